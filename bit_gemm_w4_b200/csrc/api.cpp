// C ABI of libmosaicq (include/mosaicq.h): validation, packing + upload,
// TMA descriptors, kernel dispatch, export and error reporting.
//
// MosaicQuant (gist.science/paper/2606.15652): "Methodology" 1. defines the
// 4-bit disaggregated weight W ~= Q(W) + R built once by mq_pack;
// "Methodology" 3. (ZipperEngine) defines the fused product mq_linear runs.

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <string>
#include <vector>

#include "internal.h"
#include "kernels.h"

struct mq_weight {
    int device = -1;
    mq::DeviceWeight d{};
    int64_t max_row_nnz = 0;
    int64_t device_bytes = 0;
    std::vector<void *> allocations;
    std::vector<int32_t> host_row_ptr;  // for residual tile statistics
    mutable std::mutex maps_mu;
    mutable std::vector<std::pair<int, int64_t>> tile_nnz;  // (tile height, max entries)
    mutable std::vector<std::pair<int, int64_t>> span_nnz;  // (CTA count, max entries)
    mutable std::vector<std::pair<int, int64_t>> span_blk;  // (CTA count, max blocks)
    std::vector<int32_t> host_blk_ptr;                      // block tiles: offsets per block-row
    mutable mq::PrefillMaps *pmaps = nullptr;
    ~mq_weight() { delete pmaps; }
};

namespace mq {

namespace {
thread_local std::string g_last_error;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

bool encode_2d(CUtensorMap *map, CUtensorMapDataType dt, int esize, const void *base,
               uint64_t inner, uint64_t outer, uint32_t box_inner, uint32_t box_outer,
               CUtensorMapSwizzle swz) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {inner * static_cast<uint64_t>(esize)};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

mq_status cuda_fail(cudaError_t e, const char *what) {
    return fail(e == cudaErrorMemoryAllocation ? MQ_ERR_OUT_OF_MEMORY : MQ_ERR_CUDA,
                std::string(what) + ": " + cudaGetErrorString(e));
}

template <class T>
mq_status upload(mq_weight *w, T **dst, const T *src, size_t count, size_t pad_bytes,
                 cudaStream_t stream) {
    size_t bytes = count * sizeof(T) + pad_bytes;
    void *p = nullptr;
    cudaError_t e = cudaMalloc(&p, bytes > 0 ? bytes : 16);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc");
    w->allocations.push_back(p);
    w->device_bytes += static_cast<int64_t>(bytes);
    if (pad_bytes) {
        e = cudaMemsetAsync(p, 0, bytes, stream);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
    }
    if (count) {
        e = cudaMemcpyAsync(p, src, count * sizeof(T), cudaMemcpyHostToDevice, stream);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyAsync");
    }
    *dst = static_cast<T *>(p);
    return MQ_OK;
}

// The residual grouped per (128-row tile, 64-column stage, 32-row quadrant)
// for the prefill kernel (layout in kernels.h, DeviceWeight::stage_ptr).
void build_stage_lists(const HostPacked &hp, std::vector<int32_t> &ptr, std::vector<uint32_t> &ent) {
    const int64_t tiles = (hp.N + 127) / 128, nk = hp.K / 64;
    const int64_t keys = tiles * nk * 4;
    ptr.assign(static_cast<size_t>(keys + 1), 0);
    ent.assign(static_cast<size_t>(hp.nnz), 0u);
    auto key = [&](int64_t n, int64_t c) { return ((n / 128) * nk + c / 64) * 4 + (n % 128) / 32; };
    for (int64_t n = 0; n < hp.N; ++n)
        for (int64_t e = hp.row_ptr[n]; e < hp.row_ptr[n + 1]; ++e) ++ptr[key(n, hp.col[e]) + 1];
    for (int64_t k = 0; k < keys; ++k) ptr[k + 1] += ptr[k];
    std::vector<int32_t> fill(ptr.begin(), ptr.end() - 1);
    for (int64_t n = 0; n < hp.N; ++n)
        for (int64_t e = hp.row_ptr[n]; e < hp.row_ptr[n + 1]; ++e) {
            const int64_t c = hp.col[e];
            const int q = static_cast<int>(((hp.val[e >> 1] >> ((e & 1) * 4)) & 0xF) ^ 8) - 8;
            // q in [-8, 7] is exact in bf16: the high half of its fp32 bits
            float f = static_cast<float>(q);
            uint32_t bits;
            std::memcpy(&bits, &f, 4);
            ent[fill[key(n, c)]++] = static_cast<uint32_t>(n % 128) |
                                     (static_cast<uint32_t>(c % 64) << 8) | (bits & 0xFFFF0000u);
        }
}

// The residual grouped per (128-row block, 256-column stage) for the wide
// decode kernel (layout in kernels.h, DeviceWeight::wide_ptr): inside a
// slice, entries are ordered by (16-row warp tile, 128-column group, MMA
// k-step) so that each warp finds the entries of one k-step contiguous.
void build_wide_lists(const HostPacked &hp, std::vector<int32_t> &ptr, std::vector<uint16_t> &off,
                      std::vector<uint16_t> &ent, int64_t &max_len) {
    const int64_t blocks = (hp.N + 127) / 128, S = (hp.K + 255) / 256, keys = blocks * S;
    // sub-key inside a slice: warp tile (8) x group (2) x k-step (8); the
    // k-step of column c in its group is (c % 32) / 4 (the nibble interleave)
    auto sub = [](int64_t n, int64_t c) {
        return ((n % 128) / 16) * 16 + ((c % 256) / 128) * 8 + (c % 32) / 4;
    };
    std::vector<int32_t> cnt(static_cast<size_t>(keys * 128 + 1), 0);
    for (int64_t n = 0; n < hp.N; ++n)
        for (int64_t e = hp.row_ptr[n]; e < hp.row_ptr[n + 1]; ++e) {
            const int64_t c = hp.col[e];
            ++cnt[((n / 128) * S + c / 256) * 128 + sub(n, c) + 1];
        }
    for (int64_t k = 0; k < keys * 128; ++k) cnt[k + 1] += cnt[k];
    ptr.assign(static_cast<size_t>(keys + 1), 0);
    off.assign(static_cast<size_t>(keys * kWideOffStride), 0);
    max_len = 0;
    for (int64_t k = 0; k <= keys; ++k) ptr[k] = cnt[k * 128];
    for (int64_t k = 0; k < keys; ++k) {
        for (int u = 0; u <= 128; ++u)
            off[k * kWideOffStride + u] = static_cast<uint16_t>(cnt[k * 128 + u] - ptr[k]);
        max_len = std::max<int64_t>(max_len, ptr[k + 1] - ptr[k]);
    }
    ent.assign(static_cast<size_t>(hp.nnz), 0);
    std::vector<int32_t> fill(cnt.begin(), cnt.end() - 1);
    for (int64_t n = 0; n < hp.N; ++n)
        for (int64_t e = hp.row_ptr[n]; e < hp.row_ptr[n + 1]; ++e) {
            const int64_t c = hp.col[e];
            const uint32_t nib = (hp.val[e >> 1] >> ((e & 1) * 4)) & 0xF;
            ent[fill[((n / 128) * S + c / 256) * 128 + sub(n, c)]++] =
                static_cast<uint16_t>((c % 256) | ((n % 16) << 8) | (nib << 12));
        }
}

// The residual grouped per (16-row tile, 128-column group) for the
// tall-layer decode kernel (layout in kernels.h, DeviceWeight::tl_ptr). An
// entry is stored as the byte where its code goes in the group's eight
// m16n8k16 A-fragment tiles (512 bytes each, one per MMA k-step; under the
// nibble interleave k-step (c % 32) / 4 covers column c, and inside a tile
// thread (g = r % 8, t = c / 32) holds it in register (r / 8) + 2 * ((c % 4)
// / 2), half c % 2), with the stored nibble above it.
void build_tile_lists(const HostPacked &hp, std::vector<int32_t> &ptr, std::vector<uint16_t> &ent) {
    const int64_t tiles = (hp.N + 15) / 16, G = hp.K / 128, keys = tiles * G;
    auto key = [&](int64_t n, int64_t c) { return (n / 16) * G + c / 128; };
    ptr.assign(static_cast<size_t>(keys + 1), 0);
    for (int64_t n = 0; n < hp.N; ++n)
        for (int64_t e = hp.row_ptr[n]; e < hp.row_ptr[n + 1]; ++e) ++ptr[key(n, hp.col[e]) + 1];
    for (int64_t k = 0; k < keys; ++k) ptr[k + 1] += ptr[k];
    ent.assign(static_cast<size_t>(hp.nnz), 0);
    std::vector<int32_t> fill(ptr.begin(), ptr.end() - 1);
    for (int64_t n = 0; n < hp.N; ++n)
        for (int64_t e = hp.row_ptr[n]; e < hp.row_ptr[n + 1]; ++e) {
            const int64_t c = hp.col[e];
            const uint32_t nib = (hp.val[e >> 1] >> ((e & 1) * 4)) & 0xF;
            const int64_t r = n % 16, cg = c % 128;
            const int64_t pos = ((cg % 32) / 4) * 512 +
                                (((r % 8) * 4 + cg / 32) * 4 + r / 8 + 2 * ((cg % 4) / 2)) * 4 + (cg % 2) * 2;
            ent[fill[key(n, c)]++] = static_cast<uint16_t>(pos | (nib << 12));
        }
}

mq_status upload_packed(const HostPacked &hp, cudaStream_t stream, mq_weight **out) {
    *out = nullptr;
    // Failure injection for tests: MQ_FAULT_ALLOC=1 makes the first device
    // allocation fail before any CUDA call is made.
    if (const char *f = std::getenv("MQ_FAULT_ALLOC"); f && std::strcmp(f, "1") == 0)
        return fail(MQ_ERR_OUT_OF_MEMORY, "device allocation failed (injected by MQ_FAULT_ALLOC=1)");
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "no usable CUDA device");
    mq_weight *w = new (std::nothrow) mq_weight();
    if (!w) return fail(MQ_ERR_OUT_OF_MEMORY, "host allocation failed");
    w->device = dev;
    DeviceWeight &d = w->d;
    d.N = hp.N;
    d.K = hp.K;
    d.G = hp.G;
    d.Gp = hp.Gp;
    d.nnz = hp.nnz;
    mq_status st = MQ_OK;
    uint32_t *qw = nullptr, *sz = nullptr;
    int32_t *rp = nullptr;
    uint16_t *col = nullptr, *rs = nullptr;
    uint8_t *val = nullptr;
    int *err = nullptr;
    int zero = 0;
    if (!st) st = upload(w, &qw, hp.qweight.data(), hp.qweight.size(), 0, stream);
    if (!st) st = upload(w, &sz, hp.sz.data(), hp.sz.size(), 0, stream);
    if (!st) st = upload(w, &rp, hp.row_ptr.data(), hp.row_ptr.size(), 0, stream);
    if (!st) st = upload(w, &col, hp.col.data(), hp.col.size(), 64, stream);
    if (!st) st = upload(w, &val, hp.val.data(), hp.val.size(), 64, stream);
    if (!st) st = upload(w, &rs, hp.rscale.data(), hp.rscale.size(), 0, stream);
    int32_t *sptr = nullptr;
    uint32_t *sent = nullptr;
    std::vector<int32_t> hptr;
    std::vector<uint32_t> hent;
    if (!st && hp.nnz > 0) {
        build_stage_lists(hp, hptr, hent);
        st = upload(w, &sptr, hptr.data(), hptr.size(), 0, stream);
        if (!st) st = upload(w, &sent, hent.data(), hent.size(), 0, stream);
    }
    int32_t *wptr = nullptr;
    uint16_t *woff = nullptr, *went = nullptr;
    std::vector<int32_t> hwptr;
    std::vector<uint16_t> hwoff, hwent;
    int64_t wide_max = 0;
    if (!st && hp.nnz > 0) {
        build_wide_lists(hp, hwptr, hwoff, hwent, wide_max);
        st = upload(w, &wptr, hwptr.data(), hwptr.size(), 64, stream);
        if (!st) st = upload(w, &woff, hwoff.data(), hwoff.size(), 0, stream);
        if (!st) st = upload(w, &went, hwent.data(), hwent.size(), 64, stream);
    }
    int32_t *tptr = nullptr;
    uint16_t *tent = nullptr;
    if (!st && hp.nnz > 0) {
        std::vector<int32_t> htptr;
        std::vector<uint16_t> htent;
        build_tile_lists(hp, htptr, htent);
        st = upload(w, &tptr, htptr.data(), htptr.size(), 0, stream);
        if (!st) st = upload(w, &tent, htent.data(), htent.size(), 64, stream);
    }
    int32_t *bptr = nullptr;
    uint16_t *bcol = nullptr;
    uint32_t *bq = nullptr, *bmap = nullptr;
    HostBlocks hb;
    if (!st && block_tiles_host(hp, hb)) {
        st = upload(w, &bptr, hb.ptr.data(), hb.ptr.size(), 0, stream);
        if (!st) st = upload(w, &bcol, hb.col.data(), hb.col.size(), 64, stream);
        if (!st) st = upload(w, &bq, hb.q.data(), hb.q.size(), 0, stream);
        if (!st) st = upload(w, &bmap, hb.map.data(), hb.map.size(), 0, stream);
    }
    if (!st) st = upload(w, &err, &zero, 1, 0, stream);
    if (!st) {
        e = cudaStreamSynchronize(stream);
        if (e != cudaSuccess) st = cuda_fail(e, "upload");
    }
    if (st) {
        mq_free(w);
        return st;
    }
    d.qweight = qw;
    d.sz = sz;
    d.row_ptr = rp;
    d.col = col;
    d.val = val;
    d.rscale = rs;
    d.stage_ptr = sptr;
    d.stage_ent = sent;
    d.wide_ptr = wptr;
    d.wide_off = woff;
    d.wide_ent = went;
    d.wide_max = wide_max;
    d.tl_ptr = tptr;
    d.tl_ent = tent;
    d.blk_ptr = bptr;
    d.blk_col = bcol;
    d.blk_q = bq;
    d.blk_map = bmap;
    d.nblk = bq ? hb.nblk : 0;
    d.blk_words = bq ? hb.map_words : 0;
    if (bq) w->host_blk_ptr = hb.ptr;
    d.err = err;
    w->host_row_ptr = hp.row_ptr;
    for (int64_t n = 0; n < hp.N; ++n)
        w->max_row_nnz = std::max<int64_t>(w->max_row_nnz, hp.row_ptr[n + 1] - hp.row_ptr[n]);
    *out = w;
    return MQ_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

void set_error(const std::string &msg) { g_last_error = msg; }

mq_status fail(mq_status s, const std::string &msg) {
    g_last_error = msg;
    return s;
}

const DeviceWeight &weight_device(const mq_weight *w) { return w->d; }

int sm_count() {
    static int sms[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!sms[dev] && cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        sms[dev] = 148;
    return sms[dev];
}

int64_t max_tile_nnz(const mq_weight *w, int bn) {
    std::lock_guard<std::mutex> lock(w->maps_mu);
    for (const auto &e : w->tile_nnz)
        if (e.first == bn) return e.second;
    int64_t mx = 0;
    for (int64_t r = 0; r < w->d.N; r += bn) {
        const int64_t r1 = std::min<int64_t>(w->d.N, r + bn);
        mx = std::max<int64_t>(mx, w->host_row_ptr[r1] - w->host_row_ptr[r]);
    }
    w->tile_nnz.emplace_back(bn, mx);
    return mx;
}

int64_t max_span_nnz(const mq_weight *w, int64_t ntile, int parts) {
    std::lock_guard<std::mutex> lock(w->maps_mu);
    for (const auto &e : w->span_nnz)
        if (e.first == parts) return e.second;
    int64_t mx = 0;
    for (int64_t b = 0; b < parts; ++b) {
        const int64_t r0 = std::min<int64_t>(w->d.N, 16 * (ntile * b / parts));
        const int64_t r1 = std::min<int64_t>(w->d.N, 16 * (ntile * (b + 1) / parts));
        mx = std::max<int64_t>(mx, w->host_row_ptr[r1] - w->host_row_ptr[r0]);
    }
    w->span_nnz.emplace_back(parts, mx);
    return mx;
}

int64_t max_span_blocks(const mq_weight *w, int64_t ntile, int parts) {
    if (w->host_blk_ptr.empty()) return 0;
    std::lock_guard<std::mutex> lock(w->maps_mu);
    for (const auto &e : w->span_blk)
        if (e.first == parts) return e.second;
    int64_t mx = 0;
    const int64_t nbr = static_cast<int64_t>(w->host_blk_ptr.size()) - 1;
    for (int64_t b = 0; b < parts; ++b) {
        const int64_t t0 = std::min<int64_t>(nbr, ntile * b / parts);
        const int64_t t1 = std::min<int64_t>(nbr, ntile * (b + 1) / parts);
        mx = std::max<int64_t>(mx, w->host_blk_ptr[t1] - w->host_blk_ptr[t0]);
    }
    w->span_blk.emplace_back(parts, mx);
    return mx;
}

const PrefillMaps *prefill_maps(const mq_weight *w) {
    std::lock_guard<std::mutex> lock(w->maps_mu);
    if (w->pmaps) return w->pmaps;
    PrefillMaps *m = new (std::nothrow) PrefillMaps();
    if (!m) return nullptr;
    const DeviceWeight &d = w->d;
    m->pw = static_cast<int>(std::min<int64_t>(32, d.K / 8));
    if (!encode_2d(&m->w, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, d.qweight, d.K / 8, d.N, m->pw, 128,
                   m->pw == 32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE)) {
        delete m;
        fail(MQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for the prefill maps");
        return nullptr;
    }
    w->pmaps = m;
    return m;
}

bool encode_x_map(CUtensorMap *map, const void *X, int64_t M, int64_t K, int chunks) {
    // X [M][K] viewed as [K/64][M][64]: one box is `chunks` consecutive
    // 64-column tiles [128 rows][64], each 128-byte swizzled
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(M), static_cast<cuuint64_t>(K / 64)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(K) * 2, 128};
    cuuint32_t box[3] = {64, 128, static_cast<cuuint32_t>(chunks)};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(X), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool encode_codes_map(CUtensorMap *map, const void *codes, int64_t M, int64_t K, int chunks) {
    // int8 activation codes [M][K] viewed as [K/128][M][128]: one box is
    // `chunks` consecutive 128-column tiles [128 rows][128 bytes], each
    // 128-byte swizzled (the same 16 KB tile as 64 bf16 columns)
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(M), static_cast<cuuint64_t>(K / 128)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(K), 128};
    cuuint32_t box[3] = {128, 128, static_cast<cuuint32_t>(chunks)};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(codes), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace mq

using namespace mq;

extern "C" {

const char *mq_strerror(mq_status s) {
    switch (s) {
        case MQ_OK: return "ok";
        case MQ_ERR_INVALID_ARG: return "invalid argument";
        case MQ_ERR_UNSUPPORTED: return "unsupported";
        case MQ_ERR_OUT_OF_MEMORY: return "out of memory";
        case MQ_ERR_CUDA: return "CUDA error";
        case MQ_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

const char *mq_last_error(void) { return g_last_error.c_str(); }

mq_status mq_residual_nnz(int64_t N, int64_t K, const mq_pack_opts *opts, int64_t *nnz) {
    if (!nnz) return fail(MQ_ERR_INVALID_ARG, "nnz is NULL");
    if (mq_status st = check_shape(N, K, opts)) return st;
    *nnz = opts->residual_blocks == 1
               ? residual_blocks_selected(N, K, opts->block_fraction) * kBlockRows * kBlockCols
               : N * residual_count(K, opts->residual_density);
    return MQ_OK;
}

mq_status mq_pack_host(const float *W_host, int64_t N, int64_t K, const mq_pack_opts *opts,
                       mq_host_packed *out) {
    if (!W_host || !out) return fail(MQ_ERR_INVALID_ARG, "NULL pointer");
    if (mq_status st = check_shape(N, K, opts)) return st;
    if (!out->qweight || !out->sz || !out->row_ptr || !out->rscale)
        return fail(MQ_ERR_INVALID_ARG, "an output buffer is NULL");
    HostDecomp d;
    if (mq_status st = decompose_host(W_host, N, K, *opts, d)) return st;
    if (!d.col.empty() && (!out->col || !out->val))
        return fail(MQ_ERR_INVALID_ARG, "col/val buffers are NULL");
    HostPacked p;
    pack_host(view_of(d), p);
    std::memcpy(out->qweight, p.qweight.data(), p.qweight.size() * 4);
    for (int64_t n = 0; n < N; ++n)
        std::memcpy(out->sz + n * p.G, p.sz.data() + n * p.Gp, p.G * 4);
    std::memcpy(out->row_ptr, p.row_ptr.data(), p.row_ptr.size() * 4);
    if (p.nnz) {
        std::memcpy(out->col, p.col.data(), p.col.size() * 2);
        std::memcpy(out->val, p.val.data(), p.val.size());
    }
    std::memcpy(out->rscale, p.rscale.data(), p.rscale.size() * 2);
    return MQ_OK;
}

mq_status mq_prefill_lists_host(int64_t N, int64_t K, const int32_t *row_ptr, const uint16_t *col,
                                const uint8_t *val, int32_t *ptr, uint32_t *ent) {
    if (N <= 0 || K <= 0 || K % 64) return fail(MQ_ERR_INVALID_ARG, "N, K: positive, K a multiple of 64");
    if (!row_ptr || !ptr) return fail(MQ_ERR_INVALID_ARG, "row_ptr or ptr is NULL");
    const int64_t nnz = row_ptr[N];
    if (row_ptr[0] != 0 || nnz < 0) return fail(MQ_ERR_INVALID_ARG, "row_ptr must start at 0");
    for (int64_t n = 0; n < N; ++n)
        if (row_ptr[n + 1] < row_ptr[n]) return fail(MQ_ERR_INVALID_ARG, "row_ptr must not decrease");
    if (nnz > 0 && (!col || !val || !ent)) return fail(MQ_ERR_INVALID_ARG, "col, val or ent is NULL");
    for (int64_t e = 0; e < nnz; ++e)
        if (col[e] >= K) return fail(MQ_ERR_INVALID_ARG, "a column is not below K");
    HostPacked hp;
    hp.N = N;
    hp.K = K;
    hp.nnz = nnz;
    hp.row_ptr.assign(row_ptr, row_ptr + N + 1);
    hp.col.assign(col, col + nnz);
    hp.val.assign(val, val + (nnz + 1) / 2);
    std::vector<int32_t> hptr;
    std::vector<uint32_t> hent;
    build_stage_lists(hp, hptr, hent);
    std::memcpy(ptr, hptr.data(), hptr.size() * 4);
    if (nnz) std::memcpy(ent, hent.data(), hent.size() * 4);
    return MQ_OK;
}

mq_status mq_tile_lists_host(int64_t N, int64_t K, const int32_t *row_ptr, const uint16_t *col,
                             const uint8_t *val, int32_t *ptr, uint16_t *ent) {
    if (N <= 0 || K <= 0 || K % 128) return fail(MQ_ERR_INVALID_ARG, "N, K: positive, K a multiple of 128");
    if (!row_ptr || !ptr) return fail(MQ_ERR_INVALID_ARG, "a buffer is NULL");
    const int64_t nnz = row_ptr[N];
    if (row_ptr[0] != 0 || nnz < 0) return fail(MQ_ERR_INVALID_ARG, "row_ptr must start at 0");
    for (int64_t n = 0; n < N; ++n)
        if (row_ptr[n + 1] < row_ptr[n]) return fail(MQ_ERR_INVALID_ARG, "row_ptr must not decrease");
    if (nnz > 0 && (!col || !val || !ent)) return fail(MQ_ERR_INVALID_ARG, "col, val or ent is NULL");
    for (int64_t e = 0; e < nnz; ++e)
        if (col[e] >= K) return fail(MQ_ERR_INVALID_ARG, "a column is not below K");
    HostPacked hp;
    hp.N = N;
    hp.K = K;
    hp.nnz = nnz;
    hp.row_ptr.assign(row_ptr, row_ptr + N + 1);
    hp.col.assign(col, col + nnz);
    hp.val.assign(val, val + (nnz + 1) / 2);
    std::vector<int32_t> hptr;
    std::vector<uint16_t> hent;
    build_tile_lists(hp, hptr, hent);
    std::memcpy(ptr, hptr.data(), hptr.size() * 4);
    if (nnz) std::memcpy(ent, hent.data(), hent.size() * 2);
    return MQ_OK;
}

mq_status mq_wide_lists_host(int64_t N, int64_t K, const int32_t *row_ptr, const uint16_t *col,
                             const uint8_t *val, int32_t *ptr, uint16_t *off, uint16_t *ent,
                             int64_t *max_len) {
    if (N <= 0 || K <= 0 || K % 128) return fail(MQ_ERR_INVALID_ARG, "N, K: positive, K a multiple of 128");
    if (!row_ptr || !ptr || !off || !max_len) return fail(MQ_ERR_INVALID_ARG, "a buffer is NULL");
    const int64_t nnz = row_ptr[N];
    if (row_ptr[0] != 0 || nnz < 0) return fail(MQ_ERR_INVALID_ARG, "row_ptr must start at 0");
    for (int64_t n = 0; n < N; ++n)
        if (row_ptr[n + 1] < row_ptr[n]) return fail(MQ_ERR_INVALID_ARG, "row_ptr must not decrease");
    if (nnz > 0 && (!col || !val || !ent)) return fail(MQ_ERR_INVALID_ARG, "col, val or ent is NULL");
    for (int64_t e = 0; e < nnz; ++e)
        if (col[e] >= K) return fail(MQ_ERR_INVALID_ARG, "a column is not below K");
    HostPacked hp;
    hp.N = N;
    hp.K = K;
    hp.nnz = nnz;
    hp.row_ptr.assign(row_ptr, row_ptr + N + 1);
    hp.col.assign(col, col + nnz);
    hp.val.assign(val, val + (nnz + 1) / 2);
    std::vector<int32_t> hptr;
    std::vector<uint16_t> hoff, hent;
    build_wide_lists(hp, hptr, hoff, hent, *max_len);
    std::memcpy(ptr, hptr.data(), hptr.size() * 4);
    std::memcpy(off, hoff.data(), hoff.size() * 2);
    if (nnz) std::memcpy(ent, hent.data(), hent.size() * 2);
    return MQ_OK;
}

mq_status mq_pack(const float *W_host, int64_t N, int64_t K, const mq_pack_opts *opts,
                  mq_stream stream, mq_weight **out) {
    if (!out) return fail(MQ_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (!W_host) return fail(MQ_ERR_INVALID_ARG, "W is NULL");
    if (mq_status st = check_shape(N, K, opts)) return st;
    HostDecomp d;
    if (mq_status st = decompose_host(W_host, N, K, *opts, d)) return st;
    HostPacked p;
    try {
        pack_host(view_of(d), p);
    } catch (const std::bad_alloc &) {
        return fail(MQ_ERR_OUT_OF_MEMORY, "host allocation for packing failed");
    }
    return upload_packed(p, reinterpret_cast<cudaStream_t>(stream), out);
}

mq_status mq_pack_decomposed(const mq_decomp *dec, mq_stream stream, mq_weight **out) {
    if (!out) return fail(MQ_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (mq_status st = validate_decomp(dec)) return st;
    HostPacked p;
    try {
        pack_host(*dec, p);
    } catch (const std::bad_alloc &) {
        return fail(MQ_ERR_OUT_OF_MEMORY, "host allocation for packing failed");
    }
    return upload_packed(p, reinterpret_cast<cudaStream_t>(stream), out);
}

void mq_free(mq_weight *w) {
    if (!w) return;
    int prev = -1;
    bool switched = false;
    if (w->device >= 0 && cudaGetDevice(&prev) == cudaSuccess && prev != w->device)
        switched = cudaSetDevice(w->device) == cudaSuccess;
    for (void *p : w->allocations) cudaFree(p);
    if (switched) cudaSetDevice(prev);
    delete w;
}

mq_status mq_get_info(const mq_weight *w, mq_info *out) {
    if (!w || !out) return fail(MQ_ERR_INVALID_ARG, "NULL pointer");
    out->N = w->d.N;
    out->K = w->d.K;
    out->nnz = w->d.nnz;
    out->group_size = kGroup;
    out->device = w->device;
    out->device_bytes = w->device_bytes;
    out->max_row_nnz = w->max_row_nnz;
    return MQ_OK;
}

mq_status mq_export(const mq_weight *w, mq_host_packed *out) {
    if (!w || !out) return fail(MQ_ERR_INVALID_ARG, "NULL pointer");
    if (!out->qweight || !out->sz || !out->row_ptr || !out->rscale ||
        (w->d.nnz && (!out->col || !out->val)))
        return fail(MQ_ERR_INVALID_ARG, "an output buffer is NULL");
    int prev = -1;
    if (cudaGetDevice(&prev) != cudaSuccess) return fail(MQ_ERR_CUDA, "cudaGetDevice failed");
    if (prev != w->device && cudaSetDevice(w->device) != cudaSuccess)
        return fail(MQ_ERR_CUDA, "cudaSetDevice failed");
    const DeviceWeight &d = w->d;
    cudaError_t e = cudaDeviceSynchronize();
    auto cp = [&](void *dst, const void *src, size_t bytes) {
        if (e == cudaSuccess && bytes) e = cudaMemcpy(dst, src, bytes, cudaMemcpyDeviceToHost);
    };
    cp(out->qweight, d.qweight, size_t(d.N) * d.K / 8 * 4);
    if (e == cudaSuccess)
        e = cudaMemcpy2D(out->sz, d.G * 4, d.sz, d.Gp * 4, d.G * 4, d.N, cudaMemcpyDeviceToHost);
    cp(out->row_ptr, d.row_ptr, size_t(d.N + 1) * 4);
    cp(out->col, d.col, size_t(d.nnz) * 2);
    cp(out->val, d.val, size_t(d.nnz + 1) / 2);
    cp(out->rscale, d.rscale, size_t(d.N) * 2);
    if (prev != w->device) cudaSetDevice(prev);
    if (e != cudaSuccess) return cuda_fail(e, "mq_export");
    return MQ_OK;
}

namespace {
mq_status copy_blocks_out(const HostBlocks &b, int32_t *blk_ptr, uint16_t *blk_col, uint32_t *blk_q,
                          int64_t *nblk) {
    *nblk = b.nblk;
    if (!blk_ptr) return MQ_OK;
    if (!blk_col || !blk_q) return fail(MQ_ERR_INVALID_ARG, "an output buffer is NULL");
    std::memcpy(blk_ptr, b.ptr.data(), b.ptr.size() * 4);
    std::memcpy(blk_col, b.col.data(), b.col.size() * 2);
    std::memcpy(blk_q, b.q.data(), b.q.size() * 4);
    return MQ_OK;
}
}  // namespace

mq_status mq_block_tiles_host(const mq_decomp *d, int32_t *blk_ptr, uint16_t *blk_col,
                              uint32_t *blk_q, int64_t *nblk) {
    if (!d || !nblk) return fail(MQ_ERR_INVALID_ARG, "NULL pointer");
    if (mq_status st = validate_decomp(d)) return st;
    HostPacked p;
    pack_host(*d, p);
    HostBlocks b;
    if (!block_tiles_host(p, b)) {
        *nblk = 0;
        return fail(MQ_ERR_UNSUPPORTED, "the residual is not made of whole 16 x 64 blocks");
    }
    return copy_blocks_out(b, blk_ptr, blk_col, blk_q, nblk);
}

mq_status mq_export_blocks(const mq_weight *w, int32_t *blk_ptr, uint16_t *blk_col, uint32_t *blk_q,
                           int64_t *nblk) {
    if (!w || !nblk) return fail(MQ_ERR_INVALID_ARG, "NULL pointer");
    const DeviceWeight &d = w->d;
    if (!d.blk_q) {
        *nblk = 0;
        return fail(MQ_ERR_UNSUPPORTED, "the weight has no block tiles");
    }
    *nblk = d.nblk;
    if (!blk_ptr) return MQ_OK;
    if (!blk_col || !blk_q) return fail(MQ_ERR_INVALID_ARG, "an output buffer is NULL");
    int prev = -1;
    if (cudaGetDevice(&prev) != cudaSuccess) return fail(MQ_ERR_CUDA, "cudaGetDevice failed");
    if (prev != w->device && cudaSetDevice(w->device) != cudaSuccess)
        return fail(MQ_ERR_CUDA, "cudaSetDevice failed");
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaMemcpy(blk_ptr, d.blk_ptr, size_t(d.N / 16 + 1) * 4, cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && d.nblk) e = cudaMemcpy(blk_col, d.blk_col, size_t(d.nblk) * 2, cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && d.nblk) e = cudaMemcpy(blk_q, d.blk_q, size_t(d.nblk) * 512, cudaMemcpyDeviceToHost);
    if (prev != w->device) cudaSetDevice(prev);
    if (e != cudaSuccess) return cuda_fail(e, "mq_export_blocks");
    return MQ_OK;
}

mq_status mq_device_error(const mq_weight *w, mq_stream stream, int32_t *code) {
    if (!w || !code) return fail(MQ_ERR_INVALID_ARG, "NULL pointer");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(s);
    int v = 0;
    if (e == cudaSuccess) e = cudaMemcpy(&v, w->d.err, 4, cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && v) e = cudaMemset(w->d.err, 0, 4);
    if (e != cudaSuccess) return cuda_fail(e, "mq_device_error");
    *code = v;
    return v ? fail(MQ_ERR_DEVICE_TIMEOUT, "a kernel gave up a bounded wait") : MQ_OK;
}

namespace {

// Y = X * W^T over consecutive 16-token slices, one decode launch each.
mq_status decode_slices(const mq_weight *w, const void *X, int64_t M, void *Y, cudaStream_t s) {
    const uint16_t *x = static_cast<const uint16_t *>(X);
    uint16_t *y = static_cast<uint16_t *>(Y);
    for (int64_t m0 = 0; m0 < M; m0 += 16) {
        const int mm = static_cast<int>(std::min<int64_t>(16, M - m0));
        const mq_status st = launch_decode(w, x + m0 * w->d.K, mm, y + m0 * w->d.N, s);
        if (st) return st;
    }
    return MQ_OK;
}

// For 17..64 tokens: whether 16-token decode slices beat the prefill kernel,
// whose one 128-token tile then leaves most SMs idle on short layers. Both
// sides are estimates fitted to measurements on B200 (the 7B and 70B shapes
// at 32 and 64 tokens, where they pick the faster side in every case): a
// 16-token decode launch reads the packed weight at about 0.8 TB/s (1.33 TB/s
// on layers the tall-layer kernel takes: at least eight 16-row tiles per SM);
// the prefill kernel spends about 12.8 ns per K column for each wave of
// 128-row tiles over the SMs.
bool slices_beat_prefill(const mq_weight *w, int64_t M) {
    const DeviceWeight &d = w->d;
    const int64_t sms = sm_count();
    const double bytes = 0.5 * d.N * d.K + 4.0 * d.N * d.G + 2.5 * d.nnz;
    const bool tall = (d.N + 15) / 16 >= 8 * sms;
    const double t_slice = bytes / (tall ? 1.33e12 : 0.8e12);
    const int64_t waves = ((d.N + 127) / 128 + sms - 1) / sms;
    const double t_prefill = static_cast<double>(waves) * d.K * 12.8e-9;
    return static_cast<double>((M + 15) / 16) * t_slice < t_prefill;
}

}  // namespace

mq_status mq_linear_path(const mq_weight *w, const void *X, int64_t M, void *Y, mq_stream stream,
                         mq_path path) {
    if (!w) return fail(MQ_ERR_INVALID_ARG, "weight handle is NULL");
    if (M < 0) return fail(MQ_ERR_INVALID_ARG, "M must be >= 0");
    if (M == 0) return MQ_OK;
    if (!X || !Y) return fail(MQ_ERR_INVALID_ARG, "X or Y is NULL");
    if (!aligned16(X) || !aligned16(Y)) return fail(MQ_ERR_INVALID_ARG, "X and Y must be 16-byte aligned");
    if (M > (int64_t(1) << 31) - 1) return fail(MQ_ERR_INVALID_ARG, "M too large");
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(MQ_ERR_CUDA, "cudaGetDevice failed");
    if (dev != w->device)
        return fail(MQ_ERR_INVALID_ARG, "the current device is not the device that packed the weight");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (path == MQ_PATH_AUTO) {
        if (M <= 16) {
            // the decode kernels, unless X's slice cannot fit them (very long K)
            const mq_status st = launch_decode(w, X, static_cast<int>(M), Y, s);
            if (st != MQ_ERR_UNSUPPORTED) return st;
        } else if (M <= 64 && slices_beat_prefill(w, M)) {
            // a slice the decode kernels cannot take: the prefill kernel then
            // computes every row (it rewrites any slice already done)
            const mq_status st = decode_slices(w, X, M, Y, s);
            if (st != MQ_ERR_UNSUPPORTED) return st;
        }
        return launch_prefill(w, X, M, Y, s);
    }
    switch (path) {
        case MQ_PATH_DECODE:
            // more than 16 tokens: consecutive 16-token slices of X and Y, one
            // decode launch each (each reads the weight again)
            return decode_slices(w, X, M, Y, s);
        case MQ_PATH_PREFILL:
            return launch_prefill(w, X, M, Y, s);
        default:
            return fail(MQ_ERR_INVALID_ARG, "unknown path");
    }
}

mq_status mq_linear_unfused(const mq_weight *w, const void *X, int64_t M, void *Y,
                            void *workspace, size_t workspace_bytes, mq_stream stream) {
    if (!w) return fail(MQ_ERR_INVALID_ARG, "weight handle is NULL");
    if (M < 0) return fail(MQ_ERR_INVALID_ARG, "M must be >= 0");
    if (M == 0) return MQ_OK;
    if (!X || !Y || !workspace) return fail(MQ_ERR_INVALID_ARG, "X, Y or workspace is NULL");
    if (!aligned16(X) || !aligned16(Y) || !aligned16(workspace))
        return fail(MQ_ERR_INVALID_ARG, "X, Y and workspace must be 16-byte aligned");
    if (M > (int64_t(1) << 31) - 1) return fail(MQ_ERR_INVALID_ARG, "M too large");
    if (workspace_bytes < static_cast<size_t>(M) * static_cast<size_t>(w->d.N) * 4)
        return fail(MQ_ERR_INVALID_ARG, "workspace smaller than M*N*4 bytes");
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(MQ_ERR_CUDA, "cudaGetDevice failed");
    if (dev != w->device)
        return fail(MQ_ERR_INVALID_ARG, "the current device is not the device that packed the weight");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    float *part = static_cast<float *>(workspace);
    mq_status st = (M <= 16) ? launch_decode(w, X, static_cast<int>(M), Y, s, part)
                             : launch_prefill(w, X, M, Y, s, part);
    if (st) return st;
    return launch_residual_merge(w, X, M, part, Y, s);
}

mq_status mq_linear(const mq_weight *w, const void *X, int64_t M, void *Y, mq_stream stream) {
    return mq_linear_path(w, X, M, Y, stream, MQ_PATH_AUTO);
}

mq_status mq_linear_prefetch(const mq_weight *w, const void *X, int64_t M, void *Y,
                             const mq_weight *next, mq_stream stream) {
    if (!next || M > 16 || M <= 0) return mq_linear_path(w, X, M, Y, stream, MQ_PATH_AUTO);
    if (!w) return fail(MQ_ERR_INVALID_ARG, "weight handle is NULL");
    if (!X || !Y) return fail(MQ_ERR_INVALID_ARG, "X or Y is NULL");
    if (!aligned16(X) || !aligned16(Y)) return fail(MQ_ERR_INVALID_ARG, "X and Y must be 16-byte aligned");
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(MQ_ERR_CUDA, "cudaGetDevice failed");
    if (dev != w->device)
        return fail(MQ_ERR_INVALID_ARG, "the current device is not the device that packed the weight");
    if (next->device != w->device)
        return fail(MQ_ERR_INVALID_ARG, "the next weight lives on another device");
    L2Prefetch pf;
    pf.p[0] = next->d.qweight;
    pf.bytes[0] = next->d.N * next->d.K / 2;
    pf.p[1] = next->d.sz;
    pf.bytes[1] = next->d.N * next->d.Gp * 4;
    return launch_decode(w, X, static_cast<int>(M), Y, reinterpret_cast<cudaStream_t>(stream), nullptr, pf);
}

mq_status mq_quantize_activations(const void *X, int64_t M, int64_t K, void *codes, float *scales,
                                  mq_stream stream) {
    if (M < 0) return fail(MQ_ERR_INVALID_ARG, "M must be >= 0");
    if (K <= 0 || K % 8 || K > (int64_t(1) << 30))
        return fail(MQ_ERR_INVALID_ARG, "K must be a positive multiple of 8");
    if (M == 0) return MQ_OK;
    if (M > (int64_t(1) << 31) - 1) return fail(MQ_ERR_INVALID_ARG, "M too large");
    if (!X || !codes || !scales) return fail(MQ_ERR_INVALID_ARG, "X, codes or scales is NULL");
    if (!aligned16(X) || !aligned16(codes) || !aligned16(scales))
        return fail(MQ_ERR_INVALID_ARG, "X, codes and scales must be 16-byte aligned");
    return launch_quantize(X, M, K, codes, scales, reinterpret_cast<cudaStream_t>(stream), false);
}

mq_status mq_selftest_bounded_wait(int64_t limit_cycles, int32_t *results) {
    if (!results) return fail(MQ_ERR_INVALID_ARG, "results is NULL");
    if (limit_cycles <= 0 || limit_cycles > (int64_t(1) << 31))
        return fail(MQ_ERR_INVALID_ARG, "limit_cycles must be in (0, 2^31]");
    return selftest_bounded_wait(limit_cycles, results);
}

int64_t mq_w4a4_workspace_bytes(const mq_weight *w, int64_t M) {
    if (!w || M <= 0) return 0;
    return (M * w->d.K + 15) / 16 * 16 + (M * 4 + 15) / 16 * 16;
}

mq_status mq_linear_w4a4(const mq_weight *w, const void *X, int64_t M, void *Y, void *workspace,
                         size_t workspace_bytes, mq_stream stream) {
    if (!w) return fail(MQ_ERR_INVALID_ARG, "weight handle is NULL");
    if (M < 0) return fail(MQ_ERR_INVALID_ARG, "M must be >= 0");
    if (M == 0) return MQ_OK;
    if (!X || !Y || !workspace) return fail(MQ_ERR_INVALID_ARG, "X, Y or workspace is NULL");
    if (!aligned16(X) || !aligned16(Y) || !aligned16(workspace))
        return fail(MQ_ERR_INVALID_ARG, "X, Y and workspace must be 16-byte aligned");
    if (workspace_bytes < static_cast<size_t>(mq_w4a4_workspace_bytes(w, M)))
        return fail(MQ_ERR_INVALID_ARG, "workspace smaller than mq_w4a4_workspace_bytes");
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(MQ_ERR_CUDA, "cudaGetDevice failed");
    if (dev != w->device)
        return fail(MQ_ERR_INVALID_ARG, "the current device is not the device that packed the weight");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int8_t *codes = static_cast<int8_t *>(workspace);
    float *scales = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) +
                                              (M * w->d.K + 15) / 16 * 16);
    if (M > (int64_t(1) << 23)) return fail(MQ_ERR_UNSUPPORTED, "W4A4: M above 2^23");
    mq_status st = launch_quantize(X, M, w->d.K, codes, scales, s, true);
    if (st) return st;
    // M <= 16: the narrow and wide decode kernels; above, the tcgen05 prefill kernel
    if (M <= 16) return launch_decode_a4(w, codes, scales, static_cast<int>(M), Y, s);
    return launch_prefill_a4(w, codes, scales, M, Y, s);
}

}  // extern "C"
