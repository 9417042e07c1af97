// Prefill kernel: Y[M][N] = X[M][K] * W_hat^T on the 5th-generation tensor
// cores (tcgen05, TMEM, TMA), one fused pass for any M.
//
// MosaicQuant "Methodology" 3. (ZipperEngine): the sparse residual is
// integrated into the dense 4-bit GEMM kernel; dense compute, sparse
// compensation and the reduction-add run as one overlapped pipeline on
// tensor cores, CUDA cores and HBM.
//
// One CTA computes a 128-token x 128-row output tile over all of K, in
// stages of 64 columns, with warp roles:
//   warp 0      TMA producer: the X tile [128 tokens][64] (128-byte swizzle)
//               and the packed codes [128 rows][8 words] of each stage into
//               a deep ring (S1 stages), plus the tile's scale/zero words
//               once, as [groups/4][128 rows][4 words] boxes.
//   warp 1      allocates tensor memory and issues tcgen05.mma (one thread).
//   warps 2..9  epilogue, two per tensor-memory lane quadrant (thread =
//               token), each owning 64 of the tile's 128 columns.
//   warps 10..13 dequant, thread = weight row: the 8 packed words of the row
//               become its 64 exact bf16 codes (q - z), written straight into
//               the 128-byte-swizzled K-major operand layout; the row's
//               residual entries of the stage are written as exact bf16
//               codes q_r into a second operand tile (zeros elsewhere).
// Per stage the MMA thread issues 4 K=16 steps of the dense tile into the
// TMEM buffer of the current 128-column group and 4 steps of the residual
// tile into a TMEM accumulator that spans all of K. Every product is exact
// (integer codes times bf16 x) and accumulates in fp32. When a group's two
// stages are done the epilogue reads its partial sums from TMEM and adds
// s[n][g] * partial to per-thread fp32 accumulators (the per-group rescale
// the fp16 group scales require); the next group's MMAs run meanwhile into
// the other buffer. After the last stage the residual accumulator is scaled
// by s_r[n] and added (the reduction-add), and the tile is stored as bf16.
// The residual's exact codes make it a second dense MMA per stage; rows
// whose residual is empty still pay for it (the cost a block-sparse
// residual allocation would avoid).

#include "common.cuh"
#include "internal.h"
#include "kernels.h"

namespace mq {
namespace {

constexpr int BM = 128, BN = 128, BK = 64;
constexpr int MAX_S1 = 8;  // TMA ring depth (runtime S1 <= MAX_S1)
constexpr int THREADS = 448;
constexpr int W_TMA = 0, W_MMA = 1, W_EPI0 = 2, W_DQ0 = 10;
constexpr int EPI_WARPS = 8, EPI_COLS = BN / 2;  // two warps per lane quadrant
constexpr int A_BYTES = BM * BK * 2;  // X tile
constexpr int B_BYTES = BN * BK * 2;  // one dequantized operand tile
constexpr int P_BYTES = BN * BK / 2;  // packed codes
constexpr int T_BYTES = A_BYTES + P_BYTES;  // one TMA stage: A at 0, P after it
constexpr int OFF_P = A_BYTES;
constexpr int BB_BYTES = 2 * B_BYTES;  // one operand buffer: dense at 0, residual after
constexpr uint32_t TMEM_COLS = 512;  // D[2] at 0 / 128, residual at 256
static_assert(T_BYTES % 1024 == 0 && BB_BYTES % 1024 == 0, "1024-byte swizzle alignment");

struct PrefillParams {
    CUtensorMap tm_x;   // X [M][K] bf16, box [128][64], 128B swizzle
    CUtensorMap tm_w;   // qweight [N][K/8] u32, box [128][8]
    CUtensorMap tm_sz;  // sz [N][Gp] u32, box [128][4]
    const int32_t *row_ptr;
    const uint16_t *col;
    const uint8_t *val;
    const uint16_t *rscale;
    __nv_bfloat16 *Y;
    float *Yf;
    int *err;
    int M, N, K, G, Gp;
    int with_residual;
    int csr_cap;  // residual entries the shared-memory slice holds (0: read global)
    int S1;       // TMA ring depth
    int S2;       // operand ring depth (2 or 3)
};

struct SmemLayout {
    int bring, sz, sfr, srs, rflag, bars, tmem_slot, abort, col, val, total;
    __host__ __device__ SmemLayout(int S1, int S2, int Gp, int csr_cap) {
        bring = S1 * T_BYTES;          // the TMA ring starts at 0
        sz = bring + S2 * BB_BYTES;
        sfr = sz + BN * Gp * 4;
        srs = sfr + 2 * BN * 4;
        rflag = srs + BN * 4;
        bars = rflag + 3 * 4 * 4;
        tmem_slot = bars + (3 * MAX_S1 + 12) * 8;
        abort = tmem_slot + 16;
        col = abort + 16;
        val = col + (csr_cap > 0 ? (csr_cap * 2 + 32 + 15) / 16 * 16 : 0);
        total = val + (csr_cap > 0 ? (csr_cap / 2 + 32 + 15) / 16 * 16 : 0);
    }
};

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
                 : "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t *slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (stride byte offset), leading byte offset 16 (unused for
// this layout), descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
           (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
           (static_cast<uint64_t>(2) << 61);
}

// Instruction descriptor: bf16 x bf16 -> fp32, both K-major, M = 128, N = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
                            (static_cast<uint32_t>(BM >> 4) << 24);

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// 32 lanes x 32 columns of 32-bit values: thread i gets lane (base + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
        "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 lanes x 16 columns of 32-bit values: thread i gets lane (base + i).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void sts128(void *p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(smem_u32(p)), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

__device__ __forceinline__ void sts16(void *p, uint16_t v) {
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(smem_u32(p)), "h"(v) : "memory");
}

__global__ void __launch_bounds__(THREADS, 1) prefill_kernel(const __grid_constant__ PrefillParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const SmemLayout L(p.S1, p.S2, p.Gp, p.csr_cap);
    const int S1 = p.S1, S2 = p.S2;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * BN, m0 = blockIdx.y * BM;
    const int nk = p.K / BK;
    const int G = p.G, Gp = p.Gp;

    const uint32_t *sz_s = reinterpret_cast<const uint32_t *>(smem + L.sz);
    float *sfr = reinterpret_cast<float *>(smem + L.sfr);  // [2][BN] group scales
    float *srs = reinterpret_cast<float *>(smem + L.srs);  // [BN] residual scales
    volatile uint32_t *rflag = reinterpret_cast<volatile uint32_t *>(smem + L.rflag);  // [S2][4]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bars);
    uint64_t *full = bars;                 // [S1] TMA stage landed
    uint64_t *empty = bars + MAX_S1;       // [S1] MMAs reading the TMA stage done
    uint64_t *bready = bars + 2 * MAX_S1;  // [S2] operand buffer written
    uint64_t *bempty = bready + 3;         // [S2] MMAs reading the operand buffer done
    uint64_t *dfull = bready + 6;          // [2] group partial ready in TMEM
    uint64_t *dempty = bready + 8;         // [2] epilogue done with the TMEM buffer
    uint64_t *sready = bready + 10;        // [2] group scales written
    uint64_t *rfull = bready + 12;         // residual accumulator complete
    uint64_t *szbar = reinterpret_cast<uint64_t *>(smem + L.tmem_slot + 8);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L.tmem_slot);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L.abort);

    if (threadIdx.x == 0) {
        for (int s = 0; s < S1; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < S2; ++b) {
            mbar_init(&bready[b], 4);
            mbar_init(&bempty[b], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&dfull[b], 1);
            mbar_init(&dempty[b], EPI_WARPS);
            mbar_init(&sready[b], 4);
        }
        mbar_init(rfull, 1);
        mbar_init(szbar, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == W_MMA) tmem_alloc(tmem_slot, TMEM_COLS);
    for (int i = threadIdx.x; i < BN; i += THREADS)
        srs[i] = (n0 + i < p.N) ? half_bits_to_f32(p.rscale[n0 + i]) : 0.f;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == W_TMA) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            prefetch_tensormap(&p.tm_x);
            prefetch_tensormap(&p.tm_w);
            prefetch_tensormap(&p.tm_sz);
            mbar_arrive_expect_tx(szbar, BN * Gp * 4);
            for (int j = 0; j < Gp / 4; ++j)
                tma_load_2d(smem + L.sz + j * BN * 16, &p.tm_sz, szbar, 4 * j, n0);
            int issued = 0;
            for (int i = 0; i < nk; ++i) {
                const int s = i % S1;
                if (i >= S1 &&
                    !mbar_wait(&empty[s], ((i / S1) - 1) & 1, p.err, kErrWaitEmpty, abort_flag))
                    break;
                uint8_t *st = smem + s * T_BYTES;
                mbar_arrive_expect_tx(&full[s], T_BYTES);
                tma_load_2d(st, &p.tm_x, &full[s], i * BK, m0);
                tma_load_2d(st + OFF_P, &p.tm_w, &full[s], i * (BK / 8), n0);
                issued = i + 1;
            }
            for (int i = max(0, issued - S1); i < issued; ++i)
                mbar_wait(&full[i % S1], (i / S1) & 1, p.err, kErrWaitDrain, abort_flag);
            mbar_wait(szbar, 0, p.err, kErrWaitDrain, abort_flag);
        }
    } else if (warp == W_MMA) {
        // ---------------------------------------------------------- MMA issue
        if (lane == 0) {
            for (int i = 0; i < nk; ++i) {
                const int s = i % S1, g = i >> 1, b = g & 1, bb = i % S2;
                if ((i & 1) == 0 && g >= 2 &&
                    !mbar_wait(&dempty[b], ((g >> 1) - 1) & 1, p.err, kErrWaitMma, abort_flag))
                    break;
                if (!mbar_wait(&full[s], (i / S1) & 1, p.err, kErrWaitFull, abort_flag)) break;
                if (!mbar_wait(&bready[bb], (i / S2) & 1, p.err, kErrWaitFull, abort_flag)) break;
                tc_fence_after();
                const uint32_t bbuf = smem_u32(smem + L.bring + bb * BB_BYTES);
                const uint64_t ad = sw128_desc(smem_u32(smem + s * T_BYTES));
                const uint64_t bd = sw128_desc(bbuf);
                const uint64_t br = sw128_desc(bbuf + B_BYTES);
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk)
                    mma_f16(tmem + b * BN, ad + 2 * kk, bd + 2 * kk, ((i & 1) | kk) ? 1u : 0u);
                // stage 0 always runs, so the residual accumulator is initialized
                if (p.with_residual &&
                    (rflag[4 * bb] | rflag[4 * bb + 1] | rflag[4 * bb + 2] | rflag[4 * bb + 3])) {
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        mma_f16(tmem + 2 * BN, ad + 2 * kk, br + 2 * kk, (i | kk) ? 1u : 0u);
                }
                mma_commit(&empty[s]);
                mma_commit(&bempty[bb]);
                if (i & 1) mma_commit(&dfull[b]);
            }
            mma_commit(rfull);
            // every issued MMA has finished before tensor memory is released
            mbar_wait(rfull, 0, p.err, kErrWaitDrain, abort_flag);
        }
    } else if (warp >= W_DQ0) {
        // ---------------------------------------------------------- dequant
        const int n = (warp - W_DQ0) * 32 + lane;  // row within the tile
        const int row = n0 + n;
        const bool valid = row < p.N;
        const bool res = p.with_residual != 0;
        int cur = 0, end = 0;
        const uint16_t *colp = p.col;  // residual columns, global or staged
        const uint8_t *valp = p.val;
        int cb = 0, vb = 0;            // index bases of the staged slice
        if (res) {
            if (valid) {
                cur = p.row_ptr[row];
                end = p.row_ptr[row + 1];
            }
            if (p.csr_cap > 0) {
                // stage this tile's CSR slice while the first TMA stages land
                const int e_b = p.row_ptr[n0], e_e = p.row_ptr[min(n0 + BN, p.N)];
                cb = e_b & ~7;
                vb = (e_b >> 1) & ~15;
                const int t = threadIdx.x - W_DQ0 * 32;
                const int nc16 = (e_e > e_b) ? ((e_e - cb) * 2 + 15) / 16 : 0;
                const int nv16 = (e_e > e_b) ? (((e_e + 1) >> 1) - vb + 15) / 16 : 0;
                for (int k = t; k < nc16; k += 128) cp_async16(smem + L.col + 16 * k, p.col + cb + 8 * k);
                for (int k = t; k < nv16; k += 128) cp_async16(smem + L.val + 16 * k, p.val + vb + 16 * k);
                asm volatile("cp.async.wait_all;" ::: "memory");
                asm volatile("bar.sync 1, 128;" ::: "memory");
                colp = reinterpret_cast<const uint16_t *>(smem + L.col) - cb;
                valp = smem + L.val - vb;
            }
        }
        int nextc = (cur < end) ? static_cast<int>(colp[cur]) : 0x7fffffff;
        uint32_t clean = 0;  // operand buffers whose residual rows of this warp are zero
        bool ok = mbar_wait_warp(szbar, 0, p.err, kErrWaitFull, abort_flag);
        for (int i = 0; ok && i < nk; ++i) {
            const int s = i % S1, g = i >> 1, b = g & 1, bb = i % S2;
            const uint32_t szw = sz_s[((g >> 2) * BN + n) * 4 + (g & 3)];
            if ((i & 1) == 0) {
                if (g >= 2 && !mbar_wait_warp(&dempty[b], ((g >> 1) - 1) & 1, p.err, kErrWaitMma,
                                              abort_flag))
                    break;
                sfr[b * BN + n] = half_bits_to_f32(szw);
                __syncwarp();
                if (lane == 0) mbar_arrive(&sready[b]);
            }
            if (!mbar_wait_warp(&full[s], (i / S1) & 1, p.err, kErrWaitFull, abort_flag)) break;
            if (i >= S2 &&
                !mbar_wait_warp(&bempty[bb], ((i / S2) - 1) & 1, p.err, kErrWaitMma, abort_flag))
                break;
            uint8_t *st = smem + s * T_BYTES;
            uint8_t *bbuf = smem + L.bring + bb * BB_BYTES;
            const uint32_t z = static_cast<uint32_t>(half_bits_to_f32(szw >> 16));
            const uint32_t zz = (0x4300u | z) * 0x00010001u;  // bf16x2 (128 + z)
            const uint4 w0 = lds128(st + OFF_P + n * 32);
            const uint4 w1 = lds128(st + OFF_P + n * 32 + 16);
            const uint32_t words[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
            uint8_t *brow = bbuf + n * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint32_t wd = words[c];
                sts128(brow + ((c ^ (n & 7)) << 4), bf16x2_sub(nib_pair_bias128(wd), zz),
                       bf16x2_sub(nib_pair_bias128(wd >> 4), zz),
                       bf16x2_sub(nib_pair_bias128(wd >> 8), zz),
                       bf16x2_sub(nib_pair_bias128(wd >> 12), zz));
            }
            bool has = false;
            if (res) {
                const int k_end = (i + 1) * BK;
                has = __any_sync(0xffffffffu, nextc < k_end) || i == 0;
                const uint32_t sbit = 1u << bb;
                if (has || !(clean & sbit)) {
                    uint8_t *rrow = bbuf + B_BYTES + n * 128;
#pragma unroll
                    for (int c = 0; c < 8; ++c) sts128(rrow + ((c ^ (n & 7)) << 4), 0u, 0u, 0u, 0u);
                    while (nextc < k_end) {
                        const int cl = nextc - i * BK;
                        const uint32_t byte = valp[cur >> 1];
                        const int qv = static_cast<int>(((byte >> ((cur & 1) * 4)) & 0xF) ^ 8) - 8;
                        const __nv_bfloat16 qb = __float2bfloat16_rn(static_cast<float>(qv));
                        sts16(rrow + (((cl >> 3) ^ (n & 7)) << 4) + (cl & 7) * 2,
                              __bfloat16_as_ushort(qb));
                        ++cur;
                        nextc = (cur < end) ? static_cast<int>(colp[cur]) : 0x7fffffff;
                    }
                    clean = has ? (clean & ~sbit) : (clean | sbit);
                }
            }
            if (lane == 0) rflag[4 * bb + (warp - W_DQ0)] = has ? 1u : 0u;
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bready[bb]);
        }
    } else {
        // ---------------------------------------------------------- epilogue
        const int q = warp & 3;                        // tensor-memory lane quadrant
        const int cb = ((warp - W_EPI0) >> 2) * EPI_COLS;  // first column of this warp
        const int r = 32 * q + lane;                   // token within the tile
        const uint32_t tl = tmem + (static_cast<uint32_t>(32 * q) << 16) + cb;
        float acc[EPI_COLS];
#pragma unroll
        for (int j = 0; j < EPI_COLS; ++j) acc[j] = 0.f;
        bool ok = true;
        for (int g = 0; g < G; ++g) {
            const int b = g & 1;
            if (!mbar_wait_warp(&dfull[b], (g >> 1) & 1, p.err, kErrWaitMma, abort_flag) ||
                !mbar_wait_warp(&sready[b], (g >> 1) & 1, p.err, kErrWaitMma, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const float *sc = sfr + b * BN + cb;
#pragma unroll
            for (int c0 = 0; c0 < EPI_COLS; c0 += 16) {
                float v[16];
                tmem_ld16(tl + b * BN + c0, v);
#pragma unroll
                for (int j = 0; j < 16; ++j) acc[c0 + j] = fmaf(sc[c0 + j], v[j], acc[c0 + j]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&dempty[b]);
        }
        if (ok && mbar_wait_warp(rfull, 0, p.err, kErrWaitMma, abort_flag)) {
            tc_fence_after();
            if (p.with_residual) {
#pragma unroll
                for (int c0 = 0; c0 < EPI_COLS; c0 += 16) {
                    float v[16];
                    tmem_ld16(tl + 2 * BN + c0, v);
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        acc[c0 + j] = fmaf(srs[cb + c0 + j], v[j], acc[c0 + j]);
                }
            }
            const int tok = m0 + r;
            const int nb = n0 + cb;
            if (tok < p.M) {
                if (p.Yf) {
                    float *yr = p.Yf + static_cast<size_t>(tok) * p.N + nb;
#pragma unroll
                    for (int j = 0; j < EPI_COLS; ++j)
                        if (nb + j < p.N) yr[j] = acc[j];
                } else {
                    __nv_bfloat16 *yr = p.Y + static_cast<size_t>(tok) * p.N + nb;
                    if (nb + EPI_COLS <= p.N && (p.N & 7) == 0) {
#pragma unroll
                        for (int j = 0; j < EPI_COLS; j += 8) {
                            uint32_t pk[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                __nv_bfloat162 h =
                                    __floats2bfloat162_rn(acc[j + 2 * e], acc[j + 2 * e + 1]);
                                pk[e] = *reinterpret_cast<uint32_t *>(&h);
                            }
                            *reinterpret_cast<uint4 *>(yr + j) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < EPI_COLS; ++j)
                            if (nb + j < p.N) yr[j] = __float2bfloat16_rn(acc[j]);
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == W_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace

mq_status launch_prefill(const mq_weight *w, const void *X, int64_t M, void *Y,
                         cudaStream_t stream, float *partial) {
    const DeviceWeight &d = weight_device(w);
    if (d.Gp > 256) return fail(MQ_ERR_UNSUPPORTED, "prefill kernel: K above 32768");
    if (M > (int64_t(1) << 23)) return fail(MQ_ERR_UNSUPPORTED, "prefill kernel: M above 2^23");
    const PrefillMaps *pm = prefill_maps(w);
    if (!pm) return MQ_ERR_CUDA;
    PrefillParams p;
    if (!encode_x_map(&p.tm_x, X, M, d.K))
        return fail(MQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for X");
    p.tm_w = pm->w;
    p.tm_sz = pm->sz;
    p.row_ptr = d.row_ptr;
    p.col = d.col;
    p.val = d.val;
    p.rscale = d.rscale;
    p.Y = static_cast<__nv_bfloat16 *>(Y);
    p.Yf = partial;
    p.err = d.err;
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(d.N);
    p.K = static_cast<int>(d.K);
    p.G = static_cast<int>(d.G);
    p.Gp = static_cast<int>(d.Gp);
    p.with_residual = (partial == nullptr && d.nnz > 0) ? 1 : 0;
    p.csr_cap = 0;
    int cap = 0;
    if (p.with_residual) {
        const MapSet *ms = weight_maps(w, BN, 4);
        if (!ms) return MQ_ERR_CUDA;
        cap = static_cast<int>(ms->max_tile_nnz);
    }
    // deepest TMA ring that fits, keeping the residual slice in shared memory if possible
    const int budget = 227 * 1024 - 1024;
    p.S1 = 0;
    // prefer 3 operand buffers, then the deepest TMA ring (at least 4)
    for (int s2 = 3; s2 >= 2 && !p.S1; --s2)
        for (int s1 = MAX_S1; s1 >= (s2 == 3 ? 4 : 3) && !p.S1; --s1) {
            if (SmemLayout(s1, s2, p.Gp, cap).total <= budget) {
                p.S1 = s1;
                p.S2 = s2;
                p.csr_cap = cap;
            } else if (s2 == 2 && s1 <= 4 && SmemLayout(s1, s2, p.Gp, 0).total <= budget) {
                p.S1 = s1;
                p.S2 = s2;
            }
        }
    if (!p.S1) return fail(MQ_ERR_UNSUPPORTED, "prefill kernel: shared memory");
    const SmemLayout L(p.S1, p.S2, p.Gp, p.csr_cap);
    const int smem = L.total + 1024;
    if (smem > 227 * 1024) return fail(MQ_ERR_UNSUPPORTED, "prefill kernel: shared memory");
    static bool configured[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(MQ_ERR_CUDA, "cudaGetDevice failed");
    if (dev >= 0 && dev < 64 && !configured[dev]) {
        if (cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 227 * 1024) != cudaSuccess)
            return fail(MQ_ERR_CUDA, "cudaFuncSetAttribute failed for the prefill kernel");
        configured[dev] = true;
    }
    dim3 grid(static_cast<unsigned>((d.N + BN - 1) / BN), static_cast<unsigned>((M + BM - 1) / BM));
    prefill_kernel<<<grid, THREADS, smem, stream>>>(p);
    cudaError_t e = cudaPeekAtLastError();
    if (e != cudaSuccess)
        return fail(MQ_ERR_CUDA, std::string("prefill launch: ") + cudaGetErrorString(e));
    return MQ_OK;
}

}  // namespace mq
