// Kernel launch interface between the C ABI (api.cpp) and the CUDA sources.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/mosaicq.h"

struct mq_weight;

namespace mq {

// Row-offset table stride of the wide decode kernel's residual slices: 129
// u16 offsets padded to 272 bytes, so every table starts 16-byte aligned.
constexpr int kWideOffStride = 136;

// Device buffers of one packed weight (all on one GPU).
struct DeviceWeight {
    int64_t N, K, G, Gp, nnz;
    const uint32_t *qweight;  // [N][K/8]
    const uint32_t *sz;       // [N][Gp]
    const int32_t *row_ptr;   // [N+1]
    const uint16_t *col;      // [nnz] (+ padding)
    const uint8_t *val;       // [(nnz+1)/2] (+ padding)
    const uint16_t *rscale;   // [N]
    // The residual again, grouped for the prefill kernel: per (128-row tile,
    // 64-column stage, 32-row quadrant) the entries as words
    // row-in-tile | column-in-stage << 8 | bf16 bits of q_r << 16, ordered by
    // (tile, stage, quadrant, row, column); stage_ptr[(tile * K/64 + stage) * 4
    // + quadrant] is the first entry of each group (one more entry at the end).
    const int32_t *stage_ptr;   // [ceil(N/128) * K/64 * 4 + 1], NULL when nnz = 0
    const uint32_t *stage_ent;  // [nnz]
    // The residual again, grouped for the wide decode kernel: per (128-row
    // block, 256-column stage) a slice of u16 entries column-in-stage |
    // row-in-warp-tile << 8 | (q_r & 0xF) << 12, ordered by (block, stage,
    // 16-row warp tile, 128-column group, MMA k-step) where the k-step of
    // column c of a group is (c % 32) / 4. wide_ptr[block * S + stage] is the
    // first entry of a slice (S = ceil(K/256), one more entry at the end);
    // wide_off[(block * S + stage) * kWideOffStride + u], u = 0..128, is where
    // sub-list u = warp * 16 + group * 8 + k-step starts inside its slice
    // (u = 128: the slice length). NULL when nnz = 0.
    const int32_t *wide_ptr;   // [ceil(N/128) * S + 1]
    const uint16_t *wide_off;  // [ceil(N/128) * S * kWideOffStride]
    const uint16_t *wide_ent;  // [nnz] (+ padding)
    int64_t wide_max;          // longest slice, entries
    // The residual again, grouped for the tall-layer decode kernel: per
    // (16-row tile, 128-column group) key tile * G + group a list of u16
    // entries, in CSR order inside a key: the byte offset of the code in the
    // group's eight 512-byte m16n8k16 A-fragment tiles (12 bits: k-step * 512
    // + the fragment position of (row % 16, column % 128)) | (q_r & 0xF) << 12.
    // tl_ptr[key] is the first entry of a key (one more at the end). NULL
    // when nnz = 0.
    const int32_t *tl_ptr;     // [ceil(N/16) * G + 1]
    const uint16_t *tl_ent;    // [nnz] (+ padding)
    // The residual again as block tiles, when it consists of whole 16 x 64
    // blocks (block allocation; NULL otherwise): per 16-row block-row the
    // offsets of its blocks, their column-block indices, 512 bytes of
    // offset-binary codes q_r + 8 per block (16 rows x 8 words in the base
    // codes' nibble interleave), and a bitmap of each block-row's column-
    // blocks (blk_words 32-bit words per block-row).
    const int32_t *blk_ptr;    // [N/16 + 1]
    const uint16_t *blk_col;   // [nblk]
    const uint32_t *blk_q;     // [nblk][16][8]
    const uint32_t *blk_map;   // [N/16][blk_words]
    int64_t nblk, blk_words;
    int *err;                 // device error word
};

// Most blocks over `parts` contiguous runs of 16-row tiles (as for
// max_span_nnz); 0 when the weight has no block tiles.
int64_t max_span_blocks(const mq_weight *w, int64_t ntile, int parts);

// Largest residual entry count over the bn-row tiles of a handle (cached per
// tile height; the decode kernels size their shared-memory CSR slice with it).
int64_t max_tile_nnz(const mq_weight *w, int bn);

// Largest residual entry count over `parts` contiguous runs of 16-row tiles,
// run b holding tiles [ntile * b / parts, ntile * (b + 1) / parts) (cached
// per part count; the streaming decode kernel stages a run's CSR slice).
int64_t max_span_nnz(const mq_weight *w, int64_t ntile, int parts);

// Tensor maps of the prefill kernel (built once per handle).
struct PrefillMaps {
    CUtensorMap w;  // qweight, box [128 rows][pw words]; 128-byte swizzle when pw = 32
    int pw;         // words per row of a box: min(32, K / 8), four or two 64-column stages
};
const PrefillMaps *prefill_maps(const mq_weight *w);

// bf16 X [M][K] row-major as a 3D view [K/64][M][64]; one box holds `chunks`
// consecutive [128 rows][64 columns] tiles, each 128-byte swizzled.
bool encode_x_map(CUtensorMap *map, const void *X, int64_t M, int64_t K, int chunks);
// int8 activation codes [M][K] (K a multiple of 128) as the prefill kernel's
// W4A4 X operand: boxes of `chunks` 128-column tiles [128][128 bytes].
bool encode_codes_map(CUtensorMap *map, const void *codes, int64_t M, int64_t K, int chunks);
const DeviceWeight &weight_device(const mq_weight *w);

// Streaming multiprocessors of the current device (cached per device).
int sm_count();

// Up to two regions of another weight (the next layer's packed codes and
// scale words) that a decode launch brings into L2 while it runs: each CTA
// issues one bulk L2 prefetch of its share. Addresses 16-byte aligned,
// sizes multiples of 16; a size of 0 skips a region.
struct L2Prefetch {
    const void *p[2] = {nullptr, nullptr};
    long long bytes[2] = {0, 0};
};

// Decode kernels (decode.cu): M in [1, 16]. With `partial` set the residual
// is skipped and the dense base alone is written as fp32 to `partial`
// (the unfused path's first half); else Y (bf16) gets the fused result.
mq_status launch_decode(const mq_weight *w, const void *X, int M, void *Y, cudaStream_t stream,
                        float *partial = nullptr, const L2Prefetch &pf = L2Prefetch());

// Streaming decode kernel (decode_stream.cu) for M <= 16: persistent, one
// CTA per SM over contiguous 16-row tiles, a per-thread cp.async prefetch
// ring. `partial` and `pf` as for launch_decode. Returns
// MQ_ERR_UNSUPPORTED (without setting an error message) when X does not fit
// its shared memory, or when it would leave one CTA per SM over more than
// one wave; the caller then takes the tall-layer or register kernel.
mq_status launch_decode_stream(const mq_weight *w, const void *X, int M, void *Y,
                               cudaStream_t stream, float *partial = nullptr,
                               const L2Prefetch &pf = L2Prefetch());

// Tall-layer decode kernel (decode_tall.cu) for 2 <= M <= 16 on layers of
// at least two 16-row tiles per CTA at two CTAs per SM: X from L2, a
// per-thread item ring, the residual as tensor-core k-steps from the
// per-tile lists (DeviceWeight::tl_ptr). `partial` and `pf` as for
// launch_decode. Returns MQ_ERR_UNSUPPORTED (without setting an error
// message) for other layers or when a CTA's lists or scale words do not fit
// its shared memory.
mq_status launch_decode_tall(const mq_weight *w, const void *X, int M, void *Y,
                             cudaStream_t stream, float *partial = nullptr,
                             const L2Prefetch &pf = L2Prefetch());

// Wide decode kernel (decode_wide.cu) for 8 < M <= 16; `partial` as for
// decode. Returns MQ_ERR_UNSUPPORTED (without setting an error message) when
// its stage ring cannot hold a residual slice, and the caller falls back to
// launch_decode.
// `force` also takes layers whose blocks do not fill the GPU (the fallback
// when the narrow kernel cannot hold X's slice of a very long K).
mq_status launch_decode_wide(const mq_weight *w, const void *X, int M, void *Y,
                             cudaStream_t stream, float *partial = nullptr,
                             const L2Prefetch &pf = L2Prefetch(), bool force = false);

// The wide decode kernel's W4A4 form (8 < M <= 16, layers whose 128-row
// blocks fill the GPU): activation codes with each 8-column chunk's bytes in
// the packed codes' k order, fp32 scales [M]. MQ_ERR_UNSUPPORTED (no
// message) when it does not take the call.
mq_status launch_decode_wide_a4(const mq_weight *w, const int8_t *codes, const float *xscale,
                                int M, void *Y, cudaStream_t stream);

// Prefill kernel (prefill.cu): any M >= 1; `partial` as for decode.
mq_status launch_prefill(const mq_weight *w, const void *X, int64_t M, void *Y,
                         cudaStream_t stream, float *partial = nullptr);

// The prefill kernel's W4A4 form (K a multiple of 256): permuted int8
// activation codes [M][K] and fp32 scales [M]; int8 tensor-core MMAs.
mq_status launch_prefill_a4(const mq_weight *w, const int8_t *codes, const float *xscale, int64_t M,
                            void *Y, cudaStream_t stream);

// W4A4 (w4a4.cu): per-token int4 quantization of bf16 X into int8 codes
// [M][K] (with `permuted`, each 8-column chunk's bytes in the order
// (0,4,1,5,2,6,3,7), the form the W4A4 kernels read) and fp32 scales [M];
// then the fused W4A4 product for M <= 16 from permuted codes (Y bf16).
mq_status launch_quantize(const void *X, int64_t M, int64_t K, void *codes, float *scales,
                          cudaStream_t stream, bool permuted);
mq_status launch_decode_a4(const mq_weight *w, const int8_t *codes, const float *xscale, int M,
                           void *Y, cudaStream_t stream);

// Self-test of the bounded mbarrier wait (selftest.cu): results[0..3] =
// {a completed phase was seen, the stuck wait returned true, a later wait
// returned true, the error word}; expected {1, 0, 0, kErrWaitEmpty}.
mq_status selftest_bounded_wait(long long limit, int32_t *results);

// Separate residual kernel (residual.cu): Y = bf16(partial + X * R^T).
mq_status launch_residual_merge(const mq_weight *w, const void *X, int64_t M,
                                const float *partial, void *Y, cudaStream_t stream);

}  // namespace mq
