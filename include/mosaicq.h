/*
 * mosaicq.h - C ABI of libmosaicq, a B200 (sm_100a) fused W4 + sparse-residual
 * linear layer.
 *
 * Method: MosaicQuant (gist.science/paper/2606.15652, "Methodology").
 *   1. Inlier-Outlier Disaggregation: a weight matrix W is split as
 *      W ~= Q(W) + R, a dense 4-bit base Q that captures the inliers and a
 *      sparse 4-bit residual R that compensates the quantization error the
 *      outliers leave; both parts stay 4-bit.
 *   3. ZipperEngine: the residual is computed inside the dense 4-bit GEMM
 *      kernel instead of a separate kernel that would reload activations and
 *      merge partial outputs; dense compute, sparse compensation and the
 *      reduction-add run as one pipelined pass.
 *   Problem statement as this library reads it: build the 4-bit form of W
 *   once (mq_pack), then compute Y = X * W_hat^T many times (mq_linear).
 *
 * Encoding (the pages fix none; this library fixes it):
 *   base     int4 asymmetric, group 128 along K, one fp16 scale s and one
 *            fp16 zero point z (an integer 0..15) per (row, group):
 *            deq = (q - z) * s.
 *   residual per-row CSR of int4 codes q_r in [-8, 7] with one fp16 scale
 *            s_r per row; row n keeps its k_n = floor(rho*K + 0.5) largest
 *            |W - deq| entries (ties to the smaller column).
 *            W_hat = deq + scatter(q_r * s_r).
 *   product  exact products, fp32 accumulation, bf16 output (RNE).
 *
 * Conventions for every call:
 *   - Status codes are returned; nothing aborts. mq_last_error() gives a
 *     one-line reason for the most recent failure on the calling thread.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).
 *   - Host pointers are CPU memory owned by the caller; device pointers are
 *     CUDA global memory on the device that packed the weight.
 *   - mq_linear* never allocate; mq_pack / mq_pack_decomposed own every
 *     device buffer of a handle until mq_free.
 *   - There is no CPU fallback: a missing or unusable GPU is an error.
 */
#ifndef MOSAICQ_H
#define MOSAICQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *mq_stream; /* identical to cudaStream_t */
typedef struct mq_weight mq_weight;    /* opaque; owns one packed W on one GPU */

typedef enum {
    MQ_OK = 0,
    MQ_ERR_INVALID_ARG = 1,    /* bad pointer, size, value, alignment or device */
    MQ_ERR_UNSUPPORTED = 2,    /* a valid request this build does not serve */
    MQ_ERR_OUT_OF_MEMORY = 3,  /* a device or host allocation failed */
    MQ_ERR_CUDA = 4,           /* a CUDA runtime / driver call failed */
    MQ_ERR_DEVICE_TIMEOUT = 5  /* a kernel gave up a bounded wait */
} mq_status;

/* Which kernel mq_linear_path runs. MQ_PATH_AUTO is what mq_linear does:
 * DECODE for M <= 16; for 17 <= M <= 64 DECODE (16-token slices) where an
 * estimate of both sides' times, fitted to B200 measurements, favours it,
 * else PREFILL; PREFILL for M > 64. */
typedef enum {
    MQ_PATH_AUTO = 0,
    MQ_PATH_DECODE = 1,  /* the decode kernels (mma.sync); M > 16 in 16-token slices */
    MQ_PATH_PREFILL = 2  /* tcgen05 / TMEM / TMA tensor-core kernel; any M >= 1 */
} mq_path;

typedef struct {
    int32_t group_size;      /* must be 128, else MQ_ERR_UNSUPPORTED */
    double residual_density; /* rho in [0, 1]; k_n = floor(rho*K + 0.5) per row
                                (row mode only) */
    /* Residual allocation ("Methodology" 2, Block-Wise Residual Allocation):
     * 0 = row mode: each row keeps its k_n largest |W - deq| entries;
     * 1 = block mode: W is cut into 16-row x 64-column blocks, each scored by
     *     the Hessian-weighted squared error it would remove,
     *       delta(b) = sum over (n, k) in b of (E[n][k] * E[n][k]) * h[k]
     *     (E = W - deq, h = channel_weight, summed in fp64 row by row, column
     *     by column), and the floor(block_fraction * blocks + 0.5) blocks of
     *     largest delta (ties to the smaller block index, blocks numbered
     *     row-block major) carry a residual on every entry. Needs N % 16 == 0.
     * In both modes a row's residual has one fp16 scale s_r = fp16(max |E| / 7)
     * over its residual entries and codes clamp(rne(E / s_r), -8, 7). */
    int32_t residual_blocks;
    double block_fraction;       /* block mode: in [0, 1] */
    const float *channel_weight; /* block mode: K finite weights >= 0, the
                                    diagonal Hessian estimate of the input
                                    channels (sum over calibration tokens of
                                    x_k^2); NULL weighs every channel 1.
                                    Read during the call only. */
} mq_pack_opts;

/* One decomposition in unpacked host form (caller-owned arrays). */
typedef struct {
    int64_t N, K;            /* rows (output features), columns (inputs) */
    const uint8_t *q;        /* [N][K] base codes 0..15 */
    const uint16_t *s;       /* [N][K/128] fp16 bits of the group scales (finite) */
    const uint16_t *z;       /* [N][K/128] fp16 bits of the zero points (integers 0..15) */
    const int64_t *row_ptr;  /* [N+1] residual CSR offsets: row_ptr[0] = 0, non-decreasing */
    const int32_t *col;      /* [nnz] residual columns, strictly ascending per row, < K */
    const int8_t *qr;        /* [nnz] residual codes in [-8, 7] */
    const uint16_t *sr;      /* [N] fp16 bits of the residual scales (finite) */
} mq_decomp;

/* Caller-owned host buffers of the packed layout. Element counts: qweight
 * N*K/8, sz N*K/128, row_ptr N+1, col nnz, val (nnz+1)/2, rscale N. */
typedef struct {
    uint32_t *qweight; /* word w of row n: bits [4j,4j+4) = q[n][8w + pi(j)],
                          pi = (0,2,4,6,1,3,5,7) */
    uint32_t *sz;      /* fp16 bits of s (low half) | fp16 bits of z (high half) */
    int32_t *row_ptr;  /* CSR offsets */
    uint16_t *col;     /* CSR columns */
    uint8_t *val;      /* entry e: byte e>>1, low nibble when e is even;
                          two's complement int4; an odd tail pads with 0 */
    uint16_t *rscale;  /* fp16 bits of s_r */
} mq_host_packed;

typedef struct {
    int64_t N, K, nnz;
    int32_t group_size;
    int32_t device;        /* CUDA ordinal that holds the buffers */
    int64_t device_bytes;  /* device memory the handle owns */
    int64_t max_row_nnz;   /* largest residual row */
} mq_info;

/* Decompose fp32 W[N][K] (host, row-major), pack it and upload it to the
 * current device on `stream`. Returns after the upload completed; W may be
 * freed then. *out = NULL on any error.
 * Errors: INVALID_ARG for NULL pointers, N or K <= 0, K % 128 != 0,
 * K > 65536, rho outside [0, 1], NaN/Inf in W, a scale that overflows fp16,
 * and in block mode N % 16 != 0, block_fraction outside [0, 1] or a negative
 * or non-finite channel weight; UNSUPPORTED for group_size != 128 or an
 * unknown residual_blocks; OUT_OF_MEMORY; CUDA. */
mq_status mq_pack(const float *W_host, int64_t N, int64_t K,
                  const mq_pack_opts *opts, mq_stream stream, mq_weight **out);
/* (For tests: with the environment variable MQ_FAULT_ALLOC=1, mq_pack and
 * mq_pack_decomposed fail with OUT_OF_MEMORY at their first device
 * allocation, before any CUDA call.) */

/* Y[M][N] = X[M][K] * W_hat^T on `stream`, asynchronously: no host sync, no
 * allocation. X and Y are bf16, row-major, device memory of the packing
 * device, 16-byte aligned; Y is overwritten and must not overlap X. The
 * handle is read-only here, so concurrent calls on different streams are
 * safe. M = 0 launches nothing. Every K that mq_pack accepts (up to 65536)
 * is served at every M.
 * Errors: INVALID_ARG for a NULL handle, NULL X/Y with M > 0, M < 0,
 * misaligned X/Y or a current device other than the packing device;
 * UNSUPPORTED for M above 2^23 (more than M = 16 runs the prefill kernel,
 * whose token tiles are counted in 32 bits) or a device ordinal above 63;
 * CUDA when a launch fails. */
mq_status mq_linear(const mq_weight *w, const void *X_dev, int64_t M,
                    void *Y_dev, mq_stream stream);

/* mq_linear, and while it runs, the packed codes and scale words of `next`
 * (the layer that follows on this stream) are requested into the GPU's L2
 * cache: each CTA of the decode kernel issues one bulk L2 prefetch of its
 * share. A decode launch of one layer leaves most of the HBM bandwidth idle
 * (it waits on latency), so the next layer's weights arrive meanwhile and
 * its own launch reads them from L2. The result is that of mq_linear; `next`
 * is only read. For M > 16, or next = NULL, this is mq_linear.
 * Errors as mq_linear, plus INVALID_ARG when `next` lives on another
 * device. */
mq_status mq_linear_prefetch(const mq_weight *w, const void *X_dev, int64_t M, void *Y_dev,
                             const mq_weight *next, mq_stream stream);

/* As mq_linear with an explicit kernel choice (mq_linear: the decode
 * kernels for M <= 16 unless X's slice of a very long K exceeds their shared
 * memory, 16-token decode slices or the prefill kernel for 17..64 tokens as
 * MQ_PATH_AUTO describes, the prefill kernel above). MQ_PATH_DECODE with M > 16 runs
 * consecutive 16-token slices of X and Y, one decode launch each (the weight
 * is read once per slice); UNSUPPORTED when the decode kernels cannot take
 * a slice. */
mq_status mq_linear_path(const mq_weight *w, const void *X_dev, int64_t M,
                         void *Y_dev, mq_stream stream, mq_path path);

/* The split execution the fused pass avoids ("Methodology" 3.: a separate
 * residual kernel reloads the activations and merges partial outputs), kept
 * as the comparison the fused kernels are measured against. The dense base
 * kernel writes fp32 partial outputs into `workspace`, then a second kernel
 * re-reads X, adds the residual to the partials and writes bf16 Y (one
 * rounding, so the result meets the same bounds as mq_linear).
 * workspace: caller-owned device memory of at least M*N*4 bytes, 16-byte
 * aligned, not shared with a concurrent call. Errors as mq_linear, plus
 * INVALID_ARG for a NULL, misaligned or too small workspace. */
mq_status mq_linear_unfused(const mq_weight *w, const void *X_dev, int64_t M,
                            void *Y_dev, void *workspace, size_t workspace_bytes,
                            mq_stream stream);

/* Largest M*N mq_linear_unfused_noalloc accepts (its built-in scratch). */
#define MQ_UNFUSED_NOALLOC_MAX_OUTPUTS (2 * 1024 * 1024)

/* mq_linear_unfused for callers that cannot allocate device memory. The
 * paper has no counterpart: this is a deployment variant of the unfused
 * comparison path. Some callers cannot hand out a workspace or call
 * cudaMalloc: code that runs inside a fixed memory budget or a pool it does
 * not own, plugins that only receive their input and output buffers, hosts
 * that route every device allocation through their own allocator. This call
 * keeps the M*N fp32 partial outputs in a fixed array inside the library
 * (MQ_UNFUSED_NOALLOC_MAX_OUTPUTS floats, 8 MiB, held on every GPU that
 * loads the library until the process exits) and performs no allocation of
 * any kind. Results match mq_linear_unfused.
 * The first call on each device looks up the array's device address with
 * that device current, and looks it up again when called under another
 * CUDA context of the device (after cudaDeviceReset, or with a non-primary
 * context current); make such first calls before any stream capture. All calls on a
 * device share the array, which keeps the last call's contents (nothing in
 * it needs to start at zero); calls whose GPU work overlaps in time race.
 * Errors as mq_linear, plus INVALID_ARG when M*N exceeds
 * MQ_UNFUSED_NOALLOC_MAX_OUTPUTS and CUDA when the address lookup fails. */
mq_status mq_linear_unfused_noalloc(const mq_weight *w, const void *X_dev,
                                    int64_t M, void *Y_dev, mq_stream stream);

/* --- W4A4: activations quantized to 4 bits as well ---
 * MosaicQuant "Methodology" 3. (ZipperEngine) starts its pipeline with a
 * quantization stage, and "Experimental Results" evaluate the method as
 * W4A4. The pages fix no activation format; this library reads it as
 * per-token symmetric int4:
 *   s_x[m] = fp32(max_k |x[m][k]| / 7), one IEEE fp32 division (1 when the
 *            token is all zeros);
 *   c[m][k] = clamp(rne(fp32(x[m][k] / s_x[m])), -8, 7), again one IEEE
 *            fp32 division and round-half-to-even;
 *   Y[m][n] = s_x[m] * (sum_g s[n][g] * sum_{k in g} (q - z) * c[m][k]
 *                       + s_r[n] * sum_{residual entries} q_r * c[m][col]),
 * the integer sums exact (int32), the scaling in fp32, Y stored as bf16. */

/* The quantization stage alone: per-token scales and codes of bf16 X.
 * X_dev: bf16 [M][K] row-major, 16-byte aligned, K a positive multiple of 8.
 * codes_dev: int8 [M][K] row-major, scales_dev: float [M]; both caller-owned
 * device memory, 16-byte aligned, written asynchronously on `stream`.
 * M = 0 launches nothing. Errors: INVALID_ARG for NULL or misaligned
 * pointers with M > 0, M < 0, or K not a positive multiple of 8; CUDA. */
mq_status mq_quantize_activations(const void *X_dev, int64_t M, int64_t K, void *codes_dev,
                                  float *scales_dev, mq_stream stream);

/* Device bytes of the workspace mq_linear_w4a4 needs for M tokens of this
 * weight (the codes and scales of X). 0 for a NULL handle or M <= 0. */
int64_t mq_w4a4_workspace_bytes(const mq_weight *w, int64_t M);

/* Y[M][N] for the W4A4 reading above: quantizes X into `workspace`, then
 * one fused pass computes the dense int4 x int4 base (int8 tensor-core MMAs,
 * exact int32 group sums), the int4 x int4 residual and the scaling.
 * X, Y as for mq_linear; workspace: caller-owned device memory of at least
 * mq_w4a4_workspace_bytes(w, M) bytes, 16-byte aligned, not shared with a
 * concurrent call. Asynchronous, no allocation. M <= 16 runs the decode
 * kernels (int8 mma.sync); larger M the prefill kernel (tcgen05 kind::i8
 * MMAs into int32 in tensor memory), which needs K to be a multiple of 256:
 * UNSUPPORTED otherwise, and for M above 2^23. Errors as mq_linear, plus
 * INVALID_ARG for a NULL, misaligned or too small workspace. */
mq_status mq_linear_w4a4(const mq_weight *w, const void *X_dev, int64_t M, void *Y_dev,
                         void *workspace, size_t workspace_bytes, mq_stream stream);

/* Release every buffer of the handle. NULL-safe. Waits for no stream: the
 * caller makes sure no call using the handle is still in flight. */
void mq_free(mq_weight *w);

/* --- support for tests and benchmarks (not needed for inference) --- */

/* Failure detection self-test, on the current device, synchronous: runs the
 * bounded mbarrier wait every pipeline uses on a barrier phase that nobody
 * completes, with a limit of `limit_cycles` clock cycles (at most 2^31; the
 * pipelines use 2e9). results[0..3] = {a wait on a completed phase returned
 * true, the stuck wait returned true, a wait after it returned true, the
 * error code recorded}; a working wait gives {1, 0, 0, 2}: the stuck wait
 * gave up, recorded code 2 and made the later wait return at once. The GPU
 * is never hung: the stuck wait ends after its limit.
 * Errors: INVALID_ARG for NULL results or a limit outside (0, 2^31]; CUDA. */
mq_status mq_selftest_bounded_wait(int64_t limit_cycles, int32_t *results);

/* A measuring aid with no counterpart in the paper: one pure streaming read
 * of `bytes` bytes at buf_dev (device memory, 16-byte aligned, bytes a
 * positive multiple of 16), shaped for the attainable HBM read bandwidth: a
 * persistent grid of two CTAs per SM over contiguous stretches, eight
 * 16-byte streaming loads in flight per thread, programmatic dependent
 * launch (the next launch is released at once; this one waits for its
 * predecessor only before its last write). sink_dev (4 bytes, device) is
 * written only on a data pattern that practically never occurs, so the
 * loads cannot be dropped. Asynchronous on `stream`; the caller owns both
 * buffers. A graph of these launches with a decode step's byte counts gives
 * the read ceiling for that chain of launches.
 * Errors: INVALID_ARG for NULL or misaligned pointers or a bad size; CUDA
 * when the launch fails. */
mq_status mq_read_probe(const void *buf_dev, int64_t bytes, void *sink_dev, mq_stream stream);

/* Residual entries a pack with these options produces: N * k_n in row mode,
 * (selected blocks) * 1024 in block mode. */
mq_status mq_residual_nnz(int64_t N, int64_t K, const mq_pack_opts *opts,
                          int64_t *nnz);

/* Decompose and pack on the host only (no CUDA call at all) into caller
 * buffers sized with mq_residual_nnz. Same validation as mq_pack. */
mq_status mq_pack_host(const float *W_host, int64_t N, int64_t K,
                       const mq_pack_opts *opts, mq_host_packed *out);

/* Test support, no CUDA call: the residual of a host pack regrouped as the
 * prefill kernel reads it. row_ptr [N+1], col [nnz], val [(nnz+1)/2] are the
 * packed CSR (mq_pack_host) of an N x K weight, K a multiple of 64. Writes
 * ptr: int32 [ceil(N/128) * (K/64) * 4 + 1], the first entry of each
 * (128-row tile, 64-column stage, 32-row quadrant) group in that order, and
 * ent: uint32 [nnz], each entry as row-in-tile | column-in-stage << 8 |
 * bf16 bits of q_r << 16, ordered by (group, row, column). INVALID_ARG for
 * a bad shape, NULL buffers, a malformed row_ptr or a column not below K. */
mq_status mq_prefill_lists_host(int64_t N, int64_t K, const int32_t *row_ptr, const uint16_t *col,
                                const uint8_t *val, int32_t *ptr, uint32_t *ent);

/* Test support, no CUDA call: the residual of a host pack regrouped as the
 * wide decode kernel reads it, per (128-row block, 256-column stage) slice
 * (S = ceil(K/256) stages, K a multiple of 128). Inside a slice the entries
 * are ordered by the sub-key (row % 128) / 16 * 16 + (column % 256) / 128 * 8
 * + (column % 32) / 4 (warp tile, 128-column group, MMA k-step), then by row
 * and column. Writes ptr: int32 [ceil(N/128) * S + 1] slice starts; off:
 * uint16 [ceil(N/128) * S * 136], off[slice * 136 + u] (u = 0..128) the start
 * of sub-key u inside the slice; ent: uint16 [nnz], each entry as
 * column % 256 | (row % 16) << 8 | stored nibble << 12; *max_len the longest
 * slice. Errors as mq_prefill_lists_host. */
mq_status mq_wide_lists_host(int64_t N, int64_t K, const int32_t *row_ptr, const uint16_t *col,
                             const uint8_t *val, int32_t *ptr, uint16_t *off, uint16_t *ent,
                             int64_t *max_len);

/* Test support, no CUDA call: the residual of a host pack regrouped as the
 * tall-layer decode kernel reads it, per key row / 16 * (K/128) + column /
 * 128 (16-row tile, 128-column group), K a multiple of 128. Each entry is
 * stored as the byte it takes in the group's eight m16n8k16 bf16 A-fragment
 * tiles (512 bytes per MMA k-step; k-step (column % 32) / 4, where under the
 * packed codes' nibble interleave thread t = (column % 128) / 32 of row group
 * row % 8 holds it in register row % 16 / 8 + 2 * ((column % 4) / 2), half
 * column % 2): ((column % 32) / 4) * 512 + ((row % 8) * 4 + t) * 16 +
 * register * 4 + half * 2, with the stored nibble << 12. Writes ptr: int32
 * [ceil(N/16) * (K/128) + 1] key starts; ent: uint16 [nnz] in CSR order
 * inside a key. Errors as mq_prefill_lists_host. */
mq_status mq_tile_lists_host(int64_t N, int64_t K, const int32_t *row_ptr, const uint16_t *col,
                             const uint8_t *val, int32_t *ptr, uint16_t *ent);

/* Pack a given decomposition (validated: code ranges, integer zero points
 * 0..15, finite scales, CSR structure) and upload it like mq_pack. */
mq_status mq_pack_decomposed(const mq_decomp *d, mq_stream stream,
                             mq_weight **out);

/* Shape and footprint of a handle. */
mq_status mq_get_info(const mq_weight *w, mq_info *out);

/* Copy the packed bytes of a handle back into caller host buffers (sized
 * from mq_get_info). Synchronous: waits for the device. */
mq_status mq_export(const mq_weight *w, mq_host_packed *out);

/* Block tiles. When a residual consists of whole 16-row x 64-column blocks
 * on the block grid (the block allocation of "Methodology" 2., Block-Wise
 * Residual Allocation: mq_pack with residual_blocks = 1, or such a
 * decomposition given to mq_pack_decomposed), the library also holds it as
 * block tiles, which the decode kernels run as extra tensor-core passes:
 *   blk_ptr i32 [N/16 + 1]: offsets of each 16-row block-row's blocks;
 *   blk_col u16 [nblk]: the column-block index cb of each block (columns
 *     64*cb .. 64*cb + 63), ascending within a block-row;
 *   blk_q u32 [nblk][16][8]: word w of row r holds, in bits [4j, 4j+4),
 *     u = q_r + 8 (offset binary 0..15) of column 64*cb + 8w + pi(j),
 *     pi = (0,2,4,6,1,3,5,7) as for qweight.
 * The CSR (mq_export) holds the same codes.
 *
 * mq_block_tiles_host computes the tiles of a decomposition on the host (no
 * CUDA call); mq_export_blocks copies a packed weight's tiles to the host
 * (synchronizing its device). Both write *nblk; with blk_ptr = NULL they
 * stop there (a size query), else the three caller-owned buffers must hold
 * N/16 + 1, nblk and nblk * 128 elements.
 * Errors: INVALID_ARG for a NULL d/w or nblk, a NULL buffer when blk_ptr is
 * given, or an invalid decomposition; UNSUPPORTED when the residual is not
 * made of whole blocks (or is empty); CUDA for a failed copy. */
mq_status mq_block_tiles_host(const mq_decomp *d, int32_t *blk_ptr, uint16_t *blk_col,
                              uint32_t *blk_q, int64_t *nblk);
mq_status mq_export_blocks(const mq_weight *w, int32_t *blk_ptr, uint16_t *blk_col,
                           uint32_t *blk_q, int64_t *nblk);

/* Read and clear the handle's device error word: 0 when every kernel since
 * the last read finished its waits, else the code of the wait that gave up.
 * Synchronizes `stream`. Returns MQ_ERR_DEVICE_TIMEOUT when non-zero. */
mq_status mq_device_error(const mq_weight *w, mq_stream stream, int32_t *code);

/* Static text for a status code. */
const char *mq_strerror(mq_status s);

/* One-line reason for the calling thread's most recent failure ("" if none). */
const char *mq_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* MOSAICQ_H */
