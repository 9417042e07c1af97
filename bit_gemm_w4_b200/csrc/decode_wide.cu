// Wide decode kernel: Y[M][N] = X[M][K] * W_hat^T for 8 < M <= 16, one fused
// pass.
//
// MosaicQuant "Methodology" 3. (ZipperEngine): the dense 4-bit base and the
// sparse residual are computed in the same pass over the staged activations
// and meet in one reduction-add.
//
// At 16 tokens X is a quarter as large as the packed codes it meets, so
// staging a CTA's whole slice of X up front (as the narrow decode kernel
// does) costs about as much shared-memory fill as the weights, and long K
// must be split over clusters to fit. This kernel streams instead:
//   * A CTA owns a 128-row block (8 warps x 16 rows) and walks its K range in
//     stages of 256 columns through a ring of NS shared-memory slots. A slot
//     holds one stage of X (up to 16 tokens), the block's packed codes and
//     scale words for the stage, and the block's residual entries whose
//     columns fall in the stage (grouped per block and stage on the host).
//   * Every copy is a cp.async issued NS-1 stages ahead, so the HBM stream
//     never waits for compute. Codes and scale words are copied by the
//     threads that read them back; X and the residual by all threads, which
//     then meet at one barrier per stage.
//   * Dense branch: warp w turns its 16 rows' nibbles into exact bf16 codes
//     (q - z), accumulates the products with mma.sync m16n8k16 in fp32 and
//     rescales each 128-column group by s in fp32.
//   * Sparse branch, on the tensor cores as well: the host orders a warp's
//     residual entries of a stage by MMA k-step, so for every k-step that
//     holds entries the warp's lanes scatter them as exact bf16 codes into a
//     zeroed 512-byte tile laid out in A-fragment order, read their fragment
//     back, clear it, and issue one more mma.sync on the X fragments the
//     dense branch already holds. The cost follows the entry count however
//     the entries cluster (an outlier-inflated group can put a row's whole
//     residual in one stage), and k-steps without entries cost nothing. The
//     fp32 sum is multiplied by s_r at the end.
//   * Reduction-add: dense sums and s_r times the residual sums meet in a
//     [128][16] fp32 tile and are stored once as bf16.
//   * The kernel is used when the 128-row blocks alone fill the GPU (one CTA
//     per block, two per SM); smaller layers keep the narrow kernel, whose
//     K split serves them better.
// X rows in a slot are 16 bytes longer than 256 columns, and their 16-byte
// chunks are permuted (chunk c sits at c ^ 2 * ((c >> 3) & 1)), so the
// fragment loads of a warp touch distinct banks. The k order inside a group
// follows the same permutation as the narrow kernel (the nibble interleave
// of the packed codes), applied to X and W alike.
//
// Launches use programmatic dependent launch: codes, scales and residual
// entries (which no earlier kernel writes) are requested before
// griddepcontrol.wait; X is read and Y written only after it.
//
// The same ring serves the W4A4 variant (A4 = true): a slot then holds the
// int8 activation codes of the stage (each 8-column chunk's bytes already in
// the packed codes' k order), the dense branch turns nibbles into int8 q - z
// and sums each group exactly with mma.sync m16n8k32 s8, the residual
// k-steps become int8 fragments, and Y = s_x * (sum_g s_g D_g + s_r R).

#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "kernels.h"

namespace mq {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kBN = 16 * kWarps;             // rows per CTA
constexpr int kKC = 256;                     // columns per stage (two groups)
constexpr int kMX = 16;                      // token capacity
constexpr int kWBytes = kBN * (kKC / 2);     // [warp][group][16 rows][64 B]
constexpr int kSZBytes = kBN * 2 * 4;        // [warp][group][16 rows] u32
constexpr int kOffBytes = kWideOffStride * 2;
// A slot: codes, scale words, residual offsets, residual entries, then X.
constexpr int kSZOff = kWBytes, kOffOff = kSZOff + kSZBytes, kEntOff = kOffOff + kOffBytes;
// X row stride in a slot (bytes): bf16, or int8 codes (W4A4)
template <bool A4>
__host__ __device__ constexpr int x_row_stride() { return A4 ? kKC + 16 : kKC * 2 + 16; }
constexpr int kSmemLimit = 112 * 1024;       // two CTAs per SM

struct WideParams {
    const uint32_t *qweight;  // [N][K/8]
    const uint32_t *sz;       // [N][Gp]
    const __nv_bfloat16 *X;   // [M][K]
    const int8_t *codes;      // [M][K] activation codes (W4A4), chunk bytes permuted
    const float *xscale;      // [M] activation scales (W4A4)
    __nv_bfloat16 *Y;         // [M][N]
    float *Yf;                // fp32 dense-only output (unfused path) or null
    const int32_t *wptr;
    const uint16_t *woff;
    const uint16_t *went;
    const uint16_t *rscale;
    int M, N, K, G, Gp;
    uint32_t bias;  // kBiasBf16, or kBiasI8 for int8 codes (held in a register)
    int S;           // stages over all of K
    int ent_bytes;   // residual entry bytes of one slot; 0 = no residual
    int x_off;       // X's offset in a slot (kEntOff + ent_bytes)
    int slot_bytes;  // bytes of one ring slot
    L2Prefetch pf;   // the next layer's weight, brought into L2 meanwhile
};

// Bytes in front of the ring: the CTA's slice-start table, copied in 16-byte
// chunks from a 4-entry-aligned start, then one residual fragment tile per
// warp.
__host__ __device__ constexpr int wtab_bytes(int spr) { return ((spr + 8) / 4 + 1) * 16; }
constexpr int kFrag = 512;               // 16 rows x 16 k-slots of bf16, A-fragment order
constexpr int kTileBytes = 4 * kFrag;    // the fragments of four k-steps
__host__ __device__ constexpr int ring_offset(int spr) { return wtab_bytes(spr) + kWarps * kTileBytes; }

// The same for the int8 m16n8k32 A layout (W4A4): column c of a group sits
// at byte ((c & 3) << 1) | ((c >> 2) & 1) of its 8-column chunk in the
// packed codes' k order; positions 0..3 go to registers (r / 8), 4..7 to
// 2 + (r / 8), of thread (g = r % 8, t = c / 32); k-step (c % 32) / 8.
__device__ __forceinline__ int tile_pos_a4(int r, int c) {
    const int pos = ((c & 3) << 1) | ((c >> 2) & 1);
    return ((r & 7) * 4 + (c >> 5)) * 16 + ((r >> 3) + ((pos >> 2) << 1)) * 4 + (pos & 3);
}

template <bool A4, int NS>
__global__ void __launch_bounds__(kThreads, 2)
    decode_wide_kernel(const __grid_constant__ WideParams p) {
    constexpr int XRS = x_row_stride<A4>();
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t bias = p.bias;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int M = p.M, N = p.N, K = p.K, G = p.G;
    const int blk = blockIdx.x;
    const int n0 = blk * kBN;
    const int j_lo = 0, nj = p.S;
    const bool with_res = p.ent_bytes > 0;

    int32_t *wtab = reinterpret_cast<int32_t *>(smem);
    const int key0 = blk * p.S + j_lo, kbase = key0 & ~3;
    uint8_t *const rtile = smem + wtab_bytes(p.S) + warp * kTileBytes;
    uint8_t *const slots = smem + ring_offset(p.S);
    auto slot_of = [&](int i) { return slots + (i % NS) * p.slot_bytes; };

    // sources of this thread's codes (rows g, g+8 of the warp) and scales
    const size_t wrow = static_cast<size_t>(K) / 8;
    const int ra = min(n0 + 16 * warp + g, N - 1), rb = min(n0 + 16 * warp + g + 8, N - 1);
    const uint32_t *w0 = p.qweight + static_cast<size_t>(ra) * wrow + 4 * t;
    const uint32_t *w1 = p.qweight + static_cast<size_t>(rb) * wrow + 4 * t;
    const int zrow = lane & 15, zj = lane >> 4;
    const uint32_t *szp =
        p.sz + static_cast<size_t>(min(n0 + 16 * warp + zrow, N - 1)) * p.Gp + zj;

    auto issue_weights = [&](int i) {
        uint8_t *sl = slot_of(i);
        const int j = j_lo + i;
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
            const int gi = 2 * j + jj;
            if (gi < G) {
                uint8_t *wd = sl + (warp * 2 + jj) * 16 * 64 + 16 * t;
                cp_async16(wd + g * 64, w0 + gi * 16);
                cp_async16(wd + (g + 8) * 64, w1 + gi * 16);
            }
        }
        if (2 * j + zj < G)
            cp_async4(sl + kSZOff + ((warp * 2 + zj) * 16 + zrow) * 4, szp + 2 * j);
    };
    auto issue_residual = [&](int i) {
        uint8_t *sl = slot_of(i);
        const int key = blk * p.S + j_lo + i;
        if (threadIdx.x < kOffBytes / 16)
            cp_async16(sl + kOffOff + 16 * threadIdx.x,
                       p.woff + static_cast<size_t>(key) * kWideOffStride + 8 * threadIdx.x);
        const int eb = wtab[key - kbase], ee = wtab[key - kbase + 1];
        const int base = eb & ~7, n16 = (ee - base + 7) >> 3;
        uint8_t *ed = sl + kEntOff;
        for (int c = threadIdx.x; c < n16; c += kThreads) cp_async16(ed + 16 * c, p.went + base + 8 * c);
    };
    auto issue_x = [&](int i) {
        uint8_t *sx = slot_of(i) + p.x_off;
        const int k0 = (j_lo + i) * kKC;
        if constexpr (A4) {
            // 16 chunks of 16 codes per token row, one per thread
            const int tok = threadIdx.x >> 4, c = threadIdx.x & 15;
            if (tok < M && 16 * c < K - k0)
                cp_async16(sx + tok * XRS + 16 * c, p.codes + static_cast<size_t>(tok) * K + k0 + 16 * c);
        } else {
            const int chunks = min(kKC, K - k0) / 8;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int idx = threadIdx.x + kThreads * u;
                const int tok = idx >> 5, c = idx & 31;
                if (tok < M && c < chunks)
                    cp_async16(sx + tok * XRS + xchunk(c) * 16,
                               p.X + static_cast<size_t>(tok) * K + k0 + 8 * c);
            }
        }
    };

    // ---------------------------------------------- prologue
    if (with_res) {
        const int cnt = key0 + nj + 1 - kbase;
        for (int c = threadIdx.x; 4 * c < cnt; c += kThreads) cp_async16(wtab + 4 * c, p.wptr + kbase + 4 * c);
        cp_async_commit();
    }
    for (int i = 0; i < NS - 1; ++i)
        if (i < nj) issue_weights(i);
    if (threadIdx.x == 0) l2_prefetch_share(p.pf, blk, static_cast<int>(gridDim.x));
    pdl_launch_dependents();
    if (with_res) {
        cp_async_wait_group<0>();  // the table only: the copies above are not committed yet
        __syncthreads();
        for (int i = 0; i < NS - 1; ++i)
            if (i < nj) issue_residual(i);
    }
    pdl_wait();  // X may come from the previous kernel; Y may still be read by it
    for (int i = 0; i < NS - 1; ++i) {
        if (i < nj) issue_x(i);
        cp_async_commit();
    }

    // ---------------------------------------------- stages
    float acc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
    // sparse branch, in the accumulator layout of acc (fp32 sums of exact
    // bf16 products, or exact int32 sums for W4A4)
    using RAcc = typename std::conditional<A4, int, float>::type;
    RAcc racc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) racc[nt][i] = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) sts128(rtile + u * kFrag + 16 * lane, make_uint4(0u, 0u, 0u, 0u));
    __syncwarp();

    for (int i = 0; i < nj; ++i) {
        cp_async_wait_group<NS - 2>();
        __syncthreads();  // stage i is visible to all; slot (i - 1) % NS is free
        if (i + NS - 1 < nj) {
            issue_weights(i + NS - 1);
            if (with_res) issue_residual(i + NS - 1);
            issue_x(i + NS - 1);
        }
        cp_async_commit();

        const uint8_t *sl = slot_of(i);
        const uint8_t *sx = sl + p.x_off;
        const int j = j_lo + i;
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
            const int gi = 2 * j + jj;
            if (gi >= G) break;
            // ---------------------------------------- dense branch
            const uint8_t *wd = sl + (warp * 2 + jj) * 16 * 64 + 16 * t;
            const uint4 wa = lds128(wd + g * 64), wb = lds128(wd + (g + 8) * 64);
            const uint32_t *zs = reinterpret_cast<const uint32_t *>(sl + kSZOff) + (warp * 2 + jj) * 16;
            const uint32_t sz0 = zs[g], sz1 = zs[g + 8];
            const float s0 = half_bits_to_f32(sz0), s1 = half_bits_to_f32(sz1);
            const uint32_t z0 = static_cast<uint32_t>(half_bits_to_f32(sz0 >> 16));
            const uint32_t z1 = static_cast<uint32_t>(half_bits_to_f32(sz1 >> 16));
            const uint32_t wr0[4] = {wa.x, wa.y, wa.z, wa.w};
            const uint32_t wr1[4] = {wb.x, wb.y, wb.z, wb.w};
            // X fragments of tokens g and g + 8 (16 words of bf16 pairs, or 8
            // words of int8 codes)
            constexpr int XW = A4 ? 8 : 16;
            uint32_t xb[2][XW];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const int tok = g + 8 * nt;
                if (tok < M) {
                    const uint8_t *xr = sx + tok * XRS;
#pragma unroll
                    for (int q = 0; q < XW / 4; ++q) {
                        const uint4 v = A4 ? lds128(xr + jj * 128 + 32 * t + 16 * q)
                                           : lds128(xr + xchunk(16 * jj + 4 * t + q) * 16);
                        xb[nt][4 * q + 0] = v.x;
                        xb[nt][4 * q + 1] = v.y;
                        xb[nt][4 * q + 2] = v.z;
                        xb[nt][4 * q + 3] = v.w;
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < XW; ++q) xb[nt][q] = 0u;
                }
            }
            if constexpr (A4) {
                const uint32_t zz0 = z0 * 0x01010101u, zz1 = z1 * 0x01010101u;
                int d[2][4];
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int q = 0; q < 4; ++q) d[nt][q] = 0;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    uint32_t a[4];
                    a[0] = codes_minus_zero_r(wr0[ks], zz0, bias);
                    a[1] = codes_minus_zero_r(wr1[ks], zz1, bias);
                    a[2] = codes_minus_zero_r(wr0[ks] >> 4, zz0, bias);
                    a[3] = codes_minus_zero_r(wr1[ks] >> 4, zz1, bias);
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) mma_s8_16832(d[nt], a, xb[nt][2 * ks], xb[nt][2 * ks + 1]);
                }
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    acc[nt][0] = fmaf(s0, static_cast<float>(d[nt][0]), acc[nt][0]);
                    acc[nt][1] = fmaf(s0, static_cast<float>(d[nt][1]), acc[nt][1]);
                    acc[nt][2] = fmaf(s1, static_cast<float>(d[nt][2]), acc[nt][2]);
                    acc[nt][3] = fmaf(s1, static_cast<float>(d[nt][3]), acc[nt][3]);
                }
            } else {
                const uint32_t zz0 = (0x4300u | z0) * 0x00010001u;  // bf16x2 (128+z)
                const uint32_t zz1 = (0x4300u | z1) * 0x00010001u;
                float c[2][4];
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int q = 0; q < 4; ++q) c[nt][q] = 0.f;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t a_lo = wr0[ks >> 1] >> (8 * (ks & 1));
                    const uint32_t b_lo = wr1[ks >> 1] >> (8 * (ks & 1));
                    uint32_t a[4];
                    a[0] = bf16x2_sub(mask_or<0x000F000Fu>(a_lo, bias), zz0);
                    a[1] = bf16x2_sub(mask_or<0x000F000Fu>(b_lo, bias), zz1);
                    a[2] = bf16x2_sub(mask_or<0x000F000Fu>(a_lo >> 4, bias), zz0);
                    a[3] = bf16x2_sub(mask_or<0x000F000Fu>(b_lo >> 4, bias), zz1);
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
                        mma_bf16_16816(c[nt], a, xb[nt][2 * ks], xb[nt][2 * ks + 1], c[nt]);
                }
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    acc[nt][0] = fmaf(s0, c[nt][0], acc[nt][0]);
                    acc[nt][1] = fmaf(s0, c[nt][1], acc[nt][1]);
                    acc[nt][2] = fmaf(s1, c[nt][2], acc[nt][2]);
                    acc[nt][3] = fmaf(s1, c[nt][3], acc[nt][3]);
                }
            }
            // ---------------------------------------- sparse branch
            // the warp's entries of this group, scattered into fragment tiles
            // a half-group (four bf16 k-steps, two int8 k-steps) at a time;
            // k-steps without entries issue no MMA
            if (with_res) {
                const uint16_t *offw =
                    reinterpret_cast<const uint16_t *>(sl + kOffOff) + warp * 16 + jj * 8;
                const uint16_t *ent = reinterpret_cast<const uint16_t *>(sl + kEntOff) +
                                      (wtab[blk * p.S + j - kbase] & 7);
                int o[9];
#pragma unroll
                for (int q = 0; q < 9; ++q) o[q] = static_cast<int>(lds_u16(offw + q));
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    if (o[4 * h + 4] > o[4 * h]) {  // the same for every lane
                        for (int e = o[4 * h] + lane; e < o[4 * h + 4]; e += 32) {
                            const uint32_t v = lds_u16(ent + e);
                            const int c = static_cast<int>(v & 0x7Fu);
                            const int r = static_cast<int>((v >> 8) & 0xFu);
                            const int q = static_cast<int>(((v >> 12) & 0xFu) ^ 8u) - 8;
                            if constexpr (A4)
                                sts_u8(rtile + ((c >> 3) & 1) * kFrag + tile_pos_a4(r, c),
                                       static_cast<uint32_t>(q) & 0xFFu);
                            else
                                sts_u16(rtile + (((c & 31) >> 2) & 3) * kFrag + tile_pos(r, c),
                                        __float_as_uint(static_cast<float>(q)) >> 16);
                        }
                        __syncwarp();
                        constexpr int KPH = A4 ? 2 : 4;  // k-steps per half-group
#pragma unroll
                        for (int u = 0; u < KPH; ++u) {
                            const int ks = KPH * h + u;  // k-step of the group
                            const int l0 = A4 ? 2 * ks : ks, l1 = A4 ? 2 * ks + 2 : ks + 1;
                            if (o[l1] > o[l0]) {
                                const uint4 f = lds128(rtile + u * kFrag + 16 * lane);
                                sts128(rtile + u * kFrag + 16 * lane, make_uint4(0u, 0u, 0u, 0u));
                                const uint32_t fa[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
                                for (int nt = 0; nt < 2; ++nt) {
                                    if constexpr (A4)
                                        mma_s8_16832(racc[nt], fa, xb[nt][2 * ks], xb[nt][2 * ks + 1]);
                                    else
                                        mma_bf16_16816(racc[nt], fa, xb[nt][2 * ks],
                                                       xb[nt][2 * ks + 1], racc[nt]);
                                }
                            }
                        }
                        __syncwarp();
                    }
                }
            }
        }
    }

    // ---------------------------------------------- reduction-add
    cp_async_wait_all();
    __syncthreads();  // every slot is idle: the result tile reuses them
    float *res = reinterpret_cast<float *>(slots);  // [kBN][kMX]
    float sra = 0.f, srb = 0.f;
    if (with_res) {
        const int na = n0 + 16 * warp + g, nb = na + 8;
        if (na < N) sra = half_bits_to_f32(p.rscale[na]);
        if (nb < N) srb = half_bits_to_f32(p.rscale[nb]);
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int row = 16 * warp + g + ((i < 2) ? 0 : 8);
            const int tok = 8 * nt + 2 * t + (i & 1);
            float y = fmaf(i < 2 ? sra : srb, static_cast<float>(racc[nt][i]), acc[nt][i]);
            if constexpr (A4) y *= tok < M ? p.xscale[tok] : 0.f;
            res[row * kMX + tok] = y;
        }
    __syncthreads();
    for (int idx = threadIdx.x; idx < M * kBN; idx += kThreads) {
        const int m = idx / kBN, r = idx % kBN, n = n0 + r;
        const float y = res[r * kMX + m];
        if (n < N) {
            if (p.Yf)
                p.Yf[static_cast<size_t>(m) * N + n] = y;
            else
                p.Y[static_cast<size_t>(m) * N + n] = __float2bfloat16_rn(y);
        }
    }
}

template <bool A4, int NS>
mq_status run(const WideParams &p, int smem, int blocks, cudaStream_t stream) {
    auto kern = decode_wide_kernel<A4, NS>;
    static bool configured[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(MQ_ERR_CUDA, "cudaGetDevice failed");
    if (dev >= 0 && dev < 64 && !configured[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit) !=
                cudaSuccess ||
            cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared) != cudaSuccess)
            return fail(MQ_ERR_CUDA, "cudaFuncSetAttribute failed for the wide decode kernel");
        configured[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(blocks));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = stream;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p);
    if (e != cudaSuccess)
        return fail(MQ_ERR_CUDA, std::string("wide decode launch: ") + cudaGetErrorString(e));
    return MQ_OK;
}

// Fills the shared part of the parameters and picks the ring depth; returns
// MQ_ERR_UNSUPPORTED (no message) when the kernel should not or cannot take
// the call.
template <bool A4>
mq_status launch(WideParams &p, const DeviceWeight &d, int M, bool with_res, bool force,
                 cudaStream_t stream) {
    if (M <= 8 || M > kMX) return MQ_ERR_UNSUPPORTED;
    p.qweight = d.qweight;
    p.sz = d.sz;
    p.wptr = d.wide_ptr;
    p.woff = d.wide_off;
    p.went = d.wide_ent;
    p.rscale = d.rscale;
    p.M = M;
    p.N = static_cast<int>(d.N);
    p.K = static_cast<int>(d.K);
    p.G = static_cast<int>(d.G);
    p.Gp = static_cast<int>(d.Gp);
    p.bias = A4 ? kBiasI8 : kBiasBf16;
    p.S = static_cast<int>((d.K + kKC - 1) / kKC);
    const int64_t blocks = (d.N + kBN - 1) / kBN;
    if (blocks < sm_count() && !force) return MQ_ERR_UNSUPPORTED;  // the narrow kernels serve small layers
    p.ent_bytes = with_res ? static_cast<int>(((d.wide_max + 15) / 8 + 1) * 16) : 0;
    if (with_res && (!d.wide_ptr || !d.wide_off || !d.wide_ent)) return MQ_ERR_UNSUPPORTED;
    p.x_off = kEntOff + p.ent_bytes;
    p.slot_bytes = (p.x_off + kMX * x_row_stride<A4>() + 127) / 128 * 128;
    int ns = 4;
    while (ns >= 2 && ring_offset(p.S) + ns * p.slot_bytes > kSmemLimit) --ns;
    if (ns < 2) return MQ_ERR_UNSUPPORTED;  // a residual slice too long for the ring
    const int smem = ring_offset(p.S) + ns * p.slot_bytes;
    switch (ns) {
        case 4: return run<A4, 4>(p, smem, static_cast<int>(blocks), stream);
        case 3: return run<A4, 3>(p, smem, static_cast<int>(blocks), stream);
        default: return run<A4, 2>(p, smem, static_cast<int>(blocks), stream);
    }
}

}  // namespace

mq_status launch_decode_wide(const mq_weight *w, const void *X, int M, void *Y,
                             cudaStream_t stream, float *partial, const L2Prefetch &pf,
                             bool force) {
    const DeviceWeight &d = weight_device(w);
    WideParams p{};
    p.X = static_cast<const __nv_bfloat16 *>(X);
    p.Y = static_cast<__nv_bfloat16 *>(Y);
    p.Yf = partial;
    p.pf = pf;
    return launch<false>(p, d, M, partial == nullptr && d.nnz > 0, force, stream);
}

mq_status launch_decode_wide_a4(const mq_weight *w, const int8_t *codes, const float *xscale,
                                int M, void *Y, cudaStream_t stream) {
    const DeviceWeight &d = weight_device(w);
    WideParams p{};
    p.codes = codes;
    p.xscale = xscale;
    p.Y = static_cast<__nv_bfloat16 *>(Y);
    return launch<true>(p, d, M, d.nnz > 0, false, stream);
}

}  // namespace mq
