// Streaming decode kernel: Y[M][N] = X[M][K] * W_hat^T for M <= 16 where X
// fits its shared memory, one fused pass over the packed weight (at 9-16
// tokens two 8-token MMA column tiles share each converted code fragment).
//
// MosaicQuant "Methodology" 3. (ZipperEngine): the sparse residual is
// computed inside the dense 4-bit GEMM pass over the same activations, and
// the dense and sparse parts meet in one reduction-add.
//
// At a few tokens the layer is a read of the packed weight, and a decode
// step is a chain of such launches. The kernel is shaped so that the chain
// streams HBM without gaps:
//   * Persistent: one CTA per SM, each owning a contiguous run of NT or
//     NT - 1 16-row tiles (NT <= 8, a template parameter), so a CTA's bytes
//     are one contiguous stretch of every packed array.
//   * Small footprint (256 threads, at most 128 registers, under 100 KB of
//     shared memory for the 7B-sized layers), so the next launch's CTAs fit
//     beside this one's. With programmatic dependent launch every CTA
//     releases the next grid at its first instruction; the next layer's
//     weight stream then runs while this layer computes and drains, and only
//     its read of X waits for this grid.
//   * Every thread prefetches its own share of the packed codes through a
//     private ring of D groups x NT tiles of cp.async stages in shared memory
//     (no barrier between threads; each thread waits for its own copies). A
//     slot is refilled with the item D groups ahead as soon as it has been
//     consumed; slots, tiles and the wait depth are all compile-time
//     constants, so the stream costs a few instructions per item.
//   * The run's scale/zero words, its CSR slice (row offsets, columns,
//     codes) and X are copied into shared memory once.
//   * Warp w takes groups w, w+8, ... : for each group it loads the X
//     fragment once, then walks the run's tiles (its rows g and g+8, 16
//     bytes of each), keeping one fp32 accumulator set per tile in
//     registers. Each group's nibbles become exact bf16 codes q - z (a mask
//     into the mantissa of 128.0, then a subtraction of 128 + z); mma.sync
//     m16n8k16 sums the exact products in fp32 and the group's partial is
//     scaled by s in fp32. Subtracting (128 + z) * sum(x) once per group
//     instead would save the subtraction, but the fp32 sums of (128 + q) * x
//     then lose about 1e-5 absolute to cancellation, more than the
//     per-element tolerance allows on small outputs.
//   * Residual: after the dense pass, each half-warp walks the CSR entries of
//     one row per tile (16 lanes per row), gathers x[m][col] from shared
//     memory and reduces with shuffles; s_r times the sum joins the
//     reduction.
//   * Reduction-add: the eight warps' partials and the residual meet in
//     shared memory and are stored once as bf16.
// The k order inside a group is permuted so that each thread's 16-byte load
// of packed codes feeds its own mma fragments with no shuffles: k-step s'
// (0..7) of thread (g, t) covers columns 32t + 4s' + {0,1} and 32t + 4s' +
// {2,3}; X is read in the same order, so the sum over k is unchanged.
// X rows in shared memory are 16 bytes longer than K columns and each
// group's 16-byte chunks are permuted (chunk c sits at c ^ 2 * ((c >> 3) &
// 1)); scale/zero rows are padded to an odd multiple of four words. Both
// keep a warp's shared-memory loads on distinct banks.

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "kernels.h"

namespace mq {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kTMax = 8;     // most tiles per CTA (one accumulator set each)
constexpr int kMaxSmem = 227 * 1024;
constexpr int kTwoPerSm = 113 * 1024;  // shared memory of each of two CTAs per SM
constexpr int kCsrBudget = 24 * 1024;    // shared memory for a CTA's CSR slice
constexpr int kBlockBudget = 48 * 1024;  // shared memory for a CTA's block tiles

// Groups of prefetch ahead for NT tiles per CTA: eight to ten items per
// thread (64-80 KB per CTA in flight), or one group for NT > 5; half as many
// at 16 tokens, where X takes most of the shared memory.
__host__ __device__ constexpr int groups_ahead(int nt, bool wide_x = false) {
    return wide_x ? (nt >= 3 ? 1 : nt == 2 ? 2 : 4)
                  : (nt >= 6 ? 1 : nt >= 4 ? 2 : nt == 3 ? 3 : nt == 2 ? 4 : 8);
}

struct StreamParams {
    const uint32_t *qweight;  // [N][K/8]
    const uint32_t *sz;       // [N][Gp]
    const __nv_bfloat16 *X;   // [M][K]
    __nv_bfloat16 *Y;         // [M][N]
    float *Yf;                // fp32 dense-only output (unfused path) or null
    const int32_t *row_ptr;
    const uint16_t *col;
    const uint8_t *val;
    const uint16_t *rscale;
    int M, N, K, G, Gp;
    int ntile;      // ceil(N / 16)
    int csr_cap;    // most residual entries of a CTA's run; 0: no CSR walk
    // block tiles of a block-allocated residual (blk_cap > 0: the most blocks
    // of a CTA's run; the residual then runs as tensor-core passes and the
    // CSR is not read)
    const int32_t *blk_ptr;
    const uint32_t *blk_q;
    const uint32_t *blk_map;
    int blk_words, blk_cap;
    // 0x43004300 (bf16x2 128.0, 128.0), passed at run time so that it sits in
    // a register and each code pair costs one LOP3 (mask and OR)
    uint32_t bias;
    L2Prefetch pf;  // another weight, brought into L2 meanwhile
};


// Shared-memory layout (bytes), identical on host and device.
struct StreamLayout {
    int ring, x, xrs, szs, red, res, rsf, rp, col, val, bq, bmap, bpre, total;
    __host__ __device__ StreamLayout(int M, int K, int Gp, int csr_cap, int nt, int blk_cap = 0,
                                     int blk_words = 0) {
        ring = 0;                                                       // [D * NT][2][kThreads][16 B]
        x = ring + groups_ahead(nt, M > 8) * nt * 2 * kThreads * 16;   // [M][xrs]
        xrs = K * 2 + 16;
        szs = x + (M * xrs + 15) / 16 * 16;                    // [NT * 16][sz_stride] words
        red = szs + nt * 16 * sz_stride(Gp) * 4;               // [NT][warp][M][16] fp32
        res = red + nt * kWarps * M * 16 * 4;                  // [NT][M][16] fp32
        rsf = res + nt * M * 16 * 4;                           // [NT * 16] fp32 s_r
        rp = rsf + nt * 16 * 4;                                // [NT * 16 + 1] i32
        col = rp + (csr_cap > 0 ? (nt * 16 + 1) * 4 + 15 : 0) / 16 * 16;
        val = col + (csr_cap > 0 ? csr_cap * 2 + 32 : 0);
        bq = val + (csr_cap > 0 ? csr_cap / 2 + 48 : 0);                  // [blk_cap][512 B]
        bmap = bq + blk_cap * 512;                                        // [NT][blk_words] bitmaps
        bpre = bmap + (blk_cap > 0 ? nt * blk_words * 4 : 0);            // [NT][blk_words] block counts before each word
        total = bpre + (blk_cap > 0 ? nt * blk_words * 4 : 0);
    }
};



template <int MX, int NT, bool BLK>
__global__ void __launch_bounds__(kThreads, 2) decode_stream_kernel(const __grid_constant__ StreamParams p) {
    constexpr int NTOK = MX > 8 ? 2 : 1;  // 8-token MMA column tiles
    constexpr int D = groups_ahead(NT, MX > 8);
    constexpr int R = D * NT;  // ring slots (items) per thread
    extern __shared__ __align__(16) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int M = MX == 1 ? 1 : p.M, N = p.N, K = p.K, G = p.G;
    const StreamLayout L(M, K, p.Gp, p.csr_cap, NT, p.blk_cap, p.blk_words);
    const int SZS = sz_stride(p.Gp);
    const int t0 = static_cast<int>(static_cast<long long>(p.ntile) * blockIdx.x / gridDim.x);
    const int t1 = static_cast<int>(static_cast<long long>(p.ntile) * (blockIdx.x + 1) / gridDim.x);
    const int nt = t1 - t0;      // NT or NT - 1
    const bool full = nt == NT;  // only tile NT - 1 can be missing
    const int gpw = warp < G ? (G - warp + kWarps - 1) / kWarps : 0;  // groups of this warp
    const bool resid = p.csr_cap > 0;
    // the block-tile residual path exists only in its own instantiations, so
    // that the row-residual kernels carry none of its code
    constexpr bool blocks = BLK;

    // ------------------------------------------------ the weight stream
    // Row offsets (words) of this thread's rows g and g+8 in each tile, and
    // its 16-byte column within a group.
    uint32_t off0[NT], off1[NT];
    const uint32_t wrow = static_cast<uint32_t>(K / 8);
#pragma unroll
    for (int k = 0; k < NT; ++k) {
        off0[k] = static_cast<uint32_t>(min((t0 + k) * 16 + g, N - 1)) * wrow;
        off1[k] = static_cast<uint32_t>(min((t0 + k) * 16 + g + 8, N - 1)) * wrow;
    }
    const uint32_t *qbase = p.qweight + warp * 16 + 4 * t;
    uint8_t *ring = smem + L.ring + threadIdx.x * 16;
    // item (group j of this warp, tile k) into the slot at dst (a copy that
    // is not live writes zeros: a source size of 0; the address stays in
    // bounds)
    auto issue = [&](int j, int k, uint8_t *dst) {
        // past the warp's last group the copy repeats that group (clamped
        // below: an L2 hit, never consumed), so only a warp without groups
        // and a CTA's missing last tile copy nothing
        const bool live = gpw > 0 && (k + 1 < NT || full);
        const uint32_t *src = qbase + min(j, gpw - 1) * (kWarps * 16);
        cp_async16_if(dst, src + off0[k], live);
        cp_async16_if(dst + kThreads * 16, src + off1[k], live);
        cp_async_commit();
    };
#pragma unroll
    for (int d = 0; d < D; ++d)
#pragma unroll
        for (int k = 0; k < NT; ++k) issue(d, k, ring + (d * NT + k) * (2 * kThreads * 16));
    pdl_launch_dependents();
    if (threadIdx.x == 0) {
        l2_prefetch_share(p.pf, blockIdx.x, gridDim.x);
        // X into L2 ahead of the wait: L2 is coherent, so a write of X by the
        // previous grid after this prefetch still reaches the reads below
        const long long xb = static_cast<long long>(M) * K * 2;
        for (long long o = 0; o < xb; o += 1 << 16) {
            const unsigned n = static_cast<unsigned>(xb - o < (1 << 16) ? xb - o : (1 << 16));
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<const char *>(p.X) + o), "r"(n)
                         : "memory");
        }
    }

    // ------------------------------------------------ the run's scale/zero words and CSR slice
    const int n_lo = t0 * 16, n_hi = min(t1 * 16, N);
    {
        const int q4 = p.Gp / 4;  // 16-byte chunks per scale/zero row
        for (int i = threadIdx.x; i < (n_hi - n_lo) * q4; i += kThreads) {
            const int r = i / q4, q = i - r * q4;
            cp_async16(smem + L.szs + (r * SZS + 4 * q) * 4,
                       p.sz + static_cast<size_t>(n_lo + r) * p.Gp + 4 * q);
        }
    }
    int col_base = 0, val_base = 0;
    if (resid) {
        for (int i = threadIdx.x; i <= n_hi - n_lo; i += kThreads)
            cp_async4(smem + L.rp + 4 * i, p.row_ptr + n_lo + i);
        const int e_lo = p.row_ptr[n_lo], e_hi = p.row_ptr[n_hi];
        col_base = e_lo & ~7;
        val_base = (e_lo >> 1) & ~15;
        const int ncol16 = ((e_hi - col_base) * 2 + 15) / 16;
        const int nval16 = (((e_hi + 1) >> 1) - val_base + 15) / 16;
        for (int i = threadIdx.x; i < ncol16; i += kThreads)
            cp_async16(smem + L.col + 16 * i, p.col + col_base + 8 * i);
        for (int i = threadIdx.x; i < nval16; i += kThreads)
            cp_async16(smem + L.val + 16 * i, p.val + val_base + 16 * i);
    }
    int b_lo = 0;
    if (blocks) {
        // the run's block tiles (contiguous) and its block-rows' bitmaps
        b_lo = p.blk_ptr[t0];
        const int nb16 = (p.blk_ptr[t1] - b_lo) * 32;  // 16-byte pieces
        for (int i = threadIdx.x; i < nb16; i += kThreads)
            cp_async16(smem + L.bq + 16 * i, p.blk_q + static_cast<size_t>(b_lo) * 128 + 4 * i);
        for (int i = threadIdx.x; i < nt * p.blk_words; i += kThreads)
            cp_async4(smem + L.bmap + 4 * i, p.blk_map + static_cast<size_t>(t0) * p.blk_words + i);
    }
    cp_async_commit();
    if (resid || blocks)
        for (int i = threadIdx.x; i < n_hi - n_lo; i += kThreads)
            reinterpret_cast<float *>(smem + L.rsf)[i] = half_bits_to_f32(p.rscale[n_lo + i]);
    if (blocks)
        // each tile's blocks before each bitmap word, counted from the run's first block
        for (int k = threadIdx.x; k < nt; k += kThreads) {
            int c = p.blk_ptr[t0 + k] - b_lo;
            for (int wd = 0; wd < p.blk_words; ++wd) {
                reinterpret_cast<int *>(smem + L.bpre)[k * p.blk_words + wd] = c;
                c += __popc(p.blk_map[static_cast<size_t>(t0 + k) * p.blk_words + wd]);
            }
        }

    // ------------------------------------------------ X
    pdl_wait();  // X may come from the previous kernel; Y may still be read by it
    {
        const int chunks = K / 8;  // 16-byte chunks per token row
        for (int m = 0; m < M; ++m)
            for (int c = threadIdx.x; c < chunks; c += kThreads)
                cp_async16(smem + L.x + m * L.xrs + (c >> 4) * 256 + xchunk(c & 15) * 16,
                           p.X + static_cast<size_t>(m) * K + 8 * c);
        cp_async_commit();
    }
    cp_async_wait_all();
    __syncthreads();

    const uint8_t *xs = smem + L.x;
    const uint32_t *szs = reinterpret_cast<const uint32_t *>(smem + L.szs);
    const uint32_t *bmapw = reinterpret_cast<const uint32_t *>(smem + L.bmap);
    const int *bpre = reinterpret_cast<const int *>(smem + L.bpre);
    const float *rsfs = reinterpret_cast<const float *>(smem + L.rsf);
    float *red = reinterpret_cast<float *>(smem + L.red);
    float *res = reinterpret_cast<float *>(smem + L.res);

    // ------------------------------------------------ dense pass
    float acc[NT][NTOK][4];
#pragma unroll
    for (int k = 0; k < NT; ++k)
#pragma unroll
        for (int n8 = 0; n8 < NTOK; ++n8)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[k][n8][i] = 0.f;
    uint32_t xb[NTOK][16];
#pragma unroll
    for (int n8 = 0; n8 < NTOK; ++n8)
#pragma unroll
        for (int i = 0; i < 16; ++i) xb[n8][i] = 0u;
    // one group per iteration, not unrolled over the ring's D groups (a
    // smaller loop body: fewer instruction-cache misses), with the group's
    // ring slots found from d = j mod D at run time
#pragma unroll 1
    for (int j = 0, d = 0; j < gpw; ++j, d = d + 1 == D ? 0 : d + 1) {
        uint8_t *const slots = ring + d * (NT * 2 * kThreads * 16);
        {
            {
                const int gi = warp + kWarps * j;
#pragma unroll
                for (int n8 = 0; n8 < NTOK; ++n8) {
                    const int tok = g + 8 * n8;
                    // lanes whose token column is live
                    if (MX == 1 ? g == 0 : tok < M) {
                        const uint8_t *xp = xs + tok * L.xrs + gi * 256;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const uint4 v = *reinterpret_cast<const uint4 *>(xp + xchunk(4 * t + i) * 16);
                            xb[n8][4 * i + 0] = v.x;
                            xb[n8][4 * i + 1] = v.y;
                            xb[n8][4 * i + 2] = v.z;
                            xb[n8][4 * i + 3] = v.w;
                        }
                    }
                }
                // k-step ks of the group for every 8-token tile: even steps into
                // ca, odd ones into cb (two independent accumulator chains)
                auto mma_acc = [&](float (&ca)[NTOK][4], float (&cb)[NTOK][4], const uint32_t (&a)[4],
                                   int ks) {
#pragma unroll
                    for (int n8 = 0; n8 < NTOK; ++n8) {
                        if (ks & 1)
                            mma_pure(cb[n8], a, xb[n8][2 * ks], xb[n8][2 * ks + 1]);
                        else
                            mma_pure(ca[n8], a, xb[n8][2 * ks], xb[n8][2 * ks + 1]);
                    }
                };
                // acc[k] += scale * partial, rows g (scale s0) and g + 8 (s1)
                auto scale_add = [&](int k, const float (&ca)[NTOK][4], const float (&cb)[NTOK][4],
                                     float s0, float s1) {
#pragma unroll
                    for (int n8 = 0; n8 < NTOK; ++n8) {
                        acc[k][n8][0] = fmaf(s0, ca[n8][0] + cb[n8][0], acc[k][n8][0]);
                        acc[k][n8][2] = fmaf(s1, ca[n8][2] + cb[n8][2], acc[k][n8][2]);
                        if (MX > 1) {  // token columns 2t + 1 (none live at one token)
                            acc[k][n8][1] = fmaf(s0, ca[n8][1] + cb[n8][1], acc[k][n8][1]);
                            acc[k][n8][3] = fmaf(s1, ca[n8][3] + cb[n8][3], acc[k][n8][3]);
                        }
                    }
                };
                // the residual blocks of tile k in group gi (column-blocks 2gi and
                // 2gi + 1; lanes t = 0, 1 hold the first, t = 2, 3 the second):
                // one more pass over the group's X fragment with offset-binary
                // codes q_r + 8 (8, a zero residual, where a half has no
                // block), scaled by each row's s_r
                auto block_pass = [&](int k, int gi) {
                    const int cb0 = 2 * gi;
                    const uint32_t word = bmapw[k * p.blk_words + (cb0 >> 5)];
                    const uint32_t two = (word >> (cb0 & 31)) & 3u;
                    if (two == 0) return;
                    const int lb0 = bpre[k * p.blk_words + (cb0 >> 5)] + __popc(word & ((1u << (cb0 & 31)) - 1u));
                    const int h = t >> 1;
                    const bool present = (two >> h) & 1u;
                    const int lb = lb0 + (h ? static_cast<int>(two & 1u) : 0);
                    uint4 ba = make_uint4(0x88888888u, 0x88888888u, 0x88888888u, 0x88888888u), bb = ba;
                    if (present) {
                        const uint8_t *bsrc = smem + L.bq + lb * 512 + (t & 1) * 16;
                        ba = *reinterpret_cast<const uint4 *>(bsrc + g * 32);
                        bb = *reinterpret_cast<const uint4 *>(bsrc + (g + 8) * 32);
                    }
                    const uint32_t bias = p.bias;
                    const uint32_t zz = 0x43084308u;  // bf16x2 (136, 136): u - 8 = q_r exactly
                    float ca[NTOK][4] = {}, cb[NTOK][4] = {};
                    const uint32_t wr0[4] = {ba.x, ba.y, ba.z, ba.w};
                    const uint32_t wr1[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t a_lo = wr0[ks >> 1] >> (8 * (ks & 1));
                        const uint32_t b_lo = wr1[ks >> 1] >> (8 * (ks & 1));
                        uint32_t a[4];
                        a[0] = bf16x2_sub(nib_pair(a_lo, bias), zz);
                        a[1] = bf16x2_sub(nib_pair(b_lo, bias), zz);
                        a[2] = bf16x2_sub(nib_pair(a_lo >> 4, bias), zz);
                        a[3] = bf16x2_sub(nib_pair(b_lo >> 4, bias), zz);
                        mma_acc(ca, cb, a, ks);
                    }
                    scale_add(k, ca, cb, rsfs[k * 16 + g], rsfs[k * 16 + g + 8]);
                };
                // one item: tile k of group gi, from ring slot d * NT + k
                auto item = [&](int k) {
                    const uint8_t *src = slots + k * (2 * kThreads * 16);
                    const uint4 wa = *reinterpret_cast<const uint4 *>(src);
                    const uint4 wb = *reinterpret_cast<const uint4 *>(src + kThreads * 16);
                    const uint32_t sz0 = szs[(k * 16 + g) * SZS + gi];
                    const uint32_t sz1 = szs[(k * 16 + g + 8) * SZS + gi];
                    const uint32_t zz0 = zero_pair(sz0), zz1 = zero_pair(sz1);
                    const uint32_t bias = p.bias;
                    // two accumulator chains (even and odd k-steps) per token tile
                    float ca[NTOK][4] = {}, cb[NTOK][4] = {};
                    const uint32_t wr0[4] = {wa.x, wa.y, wa.z, wa.w};
                    const uint32_t wr1[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t a_lo = wr0[ks >> 1] >> (8 * (ks & 1));
                        const uint32_t b_lo = wr1[ks >> 1] >> (8 * (ks & 1));
                        uint32_t a[4];
                        a[0] = bf16x2_sub(nib_pair(a_lo, bias), zz0);
                        a[1] = bf16x2_sub(nib_pair(b_lo, bias), zz1);
                        a[2] = bf16x2_sub(nib_pair(a_lo >> 4, bias), zz0);
                        a[3] = bf16x2_sub(nib_pair(b_lo >> 4, bias), zz1);
                        mma_acc(ca, cb, a, ks);
                    }
                    scale_add(k, ca, cb, half_bits_to_f32(sz0), half_bits_to_f32(sz1));
                    if constexpr (BLK) block_pass(k, gi);
                };
                // items in pairs after one wait, so that the two interleave;
                // each slot is refilled D groups ahead once its values are used
#pragma unroll
                for (int k = 0; k < NT; k += 2) {
                    if (k + 1 < NT) {
                        cp_async_wait_group<R - 2>();
                        item(k);
                        if (k + 2 < NT || full) item(k + 1);
                        issue(j + D, k, slots + k * (2 * kThreads * 16));
                        issue(j + D, k + 1, slots + (k + 1) * (2 * kThreads * 16));
                    } else {
                        cp_async_wait_group<R - 1>();
                        if (full) item(k);
                        issue(j + D, k, slots + k * (2 * kThreads * 16));
                    }
                }
            }
        }
    }
    // this warp's partial sums: red[k][warp][m][row]
#pragma unroll
    for (int k = 0; k < NT; ++k) {
        if (k < nt) {
            float *rw = red + ((k * kWarps + warp) * M) * 16;
#pragma unroll
            for (int n8 = 0; n8 < NTOK; ++n8) {
                const int m0 = 8 * n8 + 2 * t;
                if (m0 < M) {
                    rw[m0 * 16 + g] = acc[k][n8][0];
                    rw[m0 * 16 + g + 8] = acc[k][n8][2];
                }
                if (MX > 1 && m0 + 1 < M) {
                    rw[(m0 + 1) * 16 + g] = acc[k][n8][1];
                    rw[(m0 + 1) * 16 + g + 8] = acc[k][n8][3];
                }
            }
        }
    }

    // ------------------------------------------------ residual: one row per half-warp and tile
    if (resid) {
        const int32_t *rps = reinterpret_cast<const int32_t *>(smem + L.rp);
        const uint16_t *cols = reinterpret_cast<const uint16_t *>(smem + L.col);
        const uint8_t *vals = smem + L.val;
        const int rl = lane & 15, hw = 2 * warp + (lane >> 4);
        const float *rsf = reinterpret_cast<const float *>(smem + L.rsf);
        // q_r * x[m][c] for entry e of the staged slice
        auto entry = [&](int e, float (&r)[MX]) {
            const int cl = cols[e - col_base];
            const uint32_t byte = vals[(e >> 1) - val_base];
            const float q = static_cast<float>(static_cast<int>(((byte >> ((e & 1) * 4)) & 0xF) ^ 8) - 8);
            const uint16_t *xe = reinterpret_cast<const uint16_t *>(
                xs + (cl >> 7) * 256 + xchunk((cl & 127) >> 3) * 16 + (cl & 7) * 2);
#pragma unroll
            for (int m = 0; m < MX; ++m)
                if (MX == 1 || m < M) r[m] = fmaf(q, bf16_bits_to_f32(xe[m * (L.xrs / 2)]), r[m]);
        };
        if constexpr (MX == 1) {
            // one token: the rows of all tiles at once, so that their shared-
            // memory reads overlap; the first two entries of each lane inline,
            // longer rows in a loop
            int a[NT], b[NT];
            float r[NT][1];
#pragma unroll
            for (int k = 0; k < NT; ++k) {
                const int row = (t0 + k) * 16 + hw;
                const bool ok = (k + 1 < NT || full) && row < N;
                a[k] = ok ? rps[row - n_lo] : 0;
                b[k] = ok ? rps[row - n_lo + 1] : 0;
                r[k][0] = 0.f;
                if (a[k] + rl < b[k]) entry(a[k] + rl, r[k]);
                if (a[k] + rl + 16 < b[k]) entry(a[k] + rl + 16, r[k]);
            }
#pragma unroll
            for (int k = 0; k < NT; ++k)
#pragma unroll 1
                for (int e = a[k] + rl + 32; e < b[k]; e += 16) entry(e, r[k]);
#pragma unroll
            for (int off = 8; off > 0; off >>= 1)
#pragma unroll
                for (int k = 0; k < NT; ++k) r[k][0] += __shfl_xor_sync(0xffffffffu, r[k][0], off);
            if (rl == 0) {
#pragma unroll
                for (int k = 0; k < NT; ++k) {
                    const int row = (t0 + k) * 16 + hw;
                    if (k + 1 < NT || full) res[k * 16 + hw] = b[k] > a[k] ? rsf[row - n_lo] * r[k][0] : 0.f;
                }
            }
        } else {
#pragma unroll 1
            for (int k = 0; k < nt; ++k) {
                const int row = (t0 + k) * 16 + hw;
                int a = 0, b = 0;
                if (row < N) {
                    a = rps[row - n_lo];
                    b = rps[row - n_lo + 1];
                }
                float r[MX];
#pragma unroll
                for (int m = 0; m < MX; ++m) r[m] = 0.f;
#pragma unroll 1
                for (int e = a + rl; e < b; e += 16) entry(e, r);
#pragma unroll
                for (int off = 8; off > 0; off >>= 1)
#pragma unroll
                    for (int m = 0; m < MX; ++m) r[m] += __shfl_xor_sync(0xffffffffu, r[m], off);
                if (rl < M) {
                    float v = r[0];
#pragma unroll
                    for (int m = 1; m < MX; ++m)
                        if (m == rl) v = r[m];
                    res[(k * M + rl) * 16 + hw] = b > a ? rsf[row - n_lo] * v : 0.f;
                }
            }
        }
    }
    __syncthreads();

    // ------------------------------------------------ reduction-add and store
    for (int o = threadIdx.x; o < nt * M * 16; o += kThreads) {
        const int k = o / (M * 16), rem = o - k * M * 16, m = rem >> 4, rr = rem & 15;
        const int n = (t0 + k) * 16 + rr;
        float y = resid ? res[(k * M + m) * 16 + rr] : 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) y += red[((k * kWarps + w) * M + m) * 16 + rr];
        if (n < N) {
            if (p.Yf)
                p.Yf[static_cast<size_t>(m) * N + n] = y;
            else
                p.Y[static_cast<size_t>(m) * N + n] = __float2bfloat16_rn(y);
        }
    }
    cp_async_wait_all();
}

template <int MX, bool BLK>
void *kernel_for(int nt) {
    if constexpr (MX > 8) {  // 16 tokens: X takes the shared memory of more tiles
        switch (nt) {
            case 1: return reinterpret_cast<void *>(decode_stream_kernel<MX, 1, BLK>);
            case 2: return reinterpret_cast<void *>(decode_stream_kernel<MX, 2, BLK>);
            case 3: return reinterpret_cast<void *>(decode_stream_kernel<MX, 3, BLK>);
            case 4: return reinterpret_cast<void *>(decode_stream_kernel<MX, 4, BLK>);
            default: return nullptr;
        }
    } else {
        switch (nt) {
            case 1: return reinterpret_cast<void *>(decode_stream_kernel<MX, 1, BLK>);
            case 2: return reinterpret_cast<void *>(decode_stream_kernel<MX, 2, BLK>);
            case 3: return reinterpret_cast<void *>(decode_stream_kernel<MX, 3, BLK>);
            case 4: return reinterpret_cast<void *>(decode_stream_kernel<MX, 4, BLK>);
            case 5: return reinterpret_cast<void *>(decode_stream_kernel<MX, 5, BLK>);
            case 6: return reinterpret_cast<void *>(decode_stream_kernel<MX, 6, BLK>);
            case 7: return reinterpret_cast<void *>(decode_stream_kernel<MX, 7, BLK>);
            default: return reinterpret_cast<void *>(decode_stream_kernel<MX, 8, BLK>);
        }
    }
}

}  // namespace

mq_status launch_decode_stream(const mq_weight *w, const void *X, int M, void *Y,
                               cudaStream_t stream, float *partial, const L2Prefetch &pf) {
    const DeviceWeight &d = weight_device(w);
    if (M < 1 || M > 16) return MQ_ERR_UNSUPPORTED;
    const int64_t ntile = (d.N + 15) / 16;
    // one CTA per SM with NT = ceil(tiles / SMs) tiles each, or more CTAs of
    // kTMax tiles for layers taller than kTMax tiles per SM
    int64_t grid = std::min<int64_t>(ntile, sm_count());
    if ((ntile + grid - 1) / grid > kTMax) grid = (ntile + kTMax - 1) / kTMax;
    const int nt = static_cast<int>((ntile + grid - 1) / grid);
    const bool with_residual = partial == nullptr && d.nnz > 0;
    // a block-allocated residual runs from its block tiles, a row residual
    // from the CSR; a CTA's share too long for its shared-memory budget: the
    // register kernel takes the call
    const bool use_blocks = with_residual && d.blk_q != nullptr;
    const int64_t bspan = use_blocks ? max_span_blocks(w, ntile, static_cast<int>(grid)) : 0;
    if (bspan * 512 > kBlockBudget) return MQ_ERR_UNSUPPORTED;
    const int64_t span = (with_residual && !use_blocks) ? max_span_nnz(w, ntile, static_cast<int>(grid)) : 0;
    if (span * 5 / 2 + 96 > kCsrBudget) return MQ_ERR_UNSUPPORTED;
    StreamParams p;
    p.qweight = d.qweight;
    p.sz = d.sz;
    p.X = static_cast<const __nv_bfloat16 *>(X);
    p.Y = static_cast<__nv_bfloat16 *>(Y);
    p.Yf = partial;
    p.row_ptr = d.row_ptr;
    p.col = d.col;
    p.val = d.val;
    p.rscale = d.rscale;
    p.M = M;
    p.N = static_cast<int>(d.N);
    p.K = static_cast<int>(d.K);
    p.G = static_cast<int>(d.G);
    p.Gp = static_cast<int>(d.Gp);
    p.ntile = static_cast<int>(ntile);
    p.csr_cap = (with_residual && !use_blocks) ? static_cast<int>(std::max<int64_t>(span, 1)) : 0;
    p.blk_ptr = d.blk_ptr;
    p.blk_q = d.blk_q;
    p.blk_map = d.blk_map;
    p.blk_words = static_cast<int>(d.blk_words);
    p.blk_cap = use_blocks ? static_cast<int>(std::max<int64_t>(bspan, 1)) : 0;
    p.bias = 0x43004300u;
    p.pf = pf;
    const StreamLayout L(M, p.K, p.Gp, p.csr_cap, nt, p.blk_cap, p.blk_words);
    if (L.total > kMaxSmem) return MQ_ERR_UNSUPPORTED;
    // one CTA per SM (X takes the shared memory of two) and more CTAs than
    // SMs: a second wave; the tall-layer kernel, which reads X from L2, or
    // the register kernels take the call
    if (L.total > kTwoPerSm && grid > sm_count()) return MQ_ERR_UNSUPPORTED;
    const int mx = M == 1 ? 0 : M <= 8 ? 1 : 2;
    void *kern = use_blocks ? (mx == 0 ? kernel_for<1, true>(nt) : mx == 1 ? kernel_for<8, true>(nt)
                                                                         : kernel_for<16, true>(nt))
                            : (mx == 0 ? kernel_for<1, false>(nt) : mx == 1 ? kernel_for<8, false>(nt)
                                                                           : kernel_for<16, false>(nt));
    if (!kern) return MQ_ERR_UNSUPPORTED;
    static bool configured[64][2][3][kTMax + 1] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(MQ_ERR_CUDA, "cudaGetDevice failed");
    if (dev >= 0 && dev < 64 && !configured[dev][use_blocks][mx][nt]) {
        // the largest shared-memory carveout for every decode kernel, so that
        // consecutive launches of different layers can share an SM without
        // waiting for it to drain and be reconfigured
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem) !=
                cudaSuccess ||
            cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared) != cudaSuccess)
            return fail(MQ_ERR_CUDA, "cudaFuncSetAttribute failed for the streaming decode kernel");
        configured[dev][use_blocks][mx][nt] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(L.total);
    cfg.stream = stream;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    void *args[] = {&p};
    const cudaError_t e = cudaLaunchKernelExC(&cfg, kern, args);
    if (e != cudaSuccess)
        return fail(MQ_ERR_CUDA, std::string("streaming decode launch: ") + cudaGetErrorString(e));
    return MQ_OK;
}

}  // namespace mq
