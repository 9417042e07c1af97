// Tall-layer decode kernel: Y[M][N] = X[M][K] * W_hat^T for 2 <= M <= 16 on
// layers tall enough to give every CTA two or more 16-row tiles at two CTAs
// per SM (a 70B MLP projection, 28672 x 8192: six or seven), one fused pass.
//
// MosaicQuant "Methodology" 3. (ZipperEngine): the sparse residual is
// computed inside the dense 4-bit GEMM pass over the same activations, and
// the dense and sparse parts meet in one reduction-add.
//
// The streaming decode kernel (decode_stream.cu) stages X in shared memory.
// At 16 tokens and K = 8192 X alone is 256 KB, more than an SM holds, and
// even at 2-8 tokens it leaves one CTA per SM for grids of two waves. Here
// nothing of X is staged:
//   * Persistent grid of two CTAs per SM (NT = 2..8 contiguous 16-row tiles
//     each); warp w takes groups w, w + 8, ... of every tile of its CTA, as
//     in the streaming kernel, so a group's X fragment is used by one warp
//     only. That warp loads it straight from L2 (16-byte loads of 64
//     contiguous bytes per lane and token) at the start of the group and
//     keeps it in registers across the tiles. At 9-16 tokens two sets of four
//     warps split the CTA's tiles and each warp takes every fourth group:
//     eight accumulator registers per tile and 8-token column tile would not
//     fit beside the 32-register X fragment otherwise.
//   * The packed codes stream through a per-thread cp.async ring of R items
//     (R = 4 or 8, an item being one tile of one group), refilled as soon as
//     an item is consumed; the slot of item (group j, tile k) is
//     (j * NTW + k) mod R (NTW: the warp's tiles), found at run time once per
//     group, and the item refilled into it, R items later, has a tile index
//     known at compile time. Items run in pairs after one wait. No barrier
//     between threads.
//   * Dense part, per item: exact bf16 codes q - z (a mask into the mantissa
//     of 128.0, then a subtraction of 128 + z), mma.sync m16n8k16 in fp32 for
//     one or two 8-token column tiles, the group partial scaled by s in fp32.
//   * Residual, per item, on the tensor cores: the host groups the residual
//     per (tile, group) (DeviceWeight::tl_ptr), each entry carrying its byte
//     in the A fragments; the CTA stages its run's lists once. The warp's
//     lanes scatter an item's entries as exact bf16 codes into eight zeroed
//     512-byte fragment tiles, and each k-step that received an entry costs
//     one more mma.sync per token tile on the X fragment already in
//     registers; the sums are scaled by the row's s_r and added in. The
//     residual runs after the group's dense items, in a loop over the tiles
//     that is not unrolled (the unrolled form outgrew the instruction cache).
//   * Reduction-add: each warp writes its tiles' sums into its group lane's
//     slot in shared memory; the slots are summed in a fixed order and the
//     result is stored once as bf16.
// The k order inside a group is the packed codes' nibble interleave: k-step s
// of thread (g, t) covers columns 32t + 4s + {0,1} and 32t + 4s + {2,3}, so
// thread t's X fragment of a group is columns 32t .. 32t + 31 of its tokens.
//
// Launches use programmatic dependent launch: the ring, the scale/zero words
// and the residual lists (which no earlier kernel writes) are requested
// before griddepcontrol.wait; X is read and Y written only after it.

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "kernels.h"

namespace mq {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kTMin = 2;                   // fewest tiles per CTA (X is read once per CTA and group)
constexpr int kTMax = 8;                   // most tiles per CTA (one accumulator set each)
constexpr int kSlotBytes = 2 * kThreads * 16;  // one item: 16 bytes of rows g and g + 8 per thread
constexpr int kFragBytes = 8 * 512;        // per warp: the A fragments of a group's eight k-steps
constexpr int kTwoPerSm = 113 * 1024;      // shared memory of each of two CTAs per SM
constexpr int kEntBudget = 24 * 1024;      // shared memory for a CTA's residual entries

struct TallParams {
    const uint32_t *qweight;  // [N][K/8]
    const uint32_t *sz;       // [N][Gp]
    const __nv_bfloat16 *X;   // [M][K]
    __nv_bfloat16 *Y;         // [M][N]
    float *Yf;                // fp32 dense-only output (unfused path) or null
    const int32_t *tl_ptr;    // residual lists per (16-row tile, group)
    const uint16_t *tl_ent;
    const uint16_t *rscale;
    int M, N, K, G, Gp;
    int ntile;    // ceil(N / 16)
    int ent_cap;  // most residual entries of a CTA's run; 0: no residual
    // 0x43004300 (bf16x2 128.0, 128.0), passed at run time so that it sits in
    // a register and each code pair costs one LOP3 (mask and OR)
    uint32_t bias;
    L2Prefetch pf;  // another weight, brought into L2 meanwhile
};

// Warps sharing one set of tiles (each taking every GL-th group): all eight,
// or at 9-16 tokens two sets of four, each over half of the CTA's tiles, so
// that a warp's accumulators (8 registers per tile at 16 tokens) fit beside
// its X fragment.
__host__ __device__ constexpr int group_lanes(int mx) { return mx > 8 ? kWarps / 2 : kWarps; }

// Scale/zero rows in shared memory: with Gp a multiple of 32, Gp words per
// row and 16-byte chunk q of row r stored at chunk q ^ (r % 8), so that the
// eight rows a warp reads at once (g = 0..7) fall on distinct banks; else the
// rows are padded to an odd multiple of four words.
__host__ __device__ inline bool sz_swizzled(int Gp) { return Gp % 32 == 0; }
__host__ __device__ inline int tall_sz_stride(int Gp) { return sz_swizzled(Gp) ? Gp : sz_stride(Gp); }

// Shared-memory layout (bytes), identical on host and device. After the
// dense pass the reduction buffer [GL][NT][M][16] fp32 reuses it from 0.
struct TallLayout {
    int ring, szs, toff, tent, frag, rsf, total;
    __host__ __device__ TallLayout(int M, int G, int Gp, int nt, int R, int ent_cap) {
        const bool resid = ent_cap > 0;
        ring = 0;                                               // [R][2][kThreads][16 B]
        szs = ring + R * kSlotBytes;                            // [NT * 16][tall_sz_stride] words
        toff = szs + nt * 16 * tall_sz_stride(Gp) * 4;          // [NT * G + 1] u16
        tent = toff + (resid ? ((nt * G + 1) * 2 + 15) / 16 * 16 : 0);
        frag = tent + (resid ? ((ent_cap + 8) * 2 + 15) / 16 * 16 : 0);  // from a 16-byte aligned start
        rsf = frag + (resid ? kWarps * kFragBytes : 0);          // [kWarps][8][512 B]
        total = rsf + (resid ? nt * 16 * 4 : 0);                 // [NT * 16] fp32 s_r
        const int red = group_lanes(M) * nt * M * 16 * 4;
        if (total < red) total = red;
    }
};

template <int MX, int NT, int R>
__global__ void __launch_bounds__(kThreads, 2) decode_tall_kernel(const __grid_constant__ TallParams p) {
    static_assert((R & (R - 1)) == 0 && R >= 4, "the ring holds a power of two of at least four items");
    constexpr int NTOK = MX > 8 ? 2 : 1;       // 8-token MMA column tiles
    constexpr int GL = group_lanes(MX);        // warps per tile set
    constexpr int NTW = (NT * GL + kWarps - 1) / kWarps;  // tiles per warp
    extern __shared__ __align__(16) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int M = p.M, N = p.N, K = p.K, G = p.G;
    const TallLayout L(M, G, p.Gp, NT, R, p.ent_cap);
    const int SZS = tall_sz_stride(p.Gp);
    const bool swz = sz_swizzled(p.Gp);
    const int t0 = static_cast<int>(static_cast<long long>(p.ntile) * blockIdx.x / gridDim.x);
    const int t1 = static_cast<int>(static_cast<long long>(p.ntile) * (blockIdx.x + 1) / gridDim.x);
    const int nt = t1 - t0;  // NT or NT - 1
    // this warp's group lane, first tile and tile count: with two tile sets,
    // the CTA's nt tiles split ceil(nt / 2) + floor(nt / 2)
    const int gl = warp % GL, kt0 = GL == kWarps ? 0 : (warp / GL) * ((nt + 1) / 2);
    const int nv = GL == kWarps ? nt : (warp < GL ? (nt + 1) / 2 : nt / 2);
    const int gpw = gl < G ? (G - gl + GL - 1) / GL : 0;  // its groups
    const bool resid = p.ent_cap > 0;
    pdl_launch_dependents();

    // ------------------------------------------------ the run's scale/zero words and residual lists
    const int n_lo = t0 * 16, n_hi = min(t1 * 16, N);
    {
        const int q4 = p.Gp / 4;  // 16-byte chunks per scale/zero row
        for (int i = threadIdx.x; i < (n_hi - n_lo) * q4; i += kThreads) {
            const int r = i / q4, q = i - r * q4;
            cp_async16(smem + L.szs + (r * SZS + 4 * (swz ? q ^ (r & 7) : q)) * 4,
                       p.sz + static_cast<size_t>(n_lo + r) * p.Gp + 4 * q);
        }
    }
    if (resid) {
        const int k_lo = t0 * G, k_hi = k_lo + nt * G;
        const int e_lo = p.tl_ptr[k_lo], e_hi = p.tl_ptr[k_hi];
        const int e_base = e_lo & ~7;
        const int n16 = ((e_hi - e_base) * 2 + 15) / 16;
        for (int i = threadIdx.x; i < n16; i += kThreads)
            cp_async16(smem + L.tent + 16 * i, p.tl_ent + e_base + 8 * i);
        // list starts relative to the staged entries (they fit in 16 bits)
        uint16_t *toff = reinterpret_cast<uint16_t *>(smem + L.toff);
        for (int i = threadIdx.x; i <= k_hi - k_lo; i += kThreads)
            toff[i] = static_cast<uint16_t>(p.tl_ptr[k_lo + i] - e_base);
        float *rsf = reinterpret_cast<float *>(smem + L.rsf);
        for (int i = threadIdx.x; i < n_hi - n_lo; i += kThreads) rsf[i] = half_bits_to_f32(p.rscale[n_lo + i]);
        // the fragment tiles start zeroed; each k-step clears what it used
        for (int i = threadIdx.x; i < kWarps * kFragBytes / 16; i += kThreads)
            sts128(smem + L.frag + 16 * i, make_uint4(0u, 0u, 0u, 0u));
    }
    cp_async_commit();

    // ------------------------------------------------ the weight stream
    // This thread's rows g and g + 8 of its tile k are row0 + 16k and row0 +
    // 16k + 8 (clamped to the last row), and its 16-byte column in a group.
    const int row0 = (t0 + kt0) * 16 + g;
    const uint32_t wrow = static_cast<uint32_t>(K / 8);
    const uint32_t *qbase = p.qweight + gl * 16 + 4 * t;
    uint8_t *const ring = smem + L.ring + threadIdx.x * 16;
    // item (group j of this warp, tile k) into the slot at dst (a copy that
    // is not live writes zeros: a source size of 0; the address stays in
    // bounds)
    auto issue = [&](int j, int k, uint8_t *dst) {
        // past the warp's last group the copy repeats that group (clamped
        // below: an L2 hit, never consumed)
        const bool live = gpw > 0 && k < nv;
        const uint32_t *src = qbase + min(j, max(gpw - 1, 0)) * (GL * 16);
        const uint32_t o0 = static_cast<uint32_t>(min(row0 + 16 * k, N - 1)) * wrow;
        const uint32_t o1 = static_cast<uint32_t>(min(row0 + 16 * k + 8, N - 1)) * wrow;
        cp_async16_if(dst, src + o0, live);
        cp_async16_if(dst + kThreads * 16, src + o1, live);
        cp_async_commit();
    };
#pragma unroll
    for (int i = 0; i < R; ++i) issue(i / NTW, i % NTW, ring + i * kSlotBytes);
    if (threadIdx.x == 0) l2_prefetch_share(p.pf, blockIdx.x, gridDim.x);
    pdl_wait();  // X may come from the previous kernel; Y may still be read by it
    cp_async_wait_group<R>();  // the staged words and lists (committed before the ring)
    __syncthreads();

    const uint32_t *szw = reinterpret_cast<const uint32_t *>(smem + L.szs) + (kt0 * 16 + g) * SZS;
    const uint16_t *tow = reinterpret_cast<const uint16_t *>(smem + L.toff) + kt0 * G;
    const uint16_t *tent = reinterpret_cast<const uint16_t *>(smem + L.tent);
    const float *rsw = reinterpret_cast<const float *>(smem + L.rsf) + kt0 * 16 + g;
    uint8_t *const frag = smem + L.frag + warp * kFragBytes;

    // ------------------------------------------------ dense pass with the residual
    float acc[NTW][NTOK][4];
#pragma unroll
    for (int k = 0; k < NTW; ++k)
#pragma unroll
        for (int n8 = 0; n8 < NTOK; ++n8)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[k][n8][i] = 0.f;
    uint32_t xb[NTOK][16];
#pragma unroll
    for (int n8 = 0; n8 < NTOK; ++n8)
#pragma unroll
        for (int i = 0; i < 16; ++i) xb[n8][i] = 0u;
    int base = 0;  // ring slot of item (j, 0): (j * NTW) mod R
#pragma unroll 1
    for (int j = 0; j < gpw; ++j, base = (base + NTW) & (R - 1)) {
        const int gi = gl + GL * j;
        // the group's word in this thread's scale/zero rows (g and g + 8 of
        // each tile: both r % 8 = g under the swizzle)
        const int gis = swz ? ((((gi >> 2) ^ g) << 2) | (gi & 3)) : gi;
        // X fragment of the group for tokens g and g + 8: columns 32t .. 32t + 31
#pragma unroll
        for (int n8 = 0; n8 < NTOK; ++n8) {
            const int tok = g + 8 * n8;
            if (tok < M) {
                const uint32_t *xp = reinterpret_cast<const uint32_t *>(
                    p.X + static_cast<size_t>(tok) * K + gi * 128 + 32 * t);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint4 v = ldg_stream(xp + 4 * i);
                    xb[n8][4 * i + 0] = v.x;
                    xb[n8][4 * i + 1] = v.y;
                    xb[n8][4 * i + 2] = v.z;
                    xb[n8][4 * i + 3] = v.w;
                }
            }
        }
        auto slot = [&](int k) { return ring + ((base + k) & (R - 1)) * kSlotBytes; };
        // acc[k] += s * c, rows g (scale s0) and g + 8 (s1)
        auto scale_add = [&](int k, const float (&c)[NTOK][4], float s0, float s1) {
#pragma unroll
            for (int n8 = 0; n8 < NTOK; ++n8) {
                acc[k][n8][0] = fmaf(s0, c[n8][0], acc[k][n8][0]);
                acc[k][n8][1] = fmaf(s0, c[n8][1], acc[k][n8][1]);
                acc[k][n8][2] = fmaf(s1, c[n8][2], acc[k][n8][2]);
                acc[k][n8][3] = fmaf(s1, c[n8][3], acc[k][n8][3]);
            }
        };
        // the residual code sums rc of tile k (a run-time index) in group gi:
        // scatter the item's entries into the fragment tiles of the group's
        // eight k-steps (each entry carries its byte there), then one MMA per
        // token tile for each k-step that received one (two accumulator chains
        // at one token tile), the lanes clearing their fragment after reading
        // it; false when the item has no entries
        auto residual = [&](int k, float (&rc)[NTOK][4]) {
            const uint16_t *to = tow + k * G + gi;
            const int e0 = to[0], e1 = to[1];
            if (e1 == e0) return false;  // the same for every lane
            uint32_t used = 0;  // k-steps that received an entry
            for (int e = e0 + lane; e < e1; e += 32) {
                const uint32_t v = tent[e];
                const uint32_t pos = v & 0xFFFu;
                const int q = static_cast<int>((v >> 12) ^ 8u) - 8;
                sts_u16(frag + pos, __float_as_uint(static_cast<float>(q)) >> 16);
                used |= 1u << (pos >> 9);
            }
            used = __reduce_or_sync(0xffffffffu, used);
            __syncwarp();
            float rd[NTOK][4];
#pragma unroll
            for (int n8 = 0; n8 < NTOK; ++n8)
#pragma unroll
                for (int i = 0; i < 4; ++i) rd[n8][i] = 0.f;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                if ((used >> ks) & 1u) {
                    const uint4 f = lds128(frag + ks * 512 + 16 * lane);
                    sts128(frag + ks * 512 + 16 * lane, make_uint4(0u, 0u, 0u, 0u));
                    const uint32_t fa[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
                    for (int n8 = 0; n8 < NTOK; ++n8) {
                        if (NTOK == 1 && (ks & 1))
                            mma_pure(rd[n8], fa, xb[n8][2 * ks], xb[n8][2 * ks + 1]);
                        else
                            mma_pure(rc[n8], fa, xb[n8][2 * ks], xb[n8][2 * ks + 1]);
                    }
                }
            }
            __syncwarp();
            if (NTOK == 1) {
#pragma unroll
                for (int i = 0; i < 4; ++i) rc[0][i] += rd[0][i];
            }
            return true;
        };
        // the dense part of one item: tile k of group gi
        auto item = [&](int k) {
            const uint8_t *src = slot(k);
            const uint4 wa = *reinterpret_cast<const uint4 *>(src);
            const uint4 wb = *reinterpret_cast<const uint4 *>(src + kThreads * 16);
            const uint32_t sz0 = szw[k * 16 * SZS + gis];
            const uint32_t sz1 = szw[(k * 16 + 8) * SZS + gis];
            const uint32_t zz0 = zero_pair(sz0), zz1 = zero_pair(sz1);
            const uint32_t bias = p.bias;
            // one accumulator chain per token tile
            float c[NTOK][4];
#pragma unroll
            for (int n8 = 0; n8 < NTOK; ++n8)
#pragma unroll
                for (int i = 0; i < 4; ++i) c[n8][i] = 0.f;
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
#pragma unroll
                for (int n8 = 0; n8 < NTOK; ++n8) mma_pure(c[n8], a, xb[n8][2 * ks], xb[n8][2 * ks + 1]);
            }
            scale_add(k, c, half_bits_to_f32(sz0), half_bits_to_f32(sz1));
        };
        // items in pairs after one wait, so that the two interleave; each slot
        // is refilled with the item R later once its values are used. A CTA
        // holds NT or NT - 1 tiles, so a warp holds at least NTW - 2 of its
        // NTW: only the last two are tested (at run time).
        auto present = [&](int k) { return k < NTW - 2 || k < nv; };
#pragma unroll
        for (int k = 0; k < NTW; k += 2) {
            if (k + 1 < NTW) {
                cp_async_wait_group<R - 2>();
                if (present(k)) item(k);
                if (present(k + 1)) item(k + 1);
                issue(j + (k + R) / NTW, (k + R) % NTW, slot(k));
                issue(j + (k + 1 + R) / NTW, (k + 1 + R) % NTW, slot(k + 1));
            } else {
                cp_async_wait_group<R - 1>();
                if (present(k)) item(k);
                issue(j + (k + R) / NTW, (k + R) % NTW, slot(k));
            }
        }
        // the group's residual, tile by tile in a loop that is not unrolled
        // (its code once, not once per tile: the unrolled form outgrew the
        // instruction cache), each tile's sums scaled by s_r into its
        // accumulators through a branch on the tile index
        if (resid) {
#pragma unroll 1
            for (int k = 0; k < nv; ++k) {
                float rc[NTOK][4];
#pragma unroll
                for (int n8 = 0; n8 < NTOK; ++n8)
#pragma unroll
                    for (int i = 0; i < 4; ++i) rc[n8][i] = 0.f;
                if (residual(k, rc)) {
                    const float r0 = rsw[k * 16], r1 = rsw[k * 16 + 8];
#pragma unroll
                    for (int kk = 0; kk < NTW; ++kk)
                        if (kk == k) scale_add(kk, rc, r0, r1);
                }
            }
        }
    }

    // ------------------------------------------------ reduction-add and store
    cp_async_wait_all();  // the zero fills past the end land before the ring is reused
    __syncthreads();
    // slot gl holds the partial sums of this warp's tiles (no two warps share
    // a tile and a slot); the slots are summed in a fixed order
    float *red = reinterpret_cast<float *>(smem);  // [GL][NT][M][16]
    const int slot_floats = NT * M * 16;
    {
        float *rw = red + gl * slot_floats;
#pragma unroll
        for (int k = 0; k < NTW; ++k) {
            if (k < nv) {
#pragma unroll
                for (int n8 = 0; n8 < NTOK; ++n8) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int m = 8 * n8 + 2 * t + (i & 1), row = g + ((i >> 1) << 3);
                        if (m < M) rw[((kt0 + k) * M + m) * 16 + row] = acc[k][n8][i];
                    }
                }
            }
        }
    }
    __syncthreads();
    for (int o = threadIdx.x; o < nt * M * 16; o += kThreads) {
        const int k = o / (M * 16), rem = o - k * M * 16, m = rem >> 4, rr = rem & 15;
        const int n = (t0 + k) * 16 + rr;
        float y = red[o];
#pragma unroll
        for (int s2 = 1; s2 < GL; ++s2) y += red[s2 * slot_floats + o];

        if (n < N) {
            if (p.Yf)
                p.Yf[static_cast<size_t>(m) * N + n] = y;
            else
                p.Y[static_cast<size_t>(m) * N + n] = __float2bfloat16_rn(y);
        }
    }
}

template <int MX, int R>
void *kernel_for(int nt) {
    switch (nt) {
        case 2: return reinterpret_cast<void *>(decode_tall_kernel<MX, 2, R>);
        case 3: return reinterpret_cast<void *>(decode_tall_kernel<MX, 3, R>);
        case 4: return reinterpret_cast<void *>(decode_tall_kernel<MX, 4, R>);
        case 5: return reinterpret_cast<void *>(decode_tall_kernel<MX, 5, R>);
        case 6: return reinterpret_cast<void *>(decode_tall_kernel<MX, 6, R>);
        case 7: return reinterpret_cast<void *>(decode_tall_kernel<MX, 7, R>);
        case 8: return reinterpret_cast<void *>(decode_tall_kernel<MX, 8, R>);
        default: return nullptr;
    }
}

}  // namespace

mq_status launch_decode_tall(const mq_weight *w, const void *X, int M, void *Y, cudaStream_t stream,
                             float *partial, const L2Prefetch &pf) {
    const DeviceWeight &d = weight_device(w);
    if (M < 2 || M > 16 || d.K % 128) return MQ_ERR_UNSUPPORTED;
    const int64_t ntile = (d.N + 15) / 16;
    // two CTAs per SM with NT = ceil(tiles / (2 SMs)) tiles each, at least
    // kTMin (X is read once per CTA and group: fewer tiles make that read
    // outweigh the codes), at most kTMax (then more CTAs than two per SM)
    const int64_t slots = 2 * static_cast<int64_t>(sm_count());
    if (ntile < kTMin * slots) return MQ_ERR_UNSUPPORTED;
    int64_t grid = slots;
    if ((ntile + grid - 1) / grid > kTMax) grid = (ntile + kTMax - 1) / kTMax;
    const int nt = static_cast<int>((ntile + grid - 1) / grid);
    const bool with_residual = partial == nullptr && d.nnz > 0;
    if (with_residual && (!d.tl_ptr || !d.tl_ent)) return MQ_ERR_UNSUPPORTED;
    // a CTA's residual lists must fit their shared-memory budget
    const int64_t span = with_residual ? max_span_nnz(w, ntile, static_cast<int>(grid)) : 0;
    if (span * 2 + 16 > kEntBudget) return MQ_ERR_UNSUPPORTED;
    TallParams p;
    p.qweight = d.qweight;
    p.sz = d.sz;
    p.X = static_cast<const __nv_bfloat16 *>(X);
    p.Y = static_cast<__nv_bfloat16 *>(Y);
    p.Yf = partial;
    p.tl_ptr = d.tl_ptr;
    p.tl_ent = d.tl_ent;
    p.rscale = d.rscale;
    p.M = M;
    p.N = static_cast<int>(d.N);
    p.K = static_cast<int>(d.K);
    p.G = static_cast<int>(d.G);
    p.Gp = static_cast<int>(d.Gp);
    p.ntile = static_cast<int>(ntile);
    p.ent_cap = with_residual ? static_cast<int>(std::max<int64_t>(span, 1)) : 0;
    p.bias = kBiasBf16;
    p.pf = pf;
    // the deeper ring when both it and the rest fit two CTAs per SM
    int R = 8;
    if (TallLayout(M, p.G, p.Gp, nt, R, p.ent_cap).total > kTwoPerSm) R = 4;
    const TallLayout L(M, p.G, p.Gp, nt, R, p.ent_cap);
    if (L.total > kTwoPerSm) return MQ_ERR_UNSUPPORTED;
    const int mx = M <= 8 ? 0 : 1;
    void *kern = R == 8 ? (mx ? kernel_for<16, 8>(nt) : kernel_for<8, 8>(nt))
                        : (mx ? kernel_for<16, 4>(nt) : kernel_for<8, 4>(nt));
    if (!kern) return MQ_ERR_UNSUPPORTED;
    static bool configured[64][2][2][kTMax + 1] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(MQ_ERR_CUDA, "cudaGetDevice failed");
    const int ri = R == 8 ? 1 : 0;
    if (dev >= 0 && dev < 64 && !configured[dev][ri][mx][nt]) {
        // the largest shared-memory carveout, as for every decode kernel, so
        // that consecutive launches of different layers can share an SM
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kTwoPerSm) !=
                cudaSuccess ||
            cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared) != cudaSuccess)
            return fail(MQ_ERR_CUDA, "cudaFuncSetAttribute failed for the tall-layer decode kernel");
        configured[dev][ri][mx][nt] = true;
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
        return fail(MQ_ERR_CUDA, std::string("tall-layer decode launch: ") + cudaGetErrorString(e));
    return MQ_OK;
}

}  // namespace mq
