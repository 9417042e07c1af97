// Decode kernel: Y[M][N] = X[M][K] * W_hat^T for M <= 16, one fused pass.
//
// MosaicQuant "Methodology" 3. (ZipperEngine): the sparse residual is
// computed inside the dense 4-bit GEMM kernel, over the same staged
// activations, and the dense and sparse parts meet in one reduction-add; no
// second kernel reloads X or merges partial outputs.
//
// For M <= 16 the layer is bound by streaming the packed weight from HBM, so
// the kernel is built around keeping HBM busy from its first instruction:
//   * A CTA owns BN = 16*RT output rows and the K range of its cluster rank
//     (CS CTAs of a cluster split K when X would not fit shared memory).
//     Warp (rt, s) owns rows [16rt, 16rt+16) and every S-th group of 128
//     columns, so the S warps of a row tile read adjacent 64-byte segments.
//   * Packed codes and scale/zero words go straight from HBM into registers
//     (16-byte streaming loads, batches of BG groups, double-buffered); the
//     first batch is in flight before anything else happens.
//   * Meanwhile all threads stage X (the CTA's K range) and, when it is
//     small enough, the tile's CSR slice into shared memory with cp.async.
//   * Sparse branch, a warp-cooperative CSR walk: a team of THREADS/BN
//     consecutive lanes owns one row. Its lanes split the tokens into groups
//     of four and stride over the row's entries in this CTA's K range (a
//     binary search on the ascending columns finds that range when K is
//     split); the partial sums meet in a shuffle reduction and s_r * sum
//     q_r * x is left in shared memory. Long rows (a block-allocated
//     residual) are spread over the team instead of one thread.
//   * Dense branch: each group's nibbles become exact bf16 codes (q - z) in
//     registers (OR into the mantissa of 128.0, subtract 128 + z), 8
//     mma.sync m16n8k16 accumulate the exact products in fp32, and s times
//     the group's partial is added to the running fp32 sum.
//   * Reduction-add: split-K partials of the S warps, the residual and (for
//     CS > 1) the other ranks' partials read over DSMEM are summed in fp32
//     and stored once as bf16.
// The k order inside a group is permuted so that each thread's 16-byte load
// of packed codes feeds its own mma fragments with no shuffles: k-step s'
// (0..7) of thread (g, t) covers columns 32t + 4s' + {0,1} (fragment k 2t,
// 2t+1) and 32t + 4s' + {2,3} (fragment k 2t+8, 2t+9); X is read with the
// same permutation, so the sum over k is unchanged.
//
// Launches use programmatic dependent launch: the weight stream (which no
// earlier kernel writes) starts at once; griddepcontrol.wait precedes the
// first read of X and the first write of Y.

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "kernels.h"

namespace mq {
namespace {

struct DecodeParams {
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
    uint32_t bias;  // kBiasBf16, or kBiasI8 for int8 codes (held in a register)
    int csr_cap;  // residual entries staged in shared memory (0: read from global)
    int with_residual;
    L2Prefetch pf;  // the next layer's weight, brought into L2 meanwhile
};

template <int MX, int RT, int S, int BG, int CS>
struct Cfg {
    static constexpr int NT = (MX + 7) / 8;  // n8 tiles of tokens
    static constexpr int BN = 16 * RT;       // rows per CTA
    static constexpr int WARPS = RT * S;
    static constexpr int THREADS = WARPS * 32;
    // sparse branch: a team of TEAM lanes per row, TG token groups of TPG
    // tokens, E lanes per group striding over the row's entries
    static constexpr int TEAM = THREADS / BN;
    static constexpr int TPG = MX < 4 ? MX : 4;
    static constexpr int TG = MX / TPG;
    static constexpr int E = TEAM / TG;
    static_assert(THREADS % BN == 0 && TEAM <= 32 && 32 % TEAM == 0, "row teams inside a warp");
    static_assert(MX % TPG == 0 && TEAM % TG == 0 && (E & (E - 1)) == 0, "team split");
    static_assert(CS == 1 || CS == 2 || CS == 4 || CS == 8, "cluster size");
};

// Shared-memory layout (bytes), identical on host and device.
struct Layout {
    int xrs, kc, x, red, res, col, val, total;
    __host__ __device__ Layout(int M, int K, int G, int CS, int S, int MX, int BN, int csr_cap) {
        const int gpc = (G + CS - 1) / CS;
        kc = gpc * 128;                // columns of one rank's K range
        xrs = kc * 2 + 16;             // X row stride
        x = 0;
        red = (M * xrs + 15) / 16 * 16;
        res = red + S * MX * BN * 4;
        col = res + BN * MX * 4;
        val = col + (csr_cap * 2 + 32 + 15) / 16 * 16;
        total = val + (csr_cap / 2 + 32 + 15) / 16 * 16;
    }
};

template <int BG>
struct Batch {
    uint4 w[BG][2];
    uint32_t sz[BG][2];
};

template <int MX, int RT, int S, int BG, int CS>
__global__ void __launch_bounds__(Cfg<MX, RT, S, BG, CS>::THREADS)
    decode_kernel(const __grid_constant__ DecodeParams p) {
    using C = Cfg<MX, RT, S, BG, CS>;
    constexpr int NT = C::NT, BN = C::BN;
    extern __shared__ __align__(16) uint8_t smem[];
    const uint32_t bias = p.bias;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int rt = warp / S, s = warp % S;
    const int M = p.M, N = p.N, K = p.K, G = p.G;
    const int crank = CS > 1 ? static_cast<int>(cluster_rank()) : 0;
    const int tile = blockIdx.x / CS;
    const int n0 = tile * BN;
    const Layout L(M, K, G, CS, S, MX, BN, p.csr_cap);
    const int gpc = L.kc / 128;
    const int g_lo = min(G, crank * gpc), g_hi = min(G, g_lo + gpc);

    // ---------------------------------------------- start the weight stream
    const int r0 = n0 + 16 * rt + g, r1 = r0 + 8;
    const size_t wrow = static_cast<size_t>(K) / 8;
    const uint32_t *w0p = p.qweight + static_cast<size_t>(min(r0, N - 1)) * wrow + 4 * t;
    const uint32_t *w1p = p.qweight + static_cast<size_t>(min(r1, N - 1)) * wrow + 4 * t;
    const uint32_t *s0p = p.sz + static_cast<size_t>(min(r0, N - 1)) * p.Gp;
    const uint32_t *s1p = p.sz + static_cast<size_t>(min(r1, N - 1)) * p.Gp;
    const int ngw = (g_hi - g_lo - s + S - 1) / S;  // groups of this warp (may be <= 0)
    const int nb = ngw > 0 ? (ngw + BG - 1) / BG : 0;

    auto load = [&](Batch<BG> &b, int bi) {
#pragma unroll
        for (int u = 0; u < BG; ++u) {
            const int gi = g_lo + s + S * (bi * BG + u);
            if (gi < g_hi) {
                b.w[u][0] = ldg_stream(w0p + gi * 16);
                b.w[u][1] = ldg_stream(w1p + gi * 16);
                b.sz[u][0] = ldg_nc(s0p + gi);
                b.sz[u][1] = ldg_nc(s1p + gi);
            }
        }
    };
    Batch<BG> A, B;
    if (nb > 0) load(A, 0);
    if (threadIdx.x == 0 && crank == 0) l2_prefetch_share(p.pf, tile, static_cast<int>(gridDim.x) / CS);
    pdl_launch_dependents();

    // ---------------------------------------------- stage X and the CSR slice
    float *red = reinterpret_cast<float *>(smem + L.red);
    float *res = reinterpret_cast<float *>(smem + L.res);
    const int r_t = threadIdx.x / C::TEAM, tl = threadIdx.x % C::TEAM;
    const int row_t = n0 + r_t;
    int e_b = 0, e_e = 0, ra = 0, rb = 0;
    if (p.with_residual) {
        e_b = p.row_ptr[n0];
        e_e = p.row_ptr[min(n0 + BN, N)];
        if (row_t < N) {
            ra = p.row_ptr[row_t];
            rb = p.row_ptr[row_t + 1];
        }
    }
    const bool staged = p.csr_cap > 0;
    const int col_base = e_b & ~7, val_base = (e_b >> 1) & ~15;
    if (staged && e_e > e_b) {
        const int ncol16 = ((e_e - col_base) * 2 + 15) / 16;
        const int nval16 = (((e_e + 1) >> 1) - val_base + 15) / 16;
        for (int i = threadIdx.x; i < ncol16; i += C::THREADS)
            cp_async16(smem + L.col + 16 * i, p.col + col_base + 8 * i);
        for (int i = threadIdx.x; i < nval16; i += C::THREADS)
            cp_async16(smem + L.val + 16 * i, p.val + val_base + 16 * i);
    }
    pdl_wait();  // X may come from the previous kernel; Y may still be read by it
    {
        const int k_lo = g_lo * 128, per_row = (g_hi - g_lo) * 16;  // 16-byte chunks
        for (int m = 0; m < M; ++m)
            for (int c = threadIdx.x; c < per_row; c += C::THREADS)
                cp_async16(smem + L.x + m * L.xrs + 16 * c,
                           p.X + static_cast<size_t>(m) * K + k_lo + 8 * c);
    }
    cp_async_wait_all();
    __syncthreads();

    // ---------------------------------------------- sparse branch
    {
        constexpr int E = C::E, TPG = C::TPG;
        const uint16_t *colp =
            staged ? reinterpret_cast<const uint16_t *>(smem + L.col) : p.col;
        const uint8_t *valp = staged ? smem + L.val : p.val;
        const int coff = staged ? col_base : 0, voff = staged ? val_base : 0;
        const int tg = tl / E, el = tl % E;
        float acc[TPG];
#pragma unroll
        for (int j = 0; j < TPG; ++j) acc[j] = 0.f;
        float sr = 0.f;
        if (rb > ra) {
            const int k_lo = g_lo * 128;
            int a = ra, b = rb;
            if constexpr (CS > 1) {
                a = col_lower_bound(colp, coff, a, b, k_lo);
                b = col_lower_bound(colp, coff, a, b, g_hi * 128);
            }
            sr = half_bits_to_f32(p.rscale[row_t]);
            const uint16_t *xs = reinterpret_cast<const uint16_t *>(smem + L.x);
            for (int e0 = a + el; e0 < b; e0 += 4 * E) {
                int c[4];
                float q[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int idx = e0 + u * E;
                    const bool ok = idx < b;
                    c[u] = ok ? static_cast<int>(colp[idx - coff]) - k_lo : 0;
                    const uint32_t byte = ok ? valp[(idx >> 1) - voff] : 0u;
                    q[u] = ok ? static_cast<float>(
                                    static_cast<int>(((byte >> ((idx & 1) * 4)) & 0xF) ^ 8) - 8)
                              : 0.f;
                }
#pragma unroll
                for (int j = 0; j < TPG; ++j) {
                    const int tok = tg * TPG + j;
                    if (tok < M) {
                        const uint16_t *xr = xs + tok * (L.xrs / 2);
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            acc[j] = fmaf(q[u], bf16_bits_to_f32(xr[c[u]]), acc[j]);
                    }
                }
            }
        }
        // every lane reaches the reduction; E lanes of a token group are adjacent
#pragma unroll
        for (int off = E / 2; off > 0; off >>= 1)
#pragma unroll
            for (int j = 0; j < TPG; ++j) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], off);
        if (el == 0) {
#pragma unroll
            for (int j = 0; j < TPG; ++j) res[r_t * MX + tg * TPG + j] = sr * acc[j];
        }
    }

    // ---------------------------------------------- dense branch
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;

    auto compute = [&](const Batch<BG> &b, int bi) {
#pragma unroll
        for (int u = 0; u < BG; ++u) {
            const int gi = g_lo + s + S * (bi * BG + u);
            if (gi >= g_hi) break;
            const float s0 = half_bits_to_f32(b.sz[u][0]), s1 = half_bits_to_f32(b.sz[u][1]);
            const uint32_t z0 = static_cast<uint32_t>(half_bits_to_f32(b.sz[u][0] >> 16));
            const uint32_t z1 = static_cast<uint32_t>(half_bits_to_f32(b.sz[u][1] >> 16));
            const uint32_t zz0 = (0x4300u | z0) * 0x00010001u;  // bf16x2 (128+z)
            const uint32_t zz1 = (0x4300u | z1) * 0x00010001u;
            uint32_t xb[NT][16];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int tok = g + 8 * nt;
                if (tok < M) {
                    const uint8_t *xp = smem + L.x + tok * L.xrs + (gi - g_lo) * 256 + 64 * t;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint4 v = lds128(xp + 16 * i);
                        xb[nt][4 * i + 0] = v.x;
                        xb[nt][4 * i + 1] = v.y;
                        xb[nt][4 * i + 2] = v.z;
                        xb[nt][4 * i + 3] = v.w;
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) xb[nt][i] = 0u;
                }
            }
            float c[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) c[nt][i] = 0.f;
            const uint32_t wr0[4] = {b.w[u][0].x, b.w[u][0].y, b.w[u][0].z, b.w[u][0].w};
            const uint32_t wr1[4] = {b.w[u][1].x, b.w[u][1].y, b.w[u][1].z, b.w[u][1].w};
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
                for (int nt = 0; nt < NT; ++nt)
                    mma_bf16_16816(c[nt], a, xb[nt][2 * ks], xb[nt][2 * ks + 1], c[nt]);
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                acc[nt][0] = fmaf(s0, c[nt][0], acc[nt][0]);
                acc[nt][1] = fmaf(s0, c[nt][1], acc[nt][1]);
                acc[nt][2] = fmaf(s1, c[nt][2], acc[nt][2]);
                acc[nt][3] = fmaf(s1, c[nt][3], acc[nt][3]);
            }
        }
    };

    for (int bi = 0; bi < nb; bi += 2) {
        if (bi + 1 < nb) load(B, bi + 1);
        compute(A, bi);
        if (bi + 1 < nb) {
            if (bi + 2 < nb) load(A, bi + 2);
            compute(B, bi + 1);
        }
    }

    // ---------------------------------------------- reduction-add
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int tok = 8 * nt + 2 * t + (i & 1);
            const int row = 16 * rt + g + ((i < 2) ? 0 : 8);
            if (tok < MX) red[(s * MX + tok) * BN + row] = acc[nt][i];
        }
    __syncthreads();
    // this CTA's fp32 sums, kept in the residual buffer for the cluster
    for (int idx = threadIdx.x; idx < M * BN; idx += C::THREADS) {
        const int m = idx / BN, r = idx % BN;
        float y = res[r * MX + m];
#pragma unroll
        for (int k = 0; k < S; ++k) y += red[(k * MX + m) * BN + r];
        res[r * MX + m] = y;
    }
    if constexpr (CS > 1)
        cluster_sync();
    else
        __syncthreads();
    if (crank == 0) {
        for (int idx = threadIdx.x; idx < M * BN; idx += C::THREADS) {
            const int m = idx / BN, r = idx % BN, n = n0 + r;
            float y = res[r * MX + m];
            if constexpr (CS > 1) {
#pragma unroll
                for (int k = 1; k < CS; ++k) y += ld_dsmem_f32(&res[r * MX + m], k);
            }
            if (n < N) {
                if (p.Yf)
                    p.Yf[static_cast<size_t>(m) * N + n] = y;
                else
                    p.Y[static_cast<size_t>(m) * N + n] = __float2bfloat16_rn(y);
            }
        }
    }
    // the other ranks keep their shared memory alive until rank 0 has read it
    if constexpr (CS > 1) cluster_sync();
}

template <int MX, int RT, int S, int BG, int CS>
mq_status run(const mq_weight *w, const void *X, int M, void *Y, cudaStream_t stream,
              float *partial, const L2Prefetch &pf) {
    using C = Cfg<MX, RT, S, BG, CS>;
    const DeviceWeight &d = weight_device(w);
    const bool with_residual = partial == nullptr;
    const int64_t tile_nnz = with_residual ? max_tile_nnz(w, C::BN) : 0;
    DecodeParams p;
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
    p.bias = kBiasBf16;
    p.with_residual = with_residual ? 1 : 0;
    p.pf = pf;
    // The tile's CSR slice is staged in shared memory while that keeps two
    // CTAs per SM; a longer slice (a dense or block-allocated residual) is
    // read from global memory by the walk instead.
    constexpr int kStagedLimit = 100 * 1024;
    p.csr_cap = static_cast<int>(std::min<int64_t>(tile_nnz, int64_t(1) << 24));
    if (Layout(M, p.K, p.G, CS, S, MX, C::BN, p.csr_cap).total > kStagedLimit) p.csr_cap = 0;
    const Layout L(M, p.K, p.G, CS, S, MX, C::BN, p.csr_cap);
    if (L.total > 227 * 1024)
        return fail(MQ_ERR_UNSUPPORTED, "decode kernel: the X slice exceeds shared memory");
    auto kern = decode_kernel<MX, RT, S, BG, CS>;
    static bool configured[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(MQ_ERR_CUDA, "cudaGetDevice failed");
    if (dev >= 0 && dev < 64 && !configured[dev]) {
        // the largest shared-memory carveout, as for every decode kernel, so
        // that consecutive launches of different layers can share an SM
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) !=
                cudaSuccess ||
            cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared) != cudaSuccess)
            return fail(MQ_ERR_CUDA, "cudaFuncSetAttribute failed for the decode kernel");
        configured[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((d.N + C::BN - 1) / C::BN) * CS);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = static_cast<size_t>(L.total);
    cfg.stream = stream;
    cudaLaunchAttribute attrs[2];
    int na = 0;
    attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
    if (CS > 1) {
        attrs[na].id = cudaLaunchAttributeClusterDimension;
        attrs[na].val.clusterDim.x = CS;
        attrs[na].val.clusterDim.y = 1;
        attrs[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = attrs;
    cfg.numAttrs = na;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p);
    if (e != cudaSuccess)
        return fail(MQ_ERR_CUDA, std::string("decode launch: ") + cudaGetErrorString(e));
    return MQ_OK;
}

// Smallest power-of-two K split (at most 8, a portable cluster) whose X
// slice fits the shared-memory budget.
int k_split(int M, int64_t K) {
    const int64_t budget = 96 * 1024;
    int cs = 1;
    while (cs < 8 && static_cast<int64_t>(M) * ((K / 128 + cs - 1) / cs) * 256 > budget) cs *= 2;
    return cs;
}

template <int MX, int RT, int S, int BG>
mq_status run_cs(const mq_weight *w, const void *X, int M, void *Y, cudaStream_t stream,
                 float *partial, const L2Prefetch &pf) {
    switch (k_split(M, weight_device(w).K)) {
        case 1: return run<MX, RT, S, BG, 1>(w, X, M, Y, stream, partial, pf);
        case 2: return run<MX, RT, S, BG, 2>(w, X, M, Y, stream, partial, pf);
        case 4: return run<MX, RT, S, BG, 4>(w, X, M, Y, stream, partial, pf);
        default: return run<MX, RT, S, BG, 8>(w, X, M, Y, stream, partial, pf);
    }
}

}  // namespace

mq_status launch_decode(const mq_weight *w, const void *X, int M, void *Y, cudaStream_t stream,
                        float *partial, const L2Prefetch &pf) {
    {
        // the streaming kernel, when X (and a CTA's residual share) fits its
        // shared memory without leaving a second wave of CTAs
        const mq_status st = launch_decode_stream(w, X, M, Y, stream, partial, pf);
        if (st != MQ_ERR_UNSUPPORTED) return st;
    }
    if (M > 1) {
        // tall layers whose X does not fit: X from L2
        const mq_status st = launch_decode_tall(w, X, M, Y, stream, partial, pf);
        if (st != MQ_ERR_UNSUPPORTED) return st;
    }
    if (M > 8) {
        // 9-16 tokens on tall layers the tall-layer kernel declined (a CTA's
        // residual lists beyond their shared-memory budget)
        const mq_status st = launch_decode_wide(w, X, M, Y, stream, partial, pf);
        if (st != MQ_ERR_UNSUPPORTED) return st;
    }
    if (M == 1) {
        // More 16-row tiles than two 8-warp CTAs per SM hold at once: 4-warp
        // CTAs (four per SM) overlap their waves better (11008 x 4096:
        // 10.5 us against 13.5 us); otherwise 8 warps per tile stream more.
        if ((weight_device(w).N + 15) / 16 > 2 * static_cast<int64_t>(sm_count()))
            return run_cs<1, 1, 4, 4>(w, X, M, Y, stream, partial, pf);
        return run_cs<1, 1, 8, 4>(w, X, M, Y, stream, partial, pf);
    }
    if (M <= 8) return run_cs<8, 2, 4, 2>(w, X, M, Y, stream, partial, pf);
    const mq_status st = run_cs<16, 4, 2, 2>(w, X, M, Y, stream, partial, pf);
    // X's slice of a very long K does not fit: the wide kernel streams X
    if (st == MQ_ERR_UNSUPPORTED) return launch_decode_wide(w, X, M, Y, stream, partial, pf, true);
    return st;
}

}  // namespace mq
