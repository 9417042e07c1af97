// W4A4: activations quantized to 4 bits as well, M <= 16.
//
// MosaicQuant "Methodology" 3. (ZipperEngine) begins its pipeline with a
// quantization stage ahead of the dense computation, the sparse
// compensation and the reduction-add; "Experimental Results" evaluate the
// method as W4A4. Two launches on one stream (the second with programmatic
// dependent launch, so its weight stream starts while the first runs):
//
//   quantize_kernel: one CTA per token. The absolute maximum of the token's
//     bf16 values gives s_x = fp32(a / 7) (IEEE division; 1 for a zero
//     token), then every code is clamp(rne(fp32(x / s_x)), -8, 7), written as
//     int8 [M][K].
//
//   decode_a4_kernel (M <= 8, and up to 16 on layers too small for the wide
//     kernel's W4A4 form, decode_wide.cu): the narrow decode kernel's layout (a CTA owns 16*RT rows,
//     its warps split the K groups, codes stream from HBM into registers) with
//     integer tensor-core MMAs. A thread's 16-byte load of packed codes holds,
//     per k-step of 32, one word of row g and one of row g+8; masking the low
//     and the high nibbles gives four bytes each, and (v | 0x80) - z, then
//     ^ 0x80, per byte turns them into the int8 codes q - z with no carries
//     between bytes. mma.sync m16n8k32 s8 x s8 -> s32 sums each group exactly;
//     the group scale is applied in fp32. The quantization kernel writes the
//     activation codes with the bytes of every 8-column chunk permuted as
//     (0,4,1,5,2,6,3,7), the order the nibble interleave of the packed codes
//     puts the weight bytes in, so both operands meet at the same k.
//     The residual is walked as in the narrow kernel (a team of lanes per
//     row, shuffle reduction) with exact integer products q_r * c, and
//     Y = s_x * (sum_g s_g * D_g + s_r * R) is stored once as bf16.

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "kernels.h"

namespace mq {
namespace {

// ---------------------------------------------------------------- quantization
constexpr int kQThreads = 256;

struct QuantizeArgs {
    const __nv_bfloat16 *X;  // [M][K]
    int K;
    int8_t *codes;           // [M][K]
    float *scales;           // [M]
    int permute;             // store each 8-column chunk's codes in the order (0,4,1,5,2,6,3,7)
};

__global__ void __launch_bounds__(kQThreads) quantize_kernel(const __grid_constant__ QuantizeArgs qa) {
    const __nv_bfloat16 *X = qa.X;
    const int K = qa.K;
    int8_t *codes = qa.codes;
    float *scales = qa.scales;
    __shared__ float wmax[kQThreads / 32];
    const int m = blockIdx.x;
    const uint4 *xr = reinterpret_cast<const uint4 *>(X + static_cast<size_t>(m) * K);
    const int nc = K / 8;
    pdl_launch_dependents();
    pdl_wait();  // X may come from the previous kernel
    float a = 0.f;
    for (int c = threadIdx.x; c < nc; c += kQThreads) {
        const uint4 v = xr[c];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            a = fmaxf(a, fabsf(bf16_bits_to_f32(w[i] & 0xFFFFu)));
            a = fmaxf(a, fabsf(bf16_bits_to_f32(w[i] >> 16)));
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = a;
    __syncthreads();
    a = wmax[0];
#pragma unroll
    for (int i = 1; i < kQThreads / 32; ++i) a = fmaxf(a, wmax[i]);
    const float s = a > 0.f ? __fdiv_rn(a, 7.0f) : 1.0f;
    if (threadIdx.x == 0) scales[m] = s;
    uint2 *cr = reinterpret_cast<uint2 *>(codes + static_cast<size_t>(m) * K);
    for (int c = threadIdx.x; c < nc; c += kQThreads) {
        const uint4 v = xr[c];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t out[2] = {0u, 0u};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t b16 = (i & 1) ? (w[i >> 1] >> 16) : (w[i >> 1] & 0xFFFFu);
            int q = __float2int_rn(__fdiv_rn(bf16_bits_to_f32(b16), s));
            q = min(7, max(-8, q));
            const int pos = qa.permute ? (((i & 3) << 1) | (i >> 2)) : i;
            out[pos >> 2] |= (static_cast<uint32_t>(q) & 0xFFu) << (8 * (pos & 3));
        }
        cr[c] = make_uint2(out[0], out[1]);
    }
}

// ---------------------------------------------------------------- fused W4A4 product
struct A4Params {
    const uint32_t *qweight;  // [N][K/8]
    const uint32_t *sz;       // [N][Gp]
    const int8_t *codes;      // [M][K] activation codes
    const float *xscale;      // [M]
    __nv_bfloat16 *Y;         // [M][N]
    const int32_t *row_ptr;
    const uint16_t *col;
    const uint8_t *val;
    const uint16_t *rscale;
    int M, N, K, G, Gp;
    uint32_t bias;  // kBiasBf16, or kBiasI8 for int8 codes (held in a register)
    int csr_cap;  // residual entries staged in shared memory (0: read from global)
};

template <int MX, int RT, int S, int BG, int CS>
struct A4Cfg {
    static constexpr int NT = MX / 8;   // n8 token tiles
    static constexpr int BN = 16 * RT;  // rows per CTA
    static constexpr int WARPS = RT * S;
    static constexpr int THREADS = WARPS * 32;
    static constexpr int TEAM = THREADS / BN;  // residual lanes per row
    static constexpr int TPG = 4;              // tokens per token group
    static constexpr int TG = MX / TPG;
    static constexpr int E = TEAM / TG;        // lanes per token group striding entries
    static_assert(MX == 8 || MX == 16, "token tiles of 8");
    static_assert(THREADS % BN == 0 && TEAM <= 32 && 32 % TEAM == 0 && TEAM % TG == 0, "teams");
    static_assert((E & (E - 1)) == 0, "power-of-two entry lanes");
    static_assert(CS == 1 || CS == 2 || CS == 4 || CS == 8, "cluster size");
};

// Shared-memory layout (bytes), identical on host and device.
struct A4Layout {
    int xrs, kc, x, red, res, col, val, total;
    __host__ __device__ A4Layout(int M, int G, int CS, int S, int MX, int BN, int csr_cap) {
        const int gpc = (G + CS - 1) / CS;
        kc = gpc * 128;   // columns of one rank's K range
        xrs = kc + 16;    // code row stride
        x = 0;
        red = (M * xrs + 15) / 16 * 16;
        res = red + S * MX * BN * 4;
        col = res + BN * MX * 4;
        val = col + (csr_cap * 2 + 32 + 15) / 16 * 16;
        total = val + (csr_cap / 2 + 32 + 15) / 16 * 16;
    }
};

template <int BG>
struct A4Batch {
    uint4 w[BG][2];
    uint32_t sz[BG][2];
};

// Byte of activation column `rel` (relative to the staged range) inside its
// permuted 8-column chunk.
__device__ __forceinline__ int xpos(int rel) {
    return (rel & ~7) | ((rel & 3) << 1) | ((rel >> 2) & 1);
}

template <int MX, int RT, int S, int BG, int CS>
__global__ void __launch_bounds__(A4Cfg<MX, RT, S, BG, CS>::THREADS)
    decode_a4_kernel(const __grid_constant__ A4Params p) {
    using C = A4Cfg<MX, RT, S, BG, CS>;
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
    const A4Layout L(M, G, CS, S, MX, BN, p.csr_cap);
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
    auto load = [&](A4Batch<BG> &b, int bi) {
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
    A4Batch<BG> A, B;
    if (nb > 0) load(A, 0);
    pdl_launch_dependents();

    // ---------------------------------------------- stage the codes of X and the CSR slice
    float *red = reinterpret_cast<float *>(smem + L.red);
    float *res = reinterpret_cast<float *>(smem + L.res);
    const int r_t = threadIdx.x / C::TEAM, tml = threadIdx.x % C::TEAM;
    const int row_t = n0 + r_t;
    int e_b = 0, e_e = 0, ra = 0, rb = 0;
    e_b = p.row_ptr[n0];
    e_e = p.row_ptr[min(n0 + BN, N)];
    if (row_t < N) {
        ra = p.row_ptr[row_t];
        rb = p.row_ptr[row_t + 1];
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
    pdl_wait();  // the codes of X come from the quantization kernel
    {
        // the codes arrive with each 8-column chunk already permuted
        const int k_lo = g_lo * 128, per_row = (g_hi - g_lo) * 8;  // 16-byte chunks
        for (int m = 0; m < M; ++m)
            for (int c = threadIdx.x; c < per_row; c += C::THREADS)
                cp_async16(smem + L.x + m * L.xrs + 16 * c, p.codes + static_cast<size_t>(m) * K + k_lo + 16 * c);
    }
    cp_async_wait_all();
    __syncthreads();

    // ---------------------------------------------- sparse branch (exact integers)
    {
        constexpr int E = C::E, TPG = C::TPG;
        const uint16_t *colp = staged ? reinterpret_cast<const uint16_t *>(smem + L.col) : p.col;
        const uint8_t *valp = staged ? smem + L.val : p.val;
        const int coff = staged ? col_base : 0, voff = staged ? val_base : 0;
        const int tg = tml / E, el = tml % E;
        int racc[TPG];
#pragma unroll
        for (int j = 0; j < TPG; ++j) racc[j] = 0;
        if (rb > ra) {
            const int k_lo = g_lo * 128;
            int a = ra, b = rb;
            if constexpr (CS > 1) {
                a = col_lower_bound(colp, coff, a, b, k_lo);
                b = col_lower_bound(colp, coff, a, b, g_hi * 128);
            }
            const int8_t *xs = reinterpret_cast<const int8_t *>(smem + L.x);
            for (int e0 = a + el; e0 < b; e0 += 4 * E) {
                int c[4], q[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int idx = e0 + u * E;
                    const bool ok = idx < b;
                    c[u] = ok ? xpos(static_cast<int>(colp[idx - coff]) - k_lo) : 0;
                    const uint32_t byte = ok ? valp[(idx >> 1) - voff] : 0u;
                    q[u] = ok ? static_cast<int>(((byte >> ((idx & 1) * 4)) & 0xF) ^ 8) - 8 : 0;
                }
#pragma unroll
                for (int j = 0; j < TPG; ++j) {
                    const int tok = tg * TPG + j;
                    if (tok < M) {
                        const int8_t *xr = xs + tok * L.xrs;
#pragma unroll
                        for (int u = 0; u < 4; ++u) racc[j] += q[u] * static_cast<int>(xr[c[u]]);
                    }
                }
            }
        }
#pragma unroll
        for (int off = E / 2; off > 0; off >>= 1)
#pragma unroll
            for (int j = 0; j < TPG; ++j) racc[j] += __shfl_xor_sync(0xffffffffu, racc[j], off);
        if (el == 0) {
            const float sr = row_t < N ? half_bits_to_f32(p.rscale[row_t]) : 0.f;
#pragma unroll
            for (int j = 0; j < TPG; ++j)
                res[r_t * MX + tg * TPG + j] = sr * static_cast<float>(racc[j]);
        }
    }

    // ---------------------------------------------- dense branch (exact group sums)
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;

    auto compute = [&](const A4Batch<BG> &b, int bi) {
#pragma unroll
        for (int u = 0; u < BG; ++u) {
            const int gi = g_lo + s + S * (bi * BG + u);
            if (gi >= g_hi) break;
            const float s0 = half_bits_to_f32(b.sz[u][0]), s1 = half_bits_to_f32(b.sz[u][1]);
            const uint32_t z0 = static_cast<uint32_t>(half_bits_to_f32(b.sz[u][0] >> 16));
            const uint32_t z1 = static_cast<uint32_t>(half_bits_to_f32(b.sz[u][1] >> 16));
            const uint32_t zz0 = z0 * 0x01010101u, zz1 = z1 * 0x01010101u;
            uint32_t xb[NT][8];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int tok = g + 8 * nt;
                if (tok < M) {
                    const uint8_t *xp = smem + L.x + tok * L.xrs + (gi - g_lo) * 128 + 32 * t;
                    const uint4 v0 = lds128(xp), v1 = lds128(xp + 16);
                    xb[nt][0] = v0.x;
                    xb[nt][1] = v0.y;
                    xb[nt][2] = v0.z;
                    xb[nt][3] = v0.w;
                    xb[nt][4] = v1.x;
                    xb[nt][5] = v1.y;
                    xb[nt][6] = v1.z;
                    xb[nt][7] = v1.w;
                } else {
#pragma unroll
                    for (int q = 0; q < 8; ++q) xb[nt][q] = 0u;
                }
            }
            int d[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int q = 0; q < 4; ++q) d[nt][q] = 0;
            const uint32_t wr0[4] = {b.w[u][0].x, b.w[u][0].y, b.w[u][0].z, b.w[u][0].w};
            const uint32_t wr1[4] = {b.w[u][1].x, b.w[u][1].y, b.w[u][1].z, b.w[u][1].w};
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                uint32_t a[4];
                a[0] = codes_minus_zero_r(wr0[ks], zz0, bias);
                a[1] = codes_minus_zero_r(wr1[ks], zz1, bias);
                a[2] = codes_minus_zero_r(wr0[ks] >> 4, zz0, bias);
                a[3] = codes_minus_zero_r(wr1[ks] >> 4, zz1, bias);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma_s8_16832(d[nt], a, xb[nt][2 * ks], xb[nt][2 * ks + 1]);
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                acc[nt][0] = fmaf(s0, static_cast<float>(d[nt][0]), acc[nt][0]);
                acc[nt][1] = fmaf(s0, static_cast<float>(d[nt][1]), acc[nt][1]);
                acc[nt][2] = fmaf(s1, static_cast<float>(d[nt][2]), acc[nt][2]);
                acc[nt][3] = fmaf(s1, static_cast<float>(d[nt][3]), acc[nt][3]);
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

    // ---------------------------------------------- reduction-add and scaling
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int tok = 8 * nt + 2 * t + (i & 1);
            const int row = 16 * rt + g + ((i < 2) ? 0 : 8);
            red[(s * MX + tok) * BN + row] = acc[nt][i];
        }
    __syncthreads();
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
            if (n < N) p.Y[static_cast<size_t>(m) * N + n] = __float2bfloat16_rn(y * p.xscale[m]);
        }
    }
    // the other ranks keep their shared memory alive until rank 0 has read it
    if constexpr (CS > 1) cluster_sync();
}

template <typename Kern, typename P>
mq_status launch_pdl(Kern kern, const P &p, dim3 grid, int threads, size_t smem, int cs,
                     cudaStream_t stream, const char *what) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attrs[2];
    int na = 0;
    attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
    if (cs > 1) {
        attrs[na].id = cudaLaunchAttributeClusterDimension;
        attrs[na].val.clusterDim.x = cs;
        attrs[na].val.clusterDim.y = 1;
        attrs[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = attrs;
    cfg.numAttrs = na;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p);
    if (e != cudaSuccess) return fail(MQ_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
    return MQ_OK;
}

template <int MX, int RT, int S, int BG, int CS>
mq_status run_a4(const mq_weight *w, const int8_t *codes, const float *xscale, int M, void *Y,
                 cudaStream_t stream) {
    using C = A4Cfg<MX, RT, S, BG, CS>;
    const DeviceWeight &d = weight_device(w);
    const int64_t tile_nnz = d.nnz > 0 ? max_tile_nnz(w, C::BN) : 0;
    A4Params p;
    p.qweight = d.qweight;
    p.sz = d.sz;
    p.codes = codes;
    p.xscale = xscale;
    p.Y = static_cast<__nv_bfloat16 *>(Y);
    p.row_ptr = d.row_ptr;
    p.col = d.col;
    p.val = d.val;
    p.rscale = d.rscale;
    p.M = M;
    p.N = static_cast<int>(d.N);
    p.K = static_cast<int>(d.K);
    p.G = static_cast<int>(d.G);
    p.Gp = static_cast<int>(d.Gp);
    p.bias = kBiasI8;
    // stage the tile's CSR slice while that keeps two CTAs per SM
    p.csr_cap = static_cast<int>(std::min<int64_t>(tile_nnz, int64_t(1) << 24));
    if (A4Layout(M, p.G, CS, S, MX, C::BN, p.csr_cap).total > 100 * 1024) p.csr_cap = 0;
    const A4Layout L(M, p.G, CS, S, MX, C::BN, p.csr_cap);
    if (L.total > 227 * 1024)
        return fail(MQ_ERR_UNSUPPORTED, "W4A4 decode kernel: the code slice exceeds shared memory");
    auto kern = decode_a4_kernel<MX, RT, S, BG, CS>;
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
            return fail(MQ_ERR_CUDA, "cudaFuncSetAttribute failed for the W4A4 decode kernel");
        configured[dev] = true;
    }
    const dim3 grid(static_cast<unsigned>((d.N + C::BN - 1) / C::BN) * CS);
    return launch_pdl(kern, p, grid, C::THREADS, static_cast<size_t>(L.total), CS, stream,
                      "W4A4 decode launch");
}

// Smallest power-of-two K split (at most 8) whose code slice fits 96 KB.
int a4_split(int M, int64_t K) {
    int cs = 1;
    while (cs < 8 && static_cast<int64_t>(M) * ((K / 128 + cs - 1) / cs) * 128 > 96 * 1024) cs *= 2;
    return cs;
}

template <int MX, int RT, int S, int BG>
mq_status run_a4_cs(const mq_weight *w, const int8_t *codes, const float *xscale, int M, void *Y,
                    cudaStream_t stream) {
    switch (a4_split(M, weight_device(w).K)) {
        case 1: return run_a4<MX, RT, S, BG, 1>(w, codes, xscale, M, Y, stream);
        case 2: return run_a4<MX, RT, S, BG, 2>(w, codes, xscale, M, Y, stream);
        case 4: return run_a4<MX, RT, S, BG, 4>(w, codes, xscale, M, Y, stream);
        default: return run_a4<MX, RT, S, BG, 8>(w, codes, xscale, M, Y, stream);
    }
}

}  // namespace

mq_status launch_quantize(const void *X, int64_t M, int64_t K, void *codes, float *scales,
                          cudaStream_t stream, bool permuted) {
    if (M <= 0) return MQ_OK;
    QuantizeArgs a{static_cast<const __nv_bfloat16 *>(X), static_cast<int>(K),
                   static_cast<int8_t *>(codes), scales, permuted ? 1 : 0};
    return launch_pdl(quantize_kernel, a, dim3(static_cast<unsigned>(M)), kQThreads, 0, 1, stream,
                      "activation quantization launch");
}

mq_status launch_decode_a4(const mq_weight *w, const int8_t *codes, const float *xscale, int M,
                           void *Y, cudaStream_t stream) {
    if (M > 8) {
        const mq_status st = launch_decode_wide_a4(w, codes, xscale, M, Y, stream);
        if (st != MQ_ERR_UNSUPPORTED) return st;
    }
    if (M == 1) {
        // as for the W4A16 kernel: 4-warp CTAs when the 16-row tiles exceed
        // two 8-warp CTAs per SM
        if ((weight_device(w).N + 15) / 16 > 2 * static_cast<int64_t>(sm_count()))
            return run_a4_cs<8, 1, 4, 4>(w, codes, xscale, M, Y, stream);
        return run_a4_cs<8, 1, 8, 4>(w, codes, xscale, M, Y, stream);
    }
    if (M <= 8) return run_a4_cs<8, 2, 4, 2>(w, codes, xscale, M, Y, stream);
    return run_a4_cs<16, 4, 2, 2>(w, codes, xscale, M, Y, stream);
}

}  // namespace mq
