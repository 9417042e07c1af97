// Decode kernel: Y[M][N] = X[M][K] * W_hat^T for M <= 16, one fused pass.
//
// MosaicQuant "Methodology" 3. (ZipperEngine): the sparse residual is
// computed inside the dense 4-bit GEMM kernel, in the same pass over the
// activations, and the dense and sparse parts meet in one reduction-add; no
// second kernel reloads X or merges partial outputs.
//
// For M <= 16 the layer is bound by streaming the packed weight from HBM.
// Per CTA (BN = 16*RT output rows, all of K):
//   * one producer warp streams stages of GS = S*GW groups of 128 columns:
//     TMA boxes of the packed codes ([BN][16 words] per group), of the
//     scale/zero words ([BN][GS]) and 1D bulk copies of the X chunk
//     ([M][128*GS] bf16), all completing on one mbarrier per stage;
//   * RT*S consumer warps; warp (rt, s) owns rows [16rt, 16rt+16) and the
//     groups s*GW .. s*GW+GW-1 of every stage. For each group it turns the
//     packed nibbles into exact bf16 codes (q - z) in registers (OR into the
//     mantissa of 128.0, subtract 128 + z), runs 8 mma.sync m16n8k16 with
//     fp32 accumulation of the exact products, and adds s * partial into its
//     running fp32 accumulator; then it walks the CSR residual entries of its
//     two rows whose columns fall in that group (cursor per row, columns
//     ascending) and adds s_r * q_r * x from the X chunk already in shared
//     memory: the "zipper" merge of dense and sparse work in one pass;
//   * split-K partials of the S warps of a row tile meet in shared memory
//     and one bf16 store writes Y (coalesced along N).
// The k order inside a group is permuted so that each thread's 16-byte load
// of packed codes feeds its own mma fragments with no shuffles: k-step s'
// (0..7) of thread (g, t) covers columns 32t + 4s' + {0,1} (fragment k 2t,
// 2t+1) and 32t + 4s' + {2,3} (fragment k 2t+8, 2t+9); X is read with the
// same permutation, so the sum over k is unchanged.

#include "common.cuh"
#include "internal.h"
#include "kernels.h"

namespace mq {
namespace {

struct DecodeParams {
    CUtensorMap tm_w;   // qweight [N][K/8] u32, box [BN][16]
    CUtensorMap tm_sz;  // sz [N][Gp] u32, box [BN][GS]
    const __nv_bfloat16 *X;
    __nv_bfloat16 *Y;
    float *Yf;          // fp32 dense-only output (unfused path) or null
    const int32_t *row_ptr;
    const uint16_t *col;
    const uint8_t *val;
    const uint16_t *rscale;
    int *err;
    int M, N, K, G;
    int csr_col_bytes;  // shared-memory capacity reserved for the residual slice
    int with_residual;
};

template <int MX, int RT, int S, int GW, int STAGES>
struct Cfg {
    static constexpr int NT = (MX + 7) / 8;      // n8 tiles of tokens
    static constexpr int BN = 16 * RT;            // rows per CTA
    static constexpr int GS = S * GW;             // groups per stage
    static constexpr int WARPS = RT * S;          // consumer warps
    static constexpr int THREADS = (WARPS + 1) * 32;
    static constexpr int W_BOX = BN * 64;         // bytes of one group's codes
    static constexpr int W_STAGE = GS * W_BOX;
    static constexpr int SZ_STAGE = BN * GS * 4;
    static constexpr int XRS = GS * 256 + 64;     // X row stride in bytes
    static constexpr int X_STAGE = MX * XRS;
    static constexpr int STAGE = (W_STAGE + SZ_STAGE + X_STAGE + 127) / 128 * 128;
    static constexpr int RED = S * MX * BN * 4;   // split-K reduction buffer
    static constexpr int PIPE = STAGE * STAGES > RED ? STAGE * STAGES : RED;
    static constexpr int ROWPTR_OFF = PIPE;
    static constexpr int RSCALE_OFF = ROWPTR_OFF + ((BN + 1) * 4 + 15) / 16 * 16;
    static constexpr int CSR_OFF = RSCALE_OFF + BN * 4;
    static_assert(GS % 4 == 0, "the sz box needs a 16-byte inner extent");
    static_assert(STAGE % 128 == 0, "stages stay 128-byte aligned");
    __host__ __device__ static constexpr int val_bytes(int col_bytes) { return col_bytes / 4 + 32; }
    __host__ __device__ static constexpr int bar_off(int col_bytes) {
        return (CSR_OFF + col_bytes + val_bytes(col_bytes) + 15) / 16 * 16;
    }
    __host__ __device__ static constexpr int smem_bytes(int col_bytes) {
        return bar_off(col_bytes) + (2 * STAGES + 1) * 8 + 16;
    }
};

template <int MX, int RT, int S, int GW, int STAGES>
__global__ void __launch_bounds__(Cfg<MX, RT, S, GW, STAGES>::THREADS, 1)
    decode_kernel(const __grid_constant__ DecodeParams p) {
    using C = Cfg<MX, RT, S, GW, STAGES>;
    constexpr int NT = C::NT, BN = C::BN, GS = C::GS, WARPS = C::WARPS;
    extern __shared__ __align__(128) uint8_t smem[];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * BN;
    const int M = p.M, N = p.N, K = p.K, G = p.G;
    const int nst = (G + GS - 1) / GS;

    int *rowptr_s = reinterpret_cast<int *>(smem + C::ROWPTR_OFF);
    float *rscale_s = reinterpret_cast<float *>(smem + C::RSCALE_OFF);
    uint16_t *col_s = reinterpret_cast<uint16_t *>(smem + C::CSR_OFF);
    uint8_t *val_s = smem + C::CSR_OFF + p.csr_col_bytes;
    const int bar_off = C::bar_off(p.csr_col_bytes);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + bar_off);
    uint64_t *empty = full + STAGES;
    uint64_t *csr_bar = empty + STAGES;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(csr_bar + 1);

    auto stage_w = [&](int st, int gl) {
        return reinterpret_cast<const uint32_t *>(smem + st * C::STAGE + gl * C::W_BOX);
    };
    auto stage_sz = [&](int st) {
        return reinterpret_cast<const uint32_t *>(smem + st * C::STAGE + C::W_STAGE);
    };
    auto stage_x = [&](int st, int m) {
        return smem + st * C::STAGE + C::W_STAGE + C::SZ_STAGE + m * C::XRS;
    };

    // Stage j of the pipeline: the packed codes of groups [j*GS, j*GS+GS),
    // their scale/zero words and the matching X columns.
    auto issue_stage = [&](int j) {
        const int st = j % STAGES;
        const int g0 = j * GS, ng = min(GS, G - g0);
        const uint32_t xbytes = ng * 256;
        mbar_arrive_expect_tx(&full[st], ng * C::W_BOX + C::SZ_STAGE + M * xbytes);
        for (int gl = 0; gl < ng; ++gl)
            tma_load_2d(const_cast<uint32_t *>(stage_w(st, gl)), &p.tm_w, &full[st],
                        (g0 + gl) * 16, n0);
        tma_load_2d(const_cast<uint32_t *>(stage_sz(st)), &p.tm_sz, &full[st], g0, n0);
        for (int m = 0; m < M; ++m)
            bulk_load(stage_x(st, m), p.X + size_t(m) * K + size_t(g0) * 128, xbytes, &full[st]);
    };

    const bool producer = (warp == WARPS) && (lane == 0);
    const int first = min(STAGES, nst);
    if (producer) {
        // start streaming at once; nothing below depends on the CSR offsets
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], WARPS);
        }
        mbar_init(csr_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&p.tm_w);
        prefetch_tensormap(&p.tm_sz);
        for (int j = 0; j < first; ++j) issue_stage(j);
    }
    for (int i = threadIdx.x; i <= BN; i += C::THREADS)
        rowptr_s[i] = p.with_residual ? p.row_ptr[min(n0 + i, N)] : 0;
    for (int i = threadIdx.x; i < BN; i += C::THREADS)
        rscale_s[i] = (n0 + i < N) ? half_bits_to_f32(p.rscale[n0 + i]) : 0.f;
    __syncthreads();

    const int e_begin = rowptr_s[0], e_end = rowptr_s[BN];
    const int col_base = e_begin & ~7;          // 16-byte aligned u16 index
    const int val_base = (e_begin >> 1) & ~15;  // 16-byte aligned byte index

    if (warp == WARPS) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            if (e_end > e_begin) {
                uint32_t cb = ((e_end - col_base) * 2 + 15) & ~15;
                uint32_t vb = ((((e_end + 1) >> 1) - val_base) + 15) & ~15;
                mbar_arrive_expect_tx(csr_bar, cb + vb);
                bulk_load(col_s, p.col + col_base, cb, csr_bar);
                bulk_load(val_s, p.val + val_base, vb, csr_bar);
            } else {
                mbar_arrive(csr_bar);
            }
            int issued = first;
            for (int j = first; j < nst; ++j) {
                const int st = j % STAGES;
                if (!mbar_wait(&empty[st], ((j / STAGES) - 1) & 1, p.err, kErrWaitEmpty, abort_flag))
                    break;
                issue_stage(j);
                issued = j + 1;
            }
            // no copy may still be landing in shared memory when the block exits
            for (int j = max(0, issued - STAGES); j < issued; ++j)
                mbar_wait(&full[j % STAGES], (j / STAGES) & 1, p.err, kErrWaitDrain, abort_flag);
            mbar_wait(csr_bar, 0, p.err, kErrWaitDrain, abort_flag);
        }
    } else {
        // ------------------------------------------------------ consumers
        const int rt = warp / S, s = warp % S;
        const int g = lane >> 2, t = lane & 3;
        const int r0 = 16 * rt + g, r1 = r0 + 8;
        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;
        int cur0 = rowptr_s[r0], end0 = rowptr_s[r0 + 1];
        int cur1 = rowptr_s[r1], end1 = rowptr_s[r1 + 1];
        const float sr0 = rscale_s[r0], sr1 = rscale_s[r1];
        bool csr_ready = false;

        for (int j = 0; j < nst; ++j) {
            const int st = j % STAGES;
            if (!mbar_wait_warp(&full[st], (j / STAGES) & 1, p.err, kErrWaitFull, abort_flag)) break;
            if (!csr_ready) {
                if (!mbar_wait_warp(csr_bar, 0, p.err, kErrWaitCsr, abort_flag)) break;
                csr_ready = true;
            }
            const uint8_t *xst = stage_x(st, 0);
#pragma unroll
            for (int gw = 0; gw < GW; ++gw) {
                const int gl = s * GW + gw, gi = j * GS + gl;
                if (gi >= G) break;
                const uint32_t *wt = stage_w(st, gl);
                const uint4 w0 = lds128(wt + r0 * 16 + 4 * t);
                const uint4 w1 = lds128(wt + r1 * 16 + 4 * t);
                const uint32_t sz0 = stage_sz(st)[r0 * GS + gl];
                const uint32_t sz1 = stage_sz(st)[r1 * GS + gl];
                const float s0 = half_bits_to_f32(sz0), s1 = half_bits_to_f32(sz1);
                const uint32_t z0 = static_cast<uint32_t>(half_bits_to_f32(sz0 >> 16));
                const uint32_t z1 = static_cast<uint32_t>(half_bits_to_f32(sz1 >> 16));
                const uint32_t zz0 = (0x4300u | z0) * 0x00010001u;  // bf16x2 (128+z)
                const uint32_t zz1 = (0x4300u | z1) * 0x00010001u;

                uint32_t xb[NT][16];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int tok = g + 8 * nt;
                    if (tok < M) {
                        const uint8_t *xp = xst + tok * C::XRS + gl * 256 + 64 * t;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            uint4 v = lds128(xp + 16 * i);
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
                const uint32_t wr0[4] = {w0.x, w0.y, w0.z, w0.w};
                const uint32_t wr1[4] = {w1.x, w1.y, w1.z, w1.w};
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t a_lo = wr0[ks >> 1] >> (8 * (ks & 1));
                    const uint32_t b_lo = wr1[ks >> 1] >> (8 * (ks & 1));
                    uint32_t a[4];
                    a[0] = bf16x2_sub(nib_pair_bias128(a_lo), zz0);
                    a[1] = bf16x2_sub(nib_pair_bias128(b_lo), zz1);
                    a[2] = bf16x2_sub(nib_pair_bias128(a_lo >> 4), zz0);
                    a[3] = bf16x2_sub(nib_pair_bias128(b_lo >> 4), zz1);
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

                // residual entries of rows r0, r1 inside this group
                const int k0 = gi * 128, kst = j * GS * 128;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    int &cur = h ? cur1 : cur0;
                    const int end = h ? end1 : end0;
                    const float sr = h ? sr1 : sr0;
                    while (cur < end) {
                        const int col = col_s[cur - col_base];
                        if (col >= k0 + 128) break;
                        if (col >= k0) {
                            const uint32_t byte = val_s[(cur >> 1) - val_base];
                            const int q = static_cast<int>(((byte >> ((cur & 1) * 4)) & 0xF) ^ 8) - 8;
                            const float sq = sr * static_cast<float>(q);
                            const int kk = col - kst;
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                                for (int i = 0; i < 2; ++i) {
                                    const int tok = 8 * nt + 2 * t + i;
                                    if (tok < M) {
                                        const uint16_t xv = reinterpret_cast<const uint16_t *>(
                                            xst + tok * C::XRS)[kk];
                                        acc[nt][2 * h + i] =
                                            fmaf(sq, bf16_bits_to_f32(xv), acc[nt][2 * h + i]);
                                    }
                                }
                        }
                        ++cur;
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
        __syncwarp();
        // all stages are consumed; hand the partials to the reduction below
        asm volatile("bar.sync 1, %0;" ::"n"(WARPS * 32) : "memory");
        float *red = reinterpret_cast<float *>(smem);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int tok = 8 * nt + 2 * t + (i & 1);
                const int row = (i < 2) ? r0 : r1;
                if (tok < MX) red[(s * MX + tok) * BN + row] = acc[nt][i];
            }
    }
    __syncthreads();
    if (*abort_flag) return;
    const float *red = reinterpret_cast<const float *>(smem);
    for (int idx = threadIdx.x; idx < M * BN; idx += C::THREADS) {
        const int m = idx / BN, r = idx % BN, n = n0 + r;
        if (n >= N) continue;
        float y = 0.f;
#pragma unroll
        for (int s = 0; s < S; ++s) y += red[(s * MX + m) * BN + r];
        if (p.Yf)
            p.Yf[size_t(m) * N + n] = y;
        else
            p.Y[size_t(m) * N + n] = __float2bfloat16_rn(y);
    }
}

template <int MX, int RT, int S, int GW, int STAGES>
mq_status run(const mq_weight *w, const void *X, int M, void *Y, cudaStream_t stream,
              float *partial) {
    const bool with_residual = partial == nullptr;
    using C = Cfg<MX, RT, S, GW, STAGES>;
    const DeviceWeight &d = weight_device(w);
    const MapSet *maps = weight_maps(w, C::BN, C::GS);
    if (!maps) return MQ_ERR_CUDA;
    int64_t tile_nnz = with_residual ? maps->max_tile_nnz : 0;
    int col_bytes = static_cast<int>((tile_nnz * 2 + 16 + 15) / 16 * 16);
    const int smem = C::smem_bytes(col_bytes);
    if (smem > 227 * 1024)
        return fail(MQ_ERR_UNSUPPORTED, "residual rows too dense for the decode kernel's "
                                        "shared-memory slice");
    auto kern = decode_kernel<MX, RT, S, GW, STAGES>;
    static int configured = 0;
    if (smem > configured) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) !=
            cudaSuccess)
            return fail(MQ_ERR_CUDA, "cudaFuncSetAttribute failed for the decode kernel");
        configured = 227 * 1024;
    }
    DecodeParams p;
    p.tm_w = maps->w;
    p.tm_sz = maps->sz;
    p.X = static_cast<const __nv_bfloat16 *>(X);
    p.Y = static_cast<__nv_bfloat16 *>(Y);
    p.Yf = partial;
    p.row_ptr = d.row_ptr;
    p.col = d.col;
    p.val = d.val;
    p.rscale = d.rscale;
    p.err = d.err;
    p.M = M;
    p.N = static_cast<int>(d.N);
    p.K = static_cast<int>(d.K);
    p.G = static_cast<int>(d.G);
    p.csr_col_bytes = col_bytes;
    p.with_residual = with_residual ? 1 : 0;
    dim3 grid(static_cast<unsigned>((d.N + C::BN - 1) / C::BN));
    kern<<<grid, C::THREADS, smem, stream>>>(p);
    cudaError_t e = cudaPeekAtLastError();
    if (e != cudaSuccess) return fail(MQ_ERR_CUDA, std::string("decode launch: ") + cudaGetErrorString(e));
    return MQ_OK;
}

}  // namespace

mq_status launch_decode(const mq_weight *w, const void *X, int M, void *Y, cudaStream_t stream,
                        float *partial) {
    if (M == 1) return run<1, 1, 8, 1, 4>(w, X, M, Y, stream, partial);
    if (M <= 8) return run<8, 2, 4, 1, 4>(w, X, M, Y, stream, partial);
    return run<16, 4, 2, 2, 3>(w, X, M, Y, stream, partial);
}

}  // namespace mq
