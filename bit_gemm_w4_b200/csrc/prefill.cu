// Prefill kernel: Y[M][N] = X[M][K] * W_hat^T on the 5th-generation tensor
// cores (tcgen05, TMEM, TMA), one fused pass for any M.
//
// MosaicQuant "Methodology" 3. (ZipperEngine): the sparse residual is
// integrated into the dense 4-bit GEMM kernel; dense compute, sparse
// compensation and the reduction-add run as one overlapped pipeline on
// tensor cores, CUDA cores and HBM.
//
// The kernel is persistent: one CTA per SM walks a contiguous range of
// 128-row x 128-token output tiles (consecutive tiles share their weight
// rows), each over all of K in stages of 64 columns; the pipelines below run
// on across tile boundaries, so a tile's first stages load and dequantize
// while the previous tile's last MMAs and epilogue finish. The weight is the MMA's A operand and lives in
// tensor memory, X is the B operand and streams through shared memory
// (D[row][token] = sum_k A[row][k] * X[token][k]), so the dequantized codes
// never touch shared memory: the only shared-memory traffic per stage is the
// TMA write of X and of the packed codes and the tensor core's read of X.
// Warp roles:
//   warp 0      TMA producer (one thread). One thread's copies complete one
//               after another, so few large copies are issued: the X tiles
//               [128 tokens][64] (128-byte swizzle) of CX consecutive stages
//               per copy (X seen as a 3D tensor [K/64][M][64]) into a ring of
//               XS slots, and the packed codes of four stages per copy
//               ([128 rows][32 words], 128-byte swizzle) into two slots.
//   warp 1      allocates tensor memory and issues tcgen05.mma (one thread).
//   warps 2..9  epilogue, two per tensor-memory lane quadrant (thread =
//               weight row), each owning 64 of the tile's 128 tokens.
//   warps 10..13 dequant, thread = weight row (its tensor-memory lane; scale
//               and zero words and the CSR entries come through L1): the 8
//               packed words of the row become its 64 exact bf16 codes
//               (q - z), stored into a tensor-memory operand slot with one
//               tcgen05.st. The row's residual entries of the stage are
//               scattered as exact bf16 codes q_r into a shared-memory tile
//               (128-byte swizzle, K-major) that is otherwise zero; when the
//               slot comes round again the warp zeroes its 32 rows of it.
// Tensor memory (512 columns): the group partials D[2] at 0 / 128, the
// residual accumulator R at 256 and four 32-column operand slots at 384, or,
// without a residual, eight operand slots at 256.
// Per stage the MMA thread issues 4 K=16 steps of the dense codes (A from
// tensor memory) into the TMEM buffer of the current 128-column group and,
// when any of the tile's rows has a residual entry in the stage, 4 steps of
// the residual tile (A from shared memory) into R. Every product is exact
// (integer codes times bf16 x) and accumulates in fp32. When a group's two
// stages are done the epilogue reads its partial sums and adds
// s[n][g] * partial to per-thread fp32 accumulators (the per-group rescale
// the fp16 group scales require; one scale per thread); the next group's
// MMAs run meanwhile into the other buffer. After a tile's last stage R is
// scaled by s_r[n] and added (the reduction-add) and the tile is stored as
// bf16, while the next tile's MMAs already run.
//
// W4A4 form (the pipeline's quantization stage in front, per-token int4
// activation codes): X is the int8 codes, each 8-column chunk already in the
// packed codes' k order, and a stage is 128 columns, one quantization group,
// so the X tile and the operand slot keep their sizes. The dequant warps write
// int8 codes q - z (a carry-free byte subtraction), the MMAs are kind::i8
// (s8 x s8 -> s32, exact) and every stage commits its own group partial; the
// epilogue converts the int32 sums to fp32 exactly, applies s[n][g] and s_r[n]
// and multiplies by the token's scale s_x when it stores Y.

#include "common.cuh"
#include "internal.h"
#include "kernels.h"

namespace mq {
namespace {

constexpr int BM = 128;  // tokens per tile (the MMA's N)
constexpr int BN = 128;  // weight rows per tile (the MMA's M, tensor-memory lanes)
constexpr int BK = 64;
constexpr int MAX_XS = 4;  // X ring slots (runtime XS <= MAX_XS)
constexpr int THREADS = 448;
constexpr int W_TMA = 0, W_MMA = 1, W_EPI0 = 2, W_DQ0 = 10;
constexpr int EPI_WARPS = 8, EPI_TOK = BM / 2;  // two warps per lane quadrant
constexpr int X_BYTES = BM * BK * 2;  // X tile
constexpr int T_BYTES = X_BYTES;      // one TMA stage
constexpr int PSLOT_BYTES = BN * 32 * 4;  // packed codes of up to four stages
constexpr int NPSLOT = 2;
constexpr int R_BYTES = BN * BK * 2;  // one residual code tile
constexpr int NSLOT = 4;   // operand slots with the residual (dense in TMEM, residual in smem)
constexpr int MAX_NS = 8;  // operand slots without it (R's columns hold four more)
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t T_D = 0, T_R = 256;  // column bases; the operand slots end the columns
constexpr uint32_t A_SLOT = 32;         // columns per operand slot
static_assert(T_BYTES % 1024 == 0 && R_BYTES % 1024 == 0, "1024-byte swizzle alignment");
static_assert(2 * T_BYTES >= BM * BN * 2, "the output tile is staged in the TMA ring");

struct PrefillParams {
    CUtensorMap tm_x;  // X [M][K] bf16 (box [128][64]) or int8 codes (box [128][128]), 128B swizzle
    CUtensorMap tm_w;  // qweight [N][K/8] u32, box [128][8]
    const int32_t *stage_ptr;   // residual groups per (tile, stage, quadrant)
    const uint32_t *stage_ent;
    const uint16_t *rscale;
    const uint32_t *sz;  // [N][Gp] scale | zero << 16
    const float *xscale;  // [M] per-token activation scales (W4A4), else NULL
    __nv_bfloat16 *Y;
    float *Yf;
    int *err;
    int M, N, K, G, Gp;
    int with_residual;
    int XS;       // X ring slots
    int CX;       // stages per X copy (2 or 4)
    int pw;       // words per row of a packed-code box (32, or 16 when K = 128)
    int m_tiles;  // token tiles; tile t covers rows (t / m_tiles) and tokens (t % m_tiles)
    int tiles;
    uint32_t bias;  // kBiasBf16, or kBiasI8 for the W4A4 form (held in a register)
};

struct SmemLayout {
    int pring, rtile, rflag, bars, tmem_slot, abort, total;
    __host__ __device__ SmemLayout(int XS, int CX, bool residual) {
        pring = XS * CX * T_BYTES;  // the X ring starts at 0
        rtile = pring + NPSLOT * PSLOT_BYTES;
        rflag = rtile + (residual ? NSLOT * R_BYTES : 0);
        bars = rflag + MAX_NS * 4 * 4;
        tmem_slot = bars + (2 * MAX_XS + MAX_NS + 2 * NPSLOT + 8) * 8;
        abort = tmem_slot + 16;
        total = abort + 16;
    }
};

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

// Instruction descriptors, both operands K-major, M = 128, N = 128:
// bf16 x bf16 -> fp32 (kind::f16), and s8 x s8 -> s32 (kind::i8, W4A4).
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
                            (static_cast<uint32_t>(BM >> 4) << 24);
constexpr uint32_t kIdescI8 = (2u << 4) | (1u << 7) | (1u << 10) |
                              (static_cast<uint32_t>(BN >> 3) << 17) | (static_cast<uint32_t>(BM >> 4) << 24);

// D[tmem] (+)= A[smem] * B[smem]^T, both K-major shared-memory tiles; A4
// selects the int8 kind (32 k per step) over bf16 (16 k per step).
template <bool A4>
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t accumulate) {
    if constexpr (A4)
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(kIdescI8), "r"(accumulate)
            : "memory");
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate)
            : "memory");
}

__device__ __forceinline__ void sts16(void *p, uint16_t v) {
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(smem_u32(p)), "h"(v) : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T: A is M x 16 bf16 in tensor memory (lane =
// row, two codes per 32-bit column), B an N x 16 K-major shared-memory tile.
template <bool A4>
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                       uint32_t accumulate) {
    if constexpr (A4)
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
            "r"(a_tmem), "l"(bdesc), "r"(kIdescI8), "r"(accumulate)
            : "memory");
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
            "r"(a_tmem), "l"(bdesc), "r"(kIdesc), "r"(accumulate)
            : "memory");
}

// An int32 of magnitude below 2^22 as fp32, exactly, with two adds: placed in
// the mantissa of 1.5 * 2^23 (ulp 1) and the bias taken off again.
__device__ __forceinline__ float small_int_to_f32(uint32_t bits) {
    return __int_as_float(static_cast<int>(bits) + 0x4B400000) - 12582912.0f;
}

// 32 lanes x 32 columns of 32-bit values: thread i writes lane (base + i).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
        "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
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

// NS operand slots, handed over in pairs: 4 when the residual is fused (its
// accumulator takes tensor-memory columns 256..383), else 8.
// A4: the W4A4 form. X is int8 activation codes (each 8-column chunk in the
// packed codes' k order), a stage is 128 columns (one quantization group, the
// same 16 KB X tile and 32 tensor-memory columns as 64 bf16 columns), the
// dequant warps write int8 codes q - z, the MMAs are kind::i8 into int32, and
// the epilogue scales by s[n][g], s_r[n] and the token's s_x.
template <int NS, bool A4>
__global__ void __launch_bounds__(THREADS, 1) prefill_kernel(const __grid_constant__ PrefillParams p) {
    static_assert(NS == NSLOT || NS == MAX_NS, "operand slot count");
    constexpr int SK = A4 ? 128 : BK;  // K columns per stage
    constexpr int WPS = SK / 8;        // packed words per row and stage
    constexpr int NP = NS / 2;                         // slot pairs
    constexpr int NS_LOG = NS == 8 ? 3 : 2;
    constexpr uint32_t T_A = TMEM_COLS - NS * A_SLOT;  // first operand slot column
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const bool res = NS == NSLOT && p.with_residual != 0;
    const SmemLayout L(p.XS, p.CX, res);
    const int XS = p.XS, CX = p.CX;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nk = p.K / SK;     // stages per tile (even: K is a multiple of 256 for A4)
    const int nls = p.K / BK;    // residual list stages per tile (64 columns each)
    const int G = p.G, Gp = p.Gp;
    // this CTA's tiles
    const int t_begin = static_cast<int>(static_cast<long long>(blockIdx.x) * p.tiles / gridDim.x);
    const int t_end = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * p.tiles / gridDim.x);

    volatile uint32_t *rflag = reinterpret_cast<volatile uint32_t *>(smem + L.rflag);  // [NS][4]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.bars);
    uint64_t *full = bars;                 // [XS] X copy landed
    uint64_t *empty = bars + MAX_XS;       // [XS] MMAs reading the X copy done
    // operand slots go back and forth in pairs (one 128-column group)
    uint64_t *bready = bars + 2 * MAX_XS;   // [NP] operand slot pair written
    uint64_t *bempty = bready + MAX_NS / 2;  // [NP] MMAs reading the slot pair done
    uint64_t *dfull = bempty + MAX_NS / 2;   // [2] group partial ready in TMEM
    uint64_t *dempty = dfull + 2;          // [2] epilogue done with the TMEM buffer
    uint64_t *rfull = dempty + 2;          // every MMA of the tile complete
    uint64_t *rempty = rfull + 1;          // epilogue done with the tile's R
    uint64_t *pfull = rempty + 1;          // [NPSLOT] packed codes landed
    uint64_t *pempty = pfull + NPSLOT;     // [NPSLOT] dequant done with the packed codes
    static_assert(NPSLOT == 2, "slot arithmetic below uses shifts");
    const int spl = p.pw / WPS;            // stages per packed-code load
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L.tmem_slot);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L.abort);

    if (threadIdx.x == 0) {
        for (int s = 0; s < XS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < NP; ++b) {
            mbar_init(&bready[b], 4);
            mbar_init(&bempty[b], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&dfull[b], 1);
            mbar_init(&dempty[b], EPI_WARPS);
        }
        mbar_init(rfull, 1);
        mbar_init(rempty, EPI_WARPS);
        for (int b = 0; b < NPSLOT; ++b) {
            mbar_init(&pfull[b], 1);
            mbar_init(&pempty[b], 4);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (res) {
        // the residual code tiles start zeroed; afterwards only written entries are cleared
        for (int i = threadIdx.x; i < NSLOT * R_BYTES / 16; i += THREADS)
            reinterpret_cast<uint4 *>(smem + L.rtile)[i] = make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async();
    }
    if (warp == W_MMA) tmem_alloc(tmem_slot, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == W_TMA) {
        // ---------------------------------------------------------- producer
        // Slot indices and phases advance as counters: a lone thread would
        // pay the full latency of every integer division by a runtime value.
        if (lane == 0) {
            prefetch_tensormap(&p.tm_x);
            prefetch_tensormap(&p.tm_w);
            int xs = 0, xround = 0;  // X slot of the next copy, times the ring wrapped
            int pc = 0, xc = 0;      // packed-code and X copies issued
            bool ok = true;
            for (int t = t_begin; ok && t < t_end; ++t) {
                const int n0 = (t / p.m_tiles) * BN, m0 = (t % p.m_tiles) * BM;
                for (int i = 0, pi = 0, xi = 0; i < nk; ++i) {
                    if (pi == 0) {
                        const int ps = pc & (NPSLOT - 1);
                        if (pc >= NPSLOT && !mbar_wait(&pempty[ps], ((pc >> 1) - 1) & 1, p.err,
                                                       kErrWaitEmpty, abort_flag)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&pfull[ps], BN * p.pw * 4);
                        tma_load_2d(smem + L.pring + ps * PSLOT_BYTES, &p.tm_w, &pfull[ps], i * WPS, n0);
                        ++pc;
                    }
                    if (++pi == spl) pi = 0;
                    if (xi == 0) {
                        if (xround > 0 &&
                            !mbar_wait(&empty[xs], (xround - 1) & 1, p.err, kErrWaitEmpty, abort_flag)) {
                            ok = false;
                            break;
                        }
                        // CX tiles; past the end of K the box reads zeros (and still
                        // counts its full size)
                        mbar_arrive_expect_tx(&full[xs], CX * T_BYTES);
                        tma_load_3d(smem + xs * (CX * T_BYTES), &p.tm_x, &full[xs], 0, m0, i);
                        ++xc;
                        if (++xs == XS) {
                            xs = 0;
                            ++xround;
                        }
                    }
                    if (++xi == CX) xi = 0;
                }
            }
            // no copy may still be in flight when the CTA exits: wait for the last
            // XS X copies and the last two packed-code copies
            for (int j = 0, s = xs, r = xround; j < XS && j < xc; ++j) {
                if (--s < 0) {
                    s = XS - 1;
                    --r;
                }
                mbar_wait(&full[s], r & 1, p.err, kErrWaitDrain, abort_flag);
            }
            for (int j = max(0, pc - NPSLOT); j < pc; ++j)
                mbar_wait(&pfull[j & (NPSLOT - 1)], (j >> 1) & 1, p.err, kErrWaitDrain, abort_flag);
        }
    } else if (warp == W_MMA) {
        // ---------------------------------------------------------- MMA issue
        if (lane == 0) {
            int it = 0, gg0 = 0;
            int xs = 0, xround = 0;  // X slot being read, times the ring wrapped
            bool ok = true;
            for (int t = t_begin, j = 0; ok && t < t_end; ++t, ++j, gg0 += G) {
                // two stages (one operand slot pair; one group, or two for A4) per step
                for (int i = 0, xi = 0; i < nk; i += 2, it += 2) {
                    const int pp = (it >> 1) & (NP - 1);
                    int gg = gg0 + (i >> 1), b = gg & 1;
                    if (!A4 && gg >= 2 &&
                        !mbar_wait(&dempty[b], ((gg >> 1) - 1) & 1, p.err, kErrWaitMma, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if ((xi == 0 && !mbar_wait(&full[xs], xround & 1, p.err, kErrWaitFull, abort_flag)) ||
                        !mbar_wait(&bready[pp], (it >> NS_LOG) & 1, p.err, kErrWaitFull, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if constexpr (A4) {  // each stage is a group of its own
                            gg = gg0 + i + h;
                            b = gg & 1;
                            if (gg >= 2 && !mbar_wait(&dempty[b], ((gg >> 1) - 1) & 1, p.err,
                                                      kErrWaitMma, abort_flag)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                        }
                        const int a = (it + h) & (NS - 1);
                        const uint64_t xd = sw128_desc(smem_u32(smem + (xs * CX + xi + h) * T_BYTES));
                        const uint32_t at = tmem + T_A + a * A_SLOT;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_ts<A4>(tmem + T_D + b * BM, at + 8 * kk, xd + 2 * kk,
                                       ((A4 ? 0 : h) | kk) ? 1u : 0u);
                        // stage 0 always runs, so R is initialized; it may be
                        // overwritten once the epilogue has read the previous tile's R
                        if (res && (rflag[4 * a] | rflag[4 * a + 1] | rflag[4 * a + 2] | rflag[4 * a + 3])) {
                            if (i + h == 0 && j > 0) {
                                if (!mbar_wait(rempty, (j - 1) & 1, p.err, kErrWaitMma, abort_flag)) {
                                    ok = false;
                                    break;
                                }
                                tc_fence_after();
                            }
                            const uint64_t rd = sw128_desc(smem_u32(smem + L.rtile + a * R_BYTES));
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                mma_ss<A4>(tmem + T_R, rd + 2 * kk, xd + 2 * kk, ((i + h) | kk) ? 1u : 0u);
                        }
                        if constexpr (A4) mma_commit(&dfull[b]);
                    }
                    if (!ok) break;
                    xi += 2;
                    if (xi == CX || i + 2 == nk) {
                        mma_commit(&empty[xs]);
                        xi = 0;
                        if (++xs == XS) {
                            xs = 0;
                            ++xround;
                        }
                    }
                    mma_commit(&bempty[pp]);
                    if constexpr (!A4) mma_commit(&dfull[b]);
                }
                // the epilogue waits for each tile's completion with the tile's parity,
                // so it must have taken the previous one first
                if (ok && !res && j > 0 &&
                    !mbar_wait(rempty, (j - 1) & 1, p.err, kErrWaitMma, abort_flag))
                    ok = false;
                if (ok) mma_commit(rfull);
                if (ok && t + 1 == t_end)  // every MMA has finished before TMEM is released
                    mbar_wait(rfull, j & 1, p.err, kErrWaitDrain, abort_flag);
            }
        }
    } else if (warp >= W_DQ0) {
        // ---------------------------------------------------------- dequant
        const int q = warp & 3;        // tensor-memory lane quadrant
        const int n = 32 * q + lane;   // weight row within the tile (= lane)
        const uint32_t tl = tmem + (static_cast<uint32_t>(32 * q) << 16) + T_A;
        int it = 0, pc = 0;
        bool ok = true;
        for (int t = t_begin; ok && t < t_end; ++t) {
            const int row = (t / p.m_tiles) * BN + n;
            const bool valid = row < p.N;
            const uint32_t *szrow = p.sz + static_cast<size_t>(row) * Gp;
            const int32_t *gptr = res ? p.stage_ptr + (static_cast<size_t>(t / p.m_tiles) * nls) * 4 + q : nullptr;
            // The residual entries are requested ahead of use: a stage's group
            // bounds two stages early, its first entry per lane one stage early,
            // so neither global load sits on the path from the waits to the MMA.
            // A stage holds NSUB of the 64-column lists (two for A4's 128 columns).
            constexpr int NSUB = A4 ? 2 : 1;
            int na[NSUB][2], nb[NSUB][2];
            uint32_t nv[NSUB];
#pragma unroll
            for (int u = 0; u < NSUB; ++u) {
                na[u][0] = na[u][1] = nb[u][0] = nb[u][1] = 0;
                nv[u] = 0u;
                if (res) {
                    na[u][0] = __ldg(gptr + 4 * u);
                    na[u][1] = __ldg(gptr + 4 * u + 1);
                    if (na[u][0] + lane < na[u][1]) nv[u] = __ldg(p.stage_ent + na[u][0] + lane);
                    if (nk > 1) {
                        nb[u][0] = __ldg(gptr + 4 * (NSUB + u));
                        nb[u][1] = __ldg(gptr + 4 * (NSUB + u) + 1);
                    }
                }
            }
            // scale / zero words four groups per 16-byte load (rows are padded to a
            // multiple of four groups), the next four requested when these are
            // taken, so the loads are few and their latency is hidden
            uint4 sz4 = make_uint4(0u, 0u, 0u, 0u);
            uint4 sz4_next = valid ? __ldg(reinterpret_cast<const uint4 *>(szrow)) : sz4;
            uint32_t szw = 0u;
            constexpr int SPG = A4 ? 1 : 2;  // stages per quantization group
            for (int i = 0, pi = 0; i < nk; ++i, ++it) {
                const int a = it & (NS - 1), ps = pc & (NPSLOT - 1);
                if (i % SPG == 0) {
                    const int g = i / SPG;
                    if ((g & 3) == 0) {
                        sz4 = sz4_next;
                        if (valid && g + 4 < Gp)
                            sz4_next = __ldg(reinterpret_cast<const uint4 *>(szrow + g + 4));
                    }
                    szw = (g & 2) ? ((g & 1) ? sz4.w : sz4.z) : ((g & 1) ? sz4.y : sz4.x);
                }
                // this warp's residual groups of the stage and their first entries per lane
                int g[NSUB][2];
                uint32_t v0[NSUB];
#pragma unroll
                for (int u = 0; u < NSUB; ++u) {
                    g[u][0] = na[u][0];
                    g[u][1] = na[u][1];
                    v0[u] = nv[u];
                    if (res) {
                        na[u][0] = nb[u][0];
                        na[u][1] = nb[u][1];
                        nv[u] = (i + 1 < nk && na[u][0] + lane < na[u][1])
                                    ? __ldg(p.stage_ent + na[u][0] + lane) : 0u;
                        if (i + 2 < nk) {
                            nb[u][0] = __ldg(gptr + 4 * (NSUB * (i + 2) + u));
                            nb[u][1] = __ldg(gptr + 4 * (NSUB * (i + 2) + u) + 1);
                        }
                    }
                }
                if ((pi == 0 &&
                     !mbar_wait_warp(&pfull[ps], (pc >> 1) & 1, p.err, kErrWaitFull, abort_flag)) ||
                    ((it & 1) == 0 && it >= NS &&
                     !mbar_wait_warp(&bempty[(it >> 1) & (NP - 1)], ((it >> NS_LOG) - 1) & 1, p.err,
                                     kErrWaitMma, abort_flag))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t z = static_cast<uint32_t>(half_bits_to_f32(szw >> 16));
                // this stage's 16-byte chunks of the row (128-byte swizzle when pw = 32):
                // two for 64 bf16 columns, four for 128 int8 columns
                const uint8_t *prow = smem + L.pring + ps * PSLOT_BYTES + n * (p.pw * 4);
                const int c0 = (WPS / 4) * pi, sw = (p.pw == 32) ? (n & 7) : 0;
                uint32_t words[WPS];
#pragma unroll
                for (int u = 0; u < WPS / 4; ++u) {
                    const uint4 wv = lds128(prow + (((c0 + u) ^ sw) << 4));
                    words[4 * u] = wv.x;
                    words[4 * u + 1] = wv.y;
                    words[4 * u + 2] = wv.z;
                    words[4 * u + 3] = wv.w;
                }
                if (++pi == spl || i == nk - 1) {
                    pi = 0;
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&pempty[ps]);
                    ++pc;
                }
                uint32_t codes[32];
                const uint32_t bias = p.bias;
                if constexpr (A4) {
                    // a word's low nibbles are its columns in positions 0-3 of the
                    // chunk's code order, the high nibbles positions 4-7: one
                    // tensor-memory column of four int8 codes q - z each
                    const uint32_t zz = z * 0x01010101u;
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        codes[2 * c] = codes_minus_zero_r(words[c], zz, bias);
                        codes[2 * c + 1] = codes_minus_zero_r(words[c] >> 4, zz, bias);
                    }
                } else {
                    const uint32_t zz = (0x4300u | z) * 0x00010001u;  // bf16x2 (128 + z)
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        // pair j of word c holds columns (8c + 2j, 8c + 2j + 1)
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj)
                            codes[4 * c + jj] = bf16x2_sub(mask_or<0x000F000Fu>(words[c] >> (4 * jj), bias), zz);
                    }
                }
                tmem_st32(tl + a * A_SLOT, codes);
                bool has = false;
                if (res) {
                    uint8_t *rt = smem + L.rtile + a * R_BYTES;
                    // zero this warp's 32 rows of the slot (the stage that used it
                    // NSLOT stages ago may have left entries there), then write the
                    // stage's entries; an entry word holds row, column and the bf16
                    // code ready to store
                    if (it >= NSLOT) {
                        uint8_t *rq = rt + 32 * q * 128;
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            sts128(rq + 512 * k + 16 * lane, make_uint4(0u, 0u, 0u, 0u));
                    }
                    __syncwarp();
                    int cnt = 0;
#pragma unroll
                    for (int u = 0; u < NSUB; ++u) {
                        cnt += g[u][1] - g[u][0];
                        for (int e = g[u][0] + lane; e < g[u][1]; e += 32) {
                            const uint32_t v = (e == g[u][0] + lane) ? v0[u] : __ldg(p.stage_ent + e);
                            const int r = v & 127, c = ((v >> 8) & 63) + 64 * u;
                            if constexpr (A4) {
                                // an int8 code goes to its column's position in the
                                // chunk's code order
                                const int cp = (c & ~7) | ((c & 3) << 1) | ((c >> 2) & 1);
                                const int q8 = static_cast<int>(bf16_bits_to_f32(v >> 16));
                                sts_u8(rt + r * 128 + (((cp >> 4) ^ (r & 7)) << 4) + (cp & 15),
                                       static_cast<uint8_t>(q8 & 0xFF));
                            } else {
                                sts16(rt + r * 128 + (((c >> 3) ^ (r & 7)) << 4) + (c & 7) * 2,
                                      static_cast<uint16_t>(v >> 16));
                            }
                        }
                    }
                    // stage 0 of a tile always runs its residual MMAs (R starts there)
                    has = cnt > 0 || i == 0;
                    fence_proxy_async();  // the tile is read by the tensor core
                }
                if (lane == 0) rflag[4 * a + q] = has ? 1u : 0u;
                if (it & 1) {  // the pair's second stage: hand the pair over
                    tmem_st_wait();  // both stages' codes are in tensor memory
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bready[(it >> 1) & (NP - 1)]);
                }
            }
        }
    } else {
        // ---------------------------------------------------------- epilogue
        const int q = warp & 3;                            // tensor-memory lane quadrant
        const int tb = ((warp - W_EPI0) >> 2) * EPI_TOK;  // first token of this warp
        const int n = 32 * q + lane;                       // weight row within the tile
        const uint32_t tl = tmem + (static_cast<uint32_t>(32 * q) << 16) + tb;
        int gg = 0;
        bool ok = true;
        for (int t = t_begin, j = 0; ok && t < t_end; ++t, ++j) {
            const int n0 = (t / p.m_tiles) * BN, m0 = (t % p.m_tiles) * BM;
            const int row = n0 + n;
            const bool valid = row < p.N;
            float acc[EPI_TOK];
#pragma unroll
            for (int c = 0; c < EPI_TOK; ++c) acc[c] = 0.f;
            for (int g = 0; g < G; ++g, ++gg) {
                const int b = gg & 1;
                const uint32_t szw = valid ? __ldg(p.sz + static_cast<size_t>(row) * Gp + g) : 0u;
                if (!mbar_wait_warp(&dfull[b], (gg >> 1) & 1, p.err, kErrWaitMma, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float sc = half_bits_to_f32(szw & 0xFFFFu);
#pragma unroll
                for (int c0 = 0; c0 < EPI_TOK; c0 += 32) {
                    float v[32];
                    tmem_ld32(tl + T_D + b * BM + c0, v);
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        // A4: an exact int32 group sum, at most 128 * 15 * 8 in magnitude
                        const float d = A4 ? small_int_to_f32(__float_as_uint(v[c])) : v[c];
                        acc[c0 + c] = fmaf(sc, d, acc[c0 + c]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&dempty[b]);
            }
            if (!ok || !mbar_wait_warp(rfull, j & 1, p.err, kErrWaitMma, abort_flag)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (res) {
                const float sr = valid ? half_bits_to_f32(__ldg(p.rscale + row)) : 0.f;
#pragma unroll
                for (int c0 = 0; c0 < EPI_TOK; c0 += 32) {
                    float v[32];
                    tmem_ld32(tl + T_R + c0, v);
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        // A4: an exact int32 sum of at most K products of magnitude 64
                        const float d = A4 ? small_int_to_f32(__float_as_uint(v[c])) : v[c];
                        acc[c0 + c] = fmaf(sr, d, acc[c0 + c]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(rempty);
            // a warp writes 32 consecutive outputs of one token per store
            if (valid) {
                const int nt = min(EPI_TOK, p.M - (m0 + tb));
                if (p.Yf) {
                    float *yc = p.Yf + static_cast<size_t>(m0 + tb) * p.N + row;
#pragma unroll
                    for (int c = 0; c < EPI_TOK; ++c)
                        if (c < nt) yc[static_cast<size_t>(c) * p.N] = acc[c];
                } else if (A4) {
                    // Y = s_x[token] * (sum_g s_g D_g + s_r R); the token's scale is
                    // the same for every lane of the warp
                    __nv_bfloat16 *yc = p.Y + static_cast<size_t>(m0 + tb) * p.N + row;
                    const float *xs = p.xscale + m0 + tb;
#pragma unroll
                    for (int c = 0; c < EPI_TOK; ++c)
                        if (c < nt) yc[static_cast<size_t>(c) * p.N] = __float2bfloat16_rn(acc[c] * __ldg(xs + c));
                } else {
                    __nv_bfloat16 *yc = p.Y + static_cast<size_t>(m0 + tb) * p.N + row;
#pragma unroll
                    for (int c = 0; c < EPI_TOK; ++c)
                        if (c < nt) yc[static_cast<size_t>(c) * p.N] = __float2bfloat16_rn(acc[c]);
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

namespace {

// The shared launch path: A4 takes int8 activation codes and their per-token
// scales in place of bf16 X.
template <bool A4>
mq_status launch_prefill_impl(const mq_weight *w, const void *X, const float *xscale, int64_t M,
                              void *Y, cudaStream_t stream, float *partial) {
    const DeviceWeight &d = weight_device(w);
    if (M > (int64_t(1) << 23)) return fail(MQ_ERR_UNSUPPORTED, "prefill kernel: M above 2^23");
    if (A4 && d.K % 256) return fail(MQ_ERR_UNSUPPORTED, "W4A4 prefill kernel: K must be a multiple of 256");
    const PrefillMaps *pm = prefill_maps(w);
    if (!pm) return MQ_ERR_CUDA;
    PrefillParams p;
    p.with_residual = (partial == nullptr && d.nnz > 0) ? 1 : 0;
    // four stages per X copy; two when the residual tiles take their share of
    // shared memory (a deeper ring of smaller copies)
    p.CX = p.with_residual ? 2 : 4;
    if (!(A4 ? encode_codes_map(&p.tm_x, X, M, d.K, p.CX) : encode_x_map(&p.tm_x, X, M, d.K, p.CX)))
        return fail(MQ_ERR_CUDA, "cuTensorMapEncodeTiled failed for X");
    p.xscale = xscale;
    p.tm_w = pm->w;
    p.pw = pm->pw;
    p.stage_ptr = d.stage_ptr;
    p.stage_ent = d.stage_ent;
    p.rscale = d.rscale;
    p.sz = d.sz;
    p.Y = static_cast<__nv_bfloat16 *>(Y);
    p.Yf = partial;
    p.err = d.err;
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(d.N);
    p.K = static_cast<int>(d.K);
    p.G = static_cast<int>(d.G);
    p.Gp = static_cast<int>(d.Gp);
    p.bias = A4 ? kBiasI8 : kBiasBf16;
    p.m_tiles = static_cast<int>((M + BM - 1) / BM);
    const int64_t tiles = ((d.N + BN - 1) / BN) * static_cast<int64_t>(p.m_tiles);
    if (tiles > (int64_t(1) << 30)) return fail(MQ_ERR_UNSUPPORTED, "prefill kernel: too many tiles");
    p.tiles = static_cast<int>(tiles);
    // the deepest X ring that fits
    const int budget = 227 * 1024 - 1024;
    p.XS = 0;
    for (int xs = MAX_XS; xs >= 2 && !p.XS; --xs)
        if (SmemLayout(xs, p.CX, p.with_residual != 0).total <= budget) p.XS = xs;
    if (!p.XS) return fail(MQ_ERR_UNSUPPORTED, "prefill kernel: shared memory");
    const int smem = SmemLayout(p.XS, p.CX, p.with_residual != 0).total + 1024;
    static bool configured[64] = {};
    static int sms[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return fail(MQ_ERR_CUDA, "cudaGetDevice failed");
    if (dev < 0 || dev >= 64) return fail(MQ_ERR_UNSUPPORTED, "device ordinal above 63");
    if (!configured[dev]) {
        if (cudaFuncSetAttribute(prefill_kernel<NSLOT, A4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 227 * 1024) != cudaSuccess ||
            cudaFuncSetAttribute(prefill_kernel<MAX_NS, A4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 227 * 1024) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            sms[dev] <= 0)
            return fail(MQ_ERR_CUDA, "prefill kernel: device setup failed");
        configured[dev] = true;
    }
    // one CTA per SM (its shared memory and 512 TMEM columns allow no second)
    const int grid = static_cast<int>(std::min<int64_t>(tiles, sms[dev]));
    if (p.with_residual)
        prefill_kernel<NSLOT, A4><<<grid, THREADS, smem, stream>>>(p);
    else
        prefill_kernel<MAX_NS, A4><<<grid, THREADS, smem, stream>>>(p);
    cudaError_t e = cudaPeekAtLastError();
    if (e != cudaSuccess)
        return fail(MQ_ERR_CUDA, std::string("prefill launch: ") + cudaGetErrorString(e));
    return MQ_OK;
}

}  // namespace

mq_status launch_prefill(const mq_weight *w, const void *X, int64_t M, void *Y,
                         cudaStream_t stream, float *partial) {
    return launch_prefill_impl<false>(w, X, nullptr, M, Y, stream, partial);
}

mq_status launch_prefill_a4(const mq_weight *w, const int8_t *codes, const float *xscale, int64_t M,
                            void *Y, cudaStream_t stream) {
    return launch_prefill_impl<true>(w, codes, xscale, M, Y, stream, nullptr);
}

}  // namespace mq
