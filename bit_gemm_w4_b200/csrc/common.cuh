// Device helpers for sm_100a: mbarriers with bounded waits, TMA tiled and
// bulk copies, legacy mma.sync, bf16x2 arithmetic. Inline PTX only.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "kernels.h"

namespace mq {

// Error codes a kernel leaves in the handle's device error word.
enum DeviceError : int {
    kErrNone = 0,
    kErrWaitFull = 1,    // a consumer gave up waiting for a pipeline stage
    kErrWaitEmpty = 2,   // the producer gave up waiting for a free stage
    kErrWaitCsr = 3,     // the residual slice never arrived
    kErrWaitMma = 4,     // a tensor-core commit never arrived
    kErrWaitDrain = 5,   // copies still in flight at exit
    kErrTmem = 6,        // tensor-memory allocation failed
};

// ~1 s at 2 GHz: far beyond any legitimate wait, short enough to keep the
// context usable if a pipeline is ever broken.
constexpr long long kWaitCycles = 2000000000LL;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
            smem_u32(bar)),
        "r"(bytes)
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete. A tight try_wait
// loop (the instruction itself suspends the thread for a while) that looks
// at the clock only every 256 polls; gives up after `limit` cycles
// (kWaitCycles unless a self-test asks for less) or once *abort is set,
// records `code` in *err (global or shared memory) and sets *abort so that
// every later wait of the block returns immediately.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, int *err, int code,
                                          volatile int *abort, long long limit = kWaitCycles) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if (clock64() - t0 > limit) {
            atomicCAS(err, 0, code);
            *abort = 1;
            return false;
        }
    }
}

// One lane of the warp polls; the rest wait at __syncwarp, which orders the
// data the completed phase made visible to lane 0 before their reads.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t *bar, uint32_t parity, int *err, int code,
                                               volatile int *abort) {
    int ok = 1;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, err, code, abort) ? 1 : 0;
    __syncwarp();
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// ---------------------------------------------------------------- TMA
// 3D tiled load of a box into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int x, int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
        : "memory");
}

// 2D tiled load of a box into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- streaming loads
// 16 bytes from HBM that no kernel reuses: read-only path, no L1 allocation.
__device__ __forceinline__ uint4 ldg_stream(const uint32_t *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ldg_nc(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

// ---------------------------------------------------------------- L2 prefetch
// Share `part` of `parts` of each region of pf, requested into L2 with bulk
// prefetches (asynchronous, nothing waits for them).
__device__ __forceinline__ void l2_prefetch_share(const L2Prefetch &pf, int part, int parts) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const long long bytes = pf.bytes[r];
        if (bytes <= 0) continue;
        const long long chunk = ((bytes + parts - 1) / parts + 15) & ~15ll;
        const long long off = part * chunk;
        if (off >= bytes) continue;
        long long n = bytes - off < chunk ? bytes - off : chunk;
        const char *ptr = static_cast<const char *>(pf.p[r]) + off;
        while (n > 0) {
            const unsigned piece = static_cast<unsigned>(n < (1ll << 20) ? n : (1ll << 20));
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(ptr), "r"(piece) : "memory");
            ptr += piece;
            n -= piece;
        }
    }
}

// ---------------------------------------------------------------- cp.async, clusters, PDL
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
                 : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_all;" ::: "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile(
        "barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
            : "memory");
}

__device__ __forceinline__ float ld_dsmem_f32(const void *local, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
                 : "=r"(remote)
                 : "r"(smem_u32(local)), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}

__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src)
                 : "memory");
}

__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}

// Waits until at most N committed cp.async groups of this thread are pending.
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Programmatic dependent launch: wait for the previous grid's results / let
// the next grid start its prologue.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" :::);
}

// ---------------------------------------------------------------- CSR
// First index in [lo, hi) whose column is >= key (columns ascend in a row).
__device__ __forceinline__ int col_lower_bound(const uint16_t *colp, int coff, int lo, int hi,
                                               int key) {
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (static_cast<int>(colp[mid - coff]) < key)
            lo = mid + 1;
        else
            hi = mid;
    }
    return lo;
}


// ---------------------------------------------------------------- math
// The bias words of the code conversions, bf16x2 (128, 128) and the int8
// sign-bias bytes. Kernels take them as launch parameters: held in a
// register, (w & mask) | bias is one LOP3, where a second 32-bit immediate
// would cost a second one.
constexpr uint32_t kBiasBf16 = 0x43004300u;
constexpr uint32_t kBiasI8 = 0x80808080u;

template <uint32_t kMask>
__device__ __forceinline__ uint32_t mask_or(uint32_t w, uint32_t bias) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(w), "n"(kMask), "r"(bias));
    return d;
}

// Four int8 bytes q - z from the low nibble of each byte of w, with the
// sign-bias word in a register (kBiasI8): (nibble | 0x80) - z never borrows
// across bytes (z <= 15), and ^ 0x80 restores the sign; two LOP3s and one
// add.
__device__ __forceinline__ uint32_t codes_minus_zero_r(uint32_t w, uint32_t zz4, uint32_t bias8) {
    return (mask_or<0x0F0F0F0Fu>(w, bias8) - zz4) ^ bias8;
}

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// D = A * B + C, m16n8k16, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1, const float (&c)[4]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%11,%12,%13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]),
          "f"(c[2]), "f"(c[3]));
}

// D = A * B + C, m16n8k32, s8 inputs, s32 accumulate (exact).
__device__ __forceinline__ void mma_s8_16832(int (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                             uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b16) {
    return __uint_as_float(b16 << 16);
}

__device__ __forceinline__ float half_bits_to_f32(uint32_t h) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(h & 0xFFFFu)));
}

__device__ __forceinline__ uint32_t lds_u16(const void *p) {
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(smem_u32(p)));
    return v;
}

__device__ __forceinline__ void sts_u8(void *p, uint32_t v) {
    asm volatile("st.shared.u8 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}

__device__ __forceinline__ void sts_u16(void *p, uint32_t v) {
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(smem_u32(p)), "h"(static_cast<unsigned short>(v))
                 : "memory");
}

__device__ __forceinline__ void sts128(void *p, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(smem_u32(p)), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ uint4 lds128(const void *p) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(smem_u32(p)));
    return v;
}

// ---- shared by the streaming decode kernels

// bf16x2 (128 + q_lo, 128 + q_hi) for the nibbles at bits [0,4) and [16,20)
// of w, with the bias word in a register: one LOP3.
__device__ __forceinline__ uint32_t nib_pair(uint32_t w, uint32_t bias) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(w), "n"(0x000F000F), "r"(bias));
    return d;
}

// bf16x2 (128 + z, 128 + z) from a scale/zero word (fp16 s low, fp16 z high,
// z an integer 0..15): adding 1024 in fp16 puts z in the low mantissa bits.
__device__ __forceinline__ uint32_t zero_pair(uint32_t szw) {
    uint32_t h;
    asm("add.rn.f16x2 %0, %1, %2;" : "=r"(h) : "r"(szw), "r"(0x64006400u));
    return (__byte_perm(h, 0, 0x3232) & 0x000F000Fu) | 0x43004300u;
}

// cp.async of 16 bytes, or of none (zero fill) when `live` is false.
__device__ __forceinline__ void cp_async16_if(void *dst, const void *src, bool live) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
                 "r"(live ? 16 : 0)
                 : "memory");
}

// D += A * B, m16n8k16 bf16 -> fp32, as a pure function of its operands (not
// volatile), so that the compiler may interleave independent items.
__device__ __forceinline__ void mma_pure(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// scale/zero row stride in shared memory (words): Gp, or Gp + 4, whichever
// is an odd multiple of four
__host__ __device__ inline int sz_stride(int Gp) { return ((Gp >> 2) & 1) ? Gp : Gp + 4; }

// 16-byte chunk c of a 128-column group of X sits at xchunk(c) in shared
// memory, so that a warp's fragment loads touch distinct banks.
__device__ __forceinline__ int xchunk(int c) { return c ^ (((c >> 3) & 1) << 1); }

// Byte offset in a fragment tile of the code at row r (0..15), column c of a
// 128-column group: thread (g = r % 8, t = c / 32) holds it in register
// (r / 8) + 2 * ((c % 4) / 2), half c % 2 (the m16n8k16 A layout under the
// packed codes' k order, where k-step (c % 32) / 4 covers column c).
__device__ __forceinline__ int tile_pos(int r, int c) {
    return (((r & 7) * 4 + (c >> 5)) * 4 + (r >> 3) + 2 * ((c & 3) >> 1)) * 4 + (c & 1) * 2;
}

}  // namespace mq
