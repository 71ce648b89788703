// common.cuh -- shared device helpers and constants of libmoeq (sm_100a).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "moeq.h"

namespace moeq {

// ------------------------------------------------------------- tracing --
// Build with -DMOEQ_TRACE to record %globaltimer stamps per CTA at phase
// boundaries (g_trace[kernel][cta][point]); otherwise these compile to nothing.
#ifdef MOEQ_TRACE
__device__ unsigned long long g_trace[4][1024][16];
#define MOEQ_STAMP(K, I)                                                               \
    do {                                                                              \
        if (threadIdx.x == 0) {                                                       \
            unsigned long long t_;                                                    \
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                    \
            g_trace[K][blockIdx.x][I] = t_;                                           \
        }                                                                             \
    } while (0)
#define MOEQ_STAMP_MAX(K, I)                                                           \
    do {                                                                              \
        if ((threadIdx.x & 31) == 0) {                                                \
            unsigned long long t_;                                                    \
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                    \
            atomicMax(&g_trace[K][blockIdx.x][I], t_);                                \
        }                                                                             \
    } while (0)
#else
#define MOEQ_STAMP(K, I) do { } while (0)
#define MOEQ_STAMP_MAX(K, I) do { } while (0)
#endif

// ---------------------------------------------------------------- shapes --
constexpr int kGroup = 64;       // codes per affine group (scale, bias)
constexpr int kWinK = 256;       // codes per window: 4 groups, one 8-column accumulator
constexpr int kMmaPerWin = 8;    // m16n8k32 steps per window
constexpr int kImgWinEntries = kMmaPerWin * 32;  // uint2 operand words per window
constexpr int kTileRows = 16;    // output rows per warp tile (MMA M)
constexpr int kFfnWarps = 16;  // 512 threads, up to 128 registers each
constexpr int kFfnThreads = kFfnWarps * 32;
constexpr int kQuantMax = 32000; // |fixed-point activation| bound, fits hi/lo int8 split
constexpr int kMaxTopK = 32;
constexpr int kMaxExperts = 1024;
constexpr int kMaxDim = 8192;    // hidden and inter limits
constexpr int kMaxImgSlots = 4;  // expert-output images held at once by the down kernel

// ------------------------------------------------------------- pointers --
struct QMatDev {
    const uint32_t *codes;
    const uint16_t *scale;  // bf16 bits
    const uint16_t *bias;   // bf16 bits
};
struct QExpertDev {
    QMatDev gate, up, down;
};
static_assert(sizeof(QExpertDev) == sizeof(moe_qexpert), "slot entry layout");

// Workspace: a 256-byte header (status word) then one fixed-size block per
// token, so a token's counters sit at the same offset whatever T a call uses.
struct WsLayout {
    size_t tok_stride;  // bytes per token block
    size_t route_cnt;   // u32
    size_t ready;       // u32: 1 once the gate/up kernel has published the token's experts
    size_t logits;      // f64 [E+1]
    size_t topk_idx;    // i32 [k]
    size_t topk_w;      // f32 [k]
    size_t gamma;       // f32
    size_t ximg;        // uint2 [nwin(H)*256]: operand image of x (layer call: built by the router kernel)
    size_t xsg;         // f32 [H/64]: group sums of x
    size_t xdg;         // f32 [H/64]: fixed-point steps of x's groups
    size_t rx;          // QExpertDev [S]: the token's experts, resolved once by the gate/up kernel
    size_t rok;         // i32 [S]: 1 where rx is usable
    size_t h;           // f32 [S][I]
};
constexpr size_t kWsHeader = 256;

// Header: status word at byte 0, grid-sync counters of the fused layer
// kernel at byte 64 (kept at zero between calls by the kernel itself).
constexpr size_t kWsSyncOffset = 64;
constexpr int kWsSyncCount = 4;  // barrier 1, barrier 2, exit, spare

struct WsPtrs {
    unsigned char *base;  // token block 0
    WsLayout L;
    int *status;
    unsigned *sync;
    __device__ __host__ unsigned char *tok(int t) const { return base + (size_t)t * L.tok_stride; }
    __device__ __host__ unsigned *route_cnt(int t) const { return (unsigned *)(tok(t) + L.route_cnt); }
    __device__ __host__ unsigned *ready(int t) const { return (unsigned *)(tok(t) + L.ready); }
    __device__ __host__ double *logits(int t) const { return (double *)(tok(t) + L.logits); }
    __device__ __host__ int *topk_idx(int t) const { return (int *)(tok(t) + L.topk_idx); }
    __device__ __host__ float *topk_w(int t) const { return (float *)(tok(t) + L.topk_w); }
    __device__ __host__ float *gamma(int t) const { return (float *)(tok(t) + L.gamma); }
    __device__ __host__ uint2 *ximg(int t) const { return (uint2 *)(tok(t) + L.ximg); }
    __device__ __host__ float *xsg(int t) const { return (float *)(tok(t) + L.xsg); }
    __device__ __host__ float *xdg(int t) const { return (float *)(tok(t) + L.xdg); }
    __device__ __host__ QExpertDev *rx(int t) const { return (QExpertDev *)(tok(t) + L.rx); }
    __device__ __host__ int *rok(int t) const { return (int *)(tok(t) + L.rok); }
    __device__ __host__ float *h(int t) const { return (float *)(tok(t) + L.h); }
};

// -------------------------------------------------------------- device ---
__device__ __forceinline__ void griddep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Streaming 16-byte load of read-once weight data: bypass L1, ask L2 for a
// 256-byte prefetch around the access.
// (volatile: the loads stay where they are written, ahead of the math that
// uses the previous item, instead of being sunk next to their first use.)
__device__ __forceinline__ uint4 ldg_stream(const uint32_t *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ uint32_t ldg_u16(const uint16_t *p) {
    unsigned short v;
    asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) {
    return __uint_as_float(b << 16);
}

// D = A(16x32, u8 codes) * B(32x8, s8 activations) + D, int32 accumulate.
__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t u4_word(const uint4 &v, int i) {
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max_f32(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum_f32(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ void flag_status(int *status, int bit) {
    if (status) atomicOr(status, bit);
}

// A slot entry is usable when all nine pointers are non-NULL and the code
// arrays are 16-byte aligned (they are read with 16-byte vector loads).
__device__ __forceinline__ bool qmat_ok(const QMatDev &m) {
    return m.codes && m.scale && m.bias && ((reinterpret_cast<uintptr_t>(m.codes) & 15u) == 0) &&
           ((reinterpret_cast<uintptr_t>(m.scale) & 1u) == 0) &&
           ((reinterpret_cast<uintptr_t>(m.bias) & 1u) == 0);
}

__device__ __forceinline__ void st_release_u32(unsigned *p, unsigned v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// 16-byte asynchronous global -> shared copy (no registers held while in
// flight); cp_async_wait_all waits for this thread's copies.
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<unsigned>(__cvta_generic_to_shared(smem_dst))),
                 "l"(gmem_src)
                 : "memory");
}
__device__ __forceinline__ void cp_async8(void *smem_dst, const void *gmem_src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(static_cast<unsigned>(__cvta_generic_to_shared(smem_dst))),
                 "l"(gmem_src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// ------------------------------------------------- mbarriers and TMA bulk --

constexpr unsigned long long kWaitLimitNs = 1000000000ull;  // 1 s bound on any wait

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, unsigned parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits for the phase with the given parity; gives up after kWaitLimitNs,
// sets MOE_DEV_TIMEOUT and returns false (the caller carries on, so no
// thread is left waiting on it).
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, unsigned parity, int *status) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            flag_status(status, MOE_DEV_TIMEOUT);
            return false;
        }
    }
    return true;
}

// 1-D bulk copy global -> this CTA's shared memory, completing bytes on bar.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void tma_load_1d(void *dst, const void *src, unsigned bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void prefetch_l2(const void *src, unsigned bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Named barrier among `count` threads (a multiple of 32), id 1..15.
__device__ __forceinline__ void named_bar(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

}  // namespace moeq
