// Device-side helpers shared by the sm_100a kernels: element conversion, the
// exponentials used by the scan, and TMA / mbarrier primitives with bounded waits.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssm {

// ---------------------------------------------------------------- elements --

template <typename T> struct Elem;
template <> struct Elem<float> {
    static __device__ __forceinline__ float load(const float* p) { return *p; }
    static __device__ __forceinline__ float to_f(float v) { return v; }
    static __device__ __forceinline__ float from_f(float v) { return v; }
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16* p) {
        return __bfloat162float(*p);
    }
    static __device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
    static __device__ __forceinline__ __nv_bfloat16 from_f(float v) {
        return __float2bfloat16_rn(v);
    }
};

// ------------------------------------------------------------------- math --

// 2^x on the SFU (one MUFU.EX2). Inputs far below -126 flush to 0, which is the
// limit the recurrence wants for a fully decayed state.
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

constexpr float kLog2e = 1.4426950408889634f;

// softplus(x) = log(1 + e^x) = max(x, 0) + log1p(e), e = exp(-|x|) in (0, 1].
// log1p(e) = e * P(e) with P a degree-8 polynomial fitted by the Remez exchange
// algorithm to log1p(e)/e on [0, 1] (max relative error 3.0e-8, below fp32's half
// ulp), so the result keeps full relative accuracy for small e, where log(1 + e)
// evaluated directly would lose the low bits of e. One SFU op (the exp), nine FMAs.
__device__ __forceinline__ float softplus(float x) {
    const float e = ex2(-fabsf(x) * kLog2e);
    float q = 0.00523268878685f;
    q = fmaf(q, e, -0.029505215033f);
    q = fmaf(q, e, 0.0782259097531f);
    q = fmaf(q, e, -0.13663241868f);
    q = fmaf(q, e, 0.191060047105f);
    q = fmaf(q, e, -0.248429816251f);
    q = fmaf(q, e, 0.33319096724f);
    q = fmaf(q, e, -0.499994931362f);
    q = fmaf(q, e, 0.99999996988f);
    return fmaxf(x, 0.f) + e * q;
}

// silu(v) = v * sigmoid(v) = v / (1 + e^-v): one SFU exp and one SFU reciprocal
// (__fdividef); tends to 0 for v -> -inf (1 + e^-v overflows to inf, v / inf = 0).
__device__ __forceinline__ float silu(float v) { return __fdividef(v, 1.f + ex2(-v * kLog2e)); }

// ------------------------------------------------------ packed fp32 pairs --
// sm_100 executes add/mul/fma on two fp32 lanes of a 64-bit register pair as one
// instruction (.f32x2); the pipe throughput per element is unchanged, but issue
// slots are halved.

__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float2 upk2(uint64_t r) {
    float2 v;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(v.x), "=f"(v.y) : "l"(r));
    return v;
}
__device__ __forceinline__ float lo2(uint64_t r) { return upk2(r).x; }
__device__ __forceinline__ float hi2(uint64_t r) { return upk2(r).y; }
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// 1/x on the SFU (max error about 1 ulp).
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// silu on a pair of values: v / (1 + e^-v), two SFU exps and two SFU reciprocals.
__device__ __forceinline__ uint64_t silu2(uint64_t v) {
    const float2 f = upk2(v);
    const uint64_t e = pk2(ex2(-f.x * kLog2e), ex2(-f.y * kLog2e));
    const float2 den = upk2(add2(e, pk2(1.f, 1.f)));
    return mul2(v, pk2(rcp_approx(den.x), rcp_approx(den.y)));
}

// silu on a pair with one SFU op per value instead of two: e = 2^(-|v| log2 e) in (0, 1]
// on the SFU, then r = 1 / (1 + e) on the FMA pipe by Newton's iteration for the
// reciprocal, r <- r (2 - (1 + e) r), started from the linear minimax approximation
// 24/17 - 8/17 (1 + e) of 1 / (1 + e) on [1, 2] (relative error at most 1/17, squared by
// every step: after 2 steps 1.2e-5, after 3 steps 1.5e-10). sigmoid(v) = r for v >= 0 and
// e r for v < 0 (there e = e^v). v -> -inf: e flushes to 0 and silu to -0.
template <int ITERS>
__device__ __forceinline__ uint64_t silu2_fma(uint64_t v) {
    const float2 f = upk2(v);
    const uint64_t e = pk2(ex2(-fabsf(f.x) * kLog2e), ex2(-fabsf(f.y) * kLog2e));
    const uint64_t nd = fma2(e, pk2(-1.f, -1.f), pk2(-1.f, -1.f));      // -(1 + e)
    uint64_t r = fma2(nd, pk2(8.f / 17.f, 8.f / 17.f), pk2(24.f / 17.f, 24.f / 17.f));
#pragma unroll
    for (int i = 0; i < ITERS; ++i) r = mul2(r, fma2(nd, r, pk2(2.f, 2.f)));
    const float2 ee = upk2(e);
    const uint64_t m = pk2(f.x >= 0.f ? 1.f : ee.x, f.y >= 0.f ? 1.f : ee.y);
    return mul2(v, mul2(m, r));
}

// softplus on a pair (same polynomial as softplus()).
__device__ __forceinline__ uint64_t softplus2(uint64_t x2) {
    const float2 x = upk2(x2);
    const uint64_t e = pk2(ex2(-fabsf(x.x) * kLog2e), ex2(-fabsf(x.y) * kLog2e));
    uint64_t q = pk2(0.00523268878685f, 0.00523268878685f);
    q = fma2(q, e, pk2(-0.029505215033f, -0.029505215033f));
    q = fma2(q, e, pk2(0.0782259097531f, 0.0782259097531f));
    q = fma2(q, e, pk2(-0.13663241868f, -0.13663241868f));
    q = fma2(q, e, pk2(0.191060047105f, 0.191060047105f));
    q = fma2(q, e, pk2(-0.248429816251f, -0.248429816251f));
    q = fma2(q, e, pk2(0.33319096724f, 0.33319096724f));
    q = fma2(q, e, pk2(-0.499994931362f, -0.499994931362f));
    q = fma2(q, e, pk2(0.99999996988f, 0.99999996988f));
    return fma2(e, q, pk2(fmaxf(x.x, 0.f), fmaxf(x.y, 0.f)));
}

// Element i (a compile-time index once unrolled) of a run of 16-byte chunks of T,
// widened to fp32 (a bf16 value is the high half of an fp32 bit pattern).
template <typename T, int N>
__device__ __forceinline__ float chunk_elem(const uint4 (&w)[N], int i) {
    constexpr int EPC = 16 / (int)sizeof(T);
    const uint4 c = w[i / EPC];
    if constexpr (sizeof(T) == 2) {
        const int k = (i % 8) / 2;
        const uint32_t word = k == 0 ? c.x : k == 1 ? c.y : k == 2 ? c.z : c.w;
        return __uint_as_float((i & 1) ? (word & 0xffff0000u) : (word << 16));
    } else {
        const int k = i % 4;
        return __uint_as_float(k == 0 ? c.x : k == 1 ? c.y : k == 2 ? c.z : c.w);
    }
}

// ------------------------------------------------------- shared / barriers --

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
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

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Wait budget of a single mbarrier wait. A TMA tile lands in microseconds; a wait
// that lasts this long means the copy will not complete.
constexpr uint64_t kWaitLimitNs = 1000000000ull;   // 1 s

// Device-side error word of this translation unit, set when a bounded wait runs out.
// Every unit that includes the device headers names its own (SSM_ERROR_WORD) and
// ssm_device_error() reads and clears them all.
#ifndef SSM_ERROR_WORD
#error "define SSM_ERROR_WORD (this unit's device error word) before the device headers"
#endif
__device__ int SSM_ERROR_WORD = 0;

// Arrive on an mbarrier (release semantics at CTA scope).
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Named barrier over a subset of the CTA's warps (`count` threads, a multiple of 32).
__device__ __forceinline__ void named_bar_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Named barrier that also ORs a predicate over the participating threads; every
// participant gets the same result (used to take an abort decision uniformly).
__device__ __forceinline__ bool named_bar_or(int id, int count, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.cta.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}

// try_wait with a suspend-time hint: the thread may sleep in hardware until the phase
// completes or about `hint_ns` pass, instead of spinning and taking issue slots.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity,
                                                    uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Bounded wait on an mbarrier phase. Returns false (and records the error) when
// the budget runs out; the caller must then leave the kernel uniformly.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait_sleep(bar, parity, 20000u)) {
        if (globaltimer_ns() - t0 > limit_ns) {
            atomicExch(&SSM_ERROR_WORD, 1);
            return false;
        }
    }
    return true;
}

// ---------------------------------------------------------------------- TMA --

// 3-D tiled TMA load into this CTA's shared memory, completing on `bar`.
// The innermost coordinate c0 times the element size must be a multiple of 16 B.
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1, int32_t c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}

// 1-D bulk copy global -> this CTA's shared memory, completing on `bar`.
// Both addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes,
                                          uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes),
        "r"(smem_u32(bar))
        : "memory");
}

// 1-D bulk copy shared -> global (bulk-group completion).
__device__ __forceinline__ void bulk_store(void* gdst, const void* smem_src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                 ::"l"(reinterpret_cast<uint64_t>(gdst)), "r"(smem_u32(smem_src)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until the committed bulk stores have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Order this thread's generic-proxy shared-memory writes before later async-proxy reads.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Programmatic dependent launch: block until the grids this one depends on in the
// stream have completed and their writes are visible (a no-op for a launch without the
// programmatic attribute), then allow the next grid to start launching; its CTAs take
// the SMs this grid's last wave frees and wait there the same way.
__device__ __forceinline__ void grid_dependency_sync() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" :::);
}

// Launch with the programmatic-stream-serialization attribute (for kernels that begin
// with grid_dependency_sync).
template <typename... Args>
__host__ cudaError_t launch_dependent(void (*k)(Args...), dim3 grid, dim3 block, size_t smem,
                                      cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k, args...);
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

}  // namespace ssm
