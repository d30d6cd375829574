// common.cuh -- device helpers shared by the decode and prefill kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"
#include "moe_ffn.h"

namespace moe {

constexpr int kWarp = 32;

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

// Low and high bf16 halves of a 32-bit word.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float v)
{
    __nv_bfloat16 b = __float2bfloat16_rn(v);
    return *reinterpret_cast<uint16_t *>(&b);
}

// Two e4m3 codes (low byte first) -> two floats, through the hardware
// e4m3x2 -> f16x2 conversion (exact: every e4m3 value is an f16 value).
__device__ __forceinline__ float2 e4m3x2_to_f32x2(uint16_t two)
{
    __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two), __NV_E4M3);
    return __half22float2(*reinterpret_cast<__half2 *>(&h));
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

// 16-byte global load that bypasses L1 allocation (streamed weights).
__device__ __forceinline__ uint4 ld_stream_v4(const void *p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Programmatic dependent launch controls (no-ops when launched without the
// attribute).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" :::); }

// ------------------------------------------------------------ mbarriers

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Make mbarrier initialisation visible to the async (bulk-copy) proxy.
__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// One bounded probe of an mbarrier phase; the thread may sleep in it for up
// to ~1 us (suspend-time hint) instead of spinning.
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(1000)
        : "memory");
    return ok != 0;
}

// Non-blocking probe of an mbarrier phase.
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for phase `parity` of an mbarrier for at most limit_ns of wall time.
// Returns false if the limit ran out.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint64_t limit_ns)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        for (int i = 0; i < 8; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
}

// mbar_wait that spins instead of sleeping in the probe: for a thread whose
// wait is on the critical path and whose warp has nothing else to do.
__device__ __forceinline__ bool mbar_wait_spin(uint64_t *bar, uint32_t parity, uint64_t limit_ns)
{
    if (mbar_test_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        for (int i = 0; i < 32; ++i)
            if (mbar_test_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
}

// Bring [p, p + bytes) into L2 (asynchronous, no completion to wait for).
// p 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Order this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (bulk copy) accesses.
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Bulk (non-tensor) copy global -> shared, completing on an mbarrier.  Both
// addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// The same with an L2 evict-first hint (streamed weights).
__device__ __forceinline__ void bulk_g2s_stream(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                                uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], "
        "%4;" ::"r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// Named barrier over the first `count` threads of the CTA (id 1..15).
__device__ __forceinline__ void named_barrier(int id, int count)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.expect_tx.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

// Phase tracing for development builds (compiled with -DMOE_PHASE_TRACE):
// the calling thread records %globaltimer at a numbered point of kernel
// `kid` for its CTA.  Expands to nothing in the library build.
#ifdef MOE_PHASE_TRACE
static __device__ unsigned long long *g_moe_trace;  // one per translation unit
#define MOE_TRACE(kid, slot)                                                                    \
    do {                                                                                        \
        if (g_moe_trace)                                                                        \
            g_moe_trace[((size_t)(kid) * 4096 + blockIdx.x + blockIdx.y * gridDim.x) * 16 + (slot)] = \
                globaltimer_ns();                                                               \
    } while (0)
#else
#define MOE_TRACE(kid, slot) \
    do {                     \
    } while (0)
#endif

// D += A * B on the tensor cores: m16n8k32, e4m3 x e4m3 -> f32.
//   a0: row g, k 4t..4t+3    a1: row g+8, k 4t..4t+3
//   a2: row g, k 16+4t..     a3: row g+8, k 16+4t..
//   b0: col g, k 4t..4t+3    b1: col g, k 16+4t..
//   d0,d1: row g, cols 2t, 2t+1     d2,d3: row g+8, cols 2t, 2t+1
// (g = lane / 4, t = lane % 4).
__device__ __forceinline__ void mma_e4m3_16832(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two floats -> two e4m3 codes (round to nearest even, saturating), low
// byte first.
__device__ __forceinline__ uint16_t f32x2_to_e4m3x2(float lo, float hi)
{
    return static_cast<uint16_t>(__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

// The activation format of the tensor-core GEMVs: for each 128-wide block of
// a row, s = amax/448 (1 for an all-zero block), hi = e4m3(v/s) and
// lo = e4m3(v/s - hi), so that v ~ s * (hi + lo).  One thread quantises 4
// consecutive values given the block's scale reciprocal; returns the four
// hi codes and the four lo codes packed low byte first.
__device__ __forceinline__ void quant4_hilo(float4 v, float inv_s, uint32_t &hi, uint32_t &lo)
{
    const float a = v.x * inv_s, b = v.y * inv_s, c = v.z * inv_s, d = v.w * inv_s;
    const uint16_t h01 = f32x2_to_e4m3x2(a, b), h23 = f32x2_to_e4m3x2(c, d);
    const float2 f01 = e4m3x2_to_f32x2(h01), f23 = e4m3x2_to_f32x2(h23);
    const uint16_t l01 = f32x2_to_e4m3x2(a - f01.x, b - f01.y), l23 = f32x2_to_e4m3x2(c - f23.x, d - f23.y);
    hi = (uint32_t)h01 | ((uint32_t)h23 << 16);
    lo = (uint32_t)l01 | ((uint32_t)l23 << 16);
}

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    return v;
}

// Nearest bf16 of a double, ties to even, rounded once from the double (not
// through float): for |v| in the normal bf16 range the double's fraction is
// rounded at its 8th significant bit; below it, at the subnormal step 2^-133.
__device__ __forceinline__ uint16_t f64_to_bf16_rn(double v)
{
    unsigned long long u = (unsigned long long)__double_as_longlong(v);
    const uint16_t sign = (uint16_t)((u >> 48) & 0x8000u);
    unsigned long long a = u & 0x7FFFFFFFFFFFFFFFull;
    if (a >= 0x7FF0000000000000ull) return f32_to_bf16_bits((float)v);  // inf, NaN
    if (a >= 0x3810000000000000ull) {                                     // >= 2^-126
        a += 0x00000FFFFFFFFFFFull + ((a >> 45) & 1ull);
        a &= ~0x00001FFFFFFFFFFFull;
        const float f = (float)__longlong_as_double((long long)a);        // exact, or inf past the range
        return (uint16_t)(sign | (uint16_t)(__float_as_uint(f) >> 16));
    }
    const double m = rint(__longlong_as_double((long long)a) * 0x1p133);  // subnormal steps, ties to even
    return (uint16_t)(sign | (uint16_t)m);
}

__device__ __forceinline__ int atomic_add_acq_rel_gpu(int32_t *p, int v)
{
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// Record a device-side error in the workspace status word (first one wins).
__device__ __forceinline__ void set_status(int32_t *counters, int32_t code)
{
    atomicCAS(&counters[kCtrStatus], 0, code);
}

// Order-preserving 32-bit key of a float (larger key = larger value).
__device__ __forceinline__ uint32_t ordered_key(float f)
{
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k)
{
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Router top-k key of a logit: larger is better; NaN ranks below every
// number (key 1) and 0 marks an empty slot.
__device__ __forceinline__ uint32_t topk_key(float l) { return isnan(l) ? 1u : max(ordered_key(l), 2u); }

// Default bound on any wait inside a kernel (wall time).
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ float sigmoidf_(float z) { return 1.0f / (1.0f + expf(-z)); }
__device__ __forceinline__ float siluf_(float a) { return a / (1.0f + expf(-a)); }

}  // namespace moe
