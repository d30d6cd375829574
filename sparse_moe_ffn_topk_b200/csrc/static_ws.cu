// static_ws.cu -- the layer step without a caller-provided workspace.
//
// Some callers cannot allocate device memory at all: code that runs inside a
// host application whose memory manager owns every device allocation (a
// serving engine's fixed pool, a plugin that must not grow the process's
// device footprint), or code that must never take the allocation path
// (which can synchronise the device) in the middle of its work.  For them,
// moe_ffn_forward_static uses scratch memory that the library itself holds
// for the lifetime of the process: one statically sized device array per
// GPU, created when the library's device code is loaded on that GPU.
//
// The array's status word (the word a bounded wait inside a kernel sets to
// MOE_ETIMEOUT) is not cleared by the calls: it stays set until
// moe_static_device_status reports it, so a timeout in one call cannot be
// erased by the next one.
#include <cuda.h>

#include <mutex>

#include "internal.h"

namespace moe {
namespace {

// The scratch array: every GPU that loads this library holds it until the
// process exits.  Calls whose workspace (moe_workspace_bytes) exceeds it are
// rejected.
constexpr size_t kStaticScratchBytes = size_t(16) << 20;  // 16 MiB
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// The array's device address, per device and per context: after a context
// is torn down and created again (cudaDeviceReset anywhere in the process)
// the module is loaded again and the address is looked up again.
struct Cached {
    CUcontext ctx = nullptr;
    void *ptr = nullptr;
};
std::mutex g_mu;
Cached g_cache[64];

using CtxGetCurrentFn = CUresult (*)(CUcontext *);

CtxGetCurrentFn ctx_get_current()
{
    static CtxGetCurrentFn fn = [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return static_cast<CtxGetCurrentFn>(nullptr);
        return reinterpret_cast<CtxGetCurrentFn>(f);
    }();
    return fn;
}

// The array's device address on the current device and context.  In host
// code the array's name is only a host-side stand-in; the device address
// comes from cudaGetSymbolAddress with the device current.
int scratch_address(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ECUDA;
    CtxGetCurrentFn get = ctx_get_current();
    if (!get) return MOE_ECUDA;
    CUcontext ctx = nullptr;
    if (get(&ctx) != CUDA_SUCCESS) return MOE_ECUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    Cached &c = g_cache[dev];
    if (!ctx || c.ctx != ctx || !c.ptr) {
        // The lookup also makes the device's primary context current (on the
        // first CUDA call of a thread no context is current yet).
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return MOE_ECUDA;
        if (get(&ctx) != CUDA_SUCCESS || !ctx) return MOE_ECUDA;
        c.ctx = ctx;
        c.ptr = p;
    }
    *out = c.ptr;
    return MOE_OK;
}

// A CUDA failure in this file: sticky, like every other CUDA error.
int cuda_failed(cudaError_t e)
{
    return finish(e == cudaSuccess ? cudaErrorUnknown : e);
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

MOE_API size_t moe_static_scratch_bytes(void) { return kStaticScratchBytes; }

MOE_API int moe_ffn_forward_static(const moe_dims *d, const uint16_t *x, int32_t rows, const uint16_t *router_w,
                                   const uint8_t *expert_w8, const float *expert_scales,
                                   const moe_fp8_expert *shared_w, const uint16_t *shared_gate, uint16_t *out,
                                   const uint16_t *residual, const float *router_bias, void *stream)
{
    int st = check_forward_args(d, x, rows, router_w, expert_w8, expert_scales, shared_w, shared_gate, out,
                                residual, router_bias, MOE_PATH_AUTO, nullptr, nullptr, nullptr, false);
    if (st) return st;
    if (rows == 0) return enter();  // a no-op: no pointer is read
    const size_t need = moe_workspace_bytes(d, rows);
    if (need == 0) return MOE_EUNSUPPORTED;
    if (need > kStaticScratchBytes) return MOE_EWORKSPACE;  // beyond the built-in scratch
    st = enter();
    if (st) return st;
    void *ws = nullptr;
    st = scratch_address(&ws);
    if (st != MOE_OK) return cuda_failed(cudaGetLastError());
    // The array keeps whatever the previous call left: the counters must
    // start at zero, all but the status word, which keeps a pending
    // MOE_ETIMEOUT until moe_static_device_status has reported it.
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t *ctr = static_cast<int32_t *>(ws);
    cudaError_t e = cudaMemsetAsync(ctr, 0, sizeof(int32_t) * kCtrStatus, s);
    if (e == cudaSuccess)
        e = cudaMemsetAsync(ctr + kCtrStatus + 1, 0, sizeof(int32_t) * (kCounters - kCtrStatus - 1), s);
    if (e != cudaSuccess) return cuda_failed(e);
    return run_forward(d, x, rows, router_w, expert_w8, expert_scales, shared_w, shared_gate, out, residual,
                       router_bias, ws, stream, MOE_PATH_AUTO, nullptr, nullptr, nullptr, nullptr, 0.0);
}

MOE_API int moe_static_device_status(void *stream)
{
    int st = enter();
    if (st) return st;
    void *ws = nullptr;
    if (scratch_address(&ws) != MOE_OK) return cuda_failed(cudaGetLastError());
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t v = 0;
    int32_t *word = static_cast<int32_t *>(ws) + kCtrStatus;
    cudaError_t e = cudaMemcpyAsync(&v, word, sizeof v, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e == cudaSuccess && v != MOE_OK) {
        e = cudaMemsetAsync(word, 0, sizeof v, s);  // reported once
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    }
    if (e != cudaSuccess) return cuda_failed(e);
    return v;
}

MOE_API int moe_debug_wait_timeout_static(int32_t limit_us, void *stream)
{
    int st = enter();
    if (st) return st;
    void *ws = nullptr;
    if (scratch_address(&ws) != MOE_OK) return cuda_failed(cudaGetLastError());
    if (limit_us < 1) limit_us = 1;
    if (limit_us > 2000000) limit_us = 2000000;
    return finish(launch_wait_probe(static_cast<int32_t *>(ws), (uint64_t)limit_us * 1000ull,
                                    static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
