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
#include <mutex>

#include "internal.h"

namespace moe {
namespace {

// The scratch array: every GPU that loads this library holds it until the
// process exits.  Calls whose workspace (moe_workspace_bytes) exceeds it are
// rejected.
constexpr size_t kStaticScratchBytes = size_t(16) << 20;  // 16 MiB
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_mu;
void *g_ptr[64] = {};  // the array's device address, per device

// The array's device address on the current device (looked up once per
// device; the name itself is a host-side stand-in, not a device address).
int scratch_address(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ECUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return MOE_ECUDA;
        g_ptr[dev] = p;
    }
    *out = g_ptr[dev];
    return MOE_OK;
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
    if (!d || rows < 0) return MOE_EINVAL;
    if (rows == 0) return moe_ffn_forward(d, x, rows, router_w, expert_w8, expert_scales, shared_w, shared_gate,
                                          out, residual, router_bias, nullptr, 0, stream);
    const size_t need = moe_workspace_bytes(d, rows);
    if (need == 0) return MOE_EUNSUPPORTED;
    if (need > kStaticScratchBytes) return MOE_EWORKSPACE;  // beyond the built-in scratch
    void *ws = nullptr;
    int rc = scratch_address(&ws);
    if (rc != MOE_OK) {
        cudaGetLastError();
        return rc;
    }
    // The array keeps whatever the previous call left; the counters and the
    // status word must start at zero.
    if (cudaMemsetAsync(ws, 0, sizeof(int32_t) * kCounters, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ECUDA;
    }
    return moe_ffn_forward(d, x, rows, router_w, expert_w8, expert_scales, shared_w, shared_gate, out, residual,
                           router_bias, ws, kStaticScratchBytes, stream);
}

}  // extern "C"
