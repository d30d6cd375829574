// moe_api.cu -- the C ABI declared in include/moe_ffn.h.
//
// Host side only: argument checks, workspace carving, path selection, the
// sticky status and the host fault knob.  Every step of the layer runs in
// the kernels of decode.cu and prefill.cu.
#include <algorithm>
#include <atomic>
#include <mutex>

#include "internal.h"
#include "launch.h"

namespace moe {

namespace {

std::atomic<int> g_status{MOE_OK};
std::atomic<int> g_fault_countdown{0};

std::mutex g_dev_mu;
DeviceInfo g_dev[64];
bool g_dev_ready[64] = {};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_dims(const moe_dims *d)
{
    if (!d) return MOE_EINVAL;
    if (d->hidden <= 0 || d->n_experts <= 0 || d->top_k <= 0 || d->inter <= 0 || d->shared_inter <= 0)
        return MOE_EUNSUPPORTED;
    if (d->hidden % 128 || d->inter % 128 || d->shared_inter % 128) return MOE_EUNSUPPORTED;
    if (d->top_k > d->n_experts || d->top_k > kMaxTopK || d->n_experts > kMaxExperts) return MOE_EUNSUPPORTED;
    if (d->hidden / 8 > kMaxBlendBlocks) return MOE_EUNSUPPORTED;
    return MOE_OK;
}

}  // namespace

// Common entry: sticky status and the host fault knob.
int enter()
{
    if (g_status.load() != MOE_OK) return MOE_ECUDA;
    int n = g_fault_countdown.load();
    while (n > 0) {
        if (g_fault_countdown.compare_exchange_weak(n, n - 1)) {
            if (n == 1) {
                g_status.store(MOE_ECUDA);
                return MOE_ECUDA;
            }
            break;
        }
    }
    return MOE_OK;
}

int finish(cudaError_t e)
{
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) {
        g_status.store(MOE_ECUDA);
        return MOE_ECUDA;
    }
    return MOE_OK;
}

TimingSession &timing_session()
{
    static thread_local TimingSession ts;
    return ts;
}

bool valid_path(int32_t path)
{
    return path == MOE_PATH_AUTO || path == MOE_PATH_DECODE || path == MOE_PATH_PREFILL ||
           path == MOE_PATH_PREFILL_NARROW;
}

// MOE_PATH_AUTO's choice for a row count: the decode kernels for a few
// rows, the narrow grouped GEMMs while an expert averages at most
// MOE_AUTO_NARROW_MAX_PAIRS routed rows, the 128-row token tiles above.
int32_t resolve_path(const moe_dims &d, int32_t rows, int32_t path)
{
    if (path != MOE_PATH_AUTO) return path;
    if (rows <= MOE_AUTO_DECODE_MAX_ROWS || !prefill_available()) return MOE_PATH_DECODE;
    if (narrow_supported(d) && (int64_t)rows * d.top_k <= (int64_t)MOE_AUTO_NARROW_MAX_PAIRS * d.n_experts)
        return MOE_PATH_PREFILL_NARROW;
    return MOE_PATH_PREFILL;
}

int kernel_launches(const moe_dims &d, int32_t rows, int32_t path)
{
    if (rows <= 0) return 0;
    path = resolve_path(d, rows, path);
    if (path == MOE_PATH_PREFILL || path == MOE_PATH_PREFILL_NARROW) return prefill_kernel_launches(d, rows);
    const int per = step_rows_per_launch(d, device_info().sm_count);
    return per > 0 ? (rows + per - 1) / per : 0;  // one decode-step launch per `per` rows
}

const DeviceInfo &device_info()
{
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (!g_dev_ready[dev]) {
        DeviceInfo &i = g_dev[dev];
        cudaDeviceGetAttribute(&i.sm_count, cudaDevAttrMultiProcessorCount, dev);
        cudaDeviceGetAttribute(&i.cc_major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&i.cc_minor, cudaDevAttrComputeCapabilityMinor, dev);
        int smem = 0;
        cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        i.max_smem_optin = (size_t)smem;
        if (i.sm_count <= 0) i.sm_count = 148;  // no device to ask (host-only queries): a B200's count
        g_dev_ready[dev] = true;
    }
    return g_dev[dev];
}

// Argument checks of a forward call that need no workspace (host only).
int check_forward_args(const moe_dims *d, const uint16_t *x, int32_t rows, const uint16_t *router_w,
                       const uint8_t *expert_w8, const float *expert_scales, const moe_fp8_expert *shared_w,
                       const uint16_t *shared_gate, const uint16_t *out, const uint16_t *residual,
                       const float *router_bias, int32_t path, const int32_t *topk_idx_out,
                       const float *topk_w_out, const float *shared_gate_sig_out, bool out_may_alias_x)
{
    int st = check_dims(d);
    if (st) return st;
    if (rows < 0) return MOE_EINVAL;
    if (!valid_path(path)) return MOE_EINVAL;
    if (rows == 0) return MOE_OK;
    if (!x || !router_w || !expert_w8 || !expert_scales || !shared_w || !shared_w->w8 ||
        !shared_w->scales || !shared_gate || !out)
        return MOE_EINVAL;
    if (!aligned16(x) || !aligned16(router_w) || !aligned16(expert_w8) || !aligned16(expert_scales) ||
        !aligned16(shared_w->w8) || !aligned16(shared_w->scales) || !aligned16(shared_gate) ||
        !aligned16(out) || (residual && !aligned16(residual)) ||
        (router_bias && !aligned16(router_bias)) || (topk_idx_out && !aligned16(topk_idx_out)) ||
        (topk_w_out && !aligned16(topk_w_out)) || (shared_gate_sig_out && !aligned16(shared_gate_sig_out)))
        return MOE_EINVAL;
    if (!out_may_alias_x && static_cast<const void *>(out) == static_cast<const void *>(x)) return MOE_EINVAL;
    return MOE_OK;
}

// The layer step on a checked, large-enough workspace, after enter().
int run_forward(const moe_dims *d, const uint16_t *x, int32_t rows, const uint16_t *router_w,
                const uint8_t *expert_w8, const float *expert_scales, const moe_fp8_expert *shared_w,
                const uint16_t *shared_gate, uint16_t *out, const uint16_t *residual, const float *router_bias,
                void *ws, void *stream, int32_t path, int32_t *topk_idx_out, float *topk_w_out,
                float *shared_gate_sig_out, const uint16_t *norm_w, double eps)
{
    if (rows == 0) return MOE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    path = resolve_path(*d, rows, path);
    if (path == MOE_PATH_PREFILL || path == MOE_PATH_PREFILL_NARROW) {
        if (norm_w) {
            // the norm as its own kernel; the layer reads its output, the residual is the input rows
            uint16_t *xn = reinterpret_cast<uint16_t *>(static_cast<char *>(ws) + norm_buffer_offset(*d, rows));
            if (launch_rmsnorm(x, norm_w, eps, d->hidden, rows, xn, s) != cudaSuccess) return finish(cudaGetLastError());
            residual = x;
            x = xn;
        }
        int rc = prefill_forward(*d, x, rows, router_w, expert_w8, expert_scales, shared_w->w8,
                                 shared_w->scales, shared_gate, out, residual, router_bias, ws, s,
                                 topk_idx_out, topk_w_out, shared_gate_sig_out, path == MOE_PATH_PREFILL_NARROW);
        if (rc == MOE_ECUDA) g_status.store(MOE_ECUDA);
        return rc;
    }

    const DecodeLayout L = decode_layout(*d, rows);
    char *base = static_cast<char *>(ws);
    int32_t *tidx = topk_idx_out ? topk_idx_out : reinterpret_cast<int32_t *>(base + L.topk_idx);
    float *tw = topk_w_out ? topk_w_out : reinterpret_cast<float *>(base + L.topk_w);
    float *gs = shared_gate_sig_out ? shared_gate_sig_out : reinterpret_cast<float *>(base + L.gsig);
    const int per = step_rows_per_launch(*d, device_info().sm_count);
    if (per < 1) return MOE_EUNSUPPORTED;
    const int H = d->hidden, K = d->top_k;
    for (int r0 = 0; r0 < rows; r0 += per) {
        StepLaunch a;
        a.d = d;
        a.rows = std::min(per, rows - r0);
        a.x = x + (size_t)r0 * H;
        a.norm_w = norm_w;
        a.eps = eps;
        a.router_w = router_w;
        a.router_bias = router_bias;
        a.shared_gate = shared_gate;
        a.expert_w8 = expert_w8;
        a.expert_scales = expert_scales;
        a.shared_w8 = shared_w->w8;
        a.shared_scales = shared_w->scales;
        a.residual = norm_w ? a.x : residual ? residual + (size_t)r0 * H : nullptr;
        a.out = out + (size_t)r0 * H;
        a.topk_idx = tidx + (size_t)r0 * K;
        a.topk_w = tw + (size_t)r0 * K;
        a.gsig = gs + r0;
        a.logits = reinterpret_cast<float *>(base + L.logits);
        a.logits_ld = L.ld;
        a.hterm = reinterpret_cast<unsigned char *>(base + L.hterm);
        a.hsc = reinterpret_cast<float *>(base + L.hsc);
        a.counters = reinterpret_cast<int32_t *>(base + L.counters);
        const cudaError_t e = launch_decode_step(a, s);
        if (e != cudaSuccess) return finish(e);
    }
    return finish(cudaSuccess);
}

}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_workspace_bytes(const moe_dims *d, int32_t max_rows)
{
    if (check_dims(d) != MOE_OK || max_rows < 0) return 0;
    return workspace_bytes(*d, max_rows < 1 ? 1 : max_rows);
}

int moe_workspace_init(void *ws, size_t ws_bytes, void *stream)
{
    int st = enter();
    if (st) return st;
    if (!ws && ws_bytes) return MOE_EINVAL;
    if (!ws_bytes) return MOE_OK;
    return finish(cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream)));
}

int moe_router_topk(const moe_dims *d, const uint16_t *x, int32_t rows, const uint16_t *router_w,
                    const float *router_bias, const uint16_t *shared_gate, int32_t *topk_idx,
                    float *topk_w, float *shared_gate_sig, void *ws, size_t ws_bytes, void *stream)
{
    int st = check_dims(d);
    if (st) return st;
    if (rows < 0) return MOE_EINVAL;
    if (rows == 0) return enter();  // a no-op: no pointer is read
    if (!x || !router_w || !shared_gate || !topk_idx || !topk_w || !shared_gate_sig || !ws) return MOE_EINVAL;
    if (!aligned16(x) || !aligned16(router_w) || !aligned16(shared_gate) || !aligned16(ws) ||
        (router_bias && !aligned16(router_bias)) || !aligned16(topk_idx) || !aligned16(topk_w) ||
        !aligned16(shared_gate_sig))
        return MOE_EINVAL;
    if (ws_bytes < workspace_bytes(*d, rows < 1 ? 1 : rows)) return MOE_EWORKSPACE;
    st = enter();
    if (st) return st;
    if (rows == 0) return MOE_OK;
    const DecodeLayout L = decode_layout(*d, rows);
    char *base = static_cast<char *>(ws);
    RouterLaunch a;
    a.d = d;
    a.x = x;
    a.rows = rows;
    a.router_w = router_w;
    a.router_bias = router_bias;
    a.shared_gate = shared_gate;
    a.topk_idx = topk_idx;
    a.topk_w = topk_w;
    a.gsig = shared_gate_sig;
    a.logits = reinterpret_cast<float *>(base + L.logits);
    a.counters = reinterpret_cast<int32_t *>(base + L.counters);
    return finish(launch_router_topk(a, static_cast<cudaStream_t>(stream)));
}

int moe_ffn_forward_path(const moe_dims *d, const uint16_t *x, int32_t rows, const uint16_t *router_w,
                         const uint8_t *expert_w8, const float *expert_scales,
                         const moe_fp8_expert *shared_w, const uint16_t *shared_gate, uint16_t *out,
                         const uint16_t *residual, const float *router_bias, void *ws, size_t ws_bytes,
                         void *stream, int32_t path, int32_t *topk_idx_out, float *topk_w_out,
                         float *shared_gate_sig_out)
{
    int st = check_forward_args(d, x, rows, router_w, expert_w8, expert_scales, shared_w, shared_gate, out,
                                residual, router_bias, path, topk_idx_out, topk_w_out, shared_gate_sig_out, false);
    if (st) return st;
    if (rows == 0) return enter();  // a no-op: no pointer is read
    if (!ws || !aligned16(ws)) return MOE_EINVAL;
    if (ws_bytes < workspace_bytes(*d, rows)) return MOE_EWORKSPACE;
    st = enter();
    if (st) return st;
    return run_forward(d, x, rows, router_w, expert_w8, expert_scales, shared_w, shared_gate, out, residual,
                       router_bias, ws, stream, path, topk_idx_out, topk_w_out, shared_gate_sig_out, nullptr, 0.0);
}

int moe_ffn_forward_norm(const moe_dims *d, const uint16_t *resid, int32_t rows, const uint16_t *norm_w, float eps,
                         const uint16_t *router_w, const uint8_t *expert_w8, const float *expert_scales,
                         const moe_fp8_expert *shared_w, const uint16_t *shared_gate, uint16_t *out,
                         const float *router_bias, void *ws, size_t ws_bytes, void *stream, int32_t path)
{
    int st = check_forward_args(d, resid, rows, router_w, expert_w8, expert_scales, shared_w, shared_gate, out,
                                nullptr, router_bias, path, nullptr, nullptr, nullptr, true);
    if (st) return st;
    if (rows == 0) return enter();  // a no-op: no pointer is read
    if (!norm_w || !aligned16(norm_w) || !(eps >= 0.f) || !ws || !aligned16(ws)) return MOE_EINVAL;
    if (ws_bytes < workspace_bytes(*d, rows)) return MOE_EWORKSPACE;
    st = enter();
    if (st) return st;
    return run_forward(d, resid, rows, router_w, expert_w8, expert_scales, shared_w, shared_gate, out, nullptr,
                       router_bias, ws, stream, path, nullptr, nullptr, nullptr, norm_w, (double)eps);
}

int moe_ffn_forward(const moe_dims *d, const uint16_t *x, int32_t rows, const uint16_t *router_w,
                    const uint8_t *expert_w8, const float *expert_scales, const moe_fp8_expert *shared_w,
                    const uint16_t *shared_gate, uint16_t *out, const uint16_t *residual,
                    const float *router_bias, void *ws, size_t ws_bytes, void *stream)
{
    return moe_ffn_forward_path(d, x, rows, router_w, expert_w8, expert_scales, shared_w, shared_gate, out,
                                residual, router_bias, ws, ws_bytes, stream, MOE_PATH_AUTO, nullptr,
                                nullptr, nullptr);
}

// The device address of pinned, device-addressable host memory, else null.
static void *host_device_address(const void *p)
{
    cudaPointerAttributes a{};
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();  // a plain host pointer: not an error to keep
        return nullptr;
    }
    return a.type == cudaMemoryTypeHost ? a.devicePointer : nullptr;
}

int moe_ffn_forward_host(const moe_dims *d, const uint16_t *x_host, int32_t rows, const uint16_t *router_w,
                         const uint8_t *expert_w8, const float *expert_scales, const moe_fp8_expert *shared_w,
                         const uint16_t *shared_gate, uint16_t *out_host, const float *router_bias, void *ws,
                         size_t ws_bytes, void *stream)
{
    int st = check_forward_args(d, x_host, rows, router_w, expert_w8, expert_scales, shared_w, shared_gate,
                                out_host, nullptr, router_bias, MOE_PATH_AUTO, nullptr, nullptr, nullptr, false);
    if (st) return st;
    if (rows == 0) return enter();  // a no-op: no pointer is read
    if (!ws || !aligned16(ws)) return MOE_EINVAL;
    if (ws_bytes < workspace_bytes(*d, rows)) return MOE_EWORKSPACE;
    const void *xd = host_device_address(x_host);
    void *od = host_device_address(out_host);
    if (!xd || !od || !aligned16(xd) || !aligned16(od)) return MOE_EINVAL;
    st = enter();
    if (st) return st;
    // x into the workspace's row buffer (the one the normalised entry uses)
    uint16_t *xs = reinterpret_cast<uint16_t *>(static_cast<char *>(ws) + norm_buffer_offset(*d, rows));
    const cudaError_t e =
        launch_host_rows_in(xd, xs, (size_t)rows * d->hidden * 2, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return finish(e);
    return run_forward(d, xs, rows, router_w, expert_w8, expert_scales, shared_w, shared_gate,
                       static_cast<uint16_t *>(od), nullptr, router_bias, ws, stream, MOE_PATH_AUTO, nullptr,
                       nullptr, nullptr, nullptr, 0.0);
}

int moe_ffn_forward_nvfp4(const moe_dims *d, const uint16_t *x, int32_t rows, const uint16_t *router_w,
                          const uint8_t *expert_w4, const uint8_t *expert_sf, const float *expert_gs,
                          const moe_nvfp4_expert *shared, const uint16_t *shared_gate, uint16_t *out,
                          const uint16_t *residual, const float *router_bias, void *ws, size_t ws_bytes,
                          void *stream)
{
    int st = check_dims(d);
    if (st) return st;
    if (rows < 0) return MOE_EINVAL;
    if (rows == 0) return enter();  // a no-op: no pointer is read
    const auto a4 = [](const void *q) { return (reinterpret_cast<uintptr_t>(q) & 3u) == 0; };
    if (!x || !router_w || !expert_w4 || !expert_sf || !expert_gs || !shared || !shared->w4 || !shared->sf ||
        !shared->gs || !shared_gate || !out || !ws)
        return MOE_EINVAL;
    if (!aligned16(x) || !aligned16(router_w) || !aligned16(expert_w4) || !aligned16(expert_sf) ||
        !a4(expert_gs) || !aligned16(shared->w4) || !aligned16(shared->sf) || !a4(shared->gs) ||
        !aligned16(shared_gate) || !aligned16(out) || (residual && !aligned16(residual)) ||
        (router_bias && !aligned16(router_bias)) || !aligned16(ws))
        return MOE_EINVAL;
    if (static_cast<const void *>(out) == static_cast<const void *>(x)) return MOE_EINVAL;
    if (ws_bytes < workspace_bytes(*d, rows)) return MOE_EWORKSPACE;
    st = enter();
    if (st) return st;
    const DecodeLayout L = decode_layout(*d, rows);
    char *base = static_cast<char *>(ws);
    Nvfp4Launch a;
    a.d = d;
    a.x = x;
    a.rows = rows;
    a.router_w = router_w;
    a.router_bias = router_bias;
    a.shared_gate = shared_gate;
    a.w4 = expert_w4;
    a.sf = expert_sf;
    a.gs = expert_gs;
    a.sw4 = shared->w4;
    a.ssf = shared->sf;
    a.sgs = shared->gs;
    a.residual = residual;
    a.out = out;
    a.topk_idx = reinterpret_cast<int32_t *>(base + L.topk_idx);
    a.topk_w = reinterpret_cast<float *>(base + L.topk_w);
    a.gsig = reinterpret_cast<float *>(base + L.gsig);
    a.logits = reinterpret_cast<float *>(base + L.logits);
    a.h = reinterpret_cast<float *>(base + L.hterm);  // h of a chunk of rows fits the step's term region
    a.counters = reinterpret_cast<int32_t *>(base + L.counters);
    return finish(launch_nvfp4_forward(a, static_cast<cudaStream_t>(stream)));
}

int32_t moe_auto_path(const moe_dims *d, int32_t rows)
{
    if (check_dims(d) != MOE_OK || rows < 0) return MOE_EINVAL;
    return resolve_path(*d, rows, MOE_PATH_AUTO);
}

int32_t moe_kernel_launches(const moe_dims *d, int32_t rows, int32_t path)
{
    if (check_dims(d) != MOE_OK || rows < 0) return 0;
    if (!valid_path(path)) return 0;
    return kernel_launches(*d, rows, path);
}

int moe_ffn_forward_timed(const moe_dims *d, const uint16_t *x, int32_t rows, const uint16_t *router_w,
                          const uint8_t *expert_w8, const float *expert_scales, const moe_fp8_expert *shared_w,
                          const uint16_t *shared_gate, uint16_t *out, const uint16_t *residual,
                          const float *router_bias, void *ws, size_t ws_bytes, void *stream, int32_t path,
                          void *const *events, int32_t n_events)
{
    if (!events || check_dims(d) != MOE_OK || rows < 0) return !events ? MOE_EINVAL : check_dims(d);
    const int need = kernel_launches(*d, rows, path);
    if (n_events < need + 1) return MOE_EINVAL;
    for (int i = 0; i < need + 1; ++i)
        if (!events[i]) return MOE_EINVAL;
    TimingSession &ts = timing_session();
    ts.events = reinterpret_cast<cudaEvent_t *>(const_cast<void **>(events));
    ts.n_events = need + 1;
    ts.next = 0;
    ts.overflow = false;
    int rc = moe_ffn_forward_path(d, x, rows, router_w, expert_w8, expert_scales, shared_w, shared_gate, out,
                                  residual, router_bias, ws, ws_bytes, stream, path, nullptr, nullptr, nullptr);
    const int recorded = ts.next;
    ts = TimingSession{};
    if (rc != MOE_OK || rows == 0) return rc;
    if (recorded != need) return MOE_EINVAL;
    return finish(cudaEventRecord(static_cast<cudaEvent_t>(events[need]), static_cast<cudaStream_t>(stream)));
}

int moe_device_status(const void *ws, size_t ws_bytes, void *stream)
{
    if (!ws || ws_bytes < sizeof(int32_t) * kCounters || !aligned16(ws)) return MOE_EINVAL;
    int32_t v = 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(&v, static_cast<const int32_t *>(ws) + kCtrStatus, sizeof v,
                                    cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) {
        g_status.store(MOE_ECUDA);
        return MOE_ECUDA;
    }
    return v;
}

int moe_debug_wait_timeout(void *ws, size_t ws_bytes, int32_t limit_us, void *stream)
{
    if (!ws || ws_bytes < sizeof(int32_t) * kCounters || !aligned16(ws)) return MOE_EINVAL;
    int st = enter();
    if (st) return st;
    if (limit_us < 1) limit_us = 1;
    if (limit_us > 2000000) limit_us = 2000000;
    return finish(launch_wait_probe(static_cast<int32_t *>(ws), (uint64_t)limit_us * 1000ull,
                                    static_cast<cudaStream_t>(stream)));
}

int moe_status(void) { return g_status.load(); }

void moe_reset_status(void)
{
    cudaGetLastError();
    g_status.store(MOE_OK);
    g_fault_countdown.store(0);
}

const char *moe_status_string(int status)
{
    switch (status) {
    case MOE_OK: return "ok";
    case MOE_EINVAL: return "invalid argument (null or misaligned pointer, negative rows, bad path)";
    case MOE_EUNSUPPORTED: return "unsupported dimensions (H, I, Is multiples of 128; k <= min(E, 32); E <= 1024)";
    case MOE_EWORKSPACE: return "workspace too small (see moe_workspace_bytes)";
    case MOE_ECUDA: return "CUDA error (sticky until moe_reset_status)";
    case MOE_ETIMEOUT: return "a bounded wait inside a kernel ran out (re-initialise the workspace)";
    default: return "unknown status";
    }
}

void moe_debug_inject_fault(int32_t n) { g_fault_countdown.store(n > 0 ? n : 0); }

}  // extern "C"
