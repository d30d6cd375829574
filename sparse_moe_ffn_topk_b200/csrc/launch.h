// launch.h -- kernel launch helper shared by the decode and prefill paths.
//
// Kernels are launched with programmatic dependent launch (each kernel calls
// griddepcontrol.wait before it reads what its predecessor wrote, and
// griddepcontrol.launch_dependents once it has), so a dependent kernel's CTAs
// are resident and prefetching when its predecessor finishes.
//
// When a per-kernel timing session is active on this thread
// (moe_ffn_forward_timed), an event is recorded on the stream before every
// launch and programmatic dependent launch is switched off, so that the
// interval between two events is one kernel's execution.
#pragma once

#include <cuda_runtime.h>

namespace moe {

struct TimingSession {
    cudaEvent_t *events = nullptr;
    int n_events = 0;
    int next = 0;
    bool overflow = false;
};

TimingSession &timing_session();

template <typename P>
cudaError_t launch_kernel(void (*kernel)(P), dim3 grid, dim3 block, size_t smem, cudaStream_t s, const P &p)
{
    TimingSession &ts = timing_session();
    const bool timed = ts.events != nullptr;
    if (timed) {
        if (ts.next >= ts.n_events - 1) {
            ts.overflow = true;
            return cudaErrorInvalidValue;
        }
        cudaError_t e = cudaEventRecord(ts.events[ts.next++], s);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = timed ? 0 : 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, p);
}

}  // namespace moe
