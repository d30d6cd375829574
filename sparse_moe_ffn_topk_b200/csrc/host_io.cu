// host_io.cu -- the input copy of the host-buffer entry (moe_ffn_forward_host):
// the rows of x from pinned host memory into the workspace, read by the GPU
// itself over the host link, so that a step needs no copy-engine transfer and
// the forward's first kernel can start its weight-only prologue meanwhile.
// (The forward kernels store out straight into the caller's pinned buffer.)
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

struct HostRowsIn {
    const uint4 *src;  // pinned host memory, as the device sees it
    uint4 *dst;        // workspace
    size_t n16;        // 16-byte words
};

__global__ void __launch_bounds__(256) host_rows_in_kernel(const HostRowsIn p)
{
    pdl_trigger();  // the next kernel may start its prologue; its wait still sees these stores
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < p.n16; i += (size_t)gridDim.x * blockDim.x)
        p.dst[i] = __ldcv(p.src + i);  // fetched again every call: the host rewrites the buffer between calls
}

}  // namespace

cudaError_t launch_host_rows_in(const void *src_dev, void *dst, size_t bytes, cudaStream_t s)
{
    HostRowsIn p;
    p.src = static_cast<const uint4 *>(src_dev);
    p.dst = static_cast<uint4 *>(dst);
    p.n16 = bytes / 16;
    const size_t blocks = (p.n16 + 255) / 256;
    const unsigned grid = (unsigned)(blocks < 4 * 148 ? (blocks ? blocks : 1) : 4 * 148);
    // a plain launch (no programmatic serialization): the copy must not start
    // before every earlier kernel on the stream, which may still read dst,
    // has finished
    host_rows_in_kernel<<<grid, 256, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace moe
