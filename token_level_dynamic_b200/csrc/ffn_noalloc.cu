// ffn_noalloc.cu -- wide_ffn_masked_noalloc: the decode FFN for callers that
// cannot allocate device memory.
//
// Some callers have no way to provide device scratch: a host framework that
// owns the whole device memory pool and hands out no workspace, or a
// latency-critical loop where cudaMalloc/cudaFree would synchronise the
// device.  This entry point runs the same decode kernels as
// wide_ffn_masked's decode path, but keeps their scratch -- the fp32
// intermediate h = silu(gate) * up of up to 32 tokens, and the two words of
// the fused kernel's grid barrier -- in the file-scope device arrays below
// instead of a caller workspace.
//
// The array is a module global: every GPU that loads the library holds
// WIDE_NOALLOC_SCRATCH_BYTES of device memory for it until the process exits.
// All calls on a device share it and it keeps the last call's contents.  The
// kernels write every entry they later read (kept (token, group) pairs only),
// so nothing in it needs clearing between calls; but two calls whose work
// overlaps on the GPU (different streams without ordering) race on it.
#include <cuda_runtime.h>
#include <mutex>

#include "host.h"
#include "wide.h"

static __device__ __align__(256) float g_noalloc_scratch[WIDE_NOALLOC_SCRATCH_BYTES / sizeof(float)];
static __device__ __align__(256) uint32_t g_noalloc_bar[64];

namespace wide {
namespace {

// Device addresses of this device's copies of g_noalloc_scratch and
// g_noalloc_bar.  In host code the arrays' names are only host-side
// stand-ins, so the addresses are looked up with cudaGetSymbolAddress once
// per device, with that device current.
bool noalloc_arrays(float **scratch, uint32_t **bar)
{
    static std::mutex mu;
    static void *ptrs[64][2] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return false;
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[dev][0]) {
        void *p = nullptr, *q = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess ||
            cudaGetSymbolAddress(&q, g_noalloc_bar) != cudaSuccess)
            return false;
        ptrs[dev][0] = p;
        ptrs[dev][1] = q;
    }
    *scratch = static_cast<float *>(ptrs[dev][0]);
    *bar = static_cast<uint32_t *>(ptrs[dev][1]);
    return true;
}

}  // namespace
}  // namespace wide

using namespace wide;

extern "C" int wide_ffn_masked_noalloc(const void *d_x, const void *d_w_gate, const void *d_w_up,
                                       const void *d_w_down, const uint32_t *d_group_mask,
                                       void *d_out, const wide_ffn_dims *d, void *stream)
{
    if (!ffn_dims_ok(d))
        return WIDE_EINVAL;
    if (d->path != WIDE_PATH_AUTO && d->path != WIDE_PATH_DECODE)
        return WIDE_EUNSUPPORTED;
    if (d->tokens == 0)
        return WIDE_OK;
    if (!d_x || !d_w_gate || !d_w_up || !d_w_down || !d_group_mask || !d_out)
        return WIDE_EINVAL;
    if (!ffn_shape_supported(d, WIDE_PATH_DECODE))
        return WIDE_EUNSUPPORTED;
    if (!aligned16(d_x) || !aligned16(d_w_gate) || !aligned16(d_w_up) || !aligned16(d_w_down) ||
        !aligned16(d_out))
        return WIDE_EUNSUPPORTED;
    if (ffn_decode_h_bytes(d) > (size_t)WIDE_NOALLOC_SCRATCH_BYTES)
        return WIDE_ETOOLARGE;
    float *scratch = nullptr;
    uint32_t *bar = nullptr;
    if (!noalloc_arrays(&scratch, &bar))
        return WIDE_CUDA_FAIL();
    return ffn_decode_run(d_x, d_w_gate, d_w_up, d_w_down, d_group_mask, d_out, d, scratch, bar,
                          static_cast<cudaStream_t>(stream));
}
