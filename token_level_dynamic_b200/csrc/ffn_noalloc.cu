// ffn_noalloc.cu -- wide_ffn_masked_noalloc: the decode FFN for callers that
// cannot allocate device memory.
//
// Some callers have no way to provide device scratch: a host framework that
// owns the whole device memory pool and hands out no workspace, or a
// latency-critical loop where cudaMalloc/cudaFree would synchronise the
// device.  This entry point runs the same decode kernels as
// wide_ffn_masked's decode path, but keeps their scratch in the file-scope
// device arrays below instead of a caller workspace: for the channel-split
// kernel (bf16, the usual case) its fp32 [T][hidden] accumulator and arrival
// counter, for the GEMV kernels (fp32, and bf16 shapes outside the split
// kernel's limits) the fp32 intermediate h = silu(gate) * up of up to 32
// tokens.  The second array holds the barrier words the decode path's
// interface carries (unused by the current kernels).
//
// The arrays are module globals: every GPU that loads the library holds
// WIDE_NOALLOC_SCRATCH_BYTES (+ 256) bytes of device memory for them until
// the process exits.  All calls on a device share them and they keep the
// last call's contents.  No call depends on those contents: the split
// kernel's launch zeroes, on the stream, the accumulator and counter it is
// about to use, and the GEMV kernels read h only at the (token, group) pairs
// the same call wrote.  Two calls whose work overlaps on the GPU (different
// streams without ordering) race on the arrays.
//
// In host code the arrays' names are host-side stand-ins, not device
// addresses: the addresses are looked up with cudaGetSymbolAddress, with the
// device current, once per device and CUDA context (device_symbol_address),
// so after a cudaDeviceReset the next call looks them up again.  The first
// call on a device (or in a new context) does that lookup; make it before
// any stream capture.
#include <cuda_runtime.h>
#include <mutex>

#include "host.h"
#include "wide.h"

static __device__ __align__(256) float g_noalloc_scratch[WIDE_NOALLOC_SCRATCH_BYTES / sizeof(float)];
static __device__ __align__(256) uint32_t g_noalloc_bar[64];

namespace wide {
namespace {

// Device addresses of this device's copies of g_noalloc_scratch and
// g_noalloc_bar (see device_symbol_address).
bool noalloc_arrays(float **scratch, uint32_t **bar)
{
    static DeviceSymbolCache cs, cb;
    *scratch = static_cast<float *>(device_symbol_address(cs, &g_noalloc_scratch));
    *bar = static_cast<uint32_t *>(device_symbol_address(cb, &g_noalloc_bar));
    return *scratch && *bar;
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
    return ffn_decode_run(d_x, d_w_gate, d_w_up, d_w_down, d_group_mask, d_out, d, scratch,
                          WIDE_NOALLOC_SCRATCH_BYTES, bar, static_cast<cudaStream_t>(stream));
}
