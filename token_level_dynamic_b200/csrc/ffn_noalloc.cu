// ffn_noalloc.cu -- wide_ffn_masked_noalloc: the decode FFN for callers that
// cannot allocate device memory.
//
// Some callers have no way to provide device scratch: a host framework that
// owns the whole device memory pool and hands out no workspace, or a
// latency-critical loop where cudaMalloc/cudaFree would synchronise the
// device.  This entry point runs the same decode kernels as
// wide_ffn_masked's decode path, but keeps their scratch in the file-scope
// device array below instead of a caller workspace: for the persistent
// kernels (bf16, the usual case) their fp32 accumulator and arrival counter,
// for the GEMV kernels (fp32, and bf16 shapes outside the persistent
// kernels' limits) the fp32 intermediate h = silu(gate) * up of up to 32
// tokens.
//
// The array is a module global: every GPU that loads the library holds
// WIDE_NOALLOC_SCRATCH_BYTES bytes of device memory for it until the
// process exits.  All calls on a device share it and it keeps the last
// call's contents.  No call depends on those contents: a persistent
// kernel's launch zeroes, on the stream, the accumulator and counter it is
// about to use, and the GEMV kernels read h only at the (token, group) pairs
// the same call wrote.  Two calls whose work overlaps on the GPU (different
// streams without ordering) race on the array.
//
// In host code the array's name is a host-side stand-in, not a device
// address: the address is looked up with cudaGetSymbolAddress, with the
// device current, once per device and CUDA context (device_symbol_address),
// so after a cudaDeviceReset the next call looks it up again.  The first
// call on a device (or in a new context) does that lookup; make it before
// any stream capture.
#include <cuda_runtime.h>
#include <mutex>

#include "host.h"
#include "wide.h"

static __device__ __align__(256) float g_noalloc_scratch[WIDE_NOALLOC_SCRATCH_BYTES / sizeof(float)];

namespace wide {
namespace {

// Device address of this device's copy of g_noalloc_scratch (see
// device_symbol_address).
float *noalloc_scratch()
{
    static DeviceSymbolCache cs;
    return static_cast<float *>(device_symbol_address(cs, &g_noalloc_scratch));
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
    float *scratch = noalloc_scratch();
    if (!scratch)
        return WIDE_CUDA_FAIL();
    return ffn_decode_run(d_x, d_w_gate, d_w_up, d_w_down, d_group_mask, d_out, d, scratch,
                          WIDE_NOALLOC_SCRATCH_BYTES, static_cast<cudaStream_t>(stream));
}
