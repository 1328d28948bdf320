// norm.cu -- RMSNorm over rows (the Llama block's input norms):
// y[t] = x[t] / sqrt(mean(x[t]^2) + eps) * gamma, accumulated in fp32, bf16 out.
#include "common.cuh"
#include "host.h"

namespace wide {
namespace {

template <typename TX>
__global__ void __launch_bounds__(256)
    rmsnorm_rows(const TX *__restrict__ x, const __nv_bfloat16 *__restrict__ gamma,
                 __nv_bfloat16 *__restrict__ y, int H, float eps)
{
    __shared__ float red[8];
    const int t = blockIdx.x;
    const TX *xr = x + (size_t)t * H;
    float ss = 0.f;
    for (int k = threadIdx.x; k < H; k += 256) {
        const float v = to_f32(xr[k]);
        ss = fmaf(v, v, ss);
    }
    for (int off = 16; off; off >>= 1)
        ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if ((threadIdx.x & 31) == 0)
        red[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
    for (int w = 0; w < 8; ++w)
        tot += red[w];
    const float r = 1.0f / sqrtf(tot / (float)H + eps);
    for (int k = threadIdx.x; k < H; k += 256)
        y[(size_t)t * H + k] = __float2bfloat16_rn(to_f32(xr[k]) * r * __bfloat162float(gamma[k]));
}

}  // namespace

int rmsnorm_bf16_launch(const void *x, const void *gamma, void *y, int T, int H, float eps,
                        cudaStream_t s)
{
    if (T <= 0)
        return WIDE_OK;
    LaunchScope scope(KID_RMSNORM, s);
    rmsnorm_rows<__nv_bfloat16><<<T, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(x),
                                                  static_cast<const __nv_bfloat16 *>(gamma),
                                                  static_cast<__nv_bfloat16 *>(y), H, eps);
    return launch_status();
}

int rmsnorm_f32_launch(const float *x, const void *gamma, void *y, int T, int H, float eps,
                       cudaStream_t s)
{
    if (T <= 0)
        return WIDE_OK;
    LaunchScope scope(KID_RMSNORM, s);
    rmsnorm_rows<float><<<T, 256, 0, s>>>(x, static_cast<const __nv_bfloat16 *>(gamma),
                                          static_cast<__nv_bfloat16 *>(y), H, eps);
    return launch_status();
}

}  // namespace wide
