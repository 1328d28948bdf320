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

// The same for H = NCH * 2048 (H <= 8192): thread i caches the 8-element
// chunks i, i + 256, ... of its row in registers, so the row is read once
// with 16-byte loads and written with 16-byte stores.
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&v)[8])
{
    bf16x8_to_f32(*reinterpret_cast<const uint4 *>(p), v);
}
__device__ __forceinline__ void load8(const float *p, float (&v)[8])
{
    const float4 a = reinterpret_cast<const float4 *>(p)[0], b = reinterpret_cast<const float4 *>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

template <typename TX, int NCH>
__global__ void __launch_bounds__(256)
    rmsnorm_rows_vec(const TX *__restrict__ x, const __nv_bfloat16 *__restrict__ gamma,
                     __nv_bfloat16 *__restrict__ y, int H, float eps)
{
    __shared__ float red[8];
    const int t = blockIdx.x, tid = threadIdx.x;
    const TX *xr = x + (size_t)t * H;
    float v[NCH][8];
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        load8(xr + (size_t)(c * 256 + tid) * 8, v[c]);
#pragma unroll
        for (int e = 0; e < 8; ++e)
            ss = fmaf(v[c][e], v[c][e], ss);
    }
    for (int off = 16; off; off >>= 1)
        ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if ((tid & 31) == 0)
        red[tid >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w)
        tot += red[w];
    const float r = 1.0f / sqrtf(tot / (float)H + eps);
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        const int k = (c * 256 + tid) * 8;
        float gv[8];
        load8(gamma + k, gv);
        uint4 o;
        uint32_t *ow = reinterpret_cast<uint32_t *>(&o);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 p2 = __floats2bfloat162_rn(v[c][2 * e] * r * gv[2 * e],
                                                            v[c][2 * e + 1] * r * gv[2 * e + 1]);
            ow[e] = *reinterpret_cast<const uint32_t *>(&p2);
        }
        *reinterpret_cast<uint4 *>(y + (size_t)t * H + k) = o;
    }
}

template <typename TX>
int rmsnorm_launch(const TX *x, const __nv_bfloat16 *gamma, __nv_bfloat16 *y, int T, int H,
                   float eps, cudaStream_t s)
{
    LaunchScope scope(KID_RMSNORM, s);
    const bool vec = H % 2048 == 0 && H <= 8192 &&
                     ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(gamma) |
                       reinterpret_cast<uintptr_t>(y)) & 15u) == 0;
    if (vec && H == 2048)
        rmsnorm_rows_vec<TX, 1><<<T, 256, 0, s>>>(x, gamma, y, H, eps);
    else if (vec && H == 4096)
        rmsnorm_rows_vec<TX, 2><<<T, 256, 0, s>>>(x, gamma, y, H, eps);
    else if (vec && H == 6144)
        rmsnorm_rows_vec<TX, 3><<<T, 256, 0, s>>>(x, gamma, y, H, eps);
    else if (vec && H == 8192)
        rmsnorm_rows_vec<TX, 4><<<T, 256, 0, s>>>(x, gamma, y, H, eps);
    else
        rmsnorm_rows<TX><<<T, 256, 0, s>>>(x, gamma, y, H, eps);
    return launch_status();
}

}  // namespace

int rmsnorm_bf16_launch(const void *x, const void *gamma, void *y, int T, int H, float eps,
                        cudaStream_t s)
{
    if (T <= 0)
        return WIDE_OK;
    return rmsnorm_launch(static_cast<const __nv_bfloat16 *>(x),
                          static_cast<const __nv_bfloat16 *>(gamma),
                          static_cast<__nv_bfloat16 *>(y), T, H, eps, s);
}

int rmsnorm_f32_launch(const float *x, const void *gamma, void *y, int T, int H, float eps,
                       cudaStream_t s)
{
    if (T <= 0)
        return WIDE_OK;
    return rmsnorm_launch(x, static_cast<const __nv_bfloat16 *>(gamma),
                          static_cast<__nv_bfloat16 *>(y), T, H, eps, s);
}

}  // namespace wide
