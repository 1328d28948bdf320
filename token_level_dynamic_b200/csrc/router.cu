// router.cu -- the bottleneck router that produces the packed group masks.
//
// WIDE, technical summary section 2.A ("router architecture"): a light
// bottleneck router maps a block's input activations to one execute/skip
// decision per group.  Here:  z = act(x W_r1^T),  logit = z W_r2^T + b_r2,
// execute = logit > 0, written as the packed token-major mask words that
// every masked kernel reads.
//
// More than 32 tokens: one launch of gather_gemm in router mode
// (prefill_gemm.cu): every 128-token tile of x (TMA) times all of W_r1 (N =
// bottleneck width) on tcgen05, fp32 in tensor memory; its epilogue applies
// the activation and the W_r2 products on CUDA cores, one token per thread,
// and stores the mask words directly.
//
// Up to 32 tokens (decode): route_small, CUDA cores, clusters of 8 CTAs.  A
// cluster takes 2 tokens; CTA k of it takes bottleneck units
// [k R/8, (k+1) R/8).  One thread bulk-copies those rows of W_r1 and the
// cluster's x rows into shared memory (all in flight at once, one mbarrier)
// while the others stage the matching columns of W_r2 as fp32; then each
// warp forms z for its units and each thread partial logits [2][G] for its
// share, in shared memory.  After a cluster barrier every CTA sums the 8
// partials of its share of the (token, mask word) items through distributed
// shared memory, adds the bias and takes the decisions with a warp ballot
// (lane j = group 32 w + j).  W_r1 is read from HBM once per call (the
// clusters of a batch share it through L2).
#include "common.cuh"
#include "host.h"

#include <cooperative_groups.h>

namespace wide {

namespace cg = cooperative_groups;

namespace {
constexpr int kBM = 128;
constexpr int kRTok = 2;         // tokens per cluster
constexpr int kRCluster = 8;     // CTAs per cluster
constexpr int kRThreads = 256;
constexpr int kRMaxTokens = 32;  // route_small's range

__device__ __forceinline__ float router_act(float v, int act)
{
    return act == WIDE_ACT_SILU ? silu_f32(v) : fmaxf(v, 0.f);
}

// Shared memory, in order: mbarrier (16 bytes), W_r1 rows [R/8][H] bf16,
// x [kRTok][H] bf16, W_r2 columns [G][R/8] fp32, z [kRTok][R/8] fp32,
// partial logits [kRTok][G] fp32.
size_t route_small_smem(int H, int R, int G)
{
    const size_t RB = (size_t)(R / kRCluster);
    return 16 + RB * H * 2 + (size_t)kRTok * H * 2 + (size_t)G * RB * 4 + kRTok * RB * 4 +
           (size_t)kRTok * G * 4;
}

__global__ void __launch_bounds__(kRThreads, 1)
    route_small(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ w1,
                const __nv_bfloat16 *__restrict__ w2, const float *__restrict__ b2,
                uint32_t *__restrict__ mask, float *__restrict__ logits, int T, int H, int R,
                int G, int act, int32_t *status)
{
    extern __shared__ __align__(16) uint8_t sm[];
    cg::cluster_group cluster = cg::this_cluster();
    const int k = (int)cluster.block_rank();
    const int t0 = (int)(blockIdx.x / kRCluster) * kRTok;
    const int nt = min(kRTok, T - t0);
    const int RB = R / kRCluster, r0 = k * RB;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm);
    __nv_bfloat16 *w1s = reinterpret_cast<__nv_bfloat16 *>(sm + 16);
    __nv_bfloat16 *xs = w1s + (size_t)RB * H;
    float *w2s = reinterpret_cast<float *>(xs + (size_t)kRTok * H);
    float *zs = w2s + G * RB;
    float *ps = zs + kRTok * RB;

    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
        const uint32_t row_bytes = (uint32_t)H * 2u;
        mbar_arrive_expect_tx(bar, row_bytes * (uint32_t)(RB + nt));
        for (int rr = 0; rr < RB; ++rr)
            bulk_load(w1s + (size_t)rr * H, w1 + (size_t)(r0 + rr) * H, row_bytes, bar);
        for (int tt = 0; tt < nt; ++tt)
            bulk_load(xs + (size_t)tt * H, x + (size_t)(t0 + tt) * H, row_bytes, bar);
    }
    // x rows past T are zeros
    const int hc = H / 8;
    for (int i = nt * hc + threadIdx.x; i < kRTok * hc; i += kRThreads)
        reinterpret_cast<uint4 *>(xs)[i] = make_uint4(0u, 0u, 0u, 0u);
    // (W_r2 loads issued in batches of 8 per thread before their stores, so
    // a thread has 8 requests in flight instead of one)
    // this CTA's columns of W_r2 as fp32, [g][rr]
    const int np = G * (RB / 2);
    for (int i0 = threadIdx.x; i0 < np; i0 += 8 * kRThreads) {
        __nv_bfloat162 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = i0 + u * kRThreads;
            const int g = i / (RB / 2), p = i - g * (RB / 2);
            if (i < np)
                v[u] = reinterpret_cast<const __nv_bfloat162 *>(w2 + (size_t)g * R + r0)[p];
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = i0 + u * kRThreads;
            if (i < np) {
                const float2 f = __bfloat1622float2(v[u]);
                w2s[2 * i] = f.x;
                w2s[2 * i + 1] = f.y;
            }
        }
    }
    __syncthreads();  // barrier initialised, W_r2 staged
    if (!mbar_wait(bar, 0))
        set_status(status, WIDE_DEV_TIMEOUT);

    // z[tt][rr] = act(x[t0 + tt] . W_r1[r0 + rr]): one warp per unit
    for (int rr = warp; rr < RB; rr += kRThreads / 32) {
        const uint4 *wr = reinterpret_cast<const uint4 *>(w1s + (size_t)rr * H);
        float acc[kRTok] = {};
#pragma unroll 4
        for (int ch = lane; ch < hc; ch += 32) {
            float wv[8];
            bf16x8_to_f32(wr[ch], wv);
#pragma unroll
            for (int tt = 0; tt < kRTok; ++tt) {
                float xv[8];
                bf16x8_to_f32(reinterpret_cast<const uint4 *>(xs + (size_t)tt * H)[ch], xv);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    acc[tt] = fmaf(wv[e], xv[e], acc[tt]);
            }
        }
#pragma unroll
        for (int tt = 0; tt < kRTok; ++tt) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                acc[tt] += __shfl_xor_sync(0xffffffffu, acc[tt], o);
        }
        if (lane < kRTok)
            zs[lane * RB + rr] = router_act(acc[lane], act);
    }
    __syncthreads();

    // partial logits of this CTA's units: ps[tt][g] = z[tt] . W_r2[g][r0 : r0 + RB]
    for (int i = threadIdx.x; i < kRTok * G; i += kRThreads) {
        const int tt = i / G, g = i - tt * G;
        const float *wg = w2s + g * RB;
        const float *z = zs + tt * RB;
        float acc = 0.f;
        for (int rr = 0; rr < RB; ++rr)
            acc = fmaf(z[rr], wg[rr], acc);
        ps[i] = acc;
    }
    cluster.sync();

    // sum the 8 partials of item (tt, wd), items dealt round-robin to warps
    const int nw = (G + 31) >> 5;
    for (int it = k * (kRThreads / 32) + warp; it < nt * nw; it += kRCluster * (kRThreads / 32)) {
        const int tt = it / nw, wd = it - tt * nw;
        const int g = wd * 32 + lane;
        float lg = 0.f;
        if (g < G) {
            lg = b2 ? b2[g] : 0.f;
#pragma unroll
            for (int q = 0; q < kRCluster; ++q)
                lg += cluster.map_shared_rank(ps, q)[tt * G + g];
        }
        const uint32_t bits = __ballot_sync(0xffffffffu, g < G && lg > 0.f);
        if (lane == 0)
            mask[(size_t)(t0 + tt) * nw + wd] = bits;
        if (logits && g < G)
            logits[(size_t)(t0 + tt) * G + g] = lg;
    }
    cluster.sync();  // no CTA leaves while another still reads its partials
}

int route_small_launch(const void *x, const void *w1, const void *w2, const float *b2,
                       uint32_t *mask, float *logits, int T, int H, int R, int G, int act,
                       cudaStream_t s)
{
    const size_t smem = route_small_smem(H, R, G);
    if (!raise_smem_limit(reinterpret_cast<const void *>(route_small), smem))
        return WIDE_CUDA_FAIL();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(((T + kRTok - 1) / kRTok) * kRCluster));
    cfg.blockDim = dim3(kRThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kRCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    LaunchScope scope(KID_ROUTER_SMALL, s);
    if (cudaLaunchKernelEx(&cfg, route_small, static_cast<const __nv_bfloat16 *>(x),
                           static_cast<const __nv_bfloat16 *>(w1),
                           static_cast<const __nv_bfloat16 *>(w2), b2, mask, logits, T, H, R, G,
                           act, status_ptr()) != cudaSuccess)
        return WIDE_CUDA_FAIL();
    return WIDE_OK;
}
}  // namespace

int route_launch(const void *x, const void *w_r1, const void *w_r2, const float *b_r2,
                 uint32_t *mask, float *logits, const wide_router_dims *d, cudaStream_t s)
{
    const int64_t T = d->tokens, H = d->hidden, R = d->bottleneck, G = d->groups;
    if (T <= kRMaxTokens && route_small_smem((int)H, (int)R, (int)G) <= 227u * 1024u)
        return route_small_launch(x, w_r1, w_r2, b_r2, mask, logits, (int)T, (int)H, (int)R,
                                  (int)G, d->act, s);
    CUtensorMap tw, tx;
    // W_r1 in two boxes of R/2 rows x 64 columns, x in boxes of 128 rows x 64
    // columns (128-byte swizzle, the tensor cores' operand layout)
    if (!make_tmap_2d(&tw, w_r1, (uint64_t)R, (uint64_t)H, (uint64_t)H, 2, (uint32_t)(R / 2), 64,
                      true) ||
        !make_tmap_2d(&tx, x, (uint64_t)T, (uint64_t)H, (uint64_t)H, 2, kBM, 64, true))
        return WIDE_CUDA_FAIL();
    GemmArgs ga = {};
    ga.a = static_cast<const __nv_bfloat16 *>(x);
    ga.T = (int)T;
    ga.K = (int)H;
    ga.m_tiles = (int)((T + kBM - 1) / kBM);
    ga.w_r2 = static_cast<const __nv_bfloat16 *>(w_r2);
    ga.b_r2 = b_r2;
    ga.mask_out = mask;
    ga.logits_out = logits;
    ga.rn = (int)R;
    ga.n_groups = (int)G;
    ga.act = d->act;
    ga.status = status_ptr();
    return gather_gemm_launch(GEMM_ROUTER, tw, tx, ga, ga.m_tiles, KID_ROUTER, s);
}

}  // namespace wide

using namespace wide;

int wide_route(const void *d_x, const void *d_w_r1, const void *d_w_r2, const float *d_b_r2,
               uint32_t *d_mask, float *d_logits, const wide_router_dims *d, void *stream)
{
    if (!d || d->tokens < 0 || d->hidden <= 0 || d->bottleneck <= 0 || d->groups <= 0 ||
        (d->act != WIDE_ACT_RELU && d->act != WIDE_ACT_SILU))
        return WIDE_EINVAL;
    if (d->tokens == 0)
        return WIDE_OK;
    if (!d_x || !d_w_r1 || !d_w_r2 || !d_mask)
        return WIDE_EINVAL;
    if (d->hidden % 64 != 0 || d->bottleneck % 32 != 0 || d->bottleneck > 256 ||
        d->groups > 1024 || d->tokens * d->hidden >= ((int64_t)1 << 31))
        return WIDE_EUNSUPPORTED;
    if (!aligned16(d_x) || !aligned16(d_w_r1) || !aligned16(d_w_r2) ||
        (reinterpret_cast<uintptr_t>(d_mask) & 3u) != 0 ||
        (d_b_r2 && (reinterpret_cast<uintptr_t>(d_b_r2) & 3u) != 0) ||
        (d_logits && (reinterpret_cast<uintptr_t>(d_logits) & 3u) != 0))
        return WIDE_EUNSUPPORTED;
    return route_launch(d_x, d_w_r1, d_w_r2, d_b_r2, d_mask, d_logits, d,
                        static_cast<cudaStream_t>(stream));
}
