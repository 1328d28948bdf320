// router.cu -- the bottleneck router that produces the packed group masks.
//
// WIDE, technical summary section 2.A ("router architecture"): a light
// bottleneck router maps a block's input activations to one execute/skip
// decision per group.  Here:  z = act(x W_r1^T),  logit = z W_r2^T + b_r2,
// execute = logit > 0, written as the packed token-major mask words that
// every masked kernel reads.
//
// One launch of gather_gemm in router mode (prefill_gemm.cu): every 128-token
// tile of x times all of W_r1 (N = bottleneck width) on tcgen05, fp32 in
// tensor memory; its epilogue applies the activation and the W_r2 products on
// CUDA cores, one token per thread, and stores the mask words directly.
#include "common.cuh"
#include "host.h"

namespace wide {

namespace {
constexpr int kBM = 128;
}

int route_launch(const void *x, const void *w_r1, const void *w_r2, const float *b_r2,
                 uint32_t *mask, float *logits, const wide_router_dims *d, cudaStream_t s)
{
    const int64_t T = d->tokens, H = d->hidden, R = d->bottleneck, G = d->groups;
    CUtensorMap tw;
    // W_r1 in two boxes of R/2 rows x 64 columns (128-byte swizzle)
    if (!make_tmap_2d(&tw, w_r1, (uint64_t)R, (uint64_t)H, (uint64_t)H, 2, (uint32_t)(R / 2), 64,
                      true))
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
    return gather_gemm_launch(GEMM_ROUTER, tw, tw, ga, ga.m_tiles, KID_ROUTER, s);
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
