// ffn_prefill.cu -- the masked SwiGLU FFN for many tokens (prefill).
//
// WIDE, technical summary sections 2.B and 2.C.  After wide_reorder (per
// group stable partition, signature order, per-tile unions; no host sync):
//   gather_gemm      SwiGLU mode: each (group, row tile) work item gathers
//                    its active token rows and multiplies them by the
//                    group's [W_gate; W_up] slab on tcgen05; the epilogue
//                    writes silu(gate) * up into H at signature-order rows
//                    (only kept (token, group) pairs are ever written)
//   tile_union_gemm  out = H W_down^T over each signature tile's union of
//                    kept groups, written at the tokens' own rows; a row
//                    whose token skips a group enters that group's K steps
//                    as zeros (set in shared memory; H there is never
//                    written)
// The kernels live in prefill_gemm.cu.
#include "common.cuh"
#include "host.h"

namespace wide {

namespace {
constexpr int kBM = 128;
}

size_t ffn_prefill_workspace(const wide_ffn_dims *d)
{
    const size_t wl = wide_worklist_bytes(d->tokens, d->inter / d->group_size, kBM);
    if (wl == 0)
        return 0;
    return align_up(wl, 1024) + align_up((size_t)d->tokens * (size_t)d->inter * 2, 1024);
}

int ffn_prefill_core(const void *x, const void *wg, const void *wu, const void *wd,
                     const uint32_t *mask, const FfnPrefillOut &o, int64_t T, int64_t H,
                     int64_t I, int64_t gs, const wide_worklist *ext_wl, void *ws,
                     cudaStream_t s)
{
    const int64_t G = I / gs;
    const size_t wl_bytes = wide_worklist_bytes(T, G, kBM);
    wide_worklist wl;
    int rc = WIDE_OK;
    if (ext_wl)
        wl = *ext_wl;
    else if ((rc = wide_worklist_carve(ws, wl_bytes, T, G, kBM, &wl)))
        return rc;
    __nv_bfloat16 *hbuf =
        reinterpret_cast<__nv_bfloat16 *>(static_cast<char *>(ws) + align_up(wl_bytes, 1024));

    CUtensorMap tg, tu, th, td;
    if (!make_tmap_2d(&tg, wg, I, H, H, 2, (uint32_t)gs, 64, true) ||
        !make_tmap_2d(&tu, wu, I, H, H, 2, (uint32_t)gs, 64, true) ||
        !make_tmap_2d(&th, hbuf, T, I, I, 2, kBM, 64, true) ||
        !make_tmap_2d(&td, wd, H, I, I, 2, 256, 64, true))
        return WIDE_CUDA_FAIL();

    if (!ext_wl && (rc = reorder_launch(mask, T, G, kBM, &wl, s)))
        return rc;

    GemmArgs ga = {};
    ga.a = static_cast<const __nv_bfloat16 *>(x);
    ga.count = wl.count;
    ga.perm = wl.perm;
    ga.items = wl.items;
    ga.n_items_p = wl.n_items;
    ga.sig_pos = wl.sig_pos;
    ga.out0 = hbuf;
    ga.T = (int)T;
    ga.K = (int)H;
    ga.out_ld = (int)I;
    ga.gs = (int)gs;
    ga.status = status_ptr();
    const int max_items = (int)(G * ((T + kBM - 1) / kBM));
    if ((rc = gather_gemm_launch(GEMM_SWIGLU, tg, tu, ga, max_items, KID_PREFILL_GATEUP, s)))
        return rc;

    UnionArgs ua = {};
    ua.tile_union = wl.tile_union;
    ua.sig_perm = wl.sig_perm;
    ua.mask = mask;
    ua.h = hbuf;
    ua.T = (int)T;
    ua.N = (int)H;
    ua.W = (int)((G + 31) / 32);
    ua.gs = (int)gs;
    ua.ld = (int)I;
    ua.out_sum = o.out_sum;
    ua.res_f32 = o.res_f32;
    ua.out_total = o.out_total;
    ua.status = status_ptr();
    return tile_union_gemm_launch(th, td, ua, KID_PREFILL_DOWN, s);
}

int ffn_prefill_launch(const void *x, const void *wg, const void *wu, const void *wd,
                       const uint32_t *mask, void *out, const wide_ffn_dims *d,
                       const wide_worklist *ext_wl, void *ws, cudaStream_t s)
{
    FfnPrefillOut o = {};
    o.out_sum = static_cast<__nv_bfloat16 *>(out);
    return ffn_prefill_core(x, wg, wu, wd, mask, o, d->tokens, d->hidden, d->inter,
                            d->group_size, ext_wl, ws, s);
}

}  // namespace wide
