// attn_decode.cu -- the masked attention half of a decode step, and the
// whole decode layer.
//
// WIDE, technical summary section 2.A: attention prunes groups of query
// heads aligned with GQA, chosen per token.  A token that skips group j does
// not compute the query heads of j, attends nothing with them, and the
// o_proj columns of those heads are not read for it.  Every token's K and V
// are still computed and appended to the cache (later queries need them).
//
// Kernels (T <= 32 tokens, one new token per sequence):
//   decode_qkv    GEMV over the Wq rows of the batch's kept head groups and
//                 all Wk/Wv rows.  RMSNorm is folded in: x * gamma is staged
//                 in shared memory, each CTA of the K-split cluster also sums
//                 x^2 over its slice, and after the cluster-wide reduction the
//                 dot products are scaled by 1 / sqrt(mean(x^2) + eps).  RoPE
//                 (rotate-half pairs (c, c + hd/2), angles in double) is then
//                 applied to q and k; q goes to a workspace, k and v to the
//                 caches at position cache_len.
//   decode_attn   one 8-CTA cluster per (sequence, KV head) the sequence's
//                 token keeps (a skipped group's cluster exits at once and
//                 reads no K/V); CTA s takes one slice of the keys, computes
//                 scores, a partial softmax and P.V for the group's query
//                 heads; the slices are merged with log-sum-exp weights
//                 through distributed shared memory.
// o_proj and the FFN run through the decode down/gate-up GEMVs (groups of
// rep*head_dim o_proj columns), with the residual adds in their epilogues.
#include <cooperative_groups.h>

#include "common.cuh"
#include "host.h"

namespace cg = cooperative_groups;

namespace wide {
namespace {

constexpr int kHD = 128;           // head dimension this path is built for
constexpr int kStages = 3;
constexpr int kNTok = 32;
constexpr int kSplits = 8;         // key slices (cluster size) in decode_attn
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    const uint32_t a = smem_u32(p);
    return p + (((a + 1023u) & ~1023u) - a);
}

__device__ __forceinline__ uint32_t token_group_mask(const uint32_t *mask, int T, int W, int g)
{
    const int lane = threadIdx.x & 31;
    const uint32_t a = lane < T ? (mask[(size_t)lane * W + (g >> 5)] >> (g & 31)) & 1u : 0u;
    return __ballot_sync(0xffffffffu, a);
}

// ------------------------------------------------------------- decode_qkv
struct QkvArgs {
    const __nv_bfloat16 *x;        // [T][H]
    const __nv_bfloat16 *gamma;    // [H]
    const uint32_t *head_mask;     // [T][Wh]
    float *q;                      // [T][n_q * hd]
    __nv_bfloat16 *k_cache;        // [n_seq][n_kv][cap][hd]
    __nv_bfloat16 *v_cache;
    int T, H, n_q, n_kv, Wh, kslice;
    int64_t cache_len, cache_cap;
    float eps;
    double theta;
    int32_t *status;
};

__global__ void __launch_bounds__(kHD)
    decode_qkv(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const QkvArgs a)
{
    constexpr uint32_t kTile = kHD * 128u;    // 128 rows x 64 bf16
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *stages = smem;                                          // [kStages][kTile]
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kStages * kTile);
    int *act = reinterpret_cast<int *>(full + kStages);              // [32]
    float *pss = reinterpret_cast<float *>(act + kNTok);             // [32] partial sum x^2
    float *rv = pss + kNTok;                                          // [hd] roped exchange
    float *xs = reinterpret_cast<float *>(smem + kStages * kTile + 1024);  // [nact][kslice]

    cg::cluster_group cluster = cg::this_cluster();
    const int KS = (int)gridDim.x;
    const int s = (int)blockIdx.x;
    const int rb = (int)blockIdx.y;         // row block: q heads, then k heads, then v heads
    const int c = (int)threadIdx.x;
    const int rep = a.n_q / a.n_kv;

    int kind, head;
    const CUtensorMap *map;
    if (rb < a.n_q) {
        kind = 0; head = rb; map = &tm_q;
    } else if (rb < a.n_q + a.n_kv) {
        kind = 1; head = rb - a.n_q; map = &tm_k;
    } else {
        kind = 2; head = rb - a.n_q - a.n_kv; map = &tm_v;
    }
    const uint32_t all = a.T >= 32 ? 0xffffffffu : ((1u << a.T) - 1u);
    const uint32_t tmask = kind == 0 ? token_group_mask(a.head_mask, a.T, a.Wh, head / rep) : all;
    if (tmask == 0u)
        return;  // no token of the batch keeps this query head's group
    const int nact = __popc(tmask);
    const int k0 = s * a.kslice;
    const int ntile = a.kslice / 64;

    if (c < 32 && ((tmask >> c) & 1u))
        act[__popc(tmask & ((1u << c) - 1u))] = c;
    if (c < kNTok)
        pss[c] = 0.f;
    if (c == 0) {
        for (int st = 0; st < kStages; ++st)
            mbar_init(&full[st], 1);
        fence_mbar_init();
        tma_prefetch_desc(map);
    }
    __syncthreads();

    auto issue = [&](int kt) {
        const int st = kt % kStages;
        mbar_arrive_expect_tx(&full[st], kTile);
        tma_load_2d(stages + st * kTile, map, k0 + kt * 64, head * kHD, &full[st]);
    };
    int issued = 0;
    if (c == 0)
        for (; issued < kStages && issued < ntile; ++issued)
            issue(issued);

    // x * gamma over this K slice (fp32), and partial sums of x^2 per token
    const int cpr = a.kslice / 8;
    for (int idx = c; idx < nact * cpr; idx += kHD) {
        const int i = idx / cpr, q = idx % cpr;
        const int kk = k0 + q * 8;
        float xv[8], gv[8];
        bf16x8_to_f32(*reinterpret_cast<const uint4 *>(a.x + (size_t)act[i] * a.H + kk), xv);
        bf16x8_to_f32(*reinterpret_cast<const uint4 *>(a.gamma + kk), gv);
        float sq = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            sq = fmaf(xv[e], xv[e], sq);
            xs[i * a.kslice + q * 8 + e] = xv[e] * gv[e];
        }
        atomicAdd(&pss[i], sq);
    }
    __syncthreads();

    float acc[kNTok];
#pragma unroll
    for (int i = 0; i < kNTok; ++i)
        acc[i] = 0.f;
    bool timeout = false;
    int consumed = 0;
    for (int kt = 0; kt < ntile; ++kt) {
        const int st = kt % kStages;
        if (!mbar_wait(&full[st], (uint32_t)(kt / kStages) & 1u))
            timeout = true;
        if (!timeout) {
            const uint8_t *tw = stages + st * kTile;
#pragma unroll 2
            for (int j = 0; j < 8; ++j) {
                float w[8];
                bf16x8_to_f32(*reinterpret_cast<const uint4 *>(tw + swz128(c, j)), w);
                const float *xk = xs + kt * 64 + j * 8;
#pragma unroll
                for (int i = 0; i < kNTok; ++i) {
                    if (i >= nact)
                        break;
                    const float4 x0 = *reinterpret_cast<const float4 *>(xk + i * a.kslice);
                    const float4 x1 = *reinterpret_cast<const float4 *>(xk + i * a.kslice + 4);
                    acc[i] = fmaf(w[0], x0.x, acc[i]);
                    acc[i] = fmaf(w[1], x0.y, acc[i]);
                    acc[i] = fmaf(w[2], x0.z, acc[i]);
                    acc[i] = fmaf(w[3], x0.w, acc[i]);
                    acc[i] = fmaf(w[4], x1.x, acc[i]);
                    acc[i] = fmaf(w[5], x1.y, acc[i]);
                    acc[i] = fmaf(w[6], x1.z, acc[i]);
                    acc[i] = fmaf(w[7], x1.w, acc[i]);
                }
            }
        }
        consumed = kt + 1;
        if (__syncthreads_or(timeout)) {
            timeout = true;
            break;
        }
        if (c == 0 && issued < ntile)
            issue(issued++);
    }
    if (timeout) {
        if (c == 0) {
            set_status(a.status, WIDE_DEV_TIMEOUT);
            for (int kt = consumed; kt < issued; ++kt)
                mbar_wait(&full[kt % kStages], (uint32_t)(kt / kStages) & 1u);
        }
        __syncthreads();
    }

    float *part = reinterpret_cast<float *>(stages);   // [kNTok][hd]
#pragma unroll
    for (int i = 0; i < kNTok; ++i) {
        if (i >= nact)
            break;
        part[i * kHD + c] = timeout ? 0.f : acc[i];
    }
    cluster.sync();
    const int half = kHD / 2;
    const int pi = c % half;
    // RoPE inverse frequency theta^(-2 pi / hd) for this thread's pair
    const double inv = exp(-(2.0 * pi / kHD) * log(a.theta));
    for (int i = s; i < nact; i += KS) {
        float dot = 0.f, ss = 0.f;
        for (int q = 0; q < KS; ++q) {
            dot += cluster.map_shared_rank(part, q)[i * kHD + c];
            ss += cluster.map_shared_rank(pss, q)[i];
        }
        const float val = dot / sqrtf(ss / (float)a.H + a.eps);
        const int t = act[i];
        const int64_t pos = a.cache_len;     // one new token per sequence
        float outv = val;
        if (kind != 2) {
            rv[c] = val;
            __syncthreads();
            const float partner = rv[c ^ half];
            double sn, cs;
            sincos((double)pos * inv, &sn, &cs);
            outv = c < half ? (float)(val * cs - partner * sn) : (float)(val * cs + partner * sn);
            __syncthreads();
        }
        if (kind == 0) {
            a.q[(size_t)t * a.n_q * kHD + (size_t)head * kHD + c] = outv;
        } else {
            __nv_bfloat16 *cache = kind == 1 ? a.k_cache : a.v_cache;
            const size_t at = (((size_t)t * a.n_kv + head) * (size_t)a.cache_cap + (size_t)pos) * kHD;
            cache[at + c] = __float2bfloat16_rn(outv);
        }
    }
    cluster.sync();
}

// ------------------------------------------------------------ decode_attn
struct AttnArgs {
    const float *q;                // [T][n_q * hd], RoPE applied
    const __nv_bfloat16 *k_cache;  // [n_seq][n_kv][cap][hd]
    const __nv_bfloat16 *v_cache;
    const uint32_t *head_mask;     // [T][Wh]
    float *o;                      // [T][n_q * hd], token pairs interleaved (il2)
    int n_q, n_kv, Wh;
    int64_t nkeys, cache_cap;      // keys per sequence (cache_len + 1)
    float scale_log2;              // log2(e) / sqrt(hd)
};

__global__ void __launch_bounds__(kHD)
    decode_attn(const AttnArgs a)
{
    extern __shared__ float sm[];
    cg::cluster_group cluster = cg::this_cluster();
    const int s = (int)blockIdx.x;          // key slice (cluster rank)
    const int j = (int)blockIdx.y;          // KV head
    const int b = (int)blockIdx.z;          // sequence (= token)
    const int tid = (int)threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int rep = a.n_q / a.n_kv;         // query heads per group (<= 4 here)
    if (((a.head_mask[(size_t)b * a.Wh + (j >> 5)] >> (j & 31)) & 1u) == 0u) {
        // the token skips this head group: no K/V bytes are read; its output
        // is 0 (o_proj reads 4-token blocks without per-token predication)
        if (s < rep)
            a.o[il2(b, (size_t)(j * rep + s) * kHD + tid, (size_t)a.n_q * kHD)] = 0.f;
        return;
    }

    const int64_t C = (a.nkeys + kSplits - 1) / kSplits;
    const int64_t kb = s * C, ke = min(a.nkeys, kb + C);
    const int nk = (int)(ke > kb ? ke - kb : 0);
    float *qs = sm;                        // [rep][hd]
    float *sc = qs + rep * kHD;            // [rep][C]
    float *ml = sc + rep * C;              // [rep][2]: max, sum
    float *os = ml + 2 * rep;              // [rep][hd]

    for (int i = tid; i < rep * kHD; i += kHD)
        qs[i] = a.q[(size_t)b * a.n_q * kHD + (size_t)j * rep * kHD + i] * a.scale_log2;
    __syncthreads();

    const size_t base = ((size_t)b * a.n_kv + j) * (size_t)a.cache_cap * kHD;
    // scores (log2 domain): one key per thread at a time
    for (int kk = tid; kk < nk; kk += kHD) {
        const uint4 *kr = reinterpret_cast<const uint4 *>(a.k_cache + base + (size_t)(kb + kk) * kHD);
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
        for (int ch = 0; ch < kHD / 8; ++ch) {
            float kv[8];
            bf16x8_to_f32(__ldg(kr + ch), kv);
#pragma unroll
            for (int hh = 0; hh < 4; ++hh) {
                if (hh < rep) {
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        d[hh] = fmaf(kv[e], qs[hh * kHD + ch * 8 + e], d[hh]);
                }
            }
        }
        for (int hh = 0; hh < rep; ++hh)
            sc[hh * C + kk] = d[hh];
    }
    __syncthreads();
    // per-head max and sum over this slice: warp w handles head w
    if (warp < rep) {
        float m = -INFINITY;
        for (int kk = lane; kk < nk; kk += 32)
            m = fmaxf(m, sc[warp * C + kk]);
        for (int off = 16; off; off >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        float l = 0.f;
        for (int kk = lane; kk < nk; kk += 32) {
            const float p = nk > 0 ? exp2f(sc[warp * C + kk] - m) : 0.f;
            sc[warp * C + kk] = p;
            l += p;
        }
        for (int off = 16; off; off >>= 1)
            l += __shfl_xor_sync(0xffffffffu, l, off);
        if (lane == 0) {
            ml[2 * warp] = m;
            ml[2 * warp + 1] = l;
        }
    }
    __syncthreads();
    // P.V: thread tid owns output dimension tid
    float o[4] = {0.f, 0.f, 0.f, 0.f};
    for (int kk = 0; kk < nk; ++kk) {
        const float v = __bfloat162float(a.v_cache[base + (size_t)(kb + kk) * kHD + tid]);
#pragma unroll
        for (int hh = 0; hh < 4; ++hh)
            if (hh < rep)
                o[hh] = fmaf(sc[hh * C + kk], v, o[hh]);
    }
    for (int hh = 0; hh < rep; ++hh)
        os[hh * kHD + tid] = o[hh];
    cluster.sync();
    // merge the slices: rank r combines query head r of the group
    if (s < rep) {
        const int hh = s;
        float M = -INFINITY;
        for (int q = 0; q < kSplits; ++q)
            M = fmaxf(M, cluster.map_shared_rank(ml, q)[2 * hh]);
        float L = 0.f, acc = 0.f;
        for (int q = 0; q < kSplits; ++q) {
            const float *rml = cluster.map_shared_rank(ml, q);
            const float w = rml[2 * hh + 1] > 0.f ? exp2f(rml[2 * hh] - M) : 0.f;
            L += w * rml[2 * hh + 1];
            acc += w * cluster.map_shared_rank(os, q)[hh * kHD + tid];
        }
        a.o[il2(b, (size_t)(j * rep + hh) * kHD + tid, (size_t)a.n_q * kHD)] = acc / L;
    }
    cluster.sync();
}

template <typename... KArgs, typename... Args>
int launch_cluster(int32_t kid, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                   int cluster_x, cudaStream_t s, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cluster_x;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (!raise_smem_limit(reinterpret_cast<const void *>(kernel), smem))
        return WIDE_CUDA_FAIL();
    LaunchScope scope(kid, s);
    if (cudaLaunchKernelEx(&cfg, kernel, args...) != cudaSuccess)
        return WIDE_CUDA_FAIL();
    return WIDE_OK;
}

struct DecodeWs {
    float *q, *o, *h1, *hffn;
    __nv_bfloat16 *xn2;
    uint32_t *bar;
    size_t total;
};

DecodeWs decode_ws(const wide_layer_dims *d, void *base)
{
    const size_t T = (size_t)d->n_seq;
    const size_t qd = (size_t)d->n_q_heads * d->head_dim;
    DecodeWs w = {};
    char *p = static_cast<char *>(base);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        char *at = p ? p + off : nullptr;
        off += align_up(bytes > 0 ? bytes : 1, 256);
        return at;
    };
    const size_t Tp = (T + 1) / 2 * 2;                 // interleaved token pairs
    w.q = reinterpret_cast<float *>(take(T * qd * 4));
    w.o = reinterpret_cast<float *>(take(Tp * qd * 4));
    w.h1 = reinterpret_cast<float *>(take(T * (size_t)d->hidden * 4));
    w.hffn = reinterpret_cast<float *>(take(Tp * (size_t)d->inter * 4));
    w.xn2 = reinterpret_cast<__nv_bfloat16 *>(take(T * (size_t)d->hidden * 2));
    w.bar = reinterpret_cast<uint32_t *>(take(256));
    w.total = off;
    return w;
}

}  // namespace

bool layer_decode_supported(const wide_layer_dims *d)
{
    return d->seq_len == 1 && d->n_seq >= 1 && d->n_seq <= kNTok && d->head_dim == kHD &&
           d->n_q_heads % d->n_kv_heads == 0 && d->n_q_heads / d->n_kv_heads <= 4 &&
           d->n_kv_heads <= 1024 && d->hidden % 512 == 0 &&
           d->inter % d->ffn_group_size == 0 &&
           (d->ffn_group_size == 64 || d->ffn_group_size == 128) &&
           ((d->n_q_heads / d->n_kv_heads) * kHD == 128 ||
            (d->n_q_heads / d->n_kv_heads) * kHD == 256 ||
            (d->n_q_heads / d->n_kv_heads) * kHD == 512) &&
           d->cache_cap >= d->cache_len + 1 && d->cache_len >= 0;
}

size_t layer_decode_workspace(const wide_layer_dims *d) { return decode_ws(d, nullptr).total; }

int layer_decode_launch(const LayerPtrs &p, const wide_layer_dims *d, void *ws, cudaStream_t s)
{
    const int T = (int)d->n_seq, H = (int)d->hidden, I = (int)d->inter;
    const int n_q = d->n_q_heads, n_kv = d->n_kv_heads, rep = n_q / n_kv;
    const int qd = n_q * kHD;
    const int Wh = (n_kv + 31) / 32;
    DecodeWs w = decode_ws(d, ws);

    // 1. QKV (+ RMSNorm, RoPE, cache append)
    CUtensorMap tq, tk, tv;
    if (!make_tmap_2d(&tq, p.wq, qd, H, H, 2, kHD, 64, true) ||
        !make_tmap_2d(&tk, p.wk, (uint64_t)n_kv * kHD, H, H, 2, kHD, 64, true) ||
        !make_tmap_2d(&tv, p.wv, (uint64_t)n_kv * kHD, H, H, 2, kHD, 64, true))
        return WIDE_CUDA_FAIL();
    int KS = 8;
    while (KS > 1 && H % (KS * 64) != 0)
        KS >>= 1;
    QkvArgs qa;
    qa.x = static_cast<const __nv_bfloat16 *>(p.x);
    qa.gamma = static_cast<const __nv_bfloat16 *>(p.gamma1);
    qa.head_mask = p.head_mask;
    qa.q = w.q;
    qa.k_cache = static_cast<__nv_bfloat16 *>(p.k_cache);
    qa.v_cache = static_cast<__nv_bfloat16 *>(p.v_cache);
    qa.T = T;
    qa.H = H;
    qa.n_q = n_q;
    qa.n_kv = n_kv;
    qa.Wh = Wh;
    qa.kslice = H / KS;
    qa.cache_len = d->cache_len;
    qa.cache_cap = d->cache_cap;
    qa.eps = d->eps;
    qa.theta = (double)d->rope_theta;
    qa.status = status_ptr();
    const size_t smem_qkv = 1024 + kStages * kHD * 128 + 1024 + (size_t)T * qa.kslice * 4;
    int rc = launch_cluster(KID_DECODE_QKV, decode_qkv, dim3(KS, n_q + 2 * n_kv), dim3(kHD),
                            smem_qkv, KS, s, tq, tk, tv, qa);
    if (rc)
        return rc;

    // 2. attention over the cache, kept head groups only
    AttnArgs aa;
    aa.q = w.q;
    aa.k_cache = static_cast<const __nv_bfloat16 *>(p.k_cache);
    aa.v_cache = static_cast<const __nv_bfloat16 *>(p.v_cache);
    aa.head_mask = p.head_mask;
    aa.o = w.o;
    aa.n_q = n_q;
    aa.n_kv = n_kv;
    aa.Wh = Wh;
    aa.nkeys = d->cache_len + 1;
    aa.cache_cap = d->cache_cap;
    aa.scale_log2 = kLog2e / sqrtf((float)kHD);
    const int64_t C = (aa.nkeys + kSplits - 1) / kSplits;
    const size_t smem_att = ((size_t)rep * kHD * 2 + (size_t)rep * C + 2 * rep) * 4;
    rc = launch_cluster(KID_DECODE_ATTN, decode_attn, dim3(kSplits, n_kv, T), dim3(kHD), smem_att,
                        kSplits, s, aa);
    if (rc)
        return rc;

    // 3. o_proj over kept groups' columns; h1 = x + attn_out (fp32)
    DownOutputs oo = {};
    oo.out_sum = p.attn_out;
    if (p.ffn) {
        oo.res_in = p.x;
        oo.out_total_f32 = w.h1;
    }
    rc = decode_down_bf16(p.wo, w.o, p.head_mask, oo, T, H, qd, rep * kHD, s);
    if (rc || !p.ffn)
        return rc;

    // 4-6. FFN input norm and masked FFN; out = h1 + ffn_out
    const int gsf = (int)d->ffn_group_size;
    DownOutputs fo = {};
    fo.out_sum = p.ffn_out;
    fo.res_f32 = w.h1;
    fo.out_total = p.out;
    if (decode_ffn_fused_preferred(T, H, I, gsf)) {
        // one persistent kernel: the norm is applied while x is staged
        FusedInput in = {};
        in.x_f32 = w.h1;
        in.gamma = p.gamma2;
        in.eps = d->eps;
        in.w_gate = p.w_gate;
        in.w_up = p.w_up;
        in.w_down = p.w_down;
        in.mask = p.ffn_mask;
        return decode_ffn_fused(in, fo, T, H, I, gsf, w.hffn, w.bar, s);
    }
    if ((rc = rmsnorm_f32_launch(w.h1, p.gamma2, w.xn2, T, H, d->eps, s)))
        return rc;
    rc = decode_gateup_bf16(w.xn2, p.w_gate, p.w_up, p.ffn_mask, w.hffn, T, H, I, gsf, s);
    if (rc)
        return rc;
    return decode_down_bf16(p.w_down, w.hffn, p.ffn_mask, fo, T, H, I, gsf, s);
}

}  // namespace wide
