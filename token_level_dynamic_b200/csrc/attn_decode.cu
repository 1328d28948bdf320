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
//   decode_attn   one CTA per (key slice of <= 128 keys, KV head, sequence);
//                 a group the sequence's token skips reads no K/V.  A kept
//                 slice bulk-copies its K and V rows into shared memory,
//                 computes scores, a partial softmax and P.V for the group's
//                 query heads; the last slice of a (sequence, group) to
//                 finish merges all slices with log-sum-exp weights.
// o_proj and the FFN run through the decode down/gate-up GEMVs (groups of
// rep*head_dim o_proj columns), with the residual adds in their epilogues.
#include <cooperative_groups.h>

#include "common.cuh"
#include "host.h"

namespace cg = cooperative_groups;

namespace wide {
namespace {

constexpr int kHD = 128;           // head dimension this path is built for
constexpr int kNTok = 32;
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
// Grid (KS key slices, 2 n_kv + n_q row blocks of hd rows), clusters of KS
// CTAs along the slices.  Row blocks are the K heads, the V heads, then the
// query heads; a query head whose group no token keeps exits at once.
// The CTA's active tokens (those that keep the head's group; every token
// for K and V) are compacted and staged, times gamma, as fp32 token pairs;
// its hd x kslice weight slab streams through a TMA ring of 64-column
// tiles (128-byte swizzle).
//
// Thread (row quad rq = tid / 8, chunk jc = tid % 8) accumulates rows
// 4 rq .. 4 rq + 3 over the 8 columns of chunk jc of every tile, for every
// token pair at once: packed fp32x2 FMAs whose first operand is one weight
// in both halves and whose second is that column's x of the two tokens.
// The 8 lanes of a quad read 128 contiguous bytes of x and of each weight
// row (distinct banks); the 4 quads of a warp read the same x (broadcast).
// Sums over the 8 chunk lanes are formed by shuffles that halve what a lane
// carries at each step; the slices' partial sums (and of x^2 for the norm)
// then meet through distributed shared memory.
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

constexpr int kQkvThreads = 256;
constexpr int kQkvStages = 4;
constexpr uint32_t kQkvTile = kHD * 128u;     // 128 rows x 64 bf16

// Sums v[0..N) over the 8 lanes that differ in lane bits 0..2, halving what a
// lane carries at each step; afterwards lane l holds in v[0..N/8) the sums of
// entries (l & 7) * (N / 8) + i.
template <int N>
__device__ __forceinline__ void sum8_scatter(float (&v)[N], int lane)
{
#pragma unroll
    for (int lv = 0; lv < 3; ++lv) {
        const int o = 4 >> lv;
        const bool hi = (lane & o) != 0;
        const int n = N >> (lv + 1);
#pragma unroll
        for (int i = 0; i < N / 2; ++i) {
            if (i < n) {
                const float send = hi ? v[i] : v[i + n];
                const float keep = hi ? v[i + n] : v[i];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
        }
    }
}

// Accumulates one 64-column tile for NP token pairs: rows w[0..3] (16-byte
// chunks of this thread's 8 columns), x of the tile at xt (pair tp, column
// pair cp at xt + (tp * 4 + cp) * 128).
template <int NP>
__device__ __forceinline__ void qkv_tile(const uint4 (&w)[4], const uint8_t *xt,
                                         float2 (&acc)[4][NP])
{
#pragma unroll
    for (int cp = 0; cp < 4; ++cp) {
        float2 d0[4], d1[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            d0[r] = dup_lo(word(w[r], cp));
            d1[r] = dup_hi(word(w[r], cp));
        }
#pragma unroll
        for (int tp = 0; tp < NP; ++tp) {
            const float4 xv = *reinterpret_cast<const float4 *>(xt + (tp * 4 + cp) * 128);
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                acc[r][tp] = __ffma2_rn(d0[r], make_float2(xv.x, xv.y), acc[r][tp]);
                acc[r][tp] = __ffma2_rn(d1[r], make_float2(xv.z, xv.w), acc[r][tp]);
            }
        }
    }
}

// The main loop for NP token pairs, then the chunk-lane sums written to
// part[token][row] (token < nact).
template <int NP>
__device__ __forceinline__ bool qkv_main(const CUtensorMap *map, uint8_t *stages, uint64_t *full,
                                         const uint8_t *xs, float *part, int ntile, int k0,
                                         int head, int nact, int npt, int tid)
{
    const int rq = tid >> 3, jc = tid & 7, lane = tid & 31;
    float2 acc[4][NP];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int tp = 0; tp < NP; ++tp)
            acc[r][tp] = make_float2(0.f, 0.f);
    bool timeout = false;
    int consumed = 0, issued = min(kQkvStages, ntile);
    for (int kt = 0; kt < ntile; ++kt) {
        const int st = kt % kQkvStages;
        if (!mbar_wait(&full[st], (uint32_t)(kt / kQkvStages) & 1u))
            timeout = true;
        if (!timeout) {
            const uint8_t *tw = stages + st * kQkvTile;
            uint4 w[4];
#pragma unroll
            for (int r = 0; r < 4; ++r)
                w[r] = *reinterpret_cast<const uint4 *>(tw + swz128(4 * rq + r, jc));
            qkv_tile<NP>(w, xs + (size_t)kt * npt * 512 + jc * 16, acc);
        }
        consumed = kt + 1;
        if (__syncthreads_or(timeout)) {
            timeout = true;
            break;
        }
        if (tid == 0 && issued < ntile) {
            const int s2 = issued % kQkvStages;
            mbar_arrive_expect_tx(&full[s2], kQkvTile);
            tma_load_2d(stages + s2 * kQkvTile, map, k0 + issued * 64, head * kHD, &full[s2]);
            ++issued;
        }
    }
    if (timeout) {
        if (tid == 0)
            for (int kt = consumed; kt < issued; ++kt)
                mbar_wait(&full[kt % kQkvStages], (uint32_t)(kt / kQkvStages) & 1u);
        __syncthreads();
        return false;
    }
    // sums over the 8 chunk lanes: entry r * 2NP + t is (row 4 rq + r, token t)
    constexpr int N = 8 * NP;
    float v[N];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int tp = 0; tp < NP; ++tp) {
            v[r * 2 * NP + 2 * tp] = acc[r][tp].x;
            v[r * 2 * NP + 2 * tp + 1] = acc[r][tp].y;
        }
    sum8_scatter<N>(v, lane);
#pragma unroll
    for (int i = 0; i < N / 8; ++i) {
        const int m = jc * (N / 8) + i;
        const int r = m / (2 * NP), t = m % (2 * NP);
        if (t < nact)
            part[t * kHD + 4 * rq + r] = v[i];
    }
    return true;
}

template <int NPMAX>
__global__ void __launch_bounds__(kQkvThreads, NPMAX > 8 ? 1 : 2)
    decode_qkv(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const QkvArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *stages = smem;                                          // [stages][tile]
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kQkvStages * kQkvTile);
    int *act = reinterpret_cast<int *>(full + kQkvStages);           // [32]
    float *pss = reinterpret_cast<float *>(act + kNTok);             // [32] partial sum x^2
    float *rv = pss + kNTok;                                          // [2][hd] RoPE exchange
    uint8_t *xs = reinterpret_cast<uint8_t *>(rv + 2 * kHD);         // x pairs, 16-byte aligned
    float *part = reinterpret_cast<float *>(stages);  // [nact][hd], once the ring is drained

    cg::cluster_group cluster = cg::this_cluster();
    const int KS = (int)gridDim.x;
    const int s = (int)blockIdx.x;
    const int rb = (int)blockIdx.y;
    const int tid = (int)threadIdx.x;
    const int rep = a.n_q / a.n_kv;

    int kind, head;
    const CUtensorMap *map;
    // K and V heads first: they carry every token, so they are the longest
    // CTAs and should not be left for the last wave
    if (rb < a.n_kv) {
        kind = 1; head = rb; map = &tm_k;
    } else if (rb < 2 * a.n_kv) {
        kind = 2; head = rb - a.n_kv; map = &tm_v;
    } else {
        kind = 0; head = rb - 2 * a.n_kv; map = &tm_q;
    }
    const uint32_t all = a.T >= 32 ? 0xffffffffu : ((1u << a.T) - 1u);
    const uint32_t tmask = kind == 0 ? token_group_mask(a.head_mask, a.T, a.Wh, head / rep) : all;
    if (tmask == 0u)
        return;  // no token of the batch keeps this query head's group (whole cluster)
    const int nact = __popc(tmask);
    const int np = (nact + 1) >> 1;                                   // token pairs
    const int npb = np <= 1 ? 1 : np <= 2 ? 2 : np <= 4 ? 4 : np <= 8 ? 8 : 16;
    const int k0 = s * a.kslice;
    const int ntile = a.kslice / 64;

    if (tid < 32 && ((tmask >> tid) & 1u))
        act[__popc(tmask & ((1u << tid) - 1u))] = tid;
    if (tid < kNTok)
        pss[tid] = 0.f;
    if (tid == 0) {
        for (int st = 0; st < kQkvStages; ++st)
            mbar_init(&full[st], 1);
        fence_mbar_init();
        tma_prefetch_desc(map);
        for (int kt = 0; kt < kQkvStages && kt < ntile; ++kt) {
            mbar_arrive_expect_tx(&full[kt], kQkvTile);
            tma_load_2d(stages + kt * kQkvTile, map, k0 + kt * 64, head * kHD, &full[kt]);
        }
    }
    __syncthreads();

    // x * gamma over this K slice as fp32 token pairs: the 16-byte unit at
    // xs + ((tile * npb + pair) * 4 + column pair) * 128 + chunk * 16 holds
    // columns 2cp, 2cp + 1 of the chunk for tokens 2 pair, 2 pair + 1 (a
    // missing odd partner is 0); partial sums of x^2 per token.
    const int cpr = a.kslice / 8;
    for (int idx = tid; idx < npb * cpr; idx += kQkvThreads) {
        const int tp = idx / cpr, q8 = idx % cpr;
        const int kk = k0 + q8 * 8;
        float gv[8], x0[8], x1[8];
        bf16x8_to_f32(*reinterpret_cast<const uint4 *>(a.gamma + kk), gv);
        const int i0 = 2 * tp, i1 = 2 * tp + 1;
        float sq0 = 0.f, sq1 = 0.f;
        if (i0 < nact) {
            bf16x8_to_f32(*reinterpret_cast<const uint4 *>(a.x + (size_t)act[i0] * a.H + kk), x0);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) x0[e] = 0.f;
        }
        if (i1 < nact) {
            bf16x8_to_f32(*reinterpret_cast<const uint4 *>(a.x + (size_t)act[i1] * a.H + kk), x1);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) x1[e] = 0.f;
        }
        const int kt = q8 >> 3, jc = q8 & 7;
        uint8_t *dst = xs + ((size_t)(kt * npb + tp) * 4) * 128 + jc * 16;
#pragma unroll
        for (int cp = 0; cp < 4; ++cp) {
            const int c0 = 2 * cp, c1 = 2 * cp + 1;
            *reinterpret_cast<float4 *>(dst + cp * 128) =
                make_float4(x0[c0] * gv[c0], x1[c0] * gv[c0], x0[c1] * gv[c1], x1[c1] * gv[c1]);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            sq0 = fmaf(x0[e], x0[e], sq0);
            sq1 = fmaf(x1[e], x1[e], sq1);
        }
        if (i0 < nact)
            atomicAdd(&pss[i0], sq0);
        if (i1 < nact)
            atomicAdd(&pss[i1], sq1);
    }
    __syncthreads();

    bool ok;
    if (NPMAX >= 16 && npb == 16)
        ok = qkv_main<(NPMAX >= 16 ? 16 : 1)>(map, stages, full, xs, part, ntile, k0, head, nact, npb, tid);
    else if (npb == 8)
        ok = qkv_main<8>(map, stages, full, xs, part, ntile, k0, head, nact, npb, tid);
    else if (npb == 4)
        ok = qkv_main<4>(map, stages, full, xs, part, ntile, k0, head, nact, npb, tid);
    else if (npb == 2)
        ok = qkv_main<2>(map, stages, full, xs, part, ntile, k0, head, nact, npb, tid);
    else
        ok = qkv_main<1>(map, stages, full, xs, part, ntile, k0, head, nact, npb, tid);
    if (!ok) {
        if (tid == 0)
            set_status(a.status, WIDE_DEV_TIMEOUT);
        for (int i = tid; i < nact * kHD; i += kQkvThreads)
            part[i] = 0.f;
    }
    cluster.sync();

    // tokens s, s + KS, ... of the active list: the two halves of the block
    // take alternate ones; thread c of a half owns row c of the head
    const int half = tid / kHD, c = tid % kHD;
    const int hh = kHD / 2, pi = c % hh;
    const int64_t pos = a.cache_len;          // one new token per sequence
    double sn = 0.0, cs = 1.0;
    if (kind != 2) {
        // RoPE angle pos * theta^(-2 pi / hd) of this thread's pair
        const double inv = exp(-(2.0 * pi / kHD) * log(a.theta));
        sincos((double)pos * inv, &sn, &cs);
    }
    const int per = (nact - s + KS - 1) / KS;     // tokens of this CTA (may be <= 0)
    for (int k = 0; k < (per + 1) / 2; ++k) {
        const int i = s + KS * (2 * k + half);
        const bool have = i < nact;
        float val = 0.f;
        if (have) {
            float dot = 0.f, ss = 0.f;
            for (int q = 0; q < KS; ++q) {
                dot += cluster.map_shared_rank(part, q)[i * kHD + c];
                ss += cluster.map_shared_rank(pss, q)[i];
            }
            val = dot / sqrtf(ss / (float)a.H + a.eps);
        }
        float outv = val;
        if (kind != 2) {
            rv[half * kHD + c] = val;
            __syncthreads();
            const float partner = rv[half * kHD + (c ^ hh)];
            outv = c < hh ? (float)(val * cs - partner * sn) : (float)(val * cs + partner * sn);
            __syncthreads();
        }
        if (have) {
            const int t = act[i];
            if (kind == 0) {
                a.q[(size_t)t * a.n_q * kHD + (size_t)head * kHD + c] = outv;
            } else {
                __nv_bfloat16 *cache = kind == 1 ? a.k_cache : a.v_cache;
                const size_t at =
                    (((size_t)t * a.n_kv + head) * (size_t)a.cache_cap + (size_t)pos) * kHD;
                cache[at + c] = __float2bfloat16_rn(outv);
            }
        }
    }
    cluster.sync();
}

// ------------------------------------------------------------ decode_attn
// One CTA per (key slice s of <= 128 keys, KV head j, sequence b).  A sequence whose token
// skips group j reads no K/V bytes: slice 0 of the pair writes the group's
// zero output and every slice exits.  A kept pair's CTA bulk-copies its
// slice of the K and V slabs (contiguous rows of the [cap][hd] cache) into
// shared memory, computes the scores of its keys for the group's query
// heads (8 lanes per key, 4 keys per warp at a time), a partial softmax
// (slice max m, sum l) and the unnormalised P.V, and stores them to the
// workspace.  The last slice of a pair to finish (an arrival counter,
// zeroed on the stream before QKV) merges the slices with log-sum-exp
// weights:  o = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s.
struct AttnArgs {
    const float *q;                // [T][n_q * hd], RoPE applied
    const __nv_bfloat16 *k_cache;  // [n_seq][n_kv][cap][hd]
    const __nv_bfloat16 *v_cache;
    const uint32_t *head_mask;     // [T][Wh]
    float *o;                      // [T][n_q * hd], token pairs interleaved (il2)
    float *part_o;                 // [T][n_kv][S][rep][hd] unnormalised slice outputs
    float2 *part_ml;               // [T][n_kv][S][rep] slice (max, sum), log2 domain
    uint32_t *arrived;             // [T][n_kv] slices done (0 at launch)
    int n_q, n_kv, Wh, S, C;       // key slices and keys per slice (<= kAttnMaxC)
    int64_t nkeys, cache_cap;      // keys per sequence (cache_len + 1)
    float scale_log2;              // log2(e) / sqrt(hd)
    int32_t *status;
};

constexpr int kAttnMaxC = 128;

template <int REP>
__global__ void __launch_bounds__(kHD)
    decode_attn(const AttnArgs a)
{
    extern __shared__ __align__(128) uint8_t sm_attn[];
    const int s = (int)blockIdx.x;          // key slice
    const int j = (int)blockIdx.y;          // KV head
    const int b = (int)blockIdx.z;          // sequence (= token)
    const int tid = (int)threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const size_t qd = (size_t)a.n_q * kHD;
    if (((a.head_mask[(size_t)b * a.Wh + (j >> 5)] >> (j & 31)) & 1u) == 0u) {
        // the token skips this head group: its output is 0 (the o_proj GEMV
        // reads token pairs without per-token predication)
        if (s == 0)
            for (int hh = 0; hh < REP; ++hh)
                a.o[il2(b, (size_t)(j * REP + hh) * kHD + tid, qd)] = 0.f;
        return;
    }
    const int64_t kb = (int64_t)s * a.C;
    const int nk = (int)max((int64_t)0, min(a.nkeys, kb + a.C) - kb);
    uint8_t *ks = sm_attn;                                        // [C][hd] bf16
    uint8_t *vs = ks + (size_t)a.C * kHD * 2;                     // [C][hd] bf16
    // K and V, later the merge's per-slice weights: the larger of the two
    const size_t area = max((size_t)a.C * kHD * 4, ((size_t)a.S * REP * 8 + 15) & ~(size_t)15);
    float *pv = reinterpret_cast<float *>(ks + area);             // [C][4] scores, then P
    float *sml = pv + 4 * a.C;                                    // [REP][2]
    uint64_t *bar = reinterpret_cast<uint64_t *>(sml + 8);
    __shared__ int s_last;

    const size_t slab = ((size_t)b * a.n_kv + j) * (size_t)a.cache_cap * kHD;
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
        if (nk > 0) {
            const uint32_t bytes = (uint32_t)nk * kHD * 2u;
            mbar_arrive_expect_tx(bar, 2u * bytes);
            bulk_load(ks, a.k_cache + slab + (size_t)kb * kHD, bytes, bar);
            bulk_load(vs, a.v_cache + slab + (size_t)kb * kHD, bytes, bar);
        }
    }
    // this lane's query dims: chunk dc (dims 8 dc ..) and chunk dc + 8 of each head
    const int kq = lane >> 3, dc = lane & 7;
    float qa[REP][8], qb[REP][8];
    const float *qrow = a.q + (size_t)b * qd + (size_t)j * REP * kHD;
#pragma unroll
    for (int hh = 0; hh < REP; ++hh)
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            qa[hh][e] = qrow[hh * kHD + dc * 8 + e] * a.scale_log2;
            qb[hh][e] = qrow[hh * kHD + 64 + dc * 8 + e] * a.scale_log2;
        }
    __syncthreads();                        // barrier initialised
    bool ok = true;
    if (nk > 0)
        ok = mbar_wait(bar, 0u);
    if (!ok && tid == 0) {
        // the copies have not landed: report, give them one more bounded
        // wait before this CTA exits, and leave this slice empty
        set_status(a.status, WIDE_DEV_TIMEOUT);
        mbar_wait(bar, 0u);
    }
    const int nkv = ok ? nk : 0;

    // scores (log2 domain) of keys warp*4 + kq, + 16, ...
    for (int k0 = warp * 4; k0 < nkv; k0 += 16) {
        const int kk = k0 + kq;
        const bool valid = kk < nkv;
        float d[REP];
#pragma unroll
        for (int hh = 0; hh < REP; ++hh)
            d[hh] = 0.f;
        if (valid) {
            float ka[8], kb8[8];
            bf16x8_to_f32(*reinterpret_cast<const uint4 *>(ks + (size_t)kk * 256 + dc * 16), ka);
            bf16x8_to_f32(*reinterpret_cast<const uint4 *>(ks + (size_t)kk * 256 + 128 + dc * 16), kb8);
#pragma unroll
            for (int hh = 0; hh < REP; ++hh)
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    d[hh] = fmaf(qa[hh][e], ka[e], d[hh]);
                    d[hh] = fmaf(qb[hh][e], kb8[e], d[hh]);
                }
        }
#pragma unroll
        for (int hh = 0; hh < REP; ++hh) {
            d[hh] += __shfl_xor_sync(0xffffffffu, d[hh], 1);
            d[hh] += __shfl_xor_sync(0xffffffffu, d[hh], 2);
            d[hh] += __shfl_xor_sync(0xffffffffu, d[hh], 4);
        }
        if (valid && dc == 0)
#pragma unroll
            for (int hh = 0; hh < REP; ++hh)
                pv[kk * 4 + hh] = d[hh];
    }
    __syncthreads();
    // slice max and sum per head: warp hh takes head hh
    if (warp < REP) {
        float m = -INFINITY;
        for (int kk = lane; kk < nkv; kk += 32)
            m = fmaxf(m, pv[kk * 4 + warp]);
        for (int off = 16; off; off >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        float l = 0.f;
        for (int kk = lane; kk < nkv; kk += 32) {
            const float p = exp2f(pv[kk * 4 + warp] - m);
            pv[kk * 4 + warp] = p;
            l += p;
        }
        for (int off = 16; off; off >>= 1)
            l += __shfl_xor_sync(0xffffffffu, l, off);
        if (lane == 0) {
            sml[2 * warp] = m;
            sml[2 * warp + 1] = l;
        }
    }
    __syncthreads();
    // P.V: thread tid owns output dim tid
    float o[REP];
#pragma unroll
    for (int hh = 0; hh < REP; ++hh)
        o[hh] = 0.f;
    const __nv_bfloat16 *vcol = reinterpret_cast<const __nv_bfloat16 *>(vs) + tid;
#pragma unroll 4
    for (int kk = 0; kk < nkv; ++kk) {
        const float v = __bfloat162float(vcol[(size_t)kk * kHD]);
        const float4 p = *reinterpret_cast<const float4 *>(pv + kk * 4);
        o[0] = fmaf(p.x, v, o[0]);
        if (REP > 1) o[1] = fmaf(p.y, v, o[1]);
        if (REP > 2) o[2] = fmaf(p.z, v, o[2]);
        if (REP > 3) o[3] = fmaf(p.w, v, o[3]);
    }
    const size_t pair = (size_t)b * a.n_kv + j;
    const size_t slot = (pair * a.S + s) * REP;
#pragma unroll
    for (int hh = 0; hh < REP; ++hh)
        a.part_o[(slot + hh) * kHD + tid] = o[hh];
    if (tid < REP)
        a.part_ml[slot + tid] = make_float2(sml[2 * tid], sml[2 * tid + 1]);

    // the last slice of this (sequence, group) to finish merges them all
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        s_last = atomicAdd(&a.arrived[pair], 1u) == (uint32_t)(a.S - 1);
    }
    __syncthreads();
    if (!s_last)
        return;
    __threadfence();
    // every slice's (max, sum) into shared memory (the K/V tiles' space), then
    // each slice's weight 2^(m_s - M) per head
    float2 *wml = reinterpret_cast<float2 *>(ks);                 // [S][REP]
    const float2 *ml = a.part_ml + pair * a.S * REP;
    for (int i = tid; i < a.S * REP; i += kHD)
        wml[i] = __ldcg(&ml[i]);
    __syncthreads();
    if (tid < REP) {
        float M = -INFINITY;
        for (int q = 0; q < a.S; ++q)
            M = fmaxf(M, wml[q * REP + tid].x);
        float L = 0.f;
        for (int q = 0; q < a.S; ++q) {
            const float2 v = wml[q * REP + tid];
            const float w = v.y > 0.f ? exp2f(v.x - M) : 0.f;
            wml[q * REP + tid].x = w;
            L += w * v.y;
        }
        sml[2 * tid + 1] = L;
    }
    __syncthreads();
    const float *po = a.part_o + pair * a.S * REP * kHD + tid;
    float acc[REP];
#pragma unroll
    for (int hh = 0; hh < REP; ++hh)
        acc[hh] = 0.f;
#pragma unroll 4
    for (int q = 0; q < a.S; ++q)
#pragma unroll
        for (int hh = 0; hh < REP; ++hh)
            acc[hh] = fmaf(wml[q * REP + hh].x, __ldcg(po + ((size_t)q * REP + hh) * kHD), acc[hh]);
#pragma unroll
    for (int hh = 0; hh < REP; ++hh) {
        const float L = sml[2 * hh + 1];
        a.o[il2(b, (size_t)(j * REP + hh) * kHD + tid, qd)] = L > 0.f ? acc[hh] / L : 0.f;
    }
    if (tid == 0)
        a.arrived[pair] = 0u;               // ready for the next call
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
    float *q, *o, *h1, *hffn, *part_o;
    size_t hffn_bytes;
    float2 *part_ml;
    __nv_bfloat16 *xn2;
    uint32_t *bar, *arrived;
    int S, C;                       // attention key slices, keys per slice
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
    // FFN h, or a persistent kernel's accumulator (the o_proj's too)
    const size_t hffn_bytes = Tp * (size_t)d->inter * 4;
    const size_t acc_bytes = decode_ffn_tc_scratch((int)T, (int)d->hidden);
    w.hffn_bytes = hffn_bytes > acc_bytes ? hffn_bytes : acc_bytes;
    w.hffn = reinterpret_cast<float *>(take(w.hffn_bytes));
    w.xn2 = reinterpret_cast<__nv_bfloat16 *>(take(T * (size_t)d->hidden * 2));
    w.bar = reinterpret_cast<uint32_t *>(take(256));
    const int64_t nkeys = d->cache_len + 1;
    w.S = (int)((nkeys + kAttnMaxC - 1) / kAttnMaxC);
    w.C = (int)((nkeys + w.S - 1) / w.S);
    const size_t rep = (size_t)(d->n_q_heads / d->n_kv_heads);
    const size_t slots = T * (size_t)d->n_kv_heads * (size_t)w.S * rep;
    w.part_o = reinterpret_cast<float *>(take(slots * d->head_dim * 4));
    w.part_ml = reinterpret_cast<float2 *>(take(slots * 8));
    w.arrived = reinterpret_cast<uint32_t *>(take(T * (size_t)d->n_kv_heads * 4));
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
           d->cache_cap >= d->cache_len + 1 && d->cache_len >= 0 &&
           d->cache_len < 131072;   // bounds the attention merge's shared memory (64 KB)
}

size_t layer_decode_workspace(const wide_layer_dims *d) { return decode_ws(d, nullptr).total; }

int layer_decode_launch(const LayerPtrs &p, const wide_layer_dims *d, void *ws, cudaStream_t s)
{
    const int T = (int)d->n_seq, H = (int)d->hidden, I = (int)d->inter;
    const int n_q = d->n_q_heads, n_kv = d->n_kv_heads, rep = n_q / n_kv;
    const int qd = n_q * kHD;
    const int Wh = (n_kv + 31) / 32;
    DecodeWs w = decode_ws(d, ws);

    // attention slice counters start at zero (the merging slice also resets
    // its counter, but the workspace may come from anywhere)
    if (cudaMemsetAsync(w.arrived, 0, (size_t)T * n_kv * sizeof(uint32_t), s) != cudaSuccess)
        return WIDE_CUDA_FAIL();

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
    // x pairs of the largest token count a row block can have (T)
    const int np = (T + 1) / 2;
    const int npb = np <= 1 ? 1 : np <= 2 ? 2 : np <= 4 ? 4 : np <= 8 ? 8 : 16;
    const size_t smem_qkv = 1024 + kQkvStages * (size_t)kQkvTile + 32 + 2 * kNTok * 4 +
                            2 * kHD * 4 + (size_t)qa.kslice * npb * 8;
    int rc = npb > 8 ? launch_cluster(KID_DECODE_QKV, decode_qkv<16>, dim3(KS, n_q + 2 * n_kv),
                                      dim3(kQkvThreads), smem_qkv, KS, s, tq, tk, tv, qa)
                     : launch_cluster(KID_DECODE_QKV, decode_qkv<8>, dim3(KS, n_q + 2 * n_kv),
                                      dim3(kQkvThreads), smem_qkv, KS, s, tq, tk, tv, qa);
    if (rc)
        return rc;

    // 2. attention over the cache, kept head groups only
    AttnArgs aa;
    aa.q = w.q;
    aa.k_cache = static_cast<const __nv_bfloat16 *>(p.k_cache);
    aa.v_cache = static_cast<const __nv_bfloat16 *>(p.v_cache);
    aa.head_mask = p.head_mask;
    aa.o = w.o;
    aa.part_o = w.part_o;
    aa.part_ml = w.part_ml;
    aa.arrived = w.arrived;
    aa.n_q = n_q;
    aa.n_kv = n_kv;
    aa.Wh = Wh;
    aa.S = w.S;
    aa.C = w.C;
    aa.nkeys = d->cache_len + 1;
    aa.cache_cap = d->cache_cap;
    aa.scale_log2 = kLog2e / sqrtf((float)kHD);
    aa.status = status_ptr();
    const size_t kv_area = (size_t)w.C * kHD * 4, merge_area = ((size_t)w.S * rep * 8 + 15) & ~15;
    const size_t smem_att = (kv_area > merge_area ? kv_area : merge_area) + (size_t)w.C * 16 + 32 + 8;
    void (*attn)(AttnArgs) = rep == 4 ? decode_attn<4> : rep == 2 ? decode_attn<2> : decode_attn<1>;
    if (!raise_smem_limit(reinterpret_cast<const void *>(attn), smem_att))
        return WIDE_CUDA_FAIL();
    {
        LaunchScope scope(KID_DECODE_ATTN, s);
        attn<<<dim3(w.S, n_kv, T), kHD, smem_att, s>>>(aa);
        if (cudaGetLastError() != cudaSuccess)
            return WIDE_CUDA_FAIL();
    }

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
    const size_t hcap = w.hffn_bytes;
    // the dispatcher reads the packed copy where the tensor-core kernel runs
    const void *pk = p.ffn_packed;
    if (decode_ffn_persistent_available(T, H, I, gsf, hcap, pk)) {
        if ((rc = rmsnorm_f32_launch(w.h1, p.gamma2, w.xn2, T, H, d->eps, s)))
            return rc;
        return decode_ffn_persistent(w.xn2, p.w_gate, p.w_up, p.w_down, p.ffn_mask, fo, T, H, I,
                                     gsf, w.hffn, hcap, s, pk);
    }
    if ((rc = rmsnorm_f32_launch(w.h1, p.gamma2, w.xn2, T, H, d->eps, s)))
        return rc;
    rc = decode_gateup_bf16(w.xn2, p.w_gate, p.w_up, p.ffn_mask, w.hffn, T, H, I, gsf, s);
    if (rc)
        return rc;
    return decode_down_bf16(p.w_down, w.hffn, p.ffn_mask, fo, T, H, I, gsf, s);
}

}  // namespace wide
