// ffn_decode.cu -- masked SwiGLU FFN for small token counts (decode).
//
// WIDE, technical summary section 2.A (contiguous FFN channel groups chosen
// per token) and section 2.C (block-level early exit, intra-block skipping)
// applied to the bandwidth-bound decode case: the weights of a channel group
// are streamed from HBM once per call, and only when at least one token of
// the batch executes the group (the batch's union); inside a streamed tile,
// only the tokens that execute the group do arithmetic.
//
// gate/up kernel: grid (KS, G), cluster (KS, 1, 1), GS threads.
//   The cluster owns channel group g; CTA s owns the K-slice
//   [s*H/KS, (s+1)*H/KS).  If no token executes g the cluster exits at once
//   (block-level skip).  Gate and up tiles (GS rows x 128 bytes, 128-byte
//   swizzle) arrive by TMA through a 3-stage mbarrier ring; thread c owns
//   channel c of the group and accumulates, in fp32, the gate and up dot
//   products of every executing token against x held in shared memory as
//   fp32.  The KS partial sums are added through distributed shared memory,
//   and h = silu(gate) * up is written (fp32) for executing tokens only.
// down kernel: grid (KS, H/128), cluster (KS, 1, 1), 128 threads.
//   CTA (s, nb) owns output rows [nb*128, nb*128+128) and the groups of
//   slice s.  It streams W_down tiles (128 rows x 128 bytes) only for groups
//   some token executes, with the matching h tile, and thread n adds
//   h[t][c] * W_down[n][c] only for tokens t that execute the group.  The KS
//   partial outputs are added through distributed shared memory.
//
// Tokens are processed 32 at a time (one mask bit per lane), two at a time
// per packed fp32x2 FMA: x (staged in shared memory) and h (the fp32 [T][I]
// intermediate, and the attention output that o_proj reads) are stored with
// token pairs interleaved (il2), so one register pair holds the same column
// of two tokens and the weight element is duplicated across the pair.
#include <cooperative_groups.h>

#include "common.cuh"
#include "host.h"

namespace cg = cooperative_groups;

namespace wide {
namespace {

constexpr int kNTok = 32;
constexpr int kStages = 3;
constexpr int kDownRows = 128;

template <typename TIn> struct ElemTraits;
template <> struct ElemTraits<__nv_bfloat16> {
    static constexpr int EPC = 8;  // elements per 16-byte chunk
};
template <> struct ElemTraits<float> {
    static constexpr int EPC = 4;
};

template <typename TIn>
__device__ __forceinline__ void chunk_to_f32(const uint4 v, float (&f)[ElemTraits<TIn>::EPC]);
template <>
__device__ __forceinline__ void chunk_to_f32<__nv_bfloat16>(const uint4 v, float (&f)[8])
{
    bf16x8_to_f32(v, f);
}
template <> __device__ __forceinline__ void chunk_to_f32<float>(const uint4 v, float (&f)[4])
{
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
}

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    const uint32_t a = smem_u32(p);
    return p + (((a + 1023u) & ~1023u) - a);
}

// Token mask of group g over tokens [0, T), T <= 32 (one lane per token).
__device__ __forceinline__ uint32_t group_token_mask(const uint32_t *mask, int T, int W, int g)
{
    const int lane = threadIdx.x & 31;
    const uint32_t a = lane < T ? (mask[(size_t)lane * W + (g >> 5)] >> (g & 31)) & 1u : 0u;
    return __ballot_sync(0xffffffffu, a);
}

// One weight chunk (EPC elements of two rows wa, wb) times the x chunks of
// NP token pairs (xk2: pair 0 of the chunk in the interleaved layout, pair
// stride ld2 floats): 2*NP independent packed accumulation chains.
template <int EPC, int NP>
__device__ __forceinline__ void fma2_pairs(const float (&wa)[EPC], const float (&wb)[EPC],
                                           const float *xk2, int ld2, float2 *a, float2 *b)
{
#pragma unroll
    for (int e = 0; e < EPC; e += 2) {
        float4 xv[NP];
#pragma unroll
        for (int p = 0; p < NP; ++p)
            xv[p] = *reinterpret_cast<const float4 *>(xk2 + p * ld2 + e * 2);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const float2 wa2 = make_float2(wa[e + q], wa[e + q]);
            const float2 wb2 = make_float2(wb[e + q], wb[e + q]);
#pragma unroll
            for (int p = 0; p < NP; ++p) {
                const float2 xp = q == 0 ? make_float2(xv[p].x, xv[p].y)
                                         : make_float2(xv[p].z, xv[p].w);
                a[p] = __ffma2_rn(wa2, xp, a[p]);
                b[p] = __ffma2_rn(wb2, xp, b[p]);
            }
        }
    }
}

// One weight row chunk times the h chunks of NP token pairs.
template <int EPC, int NP>
__device__ __forceinline__ void fma1_pairs(const float (&w)[EPC], const float *hk2, int ld2,
                                           float2 *acc)
{
#pragma unroll
    for (int e = 0; e < EPC; e += 2) {
        float4 hv[NP];
#pragma unroll
        for (int p = 0; p < NP; ++p)
            hv[p] = *reinterpret_cast<const float4 *>(hk2 + p * ld2 + e * 2);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const float2 w2 = make_float2(w[e + q], w[e + q]);
#pragma unroll
            for (int p = 0; p < NP; ++p)
                acc[p] = __ffma2_rn(w2, q == 0 ? make_float2(hv[p].x, hv[p].y)
                                               : make_float2(hv[p].z, hv[p].w),
                                    acc[p]);
        }
    }
}

// Warp 0 of a decode CTA streams weight (and h) tiles through the stage
// ring; the consumer warps release a stage by one arrive per warp on its
// empty barrier, so the producer runs ahead without a block-wide barrier.
struct Ring {
    uint64_t *full, *empty;
};

// gate/up: block = 32 + 2*GS threads.  Warp 0 = TMA producer.  Consumer
// thread (half, c) owns channel c of group g (its gate and up rows) and the
// 16-byte chunks half*4 .. half*4+3 of every 128-byte K tile row.  Tokens
// are taken TB at a time from the group's executing tokens (x rows past
// them are zero), so consecutive FMAs are independent.
template <typename TIn, int GS, int TB>
__global__ void __launch_bounds__(32 + 2 * GS)
    ffn_decode_gateup(const __grid_constant__ CUtensorMap tm_gate,
                      const __grid_constant__ CUtensorMap tm_up, const TIn *__restrict__ x,
                      const uint32_t *__restrict__ mask, float *__restrict__ h, int T, int H,
                      int I, int W, int kslice, int32_t *status)
{
    constexpr int EPC = ElemTraits<TIn>::EPC;
    constexpr int KT = 8 * EPC;                 // elements in one 128-byte tile row
    constexpr uint32_t kTileBytes = GS * 128u;  // one operand tile
    constexpr int kConsumerWarps = 2 * GS / 32;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    uint8_t *stages = smem;                                          // [kStages][2][GS][128]
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kStages * 2 * kTileBytes);
    uint64_t *empty = full + kStages;
    int *act = reinterpret_cast<int *>(empty + kStages);             // [32]
    float *xs = reinterpret_cast<float *>(smem + kStages * 2 * kTileBytes + 512);  // [nactTB][kslice]

    cg::cluster_group cluster = cg::this_cluster();
    const int KS = (int)gridDim.x;
    const int s = (int)blockIdx.x;
    const int g = (int)blockIdx.y;
    const int tid = (int)threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int ct = tid - 32;                    // consumer index (valid when warp > 0)
    const int c = ct % GS, half = ct / GS;

    // mask bits at or above G are ignored by both kernels; one CTA reports them
    if (g == 0 && s == 0 && (I / GS) % 32 != 0) {
        const int G = I / GS;
        for (int t = tid; t < T; t += 32 + 2 * GS)
            if ((mask[(size_t)t * W + W - 1] >> (G & 31)) != 0u)
                set_status(status, WIDE_DEV_BAD_MASK);
    }
    const uint32_t tmask = group_token_mask(mask, T, W, g);
    if (tmask == 0u)
        return;  // block-level skip: the whole cluster leaves together
    const int nact = __popc(tmask);
    const int nactb = (nact + TB - 1) / TB * TB;
    const int k0 = s * kslice;
    const int ntile = kslice / KT;

    if (tid < 32 && ((tmask >> tid) & 1u))
        act[__popc(tmask & ((1u << tid) - 1u))] = tid;
    if (tid == 0) {
        for (int st = 0; st < kStages; ++st) {
            mbar_init(&full[st], 1);
            mbar_init(&empty[st], kConsumerWarps);
        }
        fence_mbar_init();
        tma_prefetch_desc(&tm_gate);
        tma_prefetch_desc(&tm_up);
    }
    __syncthreads();

    auto issue = [&](int kt) {
        const int st = kt % kStages;
        uint8_t *dst = stages + st * 2 * kTileBytes;
        mbar_arrive_expect_tx(&full[st], 2 * kTileBytes);
        tma_load_2d(dst, &tm_gate, k0 + kt * KT, g * GS, &full[st]);
        tma_load_2d(dst + kTileBytes, &tm_up, k0 + kt * KT, g * GS, &full[st]);
    };
    // the first ring's worth of tiles goes out before x is staged (no slot
    // is in use yet, so nothing to wait for)
    if (tid == 0)
        for (int kt = 0; kt < kStages && kt < ntile; ++kt)
            issue(kt);

    // x of the executing tokens over this K-slice, widened to fp32
    const int chunks_per_row = kslice / EPC;
    for (int idx = tid; idx < nactb * chunks_per_row; idx += 32 + 2 * GS) {
        const int i = idx / chunks_per_row, q = idx % chunks_per_row;
        float f[EPC];
        if (i < nact) {
            const uint4 v =
                *reinterpret_cast<const uint4 *>(x + (size_t)act[i] * H + k0 + q * EPC);
            chunk_to_f32<TIn>(v, f);
        } else {
#pragma unroll
            for (int e = 0; e < EPC; ++e)
                f[e] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < EPC; ++e)
            xs[il2(i, (size_t)q * EPC + e, kslice)] = f[e];
    }
    __syncthreads();

    bool timeout = false;
    if (warp == 0) {
        // ---------------------------------------------- TMA producer
        if (lane == 0) {
            for (int kt = kStages; kt < ntile; ++kt) {
                const int st = kt % kStages;
                if (!mbar_wait(&empty[st], (uint32_t)(kt / kStages - 1) & 1u)) {
                    timeout = true;
                    break;
                }
                issue(kt);
            }
        }
    }

    float2 accg[kNTok / 2], accu[kNTok / 2];     // token pairs
#pragma unroll
    for (int i = 0; i < kNTok / 2; ++i) {
        accg[i] = make_float2(0.f, 0.f);
        accu[i] = make_float2(0.f, 0.f);
    }
    if (warp > 0) {
        // ---------------------------------------------- consumers
        for (int kt = 0; kt < ntile; ++kt) {
            const int st = kt % kStages;
            if (!mbar_wait(&full[st], (uint32_t)(kt / kStages) & 1u)) {
                timeout = true;
                break;
            }
            const uint8_t *tg = stages + st * 2 * kTileBytes;
            const uint8_t *tu = tg + kTileBytes;
#pragma unroll 1
            for (int jj = 0; jj < 4; ++jj) {
                const int j = half * 4 + jj;
                float wg[EPC], wu[EPC];
                chunk_to_f32<TIn>(*reinterpret_cast<const uint4 *>(tg + swz128(c, j)), wg);
                chunk_to_f32<TIn>(*reinterpret_cast<const uint4 *>(tu + swz128(c, j)), wu);
                const float *xk2 = xs + (size_t)(kt * KT + j * EPC) * 2;
#pragma unroll
                for (int i0 = 0; i0 < kNTok; i0 += TB) {
                    if (i0 >= nactb)
                        break;
                    fma2_pairs<EPC, TB / 2>(wg, wu, xk2 + (size_t)i0 * kslice, 2 * kslice,
                                            &accg[i0 / 2], &accu[i0 / 2]);
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&empty[st]);
        }
    }
    if (__syncthreads_or(timeout)) {
        timeout = true;
        if (tid == 0) {
            set_status(status, WIDE_DEV_TIMEOUT);
            // let copies in flight land before the stage memory is reused
            for (int st = 0; st < kStages && st < ntile; ++st) {
                const int last = st + (ntile - 1 - st) / kStages * kStages;
                mbar_wait(&full[st], (uint32_t)(last / kStages) & 1u);
            }
        }
        __syncthreads();
    }

    // partial sums -> this CTA's shared memory, then a cluster-wide add
    float *pg = reinterpret_cast<float *>(stages);  // [2][kNTok][GS]
    float *pu = pg + 2 * kNTok * GS;
    if (warp > 0) {
#pragma unroll
        for (int i = 0; i < kNTok; ++i) {
            if (i >= nact)
                break;
            const float2 g2 = accg[i >> 1], u2 = accu[i >> 1];
            pg[(half * kNTok + i) * GS + c] = timeout ? 0.f : ((i & 1) ? g2.y : g2.x);
            pu[(half * kNTok + i) * GS + c] = timeout ? 0.f : ((i & 1) ? u2.y : u2.x);
        }
    }
    cluster.sync();
    if (warp > 0 && half == 0) {
        for (int i = s; i < nact; i += KS) {
            float gs = 0.f, us = 0.f;
            for (int q = 0; q < KS; ++q) {
                const float *rg = cluster.map_shared_rank(pg, q);
                const float *ru = cluster.map_shared_rank(pu, q);
                gs += rg[i * GS + c] + rg[(kNTok + i) * GS + c];
                us += ru[i * GS + c] + ru[(kNTok + i) * GS + c];
            }
            h[il2(act[i], (size_t)g * GS + c, I)] = silu_f32(gs) * us;
        }
    } else if (warp > 0) {
        // tokens that skip this group get h = 0, so that the down projection
        // can run token blocks without per-token predication
        for (int t = s; t < T; t += KS)
            if (((tmask >> t) & 1u) == 0u)
                h[il2(t, (size_t)g * GS + c, I)] = 0.f;
    }
    cluster.sync();
}

// down: block = 32 + 256 threads.  Warp 0 = TMA producer (W_down tile and
// the matching h tile per stage).  Consumer thread (half, n) owns output row
// nb*128 + n and the chunks half*4 .. half*4+3 of every streamed row.  The K
// loop visits only groups some token keeps; inside a group, blocks of TB
// tokens none of which keeps the group are skipped (h is 0 for skipped
// pairs, written by the gate/up kernel or the attention kernel).
template <typename TIn, int GS, int TB>
__global__ void __launch_bounds__(32 + 2 * kDownRows)
    ffn_decode_down(const __grid_constant__ CUtensorMap tm_down,
                    const __grid_constant__ CUtensorMap tm_h, const uint32_t *__restrict__ mask,
                    const DownOutputs o, int T, int H, int I, int W, int G, int32_t *status)
{
    constexpr int EPC = ElemTraits<TIn>::EPC;
    constexpr int KT = 8 * EPC;
    constexpr int TPG = GS / KT;                          // tiles per group
    constexpr uint32_t kWBytes = kDownRows * 128u;        // W_down tile
    constexpr int kConsumerWarps = 2 * kDownRows / 32;
    constexpr uint32_t kBlockMask = TB >= 32 ? 0xffffffffu : ((1u << TB) - 1u);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    const int TT = (T + TB - 1) / TB * TB;                // TB is even
    const int TP = (T + 1) / 2;                           // token pairs TMA writes
    const uint32_t hbytes = (uint32_t)TP * 2u * KT * 4u;  // h tile: [TP][KT][2] fp32
    const uint32_t hstride = (uint32_t)TT * KT * 4u;
    const uint32_t stage_bytes = kWBytes + ((hstride + 1023u) & ~1023u);
    uint8_t *stages = smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kStages * stage_bytes);
    uint64_t *empty = full + kStages;
    uint32_t *gmask = reinterpret_cast<uint32_t *>(empty + kStages);  // [gq]
    int *live = reinterpret_cast<int *>(gmask + 1024);               // [gq]
    __shared__ int n_live;

    cg::cluster_group cluster = cg::this_cluster();
    const int KS = (int)gridDim.x;
    const int s = (int)blockIdx.x;
    const int nb = (int)blockIdx.y;
    const int tid = (int)threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int ct = tid - 32;
    const int n = ct % kDownRows, half = ct / kDownRows;
    const int gq = (G + KS - 1) / KS;
    const int gbeg = s * gq, gend = min(G, gbeg + gq);

    for (int gi = warp; gi < gend - gbeg; gi += (32 + 2 * kDownRows) / 32) {
        const uint32_t m = group_token_mask(mask, T, W, gbeg + gi);
        if (lane == 0)
            gmask[gi] = m;
    }
    if (tid == 0) {
        for (int st = 0; st < kStages; ++st) {
            mbar_init(&full[st], 1);
            mbar_init(&empty[st], kConsumerWarps);
        }
        fence_mbar_init();
        tma_prefetch_desc(&tm_down);
        tma_prefetch_desc(&tm_h);
    }
    // token pairs TP..TT/2-1 of every h stage stay zero (TMA writes pairs < TP)
    if (TT / 2 > TP) {
        for (int st = 0; st < kStages; ++st)
            for (int i = tid; i < (TT / 2 - TP) * 2 * KT; i += 32 + 2 * kDownRows)
                reinterpret_cast<float *>(stages + st * stage_bytes + kWBytes)[TP * 2 * KT + i] =
                    0.f;
    }
    __syncthreads();
    if (tid == 0) {
        int k = 0;
        for (int gi = 0; gi < gend - gbeg; ++gi)
            if (gmask[gi])
                live[k++] = gi;
        n_live = k;
    }
    __syncthreads();
    const int ntile = n_live * TPG;

    bool timeout = false;
    float2 acc[kNTok / 2];                                // token pairs
#pragma unroll
    for (int t = 0; t < kNTok / 2; ++t)
        acc[t] = make_float2(0.f, 0.f);
    if (warp == 0) {
        if (lane == 0) {
            for (int kt = 0; kt < ntile; ++kt) {
                const int st = kt % kStages;
                if (kt >= kStages && !mbar_wait(&empty[st], (uint32_t)(kt / kStages - 1) & 1u)) {
                    timeout = true;
                    break;
                }
                const int gg = gbeg + live[kt / TPG];
                const int col = gg * GS + (kt % TPG) * KT;
                uint8_t *dst = stages + st * stage_bytes;
                mbar_arrive_expect_tx(&full[st], kWBytes + hbytes);
                tma_load_2d(dst, &tm_down, col, nb * kDownRows, &full[st]);
                tma_load_2d(dst + kWBytes, &tm_h, 2 * col, 0, &full[st]);   // interleaved pairs
            }
        }
    } else {
        for (int kt = 0; kt < ntile; ++kt) {
            const int st = kt % kStages;
            if (!mbar_wait(&full[st], (uint32_t)(kt / kStages) & 1u)) {
                timeout = true;
                break;
            }
            const uint32_t tm = gmask[live[kt / TPG]];
            const uint8_t *tw = stages + st * stage_bytes;
            const float *hs = reinterpret_cast<const float *>(tw + kWBytes);
#pragma unroll 1
            for (int jj = 0; jj < 4; ++jj) {
                const int j = half * 4 + jj;
                float w[EPC];
                chunk_to_f32<TIn>(*reinterpret_cast<const uint4 *>(tw + swz128(n, j)), w);
#pragma unroll
                for (int t0 = 0; t0 < kNTok; t0 += TB) {
                    if (t0 >= TT)
                        break;
                    if (((tm >> t0) & kBlockMask) == 0u)
                        continue;
                    fma1_pairs<EPC, TB / 2>(w, hs + (size_t)(t0 / 2) * 2 * KT + j * EPC * 2,
                                            2 * KT, &acc[t0 / 2]);
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&empty[st]);
        }
    }
    if (__syncthreads_or(timeout)) {
        timeout = true;
        if (tid == 0) {
            set_status(status, WIDE_DEV_TIMEOUT);
            for (int st = 0; st < kStages && st < ntile; ++st) {
                const int last = st + (ntile - 1 - st) / kStages * kStages;
                mbar_wait(&full[st], (uint32_t)(last / kStages) & 1u);
            }
        }
        __syncthreads();
    }

    float *part = reinterpret_cast<float *>(stages);  // [2][kNTok][128]
    if (warp > 0) {
#pragma unroll
        for (int t = 0; t < kNTok; ++t) {
            if (t >= T)
                break;
            part[(half * kNTok + t) * kDownRows + n] =
                timeout ? 0.f : ((t & 1) ? acc[t >> 1].y : acc[t >> 1].x);
        }
    }
    cluster.sync();
    if (warp > 0 && half == 0) {
        for (int t = s; t < T; t += KS) {
            float sum = 0.f;
            for (int q = 0; q < KS; ++q) {
                const float *rp = cluster.map_shared_rank(part, q);
                sum += rp[t * kDownRows + n] + rp[(kNTok + t) * kDownRows + n];
            }
            const size_t at = (size_t)t * H + (size_t)nb * kDownRows + n;
            if (o.out_sum)
                static_cast<TIn *>(o.out_sum)[at] = from_f32<TIn>(sum);
            if (o.out_total || o.out_total_f32) {
                float tot = sum;
                if (o.res_in)
                    tot += to_f32(static_cast<const TIn *>(o.res_in)[at]);
                if (o.res_f32)
                    tot += o.res_f32[at];
                if (o.out_total)
                    static_cast<TIn *>(o.out_total)[at] = from_f32<TIn>(tot);
                if (o.out_total_f32)
                    o.out_total_f32[at] = tot;
            }
        }
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

template <typename TIn, int GS>
int gateup_chunk(const TIn *x, const TIn *wg, const TIn *wu, const uint32_t *mask, float *h, int T,
                 int H, int I, cudaStream_t s)
{
    constexpr int EPC = ElemTraits<TIn>::EPC;
    constexpr int KT = 8 * EPC;
    const int G = I / GS, W = (G + 31) / 32;
    int KS = 8;
    while (KS > 1 && (H % (KS * KT)) != 0)
        KS >>= 1;
    const int kslice = H / KS;
    CUtensorMap tg, tu;
    if (!make_tmap_2d(&tg, wg, I, H, H, sizeof(TIn), GS, KT, true) ||
        !make_tmap_2d(&tu, wu, I, H, H, sizeof(TIn), GS, KT, true))
        return WIDE_CUDA_FAIL();
    const int TB = T >= 8 ? 8 : (T >= 4 ? 4 : 2);      // even: tokens go in pairs
    const size_t TT = (size_t)((T + TB - 1) / TB * TB);
    const size_t smem1 = 1024 + kStages * 2 * GS * 128 + 512 + TT * kslice * 4;
    const dim3 grid(KS, G), block(32 + 2 * GS);
#define WIDE_GU(TBV)                                                                               \
    launch_cluster(KID_DECODE_GATEUP, ffn_decode_gateup<TIn, GS, TBV>, grid, block, smem1, KS, s, \
                   tg, tu, x, mask, h, T, H, I, W, kslice, status_ptr())
    if (TB == 8)
        return WIDE_GU(8);
    if (TB == 4)
        return WIDE_GU(4);
    return WIDE_GU(2);
#undef WIDE_GU
}

template <typename TIn, int GS>
int down_chunk(const TIn *wd, const float *h, const uint32_t *mask, const DownOutputs &o, int T,
               int H, int I, cudaStream_t s)
{
    constexpr int EPC = ElemTraits<TIn>::EPC;
    constexpr int KT = 8 * EPC;
    const int G = I / GS, W = (G + 31) / 32;
    CUtensorMap td, th;
    // h holds token pairs interleaved: [ceil(T/2)][I][2] fp32, i.e. rows of
    // 2*I floats; a box is the KT columns of a tile for every pair
    const int TP = (T + 1) / 2;
    if (!make_tmap_2d(&td, wd, H, I, I, sizeof(TIn), kDownRows, KT, true) ||
        !make_tmap_2d(&th, h, TP, 2 * (uint64_t)I, 2 * (uint64_t)I, 4, TP, 2 * KT, false))
        return WIDE_CUDA_FAIL();
    const int KSd = G < 8 ? G : 8;
    const int TB = T >= 8 ? 8 : (T >= 4 ? 4 : 2);      // even: tokens go in pairs
    const size_t hb = (size_t)((T + TB - 1) / TB * TB) * KT * 4;
    const size_t stage = (size_t)kDownRows * 128 + ((hb + 1023) & ~(size_t)1023);
    const size_t smem2 = 1024 + kStages * stage + 64 + 1024 * 4 + 1024 * 4;
    const dim3 grid(KSd, H / kDownRows), block(32 + 2 * kDownRows);
#define WIDE_DN(TBV)                                                                               \
    launch_cluster(KID_DECODE_DOWN, ffn_decode_down<TIn, GS, TBV>, grid, block, smem2, KSd, s, td, \
                   th, mask, o, T, H, I, W, G, status_ptr())
    if (TB == 8)
        return WIDE_DN(8);
    if (TB == 4)
        return WIDE_DN(4);
    return WIDE_DN(2);
#undef WIDE_DN
}

template <typename TIn, int GS>
int decode_chunk(const TIn *x, const TIn *wg, const TIn *wu, const TIn *wd, const uint32_t *mask,
                 TIn *out, int T, int H, int I, float *h, cudaStream_t s)
{
    int rc = gateup_chunk<TIn, GS>(x, wg, wu, mask, h, T, H, I, s);
    if (rc)
        return rc;
    DownOutputs o = {};
    o.out_sum = out;
    return down_chunk<TIn, GS>(wd, h, mask, o, T, H, I, s);
}

template <typename TIn, int GS>
int decode_all(const void *x, const void *wg, const void *wu, const void *wd,
               const uint32_t *mask, void *out, const wide_ffn_dims *d, void *ws,
               cudaStream_t s)
{
    const int64_t T = d->tokens, H = d->hidden, I = d->inter;
    const int W = (int)((I / GS + 31) / 32);
    for (int64_t t0 = 0; t0 < T; t0 += kNTok) {
        const int Tc = (int)(T - t0 < kNTok ? T - t0 : kNTok);
        int rc = decode_chunk<TIn, GS>(
            static_cast<const TIn *>(x) + t0 * H, static_cast<const TIn *>(wg),
            static_cast<const TIn *>(wu), static_cast<const TIn *>(wd), mask + t0 * W,
            static_cast<TIn *>(out) + t0 * H, Tc, (int)H, (int)I, static_cast<float *>(ws), s);
        if (rc)
            return rc;
    }
    return WIDE_OK;
}

}  // namespace

int decode_gateup_bf16(const void *x, const void *wg, const void *wu, const uint32_t *mask,
                       float *h, int T, int H, int I, int gs, cudaStream_t s)
{
    if (T <= 0 || T > kNTok)
        return WIDE_EINVAL;
    const auto *xb = static_cast<const __nv_bfloat16 *>(x);
    const auto *gb = static_cast<const __nv_bfloat16 *>(wg);
    const auto *ub = static_cast<const __nv_bfloat16 *>(wu);
    if (gs == 128)
        return gateup_chunk<__nv_bfloat16, 128>(xb, gb, ub, mask, h, T, H, I, s);
    if (gs == 64)
        return gateup_chunk<__nv_bfloat16, 64>(xb, gb, ub, mask, h, T, H, I, s);
    return WIDE_EUNSUPPORTED;
}

int decode_down_bf16(const void *wd, const float *h, const uint32_t *mask, const DownOutputs &o,
                     int T, int H, int I, int gs, cudaStream_t s)
{
    if (T <= 0 || T > kNTok)
        return WIDE_EINVAL;
    const auto *db = static_cast<const __nv_bfloat16 *>(wd);
    if (gs == 128)
        return down_chunk<__nv_bfloat16, 128>(db, h, mask, o, T, H, I, s);
    if (gs == 64)
        return down_chunk<__nv_bfloat16, 64>(db, h, mask, o, T, H, I, s);
    if (gs == 256)
        return down_chunk<__nv_bfloat16, 256>(db, h, mask, o, T, H, I, s);
    if (gs == 512)
        return down_chunk<__nv_bfloat16, 512>(db, h, mask, o, T, H, I, s);
    return WIDE_EUNSUPPORTED;
}

size_t ffn_decode_h_bytes(const wide_ffn_dims *d)
{
    // h of up to 32 tokens, token pairs interleaved (an odd count rounds
    // up); at least the persistent kernels' fp32 [T][H] accumulator
    const int64_t T = d->tokens < kNTok ? d->tokens : kNTok;
    const int64_t Tp = T > 0 ? (T + 1) / 2 * 2 : 2;
    const size_t T4 = (size_t)(T > 0 ? T + 3 : 4) / 4 * 4;    // the tensor-core kernel's [H][T4]
    const size_t h = (size_t)Tp * (size_t)d->inter, acc = T4 * d->hidden;
    return align_up((h > acc ? h : acc) * sizeof(float), 256);
}

// h scratch, then 256 bytes: a persistent kernel's accumulator may take all
// of h_bytes, its arrival counter sits after it
size_t ffn_decode_workspace(const wide_ffn_dims *d) { return ffn_decode_h_bytes(d) + 256; }

int ffn_decode_run(const void *x, const void *wg, const void *wu, const void *wd,
                   const uint32_t *mask, void *out, const wide_ffn_dims *d, float *h,
                   size_t h_cap, cudaStream_t s, const void *packed)
{
    if (d->tokens == 0)
        return WIDE_OK;
    const int64_t gs = d->group_size;
    if (d->dtype == WIDE_BF16) {
        const int H = (int)d->hidden, I = (int)d->inter;
        const int64_t T = d->tokens;
        if (decode_ffn_persistent_available(T, H, I, (int)gs, h_cap, packed)) {
            DownOutputs o = {};
            o.out_sum = out;
            return decode_ffn_persistent(x, wg, wu, wd, mask, o, T, H, I, (int)gs, h, h_cap, s,
                                         packed);
        }
        if (gs == 128)
            return decode_all<__nv_bfloat16, 128>(x, wg, wu, wd, mask, out, d, h, s);
        if (gs == 64)
            return decode_all<__nv_bfloat16, 64>(x, wg, wu, wd, mask, out, d, h, s);
    } else {
        if (gs == 128)
            return decode_all<float, 128>(x, wg, wu, wd, mask, out, d, h, s);
        if (gs == 64)
            return decode_all<float, 64>(x, wg, wu, wd, mask, out, d, h, s);
        if (gs == 32)
            return decode_all<float, 32>(x, wg, wu, wd, mask, out, d, h, s);
    }
    return WIDE_EUNSUPPORTED;
}

int ffn_decode_launch(const void *x, const void *wg, const void *wu, const void *wd,
                      const uint32_t *mask, void *out, const wide_ffn_dims *d, void *ws,
                      cudaStream_t s, const void *packed)
{
    // h and the 256 bytes after it: ffn_decode_h_bytes + 256 contiguous bytes
    return ffn_decode_run(x, wg, wu, wd, mask, out, d, static_cast<float *>(ws),
                          ffn_decode_h_bytes(d) + 256, s, packed);
}

}  // namespace wide
