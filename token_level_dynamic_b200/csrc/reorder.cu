// reorder.cu -- device-side mask reordering (WIDE, technical summary
// section 2.B: per routing group, sort the binary mask along the token
// dimension M so that active tokens form a contiguous prefix).
//
// A memset of the rank counters and three launches, no host
// synchronisation:
//   k1  blocks [0, G)        stable partition of group g's token column
//                            (32-token ballots, one block scan per segment)
//       blocks [G, G+tiles)  signature buckets: the top B = min(12, G) bits
//                            of each token's key (the mask row read as one
//                            big-endian number); a histogram of them
//   k2  blocks [0, tiles)    exclusive scan of the histogram (every block
//                            for itself), then each token's slot in its
//                            bucket's member list (any order inside a bucket)
//       block  tiles         (group, tile) work items from count[]
//   k3  blocks [0, tiles*S)  signature rank of the tokens at member-list
//                            positions [256 i, 256 i + 256): the bucket's
//                            offset plus the members of the same bucket
//                            whose key sorts before (ties by token index);
//                            the bucket range of a block is split over S
//                            blocks whose counts meet by atomics, and the
//                            last of them scatters sig_perm and sig_pos and
//                            ORs the rows into tile_union.
// Comparing a token only against its own bucket turns the O(T^2) rank into
// the sum of squared bucket sizes; with every key equal it is O(T^2) again,
// spread over tiles * S blocks.
#include "common.cuh"
#include "host.h"

namespace wide {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kSeg = 8192;                  // partition: tokens per segment
constexpr int kPerWarp = kSeg / kWarps;     // 1024 tokens = 32 ballots per warp
constexpr int kBucketBits = 12;
constexpr int kNB = 1 << kBucketBits;       // histogram bins

__device__ __forceinline__ uint32_t lanemask_lt()
{
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Word i of a key of up to 4 words held in a uint4 (i < 4).
__device__ __forceinline__ uint32_t kw4(const uint4 k, int i)
{
    return i == 0 ? k.x : i == 1 ? k.y : i == 2 ? k.z : k.w;
}

// The top B bits of a G-bit key (bit g of the key = group g; group G-1 is
// the most significant), from the words of the key in a uint4 (G <= 128).
__device__ __forceinline__ int bucket4(const uint4 k, int G, int B)
{
    const int lo = G - B, wl = lo >> 5, sh = lo & 31;
    const uint64_t v = ((uint64_t)(wl + 1 < 4 ? kw4(k, wl + 1) : 0u) << 32) | kw4(k, wl);
    return (int)((v >> sh) & ((1u << B) - 1u));
}

// Same for a key of any width read from memory.
__device__ __forceinline__ int bucket_mem(const uint32_t *key, int W, int G, int B)
{
    const int lo = G - B, wl = lo >> 5, sh = lo & 31;
    const uint64_t v = ((uint64_t)(wl + 1 < W ? key[wl + 1] : 0u) << 32) | key[wl];
    return (int)((v >> sh) & ((1u << B) - 1u));
}

// Scratch words: [hist kNB][fill kNB][arrive tiles][acc T] (zeroed by the
// memset), then [members T][off kNB].
struct RScratch {
    int32_t *hist, *fill, *arrive, *acc, *members, *off;
};
__host__ __device__ inline RScratch rscratch(int32_t *base, int T)
{
    const int tiles = (T + kThreads - 1) / kThreads;
    RScratch r;
    r.hist = base;
    r.fill = r.hist + kNB;
    r.arrive = r.fill + kNB;
    r.acc = r.arrive + tiles;
    r.members = r.acc + T;
    r.off = r.members + T;
    return r;
}

__global__ void __launch_bounds__(kThreads)
    reorder_k1(const uint32_t *__restrict__ mask, int T, int G, int W, int tile_m, int B,
               int32_t *__restrict__ count, int32_t *__restrict__ perm, RScratch sc,
               uint32_t *__restrict__ tile_union, int32_t *status)
{
    __shared__ int warp_act[kWarps], s_total;
    __shared__ uint32_t seg_bal[kWarps][kPerWarp / 32];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;

    if (blockIdx.x < (unsigned)G) {
        // ---- stable partition of group g.  The tokens are taken in
        // segments of kSeg; within a segment warp w owns kSeg / kWarps
        // consecutive tokens.  Pass 1 stores each 32-token ballot of group
        // g's bit in shared memory and counts per warp; one block scan gives
        // every warp its offsets among the active and the inactive tokens;
        // pass 2 writes the positions from the stored ballots.
        const int g = blockIdx.x, w = g >> 5;
        const uint32_t bit = 1u << (g & 31);
        if (g == 0) {
            const int nt = (T + tile_m - 1) / tile_m;
            for (int i = tid; i < nt * W; i += kThreads)
                tile_union[i] = 0u;
        }
        // the group's active count (the inactive prefix starts after it): a
        // counting pass first, unless one segment holds every token
        if (T > kSeg) {
            int c = 0;
            for (int t = tid; t < T; t += kThreads)
                c += (mask[(size_t)t * W + w] & bit) ? 1 : 0;
            for (int off = 16; off; off >>= 1)
                c += __shfl_xor_sync(0xffffffffu, c, off);
            if (lane == 0)
                warp_act[wid] = c;
            __syncthreads();
            if (tid == 0) {
                int tot = 0;
                for (int i = 0; i < kWarps; ++i)
                    tot += warp_act[i];
                s_total = tot;
            }
            __syncthreads();
        }
        int act_base = 0;                   // active tokens in earlier segments
        for (int seg = 0; seg < T; seg += kSeg) {
            const int w0 = seg + wid * kPerWarp;
            int cnt = 0;
#pragma unroll 8
            for (int i = 0; i < kPerWarp / 32; ++i) {
                const int t = w0 + i * 32 + lane;
                const bool a = t < T && (mask[(size_t)t * W + w] & bit);
                const uint32_t ba = __ballot_sync(0xffffffffu, a);
                if (lane == 0)
                    seg_bal[wid][i] = ba;
                cnt += __popc(ba);
            }
            if (lane == 0)
                warp_act[wid] = cnt;
            __syncthreads();
            int before = 0, seg_act = 0;
#pragma unroll
            for (int i = 0; i < kWarps; ++i) {
                before += i < wid ? warp_act[i] : 0;
                seg_act += warp_act[i];
            }
            const int total = T > kSeg ? s_total : seg_act;
            int act_off = act_base + before;
            int ina_off = (w0 - act_base - before);   // inactive tokens before this warp
            for (int i = 0; i < kPerWarp / 32; ++i) {
                const int t = w0 + i * 32 + lane;
                const uint32_t ba = seg_bal[wid][i];
                const int na = __popc(ba & lanemask_lt());
                if (t < T) {
                    const bool a = (ba >> lane) & 1u;
                    perm[(size_t)g * T + (a ? act_off + na : total + ina_off + (lane - na))] = t;
                }
                const int n = __popc(ba);
                act_off += n;
                ina_off += min(32, max(0, T - (w0 + i * 32))) - n;
            }
            act_base += seg_act;
            __syncthreads();
        }
        if (tid == 0)
            count[g] = act_base;
        return;
    }

    // ---- signature buckets and their histogram
    const int t = ((int)blockIdx.x - G) * kThreads + tid;
    if (t < T) {
        const uint32_t *key = mask + (size_t)t * W;
        if ((G & 31) != 0 && (key[W - 1] >> (G & 31)) != 0u)
            set_status(status, WIDE_DEV_BAD_MASK);
        atomicAdd(&sc.hist[bucket_mem(key, W, G, B)], 1);
    }
}

// Exclusive scan of the histogram into off_s (kThreads threads, kNB bins).
__device__ __forceinline__ void scan_hist(const int32_t *hist, int32_t *off_s, int *wsum)
{
    constexpr int per = kNB / kThreads;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    int v[per], sum = 0;
#pragma unroll
    for (int i = 0; i < per; ++i) {
        v[i] = __ldcg(&hist[tid * per + i]);
        sum += v[i];
    }
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off)
            incl += x;
    }
    if (lane == 31)
        wsum[wid] = incl;
    __syncthreads();
    int base = incl - sum;
    for (int i = 0; i < wid; ++i)
        base += wsum[i];
#pragma unroll
    for (int i = 0; i < per; ++i) {
        off_s[tid * per + i] = base;
        base += v[i];
    }
    __syncthreads();
}

__global__ void __launch_bounds__(kThreads)
    reorder_k2(const uint32_t *__restrict__ mask, int T, int G, int W, int tile_m, int B,
               const int32_t *__restrict__ count, RScratch sc, int32_t *__restrict__ items,
               int32_t *__restrict__ n_items)
{
    __shared__ int32_t off_s[kNB];
    __shared__ int wsum[kWarps];
    const int tid = threadIdx.x;
    const int tiles = (T + kThreads - 1) / kThreads;
    if (blockIdx.x < (unsigned)tiles) {
        scan_hist(sc.hist, off_s, wsum);
        if (blockIdx.x == 0)
            for (int i = tid; i < kNB; i += kThreads)
                sc.off[i] = off_s[i];
        const int t = blockIdx.x * kThreads + tid;
        if (t < T) {
            const int b = bucket_mem(mask + (size_t)t * W, W, G, B);
            sc.members[off_s[b] + atomicAdd(&sc.fill[b], 1)] = t;
        }
        return;
    }
    // ---- work items, group-major: exclusive scan of ceil(count[g] / tile_m)
    __shared__ int sh[kThreads];
    const int per = (G + kThreads - 1) / kThreads;
    const int g0 = tid * per, g1 = min(G, g0 + per);
    int local = 0;
    for (int g = g0; g < g1; ++g)
        local += (count[g] + tile_m - 1) / tile_m;
    sh[tid] = local;
    __syncthreads();
    for (int d = 1; d < kThreads; d <<= 1) {
        const int v = tid >= d ? sh[tid - d] : 0;
        __syncthreads();
        sh[tid] += v;
        __syncthreads();
    }
    int off = sh[tid] - local;
    for (int g = g0; g < g1; ++g) {
        const int n = (count[g] + tile_m - 1) / tile_m;
        for (int i = 0; i < n; ++i) {
            items[2 * (off + i)] = g;
            items[2 * (off + i) + 1] = i;
        }
        off += n;
    }
    if (tid == kThreads - 1)
        n_items[0] = sh[kThreads - 1];
}

// k3: ranks of the tokens at member-list positions [256 i, 256 i + 256),
// split sp of S over the block's bucket range.  WIDE keys (W > 4) are
// staged and compared word by word; narrower ones as two 64-bit halves.
template <bool kWide>
__global__ void __launch_bounds__(kThreads)
    reorder_k3(const uint32_t *__restrict__ mask, int T, int G, int W, int tile_m, int B, int S,
               RScratch sc, int32_t *__restrict__ sig_perm, int32_t *__restrict__ sig_pos,
               uint32_t *__restrict__ tile_union)
{
    extern __shared__ __align__(16) uint32_t dyn[];   // staged keys: [kThreads][4] or [kThreads][W]
    __shared__ int s_b[kThreads], s_t[kThreads];
    __shared__ int s_r0, s_r1, s_last;
    const int tid = threadIdx.x;
    const int i = (int)blockIdx.x / S, sp = (int)blockIdx.x % S;
    const int p0 = i * kThreads, p1 = min(T, p0 + kThreads);
    const int p = p0 + tid;
    const bool own = p < p1;
    const int t = own ? sc.members[p] : -1;
    const uint32_t *tkey = mask + (size_t)(own ? t : 0) * W;
    uint4 k4 = make_uint4(0u, 0u, 0u, 0u);
    if (!kWide && own) {
        k4.x = tkey[0];
        if (W > 1) k4.y = tkey[1];
        if (W > 2) k4.z = tkey[2];
        if (W > 3) k4.w = tkey[3];
    }
    const int bt = own ? (kWide ? bucket_mem(tkey, W, G, B) : bucket4(k4, G, B)) : -1;
    const uint64_t th = ((uint64_t)k4.w << 32) | k4.z, tl = ((uint64_t)k4.y << 32) | k4.x;
    if (tid == 0) {
        const int bf = bucket_mem(mask + (size_t)sc.members[p0] * W, W, G, B);
        const int bl = bucket_mem(mask + (size_t)sc.members[p1 - 1] * W, W, G, B);
        s_r0 = __ldcg(&sc.off[bf]);
        s_r1 = __ldcg(&sc.off[bl]) + __ldcg(&sc.hist[bl]);
    }
    __syncthreads();
    const int r0 = s_r0, n = s_r1 - s_r0;
    const int lo = r0 + (int)((int64_t)n * sp / S), hi = r0 + (int)((int64_t)n * (sp + 1) / S);
    int less = 0;
    for (int ub = lo; ub < hi; ub += kThreads) {
        __syncthreads();
        {
            const int u = ub + tid;
            int bu = -2, tu = 0;
            if (u < hi) {
                tu = sc.members[u];
                const uint32_t *uk = mask + (size_t)tu * W;
                if (kWide) {
                    for (int ww = 0; ww < W; ++ww)
                        dyn[(size_t)tid * W + ww] = uk[ww];
                    bu = bucket_mem(uk, W, G, B);
                } else {
                    uint4 q = make_uint4(uk[0], W > 1 ? uk[1] : 0u, W > 2 ? uk[2] : 0u,
                                         W > 3 ? uk[3] : 0u);
                    reinterpret_cast<uint4 *>(dyn)[tid] = q;
                    bu = bucket4(q, G, B);
                }
            }
            s_b[tid] = bu;
            s_t[tid] = tu;
        }
        __syncthreads();
        const int m = min(kThreads, hi - ub);
        if (own) {
            if (!kWide) {
                const uint4 *uk4 = reinterpret_cast<const uint4 *>(dyn);
#pragma unroll 4
                for (int j = 0; j < m; ++j) {
                    const uint4 k = uk4[j];
                    const uint64_t uh = ((uint64_t)k.w << 32) | k.z, ul = ((uint64_t)k.y << 32) | k.x;
                    const bool lt = (uh < th) | ((uh == th) & ((ul < tl) | ((ul == tl) & (s_t[j] < t))));
                    less += (s_b[j] == bt) & lt;
                }
            } else {
                for (int j = 0; j < m; ++j) {
                    if (s_b[j] != bt)
                        continue;
                    int c = 0;
                    for (int ww = W - 1; ww >= 0; --ww) {
                        const uint32_t ku = dyn[(size_t)j * W + ww], kt = tkey[ww];
                        if (ku != kt) {
                            c = ku < kt ? -1 : 1;
                            break;
                        }
                    }
                    less += (c < 0) || (c == 0 && s_t[j] < t);
                }
            }
        }
    }
    if (own && less)
        atomicAdd(&sc.acc[p], less);
    // the last split of this position block writes the ranks
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        s_last = atomicAdd(&sc.arrive[i], 1) == S - 1;
    }
    __syncthreads();
    if (!s_last)
        return;
    __threadfence();
    if (own) {
        const int r = __ldcg(&sc.off[bt]) + __ldcg(&sc.acc[p]);
        sig_perm[r] = t;
        sig_pos[t] = r;
        const int tile = r / tile_m;
        for (int w = 0; w < W; ++w) {
            const uint32_t k = tkey[w];
            if (k)
                atomicOr(&tile_union[(size_t)tile * W + w], k);
        }
    }
}

}  // namespace

int reorder_splits(int64_t T)
{
    const int64_t tiles = (T + kThreads - 1) / kThreads;
    if (tiles <= 0)
        return 1;
    const int64_t S = (2 * 148 + tiles - 1) / tiles;
    return (int)(S < 1 ? 1 : (S > 16 ? 16 : S));
}

size_t reorder_scratch_bytes(int64_t T)
{
    const int64_t tiles = (T + kThreads - 1) / kThreads;
    return sizeof(int32_t) * (size_t)(3 * kNB + tiles + 2 * T);
}

int reorder_launch(const uint32_t *mask, int64_t T, int64_t G, int32_t tile_m,
                   const wide_worklist *wl, cudaStream_t s)
{
    const int W = (int)((G + 31) / 32);
    const int S = wl->scratch_splits;
    const int B = (int)(G < kBucketBits ? G : kBucketBits);
    const int tiles = (int)((T + kThreads - 1) / kThreads);
    const RScratch sc = rscratch(wl->scratch, (int)T);
    // hist, fill, arrive and acc start at zero
    if (cudaMemsetAsync(wl->scratch, 0, sizeof(int32_t) * (size_t)(2 * kNB + tiles + T), s) !=
        cudaSuccess)
        return WIDE_CUDA_FAIL();
    {
        LaunchScope scope(KID_REORDER_PARTITION_RANK, s);
        reorder_k1<<<(unsigned)(G + tiles), kThreads, 0, s>>>(
            mask, (int)T, (int)G, W, tile_m, B, wl->count, wl->perm, sc, wl->tile_union,
            status_ptr());
    }
    int rc = launch_status();
    if (rc)
        return rc;
    {
        LaunchScope scope(KID_REORDER_FINISH, s);
        reorder_k2<<<(unsigned)(tiles + 1), kThreads, 0, s>>>(mask, (int)T, (int)G, W, tile_m, B,
                                                             wl->count, sc, wl->items,
                                                             wl->n_items);
    }
    if ((rc = launch_status()))
        return rc;
    if (tiles == 0)
        return WIDE_OK;
    {
        LaunchScope scope(KID_REORDER_FINISH, s);
        if (W > 4) {
            const size_t smem = (size_t)kThreads * W * sizeof(uint32_t);
            if (!raise_smem_limit(reinterpret_cast<const void *>(reorder_k3<true>), smem))
                return WIDE_CUDA_FAIL();
            reorder_k3<true><<<(unsigned)(tiles * S), kThreads, smem, s>>>(
                mask, (int)T, (int)G, W, tile_m, B, S, sc, wl->sig_perm, wl->sig_pos,
                wl->tile_union);
        } else {
            reorder_k3<false><<<(unsigned)(tiles * S), kThreads, kThreads * 16, s>>>(
                mask, (int)T, (int)G, W, tile_m, B, S, sc, wl->sig_perm, wl->sig_pos,
                wl->tile_union);
        }
    }
    return launch_status();
}

}  // namespace wide
