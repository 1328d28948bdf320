// reorder.cu -- device-side mask reordering (WIDE, technical summary
// section 2.B: per routing group, sort the binary mask along the token
// dimension M so that active tokens form a contiguous prefix).
//
// Two launches, no host synchronisation:
//   k1  blocks [0, G)            stable partition of group g's token column
//                                (ballot + block prefix scan, two passes)
//       blocks [G, G + tiles*S)  partial signature ranks: token t counts the
//                                tokens u of one slice whose mask row sorts
//                                before its own (big-endian key, ties by index)
//   k2  blocks [0, tiles)        rank = sum of partials; scatter sig_perm,
//                                sig_pos; OR rows into tile_union
//       block  tiles             (group, tile) work items from count[]
#include "common.cuh"
#include "host.h"

namespace wide {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ uint32_t lanemask_lt()
{
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

__global__ void __launch_bounds__(kThreads)
    reorder_k1(const uint32_t *__restrict__ mask, int T, int G, int W, int tile_m, int S,
               int32_t *__restrict__ count, int32_t *__restrict__ perm,
               int32_t *__restrict__ scratch, uint32_t *__restrict__ tile_union,
               int32_t *status)
{
    __shared__ int warp_act[kWarps], warp_val[kWarps];
    extern __shared__ __align__(16) uint32_t dyn_keys[];  // [2][W][kThreads], or uint4[kThreads]
    uint32_t *ukeys = dyn_keys, *tkeys = dyn_keys + W * kThreads;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;

    if (blockIdx.x < (unsigned)G) {
        // ---- stable partition of group g
        const int g = blockIdx.x, w = g >> 5;
        const uint32_t bit = 1u << (g & 31);
        if (g == 0) {
            const int nt = (T + tile_m - 1) / tile_m;
            for (int i = tid; i < nt * W; i += kThreads)
                tile_union[i] = 0u;
        }
        int cnt = 0;
        for (int base = 0; base < T; base += kThreads) {
            const int t = base + tid;
            const int a = (t < T) && (mask[(size_t)t * W + w] & bit);
            cnt += __syncthreads_count(a);
        }
        int act_off = 0, ina_off = cnt;
        for (int base = 0; base < T; base += kThreads) {
            const int t = base + tid;
            const bool valid = t < T;
            const bool a = valid && (mask[(size_t)t * W + w] & bit);
            const uint32_t ba = __ballot_sync(0xffffffffu, a);
            const uint32_t bv = __ballot_sync(0xffffffffu, valid);
            if (lane == 0) {
                warp_act[wid] = __popc(ba);
                warp_val[wid] = __popc(bv);
            }
            __syncthreads();
            int pa = 0, pv = 0, ta = 0, tv = 0;
#pragma unroll
            for (int i = 0; i < kWarps; ++i) {
                if (i < wid) {
                    pa += warp_act[i];
                    pv += warp_val[i];
                }
                ta += warp_act[i];
                tv += warp_val[i];
            }
            const int ra = pa + __popc(ba & lanemask_lt());
            const int rv = pv + __popc(bv & lanemask_lt());
            if (valid) {
                const int pos = a ? act_off + ra : ina_off + (rv - ra);
                perm[(size_t)g * T + pos] = t;
            }
            act_off += ta;
            ina_off += tv - ta;
            __syncthreads();
        }
        if (tid == 0)
            count[g] = cnt;
        return;
    }

    // ---- partial signature ranks
    const int rb = blockIdx.x - G;
    const int ti = rb / S, s = rb % S;
    const int t = ti * kThreads + tid;
    const int chunk = (T + S - 1) / S;
    const int u0 = s * chunk, u1 = min(T, u0 + chunk);
    if (t < T) {
        for (int ww = 0; ww < W; ++ww)
            tkeys[ww * kThreads + tid] = mask[(size_t)t * W + ww];
        if (s == 0 && (G & 31) != 0 && (mask[(size_t)t * W + W - 1] >> (G & 31)) != 0u)
            set_status(status, WIDE_DEV_BAD_MASK);
    }
    int less = 0;
    if (W <= 4) {
        // keys of up to 128 bits: the slice's keys as uint4 in shared memory
        // (one broadcast load per comparison), this token's key in registers,
        // compared as two 64-bit halves (word W-1 most significant)
        uint4 *uk4 = reinterpret_cast<uint4 *>(dyn_keys);
        uint32_t tw[4] = {0u, 0u, 0u, 0u};
        if (t < T)
            for (int ww = 0; ww < W; ++ww)
                tw[ww] = mask[(size_t)t * W + ww];
        const uint64_t th = ((uint64_t)tw[3] << 32) | tw[2], tl = ((uint64_t)tw[1] << 32) | tw[0];
        for (int ub = u0; ub < u1; ub += kThreads) {
            __syncthreads();
            {
                const int u = ub + tid;
                uint32_t kw[4] = {0u, 0u, 0u, 0u};
                if (u < u1)
                    for (int ww = 0; ww < W; ++ww)
                        kw[ww] = mask[(size_t)u * W + ww];
                uk4[tid] = make_uint4(kw[0], kw[1], kw[2], kw[3]);
            }
            __syncthreads();
            const int n = min(kThreads, u1 - ub);
#pragma unroll 4
            for (int j = 0; j < n; ++j) {
                const uint4 k = uk4[j];
                const uint64_t uh = ((uint64_t)k.w << 32) | k.z, ul = ((uint64_t)k.y << 32) | k.x;
                less += (uh < th) | ((uh == th) & ((ul < tl) | ((ul == tl) & (ub + j < t))));
            }
        }
        if (t < T)
            scratch[(size_t)s * T + t] = less;
        return;
    }
    for (int ub = u0; ub < u1; ub += kThreads) {
        __syncthreads();
        for (int idx = tid; idx < kThreads * W; idx += kThreads) {
            const int j = idx % kThreads, ww = idx / kThreads, u = ub + j;
            ukeys[ww * kThreads + j] = (u < u1) ? mask[(size_t)u * W + ww] : 0u;
        }
        __syncthreads();
        const int n = min(kThreads, u1 - ub);
        if (t < T) {
            for (int j = 0; j < n; ++j) {
                int c = 0;
                for (int ww = W - 1; ww >= 0; --ww) {
                    const uint32_t ku = ukeys[ww * kThreads + j];
                    const uint32_t kt = tkeys[ww * kThreads + tid];
                    if (ku != kt) {
                        c = ku < kt ? -1 : 1;
                        break;
                    }
                }
                less += (c < 0) || (c == 0 && ub + j < t);
            }
        }
    }
    if (t < T)
        scratch[(size_t)s * T + t] = less;
}

__global__ void __launch_bounds__(kThreads)
    reorder_k2(const uint32_t *__restrict__ mask, int T, int G, int W, int tile_m, int S,
               const int32_t *__restrict__ count, const int32_t *__restrict__ scratch,
               int32_t *__restrict__ items, int32_t *__restrict__ n_items,
               int32_t *__restrict__ sig_perm, int32_t *__restrict__ sig_pos,
               uint32_t *__restrict__ tile_union)
{
    const int tid = threadIdx.x;
    const int tiles = (T + kThreads - 1) / kThreads;
    if (blockIdx.x < (unsigned)tiles) {
        const int t = blockIdx.x * kThreads + tid;
        if (t < T) {
            int r = 0;
            for (int s = 0; s < S; ++s)
                r += scratch[(size_t)s * T + t];
            sig_perm[r] = t;
            sig_pos[t] = r;
            const int tile = r / tile_m;
            for (int w = 0; w < W; ++w) {
                const uint32_t k = mask[(size_t)t * W + w];
                if (k)
                    atomicOr(&tile_union[(size_t)tile * W + w], k);
            }
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

}  // namespace

int reorder_splits(int64_t T)
{
    const int64_t tiles = (T + kThreads - 1) / kThreads;
    if (tiles <= 0)
        return 1;
    int64_t S = (4 * 148 + tiles - 1) / tiles;
    S = S < 1 ? 1 : (S > 64 ? 64 : S);
    const int64_t cap = T / 32 > 1 ? T / 32 : 1;
    return (int)(S > cap ? cap : S);
}

int reorder_launch(const uint32_t *mask, int64_t T, int64_t G, int32_t tile_m,
                   const wide_worklist *wl, cudaStream_t s)
{
    const int W = (int)((G + 31) / 32);
    const int S = wl->scratch_splits;
    const int tiles = (int)((T + kThreads - 1) / kThreads);
    // [2][W][kThreads] words (the keys of the generic path; the prologue
    // writes this token's key there for every W), at least uint4[kThreads]
    const size_t smem = (size_t)(2 * W > 4 ? 2 * W : 4) * kThreads * sizeof(uint32_t);
    if (!raise_smem_limit(reinterpret_cast<const void *>(reorder_k1), smem))
        return WIDE_CUDA_FAIL();
    {
        LaunchScope scope(KID_REORDER_PARTITION_RANK, s);
        reorder_k1<<<(unsigned)(G + (int64_t)tiles * S), kThreads, smem, s>>>(
            mask, (int)T, (int)G, W, tile_m, S, wl->count, wl->perm, wl->scratch,
            wl->tile_union, status_ptr());
    }
    int rc = launch_status();
    if (rc)
        return rc;
    {
        LaunchScope scope(KID_REORDER_FINISH, s);
        reorder_k2<<<(unsigned)(tiles + 1), kThreads, 0, s>>>(
            mask, (int)T, (int)G, W, tile_m, S, wl->count, wl->scratch, wl->items, wl->n_items,
            wl->sig_perm, wl->sig_pos, wl->tile_union);
    }
    return launch_status();
}

}  // namespace wide
