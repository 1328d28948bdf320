// ffn_decode_fused.cu -- the bf16 decode FFN as one persistent kernel.
//
// WIDE, technical summary section 2.A (each token keeps its own contiguous
// FFN channel groups) and section 2.C (block-level skipping), for decode
// batches of up to 32 tokens: the weights of the groups some token of the
// batch keeps (the batch's union) are streamed from HBM once, and no other
// weight byte is read.
//
// One CTA per SM, all resident at once (cooperative launch).
//   Phase 1: h[t][i] = silu(x[t] . W_gate[i]) * (x[t] . W_up[i]) for every
//     row i of the union (0 where token t skips i's group).  The union's
//     rows, in group order, are cut into one contiguous range per CTA in
//     units of 8 rows.  A stage holds 8 rows of W_gate and of W_up over a
//     window of KW = 1024 columns (when H is not a multiple of 1024, KW is
//     512 or 256 and a stage holds 1024 / KW units), fetched as one 3-D TMA copy
//     per unit and matrix: long contiguous row pieces stream far better than
//     2-D boxes of short rows.
//   Grid barrier: an arrival counter (zeroed on the stream before the
//     launch) that the producer of every CTA polls, bounded.
//   Phase 2: out[t][n] = sum over the union's columns i of h[t][i] *
//     W_down[n][i].  The H output rows are cut into one contiguous range per
//     CTA; the CTA walks the union's groups.
// Batches of more than 8 tokens are cut into blocks of 8; the CTAs of one
// row range (one per token block, adjacent in the grid) read the same weight
// tiles at about the same time, so HBM serves each tile once and L2 the rest.
//
// Warp 0 (one lane) streams every tile by TMA through an mbarrier ring.  It
// issues phase 2's W_down tiles as soon as ring slots free up, before the
// grid barrier; only their h tiles wait for the barrier.  Warps 1..8 compute
// in fp32 on CUDA cores: thread (row r of 4, lane c of 8) of a warp takes
// 16-byte column chunks c and c+8 of a 128-column piece -- in phase 1 the
// gate and up rows of one row of a unit over two adjacent pieces, in phase 2
// rows r + 4w + 32k of its range over each group; the 8 lanes of a row read
// 128 contiguous bytes, and the x (or h) chunk is shared by the rows of the
// warp (broadcast reads).  Products are formed two columns at a time with
// packed fp32 FMAs (even and odd columns accumulate apart); the x of 4
// tokens is loaded first and the accumulators are updated one column pair
// at a time, so consecutive FMAs into one accumulator are far apart.  In
// phase 1 the warps of a stage split its columns, so a unit's sums are
// added over the 8 lanes by shuffles and over the warps in shared memory.
#include "common.cuh"
#include "host.h"

#include <mutex>

namespace wide {
namespace {

constexpr int kFTok = 8;                    // tokens per CTA (one token block)
constexpr int kFWarps = 8;                  // consumer warps
constexpr int kFThreads = 32 * (kFWarps + 1);
constexpr int kFStageCols = 1024;           // phase 1: window columns x units per stage
constexpr uint32_t kFSlotMin = 2u * 8u * kFStageCols * 2u;   // gate + up: 32 KB
constexpr int kFMaxSlots = 8;
constexpr int kFMaxG = 1024;                // groups (union words fit one warp)
constexpr int kFMaxR2 = 3;                  // phase 2: row sets (32 rows each) per thread
constexpr int kFTQ = 4;                     // tokens whose x is held in registers at once
constexpr int kFMaxMaskWords = 1024;        // T * W

struct FusedArgs {
    const __nv_bfloat16 *x;      // [T][H] FFN input (null when xf is given)
    const float *xf;             // [T][H] fp32 rows normalised in the kernel, or null
    const __nv_bfloat16 *gamma;  // RMSNorm gain used with xf
    float eps;
    const uint32_t *mask;        // [T][W] packed group bits
    float *h;                    // [T][I] fp32 scratch
    uint32_t *bar;               // grid barrier arrival counter (0 at launch)
    DownOutputs o;
    int T, H, I, W, G, gs;
    int TG, P;                   // token blocks; row ranges (grid = P * TG)
    int kw;                      // phase-1 window columns (divides H, multiple of 128)
    int nslots;
    uint32_t slot_bytes;
    uint32_t w2_bytes;           // one W_down box (rows_box rows x gs columns)
    uint32_t h2_bytes;           // one h box (TB tokens x gs columns, fp32)
    uint32_t h2_off;             // offset of the h boxes inside a phase-2 slot
    int ng2;                     // groups per phase-2 stage
    int32_t *status;
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    const uint32_t a = smem_u32(p);
    return p + (((a + 1023u) & ~1023u) - a);
}

__device__ __forceinline__ uint4 lds128(const uint8_t *p)
{
    return *reinterpret_cast<const uint4 *>(p);
}
__device__ __forceinline__ float4 lds128f(const uint8_t *p)
{
    return *reinterpret_cast<const float4 *>(p);
}

// The 8 bf16 of one chunk as 4 fp32 pairs (columns 2i, 2i+1).  Lanes whose
// x (or h) reads start with the upper half of the chunk (sw = 1) get the
// pairs in the matching order: 4..7 first, then 0..3.  (Lanes c and c+4
// read x chunks 128 bytes apart; starting them on opposite halves keeps the
// 8 distinct 16-byte reads of a warp in distinct banks.)
__device__ __forceinline__ void widen_pairs(const uint4 v, int sw, float2 (&w)[4])
{
    const uint32_t a0 = sw ? v.z : v.x, a1 = sw ? v.w : v.y;
    const uint32_t b0 = sw ? v.x : v.z, b1 = sw ? v.y : v.w;
    w[0] = make_float2(__uint_as_float(a0 << 16), __uint_as_float(a0 & 0xffff0000u));
    w[1] = make_float2(__uint_as_float(a1 << 16), __uint_as_float(a1 & 0xffff0000u));
    w[2] = make_float2(__uint_as_float(b0 << 16), __uint_as_float(b0 & 0xffff0000u));
    w[3] = make_float2(__uint_as_float(b1 << 16), __uint_as_float(b1 & 0xffff0000u));
}

// The two float pairs of one float4.
__device__ __forceinline__ float2 lo2(const float4 v) { return make_float2(v.x, v.y); }
__device__ __forceinline__ float2 hi2(const float4 v) { return make_float2(v.z, v.w); }

// Sum over the 8 lanes of a row group (lanes 8r .. 8r+7).
__device__ __forceinline__ float sum8(float v)
{
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    return v;
}

__device__ __forceinline__ void fence_proxy_async_global()
{
    asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ void consumer_sync()
{
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kFWarps) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t *p)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void red_add_release_gpu(uint32_t *p, uint32_t v)
{
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Phase 1, one stage, one thread: row `row` of its unit of W_gate (sg) and
// W_up (su) (row stride rs bytes in the slot), chunks c and c+8 of each of
// its two 128-column pieces (xq: x at the first piece), TB tokens.
template <int TB>
__device__ __forceinline__ void p1_stage(const uint8_t *sg, const uint8_t *su, const uint8_t *xq,
                                         int H, uint32_t rs, int row, int c, int sw,
                                         float2 (&ag)[TB], float2 (&au)[TB])
{
    constexpr int TQ = TB < kFTQ ? TB : kFTQ;
    const uint32_t xo1 = sw ? 16u : 0u, xo2 = 16u - xo1;
#pragma unroll
    for (int q = 0; q < 4; ++q) {              // chunks c, c+8 of piece 0, then of piece 1
        const int j = c + 8 * q;
        float2 wg[4], wu[4];
        widen_pairs(lds128(sg + row * rs + j * 16), sw, wg);
        widen_pairs(lds128(su + row * rs + j * 16), sw, wu);
        const uint8_t *xj = xq + j * 32;
#pragma unroll
        for (int t0 = 0; t0 < TB; t0 += TQ) {
            float4 x1[TQ], x2[TQ];
#pragma unroll
            for (int t = 0; t < TQ; ++t) {
                x1[t] = lds128f(xj + (size_t)(t0 + t) * H * 4 + xo1);
                x2[t] = lds128f(xj + (size_t)(t0 + t) * H * 4 + xo2);
            }
#pragma unroll
            for (int t = 0; t < TQ; ++t) {
                ag[t0 + t] = __ffma2_rn(wg[0], lo2(x1[t]), ag[t0 + t]);
                au[t0 + t] = __ffma2_rn(wu[0], lo2(x1[t]), au[t0 + t]);
            }
#pragma unroll
            for (int t = 0; t < TQ; ++t) {
                ag[t0 + t] = __ffma2_rn(wg[1], hi2(x1[t]), ag[t0 + t]);
                au[t0 + t] = __ffma2_rn(wu[1], hi2(x1[t]), au[t0 + t]);
            }
#pragma unroll
            for (int t = 0; t < TQ; ++t) {
                ag[t0 + t] = __ffma2_rn(wg[2], lo2(x2[t]), ag[t0 + t]);
                au[t0 + t] = __ffma2_rn(wu[2], lo2(x2[t]), au[t0 + t]);
            }
#pragma unroll
            for (int t = 0; t < TQ; ++t) {
                ag[t0 + t] = __ffma2_rn(wg[3], hi2(x2[t]), ag[t0 + t]);
                au[t0 + t] = __ffma2_rn(wu[3], hi2(x2[t]), au[t0 + t]);
            }
        }
    }
}

// Phase 2, one group of one stage: rows rw + 32 k (k < R2) of the range (rows
// past the box's last row rmax read that row; their sums are discarded), the
// gs columns of the group, TB tokens.
template <int TB, int R2>
__device__ __forceinline__ void p2_group(const uint8_t *wb, const uint8_t *hb, int gs, int rw,
                                         int rmax, int c, int sw, float2 (&acc)[kFMaxR2][TB])
{
    constexpr int TQ = TB < kFTQ ? TB : kFTQ;
    const uint32_t xo1 = sw ? 16u : 0u, xo2 = 16u - xo1;
    for (int q = 0; q < gs / 64; ++q) {
        const int j = c + 8 * q;
        float2 w[R2][4];
#pragma unroll
        for (int rr = 0; rr < R2; ++rr)
            widen_pairs(lds128(wb + (size_t)min(rw + 32 * rr, rmax) * gs * 2 + j * 16), sw,
                        w[rr]);
        const uint8_t *hq = hb + j * 32;
#pragma unroll
        for (int t0 = 0; t0 < TB; t0 += TQ) {
            float4 x1[TQ], x2[TQ];
#pragma unroll
            for (int t = 0; t < TQ; ++t) {
                x1[t] = lds128f(hq + (size_t)(t0 + t) * gs * 4 + xo1);
                x2[t] = lds128f(hq + (size_t)(t0 + t) * gs * 4 + xo2);
            }
#pragma unroll
            for (int p = 0; p < 4; ++p)
#pragma unroll
                for (int t = 0; t < TQ; ++t)
#pragma unroll
                    for (int rr = 0; rr < R2; ++rr) {
                        const float2 xv = p == 0 ? lo2(x1[t]) : p == 1 ? hi2(x1[t])
                                        : p == 2 ? lo2(x2[t]) : hi2(x2[t]);
                        acc[rr][t0 + t] = __ffma2_rn(w[rr][p], xv, acc[rr][t0 + t]);
                    }
        }
    }
}

// One CTA of 9 warps per SM.  The register file is split between the SM's
// four sub-partitions and one of them holds 3 of the 9 warps, so a thread
// gets at most 16384 / 96 registers; the launch bounds let ptxas apply that.
template <int TB>
__global__ void __launch_bounds__(kFThreads, 1)
    ffn_decode_fused(const __grid_constant__ CUtensorMap tm_gate,
                     const __grid_constant__ CUtensorMap tm_up,
                     const __grid_constant__ CUtensorMap tm_down,
                     const __grid_constant__ CUtensorMap tm_h, const FusedArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    const int NS = a.nslots;
    uint8_t *slots = smem;
    float *xs = reinterpret_cast<float *>(smem + (size_t)NS * a.slot_bytes);   // [TB][H]
    float *red = xs + (size_t)TB * a.H;              // [2][4 piece pairs][8 rows][2][TB]
    uint32_t *mall = reinterpret_cast<uint32_t *>(red + 2 * 4 * 8 * 2 * TB);  // [T][W]
    int *live = reinterpret_cast<int *>(mall + a.T * a.W);                      // [G]
    uint64_t *full = reinterpret_cast<uint64_t *>(
        (reinterpret_cast<uintptr_t>(live + a.G) + 7) & ~(uintptr_t)7);
    uint64_t *empty = full + NS;
    __shared__ int s_nlive, s_err;

    const int tid = (int)threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ri = (int)blockIdx.x / a.TG, tb = (int)blockIdx.x % a.TG;
    const int t0 = tb * kFTok;
    const int bt = min(a.T - t0, TB);                // tokens of this CTA (>= 1)
    const int H = a.H, gs = a.gs, W = a.W;

    // ---- the mask (one round trip), then the batch's union as a list
    for (int i = tid; i < a.T * W; i += kFThreads)
        mall[i] = a.mask[i];
    if (tid == 0) {
        s_err = 0;
        for (int i = 0; i < NS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kFWarps);
        }
        fence_mbar_init();
        tma_prefetch_desc(&tm_gate);
        tma_prefetch_desc(&tm_up);
        tma_prefetch_desc(&tm_down);
        tma_prefetch_desc(&tm_h);
    }
    __syncthreads();
    if (warp == 0) {
        uint32_t u = 0;
        bool bad = false;
        if (lane < W) {
            for (int t = 0; t < a.T; ++t)
                u |= mall[t * W + lane];
            const int left = a.G - lane * 32;
            const uint32_t valid = left >= 32 ? 0xffffffffu : ((1u << left) - 1u);
            bad = (u & ~valid) != 0u;
            u &= valid;
        }
        const int pc = __popc(u);
        int base = pc;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, base, off);
            if (lane >= off)
                base += v;
        }
        const int total = __shfl_sync(0xffffffffu, base, 31);
        base -= pc;
        for (uint32_t m = u; m; m &= m - 1u)
            live[base++] = lane * 32 + __ffs(m) - 1;
        if (__any_sync(0xffffffffu, bad) && lane == 0)
            set_status(a.status, WIDE_DEV_BAD_MASK);
        if (lane == 0)
            s_nlive = total;
    }
    __syncthreads();

    const int n_live = s_nlive;
    const int KW = a.kw, nks = KW / 128, NUS = kFStageCols / KW;
    const int N8 = n_live * gs / 8;                      // union rows in units of 8
    const int u0 = (int)((int64_t)ri * N8 / a.P), u1 = (int)((int64_t)(ri + 1) * N8 / a.P);
    const int nRB = (u1 - u0 + NUS - 1) / NUS;           // phase-1 row blocks
    const int NKW = H / KW;
    const int n1 = nRB * NKW;
    const int j0 = (int)((int64_t)ri * H / a.P), j1 = (int)((int64_t)(ri + 1) * H / a.P);
    const int n2rows = j1 - j0;
    const int n2s = n2rows > 0 ? (n_live + a.ng2 - 1) / a.ng2 : 0;
    const int total = n1 + n2s;
    const uint32_t box1 = 8u * (uint32_t)KW * 2u;        // one 8-row unit of one matrix

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            bool passed = false, err = false;
            int hnext = n1;   // first phase-2 stage whose h tiles are not issued yet
            auto issue_h = [&](int k) {
                const int s2 = k - n1, slot = k % NS;
                uint8_t *sb = slots + (size_t)slot * a.slot_bytes + a.h2_off;
                const int gb = s2 * a.ng2, ge = min(n_live, gb + a.ng2);
                for (int i = gb; i < ge; ++i)
                    tma_load_2d(sb + (size_t)(i - gb) * a.h2_bytes, &tm_h, live[i] * gs, t0,
                                &full[slot]);
            };
            auto grid_done = [&]() {
                if (!passed && ld_acquire_gpu(a.bar) >= gridDim.x) {
                    passed = true;
                    fence_proxy_async_global();
                }
                return passed;
            };
            for (int k = 0; k < total && !err; ++k) {
                const int slot = k % NS;
                if (k >= NS) {
                    const uint32_t par = (uint32_t)(k / NS - 1) & 1u;
                    const uint64_t tw = globaltimer();
                    for (uint32_t it = 0;; ++it) {
                        if (mbar_try_wait(&empty[slot], par))
                            break;
                        if (k > n1 && hnext < k && grid_done())
                            for (; hnext < k; ++hnext)
                                issue_h(hnext);
                        if ((it & 255u) == 255u && globaltimer() - tw > kWaitLimitNs) {
                            err = true;
                            break;
                        }
                    }
                    if (err)
                        break;
                }
                uint8_t *sb = slots + (size_t)slot * a.slot_bytes;
                if (k < n1) {
                    const int rb = k / NKW, kw = k % NKW;
                    const int ub = u0 + rb * NUS, nu = min(NUS, u1 - ub);
                    mbar_arrive_expect_tx(&full[slot], 2u * (uint32_t)nu * box1);
                    for (int i = 0; i < nu; ++i) {
                        const int lr = (ub + i) * 8;
                        const int grow = live[lr / gs] * gs + lr % gs;
                        tma_load_3d(sb + (size_t)i * box1, &tm_gate, 0, kw * (KW / 64), grow,
                                    &full[slot]);
                        tma_load_3d(sb + kFSlotMin / 2 + (size_t)i * box1, &tm_up, 0,
                                    kw * (KW / 64), grow, &full[slot]);
                    }
                } else {
                    const int s2 = k - n1;
                    const int gb = s2 * a.ng2, ge = min(n_live, gb + a.ng2);
                    mbar_arrive_expect_tx(&full[slot],
                                          (uint32_t)(ge - gb) * (a.w2_bytes + a.h2_bytes));
                    for (int i = gb; i < ge; ++i)
                        tma_load_2d(sb + (size_t)(i - gb) * a.w2_bytes, &tm_down, live[i] * gs,
                                    j0, &full[slot]);
                    if (hnext == k && passed) {   // no poll here: the waits above poll
                        issue_h(k);
                        ++hnext;
                    }
                }
            }
            // h tiles still waiting for the grid barrier
            if (!err && hnext < total) {
                const uint64_t tw = globaltimer();
                for (uint32_t it = 0; !grid_done(); ++it) {
                    if ((it & 255u) == 255u && globaltimer() - tw > kWaitLimitNs) {
                        err = true;
                        break;
                    }
                }
                if (passed)
                    for (; hnext < total; ++hnext)
                        issue_h(hnext);
            }
            if (err) {
                set_status(a.status, WIDE_DEV_TIMEOUT);
                atomicExch(&s_err, 1);
            }
        }
    } else {
        // ------------------------------------------------ consumers
        const int ct = tid - 32, cw = ct >> 5;
        const int r = lane >> 3;                // row of 4 in the warp
        const int c = lane & 7, sw = (c >> 2) & 1;
        bool ok = true;
        auto wait_full = [&](int k) {
            if (ok && !mbar_wait(&full[k % NS], (uint32_t)(k / NS) & 1u)) {
                ok = false;
                set_status(a.status, WIDE_DEV_TIMEOUT);
                atomicExch(&s_err, 1);
            }
        };
        auto release = [&](int k) {
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&empty[k % NS]);
        };

        // x of this CTA's tokens, fp32 (rows bt..TB-1 zero)
        if (a.xf) {
            // RMSNorm fused: warp cw normalises token cw (bf16-rounded, as a
            // bf16 layer feeds its FFN)
            for (int t = cw; t < TB; t += kFWarps) {
                float *xr = xs + (size_t)t * H;
                if (t >= bt) {
                    for (int k = lane * 4; k < H; k += 128)
                        *reinterpret_cast<float4 *>(xr + k) = make_float4(0.f, 0.f, 0.f, 0.f);
                    continue;
                }
                const float *src = a.xf + (size_t)(t0 + t) * H;
                float ss = 0.f;
                for (int k = lane * 4; k < H; k += 128) {
                    const float4 v = *reinterpret_cast<const float4 *>(src + k);
                    ss = fmaf(v.x, v.x, ss);
                    ss = fmaf(v.y, v.y, ss);
                    ss = fmaf(v.z, v.z, ss);
                    ss = fmaf(v.w, v.w, ss);
                }
                for (int off = 16; off; off >>= 1)
                    ss += __shfl_xor_sync(0xffffffffu, ss, off);
                const float rn = 1.0f / sqrtf(ss / (float)H + a.eps);
                for (int k = lane * 4; k < H; k += 128) {
                    const float4 v = *reinterpret_cast<const float4 *>(src + k);
                    const uint2 gw = *reinterpret_cast<const uint2 *>(a.gamma + k);
                    float4 y;
                    y.x = __bfloat162float(__float2bfloat16_rn(
                        v.x * rn * __uint_as_float(gw.x << 16)));
                    y.y = __bfloat162float(__float2bfloat16_rn(
                        v.y * rn * __uint_as_float(gw.x & 0xffff0000u)));
                    y.z = __bfloat162float(__float2bfloat16_rn(
                        v.z * rn * __uint_as_float(gw.y << 16)));
                    y.w = __bfloat162float(__float2bfloat16_rn(
                        v.w * rn * __uint_as_float(gw.y & 0xffff0000u)));
                    *reinterpret_cast<float4 *>(xr + k) = y;
                }
            }
        } else {
            // all loads of a batch go out before any is used
            constexpr int kB = 8;
            const int cpr = H / 8, n = TB * cpr;
            for (int i0 = ct; i0 < n; i0 += 32 * kFWarps * kB) {
                uint4 v[kB];
#pragma unroll
                for (int u = 0; u < kB; ++u) {
                    const int i = i0 + u * 32 * kFWarps;
                    const int t = i / cpr, q = i % cpr;
                    v[u] = (i < n && t < bt) ? *reinterpret_cast<const uint4 *>(
                                                   a.x + (size_t)(t0 + t) * H + q * 8)
                                             : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int u = 0; u < kB; ++u) {
                    const int i = i0 + u * 32 * kFWarps;
                    if (i < n) {
                        const int t = i / cpr, q = i % cpr;
                        float f[8];
                        bf16x8_to_f32(v[u], f);
                        float *d = xs + (size_t)t * H + q * 8;
                        *reinterpret_cast<float4 *>(d) = make_float4(f[0], f[1], f[2], f[3]);
                        *reinterpret_cast<float4 *>(d + 4) = make_float4(f[4], f[5], f[6], f[7]);
                    }
                }
            }
        }
        consumer_sync();

        // ---- phase 1
        // warp cw: row (cw & 1) * 4 + r of unit ui, 128-column pieces ks, ks+1
        const int pw = cw >> 1;                    // piece pair 0..3
        const int ui = (2 * pw) / nks, ks = (2 * pw) % nks;
        const int row = (cw & 1) * 4 + r;
        const int nps = nks / 2;                   // piece pairs per unit
        const uint32_t rs = (uint32_t)KW * 2u;     // row stride of a unit in the slot
        const uint8_t *xbase = reinterpret_cast<const uint8_t *>(xs) + ks * 512;
        int k = 0;
        for (int rb = 0; rb < nRB; ++rb) {
            const int ub = u0 + rb * NUS, nu = min(NUS, u1 - ub);
            float2 ag[TB], au[TB];
#pragma unroll
            for (int t = 0; t < TB; ++t) {
                ag[t] = make_float2(0.f, 0.f);
                au[t] = make_float2(0.f, 0.f);
            }
            for (int kw = 0; kw < NKW; ++kw, ++k) {
                wait_full(k);
                if (ui < nu) {
                    const uint8_t *sg = slots + (size_t)(k % NS) * a.slot_bytes +
                                        (size_t)ui * box1 + ks * 256;
                    p1_stage<TB>(sg, sg + kFSlotMin / 2, xbase + (size_t)kw * KW * 4, H, rs, row,
                                 c, sw, ag, au);
                }
                release(k);
            }
            // lane sums, then the piece pairs of a unit through shared memory
            float *rd = red + (rb & 1) * (4 * 8 * 2 * TB);
#pragma unroll
            for (int t = 0; t < TB; ++t) {
                const float g = sum8(ag[t].x + ag[t].y);
                const float u = sum8(au[t].x + au[t].y);
                if (c == (t & 7)) {
                    float *e = rd + ((pw * 8 + row) * 2) * TB + t;
                    e[0] = g;
                    e[TB] = u;
                }
            }
            consumer_sync();
            for (int i = ct; i < nu * 8 * TB; i += 32 * kFWarps) {
                const int un = i / (8 * TB), rrow = (i / TB) % 8, t = i % TB;
                float g = 0.f, u = 0.f;
                for (int s = 0; s < nps; ++s) {
                    const float *e = rd + (((un * nps + s) * 8 + rrow) * 2) * TB + t;
                    g += e[0];
                    u += e[TB];
                }
                if (t < bt) {
                    const int lr = (ub + un) * 8 + rrow;
                    const int grp = live[lr / gs];
                    const bool keep = (mall[(t0 + t) * W + (grp >> 5)] >> (grp & 31)) & 1u;
                    a.h[(size_t)(t0 + t) * a.I + grp * gs + lr % gs] =
                        keep ? silu_f32(g) * u : 0.f;
                }
            }
        }

        // ---- grid barrier (arrive); the producer waits for it
        fence_proxy_async_global();
        consumer_sync();
        if (ct == 0) {
            __threadfence();
            red_add_release_gpu(a.bar, 1u);
        }

        // ---- phase 2
        if (n2rows > 0) {
            const int R2 = (n2rows + 31) / 32;
            const int rw = cw * 4 + r;             // rows rw + 32 k
            const int rmax = n2rows - 1;
            float2 acc[kFMaxR2][TB];
#pragma unroll
            for (int rr = 0; rr < kFMaxR2; ++rr)
#pragma unroll
                for (int t = 0; t < TB; ++t)
                    acc[rr][t] = make_float2(0.f, 0.f);
            for (int s2 = 0; s2 < n2s; ++s2, ++k) {
                wait_full(k);
                const uint8_t *sb = slots + (size_t)(k % NS) * a.slot_bytes;
                const int gb = s2 * a.ng2, ge = min(n_live, gb + a.ng2);
                for (int i = 0; i < ge - gb; ++i) {
                    const uint8_t *wb = sb + (size_t)i * a.w2_bytes;
                    const uint8_t *hb = sb + a.h2_off + (size_t)i * a.h2_bytes;
                    if (R2 == 1)       // R2 <= kFMaxR2 = 3 (rows_box <= 96)
                        p2_group<TB, 1>(wb, hb, gs, rw, rmax, c, sw, acc);
                    else if (R2 == 2)
                        p2_group<TB, 2>(wb, hb, gs, rw, rmax, c, sw, acc);
                    else
                        p2_group<TB, 3>(wb, hb, gs, rw, rmax, c, sw, acc);
                }
                release(k);
            }
#pragma unroll
            for (int rr = 0; rr < kFMaxR2; ++rr) {
                if (rr >= R2)
                    break;
                const int row = rr * 32 + rw;
#pragma unroll
                for (int t = 0; t < TB; ++t) {
                    const float v = sum8(acc[rr][t].x + acc[rr][t].y);
                    if (row < n2rows && c == (t & 7) && t < bt) {
                        const size_t at = (size_t)(t0 + t) * H + j0 + row;
                        const DownOutputs &o = a.o;
                        if (o.out_sum)
                            static_cast<__nv_bfloat16 *>(o.out_sum)[at] = __float2bfloat16_rn(v);
                        if (o.out_total || o.out_total_f32) {
                            float tot = v;
                            if (o.res_in)
                                tot += __bfloat162float(
                                    static_cast<const __nv_bfloat16 *>(o.res_in)[at]);
                            if (o.res_f32)
                                tot += o.res_f32[at];
                            if (o.out_total)
                                static_cast<__nv_bfloat16 *>(o.out_total)[at] =
                                    __float2bfloat16_rn(tot);
                            if (o.out_total_f32)
                                o.out_total_f32[at] = tot;
                        }
                    }
                }
            }
        }
    }

    // after an error, let this CTA's copies in flight land before exit
    __syncthreads();
    if (s_err && tid == 0) {
        for (int k = total - 1; k >= 0 && k >= total - NS; --k)
            mbar_wait(&full[k % NS], (uint32_t)(k / NS) & 1u);
    }
}

struct DevInfo {
    int sms = 0, optin = 0;
};

DevInfo dev_info()
{
    static std::mutex mu;
    static DevInfo info[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return DevInfo{};
    std::lock_guard<std::mutex> lock(mu);
    if (info[dev].sms == 0) {
        cudaDeviceGetAttribute(&info[dev].sms, cudaDevAttrMultiProcessorCount, dev);
        cudaDeviceGetAttribute(&info[dev].optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    }
    return info[dev];
}

int tok_block(int T) { return T <= 1 ? 1 : (T <= 2 ? 2 : (T <= 4 ? 4 : 8)); }

// Launch geometry of one call; false if the shape does not fit the kernel.
struct FusedPlan {
    int TB, TG, P, kw, rows_box, ng2, nslots;
    uint32_t slot_bytes, w2_bytes, h2_bytes, h2_off;
    size_t smem;
};

bool plan_fused(int T, int H, int I, int gs, FusedPlan *p)
{
    if (T < 1 || T > 32 || H % 256 != 0 || gs % 64 != 0 || gs > 256 || I % gs != 0)
        return false;
    const int G = I / gs, W = (G + 31) / 32;
    if (G > kFMaxG || T * W > kFMaxMaskWords)
        return false;
    const DevInfo di = dev_info();
    if (di.sms <= 0)
        return false;
    p->TB = tok_block(T);
    p->TG = (T + kFTok - 1) / kFTok;
    p->P = di.sms / p->TG;
    if (p->P < 1)
        return false;
    p->kw = kFStageCols;
    while (H % p->kw != 0)
        p->kw >>= 1;                              // 1024, 512 or 256 (two pieces per warp)
    p->rows_box = (H + p->P - 1) / p->P;
    if (p->rows_box > 32 * kFMaxR2)
        return false;
    p->w2_bytes = (uint32_t)p->rows_box * gs * 2u;
    p->h2_bytes = (uint32_t)p->TB * gs * 4u;
    const uint32_t per_group = p->w2_bytes + p->h2_bytes;
    p->ng2 = (int)(kFSlotMin / per_group);
    if (p->ng2 < 1)
        p->ng2 = 1;
    p->h2_off = (uint32_t)p->ng2 * p->w2_bytes;
    uint32_t slot = (uint32_t)p->ng2 * per_group;
    if (slot < kFSlotMin)
        slot = kFSlotMin;
    p->slot_bytes = (slot + 1023u) & ~1023u;
    const size_t fixed = 1024 + (size_t)p->TB * H * 4 + (size_t)2 * 4 * 8 * 2 * p->TB * 4 +
                         (size_t)T * W * 4 + (size_t)G * 4 + 8 + 2 * kFMaxSlots * 8;
    if ((size_t)di.optin <= fixed + 64)
        return false;
    int ns = (int)(((size_t)di.optin - fixed - 64) / p->slot_bytes);
    if (ns > kFMaxSlots)
        ns = kFMaxSlots;
    if (ns < 2)
        return false;
    p->nslots = ns;
    p->smem = fixed + (size_t)ns * p->slot_bytes;
    return true;
}

template <int TB>
int launch_fused(const FusedPlan &pl, const CUtensorMap &tg, const CUtensorMap &tu,
                 const CUtensorMap &td, const CUtensorMap &th, const FusedArgs &a,
                 cudaStream_t s)
{
    auto kernel = ffn_decode_fused<TB>;
    if (!raise_smem_limit(reinterpret_cast<const void *>(kernel), pl.smem))
        return WIDE_CUDA_FAIL();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.P * pl.TG);
    cfg.blockDim = dim3(kFThreads);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    LaunchScope scope(KID_DECODE_FFN_FUSED, s);
    if (cudaLaunchKernelEx(&cfg, kernel, tg, tu, td, th, a) != cudaSuccess)
        return WIDE_CUDA_FAIL();
    return WIDE_OK;
}

}  // namespace

bool decode_ffn_fused_supported(int T, int H, int I, int gs)
{
    FusedPlan p;
    return plan_fused(T, H, I, gs, &p);
}

// Measured on B200 (3B FFN, 50% keep): the fused kernel beats the two GEMV
// kernels of ffn_decode.cu for up to 8 tokens per call (one token block);
// for more tokens the extra h traffic of its phase 2 makes it slower.
bool decode_ffn_fused_preferred(int T, int H, int I, int gs)
{
    return T <= kFTok && decode_ffn_fused_supported(T, H, I, gs);
}

int decode_ffn_fused(const FusedInput &in, const DownOutputs &o, int T, int H, int I, int gs,
                     float *h, uint32_t *bar, cudaStream_t s)
{
    FusedPlan pl;
    if (!plan_fused(T, H, I, gs, &pl))
        return WIDE_EUNSUPPORTED;
    const int G = I / gs;
    CUtensorMap tg, tu, td, th;
    if (!make_tmap_rows3d(&tg, in.w_gate, I, H, H, pl.kw / 64, 8) ||
        !make_tmap_rows3d(&tu, in.w_up, I, H, H, pl.kw / 64, 8) ||
        !make_tmap_2d(&td, in.w_down, H, I, I, 2, pl.rows_box, gs, false) ||
        !make_tmap_2d(&th, h, T, I, I, 4, pl.TB, gs, false))
        return WIDE_CUDA_FAIL();
    FusedArgs a = {};
    a.x = static_cast<const __nv_bfloat16 *>(in.x);
    a.xf = in.x_f32;
    a.gamma = static_cast<const __nv_bfloat16 *>(in.gamma);
    a.eps = in.eps;
    a.mask = in.mask;
    a.h = h;
    a.bar = bar;
    a.o = o;
    a.T = T;
    a.H = H;
    a.I = I;
    a.G = G;
    a.W = (G + 31) / 32;
    a.gs = gs;
    a.TG = pl.TG;
    a.P = pl.P;
    a.kw = pl.kw;
    a.nslots = pl.nslots;
    a.slot_bytes = pl.slot_bytes;
    a.w2_bytes = pl.w2_bytes;
    a.h2_bytes = pl.h2_bytes;
    a.h2_off = pl.h2_off;
    a.ng2 = pl.ng2;
    a.status = status_ptr();
    if (cudaMemsetAsync(bar, 0, sizeof(uint32_t), s) != cudaSuccess)
        return WIDE_CUDA_FAIL();
    switch (pl.TB) {
    case 1: return launch_fused<1>(pl, tg, tu, td, th, a, s);
    case 2: return launch_fused<2>(pl, tg, tu, td, th, a, s);
    case 4: return launch_fused<4>(pl, tg, tu, td, th, a, s);
    default: return launch_fused<8>(pl, tg, tu, td, th, a, s);
    }
}

}  // namespace wide
