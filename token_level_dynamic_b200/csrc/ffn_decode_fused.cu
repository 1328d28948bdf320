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
//     units of 8 rows.  A stage holds SR rows of W_gate and of W_up over a
//     window of KW columns (16 x 512, or 32 x 256 when H is not a multiple
//     of 512), fetched as one 3-D TMA copy of 8 rows per unit and matrix:
//     long contiguous row pieces stream far better than 2-D boxes of short
//     rows.
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
// grid barrier; only their h tiles wait for the barrier.  Warps 1..16 compute
// in fp32 on CUDA cores with packed fp32x2 FMAs over token PAIRS: one
// register pair holds the running sums of tokens 2p and 2p+1, the x (or h)
// operand is the pair's two values of one column and the weight operand is
// that column's weight in both halves.  So a 16-byte weight chunk (8
// columns of one row) read from shared memory serves every token, and a
// 16-byte read of x serves 2 tokens x 2 columns of every row the thread
// holds.
//   Phase 1: a thread holds 2 rows of W_gate and the same 2 rows of W_up (4
//     weight rows) at one 8-column chunk of the window; the 8 lanes of a
//     quarter warp take 8 adjacent chunks of one row (128 contiguous bytes).
//     x is staged once as bf16 token pairs [pair][column][2], its two 16-byte
//     halves of a chunk swapped in every other group of 4 chunks, so the 8
//     lanes of a quarter warp read 8 distinct banks.  A warp's rows lie in
//     one group, so the token pairs in which neither token keeps it are
//     left out of its FMAs (their h is written as 0).  The partial sums are
//     added over the chunks of a row (lane shuffles that halve the values a
//     lane carries at every step, then shared memory between the two warps
//     of a row for 512-column windows) once per row block.
//   Phase 2: a thread holds up to 4 rows of the CTA's W_down range at one
//     8-column chunk of a group; several sets of whole warps ("instances")
//     take different groups, run ahead of one another as far as the ring
//     allows, and their sums meet in shared memory at the end.  h
//     is written by phase 1 as fp32 token pairs and copied per group by a
//     3-D TMA box with 128-byte swizzle, which leaves the 8 lanes of a
//     quarter warp reading 8 distinct banks.
#include "common.cuh"
#include "host.h"

#include <atomic>
#include <mutex>

namespace wide {
namespace {

constexpr int kFTok = 8;                    // tokens per CTA (one token block)
constexpr int kFWarps = 16;                 // consumer warps
constexpr int kFCons = 32 * kFWarps;        // consumer threads
constexpr int kFThreads = kFCons + 32;
constexpr int kFStageElems = 8192;          // phase 1: rows x window columns per stage
constexpr uint32_t kFSlotMin = 2u * kFStageElems * 2u;   // gate + up: 32 KB
constexpr int kFMaxSlots = 8;
constexpr int kFMaxG = 1024;                // groups (union words fit one warp)
constexpr int kFMaxRT = 4;                  // phase 2: rows per thread
constexpr int kFRedFloats = 2048;           // cross-warp / cross-instance sums
constexpr int kFMaxMaskWords = 1024;        // T * W

struct FusedArgs {
    const __nv_bfloat16 *x;      // [T][H] FFN input (null when xf is given)
    const float *xf;             // [T][H] fp32 rows normalised in the kernel, or null
    const __nv_bfloat16 *gamma;  // RMSNorm gain used with xf
    float eps;
    const uint32_t *mask;        // [T][W] packed group bits
    float *h;                    // [T][I] fp32 scratch, token pairs interleaved
    uint32_t *bar;               // grid barrier arrival counter (0 at launch)
    DownOutputs o;
    int T, H, I, W, G, gs;
    int TG, P;                   // token blocks; row ranges (grid = P * TG)
    int kw;                      // phase-1 window columns (512 or 256)
    int rt, nr, ni;              // phase 2: rows per thread, row sets, instances
    int nslots;
    uint32_t slot_bytes;
    uint32_t w2_bytes;           // one W_down box (rows_box rows x gs columns)
    uint32_t h2_bytes;           // one h box (token pairs x gs columns, fp32)
    uint32_t h2_stride;          // h boxes' spacing in a slot (1024-byte multiple)
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

// The two float pairs of one float4.
__device__ __forceinline__ float2 lo2(const float4 v) { return make_float2(v.x, v.y); }
__device__ __forceinline__ float2 hi2(const float4 v) { return make_float2(v.z, v.w); }

__device__ __forceinline__ void fence_proxy_async_global()
{
    asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ void consumer_sync()
{
    asm volatile("bar.sync 1, %0;" ::"n"(kFCons) : "memory");
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

// Halving steps of lane_reduce: as many as the lanes allow while KEEP values
// are left per lane.
__host__ __device__ constexpr int scatter_levels(int ratio, int lv)
{
    int s = 0;
    while (s < lv && (2 << s) <= ratio)
        ++s;
    return s;
}

// Sums v[0..N) over the 2^LV lanes that differ in lane bits [0, LV).  The
// first S = scatter_levels(N / KEEP, LV) steps halve what a lane carries
// (a lane keeps the half its bit selects and receives its partner's copy of
// it), the remaining LV - S steps add whole arrays.  Afterwards lane l holds
// in v[0..N >> S) the sums of entries
//   m = ((l >> (LV - S)) & (2^S - 1)) * (N >> S) + j.
template <int N, int LV, int KEEP>
__device__ __forceinline__ void lane_reduce(float (&v)[N], int lane)
{
    constexpr int S = scatter_levels(N / KEEP, LV);
#pragma unroll
    for (int l = 0; l < S; ++l) {
        const int o = 1 << (LV - 1 - l);
        const bool hi = (lane & o) != 0;
        const int n = N >> (l + 1);
#pragma unroll
        for (int i = 0; i < N / 2; ++i) {
            if (i < n) {
                const float send = hi ? v[i] : v[i + n];
                const float keep = hi ? v[i + n] : v[i];
                v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
        }
    }
    constexpr int R = N >> S;
#pragma unroll
    for (int l = S; l < LV; ++l) {
        const int o = 1 << (LV - 1 - l);
#pragma unroll
        for (int i = 0; i < R; ++i)
            v[i] += __shfl_xor_sync(0xffffffffu, v[i], o);
    }
}

// Phase 1, one stage, one thread: rows 0 and 1 of W_gate at sg and of W_up
// at su (row stride rs bytes), one 8-column chunk; the x half holding the
// chunk's columns 4 h .. 4 h + 3 of token pair p at xk + p * xpair + xo[h].
// Only the first NA accumulator slots are computed: slot k holds token pair
// (ppk >> 4k) & 15, the pairs with a token that keeps the unit's group.
template <int NP, int NA>
__device__ __forceinline__ void p1_stage(const uint8_t *sg, const uint8_t *su, uint32_t rs,
                                         const uint8_t *xk, uint32_t xpair, const uint32_t (&xo)[2],
                                         uint32_t ppk, float2 (&ag)[2][NP], float2 (&au)[2][NP])
{
    uint4 g[2], u[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        g[i] = lds128(sg + i * rs);
        u[i] = lds128(su + i * rs);
    }
#pragma unroll
    for (int p2 = 0; p2 < 2; ++p2) {             // columns 4 p2 .. 4 p2 + 3 of the chunk
        uint4 xr[NA];
#pragma unroll
        for (int tp = 0; tp < NA; ++tp)
            xr[tp] = lds128(xk + ((ppk >> (4 * tp)) & 15u) * xpair + xo[p2]);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
            float2 xv[NA];
#pragma unroll
            for (int tp = 0; tp < NA; ++tp) {
                const uint32_t wx = word(xr[tp], cc);
                xv[tp] = make_float2(bf_lo(wx), bf_hi(wx));
            }
            const int wi = 2 * p2 + (cc >> 1);    // weight word of column 4 p2 + cc
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const float2 d = (cc & 1) ? dup_hi(word(g[i], wi)) : dup_lo(word(g[i], wi));
#pragma unroll
                for (int tp = 0; tp < NA; ++tp)
                    ag[i][tp] = __ffma2_rn(d, xv[tp], ag[i][tp]);
            }
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const float2 d = (cc & 1) ? dup_hi(word(u[i], wi)) : dup_lo(word(u[i], wi));
#pragma unroll
                for (int tp = 0; tp < NA; ++tp)
                    au[i][tp] = __ffma2_rn(d, xv[tp], au[i][tp]);
            }
        }
    }
}

// p1_stage for the run-time number of active slots na (1 <= na <= NP).
template <int NP>
__device__ __forceinline__ void p1_dispatch(int na, const uint8_t *sg, const uint8_t *su,
                                            uint32_t rs, const uint8_t *xk, uint32_t xpair,
                                            const uint32_t (&xo)[2], uint32_t ppk,
                                            float2 (&ag)[2][NP], float2 (&au)[2][NP])
{
    constexpr int N2 = NP < 2 ? NP : 2, N3 = NP < 3 ? NP : 3;
    if (na >= NP)
        p1_stage<NP, NP>(sg, su, rs, xk, xpair, xo, ppk, ag, au);
    else if (na == 1)
        p1_stage<NP, 1>(sg, su, rs, xk, xpair, xo, ppk, ag, au);
    else if (na == 2)
        p1_stage<NP, N2>(sg, su, rs, xk, xpair, xo, ppk, ag, au);
    else if (na == 3)
        p1_stage<NP, N3>(sg, su, rs, xk, xpair, xo, ppk, ag, au);
}

// Phase 2, one group: this thread's rows of the W_down box at wb (row k at
// wb + min(wbase + k wrs, wmax), k < RT) and the group's h box at hb, whose 16-byte unit
// holding columns 2p, 2p+1 of this thread's chunk for token pair tp sits at
// hb + (hoff[tp] ^ 16 p) (128-byte swizzle: the unit index within its
// 128-byte row is XOR-ed with the row index).
template <int NP, int RT>
__device__ __forceinline__ void p2_group(const uint8_t *wb, uint32_t wbase, uint32_t wrs,
                                         uint32_t wmax, const uint8_t *hb,
                                         const uint32_t (&hoff)[NP], float2 (&acc)[kFMaxRT][NP])
{
    uint4 w[RT];
#pragma unroll
    for (int k = 0; k < RT; ++k)
        w[k] = lds128(wb + min(wbase + (uint32_t)k * wrs, wmax));
#pragma unroll
    for (int p = 0; p < 4; ++p) {                 // columns 2p, 2p+1 of the chunk
        float4 hx[NP];
#pragma unroll
        for (int tp = 0; tp < NP; ++tp)
            hx[tp] = lds128f(hb + (hoff[tp] ^ (uint32_t)(p << 4)));
#pragma unroll
        for (int e = 0; e < 2; ++e)
#pragma unroll
            for (int k = 0; k < RT; ++k) {
                const float2 d = e ? dup_hi(word(w[k], p)) : dup_lo(word(w[k], p));
#pragma unroll
                for (int tp = 0; tp < NP; ++tp)
                    acc[k][tp] = __ffma2_rn(d, e ? hi2(hx[tp]) : lo2(hx[tp]), acc[k][tp]);
            }
    }
}

// Phase 2's sums over the chunk lanes of a row set (2^LV = gs / 8 lanes),
// written to red2[instance][row][token] (one writer per value).
template <int NP, int LV>
__device__ __forceinline__ void p2_reduce(float2 (&acc)[kFMaxRT][NP], int ch2, bool act, int gi,
                                          int row0, int rt, int n2rows, int rstride, float *red2)
{
    constexpr int TBP = 2 * NP, N = kFMaxRT * TBP;
    float v[N];
#pragma unroll
    for (int k = 0; k < kFMaxRT; ++k)
#pragma unroll
        for (int tp = 0; tp < NP; ++tp) {
            v[k * TBP + 2 * tp] = acc[k][tp].x;
            v[k * TBP + 2 * tp + 1] = acc[k][tp].y;
        }
    lane_reduce<N, LV, 1>(v, ch2);
    constexpr int S = scatter_levels(N, LV), R = N >> S;
    const bool owner = (ch2 & ((1 << (LV - S)) - 1)) == 0;
    const int mb = ((ch2 >> (LV - S)) & ((1 << S) - 1)) * R;
#pragma unroll
    for (int j = 0; j < R; ++j) {
        const int m = mb + j, k = m / TBP, t = m % TBP, row = row0 + k;
        if (act && owner && k < rt && row < n2rows)
            red2[((size_t)gi * rstride + row) * TBP + t] = v[j];
    }
}

// One CTA of 17 warps per SM.  The register file is split between the SM's
// four sub-partitions and one of them holds 5 of the 17 warps, so a thread
// gets at most 16384 / 160 registers, 96 in the allocation granularity.
template <int TB>
__global__ void __maxnreg__(96)
    ffn_decode_fused(const __grid_constant__ CUtensorMap tm_gate,
                     const __grid_constant__ CUtensorMap tm_up,
                     const __grid_constant__ CUtensorMap tm_down,
                     const __grid_constant__ CUtensorMap tm_h, const FusedArgs a)
{
    constexpr int TBP = TB < 2 ? 2 : TB;             // tokens rounded up to whole pairs
    constexpr int NP = TBP / 2;                      // token pairs
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    const int NS = a.nslots;
    uint8_t *slots = smem;
    // x as bf16 token pairs: [NP][H / 8 chunks][2 halves][4 columns][2 tokens]
    uint8_t *xs = smem + (size_t)NS * a.slot_bytes;
    float *red = reinterpret_cast<float *>(xs + (size_t)TBP * a.H * 2);
    uint32_t *mall = reinterpret_cast<uint32_t *>(red + kFRedFloats);   // [T][W]
    int *live = reinterpret_cast<int *>(mall + a.T * a.W);                      // [G]
    uint64_t *full = reinterpret_cast<uint64_t *>(
        (reinterpret_cast<uintptr_t>(live + a.G) + 7) & ~(uintptr_t)7);
    uint64_t *empty = full + NS;
    __shared__ int s_nlive, s_err;
    __shared__ float s_rn[kFTok];

    const int tid = (int)threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ri = (int)blockIdx.x / a.TG, tb = (int)blockIdx.x % a.TG;
    const int t0 = tb * kFTok;
    const int bt = min(a.T - t0, TB);                // tokens of this CTA (>= 1)
    const int H = a.H, gs = a.gs, W = a.W;

    // ---- x of this CTA's tokens toward L2 (the staging below needs the
    // union first; its loads then find x in L2), the mask (one round trip),
    // then the batch's union as a list
    if (!a.xf && tid >= 32) {
        const char *xb = reinterpret_cast<const char *>(a.x + (size_t)t0 * H);
        for (int i = tid - 32; i < bt * H * 2 / 128; i += kFCons)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(xb + (size_t)i * 128));
    }
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
    const int KW = a.kw, NUS = kFStageElems / 8 / KW;   // 8-row units per stage
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
                    tma_load_3d(sb + (size_t)(i - gb) * a.h2_stride, &tm_h, 0, live[i] * gs / 16,
                                t0 / 2, &full[slot]);
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
        bool ok = true;
        // ring position: slot index, its phase parity and its base address
        int slot = 0;
        uint32_t par = 0;
        const uint8_t *sp = slots;
        const uint32_t slot_bytes = a.slot_bytes;
        auto wait_full = [&]() {
            if (ok && !mbar_wait(&full[slot], par)) {
                ok = false;
                set_status(a.status, WIDE_DEV_TIMEOUT);
                atomicExch(&s_err, 1);
            }
        };
        auto release = [&]() {
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&empty[slot]);
            sp += slot_bytes;
            if (++slot == NS) {
                slot = 0;
                par ^= 1u;
                sp = slots;
            }
        };

        // ---- x of this CTA's tokens as bf16 token pairs (tokens bt.. zero)
        if (a.xf) {
            // RMSNorm fused: warp cw finds 1 / rms of token cw; the values
            // are rounded to bf16, as a bf16 layer feeds its FFN
            for (int t = cw; t < bt; t += kFWarps) {
                const float *src = a.xf + (size_t)(t0 + t) * H;
                float ss = 0.f;
#pragma unroll 8
                for (int k = lane * 4; k < H; k += 128) {
                    const float4 v = *reinterpret_cast<const float4 *>(src + k);
                    ss = fmaf(v.x, v.x, ss);
                    ss = fmaf(v.y, v.y, ss);
                    ss = fmaf(v.z, v.z, ss);
                    ss = fmaf(v.w, v.w, ss);
                }
                for (int off = 16; off; off >>= 1)
                    ss += __shfl_xor_sync(0xffffffffu, ss, off);
                if (lane == 0)
                    s_rn[t] = 1.0f / sqrtf(ss / (float)H + a.eps);
            }
            consumer_sync();
        }
        {
            // one 16-byte unit per step: 4 columns of one token pair; the
            // global loads of kXB steps go out before any is used
            constexpr int kXB = 8;
            const int nu4 = H / 4, n = NP * nu4;
            for (int i0 = ct; i0 < n; i0 += kFCons * kXB) {
                uint2 v2[kXB][2];
#pragma unroll
                for (int q = 0; q < kXB; ++q) {
                    const int i = i0 + q * kFCons;
                    const int tp = i / nu4, u4 = i % nu4;
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int t = 2 * tp + e;
                        v2[q][e] = make_uint2(0u, 0u);
                        if (i >= n || t >= bt)
                            continue;
                        if (a.xf) {
                            const float4 v = *reinterpret_cast<const float4 *>(
                                a.xf + (size_t)(t0 + t) * H + 4 * u4);
                            const uint2 gw = *reinterpret_cast<const uint2 *>(a.gamma + 4 * u4);
                            const float rn = s_rn[t];
                            const __nv_bfloat162 p0 = __floats2bfloat162_rn(
                                v.x * rn * bf_lo(gw.x), v.y * rn * bf_hi(gw.x));
                            const __nv_bfloat162 p1 = __floats2bfloat162_rn(
                                v.z * rn * bf_lo(gw.y), v.w * rn * bf_hi(gw.y));
                            v2[q][e].x = *reinterpret_cast<const uint32_t *>(&p0);
                            v2[q][e].y = *reinterpret_cast<const uint32_t *>(&p1);
                        } else {
                            v2[q][e] = *reinterpret_cast<const uint2 *>(
                                a.x + (size_t)(t0 + t) * H + 4 * u4);
                        }
                    }
                }
#pragma unroll
                for (int q = 0; q < kXB; ++q) {
                    const int i = i0 + q * kFCons;
                    if (i >= n)
                        break;
                    const int tp = i / nu4, u4 = i % nu4;
                    uint4 o;
                    o.x = __byte_perm(v2[q][0].x, v2[q][1].x, 0x5410);
                    o.y = __byte_perm(v2[q][0].x, v2[q][1].x, 0x7632);
                    o.z = __byte_perm(v2[q][0].y, v2[q][1].y, 0x5410);
                    o.w = __byte_perm(v2[q][0].y, v2[q][1].y, 0x7632);
                    *reinterpret_cast<uint4 *>(xs + (size_t)tp * H * 4 + (u4 >> 1) * 32 +
                                               (((u4 & 1) ^ ((u4 >> 3) & 1)) << 4)) = o;
                }
            }
        }
        consumer_sync();

        // ---- phase 1
        // thread: row set rsi (rows 2 rsi, 2 rsi + 1 of a stage), chunk ch
        const int CPR = KW / 8, NWR = CPR / 32;         // chunks per row, warps per row
        const int rsi = ct / CPR, ch = ct % CPR;
        const uint32_t rs = (uint32_t)KW * 2u;           // row stride in the slot
        const uint32_t wofs = (uint32_t)rsi * 2u * rs + (uint32_t)ch * 16u;
        const uint32_t swb = ((uint32_t)ch >> 2) & 1u;
        const uint32_t xo[2] = {(uint32_t)ch * 32u + (swb << 4), (uint32_t)ch * 32u + ((swb ^ 1u) << 4)};
        const uint32_t xpair = (uint32_t)H * 4u, xwin = (uint32_t)KW * 4u;
        constexpr int S1 = scatter_levels(2 * TBP, 5);   // (gate, up) of one (row, token) left
        float2 *red1 = reinterpret_cast<float2 *>(red);  // [2][8 row sets][32 lanes]
        for (int rb = 0; rb < nRB; ++rb) {
            const int ub = u0 + rb * NUS, nu = min(NUS, u1 - ub);
            const bool act = (rsi >> 2) < nu;
            // token pairs with a token that keeps this unit's group first
            // (4 bits per slot in ppk), na of them; the rest are skipped
            uint32_t ppk = 0u;
            int na = 0;
            if (act) {
                const int grp0 = live[((ub + (rsi >> 2)) * 8) / gs];
                uint32_t dl = 0u;
                int nd = 0;
#pragma unroll
                for (int tp = 0; tp < NP; ++tp) {
                    bool k = false;
#pragma unroll
                    for (int e = 0; e < 2; ++e)
                        if (2 * tp + e < bt)
                            k |= ((mall[(t0 + 2 * tp + e) * W + (grp0 >> 5)] >> (grp0 & 31)) & 1u) != 0u;
                    if (k)
                        ppk |= (uint32_t)tp << (4 * na++);
                    else
                        dl |= (uint32_t)tp << (4 * nd++);
                }
                ppk |= dl << (4 * na);
            }
            float2 ag[2][NP], au[2][NP];
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
                for (int tp = 0; tp < NP; ++tp) {
                    ag[i][tp] = make_float2(0.f, 0.f);
                    au[i][tp] = make_float2(0.f, 0.f);
                }
            const uint8_t *xk = xs;
            for (int kw = 0; kw < NKW; ++kw, xk += xwin) {
                wait_full();
                if (na > 0)
                    p1_dispatch<NP>(na, sp + wofs, sp + kFSlotMin / 2 + wofs, rs, xk, xpair, xo,
                                    ppk, ag, au);
                release();
            }
            // sums over the chunks of the row: lanes, then the warps of a row
            float v[4 * TBP];
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
                for (int tp = 0; tp < NP; ++tp) {
                    v[((i * TBP) + 2 * tp) * 2 + 0] = ag[i][tp].x;
                    v[((i * TBP) + 2 * tp) * 2 + 1] = au[i][tp].x;
                    v[((i * TBP) + 2 * tp + 1) * 2 + 0] = ag[i][tp].y;
                    v[((i * TBP) + 2 * tp + 1) * 2 + 1] = au[i][tp].y;
                }
            lane_reduce<4 * TBP, 5, 2>(v, lane);
            float g = v[0], u = v[1];
            if (NWR == 2) {
                float2 *r1 = red1 + (rb & 1) * 256 + rsi * 32 + lane;
                if (cw & 1)
                    *r1 = make_float2(g, u);
                consumer_sync();
                if (!(cw & 1)) {
                    const float2 o = *r1;
                    g += o.x;
                    u += o.y;
                }
            }
            const bool owner =
                (NWR == 1 || !(cw & 1)) && (lane & ((1 << (5 - S1)) - 1)) == 0;
            if (act && owner) {
                const int combo = lane >> (5 - S1);      // row * TBP + slot token
                const int r = combo / TBP, ts = combo % TBP;
                const int t = 2 * (int)((ppk >> (4 * (ts >> 1))) & 15u) + (ts & 1);
                if (t < bt) {
                    const int lr = ub * 8 + rsi * 2 + r;
                    const int grp = live[lr / gs];
                    const bool keep = (mall[(t0 + t) * W + (grp >> 5)] >> (grp & 31)) & 1u;
                    a.h[il2(t0 + t, (size_t)grp * gs + lr % gs, (size_t)a.I)] =
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
        // thread: instance gi (groups gi, gi + NI, ...), rows row0 .. row0 +
        // RT - 1 of the range, chunk ch2 of each group
        const int CPR2 = gs / 8, RT = a.rt, NR = a.nr, NI = a.ni, TPI = CPR2 * NR;
        const int gi = ct / TPI, rem = ct % TPI, ch2 = rem % CPR2;
        const int row0 = (rem / CPR2) * RT, rmax = n2rows - 1;
        const bool act2 = gi < NI;
        // this thread's offsets in a group's W_down box (rows past rmax read
        // row rmax; their sums are discarded) and h box
        const uint32_t wrs = (uint32_t)gs * 2u;
        const uint32_t wbase = (uint32_t)row0 * wrs + (uint32_t)ch2 * 16u;
        const uint32_t wmax = (uint32_t)rmax * wrs + (uint32_t)ch2 * 16u;
        uint32_t hoff[NP];
#pragma unroll
        for (int tp = 0; tp < NP; ++tp) {
            const uint32_t idx = (uint32_t)tp * ((uint32_t)gs / 2u) + (uint32_t)ch2 * 4u;
            const uint32_t r = idx >> 3;
            hoff[tp] = r * 128u + (((idx ^ r) & 7u) << 4);
        }
        float2 acc[kFMaxRT][NP];
#pragma unroll
        for (int r = 0; r < kFMaxRT; ++r)
#pragma unroll
            for (int tp = 0; tp < NP; ++tp)
                acc[r][tp] = make_float2(0.f, 0.f);
        const uint32_t w2b = a.w2_bytes, h2s = a.h2_stride, h2o = a.h2_off;
        int gnext = gi;                              // this instance's next union group
        for (int gb = 0; gb < n_live && n2rows > 0; gb += a.ng2) {
            const int ge = min(n_live, gb + a.ng2);
            wait_full();
            for (; act2 && gnext < ge; gnext += NI) {
                const uint8_t *wb = sp + (uint32_t)(gnext - gb) * w2b;
                const uint8_t *hb = sp + h2o + (uint32_t)(gnext - gb) * h2s;
                switch (RT) {      // 1 <= RT <= kFMaxRT
                case 4: p2_group<NP, 4>(wb, wbase, wrs, wmax, hb, hoff, acc); break;
                case 3: p2_group<NP, 3>(wb, wbase, wrs, wmax, hb, hoff, acc); break;
                case 2: p2_group<NP, 2>(wb, wbase, wrs, wmax, hb, hoff, acc); break;
                default: p2_group<NP, 1>(wb, wbase, wrs, wmax, hb, hoff, acc); break;
                }
            }
            release();
        }
        const int rstride = NR * RT;
        if (CPR2 == 8)
            p2_reduce<NP, 3>(acc, ch2, act2, gi, row0, RT, n2rows, rstride, red);
        else if (CPR2 == 16)
            p2_reduce<NP, 4>(acc, ch2, act2, gi, row0, RT, n2rows, rstride, red);
        else
            p2_reduce<NP, 5>(acc, ch2, act2, gi, row0, RT, n2rows, rstride, red);
        consumer_sync();
        for (int idx = ct; idx < n2rows * bt; idx += kFCons) {
            const int row = idx % n2rows, t = idx / n2rows;
            float v = 0.f;
            for (int q = 0; q < NI; ++q)
                v += red[((size_t)q * rstride + row) * TBP + t];
            const size_t at = (size_t)(t0 + t) * H + j0 + row;
            const DownOutputs &o = a.o;
            if (o.out_sum)
                static_cast<__nv_bfloat16 *>(o.out_sum)[at] = __float2bfloat16_rn(v);
            if (o.out_total || o.out_total_f32) {
                float tot = v;
                if (o.res_in)
                    tot += __bfloat162float(static_cast<const __nv_bfloat16 *>(o.res_in)[at]);
                if (o.res_f32)
                    tot += o.res_f32[at];
                if (o.out_total)
                    static_cast<__nv_bfloat16 *>(o.out_total)[at] = __float2bfloat16_rn(tot);
                if (o.out_total_f32)
                    o.out_total_f32[at] = tot;
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
    int TB, TG, P, kw, rows_box, rt, nr, ni, ng2, nslots;
    uint32_t slot_bytes, w2_bytes, h2_bytes, h2_stride, h2_off;
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
    const int TBP = p->TB < 2 ? 2 : p->TB;
    p->TG = (T + kFTok - 1) / kFTok;
    p->P = di.sms / p->TG;
    if (p->P < 1)
        return false;
    p->kw = H % 512 == 0 ? 512 : 256;
    p->rows_box = (H + p->P - 1) / p->P;
    // phase 2: NI = 512 / TPI instances of TPI threads (whole warps, so no
    // warp holds two instances that work on different groups), each NR =
    // TPI / (gs / 8) row sets of RT = ceil(rows / NR) <= 4 rows.  Time per
    // thread ~ (RT + 2) / NI (the 2: the h reads of a group, shared by its
    // rows).
    const int cpr2 = gs / 8;
    double best = 0.0;
    p->rt = 0;
    for (int tpi = 32; tpi <= kFCons; tpi *= 2) {
        const int nr = tpi / cpr2;
        const int rt = (p->rows_box + nr - 1) / nr;
        if (rt > kFMaxRT)
            continue;
        const int ni = kFCons / tpi;
        const double cost = (double)(rt + 2) / ni;
        if (p->rt == 0 || cost < best) {
            best = cost;
            p->rt = rt;
            p->nr = nr;
            p->ni = ni;
        }
    }
    if (p->rt == 0 || p->ni * p->nr * p->rt * TBP > kFRedFloats)
        return false;
    p->w2_bytes = (uint32_t)p->rows_box * gs * 2u;
    p->h2_bytes = (uint32_t)TBP * gs * 4u;
    p->h2_stride = (p->h2_bytes + 1023u) & ~1023u;    // 128-byte swizzle: 1024-aligned boxes
    const size_t fixed = 1024 + (size_t)TBP * H * 2 + (size_t)kFRedFloats * 4 +
                         (size_t)T * W * 4 + (size_t)G * 4 + 8 + 2 * kFMaxSlots * 8;
    if ((size_t)di.optin <= fixed + 64)
        return false;
    // ring slots for ng phase-2 groups per stage (at least a phase-1 stage)
    auto layout = [&](int ng, uint32_t *h2_off, uint32_t *slot_bytes) {
        *h2_off = ((uint32_t)ng * p->w2_bytes + 1023u) & ~1023u;
        uint32_t slot = *h2_off + (uint32_t)ng * p->h2_stride;
        if (slot < kFSlotMin)
            slot = kFSlotMin;
        *slot_bytes = (slot + 1023u) & ~1023u;
        const int ns = (int)(((size_t)di.optin - fixed - 64) / *slot_bytes);
        return ns > kFMaxSlots ? kFMaxSlots : ns;
    };
    p->ng2 = (int)(kFSlotMin / (p->w2_bytes + p->h2_stride));
    if (p->ng2 < 1)
        p->ng2 = 1;
    int ns = layout(p->ng2, &p->h2_off, &p->slot_bytes);
    if (p->ng2 == 1) {
        // two groups per phase-2 stage when the larger slots cost no slot
        uint32_t off2, sb2;
        const int ns2 = layout(2, &off2, &sb2);
        if (ns2 >= ns && ns2 >= 2) {
            p->ng2 = 2;
            p->h2_off = off2;
            p->slot_bytes = sb2;
            ns = ns2;
        }
    }
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

namespace {
std::atomic<int> g_decode_mode{WIDE_DECODE_AUTO};
}

// Measured on B200 (3B FFN at 50% keep and 8B FFN at 72% keep, 1..32
// tokens): the fused kernel beats the two GEMV kernels of ffn_decode.cu at
// every token count it supports (by 1-26%), so AUTO takes it wherever its
// shape limits allow.
bool decode_ffn_fused_preferred(int T, int H, int I, int gs)
{
    const int mode = g_decode_mode.load(std::memory_order_relaxed);
    if (mode == WIDE_DECODE_GEMV)
        return false;
    return decode_ffn_fused_supported(T, H, I, gs);
}

int wide_get_decode_ffn_path_mode() { return g_decode_mode.load(std::memory_order_relaxed); }

int decode_ffn_fused(const FusedInput &in, const DownOutputs &o, int T, int H, int I, int gs,
                     float *h, uint32_t *bar, cudaStream_t s)
{
    FusedPlan pl;
    if (!plan_fused(T, H, I, gs, &pl))
        return WIDE_EUNSUPPORTED;
    const int G = I / gs;
    CUtensorMap tg, tu, td, th;
    const int TBP = pl.TB < 2 ? 2 : pl.TB;
    if (!make_tmap_rows3d(&tg, in.w_gate, I, H, H, pl.kw / 64, 8) ||
        !make_tmap_rows3d(&tu, in.w_up, I, H, H, pl.kw / 64, 8) ||
        !make_tmap_2d(&td, in.w_down, H, I, I, 2, pl.rows_box, gs, false) ||
        !make_tmap_f32_pairs(&th, h, (T + 1) / 2, I, gs, TBP / 2))
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
    a.rt = pl.rt;
    a.nr = pl.nr;
    a.ni = pl.ni;
    a.nslots = pl.nslots;
    a.slot_bytes = pl.slot_bytes;
    a.w2_bytes = pl.w2_bytes;
    a.h2_bytes = pl.h2_bytes;
    a.h2_stride = pl.h2_stride;
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

extern "C" int wide_set_decode_ffn_path(int mode)
{
    if (mode != WIDE_DECODE_AUTO && mode != WIDE_DECODE_FUSED && mode != WIDE_DECODE_GEMV &&
        mode != wide::kDecodeFusedOld)
        return WIDE_EINVAL;
    return wide::g_decode_mode.exchange(mode);
}
