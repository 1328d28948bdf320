// ffn_decode_split.cu -- the bf16 decode FFN as one persistent kernel in
// which every CTA owns a slice of the batch's kept channels.
//
// WIDE, technical summary section 2.A (each token keeps its own contiguous
// FFN channel groups) and section 2.C (block-level skipping), for decode
// batches of up to 32 tokens.  Only the weights of the groups some token of
// the batch keeps (the batch's union) are read from HBM, each byte once, and
// a (token, group) pair the token skips costs no multiply.
//
// Work split.  The union's groups are dealt out to the CTAs (one per SM):
// with at least as many CTAs as live groups, each group's channels are cut
// into contiguous ranges of 8-channel units for ceil-or-floor(P / U) CTAs;
// with fewer, a CTA takes whole groups.  An "item" is one (group, channel
// range).  For its item a CTA computes, with no data from any other CTA,
//   phase A  h[t][c] = silu(x[t] . W_gate[c]) * (x[t] . W_up[c]) for the
//            item's channels c and the tokens t that keep the group, and
//   phase B  the item's share of the down projection,
//            part[t][n] = sum over the item's c of h[t][c] * W_down[n][c],
//            for every output row n, added into an fp32 accumulator in
//            global memory with red.add (the accumulator and the arrival
//            counter are zeroed on the stream before the launch).
// After its last item a CTA counts itself in; once every CTA has (a
// bounded wait on the counter), each CTA converts its slice of the
// accumulator into the call's outputs (bf16 sum, plus residuals).  No CTA
// ever waits for another CTA's h: W_down streams right behind W_gate/W_up.
//
// Token compaction.  The item's group has its own active tokens t_0 < t_1 <
// ... (at most 32); they are paired (t_0, t_1), (t_2, t_3), ... and every
// packed fp32x2 FMA serves one pair, so a token that skips the group costs
// nothing (an odd count leaves one padding slot, zero throughout).
//
// Warp 0 (one lane) streams every stage by TMA through an mbarrier ring:
//   phase A stage: a KW-column window of the pass's W_gate and W_up rows
//     (up to S = 4096 / KW channels, one 32-row box each for a full pass,
//     16 KB) and the same window of x for all T tokens (bf16, as loaded);
//   phase B stage: 1024 rows x 8 channels of W_down (16 KB, one 3-D box).
// Warp 1 turns each phase-A window's x rows into the item's token pairs in
// fp32 ("x32": for every column, one pair's two values side by side) in the
// stage's own x32 area and hands every stage on (xready).  Warps 2..17
// compute; each waits only for its stage's xready, so the consumer warps
// drift apart by up to the ring's depth instead of moving in lockstep.
//   Phase A thread: one channel of the pass (its W_gate and W_up rows) at one
//     8-column chunk of the window (KW / 8 chunk lanes per channel), all of
//     the item's token pairs; sums over the chunk lanes by shuffles at the end
//     of the pass.
//   Phase B thread: rows r and r + 512 of the 1024-row block, the stage's 8
//     channels, all pairs; the 8-channel h pieces are the same for every
//     thread (broadcast reads).
// In both phases a thread holds two bf16 weight rows of one 8-column chunk
// and runs, per column, one packed FMA per (row, pair): the weight widened
// into both halves of a register pair, the operand the pair's two values.
#include "common.cuh"
#include "host.h"

#include <atomic>
#include <mutex>

namespace wide {
namespace {

// Consumer warps and the weight rows each consumer thread owns (the gate
// and up rows of kSRows / 2 channels in phase A, kSRows output rows in phase
// B): 8 x 4 or 16 x 2.  A CTA is the consumers plus 3 warps; with 8
// consumer warps a sub-partition holds 3 warps, so a thread may use 168
// registers, with 16 it holds 5 (96 registers).
#ifndef WIDE_SPLIT_WARPS
#define WIDE_SPLIT_WARPS 8
#endif
constexpr int kSWarps = WIDE_SPLIT_WARPS;     // consumer warps
constexpr int kSRows = 32 / kSWarps;          // weight rows per consumer thread
constexpr int kSMaxReg = kSWarps == 8 ? 168 : 96;
constexpr int kSCons = 32 * kSWarps;          // consumer threads
constexpr int kSThreads = kSCons + 96;        // + the TMA producer and two x converter warps
constexpr int kSMaxTok = kSplitMaxTok;        // tokens per launch (a larger batch: several)
constexpr int kSRowBlk = kSCons * kSRows;     // phase-B rows per block (1024)
constexpr int kSDownBox = 256;                // rows per W_down TMA box
constexpr int kSMaxSlots = 8;
constexpr int kSMaxG = 1024;
constexpr int kSMaxMaskWords = 1024;          // T * W
constexpr int kSMaxItems = 8;                 // items per CTA (ceil(U / P))

struct SplitArgs {
    const uint32_t *mask;   // [T][W] packed group bits
    float *acc;             // [T][H] fp32 accumulator (0 at launch)
    uint32_t *done;         // arrival counter (0 at launch)
    DownOutputs o;
    int T, H, I, W, G, gs;
    int nslots;
    uint32_t slot_bytes;    // weights + x (bf16) + x32
    uint32_t xb_off;        // x window inside a slot
    uint32_t x32_off;       // token-pair x inside a slot
    int bch;                // channels of W_down per phase-B stage (8 or 16)
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
__device__ __forceinline__ float2 lo2(const float4 v) { return make_float2(v.x, v.y); }
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&v);
}
__device__ __forceinline__ float2 hi2(const float4 v) { return make_float2(v.z, v.w); }

__device__ __forceinline__ void consumer_sync()
{
    asm volatile("bar.sync 1, %0;" ::"n"(kSCons) : "memory");
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
__device__ __forceinline__ void red_add_f32(float *p, float v)
{
    asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
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

// Sums v[0..N) (float pairs) over the 2^LV lanes that differ in lane bits
// [0, LV).  The first S = scatter_levels(N / KEEP, LV) steps halve what a
// lane carries (a lane keeps the half its bit selects and receives its
// partner's copy of it), the remaining LV - S steps add whole arrays.
// Afterwards lane l holds in v[0..N >> S) the sums of entries
//   m = ((l >> (LV - S)) & (2^S - 1)) * (N >> S) + j.
// (Works on the float2 array itself: viewing it as floats would take its
// address and move it out of registers.)
template <int N, int LV, int KEEP>
__device__ __forceinline__ void lane_reduce2(float2 (&v)[N], int lane)
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
                const float2 send = hi ? v[i] : v[i + n];
                const float2 keep = hi ? v[i + n] : v[i];
                v[i].x = keep.x + __shfl_xor_sync(0xffffffffu, send.x, o);
                v[i].y = keep.y + __shfl_xor_sync(0xffffffffu, send.y, o);
            }
        }
    }
    constexpr int R = N >> S;
#pragma unroll
    for (int l = S; l < LV; ++l) {
        const int o = 1 << (LV - 1 - l);
#pragma unroll
        for (int i = 0; i < R; ++i) {
            v[i].x += __shfl_xor_sync(0xffffffffu, v[i].x, o);
            v[i].y += __shfl_xor_sync(0xffffffffu, v[i].y, o);
        }
    }
}

// Four bf16 weight rows (w[0..3]: 8 consecutive columns each) times the
// token pairs' operand over those columns: pair p's values of columns 2q,
// 2q + 1 are the 16 bytes at ob + p * pstride + q * QS (lo half column 2q,
// hi half column 2q + 1; in each half, the pair's two tokens).  Row r's sums
// for pair p accumulate in acc[4p + r].  NA pairs, NA <= NP.
// Per column pair, every pair's operand is loaded first, then the low
// column's FMAs run for all pairs and rows, then the high column's, so two
// updates of one accumulator are 4 * NA FMAs apart (no stall on the
// previous result).
template <int NP, int NA, int QS>
__device__ __forceinline__ void rows4(const uint4 (&w)[kSRows], const uint8_t *ob,
                                      uint32_t pstride, float2 (&acc)[kSRows * NP])
{
    constexpr int R = kSRows;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        float4 v[NA];
#pragma unroll
        for (int p = 0; p < NA; ++p)
            v[p] = lds128f(ob + p * pstride + q * QS);
        float2 d[R];
#pragma unroll
        for (int r = 0; r < R; ++r)
            d[r] = dup_lo(word(w[r], q));
#pragma unroll
        for (int p = 0; p < NA; ++p)
#pragma unroll
            for (int r = 0; r < R; ++r)
                acc[R * p + r] = __ffma2_rn(d[r], lo2(v[p]), acc[R * p + r]);
#pragma unroll
        for (int r = 0; r < R; ++r)
            d[r] = dup_hi(word(w[r], q));
#pragma unroll
        for (int p = 0; p < NA; ++p)
#pragma unroll
            for (int r = 0; r < R; ++r)
                acc[R * p + r] = __ffma2_rn(d[r], hi2(v[p]), acc[R * p + r]);
    }
}

// rows4 for the run-time pair count np (1 <= np <= NP).
template <int NP, int QS>
__device__ __forceinline__ void rows4_np(int np, const uint4 (&w)[kSRows], const uint8_t *ob,
                                         uint32_t pstride, float2 (&acc)[kSRows * NP])
{
#define WIDE_ROWS4_CASE(n)                                                                          \
    case n:                                                                                        \
        if constexpr (n <= NP)                                                                     \
            rows4<NP, n, QS>(w, ob, pstride, acc);                                                 \
        break;
    switch (np) {
        WIDE_ROWS4_CASE(1) WIDE_ROWS4_CASE(2) WIDE_ROWS4_CASE(3) WIDE_ROWS4_CASE(4)
        WIDE_ROWS4_CASE(5) WIDE_ROWS4_CASE(6) WIDE_ROWS4_CASE(7) WIDE_ROWS4_CASE(8)
    default:
        break;
    }
#undef WIDE_ROWS4_CASE
}

// Phase A for up to 8 tokens, column-pair form: the thread's weight rows' 8
// columns (w[r]: gate and up of its channels) against the n active tokens'
// fp32 x (token i's 8 columns: 16 bytes at xw + xr[i], 16 more 1 KB
// further).  The packed FMA takes two adjacent columns: a weight word widens
// into one register pair (one byte permute per element), the token's two x
// values are a register pair already, and acc[R i + r] collects token i's
// row-r sums over even and odd columns (added at the end of the pass).
template <int NT, int NA>
__device__ __forceinline__ void colpair4(const uint4 (&w)[kSRows], const uint8_t *xw,
                                         const uint32_t (&xr)[NT], float2 (&acc)[kSRows * NT])
{
    constexpr int R = kSRows;
    float2 wv[R][4];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int q = 0; q < 4; ++q)
            wv[r][q] = make_float2(bf_lo(word(w[r], q)), bf_hi(word(w[r], q)));
#pragma unroll
    for (int i = 0; i < NA; ++i) {
        const float4 a = lds128f(xw + xr[i]), b = lds128f(xw + xr[i] + 1024);
        const float2 x2[4] = {lo2(a), hi2(a), lo2(b), hi2(b)};
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int r = 0; r < R; ++r)
                acc[R * i + r] = __ffma2_rn(wv[r][q], x2[q], acc[R * i + r]);
    }
}

template <int NT>
__device__ __forceinline__ void colpair4_n(int n, const uint4 (&w)[kSRows], const uint8_t *xw,
                                           const uint32_t (&xr)[NT], float2 (&acc)[kSRows * NT])
{
#define WIDE_COLPAIR_CASE(m)                                                                       \
    case m:                                                                                        \
        if constexpr (m <= NT)                                                                     \
            colpair4<NT, m>(w, xw, xr, acc);                                                       \
        break;
    switch (n) {
        WIDE_COLPAIR_CASE(1) WIDE_COLPAIR_CASE(2) WIDE_COLPAIR_CASE(3) WIDE_COLPAIR_CASE(4)
        WIDE_COLPAIR_CASE(5) WIDE_COLPAIR_CASE(6) WIDE_COLPAIR_CASE(7) WIDE_COLPAIR_CASE(8)
    default:
        break;
    }
#undef WIDE_COLPAIR_CASE
}

// Geometry of the kernel by pairs per group (NP).
// A consumer thread owns two channels of the pass (the gate and up rows of
// each: four weight rows) at one chunk lane.
//   NP <= 4 (up to 8 tokens; the weight stream sets the pace): 512-column
//     windows (1 KB of every weight row per copy: long row pieces stream far
//     better than 256-byte ones), one warp per channel pair (each lane two
//     8-column chunks), 16 channels per pass, the column-pair form on the
//     window's x widened to fp32 per token by the converters.
//   NP == 8 (9..16 tokens; the multiplies set the pace): 128-column windows
//     (the x32 area of a window grows with NP), a half warp per channel
//     pair, 32 channels per pass, token pairs from x32.
template <int NP> struct SplitCfg {
    static constexpr bool kWide = NP <= 4;
    static constexpr int KW = kWide ? 512 : 128;      // window columns
    static constexpr int CL = kWide ? 32 : 16;        // chunk lanes per channel
    static constexpr int LV = kWide ? 5 : 4;          // log2(CL)
    static constexpr int CPL = KW / (8 * CL);         // chunks per lane per window
    static constexpr int S = kSCons / CL * kSRows / 2; // channels per pass
    static constexpr int WB = 2 * S * KW * 2;         // weight bytes per phase-A stage
};

// One item of this CTA: live-list index of the group and its 8-channel
// units [u0, u1).
struct Item {
    int li, u0, u1;
};

// The items of CTA c of P for U live groups of gs channels; returns their
// count (0..kSMaxItems).  cw[0..U] are the live groups' cumulative work
// weights (cw[0] = 0).  With at least as many CTAs as groups, every group
// gets one CTA and the other P - U are dealt out in proportion to the
// weights (group i: K(i + 1) - K(i) CTAs, K(i) = i + floor((P - U) cw[i] /
// cw[U])); its units are then cut evenly over its CTAs.
__device__ __forceinline__ int cta_items(int c, int P, int U, int gs, const int *cw,
                                         Item (&it)[kSMaxItems])
{
    if (U <= 0)
        return 0;
    const int units = gs / 8;
    if (P >= U) {
        const int64_t R = P - U, Wt = cw[U] > 0 ? cw[U] : 1;
        auto K = [&](int i) { return i + (int)(R * cw[i] / Wt); };
        int lo = 0, hi = U - 1;                    // the last i with K(i) <= c
        while (lo < hi) {
            const int mid = (lo + hi + 1) / 2;
            if (K(mid) <= c)
                lo = mid;
            else
                hi = mid - 1;
        }
        const int i = lo;
        const int f = K(i), e = K(i + 1);
        const int k = e - f, j = c - f;
        it[0].li = i;
        it[0].u0 = j * units / k;
        it[0].u1 = (j + 1) * units / k;
        return it[0].u1 > it[0].u0 ? 1 : 0;
    }
    const int g0 = (int)((int64_t)c * U / P), g1 = (int)((int64_t)(c + 1) * U / P);
    int n = 0;
    for (int g = g0; g < g1 && n < kSMaxItems; ++g, ++n) {
        it[n].li = g;
        it[n].u0 = 0;
        it[n].u1 = units;
    }
    return n;
}

// One CTA of 11 warps per SM (TMA producer, two x converters, 8 consumer
// warps); a sub-partition holds 3 of them, so a thread gets at most
// 16384 / 96 registers, 168 in the allocation granularity: room for the
// accumulators of 4 rows x 8 token pairs without spilling.
template <int NP>
__global__ void __maxnreg__(kSMaxReg)
    ffn_decode_split(const __grid_constant__ CUtensorMap tm_gate,
                     const __grid_constant__ CUtensorMap tm_up,
                     const __grid_constant__ CUtensorMap tm_gate8,
                     const __grid_constant__ CUtensorMap tm_up8,
                     const __grid_constant__ CUtensorMap tm_x,
                     const __grid_constant__ CUtensorMap tm_down, const SplitArgs a)
{
    using C = SplitCfg<NP>;
    constexpr int KW = C::KW, CL = C::CL, S = C::S, WB = C::WB;
    static_assert(C::CPL * CL * 8 == KW && (1 << C::LV) == CL, "window geometry");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    const int NS = a.nslots;
    const int T = a.T, H = a.H, gs = a.gs, W = a.W;
    uint8_t *slots = smem;
    float *hs = reinterpret_cast<float *>(smem + (size_t)NS * a.slot_bytes);   // [NP][gs][2]
    uint32_t *mall = reinterpret_cast<uint32_t *>(hs + (size_t)NP * gs * 2);   // [T][W]
    int *live = reinterpret_cast<int *>(mall + T * W);                         // [G]
    int *cw = live + a.G;                                                      // [G + 1]
    int *toks = cw + a.G + 1;                                                  // [items][32]
    uint64_t *full = reinterpret_cast<uint64_t *>(
        (reinterpret_cast<uintptr_t>(toks + kSMaxItems * kSMaxTok) + 7) & ~(uintptr_t)7);
    uint64_t *empty = full + NS;
    uint64_t *xready = empty + NS;
    __shared__ int s_nlive, s_err, s_issued, s_nitems, s_ntok[kSMaxItems];
    __shared__ Item s_items[kSMaxItems];

    const int tid = (int)threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int P = (int)gridDim.x, c = (int)blockIdx.x;

    for (int i = tid; i < T * W; i += kSThreads)
        mall[i] = a.mask[i];
    if (tid == 0) {
        s_err = 0;
        s_issued = 0;
        for (int i = 0; i < NS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&xready[i], 2);
            mbar_init(&empty[i], kSWarps);
        }
        fence_mbar_init();
        tma_prefetch_desc(&tm_gate);
        tma_prefetch_desc(&tm_up);
        tma_prefetch_desc(&tm_x);
        tma_prefetch_desc(&tm_down);
    }
    __syncthreads();
    // the batch's union of groups as a list (warp 0)
    if (warp == 0) {
        uint32_t u = 0;
        bool bad = false;
        if (lane < W) {
            for (int t = 0; t < T; ++t)
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
    // work weight of every live group: 16 + its active tokens (the weight
    // stream costs a group the same whatever its tokens; each token adds
    // about a sixteenth in multiplies), then the cumulative sums (warp 0)
    {
        const int U = s_nlive;
        for (int li = tid; li < U; li += kSThreads) {
            const int g = live[li];
            int n = 0;
            for (int t = 0; t < T; ++t)
                n += (mall[t * W + (g >> 5)] >> (g & 31)) & 1u;
            cw[li + 1] = 16 + n;
        }
        __syncthreads();
        if (warp == 0) {
            const int per = (U + 31) / 32, b0 = min(U, lane * per), b1 = min(U, b0 + per);
            int sum = 0;
            for (int i = b0; i < b1; ++i)
                sum += cw[i + 1];
            int incl = sum;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off)
                    incl += v;
            }
            int run = incl - sum;
            for (int i = b0; i < b1; ++i) {
                run += cw[i + 1];
                cw[i + 1] = run;
            }
            if (lane == 0)
                cw[0] = 0;
        }
    }
    __syncthreads();
    // this CTA's items and each item's active tokens, ascending (warp 1:
    // one ballot per item)
    if (warp == 1) {
        Item its[kSMaxItems];
        const int n_it = cta_items(c, P, s_nlive, gs, cw, its);
        if (lane == 0) {
            s_nitems = n_it;
            for (int k = 0; k < n_it; ++k)
                s_items[k] = its[k];
        }
        for (int k = 0; k < n_it; ++k) {
            const int g = live[its[k].li];
            const bool keep = lane < T && ((mall[lane * W + (g >> 5)] >> (g & 31)) & 1u) != 0u;
            const uint32_t b = __ballot_sync(0xffffffffu, keep);
            if (keep)
                toks[k * kSMaxTok + __popc(b & ((1u << lane) - 1u))] = lane;
            if (lane == 0)
                s_ntok[k] = __popc(b);
        }
    }
    __syncthreads();

    const int NW = H / KW;                       // windows per pass
    const int NRB = (H + kSRowBlk - 1) / kSRowBlk;
    const int n_items = s_nitems;
    const Item *items = s_items;
    auto passes = [&](const Item &it) { return ((it.u1 - it.u0) * 8 + S - 1) / S; };
    auto slot_of = [&](int kk) { return slots + (size_t)(kk % NS) * a.slot_bytes; };
    auto par_of = [&](int kk) { return (uint32_t)(kk / NS) & 1u; };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            bool err = false;
            int k = 0;
            auto acquire = [&](int kk) {
                if (kk >= NS && !err) {
                    if (!mbar_wait(&empty[kk % NS], (uint32_t)(kk / NS - 1) & 1u))
                        err = true;
                }
                return !err;
            };
            for (int ii = 0; ii < n_items && !err; ++ii) {
                const Item it = items[ii];
                const int g = live[it.li];
                const int c0 = g * gs + it.u0 * 8, nch = (it.u1 - it.u0) * 8;
                for (int ps = 0; ps * S < nch && !err; ++ps) {
                    const int ns = min(S, nch - ps * S), row0 = c0 + ps * S;
                    for (int w = 0; w < NW; ++w, ++k) {
                        if (!acquire(k))
                            break;
                        uint64_t *fb = &full[k % NS];
                        uint8_t *sb = slot_of(k);
                        mbar_arrive_expect_tx(fb, 2u * (uint32_t)ns * KW * 2u + (uint32_t)T * KW * 2u);
                        if (ns == S) {
                            tma_load_3d(sb, &tm_gate, 0, w * (KW / 64), row0, fb);
                            tma_load_3d(sb + WB / 2, &tm_up, 0, w * (KW / 64), row0, fb);
                        } else {
                            for (int u = 0; u < ns / 8; ++u) {
                                tma_load_3d(sb + (size_t)u * 8 * KW * 2, &tm_gate8, 0,
                                            w * (KW / 64), row0 + 8 * u, fb);
                                tma_load_3d(sb + WB / 2 + (size_t)u * 8 * KW * 2, &tm_up8, 0,
                                            w * (KW / 64), row0 + 8 * u, fb);
                            }
                        }
                        tma_load_3d(sb + a.xb_off, &tm_x, 0, w * (KW / 64), 0, fb);
                    }
                }
                const int BC = a.bch, nbs = (nch + BC - 1) / BC;
                for (int rb = 0; rb < NRB && !err; ++rb) {
                    for (int cc = 0; cc < nbs; ++cc, ++k) {
                        if (!acquire(k))
                            break;
                        uint64_t *fb = &full[k % NS];
                        mbar_arrive_expect_tx(fb, (uint32_t)kSRowBlk * BC * 2u);
                        tma_load_3d(slot_of(k), &tm_down, c0 + BC * cc, 0,
                                    rb * (kSRowBlk / kSDownBox), fb);
                    }
                }
            }
            s_issued = k;
            if (err) {
                set_status(a.status, WIDE_DEV_TIMEOUT);
                atomicExch(&s_err, 1);
            }
        }
    } else if (warp <= 2) {
        // ------------------------------------------------ x converters
        // For every phase-A stage: the item's token pairs of the stage's x
        // window, in fp32, into the stage's x32 area: [pair][q][chunk][16
        // bytes], the 16 bytes holding columns 8 * chunk + 2q, + 1 of the
        // pair (the chunk lanes of a channel then read contiguous bytes).
        // Every stage (phase B too) is handed on through xready.
        {
            const int cv = warp - 1;
            bool ok = true;
            int k = 0;
            auto pass_on = [&](int kk) {
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&xready[kk % NS]);
            };
            auto wait_full = [&](int kk) {
                if (ok && !mbar_wait(&full[kk % NS], par_of(kk))) {
                    ok = false;
                    set_status(a.status, WIDE_DEV_TIMEOUT);
                    atomicExch(&s_err, 1);
                }
            };
            for (int ii = 0; ii < n_items; ++ii) {
                const Item it = items[ii];
                const int n = s_ntok[ii], np = (n + 1) / 2;
                const int *tk = toks + ii * kSMaxTok;
                const int nA = passes(it) * NW;
                const int nB = NRB * (((it.u1 - it.u0) * 8 + a.bch - 1) / a.bch);
                for (int kA = 0; kA < nA; ++kA, ++k) {
                    wait_full(k);
                    if (ok && C::kWide) {
                        // every token's 512 columns in fp32: [t][half][64
                        // chunks][16 bytes], half 0 the chunk's first 4
                        // columns (the lanes of a warp then read 512
                        // contiguous bytes); one (token, chunk) per lane and
                        // step: a 16-byte read, two 16-byte writes
                        const uint8_t *xb = slot_of(k) + a.xb_off;
                        uint8_t *x32 = slot_of(k) + a.x32_off;
                        for (int u = cv * 32 + lane; u < T * (KW / 8); u += 64) {
                            const int t = u / (KW / 8), l = u % (KW / 8);
                            const uint4 xv = lds128(xb + (size_t)t * KW * 2 + l * 16);
                            uint8_t *dst = x32 + (size_t)t * KW * 4 + l * 16;
                            *reinterpret_cast<float4 *>(dst) =
                                make_float4(bf_lo(xv.x), bf_hi(xv.x), bf_lo(xv.y), bf_hi(xv.y));
                            *reinterpret_cast<float4 *>(dst + KW * 2) =
                                make_float4(bf_lo(xv.z), bf_hi(xv.z), bf_lo(xv.w), bf_hi(xv.w));
                        }
                    } else if (ok) {
                        // one (pair, 8-column chunk) per lane and step: two
                        // 16-byte reads, four 16-byte writes
                        const uint8_t *xb = slot_of(k) + a.xb_off;
                        uint8_t *x32 = slot_of(k) + a.x32_off;
                        for (int u = cv * 32 + lane; u < np * (KW / 8); u += 64) {
                            const int pp = u / (KW / 8), l = u % (KW / 8);
                            const int ta = tk[2 * pp], tb = 2 * pp + 1 < n ? tk[2 * pp + 1] : -1;
                            const uint4 xa = lds128(xb + (size_t)ta * KW * 2 + l * 16);
                            const uint4 xv = tb >= 0 ? lds128(xb + (size_t)tb * KW * 2 + l * 16)
                                                     : make_uint4(0u, 0u, 0u, 0u);
                            uint8_t *dst = x32 + (size_t)pp * KW * 8 + l * 16;
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                *reinterpret_cast<float4 *>(dst + q * (KW / 8) * 16) =
                                    make_float4(bf_lo(word(xa, q)), bf_lo(word(xv, q)),
                                                bf_hi(word(xa, q)), bf_hi(word(xv, q)));
                        }
                    }
                    pass_on(k);
                }
                for (int kB = 0; kB < nB; ++kB, ++k) {
                    wait_full(k);
                    pass_on(k);
                }
            }
        }
    } else {
        // ------------------------------------------------ consumers
        const int ct = tid - 96;
        bool ok = true;
        uint64_t *ready = xready;                  // the converters hand every stage on
        auto wait_ready = [&](int kk) {
            if (ok && !mbar_wait(&ready[kk % NS], par_of(kk))) {
                ok = false;
                set_status(a.status, WIDE_DEV_TIMEOUT);
                atomicExch(&s_err, 1);
            }
        };
        auto release = [&](int kk) {
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&empty[kk % NS]);
        };

        constexpr int R = kSRows, RC = kSRows / 2;   // rows, channels per thread
        const int sp = ct / CL, cl = ct % CL;      // phase A: channel set of the pass, chunk lane
        float2 acc[R * NP];
        int k = 0;
        for (int ii = 0; ii < n_items; ++ii) {
            const Item it = items[ii];
            const int n = s_ntok[ii], np = (n + 1) / 2;
            const int nch = (it.u1 - it.u0) * 8;
            const int *tk = toks + ii * kSMaxTok;
            // ---- phase A
            for (int ps = 0; ps * S < nch; ++ps) {
                const int ns = min(S, nch - ps * S);
                const bool act = RC * sp < ns;       // ns is a multiple of 8
#pragma unroll
                for (int e = 0; e < R * NP; ++e)
                    acc[e] = make_float2(0.f, 0.f);
                if constexpr (C::kWide) {
                    constexpr int NT = 2 * NP;      // tokens of a group, at most
                    float2 acw[R * NT];
#pragma unroll
                    for (int e = 0; e < R * NT; ++e)
                        acw[e] = make_float2(0.f, 0.f);
                    uint32_t xr[NT];
#pragma unroll
                    for (int i = 0; i < NT; ++i)
                        xr[i] = (uint32_t)(i < n ? tk[i] : 0) * KW * 4u;
                    for (int w = 0; w < NW; ++w, ++k) {
                        wait_ready(k);
                        if (ok && act) {
                            const uint8_t *sb = slot_of(k);
#pragma unroll
                            for (int h = 0; h < C::CPL; ++h) {
                                const int ch = cl + h * CL;
                                const size_t r0 = (size_t)(RC * sp) * KW * 2 + ch * 16;
                                uint4 wr[R];
#pragma unroll
                                for (int c2 = 0; c2 < RC; ++c2) {
                                    wr[2 * c2] = lds128(sb + r0 + c2 * KW * 2);
                                    wr[2 * c2 + 1] = lds128(sb + WB / 2 + r0 + c2 * KW * 2);
                                }
                                colpair4_n<NT>(n, wr, sb + a.x32_off + ch * 16, xr, acw);
                            }
                        }
                        release(k);
                    }
                    // token i's (gate, up) sums of channel c (acw[R i + 2c],
                    // acw[R i + 2c + 1], each over even and odd columns) over
                    // the chunk lanes; the owners write h (token i is slot
                    // i & 1 of pair i / 2)
                    float2 gu[RC * NT];
#pragma unroll
                    for (int i = 0; i < NT; ++i)
#pragma unroll
                        for (int cc = 0; cc < RC; ++cc)
                            gu[RC * i + cc] = make_float2(acw[R * i + 2 * cc].x + acw[R * i + 2 * cc].y,
                                                          acw[R * i + 2 * cc + 1].x +
                                                              acw[R * i + 2 * cc + 1].y);
                    lane_reduce2<RC * NT, C::LV, 1>(gu, lane);
                    constexpr int LV = C::LV, Sl = scatter_levels(RC * NT, LV),
                                  RR = (RC * NT) >> Sl;
                    if (act && (cl & ((1 << (LV - Sl)) - 1)) == 0) {
                        const int mb = ((cl >> (LV - Sl)) & ((1 << Sl) - 1)) * RR;
#pragma unroll
                        for (int e = 0; e < RR; ++e) {
                            const int m = mb + e, i = m / RC;
                            const int chl = ps * S + RC * sp + m % RC;
                            if (i < n)
                                hs[((size_t)(i >> 1) * nch + chl) * 2 + (i & 1)] =
                                    silu_f32(gu[e].x) * gu[e].y;
                        }
                    }
                } else {
                    for (int w = 0; w < NW; ++w, ++k) {
                        wait_ready(k);
                        if (ok && act) {
                            const uint8_t *sb = slot_of(k);
                            const size_t r0 = (size_t)(RC * sp) * KW * 2 + cl * 16;
                            uint4 wr[R];
#pragma unroll
                            for (int c2 = 0; c2 < RC; ++c2) {
                                wr[2 * c2] = lds128(sb + r0 + c2 * KW * 2);
                                wr[2 * c2 + 1] = lds128(sb + WB / 2 + r0 + c2 * KW * 2);
                            }
                            rows4_np<NP, KW * 2>(np, wr, sb + a.x32_off + cl * 16,
                                                 (uint32_t)KW * 8u, acc);
                        }
                        release(k);
                    }
                    // sums over the chunk lanes, in place: acc[R p + 2c] is
                    // pair p's gate sums of channel c, acc[R p + 2c + 1] its
                    // up sums (each: the pair's two token slots); the owners
                    // write h for this pass's channels
                    constexpr int N = R * NP, LV = C::LV;
                    lane_reduce2<N, LV, 2>(acc, lane);
                    constexpr int Sl = scatter_levels(N / 2, LV), RR = N >> Sl;
                    if (act && (cl & ((1 << (LV - Sl)) - 1)) == 0) {
                        const int mb = ((cl >> (LV - Sl)) & ((1 << Sl) - 1)) * RR;
#pragma unroll
                        for (int e = 0; e < RR; e += 2) {
                            const int m = mb + e, p = m / R;
                            const int chl = ps * S + RC * sp + (m % R) / 2;
                            if (p < np)
                                *reinterpret_cast<float2 *>(hs + ((size_t)p * nch + chl) * 2) =
                                    make_float2(silu_f32(acc[e].x) * acc[e + 1].x,
                                                silu_f32(acc[e].y) * acc[e + 1].y);
                        }
                    }
                }
            }
            consumer_sync();                       // h of the item complete
            // ---- phase B
            const int BC = a.bch, nbs = (nch + BC - 1) / BC;
            for (int rb = 0; rb < NRB; ++rb) {
#pragma unroll
                for (int e = 0; e < R * NP; ++e)
                    acc[e] = make_float2(0.f, 0.f);
                for (int cc = 0; cc < nbs; ++cc, ++k) {
                    wait_ready(k);
                    if (ok) {
                        // rows ct + 256 j (j = 0..3) of the stage's 1024 rows
                        // of BC channels; with 16 channels a lane takes the
                        // two 8-channel halves in an order set by lane bit 2,
                        // so the warp's 16-byte reads hit 8 distinct bank
                        // groups
                        const uint8_t *sb = slot_of(k);
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            if (hh * 8 >= BC)
                                break;
                            const int half = BC == 16 ? (hh ^ ((lane >> 2) & 1)) : 0;
                            const int c8 = cc * BC + half * 8;     // channel within the item
                            if (c8 >= nch)
                                continue;
                            uint4 wr[R];
#pragma unroll
                            for (int j = 0; j < R; ++j)
                                wr[j] = lds128(sb + (size_t)(ct + kSCons * j) * BC * 2 + half * 16);
                            rows4_np<NP, 16>(np, wr, reinterpret_cast<const uint8_t *>(hs) + c8 * 8,
                                             (uint32_t)nch * 8u, acc);
                        }
                    }
                    release(k);
                }
                if (ok) {
                    // compile-time pair indices: a run-time index into acc
                    // would move the accumulators to local memory
#pragma unroll
                    for (int p = 0; p < NP; ++p) {
                        if (p >= np)
                            break;
                        const int ta = tk[2 * p], tb = 2 * p + 1 < n ? tk[2 * p + 1] : -1;
#pragma unroll
                        for (int j = 0; j < R; ++j) {
                            const int r = rb * kSRowBlk + ct + kSCons * j;
                            if (r < H) {
                                red_add_f32(a.acc + (size_t)ta * H + r, acc[R * p + j].x);
                                if (tb >= 0)
                                    red_add_f32(a.acc + (size_t)tb * H + r, acc[R * p + j].y);
                            }
                        }
                    }
                }
            }
            consumer_sync();                       // before the next item's h
        }
        __threadfence();
    }

    // ---- every CTA counted in, then this CTA's slice of the outputs
    __syncthreads();
    __shared__ int s_go;
    if (tid == 0) {
        int go = 0;
        red_add_release_gpu(a.done, 1u);
        if (!s_err) {
            const uint64_t t0 = globaltimer();
            for (uint32_t it = 0;; ++it) {
                if (ld_acquire_gpu(a.done) >= (uint32_t)P) {
                    go = 1;
                    break;
                }
                if ((it & 255u) == 255u && globaltimer() - t0 > kWaitLimitNs) {
                    set_status(a.status, WIDE_DEV_TIMEOUT);
                    break;
                }
            }
        }
        s_go = go;
    }
    __syncthreads();
    if (s_go) {
        const int64_t Q = (int64_t)T * H / 4;
        const int64_t q0 = (int64_t)c * Q / P, q1 = (int64_t)(c + 1) * Q / P;
        const DownOutputs &o = a.o;
        for (int64_t q = q0 + tid; q < q1; q += kSThreads) {
            const float4 v = __ldcg(reinterpret_cast<const float4 *>(a.acc) + q);
            const float s4[4] = {v.x, v.y, v.z, v.w};
            const size_t at = (size_t)q * 4;
            if (o.out_sum) {
                uint2 pk;
                pk.x = pack_bf16x2(s4[0], s4[1]);
                pk.y = pack_bf16x2(s4[2], s4[3]);
                *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(o.out_sum) + at) = pk;
            }
            if (o.out_total || o.out_total_f32) {
                float tot[4] = {s4[0], s4[1], s4[2], s4[3]};
                if (o.res_in) {
                    const uint2 r = *reinterpret_cast<const uint2 *>(
                        static_cast<const __nv_bfloat16 *>(o.res_in) + at);
                    tot[0] += bf_lo(r.x);
                    tot[1] += bf_hi(r.x);
                    tot[2] += bf_lo(r.y);
                    tot[3] += bf_hi(r.y);
                }
                if (o.res_f32) {
                    const float4 r = *reinterpret_cast<const float4 *>(o.res_f32 + at);
                    tot[0] += r.x;
                    tot[1] += r.y;
                    tot[2] += r.z;
                    tot[3] += r.w;
                }
                if (o.out_total) {
                    uint2 pk;
                    pk.x = pack_bf16x2(tot[0], tot[1]);
                    pk.y = pack_bf16x2(tot[2], tot[3]);
                    *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(o.out_total) + at) = pk;
                }
                if (o.out_total_f32)
                    *reinterpret_cast<float4 *>(o.out_total_f32 + at) =
                        make_float4(tot[0], tot[1], tot[2], tot[3]);
            }
        }
    }

    // after an error, let this CTA's copies in flight land before exit
    if (s_err && tid == 0) {
        const int issued = s_issued;
        for (int kk = issued - 1; kk >= 0 && kk >= issued - NS; --kk)
            mbar_wait(&full[kk % NS], (uint32_t)(kk / NS) & 1u);
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

int pairs_tmpl(int T)
{
    const int np = (T + 1) / 2;
    return np <= 1 ? 1 : np <= 2 ? 2 : np <= 4 ? 4 : np <= 8 ? 8 : 16;
}

// Launch geometry of one call; false if the shape does not fit the kernel.
struct SplitPlan {
    int NP, P, kw, nslots, bch;
    uint32_t slot_bytes, xb_off, x32_off;
    size_t smem;
};

template <int NP> struct PlanOf {
    static constexpr int KW = SplitCfg<NP>::KW, WB = SplitCfg<NP>::WB;
};

bool plan_split(int T, int H, int I, int gs, SplitPlan *p)
{
    if (T < 1 || T > kSMaxTok || H % 256 != 0 || gs % 8 != 0 || gs < 8 || gs > 256 ||
        I % gs != 0)
        return false;
    const int G = I / gs, W = (G + 31) / 32;
    if (G > kSMaxG || T * W > kSMaxMaskWords)
        return false;
    const DevInfo di = dev_info();
    if (di.sms <= 0)
        return false;
    p->P = di.sms;
    if ((G + p->P - 1) / p->P > kSMaxItems)
        return false;
    p->NP = pairs_tmpl(T);
    // the 512-column variant needs whole windows; otherwise the fp32-operand
    // variant (a larger pair template is always valid)
    if (p->NP <= 4 && H % 512 != 0)
        p->NP = 8;
    int KW, WB;
    switch (p->NP) {
    case 1: KW = PlanOf<1>::KW; WB = PlanOf<1>::WB; break;
    case 2: KW = PlanOf<2>::KW; WB = PlanOf<2>::WB; break;
    case 4: KW = PlanOf<4>::KW; WB = PlanOf<4>::WB; break;
    default: KW = PlanOf<8>::KW; WB = PlanOf<8>::WB; break;
    }
    if (H % KW != 0)
        return false;
    p->kw = KW;
    // weights, the x window, then x32
    const uint32_t xb = ((uint32_t)T * KW * 2u + 1023u) & ~1023u;
    p->xb_off = (uint32_t)WB;
    p->x32_off = (uint32_t)WB + xb;
    uint32_t slot = p->x32_off + (p->NP <= 4 ? (uint32_t)T * KW * 4u : (uint32_t)p->NP * KW * 8u);
    // phase-B stages of 16 channels (32 bytes of every W_down row: 1024 row
    // pieces of 16 bytes take about as long to copy as 1024 of 32), so a
    // slot holds at least 32 KB
    p->bch = 16;
    if (slot < (uint32_t)kSRowBlk * 32u)
        slot = (uint32_t)kSRowBlk * 32u;
    p->slot_bytes = (slot + 1023u) & ~1023u;
    const size_t fixed = 1024 + (size_t)p->NP * gs * 8 + (size_t)T * W * 4 + (size_t)G * 8 + 4 +
                         (size_t)kSMaxItems * kSMaxTok * 4 + 8 + 3 * kSMaxSlots * 8;
    if ((size_t)di.optin <= fixed + 64)
        return false;
    int ns = (int)(((size_t)di.optin - fixed - 64) / p->slot_bytes);
    if (ns > kSMaxSlots)
        ns = kSMaxSlots;
    if (ns < 2)
        return false;
    p->nslots = ns;
    p->smem = fixed + (size_t)ns * p->slot_bytes;
    return true;
}

struct SplitMaps {
    CUtensorMap gate, up, gate8, up8, x, down;
};

template <int NP>
int launch_split(const SplitPlan &pl, const SplitMaps &m, const SplitArgs &a, cudaStream_t s)
{
    auto kernel = ffn_decode_split<NP>;
    if (!raise_smem_limit(reinterpret_cast<const void *>(kernel), pl.smem))
        return WIDE_CUDA_FAIL();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.P);
    cfg.blockDim = dim3(kSThreads);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    LaunchScope scope(KID_DECODE_FFN_SPLIT, s);
    if (cudaLaunchKernelEx(&cfg, kernel, m.gate, m.up, m.gate8, m.up8, m.x, m.down, a) !=
        cudaSuccess)
        return WIDE_CUDA_FAIL();
    return WIDE_OK;
}

}  // namespace

size_t decode_ffn_split_scratch(int T, int H)
{
    return align_up((size_t)T * H * sizeof(float), 256) + 256;
}

bool decode_ffn_split_supported(int T, int H, int I, int gs)
{
    SplitPlan p;
    return plan_split(T, H, I, gs, &p);
}

namespace {
std::atomic<int> g_decode_mode{WIDE_DECODE_AUTO};

// Which persistent kernel runs a bf16 decode FFN of T tokens (launches of
// at most kTcMaxTok or kSplitMaxTok tokens) with `cap` bytes of scratch:
// 3 the tensor-core kernel on the packed copy, 2 the tensor-core kernel on
// the nn.Linear weights, 1 the channel-split kernel, 0 none (the GEMV
// kernels run).  `linear`: the nn.Linear weights are at hand (the split and
// GEMV kernels need them).  AUTO: the channel-split kernel for up to 8
// tokens (there it is the fastest on B200), the tensor-core kernel above,
// on the packed copy when there is one.  TC and FUSED force the tensor-core
// and the channel-split kernel where they apply; GEMV forces the GEMVs
// (group size 32 has none: AUTO's choice).
int persistent_choice(int64_t T, int H, int I, int gs, size_t cap, const void *packed, bool linear)
{
    const int mode = g_decode_mode.load(std::memory_order_relaxed);
    const int Ttc = (int)(T < kTcMaxTok ? T : kTcMaxTok);
    const int Tsp = (int)(T < kSplitMaxTok ? T : kSplitMaxTok);
    const bool tc_fits = Ttc >= 1 && decode_ffn_tc_scratch(Ttc, H) <= cap;
    const bool tcp = packed && tc_fits && decode_ffn_tc_packed_supported(Ttc, H, I, gs);
    const bool tcl = linear && tc_fits && decode_ffn_tc_supported(Ttc, H, I, gs);
    const bool sp = linear && Tsp >= 1 && decode_ffn_split_supported(Tsp, H, I, gs) &&
                    decode_ffn_split_scratch(Tsp, H) <= cap;
    const int tc = tcp ? 3 : tcl ? 2 : 0;
    if (mode == WIDE_DECODE_FUSED)
        return sp ? 1 : tc;
    if (mode == WIDE_DECODE_TC)
        return tc ? tc : sp ? 1 : 0;
    if (mode == WIDE_DECODE_GEMV && gs != 32 && linear)
        return 0;
    if (sp && T <= 8)
        return 1;
    return tc ? tc : sp ? 1 : 0;
}
}  // namespace

bool decode_ffn_persistent_available(int64_t T, int H, int I, int gs, size_t cap,
                                     const void *packed, bool linear)
{
    return persistent_choice(T, H, I, gs, cap, packed, linear) != 0;
}

int decode_ffn_persistent(const void *x, const void *wg, const void *wu, const void *wd,
                          const uint32_t *mask, const DownOutputs &o, int64_t T, int H, int I,
                          int gs, void *scratch, size_t cap, cudaStream_t s, const void *packed)
{
    const bool linear = wg && wu && wd;
    if (persistent_choice(T, H, I, gs, cap, packed, linear) == 0)
        return WIDE_EUNSUPPORTED;
    const int W = (I / gs + 31) / 32;
    auto at = [](const void *p, int64_t off, size_t elem) -> const char * {
        return p ? static_cast<const char *>(p) + off * (int64_t)elem : nullptr;
    };
    // the kernel is chosen per launch from the tokens left (AUTO: a tail of
    // up to 8 tokens goes to the channel-split kernel)
    for (int64_t t0 = 0; t0 < T;) {
        const int which = persistent_choice(T - t0, H, I, gs, cap, packed, linear);
        if (which == 0)
            return WIDE_EUNSUPPORTED;
        const int per = which >= 2 ? kTcMaxTok : kSplitMaxTok;
        const int Tc = (int)(T - t0 < per ? T - t0 : per);
        const int64_t e = t0 * H;
        DownOutputs c = {};
        c.out_sum = const_cast<char *>(at(o.out_sum, e, 2));
        c.res_in = at(o.res_in, e, 2);
        c.res_f32 = reinterpret_cast<const float *>(at(o.res_f32, e, 4));
        c.out_total = const_cast<char *>(at(o.out_total, e, 2));
        c.out_total_f32 = reinterpret_cast<float *>(const_cast<char *>(at(o.out_total_f32, e, 4)));
        const void *xc = at(x, e, 2);
        const int rc = which >= 2
                           ? decode_ffn_tc(xc, wg, wu, wd, which == 3 ? packed : nullptr,
                                           mask + t0 * W, c, Tc, H, I, gs, scratch, s)
                           : decode_ffn_split(xc, wg, wu, wd, mask + t0 * W, c, Tc, H, I, gs,
                                             scratch, s);
        if (rc)
            return rc;
        t0 += Tc;
    }
    return WIDE_OK;
}

int decode_ffn_split(const void *x, const void *wg, const void *wu, const void *wd,
                     const uint32_t *mask, const DownOutputs &o, int T, int H, int I, int gs,
                     void *scratch, cudaStream_t s)
{
    SplitPlan pl;
    if (!plan_split(T, H, I, gs, &pl))
        return WIDE_EUNSUPPORTED;
    const int G = I / gs;
    // W_down as {channels, 256 rows, H / 256 row blocks}: one box of 8
    // channels x 1024 rows per phase-B stage
    SplitMaps m;
    const uint64_t ddims[3] = {(uint64_t)I, (uint64_t)kSDownBox, (uint64_t)(H / kSDownBox)};
    const uint64_t dstr[2] = {(uint64_t)I * 2, (uint64_t)I * 2 * kSDownBox};
    const uint32_t dbox[3] = {(uint32_t)pl.bch, kSDownBox, kSRowBlk / kSDownBox};
    // W_gate / W_up rows and x rows as {64, cols / 64, rows}: a box copies
    // whole KW-column pieces of rows (1 KB each in the 512-column variant)
    const uint32_t kwc = (uint32_t)pl.kw / 64,
                   S = (uint32_t)(kSCons / (pl.kw == 512 ? 32 : 16) * kSRows / 2);
    if (!make_tmap_rows3d(&m.gate, wg, I, H, H, kwc, S) ||
        !make_tmap_rows3d(&m.up, wu, I, H, H, kwc, S) ||
        !make_tmap_rows3d(&m.gate8, wg, I, H, H, kwc, 8) ||
        !make_tmap_rows3d(&m.up8, wu, I, H, H, kwc, 8) ||
        !make_tmap_rows3d(&m.x, x, T, H, H, kwc, T) ||
        !make_tmap_3d(&m.down, wd, ddims, dstr, dbox, 2))
        return WIDE_CUDA_FAIL();
    SplitArgs a = {};
    a.mask = mask;
    a.acc = static_cast<float *>(scratch);
    const size_t acc_bytes = align_up((size_t)T * H * sizeof(float), 256);
    a.done = reinterpret_cast<uint32_t *>(static_cast<char *>(scratch) + acc_bytes);
    a.o = o;
    a.T = T;
    a.H = H;
    a.I = I;
    a.G = G;
    a.W = (G + 31) / 32;
    a.gs = gs;
    a.nslots = pl.nslots;
    a.slot_bytes = pl.slot_bytes;
    a.xb_off = pl.xb_off;
    a.x32_off = pl.x32_off;
    a.bch = pl.bch;
    a.status = status_ptr();
    if (cudaMemsetAsync(scratch, 0, acc_bytes + sizeof(uint32_t), s) != cudaSuccess)
        return WIDE_CUDA_FAIL();
    switch (pl.NP) {
    case 1: return launch_split<1>(pl, m, a, s);
    case 2: return launch_split<2>(pl, m, a, s);
    case 4: return launch_split<4>(pl, m, a, s);
    default: return launch_split<8>(pl, m, a, s);
    }
}

}  // namespace wide

extern "C" int wide_set_decode_ffn_path(int mode)
{
    if (mode != WIDE_DECODE_AUTO && mode != WIDE_DECODE_FUSED && mode != WIDE_DECODE_GEMV &&
        mode != WIDE_DECODE_TC)
        return WIDE_EINVAL;
    return wide::g_decode_mode.exchange(mode);
}
