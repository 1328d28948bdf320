// attn_prefill.cu -- causal attention over compacted queries on tcgen05, and
// the whole masked prefill layer.
//
// WIDE, technical summary section 2.A (per-token GQA head groups) with the
// reordering of section 2.B: the tokens that keep head group j form the
// prefix perm_a[j][0 : count_a[j]) in ascending token order, so the queries
// of group j in sequence s are one contiguous range of that prefix.  Their
// RoPE'd query rows were written contiguously (compacted, group-major) by
// the Q projection, and attention works on dense 128-query tiles of that
// range; skipped (token, group) pairs are never computed.
//
// prefill_attn: one CTA per (query tile, query head of the group, sequence x
// KV head); warps 0-3 run the softmax (thread r = query row r = TMEM lane r),
// one thread of warp 4 issues the tensor-core MMAs, one thread of warp 5 the
// Q and K copies and one of warp 6 the V copies; two CTAs per SM (112 KB of
// shared memory and 256 TMEM columns each).  The roles hand work over through
// mbarriers only (no block-wide barrier inside the loop), and each role
// blocks only on the barrier of its own next step, so no MMA waits for the
// completion of an earlier one: the issuer queues S(t) as soon as K(t) has
// landed and the softmax has read S(t-2), then P(t-1) V(t-1) as soon as P(t-1)
// is written.  Per 64-key tile up to the tile's last query position:
//   S  = Q K^T           tcgen05, M=128 N=64 K=128, fp32 in one of two
//                        64-column TMEM buffers; S of the next tile is issued
//                        before this tile's softmax runs
//   P  = online softmax of S with the causal mask (key position <= query
//        position; tiles wholly below the diagonal skip the test), exp2
//        domain; P is written as bf16 to a 128B-swizzled K-major tile
//   O += P V             tcgen05, B = V read MN-major from the cache tile,
//                        O accumulated in TMEM columns 128..255 across tiles.
//        Each row keeps its reference max m_ref: P = exp2(s - m_ref) as long
//        as the row's running max stays within 8 (log2 units) of m_ref, so
//        P <= 256; when it grows further the row's O and sum are rescaled
//        (TMEM load, multiply, store) and m_ref moves up.  Rescales are rare
//        after the first tiles, so O never passes through registers per tile.
// K and V tiles are double-buffered: K(t) is copied once S(t-2) has
// completed, V(t) once P(t-2) V(t-2) has.
// Then O / l is written (bf16) at the token's signature-order row of the
// o_proj input.  Tiles with no query (ragged counts) exit at once.
#include "common.cuh"
#include "host.h"
#include "umma.cuh"

namespace wide {
namespace {

constexpr int kHD = 128;
constexpr int kBQ = 128;       // queries per tile
constexpr int kBKV = 64;       // keys per tile
constexpr uint32_t kQHalf = 128 * 128;  // Q: one 64-column half, 128 rows (16 KB)
constexpr uint32_t kQTile = 2 * kQHalf;
constexpr uint32_t kKHalf = 64 * 128;   // K or V: one 64-column half, 64 rows (8 KB)
constexpr uint32_t kKTile = 2 * kKHalf;
constexpr uint32_t kPTile = 128 * 128;  // P: 128 rows x 64 keys (16 KB)
constexpr float kLog2e = 1.4426950408889634f;

// 2^x by the SFU's approximate base-2 exponential (PTX ex2.approx; results
// below the normal range flush to 0, which a probability in bf16 loses anyway)
__device__ __forceinline__ float exp2_sfu(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

struct AttnPArgs {
    const int32_t *count, *perm, *sig_pos;   // head-group work list
    int T, seq_len, n_kv, rep, qcols, ocols;
    int n_seq, q_tiles;                      // grid: q_tiles x rep x n_seq x n_kv CTAs
    int64_t cache_cap;
    float scale_log2;                        // log2(e) / sqrt(hd)
    __nv_bfloat16 *o_sig;                    // [T][n_q * hd]
    int32_t *status;
};

// Barrier phases: every barrier of a pair alternates by tile (tile t uses
// [t & 1], phase t >> 1), so a waiter for tile t's phase can never see the
// barrier two phases further on: that phase belongs to tile t + 2, whose
// copy or MMA needs a step the waiter itself takes after this wait.
struct __align__(8) ACtl {
    uint64_t bar_q, bar_k[2], bar_v[2], bar_s[2], bar_pv[2];
    uint64_t s_free[2];   // softmax warps have read S buffer b (4 warp arrivals)
    uint64_t p_full;      // softmax warps wrote P and rescaled O (4 warp arrivals)
    uint64_t bar_end;     // error path: every MMA of the issuer has completed
    uint32_t tmem_base;
    int bound[2], pmax;
    int abort;
};
constexpr int kSoftWarps = 4;
constexpr int kMmaWarp = kSoftWarps, kKWarp = kSoftWarps + 1, kVWarp = kSoftWarps + 2;
constexpr int kAttnThreads = 32 * (kSoftWarps + 3);

// Q | K[2] | V[2] | P | control.  No alignment slack: the kernel checks that
// the dynamic shared memory starts 1024-byte aligned (it does when nothing
// else is in shared memory) and reports WIDE_DEV_LAYOUT otherwise, so that
// two CTAs fit one SM.
constexpr uint32_t kOffK = kQTile, kOffV = kOffK + 2 * kKTile, kOffP = kOffV + 2 * kKTile;
constexpr uint32_t kOffCtl = kOffP + kPTile;
constexpr size_t kAttnSmem = kOffCtl + sizeof(ACtl);

// First index i in [0, n) with v[i] >= key (v ascending; n if none), by one
// warp: each round the 32 lanes test 32 evenly spaced entries of the current
// range [lo, hi], which shrinks it about 32-fold (a 4096-entry list takes 3
// rounds of loads instead of the 12 dependent loads of a one-thread search).
// Invariant: v[lo - 1] < key (or lo = 0) and v[hi] >= key (or hi = n).
__device__ __forceinline__ int warp_lower_bound(const int32_t *v, int n, int key, int lane)
{
    int lo = 0, hi = n;
    while (hi > lo) {
        const int step = (hi - lo + 32) / 32;         // 32 probes reach hi
        const int p = lo + (lane + 1) * step - 1;
        const bool ge = p >= hi || v[p] >= key;
        const int f = __ffs(__ballot_sync(0xffffffffu, ge)) - 1;   // lane 31 always tests true
        const int pf = lo + (f + 1) * step - 1;
        hi = min(pf, hi);
        lo += f * step;                                // just past the last probe below key
    }
    return lo;
}

// A bounded wait shared by all warps of the CTA: gives up on timeout (and
// tells the others through ctl->abort) or when another warp gave up.
__device__ __forceinline__ bool attn_wait(uint64_t *bar, uint32_t parity, ACtl *ctl,
                                          int32_t *status)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = globaltimer();
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity))
            return true;
        if (*(volatile int *)&ctl->abort)
            return false;
        if (globaltimer() - t0 > kWaitLimitNs) {
            set_status(status, WIDE_DEV_TIMEOUT);
            *(volatile int *)&ctl->abort = 1;
            return false;
        }
    }
}

__global__ void __launch_bounds__(kAttnThreads, 2)
    prefill_attn(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const AttnPArgs a)
{
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (smem_u32(smem) & 1023u) {
        if (tid == 0)
            set_status(a.status, WIDE_DEV_LAYOUT);
        return;
    }
    uint8_t *sq = smem, *sp = smem + kOffP;
    ACtl *ctl = reinterpret_cast<ACtl *>(smem + kOffCtl);
    // one-dimensional grid, query tile slowest and in descending order: the
    // tiles with the most key steps start first and the short ones fill in
    // at the end (empty tiles, the highest, come first and exit at once)
    const int nsk = a.n_seq * a.n_kv, per_qt = nsk * a.rep;
    const int qt = a.q_tiles - 1 - (int)(blockIdx.x / (unsigned)per_qt);
    const int rem = (int)(blockIdx.x % (unsigned)per_qt);
    const int hh = rem / nsk, s = (rem % nsk) / a.n_kv, j = rem % a.n_kv;
    const int32_t *pj = a.perm + (size_t)j * a.T;

    // this sequence's queries of group j: [lo, hi) of the group's token list
    // (warp 0 finds lo, warp 1 hi, at the same time)
    if (warp < 2) {
        const int r = warp_lower_bound(pj, a.count[j], (s + warp) * a.seq_len, lane);
        if (lane == 0)
            ctl->bound[warp] = r;
    }
    if (tid == 0) {
        ctl->abort = 0;
        mbar_init(&ctl->bar_q, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->bar_k[b], 1);
            mbar_init(&ctl->bar_v[b], 1);
            mbar_init(&ctl->bar_s[b], 1);
            mbar_init(&ctl->bar_pv[b], 1);
            mbar_init(&ctl->s_free[b], kSoftWarps);
        }
        mbar_init(&ctl->p_full, kSoftWarps);
        mbar_init(&ctl->bar_end, 1);
        fence_mbar_init();
    }
    __syncthreads();
    const int lo = ctl->bound[0], nq = ctl->bound[1] - lo;
    if (qt * kBQ >= nq)
        return;  // no query of this group in this tile: nothing to compute
    if (warp == 0) {
        umma::tmem_alloc(&ctl->tmem_base, 256);
        umma::tmem_relinquish();
    } else if (tid == 32) {
        // position of the tile's last query: how far its keys reach
        ctl->pmax = pj[min(lo + nq - 1, lo + (qt + 1) * kBQ - 1)] - s * a.seq_len;
    }
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem = ctl->tmem_base;
    const int pmax = ctl->pmax;
    const uint32_t t_pv = tmem + 128;             // S buffers at columns 0 and 64
    const int64_t kvrow0 = ((int64_t)s * a.n_kv + j) * a.cache_cap;
    const int nkt = pmax / kBKV + 1;

    if (warp == kMmaWarp) {
        // ---------------------------------------- MMA issuer (one lane)
        // Program order S(0), then per t: S(t+1), P(t) V(t).  Each MMA group
        // completes on its own barrier; the issuer never waits for one.
        if (lane == 0) {
            constexpr uint32_t idesc_s = umma::idesc_bf16_f32(kBQ, kBKV);
            constexpr uint32_t idesc_pv = umma::idesc_bf16_f32_bmn(kBQ, kHD);
            const uint32_t q0 = smem_u32(sq), p0 = smem_u32(sp);
            auto issue_s = [&](int t) {
                const uint32_t k0 = smem_u32(smem + kOffK + (t & 1) * kKTile);
#pragma unroll
                for (int k = 0; k < kHD / 16; ++k) {
                    const uint32_t qo = (uint32_t)(k >> 2) * kQHalf + (uint32_t)(k & 3) * 32u;
                    const uint32_t ko = (uint32_t)(k >> 2) * kKHalf + (uint32_t)(k & 3) * 32u;
                    umma::mma_bf16(tmem + (uint32_t)(t & 1) * kBKV,
                                   umma::desc_kmajor_sw128(q0 + qo),
                                   umma::desc_kmajor_sw128(k0 + ko), idesc_s, k != 0);
                }
                umma::commit(&ctl->bar_s[t & 1]);
            };
            // S(t): K(t) landed and the softmax has read S(t-2) (same buffer)
            auto ready_s = [&](int t) {
                return attn_wait(&ctl->bar_k[t & 1], (uint32_t)(t >> 1) & 1u, ctl, a.status) &&
                       (t < 2 || attn_wait(&ctl->s_free[t & 1], (uint32_t)((t - 2) >> 1) & 1u, ctl,
                                           a.status));
            };
            bool ok = attn_wait(&ctl->bar_q, 0, ctl, a.status) && ready_s(0);
            if (ok) {
                umma::fence_after_sync();
                issue_s(0);
            }
            for (int t = 0; t < nkt && ok; ++t) {
                if (t + 1 < nkt) {
                    if (!(ok = ready_s(t + 1)))
                        break;
                    umma::fence_after_sync();
                    issue_s(t + 1);
                }
                // O += P(t) V(t): P(t) written (which the softmax does only
                // after P(t-1) V(t-1) completed) and V(t) landed
                ok = attn_wait(&ctl->p_full, (uint32_t)t & 1u, ctl, a.status) &&
                     attn_wait(&ctl->bar_v[t & 1], (uint32_t)(t >> 1) & 1u, ctl, a.status);
                if (!ok)
                    break;
                const int kmax = a.seq_len - 1 - t * kBKV;   // last valid key row in tile
                uint8_t *sv = smem + kOffV + (t & 1) * kKTile;
                if (kmax < kBKV - 1) {
                    // keys past the sequence's end may be uninitialised cache
                    // memory: clear those V rows so that 0 * garbage cannot
                    // reach P V
                    for (int rr = max(kmax + 1, 0); rr < kBKV; ++rr)
                        for (int c = 0; c < 16; ++c)
                            *reinterpret_cast<uint4 *>(sv + (c >> 3) * kKHalf + rr * 128 +
                                                       (c & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
                    fence_proxy_async_smem();
                }
                umma::fence_after_sync();
                const uint32_t v0 = smem_u32(sv);
#pragma unroll
                for (int k = 0; k < kBKV / 16; ++k) {
                    const uint32_t aoff = (uint32_t)k * 32u;          // 16 keys of the P row
                    const uint32_t boff = (uint32_t)k * 16u * 128u;   // 16 key rows of V
                    umma::mma_bf16(t_pv, umma::desc_kmajor_sw128(p0 + aoff),
                                   umma::desc_mnmajor_sw128(v0 + boff, kKHalf), idesc_pv,
                                   (t | k) != 0);
                }
                umma::commit(&ctl->bar_pv[t & 1]);
            }
            if (!ok) {
                // let every MMA issued so far complete before TMEM is freed
                umma::commit(&ctl->bar_end);
                mbar_wait(&ctl->bar_end, 0);
            }
        }
    } else if (warp == kKWarp || warp == kVWarp) {
        // ---------------------------------------- TMA copies (one lane each)
        // K(t) [V(t)] overwrites the buffer of K(t-2) [V(t-2)] once S(t-2)
        // [P(t-2) V(t-2)] has completed.
        if (lane == 0) {
            const bool is_k = warp == kKWarp;
            const CUtensorMap *tm = is_k ? &tm_k : &tm_v;
            uint8_t *buf0 = smem + (is_k ? kOffK : kOffV);
            uint64_t *full = is_k ? ctl->bar_k : ctl->bar_v;
            uint64_t *done = is_k ? ctl->bar_s : ctl->bar_pv;
            if (is_k) {
                mbar_arrive_expect_tx(&ctl->bar_q, kQTile);
                const int qrow = j * a.T + lo + qt * kBQ;
                tma_load_2d(sq, &tm_q, hh * kHD, qrow, &ctl->bar_q);
                tma_load_2d(sq + kQHalf, &tm_q, hh * kHD + 64, qrow, &ctl->bar_q);
            }
            int n = 0;                   // copies issued
            for (; n < nkt; ++n) {
                if (n >= 2 && !attn_wait(&done[n & 1], (uint32_t)((n - 2) >> 1) & 1u, ctl, a.status))
                    break;
                uint8_t *dst = buf0 + (n & 1) * kKTile;
                const int krow = (int)(kvrow0 + (int64_t)n * kBKV);
                mbar_arrive_expect_tx(&full[n & 1], kKTile);
                tma_load_2d(dst, tm, 0, krow, &full[n & 1]);
                tma_load_2d(dst + kKHalf, tm, 64, krow, &full[n & 1]);
            }
            if (n < nkt) {
                // error path: the last copy into each buffer must land before exit
                for (int t = n - 1; t >= 0 && t >= n - 2; --t)
                    mbar_wait(&full[t & 1], (uint32_t)(t >> 1) & 1u);
                if (is_k)
                    mbar_wait(&ctl->bar_q, 0);
            }
        }
    } else {
        // ---------------------------------------- softmax warps (rows 0..127)
        const int nvalid = min(kBQ, nq - qt * kBQ);
        const int idx = lo + qt * kBQ + tid;          // row of this thread
        const bool live = tid < nvalid;
        const int tok = live ? pj[idx] : 0;
        const int pos = live ? tok - s * a.seq_len : -1;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const float sc = a.scale_log2;
        float m_ref = -INFINITY, l = 0.f;     // row reference max (log2 units), sum
        bool ok = true;
        for (int kt = 0; kt < nkt; ++kt) {
            const int b = kt & 1;
            bool w = attn_wait(&ctl->bar_s[b], (uint32_t)(kt >> 1) & 1u, ctl, a.status);
            if (!__all_sync(0xffffffffu, w)) {
                ok = false;
                break;
            }
            umma::fence_after_sync();
            // this row's 64 scores of the tile; then S buffer b is free
            const uint32_t ts = tmem + (uint32_t)b * kBKV + lane_off;
            float v[kBKV];
            umma::tmem_ld32(ts, *reinterpret_cast<float(*)[32]>(&v[0]));
            umma::tmem_ld32(ts + 32, *reinterpret_cast<float(*)[32]>(&v[32]));
            umma::tmem_ld_wait();
            umma::fence_before_sync();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&ctl->s_free[b]);
            const int k0 = kt * kBKV;
            const bool full = live && k0 + kBKV - 1 <= pos;   // no key of the tile masked
            if (!full) {
#pragma unroll
                for (int e = 0; e < kBKV; ++e)
                    if (!(live && k0 + e <= pos))
                        v[e] = -INFINITY;
            }
            // row max over 8 independent chains
            float vm[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
                vm[e] = v[e];
#pragma unroll
            for (int e = 8; e < kBKV; ++e)
                vm[e & 7] = fmaxf(vm[e & 7], v[e]);
            const float vmax = fmaxf(fmaxf(fmaxf(vm[0], vm[1]), fmaxf(vm[2], vm[3])),
                                     fmaxf(fmaxf(vm[4], vm[5]), fmaxf(vm[6], vm[7])));
            const float mt = vmax * sc;                       // -inf if no key is visible
            // move the reference max when the running max passes it by > 8
            float alpha = 1.f;
            if (mt > m_ref + 8.f) {
                alpha = kt > 0 ? exp2f(m_ref - mt) : 0.f;
                m_ref = mt;
            }
            // probabilities (bf16 pairs) while the previous tile's P V may
            // still run: only storing P and rescaling O wait for it
            const float mb = m_ref > -INFINITY ? m_ref : 0.f;
            float ls[4] = {0.f, 0.f, 0.f, 0.f};
            uint32_t pw[kBKV / 2];
#pragma unroll
            for (int e = 0; e < kBKV; e += 2) {
                const float p0 = exp2_sfu(fmaf(v[e], sc, -mb)),
                            p1 = exp2_sfu(fmaf(v[e + 1], sc, -mb));
                ls[(e >> 1) & 3] += p0 + p1;
                const __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
                pw[e / 2] = *reinterpret_cast<const uint32_t *>(&b2);
            }
            // the previous tile's P V is done: P is free, O is stable
            if (kt > 0) {
                w = attn_wait(&ctl->bar_pv[(kt - 1) & 1], (uint32_t)((kt - 1) >> 1) & 1u, ctl,
                              a.status);
                if (!__all_sync(0xffffffffu, w)) {
                    ok = false;
                    break;
                }
                umma::fence_after_sync();
            }
            if (kt > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
                for (int c = 0; c < kHD / 32; ++c) {
                    float ov[32];
                    umma::tmem_ld32(t_pv + lane_off + c * 32, ov);
                    umma::tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        ov[e] *= alpha;
                    umma::tmem_st32(t_pv + lane_off + c * 32, ov);
                }
                umma::tmem_st_wait();
            }
            // P (bf16, swizzled K-major); masked keys give 0
#pragma unroll
            for (int g8 = 0; g8 < kBKV / 8; ++g8)
                *reinterpret_cast<uint4 *>(sp + swz128(tid, g8)) =
                    make_uint4(pw[4 * g8], pw[4 * g8 + 1], pw[4 * g8 + 2], pw[4 * g8 + 3]);
            l = l * alpha + ((ls[0] + ls[1]) + (ls[2] + ls[3]));
            fence_proxy_async_smem();       // P written by threads, read by the tensor core
            umma::fence_before_sync();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&ctl->p_full);
        }
        if (ok) {
            const bool w = attn_wait(&ctl->bar_pv[(nkt - 1) & 1], (uint32_t)((nkt - 1) >> 1) & 1u,
                                     ctl, a.status);
            ok = __all_sync(0xffffffffu, w);
        }
        if (ok) {
            umma::fence_after_sync();
            // O / l (the TMEM loads are warp-collective)
            const float inv = live ? 1.f / l : 0.f;
            __nv_bfloat16 *dst = a.o_sig + (size_t)(live ? a.sig_pos[tok] : 0) * a.ocols +
                                 (size_t)(j * a.rep + hh) * kHD;
#pragma unroll 1
            for (int c = 0; c < kHD / 32; ++c) {
                float ov[32];
                umma::tmem_ld32(t_pv + lane_off + c * 32, ov);
                umma::tmem_ld_wait();
                if (live) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        __nv_bfloat162 b0 =
                            __floats2bfloat162_rn(ov[q * 8] * inv, ov[q * 8 + 1] * inv);
                        __nv_bfloat162 b1 =
                            __floats2bfloat162_rn(ov[q * 8 + 2] * inv, ov[q * 8 + 3] * inv);
                        __nv_bfloat162 b2 =
                            __floats2bfloat162_rn(ov[q * 8 + 4] * inv, ov[q * 8 + 5] * inv);
                        __nv_bfloat162 b3 =
                            __floats2bfloat162_rn(ov[q * 8 + 6] * inv, ov[q * 8 + 7] * inv);
                        reinterpret_cast<uint4 *>(dst + c * 32)[q] = make_uint4(
                            *reinterpret_cast<uint32_t *>(&b0), *reinterpret_cast<uint32_t *>(&b1),
                            *reinterpret_cast<uint32_t *>(&b2), *reinterpret_cast<uint32_t *>(&b3));
                    }
                }
            }
        }
    }
    umma::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        umma::fence_after_sync();
        umma::tmem_dealloc(tmem, 256);
    }
}

struct PrefillWs {
    char *wl_a;
    __nv_bfloat16 *xn, *qc, *o_sig;
    float *h1;
    char *ffn;
    size_t wl_bytes, total;
};

PrefillWs prefill_ws(const wide_layer_dims *d, void *base)
{
    const size_t T = (size_t)(d->n_seq * d->seq_len);
    const size_t H = (size_t)d->hidden;
    const size_t qd = (size_t)d->n_q_heads * d->head_dim;
    const size_t qcols = qd / d->n_kv_heads;
    PrefillWs w = {};
    char *p = static_cast<char *>(base);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        char *at = p ? p + off : nullptr;
        off += align_up(bytes > 0 ? bytes : 1, 1024);
        return at;
    };
    w.wl_bytes = wide_worklist_bytes((int64_t)T, d->n_kv_heads, kBQ);
    w.wl_a = take(w.wl_bytes);
    w.xn = reinterpret_cast<__nv_bfloat16 *>(take(T * H * 2));
    w.qc = reinterpret_cast<__nv_bfloat16 *>(take((size_t)d->n_kv_heads * T * qcols * 2));
    w.o_sig = reinterpret_cast<__nv_bfloat16 *>(take(T * qd * 2));
    w.h1 = reinterpret_cast<float *>(take(T * H * 4));
    wide_ffn_dims fd = {(int64_t)T, (int64_t)H, d->inter, d->ffn_group_size, WIDE_BF16,
                        WIDE_PATH_PREFILL};
    w.ffn = take(ffn_prefill_workspace(&fd));
    w.total = off;
    return w;
}

}  // namespace

bool layer_prefill_supported(const wide_layer_dims *d)
{
    const int64_t T = d->n_seq * d->seq_len;
    const int rep = d->n_kv_heads > 0 ? d->n_q_heads / d->n_kv_heads : 0;
    return d->cache_len == 0 && d->seq_len >= 1 && T >= 1 && T <= (1 << 24) &&
           d->head_dim == kHD && d->n_kv_heads >= 2 && d->n_kv_heads % 2 == 0 &&
           d->n_kv_heads <= 1024 && (rep == 2 || rep == 4) && d->hidden % 256 == 0 &&
           (d->ffn_group_size == 64 || d->ffn_group_size == 128 ||
            (d->ffn_group_size == 32 && d->inter % 64 == 0)) &&
           d->inter % d->ffn_group_size == 0 && d->inter / d->ffn_group_size <= 1024 &&
           d->cache_cap >= d->seq_len && (int64_t)d->n_kv_heads * T <= (1ll << 31) / 512;
}

size_t layer_prefill_workspace(const wide_layer_dims *d) { return prefill_ws(d, nullptr).total; }

int layer_prefill_launch(const LayerPtrs &p, const wide_layer_dims *d, void *ws, cudaStream_t s)
{
    const int64_t T = d->n_seq * d->seq_len, H = d->hidden;
    const int n_q = d->n_q_heads, n_kv = d->n_kv_heads, rep = n_q / n_kv;
    const int qd = n_q * kHD, qcols = rep * kHD;
    PrefillWs w = prefill_ws(d, ws);
    int rc;

    // 1. head-group mask reordering (no host sync)
    wide_worklist wl;
    if ((rc = wide_worklist_carve(w.wl_a, w.wl_bytes, T, n_kv, kBQ, &wl)))
        return rc;
    if ((rc = reorder_launch(p.head_mask, T, n_kv, kBQ, &wl, s)))
        return rc;

    // 2. attention input norm
    if ((rc = rmsnorm_bf16_launch(p.x, p.gamma1, w.xn, (int)T, (int)H, d->eps, s)))
        return rc;

    // 3. Q for kept (token, group) pairs, compacted per group, RoPE applied
    CUtensorMap tq, tk, tv, tqc, tkc, tvc, to_a, to_b;
    const uint64_t kv_rows = (uint64_t)d->n_seq * n_kv * d->cache_cap;
    if (!make_tmap_2d(&tq, p.wq, qd, H, H, 2, 128, 64, true) ||
        !make_tmap_2d(&tk, p.wk, (uint64_t)n_kv * kHD, H, H, 2, 128, 64, true) ||
        !make_tmap_2d(&tv, p.wv, (uint64_t)n_kv * kHD, H, H, 2, 128, 64, true) ||
        !make_tmap_2d(&tqc, w.qc, (uint64_t)n_kv * T, qcols, qcols, 2, kBQ, 64, true) ||
        !make_tmap_2d(&tkc, p.k_cache, kv_rows, kHD, kHD, 2, kBKV, 64, true) ||
        !make_tmap_2d(&tvc, p.v_cache, kv_rows, kHD, kHD, 2, kBKV, 64, true) ||
        !make_tmap_2d(&to_a, w.o_sig, T, qd, qd, 2, 128, 64, true) ||
        !make_tmap_2d(&to_b, p.wo, H, qd, qd, 2, 256, 64, true))
        return WIDE_CUDA_FAIL();
    const float log2_theta = log2f(d->rope_theta);
    GemmArgs ga = {};
    ga.a = w.xn;
    ga.count = wl.count;
    ga.perm = wl.perm;
    ga.items = wl.items;
    ga.n_items_p = wl.n_items;
    ga.sig_pos = wl.sig_pos;
    ga.out0 = w.qc;
    ga.T = (int)T;
    ga.K = (int)H;
    ga.group_cols = qcols;
    ga.seq_len = (int)d->seq_len;
    ga.n_kv = n_kv;
    ga.cache_len = 0;
    ga.cache_cap = d->cache_cap;
    ga.log2_theta = log2_theta;
    ga.status = status_ptr();
    const int m_tiles = (int)((T + 127) / 128);
    if ((rc = gather_gemm_launch(GEMM_ROPE_Q, tq, tq, ga, (qcols / 256) * n_kv * m_tiles,
                                 KID_PREFILL_Q, s)))
        return rc;

    // 4. K and V for every token, RoPE on K, into the caches
    GemmArgs gk = ga;
    gk.out0 = static_cast<__nv_bfloat16 *>(p.k_cache);
    gk.out1 = static_cast<__nv_bfloat16 *>(p.v_cache);
    gk.kv_blocks = n_kv;          // n_kv/2 blocks of two K heads, then of two V heads
    gk.m_tiles = m_tiles;
    if ((rc = gather_gemm_launch(GEMM_KV, tk, tv, gk, n_kv * m_tiles, KID_PREFILL_KV, s)))
        return rc;

    // 5. attention on compacted queries -> o_sig (rows of kept pairs only)
    AttnPArgs aa;
    aa.count = wl.count;
    aa.perm = wl.perm;
    aa.sig_pos = wl.sig_pos;
    aa.T = (int)T;
    aa.seq_len = (int)d->seq_len;
    aa.n_kv = n_kv;
    aa.rep = rep;
    aa.n_seq = (int)d->n_seq;
    aa.q_tiles = (int)((d->seq_len + kBQ - 1) / kBQ);
    aa.qcols = qcols;
    aa.ocols = qd;
    aa.cache_cap = d->cache_cap;
    aa.scale_log2 = kLog2e / sqrtf((float)kHD);
    aa.o_sig = w.o_sig;
    aa.status = status_ptr();
    if (!raise_smem_limit(reinterpret_cast<const void *>(prefill_attn), kAttnSmem))
        return WIDE_CUDA_FAIL();
    {
        LaunchScope scope(KID_PREFILL_ATTN, s);
        const unsigned grid = (unsigned)aa.q_tiles * (unsigned)rep * (unsigned)(d->n_seq * n_kv);
        prefill_attn<<<grid, kAttnThreads, kAttnSmem, s>>>(tqc, tkc, tvc, aa);
    }
    if ((rc = launch_status()))
        return rc;

    // 6. o_proj over each signature tile's kept groups; h1 = x + attn (fp32)
    UnionArgs ua = {};
    ua.tile_union = wl.tile_union;
    ua.sig_perm = wl.sig_perm;
    ua.mask = p.head_mask;
    ua.h = w.o_sig;
    ua.T = (int)T;
    ua.N = (int)H;
    ua.W = (n_kv + 31) / 32;
    ua.gs = qcols;
    ua.ld = qd;
    ua.out_sum = static_cast<__nv_bfloat16 *>(p.attn_out);
    if (p.ffn) {
        ua.res_in = static_cast<const __nv_bfloat16 *>(p.x);
        ua.out_total_f32 = w.h1;
    }
    ua.status = status_ptr();
    if ((rc = tile_union_gemm_launch(to_a, to_b, ua, KID_PREFILL_OPROJ, s)) || !p.ffn)
        return rc;

    // 7. FFN input norm, masked FFN, out = h1 + ffn_out
    if ((rc = rmsnorm_f32_launch(w.h1, p.gamma2, w.xn, (int)T, (int)H, d->eps, s)))
        return rc;
    FfnPrefillOut fo = {};
    fo.out_sum = static_cast<__nv_bfloat16 *>(p.ffn_out);
    fo.res_f32 = w.h1;
    fo.out_total = static_cast<__nv_bfloat16 *>(p.out);
    return ffn_prefill_core(w.xn, p.w_gate, p.w_up, p.w_down, p.ffn_mask, fo, T, H, d->inter,
                            d->ffn_group_size, nullptr, w.ffn, s);
}

}  // namespace wide
