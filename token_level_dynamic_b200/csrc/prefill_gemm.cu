// prefill_gemm.cu -- the tcgen05 grouped GEMMs of the prefill path.
//
// WIDE, technical summary section 2.B: after mask reordering, the active
// tokens of group g are the prefix perm[g][0 : count[g]), so each group is a
// dense GEMM over ceil(count[g] / 128) row tiles with a known active prefix;
// section 2.C: tiles with no active token are never issued (block-level
// skip) and rows past the active prefix are not loaded (load-stage skip).
//
// gather_gemm<mode>: persistent, warp-specialised, M=128 x N=256 tiles.
//   warp 0     weight producer: two 128-row TMA tiles (128-byte swizzle) per
//              64-column K stage
//   warp 1     TMEM owner (512 columns: two 256-column fp32 accumulators, so
//              the epilogue of one tile overlaps the MMAs of the next) and
//              single-thread tcgen05.mma issuer
//   warps 2-5  epilogue (warp w reads TMEM lanes 32 * (w % 4) .. +31)
//   warps 6-7  row gather: 16-byte cp.async copies of the tile's token rows
//              straight into the swizzled operand layout, 8 consecutive lanes
//              per 128-byte row piece so each warp instruction makes 4
//              coalesced requests; each thread's copy completions arrive on
//              the stage barrier
//   modes
//     Router  dense: every 128-token tile of x (one TMA box per K stage;
//             the gather warps only arrive) times all of W_r1 (N = the
//             bottleneck width); epilogue: activation, W_r2 products and
//             the packed execute bits (router_epilogue)
//     SwiGLU  work item (g, i) of the FFN work list; B = [W_gate[g]; W_up[g]]
//             (N = 2 gs: 256 for 128-channel groups, 128 for 64);
//             epilogue h = silu(gate) * up, stored bf16 at the token's
//             signature-order row of H.
//     RopeQ   work item (j, i) of the head-group work list, 256-column part
//             hf of the group (group_cols / 256 parts); B = 256 rows of Wq
//             for two query heads of group j; epilogue RoPE,
//             stored bf16 at row i*128 + r of group j's compacted q buffer.
//     KV      dense: every token tile times 256 rows of Wk (two KV heads,
//             RoPE in the epilogue) or Wv; stored into the caches.
// tile_union_gemm: persistent, M=128 tokens of one signature tile x N=256
//   outputs; the K loop visits only the groups (gs columns each) in the
//   tile's union of kept groups (block-level skip).  Warp 0 loads the A tile
//   (the tokens' rows of H, stored in signature order) and the weight tile
//   (B) by TMA; warps 6-7 then overwrite, in shared memory, the rows whose
//   token skips the group with zeros before the stage goes to the MMA, so
//   those rows contribute nothing and H entries of skipped pairs are never
//   written (no zeroing pass over H in HBM).  Gathering only the active rows
//   with 16-byte cp.async copies instead (source size 0 for a skipped row)
//   measured 1.8x slower on the 8B FFN: H streams from DRAM, and per-thread
//   copies behind a 4-stage ring do not cover that latency the way TMA
//   boxes do.  Epilogue: projection and/or projection plus residuals (bf16
//   and fp32), written at the tokens' own rows.
//
// Every mbarrier wait is bounded; on expiry the kernel records
// WIDE_DEV_TIMEOUT, drains what it issued (bounded), frees TMEM and returns.
#include "common.cuh"
#include "host.h"
#include "umma.cuh"

namespace wide {
namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kBN = 256;
constexpr int kStages = 4;
constexpr uint32_t kATile = kBM * 128;
constexpr uint32_t kBTile = kBN * 128;
constexpr uint32_t kStageBytes = kATile + kBTile;
// The router with a bottleneck of at most 128 rows splits the same ring bytes
// into 6 slots of 32 KB (A tile + 128-row B tile).  Measured as fast as 4
// slots of 48 KB: the router's time is not set by the ring depth.
constexpr int kRouterStages = 6;
constexpr uint32_t kRouterStageBytes = kATile + 128u * 128u;
constexpr int kMaxStages = 6;
static_assert(kRouterStages * kRouterStageBytes <= kStages * kStageBytes, "router ring");
constexpr int kThreadsDown = 256;
constexpr int kThreadsGather = 256;
constexpr int kGatherThreads = 64;
constexpr uint32_t kTmemCols = 512;
constexpr int kHD = 128;

struct __align__(8) Ctl {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t drain;
    uint64_t fixed[kMaxStages];   // tile_union_gemm: skipped rows zeroed
    uint32_t tmem_base;
    int abort;
    int trow[2][kBM / 2]; // gather warp w: offsets of its rows' tokens (-1: none)
};

constexpr size_t kSmemBytes = 1024 + kStages * kStageBytes + sizeof(Ctl);

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    const uint32_t a = smem_u32(p);
    return p + (((a + 1023u) & ~1023u) - a);
}

__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, Ctl *ctl,
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

__device__ __forceinline__ void store_bf16x32(__nv_bfloat16 *dst, const float (&v)[32])
{
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        __nv_bfloat162 p = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t *>(&p);
    }
    uint4 *d = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i)
        d[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
}

__device__ __forceinline__ void init_ctl(Ctl *ctl, uint32_t full_count)
{
    for (int s = 0; s < kMaxStages; ++s) {
        mbar_init(&ctl->full[s], full_count);
        mbar_init(&ctl->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
        mbar_init(&ctl->tfull[a], 1);
        mbar_init(&ctl->tempty[a], 128);
    }
    mbar_init(&ctl->drain, 1);
    ctl->abort = 0;
    fence_mbar_init();
}

// Rotate-half RoPE of a head held as 128 fp32 TMEM columns starting at
// taddr; writes the rotated head as bf16 to dst[0..127].  Angles are
// pos * theta^(-2p/128) in fp32, p the pair index.
__device__ __forceinline__ void rope_head_store(uint32_t taddr, int pos, float log2_theta,
                                                __nv_bfloat16 *dst, bool store)
{
#pragma unroll 1
    for (int cc = 0; cc < 2; ++cc) {
        float x1[32], x2[32];
        umma::tmem_ld32(taddr + cc * 32, x1);
        umma::tmem_ld32(taddr + 64 + cc * 32, x2);
        umma::tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            const int p = cc * 32 + e;
            const float inv = exp2f(-(float)(2 * p) / (float)kHD * log2_theta);
            float sn, cs;
            sincosf((float)pos * inv, &sn, &cs);
            const float a = x1[e], b = x2[e];
            x1[e] = a * cs - b * sn;
            x2[e] = b * cs + a * sn;
        }
        if (store) {
            store_bf16x32(dst + cc * 32, x1);
            store_bf16x32(dst + 64 + cc * 32, x2);
        }
    }
}

__device__ __forceinline__ void copy_head_store(uint32_t taddr, __nv_bfloat16 *dst, bool store)
{
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
        float v[32];
        umma::tmem_ld32(taddr + cc * 32, v);
        umma::tmem_ld_wait();
        if (store)
            store_bf16x32(dst + cc * 32, v);
    }
}

// Router epilogue.  A W_r2 block is 32 groups x 32 bottleneck units; lane l
// of a warp loads group (32 wd + l)'s 64 bytes of chunk c (zeros past G).
__device__ __forceinline__ void w2_block_load(const GemmArgs &a, int wd, int c, int lane,
                                              uint4 (&v)[4])
{
    const int g = wd * 32 + lane;
    if (g < a.n_groups) {
        const uint4 *p = reinterpret_cast<const uint4 *>(a.w_r2 + (size_t)g * a.rn + c * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q)
            v[q] = __ldg(p + q);
    } else {
#pragma unroll
        for (int q = 0; q < 4; ++q)
            v[q] = make_uint4(0u, 0u, 0u, 0u);
    }
}

// One token row (TMEM lane) per thread: z = act(the row's rn accumulator
// columns), logit[g] = b_r2[g] + z . W_r2[g], execute bit = logit > 0.  Each
// thread builds its token's mask words itself, 32 groups at a time; the z
// chunks are re-read from TMEM for every word.  W_r2 goes through this
// warp's own fp32 block in shared memory (rows of kRW2Stride floats, so the
// lanes' row stores hit distinct banks; the FMA loop reads it as broadcasts),
// and the next block is fetched into registers while this one is used.
// Packed fp32x2 FMAs keep even and odd bottleneck units in two partial sums.
// Called by whole warps (tcgen05.ld is warp-collective); only live rows store.
constexpr int kRW2Stride = 36;
constexpr uint32_t kRouterScratch = 4u * 32u * kRW2Stride * 4u + 16u;
static_assert(kSmemBytes + kRouterScratch <= 232448, "router mode exceeds 227 KB of shared memory");

__device__ __forceinline__ void router_epilogue(const GemmArgs &a, uint32_t taddr, int t,
                                                bool live, float *ws, int lane)
{
    const int G = a.n_groups, nw = (G + 31) >> 5, nc = a.rn >> 5, nblk = nw * nc;
    uint4 nx[4];
    w2_block_load(a, 0, 0, lane, nx);
#pragma unroll 1
    for (int wd = 0; wd < nw; ++wd) {
        const int g0 = wd * 32;
        const int ng = min(32, G - g0);
        float2 acc[32];
#pragma unroll
        for (int j = 0; j < 32; ++j)
            acc[j] = make_float2((a.b_r2 && j < ng) ? __ldg(a.b_r2 + g0 + j) : 0.f, 0.f);
#pragma unroll 1
        for (int c = 0; c < nc; ++c) {
            __syncwarp();
            float *row = ws + lane * kRW2Stride;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float f[8];
                bf16x8_to_f32(nx[q], f);
                *reinterpret_cast<float4 *>(row + 8 * q) = make_float4(f[0], f[1], f[2], f[3]);
                *reinterpret_cast<float4 *>(row + 8 * q + 4) = make_float4(f[4], f[5], f[6], f[7]);
            }
            __syncwarp();
            const int nb = wd * nc + c + 1;
            if (nb < nblk)
                w2_block_load(a, nb / nc, nb % nc, lane, nx);
            float z[32];
            umma::tmem_ld32(taddr + c * 32, z);
            umma::tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e)
                z[e] = a.act == WIDE_ACT_SILU ? silu_f32(z[e]) : fmaxf(z[e], 0.f);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float4 *wr = reinterpret_cast<const float4 *>(ws + j * kRW2Stride);
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4) {
                    const float4 w = wr[e4];
                    acc[j] = __ffma2_rn(make_float2(z[4 * e4], z[4 * e4 + 1]),
                                        make_float2(w.x, w.y), acc[j]);
                    acc[j] = __ffma2_rn(make_float2(z[4 * e4 + 2], z[4 * e4 + 3]),
                                        make_float2(w.z, w.w), acc[j]);
                }
            }
        }
        uint32_t bits = 0;
        float lg[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            lg[j] = acc[j].x + acc[j].y;
            if (j < ng && lg[j] > 0.f)
                bits |= 1u << j;
        }
        if (live) {
            a.mask_out[(size_t)t * nw + wd] = bits;
            if (a.logits_out) {
                float *lo = a.logits_out + (size_t)t * G + g0;
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (j < ng)
                        lo[j] = lg[j];
            }
        }
    }
}

// --------------------------------------------------------- gather_gemm
struct Work {
    int g, base, nrows, hf, nb;
};

template <int MODE>
__device__ __forceinline__ int n_work(const GemmArgs &a, int n_items)
{
    if (MODE == GEMM_SWIGLU)
        return n_items;
    if (MODE == GEMM_ROPE_Q)
        return (a.group_cols / kBN) * n_items;    // 256-column parts per group
    if (MODE == GEMM_ROUTER)
        return a.m_tiles;
    return a.kv_blocks * a.m_tiles;
}

template <int MODE>
__device__ __forceinline__ Work decode_work(const GemmArgs &a, int it)
{
    Work w;
    w.hf = 0;
    w.nb = 0;
    if (MODE == GEMM_KV || MODE == GEMM_ROUTER) {
        w.nb = it / a.m_tiles;
        const int ti = it % a.m_tiles;
        w.g = 0;
        w.base = ti * kBM;
        w.nrows = min(kBM, a.T - w.base);
        return w;
    }
    int item = it;
    if (MODE == GEMM_ROPE_Q) {
        const int parts = a.group_cols / kBN;
        item = it / parts;
        w.hf = it % parts;
    }
    w.g = a.items[2 * item];
    w.base = a.items[2 * item + 1] * kBM;
    w.nrows = min(kBM, a.count[w.g] - w.base);
    return w;
}

// token of tile row r (r < nrows)
template <int MODE>
__device__ __forceinline__ int row_token(const GemmArgs &a, const Work &w, int r)
{
    if (MODE == GEMM_KV || MODE == GEMM_ROUTER)
        return w.base + r;
    return a.perm[(size_t)w.g * a.T + w.base + r];
}

template <int MODE>
__global__ void __launch_bounds__(kThreadsGather, 1)
    gather_gemm(const __grid_constant__ CUtensorMap tm0, const __grid_constant__ CUtensorMap tm1,
                const GemmArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    Ctl *ctl = reinterpret_cast<Ctl *>(smem + kStages * kStageBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_items = (MODE == GEMM_KV || MODE == GEMM_ROUTER) ? 0 : *a.n_items_p;
    const int nw = n_work<MODE>(a, n_items);
    const int KT = a.K / kBK;
    // ring: kStages slots of kStageBytes, or the router's 6 smaller slots
    const bool small_slots = MODE == GEMM_ROUTER && a.rn <= 128;
    const uint32_t nst = small_slots ? (uint32_t)kRouterStages : (uint32_t)kStages;
    const uint32_t sbytes = small_slots ? kRouterStageBytes : kStageBytes;

    if (threadIdx.x == 0) {
        // one arrive (with the weight bytes) from the producer plus one
        // cp.async-completion arrive from each gather thread
        init_ctl(ctl, 1 + kGatherThreads);
        tma_prefetch_desc(&tm0);
        tma_prefetch_desc(&tm1);
    }
    if (warp == 1) {
        umma::tmem_alloc(&ctl->tmem_base, kTmemCols);
        umma::tmem_relinquish();
    }
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem = ctl->tmem_base;

    if (warp == 0) {
        // -------------------------------------------- weight producer
        uint32_t stage = 0, phase = 0, issued = 0;
        bool ok = true;
        for (int it = blockIdx.x; it < nw && ok; it += gridDim.x) {
            const Work w = decode_work<MODE>(a, it);
            const CUtensorMap *m0 = &tm0, *m1 = &tm1;
            int r0, r1;
            uint32_t b_rows = kBN;                           // rows of the B tile
            if (MODE == GEMM_SWIGLU) {
                r0 = r1 = w.g * a.gs;                        // [W_gate[g]; W_up[g]]
                b_rows = 2 * a.gs;
            } else if (MODE == GEMM_ROPE_Q) {
                r0 = w.g * a.group_cols + w.hf * kBN;        // two query heads of group g
                r1 = r0 + 128;
                m1 = &tm0;
            } else if (MODE == GEMM_ROUTER) {
                r0 = 0;                                      // all of W_r1, two halves
                r1 = a.rn / 2;
                m1 = &tm0;
                b_rows = a.rn;
            } else {
                const int half = a.kv_blocks / 2;            // first half: Wk, then Wv
                const bool is_k = w.nb < half;
                m0 = m1 = is_k ? &tm0 : &tm1;
                r0 = (is_k ? w.nb : w.nb - half) * kBN;
                r1 = r0 + 128;
            }
            for (int kt = 0; kt < KT && ok; ++kt) {
                if (lane == 0) {
                    if (!wait_or_abort(&ctl->empty[stage], phase ^ 1u, ctl, a.status)) {
                        ok = false;
                    } else {
                        uint8_t *b = smem + stage * sbytes + kATile;
                        // router: the token rows are contiguous, so the A tile
                        // is one TMA box of x as well (rows past T read zeros)
                        mbar_arrive_expect_tx(&ctl->full[stage],
                                              b_rows * 128u + (MODE == GEMM_ROUTER ? kATile : 0u));
                        if (MODE == GEMM_ROUTER)
                            tma_load_2d(smem + stage * sbytes, &tm1, kt * kBK, w.base,
                                        &ctl->full[stage]);
                        tma_load_2d(b, m0, kt * kBK, r0, &ctl->full[stage]);
                        tma_load_2d(b + b_rows * 64u, m1, kt * kBK, r1, &ctl->full[stage]);
                        ++issued;
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (++stage == nst) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (!ok && lane == 0) {
            for (uint32_t s = 0; s < nst && s < issued; ++s) {
                const uint32_t uses = (issued - s + nst - 1) / nst;
                mbar_wait(&ctl->full[s], (uses - 1u) & 1u);
            }
        }
    } else if (warp >= 6) {
        // -------------------------------------------- token-row gather
        // gather warp gw, lane l copies chunk l % 8 of rows 4 gw + l / 8 + 8 i
        // (i < 16) of each stage: lanes 8j .. 8j+7 cover one 128-byte row
        // piece.  Each warp looks up its own rows' tokens, so the two warps
        // never wait for each other; wait results are made warp-uniform.
        const int gw = warp - 6, lq = lane >> 3, cc = lane & 7;
        const int lr = 4 * gw + lq;
        int *trow = ctl->trow[gw];
        uint32_t stage = 0, phase = 0;
        bool ok = true;
        for (int it = blockIdx.x; it < nw && ok; it += gridDim.x) {
            const Work w = decode_work<MODE>(a, it);
            __syncwarp();
            for (int x = lane; x < kBM / 2; x += 32) {
                const int r = (x >> 2) * 8 + 4 * gw + (x & 3);
                // router: A arrives by TMA; these warps only arrive per stage
                trow[x] = (MODE != GEMM_ROUTER && r < w.nrows) ? row_token<MODE>(a, w, r) * a.K
                                                                : -1;
            }
            __syncwarp();
            int off[kBM / 8];
#pragma unroll
            for (int i = 0; i < kBM / 8; ++i)
                off[i] = trow[i * 4 + lq];
            for (int kt = 0; kt < KT; ++kt) {
                const bool got = wait_or_abort(&ctl->empty[stage], phase ^ 1u, ctl, a.status);
                if (!__all_sync(0xffffffffu, got)) {
                    ok = false;
                    break;
                }
                const uint32_t sa = smem_u32(smem + stage * sbytes);
                const __nv_bfloat16 *src = a.a + kt * kBK + 8 * cc;
#pragma unroll
                for (int i = 0; i < kBM / 8; ++i)
                    if (off[i] >= 0)
                        cp_async16(sa + swz128(lr + 8 * i, cc), src + off[i]);
                cp_async_arrive_noinc(&ctl->full[stage]);
                if (++stage == nst) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        cp_async_wait_all();
    } else if (warp == 1) {
        // -------------------------------------------- MMA issuer
        // SwiGLU: N = gate rows + up rows of one group (2 gs); router: the
        // bottleneck width; else 256
        const uint32_t nd = MODE == GEMM_SWIGLU   ? 2u * (uint32_t)a.gs
                            : MODE == GEMM_ROUTER ? (uint32_t)a.rn
                                                  : (uint32_t)kBN;
        const uint32_t idesc = umma::idesc_bf16_f32(kBM, nd);
        // MMA-stage skip: a group's tile with at most 64 active tokens (its
        // rows are the tile's first rows) runs M = 64 MMAs
        const uint32_t idesc64 = umma::idesc_bf16_f32(64, nd);
        uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
        bool ok = true;
        for (int it = blockIdx.x; it < nw && ok; it += gridDim.x) {
            if (lane == 0) {
                const bool m64 = (MODE == GEMM_SWIGLU || MODE == GEMM_ROPE_Q) &&
                                 decode_work<MODE>(a, it).nrows <= 64;
                const uint32_t id = m64 ? idesc64 : idesc;
                if (!wait_or_abort(&ctl->tempty[acc], acc_phase ^ 1u, ctl, a.status))
                    ok = false;
                umma::fence_after_sync();
                const uint32_t d = tmem + acc * (uint32_t)kBN;
                for (int kt = 0; kt < KT && ok; ++kt) {
                    if (!wait_or_abort(&ctl->full[stage], phase, ctl, a.status)) {
                        ok = false;
                        break;
                    }
                    // the A tile was written by cp.async (generic proxy) and
                    // is read by the tensor core (async proxy)
                    fence_proxy_async_smem();
                    umma::fence_after_sync();
                    const uint32_t sa = smem_u32(smem + stage * sbytes);
                    const uint32_t sb = sa + kATile;
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k)
                        umma::mma_bf16(d, umma::desc_kmajor_sw128(sa + 32u * k),
                                       umma::desc_kmajor_sw128(sb + 32u * k), id,
                                       (kt | k) != 0);
                    umma::commit(&ctl->empty[stage]);
                    if (++stage == nst) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok)
                    umma::commit(&ctl->tfull[acc]);
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
        if (lane == 0) {
            umma::commit(&ctl->drain);
            mbar_wait(&ctl->drain, 0);
        }
        __syncwarp();
    } else {
        // -------------------------------------------- epilogue (warps 2-5)
        const int q = warp & 3;
        uint32_t acc = 0, acc_phase = 0;
        for (int it = blockIdx.x; it < nw; it += gridDim.x) {
            const Work w = decode_work<MODE>(a, it);
            // tile row of this thread: the TMEM lane at M = 128; at M = 64
            // (tiles of at most 64 rows) row m sits in lane (m % 16) + 32 (m /
            // 16), so lanes 0..15 of warp q hold rows 16 q .. 16 q + 15
            const bool m64 = (MODE == GEMM_SWIGLU || MODE == GEMM_ROPE_Q) && w.nrows <= 64;
            const int r = m64 ? (lane < 16 ? q * 16 + lane : kBM) : q * 32 + lane;
            const bool live = r < w.nrows;
            const int t = live ? row_token<MODE>(a, w, r) : 0;
            if (!wait_or_abort(&ctl->tfull[acc], acc_phase, ctl, a.status))
                break;
            umma::fence_after_sync();
            const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + acc * (uint32_t)kBN;
            if (MODE == GEMM_SWIGLU) {
                __nv_bfloat16 *dst = a.out0 + (size_t)(live ? a.sig_pos[t] : 0) * a.out_ld +
                                     (size_t)w.g * a.gs;
#pragma unroll 1
                for (int c = 0; c < a.gs / 32; ++c) {
                    float gv[32], uv[32];
                    umma::tmem_ld32(taddr + c * 32, gv);
                    umma::tmem_ld32(taddr + a.gs + c * 32, uv);
                    umma::tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        gv[e] = silu_f32(gv[e]) * uv[e];
                    if (live)
                        store_bf16x32(dst + c * 32, gv);
                }
            } else if (MODE == GEMM_ROUTER) {
                // this warp's W_r2 block in shared memory, after the Ctl block
                float *ws = reinterpret_cast<float *>(
                                smem + ((kStages * kStageBytes + sizeof(Ctl) + 15) & ~(size_t)15)) +
                            q * 32 * kRW2Stride;
                if (__any_sync(0xffffffffu, live))
                    router_epilogue(a, taddr, t, live, ws, lane);
            } else if (MODE == GEMM_ROPE_Q) {
                const int pos = (int)(t % a.seq_len + a.cache_len);
                __nv_bfloat16 *dst = a.out0 + ((size_t)w.g * a.T + w.base + r) * a.group_cols +
                                     (size_t)w.hf * kBN;
                rope_head_store(taddr, pos, a.log2_theta, dst, live);
                rope_head_store(taddr + kHD, pos, a.log2_theta, dst + kHD, live);
            } else {
                const int half = a.kv_blocks / 2;
                const bool is_k = w.nb < half;
                const int seq = t / a.seq_len;
                const int pos = (int)(t % a.seq_len + a.cache_len);
                __nv_bfloat16 *cache = is_k ? a.out0 : a.out1;
#pragma unroll 1
                for (int h = 0; h < 2; ++h) {
                    const int kvh = (is_k ? w.nb : w.nb - half) * 2 + h;
                    __nv_bfloat16 *dst =
                        cache + (((size_t)seq * a.n_kv + kvh) * (size_t)a.cache_cap + pos) * kHD;
                    if (is_k)
                        rope_head_store(taddr + h * kHD, pos, a.log2_theta, dst, live);
                    else
                        copy_head_store(taddr + h * kHD, dst, live);
                }
            }
            umma::fence_before_sync();
            mbar_arrive(&ctl->tempty[acc]);
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    }

    umma::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        umma::fence_after_sync();
        umma::tmem_dealloc(tmem, kTmemCols);
    }
}

// ----------------------------------------------------- tile_union_gemm
__global__ void __launch_bounds__(kThreadsDown, 1)
    tile_union_gemm(const __grid_constant__ CUtensorMap tm_a,
                    const __grid_constant__ CUtensorMap tm_b, const UnionArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    Ctl *ctl = reinterpret_cast<Ctl *>(smem + kStages * kStageBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_sig = (a.T + kBM - 1) / kBM;
    const int n_tiles = n_sig * (a.N / kBN);
    // K stages per group; 32-channel groups go in pairs (2p, 2p + 1), one
    // 64-column stage per pair that holds either group (the pair's word bits
    // folded onto the even bit)
    const bool pairs = a.gs == 32;
    const int spg = pairs ? 1 : a.gs / kBK;
    auto stage_bits = [&](uint32_t bits) {
        return pairs ? (bits | (bits >> 1)) & 0x55555555u : bits;
    };

    if (threadIdx.x == 0) {
        // full: the producer's arrive with the A and B bytes; fixed: one
        // arrive per zero-filling thread once its rows of the stage are done
        init_ctl(ctl, 1);
        for (int st = 0; st < kStages; ++st)
            mbar_init(&ctl->fixed[st], kGatherThreads);
        fence_mbar_init();
        tma_prefetch_desc(&tm_a);
        tma_prefetch_desc(&tm_b);
    }
    if (warp == 1) {
        umma::tmem_alloc(&ctl->tmem_base, kTmemCols);
        umma::tmem_relinquish();
    }
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem = ctl->tmem_base;

    // all signature tiles of one output block, then the next block, so that
    // concurrently running CTAs share the weight slab
    auto coords = [&](int tile, int &s, int &nb) {
        nb = tile / n_sig;
        s = tile % n_sig;
    };
    auto uword = [&](int s, int w) { return a.tile_union[(size_t)s * a.W + w]; };

    if (warp == 0) {
        // -------------------------------------------- weight producer
        uint32_t stage = 0, phase = 0, issued = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
            int s, nb;
            coords(tile, s, nb);
            for (int w = 0; w < a.W && ok; ++w) {
                uint32_t bits = stage_bits(uword(s, w));
                while (bits && ok) {
                    const int g = w * 32 + __ffs(bits) - 1;
                    bits &= bits - 1u;
                    for (int sub = 0; sub < spg && ok; ++sub) {
                        if (lane == 0) {
                            if (!wait_or_abort(&ctl->empty[stage], phase ^ 1u, ctl, a.status)) {
                                ok = false;
                            } else {
                                uint8_t *sa = smem + stage * kStageBytes;
                                mbar_arrive_expect_tx(&ctl->full[stage], kStageBytes);
                                const int col = g * a.gs + sub * kBK;
                                tma_load_2d(sa, &tm_a, col, s * kBM, &ctl->full[stage]);
                                tma_load_2d(sa + kATile, &tm_b, col, nb * kBN, &ctl->full[stage]);
                                ++issued;
                            }
                        }
                        ok = __shfl_sync(0xffffffffu, ok, 0);
                        if (++stage == kStages) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                }
            }
        }
        if (!ok && lane == 0) {
            for (uint32_t s = 0; s < kStages && s < issued; ++s) {
                const uint32_t uses = (issued - s + kStages - 1) / kStages;
                mbar_wait(&ctl->full[s], (uses - 1u) & 1u);
            }
        }
    } else if (warp >= 6) {
        // -------------------------------------------- skipped rows to zero
        // warp gw, lane l handles chunk l % 8 of rows 4 gw + l / 8 + 8 i
        // (i < 16) of each stage (lanes 8j .. 8j+7 cover one 128-byte row
        // piece).  Row r of signature tile s is H row s * 128 + r; its token
        // sig_perm[s * 128 + r] decides, per group, whether the loaded row
        // stays or is overwritten with zeros (rows past T too: the TMA box
        // already read zeros there).
        const int gw = warp - 6, lq = lane >> 3, cc = lane & 7;
        const int lr = 4 * gw + lq;
        uint32_t stage = 0, phase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
            int s, nb;
            coords(tile, s, nb);
            int tok[kBM / 8];
#pragma unroll
            for (int i = 0; i < kBM / 8; ++i) {
                const int sr = s * kBM + lr + 8 * i;
                tok[i] = sr < a.T ? a.sig_perm[sr] : -1;
            }
            for (int w = 0; w < a.W && ok; ++w) {
                uint32_t bits = stage_bits(uword(s, w));
                if (!bits)
                    continue;
                uint32_t mw[kBM / 8];
#pragma unroll
                for (int i = 0; i < kBM / 8; ++i)
                    mw[i] = tok[i] >= 0 ? a.mask[(size_t)tok[i] * a.W + w] : 0u;
                while (bits && ok) {
                    const int gb = __ffs(bits) - 1;
                    bits &= bits - 1u;
                    for (int sub = 0; sub < spg; ++sub) {
                        const bool got = wait_or_abort(&ctl->full[stage], phase, ctl, a.status);
                        if (!__all_sync(0xffffffffu, got)) {
                            ok = false;
                            break;
                        }
                        uint8_t *sa = smem + stage * kStageBytes;
                        // chunk cc holds channels 8 cc .. 8 cc + 7 of the
                        // stage: of group gb, or with 32-channel pairs of
                        // group gb + cc / 4
                        const int gbit = pairs ? gb + (cc >> 2) : gb;
#pragma unroll
                        for (int i = 0; i < kBM / 8; ++i)
                            if (!((mw[i] >> gbit) & 1u))
                                *reinterpret_cast<uint4 *>(sa + swz128(lr + 8 * i, cc)) =
                                    make_uint4(0u, 0u, 0u, 0u);
                        // the zeros are written by the generic proxy and read
                        // by the tensor core (async proxy)
                        fence_proxy_async_smem();
                        mbar_arrive(&ctl->fixed[stage]);
                        if (++stage == kStages) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                }
            }
        }
    } else if (warp == 1) {
        constexpr uint32_t idesc = umma::idesc_bf16_f32(kBM, kBN);
        uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
            int s, nb;
            coords(tile, s, nb);
            if (lane == 0) {
                if (!wait_or_abort(&ctl->tempty[acc], acc_phase ^ 1u, ctl, a.status))
                    ok = false;
                umma::fence_after_sync();
                const uint32_t d = tmem + acc * (uint32_t)kBN;
                int kstep = 0;
                for (int w = 0; w < a.W && ok; ++w) {
                    const int nsteps = __popc(stage_bits(uword(s, w))) * spg;
                    for (int n = 0; n < nsteps && ok; ++n) {
                        // fixed completes once the zero-filling warps (which
                        // waited for full) are done with the stage
                        if (!wait_or_abort(&ctl->fixed[stage], phase, ctl, a.status)) {
                            ok = false;
                            break;
                        }
                        umma::fence_after_sync();
                        const uint32_t sa = smem_u32(smem + stage * kStageBytes);
                        const uint32_t sb = sa + kATile;
#pragma unroll
                        for (int k = 0; k < kBK / 16; ++k)
                            umma::mma_bf16(d, umma::desc_kmajor_sw128(sa + 32u * k),
                                           umma::desc_kmajor_sw128(sb + 32u * k), idesc,
                                           (kstep | k) != 0);
                        umma::commit(&ctl->empty[stage]);
                        ++kstep;
                        if (++stage == kStages) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                }
                if (ok)
                    umma::commit(&ctl->tfull[acc]);
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
        if (lane == 0) {
            umma::commit(&ctl->drain);
            mbar_wait(&ctl->drain, 0);
        }
        __syncwarp();
    } else {
        const int q = warp & 3;
        const int r = q * 32 + lane;
        uint32_t acc = 0, acc_phase = 0;
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
            int s, nb;
            coords(tile, s, nb);
            int nk = 0;
            for (int w = 0; w < a.W; ++w)
                nk += __popc(uword(s, w));
            const int sr = s * kBM + r;
            const long long orow = sr < a.T ? (long long)a.sig_perm[sr] : -1;
            if (!wait_or_abort(&ctl->tfull[acc], acc_phase, ctl, a.status))
                break;
            umma::fence_after_sync();
            const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + acc * (uint32_t)kBN;
#pragma unroll 1
            for (int c = 0; c < kBN / 32; ++c) {
                float v[32];
                if (nk > 0) {
                    umma::tmem_ld32(taddr + c * 32, v);
                    umma::tmem_ld_wait();
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        v[e] = 0.f;
                }
                if (orow < 0)
                    continue;
                const size_t at = (size_t)orow * a.N + (size_t)nb * kBN + c * 32;
                if (a.out_sum)
                    store_bf16x32(a.out_sum + at, v);
                if (a.out_total || a.out_total_f32) {
                    if (a.res_in) {
#pragma unroll
                        for (int e = 0; e < 32; e += 8) {
                            float rv[8];
                            bf16x8_to_f32(*reinterpret_cast<const uint4 *>(a.res_in + at + e), rv);
#pragma unroll
                            for (int k = 0; k < 8; ++k)
                                v[e + k] += rv[k];
                        }
                    }
                    if (a.res_f32) {
#pragma unroll
                        for (int e = 0; e < 32; e += 4) {
                            const float4 rv = *reinterpret_cast<const float4 *>(a.res_f32 + at + e);
                            v[e] += rv.x;
                            v[e + 1] += rv.y;
                            v[e + 2] += rv.z;
                            v[e + 3] += rv.w;
                        }
                    }
                    if (a.out_total)
                        store_bf16x32(a.out_total + at, v);
                    if (a.out_total_f32) {
#pragma unroll
                        for (int e = 0; e < 32; e += 4)
                            *reinterpret_cast<float4 *>(a.out_total_f32 + at + e) =
                                make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
                    }
                }
            }
            umma::fence_before_sync();
            mbar_arrive(&ctl->tempty[acc]);
            if (++acc == 2) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
    }

    umma::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        umma::fence_after_sync();
        umma::tmem_dealloc(tmem, kTmemCols);
    }
}

int num_sms()
{
    static int n[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return 0;
    if (!n[dev])
        cudaDeviceGetAttribute(&n[dev], cudaDevAttrMultiProcessorCount, dev);
    return n[dev];
}

}  // namespace

int gather_gemm_launch(int mode, const CUtensorMap &tm0, const CUtensorMap &tm1,
                       const GemmArgs &a, int max_work, int32_t kid, cudaStream_t s)
{
    const int sms = num_sms();
    if (sms <= 0 || max_work < 0)
        return WIDE_CUDA_FAIL();
    if (max_work == 0)
        return WIDE_OK;
    if ((int64_t)a.T * a.K >= (int64_t)1 << 31)      // row offsets are 32-bit
        return WIDE_EUNSUPPORTED;
    const int grid = max_work < sms ? max_work : sms;
    const void *k = mode == GEMM_SWIGLU   ? reinterpret_cast<const void *>(gather_gemm<GEMM_SWIGLU>)
                    : mode == GEMM_ROPE_Q ? reinterpret_cast<const void *>(gather_gemm<GEMM_ROPE_Q>)
                    : mode == GEMM_ROUTER ? reinterpret_cast<const void *>(gather_gemm<GEMM_ROUTER>)
                                          : reinterpret_cast<const void *>(gather_gemm<GEMM_KV>);
    const size_t smem = mode == GEMM_ROUTER ? kSmemBytes + kRouterScratch : kSmemBytes;
    if (!raise_smem_limit(k, smem))
        return WIDE_CUDA_FAIL();
    LaunchScope scope(kid, s);
    if (mode == GEMM_SWIGLU)
        gather_gemm<GEMM_SWIGLU><<<grid, kThreadsGather, kSmemBytes, s>>>(tm0, tm1, a);
    else if (mode == GEMM_ROPE_Q)
        gather_gemm<GEMM_ROPE_Q><<<grid, kThreadsGather, kSmemBytes, s>>>(tm0, tm1, a);
    else if (mode == GEMM_ROUTER)
        gather_gemm<GEMM_ROUTER><<<grid, kThreadsGather, smem, s>>>(tm0, tm1, a);
    else
        gather_gemm<GEMM_KV><<<grid, kThreadsGather, kSmemBytes, s>>>(tm0, tm1, a);
    return launch_status();
}

int tile_union_gemm_launch(const CUtensorMap &tm_a, const CUtensorMap &tm_b, const UnionArgs &a,
                           int32_t kid, cudaStream_t s)
{
    const int sms = num_sms();
    if (sms <= 0)
        return WIDE_CUDA_FAIL();
    const int64_t tiles = (int64_t)((a.T + kBM - 1) / kBM) * (a.N / kBN);
    if (tiles == 0)
        return WIDE_OK;
    const int grid = (int)(tiles < sms ? tiles : sms);
    if (!raise_smem_limit(reinterpret_cast<const void *>(tile_union_gemm), kSmemBytes))
        return WIDE_CUDA_FAIL();
    LaunchScope scope(kid, s);
    tile_union_gemm<<<grid, kThreadsDown, kSmemBytes, s>>>(tm_a, tm_b, a);
    return launch_status();
}

}  // namespace wide
