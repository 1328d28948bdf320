// ffn_decode_tc.cu -- the bf16 decode FFN of up to 32 tokens on the 5th-
// generation tensor cores, as one persistent kernel in which every CTA owns
// a slice of the batch's kept channels.
//
// WIDE, technical summary section 2.A (each token keeps its own contiguous
// FFN channel groups) and section 2.C (block-level skipping): only the
// weights of the groups some token of the batch keeps (the batch's union)
// are read from HBM, each byte once.  With 8 to 32 tokens the work over the
// union is a dense contraction that the CUDA cores cannot feed at HBM speed
// (16 multiply-adds per weight byte at 32 tokens); on the tensor cores it is
// a weight stream again.  A token's skipped groups are zeroed in h, so they
// add exactly nothing to the output, as the definition requires.
//
// Work split.  The union's channels, taken as 16-channel chunks in group
// order, are cut into P contiguous ranges (one per CTA, P = the SM count):
// ranges differ by at most one chunk.  A CTA walks its range in windows of
// up to 64 channels that are contiguous in memory and do not cross a
// 64-channel boundary, and computes, with no data from any other CTA,
//   phase 1  for each window, G[c][t] = W_gate[c] . x[t] and U[c][t] =
//            W_up[c] . x[t] on the tensor cores (N = TP, the tokens padded
//            to 16 or 32; the x rows past T read as zero), then h[t][c] =
//            silu(G) * U for the tokens that keep c's group, 0 otherwise,
//            rounded to bf16 into a shared-memory operand per chunk;
//   phase 2  for each 128-row block of output rows n, D2[n][t] = the sum
//            over ALL its chunks' channels c of W_down[n][c] * h[t][c]
//            (M = 128 MMAs, K = 16 per chunk, into one TMEM accumulator),
//            added once into an fp32 accumulator in global memory with
//            vector atomics (layout [n][T4], T4 = T rounded up to 4).
// After its last block a CTA counts itself in; once every CTA has (a
// bounded wait on the counter; the launch is cooperative), each CTA
// converts its slice of the accumulator into the call's outputs.  Every
// CTA adds into every output once, so the atomics are P * H * T adds; the
// CTAs start their block walk at different blocks to spread them.
//
// Roles (6 warps):  warp 0 streams every stage by TMA through an mbarrier
// ring; warp 1 issues the MMAs (one thread) and owns TMEM; warps 2..5 drain
// TMEM.  A tcgen05.mma at N = 16..32 costs about as much to issue and run
// as it does work, so the layouts keep MMAs few: one per K step of 16 per
// window in phase 1 (packed weights) and one per chunk and block in phase 2.
//
// Weights come in one of two layouts (the template flag PACKED):
//   packed      the wide_ffn_pack copy: W_gate and W_up interleaved in
//               64-channel panels, K-step-major (per K step of a panel,
//               four groups of 16 gate rows then 16 up rows), and W_down
//               in 16-channel column panels [I / 16][H][16].  Every box is
//               one contiguous run, and one M = 128 MMA covers the gate and
//               up rows of a window (rows 32q..32q+15 gate, +16..+31 up of
//               chunk q);
//   nn.Linear   W_gate, W_up [I][H] and W_down [H][I] as given: boxes of
//               128-byte row pieces (about half the HBM bandwidth), two
//               M = 64 MMAs (gate, up) per K step of 16.
//
// Stage layouts (slots of 24 KB at TP = 16, 32 KB at TP = 32; R = the
// window's channels, KC = 64 / R K steps of 64 columns):
//   phase 1  weights [KC][2R rows][128 B] (packed) or W_gate [KC][R][128 B]
//            then W_up the same (nn.Linear), from 16 KB; then x
//            [KC][TP][128 B]; 128-byte swizzle.  An MMA reads 128 (64) rows
//            from a K step's first row: rows past the window's are other
//            bytes of the CTA's shared memory and only feed accumulator
//            rows that are never read;
//   phase 2  for one output block, the W_down tiles of a group of the CTA's
//            windows (at most slot / 4 KB chunks): per chunk 128 rows x 16
//            channels, 32-byte swizzle (packed), or per window 128 rows x R
//            channels with the swizzle of width 2R bytes (nn.Linear).
#include "common.cuh"
#include "host.h"
#include "umma.cuh"

namespace wide {
namespace {

constexpr int kTThreads = 192;        // TMA warp, MMA warp, 4 epilogue warps
constexpr int kTEpi = 128;            // epilogue threads
constexpr int kTChunk = 16;           // channels per chunk
constexpr int kTMaxTok = kTcMaxTok;   // tokens per launch
constexpr int kTMaxChunks = 16;       // chunks per CTA (so also windows and phase-2 groups)
constexpr int kTMaxSlots = 10;
constexpr int kTNB = 8;               // phase-2 accumulators in TMEM
constexpr int kTMaxG = 1024;
constexpr int kTMaxMaskWords = 1024;  // T * W
constexpr uint32_t kTTmemCols = 512;

__host__ __device__ constexpr uint32_t tc_slot_bytes(int TP) { return TP == 16 ? 24576u : 32768u; }

struct TcArgs {
    const uint32_t *mask;   // [T][W] packed group bits
    float *acc;             // [H][T4] fp32 accumulator (0 at launch)
    uint32_t *done;         // arrival counter (0 at launch)
    DownOutputs o;
    int T, T4, H, I, W, G, gs;
    int nslots;
    int32_t *status;
};

// Tensor maps, indexed by log2 of a window's chunk count (R = 16, 32, 64
// channels).  Packed: g = interleaved W_gate / W_up boxes {64, 2R, 64 / R,
// 1}, d = W_down boxes {16, 128, 1, R / 16}.  nn.Linear: g / u = boxes {64,
// R, 64 / R}, d = W_down boxes {R, 128, 1}.  x: boxes {64, TP, 64 / R}.
struct TcMaps {
    CUtensorMap g[3], u[3], x[3], d[3];
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    const uint32_t a = smem_u32(p);
    return p + (((a + 1023u) & ~1023u) - a);
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
// Barrier of the 128 epilogue threads that also ORs a flag over them, so an
// error seen by any thread is seen by all and they leave their loop
// together (a thread left behind at the barrier would wait for ever).
__device__ __forceinline__ bool epi_sync_or(bool v)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 1, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "n"(kTEpi)
        : "memory");
    return r != 0u;
}

// K-major shared-memory descriptor of a tile whose rows are `bytes` long
// (32, 64 or 128), written with the swizzle of the same width: 8-row atoms
// of 8 * bytes, layout codes 6 (32-byte), 4 (64-byte), 2 (128-byte).  A K
// step of 16 inside a row moves the start address field by 2.
__device__ __forceinline__ uint64_t desc_kmajor_rows(uint32_t saddr, int bytes)
{
    const uint64_t code = bytes == 128 ? 2u : bytes == 64 ? 4u : 6u;
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(((uint32_t)bytes * 8u) >> 4) << 32) |
           ((uint64_t)1 << 46) | (code << 61);
}

// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16])
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; ++i)
        v[i] = __uint_as_float(r[i]);
}
template <int TP> __device__ __forceinline__ void tmem_ld_tp(uint32_t taddr, float (&v)[TP]);
template <> __device__ __forceinline__ void tmem_ld_tp<16>(uint32_t taddr, float (&v)[16])
{
    tmem_ld16(taddr, v);
}
template <> __device__ __forceinline__ void tmem_ld_tp<32>(uint32_t taddr, float (&v)[32])
{
    umma::tmem_ld32(taddr, v);
}

struct Win {
    int row0;   // first channel (row of W_gate / W_up, column of W_down)
    int nck;    // 16-channel chunks: 1, 2 or 4
    int q0;     // index of its first chunk among the CTA's chunks
};
struct Grp {    // consecutive windows whose W_down tiles share a phase-2 stage
    int w0, w1; // windows [w0, w1)
    int q0, nq; // their chunks
};

template <int TP, bool PACKED>
__global__ void __launch_bounds__(kTThreads, 1)
    ffn_decode_tc(const __grid_constant__ TcMaps maps, const TcArgs a)
{
    constexpr uint32_t SLOT = tc_slot_bytes(TP);
    constexpr int GC = (int)(SLOT / 4096);          // chunks per phase-2 stage
    constexpr uint32_t kD2 = 4 * TP;                 // TMEM: 2 x (gate, up) x TP, then D2
    static_assert(kD2 + kTNB * TP <= kTTmemCols, "TMEM columns");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    const int NS = a.nslots;
    const int T = a.T, T4 = a.T4, H = a.H, gs = a.gs, W = a.W;
    uint8_t *slots = smem;                                        // NS x SLOT
    uint8_t *hall = slots + (size_t)NS * SLOT;                    // [kTMaxChunks][TP][32 B]
    uint32_t *mall = reinterpret_cast<uint32_t *>(hall + kTMaxChunks * TP * 32);   // [T][W]
    int *live = reinterpret_cast<int *>(mall + T * W);                             // [G]
    Win *wins = reinterpret_cast<Win *>(live + a.G);                               // [kTMaxChunks]
    Grp *grps = reinterpret_cast<Grp *>(wins + kTMaxChunks);                       // [kTMaxChunks]
    uint64_t *bars = reinterpret_cast<uint64_t *>(
        (reinterpret_cast<uintptr_t>(grps + kTMaxChunks) + 7) & ~(uintptr_t)7);
    uint64_t *full = bars;                 // [NS]  TMA -> MMA
    uint64_t *empty = full + NS;           // [NS]  MMA -> TMA
    uint64_t *d1_full = empty + NS;        // [2]   MMA -> epilogue
    uint64_t *d1_empty = d1_full + 2;      // [2]   epilogue -> MMA
    uint64_t *h_ready = d1_empty + 2;      // [1]   epilogue -> MMA: every chunk's h written
    uint64_t *d2_full = h_ready + 1;       // [kTNB]
    uint64_t *d2_empty = d2_full + kTNB;   // [kTNB]
    uint64_t *fin = d2_empty + kTNB;       // [1]   every MMA of the CTA done
    __shared__ int s_nlive, s_nwin, s_ngrp, s_issued;
    __shared__ volatile int s_err;
    __shared__ uint32_t s_tmem;

    const int tid = (int)threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int P = (int)gridDim.x, c = (int)blockIdx.x;

    for (int i = tid; i < T * W; i += kTThreads)
        mall[i] = a.mask[i];
    if (tid == 0) {
        s_err = 0;
        s_issued = 0;
        for (int i = 0; i < NS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&d1_full[i], 1);
            mbar_init(&d1_empty[i], kTEpi);
        }
        mbar_init(h_ready, kTEpi);
        for (int i = 0; i < kTNB; ++i) {
            mbar_init(&d2_full[i], 1);
            mbar_init(&d2_empty[i], kTEpi);
        }
        mbar_init(fin, 1);
        fence_mbar_init();
        for (int i = 0; i < 3; ++i) {
            tma_prefetch_desc(&maps.g[i]);
            tma_prefetch_desc(&maps.x[i]);
            tma_prefetch_desc(&maps.d[i]);
            if (!PACKED)
                tma_prefetch_desc(&maps.u[i]);
        }
    }
    if (warp == 1) {
        umma::tmem_alloc(&s_tmem, kTTmemCols);
        umma::tmem_relinquish();
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
    // this CTA's chunk range, its windows and the phase-2 groups (one thread)
    if (tid == 0) {
        const int cpg = gs / kTChunk;
        const int64_t n = (int64_t)s_nlive * cpg;
        const int q0 = (int)(n * c / P), q1 = (int)(n * (c + 1) / P);
        auto row_of = [&](int q) { return live[q / cpg] * gs + (q % cpg) * kTChunk; };
        int nw = 0, nq = 0;
        for (int q = q0; q < q1 && nw < kTMaxChunks;) {
            const int r = row_of(q);
            const int lim = 4 - ((r / kTChunk) & 3);   // stay inside a 64-channel block
            int L = 1;
            while (L < lim && q + L < q1 && row_of(q + L) == r + kTChunk * L)
                ++L;
            if (L == 3)
                L = 2;
            wins[nw].row0 = r;
            wins[nw].nck = L;
            wins[nw].q0 = nq;
            ++nw;
            nq += L;
            q += L;
        }
        int ng = 0;
        for (int w0 = 0; w0 < nw;) {
            int w1 = w0, k = 0;
            while (w1 < nw && k + wins[w1].nck <= GC)
                k += wins[w1++].nck;
            grps[ng].w0 = w0;
            grps[ng].w1 = w1;
            grps[ng].q0 = wins[w0].q0;
            grps[ng].nq = k;
            ++ng;
            w0 = w1;
        }
        s_nwin = nw;
        s_ngrp = ng;
    }
    __syncthreads();

    const int nw = s_nwin, ng = s_ngrp;
    const int KS = H / 64;          // 64-column K steps
    const int MB = H / 128;         // 128-row output blocks
    const uint32_t tmem = s_tmem;
    auto slot_of = [&](int kk) { return slots + (size_t)(kk % NS) * SLOT; };
    auto lg = [](int nck) { return nck == 1 ? 0 : nck == 2 ? 1 : 2; };
    // Every CTA walks the K steps and the output blocks from its own
    // starting point (rotated by its index), so the CTAs do not all read
    // the same x lines, nor add into the same accumulator lines, at once.
    auto rot = [c](int st, int n) { return (st + c) % n; };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            bool err = false;
            int k = 0;
            auto acquire = [&](int kk) {
                if (kk >= NS && !err) {
                    if (s_err || !mbar_wait(&empty[kk % NS], (uint32_t)(kk / NS - 1) & 1u))
                        err = true;
                }
                return !err;
            };
            for (int j = 0; j < nw && !err; ++j) {
                const Win w = wins[j];
                const int li = lg(w.nck), KC = 4 >> li, R = 16 << li;
                const int n1 = (KS + KC - 1) / KC;
                for (int st = 0; st < n1; ++st, ++k) {
                    const int ks = rot(st, n1) * KC;
                    if (!acquire(k))
                        break;
                    uint64_t *fb = &full[k % NS];
                    uint8_t *sb = slot_of(k);
                    mbar_arrive_expect_tx(fb, (uint32_t)(2 * 64 + KC * TP) * 128u);
                    if (PACKED) {
                        // the window's 16-channel groups, gate and up interleaved
                        tma_load_4d(sb, &maps.g[li], 0, 2 * (w.row0 & 63), ks, w.row0 >> 6, fb);
                    } else {
                        tma_load_3d(sb, &maps.g[li], 0, w.row0, ks, fb);
                        tma_load_3d(sb + KC * R * 128, &maps.u[li], 0, w.row0, ks, fb);
                    }
                    tma_load_3d(sb + 2 * 64 * 128, &maps.x[li], 0, 0, ks, fb);
                }
            }
            for (int st = 0; st < MB && !err; ++st) {
                const int mb = rot(st, MB);
                for (int g = 0; g < ng && !err; ++g, ++k) {
                    if (!acquire(k))
                        break;
                    const Grp gr = grps[g];
                    uint64_t *fb = &full[k % NS];
                    uint8_t *sb = slot_of(k);
                    mbar_arrive_expect_tx(fb, (uint32_t)gr.nq * 4096u);
                    for (int j = gr.w0; j < gr.w1; ++j) {
                        const Win w = wins[j];
                        uint8_t *dst = sb + (size_t)(w.q0 - gr.q0) * 4096;
                        if (PACKED)
                            tma_load_4d(dst, &maps.d[lg(w.nck)], 0, 0, mb, w.row0 >> 4, fb);
                        else
                            tma_load_3d(dst, &maps.d[lg(w.nck)], w.row0, 0, mb, fb);
                    }
                }
            }
            s_issued = k;
            if (err)
                s_err = 1;
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            bool err = false;
            int k = 0;
            constexpr uint32_t id64 = umma::idesc_bf16_f32(64, TP);
            constexpr uint32_t id128 = umma::idesc_bf16_f32(128, TP);
            auto wait = [&](uint64_t *bar, uint32_t par) {
                if (!err && (s_err || !mbar_wait(bar, par)))
                    err = true;
                return !err;
            };
            for (int j = 0; j < nw && !err; ++j) {
                const Win w = wins[j];
                const int li = lg(w.nck), KC = 4 >> li, R = 16 << li;
                const int b1 = j & 1;
                if (j >= 2 && !wait(&d1_empty[b1], (uint32_t)((j >> 1) - 1) & 1u))
                    break;
                umma::fence_after_sync();
                const uint32_t dg = tmem + (uint32_t)(b1 * 2 * TP), du = dg + TP;
                const int n1 = (KS + KC - 1) / KC;
                for (int st = 0; st < n1; ++st, ++k) {
                    const int ks = rot(st, n1) * KC;
                    if (!wait(&full[k % NS], (uint32_t)(k / NS) & 1u))
                        break;
                    umma::fence_after_sync();
                    const uint32_t sa = smem_u32(slot_of(k));
                    const int nkc = KS - ks < KC ? KS - ks : KC;
                    for (int kc = 0; kc < nkc; ++kc) {
                        const uint32_t acc0 = (st | kc) != 0 ? 1u : 0u;
                        const uint64_t bd = umma::desc_kmajor_sw128(sa + 2 * 64 * 128 + kc * TP * 128);
                        if (PACKED) {
                            const uint64_t ad = umma::desc_kmajor_sw128(sa + kc * 2 * R * 128);
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                umma::mma_bf16(dg, ad + 2 * kk, bd + 2 * kk, id128, kk ? 1u : acc0);
                        } else {
                            const uint64_t agd = umma::desc_kmajor_sw128(sa + kc * R * 128),
                                           aud = umma::desc_kmajor_sw128(sa + (KC + kc) * R * 128);
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                umma::mma_bf16(dg, agd + 2 * kk, bd + 2 * kk, id64, kk ? 1u : acc0);
                                umma::mma_bf16(du, aud + 2 * kk, bd + 2 * kk, id64, kk ? 1u : acc0);
                            }
                        }
                    }
                    umma::commit(&empty[k % NS]);
                }
                if (err)
                    break;
                umma::commit(&d1_full[b1]);
            }
            // phase 2: one accumulator per output block over all the CTA's chunks
            if (!err && nw > 0 && wait(h_ready, 0)) {
                umma::fence_after_sync();
                const uint32_t sh = smem_u32(hall);
                for (int st = 0; st < MB && !err; ++st) {
                    const int b2 = st % kTNB;
                    if (st >= kTNB && !wait(&d2_empty[b2], (uint32_t)(st / kTNB - 1) & 1u))
                        break;
                    umma::fence_after_sync();
                    const uint32_t d = tmem + kD2 + (uint32_t)(b2 * TP);
                    for (int g = 0; g < ng; ++g, ++k) {
                        if (!wait(&full[k % NS], (uint32_t)(k / NS) & 1u))
                            break;
                        umma::fence_after_sync();
                        const Grp gr = grps[g];
                        const uint32_t sa = smem_u32(slot_of(k));
                        for (int j = gr.w0; j < gr.w1; ++j) {
                            const Win w = wins[j];
                            const uint32_t at = sa + (uint32_t)((w.q0 - gr.q0) * 4096);
                            const int rb = PACKED ? 32 : w.nck * 32;
                            const uint64_t a0 = desc_kmajor_rows(at, rb);
                            for (int kk = 0; kk < w.nck; ++kk) {
                                // packed: chunk tiles 4 KB apart (start field + 256);
                                // nn.Linear: a K step of 16 inside the window's rows
                                const uint64_t ad = a0 + (PACKED ? (uint64_t)(kk * 256) : (uint64_t)(2 * kk));
                                const uint64_t bd =
                                    desc_kmajor_rows(sh + (uint32_t)((w.q0 + kk) * TP * 32), 32);
                                umma::mma_bf16(d, ad, bd, id128, (g | (j - gr.w0) | kk) ? 1u : 0u);
                            }
                        }
                        umma::commit(&empty[k % NS]);
                    }
                    if (err)
                        break;
                    umma::commit(&d2_full[b2]);
                }
            }
            // every MMA issued so far has completed once fin fires
            if (k > 0) {
                umma::commit(fin);
                mbar_wait(fin, 0);
            }
            if (err)
                s_err = 1;
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue (warps 2..5)
        // Warp `quad` reads TMEM lanes 32 * quad .. + 31.  Phase 1, packed:
        // one M = 128 accumulator, lanes 0..15 the gate and 16..31 the up
        // values of the window's channels 16 * quad + (lane & 15).  Phase 1,
        // nn.Linear: two M = 64 accumulators (row m in lane (m % 16) + 32 *
        // (m / 16)), so lanes 0..15 hold gate in one and up in the other.
        // Phase 2: row n of a 128-row block is lane n.  Every exit decision
        // goes through epi_sync_or, so the four warps take the same path
        // through their named barrier.
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        bool err = false;
        auto wait = [&](uint64_t *bar, uint32_t par) {
            if (!err && (s_err || !mbar_wait(bar, par)))
                err = true;
            return !err;
        };
        for (int j = 0; j < nw; ++j) {
            const int b1 = j & 1;
            const Win w = wins[j];
            float v[TP], o[TP];
            // tcgen05.ld is warp-wide: the warp takes it only if every lane's wait ended
            if (__all_sync(0xffffffffu, wait(&d1_full[b1], (uint32_t)(j >> 1) & 1u))) {
                umma::fence_after_sync();
                const uint32_t base = tmem + lane_off + (uint32_t)(b1 * 2 * TP);
                tmem_ld_tp<TP>(base, v);
                if (!PACKED)
                    tmem_ld_tp<TP>(base + TP, o);
                umma::tmem_ld_wait();
            } else {
                err = true;
#pragma unroll
                for (int t = 0; t < TP; ++t)
                    v[t] = o[t] = 0.f;
            }
            umma::fence_before_sync();
            mbar_arrive(&d1_empty[b1]);
            if (PACKED) {
#pragma unroll
                for (int t = 0; t < TP; ++t)
                    o[t] = __shfl_xor_sync(0xffffffffu, v[t], 16);
            }
            // packed: both halves of the warp hold (gate, up) of channel
            // 16 * quad + (lane & 15) and write h for half of the tokens each;
            // nn.Linear: lanes 0..15 write all tokens
            const bool hi = lane >= 16;
            const int cw = quad * 16 + (lane & 15);          // channel within the window
            if (!err && (PACKED || !hi)) {
                const bool live_ch = quad < w.nck;
                const int grp = (w.row0 + cw) / gs;
                const uint32_t *mcol = mall + (grp >> 5);
                const uint32_t bit = 1u << (grp & 31);
                // chunk tile [TP][16] with 32-byte rows, 32-byte swizzle (the
                // 16-byte half of row t is flipped when bit 2 of t is set)
                uint8_t *hp = hall + (size_t)(w.q0 + quad) * TP * 32;
                const int cc = cw & 15;
                constexpr int TH = PACKED ? TP / 2 : TP;
#pragma unroll
                for (int t2 = 0; t2 < TH; ++t2) {
                    const int t = (PACKED && hi) ? t2 + TP / 2 : t2;
                    const float gv = PACKED ? (hi ? o[t2 + TP / 2] : v[t2]) : v[t2];
                    const float uv = PACKED ? (hi ? v[t2 + TP / 2] : o[t2]) : o[t2];
                    float hv = 0.f;
                    if (t < T && (mcol[t * W] & bit))
                        hv = silu_f32(gv) * uv;
                    if (live_ch)
                        *reinterpret_cast<__nv_bfloat16 *>(
                            hp + t * 32 + ((((cc >> 3) ^ (t >> 2)) & 1) << 4) + (cc & 7) * 2) =
                            __float2bfloat16_rn(hv);
                }
            }
            err = epi_sync_or(err);
            if (err)
                break;
        }
        if (!err && nw > 0) {
            fence_proxy_async_smem();
            mbar_arrive(h_ready);
            for (int st = 0; st < MB; ++st) {
                const int b2 = st % kTNB, mb = rot(st, MB);
                float v[TP];
                if (!__all_sync(0xffffffffu, wait(&d2_full[b2], (uint32_t)(st / kTNB) & 1u))) {
                    err = true;
                    break;
                }
                umma::fence_after_sync();
                tmem_ld_tp<TP>(tmem + lane_off + kD2 + (uint32_t)(b2 * TP), v);
                umma::tmem_ld_wait();
                umma::fence_before_sync();
                mbar_arrive(&d2_empty[b2]);
                float *dst = a.acc + (size_t)(mb * 128 + row) * T4;
#pragma unroll
                for (int t4 = 0; t4 < TP / 4; ++t4)
                    if (4 * t4 < T)
                        atomicAdd(reinterpret_cast<float4 *>(dst) + t4,
                                  make_float4(v[4 * t4], v[4 * t4 + 1], v[4 * t4 + 2], v[4 * t4 + 3]));
            }
        }
        if (err)
            s_err = 1;
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
        } else {
            set_status(a.status, WIDE_DEV_TIMEOUT);
        }
        s_go = go;
    }
    __syncthreads();
    if (s_go) {
        // this CTA's output rows n (acc is [n][T4]; out is [t][n])
        const int n0 = (int)((int64_t)c * H / P), n1 = (int)((int64_t)(c + 1) * H / P);
        const DownOutputs &o = a.o;
        for (int idx = tid; idx < (n1 - n0) * T; idx += kTThreads) {
            const int t = idx / (n1 - n0), n = n0 + idx % (n1 - n0);
            const float s = __ldcg(a.acc + (size_t)n * T4 + t);
            const size_t at = (size_t)t * H + n;
            if (o.out_sum)
                static_cast<__nv_bfloat16 *>(o.out_sum)[at] = __float2bfloat16_rn(s);
            if (o.out_total || o.out_total_f32) {
                float tot = s;
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
    if (s_err && tid == 0) {
        const int issued = s_issued;
        for (int kk = issued - 1; kk >= 0 && kk >= issued - NS; --kk)
            mbar_wait(&full[kk % NS], (uint32_t)(kk / NS) & 1u);
    }
    __syncthreads();
    if (warp == 1)
        umma::tmem_dealloc(tmem, kTTmemCols);
}

struct TcPlan {
    int TP, P, nslots;
    size_t smem;
};

bool plan_tc(int T, int H, int I, int gs, TcPlan *p)
{
    if (T < 1 || T > kTMaxTok || H < 128 || H % 128 != 0 || gs % kTChunk != 0 || gs < 16 ||
        gs > 256 || I % gs != 0)
        return false;
    const int G = I / gs, W = (G + 31) / 32;
    if (G > kTMaxG || T * W > kTMaxMaskWords)
        return false;
    int dev = 0, sms = 0, optin = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess ||
        sms <= 0)
        return false;
    p->P = sms;
    // a CTA's range holds at most ceil(I / 16 / P) chunks (one window each at worst)
    if (((int64_t)I / kTChunk + sms - 1) / sms > kTMaxChunks)
        return false;
    p->TP = T <= 16 ? 16 : 32;
    const uint32_t slot = tc_slot_bytes(p->TP);
    const size_t fixed = 1024 + (size_t)kTMaxChunks * p->TP * 32 + (size_t)T * W * 4 +
                         (size_t)G * 4 + kTMaxChunks * (sizeof(Win) + sizeof(Grp)) + 8 +
                         (2 * kTMaxSlots + 5 + 2 * kTNB + 1) * 8 + 256;
    if ((size_t)optin <= fixed + 2 * slot)
        return false;
    int ns = (int)(((size_t)optin - fixed) / slot);
    if (ns > kTMaxSlots)
        ns = kTMaxSlots;
    p->nslots = ns;
    p->smem = fixed + (size_t)ns * slot;
    return true;
}

template <int TP, bool PACKED>
int launch_tc(const TcPlan &pl, const TcMaps &m, const TcArgs &a, cudaStream_t s)
{
    auto kernel = ffn_decode_tc<TP, PACKED>;
    if (!raise_smem_limit(reinterpret_cast<const void *>(kernel), pl.smem))
        return WIDE_CUDA_FAIL();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.P);
    cfg.blockDim = dim3(kTThreads);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    LaunchScope scope(KID_DECODE_FFN_TC, s);
    if (cudaLaunchKernelEx(&cfg, kernel, m, a) != cudaSuccess)
        return WIDE_CUDA_FAIL();
    return WIDE_OK;
}

}  // namespace

size_t decode_ffn_tc_scratch(int T, int H)
{
    const size_t T4 = ((size_t)T + 3) / 4 * 4;
    return align_up(T4 * H * sizeof(float), 256) + 256;
}

bool decode_ffn_tc_supported(int T, int H, int I, int gs)
{
    TcPlan p;
    return plan_tc(T, H, I, gs, &p);
}

bool decode_ffn_tc_packed_supported(int T, int H, int I, int gs)
{
    return I % 64 == 0 && decode_ffn_tc_supported(T, H, I, gs);
}

int decode_ffn_tc(const void *x, const void *wg, const void *wu, const void *wd,
                  const void *packed, const uint32_t *mask, const DownOutputs &o, int T, int H,
                  int I, int gs, void *scratch, cudaStream_t s)
{
    TcPlan pl;
    if (!plan_tc(T, H, I, gs, &pl) || (packed && I % 64 != 0))
        return WIDE_EUNSUPPORTED;
    const int G = I / gs;
    TcMaps m;
    const uint64_t KS = (uint64_t)H / 64;
    const char *pk = static_cast<const char *>(packed);
    const size_t mat = (size_t)I * H * 2;
    for (int li = 0; li < 3; ++li) {
        const uint32_t R = 16u << li, KC = 4u >> li;
        // x as {64 columns, T rows, H / 64 K steps}: a box lands as
        // [K step][TP rows][128 bytes] (rows past T read as zero)
        const uint64_t xdims[3] = {64, (uint64_t)T, KS}, rstr[2] = {(uint64_t)H * 2, 128};
        const uint32_t xbox[3] = {64, (uint32_t)pl.TP, KC};
        if (!make_tmap_3d_swz(&m.x[li], x, xdims, rstr, xbox, 128))
            return WIDE_CUDA_FAIL();
        if (packed) {
            // interleaved W_gate / W_up panels {64 columns, 128 rows (4 groups
            // of 16 gate then 16 up rows), K steps, panels}: the box's 2R rows
            // of one K step are 2R * 128 contiguous bytes.  W_down panels {16
            // channels, 128 rows, H / 128 blocks, I / 16 chunks}: a window's
            // chunks of one block are 4 KB pieces.
            const uint64_t gdims[4] = {64, 128, KS, (uint64_t)I / 64};
            const uint64_t gstr[3] = {128, 16384, (uint64_t)H * 256};
            const uint32_t gbox[4] = {64, 2 * R, KC, 1};
            const uint64_t ddims[4] = {16, 128, (uint64_t)H / 128, (uint64_t)I / 16};
            const uint64_t dstr[3] = {32, 4096, (uint64_t)H * 32};
            const uint32_t dbox[4] = {16, 128, 1, 1u << li};
            if (!make_tmap_4d_swz(&m.g[li], pk, gdims, gstr, gbox, 128) ||
                !make_tmap_4d_swz(&m.d[li], pk + 2 * mat, ddims, dstr, dbox, 32))
                return WIDE_CUDA_FAIL();
            m.u[li] = m.g[li];
        } else {
            // W_gate / W_up as {64 columns, rows, K steps}: a box lands as
            // [K step][R rows][128 bytes] (the rows dimension's stride, H * 2
            // bytes, is larger than the K steps' 128).  W_down as {I columns,
            // 128 rows, H / 128 blocks}: [128 rows][R channels].
            const uint64_t wdims[3] = {64, (uint64_t)I, KS};
            const uint32_t wbox[3] = {64, R, KC};
            const uint64_t ddims[3] = {(uint64_t)I, 128, (uint64_t)H / 128};
            const uint64_t dstr[2] = {(uint64_t)I * 2, (uint64_t)I * 2 * 128};
            const uint32_t dbox[3] = {R, 128, 1};
            if (!make_tmap_3d_swz(&m.g[li], wg, wdims, rstr, wbox, 128) ||
                !make_tmap_3d_swz(&m.u[li], wu, wdims, rstr, wbox, 128) ||
                !make_tmap_3d_swz(&m.d[li], wd, ddims, dstr, dbox, 2 * R))
                return WIDE_CUDA_FAIL();
        }
    }
    TcArgs a = {};
    a.mask = mask;
    a.acc = static_cast<float *>(scratch);
    a.T = T;
    a.T4 = (T + 3) / 4 * 4;
    const size_t acc_bytes = align_up((size_t)a.T4 * H * sizeof(float), 256);
    a.done = reinterpret_cast<uint32_t *>(static_cast<char *>(scratch) + acc_bytes);
    a.o = o;
    a.H = H;
    a.I = I;
    a.G = G;
    a.W = (G + 31) / 32;
    a.gs = gs;
    a.nslots = pl.nslots;
    a.status = status_ptr();
    if (cudaMemsetAsync(scratch, 0, acc_bytes + sizeof(uint32_t), s) != cudaSuccess)
        return WIDE_CUDA_FAIL();
    if (packed)
        return pl.TP == 16 ? launch_tc<16, true>(pl, m, a, s) : launch_tc<32, true>(pl, m, a, s);
    return pl.TP == 16 ? launch_tc<16, false>(pl, m, a, s) : launch_tc<32, false>(pl, m, a, s);
}

}  // namespace wide
