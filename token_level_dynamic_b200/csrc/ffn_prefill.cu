// ffn_prefill.cu -- masked SwiGLU FFN for many tokens (prefill) on the
// 5th-generation tensor cores (tcgen05, TMEM accumulators, TMA operands).
//
// WIDE, technical summary section 2.B: after mask reordering, group g's
// active tokens form the prefix perm[g][0 : count[g]), so group g is a dense
// GEMM over ceil(count[g] / 128) tiles of known active prefix; section 2.C:
// a tile with no active token is never issued (block-level skip), rows past
// the active prefix of a partial tile are not loaded (load-stage skip).
//
// Three launches after wide_reorder, no host synchronisation:
//   zero_dead   writes zeros into the H rows of (token, group) pairs the
//               token skips, so that the down projection can treat every
//               tile of H as dense.
//   gateup      persistent, warp-specialised.  Work item (g, i) = rows
//               perm[g][128 i : 128 i + 128) of x (gathered 16 bytes at a time
//               with cp.async by two warps, straight into the swizzled
//               operand layout) times the 256-row slab [W_gate[g]; W_up[g]]
//               (TMA); one
//               M=128, N=256, K=16 tcgen05 MMA per 16 columns of K into an
//               fp32 TMEM accumulator (two accumulators, 512 columns, so the
//               epilogue of one item overlaps the MMAs of the next).  The
//               epilogue computes silu(gate) * up and stores bf16 rows of H
//               at the tokens' signature-order positions.
//   down        persistent.  Tile (s, nb) = 128 tokens of signature tile s
//               times 256 output columns; the K loop visits only the groups
//               in tile_union[s] (block-level skip on K); inactive rows of a
//               visited group are the zeros written by zero_dead.  The
//               epilogue writes bf16 rows of out at the tokens' own rows.
//
// Warp roles in both tcgen05 kernels: warp 0 = TMA producer, warp 1 = TMEM
// owner and single-thread MMA issuer, warps 2..5 = epilogue (warp w reads
// TMEM lanes 32 * (w % 4) .. +31); gate/up adds warps 6..7 for the row gather.  Every mbarrier wait is
// bounded; on expiry the kernel records WIDE_DEV_TIMEOUT, drains what it
// issued (bounded), frees its TMEM and returns.
#include "common.cuh"
#include "host.h"
#include "umma.cuh"

namespace wide {
namespace {

constexpr int kBM = 128;            // rows (tokens) per tile
constexpr int kBK = 64;             // K per pipeline stage (128 bytes of bf16)
constexpr int kGS = 128;            // channels per group on this path
constexpr int kBN = 256;            // MMA N
constexpr int kStages = 4;
constexpr uint32_t kATile = kBM * 128;   // 16 KB
constexpr uint32_t kBTile = kBN * 128;   // 32 KB
constexpr uint32_t kStageBytes = kATile + kBTile;
constexpr int kThreads = 192;      // down kernel: producer, MMA, 4 epilogue warps
constexpr int kThreadsGU = 256;    // gate/up: + 2 warps that gather x rows with cp.async
constexpr int kGatherThreads = 64;
constexpr uint32_t kTmemCols = 512;

struct __align__(8) Ctl {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

constexpr size_t kSmemBytes = 1024 + kStages * kStageBytes + sizeof(Ctl);

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    const uint32_t a = smem_u32(p);
    return p + (((a + 1023u) & ~1023u) - a);
}

// Bounded wait that also observes the CTA-wide abort flag.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, Ctl *ctl,
                                              int32_t *status)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((it & 255u) == 0) {
            if (*(volatile int *)&ctl->abort)
                return false;
            if (globaltimer() - t0 > kWaitLimitNs) {
                set_status(status, WIDE_DEV_TIMEOUT);
                *(volatile int *)&ctl->abort = 1;
                return false;
            }
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

// ------------------------------------------------------------- zero_dead
// One block per token; 16 threads clear the 256 bytes of one skipped group.
__global__ void __launch_bounds__(128)
    prefill_zero_dead(const uint32_t *__restrict__ mask, const int32_t *__restrict__ sig_pos,
                      __nv_bfloat16 *__restrict__ hbuf, int T, int I, int G, int W)
{
    const int t = blockIdx.x;
    if (t >= T)
        return;
    const size_t row = (size_t)sig_pos[t] * I;
    const int sub = threadIdx.x & 15;
    for (int g = threadIdx.x >> 4; g < G; g += 8) {
        if ((mask[(size_t)t * W + (g >> 5)] >> (g & 31)) & 1u)
            continue;
        uint4 *d = reinterpret_cast<uint4 *>(hbuf + row + (size_t)g * kGS);
        d[sub] = make_uint4(0u, 0u, 0u, 0u);
    }
}

// --------------------------------------------------------------- gate/up
__global__ void __launch_bounds__(kThreadsGU, 1)
    prefill_gateup(const __nv_bfloat16 *__restrict__ x, const __grid_constant__ CUtensorMap tm_g,
                   const __grid_constant__ CUtensorMap tm_u, const int32_t *__restrict__ count,
                   const int32_t *__restrict__ perm, const int32_t *__restrict__ items,
                   const int32_t *__restrict__ n_items_p, const int32_t *__restrict__ sig_pos,
                   __nv_bfloat16 *__restrict__ hbuf, int T, int H, int I, int32_t *status)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    Ctl *ctl = reinterpret_cast<Ctl *>(smem + kStages * kStageBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_items = *n_items_p;
    const int KT = H / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            // one arrive (with the weight-tile bytes) from the TMA producer
            // plus one cp.async-completion arrive from each gather thread
            mbar_init(&ctl->full[s], 1 + kGatherThreads);
            mbar_init(&ctl->empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&ctl->tfull[a], 1);
            mbar_init(&ctl->tempty[a], 128);
        }
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_g);
        tma_prefetch_desc(&tm_u);
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
        // ------------------------------------------------ weight producer
        // The 256-row slab [W_gate[g]; W_up[g]] of each K stage by TMA.
        uint32_t stage = 0, phase = 0, issued = 0;
        bool ok = true;
        for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
            const int g = items[2 * it];
            for (int kt = 0; kt < KT && ok; ++kt) {
                if (lane == 0) {
                    if (!wait_or_abort(&ctl->empty[stage], phase ^ 1u, ctl, status)) {
                        ok = false;
                    } else {
                        uint8_t *b = smem + stage * kStageBytes + kATile;
                        mbar_arrive_expect_tx(&ctl->full[stage], kBTile);
                        tma_load_2d(b, &tm_g, kt * kBK, g * kGS, &ctl->full[stage]);
                        tma_load_2d(b + kBTile / 2, &tm_u, kt * kBK, g * kGS, &ctl->full[stage]);
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
        if (!ok && lane == 0) {
            // let copies still in flight land before the CTA's smem goes away:
            // stage s was armed for the issued uses s, s + kStages, ...
            for (uint32_t s = 0; s < kStages && s < issued; ++s) {
                const uint32_t uses = (issued - s + kStages - 1) / kStages;
                mbar_wait(&ctl->full[s], (uses - 1u) & 1u);
            }
        }
    } else if (warp >= 6) {
        // ------------------------------------------------ x-row gather
        // Load-stage skipping: thread p copies tile rows p and p + 64 of
        // the item -- the tokens perm[g][128 i + row] -- 16 bytes at a time
        // into the 128-byte-swizzled A tile; rows past the active prefix
        // are not loaded (their accumulator rows are never stored).  Each
        // thread's cp.async completions arrive on the stage's barrier.
        const int p = threadIdx.x - 6 * 32;
        uint32_t stage = 0, phase = 0;
        bool ok = true;
        for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
            const int g = items[2 * it], ti = items[2 * it + 1];
            const int base = ti * kBM;
            const int nrows = min(kBM, count[g] - base);
            const int32_t *prow = perm + (size_t)g * T + base;
            const __nv_bfloat16 *src0 = p < nrows ? x + (size_t)prow[p] * H : nullptr;
            const __nv_bfloat16 *src1 = p + 64 < nrows ? x + (size_t)prow[p + 64] * H : nullptr;
            for (int kt = 0; kt < KT && ok; ++kt) {
                if (!wait_or_abort(&ctl->empty[stage], phase ^ 1u, ctl, status)) {
                    ok = false;
                    break;
                }
                const uint32_t a = smem_u32(smem + stage * kStageBytes);
                const int k0 = kt * kBK;
                if (src0) {
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        cp_async16(a + swz128(p, c), src0 + k0 + 8 * c);
                }
                if (src1) {
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        cp_async16(a + swz128(p + 64, c), src1 + k0 + 8 * c);
                }
                cp_async_arrive_noinc(&ctl->full[stage]);
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        cp_async_wait_all();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        constexpr uint32_t idesc = umma::idesc_bf16_f32(kBM, kBN);
        uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
        bool ok = true;
        for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
            if (lane == 0) {
                if (!wait_or_abort(&ctl->tempty[acc], acc_phase ^ 1u, ctl, status))
                    ok = false;
                umma::fence_after_sync();
                const uint32_t d = tmem + acc * (uint32_t)kBN;
                for (int kt = 0; kt < KT && ok; ++kt) {
                    if (!wait_or_abort(&ctl->full[stage], phase, ctl, status)) {
                        ok = false;
                        break;
                    }
                    // the A tile was written by cp.async (generic proxy) and is
                    // read by the tensor core (async proxy)
                    fence_proxy_async_smem();
                    umma::fence_after_sync();
                    const uint32_t a = smem_u32(smem + stage * kStageBytes);
                    const uint32_t b = a + kATile;
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k)
                        umma::mma_bf16(d, umma::desc_kmajor_sw128(a + 32u * k),
                                       umma::desc_kmajor_sw128(b + 32u * k), idesc,
                                       (kt | k) != 0);
                    umma::commit(&ctl->empty[stage]);
                    if (++stage == kStages) {
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
            // every MMA this thread issued has completed once this arrives
            umma::commit(&ctl->drain);
            mbar_wait(&ctl->drain, 0);
        }
        __syncwarp();
    } else if (warp >= 2 && warp <= 5) {
        // ------------------------------------------------ epilogue
        const int q = warp & 3;             // TMEM lane quadrant of this warp
        const int j = q * 32 + lane;        // tile row = TMEM lane
        uint32_t acc = 0, acc_phase = 0;
        for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
            const int g = items[2 * it], ti = items[2 * it + 1];
            const int base = ti * kBM;
            const int nrows = min(kBM, count[g] - base);
            long long out_row = -1;
            if (j < nrows)
                out_row = sig_pos[perm[(size_t)g * T + base + j]];
            if (!wait_or_abort(&ctl->tfull[acc], acc_phase, ctl, status))
                break;
            umma::fence_after_sync();
            const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + acc * (uint32_t)kBN;
#pragma unroll 1
            for (int c = 0; c < kGS / 32; ++c) {
                float gv[32], uv[32];
                umma::tmem_ld32(taddr + c * 32, gv);
                umma::tmem_ld32(taddr + kGS + c * 32, uv);
                umma::tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    gv[e] = silu_f32(gv[e]) * uv[e];
                if (out_row >= 0)
                    store_bf16x32(hbuf + out_row * I + (size_t)g * kGS + c * 32, gv);
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

// ------------------------------------------------------------------ down
__global__ void __launch_bounds__(kThreads, 1)
    prefill_down(const __grid_constant__ CUtensorMap tm_h, const __grid_constant__ CUtensorMap tm_d,
                 const uint32_t *__restrict__ tile_union, const int32_t *__restrict__ sig_perm,
                 __nv_bfloat16 *__restrict__ out, int T, int H, int I, int W, int32_t *status)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1024(smem_raw);
    Ctl *ctl = reinterpret_cast<Ctl *>(smem + kStages * kStageBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_sig = (T + kBM - 1) / kBM;
    const int n_nb = H / kBN;
    const int n_tiles = n_sig * n_nb;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&ctl->tfull[a], 1);
            mbar_init(&ctl->tempty[a], 128);
        }
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tm_h);
        tma_prefetch_desc(&tm_d);
    }
    if (warp == 1) {
        umma::tmem_alloc(&ctl->tmem_base, kTmemCols);
        umma::tmem_relinquish();
    }
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    const uint32_t tmem = ctl->tmem_base;

    // tile order: all signature tiles of one output-column block, then the
    // next block, so concurrently running CTAs share the W_down slab
    auto tile_coords = [&](int tile, int &s, int &nb) {
        nb = tile / n_sig;
        s = tile % n_sig;
    };
    auto union_word = [&](int s, int w) { return tile_union[(size_t)s * W + w]; };

    if (warp == 0) {
        uint32_t stage = 0, phase = 0, issued = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
            int s, nb;
            tile_coords(tile, s, nb);
            for (int w = 0; w < W && ok; ++w) {
                uint32_t bits = union_word(s, w);
                while (bits && ok) {
                    const int g = w * 32 + __ffs(bits) - 1;
                    bits &= bits - 1u;
                    for (int half = 0; half < kGS / kBK && ok; ++half) {
                        if (lane == 0) {
                            if (!wait_or_abort(&ctl->empty[stage], phase ^ 1u, ctl, status)) {
                                ok = false;
                            } else {
                                uint8_t *a = smem + stage * kStageBytes;
                                mbar_arrive_expect_tx(&ctl->full[stage], kStageBytes);
                                const int col = g * kGS + half * kBK;
                                tma_load_2d(a, &tm_h, col, s * kBM, &ctl->full[stage]);
                                tma_load_2d(a + kATile, &tm_d, col, nb * kBN, &ctl->full[stage]);
                            }
                        }
                        ok = __shfl_sync(0xffffffffu, ok, 0);
                        issued += ok ? 1u : 0u;
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
    } else if (warp == 1) {
        constexpr uint32_t idesc = umma::idesc_bf16_f32(kBM, kBN);
        uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
            int s, nb;
            tile_coords(tile, s, nb);
            if (lane == 0) {
                if (!wait_or_abort(&ctl->tempty[acc], acc_phase ^ 1u, ctl, status))
                    ok = false;
                umma::fence_after_sync();
                const uint32_t d = tmem + acc * (uint32_t)kBN;
                int kstep = 0;
                for (int w = 0; w < W && ok; ++w) {
                    int nbits = __popc(union_word(s, w));
                    for (int n = 0; n < nbits * (kGS / kBK) && ok; ++n) {
                        if (!wait_or_abort(&ctl->full[stage], phase, ctl, status)) {
                            ok = false;
                            break;
                        }
                        umma::fence_after_sync();
                        const uint32_t a = smem_u32(smem + stage * kStageBytes);
                        const uint32_t b = a + kATile;
#pragma unroll
                        for (int k = 0; k < kBK / 16; ++k)
                            umma::mma_bf16(d, umma::desc_kmajor_sw128(a + 32u * k),
                                           umma::desc_kmajor_sw128(b + 32u * k), idesc,
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
        const int j = q * 32 + lane;
        uint32_t acc = 0, acc_phase = 0;
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
            int s, nb;
            tile_coords(tile, s, nb);
            int nk = 0;
            for (int w = 0; w < W; ++w)
                nk += __popc(union_word(s, w));
            const int r = s * kBM + j;
            const long long orow = r < T ? (long long)sig_perm[r] : -1;
            if (!wait_or_abort(&ctl->tfull[acc], acc_phase, ctl, status))
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
                if (orow >= 0)
                    store_bf16x32(out + orow * H + (size_t)nb * kBN + c * 32, v);
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

size_t ffn_prefill_workspace(const wide_ffn_dims *d)
{
    const size_t wl = wide_worklist_bytes(d->tokens, d->inter / d->group_size, kBM);
    if (wl == 0)
        return 0;
    return align_up(wl, 1024) + align_up((size_t)d->tokens * (size_t)d->inter * 2, 1024);
}

int ffn_prefill_launch(const void *x, const void *wg, const void *wu, const void *wd,
                       const uint32_t *mask, void *out, const wide_ffn_dims *d, void *ws,
                       cudaStream_t s)
{
    const int64_t T = d->tokens, H = d->hidden, I = d->inter;
    const int64_t G = I / kGS;
    const int W = (int)((G + 31) / 32);
    const size_t wl_bytes = wide_worklist_bytes(T, G, kBM);
    wide_worklist wl;
    int rc = wide_worklist_carve(ws, wl_bytes, T, G, kBM, &wl);
    if (rc)
        return rc;
    __nv_bfloat16 *hbuf =
        reinterpret_cast<__nv_bfloat16 *>(static_cast<char *>(ws) + align_up(wl_bytes, 1024));

    CUtensorMap tg, tu, th, td;
    if (!make_tmap_2d(&tg, wg, I, H, H, 2, kGS, kBK, true) ||
        !make_tmap_2d(&tu, wu, I, H, H, 2, kGS, kBK, true) ||
        !make_tmap_2d(&th, hbuf, T, I, I, 2, kBM, kBK, true) ||
        !make_tmap_2d(&td, wd, H, I, I, 2, kBN, kBK, true))
        return WIDE_ECUDA;

    rc = reorder_launch(mask, T, G, kBM, &wl, s);
    if (rc)
        return rc;
    {
        LaunchScope scope(KID_PREFILL_ZERO, s);
        prefill_zero_dead<<<(unsigned)T, 128, 0, s>>>(mask, wl.sig_pos, hbuf, (int)T, (int)I,
                                                      (int)G, W);
    }
    if ((rc = launch_status()))
        return rc;
    const int sms = num_sms();
    if (sms <= 0)
        return WIDE_ECUDA;
    if (!raise_smem_limit(reinterpret_cast<const void *>(prefill_gateup), kSmemBytes) ||
        !raise_smem_limit(reinterpret_cast<const void *>(prefill_down), kSmemBytes))
        return WIDE_ECUDA;
    {
        const int64_t max_items = G * ((T + kBM - 1) / kBM);
        const int grid = (int)(max_items < sms ? max_items : sms);
        LaunchScope scope(KID_PREFILL_GATEUP, s);
        prefill_gateup<<<grid, kThreadsGU, kSmemBytes, s>>>(
            static_cast<const __nv_bfloat16 *>(x), tg, tu, wl.count, wl.perm, wl.items, wl.n_items, wl.sig_pos, hbuf, (int)T, (int)H,
            (int)I, status_ptr());
    }
    if ((rc = launch_status()))
        return rc;
    {
        const int64_t tiles = ((T + kBM - 1) / kBM) * (H / kBN);
        const int grid = (int)(tiles < sms ? tiles : sms);
        LaunchScope scope(KID_PREFILL_DOWN, s);
        prefill_down<<<grid, kThreads, kSmemBytes, s>>>(th, td, wl.tile_union, wl.sig_perm,
                                                        static_cast<__nv_bfloat16 *>(out),
                                                        (int)T, (int)H, (int)I, W, status_ptr());
    }
    return launch_status();
}

}  // namespace wide
