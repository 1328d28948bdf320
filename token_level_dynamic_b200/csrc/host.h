// host.h -- host-side helpers shared by the libwide entry points.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <mutex>

#include "wide.h"

namespace wide {

// Device address of this device's status word (looked up once per device
// and context).
int32_t *status_ptr();

// The device address of a module-scope __device__ variable on the current
// device.  In host code such a variable's name is only a host-side stand-in;
// its device address is looked up with cudaGetSymbolAddress, with the device
// current, once per (device, context): a cudaDeviceReset ends the context and
// the module's memory with it, and the next call looks the address up again
// in the new context.  Returns null if the lookup fails.
struct DeviceSymbolCache {
    std::mutex mu;
    void *ptr[64] = {};
    unsigned long long ctx[64] = {};
};
void *device_symbol_address(DeviceSymbolCache &cache, const void *symbol);
// Unique id of the current CUDA context (cuCtxGetId), 0 if there is none.
unsigned long long current_context_id();

// Encodes a 2-D row-major tensor map: `rows` x `cols` elements of
// `elem_bytes` bytes, row pitch `pitch_elems`, box `box_rows` x `box_cols`,
// 128-byte swizzle when `swizzle128` (box_cols * elem_bytes must be 128 then).
// Returns false if the driver rejects it.
bool make_tmap_2d(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                  uint64_t pitch_elems, uint32_t elem_bytes, uint32_t box_rows, uint32_t box_cols,
                  bool swizzle128);

// Encodes a bf16 row-major matrix (`rows` x `cols`, row pitch `pitch_elems`,
// cols % 64 == 0) as the 3-D tensor {64, cols / 64, rows}: a box
// {64, box_chunks, box_rows} copies box_rows rows of 64 * box_chunks
// consecutive elements each, landing as [box_rows][64 * box_chunks] in shared
// memory (no swizzle).  Long rows per copy stream better than 2-D boxes of
// short rows.
// As make_tmap_2d for bf16, with the shared-memory swizzle of the given
// width in bytes (0, 32, 64 or 128; the box's row must not be wider).
bool make_tmap_2d_swz(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                      uint64_t pitch_elems, uint32_t box_rows, uint32_t box_cols,
                      uint32_t swizzle_bytes);

// A bf16 3-D tensor (dims innermost first, byte strides of dims 1 and 2 in
// any order) with the given shared-memory swizzle (0, 32, 64 or 128 bytes).
bool make_tmap_3d_swz(CUtensorMap *map, const void *base, const uint64_t (&dims)[3],
                      const uint64_t (&strides)[2], const uint32_t (&box)[3],
                      uint32_t swizzle_bytes);

// The same for a 4-D tensor (byte strides of dims 1..3).
bool make_tmap_4d_swz(CUtensorMap *map, const void *base, const uint64_t (&dims)[4],
                      const uint64_t (&strides)[3], const uint32_t (&box)[4],
                      uint32_t swizzle_bytes);

bool make_tmap_rows3d(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                      uint64_t pitch_elems, uint32_t box_chunks, uint32_t box_rows);

// Encodes a 3-D tensor: dims (innermost first), byte strides of dims 1 and
// 2, box extents, no swizzle; bf16 (elem_bytes 2) or fp32 (4).
bool make_tmap_3d(CUtensorMap *map, const void *base, const uint64_t (&dims)[3],
                  const uint64_t (&strides)[2], const uint32_t (&box)[3], uint32_t elem_bytes);

// Encodes an fp32 [T][cols] activation stored with token pairs interleaved
// (row t/2 holds 2 * cols floats: tokens t and t+1 side by side per column)
// as the 3-D tensor {32, 2 * cols / 32, pairs} with 128-byte swizzle: a box
// {32, box_cols / 16, box_pairs} copies box_cols columns of box_pairs token
// pairs, landing as box_pairs x (box_cols / 16) rows of 128 bytes whose
// 16-byte chunks are XOR-permuted by (row & 7).  cols % 16 == 0.
bool make_tmap_f32_pairs(CUtensorMap *map, const float *base, uint64_t pairs, uint64_t cols,
                         uint32_t box_cols, uint32_t box_pairs);

// Raises a kernel's dynamic shared memory limit to at least `bytes` (once
// per kernel, device and size).
bool raise_smem_limit(const void *kernel, size_t bytes);

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Records "file:line: <last CUDA error>" as the calling thread's last error
// (wide_last_error), clears the CUDA error and returns WIDE_ECUDA.
int cuda_fail(const char *file, int line);
#define WIDE_CUDA_FAIL() ::wide::cuda_fail(__FILE__, __LINE__)

// Maps the last CUDA error to a WIDE code (and clears it).
#define launch_status()                                                                            \
    (cudaPeekAtLastError() == cudaSuccess ? WIDE_OK : WIDE_CUDA_FAIL())

// Kernel ids reported by the profiler (wide_kernel_name).
enum KernelId : int32_t {
    KID_REORDER_PARTITION_RANK = 1,
    KID_REORDER_FINISH = 2,
    KID_DECODE_GATEUP = 3,
    KID_DECODE_DOWN = 4,
    KID_PREFILL_GATEUP = 6,
    KID_PREFILL_DOWN = 7,
    KID_DECODE_QKV = 8,
    KID_DECODE_ATTN = 9,
    KID_RMSNORM = 10,
    KID_PREFILL_Q = 11,
    KID_PREFILL_KV = 12,
    KID_PREFILL_ATTN = 13,
    KID_PREFILL_OPROJ = 14,
    KID_ROUTER = 16,
    KID_ROUTER_SMALL = 17,
    KID_DECODE_FFN_SPLIT = 18,
    KID_DECODE_FFN_TC = 19,
    KID_FFN_PACK = 20,
};

// Pointers of one masked-layer call (FFN pointers unused when !ffn).
struct LayerPtrs {
    const void *x, *gamma1, *wq, *wk, *wv, *wo, *gamma2, *w_gate, *w_up, *w_down;
    void *k_cache, *v_cache;
    const uint32_t *head_mask, *ffn_mask;
    void *out, *attn_out, *ffn_out;
    bool ffn;
    const void *ffn_packed;   // wide_ffn_pack copy of the FFN weights, or NULL
};

// Brackets one kernel launch: counts it and, while profiling is on, records
// a begin event in the constructor and an end event in the destructor.
class LaunchScope {
  public:
    LaunchScope(int32_t kernel_id, cudaStream_t s);
    ~LaunchScope();

  private:
    int slot_;
    cudaStream_t s_;
};

// Whether *wl is a carved work list for (T, G, tile_m) with every array set.
bool worklist_matches(const wide_worklist *wl, int64_t T, int64_t G, int32_t tile_m);

// FFN argument checks shared by the FFN entry points (api.cu).
bool ffn_dims_ok(const wide_ffn_dims *d);
int ffn_path(const wide_ffn_dims *d);
bool ffn_shape_supported(const wide_ffn_dims *d, int path);

// Outputs of the decode down-projection GEMV (each pointer may be null):
// out_sum = the projection; out_total (element type of the weights) and
// out_total_f32 = the projection plus the residuals res_in (element type of
// the weights) and res_f32.  All [T][H] row-major.
struct DownOutputs {
    void *out_sum;
    const void *res_in;
    const float *res_f32;
    void *out_total;
    float *out_total_f32;
};

// ---- tcgen05 grouped GEMMs of the prefill path (prefill_gemm.cu)
enum GemmMode : int { GEMM_SWIGLU = 0, GEMM_ROPE_Q = 1, GEMM_KV = 2, GEMM_ROUTER = 3 };

struct GemmArgs {
    const __nv_bfloat16 *a;                   // [T][K] activation rows
    const int32_t *count, *perm, *items, *n_items_p, *sig_pos;  // work list (gathered modes)
    __nv_bfloat16 *out0, *out1;
    int T, K;
    int out_ld;          // SwiGLU: row stride of H (= inter)
    int gs;              // SwiGLU: channels per group (64 or 128)
    int group_cols;      // RoPE-Q: columns of one head group (rep * head_dim)
    int seq_len, n_kv, kv_blocks, m_tiles;
    int64_t cache_len, cache_cap;
    float log2_theta;
    // Router: B = W_r1 [rn][K]; the epilogue computes act(z) W_r2^T + b_r2
    // for the tile's tokens and writes the packed execute bits.
    const __nv_bfloat16 *w_r2;   // [G][rn]
    const float *b_r2;           // [G] or null
    uint32_t *mask_out;          // [T][ceil(G/32)]
    float *logits_out;           // [T][G] or null
    int rn, n_groups, act;
    int32_t *status;
};

struct UnionArgs {
    const uint32_t *tile_union;
    const int32_t *sig_perm;
    const uint32_t *mask;            // [T][W] group bits of the tokens (token order)
    const __nv_bfloat16 *h;          // A: [T][ld] rows in signature order (loaded by tm_a)
    int T, N, W, gs, ld;
    __nv_bfloat16 *out_sum;          // projection (optional)
    const __nv_bfloat16 *res_in;     // residual, bf16 (optional)
    const float *res_f32;            // residual, fp32 (optional)
    __nv_bfloat16 *out_total;        // projection + residuals, bf16 (optional)
    float *out_total_f32;            // projection + residuals, fp32 (optional)
    int32_t *status;
};

int gather_gemm_launch(int mode, const CUtensorMap &tm0, const CUtensorMap &tm1,
                       const GemmArgs &a, int max_work, int32_t kid, cudaStream_t s);
int tile_union_gemm_launch(const CUtensorMap &tm_a, const CUtensorMap &tm_b, const UnionArgs &a,
                           int32_t kid, cudaStream_t s);
int route_launch(const void *x, const void *w_r1, const void *w_r2, const float *b_r2,
                 uint32_t *mask, float *logits, const wide_router_dims *d, cudaStream_t s);

// Internal entry points of the kernel files.
int reorder_launch(const uint32_t *mask, int64_t T, int64_t G, int32_t tile_m,
                   const wide_worklist *wl, cudaStream_t s);
// Blocks per 256-position slice of the signature-rank kernel, and the bytes
// of reorder scratch (bucket histogram, member lists, rank counters).
int reorder_splits(int64_t T);
size_t reorder_scratch_bytes(int64_t T);

size_t ffn_prefill_workspace(const wide_ffn_dims *d);
// Outputs of the prefill FFN (each optional): out_sum = FFN(x); out_total =
// FFN(x) + res_f32.
struct FfnPrefillOut {
    __nv_bfloat16 *out_sum;
    const float *res_f32;
    __nv_bfloat16 *out_total;
};
// ext_wl: a caller-built work list of the same mask (tile_m 128), or null
// to reorder inside ws.
int ffn_prefill_core(const void *x, const void *wg, const void *wu, const void *wd,
                     const uint32_t *mask, const FfnPrefillOut &o, int64_t T, int64_t H,
                     int64_t I, int64_t gs, const wide_worklist *ext_wl, void *ws,
                     cudaStream_t s);
int ffn_prefill_launch(const void *x, const void *wg, const void *wu, const void *wd,
                       const uint32_t *mask, void *out, const wide_ffn_dims *d,
                       const wide_worklist *ext_wl, void *ws, cudaStream_t s);

bool layer_prefill_supported(const wide_layer_dims *d);
size_t layer_prefill_workspace(const wide_layer_dims *d);
int layer_prefill_launch(const LayerPtrs &p, const wide_layer_dims *d, void *ws, cudaStream_t s);

// RMSNorm of rows: y = x / sqrt(mean(x^2) + eps) * gamma, bf16 out.
int rmsnorm_bf16_launch(const void *x, const void *gamma, void *y, int T, int H, float eps,
                        cudaStream_t s);
int rmsnorm_f32_launch(const float *x, const void *gamma, void *y, int T, int H, float eps,
                       cudaStream_t s);

bool layer_decode_supported(const wide_layer_dims *d);
size_t layer_decode_workspace(const wide_layer_dims *d);
int layer_decode_launch(const LayerPtrs &p, const wide_layer_dims *d, void *ws, cudaStream_t s);

size_t ffn_decode_workspace(const wide_ffn_dims *d);
// bf16 decode GEMVs for T <= 32 tokens (one chunk): gate/up writes fp32 h for
// kept (token, group) pairs; down reads h of kept pairs (group size gs).
int decode_gateup_bf16(const void *x, const void *wg, const void *wu, const uint32_t *mask,
                       float *h, int T, int H, int I, int gs, cudaStream_t s);
int decode_down_bf16(const void *wd, const float *h, const uint32_t *mask, const DownOutputs &o,
                     int T, int H, int I, int gs, cudaStream_t s);
// bf16 decode FFN of 1 <= T <= kSplitMaxTok tokens as one persistent
// cooperative kernel in which every CTA owns a slice of the batch's kept
// channels
// (ffn_decode_split.cu).  x: bf16 [T][H].  scratch: device memory of at
// least decode_ffn_split_scratch(T, H) bytes (an fp32 [T][H] accumulator and
// an arrival counter, zeroed on the stream by the call).
constexpr int kSplitMaxTok = 16;   // tokens per launch of the split kernel
size_t decode_ffn_split_scratch(int T, int H);
bool decode_ffn_split_supported(int T, int H, int I, int gs);
int decode_ffn_split(const void *x, const void *wg, const void *wu, const void *wd,
                     const uint32_t *mask, const DownOutputs &o, int T, int H, int I, int gs,
                     void *scratch, cudaStream_t s);
// bf16 decode FFN of 1 <= T <= kTcMaxTok tokens on the tensor cores, one
// persistent cooperative kernel (ffn_decode_tc.cu); arguments and scratch
// as for decode_ffn_split.
constexpr int kTcMaxTok = 32;
size_t decode_ffn_tc_scratch(int T, int H);
bool decode_ffn_tc_supported(int T, int H, int I, int gs);
// `packed` (the wide_ffn_pack layout; NULL: the nn.Linear weights wg, wu,
// wd) selects where the weights are read from.
int decode_ffn_tc(const void *x, const void *wg, const void *wu, const void *wd,
                  const void *packed, const uint32_t *mask, const DownOutputs &o, int T, int H,
                  int I, int gs, void *scratch, cudaStream_t s);
bool decode_ffn_tc_packed_supported(int T, int H, int I, int gs);

// Packed decode weights (ffn_pack.cu): W_gate and W_up in 64-row panels,
// each panel K-step-major ([I/64][H/64][64][64]), then W_down in 16-channel
// column panels ([I/16][H][16]); 3 * I * H bf16 in all.
size_t ffn_packed_bytes(int64_t H, int64_t I);
int ffn_pack_launch(const void *wg, const void *wu, const void *wd, int64_t H, int64_t I,
                    void *packed, cudaStream_t s);
// The bf16 decode FFN of any T >= 1 on whichever persistent kernel the
// wide_set_decode_ffn_path mode and the shape allow, in launches of up to 32
// (tensor-core kernel) or 16 (channel-split kernel) tokens, with `cap` bytes
// of scratch.  WIDE_EUNSUPPORTED, with nothing enqueued, when neither
// applies: the caller then runs the GEMV kernels.
// `packed`: the wide_ffn_pack copy or NULL; wg / wu / wd may be NULL when
// only the packed copy is at hand (then only the tensor-core kernel applies).
bool decode_ffn_persistent_available(int64_t T, int H, int I, int gs, size_t cap,
                                     const void *packed = nullptr, bool linear = true);
int decode_ffn_persistent(const void *x, const void *wg, const void *wu, const void *wd,
                          const uint32_t *mask, const DownOutputs &o, int64_t T, int H, int I,
                          int gs, void *scratch, size_t cap, cudaStream_t s,
                          const void *packed = nullptr);
// Bytes of the fp32 h scratch of the decode path (tokens capped at 32).
size_t ffn_decode_h_bytes(const wide_ffn_dims *d);
// Runs the decode path with h scratch of h_cap contiguous bytes at h (at
// least ffn_decode_h_bytes(d); the persistent kernels run only where their
// accumulator and counter fit in h_cap).
// packed: an optional wide_ffn_pack copy of the weights, which the
// tensor-core kernel then reads.
int ffn_decode_run(const void *x, const void *wg, const void *wu, const void *wd,
                   const uint32_t *mask, void *out, const wide_ffn_dims *d, float *h,
                   size_t h_cap, cudaStream_t s, const void *packed = nullptr);
int ffn_decode_launch(const void *x, const void *wg, const void *wu, const void *wd,
                      const uint32_t *mask, void *out, const wide_ffn_dims *d, void *ws,
                      cudaStream_t s, const void *packed = nullptr);

}  // namespace wide
