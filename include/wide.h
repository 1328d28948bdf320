/*
 * wide.h -- C ABI of libwide.so, the B200 (sm_100a) masked-layer library.
 *
 * The method: "WIDE: Boosting Adaptive LLM Inference via Token-level Dynamic
 * Width Pruning".  Every token keeps or skips its own FFN channel groups
 * (contiguous groups of the intermediate dimension D') and its own attention
 * head groups (the query heads that share one KV head), technical summary
 * section 2.A.  Execution follows the pruning-kernel co-design of the
 * abstract and section 2.C: per-group mask reordering (section 2.B), then
 * block-level skipping (a tile with no active token does nothing) and
 * intra-block skipping (inactive rows of a partly active tile are neither
 * loaded nor multiplied).  Section 1 names the two costs this removes: a
 * synchronous mask-to-index conversion on the host and explicit
 * gather-scatter copies of activations; no entry point below synchronises
 * with the host or copies activations into a compacted buffer.
 *
 * Conventions for every entry point
 *   - Pointers named d_* or documented as "device" are device pointers on the
 *     current CUDA device; the caller owns every buffer.  The library never
 *     allocates or frees device memory.
 *   - stream is a cudaStream_t passed as void*; NULL is the legacy default
 *     stream.  All work is enqueued asynchronously on it.
 *   - Return value: WIDE_OK (0) or a negative WIDE_E* code for an error the
 *     host detects before launching anything (nothing is enqueued then).
 *     Errors found on the device (a mask bit at or above G, a bounded wait
 *     that gave up) set bits of a per-device status word, read with
 *     wide_get_device_status (the only call that synchronises).
 *   - bf16 tensors are IEEE bfloat16 bit patterns; all accumulation is fp32.
 *   - Matrices are row-major.  Weights use the nn.Linear layout
 *     [out_features][in_features].
 *   - A group mask is bit-packed, token-major: uint32 words[T][W] with
 *     W = ceil(G / 32); group g of token t is bit (g % 32) of words[t][g/32];
 *     a set bit means the token executes the group.  Bits at or above G
 *     must be zero.
 *   - Outputs must not alias inputs.
 */
#ifndef WIDE_H
#define WIDE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define WIDE_ABI_VERSION 3

/* host-side status codes */
#define WIDE_OK 0
#define WIDE_EINVAL -1        /* null pointer, negative or inconsistent size */
#define WIDE_EUNSUPPORTED -2  /* a shape or alignment this build does not run */
#define WIDE_EWORKSPACE -3    /* workspace smaller than the *_workspace_bytes query */
#define WIDE_ECUDA -4         /* a CUDA runtime/driver call failed */
#define WIDE_ETOOLARGE -5     /* exceeds the fixed scratch of wide_ffn_masked_noalloc */

/* device status word bits (wide_get_device_status) */
#define WIDE_DEV_BAD_MASK 0x1 /* a mask word had a bit at or above G set */
#define WIDE_DEV_TIMEOUT 0x2  /* a bounded wait inside a kernel gave up */
#define WIDE_DEV_BAD_ITEM 0x4 /* a work-list entry was out of range */
#define WIDE_DEV_LAYOUT 0x8   /* a kernel's shared-memory alignment precondition failed */

/* element types */
#define WIDE_BF16 0
#define WIDE_F32 1

/* FFN execution path */
#define WIDE_PATH_AUTO 0      /* decode for T <= 32, prefill otherwise */
#define WIDE_PATH_DECODE 1    /* CUDA-core GEMV over the batch's union of groups */
#define WIDE_PATH_PREFILL 2   /* reorder + tcgen05 grouped GEMMs (bf16 only) */

/* ------------------------------------------------------------------ status */

/* Human-readable text for a WIDE_* host code or a device status bit set. */
const char *wide_status_string(int code);

/* ABI version of the loaded library (WIDE_ABI_VERSION). */
int wide_abi_version(void);

/* After a call returned WIDE_ECUDA: "file:line: <CUDA error text>" of the
 * failing runtime or driver call, for the calling host thread ("" if none
 * yet).  The string is owned by the library and valid until the thread's
 * next failing call. */
const char *wide_last_error(void);

/* Synchronises `stream`, then copies the current device's status word into
 * *h_status (host pointer).  0 means no device-side error since the last
 * wide_clear_device_status. */
int wide_get_device_status(int32_t *h_status, void *stream);

/* Enqueues a reset of the current device's status word on `stream`. */
int wide_clear_device_status(void *stream);

/* ------------------------------------------------------------ measurement
 *
 * Kernel timing for benchmarks.  While profiling is on (host-global switch),
 * every kernel this library launches is bracketed by a pair of CUDA events
 * recorded on the launch stream; wide_profile_read synchronises on them and
 * returns one (kernel id, milliseconds) record per launch.  Off by default;
 * the events are created once, host side (no device allocation).
 */

/* Starts recording, keeping at most max_records launches (<= 65536). */
int wide_profile_start(int32_t max_records);

/* Stops recording new launches (records already taken stay readable). */
int wide_profile_stop(void);

/* Copies up to `max` records into kernel_ids[] / ms[] (host arrays), sets
 * *n to the number copied and clears the record list. */
int wide_profile_read(int32_t *kernel_ids, float *ms, int32_t max, int32_t *n);

/* Name of a kernel id ("?" when unknown). */
const char *wide_kernel_name(int32_t kernel_id);

/* Number of kernels this library has launched in this process. */
int64_t wide_launch_count(void);

/* --------------------------------------------------------- mask reordering
 *
 * Section 2.B: for each routing group, sort the binary mask along the token
 * dimension M so that the active tokens form a contiguous prefix; a tile of
 * that order is then a dense block with a known active prefix.  The sort is
 * the stable partition (active tokens ascending, then inactive ascending).
 * Also produced, for the kernels that sum over groups (FFN down projection):
 * a signature order of the tokens -- stable sort by the mask row read as one
 * big-endian unsigned key (word W-1 most significant) -- and the OR of the
 * mask rows of each tile_m-token tile of that order.
 *
 * All arrays are device memory inside one caller buffer laid out by
 * wide_worklist_carve; sizes:
 *   count[G], perm[G][T], items[G * ceil(T/tile_m)][2] (group, tile index;
 *   group-major; only tiles that hold an active token), n_items[1],
 *   sig_perm[T], sig_pos[T] (inverse of sig_perm),
 *   tile_union[ceil(T/tile_m)][W], plus reorder scratch.
 */
typedef struct wide_worklist {
    int32_t *count;
    int32_t *perm;
    int32_t *items;
    int32_t *n_items;
    int32_t *sig_perm;
    int32_t *sig_pos;
    uint32_t *tile_union;
    int32_t *scratch;      /* bucket histogram, member lists and rank counters, owned by wide_reorder */
    int64_t tokens, groups;
    int32_t tile_m, scratch_splits;
} wide_worklist;

/* Bytes of device memory a work list for (T, G, tile_m) needs (256-byte
 * aligned sub-arrays included).  Returns 0 for invalid arguments. */
size_t wide_worklist_bytes(int64_t T, int64_t G, int32_t tile_m);

/* Lays out the work-list arrays inside the device buffer `d_base` of
 * `bytes` bytes (>= wide_worklist_bytes; 256-byte aligned) and fills *wl
 * (host struct).  Enqueues nothing. */
int wide_worklist_carve(void *d_base, size_t bytes, int64_t T, int64_t G, int32_t tile_m,
                        wide_worklist *wl);

/* Builds the work list of section 2.B on the device from d_mask[T][W]
 * (device).  T >= 0, 1 <= G <= 1024, tile_m in {64, 128}.  No host sync;
 * n_items stays on the device.  A mask bit at or above G sets
 * WIDE_DEV_BAD_MASK (the outputs are then unspecified). */
int wide_reorder(const uint32_t *d_mask, int64_t T, int64_t G, int32_t tile_m,
                 const wide_worklist *wl, void *stream);

/* -------------------------------------------------------------- masked FFN
 *
 * Section 2.A, FFN half: for every token t and kept channel group g of
 * group_size consecutive channels c,
 *     h[t][c]  = silu(x[t] . W_gate[c]) * (x[t] . W_up[c])
 *     out[t]   = sum over kept groups g, c in g:  h[t][c] * W_down[:, c]
 * Skipped groups are never computed (and their W_down columns never read
 * for that token).
 *
 * Shapes: x[T][hidden], W_gate[inter][hidden], W_up[inter][hidden],
 * W_down[hidden][inter], group_mask[T][W] with G = inter / group_size,
 * out[T][hidden]; element type `dtype` for x, weights and out.  All device.
 *
 * Supported: hidden % 128 == 0; group_size in {32, 64, 128} dividing inter;
 * G <= 1024; 16-byte aligned pointers.  The bf16 decode path with
 * group_size 32 runs on the persistent kernels only (the GEMVs take 64 and
 * 128).  WIDE_PATH_PREFILL needs bf16, group_size 64 or 128 (or 32 with
 * inter % 64 == 0: the down projection takes the groups in pairs) and
 * hidden % 256 == 0.  The fp32 type runs the CUDA-core path at any T.
 */
typedef struct wide_ffn_dims {
    int64_t tokens;        /* T */
    int64_t hidden;        /* H */
    int64_t inter;         /* I (D' on the pages) */
    int64_t group_size;    /* channels per group */
    int32_t dtype;         /* WIDE_BF16 or WIDE_F32 */
    int32_t path;          /* WIDE_PATH_* */
} wide_ffn_dims;

/* Device workspace bytes wide_ffn_masked needs for `d` (0 on bad args). */
size_t wide_ffn_workspace_bytes(const wide_ffn_dims *d);

/* Masked SwiGLU FFN.  d_workspace: device, >= wide_ffn_workspace_bytes(d)
 * bytes, 256-byte aligned, contents need not be initialised and are
 * clobbered.  Calls that share a workspace must be ordered on one stream.
 *
 * wl (host struct of device pointers, optional): a work list that
 * wide_reorder already built from this same d_group_mask with
 * tile_m == 128 and G = inter / group_size, so a caller that routes once
 * can reuse one reordering across calls (section 2.B: the reordering is a
 * function of the mask alone).  NULL: the prefill path reorders inside the
 * workspace.  With a work list the prefill path reads it and does not
 * reorder; the caller must have enqueued that wide_reorder on `stream` (or
 * ordered it before this call) and must not change the mask in between --
 * a work list built from another mask gives wrong results, not an error.
 * The work list's arrays are only read.  A work list whose tokens, groups
 * or tile_m do not match returns WIDE_EINVAL.  The decode path computes the
 * batch's union of groups inside its kernel and reads no work list; wl is
 * checked the same way there and otherwise ignored.  The workspace size
 * does not depend on wl. */
int wide_ffn_masked(const void *d_x, const void *d_w_gate, const void *d_w_up,
                    const void *d_w_down, const uint32_t *d_group_mask, void *d_out,
                    const wide_ffn_dims *d, const wide_worklist *wl, void *d_workspace,
                    size_t workspace_bytes, void *stream);

/* Kernels of the bf16 decode FFN (process-wide; the decode layer's FFN
 * follows it too).  All compute the same sums, in a different fp32 order:
 *   WIDE_DECODE_AUTO   the channel-split kernel for up to 8 tokens per
 *                      launch, the tensor-core kernel above (on a packed
 *                      copy where the call has one), each where its shape
 *                      limits allow, else the GEMVs (default)
 *   WIDE_DECODE_TC     the tensor-core kernel: one persistent kernel per launch of
 *                      up to 32 tokens (hidden % 128 == 0, group size a
 *                      multiple of 16 up to 256); each CTA owns a slice of
 *                      the union's channels, runs gate/up and its share of
 *                      the down projection as tcgen05 MMAs (h rounded to
 *                      bf16 between them) and adds that share into an fp32
 *                      accumulator with atomics, so two calls can differ in
 *                      the last fp32 bits
 *   WIDE_DECODE_FUSED  the channel-split CUDA-core kernel, launches of up to
 *                      16 tokens (hidden % 256 == 0, group size a multiple
 *                      of 8 up to 256), atomics as above
 *   WIDE_DECODE_GEMV   the gate/up GEMV kernel, then the down GEMV kernel
 *                      (bitwise repeatable); bf16 group size 32 has no GEMV
 *                      kernel and runs on a persistent kernel
 * Returns the previous mode, or WIDE_EINVAL for an unknown mode (the mode
 * is then unchanged).  Not ordered with work already enqueued: it applies
 * to calls made after it returns. */
#define WIDE_DECODE_AUTO 0
#define WIDE_DECODE_FUSED 1
#define WIDE_DECODE_GEMV 2
#define WIDE_DECODE_TC 3
int wide_set_decode_ffn_path(int mode);

/* ------------------------------------------------- packed decode weights
 *
 * The decode FFN reads every kept weight byte once per call, so it runs at
 * the speed HBM delivers the union's weights.  The tensor cores take a
 * K-major bf16 operand from shared memory in atoms of 8 rows x 128 bytes;
 * from the nn.Linear layout such a tile is 128-byte pieces of rows that lie
 * kilobytes apart, which B200 HBM serves at about half its bandwidth.  A
 * packed copy holds the same weights with every tile the decode kernel loads
 * stored as one contiguous run:
 *   W_gate, W_up  interleaved, [inter / 64][hidden / 64][4][2][16][64]:
 *                 64-channel panels, K-step-major, inside each K step four
 *                 16-channel groups of 16 W_gate rows then the same 16 W_up
 *                 rows (element [p][k][q][s][r][e] = (s ? W_up : W_gate)
 *                 [64p + 16q + r][64k + e]);
 *   W_down        [inter / 16][hidden][16] (element [c][n][e] =
 *                 W_down[n][16c + e]),
 * in that order in one buffer.  The values are copied bitwise, so results
 * equal those of the nn.Linear weights up to the fp32 summation order.
 * Pack once when the weights are loaded; the copy costs as much device
 * memory as the FFN weights.  Supported: hidden % 128 == 0, inter % 64 == 0.
 */

/* Bytes of the packed copy (3 * hidden * inter * 2), or 0 if unsupported. */
size_t wide_ffn_packed_bytes(int64_t hidden, int64_t inter);

/* Writes the packed copy of W_gate, W_up [inter][hidden] and W_down
 * [hidden][inter] (device, bf16, 16-byte aligned) into d_packed (device,
 * >= wide_ffn_packed_bytes, 256-byte aligned).  Enqueued on `stream`. */
int wide_ffn_pack(const void *d_w_gate, const void *d_w_up, const void *d_w_down, int64_t hidden,
                  int64_t inter, void *d_packed, size_t packed_bytes, void *stream);

/* The masked FFN of wide_ffn_masked, decode path, reading the packed copy
 * in the tensor-core kernel (launches of up to 32 tokens, any token count).
 * d_w_gate, d_w_up, d_w_down: the nn.Linear weights as well (all three) or
 * NULL (all three).  With them the call picks the kernel per launch as the
 * wide_set_decode_ffn_path mode says (AUTO: the channel-split kernel for up
 * to 8 tokens, where it is faster, the tensor-core kernel on the packed copy
 * above); without them the tensor-core kernel runs every launch.  bf16
 * only; d->path WIDE_PATH_AUTO or WIDE_PATH_DECODE (PREFILL:
 * WIDE_EUNSUPPORTED); group size a multiple of 16 up to 256; the same
 * workspace as wide_ffn_masked's decode path (wide_ffn_workspace_bytes with
 * path WIDE_PATH_DECODE).  Atomics order the fp32 sums differently from
 * call to call (see WIDE_DECODE_TC). */
int wide_ffn_masked_packed(const void *d_x, const void *d_packed, const void *d_w_gate,
                           const void *d_w_up, const void *d_w_down, const uint32_t *d_group_mask,
                           void *d_out, const wide_ffn_dims *d, void *d_workspace,
                           size_t workspace_bytes, void *stream);

/* --------------------------------------------------- masked attention / layer
 *
 * Section 2.A, attention half: a token that skips head group j (the
 * n_q_heads / n_kv_heads query heads sharing KV head j) computes neither
 * those query heads nor their attention, and their o_proj columns are not
 * read for it.  K and V are computed for every token and group and written
 * to the cache.  The pages fix nothing else about the layer; it is the
 * Llama pre-norm block (RMSNorm, rotate-half RoPE with base rope_theta,
 * softmax scale 1/sqrt(head_dim), SwiGLU FFN):
 *     h1  = x + o_proj(attn(RMSNorm(x) * gamma1))        (attn_out = o_proj(...))
 *     out = h1 + FFN(RMSNorm(h1) * gamma2)               (ffn_out = FFN(...))
 * with the FFN masked per token as in wide_ffn_masked.
 *
 * Token t = s * seq_len + i is token i of sequence s, at position
 * cache_len + i; its K/V go to the caches at that position.  Caches are
 * bf16 [n_seq][n_kv_heads][cache_cap][head_dim]; positions < cache_len must
 * already hold (post-RoPE) keys and values.  Masks: head_mask [T][W] over
 * n_kv_heads groups; ffn_mask [T][W] over inter / ffn_group_size groups.
 *
 * Supported: bf16; head_dim == 128; ffn_group_size in {64, 128} dividing
 * inter; and one of two forms:
 *   decode  (seq_len == 1): n_seq <= 32, n_q_heads / n_kv_heads in
 *           {1, 2, 4}, n_kv_heads <= 1024, hidden % 512 == 0,
 *           cache_len < 131072, cache_cap >= cache_len + 1;
 *   prefill (seq_len >= 1 with cache_len == 0, i.e. no earlier context):
 *           n_kv_heads even, 2..1024, n_q_heads / n_kv_heads in {2, 4},
 *           ffn_group_size 32 also (with inter % 64 == 0),
 *           hidden % 256 == 0, inter / ffn_group_size <= 1024,
 *           cache_cap >= seq_len, n_seq * seq_len <= 2^24 and
 *           n_kv_heads * n_seq * seq_len <= 2^22.
 * Dims that both forms accept (seq_len == 1, cache_len == 0) run the decode
 * form.  Anything else
 * (a prefill chunk after cached context, other head ratios) returns
 * WIDE_EUNSUPPORTED.
 */
typedef struct wide_layer_dims {
    int64_t n_seq;           /* sequences */
    int64_t seq_len;         /* new tokens per sequence (1 = decode) */
    int64_t cache_len;       /* positions already in the cache */
    int64_t cache_cap;       /* cache capacity per (sequence, KV head) */
    int64_t hidden;
    int64_t inter;           /* FFN intermediate size (ignored by wide_attn_masked) */
    int64_t ffn_group_size;
    int32_t n_q_heads, n_kv_heads, head_dim;
    float rope_theta;
    float eps;               /* RMSNorm epsilon */
} wide_layer_dims;

typedef struct wide_layer_weights {
    const void *gamma1, *wq, *wk, *wv, *wo;       /* attention half (device) */
    const void *gamma2, *w_gate, *w_up, *w_down;  /* FFN half (device) */
    const void *ffn_packed;   /* optional wide_ffn_pack copy of the FFN weights
                                 (NULL: none); the decode layer's FFN reads it
                                 where the tensor-core kernel takes the shape */
} wide_layer_weights;

/* Device workspace bytes for wide_layer_masked / wide_attn_masked (0 on
 * invalid or unsupported dims). */
size_t wide_layer_workspace_bytes(const wide_layer_dims *d);

/* The masked layer.  out [T][hidden] (required); attn_out and ffn_out
 * [T][hidden] are optional (NULL = not written).  Appends K/V to the caches.
 * Workspace: >= wide_layer_workspace_bytes(d), 256-byte aligned. */
int wide_layer_masked(const void *d_x, const wide_layer_weights *w, void *d_k_cache,
                      void *d_v_cache, const uint32_t *d_head_mask, const uint32_t *d_ffn_mask,
                      void *d_out, void *d_attn_out, void *d_ffn_out, const wide_layer_dims *d,
                      void *d_workspace, size_t workspace_bytes, void *stream);

/* The attention half only: attn_out = o_proj(attn(RMSNorm(x) * gamma1)) with
 * the head-group mask; appends K/V to the caches.  w->gamma2 and the FFN
 * weights are ignored. */
int wide_attn_masked(const void *d_x, const wide_layer_weights *w, void *d_k_cache,
                     void *d_v_cache, const uint32_t *d_head_mask, void *d_attn_out,
                     const wide_layer_dims *d, void *d_workspace, size_t workspace_bytes,
                     void *stream);

/* ------------------------------------------- FFN without device allocation
 *
 * The paper has no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory or hand the library a workspace (for
 * example code inside a host framework that owns the whole device memory
 * pool, or a latency-critical loop where cudaMalloc/cudaFree would
 * synchronise the device).
 *
 * Same operation, arguments and layouts as wide_ffn_masked on its decode
 * path (the kernels the wide_set_decode_ffn_path mode picks, over the
 * batch's union of groups), minus the workspace: the kernels' scratch (fp32
 * h for up to 32 tokens x inter channels, or a persistent kernel's fp32
 * accumulator and arrival counter) lives in a fixed device array inside the
 * library of WIDE_NOALLOC_SCRATCH_BYTES bytes, which every GPU that loads
 * the library holds until the process exits.  Limit: min(tokens, 32),
 * rounded up to an even count, * inter * 4 bytes, and min(tokens, 32)
 * rounded up to a multiple of 4, * hidden * 4 bytes, must not exceed it
 * (inter <= 16384 at 32 tokens); larger problems return WIDE_ETOOLARGE
 * before anything is enqueued.  A persistent kernel runs only where its
 * accumulator and counter fit in the array (else the GEMV kernels).  The
 * call allocates nothing.
 * Its first call on a device looks up the array's device address (once per
 * device and CUDA context, with that device current: after a
 * cudaDeviceReset the next call looks it up again); make that first call
 * before any stream capture.  All calls on a device share the array, which
 * keeps the last call's contents (no call depends on them: what a kernel
 * needs zeroed it zeroes on the stream first); calls that overlap on the GPU
 * -- on streams not ordered with each other -- race on it.
 * d->path must be WIDE_PATH_AUTO or WIDE_PATH_DECODE. */
#define WIDE_NOALLOC_SCRATCH_BYTES 2097152
int wide_ffn_masked_noalloc(const void *d_x, const void *d_w_gate, const void *d_w_up,
                            const void *d_w_down, const uint32_t *d_group_mask, void *d_out,
                            const wide_ffn_dims *d, void *stream);

/* ------------------------------------------------------------------ router
 *
 * Technical summary section 2.A, "router architecture": a light bottleneck
 * router maps a block's input activations to one binary decision per group,
 * execute or skip (Gumbel-Softmax relaxes that decision in training only).
 * The pages give no formula; this call computes, for every token t,
 *     z[t]        = act(x[t] W_r1^T)                      [rn]
 *     logit[t][g] = z[t] . W_r2[g] + b_r2[g]              (b_r2 = 0 if NULL)
 *     execute     = logit[t][g] > 0                       (0 skips)
 * and writes the decisions straight into the packed mask words that
 * wide_reorder, wide_ffn_masked and wide_layer_masked read, so no dense
 * per-(token, group) byte or float mask exists on the device.
 *
 *   d_x       bf16 [tokens][hidden], the sublayer's (normalised) input
 *   d_w_r1    bf16 [bottleneck][hidden]          (nn.Linear layout)
 *   d_w_r2    bf16 [groups][bottleneck]
 *   d_b_r2    fp32 [groups] or NULL
 *   d_mask    out: uint32 [tokens][ceil(groups / 32)]; every word written,
 *             bits at or above groups zero
 *   d_logits  out: fp32 [tokens][groups] (the values the decisions were
 *             taken on), or NULL
 * Arithmetic: for more than 32 tokens x W_r1^T runs on tcgen05 tensor
 * cores (bf16 operands, fp32 accumulation in tensor memory), for up to 32
 * on CUDA cores in fp32 (when that kernel's shared memory, about
 * (bottleneck / 4 + 4) * hidden + 4 * groups * (bottleneck / 8 + 2) bytes,
 * fits in 227 KB; otherwise on the tensor-core kernel too); the activation
 * and the W_r2 products are fp32 on CUDA cores; no intermediate is rounded
 * to bf16.  A decision can differ
 * between the two kernels, or from an fp64 evaluation, only where the logit
 * is within fp32 rounding of 0.
 * Supported: hidden a multiple of 64; bottleneck a multiple of 32 in
 * [32, 256]; groups in [1, 1024]; tokens * hidden < 2^31; d_x, d_w_r1 and
 * d_w_r2 16-byte aligned (else WIDE_EUNSUPPORTED).  tokens == 0 enqueues
 * nothing.  No workspace; nothing is allocated. */
#define WIDE_ACT_RELU 0
#define WIDE_ACT_SILU 1
typedef struct wide_router_dims {
    int64_t tokens;
    int64_t hidden;
    int64_t bottleneck;
    int64_t groups;
    int32_t act; /* WIDE_ACT_RELU or WIDE_ACT_SILU */
} wide_router_dims;

int wide_route(const void *d_x, const void *d_w_r1, const void *d_w_r2, const float *d_b_r2,
               uint32_t *d_mask, float *d_logits, const wide_router_dims *d, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* WIDE_H */
