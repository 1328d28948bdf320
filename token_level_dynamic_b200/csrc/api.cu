// api.cu -- the extern "C" entry points of libwide.so (declared in wide.h):
// argument validation, work-list layout, tensor-map encoding and the
// per-device status word.  The kernels live in the other .cu files.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdio.h>
#include <string.h>
#include <mutex>
#include <set>
#include <utility>

#include "host.h"
#include "wide.h"

// Per-device status word: each device that loads this module gets its own
// copy.  Kernels set WIDE_DEV_* bits in it; wide_get_device_status reads it.
__device__ int32_t g_wide_status;

namespace wide {

// Text of the calling thread's last CUDA failure (wide_last_error).
thread_local char g_last_error[256] = "";

int cuda_fail(const char *file, int line)
{
    const cudaError_t e = cudaGetLastError();
    const char *base = strrchr(file, '/');
    snprintf(g_last_error, sizeof g_last_error, "%s:%d: %s", base ? base + 1 : file, line,
             e == cudaSuccess ? "a CUDA driver call failed (no runtime error recorded)"
                              : cudaGetErrorString(e));
    return WIDE_ECUDA;
}

namespace {
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);
}  // namespace

unsigned long long current_context_id()
{
    static CtxGetCurrentFn get_cur = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr, *q = nullptr;
        cudaDriverEntryPointQueryResult r1, r2;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault,
                                             &r1) == cudaSuccess &&
            r1 == cudaDriverEntryPointSuccess &&
            cudaGetDriverEntryPointByVersion("cuCtxGetId", &q, 12000, cudaEnableDefault, &r2) ==
                cudaSuccess &&
            r2 == cudaDriverEntryPointSuccess) {
            get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
            get_id = reinterpret_cast<CtxGetIdFn>(q);
        }
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_cur || !get_id || get_cur(&ctx) != CUDA_SUCCESS || !ctx ||
        get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

void *device_symbol_address(DeviceSymbolCache &cache, const void *symbol)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return nullptr;
    std::lock_guard<std::mutex> lock(cache.mu);
    const unsigned long long id = current_context_id();
    if (cache.ptr[dev] && id != 0 && cache.ctx[dev] == id)
        return cache.ptr[dev];
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, symbol) != cudaSuccess)
        return nullptr;
    cache.ptr[dev] = p;
    cache.ctx[dev] = current_context_id();
    return p;
}

int32_t *status_ptr()
{
    static DeviceSymbolCache cache;
    return static_cast<int32_t *>(device_symbol_address(cache, &g_wide_status));
}

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

}  // namespace

bool make_tmap_2d(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                  uint64_t pitch_elems, uint32_t elem_bytes, uint32_t box_rows, uint32_t box_cols,
                  bool swizzle128)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn || rows == 0 || cols == 0)
        return false;
    const CUtensorMapDataType dt =
        elem_bytes == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {pitch_elems * elem_bytes};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r =
        fn(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE,
           swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_tmap_2d_swz(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                      uint64_t pitch_elems, uint32_t box_rows, uint32_t box_cols,
                      uint32_t swizzle_bytes)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn || rows == 0 || cols == 0 || box_cols * 2 > (swizzle_bytes ? swizzle_bytes : 512))
        return false;
    const CUtensorMapSwizzle sw = swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                  : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                        : CU_TENSOR_MAP_SWIZZLE_NONE;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {pitch_elems * 2};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_tmap_3d_swz(CUtensorMap *map, const void *base, const uint64_t (&dims)[3],
                      const uint64_t (&strides)[2], const uint32_t (&box)[3],
                      uint32_t swizzle_bytes)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn || box[0] * 2 > (swizzle_bytes ? swizzle_bytes : 512))
        return false;
    const CUtensorMapSwizzle sw = swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                  : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                        : CU_TENSOR_MAP_SWIZZLE_NONE;
    const cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
    const cuuint64_t st[2] = {strides[0], strides[1]};
    const cuuint32_t b[3] = {box[0], box[1], box[2]};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), d,
                          st, b, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_tmap_4d_swz(CUtensorMap *map, const void *base, const uint64_t (&dims)[4],
                      const uint64_t (&strides)[3], const uint32_t (&box)[4],
                      uint32_t swizzle_bytes)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn || box[0] * 2 > (swizzle_bytes ? swizzle_bytes : 512))
        return false;
    const CUtensorMapSwizzle sw = swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                  : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                  : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                        : CU_TENSOR_MAP_SWIZZLE_NONE;
    const cuuint64_t d[4] = {dims[0], dims[1], dims[2], dims[3]};
    const cuuint64_t st[3] = {strides[0], strides[1], strides[2]};
    const cuuint32_t b[4] = {box[0], box[1], box[2], box[3]};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), d,
                          st, b, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_tmap_rows3d(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                      uint64_t pitch_elems, uint32_t box_chunks, uint32_t box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn || rows == 0 || cols == 0 || cols % 64 != 0)
        return false;
    const cuuint64_t dims[3] = {64, cols / 64, rows};
    const cuuint64_t strides[2] = {128, pitch_elems * 2};
    const cuuint32_t box[3] = {64, box_chunks, box_rows};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r =
        fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_tmap_3d(CUtensorMap *map, const void *base, const uint64_t (&dims)[3],
                  const uint64_t (&strides)[2], const uint32_t (&box)[3], uint32_t elem_bytes)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    const CUtensorMapDataType dt =
        elem_bytes == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
    const cuuint64_t st[2] = {strides[0], strides[1]};
    const cuuint32_t b[3] = {box[0], box[1], box[2]};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r =
        fn(map, dt, 3, const_cast<void *>(base), d, st, b, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
           CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_tmap_f32_pairs(CUtensorMap *map, const float *base, uint64_t pairs, uint64_t cols,
                         uint32_t box_cols, uint32_t box_pairs)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn || pairs == 0 || cols == 0 || cols % 16 != 0 || box_cols % 16 != 0)
        return false;
    const cuuint64_t dims[3] = {32, 2 * cols / 32, pairs};
    const cuuint64_t strides[2] = {128, 2 * cols * 4};
    const cuuint32_t box[3] = {32, box_cols / 16, box_pairs};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r =
        fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float *>(base), dims, strides, box,
           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool raise_smem_limit(const void *kernel, size_t bytes)
{
    // The attribute is an upper bound, so it is raised once per (kernel,
    // device) to the device's opt-in maximum; lowering it for a smaller
    // launch would break a later, larger one.
    static std::mutex mu;
    static std::set<std::pair<const void *, int>> done;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return false;
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_pair(kernel, dev);
    int optin = 0;
    if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
        cudaSuccess)
        return false;
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess)
        return false;
    const int limit = optin - (int)fa.sharedSizeBytes;  // static + dynamic <= opt-in
    if (bytes > (size_t)limit)
        return false;
    if (done.count(key))
        return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, limit) !=
        cudaSuccess)
        return false;
    done.insert(key);
    return true;
}

namespace {

struct WorklistLayout {
    size_t count, perm, items, n_items, sig_perm, sig_pos, tile_union, scratch, total;
    int splits;
};

bool worklist_layout(int64_t T, int64_t G, int32_t tile_m, WorklistLayout *L)
{
    if (T < 0 || T > (1 << 24) || G < 1 || G > 1024 || (tile_m != 64 && tile_m != 128))
        return false;
    const size_t W = (size_t)((G + 31) / 32);
    const size_t nt = (size_t)((T + tile_m - 1) / tile_m);
    const size_t t = (size_t)T;
    L->splits = reorder_splits(T);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += align_up(bytes > 0 ? bytes : 1, 256);
        return at;
    };
    L->count = take(4 * (size_t)G);
    L->perm = take(4 * (size_t)G * t);
    L->items = take(8 * (size_t)G * nt);
    L->n_items = take(4);
    L->sig_perm = take(4 * t);
    L->sig_pos = take(4 * t);
    L->tile_union = take(4 * nt * W);
    L->scratch = take(reorder_scratch_bytes(T));
    L->total = off;
    return true;
}

}  // namespace

bool worklist_matches(const wide_worklist *wl, int64_t T, int64_t G, int32_t tile_m)
{
    WorklistLayout L;
    if (!wl || !worklist_layout(T, G, tile_m, &L))
        return false;
    if (wl->tokens != T || wl->groups != G || wl->tile_m != tile_m ||
        wl->scratch_splits != L.splits)
        return false;
    return wl->count && wl->perm && wl->items && wl->n_items && wl->sig_perm && wl->sig_pos &&
           wl->tile_union && wl->scratch;
}

bool ffn_dims_ok(const wide_ffn_dims *d)
{
    if (!d || d->tokens < 0 || d->hidden <= 0 || d->inter <= 0 || d->group_size <= 0)
        return false;
    if (d->dtype != WIDE_BF16 && d->dtype != WIDE_F32)
        return false;
    if (d->path < WIDE_PATH_AUTO || d->path > WIDE_PATH_PREFILL)
        return false;
    return d->inter % d->group_size == 0 && d->inter / d->group_size <= 1024;
}

int ffn_path(const wide_ffn_dims *d)
{
    if (d->path != WIDE_PATH_AUTO)
        return d->path;
    return (d->dtype == WIDE_F32 || d->tokens <= 32) ? WIDE_PATH_DECODE : WIDE_PATH_PREFILL;
}

bool ffn_shape_supported(const wide_ffn_dims *d, int path)
{
    if (d->hidden % 128 != 0 || d->hidden > (1 << 20) || d->inter > (1 << 22))
        return false;
    const int64_t gs = d->group_size;
    if (path == WIDE_PATH_DECODE) {
        if (d->dtype != WIDE_BF16)
            return gs == 32 || gs == 64 || gs == 128;
        // bf16 group size 32 runs on the persistent kernels only
        const int T1 = (int)(d->tokens < kSplitMaxTok ? (d->tokens > 0 ? d->tokens : 1)
                                                      : kSplitMaxTok);
        const int H = (int)d->hidden, I = (int)d->inter;
        return gs == 64 || gs == 128 ||
               (gs == 32 && (decode_ffn_split_supported(T1, H, I, 32) ||
                             decode_ffn_tc_supported(T1, H, I, 32)));
    }
    // prefill: tcgen05 kernels, 256-column output blocks; 32-channel groups
    // go through the down projection in pairs (64-column stages)
    return d->dtype == WIDE_BF16 && (gs == 64 || gs == 128 || (gs == 32 && d->inter % 64 == 0)) &&
           d->hidden % 256 == 0 && d->tokens <= (1 << 24);
}

}  // namespace wide

using namespace wide;

extern "C" {

const char *wide_status_string(int code)
{
    switch (code) {
    case WIDE_OK:
        return "ok";
    case WIDE_EINVAL:
        return "invalid argument (null pointer, negative or inconsistent size)";
    case WIDE_EUNSUPPORTED:
        return "unsupported shape, type or alignment";
    case WIDE_EWORKSPACE:
        return "workspace too small";
    case WIDE_ECUDA:
        return "CUDA runtime or driver call failed";
    case WIDE_ETOOLARGE:
        return "problem larger than the fixed scratch of wide_ffn_masked_noalloc";
    case WIDE_DEV_BAD_MASK:
        return "device: mask bit at or above G";
    case WIDE_DEV_TIMEOUT:
        return "device: bounded wait gave up";
    case WIDE_DEV_BAD_ITEM:
        return "device: work item out of range";
    case WIDE_DEV_LAYOUT:
        return "device: shared-memory alignment precondition failed";
    default:
        return code > 0 ? "device: several error bits" : "unknown status";
    }
}

int wide_abi_version(void) { return WIDE_ABI_VERSION; }

const char *wide_last_error(void) { return wide::g_last_error; }

int wide_get_device_status(int32_t *h_status, void *stream)
{
    if (!h_status)
        return WIDE_EINVAL;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return WIDE_CUDA_FAIL();
    if (cudaMemcpyFromSymbol(h_status, g_wide_status, sizeof(int32_t)) != cudaSuccess)
        return WIDE_CUDA_FAIL();
    return WIDE_OK;
}

int wide_clear_device_status(void *stream)
{
    int32_t *p = status_ptr();
    if (!p)
        return WIDE_CUDA_FAIL();
    return cudaMemsetAsync(p, 0, sizeof(int32_t), static_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? WIDE_OK
               : WIDE_CUDA_FAIL();
}

size_t wide_worklist_bytes(int64_t T, int64_t G, int32_t tile_m)
{
    WorklistLayout L;
    return worklist_layout(T, G, tile_m, &L) ? L.total : 0;
}

int wide_worklist_carve(void *d_base, size_t bytes, int64_t T, int64_t G, int32_t tile_m,
                        wide_worklist *wl)
{
    WorklistLayout L;
    if (!wl || !d_base || !worklist_layout(T, G, tile_m, &L))
        return WIDE_EINVAL;
    if ((reinterpret_cast<uintptr_t>(d_base) & 255u) != 0)
        return WIDE_EUNSUPPORTED;
    if (bytes < L.total)
        return WIDE_EWORKSPACE;
    char *b = static_cast<char *>(d_base);
    wl->count = reinterpret_cast<int32_t *>(b + L.count);
    wl->perm = reinterpret_cast<int32_t *>(b + L.perm);
    wl->items = reinterpret_cast<int32_t *>(b + L.items);
    wl->n_items = reinterpret_cast<int32_t *>(b + L.n_items);
    wl->sig_perm = reinterpret_cast<int32_t *>(b + L.sig_perm);
    wl->sig_pos = reinterpret_cast<int32_t *>(b + L.sig_pos);
    wl->tile_union = reinterpret_cast<uint32_t *>(b + L.tile_union);
    wl->scratch = reinterpret_cast<int32_t *>(b + L.scratch);
    wl->tokens = T;
    wl->groups = G;
    wl->tile_m = tile_m;
    wl->scratch_splits = L.splits;
    return WIDE_OK;
}

int wide_reorder(const uint32_t *d_mask, int64_t T, int64_t G, int32_t tile_m,
                 const wide_worklist *wl, void *stream)
{
    if (!worklist_matches(wl, T, G, tile_m) || (T > 0 && !d_mask))
        return WIDE_EINVAL;
    return reorder_launch(d_mask, T, G, tile_m, wl, static_cast<cudaStream_t>(stream));
}

size_t wide_ffn_workspace_bytes(const wide_ffn_dims *d)
{
    if (!ffn_dims_ok(d))
        return 0;
    const int path = ffn_path(d);
    if (path == WIDE_PATH_DECODE)
        return ffn_decode_workspace(d);
    return ffn_prefill_workspace(d);
}

int wide_ffn_masked(const void *d_x, const void *d_w_gate, const void *d_w_up,
                    const void *d_w_down, const uint32_t *d_group_mask, void *d_out,
                    const wide_ffn_dims *d, const wide_worklist *wl, void *d_workspace,
                    size_t workspace_bytes, void *stream)
{
    if (!ffn_dims_ok(d))
        return WIDE_EINVAL;
    if (wl && !worklist_matches(wl, d->tokens, d->inter / d->group_size, 128))
        return WIDE_EINVAL;
    if (d->tokens == 0)
        return WIDE_OK;
    if (!d_x || !d_w_gate || !d_w_up || !d_w_down || !d_group_mask || !d_out || !d_workspace)
        return WIDE_EINVAL;
    const int path = ffn_path(d);
    if (!ffn_shape_supported(d, path))
        return WIDE_EUNSUPPORTED;
    if (!aligned16(d_x) || !aligned16(d_w_gate) || !aligned16(d_w_up) || !aligned16(d_w_down) ||
        !aligned16(d_out) || (reinterpret_cast<uintptr_t>(d_workspace) & 255u) != 0)
        return WIDE_EUNSUPPORTED;
    if (workspace_bytes < wide_ffn_workspace_bytes(d))
        return WIDE_EWORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (path == WIDE_PATH_DECODE)
        return ffn_decode_launch(d_x, d_w_gate, d_w_up, d_w_down, d_group_mask, d_out, d,
                                 d_workspace, s);
    return ffn_prefill_launch(d_x, d_w_gate, d_w_up, d_w_down, d_group_mask, d_out, d, wl,
                              d_workspace, s);
}

size_t wide_ffn_packed_bytes(int64_t hidden, int64_t inter)
{
    return ffn_packed_bytes(hidden, inter);
}

int wide_ffn_pack(const void *d_w_gate, const void *d_w_up, const void *d_w_down, int64_t hidden,
                  int64_t inter, void *d_packed, size_t packed_bytes, void *stream)
{
    if (!d_w_gate || !d_w_up || !d_w_down || !d_packed || hidden <= 0 || inter <= 0)
        return WIDE_EINVAL;
    const size_t need = ffn_packed_bytes(hidden, inter);
    if (need == 0 || hidden > (1 << 20) || inter > (1 << 22))
        return WIDE_EUNSUPPORTED;
    if (packed_bytes < need)
        return WIDE_EWORKSPACE;
    if (!aligned16(d_w_gate) || !aligned16(d_w_up) || !aligned16(d_w_down) ||
        (reinterpret_cast<uintptr_t>(d_packed) & 255u) != 0)
        return WIDE_EUNSUPPORTED;
    return ffn_pack_launch(d_w_gate, d_w_up, d_w_down, hidden, inter, d_packed,
                           static_cast<cudaStream_t>(stream));
}

int wide_ffn_masked_packed(const void *d_x, const void *d_packed, const void *d_w_gate,
                           const void *d_w_up, const void *d_w_down, const uint32_t *d_group_mask,
                           void *d_out, const wide_ffn_dims *d, void *d_workspace,
                           size_t workspace_bytes, void *stream)
{
    if (!ffn_dims_ok(d))
        return WIDE_EINVAL;
    if (d->tokens == 0)
        return WIDE_OK;
    if (!d_x || !d_packed || !d_group_mask || !d_out || !d_workspace)
        return WIDE_EINVAL;
    const bool linear = d_w_gate || d_w_up || d_w_down;
    if (linear && (!d_w_gate || !d_w_up || !d_w_down))
        return WIDE_EINVAL;
    if (d->dtype != WIDE_BF16 || d->path == WIDE_PATH_PREFILL ||
        ffn_packed_bytes(d->hidden, d->inter) == 0 || d->hidden > (1 << 20) ||
        d->inter > (1 << 22))
        return WIDE_EUNSUPPORTED;
    const int H = (int)d->hidden, I = (int)d->inter, gs = (int)d->group_size;
    const int T1 = (int)(d->tokens < kTcMaxTok ? d->tokens : kTcMaxTok);
    if (!decode_ffn_tc_packed_supported(T1, H, I, gs))
        return WIDE_EUNSUPPORTED;
    if (!aligned16(d_x) || !aligned16(d_out) || (reinterpret_cast<uintptr_t>(d_packed) & 255u) ||
        (reinterpret_cast<uintptr_t>(d_workspace) & 255u) != 0 ||
        (linear && (!aligned16(d_w_gate) || !aligned16(d_w_up) || !aligned16(d_w_down))))
        return WIDE_EUNSUPPORTED;
    wide_ffn_dims dd = *d;
    dd.path = WIDE_PATH_DECODE;
    const size_t need = wide_ffn_workspace_bytes(&dd);
    if (workspace_bytes < need)
        return WIDE_EWORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (linear)   // every decode kernel is open: the dispatcher picks per launch
        return ffn_decode_launch(d_x, d_w_gate, d_w_up, d_w_down, d_group_mask, d_out, &dd,
                                 d_workspace, s, d_packed);
    DownOutputs o = {};
    o.out_sum = d_out;
    return decode_ffn_persistent(d_x, nullptr, nullptr, nullptr, d_group_mask, o, d->tokens, H, I,
                                 gs, d_workspace, need, s, d_packed);
}

static bool layer_dims_ok(const wide_layer_dims *d, bool ffn)
{
    if (!d || d->n_seq < 1 || d->seq_len < 1 || d->cache_len < 0 || d->hidden <= 0 ||
        d->n_q_heads <= 0 || d->n_kv_heads <= 0 || d->head_dim <= 0 ||
        d->n_q_heads % d->n_kv_heads != 0 || d->cache_cap < d->cache_len + d->seq_len ||
        !(d->eps >= 0.f) || !(d->rope_theta > 0.f))
        return false;
    if (ffn && (d->inter <= 0 || d->ffn_group_size <= 0 || d->inter % d->ffn_group_size != 0 ||
                d->inter / d->ffn_group_size > 1024))
        return false;
    return true;
}

static wide_layer_dims attn_only_dims(const wide_layer_dims *d)
{
    wide_layer_dims a = *d;
    a.inter = 128;
    a.ffn_group_size = 128;
    return a;
}

size_t wide_layer_workspace_bytes(const wide_layer_dims *d)
{
    if (!layer_dims_ok(d, true))
        return 0;
    if (layer_decode_supported(d))
        return layer_decode_workspace(d);
    if (layer_prefill_supported(d))
        return layer_prefill_workspace(d);
    return 0;
}

static int layer_call(const LayerPtrs &p, const wide_layer_dims *d, void *ws, size_t ws_bytes,
                      void *stream)
{
    const bool decode = layer_decode_supported(d);
    if (!decode && !layer_prefill_supported(d))
        return WIDE_EUNSUPPORTED;
    const void *ptrs[] = {p.x, p.gamma1, p.wq, p.wk, p.wv, p.wo, p.k_cache, p.v_cache};
    for (const void *q : ptrs)
        if (!q)
            return WIDE_EINVAL;
    if (!p.head_mask || !ws)
        return WIDE_EINVAL;
    if (p.ffn && (!p.gamma2 || !p.w_gate || !p.w_up || !p.w_down || !p.ffn_mask || !p.out))
        return WIDE_EINVAL;
    if (!p.ffn && !p.attn_out)
        return WIDE_EINVAL;
    const void *al[] = {p.x, p.gamma1, p.wq, p.wk, p.wv, p.wo, p.k_cache, p.v_cache};
    for (const void *q : al)
        if (!aligned16(q))
            return WIDE_EUNSUPPORTED;
    if ((p.out && !aligned16(p.out)) || (p.attn_out && !aligned16(p.attn_out)) ||
        (p.ffn_out && !aligned16(p.ffn_out)) ||
        (p.ffn && (!aligned16(p.gamma2) || !aligned16(p.w_gate) || !aligned16(p.w_up) ||
                   !aligned16(p.w_down))) ||
        (reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
        return WIDE_EUNSUPPORTED;
    if (ws_bytes < (decode ? layer_decode_workspace(d) : layer_prefill_workspace(d)))
        return WIDE_EWORKSPACE;
    if (decode)
        return layer_decode_launch(p, d, ws, static_cast<cudaStream_t>(stream));
    return layer_prefill_launch(p, d, ws, static_cast<cudaStream_t>(stream));
}

int wide_layer_masked(const void *d_x, const wide_layer_weights *w, void *d_k_cache,
                      void *d_v_cache, const uint32_t *d_head_mask, const uint32_t *d_ffn_mask,
                      void *d_out, void *d_attn_out, void *d_ffn_out, const wide_layer_dims *d,
                      void *d_workspace, size_t workspace_bytes, void *stream)
{
    if (!w || !layer_dims_ok(d, true))
        return WIDE_EINVAL;
    LayerPtrs p = {d_x, w->gamma1, w->wq, w->wk, w->wv, w->wo, w->gamma2, w->w_gate, w->w_up,
                   w->w_down, d_k_cache, d_v_cache, d_head_mask, d_ffn_mask, d_out, d_attn_out,
                   d_ffn_out, true, w->ffn_packed};
    if (w->ffn_packed && !aligned16(w->ffn_packed))
        return WIDE_EUNSUPPORTED;
    return layer_call(p, d, d_workspace, workspace_bytes, stream);
}

int wide_attn_masked(const void *d_x, const wide_layer_weights *w, void *d_k_cache,
                     void *d_v_cache, const uint32_t *d_head_mask, void *d_attn_out,
                     const wide_layer_dims *d, void *d_workspace, size_t workspace_bytes,
                     void *stream)
{
    if (!w || !layer_dims_ok(d, false))
        return WIDE_EINVAL;
    const wide_layer_dims a = attn_only_dims(d);
    LayerPtrs p = {d_x, w->gamma1, w->wq, w->wk, w->wv, w->wo, nullptr, nullptr, nullptr,
                   nullptr, d_k_cache, d_v_cache, d_head_mask, nullptr, nullptr, d_attn_out,
                   nullptr, false, nullptr};
    return layer_call(p, &a, d_workspace, workspace_bytes, stream);
}

}  // extern "C"
