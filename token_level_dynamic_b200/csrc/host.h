// host.h -- host-side helpers shared by the libwide entry points.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "wide.h"

namespace wide {

// Device address of this device's status word (looked up once per device).
int32_t *status_ptr();

// Encodes a 2-D row-major tensor map: `rows` x `cols` elements of
// `elem_bytes` bytes, row pitch `pitch_elems`, box `box_rows` x `box_cols`,
// 128-byte swizzle when `swizzle128` (box_cols * elem_bytes must be 128 then).
// Returns false if the driver rejects it.
bool make_tmap_2d(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                  uint64_t pitch_elems, uint32_t elem_bytes, uint32_t box_rows, uint32_t box_cols,
                  bool swizzle128);

// Raises a kernel's dynamic shared memory limit to at least `bytes` (once
// per kernel, device and size).
bool raise_smem_limit(const void *kernel, size_t bytes);

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Maps the last CUDA error to a WIDE code (and clears it).
inline int launch_status()
{
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? WIDE_OK : WIDE_ECUDA;
}

// Kernel ids reported by the profiler (wide_kernel_name).
enum KernelId : int32_t {
    KID_REORDER_PARTITION_RANK = 1,
    KID_REORDER_FINISH = 2,
    KID_DECODE_GATEUP = 3,
    KID_DECODE_DOWN = 4,
    KID_PREFILL_ZERO = 5,
    KID_PREFILL_GATEUP = 6,
    KID_PREFILL_DOWN = 7,
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

// FFN argument checks shared by the FFN entry points (api.cu).
bool ffn_dims_ok(const wide_ffn_dims *d);
int ffn_path(const wide_ffn_dims *d);
bool ffn_shape_supported(const wide_ffn_dims *d, int path);

// Internal entry points of the kernel files.
int reorder_launch(const uint32_t *mask, int64_t T, int64_t G, int32_t tile_m,
                   const wide_worklist *wl, cudaStream_t s);
int reorder_splits(int64_t T);

size_t ffn_prefill_workspace(const wide_ffn_dims *d);
int ffn_prefill_launch(const void *x, const void *wg, const void *wu, const void *wd,
                       const uint32_t *mask, void *out, const wide_ffn_dims *d, void *ws,
                       cudaStream_t s);

size_t ffn_decode_workspace(const wide_ffn_dims *d);
int ffn_decode_launch(const void *x, const void *wg, const void *wu, const void *wd,
                      const uint32_t *mask, void *out, const wide_ffn_dims *d, void *ws,
                      cudaStream_t s);

}  // namespace wide
