// ffn_pack.cu -- the decode FFN's packed weight layout.
//
// The tensor cores read a K-major bf16 operand from shared memory in atoms
// of 8 rows x 128 bytes (64 K elements).  Copied by TMA from the nn.Linear
// layout, such a tile is 128-byte pieces of rows kilobytes apart, which B200
// HBM serves at about half its bandwidth; the packed copy stores every tile
// the decode kernel loads as one contiguous run:
//   W_gate, W_up  interleaved, [I / 64][H / 64][4][2][16][64]: 64-channel
//                 panels, K-step-major; inside a panel's K step, 16-channel
//                 groups of 16 W_gate rows followed by the same 16 W_up rows.
//                 The R channels of one K step of a panel are then 2R * 128
//                 contiguous bytes, and one M = 128 tensor-core tile holds the
//                 gate and up rows of 64 channels;
//   W_down        [I / 16][H][16]: 16-channel column panels, so the 128-row
//                 blocks of a chunk are contiguous 4 KB pieces.
// Packing is a pure permutation of the weights (the values are copied
// bitwise), done once when the weights are loaded.
#include "common.cuh"
#include "host.h"

namespace wide {
namespace {

// One thread per 16-byte piece (8 bf16) of W_gate (which = 0) or W_up
// (which = 1): piece (r, c8) of source row r goes to panel r / 64, K step
// c8 / 8, group (r % 64) / 16, half `which`, row r % 16.
__global__ void __launch_bounds__(256)
    pack_rows(const uint4 *__restrict__ src, uint4 *__restrict__ dst, int64_t H, int64_t I,
              int which)
{
    const int64_t per_row = H / 8;
    const int64_t n = I * per_row;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / per_row, c8 = i % per_row;
        const int64_t panel = r >> 6, grp = (r >> 4) & 3, row = r & 15, ks = c8 >> 3,
                      e8 = c8 & 7;
        dst[((((panel * (H / 64) + ks) * 4 + grp) * 2 + which) * 16 + row) * 8 + e8] = src[i];
    }
}

// One thread per 16-byte piece of W_down [H][I]: piece (n, c8) holds
// channels 8 * c8 .. + 7 of output row n and goes to chunk c8 / 2, row n,
// half c8 % 2.
__global__ void __launch_bounds__(256)
    pack_down(const uint4 *__restrict__ src, uint4 *__restrict__ dst, int64_t H, int64_t I)
{
    const int64_t per_row = I / 8;
    const int64_t n = H * per_row;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = i / per_row, c8 = i % per_row;
        dst[((c8 >> 1) * H + row) * 2 + (c8 & 1)] = src[i];
    }
}

}  // namespace

size_t ffn_packed_bytes(int64_t H, int64_t I)
{
    if (H <= 0 || I <= 0 || H % 128 != 0 || I % 64 != 0)
        return 0;
    return 3 * (size_t)H * (size_t)I * 2;
}

int ffn_pack_launch(const void *wg, const void *wu, const void *wd, int64_t H, int64_t I,
                    void *packed, cudaStream_t s)
{
    const size_t mat = (size_t)H * (size_t)I * 2;
    uint4 *out = static_cast<uint4 *>(packed);
    const int64_t pieces = H * I / 8;
    const int blocks = (int)((pieces + 255) / 256 < 4096 ? (pieces + 255) / 256 : 4096);
    {
        LaunchScope scope(KID_FFN_PACK, s);
        pack_rows<<<blocks, 256, 0, s>>>(static_cast<const uint4 *>(wg), out, H, I, 0);
    }
    {
        LaunchScope scope(KID_FFN_PACK, s);
        pack_rows<<<blocks, 256, 0, s>>>(static_cast<const uint4 *>(wu), out, H, I, 1);
    }
    {
        LaunchScope scope(KID_FFN_PACK, s);
        pack_down<<<blocks, 256, 0, s>>>(static_cast<const uint4 *>(wd), out + 2 * (mat / 16), H, I);
    }
    return cudaGetLastError() == cudaSuccess ? WIDE_OK : WIDE_CUDA_FAIL();
}

}  // namespace wide
