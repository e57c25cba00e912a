// scale_layout.cu -- the sweep's row-major E4M3 scale bytes rewritten into the
// tiled layout that Blackwell's block-scaled tensor-core MMA (and cuBLASLt's
// NVFP4 GEMM with 16-element E4M3 scale vectors) reads, so that the packed
// output can be consumed by such a GEMM as it is.
//
// The tiled layout, for a scale matrix SF[rows, cols] (cols = in / 16):
//   - rows are padded to a multiple of 128 and columns to a multiple of 4,
//     the padding bytes being 0;
//   - the matrix is cut into 128 x 4 blocks of 512 bytes, stored block-row by
//     block-row: block (rb, cb) starts at byte 512 * (rb * cols_padded / 4 + cb);
//   - inside a block, scale (r, c) (r < 128, c < 4) is byte
//     (r % 32) * 16 + (r / 32) * 4 + c.
// One thread writes one 16-byte line of a block: rows r32, r32+32, r32+64,
// r32+96 of the block, four columns each.
#include "nvfp4_kernels.cuh"

namespace nvfp4 {

namespace {

__global__ void __launch_bounds__(256)
scales_to_blocked_kernel(const uint8_t* __restrict__ sf, int64_t rows, int64_t cols, int64_t ld,
                         int64_t col_blocks, int64_t lines, uint4* __restrict__ out) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < lines;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t blk = i >> 5;                 // 32 lines per block
    const int r32 = static_cast<int>(i & 31);
    const int64_t rb = blk / col_blocks;
    const int64_t cb = blk - rb * col_blocks;
    uint32_t word[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {               // q = (r / 32) within the block
      const int64_t r = rb * 128 + q * 32 + r32;
      uint32_t w = 0;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int64_t cc = cb * 4 + c;
        const uint32_t v = (r < rows && cc < cols) ? sf[r * ld + cc] : 0u;
        w |= v << (8 * c);
      }
      word[q] = w;
    }
    out[i] = make_uint4(word[0], word[1], word[2], word[3]);
  }
}

}  // namespace

size_t blocked_scales_bytes(int64_t rows, int64_t cols) {
  const int64_t rp = (rows + 127) / 128 * 128;
  const int64_t cp = (cols + 3) / 4 * 4;
  return static_cast<size_t>(rp * cp);
}

cudaError_t launch_scales_to_blocked(const uint8_t* sf, int64_t rows, int64_t cols, int64_t ld,
                                     uint8_t* out, int num_sms, cudaStream_t stream) {
  const int64_t col_blocks = (cols + 3) / 4;
  const int64_t lines = (rows + 127) / 128 * col_blocks * 32;
  if (lines == 0) return cudaSuccess;
  int64_t blocks = (lines + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  scales_to_blocked_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      sf, rows, cols, ld, col_blocks, lines, reinterpret_cast<uint4*>(out));
  return cudaGetLastError();
}

}  // namespace nvfp4
