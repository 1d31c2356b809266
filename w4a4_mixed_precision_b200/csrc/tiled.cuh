// tiled.cuh -- the tiled layout of packed INT4 weights, and the copies between
// it and the row layout that atom_quant_weights writes.
//
// Row layout (the activations' and the weights' codes as quantized):
//   qw4[n][i], n < N, i < Kd/2 = (K-128)/2; group g of row n is bytes
//   [64g, 64g+64) of the row.
// Tiled layout (the library's weight layout for the GEMMs, a one-off repack):
//   tile t = n / 128, row r = n % 128, group g < G4 = K/128 - 1:
//   qw4t[((t * G4 + g) * 128 + r) * 64 + j] = qw4[n][64g + j]   (j < 64),
//   zero for rows n >= N of the last tile.
// Each (tile, group) block is 8 KB of contiguous memory holding exactly the
// 128-row x 64-byte box the GEMMs stage per group, so a GEMM fetches it with
// one bulk copy, and the blocks of one tile's consecutive groups follow each
// other. In the row layout the same box is 128 separate 64-byte pieces, one
// per weight row, (K-128)/2 bytes apart: a pattern that DRAM serves far below
// its streaming rate, which is what paces a decode GEMM (it reads every weight
// once per call).
#pragma once

#include "ptx.cuh"

namespace atomk {

constexpr int kTileRows = 128;
constexpr uint32_t kTileBlock = kTileRows * 64;   // bytes of one (tile, group) block

// One thread per 16-byte chunk of the tiled layout (4 per 64-byte row piece).
__global__ void __launch_bounds__(256)
pack_weights_tiled_kernel(const uint8_t *__restrict__ qw4, uint8_t *__restrict__ qw4t, int64_t N,
                          int64_t row_bytes, int64_t g4, int64_t chunks) {
  for (int64_t c = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; c < chunks;
       c += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t piece = c >> 2;                  // (tile, group, row) in tiled order
    const int64_t r = piece % kTileRows, tg = piece / kTileRows;
    const int64_t g = tg % g4, t = tg / g4;
    const int64_t n = t * kTileRows + r;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (n < N) v = __ldg(reinterpret_cast<const uint4 *>(qw4 + n * row_bytes + g * 64) + (c & 3));
    reinterpret_cast<uint4 *>(qw4t)[c] = v;
  }
}

// The inverse copy (rows n < N only): tiled layout back to the row layout.
__global__ void __launch_bounds__(256)
unpack_weights_tiled_kernel(const uint8_t *__restrict__ qw4t, uint8_t *__restrict__ qw4, int64_t N,
                            int64_t row_bytes, int64_t g4, int64_t chunks) {
  for (int64_t c = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; c < chunks;
       c += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t piece = c >> 2;
    const int64_t r = piece % kTileRows, tg = piece / kTileRows;
    const int64_t g = tg % g4, t = tg / g4;
    const int64_t n = t * kTileRows + r;
    if (n < N)
      reinterpret_cast<uint4 *>(qw4 + n * row_bytes + g * 64)[c & 3] =
          __ldg(reinterpret_cast<const uint4 *>(qw4t) + c);
  }
}

}  // namespace atomk
