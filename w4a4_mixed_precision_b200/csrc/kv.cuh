// kv.cuh -- INT4 KV-cache quantization and dequantization.
//
// Reading: the Atom pages ("Atom: Low-bit Quantization for Efficient and
// Accurate LLM Serving", key facts) place the method under KV-cache
// quantization without a KV recipe; each (token, head) vector of
// head_dim = 128 elements is taken as one group and encoded like an Atom INT4
// activation group ("Atom (mixed-precision block-outlier low-bit quantization
// for serving)", fields Bits and Weight group size), with no reorder and no
// outlier channels:
//   scale = fl32(amax / 7), inv = fl32(7 / amax)  (both 0 for an all-zero group)
//   q = rint(fl32(x * inv)), ties to even; element 2i -> low nibble of byte i
//   dequantized x' = fp16_rn(fl32(q * scale))
//
// Both kernels stream: 8 lanes own one group (16 elements each), a warp four
// groups per step, grid-stride over the groups. The quantizer reads 32
// contiguous bytes per lane (two 16-byte loads; 256 coalesced bytes per
// group) and writes 8 bytes per lane; the dequantizer does the reverse.
#pragma once

#include <cuda_fp16.h>

#include <cstdint>

#include "ptx.cuh"

namespace atomk {

constexpr int kKvThreads = 256;

__global__ void __launch_bounds__(kKvThreads)
kv_quant_kernel(const __half *__restrict__ x, int64_t groups, uint8_t *__restrict__ q4,
                float *__restrict__ scales) {
  const int lane = threadIdx.x & 31, sub = lane & 7;
  const unsigned team_mask = 0xFFu << (8 * (lane >> 3));
  const int64_t stride = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 3);
  for (int64_t g = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 3; g < groups;
       g += stride) {
    const uint4 *src = reinterpret_cast<const uint4 *>(x + g * 128 + sub * 16);
    const uint4 a = __ldg(src), b = __ldg(src + 1);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    float v[16];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[j]));
      v[2 * j] = f.x;
      v[2 * j + 1] = f.y;
    }
    float amax = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(v[j]));
    amax = fmaxf(amax, __shfl_xor_sync(team_mask, amax, 4));
    amax = fmaxf(amax, __shfl_xor_sync(team_mask, amax, 2));
    amax = fmaxf(amax, __shfl_xor_sync(team_mask, amax, 1));
    float scale = 0.f, inv = 0.f;
    if (amax > 0.f) {
      scale = __fdiv_rn(amax, 7.f);
      inv = __fdiv_rn(7.f, amax);
    }
    // the low byte of fp32(1.5 * 2^23 + rint(x * inv)) is the code in two's
    // complement; the product is rounded to fp32 before the add rounds to an
    // integer (__fmul_rn / __fadd_rn are never contracted into an FMA)
    uint32_t c[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) c[j] = __float_as_uint(__fadd_rn(__fmul_rn(v[j], inv), 12582912.f));
    uint32_t out[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t ev = __byte_perm(__byte_perm(c[8 * h], c[8 * h + 2], 0x0040),
                                      __byte_perm(c[8 * h + 4], c[8 * h + 6], 0x0040), 0x5410);
      const uint32_t od = __byte_perm(__byte_perm(c[8 * h + 1], c[8 * h + 3], 0x0040),
                                      __byte_perm(c[8 * h + 5], c[8 * h + 7], 0x0040), 0x5410);
      out[h] = (ev & 0x0F0F0F0Fu) | ((od << 4) & 0xF0F0F0F0u);
    }
    *reinterpret_cast<uint2 *>(q4 + g * 64 + sub * 8) = make_uint2(out[0], out[1]);
    if (sub == 0) scales[g] = scale;
  }
}

__global__ void __launch_bounds__(kKvThreads)
kv_dequant_kernel(const uint8_t *__restrict__ q4, const float *__restrict__ scales,
                  int64_t groups, __half *__restrict__ out) {
  const int lane = threadIdx.x & 31, sub = lane & 7;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 3);
  for (int64_t g = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 3; g < groups;
       g += stride) {
    const uint2 p = __ldg(reinterpret_cast<const uint2 *>(q4 + g * 64 + sub * 8));
    const float s = __ldg(scales + g);
    const uint32_t w[2] = {p.x, p.y};
    uint32_t o[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      // byte j: element 2j in the low nibble, 2j+1 in the high nibble. A
      // nibble n is the code q = (n ^ 8) - 8; fp32(q) is made without a
      // conversion instruction, as the float with bits 0x4B400000 | (n ^ 8)
      // (= 1.5*2^23 + (n ^ 8)) minus 1.5*2^23 + 8, both steps exact. The pair
      // of products goes to fp16 in one packed round-to-nearest conversion.
      const uint32_t byte = w[j >> 2] >> (8 * (j & 3));
      const float q0 = __fsub_rn(__uint_as_float(0x4B400000u | ((byte & 0xFu) ^ 8u)), 12582920.f);
      const float q1 =
          __fsub_rn(__uint_as_float(0x4B400000u | (((byte >> 4) & 0xFu) ^ 8u)), 12582920.f);
      o[j] = pack_half2_rn(__fmul_rn(q0, s), __fmul_rn(q1, s));
    }
    uint4 *dst = reinterpret_cast<uint4 *>(out + g * 128 + sub * 16);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

}  // namespace atomk
