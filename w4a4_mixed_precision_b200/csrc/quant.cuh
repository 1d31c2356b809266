// quant.cuh -- fused outlier reorder + per-token per-128-group INT4/INT8
// quantization (one streaming pass over the fp16 rows).
//
// Method: "Atom: Low-bit Quantization for Efficient and Accurate LLM Serving"
// (paper summary: activations get a dedicated outlier path) and the record
// "Atom (mixed-precision block-outlier low-bit quantization for serving)"
// (fields "Weight group size" = 128 and "notes": every contiguous run of 128
// elements is one group quantized independently; 128 high-precision channels).
//
// Design (memory-bound, so the goal is to keep HBM busy):
//  * each CTA is persistent over rows r = blockIdx.x + i*gridDim.x; a whole
//    fp16 row is brought into shared memory by one bulk copy (TMA engine,
//    mbarrier completion), S rows in flight per CTA;
//  * the permutation is built once per CTA in shared memory (uint16 [K]) while
//    the first rows are in flight: a bitmap of the outlier channels, a block
//    scan of the non-outlier counts, then the outlier list at the tail;
//  * 8 lanes quantize one group (16 reordered elements per lane), 4 groups per
//    warp per pass: gather from the staged row through the permutation,
//    shuffle-reduce amax over the 8 lanes, one IEEE division each for scale and
//    inv, codes by round-half-even via the 1.5*2^23 add (exact for |t| < 2^22),
//    nibble packing in registers, 8-byte (INT4) or 16-byte (INT8) stores;
//  * the gather order inside a lane is rotated per lane so that the 32 lanes of
//    a warp read 32 distinct shared-memory banks.
#pragma once

#include "ptx.cuh"

namespace atomk {

constexpr int kQuantThreads = 256;
constexpr int kQuantMaxStages = 4;

struct QuantLayout {
  // Byte offsets inside dynamic shared memory.
  uint32_t bitmap, perm, stages, total;
  uint32_t row_bytes;
  int stages_n;
};

__host__ __device__ inline QuantLayout quant_layout(int K, int stages_n) {
  QuantLayout L;
  L.row_bytes = 2u * static_cast<uint32_t>(K);
  L.bitmap = 256;                                                  // after barriers and flags
  L.perm = L.bitmap + ((static_cast<uint32_t>(K) / 8u + 15u) & ~15u);
  L.stages = (L.perm + L.row_bytes + 127u) & ~127u;
  L.stages_n = stages_n;
  L.total = L.stages + static_cast<uint32_t>(stages_n) * L.row_bytes;
  return L;
}

__global__ void __launch_bounds__(kQuantThreads)
reorder_quant_kernel(const __half *__restrict__ x, int64_t rows, int K, int64_t ld,
                     const int32_t *__restrict__ outlier_idx, uint8_t *__restrict__ q4,
                     int8_t *__restrict__ q8, float *__restrict__ scales, int stages_n) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const QuantLayout L = quant_layout(K, stages_n);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem);             // [kQuantMaxStages]
  volatile int *flags = reinterpret_cast<volatile int *>(smem + 64);  // [0] bad list
  int *warp_sums = reinterpret_cast<int *>(smem + 128);            // [8]
  uint32_t *bitmap = reinterpret_cast<uint32_t *>(smem + L.bitmap);
  uint16_t *perm = reinterpret_cast<uint16_t *>(smem + L.perm);
  uint8_t *stage_base = smem + L.stages;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = K / 128, Gd = G - 1, Kd = K - 128;
  const int64_t q4_row = Kd / 2;
  const int64_t grid = gridDim.x;

  if (tid == 0) {
    for (int s = 0; s < stages_n; ++s) mbar_init(&full[s], 1);
    flags[0] = 0;
    fence_mbar_init();
  }
  for (int w = tid; w < K / 32; w += kQuantThreads) bitmap[w] = 0u;
  __syncthreads();

  // Put the first rows in flight before building the permutation.
  if (tid == 0) {
    for (int s = 0; s < stages_n; ++s) {
      const int64_t r = blockIdx.x + s * grid;
      if (r < rows) {
        mbar_arrive_expect_tx(&full[s], L.row_bytes);
        bulk_load(stage_base + s * L.row_bytes, x + r * ld, L.row_bytes, &full[s]);
      }
    }
  }

  // ---- permutation: ascending non-outlier channels, then the outlier list.
  if (tid < 128) {
    const int c = outlier_idx[tid];
    if (c < 0 || c >= K) {
      flags[0] = 1;
    } else {
      const uint32_t bit = 1u << (c & 31);
      if (atomicOr(&bitmap[c >> 5], bit) & bit) flags[0] = 1;  // repeated channel
    }
  }
  __syncthreads();
  const int nwords = K / 32;
  const int per = (nwords + kQuantThreads - 1) / kQuantThreads;
  const int w0 = min(nwords, tid * per), w1 = min(nwords, w0 + per);
  int count = 0;
  for (int w = w0; w < w1; ++w) count += __popc(~bitmap[w]);
  int incl = count;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  int base = 0;
  for (int w = 0; w < warp; ++w) base += warp_sums[w];
  int pos = base + incl - count;
  for (int w = w0; w < w1; ++w) {
    uint32_t bits = ~bitmap[w];
    while (bits) {
      const int b = __ffs(bits) - 1;
      bits &= bits - 1;
      if (pos < Kd) perm[pos] = static_cast<uint16_t>(w * 32 + b);
      ++pos;
    }
  }
  if (tid < 128) {
    const int c = outlier_idx[tid];
    if (c >= 0 && c < K) perm[Kd + tid] = static_cast<uint16_t>(c);
  }
  __syncthreads();

  if (flags[0]) {
    // Invalid outlier list: write nothing, but let the issued copies land first.
    if (tid == 0) {
      report_status(1 /* ATOM_ERR_INVALID_ARG */);
      for (int s = 0; s < stages_n; ++s)
        if (blockIdx.x + s * grid < rows) (void)mbar_wait(&full[s], 0, nullptr);
    }
    return;
  }

  // ---- per-lane work assignment (fixed for the whole kernel)
  const int sub = lane & 7;        // lane within its 8-lane group team
  const int team = lane >> 3;      // which of the warp's 4 groups
  const int rot_dense = 2 * ((sub >> 2) & 1) + 4 * team;  // even, 0..14
  const unsigned team_mask = 0xFFu << (8 * team);

  int64_t aborted_at = -1;
  for (int64_t i = 0;; ++i) {
    const int64_t r = blockIdx.x + i * grid;
    if (r >= rows) break;
    const int s = static_cast<int>(i % stages_n);
    const uint32_t parity = static_cast<uint32_t>((i / stages_n) & 1);
    const bool ok = mbar_wait(&full[s], parity, nullptr);
    if (__syncthreads_or(!ok)) {
      if (tid == 0) report_status(6 /* ATOM_ERR_TIMEOUT */);
      aborted_at = i;
      break;
    }
    const __half *row = reinterpret_cast<const __half *>(stage_base + s * L.row_bytes);

    for (int gb = 0; gb < G; gb += 32) {
      const int g = gb + warp * 4 + team;
      if (g > Gd) continue;  // whole 8-lane teams skip together
      const bool dense = g < Gd;
      const int rot = dense ? rot_dense : 0;
      const int j0 = g * 128 + sub * 16;
      float v[16];
      float amax = 0.f;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int c = perm[j0 + ((e + rot) & 15)];
        v[e] = __half2float(row[c]);
        amax = fmaxf(amax, fabsf(v[e]));
      }
      amax = fmaxf(amax, __shfl_xor_sync(team_mask, amax, 4));
      amax = fmaxf(amax, __shfl_xor_sync(team_mask, amax, 2));
      amax = fmaxf(amax, __shfl_xor_sync(team_mask, amax, 1));
      const float qmax = dense ? 7.f : 127.f;
      float scale = 0.f, inv = 0.f;
      if (amax > 0.f) {
        scale = __fdiv_rn(amax, qmax);
        inv = __fdiv_rn(qmax, amax);
      }
      // code bits: low bits of fp32(1.5*2^23 + rint(x*inv)) are the two's complement code
      uint32_t bits[16];
#pragma unroll
      for (int e = 0; e < 16; ++e)
        bits[e] = __float_as_uint(__fadd_rn(__fmul_rn(v[e], inv), 12582912.f));
      if (dense) {
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          lo |= (bits[e] & 0xFu) << (4 * e);
          hi |= (bits[e + 8] & 0xFu) << (4 * e);
        }
        // slot e holds element (e + rot) mod 16: rotate the 64-bit word left by 4*rot
        uint64_t p = (static_cast<uint64_t>(hi) << 32) | lo;
        const int sh = 4 * rot;
        if (sh) p = (p << sh) | (p >> (64 - sh));
        *reinterpret_cast<uint2 *>(q4 + r * q4_row + g * 64 + sub * 8) =
            make_uint2(static_cast<uint32_t>(p), static_cast<uint32_t>(p >> 32));
      } else {
        uint4 o;
        o.x = (bits[0] & 0xFFu) | ((bits[1] & 0xFFu) << 8) | ((bits[2] & 0xFFu) << 16) |
              ((bits[3] & 0xFFu) << 24);
        o.y = (bits[4] & 0xFFu) | ((bits[5] & 0xFFu) << 8) | ((bits[6] & 0xFFu) << 16) |
              ((bits[7] & 0xFFu) << 24);
        o.z = (bits[8] & 0xFFu) | ((bits[9] & 0xFFu) << 8) | ((bits[10] & 0xFFu) << 16) |
              ((bits[11] & 0xFFu) << 24);
        o.w = (bits[12] & 0xFFu) | ((bits[13] & 0xFFu) << 8) | ((bits[14] & 0xFFu) << 16) |
              ((bits[15] & 0xFFu) << 24);
        *reinterpret_cast<uint4 *>(q8 + r * 128 + sub * 16) = o;
      }
      if (sub == 0) scales[static_cast<int64_t>(g) * rows + r] = scale;
    }

    __syncthreads();  // every warp is done with this stage
    if (tid == 0) {
      const int64_t nr = r + stages_n * grid;
      if (nr < rows) {
        mbar_arrive_expect_tx(&full[s], L.row_bytes);
        bulk_load(stage_base + s * L.row_bytes, x + nr * ld, L.row_bytes, &full[s]);
      }
    }
  }

  // After a timeout, give the copies still in flight a bounded chance to land
  // before the CTA's shared memory is released.
  if (aborted_at >= 0 && tid == 0) {
    for (int k = 0; k < stages_n; ++k) {
      const int64_t it = aborted_at + k;
      if (blockIdx.x + it * grid < rows)
        (void)mbar_wait(&full[it % stages_n], static_cast<uint32_t>((it / stages_n) & 1), nullptr);
    }
  }
}

}  // namespace atomk
