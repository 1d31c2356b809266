// gemm.cuh -- W4A4 mixed-precision group-scaled GEMM on tcgen05 integer tensor cores.
//
//   Y[m][n] = fp16( sum_g sa[g][m] * sw[g][n] * P[g][m][n] ),
//   P[g][m][n] = sum_{k in group g} qa[m][k] * qw[n][k]   (exact int32)
//
// Method: "Atom: Low-bit Quantization for Efficient and Accurate LLM Serving"
// (abstract: low-bit integer operators for 4-bit weight-activation products;
// paper summary: per-group scales, a separate higher-precision outlier path) and
// the record "Atom (mixed-precision block-outlier low-bit quantization for
// serving)" (group 128, 128 high-precision channels; "Kernels": purpose-built
// low-bit kernels). The pages' kernels target Ampere INT4 mma; sm_100a has no
// 4-bit integer MMA, so both the INT4 groups and the INT8 outlier group run on
// tcgen05.mma kind::i8.
//
// Structure. A cluster of two CTAs on two SMs owns a 256x256 output tile and
// issues 2-SM MMAs (cta_group::2, M=256, N=256, K=32): CTA r holds A rows
// [128r, 128r+128) and W rows [128r, 128r+128) of the tile in its shared
// memory, and its TMEM receives output rows [128r, 128r+128) x 256 columns.
// The pairs are persistent over tiles (m fastest). One pipeline step per
// 128-wide K group, with these warp roles in each CTA:
//
//   loader warps 1..7  LDG the packed INT4 group (64 bytes per row) one group
//                      ahead into registers, expand each nibble to a byte
//                      holding 16*q (x << 4 & 0xF0 / x & 0xF0), store K-major
//                      with the 128-byte swizzle, plus the group's scales. For
//                      the INT8 outlier group one thread issues two TMA tile
//                      loads instead. Every loader warp arrives on the pair
//                      leader's "operands full" barrier.
//   MMA warp 0         (leader CTA only) 4 x 2-SM MMA into one of two TMEM
//                      accumulators (2 x 256 int32 columns per CTA), then
//                      commits to both CTAs' "stage empty" and "accumulator
//                      full" barriers.
//   drain warps 8..15  read the partials with the 16x256b TMEM shape (a thread
//                      holds 4 rows x 2 columns of every 8-column block),
//                      refill the accumulator with the conversion bias, and
//                      accumulate sa*sw*P into fp32 registers. After the last
//                      group of a tile: fp16 stores.
//
// Exact integer -> float: every accumulator starts at the bit pattern of
// 1.5*2^23 (0x4B400000) and the MMAs add P on top, so the drain reads
// F = 1.5*2^23 + P as a float with no integer instruction (|P| < 2^22).
// Dequantisation: with sw' = sw truncated to 22 significant bits, C*sw' is
// exact for C = 1.5*2^23, so t = fma(F, sw', -C*sw') = round(P*sw') in one
// instruction, then acc = fma(t, sa, acc); both run as packed f32x2 pairs.
// (The truncation changes sw by less than 2^-21 relative.)
//
// Nibbles are expanded as 16*q so no sign extension is needed: INT4 partials
// come out as exactly 256*P, and 1/256 is folded into sa. Both operands use
// the same expansion order inside a group (low nibbles of a 16-byte chunk,
// then its high nibbles), which permutes the K positions of a group
// identically for A and W and leaves every per-group dot product unchanged.
#pragma once

#include "ptx.cuh"

namespace atomk {

namespace gemm_cfg {
constexpr int BM = 128;          // A rows per CTA (256 per pair)
constexpr int BN = 256;          // output columns per pair tile
constexpr int BW = 128;          // W rows per CTA
constexpr int kPairM = 2 * BM;
constexpr int kStages = 6;
constexpr int kThreads = 512;
constexpr int kLoaderThreads = 224;  // warps 1..7
constexpr uint32_t kABytes = BM * 128;
constexpr uint32_t kBBytes = BW * 128;
constexpr uint32_t kSaOff = kABytes + kBBytes;
constexpr uint32_t kSwOff = kSaOff + BM * 4;
constexpr uint32_t kStageBytes = 34u * 1024u;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kBarBytes = 1024;
constexpr uint32_t kSmemBytes = kBarBytes + kStages * kStageBytes + 1024;  // + alignment slack
constexpr int kPackedChunks = (BM + BW) * 4;                                   // 16-B chunks / group
constexpr int kChunksPerThread = (kPackedChunks + kLoaderThreads - 1) / kLoaderThreads;
constexpr uint32_t kIdesc = idesc_i8(kPairM, BN);
constexpr uint32_t kBias = 0x4B400000u;  // bits of 1.5 * 2^23
constexpr float kBiasF = 12582912.0f;
constexpr int kLoaderRegs = 80;
constexpr int kDrainRegs = 176;
static_assert(kSwOff + BN * 4 <= kStageBytes, "stage overflow");
static_assert(kStageBytes % 1024 == 0, "stages must keep 1024-byte alignment");
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
static_assert(2 * 128 * (kLoaderRegs + kDrainRegs) == 65536, "register split must fill the file");
}  // namespace gemm_cfg

struct GemmParams {
  const uint8_t *qa4;
  const float *sa;
  const uint8_t *qw4;
  const float *sw;
  __half *y;           // may be null in partials mode
  int32_t *partials;   // partials mode only
  int M, N, K, G;
  int m_tiles, n_tiles, tiles;   // pair tiles of 256 x 256
};

__device__ __forceinline__ uint4 ldg_stream_v4(const void *p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p));
  return v;
}

// Predicated global stores. Keeping the predicate inside the instruction
// (rather than branching around the store) keeps the epilogue one basic block,
// which is what lets the 128 live accumulators stay in registers.
__device__ __forceinline__ void st_global_b32_if(void *p, uint32_t a, bool pred) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %2, 0;\n\t@q st.global.b32 [%0], %1;\n\t}" ::"l"(p),
      "r"(a), "r"(static_cast<uint32_t>(pred))
      : "memory");
}

__device__ __forceinline__ void st_global_v2_if(void *p, uint32_t a, uint32_t b, bool pred) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %3, 0;\n\t@q st.global.v2.b32 [%0], {%1, %2};\n\t}" ::"l"(
          p),
      "r"(a), "r"(b), "r"(static_cast<uint32_t>(pred))
      : "memory");
}

// Walks one CTA pair's (tile, group) sequence; both CTAs of a pair walk the same one.
struct TileWalk {
  int tile, g, m0, n0;
  __device__ __forceinline__ void start(const GemmParams &p) {
    tile = blockIdx.x >> 1;
    g = 0;
    set(p);
  }
  __device__ __forceinline__ void set(const GemmParams &p) {
    m0 = (tile % p.m_tiles) * gemm_cfg::kPairM;
    n0 = (tile / p.m_tiles) * gemm_cfg::BN;
  }
  __device__ __forceinline__ void next(const GemmParams &p) {
    if (++g == p.G) {
      g = 0;
      tile += gridDim.x >> 1;
      set(p);
    }
  }
};

__device__ __forceinline__ int64_t pair_iterations(const GemmParams &p) {
  const int pair = static_cast<int>(blockIdx.x >> 1), pairs = static_cast<int>(gridDim.x >> 1);
  const int mine = p.tiles > pair ? (p.tiles - pair + pairs - 1) / pairs : 0;
  return static_cast<int64_t>(mine) * p.G;
}

// ------------------------------------------------------------------ loader role

struct LoaderRegs {
  uint4 chunk[gemm_cfg::kChunksPerThread];
  float sc[3];
};

// Packed chunk i (16 bytes) of this thread for group w.g, or zeros past the matrix edge.
__device__ __forceinline__ uint4 loader_chunk(const GemmParams &p, const TileWalk &w, int rank,
                                              int lt, int i) {
  using namespace gemm_cfg;
  const int c = lt + kLoaderThreads * i;
  if (c >= kPackedChunks || w.g >= p.G - 1) return make_uint4(0u, 0u, 0u, 0u);
  // byte offsets fit in 32 bits: the host limits each packed matrix to < 2 GiB
  const uint32_t row_bytes = static_cast<uint32_t>(p.K - 128) / 2;
  const bool is_a = c < BM * 4;
  const int grow = is_a ? w.m0 + BM * rank + (c >> 2) : w.n0 + BW * rank + ((c - BM * 4) >> 2);
  if (grow >= (is_a ? p.M : p.N)) return make_uint4(0u, 0u, 0u, 0u);
  const uint32_t off =
      static_cast<uint32_t>(grow) * row_bytes + static_cast<uint32_t>(w.g) * 64u + (c & 3) * 16u;
  return ldg_stream_v4((is_a ? p.qa4 : p.qw4) + off);
}

// Scale k of this thread for group w.g: sa of row lt (lt < 128) or sw of column lt-128+96k.
__device__ __forceinline__ float loader_scale(const GemmParams &p, const TileWalk &w, int rank,
                                              int lt, int k) {
  using namespace gemm_cfg;
  if (lt < BM) {
    const int m = w.m0 + BM * rank + lt;
    return (k == 0 && m < p.M) ? __ldg(p.sa + static_cast<int64_t>(w.g) * p.M + m) : 0.f;
  }
  const int j = lt - BM + 96 * k;
  const int n = w.n0 + j;
  return (j < BN && n < p.N) ? __ldg(p.sw + static_cast<int64_t>(w.g) * p.N + n) : 0.f;
}

__device__ __forceinline__ void loader_fetch(const GemmParams &p, const TileWalk &w, int rank,
                                             int lt, LoaderRegs &r) {
#pragma unroll
  for (int i = 0; i < gemm_cfg::kChunksPerThread; ++i) r.chunk[i] = loader_chunk(p, w, rank, lt, i);
#pragma unroll
  for (int k = 0; k < 3; ++k) r.sc[k] = loader_scale(p, w, rank, lt, k);
}

// Scale layouts in a stage, ordered for the drain's 16x256b fragments:
//  sa: row r = 32q + i + 8k (i < 8, k < 4) at q*32 + i*4 + k, so a thread's four
//      rows are one 16-byte load;
//  sw: column n = 16S + 8u + 2t + e (t < 4, e, u < 2) at (4S + t)*4 + 2u + e, so a
//      thread's four columns of a 16-column block are one 16-byte load. The
//      stored value is sw truncated to 22 significant bits.
__device__ __forceinline__ int sa_slot(int r) { return (r >> 5) * 32 + (r & 7) * 4 + ((r >> 3) & 3); }
__device__ __forceinline__ int sw_slot(int n) {
  const int w = n & 15;
  return ((n >> 4) * 4 + ((w & 7) >> 1)) * 4 + ((w >> 3) << 1) + (w & 1);
}

// Expands and stores this thread's chunks and scales of group w.g into the stage,
// reloading each register for group wn.g right after it has been stored (so
// one group of loads stays in flight with a single set of registers).
__device__ __forceinline__ void loader_store_refetch(const GemmParams &p, const TileWalk &w,
                                                     const TileWalk &wn, bool refetch, int rank,
                                                     int lt, LoaderRegs &r, uint8_t *stage) {
  using namespace gemm_cfg;
  const bool int4_group = w.g < p.G - 1;
#pragma unroll
  for (int i = 0; i < kChunksPerThread; ++i) {
    const int c = lt + kLoaderThreads * i;
    if (int4_group && c < kPackedChunks) {
      const bool is_a = c < BM * 4;
      const int cc = c & 3;
      const int row = (is_a ? c : c - BM * 4) >> 2;
      uint8_t *dst = stage + (is_a ? 0u : kABytes) + row * 128;
      const uint4 v = r.chunk[i];
      const uint4 lo = make_uint4((v.x << 4) & 0xF0F0F0F0u, (v.y << 4) & 0xF0F0F0F0u,
                                  (v.z << 4) & 0xF0F0F0F0u, (v.w << 4) & 0xF0F0F0F0u);
      const uint4 hi = make_uint4(v.x & 0xF0F0F0F0u, v.y & 0xF0F0F0F0u, v.z & 0xF0F0F0F0u,
                                  v.w & 0xF0F0F0F0u);
      const int sw = row & 7;
      *reinterpret_cast<uint4 *>(dst + (((2 * cc) ^ sw) << 4)) = lo;
      *reinterpret_cast<uint4 *>(dst + (((2 * cc + 1) ^ sw) << 4)) = hi;
    }
    if (refetch) r.chunk[i] = loader_chunk(p, wn, rank, lt, i);
  }
  float *sa_s = reinterpret_cast<float *>(stage + kSaOff);
  float *sw_s = reinterpret_cast<float *>(stage + kSwOff);
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    if (lt < BM) {
      if (k == 0) sa_s[sa_slot(lt)] = r.sc[0];
    } else {
      const int j = lt - BM + 96 * k;
      if (j < BN) sw_s[sw_slot(j)] = __uint_as_float(__float_as_uint(r.sc[k]) & 0xFFFFFFFCu);
    }
    if (refetch) r.sc[k] = loader_scale(p, wn, rank, lt, k);
  }
}

// ------------------------------------------------------------------ kernel

template <bool kPartials>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(gemm_cfg::kThreads, 1)
w4a4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a8,
                 const __grid_constant__ CUtensorMap tmap_w8, const GemmParams p) {
  using namespace gemm_cfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);

  uint64_t *lfull = reinterpret_cast<uint64_t *>(smem);  // [kStages] local loaders -> drain
  uint64_t *mfull = lfull + kStages;   // [kStages] leader's: both CTAs' loaders -> MMA
  uint64_t *empty = mfull + kStages;   // [kStages] MMA commit + local drain -> loaders
  uint64_t *tfull = empty + kStages;   // [2]       MMA commit -> drain
  uint64_t *tempty = tfull + 2;        // [2]       leader's: both CTAs' drains -> MMA
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  uint8_t *stages = smem + kBarBytes;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = static_cast<int>(cluster_cta_rank());

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&lfull[s], 7);       // local loader warps
      mbar_init(&mfull[s], 14);      // loader warps of both CTAs
      mbar_init(&empty[s], 1 + 8);   // MMA commit + local drain warps
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 16);     // drain warps of both CTAs
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before_sync();
  cluster_sync();
  tc_fence_after_sync();
  const uint32_t tbase = *tmem_slot;
  const int64_t iters = pair_iterations(p);

  auto fail = [&](void) {
    report_status(6 /* ATOM_ERR_TIMEOUT */);
    *abort_flag = 1;
  };

  if (warp >= 8) {
    // ================================================================ drain
    regs_increase<kDrainRegs>();
    const int q = warp & 3;           // TMEM lane quarter this warp may access
    const int h = (warp - 8) >> 2;    // which 128-column half of the tile
    const int t0 = lane & 3;          // column pair within an 8-column block
    const int i0 = lane >> 2;         // row within a group of 8 lanes
    const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
    const uint32_t tempty_leader0 = cluster_map(&tempty[0], 0);
    const uint32_t tempty_leader1 = cluster_map(&tempty[1], 0);

    // Both accumulators start at the conversion bias.
#pragma unroll 1
    for (int b = 0; b < 2; ++b)
#pragma unroll
      for (int c = 0; c < 16; ++c)
        tmem_st_16x256b_x2_fill(tbase + lane_base + (static_cast<uint32_t>(16 * (c & 1)) << 16) +
                                    b * BN + h * 128 + 16 * (c >> 1),
                                kBias);
    tmem_st_wait();
    tc_fence_before_sync();
    __syncwarp();
    if (lane == 0) {
      mbar_arrive_cluster(tempty_leader0);
      mbar_arrive_cluster(tempty_leader1);
    }

    float2 acc[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) acc[i] = make_float2(0.f, 0.f);
    const float2 negC = make_float2(-kBiasF, -kBiasF);
    TileWalk w;
    w.start(p);
    for (int64_t it = 0; it < iters; ++it, w.next(p)) {
      const int s = static_cast<int>(it % kStages), b = static_cast<int>(it & 1);
      if (!mbar_wait(&tfull[b], static_cast<uint32_t>((it >> 1) & 1), abort_flag) ||
          !mbar_wait(&lfull[s], static_cast<uint32_t>((it / kStages) & 1), abort_flag)) {
        fail();
        break;
      }
      tc_fence_after_sync();
      const uint8_t *stage = stages + s * kStageBytes;
      float4 sa4 = *reinterpret_cast<const float4 *>(stage + kSaOff + (q * 32 + i0 * 4) * 4);
      if (w.g < p.G - 1) {  // INT4 partials are 256*P
        sa4.x *= 0.00390625f;
        sa4.y *= 0.00390625f;
        sa4.z *= 0.00390625f;
        sa4.w *= 0.00390625f;
      }
      const float *sw_s = reinterpret_cast<const float *>(stage + kSwOff);
      const uint32_t tcol = tbase + lane_base + b * BN + h * 128;

      // chunk c: 16-column block pair j = c >> 1, TMEM lane half lh = c & 1
      uint32_t ra[8], rb[8];
      tmem_ld_16x256b_x2(tcol, ra);
      tmem_ld_wait(ra);
#pragma unroll
      for (int c = 0; c < 16; c += 2) {
        const int j = c >> 1;
        const float4 s4 = *reinterpret_cast<const float4 *>(sw_s + ((8 * h + j) * 4 + t0) * 4);
        const float2 swa = make_float2(s4.x, s4.y), swb = make_float2(s4.z, s4.w);
        const float2 nca = f2_mul(swa, negC), ncb = f2_mul(swb, negC);
#pragma unroll
        for (int lh = 0; lh < 2; ++lh) {
          uint32_t(&r)[8] = lh ? rb : ra;
          uint32_t(&rn)[8] = lh ? ra : rb;
          const int cn = c + lh + 1;  // next chunk
          if (cn < 16)
            tmem_ld_16x256b_x2(
                tcol + (static_cast<uint32_t>(16 * (cn & 1)) << 16) + 16 * (cn >> 1), rn);
          // this chunk's partials are in registers: refill it with the bias
          tmem_st_16x256b_x2_fill(tcol + (static_cast<uint32_t>(16 * lh) << 16) + 16 * j, kBias);
          if (kPartials) {
            const int row0 = w.m0 + BM * rank + 32 * q + 16 * lh + i0;
            const int col = w.n0 + h * 128 + 16 * j + 2 * t0;
            const bool int4_group = w.g < p.G - 1;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int row = row0 + 8 * (e & 1);
              const int cc = col + 8 * (e >> 1);
              int32_t v0 = static_cast<int32_t>(r[2 * e] - kBias);
              int32_t v1 = static_cast<int32_t>(r[2 * e + 1] - kBias);
              if (int4_group) {
                v0 >>= 8;
                v1 >>= 8;
              }
              const bool ok = row < p.M && cc < p.N;
              st_global_v2_if(
                  p.partials + (static_cast<int64_t>(w.g) * p.M + (ok ? row : 0)) * p.N +
                      (ok ? cc : 0),
                  static_cast<uint32_t>(v0), static_cast<uint32_t>(v1), ok);
            }
          }
          float2 *a = acc + (2 * j + lh) * 4;
          const float2 f0 = make_float2(__uint_as_float(r[0]), __uint_as_float(r[1]));
          const float2 f1 = make_float2(__uint_as_float(r[2]), __uint_as_float(r[3]));
          const float2 f2 = make_float2(__uint_as_float(r[4]), __uint_as_float(r[5]));
          const float2 f3 = make_float2(__uint_as_float(r[6]), __uint_as_float(r[7]));
          const float sa_lo = lh ? sa4.z : sa4.x, sa_hi = lh ? sa4.w : sa4.y;
          a[0] = f2_fma(f2_fma(f0, swa, nca), make_float2(sa_lo, sa_lo), a[0]);
          a[1] = f2_fma(f2_fma(f1, swa, nca), make_float2(sa_hi, sa_hi), a[1]);
          a[2] = f2_fma(f2_fma(f2, swb, ncb), make_float2(sa_lo, sa_lo), a[2]);
          a[3] = f2_fma(f2_fma(f3, swb, ncb), make_float2(sa_hi, sa_hi), a[3]);
          if (cn < 16) tmem_ld_wait(rn);
        }
      }
      // the accumulator is read and refilled with the bias: hand it back
      tmem_st_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_cluster(b ? tempty_leader1 : tempty_leader0);
        mbar_arrive(&empty[s]);
      }

      if (w.g == p.G - 1) {
        // epilogue: this thread's 4 rows x 32 columns as fp16 pairs
        const bool have_y = p.y != nullptr;
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
          for (int lh = 0; lh < 2; ++lh)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int row = w.m0 + BM * rank + 32 * q + 16 * lh + i0 + 8 * (e & 1);
              const int col = w.n0 + h * 128 + 16 * j + 2 * t0 + 8 * (e >> 1);
              const bool ok = have_y && row < p.M && col < p.N;
              const float2 v = acc[(2 * j + lh) * 4 + e];
              st_global_b32_if(p.y + static_cast<int64_t>(ok ? row : 0) * p.N + (ok ? col : 0),
                               pack_half2_rn(v.x, v.y), ok);
            }
#pragma unroll
        for (int i = 0; i < 64; ++i) acc[i] = make_float2(0.f, 0.f);
      }
    }
  } else {
    regs_decrease<kLoaderRegs>();
    if (warp == 0) {
      // ============================================================== MMA issuer (leader)
      if (rank == 0 && lane == 0) {
        int64_t last = -1;
        for (int64_t it = 0; it < iters; ++it) {
          const int s = static_cast<int>(it % kStages), b = static_cast<int>(it & 1);
          if (!mbar_wait_cluster(&mfull[s], static_cast<uint32_t>((it / kStages) & 1),
                                 abort_flag) ||
              !mbar_wait_cluster(&tempty[b], static_cast<uint32_t>((it >> 1) & 1), abort_flag)) {
            fail();
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_addr = smem_addr(stages + s * kStageBytes);
          const uint64_t adesc = smem_desc_k_sw128(a_addr);
          const uint64_t bdesc = smem_desc_k_sw128(a_addr + kABytes);
          const uint32_t d = tbase + b * BN;
#pragma unroll
          for (int k = 0; k < 4; ++k) mma_i8_pair(d, adesc + 2 * k, bdesc + 2 * k, kIdesc, 1u);
          tc_commit_pair_multicast(&empty[s], 0x3);
          tc_commit_pair_multicast(&tfull[b], 0x3);
          last = it;
        }
        // nothing may still write TMEM when it is released
        if (last >= 0)
          (void)mbar_wait(&tfull[last & 1], static_cast<uint32_t>((last >> 1) & 1), nullptr);
      }
    } else {
      // ============================================================== loaders
      const int lt = threadIdx.x - 32;
      const int lwarp = warp - 1;
      TileWalk w;
      w.start(p);
      LoaderRegs cur;
      if (iters > 0) loader_fetch(p, w, rank, lt, cur);
      int64_t last_tma = -1;
      for (int64_t it = 0; it < iters; ++it) {
        const int s = static_cast<int>(it % kStages);
        TileWalk wn = w;
        wn.next(p);
        if (!mbar_wait(&empty[s], static_cast<uint32_t>(((it / kStages) & 1) ^ 1), abort_flag)) {
          fail();
          break;
        }
        uint8_t *stage = stages + s * kStageBytes;
        loader_store_refetch(p, w, wn, it + 1 < iters, rank, lt, cur, stage);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&lfull[s]);
          const uint32_t leader_full = cluster_map(&mfull[s], 0);
          if (w.g == p.G - 1 && lwarp == 0) {
            mbar_arrive_expect_tx_cluster(leader_full, kABytes + kBBytes);
            tma_load_2d_pair(stage, &tmap_a8, 0, w.m0 + BM * rank, leader_full);
            tma_load_2d_pair(stage + kABytes, &tmap_w8, 0, w.n0 + BW * rank, leader_full);
            last_tma = it;
          } else {
            mbar_arrive_cluster(leader_full);
          }
        }
        w = wn;
      }
      // after an abort, let this CTA's last tensor copy land before its memory is released
      if (*abort_flag && lane == 0 && lwarp == 0 && last_tma >= 0) {
        const int s = static_cast<int>(last_tma % kStages);
        (void)mbar_wait(&empty[s], static_cast<uint32_t>((last_tma / kStages) & 1), nullptr);
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  __syncwarp();
  cluster_sync();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc_pair(tbase, kTmemCols);
  }
}

}  // namespace atomk
