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
// Structure. A cluster of two CTAs on two SMs owns a 256x256 output tile: CTA
// r holds A rows [128r, 128r+128) and W rows [128r, 128r+128) of the tile in
// its shared memory, and its TMEM receives output rows [128r, 128r+128). Each
// 128-wide K group is issued as two column halves of 2-SM MMAs (cta_group::2,
// M=256, N=128, K=32); half h takes W rows [64h, 64h+64) from each CTA, so
// accumulator column j of half h is tile column 64h + (j mod 64) + 128*(j/64).
// Two groups in flight x two halves gives four 128-column accumulators per
// CTA, and the drain hands each half back as soon as it has read it, so the
// tensor cores never wait for a whole group to be drained. The pairs are
// persistent over tiles (m fastest). Roles in each CTA:
//
//   producer (warp 0, lane 0)  TMA copies of the group's packed INT4 tiles
//                      (128 rows x 64 bytes of A and of W), or of the INT8
//                      outlier tiles straight into MMA layout, plus the
//                      group's sa and sw vectors, into a free stage.
//   warp 1, lane 0     (leader CTA) per group and half: 4 x 2-SM MMA into a
//                      128-column TMEM accumulator, commit to both CTAs' "half
//                      full" barrier; after both halves commit to both CTAs'
//                      "stage empty" barrier.
//   unpack warps 2..7  expand each nibble of the staged packed tiles to a byte
//                      holding 16*q (x << 4 & 0xF0 / x & 0xF0), store K-major
//                      with the 128-byte swizzle, and lay the scales out for
//                      the drain; then one thread signals "operands ready"
//                      locally and, in the peer CTA, to the leader.
//   drain warps 8..15  read the partials with the 16x256b TMEM shape (a thread
//                      holds 4 rows x 2 columns of every 8-column block), release
//                      each half once read (one arrival per CTA, on the leader),
//                      and accumulate sa*sw*P into fp32 registers. After the
//                      last group of a tile: fp16 stores.
//
// Exact integer -> float: F = float with the bits P + 0x4B400000 equals
// 1.5*2^23 + P exactly for |P| < 2^22 (one integer add per element; the
// alternative of pre-filling TMEM with that bias doubles the TMEM traffic).
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
constexpr int kStages = 4;
constexpr int kThreads = 512;
constexpr int kUnpackThreads = 192;  // warps 2..7
// stage layout (bytes from a 1024-aligned stage base)
constexpr uint32_t kABytes = BM * 128;                 // unpacked / INT8 A, 128-byte swizzle
constexpr uint32_t kBBytes = BW * 128;                 // unpacked / INT8 W, 128-byte swizzle
constexpr uint32_t kPackAOff = kABytes + kBBytes;      // packed A, 128 rows x 64 B
constexpr uint32_t kPackWOff = kPackAOff + BM * 64;    // packed W, 128 rows x 64 B
constexpr uint32_t kSwLinOff = kPackWOff + BW * 64;    // sw as copied (256 floats)
constexpr uint32_t kSaLinOff = kSwLinOff + BN * 4;     // sa as copied (128 floats)
constexpr uint32_t kSwOff = kSaLinOff + BM * 4;        // sw in drain order
constexpr uint32_t kSaOff = kSwOff + BN * 4;           // sa in drain order
constexpr uint32_t kStageBytes = 52u * 1024u;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kBarBytes = 1024;
constexpr uint32_t kSmemBytes = kBarBytes + kStages * kStageBytes + 1024;  // + alignment slack
constexpr int kPackedChunks = (BM + BW) * 4;                                   // 16-B chunks / group
constexpr int kChunksPerThread = (kPackedChunks + kUnpackThreads - 1) / kUnpackThreads;
constexpr int kHalfN = BN / 2;   // columns per MMA / accumulator half
constexpr uint32_t kIdesc = idesc_i8(kPairM, kHalfN);
constexpr uint32_t kBias = 0x4B400000u;  // bits of 1.5 * 2^23
constexpr float kBiasF = 12582912.0f;
constexpr int kUnpackRegs = 56;
constexpr int kDrainRegs = 200;
static_assert(kSaOff + BM * 4 <= kStageBytes, "stage overflow");
static_assert(kStageBytes % 1024 == 0, "stages must keep 1024-byte alignment");
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
static_assert(2 * 128 * (kUnpackRegs + kDrainRegs) == 65536, "register split must fill the file");
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
  int sa_by_tma;                 // M % 4 == 0: sa rows are 16-byte aligned for TMA
};

// Predicated global stores. Keeping the predicate inside the instruction
// (rather than branching around the store) keeps the epilogue one basic block,
// which is what lets the 128 live accumulators stay in registers.
__device__ __forceinline__ void st_global_b32_if(void *p, uint32_t a, bool pred) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %2, 0;\n\t@q st.global.b32 [%0], %1;\n\t}" ::"l"(p),
      "r"(a), "r"(static_cast<uint32_t>(pred))
      : "memory");
}

__device__ __forceinline__ void st_global_v4_if(void *p, uint32_t a, uint32_t b, uint32_t c,
                                                uint32_t d, bool pred) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %5, 0;\n\t"
      "@q st.global.v4.b32 [%0], {%1, %2, %3, %4};\n\t}" ::"l"(p),
      "r"(a), "r"(b), "r"(c), "r"(d), "r"(static_cast<uint32_t>(pred))
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

// ------------------------------------------------------------------ unpack role

// Tile column of accumulator column c (0..255): c = 128h + j holds the MMA half
// h column j, which is W row 64h + (j mod 64) of CTA j/64.
__device__ __forceinline__ int tile_col(int c) {
  const int h = c >> 7, j = c & 127;
  return ((j >> 6) << 7) + (h << 6) + (j & 63);
}

// Scale layouts in a stage, ordered for the drain's 16x256b fragments:
//  sa: row r = 32q + i + 8k (i < 8, k < 4) at q*32 + i*4 + k, so a thread's four
//      rows are one 16-byte load;
//  sw: accumulator column c = 16S + 8u + 2t + e (t < 4, e, u < 2) at
//      (4S + t)*4 + 2u + e, so a thread's four columns of a 16-column block are
//      one 16-byte load. The stored value is sw of tile column tile_col(c),
//      truncated to 22 significant bits.
__device__ __forceinline__ int sa_slot(int r) { return (r >> 5) * 32 + (r & 7) * 4 + ((r >> 3) & 3); }
__device__ __forceinline__ int sw_slot(int n) {
  const int w = n & 15;
  return ((n >> 4) * 4 + ((w & 7) >> 1)) * 4 + ((w >> 3) << 1) + (w & 1);
}

// Expands this thread's share of the staged packed tiles into the swizzled
// MMA operands and lays out the scales. `sa_direct` is this thread's sa value
// when sa does not come through TMA (rows not 16-byte aligned).
__device__ __forceinline__ void unpack_stage(const GemmParams &p, const TileWalk &w, int lt,
                                             uint8_t *stage, float sa_direct) {
  using namespace gemm_cfg;
  if (w.g < p.G - 1) {
#pragma unroll
    for (int i = 0; i < kChunksPerThread; ++i) {
      const int c = lt + kUnpackThreads * i;
      if (c < kPackedChunks) {
        const bool is_a = c < BM * 4;
        const int cc = c & 3;
        const int row = (is_a ? c : c - BM * 4) >> 2;
        const uint4 v = *reinterpret_cast<const uint4 *>(
            stage + (is_a ? kPackAOff : kPackWOff) + row * 64 + cc * 16);
        uint8_t *dst = stage + (is_a ? 0u : kABytes) + row * 128;
        const uint4 lo = make_uint4((v.x << 4) & 0xF0F0F0F0u, (v.y << 4) & 0xF0F0F0F0u,
                                    (v.z << 4) & 0xF0F0F0F0u, (v.w << 4) & 0xF0F0F0F0u);
        const uint4 hi = make_uint4(v.x & 0xF0F0F0F0u, v.y & 0xF0F0F0F0u, v.z & 0xF0F0F0F0u,
                                    v.w & 0xF0F0F0F0u);
        const int sw = row & 7;
        *reinterpret_cast<uint4 *>(dst + (((2 * cc) ^ sw) << 4)) = lo;
        *reinterpret_cast<uint4 *>(dst + (((2 * cc + 1) ^ sw) << 4)) = hi;
      }
    }
  }
  if (lt < BM) {
    const float v = p.sa_by_tma ? reinterpret_cast<const float *>(stage + kSaLinOff)[lt] : sa_direct;
    reinterpret_cast<float *>(stage + kSaOff)[sa_slot(lt)] = v;
  } else {
    constexpr int kSwThreads = kUnpackThreads - BM;   // threads laying out sw
    static_assert(kSwThreads > 0, "unpack threads must cover sa and sw");
#pragma unroll
    for (int k = 0; k < (BN + kSwThreads - 1) / kSwThreads; ++k) {
      const int j = lt - BM + kSwThreads * k;
      if (j < BN) {
        const float v = reinterpret_cast<const float *>(stage + kSwLinOff)[tile_col(j)];
        reinterpret_cast<float *>(stage + kSwOff)[sw_slot(j)] =
            __uint_as_float(__float_as_uint(v) & 0xFFFFFFFCu);
      }
    }
  }
}

// sa of this thread's row for group w.g read directly from global memory (only
// used when M % 4 != 0, where the rows of sa are not 16-byte aligned for TMA).
__device__ __forceinline__ float sa_direct_load(const GemmParams &p, const TileWalk &w, int rank,
                                                int lt) {
  const int m = w.m0 + gemm_cfg::BM * rank + lt;
  return (lt < gemm_cfg::BM && m < p.M) ? __ldg(p.sa + static_cast<int64_t>(w.g) * p.M + m) : 0.f;
}

// ------------------------------------------------------------------ kernel

// Tensor maps of the operands (built on the host for each call).
struct GemmMaps {
  CUtensorMap a4;   // packed INT4 A: uint8 [M][(K-128)/2], boxes of 128 rows x 64 bytes
  CUtensorMap w4;   // packed INT4 W: uint8 [N][(K-128)/2], boxes of 128 rows x 64 bytes
  CUtensorMap a8;   // INT8 A: [M][128], boxes 128 x 128 bytes, 128-byte swizzle
  CUtensorMap w8;   // INT8 W: [N][128], boxes 128 x 128 bytes, 128-byte swizzle
  CUtensorMap sa;   // fp32 [G][M], boxes of 1 x 128 (used when M % 4 == 0)
  CUtensorMap sw;   // fp32 [G][N], boxes of 1 x 256
};

// Hardware barrier ids for the role-internal gathers (0 is __syncthreads).
constexpr uint32_t kBarDrain = 1, kBarUnpack = 2;

template <bool kPartials>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(gemm_cfg::kThreads, 1)
w4a4_gemm_kernel(const __grid_constant__ GemmMaps maps, const GemmParams p) {
  using namespace gemm_cfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);

  uint64_t *pfull = reinterpret_cast<uint64_t *>(smem);  // [kStages] TMA -> unpackers
  uint64_t *lfull = pfull + kStages;   // [kStages] unpacked (local) -> drain, MMA
  uint64_t *mfull = lfull + kStages;   // [kStages] leader only: the peer's "unpacked"
  uint64_t *empty = mfull + kStages;   // [kStages] MMA commit + local drain -> producer
  uint64_t *tfull = empty + kStages;   // [4]       accumulator (buffer b, half h) at 2b+h
  uint64_t *tempty = tfull + 4;        // [4]       leader only: both CTAs drained (b, h)
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + 4);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  uint8_t *stages = smem + kBarBytes;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = static_cast<int>(cluster_cta_rank());

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&pfull[s], 1);       // producer's expect_tx arrival (+ TMA bytes)
      mbar_init(&lfull[s], 1);       // one unpack thread after the unpack gather
      mbar_init(&mfull[s], 1);       // the peer's unpack thread
      mbar_init(&empty[s], 1 + 8);   // MMA commit + local drain warps
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 2);      // one drain thread of each CTA
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
    const int dw = warp - 8;
    const int q = dw & 3;             // TMEM lane quarter this warp may access
    const int hh = dw >> 2;           // which 64 columns of each accumulator half
    const int t0 = lane & 3;          // column pair within an 8-column block
    const int i0 = lane >> 2;         // row within a group of 8 lanes
    const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
    const bool releaser = dw == 0 && lane == 0;
    const uint32_t tempty_leader = cluster_map(&tempty[0], 0);

    float2 acc[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) acc[i] = make_float2(0.f, 0.f);
    const float2 negC = make_float2(-kBiasF, -kBiasF);
    TileWalk w;
    w.start(p);
    bool aborted = false;
    for (int64_t it = 0; it < iters && !aborted; ++it, w.next(p)) {
      const int s = static_cast<int>(it % kStages), b = static_cast<int>(it & 1);
      const uint32_t tph = static_cast<uint32_t>((it >> 1) & 1);
      const bool ok = mbar_wait(&tfull[2 * b], tph, abort_flag) &&
                      mbar_wait(&lfull[s], static_cast<uint32_t>((it / kStages) & 1), abort_flag);
      if (named_bar_any(kBarDrain, 256, !ok)) {
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
      const uint32_t tbuf = tbase + lane_base + b * BN + hh * 64;

      // chunk c = 4h + 2*j4 + lh: accumulator half h, 32 columns j4, TMEM lane half lh
      uint32_t ra[16], rb[16];
      tmem_ld_16x256b_x4(tbuf, ra);
      tmem_ld_wait(ra);
      float2 swk[4], nck[4];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint32_t(&r)[16] = (c & 1) ? rb : ra;
        uint32_t(&rn)[16] = (c & 1) ? ra : rb;
        const int h = c >> 2, j4 = (c >> 1) & 1, lh = c & 1;
        const int c0 = h * 128 + hh * 64 + 32 * j4;   // accumulator column of this chunk
        if (lh == 0) {
          const float4 s4a = *reinterpret_cast<const float4 *>(sw_s + ((c0 >> 4) * 4 + t0) * 4);
          const float4 s4b =
              *reinterpret_cast<const float4 *>(sw_s + (((c0 >> 4) + 1) * 4 + t0) * 4);
          swk[0] = make_float2(s4a.x, s4a.y);
          swk[1] = make_float2(s4a.z, s4a.w);
          swk[2] = make_float2(s4b.x, s4b.y);
          swk[3] = make_float2(s4b.z, s4b.w);
#pragma unroll
          for (int k = 0; k < 4; ++k) nck[k] = f2_mul(swk[k], negC);
        }
        if (c == 3 || c == 7) {
          // every chunk of half h is in registers: hand the half back
          tc_fence_before_sync();
          bool ok2 = true;
          if (c == 3) ok2 = mbar_wait(&tfull[2 * b + 1], tph, abort_flag);
          if (named_bar_any(kBarDrain, 256, !ok2)) {
            fail();
            aborted = true;
            break;
          }
          if (releaser) {
            if (rank == 0)
              mbar_arrive(&tempty[2 * b + h]);
            else
              mbar_arrive_cluster_relaxed(tempty_leader + 8u * (2 * b + h));
          }
          if (c == 3) tc_fence_after_sync();
        }
        if (c + 1 < 8) {
          const int cn = c + 1;
          tmem_ld_16x256b_x4(tbase + lane_base + (static_cast<uint32_t>(16 * (cn & 1)) << 16) +
                                 b * BN + (cn >> 2) * 128 + hh * 64 + 32 * ((cn >> 1) & 1),
                             rn);
        }
        if (kPartials) {
          const int row0 = w.m0 + BM * rank + 32 * q + 16 * lh + i0;
          const bool int4_group = w.g < p.G - 1;
#pragma unroll
          for (int k = 0; k < 4; ++k)
#pragma unroll
            for (int v = 0; v < 2; ++v) {
              const int row = row0 + 8 * v;
              const int col = w.n0 + tile_col(c0 + 8 * k + 2 * t0);
              int32_t v0 = static_cast<int32_t>(r[4 * k + 2 * v]);
              int32_t v1 = static_cast<int32_t>(r[4 * k + 2 * v + 1]);
              if (int4_group) {
                v0 >>= 8;
                v1 >>= 8;
              }
              const bool okp = row < p.M && col < p.N;
              st_global_v2_if(
                  p.partials + (static_cast<int64_t>(w.g) * p.M + (okp ? row : 0)) * p.N +
                      (okp ? col : 0),
                  static_cast<uint32_t>(v0), static_cast<uint32_t>(v1), okp);
            }
        }
        const float sa_lo = lh ? sa4.z : sa4.x, sa_hi = lh ? sa4.w : sa4.y;
        float2 *a = acc + c * 8;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 flo = make_float2(__uint_as_float(r[4 * k] + kBias),
                                         __uint_as_float(r[4 * k + 1] + kBias));
          const float2 fhi = make_float2(__uint_as_float(r[4 * k + 2] + kBias),
                                         __uint_as_float(r[4 * k + 3] + kBias));
          a[2 * k] = f2_fma(f2_fma(flo, swk[k], nck[k]), make_float2(sa_lo, sa_lo), a[2 * k]);
          a[2 * k + 1] =
              f2_fma(f2_fma(fhi, swk[k], nck[k]), make_float2(sa_hi, sa_hi), a[2 * k + 1]);
        }
        if (c + 1 < 8) tmem_ld_wait(rn);
      }
      if (aborted) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);  // this stage's scales are no longer needed

      if (w.g == p.G - 1) {
        // epilogue. For each 32-column chunk and row, the 4 lanes with the same
        // i0 hold 2 columns of each of the 4 8-column blocks; a 4x4 transpose
        // across those lanes gives lane t0 all 8 columns of block t0, written
        // as one 16-byte store.
        const bool have_y = p.y != nullptr;
#pragma unroll
        for (int c = 0; c < 8; ++c)
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            const int h = c >> 2, j4 = (c >> 1) & 1, lh = c & 1;
            uint32_t hb[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float2 val = acc[c * 8 + 2 * k + v];
              hb[k] = pack_half2_rn(val.x, val.y);
            }
            // round r: send block t0^r to lane t0^r, receive my block t0 from it
            uint32_t o0 = hb[0], o1 = hb[1], o2 = hb[2], o3 = hb[3];
#pragma unroll
            for (int r = 1; r < 4; ++r) {
              const int idx = t0 ^ r;
              const uint32_t send =
                  idx == 0 ? hb[0] : (idx == 1 ? hb[1] : (idx == 2 ? hb[2] : hb[3]));
              const uint32_t got = __shfl_xor_sync(0xffffffffu, send, r);
              o0 = idx == 0 ? got : o0;
              o1 = idx == 1 ? got : o1;
              o2 = idx == 2 ? got : o2;
              o3 = idx == 3 ? got : o3;
            }
            const int row = w.m0 + BM * rank + 32 * q + 16 * lh + i0 + 8 * v;
            const int col = w.n0 + tile_col(h * 128 + hh * 64 + 32 * j4 + 8 * t0);
            const bool oky = have_y && row < p.M && col < p.N;
            st_global_v4_if(p.y + static_cast<int64_t>(oky ? row : 0) * p.N + (oky ? col : 0),
                            o0, o1, o2, o3, oky);
          }
#pragma unroll
        for (int i = 0; i < 64; ++i) acc[i] = make_float2(0.f, 0.f);
      }
    }
  } else {
    regs_decrease<kUnpackRegs>();
    if (warp == 0) {
      // ============================================================== producer
      if (lane == 0) {
        TileWalk wp;
        wp.start(p);
        int64_t produced = 0;
        bool ok = true;
        for (; produced < iters; ++produced, wp.next(p)) {
          const int s = static_cast<int>(produced % kStages);
          if (!mbar_wait(&empty[s], static_cast<uint32_t>(((produced / kStages) & 1) ^ 1),
                         abort_flag)) {
            ok = false;
            break;
          }
          uint8_t *stage = stages + s * kStageBytes;
          const int arow = wp.m0 + BM * rank, wrow = wp.n0 + BW * rank;
          const bool int4_group = wp.g < p.G - 1;
          const uint32_t bytes = (int4_group ? (BM + BW) * 64u : kABytes + kBBytes) + BN * 4u +
                                 (p.sa_by_tma ? BM * 4u : 0u);
          mbar_arrive_expect_tx(&pfull[s], bytes);
          if (int4_group) {
            tma_load_2d(stage + kPackAOff, &maps.a4, wp.g * 64, arow, &pfull[s]);
            tma_load_2d(stage + kPackWOff, &maps.w4, wp.g * 64, wrow, &pfull[s]);
          } else {
            tma_load_2d(stage, &maps.a8, 0, arow, &pfull[s]);
            tma_load_2d(stage + kABytes, &maps.w8, 0, wrow, &pfull[s]);
          }
          tma_load_2d(stage + kSwLinOff, &maps.sw, wp.n0, wp.g, &pfull[s]);
          if (p.sa_by_tma) tma_load_2d(stage + kSaLinOff, &maps.sa, arow, wp.g, &pfull[s]);
        }
        if (!ok) {
          fail();
          // let the tensor copies still in flight land before shared memory is released
          for (int64_t j = (produced > kStages ? produced - kStages : 0); j < produced; ++j)
            (void)mbar_wait(&pfull[j % kStages], static_cast<uint32_t>((j / kStages) & 1), nullptr);
        }
      }
    } else if (warp == 1) {
      if (lane == 0 && rank == 0) {
        // ============================================================ MMA issuer (leader)
        int64_t last_mma = -1;
        bool ok = true;
        for (int64_t it = 0; ok && it < iters; ++it) {
          const int s = static_cast<int>(it % kStages), b = static_cast<int>(it & 1);
          const uint32_t ph = static_cast<uint32_t>((it / kStages) & 1);
          if (!mbar_wait(&lfull[s], ph, abort_flag) ||
              !mbar_wait_cluster(&mfull[s], ph, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t a_addr = smem_addr(stages + s * kStageBytes);
          const uint64_t adesc = smem_desc_k_sw128(a_addr);
#pragma unroll 1
          for (int h = 0; h < 2; ++h) {
            if (!mbar_wait_cluster(&tempty[2 * b + h], static_cast<uint32_t>(((it >> 1) & 1) ^ 1),
                                   abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after_sync();
            // half h: W rows [64h, 64h+64) of each CTA's tile
            const uint64_t bdesc = smem_desc_k_sw128(a_addr + kABytes + h * 64 * 128);
            const uint32_t d = tbase + b * BN + h * kHalfN;
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_i8_pair(d, adesc + 2 * k, bdesc + 2 * k, kIdesc, k > 0 ? 1u : 0u);
            tc_commit_pair_multicast(&tfull[2 * b + h], 0x3);
          }
          if (!ok) break;
          tc_commit_pair_multicast(&empty[s], 0x3);
          last_mma = it;
        }
        if (!ok) fail();
        // nothing may still write TMEM when it is released
        if (last_mma >= 0)
          (void)mbar_wait(&tfull[2 * (last_mma & 1) + 1],
                          static_cast<uint32_t>((last_mma >> 1) & 1), nullptr);
      }
    } else {
      // ============================================================== unpackers
      const int lt = threadIdx.x - 64;
      TileWalk w;
      w.start(p);
      float sa_d = (!p.sa_by_tma && iters > 0) ? sa_direct_load(p, w, rank, lt) : 0.f;
      const uint32_t mfull_leader = cluster_map(&mfull[0], 0);
      for (int64_t it = 0; it < iters; ++it) {
        const int s = static_cast<int>(it % kStages);
        TileWalk wn = w;
        wn.next(p);
        const bool ok = mbar_wait(&pfull[s], static_cast<uint32_t>((it / kStages) & 1), abort_flag);
        if (named_bar_any(kBarUnpack, kUnpackThreads, !ok)) {
          fail();
          break;
        }
        uint8_t *stage = stages + s * kStageBytes;
        unpack_stage(p, w, lt, stage, sa_d);
        if (!p.sa_by_tma && it + 1 < iters) sa_d = sa_direct_load(p, wn, rank, lt);
        fence_proxy_async_smem();
        named_bar_sync(kBarUnpack, kUnpackThreads);
        if (lt == 0) {
          mbar_arrive(&lfull[s]);
          if (rank == 1) mbar_arrive_cluster(mfull_leader + 8u * s);
        }
        w = wn;
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
