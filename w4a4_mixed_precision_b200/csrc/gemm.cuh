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
// 128-wide K group is four 2-SM MMAs (cta_group::2, M=256, N=256, K=32): the
// B operand is CTA 0's 128 W rows followed by CTA 1's, so accumulator column j
// is tile column j. Two groups are in flight in two 256-column TMEM
// accumulators per CTA. The pairs are persistent over tiles (m fastest).
//
// Three shared-memory rings decouple the stages, so that no stage holds a
// buffer longer than its own step needs:
//   packed ring   (TMA -> unpackers): one slot per INT4 group (128 rows x 64 B
//                 of A and of W, plus the group's sw and sa vectors); the INT8
//                 outlier group takes two slots (A8, then W8, each 128 x 128 B
//                 in the 128-byte-swizzled MMA layout). Freed by the unpackers.
//   operand ring  (unpackers -> MMA): the group's K-major, 128-byte-swizzled
//                 int8 A and W tiles. Freed by the MMA's commit.
//   scale ring    (unpackers -> drain): sa and sw laid out for the drain's
//                 TMEM fragments. Freed by the drain.
// plus one 4 KB Y staging box per drain warp (drain -> TMA store).
// Roles in each CTA:
//
//   producer (warp 0, lane 0)  TMA copies into the packed ring.
//   warp 1, lane 0     (leader CTA) per group: 4 x 2-SM MMA into a 256-column
//                      TMEM accumulator, then commits to both CTAs'
//                      "accumulator full" and "operands free" barriers.
//   unpack warps 2..7  expand each nibble of the packed tiles to a byte
//                      holding 16*q (x << 4 & 0xF0 / x & 0xF0), store K-major
//                      with the 128-byte swizzle (the INT8 group is copied),
//                      and lay the scales out for the drain; then one thread
//                      signals "operands ready" locally and, from the peer CTA,
//                      to the leader.
//   drain warps 8..15  warps 8..11 drain accumulator columns [0, 128) and
//                      12..15 columns [128, 256): each thread reads one TMEM
//                      lane (one output row) with the 32x32b shape, 16 columns
//                      per load, accumulates sa*sw*P into 128 fp32 registers,
//                      and arrives on the leader's "accumulator free" barrier
//                      once its loads are done. After the last group of a
//                      tile: fp16 Y, staged per warp in shared memory as two
//                      32x64 boxes and written by TMA tensor stores.
//
// Exact integer -> float without a conversion instruction: every accumulator
// starts at the int32 0x4B400000 (the bits of C = 1.5*2^23) and the MMAs add
// the group's partial P onto it, so the int32 in TMEM is the bit pattern of
// the float C + P, exact for |P| < 2^22 (INT4 groups: |256 P| <= 1.6e6; INT8
// group: |P| <= 2.1e6). The bias is written by the tensor core itself: each
// group starts with one fp16 MMA (K = 16, accumulate off) of two constant
// tiles whose only nonzero column holds 6144 in A and 2048 in B, so every
// accumulator element becomes the fp32 6144 * 2048 = 1.5*2^23 exactly, and the
// group's integer MMAs then accumulate onto those bits. (Re-arming the columns
// with TMEM stores from the drain cost the drain ~20 % of its time per group.)
// Dequantisation: with sa' = sa truncated to 22 significant bits, C*sa' is
// exact for C = 1.5*2^23, so t = fma(F, sa', -C*sa') = round(P*sa') in one
// instruction, then acc = fma(t, sw, acc); both run as packed f32x2 pairs.
// (The truncation changes sa by less than 2^-21 relative.)
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
constexpr int kThreads = 512;
constexpr int kUnpackThreads = 192;  // warps 2..7
constexpr int kUnpackWarps = kUnpackThreads / 32;
constexpr int kNP = 4;           // packed ring slots
constexpr int kNU = 3;           // operand ring slots
constexpr int kNS = 6;           // scale ring slots
// packed slot: INT4 A at 0, INT4 W at kPackWOff; or one INT8 tile at 0
constexpr uint32_t kPackWOff = BM * 64;
constexpr uint32_t kSwLinOff = 16384;                  // sw as copied (256 floats)
constexpr uint32_t kSaLinOff = kSwLinOff + BN * 4;     // sa as copied (128 floats)
constexpr uint32_t kPSlot = 18u * 1024u;
// operand slot: A then W, int8, K-major, 128-byte swizzle
constexpr uint32_t kABytes = BM * 128;
constexpr uint32_t kBBytes = BW * 128;
constexpr uint32_t kUSlot = kABytes + kBBytes;
// scale slot: sa then sw, in drain order
constexpr uint32_t kSwOff = BM * 4;
constexpr uint32_t kSSlot = (BM + BN) * 4;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kBarBytes = 1024;
constexpr uint32_t kUOff = kBarBytes;                    // from the 1024-aligned base
constexpr uint32_t kPOff = kUOff + kNU * kUSlot;
constexpr uint32_t kSOff = kPOff + kNP * kPSlot;
// Y staging: one 32-row x 64-column fp16 box (128-byte swizzle) per drain warp
constexpr uint32_t kYSlot = 32 * 128;
constexpr uint32_t kYOff = (kSOff + kNS * kSSlot + 1023u) & ~1023u;
// bias tiles of the fp16 bias MMA: A then B, each 128 rows x 16 fp16 (K-major,
// no swizzle: core matrices of 8 rows x 16 B, K-adjacent 128 B apart, row
// groups 256 B apart)
constexpr uint32_t kBiasTile = 128 * 32;
constexpr uint32_t kBiasOff = kYOff + 8 * kYSlot;
constexpr uint32_t kBiasLbo = 128, kBiasSbo = 256;
constexpr uint32_t kIdescBias = idesc_f16(2 * 128, 256);
constexpr uint32_t kSmemBytes = kBiasOff + 2 * kBiasTile + 1024;  // + alignment slack
constexpr int kPackedChunks = (BM + BW) * 4;                    // 16-B chunks per INT4 group
constexpr int kChunksPerThread = (kPackedChunks + kUnpackThreads - 1) / kUnpackThreads;
constexpr int kInt8Chunks = (kABytes + kBBytes) / 16;           // 16-B chunks of an INT8 group
constexpr int kHalfN = BN / 2;   // accumulator columns per drain warp
constexpr uint32_t kIdesc = idesc_i8(kPairM, BN);
constexpr uint32_t kBias = 0x4B400000u;  // bits of 1.5 * 2^23
constexpr float kBiasF = 12582912.0f;
constexpr int kUnpackRegs = 72;
constexpr int kDrainRegs = 184;
static_assert(kSaLinOff + BM * 4 <= kPSlot, "packed slot overflow");
static_assert(kABytes <= kSwLinOff && kBBytes <= kSwLinOff, "INT8 tile must fit a packed slot");
static_assert(kPSlot % 1024 == 0 && kUSlot % 1024 == 0, "slots must keep 1024-byte alignment");
static_assert(kSOff % 16 == 0 && kSSlot % 16 == 0, "scale slots must be 16-byte aligned");
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
static_assert(kYOff % 1024 == 0 && kYSlot % 1024 == 0, "Y staging must keep 1024-byte alignment");
static_assert(2 * 128 * (kUnpackRegs + kDrainRegs) == 65536, "register split must fill the file");
}  // namespace gemm_cfg

struct GemmParams {
  const uint8_t *qa4;
  const float *sa;
  const uint8_t *qw4;
  const float *sw;
  __half *y;           // may be null in partials mode; null in quant-out mode
  int32_t *partials;   // partials mode only
  uint8_t *qy4;        // quant-out mode: Y's INT4 codes [M][(N-128)/2],
  int8_t *qy8;         //   INT8 codes of its last 128 columns [M][128],
  float *sy;           //   and group scales [N/128][M]
  float *ws;           // splits > 1: fp32 partial outputs [splits][M][N]
  const uint8_t *qw4t; // packed INT4 W in the tiled layout (tiled.cuh), or null: row layout by TMA
  int w_tiles;         // 128-row weight tiles, ceil(N / 128)
  int M, N, K, G;
  int m_tiles, n_tiles, tiles;   // pair tiles of 256 x 256
  int splits;                    // K splits per tile (1: no split)
  int items;                     // tiles * splits
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

// 8-byte store of an fp32 pair, passed as two f32 operands (the accumulator
// pairs live in 64-bit registers for the f32x2 arithmetic; handing them over
// as 32-bit integer operands made the compiler spill the accumulators).
__device__ __forceinline__ void st_global_f2_if(void *p, float2 v, bool pred) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %3, 0;\n\t@q st.global.v2.f32 [%0], {%1, %2};\n\t}" ::"l"(
          p),
      "f"(v.x), "f"(v.y), "r"(static_cast<uint32_t>(pred))
      : "memory");
}

__device__ __forceinline__ void st_global_v2_if(void *p, uint32_t a, uint32_t b, bool pred) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %3, 0;\n\t@q st.global.v2.b32 [%0], {%1, %2};\n\t}" ::"l"(
          p),
      "r"(a), "r"(b), "r"(static_cast<uint32_t>(pred))
      : "memory");
}

// Walks one CTA pair's (item, group) sequence; both CTAs of a pair walk the
// same one. An item is one output tile and one of its `splits` K ranges: item
// i is tile i / splits, split i % splits, groups [split*G/splits,
// (split+1)*G/splits). The pairs take items round-robin.
struct TileWalk {
  int item, g, g_end, split, m0, n0;
  __device__ __forceinline__ void start(const GemmParams &p) {
    item = blockIdx.x >> 1;
    set(p);
  }
  __device__ __forceinline__ void set(const GemmParams &p) {
    const int tile = item / p.splits;
    split = item - tile * p.splits;
    m0 = (tile % p.m_tiles) * gemm_cfg::kPairM;
    n0 = (tile / p.m_tiles) * gemm_cfg::BN;
    g = split * p.G / p.splits;
    g_end = (split + 1) * p.G / p.splits;
  }
  __device__ __forceinline__ bool last() const { return g == g_end - 1; }
  __device__ __forceinline__ void next(const GemmParams &p) {
    if (++g == g_end) {
      item += gridDim.x >> 1;
      set(p);
    }
  }
};

// Position in a ring of n slots: slot index and the parity of the slot's
// current use (flips each time the index wraps).
struct RingPos {
  int idx = 0;
  uint32_t phase = 0;
  __device__ __forceinline__ void next(int n) {
    if (++idx == n) {
      idx = 0;
      phase ^= 1u;
    }
  }
};

__device__ __forceinline__ int64_t pair_iterations(const GemmParams &p) {
  const int pair = static_cast<int>(blockIdx.x >> 1), pairs = static_cast<int>(gridDim.x >> 1);
  if (p.splits == 1) {
    const int mine = p.items > pair ? (p.items - pair + pairs - 1) / pairs : 0;
    return static_cast<int64_t>(mine) * p.G;
  }
  int64_t n = 0;
  for (int it = pair; it < p.items; it += pairs) {
    const int s = it % p.splits;
    n += (s + 1) * p.G / p.splits - s * p.G / p.splits;
  }
  return n;
}

// ------------------------------------------------------------------ unpack role

// Scale slot layout: sa by local row (128 floats), then sw by tile column (256
// floats), so a drain thread, which owns one row, reads its sa once and the sw
// of 16 consecutive columns as four 16-byte broadcast loads.
// One INT4 group: expands this thread's share of the packed tiles in `pk`
// into the swizzled int8 operands in `op`.
__device__ __forceinline__ void unpack_int4(int lt, const uint8_t *pk, uint8_t *op) {
  using namespace gemm_cfg;
#pragma unroll
  for (int i = 0; i < kChunksPerThread; ++i) {
    const int c = lt + kUnpackThreads * i;
    if (c < kPackedChunks) {
      const bool is_a = c < BM * 4;
      const int cc = c & 3;
      const int row = (is_a ? c : c - BM * 4) >> 2;
      const uint4 v =
          *reinterpret_cast<const uint4 *>(pk + (is_a ? 0u : kPackWOff) + row * 64 + cc * 16);
      uint8_t *dst = op + (is_a ? 0u : kABytes) + row * 128;
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

// The INT8 outlier group: both tiles arrived already in the swizzled MMA
// layout (A8 in `pk_a`, W8 in `pk_w`, both 1024-byte aligned like `op`), so
// they are copied byte for byte.
__device__ __forceinline__ void copy_int8(int lt, const uint8_t *pk_a, const uint8_t *pk_w,
                                          uint8_t *op) {
  using namespace gemm_cfg;
  for (int c = lt; c < kInt8Chunks; c += kUnpackThreads) {
    const bool is_a = c < static_cast<int>(kABytes / 16);
    const uint32_t off = (is_a ? c : c - kABytes / 16) * 16u;
    *reinterpret_cast<uint4 *>(op + (is_a ? 0u : kABytes) + off) =
        *reinterpret_cast<const uint4 *>((is_a ? pk_a : pk_w) + off);
  }
}

// A W4A8 INT4 group: the INT8 activation tile arrived already in the swizzled
// MMA layout (`pk_a`) and is copied; the packed INT4 weight tile (`pk_w`, 128
// rows x 64 bytes) is unpacked to bytes holding 16*q. Unlike unpack_int4, which
// writes a chunk's even elements before its odd ones (harmless there: A and W
// share that order), the elements keep their natural K order here, to match A.
__device__ __forceinline__ void copy_a8_unpack_w4(int lt, const uint8_t *pk_a, const uint8_t *pk_w,
                                                  uint8_t *op) {
  using namespace gemm_cfg;
  constexpr int kAChunks = static_cast<int>(kABytes / 16);
  for (int c = lt; c < kAChunks + BW * 4; c += kUnpackThreads) {
    if (c < kAChunks) {
      *reinterpret_cast<uint4 *>(op + c * 16u) = *reinterpret_cast<const uint4 *>(pk_a + c * 16u);
    } else {
      const int cw = c - kAChunks, row = cw >> 2, cc = cw & 3;
      const uint4 v = *reinterpret_cast<const uint4 *>(pk_w + row * 64 + cc * 16);
      uint8_t *dst = op + kABytes + row * 128;
      // packed byte i holds elements 2i (low nibble) and 2i+1: L byte i = 16*q[2i],
      // H byte i = 16*q[2i+1]; interleave them back into element order
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t o[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t L = (w[j] << 4) & 0xF0F0F0F0u, H = w[j] & 0xF0F0F0F0u;
        o[2 * j] = __byte_perm(L, H, 0x5140);       // elements 8j .. 8j+3
        o[2 * j + 1] = __byte_perm(L, H, 0x7362);   // elements 8j+4 .. 8j+7
      }
      const int sw = row & 7;
      *reinterpret_cast<uint4 *>(dst + (((2 * cc) ^ sw) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
      *reinterpret_cast<uint4 *>(dst + (((2 * cc + 1) ^ sw) << 4)) =
          make_uint4(o[4], o[5], o[6], o[7]);
    }
  }
}

// Lays the group's scales out for the drain (threads 0..127: sa; 128..191: sw).
// `sa_direct` is this thread's sa value when sa does not come through TMA.
__device__ __forceinline__ void layout_scales(const GemmParams &p, int lt, const uint8_t *pk,
                                              uint8_t *ss, float sa_direct) {
  using namespace gemm_cfg;
  if (lt < BM) {
    reinterpret_cast<float *>(ss)[lt] =
        p.sa_by_tma ? reinterpret_cast<const float *>(pk + kSaLinOff)[lt] : sa_direct;
  } else {
    constexpr int kSwThreads = kUnpackThreads - BM;   // threads laying out sw
    static_assert(kSwThreads > 0, "unpack threads must cover sa and sw");
#pragma unroll
    for (int k = 0; k < (BN + kSwThreads - 1) / kSwThreads; ++k) {
      const int j = lt - BM + kSwThreads * k;
      if (j < BN)
        reinterpret_cast<float *>(ss + kSwOff)[j] =
            reinterpret_cast<const float *>(pk + kSwLinOff)[j];
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
  CUtensorMap y;    // fp16 Y [M][N], boxes of 32 rows x 64 columns, 128-byte swizzle (stores)
};

// Hardware barrier ids for the role-internal gathers (0 is __syncthreads).

// kA8: W4A8, the activations are INT8 in every group ([M][K], loaded per
// group like the INT8 outlier tile); the INT4 weight groups unpack as usual.
template <bool kPartials, bool kQuantOut = false, bool kA8 = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(gemm_cfg::kThreads, 1)
w4a4_gemm_kernel(const __grid_constant__ GemmMaps maps, const GemmParams p) {
  using namespace gemm_cfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);

  uint64_t *pfull = reinterpret_cast<uint64_t *>(smem);  // [kNP] TMA -> unpackers
  uint64_t *pempty = pfull + kNP;      // [kNP] unpackers -> producer
  uint64_t *ufull = pempty + kNP;      // [kNU] operands ready (local) -> MMA
  uint64_t *mfull = ufull + kNU;       // [kNU] leader only: the peer's operands ready
  uint64_t *uempty = mfull + kNU;      // [kNU] MMA commit -> unpackers (both CTAs)
  uint64_t *sfull = uempty + kNU;      // [kNS] scales ready -> drain
  uint64_t *sempty = sfull + kNS;      // [kNS] drain -> unpackers
  uint64_t *tfull = sempty + kNS;      // [2]   accumulator buffer b complete
  uint64_t *tempty = tfull + 2;        // [2]   leader only: buffer b drained by both CTAs
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  uint8_t *uring = smem + kUOff;
  uint8_t *pring = smem + kPOff;
  uint8_t *sring = smem + kSOff;
  uint8_t *ystage = smem + kYOff;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = static_cast<int>(cluster_cta_rank());

  // the bias tiles: element (row, k = 0) = 6144 (A) or 2048 (B), all else 0
  for (int i = threadIdx.x; i < static_cast<int>(2 * kBiasTile / 16); i += kThreads) {
    const int t = i / static_cast<int>(kBiasTile / 16), j = (i >> 3) & 1;
    const uint32_t v = j == 0 ? (t == 0 ? 0x6E00u : 0x6800u) : 0u;   // fp16 6144 / 2048
    reinterpret_cast<uint4 *>(smem + kBiasOff)[i] = make_uint4(v, 0u, 0u, 0u);
  }
  fence_proxy_async_smem();

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNP; ++s) {
      mbar_init(&pfull[s], 1);       // producer's expect_tx arrival (+ TMA bytes)
      mbar_init(&pempty[s], kUnpackWarps);   // lane 0 of each unpack warp
    }
    for (int s = 0; s < kNU; ++s) {
      mbar_init(&ufull[s], kUnpackWarps);    // lane 0 of each local unpack warp
      mbar_init(&mfull[s], kUnpackWarps);    // lane 0 of each of the peer's unpack warps
      mbar_init(&uempty[s], 1);      // the MMA commit
    }
    for (int s = 0; s < kNS; ++s) {
      mbar_init(&sfull[s], kUnpackWarps);    // lane 0 of each unpack warp
      mbar_init(&sempty[s], 8);      // one lane of each drain warp
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 16);     // lane 0 of each of the 8 drain warps in each CTA
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
    // Warp 8 + 4*hh + q owns TMEM lanes [32q, 32q+32) (the hardware's lane
    // quarter for its warp) of accumulator half hh: thread `lane` holds row
    // 32q + lane, columns [128hh, 128hh+128) of the accumulator, as 64 fp32
    // pairs. The two halves are drained and released independently.
    regs_increase<kDrainRegs>();
    const int dw = warp - 8;
    const int q = dw & 3;
    const int hh = dw >> 2;
    const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
    const uint32_t tempty_leader = cluster_map(&tempty[0], 0);
    const int lrow = 32 * q + lane;   // row within the CTA's 128

    float2 acc[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) acc[i] = make_float2(0.f, 0.f);
    TileWalk w;
    w.start(p);
    RingPos sr;
    for (int64_t it = 0; it < iters; ++it, w.next(p), sr.next(kNS)) {
      const int b = static_cast<int>(it & 1), sl = sr.idx;
      const uint32_t tph = static_cast<uint32_t>((it >> 1) & 1);
      // Both phases have usually completed by now: test them with two
      // back-to-back try_waits and enter the (inline, timed) waits only if one
      // has not; the inline wait alone costs ~160 cycles even on a completed
      // phase, twice per group.
      bool ok = mbar_try_wait(&tfull[b], tph) & mbar_try_wait(&sfull[sl], sr.phase);
      if (!ok)
        ok = mbar_wait_inline(&tfull[b], tph, abort_flag) &&
             mbar_wait_inline(&sfull[sl], sr.phase, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) fail();
        break;
      }
      tc_fence_after_sync();
      const uint8_t *ss = sring + sl * kSSlot;
      // t = fma(F, sa', -C*sa') = P*sa' exactly-rounded, with sa' = sa (times
      // 1/256 for the INT4 groups, whose partials are 256*P) truncated to 22
      // significant bits so that C*sa' is exact; then acc += t * sw.
      float sa = reinterpret_cast<const float *>(ss)[lrow];
      if (w.g < p.G - 1) sa *= kA8 ? 0.0625f : 0.00390625f;
      sa = __uint_as_float(__float_as_uint(sa) & 0xFFFFFFFCu);
      const float2 sa2 = make_float2(sa, sa);
      const float2 nc2 = make_float2(-kBiasF * sa, -kBiasF * sa);
      const float4 *sw4 = reinterpret_cast<const float4 *>(ss + kSwOff) + hh * 32;
      const uint32_t tcol = tbase + lane_base + b * BN + hh * kHalfN;

      uint32_t ra[16], rb[16];
      tmem_ld_x16(tcol, ra);
      tmem_ld_wait(ra);
#pragma unroll
      for (int c = 0; c < 8; ++c) {   // 16 accumulator columns per chunk
        uint32_t(&r)[16] = (c & 1) ? rb : ra;
        uint32_t(&rn)[16] = (c & 1) ? ra : rb;
        if (c + 1 < 8) tmem_ld_x16(tcol + 16 * (c + 1), rn);
        if (kPartials) {
          // 16 consecutive tile columns; N % 8 == 0, so each 4-column store is
          // wholly inside or wholly outside the matrix.
          const int row = w.m0 + BM * rank + lrow;
          const int col0 = w.n0 + hh * kHalfN + 16 * c;
          const int sh = w.g < p.G - 1 ? (kA8 ? 4 : 8) : 0;
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const int col = col0 + 4 * v;
            const bool okp = row < p.M && col < p.N;
            int32_t *dst = p.partials +
                           (static_cast<int64_t>(w.g) * p.M + (okp ? row : 0)) * p.N + (okp ? col : 0);
            st_global_v4_if(dst, static_cast<uint32_t>(static_cast<int32_t>(r[4 * v] - kBias) >> sh),
                            static_cast<uint32_t>(static_cast<int32_t>(r[4 * v + 1] - kBias) >> sh),
                            static_cast<uint32_t>(static_cast<int32_t>(r[4 * v + 2] - kBias) >> sh),
                            static_cast<uint32_t>(static_cast<int32_t>(r[4 * v + 3] - kBias) >> sh),
                            okp);
          }
        }
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const float4 s4 = sw4[4 * c + v];
          float2 *a = acc + 8 * c + 2 * v;
          const float2 f0 = make_float2(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]));
          const float2 f1 = make_float2(__uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
          a[0] = f2_fma(f2_fma(f0, sa2, nc2), make_float2(s4.x, s4.y), a[0]);
          a[1] = f2_fma(f2_fma(f1, sa2, nc2), make_float2(s4.z, s4.w), a[1]);
        }
        if (c + 1 < 8) tmem_ld_wait(rn);
      }
      // this warp's lanes of the half are in registers: hand them back (the
      // next group's bias MMA rewrites them), and the group's scales with them
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0)
          mbar_arrive(&tempty[b]);
        else
          mbar_arrive_cluster_relaxed(tempty_leader + 8u * b);
        mbar_arrive(&sempty[sl]);
      }

      if constexpr (kQuantOut) {
        if (w.last()) {
          // epilogue that writes the next layer's activation codes of Y instead
          // of Y. This thread's row and 128 columns are one group of Y; Y's
          // columns are taken to be in the next layer's reordered channel order
          // already, its last 128 columns being the INT8 outlier group. The
          // steps are those of the activation quantizer applied to fp16 Y: amax
          // of the fp16 values, scale = fl(amax/qmax), inv = fl(qmax/amax),
          // codes = low byte of fl(fl(y*inv) + 1.5*2^23) (round half to even),
          // element 2i in the low nibble of byte i.
          const int row = w.m0 + BM * rank + lrow;
          const int gy = (w.n0 >> 7) + hh;
          const int Gy = p.N >> 7;
          const bool in = row < p.M && gy < Gy;
          const bool dense = gy < Gy - 1;
          float amax = 0.f;
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            const float2 f = __half22float2(__floats2half2_rn(acc[i].x, acc[i].y));
            acc[i] = f;
            amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
          }
          const float qmax = dense ? 7.f : 127.f;
          float scale = 0.f, inv = 0.f;
          if (amax > 0.f) {
            scale = __fdiv_rn(amax, qmax);
            inv = __fdiv_rn(qmax, amax);
          }
          const int64_t r = in ? row : 0;
          uint8_t *d4 = p.qy4 + r * static_cast<int64_t>((p.N - 128) >> 1) + (dense && in ? gy : 0) * 64;
          int8_t *d8 = p.qy8 + r * 128;
#pragma unroll
          for (int blk = 0; blk < 4; ++blk) {   // 32 columns: 16 bytes of INT4 or 32 of INT8 codes
            uint32_t w4[4], w8[8];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t bt[8];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 f = acc[16 * blk + 4 * c + e];
                bt[2 * e] = __float_as_uint(__fadd_rn(__fmul_rn(f.x, inv), 12582912.f));
                bt[2 * e + 1] = __float_as_uint(__fadd_rn(__fmul_rn(f.y, inv), 12582912.f));
              }
              const uint32_t ev = low_bytes4(bt[0], bt[2], bt[4], bt[6]);
              const uint32_t od = low_bytes4(bt[1], bt[3], bt[5], bt[7]);
              w4[c] = (ev & 0x0F0F0F0Fu) | ((od << 4) & 0xF0F0F0F0u);
              w8[2 * c] = low_bytes4(bt[0], bt[1], bt[2], bt[3]);
              w8[2 * c + 1] = low_bytes4(bt[4], bt[5], bt[6], bt[7]);
            }
            st_global_v4_if(d4 + 16 * blk, w4[0], w4[1], w4[2], w4[3], in && dense);
            st_global_v4_if(d8 + 32 * blk, w8[0], w8[1], w8[2], w8[3], in && !dense);
            st_global_v4_if(d8 + 32 * blk + 16, w8[4], w8[5], w8[6], w8[7], in && !dense);
          }
          if (in) p.sy[static_cast<int64_t>(gy) * p.M + row] = scale;
#pragma unroll
          for (int i = 0; i < 64; ++i) acc[i] = make_float2(0.f, 0.f);
        }
      } else if (w.last()) {
        // epilogue, 8 columns of this thread's row per step. fp16 Y goes out
        // through shared memory and the TMA, 64 columns at a time: each thread
        // writes its row of the warp's 32 x 64 box (128-byte swizzle: 16-byte
        // chunk j of row r sits at chunk j ^ (r & 7)), then one lane stores
        // the box (the rows and columns past M and N are not written). When K
        // is split, this split's fp32 partial tile goes out instead, as
        // predicated 8-byte stores. One loop without branches around the
        // accumulator reads: the compiler spills them otherwise.
        const bool to_y = p.splits == 1 && p.y != nullptr, to_ws = p.splits > 1;
        const int row = w.m0 + BM * rank + lrow;
        const int row0 = w.m0 + BM * rank + 32 * q;   // the warp's first row
        float *ws_row = p.ws + (static_cast<int64_t>(w.split) * p.M + (row < p.M ? row : 0)) * p.N;
        uint8_t *ybuf = ystage + dw * kYSlot;
        // Y is written once and not read here: first out of L2
        const uint64_t y_policy = l2_policy_evict_first();
#pragma unroll
        for (int v = 0; v < 16; ++v) {
          if ((v & 7) == 0) {
            if (lane == 0) bulk_wait_group_read0();   // the previous box has left the buffer
            __syncwarp();
          }
          const int col = w.n0 + kHalfN * hh + 8 * v;
          const float2 *a = acc + 4 * v;
          const bool in = row < p.M && col < p.N;
          const int cc = in ? col : 0;
          st_shared_v4(ybuf + lane * 128 + (((v & 7) ^ (lane & 7)) << 4),
                       pack_half2_rn(a[0].x, a[0].y), pack_half2_rn(a[1].x, a[1].y),
                       pack_half2_rn(a[2].x, a[2].y), pack_half2_rn(a[3].x, a[3].y));
#pragma unroll
          for (int k = 0; k < 4; ++k) st_global_f2_if(ws_row + cc + 2 * k, a[k], in && to_ws);
          if ((v & 7) == 7) {
            fence_proxy_async_smem();
            __syncwarp();
            const int col0 = w.n0 + kHalfN * hh + 64 * (v >> 3);
            if (lane == 0 && to_y && row0 < p.M && col0 < p.N) {
              tma_store_2d_hint(&maps.y, ybuf, col0, row0, y_policy);
              bulk_commit_group();
            }
          }
        }
#pragma unroll
        for (int i = 0; i < 64; ++i) acc[i] = make_float2(0.f, 0.f);
      }
    }
    // the Y boxes must be out of shared memory before the CTA exits
    if (lane == 0) bulk_wait_group0();
  } else {
    regs_decrease<kUnpackRegs>();
    if (warp == 0) {
      // ============================================================== producer
      if (lane == 0) {
        // A's tiles are read again for every column of output tiles: keep
        // them in L2 ahead of the streaming Y writes
        const uint64_t a_policy = l2_policy_evict_last();
        TileWalk wp;
        wp.start(p);
        int64_t ls = 0;   // packed-ring load steps issued
        RingPos pr;
        bool ok = true;
        for (int64_t it = 0; ok && it < iters; ++it, wp.next(p)) {
          const int arow = wp.m0 + BM * rank, wrow = wp.n0 + BW * rank;
          const bool int4_group = wp.g < p.G - 1;
          const bool two_slots = kA8 || !int4_group;   // INT8 A tile in its own slot
          for (int part = 0; part < (two_slots ? 2 : 1); ++part) {
            const int s = pr.idx;
            if (!mbar_wait(&pempty[s], pr.phase ^ 1u, abort_flag)) {
              ok = false;
              break;
            }
            uint8_t *slot = pring + s * kPSlot;
            // The packed INT4 W tile: one 8 KB bulk copy from the tiled layout,
            // or a TMA box of the row layout. A tiled W tile past the last
            // weight tile (a pair tile that overhangs N by 128 rows or more) is
            // not fetched: its rows only feed output columns >= N.
            const int wt = wrow / BW;
            const bool w_fetch = p.qw4t == nullptr || wt < p.w_tiles;
            auto load_w4 = [&](uint8_t *dst) {
              if (p.qw4t != nullptr) {
                if (w_fetch)
                  bulk_load(dst, p.qw4t + (static_cast<int64_t>(wt) * (p.G - 1) + wp.g) * (BW * 64),
                            BW * 64u, &pfull[s]);
              } else {
                tma_load_2d(dst, &maps.w4, wp.g * 64, wrow, &pfull[s]);
              }
            };
            const uint32_t w4_bytes = w_fetch ? BW * 64u : 0u;
            if (part == 0) {
              const uint32_t bytes = (two_slots ? kABytes : BM * 64u + w4_bytes) + BN * 4u +
                                     (p.sa_by_tma ? BM * 4u : 0u);
              mbar_arrive_expect_tx(&pfull[s], bytes);
              if (!two_slots) {
                tma_load_2d_hint(slot, &maps.a4, wp.g * 64, arow, &pfull[s], a_policy);
                load_w4(slot + kPackWOff);
              } else {
                // W4A4: the INT8 outlier tile of A ([M][128]); W4A8: group g of A ([M][K])
                tma_load_2d_hint(slot, &maps.a8, kA8 ? wp.g * 128 : 0, arow, &pfull[s], a_policy);
              }
              tma_load_2d(slot + kSwLinOff, &maps.sw, wp.n0, wp.g, &pfull[s]);
              if (p.sa_by_tma) tma_load_2d(slot + kSaLinOff, &maps.sa, arow, wp.g, &pfull[s]);
            } else if (int4_group) {
              // W4A8: the packed INT4 weight tile in the second slot
              mbar_arrive_expect_tx(&pfull[s], w4_bytes);
              load_w4(slot);
            } else {
              mbar_arrive_expect_tx(&pfull[s], kBBytes);
              tma_load_2d(slot, &maps.w8, 0, wrow, &pfull[s]);
            }
            ++ls;
            pr.next(kNP);
          }
        }
        if (!ok) {
          fail();
          // let the tensor copies still in flight land before shared memory is released
          for (int64_t j = (ls > kNP ? ls - kNP : 0); j < ls; ++j)
            (void)mbar_wait(&pfull[j % kNP], static_cast<uint32_t>((j / kNP) & 1), nullptr);
        }
      }
    } else if (warp == 1) {
      if (lane == 0 && rank == 0) {
        // ============================================================ MMA issuer (leader)
        // The peer CTA arrives on mfull (after its proxy fence) and on tempty
        // (after tcgen05.wait::ld and the tcgen05 fence); both are waited on
        // with CTA-scope acquire: a cluster-scope acquire costs hundreds of
        // cycles per wait on B200 and orders nothing more here.
        int64_t last_mma = -1;
        bool ok = true;
        RingPos ur;
        const uint64_t bias_adesc =
            smem_desc_k_noswizzle(smem_addr(smem + kBiasOff), kBiasLbo, kBiasSbo);
        const uint64_t bias_bdesc =
            smem_desc_k_noswizzle(smem_addr(smem + kBiasOff + kBiasTile), kBiasLbo, kBiasSbo);
        for (int64_t it = 0; ok && it < iters; ++it, ur.next(kNU)) {
          const int u = ur.idx, b = static_cast<int>(it & 1);
          const uint32_t ph = ur.phase;
          if (!mbar_wait(&ufull[u], ph, abort_flag) ||
              !mbar_wait(&mfull[u], ph, abort_flag)) {
            ok = false;
            break;
          }
          if (!mbar_wait(&tempty[b], static_cast<uint32_t>(((it >> 1) & 1) ^ 1), abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_addr = smem_addr(uring + u * kUSlot);
          const uint64_t adesc = smem_desc_k_sw128(a_addr);
          const uint64_t bdesc = smem_desc_k_sw128(a_addr + kABytes);
          const uint32_t d = tbase + b * BN;
          // the group's accumulator starts at the conversion bias (see above)
          mma_f16_pair(d, bias_adesc, bias_bdesc, kIdescBias, 0u);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_i8_pair(d, adesc + 2 * k, bdesc + 2 * k, kIdesc, 1u);
          tc_commit_pair_multicast(&tfull[b], 0x3);
          tc_commit_pair_multicast(&uempty[u], 0x3);
          last_mma = it;
        }
        if (!ok) fail();
        // nothing may still write TMEM when it is released
        if (last_mma >= 0)
          (void)mbar_wait(&tfull[last_mma & 1],
                          static_cast<uint32_t>((last_mma >> 1) & 1), nullptr);
      }
    } else {
      // ============================================================== unpackers
      const int lt = threadIdx.x - 64;
      TileWalk w;
      w.start(p);
      float sa_d = (!p.sa_by_tma && iters > 0) ? sa_direct_load(p, w, rank, lt) : 0.f;
      const uint32_t mfull_leader = cluster_map(&mfull[0], 0);
      RingPos ur, sr, pr;   // operand, scale and packed rings
      for (int64_t it = 0; it < iters; ++it, ur.next(kNU), sr.next(kNS)) {
        const int u = ur.idx, sl = sr.idx;
        const bool int4_group = w.g < p.G - 1;
        const bool two_slots = kA8 || !int4_group;
        const RingPos p0 = pr;
        RingPos p1 = pr;
        p1.next(kNP);
        const int s0 = p0.idx, s1 = p1.idx;
        TileWalk wn = w;
        wn.next(p);
        bool ok = mbar_try_wait(&uempty[u], ur.phase ^ 1u) &
                  mbar_try_wait(&sempty[sl], sr.phase ^ 1u) & mbar_try_wait(&pfull[s0], p0.phase);
        if (!ok)
          ok = mbar_wait(&uempty[u], ur.phase ^ 1u, abort_flag) &&
               mbar_wait(&sempty[sl], sr.phase ^ 1u, abort_flag) &&
               mbar_wait(&pfull[s0], p0.phase, abort_flag);
        if (ok && two_slots) ok = mbar_wait(&pfull[s1], p1.phase, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) {
          if (lane == 0) fail();
          break;
        }
        const uint8_t *pk = pring + s0 * kPSlot;
        uint8_t *op = uring + u * kUSlot;
        if (!two_slots)
          unpack_int4(lt, pk, op);
        else if (int4_group)
          copy_a8_unpack_w4(lt, pk, pring + s1 * kPSlot, op);
        else
          copy_int8(lt, pk, pring + s1 * kPSlot, op);
        layout_scales(p, lt, pk, sring + sl * kSSlot, sa_d);
        if (!p.sa_by_tma && it + 1 < iters) sa_d = sa_direct_load(p, wn, rank, lt);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&pempty[s0]);
          if (two_slots) mbar_arrive(&pempty[s1]);
          mbar_arrive(&sfull[sl]);
          if (rank == 0)
            mbar_arrive(&ufull[u]);
          else
            mbar_arrive_remote(mfull_leader + 8u * u);
        }
        pr = p1;
        if (two_slots) pr.next(kNP);
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

// Sums the fp32 partial tiles of a split GEMM in split order and writes fp16
// Y: thread t handles columns [8t, 8t + 8) of the flattened [M][N] output
// (N % 8 == 0).
__global__ void __launch_bounds__(256)
splitk_reduce_kernel(const float *__restrict__ ws, __half *__restrict__ y, int64_t count8,
                     int64_t mn, int splits) {
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < count8;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float4 a = __ldg(reinterpret_cast<const float4 *>(ws) + 2 * t);
    float4 b = __ldg(reinterpret_cast<const float4 *>(ws) + 2 * t + 1);
    for (int s = 1; s < splits; ++s) {
      const float4 *src = reinterpret_cast<const float4 *>(ws + s * mn) + 2 * t;
      const float4 c = __ldg(src), d = __ldg(src + 1);
      a.x += c.x; a.y += c.y; a.z += c.z; a.w += c.w;
      b.x += d.x; b.y += d.y; b.z += d.z; b.w += d.w;
    }
    uint4 o;
    o.x = pack_half2_rn(a.x, a.y);
    o.y = pack_half2_rn(a.z, a.w);
    o.z = pack_half2_rn(b.x, b.y);
    o.w = pack_half2_rn(b.z, b.w);
    reinterpret_cast<uint4 *>(y)[t] = o;
  }
}

}  // namespace atomk
