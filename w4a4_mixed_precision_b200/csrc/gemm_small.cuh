// gemm_small.cuh -- the W4A4 GEMM for a few tokens (M <= 64, decode).
//
// Same arithmetic as w4a4_gemm_kernel (gemm.cuh): exact int32 per-group
// partials P_g on the tensor cores and Y = sum_g sa * sw * P_g in fp32, with
// every element computed by the same fp32 operations in the same group order
// (so an unsplit call gives bit-identical Y). What changes is the shape of the
// work. A 256x256 tile would leave at most 64 of its rows valid and drain 256
// columns per group; here the weights are the MMA's M side and the tokens its
// N side:
//
//   one CTA owns 128 weight rows (output columns n0..n0+127) and one range of
//   K groups; per group, four tcgen05.mma.cta_group::1.kind::i8 with M = 128
//   (weight rows), N = NT (the tokens rounded up to 16, 32 or 64), K = 32
//   accumulate into one of four NT-column TMEM accumulators; K is split so
//   that about one CTA per SM works. The K ranges of one weight tile are one
//   thread-block cluster (at most 8 CTAs): each parks its fp32 partial tile in
//   its own shared memory, and after a cluster barrier every CTA sums a slice
//   of the tile over all of them through distributed shared memory, in K-range
//   order, with the same fp32 additions as the ordered split-K reduction of
//   gemm.cuh, and writes fp16 Y.
//
// A decode GEMM moves little data per SM (tens of KB) and does little work per
// group, so what sets its time is how early the weights are requested and how
// short each group's path is:
//  * the packed ring has 8 slots, so the producer puts up to 8 groups of
//    weights in flight at once (all of a K range of 8 groups at the start);
//    each slot carries the group's packed W and A tiles and its sw by TMA, and
//    its sa by 4-byte asynchronous copies from the producer warp's lanes (sa
//    rows are M floats, which a TMA cannot address for M % 4 != 0; a register
//    prefetch of them by plain loads made the producer wait on each group's
//    loads and paced the whole kernel at ~0.6 us per group);
//  * the producer starts as soon as the barriers exist: the TMEM allocation
//    runs beside the first loads;
//  * NT/16 drain warps per TMEM lane quarter, each with 16 token columns, so a
//    group costs each drain warp one 16-column TMEM load; an fp16 MMA of
//    constant tiles starts each group's accumulator at the conversion bias (as
//    in gemm.cuh), so the drain writes nothing back to TMEM;
//  * the unpack, MMA and drain roles advance two INT4 groups per step, so each
//    crosses one barrier hand-off per two groups (a hand-off costs a few
//    hundred ns on this part, about as much as a group's work);
//  * four accumulators, two steps of two;
//  * the split-K reduction gives each CTA a slice of 4-row quads: one 16-byte
//    distributed-shared-memory load per K range, all issued before the first
//    add (in K-range order), one 8-byte store of 4 fp16 values;
//  * launched with programmatic stream serialization: the set-up runs while
//    the previous kernel in the stream finishes, and nothing reads an input
//    or writes an output before griddepcontrol.wait.
//
// Roles: warp 0 producer (lane 0 issues the tensor copies, all lanes the sa
// copies); warp 1 allocates TMEM, its lane 0 issues the MMAs; warps 2..7 unpack
// (nibbles to 16*q bytes, K-major, 128-byte swizzle, as in gemm.cuh; the INT8
// outlier group is copied) and lay the scales out; warps 8.. drain.
#pragma once

#include "gemm.cuh"

namespace atomk {

namespace small_cfg {
constexpr int BW = 128;                 // weight rows (output columns) per CTA
constexpr int kMaxTokens = 64;          // token rows per call
constexpr int kUnpackThreads = 192;     // warps 2..7
constexpr int kUnpackWarps = kUnpackThreads / 32;
constexpr int kFirstDrainWarp = 8;
constexpr int kNP = 8;                  // packed slots (groups of weights in flight)
constexpr int kNU = 4;                  // operand slots (one group each)
constexpr int kNS = 8;                  // scale slots
constexpr int kNB = 4;                  // TMEM accumulators, kMaxTokens columns apart
constexpr int kMaxSplits = 8;           // most K ranges of a tile (a portable cluster)
// The unpack, MMA and drain roles advance in steps of two INT4 groups (one
// when a K range has an odd INT4 group left, and the INT8 group alone): each
// step takes a pair of operand slots, a pair of scale slots and a pair of
// accumulators, with one barrier per pair.
constexpr int kUS = kNU / 2, kSS = kNS / 2, kBS = kNB / 2;
// packed slot (1024-byte aligned). INT4 group: W4 (128 rows x 64 B) at 0, A4
// (64 x 64 B) at kPackAOff. The INT8 group takes two slots; slot h holds W8
// rows [64h, 64h+64) (64 x 128 B, 128-byte swizzle) at 0 and A8 rows
// [32h, 32h+32) (32 x 128 B, swizzled) at kPackAOff. A group's first slot also
// holds its sw (128 floats, by TMA) and sa (64 floats, by the producer's copies).
constexpr uint32_t kPackAOff = 8192;
constexpr uint32_t kPackSwOff = 12288;
constexpr uint32_t kPackSaOff = kPackSwOff + BW * 4;
constexpr uint32_t kPSlot = 13 * 1024;
// operand slot: int8 W (128 x 128 B) then int8 A (64 x 128 B), K-major, 128-byte swizzle
constexpr uint32_t kOpAOff = BW * 128;
constexpr uint32_t kUSlot = kOpAOff + kMaxTokens * 128;
// scale slot: per token pair (sa'[2j], sa'[2j+1], -C*sa'[2j], -C*sa'[2j+1]), then sw by weight row
constexpr uint32_t kSwOff = kMaxTokens * 8;
constexpr uint32_t kSSlot = kSwOff + BW * 4;
constexpr uint32_t kBarBytes = 1024;
constexpr uint32_t kPOff = kBarBytes;
constexpr uint32_t kUOff = kPOff + kNP * kPSlot;
constexpr uint32_t kSOff = kUOff + kNU * kUSlot;
// bias tiles of the fp16 MMA: A (BW rows) then B (kMaxTokens rows), 16 fp16
// per row, K-major without swizzle (core matrices of 8 rows x 16 bytes)
constexpr uint32_t kBiasOff = kSOff + kNS * kSSlot;
constexpr uint32_t kBiasA = BW * 32, kBiasB = kMaxTokens * 32;
constexpr uint32_t kBiasLbo = 128, kBiasSbo = 256;
constexpr uint32_t kSmemBytes = kBiasOff + kBiasA + kBiasB + 1024;   // + alignment slack
constexpr uint32_t kTmemCols = kNB * kMaxTokens;
constexpr uint32_t kInt4Bytes = BW * 64 + kMaxTokens * 64 + BW * 4;   // TMA bytes of an INT4 slot
constexpr uint32_t kInt8Bytes0 = 64 * 128 + 32 * 128 + BW * 4;       // first INT8 slot
constexpr uint32_t kInt8Bytes1 = 64 * 128 + 32 * 128;                // second INT8 slot
constexpr int kPackedChunks = (BW + kMaxTokens) * 4;            // 16-byte chunks, INT4 group
constexpr int kInt8Chunks = (BW + kMaxTokens) * 8;              // 16-byte chunks, INT8 group
__host__ __device__ constexpr int threads_for(int NT) { return 32 * (kFirstDrainWarp + NT / 4); }
static_assert(kPSlot % 1024 == 0 && kUSlot % 1024 == 0 && kOpAOff % 1024 == 0, "1024-byte slots");
static_assert(kPackAOff + kMaxTokens * 64 <= kPackSwOff && kPackSaOff + kMaxTokens * 4 <= kPSlot,
              "packed slot");
static_assert(kPackedChunks % kUnpackThreads == 0 && kInt8Chunks % kUnpackThreads == 0, "chunks");
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
static_assert(kTmemCols == 256, "TMEM allocation is a power of two");
}  // namespace small_cfg

struct SmallMaps {
  CUtensorMap w4;   // packed INT4 W: uint8 [N][(K-128)/2], boxes of 128 rows x 64 bytes
  CUtensorMap a4;   // packed INT4 A: uint8 [M][(K-128)/2], boxes of 64 rows x 64 bytes
  CUtensorMap w8;   // INT8 W: [N][128], boxes 64 x 128 bytes, 128-byte swizzle
  CUtensorMap a8;   // INT8 A: [M][128], boxes 32 x 128 bytes, 128-byte swizzle
  CUtensorMap sw;   // fp32 [G][N], boxes of 1 x 128
};

struct SmallParams {
  const float *sa;   // [G][M]
  const float *sw;   // [G][N]
  __half *y;         // may be null in partials mode
  int32_t *partials; // partials mode only: int32 [G][M][N]
  const uint8_t *qw4t;  // packed INT4 W in the tiled layout (tiled.cuh), or null: row layout by TMA
  int M, N, K, G;
  int n_tiles, splits, items;   // splits > 1: one item per CTA, a cluster of `splits` CTAs per tile
};

// The (item, group) sequence of one CTA; every role walks the same one. Item i
// is weight tile i / splits and K range i % splits.
struct SmallWalk {
  int item, g, g_end, split, n0;
  __device__ __forceinline__ void set(const SmallParams &p) {
    const int tile = item / p.splits;
    split = item - tile * p.splits;
    n0 = tile * small_cfg::BW;
    g = split * p.G / p.splits;
    g_end = (split + 1) * p.G / p.splits;
  }
  __device__ __forceinline__ void start(const SmallParams &p) {
    item = blockIdx.x;
    set(p);
  }
  __device__ __forceinline__ bool last() const { return g == g_end - 1; }
  __device__ __forceinline__ void next(const SmallParams &p) {
    if (++g == g_end) {
      item += gridDim.x;
      set(p);
    }
  }
};

__device__ __forceinline__ int64_t small_iterations(const SmallParams &p) {
  int64_t n = 0;
  for (int it = blockIdx.x; it < p.items; it += gridDim.x) {
    const int s = it % p.splits;
    n += (s + 1) * p.G / p.splits - s * p.G / p.splits;
  }
  return n;
}

// The step sequence of the unpack, MMA and drain roles: w at a step's first
// group, n groups in it (2 when the next group is an INT4 group of the same K
// range, else 1).
struct SmallStep {
  SmallWalk w;
  int n;
  __device__ __forceinline__ void fix(const SmallParams &p) {
    n = (w.g + 1 < w.g_end && w.g + 1 < p.G - 1) ? 2 : 1;
  }
  __device__ __forceinline__ void start(const SmallParams &p) {
    w.start(p);
    fix(p);
  }
  __device__ __forceinline__ bool last() const { return w.g + n == w.g_end; }
  __device__ __forceinline__ void next(const SmallParams &p) {
    for (int i = 0; i < n; ++i) w.next(p);
    fix(p);
  }
};

__device__ __forceinline__ int64_t small_steps(const SmallParams &p) {
  int64_t n = 0;
  for (int it = blockIdx.x; it < p.items; it += gridDim.x) {
    const int s = it % p.splits;
    const int g1 = (s + 1) * p.G / p.splits;
    for (int g = s * p.G / p.splits; g < g1; ++n) g += (g + 1 < g1 && g + 1 < p.G - 1) ? 2 : 1;
  }
  return n;
}

// kPartials: also write each group's exact int32 partial sums P[g][m][n] (the
// debug entry point), read from the biased accumulator before the scale
// arithmetic: P = (bits - bias) >> 8 for an INT4 group (the tiles hold 16*q, so
// the MMA sums 256*P), bits - bias for the INT8 group.
template <int NT, bool kPartials = false>
__global__ void __launch_bounds__(small_cfg::threads_for(NT), 1)
w4a4_gemm_small_kernel(const __grid_constant__ SmallMaps maps, const SmallParams p) {
  using namespace small_cfg;
  static_assert(NT == 16 || NT == 32 || NT == 64, "token tile");
  constexpr uint32_t kIdescSmall = idesc_i8(BW, NT);
  constexpr uint32_t kIdescBias = idesc_f16(BW, NT);
  constexpr int kDrainWarps = NT / 4;   // NT/16 per TMEM lane quarter
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);

  uint64_t *pfull = reinterpret_cast<uint64_t *>(smem);   // [kNP] TMA + sa -> unpackers
  uint64_t *pempty = pfull + kNP;                         // [kNP] unpackers -> producer
  uint64_t *ufull = pempty + kNP;                         // [kUS] operand pair ready -> MMA
  uint64_t *uempty = ufull + kUS;                         // [kUS] MMA commit -> unpackers
  uint64_t *sfull = uempty + kUS;                         // [kSS] scale pair ready -> drain
  uint64_t *sempty = sfull + kSS;                         // [kSS] drain -> unpackers
  uint64_t *tfull = sempty + kSS;                         // [kBS] accumulator pair complete
  uint64_t *tempty = tfull + kBS;                         // [kBS] accumulator pair drained
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + kBS);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  uint8_t *pring = smem + kPOff;
  uint8_t *uring = smem + kUOff;
  uint8_t *sring = smem + kSOff;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  launch_dependents();   // the next kernel may start its set-up beside this one
  // barriers: lane i of warp 0 initialises entry i of each ring's pair
  static_assert(kNP <= 32 && kUS <= 32 && kSS <= 32 && kBS <= 32, "barrier init");
  if (warp == 0) {
    if (lane < kNP) {
      mbar_init(&pfull[lane], 33);  // 32 lanes' sa-copy arrivals + the expect_tx arrival
      mbar_init(&pempty[lane], kUnpackWarps);
    }
    if (lane < kUS) {
      mbar_init(&ufull[lane], kUnpackWarps);
      mbar_init(&uempty[lane], 1);
    }
    if (lane < kSS) {
      mbar_init(&sfull[lane], kUnpackWarps);
      mbar_init(&sempty[lane], kDrainWarps);
    }
    if (lane < kBS) {
      mbar_init(&tfull[lane], 1);
      mbar_init(&tempty[lane], kDrainWarps);
    }
    if (lane == 0) *abort_flag = 0;
    fence_mbar_init();
  }
  // the bias tiles: element (row, k = 0) = 6144 (A) or 2048 (B), all else 0
  for (int i = threadIdx.x; i < static_cast<int>((kBiasA + kBiasB) / 16); i += threads_for(NT)) {
    const int t = i >= static_cast<int>(kBiasA / 16), j = (i >> 3) & 1;
    const uint32_t v = j == 0 ? (t == 0 ? 0x6E00u : 0x6800u) : 0u;   // fp16 6144 / 2048
    reinterpret_cast<uint4 *>(smem + kBiasOff)[i] = make_uint4(v, 0u, 0u, 0u);
  }
  fence_proxy_async_smem();
  __syncthreads();
  // the set-up above touches no input or output: from here on, the kernel
  // before this one in the stream has completed
  grid_dependency_wait();
  const int64_t iters = small_iterations(p);   // groups (producer)
  const int64_t steps = small_steps(p);        // steps (unpack, MMA, drain)

  // TMEM: allocated by warp 1 while the producer already loads; warp 1 and the
  // drain warps meet at named barrier 1 to learn its address
  uint32_t tbase = 0;
  if (warp == 1 || warp >= kFirstDrainWarp) {
    if (warp == 1) {
      tmem_alloc(tmem_slot, kTmemCols);
      tmem_relinquish();
      tc_fence_before_sync();
    }
    named_bar_sync(1, 32 * (1 + kDrainWarps));
    tc_fence_after_sync();
    tbase = *tmem_slot;
  }

  auto fail = [&](void) {
    report_status(6 /* ATOM_ERR_TIMEOUT */);
    *abort_flag = 1;
  };

  if (warp >= kFirstDrainWarp) {
    // ================================================================ drain
    // Warp 8 + 4s + q owns TMEM lanes [32q, 32q+32) and token columns
    // [16s, 16s+16): thread `lane` holds weight row n0 + 32q + lane and the
    // accumulators of those 16 tokens.
    const int dw = warp - kFirstDrainWarp;
    const int q = dw & 3, s = dw >> 2;
    const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
    const int lrow = 32 * q + lane;
    float2 acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = make_float2(0.f, 0.f);
    SmallStep st;
    st.start(p);
    RingPos sr, br;
    for (int64_t it = 0; it < steps; ++it, st.next(p), sr.next(kSS), br.next(kBS)) {
      const int b = br.idx, sl = sr.idx;
      bool ok = mbar_try_wait(&tfull[b], br.phase) & mbar_try_wait(&sfull[sl], sr.phase);
      if (!ok)
        ok = mbar_wait(&tfull[b], br.phase, abort_flag) && mbar_wait(&sfull[sl], sr.phase, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) fail();
        break;
      }
      tc_fence_after_sync();
      // the step's groups in order: accumulator 2b + j, scale slot 2sl + j
      for (int j = 0; j < st.n; ++j) {
        const int g = st.w.g + j;
        const uint8_t *ss = sring + (2 * sl + j) * kSSlot;
        // per token pair: (sa'[2j], sa'[2j+1], -C*sa'[2j], -C*sa'[2j+1]); sa' as in gemm.cuh
        const float4 *sap = reinterpret_cast<const float4 *>(ss) + 8 * s;
        const float swr = reinterpret_cast<const float *>(ss + kSwOff)[lrow];
        const float2 sw2 = make_float2(swr, swr);
        const uint32_t tcol = tbase + lane_base + (2 * b + j) * kMaxTokens + 16 * s;
        uint32_t r[16];
        tmem_ld_x16(tcol, r);
        tmem_ld_wait(r);
        if (kPartials) {
          // weight row n, tokens 16s .. 16s+15; consecutive lanes write
          // consecutive n of one token row
          const int n = st.w.n0 + lrow;
          const int sh = g < p.G - 1 ? 8 : 0;
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int m = 16 * s + e;
            if (n < p.N && m < p.M)
              p.partials[(static_cast<int64_t>(g) * p.M + m) * p.N + n] =
                  static_cast<int32_t>(r[e] - gemm_cfg::kBias) >> sh;
          }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {   // token pair 8s + k: tokens 16s + 2k, 16s + 2k + 1
          const float4 s4 = sap[k];
          const float2 f = make_float2(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1]));
          acc[k] = f2_fma(f2_fma(f, make_float2(s4.x, s4.y), make_float2(s4.z, s4.w)), sw2, acc[k]);
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&tempty[b]);
        mbar_arrive(&sempty[sl]);
      }
      if (st.last()) {
        // this K range of the item is complete: write the thread's row of Y
        // (tokens m < M); with a split, park the range's fp32 partial tile
        // [token][weight row] in the operand ring, which no MMA reads any more
        // (the item is the CTA's only one). Consecutive lanes take consecutive
        // columns.
        const int n = st.w.n0 + lrow;
        const bool row_ok = n < p.N;
        float *part = reinterpret_cast<float *>(uring);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int m = 16 * s + 2 * k + h;
            const float v = h ? acc[k].y : acc[k].x;
            if (p.splits > 1)
              part[m * BW + lrow] = v;
            else if (row_ok && m < p.M && p.y != nullptr)
              p.y[static_cast<int64_t>(m) * p.N + n] = __float2half_rn(v);
          }
          acc[k] = make_float2(0.f, 0.f);
        }
      }
    }
  } else if (warp == 0) {
    // ================================================================ producer
    // Lane 0 issues the tensor copies. Every lane copies sa for tokens
    // 2*lane, 2*lane + 1 of the group into the group's first slot with 4-byte
    // asynchronous copies, and arrives on the slot's barrier when they land
    // (the barrier counts 32 such arrivals and lane 0's expect-tx arrival).
    SmallWalk wp;
    wp.start(p);
    RingPos pr;
    int64_t ls = 0;
    bool ok = true;   // uniform across the warp (every wait is voted)
    for (int64_t it = 0; ok && it < iters; ++it, wp.next(p)) {
      const bool int4_group = wp.g < p.G - 1;
      for (int part = 0; ok && part < (int4_group ? 1 : 2); ++part) {
        const int s = pr.idx;
        ok = __all_sync(0xffffffffu, mbar_wait(&pempty[s], pr.phase ^ 1u, abort_flag));
        if (!ok) break;
        uint8_t *slot = pring + s * kPSlot;
        if (part == 0) {
          const float *src = p.sa + static_cast<int64_t>(wp.g) * p.M;
          const uint32_t dst = smem_addr(slot + kPackSaOff) + 8u * lane;
          if (2 * lane < p.M) cp_async_4(dst, src + 2 * lane);
          if (2 * lane + 1 < p.M) cp_async_4(dst + 4u, src + 2 * lane + 1);
        }
        cp_async_mbar_arrive_noinc(&pfull[s]);
        if (lane == 0) {
          if (int4_group) {
            mbar_arrive_expect_tx(&pfull[s], kInt4Bytes);
            if (p.qw4t != nullptr)   // the tile's 8 KB block of the tiled layout
              bulk_load(slot, p.qw4t + (static_cast<int64_t>(wp.n0 / BW) * (p.G - 1) + wp.g) *
                                           (BW * 64),
                        BW * 64u, &pfull[s]);
            else
              tma_load_2d(slot, &maps.w4, wp.g * 64, wp.n0, &pfull[s]);
            tma_load_2d(slot + kPackAOff, &maps.a4, wp.g * 64, 0, &pfull[s]);
          } else {
            mbar_arrive_expect_tx(&pfull[s], part == 0 ? kInt8Bytes0 : kInt8Bytes1);
            tma_load_2d(slot, &maps.w8, 0, wp.n0 + 64 * part, &pfull[s]);
            tma_load_2d(slot + kPackAOff, &maps.a8, 0, 32 * part, &pfull[s]);
          }
          if (part == 0) tma_load_2d(slot + kPackSwOff, &maps.sw, wp.n0, wp.g, &pfull[s]);
        }
        ++ls;
        pr.next(kNP);
      }
    }
    if (!ok && lane == 0) {
      fail();
      for (int64_t j = (ls > kNP ? ls - kNP : 0); j < ls; ++j)
        (void)mbar_wait(&pfull[j % kNP], static_cast<uint32_t>((j / kNP) & 1), nullptr);
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      int64_t last_mma = -1;
      int last_b = 0;
      uint32_t last_ph = 0;
      bool ok = true;
      RingPos ur, br;
      const uint64_t bias_adesc =
          smem_desc_k_noswizzle(smem_addr(smem + kBiasOff), kBiasLbo, kBiasSbo);
      const uint64_t bias_bdesc =
          smem_desc_k_noswizzle(smem_addr(smem + kBiasOff + kBiasA), kBiasLbo, kBiasSbo);
      SmallStep st;
      st.start(p);
      for (int64_t it = 0; ok && it < steps; ++it, ur.next(kUS), br.next(kBS), st.next(p)) {
        const int u = ur.idx, b = br.idx;
        if (!(mbar_try_wait(&ufull[u], ur.phase) & mbar_try_wait(&tempty[b], br.phase ^ 1u)) &&
            (!mbar_wait(&ufull[u], ur.phase, abort_flag) ||
             !mbar_wait(&tempty[b], br.phase ^ 1u, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        for (int j = 0; j < st.n; ++j) {
          const uint32_t op = smem_addr(uring + (2 * u + j) * kUSlot);
          const uint64_t adesc = smem_desc_k_sw128(op);             // weights, 128 rows
          const uint64_t bdesc = smem_desc_k_sw128(op + kOpAOff);   // tokens, NT rows
          const uint32_t d = tbase + (2 * b + j) * kMaxTokens;
          // the accumulator starts at the conversion bias (fp16 MMA of the constant tiles)
          mma_f16(d, bias_adesc, bias_bdesc, kIdescBias, 0u);
#pragma unroll
          for (int k = 0; k < 4; ++k) mma_i8(d, adesc + 2 * k, bdesc + 2 * k, kIdescSmall, 1u);
        }
        tc_commit(&tfull[b]);
        tc_commit(&uempty[u]);
        last_mma = it;
        last_b = b;
        last_ph = br.phase;
      }
      if (!ok) fail();
      // nothing may still write TMEM when it is released
      if (last_mma >= 0) (void)mbar_wait(&tfull[last_b], last_ph, nullptr);
    }
  } else {
    // ================================================================ unpackers
    const int lt = threadIdx.x - 64;
    SmallStep st;
    st.start(p);
    RingPos ur, sr, pr;
    for (int64_t it = 0; it < steps; ++it, ur.next(kUS), sr.next(kSS), st.next(p)) {
      const int u = ur.idx, sl = sr.idx;
      const int n = st.n;
      const bool int4_step = st.w.g < p.G - 1;
      const bool two = !int4_step || n == 2;   // the step takes two packed slots
      const RingPos p0 = pr;
      RingPos p1 = pr;
      p1.next(kNP);
      bool ok = mbar_try_wait(&uempty[u], ur.phase ^ 1u) &
                mbar_try_wait(&sempty[sl], sr.phase ^ 1u) & mbar_try_wait(&pfull[p0.idx], p0.phase);
      if (!ok)
        ok = mbar_wait(&uempty[u], ur.phase ^ 1u, abort_flag) &&
             mbar_wait(&sempty[sl], sr.phase ^ 1u, abort_flag) &&
             mbar_wait(&pfull[p0.idx], p0.phase, abort_flag);
      if (ok && two) ok = mbar_wait(&pfull[p1.idx], p1.phase, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) fail();
        break;
      }
      const uint8_t *pk0 = pring + p0.idx * kPSlot, *pk1 = pring + p1.idx * kPSlot;
      if (int4_step) {
        // nibbles -> bytes holding 16*q, K-major with the 128-byte swizzle;
        // group j of the step into operand slot 2u + j. Every shared-memory
        // load of the step goes out before the first store.
        constexpr int kCh = kPackedChunks / kUnpackThreads;
        uint4 v[2][kCh];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          if (j < n) {
#pragma unroll
            for (int i = 0; i < kCh; ++i) {
              const int c = lt + kUnpackThreads * i;
              const bool is_w = c < BW * 4;
              const int row = (is_w ? c : c - BW * 4) >> 2, cc = c & 3;
              v[j][i] = *reinterpret_cast<const uint4 *>((j ? pk1 : pk0) + (is_w ? 0u : kPackAOff) +
                                                          row * 64 + cc * 16);
            }
          }
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          if (j < n) {
            uint8_t *op = uring + (2 * u + j) * kUSlot;
#pragma unroll
            for (int i = 0; i < kCh; ++i) {
              const int c = lt + kUnpackThreads * i;
              const bool is_w = c < BW * 4;
              const int row = (is_w ? c : c - BW * 4) >> 2, cc = c & 3;
              const uint4 x = v[j][i];
              uint8_t *dst = op + (is_w ? 0u : kOpAOff) + row * 128;
              const uint4 lo = make_uint4((x.x << 4) & 0xF0F0F0F0u, (x.y << 4) & 0xF0F0F0F0u,
                                          (x.z << 4) & 0xF0F0F0F0u, (x.w << 4) & 0xF0F0F0F0u);
              const uint4 hi = make_uint4(x.x & 0xF0F0F0F0u, x.y & 0xF0F0F0F0u,
                                          x.z & 0xF0F0F0F0u, x.w & 0xF0F0F0F0u);
              const int swz = row & 7;
              *reinterpret_cast<uint4 *>(dst + (((2 * cc) ^ swz) << 4)) = lo;
              *reinterpret_cast<uint4 *>(dst + (((2 * cc + 1) ^ swz) << 4)) = hi;
            }
          }
        }
      } else {
        // the INT8 group arrived already swizzled, in halves: slot p0 holds W8
        // rows 0..63 and A8 rows 0..31, slot p1 the rest. 64 and 32 rows are
        // whole 1024-byte swizzle atoms, so the halves are copied byte for byte.
        uint8_t *op = uring + 2 * u * kUSlot;
#pragma unroll
        for (int i = 0; i < kInt8Chunks / kUnpackThreads; ++i) {
          const int c = lt + kUnpackThreads * i;
          const bool is_w = c < BW * 8;
          const int cw = is_w ? c : c - BW * 8;               // chunk within W8 (1024) or A8 (512)
          const int half_chunks = is_w ? BW * 4 : kMaxTokens * 4;
          const int h = cw >= half_chunks;
          const uint32_t off = (cw - h * half_chunks) * 16u;
          const uint8_t *src = (h ? pk1 : pk0) + (is_w ? 0u : kPackAOff) + off;
          uint8_t *dst = op + (is_w ? 0u : kOpAOff) + h * half_chunks * 16u + off;
          *reinterpret_cast<uint4 *>(dst) = *reinterpret_cast<const uint4 *>(src);
        }
      }
      // scales of group j into scale slot 2sl + j: sw of the tile's weight
      // rows, and per token pair (sa'[2k], sa'[2k+1], -C*sa'[2k],
      // -C*sa'[2k+1]) with sa' = sa (times 1/256 for an INT4 group) truncated
      // to 22 significant bits, the same fp32 steps as gemm.cuh's drain
      for (int j = 0; j < n; ++j) {
        const uint8_t *pk = j ? pk1 : pk0;
        uint8_t *ss = sring + (2 * sl + j) * kSSlot;
        if (lt < BW) {
          reinterpret_cast<float *>(ss + kSwOff)[lt] =
              reinterpret_cast<const float *>(pk + kPackSwOff)[lt];
        } else if (lt < BW + kMaxTokens / 2) {
          const int k = lt - BW;
          const float2 sa = reinterpret_cast<const float2 *>(pk + kPackSaOff)[k];
          float sv[2] = {sa.x, sa.y};
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            float x = sv[h];
            if (int4_step) x *= 0.00390625f;
            sv[h] = __uint_as_float(__float_as_uint(x) & 0xFFFFFFFCu);
          }
          reinterpret_cast<float4 *>(ss)[k] =
              make_float4(sv[0], sv[1], -gemm_cfg::kBiasF * sv[0], -gemm_cfg::kBiasF * sv[1]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&pempty[p0.idx]);
        if (two) mbar_arrive(&pempty[p1.idx]);
        mbar_arrive(&sfull[sl]);
        mbar_arrive(&ufull[u]);
      }
      pr = p1;
      if (two) pr.next(kNP);
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tbase, kTmemCols);
  }
  if (p.splits > 1) {
    // cluster of the tile's K ranges (rank = K range): sum the partial tiles
    // in range order, a slice of the weight rows per CTA
    cluster_sync();
    const int S = p.splits;
    const int rank = static_cast<int>(cluster_cta_rank());
    const int n0 = (static_cast<int>(blockIdx.x) / S) * BW;
    // this CTA's slice: weight-row quads [qlo, qlo + nq) of the tile's BW/4
    const int qlo = rank * (BW / 4) / S, nq = (rank + 1) * (BW / 4) / S - qlo;
    const int lo = 4 * qlo;
    const float *part = reinterpret_cast<const float *>(uring);
    // one thread per token and quad of weight rows: a 16-byte load from each
    // K range's tile (all issued before the first add), the ranges added in
    // order, one 8-byte store of 4 fp16 values (rows and N are multiples of 4)
    const int total = p.M * nq;
    for (int e = threadIdx.x; e < total; e += threads_for(NT)) {
      const int m = e / nq, row = lo + 4 * (e - m * nq);
      const float *src = part + m * BW + row;
      float4 v[kMaxSplits];
#pragma unroll
      for (int r = 0; r < kMaxSplits; ++r)
        if (r < S) v[r] = ld_shared_cluster_v4(cluster_map(src, r));
      float4 a = v[0];
#pragma unroll
      for (int r = 1; r < kMaxSplits; ++r) {
        if (r < S) {
          a.x += v[r].x;
          a.y += v[r].y;
          a.z += v[r].z;
          a.w += v[r].w;
        }
      }
      __half *dst = p.y + static_cast<int64_t>(m) * p.N + n0 + row;
      const __half2 h01 = __floats2half2_rn(a.x, a.y), h23 = __floats2half2_rn(a.z, a.w);
      if (n0 + row + 3 < p.N) {
        *reinterpret_cast<uint2 *>(dst) = make_uint2(*reinterpret_cast<const uint32_t *>(&h01),
                                                     *reinterpret_cast<const uint32_t *>(&h23));
      } else {
        const float f[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (n0 + row + c < p.N) dst[c] = __float2half_rn(f[c]);
      }
    }
    cluster_sync();   // no CTA leaves while a peer may still read its tile
  }
}

}  // namespace atomk
