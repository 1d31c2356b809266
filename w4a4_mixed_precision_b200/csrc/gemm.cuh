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
// 4-bit integer MMA, so this kernel runs both the INT4 groups and the INT8
// outlier group on tcgen05.mma kind::i8.
//
// One CTA per SM, persistent over 128x256 output tiles (m fastest, so the
// CTAs in flight share one weight tile column and all of A stays in L2).
// Per tile, one pipeline step per 128-wide K group:
//
//   loader warps 1..7  LDG the packed INT4 group (A 128x64 B, W 256x64 B) one
//                      group ahead into registers, expand each nibble to a byte
//                      holding 16*q (x & 0xF0 / x << 4), store K-major with the
//                      128-byte swizzle, plus the group's sa/sw scales. For the
//                      INT8 outlier group one thread issues two TMA tile loads
//                      (128x128 and 256x128 bytes, 128-byte swizzle) instead.
//   MMA warp 0         4 x tcgen05.mma kind::i8 (M=128, N=256, K=32) into one of
//                      two TMEM accumulators (2 x 256 int32 columns), then
//                      commits to the stage's "empty" and the accumulator's
//                      "full" mbarriers.
//   drain warps 8..15  tcgen05.ld the int32 partials (8 columns at a time,
//                      double-buffered), release the accumulator, convert
//                      exactly (int + 0x4B400000 reinterpreted, minus 1.5*2^23)
//                      and accumulate sa*sw*P in fp32 registers with packed
//                      f32x2 math. After the last group: fp16 store of the tile.
//
// Nibbles are expanded as 16*q so no sign extension is needed: INT4 partials
// come out as exactly 256*P (|256*P| <= 256*128*64 < 2^22), and the factor
// 1/256 is folded into sa. Both operands use the same expansion order inside a
// group (low nibbles of a 16-byte chunk, then high nibbles), which only
// permutes the K positions of a group identically for A and W, so every
// per-group dot product is unchanged.
#pragma once

#include "ptx.cuh"

namespace atomk {

namespace gemm_cfg {
constexpr int BM = 128;
constexpr int BN = 256;
constexpr int kStages = 4;
constexpr int kThreads = 512;
constexpr int kLoaderThreads = 224;  // warps 1..7
constexpr uint32_t kABytes = BM * 128;
constexpr uint32_t kBBytes = BN * 128;
constexpr uint32_t kSaOff = kABytes + kBBytes;
constexpr uint32_t kSwOff = kSaOff + BM * 4;
constexpr uint32_t kStageBytes = 50u * 1024u;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kBarBytes = 1024;
constexpr uint32_t kSmemBytes = kBarBytes + kStages * kStageBytes + 1024;  // + alignment slack
constexpr int kPackedChunks = (BM + BN) * 4;                                   // 16-B chunks / group
constexpr int kChunksPerThread = (kPackedChunks + kLoaderThreads - 1) / kLoaderThreads;
constexpr uint32_t kIdesc = idesc_i8(BM, BN);
constexpr int kLoaderRegs = 104;
constexpr int kDrainRegs = 152;
static_assert(kSwOff + BN * 4 <= kStageBytes, "stage overflow");
static_assert(kStageBytes % 1024 == 0, "stages must keep 1024-byte alignment");
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
  int m_tiles, n_tiles, tiles;
};

__device__ __forceinline__ uint4 ldg_stream_v4(const void *p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p));
  return v;
}

// Predicated 16-byte global store. Keeping the predicate inside the
// instruction (rather than branching around the store) keeps the epilogue one
// basic block, which is what lets the 128 live accumulators stay in registers.
__device__ __forceinline__ void st_global_v4_if(void *p, uint32_t a, uint32_t b, uint32_t c,
                                                uint32_t d, bool pred) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %5, 0;\n\t"
      "@q st.global.v4.b32 [%0], {%1, %2, %3, %4};\n\t}" ::"l"(p),
      "r"(a), "r"(b), "r"(c), "r"(d), "r"(static_cast<uint32_t>(pred))
      : "memory");
}

// Walks this CTA's (tile, group) sequence.
struct TileWalk {
  int tile, g, m0, n0;
  __device__ __forceinline__ void start(const GemmParams &p) {
    tile = blockIdx.x;
    g = 0;
    set(p);
  }
  __device__ __forceinline__ void set(const GemmParams &p) {
    m0 = (tile % p.m_tiles) * gemm_cfg::BM;
    n0 = (tile / p.m_tiles) * gemm_cfg::BN;
  }
  __device__ __forceinline__ void next(const GemmParams &p) {
    if (++g == p.G) {
      g = 0;
      tile += gridDim.x;
      set(p);
    }
  }
};

__device__ __forceinline__ int64_t local_iterations(const GemmParams &p) {
  const int my_tiles =
      (p.tiles > static_cast<int>(blockIdx.x))
          ? (p.tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                static_cast<int>(gridDim.x)
          : 0;
  return static_cast<int64_t>(my_tiles) * p.G;
}

// ------------------------------------------------------------------ loader role

struct LoaderRegs {
  uint4 chunk[gemm_cfg::kChunksPerThread];
  float sc[3];
};

__device__ __forceinline__ void loader_fetch(const GemmParams &p, const TileWalk &w, int lt,
                                             LoaderRegs &r) {
  using namespace gemm_cfg;
  const int64_t row_bytes = (p.K - 128) / 2;
  if (w.g < p.G - 1) {
#pragma unroll
    for (int i = 0; i < kChunksPerThread; ++i) {
      const int c = lt + kLoaderThreads * i;
      r.chunk[i] = make_uint4(0u, 0u, 0u, 0u);
      if (c < kPackedChunks) {
        const bool is_a = c < BM * 4;
        const int cc = c & 3;
        const int row = (is_a ? c : c - BM * 4) >> 2;
        const int grow = (is_a ? w.m0 : w.n0) + row;
        if (grow < (is_a ? p.M : p.N)) {
          const uint8_t *src = (is_a ? p.qa4 : p.qw4) + grow * row_bytes + w.g * 64 + cc * 16;
          r.chunk[i] = ldg_stream_v4(src);
        }
      }
    }
  }
  if (lt < BM) {
    const int m = w.m0 + lt;
    r.sc[0] = (m < p.M) ? __ldg(p.sa + static_cast<int64_t>(w.g) * p.M + m) : 0.f;
  } else {
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      const int j = lt - BM + 96 * k;
      const int n = w.n0 + j;
      r.sc[k] = (j < BN && n < p.N) ? __ldg(p.sw + static_cast<int64_t>(w.g) * p.N + n) : 0.f;
    }
  }
}

__device__ __forceinline__ void loader_store(const GemmParams &p, const TileWalk &w, int lt,
                                             const LoaderRegs &r, uint8_t *stage) {
  using namespace gemm_cfg;
  if (w.g < p.G - 1) {
#pragma unroll
    for (int i = 0; i < kChunksPerThread; ++i) {
      const int c = lt + kLoaderThreads * i;
      if (c < kPackedChunks) {
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
    }
  }
  float *sa_s = reinterpret_cast<float *>(stage + kSaOff);
  float *sw_s = reinterpret_cast<float *>(stage + kSwOff);
  if (lt < BM) {
    sa_s[lt] = r.sc[0];
  } else {
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      const int j = lt - BM + 96 * k;
      if (j < BN) sw_s[j] = r.sc[k];
    }
  }
}

// ------------------------------------------------------------------ drain helpers

// acc[0..3] += sa * sw[0..7] * P[0..7] for one 8-column chunk of this thread's row.
__device__ __forceinline__ void drain_chunk(const uint32_t (&r)[8], const float *sw_chunk,
                                            float2 sa2, float2 *acc) {
  const float2 neg = make_float2(-12582912.f, -12582912.f);
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const float4 s4 = *reinterpret_cast<const float4 *>(sw_chunk + 4 * q);
    // exact int -> float for |P| < 2^22: the bits of 1.5*2^23 + P, minus 1.5*2^23
    float2 p0 = make_float2(__uint_as_float(r[4 * q + 0] + 0x4B400000u),
                            __uint_as_float(r[4 * q + 1] + 0x4B400000u));
    float2 p1 = make_float2(__uint_as_float(r[4 * q + 2] + 0x4B400000u),
                            __uint_as_float(r[4 * q + 3] + 0x4B400000u));
    p0 = f2_add(p0, neg);
    p1 = f2_add(p1, neg);
    const float2 s0 = f2_mul(sa2, make_float2(s4.x, s4.y));
    const float2 s1 = f2_mul(sa2, make_float2(s4.z, s4.w));
    acc[2 * q] = f2_fma(p0, s0, acc[2 * q]);
    acc[2 * q + 1] = f2_fma(p1, s1, acc[2 * q + 1]);
  }
}

__device__ __forceinline__ void store_partials_chunk(const GemmParams &p, const uint32_t (&r)[8],
                                                     int m, int n, int g) {
  if (m >= p.M || n >= p.N) return;  // N % 8 == 0: a chunk is wholly in or out
  const bool int4_group = g < p.G - 1;
  int32_t v[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int32_t x = static_cast<int32_t>(r[j]);
    v[j] = int4_group ? (x >> 8) : x;   // INT4 groups hold exactly 256*P
  }
  int32_t *dst = p.partials + (static_cast<int64_t>(g) * p.M + m) * p.N + n;
  *reinterpret_cast<int4 *>(dst) = make_int4(v[0], v[1], v[2], v[3]);
  *reinterpret_cast<int4 *>(dst + 4) = make_int4(v[4], v[5], v[6], v[7]);
}

// ------------------------------------------------------------------ kernel

template <bool kPartials>
__global__ void __launch_bounds__(gemm_cfg::kThreads, 1)
w4a4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a8,
                 const __grid_constant__ CUtensorMap tmap_w8, const GemmParams p) {
  using namespace gemm_cfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);

  uint64_t *full = reinterpret_cast<uint64_t *>(smem);  // [kStages]  loaders -> MMA
  uint64_t *empty = full + kStages;                      // [kStages]  MMA + drain -> loaders
  uint64_t *tfull = empty + kStages;                     // [2]        MMA -> drain
  uint64_t *tempty = tfull + 2;                          // [2]        drain -> MMA
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  uint8_t *stages = smem + kBarBytes;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 7);       // one arrival per loader warp
      mbar_init(&empty[s], 1 + 8);  // MMA commit + one arrival per drain warp
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 8);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tbase = *tmem_slot;
  const int64_t iters = local_iterations(p);

  auto fail = [&](void) {
    report_status(6 /* ATOM_ERR_TIMEOUT */);
    *abort_flag = 1;
  };

  if (warp >= 8) {
    // ================================================================ drain
    regs_increase<kDrainRegs>();
    const int q = warp & 3;           // TMEM lane quarter this warp may access
    const int h = (warp - 8) >> 2;    // which 128-column half of the tile
    const int row = 32 * q + lane;
    float2 acc[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) acc[i] = make_float2(0.f, 0.f);
    TileWalk w;
    w.start(p);
    for (int64_t it = 0; it < iters; ++it, w.next(p)) {
      const int s = static_cast<int>(it % kStages), b = static_cast<int>(it & 1);
      if (!mbar_wait(&tfull[b], static_cast<uint32_t>((it >> 1) & 1), abort_flag) ||
          !mbar_wait(&full[s], static_cast<uint32_t>((it / kStages) & 1), abort_flag)) {
        fail();
        break;
      }
      tc_fence_after_sync();
      const uint8_t *stage = stages + s * kStageBytes;
      float sa_v = reinterpret_cast<const float *>(stage + kSaOff)[row];
      if (w.g < p.G - 1) sa_v *= 0.00390625f;  // INT4 partials are 256*P
      const float2 sa2 = make_float2(sa_v, sa_v);
      const float *sw_s = reinterpret_cast<const float *>(stage + kSwOff) + h * 128;
      const uint32_t taddr = tbase + (static_cast<uint32_t>(32 * q) << 16) + b * BN + h * 128;
      const int m = w.m0 + row;
      uint32_t ra[8], rb[8];
      tmem_ld_x8(taddr, ra);
      tmem_ld_wait(ra);
#pragma unroll
      for (int c = 0; c < 16; c += 2) {
        tmem_ld_x8(taddr + 8 * (c + 1), rb);
        drain_chunk(ra, sw_s + 8 * c, sa2, acc + 4 * c);
        if (kPartials) store_partials_chunk(p, ra, m, w.n0 + h * 128 + 8 * c, w.g);
        tmem_ld_wait(rb);
        if (c + 2 < 16) {
          tmem_ld_x8(taddr + 8 * (c + 2), ra);
        } else {
          // every column of this accumulator is in registers: hand it back
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[b]);
        }
        drain_chunk(rb, sw_s + 8 * (c + 1), sa2, acc + 4 * (c + 1));
        if (kPartials) store_partials_chunk(p, rb, m, w.n0 + h * 128 + 8 * (c + 1), w.g);
        if (c + 2 < 16) tmem_ld_wait(ra);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);

      if (w.g == p.G - 1) {
        // epilogue: fp16 row segment of 128 columns
        {
          const bool row_ok = p.y != nullptr && m < p.M;
          __half *dst = p.y + static_cast<int64_t>(row_ok ? m : 0) * p.N + w.n0 + h * 128;
#pragma unroll
          for (int c8 = 0; c8 < 16; ++c8)
            st_global_v4_if(dst + 8 * c8, pack_half2_rn(acc[4 * c8 + 0].x, acc[4 * c8 + 0].y),
                            pack_half2_rn(acc[4 * c8 + 1].x, acc[4 * c8 + 1].y),
                            pack_half2_rn(acc[4 * c8 + 2].x, acc[4 * c8 + 2].y),
                            pack_half2_rn(acc[4 * c8 + 3].x, acc[4 * c8 + 3].y),
                            row_ok && (w.n0 + h * 128 + 8 * c8 < p.N));
        }
#pragma unroll
        for (int i = 0; i < 64; ++i) acc[i] = make_float2(0.f, 0.f);
      }
    }
  } else {
    regs_decrease<kLoaderRegs>();
    if (warp == 0) {
      // ============================================================== MMA issuer
      if (lane == 0) {
        int64_t last = -1;
        for (int64_t it = 0; it < iters; ++it) {
          const int s = static_cast<int>(it % kStages), b = static_cast<int>(it & 1);
          if (!mbar_wait(&full[s], static_cast<uint32_t>((it / kStages) & 1), abort_flag) ||
              !mbar_wait(&tempty[b], static_cast<uint32_t>(((it >> 1) & 1) ^ 1), abort_flag)) {
            fail();
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_addr = smem_addr(stages + s * kStageBytes);
          const uint64_t adesc = smem_desc_k_sw128(a_addr);
          const uint64_t bdesc = smem_desc_k_sw128(a_addr + kABytes);
          const uint32_t d = tbase + b * BN;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_i8(d, adesc + 2 * k, bdesc + 2 * k, kIdesc, k > 0 ? 1u : 0u);
          tc_commit(&empty[s]);
          tc_commit(&tfull[b]);
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
      LoaderRegs cur, nxt;
      if (iters > 0) loader_fetch(p, w, lt, cur);
      int64_t last_tma = -1;
      for (int64_t it = 0; it < iters; ++it) {
        const int s = static_cast<int>(it % kStages);
        TileWalk wn = w;
        wn.next(p);
        if (it + 1 < iters) loader_fetch(p, wn, lt, nxt);
        if (!mbar_wait(&empty[s], static_cast<uint32_t>(((it / kStages) & 1) ^ 1), abort_flag)) {
          fail();
          break;
        }
        uint8_t *stage = stages + s * kStageBytes;
        loader_store(p, w, lt, cur, stage);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (w.g == p.G - 1 && lwarp == 0) {
            mbar_arrive_expect_tx(&full[s], kABytes + kBBytes);
            tma_load_2d(stage, &tmap_a8, 0, w.m0, &full[s]);
            tma_load_2d(stage + kABytes, &tmap_w8, 0, w.n0, &full[s]);
            last_tma = it;
          } else {
            mbar_arrive(&full[s]);
          }
        }
        cur = nxt;
        w = wn;
      }
      if (*abort_flag && lane == 0 && lwarp == 0 && last_tma >= 0)
        (void)mbar_wait(&full[last_tma % kStages],
                        static_cast<uint32_t>((last_tma / kStages) & 1), nullptr);
    }
  }

  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tbase, kTmemCols);
  }
}

}  // namespace atomk
