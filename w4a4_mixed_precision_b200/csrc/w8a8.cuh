// w8a8.cuh -- INT8 x INT8 GEMM with per-row activation scales and
// per-column weight scales (the W8A8 comparator of the W4A4 path):
//
//   Y[m, n] = fp16( float(P[m, n]) * (sa[m] * sw[n]) ),  P = sum_k qa[m, k] * qw[n, k]
//
// with P the exact int32 dot product over all of K (no groups). A per-tensor
// scale is the special case of constant sa and sw.
//
// Method context: "Atom: Low-bit Quantization for Efficient and Accurate LLM
// Serving" compares its W4A4 kernels against 8-bit weight-and-activation
// serving; this kernel is that baseline built on the same Blackwell pieces as
// the W4A4 GEMM, so the two can be measured side by side.
//
// Structure. A cluster of two CTAs owns a 256x256 output tile per step of a
// persistent loop over tiles (m fastest). Each 128-byte step of K is one TMA
// box of A (128 rows) and one of W (128 rows) per CTA, 128-byte swizzled,
// K-major, landing directly in the MMA operand layout, and four 2-SM MMAs
// (tcgen05.mma.cta_group::2.kind::i8, M=256, N=256, K=32) accumulate it into a
// 256-column TMEM accumulator; the first MMA of a tile overwrites it. Two
// accumulators alternate between tiles, so the epilogue of one tile overlaps
// the mainloop of the next.
//
// Roles in each CTA:
//   warp 0, lane 0   TMA producer for both operands into the stage ring.
//   warp 1, lane 0   leader CTA: the MMA issuer; peer CTA: relays "stage
//                    landed" to the leader (the MMA reads both CTAs' stages).
//   warps 4..11      epilogue: warp 4 + 4*hh + q reads TMEM lanes [32q, 32q+32)
//                    (its hardware lane quarter), columns [128hh, 128hh+128),
//                    frees the accumulator once all its loads have landed,
//                    scales, converts to fp16 and writes 32x64 boxes through
//                    shared memory with TMA tensor stores.
#pragma once

#include "ptx.cuh"

namespace atomk {

namespace w8a8_cfg {
constexpr int BM = 128;            // A rows per CTA (256 per pair)
constexpr int BN = 256;            // output columns per pair tile
constexpr int BW = 128;            // W rows per CTA
constexpr int kPairM = 2 * BM;
constexpr int kThreads = 384;      // 12 warps
constexpr int kStages = 5;
constexpr uint32_t kABytes = BM * 128;
constexpr uint32_t kBBytes = BW * 128;
constexpr uint32_t kStage = kABytes + kBBytes;
constexpr uint32_t kBarBytes = 1024;
constexpr uint32_t kSOff = kBarBytes;                       // stage ring
constexpr uint32_t kYSlot = 32 * 128;                        // one 32 x 64 fp16 box
constexpr uint32_t kYOff = kSOff + kStages * kStage;         // 8 epilogue boxes
constexpr uint32_t kSmemBytes = kYOff + 8 * kYSlot + 1024;   // + alignment slack
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kIdesc = idesc_i8(kPairM, BN);
static_assert(kStage % 1024 == 0 && kYOff % 1024 == 0, "1024-byte alignment of the rings");
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
}  // namespace w8a8_cfg

struct W8A8Maps {
  CUtensorMap a;   // int8 A [M][K], boxes of 128 rows x 128 bytes, 128-byte swizzle
  CUtensorMap w;   // int8 W [N][K], boxes of 128 rows x 128 bytes, 128-byte swizzle
  CUtensorMap y;   // fp16 Y [M][N], boxes of 32 rows x 64 columns, 128-byte swizzle (stores)
};

struct W8A8Params {
  const float *sa;   // [M]
  const float *sw;   // [N]
  int M, N, K;
  int ksteps;        // ceil(K / 128)
  int m_tiles, tiles;
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(w8a8_cfg::kThreads, 1)
w8a8_gemm_kernel(const __grid_constant__ W8A8Maps maps, const W8A8Params p) {
  using namespace w8a8_cfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);

  uint64_t *full = reinterpret_cast<uint64_t *>(smem);   // [kStages] local TMA landed
  uint64_t *mfull = full + kStages;                       // [kStages] leader: peer's landed
  uint64_t *empty = mfull + kStages;                      // [kStages] MMA commit -> producers
  uint64_t *tfull = empty + kStages;                      // [2] accumulator complete
  uint64_t *tempty = tfull + 2;                           // [2] leader: accumulator read
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  uint8_t *stages = smem + kSOff;
  uint8_t *ystage = smem + kYOff;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = static_cast<int>(cluster_cta_rank());
  const int pair = static_cast<int>(blockIdx.x >> 1), pairs = static_cast<int>(gridDim.x >> 1);
  const int my_tiles = p.tiles > pair ? (p.tiles - pair + pairs - 1) / pairs : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);    // producer's expect_tx arrival (+ TMA bytes)
      mbar_init(&mfull[s], 1);   // the peer's relay
      mbar_init(&empty[s], 1);   // the MMA commit
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 16);   // lane 0 of each of the 8 epilogue warps in each CTA
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

  auto fail = [&](void) {
    report_status(6 /* ATOM_ERR_TIMEOUT */);
    *abort_flag = 1;
  };

  if (warp == 0) {
    // ================================================================ producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int64_t issued = 0;
      bool ok = true;
      for (int t = 0; ok && t < my_tiles; ++t) {
        const int tile = pair + t * pairs;
        const int m0 = (tile % p.m_tiles) * kPairM, n0 = (tile / p.m_tiles) * BN;
        for (int ks = 0; ks < p.ksteps; ++ks) {
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t *st = stages + s * kStage;
          mbar_arrive_expect_tx(&full[s], kStage);
          tma_load_2d(st, &maps.a, ks * 128, m0 + BM * rank, &full[s]);
          tma_load_2d(st + kABytes, &maps.w, ks * 128, n0 + BW * rank, &full[s]);
          ++issued;
          if (++s == kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {
        fail();
        // let the tensor copies still in flight land before shared memory is released
        for (int64_t j = (issued > kStages ? issued - kStages : 0); j < issued; ++j)
          (void)mbar_wait(&full[j % kStages], static_cast<uint32_t>((j / kStages) & 1), nullptr);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank != 0) {
      // ============================================================ relay (peer)
      const uint32_t mfull_leader = cluster_map(&mfull[0], 0);
      int s = 0;
      uint32_t ph = 0;
      const int64_t steps = static_cast<int64_t>(my_tiles) * p.ksteps;
      for (int64_t i = 0; i < steps; ++i) {
        if (!mbar_wait(&full[s], ph, abort_flag)) {
          fail();
          break;
        }
        mbar_arrive_remote(mfull_leader + 8u * s);
        if (++s == kStages) {
          s = 0;
          ph ^= 1u;
        }
      }
    } else if (lane == 0) {
      // ============================================================ MMA issuer (leader)
      int s = 0;
      uint32_t ph = 0;
      int last_tile = -1;
      bool ok = true;
      for (int t = 0; ok && t < my_tiles; ++t) {
        const int b = t & 1;
        if (!mbar_wait(&tempty[b], static_cast<uint32_t>(((t >> 1) & 1) ^ 1), abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t d = tbase + b * BN;
        for (int ks = 0; ks < p.ksteps; ++ks) {
          if (!mbar_wait(&full[s], ph, abort_flag) || !mbar_wait(&mfull[s], ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_addr = smem_addr(stages + s * kStage);
          const uint64_t adesc = smem_desc_k_sw128(a_addr);
          const uint64_t bdesc = smem_desc_k_sw128(a_addr + kABytes);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_i8_pair(d, adesc + 2 * k, bdesc + 2 * k, kIdesc, (ks | k) != 0 ? 1u : 0u);
          tc_commit_pair_multicast(&empty[s], 0x3);
          if (++s == kStages) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair_multicast(&tfull[b], 0x3);
        last_tile = t;
      }
      if (!ok) fail();
      // nothing may still write TMEM when it is released
      if (last_tile >= 0)
        (void)mbar_wait(&tfull[last_tile & 1], static_cast<uint32_t>((last_tile >> 1) & 1),
                        nullptr);
    }
  } else if (warp >= 4) {
    // ================================================================ epilogue
    const int ew = warp - 4;           // 0..7
    const int q = ew & 3;              // TMEM lane quarter (= warp % 4)
    const int hh = ew >> 2;            // column half
    const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
    const uint32_t tempty_leader = cluster_map(&tempty[0], 0);
    uint8_t *ybuf = ystage + ew * kYSlot;
    for (int t = 0; t < my_tiles; ++t) {
      const int tile = pair + t * pairs;
      const int m0 = (tile % p.m_tiles) * kPairM, n0 = (tile / p.m_tiles) * BN;
      const int b = t & 1;
      const bool ok = mbar_wait(&tfull[b], static_cast<uint32_t>((t >> 1) & 1), abort_flag);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) fail();
        break;
      }
      tc_fence_after_sync();
      const int row0 = m0 + BM * rank + 32 * q;   // this warp's first output row
      const int row = row0 + lane;
      const float sa = row < p.M ? __ldg(p.sa + row) : 0.f;
      const uint32_t tcol = tbase + lane_base + b * BN + hh * 128;
#pragma unroll
      for (int piece = 0; piece < 2; ++piece) {
        // 64 accumulator columns of this thread's row
        uint32_t r[4][16];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld_x16(tcol + 64 * piece + 16 * c, r[c]);
        // one wait retires all four loads; each call threads one load's
        // registers through it so that none of their uses moves above it
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld_wait(r[c]);
        if (piece == 1) {
          // every column of this warp's lanes is in registers: hand the
          // accumulator back for the next tile's MMAs
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) {
            if (rank == 0)
              mbar_arrive(&tempty[b]);
            else
              mbar_arrive_cluster_relaxed(tempty_leader + 8u * b);
          }
        }
        if (lane == 0) bulk_wait_group_read0();   // the previous box has left the buffer
        __syncwarp();
        const int col0 = n0 + 128 * hh + 64 * piece;
#pragma unroll
        for (int j = 0; j < 8; ++j) {   // 8 columns per 16-byte chunk of the box row
          const int col = col0 + 8 * j;
          float4 s0 = make_float4(0.f, 0.f, 0.f, 0.f), s1 = s0;
          if (col < p.N) {   // N % 8 == 0: the 8 columns are all inside or all outside
            s0 = __ldg(reinterpret_cast<const float4 *>(p.sw + col));
            s1 = __ldg(reinterpret_cast<const float4 *>(p.sw + col) + 1);
          }
          const uint32_t *v = &r[j >> 1][8 * (j & 1)];
          const float sc[8] = {sa * s0.x, sa * s0.y, sa * s0.z, sa * s0.w,
                               sa * s1.x, sa * s1.y, sa * s1.z, sa * s1.w};
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            f[e] = __int2float_rn(static_cast<int32_t>(v[e])) * sc[e];
          st_shared_v4(ybuf + lane * 128 + ((j ^ (lane & 7)) << 4), pack_half2_rn(f[0], f[1]),
                       pack_half2_rn(f[2], f[3]), pack_half2_rn(f[4], f[5]),
                       pack_half2_rn(f[6], f[7]));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && row0 < p.M && col0 < p.N) {
          tma_store_2d(&maps.y, ybuf, col0, row0);
          bulk_commit_group();
        }
      }
    }
    // the Y boxes must be out of shared memory before the CTA exits
    if (lane == 0) bulk_wait_group0();
  }

  tc_fence_before_sync();
  __syncthreads();
  cluster_sync();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc_pair(tbase, kTmemCols);
  }
}

}  // namespace atomk
