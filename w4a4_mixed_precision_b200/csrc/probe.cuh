// probe.cuh -- a tensor-core-only loop that measures the dense INT8 MMA
// throughput of the GPU it runs on, under the clocks it runs at. It is the
// second roofline denominator of the W4A4 GEMM (the first is the measured bf16
// GEMM rate times the nominal int8:bf16 ratio), not part of the hot path.
//
// Each CTA pair issues `groups` groups of four 2-SM MMAs of the GEMM's own
// shape (tcgen05.mma.cta_group::2.kind::i8, M = 256, N = 256, K = 32, operands
// K-major with the 128-byte swizzle in shared memory), alternating between two
// 256-column TMEM accumulators, with no loads, no unpack and no drain. The
// operand tiles are zero-filled once. One commit at the end tells both CTAs
// that the last MMA has completed.
#pragma once

#include "ptx.cuh"

namespace atomk {

namespace probe_cfg {
constexpr int kThreads = 128;
constexpr uint32_t kOpBytes = 128 * 128;            // one 128-row x 128-byte operand tile
// Far more shared memory than the tiles need, so that one CTA (and one TMEM
// allocation) fits per SM: pairs never compete for an SM's tensor memory.
constexpr uint32_t kSmemBytes = 160 * 1024;
static_assert(1024 + 2 * kOpBytes + 1024 <= kSmemBytes, "probe tiles");
constexpr uint32_t kIdesc = idesc_i8(256, 256);
}  // namespace probe_cfg

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(probe_cfg::kThreads, 1)
mma_i8_probe_kernel(int64_t groups) {
  using namespace probe_cfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  uint64_t *done = reinterpret_cast<uint64_t *>(smem);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
  uint8_t *ops = smem + 1024;
  const int warp = threadIdx.x >> 5;
  const int rank = static_cast<int>(cluster_cta_rank());

  for (uint32_t i = threadIdx.x; i < 2 * kOpBytes / 16; i += kThreads)
    reinterpret_cast<uint4 *>(ops)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    mbar_init(done, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before_sync();
  cluster_sync();
  tc_fence_after_sync();
  const uint32_t tbase = *tmem_slot;

  if (threadIdx.x == 32 && rank == 0 && groups > 0) {
    const uint64_t adesc = smem_desc_k_sw128(smem_addr(ops));
    const uint64_t bdesc = smem_desc_k_sw128(smem_addr(ops + kOpBytes));
    for (int64_t g = 0; g < groups; ++g) {
      const uint32_t d = tbase + static_cast<uint32_t>(g & 1) * 256u;
#pragma unroll
      for (int k = 0; k < 4; ++k) mma_i8_pair(d, adesc + 2 * k, bdesc + 2 * k, kIdesc, 1u);
    }
    tc_commit_pair_multicast(done, 0x3);
  }
  if (threadIdx.x == 0 && groups > 0 && !mbar_wait(done, 0, nullptr))
    report_status(6 /* ATOM_ERR_TIMEOUT */);
  tc_fence_before_sync();
  __syncthreads();
  cluster_sync();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc_pair(tbase, 512);
  }
}

}  // namespace atomk
