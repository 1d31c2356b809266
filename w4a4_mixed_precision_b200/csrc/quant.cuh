// quant.cuh -- fused outlier reorder + per-token per-128-group INT4/INT8
// quantization (one streaming pass over the fp16 rows).
//
// Method: "Atom: Low-bit Quantization for Efficient and Accurate LLM Serving"
// (paper summary: activations get a dedicated outlier path) and the record
// "Atom (mixed-precision block-outlier low-bit quantization for serving)"
// (fields "Weight group size" = 128 and "notes": every contiguous run of 128
// elements is one group quantized independently; 128 high-precision channels).
//
// Design (HBM-bound, so the aim is to keep HBM busy with few instructions per
// element):
//  * one CTA per SM, persistent. It runs up to three crews, each of 8
//    quantizing warps and one copy-issuing warp with its own ring of 2-4 stage
//    slots: the copy warp takes the next row of the whole launch from a row
//    counter in global memory whenever a slot of its ring is free, tags the
//    slot with the row, and brings the whole fp16 row in with one bulk copy
//    (TMA engine, mbarrier completion); each quantizing warp frees a slot
//    through its own arrival on an "empty" mbarrier. A crew or an SM that runs
//    faster thus takes more rows, and all end together: with fixed rows per
//    SM, the same few SMs ended each launch 10-15 us (a quarter of a launch)
//    after the rest. The copy warp keeps one row claimed ahead, so the
//    counter's round trip is off the refill path;
//  * the row counter is one of kQuantSlots slots that the host hands out in
//    turn, one per call; the last CTA of a launch to finish puts its slot back
//    to zero, so the slot is ready for its next call, or for the next replay
//    of a captured launch;
//  * launched with programmatic stream serialization: the barrier set-up and
//    the scale table are built while the previous kernel in the stream
//    finishes; the outlier list, the rows and the outputs are touched only
//    after griddepcontrol.wait;
//  * at start-up each CTA (once per SM, shared by its crews) turns the outlier
//    list into a gather table in shared
//    memory (uint16 [K]): for every group and lane, the byte offsets inside a
//    staged row of the 16 channels that lane quantizes, in the lane's gather
//    order. Reordered position p holds the p-th non-outlier channel for
//    p < K-128 and outlier_idx[p-(K-128)] after that (bitmap of the outliers,
//    block scan of the non-outlier counts);
//  * 8 lanes quantize one group (16 elements per lane), 4 groups per warp per
//    pass: two conflict-free 16-byte table loads, 16 gathered halves, amax by
//    shuffles over the 8 lanes; scale and inv of an INT4 group from a
//    1024-entry table of IEEE quotients by the significand of amax (see
//    kDivTable), of the INT8 group by one IEEE division each; code
//    bits from the low byte of fp32(1.5*2^23 + x*inv) (round half to even,
//    exact for |t| < 2^22), byte permutes to
//    pack, one 8-byte (INT4) or 16-byte (INT8) store per lane;
//  * a dense-group lane gathers its 16 elements rotated by an even amount that
//    depends on its position, so the 32 lanes of a warp read 32 distinct
//    shared-memory banks; the packed 8 bytes are rotated back with two byte
//    permutes.
#pragma once

#include "ptx.cuh"

namespace atomk {

constexpr int kQuantWarps = 8;                            // quantizing warps per crew
constexpr int kQuantCrews = 3;                            // crews per CTA, + 1 copy warp each
constexpr int kQuantThreads = 32 * kQuantCrews * (kQuantWarps + 1);
constexpr int kQuantMaxStages = 12;
// Header of the dynamic shared memory (byte offsets).
constexpr uint32_t kQHdrFull = 0;                            // uint64 [kQuantMaxStages]
constexpr uint32_t kQHdrEmpty = kQHdrFull + 8 * kQuantMaxStages;
constexpr uint32_t kQHdrFlags = kQHdrEmpty + 8 * kQuantMaxStages;  // int [2]: bad list, abort
constexpr uint32_t kQHdrTags = kQHdrFlags + 8;               // int64 [kQuantMaxStages]: row of each slot
constexpr uint32_t kQHdrSums = 320;                          // int [32]: block-scan partials
constexpr uint32_t kQHdrBytes = kQHdrSums + 4 * 32;
static_assert(kQHdrTags + 8 * kQuantMaxStages <= kQHdrSums, "quantizer header");
static_assert(kQuantThreads <= 1024, "quantizer block");
// Gather-table entries are 16-bit byte offsets into a staged fp16 row.
constexpr int kQuantMaxK = 32768;

// Row counters shared by the launches of one device: a launch claims rows
// from g_quant_next[slot] and counts its finished CTAs in g_quant_exits[slot];
// the last one resets both. Zero at module load.
constexpr int kQuantSlots = 1024;
__device__ unsigned long long g_quant_next[kQuantSlots];
__device__ unsigned int g_quant_exits[kQuantSlots];

// Scale and inverse scale of an INT4 group, by the significand of its
// maximum. The maximum is an fp16 value, so its fp32 significand has at most
// 10 fraction bits: 1 + f/1024 for f < 1024, times a power of two 2^E. Entry f
// holds RN((1 + f/1024)/7) and RN(7/(1 + f/1024)), each one IEEE division;
// the group's RN(amax/7) and RN(7/amax) are those entries times 2^E and 2^-E
// (a power of two scales a correctly rounded quotient exactly while it stays a
// normal number, and for fp16 inputs both always do: from 2^-27 to 2^26).
constexpr int kDivTable = 1024;

struct QuantLayout {
  // Byte offsets inside dynamic shared memory.
  uint32_t bitmap, wbase, table, divtab, stages, total;
  uint32_t row_bytes;
  int stages_n;
};

__host__ __device__ inline QuantLayout quant_layout(int K, int stages_n) {
  QuantLayout L;
  L.row_bytes = 2u * static_cast<uint32_t>(K);
  L.bitmap = kQHdrBytes;                                           // after the header
  L.wbase = L.bitmap + ((static_cast<uint32_t>(K) / 8u + 15u) & ~15u);   // int [K/32]
  L.table = L.wbase + ((static_cast<uint32_t>(K) / 8u + 15u) & ~15u);
  L.divtab = (L.table + L.row_bytes + 15u) & ~15u;                 // float2 [kDivTable]
  L.stages = (L.divtab + 8u * kDivTable + 127u) & ~127u;
  L.stages_n = stages_n;
  L.total = L.stages + static_cast<uint32_t>(stages_n) * L.row_bytes;
  return L;
}

// Gather rotation of lane `sub` (0..7) in team `team` (0..3) for a dense
// group. With every group INT8 (a8) it is a whole number of 4-element words,
// so that the 16 code bytes are put back in order by moving whole words.
__device__ __forceinline__ int quant_rotation(int sub, int team, bool a8) {
  return a8 ? 4 * team : 2 * ((sub >> 2) & 1) + 4 * team;
}

// Table slot of reordered position p: group g = p/128 is quantized by team
// g%4 of some warp; lane sub = (p%128)/16 takes element e = p%16 at gather step
// (e - rot) mod 16. Slots 0..7 of all 8 lanes come first, then slots 8..15, so
// that each 8-lane team reads 128 contiguous bytes per 16-byte table load.
__device__ __forceinline__ int quant_table_index(int p, int Gd, bool a8) {
  const int g = p >> 7, sub = (p >> 4) & 7, e = p & 15;
  const int rot = (a8 || g < Gd) ? quant_rotation(sub, g & 3, a8) : 0;
  const int slot = (e - rot) & 15;
  return (((g * 2 + (slot >> 3)) * 8 + sub) << 3) + (slot & 7);
}


// The work of one CTA; every thread returns from here to the launch-end
// bookkeeping of reorder_quant_kernel.
__device__ __forceinline__ void
reorder_quant_cta(uint8_t *smem, const __half *__restrict__ x, int64_t rows, int K, int64_t ld,
                  const int32_t *__restrict__ outlier_idx, uint8_t *__restrict__ q4,
                  int8_t *__restrict__ q8, float *__restrict__ scales, int stages_n, int crews_n,
                  int a8, unsigned long long *next) {
  const QuantLayout L = quant_layout(K, stages_n * crews_n);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kQHdrFull);
  uint64_t *empty = reinterpret_cast<uint64_t *>(smem + kQHdrEmpty);
  volatile int *flags = reinterpret_cast<volatile int *>(smem + kQHdrFlags);  // [0] bad list, [1] abort
  volatile int64_t *tags = reinterpret_cast<volatile int64_t *>(smem + kQHdrTags);
  int *warp_sums = reinterpret_cast<int *>(smem + kQHdrSums);
  uint32_t *bitmap = reinterpret_cast<uint32_t *>(smem + L.bitmap);
  int *wbase = reinterpret_cast<int *>(smem + L.wbase);
  uint16_t *table = reinterpret_cast<uint16_t *>(smem + L.table);
  float2 *divtab = reinterpret_cast<float2 *>(smem + L.divtab);
  uint8_t *stage_base = smem + L.stages;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int crew = warp / (kQuantWarps + 1), cw = warp % (kQuantWarps + 1);
  const int G = K / 128, Gd = G - 1, Kd = K - 128;
  const int64_t q4_row = Kd / 2;
  launch_dependents();   // the next kernel may start its set-up beside this one

  if (tid == 0) {
    for (int s = 0; s < stages_n * crews_n; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kQuantWarps);
    }
    flags[0] = 0;
    flags[1] = 0;
    fence_mbar_init();
  }
  for (int w = tid; w < K / 32; w += kQuantThreads) bitmap[w] = 0u;
  for (int f = tid; f < kDivTable; f += kQuantThreads) {
    const float m = __uint_as_float(0x3F800000u | (static_cast<uint32_t>(f) << 13));
    divtab[f] = make_float2(__fdiv_rn(m, 7.f), __fdiv_rn(7.f, m));
  }
  __syncthreads();
  // the set-up above touches no input or output: from here on, the kernel
  // before this one in the stream has completed
  grid_dependency_wait();
  const int oc = tid < 128 ? __ldg(outlier_idx + tid) : 0;

  // This crew's ring: stages_n slots with their barriers and row tags.
  uint64_t *cfull = full + crew * stages_n;
  uint64_t *cempty = empty + crew * stages_n;
  volatile int64_t *ctags = tags + crew * stages_n;
  uint8_t *cstage = stage_base + static_cast<size_t>(crew) * stages_n * L.row_bytes;
  const bool copier = cw == kQuantWarps && lane == 0 && crew < crews_n;
  // `ahead` is the row claimed ahead: claim() puts it in flight in ring slot
  // s and takes the next one from the launch's counter; past the last row it
  // completes the slot's phase with a plain arrival and a tag >= rows instead,
  // which tells the crew to stop, and claims nothing more.
  int64_t ahead = copier ? static_cast<int64_t>(atomicAdd(next, 1ull)) : rows;
  auto claim = [&](int s) -> bool {
    const int64_t r = ahead;
    ctags[s] = r;
    if (r >= rows) {
      mbar_arrive(&cfull[s]);
      return false;
    }
    mbar_arrive_expect_tx(&cfull[s], L.row_bytes);
    bulk_load(cstage + s * L.row_bytes, x + r * ld, L.row_bytes, &cfull[s]);
    ahead = static_cast<int64_t>(atomicAdd(next, 1ull));
    return true;
  };
  // Each crew's first row goes in flight before the table is built, the rest
  // of its ring right after: rows all requested at once would land together,
  // only once the whole burst has been served.
  int issued = 0;
  bool more = true;
  if (copier) more = claim(issued++);

  // ---- gather table: ascending non-outlier channels, then the outlier list.
  if (tid < 128) {
    const int c = oc;
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
  // wbase[w]: reordered position of the first non-outlier channel of word w
  for (int w = w0, p = base + incl - count; w < w1; ++w) {
    wbase[w] = p;
    p += __popc(~bitmap[w]);
  }
  __syncthreads();
  // table entries of the non-outlier channels, a quarter word (8 channels) per item
  for (int it = tid; it < nwords * 4; it += kQuantThreads) {
    const int w = it >> 2, qtr = it & 3;
    const uint32_t nb = ~bitmap[w];
    int pos = wbase[w] + __popc(nb & ((1u << (8 * qtr)) - 1u));
    uint32_t bits = (nb >> (8 * qtr)) & 0xFFu;
    while (bits) {
      const int b = __ffs(bits) - 1;
      bits &= bits - 1;
      if (pos < Kd)
        table[quant_table_index(pos, Gd, a8)] = static_cast<uint16_t>(2 * (w * 32 + 8 * qtr + b));
      ++pos;
    }
  }
  if (tid < 128) {
    const int c = oc;
    if (c >= 0 && c < K) table[quant_table_index(Kd + tid, Gd, a8)] = static_cast<uint16_t>(2 * c);
  }
  __syncthreads();

  if (flags[0]) {
    // Invalid outlier list: write nothing, but let the issued copies land first.
    if (tid == 0) report_status(1 /* ATOM_ERR_INVALID_ARG */);
    if (copier)
      for (int s = 0; s < issued; ++s) (void)mbar_wait(&cfull[s], 0, nullptr);
    return;
  }
  if (crew >= crews_n) return;

  if (cw == kQuantWarps) {
    // ---- copy issuer of this crew: fills the rest of the ring, then refills
    // each slot as soon as the crew's 8 warps have released it, with the
    // CTA's next row.
    if (copier)
      for (; issued < stages_n && more; ++issued) more = claim(issued);
    if (copier && more) {
      int sl = 0;
      uint32_t eph = 0;
      int64_t k = issued;  // ring positions filled so far
      for (;;) {
        if (!mbar_wait(&cempty[sl], eph, &flags[1])) {
          if (!flags[1]) report_status(6 /* ATOM_ERR_TIMEOUT */);
          flags[1] = 1;
          break;
        }
        const bool go = claim(sl);
        ++k;
        if (++sl == stages_n) {
          sl = 0;
          eph ^= 1u;
        }
        if (!go) break;
      }
      if (flags[1]) {
        // after an abort, give the copies that may still be in flight (the
        // last one issued into each slot) a bounded chance to land before the
        // CTA's shared memory is released
        for (int64_t j = (k > stages_n ? k - stages_n : 0); j < k; ++j)
          (void)mbar_wait(&cfull[j % stages_n], static_cast<uint32_t>((j / stages_n) & 1), nullptr);
      }
    }
    return;
  }

  // ---- quantizing warps: warp cw of the crew; per-lane constants: group
  // g = pass*32 + 4*cw + team, elements [16*sub, 16*sub + 16) of the group.
  const int sub = lane & 7;
  const int team = lane >> 3;
  const unsigned team_mask = 0xFFu << (8 * team);
  // Byte permutes that rotate the packed dense 8 bytes left by rot/2 bytes.
  const int krot = quant_rotation(sub, team, false) >> 1;
  // INT8 groups: code words come out rotated by `wrot` words (a8 only)
  const int wrot = a8 ? team : 0;
  uint32_t sel_lo = 0, sel_hi = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    sel_lo |= static_cast<uint32_t>((j - krot) & 7) << (4 * j);
    sel_hi |= static_cast<uint32_t>((j + 4 - krot) & 7) << (4 * j);
  }

  // The crew's ring is consumed in order: slot and barrier parity advance by
  // counting; the slot's tag says which row it holds.
  int s = 0;
  uint32_t ph = 0;
  for (;;) {
    if (!__all_sync(0xffffffffu, mbar_wait(&cfull[s], ph, &flags[1]))) {
      if (lane == 0) {
        if (!flags[1]) report_status(6 /* ATOM_ERR_TIMEOUT */);
        flags[1] = 1;
      }
      break;
    }
    const int64_t r = ctags[s];
    if (r >= rows) break;
    const uint8_t *row = cstage + s * L.row_bytes;
    uint8_t *q4_r = q4 + r * q4_row;
    int8_t *q8_r = q8 + r * (a8 ? static_cast<int64_t>(K) : 128);
    float *scales_r = scales + r;

    for (int gb = 0; gb < G; gb += 32) {
      const int g = gb + cw * 4 + team;
      if (g > Gd) continue;  // whole 8-lane teams skip together
      const bool dense = !a8 && g < Gd;
      const uint16_t *tb = table + ((g * 2) * 8 + sub) * 8;
      const uint4 oa = *reinterpret_cast<const uint4 *>(tb);       // slots 0..7
      const uint4 ob = *reinterpret_cast<const uint4 *>(tb + 64);  // slots 8..15
      const uint32_t offs[8] = {oa.x, oa.y, oa.z, oa.w, ob.x, ob.y, ob.z, ob.w};
      float2 v[8];
      float amax = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        v[j].x = __half2float(*reinterpret_cast<const __half *>(row + (offs[j] & 0xFFFFu)));
        v[j].y = __half2float(*reinterpret_cast<const __half *>(row + (offs[j] >> 16)));
        amax = fmaxf(amax, fmaxf(fabsf(v[j].x), fabsf(v[j].y)));
      }
      amax = fmaxf(amax, __shfl_xor_sync(team_mask, amax, 4));
      amax = fmaxf(amax, __shfl_xor_sync(team_mask, amax, 2));
      amax = fmaxf(amax, __shfl_xor_sync(team_mask, amax, 1));
      float scale = 0.f, inv = 0.f;
      if (dense) {
        // amax = (1 + f/1024) * 2^E: entry f, exponent moved by E
        const uint32_t ab = __float_as_uint(amax);
        const float2 t = divtab[(ab >> 13) & (kDivTable - 1)];
        const uint32_t e = (ab & 0x7F800000u) - 0x3F800000u;   // E << 23 (two's complement)
        if (amax > 0.f) {
          scale = __uint_as_float(__float_as_uint(t.x) + e);
          inv = __uint_as_float(__float_as_uint(t.y) - e);
        }
      } else if (amax > 0.f) {
        scale = __fdiv_rn(amax, 127.f);
        inv = __fdiv_rn(127.f, amax);
      }
      // code bits: the low byte of fp32(1.5*2^23 + rint(x*inv)) is the two's
      // complement code. The product is rounded to fp32 before the 1.5*2^23 add
      // rounds it to an integer (separate instructions, never one FMA).
      // (Scalar instructions: the packed f32x2 multiply and add were fused
      // into one f32x2 FMA by the compiler, which skips the product's rounding.)
      uint32_t b[16];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        b[2 * j] = __float_as_uint(__fadd_rn(__fmul_rn(v[j].x, inv), 12582912.f));
        b[2 * j + 1] = __float_as_uint(__fadd_rn(__fmul_rn(v[j].y, inv), 12582912.f));
      }
      if (dense) {
        // gather slot e holds element (e + rot) mod 16 of the lane's 16
        const uint32_t ev0 = low_bytes4(b[0], b[2], b[4], b[6]);
        const uint32_t od0 = low_bytes4(b[1], b[3], b[5], b[7]);
        const uint32_t ev1 = low_bytes4(b[8], b[10], b[12], b[14]);
        const uint32_t od1 = low_bytes4(b[9], b[11], b[13], b[15]);
        const uint32_t lo = (ev0 & 0x0F0F0F0Fu) | ((od0 << 4) & 0xF0F0F0F0u);
        const uint32_t hi = (ev1 & 0x0F0F0F0Fu) | ((od1 << 4) & 0xF0F0F0F0u);
        *reinterpret_cast<uint2 *>(q4_r + g * 64 + sub * 8) =
            make_uint2(__byte_perm(lo, hi, sel_lo), __byte_perm(lo, hi, sel_hi));
      } else {
        // gather slot e holds element (e + 4*wrot) mod 16: word j of the
        // output is slot word (j - wrot) mod 4
        const uint32_t w0 = low_bytes4(b[0], b[1], b[2], b[3]);
        const uint32_t w1 = low_bytes4(b[4], b[5], b[6], b[7]);
        const uint32_t w2 = low_bytes4(b[8], b[9], b[10], b[11]);
        const uint32_t w3 = low_bytes4(b[12], b[13], b[14], b[15]);
        uint4 o;
        o.x = wrot == 0 ? w0 : wrot == 1 ? w3 : wrot == 2 ? w2 : w1;
        o.y = wrot == 0 ? w1 : wrot == 1 ? w0 : wrot == 2 ? w3 : w2;
        o.z = wrot == 0 ? w2 : wrot == 1 ? w1 : wrot == 2 ? w0 : w3;
        o.w = wrot == 0 ? w3 : wrot == 1 ? w2 : wrot == 2 ? w1 : w0;
        *reinterpret_cast<uint4 *>(q8_r + (a8 ? g * 128 : 0) + sub * 16) = o;
      }
      if (sub == 0) scales_r[static_cast<int64_t>(g) * rows] = scale;
    }

    __syncwarp();
    if (lane == 0) mbar_arrive(&cempty[s]);
    if (++s == stages_n) {
      s = 0;
      ph ^= 1u;
    }
  }
}

// One launch over all rows, its row counter in slot `slot`. Each CTA counts
// itself out once its copy warps have made their last claim; the last one
// resets the slot, when no claim of this launch can follow.
__global__ void __launch_bounds__(kQuantThreads, 1)
reorder_quant_kernel(const __half *__restrict__ x, int64_t rows, int K, int64_t ld,
                     const int32_t *__restrict__ outlier_idx, uint8_t *__restrict__ q4,
                     int8_t *__restrict__ q8, float *__restrict__ scales, int stages_n,
                     int crews_n, int a8, int slot) {
  extern __shared__ __align__(1024) uint8_t smem[];
  reorder_quant_cta(smem, x, rows, K, ld, outlier_idx, q4, q8, scales, stages_n, crews_n, a8,
                    g_quant_next + slot);
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0 && atomicAdd(g_quant_exits + slot, 1u) == gridDim.x - 1) {
    __threadfence();
    g_quant_next[slot] = 0ull;
    g_quant_exits[slot] = 0u;
  }
}

}  // namespace atomk
