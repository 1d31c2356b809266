/*
 * atom.h -- C ABI of the Atom W4A4 mixed-precision hot path on B200 (sm_100a).
 *
 * The method: "Atom: Low-bit Quantization for Efficient and Accurate LLM
 * Serving" (arXiv abstract: 4-bit weights and 4-bit activations with a
 * mixed-precision, fine-grained quantization process; paper summary: per-group
 * scales and separate higher-precision outlier channels, a dedicated outlier
 * path for activations) and the quantization record "Atom (mixed-precision
 * block-outlier low-bit quantization for serving)" (fields "Weight group size":
 * 128; "notes": every contiguous run of 128 elements is one independently
 * quantized group, and the high-precision channel size is 128).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - G = K/128 groups per row. Groups 0..G-2 are INT4 groups over the K-128
 *    non-outlier channels; group G-1 is the INT8 group over the 128 outlier
 *    channels.
 *  - Reorder: reordered position j < K-128 holds the j-th non-outlier channel
 *    in ascending channel order; positions K-128..K-1 hold outlier_idx[0..127]
 *    in list order.
 *  - Codes are symmetric, round half to even: q = rint(fp32(x * inv)) with
 *    scale = amax/qmax and inv = qmax/amax (fp32 divisions; qmax 7 or 127;
 *    amax = 0 gives scale 0 and zero codes).
 *  - q4 layout: uint8 [rows][(K-128)/2], row-contiguous; byte i holds elements
 *    2i (low nibble) and 2i+1 (high nibble) as 4-bit two's complement.
 *    q8 layout: int8 [rows][128]. scales: float32 [G][rows] (group-major).
 *  - Every pointer is device memory owned by the caller; the library never
 *    allocates, frees or synchronises. Work is enqueued on `stream`, in stream
 *    order. The quantizers and the GEMM for M <= 64 are launched with
 *    programmatic stream serialization: their set-up may run while the
 *    previous kernel in the stream finishes. They read no input and write no
 *    output before that kernel has completed, so the ordering a caller sees is
 *    plain stream order.
 *  - Errors a host check can see (null pointers, sizes, alignment, unsupported
 *    parameters) are returned before anything is launched. Errors only the
 *    device can see (a repeated or out-of-range outlier index, a bounded wait
 *    that ran out) are recorded in a device status word that
 *    atom_device_status() reads.
 *  - Inputs must be finite.
 *
 * Thread safety: the host side keeps one per-device cache of launch facts
 * (SM count, shared-memory limits, co-resident CTA pairs), filled once under a
 * lock; calls from several host threads are safe. Two kinds of device state are
 * shared by every call on a device, whatever its stream:
 *  - the device status word (see atom_device_status): an error recorded by a
 *    kernel on one stream is what the next atom_device_status() reports, even
 *    if the caller is checking a different stream's work;
 *  - the fixed scratch array of atom_w4a4_gemm_noalloc: calls of that entry
 *    point that overlap on the GPU race on it and must be ordered by the caller.
 *  - the quantizers' row counters (atom_reorder_quant, atom_quant_weights): a
 *    ring of 1024 per device, handed out one per call in call order and reset
 *    by the launch that used it. Quantizer launches whose call numbers on the
 *    device differ by a multiple of 1024 must not run at the same time (that
 *    takes 1024 or more quantizer launches in flight at once).
 * Apart from these, calls on different streams that share no output buffer and
 * no workspace may run concurrently.
 */
#ifndef ATOM_B200_H
#define ATOM_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ATOM_API __attribute__((visibility("default")))
#else
#define ATOM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; NULL means the legacy default stream. */
typedef struct CUstream_st *atom_stream_t;

typedef enum atom_status {
    ATOM_OK = 0,
    ATOM_ERR_INVALID_ARG = 1,  /* null pointer, negative size, bad outlier list */
    ATOM_ERR_SHAPE = 2,        /* K not a multiple of 128, K < 256, N not a multiple of 8, ... */
    ATOM_ERR_ALIGN = 3,        /* pointer or leading dimension not 16-byte aligned */
    ATOM_ERR_UNSUPPORTED = 4,  /* group != 128 or n_outlier != 128, or no sm_100 device */
    ATOM_ERR_CUDA = 5,         /* a CUDA runtime call or launch failed */
    ATOM_ERR_TIMEOUT = 6       /* a device-side bounded wait gave up (device status only) */
} atom_status_t;

/*
 * atom_reorder_quant -- fused activation quantizer (the online path).
 *
 * Source: Atom paper summary ("activations get a dedicated outlier path"),
 * record field "Activation scheme" (outlier channels at higher precision, dense
 * bulk 4-bit) and "notes" (group 128, 128 high-precision channels).
 *
 *   x            fp16 [M][ld_x] device, row-major; only the first K columns are read.
 *   M            rows (tokens), M >= 0 (M == 0 is a no-op).
 *   K            channels; K % 128 == 0, 256 <= K <= 32768.
 *   ld_x         row stride of x in elements, ld_x >= K, ld_x % 8 == 0.
 *   outlier_idx  int32 [n_outlier] device: distinct channels in [0, K); the list
 *                order is the order of the outlier codes in q8.
 *   n_outlier    must be 128.      group: must be 128.
 *   q4           uint8 [M][(K-128)/2] device (output).
 *   q8           int8  [M][128]       device (output).
 *   scales       float [K/128][M]     device (output).
 * Pointers x, q4, q8 must be 16-byte aligned; scales and outlier_idx 4-byte.
 * A repeated or out-of-range outlier index makes the kernel write nothing and
 * sets the device status to ATOM_ERR_INVALID_ARG.
 */
ATOM_API atom_status_t atom_reorder_quant(const void *x, int64_t M, int64_t K, int64_t ld_x,
                                 const int32_t *outlier_idx, int32_t n_outlier, int32_t group,
                                 uint8_t *q4, int8_t *q8, float *scales, atom_stream_t stream);

/*
 * atom_quant_weights -- the offline weight quantizer.
 *
 * Source: Atom paper summary ("weights are grouped into small blocks ... with
 * per-group scales"; the outlier channels get the same permutation as the
 * activations so that the contraction pairs matching channels).
 *
 * Same arguments and layouts as atom_reorder_quant with W fp16 [N][ld_w] in
 * place of x: qw4 [N][(K-128)/2], qw8 [N][128], sw [K/128][N]. The weight
 * layout is exactly the activation layout, so the oracle compares it directly.
 */
ATOM_API atom_status_t atom_quant_weights(const void *w, int64_t N, int64_t K, int64_t ld_w,
                                 const int32_t *outlier_idx, int32_t n_outlier, int32_t group,
                                 uint8_t *qw4, int8_t *qw8, float *sw, atom_stream_t stream);

/*
 * atom_w4a4_gemm -- mixed-precision group-scaled integer GEMM.
 *
 * Source: Atom abstract (low-bit integer operators for the 4-bit
 * weight-activation product) and record field "Kernels" (purpose-built low-bit
 * kernels). Computes, for every m < M and n < N,
 *
 *   Y[m][n] = fp16( sum_g sa[g][m] * sw[g][n] * P[g][m][n] ),
 *   P[g][m][n] = sum over the 128 reordered positions k of group g of qa[m][k]*qw[n][k],
 *
 * with exact int32 partials on the tensor cores and an fp32 accumulation of the
 * dequantized partials (summation order unspecified).
 *
 *   qa4, qa8, sa   activation codes/scales as written by atom_reorder_quant (M rows).
 *   qw4, qw8, sw   weight codes/scales as written by atom_quant_weights (N rows).
 *   y              fp16 [M][N] device (output), row-major.
 *   M >= 0, N >= 8 with N % 8 == 0, K as above; n_outlier == group == 128.
 *   workspace      device scratch that lets shapes whose output tiles would leave
 *                  most SMs idle (small M, e.g. decode) split K into ranges, whose
 *                  fp32 partial tiles are then summed in range order into y. For
 *                  M > 64 (up to 16 ranges of >= 4 groups) the partial tiles are
 *                  written to workspace [splits][M][N] and a second kernel on the
 *                  same stream sums them. For M <= 64 (up to 8 ranges of >= 2
 *                  groups) the ranges of a weight tile run as one thread-block
 *                  cluster that sums them in shared memory: the workspace is then
 *                  only the caller's consent to the split and is not written.
 *                  Caller-owned, 16-byte aligned, at least
 *                  atom_gemm_workspace_bytes(M, N, K) bytes; its contents need no
 *                  initialisation and are garbage afterwards. NULL, or fewer bytes,
 *                  runs without splitting K (same result up to the fp32 summation
 *                  order). Two calls that overlap on the GPU must not share a
 *                  workspace.
 * Pointers qa4, qw4, qa8, qw8, y must be 16-byte aligned; sa, sw 4-byte.
 */
ATOM_API atom_status_t atom_w4a4_gemm(const uint8_t *qa4, const int8_t *qa8, const float *sa,
                             const uint8_t *qw4, const int8_t *qw8, const float *sw,
                             void *y, int64_t M, int64_t N, int64_t K,
                             int32_t n_outlier, int32_t group,
                             void *workspace, size_t workspace_bytes, atom_stream_t stream);

/*
 * atom_w4a4_gemm_partials -- debug twin of atom_w4a4_gemm that also writes the
 * per-group integer partial sums P (same definition as above).
 *
 *   partials  int32 [K/128][M][N] device (output).
 *   y         fp16 [M][N] device (output) or NULL to skip it.
 * Runs the same tensor-core mainloop as atom_w4a4_gemm. Meant for small shapes:
 * the partials tensor is G times the size of Y.
 */
ATOM_API atom_status_t atom_w4a4_gemm_partials(const uint8_t *qa4, const int8_t *qa8, const float *sa,
                                      const uint8_t *qw4, const int8_t *qw8, const float *sw,
                                      int32_t *partials, void *y,
                                      int64_t M, int64_t N, int64_t K,
                                      int32_t n_outlier, int32_t group, atom_stream_t stream);

/*
 * W4A8 variant: INT8 activations in every group, the W4A4 weights unchanged.
 *
 * The pages set Atom's 4-bit kernels beside 8-bit activation schemes ("Atom:
 * Low-bit Quantization for Efficient and Accurate LLM Serving", abstract and
 * paper summary). This variant keeps Atom's layout and outlier reorder, and
 * quantizes every 128-channel group of the reordered activation row to INT8 with
 * the same steps as the outlier group ("Atom (mixed-precision block-outlier
 * low-bit quantization for serving)", fields Weight group size and notes):
 *   scale = fl32(amax/127), inv = fl32(127/amax) (0 for a zero group),
 *   q = rint(fl32(x*inv)), ties to even.
 *
 * atom_reorder_quant_a8: x, M, K, ld_x, outlier_idx, n_outlier, group as for
 *   atom_reorder_quant;
 *   q8      int8 [M][K] device (output), the codes in reordered channel order;
 *   scales  float [K/128][M] device (output).
 *   q8 must be 16-byte aligned; errors as atom_reorder_quant.
 */
ATOM_API atom_status_t atom_reorder_quant_a8(const void *x, int64_t M, int64_t K, int64_t ld_x,
                                            const int32_t *outlier_idx, int32_t n_outlier,
                                            int32_t group, int8_t *q8, float *scales,
                                            atom_stream_t stream);

/*
 * atom_w4a8_gemm: Y[m][n] = fp16( sum_g sa[g][m] * sw[g][n] * P[g][m][n] ) with
 * P[g][m][n] = sum_{k in g} qa8[m][k] * qw[n][k] exact in int32 (INT8 x INT4 for
 * the dense groups, INT8 x INT8 for the outlier group); fp32 accumulation of
 * the dequantized partials.
 *   qa8, sa        as written by atom_reorder_quant_a8 (M rows).
 *   qw4, qw8, sw   as written by atom_quant_weights (N rows).
 *   y              fp16 [M][N] device (output).
 *   M >= 0, N >= 8 with N % 8 == 0, K as for atom_w4a4_gemm. K is never split.
 * atom_w4a8_gemm_partials: the same, writing P as int32 [G][M][N] (debug) and,
 *   when y is not NULL, Y.
 * qa8, qw4, qw8, y, partials must be 16-byte aligned; sa, sw 4-byte.
 */
ATOM_API atom_status_t atom_w4a8_gemm(const int8_t *qa8, const float *sa, const uint8_t *qw4,
                                     const int8_t *qw8, const float *sw, void *y, int64_t M,
                                     int64_t N, int64_t K, int32_t n_outlier, int32_t group,
                                     atom_stream_t stream);
ATOM_API atom_status_t atom_w4a8_gemm_partials(const int8_t *qa8, const float *sa,
                                              const uint8_t *qw4, const int8_t *qw8,
                                              const float *sw, int32_t *partials, void *y,
                                              int64_t M, int64_t N, int64_t K,
                                              int32_t n_outlier, int32_t group,
                                              atom_stream_t stream);

/*
 * atom_w4a4_gemm_quant -- the GEMM of atom_w4a4_gemm with the next layer's
 * activation quantization fused into its epilogue: instead of fp16 Y it writes
 * the INT4/INT8 codes and scales that atom_reorder_quant would produce from Y,
 * with Y's last 128 columns as the outlier channels and no other reorder.
 *
 * The pages quantize every activation with its outlier channels moved to the
 * tail ("Atom: Low-bit Quantization for Efficient and Accurate LLM Serving",
 * paper summary: activations get a dedicated outlier path). Here that reorder is
 * assumed to be folded offline into this layer's weight rows (and their order
 * of output channels), so that Y's columns already come out in the next
 * layer's reordered order; each 128-column group of a row is then formed and
 * quantized where it is computed. For every row m and group g of Y's columns:
 *   yh   = fp16_rn(the value atom_w4a4_gemm writes, unsplit),
 *   amax = max |yh| over the group, qmax = 7 (g < N/128 - 1) or 127 (last group),
 *   scale = fl32(amax / qmax), inv = fl32(qmax / amax) (both 0 when amax == 0),
 *   q    = rint(fl32(yh * inv)), ties to even,
 * packed as atom_reorder_quant packs them.
 *
 *   qa4 ... sw     as for atom_w4a4_gemm; M >= 0, K as there.
 *   N              Y's columns = the next layer's K: N % 128 == 0, 256 <= N <= 32768.
 *   qy4            uint8 [M][(N-128)/2] device (output), INT4 codes of groups 0..N/128-2.
 *   qy8            int8  [M][128] device (output), INT8 codes of Y's last 128 columns.
 *   sy             float [N/128][M] device (output), group scales.
 * K is never split (no workspace). qy4 and qy8 must be 16-byte aligned, sy 4-byte.
 * Errors as atom_w4a4_gemm; ATOM_ERR_SHAPE for an N outside the range above.
 */
ATOM_API atom_status_t atom_w4a4_gemm_quant(const uint8_t *qa4, const int8_t *qa8,
                                           const float *sa, const uint8_t *qw4,
                                           const int8_t *qw8, const float *sw, int64_t M,
                                           int64_t N, int64_t K, int32_t n_outlier,
                                           int32_t group, uint8_t *qy4, int8_t *qy8, float *sy,
                                           atom_stream_t stream);

/*
 * Tiled weight layout -- the library's own layout of the packed INT4 weight
 * codes, a one-off repack of what atom_quant_weights writes.
 *
 * The pages fix what the codes are (4-bit groups of 128 channels with per-group
 * scales: "Atom (mixed-precision block-outlier low-bit quantization for
 * serving)", fields Bits and Weight group size; the paper summary's weight
 * blocks) but not how the weights are laid out for the kernels; the weights
 * are quantized offline, so their layout is the kernels' choice. In the row
 * layout qw4 [N][(K-128)/2], the 128-row x 64-byte piece a GEMM needs per
 * weight tile and group is 128 pieces of 64 bytes, (K-128)/2 bytes apart. The
 * tiled layout stores each (tile, group) piece as one contiguous 8 KB block:
 *
 *   qw4t[((t * G4 + g) * 128 + r) * 64 + j] = qw4[128 t + r][64 g + j]
 *   for tile t < ceil(N/128), group g < G4 = K/128 - 1, row r < 128, j < 64;
 *   rows 128 t + r >= N of the last tile are zero.
 *
 * qw8 and sw keep their layouts. A decode GEMM reads every weight once per
 * call, and reads the tiled layout as long contiguous runs instead of 64-byte
 * pieces.
 *
 * atom_tiled_weights_bytes: bytes of the tiled layout, ceil(N/128) * G4 * 8192
 *   (0 for N <= 0 or a K outside [256, 32768] or not a multiple of 128).
 * atom_pack_weights_tiled: qw4 (row layout, N rows) -> qw4t (tiled layout).
 * atom_unpack_weights_tiled: qw4t -> qw4 (rows n < N), the inverse copy.
 *   N >= 0 (0 is a no-op), K as for atom_quant_weights; both pointers device
 *   memory, 16-byte aligned; the buffers must not overlap.
 * atom_w4a4_gemm_tiled: atom_w4a4_gemm (same arguments, result and errors) with
 *   the packed INT4 weights `qw4t` in the tiled layout. Same kernels, same
 *   arithmetic in the same order: Y is bit-identical to atom_w4a4_gemm's on the
 *   row layout of the same weights, with the same workspace.
 */
ATOM_API size_t atom_tiled_weights_bytes(int64_t N, int64_t K);
ATOM_API atom_status_t atom_pack_weights_tiled(const uint8_t *qw4, int64_t N, int64_t K,
                                               uint8_t *qw4t, atom_stream_t stream);
ATOM_API atom_status_t atom_unpack_weights_tiled(const uint8_t *qw4t, int64_t N, int64_t K,
                                                 uint8_t *qw4, atom_stream_t stream);
ATOM_API atom_status_t atom_w4a4_gemm_tiled(const uint8_t *qa4, const int8_t *qa8,
                                            const float *sa, const uint8_t *qw4t,
                                            const int8_t *qw8, const float *sw, void *y,
                                            int64_t M, int64_t N, int64_t K, int32_t n_outlier,
                                            int32_t group, void *workspace,
                                            size_t workspace_bytes, atom_stream_t stream);

/*
 * Bytes of workspace atom_w4a4_gemm uses for this shape on the current device:
 * splits * M * N * 4 when it would split K, else 0 (also 0 on error).
 */
ATOM_API size_t atom_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);

/*
 * atom_w4a4_gemm_noalloc -- atom_w4a4_gemm for callers that cannot allocate
 * device memory around the call: serving runtimes that hand all device memory
 * to a fixed pool at start-up (there is nothing left to allocate from), and C
 * or embedded callers that have no device allocator of their own. (The pages
 * have no counterpart; it is a deployment convenience of this library.)
 *
 * Arguments, layouts, result and errors are those of atom_w4a4_gemm without
 * the workspace. When the shape splits K through a workspace (M > 64 with few
 * output tiles), the split's fp32 partial tiles go to a fixed 8 MiB array in
 * the library's device memory instead of a caller workspace; every GPU that
 * loads the library holds that array until the process exits. A shape whose
 * partials would need more than 8 MiB (the value atom_gemm_workspace_bytes
 * reports) returns ATOM_ERR_SHAPE before anything is launched. The call
 * allocates nothing.
 *
 * All calls on a device share the array, and a call leaves its partials in
 * it: two calls that overlap on the GPU (other streams, other host threads)
 * race and must be ordered by the caller. The first call on each device does
 * a one-time set-up with that device current (it looks up the array's device
 * address with cudaGetSymbolAddress and the kernel's launch limits); make that
 * first call before any stream capture.
 */
ATOM_API atom_status_t atom_w4a4_gemm_noalloc(const uint8_t *qa4, const int8_t *qa8,
                                              const float *sa, const uint8_t *qw4,
                                              const int8_t *qw8, const float *sw, void *y,
                                              int64_t M, int64_t N, int64_t K,
                                              int32_t n_outlier, int32_t group,
                                              atom_stream_t stream);

/*
 * atom_w8a8_gemm -- the 8-bit comparator of the W4A4 GEMM: INT8 activations
 * and weights with one scale per activation row and one per weight row,
 *
 *   y[m][n] = fp16( float(P) * (sa[m] * sw[n]) ),  P = sum_k qa[m][k] * qw[n][k]
 *
 * where P is the exact int32 dot product over all of K (no groups; a
 * per-tensor scale is constant sa and sw). Source: the Atom paper's comparison
 * of its W4A4 kernels with 8-bit weight-and-activation serving
 * ("Atom: Low-bit Quantization for Efficient and Accurate LLM Serving",
 * summary of results); the pages give no INT8 kernel, so this restates the
 * plain per-row x per-column scaled INT8 GEMM on the same tensor-core pipeline
 * as the W4A4 GEMM.
 *
 *   qa  int8 [M][K] device, row-major (row pitch K bytes).
 *   sa  fp32 [M] device.
 *   qw  int8 [N][K] device, row-major.
 *   sw  fp32 [N] device.
 *   y   fp16 [M][N] device (output), row-major, written in full.
 * Preconditions (else ATOM_ERR_SHAPE before any launch): K % 16 == 0,
 * 16 <= K <= 131072 (the int32 sum cannot overflow), N % 8 == 0. M = 0 or
 * N = 0 is a no-op. qa, qw, y and sw must be 16-byte aligned, sa 4-byte
 * (else ATOM_ERR_ALIGN). Stream-ordered, allocates nothing; the result is
 * deterministic.
 */
ATOM_API atom_status_t atom_w8a8_gemm(const int8_t *qa, const float *sa, const int8_t *qw,
                                      const float *sw, void *y, int64_t M, int64_t N,
                                      int64_t K, atom_stream_t stream);

/*
 * atom_kv_quant / atom_kv_dequant -- INT4 KV cache, one group per (token, head)
 * vector of head_dim = 128 elements. The pages place Atom under KV-cache
 * quantization ("Atom: Low-bit Quantization for Efficient and Accurate LLM
 * Serving", key facts) without a KV recipe; the reading used is the Atom INT4
 * group encoding ("Atom (mixed-precision block-outlier low-bit quantization
 * for serving)", Bits and Weight group size) with no reorder and no outliers:
 *
 *   scale[g] = fl32(amax / 7), inv = fl32(7 / amax)   (0, 0 for an all-zero group)
 *   q = rint(fl32(x * inv)) in [-7, 7], ties to even
 *   q4[g][i] = (q[2i] & 0xF) | (q[2i+1] << 4)
 *   atom_kv_dequant: out[g][j] = fp16_rn(fl32(q[j] * scale[g]))
 *
 *   x, out   fp16 [groups][128] device (a cache [tokens][heads][128] flattened).
 *   q4       uint8 [groups][64] device.
 *   scales   fp32 [groups] device.
 * groups = 0 is a no-op; negative groups or a null pointer ->
 * ATOM_ERR_INVALID_ARG; x and out must be 16-byte aligned, q4 8-byte, scales
 * 4-byte (else ATOM_ERR_ALIGN). Inputs must be finite. Stream-ordered,
 * allocates nothing.
 */
ATOM_API atom_status_t atom_kv_quant(const void *x, int64_t groups, uint8_t *q4, float *scales,
                                     atom_stream_t stream);
ATOM_API atom_status_t atom_kv_dequant(const uint8_t *q4, const float *scales, int64_t groups,
                                       void *out, atom_stream_t stream);

/*
 * atom_probe_mma_i8 -- a measurement aid (the pages have no counterpart): the
 * dense INT8 tensor-core rate of this GPU, the second roofline denominator of
 * the W4A4 GEMM. Every CTA pair the GPU holds at once (one CTA per SM) issues
 * `groups` groups of four tcgen05.mma.cta_group::2.kind::i8 of the GEMM's shape
 * (M = 256, N = 256, K = 32, zero-filled operands in shared memory) into two
 * alternating TMEM accumulators, with no loads and no dequantization. The
 * launch performs 2 * 256 * 256 * 128 * groups * (*pairs_out) integer
 * operations; the caller times it on `stream`.
 *
 *   groups     1 <= groups <= 2^20 (else ATOM_ERR_INVALID_ARG).
 *   pairs_out  host int32 (output): the number of CTA pairs launched.
 * Stream-ordered, allocates nothing.
 */
ATOM_API atom_status_t atom_probe_mma_i8(int64_t groups, int32_t *pairs_out,
                                         atom_stream_t stream);

/*
 * atom_debug_wait_timeout -- a test aid for the library's failure detection
 * (the pages have no counterpart). Every pipeline wait in the GEMM and
 * quantizer kernels is bounded: a wait that runs past its limit gives up,
 * records ATOM_ERR_TIMEOUT in the device status word and lets the kernel end,
 * instead of hanging the GPU. This entry point runs that same bounded wait
 * (the same device function) in a one-thread kernel on an mbarrier that
 * nothing ever arrives on and that no copy or MMA is tied to, with a limit of
 * `limit_ns` nanoseconds in place of the production 1 s. The kernel therefore
 * gives up after about `limit_ns`, and the next atom_device_status() reports
 * ATOM_ERR_TIMEOUT. Nothing is left in flight; the context stays usable.
 *
 *   limit_ns  0 < limit_ns <= 1e9 (else ATOM_ERR_INVALID_ARG).
 * Stream-ordered, allocates nothing.
 */
ATOM_API atom_status_t atom_debug_wait_timeout(uint64_t limit_ns, atom_stream_t stream);

/*
 * atom_device_status -- first device-detected error since the last clear on the
 * current device (ATOM_OK if none). Synchronises the current device. With
 * clear != 0 the status is reset to ATOM_OK afterwards.
 */
ATOM_API atom_status_t atom_device_status(int clear);

/* Static, human-readable name of a status code. */
ATOM_API const char *atom_status_string(atom_status_t status);

/* Library ABI version: major*10000 + minor*100 + patch. */
ATOM_API int atom_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATOM_B200_H */
