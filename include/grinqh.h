/*
 * grinqh.h -- C ABI of libgrinqh, the B200 (sm_100a) batch-1 decode path of
 * GRINQH ("Graded Input-Based Quantization Hierarchy for Efficient LLM
 * Generation"): activation-graded precision assignment, bit-plane-sparse
 * weight loading, on-chip reconstruction with midpoint bias correction, and
 * the GEMV y = W_hat^T x.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every pointer is a DEVICE pointer owned by the caller.  The library never
 *    allocates, frees or keeps device memory between calls (except the fixed
 *    scratch array of grinqh_decode_gemv_noalloc, at the end of this file).
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL means the legacy default stream).  No call synchronises with the
 *    host, so they may be captured in a CUDA graph.
 *  - fp16 values (x, s, z) are passed as their IEEE binary16 bit patterns.
 *  - The return value is a status code (below).  On failure nothing has been
 *    launched, except for GRINQH_ERR_CUDA (a launch failed); a message for the
 *    calling thread is available from grinqh_last_error().
 *  - Shapes: d_in % 128 == 0, 128 <= d_in <= 2^24; d_out % 16 == 0,
 *    16 <= d_out <= 2^24; b_max in {2, 4, 6, 8}.  P = b_max/2 planes,
 *    G = d_in/128 groups.
 *  - Row index = input channel i (reduction dimension), output index o.
 *
 * Layouts (the GRINQH notes, "Key design 2": 2-bit slices stacked from most
 * to least significant, rows stored reduction-dimension major, 16 slices per
 * 32-bit word):
 *    planes  uint32 [d_in][P][d_out/16]; word j of region (i, p) holds the
 *            p-th most significant 2-bit slice of codes q[i][16j .. 16j+15],
 *            output 16j+t in bits [2t+1 : 2t].  A row read at bit width b is
 *            the contiguous prefix of its first b/2 regions.
 *    s, z    fp16 [G][d_out]: scale and additive zero per (128-row group,
 *            output channel).
 */
#ifndef GRINQH_H
#define GRINQH_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes --------------------------------------------------------- */
#define GRINQH_OK 0
#define GRINQH_ERR_INVALID_ARG (-1)       /* null pointer, bad b_max, bad value */
#define GRINQH_ERR_UNSUPPORTED_SHAPE (-2) /* d_in / d_out outside the rules above */
#define GRINQH_ERR_WORKSPACE_TOO_SMALL (-3)
#define GRINQH_ERR_CUDA (-4)              /* a CUDA runtime call or launch failed */
#define GRINQH_ERR_DEVICE (-5)            /* a device-side check set the error word */

/* Library version, major * 1000 + minor. */
int grinqh_version(void);

/* Message describing the last failing call made by this host thread ("" if
 * none).  The pointer stays valid until the thread's next library call. */
const char *grinqh_last_error(void);

/* Bytes of device workspace that grinqh_assign + grinqh_gemv need for one
 * (d_in, d_out, b_max) linear layer; 0 for an unsupported shape.  The
 * workspace carries the compacted unit stream from assign to gemv, the
 * split-K partial sums, the split-K arrival counters and a device error word.
 * It MUST be zero-filled once after allocation (e.g. cudaMemsetAsync); every
 * call leaves its split-K state (counters, and the fused decode's partial
 * words) and the error word back at zero.  One workspace
 * may serve several layers in sequence on one stream (size it for the
 * largest), but calls that overlap in time need distinct workspaces. */
size_t grinqh_workspace_bytes(int d_in, int d_out, int b_max);

/* Offline bit-plane packing ("Key design 2").
 *   q       uint8 [d_in][d_out], codes of the b_max-bit base quantizer
 *           (only their low b_max bits are packed; higher bits are ignored).
 *   planes  uint32 [d_in][P][d_out/16] out, layout above.
 * Deterministic; one kernel. */
int grinqh_pack(const uint8_t *q, int d_in, int d_out, int b_max, uint32_t *planes,
                void *stream);

/* Inverse of grinqh_pack (a test and inspection aid): q_out = codes. */
int grinqh_unpack(const uint32_t *planes, int d_in, int d_out, int b_max, uint8_t *q_out,
                  void *stream);

/* Runtime precision assignment and row compaction ("Key design 1").
 *   x        fp16 [d_in] decode-time input vector.
 *   theta    fp32 [P] thresholds theta_1..theta_P (meant to be increasing):
 *            b_i = 2 * #{k : theta_k <= |x_i|}, compared in fp32 on the
 *            exactly converted |x_i|.  So a tie takes the higher level, -0 has
 *            |x| = 0, +-Inf gets b_max and NaN gets b = 0.
 *   phi      fp32 [P+1] midpoint offsets per level k (width 2k), or NULL for
 *            the default of "Key design 3": phi_k = 2^(b_max-2k-1) for
 *            2k < b_max and 0 at full width (nothing is truncated there).
 *            phi[0] is never used.
 *   b        uint8 [d_in] out: bit width of each input channel.
 *   lists    int32 [P][d_in] out: list p holds, ascending, every i with
 *            b_i > 2p (rows whose p-th plane is read); entries past
 *            counts[p] are left untouched.
 *   counts   int32 [P] out: lengths of the lists.
 *   grp_sums fp32 [2][G] out: X_g = sum of x_i and Phi_g = sum of
 *            x_i * phi_{b_i/2} over rows of group g with b_i > 0.
 *   ws       workspace of grinqh_workspace_bytes(d_in, d_out, b_max) bytes
 *            for the d_out of the grinqh_gemv that follows; assign writes
 *            the group-ordered unit stream there.
 * b, lists and counts are bit-exact functions of (x, theta); grp_sums are
 * sums in a fixed order (deterministic). */
int grinqh_assign(const uint16_t *x, const float *theta, int d_in, int b_max, const float *phi,
                  uint8_t *b, int32_t *lists, int32_t *counts, float *grp_sums, void *ws,
                  size_t ws_bytes, void *stream);

/* The fused plane-sparse reconstruct-and-GEMV (GRINQH notes, "Method /
 * overall framework" stages 2-3 and the custom GEMV operator):
 *   y_o = sum over i with b_i > 0 of x_i * w_hat(i, o),
 *   w_hat(i, o) = s[g][o] * (Q(i, o) + phi_{b_i/2}) + z[g][o],  g = i/128,
 * where Q is the code with its low b_max - b_i bits cleared, rebuilt from the
 * first b_i/2 planes only (the others, and every plane of a b_i = 0 row, are
 * never read).  Consumes the unit stream that grinqh_assign left in `ws`
 * (same d_in, b_max; the workspace must be sized for this d_out) and its
 * grp_sums.  Writes every y[o] (fp32 [d_out]); no pre-zeroing needed.
 * Deterministic (fixed-order split-K reduction). */
int grinqh_gemv(const uint32_t *planes, const uint16_t *s, const uint16_t *z,
                const float *grp_sums, int d_in, int d_out, int b_max, float *y, void *ws,
                size_t ws_bytes, void *stream);

/* The whole decode step in one kernel (the GRINQH notes, "Method / overall
 * framework" stages 1-3: grinqh_assign followed by grinqh_gemv, fused): every
 * CTA derives the precision assignment and the per-plane compaction it needs
 * from x and theta itself, so no unit stream goes through device memory and
 * no second launch waits on the first.
 *   planes, s, z  the packed layer, as for grinqh_gemv.
 *   x, theta, phi as for grinqh_assign.
 *   y             fp32 [d_out] out, the same value grinqh_gemv computes after
 *                 grinqh_assign (within the rounding of a different summation
 *                 order); every y[o] is written.
 *   b, lists, counts, grp_sums  optional outputs with exactly the contents
 *                 grinqh_assign writes (bit-exact, grp_sums in the same order);
 *                 pass NULL for any of them to skip it.
 *   ws            workspace of grinqh_workspace_bytes(d_in, d_out, b_max)
 *                 bytes (zero-filled once; left zeroed), used for the split-K
 *                 partial sums and counters only.
 * Limits: d_in <= 65536 (GRINQH_ERR_UNSUPPORTED_SHAPE otherwise; use
 * grinqh_assign + grinqh_gemv there).  Deterministic.
 * Launch overlap: the kernel may start while the kernel before it on `stream`
 * is still finishing (programmatic dependent launch), and it reads theta and
 * phi before waiting for that kernel; x, planes, s and z are read only after
 * the wait, and every output is written after it.  So theta and phi must not
 * be written by the kernel launched immediately before this call on the same
 * stream (a copy, an event or any other kernel in between lifts this).
 * Launch: cooperative (every CTA is resident at once; the launch waits for room
 * on the GPU, and fails with GRINQH_ERR_CUDA if the grid cannot fit, e.g. under
 * an SM-limited MPS client), so the split-K waits between the CTAs of one output
 * tile always end, whatever else the GPU runs.
 * Device errors (grinqh_check_device_error): 3 if a split-K wait gave up (about
 * half a second; never on a correct launch) or a split-K partial word of the
 * workspace was not zero when the call started (the workspace was not left
 * zeroed: after any device error, let grinqh_check_device_error clear it); 5 if
 * a wait inside the kernel's copy/MMA pipeline gave up (about a second; never on
 * a correct launch).  In both cases y is not valid. */
int grinqh_decode_gemv(const uint32_t *planes, const uint16_t *s, const uint16_t *z,
                       const uint16_t *x, const float *theta, const float *phi, int d_in,
                       int d_out, int b_max, float *y, uint8_t *b, int32_t *lists,
                       int32_t *counts, float *grp_sums, void *ws, size_t ws_bytes,
                       void *stream);

/* ---- Grouped decode (several independent linears in one launch) -------------
 * The linears of a decoder layer that do not depend on each other -- q, k and
 * v, or gate and up -- each run as grinqh_decode_gemv would (every linear its
 * own x, theta, phi and y), but in one kernel launch: the GPU's CTAs are split
 * between them in proportion to their plane bytes, so the launch's fixed costs
 * (the wait on the kernel before, the per-CTA front end, the split-K tail) are
 * paid once for the group.  The optional outputs (b, lists, counts, group sums)
 * are not produced.  Each linear obeys the rules of grinqh_decode_gemv (d_in
 * <= 65536, alignment, theta and phi not written by the kernel launched just
 * before).  y of a linear equals its single-call y within the summation-order
 * rounding (its CTAs take different row slices).
 *   n      1 .. GRINQH_MAX_GROUP linears.
 *   lins   host array of n descriptors (read during the call only).
 *   ws     workspace of grinqh_group_workspace_bytes() bytes (zero-filled once;
 *          left zeroed), not shared with a concurrent call. */
#define GRINQH_MAX_GROUP 4
typedef struct grinqh_linear {
  const uint32_t *planes; /* as for grinqh_decode_gemv */
  const uint16_t *s;
  const uint16_t *z;
  const uint16_t *x;
  const float *theta;
  const float *phi; /* NULL: the default table */
  int d_in;
  int d_out;
  int b_max;
  float *y; /* fp32 [d_out] out */
} grinqh_linear;
size_t grinqh_group_workspace_bytes(void);
int grinqh_decode_gemv_group(int n, const grinqh_linear *lins, void *ws, size_t ws_bytes,
                             void *stream);

/* ---- Small-batch decode (B <= 8 tokens sharing one read of the planes) --------
 * GRINQH notes, "Limitations and outlook": beyond batch 1 the requests' active
 * channels differ.  Every token t of the batch gets its own widths
 * b_t(i) = 2 #{k : theta_k <= |x_t(i)|} and its own
 *   y[t][o] = sum over i with b_t(i) > 0 of x[t][i] * w_hat_t(i, o),
 *   w_hat_t(i, o) = s[g][o] * (Q_t(i, o) + phi_{b_t(i)/2}) + z[g][o],
 * exactly what grinqh_decode_gemv computes for that token alone (within the
 * rounding of a different summation order).  Row i's planes are read once, for
 * the largest width any token gives it, and each field is decoded once.
 *   planes, s, z  the packed layer, as for grinqh_decode_gemv.
 *   x             fp16 [B][d_in], row t the input of token t (16-byte aligned).
 *   theta, phi    as for grinqh_assign (one threshold set for the batch).
 *   B             1 .. GRINQH_MAX_BATCH tokens.
 *   y             fp32 [B][d_out] out; every element is written.
 *   u             uint8 [d_in] out, or NULL: the union widths u_i = max_t b_t(i)
 *                 (the planes read for row i), bit-exact.
 *   ws            at least grinqh_batch_workspace_bytes() bytes, zero-filled once
 *                 after allocation and left zeroed by every call; not shared
 *                 with a concurrent call.
 * Limits: d_in <= 65536.  Deterministic.  Launch overlap and device errors as
 * for grinqh_decode_gemv (theta and phi are read before the wait on the kernel
 * launched just before). */
#define GRINQH_MAX_BATCH 8
size_t grinqh_batch_workspace_bytes(void);
int grinqh_decode_gemv_batch(const uint32_t *planes, const uint16_t *s, const uint16_t *z,
                             const uint16_t *x, const float *theta, const float *phi, int B,
                             int d_in, int d_out, int b_max, float *y, uint8_t *u, void *ws,
                             size_t ws_bytes, void *stream);

/* ---- Prefill GEMM (every row at the full width b_max) -------------------------
 * The pages' other phase: for a block of T tokens every input channel runs at
 * the base width, so all P planes are read and
 *   Y[t][o] = sum_i X[t][i] * (s[g][o] * (q[i][o] + phi_P) + z[g][o]),  g = i/128,
 * q the full b_max-bit code.  Each w_hat is rounded once to fp16: one fused
 * fp16 multiply-add s q + z of the exact code when phi_P = 0 (the correctly
 * rounded value, relative error <= 2^-11, inside the decode tolerance), and
 * fmaf(s, q + phi_P, z) in fp32 when an explicit phi_P != 0; the products run
 * on the tensor cores with fp32 accumulation, and the partial sums of the d_in
 * ranges are added into Y (so the last bits of Y depend on their order).
 *   planes, s, z  the packed layer, as for grinqh_decode_gemv; d_out must be a
 *                 multiple of 128 (GRINQH_ERR_UNSUPPORTED_SHAPE otherwise).
 *   x             fp16 [T][d_in] (16-byte aligned), T in [1, 65536].
 *   phi           fp32 [b_max/2 + 1] or NULL (phi_P = 0).
 *   y             fp32 [T][d_out] out (cleared by the call, then accumulated).
 *   ws            at least grinqh_prefill_workspace_bytes() bytes (its device
 *                 error word; 4 if a wait on the tensor cores gave up). */
size_t grinqh_prefill_workspace_bytes(void);
int grinqh_prefill_gemm(const uint32_t *planes, const uint16_t *s, const uint16_t *z,
                        const uint16_t *x, const float *phi, int T, int d_in, int d_out,
                        int b_max, float *y, void *ws, size_t ws_bytes, void *stream);

/* Reads and clears the device error word of `ws` (synchronises `stream`).
 * Returns GRINQH_OK, or GRINQH_ERR_DEVICE with the device code in
 * grinqh_last_error(); in that case it also zeroes the workspace's split-K
 * state (its fixed-offset part), which a failed call may have left behind. */
int grinqh_check_device_error(void *ws, void *stream);

/* ---- Dense 4-bit comparator (not a GRINQH step) ------------------------------
 * The fixed-width baseline of the GRINQH notes' throughput table ("4-bit
 * MARLIN"), rebuilt here on the same shape, group size and fp16 s/z so the
 * two kernels can be timed side by side.
 *   w4 uint32 [d_in][d_out/8]: word j of row i holds 4-bit codes of outputs
 *      8j..8j+7, output 8j+t in bits [4t+3 : 4t].
 *   y_o = sum_i x_i * (s[g][o] * q4(i, o) + z[g][o]).  */
int grinqh_pack_dense4(const uint8_t *q4, int d_in, int d_out, uint32_t *w4, void *stream);
size_t grinqh_dense4_workspace_bytes(int d_in, int d_out);
int grinqh_gemv_dense4(const uint32_t *w4, const uint16_t *s, const uint16_t *z,
                       const uint16_t *x, int d_in, int d_out, float *y, void *ws,
                       size_t ws_bytes, void *stream);

/* ---- Decode GEMV without any device allocation (no counterpart in the paper:
 * the GRINQH notes describe no such interface) ----------------------------------
 * For callers that cannot allocate device memory -- a host framework that owns
 * every byte of device memory and only hands its plug-ins streams and tensors,
 * or a latency-critical path that must never enter the allocator.  It runs
 * the fused decode kernel (grinqh_decode_gemv without its optional outputs),
 * keeping its split-K partial sums and its device error word in a fixed
 * array of about 1 MB that the library reserves
 * on every GPU that loads it and holds until exit; it calls no
 * cudaMalloc/cudaFree.
 *   planes, s, z  the packed layer (as for grinqh_gemv); x, theta, phi as for
 *                 grinqh_assign; y fp32 [d_out] out.
 *   Limits: those of grinqh_decode_gemv (d_in <= 65536); larger shapes return
 *   GRINQH_ERR_UNSUPPORTED_SHAPE with a message, and nothing is queued on any
 *   failed call.  The array holds the split-K state of every accepted shape.
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  Every call shares the one array (a completed
 * call leaves its split-K words at zero; a call is one kernel launch and
 * nothing else), so calls that overlap on the GPU -- several streams, or
 * several host threads on one device -- race and must be serialised by the
 * caller.  The device error word is not cleared by a call:
 * it keeps the first device error (codes as for grinqh_decode_gemv) until
 * grinqh_noalloc_check_device_error reads it. */
int grinqh_decode_gemv_noalloc(const uint32_t *planes, const uint16_t *s, const uint16_t *z,
                               const uint16_t *x, const float *theta, const float *phi,
                               int d_in, int d_out, int b_max, float *y, void *stream);

/* Reads the no-allocation path's device error word on the current device
 * (synchronises `stream`).  Returns GRINQH_OK, or GRINQH_ERR_DEVICE with the
 * code in grinqh_last_error(); in that case it also clears the word and the
 * split-K state a failed call may have left. */
int grinqh_noalloc_check_device_error(void *stream);

/* Device address and size in bytes of the no-allocation path's fixed array on
 * the current device, for inspection and tests (the library owns its
 * contents: the error word is the first int). */
int grinqh_noalloc_scratch(void **ptr, size_t *bytes);

#ifdef __cplusplus
}
#endif

#endif /* GRINQH_H */
