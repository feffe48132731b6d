// api.cu -- the extern "C" boundary of libgrinqh: argument checks, status
// codes, the per-thread error message, and dispatch to the launchers.
#include <stdarg.h>
#include <stdio.h>

#include <atomic>

#include "grinqh_internal.cuh"

namespace {

thread_local char g_msg[512];

int fail(int code, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof g_msg, fmt, ap);
  va_end(ap);
  return code;
}

int ok() {
  g_msg[0] = '\0';
  return GRINQH_OK;
}

int cuda_status(cudaError_t e, const char *what) {
  if (e != cudaSuccess) return fail(GRINQH_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return ok();
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_bmax(int b_max) {
  if (b_max != 2 && b_max != 4 && b_max != 6 && b_max != 8)
    return fail(GRINQH_ERR_INVALID_ARG, "b_max must be 2, 4, 6 or 8 (got %d)", b_max);
  return GRINQH_OK;
}

int check_din(int d_in) {
  if (d_in < 128 || d_in > (1 << 24) || d_in % 128 != 0)
    return fail(GRINQH_ERR_UNSUPPORTED_SHAPE,
                "d_in must be a multiple of 128 in [128, 2^24] (got %d)", d_in);
  return GRINQH_OK;
}

int check_dout(int d_out) {
  if (d_out < 16 || d_out > (1 << 24) || d_out % 16 != 0)
    return fail(GRINQH_ERR_UNSUPPORTED_SHAPE,
                "d_out must be a multiple of 16 in [16, 2^24] (got %d)", d_out);
  return GRINQH_OK;
}

int check_ptr(const void *p, size_t align, const char *name) {
  if (p == nullptr) return fail(GRINQH_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned(p, align))
    return fail(GRINQH_ERR_INVALID_ARG, "%s must be %zu-byte aligned", name, align);
  return GRINQH_OK;
}

#define TRY(expr)                   \
  do {                              \
    int _rc = (expr);               \
    if (_rc != GRINQH_OK) return _rc; \
  } while (0)

}  // namespace

namespace grinqh {
int record_error(int code, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof g_msg, fmt, ap);
  va_end(ap);
  return code;
}

int check_decode_args(const uint32_t *planes, const uint16_t *s, const uint16_t *z,
                      const uint16_t *x, const float *theta, const float *phi, int d_in, int d_out,
                      int b_max, const float *y, const int32_t *lists, const int32_t *counts,
                      const float *grp_sums, const char *who) {
  TRY(check_bmax(b_max));
  TRY(check_din(d_in));
  TRY(check_dout(d_out));
  if (d_in > kDecodeMaxDin)
    return fail(GRINQH_ERR_UNSUPPORTED_SHAPE,
                "%s: d_in must be <= %d (got %d); use grinqh_assign + grinqh_gemv", who,
                kDecodeMaxDin, d_in);
  TRY(check_ptr(planes, (d_out / 16) % 4 == 0 ? 16 : 4, "planes"));
  TRY(check_ptr(s, 16, "s"));
  TRY(check_ptr(z, 16, "z"));
  TRY(check_ptr(x, 16, "x"));
  TRY(check_ptr(theta, 4, "theta"));
  if (phi) TRY(check_ptr(phi, 4, "phi"));
  TRY(check_ptr(y, 4, "y"));
  if (lists) TRY(check_ptr(lists, 4, "lists"));
  if (counts) TRY(check_ptr(counts, 4, "counts"));
  if (grp_sums) TRY(check_ptr(grp_sums, 4, "grp_sums"));
  return GRINQH_OK;
}

cudaError_t ensure_smem_attr(const void *kernel, size_t bytes) {
  // One bit per (device, kernel slot); a handful of kernels use this.
  static std::atomic<unsigned long long> done[64];
  static const void *slots[16];
  static std::atomic<int> n_slots{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int slot = -1;
  for (int i = 0; i < n_slots.load(); ++i)
    if (slots[i] == kernel) slot = i;
  if (slot < 0) {
    slot = n_slots.fetch_add(1);
    if (slot >= 16) return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    slots[slot] = kernel;
  }
  const unsigned long long bit = 1ull << slot;
  if (dev < 64 && (done[dev].load() & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess && dev < 64) done[dev].fetch_or(bit);
  return e;
}
}  // namespace grinqh

extern "C" {

int grinqh_version(void) { return 1000; }

const char *grinqh_last_error(void) { return g_msg; }

size_t grinqh_workspace_bytes(int d_in, int d_out, int b_max) {
  if (check_bmax(b_max) || check_din(d_in) || check_dout(d_out)) return 0;
  return grinqh::ws_layout(d_in, d_out, b_max).total;
}

int grinqh_pack(const uint8_t *q, int d_in, int d_out, int b_max, uint32_t *planes,
                void *stream) {
  TRY(check_bmax(b_max));
  TRY(check_din(d_in));
  TRY(check_dout(d_out));
  TRY(check_ptr(q, 16, "q"));
  TRY(check_ptr(planes, 4, "planes"));
  return cuda_status(grinqh::launch_pack(q, d_in, d_out, b_max, planes, (cudaStream_t)stream),
                     "grinqh_pack launch");
}

int grinqh_unpack(const uint32_t *planes, int d_in, int d_out, int b_max, uint8_t *q_out,
                  void *stream) {
  TRY(check_bmax(b_max));
  TRY(check_din(d_in));
  TRY(check_dout(d_out));
  TRY(check_ptr(planes, 4, "planes"));
  TRY(check_ptr(q_out, 16, "q_out"));
  return cuda_status(
      grinqh::launch_unpack(planes, d_in, d_out, b_max, q_out, (cudaStream_t)stream),
      "grinqh_unpack launch");
}

int grinqh_assign(const uint16_t *x, const float *theta, int d_in, int b_max, const float *phi,
                  uint8_t *b, int32_t *lists, int32_t *counts, float *grp_sums, void *ws,
                  size_t ws_bytes, void *stream) {
  TRY(check_bmax(b_max));
  TRY(check_din(d_in));
  TRY(check_ptr(x, 16, "x"));
  TRY(check_ptr(theta, 4, "theta"));
  if (phi) TRY(check_ptr(phi, 4, "phi"));
  TRY(check_ptr(b, 1, "b"));
  TRY(check_ptr(lists, 4, "lists"));
  TRY(check_ptr(counts, 4, "counts"));
  TRY(check_ptr(grp_sums, 4, "grp_sums"));
  TRY(check_ptr(ws, 256, "ws"));
  const size_t need = grinqh::ws_layout(d_in, 16, b_max).stream_end;  // header + unit stream
  if (ws_bytes < need)
    return fail(GRINQH_ERR_WORKSPACE_TOO_SMALL, "workspace of %zu bytes, assign needs %zu",
                ws_bytes, need);
  return cuda_status(grinqh::launch_assign(x, theta, d_in, b_max, phi, b, lists, counts,
                                           grp_sums, ws, (cudaStream_t)stream),
                     "grinqh_assign launch");
}

int grinqh_gemv(const uint32_t *planes, const uint16_t *s, const uint16_t *z,
                const float *grp_sums, int d_in, int d_out, int b_max, float *y, void *ws,
                size_t ws_bytes, void *stream) {
  TRY(check_bmax(b_max));
  TRY(check_din(d_in));
  TRY(check_dout(d_out));
  TRY(check_ptr(planes, (d_out / 16) % 4 == 0 ? 16 : 4, "planes"));
  TRY(check_ptr(s, 16, "s"));
  TRY(check_ptr(z, 16, "z"));
  TRY(check_ptr(grp_sums, 4, "grp_sums"));
  TRY(check_ptr(y, 4, "y"));
  TRY(check_ptr(ws, 256, "ws"));
  const size_t need = grinqh::ws_layout(d_in, d_out, b_max).total;
  if (ws_bytes < need)
    return fail(GRINQH_ERR_WORKSPACE_TOO_SMALL, "workspace of %zu bytes, gemv needs %zu",
                ws_bytes, need);
  return cuda_status(grinqh::launch_gemv(planes, s, z, grp_sums, d_in, d_out, b_max, y, ws,
                                         (cudaStream_t)stream),
                     "grinqh_gemv launch");
}

int grinqh_decode_gemv(const uint32_t *planes, const uint16_t *s, const uint16_t *z,
                       const uint16_t *x, const float *theta, const float *phi, int d_in,
                       int d_out, int b_max, float *y, uint8_t *b, int32_t *lists,
                       int32_t *counts, float *grp_sums, void *ws, size_t ws_bytes,
                       void *stream) {
  TRY(grinqh::check_decode_args(planes, s, z, x, theta, phi, d_in, d_out, b_max, y, lists, counts,
                                grp_sums, "grinqh_decode_gemv"));
  TRY(check_ptr(ws, 256, "ws"));
  const size_t need = grinqh::ws_layout(d_in, d_out, b_max).total;
  if (ws_bytes < need)
    return fail(GRINQH_ERR_WORKSPACE_TOO_SMALL, "workspace of %zu bytes, decode needs %zu",
                ws_bytes, need);
  return cuda_status(grinqh::launch_decode(planes, s, z, x, theta, phi, d_in, d_out, b_max, y,
                                           b, lists, counts, grp_sums, ws,
                                           (cudaStream_t)stream),
                     "grinqh_decode_gemv launch");
}

size_t grinqh_batch_workspace_bytes(void) { return grinqh::batch_ws_bytes(); }

int grinqh_decode_gemv_batch(const uint32_t *planes, const uint16_t *s, const uint16_t *z,
                             const uint16_t *x, const float *theta, const float *phi, int B,
                             int d_in, int d_out, int b_max, float *y, uint8_t *u, void *ws,
                             size_t ws_bytes, void *stream) {
  if (B < 1 || B > GRINQH_MAX_BATCH)
    return fail(GRINQH_ERR_INVALID_ARG, "grinqh_decode_gemv_batch: B must be in [1, %d] (got %d)",
                GRINQH_MAX_BATCH, B);
  TRY(grinqh::check_decode_args(planes, s, z, x, theta, phi, d_in, d_out, b_max, y, nullptr,
                                nullptr, nullptr, "grinqh_decode_gemv_batch"));
  TRY(check_ptr(ws, 256, "ws"));
  if (ws_bytes < grinqh::batch_ws_bytes())
    return fail(GRINQH_ERR_WORKSPACE_TOO_SMALL, "workspace of %zu bytes, batch decode needs %zu",
                ws_bytes, grinqh::batch_ws_bytes());
  return cuda_status(grinqh::launch_decode_batch(planes, s, z, x, theta, phi, B, d_in, d_out,
                                                 b_max, y, u, ws, (cudaStream_t)stream),
                     "grinqh_decode_gemv_batch launch");
}

size_t grinqh_prefill_workspace_bytes(void) { return grinqh::prefill_ws_bytes(); }

int grinqh_prefill_gemm(const uint32_t *planes, const uint16_t *s, const uint16_t *z,
                        const uint16_t *x, const float *phi, int T, int d_in, int d_out,
                        int b_max, float *y, void *ws, size_t ws_bytes, void *stream) {
  TRY(check_bmax(b_max));
  TRY(check_din(d_in));
  TRY(check_dout(d_out));
  if (d_out % 128 != 0)
    return fail(GRINQH_ERR_UNSUPPORTED_SHAPE,
                "grinqh_prefill_gemm: d_out must be a multiple of 128 (got %d)", d_out);
  if (T < 1 || T > 65536)
    return fail(GRINQH_ERR_UNSUPPORTED_SHAPE, "grinqh_prefill_gemm: T must be in [1, 65536] (got %d)",
                T);
  TRY(check_ptr(planes, 16, "planes"));
  TRY(check_ptr(s, 16, "s"));
  TRY(check_ptr(z, 16, "z"));
  TRY(check_ptr(x, 16, "x"));
  if (phi) TRY(check_ptr(phi, 4, "phi"));
  TRY(check_ptr(y, 4, "y"));
  TRY(check_ptr(ws, 256, "ws"));
  if (ws_bytes < grinqh::prefill_ws_bytes())
    return fail(GRINQH_ERR_WORKSPACE_TOO_SMALL, "workspace of %zu bytes, prefill needs %zu",
                ws_bytes, grinqh::prefill_ws_bytes());
  return cuda_status(grinqh::launch_prefill(planes, s, z, x, phi, T, d_in, d_out, b_max, y, ws,
                                            (cudaStream_t)stream),
                     "grinqh_prefill_gemm launch");
}

size_t grinqh_group_workspace_bytes(void) { return grinqh::group_ws_bytes(); }

int grinqh_decode_gemv_group(int n, const grinqh_linear *lins, void *ws, size_t ws_bytes,
                             void *stream) {
  if (n < 1 || n > GRINQH_MAX_GROUP)
    return fail(GRINQH_ERR_INVALID_ARG, "grinqh_decode_gemv_group: n must be in [1, %d] (got %d)",
                GRINQH_MAX_GROUP, n);
  TRY(check_ptr(lins, alignof(grinqh_linear), "lins"));
  long long tiles = 0;
  for (int j = 0; j < n; ++j) {
    const grinqh_linear &l = lins[j];
    TRY(check_bmax(l.b_max));
    TRY(check_din(l.d_in));
    TRY(check_dout(l.d_out));
    if (l.d_in > grinqh::kDecodeMaxDin)
      return fail(GRINQH_ERR_UNSUPPORTED_SHAPE,
                  "grinqh_decode_gemv_group: linear %d: d_in must be <= %d (got %d)", j,
                  grinqh::kDecodeMaxDin, l.d_in);
    TRY(check_ptr(l.planes, (l.d_out / 16) % 4 == 0 ? 16 : 4, "planes"));
    TRY(check_ptr(l.s, 16, "s"));
    TRY(check_ptr(l.z, 16, "z"));
    TRY(check_ptr(l.x, 16, "x"));
    TRY(check_ptr(l.theta, 4, "theta"));
    if (l.phi) TRY(check_ptr(l.phi, 4, "phi"));
    TRY(check_ptr(l.y, 4, "y"));
    tiles += (l.d_out + 1023) / 1024;
  }
  if (tiles > grinqh::kMaxTiles)
    return fail(GRINQH_ERR_UNSUPPORTED_SHAPE, "grinqh_decode_gemv_group: too many output tiles (%lld)",
                tiles);
  TRY(check_ptr(ws, 256, "ws"));
  if (ws_bytes < grinqh::group_ws_bytes())
    return fail(GRINQH_ERR_WORKSPACE_TOO_SMALL, "workspace of %zu bytes, a group needs %zu",
                ws_bytes, grinqh::group_ws_bytes());
  return cuda_status(grinqh::launch_decode_group(n, lins, ws, (cudaStream_t)stream),
                     "grinqh_decode_gemv_group launch");
}

int grinqh_check_device_error(void *ws, void *stream) {
  TRY(check_ptr(ws, 256, "ws"));
  int code = 0;
  const int zero = 0;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemcpyAsync(&code, ws, sizeof code, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess)
    e = code == 0 ? cudaMemcpyAsync(ws, &zero, sizeof zero, cudaMemcpyHostToDevice, st)
                  // a failed call may have left split-K state: clear the fixed-offset part
                  : cudaMemsetAsync(ws, 0, grinqh::ws_fixed_end(), st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  TRY(cuda_status(e, "grinqh_check_device_error"));
  if (code != 0) return fail(GRINQH_ERR_DEVICE, "device error code %d", code);
  return ok();
}

int grinqh_pack_dense4(const uint8_t *q4, int d_in, int d_out, uint32_t *w4, void *stream) {
  TRY(check_din(d_in));
  TRY(check_dout(d_out));
  TRY(check_ptr(q4, 8, "q4"));
  TRY(check_ptr(w4, 4, "w4"));
  return cuda_status(grinqh::launch_pack_dense4(q4, d_in, d_out, w4, (cudaStream_t)stream),
                     "grinqh_pack_dense4 launch");
}

size_t grinqh_dense4_workspace_bytes(int d_in, int d_out) {
  if (check_din(d_in) || check_dout(d_out)) return 0;
  return grinqh::dense4_ws_bytes(d_in, d_out);
}

int grinqh_gemv_dense4(const uint32_t *w4, const uint16_t *s, const uint16_t *z,
                       const uint16_t *x, int d_in, int d_out, float *y, void *ws,
                       size_t ws_bytes, void *stream) {
  TRY(check_din(d_in));
  TRY(check_dout(d_out));
  TRY(check_ptr(w4, (d_out / 8) % 4 == 0 ? 16 : 4, "w4"));
  TRY(check_ptr(s, 16, "s"));
  TRY(check_ptr(z, 16, "z"));
  TRY(check_ptr(x, 2, "x"));
  TRY(check_ptr(y, 4, "y"));
  TRY(check_ptr(ws, 256, "ws"));
  const size_t need = grinqh::dense4_ws_bytes(d_in, d_out);
  if (ws_bytes < need)
    return fail(GRINQH_ERR_WORKSPACE_TOO_SMALL, "workspace of %zu bytes, dense4 needs %zu",
                ws_bytes, need);
  return cuda_status(
      grinqh::launch_gemv_dense4(w4, s, z, x, d_in, d_out, y, ws, (cudaStream_t)stream),
      "grinqh_gemv_dense4 launch");
}

}  // extern "C"
