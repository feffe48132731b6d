// grinqh_internal.cuh -- definitions shared by the CUDA sources of libgrinqh.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "grinqh.h"

namespace grinqh {

constexpr int kGroup = 128;            // rows per (s, z) group
constexpr int kTileOut = 512;          // outputs per gemv CTA tile
constexpr int kTileWords = kTileOut / 16;
constexpr int kAssignChunk = 1024;     // input channels per assign CTA (8 groups)
constexpr int kAssignThreads = 256;    // one warp per group
constexpr int kMaxCtaUnits = 8192;     // bound on units per gemv CTA (sets the split floor)
constexpr int kNumSMs = 148;
constexpr int kMaxTiles = (1 << 24) / kTileOut;  // d_out <= 2^24
constexpr int kMaxCtas = 256;                   // gemv grid: one CTA per SM, at most this many
constexpr int kDecodeTileOut = 1024;            // outputs per tile of the fused decode kernel
constexpr int kDecodeMaxDin = 65536;            // largest d_in of the fused decode kernel

// Device error codes written to the workspace error word.
constexpr int kDevErrStreamMismatch = 1;  // gemv saw a unit stream of another d_in / b_max
constexpr int kDevErrBadUnit = 2;         // a unit record outside [0, d_in) x [0, P) (skipped)
constexpr int kDevErrSplitKTimeout = 3;   // decode: a split-K wait gave up, or a partial word
                                          // was not zero before the launch (see decode.cu)
constexpr int kDevErrPrefillTimeout = 4;  // prefill: a wait on the tensor cores gave up
constexpr int kDevErrPipeTimeout = 5;     // decode: a wait on the copy/MMA pipeline gave up

// Workspace header (first 256 bytes of the workspace).
struct WsHeader {
  int error;        // first device error code (0 = none)
  int total_units;  // U = sum over rows of b_i/2, written by assign
  int d_in;         // shape of the assign call that wrote the stream
  int b_max;
  int pad[60];
};
static_assert(sizeof(WsHeader) == 256, "header size");

inline __host__ __device__ size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Workspace layout.  The header, the split-K counters of grinqh_gemv and the
// split-K partial words of the fused decode sit at fixed offsets for every
// shape, so one workspace can serve layers of different shapes in turn: the
// counters and the decode's partial words return to zero after every call,
// whatever its shape.
struct WsLayout {
  size_t counters;    // uint32 [kMaxTiles]: split-K arrival counters (fixed offset)
  size_t dpartials;   // u32 [kMaxCtas][kDecodeTileOut]: the fused decode's tagged partial
                      // words (fixed offset; zero between calls)
  size_t unit_code;   // int32 [P * d_in]: row << 3 | first_of_group << 2 | plane
  size_t unit_x;      // fp32 [P * d_in]: x_row * 4^(P-1-plane)
  size_t stream_end;  // end of what grinqh_assign writes
  size_t partials;    // fp32 [kMaxCtas][2][kTileOut]: partial tile segments of gemv CTAs
  size_t total;
  int tiles;
};

inline WsLayout ws_layout(int d_in, int d_out, int b_max) {
  WsLayout L;
  int P = b_max / 2;
  size_t n_units = (size_t)d_in * P;
  L.tiles = (d_out + kTileOut - 1) / kTileOut;
  L.counters = sizeof(WsHeader);
  L.dpartials = align256(L.counters + (size_t)kMaxTiles * 4);
  L.unit_code = align256(L.dpartials + (size_t)kMaxCtas * kDecodeTileOut * 4);
  L.unit_x = align256(L.unit_code + n_units * 4);
  L.stream_end = align256(L.unit_x + n_units * 4);
  L.partials = L.stream_end;
  L.total = align256(L.partials + (size_t)kMaxCtas * 2 * kTileOut * 4);
  return L;
}

// End of the workspace's fixed-offset part (header, counters, decode partial words):
// every call leaves it zero except the error word; after a device error it is
// cleared again.
inline size_t ws_fixed_end() { return ws_layout(128, 16, 2).unit_code; }

// ---- precision assignment on 8 consecutive rows (shared by assign and decode) --------
//
// b_i = 2 #{k : theta_k <= |x_i|}.  With the thresholds sorted ascending (NaN
// last: a NaN threshold never counts), b_i > 2p holds exactly when the p-th
// smallest threshold is <= |x_i|; and since |x_i| is an fp16 value, |x_i| >=
// theta holds exactly when |x_i| >= (theta rounded up to fp16).  So one packed
// fp16 comparison per two rows and plane gives the plane masks bit-exactly.

// Sorted, fp16-rounded-up thresholds from the P raw values in th (entries past P
// must be NaN, as must NaN thresholds stay): ascending, NaN last.
__device__ __forceinline__ void sort_thresholds(float (&th)[4], __half2 (&t2)[4]) {
  auto cs = [](float &x, float &y) {
    const bool sw = (x != x) ? (y == y) : (y < x);
    if (sw) {
      const float t = x;
      x = y;
      y = t;
    }
  };
  cs(th[0], th[1]);
  cs(th[2], th[3]);
  cs(th[0], th[2]);
  cs(th[1], th[3]);
  cs(th[1], th[2]);
#pragma unroll
  for (int k = 0; k < 4; ++k) t2[k] = __half2half2(__float2half_ru(th[k]));
}

// Sorted, fp16-rounded-up thresholds; entries past P (and NaN thresholds) are NaN.
__device__ __forceinline__ void make_thresholds(const float *theta, int P, __half2 (&t2)[4]) {
  float th[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) th[k] = (k < P) ? theta[k] : __int_as_float(0x7fc00000);
  sort_thresholds(th, t2);
}

// mask[p] bit e = (row e of the 8 rows in xw has b > 2p); rows in memory order.
__device__ __forceinline__ void plane_masks8(uint4 xw, const __half2 (&t2)[4], int P,
                                             uint32_t (&mask)[4]) {
  const uint32_t w[4] = {xw.x & 0x7fff7fffu, xw.y & 0x7fff7fffu, xw.z & 0x7fff7fffu,
                         xw.w & 0x7fff7fffu};
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    uint32_t v = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      v |= (__hge2_mask(*reinterpret_cast<const __half2 *>(&w[j]), t2[p]) & 0x00010001u) << (2 * j);
    mask[p] = (p < P) ? ((v | (v >> 15)) & 0xFFu) : 0u;
  }
}

// The mask of one plane: bit e = (row e has b > 2p), t = that plane's threshold.
__device__ __forceinline__ uint32_t plane_mask8(uint4 xw, __half2 t) {
  const uint32_t w[4] = {xw.x & 0x7fff7fffu, xw.y & 0x7fff7fffu, xw.z & 0x7fff7fffu,
                         xw.w & 0x7fff7fffu};
  uint32_t v = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j)
    v |= (__hge2_mask(*reinterpret_cast<const __half2 *>(&w[j]), t) & 0x00010001u) << (2 * j);
  return (v | (v >> 15)) & 0xFFu;
}

// Level (b/2) of row e from its plane masks.
__device__ __forceinline__ int row_level(const uint32_t (&mask)[4], int e) {
  return (int)(((mask[0] >> e) & 1u) + ((mask[1] >> e) & 1u) + ((mask[2] >> e) & 1u) +
               ((mask[3] >> e) & 1u));
}

__device__ __forceinline__ float pick_phi(const float (&phi)[5], int k) {
  float r = phi[0];
#pragma unroll
  for (int j = 1; j < 5; ++j) r = (k == j) ? phi[j] : r;
  return r;
}

// X_g = sum of x and Phi_g = sum of x phi_{b/2} over the active rows of a
// 128-row group held by 16 consecutive lanes (8 rows each): each lane sums its
// rows in order, then the 16 lanes are added pairwise (xor 8, 4, 2, 1).  Every
// lane of the warp must call it (the shuffles span the whole warp).
__device__ __forceinline__ void group_sums8(uint4 xw, const uint32_t (&mask)[4],
                                            const float (&phi)[5], float &X, float &Phi) {
  const uint32_t w[4] = {xw.x, xw.y, xw.z, xw.w};
  float xs = 0.0f, ps = 0.0f;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int lev = row_level(mask, e);
    const float xv = __half2float(__ushort_as_half((uint16_t)(w[e >> 1] >> (16 * (e & 1)))));
    if (lev > 0) {
      xs += xv;
      ps = __fmaf_rn(xv, pick_phi(phi, lev), ps);
    }
  }
#pragma unroll
  for (int off = 8; off > 0; off >>= 1) {
    xs += __shfl_xor_sync(0xffffffffu, xs, off);
    ps += __shfl_xor_sync(0xffffffffu, ps, off);
  }
  X = xs;
  Phi = ps;
}

// Sets the calling thread's message (grinqh_last_error) and returns `code`.
int record_error(int code, const char *fmt, ...);

// Raises a kernel's dynamic shared memory limit to `bytes`, once per device
// and kernel (the attribute is per device context).
cudaError_t ensure_smem_attr(const void *kernel, size_t bytes);

// Launchers (host side, defined in the .cu files).  They assume validated
// arguments and return the cudaError_t of the launch.
cudaError_t launch_pack(const uint8_t *q, int d_in, int d_out, int b_max, uint32_t *planes,
                        cudaStream_t st);
cudaError_t launch_unpack(const uint32_t *planes, int d_in, int d_out, int b_max, uint8_t *q,
                          cudaStream_t st);
cudaError_t launch_assign(const uint16_t *x, const float *theta, int d_in, int b_max,
                          const float *phi, uint8_t *b, int32_t *lists, int32_t *counts,
                          float *grp_sums, void *ws, cudaStream_t st);
cudaError_t launch_gemv(const uint32_t *planes, const uint16_t *s, const uint16_t *z,
                        const float *grp_sums, int d_in, int d_out, int b_max, float *y,
                        void *ws, cudaStream_t st);
cudaError_t launch_decode(const uint32_t *planes, const uint16_t *s, const uint16_t *z,
                          const uint16_t *x, const float *theta, const float *phi, int d_in,
                          int d_out, int b_max, float *y, uint8_t *b, int32_t *lists,
                          int32_t *counts, float *grp_sums, void *ws, cudaStream_t st);
// The same launch with the split-K state at explicit addresses: `partials`
// (kMaxCtas x 1024 words, zero; left zero) and the device error word.
cudaError_t launch_decode_split(const uint32_t *planes, const uint16_t *s, const uint16_t *z,
                                const uint16_t *x, const float *theta, const float *phi, int d_in,
                                int d_out, int b_max, float *y, uint8_t *b, int32_t *lists,
                                int32_t *counts, float *grp_sums, float *partials, int *error,
                                cudaStream_t st);
// Argument checks of grinqh_decode_gemv (everything but the workspace): GRINQH_OK
// or the status it returns, with the message set.
int check_decode_args(const uint32_t *planes, const uint16_t *s, const uint16_t *z,
                      const uint16_t *x, const float *theta, const float *phi, int d_in, int d_out,
                      int b_max, const float *y, const int32_t *lists, const int32_t *counts,
                      const float *grp_sums, const char *who);
cudaError_t launch_decode_group(int n, const grinqh_linear *lins, void *ws, cudaStream_t st);
size_t batch_ws_bytes();
cudaError_t launch_decode_batch(const uint32_t *planes, const uint16_t *s, const uint16_t *z,
                                const uint16_t *x, const float *theta, const float *phi, int B,
                                int d_in, int d_out, int b_max, float *y, uint8_t *u, void *ws,
                                cudaStream_t st);
size_t group_ws_bytes();
cudaError_t launch_prefill(const uint32_t *planes, const uint16_t *s, const uint16_t *z,
                           const uint16_t *x, const float *phi, int T, int d_in, int d_out,
                           int b_max, float *y, void *ws, cudaStream_t st);
size_t prefill_ws_bytes();
cudaError_t launch_pack_dense4(const uint8_t *q4, int d_in, int d_out, uint32_t *w4,
                               cudaStream_t st);
size_t dense4_ws_bytes(int d_in, int d_out);
cudaError_t launch_gemv_dense4(const uint32_t *w4, const uint16_t *s, const uint16_t *z,
                               const uint16_t *x, int d_in, int d_out, float *y, void *ws,
                               cudaStream_t st);

}  // namespace grinqh
