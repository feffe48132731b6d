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

// Device error codes written to the workspace error word.
constexpr int kDevErrStreamMismatch = 1;  // gemv saw a unit stream of another d_in / b_max
constexpr int kDevErrBadUnit = 2;         // a unit record outside [0, d_in) x [0, P) (skipped)

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

// Workspace layout.  The header and the split-K counters sit at fixed offsets
// for every shape, so one workspace can serve layers of different shapes in
// turn: the counters return to zero after every gemv, whatever its shape.
struct WsLayout {
  size_t counters;    // uint32 [kMaxTiles]: split-K arrival counters (fixed offset)
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
  L.unit_code = align256(L.counters + (size_t)kMaxTiles * 4);
  L.unit_x = align256(L.unit_code + n_units * 4);
  L.stream_end = align256(L.unit_x + n_units * 4);
  L.partials = L.stream_end;
  L.total = align256(L.partials + (size_t)kMaxCtas * 2 * kTileOut * 4);
  return L;
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
cudaError_t launch_pack_dense4(const uint8_t *q4, int d_in, int d_out, uint32_t *w4,
                               cudaStream_t st);
size_t dense4_ws_bytes(int d_in, int d_out);
cudaError_t launch_gemv_dense4(const uint32_t *w4, const uint16_t *s, const uint16_t *z,
                               const uint16_t *x, int d_in, int d_out, float *y, void *ws,
                               cudaStream_t st);

}  // namespace grinqh
