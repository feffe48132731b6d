// noalloc.cu -- grinqh_decode_gemv_noalloc: the decode GEMV with no device
// allocation at all, for callers that cannot allocate device memory.
//
// Some hosts hand a library a stream and the tensors they own and nothing
// else: an inference server or game engine that manages every byte of device
// memory itself and does not let plug-ins call cudaMalloc, or a latency-
// critical path that must never reach the allocator (cudaMalloc can
// synchronise the device).  Such a caller cannot provide the workspace that
// grinqh_decode_gemv needs.  This entry point runs the fused decode kernel
// (without its optional outputs) and keeps what is neither an input nor the
// output -- the split-K partial sums, their arrival counters and the error
// word -- in one fixed-size array that the library reserves on every GPU that
// loads it and holds until the process exits.
#include <mutex>

#include "grinqh_internal.cuh"

namespace grinqh {
namespace {

constexpr int kNoAllocMaxDin = 32768;   // largest d_in this entry point accepts
constexpr int kNoAllocMaxDout = 32768;  // largest d_out

constexpr size_t a256(size_t v) { return (v + 255) & ~size_t(255); }
// The workspace layout of grinqh_workspace_bytes at the largest accepted shape
// (header, counters, the two-call path's unit stream, partial sums).
constexpr size_t kNoAllocBytes =
    a256(a256(a256(a256(sizeof(WsHeader) + (size_t)kMaxTiles * 4) + (size_t)kNoAllocMaxDin * 16) +
              (size_t)kNoAllocMaxDin * 16) +
         (size_t)kMaxCtas * 2 * kTileOut * 4);

// The scratch (about 2.2 MB).  In host code this name is only a host-side
// stand-in; kernels get the device address from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

std::mutex g_mu;
void *g_addr[64] = {nullptr};

// Device address of the scratch on the current device, looked up once per
// device while that device is current.
cudaError_t scratch_address(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_addr[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace grinqh

extern "C" int grinqh_decode_gemv_noalloc(const uint32_t *planes, const uint16_t *s,
                                          const uint16_t *z, const uint16_t *x,
                                          const float *theta, const float *phi, int d_in,
                                          int d_out, int b_max, float *y, void *stream) {
  using namespace grinqh;
  if (grinqh_workspace_bytes(d_in, d_out, b_max) == 0)
    return GRINQH_ERR_UNSUPPORTED_SHAPE;  // message set by the shape check
  if (d_in > kNoAllocMaxDin || d_out > kNoAllocMaxDout)
    return record_error(GRINQH_ERR_UNSUPPORTED_SHAPE,
                        "grinqh_decode_gemv_noalloc: d_in and d_out must be <= 32768 (its fixed "
                        "scratch); got d_in=%d d_out=%d",
                        d_in, d_out);
  void *base = nullptr;
  cudaError_t e = scratch_address(&base);
  if (e != cudaSuccess)
    return record_error(GRINQH_ERR_CUDA, "grinqh_decode_gemv_noalloc: scratch address: %s",
                        cudaGetErrorString(e));
  char *sc = static_cast<char *>(base);
  // Every call shares the array, which keeps the last call's contents.  The
  // kernel leaves its counters at zero, but the error word and the counters of a
  // call that gave up would stay set: they are cleared first.  (The clear also
  // keeps the kernel from overlapping the kernel before it on the stream.)
  const WsLayout L = ws_layout(d_in, d_out, b_max);
  e = cudaMemsetAsync(sc, 0, L.counters + (size_t)L.tiles * 4, (cudaStream_t)stream);
  if (e != cudaSuccess)
    return record_error(GRINQH_ERR_CUDA, "grinqh_decode_gemv_noalloc: clearing scratch: %s",
                        cudaGetErrorString(e));
  return grinqh_decode_gemv(planes, s, z, x, theta, phi, d_in, d_out, b_max, y, nullptr, nullptr,
                            nullptr, nullptr, sc, kNoAllocBytes, stream);
}
