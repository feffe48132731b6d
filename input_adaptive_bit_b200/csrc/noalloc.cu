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
// output -- the split-K partial sums and the device error word -- in one
// fixed-size array that the library reserves
// on every GPU that loads it and holds until the process exits.
#include <mutex>

#include "grinqh_internal.cuh"

namespace grinqh {
namespace {

// Scratch layout: the error word (a 256-byte header), then the split-K partial
// words of up to kMaxCtas CTAs (zero between calls).  None of it depends on the
// shape, so the scratch serves every shape grinqh_decode_gemv takes.
constexpr size_t kNaPartials = 256;
constexpr size_t kNoAllocBytes = kNaPartials + (size_t)kMaxCtas * 1024 * 4;  // about 1 MB
static_assert(kNaPartials % 256 == 0, "aligned regions");

// The scratch.  In host code this name is only a host-side stand-in; kernels
// get the device address from cudaGetSymbolAddress.
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
  // every check first: nothing is queued on a failed call
  const int rc = check_decode_args(planes, s, z, x, theta, phi, d_in, d_out, b_max, y, nullptr,
                                   nullptr, nullptr, "grinqh_decode_gemv_noalloc");
  if (rc != GRINQH_OK) return rc;
  void *base = nullptr;
  cudaError_t e = scratch_address(&base);
  if (e != cudaSuccess)
    return record_error(GRINQH_ERR_CUDA, "grinqh_decode_gemv_noalloc: scratch address: %s",
                        cudaGetErrorString(e));
  char *sc = static_cast<char *>(base);
  // Every call shares the array.  A completed call leaves its partial words at
  // zero; the error word keeps the first error until it is read (and the read
  // clears the whole array again).
  e = launch_decode_split(planes, s, z, x, theta, phi, d_in, d_out, b_max, y, nullptr, nullptr,
                          nullptr, nullptr, reinterpret_cast<float *>(sc + kNaPartials),
                          reinterpret_cast<int *>(sc), (cudaStream_t)stream);
  if (e != cudaSuccess)
    return record_error(GRINQH_ERR_CUDA, "grinqh_decode_gemv_noalloc launch: %s",
                        cudaGetErrorString(e));
  return record_error(GRINQH_OK, "");
}

extern "C" int grinqh_noalloc_check_device_error(void *stream) {
  using namespace grinqh;
  void *base = nullptr;
  cudaError_t e = scratch_address(&base);
  if (e != cudaSuccess)
    return record_error(GRINQH_ERR_CUDA, "grinqh_noalloc_check_device_error: scratch address: %s",
                        cudaGetErrorString(e));
  cudaStream_t st = (cudaStream_t)stream;
  int code = 0;
  e = cudaMemcpyAsync(&code, base, sizeof code, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess && code != 0) {
    // clear the error word and the split-K words a failed call may have left
    e = cudaMemsetAsync(base, 0, kNoAllocBytes, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  }
  if (e != cudaSuccess)
    return record_error(GRINQH_ERR_CUDA, "grinqh_noalloc_check_device_error: %s",
                        cudaGetErrorString(e));
  if (code != 0) return record_error(GRINQH_ERR_DEVICE, "device error code %d", code);
  return record_error(GRINQH_OK, "");
}

extern "C" int grinqh_noalloc_scratch(void **ptr, size_t *bytes) {
  using namespace grinqh;
  if (ptr == nullptr || bytes == nullptr)
    return record_error(GRINQH_ERR_INVALID_ARG, "grinqh_noalloc_scratch: ptr and bytes must not be NULL");
  void *base = nullptr;
  cudaError_t e = scratch_address(&base);
  if (e != cudaSuccess)
    return record_error(GRINQH_ERR_CUDA, "grinqh_noalloc_scratch: scratch address: %s",
                        cudaGetErrorString(e));
  *ptr = base;
  *bytes = kNoAllocBytes;
  return record_error(GRINQH_OK, "");
}
