// pack.cu -- offline bit-plane interleaving of b_max-bit codes ("GRINQH:
// Graded Input-Based Quantization Hierarchy", Key design 2: each code is cut
// into 2-bit slices stacked from most to least significant, the matrix is
// stored reduction-dimension major, 16 slices share one 32-bit word).
//
// One thread per (row i, word j): it reads the 16 codes of outputs
// 16j..16j+15 with one 128-bit load and writes one word per plane.  Every
// plane write is coalesced across the threads of a row.
#include "grinqh_internal.cuh"

namespace grinqh {
namespace {

__global__ void __launch_bounds__(256) pack_kernel(const uint8_t *__restrict__ q, int d_in,
                                                   int d_out, int P,
                                                   uint32_t *__restrict__ planes) {
  const int W = d_out >> 4;
  const long long total = (long long)d_in * W;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const long long i = idx / W;
    const int j = (int)(idx - i * W);
    const uint4 c = *reinterpret_cast<const uint4 *>(q + i * d_out + 16 * j);
    const uint32_t cw[4] = {c.x, c.y, c.z, c.w};  // 4 codes per 32-bit lane, low byte first
    for (int p = 0; p < P; ++p) {
      const int sh = 2 * (P - 1 - p);  // bit offset of this plane's slice inside a code
      uint32_t word = 0;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t slice = (cw[k] >> (8 * e + sh)) & 3u;
          word |= slice << (2 * (4 * k + e));
        }
      }
      planes[(i * P + p) * W + j] = word;
    }
  }
}

__global__ void __launch_bounds__(256) unpack_kernel(const uint32_t *__restrict__ planes,
                                                     int d_in, int d_out, int P,
                                                     uint8_t *__restrict__ q) {
  const int W = d_out >> 4;
  const long long total = (long long)d_in * W;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const long long i = idx / W;
    const int j = (int)(idx - i * W);
    uint32_t cw[4] = {0u, 0u, 0u, 0u};
    for (int p = 0; p < P; ++p) {
      const uint32_t word = planes[(i * P + p) * W + j];
      const int sh = 2 * (P - 1 - p);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t slice = (word >> (2 * (4 * k + e))) & 3u;
          cw[k] |= slice << (8 * e + sh);
        }
      }
    }
    *reinterpret_cast<uint4 *>(q + i * d_out + 16 * j) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
  }
}

int grid_for(long long work) {
  long long blocks = (work + 255) / 256;
  const long long cap = 148LL * 16;
  return (int)(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

}  // namespace

cudaError_t launch_pack(const uint8_t *q, int d_in, int d_out, int b_max, uint32_t *planes,
                        cudaStream_t st) {
  pack_kernel<<<grid_for((long long)d_in * (d_out / 16)), 256, 0, st>>>(q, d_in, d_out,
                                                                        b_max / 2, planes);
  return cudaGetLastError();
}

cudaError_t launch_unpack(const uint32_t *planes, int d_in, int d_out, int b_max, uint8_t *q,
                          cudaStream_t st) {
  unpack_kernel<<<grid_for((long long)d_in * (d_out / 16)), 256, 0, st>>>(planes, d_in, d_out,
                                                                          b_max / 2, q);
  return cudaGetLastError();
}

}  // namespace grinqh
