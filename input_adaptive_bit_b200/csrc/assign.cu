// assign.cu -- runtime precision assignment and row compaction.
//
// "GRINQH: Graded Input-Based Quantization Hierarchy", Key design 1: each
// input channel's |x_i| is compared with the layer's static increasing
// thresholds; the number of thresholds at or below |x_i| picks its bit width
// b_i in {0, 2, ..., b_max}; a b_i = 0 channel's weight row is never loaded.
// Key design 3 supplies phi, folded here into the per-group sums.
//
// One CTA of 8 warps per 1024 input channels; warp w owns group g = 8c + w
// (128 channels, 4 per lane).  Per plane p the warp ballots "b_i > 2p" for its
// four 32-channel blocks; popc of the ballots gives each row's position inside
// the group.  The offset of the group inside the global per-plane lists needs
// the counts of every earlier channel: each CTA recounts them directly from x
// (a few tens of KB at most), so no CTA ever waits for another.
//
// Outputs: b, the per-plane lists and counts (the observable contract), the
// group sums X_g / Phi_g, and, in the workspace, the unit stream that the GEMV
// walks: every (row, plane) pair with b_row > 2*plane, ordered by group, then
// plane, then row, each with its scaled input x_row * 4^(P-1-plane).
#include "grinqh_internal.cuh"

namespace grinqh {
namespace {

constexpr int kWarps = kAssignThreads / 32;

struct AssignArgs {
  const uint16_t *x;
  const float *theta;
  const float *phi;  // may be null: default table
  int d_in, b_max, P, G;
  uint8_t *b;
  int32_t *lists;
  int32_t *counts;
  float *grp_sums;
  WsHeader *hdr;
  int32_t *unit_code;
  float *unit_x;
};

__device__ __forceinline__ int level_count(float a, const float (&th)[4], int P) {
  int c = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k) c += (k < P && th[k] <= a) ? 1 : 0;  // NaN: every test false
  return c;
}

__device__ __forceinline__ float half_bits_to_float(uint16_t h) {
  return __half2float(__ushort_as_half(h));
}

__global__ void __launch_bounds__(kAssignThreads) assign_kernel(AssignArgs a) {
  __shared__ int s_prefix[kWarps][4];   // per-warp partial counts of earlier channels
  __shared__ int s_gcnt[kWarps][4];     // per-warp (group) counts per plane
  const int P = a.P;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // x may be written by the kernel launched just before (the previous layer):
  // wait for it, then let the GEMV that consumes our outputs launch early.
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");

  float th[4], phi[5];
#pragma unroll
  for (int k = 0; k < 4; ++k) th[k] = (k < P) ? a.theta[k] : 0.0f;
#pragma unroll
  for (int k = 0; k <= 4; ++k) {
    float def = (2 * k < a.b_max) ? __int_as_float((127 + a.b_max - 2 * k - 1) << 23) : 0.0f;
    phi[k] = (k <= P) ? (a.phi ? a.phi[k] : def) : 0.0f;
  }

  // ---- counts of every channel before this CTA's chunk, per plane ----------
  const int chunk0 = blockIdx.x * kAssignChunk;
  int pre[4] = {0, 0, 0, 0};
  {
    // 8 fp16 per 128-bit load; chunk0 is a multiple of 1024 so loads stay aligned
    const uint4 *xv = reinterpret_cast<const uint4 *>(a.x);
    for (int v = threadIdx.x; v < chunk0 / 8; v += kAssignThreads) {
      const uint4 pk = xv[v];
      const uint32_t w4[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint16_t h = (uint16_t)(w4[e >> 1] >> (16 * (e & 1)));
        const int c = level_count(fabsf(half_bits_to_float(h)), th, P);
#pragma unroll
        for (int p = 0; p < 4; ++p) pre[p] += (c > p) ? 1 : 0;
      }
    }
#pragma unroll
    for (int p = 0; p < 4; ++p) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) pre[p] += __shfl_xor_sync(0xffffffffu, pre[p], off);
    }
    if (lane == 0) {
#pragma unroll
      for (int p = 0; p < 4; ++p) s_prefix[warp][p] = pre[p];
    }
  }

  // ---- this warp's group ------------------------------------------------------
  const int g = blockIdx.x * kWarps + warp;
  const bool has_group = g < a.G;
  int cnt[4];
  uint32_t mask[4][4];  // [block r][plane p]
  float xf[4];
  int gc[4] = {0, 0, 0, 0};
  if (has_group) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int i = g * kGroup + 32 * r + lane;
      const uint16_t h = a.x[i];
      xf[r] = half_bits_to_float(h);
      cnt[r] = level_count(fabsf(xf[r]), th, P);
      a.b[i] = (uint8_t)(2 * cnt[r]);
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        mask[r][p] = __ballot_sync(0xffffffffu, cnt[r] > p);
        gc[p] += __popc(mask[r][p]);
      }
    }
    // X_g, Phi_g in the fixed order of group_sums8 (16 lanes x 8 rows), the
    // order the fused decode kernel uses too; lanes 16-31 repeat lanes 0-15
    __half2 t2[4];
    make_thresholds(a.theta, P, t2);
    const uint4 xw =
        __ldg(reinterpret_cast<const uint4 *>(a.x + g * kGroup + 8 * (lane & 15)));
    uint32_t mk[4];
    plane_masks8(xw, t2, P, mk);
    float X, Phi;
    group_sums8(xw, mk, phi, X, Phi);
    if (lane == 0) {
      a.grp_sums[g] = X;
      a.grp_sums[a.G + g] = Phi;
    }
  }
  if (lane == 0) {
#pragma unroll
    for (int p = 0; p < 4; ++p) s_gcnt[warp][p] = gc[p];
  }
  __syncthreads();

  // global list offsets of this group per plane, and its unit offset
  int loff[4], uoff = 0;
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    int v = 0;
    for (int w = 0; w < kWarps; ++w) v += s_prefix[w][p];  // earlier CTAs
    for (int w = 0; w < warp; ++w) v += s_gcnt[w][p];       // earlier groups of this CTA
    loff[p] = v;
    uoff += (p < P) ? v : 0;
  }

  if (has_group) {
    // units of plane p start after the units of planes < p of this group
    int ubase[4];
    int acc = uoff;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      ubase[p] = acc;
      acc += (p < P) ? gc[p] : 0;
    }
    const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      if (p >= P) break;
      const float scale = __int_as_float((127 + 2 * (P - 1 - p)) << 23);  // 4^(P-1-p)
      int run = 0;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int i = g * kGroup + 32 * r + lane;
        if (cnt[r] > p) {
          const int pos = run + __popc(mask[r][p] & lt);
          a.lists[(size_t)p * a.d_in + loff[p] + pos] = i;
          const int first = (p == 0 && pos == 0) ? 1 : 0;
          a.unit_code[ubase[p] + pos] = (i << 3) | (first << 2) | p;
          a.unit_x[ubase[p] + pos] = xf[r] * scale;
        }
        run += __popc(mask[r][p]);
      }
    }
  }

  // the last CTA knows the totals
  if (blockIdx.x == gridDim.x - 1 && threadIdx.x == 0) {
    int total_units = 0;
    for (int p = 0; p < P; ++p) {
      int v = 0;
      for (int w = 0; w < kWarps; ++w) v += s_prefix[w][p] + s_gcnt[w][p];
      a.counts[p] = v;
      total_units += v;
    }
    a.hdr->total_units = total_units;
    a.hdr->d_in = a.d_in;
    a.hdr->b_max = a.b_max;
  }
}

}  // namespace

cudaError_t launch_assign(const uint16_t *x, const float *theta, int d_in, int b_max,
                          const float *phi, uint8_t *b, int32_t *lists, int32_t *counts,
                          float *grp_sums, void *ws, cudaStream_t st) {
  AssignArgs a;
  const WsLayout L = ws_layout(d_in, 16, b_max);  // stream offsets do not depend on d_out
  a.x = x;
  a.theta = theta;
  a.phi = phi;
  a.d_in = d_in;
  a.b_max = b_max;
  a.P = b_max / 2;
  a.G = d_in / kGroup;
  a.b = b;
  a.lists = lists;
  a.counts = counts;
  a.grp_sums = grp_sums;
  a.hdr = reinterpret_cast<WsHeader *>(ws);
  a.unit_code = reinterpret_cast<int32_t *>(static_cast<char *>(ws) + L.unit_code);
  a.unit_x = reinterpret_cast<float *>(static_cast<char *>(ws) + L.unit_x);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((d_in + kAssignChunk - 1) / kAssignChunk);
  cfg.blockDim = dim3(kAssignThreads);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, assign_kernel, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace grinqh
