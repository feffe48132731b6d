// dense4.cu -- in-library dense 4-bit GEMV, the fixed-width comparator.
//
// The GRINQH notes' throughput table ("hardware throughput and ablation")
// measures GRINQH against a 4-bit fixed-width kernel on the same projection.
// This is that comparator rebuilt on the same machinery: every row is read,
// 8 nibbles per 32-bit word, w_hat = s * q4 + z with the same 128-row fp16
// s/z grouping, y = W_hat^T x.  It is not a GRINQH step.
//
// Layout: w4 uint32 [d_in][d_out/8], output 8j+t of row i in bits [4t+3:4t]
// of word j.  CTA (tile of 512 outputs, split) reads a contiguous range of
// rows; a row's tile segment is 256 contiguous bytes, 16 lanes x 16 bytes.
// Nibbles are rebuilt like the 2-bit fields of gemv.cu:
// as_float((w & (15 << 4t)) | 0x4B000000) - 2^23 == nibble * 16^t for t <= 4,
// nibbles 5..7 from w >> 20.
#include "grinqh_internal.cuh"

namespace grinqh {
namespace {

constexpr int kThreads = 256;
constexpr int kWarpsPerCta = kThreads / 32;
constexpr int kStages = 12;
constexpr int kTileWords4 = kTileOut / 8;  // 64 words of 8 nibbles per row and tile
constexpr int kVec = 4;
constexpr int kLanes = kTileWords4 / kVec;  // 16 lanes per row segment
constexpr int kSpw = 32 / kLanes;           // 2 row streams per warp

struct Dense4Args {
  const uint32_t *w4;
  const uint16_t *s, *z, *x;
  float *y;
  int d_in, d_out, W4, splits;
  unsigned *counters;
  float *partials;
};

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}
__device__ __forceinline__ void cp_async16(void *dst, const void *src, int src_bytes) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(d), "l"(src),
               "r"(src_bytes));
}
__device__ __forceinline__ void cp_async4(void *dst, const void *src, int src_bytes) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(d), "l"(src),
               "r"(src_bytes));
}

__device__ __forceinline__ int nib_pos(int t) { return t <= 4 ? t : t - 5; }

__device__ __forceinline__ void accumulate_word4(float (&acc)[8], uint32_t w, float xv) {
  const uint32_t w2 = w >> 20;
  float m[8];
#pragma unroll
  for (int t = 0; t < 8; ++t)
    m[t] = __uint_as_float(((t <= 4 ? w : w2) & (15u << (4 * nib_pos(t)))) | 0x4B000000u);
  const float2 neg = make_float2(-8388608.0f, -8388608.0f);
  const float2 x2 = make_float2(xv, xv);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 f = __fadd2_rn(make_float2(m[2 * k], m[2 * k + 1]), neg);
    const float2 r = __ffma2_rn(x2, f, make_float2(acc[2 * k], acc[2 * k + 1]));
    acc[2 * k] = r.x;
    acc[2 * k + 1] = r.y;
  }
}

__device__ __forceinline__ void load8_half(const uint16_t *p, float (&v)[8]) {
  const uint4 a = *reinterpret_cast<const uint4 *>(p);
  const uint32_t u[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&u[k]));
    v[2 * k] = f.x;
    v[2 * k + 1] = f.y;
  }
}

template <bool ALIGNED>
__global__ void __launch_bounds__(kThreads, 1) dense4_kernel(Dense4Args a) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint32_t *ring = reinterpret_cast<uint32_t *>(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int sub = lane / kLanes, li = lane % kLanes;
  const int tile = blockIdx.x, split = blockIdx.y;
  const int word0 = tile * kTileWords4 + li * kVec;
  const int nvalid = max(0, min(kVec, a.W4 - word0));

  const int r_begin = (int)((long long)split * a.d_in / a.splits);
  const int r_end = (int)((long long)(split + 1) * a.d_in / a.splits);
  const int n = r_end - r_begin;
  const int wa = r_begin + (int)((long long)warp * n / kWarpsPerCta);
  const int wb = r_begin + (int)((long long)(warp + 1) * n / kWarpsPerCta);
  const int first = wa + sub;
  const int count = wb > first ? (wb - first + kSpw - 1) / kSpw : 0;

  float acc[kVec][8], yacc[kVec][8];
#pragma unroll
  for (int v = 0; v < kVec; ++v)
#pragma unroll
    for (int t = 0; t < 8; ++t) acc[v][t] = yacc[v][t] = 0.0f;
  float xsum = 0.0f;
  int g_cur = -1;

  auto issue = [&](int row, int slot) {
    const uint32_t *src = a.w4 + (size_t)row * a.W4 + word0;
    uint32_t *dst = ring + ((size_t)slot * kThreads + tid) * kVec;
    if (ALIGNED) {
      cp_async16(dst, nvalid > 0 ? (const void *)src : (const void *)a.w4, 4 * nvalid);
    } else {
#pragma unroll
      for (int v = 0; v < kVec; ++v)
        cp_async4(dst + v, v < nvalid ? (const void *)(src + v) : (const void *)a.w4,
                  v < nvalid ? 4 : 0);
    }
  };
  auto flush = [&](int g) {
#pragma unroll
    for (int v = 0; v < kVec; ++v) {
      if (v < nvalid) {
        float sv[8], zv[8];
        load8_half(a.s + (size_t)g * a.d_out + 8 * (word0 + v), sv);
        load8_half(a.z + (size_t)g * a.d_out + 8 * (word0 + v), zv);
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const float up = __int_as_float((127 + 4 * nib_pos(t)) << 23);  // 16^pos
          yacc[v][t] = fmaf(sv[t], acc[v][t], fmaf(zv[t] * xsum, up, yacc[v][t]));
        }
      }
#pragma unroll
      for (int t = 0; t < 8; ++t) acc[v][t] = 0.0f;
    }
    xsum = 0.0f;
  };

#pragma unroll
  for (int k = 0; k < kStages - 1; ++k) {
    if (k < count) issue(first + k * kSpw, k);
    cp_async_commit();
  }
  for (int k = 0; k < count; ++k) {
    const int kn = k + kStages - 1;
    if (kn < count) issue(first + kn * kSpw, kn % kStages);
    cp_async_commit();
    cp_async_wait<kStages - 1>();
    const int row = first + k * kSpw;
    const int g = row >> 7;
    if (g != g_cur) {
      if (g_cur >= 0) flush(g_cur);
      g_cur = g;
    }
    const float xv = __half2float(__ushort_as_half(a.x[row]));
    xsum += xv;
    const uint4 q = *reinterpret_cast<const uint4 *>(ring + ((size_t)(k % kStages) * kThreads + tid) * kVec);
    accumulate_word4(acc[0], q.x, xv);
    accumulate_word4(acc[1], q.y, xv);
    accumulate_word4(acc[2], q.z, xv);
    accumulate_word4(acc[3], q.w, xv);
  }
  cp_async_wait<0>();
  if (g_cur >= 0) flush(g_cur);

#pragma unroll
  for (int off = kLanes; off < 32; off <<= 1)
#pragma unroll
    for (int v = 0; v < kVec; ++v)
#pragma unroll
      for (int t = 0; t < 8; ++t) yacc[v][t] += __shfl_xor_sync(0xffffffffu, yacc[v][t], off);

  __syncthreads();
  float *red = reinterpret_cast<float *>(smem);  // [warps][kTileOut]
  if (sub == 0) {
#pragma unroll
    for (int v = 0; v < kVec; ++v)
#pragma unroll
      for (int t = 0; t < 8; t += 4)
        *reinterpret_cast<float4 *>(&red[warp * kTileOut + 8 * (li * kVec + v) + t]) =
            make_float4(yacc[v][t], yacc[v][t + 1], yacc[v][t + 2], yacc[v][t + 3]);
  }
  __syncthreads();

  __shared__ int s_last;
  float val[kTileOut / kThreads];
#pragma unroll
  for (int e = 0; e < kTileOut / kThreads; ++e) {
    const int ol = tid + e * kThreads;
    float sum = 0.0f;
#pragma unroll
    for (int w = 0; w < kWarpsPerCta; ++w) sum += red[w * kTileOut + ol];
    val[e] = sum * __int_as_float((127 - 4 * nib_pos(ol & 7)) << 23);
  }
  const int obase = tile * kTileOut;
  if (a.splits == 1) {
#pragma unroll
    for (int e = 0; e < kTileOut / kThreads; ++e) {
      const int o = obase + tid + e * kThreads;
      if (o < a.d_out) a.y[o] = val[e];
    }
    return;
  }
#pragma unroll
  for (int e = 0; e < kTileOut / kThreads; ++e) {
    const int o = obase + tid + e * kThreads;
    if (o < a.d_out) a.partials[(size_t)split * a.d_out + o] = val[e];
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicInc(&a.counters[tile], (unsigned)(a.splits - 1)) ==
                          (unsigned)(a.splits - 1));
  __syncthreads();
  if (!s_last) return;
  __threadfence();
#pragma unroll
  for (int e = 0; e < kTileOut / kThreads; ++e) {
    const int o = obase + tid + e * kThreads;
    if (o < a.d_out) {
      float sum = 0.0f;
      for (int sp = 0; sp < a.splits; ++sp) sum += __ldcg(&a.partials[(size_t)sp * a.d_out + o]);
      a.y[o] = sum;
    }
  }
}

__global__ void __launch_bounds__(256) pack_dense4_kernel(const uint8_t *__restrict__ q4, int d_in,
                                                          int d_out, uint32_t *__restrict__ w4) {
  const int W4 = d_out >> 3;
  const long long total = (long long)d_in * W4;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const long long i = idx / W4;
    const int j = (int)(idx - i * W4);
    const uint2 c = *reinterpret_cast<const uint2 *>(q4 + i * d_out + 8 * j);
    uint32_t word = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      word |= ((c.x >> (8 * e)) & 15u) << (4 * e);
      word |= ((c.y >> (8 * e)) & 15u) << (4 * (e + 4));
    }
    w4[i * W4 + j] = word;
  }
}

struct Dense4Plan {
  int tiles, splits;
  size_t counters, partials, total;
};

Dense4Plan dense4_plan(int d_in, int d_out) {
  Dense4Plan p;
  p.tiles = (d_out + kTileOut - 1) / kTileOut;
  int s = (2 * kNumSMs) / p.tiles;
  if (s < 1) s = 1;
  if (s > d_in / 32) s = d_in / 32;  // keep >= 32 rows per split
  if (s < 1) s = 1;
  p.splits = s;
  p.counters = 0;
  p.partials = align256((size_t)p.tiles * 4);
  p.total = align256(p.partials + (s > 1 ? (size_t)s * d_out * 4 : 0));
  return p;
}

}  // namespace

size_t dense4_ws_bytes(int d_in, int d_out) { return dense4_plan(d_in, d_out).total; }

cudaError_t launch_pack_dense4(const uint8_t *q4, int d_in, int d_out, uint32_t *w4,
                               cudaStream_t st) {
  long long blocks = ((long long)d_in * (d_out / 8) + 255) / 256;
  if (blocks > 148LL * 16) blocks = 148LL * 16;
  if (blocks < 1) blocks = 1;
  pack_dense4_kernel<<<(int)blocks, 256, 0, st>>>(q4, d_in, d_out, w4);
  return cudaGetLastError();
}

cudaError_t launch_gemv_dense4(const uint32_t *w4, const uint16_t *s, const uint16_t *z,
                               const uint16_t *x, int d_in, int d_out, float *y, void *ws,
                               cudaStream_t st) {
  const Dense4Plan p = dense4_plan(d_in, d_out);
  Dense4Args a;
  char *w = static_cast<char *>(ws);
  a.w4 = w4;
  a.s = s;
  a.z = z;
  a.x = x;
  a.y = y;
  a.d_in = d_in;
  a.d_out = d_out;
  a.W4 = d_out / 8;
  a.splits = p.splits;
  a.counters = reinterpret_cast<unsigned *>(w + p.counters);
  a.partials = reinterpret_cast<float *>(w + p.partials);
  const size_t smem = (size_t)kStages * kThreads * kVec * 4;
  const bool aligned = a.W4 % 4 == 0;
  const void *fn = aligned ? (const void *)dense4_kernel<true> : (const void *)dense4_kernel<false>;
  cudaError_t e = ensure_smem_attr(fn, smem);
  if (e != cudaSuccess) return e;
  if (aligned)
    dense4_kernel<true><<<dim3(p.tiles, p.splits), kThreads, smem, st>>>(a);
  else
    dense4_kernel<false><<<dim3(p.tiles, p.splits), kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace grinqh
