// gemv.cu -- the fused plane-sparse reconstruct-and-GEMV of GRINQH decode.
//
// What it computes ("GRINQH: Graded Input-Based Quantization Hierarchy",
// Method / overall framework, Key designs 2 and 3):
//   y_o = sum_{i : b_i > 0} x_i * (s_{g,o} * (Q_{i,o} + phi_{b_i}) + z_{g,o}),
// where Q is rebuilt from only the first b_i/2 bit planes of row i.
//
// How (B200 design, not the pages' Triton kernel):
//  * Group factorisation.  With A_{g,o} = sum_{i in g, b_i>0} x_i Q_{i,o},
//    y_o = sum_g [ s_{g,o} (A_{g,o} + Phi_g) + z_{g,o} X_g ], so the inner loop
//    is one FMA per 2-bit field: A += (x_i 4^(P-1-p)) * slice, with X_g / Phi_g
//    precomputed by grinqh_assign.
//  * Work = tiles x units, where a unit is one (row, plane) pair of the unit
//    stream of grinqh_assign (ordered by group, plane, row) and a tile is 512
//    outputs, so a (unit, tile) item is one contiguous 128-byte segment of a
//    row's plane region.  The tiles x U items are cut into one equal,
//    contiguous range per SM ("stream-K"): a single wave, balanced whatever
//    the shape or the sparsity pattern.  A range covers whole tiles plus at
//    most two partial tile segments.
//  * Inside a CTA each warp takes a contiguous piece of a round of up to
//    kRoundUnits units and its four 8-lane subgroups take every 4th unit; each
//    lane copies its 16-byte share of a unit into a private shared-memory ring
//    with cp.async (kStages deep), so ~45 KB per SM are in flight without
//    holding registers.  The s/z rows of the round's groups are staged in
//    shared memory alongside, so flushing a group never waits on memory.
//  * Field rebuild without conversions: for field t of word w,
//    as_float((w & (3 << 2t)) | 0x4B000000) - 2^23 == slice * 4^t exactly
//    (IEEE-754 single: exponent 2^23, the slice sits in the mantissa), fields
//    11..15 from w >> 22.  The 4^t factor is removed once per output at the
//    end.  Pairs of fields go through the packed f32x2 add/FMA of sm_100.
//  * Partial tile segments are summed by the last contributing CTA to arrive
//    (atomicInc on a self-resetting per-tile counter) in CTA order, so y is
//    deterministic.  Whole tiles are written directly.
//  * Programmatic dependent launch: the kernel waits on grinqh_assign with
//    griddepcontrol.wait, so its launch overlaps the tail of assign.
#include "grinqh_internal.cuh"

namespace grinqh {
namespace {

constexpr int kThreads = 256;
constexpr int kWarpsPerCta = kThreads / 32;
constexpr int kStages = 12;          // cp.async ring depth per lane
constexpr int kRoundUnits = 1024;    // unit records staged in shared memory per round
constexpr int kRoundGroups = 8;      // s/z rows staged per round
constexpr int kVec = 4;              // words per lane and unit (16 bytes)
constexpr int kLanes = kTileWords / kVec;  // 8 lanes per unit
constexpr int kSpw = 32 / kLanes;          // 4 subgroups per warp

// shared memory map (bytes)
constexpr size_t kSmRecCode = 0;
constexpr size_t kSmRecX = kSmRecCode + kRoundUnits * 4;
constexpr size_t kSmS = kSmRecX + kRoundUnits * 4;
constexpr size_t kSmZ = kSmS + kRoundGroups * kTileOut * 2;
constexpr size_t kSmRing = kSmZ + kRoundGroups * kTileOut * 2;
constexpr size_t kSmBytes = kSmRing + (size_t)kStages * kThreads * kVec * 4;
static_assert((size_t)kWarpsPerCta * kTileOut * 4 <= (size_t)kStages * kThreads * kVec * 4,
              "the reduction buffer reuses the ring");

struct GemvArgs {
  const uint32_t *planes;
  const uint16_t *s;
  const uint16_t *z;
  const float *grp_sums;
  float *y;
  int d_in, d_out, P, W, G, tiles;
  WsHeader *hdr;
  const int32_t *unit_code;
  const float *unit_x;
  unsigned *counters;
  float *partials;  // [gridDim.x][2][kTileOut]
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

// 2^23 + slice * 4^(sh/2): the slice at bit sh of w moved into a float mantissa.
__device__ __forceinline__ float magic_field(uint32_t w, int sh) {
  return __uint_as_float((w & (3u << sh)) | 0x4B000000u);
}

// Field t of a word is accumulated scaled by 4^pos(t): pos = t for t <= 10,
// t - 11 for t >= 11.
__device__ __forceinline__ int field_pos(int t) { return t <= 10 ? t : t - 11; }

// acc[t] += xp * slice_t * 4^pos(t) for the 16 fields of w.
__device__ __forceinline__ void accumulate_word(float (&acc)[16], uint32_t w, float xp) {
  const uint32_t w2 = w >> 22;
  float m[16];
#pragma unroll
  for (int t = 0; t < 16; ++t)
    m[t] = (t <= 10) ? magic_field(w, 2 * t) : magic_field(w2, 2 * (t - 11));
  const float2 neg = make_float2(-8388608.0f, -8388608.0f);
  const float2 x2 = make_float2(xp, xp);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float2 f = __fadd2_rn(make_float2(m[2 * k], m[2 * k + 1]), neg);
    const float2 r = __ffma2_rn(x2, f, make_float2(acc[2 * k], acc[2 * k + 1]));
    acc[2 * k] = r.x;
    acc[2 * k + 1] = r.y;
  }
}

// 16 consecutive fp16 values from shared memory (32 bytes, 16-byte aligned).
__device__ __forceinline__ void lds16_half(const uint16_t *p, float (&v)[16]) {
  const uint4 a = *reinterpret_cast<const uint4 *>(p);
  const uint4 b = *reinterpret_cast<const uint4 *>(p + 8);
  const uint32_t u[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&u[k]));
    v[2 * k] = f.x;
    v[2 * k + 1] = f.y;
  }
}

// Start of CTA c's range of the tiles x U items.
__device__ __forceinline__ long long range_start(long long c, long long work, long long C) {
  return c * work / C;
}
// The CTA whose range contains item pos (ranges may be empty; pos < work).
__device__ __forceinline__ int cta_of(long long pos, long long work, int C) {
  long long c = pos * C / work;
  while (c + 1 < C && range_start(c + 1, work, C) <= pos) ++c;
  while (c > 0 && range_start(c, work, C) > pos) --c;
  return (int)c;
}

template <bool ALIGNED>
__global__ void __launch_bounds__(kThreads, 1) gemv_kernel(GemvArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  int32_t *rec_code = reinterpret_cast<int32_t *>(smem + kSmRecCode);
  float *rec_x = reinterpret_cast<float *>(smem + kSmRecX);
  uint16_t *s_st = reinterpret_cast<uint16_t *>(smem + kSmS);
  uint16_t *z_st = reinterpret_cast<uint16_t *>(smem + kSmZ);
  uint32_t *ring = reinterpret_cast<uint32_t *>(smem + kSmRing);
  __shared__ int s_nround, s_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int sub = lane / kLanes, li = lane % kLanes;
  const int C = gridDim.x, c = blockIdx.x;  // C <= kMaxCtas (partials slots)

  // everything below reads what grinqh_assign wrote
  asm volatile("griddepcontrol.wait;\n" ::: "memory");

  int U = a.hdr->total_units;
  if (a.hdr->d_in != a.d_in || a.hdr->b_max != 2 * a.P) {
    // the stream was written for another layer: report it and produce zeros
    if (tid == 0 && c == 0) atomicCAS(&a.hdr->error, 0, kDevErrStreamMismatch);
    U = 0;
  }
  if (U < 0 || U > a.d_in * a.P) {
    if (tid == 0 && c == 0) atomicCAS(&a.hdr->error, 0, kDevErrBadUnit);
    U = 0;
  }
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");

  if (U == 0) {  // no active row anywhere: y = 0 exactly
    for (int t = c; t < a.tiles; t += C)
      for (int e = tid; e < kTileOut; e += kThreads) {
        const int o = t * kTileOut + e;
        if (o < a.d_out) a.y[o] = 0.0f;
      }
    return;
  }

  const long long work = (long long)a.tiles * U;
  // Only the first C_eff CTAs take work, so that every range is non-empty and
  // every CTA counted as a contributor of a tile really arrives at its counter.
  const int C_eff = (int)min((long long)C, work);
  if (c >= C_eff) return;
  const long long r_start = range_start(c, work, C_eff), r_end = range_start(c + 1, work, C_eff);

  for (long long pos = r_start; pos < r_end;) {
    const int tile = (int)(pos / U);
    const long long seg_end = min(r_end, (long long)(tile + 1) * U);
    const int u0 = (int)(pos - (long long)tile * U), u1 = (int)(seg_end - (long long)tile * U);
    pos = seg_end;

    const int word0 = tile * kTileWords + li * kVec;
    const int nvalid = max(0, min(kVec, a.W - word0));
    const int o_lane = li * kVec * 16;  // this lane's first output inside the tile

    float acc[kVec][16], yacc[kVec][16];
#pragma unroll
    for (int v = 0; v < kVec; ++v)
#pragma unroll
      for (int t = 0; t < 16; ++t) acc[v][t] = yacc[v][t] = 0.0f;
    int g_cur = -1, g_lo = 0;

    auto flush = [&](int g) {
      const uint16_t *srow = s_st + (g - g_lo) * kTileOut + o_lane;
#pragma unroll
      for (int v = 0; v < kVec; ++v) {
        float sv[16];
        lds16_half(srow + 16 * v, sv);
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          yacc[v][t] = fmaf(sv[t], acc[v][t], yacc[v][t]);
          acc[v][t] = 0.0f;
        }
      }
    };

    for (int r = u0; r < u1;) {
      const int n = min(kRoundUnits, u1 - r);
      __syncthreads();  // the previous round no longer reads the staged data
      if (tid == 0) s_nround = n;
      for (int k = tid; k < n; k += kThreads) {
        int code = a.unit_code[r + k];
        float xp = a.unit_x[r + k];
        if ((code >> 3) >= a.d_in || code < 0 || (code & 3) >= a.P) {
          atomicCAS(&a.hdr->error, 0, kDevErrBadUnit);
          code = 0;  // row 0, plane 0 with x' = 0: contributes nothing
          xp = 0.0f;
        }
        rec_code[k] = code;
        rec_x[k] = xp;
      }
      __syncthreads();
      // cut the round where its groups stop fitting the staged s/z rows
      g_lo = rec_code[0] >> 10;
      for (int k = tid; k < n; k += kThreads)
        if ((rec_code[k] >> 10) >= g_lo + kRoundGroups) atomicMin(&s_nround, k);
      __syncthreads();
      const int nr = s_nround;
      const int ng = (rec_code[nr - 1] >> 10) - g_lo + 1;
      // stage s and z rows of groups g_lo .. g_lo+ng-1 for this tile (16-byte chunks)
      {
        const int chunks = ng * (kTileOut / 8);  // 64 chunks of 8 halves per row
        for (int k = tid; k < 2 * chunks; k += kThreads) {
          const int which = k / chunks, kk = k % chunks;
          const int gi = kk / (kTileOut / 8), ci = kk % (kTileOut / 8);
          const int o = tile * kTileOut + ci * 8;
          const uint16_t *src = (which ? a.z : a.s) + (size_t)(g_lo + gi) * a.d_out + o;
          uint16_t *dst = (which ? z_st : s_st) + gi * kTileOut + ci * 8;
          // rows start on 32-byte boundaries (d_out % 16 == 0); past d_out: zero fill
          const int bytes = o < a.d_out ? 16 : 0;
          cp_async16(dst, bytes > 0 ? (const void *)src : (const void *)a.s, bytes);
        }
        cp_async_commit();
      }

      const int wa = (int)((long long)warp * nr / kWarpsPerCta);
      const int wb = (int)((long long)(warp + 1) * nr / kWarpsPerCta);
      const int first = wa + sub;
      const int count = wb > first ? (wb - first + kSpw - 1) / kSpw : 0;

      auto issue = [&](int k, int slot_i) {
        const int code = rec_code[first + k * kSpw];
        const int row = code >> 3, p = code & 3;
        const uint32_t *src = a.planes + ((size_t)row * a.P + p) * a.W + word0;
        uint32_t *dst = ring + ((size_t)slot_i * kThreads + tid) * kVec;
        if (ALIGNED) {
          cp_async16(dst, nvalid > 0 ? (const void *)src : (const void *)a.planes, 4 * nvalid);
        } else {
#pragma unroll
          for (int v = 0; v < kVec; ++v)
            cp_async4(dst + v, v < nvalid ? (const void *)(src + v) : (const void *)a.planes,
                      v < nvalid ? 4 : 0);
        }
      };

#pragma unroll
      for (int k = 0; k < kStages - 1; ++k) {
        if (k < count) issue(k, k);
        cp_async_commit();
      }
      cp_async_wait<kStages - 1>();  // this thread's s/z chunks have landed
      __syncthreads();               // ... and everybody else's

      for (int k = 0; k < count; ++k) {
        const int kn = k + kStages - 1;
        if (kn < count) issue(kn, kn % kStages);
        cp_async_commit();
        cp_async_wait<kStages - 1>();
        const int u = first + k * kSpw;
        const int code = rec_code[u];
        const float xp = rec_x[u];
        const int g = code >> 10;
        if (g != g_cur) {
          if (g_cur >= 0) flush(g_cur);
          g_cur = g;
        }
        if (code & 4) {  // first unit of its group: add s*Phi_g + z*X_g once
          const float X = a.grp_sums[g], Phi = a.grp_sums[a.G + g];
          const uint16_t *srow = s_st + (g - g_lo) * kTileOut + o_lane;
          const uint16_t *zrow = z_st + (g - g_lo) * kTileOut + o_lane;
#pragma unroll
          for (int v = 0; v < kVec; ++v) {
            float sv[16], zv[16];
            lds16_half(srow + 16 * v, sv);
            lds16_half(zrow + 16 * v, zv);
#pragma unroll
            for (int t = 0; t < 16; ++t) {
              const float up = __int_as_float((127 + 2 * field_pos(t)) << 23);  // 4^pos(t)
              yacc[v][t] = fmaf(fmaf(sv[t], Phi, zv[t] * X), up, yacc[v][t]);
            }
          }
        }
        const uint4 q = *reinterpret_cast<const uint4 *>(
            ring + ((size_t)(k % kStages) * kThreads + tid) * kVec);
        accumulate_word(acc[0], q.x, xp);
        accumulate_word(acc[1], q.y, xp);
        accumulate_word(acc[2], q.z, xp);
        accumulate_word(acc[3], q.w, xp);
      }
      cp_async_wait<0>();
      if (g_cur >= 0) {  // the next round restages s/z: flush while this one is live
        flush(g_cur);
        g_cur = -1;
      }
      r += nr;
    }

    // ---- reduce the subgroups of a warp, then the warps of the CTA ------------
#pragma unroll
    for (int off = kLanes; off < 32; off <<= 1)
#pragma unroll
      for (int v = 0; v < kVec; ++v)
#pragma unroll
        for (int t = 0; t < 16; ++t) yacc[v][t] += __shfl_xor_sync(0xffffffffu, yacc[v][t], off);
    __syncthreads();  // every cp.async has landed and the ring is free
    float *red = reinterpret_cast<float *>(ring);  // [warps][kTileOut]
    if (sub == 0) {
#pragma unroll
      for (int v = 0; v < kVec; ++v)
#pragma unroll
        for (int t = 0; t < 16; t += 4)
          *reinterpret_cast<float4 *>(&red[warp * kTileOut + o_lane + 16 * v + t]) =
              make_float4(yacc[v][t], yacc[v][t + 1], yacc[v][t + 2], yacc[v][t + 3]);
    }
    __syncthreads();
    float val[kTileOut / kThreads];
#pragma unroll
    for (int e = 0; e < kTileOut / kThreads; ++e) {
      const int ol = tid + e * kThreads;
      float sum = 0.0f;
#pragma unroll
      for (int w = 0; w < kWarpsPerCta; ++w) sum += red[w * kTileOut + ol];
      val[e] = sum * __int_as_float((127 - 2 * field_pos(ol & 15)) << 23);  // 4^-pos
    }
    const int obase = tile * kTileOut;
    if (u0 == 0 && u1 == U) {  // the whole tile is ours
#pragma unroll
      for (int e = 0; e < kTileOut / kThreads; ++e) {
        const int o = obase + tid + e * kThreads;
        if (o < a.d_out) a.y[o] = val[e];
      }
      continue;
    }
    // a partial segment: publish it, and let the tile's last contributor sum
    // slot 0 holds the segment of the first tile of a range, slot 1 that of its last
    const int slot = (tile == (int)(r_start / U)) ? 0 : 1;
    float *mine = a.partials + ((size_t)c * 2 + slot) * kTileOut;
#pragma unroll
    for (int e = 0; e < kTileOut / kThreads; ++e) mine[tid + e * kThreads] = val[e];
    const int c_first = cta_of((long long)tile * U, work, C_eff);
    const int c_last = cta_of((long long)(tile + 1) * U - 1, work, C_eff);
    __threadfence();
    __syncthreads();
    if (tid == 0)
      s_last = atomicInc(&a.counters[tile], (unsigned)(c_last - c_first)) ==
               (unsigned)(c_last - c_first);
    __syncthreads();
    if (s_last) {
      __threadfence();
#pragma unroll
      for (int e = 0; e < kTileOut / kThreads; ++e) {
        const int ol = tid + e * kThreads;
        float sum = 0.0f;
        for (int cc = c_first; cc <= c_last; ++cc) {
          // CTA cc used slot 0 for the first tile of its range, slot 1 for its last
          const int cc_first_tile = (int)(range_start(cc, work, C_eff) / U);
          const int sl = (tile == cc_first_tile) ? 0 : 1;
          sum += __ldcg(a.partials + ((size_t)cc * 2 + sl) * kTileOut + ol);
        }
        const int o = obase + ol;
        if (o < a.d_out) a.y[o] = sum;
      }
    }
  }
}

int device_sms() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return kNumSMs;
  if (dev < 64 && cached[dev]) return cached[dev];
  int n = kNumSMs;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n = kNumSMs;
  if (n > kMaxCtas) n = kMaxCtas;
  if (dev < 64) cached[dev] = n;
  return n;
}

template <bool ALIGNED>
cudaError_t launch_variant(const GemvArgs &a, cudaStream_t st) {
  cudaError_t e = ensure_smem_attr((const void *)gemv_kernel<ALIGNED>, kSmBytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(device_sms());
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemv_kernel<ALIGNED>, a);
}

}  // namespace

cudaError_t launch_gemv(const uint32_t *planes, const uint16_t *s, const uint16_t *z,
                        const float *grp_sums, int d_in, int d_out, int b_max, float *y,
                        void *ws, cudaStream_t st) {
  const WsLayout L = ws_layout(d_in, d_out, b_max);
  GemvArgs a;
  char *w = static_cast<char *>(ws);
  a.planes = planes;
  a.s = s;
  a.z = z;
  a.grp_sums = grp_sums;
  a.y = y;
  a.d_in = d_in;
  a.d_out = d_out;
  a.P = b_max / 2;
  a.W = d_out / 16;
  a.G = d_in / kGroup;
  a.tiles = L.tiles;
  a.hdr = reinterpret_cast<WsHeader *>(w);
  a.unit_code = reinterpret_cast<const int32_t *>(w + L.unit_code);
  a.unit_x = reinterpret_cast<const float *>(w + L.unit_x);
  a.counters = reinterpret_cast<unsigned *>(w + L.counters);
  a.partials = reinterpret_cast<float *>(w + L.partials);
  cudaError_t e = (a.W % 4 == 0) ? launch_variant<true>(a, st) : launch_variant<false>(a, st);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace grinqh
