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
//    row's plane region.  Each tile's U units are cut into m equal contiguous
//    ranges, m = floor(CTAs / tiles) (at most U), one range per CTA: a single
//    wave with one segment per CTA, balanced whatever the sparsity pattern.
//    With more tiles than CTAs, CTAs take whole tiles in turn.
//  * Inside a CTA each warp takes a contiguous piece of a round of up to
//    kRoundUnits units and its four 8-lane subgroups take every 4th unit; each
//    lane copies its 16-byte share of a unit into a private shared-memory ring
//    with cp.async (kStages deep), so ~45 KB per SM are in flight without
//    holding registers.  The s/z rows of the round's groups are staged in
//    shared memory alongside, so flushing a group never waits on memory.
//  * Field rebuild, two fields per logic op.  Output t of a word sits in bits
//    [2t+1:2t]; outputs t and t+8 are 16 bits apart, so one shifted copy of the
//    word and one LOP3 put both slices into the top mantissa bits (position 4,
//    bits 9:8, or position 3, bits 7:6) of the two halves of a half2 whose
//    exponent field is 15 + 2k (k = P-1-plane): each half is then exactly
//    4^k (1 + slice 4^pos / 1024).  A mixed-precision FMA (fp16 x fp16 + fp32,
//    sm_100) multiplies it by fp16 x exactly and adds in fp32.  Four shifts,
//    eight LOP3 and sixteen FMAs cover a word: 1.75 instructions per field.
//    The constant part x 4^k of every product is the same for all outputs of
//    a lane, so it is summed once per unit and subtracted at each flush; the
//    slice sits in the top bits of the mantissa, so this costs at most four
//    of fp32's 24 bits.
//  * The m partial sums of a tile are added by the last of its CTAs to
//    arrive (atomicInc on a self-resetting per-tile counter), in CTA order,
//    after staging all of them in shared memory with one cp.async round trip,
//    so y is deterministic.  A tile with m = 1 is written directly.
//  * Programmatic dependent launch: the kernel waits on grinqh_assign with
//    griddepcontrol.wait, so its launch overlaps the tail of assign.
#include "grinqh_internal.cuh"

namespace grinqh {
namespace {

constexpr int kThreads = 256;
constexpr int kWarpsPerCta = kThreads / 32;
constexpr int kStages = 16;          // cp.async ring depth per lane (power of two)
constexpr int kRoundUnits = 1024;    // unit records staged in shared memory per round
constexpr int kRoundGroups = 8;      // s/z rows staged per round
constexpr int kVec = 4;              // words per lane and unit (16 bytes)
constexpr int kLanes = kTileWords / kVec;  // 8 lanes per unit
constexpr int kSpw = 32 / kLanes;          // 4 subgroups per warp
constexpr int kFixupChunk = 16;            // contributor partials staged per fixup pass

// shared memory map (bytes)
constexpr size_t kSmRawCode = 0;                                  // int32 [kRoundUnits]
constexpr size_t kSmRawX = kSmRawCode + kRoundUnits * 4;           // fp32  [kRoundUnits]
constexpr size_t kSmRec = kSmRawX + kRoundUnits * 4;               // int4  [kRoundUnits]
constexpr size_t kSmXh = kSmRec + kRoundUnits * 16;                // fp16  [kRoundUnits]
constexpr size_t kSmS = kSmXh + kRoundUnits * 2;                   // fp16  [kRoundGroups][kTileOut]
constexpr size_t kSmZ = kSmS + kRoundGroups * kTileOut * 2;
constexpr size_t kSmRing = kSmZ + kRoundGroups * kTileOut * 2;     // [kStages][kThreads][kVec] words
constexpr size_t kRingBytes = (size_t)kStages * kThreads * kVec * 4;
constexpr size_t kSmBytes = kSmRing + kRingBytes;
static_assert((size_t)kWarpsPerCta * kSpw * kTileOut * 4 <= kRingBytes, "reduction buffer in the ring");
static_assert((size_t)kFixupChunk * kTileOut * 4 <= kRingBytes, "fixup staging in the ring");
static_assert((kStages & (kStages - 1)) == 0, "ring slots are taken modulo kStages");

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
  float *partials;  // [gridDim.x][2][kTileOut] (slot 0 used)
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

// (x & MASK) | magic in one logic instruction (magic is a runtime register).
template <uint32_t MASK>
__device__ __forceinline__ uint32_t pick(uint32_t x, uint32_t magic) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(x), "n"(MASK), "r"(magic));
  return d;
}

// a0 += xh * lo(h), a1 += xh * hi(h): exact fp16 products, fp32 sums.
__device__ __forceinline__ void fma_pair(float &a0, float &a1, uint32_t h, uint16_t xh) {
  asm("{.reg .b16 lo, hi;\n"
      " mov.b32 {lo, hi}, %2;\n"
      " fma.rn.f32.f16 %0, %3, lo, %0;\n"
      " fma.rn.f32.f16 %1, %3, hi, %1;}\n"
      : "+f"(a0), "+f"(a1)
      : "r"(h), "h"(xh));
}

// Field t of a word lands at half position pos(t) = 4 (t even) or 3 (t odd);
// its accumulator holds 4^k (1 + slice 4^pos / 1024) per unit, so the true
// plane-weighted sum is (acc - offset) * 1024 / 4^pos = (acc - offset) * field_scale(t).
__device__ __forceinline__ float field_scale(int t) { return (t & 1) ? 16.0f : 4.0f; }

constexpr uint32_t kPos4 = 0x03000300u;  // bits 9:8 of both halves
constexpr uint32_t kPos3 = 0x00C000C0u;  // bits 7:6 of both halves

// acc[t] += xh * 4^k (1 + slice_t 4^pos(t) / 1024) for the 16 fields of w.
__device__ __forceinline__ void accumulate_word(float (&acc)[16], uint32_t w, uint32_t magic,
                                                uint16_t xh) {
  const uint32_t c1 = w << 4, c2 = w << 8, c3 = w >> 4, c4 = w >> 8;
  // pair (t, t+8): t=0 from w<<8 @4, t=1 from w<<4 @3, t=2 from w<<4 @4,
  // t=3 from w @3, t=4 from w @4, t=5 from w>>4 @3, t=6 from w>>4 @4, t=7 from w>>8 @3
  fma_pair(acc[0], acc[8], pick<kPos4>(c2, magic), xh);
  fma_pair(acc[1], acc[9], pick<kPos3>(c1, magic), xh);
  fma_pair(acc[2], acc[10], pick<kPos4>(c1, magic), xh);
  fma_pair(acc[3], acc[11], pick<kPos3>(w, magic), xh);
  fma_pair(acc[4], acc[12], pick<kPos4>(w, magic), xh);
  fma_pair(acc[5], acc[13], pick<kPos3>(c3, magic), xh);
  fma_pair(acc[6], acc[14], pick<kPos4>(c3, magic), xh);
  fma_pair(acc[7], acc[15], pick<kPos3>(c4, magic), xh);
}

__device__ __forceinline__ unsigned long long __umul64wide(unsigned a, unsigned b) {
  return (unsigned long long)a * b;  // one widening multiply
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

template <bool ALIGNED>
__global__ void __launch_bounds__(kThreads, 1) gemv_kernel(GemvArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  int32_t *raw_code = reinterpret_cast<int32_t *>(smem + kSmRawCode);
  float *raw_x = reinterpret_cast<float *>(smem + kSmRawX);
  int4 *rec = reinterpret_cast<int4 *>(smem + kSmRec);  // {region, x 4^k bits, magic, g | first<<31}
  uint16_t *rec_xh = reinterpret_cast<uint16_t *>(smem + kSmXh);
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

  // m CTAs per tile, each with a contiguous range of the tile's units (m <= U,
  // so no range is empty); with more tiles than CTAs, whole tiles in turn
  const int m = a.tiles >= C ? 1 : min(C / a.tiles, U);
  const int C_eff = a.tiles >= C ? C : a.tiles * m;
  if (c >= C_eff) return;

  for (int tile = c / m; tile < a.tiles; tile += C_eff / m) {
    const int part = c % m;
    const int u0 = (int)((long long)part * U / m), u1 = (int)((long long)(part + 1) * U / m);

    const int word0 = tile * kTileWords + li * kVec;
    const int nvalid = max(0, min(kVec, a.W - word0));
    const int o_lane = li * kVec * 16;  // this lane's first output inside the tile
    // plane word (region r, this lane) = lane_base + r * lane_stride; a lane past
    // d_out reads nothing (zero-byte copies from a valid address)
    const uint32_t *lane_base = a.planes + (nvalid > 0 ? word0 : 0);
    const unsigned lane_stride = nvalid > 0 ? (unsigned)a.W : 0u;

    float acc[kVec][16], yacc[kVec][16];
#pragma unroll
    for (int v = 0; v < kVec; ++v)
#pragma unroll
      for (int t = 0; t < 16; ++t) acc[v][t] = yacc[v][t] = 0.0f;
    float x_off = 0.0f;  // sum of x 4^k over the units in acc
    int g_cur = -1, g_lo = 0;

    // yacc[t] += s_t * (acc[t] - x_off) in the domain scaled by 1 / field_scale(t)
    auto flush = [&]() {
      if (g_cur >= 0) {
        const uint16_t *srow = s_st + (g_cur - g_lo) * kTileOut + o_lane;
#pragma unroll
        for (int v = 0; v < kVec; ++v) {
          float sv[16];
          lds16_half(srow + 16 * v, sv);
#pragma unroll
          for (int t = 0; t < 16; ++t) yacc[v][t] = fmaf(sv[t], acc[v][t] - x_off, yacc[v][t]);
        }
      }
#pragma unroll
      for (int v = 0; v < kVec; ++v)
#pragma unroll
        for (int t = 0; t < 16; ++t) acc[v][t] = 0.0f;
      x_off = 0.0f;
    };

    for (int r = u0; r < u1;) {
      const int n = min(kRoundUnits, u1 - r);
      __syncthreads();  // the previous round no longer reads the staged data
      if (tid == 0) s_nround = n;
      // raw records of the round: one round trip
      for (int k = tid; k < n; k += kThreads) {
        cp_async4(raw_code + k, a.unit_code + r + k, 4);
        cp_async4(raw_x + k, a.unit_x + r + k, 4);
      }
      cp_async_commit();
      cp_async_wait<0>();
      __syncthreads();
      // digest once per CTA: plane region, half2 magic, fp16 x, group and first flag
      g_lo = min(max(raw_code[0] >> 10, 0), a.G - 1);  // a sorted stream starts at its lowest group
      for (int k = tid; k < n; k += kThreads) {
        int code = raw_code[k];
        float xp = raw_x[k];
        if ((code >> 3) >= a.d_in || code < 0 || (code & 3) >= a.P || (code >> 10) < g_lo) {
          atomicCAS(&a.hdr->error, 0, kDevErrBadUnit);
          code = (g_lo << 10);  // row 128 g_lo, plane 0 with x' = 0: contributes nothing
          xp = 0.0f;
        }
        const int row = code >> 3, p = code & 3, kpl = a.P - 1 - p, g = code >> 10;
        rec[k] = make_int4(row * a.P + p, __float_as_int(xp), (15 + 2 * kpl) * 0x04000400,
                           g | ((code & 4) << 29));
        rec_xh[k] = __half_as_ushort(__float2half_rn(xp * __int_as_float((127 - 2 * kpl) << 23)));
        if (g >= g_lo + kRoundGroups) atomicMin(&s_nround, k);
      }
      __syncthreads();
      const int nr = s_nround;
      const int ng = (rec[nr - 1].w & 0x7fffffff) - g_lo + 1;
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

      // warp w takes units [wa, wb); in iteration k its subgroup sub takes wa + 4k + sub
      const int wa = (int)((long long)warp * nr / kWarpsPerCta);
      const int wb = (int)((long long)(warp + 1) * nr / kWarpsPerCta);
      const int iters = (wb - wa + kSpw - 1) / kSpw;  // the same for the whole warp
      uint32_t *my_ring = ring + (size_t)tid * kVec;   // slot i at my_ring + i * kThreads * kVec

      auto issue = [&](int k) {
        const int u = wa + k * kSpw + sub;
        if (u < wb) {
          const unsigned region = (unsigned)rec[u].x;  // row * P + plane < 2^26
          uint32_t *dst = my_ring + (k & (kStages - 1)) * (kThreads * kVec);
          const uint32_t *src = lane_base + __umul64wide(region, lane_stride);
          if (ALIGNED) {
            cp_async16(dst, src, 4 * nvalid);
          } else {
#pragma unroll
            for (int v = 0; v < kVec; ++v)
              cp_async4(dst + v, v < nvalid ? (const void *)(src + v) : (const void *)a.planes,
                        v < nvalid ? 4 : 0);
          }
        }
      };

#pragma unroll
      for (int k = 0; k < kStages - 1; ++k) {
        if (k < iters) issue(k);
        cp_async_commit();
      }
      cp_async_wait<kStages - 1>();  // this thread's s/z chunks have landed
      __syncthreads();               // ... and everybody else's

      for (int k = 0; k < iters; ++k) {
        if (k + kStages - 1 < iters) issue(k + kStages - 1);
        cp_async_commit();
        cp_async_wait<kStages - 1>();
        const int u = wa + k * kSpw + sub;
        const bool active = u < wb;
        const int4 rc = rec[active ? u : wa];
        const int g = rc.w & 0x7fffffff;
        // warp-uniform group change: every lane flushes its own group's partial sums
        if (__any_sync(0xffffffffu, active && g != g_cur)) {
          flush();
          if (active) g_cur = g;
        }
        if (__any_sync(0xffffffffu, active && rc.w < 0)) {
          if (active && rc.w < 0) {  // first unit of its group: add s*Phi_g + z*X_g once
            const float X = a.grp_sums[g], Phi = a.grp_sums[a.G + g];
            const uint16_t *srow = s_st + (g - g_lo) * kTileOut + o_lane;
            const uint16_t *zrow = z_st + (g - g_lo) * kTileOut + o_lane;
#pragma unroll
            for (int v = 0; v < kVec; ++v) {
              float sv[16], zv[16];
              lds16_half(srow + 16 * v, sv);
              lds16_half(zrow + 16 * v, zv);
#pragma unroll
              for (int t = 0; t < 16; ++t)
                yacc[v][t] = fmaf(fmaf(sv[t], Phi, zv[t] * X), 1.0f / field_scale(t), yacc[v][t]);
            }
          }
        }
        if (active) {
          const uint16_t xh = rec_xh[u];
          const uint32_t magic = (uint32_t)rc.z;
          x_off += __int_as_float(rc.y);
          const uint4 q = *reinterpret_cast<const uint4 *>(
              my_ring + (k & (kStages - 1)) * (kThreads * kVec));
          accumulate_word(acc[0], q.x, magic, xh);
          accumulate_word(acc[1], q.y, magic, xh);
          accumulate_word(acc[2], q.z, magic, xh);
          accumulate_word(acc[3], q.w, magic, xh);
        }
      }
      cp_async_wait<0>();
      flush();  // the next round restages s/z: flush while this one is live
      g_cur = -1;
      r += nr;
    }

    // ---- reduce the 32 subgroups of the CTA through shared memory ----------------
    __syncthreads();  // every cp.async has landed and the ring is free
    float *red = reinterpret_cast<float *>(ring);  // [warp * kSpw + sub][kTileOut]
    {
      float *mine = red + (warp * kSpw + sub) * kTileOut + o_lane;
#pragma unroll
      for (int v = 0; v < kVec; ++v)
#pragma unroll
        for (int t = 0; t < 16; t += 4)
          *reinterpret_cast<float4 *>(mine + 16 * v + t) =
              make_float4(yacc[v][t], yacc[v][t + 1], yacc[v][t + 2], yacc[v][t + 3]);
    }
    __syncthreads();
    float val[kTileOut / kThreads];
#pragma unroll
    for (int e = 0; e < kTileOut / kThreads; ++e) {
      const int ol = tid + e * kThreads;
      float sum = 0.0f;
#pragma unroll 8
      for (int sg = 0; sg < kWarpsPerCta * kSpw; ++sg) sum += red[sg * kTileOut + ol];
      val[e] = sum * field_scale(ol & 15);
    }
    const int obase = tile * kTileOut;
    if (m == 1) {  // the whole tile is ours
#pragma unroll
      for (int e = 0; e < kTileOut / kThreads; ++e) {
        const int o = obase + tid + e * kThreads;
        if (o < a.d_out) a.y[o] = val[e];
      }
      continue;
    }
    // one of m partial sums: publish it; the tile's last CTA to arrive adds them
    float *mine = a.partials + (size_t)c * 2 * kTileOut;
#pragma unroll
    for (int e = 0; e < kTileOut / kThreads; ++e) mine[tid + e * kThreads] = val[e];
    const int c_first = tile * m;
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicInc(&a.counters[tile], (unsigned)(m - 1)) == (unsigned)(m - 1);
    __syncthreads();
    if (s_last) {
      __threadfence();
      float sum[kTileOut / kThreads];
#pragma unroll
      for (int e = 0; e < kTileOut / kThreads; ++e) sum[e] = 0.0f;
      float *stage = reinterpret_cast<float *>(ring);  // [kFixupChunk][kTileOut]
      for (int c0 = 0; c0 < m; c0 += kFixupChunk) {
        const int nc = min(kFixupChunk, m - c0);
        __syncthreads();  // the previous chunk (or the reduction) no longer reads the stage
        for (int k = tid; k < nc * (kTileOut / 4); k += kThreads) {
          const int ci = k / (kTileOut / 4), q4 = k % (kTileOut / 4);
          cp_async16(stage + ci * kTileOut + q4 * 4,
                     a.partials + (size_t)(c_first + c0 + ci) * 2 * kTileOut + q4 * 4, 16);
        }
        cp_async_commit();
        cp_async_wait<0>();
        __syncthreads();
        for (int ci = 0; ci < nc; ++ci)
#pragma unroll
          for (int e = 0; e < kTileOut / kThreads; ++e)
            sum[e] += stage[ci * kTileOut + tid + e * kThreads];
      }
#pragma unroll
      for (int e = 0; e < kTileOut / kThreads; ++e) {
        const int o = obase + tid + e * kThreads;
        if (o < a.d_out) a.y[o] = sum[e];
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
