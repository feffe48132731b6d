// decode.cu -- the fused GRINQH batch-1 decode step in one kernel: precision
// assignment, per-plane compaction, plane-sparse load, rebuild and GEMV.
//
// What it computes ("GRINQH: Graded Input-Based Quantization Hierarchy",
// Method / overall framework and Key designs 1-3):
//   b_i = 2 #{k : theta_k <= |x_i|},
//   y_o = sum_{i : b_i > 0} x_i (s_{g,o} (Q_{i,o} + phi_{b_i}) + z_{g,o}),
// with Q rebuilt from the first b_i/2 bit planes of row i only.
//
// How (B200 design):
//  * Factorisation per 128-row group g:
//      y_o = sum_g s_{g,o} (A_{g,o} + Phi_g) + z_{g,o} X_g,
//      A_{g,o} = sum over units (i, p) of group g of x_i 4^(P-1-p) slice_p(i, o),
//    where a unit is one (row, plane) pair with b_i > 2p and slice_p is the
//    2-bit field of plane p.  X_g, Phi_g are per-group sums of x and x phi.
//  * Units are ordered by group, plane, row (the order of the per-plane lists
//    within a group).  Every CTA derives the whole order itself from x and
//    theta: it counts each group's units per plane (one warp per group), scans
//    the counts, and then compacts only the groups its own range touches.  No
//    other kernel and no global round trip sit between x and the GEMV.
//  * Work = 1024-output tiles x unit ranges.  A unit's tile segment is 256
//    contiguous bytes of its plane region.  Each tile's U units are cut into
//    m = floor(CTAs / tiles) equal contiguous ranges, one per CTA (one wave,
//    balanced whatever the sparsity); the m partial tiles are added by the
//    last CTA to arrive, in CTA order (deterministic).
//  * A CTA walks its range in rounds of at most 1024 units and 8 groups.  The
//    segments stream through an 8-stage shared-memory ring (cp.async, 16 B per
//    thread and copy, one barrier per 32 units).
//  * The contraction runs on the tensor cores as m16n8k16 MMAs with fp32
//    accumulation: A (16 outputs x 16 units) is built in registers straight
//    from the packed words -- a byte permute pairs the same 16 outputs of two
//    units, one AND per register isolates a 2-bit field pair in the low
//    mantissa bits of two fp16 subnormals, exactly slice * 2^(pos-24) -- and B
//    (16 units x 8) holds x 4^(P-1-p) 2^-c_g in column (g mod 8), so the 8
//    columns keep the 8 groups of a round apart and the group scales s are
//    applied once per round, not per unit.  One warp covers 128 outputs with
//    8 MMAs per 16 units: 4 shared loads, 4 permutes, 4 shifts, 32 ANDs and
//    8 MMAs per 512 bytes of planes, against about 240 instructions for a
//    scalar fp32 decode of the same bytes.
#include "grinqh_internal.cuh"

namespace grinqh {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBlocks = 8;            // 128-output blocks of a tile; warps w and w + 8 share one
constexpr int kTile = 1024;           // outputs per CTA tile (8 blocks x 128)
constexpr int kTileW = kTile / 16;    // 64 words = 256 bytes per unit and tile
constexpr int kRow = kTileW + 4;      // shared words per unit row: conflict-free fragment loads
constexpr int kK = 16;                // units per MMA k-step
constexpr int kStage = 64;            // units per ring stage (4 k-steps, 2 per warp)
constexpr int kRing = 8;              // ring stages
constexpr int kRingEarly = 6;         // stages issued before the x cache (on the last slots) is freed
constexpr int kRound = 1024;          // units per round
constexpr int kSlots = 8;             // groups per round (the MMA n dimension)
constexpr int kMaxG = kDecodeMaxDin / kGroup;
constexpr int kXCache = 16384;        // rows of x held in shared memory (larger d_in: in chunks)
constexpr int kGT = 16;               // front-end threads per group (8 rows each)

// shared memory map (bytes)
constexpr size_t kStageBytes = (size_t)kStage * kRow * 4;
constexpr size_t kSmRing = 0;                                               // u32 [kRing][kStage][kRow]
constexpr size_t kSmX = kSmRing + (size_t)kRingEarly * kStageBytes;         // fp16 [kXCache], aliases
                                                                            // ring slots >= kRingEarly
constexpr size_t kSmRegion = kSmRing + (size_t)kRing * kStageBytes;         // i32 [kRound]
constexpr size_t kSmUx = kSmRegion + kRound * 4;                            // u32 [kRound]: xh | slot << 16
constexpr size_t kSmBfrag = kSmUx + kRound * 4;                             // uint2 [kRound / kK][32]
constexpr size_t kSmS = kSmBfrag + (size_t)(kRound / kK) * 32 * 8;          // fp16 [kSlots][kTile]
constexpr size_t kSmZ = kSmS + (size_t)kSlots * kTile * 2;                  // fp16 [kSlots][kTile]
constexpr size_t kSmCnt = kSmZ + (size_t)kSlots * kTile * 2;                // u32 [kMaxG]: plane counts, bytes
constexpr size_t kSmLoff = kSmCnt + (size_t)kMaxG * 4;                      // int4 [kMaxG]: list offsets
constexpr size_t kSmGoff = kSmLoff + (size_t)kMaxG * 16;                    // i32 [kMaxG + 4]: unit offsets
constexpr size_t kSmSlot = kSmGoff + (size_t)(kMaxG + 4) * 4;               // SlotInfo [kSlots]
constexpr size_t kSmWsum = kSmSlot + kSlots * 16;                           // int4 [kWarps]
constexpr size_t kSmRed = kSmWsum + kWarps * 16;                            // fp32 [kTile]: odd-k warps
constexpr size_t kSmBytes = kSmRed + (size_t)kTile * 4;
static_assert(kSmBytes <= 227 * 1024, "shared memory");
static_assert((size_t)kXCache * 2 <= (size_t)(kRing - kRingEarly) * kStageBytes, "x cache fits");
static_assert(kSmRing % 16 == 0 && kSmX % 16 == 0 && kSmS % 16 == 0 && kSmZ % 16 == 0 &&
                  kSmBfrag % 16 == 0 && kSmCnt % 16 == 0 && kSmLoff % 16 == 0 && kSmSlot % 16 == 0 &&
                  kSmWsum % 16 == 0 && kSmRed % 16 == 0,
              "16-byte aligned regions");
static_assert(kStage * 16 == 2 * kThreads, "two 16-byte copies per thread and stage");
static_assert(kStage == 4 * kK && kWarps == 2 * kBlocks, "two k-steps per warp and stage");
static_assert(kSlots * kGT <= kThreads && kMaxG == kThreads, "thread mappings");

struct SlotInfo {
  int c;       // the group's B-column scale exponent: B holds x 4^(P-1-p) 2^-c
  float X;     // sum of x over the group's active rows (added if `first`)
  float Phi;   // sum of x phi_{b/2} over the group's active rows
  int first;   // the group's first unit lies in this round: add s Phi + z X here
};

struct DecodeArgs {
  const uint32_t *planes;
  const uint16_t *s;
  const uint16_t *z;
  const uint16_t *x;
  const float *theta;
  const float *phi;  // may be null: the default table
  int d_in, d_out, b_max, P, W, G, tiles;
  float *y;
  uint8_t *b;         // optional outputs (null: not written)
  int32_t *lists;
  int32_t *counts;
  float *grp_sums;
  unsigned *counters;
  float *partials;    // [gridDim.x][kTile]
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
__device__ __forceinline__ void cp_async4(void *dst, const void *src) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(d), "l"(src));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// D += A B, m16n8k16, fp16 operands, fp32 accumulators.
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float h2f(uint16_t h) { return __half2float(__ushort_as_half(h)); }

// 2^e as a float, for |e| well inside the normal range.
__device__ __forceinline__ float exp2i(int e) { return __int_as_float((127 + e) << 23); }

// Bit position of output t's 2-bit field inside its fp16 half after the
// extraction below: t' = t mod 8; t' <= 4 stays at 2t', t' >= 5 is shifted
// down by 6 (so it stays inside the 10 mantissa bits).
__host__ __device__ constexpr int field_pos(int t) {
  return (t & 7) <= 4 ? 2 * (t & 7) : 2 * (t & 7) - 6;
}

template <bool ALIGNED>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(DecodeArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  uint32_t *ring = reinterpret_cast<uint32_t *>(smem + kSmRing);
  uint16_t *xc = reinterpret_cast<uint16_t *>(smem + kSmX);
  int32_t *s_region = reinterpret_cast<int32_t *>(smem + kSmRegion);
  uint32_t *s_ux = reinterpret_cast<uint32_t *>(smem + kSmUx);
  uint2 *s_bfrag = reinterpret_cast<uint2 *>(smem + kSmBfrag);
  uint16_t *s_st = reinterpret_cast<uint16_t *>(smem + kSmS);
  uint16_t *z_st = reinterpret_cast<uint16_t *>(smem + kSmZ);
  uint32_t *s_cnt = reinterpret_cast<uint32_t *>(smem + kSmCnt);
  int4 *s_loff = reinterpret_cast<int4 *>(smem + kSmLoff);
  int *s_goff = reinterpret_cast<int *>(smem + kSmGoff);
  SlotInfo *s_slot = reinterpret_cast<SlotInfo *>(smem + kSmSlot);
  int4 *s_wsum = reinterpret_cast<int4 *>(smem + kSmWsum);
  float *s_red = reinterpret_cast<float *>(smem + kSmRed);
  __shared__ int s_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int fg = lane >> 2, tq = lane & 3;  // MMA fragment row group and column pair
  const int ob = warp & (kBlocks - 1);      // the warp's 128-output block of the tile
  const int kp = warp / kBlocks;            // ... and its k-step parity
  const int gsub = tid & (kGT - 1);         // front end: lane of a 16-thread group team
  const int C = gridDim.x, c = blockIdx.x;
  const int P = a.P, G = a.G;

  // x, theta and the weights may be written by the kernel launched just before
  asm volatile("griddepcontrol.wait;\n" ::: "memory");

  __half2 t2[4];
  make_thresholds(a.theta, P, t2);
  float phi[5];
#pragma unroll
  for (int k = 0; k <= 4; ++k) {
    const float def = (2 * k < a.b_max) ? exp2i(a.b_max - 2 * k - 1) : 0.0f;
    phi[k] = (k <= P) ? (a.phi ? a.phi[k] : def) : 0.0f;
  }

  // rows 128 g + 8 gsub .. + 7 of x: from the shared cache while it holds them
  int xc_base = 0;
  bool xc_valid = true;
  auto load8 = [&](int g) -> uint4 {
    const int row = g * kGroup + 8 * gsub;
    if (xc_valid && row >= xc_base && row < xc_base + kXCache)
      return *reinterpret_cast<const uint4 *>(xc + (row - xc_base));
    return __ldg(reinterpret_cast<const uint4 *>(a.x + row));
  };

  // ---- units per (group, plane) ----------------------------------------------------
  // x goes to shared memory in one cp.async wave per chunk of kXCache rows; 16
  // threads count a group (8 rows each), the four plane counts (each <= 128)
  // packed into the bytes of one word; two groups per team and pass.
  for (int base = 0; base < a.d_in; base += kXCache) {
    const int rows = min(kXCache, a.d_in - base);
    if (base > 0) __syncthreads();  // the previous chunk is counted
    for (int q = tid; q < rows / 8; q += kThreads) cp_async16(xc + 8 * q, a.x + base + 8 * q, 16);
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    xc_base = base;
    const int g_lo = base / kGroup, g_hi = (base + rows) / kGroup;
    for (int g0 = g_lo; g0 < g_hi; g0 += 2 * (kThreads / kGT)) {
      const int ga = g0 + (tid >> 4), gb = ga + kThreads / kGT;
      uint32_t pa = 0, pb = 0;
      uint32_t ma[4], mb[4];
      plane_masks8(ga < g_hi ? load8(ga) : make_uint4(0, 0, 0, 0), t2, P, ma);
      plane_masks8(gb < g_hi ? load8(gb) : make_uint4(0, 0, 0, 0), t2, P, mb);
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        pa += (uint32_t)__popc(ma[p]) << (8 * p);
        pb += (uint32_t)__popc(mb[p]) << (8 * p);
      }
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) {
        pa += __shfl_xor_sync(0xffffffffu, pa, off);
        pb += __shfl_xor_sync(0xffffffffu, pb, off);
      }
      if (gsub == 0 && ga < g_hi) s_cnt[ga] = pa;
      if (gsub == 0 && gb < g_hi) s_cnt[gb] = pb;
    }
  }
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  __syncthreads();

  // ---- exclusive scans over groups: per-plane list offsets and unit offsets ----
  {
    const int g0 = tid;  // kMaxG = kThreads
    auto unpack = [](uint32_t v) {
      return make_int4(v & 255u, (v >> 8) & 255u, (v >> 16) & 255u, v >> 24);
    };
    const int4 z4 = make_int4(0, 0, 0, 0);
    const int4 v0 = g0 < G ? unpack(s_cnt[g0]) : z4;
    int4 inc = v0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      int4 t;
      t.x = __shfl_up_sync(0xffffffffu, inc.x, off);
      t.y = __shfl_up_sync(0xffffffffu, inc.y, off);
      t.z = __shfl_up_sync(0xffffffffu, inc.z, off);
      t.w = __shfl_up_sync(0xffffffffu, inc.w, off);
      if (lane >= off) inc = make_int4(inc.x + t.x, inc.y + t.y, inc.z + t.z, inc.w + t.w);
    }
    if (lane == 31) s_wsum[warp] = inc;
    __syncthreads();
    int4 pre = z4, tot = z4;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const int4 t = s_wsum[w];
      if (w < warp) pre = make_int4(pre.x + t.x, pre.y + t.y, pre.z + t.z, pre.w + t.w);
      tot = make_int4(tot.x + t.x, tot.y + t.y, tot.z + t.z, tot.w + t.w);
    }
    const int4 ex0 = make_int4(pre.x + inc.x - v0.x, pre.y + inc.y - v0.y,
                               pre.z + inc.z - v0.z, pre.w + inc.w - v0.w);
    if (g0 < G) {
      s_loff[g0] = ex0;
      s_goff[g0] = ex0.x + ex0.y + ex0.z + ex0.w;
    }
    if (tid == 0) {
      s_goff[G] = tot.x + tot.y + tot.z + tot.w;
      if (c == 0 && a.counts) {
        if (P > 0) a.counts[0] = tot.x;
        if (P > 1) a.counts[1] = tot.y;
        if (P > 2) a.counts[2] = tot.z;
        if (P > 3) a.counts[3] = tot.w;
      }
    }
    __syncthreads();
  }
  const int U = s_goff[G];

  // ---- optional outputs (b, lists, group sums) -------------------------------------
  // team t (16 threads) of CTA c writes group c + C t, so the work is spread one
  // group per CTA first; run where it hides under memory latency (after a
  // round's first copies are issued), by CTAs without GEMV work first thing
  bool outputs_pending = a.b || a.lists || a.grp_sums;
  auto write_outputs = [&]() {
    outputs_pending = false;
    // the same number of passes for every thread (the shuffles span whole warps)
    for (int g0 = 0; g0 < G; g0 += C * (kThreads / kGT)) {
      const int g = g0 + c + C * (tid >> 4);
      const bool act = g < G;
      const uint4 xw = act ? load8(g) : make_uint4(0, 0, 0, 0);
      uint32_t mk[4];
      plane_masks8(xw, t2, P, mk);
      const int row0 = g * kGroup + 8 * gsub;
      if (a.grp_sums) {
        float X, Phi;
        group_sums8(xw, mk, phi, X, Phi);
        if (act && gsub == 0) {
          a.grp_sums[g] = X;
          a.grp_sums[G + g] = Phi;
        }
      }
      if (a.b && act) {
#pragma unroll
        for (int e = 0; e < 8; ++e) a.b[row0 + e] = (uint8_t)(2 * row_level(mk, e));
      }
      if (a.lists) {
        uint32_t cnt = 0;
#pragma unroll
        for (int p = 0; p < 4; ++p) cnt += (uint32_t)__popc(mk[p]) << (8 * p);
        uint32_t inc = cnt;
#pragma unroll
        for (int off = 1; off < kGT; off <<= 1) {
          const uint32_t t = __shfl_up_sync(0xffffffffu, inc, off, kGT);
          if (gsub >= off) inc += t;
        }
        const uint32_t pre = inc - cnt;
        if (act) {
          const int4 lo = s_loff[g];
          const int lofs[4] = {lo.x, lo.y, lo.z, lo.w};
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            if (p >= P) break;
            int pos = lofs[p] + (int)((pre >> (8 * p)) & 255u);
            int32_t *lp = a.lists + (size_t)p * a.d_in;
#pragma unroll
            for (int e = 0; e < 8; ++e)
              if ((mk[p] >> e) & 1u) lp[pos++] = row0 + e;
          }
        }
      }
    }
  };

  if (U == 0) {  // no active row: y = 0 exactly
    if (outputs_pending) write_outputs();
    for (int o = c * kThreads + tid; o < a.d_out; o += C * kThreads) a.y[o] = 0.0f;
    return;
  }

  // m CTAs per tile (m <= U, so no range is empty); more tiles than CTAs: whole tiles in turn
  const int m = a.tiles >= C ? 1 : min(C / a.tiles, U);
  const int C_eff = a.tiles >= C ? C : a.tiles * m;
  if (c >= C_eff) {
    if (outputs_pending) write_outputs();
    return;
  }

  for (int tile = c / m; tile < a.tiles; tile += C_eff / m) {
    const int part = c % m;
    // U <= 2^18 and part < 256: the products fit 32 bits
    const int u0 = part * U / m, u1 = (part + 1) * U / m;
    const int wbase = tile * kTileW;  // first word of the tile in a plane region

    float yacc[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) yacc[t] = 0.0f;

    for (int r0 = u0, r1; r0 < u1; r0 = r1) {
      // the round: units [r0, r1) of at most kRound units and kSlots groups
      int lo = 0, hi = G;  // largest g with goff[g] <= r0 (a non-empty group holds r0)
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_goff[mid] <= r0) lo = mid; else hi = mid;
      }
      const int g_first = lo, g_end = min(g_first + kSlots, G), ng = g_end - g_first;
      r1 = min(u1, min(r0 + kRound, s_goff[g_end]));
      const int n = r1 - r0, n_pad = (n + kK - 1) & ~(kK - 1);
      const int n_steps = n_pad / kK, n_stages = (n_pad + kStage - 1) / kStage;

      __syncthreads();  // the previous round no longer reads the staged data

      // stage s and z rows of the round's groups for this tile (rows past d_out: zero)
#pragma unroll
      for (int i = 0; i < 2 * kSlots * (kTile / 8) / kThreads; ++i) {
        const int q = tid + i * kThreads;  // [which][slot][chunk of 8 halves]
        const int which = q / (kSlots * (kTile / 8)), gi = (q / (kTile / 8)) % kSlots;
        const int ci = q % (kTile / 8), o = tile * kTile + ci * 8;
        if (gi < ng) {
          const uint16_t *src = (which ? a.z : a.s) + (size_t)(g_first + gi) * a.d_out + o;
          uint16_t *dst = (which ? z_st : s_st) + gi * kTile + ci * 8;
          cp_async16(dst, o < a.d_out ? (const void *)src : (const void *)a.s, o < a.d_out ? 16 : 0);
        }
      }
      cp_async_commit();

      // compaction of the round's groups: a 16-thread team per group slot
      if (tid < kSlots * kGT) {
        const int gi = tid >> 4, g = g_first + gi;
        const bool act = gi < ng && s_goff[g] < r1 && s_goff[g + 1] > r0;
        const uint4 xw = act ? load8(g) : make_uint4(0, 0, 0, 0);
        uint32_t mk[4];
        plane_masks8(xw, t2, P, mk);
        // B-column scale: the largest active |x| times 4^(P-1) stays below 2^16
        const uint32_t w[4] = {xw.x, xw.y, xw.z, xw.w};
        uint32_t amax = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if ((mk[0] >> e) & 1u) amax = max(amax, (w[e >> 1] >> (16 * (e & 1))) & 0x7fffu);
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        const int cg = (amax >= 0x7c00u) ? 0 : max(0, (int)(amax >> 10) - 15 + 2 * P - 16);
        float X, Phi;
        group_sums8(xw, mk, phi, X, Phi);
        uint32_t cnt = 0;
#pragma unroll
        for (int p = 0; p < 4; ++p) cnt += (uint32_t)__popc(mk[p]) << (8 * p);
        uint32_t inc = cnt;
#pragma unroll
        for (int off = 1; off < kGT; off <<= 1) {
          const uint32_t t = __shfl_up_sync(0xffffffffu, inc, off, kGT);
          if (gsub >= off) inc += t;
        }
        const uint32_t pre = inc - cnt;
        if (act) {
          const uint32_t gc = s_cnt[g];
          int pbase = s_goff[g];
          const int row0 = g * kGroup + 8 * gsub;
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            if (p >= P) break;
            int u = pbase + (int)((pre >> (8 * p)) & 255u);
            const float xscale = exp2i(2 * (P - 1 - p) - cg);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              if ((mk[p] >> e) & 1u) {
                if (u >= r0 && u < r1) {
                  const float xv = h2f((uint16_t)(w[e >> 1] >> (16 * (e & 1))));
                  s_region[u - r0] = (row0 + e) * P + p;
                  s_ux[u - r0] = (uint32_t)__half_as_ushort(__float2half_rn(xv * xscale)) |
                                 ((uint32_t)gi << 16);
                }
                ++u;
              }
            }
            pbase += (int)((gc >> (8 * p)) & 255u);
          }
        }
        if (gsub == 0) {
          SlotInfo si = {0, 0.0f, 0.0f, 0};
          if (act) {
            si.c = cg;
            si.X = X;
            si.Phi = Phi;
            si.first = (s_goff[g] >= r0 && s_goff[g] < r1) ? 1 : 0;
          }
          s_slot[gi] = si;
        }
      }
      for (int k = n + tid; k < n_pad; k += kThreads) {  // padding units: no load, B = 0
        s_region[k] = -1;
        s_ux[k] = 0u;
      }
      __syncthreads();

      // ring: stage st holds units 32 st .. 32 st + 31 of the round
      auto issue = [&](int st) {
        uint32_t *dst_stage = ring + (size_t)(st % kRing) * (kStage * kRow);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int q = tid + h * kThreads, ul = q >> 4, part16 = q & 15;
          const int k = st * kStage + ul;
          const int region = k < n_pad ? s_region[k] : -1;
          const int word = wbase + part16 * 4;
          uint32_t *dst = dst_stage + ul * kRow + part16 * 4;
          if (region >= 0) {
            const uint32_t *src = a.planes + (size_t)region * a.W + word;
            if (ALIGNED) {
              if (word < a.W) cp_async16(dst, src, 16);
            } else {
#pragma unroll
              for (int v = 0; v < 4; ++v)
                if (word + v < a.W) cp_async4(dst + v, src + v);
            }
          }
        }
      };
      // the first kRingEarly stages, then (x cache released) the rest of the prologue
#pragma unroll 1
      for (int st = 0; st < kRingEarly; ++st) {
        if (st < n_stages) issue(st);
        cp_async_commit();
      }
      if (outputs_pending) write_outputs();  // while the first copies are in flight
      __syncthreads();                       // nobody reads the x cache any more
      xc_valid = false;
#pragma unroll 1
      for (int st = kRingEarly; st < kRing - 1; ++st) {
        if (st < n_stages) issue(st);
        cp_async_commit();
      }

      // B fragments per k-step: lane (fg, tq) holds B[2tq, 2tq+1][fg] and B[2tq+8, 2tq+9][fg];
      // B[k][col] = x'' of unit k if the unit's group slot is col, else 0
      for (int q = tid; q < n_steps * 32; q += kThreads) {
        const int kk = q >> 5, L = q & 31, col = L >> 2, t2i = 2 * (L & 3);
        const uint32_t *ux = s_ux + kk * kK;
        auto bh = [&](uint32_t e) -> uint32_t { return ((int)(e >> 16) == col) ? (e & 0xffffu) : 0u; };
        s_bfrag[q] = make_uint2(bh(ux[t2i]) | (bh(ux[t2i + 1]) << 16),
                                bh(ux[t2i + 8]) | (bh(ux[t2i + 9]) << 16));
      }

      float d[8][4];
#pragma unroll
      for (int bk = 0; bk < 8; ++bk) d[bk][0] = d[bk][1] = d[bk][2] = d[bk][3] = 0.0f;

      for (int st = 0; st < n_stages; ++st) {
        cp_async_wait<kRing - 2>();  // this thread's copies of stage st (and s/z) landed
        __syncthreads();             // everybody's; and stage st-1 is no longer read
        if (st + kRing - 1 < n_stages) issue(st + kRing - 1);
        cp_async_commit();
        const uint32_t *sb = ring + (size_t)(st % kRing) * (kStage * kRow);
        // this warp's k-steps of the stage: h = kp and kp + 2; operands of both first
        uint32_t wv[2][4];
        uint2 bv[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int h = kp + 2 * i, kk = kStage / kK * st + h;
          const uint32_t *pw = sb + (h * kK + 2 * tq) * kRow + 8 * ob + fg;
          wv[i][0] = pw[0];
          wv[i][1] = pw[kRow];
          wv[i][2] = pw[8 * kRow];
          wv[i][3] = pw[9 * kRow];
          bv[i] = s_bfrag[min(kk, n_steps - 1) * 32 + lane];
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int kk = kStage / kK * st + kp + 2 * i;
          if (kk < n_steps) {
            const uint32_t w0 = wv[i][0], w1 = wv[i][1], w2 = wv[i][2], w3 = wv[i][3];
            const uint2 bb = bv[i];
            // m0/m1: outputs 0-7 / 8-15 of units 2tq (low half) and 2tq+1 (high half);
            // m2/m3: the same for units 2tq+8 and 2tq+9; nX = mX >> 6 for t' >= 5
            const uint32_t m0 = prmt(w0, w1, 0x5410u), m1 = prmt(w0, w1, 0x7632u);
            const uint32_t m2 = prmt(w2, w3, 0x5410u), m3 = prmt(w2, w3, 0x7632u);
            const uint32_t n0 = m0 >> 6, n1 = m1 >> 6, n2 = m2 >> 6, n3 = m3 >> 6;
            constexpr uint32_t F = 0x00030003u;
            // block bk: rows fg (output t = 2bk) and fg+8 (t = 2bk+1) of word fg
            mma16816(d[0], m0 & (F << 0), m0 & (F << 2), m2 & (F << 0), m2 & (F << 2), bb.x, bb.y);
            mma16816(d[1], m0 & (F << 4), m0 & (F << 6), m2 & (F << 4), m2 & (F << 6), bb.x, bb.y);
            mma16816(d[2], m0 & (F << 8), n0 & (F << 4), m2 & (F << 8), n2 & (F << 4), bb.x, bb.y);
            mma16816(d[3], n0 & (F << 6), n0 & (F << 8), n2 & (F << 6), n2 & (F << 8), bb.x, bb.y);
            mma16816(d[4], m1 & (F << 0), m1 & (F << 2), m3 & (F << 0), m3 & (F << 2), bb.x, bb.y);
            mma16816(d[5], m1 & (F << 4), m1 & (F << 6), m3 & (F << 4), m3 & (F << 6), bb.x, bb.y);
            mma16816(d[6], m1 & (F << 8), n1 & (F << 4), m3 & (F << 8), n3 & (F << 4), bb.x, bb.y);
            mma16816(d[7], n1 & (F << 6), n1 & (F << 8), n3 & (F << 6), n3 & (F << 8), bb.x, bb.y);
          }
        }
      }
      cp_async_wait<0>();

      // flush: y_t += s (D 2^(24 - pos(t) + c) [+ Phi]) [+ z X] for the lane's two slots
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        const int j = 2 * tq + jj;
        if (j < ng) {
          const SlotInfo si = s_slot[j];
          const uint16_t *srow = s_st + j * kTile + 128 * ob + 16 * fg;
          const uint16_t *zrow = z_st + j * kTile + 128 * ob + 16 * fg;
          float sv[16], zv[16];
          const uint4 s0 = *reinterpret_cast<const uint4 *>(srow);
          const uint4 s1 = *reinterpret_cast<const uint4 *>(srow + 8);
          const uint4 z0 = *reinterpret_cast<const uint4 *>(zrow);
          const uint4 z1 = *reinterpret_cast<const uint4 *>(zrow + 8);
          const uint32_t su[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
          const uint32_t zu[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float2 fs = __half22float2(*reinterpret_cast<const __half2 *>(&su[k]));
            const float2 fz = __half22float2(*reinterpret_cast<const __half2 *>(&zu[k]));
            sv[2 * k] = fs.x;
            sv[2 * k + 1] = fs.y;
            zv[2 * k] = fz.x;
            zv[2 * k + 1] = fz.y;
          }
#pragma unroll
          for (int bk = 0; bk < 8; ++bk) {
            const int t0 = 2 * bk, t1 = 2 * bk + 1;
            float v0 = d[bk][jj] * exp2i(24 - field_pos(t0) + si.c);
            float v1 = d[bk][2 + jj] * exp2i(24 - field_pos(t1) + si.c);
            if (si.first && kp == 0) {
              v0 += si.Phi;
              v1 += si.Phi;
              yacc[t0] = fmaf(zv[t0], si.X, yacc[t0]);
              yacc[t1] = fmaf(zv[t1], si.X, yacc[t1]);
            }
            yacc[t0] = fmaf(sv[t0], v0, yacc[t0]);
            yacc[t1] = fmaf(sv[t1], v1, yacc[t1]);
          }
        }
      }
    }

    // ---- reduce the 4 lanes of a quad (their slots); lane keeps 4 outputs ------
    float keep[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float send = (tq & 1) ? yacc[i] : yacc[8 + i];
      const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
      keep[i] = ((tq & 1) ? yacc[8 + i] : yacc[i]) + recv;
    }
    float fin[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float send = (tq & 2) ? keep[i] : keep[4 + i];
      const float recv = __shfl_xor_sync(0xffffffffu, send, 2);
      fin[i] = ((tq & 2) ? keep[4 + i] : keep[i]) + recv;
    }
    const int ol = 128 * ob + 16 * fg + 8 * (tq & 1) + 4 * (tq >> 1);  // first of 4 outputs
    const int obase = tile * kTile;
    // odd-k warps hand their sums to the even-k warp of the same block
    if (kp == 1) *reinterpret_cast<float4 *>(s_red + ol) = make_float4(fin[0], fin[1], fin[2], fin[3]);
    __syncthreads();
    if (kp == 0) {
      const float4 o = *reinterpret_cast<const float4 *>(s_red + ol);
      fin[0] += o.x;
      fin[1] += o.y;
      fin[2] += o.z;
      fin[3] += o.w;
    }
    if (m == 1) {
      if (kp == 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (obase + ol + i < a.d_out) a.y[obase + ol + i] = fin[i];
      }
      continue;
    }
    // one of m partial tiles: publish it; the tile's last CTA to arrive adds them
    if (kp == 0)
      *reinterpret_cast<float4 *>(a.partials + (size_t)c * kTile + ol) =
          make_float4(fin[0], fin[1], fin[2], fin[3]);
    __syncthreads();
    if (tid == 0) {
      __threadfence();  // the CTA's partial (ordered before by the barrier) is visible first
      s_last = atomicInc(&a.counters[tile], (unsigned)(m - 1)) == (unsigned)(m - 1);
    }
    __syncthreads();
    if (s_last && tid < kTile / 4) {
      __threadfence();
      const int c_first = tile * m;
      float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      const float *src = a.partials + (size_t)c_first * kTile + 4 * tid;
      for (int c0 = 0; c0 < m; c0 += 16) {
        float4 v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          v[i] = (c0 + i < m) ? __ldcg(reinterpret_cast<const float4 *>(src + (size_t)(c0 + i) * kTile))
                              : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          acc.x += v[i].x;
          acc.y += v[i].y;
          acc.z += v[i].z;
          acc.w += v[i].w;
        }
      }
      const float out[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (obase + 4 * tid + i < a.d_out) a.y[obase + 4 * tid + i] = out[i];
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
cudaError_t launch_variant(const DecodeArgs &a, cudaStream_t st) {
  cudaError_t e = ensure_smem_attr((const void *)decode_kernel<ALIGNED>, kSmBytes);
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
  return cudaLaunchKernelEx(&cfg, decode_kernel<ALIGNED>, a);
}

}  // namespace

cudaError_t launch_decode(const uint32_t *planes, const uint16_t *s, const uint16_t *z,
                          const uint16_t *x, const float *theta, const float *phi, int d_in,
                          int d_out, int b_max, float *y, uint8_t *b, int32_t *lists,
                          int32_t *counts, float *grp_sums, void *ws, cudaStream_t st) {
  const WsLayout L = ws_layout(d_in, d_out, b_max);
  char *w = static_cast<char *>(ws);
  DecodeArgs a;
  a.planes = planes;
  a.s = s;
  a.z = z;
  a.x = x;
  a.theta = theta;
  a.phi = phi;
  a.d_in = d_in;
  a.d_out = d_out;
  a.b_max = b_max;
  a.P = b_max / 2;
  a.W = d_out / 16;
  a.G = d_in / kGroup;
  a.tiles = (d_out + kTile - 1) / kTile;
  a.y = y;
  a.b = b;
  a.lists = lists;
  a.counts = counts;
  a.grp_sums = grp_sums;
  a.counters = reinterpret_cast<unsigned *>(w + L.counters);
  a.partials = reinterpret_cast<float *>(w + L.partials);
  cudaError_t e = (a.W % 4 == 0) ? launch_variant<true>(a, st) : launch_variant<false>(a, st);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace grinqh
