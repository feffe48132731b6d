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
//  * Work = 1024-output tiles x row slices.  A unit's tile segment is 256
//    contiguous bytes of its plane region.  Each tile's d_in rows are cut into
//    m = floor(CTAs / tiles) contiguous slices, one per CTA (one wave); every
//    CTA derives its own units from x and theta -- one row per lane, a ballot
//    per plane, a scan of the per-(group, plane, 32-row chunk) counts -- so no
//    other kernel and no global round trip sit between x and the GEMV.  Units
//    are ordered by group, plane, row.
//  * The m partial tiles of a tile meet in global memory: every CTA of the tile
//    publishes its partial as words that are never zero, then adds up its own
//    1/m share of the outputs over the m partials in CTA order (deterministic),
//    polling those words until they are non-zero and zeroing them once read.
//    The launch is cooperative, so all CTAs of a tile are resident together and
//    the polls end whatever else runs on the GPU.
//  * A CTA walks its range in windows of 8 groups and rounds of at most 2048
//    units.  The segments stream through an 8-stage shared-memory ring
//    (cp.async, 16 B per thread and copy, one barrier per 64-unit stage).
//  * The contraction runs on the tensor cores as m16n8k16 MMAs with fp32
//    accumulation: A (16 outputs x 16 units) is built in registers straight
//    from the packed words -- a byte permute pairs the same 16 outputs of two
//    units, one AND per register isolates a 2-bit field pair in the low
//    mantissa bits of two fp16 subnormals, exactly slice * 2^(pos-24) -- and B
//    (16 units x 8) holds x 4^(P-1-p) 2^-c_g in the column of the unit's group
//    slot j in the window (2 (j mod 4) + j / 4), so the 8 columns keep the
//    window's 8 groups apart and the group scales s are applied once per
//    round, not per unit.  One warp covers 128 outputs with
//    8 MMAs per 16 units: 4 shared loads, 4 permutes, 4 shifts, 32 ANDs and
//    8 MMAs per 512 bytes of planes, against about 240 instructions for a
//    scalar fp32 decode of the same bytes.
#include "grinqh_internal.cuh"
#include "pipeline.cuh"

namespace grinqh {
namespace {

using namespace pipe;

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBlocks = 8;            // 128-output blocks of a tile; warps w and w + 8 share one
constexpr int kTile = kDecodeTileOut;  // outputs per CTA tile (8 blocks x 128)
constexpr int kTileW = kTile / 16;    // 64 words = 256 bytes per unit and tile
constexpr int kRow = kTileW + 4;      // shared words per unit row: conflict-free fragment loads
constexpr int kK = 16;                // units per MMA k-step
constexpr int kStage = 64;            // units per ring stage (4 k-steps, 2 per warp)
constexpr int kRing = 8;              // ring stages
constexpr int kXSlot = 6;             // first ring slot of the output CTAs' x cache
constexpr int kRound = 2048;          // units per round
constexpr int kSlots = 8;             // groups per window (the MMA n dimension)
constexpr int kMaxG = kDecodeMaxDin / kGroup;
constexpr int kXCache = 16384;        // rows of x held in shared memory
constexpr int kGT = 16;               // output CTAs: threads per group, one 8-row chunk each
constexpr int kChunkRows = 32;        // GEMV front end: rows per warp chunk, one per lane
constexpr int kSpinLimit = 1 << 20;   // polls of a split-K partial word before giving up (~0.5 s)
constexpr int kOutCtas = 4;           // CTAs that write the optional outputs
constexpr int kMaxGroup = GRINQH_MAX_GROUP;  // linears of one grouped launch

// workspace of a grouped launch: the header (error word), then the partial tiles of
// every CTA (tagged words, zero between launches)
constexpr size_t kGroupWsPartials = (sizeof(WsHeader) + 255) & ~size_t(255);

// shared memory map (bytes)
constexpr size_t kStageBytes = (size_t)kStage * kRow * 4;
constexpr size_t kSmRing = 0;                                               // u32 [kRing][kStage][kRow]
constexpr size_t kSmX = kSmRing + (size_t)kXSlot * kStageBytes;             // fp16 [kXCache] (output
                                                                            // CTAs), ring slots >= kXSlot
constexpr size_t kSmRegion = kSmRing + (size_t)kRing * kStageBytes;         // i32 [kRound]
constexpr size_t kSmUx = kSmRegion + kRound * 4;                            // u32 [kRound]: xh | slot << 16
constexpr size_t kSmBfrag = kSmUx + kRound * 4;                             // uint2 [kRound / kK][32]
constexpr size_t kSmS = kSmBfrag + (size_t)(kRound / kK) * 32 * 8;          // fp16 [kSlots][kTile]
constexpr size_t kSmZ = kSmS + (size_t)kSlots * kTile * 2;                  // fp16 [kSlots][kTile]
constexpr size_t kSmSlot = kSmZ + (size_t)kSlots * kTile * 2;               // SlotInfo [kSlots]
constexpr size_t kSmRed = kSmSlot + kSlots * 16;                            // fp32 [kTile]: odd-k warps
constexpr size_t kSmChunkCnt = kSmRed + (size_t)kTile * 4;                  // i32 [kSlots][4][4]: units per
                                                                            // (slot, plane, chunk)
constexpr size_t kSmWarpSum = kSmChunkCnt + kSlots * 4 * 4 * 4;             // float4 [kWarps]: X, Phi, max|x|
constexpr size_t kSmWarpBal = kSmWarpSum + kWarps * 16;                     // u32 [kWarps][2][4]: ballots
constexpr size_t kSmWarpOff = kSmWarpBal + kWarps * 32;                     // i32 [kWarps][2][4]: first units
constexpr size_t kSmBytes = kSmWarpOff + kWarps * 32;
// the output CTAs keep their counts and scans where the GEMV CTAs have the ring
constexpr size_t kSmCnt = kSmRing;                                          // u32 [kMaxG]: plane counts, bytes
constexpr size_t kSmLoff = kSmCnt + (size_t)kMaxG * 4;                      // int4 [kMaxG]: list offsets
constexpr size_t kSmWsum = kSmLoff + (size_t)kMaxG * 16;                    // int4 [kWarps]
static_assert(kSmBytes <= 227 * 1024, "shared memory");
static_assert((size_t)(kTile / 4 + kMaxCtas) * 16 <= kSmS, "the split-K staging fits below the s/z rows");
static_assert(kTile / 4 + kMaxCtas <= 2 * (kThreads - 32), "split-K: at most two share elements per poller");
static_assert(kTile == kBlocks * 128, "a tile is 8 blocks of 128 outputs");
static_assert((size_t)kXCache * 2 <= (size_t)(kRing - kXSlot) * kStageBytes, "x cache fits");
static_assert(kSmWsum + kWarps * 16 <= kSmX, "output-CTA arrays below the x cache");
static_assert(kSmRing % 16 == 0 && kSmX % 16 == 0 && kSmS % 16 == 0 && kSmZ % 16 == 0 &&
                  kSmBfrag % 16 == 0 && kSmLoff % 16 == 0 && kSmSlot % 16 == 0 &&
                  kSmWsum % 16 == 0 && kSmRed % 16 == 0 && kSmChunkCnt % 16 == 0 &&
                  kSmWarpSum % 16 == 0 && kSmWarpBal % 16 == 0 && kSmWarpOff % 16 == 0,
              "16-byte aligned regions");
static_assert((kStage * 16) % kThreads == 0, "whole 16-byte copies per thread and stage");
static_assert(kStage % (2 * kK) == 0 && kWarps == 2 * kBlocks, "k-steps split between two warps");
static_assert(kMaxG == kThreads, "one group per thread in the output CTAs' scan");
static_assert(kGroup == 4 * kChunkRows && kWarps == 2 * kSlots, "two warps per slot, two chunks each");

struct SlotInfo {
  int c;       // the group's B-column scale exponent: B holds x 4^(P-1-p) 2^-c
  float X;     // sum of x over the active rows of the group in this CTA's row slice
  float Phi;   // sum of x phi_{b/2} over the same rows
  int pad;
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
  float *partials;    // [CTAs of this linear][kTile] tagged words, zero between launches
  int *error;         // the workspace's device error word
  int m;              // CTAs per tile (1: each CTA takes whole tiles in turn)
  int reserve_out;    // set aside the output CTAs (the single call does, whether or not
                      // outputs are asked for, so y never depends on it; a group does not)
};

// The linears of one launch: CTAs [cta_start[j], cta_start[j+1]) run linear j.
struct DecodeGroup {
  int n;
  int cta_start[kMaxGroup + 1];
  DecodeArgs lin[kMaxGroup];
};

// The optional outputs (b, lists, counts, group sums): written by CTAs that
// take no part in the GEMV, so they cost the GEMV nothing but those CTAs' SMs.
// Every output CTA counts the units of every group per plane and scans them
// (the list offsets); then CTA k of K writes the groups g = k mod K.
__device__ __forceinline__ void write_outputs(const DecodeArgs &a, unsigned char *smem, int k,
                                              int K, const __half2 (&t2)[4],
                                              const float (&phi)[5]) {
  uint16_t *xc = reinterpret_cast<uint16_t *>(smem + kSmX);
  uint32_t *s_cnt = reinterpret_cast<uint32_t *>(smem + kSmCnt);
  int4 *s_loff = reinterpret_cast<int4 *>(smem + kSmLoff);
  int4 *s_wsum = reinterpret_cast<int4 *>(smem + kSmWsum);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gsub = tid & (kGT - 1);
  const int P = a.P, G = a.G;
  int xc_base = 0;
  auto load8 = [&](int g) -> uint4 {
    const int row = g * kGroup + 8 * gsub;
    if (row >= xc_base && row < xc_base + kXCache)
      return *reinterpret_cast<const uint4 *>(xc + (row - xc_base));
    return __ldg(reinterpret_cast<const uint4 *>(a.x + row));
  };
  // units per (group, plane), x in chunks of kXCache rows
  for (int base = 0; base < a.d_in; base += kXCache) {
    const int rows = min(kXCache, a.d_in - base);
    if (base > 0) __syncthreads();
    for (int q = tid; q < rows / 8; q += kThreads) cp_async16(xc + 8 * q, a.x + base + 8 * q, 16);
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    xc_base = base;
    const int g_lo = base / kGroup, g_hi = (base + rows) / kGroup;
    for (int g0 = g_lo; g0 < g_hi; g0 += kThreads / kGT) {
      const int g = g0 + (tid >> 4);
      uint32_t mk[4] = {0u, 0u, 0u, 0u};
      if (g < g_hi) plane_masks8(load8(g), t2, P, mk);
      uint32_t packed = 0;
#pragma unroll
      for (int p = 0; p < 4; ++p) packed += (uint32_t)__popc(mk[p]) << (8 * p);
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) packed += __shfl_xor_sync(0xffffffffu, packed, off);
      if (gsub == 0 && g < g_hi) s_cnt[g] = packed;
    }
  }
  __syncthreads();
  // exclusive scans over groups: per-plane list offsets
  {
    const int g0 = tid;  // kMaxG = kThreads
    const uint32_t v = g0 < G ? s_cnt[g0] : 0u;
    const int4 v0 = make_int4(v & 255u, (v >> 8) & 255u, (v >> 16) & 255u, v >> 24);
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
    int4 pre = make_int4(0, 0, 0, 0), tot = pre;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const int4 t = s_wsum[w];
      if (w < warp) pre = make_int4(pre.x + t.x, pre.y + t.y, pre.z + t.z, pre.w + t.w);
      tot = make_int4(tot.x + t.x, tot.y + t.y, tot.z + t.z, tot.w + t.w);
    }
    if (g0 < G)
      s_loff[g0] = make_int4(pre.x + inc.x - v0.x, pre.y + inc.y - v0.y, pre.z + inc.z - v0.z,
                             pre.w + inc.w - v0.w);
    if (tid == 0 && k == 0 && a.counts) {
      if (P > 0) a.counts[0] = tot.x;
      if (P > 1) a.counts[1] = tot.y;
      if (P > 2) a.counts[2] = tot.z;
      if (P > 3) a.counts[3] = tot.w;
    }
    __syncthreads();
  }
  // team t (16 threads) of output CTA k writes group k + K (t + 32 pass)
  for (int g0 = 0; g0 + k < G; g0 += K * (kThreads / kGT)) {
    const int g = g0 + k + K * (tid >> 4);
    const bool act = g < G;
    const uint4 xw = act ? load8(g) : make_uint4(0, 0, 0, 0);
    uint32_t mk[4] = {0u, 0u, 0u, 0u};
    if (act) plane_masks8(xw, t2, P, mk);
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
}

template <bool ALIGNED, bool GROUPED>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ DecodeGroup g) {
  extern __shared__ __align__(128) unsigned char smem[];
  uint32_t *ring = reinterpret_cast<uint32_t *>(smem + kSmRing);
  int32_t *s_region = reinterpret_cast<int32_t *>(smem + kSmRegion);
  uint32_t *s_ux = reinterpret_cast<uint32_t *>(smem + kSmUx);
  uint2 *s_bfrag = reinterpret_cast<uint2 *>(smem + kSmBfrag);
  uint16_t *s_st = reinterpret_cast<uint16_t *>(smem + kSmS);
  uint16_t *z_st = reinterpret_cast<uint16_t *>(smem + kSmZ);
  SlotInfo *s_slot = reinterpret_cast<SlotInfo *>(smem + kSmSlot);
  float *s_red = reinterpret_cast<float *>(smem + kSmRed);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int fg = lane >> 2, tq = lane & 3;  // MMA fragment row group and column pair
  const int ob = warp & (kBlocks - 1);      // the warp's 128-output block of the tile
  const int kp = warp / kBlocks;            // ... and its k-step parity
  // this CTA's linear, and the CTAs that linear has (a single linear: a fixed index,
  // so its arguments are read at fixed offsets)
  int jl = 0;
  if (GROUPED) {
#pragma unroll
    for (int i = 1; i < kMaxGroup; ++i) jl += (i < g.n && (int)blockIdx.x >= g.cta_start[i]) ? 1 : 0;
  }
  const DecodeArgs &a = g.lin[jl];
  const int C = g.cta_start[jl + 1] - g.cta_start[jl], c = (int)blockIdx.x - g.cta_start[jl];
  const int P = a.P;

  // ---- what depends on the shapes only: computed before the wait below, so it
  // overlaps the tail of the kernel launched before (programmatic launch) ----
  // the last CTAs write the optional outputs, the others run the GEMV; they are
  // set aside whether or not outputs are asked for, so y does not depend on it
  const int n_out = !a.reserve_out ? 0 : (C > 2 * kOutCtas ? kOutCtas : 1);
  const int C_g = C - n_out;
  // tiles x row slices: m CTAs per tile, CTA `part` takes the 8-row chunks
  // [R8 part / m, R8 (part + 1) / m); more tiles than CTAs: whole tiles in turn
  const bool many = a.tiles >= C_g;
  const int m = many ? 1 : a.m;
  const int C_eff = many ? C_g : a.tiles * m;
  const int R8 = a.d_in / 8;
  const int part = many ? 0 : c % m;
  const int q_lo = R8 * part / m, q_hi = R8 * (part + 1) / m;  // R8 <= 2^13, part < 2^8
  const int row_lo = 8 * q_lo, row_hi = 8 * q_hi;
  const int tile_first = many ? c : c / m, tile_step = many ? C_g : a.tiles;
  const int g_first = row_lo / kGroup;
  auto window_groups = [&](int g_w) { return min(kSlots, (row_hi + kGroup - 1) / kGroup - g_w); };

  // the s and z rows of a window's groups for a tile, to shared memory (past d_out: zero)
  auto stage_sz = [&](int tile, int g_w, int ng) {
#pragma unroll
    for (int i = 0; i < 2 * kSlots * (kTile / 8) / kThreads; ++i) {
      const int q = tid + i * kThreads;  // [which][slot][chunk of 8 halves]
      const int which = q / (kSlots * (kTile / 8)), gi = (q / (kTile / 8)) % kSlots;
      const int ci = q % (kTile / 8), o = tile * kTile + ci * 8;
      if (gi < ng) {
        const uint16_t *src = (which ? a.z : a.s) + (size_t)(g_w + gi) * a.d_out + o;
        uint16_t *dst = (which ? z_st : s_st) + gi * kTile + ci * 8;
        cp_async16(dst, o < a.d_out ? (const void *)src : (const void *)a.s, o < a.d_out ? 16 : 0);
      }
    }
  };

  // ---- theta and phi are not written by the kernel launched just before (a
  // condition of the call), so they are fetched before waiting for it; x, planes,
  // s and z only after ----
  float th_raw[4], phi[5];
#pragma unroll
  for (int k = 0; k < 4; ++k) th_raw[k] = (k < P) ? a.theta[k] : __int_as_float(0x7fc00000);
#pragma unroll
  for (int k = 0; k <= 4; ++k) {
    const float def = (2 * k < a.b_max) ? exp2i(a.b_max - 2 * k - 1) : 0.0f;
    phi[k] = (k <= P) ? (a.phi ? a.phi[k] : def) : 0.0f;
  }
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");

  // the first window's x (the lane's two rows): the loads go out before anything
  // else, and the thresholds are sorted while they are in flight
  uint32_t xr_first = 0u, inb_first = 0u;
  if (c < C_eff && c < C_g) {
    const int slot = warp >> 1, cc0 = 2 * (warp & 1);
    if (slot < window_groups(g_first)) {
      const int row0 = (g_first + slot) * kGroup + kChunkRows * cc0 + lane;
#pragma unroll
      for (int ci = 0; ci < 2; ++ci) {
        const int row = row0 + kChunkRows * ci;
        if (row >= row_lo && row < row_hi) {
          xr_first |= (uint32_t)__ldg(a.x + row) << (16 * ci);
          inb_first |= 1u << ci;
        }
      }
    }
  }

  __half2 t2[4];
  sort_thresholds(th_raw, t2);

  if (c >= C_g) {
    if (a.b || a.lists || a.counts || a.grp_sums) write_outputs(a, smem, c - C_g, n_out, t2, phi);
    return;
  }
  if (c >= C_eff) return;

  int *s_ccnt = reinterpret_cast<int *>(smem + kSmChunkCnt);
  float4 *s_wsum = reinterpret_cast<float4 *>(smem + kSmWarpSum);
  uint4 *s_wbal = reinterpret_cast<uint4 *>(smem + kSmWarpBal);
  int4 *s_woff = reinterpret_cast<int4 *>(smem + kSmWarpOff);

  for (int tile = tile_first; tile < a.tiles; tile += tile_step) {
    const int wbase = tile * kTileW;  // first word of the tile in a plane region
    float yacc[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) yacc[t] = 0.0f;

    // windows of kSlots groups over the slice
    for (int g_w = g_first; g_w * kGroup < row_hi; g_w += kSlots) {
      const int ng = window_groups(g_w);
      if (g_w != g_first || tile != tile_first)
        __syncthreads();  // the previous window no longer reads the staged data

      // ---- compaction, one row per lane: warp w takes chunks cc = 2 (w mod 2) and
      // 2 (w mod 2) + 1 (32 rows each) of group slot w / 2, for every plane.  The
      // window's units are ordered by slot, plane, chunk, row (any order works
      // within a round: each unit carries its slot into B) ----
      const int slot = warp >> 1, cc0 = 2 * (warp & 1);
      const bool live = slot < ng;  // warp-uniform
      const int row0 = (g_w + slot) * kGroup + kChunkRows * cc0 + lane;  // the lane's row in chunk cc0
      uint32_t xr = 0u, inb = 0u;  // the lane's two x values (fp16 pair) and which are in the slice
      uint32_t bal[2][4] = {{0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}};
      if (g_w == g_first && tile == tile_first) {
        xr = xr_first;
        inb = inb_first;
      } else if (live) {
#pragma unroll
        for (int ci = 0; ci < 2; ++ci) {
          const int row = row0 + kChunkRows * ci;
          if (row >= row_lo && row < row_hi) {
            xr |= (uint32_t)__ldg(a.x + row) << (16 * ci);
            inb |= 1u << ci;
          }
        }
      }
      // s and z are needed only at the flush: their copies go out after the x loads
      stage_sz(tile, g_w, ng);
      cp_async_commit();
      if (live) {
        // plane p of a row is loaded when b > 2p, i.e. |x| >= the p-th smallest threshold
        float X = 0.0f, Phi = 0.0f;
        uint32_t amax = 0u;
#pragma unroll
        for (int ci = 0; ci < 2; ++ci) {
          const uint32_t xb = (xr >> (16 * ci)) & 0xffffu;
          const __half ax = __ushort_as_half((uint16_t)(xb & 0x7fffu));
          int lev = 0;
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            const bool act = ((inb >> ci) & 1u) && __hge(ax, __low2half(t2[p]));
            bal[ci][p] = __ballot_sync(0xffffffffu, act);
            lev += act ? 1 : 0;
          }
          if (lev > 0) {
            const float xv = __half2float(__ushort_as_half((uint16_t)xb));
            X += xv;
            Phi = __fmaf_rn(xv, pick_phi(phi, lev), Phi);
            amax = max(amax, xb & 0x7fffu);
          }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          X += __shfl_xor_sync(0xffffffffu, X, off);
          Phi += __shfl_xor_sync(0xffffffffu, Phi, off);
        }
        amax = __reduce_max_sync(0xffffffffu, amax);
        if (lane == 0) s_wsum[warp] = make_float4(X, Phi, __uint_as_float(amax), 0.0f);
      }
      // units per (slot, plane, chunk); lanes 0-7 write the warp's eight
#pragma unroll
      for (int ci = 0; ci < 2; ++ci)
#pragma unroll
        for (int p = 0; p < 4; ++p)
          if (lane == 4 * ci + p) s_ccnt[(4 * slot + p) * 4 + cc0 + ci] = __popc(bal[ci][p]);
      __syncthreads();

      // exclusive prefix over the (slot, plane, chunk) counts: lane L holds the four
      // chunks of (slot, plane) = (L / 4, L mod 4)
      int Nw;
      {
        const int4 cv = reinterpret_cast<const int4 *>(s_ccnt)[lane];
        const int t = cv.x + cv.y + cv.z + cv.w;
        int inc = t;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int u = __shfl_up_sync(0xffffffffu, inc, off);
          if (lane >= off) inc += u;
        }
        Nw = __shfl_sync(0xffffffffu, inc, 31);
        // first units of chunks cc0 and cc0 + 1 of the lane's (slot, plane)
        const int o0 = inc - t + (cc0 ? cv.x + cv.y : 0);
        const int o1 = o0 + (cc0 ? cv.z : cv.x);
        int offv[2][4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          offv[0][p] = __shfl_sync(0xffffffffu, o0, 4 * slot + p);
          offv[1][p] = __shfl_sync(0xffffffffu, o1, 4 * slot + p);
        }
        if (live && lane == 0) {
          s_wbal[2 * warp] = make_uint4(bal[0][0], bal[0][1], bal[0][2], bal[0][3]);
          s_wbal[2 * warp + 1] = make_uint4(bal[1][0], bal[1][1], bal[1][2], bal[1][3]);
          s_woff[2 * warp] = make_int4(offv[0][0], offv[0][1], offv[0][2], offv[0][3]);
          s_woff[2 * warp + 1] = make_int4(offv[1][0], offv[1][1], offv[1][2], offv[1][3]);
        }
      }
      // the slot's B-column scale exponent: the largest active |x| of the slot, times
      // 4^(P-1), stays below 2^16; and its group sums (for the flush)
      int cg = 0;
      if (live) {
        const float4 w0 = s_wsum[2 * slot], w1 = s_wsum[2 * slot + 1];
        const uint32_t am = max(__float_as_uint(w0.z), __float_as_uint(w1.z));
        cg = (am >= 0x7c00u) ? 0 : max(0, (int)(am >> 10) - 15 + 2 * P - 16);
        if (cc0 == 0 && lane == 0) {
          SlotInfo si;
          si.c = cg;
          si.X = w0.x + w1.x;
          si.Phi = w0.y + w1.y;
          si.pad = 0;
          s_slot[slot] = si;
        }
      }
      __syncwarp();

      for (int k0 = 0; k0 < Nw; k0 += kRound) {
        // the round is padded to whole stages with units whose B entries are 0 and
        // which load nothing: every warp runs every k-step of a stage unconditionally
        const int n = min(kRound, Nw - k0), n_pad = (n + kStage - 1) & ~(kStage - 1);
        const int n_steps = n_pad / kK, n_stages = n_pad / kStage;
        static_assert(kRound % kStage == 0, "rounds of whole stages");
        if (k0 > 0) __syncthreads();  // the previous round no longer reads the records

        // the records of the warp's units that fall in [k0, k0 + n): plane region
        // and x 4^(P-1-p) 2^-c rounded to fp16 (a power-of-two product: exact unless
        // the result is subnormal, then rounded as fp16 does) with the slot
        if (live) {
          const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
          for (int ci = 0; ci < 2; ++ci) {
            const uint4 bv = s_wbal[2 * warp + ci];
            const int4 ov = s_woff[2 * warp + ci];
            const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
            const int ow[4] = {ov.x, ov.y, ov.z, ov.w};
            const __half xh = __ushort_as_half((uint16_t)((xr >> (16 * ci)) & 0xffffu));
            const int rp = (row0 + kChunkRows * ci) * P;
#pragma unroll
            for (int p = 0; p < 4; ++p) {
              const int u = ow[p] + __popc(bw[p] & lt);
              if (((bw[p] >> lane) & 1u) && u >= k0 && u < k0 + n) {
                const __half sc = __ushort_as_half((uint16_t)((15 + 2 * (P - 1 - p) - cg) << 10));
                s_region[u - k0] = rp + p;
                s_ux[u - k0] = (uint32_t)__half_as_ushort(__hmul(xh, sc)) | ((uint32_t)slot << 16);
              }
            }
          }
        }
        for (int k = n + tid; k < n_pad; k += kThreads) {  // padding units: no load, B = 0
          s_region[k] = -1;
          s_ux[k] = 0u;
        }
        __syncthreads();

        // B fragments per k-step: lane (fg, tq) holds B[2tq, 2tq+1][fg] and B[2tq+8, 2tq+9][fg];
        // B[k][col] = x'' of unit k if the unit's group slot is col / 2 + 4 (col mod 2), else
        // 0.  So D column 2q holds slot q and column 2q+1 slot q+4, and a window of at
        // most 4 groups leaves the second slot of every lane empty (skipped by the flush)
        auto build_bfrag = [&]() {
          for (int q = tid; q < n_steps * 32; q += kThreads) {
            const int kk = q >> 5, L = q & 31, col = L >> 2, t2i = 2 * (L & 3);
            const int slot_c = (col >> 1) + 4 * (col & 1);
            const uint32_t *ux = s_ux + kk * kK;
            auto bh = [&](uint32_t e) -> uint32_t { return ((int)(e >> 16) == slot_c) ? (e & 0xffffu) : 0u; };
            s_bfrag[q] = make_uint2(bh(ux[t2i]) | (bh(ux[t2i + 1]) << 16),
                                    bh(ux[t2i + 8]) | (bh(ux[t2i + 9]) << 16));
          }
        };

        float d[8][4];
#pragma unroll
        for (int bk = 0; bk < 8; ++bk) d[bk][0] = d[bk][1] = d[bk][2] = d[bk][3] = 0.0f;

        // this warp's MMA work on ring stage st (units 64 st .. 64 st + 63 of the round,
        // held in `sb`): its k-steps h = kp and kp + 2, operands of both first
        constexpr int kStepsPerWarp = kStage / kK / 2;  // k-steps of a stage per warp
        auto compute = [&](const uint32_t *sb, int st) {
          uint32_t wv[kStepsPerWarp][4];
          uint2 bv[kStepsPerWarp];
#pragma unroll
          for (int i = 0; i < kStepsPerWarp; ++i) {
            const int h = kp + 2 * i, kk = kStage / kK * st + h;
            const uint32_t *pw = sb + (h * kK + 2 * tq) * kRow + 8 * ob + fg;
            wv[i][0] = pw[0];
            wv[i][1] = pw[kRow];
            wv[i][2] = pw[8 * kRow];
            wv[i][3] = pw[9 * kRow];
            bv[i] = s_bfrag[kk * 32 + lane];
          }
#pragma unroll
          for (int i = 0; i < kStepsPerWarp; ++i) {
            {
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
        };

        // ---- cp.async ring: 16 threads copy a unit's segment (16-byte copies; 4-byte
        // copies for layouts whose rows are not 16-byte aligned) ----
        auto issue = [&](int st) {
          uint32_t *dst_stage = ring + (size_t)(st % kRing) * (kStage * kRow);
#pragma unroll
          for (int h = 0; h < kStage * 16 / kThreads; ++h) {
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
#pragma unroll
        for (int st = 0; st < kRing - 1; ++st) {
          if (st < n_stages) issue(st);
          cp_async_commit();
        }
        build_bfrag();
        for (int st = 0; st < n_stages; ++st) {
          cp_async_wait<kRing - 2>();  // this thread's copies of stage st (and s/z) landed
          __syncthreads();             // everybody's; and stage st-1 is no longer read
          if (st + kRing - 1 < n_stages) issue(st + kRing - 1);
          cp_async_commit();
          compute(ring + (size_t)(st % kRing) * (kStage * kRow), st);
        }
        cp_async_wait<0>();

        // flush: y_t += s (D 2^(24 - pos(t) + c) [+ Phi]) [+ z X] for the lane's two slots
        // (tq and tq + 4); the slice's group terms once per window (first round, even-k warps)
        const bool terms = k0 == 0 && kp == 0;
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int j = tq + 4 * jj;
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
              if (terms) {
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
    __syncthreads();  // s_red of the previous tile is consumed
    if (kp == 1) *reinterpret_cast<float4 *>(s_red + ol) = make_float4(fin[0], fin[1], fin[2], fin[3]);
    __syncthreads();
    if (kp == 0) {
      const float4 o = *reinterpret_cast<const float4 *>(s_red + ol);
      fin[0] += o.x;
      fin[1] += o.y;
      fin[2] += o.z;
      fin[3] += o.w;
    }
    if (m == 1) {  // the whole tile's rows: y directly
      if (kp == 0 && obase + ol < a.d_out)  // d_out % 16 == 0: the 4 outputs are wholly in or out
        for (int i = 0; i < 4; ++i) a.y[obase + ol + i] = fin[i];
      continue;
    }
    // ---- split-K: the m partial tiles of a tile meet in global memory.  Every CTA
    // publishes its partial as tagged words (never zero; see tag_word), then adds up
    // its own 1/m share of the tile's outputs over the m partials in CTA order
    // (deterministic), polling each word until it is non-zero, and sets the words it
    // consumed back to zero for the next launch.  The data are their own flags: no
    // fence or counter sits between the last partial and its readers.  The launch is
    // cooperative, so every CTA of the tile is resident and every wait ends; the poll
    // bound only guards against a broken launch. ----
    const int c_first = (c / m) * m;
    uint32_t *part_w = reinterpret_cast<uint32_t *>(a.partials);
    uint32_t canary = 0u;
    if (kp == 0) {
      uint32_t *dst = part_w + (size_t)c * kTile + ol;
      const uint4 t = make_uint4(tag_word(fin[0]), tag_word(fin[1]), tag_word(fin[2]), tag_word(fin[3]));
      if (ol == 0) {
        // the partial's first word must still be zero from the last launch: a workspace
        // that was not left zeroed shows up here (checked after the share is summed)
        canary = atomicExch(dst, t.x);
        st_relaxed_u32(dst + 1, t.y);
        st_relaxed_u32(dst + 2, t.z);
        st_relaxed_u32(dst + 3, t.w);
      } else {
        st_relaxed_v4(dst, t);
      }
    }
    // this CTA's share: quads [Q part / m, Q (part + 1) / m) of the tile's Q = kTile / 4;
    // m <= kMaxCtas <= Q, so every share is non-empty, and m nq <= Q + m
    static_assert(kMaxCtas <= kTile / 4, "split-K shares");
    const int q0 = (kTile / 4) * part / m, nq = (kTile / 4) * (part + 1) / m - q0;
    float4 *s_fix = reinterpret_cast<float4 *>(smem + kSmRing);  // [m][nq]; the ring is idle
    // pollers: threads 32 and up (warp 0 holds the canary's exchange), element e of
    // the share (partial e / nq, quad e mod nq) on thread 32 + e mod (kThreads - 32)
    const int pt = tid - 32;
    auto elem = [&](int e) -> uint32_t * {
      const int cc = e / nq, qq = e - cc * nq;
      return part_w + (size_t)(c_first + cc) * kTile + 4 * (q0 + qq);
    };
    int gave_up = 0;
    if (pt >= 0) {
      for (int e = pt; e < m * nq && !gave_up; e += kThreads - 32) {
        const uint32_t *src = elem(e);
        uint4 v;
        for (int polls = 0;; ++polls) {
          v = ld_relaxed_v4(src);
          if (v.x != 0u && v.y != 0u && v.z != 0u && v.w != 0u) break;
          if (polls == kSpinLimit) {
            gave_up = 1;
            break;
          }
          __nanosleep(20);
        }
        s_fix[e] = make_float4(__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z),
                               __uint_as_float(v.w));
      }
    }
    if (__syncthreads_or(gave_up)) {
      if (tid == 0) atomicCAS(a.error, 0, kDevErrSplitKTimeout);
      continue;  // y of this share is not written; the words stay for the error path
    }
    if (pt >= 0)
      for (int e = pt; e < m * nq; e += kThreads - 32) st_relaxed_v4(elem(e), make_uint4(0u, 0u, 0u, 0u));  // consumed
    if (pt >= 0 && pt < nq) {
      float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      for (int cc = 0; cc < m; ++cc) acc = f4add(acc, s_fix[cc * nq + pt]);  // in CTA order
      const int o = obase + 4 * (q0 + pt);
      if (o < a.d_out) {
        a.y[o] = acc.x;
        a.y[o + 1] = acc.y;
        a.y[o + 2] = acc.z;
        a.y[o + 3] = acc.w;
      }
    }
    if (canary != 0u) atomicCAS(a.error, 0, kDevErrSplitKTimeout);
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

template <bool ALIGNED, bool GROUPED>
cudaError_t launch_variant(const DecodeGroup &g, cudaStream_t st) {
  cudaError_t e = ensure_smem_attr((const void *)decode_kernel<ALIGNED, GROUPED>, kSmBytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(g.cta_start[g.n]);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmBytes;
  cfg.stream = st;
  // programmatic dependent launch, and cooperative: every CTA is resident at once, so
  // the split-K waits on the other CTAs of a tile always end
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeCooperative;
  attr[1].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, decode_kernel<ALIGNED, GROUPED>, g);
}

DecodeArgs make_args(const uint32_t *planes, const uint16_t *s, const uint16_t *z,
                     const uint16_t *x, const float *theta, const float *phi, int d_in, int d_out,
                     int b_max, float *y, int n_gemv) {
  DecodeArgs a = {};
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
  a.m = a.tiles >= n_gemv ? 1 : n_gemv / a.tiles;  // CTAs per tile (1: whole tiles in turn)
  a.y = y;
  return a;
}

template <bool GROUPED>
cudaError_t launch_group(DecodeGroup &g, cudaStream_t st) {
  bool aligned = true;  // 16-byte plane copies need every linear's rows 16-byte aligned
  for (int j = 0; j < g.n; ++j) aligned = aligned && g.lin[j].W % 4 == 0;
  cudaError_t e = aligned ? launch_variant<true, GROUPED>(g, st) : launch_variant<false, GROUPED>(g, st);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const uint32_t *planes, const uint16_t *s, const uint16_t *z,
                          const uint16_t *x, const float *theta, const float *phi, int d_in,
                          int d_out, int b_max, float *y, uint8_t *b, int32_t *lists,
                          int32_t *counts, float *grp_sums, void *ws, cudaStream_t st) {
  const WsLayout L = ws_layout(d_in, d_out, b_max);
  char *w = static_cast<char *>(ws);
  return launch_decode_split(planes, s, z, x, theta, phi, d_in, d_out, b_max, y, b, lists, counts,
                             grp_sums, reinterpret_cast<float *>(w + L.dpartials),
                             &reinterpret_cast<WsHeader *>(w)->error, st);
}

cudaError_t launch_decode_split(const uint32_t *planes, const uint16_t *s, const uint16_t *z,
                                const uint16_t *x, const float *theta, const float *phi, int d_in,
                                int d_out, int b_max, float *y, uint8_t *b, int32_t *lists,
                                int32_t *counts, float *grp_sums, float *partials, int *error,
                                cudaStream_t st) {
  DecodeGroup g = {};
  g.n = 1;
  g.cta_start[0] = 0;
  const int C = device_sms();
  g.cta_start[1] = C;
  DecodeArgs &a = g.lin[0];
  a = make_args(planes, s, z, x, theta, phi, d_in, d_out, b_max, y,
                C - (C > 2 * kOutCtas ? kOutCtas : 1));
  a.b = b;
  a.lists = lists;
  a.counts = counts;
  a.grp_sums = grp_sums;
  a.partials = partials;
  a.error = error;
  a.reserve_out = 1;
  return launch_group<false>(g, st);
}

size_t group_ws_bytes() { return kGroupWsPartials + (size_t)kMaxCtas * kTile * 4; }

cudaError_t launch_decode_group(int n, const grinqh_linear *lins, void *ws, cudaStream_t st) {
  char *w = static_cast<char *>(ws);
  DecodeGroup g = {};
  g.n = n;
  // CTAs in proportion to each linear's plane bytes (tiles x d_in x P), at least one each
  const int C = device_sms();
  double tot = 0.0, wgt[kMaxGroup];
  for (int j = 0; j < n; ++j) {
    const int tiles = (lins[j].d_out + kTile - 1) / kTile;
    wgt[j] = (double)tiles * lins[j].d_in * (lins[j].b_max / 2);
    tot += wgt[j];
  }
  int cnt[kMaxGroup], used = 0;
  for (int j = 0; j < n; ++j) {
    cnt[j] = (int)((double)C * wgt[j] / tot);
    if (cnt[j] < 1) cnt[j] = 1;
    used += cnt[j];
  }
  while (used > C) {  // rounding up the small ones may overshoot: trim the largest
    int big = 0;
    for (int j = 1; j < n; ++j)
      if (cnt[j] > cnt[big]) big = j;
    --cnt[big];
    --used;
  }
  for (int j = 0; j < n; ++j) {
    const grinqh_linear &l = lins[j];
    g.cta_start[j + 1] = g.cta_start[j] + cnt[j];
    DecodeArgs &a = g.lin[j];
    a = make_args(l.planes, l.s, l.z, l.x, l.theta, l.phi, l.d_in, l.d_out, l.b_max, l.y, cnt[j]);
    a.partials = reinterpret_cast<float *>(w + kGroupWsPartials) + (size_t)g.cta_start[j] * kTile;
    a.error = &reinterpret_cast<WsHeader *>(w)->error;
    a.reserve_out = 0;
  }
  return launch_group<true>(g, st);
}

}  // namespace grinqh
