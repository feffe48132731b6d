// batch.cu -- the small-batch GRINQH decode step (B <= 8 tokens) in one kernel.
//
// What it computes ("GRINQH: Graded Input-Based Quantization Hierarchy",
// Limitations and outlook: beyond batch 1 the requests' active channels
// differ, so a batched step reads the union of their planes): every token t
// has its own widths b_t(i) = 2 #{k : theta_k <= |x_t(i)|} and its own
//   y_t,o = sum_{i : b_t(i) > 0} x_t(i) (s_{g,o} (Q_{b_t(i)}(i, o) + phi_{b_t(i)}) + z_{g,o}),
// exactly the batch-1 step token by token.  Each row's planes are read once, for
// the union width u_i = max_t b_t(i), and each 2-bit field is decoded once for
// all tokens.
//
// How (the pipeline of decode.cu, with tokens in the MMA's n dimension):
//  * A unit is a (row, plane) pair with u_i > 2p.  Its B row holds, for token t,
//    x_t(i) 4^(P-1-p) 2^-c_g where b_t(i) > 2p and 0 elsewhere: a token whose own
//    width stops above plane p does not see that plane, which is exactly the
//    truncation of Q to its width.  So one A fragment (the decoded fields) serves
//    every token, and the MMA's 8 columns are the 8 tokens.
//  * The units of a window (8 groups) are ordered by group, plane, row, and each
//    group's units are padded to a multiple of 32 (two k-steps), so every half
//    stage belongs to one group: an MMA warp scales its accumulators by the
//    group's s and adds them into its outputs when the group of the half stage
//    it starts changes.  The group
//    terms s Phi_{g,t} + z X_{g,t} (per token) are added once per window.
//  * Copies, mbarrier ring and split-K follow the batch-1 kernel: four copy warps
//    stream 256-byte segments with 16-byte cp.async copies, eight MMA warps (one
//    per 128-output block) decode them, and the partial tiles of a tile's CTAs
//    meet in global memory, where the last arrival sums them in a fixed order
//    (y is deterministic).
#include "grinqh_internal.cuh"
#include "pipeline.cuh"

namespace grinqh {
namespace {

using namespace pipe;

constexpr int kNB = 8;                          // tokens: the MMA's n dimension
constexpr int kMmaWarps = 8;                    // one per 128-output block: all k-steps of a stage
constexpr int kMmaThreads = kMmaWarps * 32;
constexpr int kCopyWarps = 4;                   // warps that stream the planes into the ring
constexpr int kCopyThreads = kCopyWarps * 32;
constexpr int kThreads = kMmaThreads + kCopyThreads;  // 12 warps: 3 per SM sub-partition, so the
                                                      // MMA warps keep 64 accumulators in registers
constexpr int kChunks = kGroup / 32;            // 32-row chunks of a group: one warp takes a group
constexpr int kBlocks = 8;
constexpr int kTile = 1024;
constexpr int kTileW = kTile / 16;
constexpr int kRow = kTileW + 4;
constexpr int kK = 16;
constexpr int kStage = 64;
constexpr int kRing = 8;
constexpr int kRound = 1024;                    // units per round
constexpr int kSlots = 8;                       // groups per window
constexpr int kChunkRows = 32;
constexpr int kPolls = 1 << 20;                 // bounded poll for a missing split-K partial
constexpr int kGrpPad = 2 * kK;
constexpr int kFixParts = 32;                   // partial tiles staged per pass of the split-K sum                 // a group's units are padded to this: a warp's half stage

// workspace: header, 64-bit arrival words, partial tiles [CTA][kNB][kTile]
constexpr size_t kWsCounters = sizeof(WsHeader);
constexpr size_t kWsPartials = (kWsCounters + (size_t)kMaxTiles * 4 + 255) & ~size_t(255);
constexpr size_t kWsBytes = kWsPartials + (size_t)kMaxCtas * kNB * kTile * 4;

// shared memory map (bytes)
constexpr size_t kStageBytes = (size_t)kStage * kRow * 4;
constexpr size_t kSmRing = 0;                                               // u32 [kRing][kStage][kRow]
constexpr size_t kSmRegion = kSmRing + (size_t)kRing * kStageBytes;         // i32 [kRound]
constexpr size_t kSmUx = kSmRegion + kRound * 4;                            // uint4 [kRound]: 8 fp16 B values
constexpr size_t kSmBfrag = kSmUx + (size_t)kRound * 16;                    // uint2 [kRound / kK][32]
constexpr size_t kSmKgrp = kSmBfrag + (size_t)(kRound / kK) * 32 * 8;       // i32 [kRound / kK]: slot of k-step
constexpr size_t kSmS = kSmKgrp + (size_t)(kRound / kK) * 4;                // fp16 [kSlots][kTile]
constexpr size_t kSmZ = kSmS + (size_t)kSlots * kTile * 2;                  // fp16 [kSlots][kTile]
constexpr size_t kSmC = kSmZ + (size_t)kSlots * kTile * 2;                  // i32 [kSlots]: column scales
constexpr size_t kSmX = kSmC + kSlots * 4;                                  // f32 [kSlots][kNB]: X_{g,t}
constexpr size_t kSmPhi = kSmX + kSlots * kNB * 4;                          // f32 [kSlots][kNB]: Phi_{g,t}
constexpr size_t kSmBase = kSmPhi + kSlots * kNB * 4;                       // i32 [kSlots + 1]: padded bases
constexpr size_t kSmChunkCnt = (kSmBase + (kSlots + 1) * 4 + 15) & ~size_t(15);  // i32 [kSlots][4][4]
constexpr size_t kSmWarpSum = kSmChunkCnt + kSlots * 4 * 4 * 4;             // f32 [kMmaWarps][2 kNB + 4]
constexpr size_t kSmWarpBal = kSmWarpSum + (size_t)kMmaWarps * (2 * kNB + 4) * 4;  // u32 [kMmaWarps][4][4]
constexpr size_t kSmWarpOff = kSmWarpBal + kMmaWarps * kChunks * 16;        // i32 [kMmaWarps][4][4]
constexpr size_t kSmXr = kSmWarpOff + kMmaWarps * kChunks * 16;             // u32 [kMmaWarps][4][kNB/2][32]:
                                                                            // the lanes' token values
constexpr size_t kSmBar = kSmXr + (size_t)kMmaWarps * kChunks * (kNB / 2) * 32 * 4;  // u64: full, empty, sz
constexpr size_t kSmMisc = kSmBar + (2 * kRing + 1) * 8;                    // i32 [4]
constexpr size_t kSmBytes = kSmMisc + 16;
static_assert(kSmBytes <= 227 * 1024, "shared memory");
static_assert((size_t)kNB * kTile * 4 <= (size_t)kRing * kStageBytes, "the CTA's partial fits the ring");
static_assert(kSmUx % 16 == 0 && kSmBfrag % 16 == 0 && kSmS % 16 == 0 && kSmZ % 16 == 0 &&
                  kSmChunkCnt % 16 == 0 && kSmWarpSum % 16 == 0 && kSmWarpBal % 16 == 0 &&
                  kSmWarpOff % 16 == 0 && kSmBar % 8 == 0,
              "aligned regions");
static_assert((kStage * 16) % kCopyThreads == 0 && kMmaWarps == kBlocks && kMmaWarps == kSlots, "layout");

struct BatchArgs {
  const uint32_t *planes;
  const uint16_t *s;
  const uint16_t *z;
  const uint16_t *x;   // [B][d_in]
  const float *theta;
  const float *phi;    // may be null: the default table
  int B, d_in, d_out, b_max, P, W, G, tiles, m;
  float *y;            // [B][d_out]
  uint8_t *u;          // optional [d_in]: union widths (null: not written)
  unsigned long long *counters;
  float *partials;     // [CTAs][kNB][kTile]
  int *error;
};

template <bool ALIGNED>
__global__ void __launch_bounds__(kThreads, 1) batch_kernel(const __grid_constant__ BatchArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  uint32_t *ring = reinterpret_cast<uint32_t *>(smem + kSmRing);
  int32_t *s_region = reinterpret_cast<int32_t *>(smem + kSmRegion);
  uint4 *s_ux = reinterpret_cast<uint4 *>(smem + kSmUx);
  uint2 *s_bfrag = reinterpret_cast<uint2 *>(smem + kSmBfrag);
  int *s_kgrp = reinterpret_cast<int *>(smem + kSmKgrp);
  uint16_t *s_st = reinterpret_cast<uint16_t *>(smem + kSmS);
  uint16_t *z_st = reinterpret_cast<uint16_t *>(smem + kSmZ);
  int *s_c = reinterpret_cast<int *>(smem + kSmC);
  float *s_X = reinterpret_cast<float *>(smem + kSmX);
  float *s_Phi = reinterpret_cast<float *>(smem + kSmPhi);
  int *s_base = reinterpret_cast<int *>(smem + kSmBase);
  int *s_ccnt = reinterpret_cast<int *>(smem + kSmChunkCnt);
  float *s_wsum = reinterpret_cast<float *>(smem + kSmWarpSum);
  uint4 *s_wbal = reinterpret_cast<uint4 *>(smem + kSmWarpBal);
  int4 *s_woff = reinterpret_cast<int4 *>(smem + kSmWarpOff);
  uint32_t *s_xr = reinterpret_cast<uint32_t *>(smem + kSmXr);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kSmBar);
  uint64_t *empty = full + kRing;
  uint64_t *sz_bar = empty + kRing;
  int *s_misc = reinterpret_cast<int *>(smem + kSmMisc);
  float *s_part = reinterpret_cast<float *>(smem + kSmRing);  // [kNB][kTile] after the loop

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool mma = warp < kMmaWarps;
  const int fg = lane >> 2, tq = lane & 3;
  const int ob = warp;  // the MMA warp's 128-output block
  const int C = (int)gridDim.x, c = (int)blockIdx.x;
  const int P = a.P, B = a.B;

  const bool many = a.tiles >= C;
  const int m = many ? 1 : a.m;
  const int C_eff = many ? C : a.tiles * m;
  const int R8 = a.d_in / 8;
  const int part = many ? 0 : c % m;
  const int q_lo = R8 * part / m, q_hi = R8 * (part + 1) / m;
  const int row_lo = 8 * q_lo, row_hi = 8 * q_hi;
  const int tile_first = many ? c : c / m, tile_step = many ? C : a.tiles;
  const int g_first = row_lo / kGroup;
  auto window_groups = [&](int g_w) { return min(kSlots, (row_hi + kGroup - 1) / kGroup - g_w); };

  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&full[i], kCopyThreads);
      mbar_init(&empty[i], kMmaWarps);
    }
    mbar_init(sz_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
  }
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
  __half2 t2[4];
  sort_thresholds(th_raw, t2);
  if (c >= C_eff) return;
  __syncthreads();

  uint64_t policy = 0;
  if (!mma) asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(policy));
  uint32_t gstage = 0, sz_phase = 0;
  bool ok = true;

  for (int tile = tile_first; tile < a.tiles; tile += tile_step) {
    const int wbase = tile * kTileW;
    const int seg_words = min(kTileW, a.W - wbase);
    float yacc[2][16];  // tokens 2 tq + jj, outputs 128 ob + 16 fg + t
#pragma unroll
    for (int t = 0; t < 16; ++t) yacc[0][t] = yacc[1][t] = 0.0f;

    for (int g_w = g_first; g_w * kGroup < row_hi; g_w += kSlots) {
      const int ng = window_groups(g_w);
      if (g_w != g_first || tile != tile_first) __syncthreads();

      const int slot = warp;  // an MMA warp takes one group of the window, 4 chunks of 32 rows
      const bool live = mma && slot < ng;
      const int row0 = (g_w + slot) * kGroup + lane;  // the lane's row in chunk 0
      // the lane's rows' token pairs (fp16 bits), kept in shared memory for the records
      auto xr_at = [&](int ci, int k) -> uint32_t & { return s_xr[((warp * kChunks + ci) * (kNB / 2) + k) * 32 + lane]; };
      uint32_t bal[kChunks][4];
#pragma unroll
      for (int ci = 0; ci < kChunks; ++ci) bal[ci][0] = bal[ci][1] = bal[ci][2] = bal[ci][3] = 0u;
      if (warp == kMmaWarps) {
        if (sz_phase > 0) ok &= mbar_wait(sz_bar, (sz_phase - 1) & 1u, a.error);
        if (lane == 0) mbar_arrive_expect_tx(sz_bar, (uint32_t)(2 * ng * seg_words * 32));
        __syncwarp();
        if (lane < 2 * ng) {
          const int which = lane & 1, gi = lane >> 1;
          const uint16_t *src = (which ? a.z : a.s) + (size_t)(g_w + gi) * a.d_out + tile * kTile;
          bulk_g2s((which ? z_st : s_st) + gi * kTile, src, (uint32_t)seg_words * 32, sz_bar, policy);
        }
      } else if (mma) {
        // ---- compaction on the union width: plane p of a row is read when some
        // token has b > 2p, i.e. the largest |x_t| (NaN left out) >= the p-th
        // smallest threshold; per-token group sums over the tokens' own widths ----
        float X[kNB], Phi[kNB];
#pragma unroll
        for (int t = 0; t < kNB; ++t) X[t] = Phi[t] = 0.0f;
        uint32_t amax_all = 0u;
        if (live) {
#pragma unroll
          for (int ci = 0; ci < kChunks; ++ci) {
            const int row = row0 + kChunkRows * ci;
            const bool in = row >= row_lo && row < row_hi;
            uint32_t amax = 0u, xp = 0u;
#pragma unroll
            for (int t = 0; t < kNB; ++t) {
              uint32_t xb = 0u;
              if (in && t < B) xb = __ldg(a.x + (size_t)t * a.d_in + row);
              xp |= xb << (16 * (t & 1));
              if (t & 1) {
                xr_at(ci, t >> 1) = xp;
                xp = 0u;
              }
              const uint32_t ab = xb & 0x7fffu;
              if (ab <= 0x7c00u) amax = max(amax, ab);  // NaN has width 0
              const __half ax = __ushort_as_half((uint16_t)ab);
              int lev = 0;
#pragma unroll
              for (int p = 0; p < 4; ++p) lev += __hge(ax, __low2half(t2[p])) ? 1 : 0;
              if (lev > 0) {
                const float xv = __half2float(__ushort_as_half((uint16_t)xb));
                X[t] += xv;
                Phi[t] = __fmaf_rn(xv, pick_phi(phi, lev), Phi[t]);
              }
            }
            const __half am = __ushort_as_half((uint16_t)amax);
            int ulev = 0;
#pragma unroll
            for (int p = 0; p < 4; ++p) {
              const bool act = in && __hge(am, __low2half(t2[p]));
              bal[ci][p] = __ballot_sync(0xffffffffu, act);
              ulev += act ? 1 : 0;
            }
            if (ulev > 0) amax_all = max(amax_all, amax);
            if (a.u && in && tile == 0) a.u[row] = (uint8_t)(2 * ulev);  // tile 0's CTAs cover every row
          }
#pragma unroll
          for (int t = 0; t < kNB; ++t)
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
              X[t] += __shfl_xor_sync(0xffffffffu, X[t], off);
              Phi[t] += __shfl_xor_sync(0xffffffffu, Phi[t], off);
            }
          amax_all = __reduce_max_sync(0xffffffffu, amax_all);
          if (lane == 0) {
            float *ws = s_wsum + warp * (2 * kNB + 4);
#pragma unroll
            for (int t = 0; t < kNB; ++t) {
              ws[t] = X[t];
              ws[kNB + t] = Phi[t];
            }
            ws[2 * kNB] = __uint_as_float(amax_all);
          }
        }
        // units per (slot, plane, chunk); lanes 0-15 write the warp's sixteen
#pragma unroll
        for (int ci = 0; ci < kChunks; ++ci)
#pragma unroll
          for (int p = 0; p < 4; ++p)
            if (lane == 4 * ci + p) s_ccnt[(4 * slot + p) * 4 + ci] = __popc(bal[ci][p]);
      }
      __syncthreads();

      // ---- unit offsets: ordered by slot, plane, chunk; each slot's units padded
      // to whole k-steps (lane L holds (slot, plane) = (L / 4, L mod 4)) ----
      int Nw = 0, cg = 0;
      if (mma) {
        const int4 cv = reinterpret_cast<const int4 *>(s_ccnt)[lane];
        const int t = cv.x + cv.y + cv.z + cv.w;
        int tot_slot = t;
        tot_slot += __shfl_xor_sync(0xffffffffu, tot_slot, 1);
        tot_slot += __shfl_xor_sync(0xffffffffu, tot_slot, 2);
        const int pad = ((tot_slot + kGrpPad - 1) & ~(kGrpPad - 1)) - tot_slot;
        const int tp = t + ((lane & 3) == 3 ? pad : 0);
        int inc = tp;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int u = __shfl_up_sync(0xffffffffu, inc, off);
          if (lane >= off) inc += u;
        }
        Nw = __shfl_sync(0xffffffffu, inc, 31);
        const int first = inc - tp;  // first unit of (slot, plane)
        // first units of the 4 chunks of the lane's (slot, plane); the warp keeps its slot's
        const int oc[kChunks] = {first, first + cv.x, first + cv.x + cv.y, first + cv.x + cv.y + cv.z};
#pragma unroll
        for (int ci = 0; ci < kChunks; ++ci) {
          int offv[4];
#pragma unroll
          for (int p = 0; p < 4; ++p) offv[p] = __shfl_sync(0xffffffffu, oc[ci], 4 * slot + p);
          if (live && lane == 0) {
            s_wbal[kChunks * warp + ci] = make_uint4(bal[ci][0], bal[ci][1], bal[ci][2], bal[ci][3]);
            s_woff[kChunks * warp + ci] = make_int4(offv[0], offv[1], offv[2], offv[3]);
          }
        }
        if (warp == 0 && (lane & 3) == 0) s_base[lane >> 2] = first;  // slot bases (p = 0)
        if (warp == 0 && lane == 0) {
          s_base[kSlots] = Nw;
          s_misc[0] = Nw;
        }
        if (live) {
          const float *w0 = s_wsum + slot * (2 * kNB + 4);
          const uint32_t am = __float_as_uint(w0[2 * kNB]);
          cg = (am >= 0x7c00u) ? 0 : max(0, (int)(am >> 10) - 15 + 2 * P - 16);
          if (lane < kNB) {
            s_X[slot * kNB + lane] = w0[lane];
            s_Phi[slot * kNB + lane] = w0[kNB + lane];
            if (lane == 0) s_c[slot] = cg;
          }
        }
      }

      // records of the MMA warp's units in [k0, k0 + n): plane region and the 8
      // token values x_t 4^(P-1-p) 2^-c (0 where the token's own width stops above
      // plane p); every entry of the round starts as padding (no load, B = 0)
      auto write_records = [&](int k0, int n, int n_pad) {
        for (int k = tid; k < n_pad; k += kMmaThreads) {
          s_region[k] = -1;
          s_ux[k] = make_uint4(0u, 0u, 0u, 0u);
        }
        sync_first<kMmaThreads>();
        if (live) {
          const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
          for (int ci = 0; ci < kChunks; ++ci) {
            const uint4 bv = s_wbal[kChunks * warp + ci];
            const int4 ov = s_woff[kChunks * warp + ci];
            const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
            const int ow[4] = {ov.x, ov.y, ov.z, ov.w};
            const int rp = (row0 + kChunkRows * ci) * P;
#pragma unroll
            for (int p = 0; p < 4; ++p) {
              const int u = ow[p] + __popc(bw[p] & lt);
              if (((bw[p] >> lane) & 1u) && u >= k0 && u < k0 + n) {
                const __half sc = __ushort_as_half((uint16_t)((15 + 2 * (P - 1 - p) - cg) << 10));
                uint32_t v[kNB / 2];
#pragma unroll
                for (int k = 0; k < kNB / 2; ++k) {
                  uint32_t pr = 0u;
#pragma unroll
                  for (int h = 0; h < 2; ++h) {
                    const uint16_t xb = (uint16_t)(xr_at(ci, k) >> (16 * h));
                    const __half ax = __ushort_as_half((uint16_t)(xb & 0x7fffu));
                    if (__hge(ax, __low2half(t2[p])))
                      pr |= (uint32_t)__half_as_ushort(__hmul(__ushort_as_half(xb), sc)) << (16 * h);
                  }
                  v[k] = pr;
                }
                s_region[u - k0] = rp + p;
                s_ux[u - k0] = make_uint4(v[0], v[1], v[2], v[3]);
              }
            }
          }
        }
      };
      auto round_size = [](int Nw_, int k0, int &n, int &n_pad) {
        n = min(kRound, Nw_ - k0);
        n_pad = (n + kStage - 1) & ~(kStage - 1);
      };
      if (mma && Nw > 0) {
        int n, n_pad;
        round_size(Nw, 0, n, n_pad);
        write_records(0, n, n_pad);
      }
      __syncthreads();
      Nw = s_misc[0];

      for (int k0 = 0; k0 < Nw; k0 += kRound) {
        int n, n_pad;
        round_size(Nw, k0, n, n_pad);
        const int n_steps = n_pad / kK, n_stages = n_pad / kStage;
        if (k0 > 0) {
          __syncthreads();
          if (mma) write_records(k0, n, n_pad);
          __syncthreads();
        }
        if (!mma) {
          // ---- copy warps: copy thread ct takes the 16-byte pieces ct + kCopyThreads j of
          // the stage (a warp's 32 lanes: two units' 256-byte segments) ----
          const int ct = tid - kMmaThreads;
          for (int st = 0; st < n_stages; ++st) {
            const uint32_t gs = gstage + st, rs = gs % kRing;
            if (gs >= kRing) ok &= mbar_wait(&empty[rs], ((gs / kRing) - 1u) & 1u, a.error);
            uint32_t *dst_stage = ring + (size_t)rs * (kStage * kRow);
#pragma unroll
            for (int j = 0; j < kStage * 16 / kCopyThreads; ++j) {
              const int q = ct + kCopyThreads * j, ul = q >> 4, part16 = q & 15;
              const int region = s_region[st * kStage + ul];
              const int word = 4 * part16;
              if (region >= 0 && word < seg_words) {
                const uint32_t *src = a.planes + (size_t)region * a.W + wbase + word;
                uint32_t *dst = dst_stage + ul * kRow + word;
                if (ALIGNED) {
                  cp_async16_hint(dst, src, policy);
                } else {
#pragma unroll
                  for (int v = 0; v < 4; ++v)
                    if (word + v < seg_words) cp_async4(dst + v, src + v);
                }
              }
            }
            cp_async_mbar_arrive(&full[rs]);  // counts once this thread's copies have landed
          }
        } else {
          // B fragments: lane (fg, tq) holds B[2tq, 2tq+1][fg] and B[2tq+8, 2tq+9][fg], column
          // fg = token fg; and the group (slot) of every k-step
          for (int q = tid; q < n_steps * 32; q += kMmaThreads) {
            const int kk = q >> 5, L = q & 31, col = L >> 2, t2i = 2 * (L & 3);
            const uint16_t *ux = reinterpret_cast<const uint16_t *>(s_ux + kk * kK);
            auto bh = [&](int u) -> uint32_t { return ux[u * kNB + col]; };
            s_bfrag[q] = make_uint2(bh(t2i) | (bh(t2i + 1) << 16), bh(t2i + 8) | (bh(t2i + 9) << 16));
            if (L == 0) {
              const int u = k0 + kk * kK;
              int gslot = kSlots;  // past the window's units: none
#pragma unroll
              for (int j = 0; j < kSlots; ++j)
                if (u >= s_base[j] && u < s_base[j + 1]) gslot = j;
              s_kgrp[kk] = gslot;
            }
          }
          sync_first<kMmaThreads>();
          ok &= mbar_wait(sz_bar, sz_phase & 1u, a.error);  // s of the window's groups

          float d[8][4];
#pragma unroll
          for (int bk = 0; bk < 8; ++bk) d[bk][0] = d[bk][1] = d[bk][2] = d[bk][3] = 0.0f;
          int cur = kSlots;  // the group the accumulators hold (none)
          // y_t += s (D 2^(24 - pos(t) + c)) for the lane's 16 outputs and 2 tokens
          auto flush = [&]() {
            if (cur < ng) {
              const __half2 *srow = reinterpret_cast<const __half2 *>(s_st + cur * kTile + 128 * ob + 16 * fg);
              const int ebase = (127 + 24 + s_c[cur]) << 23;  // 2^(24 + c) as float bits
#pragma unroll
              for (int bk = 0; bk < 8; ++bk) {
                // s 2^(24 - pos(t) + c): a power-of-two multiple of s, exact
                const float2 fs = __half22float2(srow[bk]);
                const float s0 = fs.x * __int_as_float(ebase - (field_pos(2 * bk) << 23));
                const float s1 = fs.y * __int_as_float(ebase - (field_pos(2 * bk + 1) << 23));
                yacc[0][2 * bk] = fmaf(s0, d[bk][0], yacc[0][2 * bk]);
                yacc[1][2 * bk] = fmaf(s0, d[bk][1], yacc[1][2 * bk]);
                yacc[0][2 * bk + 1] = fmaf(s1, d[bk][2], yacc[0][2 * bk + 1]);
                yacc[1][2 * bk + 1] = fmaf(s1, d[bk][3], yacc[1][2 * bk + 1]);
              }
            }
#pragma unroll
            for (int bk = 0; bk < 8; ++bk) d[bk][0] = d[bk][1] = d[bk][2] = d[bk][3] = 0.0f;
          };

          for (int st = 0; st < n_stages; ++st) {
            const uint32_t gs = gstage + st, rs = gs % kRing;
            ok &= mbar_wait(&full[rs], (gs / kRing) & 1u, a.error);
            // the stage's 4 k-steps; each half stage (2 k-steps) belongs to one group
            constexpr int kSteps = kStage / kK;
            const uint32_t *sb = ring + (size_t)rs * (kStage * kRow);
            uint32_t wv[kSteps][4];
            uint2 bv[kSteps];
#pragma unroll
            for (int h = 0; h < kSteps; ++h) {
              const int kk = kSteps * st + h;
              const uint32_t *pw = sb + (h * kK + 2 * tq) * kRow + 8 * ob + fg;
              wv[h][0] = pw[0];
              wv[h][1] = pw[kRow];
              wv[h][2] = pw[8 * kRow];
              wv[h][3] = pw[9 * kRow];
              bv[h] = s_bfrag[kk * 32 + lane];
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[rs]);  // the stage's words are in registers
#pragma unroll
            for (int h = 0; h < kSteps; ++h) {
              if (h % 2 == 0) {
                const int grp = s_kgrp[kSteps * st + h];
                if (grp != cur) {  // warp-uniform: the accumulators go to the outputs first
                  flush();
                  cur = grp;
                }
              }
              const uint32_t w0 = wv[h][0], w1 = wv[h][1], w2 = wv[h][2], w3 = wv[h][3];
              const uint2 bb = bv[h];
              const uint32_t m0 = prmt(w0, w1, 0x5410u), m1 = prmt(w0, w1, 0x7632u);
              const uint32_t m2 = prmt(w2, w3, 0x5410u), m3 = prmt(w2, w3, 0x7632u);
              const uint32_t n0 = m0 >> 6, n1 = m1 >> 6, n2 = m2 >> 6, n3 = m3 >> 6;
              constexpr uint32_t F = 0x00030003u;
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
          flush();
          // the window's group terms s Phi_{g,t} + z X_{g,t}, once (first round)
          if (k0 == 0) {
            for (int j = 0; j < ng; ++j) {
              const uint16_t *srow = s_st + j * kTile + 128 * ob + 16 * fg;
              const uint16_t *zrow = z_st + j * kTile + 128 * ob + 16 * fg;
              const float X0 = s_X[j * kNB + 2 * tq], X1 = s_X[j * kNB + 2 * tq + 1];
              const float F0 = s_Phi[j * kNB + 2 * tq], F1 = s_Phi[j * kNB + 2 * tq + 1];
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const uint4 sv = *reinterpret_cast<const uint4 *>(srow + 8 * h);
                const uint4 zv = *reinterpret_cast<const uint4 *>(zrow + 8 * h);
                const uint32_t su[4] = {sv.x, sv.y, sv.z, sv.w}, zu[4] = {zv.x, zv.y, zv.z, zv.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  const float2 fs = __half22float2(*reinterpret_cast<const __half2 *>(&su[k]));
                  const float2 fz = __half22float2(*reinterpret_cast<const __half2 *>(&zu[k]));
                  const int t0 = 8 * h + 2 * k, t1 = t0 + 1;
                  yacc[0][t0] = fmaf(fz.x, X0, fmaf(fs.x, F0, yacc[0][t0]));
                  yacc[1][t0] = fmaf(fz.x, X1, fmaf(fs.x, F1, yacc[1][t0]));
                  yacc[0][t1] = fmaf(fz.y, X0, fmaf(fs.y, F0, yacc[0][t1]));
                  yacc[1][t1] = fmaf(fz.y, X1, fmaf(fs.y, F1, yacc[1][t1]));
                }
              }
            }
          }
        }
        gstage += (uint32_t)n_stages;
      }
      ++sz_phase;
    }

    // ---- the CTA's partial tile [kNB][kTile] in the idle ring ----
    const int obase = tile * kTile;
    __syncthreads();
    if (mma) {
#pragma unroll
      for (int jj = 0; jj < 2; ++jj)
#pragma unroll
        for (int t = 0; t < 16; t += 4)
          *reinterpret_cast<float4 *>(s_part + (2 * tq + jj) * kTile + 128 * ob + 16 * fg + t) =
              make_float4(yacc[jj][t], yacc[jj][t + 1], yacc[jj][t + 2], yacc[jj][t + 3]);
    }
    __syncthreads();

    // ---- split-K (as in decode.cu): publish, count the arrival; the last arrival sums
    // the m partials of every token in CTA order, staging them in shared memory ----
    if (m == 1) {
      for (int q = tid; q < B * (kTile / 4); q += kThreads) {
        const int t = q / (kTile / 4), o4 = q % (kTile / 4);
        const float4 v = reinterpret_cast<const float4 *>(s_part + t * kTile)[o4];
        const int o = obase + 4 * o4;
        if (o < a.d_out) {
          float *yo = a.y + (size_t)t * a.d_out + o;
          yo[0] = v.x;
          yo[1] = v.y;
          yo[2] = v.z;
          yo[3] = v.w;
        }
      }
      continue;
    }
    const int c_first = (c / m) * m;
    for (int q = tid; q < B * (kTile / 4); q += kThreads) {
      const int t = q / (kTile / 4), o4 = q % (kTile / 4);
      reinterpret_cast<float4 *>(a.partials + ((size_t)c * kNB + t) * kTile)[o4] =
          reinterpret_cast<const float4 *>(s_part + t * kTile)[o4];
    }
    __syncthreads();
    if (tid == 0) {
      unsigned long long *word = a.counters + tile;
      const bool masked = m <= 32;
      const unsigned fullm = !masked ? 0u : m == 32 ? 0xffffffffu : (1u << m) - 1u;
      const unsigned long long add = (1ull << 32) | (masked ? 1ull << part : 0ull);
      asm volatile("fence.acq_rel.gpu;\n" ::: "memory");
      const unsigned long long old = atomicAdd(word, add);
      const bool last = (unsigned)(old >> 32) == (unsigned)(m - 1);
      if (last) {
        if (masked && (((unsigned)old | (unsigned)add) & fullm) != fullm) {
          int polls = 0;
          while ((unsigned)(ld_acquire64(word) & fullm) != fullm && ++polls < kPolls) __nanosleep(64);
          atomicCAS(a.error, 0, kDevErrSplitKTimeout);
        }
        asm volatile("fence.acq_rel.gpu;\n" ::: "memory");
        *reinterpret_cast<volatile unsigned long long *>(word) = 0ull;
      }
      s_misc[1] = last ? 1 : 0;
    }
    __syncthreads();
    if (s_misc[1]) {
      float4 *stage = reinterpret_cast<float4 *>(smem);  // [kFixParts][kTile / 4], the idle ring
      for (int t = 0; t < B; ++t) {
        float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        for (int k0 = 0; k0 < m; k0 += kFixParts) {
          const int np = min(kFixParts, m - k0);
          for (int q = tid; q < np * (kTile / 4); q += kThreads) {
            const int k = q / (kTile / 4), o4 = q % (kTile / 4);
            cp_async16(stage + q, a.partials + ((size_t)(c_first + k0 + k) * kNB + t) * kTile + 4 * o4, 16);
          }
          cp_async_commit();
          cp_async_wait<0>();
          __syncthreads();
          if (tid < kTile / 4)
            for (int k = 0; k < np; ++k) acc = f4add(acc, stage[k * (kTile / 4) + tid]);
          __syncthreads();
        }
        const int o = obase + 4 * tid;
        if (tid < kTile / 4 && o < a.d_out) {
          float *yo = a.y + (size_t)t * a.d_out + o;
          yo[0] = acc.x;
          yo[1] = acc.y;
          yo[2] = acc.z;
          yo[3] = acc.w;
        }
      }
    }
  }
  if (warp == kMmaWarps && sz_phase > 0) ok &= mbar_wait(sz_bar, (sz_phase - 1) & 1u, a.error);
  (void)ok;
}

int device_sms() {
  int dev = 0, n = kNumSMs;
  if (cudaGetDevice(&dev) != cudaSuccess) return kNumSMs;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n = kNumSMs;
  return n > kMaxCtas ? kMaxCtas : n;
}

template <bool ALIGNED>
cudaError_t launch(const BatchArgs &a, int C, cudaStream_t st) {
  cudaError_t e = ensure_smem_attr((const void *)batch_kernel<ALIGNED>, kSmBytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, batch_kernel<ALIGNED>, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

size_t batch_ws_bytes() { return kWsBytes; }

cudaError_t launch_decode_batch(const uint32_t *planes, const uint16_t *s, const uint16_t *z,
                                const uint16_t *x, const float *theta, const float *phi, int B,
                                int d_in, int d_out, int b_max, float *y, uint8_t *u, void *ws,
                                cudaStream_t st) {
  char *w = static_cast<char *>(ws);
  BatchArgs a = {};
  a.planes = planes;
  a.s = s;
  a.z = z;
  a.x = x;
  a.theta = theta;
  a.phi = phi;
  a.B = B;
  a.d_in = d_in;
  a.d_out = d_out;
  a.b_max = b_max;
  a.P = b_max / 2;
  a.W = d_out / 16;
  a.G = d_in / kGroup;
  a.tiles = (d_out + kTile - 1) / kTile;
  a.y = y;
  a.u = u;
  a.counters = reinterpret_cast<unsigned long long *>(w + kWsCounters);
  a.partials = reinterpret_cast<float *>(w + kWsPartials);
  a.error = &reinterpret_cast<WsHeader *>(w)->error;
  const bool aligned = a.W % 4 == 0;
  const int C = device_sms();
  a.m = a.tiles >= C ? 1 : C / a.tiles;
  return aligned ? launch<true>(a, C, st) : launch<false>(a, C, st);
}

}  // namespace grinqh
