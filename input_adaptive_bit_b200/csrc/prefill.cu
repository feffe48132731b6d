// prefill.cu -- the prefill GEMM of GRINQH: every row at the full width b_max,
// Y[t][o] = sum_i X[t][i] w_hat(i, o),  w_hat = s_{g,o} (q_{i,o} + phi_P) + z_{g,o},
// for a block of T tokens (the pages' other phase: "GRINQH: Graded Input-Based
// Quantization Hierarchy", Method / overall framework, where prefill runs the
// base b_max-bit weights densely and pays for unpacking the planes).
//
// How (B200 design):
//  * Work unit = (token block of up to 128, tile of 128 outputs, chunk of 128
//    rows = one s/z group).  The units are ordered by token block, tile, chunk
//    and cut into one contiguous range per CTA (one CTA per SM), so every SM
//    gets the same number of chunks whatever the shape; a range meets at most
//    a few tiles, and each (range, tile) piece adds its partial sums into Y,
//    which the launcher clears first.
//  * Warp roles, connected by full/empty mbarrier rings (no block-wide barrier
//    inside the loop): warps 16-19 copy the plane words and s, z of a chunk
//    into one of 4 slots with cp.async (lanes 2j and 2j+1 take the two halves
//    of one 32-byte row segment, so every sector is one request), warps 20-23
//    the X rows into one of 3 slots, each arriving on the slot's "full" barrier
//    when its copies land; warps 0-15 rebuild the chunk's A tile into one of 2
//    buffers and arrive on "A full"; warp 24 issues the MMAs and commits them
//    to "A empty", "X slot empty" and, after the last chunk of a piece,
//    "accumulator full", on which warps 0-15 run the piece's epilogue and then
//    free the accumulator.  A waiting thread sleeps in mbarrier.try_wait until
//    the phase completes.
//  * Rebuild, about 2 logic ops and 1 fp16 op per weight: each thread takes 2
//    rows of one 16-output plane word.  Per row it rotates plane p's word left
//    by 2 (P-1-p), so that output j's digit of plane p sits at bit
//    2 j + 2 (P-1-p); for each residue r = j mod 4 one masked merge of the P
//    rotated words, rotated back by 2 r, leaves the codes of outputs r, r+4,
//    r+8, r+12 as the four bytes of one register.  Byte permutes pair the
//    codes of outputs (2c, 2c+1) under the fp16 exponent of 1024, so each half
//    is exactly 1024 + q; one fp16 subtract (exact) and one fp16 FMA give
//    w_hat = RN16(s q + z), the correctly rounded fp16 of the exact value
//    (phi_P = 0, the default).  With an explicit phi_P != 0 the FMA runs in
//    fp32, fmaf(s, q + phi_P, z), rounded once to fp16.
//  * The A tile is stored MN-major (8 consecutive outputs per 16-byte row of a
//    core matrix), so a thread writes whole 16-byte rows; a warp's lanes cover
//    the 8 rows of a core matrix and the stores are free of bank conflicts.  The
//    plane-word slots are swizzled by row (16-byte chunk index XOR row mod 8)
//    for conflict-free loads of a word's P planes.
//  * The contraction runs on the 5th-generation tensor cores: tcgen05.mma
//    kind::f16, M = 128 (outputs, A MN-major) x N = tokens (B = X, K-major) x
//    K = 16, fp32 accumulators in tensor memory.  The epilogue reads D back with
//    tcgen05.ld (one output per lane, one token per column) and adds it into Y.
#include <cuda_fp16.h>

#include "grinqh_internal.cuh"

namespace grinqh {
namespace {

constexpr int kBuildWarps = 16;  // warps 0-15: rebuild and epilogue
constexpr int kPlaneWarp0 = 16;  // warps 16-19: plane words and s, z
constexpr int kXWarp0 = 20;      // warps 20-23: X rows
constexpr int kMmaWarp = 24;     // warp 24: tensor memory and MMAs
constexpr int kPThreads = 32 * (kMmaWarp + 1);
constexpr int kBuilders = 32 * kBuildWarps, kCopiers = 128;
constexpr int kPM = 128;  // outputs per tile (MMA M)
constexpr int kPN = 128;  // tokens per block (MMA N, padded to a multiple of 16)
constexpr int kPK = 128;  // rows per chunk (one s/z group)
constexpr int kRowsPerBuilder = kPK * kPM / 16 / (32 * kBuildWarps);  // rows of one plane word per thread
static_assert(kRowsPerBuilder * 32 * kBuildWarps * 16 == kPK * kPM, "every (row, word) once");
constexpr int kSP = 4;    // plane-word (and s, z) slots
constexpr int kSX = 3;    // X slots
constexpr uint32_t kWaitHintNs = 1000000;  // suspend-time hint of one try_wait (1 ms)
constexpr int kPSpinLimit = 1000;           // tries of one wait (~1 s); after a timeout a thread stops waiting

// shared memory map (bytes)
constexpr size_t kABuf = (size_t)kPM * kPK * 2;       // A tile, fp16, MN-major
constexpr size_t kXSlot = (size_t)kPN * kPK * 2;      // B tile (X), fp16, K-major
constexpr size_t kPlaneSlot = (size_t)kPK * 128;      // [row][8 x 16-byte chunks], 4 planes x 8 words
constexpr size_t kSzSlot = (size_t)2 * kPM * 2;       // s and z of the group
constexpr size_t kOffA = 0;
constexpr size_t kOffX = kOffA + 2 * kABuf;
constexpr size_t kOffPlanes = kOffX + kSX * kXSlot;
constexpr size_t kOffSz = kOffPlanes + kSP * kPlaneSlot;
constexpr size_t kPSmem = kOffSz + kSP * kSzSlot;
static_assert(kPSmem <= 227 * 1024 - 64, "shared memory");

struct PrefillArgs {
  const uint32_t *planes;
  const uint16_t *s, *z, *x;  // x: [T][d_in]
  const float *phi;            // may be null: phi_P = 0
  int T, d_in, d_out, W;
  int tiles, tblocks, G;
  float *y;                    // [T][d_out], cleared by the launcher
  int *error;
};

__device__ __forceinline__ unsigned smem_u32(const void *p) {
  return (unsigned)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void cp_async16(void *dst, const void *src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes));
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count));
}
// Waits for the phase of the given parity.  Each try_wait may suspend the thread
// for up to kWaitHintNs and returns as soon as the phase completes, so a waiting
// warp does not take issue slots from the others; at most kPSpinLimit tries.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, unsigned parity) {
  const unsigned a = smem_u32(bar);
  for (int i = 0; i < kPSpinLimit; ++i) {
    unsigned done;
    asm volatile(
        "{.reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;}\n"
        : "=r"(done)
        : "r"(a), "r"(parity), "r"(kWaitHintNs)
        : "memory");
    if (done) return true;
  }
  return false;
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}
// arrives (counting toward the expected count) once this thread's earlier cp.async copies land
__device__ __forceinline__ void cp_async_arrive(uint64_t *bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}
// K-major operand tile without swizzle: 8-row x 16-byte core matrices, the two
// K-adjacent ones 128 bytes apart (leading), 8-row groups 256 bytes apart (stride).
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3fffu) | ((uint64_t)(128 >> 4) << 16) | ((uint64_t)(256 >> 4) << 32) |
         ((uint64_t)1 << 46);
}
// MN-major operand tile without swizzle: a core matrix is 8 K rows of 16 bytes
// (8 consecutive M elements each); M-adjacent core matrices 128 bytes apart
// (stride), the two K-adjacent ones of a 16-deep slice 2048 bytes apart (leading).
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3fffu) | ((uint64_t)(2048 >> 4) << 16) | ((uint64_t)(128 >> 4) << 32) |
         ((uint64_t)1 << 46);
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
__host__ __device__ constexpr uint32_t rotl_c(uint32_t x, int s) {
  return (s & 31) ? (x << (s & 31)) | (x >> (32 - (s & 31))) : x;
}
__device__ __forceinline__ uint32_t h2_sub_fma(uint32_t h, uint32_t s2, uint32_t c2) {
  // (h - 1024) exactly, then s q + c rounded once to fp16
  const __half2 q = __hsub2(*reinterpret_cast<const __half2 *>(&h), __half2half2(__ushort_as_half(0x6400)));
  const __half2 w = __hfma2(q, *reinterpret_cast<const __half2 *>(&s2), *reinterpret_cast<const __half2 *>(&c2));
  return *reinterpret_cast<const uint32_t *>(&w);
}

// The same with an explicit phi_P != 0: fmaf(s, q + phi_P, z) in fp32, rounded
// once to fp16.  (Folding phi_P into an fp16 offset z + s phi_P would round it,
// and that one error would land on every weight of the group: where s q + z
// nearly cancels it exceeds the per-weight 2^-11.)
__device__ __forceinline__ uint32_t h2_sub_fma_phi(uint32_t h, uint32_t s2, uint32_t z2, float phi) {
  const __half2 q = __hsub2(*reinterpret_cast<const __half2 *>(&h), __half2half2(__ushort_as_half(0x6400)));
  const float2 qf = __half22float2(q);
  const float2 sf = __half22float2(*reinterpret_cast<const __half2 *>(&s2));
  const float2 zf = __half22float2(*reinterpret_cast<const __half2 *>(&z2));
  const __half2 w = __floats2half2_rn(fmaf(sf.x, qf.x + phi, zf.x), fmaf(sf.y, qf.y + phi, zf.y));
  return *reinterpret_cast<const uint32_t *>(&w);
}

// Codes (2P bits) of outputs r, r + 4, r + 8, r + 12 of a 16-output plane word
// group, one per byte, from the P words rotated as described above.
template <int P>
__device__ __forceinline__ uint32_t merge_residue(const uint32_t (&wr)[4], int r) {
  uint32_t c = 0;
#pragma unroll
  for (int p = 0; p < P; ++p) c |= wr[p] & rotl_c(0x03030303u, 2 * r + 2 * (P - 1 - p));
  return __funnelshift_r(c, c, 2 * r);
}

// one piece of a CTA's unit range: consecutive chunks of one (token block, tile)
struct Piece {
  int g0, n, m0, t0, nt, n_pad;
};
__device__ __forceinline__ Piece piece_at(const PrefillArgs &a, long long u, long long u_hi) {
  Piece pc;
  const long long tt = u / a.G;  // (token block, tile)
  pc.g0 = (int)(u - tt * a.G);
  const long long left = u_hi - u, rest = (long long)(a.G - pc.g0);
  pc.n = (int)(left < rest ? left : rest);
  const int tb = (int)(tt / a.tiles), tile = (int)(tt - (long long)tb * a.tiles);
  pc.m0 = tile * kPM;
  pc.t0 = tb * kPN;
  pc.nt = min(kPN, a.T - pc.t0);
  pc.n_pad = (pc.nt + 15) & ~15;
  return pc;
}

template <int P>
__global__ void __launch_bounds__(kPThreads, 1) prefill_kernel(const __grid_constant__ PrefillArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ uint32_t s_tmem;
  __shared__ __align__(8) uint64_t s_full_p[kSP], s_empty_p[kSP], s_full_x[kSX], s_empty_x[kSX];
  __shared__ __align__(8) uint64_t s_a_full[2], s_a_empty[2], s_acc_full, s_acc_empty, s_drain;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(&s_tmem)),
                 "r"(kPN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  if (tid == 0) {
    for (int i = 0; i < kSP; ++i) {
      mbar_init(&s_full_p[i], kCopiers);
      mbar_init(&s_empty_p[i], kBuilders);
    }
    for (int i = 0; i < kSX; ++i) {
      mbar_init(&s_full_x[i], kCopiers);
      mbar_init(&s_empty_x[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_a_full[i], kBuilders);
      mbar_init(&s_a_empty[i], 1);
    }
    mbar_init(&s_acc_full, 1);
    mbar_init(&s_acc_empty, kBuilders);
    mbar_init(&s_drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  bool ok = true;
  auto wait = [&](uint64_t *bar, uint32_t parity) {
    if (ok) ok = mbar_wait(bar, parity & 1u);
  };

  const long long U = (long long)a.tblocks * a.tiles * a.G;
  const long long u_lo = U * blockIdx.x / gridDim.x, u_hi = U * (blockIdx.x + 1) / gridDim.x;

  if (warp < kBuildWarps) {
    // ---- rebuild: rows 8 (R rg + ii) + rk, ii < R, of plane word wc; then the epilogue
    const int rk = tid & 7, wc = (tid >> 3) & 7, rg = tid >> 6;
    const float phiP = a.phi ? a.phi[P] : 0.0f;
    const uint32_t K64 = 0x64646464u;
    uint32_t ci = 0, piece = 0;
    for (long long u = u_lo; u < u_hi; ++piece) {
      const Piece pc = piece_at(a, u, u_hi);
      for (int i = 0; i < pc.n; ++i, ++ci) {
        const int sp = (int)(ci % kSP);
        wait(&s_full_p[sp], ci / kSP);
        if (ci >= 2) wait(&s_a_empty[ci & 1], (ci >> 1) - 1);
        const unsigned char *slot = smem + kOffPlanes + (size_t)sp * kPlaneSlot;
        const uint16_t *sz = reinterpret_cast<const uint16_t *>(smem + kOffSz + (size_t)sp * kSzSlot);
        unsigned char *abuf = smem + kOffA + (size_t)(ci & 1) * kABuf;
        uint32_t s2[8], z2[8];  // half2 s and z of outputs (2e, 2e + 1)
        {
          const uint4 sa = *reinterpret_cast<const uint4 *>(sz + 16 * wc);
          const uint4 sb = *reinterpret_cast<const uint4 *>(sz + 16 * wc + 8);
          const uint4 za = *reinterpret_cast<const uint4 *>(sz + kPM + 16 * wc);
          const uint4 zb = *reinterpret_cast<const uint4 *>(sz + kPM + 16 * wc + 8);
          const uint32_t sv[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
          const uint32_t zv[8] = {za.x, za.y, za.z, za.w, zb.x, zb.y, zb.z, zb.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            s2[e] = sv[e];
            z2[e] = zv[e];
          }
        }
#pragma unroll
        for (int ii = 0; ii < kRowsPerBuilder; ++ii) {
          const int k = 8 * (kRowsPerBuilder * rg + ii) + rk;
          const unsigned char *row = slot + k * 128 + (wc & 3) * 4;
          uint32_t wr[4];
#pragma unroll
          for (int p = 0; p < P; ++p) {
            const uint32_t w = *reinterpret_cast<const uint32_t *>(row + (((2 * p + (wc >> 2)) ^ rk) << 4));
            wr[p] = __funnelshift_l(w, w, 2 * (P - 1 - p));
          }
          const uint32_t c0 = merge_residue<P>(wr, 0), c1 = merge_residue<P>(wr, 1);
          const uint32_t c2r = merge_residue<P>(wr, 2), c3 = merge_residue<P>(wr, 3);
          // bytes: u01a = codes of outputs 0 1 4 5, u01b = 8 9 12 13, u23a = 2 3 6 7, u23b = 10 11 14 15
          const uint32_t u01a = prmt(c0, c1, 0x5140u), u01b = prmt(c0, c1, 0x7362u);
          const uint32_t u23a = prmt(c2r, c3, 0x5140u), u23b = prmt(c2r, c3, 0x7362u);
          uint32_t h[8];  // half2 of outputs (2e, 2e + 1)
          h[0] = prmt(u01a, K64, 0x4140u);
          h[2] = prmt(u01a, K64, 0x4342u);
          h[4] = prmt(u01b, K64, 0x4140u);
          h[6] = prmt(u01b, K64, 0x4342u);
          h[1] = prmt(u23a, K64, 0x4140u);
          h[3] = prmt(u23a, K64, 0x4342u);
          h[5] = prmt(u23b, K64, 0x4140u);
          h[7] = prmt(u23b, K64, 0x4342u);
          if (phiP == 0.0f) {
#pragma unroll
            for (int e = 0; e < 8; ++e) h[e] = h2_sub_fma(h[e], s2[e], z2[e]);
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) h[e] = h2_sub_fma_phi(h[e], s2[e], z2[e], phiP);
          }
          unsigned char *dst = abuf + (k & 7) * 16 + (k >> 3) * 2048 + (2 * wc) * 128;
          *reinterpret_cast<uint4 *>(dst) = make_uint4(h[0], h[1], h[2], h[3]);
          *reinterpret_cast<uint4 *>(dst + 128) = make_uint4(h[4], h[5], h[6], h[7]);
        }
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");  // A for the tensor cores
        mbar_arrive(&s_empty_p[sp]);
        mbar_arrive(&s_a_full[ci & 1]);
      }
      // epilogue: lane = output, column = token; warps w, w + 4, w + 8, w + 12
      // read lanes 32 (w mod 4) .. and split the columns
      wait(&s_acc_full, piece);
      tc_fence_after();
      const int quad = warp & 3, part = warp >> 2, o = pc.m0 + 32 * quad + lane;
      for (int c0 = 8 * part; c0 < pc.n_pad; c0 += 8 * (kBuildWarps / 4)) {
        uint32_t v[8];
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n"
                     : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
                       "=r"(v[7])
                     : "r"(tmem + ((uint32_t)(32 * quad) << 16) + (uint32_t)c0)
                     : "memory");
        asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (c0 + j < pc.nt) atomicAdd(a.y + (size_t)(pc.t0 + c0 + j) * a.d_out + o, __uint_as_float(v[j]));
      }
      tc_fence_before();
      mbar_arrive(&s_acc_empty);
      u += pc.n;
    }
  } else if (warp < kXWarp0) {
    // ---- plane words (thread = half hw of the 32-byte segments of rows r0 and
    // r0 + 64) and s, z
    const int pt = tid - 32 * kPlaneWarp0, hw = pt & 1, r0 = pt >> 1;
    uint32_t ci = 0;
    for (long long u = u_lo; u < u_hi;) {
      const Piece pc = piece_at(a, u, u_hi);
      for (int i = 0; i < pc.n && ok; ++i, ++ci) {
        const int sp = (int)(ci % kSP);
        if (ci >= kSP) wait(&s_empty_p[sp], ci / kSP - 1);
        if (!ok) break;  // a wait gave up: issue nothing more
        const int g = pc.g0 + i;
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const int r = r0 + 64 * rr;
          const uint32_t *src = a.planes + (size_t)(g * kPK + r) * P * a.W + pc.m0 / 16 + 4 * hw;
          unsigned char *dst = smem + kOffPlanes + (size_t)sp * kPlaneSlot + r * 128;
#pragma unroll
          for (int p = 0; p < P; ++p) cp_async16(dst + (((2 * p + hw) ^ (r & 7)) << 4), src + (size_t)p * a.W, 16);
        }
        if (pt < 32) {
          unsigned char *sz = smem + kOffSz + (size_t)sp * kSzSlot;
          const int which = pt >> 4, c = pt & 15;
          cp_async16(sz + which * kPM * 2 + 16 * c, (which ? a.z : a.s) + (size_t)g * a.d_out + pc.m0 + 8 * c,
                     16);
        }
        cp_async_arrive(&s_full_p[sp]);
      }
      u += pc.n;
    }
  } else if (warp < kMmaWarp) {
    // ---- X rows: thread = 8-row column c of the chunk, tokens tk0 + 8 j; the
    // K-major B tile puts (token t, rows 8c..8c+7) at (c / 2) n_pad 32 + (t / 8) 256
    // + (c mod 2) 128 + (t mod 8) 16
    const int xt = tid - 32 * kXWarp0, c = xt & 15, tk0 = xt >> 4;
    uint32_t ci = 0;
    for (long long u = u_lo; u < u_hi;) {
      const Piece pc = piece_at(a, u, u_hi);
      for (int i = 0; i < pc.n && ok; ++i, ++ci) {
        const int sx = (int)(ci % kSX);
        if (ci >= kSX) wait(&s_empty_x[sx], ci / kSX - 1);
        if (!ok) break;  // a wait gave up: issue nothing more
        const int k0 = (pc.g0 + i) * kPK;
        unsigned char *dst = smem + kOffX + (size_t)sx * kXSlot + (c >> 1) * pc.n_pad * 32 + (c & 1) * 128 + tk0 * 16;
        for (int j = 0; j < pc.n_pad / 8; ++j) {
          const int tk = tk0 + 8 * j;
          const bool in = tk < pc.nt;
          cp_async16(dst + j * 256, a.x + (size_t)(pc.t0 + (in ? tk : 0)) * a.d_in + k0 + 8 * c, in ? 16 : 0);
        }
        cp_async_arrive(&s_full_x[sx]);
      }
      u += pc.n;
    }
  } else if (lane == 0) {
    // ---- MMAs
    uint32_t ci = 0, piece = 0;
    for (long long u = u_lo; u < u_hi; ++piece) {
      const Piece pc = piece_at(a, u, u_hi);
      if (piece >= 1) {
        wait(&s_acc_empty, piece - 1);
        tc_fence_after();
      }
      const uint32_t idesc =
          (1u << 4) | (1u << 15) | ((uint32_t)(pc.n_pad >> 3) << 17) | ((uint32_t)(kPM >> 4) << 24);
      for (int i = 0; i < pc.n; ++i, ++ci) {
        const int sx = (int)(ci % kSX);
        wait(&s_a_full[ci & 1], ci >> 1);
        wait(&s_full_x[sx], ci / kSX);
        if (!ok) break;  // a wait gave up: issue no more MMAs
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + kOffA + (size_t)(ci & 1) * kABuf);
        const uint32_t b_addr = smem_u32(smem + kOffX + (size_t)sx * kXSlot);
#pragma unroll
        for (int h = 0; h < kPK / 16; ++h) {
          const uint64_t ad = mnmajor_desc(a_addr + h * 4096), bd = kmajor_desc(b_addr + h * pc.n_pad * 32);
          const uint32_t acc = (i == 0 && h == 0) ? 0u : 1u;
          asm volatile(
              "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
              "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem),
              "l"(ad), "l"(bd), "r"(idesc), "r"(acc)
              : "memory");
        }
        tc_commit(&s_a_empty[ci & 1]);
        tc_commit(&s_empty_x[sx]);
      }
      tc_commit(&s_acc_full);
      u += pc.n;
    }
  }

  // Before the tensor memory is freed and the CTA exits, nothing may still be in flight:
  // every thread's own cp.async copies have landed, and the MMA lane commits once
  // more and waits (bounded) for all of its MMAs -- on a correct run they are
  // complete already; after a wait that gave up this is what keeps an MMA from
  // writing tensor memory that has been freed.
  asm volatile("cp.async.wait_all;\n" ::: "memory");
  if (warp == kMmaWarp && lane == 0) {
    tc_commit(&s_drain);
    if (!mbar_wait(&s_drain, 0)) ok = false;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kPN) : "memory");
  }
  if (!ok) atomicCAS(a.error, 0, kDevErrPrefillTimeout);
}

template <int P>
cudaError_t launch_p(const PrefillArgs &a, int ctas, cudaStream_t st) {
  cudaError_t e = ensure_smem_attr((const void *)prefill_kernel<P>, kPSmem);
  if (e != cudaSuccess) return e;
  prefill_kernel<P><<<ctas, kPThreads, kPSmem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

size_t prefill_ws_bytes() { return sizeof(WsHeader); }

cudaError_t launch_prefill(const uint32_t *planes, const uint16_t *s, const uint16_t *z,
                           const uint16_t *x, const float *phi, int T, int d_in, int d_out,
                           int b_max, float *y, void *ws, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(y, 0, (size_t)T * d_out * sizeof(float), st);
  if (e != cudaSuccess) return e;
  PrefillArgs a = {};
  a.planes = planes;
  a.s = s;
  a.z = z;
  a.x = x;
  a.phi = phi;
  a.T = T;
  a.d_in = d_in;
  a.d_out = d_out;
  a.W = d_out / 16;
  a.tiles = d_out / kPM;
  a.tblocks = (T + kPN - 1) / kPN;
  a.G = d_in / kPK;
  a.y = y;
  a.error = &reinterpret_cast<WsHeader *>(ws)->error;
  int sms = kNumSMs;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long units = (long long)a.tblocks * a.tiles * a.G;
  const int ctas = (int)(units < sms ? units : sms);
  switch (b_max / 2) {
    case 1: return launch_p<1>(a, ctas, st);
    case 2: return launch_p<2>(a, ctas, st);
    case 3: return launch_p<3>(a, ctas, st);
    default: return launch_p<4>(a, ctas, st);
  }
}

}  // namespace grinqh
