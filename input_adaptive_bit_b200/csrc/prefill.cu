// prefill.cu -- the prefill GEMM of GRINQH: every row at the full width b_max,
// Y[t][o] = sum_i X[t][i] w_hat(i, o),  w_hat = s_{g,o} (q_{i,o} + phi_P) + z_{g,o},
// for a block of T tokens (the pages' other phase: "GRINQH: Graded Input-Based
// Quantization Hierarchy", Method / overall framework, where prefill runs the
// base b_max-bit weights densely and pays for unpacking the planes).
//
// How (B200 design):
//  * CTA tile = 128 outputs x up to 128 tokens x a 128-row-aligned slice of d_in
//    (split-K over the grid; the slices' partial sums are added into Y, which the
//    launcher clears first).
//  * Per stage of 128 rows (one s/z group): the plane words of the tile's 128
//    outputs, the token block's X rows and the group's s, z go to shared memory
//    with cp.async; every thread rebuilds 8 outputs x 8 rows of w_hat (all P
//    planes, fp32 arithmetic, rounded once to fp16: a relative error of at most
//    2^-11 per weight) into the A tile.
//  * The contraction runs on the 5th-generation tensor cores: tcgen05.mma
//    kind::f16, M = 128 (outputs) x N = tokens x K = 16, both operands K-major in
//    shared memory (8 x 16-byte core matrices, no swizzle), fp32 accumulators in
//    tensor memory.  One thread issues the 8 MMAs of a stage and commits them to
//    an mbarrier; the stage's buffers are rebuilt only after that barrier
//    completes (double buffering).  The epilogue reads D back with tcgen05.ld
//    (one output per lane, one token per column).
#include <type_traits>

#include "grinqh_internal.cuh"

namespace grinqh {
namespace {

constexpr int kPThreads = 256;
constexpr int kPM = 128;          // outputs per CTA tile (MMA M)
constexpr int kPN = 128;          // tokens per CTA tile (MMA N, padded to a multiple of 16)
constexpr int kPK = 128;          // rows per stage (one s/z group)
constexpr int kPSpinLimit = 1 << 22;

// shared memory of one stage (bytes)
constexpr size_t kPWords = (size_t)kPK * 4 * (kPM / 16) * 4;  // plane words [row][plane][8]
constexpr size_t kPA = (size_t)kPM * kPK * 2;                 // A tile, fp16, K-major
constexpr size_t kPB = (size_t)kPN * kPK * 2;                 // B tile, fp16, K-major
constexpr size_t kPSZ = (size_t)2 * kPM * 2;                  // s and z of the group
constexpr size_t kPStage = kPWords + kPA + kPB + kPSZ;
constexpr size_t kPSmem = 2 * kPStage;
static_assert(kPSmem <= 227 * 1024, "shared memory");
static_assert(kPWords % 128 == 0 && kPA % 128 == 0 && kPB % 128 == 0, "aligned regions");

struct PrefillArgs {
  const uint32_t *planes;
  const uint16_t *s, *z, *x;  // x: [T][d_in]
  const float *phi;            // may be null: phi_P = 0
  int T, d_in, d_out, b_max, P, W;
  int k_slices;                // CTAs along d_in per output tile
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
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
__device__ __forceinline__ void cp_async_wait0() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }
__device__ __forceinline__ void mbar_init(uint64_t *bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, unsigned parity) {
  const unsigned a = smem_u32(bar);
  for (int i = 0; i < kPSpinLimit; ++i) {
    unsigned done;
    asm volatile(
        "{.reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;}\n"
        : "=r"(done)
        : "r"(a), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
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
// byte offset of element (row, k) in a K-major tile of `rows` rows and kPK columns:
// k-steps of 16 are consecutive sub-tiles of rows x 32 bytes
__device__ __forceinline__ uint32_t kmajor_off(int row, int k, int rows) {
  return (uint32_t)((k >> 4) * rows * 32 + (row >> 3) * 256 + ((k >> 3) & 1) * 128 + (row & 7) * 16 +
                    (k & 7) * 2);
}

__global__ void __launch_bounds__(kPThreads, 1) prefill_kernel(const __grid_constant__ PrefillArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ uint32_t s_tmem;
  __shared__ __align__(8) uint64_t s_bar[2];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = blockIdx.x * kPM;                  // first output of the tile
  const int slice = blockIdx.y, t0 = blockIdx.z * kPN;  // d_in slice, first token
  const int nt = min(kPN, a.T - t0);                 // tokens of this block
  const int n_pad = (nt + 15) & ~15;                 // MMA N
  const int P = a.P;
  // this CTA's rows: groups [G slice / S, G (slice + 1) / S)
  const int G = a.d_in / kPK;
  const int g_lo = G * slice / a.k_slices, g_hi = G * (slice + 1) / a.k_slices;
  float phiP = a.phi ? a.phi[P] : 0.0f;

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(&s_tmem)),
                 "r"(kPN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  if (tid == 0) {
    mbar_init(&s_bar[0], 1);
    mbar_init(&s_bar[1], 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  bool ok = true;

  auto stage_ptr = [&](int b) { return smem + (size_t)b * kPStage; };
  // copies of stage (group g) into buffer b
  auto issue = [&](int g, int b) {
    unsigned char *base = stage_ptr(b);
    uint32_t *words = reinterpret_cast<uint32_t *>(base);
    unsigned char *bt = base + kPWords + kPA;
    uint16_t *sz = reinterpret_cast<uint16_t *>(base + kPWords + kPA + kPB);
    const int k0 = g * kPK;
    // plane words: [row][plane][8 words] = 2 x 16 bytes per (row, plane)
    for (int q = tid; q < kPK * P * 2; q += kPThreads) {
      const int half = q & 1, rp = q >> 1, r = rp / P, p = rp - r * P;
      const uint32_t *src = a.planes + ((size_t)(k0 + r) * P + p) * a.W + m0 / 16 + 4 * half;
      cp_async16(words + (r * 4 + p) * 8 + 4 * half, src, 16);
    }
    // X rows of the token block, 8 columns (16 bytes) per copy; tokens past T: zero
    for (int q = tid; q < n_pad * (kPK / 8); q += kPThreads) {
      const int n = q / (kPK / 8), c = q - n * (kPK / 8);
      const bool in = n < nt;
      const uint16_t *src = a.x + (size_t)(t0 + (in ? n : 0)) * a.d_in + k0 + 8 * c;
      cp_async16(bt + kmajor_off(n, 8 * c, n_pad), src, in ? 16 : 0);
    }
    // s and z of group g for the tile's outputs
    if (tid < 2 * (kPM / 8)) {
      const int which = tid / (kPM / 8), c = tid - which * (kPM / 8);
      cp_async16(sz + which * kPM + 8 * c, (which ? a.z : a.s) + (size_t)g * a.d_out + m0 + 8 * c, 16);
    }
    cp_async_commit();
  };
  // rebuild w_hat of buffer b into its A tile: thread (og, rg) takes outputs
  // 8 og .. 8 og + 7 and rows 8 rg .. 8 rg + 7
  auto build = [&](int b) {
    unsigned char *base = stage_ptr(b);
    const uint32_t *words = reinterpret_cast<const uint32_t *>(base);
    unsigned char *at = base + kPWords;
    const uint16_t *sz = reinterpret_cast<const uint16_t *>(base + kPWords + kPA + kPB);
    const int og = tid & 15, rg = tid >> 4;
    float sv[8], zv[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      sv[e] = __half2float(__ushort_as_half(sz[8 * og + e]));
      zv[e] = __half2float(__ushort_as_half(sz[kPM + 8 * og + e]));
    }
    uint32_t packed[8][4];  // [output e][row pair]
#pragma unroll
    for (int rr = 0; rr < 8; ++rr) {
      const int r = 8 * rg + rr;
      uint32_t q[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
      for (int p = 0; p < P; ++p) {
        const uint32_t w = words[(r * 4 + p) * 8 + (og >> 1)] >> (16 * (og & 1));
        const int sh = 2 * (P - 1 - p);
#pragma unroll
        for (int e = 0; e < 8; ++e) q[e] |= ((w >> (2 * e)) & 3u) << sh;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float wv = fmaf(sv[e], (float)q[e] + phiP, zv[e]);
        const uint32_t h = (uint32_t)__half_as_ushort(__float2half_rn(wv));
        if (rr & 1)
          packed[e][rr >> 1] |= h << 16;
        else
          packed[e][rr >> 1] = h;
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e)
      *reinterpret_cast<uint4 *>(at + kmajor_off(8 * og + e, 8 * rg, kPM)) =
          make_uint4(packed[e][0], packed[e][1], packed[e][2], packed[e][3]);
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");  // for the tensor cores
  };
  const uint32_t idesc = (1u << 4) | ((uint32_t)(n_pad >> 3) << 17) | ((uint32_t)(kPM >> 4) << 24);
  auto mma_stage = [&](int b, bool first) {
    const uint32_t a_addr = smem_u32(stage_ptr(b) + kPWords);
    const uint32_t b_addr = smem_u32(stage_ptr(b) + kPWords + kPA);
    tc_fence_after();
#pragma unroll
    for (int h = 0; h < kPK / 16; ++h) {
      const uint64_t ad = kmajor_desc(a_addr + h * kPM * 32), bd = kmajor_desc(b_addr + h * n_pad * 32);
      const uint32_t acc = (first && h == 0) ? 0u : 1u;
      asm volatile(
          "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
          "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem),
          "l"(ad), "l"(bd), "r"(idesc), "r"(acc)
          : "memory");
    }
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                     smem_u32(&s_bar[b]))
                 : "memory");
  };

  // ---- pipeline over the slice's groups: copy g+1 while building and multiplying g
  unsigned ph0 = 0u, ph1 = 0u;  // parity of the next phase of s_bar[0] / s_bar[1]
  auto wait_buf = [&](int b) {
    if (b == 0) {
      ok = mbar_wait(&s_bar[0], ph0) && ok;
      ph0 ^= 1u;
    } else {
      ok = mbar_wait(&s_bar[1], ph1) && ok;
      ph1 ^= 1u;
    }
  };
  const int ng = g_hi - g_lo;
  if (ng > 0) issue(g_lo, 0);
  for (int i = 0; i < ng; ++i) {
    const int b = i & 1;
    cp_async_wait0();
    __syncthreads();  // stage i's copies landed for everyone
    if (i + 1 < ng) {
      if (i >= 1) wait_buf(b ^ 1);  // buffer b^1 was last multiplied at stage i-1
      issue(g_lo + i + 1, b ^ 1);
    }
    build(b);
    tc_fence_before();
    __syncthreads();  // the A tile is complete
    if (tid == 0) mma_stage(b, i == 0);
  }
  // wait for the MMAs still in flight (the last one or two stages)
  if (ng > 0) {
    const int bl = (ng - 1) & 1;
    if (ng >= 2) wait_buf(bl ^ 1);
    wait_buf(bl);
  }
  tc_fence_after();

  // ---- epilogue: lane = output, column = token; the 4 warps of a quadrant pair
  // split the columns (warps w and w + 4 read lanes 32 (w mod 4) ..)
  if (ng > 0) {
    const int quad = warp & 3, half = warp >> 2, o = m0 + 32 * quad + lane;
    for (int c0 = 8 * half; c0 < n_pad; c0 += 16) {
      uint32_t v[8];
      asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n"
                   : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
                     "=r"(v[7])
                   : "r"(tmem + ((uint32_t)(32 * quad) << 16) + (uint32_t)c0)
                   : "memory");
      asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (c0 + j < nt) atomicAdd(a.y + (size_t)(t0 + c0 + j) * a.d_out + o, __uint_as_float(v[j]));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kPN) : "memory");
  }
  if (!ok && tid == 0) atomicCAS(a.error, 0, kDevErrPrefillTimeout);
}

}  // namespace

size_t prefill_ws_bytes() { return sizeof(WsHeader); }

cudaError_t launch_prefill(const uint32_t *planes, const uint16_t *s, const uint16_t *z,
                           const uint16_t *x, const float *phi, int T, int d_in, int d_out,
                           int b_max, float *y, void *ws, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(y, 0, (size_t)T * d_out * sizeof(float), st);
  if (e != cudaSuccess) return e;
  e = ensure_smem_attr((const void *)prefill_kernel, kPSmem);
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
  a.b_max = b_max;
  a.P = b_max / 2;
  a.W = d_out / 16;
  a.y = y;
  a.error = &reinterpret_cast<WsHeader *>(ws)->error;
  int sms = kNumSMs;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int tiles = d_out / kPM, tblocks = (T + kPN - 1) / kPN, groups = d_in / kPK;
  int k_slices = (sms + tiles * tblocks - 1) / (tiles * tblocks);  // about one wave
  if (k_slices > groups) k_slices = groups;
  if (k_slices < 1) k_slices = 1;
  a.k_slices = k_slices;
  prefill_kernel<<<dim3(tiles, k_slices, tblocks), kPThreads, kPSmem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace grinqh
