// Gauge-training statistics with the gauge folded into the channel DCT, on
// tcgen05 with tensor memory holding one operand of each GEMM (bf16 input,
// d_head = 128, whole 128-token tiles).
//
// Codec-Gauge, Method (frequency-distribution objective): every 16 x 128 block
// of X' = G X gets U = C_16 X' C_d^T, L_freq = sum r U^2 / sum U^2 and
// L_rate = mean log(1 + |U| / tau) (assumed form), and the objective's
// gradient flows back to the group gauges.
//
// Restructured so the channel frequency v is the tensor-memory lane:
//   U1^T = M x^T with M = C_d blockdiag(G)   (one GEMM per 128-token tile: the
//        gauge is folded into the DCT matrix; x is bf16, exact, streamed by
//        TMA; M sits in tensor memory as two bf16 terms, M = M_hi + M_lo to
//        2^-17, as the A operand),
// so a thread owning lane v holds its channel-frequency row over the tile's
// tokens and the 16-point token DCT of every block is local to the thread.
// With the gradient:
//   dU1^T[v][t] = sum_u C_16[u][t] dU[v][u]   (thread-local again), written
//        back into tensor memory as two bf16 terms, and
//   dM += dU1^T x                             (a second GEMM per tile, A from
//        tensor memory, x from the same shared-memory stage, MN-major),
//   dG_r[i][j] = sum_v C_d[v][16 r + i] dM[v][16 r + j]   (once per slice).
//
// With dL/dG (the first kernel below; the statistics-only kernel follows it)
// the roles are (one CTA per SM; the work unit is half a head slice when the
// slice has an even number of tiles, else the whole slice, and each unit's dG
// partial is a fixed-order sum): warp 0 streams x tiles (two 16 KB boxes, 128-byte
// swizzle, no multicast) into a 4-stage ring and stages each slice's G; warp 1
// allocates tensor memory and issues the MMAs; warps 2..9 (channel quarter =
// warp mod 4, token half = (warp - 2) / 4) build M, run the token DCT, the
// statistics and the gradient.  Tensor memory: [0,128) U1^T, [128,256) M,
// [256,384) dU1^T, [384,512) dM.  Every mbarrier wait is bounded in time.
#include <cuda.h>

#include <utility>

#include "cg_kernels.cuh"

namespace cg {

namespace {

constexpr int kD = 128, kTile = 128, kStages = 4;
constexpr int kXBytes = kTile * kD * 2;
constexpr int kWorkerWarps = 8;
constexpr int kThreads = (2 + kWorkerWarps) * 32;
constexpr uint32_t kColU = 0, kColM = 128, kColDU = 256, kColDM = 384;
constexpr int kDmPitch = kD + 1;
// smem: 1024 align + ring + 2 G + dM staging + reductions + barriers
constexpr int kSmem = 1024 + kStages * kXBytes + 2 * 8192 + kD * kDmPitch * 4 + 2 * 2 * 4 * 12 * 4 + 2 * 512 * 4 + 256;

// Orthonormal DCT-II coefficients C_16[u][t] for t < 8 (the other half follows
// from C_16[u][15 - t] = (-1)^u C_16[u][t]): 1/4 for u = 0, else
// sqrt(1/8) cos(pi (2 t + 1) u / 32), folded onto sqrt(1/8) cos(k pi / 32), 0 <= k <= 16.
constexpr float kCosPi32[17] = {0.3535533845424652f, 0.3518509268760681f, 0.34675997495651245f, 0.3383294939994812f,
                                0.3266407549381256f, 0.31180626153945923f, 0.29396888613700867f, 0.2733004689216614f,
                                0.25f, 0.22429189085960388f, 0.19642373919487f, 0.16666391491889954f,
                                0.13529902696609497f, 0.10263112932443619f, 0.06897484511137009f, 0.034654293209314346f,
                                0.0f};
constexpr float c16_value(int u, int t) {
  int k = ((2 * t + 1) * u) % 64;  // cos(k pi / 32), period 64
  if (k > 32) k = 64 - k;          // cos(2 pi - a) = cos a
  float sg = 1.0f;
  if (k > 16) {                    // cos(pi - a) = -cos a
    k = 32 - k;
    sg = -1.0f;
  }
  return u == 0 ? 0.25f : sg * kCosPi32[k];
}

// Compile-time loop: the body sees its index as a constant expression, so the
// DCT coefficients below become immediates.
template <typename F, int... I>
__device__ __forceinline__ void unroll_seq(F&& f, std::integer_sequence<int, I...>) {
  (f(std::integral_constant<int, I>{}), ...);
}
template <int N, typename F>
__device__ __forceinline__ void unroll_n(F&& f) {
  unroll_seq(f, std::make_integer_sequence<int, N>{});
}
__device__ __forceinline__ float2 dup2(float c) { return make_float2(c, c); }
__device__ __forceinline__ float2 sub2(float2 a, float2 b) { return __ffma2_rn(b, dup2(-1.0f), a); }
// log2 of an argument >= 1 (never subnormal, so flushing changes nothing)
__device__ __forceinline__ float lg2_ftz(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 16-point orthonormal DCT-II of two token blocks at once (block A in .x, block B
// in .y), by partial butterflies on the symmetry C_16[u][15 - t] = (-1)^u C_16[u][t]:
// sums a and differences b of mirrored tokens; the odd frequencies are the 8 x 8
// half of C_16 on b; the even ones an 8-point DCT of a, split the same way twice
// (c, e = a[t] +- a[7 - t]; f, g = c[t] +- c[3 - t]).  100 paired operations per
// 32 coefficients against 256 scalar ones for the plain matrix product.
__device__ __forceinline__ void dct16_pair(const float* sa, const float* sb, float2 (&U)[16]) {
  float2 a[8], b[8];
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    a[t] = make_float2(sa[t] + sa[15 - t], sb[t] + sb[15 - t]);
    b[t] = make_float2(sa[t] - sa[15 - t], sb[t] - sb[15 - t]);
  }
  unroll_n<8>([&](auto k) {  // u = 1, 3, .., 15
    constexpr int u = 2 * decltype(k)::value + 1;
    constexpr float c0 = c16_value(u, 0);
    float2 acc = __fmul2_rn(dup2(c0), b[0]);
    unroll_n<7>([&](auto t1) {
      constexpr int t = decltype(t1)::value + 1;
      constexpr float ct = c16_value(u, t);
      acc = __ffma2_rn(dup2(ct), b[t], acc);
    });
    U[u] = acc;
  });
  float2 c[4], e[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    c[t] = __fadd2_rn(a[t], a[7 - t]);
    e[t] = sub2(a[t], a[7 - t]);
  }
  unroll_n<4>([&](auto k) {  // u = 2, 6, 10, 14
    constexpr int u = 4 * decltype(k)::value + 2;
    constexpr float c0 = c16_value(u, 0);
    float2 acc = __fmul2_rn(dup2(c0), e[0]);
    unroll_n<3>([&](auto t1) {
      constexpr int t = decltype(t1)::value + 1;
      constexpr float ct = c16_value(u, t);
      acc = __ffma2_rn(dup2(ct), e[t], acc);
    });
    U[u] = acc;
  });
  const float2 f0 = __fadd2_rn(c[0], c[3]), f1 = __fadd2_rn(c[1], c[2]);
  const float2 g0 = sub2(c[0], c[3]), g1 = sub2(c[1], c[2]);
  unroll_n<2>([&](auto k) {  // u = 4, 12
    constexpr int u = 8 * decltype(k)::value + 4;
    constexpr float c0 = c16_value(u, 0), c1 = c16_value(u, 1);
    U[u] = __ffma2_rn(dup2(c1), g1, __fmul2_rn(dup2(c0), g0));
  });
  U[0] = __fmul2_rn(dup2(0.25f), __fadd2_rn(f0, f1));  // C_16[0][t] = 1/4
  U[8] = __fmul2_rn(dup2(0.25f), sub2(f0, f1));        // C_16[8][t] = 1/4, -1/4 for t = 0, 1
}

// The transpose of dct16_pair, s[t] = sum_u C_16[u][t] dU[u] for two blocks at once: the
// same butterflies taken backwards (odd frequencies onto the differences b, u = 2 mod 4
// onto e, u = 4, 12 onto g, u = 0, 8 onto f, then the sums and differences undone).
__device__ __forceinline__ void idct16_pair(const float2 (&dU)[16], float2 (&s)[16]) {
  float2 db[8], de[4], dg[2];
  unroll_n<8>([&](auto tt) {
    constexpr int t = decltype(tt)::value;
    constexpr float c1 = c16_value(1, t);
    float2 acc = __fmul2_rn(dup2(c1), dU[1]);
    unroll_n<7>([&](auto k1) {
      constexpr int u = 2 * decltype(k1)::value + 3;
      constexpr float cu = c16_value(u, t);
      acc = __ffma2_rn(dup2(cu), dU[u], acc);
    });
    db[t] = acc;
  });
  unroll_n<4>([&](auto tt) {
    constexpr int t = decltype(tt)::value;
    constexpr float c2 = c16_value(2, t);
    float2 acc = __fmul2_rn(dup2(c2), dU[2]);
    unroll_n<3>([&](auto k1) {
      constexpr int u = 4 * decltype(k1)::value + 6;
      constexpr float cu = c16_value(u, t);
      acc = __ffma2_rn(dup2(cu), dU[u], acc);
    });
    de[t] = acc;
  });
  unroll_n<2>([&](auto tt) {
    constexpr int t = decltype(tt)::value;
    constexpr float c4 = c16_value(4, t), c12 = c16_value(12, t);
    dg[t] = __ffma2_rn(dup2(c12), dU[12], __fmul2_rn(dup2(c4), dU[4]));
  });
  const float2 df0 = __fmul2_rn(dup2(0.25f), __fadd2_rn(dU[0], dU[8]));
  const float2 df1 = __fmul2_rn(dup2(0.25f), sub2(dU[0], dU[8]));
  const float2 dc[4] = {__fadd2_rn(df0, dg[0]), __fadd2_rn(df1, dg[1]), sub2(df1, dg[1]), sub2(df0, dg[0])};
  float2 da[8];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    da[t] = __fadd2_rn(dc[t], de[t]);
    da[7 - t] = sub2(dc[t], de[t]);
  }
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    s[t] = __fadd2_rn(da[t], db[t]);
    s[15 - t] = sub2(da[t], db[t]);
  }
}

// Per-block sums over the 16 frequencies of a thread's channel frequency v, for the
// two blocks of a pair: E = sum U^2, F = sum r_uv U^2, R = sum log2(1 + |U| / tau).
// The logarithms are taken four at a time (log2 of the product of four arguments);
// a product overflows only when some |U| / tau is beyond about 2^32, and then the
// block's R is taken again two arguments at a time.
__device__ __forceinline__ void pair_sums(const float2 (&U)[16], const float2 (&rad2)[16], float inv_tau, float2& E,
                                          float2& F, float2& R) {
  auto arg = [&](int u) {
    return make_float2(__fmaf_rn(fabsf(U[u].x), inv_tau, 1.0f), __fmaf_rn(fabsf(U[u].y), inv_tau, 1.0f));
  };
  float2 p01 = make_float2(1.0f, 1.0f);
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const float2 e2 = __fmul2_rn(U[u], U[u]);
    if (u == 0) {
      E = e2;
      F = __fmul2_rn(rad2[0], e2);
    } else {
      E = __fadd2_rn(E, e2);
      F = __ffma2_rn(rad2[u], e2, F);
    }
    if ((u & 3) == 1) p01 = __fmul2_rn(arg(u - 1), arg(u));
    if ((u & 3) == 3) {
      const float2 q = __fmul2_rn(p01, __fmul2_rn(arg(u - 1), arg(u)));
      const float2 l = make_float2(lg2_ftz(q.x), lg2_ftz(q.y));
      R = u == 3 ? l : __fadd2_rn(R, l);
    }
  }
  if (!(fmaxf(R.x, R.y) < INFINITY)) {
#pragma unroll
    for (int u = 0; u < 16; u += 2) {
      const float2 q = __fmul2_rn(arg(u), arg(u + 1));
      const float2 l = make_float2(lg2_ftz(q.x), lg2_ftz(q.y));
      R = u == 0 ? l : __fadd2_rn(R, l);
    }
  }
}

// Sum of 12 per-lane values over a warp: afterwards lane l holds the total of
// value l >> 1 (l >> 1 < 12).  Each exchange halves the values a lane carries.
__device__ __forceinline__ float warp_sum12(const float (&p)[12], int lane) {
  float a8[8], a4[4], a2[2];
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const float lo = p[m], hi = m + 8 < 12 ? p[m + 8] : 0.0f;
    const bool up = lane & 16;
    a8[m] = (up ? hi : lo) + __shfl_xor_sync(0xffffffffu, up ? lo : hi, 16);
  }
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const bool up = lane & 8;
    a4[m] = (up ? a8[m + 4] : a8[m]) + __shfl_xor_sync(0xffffffffu, up ? a8[m] : a8[m + 4], 8);
  }
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    const bool up = lane & 4;
    a2[m] = (up ? a4[m + 2] : a4[m]) + __shfl_xor_sync(0xffffffffu, up ? a4[m] : a4[m + 2], 4);
  }
  const bool up = lane & 2;
  float r = (up ? a2[1] : a2[0]) + __shfl_xor_sync(0xffffffffu, up ? a2[0] : a2[1], 2);
  return r + __shfl_xor_sync(0xffffffffu, r, 1);
}

__device__ __forceinline__ uint64_t kdesc(uint32_t addr) {  // K-major, 128-byte swizzle
  uint64_t d = (uint64_t)((addr & 0x3FFFFu) >> 4);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}
__device__ __forceinline__ uint64_t mndesc(uint32_t addr) {  // MN-major, 128-byte swizzle, 64-element halves 16 KB apart
  uint64_t d = (uint64_t)((addr & 0x3FFFFu) >> 4);
  d |= (uint64_t)(16384 >> 4) << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}
constexpr uint32_t idesc(bool b_mn) {  // D fp32, A / B bf16, A from tensor memory, M = N = 128
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn ? 1u : 0u) << 16) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
}
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a_tmem, uint64_t bdesc, uint32_t id, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d),
      "r"(a_tmem), "l"(bdesc), "r"(id), "r"(acc));
}
__device__ __forceinline__ void commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
      "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
// split fp32 pairs into bf16 hi and lo pairs (x = hi + lo to 2^-17)
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16x2(x0, x1);
  lo = pack_bf16x2(x0 - bf16lo(hi), x1 - bf16hi(hi));
}
// Orthonormal DCT-II C_d[v][c] (d = 128) from cosk[k] = cos(k pi / 256), k = 0..128,
// a table each CTA fills once: the angle (2 c + 1) v pi / 256 is folded onto [0, pi / 2].
constexpr int kCosTab = 2 * 512;  // cos(k pi / 256) for a full period, each entry twice (a packed pair)
__device__ __forceinline__ float cd_tab(const float* cosk, int v, int c) {
  return (v == 0 ? 0.08838834764831845f : 0.125f) * cosk[2 * (((2 * c + 1) * v) & 511)];  // sqrt(1/128), sqrt(2/128)
}
__device__ __forceinline__ void fill_cos_table(float* cosk, int wid) {  // wid = 0 .. 255
  for (int k = wid; k < 512; k += 256) {
    const float c = cospif((float)k / 256.0f);
    cosk[2 * k] = c;
    cosk[2 * k + 1] = c;
  }
}
// Channels 16 r .. 16 r + 15 of row v of M = C_d blockdiag(G) (C_d alone without a
// gauge), M[v][16 r + j] = sum_i C_d[v][16 r + i] G_r[i][j], as bf16 hi / lo pairs.
// The angle index (2 c + 1) v steps by 2 v from one channel to the next; the products
// run on fp32 pairs (two output channels per instruction).
__device__ __forceinline__ void m_group(const float* cosk, const float* G, bool has_g, int v, int r, uint32_t (&h8)[8],
                                        uint32_t (&l8)[8]) {
  const float2 sc = dup2(v == 0 ? 0.08838834764831845f : 0.125f);
  const float2* cos2 = reinterpret_cast<const float2*>(cosk);
  int k = ((32 * r + 1) * v) & 511;
  float2 m2[8];
  if (has_g) {
#pragma unroll
    for (int ii = 0; ii < 16; ++ii) {
      const float2 cc = cos2[k];
      k = (k + 2 * v) & 511;
      const float4* row = reinterpret_cast<const float4*>(G + (r * 16 + ii) * 16);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 g = row[q];
        const float2 g01 = make_float2(g.x, g.y), g23 = make_float2(g.z, g.w);
        m2[2 * q] = ii == 0 ? __fmul2_rn(cc, g01) : __ffma2_rn(cc, g01, m2[2 * q]);
        m2[2 * q + 1] = ii == 0 ? __fmul2_rn(cc, g23) : __ffma2_rn(cc, g23, m2[2 * q + 1]);
      }
    }
  } else {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float c0 = cos2[k].x;
      k = (k + 2 * v) & 511;
      m2[q] = make_float2(c0, cos2[k].x);
      k = (k + 2 * v) & 511;
    }
  }
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float2 m = __fmul2_rn(sc, m2[q]);
    split2(m.x, m.y, h8[q], l8[q]);
  }
}

struct TmArgs {
  KvGeom k;
  int has_g, want_grad;
  int pieces;  // work units per head slice (dL/dG kernel)
  float lambda_f, lambda_r, tau;
  double inv_nblk, inv_ncoef;
  const float* G;
  float* lfreq;
  float* lrate;
  float* dg_part;
  unsigned int* status;
};

}  // namespace

__global__ void __launch_bounds__(kThreads, 1) spectral_tmem_kernel(const __grid_constant__ CUtensorMap tmap, TmArgs a) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  unsigned char* xs = base;                                            // ring of x tiles
  float* gs = reinterpret_cast<float*>(xs + kStages * kXBytes);        // 2 x [8][16][16] G
  float* dms = gs + 2 * 2048;                                          // [128][129] dM staging
  float* red = dms + kD * kDmPitch;                                    // [2 tile parity][2 half][4 quarter][12]
  float* cosk = red + 2 * 2 * 4 * 12;                                  // cos(k pi / 256)
  uint64_t* bars = reinterpret_cast<uint64_t*>(cosk + kCosTab);
  uint64_t* x_full = bars;
  uint64_t* x_empty = bars + kStages;
  uint64_t* g_full = bars + 2 * kStages;       // [2]
  uint64_t* g_empty = g_full + 2;              // [2]
  uint64_t* m_full = g_empty + 2;
  uint64_t* m_empty = m_full + 1;
  uint64_t* u_full = m_empty + 1;
  uint64_t* u_empty = u_full + 1;
  uint64_t* du_full = u_empty + 1;
  uint64_t* du_empty = du_full + 1;
  uint64_t* dm_full = du_empty + 1;
  uint64_t* dm_empty = dm_full + 1;
  uint64_t* mma_done = dm_empty + 1;
  uint32_t* tmem_base = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile uint32_t* abort_flag = tmem_base + 1;  // set by the first wait that gives up
  // After one wait has given up, the later ones are skipped, so a broken
  // pipeline costs one time limit per role, not one per tile.
  auto wait = [&](uint64_t* bar, uint32_t parity) {
    if (*abort_flag) return;
    if (!mbar_wait(bar, parity, a.status)) *abort_flag = 1u;
  };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Work unit: a piece of a head slice, tiles / pieces consecutive 128-token tiles
  // (half a slice when the tile count is even), each with its own dG partial.
  const long long units = a.k.slices() * a.pieces;
  const int tiles = a.k.T / kTile / a.pieces;  // tiles per piece
  const int n_my = (int)((units - blockIdx.x + gridDim.x - 1) / gridDim.x);  // pieces of this CTA

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&x_full[s], 1);
      mbar_init(&x_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&g_full[s], 1);
      mbar_init(&g_empty[s], kWorkerWarps);
    }
    mbar_init(m_full, kWorkerWarps);
    mbar_init(m_empty, 1);
    mbar_init(u_full, 1);
    mbar_init(u_empty, kWorkerWarps);
    mbar_init(du_full, kWorkerWarps);
    mbar_init(du_empty, 1);
    mbar_init(dm_full, 1);
    mbar_init(dm_empty, kWorkerWarps);
    mbar_init(mma_done, 1);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp >= 2) fill_cos_table(cosk, threadIdx.x - 64);
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_base)), "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_base;

  if (warp == 0) {
    // ---------------- producer: G of each slice, x tiles ----------------
    if (lane == 0) {
      int i = 0, g_issued = 0;
      for (int si = 0; si < n_my && !*abort_flag; ++si) {
        const long long unit = blockIdx.x + (long long)si * gridDim.x, slice = unit / a.pieces;
        const int t0 = (int)(unit % a.pieces) * tiles;  // first tile of the piece within its slice
        if (a.has_g) {
          const int gb = si & 1;
          wait(&g_empty[gb], ((uint32_t)(si >> 1) & 1u) ^ 1u);
          int l, sk, b, h;
          slice_coords(slice, a.k, l, sk, b, h);
          mbar_arrive_expect_tx(&g_full[gb], 8192);
          bulk_g2s(gs + gb * 2048, a.G + gauge_set(l, sk, h, a.k) * 2048, 8192, &g_full[gb]);
          g_issued = si + 1;
        }
        for (int j = 0; j < tiles && !*abort_flag; ++j, ++i) {
          const int s = i % kStages;
          wait(&x_empty[s], ((uint32_t)(i / kStages) & 1u) ^ 1u);
          mbar_arrive_expect_tx(&x_full[s], kXBytes);
          const int row0 = (int)(slice * a.k.T + (long long)(t0 + j) * kTile);
          tma_load_2d(xs + s * kXBytes, &tmap, 0, row0, &x_full[s]);
          tma_load_2d(xs + s * kXBytes + 16384, &tmap, 64, row0, &x_full[s]);
        }
      }
      // Drain: the last copy into every stage and G buffer has landed before the
      // CTA can exit (immediate unless a wait above gave up).
      for (int s = 0; s < kStages && s < i; ++s) {
        const int last = ((i - 1 - s) / kStages) * kStages + s;
        mbar_wait(&x_full[s], (uint32_t)(last / kStages) & 1u, a.status);
      }
      for (int si = g_issued - 2 < 0 ? 0 : g_issued - 2; si < g_issued; ++si)
        mbar_wait(&g_full[si & 1], (uint32_t)(si >> 1) & 1u, a.status);
    }
  } else if (warp == 1) {
    // ---------------- MMA issue (one thread) ----------------
    // Tile f's forward GEMM is issued as soon as its x stage is loaded and the
    // workers have read tile f-1's U1, i.e. before tile f-1's backward GEMM, except
    // at the start of a slice with a gauge: its M is built only after the previous
    // slice's dG, which needs the previous backward first.
    if (lane == 0) {
      const int N = n_my * tiles;
      int f = 0;  // next forward GEMM to issue
      auto forward = [&](int t) {
        const int si = t / tiles, j = t % tiles, s = t % kStages;
        if (j == 0 && (si == 0 || a.has_g)) wait(m_full, (uint32_t)(a.has_g ? si : 0) & 1u);
        wait(&x_full[s], (uint32_t)(t / kStages) & 1u);
        wait(u_empty, ((uint32_t)t & 1u) ^ 1u);
        fence_after();
        const uint32_t xa = smem_u32(xs + s * kXBytes);
        // U1^T[v][t] = sum_c M[v][c] x[t][c]: A = M (tensor memory), B = x (K-major)
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t bd = kdesc(xa + (k >> 2) * 16384 + (k & 3) * 32);
          mma_ts(tmem + kColU, tmem + kColM + 8 * k, bd, idesc(false), k > 0);
          mma_ts(tmem + kColU, tmem + kColM + 64 + 8 * k, bd, idesc(false), 1);
        }
        commit(u_full);
        if (a.has_g && j == tiles - 1) commit(m_empty);  // this slice's M is no longer read
      };
      for (int i = 0; i < N && !*abort_flag; ++i) {  // after a wait gave up, nothing more is issued
        if (f == i) forward(f++);
        if (f < N && (f % tiles != 0 || !a.has_g)) forward(f++);
        const int si = i / tiles, j = i % tiles, s = i % kStages;
        if (a.want_grad) {
          wait(du_full, (uint32_t)i & 1u);
          if (j == 0 && si > 0) wait(dm_empty, (uint32_t)(si - 1) & 1u);
          fence_after();
          const uint32_t xa = smem_u32(xs + s * kXBytes);
          // dM[v][c] += sum_t dU1^T[v][t] x[t][c]: A = dU1^T (tensor memory), B = x (MN-major)
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint64_t bd = mndesc(xa + k * 2048);
            mma_ts(tmem + kColDM, tmem + kColDU + 8 * k, bd, idesc(true), (j > 0 || k > 0) ? 1u : 0u);
            mma_ts(tmem + kColDM, tmem + kColDU + 64 + 8 * k, bd, idesc(true), 1);
          }
          commit(du_empty);
          if (j == tiles - 1) commit(dm_full);
        }
        commit(&x_empty[s]);  // tile i's stage: both of its GEMMs have been issued before this commit
      }
      commit(mma_done);  // every MMA has completed before tensor memory is freed
      mbar_wait(mma_done, 0u, a.status);
    }
  } else {
    // ---------------- workers: thread = channel frequency v (tensor-memory lane), token half ----------------
    const int wq = warp & 3, hf = (warp - 2) >> 2, wid = threadIdx.x - 64;  // wid 0..255
    const int v = 32 * wq + lane;
    const uint32_t lrow = (uint32_t)(32 * wq) << 16;
    const float inv_tau = 1.0f / a.tau;
    float2 rad2[16];
    {
      const float rv = (float)v / (kD - 1);
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const float ru = (float)u / 15.0f;
        rad2[u] = dup2(sqrtf(ru * ru + rv * rv) * 0.70710678118654752f);
      }
    }
    int i = 0;
    for (int si = 0; si < n_my; ++si) {
      const long long unit = blockIdx.x + (long long)si * gridDim.x, slice = unit / a.pieces;
      const int t0 = (int)(unit % a.pieces) * tiles;
      if (si == 0 || a.has_g) {
        // M[v][c] = sum_i C_d[v][16 r + i] G_r[i][j] for this thread's 64 channels c = 64 hf ..
        if (a.has_g) wait(&g_full[si & 1], (uint32_t)(si >> 1) & 1u);
        if (si > 0) wait(m_empty, (uint32_t)(si - 1) & 1u);
        __syncwarp();
        fence_after();
        const float* G = gs + (si & 1) * 2048;
#pragma unroll 1
        for (int r4 = 0; r4 < 4; ++r4) {
          const int r = 4 * hf + r4;
          uint32_t h8[8], l8[8];
          m_group(cosk, G, a.has_g, v, r, h8, l8);
          st8(tmem + lrow + kColM + 8 * r, h8);        // channels 16 r .. 16 r + 15: column pairs 8 r ..
          st8(tmem + lrow + kColM + 64 + 8 * r, l8);
        }
        wait_st();
        fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(m_full);
          if (a.has_g) mbar_arrive(&g_empty[si & 1]);
        }
      }
      for (int j = 0; j < tiles; ++j, ++i) {
        // U1^T row v, tokens 64 hf .. 64 hf + 63
        wait(u_full, (uint32_t)i & 1u);
        __syncwarp();
        fence_after();
        float x[64];
        ld32(tmem + lrow + kColU + 64 * hf, x);
        ld32(tmem + lrow + kColU + 64 * hf + 32, x + 32);
        wait_ld();
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(u_empty);
        // token DCT of the four 16-token blocks (even / odd halves), and this v's share of the sums
        float part[12];  // per block kb: sum U^2, sum r U^2, sum log2(1 + |U|/tau) at 3 kb
#pragma unroll
        for (int p = 0; p < 2; ++p) {  // blocks 2 p and 2 p + 1 as fp32 pairs
          float2 U[16], E, F, R;
          dct16_pair(x + 32 * p, x + 32 * p + 16, U);
          pair_sums(U, rad2, inv_tau, E, F, R);
#pragma unroll
          for (int u = 0; u < 16; ++u) {  // U in place of the blocks' columns
            x[32 * p + u] = U[u].x;
            x[32 * p + 16 + u] = U[u].y;
          }
          part[6 * p] = E.x;
          part[6 * p + 1] = F.x;
          part[6 * p + 2] = R.x;
          part[6 * p + 3] = E.y;
          part[6 * p + 4] = F.y;
          part[6 * p + 5] = R.y;
        }
        const float tot = warp_sum12(part, lane);
        float* rb = red + ((i & 1) * 2 + hf) * 48;  // [quarter][12] of this tile parity and half
        if (!(lane & 1) && (lane >> 1) < 12) rb[wq * 12 + (lane >> 1)] = tot;
        named_bar_sync(2 + hf, 128);
        float E[4], F[4], R[4], lf[4];
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
          E[kb] = (rb[0 * 12 + 3 * kb] + rb[1 * 12 + 3 * kb]) + (rb[2 * 12 + 3 * kb] + rb[3 * 12 + 3 * kb]);
          F[kb] = (rb[0 * 12 + 3 * kb + 1] + rb[1 * 12 + 3 * kb + 1]) + (rb[2 * 12 + 3 * kb + 1] + rb[3 * 12 + 3 * kb + 1]);
          R[kb] = (rb[0 * 12 + 3 * kb + 2] + rb[1 * 12 + 3 * kb + 2]) + (rb[2 * 12 + 3 * kb + 2] + rb[3 * 12 + 3 * kb + 2]);
          lf[kb] = E[kb] > 0.0f ? __fdividef(F[kb], E[kb]) : 0.0f;
        }
        if (wq == 0 && lane == 0) {
          const long long blk0 = slice * (a.k.T / 16) + (long long)(t0 + j) * 8 + 4 * hf;
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
            a.lfreq[blk0 + kb] = lf[kb];
            a.lrate[blk0 + kb] = R[kb] * 0.69314718055994531f / (16.0f * kD);
          }
        }
        if (!a.want_grad) continue;
        // dL/dU, then dU1^T[v][t] = sum_u C_16[u][t] dU[u], into tensor memory as bf16 hi + lo
        if (i > 0) wait(du_empty, (uint32_t)(i - 1) & 1u);
        __syncwarp();
        fence_after();
        const float cr = (float)(a.lambda_r * a.inv_ncoef);
        const float cf0 = (float)(2.0 * a.lambda_f * a.inv_nblk);
#pragma unroll
        for (int p = 0; p < 2; ++p) {  // blocks 2 p and 2 p + 1 as fp32 pairs
          float2 dU[16], d1[16];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int kb = 2 * p + h;
            const float cf = E[kb] > 0.0f ? __fdividef(cf0, E[kb]) : 0.0f;
#pragma unroll
            for (int u = 0; u < 16; ++u) {
              const float U = x[16 * kb + u];
              const float sg = U > 0.0f ? 1.0f : (U < 0.0f ? -1.0f : 0.0f);
              const float g = __fmaf_rn(cf * U, rad2[u].x - lf[kb], __fdividef(cr * sg, a.tau + fabsf(U)));
              if (h == 0) dU[u].x = g;
              else dU[u].y = g;
            }
          }
          idct16_pair(dU, d1);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t h8[8], l8[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float2 e0 = d1[2 * q], e1 = d1[2 * q + 1];
              split2(h ? e0.y : e0.x, h ? e1.y : e1.x, h8[q], l8[q]);
            }
            st8(tmem + lrow + kColDU + 32 * hf + 8 * (2 * p + h), h8);
            st8(tmem + lrow + kColDU + 64 + 32 * hf + 8 * (2 * p + h), l8);
          }
        }
        wait_st();
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(du_full);
        if (j == tiles - 1) {
          // dG_r[i][j] = sum_v C_d[v][16 r + i] dM[v][16 r + j] for this piece
          wait(dm_full, (uint32_t)si & 1u);
          __syncwarp();
          fence_after();
          float dm[64];
          ld32(tmem + lrow + kColDM + 64 * hf, dm);
          ld32(tmem + lrow + kColDM + 64 * hf + 32, dm + 32);
          wait_ld();
          fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(dm_empty);
#pragma unroll
          for (int c = 0; c < 64; ++c) dms[v * kDmPitch + 64 * hf + c] = dm[c];
          named_bar_sync(1, kWorkerWarps * 32);
          {
            const int ri = wid >> 1, r = ri >> 4, ii = ri & 15, j0 = 8 * (wid & 1);
            float acc[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] = 0.0f;
#pragma unroll 4
            for (int vv = 0; vv < kD; ++vv) {
              const float c = cd_tab(cosk, vv, 16 * r + ii);
              const float* row = dms + vv * kDmPitch + 16 * r + j0;
#pragma unroll
              for (int q = 0; q < 8; ++q) acc[q] = __fmaf_rn(c, row[q], acc[q]);
            }
            float* dst = a.dg_part + unit * (long long)kD * 16 + (r * 16 + ii) * 16 + j0;
#pragma unroll
            for (int q = 0; q < 8; ++q) dst[q] = acc[q];
          }
          named_bar_sync(1, kWorkerWarps * 32);  // dms is rewritten at the next piece's end
        }
      }
    }
  }
  fence_before();
  __syncthreads();
  if (warp == 1) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

// ---------------------------------------------------------------------------
// Statistics without dL/dG.  The 128-token tiles of all head slices are split
// into contiguous ranges, one per CTA (a range may start inside a slice and
// cross into the next ones, each with its own gauge), instead of whole slices,
// and U1^T is double-buffered in tensor memory so the GEMM of tile i + 1 runs
// while the workers take tile i's token DCT and statistics.  M is double-buffered
// too: the workers build the next slice's M during the current slice's last tiles
// (each token part at its own tile, from a G the producer loads a slice ahead), so
// the GEMM of the next slice's first tile overlaps the current slice's statistics.
// bf16 input: 16 worker warps, lane quarter = warp mod 4, token part (32 tokens) =
// (warp - 2) / 4.  fp32 input: 8 worker warps, token halves of 64 tokens.
// Tensor memory: [0,128) and [384,512) M (bf16 hi, lo), [128,256) and [256,384) U1^T.
namespace {

constexpr uint32_t kFColM0 = 0, kFColM1 = 384, kFColU1 = 128;
__device__ __forceinline__ uint32_t fwd_mcol(int q) { return (q & 1) ? kFColM1 : kFColM0; }
constexpr int kRedPitch = 132;  // [3 x blocks][kRedPitch] partial sums of a token part, by channel frequency v
// bf16 input: a 4-stage ring of bf16 tiles, block sums finished in shared memory.  fp32 input:
// a 2-stage ring of fp32 tiles (four 32-channel TMA boxes each), the current tile split by the
// workers into bf16 hi and lo tiles (x = hi + lo to 2^-17), block sums by the warp butterfly.
template <bool F32>
struct FwdCfg {
  static constexpr int WW = F32 ? 8 : 16;         // worker warps: 4 lane quarters x PARTS token parts
  static constexpr int PARTS = WW / 4;
  static constexpr int TPP = kTile / PARTS;       // tokens of a tile per part (64 or 32)
  static constexpr int BPP = TPP / 16;            // 16-token blocks per part
  static constexpr int THREADS = (2 + WW) * 32;
  static constexpr int NST = F32 ? 2 : kStages;
  static constexpr int STAGE = F32 ? 4 * 16384 : kXBytes;
  static constexpr int CONV = F32 ? 2 * kXBytes : 0;
  static constexpr int RED = F32 ? 2 * 2 * 4 * 12 : 2 * PARTS * 3 * BPP * kRedPitch;  // floats
  static constexpr int SMEM = 1024 + NST * STAGE + CONV + 2 * 8192 + RED * 4 + kCosTab * 4 + 256;
};


}  // namespace

template <bool F32>
__global__ void __launch_bounds__(FwdCfg<F32>::THREADS, 1) spectral_fwd_kernel(const __grid_constant__ CUtensorMap tmap, TmArgs a) {
  using C = FwdCfg<F32>;
  constexpr int NST = C::NST, WW = C::WW, PARTS = C::PARTS, TPP = C::TPP, BPP = C::BPP;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  unsigned char* xs = base;                                  // ring of input tiles
  unsigned char* cvt = xs + NST * C::STAGE;                  // fp32 input: bf16 hi tile, then lo tile
  float* gs = reinterpret_cast<float*>(cvt + C::CONV);       // 2 x [8][16][16] G
  float* red = gs + 2 * 2048;                                // block sums (see FwdCfg)
  float* cosk = red + C::RED;                                // cos(k pi / 256)
  uint64_t* bars = reinterpret_cast<uint64_t*>(cosk + kCosTab);
  uint64_t* x_full = bars;
  uint64_t* x_empty = bars + NST;
  uint64_t* g_full = bars + 2 * NST;      // [2]
  uint64_t* g_empty = g_full + 2;         // [2]
  uint64_t* m_full = g_empty + 2;         // [2]
  uint64_t* m_empty = m_full + 2;         // [2]
  uint64_t* u_full = m_empty + 2;         // [2]
  uint64_t* u_empty = u_full + 2;         // [2]
  uint64_t* mma_done = u_empty + 2;
  uint64_t* conv_full = mma_done + 1;     // fp32 input: the current tile's hi and lo tiles are written
  uint32_t* tmem_base = reinterpret_cast<uint32_t*>(conv_full + 1);
  volatile uint32_t* abort_flag = tmem_base + 1;
  auto wait = [&](uint64_t* bar, uint32_t parity) {
    if (*abort_flag) return;
    if (!mbar_wait(bar, parity, a.status)) *abort_flag = 1u;
  };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles = a.k.T / kTile;
  const long long total = a.k.slices() * tiles;
  const long long g0 = total * blockIdx.x / gridDim.x;
  const int n_t = (int)(total * (blockIdx.x + 1) / gridDim.x - g0);  // tiles of this CTA

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&x_full[s], 1);
      mbar_init(&x_empty[s], F32 ? WW : 1);  // freed by the split (fp32) or the GEMM (bf16)
    }
    mbar_init(conv_full, WW);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&g_full[s], 1);
      mbar_init(&g_empty[s], WW);
      mbar_init(&u_full[s], 1);
      mbar_init(&u_empty[s], WW);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&m_full[s], WW);
      mbar_init(&m_empty[s], 1);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0u;
    fence_mbar_init();
  }
  if (warp >= 2 && threadIdx.x < 64 + 256) fill_cos_table(cosk, threadIdx.x - 64);
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_base)), "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      int ls = -1, issued = 0, gq = 0;  // gq: G loads issued, for slices 0 .. gq - 1 of this range
      const int n_sl = (int)((g0 + n_t - 1) / tiles - g0 / tiles) + 1;  // slices this range touches
      // G of the range's q-th slice into buffer q & 1, once the workers have built the
      // M of slice q - 2 from it
      auto load_g = [&](int q) {
        const int gb = q & 1;
        wait(&g_empty[gb], ((uint32_t)(q >> 1) & 1u) ^ 1u);
        int l, sk, b, h;
        slice_coords(g0 / tiles + q, a.k, l, sk, b, h);
        mbar_arrive_expect_tx(&g_full[gb], 8192);
        bulk_g2s(gs + gb * 2048, a.G + gauge_set(l, sk, h, a.k) * 2048, 8192, &g_full[gb]);
      };
      int j = (int)(g0 % tiles) - 1;  // tile index within its slice, advanced per tile
      for (int i = 0; i < n_t && !*abort_flag; ++i) {  // after a wait gave up, nothing more is issued
        const long long gt = g0 + i;
        if (++j == tiles) j = 0;
        if (a.has_g && (i == 0 || j == 0)) {  // a slice starts: its G and the next slice's are on the way
          ++ls;
          while (gq <= ls + 1 && gq < n_sl && !*abort_flag) load_g(gq++);
        }
        const int s = i % NST;
        wait(&x_empty[s], ((uint32_t)(i / NST) & 1u) ^ 1u);
        mbar_arrive_expect_tx(&x_full[s], C::STAGE);
        const int row0 = (int)(gt * kTile);
        if constexpr (F32) {  // four boxes of 32 fp32 channels (128-byte rows)
#pragma unroll
          for (int b = 0; b < 4; ++b) tma_load_2d(xs + s * C::STAGE + b * 16384, &tmap, 32 * b, row0, &x_full[s]);
        } else {
          tma_load_2d(xs + s * C::STAGE, &tmap, 0, row0, &x_full[s]);
          tma_load_2d(xs + s * C::STAGE + 16384, &tmap, 64, row0, &x_full[s]);
        }
        issued = i + 1;
      }
      // Drain: the last copy into every stage and G buffer has landed before the
      // CTA can exit (immediate unless a wait above gave up).
      for (int s = 0; s < NST && s < issued; ++s) {
        const int last = ((issued - 1 - s) / NST) * NST + s;
        mbar_wait(&x_full[s], (uint32_t)(last / NST) & 1u, a.status);
      }
      for (int q = gq - 2 < 0 ? 0 : gq - 2; q < gq; ++q) mbar_wait(&g_full[q & 1], (uint32_t)(q >> 1) & 1u, a.status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int lsm = -1;
      int j = (int)(g0 % tiles) - 1;
      for (int i = 0; i < n_t && !*abort_flag; ++i) {  // after a wait gave up, nothing more is issued
        if (++j == tiles) j = 0;
        const int s = i % NST, ub = i & 1;
        if (i == 0 || j == 0) {
          ++lsm;
          // slice lsm's M (with a gauge, buffer lsm & 1; without, one M in buffer 0)
          if (a.has_g || i == 0) wait(&m_full[lsm & 1], (uint32_t)(a.has_g ? lsm >> 1 : 0) & 1u);
        }
        if constexpr (F32) wait(conv_full, (uint32_t)i & 1u);  // tile i's hi and lo tiles
        else wait(&x_full[s], (uint32_t)(i / NST) & 1u);
        wait(&u_empty[ub], ((uint32_t)(i >> 1) & 1u) ^ 1u);
        fence_after();
        const uint32_t d = tmem + kFColU1 + 128 * ub;
        const uint32_t mc = tmem + fwd_mcol(a.has_g ? lsm : 0);
        if constexpr (F32) {  // U1^T = M_hi x_hi + M_lo x_hi + M_hi x_lo
          const uint32_t ha = smem_u32(cvt), la = smem_u32(cvt + kXBytes);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t ko = (k >> 2) * 16384 + (k & 3) * 32;
            mma_ts(d, mc + 8 * k, kdesc(ha + ko), idesc(false), k > 0);
            mma_ts(d, mc + 64 + 8 * k, kdesc(ha + ko), idesc(false), 1);
            mma_ts(d, mc + 8 * k, kdesc(la + ko), idesc(false), 1);
          }
        } else {
          const uint32_t xa = smem_u32(xs + s * C::STAGE);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint64_t bd = kdesc(xa + (k >> 2) * 16384 + (k & 3) * 32);
            mma_ts(d, mc + 8 * k, bd, idesc(false), k > 0);
            mma_ts(d, mc + 64 + 8 * k, bd, idesc(false), 1);
          }
        }
        commit(&u_full[ub]);
        if constexpr (!F32) commit(&x_empty[s]);
        if (a.has_g && (j == tiles - 1 || i == n_t - 1)) commit(&m_empty[lsm & 1]);
      }
      commit(mma_done);
      mbar_wait(mma_done, 0u, a.status);
    }
  } else {
    // worker warp: lane quarter wq (tensor-memory lanes 32 wq ..), token part hf of the tile
    const int wq = warp & 3, hf = (warp - 2) >> 2;
    const int v = 32 * wq + lane;
    const uint32_t lrow = (uint32_t)(32 * wq) << 16;
    const float inv_tau = 1.0f / a.tau;
    float2 rad2[16];
    {
      const float rv = (float)v / (kD - 1);
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const float ru = (float)u / 15.0f;
        rad2[u] = dup2(sqrtf(ru * ru + rv * rv) * 0.70710678118654752f);
      }
    }
    // M of the q-th slice of this CTA's range into buffer q & 1, once that buffer's
    // previous slice (q - 2) has had all its GEMMs
    auto build_m = [&](int q) {
      if (a.has_g) wait(&g_full[q & 1], (uint32_t)(q >> 1) & 1u);
      if (q >= 2) wait(&m_empty[q & 1], (uint32_t)((q - 2) >> 1) & 1u);
      __syncwarp();
      fence_after();
      const float* G = gs + (q & 1) * 2048;
      const uint32_t mc = tmem + lrow + fwd_mcol(q);
#pragma unroll 1
      for (int r4 = 0; r4 < 8 / PARTS; ++r4) {  // channel groups 16 r .. 16 r + 15 of this part
        const int r = (8 / PARTS) * hf + r4;
        uint32_t h8[8], l8[8];
        m_group(cosk, G, a.has_g, v, r, h8, l8);
        st8(mc + 8 * r, h8);
        st8(mc + 64 + 8 * r, l8);
      }
      wait_st();
      fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&m_full[q & 1]);
        if (a.has_g) mbar_arrive(&g_empty[q & 1]);
      }
    };
    // fp32 input: split tile ti (its stage of the ring) into the bf16 hi and lo tiles the
    // GEMM reads, in the same swizzled K-major layout as a bf16 TMA tile.  Worker wid takes
    // row wid / 2, channels 64 (wid & 1) .. + 63: 16 fp32 chunks of 16 bytes (chunk c of a
    // 32-channel box at position c ^ (row & 7)) become 8 bf16 chunks in each tile.
    auto split_tile = [&](int ti) {
      const int s = ti % NST;
      wait(&x_full[s], (uint32_t)(ti / NST) & 1u);
      const int wid = threadIdx.x - 64, r = wid >> 1, hh = wid & 1;
      const unsigned char* src = xs + s * C::STAGE + r * 128;
      unsigned char* hi_t = cvt + hh * 16384 + r * 128;
      unsigned char* lo_t = hi_t + kXBytes;
#pragma unroll
      for (int q = 0; q < 8; ++q) {  // bf16 chunk q: channels 64 hh + 8 q .. + 7
        const int b = 2 * hh + (q >> 2), c0 = 2 * (q & 3);  // fp32 box, first 4-channel chunk in it
        const float4 f0 = *reinterpret_cast<const float4*>(src + b * 16384 + ((c0 ^ (r & 7)) << 4));
        const float4 f1 = *reinterpret_cast<const float4*>(src + b * 16384 + (((c0 + 1) ^ (r & 7)) << 4));
        uint4 h, l;
        split2(f0.x, f0.y, h.x, l.x);
        split2(f0.z, f0.w, h.y, l.y);
        split2(f1.x, f1.y, h.z, l.z);
        split2(f1.z, f1.w, h.w, l.w);
        const int o = (q ^ (r & 7)) << 4;
        *reinterpret_cast<uint4*>(hi_t + o) = h;
        *reinterpret_cast<uint4*>(lo_t + o) = l;
      }
      fence_proxy_async_smem();  // the tiles are read by the tensor cores
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(conv_full);
        mbar_arrive(&x_empty[s]);
      }
    };
    if (n_t > 0) build_m(0);
    if constexpr (F32) {
      if (n_t > 0) split_tile(0);
    }
    int ls = 0;
    int j = (int)(g0 % tiles) - 1;  // tile index within its slice, advanced per tile (no division)
    int j0 = j + 1;                 // the slice's first tile in this CTA's range
    for (int i = 0; i < n_t; ++i) {
      const long long gt = g0 + i;
      if (++j == tiles) j = 0;
      const int ub = i & 1;
      if (i > 0 && j == 0) {
        ++ls;
        j0 = 0;
      }
      // This warp's rows of the next slice's M, before this tile's statistics.  The
      // token parts take their turns over the slice's last PARTS tiles, so that while
      // one warp per SMSP builds, the other warps keep the arithmetic pipes busy.
      if (a.has_g && i + (tiles - j) < n_t && j == max(tiles - 1 - hf, j0)) build_m(ls + 1);
      wait(&u_full[ub], (uint32_t)(i >> 1) & 1u);
      __syncwarp();
      fence_after();
      float x[TPP];
#pragma unroll
      for (int c = 0; c < TPP / 32; ++c) ld32(tmem + lrow + kFColU1 + 128 * ub + TPP * hf + 32 * c, x + 32 * c);
      wait_ld();
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&u_empty[ub]);
      // fp32 input: tile i's GEMM is done with the hi and lo tiles, so tile i + 1 is split
      // now and its GEMM overlaps this tile's statistics
      if constexpr (F32) {
        if (i + 1 < n_t) split_tile(i + 1);
      }
      float part[3 * BPP];  // per block kb of the part: E, F, R at 3 kb
#pragma unroll
      for (int p = 0; p < BPP / 2; ++p) {  // blocks 2 p and 2 p + 1 as fp32 pairs
        float2 U[16], E, F, R;
        dct16_pair(x + 32 * p, x + 32 * p + 16, U);
        pair_sums(U, rad2, inv_tau, E, F, R);
        part[6 * p] = E.x;
        part[6 * p + 1] = F.x;
        part[6 * p + 2] = R.x;
        part[6 * p + 3] = E.y;
        part[6 * p + 4] = F.y;
        part[6 * p + 5] = R.y;
      }
      if constexpr (F32) {  // the halving butterfly, then the quarters' sums
        static_assert(!F32 || BPP == 4, "the fp32 input's reduction takes 4 blocks per part");
        const float tot = warp_sum12(part, lane);
        float* rb = red + ((i & 1) * 2 + hf) * 48;
        if (!(lane & 1) && (lane >> 1) < 12) rb[wq * 12 + (lane >> 1)] = tot;
        named_bar_sync(2 + hf, 128);
        if (wq == 0 && lane < 4) {
          const int kb = lane;
          const float E = (rb[0 * 12 + 3 * kb] + rb[1 * 12 + 3 * kb]) + (rb[2 * 12 + 3 * kb] + rb[3 * 12 + 3 * kb]);
          const float F = (rb[0 * 12 + 3 * kb + 1] + rb[1 * 12 + 3 * kb + 1]) + (rb[2 * 12 + 3 * kb + 1] + rb[3 * 12 + 3 * kb + 1]);
          const float R = (rb[0 * 12 + 3 * kb + 2] + rb[1 * 12 + 3 * kb + 2]) + (rb[2 * 12 + 3 * kb + 2] + rb[3 * 12 + 3 * kb + 2]);
          const long long blk = gt * 8 + 4 * hf + kb;
          a.lfreq[blk] = E > 0.0f ? F / E : 0.0f;
          a.lrate[blk] = R * 0.69314718055994531f / (16.0f * kD);
        }
      } else {
        float* rb = red + ((i & 1) * PARTS + hf) * (3 * BPP * kRedPitch);
#pragma unroll
        for (int q = 0; q < 3 * BPP; ++q) rb[q * kRedPitch + v] = part[q];
        named_bar_sync(2 + hf, 128);
        // One warp per part finishes the sums, the parts' reducers on different SMSPs
        // (quarter 2 + hf mod 4): LPB lanes per block, lane LPB kb + s adding the CPL
        // channel frequencies v = CPL s .. CPL s + CPL - 1 of block kb.
        if (wq == ((2 + hf) & 3)) {
          constexpr int LPB = 32 / BPP, CPL = kD / LPB;
          const int kb = lane / LPB, sx = lane % LPB;
          float acc[3];
#pragma unroll
          for (int c = 0; c < 3; ++c) {
            const float4* src = reinterpret_cast<const float4*>(rb + (3 * kb + c) * kRedPitch + CPL * sx);
            float4 q4[CPL / 4];
#pragma unroll
            for (int w = 0; w < CPL / 4; ++w) q4[w] = src[w];
            float s4[CPL / 4];
#pragma unroll
            for (int w = 0; w < CPL / 4; ++w) s4[w] = (q4[w].x + q4[w].y) + (q4[w].z + q4[w].w);
#pragma unroll
            for (int w2 = 1; w2 < CPL / 4; w2 <<= 1)
#pragma unroll
              for (int w = 0; w < CPL / 4; w += 2 * w2) s4[w] += s4[w + w2];
            acc[c] = s4[0];
#pragma unroll
            for (int o = 1; o < LPB; o <<= 1) acc[c] += __shfl_xor_sync(0xffffffffu, acc[c], o);
          }
          if (sx == 0) {
            const long long blk = gt * 8 + BPP * hf + kb;
            a.lfreq[blk] = acc[0] > 0.0f ? acc[1] / acc[0] : 0.0f;
            a.lrate[blk] = acc[2] * 0.69314718055994531f / (16.0f * kD);
          }
        }
      }
    }
  }
  fence_before();
  __syncthreads();
  if (warp == 1) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

bool spectral_tmem_supported(const KvGeom& k, int x_fp32) { return !x_fp32 && k.d == kD && k.T % kTile == 0; }
bool spectral_fwd_f32_supported(const KvGeom& k) { return k.d == kD && k.T % kTile == 0; }
int spectral_tmem_pieces(const KvGeom& k) { return (k.d == kD && k.T % (2 * kTile) == 0) ? 2 : 1; }

cudaError_t launch_spectral_tmem(const KvGeom& k, int x_fp32, const void* x, const float* G, float lambda_f,
                                 float lambda_r, float tau, float* lfreq, float* lrate, float* dg_part,
                                 unsigned int* status, int num_sms, cudaStream_t st) {
  if (x_fp32 && dg_part) return cudaErrorInvalidValue;  // fp32 input: statistics only
  alignas(64) CUtensorMap tmap;
  const uint64_t rows = (uint64_t)k.slices() * k.T;
  if (x_fp32 ? !make_tmap_2d_f32(&tmap, x, rows, kD, 32, kTile) : !make_tmap_2d_bf16(&tmap, x, rows, kD, 64, kTile))
    return cudaErrorInvalidValue;
  TmArgs a;
  a.k = k;
  a.has_g = G != nullptr;
  a.want_grad = dg_part != nullptr;
  a.lambda_f = lambda_f;
  a.lambda_r = lambda_r;
  a.tau = tau;
  const double nblk = (double)k.slices() * (k.T / 16);
  a.inv_nblk = 1.0 / nblk;
  a.inv_ncoef = 1.0 / (nblk * 16.0 * kD);
  a.G = G;
  a.lfreq = lfreq;
  a.lrate = lrate;
  a.dg_part = dg_part;
  a.status = status;
  if (dg_part == nullptr) {  // statistics only: tile-balanced ranges
    auto kern = x_fp32 ? spectral_fwd_kernel<true> : spectral_fwd_kernel<false>;
    const int smem = x_fp32 ? FwdCfg<true>::SMEM : FwdCfg<false>::SMEM;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const long long tiles = k.slices() * (k.T / kTile);
    const int grid = (int)(tiles < num_sms ? tiles : num_sms);
    kern<<<grid, x_fp32 ? FwdCfg<true>::THREADS : FwdCfg<false>::THREADS, smem, st>>>(tmap, a);
    return cudaGetLastError();
  }
  a.pieces = spectral_tmem_pieces(k);
  cudaError_t e = cudaFuncSetAttribute(spectral_tmem_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  const long long units = k.slices() * a.pieces;
  const int grid = (int)(units < num_sms ? units : num_sms);
  spectral_tmem_kernel<<<grid, kThreads, kSmem, st>>>(tmap, a);
  return cudaGetLastError();
}

}  // namespace cg
