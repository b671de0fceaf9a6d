// Fused gauge + block-uniform quantize + pack for g = 16 and d_head = 128 on
// the 5th-generation tensor cores, with codes identical to the exact encoder.
//
// Codec-Gauge, Method: explicit gauge application costs O(N_KV g) multiply-
// adds (16 per value here); Experimental setup: block-uniform backend with one
// range per 16 tokens x 16 channels.
//
// The codec defines the gauged value the quantizer sees as the fp32 FMA chain
//   acc = +0;  acc = fl32(G[i][j] x[j] + acc) for j = 0..15;  y_i = acc,
// and that chain costs 16 FP32-pipe operations per value, more than the HBM
// time of the whole codec at full clock.  Here the contraction runs on the
// tensor cores instead and the chain is evaluated only where it can change a
// decision:
//   * G (fp32) is split exactly into three bf16 terms hi + mid + lo (each
//     residual of an RNE rounding has at most 8 significant bits left), so
//     with x in bf16 every product is exact and the tensor-core sum
//     y_tc = sum_j x_j (hi + mid + lo)_ij differs from the exact dot product
//     only by accumulation rounding;
//   * an a-priori bound A = kA * max_rows |y_tc row|_2 over the block bounds
//     |y_tc - y| for every value of a 16 x 16 block, where y is the fp32 chain:
//       |y - x.G_i| <= 16 u sum_j |G_ij x_j|   (chain, u = 2^-24),
//       |y_tc - x.G_i| <= E sum_j |G_ij x_j|   (tensor-core accumulation,
//                                                E = 2^-20 assumed),
//       sum_j |G_ij x_j| <= |G_i|_2 |x|_2 <= |x.G|_2 (1 + 16 e)
//     for a gauge whose rows are orthonormal to e (checked per head slice
//     while G is staged; a gauge that is not orthogonal to 2^-12 gets A = inf,
//     i.e. every value is evaluated exactly);
//   * the zero point z = fp16(min) and step s = fp16(fl(fl(max - min)/qmax))
//     are decided when both ends of [min - A, min + A] (and of the range
//     interval) round to the same fp16 values.  Otherwise the block's min and
//     max are made exact: every value within 2A of the tensor-core minimum
//     (maximum) is re-evaluated with the chain (the exact extreme is always
//     among them) and the range reduced again;
//   * a code is decided when t = fl(fl(y_tc - z) / s) is further than
//     delta = (A + 2^-21 Q)/s (1 + 2^-18) from the nearest rounding boundary
//     k + 1/2, which bounds |t_tc - t_exact|; the few values within delta are
//     re-evaluated with the chain and quantized again.
// So codes, steps and zero points equal the exact encoder's bit for bit, as long as
// the assumed E holds; every value the chain re-evaluates is checked against A, and
// a value outside it ORs kStatusBound into the device status word (reported by
// cg_sync_status as CG_ERR_BOUND), so a violation on real data does not pass
// silently.  The
// optional fp32 gauged output holds the values actually quantized (y_tc, with
// the chain's value wherever it was evaluated), within A of the chain.
//
// Structure (persistent, one CTA per SM, contiguous ranges of 128-token
// blocks in (layer, K/V, batch, head, token) order):
//   * warp 0 streams x blocks (128 x 128 bf16 = 32 KB as two 16 KB TMA boxes,
//     128-byte swizzle, no multicast) into a 5-stage ring, and stages each
//     head slice's G: the fp32 copy for the chain and the three bf16 terms in
//     the swizzled K-major layout of the B operand (released to the MMA
//     warp), then the orthogonality check (released to the epilogue); two
//     buffers, so the next slice's G is staged while the current one is used;
//   * warp 1 issues 24 tcgen05.mma per block (8 groups x 3 terms, M = 128,
//     N = 16, K = 16, bf16 x bf16 -> fp32) into one of four 128-column TMEM
//     accumulators (group r writes columns 16r .. 16r+15);
//   * warps 2..13 are three epilogue warpgroups taking blocks in turn (thread
//     = token row): tcgen05.ld, per-group row ranges, a transposing half-warp
//     reduction that leaves block (tile, r) on lanes 2r, 2r+1 of the tile's
//     half-warp, which compute its parameters once; then quantize, check,
//     pack and store; the chain, where needed, reads x from global memory
//     (the x stage is released as soon as the tensor cores have read it).
// Every wait on an mbarrier is bounded in time.
#include <cuda.h>

#include "cg_kernels.cuh"

namespace cg {

namespace {

constexpr int D = 128;
constexpr int kXStages = 5;
constexpr int kXBytes = 128 * D * 2;       // one 128-token block of bf16
constexpr int kBBytes = 6 * 2048;          // bf16 terms: 6 swizzled regions of 16 rows x 128 B
constexpr int kGBytes = 8 * 16 * 16 * 4;   // fp32 G of one head slice
constexpr int kEpiGroups = 3;              // epilogue warpgroups, taking blocks in turn
constexpr int kEpiWarps = 4 * kEpiGroups;
constexpr int kThreads = (kEpiWarps + 2) * 32;
constexpr int kTmemCols = 512;             // four 128-column fp32 accumulators
constexpr float kMagic = 12582912.0f;      // 1.5 * 2^23: adding it rounds to an integer (RNE)
// tcgen05 instruction descriptor: D fp32, A and B bf16, both K-major, N = 16, M = 128
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((16u >> 3) << 17) | ((128u >> 4) << 24);
// |y_tc - y_chain| <= kA0 (1 + 16 e) |y_tc row|_2 for every value of a row of a
// group: (E + 16 u) with E = 2^-20 and u = 2^-24, times 1.001 for the second-
// order terms and the fp32 evaluation of the row norm.  (Measured against an
// fp64 reference on 10^8 values: max |y_tc - x.G_i| / sum_j |G_ij x_j| is
// 2^-22.0, the chain's 2^-21.1, and max |y_tc - y_chain| / |y_tc row|_2 is
// 2^-21.2.)
constexpr float kA0 = (0x1p-20f + 0x1p-20f) * 1.001f;
constexpr float kOrthoMax = 0x1p-12f;

__device__ __forceinline__ uint64_t sw128_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr & 0x3FFFFu) >> 4);  // start address
  d |= (uint64_t)1 << 16;                         // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;               // stride byte offset: 1024 B between 8-row groups
  d |= (uint64_t)1 << 46;                         // descriptor version
  d |= (uint64_t)2 << 61;                         // layout: 128-byte swizzle
  return d;
}
__device__ __forceinline__ void umma_bf16_n16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
          tmem_d),
      "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate));
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
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
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// Mark v as written here, so that no use of v can be scheduled before this
// point (a TMEM load writes its registers asynchronously, until the wait).
__device__ __forceinline__ void reg_fence16(float* v) {
  asm volatile(""
               : "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]), "+f"(v[6]), "+f"(v[7]),
                 "+f"(v[8]), "+f"(v[9]), "+f"(v[10]), "+f"(v[11]), "+f"(v[12]), "+f"(v[13]), "+f"(v[14]), "+f"(v[15]));
}
// Wait for this thread's TMEM loads; the n floats at v (n = 16 or 32) were
// their destination.
template <int N>
__device__ __forceinline__ void tmem_wait_ld_into(float* v) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  reg_fence16(v);
  if constexpr (N == 32) reg_fence16(v + 16);
}

__device__ __forceinline__ float min3f(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ void minmax16(const float* y, float& mn, float& mx) {
  mn = min3f(min3f(min3f(y[0], y[1], y[2]), min3f(y[3], y[4], y[5]), min3f(y[6], y[7], y[8])),
             min3f(y[9], y[10], y[11]), min3f(y[12], y[13], fminf(y[14], y[15])));
  mx = max3f(max3f(max3f(y[0], y[1], y[2]), max3f(y[3], y[4], y[5]), max3f(y[6], y[7], y[8])),
             max3f(y[9], y[10], y[11]), max3f(y[12], y[13], fmaxf(y[14], y[15])));
}

// Row statistics of one group: min, max and the squared norm sum_k y_k^2.
__device__ __forceinline__ void stats16(const float* y, float& mn, float& mx, float& ss) {
  minmax16(y, mn, mx);
  f2_t acc = f2_make(0.0f, 0.0f);
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const f2_t p = f2_make(y[2 * m], y[2 * m + 1]);
    acc = f2_fma(p, p, acc);
  }
  float lo, hi;
  f2_split(acc, lo, hi);
  ss = lo + hi;
}

// fp16 bits of the zero point and step the quantizer would derive from a range
// end / width (the same operations as quant_params, monotone in the argument).
__device__ __forceinline__ uint16_t z_bits(float mn) {
  mn = __fadd_rn(mn, 0.0f);  // a zero minimum is +0
  return __half_as_ushort(__float2half_rn(fminf(fmaxf(mn, -65504.0f), 65504.0f)));
}
// The step from a range width: fp16(min(fl32(rng / qmax), 65504)).  The fp32
// quotient is q0 = fl(rng c), c = fl(1/qmax), corrected once with the exact
// residual fma(-q0, qmax, rng): for qmax = 3, 7, 15, 63 and 255 this equals the
// correctly rounded rng / qmax for every fp32 rng (checked exhaustively over
// all 2^31 non-negative values, and odd-symmetric).
template <int QMAX>
__device__ __forceinline__ uint16_t s_bits(float rng) {
  constexpr float c = (float)(1.0 / QMAX);
  const float q0 = __fmul_rn(rng, c);
  const float q = __fmaf_rn(__fmaf_rn(-q0, (float)QMAX, rng), c, q0);
  return __half_as_ushort(__float2half_rn(fminf(q, 65504.0f)));
}

// The exact gauged value: output i of group r of the token whose 128 bf16
// channels start at xrow, as the fp32 FMA chain in index order from +0.  (x
// comes from global memory, most likely L2: the shared-memory copy of the
// block is released as soon as the tensor cores have read it.)
__device__ __forceinline__ float chain_y(const uint16_t* xrow, const float* gf, int r, int i) {
  const uint4 c0 = __ldg(reinterpret_cast<const uint4*>(xrow + 16 * r));
  const uint4 c1 = __ldg(reinterpret_cast<const uint4*>(xrow + 16 * r + 8));
  const float4* g = reinterpret_cast<const float4*>(gf + (16 * r + i) * 16);
  const float4 g0 = g[0], g1 = g[1], g2 = g[2], g3 = g[3];
  float acc = 0.0f;
  acc = __fmaf_rn(g0.x, bf16lo(c0.x), acc);
  acc = __fmaf_rn(g0.y, bf16hi(c0.x), acc);
  acc = __fmaf_rn(g0.z, bf16lo(c0.y), acc);
  acc = __fmaf_rn(g0.w, bf16hi(c0.y), acc);
  acc = __fmaf_rn(g1.x, bf16lo(c0.z), acc);
  acc = __fmaf_rn(g1.y, bf16hi(c0.z), acc);
  acc = __fmaf_rn(g1.z, bf16lo(c0.w), acc);
  acc = __fmaf_rn(g1.w, bf16hi(c0.w), acc);
  acc = __fmaf_rn(g2.x, bf16lo(c1.x), acc);
  acc = __fmaf_rn(g2.y, bf16hi(c1.x), acc);
  acc = __fmaf_rn(g2.z, bf16lo(c1.y), acc);
  acc = __fmaf_rn(g2.w, bf16hi(c1.y), acc);
  acc = __fmaf_rn(g3.x, bf16lo(c1.z), acc);
  acc = __fmaf_rn(g3.y, bf16hi(c1.z), acc);
  acc = __fmaf_rn(g3.z, bf16lo(c1.w), acc);
  acc = __fmaf_rn(g3.w, bf16hi(c1.w), acc);
  return acc;
}

// Pack 16 codes, given as bit patterns whose low byte is the code, into the
// 16 * BITS-bit little-endian row chunk and store it (dst aligned to the
// chunk's natural alignment: 2 B for 3 bits, 4 B for 2 and 6, 8 B for 4, 16 B for 8).
template <int BITS>
__device__ __forceinline__ void store_row16(uint8_t* dst, const uint32_t (&rb)[16]) {
  if constexpr (BITS == 4) {
    uint32_t w[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {  // even codes' bytes, odd codes' bytes, then nibbles
      const uint32_t* q = rb + 8 * h;
      const uint32_t ev = __byte_perm(__byte_perm(q[0], q[2], 0x0040), __byte_perm(q[4], q[6], 0x0040), 0x5410);
      const uint32_t od = __byte_perm(__byte_perm(q[1], q[3], 0x0040), __byte_perm(q[5], q[7], 0x0040), 0x5410);
      w[h] = (ev & 0x0F0F0F0Fu) | ((od << 4) & 0xF0F0F0F0u);
    }
    *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
  } else if constexpr (BITS == 8) {
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      w[k] = __byte_perm(__byte_perm(rb[4 * k], rb[4 * k + 1], 0x0040), __byte_perm(rb[4 * k + 2], rb[4 * k + 3], 0x0040),
                         0x5410);
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  } else if constexpr (BITS == 2) {
    uint32_t w = 0;
#pragma unroll
    for (int k = 0; k < 16; ++k) w |= (rb[k] & 3u) << (2 * k);
    *reinterpret_cast<uint32_t*>(dst) = w;
  } else if constexpr (BITS == 3) {
    uint64_t c = 0;
#pragma unroll
    for (int k = 0; k < 16; ++k) c |= (uint64_t)(rb[k] & 7u) << (3 * k);
    uint16_t* p = reinterpret_cast<uint16_t*>(dst);
    p[0] = (uint16_t)c;
    p[1] = (uint16_t)(c >> 16);
    p[2] = (uint16_t)(c >> 32);
  } else {  // 6 bits: 96 bits
    uint32_t w[3] = {0u, 0u, 0u};
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const uint32_t q = rb[k] & 63u;
      const int bit = 6 * k;
      w[bit >> 5] |= q << (bit & 31);
      if ((bit & 31) > 26) w[(bit >> 5) + 1] |= q >> (32 - (bit & 31));
    }
    uint32_t* p = reinterpret_cast<uint32_t*>(dst);
    p[0] = w[0];
    p[1] = w[1];
    p[2] = w[2];
  }
}

// Codes of one row of a group: rb[k] = bits of rne(t_k) + 1.5 * 2^23 (low byte
// = the code) with t = fma(y, inv, fl(-z inv)) (within 2^-22 (|y| + |z|) inv of
// fl(fl(y - z) * inv), which the decision margin covers), clamped to [0, qmax]
// when CLAMP.  Returns max_k |t_k - rne(t_k)| (exact: Fast2Sum against the
// magic number).
template <bool CLAMP, int QMAX>
__device__ __forceinline__ float quant16(const float (&y)[16], float zf, float inv, uint32_t (&rb)[16]) {
  const float nzi = -zf * inv;
  const f2_t nzi2 = f2_make(nzi, nzi), inv2 = f2_make(inv, inv);
  const f2_t mg2 = f2_make(kMagic, kMagic), nmg2 = f2_make(-kMagic, -kMagic), m1 = f2_make(-1.0f, -1.0f);
  float fmx = 0.0f;
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    f2_t t2 = f2_fma(f2_make(y[2 * m], y[2 * m + 1]), inv2, nzi2);
    if constexpr (CLAMP) {
      float lo, hi;
      f2_split(t2, lo, hi);
      t2 = f2_make(fminf(fmaxf(lo, 0.0f), (float)QMAX), fminf(fmaxf(hi, 0.0f), (float)QMAX));
    }
    const f2_t r2 = f2_add(t2, mg2);
    const f2_t fr2 = f2_fma(f2_add(r2, nmg2), m1, t2);  // t - rne(t)
    float flo, fhi, rlo, rhi;
    f2_split(fr2, flo, fhi);
    f2_split(r2, rlo, rhi);
    rb[2 * m] = __float_as_uint(rlo);
    rb[2 * m + 1] = __float_as_uint(rhi);
    fmx = max3f(fmx, fabsf(flo), fabsf(fhi));
  }
  return fmx;
}

// Exact range of the undecided blocks of a warp (bit lane 2r + 16 h of `und`:
// block (tile h, group r)): every value within 2A of a block's tensor-core
// minimum (maximum) is re-evaluated with the chain (the exact extreme is among
// them, since no other value can lie below min_tc + A), then the block range
// is reduced again.  Returns this lane's (mn, mx), exact where its block was
// undecided.  Called by the whole warp; out of line, as it is rarely needed.
__device__ __noinline__ float2 exact_range(const uint16_t* xrow, const float* gf, uint32_t taddr, uint32_t und,
                                           float mn, float mx, float A, unsigned int* status) {
  const unsigned FULL = 0xffffffffu;
  const int lane = threadIdx.x & 31, r_own = (lane & 15) >> 1;
  uint32_t gm = 0;
  for (uint32_t m = und; m; m &= m - 1) gm |= 1u << (((__ffs(m) - 1) & 15) >> 1);
  while (gm) {
    const int r = __ffs(gm) - 1;
    gm &= gm - 1;
    const int src = (lane & 16) + 2 * r;
    const float bmn = __shfl_sync(FULL, mn, src), bmx = __shfl_sync(FULL, mx, src);
    const float bA = __shfl_sync(FULL, A, src);
    const bool bund = (und >> src) & 1u;
    float y[16];
    tmem_ld16(taddr + 16 * r, y);
    tmem_wait_ld();
    float lo_t = __int_as_float(0xff800000), hi_t = __int_as_float(0x7f800000);
    if (bund) {
      lo_t = __fadd_ru(bmn, __fmul_ru(2.0f, bA));
      hi_t = __fsub_rd(bmx, __fmul_ru(2.0f, bA));
    }
    uint32_t cand = 0;
#pragma unroll
    for (int k = 0; k < 16; ++k) cand |= (y[k] <= lo_t || y[k] >= hi_t) ? (1u << k) : 0u;
    while (__any_sync(FULL, cand != 0)) {
      if (cand) {
        const int k0 = __ffs(cand) - 1;
        cand &= cand - 1;
        const float e = chain_y(xrow, gf, r, k0);
#pragma unroll
        for (int k = 0; k < 16; ++k)
          if (k == k0) {
            if (!(fabsf(y[k] - e) <= bA)) atomicOr(status, kStatusBound);  // the assumed bound failed
            y[k] = e;
          }
      }
    }
    float emn, emx;
    minmax16(y, emn, emx);
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) {
      emn = fminf(emn, __shfl_xor_sync(FULL, emn, o));
      emx = fmaxf(emx, __shfl_xor_sync(FULL, emx, o));
    }
    if (bund && r_own == r) {
      mn = emn;
      mx = emx;
    }
  }
  return make_float2(mn, mx);
}

// One row of a group on the slow path: quantize with clamping where the block
// needs it (th < -2 carries that, with the margin shifted by -4), re-evaluate
// the chain for every value within the margin of a rounding boundary, pack and
// store.  Reloads the group's accumulator columns.  Called by the whole warp;
// out of line, as it is rarely needed.
template <int BITS>
__device__ __noinline__ void slow_group(const uint16_t* xrow, const float* gf, uint32_t taddr_r, int r, float zf,
                                        float inv, float th, float A, bool tile_ok, uint8_t* crow_r, float* grow,
                                        unsigned int* status) {
  constexpr int QMAX = (1 << BITS) - 1;
  const unsigned FULL = 0xffffffffu;
  float y[16];
  tmem_ld16(taddr_r, y);
  tmem_wait_ld();
  const bool clamp = th < -2.0f;
  if (clamp) th += 4.0f;
  const float nzi = -zf * inv;  // as in quant16
  uint32_t rb[16];
  uint32_t pend = 0;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    float t = __fmaf_rn(y[k], inv, nzi);
    if (clamp) t = fminf(fmaxf(t, 0.0f), (float)QMAX);
    const float rr = __fadd_rn(t, kMagic);
    rb[k] = __float_as_uint(rr);
    if (tile_ok && fabsf(__fsub_rn(t, __fsub_rn(rr, kMagic))) >= th) pend |= 1u << k;
  }
  while (__any_sync(FULL, pend != 0)) {
    if (pend) {
      const int k0 = __ffs(pend) - 1;
      pend &= pend - 1;
      const float e = chain_y(xrow, gf, r, k0);
      float t = __fmul_rn(__fsub_rn(e, zf), inv);
      t = fminf(fmaxf(t, 0.0f), (float)QMAX);
      const uint32_t rr = __float_as_uint(__fadd_rn(t, kMagic));
#pragma unroll
      for (int k = 0; k < 16; ++k)
        if (k == k0) {
          if (!(fabsf(y[k] - e) <= A)) atomicOr(status, kStatusBound);  // the assumed bound failed
          rb[k] = rr;
          y[k] = e;
        }
    }
  }
  if (tile_ok) {
    store_row16<BITS>(crow_r, rb);
    if (grow) {
#pragma unroll
      for (int k = 0; k < 4; ++k)
        reinterpret_cast<float4*>(grow)[k] = make_float4(y[4 * k], y[4 * k + 1], y[4 * k + 2], y[4 * k + 3]);
    }
  }
}

struct TcSmem {
  unsigned char* xs;  // kXStages x 32 KB, 1024-aligned
  unsigned char* bs;  // 2 x 12 KB bf16 terms, 1024-aligned
  float* gf;          // 2 x 2048 fp32 G
  float* ka;          // 2: error-bound factor of the staged slice
  uint64_t* x_full;
  uint64_t* x_empty;
  uint64_t* g_full;
  uint64_t* g_empty;
  uint64_t* k_full;
  uint64_t* t_full;
  uint64_t* t_empty;
  uint32_t* tmem_base;
};
__device__ inline TcSmem tc_carve(unsigned char* raw) {
  TcSmem s;
  unsigned char* base = reinterpret_cast<unsigned char*>(((uintptr_t)raw + 1023) & ~(uintptr_t)1023);
  s.xs = base;
  s.bs = base + kXStages * kXBytes;
  s.gf = reinterpret_cast<float*>(s.bs + 2 * kBBytes);
  s.ka = s.gf + 2 * 2048;
  uint64_t* bars = reinterpret_cast<uint64_t*>(s.ka + 4);
  s.x_full = bars;
  s.x_empty = bars + kXStages;
  s.g_full = bars + 2 * kXStages;
  s.g_empty = s.g_full + 2;
  s.k_full = s.g_empty + 2;
  s.t_full = s.k_full + 2;
  s.t_empty = s.t_full + 4;
  s.tmem_base = reinterpret_cast<uint32_t*>(s.t_empty + 4);
  return s;
}
constexpr int kTcSmem = 1024 + kXStages * kXBytes + 2 * kBBytes + 2 * kGBytes + 16 + (2 * kXStages + 14) * 8 + 16;

// bf16 term k (0 = hi, 1 = mid, 2 = lo) of G_r lives in region 2k + (r >> 2),
// 32-byte column chunk r & 3 of its 128-byte rows (row n = output channel).
__device__ __forceinline__ uint32_t b_offset(int k, int r, int n, int j) {
  const int chunk = 2 * (r & 3) + (j >> 3);
  return (2 * k + (r >> 2)) * 2048 + n * 128 + ((chunk ^ (n & 7)) << 4) + (j & 7) * 2;
}

__device__ __forceinline__ uint16_t bf16_rne_bits(float v) { return __bfloat16_as_ushort(__float2bfloat16_rn(v)); }

}  // namespace

template <int BITS>
__global__ void __launch_bounds__(512, 1)  // 448 threads; the bound caps registers at 128 (4 warps per scheduler)
    encode_tc16_kernel(const __grid_constant__ CUtensorMap tmap, CodecArgs a) {
  constexpr int QMAX = (1 << BITS) - 1;
  extern __shared__ unsigned char smem_raw[];
  const TcSmem sm = tc_carve(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bps = (a.nt + 127) / 128;  // 128-token blocks per head slice
  const long long total = (long long)bps * a.k.slices();
  const long long b0 = total * blockIdx.x / gridDim.x;
  const long long b1 = total * (blockIdx.x + 1) / gridDim.x;
  const int n_blocks = (int)(b1 - b0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kXStages; ++s) {
      mbar_init(&sm.x_full[s], 1);
      mbar_init(&sm.x_empty[s], 1);  // released when the tensor cores have read the block
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.g_full[s], 1);
      mbar_init(&sm.g_empty[s], 1 + kEpiWarps);  // tensor cores done with B, every epilogue warp past the slice
      mbar_init(&sm.k_full[s], 1);
    }
    for (int s = 0; s < 4; ++s) {
      mbar_init(&sm.t_full[s], 1);
      mbar_init(&sm.t_empty[s], 4);
    }
    fence_mbar_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(sm.tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_base;

  if (warp == 0) {
    // ---------------- x blocks (TMA) + G staging ----------------
    long long slice = b0 / bps;
    int bq = (int)(b0 - slice * bps);
    int gcount = 0;
    for (int i = 0; i < n_blocks; ++i) {
      if (i == 0 || bq == 0) {
        const int gb = gcount & 1;
        mbar_wait(&sm.g_empty[gb], ((uint32_t)(gcount >> 1) & 1u) ^ 1u, a.status);
        int l, sk, b, h;
        slice_coords(slice, a.k, l, sk, b, h);
        const float4* Gp = reinterpret_cast<const float4*>(a.G + gauge_set(l, sk, h, a.k) * 8 * 256);
        float* gf = sm.gf + gb * 2048;
        unsigned char* bdst = sm.bs + gb * kBBytes;
#pragma unroll 1
        for (int k8 = 0; k8 < 16; k8 += 8) {
        float4 gv[8];  // half of the slice's G, all loads in flight at once
#pragma unroll
        for (int k = 0; k < 8; ++k) gv[k] = __ldg(Gp + lane + 32 * (k8 + k));
#pragma unroll
        for (int k = 0; k < 8; ++k) {  // float4 e: 4 consecutive entries of one row of one group
          const int e = lane + 32 * (k8 + k);
          const float4 v = gv[k];
          reinterpret_cast<float4*>(gf)[e] = v;
          const int r = e >> 6, n = (e >> 2) & 15, j0 = (e & 3) * 4;
          const float g[4] = {v.x, v.y, v.z, v.w};
          uint32_t t[3][2];
#pragma unroll
          for (int p = 0; p < 2; ++p) {
            uint32_t hb[2], mb[2], lb[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const float x = g[2 * p + q];
              const uint16_t hi = bf16_rne_bits(x);
              const float r1 = x - __uint_as_float((uint32_t)hi << 16);  // exact
              const uint16_t mid = bf16_rne_bits(r1);
              const float r2 = r1 - __uint_as_float((uint32_t)mid << 16);  // exact, 8 significant bits at most
              hb[q] = hi;
              mb[q] = mid;
              lb[q] = bf16_rne_bits(r2);
            }
            t[0][p] = hb[0] | (hb[1] << 16);
            t[1][p] = mb[0] | (mb[1] << 16);
            t[2][p] = lb[0] | (lb[1] << 16);
          }
#pragma unroll
          for (int k3 = 0; k3 < 3; ++k3)
            *reinterpret_cast<uint2*>(bdst + b_offset(k3, r, n, j0)) = make_uint2(t[k3][0], t[k3][1]);
        }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.g_full[gb]);  // B operand and fp32 copy ready
        // orthogonality of the staged rows, e = max |G_r G_r^T - I| over the 8
        // groups (lane: rows 4q .. 4q+3 of group r against all 16 rows); only
        // the epilogue needs it
        float emax = 0.0f;
        {
          const int r = lane >> 2, q = lane & 3;
#pragma unroll 1
          for (int i2 = 0; i2 < 4; i2 += 2) {
          float ar[2][16];
#pragma unroll
          for (int ii = 0; ii < 2; ++ii)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const float4 u = reinterpret_cast<const float4*>(gf + (16 * r + 4 * q + i2 + ii) * 16)[c];
              ar[ii][4 * c] = u.x;
              ar[ii][4 * c + 1] = u.y;
              ar[ii][4 * c + 2] = u.z;
              ar[ii][4 * c + 3] = u.w;
            }
#pragma unroll 1
          for (int kk = 0; kk < 16; ++kk) {
            float ck[16];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const float4 u = reinterpret_cast<const float4*>(gf + (16 * r + kk) * 16)[c];
              ck[4 * c] = u.x;
              ck[4 * c + 1] = u.y;
              ck[4 * c + 2] = u.z;
              ck[4 * c + 3] = u.w;
            }
#pragma unroll
            for (int ii = 0; ii < 2; ++ii) {
              float dsum = 0.0f;
#pragma unroll
              for (int jj = 0; jj < 16; ++jj) dsum = __fmaf_rn(ar[ii][jj], ck[jj], dsum);
              if (4 * q + i2 + ii == kk) dsum -= 1.0f;
              emax = fmaxf(emax, fabsf(dsum));
            }
          }
          }
        }
        const uint32_t eb = __reduce_max_sync(0xffffffffu, __float_as_uint(emax));  // non-negative: bits order as values
        if (lane == 0) {
          const float e = __uint_as_float(eb) + 0x1p-20f;  // plus the rounding of the check itself
          sm.ka[gb] = (e <= kOrthoMax) ? kA0 * (1.0f + 16.0f * e) : __int_as_float(0x7f800000);
          mbar_arrive(&sm.k_full[gb]);
        }
        ++gcount;
      }
      if (lane == 0) {
        const int s = i % kXStages;
        mbar_wait(&sm.x_empty[s], ((uint32_t)(i / kXStages) & 1u) ^ 1u, a.status);
        mbar_arrive_expect_tx(&sm.x_full[s], kXBytes);
        const int row0 = (int)(slice * a.k.T + a.t0 + 128LL * bq);
        tma_load_2d(sm.xs + s * kXBytes, &tmap, 0, row0, &sm.x_full[s]);
        tma_load_2d(sm.xs + s * kXBytes + 16384, &tmap, 64, row0, &sm.x_full[s]);
      }
      __syncwarp();
      if (++bq == bps) {
        bq = 0;
        ++slice;
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issue (one thread) ----------------
    if (lane == 0) {
      long long slice = b0 / bps;
      int bq = (int)(b0 - slice * bps);
      int gcount = 0;
      for (int i = 0; i < n_blocks; ++i) {
        const int gb = gcount & 1;
        if (i == 0 || bq == 0) mbar_wait(&sm.g_full[gb], (uint32_t)(gcount >> 1) & 1u, a.status);
        const int s = i % kXStages, buf = i & 3;
        mbar_wait(&sm.x_full[s], (uint32_t)(i / kXStages) & 1u, a.status);
        mbar_wait(&sm.t_empty[buf], ((uint32_t)(i >> 2) & 1u) ^ 1u, a.status);
        tc_fence_after();
        // descriptors of the stage's x block and of the slice's B terms; an
        // operand at byte offset o is the descriptor plus o / 16 (start-address field)
        const uint64_t xd = sw128_desc(smem_u32(sm.xs + s * kXBytes));
        const uint64_t bd = sw128_desc(smem_u32(sm.bs + gb * kBBytes));
        const uint32_t td = tmem + buf * 128;
        // lo, mid, hi (small terms first); consecutive MMAs write different groups'
        // accumulators, so they do not wait for one another
#pragma unroll
        for (int k = 2; k >= 0; --k) {
#pragma unroll
          for (int r = 0; r < 8; ++r)
            umma_bf16_n16(td + 16 * r, xd + (((r >> 2) * 16384 + (r & 3) * 32) >> 4),
                          bd + (((2 * k + (r >> 2)) * 2048 + (r & 3) * 32) >> 4), k == 2 ? 0u : 1u);
        }
        umma_commit(&sm.x_empty[s]);
        umma_commit(&sm.t_full[buf]);
        const bool last_of_slice = (bq + 1 == bps) || (i + 1 == n_blocks);
        if (last_of_slice) {
          umma_commit(&sm.g_empty[gb]);
          ++gcount;
        }
        if (++bq == bps) {
          bq = 0;
          ++slice;
        }
      }
    }
  } else {
    // ---------------- epilogue: three warpgroups, thread = token row ----------------
    const int wg = (warp - 2) >> 2;
    const int quarter = warp & 3;  // TMEM lanes this warp may read
    const int row = 32 * quarter + lane;
    const int j16 = lane & 15;
    const int r_own = j16 >> 1;  // group whose block parameters this lane computes
    const unsigned FULL = 0xffffffffu;
    const long long slice_code_bytes = (long long)a.k.T * D * BITS / 8;
    long long slice = b0 / bps;
    int bq = (int)(b0 - slice * bps);
    int gcount = 0;
    for (int i = 0; i < n_blocks; ++i) {
      const int gb = gcount & 1;
      if (i == 0 || bq == 0) mbar_wait(&sm.k_full[gb], (uint32_t)(gcount >> 1) & 1u, a.status);
      const bool last_of_slice = (bq + 1 == bps) || (i + 1 == n_blocks);
      if (i % kEpiGroups == wg) {
        const int buf = i & 3;
        mbar_wait(&sm.t_full[buf], (uint32_t)(i >> 2) & 1u, a.status);
        tc_fence_after();
        const float* gf = sm.gf + gb * 2048;
        const float kA = sm.ka[gb];
        const int valid = min(128, a.nt - 128 * bq);
        const bool tile_ok = row < valid;  // valid is a multiple of 16: whole half-warps agree
        const int tok = a.t0 + 128 * bq + row;
        // the token's input channels, for the chain (an address only: valid rows read it)
        const uint16_t* xrow = a.kv + (slice * a.k.T + (tile_ok ? tok : a.t0)) * D;
        const long long tile = slice * (a.k.T / 16) + tok / 16;
        const uint32_t taddr = tmem + buf * 128 + ((uint32_t)(32 * quarter) << 16);

        // ---- pass 1: row ranges of the 8 groups, then the block ranges ----
        float mnr[8], mxr[8], ssr[8];
        {
          float va[32], vb[32];  // two groups at a time; the next two load meanwhile
          tmem_ld32(taddr, va);
#pragma unroll
          for (int c = 0; c < 4; c += 2) {
            tmem_wait_ld_into<32>(va);
            tmem_ld32(taddr + 32 * (c + 1), vb);
            stats16(va, mnr[2 * c], mxr[2 * c], ssr[2 * c]);
            stats16(va + 16, mnr[2 * c + 1], mxr[2 * c + 1], ssr[2 * c + 1]);
            tmem_wait_ld_into<32>(vb);
            if (c + 2 < 4) tmem_ld32(taddr + 32 * (c + 2), va);
            stats16(vb, mnr[2 * c + 2], mxr[2 * c + 2], ssr[2 * c + 2]);
            stats16(vb + 16, mnr[2 * c + 3], mxr[2 * c + 3], ssr[2 * c + 3]);
          }
        }
        // transposing reduction over the 16 rows of a tile (min, max, and the
        // largest row norm): after it, lanes 2r and 2r+1 of each half-warp
        // hold block (tile, r)
        float mn, mx, ss;
        {
          const bool up8 = j16 & 8, up4 = j16 & 4, up2 = j16 & 2;
          float n4[4], x4[4], q4[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float sn = up8 ? mnr[k] : mnr[k + 4], kn = up8 ? mnr[k + 4] : mnr[k];
            const float sx = up8 ? mxr[k] : mxr[k + 4], kx = up8 ? mxr[k + 4] : mxr[k];
            const float sq = up8 ? ssr[k] : ssr[k + 4], kq = up8 ? ssr[k + 4] : ssr[k];
            n4[k] = fminf(kn, __shfl_xor_sync(FULL, sn, 8));
            x4[k] = fmaxf(kx, __shfl_xor_sync(FULL, sx, 8));
            q4[k] = fmaxf(kq, __shfl_xor_sync(FULL, sq, 8));
          }
          float n2[2], x2[2], q2[2];
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const float sn = up4 ? n4[k] : n4[k + 2], kn = up4 ? n4[k + 2] : n4[k];
            const float sx = up4 ? x4[k] : x4[k + 2], kx = up4 ? x4[k + 2] : x4[k];
            const float sq = up4 ? q4[k] : q4[k + 2], kq = up4 ? q4[k + 2] : q4[k];
            n2[k] = fminf(kn, __shfl_xor_sync(FULL, sn, 4));
            x2[k] = fmaxf(kx, __shfl_xor_sync(FULL, sx, 4));
            q2[k] = fmaxf(kq, __shfl_xor_sync(FULL, sq, 4));
          }
          {
            const float sn = up2 ? n2[0] : n2[1], kn = up2 ? n2[1] : n2[0];
            const float sx = up2 ? x2[0] : x2[1], kx = up2 ? x2[1] : x2[0];
            const float sq = up2 ? q2[0] : q2[1], kq = up2 ? q2[1] : q2[0];
            mn = fminf(kn, __shfl_xor_sync(FULL, sn, 2));
            mx = fmaxf(kx, __shfl_xor_sync(FULL, sx, 2));
            ss = fmaxf(kq, __shfl_xor_sync(FULL, sq, 2));
          }
          mn = fminf(mn, __shfl_xor_sync(FULL, mn, 1));
          mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 1));
          ss = fmaxf(ss, __shfl_xor_sync(FULL, ss, 1));
        }
        // ---- block (tile, r_own): error bound, decidability of z and s ----
        const float M = fmaxf(fabsf(mn), fabsf(mx));
        const bool finite_bound = kA < 1.0f;
        const float A = finite_bound ? __fmul_ru(kA, __fsqrt_ru(ss)) : __int_as_float(0x7f800000);
        // z and s are decided when both ends of the interval the exact extreme lies in
        // give the same fp16 values (the maps are monotone)
        bool decided = false;
        uint16_t zh = 0, sh = 0;
        if (finite_bound) {
          const float lo_mn = __fsub_rd(mn, A), hi_mn = __fadd_ru(mn, A);
          const float lo_mx = __fsub_rd(mx, A), hi_mx = __fadd_ru(mx, A);
          zh = z_bits(lo_mn);
          sh = s_bits<QMAX>(__fsub_rd(lo_mx, hi_mn));
          decided = zh == z_bits(hi_mn) && sh == s_bits<QMAX>(__fsub_ru(hi_mx, lo_mn));
        }
        const uint32_t und = __ballot_sync(FULL, (lane & 1) == 0 && !decided && tile_ok);
        if (und) {
          const float2 e = exact_range(xrow, gf, taddr, und, mn, mx, A, a.status);
          mn = e.x;
          mx = e.y;
        }
        if (!decided) {  // mn, mx exact now (or the block is not written)
          zh = z_bits(mn);
          sh = s_bits<QMAX>(__fsub_rn(mx, mn));
        }
        QParams qp;
        qp.zh = zh;
        qp.sh = sh;
        qp.zf = __half2float(__ushort_as_half(zh));
        qp.sf = __half2float(__ushort_as_half(sh));
        qp.inv = (qp.sf != 0.0f) ? __frcp_rn(qp.sf) : 0.0f;
        // decision margin in t units, and whether the block needs clamping
        float thr;
        {
          const float Q = M + (finite_bound ? A : 0.0f) + fabsf(qp.zf);
          const float delta = finite_bound ? qp.inv * (A + 0x1p-21f * Q) * (1.0f + 0x1p-18f)
                                           : __int_as_float(0x7f800000);
          const float t_lo = __fmul_rn(__fsub_rn(mn, qp.zf), qp.inv), t_hi = __fmul_rn(__fsub_rn(mx, qp.zf), qp.inv);
          const bool inrange = (t_lo >= -0.5f + delta) && (t_hi <= (float)QMAX + 0.5f - delta);
          // a value with |t - rne(t)| >= thr is re-evaluated (thr <= 0 re-evaluates all);
          // thr in [-1, 0.5] travels shifted by -4 when the block needs clamping
          thr = fmaxf(0.5f - delta, -1.0f);
          if (!inrange) thr -= 4.0f;
        }
        if (tile_ok && (lane & 1) == 0) {
          const long long bidx = tile * 8 + r_own;
          a.scales[bidx] = qp.sh;
          a.zeros[bidx] = qp.zh;
        }

        // ---- pass 2, one group per iteration: quantize, check, repair, pack, store ----
        uint8_t* crow = a.codes + slice * slice_code_bytes + (tile - slice * (a.k.T / 16)) * (8 * 32 * BITS) +
                        j16 * (2 * BITS);
#pragma unroll 1
        for (int r = 0; r < 8; ++r) {
          float y[16];
          tmem_ld16(taddr + 16 * r, y);
          const int src = (lane & 16) + 2 * r;
          const float zf = __shfl_sync(FULL, qp.zf, src);
          const float inv = __shfl_sync(FULL, qp.inv, src);
          const float th = __shfl_sync(FULL, thr, src);
          const float Ab = __shfl_sync(FULL, A, src);
          tmem_wait_ld_into<16>(y);
          uint32_t rb[16];
          const float fmx = quant16<false, QMAX>(y, zf, inv, rb);
          float* grow = a.gauged ? a.gauged + (slice * a.k.T + tok) * D + 16 * r : nullptr;
          if (__any_sync(FULL, tile_ok && (th < -2.0f || fmx >= th))) {
            // a block needs clamping or holds values near a rounding boundary
            slow_group<BITS>(xrow, gf, taddr + 16 * r, r, zf, inv, th, Ab, tile_ok, crow + r * (32 * BITS), grow,
                             a.status);
          } else if (tile_ok) {
            store_row16<BITS>(crow + r * (32 * BITS), rb);
            if (grow) {
#pragma unroll
              for (int k = 0; k < 4; ++k)
                reinterpret_cast<float4*>(grow)[k] = make_float4(y[4 * k], y[4 * k + 1], y[4 * k + 2], y[4 * k + 3]);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&sm.t_empty[buf]);
        }
      }
      if (last_of_slice) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.g_empty[gb]);
        ++gcount;
      }
      if (++bq == bps) {
        bq = 0;
        ++slice;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
}

namespace {
template <int BITS>
cudaError_t tc16_launch(const CodecArgs& a, int num_sms, cudaStream_t st) {
  alignas(64) CUtensorMap tmap;
  const uint64_t rows = (uint64_t)a.k.slices() * a.k.T;
  if (!make_tmap_2d_bf16(&tmap, a.kv, rows, 128, 64, 128)) return cudaErrorInvalidValue;
  auto kern = encode_tc16_kernel<BITS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmem);
  if (e != cudaSuccess) return e;
  const long long total = (long long)((a.nt + 127) / 128) * a.k.slices();
  const int grid = (int)(total < num_sms ? total : num_sms);
  kern<<<grid, kThreads, kTcSmem, st>>>(tmap, a);
  return cudaGetLastError();
}
}  // namespace

bool encode_tc16_supported(const CodecArgs& a) { return a.g == 16 && a.k.d == 128 && a.W == 16 && !a.kivi; }

cudaError_t launch_encode_tc16(const CodecArgs& a, int num_sms, cudaStream_t st) {
  if (a.nt == 0) return cudaSuccess;
  if (!encode_tc16_supported(a)) return cudaErrorInvalidValue;
  switch (a.bits) {
    case 2: return tc16_launch<2>(a, num_sms, st);
    case 3: return tc16_launch<3>(a, num_sms, st);
    case 4: return tc16_launch<4>(a, num_sms, st);
    case 6: return tc16_launch<6>(a, num_sms, st);
    case 8: return tc16_launch<8>(a, num_sms, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace cg
