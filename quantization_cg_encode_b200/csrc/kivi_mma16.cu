// KIVI-style encoder, default engine for g = 16 (d_head 64 or 128): the gauge
// on the warp-level tensor cores, then KIVI's ranges on the exact fp32
// quantizer.
//
// Codec-Gauge, Experimental setup: the KIVI-style backend takes per-channel
// key ranges and per-token value ranges (32 tokens / 32 channels here);
// Codec-Gauge, Method: the gauge is applied before the backend.  As in the
// block-uniform default engine, the gauged values are this kernel's own
// contraction y = (G_hi + G_lo) x (G split into two bf16 terms, x bf16 exact,
// fp32 accumulation: within 2^-16 sum_j |G_ij x_j| of G x), and the codes,
// steps and zero points are the quantizer's exact fp32 result for those y.
//
// One CTA of 8 warps takes units of TOK = 8192 / d tokens of one head slice
// (grid-stride), in three phases per unit:
//   1. the unit's bf16 rows sit in a padded shared tile (the next unit's rows
//      are already in registers, loaded while the previous unit was quantized);
//   2. warp w runs ldmatrix + mma.sync (m16n8k16, G_lo then G_hi) over its
//      16-token tiles of channel group w mod (d / 16) and writes y (fp32) to a
//      second shared tile (and, on request, to the gauged output);
//   3. every thread takes one range, as a lane does in the chain engine: keys:
//      channel c over 32 tokens; values: one token over 32 channels; min / max,
//      the quantizer's fp16 step and zero point, codes packed little-endian
//      into the range's record (token- or channel-ascending).
#include "cg_kernels.cuh"

namespace cg {

namespace {

constexpr int kKWarps = 8;
constexpr int kKThreads = kKWarps * 32;

template <int D>
struct KivCfg {
  static constexpr int NG = D / 16;
  static constexpr int TOK = 8192 / D;       // tokens per unit: 64 (d = 128) or 128 (d = 64)
  static constexpr int TILES = TOK / 16;
  static constexpr int WPG = kKWarps / NG;   // warps per channel group: 1 or 2
  static constexpr int TPW = TILES / WPG;    // tiles per warp: 4
  static constexpr int XP = D * 2 + 16;      // bf16 tile row pitch in bytes (ldmatrix rows on distinct banks)
  static constexpr int YP = D + 4;           // fp32 tile row pitch in floats
  static constexpr int LOADS = TOK * D * 2 / 16 / kKThreads;  // 16-byte loads per thread per unit: 4
  static constexpr int SMEM = TOK * XP + TOK * YP * 4;
};

constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23: t + kMagic rounds t to an integer (RNE) in the low bits

// One range of 32 values v: the quantizer's fp16 step and zero point from its
// extremes, then q = clamp(rne(fl(fl(v - z) * fl(1 / s))), 0, qmax) packed
// little-endian (code k at bits [k b, k b + b)).  t is monotone in v, so the
// clamp is needed only when the extremes' t fall outside [-0.5, qmax + 0.5);
// the rounding is the magic-number add on packed fp32 pairs.
template <int BITS>
__device__ __forceinline__ QParams quantize_pack32(const float (&v)[32], double inv_qmax, uint32_t (&words)[BITS]) {
  constexpr int QMAX = (1 << BITS) - 1;
  float m1[11], x1[11];  // tree: 32 -> 11 -> 4 -> 2 -> 1
#pragma unroll
  for (int k = 0; k < 10; ++k) {
    m1[k] = min3f(v[3 * k], v[3 * k + 1], v[3 * k + 2]);
    x1[k] = max3f(v[3 * k], v[3 * k + 1], v[3 * k + 2]);
  }
  m1[10] = fminf(v[30], v[31]);
  x1[10] = fmaxf(v[30], v[31]);
  const float m2a = min3f(m1[0], m1[1], m1[2]), m2b = min3f(m1[3], m1[4], m1[5]), m2c = min3f(m1[6], m1[7], m1[8]);
  const float x2a = max3f(x1[0], x1[1], x1[2]), x2b = max3f(x1[3], x1[4], x1[5]), x2c = max3f(x1[6], x1[7], x1[8]);
  const float mn = fminf(min3f(m2a, m2b, m2c), fminf(m1[9], m1[10]));
  const float mx = fmaxf(max3f(x2a, x2b, x2c), fmaxf(x1[9], x1[10]));
  const QParams qp = quant_params(mn, mx, inv_qmax);
  const float t_lo = __fmul_rn(__fsub_rn(mn, qp.zf), qp.inv), t_hi = __fmul_rn(__fsub_rn(mx, qp.zf), qp.inv);
  const bool clampit = !(t_lo >= -0.5f && t_hi < (float)QMAX + 0.5f);
  const f2_t nz2 = f2_make(-qp.zf, -qp.zf), iv2 = f2_make(qp.inv, qp.inv), mg2 = f2_make(kMagic, kMagic);
#pragma unroll
  for (int w = 0; w < BITS; ++w) words[w] = 0;
#pragma unroll
  for (int k = 0; k < 32; k += 2) {
    float t0, t1;
    f2_split(f2_mul(f2_add(f2_make(v[k], v[k + 1]), nz2), iv2), t0, t1);
    if (clampit) {
      t0 = fminf(fmaxf(t0, 0.0f), (float)QMAX);
      t1 = fminf(fmaxf(t1, 0.0f), (float)QMAX);
    }
    float r0, r1;
    f2_split(f2_add(f2_make(t0, t1), mg2), r0, r1);
    const uint32_t q[2] = {__float_as_uint(r0) & (uint32_t)QMAX, __float_as_uint(r1) & (uint32_t)QMAX};
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int bit = (k + e) * BITS;
      words[bit >> 5] |= q[e] << (bit & 31);
      if ((bit & 31) + BITS > 32) words[(bit >> 5) + 1] |= q[e] >> (32 - (bit & 31));
    }
  }
  return qp;
}

}  // namespace

template <int D, int BITS>
__global__ void __launch_bounds__(kKThreads, 3) kivi_mma16_encode_kernel(CodecArgs a) {
  using C = KivCfg<D>;
  constexpr int QMAX = (1 << BITS) - 1;
  static_assert(QMAX < 256, "codes fit the low byte of t + kMagic");
  extern __shared__ __align__(16) unsigned char kv_smem[];
  unsigned char* xs = kv_smem;                                   // [TOK][XP bytes] bf16 rows
  float* ys = reinterpret_cast<float*>(kv_smem + C::TOK * C::XP);  // [TOK][YP] gauged values

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;
  const int r = warp % C::NG, part = warp / C::NG;
  const int upsl = (a.nt + C::TOK - 1) / C::TOK;  // units per head slice
  const int units = upsl * (int)a.k.slices();      // below 2^31 (checked by the launcher)
  const double inv_qmax = 1.0 / (double)QMAX;
  const long long slice_bytes = (long long)a.k.T * D * BITS / 8;
  const long long slice_ranges = (long long)a.k.T * D / 32;

  // 16-byte piece e of a unit: row e / (D / 8), chunk e % (D / 8)
  auto load_unit = [&](int u, uint4 (&v)[C::LOADS]) {
    const int slice = u / upsl;
    const int tok0 = (u - slice * upsl) * C::TOK;
    const int rows = min(C::TOK, a.nt - tok0);
#pragma unroll
    for (int k = 0; k < C::LOADS; ++k) {
      const int e = tid + k * kKThreads, row = e / (D / 8), ch = e % (D / 8);
      v[k] = row < rows ? __ldg(reinterpret_cast<const uint4*>(a.kv + ((long long)slice * a.k.T + a.t0 + tok0 + row) * D) + ch)
                        : make_uint4(0, 0, 0, 0);
    }
  };
  auto store_unit = [&](const uint4 (&v)[C::LOADS]) {
#pragma unroll
    for (int k = 0; k < C::LOADS; ++k) {
      const int e = tid + k * kKThreads, row = e / (D / 8), ch = e % (D / 8);
      *reinterpret_cast<uint4*>(xs + row * C::XP + ch * 16) = v[k];
    }
  };

  // ldmatrix rows of lane l inside a 16 x 16 tile of group r: rows (l & 7) + 8 ((l >> 3) & 1),
  // channels 16 r + 8 (l >> 4)
  const int lrow = (lane & 7) + 8 * ((lane >> 3) & 1);
  const uint32_t xs_lane = smem_u32(xs) + lrow * C::XP + (16 * r + 8 * (lane >> 4)) * 2;

  uint32_t bh[2][2], bl[2][2];  // [n-half][b0/b1] bf16 pairs of G_hi, G_lo
  int gslice = -1, sk = 0;
  uint4 nxt[C::LOADS];
  int u = blockIdx.x;
  if (u < units) load_unit(u, nxt);
  for (; u < units; u += gridDim.x) {
    const int slice = u / upsl;
    const int tok0 = (u - slice * upsl) * C::TOK;
    const int rows = min(C::TOK, a.nt - tok0);  // a multiple of 32
    __syncthreads();  // the previous unit's phases 2 and 3 are done with both tiles
    store_unit(nxt);
    if (u + (int)gridDim.x < units) load_unit(u + gridDim.x, nxt);  // in flight during this unit
    if (slice != gslice) {
      int l, b, h;
      slice_coords(slice, a.k, l, sk, b, h);
      // B[k][n] = G[i][k], i = 4 (n >> 1) + 2 h + (n & 1) for n-half h: a thread's
      // accumulators are output channels 4c .. 4c+3 of rows g and g + 8
      const float* Gr = a.G + (gauge_set(l, sk, h, a.k) * C::NG + r) * 256;
#pragma unroll
      for (int nh = 0; nh < 2; ++nh) {
        const int i = 4 * (g >> 1) + 2 * nh + (g & 1);
        const float2 p0 = __ldg(reinterpret_cast<const float2*>(Gr + i * 16 + 2 * c));
        const float2 p1 = __ldg(reinterpret_cast<const float2*>(Gr + i * 16 + 2 * c + 8));
        const float2 p[2] = {p0, p1};
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const uint32_t hi = pack_bf16x2(p[k].x, p[k].y);
          bh[nh][k] = hi;
          bl[nh][k] = pack_bf16x2(p[k].x - bf16lo(hi), p[k].y - bf16hi(hi));  // residuals are exact
        }
      }
      gslice = slice;
    }
    __syncthreads();  // the unit's rows are in the tile

    // ---- phase 2: y = G x per 16-token tile of group r ----
#pragma unroll
    for (int j = 0; j < C::TPW; ++j) {
      const int tile = part * C::TPW + j;
      if (tile * 16 >= rows) break;  // warp-uniform
      uint32_t afr[4];
      ldmatrix_x4(afr, xs_lane + tile * 16 * C::XP);
      float acc[2][4];
#pragma unroll
      for (int nh = 0; nh < 2; ++nh) {
        mma_bf16_16816_z(acc[nh], afr, bl[nh][0], bl[nh][1]);
        mma_bf16_16816(acc[nh], afr, bh[nh][0], bh[nh][1]);
      }
      const float4 y0 = make_float4(acc[0][0], acc[0][1], acc[1][0], acc[1][1]);  // row g, channels 4c ..
      const float4 y1 = make_float4(acc[0][2], acc[0][3], acc[1][2], acc[1][3]);  // row g + 8
      const int row = tile * 16 + g;
      *reinterpret_cast<float4*>(ys + row * C::YP + 16 * r + 4 * c) = y0;
      *reinterpret_cast<float4*>(ys + (row + 8) * C::YP + 16 * r + 4 * c) = y1;
      if (a.gauged) {
        float* gp = a.gauged + ((long long)slice * a.k.T + a.t0 + tok0 + row) * D + 16 * r + 4 * c;
        *reinterpret_cast<float4*>(gp) = y0;
        *reinterpret_cast<float4*>(gp + 8 * D) = y1;
      }
    }
    __syncthreads();  // y is in the tile

    // ---- phase 3: one range per thread ----
    uint32_t words[BITS];
    if (sk == 0) {
      // keys: channel ch over the 32 tokens of group tg (record token-ascending)
      const int ch = tid % D, tg = tid / D;
      if (32 * tg < rows) {
        float yc[32];
#pragma unroll
        for (int t = 0; t < 32; ++t) yc[t] = ys[(32 * tg + t) * C::YP + ch];
        const QParams qp = quantize_pack32<BITS>(yc, inv_qmax, words);
        const long long tgroup = (a.t0 + tok0) / 32 + tg;
        const long long ridx = (long long)slice * slice_ranges + tgroup * D + ch;
        a.scales[ridx] = qp.sh;
        a.zeros[ridx] = qp.zh;
        uint32_t* rec = reinterpret_cast<uint32_t*>(a.codes + (long long)slice * slice_bytes + (tgroup * D + ch) * (4 * BITS));
#pragma unroll
        for (int w = 0; w < BITS; ++w) rec[w] = words[w];
      }
    } else {
      // values: token t over channels 32 cg .. 32 cg + 31 (record channel-ascending)
      const int t = tid / (D / 32), cgp = tid % (D / 32);
      if (t < rows) {
        float yv[32];
        const float4* src = reinterpret_cast<const float4*>(ys + t * C::YP + 32 * cgp);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float4 f = src[k];
          yv[4 * k] = f.x;
          yv[4 * k + 1] = f.y;
          yv[4 * k + 2] = f.z;
          yv[4 * k + 3] = f.w;
        }
        const QParams qp = quantize_pack32<BITS>(yv, inv_qmax, words);
        const long long tok = a.t0 + tok0 + t;
        const long long ridx = (long long)slice * slice_ranges + tok * (D / 32) + cgp;
        a.scales[ridx] = qp.sh;
        a.zeros[ridx] = qp.zh;
        uint32_t* rec = reinterpret_cast<uint32_t*>(a.codes + (long long)slice * slice_bytes + (tok * (D / 32) + cgp) * (4 * BITS));
#pragma unroll
        for (int w = 0; w < BITS; ++w) rec[w] = words[w];
      }
    }
  }
}

bool kivi_mma16_supported(const CodecArgs& a) { return a.kivi && a.g == 16 && (a.k.d == 64 || a.k.d == 128); }

namespace {

template <int D, int BITS>
cudaError_t kivi_mma16_launch(const CodecArgs& a, int num_sms, cudaStream_t st) {
  using C = KivCfg<D>;
  auto kern = kivi_mma16_encode_kernel<D, BITS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kKThreads, C::SMEM);
  if (e != cudaSuccess) return e;
  const long long units = (long long)((a.nt + C::TOK - 1) / C::TOK) * a.k.slices();
  if (units >= (1LL << 31)) return cudaErrorInvalidValue;  // unit indices are 32-bit
  const long long cap = (long long)num_sms * (per_sm > 0 ? per_sm : 1);
  const int grid = (int)(units < cap ? units : cap);
  kern<<<grid, kKThreads, C::SMEM, st>>>(a);
  return cudaGetLastError();
}

template <int D>
cudaError_t kivi_mma16_bits(const CodecArgs& a, int num_sms, cudaStream_t st) {
  switch (a.bits) {
    case 2: return kivi_mma16_launch<D, 2>(a, num_sms, st);
    case 3: return kivi_mma16_launch<D, 3>(a, num_sms, st);
    case 4: return kivi_mma16_launch<D, 4>(a, num_sms, st);
    case 6: return kivi_mma16_launch<D, 6>(a, num_sms, st);
    case 8: return kivi_mma16_launch<D, 8>(a, num_sms, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_kivi_mma16(const CodecArgs& a, int num_sms, cudaStream_t st) {
  if (a.nt == 0) return cudaSuccess;
  return a.k.d == 128 ? kivi_mma16_bits<128>(a, num_sms, st) : kivi_mma16_bits<64>(a, num_sms, st);
}

}  // namespace cg
