// KIVI-style codec with the grouped gauge fused (g = 8, 16, 32): keys are
// quantized with one range per (channel, 32 tokens), values with one range per
// (token, 32 channels).
//
// Codec-Gauge, Experimental setup: the KIVI-style backend uses per-channel key
// ranges and per-token value ranges (Liu et al. 2024c) at the same bit settings
// as the block-uniform backend; Codec-Gauge, Method: the gauge is applied
// before the backend and inverted after it, with explicit recovery.
//
// One warp owns a unit of 32 tokens x 32 channels of one head slice; lane t
// holds token t's 32 gauged values (32 / g groups).  A value range is one
// lane's 32 values.  For keys the encoder transposes the unit through shared
// memory, so that lane c holds channel c's 32 tokens: a key range is then one
// lane's values too, and lane c packs its record (token t's code at bits
// [t b, t b + b) of the little-endian bit stream) by itself.  The decoder
// gathers key codes across lanes with shuffles.
// The gauged values are the same fp32 FMA chains (j = 0..g-1 from +0) as the
// block-uniform encoder, so codes are bit-reproducible.
#include "cg_kernels.cuh"

namespace cg {

namespace {

constexpr int kWarps = 8;

struct KUnit {
  long long slice;
  int tg, cg;  // 32-token group inside [t0, t0 + nt), 32-channel group
};

__device__ inline KUnit kunit(long long u, const CodecArgs& a) {
  const int ncg = a.k.d / 32, ntg = a.nt / 32;
  KUnit k;
  k.cg = (int)(u % ncg);
  const long long r = u / ncg;
  k.tg = (int)(r % ntg);
  k.slice = r / ntg;
  return k;
}

// Stage the 32/G gauge matrices of channel group cg of slice `slice` in this
// warp's shared memory slot: Gs[rr][i][j].
template <int G>
__device__ inline void load_gauge(float* Gs, const CodecArgs& a, long long slice, int cg, int lane) {
  int l, s, b, h;
  slice_coords(slice, a.k, l, s, b, h);
  const float* src = a.G + (gauge_set(l, s, h, a.k) * (a.k.d / G) + cg * (32 / G)) * G * G;
  for (int e = lane; e < 32 * G; e += 32) Gs[e] = src[e];
  __syncwarp();
}

// The same, transposed per group (Gs[rr][j][i] = G_rr[i][j]), so that one
// 16-byte load gives four outputs' coefficients of input j.
template <int G>
__device__ inline void load_gauge_t(float* Gs, const CodecArgs& a, long long slice, int cg, int lane) {
  int l, s, b, h;
  slice_coords(slice, a.k, l, s, b, h);
  const float* src = a.G + (gauge_set(l, s, h, a.k) * (a.k.d / G) + cg * (32 / G)) * G * G;
  for (int e = lane; e < 32 * G; e += 32) {
    const int rr = e / (G * G), i = (e / G) % G, j = e % G;
    Gs[(rr * G + j) * G + i] = src[e];
  }
  __syncwarp();
}

}  // namespace

// Shared memory of the encoder per warp: its staged gauge (32 G floats) and a
// 32 x 33 fp32 transpose buffer (the padding keeps both directions free of
// bank conflicts).
template <int G>
constexpr int kivi_encode_smem() {
  return kWarps * (32 * G + 32 * 33) * 4;
}

template <int G, int BITS>
__global__ void __launch_bounds__(kWarps * 32) kivi_encode_kernel(CodecArgs a) {
  constexpr int QMAX = (1 << BITS) - 1;
  extern __shared__ __align__(16) float kivi_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* Gs = kivi_smem + warp * 32 * G;
  float* Ts = kivi_smem + kWarps * 32 * G + warp * 32 * 33;
  const long long units = a.k.slices() * (a.nt / 32) * (a.k.d / 32);
  const double inv_qmax = 1.0 / (double)QMAX;
  long long loaded = -1;
  for (long long u = (long long)blockIdx.x * kWarps + warp; u < units; u += (long long)gridDim.x * kWarps) {
    const KUnit ku = kunit(u, a);
    const long long gkey = ku.slice * 64 + ku.cg;
    if (gkey != loaded) {
      __syncwarp();
      load_gauge_t<G>(Gs, a, ku.slice, ku.cg, lane);
      loaded = gkey;
    }
    int l, s, b, h;
    slice_coords(ku.slice, a.k, l, s, b, h);
    const int tok = a.t0 + 32 * ku.tg + lane;
    const long long row = (ku.slice * a.k.T + tok) * (long long)a.k.d + 32 * ku.cg;
    // x: 32 bf16 channels of this token
    float x[32];
    {
      const uint4* src = reinterpret_cast<const uint4*>(a.kv + row);
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint4 w = src[v];
        x[8 * v + 0] = bf16lo(w.x); x[8 * v + 1] = bf16hi(w.x);
        x[8 * v + 2] = bf16lo(w.y); x[8 * v + 3] = bf16hi(w.y);
        x[8 * v + 4] = bf16lo(w.z); x[8 * v + 5] = bf16hi(w.z);
        x[8 * v + 6] = bf16lo(w.w); x[8 * v + 7] = bf16hi(w.w);
      }
    }
    // y = G x per group: fp32 FMA chain over j in index order from +0, two
    // outputs' chains per packed fma.rn.f32x2 (each half rounds as the scalar FMA)
    float y[32];
#pragma unroll
    for (int rr = 0; rr < 32 / G; ++rr) {
#pragma unroll
      for (int i = 0; i < G; i += 4) {
        f2_t acc01 = f2_make(0.0f, 0.0f), acc23 = f2_make(0.0f, 0.0f);
#pragma unroll
        for (int j = 0; j < G; ++j) {
          const float4 c = *reinterpret_cast<const float4*>(Gs + (rr * G + j) * G + i);
          const f2_t xx = f2_make(x[rr * G + j], x[rr * G + j]);
          acc01 = f2_fma(f2_make(c.x, c.y), xx, acc01);
          acc23 = f2_fma(f2_make(c.z, c.w), xx, acc23);
        }
        f2_split(acc01, y[rr * G + i], y[rr * G + i + 1]);
        f2_split(acc23, y[rr * G + i + 2], y[rr * G + i + 3]);
      }
    }
    if (a.gauged) {
      float4* dst = reinterpret_cast<float4*>(a.gauged + row);
#pragma unroll
      for (int v = 0; v < 8; ++v) dst[v] = make_float4(y[4 * v], y[4 * v + 1], y[4 * v + 2], y[4 * v + 3]);
    }
    // per (l, s, b, h): keys and values each hold T * d * bits / 8 code bytes and T * d / 32 ranges
    const long long slice_bytes = (long long)a.k.T * a.k.d * BITS / 8;
    const long long slice_ranges = (long long)a.k.T * a.k.d / 32;
    if (s == 0) {
      // ---- keys: range per channel over the 32 tokens; transpose so that lane c
      // holds channel c ----
      __syncwarp();  // the previous unit's reads of the buffer are done
#pragma unroll
      for (int c = 0; c < 32; ++c) Ts[lane * 33 + c] = y[c];
      __syncwarp();
      float yc[32];
#pragma unroll
      for (int t = 0; t < 32; ++t) yc[t] = Ts[t * 33 + lane];
      float mn = yc[0], mx = yc[0];
#pragma unroll
      for (int t = 1; t < 32; ++t) {
        mn = fminf(mn, yc[t]);
        mx = fmaxf(mx, yc[t]);
      }
      const QParams qp = quant_params(mn, mx, inv_qmax);
      const int tgroup = (a.t0 / 32) + ku.tg;
      const long long ridx = ku.slice * slice_ranges + (long long)tgroup * a.k.d + 32 * ku.cg + lane;
      a.scales[ridx] = qp.sh;
      a.zeros[ridx] = qp.zh;
      // codes: channel c's record = 32 codes, token-ascending; lane c stores record c
      uint32_t words[BITS];
#pragma unroll
      for (int w = 0; w < BITS; ++w) words[w] = 0;
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        const uint32_t q = quantize_one(yc[t], qp.zf, qp.inv, QMAX);
        const int bit = t * BITS;
        words[bit >> 5] |= q << (bit & 31);
        if ((bit & 31) + BITS > 32) words[(bit >> 5) + 1] |= q >> (32 - (bit & 31));
      }
      uint32_t* rec = reinterpret_cast<uint32_t*>(a.codes + ku.slice * slice_bytes +
                                                   ((long long)tgroup * a.k.d + 32 * ku.cg + lane) * (4 * BITS));
#pragma unroll
      for (int w = 0; w < BITS; ++w) rec[w] = words[w];
    } else {
      // ---- values: range per token over its 32 channels (this lane) ----
      float mn = y[0], mx = y[0];
#pragma unroll
      for (int c = 1; c < 32; ++c) {
        mn = fminf(mn, y[c]);
        mx = fmaxf(mx, y[c]);
      }
      const QParams qp = quant_params(mn, mx, inv_qmax);
      const long long ridx = ku.slice * slice_ranges + (long long)tok * (a.k.d / 32) + ku.cg;
      a.scales[ridx] = qp.sh;
      a.zeros[ridx] = qp.zh;
      uint32_t words[BITS];
#pragma unroll
      for (int w = 0; w < BITS; ++w) words[w] = 0;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const uint32_t q = quantize_one(y[c], qp.zf, qp.inv, QMAX);
        const int bit = c * BITS;
        words[bit >> 5] |= q << (bit & 31);
        if ((bit & 31) + BITS > 32) words[(bit >> 5) + 1] |= q >> (32 - (bit & 31));
      }
      uint32_t* rec = reinterpret_cast<uint32_t*>(a.codes + ku.slice * slice_bytes +
                                                   ((long long)tok * (a.k.d / 32) + ku.cg) * (4 * BITS));
#pragma unroll
      for (int w = 0; w < BITS; ++w) rec[w] = words[w];
    }
  }
}

template <int G, int BITS>
__global__ void __launch_bounds__(kWarps * 32) kivi_decode_kernel(CodecArgs a) {
  constexpr uint32_t M = (1u << BITS) - 1u;
  __shared__ __align__(16) float sG[kWarps][32 * G];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* Gs = sG[warp];
  const long long units = a.k.slices() * (a.nt / 32) * (a.k.d / 32);
  long long loaded = -1;
  for (long long u = (long long)blockIdx.x * kWarps + warp; u < units; u += (long long)gridDim.x * kWarps) {
    const KUnit ku = kunit(u, a);
    const long long gkey = ku.slice * 64 + ku.cg;
    if (gkey != loaded) {
      __syncwarp();
      load_gauge<G>(Gs, a, ku.slice, ku.cg, lane);
      loaded = gkey;
    }
    int l, s, b, h;
    slice_coords(ku.slice, a.k, l, s, b, h);
    const int tok = a.t0 + 32 * ku.tg + lane;
    const long long slice_bytes = (long long)a.k.T * a.k.d * BITS / 8;
    const long long slice_ranges = (long long)a.k.T * a.k.d / 32;
    float yh[32];
    if (s == 0) {
      // keys: lane c reads record c (32 tokens' codes) and its range; token t's
      // code of channel c is bits [t b, t b + b) of record c
      const int tgroup = (a.t0 / 32) + ku.tg;
      const long long ridx = ku.slice * slice_ranges + (long long)tgroup * a.k.d + 32 * ku.cg + lane;
      const float sf_c = __half2float(__ushort_as_half(a.scales_in[ridx]));
      const float zf_c = __half2float(__ushort_as_half(a.zeros_in[ridx]));
      const uint32_t* rec = reinterpret_cast<const uint32_t*>(
          a.codes_in + ku.slice * slice_bytes + ((long long)tgroup * a.k.d + 32 * ku.cg + lane) * (4 * BITS));
      uint32_t wr[BITS + 1];
#pragma unroll
      for (int w = 0; w < BITS; ++w) wr[w] = rec[w];
      wr[BITS] = 0;
      const int bit = lane * BITS;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int w = 0; w < BITS; ++w) {
          const uint32_t v = __shfl_sync(0xffffffffu, wr[w], c);
          lo = ((bit >> 5) == w) ? v : lo;
          hi = ((bit >> 5) + 1 == w) ? v : hi;
        }
        const uint32_t q = __funnelshift_r(lo, hi, bit & 31) & M;
        const float sf = __shfl_sync(0xffffffffu, sf_c, c), zf = __shfl_sync(0xffffffffu, zf_c, c);
        yh[c] = __fmaf_rn(sf, (float)q, zf);
      }
    } else {
      const long long ridx = ku.slice * slice_ranges + (long long)tok * (a.k.d / 32) + ku.cg;
      const float sf = __half2float(__ushort_as_half(a.scales_in[ridx]));
      const float zf = __half2float(__ushort_as_half(a.zeros_in[ridx]));
      const uint32_t* rec = reinterpret_cast<const uint32_t*>(a.codes_in + ku.slice * slice_bytes +
                                                              ((long long)tok * (a.k.d / 32) + ku.cg) * (4 * BITS));
      uint32_t wr[BITS + 1];
#pragma unroll
      for (int w = 0; w < BITS; ++w) wr[w] = rec[w];
      wr[BITS] = 0;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const int bit = c * BITS;
        const uint32_t q = __funnelshift_r(wr[bit >> 5], wr[(bit >> 5) + 1], bit & 31) & M;
        yh[c] = __fmaf_rn(sf, (float)q, zf);
      }
    }
    // x_hat = G^T yhat per group
    float xo[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) xo[i] = 0.0f;
#pragma unroll
    for (int rr = 0; rr < 32 / G; ++rr) {
#pragma unroll
      for (int c = 0; c < G; ++c) {
        const float* gc = Gs + (rr * G + c) * G;
#pragma unroll
        for (int i = 0; i < G; i += 4) {
          const float4 v = *reinterpret_cast<const float4*>(gc + i);
          xo[rr * G + i + 0] = __fmaf_rn(v.x, yh[rr * G + c], xo[rr * G + i + 0]);
          xo[rr * G + i + 1] = __fmaf_rn(v.y, yh[rr * G + c], xo[rr * G + i + 1]);
          xo[rr * G + i + 2] = __fmaf_rn(v.z, yh[rr * G + c], xo[rr * G + i + 2]);
          xo[rr * G + i + 3] = __fmaf_rn(v.w, yh[rr * G + c], xo[rr * G + i + 3]);
        }
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(a.kv_out + (ku.slice * a.k.T + tok) * (long long)a.k.d + 32 * ku.cg);
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      uint4 w;
      w.x = pack_bf16x2(xo[8 * v + 0], xo[8 * v + 1]);
      w.y = pack_bf16x2(xo[8 * v + 2], xo[8 * v + 3]);
      w.z = pack_bf16x2(xo[8 * v + 4], xo[8 * v + 5]);
      w.w = pack_bf16x2(xo[8 * v + 6], xo[8 * v + 7]);
      dst[v] = w;
    }
  }
}

namespace {
template <int G, int BITS>
cudaError_t kivi_launch(const CodecArgs& a, bool encode, int num_sms, cudaStream_t st) {
  const long long units = a.k.slices() * (a.nt / 32) * (a.k.d / 32);
  const long long want = (units + kWarps - 1) / kWarps;
  const int grid = (int)(want < (long long)num_sms * 8 ? want : (long long)num_sms * 8);
  if (encode) {
    auto kern = kivi_encode_kernel<G, BITS>;
    constexpr int smem = kivi_encode_smem<G>();
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, kWarps * 32, smem, st>>>(a);
  } else {
    kivi_decode_kernel<G, BITS><<<grid, kWarps * 32, 0, st>>>(a);
  }
  return cudaGetLastError();
}
template <int G>
cudaError_t kivi_bits(const CodecArgs& a, bool encode, int num_sms, cudaStream_t st) {
  switch (a.bits) {
    case 2: return kivi_launch<G, 2>(a, encode, num_sms, st);
    case 3: return kivi_launch<G, 3>(a, encode, num_sms, st);
    case 4: return kivi_launch<G, 4>(a, encode, num_sms, st);
    case 6: return kivi_launch<G, 6>(a, encode, num_sms, st);
    case 8: return kivi_launch<G, 8>(a, encode, num_sms, st);
  }
  return cudaErrorInvalidValue;
}
}  // namespace

cudaError_t launch_kivi(const CodecArgs& a, bool encode, int num_sms, cudaStream_t st) {
  if (a.nt == 0) return cudaSuccess;
  switch (a.g) {
    case 8: return kivi_bits<8>(a, encode, num_sms, st);
    case 16: return kivi_bits<16>(a, encode, num_sms, st);
    case 32: return kivi_bits<32>(a, encode, num_sms, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace cg
