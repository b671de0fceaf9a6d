// Gauge-training statistics on CUDA cores for any head width (d_head 64 or
// 128, any token count that is a multiple of 16): the same quantities as the
// tensor-core kernel (spectral.cu), one 16-token block at a time.
//
// Codec-Gauge, Method (frequency-distribution objective): every 16 x d block of
// X' = G X gets the orthonormal 2-D DCT-II U = C_16 X' C_d^T, spanning the whole
// head even when the gauge is grouped; per block L_freq = sum r_uv U^2 / sum U^2
// (0 for an all-zero block) with r_uv = sqrt((u/15)^2 + (v/(d-1))^2)/sqrt(2),
// and L_rate = mean log(1 + |U| / tau) (assumed form: the page's equation is
// truncated).  With a gradient:
//   dU = lambda_f 2 U (r - L_freq) / (E n_blk) + lambda_r sign(U) / ((tau + |U|) N_U),
//   dX' = C_16^T dU C_d,   dG_r[i][j] += sum_t dX'[t][16 r + i] x[t][16 r + j].
//
// One CTA owns whole head slices and walks their blocks in token order, so a
// slice's dG partial is a fixed-order sum and the result is deterministic.
// All arithmetic is fp32 (each output a fixed-order sum of at most d terms).
#include "cg_kernels.cuh"

namespace cg {

namespace {

constexpr int kGenThreads = 256;

struct GenArgs {
  KvGeom k;
  int x_fp32, has_g, want_grad;
  float lambda_f, lambda_r, tau;
  float inv_nblk, inv_ncoef;
  const void* x;
  const float* G;
  float* lfreq;
  float* lrate;
  float* dg_part;  // [slices][d/16][16][16]
};

template <int D>
struct GenSmem {
  static constexpr int P = D + 1;  // padded row pitch
  static constexpr int FLOATS = D * P /* C_d */ + 256 /* C_16 */ + 16 * D /* x */ + 2 * 16 * P /* two work */ +
                                (D / 16) * 256 /* G */ + D /* radius columns */ + 3 * 8 /* reductions */;
  static constexpr int BYTES = FLOATS * 4;
};

__device__ __forceinline__ float dct_c(int k, int n, int N) {
  const float a = k == 0 ? sqrtf(1.0f / N) : sqrtf(2.0f / N);
  return a * cospif((2.0f * n + 1.0f) * k / (2.0f * N));
}

// Sum of v over the CTA (256 threads), the same fixed tree on every call.
__device__ __forceinline__ float cta_sum(float v, float* red, int slot) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) red[slot * 8 + warp] = v;
  __syncthreads();
  float s = 0.0f;
#pragma unroll
  for (int w = 0; w < 8; ++w) s += red[slot * 8 + w];
  return s;
}

}  // namespace

template <int D>
__global__ void __launch_bounds__(kGenThreads) spectral_generic_kernel(GenArgs a) {
  constexpr int NG = D / 16;
  constexpr int P = GenSmem<D>::P;
  extern __shared__ float gsm[];
  float* Cd = gsm;                // [D][P]: C_d[v][c]
  float* C16 = Cd + D * P;        // [16][16]
  float* xs = C16 + 256;          // [16][D]: x of the block
  float* w1 = xs + 16 * D;        // [16][P]: X', then dV
  float* w2 = w1 + 16 * P;        // [16][P]: V = X' C_d^T, then U, then dU, then dX'
  float* Gs = w2 + 16 * P;        // [NG][16][16]
  float* rv = Gs + NG * 256;      // [D]: v / (d - 1)
  float* red = rv + D;            // [3][8]
  const int tid = threadIdx.x;

  for (int e = tid; e < D * D; e += kGenThreads) Cd[(e / D) * P + e % D] = dct_c(e / D, e % D, D);
  for (int e = tid; e < 256; e += kGenThreads) C16[e] = dct_c(e / 16, e % 16, 16);
  for (int e = tid; e < D; e += kGenThreads) rv[e] = (float)e / (float)(D - 1);
  __syncthreads();

  const long long slices = a.k.slices();
  const int nblk = a.k.T / 16;
  for (long long slice = blockIdx.x; slice < slices; slice += gridDim.x) {
    int l, sk, b, h;
    slice_coords(slice, a.k, l, sk, b, h);
    if (a.has_g)
      for (int e = tid; e < NG * 256; e += kGenThreads) Gs[e] = a.G[gauge_set(l, sk, h, a.k) * NG * 256 + e];
    // dG partial entries tid + 256 k of [NG][16][16]: each block's 16 products summed
    // afresh, then added with compensation (dg - dgc is the running sum)
    float dg[NG], dgc[NG];
#pragma unroll
    for (int k = 0; k < NG; ++k) {
      dg[k] = 0.0f;
      dgc[k] = 0.0f;
    }
    __syncthreads();

    for (int kb = 0; kb < nblk; ++kb) {
      const long long row0 = slice * a.k.T + 16LL * kb;
      // x of the block, then X' = G x per token and group (fp32 chain in index order)
      for (int e = tid; e < 16 * D; e += kGenThreads) {
        const long long idx = row0 * D + e;
        xs[e] = a.x_fp32 ? reinterpret_cast<const float*>(a.x)[idx]
                         : bf16lo((uint32_t)reinterpret_cast<const uint16_t*>(a.x)[idx]);
      }
      __syncthreads();
      for (int e = tid; e < 16 * D; e += kGenThreads) {
        const int t = e / D, c = e % D;
        float y = xs[e];
        if (a.has_g) {
          const int r = c >> 4, i = c & 15;
          const float* gi = Gs + (r * 16 + i) * 16;
          const float* xr = xs + t * D + 16 * r;
          y = 0.0f;
#pragma unroll
          for (int j = 0; j < 16; ++j) y = __fmaf_rn(gi[j], xr[j], y);
        }
        w1[t * P + c] = y;
      }
      __syncthreads();
      // V[t][v] = sum_c X'[t][c] C_d[v][c]
      for (int e = tid; e < 16 * D; e += kGenThreads) {
        const int t = e / D, v = e % D;
        const float* xr = w1 + t * P;
        const float* cr = Cd + v * P;
        float acc = 0.0f;
#pragma unroll 8
        for (int cc = 0; cc < D; ++cc) acc = __fmaf_rn(xr[cc], cr[cc], acc);
        w2[t * P + v] = acc;
      }
      __syncthreads();
      // U[u][v] = sum_t C_16[u][t] V[t][v] (column v per thread: each thread owns whole columns)
      float U[16];
      float e_sum = 0.0f, f_sum = 0.0f, r_sum = 0.0f;
      const int v = tid % D;
      const bool owner = tid < D;  // threads 0 .. D-1 own the D columns
      if (owner) {
        float col[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) col[t] = w2[t * P + v];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          float acc = 0.0f;
#pragma unroll
          for (int t = 0; t < 16; ++t) acc = __fmaf_rn(C16[u * 16 + t], col[t], acc);
          U[u] = acc;
          const float ru = (float)u / 15.0f;
          const float rad = sqrtf(ru * ru + rv[v] * rv[v]) * 0.70710678118654752f;
          const float e2 = acc * acc;
          e_sum += e2;
          f_sum = __fmaf_rn(rad, e2, f_sum);
          r_sum += log1pf(fabsf(acc) / a.tau);
        }
      }
      const float E = cta_sum(e_sum, red, 0);
      const float F = cta_sum(f_sum, red, 1);
      const float R = cta_sum(r_sum, red, 2);
      const float lf = E > 0.0f ? F / E : 0.0f;
      if (tid == 0) {
        a.lfreq[slice * nblk + kb] = lf;
        a.lrate[slice * nblk + kb] = R / (16.0f * D);
      }
      if (a.want_grad) {
        // dU, then dV[t][v] = sum_u C_16[u][t] dU[u][v] (column v, in w1)
        if (owner) {
          const float cf = E > 0.0f ? 2.0f * a.lambda_f * a.inv_nblk / E : 0.0f;
          const float cr = a.lambda_r * a.inv_ncoef;
          float dU[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const float ru = (float)u / 15.0f;
            const float rad = sqrtf(ru * ru + rv[v] * rv[v]) * 0.70710678118654752f;
            const float sg = U[u] > 0.0f ? 1.0f : (U[u] < 0.0f ? -1.0f : 0.0f);
            dU[u] = __fmaf_rn(cf * U[u], rad - lf, cr * sg / (a.tau + fabsf(U[u])));
          }
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            float acc = 0.0f;
#pragma unroll
            for (int u = 0; u < 16; ++u) acc = __fmaf_rn(C16[u * 16 + t], dU[u], acc);
            w1[t * P + v] = acc;
          }
        }
        __syncthreads();
        // dX'[t][c] = sum_v dV[t][v] C_d[v][c]  (in w2)
        for (int e = tid; e < 16 * D; e += kGenThreads) {
          const int t = e / D, c = e % D;
          const float* dr = w1 + t * P;
          float acc = 0.0f;
#pragma unroll 8
          for (int vv = 0; vv < D; ++vv) acc = __fmaf_rn(dr[vv], Cd[vv * P + c], acc);
          w2[t * P + c] = acc;
        }
        __syncthreads();
        // dG_r[i][j] += sum_t dX'[t][16 r + i] x[t][16 r + j]
#pragma unroll
        for (int k = 0; k < NG; ++k) {
          const int e = tid + kGenThreads * k, r = e >> 8, i = (e >> 4) & 15, j = e & 15;
          float acc = 0.0f;
#pragma unroll
          for (int t = 0; t < 16; ++t) acc = __fmaf_rn(w2[t * P + 16 * r + i], xs[t * D + 16 * r + j], acc);
          const float yk = __fsub_rn(acc, dgc[k]);
          const float tk = __fadd_rn(dg[k], yk);
          dgc[k] = __fsub_rn(__fsub_rn(tk, dg[k]), yk);
          dg[k] = tk;
        }
      }
      __syncthreads();  // xs, w1, w2 and red are rewritten by the next block
    }
    if (a.want_grad) {
#pragma unroll
      for (int k = 0; k < NG; ++k)
        a.dg_part[slice * (long long)NG * 256 + tid + kGenThreads * k] = __fsub_rn(dg[k], dgc[k]);
    }
    __syncthreads();  // Gs is rewritten by the next slice
  }
}

cudaError_t launch_spectral_generic(const KvGeom& k, int x_fp32, const void* x, const float* G, float lambda_f,
                                    float lambda_r, float tau, float* lfreq, float* lrate, float* dg_part,
                                    int num_sms, cudaStream_t st) {
  GenArgs a;
  a.k = k;
  a.x_fp32 = x_fp32;
  a.has_g = G != nullptr;
  a.want_grad = dg_part != nullptr;
  a.lambda_f = lambda_f;
  a.lambda_r = lambda_r;
  a.tau = tau;
  const double nblk = (double)k.slices() * (k.T / 16);
  a.inv_nblk = (float)(1.0 / nblk);
  a.inv_ncoef = (float)(1.0 / (nblk * 16.0 * k.d));
  a.x = x;
  a.G = G;
  a.lfreq = lfreq;
  a.lrate = lrate;
  a.dg_part = dg_part;
  const long long slices = k.slices();
  const int grid = (int)(slices < 4LL * num_sms ? slices : 4LL * num_sms);
  cudaError_t e;
  if (k.d == 64) {
    e = cudaFuncSetAttribute(spectral_generic_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             GenSmem<64>::BYTES);
    if (e != cudaSuccess) return e;
    spectral_generic_kernel<64><<<grid, kGenThreads, GenSmem<64>::BYTES, st>>>(a);
  } else if (k.d == 128) {
    e = cudaFuncSetAttribute(spectral_generic_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             GenSmem<128>::BYTES);
    if (e != cudaSuccess) return e;
    spectral_generic_kernel<128><<<grid, kGenThreads, GenSmem<128>::BYTES, st>>>(a);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace cg
