// Gauge training and coordinate-control support: the AdamW update of the
// gauge parameters and the per-group second-moment (Gram) matrices of a cache.
//
// Codec-Gauge, Method (gauge training): the gauge parameters are optimized with
// AdamW on the frequency-distribution objective over 4096-token windows.
// AdamW is Loshchilov & Hutter, "Decoupled weight decay regularization"
// (2019), Algorithm 2: m = b1 m + (1 - b1) g, v = b2 v + (1 - b2) g^2,
// p -= lr (m / (1 - b1^t) / (sqrt(v / (1 - b2^t)) + eps) + wd p).
//
// Codec-Gauge, Experimental setup (coordinate controls): PCA/KLT uses the
// uncentered second-moment eigenbasis at the same layer, K/V, head and group
// granularity; the Gram matrices C_r = sum_{b,t} x_{t,r} x_{t,r}^T are summed
// here (fp64, fixed order per gauge set), the eigensolver runs on the host.
#include "cg_kernels.cuh"

namespace cg {

__global__ void adamw_kernel(float* __restrict__ p, const float* __restrict__ grad, float* __restrict__ m,
                             float* __restrict__ v, long long n, float lr, float b1, float b2, float eps, float wd,
                             float inv_bc1, float inv_bc2) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const float gi = grad[i];
    const float mi = __fmaf_rn(b1, m[i], (1.0f - b1) * gi);
    const float vi = __fmaf_rn(b2, v[i], (1.0f - b2) * gi * gi);
    m[i] = mi;
    v[i] = vi;
    const float pi = p[i];
    const float upd = (mi * inv_bc1) / (sqrtf(vi * inv_bc2) + eps);
    p[i] = pi - lr * (upd + wd * pi);
  }
}

cudaError_t launch_adamw(float* p, const float* grad, float* m, float* v, long long n, float lr, float b1, float b2,
                         float eps, float wd, int step, int num_sms, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const double bc1 = 1.0 - pow((double)b1, (double)step), bc2 = 1.0 - pow((double)b2, (double)step);
  const long long blocks = (n + 255) / 256;
  const int grid = (int)(blocks < 8LL * num_sms ? blocks : 8LL * num_sms);
  adamw_kernel<<<grid, 256, 0, st>>>(p, grad, m, v, n, lr, b1, b2, eps, wd, (float)(1.0 / bc1), (float)(1.0 / bc2));
  return cudaGetLastError();
}

namespace {
constexpr int kGramThreads = 256;
constexpr int kGramTok = 32;  // tokens staged per step
}  // namespace

// One thread block per gauge set (l, s, h): sums over the batch and tokens
// [t0, t0 + nt) in order; thread e owns entries e + 256 k of [R][g][g].
template <int D, int G>
__global__ void __launch_bounds__(kGramThreads) gram_kernel(const uint16_t* __restrict__ kv, double* __restrict__ gram,
                                                            KvGeom k, int t0, int nt) {
  constexpr int R = D / G;
  constexpr int PER = R * G * G / kGramThreads;  // entries per thread
  static_assert(PER * kGramThreads == R * G * G, "entries divide evenly");
  __shared__ float xs[kGramTok][D + 1];
  const int set = blockIdx.x;  // (l * 2 + s) * H + h
  const int h = set % k.H, ls = set / k.H;
  double acc[PER];
#pragma unroll
  for (int q = 0; q < PER; ++q) acc[q] = 0.0;
  for (int b = 0; b < k.B; ++b) {
    const long long slice = ((long long)ls * k.B + b) * k.H + h;
    const uint16_t* x = kv + (slice * k.T + t0) * D;
    for (int tt = 0; tt < nt; tt += kGramTok) {
      const int ntok = min(kGramTok, nt - tt);
      __syncthreads();
      for (int e = threadIdx.x; e < ntok * D; e += kGramThreads)
        xs[e / D][e % D] = bf16lo((uint32_t)x[(long long)tt * D + e]);
      __syncthreads();
#pragma unroll
      for (int q = 0; q < PER; ++q) {
        const int e = threadIdx.x + kGramThreads * q;
        const int r = e / (G * G), i = (e / G) % G, j = e % G;
        double a = acc[q];
        for (int t = 0; t < ntok; ++t) a = fma((double)xs[t][r * G + i], (double)xs[t][r * G + j], a);
        acc[q] = a;
      }
    }
  }
#pragma unroll
  for (int q = 0; q < PER; ++q) gram[(long long)set * R * G * G + threadIdx.x + kGramThreads * q] = acc[q];
}

cudaError_t launch_gram(const KvGeom& k, int g, const uint16_t* kv, double* gram, int t0, int nt, cudaStream_t st) {
  const int sets = k.L * 2 * k.H;
  if (sets == 0) return cudaSuccess;
#define CG_GRAM(DD, GG)                                                     \
  if (k.d == DD && g == GG) {                                               \
    gram_kernel<DD, GG><<<sets, kGramThreads, 0, st>>>(kv, gram, k, t0, nt); \
    return cudaGetLastError();                                              \
  }
  CG_GRAM(128, 8) CG_GRAM(128, 16) CG_GRAM(128, 32) CG_GRAM(64, 8) CG_GRAM(64, 16) CG_GRAM(64, 32)
#undef CG_GRAM
  return cudaErrorInvalidValue;
}

}  // namespace cg
