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
constexpr int kGramThreads = 256, kGramWarps = kGramThreads / 32;
constexpr int kGramTok = 32;  // tokens staged per step
}  // namespace

// One thread block per gauge set (l, s, h): sums over the batch and tokens
// [t0, t0 + nt) in a fixed order, on the fp64 tensor cores.  C_r = X_r^T X_r is
// cut into 8 x 8 tiles (i block, j block) of every group r; warp w owns tiles
// w, w + 8, .. and accumulates each with mma.sync m8n8k4 fp64 over 4 tokens per
// step (A = X_r^T: row lane / 4, column lane % 4; B = X_r: row lane % 4, column
// lane / 4; C row lane / 4, columns 2 (lane % 4) + {0, 1}).  bf16 inputs are
// exact in fp64, so every product is exact; a staged step's missing tokens are
// zeros.  The row pitch D + 8 (floats) puts the 4 token rows of a fragment on
// disjoint banks.
template <int D, int G>
__global__ void __launch_bounds__(kGramThreads, 1) gram_kernel(const uint16_t* __restrict__ kv, double* __restrict__ gram,
                                                               KvGeom k, int t0, int nt) {
  constexpr int R = D / G, TN = G / 8, TILES = R * TN * TN, PER = TILES / kGramWarps, P = D + 8;
  constexpr int VEC = kGramTok * D / 8 / kGramThreads;  // 16-byte loads per thread per staged step
  static_assert(PER * kGramWarps == TILES, "tiles divide evenly");
  static_assert(VEC * 8 * kGramThreads == kGramTok * D, "loads divide evenly");
  __shared__ __align__(16) float xs[2][kGramTok][P];
  const int set = blockIdx.x;  // (l * 2 + s) * H + h
  const int h = set % k.H, ls = set / k.H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, lr = lane >> 2, lc = lane & 3;
  int ca[PER], cb[PER];  // fragment columns of this lane: channel of A (row block) and of B (column block)
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    const int t = warp + kGramWarps * q, r = t / (TN * TN), ti = (t / TN) % TN, tj = t % TN;
    ca[q] = r * G + 8 * ti + lr;
    cb[q] = r * G + 8 * tj + lr;
  }
  double acc[PER][2];
#pragma unroll
  for (int q = 0; q < PER; ++q) acc[q][0] = acc[q][1] = 0.0;
  // staged steps: (batch b, 32 tokens from t0 + 32 j), in order; missing tokens read as zeros
  const int nch = (nt + kGramTok - 1) / kGramTok, total = k.B * nch;
  auto fetch = [&](int ci, uint4 (&v)[VEC]) {
    const int b = ci / nch, tt = (ci % nch) * kGramTok, ntok = min(kGramTok, nt - tt);
    const long long slice = ((long long)ls * k.B + b) * k.H + h;
    const uint16_t* x = kv + (slice * k.T + t0 + tt) * D;
#pragma unroll
    for (int j = 0; j < VEC; ++j) {
      const int e = threadIdx.x + kGramThreads * j, t = e / (D / 8), c8 = e % (D / 8);
      v[j] = t < ntok ? __ldg(reinterpret_cast<const uint4*>(x + (long long)t * D) + c8) : make_uint4(0, 0, 0, 0);
    }
  };
  auto stage = [&](const uint4 (&v)[VEC], int buf) {
#pragma unroll
    for (int j = 0; j < VEC; ++j) {
      const int e = threadIdx.x + kGramThreads * j, t = e / (D / 8), c8 = e % (D / 8);
      float4* dst = reinterpret_cast<float4*>(&xs[buf][t][8 * c8]);
      dst[0] = make_float4(bf16lo(v[j].x), bf16hi(v[j].x), bf16lo(v[j].y), bf16hi(v[j].y));
      dst[1] = make_float4(bf16lo(v[j].z), bf16hi(v[j].z), bf16lo(v[j].w), bf16hi(v[j].w));
    }
  };
  if (total > 0) {
    uint4 v[VEC];
    fetch(0, v);
    stage(v, 0);
  }
  __syncthreads();
  for (int ci = 0; ci < total; ++ci) {
    uint4 v[VEC];
    if (ci + 1 < total) fetch(ci + 1, v);  // the next step's loads are in flight during this one
    const int tt = (ci % nch) * kGramTok, steps = (min(kGramTok, nt - tt) + 3) >> 2;
    for (int s4 = 0; s4 < steps; ++s4) {
      const float* row = xs[ci & 1][4 * s4 + lc];
#pragma unroll
      for (int q = 0; q < PER; ++q) {
        const double a = (double)row[ca[q]], bb = (double)row[cb[q]];
        asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
                     : "+d"(acc[q][0]), "+d"(acc[q][1])
                     : "d"(a), "d"(bb));
      }
    }
    if (ci + 1 < total) stage(v, (ci + 1) & 1);
    __syncthreads();
  }
  double* out = gram + (long long)set * R * G * G;
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    const int t = warp + kGramWarps * q, r = t / (TN * TN), ti = (t / TN) % TN, tj = t % TN;
    double* o = out + (r * G + 8 * ti + lr) * G + 8 * tj + 2 * lc;
    o[0] = acc[q][0];
    o[1] = acc[q][1];
  }
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
