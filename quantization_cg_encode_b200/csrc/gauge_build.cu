// G = exp(A - A^T) for many small matrices: one thread block per matrix.
//
// Codec-Gauge, Method (gauge parameterization): the gauge is the matrix
// exponential of the skew-symmetric A - A^T, hence orthogonal without any
// penalty term.  Scaling and squaring with a Taylor core (Higham, "The scaling
// and squaring method for the matrix exponential revisited", 2005): choose s
// with ||S / 2^s||_1 <= 1/2, evaluate the degree-14 Taylor polynomial of
// S / 2^s (truncation below 0.5^15 / 15! ~ 2e-17), square s times.  Matrices up to g = 64 are computed in fp64 and rounded once to fp32; their
// products run on the fp64 tensor cores (mma.sync m8n8k4).
// Above g = 64 three fp64 matrices do not fit in shared memory: the accumulator E
// stays fp64 there, the scaled skew matrix is held in fp32 (one rounding, about
// 6e-8 relative per entry), and each product is accumulated in fp64 registers
// (a 4 x 8 tile per thread) before it overwrites E, so no product scratch is
// needed.
#include "cg_kernels.cuh"

namespace cg {

namespace {
constexpr int kBuildThreads = 256;
constexpr int kTaylorDegree = 14;

// Row pitch (doubles) of an n x n matrix in shared memory, n % 8 == 0: a pitch of 4 mod 16
// puts the eight rows of a fragment on disjoint bank ranges (two wavefronts per load).
__host__ __device__ constexpr int mat_pitch(int n) { return n + ((4 - n) % 16 + 16) % 16; }

// C = A B for n x n fp64 matrices in shared memory (row pitch p, n % 8 == 0) on the fp64
// tensor cores: mma.sync m8n8k4, each warp taking 8 x 8 tiles of C in turn.  Fragments:
// A row lane / 4, column lane % 4; B row lane % 4, column lane / 4; C row lane / 4,
// columns 2 (lane % 4) and 2 (lane % 4) + 1.
__device__ void smem_matmul(const double* A, const double* B, double* C, int n, int p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int tn = n >> 3, nt = tn * tn, r = lane >> 2, c = lane & 3;
  for (int t0 = warp; t0 < nt; t0 += 2 * nw) {  // two tiles at a time: two independent MMA chains
    const int t1 = t0 + nw < nt ? t0 + nw : t0;
    const double* a0 = A + (8 * (t0 / tn) + r) * p + c;
    const double* b0 = B + c * p + 8 * (t0 % tn) + r;
    const double* a1 = A + (8 * (t1 / tn) + r) * p + c;
    const double* b1 = B + c * p + 8 * (t1 % tn) + r;
    double d0 = 0.0, d1 = 0.0, e0 = 0.0, e1 = 0.0;
    if (t1 != t0) {
      for (int k = 0; k < n; k += 4) {
        asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
                     : "+d"(d0), "+d"(d1)
                     : "d"(a0[k]), "d"(b0[k * p]));
        asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
                     : "+d"(e0), "+d"(e1)
                     : "d"(a1[k]), "d"(b1[k * p]));
      }
    } else {
      for (int k = 0; k < n; k += 4)
        asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
                     : "+d"(d0), "+d"(d1)
                     : "d"(a0[k]), "d"(b0[k * p]));
    }
    double* c0 = C + (8 * (t0 / tn) + r) * p + 8 * (t0 % tn) + 2 * c;
    c0[0] = d0;
    c0[1] = d1;
    if (t1 != t0) {
      double* c1 = C + (8 * (t1 / tn) + r) * p + 8 * (t1 % tn) + 2 * c;
      c1[0] = e0;
      c1[1] = e1;
    }
  }
}

// 1 / k! for k = 0 .. 14, and 0 for k = 15 (the Taylor core has degree 14)
struct InvFact {
  double v[16];
};
constexpr InvFact make_inv_fact() {
  InvFact f{};
  double x = 1.0;
  for (int k = 0; k < 15; ++k) {
    if (k > 0) x /= (double)k;
    f.v[k] = x;
  }
  f.v[15] = 0.0;
  return f;
}
__constant__ InvFact kInvFact = make_inv_fact();

// E = exp(M) for the n x n matrix M in shared memory (row pitch p; M is overwritten by
// its scaled copy X; X2, X3, X4 and W are scratch).  Scaling and squaring with the
// degree-14 Taylor core evaluated by Paterson and Stockmeyer's scheme ("On the number of
// nonscalar multiplications necessary to evaluate polynomials", 1973): with the powers
// X^2, X^3, X^4, p(X) = B0 + X^4 (B1 + X^4 (B2 + X^4 B3)), B_j = sum_i X^i / (4 j + i)!,
// so six products instead of the fourteen of Horner's rule.
__device__ void expm_smem(double* M, double* E, double* W, double* X2, double* X3, double* X4, int n, int p,
                          double* colsum, int* s_shift) {
  // ||M||_1 = max column sum of |M|
  for (int j = threadIdx.x; j < n; j += blockDim.x) {
    double acc = 0;
    for (int i = 0; i < n; ++i) acc += fabs(M[i * p + j]);
    colsum[j] = acc;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double nrm = 0;
    for (int j = 0; j < n; ++j) nrm = colsum[j] > nrm ? colsum[j] : nrm;
    int s = 0;
    while (nrm > 0.5) {
      nrm *= 0.5;
      ++s;
    }
    *s_shift = s;
  }
  __syncthreads();
  const int s = *s_shift;
  const double scale = ldexp(1.0, -s);
  for (int e = threadIdx.x; e < n * n; e += blockDim.x) {
    const int i = e / n, j = e % n;
    M[i * p + j] *= scale;
  }
  __syncthreads();
  smem_matmul(M, M, X2, n, p);
  __syncthreads();
  smem_matmul(X2, M, X3, n, p);
  smem_matmul(X2, X2, X4, n, p);
  __syncthreads();
  // E = B3, then E = B_j + X^4 E for j = 2, 1, 0
#pragma unroll
  for (int j = 3; j >= 0; --j) {
    if (j < 3) {
      smem_matmul(X4, E, W, n, p);
      __syncthreads();
    }
    const double c0 = kInvFact.v[4 * j], c1 = kInvFact.v[4 * j + 1], c2 = kInvFact.v[4 * j + 2], c3 = kInvFact.v[4 * j + 3];
    for (int e = threadIdx.x; e < n * n; e += blockDim.x) {
      const int r = e / n, c = e % n, o = r * p + c;
      double v = c1 * M[o] + c2 * X2[o] + c3 * X3[o] + (r == c ? c0 : 0.0);
      if (j < 3) v += W[o];
      E[o] = v;
    }
    __syncthreads();
  }
  for (int q = 0; q < s; ++q) {
    smem_matmul(E, E, W, n, p);
    __syncthreads();
    for (int e = threadIdx.x; e < n * n; e += blockDim.x) {
      const int i = e / n, j = e % n;
      E[i * p + j] = W[i * p + j];
    }
    __syncthreads();
  }
}

// g <= 64: fp64 in shared memory throughout; S is embedded as diag(S, 0) in n x n with n
// the next multiple of 8 (exp(diag(S, 0)) = diag(exp(S), I)).
__global__ void __launch_bounds__(kBuildThreads, 4) gauge_build_kernel(const float* __restrict__ Ain, float* __restrict__ Gout, int g) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int n = (g + 7) & ~7, p = mat_pitch(n);
  double* M = reinterpret_cast<double*>(smem_raw);  // scaled skew matrix
  double* E = M + n * p;                            // polynomial accumulator / result
  double* W = E + n * p;                            // product scratch, then the powers of M
  double* X2 = W + n * p;
  double* X3 = X2 + n * p;
  double* X4 = X3 + n * p;
  __shared__ double colsum[128];
  __shared__ int s_shift;

  const long long base = (long long)blockIdx.x * g * g;
  const float* A = Ain + base;
  for (int e = threadIdx.x; e < n * n; e += blockDim.x) {
    const int i = e / n, j = e % n;
    M[i * p + j] = (i < g && j < g) ? (double)A[i * g + j] - (double)A[j * g + i] : 0.0;
  }
  __syncthreads();
  expm_smem(M, E, W, X2, X3, X4, n, p, colsum, &s_shift);
  float* G = Gout + base;
  for (int e = threadIdx.x; e < g * g; e += blockDim.x) G[e] = (float)E[(e / g) * p + e % g];
}

// 64 < g <= 128: one 512-thread block per matrix, embedded in 128 x 128 as
// diag(S, 0) (whose exponential is diag(exp(S), I)); thread t owns rows
// 4 (t / 16) .. + 3 and columns 8 (t % 16) .. + 7 of every product.
constexpr int kG128 = 128, kG128Threads = 512;
constexpr size_t kG128Smem = (size_t)kG128 * kG128 * (sizeof(double) + sizeof(float));

// acc = X E for the 4 x 8 tile of this thread, X fp32 (Xf) or fp64 (Xd).
template <typename TX>
__device__ __forceinline__ void tile_product(const TX* X, const double* E, int r0, int c0, double (&acc)[4][8]) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0;
#pragma unroll 2
  for (int k = 0; k < kG128; ++k) {
    double xv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) xv[i] = (double)X[(r0 + i) * kG128 + k];
    const double2* er = reinterpret_cast<const double2*>(E + k * kG128 + c0);
    double ev[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const double2 t = er[q];
      ev[2 * q] = t.x;
      ev[2 * q + 1] = t.y;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = fma(xv[i], ev[j], acc[i][j]);
  }
}

__global__ void __launch_bounds__(kG128Threads) gauge_build_g128_kernel(const float* __restrict__ Ain, float* __restrict__ Gout,
                                                                         int g) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  double* E = reinterpret_cast<double*>(smem_raw);          // fp64 accumulator / result
  float* M = reinterpret_cast<float*>(E + kG128 * kG128);   // S / 2^s, fp32
  __shared__ double colsum[kG128];
  __shared__ int s_shift;
  constexpr int n = kG128;
  const long long base = (long long)blockIdx.x * g * g;
  const float* A = Ain + base;
  // ||S||_1 in fp64, S = A - A^T
  for (int j = threadIdx.x; j < n; j += blockDim.x) {
    double acc = 0.0;
    if (j < g)
      for (int i = 0; i < g; ++i) acc += fabs((double)A[i * g + j] - (double)A[j * g + i]);
    colsum[j] = acc;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double nrm = 0.0;
    for (int j = 0; j < n; ++j) nrm = fmax(nrm, colsum[j]);
    int s = 0;
    while (nrm > 0.5) {
      nrm *= 0.5;
      ++s;
    }
    s_shift = s;
  }
  __syncthreads();
  const int s = s_shift;
  const double scale = ldexp(1.0, -s);
  for (int e = threadIdx.x; e < n * n; e += blockDim.x) {
    const int i = e / n, j = e % n;
    M[e] = (i < g && j < g) ? (float)(((double)A[i * g + j] - (double)A[j * g + i]) * scale) : 0.0f;
    E[e] = i == j ? 1.0 : 0.0;
  }
  __syncthreads();
  const int r0 = 4 * (threadIdx.x / 16), c0 = 8 * (threadIdx.x % 16);
  double acc[4][8];
  // Horner: E = I + M E / k for k = degree .. 1
  for (int k = kTaylorDegree; k >= 1; --k) {
    tile_product(M, E, r0, c0, acc);
    __syncthreads();  // every read of E is done before it is overwritten
    const double rk = 1.0 / (double)k;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) E[(r0 + i) * n + c0 + j] = (r0 + i == c0 + j ? 1.0 : 0.0) + acc[i][j] * rk;
    __syncthreads();
  }
  for (int q = 0; q < s; ++q) {  // squaring
    tile_product(E, E, r0, c0, acc);
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) E[(r0 + i) * n + c0 + j] = acc[i][j];
    __syncthreads();
  }
  float* G = Gout + base;
  for (int e = threadIdx.x; e < g * g; e += blockDim.x) G[e] = (float)E[(e / g) * n + e % g];
}

// dL/dA for G = exp(S), S = A - A^T, from dL/dG, one matrix per thread block, in
// fp64.  The adjoint of the Frechet derivative E -> L_exp(S, E) is
// F -> L_exp(S^T, F) (Higham, Functions of Matrices, 2008, section 10.6), and
// L_exp(X, F) is the upper-right block of exp([[X, F], [0, X]]) (Van Loan,
// "Computing integrals involving the matrix exponential", 1978).  So
// dS = L_exp(S^T, dG) and dA = dS - dS^T.  L_exp is linear in F: dG is scaled
// to max |dG| = 2^-30 before the exponential and the result scaled back (exact
// powers of two), so the block's norm, and with it the number of squarings, is
// that of S; the upper-right block's truncation error stays relative to |dG|.
__global__ void __launch_bounds__(kBuildThreads, 4) gauge_grad_kernel(const float* __restrict__ Ain,
                                                                   const float* __restrict__ dGin,
                                                                   float* __restrict__ dAout, int g) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int n = (2 * g + 7) & ~7, p = mat_pitch(n);  // diag(block, 0) when 2 g is not a multiple of 8
  double* M = reinterpret_cast<double*>(smem_raw);
  double* E = M + n * p;
  double* W = E + n * p;
  double* X2 = W + n * p;
  double* X3 = X2 + n * p;
  double* X4 = X3 + n * p;
  __shared__ double colsum[64];
  __shared__ double dgmax[kBuildThreads / 32];
  __shared__ int s_shift;
  const long long base = (long long)blockIdx.x * g * g;
  const float* A = Ain + base;
  const float* dG = dGin + base;
  double mloc = 0.0;
  for (int e = threadIdx.x; e < g * g; e += blockDim.x) mloc = fmax(mloc, fabs((double)dG[e]));
  for (int o = 16; o >= 1; o >>= 1) mloc = fmax(mloc, __shfl_xor_sync(0xffffffffu, mloc, o));
  if ((threadIdx.x & 31) == 0) dgmax[threadIdx.x >> 5] = mloc;
  __syncthreads();
  double c = 0.0;
  for (int w = 0; w < kBuildThreads / 32; ++w) c = fmax(c, dgmax[w]);
  const double inv_c = c > 0.0 ? ldexp(1.0 / c, -30) : 0.0;
  // M = [[S^T, dG / c], [0, S^T]] with S^T[i][j] = A[j][i] - A[i][j]
  for (int e = threadIdx.x; e < n * n; e += blockDim.x) {
    const int i = e / n, j = e % n;
    double v = 0.0;
    if (i < g && j < g) v = (double)A[j * g + i] - (double)A[i * g + j];
    else if (i >= 2 * g || j >= 2 * g) v = 0.0;
    else if (i >= g && j >= g) v = (double)A[(j - g) * g + (i - g)] - (double)A[(i - g) * g + (j - g)];
    else if (i < g && j >= g) v = (double)dG[i * g + (j - g)] * inv_c;
    M[i * p + j] = v;
  }
  __syncthreads();
  expm_smem(M, E, W, X2, X3, X4, n, p, colsum, &s_shift);
  float* dA = dAout + base;
  for (int e = threadIdx.x; e < g * g; e += blockDim.x) {
    const int i = e / g, j = e % g;
    dA[e] = (float)(ldexp(c, 30) * (E[i * p + g + j] - E[j * p + g + i]));
  }
}
}  // namespace

cudaError_t launch_gauge_grad(const float* A, const float* dG, float* dA, int n_mats, int g, cudaStream_t st) {
  if (n_mats == 0) return cudaSuccess;
  if (g > 32) return cudaErrorInvalidValue;
  const int n = (2 * g + 7) & ~7;
  const size_t smem = 6 * (size_t)n * mat_pitch(n) * sizeof(double);
  cudaError_t e = cudaFuncSetAttribute(gauge_grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  gauge_grad_kernel<<<n_mats, kBuildThreads, smem, st>>>(A, dG, dA, g);
  return cudaGetLastError();
}

cudaError_t launch_gauge_build(const float* A, float* G, int n_mats, int g, cudaStream_t st) {
  if (n_mats == 0) return cudaSuccess;
  if (g <= 64) {
    const int n = (g + 7) & ~7;
    const size_t smem = 6 * (size_t)n * mat_pitch(n) * sizeof(double);
    cudaError_t e = cudaFuncSetAttribute(gauge_build_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    gauge_build_kernel<<<n_mats, kBuildThreads, smem, st>>>(A, G, g);
  } else if (g <= kG128) {
    cudaError_t e = cudaFuncSetAttribute(gauge_build_g128_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kG128Smem);
    if (e != cudaSuccess) return e;
    gauge_build_g128_kernel<<<n_mats, kG128Threads, kG128Smem, st>>>(A, G, g);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace cg
