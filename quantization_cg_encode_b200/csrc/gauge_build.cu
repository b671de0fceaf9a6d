// G = exp(A - A^T) for many small matrices: one thread block per matrix.
//
// Codec-Gauge, Method (gauge parameterization): the gauge is the matrix
// exponential of the skew-symmetric A - A^T, hence orthogonal without any
// penalty term.  Scaling and squaring with a Taylor core (Higham, "The scaling
// and squaring method for the matrix exponential revisited", 2005): choose s
// with ||S / 2^s||_1 <= 1/2, evaluate the degree-14 Taylor polynomial of
// S / 2^s by Horner's rule (truncation below 0.5^15 / 15! ~ 2e-17), square s
// times.  Matrices up to g = 64 are computed in fp64 and rounded once to fp32.
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

// C = A * B for n x n row-major matrices in shared memory.
template <typename T>
__device__ void smem_matmul(const T* A, const T* B, T* C, int n) {
  for (int e = threadIdx.x; e < n * n; e += blockDim.x) {
    const int i = e / n, j = e % n;
    T acc = 0;
    for (int k = 0; k < n; ++k) acc += A[i * n + k] * B[k * n + j];
    C[e] = acc;
  }
}

// E = exp(M) for the n x n matrix M in shared memory (M is overwritten by its
// scaled copy; W is scratch).  Scaling and squaring with the Taylor core.
template <typename T>
__device__ void expm_smem(T* M, T* E, T* W, int n, T* colsum, int* s_shift) {
  // ||M||_1 = max column sum of |M|
  for (int j = threadIdx.x; j < n; j += blockDim.x) {
    T acc = 0;
    for (int i = 0; i < n; ++i) acc += fabs(M[i * n + j]);
    colsum[j] = acc;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    T nrm = 0;
    for (int j = 0; j < n; ++j) nrm = colsum[j] > nrm ? colsum[j] : nrm;
    int s = 0;
    while (nrm > (T)0.5) {
      nrm *= (T)0.5;
      ++s;
    }
    *s_shift = s;
  }
  __syncthreads();
  const int s = *s_shift;
  const T scale = (T)ldexp(1.0, -s);
  for (int e = threadIdx.x; e < n * n; e += blockDim.x) {
    M[e] *= scale;
    E[e] = (e / n == e % n) ? (T)1 : (T)0;
  }
  __syncthreads();
  // Horner: E = I + M/k * E for k = degree .. 1
  for (int k = kTaylorDegree; k >= 1; --k) {
    smem_matmul(M, E, W, n);
    __syncthreads();
    const T rk = (T)1 / (T)k;
    for (int e = threadIdx.x; e < n * n; e += blockDim.x) E[e] = ((e / n == e % n) ? (T)1 : (T)0) + W[e] * rk;
    __syncthreads();
  }
  for (int q = 0; q < s; ++q) {
    smem_matmul(E, E, W, n);
    __syncthreads();
    for (int e = threadIdx.x; e < n * n; e += blockDim.x) E[e] = W[e];
    __syncthreads();
  }
}

template <typename T>
__global__ void __launch_bounds__(kBuildThreads) gauge_build_kernel(const float* __restrict__ Ain, float* __restrict__ Gout, int n) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  T* M = reinterpret_cast<T*>(smem_raw);  // scaled skew matrix
  T* E = M + n * n;                        // Horner accumulator / result
  T* W = E + n * n;                        // product scratch
  __shared__ T colsum[128];
  __shared__ int s_shift;

  const long long base = (long long)blockIdx.x * n * n;
  const float* A = Ain + base;
  for (int e = threadIdx.x; e < n * n; e += blockDim.x) {
    const int i = e / n, j = e % n;
    M[e] = (T)A[i * n + j] - (T)A[j * n + i];
  }
  __syncthreads();
  expm_smem(M, E, W, n, colsum, &s_shift);
  float* G = Gout + base;
  for (int e = threadIdx.x; e < n * n; e += blockDim.x) G[e] = (float)E[e];
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
// to max |dG| = 1 before the exponential and the result scaled back, so the
// scaling-and-squaring step count depends on S only.
__global__ void __launch_bounds__(kBuildThreads) gauge_grad_kernel(const float* __restrict__ Ain,
                                                                   const float* __restrict__ dGin,
                                                                   float* __restrict__ dAout, int g) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int n = 2 * g;
  double* M = reinterpret_cast<double*>(smem_raw);
  double* E = M + n * n;
  double* W = E + n * n;
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
  const double inv_c = c > 0.0 ? 1.0 / c : 0.0;
  // M = [[S^T, dG / c], [0, S^T]] with S^T[i][j] = A[j][i] - A[i][j]
  for (int e = threadIdx.x; e < n * n; e += blockDim.x) {
    const int i = e / n, j = e % n;
    double v = 0.0;
    if (i < g && j < g) v = (double)A[j * g + i] - (double)A[i * g + j];
    else if (i >= g && j >= g) v = (double)A[(j - g) * g + (i - g)] - (double)A[(i - g) * g + (j - g)];
    else if (i < g && j >= g) v = (double)dG[i * g + (j - g)] * inv_c;
    M[e] = v;
  }
  __syncthreads();
  expm_smem(M, E, W, n, colsum, &s_shift);
  float* dA = dAout + base;
  for (int e = threadIdx.x; e < g * g; e += blockDim.x) {
    const int i = e / g, j = e % g;
    dA[e] = (float)(c * (E[i * n + g + j] - E[j * n + g + i]));
  }
}
}  // namespace

cudaError_t launch_gauge_grad(const float* A, const float* dG, float* dA, int n_mats, int g, cudaStream_t st) {
  if (n_mats == 0) return cudaSuccess;
  if (g > 32) return cudaErrorInvalidValue;
  const size_t smem = 3 * (size_t)(2 * g) * (2 * g) * sizeof(double);
  cudaError_t e = cudaFuncSetAttribute(gauge_grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  gauge_grad_kernel<<<n_mats, kBuildThreads, smem, st>>>(A, dG, dA, g);
  return cudaGetLastError();
}

cudaError_t launch_gauge_build(const float* A, float* G, int n_mats, int g, cudaStream_t st) {
  if (n_mats == 0) return cudaSuccess;
  if (g <= 64) {
    const size_t smem = 3 * (size_t)g * g * sizeof(double);
    cudaError_t e = cudaFuncSetAttribute(gauge_build_kernel<double>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    gauge_build_kernel<double><<<n_mats, kBuildThreads, smem, st>>>(A, G, g);
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
