// G = exp(A - A^T) for many small matrices: one thread block per matrix.
//
// Codec-Gauge, Method (gauge parameterization): the gauge is the matrix
// exponential of the skew-symmetric A - A^T, hence orthogonal without any
// penalty term.  Scaling and squaring with a Taylor core (Higham, "The scaling
// and squaring method for the matrix exponential revisited", 2005): choose s
// with ||S / 2^s||_1 <= 1/2, evaluate the degree-14 Taylor polynomial of
// S / 2^s by Horner's rule (truncation below 0.5^15 / 15! ~ 2e-17), square s
// times.  Matrices up to g = 64 are computed in fp64 and rounded once to fp32;
// g = 128 does not fit three fp64 matrices in shared memory and runs in fp32.
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
  // ||S||_1 = max column sum of |S|
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
    s_shift = s;
  }
  __syncthreads();
  const int s = s_shift;
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
  float* G = Gout + base;
  for (int e = threadIdx.x; e < n * n; e += blockDim.x) G[e] = (float)E[e];
}
}  // namespace

cudaError_t launch_gauge_build(const float* A, float* G, int n_mats, int g, cudaStream_t st) {
  if (n_mats == 0) return cudaSuccess;
  if (g <= 64) {
    const size_t smem = 3 * (size_t)g * g * sizeof(double);
    cudaError_t e = cudaFuncSetAttribute(gauge_build_kernel<double>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    gauge_build_kernel<double><<<n_mats, kBuildThreads, smem, st>>>(A, G, g);
  } else {
    const size_t smem = 3 * (size_t)g * g * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(gauge_build_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    gauge_build_kernel<float><<<n_mats, kBuildThreads, smem, st>>>(A, G, g);
  }
  return cudaGetLastError();
}

}  // namespace cg
