// cg_spectral_stats without a caller workspace, for callers that cannot
// allocate device memory (see include/cg.h): the dL/dG partials go to a scratch
// array compiled into the library.  Nothing here allocates.
#include <mutex>

#include "cg_kernels.cuh"

namespace {

// One dG partial (d_head x g fp32: 8 KiB at d_head = 128, 4 KiB at 64) per
// head slice: 512 slices at d_head = 128, 1024 at 64.
constexpr uint64_t kScratchBytes = 8ull << 20;  // 8 MiB

// Reserved on every device that loads the library, for the life of the process.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device.  The host-side
// symbol is only a stand-in, never a device address, so it is looked up once
// per device with that device current.
cg_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CG_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return CG_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return CG_OK;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

extern "C" cg_status cg_spectral_stats_noalloc(const cg_kv_desc* kv, const cg_stats_desc* st, const void* x_dev,
                                               const float* G_dev, float* lfreq_dev, float* lrate_dev,
                                               double* totals_dev, float* dG_dev, void* stream) {
  cg_status s = cg::validate_stats(kv, st);
  if (s != CG_OK) return s;
  if (!x_dev || !lfreq_dev || !lrate_dev || !totals_dev) return CG_ERR_INVALID;
  if ((G_dev == nullptr) != (st->g == 0)) return CG_ERR_INVALID;
  if (dG_dev && !G_dev) return CG_ERR_INVALID;
  if (!aligned16(x_dev) || !aligned16(lfreq_dev) || !aligned16(lrate_dev) || !aligned16(totals_dev) ||
      (G_dev && !aligned16(G_dev)) || (dG_dev && !aligned16(dG_dev)))
    return CG_ERR_INVALID;
  const cg::KvGeom k{kv->layers, kv->batch, kv->heads, kv->tokens, kv->d_head};
  const uint64_t need = cg::spectral_workspace_bytes(k, dG_dev != nullptr);
  if (need > kScratchBytes) return CG_ERR_TOO_LARGE;
  void* scratch = nullptr;
  if (need) {
    s = scratch_address(&scratch);
    if (s != CG_OK) return s;
  }
  unsigned int* status = cg::device_status_word();
  if (!status) return CG_ERR_CUDA;
  return cg::from_cuda(cg::launch_spectral(k, st->x_is_fp32, x_dev, G_dev, st->lambda_f, st->lambda_r, st->tau,
                                           lfreq_dev, lrate_dev, totals_dev, dG_dev, scratch, status, cg::num_sms(),
                                           (cudaStream_t)stream));
}
