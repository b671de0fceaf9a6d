// C ABI of libcg (declared in include/cg.h): argument validation, buffer
// sizes, kernel dispatch and the device status word.
#include <atomic>
#include <cstring>

#include "cg_kernels.cuh"

namespace cg {
__device__ unsigned int g_status = 0;
}

using namespace cg;

namespace {
bool valid_bits(int b) { return b == 2 || b == 3 || b == 4 || b == 6 || b == 8; }
}  // namespace

namespace cg {

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

cg_status check_kv(const cg_kv_desc* kv) {
  if (!kv) return CG_ERR_INVALID;
  if (kv->layers <= 0 || kv->batch <= 0 || kv->heads <= 0 || kv->tokens <= 0 || kv->d_head <= 0) return CG_ERR_INVALID;
  if (kv->tokens % 32 != 0) return CG_ERR_INVALID;
  if (kv->d_head != 64 && kv->d_head != 128) return CG_ERR_UNSUPPORTED;
  return CG_OK;
}

cg_status check_codec(const cg_kv_desc* kv, const cg_codec_desc* c) {
  cg_status st = check_kv(kv);
  if (st != CG_OK) return st;
  if (!c) return CG_ERR_INVALID;
  const int d = kv->d_head;
  if (c->g <= 0 || d % c->g != 0) return CG_ERR_INVALID;
  if (c->g != 8 && c->g != 16 && c->g != 32 && c->g != d) return CG_ERR_UNSUPPORTED;
  if (!valid_bits(c->bits)) return CG_ERR_UNSUPPORTED;
  if (c->mode == CG_QUANT_BLOCK_UNIFORM) {
    if (c->tb != 16) return CG_ERR_UNSUPPORTED;
    if (c->range_cols <= 0 || c->range_cols % c->g != 0 || d % c->range_cols != 0) return CG_ERR_INVALID;
    if (c->range_cols != c->g && c->range_cols != d) return CG_ERR_UNSUPPORTED;
  } else if (c->mode == CG_QUANT_KIVI) {
    if (c->kivi_key_tokens != 32 || c->kivi_val_channels != 32) return CG_ERR_UNSUPPORTED;
    if (c->g > 32) return CG_ERR_UNSUPPORTED;
  } else {
    return CG_ERR_INVALID;
  }
  if (c->engine != CG_ENGINE_AUTO && c->engine != CG_ENGINE_CUDA_CORES && c->engine != CG_ENGINE_CHAIN_TENSOR)
    return CG_ERR_INVALID;
  if (c->engine == CG_ENGINE_CUDA_CORES && c->g == d) return CG_ERR_UNSUPPORTED;
  if (c->engine == CG_ENGINE_CHAIN_TENSOR &&
      !(c->g == 16 && d == 128 && c->mode == CG_QUANT_BLOCK_UNIFORM && c->range_cols == 16))
    return CG_ERR_UNSUPPORTED;
  return CG_OK;
}

}  // namespace cg

namespace {

cg_status check_range(const cg_kv_desc* kv, const cg_codec_desc* c, int t0, int nt) {
  const int step = c->mode == CG_QUANT_KIVI ? 32 : c->tb;
  if (t0 < 0 || nt < 0 || (long long)t0 + nt > kv->tokens) return CG_ERR_INVALID;
  if (t0 % step != 0 || nt % step != 0) return CG_ERR_INVALID;
  return CG_OK;
}


KvGeom geom(const cg_kv_desc* kv) { return KvGeom{kv->layers, kv->batch, kv->heads, kv->tokens, kv->d_head}; }

thread_local cudaError_t t_last_cuda = cudaSuccess;

// Device address of the status word on the current device (looked up once
// per device; a host-side symbol is not a device address).
// The status word's device address on the current device, looked up once per device.
// Concurrent first calls from several host threads may each look it up; they store the
// same value, and the atomics make that well defined.
unsigned int* status_word() {
  static std::atomic<unsigned int*> addr[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  unsigned int* a = addr[dev].load(std::memory_order_acquire);
  if (!a) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, cg::g_status) != cudaSuccess) return nullptr;
    a = (unsigned int*)p;
    addr[dev].store(a, std::memory_order_release);
  }
  return a;
}

}  // namespace

namespace cg {
int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    n = 0;
  return n > 0 ? n : 148;
}

cg_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return CG_OK;
  t_last_cuda = e;
  return CG_ERR_CUDA;
}

// Device address of the status word (for entry points defined in other files).
unsigned int* device_status_word() { return status_word(); }

// Descriptor checks shared by the spectral-statistics entry points.
cg_status validate_stats(const cg_kv_desc* kv, const cg_stats_desc* st) {
  cg_status s = check_kv(kv);
  if (s != CG_OK) return s;
  if (!st) return CG_ERR_INVALID;
  if (st->tb != 16) return CG_ERR_UNSUPPORTED;
  if (st->g != 0 && st->g != 16) return CG_ERR_UNSUPPORTED;
  if (!(st->tau > 0.0f)) return CG_ERR_INVALID;
  return CG_OK;
}
}  // namespace cg

extern "C" {

cg_status cg_sizes_for(const cg_kv_desc* kv, const cg_codec_desc* codec, cg_sizes* out) {
  cg_status st = check_codec(kv, codec);
  if (st != CG_OK) return st;
  if (!out) return CG_ERR_INVALID;
  const uint64_t heads = (uint64_t)kv->layers * 2 * kv->batch * kv->heads;
  const uint64_t n = heads * kv->tokens * kv->d_head;
  out->code_bytes = n * codec->bits / 8;
  if (codec->mode == CG_QUANT_BLOCK_UNIFORM)
    out->scale_count = heads * (kv->tokens / codec->tb) * (kv->d_head / codec->range_cols);
  else
    out->scale_count = n / 32;
  return CG_OK;
}

cg_status cg_gauge_build(const float* A_dev, float* G_dev, int32_t n_mats, int32_t g, void* stream) {
  if (n_mats < 0 || g < 2 || g > 128) return CG_ERR_INVALID;
  if (n_mats == 0) return CG_OK;
  if (!A_dev || !G_dev || !aligned16(A_dev) || !aligned16(G_dev) || A_dev == G_dev) return CG_ERR_INVALID;
  return from_cuda(launch_gauge_build(A_dev, G_dev, n_mats, g, (cudaStream_t)stream));
}

cg_status cg_gauge_grad(const float* A_dev, const float* dG_dev, float* dA_dev, int32_t n_mats, int32_t g,
                        void* stream) {
  if (n_mats < 0 || g < 2 || g > 128) return CG_ERR_INVALID;
  if (g > 32) return CG_ERR_UNSUPPORTED;
  if (n_mats == 0) return CG_OK;
  if (!A_dev || !dG_dev || !dA_dev || !aligned16(A_dev) || !aligned16(dG_dev) || !aligned16(dA_dev)) return CG_ERR_INVALID;
  if (dA_dev == A_dev || dA_dev == dG_dev) return CG_ERR_INVALID;
  return from_cuda(launch_gauge_grad(A_dev, dG_dev, dA_dev, n_mats, g, (cudaStream_t)stream));
}

cg_status cg_adamw_step(float* param_dev, const float* grad_dev, float* m_dev, float* v_dev, int64_t n,
                        const cg_adamw_desc* hp, int32_t step, void* stream) {
  if (n < 0 || !hp || step < 1) return CG_ERR_INVALID;
  if (!(hp->lr >= 0.0f) || !(hp->beta1 >= 0.0f && hp->beta1 < 1.0f) || !(hp->beta2 >= 0.0f && hp->beta2 < 1.0f) ||
      !(hp->eps > 0.0f) || !(hp->weight_decay >= 0.0f))
    return CG_ERR_INVALID;
  if (n == 0) return CG_OK;
  if (!param_dev || !grad_dev || !m_dev || !v_dev) return CG_ERR_INVALID;
  if (!aligned16(param_dev) || !aligned16(grad_dev) || !aligned16(m_dev) || !aligned16(v_dev)) return CG_ERR_INVALID;
  return from_cuda(launch_adamw(param_dev, grad_dev, m_dev, v_dev, n, hp->lr, hp->beta1, hp->beta2, hp->eps,
                                hp->weight_decay, step, num_sms(), (cudaStream_t)stream));
}

cg_status cg_group_gram(const cg_kv_desc* kv, int32_t g, const void* kv_dev, int32_t t0, int32_t nt, double* gram_dev,
                        void* stream) {
  cg_status st = check_kv(kv);
  if (st != CG_OK) return st;
  if (g <= 0 || kv->d_head % g != 0) return CG_ERR_INVALID;
  if (g != 8 && g != 16 && g != 32) return CG_ERR_UNSUPPORTED;
  if (t0 < 0 || nt < 0 || (long long)t0 + nt > kv->tokens) return CG_ERR_INVALID;
  if (!kv_dev || !gram_dev || !aligned16(kv_dev) || !aligned16(gram_dev)) return CG_ERR_INVALID;
  return from_cuda(launch_gram(geom(kv), g, (const uint16_t*)kv_dev, gram_dev, t0, nt, (cudaStream_t)stream));
}

cg_status cg_encode(const cg_kv_desc* kv, const cg_codec_desc* codec, const void* kv_dev, const float* G_dev, int32_t t0,
                    int32_t nt, uint8_t* codes_dev, void* scales_dev, void* zeros_dev, float* gauged_dev, void* stream) {
  cg_status st = check_codec(kv, codec);
  if (st != CG_OK) return st;
  st = check_range(kv, codec, t0, nt);
  if (st != CG_OK) return st;
  if (!kv_dev || !G_dev || !codes_dev || !scales_dev || !zeros_dev) return CG_ERR_INVALID;
  if (!aligned16(kv_dev) || !aligned16(G_dev) || !aligned16(codes_dev) || !aligned16(scales_dev) ||
      !aligned16(zeros_dev) || (gauged_dev && !aligned16(gauged_dev)))
    return CG_ERR_INVALID;
  if (nt == 0) return CG_OK;
  CodecArgs a;
  std::memset(&a, 0, sizeof(a));
  a.k = geom(kv);
  a.g = codec->g;
  a.bits = codec->bits;
  a.W = codec->range_cols;
  a.kivi = codec->mode == CG_QUANT_KIVI;
  a.t0 = t0;
  a.nt = nt;
  a.kv = (const uint16_t*)kv_dev;
  a.G = G_dev;
  a.codes = codes_dev;
  a.scales = (uint16_t*)scales_dev;
  a.zeros = (uint16_t*)zeros_dev;
  a.gauged = gauged_dev;
  a.status = status_word();
  if (!a.status) return CG_ERR_CUDA;
  if (a.kivi) {
    if (codec->engine == CG_ENGINE_AUTO && kivi_mma16_supported(a))
      return from_cuda(launch_kivi_mma16(a, num_sms(), (cudaStream_t)stream));
    return from_cuda(launch_kivi(a, true, num_sms(), (cudaStream_t)stream));
  }
  if (a.g == kv->d_head) {
    if (kv->d_head != 128) return CG_ERR_UNSUPPORTED;
    return from_cuda(launch_fullhead(a, true, num_sms(), (cudaStream_t)stream));
  }
  if (codec->engine == CG_ENGINE_CHAIN_TENSOR) return from_cuda(launch_encode_tc16(a, num_sms(), (cudaStream_t)stream));
  if (codec->engine == CG_ENGINE_AUTO && codec_mma16_supported(a))
    return from_cuda(launch_encode_mma16(a, num_sms(), (cudaStream_t)stream));
  if (a.g == 16) return from_cuda(launch_encode_g16(a, num_sms(), (cudaStream_t)stream));
  return from_cuda(launch_group_codec(a, true, num_sms(), (cudaStream_t)stream));
}

cg_status cg_decode(const cg_kv_desc* kv, const cg_codec_desc* codec, const uint8_t* codes_dev, const void* scales_dev,
                    const void* zeros_dev, const float* G_dev, int32_t t0, int32_t nt, void* kv_out_dev, void* stream) {
  cg_status st = check_codec(kv, codec);
  if (st != CG_OK) return st;
  st = check_range(kv, codec, t0, nt);
  if (st != CG_OK) return st;
  if (!codes_dev || !scales_dev || !zeros_dev || !G_dev || !kv_out_dev) return CG_ERR_INVALID;
  if (!aligned16(codes_dev) || !aligned16(scales_dev) || !aligned16(zeros_dev) || !aligned16(G_dev) ||
      !aligned16(kv_out_dev))
    return CG_ERR_INVALID;
  if (nt == 0) return CG_OK;
  CodecArgs a;
  std::memset(&a, 0, sizeof(a));
  a.k = geom(kv);
  a.g = codec->g;
  a.bits = codec->bits;
  a.W = codec->range_cols;
  a.kivi = codec->mode == CG_QUANT_KIVI;
  a.t0 = t0;
  a.nt = nt;
  a.G = G_dev;
  a.codes_in = codes_dev;
  a.scales_in = (const uint16_t*)scales_dev;
  a.zeros_in = (const uint16_t*)zeros_dev;
  a.kv_out = (uint16_t*)kv_out_dev;
  a.status = status_word();
  if (!a.status) return CG_ERR_CUDA;
  if (a.kivi && kivi_decode_g16_supported(a)) return from_cuda(launch_kivi_decode_g16(a, num_sms(), (cudaStream_t)stream));
  if (a.kivi) return from_cuda(launch_kivi(a, false, num_sms(), (cudaStream_t)stream));
  if (a.g == kv->d_head) {
    if (kv->d_head != 128) return CG_ERR_UNSUPPORTED;
    return from_cuda(launch_fullhead(a, false, num_sms(), (cudaStream_t)stream));
  }
  if (codec_mma16_supported(a)) return from_cuda(launch_decode_mma16(a, num_sms(), (cudaStream_t)stream));
  if (a.g == 16) return from_cuda(launch_decode_g16(a, num_sms(), (cudaStream_t)stream));
  return from_cuda(launch_group_codec(a, false, num_sms(), (cudaStream_t)stream));
}


namespace {
cg_status check_attn(const cg_kv_desc* kv, const cg_attn_desc* at) {
  cg_status s = check_kv(kv);
  if (s != CG_OK) return s;
  if (!at) return CG_ERR_INVALID;
  if (at->q_heads <= 0 || at->q_heads % kv->heads != 0) return CG_ERR_INVALID;
  const int gq = at->q_heads / kv->heads;
  if (gq != 1 && gq != 2 && gq != 4 && gq != 8) return CG_ERR_UNSUPPORTED;
  if (at->n_tokens < 16 || at->n_tokens > kv->tokens || at->n_tokens % 16 != 0) return CG_ERR_INVALID;
  if (at->layer0 < 0 || at->n_layers < 1 || (long long)at->layer0 + at->n_layers > kv->layers) return CG_ERR_INVALID;
  if (!(at->scale > 0.0f) || !(at->scale < 3.0e38f)) return CG_ERR_INVALID;
  return CG_OK;
}
}  // namespace

cg_status cg_decode_attention_workspace_size(const cg_kv_desc* kv, const cg_attn_desc* at, uint64_t* bytes) {
  cg_status s = check_attn(kv, at);
  if (s != CG_OK) return s;
  if (!bytes) return CG_ERR_INVALID;
  *bytes = attn_workspace_bytes(geom(kv), at->q_heads, at->n_layers, at->n_tokens);
  return CG_OK;
}

cg_status cg_decode_attention(const cg_kv_desc* kv, const cg_codec_desc* codec, const cg_attn_desc* at,
                              const void* q_dev, const uint8_t* codes_dev, const void* scales_dev,
                              const void* zeros_dev, const float* G_dev, float* out_dev, void* workspace_dev,
                              uint64_t workspace_bytes, void* stream) {
  cg_status s = check_codec(kv, codec);
  if (s != CG_OK) return s;
  s = check_attn(kv, at);
  if (s != CG_OK) return s;
  if (codec->mode != CG_QUANT_BLOCK_UNIFORM || codec->g != 16 || codec->range_cols != 16) return CG_ERR_UNSUPPORTED;
  if (!q_dev || !codes_dev || !scales_dev || !zeros_dev || !G_dev || !out_dev || !workspace_dev) return CG_ERR_INVALID;
  if (!aligned16(q_dev) || !aligned16(codes_dev) || !aligned16(scales_dev) || !aligned16(zeros_dev) ||
      !aligned16(G_dev) || !aligned16(out_dev) || !aligned16(workspace_dev))
    return CG_ERR_INVALID;
  if (workspace_bytes < attn_workspace_bytes(geom(kv), at->q_heads, at->n_layers, at->n_tokens)) return CG_ERR_INVALID;
  AttnArgs a;
  std::memset(&a, 0, sizeof(a));
  a.k = geom(kv);
  a.bits = codec->bits;
  a.hq = at->q_heads;
  a.n_tokens = at->n_tokens;
  a.l0 = at->layer0;
  a.n_layers = at->n_layers;
  a.scale = at->scale;
  a.q = (const uint16_t*)q_dev;
  a.codes = codes_dev;
  a.scales = (const uint16_t*)scales_dev;
  a.zeros = (const uint16_t*)zeros_dev;
  a.G = G_dev;
  a.out = out_dev;
  a.partial = (float*)workspace_dev;
  return from_cuda(launch_decode_attention(a, num_sms(), (cudaStream_t)stream));
}

cg_status cg_spectral_workspace_size(const cg_kv_desc* kv, const cg_stats_desc* st, int32_t want_grad, uint64_t* bytes) {
  cg_status s = cg::validate_stats(kv, st);
  if (s != CG_OK) return s;
  if (!bytes) return CG_ERR_INVALID;
  *bytes = spectral_workspace_bytes(geom(kv), want_grad != 0);
  return CG_OK;
}

cg_status cg_spectral_stats(const cg_kv_desc* kv, const cg_stats_desc* st, const void* x_dev, const float* G_dev,
                            float* lfreq_dev, float* lrate_dev, double* totals_dev, float* dG_dev, void* workspace_dev,
                            uint64_t workspace_bytes, void* stream) {
  cg_status s = cg::validate_stats(kv, st);
  if (s != CG_OK) return s;
  if (!x_dev || !lfreq_dev || !lrate_dev || !totals_dev) return CG_ERR_INVALID;
  if ((G_dev == nullptr) != (st->g == 0)) return CG_ERR_INVALID;
  if (dG_dev && !G_dev) return CG_ERR_INVALID;
  if (!aligned16(x_dev) || !aligned16(lfreq_dev) || !aligned16(lrate_dev) || !aligned16(totals_dev) ||
      (G_dev && !aligned16(G_dev)) || (dG_dev && !aligned16(dG_dev)))
    return CG_ERR_INVALID;
  const uint64_t need = spectral_workspace_bytes(geom(kv), dG_dev != nullptr);
  if (workspace_bytes < need || (need && (!workspace_dev || !aligned16(workspace_dev)))) return CG_ERR_INVALID;
  unsigned int* status = status_word();
  if (!status) return CG_ERR_CUDA;
  return from_cuda(launch_spectral(geom(kv), st->x_is_fp32, x_dev, G_dev, st->lambda_f, st->lambda_r, st->tau, lfreq_dev,
                                   lrate_dev, totals_dev, dG_dev, workspace_dev, status, num_sms(), (cudaStream_t)stream));
}

cg_status cg_sync_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return from_cuda(e);
  unsigned int flag = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&flag, cg::g_status, sizeof(flag));
  if (e != cudaSuccess) return from_cuda(e);
  if (flag) {
    e = cudaMemcpyToSymbol(cg::g_status, &zero, sizeof(zero));
    if (e != cudaSuccess) return from_cuda(e);
    return (flag & cg::kStatusTimeout) ? CG_ERR_TIMEOUT : CG_ERR_BOUND;
  }
  return CG_OK;
}

const char* cg_last_cuda_error(void) {
  if (t_last_cuda == cudaSuccess) return "";
  return cudaGetErrorString(t_last_cuda);
}

const char* cg_status_string(cg_status s) {
  switch (s) {
    case CG_OK: return "ok";
    case CG_ERR_INVALID: return "invalid argument";
    case CG_ERR_UNSUPPORTED: return "unsupported configuration";
    case CG_ERR_CUDA: return "CUDA error";
    case CG_ERR_TIMEOUT: return "device wait timed out";
    case CG_ERR_BOUND: return "tensor-core error bound exceeded";
    case CG_ERR_TOO_LARGE: return "request exceeds the built-in scratch size";
  }
  return "unknown status";
}

int32_t cg_version(void) { return 100; }

}  // extern "C"
