// Internal launch interface between the C ABI (cg_abi.cu) and the kernels.
#pragma once
#include "cg_common.cuh"

namespace cg {

// Arguments of one encode or decode call, after host validation.
struct CodecArgs {
  KvGeom k;
  int g, bits, W;          // gauge group, bits per value, block-uniform range width
  int kivi;                // 1: KIVI-style ranges
  int t0, nt;              // token range, multiples of 16 (32 for KIVI)
  const uint16_t* kv;      // bf16 [L][2][B][H][T][d]
  const float* G;          // fp32 [L][2][H][R][g][g]
  uint8_t* codes;
  uint16_t* scales;        // fp16 bits
  uint16_t* zeros;         // fp16 bits
  float* gauged;           // optional fp32 gauged values
  uint16_t* kv_out;        // bf16 reconstruction (decode)
  const uint8_t* codes_in; // decode input
  const uint16_t* scales_in;
  const uint16_t* zeros_in;
  unsigned int* status;     // device status word
};

cudaError_t launch_group_codec(const CodecArgs& a, bool encode, int num_sms, cudaStream_t st);
cudaError_t launch_encode_g16(const CodecArgs& a, int num_sms, cudaStream_t st);
bool encode_tc16_supported(const CodecArgs& a);
cudaError_t launch_encode_tc16(const CodecArgs& a, int num_sms, cudaStream_t st);
cudaError_t launch_decode_g16(const CodecArgs& a, int num_sms, cudaStream_t st);
bool codec_mma16_supported(const CodecArgs& a);
cudaError_t launch_encode_mma16(const CodecArgs& a, int num_sms, cudaStream_t st);
cudaError_t launch_decode_mma16(const CodecArgs& a, int num_sms, cudaStream_t st);
cudaError_t launch_kivi(const CodecArgs& a, bool encode, int num_sms, cudaStream_t st);
bool kivi_mma16_supported(const CodecArgs& a);
cudaError_t launch_kivi_mma16(const CodecArgs& a, int num_sms, cudaStream_t st);
bool kivi_decode_g16_supported(const CodecArgs& a);
cudaError_t launch_kivi_decode_g16(const CodecArgs& a, int num_sms, cudaStream_t st);
cudaError_t launch_fullhead(const CodecArgs& a, bool encode, int num_sms, cudaStream_t st);
uint64_t spectral_workspace_bytes(const KvGeom& k, bool want_grad);
unsigned int* device_status_word();
cg_status validate_stats(const cg_kv_desc* kv, const cg_stats_desc* st);
bool spectral_tmem_supported(const KvGeom& k, int x_fp32);
int spectral_tmem_pieces(const KvGeom& k);
// fp32 input is supported for the statistics without dL/dG (dg_part == nullptr).
cudaError_t launch_spectral_tmem(const KvGeom& k, int x_fp32, const void* x, const float* G, float lambda_f,
                                 float lambda_r, float tau, float* lfreq, float* lrate, float* dg_part,
                                 unsigned int* status, int num_sms, cudaStream_t st);
bool spectral_fwd_f32_supported(const KvGeom& k);
cudaError_t launch_spectral_generic(const KvGeom& k, int x_fp32, const void* x, const float* G, float lambda_f,
                                    float lambda_r, float tau, float* lfreq, float* lrate, float* dg_part,
                                    int num_sms, cudaStream_t st);
// SM count of the current device, and the C-ABI status of a CUDA error (recorded
// for cg_last_cuda_error), shared by the entry points.
int num_sms();
cg_status from_cuda(cudaError_t e);
// Host validation shared by the entry points: 16-byte alignment, the cache shape, the codec.
bool aligned16(const void* p);
cg_status check_kv(const cg_kv_desc* kv);
cg_status check_codec(const cg_kv_desc* kv, const cg_codec_desc* c);
cudaError_t launch_spectral(const KvGeom& k, int x_fp32, const void* x, const float* G, float lambda_f, float lambda_r,
                            float tau, float* lfreq, float* lrate, double* totals, float* dG, void* workspace,
                            unsigned int* status, int num_sms, cudaStream_t st);

// Arguments of one decode-attention call, after host validation.
struct AttnArgs {
  KvGeom k;
  int bits;
  int hq;                 // query heads (a multiple of H)
  int n_tokens;           // attend to tokens [0, n_tokens), a multiple of 16
  int l0, n_layers;       // layers [l0, l0 + n_layers)
  int n_chunks;           // partials per (layer, batch, query head): set by the launcher
  int chunk;              // tokens per chunk, 128 or 256: set by the launcher
  int cpc;                // chunks per CTA: set by the launcher
  float scale;            // score scale (1/sqrt(d) by default)
  const uint16_t* q;      // bf16 [n_layers][B][hq][d]
  const uint8_t* codes;   // whole cache, block-uniform 16 x 16 ranges
  const uint16_t* scales;
  const uint16_t* zeros;
  const float* G;         // fp32 [L][2][H][d/16][16][16]
  float* out;             // fp32 [n_layers][B][hq][d]
  float* partial;         // workspace
};
uint64_t attn_workspace_bytes(const KvGeom& k, int hq, int n_layers, int n_tokens);
cudaError_t launch_decode_attention(AttnArgs a, int num_sms, cudaStream_t st);

// 2-D TMA tensor map over a row-major bf16 [rows][cols] array (box_cols x
// box_rows boxes, 128-byte swizzle); `out` points to a CUtensorMap.
bool make_tmap_2d_bf16(void* out, const void* base, uint64_t rows, uint64_t cols, int box_cols, int box_rows);
bool make_tmap_2d_f32(void* out, const void* base, uint64_t rows, uint64_t cols, int box_cols, int box_rows);
cudaError_t launch_gauge_build(const float* A, float* G, int n_mats, int g, cudaStream_t st);
cudaError_t launch_gauge_grad(const float* A, const float* dG, float* dA, int n_mats, int g, cudaStream_t st);
cudaError_t launch_adamw(float* p, const float* grad, float* m, float* v, long long n, float lr, float b1, float b2,
                         float eps, float wd, int step, int num_sms, cudaStream_t st);
cudaError_t launch_gram(const KvGeom& k, int g, const uint16_t* kv, double* gram, int t0, int nt, cudaStream_t st);

}  // namespace cg
