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
cudaError_t launch_gauge_build(const float* A, float* G, int n_mats, int g, cudaStream_t st);

}  // namespace cg
