// Encode + decode of a host-resident cache, pipelined by layer over three
// streams so that both PCIe directions and the kernels overlap.
//
// Codec-Gauge, Method: the codec round trip (gauge, quantize, dequantize,
// inverse gauge), with the recovery charged in timing.  Every layout is
// layer-major ([L][2][B][H]... for the cache, the codes, the steps and zero
// points; [L][2][H]... for the gauges), so layer l of each array is one
// contiguous piece and the whole-cache entry points run on one-layer views.
#include <mutex>

#include "cg_kernels.cuh"

namespace {

constexpr int kMaxDevices = 64;

struct RtStreams {
  cudaStream_t up = nullptr, comp = nullptr, down = nullptr;
};

// The three streams of a device, created on first use and kept.
cudaError_t streams_for(RtStreams& out) {
  static std::mutex mu;
  static RtStreams table[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  RtStreams& s = table[dev];
  if (!s.up) {
    RtStreams n;
    e = cudaStreamCreateWithFlags(&n.up, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&n.comp, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&n.down, cudaStreamNonBlocking);
    if (e != cudaSuccess) {
      if (n.up) cudaStreamDestroy(n.up);
      if (n.comp) cudaStreamDestroy(n.comp);
      return e;
    }
    s = n;
  }
  out = s;
  return cudaSuccess;
}

uint64_t layer_kv_bytes(const cg_kv_desc* kv) {
  return (uint64_t)2 * kv->batch * kv->heads * kv->tokens * kv->d_head * 2;
}

}  // namespace

extern "C" {

cg_status cg_roundtrip_workspace_size(const cg_kv_desc* kv, uint64_t* bytes) {
  cg_status st = cg::check_kv(kv);
  if (st != CG_OK) return st;
  if (!bytes) return CG_ERR_INVALID;
  *bytes = 4 * layer_kv_bytes(kv);
  return CG_OK;
}

cg_status cg_roundtrip_host(const cg_kv_desc* kv, const cg_codec_desc* codec, const void* kv_host,
                            const float* G_dev, uint8_t* codes_dev, void* scales_dev, void* zeros_dev,
                            void* out_host, void* workspace_dev, uint64_t workspace_bytes, void* stream) {
  cg_status st = cg::check_codec(kv, codec);
  if (st != CG_OK) return st;
  if (!kv_host || !out_host || !G_dev || !codes_dev || !scales_dev || !zeros_dev || !workspace_dev)
    return CG_ERR_INVALID;
  if (!cg::aligned16(G_dev) || !cg::aligned16(codes_dev) || !cg::aligned16(scales_dev) || !cg::aligned16(zeros_dev) ||
      !cg::aligned16(workspace_dev))
    return CG_ERR_INVALID;
  const uint64_t kvb = layer_kv_bytes(kv);
  if (workspace_bytes < 4 * kvb) return CG_ERR_INVALID;
  cg_kv_desc one = *kv;  // one layer
  one.layers = 1;
  cg_sizes sz;
  st = cg_sizes_for(&one, codec, &sz);
  if (st != CG_OK) return st;
  const uint64_t code_b = sz.code_bytes, scale_b = sz.scale_count * 2;
  if (code_b % 16 != 0 || scale_b % 16 != 0) return CG_ERR_UNSUPPORTED;
  const uint64_t gauge_f = (uint64_t)2 * kv->heads * kv->d_head * codec->g;  // [2][H][d/g][g][g] floats
  if ((gauge_f * 4) % 16 != 0) return CG_ERR_UNSUPPORTED;

  RtStreams s;
  cudaError_t e = streams_for(s);
  if (e != cudaSuccess) return cg::from_cuda(e);
  const cudaStream_t caller = (cudaStream_t)stream;
  cudaEvent_t ev[7] = {};
  for (int i = 0; i < 7; ++i) {
    e = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming);
    if (e != cudaSuccess) {
      for (int j = 0; j < i; ++j) cudaEventDestroy(ev[j]);
      return cg::from_cuda(e);
    }
  }
  cudaEvent_t start = ev[0], up_done[2] = {ev[1], ev[2]}, comp_done[2] = {ev[3], ev[4]}, down_done[2] = {ev[5], ev[6]};
  unsigned char* ws = (unsigned char*)workspace_dev;
  unsigned char* in_buf[2] = {ws, ws + kvb};
  unsigned char* out_buf[2] = {ws + 2 * kvb, ws + 3 * kvb};
  const unsigned char* src = (const unsigned char*)kv_host;
  unsigned char* dst = (unsigned char*)out_host;

  // Enqueue everything; the first failure stops enqueueing (what is already
  // enqueued stays ordered and the caller's stream still waits for it).
  st = CG_OK;
  auto ok = [&](cudaError_t r) {
    if (r != cudaSuccess && st == CG_OK) st = cg::from_cuda(r);
    return st == CG_OK;
  };
  if (ok(cudaEventRecord(start, caller)) && ok(cudaStreamWaitEvent(s.up, start, 0)) &&
      ok(cudaStreamWaitEvent(s.comp, start, 0)) && ok(cudaStreamWaitEvent(s.down, start, 0))) {
    for (int l = 0; l < kv->layers && st == CG_OK; ++l) {
      const int b = l & 1;
      // host -> device of layer l, once the encode of layer l - 2 has read this buffer
      if (l >= 2 && !ok(cudaStreamWaitEvent(s.up, comp_done[b], 0))) break;
      if (!ok(cudaMemcpyAsync(in_buf[b], src + (uint64_t)l * kvb, kvb, cudaMemcpyHostToDevice, s.up))) break;
      if (!ok(cudaEventRecord(up_done[b], s.up))) break;
      // encode and decode of layer l, once its input is there and layer l - 2's output has left
      if (!ok(cudaStreamWaitEvent(s.comp, up_done[b], 0))) break;
      if (l >= 2 && !ok(cudaStreamWaitEvent(s.comp, down_done[b], 0))) break;
      const float* Gl = G_dev + (uint64_t)l * gauge_f;
      uint8_t* cl = codes_dev + (uint64_t)l * code_b;
      unsigned char* sl = (unsigned char*)scales_dev + (uint64_t)l * scale_b;
      unsigned char* zl = (unsigned char*)zeros_dev + (uint64_t)l * scale_b;
      st = cg_encode(&one, codec, in_buf[b], Gl, 0, kv->tokens, cl, sl, zl, nullptr, s.comp);
      if (st != CG_OK) break;
      st = cg_decode(&one, codec, cl, sl, zl, Gl, 0, kv->tokens, out_buf[b], s.comp);
      if (st != CG_OK) break;
      if (!ok(cudaEventRecord(comp_done[b], s.comp))) break;
      // device -> host of layer l
      if (!ok(cudaStreamWaitEvent(s.down, comp_done[b], 0))) break;
      if (!ok(cudaMemcpyAsync(dst + (uint64_t)l * kvb, out_buf[b], kvb, cudaMemcpyDeviceToHost, s.down))) break;
      if (!ok(cudaEventRecord(down_done[b], s.down))) break;
    }
  }
  // The caller's stream continues after everything enqueued above (each
  // internal stream ends with the event recorded here).
  cudaEvent_t tail[3] = {ev[1], ev[3], ev[5]};
  cudaStream_t tails[3] = {s.up, s.comp, s.down};
  for (int i = 0; i < 3; ++i) {
    cudaError_t r = cudaEventRecord(tail[i], tails[i]);
    if (r == cudaSuccess) r = cudaStreamWaitEvent(caller, tail[i], 0);
    if (r != cudaSuccess && st == CG_OK) st = cg::from_cuda(r);
  }
  for (int i = 0; i < 7; ++i) cudaEventDestroy(ev[i]);
  return st;
}

}  // extern "C"
