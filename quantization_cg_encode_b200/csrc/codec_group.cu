// Block-uniform codec for grouped gauges (g = 8, 16, 32), any bit width:
// the general kernels.  One thread owns one (token, channel group) of a
// 16-token tile and computes all g gauged values of it.
//
// Codec-Gauge, Problem statement and overview (channel groups) and Method
// (explicit application costs O(N_KV g) multiply-adds); Experimental setup
// (block-uniform backend: one min/max range per T_b x W block).
#include "cg_kernels.cuh"

namespace cg {

namespace {

constexpr int kThreads = 256;

// Work split: a "pass" is TPC consecutive 16-token tiles of one head slice,
// TPC = 256 / (16 R) so that one pass gives every thread one (token, group).
struct PassMap {
  int R, TPC, tiles;      // groups per head, tiles per pass, tiles in [t0, t0+nt)
  long long passes_per_slice, passes;
};

__host__ __device__ inline PassMap pass_map(const CodecArgs& a) {
  PassMap m;
  m.R = a.k.d / a.g;
  m.TPC = kThreads / (16 * m.R);
  m.tiles = a.nt / 16;
  m.passes_per_slice = (m.tiles + m.TPC - 1) / m.TPC;
  m.passes = m.passes_per_slice * a.k.slices();
  return m;
}

// Bytes of packed codes of one 16-token tile (all channel groups).
__host__ __device__ inline int tile_code_bytes(int d, int bits) { return 16 * d * bits / 8; }

// Byte offset, inside a tile's code bytes, of the chunk of g codes that token
// t of group r owns.  Element order inside a range block is token-major.
__device__ inline int chunk_byte_offset(int t, int r, int g, int W, int d, int bits) {
  if (W == g) return r * (16 * g * bits / 8) + t * (g * bits / 8);
  return (t * d + r * g) * bits / 8;  // W == d: one block per tile
}

}  // namespace

// ----------------------------------------------------------------------------------------
template <int G, int BITS>
__global__ void __launch_bounds__(kThreads) encode_group_kernel(CodecArgs a) {
  constexpr int QMAX = (1 << BITS) - 1;
  constexpr int CHUNK_BYTES = G * BITS / 8;
  __shared__ __align__(16) float sGT[128 * G];          // [R][j][i] = G[r][i][j]
  __shared__ __align__(16) uint8_t sCodes[kThreads * G * BITS / 8];
  __shared__ float sRed[2][16][16];                     // [min/max][tile][group]

  const PassMap m = pass_map(a);
  const int R = m.R, d = a.k.d, W = a.W;
  const int tid = threadIdx.x;
  const int tile_local = tid / (16 * R);
  const int r = (tid / 16) % R;
  const int t = tid % 16;
  const int tile_bytes = tile_code_bytes(d, BITS);
  const double inv_qmax = 1.0 / (double)QMAX;

  // contiguous range of passes for this CTA
  const long long p_begin = m.passes * blockIdx.x / gridDim.x;
  const long long p_end = m.passes * (blockIdx.x + 1) / gridDim.x;
  long long loaded_set = -1;

  for (long long p = p_begin; p < p_end; ++p) {
    const long long slice = p / m.passes_per_slice;
    const int tile0 = (int)(p % m.passes_per_slice) * m.TPC;
    const int tile = tile0 + tile_local;
    const bool valid = tile_local < m.TPC && tile < m.tiles;
    int l, s, b, h;
    slice_coords(slice, a.k, l, s, b, h);
    const long long gset = gauge_set(l, s, h, a.k);

    if (gset != loaded_set) {  // stage G^T of this (l, s, h) in shared memory
      __syncthreads();
      const float* Gp = a.G + gset * (long long)d * G;  // [R][g][g]
      for (int e = tid; e < d * G; e += kThreads) {
        const int rr = e / (G * G), i = (e / G) % G, j = e % G;
        sGT[rr * G * G + j * G + i] = Gp[e];
      }
      loaded_set = gset;
      __syncthreads();
    }

    const int tok = a.t0 + tile * 16 + t;
    const long long row = (slice * a.k.T + tok) * (long long)d;  // element index of (slice, tok, 0)
    float y[G];
    float mn = INFINITY, mx = -INFINITY;
    if (valid) {
      float x[G];
      const uint4* src = reinterpret_cast<const uint4*>(a.kv + row + r * G);
#pragma unroll
      for (int v = 0; v < G / 8; ++v) {
        const uint4 w = src[v];
        x[8 * v + 0] = bf16lo(w.x); x[8 * v + 1] = bf16hi(w.x);
        x[8 * v + 2] = bf16lo(w.y); x[8 * v + 3] = bf16hi(w.y);
        x[8 * v + 4] = bf16lo(w.z); x[8 * v + 5] = bf16hi(w.z);
        x[8 * v + 6] = bf16lo(w.w); x[8 * v + 7] = bf16hi(w.w);
      }
      // y_i = fp32 FMA chain over j = 0 .. g-1 in index order, from +0.
#pragma unroll
      for (int i = 0; i < G; ++i) y[i] = 0.0f;
      const float* gt = sGT + r * G * G;
#pragma unroll
      for (int j = 0; j < G; ++j) {
        const float xj = x[j];
#pragma unroll
        for (int i = 0; i < G; i += 4) {
          const float4 c = *reinterpret_cast<const float4*>(gt + j * G + i);
          y[i + 0] = __fmaf_rn(c.x, xj, y[i + 0]);
          y[i + 1] = __fmaf_rn(c.y, xj, y[i + 1]);
          y[i + 2] = __fmaf_rn(c.z, xj, y[i + 2]);
          y[i + 3] = __fmaf_rn(c.w, xj, y[i + 3]);
        }
      }
      if (a.gauged) {
        float4* dst = reinterpret_cast<float4*>(a.gauged + row + r * G);
#pragma unroll
        for (int i = 0; i < G; i += 4) dst[i / 4] = make_float4(y[i], y[i + 1], y[i + 2], y[i + 3]);
      }
#pragma unroll
      for (int i = 0; i < G; ++i) {
        mn = fminf(mn, y[i]);
        mx = fmaxf(mx, y[i]);
      }
    }
    // range of the 16 tokens of this group (16 aligned lanes)
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    if (W != G) {  // W == d: combine the R groups of the tile
      if (t == 0 && tile_local < 16) {
        sRed[0][tile_local][r] = mn;
        sRed[1][tile_local][r] = mx;
      }
      __syncthreads();
      if (tile_local < 16) {
        mn = sRed[0][tile_local][0];
        mx = sRed[1][tile_local][0];
        for (int rr = 1; rr < R; ++rr) {
          mn = fminf(mn, sRed[0][tile_local][rr]);
          mx = fmaxf(mx, sRed[1][tile_local][rr]);
        }
      }
    }
    if (valid) {
      const QParams qp = quant_params(mn, mx, inv_qmax);
      // pack this thread's g codes (token-major, LE bit stream)
      uint8_t* dst = sCodes + tile_local * tile_bytes + chunk_byte_offset(t, r, G, W, d, BITS);
      uint64_t acc = 0;
      int nbits = 0, nb = 0;
#pragma unroll
      for (int i = 0; i < G; ++i) {
        const uint32_t q = quantize_one(y[i], qp.zf, qp.inv, QMAX);
        acc |= (uint64_t)q << nbits;
        nbits += BITS;
        while (nbits >= 8) {
          dst[nb++] = (uint8_t)(acc & 0xffu);
          acc >>= 8;
          nbits -= 8;
        }
      }
      (void)CHUNK_BYTES;
      const int nblk = d / W;
      if (t == 0 && (W == G || r == 0)) {
        const long long bidx = (slice * (a.k.T / 16) + (a.t0 / 16 + tile)) * nblk + (W == G ? r : 0);
        a.scales[bidx] = qp.sh;
        a.zeros[bidx] = qp.zh;
      }
    }
    __syncthreads();
    // copy the pass's code bytes out (tiles of a slice are contiguous)
    {
      const int ntiles = min(m.TPC, m.tiles - tile0);
      const long long gofs = slice * ((long long)a.k.T * d * BITS / 8) + (long long)(a.t0 / 16 + tile0) * tile_bytes;
      const int n16 = ntiles * tile_bytes / 16;
      uint4* gdst = reinterpret_cast<uint4*>(a.codes + gofs);
      const uint4* ssrc = reinterpret_cast<const uint4*>(sCodes);
      for (int e = tid; e < n16; e += kThreads) gdst[e] = ssrc[e];
    }
    __syncthreads();
  }
}

// ----------------------------------------------------------------------------------------
template <int G, int BITS>
__global__ void __launch_bounds__(kThreads) decode_group_kernel(CodecArgs a) {
  __shared__ __align__(16) float sG[128 * G];            // [R][c][i] = G[r][c][i]
  __shared__ __align__(16) uint8_t sCodes[kThreads * G * BITS / 8];

  const PassMap m = pass_map(a);
  const int R = m.R, d = a.k.d, W = a.W;
  const int tid = threadIdx.x;
  const int tile_local = tid / (16 * R);
  const int r = (tid / 16) % R;
  const int t = tid % 16;
  const int tile_bytes = tile_code_bytes(d, BITS);

  const long long p_begin = m.passes * blockIdx.x / gridDim.x;
  const long long p_end = m.passes * (blockIdx.x + 1) / gridDim.x;
  long long loaded_set = -1;

  for (long long p = p_begin; p < p_end; ++p) {
    const long long slice = p / m.passes_per_slice;
    const int tile0 = (int)(p % m.passes_per_slice) * m.TPC;
    const int tile = tile0 + tile_local;
    const bool valid = tile_local < m.TPC && tile < m.tiles;
    const int ntiles = min(m.TPC, m.tiles - tile0);
    int l, s, b, h;
    slice_coords(slice, a.k, l, s, b, h);
    const long long gset = gauge_set(l, s, h, a.k);

    __syncthreads();  // previous pass done with sCodes / sG
    if (gset != loaded_set) {
      const float4* Gp = reinterpret_cast<const float4*>(a.G + gset * (long long)d * G);
      float4* sg4 = reinterpret_cast<float4*>(sG);
      for (int e = tid; e < d * G / 4; e += kThreads) sg4[e] = Gp[e];
      loaded_set = gset;
    }
    {
      const long long gofs = slice * ((long long)a.k.T * d * BITS / 8) + (long long)(a.t0 / 16 + tile0) * tile_bytes;
      const uint4* gsrc = reinterpret_cast<const uint4*>(a.codes_in + gofs);
      uint4* sdst = reinterpret_cast<uint4*>(sCodes);
      const int n16 = ntiles * tile_bytes / 16;
      for (int e = tid; e < n16; e += kThreads) sdst[e] = gsrc[e];
    }
    __syncthreads();
    if (!valid) continue;

    const int nblk = d / W;
    const long long bidx = (slice * (a.k.T / 16) + (a.t0 / 16 + tile)) * nblk + (W == G ? r : 0);
    const float sf = __half2float(__ushort_as_half(a.scales_in[bidx]));
    const float zf = __half2float(__ushort_as_half(a.zeros_in[bidx]));

    // unpack g codes and dequantize: yhat_c = s q_c + z
    float yh[G];
    {
      const uint8_t* src = sCodes + tile_local * tile_bytes + chunk_byte_offset(t, r, G, W, d, BITS);
      uint64_t acc = 0;
      int nbits = 0, nb = 0;
#pragma unroll
      for (int c = 0; c < G; ++c) {
        while (nbits < BITS) {
          acc |= (uint64_t)src[nb++] << nbits;
          nbits += 8;
        }
        const uint32_t q = (uint32_t)(acc & ((1u << BITS) - 1u));
        acc >>= BITS;
        nbits -= BITS;
        yh[c] = __fmaf_rn(sf, (float)q, zf);
      }
    }
    // x_hat_i = sum_c G[c][i] yhat_c   (inverse gauge G^T)
    float xo[G];
#pragma unroll
    for (int i = 0; i < G; ++i) xo[i] = 0.0f;
    const float* gg = sG + r * G * G;
#pragma unroll
    for (int c = 0; c < G; ++c) {
#pragma unroll
      for (int i = 0; i < G; i += 4) {
        const float4 v = *reinterpret_cast<const float4*>(gg + c * G + i);
        xo[i + 0] = __fmaf_rn(v.x, yh[c], xo[i + 0]);
        xo[i + 1] = __fmaf_rn(v.y, yh[c], xo[i + 1]);
        xo[i + 2] = __fmaf_rn(v.z, yh[c], xo[i + 2]);
        xo[i + 3] = __fmaf_rn(v.w, yh[c], xo[i + 3]);
      }
    }
    const int tok = a.t0 + tile * 16 + t;
    const long long row = (slice * a.k.T + tok) * (long long)d;
    uint4* dst = reinterpret_cast<uint4*>(a.kv_out + row + r * G);
#pragma unroll
    for (int v = 0; v < G / 8; ++v) {
      uint4 w;
      w.x = pack_bf16x2(xo[8 * v + 0], xo[8 * v + 1]);
      w.y = pack_bf16x2(xo[8 * v + 2], xo[8 * v + 3]);
      w.z = pack_bf16x2(xo[8 * v + 4], xo[8 * v + 5]);
      w.w = pack_bf16x2(xo[8 * v + 6], xo[8 * v + 7]);
      dst[v] = w;
    }
  }
}

// ----------------------------------------------------------------------------------------
namespace {
template <int G, int BITS>
cudaError_t launch_pair(const CodecArgs& a, bool encode, int grid, cudaStream_t st) {
  if (encode)
    encode_group_kernel<G, BITS><<<grid, kThreads, 0, st>>>(a);
  else
    decode_group_kernel<G, BITS><<<grid, kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

template <int G>
cudaError_t launch_bits(const CodecArgs& a, bool encode, int grid, cudaStream_t st) {
  switch (a.bits) {
    case 2: return launch_pair<G, 2>(a, encode, grid, st);
    case 3: return launch_pair<G, 3>(a, encode, grid, st);
    case 4: return launch_pair<G, 4>(a, encode, grid, st);
    case 6: return launch_pair<G, 6>(a, encode, grid, st);
    case 8: return launch_pair<G, 8>(a, encode, grid, st);
  }
  return cudaErrorInvalidValue;
}
}  // namespace

cudaError_t launch_group_codec(const CodecArgs& a, bool encode, int num_sms, cudaStream_t st) {
  const PassMap m = pass_map(a);
  if (m.passes == 0) return cudaSuccess;
  const long long grid = m.passes < (long long)num_sms * 4 ? m.passes : (long long)num_sms * 4;
  switch (a.g) {
    case 8: return launch_bits<8>(a, encode, (int)grid, st);
    case 16: return launch_bits<16>(a, encode, (int)grid, st);
    case 32: return launch_bits<32>(a, encode, (int)grid, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace cg
