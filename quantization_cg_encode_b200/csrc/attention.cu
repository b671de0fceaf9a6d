// Decode-step attention straight from the encoded cache (block-uniform ranges
// of 16 tokens x 16 channels, g = 16), with the inverse gauge folded into the
// query and the output.
//
// Codec-Gauge, Figure 1 / Backend compatibility: keys and values are stored in
// gauge coordinates and mapped back with G^T before attention.  With y the
// dequantized gauged vector of one group, k = G_K^T y_K and v = G_V^T y_V, so
//   q . k_t = (G_K q) . y_K,t             (per group: G_K q computed once),
//   sum_t p_t v_t = G_V^T (sum_t p_t y_V,t)  (G_V^T applied once at the end).
// Neither identity changes the result; they move the gauge from every cached
// token to the one query.  Per token only the dequantization y = s q + z of
// the codes remains.
//
// Two kernels (flash decoding):
//   partial: one CTA per (layer, batch, KV head, 256-token chunk) and all query
//     heads of the GQA group; the chunk's key and value codes, steps and zero
//     points are staged in shared memory with coalesced 16-byte loads; thread =
//     token for the scores (q' from shared memory by broadcast), a block
//     reduction for the chunk's max and exp-sum per head, thread = channel for
//     the value sums; writes (max, sum, o[d]) per (query head, chunk);
//   combine: per (layer, batch, query head): merges the chunks' partials with
//     the usual rescaling, divides by the total, applies G_V^T per group.
#include "cg_kernels.cuh"

namespace cg {

namespace {

constexpr int kChunk = 256;  // tokens per CTA
constexpr int kAttnThreads = 256;

// Code i (0..15) of one 16-code row held in little-endian 32-bit words w.
template <int BITS>
__device__ __forceinline__ uint32_t row_code(const uint32_t (&w)[4], int i) {
  const int bit = i * BITS, wd = bit >> 5, sh = bit & 31;
  uint32_t v = w[wd] >> sh;
  if (sh + BITS > 32) v |= w[wd + 1] << (32 - sh);
  return v & ((1u << BITS) - 1u);
}
// The 2*BITS bytes of row `row` of a range block in shared memory.
template <int BITS>
__device__ __forceinline__ void load_row(const uint8_t* blk, int row, uint32_t (&w)[4]) {
  const uint8_t* src = blk + row * 2 * BITS;
  if constexpr (BITS == 4) {
    const uint2 v = *reinterpret_cast<const uint2*>(src);
    w[0] = v.x; w[1] = v.y; w[2] = 0; w[3] = 0;
  } else if constexpr (BITS == 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(src);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if constexpr (BITS == 2) {
    w[0] = *reinterpret_cast<const uint32_t*>(src); w[1] = w[2] = w[3] = 0;
  } else if constexpr (BITS == 3) {  // 6 bytes, 2-byte aligned
    const uint16_t* h = reinterpret_cast<const uint16_t*>(src);
    w[0] = h[0] | ((uint32_t)h[1] << 16); w[1] = h[2]; w[2] = w[3] = 0;
  } else {                            // 6 bits: 12 bytes, 4-byte aligned
    const uint32_t* u = reinterpret_cast<const uint32_t*>(src);
    w[0] = u[0]; w[1] = u[1]; w[2] = u[2]; w[3] = 0;
  }
}
// Exact float of a small integer code: the bits 0x4B000000 | c are 2^23 + c.
__device__ __forceinline__ float code_f(uint32_t c) { return __uint_as_float(0x4B000000u | c) - 8388608.0f; }

}  // namespace

// partial[l][b][hq][chunk] = {m, l, o[D]} in gauge coordinates.
template <int D, int BITS, int GQ>
__global__ void __launch_bounds__(kAttnThreads) attn_partial_kernel(AttnArgs a) {
  constexpr int NG = D / 16;
  constexpr int BLK = 32 * BITS;                 // bytes of one 16 x 16 range block
  constexpr int CODE_BYTES = kChunk * D * BITS / 8;
  constexpr int NBLK = kChunk / 16;
  extern __shared__ __align__(16) unsigned char smem[];
  uint8_t* kc = smem;                            // key codes of the chunk
  uint8_t* vc = kc + CODE_BYTES;                 // value codes
  float* ks = reinterpret_cast<float*>(vc + CODE_BYTES + 16);  // [NBLK][NG] key steps (16 B slack: 2-byte code reads)
  float* kz = ks + NBLK * NG;
  float* vs = kz + NBLK * NG;
  float* vz = vs + NBLK * NG;
  float* qp = vz + NBLK * NG;                    // [GQ][D]: q' = G_K q * scale
  float* qsum = qp + GQ * D;                     // [GQ][NG]: sum of q' over each group
  float* p = qsum + GQ * NG;                     // [kChunk][GQ]: scores, then exp weights
  float* red = p + kChunk * GQ;                  // [8 warps][GQ]
  float* stat = red + 8 * GQ;                    // [GQ]: chunk max

  const int chunk = blockIdx.x;
  const int bh = blockIdx.y;  // b * H + h
  const int lz = blockIdx.z;  // layer index within the call
  const int l = a.l0 + lz;
  const int h = bh % a.k.H, b = bh / a.k.H;
  const int tid = threadIdx.x;
  const int t0 = chunk * kChunk;
  const int ntok = min(kChunk, a.n_tokens - t0);
  const int nblk = (ntok + 15) / 16;
  const long long slice_k = (((long long)l * 2 + 0) * a.k.B + b) * a.k.H + h;
  const long long slice_v = (((long long)l * 2 + 1) * a.k.B + b) * a.k.H + h;
  const long long slice_bytes = (long long)a.k.T * D * BITS / 8;
  const int T16 = a.k.T / 16;

  // stage codes (whole range blocks), steps and zero points
  {
    const uint4* srck = reinterpret_cast<const uint4*>(a.codes + slice_k * slice_bytes + (long long)(t0 / 16) * NG * BLK);
    const uint4* srcv = reinterpret_cast<const uint4*>(a.codes + slice_v * slice_bytes + (long long)(t0 / 16) * NG * BLK);
    const int n16 = nblk * NG * BLK / 16;
    for (int e = tid; e < n16; e += kAttnThreads) {
      reinterpret_cast<uint4*>(kc)[e] = __ldg(srck + e);
      reinterpret_cast<uint4*>(vc)[e] = __ldg(srcv + e);
    }
    for (int e = tid; e < nblk * NG; e += kAttnThreads) {
      const long long ik = (slice_k * T16 + t0 / 16) * NG + e, iv = (slice_v * T16 + t0 / 16) * NG + e;
      ks[e] = __half2float(__ushort_as_half(a.scales[ik]));
      kz[e] = __half2float(__ushort_as_half(a.zeros[ik]));
      vs[e] = __half2float(__ushort_as_half(a.scales[iv]));
      vz[e] = __half2float(__ushort_as_half(a.zeros[iv]));
    }
    // q' = scale * G_K q per group, for the GQ query heads of this KV head
    const float* Gk = a.G + gauge_set(l, 0, h, a.k) * NG * 256;
    for (int e = tid; e < GQ * D; e += kAttnThreads) {
      const int j = e / D, c = e % D, r = c >> 4, i = c & 15;
      const uint16_t* qrow = a.q + (((long long)lz * a.k.B + b) * a.hq + h * GQ + j) * D + 16 * r;
      const float* gi = Gk + (r * 16 + i) * 16;
      float acc = 0.0f;
#pragma unroll
      for (int m = 0; m < 16; ++m) acc = __fmaf_rn(gi[m], bf16lo((uint32_t)qrow[m]), acc);
      qp[e] = acc * a.scale;
    }
  }
  __syncthreads();
  for (int e = tid; e < GQ * NG; e += kAttnThreads) {
    const float* q = qp + (e / NG) * D + 16 * (e % NG);
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) s += q[i];
    qsum[e] = s;
  }
  __syncthreads();

  // scores, thread = token: sum over groups of s (q' . code) + z sum(q')
  float sc[GQ];
  const int t = tid;
  const bool live = t < ntok;
  {
#pragma unroll
    for (int j = 0; j < GQ; ++j) sc[j] = -INFINITY;
    if (live) {
#pragma unroll
      for (int j = 0; j < GQ; ++j) sc[j] = 0.0f;
      const int kb = t >> 4, row = t & 15;
#pragma unroll 1
      for (int r = 0; r < NG; ++r) {
        uint32_t w[4];
        load_row<BITS>(kc + (kb * NG + r) * BLK, row, w);
        float acc[GQ];
#pragma unroll
        for (int j = 0; j < GQ; ++j) acc[j] = 0.0f;
#pragma unroll
        for (int i4 = 0; i4 < 4; ++i4) {
          float cf[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) cf[e] = code_f(row_code<BITS>(w, 4 * i4 + e));
#pragma unroll
          for (int j = 0; j < GQ; ++j) {
            const float4 q4 = *reinterpret_cast<const float4*>(qp + j * D + 16 * r + 4 * i4);  // broadcast
            acc[j] = __fmaf_rn(q4.x, cf[0], acc[j]);
            acc[j] = __fmaf_rn(q4.y, cf[1], acc[j]);
            acc[j] = __fmaf_rn(q4.z, cf[2], acc[j]);
            acc[j] = __fmaf_rn(q4.w, cf[3], acc[j]);
          }
        }
        const float s = ks[kb * NG + r], z = kz[kb * NG + r];
#pragma unroll
        for (int j = 0; j < GQ; ++j) sc[j] += __fmaf_rn(s, acc[j], z * qsum[j * NG + r]);
      }
    }
  }
  // chunk max and exp weights per query head
  const int warp = tid >> 5, lane = tid & 31;
#pragma unroll
  for (int j = 0; j < GQ; ++j) {
    float m = sc[j];
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) red[warp * GQ + j] = m;
  }
  __syncthreads();
  if (tid < GQ) {
    float m = red[tid];
    for (int w = 1; w < 8; ++w) m = fmaxf(m, red[w * GQ + tid]);
    stat[tid] = m;
  }
  __syncthreads();
  float ls[GQ];
#pragma unroll
  for (int j = 0; j < GQ; ++j) {
    const float pj = live ? __expf(sc[j] - stat[j]) : 0.0f;
    p[t * GQ + j] = pj;
    ls[j] = pj;
  }
  __syncthreads();  // red is reused below, p is read by every thread
#pragma unroll
  for (int j = 0; j < GQ; ++j) {
    float s = ls[j];
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) red[warp * GQ + j] = s;
  }
  __syncthreads();

  // value sums in gauge coordinates, thread = channel (threads D .. 2D-1 take the
  // second half of the tokens; their sums are added in a fixed order)
  float* out = a.partial + ((((long long)lz * a.k.B + b) * a.hq + h * GQ) * a.n_chunks + chunk) * (D + 2);
  const long long head_stride = (long long)a.n_chunks * (D + 2);
  constexpr int HALVES = kAttnThreads / D;  // 2 (d = 128) or 4 (d = 64)
  const int c = tid % D, part = tid / D, r = c >> 4, i = c & 15;
  float o[GQ];
#pragma unroll
  for (int j = 0; j < GQ; ++j) o[j] = 0.0f;
  const int per = (nblk + HALVES - 1) / HALVES;
  for (int kb = part * per; kb < min(nblk, part * per + per); ++kb) {
    const uint8_t* blk = vc + (kb * NG + r) * BLK;
    const float s = vs[kb * NG + r], z = vz[kb * NG + r];
    float acc[GQ], psum[GQ];
#pragma unroll
    for (int j = 0; j < GQ; ++j) acc[j] = psum[j] = 0.0f;
#pragma unroll 4
    for (int row = 0; row < 16; ++row) {
      const int bit = (row * 16 + i) * BITS;
      const uint32_t wv = (uint32_t)blk[bit >> 3] | ((uint32_t)blk[(bit >> 3) + 1] << 8);
      const float cf = code_f((wv >> (bit & 7)) & ((1u << BITS) - 1u));
      const float* pr = p + (kb * 16 + row) * GQ;  // broadcast
#pragma unroll
      for (int j = 0; j < GQ; ++j) {
        acc[j] = __fmaf_rn(pr[j], cf, acc[j]);
        psum[j] += pr[j];
      }
    }
#pragma unroll
    for (int j = 0; j < GQ; ++j) o[j] += __fmaf_rn(s, acc[j], z * psum[j]);
  }
  // combine the token parts in order through shared memory (p is no longer needed)
  __syncthreads();
  float* po = p;  // [HALVES][GQ][D]
#pragma unroll
  for (int j = 0; j < GQ; ++j) po[(part * GQ + j) * D + c] = o[j];
  __syncthreads();
  if (part == 0) {
#pragma unroll
    for (int j = 0; j < GQ; ++j) {
      float v = po[j * D + c];
      for (int q2 = 1; q2 < HALVES; ++q2) v += po[(q2 * GQ + j) * D + c];
      out[j * head_stride + 2 + c] = v;
    }
  }
  if (tid < GQ) {
    float s = 0.0f;
    for (int w = 0; w < 8; ++w) s += red[w * GQ + tid];
    out[tid * head_stride + 0] = stat[tid];
    out[tid * head_stride + 1] = s;
  }
}

// out[l][b][hq] = G_V^T (sum_k e^(m_k - M) o_k) / (sum_k e^(m_k - M) l_k)
template <int D>
__global__ void __launch_bounds__(D) attn_combine_kernel(AttnArgs a) {
  constexpr int NG = D / 16;
  __shared__ float og[D];
  const int hq = blockIdx.x, b = blockIdx.y, lz = blockIdx.z;
  const int l = a.l0 + lz, h = hq / (a.hq / a.k.H);
  const int c = threadIdx.x;
  const float* part = a.partial + ((((long long)lz * a.k.B + b) * a.hq + hq) * a.n_chunks) * (D + 2);
  float M = -INFINITY;
  for (int k = 0; k < a.n_chunks; ++k) M = fmaxf(M, part[k * (D + 2)]);
  float Ls = 0.0f, O = 0.0f;
  for (int k = 0; k < a.n_chunks; ++k) {
    const float w = __expf(part[k * (D + 2)] - M);
    Ls = __fmaf_rn(w, part[k * (D + 2) + 1], Ls);
    O = __fmaf_rn(w, part[k * (D + 2) + 2 + c], O);
  }
  og[c] = O / Ls;
  __syncthreads();
  // x = G_V^T y per group: out[16 r + j] = sum_i G[r][i][j] y[16 r + i]
  const int r = c >> 4, j = c & 15;
  const float* Gv = a.G + (gauge_set(l, 1, h, a.k) * NG + r) * 256;
  float acc = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) acc = __fmaf_rn(Gv[i * 16 + j], og[16 * r + i], acc);
  a.out[(((long long)lz * a.k.B + b) * a.hq + hq) * D + c] = acc;
}

namespace {

template <int D, int BITS, int GQ>
cudaError_t attn_launch(const AttnArgs& a, cudaStream_t st) {
  constexpr int NG = D / 16;
  constexpr int CODE_BYTES = kChunk * D * BITS / 8;
  constexpr int NBLK = kChunk / 16;
  static_assert((kAttnThreads / D) * GQ * D == kChunk * GQ, "the value parts' sums fit where the weights were");
  const int smem_floats = 4 * NBLK * NG + GQ * D + GQ * NG + kChunk * GQ + 8 * GQ + GQ;
  const size_t smem = 2 * CODE_BYTES + 16 + 4 * (size_t)smem_floats;
  auto kern = attn_partial_kernel<D, BITS, GQ>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.n_chunks, a.k.B * a.k.H, a.n_layers);
  kern<<<grid, kAttnThreads, smem, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 cgrid(a.hq, a.k.B, a.n_layers);
  attn_combine_kernel<D><<<cgrid, D, 0, st>>>(a);
  return cudaGetLastError();
}

template <int D, int BITS>
cudaError_t attn_gq(const AttnArgs& a, cudaStream_t st) {
  switch (a.hq / a.k.H) {
    case 1: return attn_launch<D, BITS, 1>(a, st);
    case 2: return attn_launch<D, BITS, 2>(a, st);
    case 4: return attn_launch<D, BITS, 4>(a, st);
    case 8: return attn_launch<D, BITS, 8>(a, st);
  }
  return cudaErrorInvalidValue;
}

template <int D>
cudaError_t attn_bits(const AttnArgs& a, cudaStream_t st) {
  switch (a.bits) {
    case 2: return attn_gq<D, 2>(a, st);
    case 3: return attn_gq<D, 3>(a, st);
    case 4: return attn_gq<D, 4>(a, st);
    case 6: return attn_gq<D, 6>(a, st);
    case 8: return attn_gq<D, 8>(a, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

uint64_t attn_workspace_bytes(const KvGeom& k, int hq, int n_layers, int n_tokens) {
  const uint64_t chunks = (uint64_t)(n_tokens + kChunk - 1) / kChunk;
  return (uint64_t)n_layers * k.B * hq * chunks * (k.d + 2) * sizeof(float);
}

cudaError_t launch_decode_attention(AttnArgs a, cudaStream_t st) {
  a.n_chunks = (a.n_tokens + kChunk - 1) / kChunk;
  return a.k.d == 128 ? attn_bits<128>(a, st) : attn_bits<64>(a, st);
}

}  // namespace cg
