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
//   partial: one CTA per (layer, batch, KV head, run of cpc chunks of 128 or 256 tokens)
//     and all query heads of the GQA group.  Each chunk's key and value codes, steps and zero
//     points are staged in shared memory with coalesced 16-byte loads.  Both
//     contractions run on the warp-level tensor cores (mma.sync m16n8k16,
//     fp16 operands, fp32 accumulation), one MMA per 16 x 16 range block, with
//     the codes as exact small integers:
//       scores  S[t][j] = sum_r s_r (code_r q'_r)[t][j] + z_r sum(q'_r)[j]: A =
//               the block's key codes, B = q' as fp16 hi + lo terms (scaled per
//               head by a power of two into fp16's range; about 2^-22 relative),
//       values  O[c][j] = sum_blocks s (code^T p)[c][j] + z sum_t p[t][j]: A =
//               the block's value codes transposed, B = the softmax weights as
//               fp16 hi + lo terms (scaled by 2^12);
//     the block's step and zero point apply to each MMA result.  Writes (max,
//     sum, o[d]) per (query head, run of chunks);
//   combine: per (layer, batch, query head): merges the chunks' partials with
//     the usual rescaling, divides by the total, applies G_V^T per group.
#include "cg_kernels.cuh"

namespace cg {

namespace {

// Tokens per chunk: 128 (about 46 KB of shared memory per CTA at d = 128: four CTAs
// per SM) or 256 (85 KB: two per SM, half the phase synchronisations per token),
// chosen by the launcher.
constexpr int kSmallChunk = 128, kLargeChunk = 256;
constexpr int kMaxCpc = 8;   // chunks per CTA (one partial per CTA) at most; the launcher picks 1, 2, 4 or 8
constexpr int kAttnThreads = 256;

// Asynchronous global -> shared copies (16 bytes bypassing L1, or 4 bytes),
// grouped per thread; wait until at most N groups of this thread are pending.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async4(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem_dst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// 4-bit codes to exact fp16 pairs without moving single nibbles: the nibbles at bits
// 0 and 16 of w give 1024 + n (one LOP3, then minus 1024), those at bits 4 and 20 give
// 1024 + 16 n (then / 16 - 64, exact in fp16).
__device__ __forceinline__ uint32_t nib_lo_pair(uint32_t w) {
  return f16_sub1024((w & 0x000F000Fu) | 0x64006400u);
}
__device__ __forceinline__ uint32_t nib_hi_pair(uint32_t w) {
  uint32_t r;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"((w & 0x00F000F0u) | 0x64006400u), "r"(0x2C002C00u), "r"(0xD400D400u));
  return r;
}

}  // namespace

// partial[l][b][hq][split] = {m, l, o[D]} in gauge coordinates, over the token
// chunks [split cpc, split cpc + cpc) of one (layer, batch, KV head).
//
// MMA columns: for GQ <= 4 one N = 8 tile holds the hi terms of heads 0..3 in
// columns 0..3 and the lo terms in 4..7 (heads >= GQ are zero); for GQ = 8 a
// tile of hi terms and a tile of lo terms.  A thread's accumulator columns 2c,
// 2c+1 are then heads 2c, 2c+1 (hi) or their lo parts, combined by a shuffle.
// A CTA's chunks stream through two shared-memory stages (cp.async: the next
// chunk's codes, steps and zero points load while the current one computes)
// and are merged with the online softmax rescaling.
template <int D, int BITS, int GQ, int kChunk>
__global__ void __launch_bounds__(kAttnThreads) attn_partial_kernel(AttnArgs a) {
  constexpr int NG = D / 16;
  constexpr int BLK = 32 * BITS;                 // bytes of one 16 x 16 range block
  constexpr int CODE_BYTES = kChunk * D * BITS / 8;
  constexpr int NBLK = kChunk / 16;
  constexpr int NT = GQ == 8 ? 2 : 1;            // N = 8 tiles per MMA step
  constexpr int RB = NBLK * NG * 2;              // bytes of one chunk's fp16 steps (or zero points)
  constexpr int STAGE = 2 * (CODE_BYTES + 16) + 4 * RB;
  constexpr float kPScale = 4096.0f;             // p in [0, 1] -> [0, 2^12] for fp16 terms
  extern __shared__ __align__(16) unsigned char smem[];
  // stage b: [key codes | 16 | value codes | 16 | key steps | key zeros | value steps | value zeros]
  float* qp = reinterpret_cast<float*>(smem + 2 * STAGE);  // [GQ][D]: q' = scale * G_K q
  float* qsum = qp + GQ * D;                     // [GQ][NG]: sum of q' over each group
  float* qinv = qsum + GQ * NG;                  // [GQ]: 2^-e_j, the inverse of q''s fp16 scaling
  float* sc = qinv + 8;                          // [kChunk][GQ]: scores
  float* psum = sc + kChunk * GQ;                // [NBLK][GQ]: sum of p over each block
  float* red = psum + NBLK * GQ;                 // [8 warps][GQ]
  float* stat = red + 8 * GQ;                    // [GQ]: chunk max
  float* run = stat + 8;                         // [4][8]: running max, running sum, old / new weights
  float* po = run + 32;                          // [2][GQ][D]: value halves (d = 64)
  float* zsum = po + 2 * GQ * D;                 // [NBLK][GQ]: sum_r z_r sum(q'_r) of each key block
  uint32_t* bqs = reinterpret_cast<uint32_t*>(zsum + NBLK * GQ);  // [NG][NT][32 lanes][2] fp16 q'' fragments
  uint16_t* pb = reinterpret_cast<uint16_t*>(bqs + NG * NT * 64);  // [NCOL][kChunk] fp16 p terms

  const int split = blockIdx.x;
  const int bh = blockIdx.y;  // b * H + h
  const int lz = blockIdx.z;  // layer index within the call
  const int l = a.l0 + lz;
  const int h = bh % a.k.H, b = bh / a.k.H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;
  const int n_tc = (a.n_tokens + kChunk - 1) / kChunk;  // token chunks
  const int c0 = split * a.cpc, c1 = min(n_tc, c0 + a.cpc);
  const long long slice_k = (((long long)l * 2 + 0) * a.k.B + b) * a.k.H + h;
  const long long slice_v = (((long long)l * 2 + 1) * a.k.B + b) * a.k.H + h;
  const long long slice_bytes = (long long)a.k.T * D * BITS / 8;
  const int T16 = a.k.T / 16;

  // chunk -> stage st: 16-byte copies of the codes, 4-byte copies of the ranges
  auto issue = [&](int chunk, int st) {
    unsigned char* base = smem + st * STAGE;
    const int t0 = chunk * kChunk, nb = min(kChunk, a.n_tokens - t0) / 16;
    const uint8_t* srck = a.codes + slice_k * slice_bytes + (long long)(t0 / 16) * NG * BLK;
    const uint8_t* srcv = a.codes + slice_v * slice_bytes + (long long)(t0 / 16) * NG * BLK;
    const int n16 = nb * NG * BLK / 16;
    for (int e = tid; e < n16; e += kAttnThreads) {
      cp_async16(base + 16 * e, srck + 16 * e);
      cp_async16(base + CODE_BYTES + 16 + 16 * e, srcv + 16 * e);
    }
    const int n4 = nb * NG / 2;  // 4-byte words of one range array
    for (int e = tid; e < 4 * n4; e += kAttnThreads) {
      const int arr = e / n4, w = e % n4;  // key steps, key zeros, value steps, value zeros
      const uint16_t* src = (arr & 1) ? a.zeros : a.scales;
      const long long sl = (arr >> 1) ? slice_v : slice_k;
      cp_async4(base + 2 * (CODE_BYTES + 16) + arr * RB + 4 * w, src + (sl * T16 + t0 / 16) * NG + 2 * w);
    }
    cp_async_commit();
  };
  issue(c0, 0);  // the first chunk loads while q' is formed

  // q' per group, once per CTA
  {
    const float* Gk = a.G + gauge_set(l, 0, h, a.k) * NG * 256;
    for (int e = tid; e < GQ * D; e += kAttnThreads) {
      const int j = e / D, cc = e % D, r = cc >> 4, i = cc & 15;
      const uint16_t* qrow = a.q + (((long long)lz * a.k.B + b) * a.hq + h * GQ + j) * D + 16 * r;
      const float* gi = Gk + (r * 16 + i) * 16;
      float acc = 0.0f;
#pragma unroll
      for (int m = 0; m < 16; ++m) acc = __fmaf_rn(gi[m], bf16lo((uint32_t)qrow[m]), acc);
      qp[e] = acc * a.scale;
    }
    if (tid < GQ) {
      run[tid] = -INFINITY;  // running max
      run[8 + tid] = 0.0f;   // running sum
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
  if (warp < GQ) {  // fp16 scaling of head j: max |q'| * 2^e_j in [2^14, 2^15)
    float m = 0.0f;
    for (int i = lane; i < D; i += 32) m = fmaxf(m, fabsf(qp[warp * D + i]));
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    int ex = 0;
    if (m > 0.0f) frexpf(m, &ex);
    if (lane == 0) qinv[warp] = m > 0.0f ? ldexpf(1.0f, ex - 15) : 1.0f;
  }
  __syncthreads();
  // the B fragments of q'' (column n = g of tile tt holds q'' = q' 2^e of (term,
  // head); k slots 2c, 2c+1 / 2c+8, 2c+9 are channels 4c, 4c+1 / 4c+2, 4c+3 of the group,
  // or, for 4-bit codes, channels b, b+4 / b+1, b+5 with b = 8 (c >> 1) + 2 (c & 1): the
  // nibble pairs a key word yields directly)
  for (int e = tid; e < NG * NT * 32; e += kAttnThreads) {
    const int ln = e & 31, tt = (e >> 5) % NT, r = (e >> 5) / NT;
    const int gg = ln >> 2, cc = ln & 3;
    const int j = NT == 2 ? gg : (gg & 3), lo = NT == 2 ? tt : (gg >> 2);
    const bool on = j < GQ;
    const float sj = on ? 1.0f / qinv[j] : 0.0f;
    float v[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    if (on) {
      const float* qg = qp + j * D + 16 * r;
      if constexpr (BITS == 4) {
        const int bb = 8 * (cc >> 1) + 2 * (cc & 1);
        v[0] = qg[bb] * sj;
        v[1] = qg[bb + 4] * sj;
        v[2] = qg[bb + 1] * sj;
        v[3] = qg[bb + 5] * sj;
      } else {
        const float4 q4 = *reinterpret_cast<const float4*>(qg + 4 * cc);
        v[0] = q4.x * sj;
        v[1] = q4.y * sj;
        v[2] = q4.z * sj;
        v[3] = q4.w * sj;
      }
    }
    __half hv[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const __half hi = __float2half_rn(v[k]);
      hv[k] = lo ? __float2half_rn(v[k] - __half2float(hi)) : hi;
    }
    bqs[2 * e] = (uint32_t)__half_as_ushort(hv[0]) | ((uint32_t)__half_as_ushort(hv[1]) << 16);
    bqs[2 * e + 1] = (uint32_t)__half_as_ushort(hv[2]) | ((uint32_t)__half_as_ushort(hv[3]) << 16);
  }

  float orun[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // running o of this thread's (channel, head) pairs
  for (int chunk = c0, it = 0; chunk < c1; ++chunk, ++it) {
    const int st = it & 1;
    __syncthreads();  // every thread is done with the other stage (the previous chunk)
    if (chunk + 1 < c1) {
      issue(chunk + 1, st ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();  // this chunk's stage is complete
    const unsigned char* base = smem + st * STAGE;
    const uint8_t* kc = base;
    const uint8_t* vc = base + CODE_BYTES + 16;
    const __half* ks = reinterpret_cast<const __half*>(base + 2 * (CODE_BYTES + 16));
    const __half* kz = ks + RB / 2;
    const __half* vs = kz + RB / 2;
    const __half* vz = vs + RB / 2;
    const int t0 = chunk * kChunk;
    const int ntok = min(kChunk, a.n_tokens - t0);
    const int nblk = ntok / 16;  // n_tokens is a multiple of 16
    for (int e = tid; e < nblk * GQ; e += kAttnThreads) {
      const int kb = e / GQ, j = e % GQ;
      float zt = 0.0f;
#pragma unroll
      for (int r = 0; r < NG; ++r) zt = __fmaf_rn(__half2float(kz[kb * NG + r]), qsum[j * NG + r], zt);
      zsum[e] = zt;
    }
    __syncthreads();

    // ---- scores on the tensor cores: warp w takes blocks w and w + 8 ----
    {
      const int bit_g = (16 * g + 4 * c) * BITS, bit_g8 = (16 * (g + 8) + 4 * c) * BITS;
  #pragma unroll
      for (int bi = 0; bi < 2; ++bi) {
        const int kb = warp + 8 * bi;
        if (kb >= nblk) continue;  // warp-uniform
        float acc[NT][4];
  #pragma unroll
        for (int tt = 0; tt < NT; ++tt)
  #pragma unroll
          for (int e = 0; e < 4; ++e) acc[tt][e] = 0.0f;
  #pragma unroll
        for (int r = 0; r < NG; ++r) {
          const uint8_t* blk = kc + (kb * NG + r) * BLK;
          uint32_t cv[2];  // rows g, g+8: codes 4c .. 4c+3 (4 BITS bits, low aligned)
          if constexpr (BITS == 4) {  // rows g, g+8: 8 bytes each; word c >> 1, from byte c & 1
            cv[0] = *reinterpret_cast<const uint32_t*>(blk + 8 * g + 4 * (c >> 1)) >> (8 * (c & 1));
            cv[1] = *reinterpret_cast<const uint32_t*>(blk + 8 * (g + 8) + 4 * (c >> 1)) >> (8 * (c & 1));
          } else if constexpr (BITS == 8) {
            cv[0] = *reinterpret_cast<const uint32_t*>(blk + (bit_g >> 3));
            cv[1] = *reinterpret_cast<const uint32_t*>(blk + (bit_g8 >> 3));
          } else if constexpr (BITS == 2) {
            cv[0] = blk[bit_g >> 3];
            cv[1] = blk[bit_g8 >> 3];
          } else {
            const uint32_t* w0 = reinterpret_cast<const uint32_t*>(blk) + (bit_g >> 5);
            const uint32_t* w1 = reinterpret_cast<const uint32_t*>(blk) + (bit_g8 >> 5);
            cv[0] = __funnelshift_r(w0[0], w0[1], bit_g & 31);
            cv[1] = __funnelshift_r(w1[0], w1[1], bit_g8 & 31);
          }
          uint32_t afr[4];
          if constexpr (BITS == 4) {  // rows g, g+8: the word of channels 8 (c >> 1) .., from nibble 2 (c & 1)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const uint32_t u = cv[hh];
              afr[hh] = nib_lo_pair(u);      // channels b, b + 4
              afr[2 + hh] = nib_hi_pair(u);  // channels b + 1, b + 5
            }
          } else {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              constexpr uint32_t M = (1u << BITS) - 1u;
              const uint32_t v = cv[hh];
              afr[hh] = f16_sub1024(0x64006400u | (v & M) | (((v >> BITS) & M) << 16));
              afr[2 + hh] = f16_sub1024(0x64006400u | ((v >> (2 * BITS)) & M) | (((v >> (3 * BITS)) & M) << 16));
            }
          }
          const float sk = __half2float(ks[kb * NG + r]);
  #pragma unroll
          for (int tt = 0; tt < NT; ++tt) {
            const uint2 bq = *reinterpret_cast<const uint2*>(bqs + 2 * ((r * NT + tt) * 32 + lane));
            float d[4];
            mma_f16_16816_z(d, afr, bq.x, bq.y);
  #pragma unroll
            for (int e = 0; e < 4; ++e) acc[tt][e] = __fmaf_rn(sk, d[e], acc[tt][e]);
          }
        }
        // hi + lo terms; then columns 2c, 2c+1 are heads 2c, 2c+1 (threads c < 2 for GQ <= 4)
        float sv[4];
  #pragma unroll
        for (int e = 0; e < 4; ++e) {
          if constexpr (NT == 2) {
            sv[e] = acc[0][e] + acc[1][e];
          } else {
            sv[e] = acc[0][e] + __shfl_xor_sync(0xffffffffu, acc[0][e], 2);
          }
        }
  #pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = 2 * c + (e & 1), t = kb * 16 + g + 8 * (e >> 1);
          if ((NT == 2 || c < 2) && j < GQ) sc[t * GQ + j] = __fmaf_rn(sv[e], qinv[j], zsum[kb * GQ + j]);
        }
      }
    }
    __syncthreads();

    // ---- softmax over the chunk, thread = token (threads past the chunk only reduce) ----
    {
      const int t = tid;
      const bool live = t < ntok;
      const bool row = t < kChunk;  // threads past the chunk take part in the reductions only
      float sj[GQ];
  #pragma unroll
      for (int j = 0; j < GQ; ++j) {
        sj[j] = live ? sc[t * GQ + j] : -INFINITY;
        float m = sj[j];
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
        const float pj = live ? __expf(sj[j] - stat[j]) : 0.0f;
        ls[j] = pj;
        const float ps = pj * kPScale;
        const __half hi = __float2half_rn(ps);
        const __half lo = __float2half_rn(ps - __half2float(hi));
        if (row) {
          pb[j * kChunk + t] = __half_as_ushort(hi);  // lo terms: column 4 + j (GQ <= 4) or 8 + j
          pb[(NT == 2 ? 8 + j : 4 + j) * kChunk + t] = __half_as_ushort(lo);
        }
      }
      if constexpr (NT == 1) {  // unused columns of the tile are zero
        for (int j = GQ; j < 4 && row; ++j) {
          pb[j * kChunk + t] = 0;
          pb[(4 + j) * kChunk + t] = 0;
        }
      }
      __syncthreads();  // red is reused below
  #pragma unroll
      for (int j = 0; j < GQ; ++j) {
        float s16 = ls[j];  // per 16-token block (half a warp), then per warp
  #pragma unroll
        for (int o = 8; o >= 1; o >>= 1) s16 += __shfl_xor_sync(0xffffffffu, s16, o);
        if ((lane & 15) == 0 && row) psum[(t >> 4) * GQ + j] = s16;
        const float s32 = s16 + __shfl_xor_sync(0xffffffffu, s16, 16);
        if (lane == 0) red[warp * GQ + j] = s32;
      }
    }
    __syncthreads();

    // ---- value sums on the tensor cores: warp w takes group w mod NG ----
    // A = value codes transposed: row m = g is channel 2g of the group, m = g+8 is
    // channel 2g+1; k slots 2c, 2c+1 / 2c+8, 2c+9 are tokens 4c, 4c+1 / 4c+2, 4c+3.
    {
      constexpr int WPG = 8 / NG;  // warps per group: 1 (d = 128) or 2 (d = 64)
      const int r = warp % NG, part = warp / NG;
      // byte g & 3 of the first word to byte 0, of the second to byte 2 (4-bit values)
      const uint32_t vsel = (uint32_t)(g & 3) * 0x0011u + (uint32_t)(4 + (g & 3)) * 0x1100u;
      const int per = NBLK / WPG;
      float o[NT][4];
  #pragma unroll
      for (int tt = 0; tt < NT; ++tt)
  #pragma unroll
        for (int e = 0; e < 4; ++e) o[tt][e] = 0.0f;
      float oz[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // zero-point terms of this thread's (channel, head) pairs
      for (int kb = part * per; kb < min(nblk, part * per + per); ++kb) {
        const uint8_t* blk = vc + (kb * NG + r) * BLK;
        uint32_t afr[4];
        if constexpr (BITS == 4) {
          // token 4c + u is 8 bytes (16 channels); byte g holds channels 2g (low nibble) and
          // 2g + 1: pick it from two tokens' words at once, then both nibble pairs
          uint32_t w[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) w[u] = *reinterpret_cast<const uint32_t*>(blk + (4 * c + u) * 8 + 4 * (g >> 2));
          const uint32_t x01 = __byte_perm(w[0], w[1], vsel), x23 = __byte_perm(w[2], w[3], vsel);
          afr[0] = nib_lo_pair(x01);
          afr[1] = nib_hi_pair(x01);
          afr[2] = nib_lo_pair(x23);
          afr[3] = nib_hi_pair(x23);
        } else {
          uint32_t lo2[4], hi2[4];  // per token 4c + u: codes of channels 2g, 2g+1
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int bit = ((4 * c + u) * 16 + 2 * g) * BITS;
            uint32_t v;
            if constexpr (BITS == 8) {
              v = *reinterpret_cast<const uint16_t*>(blk + (bit >> 3));
            } else if constexpr (BITS == 2) {
              v = (uint32_t)blk[bit >> 3] >> (bit & 7);
            } else {
              const uint32_t* wp = reinterpret_cast<const uint32_t*>(blk) + (bit >> 5);
              v = __funnelshift_r(wp[0], wp[1], bit & 31);
            }
            constexpr uint32_t M = (1u << BITS) - 1u;
            lo2[u] = v & M;
            hi2[u] = (v >> BITS) & M;
          }
          afr[0] = f16_sub1024(0x64006400u | lo2[0] | (lo2[1] << 16));
          afr[1] = f16_sub1024(0x64006400u | hi2[0] | (hi2[1] << 16));
          afr[2] = f16_sub1024(0x64006400u | lo2[2] | (lo2[3] << 16));
          afr[3] = f16_sub1024(0x64006400u | hi2[2] | (hi2[3] << 16));
        }
        const float sv = __half2float(vs[kb * NG + r]) * (1.0f / kPScale), zv = __half2float(vz[kb * NG + r]);
  #pragma unroll
        for (int tt = 0; tt < NT; ++tt) {
          const uint2 bb = *reinterpret_cast<const uint2*>(pb + (tt * 8 + g) * kChunk + kb * 16 + 4 * c);
          float d[4];
          mma_f16_16816_z(d, afr, bb.x, bb.y);
  #pragma unroll
          for (int e = 0; e < 4; ++e) o[tt][e] = __fmaf_rn(sv, d[e], o[tt][e]);
        }
  #pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = 2 * c + (e & 1);
          if (j < GQ) oz[e] = __fmaf_rn(zv, psum[kb * GQ + j], oz[e]);
        }
      }
      float ov[4];
  #pragma unroll
      for (int e = 0; e < 4; ++e) {
        if constexpr (NT == 2) {
          ov[e] = o[0][e] + o[1][e];
        } else {
          ov[e] = o[0][e] + __shfl_xor_sync(0xffffffffu, o[0][e], 2);
        }
        ov[e] += oz[e];
      }
    // ov[e]: channel 2g + (e >> 1) of group r, head 2c + (e & 1) (d = 64: the halves added in order)
      const bool mine = (NT == 2 || c < 2) && part == 0;
      if constexpr (WPG == 2) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = 2 * c + (e & 1);
          if ((NT == 2 || c < 2) && j < GQ) po[(part * GQ + j) * D + 16 * r + 2 * g + (e >> 1)] = ov[e];
        }
      }
      // online softmax: merge this chunk into the running (max, sum, o)
      if (tid < GQ) {
        float s = 0.0f;
        for (int w = 0; w < 8; ++w) s += red[w * GQ + tid];
        const float m_old = run[tid], m_new = fmaxf(m_old, stat[tid]);
        const float w_old = __expf(m_old - m_new), w_new = __expf(stat[tid] - m_new);
        run[tid] = m_new;
        run[8 + tid] = __fmaf_rn(run[8 + tid], w_old, s * w_new);
        run[16 + tid] = w_old;
        run[24 + tid] = w_new;
      }
      __syncthreads();
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = 2 * c + (e & 1);
        if (mine && j < GQ) {
          float v = ov[e];
          if constexpr (WPG == 2) {
            const int ch = 16 * r + 2 * g + (e >> 1);
            v = po[j * D + ch] + po[(GQ + j) * D + ch];
          }
          orun[e] = __fmaf_rn(orun[e], run[16 + j], v * run[24 + j]);
        }
      }
    }
  }
  // write this split's partial
  {
    const int r = warp % NG, part = warp / NG;
    float* out = a.partial + ((((long long)lz * a.k.B + b) * a.hq + h * GQ) * a.n_chunks + split) * (D + 2);
    const long long head_stride = (long long)a.n_chunks * (D + 2);
    const bool mine = (NT == 2 || c < 2) && part == 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = 2 * c + (e & 1);
      if (mine && j < GQ) out[j * head_stride + 2 + 16 * r + 2 * g + (e >> 1)] = orun[e];
    }
    if (tid < GQ) {
      out[tid * head_stride + 0] = run[tid];
      out[tid * head_stride + 1] = run[8 + tid];
    }
  }
}

// out[l][b][hq] = G_V^T (sum_k e^(m_k - M) o_k) / (sum_k e^(m_k - M) l_k)
// (the chunk weights are formed once, in parallel, then every channel's sum
// over the chunks reads independent partials)
template <int D>
__global__ void __launch_bounds__(D) attn_combine_kernel(AttnArgs a) {
  constexpr int NG = D / 16, NW = D / 32;
  extern __shared__ float wk[];  // [n_chunks] e^(m_k - M)
  __shared__ float og[D];
  __shared__ float red[NW];
  const int hq = blockIdx.x, b = blockIdx.y, lz = blockIdx.z;
  const int l = a.l0 + lz, h = hq / (a.hq / a.k.H);
  const int c = threadIdx.x, lane = c & 31, w = c >> 5;
  const float* part = a.partial + ((((long long)lz * a.k.B + b) * a.hq + hq) * a.n_chunks) * (D + 2);
  float m = -INFINITY;
  for (int k = c; k < a.n_chunks; k += D) m = fmaxf(m, part[k * (D + 2)]);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[w] = m;
  __syncthreads();
  float M = red[0];
#pragma unroll
  for (int i = 1; i < NW; ++i) M = fmaxf(M, red[i]);
  float ls = 0.0f;
  for (int k = c; k < a.n_chunks; k += D) {
    const float wt = __expf(part[k * (D + 2)] - M);
    wk[k] = wt;
    ls = __fmaf_rn(wt, part[k * (D + 2) + 1], ls);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
  __syncthreads();  // every thread has read red; the weights are in place
  if (lane == 0) red[w] = ls;
  __syncthreads();
  float Ls = red[0];
#pragma unroll
  for (int i = 1; i < NW; ++i) Ls += red[i];
  float O = 0.0f;
#pragma unroll 4
  for (int k = 0; k < a.n_chunks; ++k) O = __fmaf_rn(wk[k], part[k * (D + 2) + 2 + c], O);
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

template <int D, int BITS, int GQ, int kChunk>
cudaError_t attn_launch(const AttnArgs& a, cudaStream_t st) {
  constexpr int NG = D / 16;
  constexpr int CODE_BYTES = kChunk * D * BITS / 8;
  constexpr int NBLK = kChunk / 16;
  constexpr int NT = GQ == 8 ? 2 : 1;
  constexpr int NCOL = 8 * NT;
  constexpr int STAGE = 2 * (CODE_BYTES + 16) + 4 * NBLK * NG * 2;
  const int smem_floats = GQ * D + GQ * NG + 8 + kChunk * GQ + NBLK * GQ + 8 * GQ + 8 + 32 + 2 * GQ * D + NBLK * GQ +
                          NG * NT * 64;
  const size_t smem = 2 * (size_t)STAGE + 4 * (size_t)smem_floats + 2 * (size_t)NCOL * kChunk;
  auto kern = attn_partial_kernel<D, BITS, GQ, kChunk>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.n_chunks, a.k.B * a.k.H, a.n_layers);  // one CTA per split of cpc chunks
  kern<<<grid, kAttnThreads, smem, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 cgrid(a.hq, a.k.B, a.n_layers);
  const size_t csmem = (size_t)a.n_chunks * sizeof(float);
  if (csmem > 48 * 1024) {
    e = cudaFuncSetAttribute(attn_combine_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)csmem);
    if (e != cudaSuccess) return e;
  }
  attn_combine_kernel<D><<<cgrid, D, csmem, st>>>(a);
  return cudaGetLastError();
}

template <int D, int BITS>
cudaError_t attn_gq(const AttnArgs& a, cudaStream_t st) {
  switch (a.hq / a.k.H) {
    case 1: return a.chunk == kLargeChunk ? attn_launch<D, BITS, 1, kLargeChunk>(a, st) : attn_launch<D, BITS, 1, kSmallChunk>(a, st);
    case 2: return a.chunk == kLargeChunk ? attn_launch<D, BITS, 2, kLargeChunk>(a, st) : attn_launch<D, BITS, 2, kSmallChunk>(a, st);
    case 4: return a.chunk == kLargeChunk ? attn_launch<D, BITS, 4, kLargeChunk>(a, st) : attn_launch<D, BITS, 4, kSmallChunk>(a, st);
    case 8: return a.chunk == kLargeChunk ? attn_launch<D, BITS, 8, kLargeChunk>(a, st) : attn_launch<D, BITS, 8, kSmallChunk>(a, st);
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
  const uint64_t chunks = (uint64_t)(n_tokens + kSmallChunk - 1) / kSmallChunk;  // at most one partial per chunk
  return (uint64_t)n_layers * k.B * hq * chunks * (k.d + 2) * sizeof(float);
}

cudaError_t launch_decode_attention(AttnArgs a, int num_sms, cudaStream_t st) {
  // A call whose CTAs of four 256-token chunks fit in one wave (two per SM) runs
  // them.  Larger calls take 128-token chunks, four CTAs per SM, as many per CTA
  // as keep at least six CTAs per SM, so that they run and merge fewer partials.
  const long long heads = (long long)a.n_layers * a.k.B * a.k.H;
  const int n_large = (a.n_tokens + kLargeChunk - 1) / kLargeChunk;
  if (heads * ((n_large + 3) / 4) <= 2LL * num_sms) {
    a.chunk = kLargeChunk;
    a.cpc = 4;
  } else {
    a.chunk = kSmallChunk;
    const int n_small = (a.n_tokens + kSmallChunk - 1) / kSmallChunk;
    a.cpc = kMaxCpc;
    while (a.cpc > 1 && heads * ((n_small + a.cpc - 1) / a.cpc) < 6LL * num_sms) a.cpc >>= 1;
  }
  a.n_chunks = ((a.n_tokens + a.chunk - 1) / a.chunk + a.cpc - 1) / a.cpc;  // partials per (layer, batch, query head)
  return a.k.d == 128 ? attn_bits<128>(a, st) : attn_bits<64>(a, st);
}

}  // namespace cg
