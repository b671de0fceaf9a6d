// KIVI-style decode for g = 16 and d_head = 128 on the tensor cores: unpack,
// dequantize and apply G^T per 16-channel group, bf16 out.
//
// Codec-Gauge, Experimental setup: KIVI-style backend (keys with one range per
// channel and 32 tokens, values with one range per token and 32 channels);
// Method: the inverse gauge restores K and V before attention, explicitly.
//
// A warp decodes a unit of 32 tokens x 128 channels of one head slice, whose
// codes (512 b bytes) and steps / zero points (128 each) are contiguous in
// both layouts.  Per 16-token tile and group, mma.sync m16n8k16 (fp16 in, fp32
// accumulate) against G split into fp16 hi + lo (2^-22):
//   * values: the step and zero point are one per token, so
//       x_hat_n = s_t sum_c q_c G[c][n] + z_t colsum_n
//     with the codes themselves as the A operand (integers, exact in fp16);
//   * keys: the step and zero point vary with the channel (and are fixed
//     over the unit's 32 tokens), so the step moves into the gauge:
//       x_hat_n = sum_c q_c (s_c G[c][n]) + sum_c z_c G[c][n],
//     with the codes again as the A operand, G'[c][n] = 2^e s_c G[c][n] split
//     into fp16 hi + lo once per unit (2^e a power of two that puts the largest
//     step near 2^13, undone exactly afterwards) and the second sum, a vector
//     per unit, added in the epilogue.
// The k order of A and B is permuted consistently (each thread reads 4
// adjacent channels), and so are the MMA rows: row g4 (+ 8) of 16-token tile
// tt is token 4 g4 + 2 tt (+ 1) of the unit, so a thread's tokens are four
// consecutive ones and each key record yields them in one read.  Each bf16
// 16-token tile goes through a padded shared-memory staging with stmatrix and
// leaves with full-line 16-byte stores.  The per-warp buffers are sized by the
// code width, so that two CTAs (16 warps) share an SM at every code width.
#include "cg_kernels.cuh"

namespace cg {

namespace {

constexpr int kWarps = 8;
constexpr int kPitch = 2 * 128 + 16;  // staging row: 256 B + 16 B pad (distinct bank groups per 8 rows)
constexpr int kStg = 16 * kPitch;     // one 16-token tile
// per warp: output staging, then two input buffers (the unit's 512 b code
// bytes + 16 B slack, steps, zero points), then the column sums of G
template <int BITS>
__host__ __device__ constexpr int in_buf_bytes() {
  return 512 * BITS + 16 + 2 * 256;
}
template <int BITS>
__host__ __device__ constexpr int warp_smem_bytes() {
  return kStg + 2 * in_buf_bytes<BITS>() + 512;
}

__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// fp16 pair {c_lo, c_hi} of two codes (< 256): 0x6400 | c is exactly 1024 + c
__device__ __forceinline__ uint32_t f16pair(uint32_t c_lo, uint32_t c_hi) {
  return f16_sub1024(0x64006400u | c_lo | (c_hi << 16));
}
__device__ __forceinline__ uint32_t f16_bits(float x) { return (uint32_t)__half_as_ushort(__float2half_rn(x)); }
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(smem)), "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async8(void* smem, const void* gmem) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"((uint32_t)__cvta_generic_to_shared(smem)), "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void stmatrix_x4(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
  asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(r0), "r"(r1),
               "r"(r2), "r"(r3)
               : "memory");
}
// 32 bits starting at bit `bit` of the little-endian stream at p (reads two words)
__device__ __forceinline__ uint32_t bits_at(const unsigned char* p, int bit) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(p) + (bit >> 5);
  return __funnelshift_r(w[0], w[1], bit & 31);
}
// The same for a field of four codes at the offsets this decoder reads: with 2, 4 or 8
// bits per code such a field never crosses a 32-bit word, so one word suffices.
template <int BITS>
__device__ __forceinline__ uint32_t field4_at(const unsigned char* p, int bit) {
  if constexpr (BITS == 2 || BITS == 4 || BITS == 8) {
    return reinterpret_cast<const uint32_t*>(p)[bit >> 5] >> (bit & 31);
  } else {
    return bits_at(p, bit);
  }
}

}  // namespace

template <int BITS>
__global__ void __launch_bounds__(kWarps * 32, 2) kivi_decode_g16_kernel(CodecArgs a) {
  constexpr int D = 128, NG = 8;
  constexpr uint32_t M = (1u << BITS) - 1u;
  constexpr int UNIT_BYTES = 512 * BITS;
  constexpr int kCodeBuf = UNIT_BYTES, kInBuf = in_buf_bytes<BITS>(), kWarpSmem = warp_smem_bytes<BITS>();
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned char* base = smem_raw + warp * kWarpSmem;
  unsigned char* stg = base;
  float* csum = reinterpret_cast<float*>(base + kStg + 2 * kInBuf);       // 128 column sums of G
  const uint32_t st_addr =
      (uint32_t)__cvta_generic_to_shared(stg) + ((lane & 7) + 8 * ((lane >> 3) & 1)) * kPitch + ((lane >> 4) * 8) * 2;
  const int g4 = lane >> 2, q4 = lane & 3;

  const int ntg = a.nt / 32;
  const long long units = a.k.slices() * ntg;
  const long long slice_bytes = (long long)a.k.T * D * BITS / 8;
  const long long slice_ranges = (long long)a.k.T * D / 32;

  uint32_t bfr[NG][2][2][2];  // [group][n-half][hi/lo][b0/b1], fp16 pairs of G
  long long loaded = -1;
  // a unit's codes, steps and zero points (contiguous in both layouts) into input buffer p
  auto prefetch = [&](long long uu, int p) {
    const long long sl = uu / ntg;
    const int tg = a.t0 / 32 + (int)(uu - sl * ntg);
    unsigned char* ib = base + kStg + p * kInBuf;
    const unsigned char* src = a.codes_in + sl * slice_bytes + (long long)tg * UNIT_BYTES;
#pragma unroll
    for (int k = 0; k < UNIT_BYTES / 512; ++k) cp_async16(ib + 16 * (32 * k + lane), src + 16 * (32 * k + lane));
    const long long r0 = sl * slice_ranges + (long long)tg * 128;
    cp_async8(ib + kCodeBuf + 16 + 8 * lane, a.scales_in + r0 + 4 * lane);
    cp_async8(ib + kCodeBuf + 16 + 256 + 8 * lane, a.zeros_in + r0 + 4 * lane);
  };
  const long long ustride = (long long)gridDim.x * kWarps;
  long long u = (long long)blockIdx.x * kWarps + warp;
  if (u < units) prefetch(u, 0);
  cp_async_commit();
  for (int it = 0; u < units; u += ustride, ++it) {
    const int p = it & 1;
    if (u + ustride < units) prefetch(u + ustride, p ^ 1);  // the next unit loads during this one
    cp_async_commit();
    cp_async_wait<1>();
    __syncwarp();
    const unsigned char* cbuf = base + kStg + p * kInBuf;
    const uint16_t* sbuf = reinterpret_cast<const uint16_t*>(cbuf + kCodeBuf + 16);
    const uint16_t* zbuf = sbuf + 128;
    const long long slice = u / ntg;
    const int tgroup = a.t0 / 32 + (int)(u - slice * ntg);
    int l, sk, b, h;
    slice_coords(slice, a.k, l, sk, b, h);
    const bool key = sk == 0;
    if (!key && slice != loaded) {  // values: G fragments and column sums of this head slice
      const float* G0 = a.G + gauge_set(l, sk, h, a.k) * NG * 256;
#pragma unroll
      for (int r = 0; r < NG; ++r) {
        const float* Gr = G0 + r * 256;  // G[c][n], row-major
#pragma unroll
        for (int nh = 0; nh < 2; ++nh) {
          const int n = 8 * nh + g4;
          float gv[4];
#pragma unroll
          for (int m = 0; m < 4; ++m) gv[m] = __ldg(Gr + (4 * q4 + m) * 16 + n);
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            hw[m] = f16_bits(gv[m]);
            lw[m] = f16_bits(gv[m] - __half2float(__ushort_as_half((unsigned short)hw[m])));
          }
          bfr[r][nh][0][0] = hw[0] | (hw[1] << 16);
          bfr[r][nh][0][1] = hw[2] | (hw[3] << 16);
          bfr[r][nh][1][0] = lw[0] | (lw[1] << 16);
          bfr[r][nh][1][1] = lw[2] | (lw[3] << 16);
        }
      }
      __syncwarp();
      for (int e = lane; e < D; e += 32) {
        const float* Gr = G0 + (e >> 4) * 256 + (e & 15);
        float acc = 0.0f;
#pragma unroll
        for (int c = 0; c < 16; ++c) acc += __ldg(Gr + c * 16);
        csum[e] = acc;
      }
      loaded = slice;
    }
    // keys: G' = 2^e s_c G per unit (fp16 hi + lo) and the bias sum_c z_c G[c][n] in csum
    float kunscale = 1.0f;
    if (key) {
      float smax = 0.0f;
#pragma unroll
      for (int m = 0; m < 4; ++m) smax = fmaxf(smax, __half2float(__ushort_as_half(sbuf[4 * lane + m])));
      smax = warp_max_f32(smax);
      float kscale = 1.0f;
      if (smax > 0.0f) {  // smax in [2^x, 2^(x+1)): scale 2^(13 - x), exact both ways (x in [-24, 15])
        const int x = (int)((__float_as_uint(smax) >> 23) & 0xffu) - 127;
        kscale = __uint_as_float((uint32_t)(127 + 13 - x) << 23);
        kunscale = __uint_as_float((uint32_t)(127 - 13 + x) << 23);
      }
      const float* G0 = a.G + gauge_set(l, sk, h, a.k) * NG * 256;
#pragma unroll
      for (int r = 0; r < NG; ++r) {
        float sc[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) sc[m] = __half2float(__ushort_as_half(sbuf[16 * r + 4 * q4 + m])) * kscale;
#pragma unroll
        for (int nh = 0; nh < 2; ++nh) {
          const float* Gc = G0 + r * 256 + (4 * q4) * 16 + 8 * nh + g4;
          float hi[4], lo[4];
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const float v = __ldg(Gc + m * 16) * sc[m];
            hi[m] = __half2float(__float2half_rn(v));
            lo[m] = v - hi[m];
          }
          const __half2 h01 = __floats2half2_rn(hi[0], hi[1]), h23 = __floats2half2_rn(hi[2], hi[3]);
          const __half2 l01 = __floats2half2_rn(lo[0], lo[1]), l23 = __floats2half2_rn(lo[2], lo[3]);
          bfr[r][nh][0][0] = *reinterpret_cast<const uint32_t*>(&h01);
          bfr[r][nh][0][1] = *reinterpret_cast<const uint32_t*>(&h23);
          bfr[r][nh][1][0] = *reinterpret_cast<const uint32_t*>(&l01);
          bfr[r][nh][1][1] = *reinterpret_cast<const uint32_t*>(&l23);
        }
      }
      {  // bias of channels n = 4 lane .. 4 lane + 3 (group lane / 4)
        const int rg = lane >> 2, n0 = 4 * (lane & 3);
        float4 bsum = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float z = __half2float(__ushort_as_half(zbuf[16 * rg + i]));
          const float4 gv = __ldg(reinterpret_cast<const float4*>(G0 + rg * 256 + i * 16 + n0));
          bsum.x = __fmaf_rn(z, gv.x, bsum.x);
          bsum.y = __fmaf_rn(z, gv.y, bsum.y);
          bsum.z = __fmaf_rn(z, gv.z, bsum.z);
          bsum.w = __fmaf_rn(z, gv.w, bsum.w);
        }
        __syncwarp();  // the previous unit's epilogue has read csum
        *reinterpret_cast<float4*>(csum + 4 * lane) = bsum;
        __syncwarp();
      }
      loaded = -1;  // csum now holds a key bias: a later value slice rebuilds its column sums
    }
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
#pragma unroll
      for (int r = 0; r < NG; ++r) {
        uint32_t pk[2][2];  // [n-half][row half], bf16 pairs
        if (!key) {
          // values: record (token, 32-channel group r / 2), channels 16 (r & 1) + 4 q4 .. + 3
          uint32_t afr[4];
          float sv[2], zv[2];
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int t = 4 * g4 + 2 * tt + half;  // MMA row g4 + 8 half of tile tt
            const int bit = ((t * 4 + (r >> 1)) * 32 + 16 * (r & 1) + 4 * q4) * BITS;
            const uint32_t v = field4_at<BITS>(cbuf, bit);
            const uint32_t c0 = v & M, c1 = (v >> BITS) & M, c2 = (v >> (2 * BITS)) & M, c3 = (v >> (3 * BITS)) & M;
            // k slots 2q, 2q+1 <- channels 4q, 4q+1;  k slots 2q+8, 2q+9 <- channels 4q+2, 4q+3
            afr[half] = f16pair(c0, c1);
            afr[2 + half] = f16pair(c2, c3);
            sv[half] = __half2float(__ushort_as_half(sbuf[t * 4 + (r >> 1)]));
            zv[half] = __half2float(__ushort_as_half(zbuf[t * 4 + (r >> 1)]));
          }
#pragma unroll
          for (int nh = 0; nh < 2; ++nh) {
            float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            mma_f16(acc, afr, bfr[r][nh][0][0], bfr[r][nh][0][1]);
            mma_f16(acc, afr, bfr[r][nh][1][0], bfr[r][nh][1][1]);
            const float2 cs2 = *reinterpret_cast<const float2*>(csum + 16 * r + 8 * nh + 2 * q4);
            pk[nh][0] = pack_bf16x2(__fmaf_rn(sv[0], acc[0], zv[0] * cs2.x), __fmaf_rn(sv[0], acc[1], zv[0] * cs2.y));
            pk[nh][1] = pack_bf16x2(__fmaf_rn(sv[1], acc[2], zv[1] * cs2.x), __fmaf_rn(sv[1], acc[3], zv[1] * cs2.y));
          }
        } else {
          // keys: record (channel c) holds the unit's 32 tokens; this thread's tokens
          // 4 g4 .. 4 g4 + 3 of channel 16 r + 4 q4 + m are 4 BITS consecutive bits
          uint32_t w[4];
#pragma unroll
          for (int m = 0; m < 4; ++m) w[m] = field4_at<BITS>(cbuf, (16 * r + 4 * q4 + m) * 32 * BITS + 4 * g4 * BITS);
          uint32_t afr[4];
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int sh = (2 * tt + half) * BITS;
            afr[half] = f16pair((w[0] >> sh) & M, (w[1] >> sh) & M);
            afr[2 + half] = f16pair((w[2] >> sh) & M, (w[3] >> sh) & M);
          }
#pragma unroll
          for (int nh = 0; nh < 2; ++nh) {
            float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            mma_f16(acc, afr, bfr[r][nh][1][0], bfr[r][nh][1][1]);
            mma_f16(acc, afr, bfr[r][nh][0][0], bfr[r][nh][0][1]);
            const float2 b2 = *reinterpret_cast<const float2*>(csum + 16 * r + 8 * nh + 2 * q4);
            pk[nh][0] = pack_bf16x2(__fmaf_rn(acc[0], kunscale, b2.x), __fmaf_rn(acc[1], kunscale, b2.y));
            pk[nh][1] = pack_bf16x2(__fmaf_rn(acc[2], kunscale, b2.x), __fmaf_rn(acc[3], kunscale, b2.y));
          }
        }
        // tiles (rows 0-7 | 8-15 of this 16-token tile) x (cols 16r .. +7 | 16r+8 .. +15)
        stmatrix_x4(st_addr + 32 * r, pk[0][0], pk[0][1], pk[1][0], pk[1][1]);
      }
      __syncwarp();
      // the tile's 16 rows of 256 B (row g + 8 h is token 4 g + 2 tt + h): each instruction writes two whole rows
      uint16_t* obase = a.kv_out + (slice * a.k.T + 32LL * tgroup) * D;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int row = 2 * k + (lane >> 4), ch = lane & 15;
        const int tok = 4 * (row & 7) + 2 * tt + (row >> 3);
        reinterpret_cast<uint4*>(obase + tok * D)[ch] = *reinterpret_cast<const uint4*>(stg + row * kPitch + ch * 16);
      }
      __syncwarp();
    }
  }
}

namespace {
template <int BITS>
cudaError_t kd_launch(const CodecArgs& a, int num_sms, cudaStream_t st) {
  constexpr int kSmem = kWarps * warp_smem_bytes<BITS>();
  // CTAs per SM: two where their shared memory (plus 1 KB reserved per CTA) fits in 228 KB (every width)
  constexpr int kCtas = 2 * (kSmem + 1024) <= 228 * 1024 ? 2 : 1;
  auto kern = kivi_decode_g16_kernel<BITS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  const long long units = a.k.slices() * (a.nt / 32);
  const long long want = (units + kWarps - 1) / kWarps;
  const int grid = (int)(want < (long long)num_sms * kCtas ? want : (long long)num_sms * kCtas);
  kern<<<grid, kWarps * 32, kSmem, st>>>(a);
  return cudaGetLastError();
}
}  // namespace

bool kivi_decode_g16_supported(const CodecArgs& a) { return a.kivi && a.g == 16 && a.k.d == 128; }

cudaError_t launch_kivi_decode_g16(const CodecArgs& a, int num_sms, cudaStream_t st) {
  if (a.nt == 0) return cudaSuccess;
  switch (a.bits) {
    case 2: return kd_launch<2>(a, num_sms, st);
    case 3: return kd_launch<3>(a, num_sms, st);
    case 4: return kd_launch<4>(a, num_sms, st);
    case 6: return kd_launch<6>(a, num_sms, st);
    case 8: return kd_launch<8>(a, num_sms, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace cg
