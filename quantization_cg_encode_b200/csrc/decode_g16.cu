// Fused unpack + dequantize + inverse gauge for g = 16 (d_head 64 or 128, any
// bit width, block-uniform ranges of 16 x 16 or 16 x d_head).
//
// Codec-Gauge, Figure 1 / Method: the inverse gauge G^T restores K and V before
// attention, and the implementation charges this explicit recovery in timing.
//
// With s and z constant over a range block (which always covers whole groups),
//   x_hat_n = sum_c G[c][n] (s q_c + z) = s (sum_c q_c G[c][n]) + z colsum_n,
// so the per-token work is a 16 x 16 contraction of exact small integers q with
// G.  It runs on the tensor cores as mma.sync m16n8k16 (fp16 in, fp32
// accumulate): A = the 16-token x 16-channel code tile (integers <= 255 are
// exact in fp16), B = G split into fp16 hi + lo parts (G = hi + lo to about
// 2^-22 relative), two n-halves, four MMAs per tile and group.  The k order of
// A and B is permuted consistently so that each thread reads 4 adjacent codes.
//
// Structure (persistent, one CTA per SM): a producer warp streams stages of up
// to 16 code tiles (contiguous, 16 KB at d = 128 and 4 bits) into a shared-
// memory ring with one 1-D bulk copy each; consumer warp r owns group r and
// stores its bf16 outputs straight to global memory; lane j of each warp reads
// the step and zero point of the stage's tile j, handed out by shuffle.
#include <cuda.h>

#include "cg_kernels.cuh"

namespace cg {

namespace {



__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// fp16 pair {c_lo, c_hi} of two codes (< 256): the fp16 bit patterns
// 0x6400 | c are exactly 1024 + c, and one exact f16x2 subtraction removes the
// 1024.  No conversion instruction is involved.
__device__ __forceinline__ uint32_t f16_sub1024(uint32_t biased) {
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(biased), "r"(0x64006400u));
  return r;
}
__device__ __forceinline__ uint32_t f16pair(uint32_t c_lo, uint32_t c_hi) {
  return f16_sub1024(0x64006400u | c_lo | (c_hi << 16));
}
// Four 4-bit codes c0..c3 (v = c0 | c1 << 4 | c2 << 8 | c3 << 12) -> fp16 pairs
// {c0, c1} and {c2, c3}, built with byte permutes.
__device__ __forceinline__ void f16pairs_nib4(uint32_t v, uint32_t& p01, uint32_t& p23) {
  const uint32_t e = (v & 0x0F0Fu) | 0x64640000u;          // bytes c0, c2, 0x64, 0x64
  const uint32_t o = ((v >> 4) & 0x0F0Fu) | 0x64640000u;   // bytes c1, c3, 0x64, 0x64
  p01 = f16_sub1024(__byte_perm(e, o, 0x6420));
  p23 = f16_sub1024(__byte_perm(e, o, 0x6521));
}
__device__ __forceinline__ uint32_t f16_bits(float x) { return (uint32_t)__half_as_ushort(__float2half_rn(x)); }

template <int D, int BITS, bool WFULL>
struct DCfg {
  static constexpr int NW = D / 16;
  static constexpr int THREADS = (NW + 1) * 32;
  static constexpr int CODE_TILE = 16 * D * BITS / 8;
  // one bulk copy moves a whole stage of tiles (>= 8 KB: smaller copies leave
  // the copy engine short of HBM bandwidth)
  static constexpr int STAGE_TILES = D == 128 ? 16 : 32;
  static constexpr int CODE_STAGE = (STAGE_TILES * CODE_TILE + 16 + 127) / 128 * 128;  // +16: slack for window reads
  static constexpr int NST = CODE_STAGE > 24 * 1024 ? 4 : 6;
  static constexpr int SMEM = 128 + NST * CODE_STAGE + 2 * NST * 8;
};

template <int D, int BITS, bool WFULL>
__global__ void __launch_bounds__(DCfg<D, BITS, WFULL>::THREADS, 1) decode_g16_kernel(CodecArgs a) {
  using C = DCfg<D, BITS, WFULL>;
  constexpr int kStages = C::NST;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* stages = reinterpret_cast<unsigned char*>(((uintptr_t)smem_raw + 127) & ~(uintptr_t)127);
  uint64_t* full = reinterpret_cast<uint64_t*>(stages + kStages * C::CODE_STAGE);
  uint64_t* empty = full + kStages;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Work unit = one stage: up to STAGE_TILES consecutive tiles of one head slice.
  const int tps = a.nt / 16;
  const int sps = (tps + C::STAGE_TILES - 1) / C::STAGE_TILES;
  const long long total = (long long)sps * a.k.slices();
  const long long u0 = total * blockIdx.x / gridDim.x;
  const long long u1 = total * (blockIdx.x + 1) / gridDim.x;
  const int n_units = (int)(u1 - u0);
  const long long slice_code_bytes = (long long)a.k.T * D * BITS / 8;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], C::NW);
    }
    fence_mbar_init();
  }
  __syncthreads();
  if (n_units == 0) return;
  long long slice0 = u0 / sps;
  const int sq0 = (int)(u0 - slice0 * sps);

  if (warp == C::NW) {  // ---------------- producer ----------------
    if (lane == 0) {
      long long slice = slice0;
      int sq = sq0;
      for (int q = 0; q < n_units; ++q) {
        const int s = q % kStages;
        mbar_wait(&empty[s], ((uint32_t)(q / kStages) & 1u) ^ 1u, a.status);
        const int nvalid = min(C::STAGE_TILES, tps - C::STAGE_TILES * sq);
        const uint32_t bytes = (uint32_t)(nvalid * C::CODE_TILE);
        mbar_arrive_expect_tx(&full[s], bytes);
        bulk_g2s(stages + s * C::CODE_STAGE,
                 a.codes_in + slice * slice_code_bytes + (long long)(a.t0 / 16 + C::STAGE_TILES * sq) * C::CODE_TILE,
                 bytes, &full[s]);
        if (++sq == sps) {
          sq = 0;
          ++slice;
        }
      }
    }
    return;
  }

  // ---------------- consumers ----------------
  const int r = warp;
  const int g4 = lane >> 2, q4 = lane & 3;
  const int nblk = WFULL ? 1 : D / 16;
  uint32_t bfr[2][2][2];  // [n-half][hi/lo][b0/b1], fp16 pairs
  float colsum[4];        // output channels 2q, 2q+1, 8+2q, 9+2q
  auto load_g = [&](long long sl) {
    int l, sk, b, h;
    slice_coords(sl, a.k, l, sk, b, h);
    const float* Gr = a.G + (gauge_set(l, sk, h, a.k) * (D / 16) + r) * 256;  // G[c][n], row-major
#pragma unroll
    for (int nh = 0; nh < 2; ++nh) {
      const int n = 8 * nh + g4;
      const float g0 = __ldg(Gr + (4 * q4 + 0) * 16 + n), g1 = __ldg(Gr + (4 * q4 + 1) * 16 + n);
      const float g2 = __ldg(Gr + (4 * q4 + 2) * 16 + n), g3 = __ldg(Gr + (4 * q4 + 3) * 16 + n);
      const uint32_t h0 = f16_bits(g0), h1 = f16_bits(g1), h2 = f16_bits(g2), h3 = f16_bits(g3);
      const float r0 = g0 - __half2float(__ushort_as_half((unsigned short)h0));
      const float r1 = g1 - __half2float(__ushort_as_half((unsigned short)h1));
      const float r2 = g2 - __half2float(__ushort_as_half((unsigned short)h2));
      const float r3 = g3 - __half2float(__ushort_as_half((unsigned short)h3));
      bfr[nh][0][0] = h0 | (h1 << 16);
      bfr[nh][0][1] = h2 | (h3 << 16);
      bfr[nh][1][0] = f16_bits(r0) | (f16_bits(r1) << 16);
      bfr[nh][1][1] = f16_bits(r2) | (f16_bits(r3) << 16);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int n = (k < 2) ? 2 * q4 + k : 8 + 2 * q4 + (k - 2);
      float acc = 0.0f;
#pragma unroll
      for (int c = 0; c < 16; ++c) acc += __ldg(Gr + c * 16 + n);
      colsum[k] = acc;
    }
  };

  // steps and zero points of a stage: lane j takes tile j (raw fp16 pairs,
  // fetched one stage ahead so the loads are in flight during the previous stage)
  auto fetch_sz = [&](long long sl, int sqq) -> uint32_t {
    const int nv = min(C::STAGE_TILES, tps - C::STAGE_TILES * sqq);
    if (lane >= nv) return 0u;
    const long long bidx = (sl * (a.k.T / 16) + a.t0 / 16 + C::STAGE_TILES * sqq + lane) * nblk + (WFULL ? 0 : r);
    return (uint32_t)__ldg(a.scales_in + bidx) | ((uint32_t)__ldg(a.zeros_in + bidx) << 16);
  };
  long long slice = slice0;
  int sq = sq0;
  load_g(slice);
  uint32_t sz_next = fetch_sz(slice, sq);
  for (int q = 0; q < n_units; ++q) {
    const int s = q % kStages;
    const int nvalid = min(C::STAGE_TILES, tps - C::STAGE_TILES * sq);
    const int tile0 = a.t0 / 16 + C::STAGE_TILES * sq;
    float sfv[1], zfv[1];
    sfv[0] = __half2float(__ushort_as_half((unsigned short)(sz_next & 0xffffu)));
    zfv[0] = __half2float(__ushort_as_half((unsigned short)(sz_next >> 16)));
    if (q + 1 < n_units) {
      const bool wrap = sq + 1 == sps;
      sz_next = fetch_sz(wrap ? slice + 1 : slice, wrap ? 0 : sq + 1);
    }
    mbar_wait(&full[s], (uint32_t)(q / kStages) & 1u, a.status);
    const unsigned char* sbase = stages + s * C::CODE_STAGE;
    uint16_t* obase = a.kv_out + (slice * a.k.T + (long long)tile0 * 16) * D + 16 * r;
    for (int tl = 0; tl < nvalid; ++tl) {
      const float sf = __shfl_sync(0xffffffffu, sfv[0], tl);
      const float zf = __shfl_sync(0xffffffffu, zfv[0], tl);
      const unsigned char* cbuf = sbase + tl * C::CODE_TILE;
      uint32_t afr[4];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int row = g4 + 8 * half;
        const int bit = (WFULL ? (row * D + 16 * r + 4 * q4) : (r * 256 + row * 16 + 4 * q4)) * BITS;
        const uint32_t* w = reinterpret_cast<const uint32_t*>(cbuf) + (bit >> 5);
        const uint32_t v = __funnelshift_r(w[0], w[1], bit & 31);
        // k slots 2q, 2q+1 <- channels 4q, 4q+1;  k slots 2q+8, 2q+9 <- channels 4q+2, 4q+3
        if constexpr (BITS == 4) {
          f16pairs_nib4(v, afr[half], afr[2 + half]);
        } else {
          constexpr uint32_t M = (1u << BITS) - 1u;
          const uint32_t c0 = v & M, c1 = (v >> BITS) & M, c2 = (v >> (2 * BITS)) & M, c3 = (v >> (3 * BITS)) & M;
          afr[half] = f16pair(c0, c1);
          afr[2 + half] = f16pair(c2, c3);
        }
      }
      float acc[2][4];
#pragma unroll
      for (int nh = 0; nh < 2; ++nh) {
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[nh][k] = 0.0f;
        mma_f16_16816(acc[nh], afr, bfr[nh][0][0], bfr[nh][0][1]);
        mma_f16_16816(acc[nh], afr, bfr[nh][1][0], bfr[nh][1][1]);
      }
      // x_hat = s * acc + z * colsum, bf16 RNE, stored straight to global memory
      uint16_t* orow = obase + (long long)tl * 16 * D;
#pragma unroll
      for (int nh = 0; nh < 2; ++nh) {
        const float cz0 = zf * colsum[2 * nh], cz1 = zf * colsum[2 * nh + 1];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int row = g4 + 8 * half;
          const float x0 = __fmaf_rn(sf, acc[nh][2 * half], cz0);
          const float x1 = __fmaf_rn(sf, acc[nh][2 * half + 1], cz1);
          *reinterpret_cast<uint32_t*>(orow + row * D + 8 * nh + 2 * q4) = pack_bf16x2(x0, x1);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    if (++sq == sps) {
      sq = 0;
      ++slice;
      if (q + 1 < n_units) load_g(slice);
    }
  }
}

template <int D, int BITS, bool WFULL>
cudaError_t launch_one(const CodecArgs& a, int num_sms, cudaStream_t st) {
  using C = DCfg<D, BITS, WFULL>;
  auto kern = decode_g16_kernel<D, BITS, WFULL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const long long total = (long long)((a.nt / 16 + C::STAGE_TILES - 1) / C::STAGE_TILES) * a.k.slices();
  const int grid = (int)(total < num_sms ? total : num_sms);
  kern<<<grid, C::THREADS, C::SMEM, st>>>(a);
  return cudaGetLastError();
}

template <int D, int BITS>
cudaError_t launch_w(const CodecArgs& a, int num_sms, cudaStream_t st) {
  return a.W == 16 ? launch_one<D, BITS, false>(a, num_sms, st) : launch_one<D, BITS, true>(a, num_sms, st);
}

template <int D>
cudaError_t launch_b(const CodecArgs& a, int num_sms, cudaStream_t st) {
  switch (a.bits) {
    case 2: return launch_w<D, 2>(a, num_sms, st);
    case 3: return launch_w<D, 3>(a, num_sms, st);
    case 4: return launch_w<D, 4>(a, num_sms, st);
    case 6: return launch_w<D, 6>(a, num_sms, st);
    case 8: return launch_w<D, 8>(a, num_sms, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode_g16(const CodecArgs& a, int num_sms, cudaStream_t st) {
  if (a.nt == 0) return cudaSuccess;
  return a.k.d == 128 ? launch_b<128>(a, num_sms, st) : launch_b<64>(a, num_sms, st);
}

}  // namespace cg
