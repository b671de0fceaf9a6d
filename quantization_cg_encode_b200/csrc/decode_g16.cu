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
// Structure (persistent, one CTA per SM, 8 warps): stages of up to 16 code
// tiles (contiguous, 16 KB at d = 128 and 4 bits) stream into a shared-memory
// ring with one 1-D bulk copy each (plus the stage's steps and zero points for
// 16 x 16 ranges); the warp that releases a stage last refills it.  Warp w decodes whole
// 16-token tiles (every group, G's fragments for all groups held in
// registers), writes the bf16 results into a padded shared-memory staging tile
// with stmatrix, and copies the tile out with 16-byte stores (the tile is 4 KB
// contiguous in the output, so each store instruction writes two whole rows).
// The steps and zero points of a stage are loaded one stage ahead.
#include <cuda.h>

#include "cg_kernels.cuh"

namespace cg {

namespace {

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
  static constexpr int NG = D / 16;          // channel groups per tile
  static constexpr int NCW = 8;              // warps (no producer warp: 8 warps of up to 255 registers fit
                                             // the 4 x 16K-register scheduler partitions)
  static constexpr int THREADS = NCW * 32;
  static constexpr int CODE_TILE = 16 * D * BITS / 8;
  // one bulk copy moves a whole stage of tiles (>= 8 KB: smaller copies leave
  // the copy engine short of HBM bandwidth)
  static constexpr int STAGE_TILES = D == 128 ? 16 : 32;
  static constexpr int TPW = STAGE_TILES / NCW;  // tiles per consumer warp and stage
  static constexpr int CODE_BYTES = (STAGE_TILES * CODE_TILE + 16 + 127) / 128 * 128;  // +16: slack for window reads
  // W = 16 at d = 128: the stage's steps and zero points travel with its codes
  // (fp16, 8 per tile: 16 bytes, so every bulk copy stays 16-byte aligned and
  // sized); otherwise each warp loads its tiles' values one stage ahead
  static constexpr bool SZ_SMEM = !WFULL && NG == 8;
  static constexpr int SZW = SZ_SMEM ? 1 : (WFULL ? 1 : NG / 2);  // 32-bit words of steps per tile in registers
  static constexpr int SZ_BYTES = SZ_SMEM ? STAGE_TILES * NG * 2 : 0;
  static constexpr int CODE_STAGE = CODE_BYTES + 2 * SZ_BYTES;
  static constexpr int NST = CODE_STAGE > 24 * 1024 ? 4 : 6;
  // bf16 staging of one output tile per consumer warp: rows padded by 16 bytes
  // so the 8 rows of an 8 x 8 stmatrix tile fall into distinct bank groups
  static constexpr int PITCH = 2 * D + 16;
  static constexpr int STG = 16 * PITCH;
  static constexpr int CSUM = NG * 16 * 4;  // column sums of G for the slice, per consumer warp
  static constexpr int SMEM = 128 + NST * CODE_STAGE + NCW * (STG + CSUM) + NST * 8 + NST * 4;
};

// Release of a ring stage by one warp (returns the number of warps that had
// released it before); acq_rel orders every warp's reads of the stage before
// the refill's bulk copy.
__device__ __forceinline__ uint32_t stage_release(uint32_t* cnt) {
  uint32_t old;
  asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], 1;" : "=r"(old) : "r"(smem_u32(cnt)) : "memory");
  return old;
}

// Four 8 x 8 bf16 tiles from the mma accumulator layout into shared memory;
// lane l gives the address of row l % 8 of tile l / 8.
__device__ __forceinline__ void stmatrix_x4(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
  asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(r0), "r"(r1),
               "r"(r2), "r"(r3)
               : "memory");
}

template <int D, int BITS, bool WFULL>
__global__ void __launch_bounds__(DCfg<D, BITS, WFULL>::THREADS, 1) decode_g16_kernel(CodecArgs a) {
  using C = DCfg<D, BITS, WFULL>;
  constexpr int kStages = C::NST;
  constexpr int NG = C::NG;
  static_assert(!C::SZ_SMEM || NG * 2 == 16, "bulk copies of steps need 16 bytes per tile");
  static_assert(C::NCW * C::TPW == C::STAGE_TILES, "every tile of a stage has a warp");
  extern __shared__ unsigned char smem_raw[];
  unsigned char* stages = reinterpret_cast<unsigned char*>(((uintptr_t)smem_raw + 127) & ~(uintptr_t)127);
  unsigned char* staging = stages + kStages * C::CODE_STAGE;
  float* csums = reinterpret_cast<float*>(staging + C::NCW * C::STG);
  uint64_t* full = reinterpret_cast<uint64_t*>(csums + C::NCW * NG * 16);
  uint32_t* released = reinterpret_cast<uint32_t*>(full + kStages);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Work unit = one stage: up to STAGE_TILES consecutive tiles of one head slice.
  const int tps = a.nt / 16;
  const int sps = (tps + C::STAGE_TILES - 1) / C::STAGE_TILES;
  const long long total = (long long)sps * a.k.slices();
  const long long u0 = total * blockIdx.x / gridDim.x;
  const long long u1 = total * (blockIdx.x + 1) / gridDim.x;
  const int n_units = (int)(u1 - u0);
  const long long slice_code_bytes = (long long)a.k.T * D * BITS / 8;

  // stage q of this CTA: up to STAGE_TILES code tiles (and, W = 16, their
  // steps and zero points) by 1-D bulk copies into ring slot q % kStages
  auto issue = [&](int q) {
    const long long u = u0 + q, sl = u / sps;
    const int sqq = (int)(u - sl * sps);
    const int st = q % kStages;
    const int nvalid = min(C::STAGE_TILES, tps - C::STAGE_TILES * sqq);
    const uint32_t bytes = (uint32_t)(nvalid * C::CODE_TILE);
    const uint32_t szb = (uint32_t)(nvalid * NG * 2);  // 16 bytes per tile (SZ_SMEM)
    mbar_arrive_expect_tx(&full[st], bytes + (C::SZ_SMEM ? 2u * szb : 0u));
    const long long tl0 = sl * (a.k.T / 16) + a.t0 / 16 + C::STAGE_TILES * sqq;
    unsigned char* sdst = stages + st * C::CODE_STAGE;
    bulk_g2s(sdst, a.codes_in + sl * slice_code_bytes + (tl0 - sl * (a.k.T / 16)) * C::CODE_TILE, bytes, &full[st]);
    if constexpr (C::SZ_SMEM) {
      bulk_g2s(sdst + C::CODE_BYTES, a.scales_in + tl0 * NG, szb, &full[st]);
      bulk_g2s(sdst + C::CODE_BYTES + C::SZ_BYTES, a.zeros_in + tl0 * NG, szb, &full[st]);
    }
  };
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      released[s] = 0;
    }
    fence_mbar_init();
    for (int q = 0; q < kStages && q < n_units; ++q) issue(q);
  }
  __syncthreads();
  if (n_units == 0) return;
  long long slice0 = u0 / sps;
  const int sq0 = (int)(u0 - slice0 * sps);

  // ---------------- consumers: warp w decodes tiles w*TPW .. w*TPW+TPW-1 of each stage ----------------
  const int g4 = lane >> 2, q4 = lane & 3;
  uint32_t bfr[NG][2][2][2];  // [group][n-half][hi/lo][b0/b1], fp16 pairs of G
  float* csum = csums + warp * NG * 16;  // this warp's copy of the column sums sum_c G[c][n]
  auto load_g = [&](long long sl) {
    int l, sk, b, h;
    slice_coords(sl, a.k, l, sk, b, h);
#pragma unroll
    for (int r = 0; r < NG; ++r) {
      const float* Gr = a.G + (gauge_set(l, sk, h, a.k) * NG + r) * 256;  // G[c][n], row-major
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
        bfr[r][nh][0][0] = h0 | (h1 << 16);
        bfr[r][nh][0][1] = h2 | (h3 << 16);
        bfr[r][nh][1][0] = f16_bits(r0) | (f16_bits(r1) << 16);
        bfr[r][nh][1][1] = f16_bits(r2) | (f16_bits(r3) << 16);
      }
    }
    __syncwarp();  // the previous slice's column sums are no longer read
    for (int e = lane; e < NG * 16; e += 32) {
      const float* Gr = a.G + (gauge_set(l, sk, h, a.k) * NG + (e >> 4)) * 256 + (e & 15);
      float acc = 0.0f;
#pragma unroll
      for (int c = 0; c < 16; ++c) acc += __ldg(Gr + c * 16);
      csum[e] = acc;
    }
    __syncwarp();
  };
  // steps and zero points of this warp's tiles of a stage as raw fp16 words
  // (W = d: one value; W = 16: NG/2 words of two), loaded one stage ahead
  auto fetch_sz = [&](long long sl, int sqq, uint32_t (&sw)[C::TPW][C::SZW], uint32_t (&zw)[C::TPW][C::SZW]) {
    const int nv = min(C::STAGE_TILES, tps - C::STAGE_TILES * sqq);
#pragma unroll
    for (int tt = 0; tt < C::TPW; ++tt) {
      const int tl = warp * C::TPW + tt;
      const long long tile = sl * (a.k.T / 16) + a.t0 / 16 + C::STAGE_TILES * sqq + tl;
      if (tl < nv) {
        if constexpr (WFULL) {
          sw[tt][0] = __ldg(a.scales_in + tile);
          zw[tt][0] = __ldg(a.zeros_in + tile);
        } else {
#pragma unroll
          for (int w = 0; w < C::SZW; ++w) {
            sw[tt][w] = __ldg(reinterpret_cast<const uint32_t*>(a.scales_in + tile * NG) + w);
            zw[tt][w] = __ldg(reinterpret_cast<const uint32_t*>(a.zeros_in + tile * NG) + w);
          }
        }
      }
    }
  };
  long long slice = slice0;
  int sq = sq0;
  load_g(slice);
  uint32_t sw[C::TPW][C::SZW], zw[C::TPW][C::SZW];
  if constexpr (!C::SZ_SMEM) fetch_sz(slice, sq, sw, zw);
  unsigned char* stg = staging + warp * C::STG;
  const uint32_t stg_s = smem_u32(stg);
  // stmatrix row addresses: lane l -> row l % 8 (+ 8 for tiles 1 and 3) of the tile, column half l / 16
  const uint32_t st_addr = stg_s + ((lane & 7) + 8 * ((lane >> 3) & 1)) * C::PITCH + ((lane >> 4) * 8) * 2;
  for (int q = 0; q < n_units; ++q) {
    const int s = q % kStages;
    const int nvalid = min(C::STAGE_TILES, tps - C::STAGE_TILES * sq);
    const int tile0 = a.t0 / 16 + C::STAGE_TILES * sq;
    uint32_t cs[C::TPW][C::SZW], cz[C::TPW][C::SZW];
    if constexpr (!C::SZ_SMEM) {
#pragma unroll
      for (int tt = 0; tt < C::TPW; ++tt)
#pragma unroll
        for (int w = 0; w < C::SZW; ++w) {
          cs[tt][w] = sw[tt][w];
          cz[tt][w] = zw[tt][w];
        }
      if (q + 1 < n_units) {  // next stage's steps and zero points, in flight during this one
        const bool wrap = sq + 1 == sps;
        fetch_sz(wrap ? slice + 1 : slice, wrap ? 0 : sq + 1, sw, zw);
      }
    }
    mbar_wait(&full[s], (uint32_t)(q / kStages) & 1u, a.status);
    const unsigned char* sbase = stages + s * C::CODE_STAGE;
#pragma unroll
    for (int tt = 0; tt < C::TPW; ++tt) {
      const int tl = warp * C::TPW + tt;
      if (tl >= nvalid) break;
      const unsigned char* cbuf = sbase + tl * C::CODE_TILE;
#pragma unroll
      for (int r = 0; r < NG; ++r) {
        float sf, zf;
        if constexpr (WFULL) {
          sf = __half2float(__ushort_as_half((unsigned short)cs[tt][0]));
          zf = __half2float(__ushort_as_half((unsigned short)cz[tt][0]));
        } else if constexpr (C::SZ_SMEM) {
          const __half* sz = reinterpret_cast<const __half*>(sbase + C::CODE_BYTES) + tl * NG + r;
          sf = __half2float(sz[0]);
          zf = __half2float(sz[C::SZ_BYTES / 2]);
        } else {
          const uint32_t ws = cs[tt][r >> 1], wz = cz[tt][r >> 1];
          sf = __half2float(__ushort_as_half((unsigned short)((r & 1) ? (ws >> 16) : (ws & 0xffffu))));
          zf = __half2float(__ushort_as_half((unsigned short)((r & 1) ? (wz >> 16) : (wz & 0xffffu))));
        }
        uint32_t afr[4];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int row = g4 + 8 * half;
          const int bit = (WFULL ? (row * D + 16 * r + 4 * q4) : (r * 256 + row * 16 + 4 * q4)) * BITS;
          const uint32_t* wp = reinterpret_cast<const uint32_t*>(cbuf) + (bit >> 5);
          uint32_t v;
          if constexpr (BITS == 4 || BITS == 8 || BITS == 2) {
            v = wp[0] >> (bit & 31);  // the 4 codes never straddle a word for these widths
          } else {
            v = __funnelshift_r(wp[0], wp[1], bit & 31);
          }
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
        uint32_t pk[2][2];  // [n-half][row half], bf16 pairs
#pragma unroll
        for (int nh = 0; nh < 2; ++nh) {
          float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
          mma_f16_16816(acc, afr, bfr[r][nh][0][0], bfr[r][nh][0][1]);
          mma_f16_16816(acc, afr, bfr[r][nh][1][0], bfr[r][nh][1][1]);
          // x_hat = s * acc + z * colsum, bf16 RNE
          const float2 cs2 = *reinterpret_cast<const float2*>(csum + 16 * r + 8 * nh + 2 * q4);
          const float cz0 = zf * cs2.x, cz1 = zf * cs2.y;
          pk[nh][0] = pack_bf16x2(__fmaf_rn(sf, acc[0], cz0), __fmaf_rn(sf, acc[1], cz1));
          pk[nh][1] = pack_bf16x2(__fmaf_rn(sf, acc[2], cz0), __fmaf_rn(sf, acc[3], cz1));
        }
        // tiles (rows 0-7 | 8-15) x (cols 16r .. +7 | 16r+8 .. +15)
        stmatrix_x4(st_addr + 32 * r, pk[0][0], pk[0][1], pk[1][0], pk[1][1]);
      }
      __syncwarp();
      // the tile's 16 rows (contiguous in the output) with 16-byte stores:
      // each instruction writes two whole rows
      uint16_t* obase = a.kv_out + (slice * a.k.T + (long long)(tile0 + tl) * 16) * D;
      constexpr int CPR = 2 * D / 16;  // 16-byte chunks per row
#pragma unroll
      for (int k = 0; k < 16 * CPR / 32; ++k) {
        const int idx = 32 * k + lane, row = idx / CPR, ch = idx % CPR;
        const uint4 v = *reinterpret_cast<const uint4*>(stg + row * C::PITCH + ch * 16);
        reinterpret_cast<uint4*>(obase + row * D)[ch] = v;
      }
      __syncwarp();
    }
    // this warp is done with stage q; the last warp to say so refills the slot
    __syncwarp();
    if (lane == 0 && stage_release(&released[s]) == C::NCW - 1) {
      released[s] = 0;
      if (q + kStages < n_units) issue(q + kStages);
    }
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
