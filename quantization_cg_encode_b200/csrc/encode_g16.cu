// Fused gauge + block-uniform quantize + pack for g = 16 (the grouped setting
// Codec-Gauge reports as representative), d_head 64 or 128, any bit width,
// ranges of 16 tokens x 16 channels or 16 tokens x d_head.
//
// Codec-Gauge, Method: explicit gauge application costs O(N_KV g) multiply-
// adds (16 per value here); Experimental setup: block-uniform backend.
//
// Structure (one CTA per SM, persistent over a contiguous range of 16-token
// tiles in (layer, K/V, batch, head, token) order, two tiles per iteration):
//   * tiles (16 tokens x d bf16, 4 KB at d = 128) stream into a 12-stage
//     shared-memory ring with 2-D TMA loads (128-byte swizzle, no multicast),
//     completion counted on mbarriers; the warp that releases a stage last
//     refills it (no producer warp: eight warps of up to 255 registers is what
//     the 4 x 16K-register scheduler partitions of an SM can hold);
//   * warp r owns channel group r: lane (t, hh) = (lane & 15, lane >> 4)
//     computes gauged outputs 8hh .. 8hh+7 of token t.  Its half of G_r lives
//     in registers as fp32 row pairs, and the exact per-output FMA chain
//     (j = 0..15, from +0) runs as packed fma.rn.f32x2, two outputs per
//     instruction with the token's x_j duplicated into both halves;
//   * the range of a 16 x 16 block is one warp: redux.sync min / max (a
//     16 x d_head range adds one exchange between the group warps);
//   * each lane stores its 8 packed codes straight to global memory (a warp
//     writes its block's bytes contiguously), so warps never wait on each other.
#include <cuda.h>

#include "cg_kernels.cuh"

namespace cg {

namespace {

constexpr int kStages = 12;

__device__ __forceinline__ float min3f(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Store the 8 * BITS-bit chunk v at dst (alignment: see the callers' offsets).
template <int BITS>
__device__ __forceinline__ void store_chunk(uint8_t* dst, uint64_t v) {
  if constexpr (BITS == 2) {
    *reinterpret_cast<uint16_t*>(dst) = (uint16_t)v;
  } else if constexpr (BITS == 4) {
    *reinterpret_cast<uint32_t*>(dst) = (uint32_t)v;
  } else if constexpr (BITS == 8) {
    *reinterpret_cast<uint2*>(dst) = make_uint2((uint32_t)v, (uint32_t)(v >> 32));
  } else if constexpr (BITS == 6) {
    uint16_t* p = reinterpret_cast<uint16_t*>(dst);
    p[0] = (uint16_t)v;
    p[1] = (uint16_t)(v >> 16);
    p[2] = (uint16_t)(v >> 32);
  } else {  // 3 bits: 3 bytes at any offset
    dst[0] = (uint8_t)v;
    dst[1] = (uint8_t)(v >> 8);
    dst[2] = (uint8_t)(v >> 16);
  }
}

template <int D, int BITS, bool WFULL>
struct Cfg {
  static constexpr int NW = D / 16;                      // warps (= channel groups)
  static constexpr int THREADS = NW * 32;
  static constexpr int TILE_BYTES = 16 * D * 2;          // bf16 input tile
  static constexpr int BOXES = D / 64;                   // 64-channel TMA boxes per tile
  static constexpr int CODE_TILE = 16 * D * BITS / 8;    // packed codes of one tile
  static constexpr int SMEM = 1024 + kStages * TILE_BYTES + kStages * 8 + kStages * 4 + 2 * 32 * 4;
};

// Pack 8 codes, given as the bit patterns of (t + 1.5 * 2^23) whose low byte is
// the code, into an 8 * BITS-bit little-endian chunk.
template <int BITS>
__device__ __forceinline__ uint64_t pack8(const uint32_t (&rb)[8]) {
  if constexpr (BITS == 4) {
    const uint32_t n01 = (rb[0] & 0x0Fu) | ((rb[1] << 4) & 0xF0u);
    const uint32_t n23 = (rb[2] & 0x0Fu) | ((rb[3] << 4) & 0xF0u);
    const uint32_t n45 = (rb[4] & 0x0Fu) | ((rb[5] << 4) & 0xF0u);
    const uint32_t n67 = (rb[6] & 0x0Fu) | ((rb[7] << 4) & 0xF0u);
    return __byte_perm(__byte_perm(n01, n23, 0x0040), __byte_perm(n45, n67, 0x0040), 0x5410);
  } else if constexpr (BITS == 8) {
    const uint32_t lo = __byte_perm(__byte_perm(rb[0], rb[1], 0x0040), __byte_perm(rb[2], rb[3], 0x0040), 0x5410);
    const uint32_t hi = __byte_perm(__byte_perm(rb[4], rb[5], 0x0040), __byte_perm(rb[6], rb[7], 0x0040), 0x5410);
    return (uint64_t)lo | ((uint64_t)hi << 32);
  } else {
    constexpr uint32_t M = (1u << BITS) - 1u;
    uint64_t c = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) c |= (uint64_t)(rb[k] & M) << (k * BITS);
    return c;
  }
}

// Codes of 8 gauged values (4 f32x2 pairs) against one block's z and 1/s.
template <int BITS>
__device__ __forceinline__ uint64_t quantize8(const f2_t (&acc)[4], float zf, float inv, bool inrange) {
  constexpr int QMAX = (1 << BITS) - 1;
  const f2_t nz2 = f2_make(-zf, -zf), inv2 = f2_make(inv, inv);
  const f2_t mg2 = f2_make(12582912.0f, 12582912.0f);  // 1.5 * 2^23: adding it rounds to an integer (RNE)
  uint32_t rb[8];
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    f2_t tt = f2_mul(f2_add(acc[m], nz2), inv2);
    if (!inrange) {
      float lo, hi;
      f2_split(tt, lo, hi);
      tt = f2_make(fminf(fmaxf(lo, 0.0f), (float)QMAX), fminf(fmaxf(hi, 0.0f), (float)QMAX));
    }
    tt = f2_add(tt, mg2);
    float lo, hi;
    f2_split(tt, lo, hi);
    rb[2 * m] = __float_as_uint(lo);
    rb[2 * m + 1] = __float_as_uint(hi);
  }
  return pack8<BITS>(rb);
}

__device__ __forceinline__ void minmax8(const f2_t (&acc)[4], float& mn, float& mx) {
  float y[8];
#pragma unroll
  for (int m = 0; m < 4; ++m) f2_split(acc[m], y[2 * m], y[2 * m + 1]);
  mn = min3f(min3f(y[0], y[1], y[2]), min3f(y[3], y[4], y[5]), fminf(y[6], y[7]));
  mx = max3f(max3f(y[0], y[1], y[2]), max3f(y[3], y[4], y[5]), fmaxf(y[6], y[7]));
}

// Release of a ring stage by one warp; the warp that releases it last refills
// it with the tile kStages further on.  acq_rel orders every warp's reads of
// the stage before the refill's TMA write.
__device__ __forceinline__ uint32_t stage_release(uint32_t* cnt) {
  uint32_t old;
  asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], 1;" : "=r"(old) : "r"(smem_u32(cnt)) : "memory");
  return old;
}

template <int D, int BITS, bool WFULL>
__global__ void __launch_bounds__(Cfg<D, BITS, WFULL>::THREADS, 1)
    encode_g16_kernel(const __grid_constant__ CUtensorMap tmap, CodecArgs a) {
  using C = Cfg<D, BITS, WFULL>;
  constexpr int QMAX = (1 << BITS) - 1;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  unsigned char* stages = base;                                   // kStages x TILE_BYTES, 1024-aligned
  uint64_t* full = reinterpret_cast<uint64_t*>(stages + kStages * C::TILE_BYTES);
  uint32_t* released = reinterpret_cast<uint32_t*>(full + kStages);
  float* red = reinterpret_cast<float*>(released + kStages);      // [2 parity][4 (mnA,mxA,mnB,mxB)][8 groups]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Work unit = a pair of consecutive tiles of one head slice (the tile count
  // per slice is even on this path); the CTA owns tiles [2 u0, 2 u1).
  const int tps = a.nt / 16;
  const int upt = tps / 2;
  const long long total = (long long)upt * a.k.slices();
  const long long u0 = total * blockIdx.x / gridDim.x;
  const long long u1 = total * (blockIdx.x + 1) / gridDim.x;
  const int n_units = (int)(u1 - u0);
  const int n_tiles = 2 * n_units;
  long long slice = u0 / upt;
  int pu = (int)(u0 - slice * upt);                               // pair index inside the slice

  // row of the CTA's j-th tile in the [rows][d] view of the cache
  auto tile_row = [&](int j) -> int {
    const unsigned gt = (unsigned)(2 * u0 + j);   // < 2^31 tiles
    const unsigned sl = gt / (unsigned)tps;
    return (int)((long long)sl * a.k.T + a.t0 + 16 * (gt - sl * (unsigned)tps));
  };
  auto issue = [&](int j) {
    const int st = j % kStages;
    mbar_arrive_expect_tx(&full[st], C::TILE_BYTES);
    const int row = tile_row(j);
#pragma unroll
    for (int b = 0; b < C::BOXES; ++b) tma_load_2d(stages + st * C::TILE_BYTES + b * 2048, &tmap, b * 64, row, &full[st]);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      released[s] = 0;
    }
    fence_mbar_init();
    for (int j = 0; j < kStages && j < n_tiles; ++j) issue(j);
  }
  __syncthreads();

  // ---------------- consumers: warp r = channel group r ----------------
  const int r = warp;
  const int t = lane & 15, hh = lane >> 4;
  const double inv_qmax = 1.0 / (double)QMAX;
  const int box = r >> 2;
  const int c0 = (r & 3) * 2;  // first 16-byte chunk of this group inside the 128-byte row
  const uint32_t rd0 = t * 128 + ((c0 ^ (t & 7)) << 4) + box * 2048;
  const uint32_t rd1 = t * 128 + (((c0 + 1) ^ (t & 7)) << 4) + box * 2048;
  const int nblk = WFULL ? 1 : D / 16;
  const int code_off = WFULL ? (t * D + 16 * r + 8 * hh) * BITS / 8 : r * (256 * BITS / 8) + t * (2 * BITS) + hh * BITS;
  const long long slice_code_bytes = (long long)a.k.T * D * BITS / 8;
  const long long slice_blocks = (long long)(a.k.T / 16) * nblk;

  f2_t gp[4][16];  // gp[m][j] = {G[8hh+2m][j], G[8hh+2m+1][j]}
  bool need_g = true;
  for (int u = 0; u < n_units; ++u) {
    if (need_g) {
      int l, sk, b, h;
      slice_coords(slice, a.k, l, sk, b, h);
      const float* Gr = a.G + (gauge_set(l, sk, h, a.k) * (D / 16) + r) * 256;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float4* row0 = reinterpret_cast<const float4*>(Gr + (8 * hh + 2 * m) * 16);
        const float4* row1 = reinterpret_cast<const float4*>(Gr + (8 * hh + 2 * m + 1) * 16);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 uu = __ldg(row0 + q), vv = __ldg(row1 + q);
          gp[m][4 * q + 0] = f2_make(uu.x, vv.x);
          gp[m][4 * q + 1] = f2_make(uu.y, vv.y);
          gp[m][4 * q + 2] = f2_make(uu.z, vv.z);
          gp[m][4 * q + 3] = f2_make(uu.w, vv.w);
        }
      }
      need_g = false;
    }
    const int tileA = a.t0 / 16 + 2 * pu;

    // ---- x of token t in group r, tiles A = 2u and B = 2u + 1 of this CTA ----
    const int jA = 2 * u, jB = 2 * u + 1;
    const int sA = jA % kStages, sB = jB % kStages;
    mbar_wait(&full[sA], (uint32_t)((jA / kStages) & 1), a.status);
    const uint4 a0 = *reinterpret_cast<const uint4*>(stages + sA * C::TILE_BYTES + rd0);
    const uint4 a1 = *reinterpret_cast<const uint4*>(stages + sA * C::TILE_BYTES + rd1);
    mbar_wait(&full[sB], (uint32_t)((jB / kStages) & 1), a.status);
    const uint4 b0 = *reinterpret_cast<const uint4*>(stages + sB * C::TILE_BYTES + rd0);
    const uint4 b1 = *reinterpret_cast<const uint4*>(stages + sB * C::TILE_BYTES + rd1);
    __syncwarp();
    if (lane == 0) {
      if (stage_release(&released[sA]) == C::NW - 1) {
        released[sA] = 0;
        if (jA + kStages < n_tiles) issue(jA + kStages);
      }
      if (stage_release(&released[sB]) == C::NW - 1) {
        released[sB] = 0;
        if (jB + kStages < n_tiles) issue(jB + kStages);
      }
    }

    // ---- gauge: exact fp32 FMA chains, tiles A and B interleaved ----
    const uint32_t wa[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    const uint32_t wb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
    f2_t accA[4], accB[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) accA[m] = accB[m] = 0ull;  // {+0, +0}
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float xa = (j & 1) ? bf16hi(wa[j >> 1]) : bf16lo(wa[j >> 1]);
      const float xb = (j & 1) ? bf16hi(wb[j >> 1]) : bf16lo(wb[j >> 1]);
      const f2_t xda = f2_make(xa, xa), xdb = f2_make(xb, xb);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        accA[m] = f2_fma(gp[m][j], xda, accA[m]);
        accB[m] = f2_fma(gp[m][j], xdb, accB[m]);
      }
    }
    if (a.gauged) {
      float* gA = a.gauged + (slice * a.k.T + (long long)tileA * 16 + t) * D + 16 * r + 8 * hh;
      float y[8];
#pragma unroll
      for (int m = 0; m < 4; ++m) f2_split(accA[m], y[2 * m], y[2 * m + 1]);
      reinterpret_cast<float4*>(gA)[0] = make_float4(y[0], y[1], y[2], y[3]);
      reinterpret_cast<float4*>(gA)[1] = make_float4(y[4], y[5], y[6], y[7]);
      {
#pragma unroll
        for (int m = 0; m < 4; ++m) f2_split(accB[m], y[2 * m], y[2 * m + 1]);
        reinterpret_cast<float4*>(gA + 16 * D)[0] = make_float4(y[0], y[1], y[2], y[3]);
        reinterpret_cast<float4*>(gA + 16 * D)[1] = make_float4(y[4], y[5], y[6], y[7]);
      }
    }

    // ---- block ranges ----
    float mnA, mxA, mnB, mxB;
    minmax8(accA, mnA, mxA);
    minmax8(accB, mnB, mxB);
    mnA = warp_min_f32(mnA);
    mxA = warp_max_f32(mxA);
    mnB = warp_min_f32(mnB);
    mxB = warp_max_f32(mxB);
    if constexpr (WFULL) {
      float* rb = red + (u & 1) * 32;
      if (lane == 0) {
        rb[r] = mnA;
        rb[8 + r] = mxA;
        rb[16 + r] = mnB;
        rb[24 + r] = mxB;
      }
      named_bar_sync(1, C::NW * 32);
      mnA = rb[0]; mxA = rb[8]; mnB = rb[16]; mxB = rb[24];
#pragma unroll
      for (int q = 1; q < C::NW; ++q) {
        mnA = fminf(mnA, rb[q]);
        mxA = fmaxf(mxA, rb[8 + q]);
        mnB = fminf(mnB, rb[16 + q]);
        mxB = fmaxf(mxB, rb[24 + q]);
      }
    }
    // block parameters: lanes 0-15 for tile A, lanes 16-31 for tile B
    const float pmn = hh ? mnB : mnA, pmx = hh ? mxB : mxA;
    const QParams qp = quant_params(pmn, pmx, inv_qmax);
    const float tlo = __fmul_rn(__fsub_rn(pmn, qp.zf), qp.inv);
    const float thi = __fmul_rn(__fsub_rn(pmx, qp.zf), qp.inv);
    // t is monotone in y: if the block's extremes round into [0, qmax], no value needs clamping
    const unsigned inr = __ballot_sync(0xffffffffu, (tlo >= -0.5f) && (thi < (float)QMAX + 0.5f));
    const float zfA = __shfl_sync(0xffffffffu, qp.zf, 0), invA = __shfl_sync(0xffffffffu, qp.inv, 0);
    const float zfB = __shfl_sync(0xffffffffu, qp.zf, 16), invB = __shfl_sync(0xffffffffu, qp.inv, 16);

    const uint64_t chA = quantize8<BITS>(accA, zfA, invA, inr & 1u);
    const uint64_t chB = quantize8<BITS>(accB, zfB, invB, (inr >> 16) & 1u);
    uint8_t* cp = a.codes + slice * slice_code_bytes + (long long)tileA * C::CODE_TILE + code_off;
    store_chunk<BITS>(cp, chA);
    store_chunk<BITS>(cp + C::CODE_TILE, chB);
    if ((lane & 15) == 0 && (!WFULL || r == 0)) {
      const long long bidx = slice * slice_blocks + (long long)(tileA + hh) * nblk + (WFULL ? 0 : r);
      a.scales[bidx] = qp.sh;
      a.zeros[bidx] = qp.zh;
    }
    if (++pu == upt) {
      pu = 0;
      ++slice;
      need_g = true;
    }
  }
}

template <int D, int BITS, bool WFULL>
cudaError_t launch_one(const CodecArgs& a, int num_sms, cudaStream_t st) {
  using C = Cfg<D, BITS, WFULL>;
  alignas(64) CUtensorMap tmap;
  const uint64_t rows = (uint64_t)a.k.slices() * a.k.T;
  if (!make_tmap_2d_bf16(&tmap, a.kv, rows, D, 64, 16)) return cudaErrorInvalidValue;
  auto kern = encode_g16_kernel<D, BITS, WFULL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const long long total = (long long)(a.nt / 32) * a.k.slices();
  const int grid = (int)(total < num_sms ? total : num_sms);
  kern<<<grid, C::THREADS, C::SMEM, st>>>(tmap, a);
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

cudaError_t launch_encode_g16(const CodecArgs& a, int num_sms, cudaStream_t st) {
  if (a.nt == 0) return cudaSuccess;
  if ((a.nt / 16) % 2 != 0) return cudaErrorInvalidValue;   // callers route odd tile counts elsewhere
  return a.k.d == 128 ? launch_b<128>(a, num_sms, st) : launch_b<64>(a, num_sms, st);
}

}  // namespace cg
