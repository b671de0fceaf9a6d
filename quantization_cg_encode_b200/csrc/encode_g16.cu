// Fused gauge + block-uniform quantize + pack for g = 16 (the grouped setting
// Codec-Gauge reports as representative), d_head 64 or 128, any bit width,
// ranges of 16 tokens x 16 channels or 16 tokens x d_head.
//
// Codec-Gauge, Method: explicit gauge application costs O(N_KV g) multiply-
// adds (16 per value here); Experimental setup: block-uniform backend.
//
// Structure (one CTA per SM, persistent over a contiguous range of 16-token
// tiles in (layer, K/V, batch, head, token) order, two tiles per iteration):
//   * stages of 4 tiles (64 tokens x d bf16, 16 KB at d = 128) stream into a
//     6-stage shared-memory ring with 2-D TMA loads of 64 x 64 boxes (8 KB per
//     copy: smaller copies leave the TMA unit short of HBM bandwidth; 128-byte
//     swizzle, no multicast), completion counted on mbarriers; the warp that
//     releases a stage last refills it (no producer warp: eight warps of up to
//     255 registers is what the 4 x 16K-register scheduler partitions hold);
//   * warp r owns channel group r: lane (t, hh) = (lane & 15, lane >> 4)
//     computes gauged outputs 8hh .. 8hh+7 of token t in all 4 tiles of a
//     stage.  Its half of G_r lives in registers as fp32 row pairs, and the
//     exact per-output FMA chain (j = 0..15, from +0) runs as packed
//     fma.rn.f32x2, two outputs per instruction with the token's x_j
//     duplicated into both halves (16 independent chains per thread);
//   * lanes 8k .. 8k+7 compute tile k's block parameters (one evaluation per
//     lane covers the stage's four blocks), shared by shuffle;
//   * the range of a 16 x 16 block is one warp: redux.sync min / max (a
//     16 x d_head range adds one exchange between the group warps);
//   * each lane stores its 8 packed codes straight to global memory (a warp
//     writes its block's bytes contiguously), so warps never wait on each other.
#include <cuda.h>

#include "cg_kernels.cuh"

namespace cg {

namespace {

constexpr int kStages = 6;   // ring stages of 4 tiles (96 KB at d = 128)

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
  static constexpr int TPS = 4;                          // 16-token tiles per ring stage
  static constexpr int STAGE_BYTES = TPS * 16 * D * 2;   // 16 KB at d = 128: one 8 KB TMA box per 64 channels
  static constexpr int BOXES = D / 64;
  static constexpr int CODE_TILE = 16 * D * BITS / 8;    // packed codes of one tile
  static constexpr int SMEM = 1024 + kStages * STAGE_BYTES + kStages * 8 + kStages * 4 + 64 * 4;
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
  unsigned char* stages = base;                                   // kStages x STAGE_BYTES, 1024-aligned
  uint64_t* full = reinterpret_cast<uint64_t*>(stages + kStages * C::STAGE_BYTES);
  uint32_t* released = reinterpret_cast<uint32_t*>(full + kStages);
  float* red = reinterpret_cast<float*>(released + kStages);      // [min / max][4 tiles][8 groups]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Work unit = one ring stage: up to 4 consecutive tiles of one head slice,
  // processed as two pairs (A, B).  The CTA owns units [u0, u1).
  const int tps = a.nt / 16;                                      // tiles per head slice
  const int sps = (tps + C::TPS - 1) / C::TPS;                    // stages per head slice
  const long long total = (long long)sps * a.k.slices();
  const long long u0 = total * blockIdx.x / gridDim.x;
  const long long u1 = total * (blockIdx.x + 1) / gridDim.x;
  const int n_units = (int)(u1 - u0);

  // rows [row, row + 64) of the [rows][d] view hold unit q's tiles
  auto unit_row = [&](int q) -> int {
    const unsigned gu = (unsigned)(u0 + q);                       // < 2^31 units
    const unsigned sl = gu / (unsigned)sps;
    return (int)((long long)sl * a.k.T + a.t0 + 64 * (gu - sl * (unsigned)sps));
  };
  auto issue = [&](int q) {
    const int st = q % kStages;
    mbar_arrive_expect_tx(&full[st], C::STAGE_BYTES);
    const int row = unit_row(q);
#pragma unroll
    for (int b = 0; b < C::BOXES; ++b)
      tma_load_2d(stages + st * C::STAGE_BYTES + b * (C::STAGE_BYTES / C::BOXES), &tmap, b * 64, row, &full[st]);
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

  const int r = warp;
  const int t = lane & 15, hh = lane >> 4;
  const double inv_qmax = 1.0 / (double)QMAX;
  const int box = r >> 2;
  const int c0 = (r & 3) * 2;  // first 16-byte chunk of this group inside the 128-byte row
  // byte offsets of token t's two chunks inside the first tile of a stage (box rows t)
  const uint32_t rd0 = box * (C::STAGE_BYTES / C::BOXES) + t * 128 + ((c0 ^ (t & 7)) << 4);
  const uint32_t rd1 = box * (C::STAGE_BYTES / C::BOXES) + t * 128 + (((c0 + 1) ^ (t & 7)) << 4);
  const int nblk = WFULL ? 1 : D / 16;
  const int code_off = WFULL ? (t * D + 16 * r + 8 * hh) * BITS / 8 : r * (256 * BITS / 8) + t * (2 * BITS) + hh * BITS;
  const long long slice_code_bytes = (long long)a.k.T * D * BITS / 8;
  const long long slice_blocks = (long long)(a.k.T / 16) * nblk;

  f2_t gp[4][16];  // gp[m][j] = {G[8hh+2m][j], G[8hh+2m+1][j]}
  auto load_g = [&](long long sl) {
    int l, sk, b, h;
    slice_coords(sl, a.k, l, sk, b, h);
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
  };
  // the warp is done reading unit q; the last warp to say so refills the stage
  auto release = [&](int q) {
    __syncwarp();
    if (lane == 0) {
      const int st = q % kStages;
      if (stage_release(&released[st]) == C::NW - 1) {
        released[st] = 0;
        if (q + kStages < n_units) issue(q + kStages);
      }
    }
  };

  // One iteration = one stage of up to 4 tiles: 16 independent FMA chains per
  // thread, then the four blocks' parameters computed by 8 lanes each.
  long long slice = u0 / sps;
  int sq = (int)(u0 - slice * sps);
  load_g(slice);
  const int kq = lane >> 3;  // tile whose block parameters this lane computes
  for (int q = 0; q < n_units; ++q) {
    const int nvalid = min(C::TPS, tps - C::TPS * sq);
    const int st = q % kStages;
    mbar_wait(&full[st], (uint32_t)(q / kStages) & 1u, a.status);
    const unsigned char* sb = stages + st * C::STAGE_BYTES;
    uint32_t w[C::TPS][8];
#pragma unroll
    for (int k = 0; k < C::TPS; ++k) {
      const uint4 v0 = *reinterpret_cast<const uint4*>(sb + k * 2048 + rd0);
      const uint4 v1 = *reinterpret_cast<const uint4*>(sb + k * 2048 + rd1);
      w[k][0] = v0.x; w[k][1] = v0.y; w[k][2] = v0.z; w[k][3] = v0.w;
      w[k][4] = v1.x; w[k][5] = v1.y; w[k][6] = v1.z; w[k][7] = v1.w;
    }
    // ---- gauge: exact fp32 FMA chains (j = 0..15 from +0), four tiles interleaved ----
    f2_t acc[C::TPS][4];
#pragma unroll
    for (int k = 0; k < C::TPS; ++k)
#pragma unroll
      for (int m = 0; m < 4; ++m) acc[k][m] = 0ull;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
#pragma unroll
      for (int k = 0; k < C::TPS; ++k) {
        const float x = (j & 1) ? bf16hi(w[k][j >> 1]) : bf16lo(w[k][j >> 1]);
        const f2_t xd = f2_make(x, x);
#pragma unroll
        for (int m = 0; m < 4; ++m) acc[k][m] = f2_fma(gp[m][j], xd, acc[k][m]);
      }
    }
    release(q);

    // ---- block ranges ----
    float mn[C::TPS], mx[C::TPS];
#pragma unroll
    for (int k = 0; k < C::TPS; ++k) {
      minmax8(acc[k], mn[k], mx[k]);
      mn[k] = warp_min_f32(mn[k]);
      mx[k] = warp_max_f32(mx[k]);
    }
    if constexpr (WFULL) {
      float* rb = red;  // [mn x 4 tiles][mx x 4 tiles] x 8 groups
      if (lane == 0) {
#pragma unroll
        for (int k = 0; k < C::TPS; ++k) {
          rb[k * 8 + r] = mn[k];
          rb[32 + k * 8 + r] = mx[k];
        }
      }
      named_bar_sync(1, C::NW * 32);
#pragma unroll
      for (int k = 0; k < C::TPS; ++k) {
        mn[k] = rb[k * 8];
        mx[k] = rb[32 + k * 8];
#pragma unroll
        for (int g = 1; g < C::NW; ++g) {
          mn[k] = fminf(mn[k], rb[k * 8 + g]);
          mx[k] = fmaxf(mx[k], rb[32 + k * 8 + g]);
        }
      }
      named_bar_sync(2, C::NW * 32);  // every warp has read rb before it is reused
    }
    // ---- block parameters: lanes 8k .. 8k+7 compute tile k's ----
    const float pmn = kq == 0 ? mn[0] : kq == 1 ? mn[1] : kq == 2 ? mn[2] : mn[3];
    const float pmx = kq == 0 ? mx[0] : kq == 1 ? mx[1] : kq == 2 ? mx[2] : mx[3];
    const QParams qp = quant_params(pmn, pmx, inv_qmax);
    const float tlo = __fmul_rn(__fsub_rn(pmn, qp.zf), qp.inv);
    const float thi = __fmul_rn(__fsub_rn(pmx, qp.zf), qp.inv);
    // t is monotone in y: if the block's extremes round into [0, qmax], no value needs clamping
    const unsigned inr = __ballot_sync(0xffffffffu, (tlo >= -0.5f) && (thi < (float)QMAX + 0.5f));

    // ---- quantize, pack, store ----
    const int tile0 = a.t0 / 16 + C::TPS * sq;
    uint8_t* cp = a.codes + slice * slice_code_bytes + (long long)tile0 * C::CODE_TILE + code_off;
#pragma unroll
    for (int k = 0; k < C::TPS; ++k) {
      const float zf = __shfl_sync(0xffffffffu, qp.zf, 8 * k);
      const float inv = __shfl_sync(0xffffffffu, qp.inv, 8 * k);
      const uint64_t ch = quantize8<BITS>(acc[k], zf, inv, (inr >> (8 * k)) & 1u);
      if (k < nvalid) store_chunk<BITS>(cp + k * C::CODE_TILE, ch);
    }
    if ((lane & 7) == 0 && kq < nvalid && (!WFULL || r == 0)) {
      const long long bidx = slice * slice_blocks + (long long)(tile0 + kq) * nblk + (WFULL ? 0 : r);
      a.scales[bidx] = qp.sh;
      a.zeros[bidx] = qp.zh;
    }
    if (a.gauged) {
#pragma unroll
      for (int k = 0; k < C::TPS; ++k) {
        if (k >= nvalid) break;
        float* gk = a.gauged + (slice * a.k.T + (long long)(tile0 + k) * 16 + t) * D + 16 * r + 8 * hh;
        float y[8];
#pragma unroll
        for (int m = 0; m < 4; ++m) f2_split(acc[k][m], y[2 * m], y[2 * m + 1]);
        reinterpret_cast<float4*>(gk)[0] = make_float4(y[0], y[1], y[2], y[3]);
        reinterpret_cast<float4*>(gk)[1] = make_float4(y[4], y[5], y[6], y[7]);
      }
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
  using C = Cfg<D, BITS, WFULL>;
  alignas(64) CUtensorMap tmap;
  const uint64_t rows = (uint64_t)a.k.slices() * a.k.T;
  if (!make_tmap_2d_bf16(&tmap, a.kv, rows, D, 64, 16 * C::TPS)) return cudaErrorInvalidValue;
  auto kern = encode_g16_kernel<D, BITS, WFULL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const long long total = (long long)((a.nt / 16 + C::TPS - 1) / C::TPS) * a.k.slices();
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
  return a.k.d == 128 ? launch_b<128>(a, num_sms, st) : launch_b<64>(a, num_sms, st);
}

}  // namespace cg
