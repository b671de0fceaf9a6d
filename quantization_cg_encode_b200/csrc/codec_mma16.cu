// Fused g = 16 codec with 16 x 16 block-uniform ranges (d_head 64 or 128) on
// the warp-level tensor-core path (mma.sync m16n8k16).
//
// Codec-Gauge, Method: explicit gauge application costs O(N_KV g) multiply-
// adds (16 per value at g = 16) and the inverse gauge G^T restores K and V
// before attention; Experimental setup: block-uniform backend, one min/max
// range per 16 tokens x 16 channels here.
//
// Encode.  The gauged values the quantizer sees are this kernel's own fp32
// tensor-core contraction y = x (G_hi + G_lo)^T: G (fp32) split into two bf16
// terms (G = G_hi + G_lo to 2^-18 relative), x exact in bf16, products exact,
// fp32 accumulation in the tensor core.  Given y, the block range, zero point,
// step and every code follow the quantizer's fp32 steps exactly:
//   mn, mx = min y, max y (a zero extreme is taken as +0),
//   z = fp16_rne(clamp(mn)), s = fp16_rne(min(fl32(fl32(mx - mn) / qmax), 65504)),
//   q = clamp(rne(fl32(fl32(y - z) * fl32(1/s))), 0, qmax)   (q = 0 if s = 0),
// so the codes, steps and zero points are bit-exact functions of the gauged
// values the kernel reports (gauged output), which themselves are within
// about 2^-17 sum_j |G_ij x_j| of the exact G x.
//
// Decode.  With s and z constant over a range block (a whole group),
//   x_hat_n = sum_c G[c][n] (s q_c + z) = s (sum_c q_c G[c][n]) + z colsum_n,
// a contraction of exact small integers (fp16) with G split into fp16 hi + lo
// (2^-22 relative), fp32 accumulation, then the affine epilogue and bf16 RNE.
//
// Work split (both kernels; persistent, one CTA per SM, 16 warps): stages of
// 128 (encode) or 256/512 (decode) consecutive tokens of one head slice stream
// into a shared-memory ring (encode: two or one 16 KB TMA boxes of bf16 with
// 128-byte swizzle, no multicast; decode: one 1-D bulk copy of the stage's
// code tiles).  Warp w owns channel group r = w mod (d/16) for the whole run:
// it keeps only that group's G fragments in registers and takes a fixed share
// of the stage's 16-token tiles, so one warp's 16 x 16 tile of a group is
// exactly one range block.  The output-channel order of the MMA is permuted
// so that a thread's accumulators are 4 adjacent channels of two token rows;
// each thread then packs its own code chunk (4, 8 bits) or the four threads of
// a row assemble it with shuffles (2, 3, 6 bits).  A warp releases its stage as
// soon as its fragments are in registers; the last warp to release a stage
// refills it.  Every wait on an mbarrier is bounded in time.
#include <cuda.h>

#include "cg_kernels.cuh"
#include "stage_ring.cuh"

namespace cg {

namespace {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23: t + kMagic rounds t to an integer (RNE) in the low bits

__device__ __forceinline__ float redux_min(float v) {
  float r;
  asm volatile("redux.sync.min.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}
__device__ __forceinline__ float redux_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}
__device__ __forceinline__ uint32_t f16_bits(float x) { return (uint32_t)__half_as_ushort(__float2half_rn(x)); }

// fp32 quotient rng / QMAX correctly rounded: q0 = fl(rng c), c = fl(1/QMAX),
// corrected once with the exact residual fma(-q0, QMAX, rng).  For QMAX = 3,
// 7, 15, 63 and 255 this equals fl32(rng / QMAX) for every fp32 rng (checked
// exhaustively over all non-negative inputs; odd-symmetric).
template <int QMAX>
__device__ __forceinline__ float div_qmax(float rng) {
  constexpr float c = (float)(1.0 / QMAX);
  const float q0 = __fmul_rn(rng, c);
  return __fmaf_rn(__fmaf_rn(-q0, (float)QMAX, rng), c, q0);
}

// The 4 codes of one token row held by a thread (channels 4c .. 4c+3 of its
// group), as the bit patterns of t + kMagic (low byte = the code), packed into
// a 4*BITS-bit little-endian chunk.
template <int BITS>
__device__ __forceinline__ uint32_t chunk4(uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
  if constexpr (BITS == 4) {
    const uint32_t e = __byte_perm(r0, r2, 0x1140);  // q0 | q2 << 8
    const uint32_t o = __byte_perm(r1, r3, 0x1140);  // q1 | q3 << 8
    return e + (o << 4);
  } else if constexpr (BITS == 8) {
    return __byte_perm(__byte_perm(r0, r1, 0x1140), __byte_perm(r2, r3, 0x1140), 0x5410);
  } else {
    constexpr uint32_t M = (1u << BITS) - 1u;
    return (r0 & M) | ((r1 & M) << BITS) | ((r2 & M) << (2 * BITS)) | ((r3 & M) << (3 * BITS));
  }
}

// Store the code chunks of rows g and g+8 of a 16 x 16 block (row = 16 codes,
// 2*BITS bytes).  `blk` is the block's first byte; c is the thread's quad
// position (channels 4c .. 4c+3), g its row.  4 and 8 bits: each thread stores
// its own chunk.  2 and 3 bits: the quad ORs its chunks into the whole row and
// lane c = 0 (row g) / c = 1 (row g+8) stores it.  6 bits: lane pairs form
// 48-bit half rows, stored by lanes c = 0, 2 (row g) and c = 1, 3 (row g+8).
template <int BITS>
__device__ __forceinline__ void store_rows(uint8_t* blk, int g, int c, uint32_t v0, uint32_t v1) {
  constexpr int RB = 2 * BITS;  // bytes per 16-code row
  const unsigned FULL = 0xffffffffu;
  if constexpr (BITS == 4) {
    *reinterpret_cast<uint16_t*>(blk + RB * g + 2 * c) = (uint16_t)v0;
    *reinterpret_cast<uint16_t*>(blk + RB * (g + 8) + 2 * c) = (uint16_t)v1;
  } else if constexpr (BITS == 8) {
    *reinterpret_cast<uint32_t*>(blk + RB * g + 4 * c) = v0;
    *reinterpret_cast<uint32_t*>(blk + RB * (g + 8) + 4 * c) = v1;
  } else if constexpr (BITS == 2) {  // 8-bit chunks, 32-bit rows
    uint32_t w0 = v0 << (8 * c), w1 = v1 << (8 * c);
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      w0 |= __shfl_xor_sync(FULL, w0, o);
      w1 |= __shfl_xor_sync(FULL, w1, o);
    }
    if (c < 2) *reinterpret_cast<uint32_t*>(blk + RB * (g + 8 * c)) = c ? w1 : w0;
  } else if constexpr (BITS == 3) {  // 12-bit chunks, 48-bit rows (2-byte aligned)
    uint64_t w0 = (uint64_t)v0 << (12 * c), w1 = (uint64_t)v1 << (12 * c);
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      w0 |= __shfl_xor_sync(FULL, w0, o);
      w1 |= __shfl_xor_sync(FULL, w1, o);
    }
    if (c < 2) {
      const uint64_t w = c ? w1 : w0;
      uint16_t* p = reinterpret_cast<uint16_t*>(blk + RB * (g + 8 * c));
      p[0] = (uint16_t)w;
      p[1] = (uint16_t)(w >> 16);
      p[2] = (uint16_t)(w >> 32);
    }
  } else {  // 6 bits: 24-bit chunks; lanes 2k, 2k+1 form half row k (48 bits, 2-byte aligned)
    uint64_t w0 = (uint64_t)v0 << (24 * (c & 1)), w1 = (uint64_t)v1 << (24 * (c & 1));
    w0 |= __shfl_xor_sync(FULL, w0, 1);
    w1 |= __shfl_xor_sync(FULL, w1, 1);
    const uint64_t w = (c & 1) ? w1 : w0;
    uint16_t* p = reinterpret_cast<uint16_t*>(blk + RB * (g + 8 * (c & 1)) + 6 * (c >> 1));
    p[0] = (uint16_t)w;
    p[1] = (uint16_t)(w >> 16);
    p[2] = (uint16_t)(w >> 32);
  }
}

template <int D>
struct EncCfg {
  static constexpr int NG = D / 16;           // channel groups
  static constexpr int UNIT = 256;            // tokens per stage
  static constexpr int TILES = UNIT / 16;     // 16-token tiles per stage
  static constexpr int WPG = kWarps / NG;     // warps per group
  static constexpr int BPW = TILES / WPG;     // range blocks per warp and stage: 8 (d = 128) or 4 (d = 64)
  static constexpr int XBYTES = UNIT * D * 2;  // one stage of bf16: 64 KB or 32 KB
  static constexpr int BOX = UNIT * 128;       // one 64-channel TMA box of the stage
  static constexpr int NST = D == 128 ? 3 : 6;
  static constexpr int SMEM = 1024 + NST * XBYTES + NST * 8 + NST * 4 + 16;
};


}  // namespace

template <int D, int BITS>
__global__ void __launch_bounds__(kThreads, 1) encode_mma16_kernel(const __grid_constant__ CUtensorMap tmap, CodecArgs a) {
  using C = EncCfg<D>;
  constexpr int QMAX = (1 << BITS) - 1;
  constexpr int NST = C::NST;
  constexpr int BPW = C::BPW;
  static_assert(BPW == 8 || BPW == 4, "one lane per block's parameters");
  extern __shared__ unsigned char smem_raw[];
  unsigned char* xs = reinterpret_cast<unsigned char*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(xs + NST * C::XBYTES);
  uint32_t* released = reinterpret_cast<uint32_t*>(full + NST);
  uint32_t* ctl = released + NST;  // [0] abort flag, [1] units issued
  volatile uint32_t* abort_v = ctl;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int r = warp % C::NG;           // this warp's channel group
  const int tq = warp / C::NG;          // its share of a stage's tiles: tq*BPW .. tq*BPW + BPW-1
  const int bps = (a.nt + C::UNIT - 1) / C::UNIT;  // stages per head slice
  const long long total = (long long)bps * a.k.slices();
  const long long u0 = total * blockIdx.x / gridDim.x;
  const long long u1 = total * (blockIdx.x + 1) / gridDim.x;
  const int n_units = (int)(u1 - u0);
  const int T16 = a.k.T / 16;

  // stage loads: slot st <- unit at cursor p
  auto issue = [&](int st, const Cursor& p) {
    mbar_arrive_expect_tx(&full[st], C::XBYTES);
    const int row0 = (int)(p.slice * a.k.T + a.t0 + (long long)C::UNIT * p.bq);
#pragma unroll
    for (int bx = 0; bx < D / 64; ++bx) tma_load_2d(xs + st * C::XBYTES + bx * C::BOX, &tmap, 64 * bx, row0, &full[st]);
  };
  Cursor cur{u0 / bps, (int)(u0 % bps)};  // the unit this CTA consumes next
  Cursor pre = cur;                        // the unit NST ahead of it (next to be loaded)
  if (threadIdx.x == 0) {
    for (int st = 0; st < NST; ++st) {
      mbar_init(&full[st], 1);
      released[st] = 0;
    }
    ctl[0] = 0u;                                   // set by the first wait that gives up
    ctl[1] = (uint32_t)(n_units < NST ? n_units : NST);  // units whose loads were issued (a prefix)
    fence_mbar_init();
  }
  __syncthreads();
  for (int q = 0; q < NST; ++q) {
    if (q < n_units && threadIdx.x == 0) issue(q, pre);
    pre.next(bps);
  }

  // ldmatrix row address of lane l inside a tile: rows (l & 7) + 8 ((l >> 3) & 1),
  // 16-byte chunk 2 (r & 3) + (l >> 4) of the 128-byte swizzled row of box r / 4
  const int lrow = (lane & 7) + 8 * ((lane >> 3) & 1);
  const uint32_t xs_lane = smem_u32(xs) + (r >> 2) * C::BOX + (tq * BPW * 16 + lrow) * 128 +
                           (((2 * (r & 3) + (lane >> 4)) ^ (lrow & 7)) << 4);

  uint32_t bh[2][2], bl[2][2];  // [n-half][b0/b1] bf16 pairs of G_hi, G_lo
  long long gslice = -1;
  int s = 0;
  uint32_t phase = 0;

  for (int q = 0; q < n_units; ++q) {
    const long long slice = cur.slice;
    if (slice != gslice) {
      // B fragments of this group: B[k][n] = G[i][k], i = 4 (n >> 1) + 2 h + (n & 1) for
      // n-half h, so a thread's accumulators are output channels 4c .. 4c+3
      int l, sk, b, h;
      slice_coords(slice, a.k, l, sk, b, h);
      const float* Gr = a.G + (gauge_set(l, sk, h, a.k) * C::NG + r) * 256;
#pragma unroll
      for (int nh = 0; nh < 2; ++nh) {
        const int i = 4 * (g >> 1) + 2 * nh + (g & 1);
        const float2 p0 = __ldg(reinterpret_cast<const float2*>(Gr + i * 16 + 2 * c));
        const float2 p1 = __ldg(reinterpret_cast<const float2*>(Gr + i * 16 + 2 * c + 8));
        const float2 p[2] = {p0, p1};
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const uint32_t hi = pack_bf16x2(p[k].x, p[k].y);
          bh[nh][k] = hi;
          bl[nh][k] = pack_bf16x2(p[k].x - bf16lo(hi), p[k].y - bf16hi(hi));  // residuals are exact
        }
      }
      gslice = slice;
    }
    const int valid = min(C::TILES, (a.nt - C::UNIT * cur.bq) / 16) - tq * BPW;  // this warp's tiles in range

    stage_wait(&full[s], phase, abort_v, a.status);
    // Every block of the stage is computed whether or not its tile lies inside
    // [t0, t0 + nt) (rows past the range are still inside the stage buffer); only
    // the stores are predicated.  With no branch per block the compiler can
    // interleave the eight blocks' dependency chains.
    // Each block's fragments go straight into its MMAs (two terms, two n-halves).
    float acc[BPW][2][4];
#pragma unroll
    for (int j = 0; j < BPW; ++j) {
      if (j >= valid) continue;
      uint32_t afr[4];
      ldmatrix_x4(afr, xs_lane + s * C::XBYTES + j * 2048);
#pragma unroll
      for (int nh = 0; nh < 2; ++nh) {
        mma_bf16_16816_z(acc[j][nh], afr, bl[nh][0], bl[nh][1]);
        mma_bf16_16816(acc[j][nh], afr, bh[nh][0], bh[nh][1]);
      }
    }
    // the stage is in registers: release it (the last warp refills the slot)
    __syncwarp();
    if (lane == 0 && stage_release(&released[s]) == kWarps - 1) {
      released[s] = 0;
      if (q + NST < n_units && !*abort_v) {  // nothing more is loaded after a wait gave up
        issue(s, pre);
        ctl[1] = (uint32_t)(q + NST + 1);  // refills run in unit order (ordered by the release atomics)
      }
    }
    pre.next(bps);

    // block ranges (a warp's 16 x 16 tile of its group is one range block); lane l
    // keeps those of block j = l mod BPW
    const int jl = lane & (BPW - 1);
    float mn = 0.0f, mx = 0.0f;
#pragma unroll
    for (int j = 0; j < BPW; ++j) {
      const float* v0 = acc[j][0];
      const float* v1 = acc[j][1];
      const float bmn = redux_min(min3f(min3f(v0[0], v0[1], v0[2]), min3f(v0[3], v1[0], v1[1]), fminf(v1[2], v1[3])));
      const float bmx = redux_max(max3f(max3f(v0[0], v0[1], v0[2]), max3f(v0[3], v1[0], v1[1]), fmaxf(v1[2], v1[3])));
      if (jl == j) {
        mn = bmn;
        mx = bmx;
      }
    }
    mn = __fadd_rn(mn, 0.0f);  // a zero extreme is +0
    mx = __fadd_rn(mx, 0.0f);
    const __half zh = __float2half_rn(fminf(fmaxf(mn, -65504.0f), 65504.0f));
    const __half sh = __float2half_rn(fminf(div_qmax<QMAX>(__fsub_rn(mx, mn)), 65504.0f));
    const float zf = __half2float(zh), sf = __half2float(sh);
    const float inv = sf != 0.0f ? __frcp_rn(sf) : 0.0f;
    // t is monotone in y: the block needs no clamping when its extremes round into [0, qmax]
    const float t_lo = __fmul_rn(__fsub_rn(mn, zf), inv), t_hi = __fmul_rn(__fsub_rn(mx, zf), inv);
    const uint32_t clampm = __ballot_sync(0xffffffffu, !(t_lo >= -0.5f && t_hi < (float)QMAX + 0.5f));
    const float nzf = -zf;
    const long long tile0 = cur.slice * T16 + a.t0 / 16 + (C::UNIT / 16) * (long long)cur.bq + tq * BPW;
    if (lane < BPW && lane < valid) {
      const long long bidx = (tile0 + lane) * C::NG + r;
      a.scales[bidx] = __half_as_ushort(sh);
      a.zeros[bidx] = __half_as_ushort(zh);
    }
    uint8_t* blk0 = a.codes + (tile0 * C::NG + r) * (32 * BITS);
    float* grow0 = a.gauged ? a.gauged + (cur.slice * a.k.T + (tile0 - cur.slice * T16) * 16 + g) * D + 16 * r + 4 * c
                            : nullptr;
#pragma unroll
    for (int j = 0; j < BPW; ++j) {
      const bool ok = j < valid;
      const float nz = __shfl_sync(0xffffffffu, nzf, j);
      const float iv = __shfl_sync(0xffffffffu, inv, j);
      const f2_t nz2 = f2_make(nz, nz), iv2 = f2_make(iv, iv), mg2 = f2_make(kMagic, kMagic);
      // rows g (e = 0, 1 of both n-halves) and g + 8 (e = 2, 3): channels 4c .. 4c+3
      float t[8];
      {
        const f2_t y[4] = {f2_make(acc[j][0][0], acc[j][0][1]), f2_make(acc[j][1][0], acc[j][1][1]),
                           f2_make(acc[j][0][2], acc[j][0][3]), f2_make(acc[j][1][2], acc[j][1][3])};
#pragma unroll
        for (int k = 0; k < 4; ++k) f2_split(f2_mul(f2_add(y[k], nz2), iv2), t[2 * k], t[2 * k + 1]);
      }
      if ((clampm >> j) & 1u) {
#pragma unroll
        for (int k = 0; k < 8; ++k) t[k] = fminf(fmaxf(t[k], 0.0f), (float)QMAX);
      }
      uint32_t rb[8];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float lo, hi;
        f2_split(f2_add(f2_make(t[2 * k], t[2 * k + 1]), mg2), lo, hi);
        rb[2 * k] = __float_as_uint(lo);
        rb[2 * k + 1] = __float_as_uint(hi);
      }
      const uint32_t v0c = chunk4<BITS>(rb[0], rb[1], rb[2], rb[3]), v1c = chunk4<BITS>(rb[4], rb[5], rb[6], rb[7]);
      if (ok) store_rows<BITS>(blk0 + j * (C::NG * 32 * BITS), g, c, v0c, v1c);
      if (grow0 && ok) {
        float* gr = grow0 + j * 16 * D;
        *reinterpret_cast<float4*>(gr) = make_float4(acc[j][0][0], acc[j][0][1], acc[j][1][0], acc[j][1][1]);
        *reinterpret_cast<float4*>(gr + 8 * D) = make_float4(acc[j][0][2], acc[j][0][3], acc[j][1][2], acc[j][1][3]);
      }
    }
    cur.next(bps);
    if (++s == NST) {
      s = 0;
      phase ^= 1u;
    }
  }
  drain_stages(full, ctl, NST, a.status);
}

namespace {

template <int D, int BITS>
struct DecCfg {
  static constexpr int NG = D / 16;
  static constexpr int UNIT = D == 128 ? 256 : 512;  // tokens per stage
  static constexpr int TILES = UNIT / 16;
  static constexpr int WPG = kWarps / NG;
  static constexpr int BPW = TILES / WPG;             // 8 blocks per warp and stage
  static constexpr int TILE_BYTES = 16 * D * BITS / 8;
  static constexpr int CBYTES = TILES * TILE_BYTES;   // one stage of codes (16 KB at 4 bits)
  static constexpr int CSLACK = 16;                   // word reads of 3 and 6-bit rows may pass the end
  static constexpr int SZB = TILES * NG * 2 + 32;     // steps (or zero points) of a stage, with alignment slack
  static constexpr int CSTAGE = CBYTES + CSLACK + 2 * SZB;
  static constexpr int NST = CBYTES >= 24 * 1024 ? 5 : 8;
  static constexpr int SMEM = 128 + NST * CSTAGE + NST * 8 + NST * 4 + 16;
};

}  // namespace

template <int D, int BITS>
__global__ void __launch_bounds__(kThreads, 1) decode_mma16_kernel(CodecArgs a) {
  using C = DecCfg<D, BITS>;
  constexpr int NST = C::NST;
  constexpr int BPW = C::BPW;
  static_assert(C::CSTAGE % 16 == 0, "stages stay 16-byte aligned");
  extern __shared__ unsigned char smem_raw[];
  unsigned char* cs = reinterpret_cast<unsigned char*>(((uintptr_t)smem_raw + 127) & ~(uintptr_t)127);
  uint64_t* full = reinterpret_cast<uint64_t*>(cs + NST * C::CSTAGE);
  uint32_t* released = reinterpret_cast<uint32_t*>(full + NST);
  uint32_t* ctl = released + NST;  // [0] abort flag, [1] units issued
  volatile uint32_t* abort_v = ctl;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int r = warp % C::NG;
  const int tq = warp / C::NG;
  const int tps = a.nt / 16;
  const int sps = (tps + C::TILES - 1) / C::TILES;  // stages per head slice
  const long long total = (long long)sps * a.k.slices();
  const long long u0 = total * blockIdx.x / gridDim.x;
  const long long u1 = total * (blockIdx.x + 1) / gridDim.x;
  const int n_units = (int)(u1 - u0);
  const long long slice_code_bytes = (long long)a.k.T * D * BITS / 8;
  const int T16 = a.k.T / 16;

  // The stage's steps and zero points are fp16 [tile][group]; their byte range
  // starts at b0 = 2 NG (slice T/16 + first tile).  The copies start at b0
  // rounded down to 16 bytes (a head slice's range is 16-byte aligned at both
  // ends, so the rounded range stays inside it); sz_off = b0 mod 16.
  auto sz_start = [&](const Cursor& p) -> long long {
    return 2LL * C::NG * (p.slice * T16 + a.t0 / 16 + (long long)C::TILES * p.bq);
  };
  auto issue = [&](int st, const Cursor& p) {
    const int nvalid = min(C::TILES, tps - C::TILES * p.bq);
    const uint32_t bytes = (uint32_t)(nvalid * C::TILE_BYTES);
    const long long b0 = sz_start(p), a0 = b0 & ~15LL;
    const uint32_t szb = (uint32_t)((b0 - a0 + 2 * C::NG * nvalid + 15) & ~15LL);
    mbar_arrive_expect_tx(&full[st], bytes + 2 * szb);
    unsigned char* dst = cs + st * C::CSTAGE;
    const long long tl0 = a.t0 / 16 + (long long)C::TILES * p.bq;
    bulk_g2s(dst, a.codes_in + p.slice * slice_code_bytes + tl0 * C::TILE_BYTES, bytes, &full[st]);
    bulk_g2s(dst + C::CBYTES + C::CSLACK, reinterpret_cast<const unsigned char*>(a.scales_in) + a0, szb, &full[st]);
    bulk_g2s(dst + C::CBYTES + C::CSLACK + C::SZB, reinterpret_cast<const unsigned char*>(a.zeros_in) + a0, szb,
             &full[st]);
  };
  Cursor cur{u0 / sps, (int)(u0 % sps)};
  Cursor pre = cur;
  if (threadIdx.x == 0) {
    for (int st = 0; st < NST; ++st) {
      mbar_init(&full[st], 1);
      released[st] = 0;
    }
    ctl[0] = 0u;                                   // set by the first wait that gives up
    ctl[1] = (uint32_t)(n_units < NST ? n_units : NST);  // units whose loads were issued (a prefix)
    fence_mbar_init();
  }
  __syncthreads();
  for (int q = 0; q < NST; ++q) {
    if (q < n_units && threadIdx.x == 0) issue(q, pre);
    pre.next(sps);
  }

  uint32_t bh[2][2], bl[2][2];  // [n-half][b0/b1] fp16 pairs of G hi, lo (k order permuted, below)
  float csum[4];                // column sums sum_c G[c][n] of this thread's 4 output channels
  long long gslice = -1;
  int s = 0;
  uint32_t phase = 0;
  // this thread's row chunk inside a block: rows g and g + 8, codes 4c .. 4c+3
  const int bit_g = (16 * g + 4 * c) * BITS, bit_g8 = (16 * (g + 8) + 4 * c) * BITS;

  for (int q = 0; q < n_units; ++q) {
    const long long slice = cur.slice;
    if (slice != gslice) {
      // A's k slots 2c, 2c+1 hold channels 4c, 4c+1 and slots 2c+8, 2c+9 hold 4c+2, 4c+3, so a
      // thread reads 4 adjacent codes; B follows: B[slot][n] = G[ch(slot)][4 (n >> 1) + 2 h + (n & 1)]
      int l, sk, b, h;
      slice_coords(slice, a.k, l, sk, b, h);
      const float* Gr = a.G + (gauge_set(l, sk, h, a.k) * C::NG + r) * 256;  // G[c][n], row-major
#pragma unroll
      for (int nh = 0; nh < 2; ++nh) {
        const int n = 4 * (g >> 1) + 2 * nh + (g & 1);
        float gv[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) gv[k] = __ldg(Gr + (4 * c + k) * 16 + n);
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const uint32_t h0 = f16_bits(gv[2 * k]), h1 = f16_bits(gv[2 * k + 1]);
          const float r0 = gv[2 * k] - __half2float(__ushort_as_half((unsigned short)h0));
          const float r1 = gv[2 * k + 1] - __half2float(__ushort_as_half((unsigned short)h1));
          bh[nh][k] = h0 | (h1 << 16);
          bl[nh][k] = f16_bits(r0) | (f16_bits(r1) << 16);
        }
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float* col = Gr + 4 * c + k;
        float sacc = 0.0f;
#pragma unroll
        for (int cc = 0; cc < 16; ++cc) sacc += __ldg(col + cc * 16);
        csum[k] = sacc;
      }
      gslice = slice;
    }
    const int valid = min(C::TILES, tps - C::TILES * cur.bq) - tq * BPW;  // this warp's tiles in range
    const long long tile0 = slice * T16 + a.t0 / 16 + (long long)C::TILES * cur.bq + tq * BPW;
    const int sz_off = (int)(sz_start(cur) & 15);

    stage_wait(&full[s], phase, abort_v, a.status);
    const unsigned char* sbase = cs + s * C::CSTAGE;
    const unsigned char* cblk = sbase + (tq * BPW * C::NG + r) * (32 * BITS);
    const __half* szp = reinterpret_cast<const __half*>(sbase + C::CBYTES + C::CSLACK + sz_off) + tq * BPW * C::NG + r;
    uint32_t cv[BPW][2];  // rows g, g+8: this thread's 4 codes (4*BITS bits, low aligned)
    float sf[BPW], zf[BPW];
#pragma unroll
    for (int j = 0; j < BPW; ++j) {
      if (j < valid) {
        const unsigned char* blk = cblk + j * (C::NG * 32 * BITS);
        if constexpr (BITS == 4) {
          cv[j][0] = *reinterpret_cast<const uint16_t*>(blk + (bit_g >> 3));
          cv[j][1] = *reinterpret_cast<const uint16_t*>(blk + (bit_g8 >> 3));
        } else if constexpr (BITS == 8) {
          cv[j][0] = *reinterpret_cast<const uint32_t*>(blk + (bit_g >> 3));
          cv[j][1] = *reinterpret_cast<const uint32_t*>(blk + (bit_g8 >> 3));
        } else if constexpr (BITS == 2) {
          cv[j][0] = blk[bit_g >> 3];
          cv[j][1] = blk[bit_g8 >> 3];
        } else {
          const uint32_t* w0 = reinterpret_cast<const uint32_t*>(blk) + (bit_g >> 5);
          const uint32_t* w1 = reinterpret_cast<const uint32_t*>(blk) + (bit_g8 >> 5);
          cv[j][0] = __funnelshift_r(w0[0], w0[1], bit_g & 31);
          cv[j][1] = __funnelshift_r(w1[0], w1[1], bit_g8 & 31);
        }
        sf[j] = __half2float(szp[j * C::NG]);
        zf[j] = __half2float(szp[j * C::NG + C::SZB / 2]);
      }
    }
    __syncwarp();
    if (lane == 0 && stage_release(&released[s]) == kWarps - 1) {
      released[s] = 0;
      if (q + NST < n_units && !*abort_v) {  // nothing more is loaded after a wait gave up
        issue(s, pre);
        ctl[1] = (uint32_t)(q + NST + 1);  // refills run in unit order (ordered by the release atomics)
      }
    }
    pre.next(sps);

    // output rows: even c writes row g, channels 4c .. 4c+7; odd c writes row g + 8,
    // channels 4c - 4 .. 4c+3 (partners swap the other row's half through a shuffle)
    const bool odd = c & 1;
    uint16_t* orow0 = a.kv_out + (slice * a.k.T + (tile0 - slice * T16) * 16 + g + (odd ? 8 : 0)) * D + 16 * r +
                      4 * (c & 2);
#pragma unroll
    for (int j = 0; j < BPW; ++j) {
      if (j >= valid) continue;
      uint32_t afr[4];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const uint32_t v = cv[j][hh];
        if constexpr (BITS == 4) {
          const uint32_t e = (v & 0x0F0Fu) | 0x64640000u;         // bytes c0, c2, 0x64, 0x64
          const uint32_t o = ((v >> 4) & 0x0F0Fu) | 0x64640000u;  // bytes c1, c3, 0x64, 0x64
          afr[hh] = f16_sub1024(__byte_perm(e, o, 0x6420));
          afr[2 + hh] = f16_sub1024(__byte_perm(e, o, 0x6521));
        } else {
          constexpr uint32_t M = (1u << BITS) - 1u;
          afr[hh] = f16_sub1024(0x64006400u | (v & M) | (((v >> BITS) & M) << 16));
          afr[2 + hh] = f16_sub1024(0x64006400u | ((v >> (2 * BITS)) & M) | (((v >> (3 * BITS)) & M) << 16));
        }
      }
      uint32_t pk[2][2];  // [row g / g+8][channels 4c,4c+1 / 4c+2,4c+3] bf16 pairs
#pragma unroll
      for (int nh = 0; nh < 2; ++nh) {
        float acc[4];
        mma_f16_16816_z(acc, afr, bl[nh][0], bl[nh][1]);
        mma_f16_16816(acc, afr, bh[nh][0], bh[nh][1]);
        const float cz0 = zf[j] * csum[2 * nh], cz1 = zf[j] * csum[2 * nh + 1];
        pk[0][nh] = pack_bf16x2(__fmaf_rn(sf[j], acc[0], cz0), __fmaf_rn(sf[j], acc[1], cz1));
        pk[1][nh] = pack_bf16x2(__fmaf_rn(sf[j], acc[2], cz0), __fmaf_rn(sf[j], acc[3], cz1));
      }
      const uint32_t send0 = odd ? pk[0][0] : pk[1][0], send1 = odd ? pk[0][1] : pk[1][1];
      const uint32_t got0 = __shfl_xor_sync(0xffffffffu, send0, 1), got1 = __shfl_xor_sync(0xffffffffu, send1, 1);
      const uint4 v = odd ? make_uint4(got0, got1, pk[1][0], pk[1][1]) : make_uint4(pk[0][0], pk[0][1], got0, got1);
      *reinterpret_cast<uint4*>(orow0 + j * 16 * D) = v;
    }
    cur.next(sps);
    if (++s == NST) {
      s = 0;
      phase ^= 1u;
    }
  }
  drain_stages(full, ctl, NST, a.status);
}

namespace {

template <int D, int BITS>
cudaError_t enc_launch(const CodecArgs& a, int num_sms, cudaStream_t st) {
  using C = EncCfg<D>;
  alignas(64) CUtensorMap tmap;
  const uint64_t rows = (uint64_t)a.k.slices() * a.k.T;
  if (!make_tmap_2d_bf16(&tmap, a.kv, rows, D, 64, C::UNIT)) return cudaErrorInvalidValue;
  auto kern = encode_mma16_kernel<D, BITS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const long long total = (long long)((a.nt + C::UNIT - 1) / C::UNIT) * a.k.slices();
  const int grid = (int)(total < num_sms ? total : num_sms);
  kern<<<grid, kThreads, C::SMEM, st>>>(tmap, a);
  return cudaGetLastError();
}

template <int D, int BITS>
cudaError_t dec_launch(const CodecArgs& a, int num_sms, cudaStream_t st) {
  using C = DecCfg<D, BITS>;
  auto kern = decode_mma16_kernel<D, BITS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const long long total = (long long)((a.nt / 16 + C::TILES - 1) / C::TILES) * a.k.slices();
  const int grid = (int)(total < num_sms ? total : num_sms);
  kern<<<grid, kThreads, C::SMEM, st>>>(a);
  return cudaGetLastError();
}

template <int D>
cudaError_t enc_bits(const CodecArgs& a, int num_sms, cudaStream_t st) {
  switch (a.bits) {
    case 2: return enc_launch<D, 2>(a, num_sms, st);
    case 3: return enc_launch<D, 3>(a, num_sms, st);
    case 4: return enc_launch<D, 4>(a, num_sms, st);
    case 6: return enc_launch<D, 6>(a, num_sms, st);
    case 8: return enc_launch<D, 8>(a, num_sms, st);
  }
  return cudaErrorInvalidValue;
}

template <int D>
cudaError_t dec_bits(const CodecArgs& a, int num_sms, cudaStream_t st) {
  switch (a.bits) {
    case 2: return dec_launch<D, 2>(a, num_sms, st);
    case 3: return dec_launch<D, 3>(a, num_sms, st);
    case 4: return dec_launch<D, 4>(a, num_sms, st);
    case 6: return dec_launch<D, 6>(a, num_sms, st);
    case 8: return dec_launch<D, 8>(a, num_sms, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool codec_mma16_supported(const CodecArgs& a) {
  return a.g == 16 && a.W == 16 && !a.kivi && (a.k.d == 64 || a.k.d == 128);
}

cudaError_t launch_encode_mma16(const CodecArgs& a, int num_sms, cudaStream_t st) {
  if (a.nt == 0) return cudaSuccess;
  if (!codec_mma16_supported(a)) return cudaErrorInvalidValue;
  return a.k.d == 128 ? enc_bits<128>(a, num_sms, st) : enc_bits<64>(a, num_sms, st);
}

cudaError_t launch_decode_mma16(const CodecArgs& a, int num_sms, cudaStream_t st) {
  if (a.nt == 0) return cudaSuccess;
  if (!codec_mma16_supported(a)) return cudaErrorInvalidValue;
  return a.k.d == 128 ? dec_bits<128>(a, num_sms, st) : dec_bits<64>(a, num_sms, st);
}

}  // namespace cg
