// Gauge-training statistics: 2-D orthonormal DCT-II spectral centroid and rate
// proxy per T_b x d block of the gauged cache, and their gradient w.r.t. G.
//
// Codec-Gauge, Method (frequency-distribution objective): X' = G X is cut into
// 16-token blocks spanning the whole head; each block gets U = C_16 X' C_d^T;
// L_freq = sum r_uv U^2 / sum U^2 with the normalized radius r_uv, the rate
// proxy L_rate = mean log(1 + |U| / tau) (assumed form: the page's equation is
// truncated), L = lambda_f mean L_freq + lambda_r mean L_rate.
//
// One CTA owns whole head slices (so each slice's dG partial comes from one CTA
// and the result is deterministic) and walks them in tiles of 128 tokens:
//   A  (4 warps, thread = token row)  X' row = G x (fp32), split into bf16
//      hi + lo, written as the swizzled K-major A operand;
//   B  (1 thread)  U1 = X' C_d^T on tcgen05 with X' = A_hi + A_lo and C_d split
//      into three bf16 terms (exact to 24 bits: an inexact transform matrix
//      would bias every token the same way and the bias would add up in dG):
//      A_hi (C_1 + C_2 + C_3) + A_lo (C_1 + C_2), fp32 accumulate in TMEM;
//   C  (thread = channel column v)  token DCT of each 16-token block, the
//      block's sums sum U^2, sum r U^2, sum log1p(|U|/tau) (warp + shared-memory
//      reduction), per-block L_freq / L_rate; with a gradient:
//        dU = lambda_f 2 U (r - L_freq) / (E n_blk) + lambda_r sign(U) / ((tau + |U|) N_U),
//      dU1 = C_16^T dU, written as the bf16 hi + lo operand;
//   D  (1 thread)  dX'^T = C_d^T dU1^T on tcgen05 (C_d read through an MN-major
//      descriptor of the same tiles);
//   E  (thread = channel c = 16 r + i)  dG_r[i][j] += sum_t dX'[t][c] x[t][16 r + j].
#include <cuda.h>

#include "cg_kernels.cuh"

namespace cg {

namespace {

constexpr int kTile = 128;      // tokens per tile
constexpr int kD = 128;         // d_head of this kernel
constexpr int kOpBytes = kTile * kD * 2;  // one bf16 128 x 128 operand: 32 KB
constexpr int kSPitch = 129;    // fp32 pitch of the 128 x 128 staging matrix
constexpr int kWorkers = 256;  // 8 worker warps; warp 8 issues the MMAs
constexpr int kSpecThreads = kWorkers + 32;

// K-major, 128-byte swizzle (rows of 128 B; 8-row atoms 1024 B apart)
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t addr) {
  uint64_t d = (uint64_t)((addr & 0x3FFFFu) >> 4);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}
// MN-major, 128-byte swizzle, over the same storage: rows are K, 64 MN
// elements per 128-byte row; the two 64-element MN halves are 16 KB apart
// (leading byte offset), 8-row K groups 1024 B apart (stride byte offset).
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t addr) {
  uint64_t d = (uint64_t)((addr & 0x3FFFFu) >> 4);
  d |= (uint64_t)(16384 >> 4) << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}
// D fp32, A / B bf16, M = N = 128; a_mn / b_mn select MN-major operands
__host__ __device__ constexpr uint32_t idesc_bf16(bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((128u >> 3) << 17) | ((128u >> 4) << 24);
}
__device__ __forceinline__ void umma(uint32_t tmem_d, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
          tmem_d),
      "l"(ad), "l"(bd), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
      "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
// byte offset of (row, col) in a swizzled 128 x 128 bf16 operand (two 64-column halves)
__device__ __forceinline__ uint32_t swz(int row, int col) {
  return (col >> 6) * 16384 + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) + (col & 7) * 2;
}
__device__ __forceinline__ uint16_t bf16_rn(float x) { return __bfloat16_as_ushort(__float2bfloat16_rn(x)); }
__device__ __forceinline__ float bf16_f(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

struct SpecArgs {
  KvGeom k;
  int x_fp32, has_g, want_grad;
  float lambda_f, lambda_r, tau;
  double inv_nblk, inv_ncoef;  // 1 / n_blocks, 1 / (n_blocks * 16 * d)
  const void* x;
  const float* G;              // [L][2][H][8][16][16] (g = 16) or null
  float* lfreq;
  float* lrate;
  float* dg_part;              // [slices][8][16][16] workspace
  unsigned int* status;
};

struct SpecSmem {
  unsigned char* c1;   // C_d = c1 + c2 + c3 (bf16 terms; rows v, cols c), swizzled
  unsigned char* c2;
  unsigned char* c3;
  unsigned char* ahi;  // X' hi / dU1 hi (rows t)
  unsigned char* alo;
  float* S;            // [128][kSPitch] fp32: U1
  float* Gs;           // [8][16][16], inside S (used in phase A only)
  float* C16;          // [16][16]
  float* red;          // [4 warps][3]
  float* blk;          // [2]: L_freq, E of the current block
  uint64_t* bars;      // a_full, t_full, d_full, t2_full
  uint32_t* tmem_base;
};
constexpr int kSpecSmem = 1024 + 5 * kOpBytes + kTile * kSPitch * 4 + (256 + 32 + 8) * 4 + 4 * 8 + 16;

__device__ inline SpecSmem spec_carve(unsigned char* raw) {
  SpecSmem s;
  unsigned char* base = reinterpret_cast<unsigned char*>(((uintptr_t)raw + 1023) & ~(uintptr_t)1023);
  s.c1 = base;
  s.c2 = base + kOpBytes;
  s.c3 = base + 2 * kOpBytes;
  s.ahi = base + 3 * kOpBytes;
  s.alo = base + 4 * kOpBytes;
  s.S = reinterpret_cast<float*>(base + 5 * kOpBytes);
  s.Gs = s.S;
  s.C16 = s.S + kTile * kSPitch;
  s.red = s.C16 + 256;
  s.blk = s.red + 32;
  s.bars = reinterpret_cast<uint64_t*>(s.blk + 8);
  s.tmem_base = reinterpret_cast<uint32_t*>(s.bars + 4);
  return s;
}

__device__ __forceinline__ float dct_coef(int k, int n, int N) {
  const float a = k == 0 ? sqrtf(1.0f / N) : sqrtf(2.0f / N);
  return a * cospif((2.0f * n + 1.0f) * k / (2.0f * N));
}

}  // namespace

__global__ void __launch_bounds__(kSpecThreads, 1) spectral_kernel(SpecArgs a) {
  extern __shared__ unsigned char smem_raw[];
  const SpecSmem sm = spec_carve(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  uint64_t* a_full = &sm.bars[0];
  uint64_t* t_full = &sm.bars[1];
  uint64_t* d_full = &sm.bars[2];
  uint64_t* t2_full = &sm.bars[3];
  const long long slices = a.k.slices();
  const int tiles = a.k.T / kTile;

  // constants: C_d (split into bf16 hi + lo), C_16
  for (int e = tid; e < kD * kD; e += kSpecThreads) {
    const int v = e / kD, c = e % kD;
    const float cf = dct_coef(v, c, kD);
    const uint16_t t1 = bf16_rn(cf);
    const float r1 = cf - bf16_f(t1);
    const uint16_t t2 = bf16_rn(r1);
    *reinterpret_cast<uint16_t*>(sm.c1 + swz(v, c)) = t1;
    *reinterpret_cast<uint16_t*>(sm.c2 + swz(v, c)) = t2;
    *reinterpret_cast<uint16_t*>(sm.c3 + swz(v, c)) = bf16_rn(r1 - bf16_f(t2));
  }
  for (int e = tid; e < 256; e += kSpecThreads) sm.C16[e] = dct_coef(e / 16, e % 16, 16);
  if (tid == 0) {
    mbar_init(a_full, kWorkers / 32);
    mbar_init(t_full, 1);
    mbar_init(d_full, kWorkers / 32);
    mbar_init(t2_full, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(sm.tmem_base)),
                 "r"(256));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  fence_proxy_async_smem();
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *sm.tmem_base;  // columns [0,128): U1 ; [128,256): dX'^T
  const uint32_t id_fwd = idesc_bf16(false, false), id_bwd = idesc_bf16(true, false);

  // normalized radius r_uv of this thread's channel-frequency column (phase C)
  float rad[16];
  {
    const float rv = (float)(tid & 127) / (kD - 1);
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const float ru = (float)u / 15.0f;
      rad[u] = sqrtf(ru * ru + rv * rv) * 0.70710678118654752f;
    }
  }
  int it = 0;  // tiles processed by this CTA (mbarrier phases)
  for (long long slice = blockIdx.x; slice < slices; slice += gridDim.x) {
    int l, sk, b, h;
    slice_coords(slice, a.k, l, sk, b, h);
    const float* Gp = a.has_g ? a.G + gauge_set(l, sk, h, a.k) * kD * 16 : nullptr;
    // dG partial of this thread's channel over the slice: each tile's 64 products are
    // summed afresh and the tile sums added in order, so the rounding grows with
    // 64 + (tiles per slice) terms rather than with the slice's token count
    float dg[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) dg[j] = 0.0f;

    for (int tile = 0; tile < tiles; ++tile, ++it) {
      const uint32_t ph = (uint32_t)(it & 1);
      const long long row0 = slice * a.k.T + (long long)tile * kTile;
      if (warp == kWorkers / 32) {
        // ---------------- MMA issue ----------------
        if (lane == 0) {
          mbar_wait(a_full, ph, a.status);
          fence_after();
          const uint32_t A0 = smem_u32(sm.ahi), A1 = smem_u32(sm.alo);
          const uint32_t C0 = smem_u32(sm.c1), C1 = smem_u32(sm.c2), C2 = smem_u32(sm.c3);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t ko = (k >> 2) * 16384 + (k & 3) * 32;
            umma(tmem, desc_kmajor(A0 + ko), desc_kmajor(C0 + ko), id_fwd, k > 0);
            umma(tmem, desc_kmajor(A0 + ko), desc_kmajor(C1 + ko), id_fwd, 1);
            umma(tmem, desc_kmajor(A0 + ko), desc_kmajor(C2 + ko), id_fwd, 1);
            umma(tmem, desc_kmajor(A1 + ko), desc_kmajor(C0 + ko), id_fwd, 1);
            umma(tmem, desc_kmajor(A1 + ko), desc_kmajor(C1 + ko), id_fwd, 1);
          }
          commit(t_full);
          if (a.want_grad) {
            mbar_wait(d_full, ph, a.status);
            fence_after();
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const uint32_t ka = k * 2048;                            // C_d as MN-major A: K rows 16k..16k+15
              const uint32_t kb = (k >> 2) * 16384 + (k & 3) * 32;     // dU1 as K-major B
              umma(tmem + 128, desc_mnmajor(C0 + ka), desc_kmajor(A0 + kb), id_bwd, k > 0);
              umma(tmem + 128, desc_mnmajor(C1 + ka), desc_kmajor(A0 + kb), id_bwd, 1);
              umma(tmem + 128, desc_mnmajor(C2 + ka), desc_kmajor(A0 + kb), id_bwd, 1);
              umma(tmem + 128, desc_mnmajor(C0 + ka), desc_kmajor(A1 + kb), id_bwd, 1);
              umma(tmem + 128, desc_mnmajor(C1 + ka), desc_kmajor(A1 + kb), id_bwd, 1);
            }
            commit(t2_full);
          }
        }
        continue;
      }
      // ---------------- A: X' row = G x, split into the bf16 operand ----------------
      if (a.has_g) {  // G of this slice, staged in the (idle) U1 buffer
        for (int e = tid; e < 2048; e += kWorkers) sm.Gs[e] = Gp[e];
        named_bar_sync(1, kWorkers);
      }
      {
        const int t = tid & 127, hf = tid >> 7;  // token row, channel half 64 hf .. 64 hf + 63
        float x[64];
        if (a.x_fp32) {
          const float4* src =
              reinterpret_cast<const float4*>(reinterpret_cast<const float*>(a.x) + (row0 + t) * kD + 64 * hf);
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const float4 v = src[q];
            x[4 * q] = v.x; x[4 * q + 1] = v.y; x[4 * q + 2] = v.z; x[4 * q + 3] = v.w;
          }
        } else {
          const uint4* src =
              reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.x) + (row0 + t) * kD + 64 * hf);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint4 w = src[q];
            x[8 * q + 0] = bf16lo(w.x); x[8 * q + 1] = bf16hi(w.x); x[8 * q + 2] = bf16lo(w.y); x[8 * q + 3] = bf16hi(w.y);
            x[8 * q + 4] = bf16lo(w.z); x[8 * q + 5] = bf16hi(w.z); x[8 * q + 6] = bf16lo(w.w); x[8 * q + 7] = bf16hi(w.w);
          }
        }
#pragma unroll
        for (int cb = 0; cb < 8; ++cb) {  // 8 channels per 16-byte chunk
          float y8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int cl = 8 * cb + e, c = 64 * hf + cl;  // local and head channel
            if (a.has_g) {
              const int rl = cl >> 4, r = c >> 4, i = c & 15;
              const float4* gi = reinterpret_cast<const float4*>(sm.Gs + (r * 16 + i) * 16);
              float acc = 0.0f;
#pragma unroll
              for (int j4 = 0; j4 < 4; ++j4) {
                const float4 g = gi[j4];
                acc = __fmaf_rn(g.x, x[16 * rl + 4 * j4], acc);
                acc = __fmaf_rn(g.y, x[16 * rl + 4 * j4 + 1], acc);
                acc = __fmaf_rn(g.z, x[16 * rl + 4 * j4 + 2], acc);
                acc = __fmaf_rn(g.w, x[16 * rl + 4 * j4 + 3], acc);
              }
              y8[e] = acc;
            } else {
              y8[e] = x[cl];
            }
          }
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint16_t h0 = bf16_rn(y8[2 * e]), h1 = bf16_rn(y8[2 * e + 1]);
            hw[e] = (uint32_t)h0 | ((uint32_t)h1 << 16);
            lw[e] = (uint32_t)bf16_rn(y8[2 * e] - bf16_f(h0)) | ((uint32_t)bf16_rn(y8[2 * e + 1] - bf16_f(h1)) << 16);
          }
          *reinterpret_cast<uint4*>(sm.ahi + swz(t, 64 * hf + 8 * cb)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(sm.alo + swz(t, 64 * hf + 8 * cb)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(a_full);
      }
      if (a.has_g) named_bar_sync(1, kWorkers);  // all rows gauged before U1 overwrites the staged G
      // ---------------- C: U1 rows to shared memory, token DCT and block statistics ----------------
      mbar_wait(t_full, ph, a.status);
      fence_after();
      {
        const int t = 32 * (warp & 3) + lane, ch = warp >> 2;  // TMEM lane quarter of this warp, column half
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          const int c4 = 2 * ch + c2;
          float v[32];
          ld32(tmem + 32 * c4 + ((uint32_t)(32 * (warp & 3)) << 16), v);
#pragma unroll
          for (int j = 0; j < 32; ++j) sm.S[t * kSPitch + 32 * c4 + j] = v[j];
        }
      }
      fence_before();
      named_bar_sync(1, kWorkers);
      {
        const int v = tid & 127, bh = tid >> 7;  // channel-frequency column, half of the tile's blocks
        const int obase = (int)(row0 / 16);       // first block index of this tile
        const float inv_tau = 1.0f / a.tau;
        float* red = sm.red + 12 * bh;
        for (int kb = 4 * bh; kb < 4 * bh + 4; ++kb) {
          float col[16], U[16];
#pragma unroll
          for (int t = 0; t < 16; ++t) col[t] = sm.S[(16 * kb + t) * kSPitch + v];
          // 16-point DCT-II through its symmetry C[u][15 - t] = (-1)^u C[u][t]:
          // even u from col[t] + col[15 - t], odd u from col[t] - col[15 - t]
          float sm8[8], df8[8];
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            sm8[t] = col[t] + col[15 - t];
            df8[t] = col[t] - col[15 - t];
          }
          float e_sum = 0.0f, f_sum = 0.0f, r_sum = 0.0f;
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const float4 c0 = reinterpret_cast<const float4*>(sm.C16 + u * 16)[0];
            const float4 c1 = reinterpret_cast<const float4*>(sm.C16 + u * 16)[1];
            float h8[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) h8[t] = (u & 1) ? df8[t] : sm8[t];  // u is a compile-time index
            float acc = c0.x * h8[0];
            acc = __fmaf_rn(c0.y, h8[1], acc);
            acc = __fmaf_rn(c0.z, h8[2], acc);
            acc = __fmaf_rn(c0.w, h8[3], acc);
            acc = __fmaf_rn(c1.x, h8[4], acc);
            acc = __fmaf_rn(c1.y, h8[5], acc);
            acc = __fmaf_rn(c1.z, h8[6], acc);
            acc = __fmaf_rn(c1.w, h8[7], acc);
            U[u] = acc;
            const float e = acc * acc;
            e_sum += e;
            f_sum = __fmaf_rn(rad[u], e, f_sum);
            r_sum += __log2f(__fmaf_rn(fabsf(acc), inv_tau, 1.0f));  // log1p(|U| / tau) / ln 2
          }
          r_sum *= 0.69314718055994531f;
          // block reduction over the 128 columns
#pragma unroll
          for (int o = 16; o >= 1; o >>= 1) {
            e_sum += __shfl_xor_sync(0xffffffffu, e_sum, o);
            f_sum += __shfl_xor_sync(0xffffffffu, f_sum, o);
            r_sum += __shfl_xor_sync(0xffffffffu, r_sum, o);
          }
          if (lane == 0) {
            red[(warp & 3) * 3 + 0] = e_sum;
            red[(warp & 3) * 3 + 1] = f_sum;
            red[(warp & 3) * 3 + 2] = r_sum;
          }
          named_bar_sync(2 + bh, 128);
          const float E = (red[0] + red[3]) + (red[6] + red[9]);
          const float F = (red[1] + red[4]) + (red[7] + red[10]);
          const float R = (red[2] + red[5]) + (red[8] + red[11]);
          const float lf = E > 0.0f ? F / E : 0.0f;
          if (v == 0) {
            a.lfreq[obase + kb] = lf;
            a.lrate[obase + kb] = R / (16.0f * kD);
          }
          if (a.want_grad) {
            // dL/dU, then dU1 = C_16^T dU, written as the bf16 hi + lo operand (rows t, K = v)
            const float cf = E > 0.0f ? (float)(2.0 * a.lambda_f * a.inv_nblk) / E : 0.0f;
            const float cr = (float)(a.lambda_r * a.inv_ncoef);
            float dU[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
              const float sg = U[u] > 0.0f ? 1.0f : (U[u] < 0.0f ? -1.0f : 0.0f);
              dU[u] = __fmaf_rn(cf * U[u], rad[u] - lf, cr * sg / (a.tau + fabsf(U[u])));
            }
            // dU1[t] = sum_u C[u][t] dU[u]: even-u part Ev and odd-u part Od of
            // t < 8 give dU1[t] = Ev + Od and dU1[15 - t] = Ev - Od
#pragma unroll
            for (int t = 0; t < 8; ++t) {
              float ev = 0.0f, od = 0.0f;
#pragma unroll
              for (int u = 0; u < 16; u += 2) {
                ev = __fmaf_rn(sm.C16[u * 16 + t], dU[u], ev);
                od = __fmaf_rn(sm.C16[(u + 1) * 16 + t], dU[u + 1], od);
              }
              const float d0 = ev + od, d1 = ev - od;
              const uint16_t h0 = bf16_rn(d0), h1 = bf16_rn(d1);
              *reinterpret_cast<uint16_t*>(sm.ahi + swz(16 * kb + t, v)) = h0;
              *reinterpret_cast<uint16_t*>(sm.alo + swz(16 * kb + t, v)) = bf16_rn(d0 - bf16_f(h0));
              *reinterpret_cast<uint16_t*>(sm.ahi + swz(16 * kb + 15 - t, v)) = h1;
              *reinterpret_cast<uint16_t*>(sm.alo + swz(16 * kb + 15 - t, v)) = bf16_rn(d1 - bf16_f(h1));
            }
          }
          named_bar_sync(2 + bh, 128);  // red reused by the next block
        }
      }
      if (!a.want_grad) continue;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(d_full);
      // ---------------- E: dG_r[i][j] += sum_t dX'[t][c] x[t][16 r + j], thread c ----------------
      mbar_wait(t2_full, ph, a.status);
      fence_after();
      {
        const int c = tid & 127, r = c >> 4, th = tid >> 7;  // channel (= TMEM lane), token half
        float dgt[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) dgt[j] = 0.0f;
        for (int c4 = 2 * th; c4 < 2 * th + 2; ++c4) {
          float v[32];
          ld32(tmem + 128 + 32 * c4 + ((uint32_t)(32 * (warp & 3)) << 16), v);  // dX'^T row c: tokens 32 c4 ..
#pragma unroll 8
          for (int tt = 0; tt < 32; ++tt) {
            const long long row = row0 + 32 * c4 + tt;
            float xs[16];
            if (a.x_fp32) {
              const float4* src = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(a.x) + row * kD + 16 * r);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const float4 w = __ldg(src + q);
                xs[4 * q] = w.x; xs[4 * q + 1] = w.y; xs[4 * q + 2] = w.z; xs[4 * q + 3] = w.w;
              }
            } else {
              const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.x) + row * kD + 16 * r);
#pragma unroll
              for (int q = 0; q < 2; ++q) {
                const uint4 w = __ldg(src + q);
                xs[8 * q + 0] = bf16lo(w.x); xs[8 * q + 1] = bf16hi(w.x); xs[8 * q + 2] = bf16lo(w.y);
                xs[8 * q + 3] = bf16hi(w.y); xs[8 * q + 4] = bf16lo(w.z); xs[8 * q + 5] = bf16hi(w.z);
                xs[8 * q + 6] = bf16lo(w.w); xs[8 * q + 7] = bf16hi(w.w);
              }
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) dgt[j] = __fmaf_rn(v[tt], xs[j], dgt[j]);
          }
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) dg[j] = __fadd_rn(dg[j], dgt[j]);
      }
      fence_before();
      named_bar_sync(1, kWorkers);
    }
    if (warp < kWorkers / 32 && a.want_grad) {  // the two token halves' partials of channel c, in a fixed order
      const int c = tid & 127;
      float* part = sm.S + c * 16;  // U1 staging is free here
      if (tid >= 128) {
#pragma unroll
        for (int j = 0; j < 16; ++j) part[j] = dg[j];
      }
      named_bar_sync(1, kWorkers);
      if (tid < 128) {
        float4* dst = reinterpret_cast<float4*>(a.dg_part + slice * (long long)kD * 16 + c * 16);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          dst[q] = make_float4(dg[4 * q] + part[4 * q], dg[4 * q + 1] + part[4 * q + 1], dg[4 * q + 2] + part[4 * q + 2],
                               dg[4 * q + 3] + part[4 * q + 3]);
      }
      named_bar_sync(1, kWorkers);  // the staging is written by the next slice's first tile
    }
  }
  fence_before();
  __syncthreads();
  if (warp == 0) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(256));
  }
}

// Deterministic totals: fixed partition of the per-block values into 1024
// threads, fp64 partial sums, fixed tree.
__global__ void __launch_bounds__(1024) spectral_totals_kernel(const float* lfreq, const float* lrate, long long n,
                                                                double lambda_f, double lambda_r, double* totals) {
  __shared__ double sf[1024], sr[1024];
  double f = 0.0, r = 0.0;
  for (long long i = threadIdx.x; i < n; i += 1024) {
    f += (double)lfreq[i];
    r += (double)lrate[i];
  }
  sf[threadIdx.x] = f;
  sr[threadIdx.x] = r;
  __syncthreads();
  for (int s = 512; s > 0; s >>= 1) {
    if ((int)threadIdx.x < s) {
      sf[threadIdx.x] += sf[threadIdx.x + s];
      sr[threadIdx.x] += sr[threadIdx.x + s];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    totals[0] = sf[0];
    totals[1] = sr[0];
    totals[2] = (double)n;
    totals[3] = lambda_f * sf[0] / (double)n + lambda_r * sr[0] / (double)n;
  }
}

// dG[l][s][h] = sum over the batch, and over the pieces of each head slice, of
// the per-piece partials, in (batch, piece) order.
__global__ void spectral_dg_reduce_kernel(const float* part, float* dG, KvGeom k, int pieces) {
  const long long per = (long long)k.d * 16;
  const long long n = (long long)k.L * 2 * k.H * per;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
    const long long set = e / per, off = e % per;
    const long long h = set % k.H, ls = set / k.H;  // ls = l * 2 + s
    float acc = 0.0f;
    for (int b = 0; b < k.B; ++b)
      for (int q = 0; q < pieces; ++q) acc += part[(((ls * k.B + b) * k.H + h) * pieces + q) * per + off];
    dG[e] = acc;
  }
}

// Partials: one per work unit of the kernel that runs (head slices, or their
// pieces on the tensor-core path); sized for the larger of the two.
uint64_t spectral_workspace_bytes(const KvGeom& k, bool want_grad) {
  return want_grad ? (uint64_t)k.slices() * spectral_tmem_pieces(k) * k.d * 16 * sizeof(float) : 0;
}

cudaError_t launch_spectral(const KvGeom& k, int x_fp32, const void* x, const float* G, float lambda_f, float lambda_r,
                            float tau, float* lfreq, float* lrate, double* totals, float* dG, void* workspace,
                            unsigned int* status, int num_sms, cudaStream_t st) {
  SpecArgs a;
  a.k = k;
  a.x_fp32 = x_fp32;
  a.has_g = G != nullptr;
  a.want_grad = dG != nullptr;
  a.lambda_f = lambda_f;
  a.lambda_r = lambda_r;
  a.tau = tau;
  const double nblk = (double)k.slices() * (k.T / 16);
  a.inv_nblk = 1.0 / nblk;
  a.inv_ncoef = 1.0 / (nblk * 16.0 * kD);
  a.x = x;
  a.G = G;
  a.lfreq = lfreq;
  a.lrate = lrate;
  a.dg_part = reinterpret_cast<float*>(workspace);
  a.status = status;
  cudaError_t e;
  if (spectral_tmem_supported(k, x_fp32) || (x_fp32 && !dG && spectral_fwd_f32_supported(k))) {
    // the gauge folded into the channel DCT (fp32 input: statistics only, x split into bf16 hi + lo)
    e = launch_spectral_tmem(k, x_fp32, x, G, lambda_f, lambda_r, tau, lfreq, lrate, dG ? a.dg_part : nullptr, status,
                             num_sms, st);
  } else if (k.d == kD && k.T % kTile == 0) {
    e = cudaFuncSetAttribute(spectral_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSpecSmem);
    if (e != cudaSuccess) return e;
    const long long slices = k.slices();
    const int grid = (int)(slices < num_sms ? slices : num_sms);
    spectral_kernel<<<grid, kSpecThreads, kSpecSmem, st>>>(a);
    e = cudaGetLastError();
  } else {  // other head widths and token counts: the CUDA-core kernel
    e = launch_spectral_generic(k, x_fp32, x, G, lambda_f, lambda_r, tau, lfreq, lrate, dG ? a.dg_part : nullptr,
                                num_sms, st);
  }
  if (e != cudaSuccess) return e;
  spectral_totals_kernel<<<1, 1024, 0, st>>>(lfreq, lrate, (long long)nblk, lambda_f, lambda_r, totals);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (dG) {
    const int pieces = spectral_tmem_supported(k, x_fp32) ? spectral_tmem_pieces(k) : 1;
    spectral_dg_reduce_kernel<<<num_sms, 256, 0, st>>>(a.dg_part, dG, k, pieces);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace cg
