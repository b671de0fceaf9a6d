// Device helpers shared by the libcg kernels (sm_100a).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/cg.h"

namespace cg {

// ---- device status word ------------------------------------------------------
// A kernel whose bounded wait runs out ORs kStatusTimeout into the status word
// (defined once in cg_abi.cu; kernels receive its device address).
// cg_sync_status() reads and clears it.
constexpr unsigned int kStatusTimeout = 1u;
// The chain-exact tensor-core encoder ORs kStatusBound when a value it re-evaluated with the
// fp32 chain lay farther from its tensor-core value than the error bound its decisions assume.
constexpr unsigned int kStatusBound = 2u;
// Wall-time bound of any device-side wait on an asynchronous copy.
constexpr unsigned long long kWaitNs = 2000000000ull;

// ---- problem geometry shared by host and device -------------------------------
struct KvGeom {
  int L, B, H, T, d;
  // number of (l, s, b, h) head slices
  __host__ __device__ long long slices() const { return (long long)L * 2 * B * H; }
};

__host__ __device__ inline void slice_coords(long long slice, const KvGeom& k, int& l, int& s, int& b, int& h) {
  h = (int)(slice % k.H);
  long long r = slice / k.H;
  b = (int)(r % k.B);
  r /= k.B;
  s = (int)(r % 2);
  l = (int)(r / 2);
}

// Index of the gauge matrix set (l, s, h) in a [L][2][H][R][g][g] array.
__host__ __device__ inline long long gauge_set(int l, int s, int h, const KvGeom& k) {
  return ((long long)l * 2 + s) * k.H + h;
}

// ---- bf16 / fp32 bit helpers -----------------------------------------------------
// Low and high bf16 of a packed pair as fp32 (exact: bf16 is the top half of fp32).
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// fp32 -> bf16 pair with round-to-nearest-even (cvt.rn.bf16x2.f32).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// ---- packed fp32 pairs (sm_100 f32x2 arithmetic) -----------------------------------
typedef unsigned long long f2_t;
__device__ __forceinline__ f2_t f2_make(float lo, float hi) {
  f2_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_split(f2_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
// d = a * b + c, two independent IEEE fp32 fused multiply-adds (RN).
__device__ __forceinline__ f2_t f2_fma(f2_t a, f2_t b, f2_t c) {
  f2_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ f2_t f2_add(f2_t a, f2_t b) {
  f2_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f2_t f2_mul(f2_t a, f2_t b) {
  f2_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// ---- warp reductions -------------------------------------------------------------
__device__ __forceinline__ float warp_min_f32(float v) {
  float r;
  asm volatile("redux.sync.min.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}
__device__ __forceinline__ float warp_max_f32(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// ---- the quantizer's block parameters -------------------------------------------------
// z = fp16_rne(clamp(mn)), s = fp16_rne(min(fl32(fl32(mx - mn) / qmax), 65504)),
// with a zero minimum or maximum taken as +0.
// The division by the integer qmax = 2^b - 1 is evaluated as the fp64 product
// r * fl64(1/qmax) rounded to fp32, which equals the correctly rounded fp32
// quotient Q = r / qmax: (i) Q is never an fp32 rounding midpoint, because a
// midpoint has a 25-bit odd significand and odd * qmax would then need more
// than the 24 bits r has; (ii) Q is at least 2^-26 / qmax (relative) away from
// every midpoint, while the fp64 product is within 2^-52 of Q.  So both round
// to the same fp32 value.  inv = fl32(1 / s), the correctly rounded reciprocal.
// 3-input fp32 min / max
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

struct QParams {
  float zf;      // fp16 zero point as fp32
  float sf;      // fp16 step as fp32
  float inv;     // fl32(1 / sf), 0 when sf == 0
  uint16_t zh, sh;
};

__device__ __forceinline__ QParams quant_params(float mn, float mx, double inv_qmax) {
  QParams p;
  mn = __fadd_rn(mn, 0.0f);  // a zero extreme is +0 (-0 + +0 = +0)
  mx = __fadd_rn(mx, 0.0f);
  float zc = fminf(fmaxf(mn, -65504.0f), 65504.0f);
  __half z = __float2half_rn(zc);
  float rng = __fsub_rn(mx, mn);
  float s32 = __double2float_rn(__dmul_rn((double)rng, inv_qmax));
  __half s = __float2half_rn(fminf(s32, 65504.0f));
  p.zf = __half2float(z);
  p.sf = __half2float(s);
  p.inv = (p.sf != 0.0f) ? __frcp_rn(p.sf) : 0.0f;
  p.zh = __half_as_ushort(z);
  p.sh = __half_as_ushort(s);
  return p;
}

// q = clamp(rne(fl32(fl32(y - z) * inv)), 0, qmax); inv == 0 gives 0.
__device__ __forceinline__ uint32_t quantize_one(float y, float zf, float inv, int qmax) {
  float t = __fmul_rn(__fsub_rn(y, zf), inv);
  int q = __float2int_rn(t);  // RNE, saturating
  q = max(q, 0);
  q = min(q, qmax);
  return (uint32_t)q;
}

// ---- bounded mbarrier / bulk-copy helpers ------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Wait for phase `parity` of `bar` to complete.  Gives up after kWaitNs of
// wall time, ORs kStatusTimeout into *status and returns false (the caller
// carries on, so every thread still reaches every barrier and the kernel ends).
__device__ __forceinline__ uint32_t mbar_try_wait(uint32_t addr, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(done)
      : "r"(addr), "r"(parity)
      : "memory");
  return done;
}
// (The first test needs no clock: the common case is a phase already complete.)
// `limit_ns` is the wall-time bound (kWaitNs unless a caller asks for less).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned int* status,
                                          unsigned long long limit_ns = kWaitNs) {
  const uint32_t addr = smem_u32(bar);
  if (mbar_try_wait(addr, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(addr, parity)) return true;
    if ((i & 255u) == 0 && global_ns() - t0 > limit_ns) {
      atomicOr(status, kStatusTimeout);
      return false;
    }
  }
}
// 1-D bulk copy global -> shared, completion counted on `bar` (bytes % 16 == 0,
// both addresses 16-byte aligned).
__device__ __forceinline__ void bulk_g2s(void* smem_dst, const void* gmem_src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// 1-D bulk copy shared -> global (bulk-group completion).
__device__ __forceinline__ void bulk_s2g(void* gmem_dst, const void* smem_src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gmem_dst), "r"(smem_u32(smem_src)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N bulk groups are still reading their shared source.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// 2-D tiled TMA load (no multicast) of box {x, y} into shared memory.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const void* tmap, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cta.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(smem_dst)),
      "l"(tmap), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
// Warp-level m16n8k16 MMA, bf16 operands, fp32 accumulators, and ldmatrix.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// d = a b (no accumulator input: C is a zero register, d is written only, so no
// zeroing of d is needed before the first product of a chain)
__device__ __forceinline__ void mma_bf16_16816_z(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
}
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
// Warp-level m16n8k16 MMA, fp16 operands, fp32 accumulators (d = a b, or d += a b).
__device__ __forceinline__ void mma_f16_16816_z(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
}
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// fp16 pair {c_lo, c_hi} of two codes < 256: the fp16 patterns 0x6400 | c are
// exactly 1024 + c, and one exact f16x2 subtraction removes the 1024.
__device__ __forceinline__ uint32_t f16_sub1024(uint32_t biased) {
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(biased), "r"(0x64006400u));
  return r;
}
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

}  // namespace cg
