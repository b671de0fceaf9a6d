// Full-head gauge (g = d_head = 128): the gauge is a dense 128 x 128
// contraction per token, run on the 5th-generation tensor cores.
//
// Codec-Gauge, Method: full-head gauges (g = d_l) give the gauge the most
// freedom; explicit application costs O(N_KV g) multiply-adds (128 per value
// here), and recovery before attention is explicit.  Experimental setup:
// block-uniform backend; with g = d_head a range block is 16 tokens x d_head.
//
// Encode, per block of 128 tokens of one head slice:
//   * a TMA warp streams x blocks (128 x 128 bf16 = 32 KB, two 16 KB boxes with
//     128-byte swizzle, no multicast) into a 4-stage shared-memory ring, and
//     writes each head slice's G as bf16 (RNE) in the same swizzled K-major
//     layout (two buffers, so the next slice's G is staged while the current
//     one is in use);
//   * one thread issues 8 tcgen05.mma (M = N = 128, K = 16, bf16 x bf16 -> fp32)
//     into one of four 128-column TMEM accumulators: y[t][i] = sum_j x[t][j] G[i][j];
//   * three epilogue warpgroups take blocks in turn (one thread per token):
//     a first pass over the row's TMEM columns gives its range, half-warp
//     shuffles the 16-token block's; a second pass quantizes, packs and
//     stores the codes 32 at a time, as the grouped encoder defines them.
// Every wait on an mbarrier is bounded in time.
#include <cuda.h>

#include "cg_kernels.cuh"

namespace cg {

namespace {

constexpr int kXStages = 4;
constexpr int kBlockBytes = 128 * 128 * 2;  // 32 KB of bf16
// encoder: three epilogue warpgroups taking blocks in turn, four TMEM accumulators
constexpr int kEncGroups = 3;
constexpr int kEncEpi = 4 * kEncGroups;
constexpr int kThreads = (kEncEpi + 2) * 32;  // 12 epilogue, 1 TMA / G, 1 MMA
// tcgen05 instruction descriptor: D fp32, A and B bf16, both K-major, N = 128, M = 128
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

// Shared-memory matrix descriptor for a K-major tile in the 128-byte swizzled
// canonical layout (rows of 128 bytes, 8-row atoms 1024 bytes apart).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr & 0x3FFFFu) >> 4);  // start address
  d |= (uint64_t)1 << 16;                         // leading byte offset (unused for swizzled K-major): 16 B
  d |= (uint64_t)(1024 >> 4) << 32;               // stride byte offset: 1024 B between 8-row groups
  d |= (uint64_t)1 << 46;                         // descriptor version
  d |= (uint64_t)2 << 61;                         // layout: 128-byte swizzle
  return d;
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
          tmem_d),
      "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate));
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
      "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Byte offset of element (row, col) of a 128 x 128 bf16 K-major tile stored
// as two 64-column halves in the 128-byte swizzled layout.
__device__ __forceinline__ uint32_t sw128_offset(int row, int col) {
  const int half = col >> 6, c = (col & 63) >> 3;
  return half * 16384 + row * 128 + ((c ^ (row & 7)) << 4) + (col & 7) * 2;
}

struct FhSmem {
  unsigned char* xs;  // kXStages x 32 KB, 1024-aligned
  unsigned char* gs;  // 2 x 32 KB
  uint64_t* x_full;
  uint64_t* x_empty;
  uint64_t* g_full;
  uint64_t* g_empty;
  uint64_t* t_full;
  uint64_t* t_empty;
  uint32_t* tmem_base;
};

__device__ inline FhSmem fh_carve(unsigned char* raw) {
  FhSmem s;
  unsigned char* base = reinterpret_cast<unsigned char*>(((uintptr_t)raw + 1023) & ~(uintptr_t)1023);
  s.xs = base;
  s.gs = base + kXStages * kBlockBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(s.gs + 2 * kBlockBytes);
  s.x_full = bars;
  s.x_empty = bars + kXStages;
  s.g_full = bars + 2 * kXStages;
  s.g_empty = s.g_full + 2;
  s.t_full = s.g_empty + 2;
  s.t_empty = s.t_full + 4;
  s.tmem_base = reinterpret_cast<uint32_t*>(s.t_empty + 4);
  return s;
}
constexpr int kFhSmem = 1024 + (kXStages + 2) * kBlockBytes + (2 * kXStages + 12) * 8 + 16;

// The BITS words of 32 packed codes at p (4 * BITS bytes; p is aligned to 16 bytes for
// BITS = 4 and 8, to 8 for BITS = 2 and 6, to 4 for BITS = 3).
template <int BITS>
__device__ __forceinline__ void store_code_words(unsigned char* p, const uint32_t (&w)[BITS]) {
  if constexpr (BITS % 4 == 0) {
#pragma unroll
    for (int k = 0; k < BITS / 4; ++k)
      reinterpret_cast<uint4*>(p)[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
  } else if constexpr (BITS % 2 == 0) {
#pragma unroll
    for (int k = 0; k < BITS / 2; ++k) reinterpret_cast<uint2*>(p)[k] = make_uint2(w[2 * k], w[2 * k + 1]);
  } else {
#pragma unroll
    for (int k = 0; k < BITS; ++k) reinterpret_cast<uint32_t*>(p)[k] = w[k];
  }
}

}  // namespace

template <int BITS>
__global__ void __launch_bounds__(512, 1)  // 448 threads; the bound caps registers at 128 (4 warps per scheduler)
    fullhead_encode_kernel(const __grid_constant__ CUtensorMap tmap, CodecArgs a) {
  constexpr int D = 128;
  constexpr int QMAX = (1 << BITS) - 1;
  extern __shared__ unsigned char smem_raw[];
  const FhSmem sm = fh_carve(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bps = (a.nt + 127) / 128;  // 128-token blocks per head slice
  const long long total = (long long)bps * a.k.slices();
  const long long b0 = total * blockIdx.x / gridDim.x;
  const long long b1 = total * (blockIdx.x + 1) / gridDim.x;
  const int n_blocks = (int)(b1 - b0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kXStages; ++s) {
      mbar_init(&sm.x_full[s], 1);
      mbar_init(&sm.x_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.g_full[s], 1);
      mbar_init(&sm.g_empty[s], 1);
    }
    for (int s = 0; s < 4; ++s) {
      mbar_init(&sm.t_full[s], 1);
      mbar_init(&sm.t_empty[s], 4);  // the four warps of the warpgroup that took the block
    }
    fence_mbar_init();
  }
  if (warp == 0) {  // TMEM: four 128-column fp32 accumulators
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(sm.tmem_base)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_base;

  if (warp == kEncEpi) {
    // ---------------- TMA x blocks + G staging ----------------
    long long slice = b0 / bps;
    int bq = (int)(b0 - slice * bps);
    int gcount = 0;  // slices staged so far
    for (int i = 0; i < n_blocks; ++i) {
      if (i == 0 || bq == 0) {  // new head slice: stage its G (bf16, swizzled K-major, rows = outputs)
        const int gb = gcount & 1;
        mbar_wait(&sm.g_empty[gb], ((uint32_t)(gcount >> 1) & 1u) ^ 1u, a.status);
        int l, sk, b, h;
        slice_coords(slice, a.k, l, sk, b, h);
        const float4* Gp = reinterpret_cast<const float4*>(a.G + gauge_set(l, sk, h, a.k) * D * D);
        unsigned char* gdst = sm.gs + gb * kBlockBytes;
        for (int e = lane; e < D * D / 8; e += 32) {  // 8 consecutive elements of one row per step
          const float4 u = __ldg(Gp + 2 * e), v = __ldg(Gp + 2 * e + 1);
          const int row = (e * 8) / D, col = (e * 8) % D;
          uint4 w;
          w.x = pack_bf16x2(u.x, u.y);
          w.y = pack_bf16x2(u.z, u.w);
          w.z = pack_bf16x2(v.x, v.y);
          w.w = pack_bf16x2(v.z, v.w);
          *reinterpret_cast<uint4*>(gdst + sw128_offset(row, col)) = w;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.g_full[gb]);
        ++gcount;
      }
      if (lane == 0) {
        const int s = i % kXStages;
        mbar_wait(&sm.x_empty[s], ((uint32_t)(i / kXStages) & 1u) ^ 1u, a.status);
        mbar_arrive_expect_tx(&sm.x_full[s], kBlockBytes);
        const int row0 = (int)(slice * a.k.T + a.t0 + 128LL * bq);
        tma_load_2d(sm.xs + s * kBlockBytes, &tmap, 0, row0, &sm.x_full[s]);
        tma_load_2d(sm.xs + s * kBlockBytes + 16384, &tmap, 64, row0, &sm.x_full[s]);
      }
      __syncwarp();
      if (++bq == bps) {
        bq = 0;
        ++slice;
      }
    }
  } else if (warp == kEncEpi + 1) {
    // ---------------- MMA issue (one thread) ----------------
    if (lane == 0) {
      long long slice = b0 / bps;
      int bq = (int)(b0 - slice * bps);
      int gcount = 0;
      for (int i = 0; i < n_blocks; ++i) {
        const int gb = gcount & 1;
        if (i == 0 || bq == 0) mbar_wait(&sm.g_full[gb], (uint32_t)(gcount >> 1) & 1u, a.status);
        const int s = i % kXStages, acc = i & 3;
        mbar_wait(&sm.x_full[s], (uint32_t)(i / kXStages) & 1u, a.status);
        mbar_wait(&sm.t_empty[acc], ((uint32_t)(i >> 2) & 1u) ^ 1u, a.status);
        tc_fence_after();
        const uint32_t xa = smem_u32(sm.xs + s * kBlockBytes), ga = smem_u32(sm.gs + gb * kBlockBytes);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t koff = (k >> 2) * 16384 + (k & 3) * 32;
          umma_bf16(tmem + acc * 128, sw128_desc(xa + koff), sw128_desc(ga + koff), k > 0 ? 1u : 0u);
        }
        umma_commit(&sm.x_empty[s]);
        umma_commit(&sm.t_full[acc]);
        const bool last_of_slice = (bq + 1 == bps) || (i + 1 == n_blocks);
        if (last_of_slice) {
          umma_commit(&sm.g_empty[gb]);
          ++gcount;
        }
        if (++bq == bps) {
          bq = 0;
          ++slice;
        }
      }
    }
  } else {
    // ---------------- epilogue: warpgroup wg takes blocks i with i % 3 == wg; thread = token row ----------------
    const int wg = warp >> 2, quarter = warp & 3;
    const int row = 32 * quarter + lane;
    const double inv_qmax = 1.0 / (double)QMAX;
    const long long slice_code_bytes = (long long)a.k.T * D * BITS / 8;
    long long slice = b0 / bps;
    int bq = (int)(b0 - slice * bps);
    for (int i = 0; i < n_blocks; ++i) {
      if (i % kEncGroups == wg) {
        const int acc = i & 3;
        mbar_wait(&sm.t_full[acc], (uint32_t)(i >> 2) & 1u, a.status);
        tc_fence_after();
        const uint32_t taddr = tmem + acc * 128 + ((uint32_t)(32 * quarter) << 16);
        const int valid = min(128, a.nt - 128 * bq);
        const int tok = a.t0 + 128 * bq + row;
        // Two 32-column accumulator loads are kept in flight in both passes: the next one is
        // issued before the current one is used (the empty asm statements pin each load's
        // registers after its wait).
        float va[32], vb[32];
        auto pin = [](float (&v)[32]) {
#pragma unroll
          for (int k = 0; k < 32; ++k) asm volatile("" : "+f"(v[k]));
        };
        // pass 1: the row's range, then the 16-token block's (16 lanes)
        float mn = __int_as_float(0x7f800000), mx = __int_as_float(0xff800000);
        auto range32 = [&](const float (&v)[32]) {
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            mn = min3f(mn, v[j], v[j + 1]);
            mx = max3f(mx, v[j], v[j + 1]);
          }
        };
        tmem_ld32(taddr, va);
        tmem_wait_ld();
        pin(va);
        tmem_ld32(taddr + 32, vb);
        range32(va);
        tmem_wait_ld();
        pin(vb);
        tmem_ld32(taddr + 64, va);
        range32(vb);
        tmem_wait_ld();
        pin(va);
        tmem_ld32(taddr + 96, vb);
        range32(va);
        tmem_wait_ld();
        pin(vb);
        range32(vb);
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) {
          mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        const QParams qp = quant_params(mn, mx, inv_qmax);
        // t is monotone in y: no clamp is needed when the block's extremes round into [0, qmax]
        const float t_lo = __fmul_rn(__fsub_rn(mn, qp.zf), qp.inv), t_hi = __fmul_rn(__fsub_rn(mx, qp.zf), qp.inv);
        const bool clampit = !(t_lo >= -0.5f && t_hi < (float)QMAX + 0.5f);
        const f2_t nz2 = f2_make(-qp.zf, -qp.zf), iv2 = f2_make(qp.inv, qp.inv), mg2 = f2_make(12582912.0f, 12582912.0f);
        // pass 2: codes of the row, 32 at a time (BITS packed words each, little-endian),
        // stored as they are made: the row's codes are bytes [r16 * 16 * BITS, +16 * BITS)
        // of its 16-token block's record
        const int tile = tok / 16, r16 = tok % 16;
        unsigned char* dst = a.codes + slice * slice_code_bytes + (long long)tile * (16 * D * BITS / 8) +
                             r16 * (D * BITS / 8);
        auto quant32 = [&](const float (&v)[32], int c) {
          if (a.gauged && row < valid) {
            float4* gd = reinterpret_cast<float4*>(a.gauged + (slice * a.k.T + tok) * D + 32 * c);
#pragma unroll
            for (int j = 0; j < 8; ++j) gd[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
          }
          uint32_t words[BITS];
#pragma unroll
          for (int w = 0; w < BITS; ++w) words[w] = 0;
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            // q = clamp(rne(fl(fl(y - z) * inv)), 0, qmax): clamped where needed, then rounded
            // (RNE) by adding 1.5 * 2^23, which leaves the integer in the low mantissa bits
            float t0, t1;
            f2_split(f2_mul(f2_add(f2_make(v[j], v[j + 1]), nz2), iv2), t0, t1);
            if (clampit) {
              t0 = fminf(fmaxf(t0, 0.0f), (float)QMAX);
              t1 = fminf(fmaxf(t1, 0.0f), (float)QMAX);
            }
            float r0, r1;
            f2_split(f2_add(f2_make(t0, t1), mg2), r0, r1);
            const uint32_t q[2] = {__float_as_uint(r0) & (uint32_t)QMAX, __float_as_uint(r1) & (uint32_t)QMAX};
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int bit = (j + e) * BITS;
              words[bit >> 5] |= q[e] << (bit & 31);
              if ((bit & 31) + BITS > 32) words[(bit >> 5) + 1] |= q[e] >> (32 - (bit & 31));
            }
          }
          if (row < valid) store_code_words<BITS>(dst + c * 4 * BITS, words);
        };
        tmem_ld32(taddr, va);
        tmem_wait_ld();
        pin(va);
        tmem_ld32(taddr + 32, vb);
        quant32(va, 0);
        tmem_wait_ld();
        pin(vb);
        tmem_ld32(taddr + 64, va);
        quant32(vb, 1);
        tmem_wait_ld();
        pin(va);
        tmem_ld32(taddr + 96, vb);
        quant32(va, 2);
        tmem_wait_ld();
        pin(vb);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.t_empty[acc]);  // the accumulator is in registers
        quant32(vb, 3);
        if (row < valid && (lane & 15) == 0) {
          const long long bidx = slice * (a.k.T / 16) + tile;
          a.scales[bidx] = qp.sh;
          a.zeros[bidx] = qp.zh;
        }
      }
      if (++bq == bps) {
        bq = 0;
        ++slice;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

// Decode, per block of 128 tokens: x_hat_t = G^T (s q_t + z) = s (G^T q_t) + z (G^T 1)
// (the range block of 16 tokens x d_head has one s and z).  Two warpgroups take
// alternate blocks, each with its own A buffer and accumulator: a warpgroup
// expands its block's codes into the A operand (exact bf16 integers, swizzled
// K-major rows in shared memory), the tensor cores contract it with
// B = G^T (bf16, swizzled K-major, column sums of the same bf16 values kept
// beside it), and the same warps then read the accumulator and write bf16,
// while the other warpgroup works on the next block.  A warpgroup's loads of
// its next block's codes are issued as soon as the current block's are
// expanded, so they are in flight during its epilogue.
namespace {
constexpr int kDecEpi = 8;  // two warpgroups taking alternate blocks: code expansion, then epilogue
constexpr int kDecThreads = (kDecEpi + 2) * 32;
constexpr int kStgPitch = 256 + 16, kStgWarp = 32 * kStgPitch;
struct FdSmem {
  unsigned char* as;  // 2 x 32 KB A tiles
  unsigned char* gs;  // 2 x 32 KB G^T tiles
  float* colsum;      // 2 x 128
  unsigned char* stg; // per epilogue warp: 32 output rows of 256 B (+16 B pad) for coalesced stores
  uint64_t* a_full;
  uint64_t* a_empty;
  uint64_t* g_full;
  uint64_t* g_empty;
  uint64_t* t_full;
  uint64_t* t_empty;
  uint32_t* tmem_base;
};
__device__ inline FdSmem fd_carve(unsigned char* raw) {
  FdSmem s;
  unsigned char* base = reinterpret_cast<unsigned char*>(((uintptr_t)raw + 1023) & ~(uintptr_t)1023);
  s.as = base;
  s.gs = base + 2 * kBlockBytes;
  s.colsum = reinterpret_cast<float*>(base + 4 * kBlockBytes);
  s.stg = reinterpret_cast<unsigned char*>(s.colsum + 256);
  uint64_t* bars = reinterpret_cast<uint64_t*>(s.stg + kDecEpi * kStgWarp);
  s.a_full = bars;
  s.a_empty = bars + 2;
  s.g_full = bars + 4;
  s.g_empty = bars + 6;
  s.t_full = bars + 8;
  s.t_empty = bars + 10;
  s.tmem_base = reinterpret_cast<uint32_t*>(bars + 12);
  return s;
}
constexpr int kFdSmem = 1024 + 4 * kBlockBytes + 256 * 4 + kDecEpi * kStgWarp + 12 * 8 + 16;

// bf16 pair of the 4-bit codes at bits 0 and 16 of v: 128 + q is exact in bf16
// (0x4300 | q), and subtracting 128 leaves q.
__device__ __forceinline__ uint32_t bf16_nib_pair(uint32_t v) {
  uint32_t r;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"((v & 0x000F000Fu) | 0x43004300u), "r"(0x43004300u));
  return r;
}
// bf16 bits of two codes (< 256, exact), packed low / high
__device__ __forceinline__ uint32_t code_pair_bf16(uint32_t q0, uint32_t q1) {
  const f2_t v = f2_add(f2_make(__uint_as_float(0x4B000000u | q0), __uint_as_float(0x4B000000u | q1)),
                        f2_make(-8388608.0f, -8388608.0f));
  float lo, hi;
  f2_split(v, lo, hi);
  return __byte_perm(__float_as_uint(lo), __float_as_uint(hi), 0x7632);
}
}  // namespace

template <int BITS>
__global__ void __launch_bounds__(kDecThreads, 1) fullhead_decode_kernel(CodecArgs a) {
  constexpr int D = 128;
  constexpr uint32_t M = (1u << BITS) - 1u;
  extern __shared__ unsigned char smem_raw[];
  const FdSmem sm = fd_carve(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bps = (a.nt + 127) / 128;
  const long long total = (long long)bps * a.k.slices();
  const long long b0 = total * blockIdx.x / gridDim.x;
  const long long b1 = total * (blockIdx.x + 1) / gridDim.x;
  const int n_blocks = (int)(b1 - b0);
  const long long slice_code_bytes = (long long)a.k.T * D * BITS / 8;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.a_full[s], 4);  // the warpgroup that takes the block
      mbar_init(&sm.a_empty[s], 1);
      mbar_init(&sm.g_full[s], 1);
      // released by the tensor cores (done reading G^T) and by the epilogue
      // warps (done reading the column sums)
      mbar_init(&sm.g_empty[s], 1 + kDecEpi);
      mbar_init(&sm.t_full[s], 1);
      mbar_init(&sm.t_empty[s], 4);
    }
    fence_mbar_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(sm.tmem_base)),
                 "r"(256));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_base;

  if (warp == kDecEpi) {
    // ---------------- G^T staging (bf16, swizzled, rows = outputs n) and column sums ----------------
    long long slice = b0 / bps;
    int bq = (int)(b0 - slice * bps);
    int gcount = 0;
    for (int i = 0; i < n_blocks; ++i) {
      if (i == 0 || bq == 0) {
        const int gb = gcount & 1;
        mbar_wait(&sm.g_empty[gb], ((uint32_t)(gcount >> 1) & 1u) ^ 1u, a.status);
        int l, sk, b, h;
        slice_coords(slice, a.k, l, sk, b, h);
        const float* Gp = a.G + gauge_set(l, sk, h, a.k) * D * D;  // G[k][n]
        unsigned char* gdst = sm.gs + gb * kBlockBytes;
        // lane owns output columns n = lane, lane+32, ...: row n of B = column n of G.  With
        // 4-bit codes the k slots of every 8-channel chunk hold channels 0, 4, 1, 5, 2, 6, 3, 7
        // (the order in which the code expansion produces them); the column sums run in
        // channel order either way.
        for (int n = lane; n < D; n += 32) {
          float cs = 0.0f;
          for (int k0 = 0; k0 < D; k0 += 8) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float g0 = __ldg(Gp + (k0 + 2 * e) * D + n), g1 = __ldg(Gp + (k0 + 2 * e + 1) * D + n);
              w[e] = pack_bf16x2(g0, g1);
              cs += __uint_as_float(w[e] << 16) + __uint_as_float(w[e] & 0xffff0000u);
            }
            if constexpr (BITS == 4) {  // pairs (0, 4), (1, 5), (2, 6), (3, 7) of the chunk
              const uint32_t p0 = __byte_perm(w[0], w[2], 0x5410), p1 = __byte_perm(w[0], w[2], 0x7632);
              const uint32_t p2 = __byte_perm(w[1], w[3], 0x5410), p3 = __byte_perm(w[1], w[3], 0x7632);
              *reinterpret_cast<uint4*>(gdst + sw128_offset(n, k0)) = make_uint4(p0, p1, p2, p3);
            } else {
              *reinterpret_cast<uint4*>(gdst + sw128_offset(n, k0)) = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
          sm.colsum[gb * 128 + n] = cs;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.g_full[gb]);
        ++gcount;
      }
      if (++bq == bps) {
        bq = 0;
        ++slice;
      }
    }
  } else if (warp == kDecEpi + 1) {
    // ---------------- MMA issue ----------------
    if (lane == 0) {
      long long slice = b0 / bps;
      int bq = (int)(b0 - slice * bps);
      int gcount = 0;
      for (int i = 0; i < n_blocks; ++i) {
        const int gb = gcount & 1, ab = i & 1;
        if (i == 0 || bq == 0) mbar_wait(&sm.g_full[gb], (uint32_t)(gcount >> 1) & 1u, a.status);
        mbar_wait(&sm.a_full[ab], (uint32_t)(i >> 1) & 1u, a.status);
        mbar_wait(&sm.t_empty[ab], ((uint32_t)(i >> 1) & 1u) ^ 1u, a.status);
        tc_fence_after();
        const uint32_t aa = smem_u32(sm.as + ab * kBlockBytes), ga = smem_u32(sm.gs + gb * kBlockBytes);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t koff = (k >> 2) * 16384 + (k & 3) * 32;
          umma_bf16(tmem + ab * 128, sw128_desc(aa + koff), sw128_desc(ga + koff), k > 0 ? 1u : 0u);
        }
        umma_commit(&sm.a_empty[ab]);
        umma_commit(&sm.t_full[ab]);
        if ((bq + 1 == bps) || (i + 1 == n_blocks)) {
          umma_commit(&sm.g_empty[gb]);
          ++gcount;
        }
        if (++bq == bps) {
          bq = 0;
          ++slice;
        }
      }
    }
  } else {
    // ---------------- warpgroup wg takes blocks i = wg, wg + 2, ...: code expansion, then epilogue;
    // thread = token row (the other warpgroup's work covers this block's MMA) ----------------
    const int wg = warp >> 2, quarter = warp & 3;
    const int row = 32 * quarter + lane;
    // this thread's codes of block (sl, q): its token row's 16 BITS bytes (rows past
    // the range repeat a valid row)
    auto load_codes = [&](long long sl, int q, uint4 (&dst)[BITS]) {
      const int valid = min(128, a.nt - 128 * q);
      const int tok = a.t0 + 128 * q + min(row, valid - 1);
      const uint4* src = reinterpret_cast<const uint4*>(a.codes_in + sl * slice_code_bytes +
                                                        (long long)(tok / 16) * (16 * D * BITS / 8) +
                                                        (tok % 16) * (D * BITS / 8));
#pragma unroll
      for (int w = 0; w < BITS; ++w) dst[w] = __ldg(src + w);
    };
    long long slice = b0 / bps;
    int bq = (int)(b0 - slice * bps);
    int gcount = 0;
    uint4 next[BITS];  // codes of this warpgroup's next block, loading while it finishes the current one
    if (wg < n_blocks) {
      long long sl = slice;
      int q = bq + wg;
      if (q >= bps) {
        q -= bps;
        ++sl;
      }
      load_codes(sl, q, next);
    }
    for (int i = 0; i < n_blocks; ++i) {
      const int gb = gcount & 1;
      const bool last_of_slice = (bq + 1 == bps) || (i + 1 == n_blocks);
      if ((i & 1) == wg) {
        const int ab = i & 1;  // == wg: each warpgroup has its own A buffer and accumulator
        const int valid = min(128, a.nt - 128 * bq);
        {  // codes of the block -> exact bf16 integers, swizzled K-major A operand
          uint32_t words[4 * BITS + 1];
#pragma unroll
          for (int w = 0; w < BITS; ++w) {
            const uint4 v = next[w];
            words[4 * w] = v.x; words[4 * w + 1] = v.y; words[4 * w + 2] = v.z; words[4 * w + 3] = v.w;
          }
          words[4 * BITS] = 0;
          if (i + 2 < n_blocks) {  // block i + 2 is this warpgroup's next
            long long sl = slice;
            int q = bq + 2;
            while (q >= bps) {  // at most twice
              q -= bps;
              ++sl;
            }
            load_codes(sl, q, next);
          }
          mbar_wait(&sm.a_empty[ab], ((uint32_t)(i >> 1) & 1u) ^ 1u, a.status);
          unsigned char* adst = sm.as + ab * kBlockBytes;
#pragma unroll
          for (int c = 0; c < 16; ++c) {  // 16-byte chunk c = channels 8c .. 8c+7
            uint4 w;
            if constexpr (BITS == 4) {
              // word c holds the chunk's 8 codes; the nibbles at bits 0 and 16 of w >> 4 e are
              // channels e and e + 4: 128 + q as bf16 by one mask, minus 128 exactly
              const uint32_t v = words[c];
              w = make_uint4(bf16_nib_pair(v), bf16_nib_pair(v >> 4), bf16_nib_pair(v >> 8), bf16_nib_pair(v >> 12));
            } else {
              uint32_t q[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const int bit = (8 * c + e) * BITS;
                q[e] = __funnelshift_r(words[bit >> 5], words[(bit >> 5) + 1], bit & 31) & M;
              }
              w = make_uint4(code_pair_bf16(q[0], q[1]), code_pair_bf16(q[2], q[3]), code_pair_bf16(q[4], q[5]),
                             code_pair_bf16(q[6], q[7]));
            }
            *reinterpret_cast<uint4*>(adst + sw128_offset(row, 8 * c)) = w;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.a_full[ab]);
        }
        const int tok = a.t0 + 128 * bq + row;
        float sf = 0.0f, zf = 0.0f;
        if (row < valid) {
          const long long bidx = slice * (a.k.T / 16) + tok / 16;
          sf = __half2float(__ushort_as_half(__ldg(a.scales_in + bidx)));
          zf = __half2float(__ushort_as_half(__ldg(a.zeros_in + bidx)));
        }
        mbar_wait(&sm.t_full[ab], (uint32_t)(i >> 1) & 1u, a.status);
        tc_fence_after();
        const uint32_t taddr = tmem + ab * 128 + ((uint32_t)(32 * quarter) << 16);
        const float* cs = sm.colsum + gb * 128;
        unsigned char* stg = sm.stg + warp * kStgWarp;
        // 32 accumulator columns c4 -> 64 bytes of this thread's staged row
        auto emit = [&](const float (&v)[32], int c4) {
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            uint4 o;
            o.x = pack_bf16x2(__fmaf_rn(sf, v[j + 0], zf * cs[32 * c4 + j + 0]), __fmaf_rn(sf, v[j + 1], zf * cs[32 * c4 + j + 1]));
            o.y = pack_bf16x2(__fmaf_rn(sf, v[j + 2], zf * cs[32 * c4 + j + 2]), __fmaf_rn(sf, v[j + 3], zf * cs[32 * c4 + j + 3]));
            o.z = pack_bf16x2(__fmaf_rn(sf, v[j + 4], zf * cs[32 * c4 + j + 4]), __fmaf_rn(sf, v[j + 5], zf * cs[32 * c4 + j + 5]));
            o.w = pack_bf16x2(__fmaf_rn(sf, v[j + 6], zf * cs[32 * c4 + j + 6]), __fmaf_rn(sf, v[j + 7], zf * cs[32 * c4 + j + 7]));
            *reinterpret_cast<uint4*>(stg + lane * kStgPitch + 2 * (32 * c4 + j)) = o;
          }
        };
        // two 32-column loads in flight: the next one is issued before the current one is used
        // (the empty asm statements pin each load's registers after its wait)
        float va[32], vb[32];
        tmem_ld32(taddr, va);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) asm volatile("" : "+f"(va[k]));
        tmem_ld32(taddr + 32, vb);
        emit(va, 0);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) asm volatile("" : "+f"(vb[k]));
        tmem_ld32(taddr + 64, va);
        emit(vb, 1);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) asm volatile("" : "+f"(va[k]));
        tmem_ld32(taddr + 96, vb);
        emit(va, 2);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) asm volatile("" : "+f"(vb[k]));
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.t_empty[ab]);  // the accumulator is in registers
        emit(vb, 3);
        __syncwarp();
        // the warp's 32 rows leave as whole 256-byte lines: two rows per instruction
        const int tok0 = a.t0 + 128 * bq + 32 * quarter;
        uint4* dst0 = reinterpret_cast<uint4*>(a.kv_out + (slice * a.k.T + tok0) * (long long)D);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const int r = 2 * k + (lane >> 4), ch = lane & 15;
          if (32 * quarter + r < valid)
            dst0[r * (D / 8) + ch] = *reinterpret_cast<const uint4*>(stg + r * kStgPitch + 16 * ch);
        }
        __syncwarp();  // the staging rows are rewritten by this warp's next block
      }
      if (last_of_slice) {  // every epilogue warp is past this slice: its G^T and column sums may go
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.g_empty[gb]);
        ++gcount;
      }
      if (++bq == bps) {
        bq = 0;
        ++slice;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(256));
  }
}

namespace {
template <int BITS>
cudaError_t fh_dec_launch(const CodecArgs& a, int num_sms, cudaStream_t st) {
  auto kern = fullhead_decode_kernel<BITS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kFdSmem);
  if (e != cudaSuccess) return e;
  const long long total = (long long)((a.nt + 127) / 128) * a.k.slices();
  const int grid = (int)(total < num_sms ? total : num_sms);
  kern<<<grid, kDecThreads, kFdSmem, st>>>(a);
  return cudaGetLastError();
}
}  // namespace

namespace {
template <int BITS>
cudaError_t fh_enc_launch(const CodecArgs& a, int num_sms, cudaStream_t st) {
  alignas(64) CUtensorMap tmap;
  const uint64_t rows = (uint64_t)a.k.slices() * a.k.T;
  if (!make_tmap_2d_bf16(&tmap, a.kv, rows, 128, 64, 128)) return cudaErrorInvalidValue;
  auto kern = fullhead_encode_kernel<BITS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kFhSmem);
  if (e != cudaSuccess) return e;
  const long long total = (long long)((a.nt + 127) / 128) * a.k.slices();
  const int grid = (int)(total < num_sms ? total : num_sms);
  kern<<<grid, kThreads, kFhSmem, st>>>(tmap, a);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_fullhead(const CodecArgs& a, bool encode, int num_sms, cudaStream_t st) {
  if (a.nt == 0) return cudaSuccess;
  if (a.k.d != 128 || a.W != 128) return cudaErrorInvalidValue;
  switch (a.bits) {
    case 2: return encode ? fh_enc_launch<2>(a, num_sms, st) : fh_dec_launch<2>(a, num_sms, st);
    case 3: return encode ? fh_enc_launch<3>(a, num_sms, st) : fh_dec_launch<3>(a, num_sms, st);
    case 4: return encode ? fh_enc_launch<4>(a, num_sms, st) : fh_dec_launch<4>(a, num_sms, st);
    case 6: return encode ? fh_enc_launch<6>(a, num_sms, st) : fh_dec_launch<6>(a, num_sms, st);
    case 8: return encode ? fh_enc_launch<8>(a, num_sms, st) : fh_dec_launch<8>(a, num_sms, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace cg
