// Block-ALS contractions on the 5th-generation tensor cores (tcgen05, sm_100a).
//
//   P  = R (W V)   : M = rows of R,    N = 64 components, K = columns of R
//   Q^T = R^T U    : M = columns of R, N = 64 components, K = rows of R
//
// The ternary operand (V or U, entries -1/0/+1) is exact in bf16.  The fp32
// residual (times w_j for P when weighted, one fp32 rounding) is split exactly
// into three bf16 parts hi + mid + lo (8 + 8 + 8 significand bits), so every
// product the tensor core forms is exact and only its fp32 accumulation rounds
// -- the same class of error as an fp32 dot product on the CUDA cores.
//
// Two kernels compute these contractions; tc_contract_rv / tc_contract_rtu
// choose between them.
//
// contract_tma_kernel (the usual path: rows of R 16-byte aligned, i.e.
// n % 4 == 0): persistent, one CTA per SM, stream-K over units of (128-row
// tile, 32-wide K chunk).  A producer thread copies fp32 chunks of R with TMA
// (and the ternary B chunks with bulk copies) into an 8-deep shared-memory
// ring; converter warps split each chunk into its bf16 parts straight into
// tensor memory; one thread issues the MMAs into one of two alternating
// 128 x 64 fp32 accumulators in tensor memory; epilogue warps read a finished
// accumulator out (tcgen05.ld) into the tile's stream-K partials
// Xp[(t S + slot) 128 + row][64] while the next segment streams.
//
// contract_kernel (the other case: n % 4 != 0, or EXTERND_CONTRACT_NO_TMA=1):
// one CTA per (128-row tile, K split); every thread loads and converts a
// chunk into the canonical no-swizzle UMMA layouts in shared memory, double
// buffered, while one thread issues the previous chunk's 3 x 2 MMAs (3 parts
// x K/16 steps); tcgen05.commit on a per-stage mbarrier tells when a stage
// may be refilled.  Outputs are split-K partials Xp[split][row][64].
//
// In both, every mbarrier wait is bounded; a wait that runs out records
// EXTERND_ERR_TIMEOUT, the CTA stops issuing, waits (bounded) for its own
// copies and MMAs in flight and frees its tensor memory.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdint>
#include <cstdlib>

#include "common.cuh"
#include "internal.h"
#include "umma_layout.cuh"

namespace externd {
namespace umma {

typedef unsigned long long u64;

constexpr int kThreads = 256;
constexpr int kPartBytes = kM * kKc * 2;   // one bf16 part of the A chunk: 8 KB
constexpr int kLboMN = kM / 8 * 128;       // MN-major: bytes between 8-k groups
constexpr int kStageBytes = 3 * kPartBytes + kBBytes;
constexpr int kSmemBytes = 2 * kStageBytes + 1024;  // 56 KB + alignment slack: 3-4 CTAs per SM
constexpr long long kWaitBudget = 2000000000LL;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// --- tcgen05 / mbarrier wrappers (PTX ISA, sm_100a) ---
__device__ __forceinline__ void tmem_alloc(uint32_t dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_init(uint32_t addr, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(addr), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ bool mbar_test(uint32_t addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(addr), "r"(parity)
      : "memory");
  return ok != 0u;
}
// bounded wait for completion of the phase with the given parity
__device__ __forceinline__ bool mbar_wait(uint32_t addr, uint32_t parity) {
  if (mbar_test(addr, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_test(addr, parity))
    if (clock64() - t0 > kWaitBudget) return false;
  return true;
}
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint32_t mbar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
      : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor, no swizzle: start address, leading-dimension
// byte offset (LBO), stride-dimension byte offset (SBO), version 1.
__device__ __forceinline__ uint64_t make_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3fffu);
  d |= (uint64_t)((lbo >> 4) & 0x3fffu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3fffu) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version for sm_100
  return d;                // base offset 0, legacy LBO mode, layout type 0 (no swizzle)
}

// Instruction descriptor, kind::f16: fp32 accumulate, bf16 A and B, M x N.
__host__ __device__ constexpr uint32_t make_idesc(int a_mn_major) {
  return (1u << 4)                      // D format: f32
         | (1u << 7)                    // A format: bf16
         | (1u << 10)                   // B format: bf16
         | ((uint32_t)a_mn_major << 15)  // A major: 0 = K, 1 = MN
         | (0u << 16)                   // B major: K
         | ((uint32_t)(kN >> 3) << 17)  // N / 8
         | ((uint32_t)(kM >> 4) << 24);  // M / 16
}

// exact three-way bf16 split of an fp32 value
__device__ __forceinline__ void split3(float x, __nv_bfloat16& h, __nv_bfloat16& md,
                                       __nv_bfloat16& l) {
  h = __float2bfloat16_rn(x);
  const float r1 = x - __bfloat162float(h);
  md = __float2bfloat16_rn(r1);
  const float r2 = r1 - __bfloat162float(md);
  l = __float2bfloat16_rn(r2);
}

__device__ __forceinline__ uint32_t pack2(__nv_bfloat16 a, __nv_bfloat16 b) {
  return (uint32_t)__bfloat16_as_ushort(a) | ((uint32_t)__bfloat16_as_ushort(b) << 16);
}

// MN-major no-swizzle offset of element (mn, k) of a [128 x kKc] bf16 tile:
// core matrices of 8 k-rows x 16 B (8 mn); MN-adjacent cores 128 B apart (SBO),
// K groups of 8 kLboMN bytes apart (LBO).
__device__ __forceinline__ uint32_t mnmaj_off(int mn, int k) {
  return (uint32_t)((mn >> 3) * 128 + (k >> 3) * kLboMN + (k & 7) * 16 + (mn & 7) * 2);
}

// Ternary B chunk: element (l, k) = sign of component l at K index k0+k, from
// 64-bit masks; K-major layout, 16 bytes (8 k) per store.
__device__ __forceinline__ void fill_b(unsigned char* bs, const u64* __restrict__ Mk,
                                       const u64* __restrict__ Sg, int k0, int klim) {
  constexpr int kGroups = kKc / 8;  // 8-element K groups per chunk
  for (int e = threadIdx.x; e < kN * kGroups; e += kThreads) {
    const int l = e / kGroups, kg = e - l * kGroups;
    uint32_t w[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      uint32_t v = 0u;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int k = kg * 8 + 2 * h + t;
        uint32_t bits = 0u;
        if (k0 + k < klim) {
          const u64 mk = Mk[k0 + k];
          if ((mk >> l) & 1ull) bits = ((Sg[k0 + k] >> l) & 1ull) ? 0xBF80u : 0x3F80u;
        }
        v |= bits << (16 * t);
      }
      w[h] = v;
    }
    *(uint4*)(bs + kmaj_off(l, kg * 8)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// MODE 0: P = R (W V) -- A = R rows [i0, i0+128), K = columns; K-major A.
// MODE 1: Q^T = R^T U -- A = R^T columns [i0, i0+128), K = rows; MN-major A.
template <int MODE>
__global__ void __launch_bounds__(kThreads, 1) contract_kernel(
    const float* __restrict__ R, int m, int n, const u64* __restrict__ Mk,
    const u64* __restrict__ Sg, const float* __restrict__ w, int bb, int klen,
    float* __restrict__ Xp, int* __restrict__ status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 1024-byte aligned base for the operand tiles
  unsigned char* smem = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ uint32_t tmem_base;
  __shared__ __align__(8) u64 mbar[2];
  __shared__ int bad;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int M = MODE == 0 ? m : n;  // output rows
  const int Kdim = MODE == 0 ? n : m;
  const int i0 = blockIdx.x * kM;
  const int split = blockIdx.y;
  const int k_begin = split * klen, k_end = min(Kdim, k_begin + klen);
  const int nchunks = k_end > k_begin ? (k_end - k_begin + kKc - 1) / kKc : 0;
  // 16-byte loads only when every row of R starts 16-byte aligned
  const bool vec4 = (n & 3) == 0 && (((uintptr_t)R) & 15) == 0;

  if (wid == 0) {
    tmem_alloc(smem_u32(&tmem_base), kN);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(smem_u32(&mbar[0]), 1);
    mbar_init(smem_u32(&mbar[1]), 1);
    fence_mbar_init();
    bad = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  const uint32_t idesc = make_idesc(MODE);
  bool ok = true;

  for (int c = 0; c < nchunks; ++c) {
    const int s = c & 1;
    unsigned char* stage = smem + s * kStageBytes;
    if (c >= 2) {  // the MMAs that read this stage (chunk c-2) must be done
      if (tid == 0 && !mbar_wait(smem_u32(&mbar[s]), (uint32_t)((c / 2 - 1) & 1))) bad = 1;
      __syncthreads();
      if (bad) {
        ok = false;
        break;
      }
    }
    const int k0 = k_begin + c * kKc;
    // ---- A chunk: fp32 -> hi/mid/lo bf16, canonical layout ----
    if (MODE == 0) {
      // tile rows r (128) x k (kKc = 32): lanes cover 8 rows x 16 k per step
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int r = (wid + 8 * (u & 1)) * 8 + (lane >> 2);
        const int k = (u >> 1) * 16 + (lane & 3) * 4;
        const int gi = i0 + r, gk = k0 + k;
        float x[4] = {0.f, 0.f, 0.f, 0.f};
        if (gi < m) {
          const float* src = R + (size_t)gi * n + gk;
          if (vec4 && gk + 3 < k_end) {
            const float4 v = *(const float4*)src;
            x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (gk + e < k_end) x[e] = src[e];
          }
          if (w) {
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (gk + e < k_end) x[e] *= w[gk + e];
          }
        }
        __nv_bfloat16 h[4], md[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) split3(x[e], h[e], md[e], lo[e]);
        const uint32_t off = kmaj_off(r, k);
        *(uint2*)(stage + off) = make_uint2(pack2(h[0], h[1]), pack2(h[2], h[3]));
        *(uint2*)(stage + kPartBytes + off) = make_uint2(pack2(md[0], md[1]), pack2(md[2], md[3]));
        *(uint2*)(stage + 2 * kPartBytes + off) =
            make_uint2(pack2(lo[0], lo[1]), pack2(lo[2], lo[3]));
      }
    } else {
      // tile mn = columns j (128) x k = rows i (kKc = 32): lanes cover 8 k x 16 mn per step
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int k = (lane >> 2) + 8 * u;
        const int mn = wid * 16 + (lane & 3) * 4;
        const int gi = k0 + k, gj = i0 + mn;
        float x[4] = {0.f, 0.f, 0.f, 0.f};
        if (gi < k_end) {
          const float* src = R + (size_t)gi * n + gj;
          if (vec4 && gj + 3 < n) {
            const float4 v = *(const float4*)src;
            x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (gj + e < n) x[e] = src[e];
          }
        }
        __nv_bfloat16 h[4], md[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) split3(x[e], h[e], md[e], lo[e]);
        const uint32_t off = mnmaj_off(mn, k);
        *(uint2*)(stage + off) = make_uint2(pack2(h[0], h[1]), pack2(h[2], h[3]));
        *(uint2*)(stage + kPartBytes + off) = make_uint2(pack2(md[0], md[1]), pack2(md[2], md[3]));
        *(uint2*)(stage + 2 * kPartBytes + off) =
            make_uint2(pack2(lo[0], lo[1]), pack2(lo[2], lo[3]));
      }
    }
    // ---- B chunk: ternary components ----
    fill_b(stage + 3 * kPartBytes, Mk, Sg, k0, k_end);
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t abase = smem_u32(stage), bbase = smem_u32(stage + 3 * kPartBytes);
#pragma unroll
      for (int p = 0; p < 3; ++p)
#pragma unroll
        for (int ks = 0; ks < kKc / 16; ++ks) {
          uint64_t ad, bd;
          if (MODE == 0)
            ad = make_desc(abase + p * kPartBytes + ks * 256, 128, kSboK);
          else
            ad = make_desc(abase + p * kPartBytes + ks * 2 * kLboMN, kLboMN, 128);
          bd = make_desc(bbase + ks * 256, 128, kSboK);
          umma_bf16(tmem, ad, bd, idesc, (c > 0 || p > 0 || ks > 0) ? 1u : 0u);
        }
      umma_commit(smem_u32(&mbar[s]));
    }
  }
  // ---- wait for the last chunk's MMAs (all earlier ones complete before) ----
  if (tid == 0 && nchunks > 0) {
    const int cl = ok ? nchunks - 1 : -1;
    if (cl >= 0) {
      if (!mbar_wait(smem_u32(&mbar[cl & 1]), (uint32_t)((cl / 2) & 1))) bad = 1;
    } else {
      // stopped early: drain whatever was issued (bounded)
      for (int s = 0; s < 2; ++s) mbar_wait(smem_u32(&mbar[s]), 0u);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (bad) {
    if (tid == 0) atomicCAS(status, 0, EXTERND_ERR_TIMEOUT);
  } else if (nchunks > 0) {
    // ---- epilogue: TMEM -> partials; warp w reads lanes 32*(w%4).., columns 32*(w/4).. ----
    const int q = wid & 3, chalf = wid >> 2;
    const int row = q * 32 + lane;
    const int gi = i0 + row;
    float* out = Xp + ((size_t)split * M + gi) * bb;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t v[16];
      const int col = chalf * 32 + h * 16;
      tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)col, v);
      if (gi < M)
#pragma unroll
        for (int t = 0; t < 16; ++t)
          if (col + t < bb) out[col + t] = __uint_as_float(v[t]);
    }
  } else {
    // empty K range: zero partials
    const int q = wid & 3, chalf = wid >> 2;
    const int gi = i0 + q * 32 + lane;
    if (gi < M)
      for (int t = 0; t < 32; ++t)
        if (chalf * 32 + t < bb) Xp[((size_t)split * M + gi) * bb + chalf * 32 + t] = 0.f;
  }
  // every warp's tensor-memory loads are complete (tcgen05.wait::ld) and
  // ordered before the barrier; the deallocating warp orders itself after it
  tc_fence_before();
  __syncthreads();
  if (wid == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kN);
  }
}


// ===========================================================================
// Pipelined, persistent variant (row stride a multiple of 16 bytes): one CTA
// per SM, each taking an equal contiguous run of the (tile, K-chunk) units of
// the contraction (stream-K partition, umma_layout.cuh), so every SM streams
// R for the whole launch.  Per chunk the producer copies into one stage of
// the fp32 ring: the 128 x 32 tile of R (TMA tensor copy), the chunk's
// ternary B operand, already laid out for the MMA (bulk copy), and, for
// P = R W V, the chunk's 32 weights (bulk copy).  Converter warps split the
// tile into the three bf16 parts, which go straight into the stage's slice of
// tensor memory -- the A operand of tcgen05.mma may live there, K-major:
// TMEM lane = output row, one 32-bit column = two consecutive K elements;
// B is read by the MMA where the copy put it.  A stage (tile, B and A slice)
// is handed back to the producer by the tcgen05.commit after its MMAs.  Two
// accumulators in tensor memory alternate between the CTA's tile
// segments, so a finished segment is read out while the next one streams.
// Warp roles:
//   warp 0        producer (one lane); allocates / frees tensor memory
//   warp 1        MMA issuer (one lane)
//   warps 2..5    epilogue: accumulator -> split-K partial of the segment
//   warps 6..21   converters, two groups of eight on alternate chunks; warp w
//                 serves TMEM lanes 32 (w % 4) .. + 31 and K half
//                 ((w - 6) / 4) % 2 of its group's chunks
// mbarriers per stage: full (copies landed), afull (A parts stored), aempty
// (tcgen05.commit after the chunk's MMAs); accf / accfree the two
// accumulators (segment's MMAs done / read out); drain the final commit.
// One CTA per SM: with two co-resident CTAs the transposed contraction
// (Q^T = R^T U) returned wrong partial sums from the CTA placed second on an
// SM (reproducible with 160-280 CTAs, varying from run to run; one CTA per
// SM was exact); the shared memory a second CTA would use deepens the ring.
// ===========================================================================
constexpr int kS32 = 8;                                 // ring depth (fp32 tile + B + A stage)
constexpr int kTileBytes32 = kM * kKc * 4;              // 16 KB fp32 tile
constexpr int kBOff = kTileBytes32;                     // B chunk within a stage
constexpr int kWOff = kTileBytes32 + kBBytes;           // weights of the chunk
constexpr int kStageBytesP = kTileBytes32 + kBBytes + 1024;  // multiple of 1024
constexpr int kAcolsStage = 3 * (kKc / 2);              // 48 TMEM columns per A stage
constexpr int kAcc0 = 0, kAstage0 = 2 * kN;             // TMEM: 2 accumulators, then A stages
constexpr int kTmemCols = 512;
constexpr int kEpiWarps = 4;
constexpr int kConvWarp0 = 2 + kEpiWarps;
constexpr int kConvGroups = 2;                          // converter groups, alternate chunks
constexpr int kThreadsP = 32 * kConvWarp0 + 256 * kConvGroups;
constexpr int kSmemP = kS32 * kStageBytesP + 1024;
static_assert(kAstage0 + kS32 * kAcolsStage <= kTmemCols, "tensor memory budget");
// A converter group waits on stage s's `full` barrier by phase parity; that is
// unambiguous only if the same group consumed the stage's previous fill (chunk
// i - kS32) and so saw it land: every group must own whole stages.
static_assert(kS32 % kConvGroups == 0, "converter groups own whole ring stages");
static_assert(kStageBytesP % 1024 == 0, "swizzled tiles need 1024-byte alignment");
static_assert(2 * (kSmemP + 1024) > 228 * 1024, "the ring must keep the kernel at one CTA per SM");
static_assert(kSmemP <= 227 * 1024, "shared memory per CTA");

struct PipeBars {
  u64 full[kS32], afull[kS32], aempty[kS32], accf[2], accfree[2], drain;
};

__device__ __forceinline__ void mbar_arrive(uint32_t addr) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(addr) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t addr, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(addr), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, int x, int y,
                                            uint32_t mbar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, "
      "{%2, %3}], [%4];" ::"r"(dst),
      "l"((uint64_t)tmap), "r"(x), "r"(y), "r"(mbar)
      : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// D (TMEM) (+)= A (TMEM) x B (shared memory descriptor)
__device__ __forceinline__ void umma_ts_bf16(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}

// Bounded wait (budget in SM cycles) that also gives up once another thread
// of the CTA has recorded a timeout in *abort.  The waits for the CTA's own
// copies and MMAs before it exits use mbar_wait (kWaitBudget) instead.
__device__ __forceinline__ bool mbar_wait_ab(uint32_t addr, uint32_t parity,
                                             volatile int* abort, long long budget) {
  if (mbar_test(addr, parity)) return true;
  const long long t0 = clock64();
  unsigned spins = 0;
  while (!mbar_test(addr, parity)) {
    if (((++spins) & 15u) == 0u && *abort) return false;
    if (clock64() - t0 > budget) {
      *abort = 1;
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t mbar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"((uint64_t)src), "r"(bytes), "r"(mbar)
      : "memory");
}

// MODE 0: P = R (W V), A rows = rows of R, K = columns (tile box 32 x 128,
//         128-byte swizzle: 16-byte group g of tile row r sits at g ^ (r % 8)).
// MODE 1: Q^T = R^T U, A rows = columns of R, K = rows (box 128 x 32, no swizzle).
// T tiles of 128 output rows, C chunks of 32 along K, U = T C units over
// gridDim.x CTAs; S = slots per tile of Xp (umma_layout.cuh).
// Bop: ternary B chunks of the K range, 4 KB per 32 K entries.
// wpad: for MODE 0 the weights, zero padded to a multiple of 32 (or null).
template <int MODE>
__global__ void __launch_bounds__(kThreadsP, 1) contract_tma_kernel(
    const __grid_constant__ CUtensorMap tmap, int m, int n, const unsigned char* __restrict__ Bop,
    const float* __restrict__ wpad, int bb, int C, long long U, int S, float* __restrict__ Xp,
    int* __restrict__ status, long long budget) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* ring = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) PipeBars bars;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int G = gridDim.x, b = blockIdx.x;
  const int M = MODE == 0 ? m : n;
  const long long u0 = sk_u0(b, U, G), u1 = sk_u0(b + 1, U, G);
  const int nunits = (int)(u1 - u0);
  const bool weighted = MODE == 0 && wpad != nullptr;
  volatile int* ab = &abort_flag;

  if (wid == 0) {
    tmem_alloc(smem_u32(&tmem_base), kTmemCols);
    tmem_relinquish();
  }
  if (tid == 32) {
    for (int s = 0; s < kS32; ++s) {
      mbar_init(smem_u32(&bars.full[s]), 1);
      mbar_init(smem_u32(&bars.afull[s]), 8);
      mbar_init(smem_u32(&bars.aempty[s]), 1);
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(smem_u32(&bars.accf[q]), 1);
      mbar_init(smem_u32(&bars.accfree[q]), kEpiWarps);
    }
    mbar_init(smem_u32(&bars.drain), 1);
    fence_mbar_init();
    abort_flag = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (wid == 0) {
    if (lane == 0) {  // ---- producer ----
      const uint32_t tx = kTileBytes32 + kBBytes + (weighted ? kKc * 4 : 0);
      int issued = 0;
      // (tile, chunk) of the current unit, advanced incrementally: a 64-bit
      // division per chunk would cost more than the chunk's MMAs
      int t = (int)(u0 / C), c = (int)(u0 - (long long)t * C);
      for (int i = 0; i < nunits; ++i, c = (c + 1 == C) ? 0 : c + 1, t += (c == 0) ? 1 : 0) {
        const int s = i % kS32;
        // stage s (fp32 tile, B, A in tensor memory) is free once the MMAs
        // of chunk i - kS32 have completed
        if (i >= kS32 && !mbar_wait_ab(smem_u32(&bars.aempty[s]), ((i / kS32) + 1) & 1, ab, budget))
          break;
        const int kk = c * kKc;
        const uint32_t fb = smem_u32(&bars.full[s]);
        const uint32_t dst = smem_u32(ring + s * kStageBytesP);
        mbar_expect_tx(fb, tx);
        if (MODE == 0)
          tma_load_2d(dst, &tmap, kk, t * kM, fb);
        else
          tma_load_2d(dst, &tmap, t * kM, kk, fb);
        bulk_load(dst + kBOff, Bop + (size_t)(kk / kKc) * kBBytes, kBBytes, fb);
        if (weighted) bulk_load(dst + kWOff, wpad + kk, kKc * 4, fb);
        ++issued;
      }
      // every issued copy must have landed before the CTA may exit
      for (int i = issued > kS32 ? issued - kS32 : 0; i < issued; ++i)
        mbar_wait(smem_u32(&bars.full[i % kS32]), (uint32_t)((i / kS32) & 1));
    }
  } else if (wid == 1) {
    if (lane == 0) {  // ---- MMA issuer ----
      const uint32_t idesc = make_idesc(0);
      int seg = 0;
      bool ok = true;
      int c = (int)(u0 % C);  // chunk of the current unit within its tile
      for (int i = 0; i < nunits && ok; ++i, c = (c + 1 == C) ? 0 : c + 1) {
        const bool first = i == 0 || c == 0;
        const bool last = i == nunits - 1 || c == C - 1;
        const int q = seg & 1;
        // the accumulator of segment seg - 2 must have been read out
        if (first && seg >= 2 &&
            !mbar_wait_ab(smem_u32(&bars.accfree[q]), ((seg >> 1) - 1) & 1, ab, budget)) {
          ok = false;
          break;
        }
        const int s = i % kS32;
        if (!mbar_wait_ab(smem_u32(&bars.afull[s]), (i / kS32) & 1, ab, budget)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + kAcc0 + q * kN;
        const uint32_t acol = tmem + kAstage0 + s * kAcolsStage;
        const uint32_t bbase = smem_u32(ring + s * kStageBytesP + kBOff);
#pragma unroll
        for (int p = 0; p < 3; ++p)
#pragma unroll
          for (int ks = 0; ks < kKc / 16; ++ks)
            umma_ts_bf16(acc, acol + p * (kKc / 2) + ks * 8, make_desc(bbase + ks * 256, 128, kSboK),
                         idesc, (!first || p > 0 || ks > 0) ? 1u : 0u);
        umma_commit(smem_u32(&bars.aempty[s]));
        if (last) {
          umma_commit(smem_u32(&bars.accf[q]));
          ++seg;
        }
      }
      // completes once every MMA issued above has finished (also after an abort)
      umma_commit(smem_u32(&bars.drain));
      mbar_wait(smem_u32(&bars.drain), 0u);
    }
  } else if (wid < kConvWarp0) {
    // ---- epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31, all 64 columns ----
    const int quad = wid & 3;
    const int t_first = nunits > 0 ? (int)(u0 / C) : 0;
    const int nsegs = nunits > 0 ? (int)((u1 - 1) / C) - t_first + 1 : 0;
    for (int sg = 0; sg < nsegs; ++sg) {
      const int q = sg & 1;
      const bool ok = mbar_wait_ab(smem_u32(&bars.accf[q]), (sg >> 1) & 1, ab, budget);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const int t = t_first + sg;
      const int slot = b - sk_first(t, C, U, G);
      const int row = quad * 32 + lane, gi = t * kM + row;
      float* out = Xp + ((size_t)((size_t)t * S + slot) * kM + row) * bb;
#pragma unroll
      for (int h = 0; h < kN / 16; ++h) {
        uint32_t v[16];
        tmem_ld16(tmem + kAcc0 + q * kN + ((uint32_t)(quad * 32) << 16) + (uint32_t)(h * 16), v);
        if (gi < M) {
          if (bb == kN) {
#pragma unroll
            for (int t4 = 0; t4 < 4; ++t4)
              *(float4*)(out + h * 16 + 4 * t4) =
                  make_float4(__uint_as_float(v[4 * t4]), __uint_as_float(v[4 * t4 + 1]),
                              __uint_as_float(v[4 * t4 + 2]), __uint_as_float(v[4 * t4 + 3]));
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e)
              if (h * 16 + e < bb) out[h * 16 + e] = __uint_as_float(v[e]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars.accfree[q]));
    }
  } else {
    // ---- converters (two groups of eight warps, alternate chunks) ----
    const int cw = wid - kConvWarp0;
    const int grp = cw >> 3;
    const int quad = wid & 3;               // TMEM lanes this warp may access
    const int kh = (cw >> 2) & 1;           // K half of each chunk
    const int row = quad * 32 + lane;       // tile row = TMEM lane
    for (int i = grp; i < nunits; i += kConvGroups) {
      const int s = i % kS32;
      // the copies of chunk i have landed; the producer waited for the MMAs of
      // chunk i - kS32 before issuing them, so A stage s is free as well
      const bool ok = mbar_wait_ab(smem_u32(&bars.full[s]), (i / kS32) & 1, ab, budget);
      if (!__all_sync(0xffffffffu, ok)) break;
      const unsigned char* st = ring + s * kStageBytesP;
      float x[16];
      if (MODE == 0) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int g = (kh * 4 + q) ^ (row & 7);
          const float4 v = *(const float4*)(st + row * 128 + g * 16);
          x[4 * q] = v.x;
          x[4 * q + 1] = v.y;
          x[4 * q + 2] = v.z;
          x[4 * q + 3] = v.w;
        }
        if (weighted) {
          const float* ws = (const float*)(st + kWOff) + kh * 16;
#pragma unroll
          for (int e = 0; e < 16; ++e) x[e] *= ws[e];
        }
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) x[e] = *(const float*)(st + (kh * 16 + e) * 512 + row * 4);
      }
      uint32_t ph[8], pm[8], pl[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        __nv_bfloat16 h0, m0, l0, h1, m1, l1;
        split3(x[2 * e], h0, m0, l0);
        split3(x[2 * e + 1], h1, m1, l1);
        ph[e] = pack2(h0, h1);
        pm[e] = pack2(m0, m1);
        pl[e] = pack2(l0, l1);
      }
      tc_fence_after();
      const uint32_t ta =
          tmem + ((uint32_t)(quad * 32) << 16) + kAstage0 + s * kAcolsStage + kh * 8;
      tmem_st8(ta, ph);
      tmem_st8(ta + kKc / 2, pm);
      tmem_st8(ta + kKc, pl);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bars.afull[s]));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (wid == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (tid == 0 && abort_flag) atomicCAS(status, 0, EXTERND_ERR_TIMEOUT);
}

}  // namespace umma

namespace {

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the driver library); resolved once.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
    else
      cudaGetLastError();
  }
  return fn;
}

// Tensor map over the row-major m x n fp32 residual: MODE 0 boxes of 128
// rows x 32 columns (128-byte swizzle), MODE 1 boxes of 32 rows x 128 columns.
// Out-of-range box elements read as zero.
bool make_tmap(CUtensorMap* tm, const float* R, int m, int n, int mode) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)n, (cuuint64_t)m};
  const cuuint64_t strides[1] = {(cuuint64_t)n * sizeof(float)};
  const cuuint32_t box0[2] = {(cuuint32_t)umma::kKc, (cuuint32_t)umma::kM};
  const cuuint32_t box1[2] = {(cuuint32_t)umma::kM, (cuuint32_t)umma::kKc};
  const cuuint32_t estr[2] = {1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, (void*)R, dims, strides,
            mode == 0 ? box0 : box1, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            mode == 0 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool tma_ok(const float* R, int n) {
  return (n % 4) == 0 && (((uintptr_t)R) & 15) == 0 && getenv("EXTERND_CONTRACT_NO_TMA") == nullptr;
}

void set_attrs() {
  using namespace umma;
  static bool attr = false;
  if (attr) return;
  attr = true;
  cudaFuncSetAttribute(contract_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  cudaFuncSetAttribute(contract_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  cudaFuncSetAttribute(contract_tma_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemP);
  cudaFuncSetAttribute(contract_tma_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemP);
}

}  // namespace

// Stream-K plan of a contraction with M output rows and K-dimension Kdim:
// G CTAs (one per SM but one, and few enough that no tile is split into more
// than kMaxSegs segments), S = most segments of any tile.
void tc_contract_plan(int M, int Kdim, int nsm, TcPlan* p) {
  using namespace umma;
  p->T = (M + kM - 1) / kM;
  p->C = (Kdim + kKc - 1) / kKc;
  p->U = (long long)p->T * p->C;
  // one SM is left to the Gram / inverse kernels that run beside the
  // contraction on a side stream: they cannot share an SM with a contraction
  // CTA (registers), so on a full grid one CTA, and with it the launch, would
  // wait for them (17 % of a 9728 x 2560 block-ALS decomposition)
  p->G = sk_ctas(p->T, p->C, nsm, kMaxSegs);
  p->S = 1;
  for (int t = 0; t < p->T; ++t) p->S = std::max(p->S, sk_nseg(t, p->C, p->U, p->G));
}

// rows of an n-column fp32 matrix at a 16-byte aligned base are TMA-addressable
bool tc_contract_tma_ok(int n) { return tma_ok(nullptr, n) && encode_fn() != nullptr; }

// Host launchers.  With a plan the TMA kernel runs and writes stream-K tile
// partials (callers check tc_contract_tma_ok first); without one the direct
// kernel writes `splits` split-K partials over K ranges of klen (a multiple
// of 32).
int tc_contract_rv(const float* R, int m, int n, const unsigned long long* Vm,
                   const unsigned long long* Vs, const unsigned char* Bop, const float* w,
                   const float* wpad, int bb, const TcPlan* p, int klen, int splits, float* Pp,
                   long long budget, cudaStream_t st) {
  using namespace umma;
  set_attrs();
  int* status = status_word_ptr();
  CUtensorMap tm;
  if (p) {
    if (!make_tmap(&tm, R, m, n, 0)) return EXTERND_ERR_CUDA;
    contract_tma_kernel<0><<<p->G, kThreadsP, kSmemP, st>>>(tm, m, n, Bop, w ? wpad : nullptr, bb,
                                                            p->C, p->U, p->S, Pp, status,
                                                            budget > 0 ? budget : kWaitBudget);
  } else {
    contract_kernel<0><<<dim3((unsigned)((m + kM - 1) / kM), (unsigned)splits), umma::kThreads,
                         kSmemBytes, st>>>(R, m, n, Vm, Vs, w, bb, klen, Pp, status);
  }
  return cudaGetLastError() == cudaSuccess ? EXTERND_OK : EXTERND_ERR_CUDA;
}

int tc_contract_rtu(const float* R, int m, int n, const unsigned long long* Um,
                    const unsigned long long* Us, const unsigned char* Bop, int bb, const TcPlan* p,
                    int klen, int splits, float* Qp, long long budget, cudaStream_t st) {
  using namespace umma;
  set_attrs();
  int* status = status_word_ptr();
  CUtensorMap tm;
  if (p) {
    if (!make_tmap(&tm, R, m, n, 1)) return EXTERND_ERR_CUDA;
    contract_tma_kernel<1><<<p->G, kThreadsP, kSmemP, st>>>(tm, m, n, Bop, nullptr, bb, p->C, p->U,
                                                            p->S, Qp, status,
                                                            budget > 0 ? budget : kWaitBudget);
  } else {
    contract_kernel<1><<<dim3((unsigned)((n + kM - 1) / kM), (unsigned)splits), umma::kThreads,
                         kSmemBytes, st>>>(R, m, n, Um, Us, nullptr, bb, klen, Qp, status);
  }
  return cudaGetLastError() == cudaSuccess ? EXTERND_OK : EXTERND_ERR_CUDA;
}

}  // namespace externd
