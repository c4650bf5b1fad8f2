// Pipe-throughput probes: how many operations of one kind an SM retires per
// clock.  They pin the arithmetic roofline of the element math of the fused
// BCE (exp, log, reciprocal or tanh per logit, plus FP32 FMA work) on the GPU
// at hand instead of taking the rates from a table.
//
// Each thread runs 8 independent dependency chains of one operation in a loop
// (enough independent work per warp to cover the pipe's latency with 32 warps
// per SM); the SM's clock64 delta over the loop gives operations per clock.
#pragma once
#include <cstdint>
#include "ptx_sm100.cuh"
#include "tile_engine.cuh"

namespace cutbce {

enum : int {
  kProbeFfma = 0,     // fma.rn.f32
  kProbeFfma2 = 1,    // fma.rn.f32x2 (two FMAs per instruction)
  kProbeEx2 = 2,      // ex2.approx.ftz.f32 (+ one FADD to stay in range)
  kProbeRcp = 3,      // rcp.approx.ftz.f32
  kProbeTanh = 4,     // tanh.approx.f32
  kProbeLg2 = 5,      // lg2.approx.ftz.f32 (+ one FADD to stay in range)
  kProbeCvtBf16x2 = 6,  // cvt.rn.bf16x2.f32 (one instruction packs two values)
  kProbeFmax = 7,     // max.f32
  kProbeAdd2 = 8,     // add.rn.f32x2 (two additions per instruction)
  kProbeIadd = 9,     // add.s32
  kProbePrmt = 10,    // prmt.b32
  kProbeEx2F16x2 = 11,   // ex2.approx.f16x2 (+ one packed add to stay in range), counted per instruction
  kProbeEx2Bf16x2 = 12,  // ex2.approx.ftz.bf16x2 (+ one packed add), counted per instruction
  kProbeTanhF16x2 = 13,  // tanh.approx.f16x2, counted per instruction
  kProbeHfma2 = 14,      // fma.rn.f16x2, counted per instruction
  kProbeCvtF16x2 = 15,   // cvt.rn.f16x2.f32, counted per instruction
  kProbeFfmaSat = 16,    // fma.rn.sat.f32
  kProbeSelp = 17,       // setp.ge.f32 + selp.f32 (one select), counted per select
  kProbeLop3 = 18,       // and.b32 with a register operand
  kProbeFmul2 = 19,      // mul.rn.f32x2, counted as two operations
  kProbeCount = 20
};

constexpr int kProbeThreads = 1024;
constexpr int kProbeChains = 8;

__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm volatile("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

__device__ __forceinline__ uint64_t fmul2_u(uint64_t a, uint64_t b) {
  uint64_t d;
  asm volatile("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm volatile("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

template <int OP>
__global__ void __launch_bounds__(kProbeThreads, 1) k_probe(int iters, unsigned long long* cycles, float* sink) {
  float a[kProbeChains];
#pragma unroll
  for (int k = 0; k < kProbeChains; ++k) a[k] = 0.25f + 1e-4f * static_cast<float>((threadIdx.x + 37 * k) & 255);
  uint64_t a2[kProbeChains];
  if (OP == kProbeFfma2 || OP == kProbeAdd2 || OP == kProbeFmul2) {
#pragma unroll
    for (int k = 0; k < kProbeChains; ++k)
      a2[k] = (static_cast<uint64_t>(__float_as_uint(a[k])) << 32) | __float_as_uint(a[k] + 0.5f);
  }
  const uint64_t m2 = (static_cast<uint64_t>(__float_as_uint(0.999f)) << 32) | __float_as_uint(0.999f);
  const uint64_t c2 = (static_cast<uint64_t>(__float_as_uint(1e-3f)) << 32) | __float_as_uint(1e-3f);
  __syncthreads();
  const long long t0 = clock64();
  for (int i = 0; i < iters; ++i) {
#pragma unroll
    for (int k = 0; k < kProbeChains; ++k) {
      if (OP == kProbeFfma) a[k] = fmaf(a[k], 0.999f, 1e-3f);
      if (OP == kProbeFfma2) a2[k] = ffma2(a2[k], m2, c2);
      if (OP == kProbeEx2) a[k] = ex2_approx(a[k]) - 1.5f;          // stays in [-1, 0.5]
      if (OP == kProbeRcp) a[k] = rcp_approx(a[k] + 1.0f);          // stays in [0.5, 1]
      if (OP == kProbeTanh) a[k] = tanh_approx(a[k]);                // stays in (-1, 1)
      if (OP == kProbeLg2) a[k] = lg2_approx(a[k] + 2.0f);           // stays in [1, 2]
      if (OP == kProbeCvtBf16x2) a[k] = __uint_as_float(pack_bf16x2(a[k], a[k]));
      if (OP == kProbeFmax) {                                        // asm: the chain must not fold
        asm volatile("max.f32 %0, %0, %1;" : "+f"(a[k]) : "f"(0.5f));
      }
      if (OP == kProbeAdd2) a2[k] = fadd2(a2[k], c2);
      if (OP == kProbeIadd) {
        uint32_t v = __float_as_uint(a[k]);
        asm volatile("add.s32 %0, %0, 257;" : "+r"(v));
        a[k] = __uint_as_float(v);
      }
      if (OP == kProbePrmt) a[k] = __uint_as_float(__byte_perm(__float_as_uint(a[k]), 0x12345678u, 0x3726u));
      if (OP == kProbeEx2F16x2 || OP == kProbeEx2Bf16x2 || OP == kProbeTanhF16x2 || OP == kProbeHfma2) {
        // two 16-bit lanes in one register; values stay in a small range
        uint32_t v = __float_as_uint(a[k]);
        if (OP == kProbeEx2F16x2) {
          asm volatile("ex2.approx.f16x2 %0, %0;" : "+r"(v));
          asm volatile("sub.f16x2 %0, %0, %1;" : "+r"(v) : "r"(0x3E003E00u));          // - 1.5
        } else if (OP == kProbeEx2Bf16x2) {
          asm volatile("ex2.approx.ftz.bf16x2 %0, %0;" : "+r"(v));
          asm volatile("sub.bf16x2 %0, %0, %1;" : "+r"(v) : "r"(0x3FC03FC0u));         // - 1.5
        } else if (OP == kProbeTanhF16x2) {
          asm volatile("tanh.approx.f16x2 %0, %0;" : "+r"(v));
        } else {
          asm volatile("fma.rn.f16x2 %0, %0, %1, %2;" : "+r"(v) : "r"(0x3BFF3BFFu), "r"(0x1A001A00u));
        }
        a[k] = __uint_as_float(v);
      }
      if (OP == kProbeCvtF16x2) {
        uint32_t v;
        asm volatile("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(v) : "f"(a[k]), "f"(a[k]));
        a[k] = __uint_as_float(v & 0x3FFFFFFFu);
      }
      if (OP == kProbeFfmaSat) asm volatile("fma.rn.sat.f32 %0, %0, %1, %2;" : "+f"(a[k]) : "f"(0.999f), "f"(1e-3f));
      if (OP == kProbeSelp) {
        asm volatile("{\n\t.reg .pred p;\n\tsetp.ge.f32 p, %0, %1;\n\tselp.f32 %0, %2, %0, p;\n\t}"
                     : "+f"(a[k]) : "f"(0.5f), "f"(0.25f));
      }
      if (OP == kProbeLop3) {
        uint32_t v = __float_as_uint(a[k]);
        asm volatile("and.b32 %0, %0, %1;" : "+r"(v) : "r"(0xFFFFFF7Fu + static_cast<uint32_t>(k)));
        a[k] = __uint_as_float(v);
      }
      if (OP == kProbeFmul2) a2[k] = fmul2_u(a2[k], m2);
    }
  }
  __syncthreads();
  const long long t1 = clock64();
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < kProbeChains; ++k)
    s += (OP == kProbeFfma2 || OP == kProbeAdd2 || OP == kProbeFmul2) ? __uint_as_float(static_cast<uint32_t>(a2[k]))
                                                                     : a[k];
  if (s == 12345.678f) sink[threadIdx.x] = s;
  if (threadIdx.x == 0) cycles[blockIdx.x] = static_cast<unsigned long long>(t1 - t0);
}

// Tensor-core probe: one thread issues `iters` bf16 tcgen05.mma instructions of
// shape 128 x N x 16 (fp32 accumulate in tensor memory, A from shared or tensor
// memory, B from shared memory K-major or MN-major), commits, and waits.  Records the SM cycles
// spent issuing and until completion; operands are zero (their values do not
// affect timing).  One CTA per SM.
template <int N, bool kATmem, bool kBMN>
__global__ void __launch_bounds__(128, 1) k_probe_mma(int iters, unsigned long long* out) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;                    // 128 x 64 bf16, 128-byte swizzle (16 KB)
  uint8_t* sB = smem + 16384;            // N x 64 bf16 (K-major) or 64 x N (MN-major), 128-byte swizzle
  __shared__ uint64_t bar;
  __shared__ uint32_t tslot;
  for (int i = threadIdx.x; i < (16384 + N * 128) / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem)[i] = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbarrier_init();
  }
  fence_proxy_async_smem();
  if ((threadIdx.x >> 5) == 0) tmem_alloc(&tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tslot;
  if (kATmem) {
    // zero the 8 TMEM columns used as A (each warp its 32 lanes)
    uint32_t z[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) z[k] = 0;
    tmem_st16(tbase + ((static_cast<uint32_t>(threadIdx.x >> 5) * 32) << 16) + 256, z);
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) {
    const uint32_t idesc = idesc_bf16_f32(128, N, false, kBMN);
    const uint32_t a_base = smem_u32(sA), b_base = smem_u32(sB);
    const long long t0 = clock64();
    for (int i = 0; i < iters; ++i) {
      const int ks = i & 3;
      // MN-major B: 16 K-rows of 128-byte atoms per step, N in 64-wide column blocks of 64 rows
      const uint64_t bd = kBMN ? smem_desc_sw128(b_base + ks * 2048, 64 * 128, 1024)
                               : smem_desc_sw128(b_base + ks * 32, 16, 1024);
      if (kATmem) {
        umma_bf16_tmem_a(tbase, tbase + 256, bd, idesc, i > 0 ? 1u : 0u);
      } else {
        const uint64_t ad = smem_desc_sw128(a_base + ks * 32, 16, 1024);
        umma_bf16(tbase, ad, bd, idesc, i > 0 ? 1u : 0u);
      }
    }
    const long long t1 = clock64();
    umma_commit(&bar);
    wait_bar_drain(&bar, 0, 2000000000LL);
    const long long t2 = clock64();
    out[2 * blockIdx.x] = static_cast<unsigned long long>(t1 - t0);
    out[2 * blockIdx.x + 1] = static_cast<unsigned long long>(t2 - t0);
  }
  tc_fence_before();
  __syncthreads();
  if ((threadIdx.x >> 5) == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// The same probe on an SM pair: 2-CTA clusters, and the even CTA of each issues
// `iters` tcgen05.mma.cta_group::2 of shape 256 x N x 16 (each CTA holds 128
// rows of A, in shared or tensor memory, and its half of B; zero operands).
// Both CTAs allocate the pair's tensor memory; neither frees it before the
// issuing CTA has seen the commit and both have passed a cluster barrier.
template <int N, bool kATmem>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(128, 1) k_probe_mma_pair(int iters, unsigned long long* out) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;                    // 128 x 64 bf16, 128-byte swizzle (16 KB)
  uint8_t* sB = smem + 16384;            // N x 64 bf16, K-major, 128-byte swizzle
  __shared__ uint64_t bar;
  __shared__ uint32_t tslot;
  for (int i = threadIdx.x; i < (16384 + N * 128) / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem)[i] = make_uint4(0, 0, 0, 0);
  const uint32_t rank = cluster_ctarank();
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbarrier_init();
  }
  fence_proxy_async_smem();
  if ((threadIdx.x >> 5) == 0) tmem_alloc_pair(&tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tslot;
  if (kATmem) {
    uint32_t z[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) z[k] = 0;
    tmem_st16(tbase + ((static_cast<uint32_t>(threadIdx.x >> 5) * 32) << 16) + 256, z);
    tmem_st_wait();
  }
  // both CTAs' operands are in place before the even CTA issues
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  if (rank == 0 && threadIdx.x == 0) {
    const uint32_t idesc = idesc_bf16_f32(256, N, false, false);
    const uint32_t a_base = smem_u32(sA), b_base = smem_u32(sB);
    const long long t0 = clock64();
    for (int i = 0; i < iters; ++i) {
      const int ks = i & 3;
      const uint64_t bd = smem_desc_sw128(b_base + ks * 32, 16, 1024);
      if (kATmem) {
        umma_bf16_pair_tmem_a(tbase, tbase + 256, bd, idesc, i > 0 ? 1u : 0u);
      } else {
        const uint64_t ad = smem_desc_sw128(a_base + ks * 32, 16, 1024);
        umma_bf16_pair(tbase, ad, bd, idesc, i > 0 ? 1u : 0u);
      }
    }
    const long long t1 = clock64();
    umma_commit_pair(&bar);
    wait_bar_drain(&bar, 0, 2000000000LL);
    const long long t2 = clock64();
    out[2 * blockIdx.x] = static_cast<unsigned long long>(t1 - t0);
    out[2 * blockIdx.x + 1] = static_cast<unsigned long long>(t2 - t0);
  }
  // the pair's MMAs are complete before either CTA frees its tensor memory
  tc_fence_before();
  cluster_sync_all();
  if ((threadIdx.x >> 5) == 0) {
    tc_fence_after();
    tmem_dealloc_pair(tbase, 512);
  }
}

}  // namespace cutbce
