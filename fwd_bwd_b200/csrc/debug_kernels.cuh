// debug_kernels.cuh -- single-CTA kernels that run one piece of the tensor-core path in
// isolation, so tests can compare it with an exact integer / float reference:
//   * debug_gemm_kernel: C = A B with the same TMA staging, shared-memory descriptors and
//     tcgen05 MMAs the attention kernels use, for every operand form they use (INT8 K-major
//     and MN-major A and B; FP16/BF16 K-major);
//   * debug_qk_kernel: the forward kernel's INT8 score product for one query tile against all
//     keys of one head, through the forward kernel's own issue_scores();
//   * mma_peak_kernel: back-to-back tcgen05 MMAs from resident shared memory, one CTA per SM,
//     so the host can time the tensor cores' sustained INT8 and 16-bit throughput (the
//     denominators of the attention kernels' rooflines);
//   * debug_wait_kernel: a bounded wait on an mbarrier that nothing arrives on, so tests can
//     drive the kernels' failure path (timeout recorded in the status word, TMEM freed, the
//     kernel returns) without hanging anything.
#pragma once

#include <stdint.h>

#include "attn_fwd.cuh"
#include "ptx.cuh"

namespace sage {
namespace dbg {

struct GemmSmem {
  uint8_t a[128 * 128 * 2];
  uint8_t b[128 * 128 * 2];
  uint64_t full, done;
  uint32_t tmem_base;
};

// kind 0: int8 -> int32; 1: fp16 -> fp32; 2: bf16 -> fp32.
// Tensor maps: A / B with the boxes the host chose for (kind, majorness, N, K).
__global__ void __launch_bounds__(128, 1)
    debug_gemm_kernel(const __grid_constant__ CUtensorMap tm_a,
                      const __grid_constant__ CUtensorMap tm_b, int kind, int a_mn, int b_mn,
                      int N, int K, void* C) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base = smem_u32(smem_raw);
  GemmSmem& sm = *reinterpret_cast<GemmSmem*>(smem_raw + ((1024u - (base & 1023u)) & 1023u));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&sm.full, 1);
    mbar_init(&sm.done, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (warp == 0) {
    tmem_alloc(&sm.tmem_base, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const int M = 128;
  if (threadIdx.x == 0) {
    if (kind == 0) {
      mbar_arrive_expect_tx(&sm.full, (M + N) * K);
      tma_load_2d(sm.a, &tm_a, 0, 0, &sm.full);
      tma_load_2d(sm.b, &tm_b, 0, 0, &sm.full);
    } else {
      mbar_arrive_expect_tx(&sm.full, (M + N) * K * 2);
      for (int at = 0; at < K / 64; ++at) {
        tma_load_2d(sm.a + at * M * 128, &tm_a, at * 64, 0, &sm.full);
        tma_load_2d(sm.b + at * N * 128, &tm_b, at * 64, 0, &sm.full);
      }
    }
    mbar_wait(&sm.full, 0, 300);
    tc_fence_after();
    const uint32_t aa = smem_u32(sm.a), ba = smem_u32(sm.b);
    if (kind == 0) {
      const uint32_t id = instr_desc(2, 1, 1, a_mn != 0, b_mn != 0, M, N);
      for (int kk = 0; kk < K / 32; ++kk) {
        uint64_t ad, bd;
        if (a_mn)  // A stored [K][M]: rows of 128 B along M, K-steps of 32 rows
          ad = smem_desc(aa + kk * 32 * M, K * M, 8 * M, kSwizzle128B);
        else       // A stored [M][K]
          ad = smem_desc(aa + kk * 32, 16, 8 * K, K == 128 ? kSwizzle128B : kSwizzle64B);
        if (b_mn)  // B stored [K][N]
          bd = smem_desc(ba + kk * 32 * N, K * N, 8 * N, N == 128 ? kSwizzle128B : kSwizzle64B);
        else       // B stored [N][K]
          bd = smem_desc(ba + kk * 32, 16, 8 * K, K == 128 ? kSwizzle128B : kSwizzle64B);
        mma_i8(tmem, ad, bd, id, kk > 0 ? 1u : 0u);
      }
    } else {
      const uint32_t ab = (kind == 2) ? 1u : 0u;
      const uint32_t id = instr_desc(1, ab, ab, false, false, M, N);
      for (int kk = 0; kk < K / 16; ++kk) {
        const uint32_t at = kk * 16 / 64, off = (kk * 16 % 64) * 2;
        mma_f16(tmem, smem_desc(aa + at * M * 128 + off, 16, 1024, kSwizzle128B),
                smem_desc(ba + at * N * 128 + off, 16, 1024, kSwizzle128B), id,
                kk > 0 ? 1u : 0u);
      }
    }
    mma_commit(&sm.done);
  }
  __syncwarp();
  mbar_wait(&sm.done, 0, 301);
  tc_fence_after();
  const int row = warp * 32 + lane;
  uint32_t* crow = reinterpret_cast<uint32_t*>(C) + static_cast<size_t>(row) * N;
  for (int c0 = 0; c0 < N; c0 += 16) {
    uint32_t v[16];
    tmem_ld16(tmem + ((warp * 32u) << 16) + c0, v);
    tmem_ld_wait();
    for (int e = 0; e < 16; ++e) crow[c0 + e] = v[e];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 128);
}

template <int D>
struct QkSmem {
  int8_t q[128 * D];
  int8_t k[64 * D];
  uint64_t full, done;
  uint32_t tmem_base;
};

// s_out[128][N] = Qc[q_tile rows] Kc^T for head bh.
template <int D>
__global__ void __launch_bounds__(128, 1)
    debug_qk_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k, int bh, int q_tile, int N,
                    int32_t* s_out) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base = smem_u32(smem_raw);
  QkSmem<D>& sm =
      *reinterpret_cast<QkSmem<D>*>(smem_raw + ((1024u - (base & 1023u)) & 1023u));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&sm.full, 1);
    mbar_init(&sm.done, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (warp == 0) {
    tmem_alloc(&sm.tmem_base, 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  for (int j = 0; j < N / 64; ++j) {
    // the forward kernel's accumulator convention: preload 1.5 * 2^23, accumulate onto it
#pragma unroll
    for (int c0 = 0; c0 < 64; c0 += 16) tmem_fill16(tmem + ((warp * 32u) << 16) + c0, kMagicBits);
    tmem_st_wait();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (threadIdx.x == 0) {
      const int bytes = (j == 0 ? 128 * D : 0) + 64 * D;
      mbar_arrive_expect_tx(&sm.full, bytes);
      if (j == 0) tma_load_2d(sm.q, &tm_q, 0, bh * N + q_tile * 128, &sm.full);
      tma_load_2d(sm.k, &tm_k, 0, bh * N + j * 64, &sm.full);
      mbar_wait(&sm.full, j & 1, 310);
      tc_fence_after();
      fwd::issue_scores<D>(tmem, sm.q, sm.k, 64, 1u);
      mma_commit(&sm.done);
    }
    __syncwarp();
    mbar_wait(&sm.done, j & 1, 311);
    tc_fence_after();
    const int row = warp * 32 + lane;
    int32_t* dst = s_out + static_cast<size_t>(row) * N + j * 64;
    for (int c0 = 0; c0 < 64; c0 += 16) {
      uint32_t v[16];
      tmem_ld16(tmem + ((warp * 32u) << 16) + c0, v);
      tmem_ld_wait();
      for (int e = 0; e < 16; ++e)
        dst[c0 + e] = static_cast<int32_t>(v[e]) - static_cast<int32_t>(kMagicBits);
    }
    tc_fence_before();
    __syncthreads();  // TMEM and the K tile are free for the next block
    tc_fence_after();
  }
  if (warp == 0) tmem_dealloc(tmem, 64);
}

struct PeakSmem {
  uint8_t a[128 * 128];  // A: 128 rows x 128 bytes, 128-byte swizzle, K-major
  uint8_t b[256 * 128];  // B: 256 rows x 128 bytes
  uint64_t done;
  uint32_t tmem_base;
};
constexpr int kPeakFillBytes = 128 * 128 + 256 * 128;

// One thread issues `groups` x 4 MMAs of M = 128, N = 256 and K = 32 bytes (kind::i8: 32
// elements; kind::f16: 16) back to back, alternating two 256-column accumulators; the
// operands are `fill`'s first 48 KB, staged once.  kind 0: int8 -> int32; 1: fp16 -> fp32;
// 2: bf16 -> fp32.
__global__ void __launch_bounds__(128, 1)
    mma_peak_kernel(const uint4* __restrict__ fill, int kind, int groups) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base = smem_u32(smem_raw);
  PeakSmem& sm = *reinterpret_cast<PeakSmem*>(smem_raw + ((1024u - (base & 1023u)) & 1023u));
  const int warp = threadIdx.x >> 5;
  uint4* dst = reinterpret_cast<uint4*>(sm.a);  // a and b are contiguous
  for (int i = threadIdx.x; i < kPeakFillBytes / 16; i += blockDim.x) dst[i] = fill[i];
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    mbar_init(&sm.done, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (warp == 0) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  if (threadIdx.x == 0) {
    const uint32_t ab = kind == 2 ? 1u : 0u;
    const uint32_t id = kind == 0 ? instr_desc(2, 1, 1, false, false, 128, 256)
                                  : instr_desc(1, ab, ab, false, false, 128, 256);
    const uint32_t aa = smem_u32(sm.a), ba = smem_u32(sm.b);
    for (int g = 0; g < groups; ++g) {
      const uint32_t acc = tmem + (g & 1) * 256;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t ad = smem_desc(aa + kk * 32, 16, 1024, kSwizzle128B);
        const uint64_t bd = smem_desc(ba + kk * 32, 16, 1024, kSwizzle128B);
        const uint32_t accum = (g >= 2 || kk > 0) ? 1u : 0u;
        if (kind == 0)
          mma_i8(acc, ad, bd, id, accum);
        else
          mma_f16(acc, ad, bd, id, accum);
      }
    }
    mma_commit(&sm.done);
    mbar_wait(&sm.done, 0, 320);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// One CTA holding TMEM waits (thread 0) on a barrier whose arrival never comes, for at most
// limit_ns; the wait records SAGE_ERR_TIMEOUT (site 330), then the CTA frees its TMEM and
// returns -- the same exit every pipeline kernel takes when one of its waits runs out.
__global__ void __launch_bounds__(128, 1) debug_wait_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_base;
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (warp == 0) {
    tmem_alloc(&tmem_base, 32);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) mbar_wait_ns(&bar, 0, 330, limit_ns);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem_base, 32);
}

}  // namespace dbg
}  // namespace sage
