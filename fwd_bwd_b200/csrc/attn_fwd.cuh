// attn_fwd.cuh -- SageBwd forward attention on sm_100a (quantization-strategy paragraph of
// "SageBwd: trainable low-bit attention": S = Q K^T and O = P V in INT8).
//
// Per CTA: two tiles of 128 query rows of one (batch, head), walking 64-key blocks.
//   warp 8      TMA producer: the Q code tiles once, then K and V code blocks through a
//               4-stage ring (K and V blocks are shared by both query tiles).
//   warp 9      MMA issuer (one thread): S_j = Qc Kc_j^T (kind::i8, M=128, N=64, into TMEM,
//               double-buffered per tile) and PV_j = Pc_j Vc_j (kind::i8, M=128, N=d).
//   warps 0-7   softmax, one query row per thread (warps 0-3 tile 0, 4-7 tile 1):
//               z = A * (sQ sK tau), causal mask, block max, p~ = exp(z - max_block),
//               P codes = rne(127 p~) written to shared memory in the tensor core's swizzled
//               K-major layout, running max / sum, and the dequantizing fold
//               O <- alpha O + PV * beta with beta = exp(max_block - max_running) sV / 127.
//   warps 10-11 idle (they complete the producer warpgroup, which gives its registers to the
//               softmax warpgroups: 256 x 232 + 128 x 40 = 64512 = 384 x 168).
// TMEM (512 columns): tile g uses columns [256g, 256g+256): S buffers at +0 and +64, PV at
// +128 (d columns, INT32).  The INT32 regions are preloaded with the bits of 1.5 * 2^23 before
// each MMA (see kMagicBits), so results read back as floats that one FMA dequantizes; the MMA
// thread writes the preload with one bf16 MMA (mma_fill_magic), so the softmax warps only read
// TMEM.
// O (float32) lives in registers; it is stored in the 16-bit type, or in float32 when
// Args::o_f32 is set (a partial result of context parallelism, merged by log-sum-exp later).
//
// Q-smoothing (template flag QS): every score of key j gains the per-key bias k_bias_j, copied
// with the K block into shared memory; the block maximum is then taken over the biased scores
// rather than over the raw INT32 values.
//
// P quantization: one scale per (query row, 64-key block).  The codes rne(127 p / max p) do
// not depend on which running maximum p was taken against, so computing them against the
// block's own maximum (as here) equals any other evaluation order in exact arithmetic.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stddef.h>
#include <stdint.h>

#include <type_traits>

#include "ptx.cuh"
#include "rowops.cuh"

namespace sage {
namespace fwd {

constexpr int BM = 128;   // query rows per tile (MMA M)
constexpr int BKV = 64;   // keys per block (= k_block)
constexpr int NT = 2;     // query tiles per CTA
constexpr int NST = 4;    // K/V pipeline stages
constexpr int kThreads = 384;
constexpr int kProducerWarp = 8, kMmaWarp = 9;
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 232;
constexpr int kOtherRegs = 40;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kOtherRegs <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");

template <int D>
struct Smem {
  int8_t q[NT][BM * D];
  int8_t k[NST][BKV * D];
  int8_t v[NST][BKV * D];
  int8_t p[NT][2][BM * BKV];
  alignas(256) uint8_t fill[kFillBytes];  // operands of the preload MMA (mma_fill_magic)
  float kb[NST][BKV];  // Q-smoothing: k_bias of the stage's keys
  uint64_t q_full;
  uint64_t k_full[NST], v_full[NST], kv_empty[NST];
  uint64_t s_full[NT][2], p_full[NT][2], pv_full[NT], pv_free[NT];
  uint32_t tmem_base;
  int abort;
};

template <int D>
constexpr size_t smem_bytes() {
  return sizeof(Smem<D>) + 1024;  // + alignment slack (tiles need 1024-byte alignment)
}

// Every TMA destination / tensor-core operand tile starts on a 1024-byte boundary.
template <int D>
constexpr bool tiles_aligned() {
  return offsetof(Smem<D>, q) % 1024 == 0 && (BM * D) % 1024 == 0 &&
         offsetof(Smem<D>, k) % 1024 == 0 && (BKV * D) % 1024 == 0 &&
         offsetof(Smem<D>, v) % 1024 == 0 && offsetof(Smem<D>, p) % 1024 == 0 &&
         (BM * BKV) % 1024 == 0 && offsetof(Smem<D>, fill) % 256 == 0;
}
static_assert(tiles_aligned<64>() && tiles_aligned<128>(), "shared-memory tiles misaligned");

struct Args {
  const float* q_scale;
  const float* k_scale;
  const float* v_scale;
  void* o;
  float* lse;
  int BH, N, q_block, causal;
  float scale_log2;  // softmax_scale * log2(e)
  int nsup;          // CTAs per head: ceil(N / 256)
  const float* k_bias;  // [BH, N] (Q-smoothing)
  float* o_f32;  // when set, O is written here in float32 [BH, N, D] instead of to `o`
};

template <int D>
__device__ __forceinline__ Smem<D>& smem_ref(uint8_t* raw) {
  const uint32_t a = smem_u32(raw);
  return *reinterpret_cast<Smem<D>*>(raw + ((1024u - (a & 1023u)) & 1023u));
}

// Issue S (+)= Qc Kc^T for one tile / block: d/32 MMAs of K = 32 bytes.  accumulate = 1 adds
// onto the preloaded accumulator.
template <int D>
__device__ __forceinline__ void issue_scores(uint32_t d_tmem, const int8_t* qs,
                                             const int8_t* ks, int n_keys, uint32_t accumulate) {
  constexpr uint32_t kSw = (D == 128) ? kSwizzle128B : kSwizzle64B;
  constexpr uint32_t kSbo = 8 * D;  // 8 rows of D bytes
  const uint32_t idesc = instr_desc(2, 1, 1, false, false, BM, n_keys);
  const uint32_t qa = smem_u32(qs), ka = smem_u32(ks);
#pragma unroll
  for (int kk = 0; kk < D / 32; ++kk) {
    mma_i8(d_tmem, smem_desc(qa + kk * 32, 16, kSbo, kSw), smem_desc(ka + kk * 32, 16, kSbo, kSw),
           idesc, (kk > 0 || accumulate) ? 1u : 0u);
  }
}

template <typename T, int D, bool QS>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, Args args) {
  extern __shared__ uint8_t smem_raw[];
  Smem<D>& sm = smem_ref<D>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = args.N;
  // head-major order (a head's CTAs share its K / V codes in L2); within a head the query
  // tiles with the most key blocks come first when causal
  const int bh = blockIdx.x / args.nsup;
  const int sidx = blockIdx.x % args.nsup;
  const int sup = args.causal ? (args.nsup - 1 - sidx) : sidx;
  int q0[NT], nb[NT];
  bool active[NT];
  int nb_max = 0;
#pragma unroll
  for (int g = 0; g < NT; ++g) {
    q0[g] = sup * (NT * BM) + g * BM;
    active[g] = q0[g] < N;
    nb[g] = active[g] ? (args.causal ? (q0[g] + BM) / BKV : N / BKV) : 0;
    nb_max = max(nb_max, nb[g]);
  }

  write_fill_operands(sm.fill, threadIdx.x, kThreads);
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    sm.abort = device_aborted() ? 1 : 0;
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int g = 0; g < NT; ++g) {
      mbar_init(&sm.s_full[g][0], 1);
      mbar_init(&sm.s_full[g][1], 1);
      mbar_init(&sm.p_full[g][0], BM);
      mbar_init(&sm.p_full[g][1], BM);
      mbar_init(&sm.pv_full[g], 1);
      mbar_init(&sm.pv_free[g], BM);
    }
    fence_barrier_init();
  }
  __syncthreads();
  if (sm.abort) return;
  if (warp == kMmaWarp) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kOtherRegs));
    if (warp == kProducerWarp && lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const int row_base = bh * N;
      int nact = 0;
      for (int g = 0; g < NT; ++g) nact += active[g] ? 1 : 0;
      mbar_arrive_expect_tx(&sm.q_full, nact * BM * D);
      for (int g = 0; g < NT; ++g)
        if (active[g]) tma_load_2d(sm.q[g], &tm_q, 0, row_base + q0[g], &sm.q_full);
      for (int j = 0; j < nb_max; ++j) {
        const int st = j % NST;
        if (j >= NST) mbar_wait(&sm.kv_empty[st], ((j / NST) - 1) & 1, 100);
        mbar_arrive_expect_tx(&sm.k_full[st], BKV * D + (QS ? BKV * 4 : 0));
        tma_load_2d(sm.k[st], &tm_k, 0, row_base + j * BKV, &sm.k_full[st]);
        if constexpr (QS)
          bulk_load(sm.kb[st], args.k_bias + row_base + j * BKV, BKV * 4, &sm.k_full[st]);
        mbar_arrive_expect_tx(&sm.v_full[st], BKV * D);
        tma_load_2d(sm.v[st], &tm_v, 0, row_base + j * BKV, &sm.v_full[st]);
      }
    } else if (warp == kMmaWarp && lane == 0) {
      constexpr uint32_t kSw = (D == 128) ? kSwizzle128B : kSwizzle64B;
      constexpr uint32_t kSbo = 8 * D;
      const uint32_t idesc_pv = instr_desc(2, 1, 1, false, true, BM, D);
      mbar_wait(&sm.q_full, 0, 101);
      mbar_wait(&sm.k_full[0], 0, 102);
      tc_fence_after();
      for (int g = 0; g < NT; ++g)
        if (nb[g] > 0) {
          mma_fill_magic(tmem + g * 256, sm.fill, BKV);
          issue_scores<D>(tmem + g * 256, sm.q[g], sm.k[0], BKV, 1u);
          mma_commit(&sm.s_full[g][0]);
        }
      for (int j = 0; j < nb_max; ++j) {
        const int st = j % NST;
        if (j + 1 < nb_max) {
          const int st1 = (j + 1) % NST;
          mbar_wait(&sm.k_full[st1], ((j + 1) / NST) & 1, 103);
          tc_fence_after();
          for (int g = 0; g < NT; ++g)
            if (j + 1 < nb[g]) {
              // buffer (j+1)&1 held S_{j-1}: read before p_full[j-1]; preloaded here
              mma_fill_magic(tmem + g * 256 + ((j + 1) & 1) * 64, sm.fill, BKV);
              issue_scores<D>(tmem + g * 256 + ((j + 1) & 1) * 64, sm.q[g], sm.k[st1], BKV,
                              1u);
              mma_commit(&sm.s_full[g][(j + 1) & 1]);
            }
        }
        mbar_wait(&sm.v_full[st], (j / NST) & 1, 104);
        for (int g = 0; g < NT; ++g) {
          if (j >= nb[g]) continue;
          mbar_wait(&sm.p_full[g][j & 1], (j >> 1) & 1, 105);
          if (j > 0) mbar_wait(&sm.pv_free[g], (j - 1) & 1, 106);
          tc_fence_after();
          const uint32_t pa = smem_u32(sm.p[g][j & 1]);
          const uint32_t va = smem_u32(sm.v[st]);
          mma_fill_magic(tmem + g * 256 + 128, sm.fill, D);
#pragma unroll
          for (int kk = 0; kk < BKV / 32; ++kk) {
            mma_i8(tmem + g * 256 + 128, smem_desc(pa + kk * 32, 16, 8 * BKV, kSwizzle64B),
                   smem_desc(va + kk * 32 * D, BKV * D, kSbo, kSw), idesc_pv, 1u);
          }
          mma_commit(&sm.pv_full[g]);
        }
        mma_commit(&sm.kv_empty[st]);
      }
    }
    __syncwarp();
    tc_fence_before();
    named_barrier_sync(15, kThreads);
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kSoftmaxRegs));
    // ---------------- softmax warps ----------------
    const int g = warp >> 2, quarter = warp & 3;
    if (active[g]) {
      const int r = quarter * 32 + lane;
      const int i = q0[g] + r;
      const int nqb = N / args.q_block, nkb = N / BKV;
      const float cq = args.q_scale[bh * nqb + i / args.q_block] * args.scale_log2;
      const float* ksc = args.k_scale + static_cast<size_t>(bh) * nkb;
      const float* vsc = args.v_scale + static_cast<size_t>(bh) * nkb;
      const uint32_t lane_base = tmem + ((quarter * 32u) << 16) + g * 256;
      // O in column pairs: the fold runs on the FMA pipe's paired (f32x2) instructions
      float2 O[D / 2];
#pragma unroll
      for (int c = 0; c < D / 2; ++c) O[c] = make_float2(0.0f, 0.0f);
      float m2 = -INFINITY, l = 0.0f, alpha_prev = 1.0f, beta_prev = 0.0f;
      int8_t* pbase = sm.p[g][0];
      float sk_next = ksc[0], sv_next = vsc[0];

      // O <- alpha O + PV_jj * beta (PV read back as 1.5*2^23 + PV), then re-preload PV
      auto fold_pv = [&](int jj) {
        const float b22 = scale22(beta_prev);
        const float nb22 = __fmul_rn(-kMagic, b22);
        mbar_wait(&sm.pv_full[g], jj & 1, 110);
        tc_fence_after();
        // 32-column chunks (one load each), double-buffered: the load of chunk c+1 is in flight
        // while chunk c is folded
        uint32_t a0[16], a1[16], b0[16], b1[16];
        tmem_ld32x(lane_base + 128, a0, a1);
        tmem_ld_wait_regs(a0, a1);
        const float2 al2 = make_float2(alpha_prev, alpha_prev);
        const float2 b2 = make_float2(b22, b22), nb2 = make_float2(nb22, nb22);
        // O = alpha O + deq(PV) for two columns per instruction (deq exact, as in deq())
        auto fold32 = [&](const uint32_t (&x0)[16], const uint32_t (&x1)[16], int c0) {
#pragma unroll
          for (int c = 0; c < 16; c += 2) {
            const float2 t = __ffma2_rn(make_float2(__uint_as_float(x0[c]),
                                                    __uint_as_float(x0[c + 1])), b2, nb2);
            O[(c0 + c) / 2] = __ffma2_rn(O[(c0 + c) / 2], al2, t);
          }
#pragma unroll
          for (int c = 0; c < 16; c += 2) {
            const float2 t = __ffma2_rn(make_float2(__uint_as_float(x1[c]),
                                                    __uint_as_float(x1[c + 1])), b2, nb2);
            O[(c0 + 16 + c) / 2] = __ffma2_rn(O[(c0 + 16 + c) / 2], al2, t);
          }
        };
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 64) {
          if (c0 + 32 < D) tmem_ld32x(lane_base + 128 + c0 + 32, b0, b1);
          fold32(a0, a1, c0);
          if (c0 + 32 < D) {
            tmem_ld_wait_regs(b0, b1);
            if (c0 + 64 < D) tmem_ld32x(lane_base + 128 + c0 + 64, a0, a1);
            fold32(b0, b1, c0 + 32);
            if (c0 + 64 < D) tmem_ld_wait_regs(a0, a1);
          }
        }
        tc_fence_before();
        mbar_arrive(&sm.pv_free[g]);
      };

      for (int j = 0; j < nb[g]; ++j) {
        const float sk = sk_next, sv = sv_next;
        if (j + 1 < nb[g]) {
          sk_next = ksc[j + 1];
          sv_next = vsc[j + 1];
        }
        const float c22 = scale22(cq * sk);
        const float nc22 = __fmul_rn(-kMagic, c22);
        const bool diag = args.causal && (j * BKV + BKV - 1 > q0[g]);
        const int key0 = j * BKV;
        mbar_wait(&sm.s_full[g][j & 1], (j >> 1) & 1, 111);
        tc_fence_after();
        const uint32_t sa = lane_base + (j & 1) * 64;
        // Q-smoothing: the block's key biases, bulk-copied with its K codes.  Waiting on the
        // stage's own barrier makes the copy visible here; the stage cannot be refilled before
        // this tile's P_j has been consumed, so the phase is still block j's.
        const float* kbj = sm.kb[j % NST];
        if constexpr (QS) mbar_wait(&sm.k_full[j % NST], (j / NST) & 1, 112);
        // pass 1: block maximum of kMagic + A (floats, ordered like A) over unmasked keys; with
        // Q-smoothing, of the biased scores themselves
        // (all 64 keys loaded at once; two maximum chains)
        // the block's 64 scores stay in registers for pass 2
        float mx;
        uint32_t a0[16], a1[16], b0[16], b1[16];
        {
          tmem_ld64x(sa, a0, a1, b0, b1);  // the block's 64 scores in one load
          tmem_ld_wait_regs4(a0, a1, b0, b1);
          float m0 = -INFINITY, m1 = -INFINITY;
          auto maxh = [&](const uint32_t (&x0)[16], const uint32_t (&x1)[16], int h, float& m) {
            if constexpr (QS) {
#pragma unroll
              for (int cc = 0; cc < 16; ++cc) {
                const int k0 = key0 + h * 32 + cc;
                float f0 = fmaf(kbj[h * 32 + cc], args.scale_log2, deq(x0[cc], c22, nc22));
                float f1 = fmaf(kbj[h * 32 + 16 + cc], args.scale_log2, deq(x1[cc], c22, nc22));
                if (diag && k0 > i) f0 = -INFINITY;
                if (diag && k0 + 16 > i) f1 = -INFINITY;
                m = fmax3(m, f0, f1);
              }
            } else if (diag) {
              float mo = -INFINITY;  // second chain (odd columns)
#pragma unroll
              for (int cc = 0; cc < 16; ++cc) {
                const int k0 = key0 + h * 32 + cc;
                const float f0 = k0 <= i ? __uint_as_float(x0[cc]) : -INFINITY;
                const float f1 = k0 + 16 <= i ? __uint_as_float(x1[cc]) : -INFINITY;
                if (cc & 1)
                  mo = fmax3(mo, f0, f1);
                else
                  m = fmax3(m, f0, f1);
              }
              m = fmaxf(m, mo);
            } else {
              float mo = -INFINITY;
#pragma unroll
              for (int cc = 0; cc < 16; cc += 2) {
                m = fmax3(m, __uint_as_float(x0[cc]), __uint_as_float(x1[cc]));
                mo = fmax3(mo, __uint_as_float(x0[cc + 1]), __uint_as_float(x1[cc + 1]));
              }
              m = fmaxf(m, mo);
            }
          };
          maxh(a0, a1, 0, m0);
          maxh(b0, b1, 1, m1);
          mx = fmaxf(m0, m1);
        }
        const bool has = mx != -INFINITY;
        float mblk;
        if constexpr (QS)
          mblk = mx;
        else
          mblk = has ? __fmaf_rn(mx, c22, nc22) : -INFINITY;  // fl(c * A_max)
        // pass 2: p~ = exp2(z - mblk), codes rne(127 p~), row sum, from the scores pass 1
        // loaded; four partial row sums keep the adds off one dependency chain; the causal mask
        // test exists only in the diagonal blocks' copy of the loop.
        int8_t* prow = pbase + (j & 1) * (BM * BKV);
        // Two keys per FMA-pipe instruction (f32x2); the exponentials stay one per key.
        float2 rs2[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
        const float2 c2 = make_float2(c22, c22), nc2 = make_float2(nc22, nc22);
        const float2 nm2 = make_float2(-mblk, -mblk);
        const float2 k127 = make_float2(127.0f, 127.0f), km2 = make_float2(kMagic, kMagic);
        auto pass2 = [&](auto masked) {
          auto conv = [&](const uint32_t (&x0)[16], const uint32_t (&x1)[16], int h) {
            uint32_t pk[8];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4) {
                float2 f[2];
#pragma unroll
                for (int e = 0; e < 4; e += 2) {
                  const int cc = q4 * 4 + e;
                  const uint32_t a_0 = half ? x1[cc] : x0[cc];
                  const uint32_t a_1 = half ? x1[cc + 1] : x0[cc + 1];
                  float2 z = __ffma2_rn(make_float2(__uint_as_float(a_0), __uint_as_float(a_1)),
                                        c2, nc2);  // exact dequantization, as deq()
                  if constexpr (QS) {
                    const float2 kb = make_float2(kbj[h * 32 + half * 16 + cc],
                                                  kbj[h * 32 + half * 16 + cc + 1]);
                    z = __ffma2_rn(kb, make_float2(args.scale_log2, args.scale_log2), z);
                  }
                  const float2 t = __fadd2_rn(z, nm2);
                  float2 p = make_float2(ex2_approx(t.x), ex2_approx(t.y));
                  if constexpr (decltype(masked)::value) {
                    const int key = key0 + h * 32 + half * 16 + cc;
                    if (key > i) p.x = 0.0f;
                    if (key + 1 > i) p.y = 0.0f;
                  }
                  rs2[e >> 1] = __fadd2_rn(rs2[e >> 1], p);
                  f[e >> 1] = __ffma2_rn(p, k127, km2);
                }
                pk[half * 4 + q4] = pack_magic4(f[0].x, f[0].y, f[1].x, f[1].y);
              }
            }
            // keys h*32 .. h*32+31 are 16-byte chunks 2h and 2h+1 of this row
            *reinterpret_cast<uint4*>(prow + swz_offset(r, 2 * h, 64)) =
                make_uint4(pk[0], pk[1], pk[2], pk[3]);
            *reinterpret_cast<uint4*>(prow + swz_offset(r, 2 * h + 1, 64)) =
                make_uint4(pk[4], pk[5], pk[6], pk[7]);
          };
          conv(a0, a1, 0);
          conv(b0, b1, 1);
        };
        if (diag)
          pass2(std::true_type{});
        else
          pass2(std::false_type{});
        const float rs = (rs2[0].x + rs2[0].y) + (rs2[1].x + rs2[1].y);
        const float m2n = fmaxf(m2, mblk);
        const float alpha = ex2_approx(m2 - m2n);
        const float eblk = has ? ex2_approx(mblk - m2n) : 0.0f;
        l = fmaf(l, alpha, eblk * rs);
        const float beta = eblk * sv * (1.0f / 127.0f);
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&sm.p_full[g][j & 1]);
        if (j > 0) fold_pv(j - 1);
        alpha_prev = alpha;
        beta_prev = beta;
        m2 = m2n;
      }
      fold_pv(nb[g] - 1);
      // epilogue: O / l in the output type, LSE = (m2 + log2 l) ln 2
      const float inv_l = 1.0f / l;
      if (args.o_f32 != nullptr) {
        // float32 partial result (context parallelism merges several of them)
        float4* of = reinterpret_cast<float4*>(args.o_f32 + (static_cast<size_t>(bh) * N + i) * D);
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 4)
          of[c0 / 4] = make_float4(O[c0 / 2].x * inv_l, O[c0 / 2].y * inv_l,
                                   O[c0 / 2 + 1].x * inv_l, O[c0 / 2 + 1].y * inv_l);
      } else {
        T* orow = reinterpret_cast<T*>(args.o) + (static_cast<size_t>(bh) * N + i) * D;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 8) {
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            f[e] = O[(c0 + e) / 2].x * inv_l;
            f[e + 1] = O[(c0 + e) / 2].y * inv_l;
          }
          *reinterpret_cast<uint4*>(orow + c0) = pack8<T>(f);
        }
      }
      args.lse[static_cast<size_t>(bh) * N + i] = (m2 + log2f(l)) * 0.69314718055994531f;
    }
    tc_fence_before();
    named_barrier_sync(15, kThreads);
  }
}

}  // namespace fwd
}  // namespace sage
