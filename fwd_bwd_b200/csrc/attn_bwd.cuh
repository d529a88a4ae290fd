// attn_bwd.cuh -- SageBwd backward attention on sm_100a ("SageBwd: trainable low-bit
// attention", quantization-strategy and error-propagation paragraphs).
//
// Per CTA: one tile of 128 keys (two 64-key K blocks) of one (batch, head), walking the tiles
// of 128 queries that can see it.  Per query tile:
//   1. S = Qc Kc^T (kind::i8) and dP = dO V^T (kind::f16 on the raw 16-bit dO and V, float32
//      accumulation -- the one matmul the page keeps in 16-bit float) into TMEM;
//   2. P = exp(z - LSE), dS = P (dP - D) (pass A, each thread one query row of 64 keys; values
//      stored back to TMEM), per-warp absmax of P and dS handed to the readers through shared
//      memory and a per-parity mbarrier (each reader forms the q_block x 64 tile maxima it
//      needs), then INT8 codes written to shared memory (pass B) in the 128-byte swizzled
//      layout, which the tensor core reads K-major (for dQ) and MN-major (for dV, dK);
//   3. dV_t = Pc^T dOc and dK_t = dSc^T Qc (kind::i8, M = 128 keys, one per q_block group),
//      dequantized by the tile scales and added to float32 accumulators in registers;
//      every INT32 accumulator region is preloaded with the bits of 1.5 * 2^23 so the results
//      read back as floats that one exact FMA dequantizes (see kMagicBits); the MMA thread
//      writes every preload with one bf16 MMA (mma_fill_magic), so the compute warps store to
//      TMEM only P and dS in pass A;
//   4. dQ_t = dSc Kc per 64-key block (kind::i8), dequantized, summed and added to a float32
//      dQ accumulator in global memory: for d = 128 computed transposed (TMEM lanes = head-dim
//      channels), staged per warp in shared memory and added by the TMA unit
//      (cp.reduce.async.bulk); for d = 64 with vector atomics.
// S and dP are double-buffered in TMEM, so the tensor core computes them for query tile i+1
// while the compute warps turn tile i into codes.
//
// Warps 0-7 compute (warpgroup h owns keys 64h .. 64h+63 in step 2 and d columns h*d/2 ..
// in steps 3-4), warp 8 is the TMA producer, warp 9 the MMA issuer, warps 10-11 idle.  The
// producer warpgroup gives registers to the compute warpgroups (setmaxnreg): at launch every
// thread holds 168, afterwards 256 x 216 + 128 x 72 = 64512 = 384 x 168.  The MMA thread keeps
// 72: with 56 it spilled and its reloads delayed the tensor-core issue; the compute warps' 216
// leave them fewer spills than 208 (-0.9% time).
// Context parallelism (Args::dk_acc set): the epilogue stores or adds the raw dK_hat / dV rows
// into float32 accumulators instead of finishing them, since other chunks of queries add
// theirs; the keys' owner applies the RMSNorm backward afterwards.
// Q-smoothing (template flag QS): pass A adds the per-key bias to the recomputed scores, and
// pass B also sums each key's dS codes over the tile's rows (one warp reduction per key), so
// the epilogue can add dK_bias = tau * (sum over tiles of sdS * column sum) * mu_Q.
// TMEM (512 columns): buffer b in {0,1} at [256b, 256b+256): [0,128) S -> P -> dV_t ->
// dQ_t(block 0); [128,256) dP -> dS -> dK_t -> dQ_t(block 1).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stddef.h>
#include <stdint.h>

#include <type_traits>

#include "ptx.cuh"
#include "rowops.cuh"

namespace sage {
namespace bwd {

constexpr int BQ = 128;   // query rows per tile
constexpr int BKT = 128;  // keys per CTA
constexpr int kThreads = 384;
constexpr int kProducerWarp = 8, kMmaWarp = 9;
constexpr int kLaunchRegs = 168;   // registers per thread the kernel must be launched with
constexpr int kComputeRegs = 216;  // compute warpgroups after setmaxnreg.inc
constexpr int kOtherRegs = 72;     // producer / MMA warpgroup after setmaxnreg.dec
static_assert(2 * 128 * kComputeRegs + 128 * kOtherRegs <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");

template <typename T>
struct IsBf16 {
  static constexpr bool value = false;
};
template <>
struct IsBf16<__nv_bfloat16> {
  static constexpr bool value = true;
};

template <int D>
struct Stage {
  int8_t qc[BQ * D];
  int8_t doc[BQ * D];
};

constexpr int kDqRows = 16;  // queries per dQ staging round (d = 128)
constexpr int kDqCols = 32;  // channels per warp in a dQ staging round (d = 128)

template <int D>
struct Smem {
  Stage<D> st[2];
  uint8_t dor[BQ * D * 2];  // raw 16-bit dO of the current tile, [D/64 atoms][128 rows][128 B]
  int8_t kc[BKT * D];
  uint8_t v[BKT * D * 2];  // raw 16-bit V, [D/64 atoms][128 rows][128 B]
  int8_t pc[BQ * BKT];     // P codes  [128 q][128 keys], 128-byte swizzle
  int8_t dsc[BQ * BKT];    // dS codes [128 q][128 keys], 128-byte swizzle
  // dQ staging for the asynchronous bulk reduction, per compute warp 4 KB:
  // d = 128: [buffer][query row][channel of the warp], 2 x 16 x 32 floats;
  // d = 64: one box of 32 query rows x 32 channels (128-byte swizzle)
  float dqs[8][2][kDqRows * kDqCols];
  alignas(256) uint8_t fill[kFillBytes];  // operands of the preload MMA (mma_fill_magic)
  alignas(16) float red_p[2][8];  // per-warp tile maxima of P, [tile parity][warp]
  alignas(16) float red_ds[2][8];  // and of |dS|
  float dot[BKT];                   // RMSNorm-backward row dot products (warpgroup 1 -> 0)
  float kb[BKT];                    // Q-smoothing: k_bias of the CTA's keys
  // Q-smoothing: per compute warp, the sum over tiles of sdS * (column sum of dSc over the
  // warp's rows) for the 64 keys of its warpgroup; one writer per element, so the totals do
  // not depend on timing
  float cs[8][64];
  uint64_t kv_full, q_full[2], q_empty[2], dor_full, dor_free;
  uint64_t sdp_full[2], pds_ready, dvdk_full, dvdk_free, dq_full, dq_free;
  uint64_t red_full[2];  // tile parity: every warp's tile maxima are in red_p / red_ds
  uint32_t tmem_base;
  int abort;
};

template <int D>
constexpr size_t smem_bytes() {
  return sizeof(Smem<D>) + 1024;
}

// Every TMA destination / tensor-core operand tile starts on a 1024-byte boundary (the
// structure itself is placed on one), as the swizzled layouts and descriptors require.
template <int D>
constexpr bool tiles_aligned() {
  return offsetof(Smem<D>, st) % 1024 == 0 && sizeof(Stage<D>) % 1024 == 0 &&
         offsetof(Stage<D>, doc) % 1024 == 0 && offsetof(Smem<D>, dor) % 1024 == 0 &&
         offsetof(Smem<D>, kc) % 1024 == 0 && offsetof(Smem<D>, v) % 1024 == 0 &&
         offsetof(Smem<D>, pc) % 1024 == 0 && offsetof(Smem<D>, dsc) % 1024 == 0 &&
         offsetof(Smem<D>, dqs) % 1024 == 0 && offsetof(Smem<D>, fill) % 256 == 0;
}
static_assert(smem_bytes<128>() <= 232448, "shared memory exceeds the per-block limit");
static_assert(tiles_aligned<64>() && tiles_aligned<128>(), "shared-memory tiles misaligned");

struct Args {
  const float* q_scale;   // [BH, N/q_block]
  const float* k_scale;   // [BH, N/64]
  const float* do_scale;  // [BH, N/q_block]
  const float* lse;       // [BH, N]
  const float* dvec;      // [BH, N]
  const void* k_raw;      // [BH, N, D] (RMSNorm backward of dk)
  const float* k_inv_rms; // [BH, N]
  void* dk;
  void* dv;
  int BH, N, q_block, causal, qknorm;
  float scale_log2;  // softmax_scale * log2(e)
  float tau;         // softmax_scale
  const float* k_bias;  // [BH, N] (Q-smoothing)
  const float* q_mean;  // [BH, D] (Q-smoothing)
  // context-parallel partial (both set, Q-smoothing off): the CTA's raw dK_hat / dV rows go to
  // these float32 [BH, N, D] accumulators instead of being finished and stored; acc_add = 0
  // stores them (the first chunk of queries), 1 adds them
  float* dk_acc;
  float* dv_acc;
  int acc_add;
};

template <int D>
__device__ __forceinline__ Smem<D>& smem_ref(uint8_t* raw) {
  const uint32_t a = smem_u32(raw);
  return *reinterpret_cast<Smem<D>*>(raw + ((1024u - (a & 1023u)) & 1023u));
}

template <typename T, int D, bool QS>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_qc,
                    const __grid_constant__ CUtensorMap tm_kc,
                    const __grid_constant__ CUtensorMap tm_doc,
                    const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_dq, Args args) {
  constexpr uint32_t kSwC = (D == 128) ? kSwizzle128B : kSwizzle64B;  // code tiles
  constexpr uint32_t kSboC = 8 * D;
  constexpr int kHalfD = D / 2;
  extern __shared__ uint8_t smem_raw[];
  Smem<D>& sm = smem_ref<D>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = args.N;
  const int nkt = N / BKT;
  // head-major order: the key tiles of one head run together and share its query-side tiles
  // and dQ accumulator in L2; within a head the tile with the most work (t = 0) comes first
  const int bh = blockIdx.x / nkt;
  const int t = blockIdx.x % nkt;
  const int i_first = args.causal ? t : 0;
  const int nq = N / BQ - i_first;
  const int G = BQ / args.q_block;  // q_block groups per query tile (1 or 2)

  write_fill_operands(sm.fill, threadIdx.x, kThreads);
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    sm.abort = device_aborted() ? 1 : 0;
    mbar_init(&sm.kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.q_full[s], 1);
      mbar_init(&sm.q_empty[s], 1);
      mbar_init(&sm.sdp_full[s], 1);
    }
    mbar_init(&sm.dor_full, 1);
    mbar_init(&sm.dor_free, 1);
    mbar_init(&sm.pds_ready, 256);
    for (int s = 0; s < 2; ++s)  // one arrival per compute warp
      mbar_init(&sm.red_full[s], 8);
    mbar_init(&sm.dvdk_full, 1);
    mbar_init(&sm.dvdk_free, 256);
    mbar_init(&sm.dq_full, 1);
    mbar_init(&sm.dq_free, 256);
    fence_barrier_init();
  }
  if constexpr (QS) {
    for (int i = threadIdx.x; i < BKT; i += kThreads) {
      sm.kb[i] = args.k_bias[static_cast<size_t>(bh) * N + t * BKT + i];
      for (int w = 0; w < 8; w += 2) sm.cs[w + (i >> 6)][i & 63] = 0.0f;
    }
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
  const int row_base = bh * N;

  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kOtherRegs));
    if (warp == kProducerWarp && lane == 0) {
      tma_prefetch_desc(&tm_qc);
      tma_prefetch_desc(&tm_kc);
      tma_prefetch_desc(&tm_doc);
      tma_prefetch_desc(&tm_do);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(&sm.kv_full, BKT * D * 3);
      tma_load_2d(sm.kc, &tm_kc, 0, row_base + t * BKT, &sm.kv_full);
      for (int a = 0; a < D / 64; ++a)
        tma_load_2d(sm.v + a * BKT * 128, &tm_v, a * 64, row_base + t * BKT, &sm.kv_full);
      for (int it = 0; it < nq; ++it) {
        const int s = it & 1;
        if (it >= 2) mbar_wait(&sm.q_empty[s], ((it >> 1) - 1) & 1, 200);
        const int row = row_base + (i_first + it) * BQ;
        mbar_arrive_expect_tx(&sm.q_full[s], BQ * D * 2);
        tma_load_2d(sm.st[s].qc, &tm_qc, 0, row, &sm.q_full[s]);
        tma_load_2d(sm.st[s].doc, &tm_doc, 0, row, &sm.q_full[s]);
        // the raw dO tile is single-buffered: wait until dP of the previous tile has read it
        if (it >= 1) mbar_wait(&sm.dor_free, (it - 1) & 1, 206);
        mbar_arrive_expect_tx(&sm.dor_full, BQ * D * 2);
        for (int a = 0; a < D / 64; ++a)
          tma_load_2d(sm.dor + a * BQ * 128, &tm_do, a * 64, row, &sm.dor_full);
      }
    } else if (warp == kMmaWarp && lane == 0) {
      const uint32_t id_s = instr_desc(2, 1, 1, false, false, BQ, BKT);
      const uint32_t ab = IsBf16<T>::value ? 1u : 0u;
      const uint32_t id_dp = instr_desc(1, ab, ab, false, false, BQ, BKT);
      const uint32_t id_mn = instr_desc(2, 1, 1, true, true, BKT, D);   // dV_t, dK_t
      const uint32_t id_dq = instr_desc(2, 1, 1, false, true, BQ, D);   // dQ_t (d = 64)
      const uint32_t id_dqt = instr_desc(2, 1, 1, true, false, D, BQ);  // dQ_t^T (d = 128)
      const uint32_t kca = smem_u32(sm.kc), va = smem_u32(sm.v);
      const uint32_t pca = smem_u32(sm.pc), dsa = smem_u32(sm.dsc);
      // S and dP of query tile `it` into TMEM buffer it & 1
      auto issue_sdp = [&](int it) {
        const int s = it & 1;
        const uint32_t dst = tmem + s * 256;
        const uint32_t qca = smem_u32(sm.st[s].qc), dora = smem_u32(sm.dor);
        mbar_wait(&sm.q_full[s], (it >> 1) & 1, 202);
        mbar_wait(&sm.dor_full, it & 1, 207);
        tc_fence_after();
        mma_fill_magic(dst, sm.fill, BKT);  // the S accumulator's preload
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk)
          mma_i8(dst, smem_desc(qca + kk * 32, 16, kSboC, kSwC),
                 smem_desc(kca + kk * 32, 16, kSboC, kSwC), id_s, 1u);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk * 16 / 64) * (BQ * 128) + (kk * 16 % 64) * 2;
          mma_f16(dst + 128, smem_desc(dora + off, 16, 1024, kSwizzle128B),
                  smem_desc(va + off, 16, 1024, kSwizzle128B), id_dp, kk > 0 ? 1u : 0u);
        }
        mma_commit(&sm.sdp_full[s]);
        mma_commit(&sm.dor_free);
      };
      mbar_wait(&sm.kv_full, 0, 201);
      issue_sdp(0);
      int dvdk_cnt = 0;
      for (int it = 0; it < nq; ++it) {
        const int s = it & 1;
        const uint32_t buf = tmem + s * 256;
        if (it + 1 < nq) {
          // buffer (it+1)&1 last held tile it-1: free once its dQ has been read out
          if (it >= 1) mbar_wait(&sm.dq_free, (it - 1) & 1, 203);
          issue_sdp(it + 1);
        }
        const uint32_t qca = smem_u32(sm.st[s].qc), doca = smem_u32(sm.st[s].doc);
        mbar_wait(&sm.pds_ready, it & 1, 204);
        tc_fence_after();
        for (int g = 0; g < G; ++g) {
          const int q0 = g * args.q_block;
          // preload dV_t ([0, D)) and dK_t ([128, 128 + D)); P / dS (pass B) and the previous
          // group's products (read-out) have been read from these columns
          if constexpr (D == 128) {
            mma_fill_magic(buf, sm.fill, 256);
          } else {
            mma_fill_magic(buf, sm.fill, D);
            mma_fill_magic(buf + 128, sm.fill, D);
          }
          for (int kk = 0; kk < args.q_block / 32; ++kk) {
            const int qr = q0 + kk * 32;
            mma_i8(buf, smem_desc(pca + qr * 128, BQ * BKT, 1024, kSwizzle128B),
                   smem_desc(doca + qr * D, BQ * D, kSboC, kSwC), id_mn, 1u);
            mma_i8(buf + 128, smem_desc(dsa + qr * 128, BQ * BKT, 1024, kSwizzle128B),
                   smem_desc(qca + qr * D, BQ * D, kSboC, kSwC), id_mn, 1u);
          }
          mma_commit(&sm.dvdk_full);
          // dK_t / dV_t are the last readers of this tile's Q and dO codes: release the stage
          if (g == G - 1) mma_commit(&sm.q_empty[s]);
          mbar_wait(&sm.dvdk_free, dvdk_cnt & 1, 205);
          ++dvdk_cnt;
          tc_fence_after();
        }
        // dQ_t per 64-key block.  d = 128: dQ_t^T = Kc[block]^T dSc[:, block]^T (M = d,
        // N = 128 queries; A = K codes read MN-major, B = dS codes K-major), so TMEM lanes are
        // head-dim channels and each warp's read-out holds 32 contiguous channels of a row.
        // d = 64: dQ_t = dSc[:, block] Kc[block] (M = 128 queries, N = d).
        if constexpr (D == 128) {
          mma_fill_magic(buf, sm.fill, 256);
        } else {
          mma_fill_magic(buf, sm.fill, D);
          mma_fill_magic(buf + 128, sm.fill, D);
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            if constexpr (D == 128)
              mma_i8(buf + hh * 128,
                     smem_desc(kca + (hh * 64 + kk * 32) * D, BKT * D, kSboC, kSwC),
                     smem_desc(dsa + hh * 64 + kk * 32, 16, 1024, kSwizzle128B), id_dqt, 1u);
            else
              mma_i8(buf + hh * 128, smem_desc(dsa + hh * 64 + kk * 32, 16, 1024, kSwizzle128B),
                     smem_desc(kca + (hh * 64 + kk * 32) * D, BKT * D, kSboC, kSwC), id_dq, 1u);
          }
        mma_commit(&sm.dq_full);
      }
    }
    // teardown: every MMA has completed once the compute warps pass this barrier
    __syncwarp();
    tc_fence_before();
    named_barrier_sync(15, kThreads);
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kComputeRegs));
    // ---------------- compute warps ----------------
    // Software-pipelined: pass A of tile it+1 (TMEM buffer (it+1)&1 only) runs between pass B
    // of tile it and the read-outs of tile it, so the tensor core computes dV_t / dK_t / dQ_t
    // of tile it meanwhile.
    const int h = warp >> 2, quarter = warp & 3;
    const int r = quarter * 32 + lane;  // TMEM lane = query row (steps 1-2, 4) / key row (3)
    const uint32_t lane_off = (quarter * 32u) << 16;
    const int nqb = N / args.q_block, nkb = N / 64;
    const float* ksc = args.k_scale + static_cast<size_t>(bh) * nkb;
    const float sk_h = ksc[2 * t + h];
    const float sk0 = ksc[2 * t], sk1 = ksc[2 * t + 1];
    const int key_base = t * BKT;
    const int wpg = args.q_block / 32;  // warps per q_block group
    const int g_row = r / args.q_block;
    // float32 dV / dK accumulators of this thread's key row, column pairs (f32x2 updates)
    float2 accv[kHalfD / 2], acck[kHalfD / 2];
#pragma unroll
    for (int c = 0; c < kHalfD / 2; ++c) accv[c] = acck[c] = make_float2(0.0f, 0.0f);
    int dvdk_cnt = 0;
    int dq_round = 0;  // dQ staging rounds so far (selects the staging buffer)

    // per-row inputs of query tile `it`: (c, lse2, D) for this thread's row
    auto row_inputs = [&](int it, float& c, float& lse2, float& dvr) {
      const int qrow = (i_first + it) * BQ + r;
      const size_t grow = static_cast<size_t>(row_base) + qrow;
      c = args.q_scale[static_cast<size_t>(bh) * nqb + qrow / args.q_block] * sk_h *
          args.scale_log2;
      lse2 = args.lse[grow] * 1.4426950408889634f;
      dvr = args.dvec[grow];
    };
    // pass A of tile it: P, dS into TMEM buffer it&1, per-warp maxima into red_*[it&1]
    auto pass_a = [&](int it, float c, float lse2, float dvr) {
      const int b = it & 1;
      const uint32_t lane_base = tmem + lane_off + b * 256;
      const int qt = i_first + it;
      const bool diag = args.causal && (qt == t);
      const float c22 = scale22(c);
      const float nc22 = __fmul_rn(-kMagic, c22);
      const float2 c2 = make_float2(c22, c22), nc2 = make_float2(nc22, nc22);
      const float2 nlse2 = make_float2(-lse2, -lse2), ndvr2 = make_float2(-dvr, -dvr);
      const float2 sl2 = make_float2(args.scale_log2, args.scale_log2);
      mbar_wait(&sm.sdp_full[b], (it >> 1) & 1, 210);
      tc_fence_after();
      float pmax = 0.0f, dsmax = 0.0f;
      // 8-column chunks, double-buffered: the TMEM loads of chunk ch+1 are in flight while
      // chunk ch computes.  The causal mask (key > query) exists only on the diagonal tile, so
      // the chunk loop is compiled twice and the off-diagonal copy carries no mask test.
      auto chunks = [&](auto masked) {
        // two keys per FMA-pipe instruction (f32x2); the exponentials stay one per key
        auto proc_a = [&](uint32_t (&sa)[8], uint32_t (&pa)[8], int col) {
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            float2 z = __ffma2_rn(make_float2(__uint_as_float(sa[e]), __uint_as_float(sa[e + 1])),
                                  c2, nc2);  // exact dequantization, as deq()
            if constexpr (QS)
              z = __ffma2_rn(make_float2(sm.kb[col + e], sm.kb[col + e + 1]), sl2, z);
            const float2 t = __fadd2_rn(z, nlse2);
            float2 p = make_float2(ex2_approx(t.x), ex2_approx(t.y));
            if constexpr (decltype(masked)::value) {
              // diagonal tile: key index - query index = col - r
              if (col + e > r) p.x = 0.0f;
              if (col + e + 1 > r) p.y = 0.0f;
            }
            const float2 ds = __fmul2_rn(
                p, __fadd2_rn(make_float2(__uint_as_float(pa[e]), __uint_as_float(pa[e + 1])),
                              ndvr2));
            dsmax = fmax3(dsmax, fabsf(ds.x), fabsf(ds.y));
            sa[e] = __float_as_uint(p.x);
            sa[e + 1] = __float_as_uint(p.y);
            pa[e] = __float_as_uint(ds.x);
            pa[e + 1] = __float_as_uint(ds.y);
          }
#pragma unroll
          for (int e = 0; e < 8; e += 2)
            pmax = fmax3(pmax, __uint_as_float(sa[e]), __uint_as_float(sa[e + 1]));
          tmem_st8(lane_base + col, sa);
          tmem_st8(lane_base + 128 + col, pa);
        };
        const int c0 = h * 64;
        uint32_t sa0[8], pa0[8], sa1[8], pa1[8];
        tmem_ld8(lane_base + c0, sa0);
        tmem_ld8(lane_base + 128 + c0, pa0);
        tmem_ld_wait_regs8(sa0, pa0);
#pragma unroll
        for (int ch = 0; ch < 8; ch += 2) {
          tmem_ld8(lane_base + c0 + 8 * ch + 8, sa1);
          tmem_ld8(lane_base + 128 + c0 + 8 * ch + 8, pa1);
          proc_a(sa0, pa0, c0 + 8 * ch);
          tmem_ld_wait_regs8(sa1, pa1);
          if (ch + 2 < 8) {
            tmem_ld8(lane_base + c0 + 8 * ch + 16, sa0);
            tmem_ld8(lane_base + 128 + c0 + 8 * ch + 16, pa0);
          }
          proc_a(sa1, pa1, c0 + 8 * ch + 8);
          if (ch + 2 < 8) tmem_ld_wait_regs8(sa0, pa0);
        }
      };
      if (diag)
        chunks(std::true_type{});
      else
        chunks(std::false_type{});
      tmem_st_wait();
      // per-warp maxima of P and |dS|; the tile maxima (q_block rows x 64 keys) are formed by
      // their readers -- pass B and the read-outs of this tile -- once every warp has arrived
      pmax = warp_max(pmax);
      dsmax = warp_max(dsmax);
      if (lane == 0) {
        sm.red_p[b][h * 4 + quarter] = pmax;
        sm.red_ds[b][h * 4 + quarter] = dsmax;
        mbar_arrive(&sm.red_full[b]);
      }
      // sm.red_*[b] is rewritten only in pass A of tile it+2, which waits for that tile's
      // S / dP, issued after every thread released tile it's dQ -- i.e. after every warp
      // finished reading them for tile it.  (Tiles 0 and 1 have their S / dP issued back to
      // back, hence the two slots.)
    };
    // maximum over the warps of q_block group g in warpgroup kh's key block (the tile's
    // absmax of P or dS): all four warps (q_block = 128) or a pair (64).  Maxima below 2^-121,
    // where the code multiplier 127 / max would overflow float32, are raised to 2^-121: such a
    // tile is quantized (and dequantized) with the scale 2^-121 / 127 instead of max / 127, so
    // its codes and scales stay finite and consistent (a zero tile keeps all-zero codes).
    auto tile_max = [&](const float* red, int g, int kh) {
      const float4 v = *reinterpret_cast<const float4*>(red + kh * 4);
      const float m = wpg == 4 ? fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w))
                               : (g == 0 ? fmaxf(v.x, v.y) : fmaxf(v.z, v.w));
      return fmaxf(m, 0x1p-121f);
    };

    // pass B's code multipliers 127 / max of tile `it` (its own row group and key half) from
    // the tile maxima, once every warp has arrived; IEEE quotients, like the read-outs' scales
    // max / 127 (an approximate reciprocal would flush a subnormal maximum to zero).  One
    // barrier per tile parity, so arrivals for tiles it and it+1 never share a phase; a warp
    // cannot arrive for tile it+2 before every thread released tile it's dQ.
    auto multipliers = [&](int it, float& ip, float& ids, float& sdsc) {
      const int b = it & 1;
      mbar_wait(&sm.red_full[b], (it >> 1) & 1, 213);
      const float tp = tile_max(sm.red_p[b], g_row, h);
      const float tds = tile_max(sm.red_ds[b], g_row, h);
      ip = __fdiv_rn(127.0f, tp);
      ids = __fdiv_rn(127.0f, tds);
      sdsc = QS ? __fdiv_rn(tds, 127.0f) : 0.0f;  // Q-smoothing column sums: this group's scale
    };

    float c_n, lse2_n, dvr_n, ip, ids, sdsc;
    row_inputs(0, c_n, lse2_n, dvr_n);
    pass_a(0, c_n, lse2_n, dvr_n);
    multipliers(0, ip, ids, sdsc);
    for (int it = 0; it < nq; ++it) {
      const int b = it & 1;
      const uint32_t lane_base = tmem + lane_off + b * 256;
      const int qt = i_first + it;
      if (it + 1 < nq) row_inputs(it + 1, c_n, lse2_n, dvr_n);  // loads in flight during pass B
      // pass B: INT8 codes into shared memory.  The TMEM loads of chunk ch+1 are in flight while
      // chunk ch is converted (two keys per FMA).
      const float2 ip2 = make_float2(ip, ip), ids2 = make_float2(ids, ids);
      const float2 km2 = make_float2(kMagic, kMagic);
      auto proc_b = [&](uint32_t (&sa)[16], uint32_t (&pa)[16], int ch) {
        uint32_t cp[4], cd[4];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          float2 fp[2], fd[2];
#pragma unroll
          for (int e = 0; e < 4; e += 2) {
            const int x = q4 * 4 + e;
            fp[e >> 1] = __ffma2_rn(make_float2(__uint_as_float(sa[x]), __uint_as_float(sa[x + 1])),
                                    ip2, km2);
            fd[e >> 1] = __ffma2_rn(make_float2(__uint_as_float(pa[x]), __uint_as_float(pa[x + 1])),
                                    ids2, km2);
          }
          cp[q4] = pack_magic4(fp[0].x, fp[0].y, fp[1].x, fp[1].y);
          cd[q4] = pack_magic4(fd[0].x, fd[0].y, fd[1].x, fd[1].y);
        }
        const uint32_t off = swz_offset(r, h * 4 + ch, 128);
        *reinterpret_cast<uint4*>(sm.pc + off) = make_uint4(cp[0], cp[1], cp[2], cp[3]);
        *reinterpret_cast<uint4*>(sm.dsc + off) = make_uint4(cd[0], cd[1], cd[2], cd[3]);
        if constexpr (QS) {
          // column sums of the dS codes over the warp's 32 rows (one q_block group, so one
          // scale), added to the per-key total; lane e carries column col + e
          float mine = 0.0f;
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int v = static_cast<int>(cd[e >> 2] << (24 - 8 * (e & 3))) >> 24;
            const int cs = __reduce_add_sync(0xFFFFFFFFu, v);
            if (lane == e) mine = static_cast<float>(cs);
          }
          if (lane < 16) sm.cs[warp][ch * 16 + lane] += mine * sdsc;
        }
      };
      {
        const int c0 = h * 64;
        uint32_t sa0[16], pa0[16], sa1[16], pa1[16];
        tmem_ld16(lane_base + c0, sa0);
        tmem_ld16(lane_base + 128 + c0, pa0);
        tmem_ld_wait_regs(sa0, pa0);
        tmem_ld16(lane_base + c0 + 16, sa1);
        tmem_ld16(lane_base + 128 + c0 + 16, pa1);
        proc_b(sa0, pa0, 0);
        tmem_ld_wait_regs(sa1, pa1);
        tmem_ld16(lane_base + c0 + 32, sa0);
        tmem_ld16(lane_base + 128 + c0 + 32, pa0);
        proc_b(sa1, pa1, 1);
        tmem_ld_wait_regs(sa0, pa0);
        tmem_ld16(lane_base + c0 + 48, sa1);
        tmem_ld16(lane_base + 128 + c0 + 48, pa1);
        proc_b(sa0, pa0, 2);
        tmem_ld_wait_regs(sa1, pa1);
        proc_b(sa1, pa1, 3);
      }
      tmem_st_wait();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&sm.pds_ready);
      // dO and Q block scales of this tile's q_block groups, used by the dV / dK read-out
      // (loaded here so that pass A hides their latency)
      float sdo_t[2], sq_t[2];
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        const size_t qb = static_cast<size_t>(bh) * nqb +
                          (qt * BQ + (g < G ? g : 0) * args.q_block) / args.q_block;
        sdo_t[g] = args.do_scale[qb];
        sq_t[g] = args.q_scale[qb];
      }
      // pass A of the next tile while the tensor core works on this one
      if (it + 1 < nq) pass_a(it + 1, c_n, lse2_n, dvr_n);
      // step 3: dV_t, dK_t (thread = key row r, d columns of warpgroup h) into registers.  The tile scales (P and dS absmax / 127,
      // IEEE quotients) come from the maxima of the key half this thread's key row is in.
      for (int g = 0; g < G; ++g) {
        const float sdo = g == 0 ? sdo_t[0] : sdo_t[1];
        const float sqg = g == 0 ? sq_t[0] : sq_t[1];
        const int kh = r >> 6;
        mbar_wait(&sm.dvdk_full, dvdk_cnt & 1, 211);
        tc_fence_after();
        // P / dS scales of this key row's half (IEEE quotients absmax / 127)
        const float sp = __fdiv_rn(tile_max(sm.red_p[b], g, kh), 127.0f);
        const float sds = __fdiv_rn(tile_max(sm.red_ds[b], g, kh), 127.0f);
        const float sv22 = scale22(sp * sdo);
        const float sk22 = scale22(sds * sqg * args.tau);
        const float nsv = __fmul_rn(-kMagic, sv22), nsk = __fmul_rn(-kMagic, sk22);
        const float2 sv2 = make_float2(sv22, sv22), nsv2 = make_float2(nsv, nsv);
        const float2 sk2 = make_float2(sk22, sk22), nsk2 = make_float2(nsk, nsk);
        // 16-column chunks; the loads of chunk c+1 are in flight while chunk c accumulates
        uint32_t tv0[16], tk0[16], tv1[16], tk1[16];
        tmem_ld16(lane_base + h * kHalfD, tv0);
        tmem_ld16(lane_base + 128 + h * kHalfD, tk0);
        tmem_ld_wait_regs(tv0, tk0);
#pragma unroll
        for (int c0 = 0; c0 < kHalfD; c0 += 16) {
          const int col = h * kHalfD + c0;
          const bool odd = (c0 / 16) & 1;
          if (c0 + 16 < kHalfD) {
            if (odd) {
              tmem_ld16(lane_base + col + 16, tv0);
              tmem_ld16(lane_base + 128 + col + 16, tk0);
            } else {
              tmem_ld16(lane_base + col + 16, tv1);
              tmem_ld16(lane_base + 128 + col + 16, tk1);
            }
          }
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            const uint32_t* tv = odd ? tv1 : tv0;
            const uint32_t* tk = odd ? tk1 : tk0;
            const float2 dv2 = __ffma2_rn(
                make_float2(__uint_as_float(tv[e]), __uint_as_float(tv[e + 1])), sv2, nsv2);
            const float2 dk2 = __ffma2_rn(
                make_float2(__uint_as_float(tk[e]), __uint_as_float(tk[e + 1])), sk2, nsk2);
            accv[(c0 + e) / 2] = __fadd2_rn(accv[(c0 + e) / 2], dv2);
            acck[(c0 + e) / 2] = __fadd2_rn(acck[(c0 + e) / 2], dk2);
          }
          if (c0 + 16 < kHalfD) {
            if (odd)
              tmem_ld_wait_regs(tv0, tk0);
            else
              tmem_ld_wait_regs(tv1, tk1);
          }
        }
        tc_fence_before();
        mbar_arrive(&sm.dvdk_free);
        ++dvdk_cnt;
      }
      // step 4: dQ, added to the float32 accumulator.  The dS scales of both key halves for this thread's dQ rows
      // are formed while the dQ MMAs run.
      const int gq = D == 128 ? (64 * h) / args.q_block : g_row;
      const float s0 = scale22(__fdiv_rn(tile_max(sm.red_ds[b], gq, 0), 127.0f) * sk0 * args.tau);
      const float s1 = scale22(__fdiv_rn(tile_max(sm.red_ds[b], gq, 1), 127.0f) * sk1 * args.tau);
      const float n0 = __fmul_rn(-kMagic, s0), n1 = __fmul_rn(-kMagic, s1);
      const float2 s02 = make_float2(s0, s0), n02 = make_float2(n0, n0);
      const float2 s12 = make_float2(s1, s1), n12 = make_float2(n1, n1);
      // and the next tile's code multipliers (its pass A is done in every warp by now)
      float ip_n = 0.0f, ids_n = 0.0f, sdsc_n = 0.0f;
      if (it + 1 < nq) multipliers(it + 1, ip_n, ids_n, sdsc_n);
      mbar_wait(&sm.dq_full, it & 1, 212);
      tc_fence_after();
      if constexpr (D == 128) {
        // thread = head-dim channel r, queries 64h .. 64h+63 of the tile (TMEM columns).
        // Each warp stages rounds of 16 queries x its 32 channels in its own shared-memory
        // buffers (double-buffered) and its lane 0 hands them to the TMA unit, which adds them
        // to the global accumulator; no warp waits for another.  The TMEM loads of round rr+1
        // are in flight while round rr is staged.
        uint32_t a0[16], a1[16];
        tmem_ld16(lane_base + 64 * h, a0);
        tmem_ld16(lane_base + 128 + 64 * h, a1);
        tmem_ld_wait_regs(a0, a1);
#pragma unroll
        for (int rr = 0; rr < 64 / kDqRows; ++rr) {
          const int q0 = 64 * h + kDqRows * rr;
          float2 v[kDqRows / 2];
#pragma unroll
          for (int e = 0; e < kDqRows; e += 2)
            v[e / 2] = __fadd2_rn(
                __ffma2_rn(make_float2(__uint_as_float(a0[e]), __uint_as_float(a0[e + 1])),
                           s02, n02),
                __ffma2_rn(make_float2(__uint_as_float(a1[e]), __uint_as_float(a1[e + 1])),
                           s12, n12));
          if (rr + 1 < 64 / kDqRows) {
            tmem_ld16(lane_base + q0 + kDqRows, a0);
            tmem_ld16(lane_base + 128 + q0 + kDqRows, a1);
          }
          float* stg = sm.dqs[warp][dq_round & 1];
          // the buffer's previous round (two rounds back) has been read by the TMA unit
          if (lane == 0) bulk_wait_read_1();
          __syncwarp();
#pragma unroll
          for (int e = 0; e < kDqRows; e += 2) {
            stg[e * kDqCols + lane] = v[e / 2].x;
            stg[(e + 1) * kDqCols + lane] = v[e / 2].y;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_reduce_add_2d(&tm_dq, stg, quarter * kDqCols, row_base + qt * BQ + q0);
            bulk_commit();
          }
          ++dq_round;
          if (rr + 1 < 64 / kDqRows) tmem_ld_wait_regs(a0, a1);
        }
      } else {
        // thread = query row r, the 32 channels of warpgroup h: staged in this warp's own box
        // (32 rows x 32 channels, 128-byte swizzle) and added to the global accumulator by the
        // TMA unit; the box's previous reduction has read it (a tile ago) before it is rewritten
        uint8_t* box = reinterpret_cast<uint8_t*>(&sm.dqs[warp][0][0]);
        if (lane == 0) bulk_wait_read_0();
        __syncwarp();
#pragma unroll
        for (int c0 = 0; c0 < kHalfD; c0 += 16) {
          uint32_t a0[16], a1[16];
          tmem_ld16(lane_base + h * kHalfD + c0, a0);
          tmem_ld16(lane_base + 128 + h * kHalfD + c0, a1);
          tmem_ld_wait_regs(a0, a1);
#pragma unroll
          for (int e = 0; e < 16; e += 4) {
            float4 v4;
            v4.x = deq(a0[e + 0], s0, n0) + deq(a1[e + 0], s1, n1);
            v4.y = deq(a0[e + 1], s0, n0) + deq(a1[e + 1], s1, n1);
            v4.z = deq(a0[e + 2], s0, n0) + deq(a1[e + 2], s1, n1);
            v4.w = deq(a0[e + 3], s0, n0) + deq(a1[e + 3], s1, n1);
            *reinterpret_cast<float4*>(box + swz_offset(lane, (c0 + e) / 4, 128)) = v4;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_2d(&tm_dq, box, h * kHalfD, row_base + qt * BQ + quarter * 32);
          bulk_commit();
        }
      }
      tc_fence_before();
      mbar_arrive(&sm.dq_free);
      ip = ip_n;
      ids = ids_n;
      sdsc = sdsc_n;
    }
    // epilogue: dv, dk from the register accumulators (thread = key row r, d half h)
    if (args.dk_acc != nullptr) {
      // partial over one query chunk: accumulate; the keys' owner applies the RMSNorm
      // backward once every chunk's contribution is in
      const size_t off = (static_cast<size_t>(row_base) + key_base + r) * D + h * kHalfD;
      float4* ka = reinterpret_cast<float4*>(args.dk_acc + off);
      float4* va = reinterpret_cast<float4*>(args.dv_acc + off);
#pragma unroll
      for (int c4 = 0; c4 < kHalfD / 4; ++c4) {
        float4 a = make_float4(0.0f, 0.0f, 0.0f, 0.0f), b = a;
        if (args.acc_add) {
          a = ka[c4];
          b = va[c4];
        }
        a.x += acck[2 * c4].x;
        a.y += acck[2 * c4].y;
        a.z += acck[2 * c4 + 1].x;
        a.w += acck[2 * c4 + 1].y;
        b.x += accv[2 * c4].x;
        b.y += accv[2 * c4].y;
        b.z += accv[2 * c4 + 1].x;
        b.w += accv[2 * c4 + 1].y;
        ka[c4] = a;
        va[c4] = b;
      }
    } else {
      const size_t krow = static_cast<size_t>(row_base) + key_base + r;
      T* dvp = reinterpret_cast<T*>(args.dv) + krow * D + h * kHalfD;
      T* dkp = reinterpret_cast<T*>(args.dk) + krow * D + h * kHalfD;
      if constexpr (QS) {
        // dK_bias = tau * (dS^T 1)_r * mu_Q, the gradient through the score bias
        named_barrier_sync(4, 256);  // every warp's column-sum additions are in
        const int kh = r >> 6;
        const float csr = (((sm.cs[kh * 4][r & 63] + sm.cs[kh * 4 + 1][r & 63]) +
                             sm.cs[kh * 4 + 2][r & 63]) + sm.cs[kh * 4 + 3][r & 63]) * args.tau;
        const float4* mq =
            reinterpret_cast<const float4*>(args.q_mean + static_cast<size_t>(bh) * D + h * kHalfD);
#pragma unroll
        for (int c0 = 0; c0 < kHalfD; c0 += 4) {
          const float4 m4 = __ldg(mq + c0 / 4);
          acck[c0 / 2].x = fmaf(csr, m4.x, acck[c0 / 2].x);
          acck[c0 / 2].y = fmaf(csr, m4.y, acck[c0 / 2].y);
          acck[c0 / 2 + 1].x = fmaf(csr, m4.z, acck[c0 / 2 + 1].x);
          acck[c0 / 2 + 1].y = fmaf(csr, m4.w, acck[c0 / 2 + 1].y);
        }
      }
      if (args.qknorm) {
        // RMSNorm backward: dk = inv * (dkhat - khat * (sum_c dkhat_c khat_c) / d), with
        // khat = k * inv recomputed from the raw row (bitwise the prologue's value)
        const float inv = args.k_inv_rms[krow];
        const T* kp = reinterpret_cast<const T*>(args.k_raw) + krow * D + h * kHalfD;
        float part = 0.0f;
#pragma unroll
        for (int c0 = 0; c0 < kHalfD; c0 += 8) {
          float x[8];
          Cvt<T>::load8(__ldg(reinterpret_cast<const uint4*>(kp + c0)), x);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float a = (e & 1) ? acck[(c0 + e) / 2].y : acck[(c0 + e) / 2].x;
            part = fmaf(a, __fmul_rn(x[e], inv), part);
          }
        }
        if (h == 1) sm.dot[r] = part;
        named_barrier_sync(3, 256);
        if (h == 0) sm.dot[r] += part;
        named_barrier_sync(3, 256);
        const float dotd = sm.dot[r] * (1.0f / D);
#pragma unroll
        for (int c0 = 0; c0 < kHalfD; c0 += 8) {
          float x[8];
          Cvt<T>::load8(__ldg(reinterpret_cast<const uint4*>(kp + c0)), x);
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            float2& a = acck[(c0 + e) / 2];
            a.x = inv * fmaf(-__fmul_rn(x[e], inv), dotd, a.x);
            a.y = inv * fmaf(-__fmul_rn(x[e + 1], inv), dotd, a.y);
          }
        }
      }
#pragma unroll
      for (int c0 = 0; c0 < kHalfD; c0 += 8) {
        float fv[8], fk[8];
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          fv[e] = accv[(c0 + e) / 2].x;
          fv[e + 1] = accv[(c0 + e) / 2].y;
          fk[e] = acck[(c0 + e) / 2].x;
          fk[e + 1] = acck[(c0 + e) / 2].y;
        }
        *reinterpret_cast<uint4*>(dvp + c0) = pack8<T>(fv);
        *reinterpret_cast<uint4*>(dkp + c0) = pack8<T>(fk);
      }
    }
    if (lane == 0) bulk_wait_all();  // this warp's dQ reductions complete
    tc_fence_before();
    named_barrier_sync(15, kThreads);
  }
}

}  // namespace bwd
}  // namespace sage
