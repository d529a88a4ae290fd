// nvfp4_bwd.cuh -- backward pass of the NVFP4 Q-Attn variant on sm_100a ("Full-Stack FP4",
// gist.science 2607.04422, section 2.4: dS runs in NVFP4, P^T dO and dO V^T in BF16; the
// quantized views of Q and K made by the prologue are reused).
//
// Per CTA: one tile of 128 keys of one (batch, head), walking the tiles of 128 queries that can
// see it (from the diagonal on when causal).  Per query tile:
//   1. S = Q K^T (kind::mxf4nvf4 from the forward's NVFP4 views: Q / K codes and block scales)
//      and dP = dO V^T (kind::f16 on the raw 16-bit dO and V) into TMEM, committed separately;
//   2. pass A (thread = query row, warpgroup h = keys 64h .. 64h+63): as soon as S lands,
//      P = exp2(S c - LSE log2 e) in the 16-bit type of dO / V into shared memory (the A operand
//      of dV += P^T dO, kind::f16, accumulated in TMEM over every query tile); once dP lands,
//      dS = P (dP - D) in registers, also written transposed to a float32 shared-memory tile;
//   3. the tile's absolute maximum of dS (every warp's maximum through shared memory) gives the
//      tile's global encode scale genc = 2688 / max, and a table of genc / e4m3(c) per scale
//      code c;
//   4. pass B: dS quantized twice with that global scale -- per query row in 16-key blocks
//      (the A operand of dQ_t = dS_k K_seq; its MMA starts while the second quantization runs)
//      and, from the transposed tile, per key row in 16-query blocks (the A operand of
//      dK_t = dS_q^T Q_seq): E2M1 codes in 64-byte swizzled rows and E4M3 block scales in the
//      tensor core's scale-factor order.  K_seq / Q_seq are the prologue's sequence views
//      (16-token blocks), multiplied by kind::mxf4nvf4;
//   5. read-outs: dQ_t * tau / (genc genc_K) is staged in shared memory (over the transposed
//      tile) and added to the float32 dQ accumulator in global memory by TMA reductions, which
//      run while the next tile starts; dK_t * tau / (genc genc_Q) goes to float32 registers.
//      The S / dQ_t and the dP / dK_t columns are released separately.
// After the last tile: dV from TMEM, dK (with the RMSNorm backward when qknorm) to global memory.
// The query tile's operands (Q codes and scales, dO, the Q sequence view) each have their own
// full / free barrier pair, so each is reloaded as soon as its last reader is done.
//
// Warps 0-7 compute, warp 8 is the TMA producer, warp 9 the MMA issuer, warps 10-11 idle (they
// complete the producer warpgroup, which gives registers to the compute warpgroups).
// TMEM (512 columns): S -> dQ_t at 0, dP -> dK_t at 128, dV at 256 (D columns), block scales
// from 384 (4 columns per 512-byte scale atom).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stddef.h>
#include <stdint.h>

#include <type_traits>

#include "nvfp4.cuh"
#include "ptx.cuh"
#include "rowops.cuh"

namespace sage {
namespace fp4 {
namespace bwd {

constexpr int BQ = 128;   // queries per tile
constexpr int BKT = 128;  // keys per CTA
constexpr int kThreads = 384;
constexpr int kCompute = 256;
constexpr int kProducerWarp = 8, kMmaWarp = 9;
constexpr int kLaunchRegs = 168, kComputeRegs = 216, kOtherRegs = 72;
static_assert(kCompute * kComputeRegs + (kThreads - kCompute) * kOtherRegs <=
                  kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");

// TMEM columns
constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColSf = 384;

template <typename T, int D>
struct Smem {
  alignas(1024) uint8_t kc[BKT * D / 2];  // K codes (B of S), resident
  alignas(1024) T v[BKT * D];             // V (B of dP), resident: D/64 boxes [128 keys][64 ch]
  alignas(1024) uint8_t ks[D * 64];       // K sequence view (B of dQ), resident: [D][64 bytes]
  alignas(1024) uint8_t qc[BQ * D / 2];   // Q codes (A of S), per query tile
  alignas(1024) T dor[BQ * D];            // dO (A of dP, B of dV): D/64 boxes [128 q][64 ch]
  alignas(1024) uint8_t qs[D * 64];       // Q sequence view (B of dK), per query tile
  alignas(1024) T p[BQ * BKT];            // P (A of dV, read MN-major): 2 atoms [128 q][64 keys]
  alignas(1024) uint8_t dsk[BQ * 64];     // dS in 16-key blocks (A of dQ): [128 q][64 bytes]
  alignas(1024) uint8_t dsq[BKT * 64];    // dS^T in 16-query blocks (A of dK): [128 keys][64 B]
  alignas(128) uint8_t ksf[D / 64 * 512];
  alignas(128) uint8_t kssf[2 * 512];
  alignas(128) uint8_t qsf[D / 64 * 512];
  alignas(128) uint8_t qssf[2 * 512];
  alignas(128) uint8_t dsksf[2 * 512];
  alignas(128) uint8_t dsqsf[2 * 512];
  // dS transposed, [key][query]; rows padded to 132 floats: the column writes of pass A and
  // the 16-byte row reads of pass B are both conflict-free.  After pass B the same bytes stage
  // the tile's dQ for the TMA reductions: per compute warp D/64 boxes of 32 query rows x 32
  // channels (4 KB, 128-byte swizzle)
  alignas(1024) float dst[BKT][BQ + 4];
  alignas(16) float red[2][8];  // per-warp max |dS|, [tile parity][warp]
  float mult[128];              // the tile's genc / E4M3 value, by scale code
  float dot[BKT];               // RMSNorm-backward row dot products (warpgroup 1 -> 0)
  uint64_t kv_full;
  // S and dP landed; P written; dS codes written (16-key blocks, 16-query blocks); dQ_t and
  // dK_t landed; the S / dQ_t and the dP / dK_t columns read out
  uint64_t s_full, dp_full, p_ready, dsk_ready, dsq_ready, dq_full, dk_full, s_free, dp_free;
  // the query tile's operands, each loaded as soon as its last reader of the previous tile
  // has completed: Q codes and scales (S), dO (dP, dV), the Q sequence view (dK)
  uint64_t q_full, q_free, do_full, do_free, qs_full, qs_free;
  uint64_t red_full[2];
  uint64_t stage_free;  // the previous tile's dQ reductions have read the staging boxes
  uint32_t tmem_base;
  int abort;
};

template <typename T, int D>
constexpr size_t smem_bytes() {
  return sizeof(Smem<T, D>) + 1024;
}
static_assert(smem_bytes<__nv_bfloat16, 128>() <= 232448, "shared memory exceeds the limit");

template <typename T, int D>
__device__ __forceinline__ Smem<T, D>& smem_ref(uint8_t* raw) {
  const uint32_t a = smem_u32(raw);
  return *reinterpret_cast<Smem<T, D>*>(raw + ((1024u - (a & 1023u)) & 1023u));
}

struct Args {
  const uint8_t* q_sf;    // [BH, N/128, D/64, 512]
  const uint8_t* k_sf;
  const uint8_t* q_sf_t;  // [BH, 1, N/64, 512]
  const uint8_t* k_sf_t;
  const float* q_genc;    // [BH]
  const float* k_genc;
  const float* lse;       // [BH, N]
  const float* dvec;      // [BH, N]
  const void* k_raw;      // [BH, N, D] (RMSNorm backward of dk)
  const float* k_inv_rms; // [BH, N]
  void* dk;
  void* dv;
  int N, causal, qknorm;
  float scale_log2;  // softmax_scale * log2(e)
  float tau;         // softmax_scale
};

// Eight E2M1 codes of values already multiplied by their block's encode factor: element 2i
// in the low nibble of byte i (hardware conversion: nearest, ties to even, saturating at 6).
__device__ __forceinline__ uint32_t e2m1x8(float2 a, float2 b, float2 c, float2 d) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y), "f"(d.x), "f"(d.y));
  return r;
}

// Four consecutive 16-element blocks of x quantized to NVFP4 with the global encode scale genc
// (the prologue's float32 steps: u = (max|x| genc) / 6, sd = e4m3(u), code = e2m1(x genc / sd)),
// in four independent chains (the scale codes first, then the multipliers, then the codes).
// mult_tab[c] = genc / e4m3_value(c) (0 for c = 0), made once per tile.  codes[b] holds block
// b's 8 code bytes (element 2i in the low nibble of byte i); the return value holds the four
// E4M3 scale bytes (block b in byte b).
__device__ __forceinline__ uint32_t quant_blocks4(const float (&x)[64], float genc,
                                                  const float* mult_tab, uint2 (&codes)[4]) {
  uint32_t sc[4];
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    float am = 0.0f;
#pragma unroll
    for (int e = 0; e < 16; e += 2) am = fmax3(am, fabsf(x[16 * b + e]), fabsf(x[16 * b + e + 1]));
    sc[b] = e4m3_code(div6_rn(__fmul_rn(am, genc)));
  }
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    const float mult = mult_tab[sc[b]];
    const float2 m2 = make_float2(mult, mult);
    float2 y[8];
#pragma unroll
    for (int e = 0; e < 8; ++e)
      y[e] = __fmul2_rn(make_float2(x[16 * b + 2 * e], x[16 * b + 2 * e + 1]), m2);
    codes[b] = make_uint2(e2m1x8(y[0], y[1], y[2], y[3]), e2m1x8(y[4], y[5], y[6], y[7]));
  }
  return sc[0] | (sc[1] << 8) | (sc[2] << 16) | (sc[3] << 24);
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_qc,
                    const __grid_constant__ CUtensorMap tm_kc,
                    const __grid_constant__ CUtensorMap tm_qs,
                    const __grid_constant__ CUtensorMap tm_ks,
                    const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_dq, Args args) {
  static_assert(D == 64 || D == 128, "head dimension");
  static_assert(sizeof(float) * BKT * (BQ + 4) >= 8 * (D / 64) * 4096, "dQ staging space");
  constexpr int DH = D / 2;
  constexpr uint32_t kSfBytes = D / 64 * 512;
  constexpr uint32_t kSwC = (D == 128) ? kSwizzle64B : kSwizzle32B;  // Q / K code tiles
  constexpr uint32_t kSboC = 8 * (D / 2);
  extern __shared__ uint8_t smem_raw[];
  Smem<T, D>& sm = smem_ref<T, D>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = args.N, nkt = N / BKT, nqt = N / BQ;
  // head-major order; within a head the key tile with the most query tiles first (causal)
  const int bh = blockIdx.x / nkt;
  const int t = blockIdx.x % nkt;
  const int i_first = args.causal ? t : 0;
  const int nq = nqt - i_first;
  // sequence-view scale atoms: [BH][1 channel group][N / 64][512]
  const size_t seq_atoms = static_cast<size_t>(bh) * (N / 64);

  if (threadIdx.x == 0) {
    sm.abort = device_aborted() ? 1 : 0;
    mbar_init(&sm.kv_full, 1);
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_free, 1);
    mbar_init(&sm.do_full, 1);
    mbar_init(&sm.do_free, 1);
    mbar_init(&sm.qs_full, 1);
    mbar_init(&sm.qs_free, 1);
    mbar_init(&sm.s_full, 1);
    mbar_init(&sm.dp_full, 1);
    mbar_init(&sm.p_ready, kCompute);
    mbar_init(&sm.dsk_ready, kCompute);
    mbar_init(&sm.dsq_ready, kCompute);
    mbar_init(&sm.dq_full, 1);
    mbar_init(&sm.dk_full, 1);
    mbar_init(&sm.s_free, kCompute);
    mbar_init(&sm.dp_free, kCompute);
    mbar_init(&sm.red_full[0], 8);
    mbar_init(&sm.red_full[1], 8);
    mbar_init(&sm.stage_free, 8);
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
  const int row_base = bh * N;
  const uint32_t sf_q = tmem + kColSf, sf_k = sf_q + 4 * (D / 64);
  const uint32_t sf_dsk = sf_k + 4 * (D / 64), sf_kseq = sf_dsk + 8;
  const uint32_t sf_dsq = sf_kseq + 8, sf_qseq = sf_dsq + 8;

  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kOtherRegs));
    if (warp == kProducerWarp && lane == 0) {
      tma_prefetch_desc(&tm_qc);
      tma_prefetch_desc(&tm_kc);
      tma_prefetch_desc(&tm_qs);
      tma_prefetch_desc(&tm_ks);
      tma_prefetch_desc(&tm_do);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_dq);
      // resident: K codes and scales, V, the K sequence view and its scales
      mbar_arrive_expect_tx(&sm.kv_full, BKT * D / 2 + kSfBytes + BKT * D * 2 + D * 64 + 1024);
      tma_load_2d(sm.kc, &tm_kc, 0, row_base + t * BKT, &sm.kv_full);
      bulk_load(sm.ksf, args.k_sf + (static_cast<size_t>(bh) * nkt + t) * kSfBytes, kSfBytes,
                &sm.kv_full);
      for (int a = 0; a < D / 64; ++a)
        tma_load_2d(sm.v + a * BKT * 64, &tm_v, a * 64, row_base + t * BKT, &sm.kv_full);
      tma_load_2d(sm.ks, &tm_ks, t * 64, bh * D, &sm.kv_full);
      bulk_load(sm.kssf, args.k_sf_t + (seq_atoms + 2 * t) * 512, 1024, &sm.kv_full);
      for (int it = 0; it < nq; ++it) {
        const int qt = i_first + it;
        if (it >= 1) mbar_wait(&sm.q_free, (it - 1) & 1, 400);
        mbar_arrive_expect_tx(&sm.q_full, BQ * D / 2 + kSfBytes);
        tma_load_2d(sm.qc, &tm_qc, 0, row_base + qt * BQ, &sm.q_full);
        bulk_load(sm.qsf, args.q_sf + (static_cast<size_t>(bh) * nqt + qt) * kSfBytes, kSfBytes,
                  &sm.q_full);
        if (it >= 1) mbar_wait(&sm.do_free, (it - 1) & 1, 406);
        mbar_arrive_expect_tx(&sm.do_full, BQ * D * 2);
        for (int a = 0; a < D / 64; ++a)
          tma_load_2d(sm.dor + a * BQ * 64, &tm_do, a * 64, row_base + qt * BQ, &sm.do_full);
        if (it >= 1) mbar_wait(&sm.qs_free, (it - 1) & 1, 407);
        mbar_arrive_expect_tx(&sm.qs_full, D * 64 + 1024);
        tma_load_2d(sm.qs, &tm_qs, qt * 64, bh * D, &sm.qs_full);
        bulk_load(sm.qssf, args.q_sf_t + (seq_atoms + 2 * qt) * 512, 1024, &sm.qs_full);
      }
    } else if (warp == kMmaWarp && lane == 0) {
      constexpr uint32_t kFmt = std::is_same<T, __nv_bfloat16>::value ? 1u : 0u;
      const uint32_t id_s = instr_desc_nvf4(BQ, BKT);
      const uint32_t id_dp = instr_desc(1, kFmt, kFmt, false, false, BQ, BKT);
      const uint32_t id_dv = instr_desc(1, kFmt, kFmt, true, true, BKT, D);
      const uint32_t id_g = instr_desc_nvf4(128, D);  // dQ_t and dK_t
      const uint32_t kca = smem_u32(sm.kc), va = smem_u32(sm.v), ksa = smem_u32(sm.ks);
      const uint32_t qca = smem_u32(sm.qc), dora = smem_u32(sm.dor), qsa = smem_u32(sm.qs);
      const uint32_t pa = smem_u32(sm.p), dska = smem_u32(sm.dsk), dsqa = smem_u32(sm.dsq);
      auto cp_atoms = [&](uint32_t col, const uint8_t* src, int n) {
        for (int a = 0; a < n; ++a)
          tmem_cp_sf(col + 4 * a, smem_desc(smem_u32(src) + 512 * a, 128, 128, kSwizzleNone));
      };
      mbar_wait(&sm.kv_full, 0, 401);
      tc_fence_after();
      cp_atoms(sf_k, sm.ksf, D / 64);
      cp_atoms(sf_kseq, sm.kssf, 2);
      for (int it = 0; it < nq; ++it) {
        // 1. S = Q K^T (NVFP4) into columns the previous tile's dQ_t has been read out of
        mbar_wait(&sm.q_full, it & 1, 402);
        if (it >= 1) mbar_wait(&sm.s_free, (it - 1) & 1, 403);
        tc_fence_after();
        cp_atoms(sf_q, sm.qsf, D / 64);
#pragma unroll
        for (int kk = 0; kk < D / 64; ++kk)
          mma_nvf4(tmem + kColS, smem_desc(qca + 32 * kk, 16, kSboC, kSwC),
                   smem_desc(kca + 32 * kk, 16, kSboC, kSwC), id_s, sf_q + 4 * kk,
                   sf_k + 4 * kk, kk > 0 ? 1u : 0u);
        mma_commit(&sm.s_full);
        mma_commit(&sm.q_free);  // the Q codes and scales have been read
        // 2. dP = dO V^T (16-bit) into columns the previous tile's dK_t has been read out of
        mbar_wait(&sm.do_full, it & 1, 408);
        if (it >= 1) mbar_wait(&sm.dp_free, (it - 1) & 1, 414);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk * 16 / 64) * (BQ * 128) + (kk * 16 % 64) * 2;
          mma_f16(tmem + kColDP, smem_desc(dora + off, 16, 1024, kSwizzle128B),
                  smem_desc(va + off, 16, 1024, kSwizzle128B), id_dp, kk > 0 ? 1u : 0u);
        }
        mma_commit(&sm.dp_full);
        // 3. dV += P^T dO: A = P read MN-major (M = keys), B = dO read MN-major (N = channels)
        mbar_wait(&sm.p_ready, it & 1, 404);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BQ / 16; ++kk)
          mma_f16(tmem + kColDV, smem_desc(pa + kk * 16 * 128, BQ * 128, 1024, kSwizzle128B),
                  smem_desc(dora + kk * 16 * 128, BQ * 128, 1024, kSwizzle128B), id_dv,
                  (it > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&sm.do_free);  // dP and dV have read dO
        // 4. dQ_t = dS_k K_seq into S's columns (S has been read: pass A precedes pass B)
        mbar_wait(&sm.dsk_ready, it & 1, 405);
        tc_fence_after();
        cp_atoms(sf_dsk, sm.dsksf, 2);
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
          mma_nvf4(tmem + kColS, smem_desc(dska + 32 * kk, 16, 512, kSwizzle64B),
                   smem_desc(ksa + 32 * kk, 16, 512, kSwizzle64B), id_g, sf_dsk + 4 * kk,
                   sf_kseq + 4 * kk, kk > 0 ? 1u : 0u);
        mma_commit(&sm.dq_full);
        // 5. dK_t = dS_q^T Q_seq into dP's columns
        mbar_wait(&sm.qs_full, it & 1, 409);
        tc_fence_after();
        cp_atoms(sf_qseq, sm.qssf, 2);
        mbar_wait(&sm.dsq_ready, it & 1, 415);
        tc_fence_after();
        cp_atoms(sf_dsq, sm.dsqsf, 2);
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
          mma_nvf4(tmem + kColDP, smem_desc(dsqa + 32 * kk, 16, 512, kSwizzle64B),
                   smem_desc(qsa + 32 * kk, 16, 512, kSwizzle64B), id_g, sf_dsq + 4 * kk,
                   sf_qseq + 4 * kk, kk > 0 ? 1u : 0u);
        mma_commit(&sm.dk_full);
        mma_commit(&sm.qs_free);  // dK has read the Q sequence view
      }
    }
    __syncwarp();
    tc_fence_before();
    named_barrier_sync(15, kThreads);
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kComputeRegs));
    // ---------------- compute warps ----------------
    const int h = warp >> 2, quarter = warp & 3;
    const int r = quarter * 32 + lane;  // TMEM lane: query row (S, dP, dQ_t) / key row (dK_t, dV)
    const uint32_t lane_base = tmem + ((quarter * 32u) << 16);
    const float qg = args.q_genc[bh], kg = args.k_genc[bh];
    const float c = __fdiv_rn(args.scale_log2, qg * kg);  // the forward's score scale
    float acck[DH];
#pragma unroll
    for (int e = 0; e < DH; ++e) acck[e] = 0.0f;

    // this row's LSE and D, loaded one tile ahead
    size_t grow_n = static_cast<size_t>(row_base) + i_first * BQ + r;
    float lse_n = args.lse[grow_n], dvr_n = args.dvec[grow_n];
    for (int it = 0; it < nq; ++it) {
      const int qt = i_first + it;
      const int b = it & 1;
      const float lse2 = lse_n * 1.4426950408889634f;
      const float dvr = dvr_n;
      if (it + 1 < nq) {
        grow_n += BQ;
        lse_n = args.lse[grow_n];
        dvr_n = args.dvec[grow_n];
      }
      const bool diag = args.causal && qt == t;
      // pass A (thread = query row r, warpgroup h = keys 64h .. 64h + 63), first P from S (the
      // dP MMA runs meanwhile), then dS from dP
      float ds[64];
      float dsmax = 0.0f;
      uint8_t* patom = reinterpret_cast<uint8_t*>(sm.p) + h * (BQ * 128);
      const float2 c2 = make_float2(c, c), nlse2 = make_float2(-lse2, -lse2);
      const float2 ndvr2 = make_float2(-dvr, -dvr);
      mbar_wait(&sm.s_full, it & 1, 410);
      tc_fence_after();
#pragma unroll
      for (int c32 = 0; c32 < 2; ++c32) {
        const int col = h * 64 + c32 * 32;
        uint32_t s0[16], s1[16];
        tmem_ld32x(lane_base + kColS + col, s0, s1);
        tmem_ld_wait_regs(s0, s1);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const uint32_t(&sx)[16] = half ? s1 : s0;
          const int cc = col + half * 16;  // first key of these 16 columns
          uint32_t w[8];
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            const float2 z = __ffma2_rn(make_float2(__uint_as_float(sx[e]), __uint_as_float(sx[e + 1])),
                                        c2, nlse2);
            // one pair in four on the FMA pipe (exp2_poly2), the rest on the MUFU unit
            float p0, p1;
            if ((e & 6) == 6) {
              const float2 p = exp2_poly2(z);
              p0 = p.x;
              p1 = p.y;
            } else {
              p0 = ex2_approx(z.x);
              p1 = ex2_approx(z.y);
            }
            if (diag && cc + e > r) p0 = 0.0f;  // key index - query index = cc + e - r
            if (diag && cc + e + 1 > r) p1 = 0.0f;
            const int j = c32 * 32 + half * 16 + e;
            ds[j] = p0;
            ds[j + 1] = p1;
            w[e / 2] = Cvt<T>::pack2(p0, p1);
          }
          // keys cc .. cc+15 are 16-byte chunks 2 c16 and 2 c16 + 1 of this row's atom
          const int c16 = c32 * 2 + half;
          *reinterpret_cast<uint4*>(patom + swz_offset(r, 2 * c16, 128)) =
              make_uint4(w[0], w[1], w[2], w[3]);
          *reinterpret_cast<uint4*>(patom + swz_offset(r, 2 * c16 + 1, 128)) =
              make_uint4(w[4], w[5], w[6], w[7]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&sm.p_ready);
      mbar_wait(&sm.dp_full, it & 1, 416);
      tc_fence_after();
#pragma unroll
      for (int c32 = 0; c32 < 2; ++c32) {
        uint32_t q0[16], q1[16];
        tmem_ld32x(lane_base + kColDP + h * 64 + c32 * 32, q0, q1);
        tmem_ld_wait_regs(q0, q1);
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const uint32_t(&px)[16] = e < 16 ? q0 : q1;
          const int j = c32 * 32 + e;
          const float2 d = __fmul2_rn(
              make_float2(ds[j], ds[j + 1]),
              __fadd2_rn(make_float2(__uint_as_float(px[e & 15]), __uint_as_float(px[(e & 15) + 1])),
                         ndvr2));
          ds[j] = d.x;
          ds[j + 1] = d.y;
          dsmax = fmax3(dsmax, fabsf(d.x), fabsf(d.y));
        }
      }
      // dS transposed into shared memory, once the previous tile's dQ reductions have read
      // the same bytes
      if (it >= 1) {
        if (lane == 0) {
          bulk_wait_read_0();
          mbar_arrive(&sm.stage_free);
        }
        mbar_wait(&sm.stage_free, (it - 1) & 1, 413);
      }
#pragma unroll
      for (int j = 0; j < 64; ++j) sm.dst[h * 64 + j][r] = ds[j];
      dsmax = warp_max(dsmax);
      __syncwarp();  // this warp's transposed dS writes precede lane 0's arrival
      if (lane == 0) {
        sm.red[b][warp] = dsmax;
        mbar_arrive(&sm.red_full[b]);
      }
      mbar_wait(&sm.red_full[b], (it >> 1) & 1, 411);
      float tmax = 0.0f;
#pragma unroll
      for (int w8 = 0; w8 < 8; ++w8) tmax = fmaxf(tmax, sm.red[b][w8]);
      const float genc = tmax > 0.0f ? __fdiv_rn(kGlobalRange, tmax) : 1.0f;
      if (threadIdx.x < 128) {
        const uint32_t code = threadIdx.x;
        sm.mult[code] = code == 0 ? 0.0f : __fdiv_rn(genc, e4m3_value(code));
      }
      named_barrier_sync(2, kCompute);
      // pass B (1): dS in 16-key blocks along this query row -> A of dQ (the dQ MMA then runs
      // during pass B (2)); the row's four scales of this key half are one 32-bit word
      {
        uint2 cd[4];
        const uint32_t scw = quant_blocks4(ds, genc, sm.mult, cd);
        *reinterpret_cast<uint4*>(sm.dsk + swz_offset(r, 2 * h, 64)) =
            make_uint4(cd[0].x, cd[0].y, cd[1].x, cd[1].y);
        *reinterpret_cast<uint4*>(sm.dsk + swz_offset(r, 2 * h + 1, 64)) =
            make_uint4(cd[2].x, cd[2].y, cd[3].x, cd[3].y);
        *reinterpret_cast<uint32_t*>(sm.dsksf + h * 512 + (r & 31) * 16 + (r >> 5) * 4) = scw;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&sm.dsk_ready);
      // pass B (2): dS^T in 16-query blocks along key row k = threadIdx % 128 (queries
      // 64 qh .. 64 qh + 63, read back from the transposed tile) -> A of dK
      {
        const int k = threadIdx.x & 127, qh = threadIdx.x >> 7;
        float y[64];
        const float4* row = reinterpret_cast<const float4*>(&sm.dst[k][qh * 64]);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float4 f4 = row[e];
          y[4 * e] = f4.x;
          y[4 * e + 1] = f4.y;
          y[4 * e + 2] = f4.z;
          y[4 * e + 3] = f4.w;
        }
        uint2 cd[4];
        const uint32_t scw = quant_blocks4(y, genc, sm.mult, cd);
        *reinterpret_cast<uint4*>(sm.dsq + swz_offset(k, 2 * qh, 64)) =
            make_uint4(cd[0].x, cd[0].y, cd[1].x, cd[1].y);
        *reinterpret_cast<uint4*>(sm.dsq + swz_offset(k, 2 * qh + 1, 64)) =
            make_uint4(cd[2].x, cd[2].y, cd[3].x, cd[3].y);
        *reinterpret_cast<uint32_t*>(sm.dsqsf + qh * 512 + (k & 31) * 16 + (k >> 5) * 4) = scw;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&sm.dsq_ready);
      // read-outs.  dQ_t (lane = query row): scaled into this warp's staging boxes; the S / dQ_t
      // columns are then released (the next tile's S MMA starts) and one lane hands the boxes
      // to the TMA unit, which adds them into the float32 dQ accumulator
      const float sq = __fdiv_rn(args.tau, __fmul_rn(genc, kg));
      const float sk = __fdiv_rn(args.tau, __fmul_rn(genc, qg));
      uint8_t* stage = reinterpret_cast<uint8_t*>(&sm.dst[0][0]) + warp * (D / 64) * 4096;
      // the staging boxes overlay the transposed tile: every thread's pass B (2) has read it
      mbar_wait(&sm.dsq_ready, it & 1, 418);
      mbar_wait(&sm.dq_full, it & 1, 412);
      tc_fence_after();
#pragma unroll
      for (int c0 = 0; c0 < DH; c0 += 32) {
        uint32_t a0[16], a1[16];
        tmem_ld32x(lane_base + kColS + h * DH + c0, a0, a1);
        tmem_ld_wait_regs(a0, a1);
        uint8_t* box = stage + (c0 / 32) * 4096;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint32_t(&a)[16] = ch < 4 ? a0 : a1;
          const int e = (ch & 3) * 4;
          *reinterpret_cast<float4*>(box + swz_offset(lane, ch, 128)) =
              make_float4(__uint_as_float(a[e]) * sq, __uint_as_float(a[e + 1]) * sq,
                          __uint_as_float(a[e + 2]) * sq, __uint_as_float(a[e + 3]) * sq);
        }
      }
      tc_fence_before();
      mbar_arrive(&sm.s_free);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
#pragma unroll
        for (int j = 0; j < D / 64; ++j)
          tma_reduce_add_2d(&tm_dq, stage + j * 4096, h * DH + 32 * j,
                            row_base + qt * BQ + quarter * 32);
        bulk_commit();
      }
      // dK_t (lane = key row) into the accumulators; then the dP / dK_t columns are released
      mbar_wait(&sm.dk_full, it & 1, 417);
      tc_fence_after();
#pragma unroll
      for (int c0 = 0; c0 < DH; c0 += 32) {
        uint32_t k0[16], k1[16];
        tmem_ld32x(lane_base + kColDP + h * DH + c0, k0, k1);
        tmem_ld_wait_regs(k0, k1);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          acck[c0 + e] = fmaf(__uint_as_float(k0[e]), sk, acck[c0 + e]);
          acck[c0 + 16 + e] = fmaf(__uint_as_float(k1[e]), sk, acck[c0 + 16 + e]);
        }
      }
      tc_fence_before();
      mbar_arrive(&sm.dp_free);
    }
    if (lane == 0) bulk_wait_all();  // this warp's dQ reductions have completed
    // epilogue: dV from TMEM, dK from the registers (thread = key row r, channels h*D/2 ..);
    // every dV MMA has completed: the last tile's dK/dQ commit follows them
    {
      const size_t krow = static_cast<size_t>(row_base) + t * BKT + r;
      T* dvp = reinterpret_cast<T*>(args.dv) + krow * D + h * DH;
      T* dkp = reinterpret_cast<T*>(args.dk) + krow * D + h * DH;
#pragma unroll
      for (int c0 = 0; c0 < DH; c0 += 16) {
        uint32_t x[16];
        tmem_ld16(lane_base + kColDV + h * DH + c0, x);
        tmem_ld_wait();
        float f[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) f[e] = __uint_as_float(x[e]);
        *reinterpret_cast<uint4*>(dvp + c0) = pack8<T>(*reinterpret_cast<float(*)[8]>(f));
        *reinterpret_cast<uint4*>(dvp + c0 + 8) = pack8<T>(*reinterpret_cast<float(*)[8]>(f + 8));
      }
      if (args.qknorm) {
        // RMSNorm backward: dk = inv * (dkhat - khat * (sum_c dkhat_c khat_c) / d), with
        // khat = k * inv recomputed from the raw row (bitwise the prologue's value)
        const float inv = args.k_inv_rms[krow];
        const T* kp = reinterpret_cast<const T*>(args.k_raw) + krow * D + h * DH;
        float part = 0.0f;
#pragma unroll
        for (int c0 = 0; c0 < DH; c0 += 8) {
          float x[8];
          Cvt<T>::load8(__ldg(reinterpret_cast<const uint4*>(kp + c0)), x);
#pragma unroll
          for (int e = 0; e < 8; ++e) part = fmaf(acck[c0 + e], __fmul_rn(x[e], inv), part);
        }
        if (h == 1) sm.dot[r] = part;
        named_barrier_sync(3, kCompute);
        if (h == 0) sm.dot[r] += part;
        named_barrier_sync(3, kCompute);
        const float dotd = sm.dot[r] * (1.0f / D);
#pragma unroll
        for (int c0 = 0; c0 < DH; c0 += 8) {
          float x[8];
          Cvt<T>::load8(__ldg(reinterpret_cast<const uint4*>(kp + c0)), x);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            acck[c0 + e] = inv * fmaf(-__fmul_rn(x[e], inv), dotd, acck[c0 + e]);
        }
      }
#pragma unroll
      for (int c0 = 0; c0 < DH; c0 += 8) {
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = acck[c0 + e];
        *reinterpret_cast<uint4*>(dkp + c0) = pack8<T>(f);
      }
    }
    tc_fence_before();
    named_barrier_sync(15, kThreads);
  }
}

}  // namespace bwd
}  // namespace fp4
}  // namespace sage
