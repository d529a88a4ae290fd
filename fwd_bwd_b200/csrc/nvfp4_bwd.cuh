// nvfp4_bwd.cuh -- backward pass of the NVFP4 Q-Attn variant on sm_100a ("Full-Stack FP4",
// gist.science 2607.04422, section 2.4: dS runs in NVFP4, P^T dO and dO V^T in BF16; the
// quantized views of Q and K made by the prologue are reused).
//
// Per CTA: one tile of 128 keys of one (batch, head), walking the tiles of 128 queries that can
// see it.  Per query tile:
//   1. S = Q K^T (kind::mxf4nvf4 from the forward's NVFP4 views: Q / K codes and block scales)
//      and dP = dO V^T (kind::f16 on the raw 16-bit dO and V) into TMEM;
//   2. pass A (thread = query row, warpgroup h = keys 64h .. 64h+63): P = exp2(S c - LSE log2 e),
//      dS = P (dP - D); P in the 16-bit type of dO / V goes to shared memory as the A operand of
//      dV += P^T dO (kind::f16, accumulated in TMEM over every query tile); dS stays in
//      registers and is also written, transposed, to a float32 shared-memory tile;
//   3. the tile's absolute maximum of dS (every warp's maximum through shared memory) gives the
//      tile's global encode scale genc = 2688 / max;
//   4. pass B: dS quantized twice with that global scale -- per query row in 16-key blocks
//      (the A operand of dQ = dS K) and, from the transposed tile, per key row in 16-query
//      blocks (the A operand of dK = dS^T Q): E2M1 codes in 64-byte swizzled rows and E4M3
//      block scales in the tensor core's scale-factor order;
//   5. dQ_t = dS_k K_seq and dK_t = dS_q^T Q_seq (kind::mxf4nvf4; K_seq / Q_seq are the
//      prologue's sequence views, 16-token blocks) into TMEM; dQ_t * tau / (genc genc_K) is
//      added to the float32 dQ accumulator in global memory, dK_t * tau / (genc genc_Q) to
//      float32 registers.
// After the last tile: dV from TMEM, dK (with the RMSNorm backward when qknorm) to global memory.
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
  float dst[BKT][BQ + 1];  // dS transposed, [key][query] (padded: conflict-free columns)
  alignas(16) float red[2][8];  // per-warp max |dS|, [tile parity][warp]
  float dot[BKT];               // RMSNorm-backward row dot products (warpgroup 1 -> 0)
  uint64_t kv_full, st_full, st_free, sdp_full, p_ready, ds_ready, dkdq_full, tmem_free;
  uint64_t red_full[2];
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
  float* dq_acc;          // [BH, N, D] float32
  void* dk;
  void* dv;
  int N, causal, qknorm;
  float scale_log2;  // softmax_scale * log2(e)
  float tau;         // softmax_scale
};

// Quantizes one 16-element block to NVFP4 with global encode scale genc (the prologue's
// float32 steps): returns the 8 code bytes (element 2i in the low nibble of byte i) and the
// E4M3 scale byte.
__device__ __forceinline__ uint2 quant_block16(const float (&x)[16], float genc, uint32_t& sc) {
  float am = 0.0f;
#pragma unroll
  for (int e = 0; e < 16; ++e) am = fmaxf(am, fabsf(x[e]));
  const float u = __fdiv_rn(__fmul_rn(am, genc), 6.0f);
  sc = e4m3_code(u);
  const float sd = e4m3_value(sc);
  const float mult = sd > 0.0f ? __fdiv_rn(genc, sd) : 0.0f;
  uint32_t w0 = 0, w1 = 0;
#pragma unroll
  for (int e = 0; e < 8; e += 2) {
    w0 |= e2m1x2(__fmul_rn(x[e], mult), __fmul_rn(x[e + 1], mult)) << (4 * e);
    w1 |= e2m1x2(__fmul_rn(x[8 + e], mult), __fmul_rn(x[9 + e], mult)) << (4 * e);
  }
  return make_uint2(w0, w1);
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_qc,
                    const __grid_constant__ CUtensorMap tm_kc,
                    const __grid_constant__ CUtensorMap tm_qs,
                    const __grid_constant__ CUtensorMap tm_ks,
                    const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_v, Args args) {
  static_assert(D == 64 || D == 128, "head dimension");
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
    mbar_init(&sm.st_full, 1);
    mbar_init(&sm.st_free, 1);
    mbar_init(&sm.sdp_full, 1);
    mbar_init(&sm.p_ready, kCompute);
    mbar_init(&sm.ds_ready, kCompute);
    mbar_init(&sm.dkdq_full, 1);
    mbar_init(&sm.tmem_free, kCompute);
    mbar_init(&sm.red_full[0], 8);
    mbar_init(&sm.red_full[1], 8);
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
        if (it >= 1) mbar_wait(&sm.st_free, (it - 1) & 1, 400);
        mbar_arrive_expect_tx(&sm.st_full, BQ * D / 2 + kSfBytes + BQ * D * 2 + D * 64 + 1024);
        tma_load_2d(sm.qc, &tm_qc, 0, row_base + qt * BQ, &sm.st_full);
        bulk_load(sm.qsf, args.q_sf + (static_cast<size_t>(bh) * nqt + qt) * kSfBytes, kSfBytes,
                  &sm.st_full);
        for (int a = 0; a < D / 64; ++a)
          tma_load_2d(sm.dor + a * BQ * 64, &tm_do, a * 64, row_base + qt * BQ, &sm.st_full);
        tma_load_2d(sm.qs, &tm_qs, qt * 64, bh * D, &sm.st_full);
        bulk_load(sm.qssf, args.q_sf_t + (seq_atoms + 2 * qt) * 512, 1024, &sm.st_full);
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
        mbar_wait(&sm.st_full, it & 1, 402);
        if (it >= 1) mbar_wait(&sm.tmem_free, (it - 1) & 1, 403);
        tc_fence_after();
        // 1. S = Q K^T (NVFP4) and dP = dO V^T (16-bit)
        cp_atoms(sf_q, sm.qsf, D / 64);
#pragma unroll
        for (int kk = 0; kk < D / 64; ++kk)
          mma_nvf4(tmem + kColS, smem_desc(qca + 32 * kk, 16, kSboC, kSwC),
                   smem_desc(kca + 32 * kk, 16, kSboC, kSwC), id_s, sf_q + 4 * kk,
                   sf_k + 4 * kk, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk * 16 / 64) * (BQ * 128) + (kk * 16 % 64) * 2;
          mma_f16(tmem + kColDP, smem_desc(dora + off, 16, 1024, kSwizzle128B),
                  smem_desc(va + off, 16, 1024, kSwizzle128B), id_dp, kk > 0 ? 1u : 0u);
        }
        mma_commit(&sm.sdp_full);
        // 2. dV += P^T dO: A = P read MN-major (M = keys), B = dO read MN-major (N = channels)
        mbar_wait(&sm.p_ready, it & 1, 404);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BQ / 16; ++kk)
          mma_f16(tmem + kColDV, smem_desc(pa + kk * 16 * 128, BQ * 128, 1024, kSwizzle128B),
                  smem_desc(dora + kk * 16 * 128, BQ * 128, 1024, kSwizzle128B), id_dv,
                  (it > 0 || kk > 0) ? 1u : 0u);
        // 5. dQ_t = dS_k K_seq into S's columns, dK_t = dS_q^T Q_seq into dP's
        mbar_wait(&sm.ds_ready, it & 1, 405);
        tc_fence_after();
        cp_atoms(sf_dsk, sm.dsksf, 2);
        cp_atoms(sf_dsq, sm.dsqsf, 2);
        cp_atoms(sf_qseq, sm.qssf, 2);
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
          mma_nvf4(tmem + kColS, smem_desc(dska + 32 * kk, 16, 512, kSwizzle64B),
                   smem_desc(ksa + 32 * kk, 16, 512, kSwizzle64B), id_g, sf_dsk + 4 * kk,
                   sf_kseq + 4 * kk, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
          mma_nvf4(tmem + kColDP, smem_desc(dsqa + 32 * kk, 16, 512, kSwizzle64B),
                   smem_desc(qsa + 32 * kk, 16, 512, kSwizzle64B), id_g, sf_dsq + 4 * kk,
                   sf_qseq + 4 * kk, kk > 0 ? 1u : 0u);
        mma_commit(&sm.dkdq_full);
        mma_commit(&sm.st_free);  // every reader of the query tile's stage has completed
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

    for (int it = 0; it < nq; ++it) {
      const int qt = i_first + it;
      const int b = it & 1;
      const size_t grow = static_cast<size_t>(row_base) + qt * BQ + r;
      const float lse2 = args.lse[grow] * 1.4426950408889634f;
      const float dvr = args.dvec[grow];
      const bool diag = args.causal && qt == t;
      mbar_wait(&sm.sdp_full, it & 1, 410);
      tc_fence_after();
      // pass A: this row's 64 keys of warpgroup h, 16 columns at a time
      float ds[64];
      float dsmax = 0.0f;
      uint8_t* patom = reinterpret_cast<uint8_t*>(sm.p) + h * (BQ * 128);
#pragma unroll
      for (int c16 = 0; c16 < 4; ++c16) {
        const int col = h * 64 + c16 * 16;
        uint32_t sx[16], px[16];
        tmem_ld16(lane_base + kColS + col, sx);
        tmem_ld16(lane_base + kColDP + col, px);
        tmem_ld_wait_regs(sx, px);
        uint32_t w[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          float p0 = ex2_approx(fmaf(__uint_as_float(sx[e]), c, -lse2));
          float p1 = ex2_approx(fmaf(__uint_as_float(sx[e + 1]), c, -lse2));
          if (diag && col + e > r) p0 = 0.0f;  // key index - query index = col - r
          if (diag && col + e + 1 > r) p1 = 0.0f;
          const float d0 = p0 * (__uint_as_float(px[e]) - dvr);
          const float d1 = p1 * (__uint_as_float(px[e + 1]) - dvr);
          ds[c16 * 16 + e] = d0;
          ds[c16 * 16 + e + 1] = d1;
          dsmax = fmax3(dsmax, fabsf(d0), fabsf(d1));
          w[e / 2] = Cvt<T>::pack2(p0, p1);
          sm.dst[col + e][r] = d0;
          sm.dst[col + e + 1][r] = d1;
        }
        // keys col .. col+15 are 16-byte chunks 2 c16 and 2 c16 + 1 of this row's atom
        *reinterpret_cast<uint4*>(patom + swz_offset(r, 2 * c16, 128)) =
            make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4*>(patom + swz_offset(r, 2 * c16 + 1, 128)) =
            make_uint4(w[4], w[5], w[6], w[7]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&sm.p_ready);
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
      // pass B (1): dS in 16-key blocks along this query row -> A of dQ
#pragma unroll
      for (int kb = 0; kb < 4; kb += 2) {
        uint32_t sc0, sc1;
        float xa[16], xb[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          xa[e] = ds[kb * 16 + e];
          xb[e] = ds[kb * 16 + 16 + e];
        }
        const uint2 ca = quant_block16(xa, genc, sc0);
        const uint2 cb = quant_block16(xb, genc, sc1);
        *reinterpret_cast<uint4*>(sm.dsk + swz_offset(r, 2 * h + kb / 2, 64)) =
            make_uint4(ca.x, ca.y, cb.x, cb.y);
        sm.dsksf[h * 512 + (r & 31) * 16 + (r >> 5) * 4 + kb] = static_cast<uint8_t>(sc0);
        sm.dsksf[h * 512 + (r & 31) * 16 + (r >> 5) * 4 + kb + 1] = static_cast<uint8_t>(sc1);
      }
      // pass B (2): dS^T in 16-query blocks along each key row -> A of dK; thread -> key
      // k = threadIdx % 128, queries 64 qh .. 64 qh + 63
      {
        const int k = threadIdx.x & 127, qh = threadIdx.x >> 7;
#pragma unroll
        for (int qb = 0; qb < 4; qb += 2) {
          uint32_t sc0, sc1;
          float xa[16], xb[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            xa[e] = sm.dst[k][qh * 64 + qb * 16 + e];
            xb[e] = sm.dst[k][qh * 64 + qb * 16 + 16 + e];
          }
          const uint2 ca = quant_block16(xa, genc, sc0);
          const uint2 cb = quant_block16(xb, genc, sc1);
          *reinterpret_cast<uint4*>(sm.dsq + swz_offset(k, 2 * qh + qb / 2, 64)) =
              make_uint4(ca.x, ca.y, cb.x, cb.y);
          sm.dsqsf[qh * 512 + (k & 31) * 16 + (k >> 5) * 4 + qb] = static_cast<uint8_t>(sc0);
          sm.dsqsf[qh * 512 + (k & 31) * 16 + (k >> 5) * 4 + qb + 1] = static_cast<uint8_t>(sc1);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&sm.ds_ready);
      // 5. read-outs: dQ_t (lane = query row) to the global accumulator, dK_t (lane = key row)
      // into registers; thread (h) takes channels h*D/2 ..
      const float sq = __fdiv_rn(args.tau, __fmul_rn(genc, kg));
      const float sk = __fdiv_rn(args.tau, __fmul_rn(genc, qg));
      mbar_wait(&sm.dkdq_full, it & 1, 412);
      tc_fence_after();
      float* dqrow = args.dq_acc + grow * D + h * DH;
#pragma unroll
      for (int c0 = 0; c0 < DH; c0 += 16) {
        uint32_t a[16], kx[16];
        tmem_ld16(lane_base + kColS + h * DH + c0, a);
        tmem_ld16(lane_base + kColDP + h * DH + c0, kx);
        tmem_ld_wait_regs(a, kx);
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
          const float4 v4 = make_float4(__uint_as_float(a[e]) * sq, __uint_as_float(a[e + 1]) * sq,
                                        __uint_as_float(a[e + 2]) * sq,
                                        __uint_as_float(a[e + 3]) * sq);
          atomicAdd(reinterpret_cast<float4*>(dqrow + c0 + e), v4);
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) acck[c0 + e] = fmaf(__uint_as_float(kx[e]), sk, acck[c0 + e]);
      }
      tc_fence_before();
      mbar_arrive(&sm.tmem_free);
    }
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
