// nvfp4.cuh -- the NVFP4 Q-Attn variant on sm_100a ("Full-Stack FP4", gist.science
// 2607.04422, section 2.4: Q K^T in NVFP4, P V in BF16; the quantized views of Q and K are made
// once and reused).  NVFP4 format ("Quartet II", allinfo.ai.kr): E2M1 values in blocks of 16
// sharing an E4M3 scale, plus one global scale.
//
// Prologue (after the INT8 path's QK-norm / K-smoothing):
//   amax pass   per (tensor, batch-head) absolute maximum G of the normalized, smoothed values
//               (atomicMax on the float bits: non-negative floats order like their bits, so
//               the result does not depend on the order of the atomics).  With K-smoothing,
//               K's G comes instead from the K-statistics pass (column extremes, see
//               prologue_kmean_kernel) and this pass reads Q only;
//   quant pass  genc = 2688 / G (1 when G = 0); per 16 channels: a = max|x|,
//               u = (a * genc) / 6, sd = e4m3(u) (nearest, ties to even, saturating at 448),
//               code = e2m1(x * (genc / sd)) (nearest, ties to even, saturating at 6, the sign
//               bit the product's); every step a correctly rounded float32 operation.
// Outputs: codes [BH, N, d/2] (channel 2i in the low nibble of byte i), block scales in the
// tensor core's scale-factor order (per 128-row tile and 64-channel chunk, 512 bytes: byte
// (r % 32) * 16 + (r / 32) * 4 + b holds row r's scale of the chunk's 16-channel block b), and
// genc [BH].  Optionally the sequence views: the same values quantized in blocks of 16 tokens
// per channel (codes [BH, d, N/2], scale atoms per 128-channel group and 64-token chunk), the
// K-major operands of the backward's dK = dS^T Q and dQ = dS K.
//
// Forward: per CTA one tile of 128 query rows of one (batch, head), walking 128-key blocks.
//   warp 8      TMA producer: Q codes and scales once, then K codes, K scales and V (16-bit)
//               through a 3-stage ring;
//   warp 9      MMA issuer (one thread): block scales copied to TMEM (tcgen05.cp), S_j = Q K_j^T
//               (kind::mxf4nvf4, scale vector 16, FP32 in TMEM; S is read into registers as
//               soon as it lands, so one buffer suffices), then PV_{j-1} = P_{j-1} V_{j-1}
//               (kind::f16 in V's type, FP32 in TMEM, double-buffered);
//   warps 0-7   softmax, two warps per query row (one per 64-key half of each block and per
//               half of the output channels): z = S * tau / (genc_Q genc_K), causal mask,
//               running max (both warps of a row take it over all 128 scores of the block),
//               p = exp2(z - m) written to shared memory in V's 16-bit type (K-major, 128-byte
//               swizzle), running sum of the float32 p, and the fold O <- alpha O + PV in
//               registers.
//   warps 10-11 idle (they complete the producer warpgroup, which gives its registers to the
//               softmax warpgroups).
// TMEM (512 columns): S at 0, PV buffers at 128 and 256, Q scales at 384, K scales at 392 and
// 400 (alternating by block).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stddef.h>
#include <stdint.h>

#include <type_traits>

#include "ptx.cuh"
#include "rowops.cuh"

namespace sage {
namespace fp4 {

// ---------------------------------------------------------------------------------------------
// Number formats
// ---------------------------------------------------------------------------------------------
// Unsigned E4M3 code of u >= 0: nearest, ties to even, 448 and above -> 448 (0x7E).  Both the
// subnormal and the normal candidate are computed and one is selected (no branches).
__device__ __forceinline__ uint32_t e4m3_code(float u) {
  // subnormal codes: m * 2^-9, m = rint(u * 512) in [0, 8] (8 is the smallest normal, 2^-6)
  const uint32_t cs = static_cast<uint32_t>(__float2int_rn(u * 512.0f));
  // normal codes: with e = floor(log2 u), u * 2^(3-e) lies in [8, 16) and is exact (a
  // power-of-two scaling); its rounding q in [8, 16] gives code ((e + 7) << 3) + (q - 8), where
  // q = 16 carries into the exponent field.  (Meaningless for u < 2^-6, where cs is taken.)
  const int e = static_cast<int>((__float_as_uint(u) >> 23) & 0xFFu) - 127;
  const int q = __float2int_rn(u * __uint_as_float(static_cast<uint32_t>(130 - e) << 23));
  const uint32_t cn = static_cast<uint32_t>(((e + 7) << 3) + (q - 8));
  const uint32_t c = u < 0.015625f ? cs : cn;
  return u >= 448.0f ? 0x7Eu : c;
}

__device__ __forceinline__ float e4m3_value(uint32_t c) {
  const uint32_t e = c >> 3, m = c & 7u;
  const float sub = static_cast<float>(m) * 0.001953125f;
  const float nrm = __uint_as_float(((e + 120u) << 23) | (m << 20));
  return e == 0 ? sub : nrm;
}

// Two E2M1 codes in one byte (lo in bits 0-3, hi in bits 4-7) by the hardware conversion:
// round to nearest, ties to even, saturating at +-6, the sign bit that of the input (a
// negative value that rounds to zero gives -0, code 8).
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %2, %1;\n\t"
      "cvt.u32.u8 %0, t;\n\t}"
      : "=r"(r)
      : "f"(lo), "f"(hi));
  return r;
}

constexpr float kGlobalRange = 2688.0f;  // 6 (largest E2M1) * 448 (largest E4M3)

// x / 6 without a division: q = x * r with r = RN(1/6), the exact residual e = x - 6 q by one
// FMA, then q + e r by a second FMA (the correction step of Markstein's division algorithm).
// The result is the correctly rounded quotient whenever that quotient is a normal float32
// (one binade decides it: power-of-two scaling is exact); for x < 6 * 2^-126 it may differ,
// but both lie far below 2^-10, so the E4M3 code taken from it is 0 either way.  Checked
// against __fdiv_rn for every non-negative float32: no E4M3 code differs.
__device__ __forceinline__ float div6_rn(float x) {
  const float r = 0.16666667f;  // RN(1/6)
  const float q = __fmul_rn(x, r);
  const float e = __fmaf_rn(-q, 6.0f, x);
  return __fmaf_rn(e, r, q);
}

// ---------------------------------------------------------------------------------------------
// Prologue
// ---------------------------------------------------------------------------------------------
struct PrologueArgs {
  const void* src[2];     // q, k
  uint8_t* codes[2];      // [BH, N, D/2]
  uint8_t* sf[2];         // [BH, N/128, D/64, 512]
  float* genc[2];         // [BH]
  float* inv_rms[2];      // [BH, N] (qknorm)
  const float* k_mean;    // [BH, D] (ksmooth)
  uint32_t* gmax;         // [2, BH] float bits, zeroed before the amax pass
  uint8_t* codes_t[2];    // sequence views (or null): [BH, D, N/2], 16-token blocks per channel
  uint8_t* sf_t[2];       // [BH, ceil(D/128), N/64, 512]
  int BH, N, qknorm, ksmooth;
  float eps;
};

// Shared memory of the quantization pass when it also writes the sequence views: the chunk's
// normalized, smoothed values (128 tokens x D channels, rows padded by one float).
template <int D>
constexpr size_t seq_smem_bytes() {
  return static_cast<size_t>(kRowsPerCta) * (D + 1) * sizeof(float);
}

// The rows of one 128-row chunk, normalized and smoothed exactly as the INT8 prologue does.
template <typename T, int D, int STEPS, int RPW, int GPW>
__device__ __forceinline__ void load_rows(const PrologueArgs& a, int which, int bh, size_t row0,
                                          int warp, int grp, int sub, uint32_t mask,
                                          bool write_inv, float (&x)[STEPS][8]) {
  const T* src = reinterpret_cast<const T*>(which == 0 ? a.src[0] : a.src[1]);
  float* inv_out = which == 0 ? a.inv_rms[0] : a.inv_rms[1];
#pragma unroll
  for (int s = 0; s < STEPS; ++s) {
    const int r = warp * RPW + s * GPW + grp;
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(src + (row0 + r) * D + sub * 8));
    Cvt<T>::load8(u, x[s]);
  }
  if (a.qknorm) {
#pragma unroll
    for (int s = 0; s < STEPS; ++s) {
      const float inv = rms_norm8<D>(x[s], a.eps, mask);
      const int r = warp * RPW + s * GPW + grp;
      if (write_inv && sub == 0 && inv_out) inv_out[row0 + r] = inv;
    }
  }
  if (which == 1 && a.ksmooth) {
    const float4* mp =
        reinterpret_cast<const float4*>(a.k_mean + static_cast<size_t>(bh) * D + sub * 8);
    const float4 m0 = mp[0], m1 = mp[1];
    const float m[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
#pragma unroll
    for (int s = 0; s < STEPS; ++s)
#pragma unroll
      for (int c = 0; c < 8; ++c) x[s][c] = __fsub_rn(x[s][c], m[c]);
  }
}

// Pass 1: per (tensor, batch-head) absolute maximum.  Grid 2 * BH * N/128, kQuantThreads.
template <typename T, int D>
__global__ void __launch_bounds__(kQuantThreads, 2) prologue_amax_kernel(PrologueArgs a) {
  constexpr int NW = kQuantThreads / 32, RPW = kRowsPerCta / NW;
  constexpr int LPR = D / 8, GPW = 32 / LPR, STEPS = RPW / GPW;
  __shared__ float red[NW];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int grp = lane / LPR, sub = lane % LPR;
  const uint32_t mask = ((LPR == 32) ? 0xFFFFFFFFu : ((1u << LPR) - 1u)) << (grp * LPR);
  const int nchunk = a.N / kRowsPerCta, per = a.BH * nchunk;
  const int which = blockIdx.x / per, rem = blockIdx.x % per;
  const int bh = rem / nchunk, ch = rem % nchunk;
  const size_t row0 = static_cast<size_t>(bh) * a.N + static_cast<size_t>(ch) * kRowsPerCta;
  float x[STEPS][8];
  load_rows<T, D, STEPS, RPW, GPW>(a, which, bh, row0, warp, grp, sub, mask, false, x);
  float am = 0.0f;
#pragma unroll
  for (int s = 0; s < STEPS; ++s)
#pragma unroll
    for (int c = 0; c < 8; ++c) am = fmaxf(am, fabsf(x[s][c]));
  am = warp_max(am);
  if (lane == 0) red[warp] = am;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = 0.0f;
#pragma unroll
    for (int w = 0; w < NW; ++w) m = fmaxf(m, red[w]);
    atomicMax(a.gmax + which * a.BH + bh, __float_as_uint(m));
  }
}

// Pass 2: codes, block scales and the global scale.  Grid 2 * BH * N/128, kQuantThreads.
template <typename T, int D>
__global__ void __launch_bounds__(kQuantThreads, 2) prologue_quant_kernel(PrologueArgs a) {
  constexpr int NW = kQuantThreads / 32, RPW = kRowsPerCta / NW;
  constexpr int LPR = D / 8, GPW = 32 / LPR, STEPS = RPW / GPW;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int grp = lane / LPR, sub = lane % LPR;
  const uint32_t mask = ((LPR == 32) ? 0xFFFFFFFFu : ((1u << LPR) - 1u)) << (grp * LPR);
  const int nchunk = a.N / kRowsPerCta, per = a.BH * nchunk;
  const int which = blockIdx.x / per, rem = blockIdx.x % per;
  const int bh = rem / nchunk, ch = rem % nchunk;
  const size_t row0 = static_cast<size_t>(bh) * a.N + static_cast<size_t>(ch) * kRowsPerCta;
  float x[STEPS][8];
  load_rows<T, D, STEPS, RPW, GPW>(a, which, bh, row0, warp, grp, sub, mask, true, x);
  const float G = __uint_as_float(a.gmax[which * a.BH + bh]);
  const float genc = G > 0.0f ? __fdiv_rn(kGlobalRange, G) : 1.0f;
  if (ch == 0 && threadIdx.x == 0) (which == 0 ? a.genc[0] : a.genc[1])[bh] = genc;
  // this lane's 8 channels are half of the 16-channel block (sub / 2)
  const int kb = sub >> 1;
  uint8_t* codes = which == 0 ? a.codes[0] : a.codes[1];
  uint8_t* sf_tile = (which == 0 ? a.sf[0] : a.sf[1]) +
                     (static_cast<size_t>(bh) * nchunk + ch) * (D / 64) * 512 + (kb >> 2) * 512 +
                     (kb & 3);
#pragma unroll
  for (int s = 0; s < STEPS; ++s) {
    float am = 0.0f;
#pragma unroll
    for (int c = 0; c < 8; ++c) am = fmaxf(am, fabsf(x[s][c]));
    am = fmaxf(am, __shfl_xor_sync(mask, am, 1));
    const float u = __fdiv_rn(__fmul_rn(am, genc), 6.0f);
    const uint32_t sc = e4m3_code(u);
    const float sd = e4m3_value(sc);
    const float mult = sd > 0.0f ? __fdiv_rn(genc, sd) : 0.0f;
    uint32_t w = 0;
#pragma unroll
    for (int c = 0; c < 8; c += 2)
      w |= e2m1x2(__fmul_rn(x[s][c], mult), __fmul_rn(x[s][c + 1], mult)) << (4 * c);
    const int r = warp * RPW + s * GPW + grp;
    *reinterpret_cast<uint32_t*>(codes + (row0 + r) * (D / 2) + sub * 4) = w;
    if ((sub & 1) == 0) sf_tile[(r & 31) * 16 + (r >> 5) * 4] = static_cast<uint8_t>(sc);
  }
  uint8_t* codes_t = which == 0 ? a.codes_t[0] : a.codes_t[1];
  if (codes_t == nullptr) return;
  // Sequence views: the same values quantized in blocks of 16 tokens per channel (the global
  // scale is the matrix maximum, as for the row views).  Item (channel c, block tb) of the
  // chunk: codes of tokens 16 tb .. 16 tb + 15 at row c, scale at the channel's atom row.
  extern __shared__ float tile[];  // [kRowsPerCta][D + 1]
#pragma unroll
  for (int s = 0; s < STEPS; ++s) {
    const int r = warp * RPW + s * GPW + grp;
#pragma unroll
    for (int c = 0; c < 8; ++c) tile[r * (D + 1) + sub * 8 + c] = x[s][c];
  }
  __syncthreads();
  uint8_t* sf_t = which == 0 ? a.sf_t[0] : a.sf_t[1];
  constexpr int NTB = kRowsPerCta / 16;  // token blocks per chunk
  constexpr int NCG = (D + 127) / 128;   // 128-channel groups (scale atoms)
  const int nq64 = a.N / 64;
#pragma unroll
  for (int item = threadIdx.x; item < D * NTB; item += kQuantThreads) {
    const int c = item / NTB, tb = item % NTB;
    float v[16];
    float am = 0.0f;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      v[e] = tile[(tb * 16 + e) * (D + 1) + c];
      am = fmaxf(am, fabsf(v[e]));
    }
    const float u = __fdiv_rn(__fmul_rn(am, genc), 6.0f);
    const uint32_t sc = e4m3_code(u);
    const float sd = e4m3_value(sc);
    const float mult = sd > 0.0f ? __fdiv_rn(genc, sd) : 0.0f;
    uint32_t w0 = 0, w1 = 0;
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      w0 |= e2m1x2(__fmul_rn(v[e], mult), __fmul_rn(v[e + 1], mult)) << (4 * e);
      w1 |= e2m1x2(__fmul_rn(v[8 + e], mult), __fmul_rn(v[9 + e], mult)) << (4 * e);
    }
    const int t0 = ch * kRowsPerCta + tb * 16;  // first token of the block
    *reinterpret_cast<uint2*>(codes_t + (static_cast<size_t>(bh) * D + c) * (a.N / 2) + t0 / 2) =
        make_uint2(w0, w1);
    const size_t atom = (static_cast<size_t>(bh) * NCG + c / 128) * nq64 + t0 / 64;
    sf_t[atom * 512 + (c & 31) * 16 + ((c & 127) >> 5) * 4 + ((t0 >> 4) & 3)] =
        static_cast<uint8_t>(sc);
  }
}

// ---------------------------------------------------------------------------------------------
// Forward
// ---------------------------------------------------------------------------------------------
constexpr int BM = 128;   // query rows per CTA (MMA M)
constexpr int BKV = 128;  // keys per block
constexpr int NST = 3;    // K / V pipeline stages
constexpr int kThreads = 384;  // 8 softmax warps, producer, MMA, 2 idle warps
constexpr int kSoftmaxThreads = 256;
constexpr int kProducerWarp = 8, kMmaWarp = 9;
// register split (setmaxnreg): the softmax warpgroups rise to 232, the producer warpgroup
// (producer, MMA and two idle warps) drops to 40; the launch gives every thread 168
constexpr int kLaunchRegs = 168, kSoftmaxRegs = 232, kOtherRegs = 40;
static_assert(kSoftmaxThreads * kSoftmaxRegs + (kThreads - kSoftmaxThreads) * kOtherRegs <=
                  kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
constexpr uint32_t kColS = 0, kColPV = 128, kColSfa = 384, kColSfb = 392;  // TMEM columns

template <typename T, int D>
struct Smem {
  alignas(1024) uint8_t q[BM * D / 2];
  alignas(1024) uint8_t k[NST][BKV * D / 2];
  alignas(1024) T v[NST][BKV * D];   // D/64 boxes of [BKV keys][64 channels]
  alignas(1024) T p[2][BM * BKV];    // 2 swizzle atoms of [BM rows][64 keys]
  alignas(128) uint8_t qsf[D / 64 * 512];
  alignas(128) uint8_t ksf[NST][D / 64 * 512];
  float lsum[2][BM];    // per key half: the rows' final partial sums
  uint64_t q_full, k_full[NST], v_full[NST], kv_empty[NST];
  uint64_t s_full, s_free, p_full[2], pv_full[2], pv_free[2];
  uint32_t tmem_base;
  int abort;
};

template <typename T, int D>
constexpr size_t smem_bytes() {
  return sizeof(Smem<T, D>) + 1024;
}

template <typename T, int D>
__device__ __forceinline__ Smem<T, D>& smem_ref(uint8_t* raw) {
  const uint32_t a = smem_u32(raw);
  return *reinterpret_cast<Smem<T, D>*>(raw + ((1024u - (a & 1023u)) & 1023u));
}

struct Args {
  const uint8_t* q_sf;
  const uint8_t* k_sf;
  const float* q_genc;
  const float* k_genc;
  void* o;
  float* lse;
  int N, causal;
  float scale_log2;  // softmax_scale * log2(e)
};

template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, Args args) {
  static_assert(D == 64 || D == 128, "head dimension");
  extern __shared__ uint8_t smem_raw[];
  Smem<T, D>& sm = smem_ref<T, D>(smem_raw);
  constexpr uint32_t kSfBytes = D / 64 * 512;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int N = args.N, nqt = N / BM;
  // head-major order; within a head, the query tiles with the most key blocks first (causal)
  const int bh = blockIdx.x / nqt, t = blockIdx.x % nqt;
  const int qt = args.causal ? nqt - 1 - t : t;
  const int q0 = qt * BM;
  const int nb = args.causal ? qt + 1 : N / BKV;

  if (threadIdx.x == 0) {
    sm.abort = device_aborted() ? 1 : 0;
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    mbar_init(&sm.s_full, 1);
    mbar_init(&sm.s_free, kSoftmaxThreads);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.p_full[b], kSoftmaxThreads);
      mbar_init(&sm.pv_full[b], 1);
      mbar_init(&sm.pv_free[b], kSoftmaxThreads);
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
    if (warp == kProducerWarp) {
      if (lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        const int row_base = bh * N;
        mbar_arrive_expect_tx(&sm.q_full, BM * D / 2 + kSfBytes);
        tma_load_2d(sm.q, &tm_q, 0, row_base + q0, &sm.q_full);
        bulk_load(sm.qsf, args.q_sf + (static_cast<size_t>(bh) * nqt + qt) * kSfBytes, kSfBytes,
                  &sm.q_full);
        for (int j = 0; j < nb; ++j) {
          const int st = j % NST;
          if (j >= NST) mbar_wait(&sm.kv_empty[st], ((j / NST) - 1) & 1, 201);
          mbar_arrive_expect_tx(&sm.k_full[st], BKV * D / 2 + kSfBytes);
          tma_load_2d(sm.k[st], &tm_k, 0, row_base + j * BKV, &sm.k_full[st]);
          bulk_load(sm.ksf[st], args.k_sf + (static_cast<size_t>(bh) * (N / BKV) + j) * kSfBytes,
                    kSfBytes, &sm.k_full[st]);
          mbar_arrive_expect_tx(&sm.v_full[st], BKV * D * 2);
  #pragma unroll
          for (int b = 0; b < D / 64; ++b)
            tma_load_2d(sm.v[st] + b * BKV * 64, &tm_v, b * 64, row_base + j * BKV, &sm.v_full[st]);
        }
      }
      __syncwarp();
    } else if (warp == kMmaWarp) {
      if (lane == 0) {
        constexpr uint32_t kSw = (D == 128) ? kSwizzle64B : kSwizzle32B;
        constexpr uint32_t kSbo = 8 * (D / 2);  // 8 rows of D/2 bytes
        constexpr uint32_t kFmt = std::is_same<T, __nv_bfloat16>::value ? 1u : 0u;
        const uint32_t idesc_s = instr_desc_nvf4(BM, BKV);
        // P (A, K-major) and V (B, MN-major) share V's 16-bit type
        const uint32_t idesc_pv = instr_desc(1, kFmt, kFmt, false, true, BM, D);
        const uint32_t qa = smem_u32(sm.q);
        mbar_wait(&sm.q_full, 0, 210);
        tc_fence_after();
  #pragma unroll
        for (int kk = 0; kk < D / 64; ++kk)
          tmem_cp_sf(tmem + kColSfa + 4 * kk,
                     smem_desc(smem_u32(sm.qsf) + 512 * kk, 128, 128, kSwizzleNone));
        auto issue_pv = [&](int jj) {
          const int st = jj % NST;
          mbar_wait(&sm.v_full[st], (jj / NST) & 1, 213);
          mbar_wait(&sm.p_full[jj & 1], (jj >> 1) & 1, 214);
          if (jj >= 2) mbar_wait(&sm.pv_free[jj & 1], ((jj - 2) >> 1) & 1, 215);
          tc_fence_after();
          const uint32_t pa = smem_u32(sm.p[jj & 1]);
          const uint32_t va = smem_u32(sm.v[st]);
  #pragma unroll
          for (int kk = 0; kk < BKV / 16; ++kk) {
            mma_f16(tmem + kColPV + (jj & 1) * 128,
                    smem_desc(pa + (kk >> 2) * (BM * 128) + (kk & 3) * 32, 16, 1024, kSwizzle128B),
                    smem_desc(va + kk * 16 * 128, BKV * 128, 1024, kSwizzle128B), idesc_pv,
                    kk > 0 ? 1u : 0u);
          }
          mma_commit(&sm.pv_full[jj & 1]);
          mma_commit(&sm.kv_empty[st]);
        };
        for (int j = 0; j < nb; ++j) {
          const int st = j % NST, b = j & 1;
          mbar_wait(&sm.k_full[st], (j / NST) & 1, 211);
          // S and the K-scale columns b served block j-1 / j-2: S is free once block j-1's
          // softmax has read it (s_free), which also orders the scale copy below after the
          // MMAs of block j-2 (s_free of block j-1 follows s_full of block j-2)
          if (j >= 1) mbar_wait(&sm.s_free, (j - 1) & 1, 212);
          tc_fence_after();
          const uint32_t sfb = tmem + kColSfb + 8 * b;
  #pragma unroll
          for (int kk = 0; kk < D / 64; ++kk)
            tmem_cp_sf(sfb + 4 * kk, smem_desc(smem_u32(sm.ksf[st]) + 512 * kk, 128, 128,
                                               kSwizzleNone));
          const uint32_t ka = smem_u32(sm.k[st]);
  #pragma unroll
          for (int kk = 0; kk < D / 64; ++kk)
            mma_nvf4(tmem + kColS, smem_desc(qa + 32 * kk, 16, kSbo, kSw),
                     smem_desc(ka + 32 * kk, 16, kSbo, kSw), idesc_s, tmem + kColSfa + 4 * kk,
                     sfb + 4 * kk, kk > 0 ? 1u : 0u);
          mma_commit(&sm.s_full);
          if (j >= 1) issue_pv(j - 1);
        }
        issue_pv(nb - 1);
      }
      __syncwarp();
    }
    tc_fence_before();
    named_barrier_sync(15, kThreads);
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kSoftmaxRegs));
    // ---------------- softmax warps ----------------
    // Two warps per TMEM lane quarter: `half` 0 takes keys 0-63 of every block and output
    // channels 0 .. D/2-1, half 1 keys 64-127 and channels D/2 .. D-1.  The row sums are
    // combined at the end through shared memory.
    const int quarter = warp & 3;
    const int half = warp >> 2;
    const int r = quarter * 32 + lane;
    const int i = q0 + r;
    const uint32_t lane_base = tmem + ((quarter * 32u) << 16);
    const int pair_bar = 1 + quarter;  // named barrier of the two warps of this quarter
    const float c = __fdiv_rn(args.scale_log2, args.q_genc[bh] * args.k_genc[bh]);
    constexpr int DH = D / 2;
    float O[DH];
#pragma unroll
    for (int cc = 0; cc < DH; ++cc) O[cc] = 0.0f;
    float m = -INFINITY, l = 0.0f, alpha_prev = 1.0f;

    auto fold_pv = [&](int jj, float a) {
      const uint32_t pv = lane_base + kColPV + (jj & 1) * 128 + half * DH;
      mbar_wait(&sm.pv_full[jj & 1], (jj >> 1) & 1, 221);
      tc_fence_after();
#pragma unroll
      for (int c0 = 0; c0 < DH; c0 += 32) {
        uint32_t x0[16], x1[16];
        tmem_ld16(pv + c0, x0);
        tmem_ld16(pv + c0 + 16, x1);
        tmem_ld_wait_regs(x0, x1);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          O[c0 + e] = fmaf(O[c0 + e], a, __uint_as_float(x0[e]));
          O[c0 + 16 + e] = fmaf(O[c0 + 16 + e], a, __uint_as_float(x1[e]));
        }
      }
      tc_fence_before();
      mbar_arrive(&sm.pv_free[jj & 1]);
    };

    // One 128-key block.  Both warps of a row read all 128 scores for the block maximum
    // (identical on both: max does not depend on the order), so they need no exchange; each
    // keeps only its own 64 for the exponentials.  MASK: the causal test, compiled only into
    // the diagonal block's copy.
    auto block = [&](int j, auto masked) {
      constexpr bool MASK = decltype(masked)::value;
      const int b = j & 1;
      const int key0 = j * BKV + half * 64, okey0 = j * BKV + (half ^ 1) * 64;
      mbar_wait(&sm.s_full, j & 1, 220);
      tc_fence_after();
      const uint32_t sa = lane_base + kColS + half * 64;
      const uint32_t so = lane_base + kColS + (half ^ 1) * 64;
      uint32_t x0[16], x1[16], x2[16], x3[16], y0[16], y1[16];
      tmem_ld16(sa, x0);
      tmem_ld16(sa + 16, x1);
      tmem_ld16(sa + 32, x2);
      tmem_ld16(sa + 48, x3);
      tmem_ld16(so, y0);
      tmem_ld16(so + 16, y1);
      tmem_ld_wait_regs(x0, x1);
      tmem_ld_wait_regs(x2, x3);
      tmem_ld_wait_regs(y0, y1);
      float m0 = -INFINITY, m1 = -INFINITY, m0b = -INFINITY, m1b = -INFINITY;  // four chains
      auto maxh = [&](const uint32_t (&xa)[16], const uint32_t (&xb)[16], int k0, float& mm) {
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float f0 = __uint_as_float(xa[e]), f1 = __uint_as_float(xb[e]);
          if (MASK && k0 + e > i) f0 = -INFINITY;
          if (MASK && k0 + 16 + e > i) f1 = -INFINITY;
          mm = fmax3(mm, f0, f1);
        }
      };
      maxh(y0, y1, okey0, m1);
      tmem_ld16(so + 32, y0);
      tmem_ld16(so + 48, y1);
      maxh(x0, x1, key0, m0);
      maxh(x2, x3, key0 + 32, m0b);
      tmem_ld_wait_regs(y0, y1);
      tc_fence_before();
      mbar_arrive(&sm.s_free);
      maxh(y0, y1, okey0 + 32, m1b);
      // block maximum of the raw scores over visible keys (c > 0 keeps the order)
      const float mn = fmaxf(m, fmaxf(fmaxf(m0, m0b), fmaxf(m1, m1b)) * c);
      const float alpha = ex2_approx(m - mn);
      // p = exp2(S c - mn) in V's type into this half's swizzle atom (64 keys), row sum
      float rs0 = 0.0f, rs1 = 0.0f;
      uint8_t* atom = reinterpret_cast<uint8_t*>(sm.p[b]) + half * (BM * 128);
      auto conv = [&](const uint32_t (&x)[16], int k16) {
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            const int kk = key0 + k16 * 16 + q2 * 8 + e;
            float p0 = ex2_approx(fmaf(__uint_as_float(x[q2 * 8 + e]), c, -mn));
            float p1 = ex2_approx(fmaf(__uint_as_float(x[q2 * 8 + e + 1]), c, -mn));
            if (MASK && kk > i) p0 = 0.0f;
            if (MASK && kk + 1 > i) p1 = 0.0f;
            rs0 += p0;
            rs1 += p1;
            w[e / 2] = Cvt<T>::pack2(p0, p1);
          }
          *reinterpret_cast<uint4*>(atom + swz_offset(r, k16 * 2 + q2, 128)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      };
      conv(x0, 0);
      conv(x1, 1);
      conv(x2, 2);
      conv(x3, 3);
      l = fmaf(l, alpha, rs0 + rs1);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&sm.p_full[b]);
      if (j > 0) fold_pv(j - 1, alpha_prev);
      alpha_prev = alpha;
      m = mn;
    };
    for (int j = 0; j < nb; ++j) {
      if (args.causal && j == qt)
        block(j, std::true_type{});
      else
        block(j, std::false_type{});
    }
    fold_pv(nb - 1, alpha_prev);
    // row sum over both halves (same order on both warps), then the epilogue: O / l in the
    // output type, LSE = (m + log2 l) ln 2
    sm.lsum[half][r] = l;
    named_barrier_sync(pair_bar, 64);
    const float lt = sm.lsum[0][r] + sm.lsum[1][r];
    const float inv_l = 1.0f / lt;
    T* orow = reinterpret_cast<T*>(args.o) + (static_cast<size_t>(bh) * N + i) * D + half * DH;
#pragma unroll
    for (int c0 = 0; c0 < DH; c0 += 8) {
      float f[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) f[e] = O[c0 + e] * inv_l;
      *reinterpret_cast<uint4*>(orow + c0) = pack8<T>(f);
    }
    if (half == 0)
      args.lse[static_cast<size_t>(bh) * N + i] = (m + log2f(lt)) * 0.69314718055994531f;
    tc_fence_before();
    named_barrier_sync(15, kThreads);
  }
}

}  // namespace fp4
}  // namespace sage
