// rowops.cuh -- HBM-bound row kernels of the SageBwd path:
//   * the prologue (QK-norm paragraph: per-token RMSNorm of q and k; K-smoothing paragraph:
//     per-channel mean of k over tokens subtracted before quantization; Triton-kernel
//     paragraph: per-block INT8 quantization of q, k, v),
//   * the backward preprocess (D = rowsum(dO o O), dO quantized per q_block tokens, dQ
//     accumulator cleared),
//   * the dQ finalize (float32 dQ accumulator -> RMSNorm backward -> 16-bit dq).
//
// Row mapping: a row of d 16-bit values is read by d/8 consecutive lanes with one 128-bit load
// each (lane l owns channels 8l .. 8l+7); a warp therefore covers 32/(d/8) rows per step.
// Reductions inside a row are xor-butterflies over those lanes.
//
// The prologue's float32 operation order is part of its definition (its codes, scales,
// inverse RMS values and K means are reproducible bit for bit):
//   RMSNorm: per lane, p = 0; p = p + x_c * x_c over its 8 channels in ascending order; then
//            p_l = p_l + p_(l xor o) for o = d/16, ..., 1; ss = p; inv = 1 / sqrt(ss/d + eps);
//            xhat = x * inv;
//   K mean:  per 64-token block, each channel summed over the block's tokens in ascending order
//            from 0; block sums added in ascending block order from 0; m = S / N;
//   quantize: s = absmax / 127, code = rint(x / s) (round half to even), s = 0 -> codes 0.
// All operations use the _rn intrinsics, which the compiler never contracts into FMAs.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "ptx.cuh"

namespace sage {

constexpr int kRowThreads = 256;  // 8 warps; a CTA handles 128 rows (16 per warp)
constexpr int kRowsPerCta = 128;
constexpr int kQuantThreads = 512;  // prologue quantization: 16 warps, 8 rows each

template <typename T>
struct Cvt;

template <>
struct Cvt<__nv_bfloat16> {
  static __device__ __forceinline__ void load8(const uint4& u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
  static __device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
};

template <>
struct Cvt<__half> {
  static __device__ __forceinline__ void load8(const uint4& u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __half2 h = *reinterpret_cast<const __half2*>(&w[i]);
      float2 t = __half22float2(h);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
  static __device__ __forceinline__ uint32_t pack2(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
};

template <typename T>
__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  return make_uint4(Cvt<T>::pack2(f[0], f[1]), Cvt<T>::pack2(f[2], f[3]),
                    Cvt<T>::pack2(f[4], f[5]), Cvt<T>::pack2(f[6], f[7]));
}

// Butterfly sum across the LPR lanes that hold one row (mask = those lanes).
template <int LPR>
__device__ __forceinline__ float row_sum(float p, uint32_t mask) {
#pragma unroll
  for (int o = LPR / 2; o >= 1; o >>= 1) p = __fadd_rn(p, __shfl_xor_sync(mask, p, o));
  return p;
}

// RMSNorm of the 8 values a lane holds (the row is spread over LPR lanes).  Returns inv.
template <int D>
__device__ __forceinline__ float rms_norm8(float (&x)[8], float eps, uint32_t mask) {
  float p = 0.0f;
#pragma unroll
  for (int c = 0; c < 8; ++c) p = __fadd_rn(p, __fmul_rn(x[c], x[c]));
  const float ss = row_sum<D / 8>(p, mask);
  const float ms = __fdiv_rn(ss, static_cast<float>(D));
  const float r = __fsqrt_rn(__fadd_rn(ms, eps));
  const float inv = __fdiv_rn(1.0f, r);
#pragma unroll
  for (int c = 0; c < 8; ++c) x[c] = __fmul_rn(x[c], inv);
  return inv;
}

// code = rint(x / s) (round half to even) as a byte (two's complement), 0 when s == 0.
// |x| <= absmax and s = RN(absmax / 127) keep |x / s| below 127.5, so no clamp is needed and
// rint is taken by adding 1.5 * 2^23 (the sum rounds the quotient to the nearest integer, ties
// to even, into the low mantissa bits), which keeps the conversion off the MUFU/XU pipe.
__device__ __forceinline__ float quant_magic(float x, float s) {
  return s > 0.0f ? __fadd_rn(__fdiv_rn(x, s), kMagic) : kMagic;
}

// The same code without a division per element: q = x * r with r = RN(1/s) is within
// 1.5 * 2^-16 of RN(x / s) for every element of the block (|x / s| < 128: both carry a relative
// error below 2^-23 and 2^-24), so rint(q) = rint(RN(x / s)) unless a half-integer lies within
// that distance of q -- then |q - rint(q)| >= 0.5 - 2^-15 and the IEEE quotient decides (ties
// included).  r_ok is false when r is not finite (s below 2^-128): every element takes the IEEE
// quotient.  Returns kMagic + code, as quant_magic.
__device__ __forceinline__ float quant_magic_r(float x, float s, float r, bool r_ok) {
  const float q = __fmul_rn(x, r);
  const float t = __fadd_rn(q, kMagic);                  // kMagic + rint(q)
  const float f = __fsub_rn(q, __fsub_rn(t, kMagic));    // q - rint(q), exact
  if (!r_ok || fabsf(f) >= 0.5f - 0x1p-15f) return quant_magic(x, s);
  return t;
}

// Eight codes by the IEEE quotient (the backward preprocess's dO codes: there the division-free
// path measured slower).
__device__ __forceinline__ uint2 quant8_div(const float (&x)[8], float s) {
  return make_uint2(pack_magic4(quant_magic(x[0], s), quant_magic(x[1], s),
                                quant_magic(x[2], s), quant_magic(x[3], s)),
                    pack_magic4(quant_magic(x[4], s), quant_magic(x[5], s),
                                quant_magic(x[6], s), quant_magic(x[7], s)));
}

// Eight codes by the division-free path (the prologue's Q, K and V codes).
__device__ __forceinline__ uint2 quant8(const float (&x)[8], float s) {
  if (!(s > 0.0f)) return make_uint2(0u, 0u);  // all-zero block: codes 0
  const float r = __frcp_rn(s);
  const bool r_ok = r < INFINITY;
  return make_uint2(pack_magic4(quant_magic_r(x[0], s, r, r_ok), quant_magic_r(x[1], s, r, r_ok),
                                quant_magic_r(x[2], s, r, r_ok), quant_magic_r(x[3], s, r, r_ok)),
                    pack_magic4(quant_magic_r(x[4], s, r, r_ok), quant_magic_r(x[5], s, r, r_ok),
                                quant_magic_r(x[6], s, r, r_ok), quant_magic_r(x[7], s, r, r_ok)));
}

// ---------------------------------------------------------------------------------------------
// Prologue pass 1 (only with smoothing): per 64-token block of k (or q), the column sums of
// khat (qhat).
// One group of D/8 lanes walks one block's 64 tokens in order.  partials: [BH * N/64, D].
// MINMAX (NVFP4 prologue): also the block's column maxima and minima, at partials +
// total_blocks * D and + 2 * total_blocks * D.
// ---------------------------------------------------------------------------------------------
template <typename T, int D, bool MINMAX = false>
__global__ void __launch_bounds__(kRowThreads) prologue_kstats_kernel(
    const T* __restrict__ k, float* __restrict__ partials, int total_blocks, int qknorm,
    float eps) {
  constexpr int LPR = D / 8, GPW = 32 / LPR;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int grp = lane / LPR, sub = lane % LPR;
  const int blk = (blockIdx.x * (kRowThreads / 32) + warp) * GPW + grp;
  if (blk >= total_blocks) return;  // whole lane groups leave together
  const uint32_t mask = ((LPR == 32) ? 0xFFFFFFFFu : ((1u << LPR) - 1u)) << (grp * LPR);
  const T* src = k + static_cast<size_t>(blk) * 64 * D + sub * 8;
  float c[8], hi[8], lo[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    c[i] = 0.0f;
    hi[i] = -INFINITY;
    lo[i] = INFINITY;
  }
#pragma unroll 4
  for (int t = 0; t < 64; ++t) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(src + static_cast<size_t>(t) * D));
    float x[8];
    Cvt<T>::load8(u, x);
    if (qknorm) rms_norm8<D>(x, eps, mask);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      c[i] = __fadd_rn(c[i], x[i]);
      if constexpr (MINMAX) {
        hi[i] = fmaxf(hi[i], x[i]);
        lo[i] = fminf(lo[i], x[i]);
      }
    }
  }
  float4* dst = reinterpret_cast<float4*>(partials + static_cast<size_t>(blk) * D + sub * 8);
  dst[0] = make_float4(c[0], c[1], c[2], c[3]);
  dst[1] = make_float4(c[4], c[5], c[6], c[7]);
  if constexpr (MINMAX) {
    const size_t plane = static_cast<size_t>(total_blocks) * D;
    dst[plane / 4] = make_float4(hi[0], hi[1], hi[2], hi[3]);
    dst[plane / 4 + 1] = make_float4(hi[4], hi[5], hi[6], hi[7]);
    dst[plane / 2] = make_float4(lo[0], lo[1], lo[2], lo[3]);
    dst[plane / 2 + 1] = make_float4(lo[4], lo[5], lo[6], lo[7]);
  }
}

// Prologue pass 2 (only with smoothing): m[bh][c] = (sum over blocks in order) / N.
// MINMAX (NVFP4 prologue): also the head's maximum of |fl(khat - m)|, as float bits in
// gmax[bh].  fl(x - m) is monotone in x, so per channel that maximum is reached at the
// channel's largest or smallest khat: no pass over the smoothed values is needed.
template <int D, bool MINMAX = false>
__global__ void prologue_kmean_kernel(const float* __restrict__ partials,
                                      float* __restrict__ k_mean, int nkb, int N,
                                      int total_blocks = 0, uint32_t* gmax = nullptr) {
  const int bh = blockIdx.x, c = threadIdx.x;
  const float* src = partials + static_cast<size_t>(bh) * nkb * D + c;
  float s = 0.0f;
  for (int t = 0; t < nkb; ++t) s = __fadd_rn(s, src[static_cast<size_t>(t) * D]);
  const float m = __fdiv_rn(s, static_cast<float>(N));
  k_mean[static_cast<size_t>(bh) * D + c] = m;
  if constexpr (MINMAX) {
    const size_t plane = static_cast<size_t>(total_blocks) * D;
    float hi = -INFINITY, lo = INFINITY;
    for (int t = 0; t < nkb; ++t) {
      hi = fmaxf(hi, src[plane + static_cast<size_t>(t) * D]);
      lo = fminf(lo, src[2 * plane + static_cast<size_t>(t) * D]);
    }
    float a = fmaxf(fabsf(__fsub_rn(hi, m)), fabsf(__fsub_rn(lo, m)));
    __shared__ float red[D / 32];
    a = warp_max(a);
    if ((c & 31) == 0) red[c >> 5] = a;
    __syncthreads();
    if (c == 0) {
      float g = 0.0f;
#pragma unroll
      for (int w = 0; w < D / 32; ++w) g = fmaxf(g, red[w]);
      gmax[bh] = __float_as_uint(g);
    }
  }
}

// Block absmax over the CTA's 128 rows held by NW warps (rows 0-63 in the first half of the
// warps, 64-127 in the second); returns the absmax of the block (of `blk` rows) this thread's
// row belongs to.
template <int NW>
__device__ __forceinline__ float block_absmax_n(float local, int blk, float* red) {
  const int warp = threadIdx.x >> 5;
  const float wm = warp_max(local);
  if ((threadIdx.x & 31) == 0) red[warp] = wm;
  __syncthreads();
  float a = 0.0f;
  if (blk == 128) {
#pragma unroll
    for (int w = 0; w < NW; ++w) a = fmaxf(a, red[w]);
  } else {
    const int w0 = (warp / (NW / 2)) * (NW / 2);
#pragma unroll
    for (int w = 0; w < NW / 2; ++w) a = fmaxf(a, red[w0 + w]);
  }
  return a;
}

struct PrologueArgs {
  const void* src[3];      // q, k, v
  int8_t* codes[3];        // q, k, v codes
  float* scale[3];         // q, k, v scales
  float* inv_rms[2];       // q, k
  const float* k_mean;     // [BH, D] (ksmooth)
  const float* q_mean;     // [BH, D] (qsmooth)
  float* k_bias;           // [BH, N] (qsmooth): mu_Q . ktilde_j
  int BH, N, q_block, qknorm, ksmooth, qsmooth;
  float eps;
};

// Prologue pass 3: one CTA per 128-token chunk of q, k or v (grid = 3 * BH * N/128):
// RMSNorm (q, k), mean subtraction (k), block absmax and quantization.
template <typename T, int D>
__global__ void __launch_bounds__(kQuantThreads, 2) prologue_quant_kernel(PrologueArgs a) {
  constexpr int NW = kQuantThreads / 32, RPW = kRowsPerCta / NW;  // warps, rows per warp
  constexpr int LPR = D / 8, GPW = 32 / LPR, STEPS = RPW / GPW;
  __shared__ float red[NW];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int grp = lane / LPR, sub = lane % LPR;
  const uint32_t mask = ((LPR == 32) ? 0xFFFFFFFFu : ((1u << LPR) - 1u)) << (grp * LPR);
  const int nchunk = a.N / kRowsPerCta;
  const int per = a.BH * nchunk;
  const int which = blockIdx.x / per;
  const int rem = blockIdx.x % per;
  const int bh = rem / nchunk, ch = rem % nchunk;
  const size_t row0 = static_cast<size_t>(bh) * a.N + static_cast<size_t>(ch) * kRowsPerCta;
  const T* src = reinterpret_cast<const T*>(a.src[which]);

  float x[STEPS][8];
#pragma unroll
  for (int s = 0; s < STEPS; ++s) {
    const int r = warp * RPW + s * GPW + grp;
    const uint4 u =
        __ldg(reinterpret_cast<const uint4*>(src + (row0 + r) * D + sub * 8));
    Cvt<T>::load8(u, x[s]);
  }
  if (which < 2 && a.qknorm) {
#pragma unroll
    for (int s = 0; s < STEPS; ++s) {
      const float inv = rms_norm8<D>(x[s], a.eps, mask);
      const int r = warp * RPW + s * GPW + grp;
      if (sub == 0) a.inv_rms[which][row0 + r] = inv;
    }
  }
  // smoothing: K's mean (ksmooth) or Q's (qsmooth) subtracted just before quantization
  const float* mean = which == 1 ? (a.ksmooth ? a.k_mean : nullptr)
                                 : (which == 0 && a.qsmooth ? a.q_mean : nullptr);
  if (mean) {
    const float4* mp = reinterpret_cast<const float4*>(mean + static_cast<size_t>(bh) * D + sub * 8);
    const float4 m0 = mp[0], m1 = mp[1];
    const float m[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
#pragma unroll
    for (int s = 0; s < STEPS; ++s)
#pragma unroll
      for (int c = 0; c < 8; ++c) x[s][c] = __fsub_rn(x[s][c], m[c]);
  }
  if (which == 1 && a.qsmooth) {
    // Q-smoothing bias of every key: k_bias_j = mu_Q . ktilde_j (lane partials + butterfly)
    const float4* mp =
        reinterpret_cast<const float4*>(a.q_mean + static_cast<size_t>(bh) * D + sub * 8);
    const float4 m0 = mp[0], m1 = mp[1];
    const float m[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
#pragma unroll
    for (int s = 0; s < STEPS; ++s) {
      float p = 0.0f;
#pragma unroll
      for (int c = 0; c < 8; ++c) p = __fadd_rn(p, __fmul_rn(m[c], x[s][c]));
      const float b = row_sum<D / 8>(p, mask);
      const int r = warp * RPW + s * GPW + grp;
      if (sub == 0) a.k_bias[row0 + r] = b;
    }
  }
  float amax = 0.0f;
#pragma unroll
  for (int s = 0; s < STEPS; ++s)
#pragma unroll
    for (int c = 0; c < 8; ++c) amax = fmaxf(amax, fabsf(x[s][c]));
  const int blk = (which == 0) ? a.q_block : 64;
  const float am = block_absmax_n<NW>(amax, blk, red);
  const float sc = __fdiv_rn(am, 127.0f);
  if (threadIdx.x == 0 || (blk == 64 && threadIdx.x == kQuantThreads / 2)) {
    const int sub_blk = (blk == 64 && threadIdx.x != 0) ? 1 : 0;
    const size_t idx = static_cast<size_t>(bh) * (a.N / blk) +
                       static_cast<size_t>(ch) * (kRowsPerCta / blk) + sub_blk;
    a.scale[which][idx] = sc;
  }
  int8_t* dst = a.codes[which];
#pragma unroll
  for (int s = 0; s < STEPS; ++s) {
    const int r = warp * RPW + s * GPW + grp;
    *reinterpret_cast<uint2*>(dst + (row0 + r) * D + sub * 8) = quant8(x[s], sc);
  }
}

// ---------------------------------------------------------------------------------------------
// Backward preprocess: D_i = sum_c dO_ic O_ic (float32), dO codes per q_block tokens (skipped
// when do_codes is null), and the float32 dQ accumulator rows cleared.  One CTA
// (kQuantThreads threads) per 128 rows.
// ---------------------------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(kQuantThreads, 2) bwd_preprocess_kernel(
    const T* __restrict__ o, const T* __restrict__ dout, float* __restrict__ Dvec,
    int8_t* __restrict__ do_codes, float* __restrict__ do_scale, float* __restrict__ dq_acc,
    int N, int q_block) {
  constexpr int NW = kQuantThreads / 32, RPW = kRowsPerCta / NW;  // warps, rows per warp
  constexpr int LPR = D / 8, GPW = 32 / LPR, STEPS = RPW / GPW;
  __shared__ float red[NW];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int grp = lane / LPR, sub = lane % LPR;
  const uint32_t mask = ((LPR == 32) ? 0xFFFFFFFFu : ((1u << LPR) - 1u)) << (grp * LPR);
  const size_t row0 = static_cast<size_t>(blockIdx.x) * kRowsPerCta;
  float x[STEPS][8];
  float amax = 0.0f;
#pragma unroll
  for (int s = 0; s < STEPS; ++s) {
    const int r = warp * RPW + s * GPW + grp;
    const size_t off = (row0 + r) * D + sub * 8;
    float y[8];
    Cvt<T>::load8(__ldg(reinterpret_cast<const uint4*>(dout + off)), x[s]);
    Cvt<T>::load8(__ldg(reinterpret_cast<const uint4*>(o + off)), y);
    float p = 0.0f;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      p = fmaf(x[s][c], y[c], p);
      amax = fmaxf(amax, fabsf(x[s][c]));
    }
    p = row_sum<LPR>(p, mask);
    if (sub == 0) Dvec[row0 + r] = p;
    float4* z = reinterpret_cast<float4*>(dq_acc + off);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  if (do_codes == nullptr) return;  // D and the cleared accumulator only
  const float am = block_absmax_n<NW>(amax, q_block, red);
  const float sc = __fdiv_rn(am, 127.0f);
  if (threadIdx.x == 0 || (q_block == 64 && threadIdx.x == kQuantThreads / 2))
    do_scale[(row0 + (threadIdx.x == 0 ? 0 : 64)) / q_block] = sc;
#pragma unroll
  for (int s = 0; s < STEPS; ++s) {
    const int r = warp * RPW + s * GPW + grp;
    *reinterpret_cast<uint2*>(do_codes + (row0 + r) * D + sub * 8) = quant8_div(x[s], sc);
  }
}

// ---------------------------------------------------------------------------------------------
// dQ finalize: dq = inv * (dqhat - qhat * (sum_c dqhat_c qhat_c) / d) when qknorm (RMSNorm
// backward, qhat = q * inv recomputed in float32), else dq = dqhat; rounded to T.
// ---------------------------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(kRowThreads) dq_finalize_kernel(
    const float* __restrict__ dq_acc, const T* __restrict__ q, const float* __restrict__ inv_rms,
    T* __restrict__ dq, int qknorm) {
  constexpr int LPR = D / 8, GPW = 32 / LPR, STEPS = 16 / GPW;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int grp = lane / LPR, sub = lane % LPR;
  const uint32_t mask = ((LPR == 32) ? 0xFFFFFFFFu : ((1u << LPR) - 1u)) << (grp * LPR);
  const size_t row0 = static_cast<size_t>(blockIdx.x) * kRowsPerCta;
#pragma unroll
  for (int s = 0; s < STEPS; ++s) {
    const int r = warp * 16 + s * GPW + grp;
    const size_t off = (row0 + r) * D + sub * 8;
    const float4 g0 = *reinterpret_cast<const float4*>(dq_acc + off);
    const float4 g1 = *reinterpret_cast<const float4*>(dq_acc + off + 4);
    float g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
    if (qknorm) {
      const float inv = inv_rms[row0 + r];
      float xh[8];
      Cvt<T>::load8(__ldg(reinterpret_cast<const uint4*>(q + off)), xh);
      float p = 0.0f;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        xh[c] = __fmul_rn(xh[c], inv);
        p = fmaf(g[c], xh[c], p);
      }
      const float dot = row_sum<LPR>(p, mask) * (1.0f / D);
#pragma unroll
      for (int c = 0; c < 8; ++c) g[c] = inv * fmaf(-xh[c], dot, g[c]);
    }
    *reinterpret_cast<uint4*>(dq + off) = pack8<T>(g);
  }
}

// ---------------------------------------------------------------------------------------------
// Merge of two attention results over disjoint key sets (context parallelism).  With
// L = ln(e^La + e^Lb), the softmax over the union of the keys gives
// O = e^(La - L) O_a + e^(Lb - L) O_b.  o_acc / lse_acc (float32, natural-log LSE; -inf marks
// an empty result) are updated in place with the partial o_part / lse_part; when `out` is
// set, the merged O is also written there in the 16-bit type.  Without a partial (o_part and
// lse_part null) the accumulator is only converted to `out`.  One thread per 8 channels of a
// row; the grid covers rows * D / 8 threads exactly (rows a multiple of 128).
// ---------------------------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(256) attn_merge_kernel(float* __restrict__ o_acc,
                                                         float* __restrict__ lse_acc,
                                                         const float* __restrict__ o_part,
                                                         const float* __restrict__ lse_part,
                                                         T* __restrict__ out) {
  constexpr int TPR = D / 8;  // threads per row (a row never straddles a warp)
  const size_t tid = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const size_t row = tid / TPR;
  const int c = static_cast<int>(tid % TPR) * 8;
  const float la = lse_acc[row];
  const float lb = lse_part != nullptr ? lse_part[row] : -INFINITY;
  const float4* pa = reinterpret_cast<const float4*>(o_acc + row * D + c);
  const float4 a0 = pa[0], a1 = pa[1];
  float f[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};  // empty partial: keep acc
  float lnew = la;
  if (lb != -INFINITY) {
    const float4* pb = reinterpret_cast<const float4*>(o_part + row * D + c);
    const float4 b0 = pb[0], b1 = pb[1];
    const float g[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
    if (la == -INFINITY) {  // empty accumulator: take the partial
#pragma unroll
      for (int e = 0; e < 8; ++e) f[e] = g[e];
      lnew = lb;
    } else {
      const float m = fmaxf(la, lb);
      const float ea = expf(la - m), eb = expf(lb - m);
      const float sum = ea + eb;
      lnew = m + logf(sum);
      const float wa = ea / sum, wb = eb / sum;
#pragma unroll
      for (int e = 0; e < 8; ++e) f[e] = fmaf(f[e], wa, g[e] * wb);
    }
  }
  float4* po = reinterpret_cast<float4*>(o_acc + row * D + c);
  po[0] = make_float4(f[0], f[1], f[2], f[3]);
  po[1] = make_float4(f[4], f[5], f[6], f[7]);
  if (out != nullptr) *reinterpret_cast<uint4*>(out + row * D + c) = pack8<T>(f);
  __syncwarp();  // every thread of the row has read lse_acc[row]
  if (c == 0) lse_acc[row] = lnew;
}

}  // namespace sage
