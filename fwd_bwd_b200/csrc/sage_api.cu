// sage_api.cu -- the C ABI of libsage (declared in include/sage.h): argument validation,
// workspace layout, TMA tensor-map construction and kernel launches.  The whole library is one
// translation unit so that every kernel shares the device status word.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>

#include "sage.h"
#include "sage_nvfp4.h"
#include "attn_bwd.cuh"
#include "attn_fwd.cuh"
#include "debug_kernels.cuh"
#include "nvfp4.cuh"
#include "nvfp4_bwd.cuh"
#include "ptx.cuh"
#include "rowops.cuh"

namespace {

using sage::kRowThreads;
using sage::kRowsPerCta;

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_params(const sage_params* p) {
  if (!p) return SAGE_ERR_INVALID_ARG;
  if (p->B <= 0 || p->H <= 0 || p->N <= 0 || p->d <= 0) return SAGE_ERR_INVALID_ARG;
  if (p->dtype != SAGE_FP16 && p->dtype != SAGE_BF16) return SAGE_ERR_INVALID_ARG;
  if (p->rms_eps < 0.0f || !std::isfinite(p->rms_eps)) return SAGE_ERR_INVALID_ARG;
  if (!std::isfinite(p->softmax_scale)) return SAGE_ERR_INVALID_ARG;
  if (p->d != 64 && p->d != 128) return SAGE_ERR_UNSUPPORTED;
  if (p->k_block != 64) return SAGE_ERR_UNSUPPORTED;
  if (p->q_block != 64 && p->q_block != 128) return SAGE_ERR_UNSUPPORTED;
  if (p->N % 128 != 0) return SAGE_ERR_UNSUPPORTED;
  if (p->qsmooth != 0 && p->qsmooth != 1) return SAGE_ERR_INVALID_ARG;
  // row indices of [B*H*N, d] tensors are passed to TMA as int32
  if (static_cast<long long>(p->B) * p->H * p->N >= (1ll << 31)) return SAGE_ERR_UNSUPPORTED;
  return SAGE_OK;
}

float tau_of(const sage_params* p) {
  return p->softmax_scale > 0.0f ? p->softmax_scale : 1.0f / std::sqrt(static_cast<float>(p->d));
}

int check_qbufs(const sage_params* p, const sage_qbufs* qb) {
  if (!qb || !qb->q_codes || !qb->k_codes || !qb->v_codes || !qb->q_scale || !qb->k_scale ||
      !qb->v_scale)
    return SAGE_ERR_INVALID_ARG;
  if (p->qknorm && (!qb->q_inv_rms || !qb->k_inv_rms)) return SAGE_ERR_INVALID_ARG;
  if (p->ksmooth && !qb->k_mean) return SAGE_ERR_INVALID_ARG;
  if (p->qsmooth && (!qb->q_mean || !qb->k_bias)) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(qb->q_codes) || !aligned16(qb->k_codes) || !aligned16(qb->v_codes))
    return SAGE_ERR_ALIGNMENT;
  if (qb->k_mean && !aligned16(qb->k_mean)) return SAGE_ERR_ALIGNMENT;
  if (p->qsmooth && (!aligned16(qb->q_mean) || !aligned16(qb->k_bias)))
    return SAGE_ERR_ALIGNMENT;
  return SAGE_OK;
}

// ---- workspace layouts ------------------------------------------------------------------
struct BwdWs {
  size_t dvec, doc, dos, dq, total;
};
BwdWs bwd_ws(const sage_params* p) {
  const size_t BH = static_cast<size_t>(p->B) * p->H, N = p->N, d = p->d;
  BwdWs w;
  w.dvec = 0;
  w.doc = align_up(w.dvec + BH * N * 4);
  w.dos = align_up(w.doc + BH * N * d);
  w.dq = align_up(w.dos + BH * (N / p->q_block) * 4);
  w.total = align_up(w.dq + BH * N * d * 4);
  return w;
}
// Column-sum partials of the smoothed tensors: K's (ksmooth) then Q's (qsmooth).
size_t prologue_partials(const sage_params* p) {
  return static_cast<size_t>(p->B) * p->H * (p->N / 64) * p->d;
}
size_t prologue_ws(const sage_params* p) {
  const int n = (p->ksmooth ? 1 : 0) + (p->qsmooth ? 1 : 0);
  return n == 0 ? 0 : align_up(n * prologue_partials(p) * 4);
}

// ---- TMA tensor maps --------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 2-D map over a row-major [rows][inner] array of 1- or 2-byte elements.
// Boxes whose rows are 64 or 128 bytes are swizzled to match the tensor cores' shared-memory
// layouts; `swizzle = false` gives a plain row-major box (float32 reduction staging).
bool make_map(CUtensorMap* m, const void* base, int elem_bytes, uint64_t inner, uint64_t rows,
              uint32_t box_inner, uint32_t box_rows, bool swizzle = true) {
  auto fn = encode_fn();
  if (!fn) return false;
  const uint32_t row_bytes_box = box_inner * elem_bytes;
  CUtensorMapSwizzle sw = !swizzle               ? CU_TENSOR_MAP_SWIZZLE_NONE
                          : row_bytes_box == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                          : row_bytes_box == 64  ? CU_TENSOR_MAP_SWIZZLE_64B
                                                 : CU_TENSOR_MAP_SWIZZLE_32B;
  const CUtensorMapDataType dt = elem_bytes == 1   ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                 : elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16
                                                   : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * elem_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int launch_status() { return cudaGetLastError() == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA; }

template <typename K>
int set_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(bytes)) == cudaSuccess
             ? SAGE_OK
             : SAGE_ERR_CUDA;
}

template <typename K>
int launch_regs(K kernel) {
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return -1;
  return fa.numRegs;
}

// ---- prologue ---------------------------------------------------------------------------
template <typename T, int D>
// part -1: statistics and quantization; 0: statistics only (the smoothing means); 1:
// quantization only, with the means already in `out`.
int run_prologue(const sage_params* p, const void* q, const void* k, const void* v,
                 const sage_qbufs* out, void* ws, cudaStream_t st, int part = -1) {
  const int BH = p->B * p->H, N = p->N;
  float* partials = reinterpret_cast<float*>(ws);
  const int total = BH * (N / 64);
  const int per_cta = (kRowThreads / 32) * (32 / (D / 8));
  // smoothing means: K's (ksmooth), then Q's (qsmooth), each from its own partials
  for (int which = 1; which >= 0 && part != 1; --which) {
    if (which == 1 ? !p->ksmooth : !p->qsmooth) continue;
    sage::prologue_kstats_kernel<T, D><<<(total + per_cta - 1) / per_cta, kRowThreads, 0, st>>>(
        reinterpret_cast<const T*>(which == 1 ? k : q), partials, total, p->qknorm,
        p->rms_eps);
    sage::prologue_kmean_kernel<D><<<BH, D, 0, st>>>(
        partials, which == 1 ? out->k_mean : out->q_mean, N / 64, N);
    partials += prologue_partials(p);
  }
  if (part == 0) return launch_status();
  sage::PrologueArgs a;
  a.src[0] = q;
  a.src[1] = k;
  a.src[2] = v;
  a.codes[0] = out->q_codes;
  a.codes[1] = out->k_codes;
  a.codes[2] = out->v_codes;
  a.scale[0] = out->q_scale;
  a.scale[1] = out->k_scale;
  a.scale[2] = out->v_scale;
  a.inv_rms[0] = out->q_inv_rms;
  a.inv_rms[1] = out->k_inv_rms;
  a.k_mean = out->k_mean;
  a.q_mean = out->q_mean;
  a.k_bias = out->k_bias;
  a.BH = BH;
  a.N = N;
  a.q_block = p->q_block;
  a.qknorm = p->qknorm;
  a.ksmooth = p->ksmooth;
  a.qsmooth = p->qsmooth;
  a.eps = p->rms_eps;
  sage::prologue_quant_kernel<T, D>
      <<<3 * BH * (N / kRowsPerCta), sage::kQuantThreads, 0, st>>>(a);
  return launch_status();
}

// ---- forward ----------------------------------------------------------------------------
template <typename T, int D>
int run_fwd(const sage_params* p, const sage_qbufs* qb, void* o, float* lse, cudaStream_t st,
            float* o_f32 = nullptr) {
  const int BH = p->B * p->H, N = p->N;
  const uint64_t rows = static_cast<uint64_t>(BH) * N;
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, qb->q_codes, 1, D, rows, D, sage::fwd::BM) ||
      !make_map(&tk, qb->k_codes, 1, D, rows, D, sage::fwd::BKV) ||
      !make_map(&tv, qb->v_codes, 1, D, rows, D, sage::fwd::BKV))
    return SAGE_ERR_CUDA;
  sage::fwd::Args a;
  a.q_scale = qb->q_scale;
  a.k_scale = qb->k_scale;
  a.v_scale = qb->v_scale;
  a.o = o;
  a.lse = lse;
  a.BH = BH;
  a.N = N;
  a.q_block = p->q_block;
  a.causal = p->causal;
  a.scale_log2 = tau_of(p) * 1.4426950408889634f;
  a.nsup = (N + sage::fwd::NT * sage::fwd::BM - 1) / (sage::fwd::NT * sage::fwd::BM);
  a.k_bias = qb->k_bias;
  a.o_f32 = o_f32;
  const size_t smem = sage::fwd::smem_bytes<D>();
  auto kern = p->qsmooth ? sage::fwd::attn_fwd_kernel<T, D, true>
                         : sage::fwd::attn_fwd_kernel<T, D, false>;
  if (set_smem(kern, smem) != SAGE_OK) return SAGE_ERR_CUDA;
  // register split between warpgroups (setmaxnreg) assumes exactly kLaunchRegs at launch
  if (launch_regs(kern) != sage::fwd::kLaunchRegs) return SAGE_ERR_UNSUPPORTED;
  kern<<<BH * a.nsup, sage::fwd::kThreads, smem, st>>>(tq, tk, tv, a);
  return launch_status();
}

// ---- backward ---------------------------------------------------------------------------
// stage 0: preprocess (D, dO codes, dQ accumulator cleared); 1: main tensor-core kernel;
// 2: dq finalize.
template <typename T, int D>
int run_bwd(int stage, const sage_params* p, const void* q, const void* k, const void* v,
            const sage_qbufs* qb, const void* o, const float* lse, const void* dout, void* dq,
            void* dk, void* dv, void* ws, cudaStream_t st, float* dk_acc = nullptr,
            float* dv_acc = nullptr, int acc_add = 0) {
  const int BH = p->B * p->H, N = p->N;
  const uint64_t rows = static_cast<uint64_t>(BH) * N;
  const BwdWs w = bwd_ws(p);
  uint8_t* wsb = reinterpret_cast<uint8_t*>(ws);
  float* dvec = reinterpret_cast<float*>(wsb + w.dvec);
  int8_t* doc = reinterpret_cast<int8_t*>(wsb + w.doc);
  float* dos = reinterpret_cast<float*>(wsb + w.dos);
  float* dqacc = reinterpret_cast<float*>(wsb + w.dq);
  if (stage == 0) {
    sage::bwd_preprocess_kernel<T, D>
        <<<static_cast<int>(rows / kRowsPerCta), sage::kQuantThreads, 0, st>>>(
            reinterpret_cast<const T*>(o), reinterpret_cast<const T*>(dout), dvec, doc, dos,
            dqacc, N, p->q_block);
    return launch_status();
  }
  if (stage == 2) {
    sage::dq_finalize_kernel<T, D><<<static_cast<int>(rows / kRowsPerCta), kRowThreads, 0, st>>>(
        dqacc, reinterpret_cast<const T*>(q), qb->q_inv_rms, reinterpret_cast<T*>(dq),
        p->qknorm);
    return launch_status();
  }
  CUtensorMap tqc, tkc, tdoc, tdo, tv, tdq;
  if (!make_map(&tqc, qb->q_codes, 1, D, rows, D, sage::bwd::BQ) ||
      !make_map(&tkc, qb->k_codes, 1, D, rows, D, sage::bwd::BKT) ||
      !make_map(&tdoc, doc, 1, D, rows, D, sage::bwd::BQ) ||
      !make_map(&tdo, dout, 2, D, rows, 64, sage::bwd::BQ) ||
      !make_map(&tv, v, 2, D, rows, 64, sage::bwd::BKT) ||
      // d = 128: 16-query x 32-channel boxes, row-major; d = 64: 32 x 32 boxes, 128-byte swizzle
      !(D == 128 ? make_map(&tdq, dqacc, 4, D, rows, sage::bwd::kDqCols, sage::bwd::kDqRows, false)
                 : make_map(&tdq, dqacc, 4, D, rows, 32, 32)))
    return SAGE_ERR_CUDA;
  sage::bwd::Args a;
  a.q_scale = qb->q_scale;
  a.k_scale = qb->k_scale;
  a.do_scale = dos;
  a.lse = lse;
  a.dvec = dvec;
  a.k_raw = k;
  a.k_inv_rms = qb->k_inv_rms;
  a.dk = dk;
  a.dv = dv;
  a.BH = BH;
  a.N = N;
  a.q_block = p->q_block;
  a.causal = p->causal;
  a.qknorm = p->qknorm;
  a.tau = tau_of(p);
  a.scale_log2 = a.tau * 1.4426950408889634f;
  a.k_bias = qb->k_bias;
  a.q_mean = qb->q_mean;
  a.dk_acc = dk_acc;
  a.dv_acc = dv_acc;
  a.acc_add = acc_add;
  const size_t smem = sage::bwd::smem_bytes<D>();
  auto kern = p->qsmooth ? sage::bwd::attn_bwd_kernel<T, D, true>
                         : sage::bwd::attn_bwd_kernel<T, D, false>;
  if (set_smem(kern, smem) != SAGE_OK) return SAGE_ERR_CUDA;
  // The kernel moves registers between warpgroups (setmaxnreg); the split is sized for a launch
  // allocation of exactly kLaunchRegs per thread.  Any other allocation could leave the
  // increasing warpgroups waiting, so refuse to launch.
  if (launch_regs(kern) != sage::bwd::kLaunchRegs) return SAGE_ERR_UNSUPPORTED;
  kern<<<BH * (N / sage::bwd::BKT), sage::bwd::kThreads, smem, st>>>(tqc, tkc, tdoc, tdo, tv, tdq,
                                                                     a);
  return launch_status();
}

// ---- context parallelism: merge of partial results, key-side finalize ---------------------
template <typename T, int D>
int run_merge(const sage_params* p, float* o_acc, float* lse_acc, const float* o_part,
              const float* lse_part, void* out, cudaStream_t st) {
  // N is a multiple of 128, so rows * D / 8 threads fill whole 256-thread blocks
  const size_t rows = static_cast<size_t>(p->B) * p->H * p->N;
  const size_t blocks = rows * (D / 8) / 256;
  sage::attn_merge_kernel<T, D><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
      o_acc, lse_acc, o_part, lse_part, reinterpret_cast<T*>(out));
  return launch_status();
}

template <typename T, int D>
int run_kv_finalize(const sage_params* p, const void* k, const sage_qbufs* qb,
                    const float* dk_acc, const float* dv_acc, void* dk, void* dv, cudaStream_t st) {
  const size_t rows = static_cast<size_t>(p->B) * p->H * p->N;
  const int grid = static_cast<int>(rows / kRowsPerCta);
  sage::dq_finalize_kernel<T, D><<<grid, kRowThreads, 0, st>>>(
      dk_acc, reinterpret_cast<const T*>(k), qb ? qb->k_inv_rms : nullptr,
      reinterpret_cast<T*>(dk), p->qknorm);
  sage::dq_finalize_kernel<T, D><<<grid, kRowThreads, 0, st>>>(
      dv_acc, nullptr, nullptr, reinterpret_cast<T*>(dv), 0);
  return launch_status();
}

int bwd_stage(int stage, const sage_params* p, const void* q, const void* k, const void* v,
              const sage_qbufs* qb, const void* o, const float* lse, const void* dout, void* dq,
              void* dk, void* dv, void* workspace, size_t workspace_bytes, void* stream) {
  int s = check_params(p);
  if (s != SAGE_OK) return s;
  if (stage < 0 || stage > 2) return SAGE_ERR_INVALID_ARG;
  if ((s = check_qbufs(p, qb)) != SAGE_OK) return s;
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return SAGE_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, o, lse, dout, dq, dk, dv, workspace};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return SAGE_ERR_ALIGNMENT;
  if (!workspace || workspace_bytes < bwd_ws(p).total) return SAGE_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool bf = p->dtype == SAGE_BF16;
  if (p->d == 128)
    return bf ? run_bwd<__nv_bfloat16, 128>(stage, p, q, k, v, qb, o, lse, dout, dq, dk, dv,
                                             workspace, st)
              : run_bwd<__half, 128>(stage, p, q, k, v, qb, o, lse, dout, dq, dk, dv, workspace,
                                     st);
  return bf ? run_bwd<__nv_bfloat16, 64>(stage, p, q, k, v, qb, o, lse, dout, dq, dk, dv,
                                          workspace, st)
            : run_bwd<__half, 64>(stage, p, q, k, v, qb, o, lse, dout, dq, dk, dv, workspace, st);
}

// ---- NVFP4 variant -----------------------------------------------------------------------
int check_fp4(const sage_params* p) {
  const int s = check_params(p);
  if (s != SAGE_OK) return s;
  return p->qsmooth ? SAGE_ERR_UNSUPPORTED : SAGE_OK;
}

int check_fp4bufs(const sage_params* p, const sage_fp4_bufs* fb) {
  if (!fb || !fb->q_fp4 || !fb->k_fp4 || !fb->q_sf || !fb->k_sf || !fb->q_genc || !fb->k_genc)
    return SAGE_ERR_INVALID_ARG;
  if (p->ksmooth && !fb->k_mean) return SAGE_ERR_INVALID_ARG;
  if ((fb->q_fp4_t == nullptr) != (fb->q_sf_t == nullptr) ||
      (fb->k_fp4_t == nullptr) != (fb->k_sf_t == nullptr))
    return SAGE_ERR_INVALID_ARG;
  const void* ptrs[] = {fb->q_fp4, fb->k_fp4, fb->q_sf, fb->k_sf, fb->q_genc, fb->k_genc,
                        fb->k_mean, fb->q_inv_rms, fb->k_inv_rms, fb->q_fp4_t, fb->k_fp4_t,
                        fb->q_sf_t, fb->k_sf_t};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return SAGE_ERR_ALIGNMENT;
  return SAGE_OK;
}

// Workspace: K-mean partials (ksmooth) then the 2 x BH global maxima.
struct Fp4Ws {
  size_t gmax, total;
};
Fp4Ws fp4_ws(const sage_params* p) {
  Fp4Ws w;
  // K statistics: column sums, maxima and minima per 64-token block (ksmooth)
  w.gmax = p->ksmooth ? align_up(3 * prologue_partials(p) * 4) : 0;
  w.total = align_up(w.gmax + 2 * static_cast<size_t>(p->B) * p->H * 4);
  return w;
}

template <typename T, int D>
int run_fp4_prologue(const sage_params* p, const void* q, const void* k, const sage_fp4_bufs* fb,
                     void* ws, cudaStream_t st) {
  const int BH = p->B * p->H, N = p->N;
  const Fp4Ws w = fp4_ws(p);
  uint8_t* wsb = reinterpret_cast<uint8_t*>(ws);
  uint32_t* gmax = reinterpret_cast<uint32_t*>(wsb + w.gmax);
  if (cudaMemsetAsync(gmax, 0, 2 * static_cast<size_t>(BH) * 4, st) != cudaSuccess)
    return SAGE_ERR_CUDA;
  if (p->ksmooth) {
    // K's mean and, from its column extremes, K's global maximum (gmax[BH + bh])
    const int total = BH * (N / 64);
    const int per_cta = (kRowThreads / 32) * (32 / (D / 8));
    float* partials = reinterpret_cast<float*>(wsb);
    sage::prologue_kstats_kernel<T, D, true>
        <<<(total + per_cta - 1) / per_cta, kRowThreads, 0, st>>>(
            reinterpret_cast<const T*>(k), partials, total, p->qknorm, p->rms_eps);
    sage::prologue_kmean_kernel<D, true><<<BH, D, 0, st>>>(partials, fb->k_mean, N / 64, N,
                                                           total, gmax + BH);
  }
  sage::fp4::PrologueArgs a;
  a.src[0] = q;
  a.src[1] = k;
  a.codes[0] = fb->q_fp4;
  a.codes[1] = fb->k_fp4;
  a.sf[0] = fb->q_sf;
  a.sf[1] = fb->k_sf;
  a.genc[0] = fb->q_genc;
  a.genc[1] = fb->k_genc;
  a.inv_rms[0] = fb->q_inv_rms;
  a.inv_rms[1] = fb->k_inv_rms;
  a.k_mean = fb->k_mean;
  a.gmax = gmax;
  a.codes_t[0] = fb->q_fp4_t;
  a.codes_t[1] = fb->k_fp4_t;
  a.sf_t[0] = fb->q_sf_t;
  a.sf_t[1] = fb->k_sf_t;
  a.BH = BH;
  a.N = N;
  a.qknorm = p->qknorm;
  a.ksmooth = p->ksmooth;
  a.eps = p->rms_eps;
  const int grid = 2 * BH * (N / kRowsPerCta);
  // the absolute-maximum pass covers Q, and K too unless the K statistics gave its maximum
  // (blocks [0, grid/2) are Q's)
  sage::fp4::prologue_amax_kernel<T, D>
      <<<p->ksmooth ? grid / 2 : grid, sage::kQuantThreads, 0, st>>>(a);
  // the sequence views stage each chunk through shared memory
  const bool seq = fb->q_fp4_t != nullptr || fb->k_fp4_t != nullptr;
  const size_t smem = seq ? sage::fp4::seq_smem_bytes<D>() : 0;
  if (seq && set_smem(sage::fp4::prologue_quant_kernel<T, D>, smem) != SAGE_OK)
    return SAGE_ERR_CUDA;
  sage::fp4::prologue_quant_kernel<T, D><<<grid, sage::kQuantThreads, smem, st>>>(a);
  return launch_status();
}

template <typename T, int D>
int run_fp4_fwd(const sage_params* p, const sage_fp4_bufs* fb, const void* v, void* o,
                float* lse, cudaStream_t st) {
  const int BH = p->B * p->H, N = p->N;
  const uint64_t rows = static_cast<uint64_t>(BH) * N;
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, fb->q_fp4, 1, D / 2, rows, D / 2, sage::fp4::BM) ||
      !make_map(&tk, fb->k_fp4, 1, D / 2, rows, D / 2, sage::fp4::BKV) ||
      !make_map(&tv, v, 2, D, rows, 64, sage::fp4::BKV))
    return SAGE_ERR_CUDA;
  sage::fp4::Args a;
  a.q_sf = fb->q_sf;
  a.k_sf = fb->k_sf;
  a.q_genc = fb->q_genc;
  a.k_genc = fb->k_genc;
  a.o = o;
  a.lse = lse;
  a.N = N;
  a.causal = p->causal;
  a.scale_log2 = tau_of(p) * 1.4426950408889634f;
  const size_t smem = sage::fp4::smem_bytes<T, D>();
  auto kern = sage::fp4::attn_fwd_kernel<T, D>;
  if (set_smem(kern, smem) != SAGE_OK) return SAGE_ERR_CUDA;
  // register split between warpgroups (setmaxnreg) assumes exactly kLaunchRegs at launch
  if (launch_regs(kern) != sage::fp4::kLaunchRegs) return SAGE_ERR_UNSUPPORTED;
  kern<<<BH * (N / sage::fp4::BM), sage::fp4::kThreads, smem, st>>>(tq, tk, tv, a);
  return launch_status();
}

// Backward workspace: D = rowsum(dO o O) [BH, N] then the float32 dQ accumulator [BH, N, d].
struct Fp4BwdWs {
  size_t dvec, dq, total;
};
Fp4BwdWs fp4_bwd_ws(const sage_params* p) {
  const size_t BH = static_cast<size_t>(p->B) * p->H, N = p->N, d = p->d;
  Fp4BwdWs w;
  w.dvec = 0;
  w.dq = align_up(BH * N * 4);
  w.total = align_up(w.dq + BH * N * d * 4);
  return w;
}

// stage 0: preprocess (D, the dQ accumulator cleared); 1: main kernel; 2: dq finalize.
template <typename T, int D>
int run_fp4_bwd(int stage, const sage_params* p, const void* q, const void* k, const void* v,
                const sage_fp4_bufs* fb, const void* o, const float* lse, const void* dout,
                void* dq, void* dk, void* dv, void* ws, cudaStream_t st) {
  const int BH = p->B * p->H, N = p->N;
  const uint64_t rows = static_cast<uint64_t>(BH) * N;
  const Fp4BwdWs w = fp4_bwd_ws(p);
  uint8_t* wsb = reinterpret_cast<uint8_t*>(ws);
  float* dvec = reinterpret_cast<float*>(wsb + w.dvec);
  float* dqacc = reinterpret_cast<float*>(wsb + w.dq);
  if (stage == 0) {
    // D and the cleared dQ accumulator (no INT8 dO codes: dO enters the MMAs in 16 bits)
    sage::bwd_preprocess_kernel<T, D>
        <<<static_cast<int>(rows / kRowsPerCta), sage::kQuantThreads, 0, st>>>(
            reinterpret_cast<const T*>(o), reinterpret_cast<const T*>(dout), dvec, nullptr,
            nullptr, dqacc, N, p->q_block);
    return launch_status();
  }
  if (stage == 2) {
    sage::dq_finalize_kernel<T, D><<<static_cast<int>(rows / kRowsPerCta), kRowThreads, 0, st>>>(
        dqacc, reinterpret_cast<const T*>(q), fb->q_inv_rms, reinterpret_cast<T*>(dq),
        p->qknorm);
    return launch_status();
  }
  CUtensorMap tqc, tkc, tqs, tks, tdo, tv, tdq;
  const uint64_t seq_rows = static_cast<uint64_t>(BH) * D;
  if (!make_map(&tqc, fb->q_fp4, 1, D / 2, rows, D / 2, sage::fp4::bwd::BQ) ||
      !make_map(&tkc, fb->k_fp4, 1, D / 2, rows, D / 2, sage::fp4::bwd::BKT) ||
      !make_map(&tqs, fb->q_fp4_t, 1, N / 2, seq_rows, 64, D) ||
      !make_map(&tks, fb->k_fp4_t, 1, N / 2, seq_rows, 64, D) ||
      !make_map(&tdo, dout, 2, D, rows, 64, sage::fp4::bwd::BQ) ||
      !make_map(&tv, v, 2, D, rows, 64, sage::fp4::bwd::BKT) ||
      !make_map(&tdq, dqacc, 4, D, rows, 32, 32))  // 32 x 32 float32 boxes, 128-byte swizzle
    return SAGE_ERR_CUDA;
  sage::fp4::bwd::Args a;
  a.q_sf = fb->q_sf;
  a.k_sf = fb->k_sf;
  a.q_sf_t = fb->q_sf_t;
  a.k_sf_t = fb->k_sf_t;
  a.q_genc = fb->q_genc;
  a.k_genc = fb->k_genc;
  a.lse = lse;
  a.dvec = dvec;
  a.k_raw = k;
  a.k_inv_rms = fb->k_inv_rms;
  a.dk = dk;
  a.dv = dv;
  a.N = N;
  a.causal = p->causal;
  a.qknorm = p->qknorm;
  a.tau = tau_of(p);
  a.scale_log2 = a.tau * 1.4426950408889634f;
  const size_t smem = sage::fp4::bwd::smem_bytes<T, D>();
  auto kern = sage::fp4::bwd::attn_bwd_kernel<T, D>;
  if (set_smem(kern, smem) != SAGE_OK) return SAGE_ERR_CUDA;
  // register split between warpgroups (setmaxnreg) assumes exactly kLaunchRegs at launch
  if (launch_regs(kern) != sage::fp4::bwd::kLaunchRegs) return SAGE_ERR_UNSUPPORTED;
  kern<<<BH * (N / sage::fp4::bwd::BKT), sage::fp4::bwd::kThreads, smem, st>>>(tqc, tkc, tqs,
                                                                             tks, tdo, tv, tdq,
                                                                             a);
  return launch_status();
}

int fp4_bwd_stage(int stage, const sage_params* p, const void* q, const void* k, const void* v,
                  const sage_fp4_bufs* fb, const void* o, const float* lse, const void* dout,
                  void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
                  void* stream) {
  int s = check_fp4(p);
  if (s != SAGE_OK) return s;
  if (stage < 0 || stage > 2) return SAGE_ERR_INVALID_ARG;
  if ((s = check_fp4bufs(p, fb)) != SAGE_OK) return s;
  if (!fb->q_fp4_t || !fb->k_fp4_t) return SAGE_ERR_INVALID_ARG;
  if (p->qknorm && (!fb->q_inv_rms || !fb->k_inv_rms)) return SAGE_ERR_INVALID_ARG;
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return SAGE_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, o, lse, dout, dq, dk, dv, workspace};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return SAGE_ERR_ALIGNMENT;
  if (!workspace || workspace_bytes < fp4_bwd_ws(p).total) return SAGE_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool bf = p->dtype == SAGE_BF16;
  if (p->d == 128)
    return bf ? run_fp4_bwd<__nv_bfloat16, 128>(stage, p, q, k, v, fb, o, lse, dout, dq, dk, dv,
                                                 workspace, st)
              : run_fp4_bwd<__half, 128>(stage, p, q, k, v, fb, o, lse, dout, dq, dk, dv,
                                         workspace, st);
  return bf ? run_fp4_bwd<__nv_bfloat16, 64>(stage, p, q, k, v, fb, o, lse, dout, dq, dk, dv,
                                              workspace, st)
            : run_fp4_bwd<__half, 64>(stage, p, q, k, v, fb, o, lse, dout, dq, dk, dv, workspace,
                                      st);
}

// ---- end-to-end pipeline over host buffers -------------------------------------------------
// One chunk slot of sage_fwd_bwd_host's device workspace: the chunk's 16-bit inputs and
// outputs, its quantized views, LSE and the prologue / backward scratch; offsets from the
// slot's start, each 256-byte aligned.
struct HostSlot {
  size_t in[4], out[4], qc, kc, vc, qs, ks, vs, qinv, kinv, kmean, qmean, kbias, lse, wpro, wbwd;
  size_t total;
};
HostSlot host_slot(const sage_params* cp) {  // cp->B = the largest chunk's batch
  const size_t BH = static_cast<size_t>(cp->B) * cp->H, N = cp->N, d = cp->d, e = BH * N * d;
  HostSlot s;
  size_t at = 0;
  auto take = [&](size_t bytes) {
    const size_t here = at;
    at = align_up(at + bytes);
    return here;
  };
  for (int i = 0; i < 4; ++i) s.in[i] = take(e * 2);
  for (int i = 0; i < 4; ++i) s.out[i] = take(e * 2);
  s.qc = take(e);
  s.kc = take(e);
  s.vc = take(e);
  s.qs = take(BH * (N / cp->q_block) * 4);
  s.ks = take(BH * (N / cp->k_block) * 4);
  s.vs = take(BH * (N / cp->k_block) * 4);
  s.qinv = take(BH * N * 4);
  s.kinv = take(BH * N * 4);
  s.kmean = take(BH * d * 4);
  s.qmean = take(BH * d * 4);
  s.kbias = take(BH * N * 4);
  s.lse = take(BH * N * 4);
  s.wpro = take(prologue_ws(cp));
  s.wbwd = take(bwd_ws(cp).total);
  s.total = at;
  return s;
}
sage_params largest_chunk(const sage_params* p, int chunks) {
  sage_params cp = *p;
  cp.B = (p->B + chunks - 1) / chunks;
  return cp;
}

// ---- prologue scratch for callers that cannot allocate -------------------------------------
// A fixed device array that sage_quant_prologue_noalloc uses instead of a caller workspace for
// the K-smoothing column sums.  Every device that loads the library holds it until exit.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

// Device address of g_noalloc_scratch in the calling thread's current context.  In host code
// the array's name is only a host-side stand-in, so kernels must be given this address.  The
// address belongs to the copy of the library's device code loaded in that context: a driver
// context other than the device's primary one, or the primary context re-created after
// cudaDeviceReset, holds its own copy at another address.  So it is looked up on every call
// (a host-side table lookup once the code is loaded there, which allocates nothing) rather than
// cached per device.
int noalloc_scratch(void** out) {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
    return SAGE_ERR_CUDA;
  *out = ptr;
  return SAGE_OK;
}

}  // namespace

extern "C" {

size_t sage_workspace_bytes(const sage_params* p, int which) {
  if (check_params(p) != SAGE_OK) return 0;
  if (which == 0) return prologue_ws(p);
  if (which == 1) return 0;
  if (which == 2) return bwd_ws(p).total;
  return 0;
}

int sage_quant_prologue(const sage_params* p, const void* q, const void* k, const void* v,
                        const sage_qbufs* out, void* workspace, size_t workspace_bytes,
                        void* stream) {
  int s = check_params(p);
  if (s != SAGE_OK) return s;
  if (!q || !k || !v) return SAGE_ERR_INVALID_ARG;
  if ((s = check_qbufs(p, out)) != SAGE_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return SAGE_ERR_ALIGNMENT;
  const size_t need = prologue_ws(p);
  if (need > 0 && (!workspace || workspace_bytes < need)) return SAGE_ERR_WORKSPACE;
  if (workspace && !aligned16(workspace)) return SAGE_ERR_ALIGNMENT;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool bf = p->dtype == SAGE_BF16;
  if (p->d == 128)
    return bf ? run_prologue<__nv_bfloat16, 128>(p, q, k, v, out, workspace, st)
              : run_prologue<__half, 128>(p, q, k, v, out, workspace, st);
  return bf ? run_prologue<__nv_bfloat16, 64>(p, q, k, v, out, workspace, st)
            : run_prologue<__half, 64>(p, q, k, v, out, workspace, st);
}

int sage_quant_prologue_noalloc(const sage_params* p, const void* q, const void* k,
                                const void* v, const sage_qbufs* out, void* stream) {
  int s = check_params(p);
  if (s != SAGE_OK) return s;
  if (!q || !k || !v) return SAGE_ERR_INVALID_ARG;
  if ((s = check_qbufs(p, out)) != SAGE_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return SAGE_ERR_ALIGNMENT;
  const size_t need = prologue_ws(p);
  if (need > kNoAllocScratchBytes) return SAGE_ERR_WORKSPACE;
  void* ws = nullptr;
  if (need > 0 && (s = noalloc_scratch(&ws)) != SAGE_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool bf = p->dtype == SAGE_BF16;
  if (p->d == 128)
    return bf ? run_prologue<__nv_bfloat16, 128>(p, q, k, v, out, ws, st)
              : run_prologue<__half, 128>(p, q, k, v, out, ws, st);
  return bf ? run_prologue<__nv_bfloat16, 64>(p, q, k, v, out, ws, st)
            : run_prologue<__half, 64>(p, q, k, v, out, ws, st);
}

int sage_attn_fwd(const sage_params* p, const sage_qbufs* qb, void* o, float* lse,
                  void* workspace, size_t workspace_bytes, void* stream) {
  (void)workspace;
  (void)workspace_bytes;
  int s = check_params(p);
  if (s != SAGE_OK) return s;
  if ((s = check_qbufs(p, qb)) != SAGE_OK) return s;
  if (!o || !lse) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(o) || !aligned16(lse)) return SAGE_ERR_ALIGNMENT;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool bf = p->dtype == SAGE_BF16;
  if (p->d == 128)
    return bf ? run_fwd<__nv_bfloat16, 128>(p, qb, o, lse, st)
              : run_fwd<__half, 128>(p, qb, o, lse, st);
  return bf ? run_fwd<__nv_bfloat16, 64>(p, qb, o, lse, st)
            : run_fwd<__half, 64>(p, qb, o, lse, st);
}

int sage_attn_bwd(const sage_params* p, const void* q, const void* k, const void* v,
                  const sage_qbufs* qb, const void* o, const float* lse, const void* dout,
                  void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
                  void* stream) {
  for (int stage = 0; stage < 3; ++stage) {
    const int s = bwd_stage(stage, p, q, k, v, qb, o, lse, dout, dq, dk, dv, workspace,
                            workspace_bytes, stream);
    if (s != SAGE_OK) return s;
  }
  return SAGE_OK;
}

int sage_attn_bwd_stage(int stage, const sage_params* p, const void* q, const void* k,
                        const void* v, const sage_qbufs* qb, const void* o, const float* lse,
                        const void* dout, void* dq, void* dk, void* dv, void* workspace,
                        size_t workspace_bytes, void* stream) {
  return bwd_stage(stage, p, q, k, v, qb, o, lse, dout, dq, dk, dv, workspace, workspace_bytes,
                   stream);
}

size_t sage_fwd_bwd_host_workspace_bytes(const sage_params* p, int chunks) {
  if (check_params(p) != SAGE_OK || chunks < 1) return 0;
  chunks = chunks < p->B ? chunks : p->B;
  const sage_params cp = largest_chunk(p, chunks);
  return 2 * host_slot(&cp).total;
}

int sage_fwd_bwd_host(const sage_params* p, const void* q, const void* k, const void* v,
                      const void* dout, void* o, void* dq, void* dk, void* dv, int chunks,
                      void* workspace, size_t workspace_bytes, void* stream_in,
                      void* stream_compute, void* stream_out) {
  int s = check_params(p);
  if (s != SAGE_OK) return s;
  if (!q || !k || !v || !dout || !o || !dq || !dk || !dv || chunks < 1)
    return SAGE_ERR_INVALID_ARG;
  chunks = chunks < p->B ? chunks : p->B;
  const sage_params cp = largest_chunk(p, chunks);
  const HostSlot L = host_slot(&cp);
  if (!workspace || workspace_bytes < 2 * L.total) return SAGE_ERR_WORKSPACE;
  if (!aligned16(workspace)) return SAGE_ERR_ALIGNMENT;
  cudaStream_t sin = reinterpret_cast<cudaStream_t>(stream_in);
  cudaStream_t scomp = reinterpret_cast<cudaStream_t>(stream_compute);
  cudaStream_t sout = reinterpret_cast<cudaStream_t>(stream_out);
  // [0]: a slot's inputs are on the device, [1]: its kernels are done, [2]: its results left
  cudaEvent_t ev[3][2] = {};
  for (auto& row : ev)
    for (auto& e : row)
      if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) s = SAGE_ERR_CUDA;
  const void* hin[4] = {q, k, v, dout};
  void* hout[4] = {o, dq, dk, dv};
  const size_t per_b = static_cast<size_t>(p->H) * p->N * p->d * 2;  // bytes per batch entry
  for (int c = 0; c < chunks && s == SAGE_OK; ++c) {
    const int b0 = static_cast<int>(static_cast<long long>(p->B) * c / chunks);
    const int b1 = static_cast<int>(static_cast<long long>(p->B) * (c + 1) / chunks);
    const int slot = c & 1;
    uint8_t* base = reinterpret_cast<uint8_t*>(workspace) + slot * L.total;
    sage_params pc = *p;
    pc.B = b1 - b0;
    const size_t bytes = static_cast<size_t>(b1 - b0) * per_b, off = b0 * per_b;
    auto ok = [&](cudaError_t e) {
      if (e != cudaSuccess && s == SAGE_OK) s = SAGE_ERR_CUDA;
    };
    // host -> device: the slot's previous chunk (c - 2) must have finished reading its inputs
    if (c >= 2) ok(cudaStreamWaitEvent(sin, ev[1][slot], 0));
    for (int i = 0; i < 4; ++i)
      ok(cudaMemcpyAsync(base + L.in[i], static_cast<const uint8_t*>(hin[i]) + off, bytes,
                         cudaMemcpyHostToDevice, sin));
    ok(cudaEventRecord(ev[0][slot], sin));
    // kernels: after the inputs arrived and chunk c - 2's results left the slot
    ok(cudaStreamWaitEvent(scomp, ev[0][slot], 0));
    if (c >= 2) ok(cudaStreamWaitEvent(scomp, ev[2][slot], 0));
    if (s != SAGE_OK) break;
    sage_qbufs qb;
    qb.q_codes = reinterpret_cast<int8_t*>(base + L.qc);
    qb.k_codes = reinterpret_cast<int8_t*>(base + L.kc);
    qb.v_codes = reinterpret_cast<int8_t*>(base + L.vc);
    qb.q_scale = reinterpret_cast<float*>(base + L.qs);
    qb.k_scale = reinterpret_cast<float*>(base + L.ks);
    qb.v_scale = reinterpret_cast<float*>(base + L.vs);
    qb.q_inv_rms = reinterpret_cast<float*>(base + L.qinv);
    qb.k_inv_rms = reinterpret_cast<float*>(base + L.kinv);
    qb.k_mean = reinterpret_cast<float*>(base + L.kmean);
    qb.q_mean = reinterpret_cast<float*>(base + L.qmean);
    qb.k_bias = reinterpret_cast<float*>(base + L.kbias);
    float* lse = reinterpret_cast<float*>(base + L.lse);
    void* din[4];
    void* dres[4];
    for (int i = 0; i < 4; ++i) {
      din[i] = base + L.in[i];
      dres[i] = base + L.out[i];
    }
    s = sage_quant_prologue(&pc, din[0], din[1], din[2], &qb, base + L.wpro, prologue_ws(&pc),
                            scomp);
    if (s == SAGE_OK) s = sage_attn_fwd(&pc, &qb, dres[0], lse, nullptr, 0, scomp);
    if (s == SAGE_OK)
      s = sage_attn_bwd(&pc, din[0], din[1], din[2], &qb, dres[0], lse, din[3], dres[1],
                        dres[2], dres[3], base + L.wbwd, bwd_ws(&pc).total, scomp);
    if (s != SAGE_OK) break;
    ok(cudaEventRecord(ev[1][slot], scomp));
    // device -> host once the kernels are done
    ok(cudaStreamWaitEvent(sout, ev[1][slot], 0));
    for (int i = 0; i < 4; ++i)
      ok(cudaMemcpyAsync(static_cast<uint8_t*>(hout[i]) + off, base + L.out[i], bytes,
                         cudaMemcpyDeviceToHost, sout));
    ok(cudaEventRecord(ev[2][slot], sout));
  }
  // whatever happened, nothing of this call is left in flight when it returns
  for (cudaStream_t st : {sin, scomp, sout})
    if (cudaStreamSynchronize(st) != cudaSuccess && s == SAGE_OK) s = SAGE_ERR_CUDA;
  for (auto& row : ev)
    for (auto& e : row)
      if (e) cudaEventDestroy(e);
  return s;
}

size_t sage_fp4_workspace_bytes(const sage_params* p, int which) {
  if (check_fp4(p) != SAGE_OK) return 0;
  return which == 0 ? fp4_ws(p).total : which == 2 ? fp4_bwd_ws(p).total : 0;
}

int sage_fp4_quant_prologue(const sage_params* p, const void* q, const void* k,
                            const sage_fp4_bufs* out, void* workspace, size_t workspace_bytes,
                            void* stream) {
  int s = check_fp4(p);
  if (s != SAGE_OK) return s;
  if (!q || !k) return SAGE_ERR_INVALID_ARG;
  if ((s = check_fp4bufs(p, out)) != SAGE_OK) return s;
  if (!aligned16(q) || !aligned16(k)) return SAGE_ERR_ALIGNMENT;
  if (!workspace || workspace_bytes < fp4_ws(p).total) return SAGE_ERR_WORKSPACE;
  if (!aligned16(workspace)) return SAGE_ERR_ALIGNMENT;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool bf = p->dtype == SAGE_BF16;
  if (p->d == 128)
    return bf ? run_fp4_prologue<__nv_bfloat16, 128>(p, q, k, out, workspace, st)
              : run_fp4_prologue<__half, 128>(p, q, k, out, workspace, st);
  return bf ? run_fp4_prologue<__nv_bfloat16, 64>(p, q, k, out, workspace, st)
            : run_fp4_prologue<__half, 64>(p, q, k, out, workspace, st);
}

int sage_fp4_attn_fwd(const sage_params* p, const sage_fp4_bufs* fb, const void* v, void* o,
                      float* lse, void* stream) {
  int s = check_fp4(p);
  if (s != SAGE_OK) return s;
  if ((s = check_fp4bufs(p, fb)) != SAGE_OK) return s;
  if (!v || !o || !lse) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(v) || !aligned16(o) || !aligned16(lse)) return SAGE_ERR_ALIGNMENT;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool bf = p->dtype == SAGE_BF16;
  if (p->d == 128)
    return bf ? run_fp4_fwd<__nv_bfloat16, 128>(p, fb, v, o, lse, st)
              : run_fp4_fwd<__half, 128>(p, fb, v, o, lse, st);
  return bf ? run_fp4_fwd<__nv_bfloat16, 64>(p, fb, v, o, lse, st)
            : run_fp4_fwd<__half, 64>(p, fb, v, o, lse, st);
}

int sage_fp4_attn_bwd(const sage_params* p, const void* q, const void* k, const void* v,
                      const sage_fp4_bufs* fb, const void* o, const float* lse, const void* dout,
                      void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
                      void* stream) {
  for (int stage = 0; stage < 3; ++stage) {
    const int s = fp4_bwd_stage(stage, p, q, k, v, fb, o, lse, dout, dq, dk, dv, workspace,
                                workspace_bytes, stream);
    if (s != SAGE_OK) return s;
  }
  return SAGE_OK;
}

int sage_fp4_attn_bwd_stage(int stage, const sage_params* p, const void* q, const void* k,
                            const void* v, const sage_fp4_bufs* fb, const void* o,
                            const float* lse, const void* dout, void* dq, void* dk, void* dv,
                            void* workspace, size_t workspace_bytes, void* stream) {
  return fp4_bwd_stage(stage, p, q, k, v, fb, o, lse, dout, dq, dk, dv, workspace,
                       workspace_bytes, stream);
}

int sage_last_device_status(void* stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return SAGE_ERR_CUDA;
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, sage::g_status, sizeof(int)) != cudaSuccess) return SAGE_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(sage::g_status, &zero, sizeof(int)) != cudaSuccess)
    return SAGE_ERR_CUDA;
  return v;
}

const char* sage_status_string(int status) {
  switch (status) {
    case SAGE_OK: return "SAGE_OK";
    case SAGE_ERR_INVALID_ARG: return "SAGE_ERR_INVALID_ARG";
    case SAGE_ERR_UNSUPPORTED: return "SAGE_ERR_UNSUPPORTED";
    case SAGE_ERR_ALIGNMENT: return "SAGE_ERR_ALIGNMENT";
    case SAGE_ERR_WORKSPACE: return "SAGE_ERR_WORKSPACE";
    case SAGE_ERR_CUDA: return "SAGE_ERR_CUDA";
    case SAGE_ERR_TIMEOUT: return "SAGE_ERR_TIMEOUT";
    default: return "SAGE_ERR_UNKNOWN";
  }
}

int sage_debug_qk_int32(const sage_params* p, const sage_qbufs* qb, int bh, int q_tile,
                        int32_t* s_out, void* stream) {
  int s = check_params(p);
  if (s != SAGE_OK) return s;
  if ((s = check_qbufs(p, qb)) != SAGE_OK) return s;
  if (!s_out) return SAGE_ERR_INVALID_ARG;
  if (bh < 0 || bh >= p->B * p->H || q_tile < 0 || q_tile >= p->N / 128)
    return SAGE_ERR_INVALID_ARG;
  const uint64_t rows = static_cast<uint64_t>(p->B) * p->H * p->N;
  CUtensorMap tq, tk;
  if (!make_map(&tq, qb->q_codes, 1, p->d, rows, p->d, 128) ||
      !make_map(&tk, qb->k_codes, 1, p->d, rows, p->d, 64))
    return SAGE_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (p->d == 128) {
    const size_t smem = sizeof(sage::dbg::QkSmem<128>) + 1024;
    if (set_smem(sage::dbg::debug_qk_kernel<128>, smem) != SAGE_OK) return SAGE_ERR_CUDA;
    sage::dbg::debug_qk_kernel<128><<<1, 128, smem, st>>>(tq, tk, bh, q_tile, p->N, s_out);
  } else {
    const size_t smem = sizeof(sage::dbg::QkSmem<64>) + 1024;
    if (set_smem(sage::dbg::debug_qk_kernel<64>, smem) != SAGE_OK) return SAGE_ERR_CUDA;
    sage::dbg::debug_qk_kernel<64><<<1, 128, smem, st>>>(tq, tk, bh, q_tile, p->N, s_out);
  }
  return launch_status();
}

int sage_debug_umma_gemm(int kind, int a_mn_major, int b_mn_major, int N, int K, const void* A,
                         const void* B, void* C, void* stream) {
  if (kind < 0 || kind > 2 || !A || !B || !C) return SAGE_ERR_INVALID_ARG;
  if ((N != 64 && N != 128) || (K != 64 && K != 128)) return SAGE_ERR_UNSUPPORTED;
  if (kind != 0 && (a_mn_major || b_mn_major)) return SAGE_ERR_UNSUPPORTED;
  if (!aligned16(A) || !aligned16(B) || !aligned16(C)) return SAGE_ERR_ALIGNMENT;
  const int M = 128;
  CUtensorMap ta, tb;
  bool ok;
  if (kind == 0) {
    ok = (a_mn_major ? make_map(&ta, A, 1, M, K, M, K) : make_map(&ta, A, 1, K, M, K, M)) &&
         (b_mn_major ? make_map(&tb, B, 1, N, K, N, K) : make_map(&tb, B, 1, K, N, K, N));
  } else {
    ok = make_map(&ta, A, 2, K, M, 64, M) && make_map(&tb, B, 2, K, N, 64, N);
  }
  if (!ok) return SAGE_ERR_CUDA;
  const size_t smem = sizeof(sage::dbg::GemmSmem) + 1024;
  if (set_smem(sage::dbg::debug_gemm_kernel, smem) != SAGE_OK) return SAGE_ERR_CUDA;
  sage::dbg::debug_gemm_kernel<<<1, 128, smem, reinterpret_cast<cudaStream_t>(stream)>>>(
      ta, tb, kind, a_mn_major, b_mn_major, N, K, C);
  return launch_status();
}

int sage_debug_wait_timeout(int limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 1000000) return SAGE_ERR_INVALID_ARG;
  sage::dbg::debug_wait_kernel<<<1, 128, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<unsigned long long>(limit_us) * 1000ull);
  return launch_status();
}

int sage_mma_peak(int kind, int n_ctas, int groups, const void* fill, size_t fill_bytes,
                  void* stream) {
  if (kind < 0 || kind > 2 || !fill) return SAGE_ERR_INVALID_ARG;
  if (n_ctas < 1 || n_ctas > 65535 || groups < 1 || groups > (1 << 26))
    return SAGE_ERR_INVALID_ARG;
  if (fill_bytes < static_cast<size_t>(sage::dbg::kPeakFillBytes)) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(fill)) return SAGE_ERR_ALIGNMENT;
  const size_t smem = sizeof(sage::dbg::PeakSmem) + 1024;
  if (set_smem(sage::dbg::mma_peak_kernel, smem) != SAGE_OK) return SAGE_ERR_CUDA;
  sage::dbg::mma_peak_kernel<<<n_ctas, 128, smem, reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint4*>(fill), kind, groups);
  return launch_status();
}

// ---- context parallelism ------------------------------------------------------------------
int sage_quant_prologue_part(const sage_params* p, const void* q, const void* k, const void* v,
                             const sage_qbufs* out, void* workspace, size_t workspace_bytes,
                             int part, void* stream) {
  int s = check_params(p);
  if (s != SAGE_OK) return s;
  if (part != 0 && part != 1) return SAGE_ERR_INVALID_ARG;
  if (p->qsmooth) return SAGE_ERR_UNSUPPORTED;
  if (!q || !k || !v) return SAGE_ERR_INVALID_ARG;
  if ((s = check_qbufs(p, out)) != SAGE_OK) return s;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return SAGE_ERR_ALIGNMENT;
  const size_t need = part == 0 ? prologue_ws(p) : 0;
  if (need > 0 && (!workspace || workspace_bytes < need)) return SAGE_ERR_WORKSPACE;
  if (workspace && !aligned16(workspace)) return SAGE_ERR_ALIGNMENT;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool bf = p->dtype == SAGE_BF16;
  if (p->d == 128)
    return bf ? run_prologue<__nv_bfloat16, 128>(p, q, k, v, out, workspace, st, part)
              : run_prologue<__half, 128>(p, q, k, v, out, workspace, st, part);
  return bf ? run_prologue<__nv_bfloat16, 64>(p, q, k, v, out, workspace, st, part)
            : run_prologue<__half, 64>(p, q, k, v, out, workspace, st, part);
}

int sage_attn_fwd_partial(const sage_params* p, const sage_qbufs* qb, float* o_part,
                          float* lse_part, void* stream) {
  int s = check_params(p);
  if (s != SAGE_OK) return s;
  if (p->qsmooth) return SAGE_ERR_UNSUPPORTED;
  if ((s = check_qbufs(p, qb)) != SAGE_OK) return s;
  if (!o_part || !lse_part) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(o_part) || !aligned16(lse_part)) return SAGE_ERR_ALIGNMENT;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool bf = p->dtype == SAGE_BF16;
  if (p->d == 128)
    return bf ? run_fwd<__nv_bfloat16, 128>(p, qb, nullptr, lse_part, st, o_part)
              : run_fwd<__half, 128>(p, qb, nullptr, lse_part, st, o_part);
  return bf ? run_fwd<__nv_bfloat16, 64>(p, qb, nullptr, lse_part, st, o_part)
            : run_fwd<__half, 64>(p, qb, nullptr, lse_part, st, o_part);
}

int sage_attn_merge(const sage_params* p, float* o_acc, float* lse_acc, const float* o_part,
                    const float* lse_part, void* out, void* stream) {
  int s = check_params(p);
  if (s != SAGE_OK) return s;
  if (!o_acc || !lse_acc || (o_part == nullptr) != (lse_part == nullptr))
    return SAGE_ERR_INVALID_ARG;
  const void* ptrs[] = {o_acc, lse_acc, o_part, lse_part, out};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return SAGE_ERR_ALIGNMENT;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool bf = p->dtype == SAGE_BF16;
  if (p->d == 128)
    return bf ? run_merge<__nv_bfloat16, 128>(p, o_acc, lse_acc, o_part, lse_part, out, st)
              : run_merge<__half, 128>(p, o_acc, lse_acc, o_part, lse_part, out, st);
  return bf ? run_merge<__nv_bfloat16, 64>(p, o_acc, lse_acc, o_part, lse_part, out, st)
            : run_merge<__half, 64>(p, o_acc, lse_acc, o_part, lse_part, out, st);
}

int sage_attn_bwd_partial(const sage_params* p, const void* v, const sage_qbufs* qb,
                          const float* lse, const void* dout, float* dk_acc, float* dv_acc,
                          int accumulate, void* workspace, size_t workspace_bytes, void* stream) {
  int s = check_params(p);
  if (s != SAGE_OK) return s;
  if (accumulate != 0 && accumulate != 1) return SAGE_ERR_INVALID_ARG;
  if (p->qsmooth) return SAGE_ERR_UNSUPPORTED;
  if ((s = check_qbufs(p, qb)) != SAGE_OK) return s;
  if (!v || !lse || !dout || !dk_acc || !dv_acc) return SAGE_ERR_INVALID_ARG;
  const void* ptrs[] = {v, lse, dout, dk_acc, dv_acc, workspace};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return SAGE_ERR_ALIGNMENT;
  if (!workspace || workspace_bytes < bwd_ws(p).total) return SAGE_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool bf = p->dtype == SAGE_BF16;
  if (p->d == 128)
    return bf ? run_bwd<__nv_bfloat16, 128>(1, p, nullptr, nullptr, v, qb, nullptr, lse, dout,
                                             nullptr, nullptr, nullptr, workspace, st, dk_acc,
                                             dv_acc, accumulate)
              : run_bwd<__half, 128>(1, p, nullptr, nullptr, v, qb, nullptr, lse, dout, nullptr,
                                     nullptr, nullptr, workspace, st, dk_acc, dv_acc, accumulate);
  return bf ? run_bwd<__nv_bfloat16, 64>(1, p, nullptr, nullptr, v, qb, nullptr, lse, dout,
                                          nullptr, nullptr, nullptr, workspace, st, dk_acc, dv_acc,
                                          accumulate)
            : run_bwd<__half, 64>(1, p, nullptr, nullptr, v, qb, nullptr, lse, dout, nullptr,
                                  nullptr, nullptr, workspace, st, dk_acc, dv_acc, accumulate);
}

int sage_kv_finalize(const sage_params* p, const void* k, const sage_qbufs* qb,
                     const float* dk_acc, const float* dv_acc, void* dk, void* dv, void* stream) {
  int s = check_params(p);
  if (s != SAGE_OK) return s;
  if (!dk_acc || !dv_acc || !dk || !dv) return SAGE_ERR_INVALID_ARG;
  if (p->qknorm && (!k || !qb || !qb->k_inv_rms)) return SAGE_ERR_INVALID_ARG;
  const void* ptrs[] = {k, dk_acc, dv_acc, dk, dv};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return SAGE_ERR_ALIGNMENT;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool bf = p->dtype == SAGE_BF16;
  if (p->d == 128)
    return bf ? run_kv_finalize<__nv_bfloat16, 128>(p, k, qb, dk_acc, dv_acc, dk, dv, st)
              : run_kv_finalize<__half, 128>(p, k, qb, dk_acc, dv_acc, dk, dv, st);
  return bf ? run_kv_finalize<__nv_bfloat16, 64>(p, k, qb, dk_acc, dv_acc, dk, dv, st)
            : run_kv_finalize<__half, 64>(p, k, qb, dk_acc, dv_acc, dk, dv, st);
}

}  // extern "C"
