/*
 * sage.h -- C ABI of libsage: SageBwd quantized attention training on NVIDIA B200 (sm_100a).
 *
 * The operation ("SageBwd: trainable low-bit attention", aitrends.kr):
 *   - QK-norm paragraph: every token vector of Q and K is RMS-normalized over the head dim;
 *   - K-smoothing paragraph: a mean over tokens is subtracted from each channel of K right
 *     before quantization;
 *   - Triton-kernel paragraph: Q, K, V (and P, dS, dO) are quantized to INT8 per block;
 *   - quantization-strategy paragraph: six of the seven attention matmuls run in INT8
 *     (S = Q K^T forward and recomputed, O = P V, dV = P^T dO, dQ = dS K, dK = dS^T Q); only
 *     dP = dO V^T runs in 16-bit float, being the most error-sensitive;
 *   - error-propagation paragraph: dQ = dS K and dK = dS^T Q carry the quantization error of dS.
 *
 * Conventions shared by every entry point
 *   Layout     All tensors are contiguous [B, H, N, d] with d innermost; per-block scales are
 *              [B, H, N / block]; per-token vectors [B, H, N]; K means [B, H, d].
 *   Pointers   Every pointer is a DEVICE pointer, allocated and owned by the caller, except
 *              the tensors of sage_fwd_bwd_host (host memory); the library never allocates,
 *              frees or retains memory.  Tensor pointers must be
 *              16-byte aligned.  Work is asynchronous on `stream` (a cudaStream_t; NULL = the
 *              legacy default stream); buffers must stay valid until the stream reaches it.
 *   Shapes     d in {64, 128}; k_block == 64; q_block in {64, 128}; N a multiple of 128.
 *   Errors     Argument errors return a negative sage_status synchronously and launch nothing.
 *              A failed launch returns SAGE_ERR_CUDA.  Kernels never trap: a device-side wait
 *              that exceeds its time limit records SAGE_ERR_TIMEOUT in a status word that
 *              sage_last_device_status() reads.  No C++ exception crosses this boundary.
 *   Threads    Calls are thread-safe as far as the CUDA runtime is; calls that share output
 *              or workspace buffers must be ordered by the caller.
 */
#ifndef SAGE_H_
#define SAGE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SAGE_OK = 0,
  SAGE_ERR_INVALID_ARG = -1, /* null pointer, non-positive size, inconsistent parameters   */
  SAGE_ERR_UNSUPPORTED = -2, /* valid but unimplemented shape (d, block sizes, N)          */
  SAGE_ERR_ALIGNMENT = -3,   /* a tensor pointer is not 16-byte aligned                    */
  SAGE_ERR_WORKSPACE = -4,   /* workspace missing or smaller than sage_workspace_bytes()   */
  SAGE_ERR_CUDA = -5,        /* a CUDA runtime / driver call failed                        */
  SAGE_ERR_TIMEOUT = -6      /* a kernel gave up waiting on a barrier (device status only) */
} sage_status;

typedef enum { SAGE_FP16 = 0, SAGE_BF16 = 1 } sage_dtype;

/* Problem description.  softmax_scale <= 0 selects 1/sqrt(d); rms_eps is the RMSNorm epsilon
 * (the page gives none; 1e-6 is the library's default in its bindings). */
typedef struct {
  int B, H, N, d;
  int dtype;   /* sage_dtype of q, k, v, o, dout, dq, dk, dv                          */
  int causal;  /* 1: key j visible to query i iff j <= i (square, top-left aligned)   */
  int qknorm;  /* 1: per-token RMSNorm of q and k before quantization                 */
  int ksmooth; /* 1: subtract the per-channel mean over tokens from k before quant.   */
  int q_block; /* tokens per Q (and dO) quantization block: 64 or 128                 */
  int k_block; /* tokens per K and V quantization block: 64                           */
  float softmax_scale;
  float rms_eps;
  int qsmooth; /* 1: Q-smoothing as well (Q-smoothing paragraph): subtract the per-channel
                  token mean mu_Q from qhat before quantization, add the per-key bias
                  k_bias_j = mu_Q . ktilde_j to the scores and the correction
                  softmax_scale * (dS^T 1) mu_Q^T to dK.  0: off.                           */
} sage_params;

/* Quantized views of Q, K, V produced once by the prologue and read by both the forward and
 * the backward pass.  Codes are int8 in [-127, 127]; scale = absmax / 127 of the block. */
typedef struct {
  int8_t *q_codes, *k_codes, *v_codes; /* [B,H,N,d]                                        */
  float *q_scale;                      /* [B,H,N/q_block]                                  */
  float *k_scale, *v_scale;            /* [B,H,N/k_block]                                  */
  float *q_inv_rms, *k_inv_rms;        /* [B,H,N]; written when qknorm (else unused, may be
                                          NULL)                                            */
  float *k_mean;                       /* [B,H,d]; written when ksmooth (else may be NULL) */
  float *q_mean;                       /* [B,H,d]; written when qsmooth (else may be NULL) */
  float *k_bias;                       /* [B,H,N]; written when qsmooth (else may be NULL) */
} sage_qbufs;

/* Bytes of scratch each call needs: which = 0 prologue, 1 forward, 2 backward.  Returns 0 for
 * invalid parameters.  The scratch is caller-owned device memory, 256-byte aligned. */
size_t sage_workspace_bytes(const sage_params* p, int which);

/* Prologue (QK-norm, K-smoothing and quantization paragraphs).  In float32:
 *   qknorm:  inv = 1/sqrt(sum(x^2)/d + eps), xhat = x * inv for every token of q and k;
 *   ksmooth: m_c = (sum over all N tokens of khat_c) / N, ktilde = khat - m;
 *   qsmooth: mu_Q the same mean of qhat, qtilde = qhat - mu_Q is what gets quantized, and
 *            k_bias_j = sum_c mu_Q,c * ktilde_jc (8-channel lane partials, products and sums
 *            rounded, combined by a butterfly over the lanes, as in the RMSNorm sum);
 *   quantize: per block of q_block (q) or k_block (k, v) tokens spanning all d channels,
 *            s = absmax/127, code = round-half-even(x / s); s = 0 and codes 0 if absmax = 0.
 * The float32 operation order is fixed, so codes, scales, inv_rms, k_mean, q_mean and k_bias
 * are reproducible bit for bit.  q, k, v: 16-bit inputs [B,H,N,d].  out: all buffers written. */
int sage_quant_prologue(const sage_params* p, const void* q, const void* k, const void* v,
                        const sage_qbufs* out, void* workspace, size_t workspace_bytes,
                        void* stream);

/* sage_quant_prologue for callers that cannot allocate device memory.  (The SageBwd page has
 * no counterpart: this is a deployment variant of the prologue, not part of the method.)
 * Some callers cannot call cudaMalloc: code embedded in a host runtime that owns every device
 * allocation through its own memory pool, code running under a fixed device-memory budget set
 * at start-up, and latency-critical host threads that must not risk the device-wide
 * synchronization cudaMalloc / cudaFree can cause.  This entry point takes no workspace: the
 * smoothing column sums go to a fixed 32 MiB array in the library's own device memory (every
 * context that loads the library's device code holds it until the context is destroyed), so
 * it supports shapes with (ksmooth + qsmooth) * B * H * (N / 64) * d * 4 <= 32 MiB (e.g.
 * B*H*N*d up to 2^29 elements with one of the two) and returns SAGE_ERR_WORKSPACE beyond
 * that, before launching anything.  Everything else -- arguments, outputs, results (bit for
 * bit) -- is as for sage_quant_prologue.  It allocates nothing.
 * Every call looks up the array's device address in the calling thread's current context (a
 * host-side lookup that allocates nothing), so calls from any context -- the device's primary
 * one or a driver context of the caller's own -- use that context's copy of the array.  The
 * library's device code, and the 32 MiB array with it, is loaded into a context by the first
 * call of any libsage entry point there (lazy module loading), and that load allocates device
 * memory and may synchronize the device: callers that cannot afford either later should make
 * one warm-up call per context at start-up, before any stream capture.  All calls in one
 * context share its array, which keeps the last call's contents; every value a call reads from
 * it is written by that same call first, so nothing needs clearing, but calls whose kernels
 * overlap on the GPU (on different streams) race on it and must be ordered by the caller. */
int sage_quant_prologue_noalloc(const sage_params* p, const void* q, const void* k,
                                const void* v, const sage_qbufs* out, void* stream);

/* Forward attention with INT8 S = Qc Kc^T and O = Pc Vc (quantization-strategy paragraph).
 * z = (A * sQ * sK + k_bias_j) * softmax_scale (k_bias_j = 0 without qsmooth); P is quantized
 * with one scale per (query row, K block);
 * o: [B,H,N,d] in dtype; lse: [B,H,N] float32, natural log-sum-exp of the scaled scores. */
int sage_attn_fwd(const sage_params* p, const sage_qbufs* qb, void* o, float* lse,
                  void* workspace, size_t workspace_bytes, void* stream);

/* Backward attention (quantization-strategy and error-propagation paragraphs): recomputes the
 * INT8 scores from the same codes, dP = dO V^T in 16-bit float with float32 accumulation,
 * dS = P (dP - rowsum(dO o O)), P and dS quantized per q_block x k_block tile, dO per q_block
 * tokens; dV = P^T dO, dK = dS^T Q, dQ = dS K in INT8 (with qsmooth, the scores carry the
 * forward's bias and dK gains softmax_scale * (sum_i dS_ij) mu_Q, the column sums taken over the
 * quantized dS tiles).  q, k, v are the raw 16-bit inputs
 * (needed for dP and the RMSNorm backward); o, lse the forward's outputs; dout = dL/do.
 * dq, dk, dv: [B,H,N,d] in dtype, gradients with respect to the raw q, k, v. */
int sage_attn_bwd(const sage_params* p, const void* q, const void* k, const void* v,
                  const sage_qbufs* qb, const void* o, const float* lse, const void* dout,
                  void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
                  void* stream);

/* The three stages sage_attn_bwd runs, for callers that schedule or time them separately;
 * same arguments as sage_attn_bwd, and they must run in order on the same workspace:
 *   stage 0  preprocess: D_i = sum_c dO_ic O_ic, dO quantized per q_block tokens, the float32
 *            dQ accumulator (in the workspace) cleared;
 *   stage 1  the tensor-core kernel: dk and dv written, dQ accumulated in the workspace;
 *   stage 2  dq from the accumulator (with the RMSNorm backward when qknorm).
 * Returns SAGE_ERR_INVALID_ARG for any other stage. */
int sage_attn_bwd_stage(int stage, const sage_params* p, const void* q, const void* k,
                        const void* v, const sage_qbufs* qb, const void* o, const float* lse,
                        const void* dout, void* dq, void* dk, void* dv, void* workspace,
                        size_t workspace_bytes, void* stream);

/* The whole step -- prologue, forward, backward -- on HOST buffers (end to end: the operator as
 * a host program calls it).  q, k, v, dout and the results o, dq, dk, dv are host pointers to
 * [B,H,N,d] 16-bit tensors; pin them (cudaHostAlloc / cudaHostRegister) for the copies to run
 * asynchronously (pageable memory works, with copies that block the host).  Every (batch, head)
 * is independent, so the batch is cut into `chunks` contiguous slices of B*c/chunks ..
 * B*(c+1)/chunks (chunks is capped at B) that flow through two device slots: slice c's
 * host-to-device copies run on stream_in, its kernels on stream_compute and its device-to-host
 * copies on stream_out, so the copies of neighbouring slices overlap slice c's kernels.  One
 * cudaMemcpyAsync per tensor and slice.  `workspace` is caller-owned device memory of at least
 * sage_fwd_bwd_host_workspace_bytes(p, chunks) bytes (16-byte aligned) holding both slots.  The
 * three streams are caller-owned (distinct streams overlap; NULL serializes everything on the
 * legacy default stream); the library creates six CUDA events for the call and destroys them
 * before returning.  The call returns once the results are in host memory (or on the first
 * error, after draining the streams); results equal sage_quant_prologue + sage_attn_fwd +
 * sage_attn_bwd run on the same data on the device.  Read sage_last_device_status() afterwards
 * for device-side timeouts. */
size_t sage_fwd_bwd_host_workspace_bytes(const sage_params* p, int chunks);
int sage_fwd_bwd_host(const sage_params* p, const void* q, const void* k, const void* v,
                      const void* dout, void* o, void* dq, void* dk, void* dv, int chunks,
                      void* workspace, size_t workspace_bytes, void* stream_in,
                      void* stream_compute, void* stream_out);

/* ---- context parallelism: one long sequence split into chunks held by different ranks ----
 * The sequence of N_total tokens is cut into W contiguous chunks of N tokens (p->N is the
 * chunk length; N_total = W * N); rank r holds tokens [r*N, (r+1)*N) of every (batch, head).
 * The blocks of every quantization (Q, K, V per block of tokens; P, dS, dO per tile) never
 * straddle a chunk boundary, so the pieces below give the single-sequence result of
 * sage_quant_prologue / sage_attn_fwd / sage_attn_bwd up to float32 rounding order.  The
 * ranks exchange data between the calls (ring order; fwd_bwd_b200/cp.py).  Q-smoothing
 * (qsmooth) is not supported here (SAGE_ERR_UNSUPPORTED).
 *
 * sage_quant_prologue_part: the prologue in two parts.  part 0: the K-smoothing statistics of
 *   this chunk only: out->k_mean = per-channel mean over the chunk's tokens of the normalized
 *   k (needs the prologue workspace; nothing else is written).  The ranks then average their
 *   means (all equal-sized chunks, so the average is the mean over all N_total tokens, the
 *   K-smoothing paragraph's mean over the sequence).  part 1: QK-norm, smoothing with the
 *   caller's out->k_mean, and the per-block codes and scales of the chunk (no workspace).
 *   Without ksmooth, part 0 does nothing and part 1 equals sage_quant_prologue. */
int sage_quant_prologue_part(const sage_params* p, const void* q, const void* k, const void* v,
                             const sage_qbufs* out, void* workspace, size_t workspace_bytes,
                             int part, void* stream);

/* sage_attn_fwd_partial: attention of this chunk's queries over ONE chunk of keys, whose codes
 *   and scales qb->k_* / qb->v_* point at (the local chunk or one received from another
 *   rank; qb->q_* are the local queries').  p->causal: 1 for the diagonal chunk (the same
 *   token range as the queries), 0 for a chunk of earlier keys; chunks of later keys are not
 *   computed under a causal mask.  o_part: float32 [B,H,N,d], normalized over this chunk's
 *   keys; lse_part: float32 [B,H,N], natural-log sum of exponentials of the scaled scores. */
int sage_attn_fwd_partial(const sage_params* p, const sage_qbufs* qb, float* o_part,
                          float* lse_part, void* stream);

/* sage_attn_merge: softmax over the union of two disjoint key sets from their partial results:
 *   L = ln(e^La + e^Lb), O = e^(La-L) O_a + e^(Lb-L) O_b, written back into (o_acc, lse_acc)
 *   (float32 [B,H,N,d] / [B,H,N]; lse = -inf marks an empty result).  When `out` is not NULL
 *   the merged O is also stored there in dtype ([B,H,N,d]).  With o_part and lse_part both
 *   NULL the accumulator is only converted to `out`. */
int sage_attn_merge(const sage_params* p, float* o_acc, float* lse_acc, const float* o_part,
                    const float* lse_part, void* out, void* stream);

/* sage_attn_bwd_partial: the backward tensor-core kernel for this chunk's queries against one
 *   chunk of keys (qb->k_*: its codes and scales, v: its raw 16-bit values for dP; p->causal
 *   as in sage_attn_fwd_partial).  Needs stage 0 of sage_attn_bwd_stage run first on the same
 *   workspace with this chunk's o, dout and the merged lse; dQ accumulates in the workspace
 *   across calls (stage 2 then finishes dq).  The keys' raw gradients (before the RMSNorm
 *   backward) go to dk_acc / dv_acc (float32 [B,H,N,d]): stored when accumulate = 0 (the first
 *   chunk of queries to see these keys), added when accumulate = 1.  They travel back to the
 *   keys' owner, which finishes them with sage_kv_finalize. */
int sage_attn_bwd_partial(const sage_params* p, const void* v, const sage_qbufs* qb,
                          const float* lse, const void* dout, float* dk_acc, float* dv_acc,
                          int accumulate, void* workspace, size_t workspace_bytes, void* stream);

/* sage_kv_finalize: dk = RMSNorm backward of dk_acc (with qknorm; k the raw keys and
 *   qb->k_inv_rms their inverse RMS from the prologue; otherwise dk = dk_acc), dv = dv_acc,
 *   both stored in dtype ([B,H,N,d]). */
int sage_kv_finalize(const sage_params* p, const void* k, const sage_qbufs* qb,
                     const float* dk_acc, const float* dv_acc, void* dk, void* dv, void* stream);

/* Synchronizes `stream`, returns the device status word of the current device (SAGE_OK or
 * SAGE_ERR_TIMEOUT) and clears it.  Returns SAGE_ERR_CUDA if the synchronization fails. */
int sage_last_device_status(void* stream);

/* Human-readable name of a sage_status value (static storage). */
const char* sage_status_string(int status);

/* ---- test support: run single pieces of the kernels' tensor-core path ---------------------
 * sage_debug_qk_int32: the forward kernel's INT8 score product for one head `bh` and one tile
 *   of 128 queries `q_tile`, against all N keys: s_out[128][N] int32 = Qc Kc^T, computed by
 *   the same shared-memory staging and tcgen05 MMA code as the forward kernel.
 * sage_debug_umma_gemm: C[M][N] = A B with M = 128, N and K in {64, 128}.
 *   kind 0: int8 x int8 -> int32; kind 1: fp16 -> fp32; kind 2: bf16 -> fp32 (K-major only).
 *   a_mn_major = 0: A stored [M][K]; 1: A stored [K][M].  b_mn_major = 0: B stored [N][K];
 *   1: B stored [K][N].  All pointers are device pointers; C is row-major [M][N]. */
int sage_debug_qk_int32(const sage_params* p, const sage_qbufs* qb, int bh, int q_tile,
                        int32_t* s_out, void* stream);
int sage_debug_umma_gemm(int kind, int a_mn_major, int b_mn_major, int N, int K, const void* A,
                         const void* B, void* C, void* stream);

/* sage_debug_wait_timeout: drives the kernels' failure path on purpose, without a fault.  One
 * CTA allocates tensor memory and waits on a shared-memory barrier that nothing ever arrives
 * on, for at most limit_us microseconds (1 .. 1e6); the wait then records SAGE_ERR_TIMEOUT in
 * the device status word, the CTA frees its tensor memory and returns, exactly as a pipeline
 * kernel does when one of its bounded waits runs out.  Until the status word is read and
 * cleared by sage_last_device_status(), the attention kernels launched afterwards on the same
 * device see the recorded failure and return at once without writing their outputs.  Returns
 * SAGE_ERR_INVALID_ARG for limit_us out of range, before launching. */
int sage_debug_wait_timeout(int limit_us, void* stream);

/* ---- measurement support: the tensor cores' own peak ---------------------------------------
 * sage_mma_peak launches n_ctas CTAs (one per SM: pass the SM count), each of which stages
 * the first 48 KB of `fill` (a device buffer of at least 49152 bytes, 16-byte aligned; give it
 * random int8 codes for kind 0 and random fp16 / bf16 values for kinds 1 / 2 so the operands
 * toggle like real data) in shared memory and issues `groups` x 4 back-to-back tcgen05 MMAs of
 * M = 128, N = 256 from it: kind 0 = kind::i8 (K = 32 per MMA, INT32 accumulation), 1 = fp16
 * and 2 = bf16 (kind::f16, K = 16, float32 accumulation).  Each CTA performs
 * groups * 4 * 2 * 128 * 256 * K operations; the caller times the launch on `stream` with CUDA
 * events.  This is the denominator of the attention kernels' rooflines (the quantization-
 * strategy paragraph's six INT8 and one 16-bit matmul run at these two rates); it computes
 * nothing the attention uses.  groups in [1, 2^26]; keep one launch well under a second (the
 * issuing thread's completion wait gives up after two seconds and records SAGE_ERR_TIMEOUT).
 * Returns SAGE_ERR_INVALID_ARG / SAGE_ERR_ALIGNMENT for bad arguments before launching. */
int sage_mma_peak(int kind, int n_ctas, int groups, const void* fill, size_t fill_bytes,
                  void* stream);

#ifdef __cplusplus
}
#endif
#endif /* SAGE_H_ */
