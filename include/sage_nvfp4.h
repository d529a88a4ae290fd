/*
 * sage_nvfp4.h -- C ABI of the NVFP4 Q-Attn variant of libsage (B200, sm_100a).
 *
 * The operation ("Full-Stack FP4", gist.science 2607.04422, section 2.4 "mixed-precision
 * attention (Q-Attn)"): the robust product Q K^T runs in NVFP4, the softmax-sensitive product
 * P V in BF16 (here: in the inputs' 16-bit type); the quantized views of Q and K are produced
 * once by sage_fp4_quant_prologue and reused.  NVFP4 ("Quartet II", allinfo.ai.kr): E2M1
 * values in blocks of 16 along the head dimension, one E4M3 scale per block, plus a global
 * scale, here one per (batch, head) matrix.
 *
 * Quantization (float32, every step correctly rounded, reproducible bit for bit):
 *   x      q or k after the optional QK-norm and K-smoothing of sage.h (same arithmetic);
 *   G      max |x| over the (batch, head) matrix; genc = 2688 / G (1 when G == 0);
 *   block  a = max |x| over 16 channels; u = (a * genc) / 6;
 *          sd = E4M3(u): round to nearest, ties to even, subnormals, 448 and above -> 448;
 *          code = E2M1(x * (genc / sd)): magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}, nearest, ties
 *          to the even code, above 6 -> 6, the sign bit that of the product (a negative value
 *          rounding to zero gives -0, code 8); sd == 0 -> genc / sd taken as 0 (codes +-0).
 *   value  E2M1(code) * sd / genc.
 *
 * Conventions are those of sage.h (device pointers owned by the caller, 16-byte alignment,
 * asynchronous on `stream`, negative sage_status on argument errors, no exceptions).
 * Supported: d in {64, 128}, N a multiple of 128, qsmooth == 0 (else SAGE_ERR_UNSUPPORTED);
 * q_block and k_block are validated as in sage.h but unused (NVFP4 blocks are 16 channels).
 */
#ifndef SAGE_NVFP4_H_
#define SAGE_NVFP4_H_

#include "sage.h"

#ifdef __cplusplus
extern "C" {
#endif

/* NVFP4 views of Q and K.  Sizes per (batch, head); all owned by the caller. */
typedef struct {
  uint8_t *q_fp4, *k_fp4;       /* [B,H,N,d/2]: E2M1 codes, channel 2i in the low nibble of
                                   byte i, channel 2i+1 in the high nibble                   */
  uint8_t *q_sf, *k_sf;         /* [B,H,N/128,d/64,512]: E4M3 block scales; per 128-row tile
                                   and 64-channel chunk, byte (r%32)*16 + (r/32)*4 + b holds
                                   row r's scale of the chunk's 16-channel block b           */
  float *q_genc, *k_genc;       /* [B,H]: global encode scales genc                         */
  float *q_inv_rms, *k_inv_rms; /* [B,H,N]: 1/rms per token (qknorm; may be NULL otherwise) */
  float *k_mean;                /* [B,H,d]: K channel means (ksmooth; else unused)          */
  /* Optional sequence views (NULL: not produced): the same values quantized along the tokens,
   * the K-major operands of dK = dS^T Q and dQ = dS K.  Global scales as above.               */
  uint8_t *q_fp4_t, *k_fp4_t;   /* [B,H,d,N/2]: channel rows, token 2i in the low nibble     */
  uint8_t *q_sf_t, *k_sf_t;     /* [B,H,ceil(d/128),N/64,512]: per 128-channel group and
                                   64-token chunk, byte (c%32)*16 + ((c%128)/32)*4 + b holds
                                   channel c's scale of the chunk's 16-token block b (rows
                                   c >= d of a group are left unwritten)                     */
} sage_fp4_bufs;

/* Workspace bytes: which = 0 prologue (K-mean partials when ksmooth, plus 2*B*H words for the
 * global maxima), 1 forward (0), 2 backward (D = rowsum(dO o O) [B,H,N] float32, then the
 * float32 dQ accumulator [B,H,N,d]).  Returns 0 for invalid parameters. */
size_t sage_fp4_workspace_bytes(const sage_params* p, int which);

/* QK-norm -> K-smoothing -> NVFP4 views of q and k (an absolute-maximum pass, then the
 * quantization pass).  q, k: [B,H,N,d] in p->dtype. */
int sage_fp4_quant_prologue(const sage_params* p, const void* q, const void* k,
                            const sage_fp4_bufs* out, void* workspace, size_t workspace_bytes,
                            void* stream);

/* Forward: S = tau * (Q K^T) from the NVFP4 views (tensor-core block-scaled MMA, FP32
 * accumulation), causal mask, online softmax, O = P V with P rounded to the 16-bit type of v
 * and FP32 accumulation.  v: [B,H,N,d] in p->dtype; o: [B,H,N,d] in p->dtype;
 * lse: [B,H,N] float32, natural log of sum_j exp(z_ij). */
int sage_fp4_attn_fwd(const sage_params* p, const sage_fp4_bufs* fb, const void* v, void* o,
                      float* lse, void* stream);

/* Backward ("Full-Stack FP4" section 2.4: dS in NVFP4; P^T dO and dO V^T in 16 bits):
 *   S = Q K^T from the forward's NVFP4 views (block-scaled MMA), P = exp(tau S - lse) (causal
 *   mask); dP = dO V^T (16-bit operands, FP32 accumulation); D = rowsum(dO o O);
 *   dS = P o (dP - D) in float32;
 *   dV = P^T dO with P rounded to the 16-bit type of v;
 *   per 128 x 128 (query, key) tile, dS is quantized twice with the tile's own global scale
 *   genc = 2688 / max|dS_tile| and the steps listed above: in 16-key blocks (dS_k) and in
 *   16-query blocks (dS_q);
 *   dQ = tau dS_k K_seq and dK = tau dS_q^T Q_seq (block-scaled MMA), K_seq / Q_seq the
 *   sequence views of fb (16-token blocks), which must be present;
 *   with qknorm, the RMSNorm backward dx = inv (dxhat - xhat (dxhat . xhat) / d) of each row.
 * q, k, v, o, dout: [B,H,N,d] in p->dtype (the raw inputs, the forward's output and the
 * output gradient); lse: the forward's [B,H,N]; dq, dk, dv: [B,H,N,d] in p->dtype.
 * Workspace: sage_fp4_workspace_bytes(p, 2) bytes, 16-byte aligned.
 * Errors: SAGE_ERR_INVALID_ARG (a null pointer, missing sequence views, or missing inverse RMS
 * with qknorm), SAGE_ERR_ALIGNMENT, SAGE_ERR_WORKSPACE, SAGE_ERR_UNSUPPORTED (qsmooth, or a
 * launch the register split cannot take), SAGE_ERR_CUDA (launch failure); a bounded wait that
 * gives up is reported by sage_last_device_status. */
int sage_fp4_attn_bwd(const sage_params* p, const void* q, const void* k, const void* v,
                      const sage_fp4_bufs* fb, const void* o, const float* lse, const void* dout,
                      void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
                      void* stream);

/* The three stages sage_fp4_attn_bwd runs, for callers that schedule or time them separately;
 * same arguments and checks as sage_fp4_attn_bwd, and they must run in order on the same
 * workspace:
 *   stage 0  D = rowsum(dO o O) into the workspace, the float32 dQ accumulator cleared;
 *   stage 1  the tensor-core kernel: dk and dv written, dQ accumulated in the workspace;
 *   stage 2  dq from the accumulator (with the RMSNorm backward when qknorm).
 * Returns SAGE_ERR_INVALID_ARG for any other stage. */
int sage_fp4_attn_bwd_stage(int stage, const sage_params* p, const void* q, const void* k,
                            const void* v, const sage_fp4_bufs* fb, const void* o,
                            const float* lse, const void* dout, void* dq, void* dk, void* dv,
                            void* workspace, size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SAGE_NVFP4_H_ */
