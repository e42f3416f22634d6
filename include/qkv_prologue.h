/*
 * qkv_prologue.h -- C ABI of the QKV projection + RMSNorm layer with its
 * tangent (B200, sm_100a): the forward-and-tangent function of the layer in
 * front of attention.
 *
 * The operation.  rCM refactors each network layer to expose forward and
 * tangent functions so that JVPs survive FSDP ("Large Scale Diffusion
 * Distillation via Score-Regularized Continuous-Time Consistency", ai.info AI
 * summary, Key Contributions 1).  For tokens x (row t = b L + l) and their
 * tangent x', with fixed weights W = [W_q; W_k; W_v] of shape [3 H d, D]:
 *
 *     y = x W^T,  y' = x' W^T
 *     r = (mean over each head's d channels of y^2 + eps)^(-1/2)
 *     q = gamma_q * y_q * r,   q' = gamma_q * (y_q' r - y_q r^3 mean(y_q y_q'))
 *     k, k' alike with gamma_k;   v = y_v,   v' = y_v'
 *
 * RMSNorm runs per head over d channels (QK-norm) with one gain vector of
 * length d for q and one for k; V is not normalised.
 *
 * Layout.  x, x_dot: bf16 [B*L, D] row-major; w_qkv: bf16 [3*H*d, D]
 * row-major (q heads, then k heads, then v heads, d rows each); gamma_q,
 * gamma_k: fp32 [d]; q, k, v, q_dot, k_dot, v_dot: bf16 [B, H, L, d], the
 * layout attn_jvp_fwd reads.  Accumulation is fp32; outputs are rounded to
 * bf16 (nearest even).
 *
 * Ownership and errors as in attn_jvp.h.  A device-side wait that gives up
 * is reported by qkv_prologue_check.
 */
#ifndef QKV_PROLOGUE_H
#define QKV_PROLOGUE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/*
 * qkv_rmsnorm_jvp -- queue the six outputs for all B*L tokens on `stream`.
 *
 *   B, L, H  >= 1, B*L and 3*H*d below 2^31
 *   D        model width, a positive multiple of 64
 *   d        head dimension, 64 or 128
 *   eps      finite, >= 0
 *
 * Returns ATTN_JVP_OK once queued, or ATTN_JVP_ERR_NULL, _SHAPE, _HEADDIM,
 * _ALIGN (bf16 pointers need 16 bytes, gains 4), _VALUE (eps, or an output
 * overlapping an input or another output) or _LAUNCH.
 */
int qkv_rmsnorm_jvp(const void *x, const void *x_dot, const void *w_qkv, const float *gamma_q,
                    const float *gamma_k, void *q, void *k, void *v, void *q_dot, void *k_dot,
                    void *v_dot, int B, int L, int H, int D, int d, float eps, void *stream);

/* As attn_jvp_check, for the prologue kernel's own status word. */
int qkv_prologue_check(void *stream, int *site);

#ifdef __cplusplus
}
#endif

#endif /* QKV_PROLOGUE_H */
