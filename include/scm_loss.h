/*
 * scm_loss.h -- C ABI of the tangent-normalised sCM loss term (B200, sm_100a).
 *
 * The operation.  rCM's sCM term uses tangent normalisation (papernotes.org
 * notes on "Large Scale Diffusion Distillation via Score-Regularized
 * Continuous-Time Consistency", 损失函数 / 训练策略; ai.info AI summary,
 * Methodology in Plain English: c = 0.1).  For every sample b, over its N
 * elements i:
 *
 *     n_b     = sum_i g_bi^2
 *     r_bi    = F_bi - F-_bi - g_bi / (n_b + c)
 *     loss_b  = sum_i r_bi^2
 *     grad_bi = 2 r_bi                    (d loss_b / d F_bi)
 *
 * F is the student's output, F- the EMA target's (no gradient), g the
 * tangent direction.  The mean over samples is the caller's.
 *
 * Layout.  f, f_ema, g and grad are dense row-major bf16 [B, N]; loss is fp32
 * [B].  Sums are fp32 in a fixed order (deterministic); grad is rounded to
 * bf16 (nearest even).
 *
 * Ownership and errors as in attn_jvp.h: caller-owned buffers, no device
 * allocation, asynchronous on `stream`, host-side checks return an
 * attn_jvp_status before anything is queued.
 */
#ifndef SCM_LOSS_H
#define SCM_LOSS_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/*
 * scm_tangent_loss -- queue loss (and grad) for all B samples on `stream`.
 *
 *   f, f_ema, g   bf16 device pointers [B, N], 16-byte aligned
 *   loss          fp32 device pointer [B], written
 *   grad          bf16 device pointer [B, N], written, or NULL (not computed)
 *   B             1 .. 65535 samples;  N  1 .. 2^40 elements per sample
 *   c             finite, >= 0 (the pages use 0.1); n_b + c = 0 gives inf/NaN
 *   stream        a cudaStream_t, or NULL for the legacy default stream
 *
 * Returns ATTN_JVP_OK once queued, ATTN_JVP_ERR_NULL (f, f_ema, g or loss
 * NULL), ATTN_JVP_ERR_SHAPE, ATTN_JVP_ERR_ALIGN, ATTN_JVP_ERR_VALUE (c not
 * finite or negative, or an output overlapping an input or the other
 * output) or ATTN_JVP_ERR_LAUNCH.  When N is a multiple of 8 the kernel
 * moves 16-byte vectors; otherwise it reads element by element (slower).
 */
int scm_tangent_loss(const void *f, const void *f_ema, const void *g, float *loss, void *grad,
                     int B, long long N, float c, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* SCM_LOSS_H */
