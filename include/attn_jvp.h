/*
 * attn_jvp.h -- C ABI of the B200 (sm_100a) attention forward + JVP library.
 *
 * The operation.  The FlashAttention-2 JVP kernel of rCM ("Large Scale
 * Diffusion Distillation via Score-Regularized Continuous-Time Consistency",
 * ai.info AI summary, Key Contributions 1 and Methodology in Plain English;
 * papernotes.org notes, 关键设计 1) folds the Jacobian-vector product into the
 * attention forward pass, for self- and cross-attention, and carries the
 * tangents through the same block-wise tiling.  For every batch b, head h and
 * query row i, over the valid keys j < n_b:
 *
 *     S_ij  = scale * q_i . k_j                 P = softmax_j(S)
 *     O_i   = sum_j P_ij v_j                    lse_i = ln sum_j exp(S_ij)
 *     S'_ij = scale * (q'_i . k_j + q_i . k'_j)
 *     O'_i  = sum_j P_ij (S'_ij - mu_i) v_j + sum_j P_ij v'_j,
 *             mu_i = sum_j P_ij S'_ij
 *
 * i.e. O' = P'V + PV' with P' = P (S' - mu), the exact directional
 * derivative of O along (Q', K', V').  The scale has no tangent.
 *
 * Layout.  Every tensor is dense, contiguous and row-major in device memory:
 *     q, q_dot, o, o_dot : bf16 [B, H, Lq, d]
 *     k, k_dot, v, v_dot : bf16 [B, H, Lk, d]
 *     lse                : fp32 [B, H, Lq]
 *     kv_len             : int32 [B] or NULL
 * K and V have the same head count as Q.  bf16 is the IEEE-754 binary32 upper
 * half; outputs are rounded to nearest even from fp32 accumulators.
 *
 * Masking.  n_b = min(Lk, kv_len[b]) clamped below at 0; with kv_len == NULL,
 * n_b = Lk.  Keys j >= n_b take no part in any output: their k, k', v, v'
 * may hold any bits (NaN included).  A row with n_b == 0 gets O = O' = 0 and
 * lse = -inf.  kv_len is read on the device, so its values are not checked
 * on the host.  There is no causal mask.
 *
 * Ownership.  The caller owns every buffer.  The library allocates no device
 * memory, keeps no per-call state, and returns as soon as the work is queued
 * on `stream` (asynchronous).  Outputs must not overlap inputs or each other.
 *
 * Errors.  Argument errors are detected on the host before anything is
 * queued; outputs are then left untouched.  Failures that only the device
 * can see (a pipeline wait that gave up) are recorded in a per-device status
 * word and reported by attn_jvp_check().
 */
#ifndef ATTN_JVP_H
#define ATTN_JVP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ATTN_JVP_OK = 0,
    ATTN_JVP_ERR_NULL = -1,    /* a required pointer is NULL                         */
    ATTN_JVP_ERR_SHAPE = -2,   /* B, H, Lq or Lk < 1, or a size past the limits below  */
    ATTN_JVP_ERR_HEADDIM = -3, /* d is not 64 or 128                                  */
    ATTN_JVP_ERR_ALIGN = -4,   /* a tensor pointer is not 16-byte aligned             */
    ATTN_JVP_ERR_LAUNCH = -5,  /* the CUDA runtime refused the launch or a query      */
    ATTN_JVP_ERR_TIMEOUT = -6, /* a device-side wait gave up (see attn_jvp_check)    */
    ATTN_JVP_ERR_VALUE = -7,   /* scale not finite, or outputs overlap inputs         */
    ATTN_JVP_ERR_SCRATCH = -8  /* attn_jvp_fwd_noalloc: the split needs more than the */
                               /* library's static scratch holds                      */
} attn_jvp_status;

/*
 * attn_jvp_fwd -- queue O, O' and lse for the whole [B, H] batch on `stream`.
 *
 *   q, k, v              bf16 device pointers (layout above)
 *   q_dot, k_dot, v_dot  bf16 device pointers, the tangents Q', K', V'
 *   o, o_dot             bf16 device pointers, written.  When both are 32-byte
 *                        aligned (as cudaMalloc and PyTorch allocations are), the
 *                        epilogue stores 32 bytes at a time; 16-byte aligned
 *                        outputs take a slower store path with the same results
 *   lse                  fp32 device pointer, written (natural log)
 *   B, H, Lq, Lk         >= 1; B*H*Lq and B*H*Lk below 2^31; Lq, Lk below 2^31
 *   d                    64 or 128
 *   scale                finite; the usual choice is 1/sqrt(d)
 *   kv_len               device int32[B] or NULL
 *   stream               a cudaStream_t, or NULL for the legacy default stream
 *
 * Returns ATTN_JVP_OK once the kernel is queued, or a negative status.
 * Thread-safe; the first call on a device also sets that device's kernel
 * attributes.
 */
int attn_jvp_fwd(const void *q, const void *k, const void *v,
                 const void *q_dot, const void *k_dot, const void *v_dot,
                 void *o, void *o_dot, float *lse,
                 int B, int H, int Lq, int Lk, int d, float scale,
                 const int32_t *kv_len, void *stream);

/*
 * attn_jvp_fwd_ex -- attn_jvp_fwd with two additions.
 *
 *   lse_dot       fp32 device pointer [B, H, Lq], written, or NULL.  It
 *                 receives the tangent of lse along (Q', K'):
 *                 lse'_i = sum_j P_ij S'_ij (the row mean mu of the JVP
 *                 above; d lse_i = sum_j P_ij dS_ij).  Rows with n_b = 0
 *                 get 0.  It is formed as c + a / l from the kernel's running
 *                 sums, so its error is of the order of the bf16 rounding of
 *                 P (s S' - c) relative to the spread of s S' over the row.
 *   k_dot, v_dot  may both be NULL, meaning K' = V' = 0 (keys and values that
 *                 do not move, such as text tokens in cross-attention).
 *                 Then S' = s Q' K^T and O' = P' V; the kernel neither loads
 *                 nor multiplies K' and V', which removes 4 of the 12 FLOP
 *                 units.  Exactly one of them NULL is ATTN_JVP_ERR_NULL.
 *
 * Everything else (layout, masking, ownership, errors) is as for
 * attn_jvp_fwd; lse_dot must not overlap any other tensor.  The row mean
 * and the zero-tangent case are the "next" items the rCM pages' kernel
 * needs for cross-attention with frozen text keys (ai.info AI summary, Key
 * Contributions 1: self- and cross-attention).
 */
int attn_jvp_fwd_ex(const void *q, const void *k, const void *v,
                    const void *q_dot, const void *k_dot, const void *v_dot,
                    void *o, void *o_dot, float *lse, float *lse_dot,
                    int B, int H, int Lq, int Lk, int d, float scale,
                    const int32_t *kv_len, void *stream);

/*
 * attn_jvp_fwd_ws -- attn_jvp_fwd_ex with the last wave of query tiles split
 * over the key range.  The kernel keeps one persistent CTA per SM; with T
 * query tiles ([ceil(Lq / 128)] * B * H) on n SMs, the last T mod n tiles
 * would leave most SMs idle for a whole tile's time.  Each of them is cut
 * instead into S = min(n / (T mod n), ceil(Lk / 64), 8) key ranges, one per
 * CTA.  Every range keeps the unnormalised online-softmax state of its keys
 * (running max m, l = sum p, a = sum p (s S' - c), the centring constant c,
 * O_acc and O'_acc) and writes it to `workspace`; the range that finishes
 * last merges the states of its tile (the same rescaling by 2^(m - max m)
 * that the online softmax applies between key tiles) and writes the
 * outputs.  No CTA waits for another.  The results equal attn_jvp_fwd_ex's
 * up to the order of the fp32 sums.  This is the FlashAttention-2 forward's
 * block-wise online softmax (rCM pages: ai.info AI summary, Key
 * Contributions 1 and Methodology in Plain English; papernotes.org notes,
 * key design 1), with blocks of keys taken by different CTAs; the pages do
 * not describe a split.
 *   workspace        device memory of at least attn_jvp_workspace_bytes(B, H,
 *                    Lq, Lk, d) bytes, 256-byte aligned, not overlapping any
 *                    other argument; caller-owned.  Its first bytes are
 *                    counters that the call zeroes (cudaMemsetAsync on
 *                    `stream`) before the kernel; the rest is overwritten.
 *                    Calls that run at the same time need separate
 *                    workspaces.  NULL is allowed when the size is 0 (no
 *                    split for this shape on this device).
 *   workspace_bytes  its size; less than needed is ATTN_JVP_ERR_VALUE.
 * Everything else is as for attn_jvp_fwd_ex.
 */
int attn_jvp_fwd_ws(const void *q, const void *k, const void *v,
                    const void *q_dot, const void *k_dot, const void *v_dot,
                    void *o, void *o_dot, float *lse, float *lse_dot,
                    int B, int H, int Lq, int Lk, int d, float scale,
                    const int32_t *kv_len, void *workspace, size_t workspace_bytes,
                    void *stream);

/*
 * attn_jvp_fwd_noalloc -- attn_jvp_fwd_ws for callers that cannot allocate
 * device memory: runtimes that own all device memory and give a kernel
 * library no allocator (only the inputs and outputs), and latency-critical
 * loops that must not call cudaMalloc, which can synchronise the device and
 * stall every stream.  The pages have no counterpart: it exists for such
 * callers.  The caller passes inputs and
 * outputs exactly as for attn_jvp_fwd_ws, but no workspace: the library uses
 * a 20 MiB array of its own in device memory, which every GPU that loads the
 * library holds until the process exits.  The call allocates nothing and
 * frees nothing.
 *   - The first call on a device looks up the array's device address (once
 *     per device, with that device current); make that first call before
 *     any stream capture on the device.
 *   - Every call on a device shares the one array: calls whose kernels can
 *     overlap on the GPU (different streams without an ordering between
 *     them) race on it and give wrong results.  The counters in it are
 *     zeroed on `stream` before each kernel; the rest is overwritten.
 *   - A shape whose split needs more than the array holds returns
 *     ATTN_JVP_ERR_SCRATCH (not reachable on a 148-SM B200, where d = 128
 *     needs at most 19.7 MB).
 * Everything else is as for attn_jvp_fwd_ws.
 */
int attn_jvp_fwd_noalloc(const void *q, const void *k, const void *v,
                         const void *q_dot, const void *k_dot, const void *v_dot,
                         void *o, void *o_dot, float *lse, float *lse_dot,
                         int B, int H, int Lq, int Lk, int d, float scale,
                         const int32_t *kv_len, void *stream);

/*
 * attn_jvp_workspace_bytes -- bytes of workspace attn_jvp_fwd_ws needs for
 * this shape on the current device (it depends on the SM count); 0 when the
 * shape gets no split or the arguments are out of range.  There are at most
 * n ranges (n SMs), so it is at most 256 + n * (4 + 2 d) * 128 * 4 bytes:
 * 19.7 MB at d = 128, 10.0 MB at d = 64 on a 148-SM B200.
 */
size_t attn_jvp_workspace_bytes(int B, int H, int Lq, int Lk, int d);

/*
 * attn_jvp_check -- take the current device's status word: a one-thread
 * kernel queued on `stream` reads and clears it in one atomic exchange, and
 * the call then synchronises `stream`.  Returns ATTN_JVP_OK,
 * ATTN_JVP_ERR_TIMEOUT if a kernel that finished before the exchange gave up
 * on a pipeline wait (its outputs are then unspecified), or
 * ATTN_JVP_ERR_LAUNCH if the launch or the synchronisation failed.  If `site`
 * is not NULL it receives the code of the first wait that gave up (0 if none).
 * The word is per device, not per stream: a check on one stream also reports
 * (and clears) a timeout of a kernel on another stream of the same device,
 * if that kernel finished before the exchange ran.  Host threads that check
 * at the same time take turns; no recorded site is lost.
 */
int attn_jvp_check(void *stream, int *site);

/* Static English text for a status code. */
const char *attn_jvp_status_string(int status);

/*
 * attn_jvp_fwd_trace -- attn_jvp_fwd in the trace build: the same results,
 * bit for bit, plus SM clock stamps (clock64) of the pipeline events of each
 * key tile, for measuring where the time of a key tile goes.  No counterpart
 * on the pages: it exists to profile the kernel.
 *   trace        device buffer of uint64 [trace_ctas][trace_tiles][11], written
 *                where a stamp is taken and left as it was elsewhere; 8-byte
 *                aligned, not overlapping any other argument
 *   trace_tiles  key tiles stamped per CTA (a CTA counts the key tiles of all
 *                its query tiles in order), >= 1
 *   trace_ctas   CTAs stamped (blockIdx < trace_ctas), >= 1; the launch has
 *                min(query tiles, SM count) CTAs
 * Events per key tile (cycles of the CTA's SM; compare within a CTA only):
 *   0 K/K' loads issued, 1 V/V' loads issued, 2 S MMAs issued, 3 P V MMAs
 *   issued, 4 P (sS' - c) V MMAs issued; then for softmax warpgroup g = 0, 1
 *   (the warpgroup's first warp): 5 + 3g S seen, 6 + 3g P signalled,
 *   7 + 3g P (sS' - c) signalled.  At d = 64 warpgroup g handles the key tiles
 *   with index % 2 == g, so only its events are stamped for them.
 * Returns what attn_jvp_fwd returns, or ATTN_JVP_ERR_NULL (trace NULL),
 * _VALUE (trace_tiles or trace_ctas < 1, or overlap), _ALIGN.
 */
int attn_jvp_fwd_trace(const void *q, const void *k, const void *v,
                       const void *q_dot, const void *k_dot, const void *v_dot,
                       void *o, void *o_dot, float *lse,
                       int B, int H, int Lq, int Lk, int d, float scale,
                       const int32_t *kv_len, void *stream,
                       unsigned long long *trace, int trace_tiles, int trace_ctas);

/*
 * attn_jvp_fwd_debug -- test hook: attn_jvp_fwd with an explicit wait limit
 * and fault-injection flags, so a test can make a device-side wait run out
 * without hanging or faulting the GPU.
 *   timeout_ns  limit for every device-side wait (0 = the default, 2 s)
 *   flags       ATTN_JVP_DEBUG_* bits; 0 behaves exactly like attn_jvp_fwd;
 *               any other bit is ATTN_JVP_ERR_VALUE
 * No counterpart on the pages: it exists to test the failure path.
 */
#define ATTN_JVP_DEBUG_STARVE_Q 1    /* never load Q/Q': the first wait on it runs out */
int attn_jvp_fwd_debug(const void *q, const void *k, const void *v,
                       const void *q_dot, const void *k_dot, const void *v_dot,
                       void *o, void *o_dot, float *lse,
                       int B, int H, int Lq, int Lk, int d, float scale,
                       const int32_t *kv_len, void *stream,
                       uint64_t timeout_ns, int flags);

/* Library version, for logs: major*10000 + minor*100 + patch (0.2.0). */
int attn_jvp_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_JVP_H */
