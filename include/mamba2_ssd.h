/*
 * mamba2_ssd.h -- C ABI of the B200 (sm_100a) Mamba2 selective scan (the SSD layer).
 *
 * The recurrence is that of the Mamba2 layer whose weight contract niverel-mamba 0.1.0
 * describes (section "The weight contract": dt_bias, A_log and D hold one value per
 * head; headdim 64, ngroups 1 and chunk_size 256 in the reference configuration
 * d_model 768, d_state 128, expand 2), i.e. the Mamba recurrence of calm-mamba 0.1.4
 * ("Mamba operator") with one scalar A, Delta and D per head and one B/C pair per group
 * of heads.  For batch row b, head h in group g = h / (nheads / ngroups), channel p < 64,
 * state n < d_state:
 *
 *   Delta_t    = softplus(dt_raw[b,t,h] + dt_bias[h]),   A = -exp(A_log[h])
 *   h[p, n]   <- exp(Delta_t * A) * h[p, n] + Delta_t * x[b,t,h,p] * B[b,t,g,n]
 *   y[b,t,h,p] = sum_n C[b,t,g,n] * h[p, n] + D[h] * x[b,t,h,p]
 *   out        = y * SiLU(z[b,t,h,p])        (only when z is given)
 *
 * x is the activation after the layer's causal conv and SiLU; the conv, the projections
 * and the gated RMSNorm of the full layer stay outside this entry point (with the norm,
 * pass z = NULL and apply the gate inside the norm).  The state starts from h_in (zero
 * when NULL).  The computation is chunked (64 steps per chunk) on the tensor cores; the
 * result equals the sequential recurrence up to rounding (niverel-mamba 0.1.0, section
 * "Measured tolerances": chunked and sequential evaluation agree).  Long sequences of few
 * (batch row, head) pairs are also cut into time segments (see the workspace below).
 *
 * Conventions are those of mamba_mixer.h (caller-owned device memory, stream-ordered,
 * host-side checks before anything is enqueued, mamba_last_error for the message):
 *
 *   Layouts   x, z, y       [batch, seqlen, nheads, headdim]    bf16
 *             dt_raw        [batch, seqlen, nheads]             bf16
 *             seq_idx       [batch, seqlen]                     int32
 *             B, C          [batch, seqlen, ngroups, d_state]   bf16
 *             A_log, D, dt_bias  [nheads]                       fp32
 *             h_in, h_out   [batch, nheads, headdim, d_state]   fp32
 *   Support   io_dtype MAMBA_BF16, headdim 64, d_state 64 or 128, ngroups >= 1 dividing
 *             nheads, batch <= 65535; batch, seqlen or nheads may be 0.
 *   Numerics  the products run with bf16 operands (the inputs exactly; the masked C B^T,
 *             the state for the inter-chunk term and Delta-weighted x are rounded once
 *             to bf16) and fp32 accumulation; the carried state is fp32.
 *   Errors    MAMBA_ERR_INVALID_ARGUMENT  NULL required pointer, negative size, ngroups
 *                                         not dividing nheads, an output overlapping an
 *                                         input (h_out == h_in exactly is allowed)
 *             MAMBA_ERR_UNSUPPORTED       dtype, headdim, d_state or batch outside the above
 *             MAMBA_ERR_ALIGNMENT         x, z, y, B, C, h_in or h_out not 16-byte
 *                                         aligned; dt_raw not 2-byte; A_log, D, dt_bias,
 *                                         seq_idx not 4-byte aligned
 *             MAMBA_ERR_WORKSPACE         workspace missing, too small, or not 256-byte
 *                                         aligned
 *             MAMBA_ERR_CUDA              a launch failed
 */
#ifndef MAMBA2_SSD_H_
#define MAMBA2_SSD_H_

#include <stddef.h>
#include <stdint.h>

#include "mamba_mixer.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
  int64_t batch;
  int64_t seqlen;
  int64_t nheads;
  int64_t headdim;
  int64_t d_state;
  int64_t ngroups;
  int32_t io_dtype; /* mamba_dtype */
  int32_t reserved; /* set to 0 */
} mamba2_dims;

/*
 * Device workspace, in bytes, that mamba2_ssd_fwd needs for `dims` (0 for invalid dims, and
 * 0 when the sequence is not split).  With few (batch row, head) pairs the sequence of each
 * pair is cut into time segments that run in parallel: a state pass leaves each segment's
 * end state (fp32, headdim x d_state) and summed decay exponent here, with a copy of h_in,
 * and the main pass starts every segment from the earlier ones folded together.
 */
MAMBA_API size_t mamba2_ssd_fwd_workspace_bytes(const mamba2_dims* dims);

/*
 * Forward of the Mamba2 scan over [0, seqlen).  Writes y (every element) and, when h_out
 * is not NULL, the state after the last step (h_in when seqlen == 0).  z, seq_idx and
 * h_in may be NULL.  seq_idx [batch, seqlen] int32 packs documents into rows: the state is
 * zeroed before every step t > 0 whose id differs from step t - 1's (niverel-mamba 0.1.0,
 * section "seq_idx strict reset"), so h_in belongs to the row's first document and h_out
 * to its last.  workspace: device memory of at least mamba2_ssd_fwd_workspace_bytes(dims) bytes,
 * 256-byte aligned, overlapping no other argument (may be NULL when that size is 0);
 * fully rewritten by every call, nothing needs clearing.  MAMBA_ERR_WORKSPACE when it is
 * missing or too small.
 */
MAMBA_API int mamba2_ssd_fwd(const mamba2_dims* dims, const void* x, const void* dt_raw,
                             const float* A_log, const void* B, const void* C, const float* D,
                             const float* dt_bias, const void* z, const int32_t* seq_idx,
                             const float* h_in, void* y, float* h_out, void* workspace,
                             size_t workspace_bytes, void* cuda_stream);

/*
 * Status of mamba2_ssd_fwd's tensor-core pass (rows without seq_idx), which waits on its own
 * asynchronous copies and products: waits for `cuda_stream`, then reads and clears the
 * library's status word for the Mamba2 scan (one per CUDA context).  Returns
 * MAMBA_ERR_TIMEOUT if a call since the last check gave up on a bounded wait (about one
 * second; its outputs are then incomplete), MAMBA_OK otherwise.  Allocates nothing.
 */
MAMBA_API int mamba2_ssd_check(void* cuda_stream);

/*
 * One decode step of the Mamba2 scan on a cached state (niverel-mamba 0.1.0, section
 * "Autoregressive decoding": step(x_t, state) returns the output and a new state, and
 * concatenated steps equal the forward).  dims->seqlen must be 1; the layouts are those of
 * mamba2_ssd_fwd with seqlen 1.  h_in is required; the new state goes to h_out, which may be
 * h_in itself (in-place update; any other overlap is MAMBA_ERR_INVALID_ARGUMENT).  z may be
 * NULL.  No workspace.
 */
MAMBA_API int mamba2_ssd_step(const mamba2_dims* dims, const void* x, const void* dt_raw,
                              const float* A_log, const void* B, const void* C, const float* D,
                              const float* dt_bias, const void* z, const float* h_in, void* y,
                              float* h_out, void* cuda_stream);

/*
 * The layer's causal depthwise conv + SiLU before the scan, over the concatenated channels
 * x | B | C (niverel-mamba 0.1.0, section "The weight contract": conv1d over d_inner +
 * 2 ngroups d_state channels, 4 taps):
 *
 *   out[b,t,c] = SiLU(conv_b[c] + sum_{k<4} conv_w[c,k] * xpad[b,t+k,c]),
 *   xpad = [conv_state_in (3 inputs, oldest first; zeros when NULL) ; xbc]
 *
 * with conv_w[c, 3] on the current input.  With seq_idx [batch, seqlen] (may be NULL) a tap
 * reads zero when an id change lies between its input's step and t (the state before step 0
 * belongs to the row's first document).  The output is split as the scan takes it:
 *
 *   xbc                          [batch, seqlen, Cc]            bf16, Cc = nheads*64 + 2*ngroups*d_state
 *   conv_w                       [Cc, 4]                        fp32 (16-byte aligned)
 *   conv_b                       [Cc]                           fp32 or NULL
 *   x                            [batch, seqlen, nheads*64]     bf16 (channels 0 .. nheads*64-1)
 *   B, C                         [batch, seqlen, ngroups*d_state] bf16 (the next two blocks)
 *   conv_state_in / _out         [batch, Cc, 3]                 bf16 or NULL
 *
 * conv_state_out receives the last 3 entries of xpad (zero where an id change lies between
 * the entry's step and the last step); it may not overlap conv_state_in.  Outputs may not
 * overlap inputs or each other.  SiLU and the sums are fp32; outputs round to nearest even.
 */
MAMBA_API int mamba2_conv_silu(const mamba2_dims* dims, const void* xbc, const float* conv_w,
                               const float* conv_b, const int32_t* seq_idx,
                               const void* conv_state_in, void* x, void* B, void* C,
                               void* conv_state_out, void* cuda_stream);

/*
 * The layer's gated RMSNorm after the scan, gate first (niverel-mamba 0.1.0, section "The
 * weight contract": norm.weight over d_inner, eps 1e-5):
 *
 *   g = y * SiLU(z);  out = g / sqrt(mean(g^2) + eps) * weight
 *
 * the mean over each group of nheads*64/ngroups consecutive channels of a (b, t).  y, z, out
 * [batch, seqlen, nheads*64] bf16 (16-byte aligned); weight [nheads*64] fp32 (16-byte
 * aligned); eps >= 0.  out may not overlap an input.  fp32 arithmetic.  dims->d_state is
 * not used (it must still be 64 or 128).
 */
MAMBA_API int mamba2_gated_rmsnorm(const mamba2_dims* dims, const void* y, const void* z,
                                   const float* weight, float eps, void* out,
                                   void* cuda_stream);

#ifdef __cplusplus
}
#endif

#endif /* MAMBA2_SSD_H_ */
