/*
 * mamba_mixer.h -- C ABI of the B200 (sm_100a) fused Mamba-1 selective-SSM mixer core.
 *
 * The operator is the "Mamba operator" of calm-mamba 0.1.4 (PyPI PKG-INFO), steps 2 and
 * 4-6; the projections of steps 1, 3, 4 (matmul) and 7 stay outside this library and
 * their outputs (x', z, dt_raw, B, C) are its inputs:
 *
 *   u[t]   = SiLU(conv_b + sum_{k<4} conv_w[k] * xpad[t+k])     step 2 (causal, left-padded)
 *   D[t]   = softplus(dt_raw[t] + dt_bias)                       step 4
 *   h[t]   = exp(D[t]*A) * h[t-1] + D[t]*B[t]*u[t],  A = -exp(A_log)
 *   y[t]   = C[t] . h[t] + D*u[t]                                 step 5 (selective scan)
 *   out[t] = y[t] * SiLU(z[t])                                    step 6 (gate)
 *
 * with xpad = [conv state (3 values, oldest first) or zeros ; x'[0..L-1]].  The decode
 * step is the same computation for one token on a cached (h, conv state) pair: calm-mamba
 * 0.1.4 (introduction: O(1) per-token state-cached generation) and niverel-mamba 0.1.0
 * (section "Autoregressive decoding": step returns a new state and mutates nothing).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Memory.    Every array argument is a DEVICE pointer owned by the caller.  The library
 *            allocates no device memory and keeps no state besides a thread-local error
 *            message.  Work is enqueued on `cuda_stream` (a cudaStream_t; NULL = the
 *            legacy default stream); calls return once the work is enqueued.
 * Layouts.   Row-major, channel-contiguous ("BLD"):
 *              x', z, dt_raw, y         [batch, seqlen, d_inner]   io dtype
 *              B, C                     [batch, seqlen, d_state]   io dtype (shared by all
 *                                                                  channels of a (b, t))
 *              A_log                    [d_inner, d_state]         fp32
 *              D, conv_b, dt_bias       [d_inner]                  fp32
 *              conv_w                   [d_inner, d_conv]          fp32
 *              h (SSM state)            [batch, d_inner, d_state]  fp32
 *              conv state               [batch, d_inner, d_conv-1] io dtype, oldest first
 * Types.     io dtype MAMBA_F32 or MAMBA_BF16; all arithmetic is fp32; outputs in the io
 *            dtype are rounded to nearest even.
 * Support.   d_conv == 4, d_state in {8, 16}, d_inner a multiple of 8; batch, seqlen and
 *            d_inner may be 0 (nothing to do beyond writing the states).
 * Errors.    Every check is made on the host before anything is enqueued; a call that
 *            returns non-OK has enqueued nothing.  There is no fallback path.
 *              MAMBA_ERR_INVALID_ARGUMENT  NULL required pointer, negative size, bad
 *                                          overlap between an output and another array
 *              MAMBA_ERR_UNSUPPORTED       d_conv, d_state, d_inner or dtype outside the
 *                                          supported set
 *              MAMBA_ERR_ALIGNMENT         an activation, state or output pointer not
 *                                          16-byte aligned, or a parameter pointer not
 *                                          4-byte aligned
 *              MAMBA_ERR_WORKSPACE         workspace smaller than
 *                                          mamba_mixer_fwd_workspace_bytes() or not
 *                                          16-byte aligned
 *              MAMBA_ERR_CUDA              a CUDA launch or query failed
 *              MAMBA_ERR_TIMEOUT           (mamba_mixer_check only) a forward kernel gave
 *                                          up on a bounded wait; see mamba_mixer_check
 *            mamba_last_error() gives a one-line message for the last non-OK return on
 *            the calling thread.
 * Waits.     The forward kernels wait on their own asynchronous copies (TMA into shared
 *            memory).  Every such wait gives up after one second, stops the CTA cleanly
 *            and records MAMBA_ERR_TIMEOUT in the workspace status word; no call hangs.
 */
#ifndef MAMBA_MIXER_H_
#define MAMBA_MIXER_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MAMBA_MIXER_ABI_VERSION 1

#if defined(__GNUC__)
#define MAMBA_API __attribute__((visibility("default")))
#else
#define MAMBA_API
#endif

typedef enum { MAMBA_F32 = 0, MAMBA_BF16 = 1 } mamba_dtype;

typedef enum {
  MAMBA_OK = 0,
  MAMBA_ERR_INVALID_ARGUMENT = 1,
  MAMBA_ERR_UNSUPPORTED = 2,
  MAMBA_ERR_ALIGNMENT = 3,
  MAMBA_ERR_WORKSPACE = 4,
  MAMBA_ERR_CUDA = 5,
  MAMBA_ERR_TIMEOUT = 6
} mamba_status;

/* Problem sizes.  io_dtype holds a mamba_dtype value. */
typedef struct {
  int64_t batch;
  int64_t seqlen;
  int64_t d_inner;
  int64_t d_state;
  int64_t d_conv;
  int32_t io_dtype;
  int32_t reserved; /* must be 0 */
} mamba_dims;

/*
 * Device workspace, in bytes, that mamba_mixer_fwd needs for `dims`: a 256-byte header
 * whose first 4 bytes are the status word, then, when the sequence is split into time
 * chunks, what the chunks hand on:
 *   - bf16 I/O (chained chunks, one launch): one flag per (32-channel tile, scan warp) and
 *     each tile's carried state, fp32 [tiles, 32, d_state]; the forward resets the flags
 *     and its unit counter (header bytes 64..67) itself on the stream;
 *   - fp32 I/O (a chunk-state pass, then the main pass): each chunk's carry aggregate
 *     (decay product and local end state, fp32 [batch, chunks-1, d_inner, d_state] each).
 * The status word must be zero before the first forward that uses the workspace (clear the
 * header once after allocating it); the library only sets it on a timeout and
 * mamba_mixer_check clears it.  Returns 0 for dims the library does not support
 * (mamba_mixer_fwd then reports why).
 */
MAMBA_API size_t mamba_mixer_fwd_workspace_bytes(const mamba_dims* dims);

/*
 * Number of kernels one mamba_mixer_fwd call with `dims` launches (1, or 2 for fp32 I/O
 * with time chunks: the chunk-state pass, then the main pass); 0 when there is nothing to
 * compute; -1 for unsupported dims.
 */
MAMBA_API int mamba_mixer_fwd_launches(const mamba_dims* dims);

/*
 * Fused forward over a whole sequence from a zero state (no initial state: the
 * niverel-mamba weight contract, section "The weight contract", has no init_states).
 * Inputs: xp, z, dt_raw, B, C, A_log, D, conv_w, conv_b (may be NULL = zero bias),
 * dt_bias.  Outputs: y [batch, seqlen, d_inner]; h_out, the SSM state after the last
 * token (may be NULL = not written); conv_state_out, the last d_conv-1 inputs of xpad
 * (zeros included when seqlen < d_conv-1; may be NULL = not written).
 * Outputs must not overlap any input or each other.  `workspace` (device, 16-byte
 * aligned, at least mamba_mixer_fwd_workspace_bytes(dims) bytes) is required.  Calls that
 * share a workspace must not overlap on the GPU.
 */
MAMBA_API int mamba_mixer_fwd(const mamba_dims* dims, const void* xp, const void* z,
                    const void* dt_raw, const void* B, const void* C, const float* A_log,
                    const float* D, const float* conv_w, const float* conv_b,
                    const float* dt_bias, void* y, float* h_out, void* conv_state_out,
                    void* workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * The fused forward over packed documents and/or from a cached state (niverel-mamba 0.1.0,
 * section "seq_idx strict reset"; the state pair is the one of section "Autoregressive
 * decoding").  Same arguments, workspace and result as mamba_mixer_fwd, plus three
 * optional inputs (each may be NULL):
 *   seq_idx        int32 [batch, seqlen], 4-byte aligned: document ids.  Wherever
 *                  seq_idx[b, t] != seq_idx[b, t-1], the conv state and the SSM state reset
 *                  to zero before token t, so a packed row equals its documents run one by
 *                  one and concatenated; boundaries need not align with anything.  The ids'
 *                  values do not matter, only where they change; position 0 never resets.
 *   h_in           fp32 [batch, d_inner, d_state], 16-byte aligned: the SSM state before
 *                  token 0 (zero when NULL), e.g. a previous call's h_out, so a long prompt
 *                  can be fed in pieces.
 *   conv_state_in  io dtype [batch, d_inner, 3], 2-byte aligned: the 3 inputs before
 *                  token 0, oldest first (zeros when NULL), e.g. a previous conv_state_out.
 * The initial state belongs to each row's first document.  h_out and conv_state_out are
 * the last document's (slots of conv_state_out older than its first token are zero).  With
 * all three NULL this is mamba_mixer_fwd.  Outputs must not overlap any input (h_in and
 * conv_state_in included: no in-place update here, since time chunks read the initial
 * state while the last chunk writes the final one).  A reset is applied as a zero decay of
 * the state: for finite states this is the reset; a non-finite state stays non-finite.
 */
MAMBA_API int mamba_mixer_fwd_packed(const mamba_dims* dims, const void* xp, const void* z,
                                     const void* dt_raw, const void* B, const void* C,
                                     const float* A_log, const float* D, const float* conv_w,
                                     const float* conv_b, const float* dt_bias,
                                     const int32_t* seq_idx, const float* h_in,
                                     const void* conv_state_in, void* y, float* h_out,
                                     void* conv_state_out, void* workspace,
                                     size_t workspace_bytes, void* cuda_stream);

/*
 * Device workspace, in bytes, that mamba_mixer_bwd needs for `dims`: a 256-byte header,
 * then the recurrence's state at the start of every 16-step tile (fp32 [batch,
 * ceil(seqlen/16), d_inner, d_state]).  0 for unsupported dims.
 */
MAMBA_API size_t mamba_mixer_bwd_workspace_bytes(const mamba_dims* dims);

/*
 * Backward of mamba_mixer_fwd (forward from a zero state, no documents), by forward
 * recompute (calm-mamba 0.1.4, section "GPU acceleration (Triton kernels)"): the gradients
 * of sum(dy * y) with respect to every input, in fp32 (the openfluke stress-test page keeps
 * boundary gradients in Float32).
 * Inputs: the forward's inputs (same layouts, io dtype activations) and dy [batch, seqlen,
 * d_inner] in the io dtype.  Outputs (fp32, device, all overwritten):
 *   dxp, dz, ddt_raw [batch, seqlen, d_inner]; dB, dC [batch, seqlen, d_state] (summed over
 *   the channels that share B and C); dA_log [d_inner, d_state]; dD, ddt_bias [d_inner];
 *   dconv_w [d_inner, d_conv]; dconv_b [d_inner] (may be NULL: not computed).
 * The sums over channels, batch rows and time use atomic additions, so the last bits of
 * those outputs may differ between runs.  Outputs must not overlap any input, each other
 * or the workspace (16-byte aligned, mamba_mixer_bwd_workspace_bytes(dims) bytes).
 */
MAMBA_API int mamba_mixer_bwd(const mamba_dims* dims, const void* xp, const void* z,
                              const void* dt_raw, const void* B, const void* C,
                              const float* A_log, const float* D, const float* conv_w,
                              const float* conv_b, const float* dt_bias, const void* dy,
                              float* dxp, float* dz, float* ddt_raw, float* dB, float* dC,
                              float* dA_log, float* dD, float* dconv_w, float* dconv_b,
                              float* ddt_bias, void* workspace, size_t workspace_bytes,
                              void* cuda_stream);

/*
 * Backward of mamba_mixer_fwd_packed: as mamba_mixer_bwd, with the forward's optional
 * seq_idx, h_in and conv_state_in (each may be NULL; see mamba_mixer_fwd_packed), and two
 * optional gradient outputs (fp32, may be NULL = not computed): dh_in [batch, d_inner,
 * d_state] and dconv_state_in [batch, d_inner, 3], the gradients of the initial state and
 * conv window (defined, as zero-input gradients, even when h_in / conv_state_in are NULL).
 * Where seq_idx changes, the conv taps before the document start pass no gradient and the
 * adjoint state stops (niverel-mamba 0.1.0, section "seq_idx strict reset").  Same
 * workspace as mamba_mixer_bwd.  Outputs must not overlap inputs, each other or the
 * workspace.
 */
MAMBA_API int mamba_mixer_bwd_packed(const mamba_dims* dims, const void* xp, const void* z,
                                     const void* dt_raw, const void* B, const void* C,
                                     const float* A_log, const float* D, const float* conv_w,
                                     const float* conv_b, const float* dt_bias,
                                     const int32_t* seq_idx, const float* h_in,
                                     const void* conv_state_in, const void* dy, float* dxp,
                                     float* dz, float* ddt_raw, float* dB, float* dC,
                                     float* dA_log, float* dD, float* dconv_w, float* dconv_b,
                                     float* ddt_bias, float* dh_in, float* dconv_state_in,
                                     void* workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * Training pair that trades memory for the backward's forward sweep.  The backward needs
 * the state at the start of every 16-step tile; mamba_mixer_bwd recomputes them (one extra
 * pass over x', dt_raw and B), while mamba_mixer_fwd_ckpt writes them during the forward
 * and mamba_mixer_bwd_ckpt reads them back.
 *
 * mamba_mixer_ckpt_bytes: bytes of that buffer, fp32 [batch, ceil(seqlen/16), d_inner,
 * d_state] (entry k = the state before step 16k; entry 0 is zero); 0 for unsupported dims.
 *
 * mamba_mixer_fwd_ckpt: mamba_mixer_fwd (same inputs, outputs, workspace and errors) that
 * also writes every entry of h_ckpt (device, 16-byte aligned, mamba_mixer_ckpt_bytes(dims)
 * bytes, overlapping no input, output or the workspace; required unless there is nothing
 * to compute).  Not for dims the forward's dt-projection or packed entry points need.
 *
 * mamba_mixer_bwd_ckpt: mamba_mixer_bwd (same arguments, outputs, workspace and errors)
 * with h_ckpt as written by mamba_mixer_fwd_ckpt on the same inputs, read only.  Its results
 * equal mamba_mixer_bwd's up to the rounding of the recomputed states.
 */
MAMBA_API size_t mamba_mixer_ckpt_bytes(const mamba_dims* dims);
MAMBA_API int mamba_mixer_fwd_ckpt(const mamba_dims* dims, const void* xp, const void* z,
                                   const void* dt_raw, const void* B, const void* C,
                                   const float* A_log, const float* D, const float* conv_w,
                                   const float* conv_b, const float* dt_bias, void* y,
                                   float* h_out, void* conv_state_out, float* h_ckpt,
                                   void* workspace, size_t workspace_bytes, void* cuda_stream);
MAMBA_API int mamba_mixer_bwd_ckpt(const mamba_dims* dims, const void* xp, const void* z,
                                   const void* dt_raw, const void* B, const void* C,
                                   const float* A_log, const float* D, const float* conv_w,
                                   const float* conv_b, const float* dt_bias,
                                   const float* h_ckpt, const void* dy, float* dxp, float* dz,
                                   float* ddt_raw, float* dB, float* dC, float* dA_log,
                                   float* dD, float* dconv_w, float* dconv_b, float* ddt_bias,
                                   void* workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * One decode step: one token for each of `batch` sequences (dims->seqlen must be 1) on a
 * cached state.  Inputs: xp, z, dt_raw [batch, 1, d_inner]; B, C [batch, 1, d_state];
 * the parameters as for mamba_mixer_fwd; h_in [batch, d_inner, d_state] fp32 and
 * conv_state_in [batch, d_inner, 3] io dtype.  Outputs: y [batch, 1, d_inner], h_out,
 * conv_state_out (the new state; both required).
 * Functional by default (distinct output buffers leave the inputs untouched).  In-place
 * update is allowed: h_out == h_in and/or conv_state_out == conv_state_in exactly; any
 * other overlap is MAMBA_ERR_INVALID_ARGUMENT.
 */
MAMBA_API int mamba_mixer_step(const mamba_dims* dims, const void* xp, const void* z,
                     const void* dt_raw, const void* B, const void* C, const float* A_log,
                     const float* D, const float* conv_w, const float* conv_b,
                     const float* dt_bias, const float* h_in, const void* conv_state_in,
                     void* y, float* h_out, void* conv_state_out, void* cuda_stream);

/*
 * The fused forward with the dt projection folded in (calm-mamba 0.1.4, section "Mamba
 * operator", step 4: dt = dt_proj(dt_low)): instead of dt_raw [batch, L, d_inner] it takes
 * dt_low [batch, L, dt_rank] (the low-rank slice of x_proj's output) and W_dt [d_inner,
 * dt_rank], both bf16 row-major and 16-byte aligned, and forms dt_raw = dt_low W_dt^T per
 * 32-step tile on the tensor cores (tcgen05, fp32 accumulation in tensor memory), kept in
 * fp32 (no bf16 rounding of dt_raw); dt_bias is added as in mamba_mixer_fwd.  Everything else
 * -- arguments, layouts, outputs, workspace (mamba_mixer_fwd_workspace_bytes of the same
 * dims), errors -- is mamba_mixer_fwd's.  bf16 I/O only (MAMBA_ERR_UNSUPPORTED otherwise);
 * dt_rank a multiple of 8 from 8 to 128 (MAMBA_ERR_UNSUPPORTED otherwise).  HBM traffic per
 * token and channel drops from 8 to 6 bytes (dt_raw is neither written by a GEMM nor read).
 */
MAMBA_API int mamba_mixer_fwd_dtproj(const mamba_dims* dims, int64_t dt_rank, const void* xp,
                                     const void* z, const void* dt_low, const void* W_dt,
                                     const void* B, const void* C, const float* A_log,
                                     const float* D, const float* conv_w, const float* conv_b,
                                     const float* dt_bias, void* y, float* h_out,
                                     void* conv_state_out, void* workspace,
                                     size_t workspace_bytes, void* cuda_stream);

/*
 * How mamba_mixer_fwd / mamba_mixer_fwd_packed split a forward with these dims (a query; it
 * launches nothing).  nchunks: time chunks per row; chunk_len: steps per chunk (the last may
 * be shorter); time_groups: time groups per CTA (1, or 4 for the two-level scan of rows with
 * few channels); chained: 1 when each chunk starts from the end state its predecessor left in
 * the workspace, 0 when chunks past the first are preceded by a chunk-state pass.  Any output
 * pointer may be NULL.  Returns MAMBA_OK, or the dims' validation error.  The pages have no
 * counterpart: it documents this library's schedule for tests and tuning.
 */
MAMBA_API int mamba_mixer_fwd_plan(const mamba_dims* dims, int* nchunks, int64_t* chunk_len,
                                   int* time_groups, int* chained);

/*
 * The status check of mamba_mixer_step, which takes no workspace: waits for `cuda_stream`,
 * then reads and clears the step's status word (library-owned, one per CUDA context).
 * Returns MAMBA_ERR_TIMEOUT if a decode step since the last check gave up on a bounded wait
 * (its outputs are then incomplete), MAMBA_OK otherwise.  Allocates nothing.
 */
MAMBA_API int mamba_mixer_step_check(void* cuda_stream);

/*
 * Waits for `cuda_stream`, then reads and clears the status word of `workspace`.
 * Returns MAMBA_ERR_TIMEOUT if a forward that used this workspace since the last check
 * gave up on a bounded wait (its outputs are then incomplete), MAMBA_OK otherwise.
 */
MAMBA_API int mamba_mixer_check(void* workspace, void* cuda_stream);

/*
 * Test hook for the bounded-wait path; not for production use.  tile >= 0 makes the CTA
 * of channel tile 0, batch row 0 and time chunk 0 of every following forward arm the
 * barrier of its time tile `tile` without issuing that tile's copies, so that its waits run
 * out (after about one second), it stops cleanly and the call's status word reads
 * MAMBA_ERR_TIMEOUT; no GPU fault is involved.  tile = -1 (the default) turns it off.
 * Process-wide; takes effect for launches enqueued after the call.
 */
MAMBA_API void mamba_mixer_set_fault_injection(int tile);

/*
 * The fused forward for callers that cannot allocate device memory.  The pages describe no
 * such entry point; it exists for this library's users.  Plugin hosts that hand over the
 * input and output buffers but no allocator, code running inside an allocator's callback,
 * and latency-critical paths that must not call cudaMalloc (it can synchronize the device)
 * cannot provide the workspace mamba_mixer_fwd asks for.  This variant takes the same
 * inputs and outputs, computes the same result, and uses a scratch array owned by the
 * library instead: 2 MiB (2097152 bytes) of device memory per GPU that loads the library,
 * held until the process exits.  It calls no cudaMalloc/cudaFree.
 * Limits and conventions:
 *   - dims whose mamba_mixer_fwd_workspace_bytes exceeds 2 MiB are rejected with
 *     MAMBA_ERR_WORKSPACE (message via mamba_last_error); use mamba_mixer_fwd for them;
 *   - the first call in each CUDA context looks up the array's device address in that
 *     context (cudaGetSymbolAddress, which also makes the device's primary context current
 *     on a thread that has none) and caches it under the context's unique id; a second
 *     context on the same device, or one re-created after a reset, does its own lookup.
 *     Make the first call in a context before any stream capture;
 *   - all calls in a context share the one array and it keeps the last call's contents:
 *     calls that overlap on the GPU (e.g. on two streams at once) race; serialize them;
 *   - a bounded-wait timeout is recorded in the array's status word, like the workspace's
 *     for mamba_mixer_fwd: mamba_mixer_noalloc_check reports and clears it.
 */
MAMBA_API int mamba_mixer_fwd_noalloc(const mamba_dims* dims, const void* xp, const void* z,
                                      const void* dt_raw, const void* B, const void* C,
                                      const float* A_log, const float* D, const float* conv_w,
                                      const float* conv_b, const float* dt_bias, void* y,
                                      float* h_out, void* conv_state_out, void* cuda_stream);

/*
 * The status check of mamba_mixer_fwd_noalloc, which has no workspace to hand to
 * mamba_mixer_check: waits for `cuda_stream`, then reads and clears the status word of the
 * library's scratch array in the current context.  Returns MAMBA_ERR_TIMEOUT if a no-alloc
 * forward since the last check gave up on a bounded wait (its outputs are then
 * incomplete), MAMBA_OK otherwise.  Allocates nothing.  No counterpart on the pages.
 */
MAMBA_API int mamba_mixer_noalloc_check(void* cuda_stream);

/* Message for the last non-OK return on this thread ("" if none). Never NULL. */
MAMBA_API const char* mamba_last_error(void);

/* Library version string, e.g. "mamba_mixer 0.1.0 (abi 1, sm_100a)". */
MAMBA_API const char* mamba_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MAMBA_MIXER_H_ */
