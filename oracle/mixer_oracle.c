/*
 * CPU oracle for the Mamba-1 selective-SSM mixer core.  TEST INFRASTRUCTURE ONLY:
 * tests, the package's smoke check and the benchmark's CPU-baseline leg call it; the
 * CUDA library never does, and this file shares nothing with it.
 *
 * It is a plain, slow, sequential restatement of the operator as calm-mamba 0.1.4
 * (PyPI PKG-INFO, section "Mamba operator") states it, steps 2 and 4-6:
 *
 *   step 2  causal depthwise conv1d (kernel d_conv, default 4), then SiLU on x'
 *   step 4  dt_proj output + bias, softplus  ->  the discretised step Delta
 *   step 5  h[t] = exp(Delta*A) * h[t-1] + Delta*B[t]*x[t];  y[t] = C[t].h[t] + D*x[t]
 *   step 6  y = y * SiLU(z)
 *
 * The projections (steps 1, 3, the matmul of 4, and 7) are outside the core: their
 * outputs x', z, dt_raw, B, C are inputs here.  The state cache for single-token
 * decoding (calm-mamba, introduction: O(1) per-token state-cached generation;
 * niverel-mamba 0.1.0, section "Autoregressive decoding": step returns a new state)
 * is the pair (h, conv_state): a decode step is this same function with L = 1 and the
 * cached pair passed in.
 *
 * Readings taken where the pages leave a step open:
 *   - A = -exp(A_log)  (the pages name A_log but never write A out);
 *   - "x[t]" in step 5 is the conv+SiLU output u[t]  (step 2 precedes step 5);
 *   - the conv is a cross-correlation over a left zero-padded sequence
 *     (section "GPU acceleration (Triton kernels)": "left-pad"):
 *       u[t] = SiLU(conv_b + sum_k conv_w[k] * xpad[t+k]),
 *       xpad = [conv_state (K-1 values, oldest first) or zeros ; x'[0..L-1]],
 *     so conv_w[K-1] multiplies the current x'[t];
 *   - conv_b may be absent (NULL means zero);
 *   - softplus(v) = log(1 + exp(v)), evaluated as max(v,0) + log1p(exp(-|v|)),
 *     the same number without overflow;  SiLU(v) = v / (1 + exp(-v));
 *   - the new conv state is the last K-1 entries of xpad (zeros included if L < K-1).
 *
 * Packed documents (niverel-mamba 0.1.0, section "seq_idx strict reset"): with an int32
 * seq_idx [batch, L], wherever seq_idx[b, t] != seq_idx[b, t-1] both the conv state and
 * the SSM state reset to zero before step t, so a packed row equals its documents run
 * one by one and concatenated.  The initial state (h_in, conv_state_in), if given,
 * belongs to the row's first document; the states returned are the last document's.
 *
 * Layouts (row-major): x', z, dt_raw, y [batch, L, d_inner]; B, C [batch, L, d_state];
 * A_log [d_inner, d_state]; D, conv_b, dt_bias [d_inner]; conv_w [d_inner, d_conv];
 * h [batch, d_inner, d_state]; conv_state [batch, d_inner, d_conv-1]; seq_idx [batch, L].
 *
 * Build: gcc -O2 -fPIC -shared -fopenmp -ffp-contract=off (no fast-math), so every
 * operation is the one written.  Channels (b, d) are independent and may run on
 * several threads; each channel is computed sequentially in time.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

#ifdef _OPENMP
#include <omp.h>
int oracle_max_threads(void) { return omp_get_max_threads(); }
#else
int oracle_max_threads(void) { return 1; }
#endif

#define REAL double
#define REXP exp
#define RLOG1P log1p
#define RFABS fabs
#define RFMAX fmax
#define ORACLE_FN(name) name##_f64
#include "mixer_oracle_impl.h"
#undef REAL
#undef REXP
#undef RLOG1P
#undef RFABS
#undef RFMAX
#undef ORACLE_FN

#define REAL float
#define REXP expf
#define RLOG1P log1pf
#define RFABS fabsf
#define RFMAX fmaxf
#define ORACLE_FN(name) name##_f32
#include "mixer_oracle_impl.h"
