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

/*
 * Backward of the operator above (fp64; the reference for the backward's parity).
 *
 * The calm-mamba page (section "GPU acceleration (Triton kernels)") says only that its
 * backward recomputes the forward; the gradients themselves are the chain rule through
 * steps 2, 4, 5 and 6, written out here step by step in reverse.  Boundary gradients are
 * fp32 on the openfluke stress-test page ("Activations and boundary gradients are
 * Float32"); this oracle computes them in fp64.
 *
 * Given dy = dLoss/dy [batch, L, d_inner], it returns dLoss with respect to every input:
 *   dxp, dz, ddt_raw [batch, L, d_inner]; dB, dC [batch, L, d_state];
 *   dA_log [d_inner, d_state]; dD, dconv_b, ddt_bias [d_inner]; dconv_w [d_inner, d_conv];
 *   and, when the forward started from a cached state (h_in, conv_state_in), dh_in
 *   [batch, d_inner, d_state] and dconv_state_in [batch, d_inner, d_conv-1].
 * All outputs are overwritten.  dconv_b may be NULL when the forward had no conv bias;
 * seq_idx, h_in, conv_state_in (forward inputs) and dh_in, dconv_state_in may be NULL.
 * With seq_idx the forward resets both states at every id change (see oracle_mixer): a
 * conv tap lying before the step's document start is zero, so it passes no gradient; the
 * state entering a reset step is zero, so the adjoint stops there.
 *
 * Per channel (b, d), with xpad = [0 (K-1) ; x'], pre_t = conv_b + sum_k w_k xpad[t+k],
 * u_t = SiLU(pre_t), v_t = dt_raw_t + dt_bias, Delta_t = softplus(v_t),
 * a_{t,n} = exp(Delta_t A_n) (A = -exp(A_log)), h_{t,n} = a_{t,n} h_{t-1,n} + Delta_t B_{t,n} u_t,
 * yc_t = sum_n C_{t,n} h_{t,n} + D u_t, y_t = yc_t g_t with g_t = SiLU(z_t):
 *   dz_t     = dy_t yc_t SiLU'(z_t),   SiLU'(v) = s (1 + v (1 - s)), s = sigmoid(v)
 *   dyc_t    = dy_t g_t
 *   dC_{t,n} += dyc_t h_{t,n};   dD += dyc_t u_t;   du_t = dyc_t D
 *   reverse in t, with the adjoint state lam_n (lam = 0 after the last step):
 *     lam_n += dyc_t C_{t,n}
 *     dB_{t,n} += lam_n Delta_t u_t;   du_t += lam_n Delta_t B_{t,n}
 *     dDelta_t += lam_n B_{t,n} u_t + lam_n h_{t-1,n} a_{t,n} A_n
 *     dA_n += lam_n h_{t-1,n} a_{t,n} Delta_t
 *     lam_n *= a_{t,n}                         (carried to step t-1)
 *   dv_t = dDelta_t sigmoid(v_t):  ddt_raw_t = dv_t,  ddt_bias += dv_t
 *   dpre_t = du_t SiLU'(pre_t):  dconv_b += dpre_t,  dconv_w_k += dpre_t xpad[t+k],
 *                                dxp_{t'} += dpre_t w_k  for xpad[t+k] = x'[t'] (t' = t+k-K+1 >= 0)
 *   dA_log_n = dA_n A_n   (dA/dA_log = -exp(A_log) = A);
 *   dh_in = lam after step 0 (the adjoint carried into the initial state);
 *   dconv_state_in_k = the gradient of xpad[k], k < K-1, collected like dxp.
 */
static double sigm(double v) { return 1.0 / (1.0 + exp(-v)); }
static double silu_d(double v) { const double s = sigm(v); return s * (1.0 + v * (1.0 - s)); }

int oracle_mixer_bwd_f64(int64_t batch, int64_t seqlen, int64_t d_inner, int64_t d_state,
                         int64_t d_conv, const double* xp, const double* z, const double* dt_raw,
                         const double* Bm, const double* Cm, const double* A_log, const double* Dv,
                         const double* conv_w, const double* conv_b, const double* dt_bias,
                         const int32_t* seq_idx, const double* h_in,
                         const double* conv_state_in, const double* dy, double* dxp, double* dz,
                         double* ddt_raw, double* dB, double* dC, double* dA_log, double* dD,
                         double* dconv_w, double* dconv_b, double* ddt_bias, double* dh_in,
                         double* dconv_state_in, int nthreads) {
  if (batch < 0 || seqlen < 0 || d_inner < 0 || d_state < 1 || d_conv < 1) return 1;
  const int64_t L = seqlen, Di = d_inner, N = d_state, K = d_conv;
  int nth = nthreads > 0 ? nthreads : oracle_max_threads();
  (void)nth;
  /* per-batch-row partial sums of the parameter gradients (rows run in parallel) */
  const int64_t np = Di * N + Di + Di * K + Di + Di;
  double* part = (double*)calloc((size_t)(batch > 0 ? batch : 1) * (size_t)np, sizeof(double));
  if (!part) return 2;
  for (int64_t i = 0; i < batch * L * N; ++i) { dB[i] = 0.0; dC[i] = 0.0; }
  int bad = 0;

#pragma omp parallel for schedule(dynamic, 1) num_threads(nth)
  for (int64_t b = 0; b < batch; ++b) {
    double* pA = part + b * np;          /* dA [Di, N] (before the chain to A_log) */
    double* pD = pA + Di * N;            /* dD [Di] */
    double* pW = pD + Di;                /* dconv_w [Di, K] */
    double* pCb = pW + Di * K;           /* dconv_b [Di] */
    double* pDb = pCb + Di;              /* ddt_bias [Di] */
    double* xpad = (double*)malloc(sizeof(double) * (size_t)(K - 1 + L));
    double* pre = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    double* u = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    double* vv = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    double* del = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    double* du = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    double* ddel = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    double* h = (double*)malloc(sizeof(double) * (size_t)((L + 1) * N));   /* h[-1..L-1] */
    double* A = (double*)malloc(sizeof(double) * (size_t)N);
    double* lam = (double*)malloc(sizeof(double) * (size_t)N);
    double* dxpad = (double*)malloc(sizeof(double) * (size_t)(K - 1 + L));
    char* rs = (char*)malloc((size_t)(L > 0 ? L : 1));      /* reset at step t */
    if (!xpad || !pre || !u || !vv || !del || !du || !ddel || !h || !A || !lam || !dxpad || !rs) {
      bad = 1;
    } else {
      for (int64_t d = 0; d < Di; ++d) {
        /* forward, keeping every intermediate; tap k of step t is live unless a reset lies
           in (its position, t] */
        for (int64_t k = 0; k < K - 1; ++k)
          xpad[k] = conv_state_in ? conv_state_in[(b * Di + d) * (K - 1) + k] : 0.0;
        for (int64_t t = 0; t < L; ++t) xpad[K - 1 + t] = xp[(b * L + t) * Di + d];
        for (int64_t t = 0; t < L; ++t)
          rs[t] = (char)(seq_idx && t > 0 && seq_idx[b * L + t] != seq_idx[b * L + t - 1]);
        for (int64_t n = 0; n < N; ++n) {
          A[n] = -exp(A_log[d * N + n]);
          h[n] = h_in ? h_in[(b * Di + d) * N + n] : 0.0;
        }
        for (int64_t t = 0; t < L; ++t) {
          double acc = conv_b ? conv_b[d] : 0.0;
          for (int64_t k = 0; k < K; ++k) {
            int live = 1;
            for (int64_t s2 = t + k - (K - 1) + 1; s2 <= t; ++s2) if (s2 >= 0 && rs[s2]) live = 0;
            if (live) acc += conv_w[d * K + k] * xpad[t + k];
          }
          pre[t] = acc;
          u[t] = acc * sigm(acc);
          vv[t] = dt_raw[(b * L + t) * Di + d] + dt_bias[d];
          del[t] = fmax(vv[t], 0.0) + log1p(exp(-fabs(vv[t])));
          for (int64_t n = 0; n < N; ++n)
            h[(t + 1) * N + n] = exp(del[t] * A[n]) * (rs[t] ? 0.0 : h[t * N + n]) +
                                 del[t] * Bm[(b * L + t) * N + n] * u[t];
        }
        /* gate and output readout */
        for (int64_t t = 0; t < L; ++t) {
          const int64_t o = (b * L + t) * Di + d;
          double yc = Dv[d] * u[t];
          for (int64_t n = 0; n < N; ++n) yc += Cm[(b * L + t) * N + n] * h[(t + 1) * N + n];
          const double zz = z[o];
          dz[o] = dy[o] * yc * silu_d(zz);
          const double dyc = dy[o] * zz * sigm(zz);
          for (int64_t n = 0; n < N; ++n) dC[(b * L + t) * N + n] += dyc * h[(t + 1) * N + n];
          pD[d] += dyc * u[t];
          du[t] = dyc * Dv[d];
          ddel[t] = 0.0;
        }
        /* reverse scan with the adjoint state */
        for (int64_t n = 0; n < N; ++n) lam[n] = 0.0;
        for (int64_t t = L - 1; t >= 0; --t) {
          const int64_t o = (b * L + t) * Di + d;
          const double zz = z[o];
          const double dyc = dy[o] * zz * sigm(zz);
          for (int64_t n = 0; n < N; ++n) {
            const double Bn = Bm[(b * L + t) * N + n], Cn = Cm[(b * L + t) * N + n];
            const double a = exp(del[t] * A[n]);
            const double hprev = rs[t] ? 0.0 : h[t * N + n];   /* the state entering step t */
            lam[n] += dyc * Cn;
            dB[(b * L + t) * N + n] += lam[n] * del[t] * u[t];
            du[t] += lam[n] * del[t] * Bn;
            ddel[t] += lam[n] * Bn * u[t] + lam[n] * hprev * a * A[n];
            pA[d * N + n] += lam[n] * hprev * a * del[t];
            lam[n] = rs[t] ? 0.0 : lam[n] * a;
          }
        }
        if (dh_in)
          for (int64_t n = 0; n < N; ++n) dh_in[(b * Di + d) * N + n] = lam[n];
        /* softplus and conv + SiLU */
        for (int64_t k = 0; k < K - 1 + L; ++k) dxpad[k] = 0.0;
        for (int64_t t = 0; t < L; ++t) {
          const int64_t o = (b * L + t) * Di + d;
          const double dv = ddel[t] * sigm(vv[t]);
          ddt_raw[o] = dv;
          pDb[d] += dv;
          const double dpre = du[t] * silu_d(pre[t]);
          pCb[d] += dpre;
          for (int64_t k = 0; k < K; ++k) {
            int live = 1;
            for (int64_t s2 = t + k - (K - 1) + 1; s2 <= t; ++s2) if (s2 >= 0 && rs[s2]) live = 0;
            if (!live) continue;
            pW[d * K + k] += dpre * xpad[t + k];
            dxpad[t + k] += dpre * conv_w[d * K + k];
          }
        }
        for (int64_t t = 0; t < L; ++t) dxp[(b * L + t) * Di + d] = dxpad[K - 1 + t];
        if (dconv_state_in)
          for (int64_t k = 0; k < K - 1; ++k)
            dconv_state_in[(b * Di + d) * (K - 1) + k] = dxpad[k];
      }
    }
    free(xpad); free(pre); free(u); free(vv); free(del); free(du); free(ddel); free(h);
    free(A); free(lam); free(dxpad); free(rs);
  }
  /* sum the rows' parameter gradients; chain dA -> dA_log */
  for (int64_t i = 0; i < Di * N; ++i) dA_log[i] = 0.0;
  for (int64_t d = 0; d < Di; ++d) {
    dD[d] = 0.0; ddt_bias[d] = 0.0;
    if (dconv_b) dconv_b[d] = 0.0;
    for (int64_t k = 0; k < K; ++k) dconv_w[d * K + k] = 0.0;
  }
  for (int64_t b = 0; b < batch; ++b) {
    const double* pA = part + b * np;
    const double* pD = pA + Di * N;
    const double* pW = pD + Di;
    const double* pCb = pW + Di * K;
    const double* pDb = pCb + Di;
    for (int64_t i = 0; i < Di * N; ++i) dA_log[i] += pA[i];
    for (int64_t d = 0; d < Di; ++d) {
      dD[d] += pD[d]; ddt_bias[d] += pDb[d];
      if (dconv_b) dconv_b[d] += pCb[d];
      for (int64_t k = 0; k < K; ++k) dconv_w[d * K + k] += pW[d * K + k];
    }
  }
  for (int64_t d = 0; d < Di; ++d)
    for (int64_t n = 0; n < N; ++n) dA_log[d * N + n] *= -exp(A_log[d * N + n]);
  free(part);
  return bad ? 2 : 0;
}
