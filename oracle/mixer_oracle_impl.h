/*
 * Body of the CPU oracle, written once and compiled for two arithmetic types.
 * mixer_oracle.c includes this file with REAL = double (the reference for parity) and
 * REAL = float (used only to show that a plain fp32 recurrence lies inside the fp32
 * tolerance band).  ORACLE_FN(name) appends the precision suffix; REXP, RLOG1P, RFABS
 * and RFMAX are the libm functions of that type.
 */

static REAL ORACLE_FN(silu)(REAL v) {
  /* SiLU(v) = v * sigmoid(v) = v / (1 + exp(-v)) */
  return v / ((REAL)1 + REXP(-v));
}

static REAL ORACLE_FN(softplus)(REAL v) {
  /* softplus(v) = log(1 + exp(v)) = max(v, 0) + log(1 + exp(-|v|)) */
  return RFMAX(v, (REAL)0) + RLOG1P(REXP(-RFABS(v)));
}

int ORACLE_FN(oracle_mixer)(int64_t batch, int64_t seqlen, int64_t d_inner, int64_t d_state,
                            int64_t d_conv, const REAL* xp, const REAL* z, const REAL* dt_raw,
                            const REAL* Bm, const REAL* Cm, const REAL* A_log, const REAL* Dv,
                            const REAL* conv_w, const REAL* conv_b, const REAL* dt_bias,
                            const int32_t* seq_idx, const REAL* h_in, const REAL* conv_state_in,
                            REAL* y, REAL* h_out,
                            REAL* conv_state_out, int nthreads) {
  if (batch < 0 || seqlen < 0 || d_inner < 0 || d_state < 1 || d_conv < 1) return 1;
  const int64_t L = seqlen, Di = d_inner, N = d_state, K = d_conv;
  const int64_t nch = batch * Di;
  int bad = 0;
  int nth = nthreads > 0 ? nthreads : oracle_max_threads();
  (void)nth;

#pragma omp parallel for schedule(dynamic, 1) num_threads(nth)
  for (int64_t ch = 0; ch < nch; ++ch) {
    const int64_t b = ch / Di, d = ch % Di;
    REAL* xpad = (REAL*)malloc(sizeof(REAL) * (size_t)(K - 1 + L));
    REAL* h = (REAL*)malloc(sizeof(REAL) * (size_t)N);
    REAL* A = (REAL*)malloc(sizeof(REAL) * (size_t)N);
    if (!xpad || !h || !A) {
      free(xpad); free(h); free(A);
      bad = 1;
      continue;
    }
    /* xpad = the K-1 cached inputs (oldest first, zeros without a cache), then x'[b,:,d] */
    for (int64_t k = 0; k < K - 1; ++k)
      xpad[k] = conv_state_in ? conv_state_in[(b * Di + d) * (K - 1) + k] : (REAL)0;
    for (int64_t t = 0; t < L; ++t) xpad[K - 1 + t] = xp[(b * L + t) * Di + d];

    for (int64_t n = 0; n < N; ++n) {
      h[n] = h_in ? h_in[(b * Di + d) * N + n] : (REAL)0;
      A[n] = -REXP(A_log[d * N + n]);               /* A = -exp(A_log) */
    }

    for (int64_t t = 0; t < L; ++t) {
      /* document reset (niverel-mamba, section "seq_idx strict reset"): where seq_idx
         changes between t-1 and t, the conv state (the K-1 inputs before t) and the SSM
         state are zero before step t */
      if (seq_idx && t > 0 && seq_idx[b * L + t] != seq_idx[b * L + t - 1]) {
        for (int64_t k = 0; k < K - 1; ++k) xpad[t + k] = (REAL)0;
        for (int64_t n = 0; n < N; ++n) h[n] = (REAL)0;
      }

      /* step 2: causal depthwise conv, then SiLU */
      REAL acc = conv_b ? conv_b[d] : (REAL)0;
      for (int64_t k = 0; k < K; ++k) acc = acc + conv_w[d * K + k] * xpad[t + k];
      const REAL u = ORACLE_FN(silu)(acc);

      /* step 4: Delta = softplus(dt_raw + dt_bias) */
      const REAL delta = ORACLE_FN(softplus)(dt_raw[(b * L + t) * Di + d] + dt_bias[d]);

      /* step 5: h[n] = exp(Delta*A[n]) * h[n] + Delta*B[t,n]*u;  y = sum_n C[t,n]*h[n] + D*u */
      const REAL* Bt = Bm + (b * L + t) * N;
      const REAL* Ct = Cm + (b * L + t) * N;
      REAL yv = (REAL)0;
      for (int64_t n = 0; n < N; ++n) {
        h[n] = REXP(delta * A[n]) * h[n] + delta * Bt[n] * u;
        yv = yv + Ct[n] * h[n];
      }
      yv = yv + Dv[d] * u;

      /* step 6: gate */
      y[(b * L + t) * Di + d] = yv * ORACLE_FN(silu)(z[(b * L + t) * Di + d]);
    }

    if (h_out)
      for (int64_t n = 0; n < N; ++n) h_out[(b * Di + d) * N + n] = h[n];
    if (conv_state_out)
      for (int64_t k = 0; k < K - 1; ++k)
        conv_state_out[(b * Di + d) * (K - 1) + k] = xpad[L + k];
    free(xpad); free(h); free(A);
  }
  return bad ? 2 : 0;
}
