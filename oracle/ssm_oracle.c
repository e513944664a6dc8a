/*
 * ssm_oracle.c -- plain fp64 CPU oracle for the selective state-space (S6) scan.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call this
 * file; only the tests, the smoke check and the benchmark's CPU-baseline leg use it.
 * It shares no code, header, table or constant with the CUDA library.
 *
 * What it computes, and where the pages define it:
 *   "Mamba: Linear-Time Sequence Modeling with Selective State Spaces" (Gu & Dao,
 *   arXiv 2312.00752; Turkish summary page), section "Yöntem" (Method):
 *     continuous SSM h'(t) = A h(t) + B x(t), y(t) = C h(t); zero-order-hold
 *     discretisation with step Δ gives Ā = exp(ΔA); the discrete recurrence is
 *     h_t = Ā h_{t-1} + B̄ x_t and the readout y_t = C h_t.
 *   Same page, section "Seçim Mekanizması (S6)": B_t and C_t are per-token vectors of
 *   length N (shared by every channel), and Δ_t = softplus(Parameter + s_Δ(x_t)); the
 *   per-channel "Parameter" is the dt_bias argument here, s_Δ(x_t) is the raw delta input.
 *   Same page, "Temel Fikirler" / "Mamba Block": the block output is multiplicatively
 *   gated; the gate used here is silu(z).
 *   "PyTorch 1ファイルでのMamba実装" (mamba-minimal news page), Hacker News comment with
 *   the sequential scan loop: the state is updated first and then read out with C_t, so
 *   y_t uses h_t (not h_{t-1}).
 *
 * Readings taken where the pages are silent (each is listed in the design notes):
 *   - Input term: B̄ x_t = Δ_t * B_t * x_t (first-order/Euler form).  The exact ZOH
 *     input term (exp(ΔA)-1)/A * B_t * x_t is available with zoh=1 (forward and backward).
 *   - A is a general real [D][N] matrix (diagonal state matrix per channel).
 *   - softplus(v) = log(1 + exp(v)), evaluated in the overflow-safe form.
 *   - The skip term D*x_t is added to y_t before the gate; z == NULL means no gate.
 *   - The initial state is zero unless h0 is given.
 *
 * Everything is double precision and plain loops in the order of the equations above;
 * the only parallelism is an OpenMP loop over independent channels (b, d).
 *
 * Layouts (all row-major, contiguous):
 *   u, delta, z, out, ypre, du, ddelta, dz, dout : [batch][dim][seqlen]
 *   B, C, dB, dC                                 : [batch][dstate][seqlen]
 *   A, dA                                        : [dim][dstate]
 *   Dskip, dt_bias, dD, ddt_bias                 : [dim]
 *   h0, hL, dhL, dh0, state                      : [batch][dim][dstate]
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* softplus(v) = log(1 + e^v), written so that neither branch overflows. */
static double sp_softplus(double v) { return v > 0.0 ? v + log1p(exp(-v)) : log1p(exp(v)); }

/* logistic sigmoid 1 / (1 + e^-v), overflow-safe. */
static double sp_sigmoid(double v) {
  if (v >= 0.0) return 1.0 / (1.0 + exp(-v));
  double e = exp(v);
  return e / (1.0 + e);
}

/* Δ_t for one channel and step: softplus(delta + dt_bias), or the plain sum when the
 * softplus flag is off (selection mechanism, Δ_t = τ_Δ(Parameter + s_Δ(x_t))). */
static double step_size(double draw, double bias, int use_softplus) {
  double v = draw + bias;
  return use_softplus ? sp_softplus(v) : v;
}

/* Coefficient multiplying B_t * x_t in the state update. */
static double input_coef(double dt, double a_dn, int zoh) {
  if (!zoh) return dt;                 /* B̄ x = Δ B x */
  if (a_dn == 0.0) return dt;          /* limit of (exp(ΔA)-1)/A as A -> 0 */
  return expm1(dt * a_dn) / a_dn;      /* ZOH: (ΔA)^-1 (exp(ΔA) - 1) Δ  for diagonal A */
}

/* d/dΔ and d/dA of the input coefficient.  Euler: (1, 0).  ZOH, c = (e^{ΔA} - 1)/A:
 * dc/dΔ = e^{ΔA};  dc/dA = (Δ e^{ΔA} - c)/A = Δ^2 ψ(ΔA) with ψ(y) = (y e^y - e^y + 1)/y^2,
 * evaluated by its Taylor series Σ_{k>=2} (k-1) y^{k-2}/k! = 1/2 + y/3 + y^2/8 + y^3/30 + ...
 * where the direct form cancels (|ΔA| < 1e-2; truncation after y^5 < 1e-15 relative). */
static void input_coef_grad(double dt, double a_dn, int zoh, double* d_dt, double* d_da) {
  if (!zoh) {
    *d_dt = 1.0;
    *d_da = 0.0;
    return;
  }
  const double y = dt * a_dn;
  *d_dt = exp(y);
  if (fabs(y) < 1e-2) {
    const double psi = 0.5 + y * (1.0 / 3.0 + y * (1.0 / 8.0 + y * (1.0 / 30.0 + y * (1.0 / 144.0 + y / 840.0))));
    *d_da = dt * dt * psi;
  } else {
    *d_da = (dt * exp(y) - expm1(y) / a_dn) / a_dn;
  }
}

static int nthreads_or_default(int nthreads) {
#ifdef _OPENMP
  return nthreads > 0 ? nthreads : omp_get_max_threads();
#else
  (void)nthreads;
  return 1;
#endif
}

int oracle_max_threads(void) { return nthreads_or_default(0); }

/*
 * Forward scan.  chans (length nchan) lists flat channel indices b*dim + d to compute;
 * chans == NULL computes every channel.  Outputs of channels not listed are untouched.
 * out: gated output; ypre (optional): the pre-gate y_t = C_t.h_t + D x_t; hL (optional).
 * Returns 0, or -1 on a NULL required argument.
 */
int oracle_scan_fwd(int batch, int dim, int seqlen, int dstate,
                    const double* u, const double* delta, const double* A,
                    const double* B, const double* C, const double* Dskip,
                    const double* z, const double* dt_bias, int delta_softplus, int zoh,
                    const double* h0, double* out, double* ypre, double* hL,
                    const int64_t* chans, int64_t nchan, int nthreads) {
  if (!u || !delta || !A || !B || !C || !out) return -1;
  const int64_t nall = (int64_t)batch * dim;
  const int64_t ncomp = chans ? nchan : nall;
  const int nt = nthreads_or_default(nthreads);
  int err = 0;
#pragma omp parallel num_threads(nt)
  {
    double* h = (double*)malloc(sizeof(double) * (size_t)(dstate > 0 ? dstate : 1));
    if (!h) {
#pragma omp atomic write
      err = -2;
    }
#pragma omp for schedule(dynamic, 1)
    for (int64_t k = 0; k < ncomp; ++k) {
      if (!h) continue;
      const int64_t ch = chans ? chans[k] : k;
      const int b = (int)(ch / dim), d = (int)(ch % dim);
      const double* uc = u + ch * seqlen;
      const double* dc = delta + ch * seqlen;
      const double* zc = z ? z + ch * seqlen : NULL;
      const double* Bb = B + (int64_t)b * dstate * seqlen;
      const double* Cb = C + (int64_t)b * dstate * seqlen;
      const double bias = dt_bias ? dt_bias[d] : 0.0;
      const double skip = Dskip ? Dskip[d] : 0.0;
      for (int n = 0; n < dstate; ++n) h[n] = h0 ? h0[ch * dstate + n] : 0.0;
      for (int t = 0; t < seqlen; ++t) {
        const double dt = step_size(dc[t], bias, delta_softplus);
        const double x = uc[t];
        double y = 0.0;
        for (int n = 0; n < dstate; ++n) {
          const double a_dn = A[(int64_t)d * dstate + n];
          const double abar = exp(dt * a_dn);                        /* Ā = exp(ΔA) */
          const double bx = input_coef(dt, a_dn, zoh) * Bb[(int64_t)n * seqlen + t] * x;
          h[n] = abar * h[n] + bx;                                   /* h_t = Ā h_{t-1} + B̄ x_t */
          y += Cb[(int64_t)n * seqlen + t] * h[n];                   /* y_t = C_t . h_t */
        }
        y += skip * x;                                               /* + D x_t */
        if (ypre) ypre[ch * seqlen + t] = y;
        out[ch * seqlen + t] = zc ? y * zc[t] * sp_sigmoid(zc[t]) : y; /* * silu(z_t) */
      }
      if (hL)
        for (int n = 0; n < dstate; ++n) hL[ch * dstate + n] = h[n];
    }
    free(h);
  }
  return err;
}

/*
 * Backward pass of the forward scan above, by the chain rule through the same recurrence run
 * in reverse time.  Written for the Euler input term (c = Δ); with zoh=1 the coefficient is
 * c_n = (e^{ΔA_n} - 1)/A_n and the terms below take c_n, dc/dΔ and dc/dA in place of Δ, 1, 0.  The pages state only that the backward pass
 * recomputes the intermediate states instead of storing them; the oracle simply keeps
 * the whole per-channel state history in host memory.
 *
 *   g_t      = dout_t * silu(z_t)                    (dL/dy_t)
 *   λ_t      = g_t C_t + Ā_{t+1} λ_{t+1},  λ_{L-1} = g_{L-1} C_{L-1} + dhL
 *   dC_t    += g_t h_t            dB_t += λ_t Δ_t x_t          (summed over channels d)
 *   du_t     = g_t D + Σ_n λ_t c_n B_t              (c_n = Δ_t for the Euler term)
 *   dΔ_t     = Σ_n λ_t (A Ā_t h_{t-1} + dc/dΔ B_t x_t)
 *   ddelta_t = dΔ_t * sigmoid(delta_t + dt_bias)  (softplus' ; 1 without softplus)
 *   dA      += λ_t (Δ_t Ā_t h_{t-1} + dc/dA B_t x_t)     dD += g_t x_t     ddt_bias += ddelta_t
 *   dz_t     = dout_t y_t silu'(z_t)   dh0 = Ā_0 λ_0
 *
 * Gradients dB, dC, dA, dD, ddt_bias are ACCUMULATED (+=) into the given arrays, which the
 * caller zeroes; per-channel outputs (du, ddelta, dz, dh0) are overwritten.  chans as in
 * the forward pass: with a channel subset, the summed gradients hold the subset's share.
 */
int oracle_scan_bwd(int batch, int dim, int seqlen, int dstate,
                    const double* u, const double* delta, const double* A,
                    const double* B, const double* C, const double* Dskip,
                    const double* z, const double* dt_bias, int delta_softplus, int zoh,
                    const double* h0, const double* dout, const double* dhL,
                    double* du, double* ddelta, double* dA, double* dB, double* dC,
                    double* dD, double* dz, double* ddt_bias, double* dh0,
                    const int64_t* chans, int64_t nchan, int nthreads) {
  if (!u || !delta || !A || !B || !C || !dout) return -1;
  const int64_t nall = (int64_t)batch * dim;
  const int64_t ncomp = chans ? nchan : nall;
  const int nt = nthreads_or_default(nthreads);
  const size_t nbc = (size_t)batch * dstate * seqlen;
  const size_t nda = (size_t)dim * dstate;
  int err = 0;
#pragma omp parallel num_threads(nt)
  {
    /* per-thread history and accumulators, summed into the outputs at the end */
    double* hist = (double*)malloc(sizeof(double) * (size_t)(seqlen + 1) * dstate);
    double* dts = (double*)malloc(sizeof(double) * (size_t)seqlen);
    double* lam = (double*)malloc(sizeof(double) * (size_t)dstate);
    double* accB = (double*)calloc(nbc, sizeof(double));
    double* accC = (double*)calloc(nbc, sizeof(double));
    double* accA = (double*)calloc(nda, sizeof(double));
    double* accD = (double*)calloc((size_t)dim, sizeof(double));
    double* accT = (double*)calloc((size_t)dim, sizeof(double));
    const int ok = hist && dts && lam && accB && accC && accA && accD && accT;
    if (!ok) {
#pragma omp atomic write
      err = -2;
    }
#pragma omp for schedule(dynamic, 1)
    for (int64_t k = 0; k < ncomp; ++k) {
      if (!ok) continue;
      const int64_t ch = chans ? chans[k] : k;
      const int b = (int)(ch / dim), d = (int)(ch % dim);
      const double* uc = u + ch * seqlen;
      const double* dc = delta + ch * seqlen;
      const double* zc = z ? z + ch * seqlen : NULL;
      const double* gc = dout + ch * seqlen;
      const double* Bb = B + (int64_t)b * dstate * seqlen;
      const double* Cb = C + (int64_t)b * dstate * seqlen;
      const double* Ad = A + (int64_t)d * dstate;
      const double bias = dt_bias ? dt_bias[d] : 0.0;
      const double skip = Dskip ? Dskip[d] : 0.0;
      /* forward: hist[(t+1)*N + n] = h_t, hist[0..N) = h_{-1} */
      for (int n = 0; n < dstate; ++n) hist[n] = h0 ? h0[ch * dstate + n] : 0.0;
      for (int t = 0; t < seqlen; ++t) {
        const double dt = step_size(dc[t], bias, delta_softplus);
        dts[t] = dt;
        for (int n = 0; n < dstate; ++n) {
          const double hp = hist[(size_t)t * dstate + n];
          hist[(size_t)(t + 1) * dstate + n] =
              exp(dt * Ad[n]) * hp + input_coef(dt, Ad[n], zoh) * Bb[(int64_t)n * seqlen + t] * uc[t];
        }
      }
      /* reverse */
      for (int n = 0; n < dstate; ++n) lam[n] = dhL ? dhL[ch * dstate + n] : 0.0;
      for (int t = seqlen - 1; t >= 0; --t) {
        const double dt = dts[t];
        const double x = uc[t];
        const double* ht = hist + (size_t)(t + 1) * dstate;
        const double* hp = hist + (size_t)t * dstate;
        double y = skip * x;
        for (int n = 0; n < dstate; ++n) y += Cb[(int64_t)n * seqlen + t] * ht[n];
        double g = gc[t];
        if (zc) {
          const double s = sp_sigmoid(zc[t]);
          g = gc[t] * zc[t] * s;
          if (dz) dz[ch * seqlen + t] = gc[t] * y * s * (1.0 + zc[t] * (1.0 - s));
        } else if (dz) {
          dz[ch * seqlen + t] = 0.0;
        }
        double s1 = 0.0, s2 = 0.0, s3 = 0.0;
        for (int n = 0; n < dstate; ++n) {
          const double Bt = Bb[(int64_t)n * seqlen + t];
          const double Ct = Cb[(int64_t)n * seqlen + t];
          const double abar = exp(dt * Ad[n]);
          const double c = input_coef(dt, Ad[n], zoh);
          double c_dt, c_da;
          input_coef_grad(dt, Ad[n], zoh, &c_dt, &c_da);
          lam[n] += g * Ct;                                /* λ_t complete */
          const double q = abar * hp[n];                   /* Ā_t h_{t-1} */
          accB[(size_t)b * dstate * seqlen + (size_t)n * seqlen + t] += lam[n] * c * x;
          accC[(size_t)b * dstate * seqlen + (size_t)n * seqlen + t] += g * ht[n];
          accA[(size_t)d * dstate + n] += lam[n] * (dt * q + c_da * Bt * x);
          s1 += lam[n] * c * Bt;
          s2 += lam[n] * Ad[n] * q;
          s3 += lam[n] * c_dt * Bt;
          lam[n] *= abar;                                  /* becomes Ā_t λ_t for step t-1 */
        }
        if (du) du[ch * seqlen + t] = g * skip + s1;
        const double ddt = x * s3 + s2;
        const double ddl = delta_softplus ? ddt * sp_sigmoid(dc[t] + bias) : ddt;
        if (ddelta) ddelta[ch * seqlen + t] = ddl;
        accD[d] += g * x;
        accT[d] += ddl;
      }
      if (dh0)
        for (int n = 0; n < dstate; ++n) dh0[ch * dstate + n] = lam[n];
    }
#pragma omp critical
    {
      if (ok) {
        if (dB) for (size_t i = 0; i < nbc; ++i) dB[i] += accB[i];
        if (dC) for (size_t i = 0; i < nbc; ++i) dC[i] += accC[i];
        if (dA) for (size_t i = 0; i < nda; ++i) dA[i] += accA[i];
        if (dD) for (int i = 0; i < dim; ++i) dD[i] += accD[i];
        if (ddt_bias) for (int i = 0; i < dim; ++i) ddt_bias[i] += accT[i];
      }
    }
    free(hist); free(dts); free(lam); free(accB); free(accC); free(accA); free(accD); free(accT);
  }
  return err;
}

/*
 * One-token recurrent (decode) step, in place on state [batch][dim][dstate]
 * (Sorular: generation keeps only a fixed D x N state per layer, no KV cache; the
 * recurrent mode processes one time step per call).  x, dt, z, out: [batch][dim];
 * B, C: [batch][dstate].  Same arithmetic as one step of oracle_scan_fwd.
 */
int oracle_state_update(int batch, int dim, int dstate, double* state,
                        const double* x, const double* dt_raw, const double* A,
                        const double* B, const double* C, const double* Dskip,
                        const double* z, const double* dt_bias, int delta_softplus, int zoh,
                        double* out, int nthreads) {
  if (!state || !x || !dt_raw || !A || !B || !C || !out) return -1;
  const int64_t nall = (int64_t)batch * dim;
  const int nt = nthreads_or_default(nthreads);
#pragma omp parallel for num_threads(nt) schedule(static)
  for (int64_t ch = 0; ch < nall; ++ch) {
    const int b = (int)(ch / dim), d = (int)(ch % dim);
    const double dt = step_size(dt_raw[ch], dt_bias ? dt_bias[d] : 0.0, delta_softplus);
    double y = 0.0;
    for (int n = 0; n < dstate; ++n) {
      double* h = state + ch * dstate + n;
      const double a_dn = A[(int64_t)d * dstate + n];
      *h = exp(dt * a_dn) * (*h) + input_coef(dt, a_dn, zoh) * B[(int64_t)b * dstate + n] * x[ch];
      y += C[(int64_t)b * dstate + n] * (*h);
    }
    y += (Dskip ? Dskip[d] : 0.0) * x[ch];
    out[ch] = z ? y * z[ch] * sp_sigmoid(z[ch]) : y;
  }
  return 0;
}
