/*
 * ssm_oracle.c -- fp64 CPU oracle for the selective scan, the SS2D
 * four-direction scan and the one-token state update.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file: only tests/, __graft_entry__.smoke() and the cpu_baseline /
 * reference legs of bench.py use it.  It shares no code, header, table or
 * helper with the CUDA library; both sides only receive the same seeded
 * inputs.
 *
 * Everything is the plain definition of the method, written out in double
 * precision, with no blocking, fusion or reordering:
 *
 *   [Minimal-scan]  "PyTorch新手也能懂：手把手拆解Mamba-minimal中的selective_scan实现"
 *                   (mhpn.cn), §2 parameter table, §3 discretisation
 *                   (§3.1 ZOH for A, §3.2 Euler for B), §4 core loop,
 *                   §5 output + D skip, §7 softplus for delta.
 *   [Mamba-step]    "代码连连看——mamba" (jiafeimiao.top), the Mamba.step()
 *                   listing, "SSM step" branch without selective_state_update:
 *                   softplus(dt + dt_proj.bias), dA = exp(dt A), dB = dt B,
 *                   state = state dA + x dB, y = state.C + D x, y * act(z).
 *   [VMamba-206]    "关于代码SS2D中的d_state设置" (VMamba issue 206):
 *                   CrossScan / CrossMerge only arrange the sequence.
 *
 * Readings where the pages are silent:
 *   - softplus is torch's F.softplus: x for x > 20, log1p(exp(x)) otherwise.
 *   - dt_bias is added before the softplus, whether or not softplus is on.
 *   - y uses the state AFTER the update of the same step ([Minimal-scan] §4:
 *     update, then contract with C).
 *   - the gate act(z) is SiLU: z / (1 + exp(-z)).
 *   - absent D / z / dt_bias mean D = 0, no gate, bias = 0.
 *   - SS2D directions: k0 row-major (l = h W + w), k1 column-major
 *     (l = w H + h), k2 = k0 reversed, k3 = k1 reversed ("cross"); the snake
 *     variant flips every odd row of k0 and odd column of k1; delta/B/C of
 *     direction k are given in that direction's scan order; A, D, dt_bias
 *     rows of direction k are k*d_in .. k*d_in + d_in - 1; the merge is the
 *     plain sum over the four directions at each pixel.
 *
 * Layouts (row-major, contiguous):
 *   u, delta, z, y : (b, L, d_in)        A : (d_in, N)
 *   B, C           : (b, L, N)           D, dt_bias : (d_in)
 *   h0, h_last     : (b, d_in, N)
 * Parity unpinned: nothing in this file (every function has pins in
 * tests/test_oracle_pins.py).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* torch.nn.functional.softplus with its defaults (beta 1, threshold 20). */
static double oracle_softplus(double x)
{
    if (x > 20.0)
        return x;
    return log1p(exp(x));
}

/* SiLU, the activation of the Mamba block's gate branch. */
static double oracle_silu(double z)
{
    return z / (1.0 + exp(-z));
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/*
 * Selective scan, [Minimal-scan] §2-§5 plus the gate of [Mamba-step].
 * For every (batch, channel): x (the state) starts at h0 (or 0), then for
 * i = 0..L-1:  deltaA = exp(delta A), deltaB_u = delta B u,
 * x = deltaA * x + deltaB_u, y = sum_n x[n] C[n];  then y = y + u D and
 * y = y * silu(z).  The last state goes to h_last when it is given.
 */
void oracle_selective_scan(const double *u, const double *delta,
                           const double *A, const double *B, const double *C,
                           const double *D, const double *z,
                           const double *dt_bias, int delta_softplus,
                           const double *h0, double *h_last, double *y,
                           int64_t b, int64_t L, int64_t d_in, int64_t N)
{
    int64_t bd;
#pragma omp parallel for schedule(dynamic, 4)
    for (bd = 0; bd < b * d_in; ++bd) {
        const int64_t ib = bd / d_in;
        const int64_t d = bd % d_in;
        double *x = (double *)malloc((size_t)(N > 0 ? N : 1) * sizeof(double));
        for (int64_t n = 0; n < N; ++n)
            x[n] = h0 ? h0[(ib * d_in + d) * N + n] : 0.0;

        for (int64_t i = 0; i < L; ++i) {
            const int64_t row = ib * L + i;
            double dt = delta[row * d_in + d];
            if (dt_bias)
                dt += dt_bias[d];
            if (delta_softplus)
                dt = oracle_softplus(dt);
            const double ui = u[row * d_in + d];

            /* §3.1: deltaA = exp(delta * A)   §3.2: deltaB_u = delta * B * u
             * §4:   x = deltaA * x + deltaB_u                              */
            for (int64_t n = 0; n < N; ++n) {
                const double deltaA = exp(dt * A[d * N + n]);
                const double deltaB_u = dt * B[row * N + n] * ui;
                x[n] = deltaA * x[n] + deltaB_u;
            }
            /* §4: y = einsum(x, C[:, i, :], 'b d n, b n -> b d') */
            double yi = 0.0;
            for (int64_t n = 0; n < N; ++n)
                yi += x[n] * C[row * N + n];
            /* §5: y = y + u * D */
            if (D)
                yi += ui * D[d];
            /* [Mamba-step]: y = y * act(z) */
            if (z)
                yi *= oracle_silu(z[row * d_in + d]);
            y[row * d_in + d] = yi;
        }
        if (h_last)
            for (int64_t n = 0; n < N; ++n)
                h_last[(ib * d_in + d) * N + n] = x[n];
        free(x);
    }
}

/*
 * One-token state update, [Mamba-step] "SSM step":
 *   dt = softplus(dt + dt_bias);  dA = exp(einsum('bd,dn->bdn', dt, A));
 *   dB = einsum('bd,bn->bdn', dt, B);  state = state * dA + x * dB;
 *   y = einsum('bdn,bn->bd', state, C) + D * x;  y = y * act(z).
 * state (b, d_in, N) is updated in place; x, dt, z, y are (b, d_in);
 * B, C are (b, N).
 */
void oracle_state_update(double *state, const double *x, const double *dt,
                         const double *A, const double *B, const double *C,
                         const double *D, const double *z,
                         const double *dt_bias, int dt_softplus, double *y,
                         int64_t b, int64_t d_in, int64_t N)
{
    int64_t bd;
#pragma omp parallel for schedule(static)
    for (bd = 0; bd < b * d_in; ++bd) {
        const int64_t ib = bd / d_in;
        const int64_t d = bd % d_in;
        double delta = dt[bd];
        if (dt_bias)
            delta += dt_bias[d];
        if (dt_softplus)
            delta = oracle_softplus(delta);
        double yi = 0.0;
        for (int64_t n = 0; n < N; ++n) {
            const double dA = exp(delta * A[d * N + n]);
            const double dB = delta * B[ib * N + n];
            double *s = &state[bd * N + n];
            *s = *s * dA + x[bd] * dB;
            yi += *s * C[ib * N + n];
        }
        if (D)
            yi += D[d] * x[bd];
        if (z)
            yi *= oracle_silu(z[bd]);
        y[bd] = yi;
    }
}

/*
 * Causal-conv1d decode step, [Mamba-step] "Conv step" without
 * causal_conv1d_update: conv_state = roll(conv_state, -1) along the window,
 * conv_state[..., -1] = x, x = sum(conv_state * weight, -1) + bias,
 * x = act(x) with act = SiLU.  conv_state (b, d_in, d_conv) is updated in
 * place; x, x_out are (b, d_in); weight is (d_in, d_conv); bias (d_in) is
 * nullable.
 */
void oracle_conv_step(double *conv_state, const double *x, const double *weight,
                      const double *bias, double *x_out, int64_t b, int64_t d_in,
                      int64_t d_conv)
{
    int64_t bd;
#pragma omp parallel for schedule(static)
    for (bd = 0; bd < b * d_in; ++bd) {
        const int64_t d = bd % d_in;
        double *cs = &conv_state[bd * d_conv];
        for (int64_t j = 0; j + 1 < d_conv; ++j)  /* roll left by one */
            cs[j] = cs[j + 1];
        cs[d_conv - 1] = x[bd];
        double acc = bias ? bias[d] : 0.0;
        for (int64_t j = 0; j < d_conv; ++j)
            acc += cs[j] * weight[d * d_conv + j];
        x_out[bd] = oracle_silu(acc);
    }
}

/*
 * Pixel visited at step l of scan direction k on an H x W grid (pixels are
 * numbered row-major, p = h W + w).  [VMamba-206]: four orders, row-major,
 * column-major and both reversed (order 0, "cross"); the snake scan the
 * issue mentions (order 1) walks odd rows right to left and odd columns
 * bottom to top, so consecutive steps stay neighbours.
 */
static int64_t oracle_ss2d_pixel(int k, int order, int64_t l, int64_t H, int64_t W)
{
    const int64_t L = H * W;
    if (k >= 2)
        l = L - 1 - l;               /* k2, k3: the reverse of k0, k1 */
    if (k == 0 || k == 2) {
        const int64_t h = l / W;     /* row-major: l = h W + w */
        int64_t w = l % W;
        if (order == 1 && h % 2 == 1)
            w = W - 1 - w;
        return h * W + w;
    }
    {
        int64_t h = l % H;           /* column-major: l = w H + h */
        const int64_t w = l / H;
        if (order == 1 && w % 2 == 1)
            h = H - 1 - h;
        return h * W + w;
    }
}

/* CrossScan: xs[b, k, l, d] = u[b, pixel_k(l), d]. */
void oracle_cross_scan(const double *u, double *xs, int64_t b, int64_t H,
                       int64_t W, int64_t d_in, int order)
{
    const int64_t L = H * W;
    for (int64_t ib = 0; ib < b; ++ib)
        for (int k = 0; k < 4; ++k)
            for (int64_t l = 0; l < L; ++l) {
                const int64_t p = oracle_ss2d_pixel(k, order, l, H, W);
                for (int64_t d = 0; d < d_in; ++d)
                    xs[((ib * 4 + k) * L + l) * d_in + d] =
                        u[(ib * L + p) * d_in + d];
            }
}

/* CrossMerge: y[b, pixel_k(l), d] = sum over k of ys[b, k, l, d]. */
void oracle_cross_merge(const double *ys, double *y, int64_t b, int64_t H,
                        int64_t W, int64_t d_in, int order)
{
    const int64_t L = H * W;
    memset(y, 0, (size_t)(b * L * d_in) * sizeof(double));
    for (int64_t ib = 0; ib < b; ++ib)
        for (int k = 0; k < 4; ++k)
            for (int64_t l = 0; l < L; ++l) {
                const int64_t p = oracle_ss2d_pixel(k, order, l, H, W);
                for (int64_t d = 0; d < d_in; ++d)
                    y[(ib * L + p) * d_in + d] +=
                        ys[((ib * 4 + k) * L + l) * d_in + d];
            }
}

/*
 * SS2D forward: CrossScan, a selective scan per (batch, direction) with the
 * direction's own A/D/dt_bias rows and its own delta/B/C, then CrossMerge.
 *   u, y        : (b, H W, d_in)
 *   delta       : (b, 4, H W, d_in), scan order of each direction
 *   B, C        : (b, 4, H W, N)
 *   A           : (4 d_in, N);  D, dt_bias : (4 d_in), nullable
 * Returns 0, or -1 when the temporaries cannot be allocated.
 */
int oracle_ss2d_scan(const double *u, const double *delta, const double *A,
                     const double *B, const double *C, const double *D,
                     const double *dt_bias, int delta_softplus, double *y,
                     int64_t b, int64_t H, int64_t W, int64_t d_in, int64_t N,
                     int order)
{
    const int64_t L = H * W;
    const size_t n_xs = (size_t)(b * 4 * L * d_in);
    double *xs = (double *)malloc(n_xs * sizeof(double));
    double *ys = (double *)malloc(n_xs * sizeof(double));
    if (!xs || !ys) {
        free(xs);
        free(ys);
        return -1;
    }
    oracle_cross_scan(u, xs, b, H, W, d_in, order);
    for (int64_t ib = 0; ib < b; ++ib)
        for (int k = 0; k < 4; ++k) {
            const int64_t seq = ib * 4 + k;
            oracle_selective_scan(xs + seq * L * d_in, delta + seq * L * d_in,
                                  A + (int64_t)k * d_in * N,
                                  B + seq * L * N, C + seq * L * N,
                                  D ? D + (int64_t)k * d_in : NULL, NULL,
                                  dt_bias ? dt_bias + (int64_t)k * d_in : NULL,
                                  delta_softplus, NULL, NULL,
                                  ys + seq * L * d_in, 1, L, d_in, N);
        }
    oracle_cross_merge(ys, y, b, H, W, d_in, order);
    free(xs);
    free(ys);
    return 0;
}

/* Derivative of oracle_softplus: the logistic sigmoid below the threshold,
 * 1 above it (the linear branch). */
static double oracle_softplus_grad(double x)
{
    if (x > 20.0)
        return 1.0;
    return 1.0 / (1.0 + exp(-x));
}

/*
 * Backward of oracle_selective_scan: the gradients of
 *     loss = sum_{i,t,d} dout[i,t,d] y[i,t,d] + sum_{i,d,n} dh_last[i,d,n] h_last[i,d,n]
 * with respect to every input, by the chain rule applied to the forward
 * recurrence above ([Minimal-scan] §3-§5 with the gate of [Mamba-step]),
 * walked backwards in time.  "Fast backward" is what the VMamba discussion
 * ([VMamba-206]) asks of a scan kernel; the gradient itself is the plain
 * definition.  For one (batch, channel), with delta_t the softplus'd step,
 * a_t[n] = exp(delta_t A[n]) and h_t the state after step t (h_{-1} = h0):
 *
 *   forward:   h_t = a_t h_{t-1} + delta_t B_t u_t,   yp_t = C_t.h_t + D u_t,
 *              y_t = yp_t silu(z_t)
 *   backward:  g_t = dout_t silu(z_t),   dz_t = dout_t yp_t silu'(z_t)
 *              lam <- lam + g_t C_t                 (lam = d loss / d h_t)
 *              dC_t += g_t h_t,  dD += g_t u_t,  du_t = g_t D
 *              ddelta_t = sum_n lam (A a_t h_{t-1} + B_t u_t)
 *              dA += lam delta_t a_t h_{t-1},  dB_t += lam delta_t u_t,
 *              du_t += sum_n lam delta_t B_t
 *              lam <- lam a_t                       (now d loss / d h_{t-1})
 *   and at the end dh0 = lam.  The gradient of the raw delta input is
 *   ddelta_t softplus'(delta + dt_bias) (or ddelta_t without softplus), and
 *   ddt_bias is its sum over batch and time.
 *
 * dB, dC sum over the channels; dA, dD, ddt_bias over batch (and time).
 * Outputs dz, dD, ddt_bias, dh0 may be NULL (not computed); dz is only
 * written when z is given.  dh_last may be NULL (zero).  Batches run in
 * parallel; the sums over batch are taken afterwards in batch order.
 * Returns 0, or -1 when scratch memory could not be allocated.
 */
int oracle_selective_scan_bwd(const double *u, const double *delta,
                              const double *A, const double *B, const double *C,
                              const double *D, const double *z,
                              const double *dt_bias, int delta_softplus,
                              const double *h0, const double *dout,
                              const double *dh_last,
                              double *du, double *ddelta, double *dA,
                              double *dB, double *dC, double *dD, double *dz,
                              double *ddt_bias, double *dh0,
                              int64_t b, int64_t L, int64_t d_in, int64_t N)
{
    /* per-batch partial sums of the per-channel gradients */
    double *pA = (double *)calloc((size_t)(b * d_in * N + 1), sizeof(double));
    double *pD = (double *)calloc((size_t)(b * d_in + 1), sizeof(double));
    double *pbias = (double *)calloc((size_t)(b * d_in + 1), sizeof(double));
    int failed = !pA || !pD || !pbias;
    if (!failed) {
        memset(dB, 0, (size_t)(b * L * N) * sizeof(double));
        memset(dC, 0, (size_t)(b * L * N) * sizeof(double));
    }

    int64_t ib;
#pragma omp parallel for schedule(dynamic, 1) reduction(|| : failed)
    for (ib = 0; ib < b; ++ib) {
        if (failed)
            continue;
        /* states after every step, plus h0 in front: hs[(t + 1) N + n] */
        double *hs = (double *)malloc((size_t)((L + 1) * N + 1) * sizeof(double));
        double *dts = (double *)malloc((size_t)(L + 1) * sizeof(double));
        double *pre = (double *)malloc((size_t)(L + 1) * sizeof(double));
        double *yp = (double *)malloc((size_t)(L + 1) * sizeof(double));
        double *lam = (double *)malloc((size_t)(N + 1) * sizeof(double));
        if (!hs || !dts || !pre || !yp || !lam) {
            failed = 1;
            free(hs); free(dts); free(pre); free(yp); free(lam);
            continue;
        }
        for (int64_t d = 0; d < d_in; ++d) {
            const int64_t bd = ib * d_in + d;
            /* forward, keeping what the backward needs */
            for (int64_t n = 0; n < N; ++n)
                hs[n] = h0 ? h0[bd * N + n] : 0.0;
            for (int64_t t = 0; t < L; ++t) {
                const int64_t row = ib * L + t;
                double x = delta[row * d_in + d];
                if (dt_bias)
                    x += dt_bias[d];
                pre[t] = x;
                dts[t] = delta_softplus ? oracle_softplus(x) : x;
                const double ut = u[row * d_in + d];
                double acc = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    const double a = exp(dts[t] * A[d * N + n]);
                    hs[(t + 1) * N + n] = a * hs[t * N + n] + dts[t] * B[row * N + n] * ut;
                    acc += hs[(t + 1) * N + n] * C[row * N + n];
                }
                if (D)
                    acc += ut * D[d];
                yp[t] = acc;
            }
            /* backward in time */
            for (int64_t n = 0; n < N; ++n)
                lam[n] = dh_last ? dh_last[bd * N + n] : 0.0;
            for (int64_t t = L - 1; t >= 0; --t) {
                const int64_t row = ib * L + t;
                const int64_t at = row * d_in + d;
                const double ut = u[at];
                double g = dout[at];
                if (z) {
                    const double zt = z[at];
                    const double s = 1.0 / (1.0 + exp(-zt));
                    if (dz)
                        dz[at] = g * yp[t] * s * (1.0 + zt * (1.0 - s));
                    g *= zt * s;
                }
                pD[bd] += g * ut;          /* defined at D = 0 when D is absent */
                double dut = D ? g * D[d] : 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    lam[n] += g * C[row * N + n];
                    dC[row * N + n] += g * hs[(t + 1) * N + n];
                }
                double ddt = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    const double a = exp(dts[t] * A[d * N + n]);
                    const double hprev = hs[t * N + n];
                    ddt += lam[n] * (A[d * N + n] * a * hprev + B[row * N + n] * ut);
                    pA[bd * N + n] += lam[n] * dts[t] * a * hprev;
                    dB[row * N + n] += lam[n] * dts[t] * ut;
                    dut += lam[n] * dts[t] * B[row * N + n];
                    lam[n] *= a;
                }
                if (delta_softplus)
                    ddt *= oracle_softplus_grad(pre[t]);
                du[at] = dut;
                ddelta[at] = ddt;
                pbias[bd] += ddt;
            }
            if (dh0)
                for (int64_t n = 0; n < N; ++n)
                    dh0[bd * N + n] = lam[n];
        }
        free(hs); free(dts); free(pre); free(yp); free(lam);
    }
    if (!failed) {
        for (int64_t d = 0; d < d_in; ++d) {
            for (int64_t n = 0; n < N; ++n) {
                double s = 0.0;
                for (int64_t i = 0; i < b; ++i)
                    s += pA[(i * d_in + d) * N + n];
                dA[d * N + n] = s;
            }
            double sD = 0.0, sb = 0.0;
            for (int64_t i = 0; i < b; ++i) {
                sD += pD[i * d_in + d];
                sb += pbias[i * d_in + d];
            }
            if (dD)
                dD[d] = sD;
            if (ddt_bias)
                ddt_bias[d] = sb;
        }
    }
    free(pA); free(pD); free(pbias);
    return failed ? -1 : 0;
}
