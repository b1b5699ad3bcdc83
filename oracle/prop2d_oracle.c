/*
 * Prop2D CPU oracle: plain, single-threaded, fp64.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the correctness reference that the
 * CUDA library is checked against.  Only the test suite, the package's
 * smoke check and the CPU-baseline leg of the benchmark may load it.  It
 * shares no code, header, table or constant with the CUDA path.
 *
 * What it computes (paper: "Scaling Parallel Sequence Models to
 * Foundation-Scale Vision Encoders", Sec. 3 "Line-scan recurrence" and the
 * papernotes.org summary of the method, "背景算子" paragraph, Eq. 2/3):
 *
 *   For each batch b, latent channel c and direction d in
 *   {top->bottom, bottom->top, left->right, right->left}, the grid is swept
 *   one line at a time.  Every position q of line l is updated in parallel
 *   from the three positions q-1, q, q+1 of the previous line:
 *
 *       h_l(q) = sum_k w_l(q,k) * h_{l-1}(q+k-1) + lambda_l(q) * x_l(q),
 *       h_{-1} = 0,
 *
 *   and the output is the gated sum over the directions that are enabled,
 *
 *       y = sum_d u_d (.) h_d                   (papernotes.org, Eq. y_c =
 *                                                 Prop2D(x_c; u, lambda, w)).
 *
 *   The tridiagonal weights are row-stochastic (Sec. 3 "Stability and
 *   connectivity"; papernotes.org normalisation formula):
 *
 *       s_k = sigmoid(wt_k)   for every slot k whose neighbour is on the grid,
 *       S   = max(sum_k s_k, eps),                      (Sec. 5.1 "Fused CUDA
 *       w_k = s_k / S.                                    normalization":
 *                                                         sigmoid, local sum,
 *                                                         clamp, divide)
 *
 * Readings taken where the pages are silent (the equation bodies of Sec. 3
 * were lost from the page text):
 *   - no skip term, h_{-1} = 0;
 *   - off-grid neighbour slots get weight 0 and are left out of the sum;
 *   - the clamp acts on the denominator, eps = 1e-6;
 *   - lambda, u and the logits are separate per direction;
 *   - slot k names the absolute orthogonal offset k-1 (-1 = up / left);
 *   - with share_w the logit field has one channel, used by every channel.
 *
 * Layouts (all contiguous, row-major):
 *   x      [B][Cc][H][W]
 *   lambda [B][4][Cc][H][W]
 *   u      [B][4][Cc][H][W]
 *   wlogit [B][4][Cw][3][H][W],   Cw = share_w ? 1 : Cc
 *   out    [B][Cc][H][W]
 * Direction slot order: 0 top->bottom, 1 bottom->top, 2 left->right,
 * 3 right->left; bit d of `dirs` enables slot d.
 *
 * Return value: 0 on success, 1 on a bad argument (nothing written).
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_EPS 1e-6

static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

/* Index of element (i, j) of plane `plane` in a [..][H][W] tensor. */
static size_t at(size_t plane, int H, int W, int i, int j) {
    return (plane * (size_t)H + (size_t)i) * (size_t)W + (size_t)j;
}

/* Row-stochastic weights of one position, following the normalisation
 * formula: sigmoid of each on-grid slot, local sum, clamp, divide.
 * `lg[k]` are the three logits, `valid[k]` says whether slot k's neighbour
 * lies on the grid. */
static void normalise(const double lg[3], const int valid[3], double w[3]) {
    double s[3];
    double sum = 0.0;
    for (int k = 0; k < 3; ++k) {
        s[k] = valid[k] ? sigmoid(lg[k]) : 0.0;
        sum += s[k];
    }
    double denom = sum > ORACLE_EPS ? sum : ORACLE_EPS;
    for (int k = 0; k < 3; ++k) w[k] = s[k] / denom;
}

/* Grid position (i, j) of line `line`, position `q` along it, for direction d. */
static void position(int d, int line, int q, int *i, int *j) {
    if (d < 2) { *i = line; *j = q; }      /* row lines: top->bottom / bottom->top */
    else       { *i = q;    *j = line; }   /* column lines: left->right / right->left */
}

int oracle_prop2d_weights_f64(const double *wlogit, int B, int Cc, int H, int W,
                              int share_w, double *w_out) {
    if (!wlogit || !w_out || B < 0 || Cc < 0 || H < 0 || W < 0) return 1;
    int Cw = share_w ? 1 : Cc;
    for (int b = 0; b < B; ++b)
        for (int d = 0; d < 4; ++d)
            for (int c = 0; c < Cw; ++c) {
                size_t base = ((size_t)(b * 4 + d) * (size_t)Cw + (size_t)c) * 3;
                for (int i = 0; i < H; ++i)
                    for (int j = 0; j < W; ++j) {
                        /* the orthogonal coordinate is j for row lines, i for column lines */
                        int q = d < 2 ? j : i;
                        int M = d < 2 ? W : H;
                        double lg[3], w[3];
                        int valid[3];
                        for (int k = 0; k < 3; ++k) {
                            valid[k] = (q + k - 1 >= 0) && (q + k - 1 < M);
                            lg[k] = valid[k] ? wlogit[at(base + k, H, W, i, j)] : 0.0;
                        }
                        normalise(lg, valid, w);
                        for (int k = 0; k < 3; ++k) w_out[at(base + k, H, W, i, j)] = w[k];
                    }
            }
    return 0;
}

int oracle_prop2d_f64(const double *x, const double *lambda, const double *wlogit,
                      const double *u, int B, int Cc, int H, int W, int dirs,
                      int share_w, double *out) {
    if (!x || !lambda || !wlogit || !u || !out) return 1;
    if (B < 0 || Cc < 0 || H < 0 || W < 0) return 1;
    if (dirs < 1 || dirs > 15) return 1;
    int Cw = share_w ? 1 : Cc;
    int maxM = H > W ? H : W;
    double *hprev = (double *)calloc((size_t)maxM + 1, sizeof(double));
    double *hcur = (double *)calloc((size_t)maxM + 1, sizeof(double));
    if (!hprev || !hcur) { free(hprev); free(hcur); return 1; }

    for (int b = 0; b < B; ++b)
        for (int c = 0; c < Cc; ++c) {
            size_t xp = (size_t)b * (size_t)Cc + (size_t)c;      /* plane of x and out */
            for (int i = 0; i < H; ++i)
                for (int j = 0; j < W; ++j) out[at(xp, H, W, i, j)] = 0.0;

            for (int d = 0; d < 4; ++d) {
                if (!(dirs & (1 << d))) continue;
                size_t gp = ((size_t)b * 4 + (size_t)d) * (size_t)Cc + (size_t)c;   /* lambda, u */
                size_t wp = (((size_t)b * 4 + (size_t)d) * (size_t)Cw +
                             (size_t)(share_w ? 0 : c)) * 3;                       /* logits */
                int L = d < 2 ? H : W;      /* number of lines swept */
                int M = d < 2 ? W : H;      /* positions per line */
                for (int q = 0; q < M; ++q) hprev[q] = 0.0;

                for (int step = 0; step < L; ++step) {
                    /* even slots sweep forward, odd slots sweep backward */
                    int line = (d % 2 == 0) ? step : L - 1 - step;
                    for (int q = 0; q < M; ++q) {
                        int i, j;
                        position(d, line, q, &i, &j);
                        double lg[3], w[3];
                        int valid[3];
                        for (int k = 0; k < 3; ++k) {
                            valid[k] = (q + k - 1 >= 0) && (q + k - 1 < M);
                            lg[k] = valid[k] ? wlogit[at(wp + k, H, W, i, j)] : 0.0;
                        }
                        normalise(lg, valid, w);
                        double acc = 0.0;
                        for (int k = 0; k < 3; ++k)
                            if (valid[k]) acc += w[k] * hprev[q + k - 1];
                        acc += lambda[at(gp, H, W, i, j)] * x[at(xp, H, W, i, j)];
                        hcur[q] = acc;
                    }
                    for (int q = 0; q < M; ++q) {
                        int i, j;
                        position(d, line, q, &i, &j);
                        out[at(xp, H, W, i, j)] += u[at(gp, H, W, i, j)] * hcur[q];
                    }
                    double *t = hprev; hprev = hcur; hcur = t;
                }
            }
        }
    free(hprev);
    free(hcur);
    return 0;
}

/*
 * Backward of Prop2D: the vector-Jacobian product of the forward above, in
 * fp64.  The pages report backward timings of their kernel (Sec. 6.1
 * "Scaling with input size, batch, and channels", Fig. 8) but print no
 * backward formulas; what follows is the plain chain rule of the forward
 * recurrence and normalisation, in reverse scan order.
 *
 * Given gy = dL/dy ([B][Cc][H][W]), for each batch b, channel c and enabled
 * direction d, with the forward lines h_l kept:
 *
 *     g_l        = u_l (.) gy_l + W_{l+1}^T g_{l+1}      (adjoint of h_l; none
 *                                                       after the last line)
 *     du_l       = gy_l (.) h_l
 *     dlambda_l  = g_l (.) x_l,      dx_l += g_l (.) lambda_l
 *     dw_l(q,k)  = g_l(q) h_{l-1}(q+k-1)                 (h_{-1} = 0)
 *
 * and through the normalisation w_k = s_k / max(sum_k s_k, eps),
 * s_k = sigmoid(wt_k), over the on-grid slots:
 *
 *     sum > eps:  ds_j = (dw_j - sum_k dw_k w_k) / sum
 *     otherwise:  ds_j = dw_j / eps          (the clamp holds the denominator)
 *     dwt_j = ds_j s_j (1 - s_j);   off-grid slots get 0.
 *
 * Readings: the derivative of max(sum, eps) is taken on the branch the
 * forward uses (sum > eps: the sum); with share_w the gradient of the one
 * logit field is the sum over the channels that use it.
 *
 * Outputs (fully written; slots of directions not in `dirs` are 0):
 *   dx [B][Cc][H][W], dlambda [B][4][Cc][H][W], dwlogit [B][4][Cw][3][H][W],
 *   du [B][4][Cc][H][W].
 * Return value: 0 on success, 1 on a bad argument.
 */
static void normalise_parts(const double lg[3], const int valid[3], double s[3], double w[3],
                            double *sum_out) {
    double total = 0.0;
    for (int k = 0; k < 3; ++k) {
        s[k] = valid[k] ? sigmoid(lg[k]) : 0.0;
        total += s[k];
    }
    normalise(lg, valid, w);
    *sum_out = total;
}

/* Position q of line `line` of direction d (M positions per line): which
 * neighbour slots are on the grid, their sigmoids, the normalised weights
 * and the local sum of the sigmoids. */
static void position_weights(const double *wlogit, size_t wplane, int H, int W, int d, int line,
                             int q, int M, int on[3], double s[3], double w[3], double *sum) {
    int i, j;
    position(d, line, q, &i, &j);
    double lg[3];
    for (int k = 0; k < 3; ++k) {
        int nb = q + k - 1;   /* neighbour position along the line */
        on[k] = nb >= 0 && nb < M;
        lg[k] = on[k] ? wlogit[at(wplane + k, H, W, i, j)] : 0.0;
    }
    normalise_parts(lg, on, s, w, sum);
}

/* The backward with the sharing of the variants: lambda, u
 * [B][gate_dirs][Cc][H][W] (gate_dirs 4, or 1 plane shared by the four
 * directions) and logits [B][4][G][3][H][W] (channel c uses field c / (Cc/G)).
 * A shared input's gradient is the sum of the gradients of its uses. */
static int prop2d_bwd_shared(const double *x, const double *lambda, const double *wlogit,
                             const double *u, const double *gy, int B, int Cc, int H, int W,
                             int dirs, int gate_dirs, int G, double *dx, double *dlambda,
                             double *dwlogit, double *du) {
    if (!x || !lambda || !wlogit || !u || !gy || !dx || !dlambda || !dwlogit || !du) return 1;
    if (B < 0 || Cc < 0 || H < 0 || W < 0) return 1;
    if (dirs < 1 || dirs > 15) return 1;
    if ((gate_dirs != 1 && gate_dirs != 4) || G < 1 || (Cc > 0 && Cc % G != 0)) return 1;
    int cpg = Cc > 0 ? Cc / G : 1;   /* channels per logit field */
    size_t HW = (size_t)H * (size_t)W;
    memset(dx, 0, (size_t)B * (size_t)Cc * HW * sizeof(double));
    memset(dlambda, 0, (size_t)B * (size_t)gate_dirs * (size_t)Cc * HW * sizeof(double));
    memset(du, 0, (size_t)B * (size_t)gate_dirs * (size_t)Cc * HW * sizeof(double));
    memset(dwlogit, 0, (size_t)B * 4 * (size_t)G * 3 * HW * sizeof(double));
    int maxM = H > W ? H : W;
    /* forward lines in scan order, the adjoint line and its carry */
    double *hist = (double *)calloc(HW + 1, sizeof(double));
    double *adj = (double *)calloc((size_t)maxM + 1, sizeof(double));
    double *carry = (double *)calloc((size_t)maxM + 1, sizeof(double));
    double *carry_next = (double *)calloc((size_t)maxM + 1, sizeof(double));
    if (!hist || !adj || !carry || !carry_next) {
        free(hist); free(adj); free(carry); free(carry_next);
        return 1;
    }

    for (int b = 0; b < B; ++b)
        for (int c = 0; c < Cc; ++c) {
            size_t xpl = (size_t)b * (size_t)Cc + (size_t)c;
            for (int d = 0; d < 4; ++d) {
                if (!(dirs & (1 << d))) continue;
                size_t gpl = ((size_t)b * (size_t)gate_dirs + (size_t)(gate_dirs == 4 ? d : 0)) *
                             (size_t)Cc + (size_t)c;
                size_t wpl = (((size_t)b * 4 + (size_t)d) * (size_t)G + (size_t)(c / cpg)) * 3;
                int L = d < 2 ? H : W;
                int M = d < 2 ? W : H;

                /* forward sweep, every line kept: hist[step * M + q] */
                for (int step = 0; step < L; ++step) {
                    int line = d % 2 ? L - 1 - step : step;   /* odd slots sweep backward */
                    const double *prev = step > 0 ? hist + (size_t)(step - 1) * M : NULL;
                    for (int q = 0; q < M; ++q) {
                        int i, j, on[3];
                        double s[3], w[3], sum;
                        position(d, line, q, &i, &j);
                        position_weights(wlogit, wpl, H, W, d, line, q, M, on, s, w, &sum);
                        double v = lambda[at(gpl, H, W, i, j)] * x[at(xpl, H, W, i, j)];
                        if (prev)
                            for (int k = 0; k < 3; ++k)
                                if (on[k]) v += w[k] * prev[q + k - 1];
                        hist[(size_t)step * M + q] = v;
                    }
                }

                /* reverse sweep of the adjoint */
                for (int q = 0; q < M; ++q) carry[q] = 0.0;
                for (int step = L - 1; step >= 0; --step) {
                    int line = d % 2 ? L - 1 - step : step;   /* odd slots sweep backward */
                    const double *hl = hist + (size_t)step * M;
                    const double *hprv = step > 0 ? hist + (size_t)(step - 1) * M : NULL;
                    for (int q = 0; q < M; ++q) {
                        int i, j;
                        position(d, line, q, &i, &j);
                        size_t e = at(gpl, H, W, i, j);
                        double gyv = gy[at(xpl, H, W, i, j)];
                        adj[q] = u[e] * gyv + carry[q];
                        du[e] += gyv * hl[q];
                        dlambda[e] += adj[q] * x[at(xpl, H, W, i, j)];
                        dx[at(xpl, H, W, i, j)] += adj[q] * lambda[e];
                        carry_next[q] = 0.0;
                    }
                    for (int q = 0; q < M; ++q) {
                        int i, j, on[3];
                        double s[3], w[3], sum;
                        position(d, line, q, &i, &j);
                        position_weights(wlogit, wpl, H, W, d, line, q, M, on, s, w, &sum);
                        double dw[3] = {0.0, 0.0, 0.0}, dot = 0.0;
                        for (int k = 0; k < 3; ++k) {
                            if (!on[k]) continue;
                            dw[k] = hprv ? adj[q] * hprv[q + k - 1] : 0.0;
                            dot += dw[k] * w[k];
                            carry_next[q + k - 1] += w[k] * adj[q];
                        }
                        for (int k = 0; k < 3; ++k) {
                            if (!on[k]) continue;
                            double ds = sum > ORACLE_EPS ? (dw[k] - dot) / sum : dw[k] / ORACLE_EPS;
                            dwlogit[at(wpl + k, H, W, i, j)] += ds * s[k] * (1.0 - s[k]);
                        }
                    }
                    double *t = carry; carry = carry_next; carry_next = t;
                }
            }
        }
    free(hist);
    free(adj);
    free(carry);
    free(carry_next);
    return 0;
}

/* Backward of Prop2D: per-direction lambda, u [B][4][Cc][H][W]; logits
 * per channel, or shared by all channels (share_w). */
int oracle_prop2d_bwd_f64(const double *x, const double *lambda, const double *wlogit,
                          const double *u, const double *gy, int B, int Cc, int H, int W,
                          int dirs, int share_w, double *dx, double *dlambda, double *dwlogit,
                          double *du) {
    return prop2d_bwd_shared(x, lambda, wlogit, u, gy, B, Cc, H, W, dirs, 4, share_w ? 1 : (Cc > 0 ? Cc : 1),
                             dx, dlambda, dwlogit, du);
}

/* Backward of the sharing variants (oracle_prop2d_ex_f64's layouts). */
int oracle_prop2d_bwd_ex_f64(const double *x, const double *lambda, const double *wlogit,
                             const double *u, const double *gy, int B, int Cc, int H, int W,
                             int dirs, int gate_dirs, int w_groups, double *dx, double *dlambda,
                             double *dwlogit, double *du) {
    return prop2d_bwd_shared(x, lambda, wlogit, u, gy, B, Cc, H, W, dirs, gate_dirs, w_groups,
                             dx, dlambda, dwlogit, du);
}

/*
 * Gate- and weight-sharing variants of the forward (the pages' "share w_i
 * across channels in all modules", Sec. 6.2 "Image classification", and the
 * channel-shared weights of Sec. 4.2, generalised):
 *
 *   gate_dirs = 4: lambda and u hold one plane per direction, [B][4][Cc][H][W];
 *   gate_dirs = 1: one lambda and one u plane serve all four directions,
 *                  [B][1][Cc][H][W];
 *   w_groups  = G (G divides Cc): the logits hold G fields per (batch,
 *                  direction), [B][4][G][3][H][W]; channel c uses field
 *                  c / (Cc / G).  G = Cc is per-channel, G = 1 is share_w.
 *
 * Everything else is the forward above.  Return value: 0 on success, 1 on a
 * bad argument.
 */
int oracle_prop2d_ex_f64(const double *x, const double *lambda, const double *wlogit,
                         const double *u, int B, int Cc, int H, int W, int dirs,
                         int gate_dirs, int w_groups, double *out) {
    if (!x || !lambda || !wlogit || !u || !out) return 1;
    if (B < 0 || Cc < 0 || H < 0 || W < 0) return 1;
    if (dirs < 1 || dirs > 15) return 1;
    if (gate_dirs != 1 && gate_dirs != 4) return 1;
    if (w_groups < 1 || (Cc > 0 && Cc % w_groups != 0)) return 1;
    int per_group = Cc > 0 ? Cc / w_groups : 1;
    int maxM = H > W ? H : W;
    double *before = (double *)calloc((size_t)maxM + 1, sizeof(double));
    double *after = (double *)calloc((size_t)maxM + 1, sizeof(double));
    if (!before || !after) { free(before); free(after); return 1; }

    for (int b = 0; b < B; ++b)
        for (int c = 0; c < Cc; ++c) {
            size_t xo = (size_t)b * (size_t)Cc + (size_t)c;
            for (int i = 0; i < H; ++i)
                for (int j = 0; j < W; ++j) out[at(xo, H, W, i, j)] = 0.0;
            for (int d = 0; d < 4; ++d) {
                if (!(dirs & (1 << d))) continue;
                /* lambda / u plane: the direction's own, or the one shared plane */
                size_t go = ((size_t)b * (size_t)gate_dirs + (size_t)(gate_dirs == 4 ? d : 0)) *
                                (size_t)Cc + (size_t)c;
                /* logit field of the channel's group */
                size_t wo = (((size_t)b * 4 + (size_t)d) * (size_t)w_groups +
                             (size_t)(c / per_group)) * 3;
                int L = d < 2 ? H : W;
                int M = d < 2 ? W : H;
                for (int q = 0; q < M; ++q) before[q] = 0.0;
                for (int step = 0; step < L; ++step) {
                    int line = d % 2 ? L - 1 - step : step;
                    for (int q = 0; q < M; ++q) {
                        int i, j, on[3];
                        double s[3], w[3], sum;
                        position(d, line, q, &i, &j);
                        position_weights(wlogit, wo, H, W, d, line, q, M, on, s, w, &sum);
                        double v = 0.0;
                        for (int k = 0; k < 3; ++k)
                            if (on[k]) v += w[k] * before[q + k - 1];
                        after[q] = v + lambda[at(go, H, W, i, j)] * x[at(xo, H, W, i, j)];
                    }
                    for (int q = 0; q < M; ++q) {
                        int i, j;
                        position(d, line, q, &i, &j);
                        out[at(xo, H, W, i, j)] += u[at(go, H, W, i, j)] * after[q];
                    }
                    double *t = before; before = after; after = t;
                }
            }
        }
    free(before);
    free(after);
    return 0;
}
