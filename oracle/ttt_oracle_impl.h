/*
 * TTT forward scan, primal form, one precision.  Included twice by
 * ttt_oracle.c: REAL=double (the oracle) and REAL=float (used only to measure
 * how much single-precision rounding grows through the recurrence).
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the bench's
 * CPU-baseline leg may call this code; the product path never does.
 *
 * Sources (page title, then section):
 *  [LR1] literature record "Learning to (Learn at Test Time): RNNs with
 *        Expressive Hidden States" (dmarx.github.io, lit-801), Key takeaways,
 *        bullet 1: state = weights W of a model f; update
 *        W_t = W_{t-1} - eta grad l(W_{t-1}; x_t); output z_t = f(theta_Q x_t; W_t).
 *  [LR2] same record, bullet 2: inner loss l(W; x_t) = ||f(theta_K x_t; W) - theta_V x_t||^2,
 *        token-dependent learning rate trained by the outer loop.
 *  [LR3] same record, bullet 3 (Theorem 1): linear f, batch GD, eta = 1/2, W0 = 0
 *        gives z_t = sum_{s<=t} (theta_V x_s)(theta_K x_s)^T (theta_Q x_t).
 *  [LR5] same record, bullet 5: mini-batch inner updates with b = 16; LayerNorm
 *        and a residual inside f.
 *  [ABS] codewithpapers.app record of the same paper, abstract: TTT-Linear
 *        (hidden state is a linear model) and TTT-MLP (a two-layer MLP).
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *  - ||.||^2 is a plain sum of squares (no 1/2, no mean), so dl/df = 2 (f - v).
 *    This is the scale under which Theorem 1 holds with eta = 1/2.
 *  - Inside a mini-batch every token's gradient is taken at the state the
 *    mini-batch started from; the running state W_t subtracts the gradients of
 *    all tokens s <= t of the mini-batch, each times its own eta_s, and the
 *    output of token t uses that W_t.  b = 1 is the per-token rule [LR1];
 *    b = T is batch GD [LR3].  When b does not divide T, the last mini-batch
 *    holds the remaining T mod b tokens.
 *  - LayerNorm: over the d features of one token, biased variance, eps inside
 *    the square root; gamma and beta are fixed (outer-loop) parameters, the
 *    inner loop updates W and b only.
 *  - GELU: the tanh form 0.5 x (1 + tanh(sqrt(2/pi)(x + 0.044715 x^3))).
 *  - Row vectors: f(x) = x W + b with W stored [in][out] row-major.
 */

#define CAT_(a, b) a##b
#define CAT(a, b) CAT_(a, b)
#define FN(name) CAT(name, SFX)

/* mean and 1/sqrt(var + eps) of one row, two passes. */
static void FN(ln_stats)(int d, const REAL* y, REAL eps, REAL* mu, REAL* s) {
    REAL m = 0, v = 0;
    for (int j = 0; j < d; j++) m += y[j];
    m /= (REAL)d;
    for (int j = 0; j < d; j++) v += (y[j] - m) * (y[j] - m);
    v /= (REAL)d;
    *mu = m;
    *s = (REAL)1 / SQRT(v + eps);
}

/* x + LN(y) with LN(y) = gamma * (y - mu) s + beta. */
static void FN(residual_ln)(int d, const REAL* x, const REAL* y, const REAL* gamma,
                            const REAL* beta, REAL eps, REAL* out) {
    REAL mu, s;
    FN(ln_stats)(d, y, eps, &mu, &s);
    for (int j = 0; j < d; j++) out[j] = x[j] + gamma[j] * (y[j] - mu) * s + beta[j];
}

/*
 * Given the pre-LN activation y of token x (LN mode), return the loss
 * ||x + LN(y) - v||^2 and write g = dl/dy.  The LayerNorm Jacobian is
 * d xhat_i / d y_j = s (delta_ij - 1/d - xhat_i xhat_j / d), so
 * g = s (gx - mean(gx) - xhat * mean(gx . xhat)) with gx = dl/dxhat = 2 gamma r.
 */
static REAL FN(ln_residual_loss_dy)(int d, const REAL* x, const REAL* v, const REAL* y,
                                    const REAL* gamma, const REAL* beta, REAL eps,
                                    REAL* xhat, REAL* g) {
    REAL mu, s, loss = 0, sum_gx = 0, sum_gxx = 0;
    FN(ln_stats)(d, y, eps, &mu, &s);
    for (int j = 0; j < d; j++) {
        xhat[j] = (y[j] - mu) * s;
        REAL r = x[j] + gamma[j] * xhat[j] + beta[j] - v[j];
        loss += r * r;
        g[j] = 2 * gamma[j] * r; /* dl/dxhat, held in g for now */
        sum_gx += g[j];
        sum_gxx += g[j] * xhat[j];
    }
    REAL mean_gx = sum_gx / (REAL)d, mean_gxx = sum_gxx / (REAL)d;
    for (int j = 0; j < d; j++) g[j] = s * (g[j] - mean_gx - xhat[j] * mean_gxx);
    return loss;
}

/* y = x W (+ b), x [din], W [din][dout]. */
static void FN(affine)(int din, int dout, const REAL* x, const REAL* W, const REAL* b, REAL* y) {
    for (int j = 0; j < dout; j++) y[j] = b ? b[j] : 0;
    for (int i = 0; i < din; i++) {
        REAL xi = x[i];
        const REAL* Wi = W + (long)i * dout;
        for (int j = 0; j < dout; j++) y[j] += xi * Wi[j];
    }
}

/* ---------------------------- TTT-Linear ---------------------------------- */

/*
 * Loss of one token and g = dl/dy for the linear inner model [ABS], [LR2], [LR5]:
 * LN mode f(x) = x + LN(x W + b); plain mode f(x) = x W.
 * scratch: 2 d.
 */
static REAL FN(linear_token_dy)(int d, int mode, REAL eps, const REAL* k, const REAL* v,
                                const REAL* W, const REAL* b, const REAL* gamma,
                                const REAL* beta, REAL* g, REAL* scratch) {
    REAL* y = scratch;
    REAL* xhat = scratch + d;
    if (mode == ORACLE_MODE_PLAIN) {
        REAL loss = 0;
        FN(affine)(d, d, k, W, NULL, y);
        for (int j = 0; j < d; j++) {
            REAL r = y[j] - v[j];
            loss += r * r;
            g[j] = 2 * r;
        }
        return loss;
    }
    FN(affine)(d, d, k, W, b, y);
    return FN(ln_residual_loss_dy)(d, k, v, y, gamma, beta, eps, xhat, g);
}

/* f(x; W, b) for the linear inner model.  scratch: d. */
static void FN(linear_apply)(int d, int mode, REAL eps, const REAL* x, const REAL* W,
                             const REAL* b, const REAL* gamma, const REAL* beta, REAL* out,
                             REAL* scratch) {
    if (mode == ORACLE_MODE_PLAIN) {
        FN(affine)(d, d, x, W, NULL, out);
        return;
    }
    FN(affine)(d, d, x, W, b, scratch);
    FN(residual_ln)(d, x, scratch, gamma, beta, eps, out);
}

/* Loss and gradients dl/dW = k^T g, dl/db = g of one token. */
REAL FN(oracle_linear_loss_grad)(int d, int mode, REAL eps, const REAL* k, const REAL* v,
                                 const REAL* W, const REAL* b, const REAL* gamma,
                                 const REAL* beta, REAL* gW, REAL* gb) {
    REAL* g = (REAL*)malloc(sizeof(REAL) * 3 * d);
    REAL loss = FN(linear_token_dy)(d, mode, eps, k, v, W, b, gamma, beta, g, g + d);
    if (gW)
        for (int i = 0; i < d; i++)
            for (int j = 0; j < d; j++) gW[(long)i * d + j] = k[i] * g[j];
    if (gb)
        for (int j = 0; j < d; j++) gb[j] = (mode == ORACLE_MODE_PLAIN) ? 0 : g[j];
    free(g);
    return loss;
}

/*
 * Causal TTT-Linear scan over [B,H,T,d], token by token, mini-batch by
 * mini-batch, with the per-token state W_t materialised [LR1], [LR5].
 * b0 / b_T may be NULL in plain mode.  Returns 0, or -1 on bad arguments.
 */
int FN(oracle_ttt_linear)(int B, int H, int T, int d, int mb, int mode, REAL eps,
                          const REAL* Q, const REAL* K, const REAL* V, const REAL* eta,
                          const REAL* W0, const REAL* b0, const REAL* gamma,
                          const REAL* beta, REAL* Z, REAL* W_T, REAL* b_T, int nthreads) {
    if (B < 0 || H < 0 || T < 0 || d <= 0 || mb <= 0) return -1;
    if (mode != ORACLE_MODE_PLAIN && mode != ORACLE_MODE_LN_RESIDUAL) return -1;
    if (nthreads <= 0) nthreads = 1;
    long nbh = (long)B * H;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (long bh = 0; bh < nbh; bh++) {
        int h = (int)(bh % H);
        const REAL* gam = gamma ? gamma + (long)h * d : NULL;
        const REAL* bet = beta ? beta + (long)h * d : NULL;
        REAL* Ws = (REAL*)malloc(sizeof(REAL) * (size_t)d * d); /* mini-batch start state */
        REAL* Wc = (REAL*)malloc(sizeof(REAL) * (size_t)d * d); /* running state W_t */
        REAL* buf = (REAL*)calloc((size_t)6 * d, sizeof(REAL));
        REAL *bs = buf, *bc = buf + d, *g = buf + 2 * d, *scratch = buf + 3 * d;
        memcpy(Ws, W0 + bh * d * d, sizeof(REAL) * (size_t)d * d);
        if (b0 && mode != ORACLE_MODE_PLAIN) memcpy(bs, b0 + bh * d, sizeof(REAL) * d);
        for (int m = 0; m < T; m += mb) {
            memcpy(Wc, Ws, sizeof(REAL) * (size_t)d * d);
            memcpy(bc, bs, sizeof(REAL) * d);
            for (int t = m; t < m + mb && t < T; t++) {
                long row = (bh * T + t) * d;
                REAL e = eta[bh * T + t];
                /* gradient of token t, taken at the mini-batch's start state */
                FN(linear_token_dy)(d, mode, eps, K + row, V + row, Ws, bs, gam, bet, g, scratch);
                /* W_t = W_{t-1} - eta_t k_t^T g_t (and b_t = b_{t-1} - eta_t g_t) */
                for (int i = 0; i < d; i++) {
                    REAL ek = e * K[row + i];
                    REAL* Wi = Wc + (long)i * d;
                    for (int j = 0; j < d; j++) Wi[j] -= ek * g[j];
                }
                if (mode != ORACLE_MODE_PLAIN)
                    for (int j = 0; j < d; j++) bc[j] -= e * g[j];
                /* output rule: z_t = f(q_t; W_t), W_t already includes token t */
                FN(linear_apply)(d, mode, eps, Q + row, Wc, bc, gam, bet, Z + row, scratch);
            }
            memcpy(Ws, Wc, sizeof(REAL) * (size_t)d * d);
            memcpy(bs, bc, sizeof(REAL) * d);
        }
        if (W_T) memcpy(W_T + bh * d * d, Ws, sizeof(REAL) * (size_t)d * d);
        if (b_T) memcpy(b_T + bh * d, bs, sizeof(REAL) * d);
        free(Ws);
        free(Wc);
        free(buf);
    }
    return 0;
}

/*
 * TTT-Linear decode: the same scan continued by T more tokens from position
 * pos0 of a mini-batch [LR1], [LR5].  The state carried between calls is the
 * running state (Wc, bc) = W_t and the state the current mini-batch started
 * from (Wm, bm), at which that mini-batch's gradients are taken.  All four are
 * read and overwritten in place; on return (Wm, bm) is the start state of the
 * mini-batch the next token falls in.  bc / bm may be NULL in plain mode.
 * Returns 0, or -1 on bad arguments.
 */
int FN(oracle_ttt_linear_decode)(int B, int H, int T, int d, int mb, int pos0, int mode, REAL eps,
                                 const REAL* Q, const REAL* K, const REAL* V, const REAL* eta,
                                 REAL* Wc_all, REAL* bc_all, REAL* Wm_all, REAL* bm_all,
                                 const REAL* gamma, const REAL* beta, REAL* Z, int nthreads) {
    if (B < 0 || H < 0 || T < 0 || d <= 0 || mb <= 0 || pos0 < 0 || pos0 >= mb) return -1;
    if (mode != ORACLE_MODE_PLAIN && mode != ORACLE_MODE_LN_RESIDUAL) return -1;
    if (nthreads <= 0) nthreads = 1;
    const int ln = mode != ORACLE_MODE_PLAIN;
    long nbh = (long)B * H;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (long bh = 0; bh < nbh; bh++) {
        int h = (int)(bh % H);
        const REAL* gam = gamma ? gamma + (long)h * d : NULL;
        const REAL* bet = beta ? beta + (long)h * d : NULL;
        REAL* Wc = Wc_all + bh * d * d;
        REAL* Wm = Wm_all + bh * d * d;
        REAL* buf = (REAL*)calloc((size_t)6 * d, sizeof(REAL));
        REAL *bc = buf, *bm = buf + d, *g = buf + 2 * d, *scratch = buf + 3 * d;
        if (ln && bc_all) memcpy(bc, bc_all + bh * d, sizeof(REAL) * d);
        if (ln && bm_all) memcpy(bm, bm_all + bh * d, sizeof(REAL) * d);
        for (int t = 0; t < T; t++) {
            if ((pos0 + t) % mb == 0) { /* a mini-batch starts at this token */
                memcpy(Wm, Wc, sizeof(REAL) * (size_t)d * d);
                memcpy(bm, bc, sizeof(REAL) * d);
            }
            long row = (bh * T + t) * d;
            REAL e = eta[bh * T + t];
            FN(linear_token_dy)(d, mode, eps, K + row, V + row, Wm, bm, gam, bet, g, scratch);
            for (int i = 0; i < d; i++) {
                REAL ek = e * K[row + i];
                REAL* Wi = Wc + (long)i * d;
                for (int j = 0; j < d; j++) Wi[j] -= ek * g[j];
            }
            if (ln)
                for (int j = 0; j < d; j++) bc[j] -= e * g[j];
            FN(linear_apply)(d, mode, eps, Q + row, Wc, bc, gam, bet, Z + row, scratch);
        }
        if ((pos0 + T) % mb == 0) { /* the next token starts a mini-batch */
            memcpy(Wm, Wc, sizeof(REAL) * (size_t)d * d);
            memcpy(bm, bc, sizeof(REAL) * d);
        }
        if (ln && bc_all) memcpy(bc_all + bh * d, bc, sizeof(REAL) * d);
        if (ln && bm_all) memcpy(bm_all + bh * d, bm, sizeof(REAL) * d);
        free(buf);
    }
    return 0;
}

/* ----------------------------- TTT-MLP ------------------------------------ */

static REAL FN(gelu)(REAL x) {
    const REAL c = (REAL)0.7978845608028654; /* sqrt(2/pi) */
    return (REAL)0.5 * x * ((REAL)1 + TANH(c * (x + (REAL)0.044715 * x * x * x)));
}

/* derivative of the tanh-form GELU above */
static REAL FN(gelu_prime)(REAL x) {
    const REAL c = (REAL)0.7978845608028654;
    REAL th = TANH(c * (x + (REAL)0.044715 * x * x * x));
    return (REAL)0.5 * ((REAL)1 + th) +
           (REAL)0.5 * x * ((REAL)1 - th * th) * c * ((REAL)1 + (REAL)3 * (REAL)0.044715 * x * x);
}

/*
 * Loss of one token for f(x) = x + LN(GELU(x W1 + b1) W2 + b2) [ABS], [LR2], [LR5];
 * writes g2 = dl/dy, g1 = dl/dz1 (z1 = x W1 + b1) and a = GELU(z1).
 * scratch: 2 d + hid.
 */
static REAL FN(mlp_token_grads)(int d, int hid, REAL eps, const REAL* k, const REAL* v,
                                const REAL* W1, const REAL* b1, const REAL* W2,
                                const REAL* b2, const REAL* gamma, const REAL* beta,
                                REAL* a, REAL* g1, REAL* g2, REAL* scratch) {
    REAL* y = scratch;
    REAL* xhat = scratch + d;
    REAL* z1 = scratch + 2 * d;
    FN(affine)(d, hid, k, W1, b1, z1);
    for (int i = 0; i < hid; i++) a[i] = FN(gelu)(z1[i]);
    FN(affine)(hid, d, a, W2, b2, y);
    REAL loss = FN(ln_residual_loss_dy)(d, k, v, y, gamma, beta, eps, xhat, g2);
    /* back through the second layer and the activation */
    for (int i = 0; i < hid; i++) {
        REAL acc = 0;
        const REAL* W2i = W2 + (long)i * d;
        for (int j = 0; j < d; j++) acc += W2i[j] * g2[j];
        g1[i] = acc * FN(gelu_prime)(z1[i]);
    }
    return loss;
}

static void FN(mlp_apply)(int d, int hid, REAL eps, const REAL* x, const REAL* W1,
                          const REAL* b1, const REAL* W2, const REAL* b2, const REAL* gamma,
                          const REAL* beta, REAL* out, REAL* scratch) {
    REAL* y = scratch;
    REAL* a = scratch + d;
    FN(affine)(d, hid, x, W1, b1, a);
    for (int i = 0; i < hid; i++) a[i] = FN(gelu)(a[i]);
    FN(affine)(hid, d, a, W2, b2, y);
    FN(residual_ln)(d, x, y, gamma, beta, eps, out);
}

REAL FN(oracle_mlp_loss_grad)(int d, int hid, REAL eps, const REAL* k, const REAL* v,
                              const REAL* W1, const REAL* b1, const REAL* W2, const REAL* b2,
                              const REAL* gamma, const REAL* beta, REAL* gW1, REAL* gb1,
                              REAL* gW2, REAL* gb2) {
    REAL* buf = (REAL*)malloc(sizeof(REAL) * (size_t)(3 * hid + 3 * d + hid));
    REAL *a = buf, *g1 = buf + hid, *g2 = buf + 2 * hid, *scratch = buf + 2 * hid + d;
    REAL loss = FN(mlp_token_grads)(d, hid, eps, k, v, W1, b1, W2, b2, gamma, beta, a, g1, g2,
                                    scratch);
    if (gW1)
        for (int i = 0; i < d; i++)
            for (int j = 0; j < hid; j++) gW1[(long)i * hid + j] = k[i] * g1[j];
    if (gb1) memcpy(gb1, g1, sizeof(REAL) * hid);
    if (gW2)
        for (int i = 0; i < hid; i++)
            for (int j = 0; j < d; j++) gW2[(long)i * d + j] = a[i] * g2[j];
    if (gb2) memcpy(gb2, g2, sizeof(REAL) * d);
    free(buf);
    return loss;
}

/* Causal TTT-MLP scan, same loop structure as the linear scan. */
int FN(oracle_ttt_mlp)(int B, int H, int T, int d, int hid, int mb, REAL eps, const REAL* Q,
                       const REAL* K, const REAL* V, const REAL* eta, const REAL* W1_0,
                       const REAL* b1_0, const REAL* W2_0, const REAL* b2_0, const REAL* gamma,
                       const REAL* beta, REAL* Z, REAL* W1_T, REAL* b1_T, REAL* W2_T,
                       REAL* b2_T, int nthreads) {
    if (B < 0 || H < 0 || T < 0 || d <= 0 || hid <= 0 || mb <= 0) return -1;
    if (nthreads <= 0) nthreads = 1;
    long nbh = (long)B * H;
    size_t nW = (size_t)d * hid;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (long bh = 0; bh < nbh; bh++) {
        int h = (int)(bh % H);
        const REAL* gam = gamma + (long)h * d;
        const REAL* bet = beta + (long)h * d;
        REAL* st = (REAL*)malloc(sizeof(REAL) * (4 * nW + 2 * (size_t)hid + 2 * (size_t)d));
        REAL *W1s = st, *W2s = st + nW, *W1c = st + 2 * nW, *W2c = st + 3 * nW;
        REAL* vec = (REAL*)malloc(sizeof(REAL) * (size_t)(4 * hid + 5 * d + 2 * d + hid));
        REAL *b1s = vec, *b1c = vec + hid, *a = vec + 2 * hid, *g1 = vec + 3 * hid;
        REAL *b2s = vec + 4 * hid, *b2c = b2s + d, *g2 = b2s + 2 * d, *scratch = b2s + 3 * d;
        memcpy(W1s, W1_0 + bh * nW, sizeof(REAL) * nW);
        memcpy(W2s, W2_0 + bh * nW, sizeof(REAL) * nW);
        memcpy(b1s, b1_0 + bh * hid, sizeof(REAL) * hid);
        memcpy(b2s, b2_0 + bh * d, sizeof(REAL) * d);
        for (int m = 0; m < T; m += mb) {
            memcpy(W1c, W1s, sizeof(REAL) * nW);
            memcpy(W2c, W2s, sizeof(REAL) * nW);
            memcpy(b1c, b1s, sizeof(REAL) * hid);
            memcpy(b2c, b2s, sizeof(REAL) * d);
            for (int t = m; t < m + mb && t < T; t++) {
                long row = (bh * T + t) * d;
                REAL e = eta[bh * T + t];
                FN(mlp_token_grads)(d, hid, eps, K + row, V + row, W1s, b1s, W2s, b2s, gam, bet,
                                    a, g1, g2, scratch);
                for (int i = 0; i < d; i++) {
                    REAL ek = e * K[row + i];
                    REAL* W1i = W1c + (long)i * hid;
                    for (int j = 0; j < hid; j++) W1i[j] -= ek * g1[j];
                }
                for (int j = 0; j < hid; j++) b1c[j] -= e * g1[j];
                for (int i = 0; i < hid; i++) {
                    REAL ea = e * a[i];
                    REAL* W2i = W2c + (long)i * d;
                    for (int j = 0; j < d; j++) W2i[j] -= ea * g2[j];
                }
                for (int j = 0; j < d; j++) b2c[j] -= e * g2[j];
                FN(mlp_apply)(d, hid, eps, Q + row, W1c, b1c, W2c, b2c, gam, bet, Z + row,
                              scratch);
            }
            memcpy(W1s, W1c, sizeof(REAL) * nW);
            memcpy(W2s, W2c, sizeof(REAL) * nW);
            memcpy(b1s, b1c, sizeof(REAL) * hid);
            memcpy(b2s, b2c, sizeof(REAL) * d);
        }
        if (W1_T) memcpy(W1_T + bh * nW, W1s, sizeof(REAL) * nW);
        if (b1_T) memcpy(b1_T + bh * hid, b1s, sizeof(REAL) * hid);
        if (W2_T) memcpy(W2_T + bh * nW, W2s, sizeof(REAL) * nW);
        if (b2_T) memcpy(b2_T + bh * d, b2s, sizeof(REAL) * d);
        free(st);
        free(vec);
    }
    return 0;
}

/*
 * TTT-MLP decode: the MLP scan continued by T tokens from position pos0 of a
 * mini-batch, as oracle_ttt_linear_decode for the linear model [LR1], [LR5],
 * [ABS].  (W1c, b1c, W2c, b2c) is the running state, (W1m, b1m, W2m, b2m)
 * the state the current mini-batch started from; all are read and
 * overwritten in place.  Returns 0, or -1 on bad arguments.
 */
int FN(oracle_ttt_mlp_decode)(int B, int H, int T, int d, int hid, int mb, int pos0, REAL eps,
                              const REAL* Q, const REAL* K, const REAL* V, const REAL* eta,
                              REAL* W1c_all, REAL* b1c_all, REAL* W2c_all, REAL* b2c_all,
                              REAL* W1m_all, REAL* b1m_all, REAL* W2m_all, REAL* b2m_all,
                              const REAL* gamma, const REAL* beta, REAL* Z, int nthreads) {
    if (B < 0 || H < 0 || T < 0 || d <= 0 || hid <= 0 || mb <= 0 || pos0 < 0 || pos0 >= mb) return -1;
    if (nthreads <= 0) nthreads = 1;
    long nbh = (long)B * H;
    size_t nW = (size_t)d * hid;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (long bh = 0; bh < nbh; bh++) {
        int h = (int)(bh % H);
        const REAL* gam = gamma + (long)h * d;
        const REAL* bet = beta + (long)h * d;
        REAL *W1c = W1c_all + bh * nW, *W2c = W2c_all + bh * nW, *b1c = b1c_all + bh * hid, *b2c = b2c_all + bh * d;
        REAL *W1m = W1m_all + bh * nW, *W2m = W2m_all + bh * nW, *b1m = b1m_all + bh * hid, *b2m = b2m_all + bh * d;
        REAL* vec = (REAL*)malloc(sizeof(REAL) * (size_t)(2 * hid + 5 * d + hid));
        REAL *a = vec, *g1 = vec + hid, *g2 = vec + 2 * hid, *scratch = g2 + d;
        for (int t = 0; t < T; t++) {
            if ((pos0 + t) % mb == 0) { /* a mini-batch starts at this token */
                memcpy(W1m, W1c, sizeof(REAL) * nW);
                memcpy(W2m, W2c, sizeof(REAL) * nW);
                memcpy(b1m, b1c, sizeof(REAL) * hid);
                memcpy(b2m, b2c, sizeof(REAL) * d);
            }
            long row = (bh * T + t) * d;
            REAL e = eta[bh * T + t];
            FN(mlp_token_grads)(d, hid, eps, K + row, V + row, W1m, b1m, W2m, b2m, gam, bet, a, g1, g2,
                                scratch);
            for (int i = 0; i < d; i++) {
                REAL ek = e * K[row + i];
                REAL* W1i = W1c + (long)i * hid;
                for (int j = 0; j < hid; j++) W1i[j] -= ek * g1[j];
            }
            for (int j = 0; j < hid; j++) b1c[j] -= e * g1[j];
            for (int i = 0; i < hid; i++) {
                REAL ea = e * a[i];
                REAL* W2i = W2c + (long)i * d;
                for (int j = 0; j < d; j++) W2i[j] -= ea * g2[j];
            }
            for (int j = 0; j < d; j++) b2c[j] -= e * g2[j];
            FN(mlp_apply)(d, hid, eps, Q + row, W1c, b1c, W2c, b2c, gam, bet, Z + row, scratch);
        }
        if ((pos0 + T) % mb == 0) { /* the next token starts a mini-batch */
            memcpy(W1m, W1c, sizeof(REAL) * nW);
            memcpy(W2m, W2c, sizeof(REAL) * nW);
            memcpy(b1m, b1c, sizeof(REAL) * hid);
            memcpy(b2m, b2c, sizeof(REAL) * d);
        }
        free(vec);
    }
    return 0;
}

#undef FN
#undef CAT
#undef CAT_
