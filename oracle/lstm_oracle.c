/*
 * lstm_oracle.c -- fp64 CPU oracle for the single-layer, unidirectional LSTM
 * forward pass and its backpropagation through time (BPTT).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
 * statement of what the GPU path computes.  Only tests/, the smoke check and
 * the cpu_baseline / reference leg of bench.py may load it.  It shares no code,
 * header, table or helper with the CUDA library, and the product path never
 * calls it.
 *
 * Source of every formula: "SingleLayerLstmGrad" (CANN ops-nn operator page):
 *   - forward-formula table (input concat, forget/input/candidate/output gate,
 *     cell state, hidden state);
 *   - "backward algorithm (time step t -> t-1)", initialisation and steps 1-6;
 *   - "gradient derivation" (cell-state chain rule, dL/dW = sum_t delta z_t^T);
 *   - parameter table (tensor shapes, layouts, optional inputs).
 *
 * Readings taken where the page is ambiguous:
 *   - W columns are [h | x], i.e. W = [W_h | W_x] with z_t = [h_{t-1}; x_t]
 *     (forward table "input concat" and step 5 "delta h_prev = delta z[1:dim h]");
 *   - gate rows are [i | f | g | o] (gate_order "ifjo", j = g) by default;
 *   - one bias b[4H];
 *   - the cell-gradient carry applies the forget gate ONCE: step 5 already sets
 *     delta c_prev = delta c_t * f_t, so step 2 adds delta c_next without a
 *     second factor f (the chain rule in "gradient derivation" fixes this);
 *   - delta h_next and delta c_next start at the dh/dc inputs (zero if absent);
 *   - dy is added at every step, including t = T-1 where dh is also added;
 *   - sequences in a batch are independent; dW and db sum over time and batch.
 *
 * Layouts (row-major, time-major, as in the parameter table):
 *   x[T][B][I], W[4H][H+I], b[4H], h0[B][H], c0[B][H], y[T][B][H],
 *   gates[T][B][4H] (post-activation i,f,g,o), cells[T][B][H],
 *   dy[T][B][H], dhT[B][H], dcT[B][H], dx[T][B][I], dW[4H][H+I], db[4H],
 *   dh0[B][H], dc0[B][H].
 *
 * Variable length ("seq_length", the parameter table's optional mask input of
 * shape [T][B][H], read as 1 = real step, 0 = padding): at a padded element
 * the state does not move -- c_t = m c~_t + (1 - m) c_{t-1} and
 * h_t = m h~_t + (1 - m) h_{t-1}, with c~, h~ the unmasked update, y_t = h_t --
 * and the backward pass is the exact gradient of that function (padding passes
 * delta h and delta c through unchanged and has zero gate gradients).  The
 * page gives no formula for the mask; this reading follows the Darknet LSTM
 * page's note that padding steps must not update the state or the gradients.
 * Mask values other than 0 and 1 are outside the reading (the backward uses
 * tanh of the saved cell state, which equals tanh c~ only where m = 1).
 *
 * Direction (the operator's "direction" attribute): "UNIDIRECTIONAL" runs the
 * recurrence over t = 0 .. T-1, "REDIRECTIONAL" (reverse = 1) over
 * t = T-1 .. 0: the step at time t then reads the state of time t+1 (initH /
 * initC before the first step, t = T-1), and hT / cT are the state after the
 * last step (t = 0).
 *
 * Gate order (the operator's "gate_order" attribute): "ifjo" (ijfo = 0) has the
 * row blocks of W, b, gates and dG in the order i, f, j (= g), o; "ijfo"
 * (ijfo = 1) in the order i, j, f, o.
 *
 * Parity is pinned (tests/test_oracle.py) by central finite differences of the
 * surrogate loss L = sum_t <dy_t, h_t> + <dhT, h_{T-1}> + <dcT, c_{T-1}>,
 * by the T = 1 closed form, the W = 0 closed form, a hand-computed example,
 * the invariants db = sum delta G and delta c_prev = delta c_t * f_t, and a
 * cross-check against torch.nn.LSTM in fp64.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Thread control for timing the oracle as a CPU baseline. */
void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Logistic sigmoid, forward-formula table; the two branches are the same
 * function written so that exp() never overflows. */
static double sigm(double a)
{
    if (a >= 0.0)
        return 1.0 / (1.0 + exp(-a));
    double e = exp(a);
    return e / (1.0 + e);
}

/* Forward pass, forward-formula table of "SingleLayerLstmGrad".
 * b, h0, c0 and mask may be NULL (zeros; no padding).  Returns 0, or -1 on bad
 * sizes / no memory. */
int oracle_lstm_fwd_ex(int T, int B, int I, int H,
                       const double *x, const double *W, const double *b,
                       const double *h0, const double *c0, const double *mask, int reverse,
                       int ijfo, double *y, double *gates, double *cells,
                       double *hT, double *cT)
{
    /* row block of each gate */
    const long BF = ijfo ? 2L * H : (long)H, BG = ijfo ? (long)H : 2L * H;
    if (T < 0 || B < 0 || I < 0 || H < 0)
        return -1;
    const long K = (long)H + I;  /* length of z_t */
    int err = 0;

#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
    for (int n = 0; n < B; ++n) {
        double *z = (double *)malloc(sizeof(double) * (K > 0 ? K : 1));
        double *a = (double *)malloc(sizeof(double) * (4L * H > 0 ? 4L * H : 1));
        double *cprev = (double *)malloc(sizeof(double) * (H > 0 ? H : 1));
        if (!z || !a || !cprev) {
            err |= 1;
            free(z); free(a); free(cprev);
            continue;
        }
        for (int j = 0; j < H; ++j) {
            z[j] = h0 ? h0[(long)n * H + j] : 0.0;      /* h_{-1} = initH */
            cprev[j] = c0 ? c0[(long)n * H + j] : 0.0;  /* c_{-1} = initC */
        }
        for (int s = 0; s < T; ++s) {
            const int t = reverse ? T - 1 - s : s;  /* time of the s-th step */
            /* input concat: z_t = [h_prev; x_t] (h_prev: the previous step's) */
            const double *xt = x + ((long)t * B + n) * I;
            const double *mt = mask ? mask + ((long)t * B + n) * H : NULL;
            for (int k = 0; k < I; ++k)
                z[H + k] = xt[k];
            /* a = W z_t + b for all four gates at once */
            for (long r = 0; r < 4L * H; ++r) {
                const double *Wr = W + r * K;
                double s = 0.0;
#pragma omp simd reduction(+ : s)
                for (long k = 0; k < K; ++k)
                    s += Wr[k] * z[k];
                if (b)
                    s += b[r];
                a[r] = s;
            }
            double *gt = gates + ((long)t * B + n) * 4L * H;
            double *ct = cells + ((long)t * B + n) * H;
            double *yt = y + ((long)t * B + n) * H;
            for (int j = 0; j < H; ++j) {
                double i_ = sigm(a[j]);               /* input gate */
                double f_ = sigm(a[BF + j]);          /* forget gate */
                double g_ = tanh(a[BG + j]);          /* candidate state */
                double o_ = sigm(a[3L * H + j]);      /* output gate */
                double c_ = f_ * cprev[j] + i_ * g_;  /* cell state */
                double h_ = o_ * tanh(c_);            /* hidden state */
                if (mt) {  /* padding keeps the previous state */
                    c_ = mt[j] * c_ + (1.0 - mt[j]) * cprev[j];
                    h_ = mt[j] * h_ + (1.0 - mt[j]) * z[j];
                }
                gt[j] = i_;
                gt[BF + j] = f_;
                gt[BG + j] = g_;
                gt[3L * H + j] = o_;
                ct[j] = c_;
                yt[j] = h_;
                cprev[j] = c_;
                z[j] = h_;  /* becomes h_{t-1} of the next step */
            }
        }
        for (int j = 0; j < H; ++j) {
            if (hT) hT[(long)n * H + j] = (T > 0) ? z[j] : (h0 ? h0[(long)n * H + j] : 0.0);
            if (cT) cT[(long)n * H + j] = cprev[j];
        }
        free(z); free(a); free(cprev);
    }
    return err ? -1 : 0;
}

int oracle_lstm_fwd(int T, int B, int I, int H,
                    const double *x, const double *W, const double *b,
                    const double *h0, const double *c0,
                    double *y, double *gates, double *cells,
                    double *hT, double *cT)
{
    return oracle_lstm_fwd_ex(T, B, I, H, x, W, b, h0, c0, NULL, 0, 0, y, gates, cells, hT, cT);
}

/* Backward pass, "backward algorithm (time step t -> t-1)" of
 * "SingleLayerLstmGrad", consuming the forward's saved y, gates and cells.
 * dy, dhT, dcT, h0, c0 and mask may be NULL (zeros; no padding).  dG is
 * optional scratch of T*B*4H doubles (allocated here when NULL); on return it
 * holds the pre-activation gate gradients [di | df | dg | do] of every step.
 * Returns 0, or -1 on bad sizes / no memory. */
int oracle_lstm_bwd_ex(int T, int B, int I, int H,
                       const double *x, const double *W,
                       const double *h0, const double *c0, const double *mask, int reverse,
                       int ijfo, const double *y, const double *gates, const double *cells,
                       const double *dy, const double *dhT, const double *dcT,
                       double *dx, double *dW, double *db,
                       double *dh0, double *dc0, double *dG)
{
    const long BF = ijfo ? 2L * H : (long)H, BG = ijfo ? (long)H : 2L * H;
    if (T < 0 || B < 0 || I < 0 || H < 0)
        return -1;
    const long K = (long)H + I;
    const long G4 = 4L * H;
    int own_dG = 0;
    if (!dG && (long)T * B * G4 > 0) {
        dG = (double *)malloc(sizeof(double) * (size_t)((long)T * B * G4));
        if (!dG)
            return -1;
        own_dG = 1;
    }
    int err = 0;

    /* Per-sequence recursion: steps 1, 2, 3, 5 and 6. */
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
    for (int n = 0; n < B; ++n) {
        double *dh_next = (double *)malloc(sizeof(double) * (H > 0 ? H : 1));
        double *dc_next = (double *)malloc(sizeof(double) * (H > 0 ? H : 1));
        double *dz = (double *)malloc(sizeof(double) * (K > 0 ? K : 1));
        double *dh_pass = (double *)malloc(sizeof(double) * (H > 0 ? H : 1));
        if (!dh_next || !dc_next || !dz || !dh_pass) {
            err |= 1;
            free(dh_next); free(dc_next); free(dz); free(dh_pass);
            continue;
        }
        /* initialisation: the gradients arriving from time T are the dh / dc
         * inputs (zero when absent); no forget factor is applied to them. */
        for (int j = 0; j < H; ++j) {
            dh_next[j] = dhT ? dhT[(long)n * H + j] : 0.0;
            dc_next[j] = dcT ? dcT[(long)n * H + j] : 0.0;
        }
        for (int s = T - 1; s >= 0; --s) {  /* steps in reverse order of the forward's */
            const int t = reverse ? T - 1 - s : s;         /* time of step s */
            const int tp = reverse ? t + 1 : t - 1;        /* time of step s - 1 */
            const double *gt = gates + ((long)t * B + n) * G4;
            const double *ct = cells + ((long)t * B + n) * H;
            const double *cp = (s > 0) ? cells + ((long)tp * B + n) * H
                                       : (c0 ? c0 + (long)n * H : NULL);
            const double *dyt = dy ? dy + ((long)t * B + n) * H : NULL;
            const double *mt = mask ? mask + ((long)t * B + n) * H : NULL;
            double *dGt = dG + ((long)t * B + n) * G4;
            for (int j = 0; j < H; ++j) {
                double i_ = gt[j], f_ = gt[BF + j], g_ = gt[BG + j], o_ = gt[3L * H + j];
                double c_ = ct[j];
                double c_prev = cp ? cp[j] : 0.0;
                double tc = tanh(c_);
                double m = mt ? mt[j] : 1.0;
                /* step 1: delta h_t = dL_t/dh_t + delta h_next; the update h~
                 * receives the share m, padding passes the rest to h_{t-1} */
                double dh_tot = (dyt ? dyt[j] : 0.0) + dh_next[j];
                double dh = m * dh_tot;
                dh_pass[j] = (1.0 - m) * dh_tot;
                /* step 2: delta c_t = delta h o (1 - tanh^2 c) + delta c_next,
                 * where delta c_next already carries the factor f_{t+1} (the
                 * update c~ receives the share m of delta c_next) */
                double dc = dh * o_ * (1.0 - tc * tc) + m * dc_next[j];
                /* step 3: pre-activation gate gradients */
                double d_o = dh * tc * o_ * (1.0 - o_);
                double d_g = dc * i_ * (1.0 - g_ * g_);
                double d_i = dc * g_ * i_ * (1.0 - i_);
                double d_f = dc * c_prev * f_ * (1.0 - f_);
                dGt[j] = d_i;
                dGt[BF + j] = d_f;
                dGt[BG + j] = d_g;
                dGt[3L * H + j] = d_o;
                /* step 5: delta c_prev = delta c_t * f_t (+ what padding passes) */
                dc_next[j] = dc * f_ + (1.0 - m) * dc_next[j];
            }
            /* step 5: delta z_t = sum over gates of W_*^T delta_* = W^T dG_t */
            for (long k = 0; k < K; ++k)
                dz[k] = 0.0;
            for (long r = 0; r < G4; ++r) {
                const double *Wr = W + r * K;
                double d = dGt[r];
                for (long k = 0; k < K; ++k)
                    dz[k] += Wr[k] * d;
            }
            /* delta x_t is the x-part of delta z_t; delta h_prev its h-part */
            double *dxt = dx + ((long)t * B + n) * I;
            for (int k = 0; k < I; ++k)
                dxt[k] = dz[H + k];
            /* step 6: carry delta h_prev into the next (earlier) step */
            for (int j = 0; j < H; ++j)
                dh_next[j] = dz[j] + dh_pass[j];
        }
        for (int j = 0; j < H; ++j) {
            if (dh0) dh0[(long)n * H + j] = dh_next[j];  /* dh_prev at t = 0 */
            if (dc0) dc0[(long)n * H + j] = dc_next[j];  /* dc_prev at t = 0 */
        }
        free(dh_next); free(dc_next); free(dz); free(dh_pass);
    }

    /* Step 4: dW = sum_{t,n} dG_{t,n} z_{t,n}^T and db = sum_{t,n} dG_{t,n},
     * with z_{t,n} = [h_{t-1}; x_t] (h_{-1} = initH).  Each row r of dW is
     * owned by one thread, so the sums are race-free. */
    if (!err) {
#pragma omp parallel for schedule(dynamic, 8)
        for (long r = 0; r < G4; ++r) {
            double *dWr = dW + r * K;
            double s_b = 0.0;
            for (long k = 0; k < K; ++k)
                dWr[k] = 0.0;
            for (int t = 0; t < T; ++t) {
                /* time of the step before time t's step (none: h_prev = initH) */
                const int tp = reverse ? t + 1 : t - 1;
                const int first = reverse ? (t == T - 1) : (t == 0);
                for (int n = 0; n < B; ++n) {
                    double d = dG[((long)t * B + n) * G4 + r];
                    s_b += d;
                    const double *hp = !first ? y + ((long)tp * B + n) * H
                                              : (h0 ? h0 + (long)n * H : NULL);
                    const double *xt = x + ((long)t * B + n) * I;
                    if (hp)
                        for (int k = 0; k < H; ++k)
                            dWr[k] += d * hp[k];
                    for (int k = 0; k < I; ++k)
                        dWr[H + k] += d * xt[k];
                }
            }
            db[r] = s_b;
        }
    }
    if (own_dG)
        free(dG);
    return err ? -1 : 0;
}

int oracle_lstm_bwd(int T, int B, int I, int H,
                    const double *x, const double *W,
                    const double *h0, const double *c0,
                    const double *y, const double *gates, const double *cells,
                    const double *dy, const double *dhT, const double *dcT,
                    double *dx, double *dW, double *db,
                    double *dh0, double *dc0, double *dG)
{
    return oracle_lstm_bwd_ex(T, B, I, H, x, W, h0, c0, NULL, 0, 0, y, gates, cells, dy, dhT,
                              dcT, dx, dW, db, dh0, dc0, dG);
}
