/*
 * wkv_oracle.c -- plain fp64 CPU oracle for the two WKV recurrences.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
 * CPU-baseline / reference arm may load or run this library.  The CUDA library
 * (wkv_recurrence_02_b200) never calls it, links it or includes anything from it;
 * the two share no code, header, table or constant.
 *
 * Every input is fp64 (bf16 / fp32 values the GPU sees are widened exactly by the
 * caller), every operation is fp64, and each recurrence is walked serially in the
 * order the pages state it.  OpenMP is used only across independent units
 * ((b,c) for WKV-4, (b,h) for WKV-6); it never reorders work inside a unit.
 *
 * Sources (page title, section):
 *  [R4]  "RWKV: Reinventing RNNs for the Transformer Era" (Chinese translation),
 *        section "利用时间结构进行时序数据处理" (exploiting temporal structure): the time
 *        decay e^{-w} and the bonus e^{u} of eq. 14; section "梯度稳定性和层堆叠"
 *        (gradient stability): the attention-like score is updated by a single-step
 *        "time-dependent softmax", which is what makes the running-max form below
 *        the method's own evaluation order.  Eq. 14 itself is missing from the page;
 *        its content (the weighted average written out in wkv4_step below) is the
 *        RWKV-4 WKV definition the page refers to.
 *  [E4]  "RWKV-5/6 (Eagle and Finch)" summary, section 4: vectors are row vectors of
 *        size D/h and matrices act on the right.
 *  [E412] same page, section 4.1.2 (Eagle time mixing): the state s is a sum of
 *        k^T v; each channel of s is decayed by the matching channel of w at every
 *        step; the learned gain u multiplies the current token's k^T v, which is
 *        added to the state; the receptance r multiplies that sum like a query.
 *        w = exp(-exp(omega)) lies in (0,1).
 *  [F422] same page, section 4.2.2 (Finch time mixing): w_t varies per token.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

/*
 * WKV-4, one channel of one sequence, [R4].
 *
 * Definition (per channel, decay rate w, bonus u, keys k_i, values v_i):
 *   wkv_t = ( sum_{i<t} e^{-(t-1-i) w + k_i} v_i + e^{u + k_t} v_t )
 *         / ( sum_{i<t} e^{-(t-1-i) w + k_i}     + e^{u + k_t}     )
 *
 * The past sums are carried as (a, b, p) with numerator = a e^p and
 * denominator = b e^p.  Each step rescales to the larger exponent (the
 * "time-dependent softmax" single-step update), so no exponential overflows.
 * After token t the state holds sum_{i<=t} e^{-(t-i) w + k_i} (v_i | 1).
 * An empty state is a = b = 0, p = -inf.
 */
static void wkv4_channel(int64_t T, int64_t stride, double w, double u,
                         const double *k, const double *v, double *y,
                         double *a_io, double *b_io, double *p_io)
{
    double a = *a_io, b = *b_io, p = *p_io;
    for (int64_t t = 0; t < T; ++t) {
        const double kt = k[t * stride];
        const double vt = v[t * stride];

        /* output: past state (not yet decayed for this step) plus the bonus term */
        double q = p > u + kt ? p : u + kt;
        double e_past = exp(p - q);        /* weight of the carried sums      */
        double e_now = exp(u + kt - q);    /* weight e^{u+k_t} of the current */
        y[t * stride] = (e_past * a + e_now * vt) / (e_past * b + e_now);

        /* state update: decay the past by e^{-w}, add e^{k_t} (v_t | 1) */
        double q2 = p - w > kt ? p - w : kt;
        double e_decay = exp(p - w - q2);
        double e_key = exp(kt - q2);
        a = e_decay * a + e_key * vt;
        b = e_decay * b + e_key;
        p = q2;
    }
    *a_io = a;
    *b_io = b;
    *p_io = p;
}

/*
 * k, v, y: [B, T, C] (channel innermost); w, u: [C].
 * s0, sT: [B, 3, C] = (a, b, p) per channel, or NULL (s0 NULL = empty state;
 * sT NULL = not written).  sT may equal s0.
 */
void oracle_wkv4(int64_t B, int64_t T, int64_t C,
                 const double *w, const double *u,
                 const double *k, const double *v,
                 const double *s0, double *y, double *sT)
{
    int64_t units = B * C;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < units; ++n) {
        int64_t bi = n / C, c = n % C;
        double a = 0.0, b = 0.0, p = -INFINITY;
        if (s0) {
            a = s0[(bi * 3 + 0) * C + c];
            b = s0[(bi * 3 + 1) * C + c];
            p = s0[(bi * 3 + 2) * C + c];
        }
        const int64_t base = bi * T * C + c;
        wkv4_channel(T, C, w[c], u[c], k + base, v + base, y + base, &a, &b, &p);
        if (sT) {
            sT[(bi * 3 + 0) * C + c] = a;
            sT[(bi * 3 + 1) * C + c] = b;
            sT[(bi * 3 + 2) * C + c] = p;
        }
    }
}

/*
 * WKV-6 (Eagle / Finch), one head of one sequence, [E4] [E412] [F422].
 *
 * S is N x N; row i = key channel (decayed by w_i), column j = value channel.
 * For each token t, in this order:
 *   o_t[j] = sum_i r_t[i] * ( S[i][j] + u[i] k_t[i] v_t[j] )
 *   S[i][j] = w_t[i] S[i][j] + k_t[i] v_t[j]
 * so the output reads the state before this token's decay, and the newest
 * past key reaches the query undecayed.
 */
static void wkv6_head(int64_t T, int64_t N, int64_t stride,
                      const double *r, const double *k, const double *v,
                      const double *w, const double *u,
                      double *S, double *y)
{
    for (int64_t t = 0; t < T; ++t) {
        const double *rt = r + t * stride;
        const double *kt = k + t * stride;
        const double *vt = v + t * stride;
        const double *wt = w + t * stride;
        double *yt = y + t * stride;
        for (int64_t j = 0; j < N; ++j) {
            double o = 0.0;
            for (int64_t i = 0; i < N; ++i)
                o += rt[i] * (S[i * N + j] + u[i] * kt[i] * vt[j]);
            yt[j] = o;
        }
        for (int64_t i = 0; i < N; ++i)
            for (int64_t j = 0; j < N; ++j)
                S[i * N + j] = wt[i] * S[i * N + j] + kt[i] * vt[j];
    }
}

/*
 * r, k, v, w, y: [B, T, H, N] (channel innermost); u: [H, N].
 * s0, sT: [B, H, N, N] (row = key channel), or NULL (s0 NULL = zero state;
 * sT NULL = not written).  sT may equal s0.  work: B*H*N*N doubles of scratch
 * owned by the caller (the oracle allocates nothing).
 */
void oracle_wkv6(int64_t B, int64_t T, int64_t H, int64_t N,
                 const double *r, const double *k, const double *v,
                 const double *w, const double *u,
                 const double *s0, double *y, double *sT, double *work)
{
    int64_t units = B * H;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < units; ++n) {
        int64_t bi = n / H, h = n % H;
        double *S = work + n * N * N;
        for (int64_t e = 0; e < N * N; ++e)
            S[e] = s0 ? s0[n * N * N + e] : 0.0;
        const int64_t base = (bi * T * H + h) * N;
        wkv6_head(T, N, H * N, r + base, k + base, v + base, w + base,
                  u + h * N, S, y + base);
        if (sT)
            for (int64_t e = 0; e < N * N; ++e)
                sT[n * N * N + e] = S[e];
    }
}

/* Eagle time mixing ("RWKV-5/6 (Eagle and Finch)" summary, section 4.1.2, and the
 * architecture overview of section 4): the WKV output of each head is normalised by a
 * LayerNorm over that head's N channels (equivalently GroupNorm over H groups), with a
 * per-channel scale ln_w and shift ln_b, and multiplied by the SiLU attention gate:
 *
 *   y = SiLU(g) * (ln_w * (o - mean) / sqrt(var + eps) + ln_b),   SiLU(g) = g / (1 + e^-g)
 *
 * mean and var (the mean of squared deviations) are taken over the N channels of one
 * (b, t, h).  o, g, y: [B,T,H,N]; ln_w, ln_b: [H,N].  The output projection that follows
 * in the model is a dense GEMM and is not part of the recurrence.
 */
void oracle_head_norm_gate(int64_t B, int64_t T, int64_t H, int64_t N, const double *o, const double *g,
                           const double *ln_w, const double *ln_b, double eps, double *y)
{
    const int64_t rows = B * T * H;
#pragma omp parallel for schedule(static)
    for (int64_t row = 0; row < rows; ++row) {
        const int64_t h = row % H;
        const double *x = o + row * N;
        double mean = 0.0;
        for (int64_t n = 0; n < N; ++n) mean += x[n];
        mean /= (double)N;
        double var = 0.0;
        for (int64_t n = 0; n < N; ++n) {
            const double d = x[n] - mean;
            var += d * d;
        }
        var /= (double)N;
        const double rstd = 1.0 / sqrt(var + eps);
        for (int64_t n = 0; n < N; ++n) {
            const double gn = g[row * N + n];
            const double gate = gn / (1.0 + exp(-gn));
            y[row * N + n] = gate * (ln_w[h * N + n] * (x[n] - mean) * rstd + ln_b[h * N + n]);
        }
    }
}

/*
 * Decay from its logit, [E412] and [F422].
 *
 * Eagle obtains the per-channel decay as w = exp(-exp(omega)) from the trainable logit
 * omega, which puts w in (0,1); Finch adds a per-token, data-dependent offset (a LoRA of
 * the token-shifted input, section 4.2.1) to omega before the same map, giving w_t per
 * token and channel.  This evaluates the map elementwise: w[i] = exp(-exp(omega[i])),
 * n elements.  omega = -inf gives 1, omega = +inf gives 0.
 */
void oracle_decay_from_logit(int64_t n, const double *omega, double *w)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) w[i] = exp(-exp(omega[i]));
}

/*
 * WKV-6 backward: the reverse-mode derivative of oracle_wkv6 ([E412], [F422]) for a loss
 * L whose gradients with respect to the outputs are dy = dL/dy [B,T,H,N] and
 * dsT = dL/dsT [B,H,N,N] (NULL = zero).  The forward pass is walked first and every state
 * it passes through is kept; then, with Lambda = dL/dS for the state after token t
 * (Lambda = dsT after the last token), the chain rule through the two forward lines
 *   o_t[j] = sum_i r_t[i] (S[i][j] + u[i] k_t[i] v_t[j]),   S' = diag(w_t) S + k_t^T v_t
 * gives, for t = T-1 down to 0 with S = the state before token t:
 *   dr_t[i] = sum_j dy_t[j] (S[i][j] + u[i] k_t[i] v_t[j])
 *   dk_t[i] = sum_j Lambda[i][j] v_t[j] + sum_j dy_t[j] r_t[i] u[i] v_t[j]
 *   dv_t[j] = sum_i Lambda[i][j] k_t[i] + sum_i dy_t[j] r_t[i] u[i] k_t[i]
 *   dw_t[i] = sum_j Lambda[i][j] S[i][j]
 *   du[i]  += sum_j dy_t[j] r_t[i] k_t[i] v_t[j]
 *   Lambda[i][j] <- w_t[i] Lambda[i][j] + r_t[i] dy_t[j]    (the gradient reaching S)
 * and ds0 = Lambda after token 0 is undone.  du is summed over the batch rows (u is
 * shared by them).  Outputs dr, dk, dv, dw: [B,T,H,N]; du: [H,N]; ds0: [B,H,N,N] or NULL.
 * work: H*(T+1)*N*N + H*N*N doubles of caller-owned scratch.
 */
void oracle_wkv6_backward(int64_t B, int64_t T, int64_t H, int64_t N,
                          const double *r, const double *k, const double *v, const double *w,
                          const double *u, const double *s0, const double *dy, const double *dsT,
                          double *dr, double *dk, double *dv, double *dw, double *du, double *ds0,
                          double *work)
{
    const int64_t NN = N * N, stride = H * N;
#pragma omp parallel for schedule(static)
    for (int64_t h = 0; h < H; ++h) {
        double *Sall = work + h * (T + 1) * NN;  /* Sall[t] = state before token t */
        double *L = work + H * (T + 1) * NN + h * NN;
        const double *uh = u + h * N;
        for (int64_t i = 0; i < N; ++i) du[h * N + i] = 0.0;
        for (int64_t bi = 0; bi < B; ++bi) {
            const int64_t n = bi * H + h, base = (bi * T * H + h) * N;
            for (int64_t e = 0; e < NN; ++e) Sall[e] = s0 ? s0[n * NN + e] : 0.0;
            for (int64_t t = 0; t < T; ++t) {
                const double *kt = k + base + t * stride, *vt = v + base + t * stride;
                const double *wt = w + base + t * stride;
                const double *S = Sall + t * NN;
                double *Sn = Sall + (t + 1) * NN;
                for (int64_t i = 0; i < N; ++i)
                    for (int64_t j = 0; j < N; ++j) Sn[i * N + j] = kt[i] * vt[j] + wt[i] * S[i * N + j];
            }
            for (int64_t e = 0; e < NN; ++e) L[e] = dsT ? dsT[n * NN + e] : 0.0;
            for (int64_t t = T - 1; t >= 0; --t) {
                const int64_t o = base + t * stride;
                const double *rt = r + o, *kt = k + o, *vt = v + o, *wt = w + o, *gt = dy + o;
                const double *S = Sall + t * NN;
                for (int64_t i = 0; i < N; ++i) {
                    double a = 0.0, b = 0.0, c = 0.0, d = 0.0;
                    for (int64_t j = 0; j < N; ++j) {
                        a += gt[j] * (S[i * N + j] + uh[i] * kt[i] * vt[j]);
                        b += L[i * N + j] * vt[j] + gt[j] * rt[i] * uh[i] * vt[j];
                        c += L[i * N + j] * S[i * N + j];
                        d += gt[j] * rt[i] * kt[i] * vt[j];
                    }
                    dr[o + i] = a;
                    dk[o + i] = b;
                    dw[o + i] = c;
                    du[h * N + i] += d;
                }
                for (int64_t j = 0; j < N; ++j) {
                    double a = 0.0;
                    for (int64_t i = 0; i < N; ++i) a += L[i * N + j] * kt[i] + gt[j] * rt[i] * uh[i] * kt[i];
                    dv[o + j] = a;
                }
                for (int64_t i = 0; i < N; ++i)
                    for (int64_t j = 0; j < N; ++j) L[i * N + j] = wt[i] * L[i * N + j] + rt[i] * gt[j];
            }
            if (ds0)
                for (int64_t e = 0; e < NN; ++e) ds0[n * NN + e] = L[e];
        }
    }
}

/*
 * Chain rule through the decay map of oracle_decay_from_logit:
 * d/domega exp(-exp(omega)) = -exp(omega) exp(-exp(omega)), so
 * domega[i] = dw[i] * (-exp(omega[i]) * exp(-exp(omega[i]))).  n elements.
 */
void oracle_decay_from_logit_grad(int64_t n, const double *omega, const double *dw, double *domega)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        const double e = exp(omega[i]);
        domega[i] = dw[i] * (-e * exp(-e));
    }
}
