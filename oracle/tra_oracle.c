/*
 * tra_oracle.c -- plain, slow, fp64 CPU oracle for the Token Radius Attention
 * hot path (entropy, budget, radius, token mask, block mask, masked attention).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes
 * or calls this file; only the test-suite, the smoke check and the CPU
 * baseline leg of the benchmark do.  It shares no code, header, table or
 * helper with the CUDA path.
 *
 * Sources (page title, then the passage):
 *   [TRA]  "Token Radius Attention for Efficient Video Generation"
 *          (gist.science technical summary): section 2 "Methodologie",
 *          Intuition I (entropy -> token budget, B ~ tau*exp(H_i)/N),
 *          Intuition II (query-centred radius, temporal decay phi(delta)),
 *          "Le Pipeline TRA" (warm-up entropy, budget -> radius, tile-major
 *          layout, radius-mask -> block-sparse mask by token voting).
 *   [TLDR] "Token Radius Attention for Efficient Video Generation"
 *          (daily-ai-frontier TL;DR): entropy -> analytic budget ->
 *          temporally decayed radius; fused entropy extraction.
 *   [BLOG] "Token Radius Attention" blog post (qwbw.cn), sections 5.1 and 9.1:
 *          frame-major token order n = (t*H + h)*W + w.
 *
 * Readings taken where the pages are silent or loose (all listed in the
 * design notes of the repository):
 *   - entropy uses the natural log (exp(H) is then the effective key count,
 *     which is what tau*exp(H_i) needs);
 *   - the budget is B_i = min(N, max(Bmin, exp(a*H_i + b))), Bhat = ceil(B);
 *     tau*exp(H) is the case a = 1, b = ln(tau) (in tokens, not density);
 *   - temporal decay is gamma^|dt| (the family exp(-gamma' * dt) with
 *     gamma = exp(-gamma')), spatial test is Chebyshev distance
 *     <= floor(r * gamma^|dt| + 1e-9), keys limited to |dt| <= Rt;
 *   - counts are taken over in-grid keys only;
 *   - "token voting" is an OR vote: a tile pair is active iff any retained
 *     token pair lies in it;
 *   - subsampled entropy: plug-in entropy over the sampled keys + ln(N/|S|);
 *   - metric 1 (the summary's "circular neighbourhoods" / 2D disk mask): the
 *     spatial test is dh^2 + dw^2 <= s^2 with the same half-width s; the
 *     count then sums, row by row, the clipped width 2*isqrt(s^2 - dh^2) + 1,
 *     and r_cap is the smallest r with s(r, Rt')^2 >= (H-1)^2 + (W-1)^2.
 *
 * Build:  gcc -O2 -fopenmp -ffp-contract=off -fno-fast-math -shared -fPIC ... -lquadmath
 * (fp-contract=off keeps r*g and +1e-9 as two separately rounded operations;
 * libquadmath gives the budget's exponential in binary128).
 *
 * Layout of every per-token array: [heads][N][...] in natural order.
 * Element arrays are passed as `const void*` with a type flag: 0 = float32,
 * 1 = bfloat16 bit patterns (uint16), 2 = float64.  All arithmetic is fp64.
 */
#include <math.h>
#include <quadmath.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <omp.h>

#define EPS_S 1e-9

/* ------------------------------------------------------------------------ */
/* element access                                                            */
/* ------------------------------------------------------------------------ */

static double load_elem(const void* p, size_t i, int type)
{
    if (type == 0) return (double)((const float*)p)[i];
    if (type == 1) {
        uint32_t bits = ((uint32_t)((const uint16_t*)p)[i]) << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return (double)f;
    }
    return ((const double*)p)[i];
}

/* ------------------------------------------------------------------------ */
/* geometry: natural order n = (t*H + h)*W + w   ([BLOG] 5.1, 9.1)           */
/* ------------------------------------------------------------------------ */

typedef struct { int T, H, W; } grid_t;

static void coords(const grid_t* g, int64_t n, int* t, int* h, int* w)
{
    *w = (int)(n % g->W);
    *h = (int)((n / g->W) % g->H);
    *t = (int)(n / ((int64_t)g->W * g->H));
}

static int64_t imin64(int64_t a, int64_t b) { return a < b ? a : b; }
static int64_t imax64(int64_t a, int64_t b) { return a > b ? a : b; }

/* ------------------------------------------------------------------------ */
/* radius pieces  ([TRA] Intuition II, "Budget-vers-Rayon")                  */
/* ------------------------------------------------------------------------ */

/* decay table g[delta] = gamma^delta for delta = 0..Rt_eff */
void oracle_decay_table(double gamma, int Rt_eff, double* g_out)
{
    for (int d = 0; d <= Rt_eff; ++d) g_out[d] = pow(gamma, (double)d);
}

/* spatial half-width at radius r and frame distance with decay g:
   floor(r*g + 1e-9), the product and the sum each rounded once */
int64_t oracle_halfwidth(int64_t r, double g)
{
    volatile double prod = (double)r * g;
    volatile double sum = prod + EPS_S;
    return (int64_t)floor(sum);
}

/* Rt' = min(Rt, T-1) */
int oracle_rt_eff(int T, int Rt) { return Rt < T - 1 ? Rt : T - 1; }

/* r_cap: the smallest r whose farthest-frame half-width reaches the grid,
   s(r, Rt') >= max(H, W) - 1, so no larger radius adds keys. */
int64_t oracle_r_cap(int T, int H, int W, double gamma, int Rt, int metric)
{
    int rte = oracle_rt_eff(T, Rt);
    double g = pow(gamma, (double)rte);
    int64_t r = 0;
    if (metric == 1) {
        /* the farthest-frame disk must reach the opposite corner of the frame */
        int64_t need2 = (int64_t)(H - 1) * (H - 1) + (int64_t)(W - 1) * (W - 1);
        for (;;) {
            int64_t s = oracle_halfwidth(r, g);
            if (s * s >= need2) return r;
            ++r;
        }
    }
    int64_t need = (H > W ? H : W) - 1;
    while (oracle_halfwidth(r, g) < need) ++r;
    return r;
}

/* the largest integer x >= 0 with x*x <= n (n >= 0), by bisection */
static int64_t isqrt_floor(int64_t n)
{
    int64_t lo = 0, hi = 1;
    while (hi * hi <= n) hi *= 2;
    while (hi - lo > 1) {
        int64_t mid = (lo + hi) / 2;
        if (mid * mid <= n) lo = mid; else hi = mid;
    }
    return lo;
}

/* c_i(r): number of in-grid keys j with |t_i-t_j| <= Rt' and Chebyshev
   distance <= s(r, |t_i - t_j|), by the clipped-rectangle formula. */
int64_t oracle_count(int T, int H, int W, double gamma, int Rt,
                     int t, int h, int w, int64_t r, int metric)
{
    int rte = oracle_rt_eff(T, Rt);
    int64_t c = 0;
    for (int dt = -rte; dt <= rte; ++dt) {
        int tt = t + dt;
        if (tt < 0 || tt >= T) continue;
        int64_t s = oracle_halfwidth(r, pow(gamma, (double)(dt < 0 ? -dt : dt)));
        int64_t hl = imax64(0, h - s), hh = imin64(H - 1, h + s);
        if (metric == 1) {
            /* disk: each key row h' holds the keys with dw^2 <= s^2 - dh^2 */
            for (int64_t hk = hl; hk <= hh; ++hk) {
                int64_t dh = hk - h;
                int64_t half = isqrt_floor(s * s - dh * dh);
                c += imin64(W - 1, w + half) - imax64(0, w - half) + 1;
            }
        } else {
            int64_t wl = imax64(0, w - s), wh = imin64(W - 1, w + s);
            c += (hh - hl + 1) * (wh - wl + 1);
        }
    }
    return c;
}

/* E3: token budget from entropy ([TRA] Intuition I).  Hent is the fp32
   entropy promoted to fp64; x = a*H + b with a*H and +b rounded separately.
   Bhat = ceil(min(N, max(Bmin, e^x))) with e^x evaluated in 113-bit binary128
   (libquadmath), so the ceiling is the exact one: for a double x != 0, e^x
   is irrational and lies farther than 2^-113 relative from every integer in
   practice, while an fp64 exponential can land on the wrong side of an
   integer it is within a few ulps of (e.g. a = 0, b = ln k).  One case is
   below binary128's resolution: for 0 < x < 2^-113, e^x = 1 + x + ... rounds
   to 1, while e^x > 1 for every x > 0, so its ceiling is 2.  x = NaN gives
   Bmin. */
int64_t oracle_budget(float Hent, double a, double b, int64_t N, int64_t Bmin)
{
    volatile double ah = a * (double)Hent;
    volatile double x = ah + b;
    if (isnan(x)) return Bmin;
    __float128 c = ceilq(expq((__float128)x));
    if (x > 0 && c < 2) c = 2;
    if (c < (__float128)Bmin) c = (__float128)Bmin;
    if (c > (__float128)N) c = (__float128)N;
    return (int64_t)c;
}

/* E3 + E4 per (head, token).  Hent[row] is the fp32 entropy of query
   queries[row] (a head-major index g*N + n; NULL = all G*N in order).
   Writes r_out[row], c_out[row] = c_i(r_i) and bhat_out[row] = ceil(B_i).
   r_i = the smallest r in [0, r_cap] with c_i(r) >= Bhat_i, found by a
   linear scan upward from 0 (the definition), else r_cap. */
void oracle_radius(const float* Hent, int G, int T, int H, int W,
                   double a, double b, double gamma, int Rt, int Bmin, int metric,
                   const int64_t* queries, int64_t n_queries,
                   int32_t* r_out, int64_t* c_out, int64_t* bhat_out)
{
    grid_t gr = {T, H, W};
    int64_t N = (int64_t)T * H * W;
    int64_t rcap = oracle_r_cap(T, H, W, gamma, Rt, metric);
    int64_t rows = queries ? n_queries : (int64_t)G * N;
    #pragma omp parallel for schedule(dynamic, 64)
    for (int64_t row = 0; row < rows; ++row) {
        int64_t gi = queries ? queries[row] : row;
        int t, h, w;
        coords(&gr, gi % N, &t, &h, &w);
        int64_t bh = oracle_budget(Hent[row], a, b, N, Bmin);
        int64_t r = 0, c = oracle_count(T, H, W, gamma, Rt, t, h, w, 0, metric);
        while (c < bh && r < rcap) {
            ++r;
            c = oracle_count(T, H, W, gamma, Rt, t, h, w, r, metric);
        }
        r_out[row] = (int32_t)r;
        if (c_out) c_out[row] = c;
        if (bhat_out) bhat_out[row] = bh;
    }
}

/* E5: token mask M_ij given the query's radius ([TRA] "Budget-vers-Rayon") */
static int token_mask(const grid_t* gr, double gamma, int rte, int metric,
                      int64_t i, int64_t j, int64_t r_i)
{
    int ti, hi, wi, tj, hj, wj;
    coords(gr, i, &ti, &hi, &wi);
    coords(gr, j, &tj, &hj, &wj);
    int dt = ti > tj ? ti - tj : tj - ti;
    if (dt > rte) return 0;
    int64_t s = oracle_halfwidth(r_i, pow(gamma, (double)dt));
    int64_t dh = hi > hj ? hi - hj : hj - hi;
    int64_t dw = wi > wj ? wi - wj : wj - wi;
    if (metric == 1) return dh * dh + dw * dw <= s * s;    /* disk */
    int64_t cheb = dh > dw ? dh : dw;
    return cheb <= s;
}

int oracle_token_mask(int T, int H, int W, double gamma, int Rt, int metric,
                      int64_t i, int64_t j, int64_t r_i)
{
    grid_t gr = {T, H, W};
    return token_mask(&gr, gamma, oracle_rt_eff(T, Rt), metric, i, j, r_i);
}

/* ------------------------------------------------------------------------ */
/* E6: block mask over tiles of the tile-major layout ([TRA] "Disposition    */
/* Tile-Major" and "Noyaux CUDA Fusionnes": distance, radius comparison,     */
/* block pruning and token voting).                                          */
/*                                                                           */
/* Query tiles are (1, qth, qtw) boxes, key tiles (1, kth, ktw) boxes of the */
/* T x H x W grid; tile index = (t*nTh + h/th)*nTw + w/tw.  For each listed  */
/* query tile and every key tile: out = 0 inactive, 1 active (some valid     */
/* retained pair), 3 active and full (every valid pair retained).            */
/* ------------------------------------------------------------------------ */
void oracle_block_mask(const int32_t* r, int G, int T, int H, int W,
                       double gamma, int Rt, int metric,
                       int qth, int qtw, int kth, int ktw,
                       const int64_t* qtiles, int64_t n_qtiles,
                       uint8_t* out)
{
    grid_t gr = {T, H, W};
    int rte = oracle_rt_eff(T, Rt);
    int64_t N = (int64_t)T * H * W;
    int qnTh = (H + qth - 1) / qth, qnTw = (W + qtw - 1) / qtw;
    int knTh = (H + kth - 1) / kth, knTw = (W + ktw - 1) / ktw;
    int64_t nQ = (int64_t)T * qnTh * qnTw, nK = (int64_t)T * knTh * knTw;
    int64_t rows = qtiles ? n_qtiles : (int64_t)G * nQ;

    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t row = 0; row < rows; ++row) {
        int64_t gq = qtiles ? qtiles[row] : row;       /* g*nQ + a */
        int64_t g = gq / nQ, a = gq % nQ;
        int at = (int)(a / ((int64_t)qnTh * qnTw));
        int ah = (int)((a / qnTw) % qnTh), aw = (int)(a % qnTw);
        for (int64_t kb = 0; kb < nK; ++kb) {
            int bt = (int)(kb / ((int64_t)knTh * knTw));
            int bh = (int)((kb / knTw) % knTh), bw = (int)(kb % knTw);
            int any = 0, all = 1;
            for (int ih = 0; ih < qth; ++ih) for (int iw = 0; iw < qtw; ++iw) {
                int hi = ah * qth + ih, wi = aw * qtw + iw;
                if (hi >= H || wi >= W) continue;
                int64_t i = ((int64_t)at * H + hi) * W + wi;
                for (int jh = 0; jh < kth; ++jh) for (int jw = 0; jw < ktw; ++jw) {
                    int hj = bh * kth + jh, wj = bw * ktw + jw;
                    if (hj >= H || wj >= W) continue;
                    int64_t j = ((int64_t)bt * H + hj) * W + wj;
                    if (token_mask(&gr, gamma, rte, metric, i, j, r[g * N + i])) any = 1;
                    else all = 0;
                }
            }
            out[row * nK + kb] = (uint8_t)(any ? (all ? 3 : 1) : 0);
        }
    }
}

/* Block mask of explicit query sets (the radius-sorted query groups of the  */
/* library's TRA_FLAG_QSORT plans): set s holds the queries                  */
/* members[s*set_size .. s*set_size + set_size) as g*N + n (-1: no query).   */
/* For every key tile of the query set's head: 0 inactive, 1 active (some    */
/* member keeps some valid key of it), 3 active and full (every member keeps */
/* every valid key of it).  A set without members is all 0.  All members of */
/* a set belong to one head.                                                 */
void oracle_block_mask_sets(const int32_t* r, int G, int T, int H, int W,
                            double gamma, int Rt, int metric, int kth, int ktw,
                            const int64_t* members, int64_t n_sets, int set_size,
                            uint8_t* out)
{
    grid_t gr = {T, H, W};
    int rte = oracle_rt_eff(T, Rt);
    int64_t N = (int64_t)T * H * W;
    int knTh = (H + kth - 1) / kth, knTw = (W + ktw - 1) / ktw;
    int64_t nK = (int64_t)T * knTh * knTw;
    (void)G;

    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t set = 0; set < n_sets; ++set) {
        const int64_t* mem = members + set * set_size;
        for (int64_t kb = 0; kb < nK; ++kb) {
            int bt = (int)(kb / ((int64_t)knTh * knTw));
            int bh = (int)((kb / knTw) % knTh), bw = (int)(kb % knTw);
            int any = 0, all = 1, some = 0;
            for (int m = 0; m < set_size; ++m) {
                int64_t gi = mem[m];
                if (gi < 0) continue;
                some = 1;
                int64_t g = gi / N, i = gi % N;
                for (int jh = 0; jh < kth; ++jh) for (int jw = 0; jw < ktw; ++jw) {
                    int hj = bh * kth + jh, wj = bw * ktw + jw;
                    if (hj >= H || wj >= W) continue;
                    int64_t j = ((int64_t)bt * H + hj) * W + wj;
                    if (token_mask(&gr, gamma, rte, metric, i, j, r[g * N + i])) any = 1;
                    else all = 0;
                }
            }
            out[set * nK + kb] = (uint8_t)(some && any ? (all ? 3 : 1) : 0);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* E1 / E2: per-query softmax entropy ([TRA] Intuition I, "Entropie-vers-    */
/* Budget"; [TLDR] fused entropy extraction).                                */
/*   s_j = q.k_j / sqrt(d);  H = ln Z - (sum_j e^{s_j-m}(s_j-m)) / Z,        */
/*   Z = sum_j e^{s_j-m}, m = max_j s_j  (equal to -sum p ln p).             */
/* key_stride = 1: all N keys.  key_stride > 1: only valid keys of key tiles */
/* (1, kth, ktw) whose tile index is a multiple of key_stride, and the       */
/* result gets + ln(N / |S|).  queries: NULL = all, else G*N-indexed list.   */
/* ------------------------------------------------------------------------ */
void oracle_entropy(const void* q, const void* k, int type,
                    int G, int T, int H, int W, int d,
                    int key_stride, int kth, int ktw,
                    const int64_t* queries, int64_t n_queries, double* H_out)
{
    grid_t gr = {T, H, W};
    int64_t N = (int64_t)T * H * W;
    int knTh = (H + kth - 1) / kth, knTw = (W + ktw - 1) / ktw;
    double sigma = 1.0 / sqrt((double)d);

    /* the sampled key set S (natural indices) */
    int64_t* keys = (int64_t*)malloc(sizeof(int64_t) * (size_t)N);
    int64_t nS = 0;
    for (int64_t j = 0; j < N; ++j) {
        int t, h, w;
        coords(&gr, j, &t, &h, &w);
        int64_t tile = ((int64_t)t * knTh + h / kth) * knTw + w / ktw;
        if (key_stride <= 1 || tile % key_stride == 0) keys[nS++] = j;
    }
    double corr = key_stride <= 1 ? 0.0 : log((double)N / (double)nS);
    int64_t rows = queries ? n_queries : (int64_t)G * N;

    #pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)nS);
        #pragma omp for schedule(dynamic, 16)
        for (int64_t row = 0; row < rows; ++row) {
            int64_t gi = queries ? queries[row] : row;
            int64_t g = gi / N;
            double m = -INFINITY;
            for (int64_t u = 0; u < nS; ++u) {
                int64_t j = keys[u];
                double acc = 0.0;
                for (int c = 0; c < d; ++c)
                    acc += load_elem(q, (size_t)gi * d + c, type)
                         * load_elem(k, ((size_t)(g * N + j)) * d + c, type);
                s[u] = acc * sigma;
                if (s[u] > m) m = s[u];
            }
            double Z = 0.0, S = 0.0;
            for (int64_t u = 0; u < nS; ++u) {
                double e = exp(s[u] - m);
                Z += e;
                S += e * (s[u] - m);
            }
            H_out[row] = log(Z) - S / Z + corr;
        }
        free(s);
    }
    free(keys);
}

/* ------------------------------------------------------------------------ */
/* E7: attention restricted to the token mask ([TRA] "Budget-vers-Rayon",    */
/* "Execution Efficace"): O_i = sum_{j in M_i} softmax_j(q_i.k_j/sqrt d) v_j */
/* out: [rows][d] fp64 for the listed queries (NULL = all G*N).              */
/* ------------------------------------------------------------------------ */
void oracle_attention(const void* q, const void* k, const void* v, int type,
                      const int32_t* r, int G, int T, int H, int W, int d,
                      double gamma, int Rt, int metric,
                      const int64_t* queries, int64_t n_queries, double* out)
{
    grid_t gr = {T, H, W};
    int rte = oracle_rt_eff(T, Rt);
    int64_t N = (int64_t)T * H * W;
    double sigma = 1.0 / sqrt((double)d);
    int64_t rows = queries ? n_queries : (int64_t)G * N;

    #pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)N);
        #pragma omp for schedule(dynamic, 16)
        for (int64_t row = 0; row < rows; ++row) {
            int64_t gi = queries ? queries[row] : row;
            int64_t g = gi / N, i = gi % N;
            double m = -INFINITY;
            for (int64_t j = 0; j < N; ++j) {
                if (!token_mask(&gr, gamma, rte, metric, i, j, r[gi])) { s[j] = -INFINITY; continue; }
                double acc = 0.0;
                for (int c = 0; c < d; ++c)
                    acc += load_elem(q, (size_t)gi * d + c, type)
                         * load_elem(k, ((size_t)(g * N + j)) * d + c, type);
                s[j] = acc * sigma;
                if (s[j] > m) m = s[j];
            }
            double Z = 0.0;
            double* o = out + (size_t)row * d;
            for (int c = 0; c < d; ++c) o[c] = 0.0;
            for (int64_t j = 0; j < N; ++j) {
                if (s[j] == -INFINITY) continue;
                double e = exp(s[j] - m);
                Z += e;
                for (int c = 0; c < d; ++c)
                    o[c] += e * load_elem(v, ((size_t)(g * N + j)) * d + c, type);
            }
            for (int c = 0; c < d; ++c) o[c] /= Z;
        }
        free(s);
    }
}

/* ------------------------------------------------------------------------ */
/* Calibration ([TRA] Intuition I: the key density a query needs follows its */
/* entropy): k_i(mass) = the smallest k whose k largest dense softmax       */
/* probabilities sum to at least mass, by an exact sort of the fp64          */
/* probabilities.  queries: NULL = all G*N, else G*N-indexed list.           */
/* ------------------------------------------------------------------------ */
static int cmp_desc(const void* a, const void* b)
{
    double x = *(const double*)a, y = *(const double*)b;
    return x < y ? 1 : (x > y ? -1 : 0);
}

void oracle_topk_count(const void* q, const void* k, int type, int G, int T, int H, int W, int d,
                       double mass, const int64_t* queries, int64_t n_queries, int64_t* k_out)
{
    int64_t N = (int64_t)T * H * W;
    double sigma = 1.0 / sqrt((double)d);
    int64_t rows = queries ? n_queries : (int64_t)G * N;
    (void)G;
    #pragma omp parallel
    {
        double* p = (double*)malloc(sizeof(double) * (size_t)N);
        #pragma omp for schedule(dynamic, 16)
        for (int64_t row = 0; row < rows; ++row) {
            int64_t gi = queries ? queries[row] : row;
            int64_t g = gi / N;
            double m = -INFINITY;
            for (int64_t j = 0; j < N; ++j) {
                double acc = 0.0;
                for (int c = 0; c < d; ++c)
                    acc += load_elem(q, (size_t)gi * d + c, type)
                         * load_elem(k, ((size_t)(g * N + j)) * d + c, type);
                p[j] = acc * sigma;
                if (p[j] > m) m = p[j];
            }
            double Z = 0.0;
            for (int64_t j = 0; j < N; ++j) { p[j] = exp(p[j] - m); Z += p[j]; }
            for (int64_t j = 0; j < N; ++j) p[j] /= Z;
            qsort(p, (size_t)N, sizeof(double), cmp_desc);
            double cum = 0.0;
            int64_t kk = N;
            for (int64_t j = 0; j < N; ++j) {
                cum += p[j];
                if (cum >= mass) { kk = j + 1; break; }
            }
            k_out[row] = kk;
        }
        free(p);
    }
}

/* ------------------------------------------------------------------------ */
/* Calibration fit ([TRA] Intuition I: the number of keys a query needs      */
/* grows log-linearly with its entropy, B ~ tau*exp(H_i), i.e. ln B is       */
/* linear in H with slope 1 and intercept ln tau; the fit generalises the    */
/* slope to a).  Ordinary least squares of y = ln k_i on x = H_i,            */
/*   ln k = a*H + b,                                                         */
/* over the rows with k_i >= 1 and a finite H_i, in two passes: the means,   */
/* then the centred sums  a = S_xy / S_xx,  b = mean(y) - a*mean(x).         */
/* r2_out (optional) = S_xy^2 / (S_xx * S_yy), the share of the variance of  */
/* ln k the line explains.  Returns the number of rows used, or -1 (nothing  */
/* written) when fewer than two rows are usable or their H are all equal.    */
/* ------------------------------------------------------------------------ */
static double fit_y(int64_t k) { return log((double)k); }

int64_t oracle_fit_log_linear(const double* H, const int64_t* k, int64_t n,
                              double* a_out, double* b_out, double* r2_out)
{
    int64_t m = 0;
    double sx = 0.0, sy = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        if (k[i] < 1 || !isfinite(H[i])) continue;
        ++m;
        sx += H[i];
        sy += fit_y(k[i]);
    }
    if (m < 2) return -1;
    double mx = sx / (double)m, my = sy / (double)m;
    double sxx = 0.0, sxy = 0.0, syy = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        if (k[i] < 1 || !isfinite(H[i])) continue;
        double dx = H[i] - mx, dy = fit_y(k[i]) - my;
        sxx += dx * dx;
        sxy += dx * dy;
        syy += dy * dy;
    }
    if (!(sxx > 0.0)) return -1;
    *a_out = sxy / sxx;
    *b_out = my - *a_out * mx;
    if (r2_out) *r2_out = syy > 0.0 ? (sxy * sxy) / (sxx * syy) : 1.0;
    return m;
}

/* threads the OpenMP runtime will use (for the reported CPU baseline) */
int oracle_num_threads(void)
{
    int n = 1;
    #pragma omp parallel
    {
        #pragma omp single
        n = omp_get_num_threads();
    }
    return n;
}
