/*
 * na_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, fp64 CPU definition of the forward pass of multi-dimensional
 * local ("generalized neighborhood" / "sliding tile") attention.  Only the
 * tests, the package's smoke check and the benchmark's CPU-baseline leg may
 * load this library; the product path never does.  It shares no code with the
 * CUDA path: its window rule, mask, softmax and block counting are written
 * here from the pages and from nothing else.
 *
 * What it computes, per (batch*head bh, query token i):
 *   z_ij  = scale * <q_i, k_j>           for every key j in the window of i
 *   m     = max_j z_ij
 *   l     = sum_j exp(z_ij - m)
 *   out_i = sum_j exp(z_ij - m) v_j / l
 *   lse_i = m + ln l
 * following "pi-Attention: Online Efficient Sparse Transformers for
 * Long-Context Modeling", section 3.1 eqs. (1)-(3) (softmax(QK^T/sqrt(d_k))V,
 * a weighted sum of values) and section 3.2 eq. (4) (pre-softmax score z_ij)
 * with the sum restricted to the neighbourhood (text after eq. (5)).  The
 * restriction is evaluated as a dense mask over all N keys of the row, the
 * convention stated under eq. (34) of the same page (invalid positions get
 * -inf before the softmax, which is the same as restricting the sum); the
 * arithmetic is only done where the mask is true, which is identical because
 * exp(-inf) = 0.
 *
 * Window rule (per grid dimension, window w, stride s, length L):
 *   g     = floor(i / s)                 stride group of coordinate i
 *   c     = g*s + floor(s/2)             the group's centre ("leader")
 *   start = clamp(c - floor(w/2), 0, L - w)
 *   window = [start, start + w)
 * and the N-d window is the Cartesian product over dimensions.  Sources:
 * "Generalized Neighborhood Attention: Multi-dimensional Sparse Attention at
 * the Speed of Light" (abstract: one family covering sliding window, strided
 * sliding window and blocked attention); "ENA: Efficient N-dimensional
 * Attention" (the pith, "What carries the argument": tokens within one tile
 * share a window that shifts tile by tile).  The pages print no formula; the
 * reading used here (a window centred on the query's stride group and clamped
 * inside the grid, so that every query sees exactly prod(w) keys) is the
 * plainest one consistent with both pages.
 *
 * Window modes (chosen per grid dimension; the rule above is "clamped"):
 *   truncated  the clamped rule's window taken before the clamp and cut to
 *              the grid: [c - floor(w/2), c - floor(w/2) + w) intersected
 *              with [0, L).  With s = 1 and w = 2k + 1 this is the
 *              bidirectional neighbourhood {j : |j - i| <= k} of
 *              "pi-Attention", section 3.2 eq. (5); queries near a border see
 *              fewer keys instead of a shifted window.
 *   causal     the w positions ending with the last position of the query's
 *              stride group, cut to the grid: [(g+1)*s - w, (g+1)*s)
 *              intersected with [0, L).  With s = 1 and w = k + 1 this is the
 *              causal neighbourhood {j : max(0, i - k) <= j <= i} of eq. (5)
 *              (self included, as the text after eq. (5) states).  For s > 1
 *              every query of a group sees the whole group (block causal).
 *   Eq. (5) has no stride; the stride readings above are this oracle's
 *   (truncated: the same centring as the clamped rule; causal: the group as
 *   the unit of causality) and coincide with eq. (5) at s = 1.
 *
 * Dilation (per grid dimension, dil >= 1): the pages name dilated patterns
 * only as related work ("pi-Attention", section 2: "strided/dilated
 * patterns") and define none.  The reading here is the plainest one that
 * keeps the rules above intact: coordinates split into dil interleaved
 * sub-sequences by residue r = i mod dil; sub-sequence r holds the
 * Lr = ceil((L - r) / dil) coordinates r, r + dil, r + 2 dil, ...; a query
 * at i = r + dil * p takes the window [lo, hi) of position p inside its
 * sub-sequence (any mode, stride in sub-sequence positions) and attends to
 * the keys r + dil * t for t in [lo, hi).  dil = 1 is the undilated rule;
 * clamped windows need w <= Lr for every r, i.e. w * dil <= L.
 *
 * Backward (the gradients of the forward pass for an upstream gradient dO of
 * out): the pages give only the forward; the gradients here are its
 * vector-Jacobian product written out with P_ij = exp(z_ij - lse_i) over the
 * same windows:
 *   dV_j  = sum_{i : j in W(i)} P_ij dO_i
 *   dP_ij = <dO_i, v_j>,  D_i = sum_j P_ij dP_ij  (= <dO_i, out_i>)
 *   dZ_ij = P_ij (dP_ij - D_i)
 *   dQ_i  = scale * sum_j dZ_ij k_j,   dK_j = scale * sum_{i : j in W(i)} dZ_ij q_i
 *
 * Block counting (empty / partial / full tiles of the N x N attention map in
 * row-major token order) follows "Hilbert-Guided Sparse Local Attention",
 * "Methodology in Plain English" (tiles labelled full, partial or empty).
 *
 * Inputs are read as the exact float32 values, the exact bfloat16 values
 * (16-bit patterns widened by a shift) or the exact IEEE 754 binary16 values
 * (decoded below from the format's definition) that the GPU receives.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define NA_ORACLE_MAXDIM 3

enum { IN_F32 = 0, IN_BF16 = 1, IN_F16 = 2, IN_E4M3 = 3 };
enum { WIN_CLAMPED = 0, WIN_TRUNCATED = 1, WIN_CAUSAL = 2 };

/* ---------------------------------------------------------------- window -- */

int na_oracle_window_start(int L, int w, int s, int i) {
    if (L < 1 || w < 1 || w > L || s < 1 || s > w || i < 0 || i >= L) return -1;
    int g = i / s;
    int c = g * s + s / 2;
    int start = c - w / 2;
    if (start < 0) start = 0;
    if (start > L - w) start = L - w;
    return start;
}

/*
 * Window of coordinate i in one dimension as the half-open range [*lo, *hi),
 * for mode WIN_CLAMPED, WIN_TRUNCATED or WIN_CAUSAL (definitions above).
 */
int na_oracle_window(int L, int w, int s, int mode, int i, int* lo, int* hi) {
    if (L < 1 || w < 1 || w > L || s < 1 || s > w || i < 0 || i >= L || !lo || !hi) return -1;
    if (mode == WIN_CLAMPED) {
        *lo = na_oracle_window_start(L, w, s, i);
        *hi = *lo + w;
        return 0;
    }
    int g = i / s;
    int a;
    if (mode == WIN_TRUNCATED)
        a = g * s + s / 2 - w / 2;
    else if (mode == WIN_CAUSAL)
        a = (g + 1) * s - w;
    else
        return -1;
    *lo = a < 0 ? 0 : a;
    *hi = a + w > L ? L : a + w;
    return 0;
}

/*
 * Dilated window of coordinate i in one dimension: the keys r + dil * t for
 * t in [*lo, *hi), with *r = i mod dil (definition above).
 */
int na_oracle_dilated_window(int L, int w, int s, int mode, int dil, int i, int* r, int* lo,
                             int* hi) {
    if (dil < 1 || L < 1 || i < 0 || i >= L || !r || !lo || !hi) return -1;
    const int res = i % dil;
    const int Lr = (L - res + dil - 1) / dil;      /* coordinates res, res + dil, ... below L */
    if (w > L / dil) return -1;                    /* every sub-sequence holds the window */
    *r = res;
    return na_oracle_window(Lr, w, s, mode, i / dil, lo, hi);
}

static int check_geometry(int ndim, const int* L, const int* w, const int* s, const int* mode,
                          const int* dil, long long* N) {
    if (ndim < 1 || ndim > NA_ORACLE_MAXDIM || !L || !w || !s) return -1;
    long long n = 1;
    for (int a = 0; a < ndim; ++a) {
        if (L[a] < 1 || w[a] < 1 || w[a] > L[a] || s[a] < 1 || s[a] > w[a]) return -1;
        if (mode && (mode[a] < WIN_CLAMPED || mode[a] > WIN_CAUSAL)) return -1;
        if (dil && (dil[a] < 1 || (long long)w[a] * dil[a] > L[a])) return -1;
        n *= L[a];
    }
    *N = n;
    return 0;
}

static void unflatten(long long t, int ndim, const int* L, int* coord) {
    for (int a = ndim - 1; a >= 0; --a) {
        coord[a] = (int)(t % L[a]);
        t /= L[a];
    }
}

/*
 * Dense membership row: mask[j] = 1 iff key token j is in the window of query
 * token t.  mode: per-dimension window modes, NULL = all clamped; dil:
 * per-dimension dilation, NULL = all 1.  Returns the number of keys in the
 * window (> 0), or -1 on invalid input.
 */
long long na_oracle_mask_row_dil(int ndim, const int* L, const int* w, const int* s,
                                 const int* mode, const int* dil, long long t, uint8_t* mask) {
    long long N;
    if (check_geometry(ndim, L, w, s, mode, dil, &N) || t < 0 || t >= N || !mask) return -1;
    int qi[NA_ORACLE_MAXDIM], lo[NA_ORACLE_MAXDIM], hi[NA_ORACLE_MAXDIM], kj[NA_ORACLE_MAXDIM];
    int res[NA_ORACLE_MAXDIM], step[NA_ORACLE_MAXDIM];
    unflatten(t, ndim, L, qi);
    for (int a = 0; a < ndim; ++a) {
        step[a] = dil ? dil[a] : 1;
        na_oracle_dilated_window(L[a], w[a], s[a], mode ? mode[a] : WIN_CLAMPED, step[a], qi[a],
                                 &res[a], &lo[a], &hi[a]);
    }
    for (int a = 0; a < ndim; ++a) kj[a] = 0;
    long long count = 0;
    for (long long j = 0; j < N; ++j) {
        int in = 1;
        for (int a = 0; a < ndim; ++a) {
            /* key coordinate kj = res + step * u with u in [lo, hi) */
            if (kj[a] % step[a] != res[a]) in = 0;
            const int u = kj[a] / step[a];
            if (u < lo[a] || u >= hi[a]) in = 0;
        }
        count += in;
        mask[j] = (uint8_t)in;
        for (int a = ndim - 1; a >= 0; --a) { /* advance the row-major key counter */
            if (++kj[a] < L[a]) break;
            kj[a] = 0;
        }
    }
    return count;
}

long long na_oracle_mask_row(int ndim, const int* L, const int* w, const int* s, const int* mode,
                             long long t, uint8_t* mask) {
    return na_oracle_mask_row_dil(ndim, L, w, s, mode, NULL, t, mask);
}

/* --------------------------------------------------------------- forward -- */

/*
 * Value of an IEEE 754 binary16 bit pattern: sign bit, 5-bit exponent field e
 * (bias 15), 10-bit fraction f.  e = 0: subnormal f * 2^-24; e = 31: infinity
 * (f = 0) or NaN; otherwise (1024 + f) * 2^(e - 25) = (1 + f/1024) * 2^(e - 15).
 */
double na_oracle_f16_value(uint16_t h) {
    const int e = (h >> 10) & 0x1f, f = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + f), e - 25);
    return (h & 0x8000) ? -v : v;
}

/*
 * Value of an OFP8 E4M3 bit pattern ("OCP 8-bit Floating Point
 * Specification", E4M3 encoding): sign bit, 4-bit exponent field e (bias 7),
 * 3-bit mantissa m.  e = 0: subnormal m * 2^-9; e = 15 with m = 7: NaN (the
 * format has no infinities); otherwise (8 + m) * 2^(e - 10) = (1 + m/8) * 2^(e - 7).
 */
double na_oracle_e4m3_value(uint8_t b) {
    const int e = (b >> 3) & 0xf, m = b & 0x7;
    double v;
    if (e == 0)
        v = ldexp((double)m, -9);
    else if (e == 15 && m == 7)
        v = NAN;
    else
        v = ldexp((double)(8 + m), e - 10);
    return (b & 0x80) ? -v : v;
}

static inline double load_in(const void* p, int dtype, size_t idx) {
    if (dtype == IN_F32) return (double)((const float*)p)[idx];
    if (dtype == IN_F16) return na_oracle_f16_value(((const uint16_t*)p)[idx]);
    if (dtype == IN_E4M3) return na_oracle_e4m3_value(((const uint8_t*)p)[idx]);
    uint32_t bits = (uint32_t)((const uint16_t*)p)[idx] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

typedef struct {
    const void *q, *k, *v;
    int dtype, ndim, d;
    const int *L, *w, *s, *mode;
    long long N, BH, W;
    double scale;
    const long long* rows;
    long long r_begin, r_end;
    double *out, *lse;
    const int* dil;
    int status;
} fwd_job;

static void* fwd_worker(void* arg) {
    fwd_job* J = (fwd_job*)arg;
    const int ndim = J->ndim, d = J->d;
    const long long N = J->N;
    double* z = (double*)malloc(sizeof(double) * (size_t)J->W);
    long long* idx = (long long*)malloc(sizeof(long long) * (size_t)J->W);
    uint8_t* mask = (uint8_t*)malloc((size_t)N);
    double* acc = (double*)malloc(sizeof(double) * (size_t)d);
    if (!z || !idx || !mask || !acc) {
        J->status = -2;
        goto done;
    }
    for (long long r = J->r_begin; r < J->r_end; ++r) {
        long long row = J->rows ? J->rows[r] : r;
        if (row < 0 || row >= J->BH * N) { J->status = -1; break; }
        long long bh = row / N, t = row % N;
        const long long inwin =
            na_oracle_mask_row_dil(ndim, J->L, J->w, J->s, J->mode, J->dil, t, mask);
        size_t qoff = (size_t)row * (size_t)d;
        long long cnt = 0;
        for (long long j = 0; j < N; ++j) {
            if (!mask[j]) continue;
            if (cnt >= J->W) { J->status = -3; goto done; }
            size_t koff = ((size_t)bh * (size_t)N + (size_t)j) * (size_t)d;
            double dot = 0.0;
            for (int c = 0; c < d; ++c)
                dot += load_in(J->q, J->dtype, qoff + c) * load_in(J->k, J->dtype, koff + c);
            z[cnt] = J->scale * dot;
            idx[cnt] = j;
            ++cnt;
        }
        /* clamped windows hold exactly prod(w) keys; every window at least one */
        if (cnt != inwin || cnt < 1 || (!J->mode && cnt != J->W)) { J->status = -3; goto done; }
        double m = -INFINITY;
        for (long long e = 0; e < cnt; ++e) if (z[e] > m) m = z[e];
        double l = 0.0;
        for (long long e = 0; e < cnt; ++e) l += exp(z[e] - m);
        for (int c = 0; c < d; ++c) acc[c] = 0.0;
        for (long long e = 0; e < cnt; ++e) {
            double p = exp(z[e] - m) / l;
            size_t voff = ((size_t)bh * (size_t)N + (size_t)idx[e]) * (size_t)d;
            for (int c = 0; c < d; ++c) acc[c] += p * load_in(J->v, J->dtype, voff + c);
        }
        for (int c = 0; c < d; ++c) J->out[(size_t)r * (size_t)d + c] = acc[c];
        J->lse[r] = m + log(l);
    }
done:
    free(z);
    free(idx);
    free(mask);
    free(acc);
    return NULL;
}

/*
 * q, k, v: [BH, N, d] with the N tokens in row-major grid order (last grid
 * dimension fastest), float32 (in_dtype 0), bfloat16 bit patterns (1) or
 * binary16 bit patterns (2).
 * mode: per-dimension window modes (WIN_*), or NULL for all clamped.
 * rows: NULL for every row 0..BH*N-1 (then nrows must be BH*N), else a list
 * of global row indices bh*N + token.  out: [nrows, d] fp64; lse: [nrows] fp64.
 * scale <= 0 means 1/sqrt(d).  Returns 0, or a negative code on bad input
 * (-1), allocation failure (-2) or a window whose key count is inconsistent (-3).
 */
int na_oracle_forward_dil(const void* q, const void* k, const void* v, int in_dtype, long long BH,
                          int ndim, const int* L, const int* w, const int* s, const int* mode,
                          const int* dil, int d, double scale, const long long* rows,
                          long long nrows, double* out, double* lse, int nthreads) {
    long long N;
    if (!q || !k || !v || !out || !lse || BH < 1 || d < 1 || nrows < 0) return -1;
    if (in_dtype < IN_F32 || in_dtype > IN_E4M3) return -1;
    if (check_geometry(ndim, L, w, s, mode, dil, &N)) return -1;
    if (!rows && nrows != BH * N) return -1;
    long long W = 1;
    for (int a = 0; a < ndim; ++a) W *= w[a];
    if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (nthreads > nrows) nthreads = (int)(nrows > 0 ? nrows : 1);
    fwd_job jobs[256];
    pthread_t th[256];
    long long per = (nrows + nthreads - 1) / nthreads;
    for (int t = 0; t < nthreads; ++t) {
        fwd_job* J = &jobs[t];
        J->q = q; J->k = k; J->v = v;
        J->dtype = in_dtype; J->ndim = ndim; J->d = d;
        J->L = L; J->w = w; J->s = s; J->mode = mode;
        J->N = N; J->BH = BH; J->W = W;
        J->scale = scale;
        J->rows = rows;
        J->r_begin = per * t < nrows ? per * t : nrows;
        J->r_end = per * (t + 1) < nrows ? per * (t + 1) : nrows;
        J->out = out; J->lse = lse;
        J->dil = dil;
        J->status = 0;
    }
    for (int t = 1; t < nthreads; ++t)
        if (pthread_create(&th[t], NULL, fwd_worker, &jobs[t]) != 0) {
            fwd_worker(&jobs[t]);
            th[t] = 0;
        }
    fwd_worker(&jobs[0]);
    for (int t = 1; t < nthreads; ++t)
        if (th[t]) pthread_join(th[t], NULL);
    for (int t = 0; t < nthreads; ++t)
        if (jobs[t].status) return jobs[t].status;
    return 0;
}

int na_oracle_forward(const void* q, const void* k, const void* v, int in_dtype, long long BH,
                      int ndim, const int* L, const int* w, const int* s, const int* mode, int d,
                      double scale, const long long* rows, long long nrows, double* out,
                      double* lse, int nthreads) {
    return na_oracle_forward_dil(q, k, v, in_dtype, BH, ndim, L, w, s, mode, NULL, d, scale, rows,
                                 nrows, out, lse, nthreads);
}

/* -------------------------------------------------------------- backward -- */

typedef struct {
    const void *q, *k, *v, *dout;
    int dtype, ndim, d;
    const int *L, *w, *s, *mode;
    long long N, W;
    double scale;
    long long bh_begin, bh_end;
    double *dq, *dk, *dv;
    const int* dil;
    int status;
} bwd_job;

static void* bwd_worker(void* arg) {
    bwd_job* J = (bwd_job*)arg;
    const int d = J->d;
    const long long N = J->N;
    double* z = (double*)malloc(sizeof(double) * (size_t)J->W);
    long long* idx = (long long*)malloc(sizeof(long long) * (size_t)J->W);
    uint8_t* mask = (uint8_t*)malloc((size_t)N);
    double* o = (double*)malloc(sizeof(double) * (size_t)d);
    double* g = (double*)malloc(sizeof(double) * (size_t)d);
    if (!z || !idx || !mask || !o || !g) { J->status = -2; goto done; }
    for (long long bh = J->bh_begin; bh < J->bh_end; ++bh) {
        const size_t hoff = (size_t)bh * (size_t)N * (size_t)d;
        for (long long t = 0; t < N; ++t) {
            const long long inwin =
                na_oracle_mask_row_dil(J->ndim, J->L, J->w, J->s, J->mode, J->dil, t, mask);
            const size_t qoff = hoff + (size_t)t * (size_t)d;
            long long cnt = 0;
            for (long long j = 0; j < N; ++j) {
                if (!mask[j]) continue;
                if (cnt >= J->W) { J->status = -3; goto done; }
                const size_t koff = hoff + (size_t)j * (size_t)d;
                double dot = 0.0;
                for (int c = 0; c < d; ++c) {
                    const double qc = load_in(J->q, J->dtype, qoff + c);
                    dot += qc * load_in(J->k, J->dtype, koff + (size_t)c);
                }
                z[cnt] = dot * J->scale;
                idx[cnt] = j;
                ++cnt;
            }
            if (cnt != inwin || cnt < 1) { J->status = -3; goto done; }
            double m = -INFINITY;
            for (long long e = 0; e < cnt; ++e) if (z[e] > m) m = z[e];
            double l = 0.0;
            for (long long e = 0; e < cnt; ++e) l += exp(z[e] - m);
            const double lse = m + log(l);
            /* out_i and D_i = <dO_i, out_i> */
            for (int c = 0; c < d; ++c) o[c] = 0.0;
            for (long long e = 0; e < cnt; ++e) {
                const double p = exp(z[e] - lse);
                const size_t voff = hoff + (size_t)idx[e] * (size_t)d;
                for (int c = 0; c < d; ++c) o[c] += p * load_in(J->v, J->dtype, voff + c);
            }
            double Di = 0.0;
            for (int c = 0; c < d; ++c) Di += load_in(J->dout, J->dtype, qoff + c) * o[c];
            for (int c = 0; c < d; ++c) g[c] = 0.0;
            for (long long e = 0; e < cnt; ++e) {
                const double p = exp(z[e] - lse);
                const size_t koff = hoff + (size_t)idx[e] * (size_t)d;
                double dp = 0.0;
                for (int c = 0; c < d; ++c)
                    dp += load_in(J->dout, J->dtype, qoff + c) * load_in(J->v, J->dtype, koff + c);
                const double dz = p * (dp - Di);
                for (int c = 0; c < d; ++c) {
                    g[c] += J->scale * dz * load_in(J->k, J->dtype, koff + (size_t)c);
                    J->dk[koff + c] += J->scale * dz * load_in(J->q, J->dtype, qoff + c);
                    J->dv[koff + c] += p * load_in(J->dout, J->dtype, qoff + c);
                }
            }
            for (int c = 0; c < d; ++c) J->dq[qoff + c] = g[c];
        }
    }
done:
    free(z); free(idx); free(mask); free(o); free(g);
    return NULL;
}

/*
 * Gradients of the forward pass for upstream gradient dout (same layout and
 * dtype as q): dq, dk, dv are [BH, N, d] fp64 (written).  mode: per-dimension
 * window modes or NULL (all clamped); dil: per-dimension dilation or NULL.
 * scale <= 0 means 1/sqrt(d).  Threads split the BH (batch, head) slices, so
 * dk and dv need no reduction across threads.  Returns 0 or a negative code
 * as na_oracle_forward.
 */
int na_oracle_backward_dil(const void* q, const void* k, const void* v, const void* dout,
                           int in_dtype, long long BH, int ndim, const int* L, const int* w,
                           const int* s, const int* mode, const int* dil, int d, double scale,
                           double* dq, double* dk, double* dv, int nthreads) {
    long long N;
    if (!q || !k || !v || !dout || !dq || !dk || !dv || BH < 1 || d < 1) return -1;
    if (in_dtype < IN_F32 || in_dtype > IN_E4M3) return -1;
    if (check_geometry(ndim, L, w, s, mode, dil, &N)) return -1;
    long long W = 1;
    for (int a = 0; a < ndim; ++a) W *= w[a];
    if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
    memset(dq, 0, sizeof(double) * (size_t)(BH * N * d));
    memset(dk, 0, sizeof(double) * (size_t)(BH * N * d));
    memset(dv, 0, sizeof(double) * (size_t)(BH * N * d));
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (nthreads > BH) nthreads = (int)BH;
    bwd_job jobs[256];
    pthread_t th[256];
    const long long per = (BH + nthreads - 1) / nthreads;
    for (int t = 0; t < nthreads; ++t) {
        bwd_job* J = &jobs[t];
        J->q = q; J->k = k; J->v = v; J->dout = dout;
        J->dtype = in_dtype; J->ndim = ndim; J->d = d;
        J->L = L; J->w = w; J->s = s; J->mode = mode;
        J->N = N; J->W = W; J->scale = scale;
        J->bh_begin = per * t < BH ? per * t : BH;
        J->bh_end = per * (t + 1) < BH ? per * (t + 1) : BH;
        J->dq = dq; J->dk = dk; J->dv = dv;
        J->dil = dil;
        J->status = 0;
    }
    for (int t = 1; t < nthreads; ++t)
        if (pthread_create(&th[t], NULL, bwd_worker, &jobs[t]) != 0) {
            bwd_worker(&jobs[t]);
            th[t] = 0;
        }
    bwd_worker(&jobs[0]);
    for (int t = 1; t < nthreads; ++t)
        if (th[t]) pthread_join(th[t], NULL);
    for (int t = 0; t < nthreads; ++t)
        if (jobs[t].status) return jobs[t].status;
    return 0;
}

int na_oracle_backward(const void* q, const void* k, const void* v, const void* dout, int in_dtype,
                       long long BH, int ndim, const int* L, const int* w, const int* s,
                       const int* mode, int d, double scale, double* dq, double* dk, double* dv,
                       int nthreads) {
    return na_oracle_backward_dil(q, k, v, dout, in_dtype, BH, ndim, L, w, s, mode, NULL, d, scale,
                                  dq, dk, dv, nthreads);
}

/*
 * Gradients on sampled rows of one (batch, head) slice bh, for parity checks
 * at sizes where the full backward is too slow: first lse_t and
 * D_t = <dO_t, out_t> for the queries t the sampled rows depend on -- the
 * query rows `qrows` themselves and every query whose window holds one of the
 * key rows `krows` (token indices within the slice) -- then dq for the query
 * rows and dk, dv for the key rows, each summed over the queries whose window
 * holds the key.  Threads split the queries of the first step and the rows of
 * the second.  Outputs [nq, d] and [nk, d] fp64.  Same definitions as
 * na_oracle_backward, which it equals on every row.
 */
typedef struct {
    const void *q, *k, *v, *dout;
    int dtype, ndim, d;
    const int *L, *w, *s, *mode;
    long long N, W, bh;
    double scale;
    const long long* list;          /* the queries whose lse_t, D_t are needed */
    long long i_begin, i_end;       /* this thread's share of `list` */
    double *lse, *delta;
    int status;
} stat_job;

static void* stat_worker(void* arg) {
    stat_job* J = (stat_job*)arg;
    const int d = J->d;
    const size_t hoff = (size_t)J->bh * (size_t)J->N * (size_t)d;
    double* z = (double*)malloc(sizeof(double) * (size_t)J->W);
    long long* idx = (long long*)malloc(sizeof(long long) * (size_t)J->W);
    uint8_t* mask = (uint8_t*)malloc((size_t)J->N);
    if (!z || !idx || !mask) { J->status = -2; goto done; }
    for (long long i = J->i_begin; i < J->i_end; ++i) {
        const long long t = J->list[i];
        na_oracle_mask_row(J->ndim, J->L, J->w, J->s, J->mode, t, mask);
        const size_t qoff = hoff + (size_t)t * (size_t)d;
        long long cnt = 0;
        for (long long j = 0; j < J->N; ++j) {
            if (!mask[j]) continue;
            if (cnt >= J->W) { J->status = -3; goto done; }
            const size_t koff = hoff + (size_t)j * (size_t)d;
            double dot = 0.0;
            for (int c = 0; c < d; ++c)
                dot += load_in(J->q, J->dtype, qoff + c) * load_in(J->k, J->dtype, koff + (size_t)c);
            z[cnt] = dot * J->scale;
            idx[cnt++] = j;
        }
        double m = -INFINITY, l = 0.0;
        for (long long e = 0; e < cnt; ++e) if (z[e] > m) m = z[e];
        for (long long e = 0; e < cnt; ++e) l += exp(z[e] - m);
        const double lse = m + log(l);
        double D = 0.0;
        for (long long e = 0; e < cnt; ++e) {
            const size_t voff = hoff + (size_t)idx[e] * (size_t)d;
            double dv = 0.0;
            for (int c = 0; c < d; ++c)
                dv += load_in(J->dout, J->dtype, qoff + c) * load_in(J->v, J->dtype, voff + c);
            D += exp(z[e] - lse) * dv;
        }
        J->lse[t] = lse;
        J->delta[t] = D;
    }
done:
    free(z); free(idx); free(mask);
    return NULL;
}

/* Does the window of query t (grid coordinates qi) hold key kj? */
static int window_holds(int ndim, const int* L, const int* w, const int* s, const int* mode,
                        const int* qi, const int* kj) {
    for (int a = 0; a < ndim; ++a) {
        int lo, hi;
        na_oracle_window(L[a], w[a], s[a], mode ? mode[a] : 0, qi[a], &lo, &hi);
        if (kj[a] < lo || kj[a] >= hi) return 0;
    }
    return 1;
}

typedef struct {
    const void *q, *k, *v, *dout;
    int dtype, ndim, d;
    const int *L, *w, *s, *mode;
    long long N, bh;
    double scale;
    const double *lse, *delta;
    const long long *qrows, *krows;
    long long q_begin, q_end, k_begin, k_end;   /* this thread's sampled rows */
    double *dq, *dk, *dv;
    int status;
} grad_job;

static void* grad_worker(void* arg) {
    grad_job* J = (grad_job*)arg;
    const int d = J->d, ndim = J->ndim, dt = J->dtype;
    const void *Q = J->q, *K = J->k, *V = J->v, *DO = J->dout;
    const size_t hoff = (size_t)J->bh * (size_t)J->N * (size_t)d;
    uint8_t* mask = (uint8_t*)malloc((size_t)J->N);
    if (!mask) { J->status = -2; return NULL; }
    /* dq of the sampled query rows */
    for (long long r = J->q_begin; r < J->q_end; ++r) {
        const long long t = J->qrows[r];
        na_oracle_mask_row(ndim, J->L, J->w, J->s, J->mode, t, mask);
        const size_t qoff = hoff + (size_t)t * (size_t)d;
        double* g = J->dq + (size_t)r * d;
        for (int c = 0; c < d; ++c) g[c] = 0.0;
        for (long long j = 0; j < J->N; ++j) {
            if (!mask[j]) continue;
            const size_t koff = hoff + (size_t)j * (size_t)d;
            double zq = 0.0, dp = 0.0;
            for (int c = 0; c < d; ++c) {
                zq += load_in(Q, dt, qoff + c) * load_in(K, dt, koff + c);
                dp += load_in(DO, dt, qoff + c) * load_in(V, dt, koff + c);
            }
            const double p = exp(J->scale * zq - J->lse[t]);
            const double dz = p * (dp - J->delta[t]);
            for (int c = 0; c < d; ++c) g[c] += J->scale * dz * load_in(K, dt, koff + c);
        }
    }
    /* dk, dv of the sampled key rows: over every query whose window holds the key */
    for (long long r = J->k_begin; r < J->k_end; ++r) {
        const long long j = J->krows[r];
        const size_t koff = hoff + (size_t)j * (size_t)d;
        double* gk = J->dk + (size_t)r * d;
        double* gv = J->dv + (size_t)r * d;
        for (int c = 0; c < d; ++c) { gk[c] = 0.0; gv[c] = 0.0; }
        int kj[NA_ORACLE_MAXDIM];
        unflatten(j, ndim, J->L, kj);
        int qi[NA_ORACLE_MAXDIM];
        for (int a = 0; a < ndim; ++a) qi[a] = 0;
        for (long long t = 0; t < J->N; ++t) {
            if (window_holds(ndim, J->L, J->w, J->s, J->mode, qi, kj)) {
                const size_t qoff = hoff + (size_t)t * (size_t)d;
                double zq = 0.0, dp = 0.0;
                for (int c = 0; c < d; ++c) {
                    zq += load_in(Q, dt, qoff + c) * load_in(K, dt, koff + c);
                    dp += load_in(DO, dt, qoff + c) * load_in(V, dt, koff + c);
                }
                const double p = exp(J->scale * zq - J->lse[t]);
                const double dz = p * (dp - J->delta[t]);
                for (int c = 0; c < d; ++c) {
                    gk[c] += J->scale * dz * load_in(Q, dt, qoff + c);
                    gv[c] += p * load_in(DO, dt, qoff + c);
                }
            }
            for (int a = ndim - 1; a >= 0; --a) { /* advance the row-major query counter */
                if (++qi[a] < J->L[a]) break;
                qi[a] = 0;
            }
        }
    }
    free(mask);
    return NULL;
}

int na_oracle_backward_sampled(const void* q, const void* k, const void* v, const void* dout,
                               int in_dtype, long long BH, long long bh, int ndim, const int* L,
                               const int* w, const int* s, const int* mode, int d, double scale,
                               const long long* qrows, long long nq, const long long* krows,
                               long long nk, double* dq, double* dk, double* dv, int nthreads) {
    long long N;
    if (!q || !k || !v || !dout || BH < 1 || bh < 0 || bh >= BH || d < 1) return -1;
    if ((nq && (!qrows || !dq)) || (nk && (!krows || !dk || !dv))) return -1;
    if (in_dtype < IN_F32 || in_dtype > IN_E4M3) return -1;
    if (check_geometry(ndim, L, w, s, mode, NULL, &N)) return -1;
    for (long long r = 0; r < nq; ++r) if (qrows[r] < 0 || qrows[r] >= N) return -1;
    for (long long r = 0; r < nk; ++r) if (krows[r] < 0 || krows[r] >= N) return -1;
    long long W = 1;
    for (int a = 0; a < ndim; ++a) W *= w[a];
    if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
    double* lse = (double*)malloc(sizeof(double) * (size_t)N);
    double* delta = (double*)malloc(sizeof(double) * (size_t)N);
    uint8_t* needed = (uint8_t*)calloc((size_t)N, 1);
    long long* list = (long long*)malloc(sizeof(long long) * (size_t)N);
    if (!lse || !delta || !needed || !list) {
        free(lse); free(delta); free(needed); free(list);
        return -2;
    }
    /* the queries whose statistics the sampled rows read */
    for (long long r = 0; r < nq; ++r) needed[qrows[r]] = 1;
    if (nk) {
        int qi[NA_ORACLE_MAXDIM];
        for (int a = 0; a < ndim; ++a) qi[a] = 0;
        for (long long t = 0; t < N; ++t) {
            for (long long r = 0; r < nk && !needed[t]; ++r) {
                int kj[NA_ORACLE_MAXDIM];
                unflatten(krows[r], ndim, L, kj);
                if (window_holds(ndim, L, w, s, mode, qi, kj)) needed[t] = 1;
            }
            for (int a = ndim - 1; a >= 0; --a) {
                if (++qi[a] < L[a]) break;
                qi[a] = 0;
            }
        }
    }
    long long nlist = 0;
    for (long long t = 0; t < N; ++t) if (needed[t]) list[nlist++] = t;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    pthread_t th[256];
    stat_job jobs[256];
    const long long per = (nlist + nthreads - 1) / nthreads;
    for (int t = 0; t < nthreads; ++t) {
        stat_job* J = &jobs[t];
        J->q = q; J->k = k; J->v = v; J->dout = dout;
        J->dtype = in_dtype; J->ndim = ndim; J->d = d;
        J->L = L; J->w = w; J->s = s; J->mode = mode;
        J->N = N; J->W = W; J->bh = bh; J->scale = scale;
        J->list = list;
        J->i_begin = per * t < nlist ? per * t : nlist;
        J->i_end = per * (t + 1) < nlist ? per * (t + 1) : nlist;
        J->lse = lse; J->delta = delta;
        J->status = 0;
    }
    for (int t = 1; t < nthreads; ++t)
        if (pthread_create(&th[t], NULL, stat_worker, &jobs[t]) != 0) {
            stat_worker(&jobs[t]);
            th[t] = 0;
        }
    stat_worker(&jobs[0]);
    for (int t = 1; t < nthreads; ++t)
        if (th[t]) pthread_join(th[t], NULL);
    int rc = 0;
    for (int t = 0; t < nthreads; ++t)
        if (jobs[t].status) rc = jobs[t].status;
    if (!rc) {
        grad_job gj[256];
        const long long pq = (nq + nthreads - 1) / nthreads, pk = (nk + nthreads - 1) / nthreads;
        for (int t = 0; t < nthreads; ++t) {
            grad_job* J = &gj[t];
            J->q = q; J->k = k; J->v = v; J->dout = dout;
            J->dtype = in_dtype; J->ndim = ndim; J->d = d;
            J->L = L; J->w = w; J->s = s; J->mode = mode;
            J->N = N; J->bh = bh; J->scale = scale;
            J->lse = lse; J->delta = delta;
            J->qrows = qrows; J->krows = krows;
            J->q_begin = pq * t < nq ? pq * t : nq;
            J->q_end = pq * (t + 1) < nq ? pq * (t + 1) : nq;
            J->k_begin = pk * t < nk ? pk * t : nk;
            J->k_end = pk * (t + 1) < nk ? pk * (t + 1) : nk;
            J->dq = dq; J->dk = dk; J->dv = dv;
            J->status = 0;
        }
        for (int t = 1; t < nthreads; ++t)
            if (pthread_create(&th[t], NULL, grad_worker, &gj[t]) != 0) {
                grad_worker(&gj[t]);
                th[t] = 0;
            }
        grad_worker(&gj[0]);
        for (int t = 1; t < nthreads; ++t)
            if (th[t]) pthread_join(th[t], NULL);
        for (int t = 0; t < nthreads; ++t)
            if (gj[t].status) rc = gj[t].status;
    }
    free(lse); free(delta); free(needed); free(list);
    return rc;
}

/* --------------------------------------------------------- block counts -- */

/*
 * Cut the N x N attention map (tokens in row-major grid order) into blk x blk
 * tiles and count empty (no query-key pair in a window), full (every pair in
 * a window) and partial tiles.  counts[0..2] = {empty, partial, full}.
 */
int na_oracle_block_counts(int ndim, const int* L, const int* w, const int* s, const int* mode,
                           long long blk, long long* counts) {
    long long N;
    if (check_geometry(ndim, L, w, s, mode, NULL, &N) || blk < 1 || !counts) return -1;
    long long nb = (N + blk - 1) / blk;
    long long* members = (long long*)calloc((size_t)(nb * nb), sizeof(long long));
    uint8_t* mask = (uint8_t*)malloc((size_t)N);
    if (!members || !mask) { free(members); free(mask); return -2; }
    for (long long t = 0; t < N; ++t) {
        na_oracle_mask_row(ndim, L, w, s, mode, t, mask);
        long long* rowblk = members + (t / blk) * nb;
        for (long long j = 0; j < N; ++j) rowblk[j / blk] += mask[j];
    }
    counts[0] = counts[1] = counts[2] = 0;
    for (long long a = 0; a < nb; ++a)
        for (long long b = 0; b < nb; ++b) {
            long long ra = (a + 1) * blk <= N ? blk : N - a * blk;
            long long cb = (b + 1) * blk <= N ? blk : N - b * blk;
            long long m = members[a * nb + b];
            counts[m == 0 ? 0 : (m == ra * cb ? 2 : 1)] += 1;
        }
    free(members);
    free(mask);
    return 0;
}
