/*
 * dsa3d_oracle.c -- plain, slow CPU oracle for 3D Deformable Slide Attention (3D-DSA).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or load this file;
 * only the test suite, the package's smoke check and the benchmark's CPU-baseline leg use it.
 * It shares no code, header, table or helper with the CUDA path.
 *
 * What it computes (MegaSlide-DiT, "Memory-Centric Adaptation and Deformable Local Attention
 * for Efficient Video Diffusion", arXiv 2607.22696, the 3D-DSA definition, Eq. 1 and the
 * softmax equation right after it):
 *
 *   out(t,i,j) = sum_{u,v,w} alpha_{u,v,w} * TrilinearSample(V, p + tau_{u,v,w} + delta)
 *   alpha      = softmax over the window taps of  q . TrilinearSample(K, ...) / sqrt(dh)
 *
 * for every attention head separately.  The DWConv3D term of Eq. 1 is the caller's and is not
 * computed here.  Every step is done directly, tap by tap: each tap's key and value are sampled
 * at its own fractional position by trilinear interpolation of the 8 surrounding tokens, then
 * dotted with q.  No work is shared between taps.  All arithmetic is in double precision except
 * the offset decode, which the readings below fix in single precision.
 *
 * Readings of the paper fixed here (the paper leaves them open):
 *   R1  One offset 3-vector (dt, dy, dx) per (token, head) slides the whole window (the
 *       "slide" of the operator's name; the paper's per-tap offset tensor is not used).
 *   R2  The regular window is centred: tap (u,v,w) in [-r_t..r_t] x [-r_h..r_h] x [-r_w..r_w]
 *       with r = (k-1)/2, so that zero offsets give plain local attention with kernel
 *       (k_t,k_h,k_w), as the fixed-window ablation states.  Window sizes are odd.
 *   R3  Score scale 1/sqrt(dh), dh = per-head width (the equation's sqrt(d) read per head).
 *   R4  Positions use grid_sample's align_corners=True convention: integer coordinate = token
 *       centre.  Offsets are decoded in single precision: i = floor(delta), f = delta - i
 *       rounded to nearest; f == 1 carries into i.  A non-finite offset, or |delta| > 2^24,
 *       makes the whole query invalid.
 *   R5  A tap whose sample position leaves the closed box [0, dim-1] on any axis is masked
 *       out of the softmax.  Corners outside the volume read as zero (they only occur with
 *       weight zero).  A query with no valid tap yields out = 0 and lse = -inf, and receives
 *       and gives zero gradient.
 *   R6  Values are sampled at the same positions as keys.  No causal mask.
 *   R7  Backward: exact derivative of the above with the validity pattern and the integer
 *       part held fixed; d/d(delta) is the derivative of the trilinear weights inside the cell
 *       [i, i+1] (the +f side at exact integers).  The softmax Jacobian's D = sum_tau P dP
 *       equals dO . out for the exact out (no rounding to the I/O type).
 *   R8  Per-tap offsets (the *_taps entry points): the paper's offset tensor with one 3-vector
 *       per window tap, offsets [heads][N][K][3] with K = kt*kh*kw in tap order (u outermost).
 *       Tap tau samples at p + tau + delta_tau; each tap's offset is decoded as in R4 on its
 *       own, and a non-finite or too large offset masks only that tap (R5 applies per tap).
 *       The offset gradient is per tap, [heads][N][K][3].  With every tap's offset equal to one
 *       per-token offset the result is that of R1.
 *   R9  The DWConv3D term of Eq. 1 (dsa3d_oracle_dwconv3d): a depthwise 3-D convolution of the
 *       layer input X [N][C], C = heads * dh, with a kernel of the window's extent
 *       (kt x kh x kw: the paper names one neighbourhood size per layer), stride 1, zero
 *       padding so the output grid equals the token grid, a bias per channel, and
 *       cross-correlation (PyTorch's conv3d convention, which the paper's implementation
 *       uses).  Its output adds to the attention output channel by channel, c = h * dh + e.
 *   R10 The offset network ("a lightweight depthwise 3D convolution followed by a linear
 *       layer"; nn.Conv3d with groups = hidden size, then pointwise convolutions): its own
 *       depthwise convolution as in R9, then one pointwise linear layer C -> heads * 3 (per
 *       token, R1) or heads * K * 3 (per tap, R8) with bias; output channel (h * 3 + a), or
 *       ((h * K + tau) * 3 + a), is offset component a of head h (and tap tau).  The pointwise
 *       layer is a matrix product and is composed in the Python module.
 *
 * Layouts: q, k, v, dout: [N][heads][dh] (token n = (t*Hp + y)*Wp + x), in fp32 or bf16 bits.
 * offsets: [heads][N][3] fp32, order (dt, dy, dx).  A query or key "item" is h*N + n.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <omp.h>

#define IO_F32 0
#define IO_BF16 1

typedef struct {
    int F, Hp, Wp, heads, dh, kt, kh, kw, io;
    int n_off;       /* offsets per (token, head): 1 (R1) or K (R8) */
    int64_t N;
    const void *q, *k, *v, *dout;
    const float *off;
} prob_t;

/* One query's decoded offset. */
typedef struct {
    int ok;          /* 0: the query is invalid (R4) */
    int64_t i[3];    /* integer parts (t, y, x)      */
    float f[3];      /* fractional parts in [0,1)    */
} decode_t;

static double rd(const void *base, int io, int64_t idx) {
    if (io == IO_F32) return (double)((const float *)base)[idx];
    uint32_t u = (uint32_t)((const uint16_t *)base)[idx] << 16;
    float x;
    memcpy(&x, &u, 4);
    return (double)x;
}

/* Decode one offset 3-vector o (R4). */
static decode_t decode_vec(const float *o) {
    decode_t d;
    d.ok = 1;
    for (int a = 0; a < 3; a++) {
        volatile float delta = o[a];
        if (!isfinite(delta) || fabsf(delta) > 16777216.0f) {
            d.ok = 0;
            d.i[a] = 0;
            d.f[a] = 0.0f;
            continue;
        }
        volatile float fl = floorf(delta);
        volatile float fr = delta - fl; /* single-precision subtraction, round to nearest */
        int64_t ii = (int64_t)fl;
        if (fr == 1.0f) {
            ii += 1;
            fr = 0.0f;
        }
        d.i[a] = ii;
        d.f[a] = fr;
    }
    return d;
}

/* The per-token offset of query n (R1). */
static decode_t decode(const prob_t *P, int h, int64_t n) {
    return decode_vec(P->off + ((int64_t)h * P->N + n) * 3);
}

/* The decoded offset of tap tau of query n: the query's own d (R1), or the tap's (R8). */
static decode_t tap_decode(const prob_t *P, int h, int64_t n, int tau, const decode_t *d) {
    if (P->n_off == 1) return *d;
    return decode_vec(P->off + (((int64_t)h * P->N + n) * P->n_off + tau) * 3);
}

/* Token coordinates of token n. */
static void coords(const prob_t *P, int64_t n, int64_t p[3]) {
    p[2] = n % P->Wp;
    p[1] = (n / P->Wp) % P->Hp;
    p[0] = n / ((int64_t)P->Wp * P->Hp);
}

static int dim_of(const prob_t *P, int a) { return a == 0 ? P->F : (a == 1 ? P->Hp : P->Wp); }

/* Tap index -> (u,v,w) with u outermost. */
static void tap_uvw(const prob_t *P, int tau, int uvw[3]) {
    int rt = (P->kt - 1) / 2, rh = (P->kh - 1) / 2, rw = (P->kw - 1) / 2;
    uvw[2] = tau % P->kw - rw;
    uvw[1] = (tau / P->kw) % P->kh - rh;
    uvw[0] = tau / (P->kw * P->kh) - rt;
}

/* Base corner of tap tau of a decoded query at p; returns 1 iff the tap is valid (R5). */
static int tap_base(const prob_t *P, const int64_t p[3], const decode_t *d, int tau, int64_t b[3]) {
    int uvw[3];
    tap_uvw(P, tau, uvw);
    int valid = d->ok;
    for (int a = 0; a < 3; a++) {
        b[a] = p[a] + uvw[a] + d->i[a];
        int64_t D = dim_of(P, a);
        if (b[a] < 0 || b[a] > D - 1) valid = 0;
        if (b[a] == D - 1 && d->f[a] != 0.0f) valid = 0;
    }
    return valid;
}

/* Trilinear weight of corner c (bit 2: t, bit 1: y, bit 0: x) and its derivative along axis a. */
static double corner_w(const float f[3], int c) {
    double w = 1.0;
    for (int a = 0; a < 3; a++) {
        int ca = (c >> (2 - a)) & 1;
        w *= ca ? (double)f[a] : 1.0 - (double)f[a];
    }
    return w;
}
static double corner_dw(const float f[3], int c, int axis) {
    double w = 1.0;
    for (int a = 0; a < 3; a++) {
        int ca = (c >> (2 - a)) & 1;
        if (a == axis) w *= ca ? 1.0 : -1.0;
        else w *= ca ? (double)f[a] : 1.0 - (double)f[a];
    }
    return w;
}

/* Token index of corner c of base b, or -1 if it lies outside the volume. */
static int64_t corner_tok(const prob_t *P, const int64_t b[3], int c) {
    int64_t cc[3];
    for (int a = 0; a < 3; a++) {
        cc[a] = b[a] + ((c >> (2 - a)) & 1);
        if (cc[a] < 0 || cc[a] >= dim_of(P, a)) return -1;
    }
    return (cc[0] * P->Hp + cc[1]) * P->Wp + cc[2];
}

/* Trilinear sample of src (head h) at base b with fractions f; also d/df_a if dsamp != NULL. */
static void sample(const prob_t *P, const void *src, int h, const int64_t b[3], const float f[3],
                   double *samp, double *dsamp, int64_t *reads) {
    int dh = P->dh;
    for (int e = 0; e < dh; e++) samp[e] = 0.0;
    if (dsamp)
        for (int e = 0; e < 3 * dh; e++) dsamp[e] = 0.0;
    for (int c = 0; c < 8; c++) {
        int64_t tok = corner_tok(P, b, c);
        if (tok < 0) continue;
        if (reads) (*reads)++;
        double w = corner_w(f, c);
        double dw[3] = {corner_dw(f, c, 0), corner_dw(f, c, 1), corner_dw(f, c, 2)};
        int64_t row = (tok * P->heads + h) * (int64_t)dh;
        for (int e = 0; e < dh; e++) {
            double x = rd(src, P->io, row + e);
            samp[e] += w * x;
            if (dsamp) {
                dsamp[0 * dh + e] += dw[0] * x;
                dsamp[1 * dh + e] += dw[1] * x;
                dsamp[2 * dh + e] += dw[2] * x;
            }
        }
    }
}

static double dot_row(const prob_t *P, const void *src, int h, int64_t n, const double *x) {
    int64_t row = (n * P->heads + h) * (int64_t)P->dh;
    double s = 0.0;
    for (int e = 0; e < P->dh; e++) s += rd(src, P->io, row + e) * x[e];
    return s;
}

/* Forward of one query: out[dh], returns lse (-inf if no valid tap).  s[] holds K scores. */
static double query_forward(const prob_t *P, int h, int64_t n, double *out, double *s, double *ktil,
                            double *vtil, int64_t *reads) {
    int K = P->kt * P->kh * P->kw, dh = P->dh;
    double scale = 1.0 / sqrt((double)dh);
    int64_t p[3], b[3];
    coords(P, n, p);
    decode_t d = decode(P, h, n);
    double m = -INFINITY;
    int any = 0;
    for (int tau = 0; tau < K; tau++) {
        const decode_t dt = tap_decode(P, h, n, tau, &d);
        if (!tap_base(P, p, &dt, tau, b)) {
            s[tau] = -INFINITY;
            continue;
        }
        sample(P, P->k, h, b, dt.f, ktil, NULL, reads);
        s[tau] = scale * dot_row(P, P->q, h, n, ktil);
        if (s[tau] > m) m = s[tau];
        any = 1;
    }
    for (int e = 0; e < dh; e++) out[e] = 0.0;
    if (!any) return -INFINITY;
    double l = 0.0;
    for (int tau = 0; tau < K; tau++) {
        if (s[tau] == -INFINITY) continue;
        double pt = exp(s[tau] - m);
        l += pt;
        const decode_t dt = tap_decode(P, h, n, tau, &d);
        tap_base(P, p, &dt, tau, b);
        sample(P, P->v, h, b, dt.f, vtil, NULL, reads);
        for (int e = 0; e < dh; e++) out[e] += pt * vtil[e];
    }
    for (int e = 0; e < dh; e++) out[e] /= l;
    return m + log(l);
}

static prob_t make_prob(int io, const void *q, const void *k, const void *v, const float *off,
                        const void *dout, int F, int Hp, int Wp, int heads, int dh, int kt, int kh,
                        int kw) {
    prob_t P;
    P.F = F; P.Hp = Hp; P.Wp = Wp; P.heads = heads; P.dh = dh;
    P.kt = kt; P.kh = kh; P.kw = kw; P.io = io;
    P.N = (int64_t)F * Hp * Wp;
    P.q = q; P.k = k; P.v = v; P.off = off; P.dout = dout;
    P.n_off = 1;
    return P;
}

static int check_args(int F, int Hp, int Wp, int heads, int dh, int kt, int kh, int kw, int io) {
    if (F < 1 || Hp < 1 || Wp < 1 || heads < 1 || dh < 1) return -1;
    if (kt < 1 || kh < 1 || kw < 1 || !(kt & 1) || !(kh & 1) || !(kw & 1)) return -1;
    if (io != IO_F32 && io != IO_BF16) return -1;
    return 0;
}

/*
 * Forward for a list of query items (h*N + n).  out: [n_items][dh], lse: [n_items].
 * Returns the number of corner-token reads performed (a work counter), or -1 on bad arguments.
 * per_tap selects the offset layout: 0 = [heads][N][3] (R1), 1 = [heads][N][K][3] (R8).
 */
static int64_t forward_impl(int io, const void *q, const void *k, const void *v, const float *off,
                            int F, int Hp, int Wp, int heads, int dh, int kt, int kh, int kw,
                            const int64_t *items, int64_t n_items, double *out, double *lse,
                            int n_threads, int per_tap) {
    if (check_args(F, Hp, Wp, heads, dh, kt, kh, kw, io)) return -1;
    prob_t P = make_prob(io, q, k, v, off, NULL, F, Hp, Wp, heads, dh, kt, kh, kw);
    int K = kt * kh * kw;
    P.n_off = per_tap ? K : 1;
    for (int64_t it = 0; it < n_items; it++)
        if (items[it] < 0 || items[it] >= P.N * heads) return -1;
    int64_t total_reads = 0;
#pragma omp parallel num_threads(n_threads > 0 ? n_threads : 1) reduction(+ : total_reads)
    {
        double *s = (double *)malloc(sizeof(double) * K);
        double *kt_ = (double *)malloc(sizeof(double) * dh);
        double *vt_ = (double *)malloc(sizeof(double) * dh);
#pragma omp for schedule(dynamic, 8)
        for (int64_t it = 0; it < n_items; it++) {
            int h = (int)(items[it] / P.N);
            int64_t n = items[it] % P.N;
            int64_t reads = 0;
            lse[it] = query_forward(&P, h, n, out + it * dh, s, kt_, vt_, &reads);
            total_reads += reads;
        }
        free(s); free(kt_); free(vt_);
    }
    return total_reads;
}

int64_t dsa3d_oracle_forward(int io, const void *q, const void *k, const void *v, const float *off,
                             int F, int Hp, int Wp, int heads, int dh, int kt, int kh, int kw,
                             const int64_t *items, int64_t n_items, double *out, double *lse,
                             int n_threads) {
    return forward_impl(io, q, k, v, off, F, Hp, Wp, heads, dh, kt, kh, kw, items, n_items, out, lse,
                        n_threads, 0);
}

/* Forward with per-tap offsets [heads][N][K][3] (R8); otherwise as dsa3d_oracle_forward. */
int64_t dsa3d_oracle_forward_taps(int io, const void *q, const void *k, const void *v,
                                  const float *off, int F, int Hp, int Wp, int heads, int dh, int kt,
                                  int kh, int kw, const int64_t *items, int64_t n_items, double *out,
                                  double *lse, int n_threads) {
    return forward_impl(io, q, k, v, off, F, Hp, Wp, heads, dh, kt, kh, kw, items, n_items, out, lse,
                        n_threads, 1);
}

/* Per-thread work arrays of the backward. */
typedef struct {
    double *s, *P, *dS, *ktil, *vtil, *dk_t, *dv_t, *out, *q, *dO;
} scratch_t;

static scratch_t scratch_new(int K, int dh) {
    scratch_t S;
    S.s = malloc(sizeof(double) * K);
    S.P = malloc(sizeof(double) * K);
    S.dS = malloc(sizeof(double) * K);
    S.ktil = malloc(sizeof(double) * dh);
    S.vtil = malloc(sizeof(double) * dh);
    S.dk_t = malloc(sizeof(double) * 3 * dh);
    S.dv_t = malloc(sizeof(double) * 3 * dh);
    S.out = malloc(sizeof(double) * dh);
    S.q = malloc(sizeof(double) * dh);
    S.dO = malloc(sizeof(double) * dh);
    return S;
}
static void scratch_free(scratch_t *S) {
    free(S->s); free(S->P); free(S->dS); free(S->ktil); free(S->vtil);
    free(S->dk_t); free(S->dv_t); free(S->out); free(S->q); free(S->dO);
}

/*
 * Softmax backward of one query: P[tau], dS[tau] (zero for masked taps), and dq, doff.
 * Returns 0 if the query has no valid tap (everything zero).
 */
static int query_backward(const prob_t *P, int h, int64_t n, scratch_t *S, double *dq,
                          double *doff_all) {
    int K = P->kt * P->kh * P->kw, dh = P->dh;
    double scale = 1.0 / sqrt((double)dh);
    int64_t p[3], b[3];
    coords(P, n, p);
    decode_t d = decode(P, h, n);
    for (int e = 0; e < dh; e++) dq[e] = 0.0;
    for (int e = 0; e < 3 * P->n_off; e++) doff_all[e] = 0.0;
    for (int tau = 0; tau < K; tau++) S->P[tau] = S->dS[tau] = 0.0;
    double lse = query_forward(P, h, n, S->out, S->s, S->ktil, S->vtil, NULL);
    if (lse == -INFINITY) return 0;
    int64_t row = (n * P->heads + h) * (int64_t)dh;
    for (int e = 0; e < dh; e++) {
        S->q[e] = rd(P->q, P->io, row + e);
        S->dO[e] = rd(P->dout, P->io, row + e);
    }
    double D = 0.0;
    for (int e = 0; e < dh; e++) D += S->dO[e] * S->out[e];
    for (int tau = 0; tau < K; tau++) {
        if (S->s[tau] == -INFINITY) continue;
        const decode_t dt = tap_decode(P, h, n, tau, &d);
        double *doff = doff_all + (P->n_off > 1 ? 3 * tau : 0); /* per query (R1) or tap (R8) */
        tap_base(P, p, &dt, tau, b);
        sample(P, P->k, h, b, dt.f, S->ktil, S->dk_t, NULL);
        sample(P, P->v, h, b, dt.f, S->vtil, S->dv_t, NULL);
        double Pt = exp(S->s[tau] - lse);
        double dP = 0.0;
        for (int e = 0; e < dh; e++) dP += S->dO[e] * S->vtil[e];
        double dS = Pt * (dP - D);
        S->P[tau] = Pt;
        S->dS[tau] = dS;
        for (int e = 0; e < dh; e++) dq[e] += scale * dS * S->ktil[e];
        for (int a = 0; a < 3; a++) {
            double qk = 0.0, ov = 0.0;
            for (int e = 0; e < dh; e++) {
                qk += S->q[e] * S->dk_t[a * dh + e];
                ov += S->dO[e] * S->dv_t[a * dh + e];
            }
            doff[a] += scale * dS * qk + Pt * ov;
        }
    }
    return 1;
}

/*
 * Backward.  dq/doff are reported for the query items q_items ([n_q][dh], [n_q][3]).
 * dk/dv are reported for the key items k_items ([n_k][dh]); each gathers the contributions of
 * every query of its head whose taps touch it.  Returns 0, or -1 on bad arguments.  With
 * per_tap (R8) the offsets are [heads][N][K][3] and doff is [n_q][K][3].
 */
static int backward_impl(int io, const void *q, const void *k, const void *v, const float *off,
                         const void *dout, int F, int Hp, int Wp, int heads, int dh, int kt,
                         int kh, int kw, const int64_t *q_items, int64_t n_q, double *dq,
                         double *doff, const int64_t *k_items, int64_t n_k, double *dk,
                         double *dv, int n_threads, int per_tap) {
    if (check_args(F, Hp, Wp, heads, dh, kt, kh, kw, io)) return -1;
    prob_t P = make_prob(io, q, k, v, off, dout, F, Hp, Wp, heads, dh, kt, kh, kw);
    int K = kt * kh * kw;
    P.n_off = per_tap ? K : 1;
    int nt = n_threads > 0 ? n_threads : 1;
    double scale = 1.0 / sqrt((double)dh);
    for (int64_t it = 0; it < n_q; it++)
        if (q_items[it] < 0 || q_items[it] >= P.N * heads) return -1;
    for (int64_t it = 0; it < n_k; it++)
        if (k_items[it] < 0 || k_items[it] >= P.N * heads) return -1;

#pragma omp parallel num_threads(nt)
    {
        scratch_t S = scratch_new(K, dh);
#pragma omp for schedule(dynamic, 4)
        for (int64_t it = 0; it < n_q; it++) {
            int h = (int)(q_items[it] / P.N);
            int64_t n = q_items[it] % P.N;
            query_backward(&P, h, n, &S, dq + it * dh, doff + it * 3 * P.n_off);
        }
        scratch_free(&S);
    }
    if (n_k == 0) return 0;

    for (int64_t e = 0; e < n_k * dh; e++) dk[e] = dv[e] = 0.0;
    /* Map each requested key token to its output row, per head. */
    int64_t *rowmap = malloc(sizeof(int64_t) * P.N * heads);
    for (int64_t e = 0; e < P.N * heads; e++) rowmap[e] = -1;
    int *head_used = calloc(heads, sizeof(int));
    for (int64_t it = 0; it < n_k; it++) {
        rowmap[k_items[it]] = it;
        head_used[k_items[it] / P.N] = 1;
    }
    /* One thread per head; queries visited in index order. */
#pragma omp parallel num_threads(nt)
    {
        scratch_t S = scratch_new(K, dh);
        double *dq_tmp = malloc(sizeof(double) * dh);
        double *doff_tmp = malloc(sizeof(double) * 3 * P.n_off);
#pragma omp for schedule(dynamic, 1)
        for (int h = 0; h < heads; h++) {
            if (!head_used[h]) continue;
            const int64_t *map = rowmap + (int64_t)h * P.N;
            for (int64_t n = 0; n < P.N; n++) {
                /* Skip queries none of whose taps' corners is a requested key. */
                int64_t p[3], b[3];
                coords(&P, n, p);
                decode_t d = decode(&P, h, n);
                if (P.n_off == 1 && !d.ok) continue;
                int touches = 0;
                for (int tau = 0; tau < K && !touches; tau++) {
                    const decode_t dt = tap_decode(&P, h, n, tau, &d);
                    if (!tap_base(&P, p, &dt, tau, b)) continue;
                    for (int c = 0; c < 8; c++) {
                        int64_t tok = corner_tok(&P, b, c);
                        if (tok >= 0 && map[tok] >= 0) { touches = 1; break; }
                    }
                }
                if (!touches) continue;
                if (!query_backward(&P, h, n, &S, dq_tmp, doff_tmp)) continue;
                for (int tau = 0; tau < K; tau++) {
                    if (S.P[tau] == 0.0 && S.dS[tau] == 0.0) continue;
                    const decode_t dt = tap_decode(&P, h, n, tau, &d);
                    tap_base(&P, p, &dt, tau, b);
                    for (int c = 0; c < 8; c++) {
                        int64_t tok = corner_tok(&P, b, c);
                        if (tok < 0 || map[tok] < 0) continue;
                        double w = corner_w(dt.f, c);
                        double gk = w * scale * S.dS[tau];
                        double gv = w * S.P[tau];
                        double *dkr = dk + map[tok] * dh, *dvr = dv + map[tok] * dh;
                        for (int e = 0; e < dh; e++) {
                            dkr[e] += gk * S.q[e];
                            dvr[e] += gv * S.dO[e];
                        }
                    }
                }
            }
        }
        free(dq_tmp);
        free(doff_tmp);
        scratch_free(&S);
    }
    free(rowmap);
    free(head_used);
    return 0;
}

int dsa3d_oracle_backward(int io, const void *q, const void *k, const void *v, const float *off,
                          const void *dout, int F, int Hp, int Wp, int heads, int dh, int kt,
                          int kh, int kw, const int64_t *q_items, int64_t n_q, double *dq,
                          double *doff, const int64_t *k_items, int64_t n_k, double *dk,
                          double *dv, int n_threads) {
    return backward_impl(io, q, k, v, off, dout, F, Hp, Wp, heads, dh, kt, kh, kw, q_items, n_q, dq,
                         doff, k_items, n_k, dk, dv, n_threads, 0);
}

/* Backward with per-tap offsets (R8): offsets [heads][N][K][3], doff [n_q][K][3]. */
int dsa3d_oracle_backward_taps(int io, const void *q, const void *k, const void *v,
                               const float *off, const void *dout, int F, int Hp, int Wp, int heads,
                               int dh, int kt, int kh, int kw, const int64_t *q_items, int64_t n_q,
                               double *dq, double *doff, const int64_t *k_items, int64_t n_k,
                               double *dk, double *dv, int n_threads) {
    return backward_impl(io, q, k, v, off, dout, F, Hp, Wp, heads, dh, kt, kh, kw, q_items, n_q, dq,
                         doff, k_items, n_k, dk, dv, n_threads, 1);
}

/*
 * One tap of one query, for cross-checks: validity, decoded base and fraction, the sampled
 * vector of src and its derivative along each fractional coordinate ([3][dh]).
 */
int dsa3d_oracle_tap(int io, const void *src, const float *off, int F, int Hp, int Wp, int heads,
                     int dh, int kt, int kh, int kw, int h, int64_t n, int tau, int64_t *base,
                     float *frac, double *samp, double *dsamp) {
    if (check_args(F, Hp, Wp, heads, dh, kt, kh, kw, io)) return -1;
    prob_t P = make_prob(io, src, src, src, off, NULL, F, Hp, Wp, heads, dh, kt, kh, kw);
    if (h < 0 || h >= heads || n < 0 || n >= P.N || tau < 0 || tau >= kt * kh * kw) return -1;
    int64_t p[3];
    coords(&P, n, p);
    decode_t d = decode(&P, h, n);
    int valid = tap_base(&P, p, &d, tau, base);
    frac[0] = d.f[0]; frac[1] = d.f[1]; frac[2] = d.f[2];
    sample(&P, src, h, base, d.f, samp, dsamp, NULL);
    return valid;
}

/*
 * Depthwise 3-D convolution: the DWConv3D term of Eq. 1 and the first layer of the offset
 * network (readings R9 and R10, MegaSlide-DiT, the 3D-DSA definition).  For every channel c of
 * X [N][C] (token n = (t*Hp + y)*Wp + x) and every output token p = (t, y, x):
 *
 *   Y[p][c] = b[c] + sum_{u<kt, v<kh, w<kw} W[c][u][v][w] * X[(t + u - r_t, y + v - r_h, x + w - r_w)][c]
 *
 * with r = (k-1)/2 and X = 0 outside the volume (zero padding; the output grid is the input
 * grid).  This is cross-correlation, the convention of PyTorch's conv3d with groups = C and
 * padding k // 2.  W is [C][kt][kh][kw] fp32, b is [C] fp32 (may be NULL: no bias), X is fp32 or
 * bf16 bits; Y is double.  Each output is summed directly over its window, tap by tap.
 */
static int conv_args(int F, int Hp, int Wp, int C, int kt, int kh, int kw, int io) {
    if (F < 1 || Hp < 1 || Wp < 1 || C < 1) return -1;
    if (kt < 1 || kh < 1 || kw < 1 || !(kt & 1) || !(kh & 1) || !(kw & 1)) return -1;
    if (io != IO_F32 && io != IO_BF16) return -1;
    return 0;
}

int dsa3d_oracle_dwconv3d(int io, const void *x, const float *w, const float *b, int F, int Hp,
                          int Wp, int C, int kt, int kh, int kw, double *y, int n_threads) {
    if (conv_args(F, Hp, Wp, C, kt, kh, kw, io)) return -1;
    const int64_t N = (int64_t)F * Hp * Wp;
    const int rt = (kt - 1) / 2, rh = (kh - 1) / 2, rw = (kw - 1) / 2;
#pragma omp parallel for schedule(static) num_threads(n_threads > 0 ? n_threads : 1)
    for (int64_t n = 0; n < N; n++) {
        const int64_t x0 = n % Wp, y0 = (n / Wp) % Hp, t0 = n / ((int64_t)Wp * Hp);
        for (int c = 0; c < C; c++) {
            double acc = b ? (double)b[c] : 0.0;
            for (int u = 0; u < kt; u++)
                for (int v = 0; v < kh; v++)
                    for (int ww = 0; ww < kw; ww++) {
                        const int64_t ts = t0 + u - rt, ys = y0 + v - rh, xs = x0 + ww - rw;
                        if (ts < 0 || ts >= F || ys < 0 || ys >= Hp || xs < 0 || xs >= Wp) continue;
                        const int64_t src = (ts * Hp + ys) * Wp + xs;
                        acc += (double)w[((int64_t)c * kt + u) * kh * kw + v * kw + ww] *
                               rd(x, io, src * C + c);
                    }
            y[n * C + c] = acc;
        }
    }
    return 0;
}

/*
 * Backward of dsa3d_oracle_dwconv3d for an upstream gradient dY [N][C] (double):
 *   dX[m][c]       = sum over outputs p and taps whose source is m of W[c][u][v][w] * dY[p][c]
 *   dW[c][u][v][w] = sum_p dY[p][c] * X[p + (u - r_t, v - r_h, w - r_w)][c]   (in-volume sources)
 *   db[c]          = sum_p dY[p][c]
 * Written as the forward's loop with each product's contributions accumulated into its
 * operands; threads own channels, so no two threads touch the same accumulator.
 */
int dsa3d_oracle_dwconv3d_backward(int io, const void *x, const float *w, const double *dy, int F,
                                   int Hp, int Wp, int C, int kt, int kh, int kw, double *dx,
                                   double *dw, double *db, int n_threads) {
    if (conv_args(F, Hp, Wp, C, kt, kh, kw, io)) return -1;
    const int64_t N = (int64_t)F * Hp * Wp;
    const int K = kt * kh * kw;
    const int rt = (kt - 1) / 2, rh = (kh - 1) / 2, rw = (kw - 1) / 2;
    for (int64_t e = 0; e < N * C; e++) dx[e] = 0.0;
    for (int64_t e = 0; e < (int64_t)C * K; e++) dw[e] = 0.0;
    for (int c = 0; c < C; c++) db[c] = 0.0;
#pragma omp parallel for schedule(static) num_threads(n_threads > 0 ? n_threads : 1)
    for (int c = 0; c < C; c++) {
        for (int64_t n = 0; n < N; n++) {
            const int64_t x0 = n % Wp, y0 = (n / Wp) % Hp, t0 = n / ((int64_t)Wp * Hp);
            const double g = dy[n * C + c];
            db[c] += g;
            for (int u = 0; u < kt; u++)
                for (int v = 0; v < kh; v++)
                    for (int ww = 0; ww < kw; ww++) {
                        const int64_t ts = t0 + u - rt, ys = y0 + v - rh, xs = x0 + ww - rw;
                        if (ts < 0 || ts >= F || ys < 0 || ys >= Hp || xs < 0 || xs >= Wp) continue;
                        const int64_t src = (ts * Hp + ys) * Wp + xs;
                        const int64_t wi = ((int64_t)c * kt + u) * kh * kw + v * kw + ww;
                        dx[src * C + c] += (double)w[wi] * g;
                        dw[wi] += g * rd(x, io, src * C + c);
                    }
        }
    }
    return 0;
}
