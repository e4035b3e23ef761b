/*
 * CPU fp64 oracle for shifted local window attention with optional K/V-pooled
 * global memory.  TEST INFRASTRUCTURE ONLY: the parity tests, the package's
 * smoke check and the benchmark's CPU-baseline leg call it.  The product path
 * (the CUDA library) never links, loads or calls this file, and this file uses
 * nothing from it.
 *
 * What it computes (plain definitions, no blocking, fusion or reordering):
 *
 *  - Shifted local window attention replaces full visual self-attention: each
 *    token attends only to the tokens of its own window, and the window
 *    partition is offset by a per-block shift ("BASA: Backend-Agnostic Sparse
 *    Attention for Fast High-Resolution Diffusion Transformers", zhichai.net
 *    topic 178635722, sections "Summary" and "The BASA Method").
 *    Reading used here (the pages give no formula): on every grid axis a with
 *    size G, window size w and shift s, token coordinate x belongs to window
 *        wid(x) = floor( ((x - s) mod G) / w ),
 *    with a cyclic wrap at the border and no extra mask.  Shift 0 is the plain
 *    partitioned window attention that the same pages contrast it with.
 *
 *  - K/V-pooled global memory: the forum review of the same paper (zhichai.net
 *    topic 178635722, reply 178634520, the four-part method list) names
 *    "K/V pooled global memory" as a second component.  Reading used here:
 *    pooled tokens are the plain means of K and V over non-overlapping
 *    pt x ph x pw cells aligned to the unshifted grid origin, and they are
 *    appended to every query's key set under one joint softmax, with no
 *    count correction.
 *
 *  - Full attention (the quadratic baseline in the same pages) is the case of
 *    one window covering the whole grid.
 *
 *  - Joint text + image attention (MM-DiT blocks such as FLUX's): the method
 *    replaces the *visual* self-attention (same pages, "The BASA Method"), so
 *    reading used here: image queries attend to their window plus every text
 *    token, text queries attend to every image and text token, each under one
 *    softmax.
 *
 *  - Grids that a window size does not divide (only with `pad` set; the pages
 *    are silent here).  Reading used here, the one shifted-window attention
 *    commonly takes: each axis is padded at its far end to the next multiple
 *    of the window, Gp = ceil(G / w) * w; the shift rolls the padded axis
 *    (wid(x) = floor(((x - s) mod Gp) / w)); padded positions hold no token,
 *    so they are neither queries nor keys, and a window holds only its real
 *    members.  With w dividing G this is the definition above.
 *
 * Arithmetic: every input value is read as a double; dot products, the
 * max-subtracted softmax and the weighted sum are all in double precision.
 *
 * Layout: all token tensors are [B, T, Hg, Wg, H, d] row-major doubles.
 * Pooled tensors are [B, T/pt, Hg/ph, Wg/pw, H, d].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
  int64_t B, H, T, Hg, Wg, d;
  int64_t wt, wh, ww;   /* window size per axis (t, rows, columns) */
  int64_t st, sh, sw;   /* shift per axis */
  int64_t pt, ph, pw;   /* pooled cell size; all zero = no global memory */
  double scale;         /* softmax scale applied to q.k */
  int64_t Hkv;          /* K/V heads (grouped-query attention); 0 = H */
  int64_t pad;          /* 1: pad axes the window does not divide (see above) */
} oracle_params;

static int64_t floor_mod(int64_t a, int64_t n) {
  int64_t r = a % n;
  return r < 0 ? r + n : r;
}

/* Padded extent of an axis: G itself, or with `pad` the next multiple of w. */
static int64_t padded(int64_t G, int64_t w, int64_t pad) {
  return pad ? (G + w - 1) / w * w : G;
}

/* 0 when the window fits the grid: w divides G on every axis, or `pad` is set. */
static int grid_ok(const oracle_params* p) {
  if (p->wt <= 0 || p->wh <= 0 || p->ww <= 0) return -1;
  if (p->pad) return 0;
  return (p->T % p->wt || p->Hg % p->wh || p->Wg % p->ww) ? -1 : 0;
}

/*
 * Members of window (it, iy, ix) in (t, row, column) order: coordinate l of
 * the window on an axis is (i * w + s + l) mod Gp; positions past the real
 * grid are padding and skipped.  Writes (t, y, x) triples, returns the count.
 */
static int64_t window_members(const oracle_params* p, int64_t it, int64_t iy, int64_t ix,
                              int64_t* tok) {
  const int64_t Tp = padded(p->T, p->wt, p->pad), Hp = padded(p->Hg, p->wh, p->pad),
                Wp = padded(p->Wg, p->ww, p->pad);
  int64_t j = 0;
  for (int64_t lt = 0; lt < p->wt; ++lt)
    for (int64_t ly = 0; ly < p->wh; ++ly)
      for (int64_t lx = 0; lx < p->ww; ++lx) {
        const int64_t tt = floor_mod(it * p->wt + p->st + lt, Tp);
        const int64_t yy = floor_mod(iy * p->wh + p->sh + ly, Hp);
        const int64_t xx = floor_mod(ix * p->ww + p->sw + lx, Wp);
        if (tt >= p->T || yy >= p->Hg || xx >= p->Wg) continue;
        tok[3 * j] = tt;
        tok[3 * j + 1] = yy;
        tok[3 * j + 2] = xx;
        ++j;
      }
  return j;
}

static int64_t tok_index(const oracle_params* p, int64_t b, int64_t t, int64_t y,
                         int64_t x, int64_t h) {
  return ((((b * p->T + t) * p->Hg + y) * p->Wg + x) * p->H + h) * p->d;
}

/* K/V tensors have Hkv heads; query head h reads K/V head h / (H / Hkv). */
static int64_t kv_heads(const oracle_params* p) { return p->Hkv > 0 ? p->Hkv : p->H; }
static int64_t kv_head(const oracle_params* p, int64_t h) { return h / (p->H / kv_heads(p)); }
static int64_t kv_index(const oracle_params* p, int64_t b, int64_t t, int64_t y, int64_t x,
                        int64_t hk) {
  return ((((b * p->T + t) * p->Hg + y) * p->Wg + x) * kv_heads(p) + hk) * p->d;
}

/* Mean of x over each pooled cell. */
void oracle_pool(const double* x, double* xp, const oracle_params* p) {
  const int64_t Pt = p->T / p->pt, Ph = p->Hg / p->ph, Pw = p->Wg / p->pw;
  const double inv = 1.0 / (double)(p->pt * p->ph * p->pw);
  for (int64_t b = 0; b < p->B; ++b)
    for (int64_t ct = 0; ct < Pt; ++ct)
      for (int64_t cy = 0; cy < Ph; ++cy)
        for (int64_t cx = 0; cx < Pw; ++cx)
          for (int64_t h = 0; h < kv_heads(p); ++h)
            for (int64_t c = 0; c < p->d; ++c) {
              double acc = 0.0;
              for (int64_t i = 0; i < p->pt; ++i)
                for (int64_t j = 0; j < p->ph; ++j)
                  for (int64_t l = 0; l < p->pw; ++l)
                    acc += x[kv_index(p, b, ct * p->pt + i, cy * p->ph + j,
                                       cx * p->pw + l, h) + c];
              int64_t o = (((((b * Pt + ct) * Ph + cy) * Pw + cx) * kv_heads(p) + h) * p->d) + c;
              xp[o] = acc * inv;
            }
}

/*
 * Output (and optionally log-sum-exp) of one query token (b, t, y, x, h).
 * kp/vp may be NULL (no global memory).  Scratch z must hold m + P doubles.
 */
static void one_query(const double* q, const double* k, const double* v,
                      const double* kp, const double* vp, int64_t P,
                      const oracle_params* p, int64_t b, int64_t t, int64_t y,
                      int64_t x, int64_t h, double* z, int64_t* tok, double* out_row,
                      double* lse_out) {
  const int64_t d = p->d;
  const double* qv = q + tok_index(p, b, t, y, x, h);
  /* window id of the query on each (padded) axis */
  const int64_t it = floor_mod(t - p->st, padded(p->T, p->wt, p->pad)) / p->wt;
  const int64_t iy = floor_mod(y - p->sh, padded(p->Hg, p->wh, p->pad)) / p->wh;
  const int64_t ix = floor_mod(x - p->sw, padded(p->Wg, p->ww, p->pad)) / p->ww;
  const int64_t m = window_members(p, it, iy, ix, tok);

  /* logits over the window members */
  int64_t j = 0;
  for (int64_t a = 0; a < m; ++a) {
    const double* kv = k + kv_index(p, b, tok[3 * a], tok[3 * a + 1], tok[3 * a + 2], kv_head(p, h));
    double s = 0.0;
    for (int64_t c = 0; c < d; ++c) s += qv[c] * kv[c];
    z[j++] = p->scale * s;
  }
  /* logits over the pooled tokens */
  for (int64_t c2 = 0; c2 < P; ++c2) {
    const double* kv = kp + ((b * P + c2) * kv_heads(p) + kv_head(p, h)) * d;
    double s = 0.0;
    for (int64_t c = 0; c < d; ++c) s += qv[c] * kv[c];
    z[j++] = p->scale * s;
  }
  const int64_t nk = m + P;
  double mx = -INFINITY;
  for (int64_t i = 0; i < nk; ++i) mx = z[i] > mx ? z[i] : mx;
  double den = 0.0;
  for (int64_t i = 0; i < nk; ++i) {
    z[i] = exp(z[i] - mx);
    den += z[i];
  }
  for (int64_t c = 0; c < d; ++c) out_row[c] = 0.0;
  j = 0;
  for (int64_t a = 0; a < m; ++a) {
    const double* vv = v + kv_index(p, b, tok[3 * a], tok[3 * a + 1], tok[3 * a + 2], kv_head(p, h));
    const double w = z[j++] / den;
    for (int64_t c = 0; c < d; ++c) out_row[c] += w * vv[c];
  }
  for (int64_t c2 = 0; c2 < P; ++c2) {
    const double* vv = vp + ((b * P + c2) * kv_heads(p) + kv_head(p, h)) * d;
    const double a = z[j++] / den;
    for (int64_t c = 0; c < d; ++c) out_row[c] += a * vv[c];
  }
  if (lse_out) *lse_out = mx + log(den);
}

/*
 * Window attention over all queries, or over a selection.
 *   kp, vp : pooled K/V ([B, P, H, d] flattened cells) or NULL for none
 *   out    : [B, T, Hg, Wg, H, d] when sel == NULL, else [nsel, d]
 *   lse    : [B, H, N] when sel == NULL, else [nsel]; may be NULL
 *   sel    : nsel triples (b, n, h) with n the flattened token index
 *            ((t * Hg + y) * Wg + x), or NULL for every query
 * Returns 0, or -1 on an invalid size.
 */
static int window_attn_keys(const double* q, const double* k, const double* v,
                            const double* kp, const double* vp, int64_t P, double* out,
                            double* lse, const oracle_params* p, const int64_t* sel,
                            int64_t nsel, int nthreads);

int oracle_window_attn(const double* q, const double* k, const double* v,
                       const double* kp, const double* vp, double* out,
                       double* lse, const oracle_params* p, const int64_t* sel,
                       int64_t nsel, int nthreads) {
  if (grid_ok(p)) return -1;
  int64_t P = 0;
  if (kp) {
    if (p->pt <= 0 || p->ph <= 0 || p->pw <= 0) return -1;
    P = (p->T / p->pt) * (p->Hg / p->ph) * (p->Wg / p->pw);
  }
  return window_attn_keys(q, k, v, kp, vp, P, out, lse, p, sel, nsel, nthreads);
}

/*
 * Window attention whose extra keys are nx given tokens kx, vx ([B, nx, H, d])
 * instead of pooled cells: the visual queries of joint text + image attention
 * (every image token sees its own window plus every text token, one softmax).
 */
int oracle_window_attn_extra(const double* q, const double* k, const double* v,
                             const double* kx, const double* vx, int64_t nx, double* out,
                             double* lse, const oracle_params* p, const int64_t* sel,
                             int64_t nsel, int nthreads) {
  if (grid_ok(p)) return -1;
  if (nx < 0 || (nx > 0 && (!kx || !vx))) return -1;
  return window_attn_keys(q, k, v, nx ? kx : NULL, nx ? vx : NULL, nx, out, lse, p, sel, nsel,
                          nthreads);
}

static int window_attn_keys(const double* q, const double* k, const double* v,
                            const double* kp, const double* vp, int64_t P, double* out,
                            double* lse, const oracle_params* p, const int64_t* sel,
                            int64_t nsel, int nthreads) {
  const int64_t N = p->T * p->Hg * p->Wg;
  const int64_t m = p->wt * p->wh * p->ww;
  const int64_t total = sel ? nsel : p->B * N * p->H;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
#pragma omp parallel
  {
    double* z = (double*)malloc(sizeof(double) * (size_t)(m + P));
    int64_t* tok = (int64_t*)malloc(sizeof(int64_t) * (size_t)m * 3);
#pragma omp for schedule(dynamic, 64)
    for (int64_t i = 0; i < total; ++i) {
      int64_t b, n, h;
      if (sel) {
        b = sel[3 * i];
        n = sel[3 * i + 1];
        h = sel[3 * i + 2];
      } else {
        b = i / (N * p->H);
        n = (i / p->H) % N;
        h = i % p->H;
      }
      const int64_t x = n % p->Wg, y = (n / p->Wg) % p->Hg, t = n / (p->Wg * p->Hg);
      double* orow = sel ? out + i * p->d : out + tok_index(p, b, t, y, x, h);
      double* l = NULL;
      if (lse) l = sel ? lse + i : lse + (b * p->H + h) * N + n;
      one_query(q, k, v, kp, vp, P, p, b, t, y, x, h, z, tok, orow, l);
    }
    free(z);
    free(tok);
  }
  return 0;
}

/*
 * The text queries of joint text + image attention: every text query attends
 * to all N image tokens and all L text tokens under one softmax (plain dense
 * attention over the concatenated key set; the window restriction applies to
 * image queries only).
 *   qt, kt, vt : [B, L, H, d]      k, v : [B, T, Hg, Wg, H, d]
 *   out_t      : [B, L, H, d]      lse_t: [B, H, L] or NULL
 */
int oracle_joint_text_attn(const double* qt, const double* kt, const double* vt,
                           const double* k, const double* v, int64_t L, double* out_t,
                           double* lse_t, const oracle_params* p, int nthreads) {
  if (L < 0) return -1;
  const int64_t N = p->T * p->Hg * p->Wg, d = p->d, H = p->H, Hk = kv_heads(p);
  const int64_t total = p->B * L * H;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
#pragma omp parallel
  {
    double* z = (double*)malloc(sizeof(double) * (size_t)(N + L + 1));
#pragma omp for schedule(dynamic, 16)
    for (int64_t i = 0; i < total; ++i) {
      const int64_t b = i / (L * H), lq = (i / H) % L, h = i % H;
      const double* qv = qt + ((b * L + lq) * H + h) * d;
      for (int64_t j = 0; j < N + L; ++j) {
        const int64_t hk = kv_head(p, h);
        const double* kv = j < N ? k + ((b * N + j) * Hk + hk) * d
                                 : kt + ((b * L + (j - N)) * Hk + hk) * d;
        double s = 0.0;
        for (int64_t c = 0; c < d; ++c) s += qv[c] * kv[c];
        z[j] = p->scale * s;
      }
      double mx = -INFINITY;
      for (int64_t j = 0; j < N + L; ++j) mx = z[j] > mx ? z[j] : mx;
      double den = 0.0;
      for (int64_t j = 0; j < N + L; ++j) {
        z[j] = exp(z[j] - mx);
        den += z[j];
      }
      double* orow = out_t + ((b * L + lq) * H + h) * d;
      for (int64_t c = 0; c < d; ++c) orow[c] = 0.0;
      for (int64_t j = 0; j < N + L; ++j) {
        const int64_t hk = kv_head(p, h);
        const double* vv = j < N ? v + ((b * N + j) * Hk + hk) * d
                                 : vt + ((b * L + (j - N)) * Hk + hk) * d;
        const double a = z[j] / den;
        for (int64_t c = 0; c < d; ++c) orow[c] += a * vv[c];
      }
      if (lse_t) lse_t[(b * H + h) * L + lq] = mx + log(den);
    }
    free(z);
  }
  return 0;
}

/* Number of OpenMP threads the oracle would use (1 without OpenMP). */
int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/*
 * Gradients of window attention for one output gradient dO: with P_ij the
 * softmax weights of query i over its keys j (the keys of its window, plus the
 * pooled tokens when a pool cell is set),
 *   dV_j = sum_i P_ij dO_i
 *   dP_ij = dO_i . V_j,   D_i = dO_i . O_i = sum_j P_ij dP_ij
 *   dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i = scale sum_j dS_ij K_j,   dK_j = scale sum_i dS_ij Q_i
 * (the chain rule through softmax(scale * Q K^T) V restricted to each query's
 * keys).  A pooled token is the mean of its cell's keys (values), so its
 * gradient, summed over every query of the batch that sees it, flows back to
 * each token of the cell divided by the cell size.  The forward quantities are
 * recomputed here from q, k, v; nothing is taken from a forward pass.  All
 * tensors [B, T, Hg, Wg, H, d] (k, v, dk, dv with Hkv heads; with Hkv < H the
 * query heads of one group add into the same dK, dV).
 */
int oracle_window_attn_bwd(const double* q, const double* k, const double* v,
                           const double* dout, double* dq, double* dk, double* dv,
                           const oracle_params* p) {
  if (grid_ok(p)) return -1;
  const int pooled = p->pt > 0 && p->ph > 0 && p->pw > 0;
  if (pooled && (p->T % p->pt || p->Hg % p->ph || p->Wg % p->pw)) return -1;
  const int64_t d = p->d, N = p->T * p->Hg * p->Wg, mmax = p->wt * p->wh * p->ww;
  const int64_t nwt = padded(p->T, p->wt, p->pad) / p->wt, nwh = padded(p->Hg, p->wh, p->pad) / p->wh,
                nww = padded(p->Wg, p->ww, p->pad) / p->ww;
  const int64_t Ph = pooled ? p->Hg / p->ph : 0, Pw = pooled ? p->Wg / p->pw : 0;
  const int64_t Pn = pooled ? (p->T / p->pt) * Ph * Pw : 0; /* pooled tokens per batch */
  const int64_t nkmax = mmax + Pn;                          /* keys of a query, at most */
  const int64_t Hk = kv_heads(p);
  memset(dq, 0, sizeof(double) * (size_t)(p->B * N * p->H * d));
  memset(dk, 0, sizeof(double) * (size_t)(p->B * N * Hk * d));
  memset(dv, 0, sizeof(double) * (size_t)(p->B * N * Hk * d));
  double *kp = NULL, *vp = NULL, *dkp = NULL, *dvp = NULL;
  if (pooled) {
    const size_t np = (size_t)(p->B * Pn * Hk * d);
    kp = (double*)malloc(sizeof(double) * np);
    vp = (double*)malloc(sizeof(double) * np);
    dkp = (double*)calloc(np, sizeof(double));
    dvp = (double*)calloc(np, sizeof(double));
    oracle_pool(k, kp, p);
    oracle_pool(v, vp, p);
  }
  int64_t* tok = (int64_t*)malloc(sizeof(int64_t) * (size_t)mmax * 3);
  double* P = (double*)malloc(sizeof(double) * (size_t)(mmax * nkmax));
  double* dS = (double*)malloc(sizeof(double) * (size_t)(mmax * nkmax));
  for (int64_t b = 0; b < p->B; ++b)
    for (int64_t h = 0; h < p->H; ++h) {
      const int64_t hk = kv_head(p, h);
      for (int64_t wi = 0; wi < nwt * nwh * nww; ++wi) {
        const int64_t it = wi / (nwh * nww), iy = (wi / nww) % nwh, ix = wi % nww;
        /* members of window (it, iy, ix), enumerated from its id */
        const int64_t m = window_members(p, it, iy, ix, tok);
        const int64_t nk = m + Pn;  /* keys of every query of this window */
        /* key c2 < m: window member c2; key m + c: pooled token c of batch b */
#define KEY(c2) ((c2) < m ? k + kv_index(p, b, tok[3 * (c2)], tok[3 * (c2) + 1], tok[3 * (c2) + 2], hk) \
                          : kp + ((b * Pn + ((c2) - m)) * Hk + hk) * d)
#define VAL(c2) ((c2) < m ? v + kv_index(p, b, tok[3 * (c2)], tok[3 * (c2) + 1], tok[3 * (c2) + 2], hk) \
                          : vp + ((b * Pn + ((c2) - m)) * Hk + hk) * d)
        for (int64_t a = 0; a < m; ++a) {  /* query a: softmax row, then dS row */
          const double* qa = q + tok_index(p, b, tok[3 * a], tok[3 * a + 1], tok[3 * a + 2], h);
          const double* ga = dout + tok_index(p, b, tok[3 * a], tok[3 * a + 1], tok[3 * a + 2], h);
          double mx = -INFINITY;
          for (int64_t c2 = 0; c2 < nk; ++c2) {
            const double* kc = KEY(c2);
            double s = 0.0;
            for (int64_t c = 0; c < d; ++c) s += qa[c] * kc[c];
            P[a * nk + c2] = p->scale * s;
            if (P[a * nk + c2] > mx) mx = P[a * nk + c2];
          }
          double den = 0.0;
          for (int64_t c2 = 0; c2 < nk; ++c2) {
            P[a * nk + c2] = exp(P[a * nk + c2] - mx);
            den += P[a * nk + c2];
          }
          double Da = 0.0;
          for (int64_t c2 = 0; c2 < nk; ++c2) {
            P[a * nk + c2] /= den;
            const double* vc = VAL(c2);
            double dp = 0.0;
            for (int64_t c = 0; c < d; ++c) dp += ga[c] * vc[c];
            dS[a * nk + c2] = dp;
            Da += P[a * nk + c2] * dp;
          }
          for (int64_t c2 = 0; c2 < nk; ++c2)
            dS[a * nk + c2] = P[a * nk + c2] * (dS[a * nk + c2] - Da);
        }
        for (int64_t a = 0; a < m; ++a) {
          double* dqa = dq + tok_index(p, b, tok[3 * a], tok[3 * a + 1], tok[3 * a + 2], h);
          const double* qa = q + tok_index(p, b, tok[3 * a], tok[3 * a + 1], tok[3 * a + 2], h);
          const double* ga = dout + tok_index(p, b, tok[3 * a], tok[3 * a + 1], tok[3 * a + 2], h);
          for (int64_t c2 = 0; c2 < nk; ++c2) {
            const double* kc = KEY(c2);
            double* dkc = c2 < m ? dk + (kc - k) : dkp + (kc - kp);
            double* dvc = c2 < m ? dv + (kc - k) : dvp + (kc - kp);
            const double ds = dS[a * nk + c2], pw = P[a * nk + c2];
            for (int64_t c = 0; c < d; ++c) {
              dqa[c] += p->scale * ds * kc[c];
              dkc[c] += p->scale * ds * qa[c];
              dvc[c] += pw * ga[c];
            }
          }
        }
#undef KEY
#undef VAL
      }
    }
  if (pooled) {  /* through the mean pooling: each cell token gets 1 / count of its cell's */
    const double inv = 1.0 / (double)(p->pt * p->ph * p->pw);
    for (int64_t b = 0; b < p->B; ++b)
      for (int64_t t = 0; t < p->T; ++t)
        for (int64_t y = 0; y < p->Hg; ++y)
          for (int64_t x = 0; x < p->Wg; ++x) {
            const int64_t cell = ((t / p->pt) * Ph + y / p->ph) * Pw + x / p->pw;
            for (int64_t hk = 0; hk < Hk; ++hk) {
              const int64_t o = kv_index(p, b, t, y, x, hk), po = ((b * Pn + cell) * Hk + hk) * d;
              for (int64_t c = 0; c < d; ++c) {
                dk[o + c] += inv * dkp[po + c];
                dv[o + c] += inv * dvp[po + c];
              }
            }
          }
    free(kp);
    free(vp);
    free(dkp);
    free(dvp);
  }
  free(tok);
  free(P);
  free(dS);
  return 0;
}

/*
 * Gradients of joint text + image attention for the output gradients dout
 * (image queries) and dout_t (text queries).  The keys of image query i are
 * the members of its shifted window and the L text tokens; the keys of text
 * query t are the N image tokens and the L text tokens; one softmax per query.
 * Per query row the chain rule of oracle_window_attn_bwd: P over the row's
 * keys, dP_j = dO . V_j, D = sum_j P_j dP_j, dS_j = P_j (dP_j - D); dQ = scale
 * sum_j dS_j K_j; every key's dK (scale dS Q) and dV (P dO) sum over all the
 * queries that see it.  Image tensors [B, T, Hg, Wg, H or Hkv, d], text tensors
 * [B, L, H or Hkv, d].
 */
static void joint_row_bwd(const double* qa, const double* ga, const double** kp,
                          const double** vp, double** dkp, double** dvp, int64_t nk, int64_t d,
                          double scale, double* z, double* dp, double* dqa) {
  double mx = -INFINITY;
  for (int64_t j = 0; j < nk; ++j) {
    double s = 0.0;
    for (int64_t c = 0; c < d; ++c) s += qa[c] * kp[j][c];
    z[j] = scale * s;
    if (z[j] > mx) mx = z[j];
  }
  double den = 0.0;
  for (int64_t j = 0; j < nk; ++j) {
    z[j] = exp(z[j] - mx);
    den += z[j];
  }
  double D = 0.0;
  for (int64_t j = 0; j < nk; ++j) {
    z[j] /= den;
    double g = 0.0;
    for (int64_t c = 0; c < d; ++c) g += ga[c] * vp[j][c];
    dp[j] = g;
    D += z[j] * g;
  }
  for (int64_t j = 0; j < nk; ++j) {
    const double ds = z[j] * (dp[j] - D);
    for (int64_t c = 0; c < d; ++c) {
      dqa[c] += scale * ds * kp[j][c];
      dkp[j][c] += scale * ds * qa[c];
      dvp[j][c] += z[j] * ga[c];
    }
  }
}

int oracle_joint_attn_bwd(const double* q, const double* k, const double* v, const double* qt,
                          const double* kt, const double* vt, int64_t L, const double* dout,
                          const double* dout_t, double* dq, double* dk, double* dv, double* dqt,
                          double* dkt, double* dvt, const oracle_params* p) {
  if (L < 0) return -1;
  if (grid_ok(p)) return -1;
  const int64_t d = p->d, N = p->T * p->Hg * p->Wg, mmax = p->wt * p->wh * p->ww;
  const int64_t nwt = padded(p->T, p->wt, p->pad) / p->wt, nwh = padded(p->Hg, p->wh, p->pad) / p->wh,
                nww = padded(p->Wg, p->ww, p->pad) / p->ww;
  const int64_t H = p->H, Hk = kv_heads(p);
  memset(dq, 0, sizeof(double) * (size_t)(p->B * N * H * d));
  memset(dk, 0, sizeof(double) * (size_t)(p->B * N * Hk * d));
  memset(dv, 0, sizeof(double) * (size_t)(p->B * N * Hk * d));
  if (L) {
    memset(dqt, 0, sizeof(double) * (size_t)(p->B * L * H * d));
    memset(dkt, 0, sizeof(double) * (size_t)(p->B * L * Hk * d));
    memset(dvt, 0, sizeof(double) * (size_t)(p->B * L * Hk * d));
  }
  const int64_t nmax = N + L;
  const double** kp = (const double**)malloc(sizeof(double*) * (size_t)nmax);
  const double** vp = (const double**)malloc(sizeof(double*) * (size_t)nmax);
  double** dkp = (double**)malloc(sizeof(double*) * (size_t)nmax);
  double** dvp = (double**)malloc(sizeof(double*) * (size_t)nmax);
  double* z = (double*)malloc(sizeof(double) * (size_t)nmax);
  double* dpv = (double*)malloc(sizeof(double) * (size_t)nmax);
  int64_t* tok = (int64_t*)malloc(sizeof(int64_t) * (size_t)mmax * 3);
  for (int64_t b = 0; b < p->B; ++b)
    for (int64_t h = 0; h < H; ++h) {
      const int64_t hk = kv_head(p, h);
      for (int64_t l = 0; l < L; ++l) {  /* the text keys, seen by every query */
        const int64_t o = ((b * L + l) * Hk + hk) * d;
        kp[N + l] = kt + o; vp[N + l] = vt + o; dkp[N + l] = dkt + o; dvp[N + l] = dvt + o;
      }
      /* image queries: their window, then the text keys */
      for (int64_t wi = 0; wi < nwt * nwh * nww; ++wi) {
        const int64_t it = wi / (nwh * nww), iy = (wi / nww) % nwh, ix = wi % nww;
        const int64_t m = window_members(p, it, iy, ix, tok);
        /* window members in key slots N - m .. N - 1, so the text keys follow */
        for (int64_t c2 = 0; c2 < m; ++c2) {
          const int64_t o = kv_index(p, b, tok[3 * c2], tok[3 * c2 + 1], tok[3 * c2 + 2], hk);
          kp[N - m + c2] = k + o; vp[N - m + c2] = v + o; dkp[N - m + c2] = dk + o;
          dvp[N - m + c2] = dv + o;
        }
        for (int64_t a = 0; a < m; ++a) {
          const int64_t qo = tok_index(p, b, tok[3 * a], tok[3 * a + 1], tok[3 * a + 2], h);
          joint_row_bwd(q + qo, dout + qo, kp + (N - m), vp + (N - m), dkp + (N - m),
                        dvp + (N - m), m + L, d, p->scale, z, dpv, dq + qo);
        }
      }
      /* text queries: every image token, then the text keys */
      for (int64_t j = 0; j < N; ++j) {
        const int64_t o = ((b * N + j) * Hk + hk) * d;
        kp[j] = k + o; vp[j] = v + o; dkp[j] = dk + o; dvp[j] = dv + o;
      }
      for (int64_t t = 0; t < L; ++t) {
        const int64_t qo = ((b * L + t) * H + h) * d;
        joint_row_bwd(qt + qo, dout_t + qo, kp, vp, dkp, dvp, N + L, d, p->scale, z, dpv,
                      dqt + qo);
      }
    }
  free(kp); free(vp); free(dkp); free(dvp); free(z); free(dpv); free(tok);
  return 0;
}
