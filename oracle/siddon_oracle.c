/*
 * FP64 oracle for the cell-constant Siddon projector pair.
 *
 * TEST INFRASTRUCTURE ONLY.  Tests, the smoke check and the CPU-baseline leg of
 * the benchmark call this code; the product library never does, and this file
 * shares no code, header or table with it.  It is deliberately plain, slow and
 * single-threaded, in double precision throughout.
 *
 * What it computes (diffct "Execution", section "Precision, training and
 * reconstruction": the cell-constant Siddon model in physical coordinates;
 * section "Batch dimensions and axis spacing": native traversal integrates in
 * physical length units with per-axis pitch):
 *
 *     y[ray] = sum over voxels j of |ray ∩ voxel j| (physical length) * x[j]
 *
 * and back projection is the transpose of the same coefficients (same page:
 * "matched interpolation/traversal coefficients").  The oracle evaluates the
 * definition directly, following Siddon's merged set of plane crossings:
 *
 *   1. expand the detector geometry to the pixel centre of ray (v, r, c);
 *   2. form the segment a -> b (cone: source -> pixel centre, a finite ray;
 *      parallel: a long line through the pixel centre along the view's
 *      direction, long enough to contain the whole volume);
 *   3. clip t in [0, 1] against the volume's three slabs;
 *   4. collect every voxel-plane crossing strictly inside (t_in, t_out), add
 *      t_in and t_out, sort;
 *   5. each consecutive pair with positive gap is one segment: its voxel is
 *      the one containing the segment midpoint, its weight the gap times |b-a|.
 *
 * Geometry readings (the pages fix no vector convention):
 *   flat pixel centre  p = det_c + (c-(n_cols-1)/2) det_u + (r-(n_rows-1)/2) det_v
 *   cylindrical (cone only): the cylinder axis passes through the source along
 *   det_v; R = |component of (det_c - src) orthogonal to det_v|; the column
 *   angle is g = (c-(n_cols-1)/2)|det_u|/R (|det_u| is the arc pitch) and
 *   p = src + ((det_c-src).v^) v^ + R (cos g w^ + sin g u^) + (r-(n_rows-1)/2) det_v
 *   with w^ = unit orthogonal part of det_c - src and u^ = det_u/|det_u|.
 *   parallel beam: src holds the ray direction.
 *   voxel (i,j,k) covers [o + i s, o + (i+1) s) per axis (half-open).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  int32_t beam;      /* 0 parallel, 1 cone */
  int32_t detector;  /* 0 flat, 1 cylindrical */
  int64_t n_views, n_rows, n_cols;
  const double *src, *det_c, *det_u, *det_v; /* [n_views][3] each, (x,y,z) */
  int64_t n[3];                              /* nx, ny, nz */
  double origin[3];
  double spacing[3];
} oracle_geom;

static double dot3(const double *a, const double *b) { return a[0] * b[0] + a[1] * b[1] + a[2] * b[2]; }
static double norm3(const double *a) { return sqrt(dot3(a, a)); }

/* Step 1: world position of the centre of pixel (r, c) in view v. */
void oracle_pixel_centre(const oracle_geom *g, int64_t v, int64_t r, int64_t c, double *p) {
  const double *s = g->src + 3 * v, *dc = g->det_c + 3 * v, *du = g->det_u + 3 * v, *dv = g->det_v + 3 * v;
  double cc = (double)c - 0.5 * (double)(g->n_cols - 1);
  double rr = (double)r - 0.5 * (double)(g->n_rows - 1);
  if (g->detector == 0) {
    for (int k = 0; k < 3; ++k) p[k] = dc[k] + cc * du[k] + rr * dv[k];
    return;
  }
  double vhat[3], w[3], what[3], uhat[3];
  double nv = norm3(dv), nu = norm3(du);
  for (int k = 0; k < 3; ++k) vhat[k] = dv[k] / nv;
  for (int k = 0; k < 3; ++k) w[k] = dc[k] - s[k];
  double axial = dot3(w, vhat);
  for (int k = 0; k < 3; ++k) w[k] -= axial * vhat[k];
  double R = norm3(w);
  for (int k = 0; k < 3; ++k) what[k] = w[k] / R;
  for (int k = 0; k < 3; ++k) uhat[k] = du[k] / nu;
  double gam = cc * nu / R;
  for (int k = 0; k < 3; ++k)
    p[k] = s[k] + axial * vhat[k] + R * (cos(gam) * what[k] + sin(gam) * uhat[k]) + rr * dv[k];
}

/* Step 2: segment endpoints a, b. */
void oracle_ray_endpoints(const oracle_geom *g, int64_t v, int64_t r, int64_t c, double *a, double *b) {
  double p[3];
  oracle_pixel_centre(g, v, r, c, p);
  if (g->beam == 1) {
    for (int k = 0; k < 3; ++k) { a[k] = g->src[3 * v + k]; b[k] = p[k]; }
    return;
  }
  const double *d = g->src + 3 * v;
  double nd = norm3(d), centre[3], diag2 = 0.0, off[3];
  for (int k = 0; k < 3; ++k) {
    double ext = (double)g->n[k] * g->spacing[k];
    centre[k] = g->origin[k] + 0.5 * ext;
    diag2 += 0.25 * ext * ext;
    off[k] = p[k] - centre[k];
  }
  double D = 2.0 * (norm3(off) + sqrt(diag2)) + 1.0;
  for (int k = 0; k < 3; ++k) { a[k] = p[k] - D * d[k] / nd; b[k] = p[k] + D * d[k] / nd; }
}

static int cmp_double(const void *x, const void *y) {
  double a = *(const double *)x, b = *(const double *)y;
  return (a > b) - (a < b);
}

/* Steps 3-5 for one ray.  Calls emit(ctx, flat voxel index, physical length)
 * once per positive-length segment.  Returns the number of segments. */
typedef void (*oracle_emit_fn)(void *ctx, int64_t idx, double w);

static int64_t trace_ray(const oracle_geom *g, int64_t v, int64_t r, int64_t c, double *ts,
                         oracle_emit_fn emit, void *ctx) {
  double a[3], b[3], d[3];
  oracle_ray_endpoints(g, v, r, c, a, b);
  for (int k = 0; k < 3; ++k) d[k] = b[k] - a[k];
  double t_in = 0.0, t_out = 1.0;
  for (int k = 0; k < 3; ++k) {
    double lo = g->origin[k], hi = g->origin[k] + (double)g->n[k] * g->spacing[k];
    if (d[k] == 0.0) {
      if (a[k] < lo || a[k] >= hi) return 0;
      continue;
    }
    double t0 = (lo - a[k]) / d[k], t1 = (hi - a[k]) / d[k];
    double tmin = t0 < t1 ? t0 : t1, tmax = t0 < t1 ? t1 : t0;
    if (tmin > t_in) t_in = tmin;
    if (tmax < t_out) t_out = tmax;
  }
  if (!(t_out > t_in)) return 0;
  int64_t m = 0;
  ts[m++] = t_in;
  ts[m++] = t_out;
  for (int k = 0; k < 3; ++k) {
    if (d[k] == 0.0) continue;
    for (int64_t q = 0; q <= g->n[k]; ++q) {
      double t = (g->origin[k] + (double)q * g->spacing[k] - a[k]) / d[k];
      if (t > t_in && t < t_out) ts[m++] = t;
    }
  }
  qsort(ts, (size_t)m, sizeof(double), cmp_double);
  double len = norm3(d);
  int64_t nseg = 0;
  for (int64_t q = 0; q + 1 < m; ++q) {
    if (!(ts[q + 1] > ts[q])) continue;
    double tm = 0.5 * (ts[q] + ts[q + 1]);
    int64_t idx[3];
    for (int k = 0; k < 3; ++k) {
      double x = (a[k] + tm * d[k] - g->origin[k]) / g->spacing[k];
      int64_t i = (int64_t)floor(x);
      if (i < 0) i = 0;
      if (i > g->n[k] - 1) i = g->n[k] - 1;
      idx[k] = i;
    }
    int64_t flat = (idx[2] * g->n[1] + idx[1]) * g->n[0] + idx[0];
    emit(ctx, flat, (ts[q + 1] - ts[q]) * len);
    ++nseg;
  }
  return nseg;
}

static double *alloc_ts(const oracle_geom *g) {
  return (double *)malloc(sizeof(double) * (size_t)(g->n[0] + g->n[1] + g->n[2] + 8));
}

/* ---- forward: y = A x over views [v0, v1) ---- */
typedef struct { const float *vol; double acc; } fwd_ctx;
static void fwd_emit(void *p, int64_t idx, double w) {
  fwd_ctx *f = (fwd_ctx *)p;
  f->acc += w * (double)f->vol[idx];
}

int oracle_forward(const oracle_geom *g, const float *vol, double *sino, int64_t v0, int64_t v1) {
  double *ts = alloc_ts(g);
  if (!ts) return -1;
  for (int64_t v = v0; v < v1; ++v)
    for (int64_t r = 0; r < g->n_rows; ++r)
      for (int64_t c = 0; c < g->n_cols; ++c) {
        fwd_ctx f = {vol, 0.0};
        trace_ray(g, v, r, c, ts, fwd_emit, &f);
        sino[((v - v0) * g->n_rows + r) * g->n_cols + c] = f.acc;
      }
  free(ts);
  return 0;
}

/* Forward for an explicit list of rays (v, r, c) given as three index arrays. */
int oracle_forward_rays(const oracle_geom *g, const float *vol, int64_t n, const int64_t *vs,
                        const int64_t *rs, const int64_t *cs, double *out) {
  double *ts = alloc_ts(g);
  if (!ts) return -1;
  for (int64_t q = 0; q < n; ++q) {
    fwd_ctx f = {vol, 0.0};
    trace_ray(g, vs[q], rs[q], cs[q], ts, fwd_emit, &f);
    out[q] = f.acc;
  }
  free(ts);
  return 0;
}

/* ---- back: x = A^T y with coefficient power 0, 1 or 2, views [v0, v1) ---- */
typedef struct { double *vol; double y; int power; } back_ctx;
static void back_emit(void *p, int64_t idx, double w) {
  back_ctx *b = (back_ctx *)p;
  double coef = b->power == 0 ? 1.0 : (b->power == 1 ? w : w * w);
  b->vol[idx] += coef * b->y;
}

/* sino holds views [v0, v1) only; vol (n voxels, double) is accumulated into. */
int oracle_back(const oracle_geom *g, const float *sino, double *vol, int64_t v0, int64_t v1, int power) {
  double *ts = alloc_ts(g);
  if (!ts) return -1;
  for (int64_t v = v0; v < v1; ++v)
    for (int64_t r = 0; r < g->n_rows; ++r)
      for (int64_t c = 0; c < g->n_cols; ++c) {
        back_ctx b = {vol, (double)sino[((v - v0) * g->n_rows + r) * g->n_cols + c], power};
        if (b.y == 0.0) continue;
        trace_ray(g, v, r, c, ts, back_emit, &b);
      }
  free(ts);
  return 0;
}

/* ---- one ray's coefficient list ---- */
typedef struct { int64_t *idx; double *w; int64_t cap, n; } seg_ctx;
static void seg_emit(void *p, int64_t idx, double w) {
  seg_ctx *s = (seg_ctx *)p;
  if (s->n < s->cap) { s->idx[s->n] = idx; s->w[s->n] = w; }
  s->n++;
}

int64_t oracle_ray_segments(const oracle_geom *g, int64_t v, int64_t r, int64_t c, int64_t *idx, double *w,
                            int64_t cap) {
  double *ts = alloc_ts(g);
  if (!ts) return -1;
  seg_ctx s = {idx, w, cap, 0};
  trace_ray(g, v, r, c, ts, seg_emit, &s);
  free(ts);
  return s.n;
}

/* ---- exact count of positive-length segments over views [v0, v1) ---- */
static void count_emit(void *p, int64_t idx, double w) { (void)idx; (void)w; ++*(int64_t *)p; }

int64_t oracle_count_updates(const oracle_geom *g, int64_t v0, int64_t v1) {
  double *ts = alloc_ts(g);
  if (!ts) return -1;
  int64_t total = 0;
  for (int64_t v = v0; v < v1; ++v)
    for (int64_t r = 0; r < g->n_rows; ++r)
      for (int64_t c = 0; c < g->n_cols; ++c) trace_ray(g, v, r, c, ts, count_emit, &total);
  free(ts);
  return total;
}
