// C-ABI entry points of libctp: geometry validation and planning on the host,
// device upload of the per-view FP64 records, and the asynchronous forward /
// adjoint calls.  See include/ctp.h for the contract of every function.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "ctp_gather.h"
#include "ctp_internal.h"

using ctp::BackLaunch;
using ctp::FwdLaunch;
using ctp::ViewRec;
using ctp::VolDesc;

struct ctp_geom {
  int device = 0;
  int beam = 0, det = 0;
  int64_t n_views = 0, n_rows = 0, n_cols = 0;
  int64_t nx = 0, ny = 0, nz = 0;
  int64_t n_rays = 0, n_vox = 0;
  bool wide_index = false;
  VolDesc vol{};
  ctp::Dims dims{};
  FwdLaunch fwd{};
  BackLaunch back{};
  BackLaunch back2{};   // batched adjoint of member pairs: the brick halved along y (same shared memory)
  int adjoint_variant = CTP_ADJOINT_BRICK;
  int n_transposed = 0;
  double collision_ratio = 0.0;
  ViewRec *d_views = nullptr;
  double *d_trig = nullptr;
  float *d_volT = nullptr;
  float4 *d_vol4 = nullptr;   // volume interleaved by 4 slices (and its y-fastest twin), shared slice walks
  int64_t n_vol4 = 0;         // float4 elements of one interleaved copy
  bool wide4 = false;         // 64-bit offsets for the interleaved copies
  unsigned long long *d_counter = nullptr;
  ctp::GatherView *d_gview = nullptr;  // gather adjoint: per-view records
  float *d_ysum = nullptr;             // gather adjoint: slice sums of the sinogram [view][column][nz4]
  ctp::GatherLaunch gather{};
  int64_t scratch_bytes = 0;
  int batch_chunk = 1;  // volumes per fused batched forward launch (y-fastest copies held)
};

namespace {

thread_local char g_detail[512] = "";

ctp_status fail(ctp_status s, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_detail, sizeof(g_detail), fmt, ap);
  va_end(ap);
  return s;
}

ctp_status cuda_fail(cudaError_t e, const char *where) {
  return fail(CTP_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

double dot(const double *a, const double *b) { return a[0] * b[0] + a[1] * b[1] + a[2] * b[2]; }
double norm(const double *a) { return std::sqrt(dot(a, a)); }
void cross(const double *a, const double *b, double *c) {
  c[0] = a[1] * b[2] - a[2] * b[1];
  c[1] = a[2] * b[0] - a[0] * b[2];
  c[2] = a[0] * b[1] - a[1] * b[0];
}
bool finite3(const double *p) { return std::isfinite(p[0]) && std::isfinite(p[1]) && std::isfinite(p[2]); }

// Inverse of the 3x3 matrix with the given columns; false if (near) singular.
bool invert_columns(const double *c0, const double *c1, const double *c2, double *inv) {
  double m[9] = {c0[0], c1[0], c2[0], c0[1], c1[1], c2[1], c0[2], c1[2], c2[2]};
  double det = m[0] * (m[4] * m[8] - m[5] * m[7]) - m[1] * (m[3] * m[8] - m[5] * m[6]) +
               m[2] * (m[3] * m[7] - m[4] * m[6]);
  double scale = norm(c0) * norm(c1) * norm(c2);
  if (!(std::fabs(det) > 1e-12 * scale) || !std::isfinite(det)) return false;
  double id = 1.0 / det;
  inv[0] = (m[4] * m[8] - m[5] * m[7]) * id;
  inv[1] = (m[2] * m[7] - m[1] * m[8]) * id;
  inv[2] = (m[1] * m[5] - m[2] * m[4]) * id;
  inv[3] = (m[5] * m[6] - m[3] * m[8]) * id;
  inv[4] = (m[0] * m[8] - m[2] * m[6]) * id;
  inv[5] = (m[2] * m[3] - m[0] * m[5]) * id;
  inv[6] = (m[3] * m[7] - m[4] * m[6]) * id;
  inv[7] = (m[1] * m[6] - m[0] * m[7]) * id;
  inv[8] = (m[0] * m[4] - m[1] * m[3]) * id;
  return true;
}

// Adjoint variant dispatch (automatic plans): the ray-scatter adjoint unless
// each distinct voxel of a warp batch receives at least this many
// contributions on average, where the sort / segment-reduce adjoint takes
// over.  Measured on B200 (256^3 cone, 90 views, 384x384 detector, source at
// 500 voxels, magnification 2 / 4 / 8 / 16 / 32 / 64, collision ratios 1.5 /
// 2.6 / 4.7 / 8.1 / 12.8 / 18.4): the scatter adjoint is 8.0x / 5.7x / 3.5x /
// 2.0x / 1.10x faster than the sort adjoint at the first five and 1.78x
// slower at the last; the crossover, interpolated log-linearly, sits at 13.5.
// The brick adjoint was slower than the scatter adjoint at every one of these
// points and on workloads 1-4 (and equal within 2 % on workload 0); it stays
// available through the plan, for bitwise-reproducible results.
constexpr double kSortMinCollisionRatio = 13.5;

constexpr double kNearLimit = 1e6;  // one endpoint within this many voxels of the centre
constexpr double kFarLimit = 1e15;  // both endpoints within this many voxels

// Voxel-scaled distance |((p - centre) / spacing)|.
double vox_dist(const double *p, const double *centre_w, const double *sp) {
  double s = 0.0;
  for (int k = 0; k < 3; ++k) {
    double d = (p[k] - centre_w[k]) / sp[k];
    s += d * d;
  }
  return std::sqrt(s);
}

// World pixel centre, same formulas the kernels use (see ViewRec).
void host_pixel(const ViewRec &V, int det, int64_t r, int64_t c, double *p) {
  if (det == CTP_DET_FLAT) {
    for (int k = 0; k < 3; ++k) p[k] = V.p00[k] + (double)c * V.du[k] + (double)r * V.dv[k];
  } else {
    double g = V.gam0 + (double)c * V.dgam;
    for (int k = 0; k < 3; ++k)
      p[k] = V.p00[k] + (double)r * V.dv[k] + V.R * (std::cos(g) * V.w[k] + std::sin(g) * V.du[k]);
  }
}

ctp_status validate_desc(const ctp_geom_desc *d) {
  if (!d) return fail(CTP_ERR_INVALID_ARGUMENT, "desc is NULL");
  if (d->beam != CTP_BEAM_PARALLEL && d->beam != CTP_BEAM_CONE)
    return fail(CTP_ERR_INVALID_ARGUMENT, "beam %d is not CTP_BEAM_PARALLEL or CTP_BEAM_CONE", d->beam);
  if (d->detector != CTP_DET_FLAT && d->detector != CTP_DET_CYLINDRICAL)
    return fail(CTP_ERR_INVALID_ARGUMENT, "detector %d is not CTP_DET_FLAT or CTP_DET_CYLINDRICAL", d->detector);
  if (d->detector == CTP_DET_CYLINDRICAL && d->beam != CTP_BEAM_CONE)
    return fail(CTP_ERR_UNSUPPORTED, "a cylindrical detector needs a cone beam");
  const int64_t lim = 0x7fffffff;
  if (d->n_views <= 0 || d->n_rows <= 0 || d->n_cols <= 0)
    return fail(CTP_ERR_INVALID_ARGUMENT, "detector sizes must be positive (views %lld rows %lld cols %lld)",
                (long long)d->n_views, (long long)d->n_rows, (long long)d->n_cols);
  if (d->nx <= 0 || d->ny <= 0 || d->nz <= 0)
    return fail(CTP_ERR_INVALID_ARGUMENT, "volume sizes must be positive (%lld, %lld, %lld)", (long long)d->nx,
                (long long)d->ny, (long long)d->nz);
  if (d->n_views > lim || d->n_rows > lim || d->n_cols > lim || d->nx > lim || d->ny > lim || d->nz > lim)
    return fail(CTP_ERR_OUT_OF_RANGE, "a size exceeds 2^31-1");
  // element counts below 2^62 (offsets are 64-bit where needed)
  const double rays = (double)d->n_views * (double)d->n_rows * (double)d->n_cols;
  const double vox = (double)d->nx * (double)d->ny * (double)d->nz;
  if (rays >= 4.6e18 || vox >= 4.6e18) return fail(CTP_ERR_OUT_OF_RANGE, "element count too large");
  const double row_blocks = (double)((d->n_rows + 7) / 8) * (double)d->n_views * (double)((d->n_cols + 31) / 32);
  if (row_blocks > 2147483647.0) return fail(CTP_ERR_OUT_OF_RANGE, "too many detector tiles for one launch");
  for (int k = 0; k < 3; ++k) {
    if (!std::isfinite(d->origin[k])) return fail(CTP_ERR_INVALID_ARGUMENT, "origin[%d] is not finite", k);
    double s = d->spacing[k];
    if (!std::isfinite(s) || s < 1e-6 || s > 1e6)
      return fail(CTP_ERR_OUT_OF_RANGE, "spacing[%d] = %g outside [1e-6, 1e6]", k, s);
  }
  double smax = std::fmax(d->spacing[0], std::fmax(d->spacing[1], d->spacing[2]));
  double smin = std::fmin(d->spacing[0], std::fmin(d->spacing[1], d->spacing[2]));
  if (smax / smin > 1e4) return fail(CTP_ERR_OUT_OF_RANGE, "largest/smallest spacing %g exceeds 1e4", smax / smin);
  if (!d->src || !d->det_c || !d->det_u || !d->det_v)
    return fail(CTP_ERR_INVALID_ARGUMENT, "a per-view vector array is NULL");
  if (d->plan) {
    const ctp_plan *p = d->plan;
    if (p->adjoint_variant < CTP_ADJOINT_AUTO || p->adjoint_variant > CTP_ADJOINT_GATHER)
      return fail(CTP_ERR_INVALID_ARGUMENT, "plan.adjoint_variant %d", p->adjoint_variant);
    for (int k = 0; k < 3; ++k)
      if (p->brick[k] < 0 || p->brick[k] > 1024) return fail(CTP_ERR_INVALID_ARGUMENT, "plan.brick[%d]", k);
    if (p->view_groups < 0) return fail(CTP_ERR_INVALID_ARGUMENT, "plan.view_groups");
    if (p->forward_layout < 0 || p->forward_layout > 2) return fail(CTP_ERR_INVALID_ARGUMENT, "plan.forward_layout");
    if (p->batch_chunk != 0 && p->batch_chunk != 1 && p->batch_chunk != 2 && p->batch_chunk != 4)
      return fail(CTP_ERR_INVALID_ARGUMENT, "plan.batch_chunk %d is not 0, 1, 2 or 4", p->batch_chunk);
    if (p->slice_rows != 0 && p->slice_rows != 1 && p->slice_rows != 2 && p->slice_rows != 4 && p->slice_rows != 8)
      return fail(CTP_ERR_INVALID_ARGUMENT, "plan.slice_rows %d is not 0, 1, 2, 4 or 8", p->slice_rows);
  }
  return CTP_OK;
}

// One view's FP64 record and its guards; for a cylindrical detector also
// the row of column cos/sin values (2 * n_cols doubles at trig_row).
ctp_status build_view(const ctp_geom_desc *d, int64_t v, ViewRec &V, double *trig_row) {
  const int64_t nr = d->n_rows, nc = d->n_cols;
  const double cc = 0.5 * (double)(nc - 1), rc = 0.5 * (double)(nr - 1);
  const double n3[3] = {(double)d->nx, (double)d->ny, (double)d->nz};
  double centre_w[3];
  for (int k = 0; k < 3; ++k) centre_w[k] = d->origin[k] + 0.5 * n3[k] * d->spacing[k];
  const double smin = std::fmin(d->spacing[0], std::fmin(d->spacing[1], d->spacing[2]));
  V = ViewRec{};
  const double *s = d->src + 3 * v, *dc = d->det_c + 3 * v, *du = d->det_u + 3 * v, *dv = d->det_v + 3 * v;
  if (!finite3(s) || !finite3(dc) || !finite3(du) || !finite3(dv))
    return fail(CTP_ERR_INVALID_ARGUMENT, "view %lld: a vector is not finite", (long long)v);
  const double nu = norm(du), nvl = norm(dv);
  if (!(nu > 0.0) || !(nvl > 0.0))
    return fail(CTP_ERR_INVALID_ARGUMENT, "view %lld: det_u and det_v must be non-zero", (long long)v);
  V.vlen = nvl;
  for (int k = 0; k < 3; ++k) V.vhat[k] = dv[k] / nvl;
  for (int k = 0; k < 3; ++k) V.dv[k] = dv[k];
  V.src_norm = norm(s);
  if (d->beam == CTP_BEAM_PARALLEL) {
    const double ns = norm(s);
    if (!(ns > 0.0)) return fail(CTP_ERR_DEGENERATE_RAY, "view %lld: zero ray direction", (long long)v);
    for (int k = 0; k < 3; ++k) {
      V.s[k] = s[k] / ns;
      V.p00[k] = dc[k] - cc * du[k] - rc * dv[k];
      V.du[k] = du[k];
      const double dvox = V.s[k] / d->spacing[k];
      V.rcp_dir[k] = dvox != 0.0 ? 1.0 / dvox : HUGE_VAL;
    }
    if (!invert_columns(du, dv, V.s, V.minv))
      return fail(CTP_ERR_DEGENERATE_RAY, "view %lld: ray direction lies in the detector plane", (long long)v);
  } else if (d->detector == CTP_DET_FLAT) {
    double n[3];
    cross(du, dv, n);
    const double nn = norm(n);
    if (!(nn > 1e-12 * nu * nvl))
      return fail(CTP_ERR_INVALID_ARGUMENT, "view %lld: det_u and det_v are parallel", (long long)v);
    for (int k = 0; k < 3; ++k) {
      V.s[k] = s[k];
      V.p00[k] = dc[k] - cc * du[k] - rc * dv[k];
      V.du[k] = du[k];
    }
    // Source / pixel coincidence: only possible if the source lies in the detector plane.
    double rel[3] = {s[0] - dc[0], s[1] - dc[1], s[2] - dc[2]};
    const double h = std::fabs(dot(rel, n)) / nn;
    const double scale = std::fmax(norm(rel), std::fmax(nu, nvl));
    double sp00[3] = {V.p00[0] - s[0], V.p00[1] - s[1], V.p00[2] - s[2]};
    if (!(h > 1e-12 * scale)) {
      // coordinates of the source in the pixel lattice
      double inv[9];
      double a[3] = {s[0] - V.p00[0], s[1] - V.p00[1], s[2] - V.p00[2]};
      if (invert_columns(du, dv, n, inv)) {
        const double cs = inv[0] * a[0] + inv[1] * a[1] + inv[2] * a[2];
        const double rs = inv[3] * a[0] + inv[4] * a[1] + inv[5] * a[2];
        const double ci = std::round(cs), ri = std::round(rs);
        if (std::fabs(cs - ci) < 1e-9 && std::fabs(rs - ri) < 1e-9 && ci >= 0 && ci < (double)nc && ri >= 0 &&
            ri < (double)nr)
          return fail(CTP_ERR_DEGENERATE_RAY, "view %lld: the source coincides with pixel (%g, %g)", (long long)v,
                      ri, ci);
      }
      V.full_footprint = 1;
    } else if (!invert_columns(sp00, du, dv, V.minv)) {
      V.full_footprint = 1;
    }
    // distance guards at the detector corners (pixel distance is convex over the plane)
    const double ds = vox_dist(s, centre_w, d->spacing);
    double dp_max = 0.0;
    for (int corner = 0; corner < 4; ++corner) {
      double p[3];
      host_pixel(V, CTP_DET_FLAT, (corner & 1) ? nr - 1 : 0, (corner & 2) ? nc - 1 : 0, p);
      dp_max = std::fmax(dp_max, vox_dist(p, centre_w, d->spacing));
    }
    if (!(ds <= kFarLimit && dp_max <= kFarLimit))
      return fail(CTP_ERR_OUT_OF_RANGE, "view %lld: an endpoint is beyond 1e15 voxels", (long long)v);
    if (!(ds <= kNearLimit || dp_max <= kNearLimit))
      return fail(CTP_ERR_OUT_OF_RANGE, "view %lld: no endpoint within 1e6 voxels of the volume centre",
                  (long long)v);
  } else {
    // cylindrical detector centred on the source's axis
    const double uhat[3] = {du[0] / nu, du[1] / nu, du[2] / nu};
    double w0[3] = {dc[0] - s[0], dc[1] - s[1], dc[2] - s[2]};
    const double axial = dot(w0, V.vhat);
    double wp[3];
    for (int k = 0; k < 3; ++k) wp[k] = w0[k] - axial * V.vhat[k];
    const double R = norm(wp);
    if (!(R > 1e-9 * std::fmax(norm(w0), 1.0)))
      return fail(CTP_ERR_DEGENERATE_RAY, "view %lld: the detector centre lies on the source's axis", (long long)v);
    if (std::fabs(dot(uhat, V.vhat)) > 1e-9)
      return fail(CTP_ERR_INVALID_ARGUMENT, "view %lld: det_u must be orthogonal to det_v", (long long)v);
    if (std::fabs(dot(uhat, wp)) > 1e-9 * R)
      return fail(CTP_ERR_INVALID_ARGUMENT, "view %lld: det_u must be orthogonal to det_c - src", (long long)v);
    V.R = R;
    for (int k = 0; k < 3; ++k) {
      V.s[k] = s[k];
      V.w[k] = wp[k] / R;
      V.du[k] = uhat[k];
    }
    V.dgam = nu / R;
    V.gam0 = -cc * V.dgam;
    V.axial0 = axial - rc * nvl;
    for (int k = 0; k < 3; ++k) V.p00[k] = s[k] + V.axial0 * V.vhat[k];
    if (trig_row)
      for (int64_t c = 0; c < nc; ++c) {
        const double g = V.gam0 + (double)c * V.dgam;
        trig_row[2 * c] = std::cos(g);
        trig_row[2 * c + 1] = std::sin(g);
      }
    // distance guards: a bound first, the exact per-pixel check only if it fails
    const double ds = vox_dist(s, centre_w, d->spacing);
    const double row_ext = std::fmax(std::fabs(V.axial0), std::fabs(V.axial0 + (double)(nr - 1) * nvl));
    const double bound = ds + (R + row_ext) / smin;
    double dp_max = bound;
    if (!(ds <= kNearLimit || bound <= kNearLimit) || !(bound <= kFarLimit)) {
      dp_max = 0.0;
      for (int64_t r = 0; r < nr; ++r)
        for (int64_t c = 0; c < nc; ++c) {
          double p[3];
          const double g = V.gam0 + (double)c * V.dgam;
          for (int k = 0; k < 3; ++k)
            p[k] = V.p00[k] + (double)r * V.dv[k] + R * (std::cos(g) * V.w[k] + std::sin(g) * V.du[k]);
          dp_max = std::fmax(dp_max, vox_dist(p, centre_w, d->spacing));
        }
    }
    if (!(ds <= kFarLimit && dp_max <= kFarLimit))
      return fail(CTP_ERR_OUT_OF_RANGE, "view %lld: an endpoint is beyond 1e15 voxels", (long long)v);
    if (!(ds <= kNearLimit || dp_max <= kNearLimit))
      return fail(CTP_ERR_OUT_OF_RANGE, "view %lld: no endpoint within 1e6 voxels of the volume centre",
                  (long long)v);
  }
  // extent of one voxel's projection, used to bound the rays per voxel
  if (d->beam == CTP_BEAM_PARALLEL) {
    for (int i = 0; i < 2; ++i)
      V.vox_ext[i] = std::fabs(V.minv[3 * i]) * d->spacing[0] + std::fabs(V.minv[3 * i + 1]) * d->spacing[1] +
                     std::fabs(V.minv[3 * i + 2]) * d->spacing[2];
  } else if (d->detector == CTP_DET_FLAT) {
    for (int i = 0; i < 3; ++i)
      V.vox_ext[i] = std::fabs(V.minv[3 * i]) * d->spacing[0] + std::fabs(V.minv[3 * i + 1]) * d->spacing[1] +
                     std::fabs(V.minv[3 * i + 2]) * d->spacing[2];
  }
  // forward gather layout: y-fastest copy when the column step runs mostly along y
  const double ux = std::fabs(du[0] / d->spacing[0]), uy = std::fabs(du[1] / d->spacing[1]),
               uz = std::fabs(du[2] / d->spacing[2]);
  V.layout = (uy > ux && uy >= uz) ? 1 : 0;
  if (d->plan && d->plan->forward_layout == 1) V.layout = 0;
  if (d->plan && d->plan->forward_layout == 2) V.layout = 1;
  return CTP_OK;
}

// Per-view records and per-view guards of all views.  Host FP64 throughout.
ctp_status build_views(const ctp_geom_desc *d, std::vector<ViewRec> &views, std::vector<double> &trig) {
  const int64_t nv = d->n_views, nc = d->n_cols;
  views.assign((size_t)nv, ViewRec{});
  if (d->detector == CTP_DET_CYLINDRICAL) trig.assign((size_t)(2 * nv * nc), 0.0);
  for (int64_t v = 0; v < nv; ++v) {
    const ctp_status st = build_view(d, v, views[(size_t)v], trig.empty() ? nullptr : trig.data() + 2 * v * nc);
    if (st != CTP_OK) return st;
  }
  return CTP_OK;
}

// Brick counts, shared-memory pitch and view groups of an adjoint launch
// whose brick is already set (kb members share each CTA).
void plan_back_groups(const ctp_geom *g, BackLaunch &p, const ctp_plan *plan, int sm_count, int kb) {
  const int64_t n[3] = {g->nx, g->ny, g->nz};
  int64_t nb = 1;
  for (int k = 0; k < 3; ++k) {
    p.nbrick[k] = (int)((n[k] + p.brick[k] - 1) / p.brick[k]);
    nb *= p.nbrick[k];
  }
  p.pitch_x = p.brick[0] + 1;
  // Resident CTAs per SM: shared memory (brick + staged footprints + the
  // 1 KB the runtime reserves per CTA) and registers (three 256-thread CTAs).
  const int64_t per_cta = (int64_t)ctp::back_brick_smem_bytes(p.brick, kb) + 6 * 1024;
  const int64_t per_sm = std::max<int64_t>(1, std::min<int64_t>(3, (228 * 1024) / per_cta));
  const int64_t slots = (int64_t)sm_count * per_sm;
  // at least four waves of CTAs, so the last partial wave costs little:
  // split the views over groups when there are too few bricks
  int groups = 1;
  if (nb < 4 * slots)
    groups = (int)std::min<int64_t>((4 * slots + nb - 1) / nb, std::max<int64_t>(1, (g->n_views + 7) / 8));
  if (plan && plan->view_groups > 0) groups = (int)std::min<int64_t>(plan->view_groups, g->n_views);
  int vpg = (int)((g->n_views + groups - 1) / groups);
  groups = (int)((g->n_views + vpg - 1) / vpg);
  p.view_groups = groups;
  p.views_per_group = vpg;
}

void plan_back(ctp_geom *g, const ctp_plan *plan, int sm_count) {
  int b[3];
  // measured on B200: flat, wide bricks amortise the per-ray FP64 entry best
  if (g->beam == CTP_BEAM_PARALLEL) {
    b[0] = 128, b[1] = 128, b[2] = 1;
  } else {
    b[0] = 64, b[1] = 64, b[2] = 4;
  }
  if (plan)
    for (int k = 0; k < 3; ++k)
      if (plan->brick[k] > 0) b[k] = plan->brick[k];
  const int64_t n[3] = {g->nx, g->ny, g->nz};
  for (int k = 0; k < 3; ++k) b[k] = (int)std::min<int64_t>(b[k], n[k]);
  BackLaunch &p = g->back;
  p.dims = g->dims;
  p.vol = g->vol;
  for (int k = 0; k < 3; ++k) p.brick[k] = b[k];
  plan_back_groups(g, p, plan, sm_count, 1);
  // member pairs: half the brick along y, so two accumulators fit the same
  // shared memory as one
  BackLaunch &p2 = g->back2;
  p2 = p;
  p2.brick[1] = (b[1] + 1) / 2;
  plan_back_groups(g, p2, plan, sm_count, 2);
}

bool is_device_pointer(const void *ptr, int device) {
  if (!ptr) return false;
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, ptr) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) && a.device == device;
}

struct DeviceGuard {
  int prev = -1;
  bool switched = false;
  cudaError_t err = cudaSuccess;
  explicit DeviceGuard(int dev) {
    err = cudaGetDevice(&prev);
    if (err == cudaSuccess && prev != dev) {
      err = cudaSetDevice(dev);
      switched = err == cudaSuccess;
    }
  }
  ~DeviceGuard() {
    if (switched) cudaSetDevice(prev);
  }
};

void free_geom(ctp_geom *g) {
  if (!g) return;
  cudaFree(g->d_views);
  cudaFree(g->d_trig);
  cudaFree(g->d_volT);
  cudaFree(g->d_vol4);
  cudaFree(g->d_counter);
  cudaFree(g->d_gview);
  cudaFree(g->d_ysum);
  delete g;
}

// Collision ratio of the sort / segment-reduce adjoint: contributions per
// distinct-voxel run of its warp batches, measured on up to 16 evenly spaced
// views with the counting form of the kernel.  Synchronous (create only).
ctp_status measure_collision_ratio(ctp_geom *g, const std::vector<ViewRec> &views, const std::vector<double> &trig,
                                   double *ratio) {
  const int64_t nv = g->n_views;
  const int64_t ns = std::min<int64_t>(nv, 16);
  std::vector<ViewRec> sv((size_t)ns);
  std::vector<double> st;
  for (int64_t i = 0; i < ns; ++i) {
    const int64_t v = ns > 1 ? (i * (nv - 1)) / (ns - 1) : 0;
    sv[(size_t)i] = views[(size_t)v];
    if (!trig.empty())
      st.insert(st.end(), trig.begin() + 2 * v * g->n_cols, trig.begin() + 2 * (v + 1) * g->n_cols);
  }
  ViewRec *d_sv = nullptr;
  double *d_st = nullptr;
  unsigned long long *d_cnt = nullptr;
  cudaStream_t stream = nullptr;
  unsigned long long h[2] = {0, 0};
  cudaError_t e = cudaMalloc((void **)&d_sv, sizeof(ViewRec) * sv.size());
  if (e == cudaSuccess && !st.empty()) e = cudaMalloc((void **)&d_st, sizeof(double) * st.size());
  if (e == cudaSuccess) e = cudaMalloc((void **)&d_cnt, 2 * sizeof(unsigned long long));
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&stream, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaMemcpyAsync(d_sv, sv.data(), sizeof(ViewRec) * sv.size(), cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess && d_st)
    e = cudaMemcpyAsync(d_st, st.data(), sizeof(double) * st.size(), cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(d_cnt, 0, 2 * sizeof(unsigned long long), stream);
  if (e == cudaSuccess) {
    FwdLaunch f = g->fwd;
    f.dims.n_views = (int32_t)ns;
    e = ctp::launch_collision_count(f, d_sv, d_st, d_cnt, g->wide_index, stream);
  }
  if (e == cudaSuccess) e = cudaMemcpyAsync(h, d_cnt, sizeof(h), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (stream) cudaStreamDestroy(stream);
  cudaFree(d_sv);
  cudaFree(d_st);
  cudaFree(d_cnt);
  if (e != cudaSuccess) return cuda_fail(e, "collision-ratio measurement");
  *ratio = h[1] ? (double)h[0] / (double)h[1] : 1.0;
  return CTP_OK;
}

}  // namespace

// CTP_DEBUG builds: a bounds check that failed in an earlier kernel makes the
// next call return CTP_ERR_OUT_OF_RANGE (the record stays until
// ctp_debug_error_word reads and clears it).  Synchronous in those builds only.
#ifdef CTP_DEBUG
std::mutex g_debug_mu;
unsigned long long g_debug_pending = 0;

unsigned long long debug_collect() {
  std::lock_guard<std::mutex> lock(g_debug_mu);
  if (!g_debug_pending) g_debug_pending = ctp::debug_take_word_kernels();
  if (!g_debug_pending) g_debug_pending = ctp::debug_take_word_grad();
  if (!g_debug_pending) g_debug_pending = ctp::debug_take_word_gather();
  return g_debug_pending;
}
#endif

ctp_status debug_check() {
#ifdef CTP_DEBUG
  const unsigned long long w = debug_collect();
  if (w)
    return fail(CTP_ERR_OUT_OF_RANGE, "bounds check failed in an earlier kernel: site %llu, index %llu", w >> 48,
                w & 0xffffffffffffull);
#endif
  return CTP_OK;
}

// Host helpers shared with the entry point that allocates nothing
// (ctp_noalloc.cu); thin wrappers over the functions above.
namespace ctp {
ctp_status host_validate(const ctp_geom_desc *d) { return validate_desc(d); }
ctp_status host_view_record(const ctp_geom_desc *d, int64_t v, ViewRec &V, double *trig_row) {
  return build_view(d, v, V, trig_row);
}
ctp_status host_error(ctp_status s, const char *msg) { return fail(s, "%s", msg); }
ctp_status host_cuda_error(cudaError_t e, const char *where) { return cuda_fail(e, where); }
bool host_is_device_pointer(const void *ptr, int device) { return is_device_pointer(ptr, device); }
void host_clear_error() { g_detail[0] = '\0'; }
}  // namespace ctp

extern "C" {

const char *ctp_version(void) { return "0.2.0"; }

ctp_status ctp_debug_error_word(uint64_t *word) {
  g_detail[0] = '\0';
  if (!word) return fail(CTP_ERR_INVALID_ARGUMENT, "word is NULL");
#ifdef CTP_DEBUG
  debug_collect();
  std::lock_guard<std::mutex> lock(g_debug_mu);
  *word = (uint64_t)g_debug_pending;
  g_debug_pending = 0;
  return CTP_OK;
#else
  *word = 0;
  return fail(CTP_ERR_UNSUPPORTED, "bounds checks are compiled only into CTP_DEBUG builds");
#endif
}

const char *ctp_status_string(ctp_status s) {
  switch (s) {
    case CTP_OK: return "ok";
    case CTP_ERR_INVALID_ARGUMENT: return "invalid argument";
    case CTP_ERR_DEGENERATE_RAY: return "degenerate ray";
    case CTP_ERR_OUT_OF_RANGE: return "out of range";
    case CTP_ERR_UNSUPPORTED: return "unsupported";
    case CTP_ERR_OUT_OF_MEMORY: return "out of device memory";
    case CTP_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

const char *ctp_last_error_detail(void) { return g_detail; }

ctp_status ctp_geom_create(const ctp_geom_desc *desc, ctp_geom **out) {
  g_detail[0] = '\0';
  if (!out) return fail(CTP_ERR_INVALID_ARGUMENT, "out is NULL");
  ctp_status st = validate_desc(desc);
  if (st != CTP_OK) return st;
  std::vector<ViewRec> views;
  std::vector<double> trig;
  st = build_views(desc, views, trig);
  if (st != CTP_OK) return st;

  ctp_geom *g = new (std::nothrow) ctp_geom();
  if (!g) return fail(CTP_ERR_OUT_OF_MEMORY, "host allocation failed");
  g->device = desc->device;
  g->beam = desc->beam;
  g->det = desc->detector;
  g->n_views = desc->n_views;
  g->n_rows = desc->n_rows;
  g->n_cols = desc->n_cols;
  g->nx = desc->nx;
  g->ny = desc->ny;
  g->nz = desc->nz;
  g->n_rays = g->n_views * g->n_rows * g->n_cols;
  g->n_vox = g->nx * g->ny * g->nz;
  g->wide_index = g->n_vox >= (int64_t)0x7fffffff;
  VolDesc &vd = g->vol;
  vd.n[0] = (int32_t)g->nx;
  vd.n[1] = (int32_t)g->ny;
  vd.n[2] = (int32_t)g->nz;
  for (int k = 0; k < 3; ++k) {
    vd.origin[k] = desc->origin[k];
    vd.spacing[k] = desc->spacing[k];
    vd.inv_spacing[k] = 1.0 / desc->spacing[k];
    vd.centre[k] = 0.5 * (double)vd.n[k];
  }
  ctp::Dims &dm = g->dims;
  dm.beam = g->beam;
  dm.det = g->det;
  dm.n_views = (int32_t)g->n_views;
  dm.n_rows = (int32_t)g->n_rows;
  dm.n_cols = (int32_t)g->n_cols;
  for (const ViewRec &V : views) g->n_transposed += V.layout != 0;
  FwdLaunch &f = g->fwd;
  f.dims = dm;
  f.vol = vd;
  f.n_col_tiles = (int32_t)((g->n_cols + 31) / 32);
  f.n_row_bands = (int32_t)((g->n_rows + 7) / 8);
  f.any_transposed = g->n_transposed > 0;
  const ctp_plan *plan = desc->plan;
  // Rays in z-planes whose rows step along z share one (x, y) walk per column.
  bool slices = g->beam == CTP_BEAM_PARALLEL && g->det == CTP_DET_FLAT;
  for (const ViewRec &V : views)
    slices = slices && V.s[2] == 0.0 && V.dv[0] == 0.0 && V.dv[1] == 0.0;
  f.row_group = 1;
  g->adjoint_variant = CTP_ADJOINT_BRICK;
  g->batch_chunk = plan && plan->batch_chunk > 0 ? plan->batch_chunk : 1;

  DeviceGuard dg(g->device);
  int sm_count = 0;
  cudaError_t de = dg.err;
  if (de == cudaSuccess) de = cudaDeviceGetAttribute(&sm_count, cudaDevAttrMultiProcessorCount, g->device);
  if (de != cudaSuccess) {
    ctp_status s = cuda_fail(de, "device query");
    delete g;
    return s;
  }
  plan_back(g, plan, sm_count);
  if (slices) {
    // the largest row group that still launches two full waves of blocks
    // (four resident per SM), unless the plan names one
    const int want = plan ? plan->slice_rows : 0;
    int rg = 1;
    if (want > 0) {
      rg = want;
    } else {
      for (int r : {4, 2}) {
        const int64_t bands = (g->n_rows + 8 * r - 1) / (8 * r);
        if (bands * g->n_views * f.n_col_tiles >= 2 * 4 * (int64_t)sm_count) {
          rg = r;
          break;
        }
      }
    }
    f.row_group = rg;
#ifndef CTP_NO_INTERLEAVE
    // four rows per walk read and add 16 bytes at once from slices interleaved by 4
    f.interleaved = rg == 4;
#endif
    g->n_vol4 = (g->nz + 3) / 4 * g->nx * g->ny;
    g->wide4 = g->wide_index || 4 * g->n_vol4 >= (int64_t)0x7fffffff;
  }
  // Gather adjoint: decoupled slices whose views all suit it, when the plan
  // names it, or automatically once its grid fills the device (four blocks
  // per SM; below that the scatter adjoint measured faster) and the volume
  // has more than 128 slices (at most one float4 group of slices per lane
  // leaves the per-(cell, view) work unamortised).
  const int forced = plan ? plan->adjoint_variant : CTP_ADJOINT_AUTO;
  std::vector<ctp::GatherView> gviews;
  std::string gather_why = "the rays do not lie in z-planes with rows stepping along z";
  const bool gather_ok = slices && ctp::build_gather_views(views, vd, g->n_cols, gviews, gather_why);
  if (forced == CTP_ADJOINT_GATHER && !gather_ok) {
    delete g;
    return fail(CTP_ERR_UNSUPPORTED, "gather adjoint: %s", gather_why.c_str());
  }
  g->gather = ctp::plan_gather(vd, dm);
  const int64_t gather_blocks = (int64_t)g->gather.tiles_x * g->gather.tiles_y * g->gather.n_zchunks;
  const bool use_gather =
      gather_ok && (forced == CTP_ADJOINT_GATHER || (forced == CTP_ADJOINT_AUTO && g->gather.nz4 > 128 &&
                                                     gather_blocks >= 4 * (int64_t)sm_count));
  if (ctp::back_brick_smem_bytes(g->back.brick) > 200 * 1024) {
    delete g;
    return fail(CTP_ERR_INVALID_ARGUMENT, "adjoint brick needs more than 200 KB of shared memory");
  }
  auto alloc = [&](void **p, size_t bytes, const char *what) -> ctp_status {
    cudaError_t e = cudaMalloc(p, bytes);
    if (e == cudaErrorMemoryAllocation) {
      cudaGetLastError();
      return fail(CTP_ERR_OUT_OF_MEMORY, "cudaMalloc(%zu) for %s failed", bytes, what);
    }
    if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc");
    g->scratch_bytes += (int64_t)bytes;
    return CTP_OK;
  };
  size_t vbytes = sizeof(ViewRec) * views.size();
  st = alloc((void **)&g->d_views, vbytes, "view records");
  if (st == CTP_OK && !trig.empty()) st = alloc((void **)&g->d_trig, sizeof(double) * trig.size(), "column angles");
  if (st == CTP_OK && f.any_transposed)
    st = alloc((void **)&g->d_volT, sizeof(float) * (size_t)g->n_vox * (size_t)g->batch_chunk,
               "y-fastest volume copies");
  if (st == CTP_OK && f.interleaved)
    st = alloc((void **)&g->d_vol4, sizeof(float4) * (size_t)g->n_vol4 * (f.any_transposed ? 2 : 1),
               "volumes interleaved by 4 slices");
  if (st == CTP_OK) st = alloc((void **)&g->d_counter, sizeof(unsigned long long), "counter");
  if (st == CTP_OK && use_gather)
    st = alloc((void **)&g->d_gview, sizeof(ctp::GatherView) * gviews.size(), "gather view records");
  if (st == CTP_OK && use_gather)
    st = alloc((void **)&g->d_ysum, sizeof(float) * (size_t)g->n_views * (size_t)g->n_cols * (size_t)g->gather.nz4,
               "slice sums of the sinogram");
  cudaError_t e = cudaSuccess;
  if (st == CTP_OK) {
    e = cudaMemcpy(g->d_views, views.data(), vbytes, cudaMemcpyHostToDevice);
    if (e == cudaSuccess && !trig.empty())
      e = cudaMemcpy(g->d_trig, trig.data(), sizeof(double) * trig.size(), cudaMemcpyHostToDevice);
    if (e == cudaSuccess && use_gather)
      e = cudaMemcpy(g->d_gview, gviews.data(), sizeof(ctp::GatherView) * gviews.size(), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = ctp::prepare_back_brick(ctp::back_brick_smem_bytes(g->back.brick));
    if (e == cudaSuccess && g->batch_chunk >= 2)
      e = ctp::prepare_back_brick(ctp::back_brick_smem_bytes(g->back2.brick, 2), 2);
    if (e != cudaSuccess) st = cuda_fail(e, "geometry upload");
  }
  if (st == CTP_OK) st = measure_collision_ratio(g, views, trig, &g->collision_ratio);
  if (st != CTP_OK) {
    free_geom(g);
    return st;
  }
  // adjoint variant: forced by the plan, else the gather where it applies,
  // else by the measured collision ratio
  if (use_gather)
    g->adjoint_variant = CTP_ADJOINT_GATHER;
  else if (forced == CTP_ADJOINT_BRICK || forced == CTP_ADJOINT_SORT || forced == CTP_ADJOINT_SCATTER)
    g->adjoint_variant = forced;
  else
    g->adjoint_variant = g->collision_ratio >= kSortMinCollisionRatio ? CTP_ADJOINT_SORT : CTP_ADJOINT_SCATTER;
  *out = g;
  return CTP_OK;
}

void ctp_geom_destroy(ctp_geom *g) {
  if (!g) return;
  DeviceGuard dg(g->device);
  cudaDeviceSynchronize();
  free_geom(g);
}

ctp_status ctp_geom_query(const ctp_geom *g, ctp_geom_info *info) {
  if (!g || !info) return fail(CTP_ERR_INVALID_ARGUMENT, "NULL argument");
  info->n_rays = g->n_rays;
  info->n_vox = g->n_vox;
  info->scratch_bytes = g->scratch_bytes;
  info->adjoint_variant = g->adjoint_variant;
  for (int k = 0; k < 3; ++k) info->brick[k] = g->back.brick[k];
  info->view_groups = g->back.view_groups;
  info->n_transposed_views = g->n_transposed;
  info->collision_ratio = g->collision_ratio;
  info->batch_chunk = g->batch_chunk;
  info->slice_rows = g->fwd.row_group;
  info->interleaved_slices = g->fwd.interleaved;
  info->reserved = 0;
  return CTP_OK;
}

ctp_status ctp_forward(const ctp_geom *g, const float *vol, float *sino, void *stream) {
  g_detail[0] = '\0';
  if (!g) return fail(CTP_ERR_INVALID_ARGUMENT, "geometry is NULL");
  DeviceGuard dg(g->device);
  if (dg.err != cudaSuccess) return cuda_fail(dg.err, "cudaSetDevice");
  if (!is_device_pointer(vol, g->device))
    return fail(CTP_ERR_INVALID_ARGUMENT, "vol is not device memory of device %d", g->device);
  if (!is_device_pointer(sino, g->device))
    return fail(CTP_ERR_INVALID_ARGUMENT, "sino is not device memory of device %d", g->device);
  {
    const ctp_status dbg = debug_check();
    if (dbg != CTP_OK) return dbg;
  }
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "pending error before ctp_forward");
  if (g->fwd.interleaved) {
    e = ctp::launch_forward_rows4(g->fwd, g->d_views, vol, g->d_vol4, g->d_vol4 + g->n_vol4, sino, g->wide4, s);
    if (e != cudaSuccess) return cuda_fail(e, "forward launch");
    return CTP_OK;
  }
  if (g->fwd.any_transposed) {
    e = ctp::launch_transpose_xy(vol, g->d_volT, g->vol, s);
    if (e != cudaSuccess) return cuda_fail(e, "transpose launch");
  }
  if (g->fwd.row_group > 1)
    e = ctp::launch_forward_rows(g->fwd, g->d_views, vol, g->d_volT, sino, g->wide_index, s);
  else
    e = ctp::launch_forward(g->fwd, g->d_views, g->d_trig, vol, g->d_volT, sino, 1, g->wide_index, s);
  if (e != cudaSuccess) return cuda_fail(e, "forward launch");
  return CTP_OK;
}

namespace {
// n_batch >= 0 and the batch's largest array below 2^62 elements.
ctp_status check_batch(const ctp_geom *g, int64_t n_batch) {
  if (n_batch < 0) return fail(CTP_ERR_INVALID_ARGUMENT, "n_batch %lld is negative", (long long)n_batch);
  const double most = (double)n_batch * (double)(g->n_vox > g->n_rays ? g->n_vox : g->n_rays);
  if (most >= 4.6e18) return fail(CTP_ERR_INVALID_ARGUMENT, "batch of %lld is too large", (long long)n_batch);
  return CTP_OK;
}
}  // namespace

ctp_status ctp_forward_batch(const ctp_geom *g, const float *vol, float *sino, int64_t n_batch, void *stream) {
  g_detail[0] = '\0';
  if (!g) return fail(CTP_ERR_INVALID_ARGUMENT, "geometry is NULL");
  ctp_status st = check_batch(g, n_batch);
  if (st != CTP_OK || n_batch == 0) return st;
  DeviceGuard dg(g->device);
  if (dg.err != cudaSuccess) return cuda_fail(dg.err, "cudaSetDevice");
  if (!is_device_pointer(vol, g->device))
    return fail(CTP_ERR_INVALID_ARGUMENT, "vol is not device memory of device %d", g->device);
  if (!is_device_pointer(sino, g->device))
    return fail(CTP_ERR_INVALID_ARGUMENT, "sino is not device memory of device %d", g->device);
  {
    const ctp_status dbg = debug_check();
    if (dbg != CTP_OK) return dbg;
  }
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "pending error before ctp_forward_batch");
  if (g->fwd.row_group > 1) {
    // decoupled slices: one (x, y) walk already serves several rows of one
    // volume, faster per member than walks shared across members
    for (int64_t b = 0; b < n_batch; ++b) {
      st = ctp_forward(g, vol + (size_t)b * (size_t)g->n_vox, sino + (size_t)b * (size_t)g->n_rays, stream);
      if (st != CTP_OK) return st;
    }
    return CTP_OK;
  }
  for (int64_t b0 = 0; b0 < n_batch;) {
    // the largest supported chunk that fits the remaining members
    int kb = g->batch_chunk;
    while (kb > 1 && b0 + kb > n_batch) kb >>= 1;
    const float *v0 = vol + (size_t)b0 * (size_t)g->n_vox;
    if (g->fwd.any_transposed)
      for (int j = 0; j < kb && e == cudaSuccess; ++j)
        e = ctp::launch_transpose_xy(v0 + (size_t)j * (size_t)g->n_vox, g->d_volT + (size_t)j * (size_t)g->n_vox,
                                     g->vol, s);
    if (e == cudaSuccess)
      e = ctp::launch_forward(g->fwd, g->d_views, g->d_trig, v0, g->d_volT, sino + (size_t)b0 * (size_t)g->n_rays,
                              kb, g->wide_index, s);
    if (e != cudaSuccess) return cuda_fail(e, "batched forward launch");
    b0 += kb;
  }
  return CTP_OK;
}

ctp_status ctp_back_batch(const ctp_geom *g, const float *sino, float *vol, int64_t n_batch, void *stream) {
  g_detail[0] = '\0';
  if (!g) return fail(CTP_ERR_INVALID_ARGUMENT, "geometry is NULL");
  ctp_status st = check_batch(g, n_batch);
  if (st != CTP_OK || n_batch == 0) return st;
  int64_t b = 0;
  if (g->batch_chunk >= 2 && g->adjoint_variant == CTP_ADJOINT_BRICK && n_batch >= 2) {
    // member pairs share each ray's set-up and walk (one launch per pair)
    DeviceGuard dg(g->device);
    if (dg.err != cudaSuccess) return cuda_fail(dg.err, "cudaSetDevice");
    if (!is_device_pointer(sino, g->device))
      return fail(CTP_ERR_INVALID_ARGUMENT, "sino is not device memory of device %d", g->device);
    if (!is_device_pointer(vol, g->device))
      return fail(CTP_ERR_INVALID_ARGUMENT, "vol is not device memory of device %d", g->device);
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "pending error before ctp_back_batch");
    for (; b + 2 <= n_batch; b += 2) {
      float *v0 = vol + (size_t)b * (size_t)g->n_vox;
      if (g->back2.view_groups > 1) e = cudaMemsetAsync(v0, 0, 2 * sizeof(float) * (size_t)g->n_vox, s);
      if (e == cudaSuccess)
        e = ctp::launch_back_brick(g->back2, g->d_views, g->d_trig, sino + (size_t)b * (size_t)g->n_rays, v0, 1, 2,
                                   g->wide_index, s);
      if (e != cudaSuccess) return cuda_fail(e, "batched adjoint launch");
    }
  }
  for (; b < n_batch; ++b) {
    st = ctp_back_power(g, sino + (size_t)b * (size_t)g->n_rays, vol + (size_t)b * (size_t)g->n_vox, 1, stream);
    if (st != CTP_OK) return st;
  }
  return CTP_OK;
}

ctp_status ctp_back(const ctp_geom *g, const float *sino, float *vol, void *stream) {
  return ctp_back_power(g, sino, vol, 1, stream);
}

ctp_status ctp_back_power(const ctp_geom *g, const float *sino, float *vol, int power, void *stream) {
  g_detail[0] = '\0';
  if (!g) return fail(CTP_ERR_INVALID_ARGUMENT, "geometry is NULL");
  if (power != 1 && power != 2) return fail(CTP_ERR_INVALID_ARGUMENT, "power %d is not 1 or 2", power);
  DeviceGuard dg(g->device);
  if (dg.err != cudaSuccess) return cuda_fail(dg.err, "cudaSetDevice");
  if (!is_device_pointer(sino, g->device))
    return fail(CTP_ERR_INVALID_ARGUMENT, "sino is not device memory of device %d", g->device);
  if (!is_device_pointer(vol, g->device))
    return fail(CTP_ERR_INVALID_ARGUMENT, "vol is not device memory of device %d", g->device);
  {
    const ctp_status dbg = debug_check();
    if (dbg != CTP_OK) return dbg;
  }
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "pending error before ctp_back");
  if (g->adjoint_variant == CTP_ADJOINT_GATHER) {
    // slice sums, then one warp per (x, y) cell writes every slice of it
    e = ctp::launch_back_gather(g->fwd, g->gather, g->d_views, g->d_gview, sino, g->d_ysum, vol, power, s);
    if (e != cudaSuccess) return cuda_fail(e, "adjoint launch");
    return CTP_OK;
  }
  const bool sorted = g->adjoint_variant == CTP_ADJOINT_SORT;
  const bool scatter = g->adjoint_variant == CTP_ADJOINT_SCATTER;
  if (scatter && g->fwd.interleaved) {
    // accumulate into the zeroed interleaved copies; their sum overwrites vol
    e = cudaMemsetAsync(g->d_vol4, 0, sizeof(float4) * (size_t)g->n_vol4 * (g->fwd.any_transposed ? 2 : 1), s);
    if (e != cudaSuccess) return cuda_fail(e, "accumulator zero-fill");
    e = ctp::launch_back_scatter_rows4(g->fwd, g->d_views, sino, vol, g->d_vol4, g->d_vol4 + g->n_vol4, power,
                                       g->wide4, s);
    if (e != cudaSuccess) return cuda_fail(e, "adjoint launch");
    return CTP_OK;
  }
  if (sorted || scatter || g->back.view_groups > 1) {
    e = cudaMemsetAsync(vol, 0, sizeof(float) * (size_t)g->n_vox, s);
    if (e == cudaSuccess && scatter && g->fwd.any_transposed)
      e = cudaMemsetAsync(g->d_volT, 0, sizeof(float) * (size_t)g->n_vox, s);
    if (e != cudaSuccess) return cuda_fail(e, "volume zero-fill");
  }
  if (scatter)
    e = ctp::launch_back_scatter(g->fwd, g->d_views, g->d_trig, sino, vol, g->d_volT, power, g->wide_index, s);
  else if (sorted)
    e = ctp::launch_back_sort(g->fwd, g->d_views, g->d_trig, sino, vol, power, g->wide_index, s);
  else
    e = ctp::launch_back_brick(g->back, g->d_views, g->d_trig, sino, vol, power, 1, g->wide_index, s);
  if (e != cudaSuccess) return cuda_fail(e, "adjoint launch");
  return CTP_OK;
}

ctp_status ctp_geometry_gradient(const ctp_geom *g, const float *vol, const float *sino_grad, double *grad,
                                 void *stream) {
  g_detail[0] = '\0';
  if (!g) return fail(CTP_ERR_INVALID_ARGUMENT, "geometry is NULL");
  DeviceGuard dg(g->device);
  if (dg.err != cudaSuccess) return cuda_fail(dg.err, "cudaSetDevice");
  if (!is_device_pointer(vol, g->device) || !is_device_pointer(sino_grad, g->device) ||
      !is_device_pointer(grad, g->device))
    return fail(CTP_ERR_INVALID_ARGUMENT, "vol, sino_grad and grad must be device memory of device %d", g->device);
  {
    const ctp_status dbg = debug_check();
    if (dbg != CTP_OK) return dbg;
  }
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "pending error before ctp_geometry_gradient");
  e = cudaMemsetAsync(grad, 0, sizeof(double) * 12 * (size_t)g->n_views, s);
  if (e == cudaSuccess && g->fwd.interleaved) {
    // decoupled slices: one (x, y) walk per 4 rows on the interleaved copies
    e = ctp::launch_interleave(g->fwd, vol, g->d_vol4, g->d_vol4 + g->n_vol4, s);
    if (e == cudaSuccess)
      e = ctp::launch_geometry_gradient_rows4(g->fwd, g->d_views, g->d_vol4, g->d_vol4 + g->n_vol4, sino_grad, grad,
                                              g->wide4, s);
    if (e != cudaSuccess) return cuda_fail(e, "geometry gradient launch");
    return CTP_OK;
  }
  if (e == cudaSuccess && g->fwd.any_transposed) e = ctp::launch_transpose_xy(vol, g->d_volT, g->vol, s);
  if (e == cudaSuccess)
    e = ctp::launch_geometry_gradient(g->fwd, g->d_views, g->d_trig, vol, g->d_volT, sino_grad, grad,
                                      g->wide_index, s);
  if (e != cudaSuccess) return cuda_fail(e, "geometry gradient launch");
  return CTP_OK;
}

ctp_status ctp_count_updates(const ctp_geom *g, int64_t *host_out, void *stream) {
  g_detail[0] = '\0';
  if (!g || !host_out) return fail(CTP_ERR_INVALID_ARGUMENT, "NULL argument");
  DeviceGuard dg(g->device);
  if (dg.err != cudaSuccess) return cuda_fail(dg.err, "cudaSetDevice");
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(g->d_counter, 0, sizeof(unsigned long long), s);
  if (e == cudaSuccess) e = ctp::launch_count(g->fwd, g->d_views, g->d_trig, g->d_counter, s);
  unsigned long long n = 0;
  if (e == cudaSuccess) e = cudaMemcpyAsync(&n, g->d_counter, sizeof(n), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "count");
  *host_out = (int64_t)n;
  return CTP_OK;
}

}  // extern "C"
