// Geometry gradients of the forward projection (sm_100a).
//
// For an upstream gradient g = dL/dy on the sinogram, the gradient of L with
// respect to each view's vectors (src, det_c, det_u, det_v) is the sum over
// the view's rays of g * dy/d(vector).  diffct "Execution", section
// "Streaming analytical reconstruction", lists geometry gradients of the
// projection beside the volume gradient (the adjoint) and costs them at one
// extra traversal; this is that traversal.
//
// The Siddon line integral of a ray is piecewise linear in its endpoints.
// Parametrise the ray as X(t) = P_a + t (P_b - P_a) with t in [t_lo, t_hi]
// (cone: the segment from the endpoint nearer the volume centre, P_a, to the
// other one, t in [0, 1]; parallel: the line through the pixel p along the
// unit direction u, t in (-inf, inf)).  Treating voxels outside the volume as
// zero, every plane crossing i of axis k at parameter t_i changes the voxel
// value by dx_i = x_before - x_after, and
//   y / |P_b - P_a| = sum_i t_i dx_i + x_end,
// with x_end the value of the voxel holding the endpoint t = 1 (zero when
// that endpoint lies outside; parallel rays have no such term).  The
// crossing parameter of the plane X_k = q moves as
//   dt_i = -((1 - t_i) dP_a,k + t_i dP_b,k) / D_k,   D = P_b - P_a,
// and the length as d|D| = u . (dP_b - dP_a) with u = D / |D|.  With the
// per-axis sums S0_k = sum dx_i and S1_k = sum t_i dx_i over that axis's
// crossings (the volume's faces included) and E = sum_k S1_k + x_end:
//   dy/dP_a = sum_k e_k |D| (S1_k - S0_k) / D_k - u E
//   dy/dP_b = -sum_k e_k |D| S1_k / D_k + u E.
// For a parallel ray (|u| = 1, t measured from the pixel):
//   dy/dp = -sum_k e_k S0_k / u_k,   dy/du = -sum_k e_k S1_k / u_k,
// and the given direction s = |s| u moves u by (I - u u^T) ds / |s|.  Axes
// with D_k = 0 have no crossings and contribute nothing (y is constant in
// that coordinate away from the voxel boundaries).
//
// A flat detector's pixel (r, c) sits at det_c + (c - cc) det_u + (r - rc)
// det_v with (rc, cc) the detector's centre, so the pixel gradient also
// gives the det_c, det_u and det_v gradients; a cylindrical detector's pixel
// is a nonlinear function of the four vectors (cylinder_chain below).  Kinks (a ray through a voxel
// edge, an endpoint on a plane) have no derivative; the formula then returns
// one of the one-sided values.
//
// Kernel: one thread per ray on the forward's grid (a block is 32 columns x 8
// rows of one view), FP64 setup shared with the projectors, an FP32
// major-axis slab walk for the per-axis crossing sums, the per-ray gradient
// in FP64, then a block reduction and 12 FP64 atomics per block into
// grad[view][4][3].
#include "ctp_ray.cuh"

namespace ctp {
namespace {

// Tuning knobs (compile-time; the defaults are the measured choices: 4 CTAs
// per SM with the setup recomputed after the walk, 2 / 1 slab unroll).
#ifndef CTP_GRAD_MIN_BLOCKS
#define CTP_GRAD_MIN_BLOCKS 4
#endif
#ifndef CTP_GRAD_UNROLL2
#define CTP_GRAD_UNROLL2 2
#endif
#ifndef CTP_GRAD_UNROLL3
#define CTP_GRAD_UNROLL3 1
#endif
constexpr int kGradUnroll2 = CTP_GRAD_UNROLL2;
constexpr int kGradUnroll3 = CTP_GRAD_UNROLL3;
constexpr int kGradCols = 32;
constexpr int kGradRows = 8;
constexpr int kGradThreads = kGradCols * kGradRows;

// Slab clip as in the projectors, also returning the axis whose faces bound
// the segment at each end (-1 where the ray's own end t_lo / t_hi does).
__device__ __forceinline__ bool clip_faces(const Ray& R, const int hi[3], double& t_in, double& t_out, int& k_in,
                                           int& k_out) {
  t_in = R.t_lo;
  t_out = R.t_hi;
  k_in = -1;
  k_out = -1;
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    if (R.D[k] == 0.0) {
      if (!(R.A[k] >= 0.0 && R.A[k] < (double)hi[k])) return false;
    } else {
      const double ta = (0.0 - R.A[k]) * R.rcp[k];
      const double tb = ((double)hi[k] - R.A[k]) * R.rcp[k];
      const double a = fmin(ta, tb), b = fmax(ta, tb);
      if (a > t_in) {
        t_in = a;
        k_in = k;
      }
      if (b < t_out) {
        t_out = b;
        k_out = k;
      }
    }
  }
  return t_out > t_in;
}

// Per-axis crossing sums of one ray in FP32:
//   S0_k = sum of dx over the crossings of axis k,
//   Sl_k = sum of dx * (distance of the crossing from the entry),
// dx = value before - value after, for the crossings strictly inside the
// clipped segment (the faces at its ends are added by the caller).  Walks
// major-axis slabs as the forward projector does: a slab between two
// successive planes of the major axis a holds at most one crossing of each
// minor axis, so it is two to four neighbouring voxels, read only where the
// crossing exists.  The warp's lanes are aligned on their entry position
// along the major axis (slab k of the loop is slab k - d of the lane), so
// neighbouring rays read the same plane in the same iteration.  Crossing
// distances are l0 + j * inc from exact integers j and the FP64 counts N
// bound every index, as in the projectors.  All 32 lanes call this; lanes
// without a ray pass active = false.  Returns the value of the voxel the
// segment ends in.
template <typename Off>
__device__ __forceinline__ float crossing_sums(bool active, const Walk& W, const int hi[3],
                                               const float* __restrict__ vol, Off off, Off s0, Off s1, Off s2,
                                               float x0, float S0[3], float Sl[3],
                                               [[maybe_unused]] long long n_vox) {
  constexpr unsigned kFull = 0xffffffffu;
  int a, b, c;
  walk_axes(W, a, b, c);
  const int Na = active ? pick3(a, W.N[0], W.N[1], W.N[2]) : 0;
  const int Nb = pick3(b, W.N[0], W.N[1], W.N[2]);
  const int Nc = pick3(c, W.N[0], W.N[1], W.N[2]);
  const float l0a = pick3(a, W.l0[0], W.l0[1], W.l0[2]), inca = pick3(a, W.inc[0], W.inc[1], W.inc[2]);
  const float l0b = pick3(b, W.l0[0], W.l0[1], W.l0[2]), incb = pick3(b, W.inc[0], W.inc[1], W.inc[2]);
  const float l0c = pick3(c, W.l0[0], W.l0[1], W.l0[2]), incc = pick3(c, W.inc[0], W.inc[1], W.inc[2]);
  const Off sa = pick3(a, s0, s1, s2), sb = pick3(b, s0, s1, s2), sc = pick3(c, s0, s1, s2);

  // slab alignment on the entry position along the major axis (travel direction)
  const int ia = pick3(a, W.i[0], W.i[1], W.i[2]);
  const int p = pick3(a, W.step[0], W.step[1], W.step[2]) > 0 ? ia : pick3(a, hi[0], hi[1], hi[2]) - 1 - ia;
  const int span_plain = __reduce_max_sync(kFull, active ? Na : -1);
  float S0a = 0.f, S0b = 0.f, S0c = 0.f, Sla = 0.f, Slb = 0.f, Slc = 0.f;
  float xe = x0;
  if (span_plain >= 0) {
    const int pmin = __reduce_min_sync(kFull, active ? p : 0x7fffffff);
    int d = active ? p - pmin : 0;
    int kmax = __reduce_max_sync(kFull, active ? d + Na : -1);
    if (kmax > 2 * span_plain + 8) {  // alignment would stretch the warp's loop too much
      d = 0;
      kmax = span_plain;
    }
    if (!active) d = 1 << 30;  // s = k - d stays negative: never inside [0, Na]
    float fs = -(float)d;      // s as a float, counted (exact for active lanes)
    const float L = W.L;
    const float fNb = (float)Nb, fNc = (float)Nc;
    float tb = Nb > 0 ? l0b : CUDART_INF_F, tc = Nc > 0 ? l0c : CUDART_INF_F;
    float fjb = 1.f, fjc = 1.f, cur = 0.f;
    if (!__any_sync(kFull, active && Nc > 0)) {
#pragma unroll kGradUnroll2
      for (int k = 0; k <= kmax; ++k, fs += 1.f) {
        const int s = k - d;
        const bool on = (unsigned)s <= (unsigned)Na;
        const bool ona = (unsigned)s < (unsigned)Na;  // a major plane ends this slab
        const float tx = ona ? fminf(fmaf(fs, inca, l0a), L) : L;
        const bool cb = on && tb < tx;
        const float m1 = fmaxf(fminf(tb, tx), cur);
        const Off o2 = off + (cb ? sb : (Off)0);
        float x1 = x0;
        if (cb && CTP_IN_BOUNDS(o2, n_vox, 13)) x1 = __ldg(vol + o2);
        float x2 = x1;
        if (ona && CTP_IN_BOUNDS(o2 + sa, n_vox, 13)) x2 = __ldg(vol + o2 + sa);
        const float d1 = x0 - x1, d2 = x1 - x2;
        S0b += d1;
        Slb = fmaf(d1, m1, Slb);
        S0a += d2;
        Sla = fmaf(d2, tx, Sla);
        if (on) {
          xe = x1;
          x0 = x2;
          off = o2 + sa;
          cur = tx;
        }
        if (cb) {
          tb = fjb < fNb ? fmaf(fjb, incb, l0b) : CUDART_INF_F;
          fjb += 1.f;
        }
      }
    } else {
#pragma unroll kGradUnroll3
      for (int k = 0; k <= kmax; ++k, fs += 1.f) {
        const int s = k - d;
        const bool on = (unsigned)s <= (unsigned)Na;
        const bool ona = (unsigned)s < (unsigned)Na;
        const float tx = ona ? fminf(fmaf(fs, inca, l0a), L) : L;
        const bool cb = on && tb < tx, cc = on && tc < tx;
        const bool bfirst = tb <= tc;
        const float m1 = fmaxf(fminf(fminf(tb, tc), tx), cur);
        const float m2 = fmaxf(fminf(fmaxf(tb, tc), tx), m1);
        const Off db = cb ? sb : (Off)0, dc = cc ? sc : (Off)0;
        const Off o2 = off + (bfirst ? db : dc);
        const Off o3 = off + db + dc;
        float x1 = x0;
        if ((cb || cc) && CTP_IN_BOUNDS(o2, n_vox, 13)) x1 = __ldg(vol + o2);
        float x2 = x1;
        if (cb && cc && CTP_IN_BOUNDS(o3, n_vox, 13)) x2 = __ldg(vol + o3);
        float x3 = x2;
        if (ona && CTP_IN_BOUNDS(o3 + sa, n_vox, 13)) x3 = __ldg(vol + o3 + sa);
        const float d1 = x0 - x1, d2 = x1 - x2, d3 = x2 - x3;
        S0b += bfirst ? d1 : d2;
        S0c += bfirst ? d2 : d1;
        Slb = fmaf(bfirst ? d1 : d2, bfirst ? m1 : m2, Slb);
        Slc = fmaf(bfirst ? d2 : d1, bfirst ? m2 : m1, Slc);
        S0a += d3;
        Sla = fmaf(d3, tx, Sla);
        if (on) {
          xe = x2;
          x0 = x3;
          off = o3 + sa;
          cur = tx;
        }
        if (cb) {
          tb = fjb < fNb ? fmaf(fjb, incb, l0b) : CUDART_INF_F;
          fjb += 1.f;
        }
        if (cc) {
          tc = fjc < fNc ? fmaf(fjc, incc, l0c) : CUDART_INF_F;
          fjc += 1.f;
        }
      }
    }
  }
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    S0[k] = k == a ? S0a : (k == b ? S0b : S0c);
    Sl[k] = k == a ? Sla : (k == b ? Slb : Slc);
  }
  return xe;
}

// Cylindrical detector: the pixel gradient G (already weighted) carried to
// the view's vectors.  With a = det_c - src, v^ = det_v / |det_v|,
// alpha = a.v^, w = a - alpha v^, R = |w|, w^ = w / R, u^ = det_u / |det_u|,
// gamma = (c - cc) |det_u| / R and rho = r - rc, the pixel is
//   p = src + alpha v^ + R (cos gamma w^ + sin gamma u^) + rho det_v.
// With t = -sin gamma w^ + cos gamma u^ (the unit tangent at the pixel),
// h = (sin gamma u^ - gamma t).G and P = I - v^ v^T:
//   dL/d det_c = (v^.G) v^ + cos gamma P G + h w^
//   dL/d src   = (source endpoint gradient) + G - dL/d det_c
//   dL/d det_u = (R gamma / |det_u|) (t.G) u^ + (R sin gamma / |det_u|) (G - (u^.G) u^)
//   dL/d det_v = P X / |det_v| + rho G,
//     X = (1 - cos gamma) ((v^.G) a + alpha G) - alpha h w^.
// (Derivatives of the unconstrained formula above, the one the projector
// evaluates; the view record holds u^, w^, v^, R, |det_u| / R and alpha.)
__device__ __forceinline__ void cylinder_chain(const ViewRec& V, const double* __restrict__ trig, const Dims& dm,
                                               int v, int c, double rho, const double gsrc[3], const double G[3],
                                               double out[12]) {
  const size_t ti = 2 * ((size_t)v * dm.n_cols + c);
  const double cg = trig[ti], sg = trig[ti + 1];
  const double gam = V.gam0 + (double)c * V.dgam;
  const double alpha = V.axial0 + 0.5 * (double)(dm.n_rows - 1) * V.vlen;  // (det_c - src).v^
  double t[3], a[3], vG = 0.0, uG = 0.0, tG = 0.0, hG = 0.0;
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    t[k] = cg * V.du[k] - sg * V.w[k];
    a[k] = alpha * V.vhat[k] + V.R * V.w[k];
    vG = fma(V.vhat[k], G[k], vG);
    uG = fma(V.du[k], G[k], uG);
    tG = fma(t[k], G[k], tG);
  }
  hG = sg * uG - gam * tG;
  double X[3], vX = 0.0;
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    X[k] = (1.0 - cg) * (vG * a[k] + alpha * G[k]) - alpha * hG * V.w[k];
    vX = fma(V.vhat[k], X[k], vX);
  }
  const double inv_dgam = 1.0 / V.dgam;  // R / |det_u|
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    const double ga = vG * V.vhat[k] + cg * (G[k] - vG * V.vhat[k]) + hG * V.w[k];
    out[k] = gsrc[k] + G[k] - ga;
    out[3 + k] = ga;
    out[6 + k] = inv_dgam * (gam * tG * V.du[k] + sg * (G[k] - uG * V.du[k]));
    out[9 + k] = (X[k] - vX * V.vhat[k]) / V.vlen + rho * G[k];
  }
}

// Block reduction of the 12 per-thread gradient entries (warps by shuffles,
// then one warp over the 8 warp sums) and one FP64 atomic per entry into
// grad[v][4][3].  Every block covers one view.
__device__ __forceinline__ void block_add_view_gradient(const double acc[12], double* __restrict__ grad, int v) {
  __shared__ double part[kGradThreads / 32][12];
  const int tid = threadIdx.y * kGradCols + threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
#pragma unroll
  for (int i = 0; i < 12; ++i) {
    double a = acc[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    if (lane == 0) part[warp][i] = a;
  }
  __syncthreads();
  if (tid < 12) {
    double a = 0.0;
#pragma unroll
    for (int w = 0; w < kGradThreads / 32; ++w) a += part[w][tid];
    if (a != 0.0) atomicAdd(grad + (size_t)v * 12 + tid, a);
  }
}

template <typename Off, bool kCyl>
__global__ void __launch_bounds__(kGradThreads, CTP_GRAD_MIN_BLOCKS) geometry_gradient_kernel(FwdLaunch P,
                                                                         const ViewRec* __restrict__ views,
                                                                         const double* __restrict__ trig,
                                                                         const float* __restrict__ vol,
                                                                         const float* __restrict__ volT,
                                                                         const float* __restrict__ gsino,
                                                                         double* __restrict__ grad) {
  const int per_band = P.dims.n_views * P.n_col_tiles;
  const int band = blockIdx.x / per_band;
  const int rem = blockIdx.x - band * per_band;
  const int v = rem / P.n_col_tiles;
  const int ct = rem - v * P.n_col_tiles;
  const int c = ct * kGradCols + threadIdx.x;
  const int r = band * kGradRows + threadIdx.y;
  const bool valid = c < P.dims.n_cols && r < P.dims.n_rows;

  const int lo[3] = {0, 0, 0};
  const int hi[3] = {P.vol.n[0], P.vol.n[1], P.vol.n[2]};
  const float gr = valid ? gsino[((size_t)v * P.dims.n_rows + r) * P.dims.n_cols + c] : 0.f;
  const int rr = valid ? r : 0, cc = valid ? c : 0;

  // Pass 1: FP64 setup, then the FP32 walk for the per-axis crossing sums.
  Walk W = {};
  bool hit;
  bool yfast;
  {
    const ViewRec& V = views[v];
    Ray R;
    make_ray(V, P.vol, trig, P.dims, v, rr, cc, R);
    double t_in = 0.0, t_out = 0.0;
    int k_in, k_out;
    hit = valid && gr != 0.f && clip_faces(R, hi, t_in, t_out, k_in, k_out);
    if (hit) entry(R, t_in, t_out, lo, hi, W);
    yfast = V.layout != 0;
  }
  // gather from the x-fastest volume or its y-fastest copy, as the forward does
  const Off nx = P.vol.n[0], ny = P.vol.n[1];
  const float* __restrict__ base = yfast ? volT : vol;
  const Off sx = yfast ? ny : (Off)1, sy = yfast ? (Off)1 : nx, sz = nx * ny;
  const Off off = (Off)W.i[2] * sz + (Off)W.i[1] * sy + (Off)W.i[0] * sx;
  const long long n_vox = (long long)P.vol.n[0] * P.vol.n[1] * P.vol.n[2];
  const float first = hit && CTP_IN_BOUNDS(off, n_vox, 14) ? __ldg(base + off) : 0.f;
  float f0[3], fl[3];
  const float last =
      crossing_sums<Off>(hit, W, hi, base, off, W.step[0] * sx, W.step[1] * sy, W.step[2] * sz, first, f0, fl, n_vox);

  // Pass 2: the same FP64 setup again (bit-identical), recomputed rather than
  // kept live through the walk so the walk runs with fewer registers; the
  // opaque copy of the record pointer keeps the compiler from merging the
  // two setups.
  const ViewRec* vp = views + v;
  asm volatile("" : "+l"(vp));
  const ViewRec& V = *vp;
  Ray R;
  const bool from_pixel = make_ray(V, P.vol, trig, P.dims, v, rr, cc, R);
  double t_in = 0.0, t_out = 0.0;
  int k_in = -1, k_out = -1;
  if (hit) clip_faces(R, hi, t_in, t_out, k_in, k_out);
  double S0[3], Sl[3];
  // the faces: entering at local distance 0, leaving at the segment's length
  const double Lseg = (t_out - t_in) * R.len;
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    S0[k] = (double)f0[k] - (k == k_in ? (double)first : 0.0) + (k == k_out ? (double)last : 0.0);
    Sl[k] = (double)fl[k] + (k == k_out ? (double)last * Lseg : 0.0);
  }
  const double x_end = k_out < 0 ? (double)last : 0.0;

  // per-ray gradients: G_src (3) and G_pix (3), weighted by g
  double gs[3] = {0.0, 0.0, 0.0}, gp[3] = {0.0, 0.0, 0.0};
  if (hit) {
    const double len = R.len, g = (double)gr;
    double S1[3], Dw[3];
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      S1[k] = fma(t_in, S0[k], Sl[k] / len);  // t_i = t_in + l_i / len
      Dw[k] = R.D[k] * P.vol.spacing[k];      // world-unit direction per unit t
    }
    if (P.dims.beam == CTP_BEAM_PARALLEL) {
      double gu[3];
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        const double q = V.s[k] != 0.0 ? -1.0 / V.s[k] : 0.0;  // V.s is the unit direction
        gp[k] = g * q * S0[k];
        gu[k] = g * q * S1[k];
      }
      const double ud = V.s[0] * gu[0] + V.s[1] * gu[1] + V.s[2] * gu[2];
#pragma unroll
      for (int k = 0; k < 3; ++k) gs[k] = (gu[k] - V.s[k] * ud) / V.src_norm;
    } else {
      const double E = S1[0] + S1[1] + S1[2] + x_end;
      double ga[3], gb[3];
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        const double q = Dw[k] != 0.0 ? len / Dw[k] : 0.0;
        const double u = Dw[k] / len;
        ga[k] = g * (q * (S1[k] - S0[k]) - u * E);
        gb[k] = g * (u * E - q * S1[k]);
      }
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        gp[k] = from_pixel ? ga[k] : gb[k];
        gs[k] = from_pixel ? gb[k] : ga[k];
      }
    }
  }
  const double cu = (double)c - 0.5 * (double)(P.dims.n_cols - 1);
  const double rv = (double)r - 0.5 * (double)(P.dims.n_rows - 1);
  double acc[12];
  if (!kCyl) {
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      acc[k] = gs[k];
      acc[3 + k] = gp[k];
      acc[6 + k] = cu * gp[k];
      acc[9 + k] = rv * gp[k];
    }
  } else {
    cylinder_chain(V, trig, P.dims, v, valid ? c : 0, rv, gs, gp, acc);
  }
  block_add_view_gradient(acc, grad, v);
}

// ------------------------------------------------ shared (x, y) slice walks --
//
// Rays in z-planes whose detector rows step along z (ctp_ray.cuh): one thread
// walks the (x, y) path of a detector column once for 4 rows, reading the 4
// rows' voxel values with one 16-byte load from the volume interleaved by 4
// slices where the rows fall in one slice group (single elements otherwise).
// The z axis is never crossed, so a slab is one or two segments; every row's
// crossing sums are the ones its own walk would give, in the same order.

__device__ __forceinline__ float4 f4sub(float4 p, float4 q) { return make_float4(p.x - q.x, p.y - q.y, p.z - q.z, p.w - q.w); }
__device__ __forceinline__ float4 f4add(float4 p, float4 q) { return make_float4(p.x + q.x, p.y + q.y, p.z + q.z, p.w + q.w); }
__device__ __forceinline__ float4 f4fma(float4 p, float t, float4 q) {
  return make_float4(fmaf(p.x, t, q.x), fmaf(p.y, t, q.y), fmaf(p.z, t, q.z), fmaf(p.w, t, q.w));
}
__device__ __forceinline__ float f4get(float4 p, int j) { return j == 0 ? p.x : (j == 1 ? p.y : (j == 2 ? p.z : p.w)); }

// crossing_sums for 4 rows at once (component j of every float4 is row j):
// S0 / Sl of the major axis a (index 0) and of the other crossed axis b
// (index 1).  load(offset) returns the 4 rows' values of the voxel column at
// that (x, y) offset.  Returns the values of the voxel the segment ends in.
#ifndef CTP_GRAD_ROWS_UNROLL
#define CTP_GRAD_ROWS_UNROLL 2
#endif
constexpr int kGradRowsUnroll = CTP_GRAD_ROWS_UNROLL;

template <typename Off, typename Load>
__device__ __forceinline__ float4 crossing_sums4(bool active, const Walk& W, const int hi[3], Off off, Off s0, Off s1,
                                                 float4 x0, float4 S0[2], float4 Sl[2], int& ka, int& kb,
                                                 Load&& load) {
  constexpr unsigned kFull = 0xffffffffu;
  int a, b, c;
  walk_axes(W, a, b, c);
  ka = a;
  kb = b;
  const int Na = active ? pick3(a, W.N[0], W.N[1], W.N[2]) : 0;
  const int Nb = pick3(b, W.N[0], W.N[1], W.N[2]);
  const float l0a = pick3(a, W.l0[0], W.l0[1], W.l0[2]), inca = pick3(a, W.inc[0], W.inc[1], W.inc[2]);
  const float l0b = pick3(b, W.l0[0], W.l0[1], W.l0[2]), incb = pick3(b, W.inc[0], W.inc[1], W.inc[2]);
  const Off sa = pick3(a, s0, s1, (Off)0), sb = pick3(b, s0, s1, (Off)0);
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
  float4 S0a = zero, S0b = zero, Sla = zero, Slb = zero;
  float4 xe = x0;
  const int ia = pick3(a, W.i[0], W.i[1], W.i[2]);
  const int p = pick3(a, W.step[0], W.step[1], W.step[2]) > 0 ? ia : pick3(a, hi[0], hi[1], hi[2]) - 1 - ia;
  const int span_plain = __reduce_max_sync(kFull, active ? Na : -1);
  if (span_plain >= 0) {
    const int pmin = __reduce_min_sync(kFull, active ? p : 0x7fffffff);
    int d = active ? p - pmin : 0;
    int kmax = __reduce_max_sync(kFull, active ? d + Na : -1);
    if (kmax > 2 * span_plain + 8) {  // alignment would stretch the warp's loop too much
      d = 0;
      kmax = span_plain;
    }
    if (!active) d = 1 << 30;
    float fs = -(float)d;
    const float L = W.L;
    const float fNb = (float)Nb;
    float tb = Nb > 0 ? l0b : CUDART_INF_F;
    float fjb = 1.f, cur = 0.f;
#pragma unroll kGradRowsUnroll
    for (int k = 0; k <= kmax; ++k, fs += 1.f) {
      const int s = k - d;
      const bool on = (unsigned)s <= (unsigned)Na;
      const bool ona = (unsigned)s < (unsigned)Na;  // a major plane ends this slab
      const float tx = ona ? fminf(fmaf(fs, inca, l0a), L) : L;
      const bool cb = on && tb < tx;
      const float m1 = fmaxf(fminf(tb, tx), cur);
      const Off o2 = off + (cb ? sb : (Off)0);
      float4 x1 = x0;
      if (cb) x1 = load(o2);
      float4 x2 = x1;
      if (ona) x2 = load(o2 + sa);
      const float4 d1 = f4sub(x0, x1), d2 = f4sub(x1, x2);
      S0b = f4add(S0b, d1);
      Slb = f4fma(d1, m1, Slb);
      S0a = f4add(S0a, d2);
      Sla = f4fma(d2, tx, Sla);
      if (on) {
        xe = x1;
        x0 = x2;
        off = o2 + sa;
        cur = tx;
      }
      if (cb) {
        tb = fjb < fNb ? fmaf(fjb, incb, l0b) : CUDART_INF_F;
        fjb += 1.f;
      }
    }
  }
  S0[0] = S0a;
  S0[1] = S0b;
  Sl[0] = Sla;
  Sl[1] = Slb;
  return xe;
}

#ifndef CTP_GRAD_ROWS_MIN_BLOCKS
#define CTP_GRAD_ROWS_MIN_BLOCKS 3
#endif

template <typename Off>
__global__ void __launch_bounds__(kSliceCols* kSliceWarps, CTP_GRAD_ROWS_MIN_BLOCKS)
    geometry_gradient_rows4_kernel(FwdLaunch P, const ViewRec* __restrict__ views, const float4* __restrict__ vol4,
                                   const float4* __restrict__ vol4T, const float* __restrict__ gsino,
                                   double* __restrict__ grad) {
  static_assert(kSliceCols * kSliceWarps == kGradThreads, "one gradient block per shared-walk block");
  int v, c, r0;
  rows_block_position<4>(P, v, c, r0);
  const bool cvalid = c < P.dims.n_cols;
  const ViewRec& V = views[v];
  const Off nx = P.vol.n[0], ny = P.vol.n[1];
  const Off plane = nx * ny;
  [[maybe_unused]] const Off n4 = (Off)((P.vol.n[2] + 3) >> 2) * plane;
  int ks[4];
  const unsigned inside = cvalid ? row_slice_index<4>(V, P.vol, r0, c, P.dims.n_rows, ks) : 0u;
  // rows with a non-zero upstream gradient (their values are read again after
  // the walk, so they hold no registers through it)
  auto upstream = [&](int j) -> float {
    return (inside & (1u << j)) ? __ldg(gsino + ((size_t)v * P.dims.n_rows + r0 + j) * P.dims.n_cols + c) : 0.f;
  };
  unsigned rows = inside;
#pragma unroll
  for (int j = 0; j < 4; ++j)
    if (!(upstream(j) != 0.f)) rows &= ~(1u << j);
  // the shared (x, y) ray, lifted into the volume's height: only the x and y
  // slabs clip it, so t_in, t_out and the entry and exit faces are every row's
  const int lo[3] = {0, 0, 0};
  const int hi[3] = {P.vol.n[0], P.vol.n[1], P.vol.n[2]};
  Walk W = {};
  bool hit;
  {
    Ray R;
    make_ray(V, P.vol, nullptr, P.dims, v, 0, cvalid ? c : 0, R);
    R.A[2] = (setup_t)0.5;
    double t_in = 0.0, t_out = 0.0;
    int k_in, k_out;
    hit = rows != 0u && clip_faces(R, hi, t_in, t_out, k_in, k_out);
    if (hit) entry(R, (setup_t)t_in, (setup_t)t_out, lo, hi, W);
  }
  const bool yfast = V.layout != 0;
  const float4* __restrict__ base4 = yfast ? vol4T : vol4;
  const float* __restrict__ base1 = reinterpret_cast<const float*>(base4);
  const Off sx = yfast ? ny : (Off)1, sy = yfast ? (Off)1 : nx;
  const Off off = (Off)W.i[1] * sy + (Off)W.i[0] * sx;
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
  float4 S0[2], Sl[2], first, last;
  int ka = 0, kb = 1;
  if (__all_sync(0xffffffffu, one_group(inside, ks) || !hit)) {
    const Off g0 = (Off)(ks[0] >> 2) * plane;
    auto load = [&](Off o) -> float4 { return CTP_IN_BOUNDS(g0 + o, n4, 19) ? __ldg(base4 + g0 + o) : zero; };
    first = hit ? load(off) : zero;
    last = crossing_sums4<Off>(hit, W, hi, off, W.step[0] * sx, W.step[1] * sy, first, S0, Sl, ka, kb, load);
  } else {
    Off e[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) e[j] = ((Off)(ks[j] >> 2) * plane) * 4 + (ks[j] & 3);
    auto load = [&](Off o) -> float4 {
      float q[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        q[j] = (inside & (1u << j)) && CTP_IN_BOUNDS(e[j] + 4 * o, 4 * n4, 20) ? __ldg(base1 + e[j] + 4 * o) : 0.f;
      return make_float4(q[0], q[1], q[2], q[3]);
    };
    first = hit ? load(off) : zero;
    last = crossing_sums4<Off>(hit, W, hi, off, W.step[0] * sx, W.step[1] * sy, first, S0, Sl, ka, kb, load);
  }
  // per-row gradients of a parallel ray (as in geometry_gradient_kernel),
  // weighted by the row's upstream gradient and summed over the 4 rows; the
  // FP64 set-up is recomputed (bit-identical) rather than kept through the walk
  const ViewRec* vp = views + v;
  asm volatile("" : "+l"(vp));
  Ray R;
  make_ray(*vp, P.vol, nullptr, P.dims, v, 0, cvalid ? c : 0, R);
  R.A[2] = (setup_t)0.5;
  double t_in = 0.0, t_out = 0.0;
  int k_in = -1, k_out = -1;
  if (hit) clip_faces(R, hi, t_in, t_out, k_in, k_out);
  double acc[12];
#pragma unroll
  for (int i = 0; i < 12; ++i) acc[i] = 0.0;
  if (hit) {
    const double Lseg = (t_out - t_in) * (double)R.len;
    const double cu = (double)c - 0.5 * (double)(P.dims.n_cols - 1);
    double q[3];
#pragma unroll
    for (int k = 0; k < 3; ++k) q[k] = V.s[k] != 0.0 ? -1.0 / V.s[k] : 0.0;  // V.s is the unit direction
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (!(rows & (1u << j))) continue;
      const double fj = (double)f4get(first, j), lj = (double)f4get(last, j), gj = (double)upstream(j);
      double gp[3], gu[3];
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        const double f0 = k == ka ? (double)f4get(S0[0], j) : (k == kb ? (double)f4get(S0[1], j) : 0.0);
        const double fl = k == ka ? (double)f4get(Sl[0], j) : (k == kb ? (double)f4get(Sl[1], j) : 0.0);
        const double s0 = f0 - (k == k_in ? fj : 0.0) + (k == k_out ? lj : 0.0);
        const double sl = fl + (k == k_out ? lj * Lseg : 0.0);
        const double s1 = fma(t_in, s0, sl / (double)R.len);
        gp[k] = gj * q[k] * s0;
        gu[k] = gj * q[k] * s1;
      }
      const double ud = V.s[0] * gu[0] + V.s[1] * gu[1] + V.s[2] * gu[2];
      const double rv = (double)(r0 + j) - 0.5 * (double)(P.dims.n_rows - 1);
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        acc[k] += (gu[k] - V.s[k] * ud) / V.src_norm;
        acc[3 + k] += gp[k];
        acc[6 + k] += cu * gp[k];
        acc[9 + k] += rv * gp[k];
      }
    }
  }
  block_add_view_gradient(acc, grad, v);
}

}  // namespace

cudaError_t launch_geometry_gradient(const FwdLaunch& p, const ViewRec* views, const double* trig, const float* vol,
                                     const float* volT, const float* gsino, double* grad, bool wide_index,
                                     cudaStream_t stream) {
  const long long blocks = (long long)p.n_row_bands * p.dims.n_views * p.n_col_tiles;
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  dim3 block(kGradCols, kGradRows);
  const unsigned nb = (unsigned)blocks;
  const bool cyl = p.dims.det != CTP_DET_FLAT;
  if (wide_index) {
    if (cyl) geometry_gradient_kernel<long long, true><<<nb, block, 0, stream>>>(p, views, trig, vol, volT, gsino, grad);
    else geometry_gradient_kernel<long long, false><<<nb, block, 0, stream>>>(p, views, trig, vol, volT, gsino, grad);
  } else {
    if (cyl) geometry_gradient_kernel<int, true><<<nb, block, 0, stream>>>(p, views, trig, vol, volT, gsino, grad);
    else geometry_gradient_kernel<int, false><<<nb, block, 0, stream>>>(p, views, trig, vol, volT, gsino, grad);
  }
  return cudaGetLastError();
}

cudaError_t launch_geometry_gradient_rows4(const FwdLaunch& p, const ViewRec* views, const float4* vol4,
                                           const float4* vol4T, const float* gsino, double* grad, bool wide_index,
                                           cudaStream_t stream) {
  const long long blocks = (long long)rows_bands(p.dims.n_rows, 4) * p.dims.n_views * rows_col_tiles(p.dims.n_cols);
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const dim3 block(kSliceCols, kSliceWarps);
  if (wide_index)
    geometry_gradient_rows4_kernel<long long><<<(unsigned)blocks, block, 0, stream>>>(p, views, vol4, vol4T, gsino,
                                                                                       grad);
  else
    geometry_gradient_rows4_kernel<int><<<(unsigned)blocks, block, 0, stream>>>(p, views, vol4, vol4T, gsino, grad);
  return cudaGetLastError();
}

// The bounds-check word of this file's kernel (CTP_DEBUG builds; 0
// elsewhere), read and cleared.  Synchronous.
unsigned long long debug_take_word_grad() {
#ifdef CTP_DEBUG
  unsigned long long w = 0, z = 0;
  if (cudaMemcpyFromSymbol(&w, g_debug_word, sizeof(w)) != cudaSuccess) return ~0ull;
  cudaMemcpyToSymbol(g_debug_word, &z, sizeof(z));
  return w;
#else
  return 0;
#endif
}

}  // namespace ctp
