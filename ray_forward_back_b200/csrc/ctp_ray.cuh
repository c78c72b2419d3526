// Per-ray FP64 setup shared by the projector kernels (ctp_kernels.cu) and the
// geometry-gradient kernel (ctp_grad.cu): pixel centre, ray, slab clipping and
// the entry voxel with its per-axis crossing counts and local FP32 crossing
// parameters.  The model is the cell-constant Siddon model in physical
// coordinates with the FP64-setup / FP32-traversal split of diffct
// "Execution", section "Precision, training and reconstruction".
#pragma once

#include <math_constants.h>

#include "ctp_internal.h"

namespace ctp {

struct Ray {
  double A[3];    // parameter origin, voxel units relative to the volume min corner
  double D[3];    // direction, voxel units per unit t
  double rcp[3];  // 1 / D (unused where D == 0)
  double len;     // physical length per unit t
  double t_lo, t_hi;
};

struct Walk {
  int i[3];       // entry voxel (absolute indices)
  int N[3];       // crossings per axis inside the clipped segment
  int step[3];    // +1 / -1 per axis
  float l0[3];    // physical distance from the entry to the first crossing per axis
  float inc[3];   // physical distance between successive crossings per axis
  float L;        // physical length of the clipped segment
};

__device__ __forceinline__ void pixel_centre(const ViewRec& V, const double* __restrict__ trig, const Dims& dm, int v,
                                             int r, int c, double p[3]) {
  if (dm.det == CTP_DET_FLAT) {
#pragma unroll
    for (int k = 0; k < 3; ++k) p[k] = fma((double)r, V.dv[k], fma((double)c, V.du[k], V.p00[k]));
  } else {
    const size_t t = 2 * ((size_t)v * dm.n_cols + c);
    const double cg = trig[t], sg = trig[t + 1];
#pragma unroll
    for (int k = 0; k < 3; ++k) p[k] = fma((double)r, V.dv[k], V.p00[k]) + V.R * fma(cg, V.w[k], sg * V.du[k]);
  }
}

// Ray of pixel (v, r, c) in voxel units.  Cone: the finite segment between the
// source and the pixel centre, parametrised from whichever endpoint is nearer
// the volume centre.  Parallel: the full line through the pixel centre.
// Returns true when the origin is the pixel (cone) or always (parallel).
__device__ __forceinline__ bool make_ray(const ViewRec& V, const VolDesc& G, const double* __restrict__ trig,
                                         const Dims& dm, int v, int r, int c, Ray& R) {
  double p[3];
  pixel_centre(V, trig, dm, v, r, c, p);
  if (dm.beam == CTP_BEAM_PARALLEL) {
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      R.A[k] = (p[k] - G.origin[k]) * G.inv_spacing[k];
      R.D[k] = V.s[k] * G.inv_spacing[k];
      R.rcp[k] = V.rcp_dir[k];
    }
    R.len = 1.0;
    R.t_lo = -CUDART_INF;
    R.t_hi = CUDART_INF;
    return true;
  } else {
    double pv[3], sv[3], dp2 = 0.0, ds2 = 0.0;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      pv[k] = (p[k] - G.origin[k]) * G.inv_spacing[k];
      sv[k] = (V.s[k] - G.origin[k]) * G.inv_spacing[k];
      const double a = pv[k] - G.centre[k], b = sv[k] - G.centre[k];
      dp2 = fma(a, a, dp2);
      ds2 = fma(b, b, ds2);
    }
    const bool from_pixel = dp2 <= ds2;
    double len2 = 0.0;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      const double dw = from_pixel ? (V.s[k] - p[k]) : (p[k] - V.s[k]);
      len2 = fma(dw, dw, len2);
      R.A[k] = from_pixel ? pv[k] : sv[k];
      R.D[k] = dw * G.inv_spacing[k];
      R.rcp[k] = 1.0 / R.D[k];
    }
    R.len = sqrt(len2);
    R.t_lo = 0.0;
    R.t_hi = 1.0;
    return from_pixel;
  }
}

// Slab clipping against the half-open box [lo, hi) (voxel units).
__device__ __forceinline__ bool clip(const Ray& R, const int lo[3], const int hi[3], double& t_in, double& t_out) {
  t_in = R.t_lo;
  t_out = R.t_hi;
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    if (R.D[k] == 0.0) {
      if (!(R.A[k] >= (double)lo[k] && R.A[k] < (double)hi[k])) return false;
    } else {
      const double ta = ((double)lo[k] - R.A[k]) * R.rcp[k];
      const double tb = ((double)hi[k] - R.A[k]) * R.rcp[k];
      t_in = fmax(t_in, fmin(ta, tb));
      t_out = fmin(t_out, fmax(ta, tb));
    }
  }
  return t_out > t_in;
}

__device__ __forceinline__ int clampi(int x, int lo, int hi) { return x < lo ? lo : (x > hi ? hi : x); }

// Entry voxel, crossing counts and local FP32 crossing parameters of the
// clipped segment [t_in, t_out] inside the box [lo, hi).
// With w64 (a per-lane record of 7 doubles at stride `stride`: l0[3],
// inc[3], L) the FP64 values behind W's FP32 l0, inc and L are kept too, for
// walks that re-anchor their local FP32 parameters along the ray.
__device__ __forceinline__ void entry(const Ray& R, double t_in, double t_out, const int lo[3], const int hi[3],
                                      Walk& W, double* w64 = nullptr, int stride = 1) {
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    const double e = fma(t_in, R.D[k], R.A[k]);
    const double x = fma(t_out, R.D[k], R.A[k]);
    const double el = fmin(fmax(e, (double)lo[k]), (double)hi[k]);
    const double xl = fmin(fmax(x, (double)lo[k]), (double)hi[k]);
    if (R.D[k] > 0.0) {
      const int i0 = clampi((int)floor(el), lo[k], hi[k] - 1);
      const int i1 = clampi((int)ceil(xl) - 1, lo[k], hi[k] - 1);
      W.i[k] = i0;
      W.N[k] = max(i1 - i0, 0);
      W.step[k] = 1;
      const double tc = ((double)(i0 + 1) - R.A[k]) * R.rcp[k];
      const double l0d = (tc - t_in) * R.len, incd = R.rcp[k] * R.len;
      W.l0[k] = (float)l0d;
      W.inc[k] = (float)incd;
      if (w64) {
        w64[k * stride] = l0d;
        w64[(3 + k) * stride] = incd;
      }
    } else if (R.D[k] < 0.0) {
      const int i0 = clampi((int)ceil(el) - 1, lo[k], hi[k] - 1);
      const int i1 = clampi((int)floor(xl), lo[k], hi[k] - 1);
      W.i[k] = i0;
      W.N[k] = max(i0 - i1, 0);
      W.step[k] = -1;
      const double tc = ((double)i0 - R.A[k]) * R.rcp[k];
      const double l0d = (tc - t_in) * R.len, incd = -R.rcp[k] * R.len;
      W.l0[k] = (float)l0d;
      W.inc[k] = (float)incd;
      if (w64) {
        w64[k * stride] = l0d;
        w64[(3 + k) * stride] = incd;
      }
    } else {
      W.i[k] = clampi((int)floor(el), lo[k], hi[k] - 1);
      W.N[k] = 0;
      W.step[k] = 1;
      W.l0[k] = CUDART_INF_F;
      W.inc[k] = CUDART_INF_F;
      if (w64) {
        w64[k * stride] = CUDART_INF;
        w64[(3 + k) * stride] = CUDART_INF;
      }
    }
  }
  const double Ld = (t_out - t_in) * R.len;
  W.L = (float)Ld;
  if (w64) w64[6 * stride] = Ld;
}

template <typename T>
__device__ __forceinline__ T pick3(int k, T a0, T a1, T a2) {
  return k == 0 ? a0 : (k == 1 ? a1 : a2);
}

// Axis roles of a walk: a = major (crossed most often, smallest spacing
// between crossings), c = the minor axis crossed least often, b = the other.
__device__ __forceinline__ void walk_axes(const Walk& W, int& a, int& b, int& c) {
  const float i0 = W.inc[0], i1 = W.inc[1], i2 = W.inc[2];
  a = (i0 <= i1 && i0 <= i2) ? 0 : (i1 <= i2 ? 1 : 2);
  if (a == 0) {
    b = i1 <= i2 ? 1 : 2;
    c = 3 - b;
  } else if (a == 1) {
    b = i0 <= i2 ? 0 : 2;
    c = 2 - b;
  } else {
    b = i0 <= i1 ? 0 : 1;
    c = 1 - b;
  }
}

}  // namespace ctp
