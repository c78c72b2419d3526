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

// Working precision of the per-ray set-up: FP64.  The CTP_FP32_SETUP build
// (an ablation for tests only, never the library's default) runs the same
// set-up in FP32, the working precision the pages report for hardware
// without FP64 (diffct "Execution", paragraph on Apple MPS).
#ifdef CTP_FP32_SETUP
using setup_t = float;
#else
using setup_t = double;
#endif

// Bounds checks of the CTP_DEBUG build: every global and shared-memory index
// of the walks and flushes is tested against its array's extent; a failing
// index is recorded (the first one per translation unit: check site in the
// top 16 bits, the index in the low 48) and its access skipped, so a bad
// index never reaches memory.  Ordinary builds compile the checks away.
#ifdef CTP_DEBUG
static __device__ unsigned long long g_debug_word;
__device__ __forceinline__ bool in_bounds(long long i, long long n, unsigned site) {
  if (i >= 0 && i < n) return true;
  atomicCAS(&g_debug_word, 0ull, ((unsigned long long)site << 48) | ((unsigned long long)i & 0xffffffffffffull));
  return false;
}
#define CTP_IN_BOUNDS(i, n, site) ::ctp::in_bounds((long long)(i), (long long)(n), (site))
#else
#define CTP_IN_BOUNDS(i, n, site) true
#endif

struct Ray {
  setup_t A[3];    // parameter origin, voxel units relative to the volume min corner
  setup_t D[3];    // direction, voxel units per unit t
  setup_t rcp[3];  // 1 / D (unused where D == 0)
  setup_t len;     // physical length per unit t
  setup_t t_lo, t_hi;
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
                                             int r, int c, setup_t p[3]) {
  using T = setup_t;
  if (dm.det == CTP_DET_FLAT) {
#pragma unroll
    for (int k = 0; k < 3; ++k) p[k] = fma((T)r, (T)V.dv[k], fma((T)c, (T)V.du[k], (T)V.p00[k]));
  } else {
    const size_t t = 2 * ((size_t)v * dm.n_cols + c);
    const T cg = (T)trig[t], sg = (T)trig[t + 1];
#pragma unroll
    for (int k = 0; k < 3; ++k)
      p[k] = fma((T)r, (T)V.dv[k], (T)V.p00[k]) + (T)V.R * fma(cg, (T)V.w[k], sg * (T)V.du[k]);
  }
}

// Ray of pixel (v, r, c) in voxel units.  Cone: the finite segment between the
// source and the pixel centre, parametrised from whichever endpoint is nearer
// the volume centre.  Parallel: the full line through the pixel centre.
// Returns true when the origin is the pixel (cone) or always (parallel).
__device__ __forceinline__ bool make_ray(const ViewRec& V, const VolDesc& G, const double* __restrict__ trig,
                                         const Dims& dm, int v, int r, int c, Ray& R) {
  using T = setup_t;
  T p[3];
  pixel_centre(V, trig, dm, v, r, c, p);
  if (dm.beam == CTP_BEAM_PARALLEL) {
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      R.A[k] = (p[k] - (T)G.origin[k]) * (T)G.inv_spacing[k];
      R.D[k] = (T)V.s[k] * (T)G.inv_spacing[k];
      R.rcp[k] = (T)V.rcp_dir[k];
    }
    R.len = (T)1;
    R.t_lo = -(T)CUDART_INF;
    R.t_hi = (T)CUDART_INF;
    return true;
  } else {
    T pv[3], sv[3], dp2 = 0, ds2 = 0;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      pv[k] = (p[k] - (T)G.origin[k]) * (T)G.inv_spacing[k];
      sv[k] = ((T)V.s[k] - (T)G.origin[k]) * (T)G.inv_spacing[k];
      const T a = pv[k] - (T)G.centre[k], b = sv[k] - (T)G.centre[k];
      dp2 = fma(a, a, dp2);
      ds2 = fma(b, b, ds2);
    }
    const bool from_pixel = dp2 <= ds2;
    T len2 = 0;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      const T dw = from_pixel ? ((T)V.s[k] - p[k]) : (p[k] - (T)V.s[k]);
      len2 = fma(dw, dw, len2);
      R.A[k] = from_pixel ? pv[k] : sv[k];
      R.D[k] = dw * (T)G.inv_spacing[k];
      R.rcp[k] = (T)1 / R.D[k];
    }
    R.len = sqrt(len2);
    R.t_lo = 0;
    R.t_hi = 1;
    return from_pixel;
  }
}

// Slab clipping against the half-open box [lo, hi) (voxel units).
__device__ __forceinline__ bool clip(const Ray& R, const int lo[3], const int hi[3], setup_t& t_in, setup_t& t_out) {
  using T = setup_t;
  t_in = R.t_lo;
  t_out = R.t_hi;
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    if (R.D[k] == (T)0) {
      if (!(R.A[k] >= (T)lo[k] && R.A[k] < (T)hi[k])) return false;
    } else {
      const T ta = ((T)lo[k] - R.A[k]) * R.rcp[k];
      const T tb = ((T)hi[k] - R.A[k]) * R.rcp[k];
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
__device__ __forceinline__ void entry(const Ray& R, setup_t t_in, setup_t t_out, const int lo[3], const int hi[3],
                                      Walk& W, double* w64 = nullptr, int stride = 1) {
  using T = setup_t;
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    const T e = fma(t_in, R.D[k], R.A[k]);
    const T x = fma(t_out, R.D[k], R.A[k]);
    const T el = fmin(fmax(e, (T)lo[k]), (T)hi[k]);
    const T xl = fmin(fmax(x, (T)lo[k]), (T)hi[k]);
    if (R.D[k] > (T)0) {
      const int i0 = clampi((int)floor(el), lo[k], hi[k] - 1);
      const int i1 = clampi((int)ceil(xl) - 1, lo[k], hi[k] - 1);
      W.i[k] = i0;
      W.N[k] = max(i1 - i0, 0);
      W.step[k] = 1;
      const T tc = ((T)(i0 + 1) - R.A[k]) * R.rcp[k];
      const T l0d = (tc - t_in) * R.len, incd = R.rcp[k] * R.len;
      W.l0[k] = (float)l0d;
      W.inc[k] = (float)incd;
      if (w64) {
        w64[k * stride] = (double)l0d;
        w64[(3 + k) * stride] = (double)incd;
      }
    } else if (R.D[k] < (T)0) {
      const int i0 = clampi((int)ceil(el) - 1, lo[k], hi[k] - 1);
      const int i1 = clampi((int)floor(xl), lo[k], hi[k] - 1);
      W.i[k] = i0;
      W.N[k] = max(i0 - i1, 0);
      W.step[k] = -1;
      const T tc = ((T)i0 - R.A[k]) * R.rcp[k];
      const T l0d = (tc - t_in) * R.len, incd = -R.rcp[k] * R.len;
      W.l0[k] = (float)l0d;
      W.inc[k] = (float)incd;
      if (w64) {
        w64[k * stride] = (double)l0d;
        w64[(3 + k) * stride] = (double)incd;
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
  const T Ld = (t_out - t_in) * R.len;
  W.L = (float)Ld;
  if (w64) w64[6 * stride] = (double)Ld;
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


// ------------------------------------------------ shared (x, y) slice walks --
//
// Shared by the projector kernels (ctp_kernels.cu) and the geometry-gradient
// kernel (ctp_grad.cu): when every ray lies in a plane of constant z (a
// parallel beam whose direction has no z component) and detector rows step
// along z only, the rays of one detector column in one view follow the same
// (x, y) path, each in the slice of its own row (the slices decouple;
// MBIRJAX "Sharding overview", section "Why cone beam").  Blocks of these
// kernels are kSliceWarps warps of kSliceCols columns x kR rows.
constexpr int kSliceCols = 32;
constexpr int kSliceWarps = 8;

// Block shape of the shared-slice kernels: 8 warps of 32 columns x kR rows,
// kRowsGroups of them stacked along the rows and 8 / kRowsGroups side by side
// along the columns.  A band (the rows of one block row) is kRowsGroups * kR
// slices deep; blocks run band by band, every view of a band before the next,
// so the slices the blocks in flight touch (the adjoint's accumulation
// working set, in both volume layouts) stay few enough for L2.
#ifndef CTP_ROWS_GROUPS
#define CTP_ROWS_GROUPS 8
#endif
constexpr int kRowsGroups = CTP_ROWS_GROUPS;
constexpr int kRowsColTiles = kSliceWarps / kRowsGroups;
static_assert(kRowsGroups * kRowsColTiles == kSliceWarps, "row groups divide the block's warps");

__host__ __device__ __forceinline__ int rows_col_tiles(int n_cols) {
  return (n_cols + kSliceCols * kRowsColTiles - 1) / (kSliceCols * kRowsColTiles);
}
__host__ __device__ __forceinline__ int rows_bands(int n_rows, int r) {
  return (n_rows + kRowsGroups * r - 1) / (kRowsGroups * r);
}

// View, column and first row of this thread in a shared-slice kernel.
template <int kR>
__device__ __forceinline__ void rows_block_position(const FwdLaunch& P, int& v, int& c, int& r0) {
  const int ctiles = rows_col_tiles(P.dims.n_cols);
  const int per_band = P.dims.n_views * ctiles;
  const int band = blockIdx.x / per_band;
  const int rem = blockIdx.x - band * per_band;
  v = rem / ctiles;
  const int ct = rem - v * ctiles;
  const int w = threadIdx.y;
  c = (ct * kRowsColTiles + w % kRowsColTiles) * kSliceCols + threadIdx.x;
  r0 = (band * kRowsGroups + w / kRowsColTiles) * kR;
}

// Slices of rows r0 .. r0 + kR - 1 of column c: bit j of the result is set
// where row r0 + j exists and its rays' height falls inside the volume (the z
// test of the ray's slab clip); ks[j] is then that slice.
template <int kR>
__device__ __forceinline__ unsigned row_slice_index(const ViewRec& V, const VolDesc& G, int r0, int c, int n_rows,
                                                    int ks[kR]) {
  unsigned mask = 0u;
#pragma unroll
  for (int j = 0; j < kR; ++j) {
    const int r = r0 + j;
    // the z component of pixel_centre's flat-detector formula and make_ray's
    // voxel-unit height, in the set-up's precision
    using T = setup_t;
    const T pz = fma((T)r, (T)V.dv[2], fma((T)c, (T)V.du[2], (T)V.p00[2]));
    const T az = (pz - (T)G.origin[2]) * (T)G.inv_spacing[2];
    const bool in = r < n_rows && az >= (T)0 && az < (T)G.n[2];
    ks[j] = in ? clampi((int)floor(az), 0, G.n[2] - 1) : 0;
    mask |= in ? 1u << j : 0u;
  }
  return mask;
}

// The same, as offsets of the slices (zoff[j] = slice * sz).
template <int kR, typename Off>
__device__ __forceinline__ unsigned row_slices(const ViewRec& V, const VolDesc& G, int r0, int c, int n_rows, Off sz,
                                               Off zoff[kR]) {
  int ks[kR];
  const unsigned mask = row_slice_index<kR>(V, G, r0, c, n_rows, ks);
#pragma unroll
  for (int j = 0; j < kR; ++j) zoff[j] = (mask & (1u << j)) ? (Off)ks[j] * sz : (Off)0;
  return mask;
}

// Shared (x, y) set-up of column c: the ray of any row, lifted into the
// volume's height (its direction has no z component, so only the x and y
// slabs clip it) and walked as slice 0.
__device__ __forceinline__ bool slice_ray(const ViewRec& V, const VolDesc& G, const Dims& dm, int v, int c, Ray& R,
                                          setup_t& t_in, setup_t& t_out) {
  make_ray(V, G, nullptr, dm, v, 0, c, R);
  R.A[2] = (setup_t)0.5;
  const int lo[3] = {0, 0, 0};
  const int hi[3] = {G.n[0], G.n[1], G.n[2]};
  return clip(R, lo, hi, t_in, t_out);
}

// slices 4g .. 4g + 3 of the rows' heights, in order
__device__ __forceinline__ bool one_group(unsigned rows, const int ks[4]) {
  return rows == 0xfu && (ks[0] & 3) == 0 && ks[1] == ks[0] + 1 && ks[2] == ks[0] + 2 && ks[3] == ks[0] + 3;
}

}  // namespace ctp
