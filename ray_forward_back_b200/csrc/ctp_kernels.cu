// CUDA kernels of the matched Siddon projector pair (sm_100a).
//
// Model: the coefficient of ray i and voxel j is the physical length of ray i
// inside voxel j (cell-constant Siddon model in physical coordinates; diffct
// "Execution", section "Precision, training and reconstruction").
//
// Precision split (same section, table row backend="numba" and the paragraph
// on segment setup): every ray is set up in FP64 -- pixel centre, the endpoint
// nearer the volume centre as parameter origin, slab clipping, entry voxel,
// per-axis crossing counts and the distance from the entry to each axis's
// first crossing -- and then traversed in FP32 with parameters measured
// locally from that entry.  The j-th crossing of axis k sits at
// l0_k + j * step_k (one FMA from exact integers), so rounding does not
// accumulate along the ray, and the per-axis crossing counts fixed in FP64
// bound every index: a walk can never leave the box it was set up in.
//
// Kernels:
//   forward_kernel     one thread per ray, gather (no write collisions);
//                      blocks ordered detector-row band -> view -> column tile so
//                      the blocks in flight touch a thin slab of the volume that
//                      stays in L2; a warp holds 32 adjacent columns so its
//                      lanes read neighbouring voxels, from an x-fastest or a
//                      y-fastest copy of the volume, whichever the view's
//                      column direction runs along; coalesced sinogram stores.
//   back_brick_kernel  one CTA owns a voxel brick in shared memory, visits every
//                      ray of its view range that can cross the brick (detector
//                      footprint of the brick per view), clips each ray to the
//                      brick in FP64 (the per-tile entry of the pages), walks it
//                      in FP32 with shared-memory atomics, and flushes the brick
//                      once with coalesced stores (plain stores when the CTA
//                      owns all views, red.global.add otherwise).
//   count_kernel       the forward traversal counting positive-length segments.
//   transpose_xy       x-fastest -> y-fastest copy of the volume.
#include <math_constants.h>

#include "ctp_internal.h"

namespace ctp {
namespace {

constexpr int kFwdCols = 32;  // threads along detector columns per block
constexpr int kFwdRows = 8;   // detector rows per block (row band height)
constexpr int kBackThreads = 256;
constexpr int kBackChunk = 8;  // views whose footprints are staged together

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
__device__ __forceinline__ void make_ray(const ViewRec& V, const VolDesc& G, const double* __restrict__ trig,
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
__device__ __forceinline__ void entry(const Ray& R, double t_in, double t_out, const int lo[3], const int hi[3],
                                      Walk& W) {
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
      W.l0[k] = (float)((tc - t_in) * R.len);
      W.inc[k] = (float)(R.rcp[k] * R.len);
    } else if (R.D[k] < 0.0) {
      const int i0 = clampi((int)ceil(el) - 1, lo[k], hi[k] - 1);
      const int i1 = clampi((int)floor(xl), lo[k], hi[k] - 1);
      W.i[k] = i0;
      W.N[k] = max(i0 - i1, 0);
      W.step[k] = -1;
      const double tc = ((double)i0 - R.A[k]) * R.rcp[k];
      W.l0[k] = (float)((tc - t_in) * R.len);
      W.inc[k] = (float)(-R.rcp[k] * R.len);
    } else {
      W.i[k] = clampi((int)floor(el), lo[k], hi[k] - 1);
      W.N[k] = 0;
      W.step[k] = 1;
      W.l0[k] = CUDART_INF_F;
      W.inc[k] = 0.f;
    }
  }
  W.L = (float)((t_out - t_in) * R.len);
}

// FP32 Siddon walk: visits (offset, physical segment length) for every voxel
// of the clipped segment in order; offsets advance by the signed strides.
template <typename Off, typename Visit>
__device__ __forceinline__ void walk(const Walk& W, Off off, Off sx, Off sy, Off sz, Visit&& visit) {
  float nx = W.N[0] > 0 ? W.l0[0] : CUDART_INF_F;
  float ny = W.N[1] > 0 ? W.l0[1] : CUDART_INF_F;
  float nz = W.N[2] > 0 ? W.l0[2] : CUDART_INF_F;
  int jx = 0, jy = 0, jz = 0;
  const int total = W.N[0] + W.N[1] + W.N[2];
  const float L = W.L;
  float cur = 0.f;
  for (int it = 0; it < total; ++it) {
    const float m = fminf(fminf(nx, ny), fminf(nz, L));
    visit(off, m - cur);
    cur = m;
    if (nx <= ny && nx <= nz) {
      off += sx;
      ++jx;
      nx = jx < W.N[0] ? fmaf((float)jx, W.inc[0], W.l0[0]) : CUDART_INF_F;
    } else if (ny <= nz) {
      off += sy;
      ++jy;
      ny = jy < W.N[1] ? fmaf((float)jy, W.inc[1], W.l0[1]) : CUDART_INF_F;
    } else {
      off += sz;
      ++jz;
      nz = jz < W.N[2] ? fmaf((float)jz, W.inc[2], W.l0[2]) : CUDART_INF_F;
    }
  }
  visit(off, L - cur);
}

// ------------------------------------------------------------------ forward --

template <typename Off>
__global__ void __launch_bounds__(kFwdCols* kFwdRows) forward_kernel(FwdLaunch P, const ViewRec* __restrict__ views,
                                                                     const double* __restrict__ trig,
                                                                     const float* __restrict__ vol,
                                                                     const float* __restrict__ volT,
                                                                     float* __restrict__ sino) {
  const int per_band = P.dims.n_views * P.n_col_tiles;
  const int band = blockIdx.x / per_band;
  const int rem = blockIdx.x - band * per_band;
  const int v = rem / P.n_col_tiles;
  const int ct = rem - v * P.n_col_tiles;
  const int c = ct * kFwdCols + threadIdx.x;
  const int r = band * kFwdRows + threadIdx.y;
  if (c >= P.dims.n_cols || r >= P.dims.n_rows) return;

  const ViewRec& V = views[v];
  Ray R;
  make_ray(V, P.vol, trig, P.dims, v, r, c, R);
  const int lo[3] = {0, 0, 0};
  const int hi[3] = {P.vol.n[0], P.vol.n[1], P.vol.n[2]};
  double t_in, t_out;
  float acc = 0.f;
  if (clip(R, lo, hi, t_in, t_out)) {
    Walk W;
    entry(R, t_in, t_out, lo, hi, W);
    const Off nx = P.vol.n[0], ny = P.vol.n[1];
    const bool yfast = V.layout != 0;
    const float* __restrict__ base = yfast ? volT : vol;
    const Off sx = yfast ? ny : (Off)1;
    const Off sy = yfast ? (Off)1 : nx;
    const Off sz = nx * ny;
    const Off off = (Off)W.i[2] * sz + (Off)W.i[1] * sy + (Off)W.i[0] * sx;
    walk<Off>(W, off, W.step[0] * sx, W.step[1] * sy, W.step[2] * sz,
              [&](Off o, float len) { acc = fmaf(len, __ldg(base + o), acc); });
  }
  sino[((size_t)v * P.dims.n_rows + r) * P.dims.n_cols + c] = acc;
}

// ------------------------------------------------------------------- count --

__global__ void __launch_bounds__(kFwdCols* kFwdRows) count_kernel(FwdLaunch P, const ViewRec* __restrict__ views,
                                                                   const double* __restrict__ trig,
                                                                   unsigned long long* __restrict__ counter) {
  const int per_band = P.dims.n_views * P.n_col_tiles;
  const int band = blockIdx.x / per_band;
  const int rem = blockIdx.x - band * per_band;
  const int v = rem / P.n_col_tiles;
  const int ct = rem - v * P.n_col_tiles;
  const int c = ct * kFwdCols + threadIdx.x;
  const int r = band * kFwdRows + threadIdx.y;
  unsigned long long n = 0;
  if (c < P.dims.n_cols && r < P.dims.n_rows) {
    Ray R;
    make_ray(views[v], P.vol, trig, P.dims, v, r, c, R);
    const int lo[3] = {0, 0, 0};
    const int hi[3] = {P.vol.n[0], P.vol.n[1], P.vol.n[2]};
    double t_in, t_out;
    if (clip(R, lo, hi, t_in, t_out)) {
      Walk W;
      entry(R, t_in, t_out, lo, hi, W);
      walk<int>(W, 0, 0, 0, 0, [&](int, float len) { n += len > 0.f ? 1ull : 0ull; });
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
  if ((threadIdx.x & 31) == 0 && n) atomicAdd(counter, n);
}

// ---------------------------------------------------------------- transpose --

__global__ void __launch_bounds__(256) transpose_xy_kernel(const float* __restrict__ in, float* __restrict__ out,
                                                           int nx, int ny) {
  __shared__ float tile[32][33];
  const size_t slice = (size_t)blockIdx.z * nx * ny;
  const int x0 = blockIdx.x * 32, y0 = blockIdx.y * 32;
  for (int j = threadIdx.y; j < 32; j += 8) {
    const int x = x0 + threadIdx.x, y = y0 + j;
    if (x < nx && y < ny) tile[j][threadIdx.x] = in[slice + (size_t)y * nx + x];
  }
  __syncthreads();
  for (int j = threadIdx.y; j < 32; j += 8) {
    const int y = y0 + threadIdx.x, x = x0 + j;
    if (x < nx && y < ny) out[slice + (size_t)x * ny + y] = tile[threadIdx.x][j];
  }
}

// -------------------------------------------------------------- back: brick --

// Detector footprint of the brick [lo, hi) in view V: a rectangle of pixels
// that contains every pixel whose ray can meet the brick.  Computed by one
// warp (lanes 0-7 project the eight corners); all lanes return the result.
__device__ void brick_footprint(const ViewRec& V, const BackLaunch& P, const int lo[3], const int hi[3], int lane,
                                int& c0, int& c1, int& r0, int& r1) {
  const int nc = P.dims.n_cols, nr = P.dims.n_rows;
  if (V.full_footprint) {
    c0 = 0, c1 = nc - 1, r0 = 0, r1 = nr - 1;
    return;
  }
  const int q = lane & 7;
  double X[3];
  const int cv[3] = {(q & 1) ? hi[0] : lo[0], (q & 2) ? hi[1] : lo[1], (q & 4) ? hi[2] : lo[2]};
#pragma unroll
  for (int k = 0; k < 3; ++k) X[k] = P.vol.origin[k] + (double)cv[k] * P.vol.spacing[k];
  double cmin, cmax, rmin, rmax;
  int bad = 0;
  if (P.dims.beam == CTP_BEAM_PARALLEL) {
    const double d[3] = {X[0] - V.p00[0], X[1] - V.p00[1], X[2] - V.p00[2]};
    cmin = cmax = V.minv[0] * d[0] + V.minv[1] * d[1] + V.minv[2] * d[2];
    rmin = rmax = V.minv[3] * d[0] + V.minv[4] * d[1] + V.minv[5] * d[2];
  } else if (P.dims.det == CTP_DET_FLAT) {
    const double d[3] = {X[0] - V.s[0], X[1] - V.s[1], X[2] - V.s[2]};
    const double lam = V.minv[0] * d[0] + V.minv[1] * d[1] + V.minv[2] * d[2];
    const double lc = V.minv[3] * d[0] + V.minv[4] * d[1] + V.minv[5] * d[2];
    const double lr = V.minv[6] * d[0] + V.minv[7] * d[1] + V.minv[8] * d[2];
    if (!(lam > 1e-12)) {
      bad = 1;
      cmin = cmax = rmin = rmax = 0.0;
    } else {
      cmin = cmax = lc / lam;
      rmin = rmax = lr / lam;
    }
  } else {
    // cylindrical: column from the angle about the source's axis, row from
    // the ray's height where it reaches radius R (bounded via rho's range).
    double Xc[3], hd2 = 0.0;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      Xc[k] = P.vol.origin[k] + 0.5 * (double)(lo[k] + hi[k]) * P.vol.spacing[k] - V.s[k];
      const double e = 0.5 * (double)(hi[k] - lo[k]) * P.vol.spacing[k];
      hd2 += e * e;
    }
    const double ac = Xc[0] * V.w[0] + Xc[1] * V.w[1] + Xc[2] * V.w[2];
    const double bc = Xc[0] * V.du[0] + Xc[1] * V.du[1] + Xc[2] * V.du[2];
    const double rel[3] = {X[0] - V.s[0], X[1] - V.s[1], X[2] - V.s[2]};
    const double a = rel[0] * V.w[0] + rel[1] * V.w[1] + rel[2] * V.w[2];
    const double b = rel[0] * V.du[0] + rel[1] * V.du[1] + rel[2] * V.du[2];
    const double h = rel[0] * V.vhat[0] + rel[1] * V.vhat[1] + rel[2] * V.vhat[2];
    const double phi = atan2(bc, ac) + atan2(ac * b - bc * a, ac * a + bc * b);
    cmin = cmax = (phi - V.gam0) / V.dgam;
    rmin = rmax = h;  // reduced below, then converted with the rho bounds
    const double rho_c = sqrt(ac * ac + bc * bc), hd = sqrt(hd2);
    if (!(rho_c - hd > 1e-9)) bad = 1;
  }
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) {
    cmin = fmin(cmin, __shfl_xor_sync(0xffffffffu, cmin, o));
    cmax = fmax(cmax, __shfl_xor_sync(0xffffffffu, cmax, o));
    rmin = fmin(rmin, __shfl_xor_sync(0xffffffffu, rmin, o));
    rmax = fmax(rmax, __shfl_xor_sync(0xffffffffu, rmax, o));
    bad |= __shfl_xor_sync(0xffffffffu, bad, o);
  }
  if (bad) {
    c0 = 0, c1 = nc - 1, r0 = 0, r1 = nr - 1;
    return;
  }
  if (P.dims.beam == CTP_BEAM_CONE && P.dims.det == CTP_DET_CYLINDRICAL) {
    double Xc[3], hd2 = 0.0;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      Xc[k] = P.vol.origin[k] + 0.5 * (double)(lo[k] + hi[k]) * P.vol.spacing[k] - V.s[k];
      const double e = 0.5 * (double)(hi[k] - lo[k]) * P.vol.spacing[k];
      hd2 += e * e;
    }
    const double ac = Xc[0] * V.w[0] + Xc[1] * V.w[1] + Xc[2] * V.w[2];
    const double bc = Xc[0] * V.du[0] + Xc[1] * V.du[1] + Xc[2] * V.du[2];
    const double rho_c = sqrt(ac * ac + bc * bc), hd = sqrt(hd2);
    const double rho_lo = rho_c - hd, rho_hi = rho_c + hd;
    const double hmin = rmin, hmax = rmax;
    const double q_lo = hmin >= 0.0 ? hmin / rho_hi : hmin / rho_lo;
    const double q_hi = hmax >= 0.0 ? hmax / rho_lo : hmax / rho_hi;
    rmin = (q_lo * V.R - V.axial0) / V.vlen;
    rmax = (q_hi * V.R - V.axial0) / V.vlen;
  }
  const double cl = fmax(floor(cmin - 1e-7), -1.0), ch = fmin(ceil(cmax + 1e-7), (double)nc);
  const double rl = fmax(floor(rmin - 1e-7), -1.0), rh = fmin(ceil(rmax + 1e-7), (double)nr);
  c0 = max((int)cl, 0);
  c1 = min((int)ch, nc - 1);
  r0 = max((int)rl, 0);
  r1 = min((int)rh, nr - 1);
}

template <typename Off>
__global__ void __launch_bounds__(kBackThreads) back_brick_kernel(BackLaunch P, const ViewRec* __restrict__ views,
                                                                  const double* __restrict__ trig,
                                                                  const float* __restrict__ sino,
                                                                  float* __restrict__ vol) {
  extern __shared__ float acc[];
  __shared__ int fp[kBackChunk][3];  // c0, r0, width per staged view
  __shared__ int pre[kBackChunk + 1];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int b = blockIdx.x;
  const int g = b % P.view_groups;
  b /= P.view_groups;
  const int bx = b % P.nbrick[0];
  b /= P.nbrick[0];
  const int by = b % P.nbrick[1];
  const int bz = b / P.nbrick[1];
  const int lo[3] = {bx * P.brick[0], by * P.brick[1], bz * P.brick[2]};
  const int hi[3] = {min(lo[0] + P.brick[0], P.vol.n[0]), min(lo[1] + P.brick[1], P.vol.n[1]),
                     min(lo[2] + P.brick[2], P.vol.n[2])};
  const int pitch = P.pitch_x;
  const int plane = pitch * P.brick[1];
  const int n_acc = plane * P.brick[2];
  for (int i = tid; i < n_acc; i += kBackThreads) acc[i] = 0.f;

  const int nr = P.dims.n_rows, nc = P.dims.n_cols;
  const int v_begin = g * P.views_per_group;
  const int v_end = min(v_begin + P.views_per_group, P.dims.n_views);
  for (int vb = v_begin; vb < v_end; vb += kBackChunk) {
    __syncthreads();  // previous chunk's footprints consumed (and accumulators zeroed)
    if (warp < kBackChunk) {
      const int v = vb + warp;
      int c0 = 0, c1 = -1, r0 = 0, r1 = -1;
      if (v < v_end) brick_footprint(views[v], P, lo, hi, lane, c0, c1, r0, r1);
      if (lane == 0) {
        const int w = c1 >= c0 ? c1 - c0 + 1 : 0;
        const int h = r1 >= r0 ? r1 - r0 + 1 : 0;
        fp[warp][0] = c0;
        fp[warp][1] = r0;
        fp[warp][2] = w;
        pre[warp + 1] = w * h;  // count, turned into a prefix sum below
      }
    }
    __syncthreads();
    if (tid == 0) {
      pre[0] = 0;
      for (int s = 0; s < kBackChunk; ++s) pre[s + 1] += pre[s];
    }
    __syncthreads();
    const int total = pre[kBackChunk];
    for (int q = tid; q < total; q += kBackThreads) {
      int s = 0;
      while (q >= pre[s + 1]) ++s;
      const int qq = q - pre[s];
      const int w = fp[s][2];
      const int rr = qq / w;
      const int r = fp[s][1] + rr, c = fp[s][0] + (qq - rr * w);
      const int v = vb + s;
      const float y = __ldg(sino + ((size_t)v * nr + r) * nc + c);
      if (y == 0.f) continue;
      Ray R;
      make_ray(views[v], P.vol, trig, P.dims, v, r, c, R);
      double t_in, t_out;
      if (!clip(R, lo, hi, t_in, t_out)) continue;
      Walk W;
      entry(R, t_in, t_out, lo, hi, W);
      const int off = ((W.i[2] - lo[2]) * P.brick[1] + (W.i[1] - lo[1])) * pitch + (W.i[0] - lo[0]);
      walk<int>(W, off, W.step[0], W.step[1] * pitch, W.step[2] * plane,
                [&](int o, float len) { atomicAdd(acc + o, len * y); });
    }
  }
  __syncthreads();

  const int ex = hi[0] - lo[0], ey = hi[1] - lo[1], ez = hi[2] - lo[2];
  const int n_out = ex * ey * ez;
  const Off nx = P.vol.n[0], ny = P.vol.n[1];
  for (int i = tid; i < n_out; i += kBackThreads) {
    const int x = i % ex;
    const int t = i / ex;
    const int yy = t % ey;
    const int z = t / ey;
    const float val = acc[(z * P.brick[1] + yy) * pitch + x];
    const Off gi = ((Off)(lo[2] + z) * ny + (Off)(lo[1] + yy)) * nx + (Off)(lo[0] + x);
    if (P.view_groups > 1) {
      if (val != 0.f) atomicAdd(vol + gi, val);
    } else {
      vol[gi] = val;
    }
  }
}

}  // namespace

// ---------------------------------------------------------------- launchers --

cudaError_t launch_transpose_xy(const float* vol, float* volT, const VolDesc& vd, cudaStream_t stream) {
  dim3 grid((vd.n[0] + 31) / 32, (vd.n[1] + 31) / 32, vd.n[2]);
  transpose_xy_kernel<<<grid, dim3(32, 8), 0, stream>>>(vol, volT, vd.n[0], vd.n[1]);
  return cudaGetLastError();
}

cudaError_t launch_forward(const FwdLaunch& p, const ViewRec* views, const double* trig, const float* vol,
                           const float* volT, float* sino, bool wide_index, cudaStream_t stream) {
  const long long blocks = (long long)p.n_row_bands * p.dims.n_views * p.n_col_tiles;
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  dim3 block(kFwdCols, kFwdRows);
  if (wide_index)
    forward_kernel<long long><<<(unsigned)blocks, block, 0, stream>>>(p, views, trig, vol, volT, sino);
  else
    forward_kernel<int><<<(unsigned)blocks, block, 0, stream>>>(p, views, trig, vol, volT, sino);
  return cudaGetLastError();
}

cudaError_t launch_count(const FwdLaunch& p, const ViewRec* views, const double* trig, unsigned long long* counter,
                         cudaStream_t stream) {
  const long long blocks = (long long)p.n_row_bands * p.dims.n_views * p.n_col_tiles;
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  count_kernel<<<(unsigned)blocks, dim3(kFwdCols, kFwdRows), 0, stream>>>(p, views, trig, counter);
  return cudaGetLastError();
}

size_t back_brick_smem_bytes(const int32_t brick[3]) {
  return sizeof(float) * (size_t)(brick[0] + 1) * brick[1] * brick[2];
}

cudaError_t prepare_back_brick(size_t smem_bytes) {
  cudaError_t e = cudaFuncSetAttribute(back_brick_kernel<int>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem_bytes);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(back_brick_kernel<long long>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)smem_bytes);
}

cudaError_t launch_back_brick(const BackLaunch& p, const ViewRec* views, const double* trig, const float* sino,
                              float* vol, bool wide_index, cudaStream_t stream) {
  const long long blocks = (long long)p.nbrick[0] * p.nbrick[1] * p.nbrick[2] * p.view_groups;
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const size_t smem = back_brick_smem_bytes(p.brick);
  cudaError_t e = prepare_back_brick(smem);
  if (e != cudaSuccess) return e;
  if (wide_index)
    back_brick_kernel<long long><<<(unsigned)blocks, kBackThreads, smem, stream>>>(p, views, trig, sino, vol);
  else
    back_brick_kernel<int><<<(unsigned)blocks, kBackThreads, smem, stream>>>(p, views, trig, sino, vol);
  return cudaGetLastError();
}

}  // namespace ctp
