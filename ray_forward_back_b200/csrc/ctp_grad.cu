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
// gives the det_c, det_u and det_v gradients.  Kinks (a ray through a voxel
// edge, an endpoint on a plane) have no derivative; the formula then returns
// one of the one-sided values.
//
// Kernel: one thread per ray on the forward's grid (a block is 32 columns x 8
// rows of one view), FP64 setup shared with the projectors, a merged Siddon
// walk that visits every crossing in order (FP32 crossing distances from
// exact integers, FP64 sums), then a block reduction and 12 FP64 atomics per
// block into grad[view][4][3].
#include "ctp_ray.cuh"

namespace ctp {
namespace {

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

__device__ __forceinline__ void add_axis(int k, double v, double& s0, double& s1, double& s2) {
  s0 += k == 0 ? v : 0.0;
  s1 += k == 1 ? v : 0.0;
  s2 += k == 2 ? v : 0.0;
}

template <typename Off>
__global__ void __launch_bounds__(kGradThreads) geometry_gradient_kernel(FwdLaunch P,
                                                                         const ViewRec* __restrict__ views,
                                                                         const double* __restrict__ trig,
                                                                         const float* __restrict__ vol,
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

  const ViewRec& V = views[v];
  Ray R;
  const bool from_pixel = make_ray(V, P.vol, trig, P.dims, v, valid ? r : 0, valid ? c : 0, R);
  const int lo[3] = {0, 0, 0};
  const int hi[3] = {P.vol.n[0], P.vol.n[1], P.vol.n[2]};
  double t_in = 0.0, t_out = 0.0;
  int k_in = -1, k_out = -1;
  const float gr = valid ? gsino[((size_t)v * P.dims.n_rows + r) * P.dims.n_cols + c] : 0.f;
  const bool hit = valid && gr != 0.f && clip_faces(R, hi, t_in, t_out, k_in, k_out);

  // per-axis sums S0_k and sum of dx * (local distance from the entry)
  double S0x = 0.0, S0y = 0.0, S0z = 0.0, Slx = 0.0, Sly = 0.0, Slz = 0.0, x_end = 0.0;
  if (hit) {
    Walk W;
    entry(R, t_in, t_out, lo, hi, W);
    const Off nx = P.vol.n[0], ny = P.vol.n[1];
    const Off sx = W.step[0], sy = W.step[1] * nx, sz = W.step[2] * nx * ny;
    Off off = (Off)W.i[2] * nx * ny + (Off)W.i[1] * nx + (Off)W.i[0];
    float cur = __ldg(vol + off);
    if (k_in >= 0) add_axis(k_in, -(double)cur, S0x, S0y, S0z);  // enters through a face at local distance 0
    // merged walk: every crossing in order of distance; an axis takes part
    // only while it has crossings left, so each axis moves exactly N_k times
    int jx = 0, jy = 0, jz = 0;
    float lx = W.l0[0], ly = W.l0[1], lz = W.l0[2];
    const int total = W.N[0] + W.N[1] + W.N[2];
    for (int n = 0; n < total; ++n) {
      const bool ex = jx < W.N[0], ey = jy < W.N[1], ez = jz < W.N[2];
      const int k = (ex && (!ey || lx <= ly) && (!ez || lx <= lz)) ? 0 : ((ey && (!ez || ly <= lz)) ? 1 : 2);
      const float l = k == 0 ? lx : (k == 1 ? ly : lz);
      off += k == 0 ? sx : (k == 1 ? sy : sz);
      const float nxt = __ldg(vol + off);
      const double dx = (double)cur - (double)nxt;
      add_axis(k, dx, S0x, S0y, S0z);
      add_axis(k, dx * (double)l, Slx, Sly, Slz);
      cur = nxt;
      if (k == 0) {
        ++jx;
        lx = fmaf((float)jx, W.inc[0], W.l0[0]);
      } else if (k == 1) {
        ++jy;
        ly = fmaf((float)jy, W.inc[1], W.l0[1]);
      } else {
        ++jz;
        lz = fmaf((float)jz, W.inc[2], W.l0[2]);
      }
    }
    if (k_out >= 0) {  // leaves through a face at local distance L
      const double L = (t_out - t_in) * R.len;
      add_axis(k_out, (double)cur, S0x, S0y, S0z);
      add_axis(k_out, (double)cur * L, Slx, Sly, Slz);
    } else {
      x_end = (double)cur;
    }
  }

  // per-ray gradients: G_src (3) and G_pix (3), weighted by g
  double gs[3] = {0.0, 0.0, 0.0}, gp[3] = {0.0, 0.0, 0.0};
  if (hit) {
    const double S0[3] = {S0x, S0y, S0z};
    const double Sl[3] = {Slx, Sly, Slz};
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
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    acc[k] = gs[k];
    acc[3 + k] = gp[k];
    acc[6 + k] = cu * gp[k];
    acc[9 + k] = rv * gp[k];
  }
  // block reduction: warps by shuffles, then one warp over the 8 warp sums
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

}  // namespace

cudaError_t launch_geometry_gradient(const FwdLaunch& p, const ViewRec* views, const double* trig, const float* vol,
                                     const float* gsino, double* grad, bool wide_index, cudaStream_t stream) {
  const long long blocks = (long long)p.n_row_bands * p.dims.n_views * p.n_col_tiles;
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  dim3 block(kGradCols, kGradRows);
  if (wide_index)
    geometry_gradient_kernel<long long><<<(unsigned)blocks, block, 0, stream>>>(p, views, trig, vol, gsino, grad);
  else
    geometry_gradient_kernel<int><<<(unsigned)blocks, block, 0, stream>>>(p, views, trig, vol, gsino, grad);
  return cudaGetLastError();
}

}  // namespace ctp
