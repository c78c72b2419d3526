// Voxel-driven (gather) adjoint for parallel beams whose slices decouple
// (sm_100a).
//
// When every ray lies in a plane of constant z and the detector rows step
// along z only, the rays of one detector column in one view share their
// (x, y) path, each in the slice its row's height falls in (MBIRJAX "Sharding
// overview", section "Why cone beam").  The adjoint of the cell-constant
// Siddon model (diffct "Execution", section "Precision, training and
// reconstruction") then factors:
//   x[z][y][x] = sum_v sum_c a_v(c; x, y) * ysum[v][c][z],
// where a_v(c; x, y) is the chord of column c's ray through cell (x, y) and
// ysum[v][c][z] sums the sinogram over the rows of column c whose height
// falls in slice z.  MBIRJAX "Projector kernels", paragraph "Forward
// scatters, back gathers", prefers a gather for the back projection: every
// output is written once by the thread that owns it, so no two threads add
// into one voxel, and the result does not depend on scheduling.
//
// Two kernels:
//  * slice_sum_kernel: one thread per (view, column) walks the rows in order
//    of rising height and writes ysum[v][c][0 .. nz4), z fastest;
//  * back_gather_kernel: one warp per cell (x, y), lanes over the slices (16
//    per lane at most, in float4 groups lane + 32 j, so that each 16-byte
//    load of a warp reads 512 contiguous bytes of one ysum column).  For
//    every view it finds the columns whose rays cross the cell from the
//    closed-form chord (a trapezoid in the ray's offset from the cell centre)
//    and adds chord (or chord squared) times the column's slice sums.
//    Blocks are 4 x 4 cells, so the 16 warps of a block read the few columns
//    of one view that cross their tile through L1.
#include <cmath>
#include <limits>

#include "ctp_gather.h"
#include "ctp_ray.cuh"

namespace ctp {

namespace {

constexpr int kGatherTileX = 4;
constexpr int kGatherTileY = 4;
constexpr int kGatherThreads = 32 * kGatherTileX * kGatherTileY;
// tiles per side of the square groups of tiles that consecutive blocks cover,
// so that the blocks in flight read the columns of a compact patch of cells
constexpr int kGatherSuper = 16;
constexpr int kSliceSumThreads = 128;

__global__ void __launch_bounds__(kSliceSumThreads)
    slice_sum_kernel(FwdLaunch P, const ViewRec* __restrict__ views, const float* __restrict__ sino, int nz4,
                     float* __restrict__ ysum) {
  const int ctiles = (P.dims.n_cols + kSliceSumThreads - 1) / kSliceSumThreads;
  const int v = blockIdx.x / ctiles;
  const int c = (blockIdx.x - v * ctiles) * kSliceSumThreads + threadIdx.x;
  const int nr = P.dims.n_rows, nc = P.dims.n_cols;
  if (v >= P.dims.n_views || c >= nc) return;
  const ViewRec& V = views[v];
  // heights rise with the row index when dv_z >= 0: the slice index of the
  // rows, taken in this order, never decreases (rounding is monotone)
  const bool up = V.dv[2] >= 0.0;
  [[maybe_unused]] const size_t total = (size_t)P.dims.n_views * nc * nz4;
  [[maybe_unused]] const size_t n_sino = (size_t)P.dims.n_views * nr * nc;
  const size_t out0 = ((size_t)v * nc + c) * nz4;
  const size_t in0 = (size_t)v * nr * nc + c;
  int cur = -1;   // slice being summed
  int next = 0;   // first slice not yet written
  float s = 0.f;
  constexpr int kU = 8;
  for (int i0 = 0; i0 < nr; i0 += kU) {
    float y[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = i0 + u;
      const int r = up ? i : nr - 1 - i;
      const size_t idx = in0 + (size_t)r * nc;
      y[u] = (i < nr && CTP_IN_BOUNDS(idx, n_sino, 21)) ? __ldg(sino + idx) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = i0 + u;
      if (i >= nr) break;
      const int r = up ? i : nr - 1 - i;
      int k[1];
      if (!row_slice_index<1>(V, P.vol, r, c, nr, k)) continue;
      if (k[0] != cur) {
        if (cur >= 0 && CTP_IN_BOUNDS(out0 + cur, total, 22)) ysum[out0 + cur] = s;
        for (int z = next; z < k[0]; ++z)
          if (CTP_IN_BOUNDS(out0 + z, total, 22)) ysum[out0 + z] = 0.f;
        cur = k[0];
        next = cur + 1;
        s = 0.f;
      }
      s += y[u];
    }
  }
  if (cur >= 0 && CTP_IN_BOUNDS(out0 + cur, total, 22)) ysum[out0 + cur] = s;
  for (int z = next; z < nz4; ++z)
    if (CTP_IN_BOUNDS(out0 + z, total, 22)) ysum[out0 + z] = 0.f;
}

template <int kJ, int kPower>
__global__ void __launch_bounds__(kGatherThreads, 2)
    back_gather_kernel(GatherLaunch P, const GatherView* __restrict__ gv, const float* __restrict__ ysum,
                       float* __restrict__ vol) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // block -> (slice chunk, group of kGatherSuper^2 tiles, tile in the group)
  const int per_chunk = gridDim.x / P.n_zchunks;
  const int zc = blockIdx.x / per_chunk;
  const int b = blockIdx.x - zc * per_chunk;
  const int sgx = (P.tiles_x + kGatherSuper - 1) / kGatherSuper;
  const int grp = b / (kGatherSuper * kGatherSuper), in_grp = b - grp * (kGatherSuper * kGatherSuper);
  const int tx = (grp % sgx) * kGatherSuper + in_grp % kGatherSuper;
  const int ty = (grp / sgx) * kGatherSuper + in_grp / kGatherSuper;
  const int x = tx * kGatherTileX + warp % kGatherTileX;
  const int y = ty * kGatherTileY + warp / kGatherTileX;
  if (tx >= P.tiles_x || ty >= P.tiles_y || x >= P.nx || y >= P.ny) return;  // no block barrier below
  const int g4 = P.nz4 >> 2;  // float4 groups per ysum column
  int q[kJ];
  bool ok[kJ];
  float4 acc[kJ];
#pragma unroll
  for (int j = 0; j < kJ; ++j) {
    q[j] = zc * 32 * kJ + lane + 32 * j;
    ok[j] = q[j] < g4;
    acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const double xd = (double)x, yd = (double)y;
  const int nc = P.n_cols;
  [[maybe_unused]] const size_t n_ysum4 = (size_t)P.n_views * nc * g4;
  const float4* __restrict__ colv = reinterpret_cast<const float4*>(ysum);  // view v's first column
  auto add = [&](float w, const float4* __restrict__ src) {
#pragma unroll
    for (int j = 0; j < kJ; ++j) {
      if (ok[j] && CTP_IN_BOUNDS((src - reinterpret_cast<const float4*>(ysum)) + q[j], n_ysum4, 23)) {
        const float4 t = __ldg(src + q[j]);
        acc[j].x = fmaf(w, t.x, acc[j].x);
        acc[j].y = fmaf(w, t.y, acc[j].y);
        acc[j].z = fmaf(w, t.z, acc[j].z);
        acc[j].w = fmaf(w, t.w, acc[j].w);
      }
    }
  };
  for (int v = 0; v < P.n_views; ++v, colv += (size_t)nc * g4) {
    const GatherView& G = gv[v];
    const double gam = fma(yd, G.gy, fma(xd, G.gx, G.g0));
    if (G.two) {
      // at most two columns cross the cell: the first candidate and the next
      const double c0 = fmax(0.0, ceil(gam - G.halfw));
      const double cmax = fmin((double)(nc - 1), floor(gam + G.halfw));
      const double d0 = G.wh - fabs((gam - c0) * G.kap);
      const double d1 = G.wh - fabs((gam - (c0 + 1.0)) * G.kap);
      const bool h0 = c0 <= cmax && d0 > 0.0;
      const bool h1 = c0 + 1.0 <= cmax && d1 > 0.0;
      if (!(h0 || h1)) continue;
      const float4* __restrict__ src0 = colv + (size_t)(int)c0 * g4;
      if (h0) {
        const float len = fminf(G.lmax, (float)d0 * G.inv_slope);
        add(kPower == 2 ? len * len : len, src0);
      }
      if (h1) {
        const float len = fminf(G.lmax, (float)d1 * G.inv_slope);
        add(kPower == 2 ? len * len : len, src0 + g4);
      }
      continue;
    }
    const int clo = (int)fmax(0.0, ceil(gam - G.halfw));
    const int chi = (int)fmin((double)(nc - 1), floor(gam + G.halfw));
    for (int c = clo; c <= chi; ++c) {
      float len;
      if (G.axis == 0) {
        const double d = G.wh - fabs((gam - (double)c) * G.kap);
        if (!(d > 0.0)) continue;
        len = fminf(G.lmax, (float)d * G.inv_slope);
      } else {
        // the minor-axis position of the ray, as the slab walk computes it
        const double am = (fma((double)c, G.dum, G.p00m) - G.om) * G.invm;
        if (floor(am) != (G.axis == 1 ? yd : xd)) continue;
        len = G.lmax;
      }
      add(kPower == 2 ? len * len : len, colv + (size_t)c * g4);
    }
  }
  const size_t plane = (size_t)P.nx * P.ny;
  const size_t xy = (size_t)y * P.nx + x;
  [[maybe_unused]] const size_t n_vox = plane * P.nz;
#pragma unroll
  for (int j = 0; j < kJ; ++j) {
    if (!ok[j]) continue;
    const float a[4] = {acc[j].x, acc[j].y, acc[j].z, acc[j].w};
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int z = 4 * q[j] + s;
      if (z < P.nz && CTP_IN_BOUNDS(z * plane + xy, n_vox, 24)) vol[z * plane + xy] = a[s];
    }
  }
}

}  // namespace

// ------------------------------------------------------------- host side --

bool build_gather_views(const std::vector<ViewRec>& views, const VolDesc& vd, int64_t n_cols,
                        std::vector<GatherView>& out, std::string& why) {
  out.assign(views.size(), GatherView{});
  const double inf = std::numeric_limits<double>::infinity();
  const double half_diag = 0.5 * std::hypot((double)vd.n[0], (double)vd.n[1]);
  for (size_t v = 0; v < views.size(); ++v) {
    const ViewRec& V = views[v];
    GatherView& G = out[v];
    const double Dx = V.s[0] * vd.inv_spacing[0], Dy = V.s[1] * vd.inv_spacing[1];
    const double adx = std::fabs(Dx), ady = std::fabs(Dy);
    const double Dn = std::hypot(Dx, Dy);
    if (!(Dn > 0.0)) {
      why = "a ray has no (x, y) direction";
      return false;
    }
    // ray position of column c in voxel units (make_ray's expression)
    auto A = [&](double c, int k) { return (std::fma(c, V.du[k], V.p00[k]) - vd.origin[k]) * vd.inv_spacing[k]; };
    // largest |t| at which a column's ray is inside the volume
    double far = 0.0;
    for (double c : {0.0, (double)(n_cols - 1)})
      far = std::fmax(far, std::hypot(A(c, 0) - vd.centre[0], A(c, 1) - vd.centre[1]));
    const double t_ext = (far + half_diag) / Dn;
    const double minor = std::fmin(adx, ady);
    int axis = 0;
    if (minor == 0.0 || minor * t_ext <= 1e-9) {
      axis = adx >= ady ? 1 : 2;
      if (minor != 0.0) {
        // the ray drifts by less than 1e-9 voxels across the volume: it stays
        // in the cell of its floor position unless it runs along a grid line
        const int k = axis == 1 ? 1 : 0;
        for (int64_t c = 0; c < n_cols; ++c) {
          const double am = A((double)c, k);
          if (am < -1.0 || am > (double)vd.n[k] + 1.0) continue;
          const double f = am - std::floor(am);
          if (std::fmin(f, 1.0 - f) < 1e-6) {
            why = "a ray of an axis view runs along a grid line";
            return false;
          }
        }
      }
    }
    const double Nx = axis == 1 ? 0.0 : -Dy;
    const double Ny = axis == 2 ? 0.0 : Dx;
    const double dux = V.du[0] * vd.inv_spacing[0], duy = V.du[1] * vd.inv_spacing[1];
    const double kap = Nx * dux + Ny * duy;
    if (!(std::fabs(kap) > 1e-9 * std::hypot(Nx, Ny) * std::hypot(dux, duy))) {
      why = "rays run along the detector's columns";
      return false;
    }
    const double wh = 0.5 * (std::fabs(Nx) + std::fabs(Ny));
    const double halfw = wh / std::fabs(kap);
    if (!(halfw <= 32.0)) {
      why = "more than 64 columns cross one cell per view";
      return false;
    }
    const double A0x = A(0.0, 0), A0y = A(0.0, 1);
    G.g0 = (Nx * (0.5 - A0x) + Ny * (0.5 - A0y)) / kap;
    G.gx = Nx / kap;
    G.gy = Ny / kap;
    G.kap = kap;
    G.halfw = halfw * (1.0 + 1e-9) + 1e-9;
    G.wh = wh;
    G.lmax = (float)std::fmin(adx > 0.0 ? 1.0 / adx : inf, ady > 0.0 ? 1.0 / ady : inf);
    G.inv_slope = axis == 0 ? (float)(1.0 / (adx * ady)) : 0.f;
    G.axis = axis;
    // at most two integers lie within halfw of any column coordinate
    G.two = axis == 0 && G.halfw < 1.0 ? 1 : 0;
    const int k = axis == 2 ? 0 : 1;
    G.p00m = V.p00[k];
    G.dum = V.du[k];
    G.om = vd.origin[k];
    G.invm = vd.inv_spacing[k];
  }
  return true;
}

GatherLaunch plan_gather(const VolDesc& vd, const Dims& dm) {
  GatherLaunch gl{};
  gl.nx = vd.n[0];
  gl.ny = vd.n[1];
  gl.nz = vd.n[2];
  gl.nz4 = (vd.n[2] + 3) / 4 * 4;
  gl.n_views = dm.n_views;
  gl.n_cols = dm.n_cols;
  gl.tiles_x = (vd.n[0] + kGatherTileX - 1) / kGatherTileX;
  gl.tiles_y = (vd.n[1] + kGatherTileY - 1) / kGatherTileY;
  const int g4 = gl.nz4 / 4;
  gl.j_groups = g4 <= 32 ? 1 : (g4 <= 64 ? 2 : 4);
  gl.n_zchunks = (g4 + 32 * gl.j_groups - 1) / (32 * gl.j_groups);
  return gl;
}

cudaError_t launch_back_gather(const FwdLaunch& p, const GatherLaunch& gl, const ViewRec* views,
                               const GatherView* gviews, const float* sino, float* ysum, float* vol, int power,
                               cudaStream_t stream) {
  const long long ctiles = (p.dims.n_cols + kSliceSumThreads - 1) / kSliceSumThreads;
  const long long sblocks = ctiles * p.dims.n_views;
  if (sblocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  if (sblocks > 0)
    slice_sum_kernel<<<(unsigned)sblocks, kSliceSumThreads, 0, stream>>>(p, views, sino, gl.nz4, ysum);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long sgx = (gl.tiles_x + kGatherSuper - 1) / kGatherSuper;
  const long long sgy = (gl.tiles_y + kGatherSuper - 1) / kGatherSuper;
  const long long blocks = sgx * sgy * kGatherSuper * kGatherSuper * gl.n_zchunks;
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const unsigned nb = (unsigned)blocks;
#define CTP_GATHER_LAUNCH(J)                                                             \
  do {                                                                                     \
    if (power == 2)                                                                        \
      back_gather_kernel<J, 2><<<nb, kGatherThreads, 0, stream>>>(gl, gviews, ysum, vol); \
    else                                                                                   \
      back_gather_kernel<J, 1><<<nb, kGatherThreads, 0, stream>>>(gl, gviews, ysum, vol); \
  } while (0)
  switch (gl.j_groups) {
    case 1:
      CTP_GATHER_LAUNCH(1);
      break;
    case 2:
      CTP_GATHER_LAUNCH(2);
      break;
    default:
      CTP_GATHER_LAUNCH(4);
      break;
  }
#undef CTP_GATHER_LAUNCH
  return cudaGetLastError();
}

unsigned long long debug_take_word_gather() {
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
