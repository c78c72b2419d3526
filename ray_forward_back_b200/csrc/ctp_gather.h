// Voxel-driven (gather) adjoint for parallel beams whose slices decouple:
// host-side plan records and launchers (ctp_gather.cu).  Not part of the
// public C ABI.
#pragma once

#include <string>
#include <vector>

#include "ctp_internal.h"

namespace ctp {

// Per-view constants of the gather, FP64, built on the host at create.
//
// In voxel units the ray of column c is A(c) + t D in the (x, y) plane (the
// same for every detector row).  With N = (-D_y, D_x) the signed offset of
// the centre m of cell (x, y) from that ray is N . (m - A(c)), which is
// linear in c: (gamma - c) kap with gamma = g0 + x gx + y gy.  The chord of
// the ray through the cell, as a function of that offset, is a trapezoid:
// lmax where |offset| <= |(|D_x| - |D_y|)| / 2, falling linearly to zero at
// wh = (|D_x| + |D_y|) / 2, with slope 1 / (|D_x| |D_y|).  Views whose ray
// direction lies on an axis (axis 1: along x, axis 2: along y, including
// directions whose drift across the volume is below 1e-9 voxels) place the
// ray by the floor of its minor-axis position, as the slab walk does.
struct __align__(16) GatherView {
  double g0, gx, gy;  // column coordinate of a cell centre
  double kap;         // offset of the cell centre per column
  double halfw;       // candidate columns: |gamma - c| <= halfw
  double wh;          // half-width of the cell's shadow across the rays
  float lmax;         // chord along the full cell in the ray's major axis
  float inv_slope;    // 1 / (|D_x| |D_y|), general views
  int32_t axis;       // 0 general, 1 along x, 2 along y
  int32_t two;        // general view whose cells at most two columns cross
  double p00m, dum, om, invm;  // axis views: minor-axis p00, du, origin and 1 / spacing
};

struct GatherLaunch {
  int32_t nx, ny, nz;
  int32_t nz4;                  // slices per sinogram column of the slice sums, nz rounded up to 4
  int32_t n_views, n_cols;
  int32_t tiles_x, tiles_y;     // cell tiles of kGatherTileX x kGatherTileY
  int32_t n_zchunks;            // slice chunks of 32 * j_groups float4 groups
  int32_t j_groups;             // float4 groups of slices per lane: 1, 2 or 4
};

// Records of every view, or false (with the reason) when some view does not
// suit the gather: a ray running along the detector's columns, columns more
// than 32 apart per voxel in the offset, or an axis view with a ray within
// 1e-6 voxels of a grid line (where the walk's rounding decides the cell).
bool build_gather_views(const std::vector<ViewRec>& views, const VolDesc& vd, int64_t n_cols,
                        std::vector<GatherView>& out, std::string& why);
GatherLaunch plan_gather(const VolDesc& vd, const Dims& dm);

// Slice sums of the sinogram: ysum[v][c][z] = sum of sino[v][r][c] over the
// rows r whose height falls in slice z (row order), 0 for slices no row
// reaches; then vol[z][y][x] = sum over views and columns of coef * ysum.
// Every voxel of vol is written (no zero-fill needed).
cudaError_t launch_back_gather(const FwdLaunch& p, const GatherLaunch& gl, const ViewRec* views,
                               const GatherView* gviews, const float* sino, float* ysum, float* vol, int power,
                               cudaStream_t stream);

// Bounds-check word of this file's kernels (CTP_DEBUG builds; 0 elsewhere).
unsigned long long debug_take_word_gather();

}  // namespace ctp
