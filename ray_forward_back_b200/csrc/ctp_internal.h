// Internal types shared by the host entry points (ctp_api.cu) and the kernels
// (ctp_kernels.cu).  Not part of the public C ABI.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "ctp.h"

namespace ctp {

// Per-view geometry in FP64, prepared on the host at create time.
//
// Pixel centre of (row r, column c), world coordinates:
//   flat:        p = p00 + c * du + r * dv
//   cylindrical: p = p00 + r * dv + R * (cos g * w + sin g * du),  g = gam0 + c * dgam
// (for the cylindrical detector du holds the unit tangent u^ and p00 the
// point on the source's axis at the height of row 0).
struct ViewRec {
  double s[3];        // cone: source position; parallel: unit ray direction
  double p00[3];
  double du[3];
  double dv[3];
  double w[3];        // cylindrical: unit radial direction of the middle column
  double vhat[3];     // unit row direction
  double rcp_dir[3];  // parallel: 1 / (direction in voxel units), +-inf where 0
  double minv[9];     // footprint matrix: parallel flat [du dv s]^-1, cone flat [p00-s du dv]^-1
  double vox_ext[3];  // one voxel's projected extent: parallel (columns, rows, -);
                      // cone flat: sum_k |minv row i, k| * spacing_k for rows i = 0, 1, 2
  double R, gam0, dgam, axial0, vlen;
  double src_norm;    // |src| as given (parallel beam: the direction's length)
  int32_t layout;     // forward gather: 0 = x-fastest volume, 1 = y-fastest copy
  int32_t full_footprint;  // 1: the footprint test cannot bound this view; scan all pixels
};

struct VolDesc {
  int32_t n[3];       // nx, ny, nz
  int32_t pad;
  double origin[3];
  double spacing[3];
  double inv_spacing[3];
  double centre[3];   // volume centre in voxel units (n / 2)
};

struct Dims {
  int32_t beam, det;
  int32_t n_views, n_rows, n_cols;
  int32_t pad;
};

struct FwdLaunch {
  Dims dims;
  VolDesc vol;
  int32_t n_col_tiles, n_row_bands;
  int32_t any_transposed;
  // Rays in z-planes with rows stepping along z: each thread walks one (x, y)
  // path for row_group rows (1 = one walk per ray).  Used by the
  // single-volume forward and the scatter adjoint.
  int32_t row_group;
  int32_t interleaved;  // row_group 4 on volumes interleaved by 4 slices (the rows4 kernels)
};

struct BackLaunch {
  Dims dims;
  VolDesc vol;
  int32_t brick[3];      // brick size
  int32_t nbrick[3];     // bricks per axis
  int32_t pitch_x;       // shared-memory row pitch (brick[0] + 1)
  int32_t view_groups;   // CTA groups over the views; >1 means atomic flush into a zeroed volume
  int32_t views_per_group;
  int32_t pad;
};

// Launchers (ctp_kernels.cu).  All enqueue on `stream` and return the launch error.
cudaError_t launch_transpose_xy(const float* vol, float* volT, const VolDesc& vd, cudaStream_t stream);
// Forward of kb (1, 2 or 4) volumes at vol, vol + n_vox, ... (their y-fastest
// copies at volT, volT + n_vox, ...) into kb sinograms at sino, sino + n_rays, ...
cudaError_t launch_forward(const FwdLaunch& p, const ViewRec* views, const double* trig, const float* vol,
                           const float* volT, float* sino, int kb, bool wide_index, cudaStream_t stream);
// Brick adjoint of kb (1 or 2) batch members: sinograms at sino, sino + n_rays,
// volumes at vol, vol + n_vox.
// The single-volume forward with one (x, y) walk per p.row_group rows.
cudaError_t launch_forward_rows(const FwdLaunch& p, const ViewRec* views, const float* vol, const float* volT,
                                float* sino, bool wide_index, cudaStream_t stream);
// Slices interleaved by 4 (element [g][y][x][s] = slice 4g + s; vol4T with x
// and y swapped): the forward interleaves vol into vol4 (and vol4T if some
// view gathers y-fastest), then walks 4 rows per thread reading 16 bytes per
// segment; the adjoint adds into the zeroed acc4 / acc4T with 16-byte
// reductions, then writes vol from them.
cudaError_t launch_interleave(const FwdLaunch& p, const float* vol, float4* vol4, float4* vol4T,
                              cudaStream_t stream);
// Geometry gradients with one (x, y) walk per 4 rows on the interleaved copies
// (written by launch_interleave first).
cudaError_t launch_geometry_gradient_rows4(const FwdLaunch& p, const ViewRec* views, const float4* vol4,
                                           const float4* vol4T, const float* gsino, double* grad, bool wide_index,
                                           cudaStream_t stream);
cudaError_t launch_forward_rows4(const FwdLaunch& p, const ViewRec* views, const float* vol, float4* vol4,
                                 float4* vol4T, float* sino, bool wide_index, cudaStream_t stream);
cudaError_t launch_back_scatter_rows4(const FwdLaunch& p, const ViewRec* views, const float* sino, float* vol,
                                      float4* acc4, float4* acc4T, int power, bool wide_index, cudaStream_t stream);
cudaError_t launch_back_brick(const BackLaunch& p, const ViewRec* views, const double* trig, const float* sino,
                              float* vol, int power, int kb, bool wide_index, cudaStream_t stream);
cudaError_t launch_count(const FwdLaunch& p, const ViewRec* views, const double* trig,
                         unsigned long long* counter, cudaStream_t stream);
cudaError_t launch_back_sort(const FwdLaunch& p, const ViewRec* views, const double* trig, const float* sino,
                             float* vol, int power, bool wide_index, cudaStream_t stream);
// Ray-driven scatter adjoint into vol (x-fastest views) and volT (y-fastest
// views), both zeroed by the caller; volT is then added into vol.
cudaError_t launch_back_scatter(const FwdLaunch& p, const ViewRec* views, const double* trig, const float* sino,
                                float* vol, float* volT, int power, bool wide_index, cudaStream_t stream);
cudaError_t launch_collision_count(const FwdLaunch& p, const ViewRec* views, const double* trig,
                                   unsigned long long* counters, bool wide_index, cudaStream_t stream);
size_t back_brick_smem_bytes(const int32_t brick[3], int kb = 1);
cudaError_t launch_geometry_gradient(const FwdLaunch& p, const ViewRec* views, const double* trig, const float* vol,
                                     const float* volT, const float* gsino, double* grad, bool wide_index,
                                     cudaStream_t stream);

// Bounds-check words of the CTP_DEBUG build (ctp_kernels.cu, ctp_grad.cu):
// read and cleared, synchronously; always 0 in other builds.
unsigned long long debug_take_word_kernels();
unsigned long long debug_take_word_grad();

// Host helpers (ctp_api.cu).
ctp_status host_validate(const ctp_geom_desc* d);
ctp_status host_view_record(const ctp_geom_desc* d, int64_t v, ViewRec& V, double* trig_row);
ctp_status host_error(ctp_status s, const char* msg);
ctp_status host_cuda_error(cudaError_t e, const char* where);
bool host_is_device_pointer(const void* ptr, int device);
void host_clear_error();
// Raise the brick adjoint's dynamic shared-memory limit on the current
// device to at least smem_bytes (kb members); never lowers it, so handles
// with larger bricks stay launchable.  Called at create only.
cudaError_t prepare_back_brick(size_t smem_bytes, int kb = 1);

}  // namespace ctp
