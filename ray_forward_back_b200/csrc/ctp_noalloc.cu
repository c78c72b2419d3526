// ctp_forward_noalloc: the forward projection for callers that cannot
// allocate device memory at all (see include/ctp.h).  Everything the call
// needs beyond the caller's volume and sinogram -- the per-view FP64 records,
// the cylindrical column table and the y-fastest copy of the volume -- lives
// in one file-scope device array of fixed size.  Nothing here allocates:
// no cudaMalloc/cudaFree, no host heap; records are built in a stack buffer,
// column rows in a static staging array, and both are copied with
// cudaMemcpyAsync (pageable source, consumed before the copy call returns).
#include <cmath>
#include <cstdio>
#include <mutex>

#include "ctp_internal.h"

namespace {

constexpr size_t kScratchBytes = CTP_NOALLOC_SCRATCH_BYTES;
constexpr int kChunk = 32;  // view records built and copied per cudaMemcpyAsync

// The scratch.  Every GPU that loads the library holds it until exit; all
// calls on a device share it and it keeps the last call's contents.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

// Serialises the host part of the calls (the staging buffer below).
std::mutex g_mu;

// Host staging for the cylindrical column table: whole views' rows of cos/sin
// pairs are packed here and sent with one copy (a static array, not heap).
constexpr size_t kTrigStage = 1 << 16;  // doubles (512 KiB)
double g_trig_stage[kTrigStage];

// Device address of g_scratch on the current device.  The host-side name is
// only a stand-in; the address is looked up on every call (no allocation, and
// no stale address after the caller resets the device).
cudaError_t scratch_address(unsigned char** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
  if (e != cudaSuccess) return e;
  *out = static_cast<unsigned char*>(p);
  return cudaSuccess;
}

size_t align256(size_t n) { return (n + 255) & ~(size_t)255; }

struct CurrentDevice {
  int prev = -1;
  bool switched = false;
  cudaError_t err = cudaSuccess;
  explicit CurrentDevice(int dev) {
    err = cudaGetDevice(&prev);
    if (err == cudaSuccess && prev != dev) {
      err = cudaSetDevice(dev);
      switched = err == cudaSuccess;
    }
  }
  ~CurrentDevice() {
    if (switched) cudaSetDevice(prev);
  }
};

}  // namespace

extern "C" ctp_status ctp_forward_noalloc(const ctp_geom_desc* desc, const float* vol, float* sino, void* stream) {
  using namespace ctp;
  host_clear_error();
  ctp_status st = host_validate(desc);
  if (st != CTP_OK) return st;
  const ctp_geom_desc& d = *desc;
  if (d.device < 0) return host_error(CTP_ERR_INVALID_ARGUMENT, "device ordinal out of range");

  // pass 1 (host only): guards of every view and the layout plan
  ViewRec rec[kChunk];
  int64_t n_transposed = 0;
  for (int64_t v = 0; v < d.n_views; ++v) {
    st = host_view_record(desc, v, rec[0], nullptr);
    if (st != CTP_OK) return st;
    n_transposed += rec[0].layout != 0;
  }
  const int64_t n_vox = d.nx * d.ny * d.nz;
  const size_t rec_bytes = align256(sizeof(ViewRec) * (size_t)d.n_views);
  const size_t trig_bytes =
      d.detector == CTP_DET_CYLINDRICAL ? align256(sizeof(double) * 2 * (size_t)(d.n_views * d.n_cols)) : 0;
  const size_t copy_bytes = n_transposed > 0 ? sizeof(float) * (size_t)n_vox : 0;
  if (rec_bytes + trig_bytes + copy_bytes > kScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "ctp_forward_noalloc needs %zu bytes of scratch (view records %zu, column table %zu, volume copy %zu); "
             "its fixed scratch holds %zu",
             rec_bytes + trig_bytes + copy_bytes, rec_bytes, trig_bytes, copy_bytes, kScratchBytes);
    return host_error(CTP_ERR_OUT_OF_RANGE, msg);
  }

  CurrentDevice cd(d.device);
  if (cd.err != cudaSuccess) return host_cuda_error(cd.err, "cudaSetDevice");
  cudaStream_t s = (cudaStream_t)stream;
  // The uploads below copy from this call's host memory, which is gone (or
  // reused) once the call returns: a graph captured from them would replay
  // stale copies, so a capturing stream is refused before anything is enqueued.
  cudaStreamCaptureStatus capturing = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(s, &capturing);
  if (e != cudaSuccess) return host_cuda_error(e, "cudaStreamIsCapturing");
  if (capturing != cudaStreamCaptureStatusNone)
    return host_error(CTP_ERR_UNSUPPORTED, "ctp_forward_noalloc does not run on a stream that is capturing");
  if (!host_is_device_pointer(vol, d.device))
    return host_error(CTP_ERR_INVALID_ARGUMENT, "vol is not device memory of the described device");
  if (!host_is_device_pointer(sino, d.device))
    return host_error(CTP_ERR_INVALID_ARGUMENT, "sino is not device memory of the described device");
  std::lock_guard<std::mutex> lock(g_mu);
  unsigned char* base = nullptr;
  e = scratch_address(&base);
  if (e != cudaSuccess) return host_cuda_error(e, "cudaGetSymbolAddress");
  ViewRec* d_views = reinterpret_cast<ViewRec*>(base);
  double* d_trig = trig_bytes ? reinterpret_cast<double*>(base + rec_bytes) : nullptr;
  float* d_copy = copy_bytes ? reinterpret_cast<float*>(base + rec_bytes + trig_bytes) : nullptr;
  e = cudaGetLastError();
  if (e != cudaSuccess) return host_cuda_error(e, "pending error before ctp_forward_noalloc");

  // pass 2: records to the scratch, kChunk views per copy; column rows of as
  // many whole views as the staging buffer holds per copy (a row wider than
  // the buffer goes in pieces)
  const size_t row = 2 * (size_t)d.n_cols;  // doubles per view
  int64_t staged_v0 = 0;
  size_t staged = 0;
  auto flush_trig = [&]() -> cudaError_t {
    if (!staged) return cudaSuccess;
    const cudaError_t err = cudaMemcpyAsync(d_trig + (size_t)staged_v0 * row, g_trig_stage, sizeof(double) * staged,
                                            cudaMemcpyHostToDevice, s);
    staged = 0;
    return err;
  };
  for (int64_t v0 = 0; v0 < d.n_views; v0 += kChunk) {
    const int n = (int)(d.n_views - v0 < kChunk ? d.n_views - v0 : kChunk);
    for (int i = 0; i < n; ++i) {
      const int64_t v = v0 + i;
      st = host_view_record(desc, v, rec[i], nullptr);
      if (st != CTP_OK) return st;
      if (!d_trig) continue;
      if (row <= kTrigStage) {
        if (staged + row > kTrigStage) {
          e = flush_trig();
          if (e != cudaSuccess) return host_cuda_error(e, "column table upload");
        }
        if (!staged) staged_v0 = v;
        for (int64_t c = 0; c < d.n_cols; ++c) {
          const double g = rec[i].gam0 + (double)c * rec[i].dgam;
          g_trig_stage[staged + 2 * c] = std::cos(g);
          g_trig_stage[staged + 2 * c + 1] = std::sin(g);
        }
        staged += row;
      } else {
        const int64_t piece = (int64_t)(kTrigStage / 2);
        for (int64_t c0 = 0; c0 < d.n_cols; c0 += piece) {
          const int64_t m = d.n_cols - c0 < piece ? d.n_cols - c0 : piece;
          for (int64_t c = 0; c < m; ++c) {
            const double g = rec[i].gam0 + (double)(c0 + c) * rec[i].dgam;
            g_trig_stage[2 * c] = std::cos(g);
            g_trig_stage[2 * c + 1] = std::sin(g);
          }
          e = cudaMemcpyAsync(d_trig + (size_t)v * row + 2 * (size_t)c0, g_trig_stage, sizeof(double) * 2 * (size_t)m,
                              cudaMemcpyHostToDevice, s);
          if (e != cudaSuccess) return host_cuda_error(e, "column table upload");
        }
      }
    }
    e = cudaMemcpyAsync(d_views + v0, rec, sizeof(ViewRec) * (size_t)n, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return host_cuda_error(e, "view record upload");
  }
  e = flush_trig();
  if (e != cudaSuccess) return host_cuda_error(e, "column table upload");

  // same launch plan as ctp_forward
  FwdLaunch f{};
  f.dims.beam = d.beam;
  f.dims.det = d.detector;
  f.dims.n_views = (int32_t)d.n_views;
  f.dims.n_rows = (int32_t)d.n_rows;
  f.dims.n_cols = (int32_t)d.n_cols;
  f.vol.n[0] = (int32_t)d.nx;
  f.vol.n[1] = (int32_t)d.ny;
  f.vol.n[2] = (int32_t)d.nz;
  for (int k = 0; k < 3; ++k) {
    f.vol.origin[k] = d.origin[k];
    f.vol.spacing[k] = d.spacing[k];
    f.vol.inv_spacing[k] = 1.0 / d.spacing[k];
    f.vol.centre[k] = 0.5 * (double)f.vol.n[k];
  }
  f.n_col_tiles = (int32_t)((d.n_cols + 31) / 32);
  f.n_row_bands = (int32_t)((d.n_rows + 7) / 8);
  f.any_transposed = n_transposed > 0;
  const bool wide = n_vox >= (int64_t)0x7fffffff;
  if (d_copy) {
    e = launch_transpose_xy(vol, d_copy, f.vol, s);
    if (e != cudaSuccess) return host_cuda_error(e, "transpose launch");
  }
  e = launch_forward(f, d_views, d_trig, vol, d_copy, sino, 1, wide, s);
  if (e != cudaSuccess) return host_cuda_error(e, "forward launch");
  return CTP_OK;
}
