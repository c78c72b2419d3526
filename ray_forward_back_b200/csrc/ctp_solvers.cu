// Iterative reconstruction on the device with the matched projector pair:
// CGLS and SIRT (diffct "Execution", section "Numerical solver API").
//
// Both keep every vector on the device and run the projections through
// ctp_forward / ctp_back on the caller's stream.  Norms are accumulated in
// FP64 by the kernels below.  The host reads back one small block of
// scalars per iteration -- the squared residual norm for the history and the
// convergence test ||y - A x|| <= atol + rtol ||y|| (initial iterate
// included), and for CGLS also the two norms the next step needs (the pages:
// "CGLS reads its two scalar norms of an iteration together").  SIRT reuses
// the residual of the previous history entry for its next update, so each
// iteration costs one forward and one back projection.
#include <cmath>
#include <cstring>

#include "ctp_internal.h"

namespace {

constexpr int kThreads = 256;
constexpr int kMaxBlocks = 148 * 8;

// device scalar slots (doubles)
enum { kGamma = 0, kDelta = 1, kGammaNew = 2, kRho = 3, kYNorm2 = 4, kSlots = 8 };

__device__ __forceinline__ double block_sum(double v) {
  __shared__ double part[kThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = v;
  __syncthreads();
  double t = 0.0;
  if (threadIdx.x < 32) {
    t = threadIdx.x < kThreads / 32 ? part[threadIdx.x] : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  }
  return t;  // valid in thread 0
}

// out += sum a_i^2
__global__ void __launch_bounds__(kThreads) norm2_kernel(const float* __restrict__ a, size_t n, double* out) {
  double acc = 0.0;
  for (size_t i = blockIdx.x * (size_t)kThreads + threadIdx.x; i < n; i += (size_t)gridDim.x * kThreads) {
    const double v = a[i];
    acc = fma(v, v, acc);
  }
  acc = block_sum(acc);
  if (threadIdx.x == 0 && acc != 0.0) atomicAdd(out, acc);
}

// r = y - q, out += sum r_i^2
__global__ void __launch_bounds__(kThreads) residual_kernel(const float* __restrict__ y, const float* __restrict__ q,
                                                            float* __restrict__ r, size_t n, double* out) {
  double acc = 0.0;
  for (size_t i = blockIdx.x * (size_t)kThreads + threadIdx.x; i < n; i += (size_t)gridDim.x * kThreads) {
    const float v = y[i] - q[i];
    r[i] = v;
    acc = fma((double)v, (double)v, acc);
  }
  acc = block_sum(acc);
  if (threadIdx.x == 0 && acc != 0.0) atomicAdd(out, acc);
}

__global__ void __launch_bounds__(kThreads) fill_kernel(float* __restrict__ a, size_t n, float v) {
  for (size_t i = blockIdx.x * (size_t)kThreads + threadIdx.x; i < n; i += (size_t)gridDim.x * kThreads) a[i] = v;
}

// a_i <- 1 / a_i where a_i > 0, else 0 (SIRT row / column weights)
__global__ void __launch_bounds__(kThreads) recip_pos_kernel(float* __restrict__ a, size_t n) {
  for (size_t i = blockIdx.x * (size_t)kThreads + threadIdx.x; i < n; i += (size_t)gridDim.x * kThreads)
    a[i] = a[i] > 0.f ? 1.f / a[i] : 0.f;
}

// t = R * r
__global__ void __launch_bounds__(kThreads) mul_kernel(const float* __restrict__ R, const float* __restrict__ r,
                                                       float* __restrict__ t, size_t n) {
  for (size_t i = blockIdx.x * (size_t)kThreads + threadIdx.x; i < n; i += (size_t)gridDim.x * kThreads)
    t[i] = R[i] * r[i];
}

// x <- x + lambda C u, clamped at 0 when asked
__global__ void __launch_bounds__(kThreads) sirt_update_kernel(float* __restrict__ x, const float* __restrict__ C,
                                                               const float* __restrict__ u, size_t n, float lambda,
                                                               int nonneg) {
  for (size_t i = blockIdx.x * (size_t)kThreads + threadIdx.x; i < n; i += (size_t)gridDim.x * kThreads) {
    float v = fmaf(lambda * C[i], u[i], x[i]);
    x[i] = nonneg ? fmaxf(v, 0.f) : v;
  }
}

// CGLS step with alpha = gamma / delta: x += alpha p (first nx entries of the
// index range), r -= alpha q (next nr entries).  alpha = 0 when delta = 0.
__global__ void __launch_bounds__(kThreads) cgls_xr_kernel(float* __restrict__ x, const float* __restrict__ p,
                                                           size_t nx, float* __restrict__ r,
                                                           const float* __restrict__ q, size_t nr,
                                                           const double* __restrict__ sc) {
  const double delta = sc[kDelta];
  const float alpha = delta > 0.0 ? (float)(sc[kGamma] / delta) : 0.f;
  for (size_t i = blockIdx.x * (size_t)kThreads + threadIdx.x; i < nx + nr; i += (size_t)gridDim.x * kThreads) {
    if (i < nx) x[i] = fmaf(alpha, p[i], x[i]);
    else r[i - nx] = fmaf(-alpha, q[i - nx], r[i - nx]);
  }
}

// p = s + beta p with beta = gamma_new / gamma
__global__ void __launch_bounds__(kThreads) cgls_p_kernel(float* __restrict__ p, const float* __restrict__ s, size_t n,
                                                          const double* __restrict__ sc) {
  const double gamma = sc[kGamma];
  const float beta = gamma > 0.0 ? (float)(sc[kGammaNew] / gamma) : 0.f;
  for (size_t i = blockIdx.x * (size_t)kThreads + threadIdx.x; i < n; i += (size_t)gridDim.x * kThreads)
    p[i] = fmaf(beta, p[i], s[i]);
}

unsigned blocks_for(size_t n) {
  const size_t b = (n + kThreads - 1) / kThreads;
  return (unsigned)(b < (size_t)kMaxBlocks ? (b ? b : 1) : (size_t)kMaxBlocks);
}

size_t align256(size_t n) { return (n + 255) & ~(size_t)255; }

struct Workspace {
  float *r = nullptr, *q = nullptr, *w = nullptr;  // sinogram-sized
  float *s = nullptr, *p = nullptr;                // volume-sized
  double* sc = nullptr;
};

size_t workspace_bytes(int64_t n_rays, int64_t n_vox, int method) {
  const size_t sino = align256(sizeof(float) * (size_t)n_rays), vol = align256(sizeof(float) * (size_t)n_vox);
  const size_t n_sino = method == CTP_SOLVER_SIRT ? 3 : 2;
  return n_sino * sino + 2 * vol + align256(sizeof(double) * kSlots);
}

Workspace carve(void* base, int64_t n_rays, int64_t n_vox, int method) {
  const size_t sino = align256(sizeof(float) * (size_t)n_rays), vol = align256(sizeof(float) * (size_t)n_vox);
  unsigned char* b = static_cast<unsigned char*>(base);
  Workspace w;
  w.r = reinterpret_cast<float*>(b);
  b += sino;
  w.q = reinterpret_cast<float*>(b);
  b += sino;
  if (method == CTP_SOLVER_SIRT) {
    w.w = reinterpret_cast<float*>(b);
    b += sino;
  }
  w.s = reinterpret_cast<float*>(b);
  b += vol;
  w.p = reinterpret_cast<float*>(b);
  b += vol;
  w.sc = reinterpret_cast<double*>(b);
  return w;
}

}  // namespace

extern "C" {

size_t ctp_solver_workspace_bytes(const ctp_geom* geom, int32_t method) {
  ctp_geom_info info;
  if (!geom || ctp_geom_query(geom, &info) != CTP_OK) return 0;
  if (method != CTP_SOLVER_CGLS && method != CTP_SOLVER_SIRT) return 0;
  return workspace_bytes(info.n_rays, info.n_vox, method);
}

ctp_status ctp_solve(const ctp_geom* geom, const float* sino, float* vol, const ctp_solver_options* opts,
                     void* workspace, size_t workspace_size, double* history, ctp_solver_result* result,
                     void* stream) {
  using namespace ctp;
  host_clear_error();
  if (!geom || !opts || !history || !result) return host_error(CTP_ERR_INVALID_ARGUMENT, "NULL argument");
  const int method = opts->method;
  if (method != CTP_SOLVER_CGLS && method != CTP_SOLVER_SIRT)
    return host_error(CTP_ERR_INVALID_ARGUMENT, "options.method is not CTP_SOLVER_CGLS or CTP_SOLVER_SIRT");
  if (opts->iterations < 0) return host_error(CTP_ERR_INVALID_ARGUMENT, "options.iterations < 0");
  if (!(opts->atol >= 0.0) || !(opts->rtol >= 0.0))
    return host_error(CTP_ERR_INVALID_ARGUMENT, "options.atol and options.rtol must be >= 0");
  if (method == CTP_SOLVER_SIRT && !std::isfinite(opts->relaxation))
    return host_error(CTP_ERR_INVALID_ARGUMENT, "options.relaxation must be finite");
  ctp_geom_info info;
  ctp_status st = ctp_geom_query(geom, &info);
  if (st != CTP_OK) return st;
  const size_t need = workspace_bytes(info.n_rays, info.n_vox, method);
  if (!workspace || workspace_size < need)
    return host_error(CTP_ERR_INVALID_ARGUMENT, "workspace missing or smaller than ctp_solver_workspace_bytes()");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0)
    return host_error(CTP_ERR_INVALID_ARGUMENT, "workspace must be 256-byte aligned");
  const size_t nr = (size_t)info.n_rays, nv = (size_t)info.n_vox;
  Workspace w = carve(workspace, info.n_rays, info.n_vox, method);
  cudaStream_t s = (cudaStream_t)stream;
  result->iterations = 0;
  result->converged = 0;
  double h[kSlots];
  cudaError_t e = cudaSuccess;
#define CTP_CHECK(expr, what)                        \
  do {                                               \
    e = (expr);                                      \
    if (e != cudaSuccess) return host_cuda_error(e, what); \
  } while (0)
#define CTP_CALL(expr)                 \
  do {                                 \
    st = (expr);                       \
    if (st != CTP_OK) return st;       \
  } while (0)
  auto read_scalars = [&]() -> cudaError_t {
    cudaError_t ee = cudaMemcpyAsync(h, w.sc, sizeof(h), cudaMemcpyDeviceToHost, s);
    if (ee == cudaSuccess) ee = cudaStreamSynchronize(s);
    return ee;
  };

  CTP_CHECK(cudaMemsetAsync(w.sc, 0, sizeof(double) * kSlots, s), "scalar reset");
  if (!opts->use_x0) CTP_CHECK(cudaMemsetAsync(vol, 0, sizeof(float) * nv, s), "initial iterate");
  // ||y||^2 and the initial residual r = y - A x0
  norm2_kernel<<<blocks_for(nr), kThreads, 0, s>>>(sino, nr, w.sc + kYNorm2);
  CTP_CALL(ctp_forward(geom, vol, w.q, stream));
  residual_kernel<<<blocks_for(nr), kThreads, 0, s>>>(sino, w.q, w.r, nr, w.sc + kRho);
  CTP_CHECK(cudaGetLastError(), "residual");
  CTP_CHECK(read_scalars(), "scalar read");
  const double ynorm = std::sqrt(h[kYNorm2]);
  const double tol = opts->atol + opts->rtol * ynorm;
  history[0] = std::sqrt(h[kRho]);
  if (history[0] <= tol) {
    result->converged = 1;
    return CTP_OK;
  }

  if (method == CTP_SOLVER_CGLS) {
    // s = A^T r, p = s, gamma = ||s||^2
    CTP_CALL(ctp_back(geom, w.r, w.s, stream));
    CTP_CHECK(cudaMemcpyAsync(w.p, w.s, sizeof(float) * nv, cudaMemcpyDeviceToDevice, s), "p = s");
    norm2_kernel<<<blocks_for(nv), kThreads, 0, s>>>(w.s, nv, w.sc + kGamma);
    CTP_CHECK(read_scalars(), "scalar read");
    double gamma = h[kGamma];
    for (int it = 1; it <= opts->iterations; ++it) {
      if (gamma == 0.0) break;
      CTP_CHECK(cudaMemsetAsync(w.sc + kDelta, 0, sizeof(double) * 3, s), "scalar reset");
      CTP_CALL(ctp_forward(geom, w.p, w.q, stream));  // q = A p
      norm2_kernel<<<blocks_for(nr), kThreads, 0, s>>>(w.q, nr, w.sc + kDelta);
      cgls_xr_kernel<<<blocks_for(nv + nr), kThreads, 0, s>>>(vol, w.p, nv, w.r, w.q, nr, w.sc);
      CTP_CALL(ctp_back(geom, w.r, w.s, stream));     // s = A^T r
      norm2_kernel<<<blocks_for(nv), kThreads, 0, s>>>(w.s, nv, w.sc + kGammaNew);
      norm2_kernel<<<blocks_for(nr), kThreads, 0, s>>>(w.r, nr, w.sc + kRho);
      CTP_CHECK(cudaGetLastError(), "CGLS kernels");
      CTP_CHECK(read_scalars(), "scalar read");       // delta, gamma_new, rho together
      if (!(h[kDelta] > 0.0)) break;                  // A p = 0: no further progress
      history[it] = std::sqrt(h[kRho]);
      result->iterations = it;
      if (history[it] <= tol) {
        result->converged = 1;
        break;
      }
      cgls_p_kernel<<<blocks_for(nv), kThreads, 0, s>>>(w.p, w.s, nv, w.sc);
      CTP_CHECK(cudaMemcpyAsync(w.sc + kGamma, w.sc + kGammaNew, sizeof(double), cudaMemcpyDeviceToDevice, s),
                "gamma update");
      gamma = h[kGammaNew];
    }
  } else {
    // weights: R = 1 / (A 1) per ray, C = 1 / (A^T 1) per voxel (0 where the sum is 0)
    float* R = w.w;
    float* C = w.s;
    float* u = w.p;
    fill_kernel<<<blocks_for(nv), kThreads, 0, s>>>(u, nv, 1.f);
    CTP_CALL(ctp_forward(geom, u, R, stream));
    recip_pos_kernel<<<blocks_for(nr), kThreads, 0, s>>>(R, nr);
    fill_kernel<<<blocks_for(nr), kThreads, 0, s>>>(w.q, nr, 1.f);
    CTP_CALL(ctp_back(geom, w.q, C, stream));
    recip_pos_kernel<<<blocks_for(nv), kThreads, 0, s>>>(C, nv);
    CTP_CHECK(cudaGetLastError(), "SIRT weights");
    for (int it = 1; it <= opts->iterations; ++it) {
      mul_kernel<<<blocks_for(nr), kThreads, 0, s>>>(R, w.r, w.q, nr);  // q = R r
      CTP_CALL(ctp_back(geom, w.q, u, stream));                        // u = A^T R r
      sirt_update_kernel<<<blocks_for(nv), kThreads, 0, s>>>(vol, C, u, nv, (float)opts->relaxation,
                                                             opts->nonnegative);
      CTP_CHECK(cudaMemsetAsync(w.sc + kRho, 0, sizeof(double), s), "scalar reset");
      CTP_CALL(ctp_forward(geom, vol, w.q, stream));                    // r = y - A x
      residual_kernel<<<blocks_for(nr), kThreads, 0, s>>>(sino, w.q, w.r, nr, w.sc + kRho);
      CTP_CHECK(cudaGetLastError(), "SIRT kernels");
      CTP_CHECK(read_scalars(), "scalar read");
      history[it] = std::sqrt(h[kRho]);
      result->iterations = it;
      if (history[it] <= tol) {
        result->converged = 1;
        break;
      }
    }
  }
#undef CTP_CHECK
#undef CTP_CALL
  return CTP_OK;
}

}  // extern "C"
