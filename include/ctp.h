/*
 * ctp — matched cell-constant Siddon projector pair for one NVIDIA B200 (sm_100a).
 *
 * Forward projection y = A x turns a voxel volume into a sinogram of ray line
 * integrals; back projection x = A^T y is its exact adjoint.  The coefficient
 * a_ij is the physical length of ray i inside voxel j: the cell-constant
 * Siddon ray-voxel intersection model in physical coordinates (diffct,
 * "Execution", section "Precision, training and reconstruction", first
 * paragraph; section "Batch dimensions and axis spacing": traversal scales
 * each world coordinate by its axis pitch and integrates in physical length
 * units).  Forward and back use the same coefficients ("matched
 * interpolation/traversal coefficients", same section), up to FP32 rounding
 * and summation order.
 *
 * Precision: per-ray clipping and entry setup in FP64, traversal and data in
 * FP32 (same page, table row backend="numba", and its paragraph on segment
 * setup from the endpoint nearer the volume centre); walks that run the
 * whole volume re-derive their FP32 parameters from the FP64 set-up every 64
 * slabs.  The forward projection is deterministic.  The ray-driven
 * adjoints (ray scatter, sort / segment-reduce) add FP32 contributions with
 * global atomics, so their last bits depend on scheduling (the pages promise
 * no bitwise determinism for scatter accumulation, same page); the gather
 * adjoint (decoupled parallel slices) sums each voxel in one thread in a
 * fixed order, and the brick adjoint, available through the plan, sums
 * exactly as 32-bit fixed point inside each block of the volume: both are
 * bitwise reproducible.
 *
 * Layouts (same page, "Batch dimensions and axis spacing"):
 *   volume    float32 [nz][ny][nx], x fastest, contiguous
 *   sinogram  float32 [n_views][n_rows][n_cols], column fastest, contiguous
 *   geometry  world coordinates (x, y, z), per-axis spacing (dx, dy, dz)
 *
 * Geometry model (the pages fix no vector convention; this is the reading):
 *   cone beam:     src[v] is the source position; each ray is the finite
 *                  segment from the source to a pixel centre.
 *   parallel beam: src[v] is the ray direction (any non-zero length); each
 *                  ray is the whole line through a pixel centre.
 *   flat detector: pixel centre p(r, c) = det_c + (c - (n_cols-1)/2) det_u
 *                                             + (r - (n_rows-1)/2) det_v
 *   cylindrical detector (cone only): the cylinder axis passes through the
 *                  source along det_v; its radius R is the distance of det_c
 *                  from that axis; |det_u| is the arc pitch; column c sits at
 *                  angle (c - (n_cols-1)/2) |det_u| / R from det_c, rows step
 *                  by det_v.  det_u must be orthogonal to det_v and to
 *                  det_c - src.
 *   volume:        voxel (i, j, k) covers [origin + (i,j,k) * spacing,
 *                  origin + (i+1,j+1,k+1) * spacing), half-open per axis.
 *
 * Calls are asynchronous: ctp_forward and ctp_back only enqueue kernels on
 * the caller's stream, never synchronise and never read device memory back
 * to the host.  Outputs are overwritten.  Input and output must not overlap.
 * A geometry handle may be used from one stream at a time (its scratch
 * buffers are shared by all calls on it); make one handle per stream for
 * concurrent use.  Errors from a kernel that already ran surface as
 * CTP_ERR_CUDA on a later call or on the caller's next synchronisation.
 */
#ifndef CTP_H
#define CTP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct ctp_geom ctp_geom; /* opaque, library-owned, immutable after create */

typedef enum {
  CTP_OK = 0,
  CTP_ERR_INVALID_ARGUMENT = 1, /* bad pointer, size, enum, non-finite vector, wrong device */
  CTP_ERR_DEGENERATE_RAY = 2,   /* a source coincides with a pixel centre, or a zero direction */
  CTP_ERR_OUT_OF_RANGE = 3,     /* distance or pitch guard violated */
  CTP_ERR_UNSUPPORTED = 4,      /* e.g. cylindrical detector with parallel beam */
  CTP_ERR_OUT_OF_MEMORY = 5,    /* device scratch could not be allocated */
  CTP_ERR_CUDA = 6              /* a CUDA runtime call failed; see ctp_last_error_detail() */
} ctp_status;

enum { CTP_BEAM_PARALLEL = 0, CTP_BEAM_CONE = 1 };
enum { CTP_DET_FLAT = 0, CTP_DET_CYLINDRICAL = 1 };

/* Adjoint variants.  AUTO picks GATHER where it applies (parallel beams
 * whose rays lie in z-planes with detector rows stepping along z: one warp
 * per (x, y) cell sums chord x slice-summed sinogram over the views and the
 * crossing columns, writing every voxel once; bitwise reproducible; MBIRJAX
 * "Projector kernels", paragraph "Forward scatters, back gathers"), its
 * grid of 4 x 4-cell blocks holds at least four blocks per SM and the volume
 * has more than 128 slices, else by
 * the collision ratio measured at create: SCATTER (one global float add per
 * ray-voxel segment, off the forward's walk) below 13.5 contributions per
 * distinct voxel of a warp batch, SORT (warp sort and segmented sum, one add
 * per distinct voxel) above.  BRICK (shared-memory fixed point per voxel
 * block) is never chosen automatically; it is bitwise reproducible on every
 * geometry.  Forcing GATHER where it does not apply fails with
 * CTP_ERR_UNSUPPORTED (ctp_last_error_detail() names the reason: another
 * beam or detector, rays leaving the z-planes, rays running along the
 * detector's columns, columns more than 64 per voxel, or a ray of a view on an
 * axis running within 1e-6 voxels of a grid line, where the slab walk's
 * rounding decides the cell). */
enum {
  CTP_ADJOINT_AUTO = 0,
  CTP_ADJOINT_BRICK = 1,
  CTP_ADJOINT_SORT = 2,
  CTP_ADJOINT_SCATTER = 3,
  CTP_ADJOINT_GATHER = 4
};

/* Optional plan overrides (all zero = library defaults). */
typedef struct {
  int32_t adjoint_variant;   /* CTP_ADJOINT_* */
  int32_t brick[3];          /* adjoint brick (bx, by, bz) in voxels; 0 = automatic */
  int32_t view_groups;       /* adjoint: split the views over this many CTA groups; 0 = automatic */
  int32_t forward_layout;    /* 0 = automatic per view, 1 = always x-fastest volume, 2 = always y-fastest */
  int32_t batch_chunk;       /* ctp_forward_batch: volumes per fused launch, 1, 2 or 4; 0 = 1.  The
                                y-fastest scratch copy (if any view uses it) grows by this factor.
                                2 or 4 also lets the brick adjoint of ctp_back_batch take member pairs
                                in one launch. */
  int32_t slice_rows;        /* parallel beams whose rays lie in z-planes and whose rows step along z:
                                detector rows that share one (x, y) path per thread, 2, 4 or 8 (one walk
                                serves that many slices); 1 = one walk per ray; 0 = automatic */
  int32_t reserved[8];
} ctp_plan;

/* Acquisition and volume description.  All pointers are HOST pointers; the
 * vectors are copied during ctp_geom_create and not referenced afterwards. */
typedef struct {
  int32_t beam;                 /* CTP_BEAM_PARALLEL | CTP_BEAM_CONE */
  int32_t detector;             /* CTP_DET_FLAT | CTP_DET_CYLINDRICAL (cone only) */
  int64_t n_views, n_rows, n_cols;
  const double *src;            /* [n_views][3] source (cone) or direction (parallel) */
  const double *det_c;          /* [n_views][3] detector centre */
  const double *det_u;          /* [n_views][3] column step (length = pitch) */
  const double *det_v;          /* [n_views][3] row step (length = pitch) */
  int64_t nx, ny, nz;           /* volume voxels */
  double origin[3];             /* world position of the min corner of voxel (0,0,0) */
  double spacing[3];            /* (dx, dy, dz), each in [1e-6, 1e6], max/min <= 1e4 */
  int32_t device;               /* CUDA device ordinal that will run the calls */
  int32_t reserved0;
  const ctp_plan *plan;         /* optional (NULL = defaults) */
} ctp_geom_desc;

/* Read-only facts about a created geometry. */
typedef struct {
  int64_t n_rays, n_vox;
  int64_t scratch_bytes;        /* device memory the handle owns */
  int32_t adjoint_variant;      /* variant ctp_back will run (BRICK, SORT, SCATTER or GATHER) */
  int32_t brick[3];
  int32_t view_groups;
  int32_t n_transposed_views;   /* views whose forward gathers from the y-fastest copy */
  double collision_ratio;       /* updates / distinct voxels per sort batch, measured at create */
  int32_t batch_chunk;          /* volumes per fused ctp_forward_batch launch */
  int32_t slice_rows;           /* detector rows per shared (x, y) walk (1 = one walk per ray) */
  int32_t interleaved_slices;   /* 1: shared walks of 4 rows run on copies interleaved by 4 slices */
  int32_t reserved;
} ctp_geom_info;

/*
 * ctp_geom_create — validate the description, copy the per-view vectors to
 * the device and allocate the handle's scratch.
 *
 * Guards (each returns an error and leaves nothing allocated), following
 * diffct "Execution": finite vectors; positive sizes; per-axis pitch in
 * [1e-6, 1e6] with largest/smallest <= 1e4 (section "Batch dimensions and axis
 * spacing"); cone beam: every view needs one ray endpoint within 1e6 voxels of
 * the volume centre and both within 1e15, distance measured as
 * |((x-cx)/dx, (y-cy)/dy, (z-cz)/dz)| (section "Precision, training and
 * reconstruction"); no source may coincide with a pixel centre (section
 * "Batch dimensions and axis spacing": finite rays are degenerate when their
 * endpoints coincide); flat detectors are checked at their corners (section
 * "Call-time trajectory validation").  Validation runs on the host before any
 * CUDA call.  *out receives the handle on success and is untouched on error.
 */
ctp_status ctp_geom_create(const ctp_geom_desc *desc, ctp_geom **out);

/* Free a handle and its device memory (synchronises the device first).  NULL is a no-op. */
void ctp_geom_destroy(ctp_geom *geom);

/* Fill *info.  Host-only, no CUDA call. */
ctp_status ctp_geom_query(const ctp_geom *geom, ctp_geom_info *info);

/*
 * ctp_forward — sino = A vol (diffct "Execution": Projector.project).
 * vol:  device pointer, float32 [nz][ny][nx], read only.
 * sino: device pointer, float32 [n_views][n_rows][n_cols], overwritten
 *       (rays that miss the volume get 0).
 * stream: a cudaStream_t (NULL = legacy default stream) on the handle's device.
 * Both pointers must be device (or managed) memory of the handle's device,
 * else CTP_ERR_INVALID_ARGUMENT.  No synchronisation.
 */
ctp_status ctp_forward(const ctp_geom *geom, const float *vol, float *sino, void *stream);

/*
 * ctp_back — vol = A^T sino, the exact transpose of ctp_forward's
 * coefficients (diffct "Execution": backward applies the matched adjoint).
 * sino: device pointer, float32 [n_views][n_rows][n_cols], read only.
 * vol:  device pointer, float32 [nz][ny][nx], overwritten.
 * Same pointer, stream and synchronisation rules as ctp_forward.  A
 * non-finite sinogram value (NaN or infinity) is not dropped: with the
 * scatter, sort and gather adjoints it reaches every voxel its ray crosses
 * (NaN, or an infinity); with the brick adjoint every voxel of each volume
 * block whose detector footprint holds it is written as NaN.
 * The gather adjoint first sums the sinogram over the rows of each column
 * that fall in one slice, into scratch the handle owns (n_views x n_cols x
 * nz rounded up to 4 floats), so calls on one handle must not overlap in
 * time (stream-order them).
 */
ctp_status ctp_back(const ctp_geom *geom, const float *sino, float *vol, void *stream);

/*
 * ctp_forward_batch / ctp_back_batch — the projections of n_batch volumes
 * (sinograms) that share one geometry, laid out one after the other:
 *   vol:  device pointer, float32 [n_batch][nz][ny][nx]
 *   sino: device pointer, float32 [n_batch][n_views][n_rows][n_cols]
 * Member b's forward output is exactly what ctp_forward gives for member b
 * alone (leading batch dimensions are preserved, diffct "Execution", section
 * "Batch dimensions and axis spacing"; empty batches included: n_batch = 0
 * does nothing and returns CTP_OK without looking at the pointers).
 * The forward walks every ray once per chunk of plan.batch_chunk members and
 * gathers from all of them, so the per-ray set-up and walk control are shared
 * across the chunk (where the geometry's slices decouple and one walk already
 * serves several detector rows, it runs member by member instead); each
 * member's sinogram is bit-identical to ctp_forward's.
 * With plan.batch_chunk >= 2 the brick adjoint takes member pairs in one
 * launch (its brick halved along y); their volumes then differ from
 * ctp_back's by fixed-point rounding only.  Otherwise, and for the scatter,
 * sort and gather adjoints, it runs member by member.  n_batch < 0, or a
 * batch whose element count exceeds 2^62, gives CTP_ERR_INVALID_ARGUMENT.
 * Same pointer, stream and synchronisation rules as ctp_forward / ctp_back.
 */
ctp_status ctp_forward_batch(const ctp_geom *geom, const float *vol, float *sino, int64_t n_batch, void *stream);
ctp_status ctp_back_batch(const ctp_geom *geom, const float *sino, float *vol, int64_t n_batch, void *stream);

/*
 * ctp_back_power — vol = (A∘A)^T sino for power 2 (every coefficient squared)
 * or A^T sino for power 1 (identical to ctp_back).  Back projection with
 * squared weights gives the diagonal of the normal operator used for
 * Hessian-diagonal preconditioning (MBIRJAX "Projector kernels", paragraph
 * "Gradient and Hessian can take different paths": back projection with the
 * weights unchanged for the gradient and squared for the Hessian diagonal).
 * Same pointer, stream and synchronisation rules as ctp_back; other powers
 * give CTP_ERR_INVALID_ARGUMENT.
 */
ctp_status ctp_back_power(const ctp_geom *geom, const float *sino, float *vol, int power, void *stream);

/*
 * ctp_geometry_gradient — gradients of a scalar loss with respect to the
 * acquisition geometry, given the loss's gradient on the sinogram:
 *   grad[v][f][k] = sum over the rays (r, c) of view v of
 *                   sino_grad[v][r][c] * d(A vol)[v][r][c] / d(vector f)_k,
 * f = 0 src, 1 det_c, 2 det_u, 3 det_v (the vectors of ctp_geom_desc; for
 * a parallel beam src is the ray direction, whose length does not matter).
 * diffct "Execution", section "Streaming analytical reconstruction": geometry
 * gradients of the projection at the cost of one extra traversal.  The line
 * integral is piecewise linear in the geometry; where a ray passes through a
 * voxel edge or an endpoint lies on a voxel face it has a kink and the result
 * is one of the one-sided derivatives.
 * vol:       device pointer, float32 [nz][ny][nx] (the forward's input), read only.
 * sino_grad: device pointer, float32 [n_views][n_rows][n_cols], read only.
 * grad:      device pointer, float64 [n_views][4][3], overwritten (zeroed,
 *            then accumulated; contents are undefined if the call fails).
 * Flat and cylindrical detectors (for the cylindrical one, the derivatives
 * of its pixel formula with respect to all four vectors, whose orthogonality
 * constraints are not imposed on the gradient).
 * Asynchronous on `stream`; summation order across blocks is not fixed, so
 * results can differ between calls in the last bits.
 */
ctp_status ctp_geometry_gradient(const ctp_geom *geom, const float *vol, const float *sino_grad, double *grad,
                                 void *stream);

/*
 * ctp_count_updates — the number of positive-length ray-voxel segments of the
 * whole acquisition (the work measure of both projectors), computed on the
 * device.  Synchronous: waits for the count and writes it to *host_out.
 */
ctp_status ctp_count_updates(const ctp_geom *geom, int64_t *host_out, void *stream);

/*
 * ctp_forward_noalloc — the forward projection sino = A vol for callers that
 * cannot allocate device memory: code running where cudaMalloc is not
 * allowed (a real-time loop with a fixed memory budget, an allocator-free
 * embedded runtime, a process whose device memory is owned by another
 * framework) and so cannot create a geometry handle either.  The pages have
 * no counterpart; this is a library convenience.
 *
 * It takes the acquisition description itself (same fields and guards as
 * ctp_geom_create) plus the caller's device buffers, and computes exactly
 * what ctp_forward computes (bit for bit), always with one walk per ray: the
 * shared slice walks of ctp_forward need scratch this call does not have.  It calls no cudaMalloc,
 * cudaFree or other allocating routine, and uses no host heap: its per-view
 * records, the cylindrical column table and the y-fastest copy of the volume
 * live in one fixed device array of CTP_NOALLOC_SCRATCH_BYTES, which every
 * GPU that loads this library holds until the process exits.  A description
 * whose records + column table + volume copy (4 bytes per voxel, needed when
 * some view's detector columns run mostly along y) exceed that size is
 * rejected with CTP_ERR_OUT_OF_RANGE and a detail message giving the sizes.
 *
 * Every call looks the array's device address up on the current device
 * (cudaGetSymbolAddress, which allocates nothing), so the address is never
 * stale, even after the caller resets the device.  The records and column
 * rows are copied with cudaMemcpyAsync from host memory of this call (a
 * stack buffer and a static staging array, not the heap), so the call may
 * wait for earlier work on `stream` before returning; for the same reason it
 * returns CTP_ERR_UNSUPPORTED, enqueuing nothing, while `stream` is being
 * captured into a graph (a replay would copy from memory the call no longer
 * owns).  All calls on a device share the one array and it keeps the last
 * call's contents: calls that overlap on the GPU (different streams, or
 * different host threads) race and corrupt each other's results; serialise
 * them on one stream (host threads are serialised inside the call, the GPU
 * work they enqueue is not).
 * vol, sino: as for ctp_forward.  The plan's forward_layout is honoured; the
 * other plan fields do not apply.
 */
#define CTP_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
ctp_status ctp_forward_noalloc(const ctp_geom_desc *desc, const float *vol, float *sino, void *stream);

/* Iterative solvers (diffct "Execution", section "Numerical solver API"). */
enum { CTP_SOLVER_CGLS = 1, CTP_SOLVER_SIRT = 2 };

typedef struct {
  int32_t method;       /* CTP_SOLVER_CGLS | CTP_SOLVER_SIRT */
  int32_t iterations;   /* run at most this many iterations */
  double atol, rtol;    /* stop when ||y - A x|| <= atol + rtol ||y||, the initial iterate included */
  double relaxation;    /* SIRT step factor lambda (1 = plain SIRT); ignored by CGLS */
  int32_t nonnegative;  /* SIRT: clamp x >= 0 after every step; ignored by CGLS */
  int32_t use_x0;       /* 1: vol holds the initial iterate; 0: start from zero */
} ctp_solver_options;

typedef struct {
  int32_t iterations;   /* completed iterations (history holds iterations + 1 entries) */
  int32_t converged;    /* 1 if the tolerance was met (possibly by the initial iterate) */
} ctp_solver_result;

/* Device workspace ctp_solve needs for this geometry and method, in bytes
 * (0 for a NULL geometry or an unknown method). */
size_t ctp_solver_workspace_bytes(const ctp_geom *geom, int32_t method);

/*
 * ctp_solve — least-squares reconstruction of vol from sino with the matched
 * pair, following diffct "Execution", section "Numerical solver API":
 *   CGLS: conjugate gradients on the normal equations (least-squares form);
 *   SIRT: x <- x + lambda C A^T R (y - A x), R and C the reciprocal row and
 *         column sums of A (0 where a sum is 0), optionally clamped at 0; the
 *         residual of each history entry is reused for the next update.
 * history (HOST, at least iterations + 1 doubles) receives ||y - A x|| of the
 * initial iterate and of every completed iteration; *result the count and
 * whether the tolerance was met.  workspace: DEVICE memory of at least
 * ctp_solver_workspace_bytes(geom, method), 256-byte aligned, owned by the
 * caller and overwritten.  sino, vol: device pointers as for ctp_forward;
 * vol is overwritten with the final iterate.
 * Synchronous: every iteration reads one block of norms back to the host
 * (the residual norm, and for CGLS the two norms of its step), so the call
 * returns when the solve is finished.
 */
ctp_status ctp_solve(const ctp_geom *geom, const float *sino, float *vol, const ctp_solver_options *opts,
                     void *workspace, size_t workspace_bytes, double *history, ctp_solver_result *result,
                     void *stream);

/*
 * ctp_debug_error_word — the bounds-check record of a CTP_DEBUG build of this
 * library (built with -DCTP_DEBUG; a test and diagnosis build, not the
 * default).  In that build every global and shared-memory index of the
 * projector kernels is checked against its array's extent before the
 * access; a failing index is recorded (site number in the top 16 bits, the
 * index in the low 48) and the access skipped, and the next ctp_forward /
 * ctp_back / ctp_back_power / ctp_forward_batch / ctp_geometry_gradient call
 * returns CTP_ERR_OUT_OF_RANGE.  This call waits for the device, stores the
 * record (0 if every index was in bounds) in *word and clears it.
 * Other builds: *word = 0 and CTP_ERR_UNSUPPORTED.  The pages have no
 * counterpart; this is the library's memory-safety check.
 */
ctp_status ctp_debug_error_word(uint64_t *word);

/* Static description of a status code. */
const char *ctp_status_string(ctp_status status);

/* Detail message of the last failing call on this host thread ("" if none). */
const char *ctp_last_error_detail(void);

/* Library version, "major.minor.patch". */
const char *ctp_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CTP_H */
