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
//                      One walk can serve 1, 2 or 4 volumes of a batch.
//   back_brick_kernel  one CTA owns a voxel brick in shared memory, visits every
//                      ray of its view range that can cross the brick (exact
//                      detector footprint of the brick per view), clips each
//                      ray to the brick in FP64 (the per-tile entry of the
//                      pages), walks it in FP32 with int32 fixed-point
//                      shared-memory atomics, and flushes the brick once per
//                      stage with coalesced stores (plain stores when the CTA
//                      owns all views, red.global.add otherwise).  Parallel
//                      beams take each window of 2048 rays in order of
//                      estimated chord length, so a warp's lanes finish
//                      together; one instance per beam type.
//   back_sort_kernel   the adjoint as a sorted segment reduction, for dense
//                      ray-voxel collisions (and, counting, the collision ratio).
//   count_kernel       the forward traversal counting positive-length segments.
//   transpose_xy       x-fastest -> y-fastest copy of the volume.
#include <map>
#include <mutex>
#include <utility>

#include "ctp_ray.cuh"

namespace ctp {
namespace {

// Tuning knobs (compile-time; the defaults are the measured choices).
#ifndef CTP_FWD_MIN_BLOCKS
#define CTP_FWD_MIN_BLOCKS 5
#endif
#ifndef CTP_SCATTER_MIN_BLOCKS
#define CTP_SCATTER_MIN_BLOCKS 5
#endif
#ifndef CTP_BACK_MIN_BLOCKS
#define CTP_BACK_MIN_BLOCKS 3
#endif
#ifndef CTP_WALK2_UNROLL
#define CTP_WALK2_UNROLL 4
#endif
#ifndef CTP_WALK3_UNROLL
#define CTP_WALK3_UNROLL 2
#endif
#ifndef CTP_LANE_WALK2_UNROLL
#define CTP_LANE_WALK2_UNROLL 8
#endif
constexpr int kWalk2Unroll = CTP_WALK2_UNROLL;
constexpr int kLaneWalk2Unroll = CTP_LANE_WALK2_UNROLL;
constexpr int kWalk3Unroll = CTP_WALK3_UNROLL;

constexpr int kFwdCols = 32;  // threads along detector columns per block
constexpr int kFwdRows = 8;   // detector rows per block (row band height)
static_assert(kFwdCols == kSliceCols && kFwdRows == kSliceWarps, "shared slice walks use the forward's block");
constexpr int kBackThreads = 256;
#ifndef CTP_BACK_STAGE
#define CTP_BACK_STAGE 64
#endif
constexpr int kBackStage = CTP_BACK_STAGE;  // views per fixed-point accumulation stage of the adjoint
constexpr int kSortWin = 2048;     // parallel adjoint: rays per length-sorted window
constexpr int kSortBuckets = 32;   // chord-length classes of the counting sort
constexpr float kRoundBias = 12582912.0f;   // 1.5 * 2^23
constexpr int kRoundBiasBits = 0x4B400000;  // its bit pattern

// FP32 Siddon walk in major-axis slabs, one lane per ray (lanes run
// independently).  Each slab between two successive planes of the major axis
// a holds at most one crossing of each minor axis, so it is one, two or three
// segments.  The walk is branch-free: every slab makes the same visit calls,
// a segment that does not exist in that slab being visited with length 0 at
// a valid offset.  visit(offset, physical length) is called for every segment
// (zero-length ones included);
// offsets move by the signed strides s0, s1, s2 of axes x, y, z.  Crossings
// are l0 + j * inc from exact integers j and the FP64 counts N cap every
// axis, so offsets never leave the clipped box; a minor crossing that rounds
// past the exit is dropped (its error is below one ulp of the walk length).
template <typename Off, typename Visit>
__device__ __forceinline__ void walk_lane(const Walk& W, Off off, Off s0, Off s1, Off s2, Visit&& visit) {
  int a, b, c;
  walk_axes(W, a, b, c);
  const int Na = pick3(a, W.N[0], W.N[1], W.N[2]);
  const int Nb = pick3(b, W.N[0], W.N[1], W.N[2]);
  const int Nc = pick3(c, W.N[0], W.N[1], W.N[2]);
  const float l0a = pick3(a, W.l0[0], W.l0[1], W.l0[2]), inca = pick3(a, W.inc[0], W.inc[1], W.inc[2]);
  const float l0b = pick3(b, W.l0[0], W.l0[1], W.l0[2]), incb = pick3(b, W.inc[0], W.inc[1], W.inc[2]);
  const float l0c = pick3(c, W.l0[0], W.l0[1], W.l0[2]), incc = pick3(c, W.inc[0], W.inc[1], W.inc[2]);
  const Off sa = pick3(a, s0, s1, s2), sb = pick3(b, s0, s1, s2), sc = pick3(c, s0, s1, s2);
  const float L = W.L;
  const float fNb = (float)Nb, fNc = (float)Nc;
  float tb = Nb > 0 ? l0b : CUDART_INF_F;
  float fjb = 1.f;
  float cur = 0.f;
  if (Nc == 0) {
    float fs = 0.f;  // s as a float, counted rather than converted each slab
#pragma unroll kLaneWalk2Unroll
    for (int s = 0; s < Na; ++s, fs += 1.f) {
      const float tx = fminf(fmaf(fs, inca, l0a), L);
      const bool cb = tb < tx;
      const float m1 = fmaxf(fminf(tb, tx), cur);
      const Off o2 = off + (cb ? sb : (Off)0);
      visit(off, m1 - cur);
      visit(o2, tx - m1);
      off = o2 + sa;
      tb = cb ? (fjb < fNb ? fmaf(fjb, incb, l0b) : CUDART_INF_F) : tb;
      fjb += cb ? 1.f : 0.f;
      cur = tx;
    }
    const bool cb = tb < L;
    const float m1 = fmaxf(fminf(tb, L), cur);
    visit(off, m1 - cur);
    visit(off + (cb ? sb : (Off)0), L - m1);
  } else {
    float tc = l0c;
    float fjc = 1.f;
    float fs = 0.f;
#pragma unroll kWalk3Unroll
    for (int s = 0; s <= Na; ++s, fs += 1.f) {
      const float tx = s < Na ? fminf(fmaf(fs, inca, l0a), L) : L;
      const bool cb = tb < tx, cc = tc < tx;
      const float m1 = fmaxf(fminf(fminf(tb, tc), tx), cur);
      const float m2 = fmaxf(fminf(fmaxf(tb, tc), tx), m1);
      const Off db = cb ? sb : (Off)0, dc = cc ? sc : (Off)0;
      const Off o2 = off + (tb <= tc ? db : dc);
      const Off o3 = off + db + dc;
      visit(off, m1 - cur);
      visit(o2, m2 - m1);
      visit(o3, tx - m2);
      tb = cb ? (fjb < fNb ? fmaf(fjb, incb, l0b) : CUDART_INF_F) : tb;
      fjb += cb ? 1.f : 0.f;
      tc = cc ? (fjc < fNc ? fmaf(fjc, incc, l0c) : CUDART_INF_F) : tc;
      fjc += cc ? 1.f : 0.f;
      off = o3 + sa;
      cur = tx;
    }
  }
}

// Branch-free FP32 Siddon walk in major-axis slabs with a warp-uniform trip
// count: every lane steps slab s = 0, 1, ... up to the warp's longest walk
// and lanes past their own last slab are predicated off, so the loop needs
// no reconvergence and unrolls cleanly.  Every slab makes the same visit
// calls (a segment absent from that slab is visited with length 0 at a valid
// offset).  The last slab of a ray ends at its exit: the (Na+1)-th major
// crossing lies at or past it, so clamping to L closes the walk (to within
// rounding of the walk length).  All 32 lanes must call this; lanes without
// a ray pass active = false.  Offsets as in walk_lane.
template <typename Off, typename Visit>
__device__ __forceinline__ void walk_warp_bf(bool active, const Walk& W, Off off, Off s0, Off s1, Off s2,
                                             Visit&& visit) {
  constexpr unsigned kFull = 0xffffffffu;
  int a, b, c;
  walk_axes(W, a, b, c);
  const int Na = active ? pick3(a, W.N[0], W.N[1], W.N[2]) : -1;
  const int Nb = pick3(b, W.N[0], W.N[1], W.N[2]);
  const int Nc = pick3(c, W.N[0], W.N[1], W.N[2]);
  const float l0a = pick3(a, W.l0[0], W.l0[1], W.l0[2]), inca = pick3(a, W.inc[0], W.inc[1], W.inc[2]);
  const float l0b = pick3(b, W.l0[0], W.l0[1], W.l0[2]), incb = pick3(b, W.inc[0], W.inc[1], W.inc[2]);
  const float l0c = pick3(c, W.l0[0], W.l0[1], W.l0[2]), incc = pick3(c, W.inc[0], W.inc[1], W.inc[2]);
  const Off sa = pick3(a, s0, s1, s2), sb = pick3(b, s0, s1, s2), sc = pick3(c, s0, s1, s2);
  const float L = W.L;
  const float fNb = (float)Nb, fNc = (float)Nc;
  const int kmax = __reduce_max_sync(kFull, Na);
  if (kmax < 0) return;
  float tb = Nb > 0 ? l0b : CUDART_INF_F;
  float fjb = 1.f, cur = 0.f;
  float fs = 0.f;  // s as a float, counted rather than converted each slab
  if (!__any_sync(kFull, active && Nc > 0)) {
#pragma unroll kLaneWalk2Unroll
    for (int s = 0; s <= kmax; ++s, fs += 1.f) {
      const bool on = s <= Na;
      const float tx = fminf(fmaf(fs, inca, l0a), L);
      const bool cb = tb < tx;
      const float m1 = fmaxf(fminf(tb, tx), cur);
      const Off o2 = off + (cb ? sb : (Off)0);
      if (on) {
        visit(off, m1 - cur);
        visit(o2, tx - m1);
        off = o2 + sa;
        tb = cb ? (fjb < fNb ? fmaf(fjb, incb, l0b) : CUDART_INF_F) : tb;
        fjb += cb ? 1.f : 0.f;
        cur = tx;
      }
    }
  } else {
    float tc = Nc > 0 ? l0c : CUDART_INF_F;
    float fjc = 1.f;
#pragma unroll kWalk3Unroll
    for (int s = 0; s <= kmax; ++s, fs += 1.f) {
      const bool on = s <= Na;
      const float tx = fminf(fmaf(fs, inca, l0a), L);
      const bool cb = tb < tx, cc = tc < tx;
      const float m1 = fmaxf(fminf(fminf(tb, tc), tx), cur);
      const float m2 = fmaxf(fminf(fmaxf(tb, tc), tx), m1);
      const Off db = cb ? sb : (Off)0, dc = cc ? sc : (Off)0;
      const Off o2 = off + (tb <= tc ? db : dc);
      const Off o3 = off + db + dc;
      if (on) {
        visit(off, m1 - cur);
        visit(o2, m2 - m1);
        visit(o3, tx - m2);
        off = o3 + sa;
        tb = cb ? (fjb < fNb ? fmaf(fjb, incb, l0b) : CUDART_INF_F) : tb;
        fjb += cb ? 1.f : 0.f;
        tc = cc ? (fjc < fNc ? fmaf(fjc, incc, l0c) : CUDART_INF_F) : tc;
        fjc += cc ? 1.f : 0.f;
        cur = tx;
      }
    }
  }
}

// FP32 Siddon walk in major-axis slabs, warp-synchronous.
//
// The major axis a is the one the ray crosses most often (smallest spacing
// between crossings), so each slab between two successive a-planes holds at
// most one crossing of each minor axis b, c: a slab is one, two or three
// segments, visited in order with predicated (not branched) extra segments.
// Lanes are aligned on absolute slab positions inside the box: a lane whose
// ray enters the box further along the major axis waits that many steps, so
// at every step all lanes of the warp (neighbouring rays) sit in the same
// slab and touch neighbouring voxels.  visit(offset, physical length) is
// called for every segment (zero-length ones included); offsets move by the
// signed strides s0, s1, s2 of axes x, y, z.  Crossings are l0 + j * inc from
// exact integers j, and the FP64 counts N cap every axis, so offsets never
// leave the clipped box; a minor crossing that rounds past the exit is
// dropped (its error is below one ulp of the walk length).
//
// Positions are measured from a local origin.  Without re-anchoring
// (kAnchor = 0) that origin is the entry, and a crossing far along the ray
// carries an FP32 error of about one ulp of its distance from the entry: a
// few 1e-5 of a voxel after a few hundred voxels.  That is harmless where
// segment errors telescope (a forward sum over one ray) but not where a
// voxel sums a few short segments of different rays (the adjoint).  With
// kAnchor = K, every K slabs each lane moves its origin to the start of its
// current slab and recomputes its local FP32 parameters there in FP64, from
// the entry's FP64 values at anc[q * kAncStride] (q = 0-2: l0 per axis,
// 3-5: inc per axis, 6: length), so positions never grow beyond K slabs.
//
// All 32 lanes must call this together; lanes without a ray pass active = false.
// With kUniform, every lane calls visit(offset, length, flag) at every segment
// slot, flag telling whether the segment exists for that lane (so the visitor
// may use warp collectives); a slot that no lane of the warp has is skipped.
// Without it, visit(offset, length, true) is called for existing segments only.
constexpr int kAncStride = kFwdCols * kFwdRows;  // one FP64 record per thread of the block, field-major
#ifndef CTP_WALK_ANCHOR
#define CTP_WALK_ANCHOR 64
#endif
constexpr int kWalkAnchor = CTP_WALK_ANCHOR;  // slabs between re-anchorings of the whole-volume adjoint walks

template <bool kAlign, bool kUniform, int kAnchor, typename Off, typename Visit>
__device__ __forceinline__ void walk(bool active, const Walk& W, const int lo[3], const int hi[3], Off off, Off s0,
                                     Off s1, Off s2, const double* __restrict__ anc, Visit&& visit) {
  static_assert(kAnchor == 0 || (kAnchor & (kAnchor - 1)) == 0, "re-anchoring period is a power of two");
  constexpr unsigned kFull = 0xffffffffu;
  const float i0 = W.inc[0], i1 = W.inc[1], i2 = W.inc[2];
  int a, b, c;
  walk_axes(W, a, b, c);
  // Rayless lanes get Na = 0 and, below, an unreachable slab window, so the
  // window test is one unsigned compare.
  const int Na = active ? pick3(a, W.N[0], W.N[1], W.N[2]) : 0;
  const int Nb = pick3(b, W.N[0], W.N[1], W.N[2]);
  const int Nc = pick3(c, W.N[0], W.N[1], W.N[2]);
  float l0a = pick3(a, W.l0[0], W.l0[1], W.l0[2]);
  float l0b = pick3(b, W.l0[0], W.l0[1], W.l0[2]);
  float l0c = pick3(c, W.l0[0], W.l0[1], W.l0[2]);
  const float inca = pick3(a, i0, i1, i2), incb = pick3(b, i0, i1, i2), incc = pick3(c, i0, i1, i2);
  const Off sa = pick3(a, s0, s1, s2), sb = pick3(b, s0, s1, s2), sc = pick3(c, s0, s1, s2);

  // slab alignment: entry position along the major axis in travel direction
  const int ia = pick3(a, W.i[0], W.i[1], W.i[2]);
  const int p = pick3(a, W.step[0], W.step[1], W.step[2]) > 0 ? ia - pick3(a, lo[0], lo[1], lo[2])
                                                               : pick3(a, hi[0], hi[1], hi[2]) - 1 - ia;
  const int span_plain = __reduce_max_sync(kFull, active ? Na : -1);
  if (span_plain < 0) return;  // no lane has a ray
  int d = 0, kmax = span_plain;
  if (kAlign) {
    const int pmin = __reduce_min_sync(kFull, active ? p : 0x7fffffff);
    d = active ? p - pmin : 0;
    const int span_aligned = __reduce_max_sync(kFull, active ? d + Na : -1);
    // alignment only pays while it does not stretch the warp's loop much
    if (span_aligned <= 2 * span_plain + 8) kmax = span_aligned;
    else d = 0;
  }
  if (!active) d = 1 << 30;  // s = k - d stays negative: never inside [0, Na]
  // s = k - d as a float, counted rather than converted each slab (exact for
  // the active lanes, whose |s| stays far below 2^24)
  float fs = -(float)d;

  float L = W.L;
  float fNb = (float)Nb, fNc = (float)Nc;
  float tb = Nb > 0 ? l0b : CUDART_INF_F;
  float tc = Nc > 0 ? l0c : CUDART_INF_F;
  float fjb = 1.f, fjc = 1.f;
  float jb0 = 0.f, jc0 = 0.f;  // entry-frame index of crossing 0 of the current frame (b, c)
  float cur = 0.f;
  // Move the local origin to the start of slab s >= 1 (major crossing s - 1).
  auto reanchor = [&](int s) {
    const double la = anc[a * kAncStride], ja = anc[(3 + a) * kAncStride];
    const double O = fma((double)(s - 1), ja, la);
    l0a = (float)(fma((double)s, ja, la) - O);
    L = (float)(anc[6 * kAncStride] - O);
    cur = 0.f;
    fs = 0.f;
    if (tb < CUDART_INF_F) {  // the pending b crossing has entry-frame index jb0 + fjb - 1
      const float db = fjb - 1.f;
      jb0 += db;
      fNb -= db;
      fjb = 1.f;
      l0b = (float)(fma((double)jb0, anc[(3 + b) * kAncStride], anc[b * kAncStride]) - O);
      tb = l0b;
    }
    if (tc < CUDART_INF_F) {
      const float dc = fjc - 1.f;
      jc0 += dc;
      fNc -= dc;
      fjc = 1.f;
      l0c = (float)(fma((double)jc0, anc[(3 + c) * kAncStride], anc[c * kAncStride]) - O);
      tc = l0c;
    }
  };
  // One slab of the two-segment walk (no lane crosses axis c).
  auto slab2 = [&](int k) {
    const int s = k - d;
    const bool on = (unsigned)s <= (unsigned)Na;
    // the (Na+1)-th major crossing lies at or past the exit: clamping to L
    // ends the last slab there (to within rounding of the walk length)
    const float tx = fminf(fmaf(fs, inca, l0a), L);
    const bool cb = on && tb < tx;
    const float m1 = fmaxf(fminf(tb, tx), cur);
    if (kUniform) {
      visit(off, m1 - cur, on);
      if (__any_sync(kFull, cb)) visit(off + sb, tx - m1, cb);
    } else {
      if (on) visit(off, m1 - cur, true);
      if (cb) visit(off + sb, tx - m1, true);
    }
    if (on) {
      off += (cb ? sb : (Off)0) + sa;
      cur = tx;
    }
    if (cb) {
      tb = fjb < fNb ? fmaf(fjb, incb, l0b) : CUDART_INF_F;
      fjb += 1.f;
    }
  };
  // One slab of the three-segment walk.
  auto slab3 = [&](int k) {
    const int s = k - d;
    const bool on = (unsigned)s <= (unsigned)Na;
    const float tx = fminf(fmaf(fs, inca, l0a), L);
    const bool cb = on && tb < tx, cc = on && tc < tx;
    if (!kUniform && !__any_sync(kFull, cc)) {
      // No lane crosses axis c in this slab (the common case: c is the axis
      // crossed least often, and the aligned lanes of a warp cross it at
      // nearly the same slab): the slab is one or two segments.
      const float m1 = fmaxf(fminf(tb, tx), cur);
      if (on) visit(off, m1 - cur, true);
      if (cb) visit(off + sb, tx - m1, true);
      if (on) {
        off += (cb ? sb : (Off)0) + sa;
        cur = tx;
      }
      if (cb) {
        tb = fjb < fNb ? fmaf(fjb, incb, l0b) : CUDART_INF_F;
        fjb += 1.f;
      }
      return;
    }
    const float m1 = fmaxf(fminf(fminf(tb, tc), tx), cur);
    const float m2 = fmaxf(fminf(fmaxf(tb, tc), tx), m1);
    const Off db = cb ? sb : (Off)0, dc = cc ? sc : (Off)0;
    const Off o2 = off + (tb <= tc ? db : dc);
    const Off o3 = off + db + dc;
    if (kUniform) {
      visit(off, m1 - cur, on);
      if (__any_sync(kFull, cb || cc)) visit(o2, m2 - m1, cb || cc);
      if (__any_sync(kFull, cb && cc)) visit(o3, tx - m2, cb && cc);
    } else {
      if (on) visit(off, m1 - cur, true);
      if (cb || cc) visit(o2, m2 - m1, true);
      if (cb && cc) visit(o3, tx - m2, true);
    }
    if (on) {
      off = o3 + sa;
      cur = tx;
    }
    if (cb) {
      tb = fjb < fNb ? fmaf(fjb, incb, l0b) : CUDART_INF_F;
      fjb += 1.f;
    }
    if (cc) {
      tc = fjc < fNc ? fmaf(fjc, incc, l0c) : CUDART_INF_F;
      fjc += 1.f;
    }
  };
  const bool three = __any_sync(kFull, active && Nc > 0);
  if (kAnchor == 0) {
    if (!three) {
#pragma unroll kWalk2Unroll
      for (int k = 0; k <= kmax; ++k, fs += 1.f) slab2(k);
    } else {
#pragma unroll kWalk3Unroll
      for (int k = 0; k <= kmax; ++k, fs += 1.f) slab3(k);
    }
  } else {
    // blocks of kAnchor slabs; every lane already inside its walk re-anchors
    // at the start of each block after the first
    for (int k0 = 0; k0 <= kmax; k0 += kAnchor) {
      if (k0 > 0) {
        const int s = k0 - d;
        if ((unsigned)s <= (unsigned)Na && s > 0) reanchor(s);
      }
      const int kend = min(k0 + kAnchor, kmax + 1);
      if (!three) {
#pragma unroll kWalk2Unroll
        for (int k = k0; k < kend; ++k, fs += 1.f) slab2(k);
      } else {
#pragma unroll kWalk3Unroll
        for (int k = k0; k < kend; ++k, fs += 1.f) slab3(k);
      }
    }
  }
}

// ------------------------------------------------------------------ forward --

// kB volumes per launch (a chunk of a batch sharing the geometry): each ray is
// walked once and every segment gathers from all kB volumes, so the FP64
// set-up and the walk control are shared; kB = 1 is the plain forward.
template <typename Off, int kB>
__global__ void __launch_bounds__(kFwdCols* kFwdRows, kB == 1 ? CTP_FWD_MIN_BLOCKS : 4)
    forward_kernel(FwdLaunch P, const ViewRec* __restrict__ views, const double* __restrict__ trig,
                   const float* __restrict__ vol, const float* __restrict__ volT, float* __restrict__ sino) {
  const int per_band = P.dims.n_views * P.n_col_tiles;
  const int band = blockIdx.x / per_band;
  const int rem = blockIdx.x - band * per_band;
  const int v = rem / P.n_col_tiles;
  const int ct = rem - v * P.n_col_tiles;
  const int c = ct * kFwdCols + threadIdx.x;
  const int r = band * kFwdRows + threadIdx.y;
  const bool valid = c < P.dims.n_cols && r < P.dims.n_rows;

  const ViewRec& V = views[v];
  Ray R;
  make_ray(V, P.vol, trig, P.dims, v, valid ? r : 0, valid ? c : 0, R);
  const int lo[3] = {0, 0, 0};
  const int hi[3] = {P.vol.n[0], P.vol.n[1], P.vol.n[2]};
  setup_t t_in = 0, t_out = 0;
  const bool hit = valid && clip(R, lo, hi, t_in, t_out);
  Walk W = {};
  if (hit) entry(R, t_in, t_out, lo, hi, W);
  const Off nx = P.vol.n[0], ny = P.vol.n[1];
  const bool yfast = V.layout != 0;
  const float* __restrict__ base = yfast ? volT : vol;
  const Off sx = yfast ? ny : (Off)1;
  const Off sy = yfast ? (Off)1 : nx;
  const Off sz = nx * ny;
  const Off off = (Off)W.i[2] * sz + (Off)W.i[1] * sy + (Off)W.i[0] * sx;
  const size_t n_vox = (size_t)P.vol.n[0] * (size_t)P.vol.n[1] * (size_t)P.vol.n[2];
  float acc[kB];
#pragma unroll
  for (int j = 0; j < kB; ++j) acc[j] = 0.f;
  walk<true, false, 0, Off>(hit, W, lo, hi, off, W.step[0] * sx, W.step[1] * sy, W.step[2] * sz, nullptr,
                         [&](Off o, float len, bool) {
                           if (CTP_IN_BOUNDS(o, n_vox, 1)) {
#pragma unroll
                             for (int j = 0; j < kB; ++j) acc[j] = fmaf(len, __ldg(base + j * n_vox + o), acc[j]);
                           }
                         });
  if (valid) {
    const size_t n_rays = (size_t)P.dims.n_views * P.dims.n_rows * P.dims.n_cols;
    const size_t i = ((size_t)v * P.dims.n_rows + r) * P.dims.n_cols + c;
    if (CTP_IN_BOUNDS(i, n_rays, 2)) {
#pragma unroll
      for (int j = 0; j < kB; ++j) sino[j * n_rays + i] = acc[j];
    }
  }
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
  const bool valid = c < P.dims.n_cols && r < P.dims.n_rows;
  unsigned long long n = 0;
  Ray R;
  make_ray(views[v], P.vol, trig, P.dims, v, valid ? r : 0, valid ? c : 0, R);
  const int lo[3] = {0, 0, 0};
  const int hi[3] = {P.vol.n[0], P.vol.n[1], P.vol.n[2]};
  setup_t t_in = 0, t_out = 0;
  const bool hit = valid && clip(R, lo, hi, t_in, t_out);
  Walk W = {};
  if (hit) entry(R, t_in, t_out, lo, hi, W);
  walk<false, false, 0, int>(hit, W, lo, hi, 0, 0, 0, 0, nullptr, [&](int, float len, bool) { n += len > 0.f ? 1ull : 0ull; });
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

// Adjoint coefficient of a segment of physical length len: len (the
// transpose of the forward projection) or len^2 (squared weights, the
// diagonal of the normal operator used for Hessian preconditioning).
template <int kPower>
__device__ __forceinline__ float coef(float len) {
  return kPower == 2 ? len * len : len;
}

// Column of the t-th ray of a footprint row of width w taken from both ends
// inwards (0, w-1, 1, w-2, ...).  With parallel rays a brick's chord profile
// along a footprint row is a trapezoid symmetric about the row centre, so
// consecutive rays in this order come in pairs of equal chords.  (The length
// sort of the parallel adjoint then groups rays across views; cone
// footprints are not symmetric and keep plain order.)
__device__ __forceinline__ int mirror_order(int t, int w) { return (t & 1) ? w - 1 - (t >> 1) : (t >> 1); }

// Detector footprint of the brick [lo, hi) in view V: a rectangle of pixels
// that contains every pixel whose ray can meet the brick.  Also returns
// nvox, an upper bound on the number of this view's rays that can meet any
// single voxel of the brick (lattice points inside the bounding rectangle of
// one voxel's projection, plus slack), used to size the fixed-point scale.
// Computed by one warp (lanes 0-7 project the eight corners); all lanes
// return the result.
__device__ void brick_footprint(const ViewRec& V, const BackLaunch& P, const int lo[3], const int hi[3], int lane,
                                int& c0, int& c1, int& r0, int& r1, int& nvox, float ucol[4]) {
  const int nc = P.dims.n_cols, nr = P.dims.n_rows;
  if (V.full_footprint) {
    c0 = 0, c1 = nc - 1, r0 = 0, r1 = nr - 1;
    nvox = nc * nr;
    return;
  }
  const int q = lane & 7;
  double X[3];
  const int cv[3] = {(q & 1) ? hi[0] : lo[0], (q & 2) ? hi[1] : lo[1], (q & 4) ? hi[2] : lo[2]};
#pragma unroll
  for (int k = 0; k < 3; ++k) X[k] = P.vol.origin[k] + (double)cv[k] * P.vol.spacing[k];
  double cmin, cmax, rmin, rmax, lam_min = 0.0;
  int bad = 0;
  // cylindrical only: distance of the brick from the source's axis
  double rho_lo = 0.0, rho_hi = 0.0;
  if (P.dims.beam == CTP_BEAM_PARALLEL) {
    const double d[3] = {X[0] - V.p00[0], X[1] - V.p00[1], X[2] - V.p00[2]};
    cmin = cmax = V.minv[0] * d[0] + V.minv[1] * d[1] + V.minv[2] * d[2];
    rmin = rmax = V.minv[3] * d[0] + V.minv[4] * d[1] + V.minv[5] * d[2];
    // sort the eight corner columns across the lanes of each group of 8
    // (bitonic); a brick whose chord depends on the column alone (rays and
    // columns in z-planes) has the chord profile of a trapezoid with corners
    // at sorted positions 0, 2, 5, 7 (each column appears twice)
    float u = (float)cmin;
#pragma unroll
    for (int k = 2; k <= 8; k <<= 1) {
#pragma unroll
      for (int j = k >> 1; j > 0; j >>= 1) {
        const float o = __shfl_xor_sync(0xffffffffu, u, j);
        const bool up = (q & k) == 0, low = (q & j) == 0;
        u = (low == up) ? fminf(u, o) : fmaxf(u, o);
      }
    }
    const int g0 = lane & ~7;
    ucol[0] = __shfl_sync(0xffffffffu, u, g0);
    ucol[1] = __shfl_sync(0xffffffffu, u, g0 + 2);
    ucol[2] = __shfl_sync(0xffffffffu, u, g0 + 5);
    ucol[3] = __shfl_sync(0xffffffffu, u, g0 + 7);
  } else if (P.dims.det == CTP_DET_FLAT) {
    const double d[3] = {X[0] - V.s[0], X[1] - V.s[1], X[2] - V.s[2]};
    const double lam = V.minv[0] * d[0] + V.minv[1] * d[1] + V.minv[2] * d[2];
    const double lc = V.minv[3] * d[0] + V.minv[4] * d[1] + V.minv[5] * d[2];
    const double lr = V.minv[6] * d[0] + V.minv[7] * d[1] + V.minv[8] * d[2];
    lam_min = lam;
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
    rho_lo = rho_c - hd;
    rho_hi = rho_c + hd;
    if (!(rho_lo > 1e-9)) bad = 1;
  }
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) {
    cmin = fmin(cmin, __shfl_xor_sync(0xffffffffu, cmin, o));
    cmax = fmax(cmax, __shfl_xor_sync(0xffffffffu, cmax, o));
    rmin = fmin(rmin, __shfl_xor_sync(0xffffffffu, rmin, o));
    rmax = fmax(rmax, __shfl_xor_sync(0xffffffffu, rmax, o));
    lam_min = fmin(lam_min, __shfl_xor_sync(0xffffffffu, lam_min, o));
    bad |= __shfl_xor_sync(0xffffffffu, bad, o);
  }
  if (bad) {
    c0 = 0, c1 = nc - 1, r0 = 0, r1 = nr - 1;
    nvox = nc * nr;
    return;
  }
  // extent (in pixels) of one voxel's projection: wc columns by wr rows
  double wc, wr;
  const double D = sqrt(P.vol.spacing[0] * P.vol.spacing[0] + P.vol.spacing[1] * P.vol.spacing[1] +
                        P.vol.spacing[2] * P.vol.spacing[2]);
  if (P.dims.beam == CTP_BEAM_PARALLEL) {
    wc = V.vox_ext[0];
    wr = V.vox_ext[1];
  } else if (P.dims.det == CTP_DET_FLAT) {
    // c = lc / lam over a voxel varies by at most (A_c + |c|max A_lam) / lam_min
    const double cm = fmax(fabs(cmin), fabs(cmax)), rm = fmax(fabs(rmin), fabs(rmax));
    wc = (V.vox_ext[1] + cm * V.vox_ext[0]) / lam_min;
    wr = (V.vox_ext[2] + rm * V.vox_ext[0]) / lam_min;
  } else {
    const double H = fmax(fabs(rmin), fabs(rmax));
    wc = 1.5707963267948966 * D / (rho_lo * V.dgam);
    wr = V.R * D * (1.0 / rho_lo + H / (rho_lo * rho_lo)) / V.vlen;
    const double hmin = rmin, hmax = rmax;
    const double q_lo = hmin >= 0.0 ? hmin / rho_hi : hmin / rho_lo;
    const double q_hi = hmax >= 0.0 ? hmax / rho_lo : hmax / rho_hi;
    rmin = (q_lo * V.R - V.axial0) / V.vlen;
    rmax = (q_hi * V.R - V.axial0) / V.vlen;
  }
  // Parallel and flat cone beams: the box projects exactly onto the hull of
  // its projected corners, so the pixels inside [min, max] (widened by 1e-7
  // pixel against FP64 rounding, which is below 1e-12 pixel here) are the
  // only ones whose rays can meet it.  The cylindrical bounds above are
  // themselves relaxations; they keep one more pixel on each side.
  const bool exact = P.dims.beam == CTP_BEAM_PARALLEL || P.dims.det == CTP_DET_FLAT;
  const double cl = fmax(exact ? ceil(cmin - 1e-7) : floor(cmin - 1e-7), -1.0);
  const double ch = fmin(exact ? floor(cmax + 1e-7) : ceil(cmax + 1e-7), (double)nc);
  const double rl = fmax(exact ? ceil(rmin - 1e-7) : floor(rmin - 1e-7), -1.0);
  const double rh = fmin(exact ? floor(rmax + 1e-7) : ceil(rmax + 1e-7), (double)nr);
  c0 = max((int)cl, 0);
  c1 = min((int)ch, nc - 1);
  r0 = max((int)rl, 0);
  r1 = min((int)rh, nr - 1);
  const long long fw_ = c1 >= c0 ? c1 - c0 + 1 : 0, fh_ = r1 >= r0 ? r1 - r0 + 1 : 0;
  const double pc = floor(fmin(wc, 1e6)) + 2.0, pr = floor(fmin(wr, 1e6)) + 2.0;
  nvox = (int)fmin(pc * pr, (double)(fw_ * fh_));
}

// Adjoint on one brick.  Ray contributions are accumulated in shared memory
// as 32-bit fixed point (native integer atomics; shared-memory float atomics
// are compare-and-swap loops on this hardware).  The views are taken in
// stages of kBackStage; per stage the scale S is set so that no voxel can
// overflow: every segment is at most one voxel diagonal long, |y| is at most
// the stage's largest footprint value, and no voxel meets more than the
// summed per-view ray bounds.  Each stage is then flushed into the FP32
// volume.  Integer sums are exact, so the result does not depend on the
// order in which threads add.
// kB members of a batch (1 or 2) share each ray's set-up and walk: member m
// reads sino + m * n_rays, accumulates in its own brick of fixed-point
// counters (acc + m * n_acc) with its own per-stage scale, and writes
// vol + m * n_vox.
template <int kPower, typename Off, bool kParallel, int kB>
__global__ void __launch_bounds__(kBackThreads, CTP_BACK_MIN_BLOCKS)
    back_brick_kernel(BackLaunch P, const ViewRec* __restrict__ views, const double* __restrict__ trig,
                      const float* __restrict__ sino, float* __restrict__ vol) {
  extern __shared__ int acc[];
  // per staged view: first column, first row, width, footprint size, ray bound
  __shared__ int fc0[kBackStage], fr0[kBackStage], fw[kBackStage], cnt[kBackStage], nvb[kBackStage];
  __shared__ int pre[kBackStage + 1];
  // parallel beams: per staged view, the chord trapezoid's outer columns and
  // inverse ramp widths; the length-sorted order of one window of rays
  __shared__ float fu0[kBackStage], fu3[kBackStage], firl[kBackStage], firr[kBackStage];
  __shared__ unsigned short sched[kSortWin];
  __shared__ int hist[kSortBuckets];
  __shared__ unsigned int s_ymax_bits[kB];
  __shared__ long long s_nsum;
  __shared__ float s_scale[kB];
  __shared__ int s_fast_round;

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
  for (int i = tid; i < kB * n_acc; i += kBackThreads) acc[i] = 0;
  const size_t n_rays = (size_t)P.dims.n_views * P.dims.n_rows * P.dims.n_cols;
  const size_t n_vox = (size_t)P.vol.n[0] * P.vol.n[1] * P.vol.n[2];
  const double diag = sqrt(P.vol.spacing[0] * P.vol.spacing[0] + P.vol.spacing[1] * P.vol.spacing[1] +
                           P.vol.spacing[2] * P.vol.spacing[2]);
  const int ex = hi[0] - lo[0], ey = hi[1] - lo[1], ez = hi[2] - lo[2];
  const int n_out = ex * ey * ez;
  const Off nx = P.vol.n[0], ny = P.vol.n[1];

  const int nr = P.dims.n_rows, nc = P.dims.n_cols;
  const int v_begin = g * P.views_per_group;
  const int v_end = min(v_begin + P.views_per_group, P.dims.n_views);
  bool first = true;
  for (int vb = v_begin; vb < v_end; vb += kBackStage) {
    const int nvs = min(kBackStage, v_end - vb);
    __syncthreads();  // previous stage flushed (and accumulators zeroed)
    for (int s = warp; s < nvs; s += kBackThreads / 32) {
      int c0 = 0, c1 = -1, r0 = 0, r1 = -1, nv = 0;
      float uc[4] = {0.f, 0.f, 0.f, 0.f};
      brick_footprint(views[vb + s], P, lo, hi, lane, c0, c1, r0, r1, nv, uc);
      if (lane == 0) {
        fu0[s] = uc[0];
        fu3[s] = uc[3];
        firl[s] = uc[1] > uc[0] ? 1.f / (uc[1] - uc[0]) : 1e30f;
        firr[s] = uc[3] > uc[2] ? 1.f / (uc[3] - uc[2]) : 1e30f;
        const int w = c1 >= c0 ? c1 - c0 + 1 : 0;
        const int h = r1 >= r0 ? r1 - r0 + 1 : 0;
        fc0[s] = c0;
        fr0[s] = r0;
        fw[s] = w;
        cnt[s] = w * h;
        nvb[s] = w * h > 0 ? nv : 0;
      }
    }
    if (tid < kB) s_ymax_bits[tid] = 0u;
    __syncthreads();
    if (warp == 0) {
      // exclusive scan of cnt[0..nvs) and the sum of the ray bounds
      constexpr int kPer = kBackStage / 32;
      int sum = 0;
      long long nsum = 0;
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int i = lane * kPer + j;
        sum += i < nvs ? cnt[i] : 0;
        nsum += i < nvs ? nvb[i] : 0;
      }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) nsum += __shfl_xor_sync(0xffffffffu, nsum, o);
      int run = incl - sum;
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int i = lane * kPer + j;
        if (i < nvs) {
          pre[i] = run;
          run += cnt[i];
        }
      }
      if (lane == 31) pre[nvs] = incl;
      if (lane == 0) s_nsum = nsum;
    }
    __syncthreads();
    const int total = pre[nvs];
    // pass 1: largest |y| of the stage's footprint rays (NaN and inf sort
    // above every finite value as unsigned bit patterns)
    {
      unsigned int mb[kB];
#pragma unroll
      for (int m = 0; m < kB; ++m) mb[m] = 0u;
      for (int q = tid; q < total; q += kBackThreads) {
        int sl = 0, sh = nvs;
        while (sh - sl > 1) {
          const int mid = (sl + sh) >> 1;
          if (pre[mid] <= q) sl = mid;
          else sh = mid;
        }
        const int qq = q - pre[sl];
        const int rr = qq / fw[sl];
        const int r = fr0[sl] + rr, c = fc0[sl] + (qq - rr * fw[sl]);
        const size_t i = ((size_t)(vb + sl) * nr + r) * nc + c;
#pragma unroll
        for (int m = 0; m < kB; ++m) mb[m] = max(mb[m], __float_as_uint(fabsf(__ldg(sino + m * n_rays + i))));
      }
#pragma unroll
      for (int m = 0; m < kB; ++m) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mb[m] = max(mb[m], __shfl_xor_sync(0xffffffffu, mb[m], o));
        if (lane == 0 && mb[m]) atomicMax(&s_ymax_bits[m], mb[m]);
      }
    }
    __syncthreads();
    if (tid == 0) {
      int fast = 1;
#pragma unroll
      for (int m = 0; m < kB; ++m) {
        const unsigned int bits = s_ymax_bits[m];
        float sc = 0.f;
        if (bits >= 0x7f800000u) {
          sc = CUDART_NAN_F;  // non-finite input: the brick is written as NaN
        } else {
          const double seg_max = kPower == 2 ? diag * diag : diag;
          const double one = (double)__uint_as_float(bits) * seg_max;  // largest single contribution / S
          const double bound = one * (double)s_nsum;
          if (bound > 0.0) {
            sc = (float)((2147483647.0 - 4194304.0) / bound);
            // one contribution below 4.0e6 < 2^22: the FMA rounding's range
            // (the margin covers segments a few FP32 ulps over the diagonal)
            if (!((double)sc * one < 4.0e6)) fast = 0;
          }
        }
        s_scale[m] = sc;
      }
      s_fast_round = fast;
    }
    __syncthreads();
    float S[kB];
    bool any_walk = false;
#pragma unroll
    for (int m = 0; m < kB; ++m) {
      S[m] = s_scale[m];
      any_walk |= S[m] > 0.f;
    }
    const bool fast_round = s_fast_round != 0;
    // pass 2: walk every ray of the stage through the brick.  A warp takes
    // 32 footprint rays, sets them up together and reconverges before the
    // next 32.  Footprint ray q of the stage: view vb + sl, then row-major in
    // its footprint rectangle; parallel beams take each row in mirror order
    // (0, w-1, 1, w-2, ...).
    auto locate = [&](int q, int& sl, int& r, int& c) {
      int sh = nvs;
      sl = 0;
      while (sh - sl > 1) {
        const int mid = (sl + sh) >> 1;
        if (pre[mid] <= q) sl = mid;
        else sh = mid;
      }
      const int qq = q - pre[sl];
      const int w = fw[sl];
      const int rr = qq / w;
      r = fr0[sl] + rr;
      c = fc0[sl] + (kParallel ? mirror_order(qq - rr * w, w) : qq - rr * w);
    };
    char* const accb = reinterpret_cast<char*>(acc);
    // Set up and walk one ray per lane (all 32 lanes call this together;
    // lanes without a ray pass valid = false).
    auto process = [&](int q, bool valid) {
      bool act = valid;
      int v = vb, r = 0, c = 0;
      float y[kB];
#pragma unroll
      for (int m = 0; m < kB; ++m) y[m] = 0.f;
      if (act) {
        int sl;
        locate(q, sl, r, c);
        v = vb + sl;
        const size_t i = ((size_t)v * nr + r) * nc + c;
        act = false;
        const bool in = CTP_IN_BOUNDS(i, n_rays, 8) && CTP_IN_BOUNDS(v, P.dims.n_views, 9);
#pragma unroll
        for (int m = 0; m < kB; ++m) {
          // a member whose stage scale is 0 or NaN adds nothing (its brick
          // is all zero, or written as NaN, at the flush); a single member
          // only gets here with a positive scale
          y[m] = in && (kB == 1 || S[m] > 0.f) ? __ldg(sino + m * n_rays + i) : 0.f;
          act |= y[m] != 0.f;
        }
      }
      Ray R;
      setup_t t_in = 0, t_out = 0;
      if (act) {
        make_ray(views[v], P.vol, trig, P.dims, v, r, c, R);
        act = clip(R, lo, hi, t_in, t_out);
      }
      Walk W = {};
      int off = 0;
      if (act) {
        entry(R, t_in, t_out, lo, hi, W);
        // byte offset into the accumulators: the shared atomics then
        // address [offset + constant] with no scaling per segment
        off = 4 * (((W.i[2] - lo[2]) * P.brick[1] + (W.i[1] - lo[1])) * pitch + (W.i[0] - lo[0]));
      }
      float yS[kB];
#pragma unroll
      for (int m = 0; m < kB; ++m) yS[m] = y[m] * S[m];
      // Round coef * yS to the nearest integer.  Where the stage's scale
      // keeps every contribution below 4.0e6 (< 2^22), one FMA does it:
      // adding 1.5 * 2^23 leaves the integer in the low mantissa bits.
      // Elsewhere (few rays per voxel, a finer scale) a conversion does.
      const int mbytes = 4 * n_acc;  // byte distance between the members' bricks
      auto visit_fma = [&](int o, float len) {
        if (!CTP_IN_BOUNDS(o >> 2, n_acc, 5)) return;
        const float w = coef<kPower>(len);
#pragma unroll
        for (int m = 0; m < kB; ++m)
          atomicAdd(reinterpret_cast<int*>(accb + m * mbytes + o),
                    __float_as_int(fmaf(w, yS[m], kRoundBias)) - kRoundBiasBits);
      };
      auto visit_cvt = [&](int o, float len) {
        if (!CTP_IN_BOUNDS(o >> 2, n_acc, 5)) return;
        const float w = coef<kPower>(len);
#pragma unroll
        for (int m = 0; m < kB; ++m)
          atomicAdd(reinterpret_cast<int*>(accb + m * mbytes + o), __float2int_rn(w * yS[m]));
      };
      // measured on B200: parallel rays (length-sorted, near-equal chords)
      // walk fastest with independent lane loops, cone rays with the
      // warp-uniform trip count
      if (kParallel) {
        if (act) {
          if (fast_round) walk_lane<int>(W, off, 4 * W.step[0], 4 * W.step[1] * pitch, 4 * W.step[2] * plane, visit_fma);
          else walk_lane<int>(W, off, 4 * W.step[0], 4 * W.step[1] * pitch, 4 * W.step[2] * plane, visit_cvt);
        }
        __syncwarp();
      } else if (fast_round) {
        walk_warp_bf<int>(act, W, off, 4 * W.step[0], 4 * W.step[1] * pitch, 4 * W.step[2] * plane, visit_fma);
      } else {
        walk_warp_bf<int>(act, W, off, 4 * W.step[0], 4 * W.step[1] * pitch, 4 * W.step[2] * plane, visit_cvt);
      }
    };
    if (any_walk && !kParallel) {
      for (int q0 = warp * 32; q0 < total; q0 += kBackThreads) process(q0 + lane, q0 + lane < total);
    } else if (any_walk) {
      // Parallel beams: windows of kSortWin rays, counting-sorted by the
      // chord estimated from the view's trapezoid, so that the 32 lanes of
      // a warp walk rays of near-equal length (chunks of consecutive rays
      // of one view span a ramp of the trapezoid).
      for (int w0 = 0; w0 < total; w0 += kSortWin) {
        const int nwin = min(kSortWin, total - w0);
        __syncthreads();  // the previous window's schedule is consumed
        if (tid < kSortBuckets) hist[tid] = 0;
        __syncthreads();
        constexpr int kPer = kSortWin / kBackThreads;  // 8 rays per thread, buckets packed 4 to a word
        static_assert(kPer == 8 && kSortBuckets <= 256, "bucket packing");
        unsigned int bk[2] = {0u, 0u};
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
          const int i = tid + j * kBackThreads;
          if (i < nwin) {
            int sl, r, c;
            locate(w0 + i, sl, r, c);
            const float fc = (float)c;
            const float e = fminf(fminf((fc - fu0[sl]) * firl[sl], (fu3[sl] - fc) * firr[sl]), 1.f);
            const unsigned int b = (unsigned int)(fmaxf(e, 0.f) * (kSortBuckets - 0.5f));
            bk[j >> 2] |= b << (8 * (j & 3));
            atomicAdd(&hist[b], 1);
          }
        }
        __syncthreads();
        if (warp == 0) {  // exclusive scan of the bucket counts
          const int n = hist[lane];
          int incl = n;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
          }
          hist[lane] = incl - n;
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
          const int i = tid + j * kBackThreads;
          if (i < nwin) sched[atomicAdd(&hist[(bk[j >> 2] >> (8 * (j & 3))) & 0xffu], 1)] = (unsigned short)i;
        }
        __syncthreads();
        for (int j0 = warp * 32; j0 < nwin; j0 += kBackThreads) {
          const bool ok = j0 + lane < nwin;
          process(w0 + (ok ? (int)sched[j0 + lane] : 0), ok);
        }
      }
    }
    __syncthreads();
    // flush the stage into the volume and clear the accumulators
    float inv[kB];
    bool nan_stage[kB];
#pragma unroll
    for (int m = 0; m < kB; ++m) {
      inv[m] = S[m] > 0.f ? 1.f / S[m] : 0.f;
      nan_stage[m] = S[m] != S[m];
    }
    for (int i = tid; i < n_out; i += kBackThreads) {
      const int x = i % ex;
      const int t = i / ex;
      const int yy = t % ey;
      const int z = t / ey;
      const int ai = (z * P.brick[1] + yy) * pitch + x;
      const Off gi = ((Off)(lo[2] + z) * ny + (Off)(lo[1] + yy)) * nx + (Off)(lo[0] + x);
      if (!CTP_IN_BOUNDS(ai, n_acc, 6) || !CTP_IN_BOUNDS(gi, n_vox, 7)) continue;
#pragma unroll
      for (int m = 0; m < kB; ++m) {
        const float val = nan_stage[m] ? CUDART_NAN_F : (float)acc[m * n_acc + ai] * inv[m];
        acc[m * n_acc + ai] = 0;
        float* const vm = vol + m * n_vox;
        if (P.view_groups > 1) {
          if (val != 0.f) atomicAdd(vm + gi, val);
        } else if (first) {
          vm[gi] = val;
        } else {
          vm[gi] += val;
        }
      }
    }
    first = false;
  }
}

// ------------------------------------------------------ back: sort / reduce --

// Bitonic sort of one (key, value) pair per lane across the warp, ascending
// by key; pairs move together and equal keys are never split or duplicated.
template <typename Key>
__device__ __forceinline__ void warp_sort_pairs(Key& key, float& val, int lane) {
  constexpr unsigned kFull = 0xffffffffu;
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const Key pk = __shfl_xor_sync(kFull, key, j);
      const float pv = __shfl_xor_sync(kFull, val, j);
      const bool ascending = (lane & k) == 0;
      const bool lower = (lane & j) == 0;
      const bool take = (lower == ascending) ? (pk < key) : (key < pk);
      if (take) {
        key = pk;
        val = pv;
      }
    }
  }
}

// One warp-wide batch of the sort / segment-reduce adjoint: the 32 lanes'
// (voxel key, contribution) pairs are grouped by key (a warp sort, skipped
// when the keys are already monotone across the lanes, which the aligned
// walk of neighbouring rays usually gives), each run of equal keys is summed
// with a segmented scan, and its last lane adds the run's sum to the volume
// with one global atomic.  With kCount nothing is written; instead the
// numbers of contributions and of runs are added to n_upd and n_runs.
template <bool kCount, typename Key>
__device__ __forceinline__ void warp_segment_reduce(Key key, float val, bool valid, float* __restrict__ vol, size_t n_vox,
                                                    unsigned long long& n_upd, unsigned long long& n_runs) {
  constexpr unsigned kFull = 0xffffffffu;
  const Key kNone = (Key)(~(unsigned long long)0 >> 1);
  const int lane = threadIdx.x & 31;
  if (!valid || !(val != 0.f)) {
    key = kNone;
    val = 0.f;
  }
  const Key kn = __shfl_down_sync(kFull, key, 1);
  const bool nondec = lane == 31 || key <= kn, noninc = lane == 31 || key >= kn;
  if (!__all_sync(kFull, nondec) && !__all_sync(kFull, noninc)) warp_sort_pairs(key, val, lane);
  const Key kp = __shfl_up_sync(kFull, key, 1);
  const Key kq = __shfl_down_sync(kFull, key, 1);
  const bool head = lane == 0 || kp != key;
  const bool tail = lane == 31 || kq != key;
  const unsigned heads = __ballot_sync(kFull, head);
  const int start = 31 - __clz(heads & (kFull >> (31 - lane)));
  float sum = val;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float t = __shfl_up_sync(kFull, sum, o);
    if (lane - o >= start) sum += t;
  }
  if (kCount) {
    const unsigned u = __ballot_sync(kFull, key != kNone);
    const unsigned r = __ballot_sync(kFull, tail && key != kNone);
    if (lane == 0) {
      n_upd += __popc(u);
      n_runs += __popc(r);
    }
  } else if (tail && key != kNone) {
    if (CTP_IN_BOUNDS(key, n_vox, 12)) atomicAdd(vol + key, sum);
  }
}

// Sort / segment-reduce adjoint: one thread per ray as in the forward
// kernel (same block order and aligned slab walk over the whole volume), the
// contributions of each warp step grouped and reduced before one global add
// per distinct voxel.  Needs the volume zeroed first.  With kCount it writes
// nothing and counts contributions and runs (the collision ratio) instead,
// treating every ray value as 1.
template <bool kCount, int kPower, typename Off>
__global__ void __launch_bounds__(kFwdCols* kFwdRows, CTP_FWD_MIN_BLOCKS)
    back_sort_kernel(FwdLaunch P, const ViewRec* __restrict__ views, const double* __restrict__ trig,
                     const float* __restrict__ sino, float* __restrict__ vol,
                     unsigned long long* __restrict__ counters) {
  const int per_band = P.dims.n_views * P.n_col_tiles;
  const int band = blockIdx.x / per_band;
  const int rem = blockIdx.x - band * per_band;
  const int v = rem / P.n_col_tiles;
  const int ct = rem - v * P.n_col_tiles;
  const int c = ct * kFwdCols + threadIdx.x;
  const int r = band * kFwdRows + threadIdx.y;
  const bool valid = c < P.dims.n_cols && r < P.dims.n_rows;
  float y = 1.f;
  if (!kCount) y = valid ? __ldg(sino + ((size_t)v * P.dims.n_rows + r) * P.dims.n_cols + c) : 0.f;
  Ray R;
  make_ray(views[v], P.vol, trig, P.dims, v, valid ? r : 0, valid ? c : 0, R);
  const int lo[3] = {0, 0, 0};
  const int hi[3] = {P.vol.n[0], P.vol.n[1], P.vol.n[2]};
  setup_t t_in = 0, t_out = 0;
  const bool hit = valid && y != 0.f && clip(R, lo, hi, t_in, t_out);
  Walk W = {};
  // the counting form only counts segments: no re-anchoring needed
  constexpr int kAnchor = kCount ? 0 : kWalkAnchor;
  __shared__ double s_anc[kAnchor ? 7 * kAncStride : 1];
  double* const anc = s_anc + (kAnchor ? threadIdx.y * kFwdCols + threadIdx.x : 0);
  if (hit) entry(R, t_in, t_out, lo, hi, W, kAnchor ? anc : nullptr, kAncStride);
  const Off nx = P.vol.n[0], sz = (Off)P.vol.n[0] * P.vol.n[1];
  const Off off = (Off)W.i[2] * sz + (Off)W.i[1] * nx + (Off)W.i[0];
  const size_t n_vox = (size_t)P.vol.n[0] * P.vol.n[1] * P.vol.n[2];
  unsigned long long n_upd = 0, n_runs = 0;
  walk<true, true, kAnchor, Off>(hit, W, lo, hi, off, (Off)W.step[0], W.step[1] * nx, W.step[2] * sz, anc,
                        [&](Off o, float len, bool f) {
                          warp_segment_reduce<kCount, Off>(o, coef<kPower>(len) * y, f, vol, n_vox, n_upd, n_runs);
                        });
  if (kCount && (threadIdx.x & 31) == 0 && (n_upd | n_runs)) {
    atomicAdd(counters, n_upd);
    atomicAdd(counters + 1, n_runs);
  }
}

// ------------------------------------------------------- back: ray scatter --

// Ray-driven scatter adjoint: the forward kernel's grid, set-up and aligned
// slab walk, with every positive-length segment added into the volume by one
// red.global.add.f32.  The warp's 32 lanes hold neighbouring rays of one view
// and, aligned on absolute slab positions, add into neighbouring voxels of one
// slab; views whose columns run along y accumulate into a y-fastest copy (as
// the forward gathers from it), so a warp's adds stay within a few sectors.
// Both accumulators must be zero on entry; transpose_add_kernel folds the copy
// into the volume afterwards.
template <int kPower, typename Off>
__global__ void __launch_bounds__(kFwdCols* kFwdRows, CTP_SCATTER_MIN_BLOCKS)
    back_scatter_kernel(FwdLaunch P, const ViewRec* __restrict__ views, const double* __restrict__ trig,
                        const float* __restrict__ sino, float* __restrict__ vol, float* __restrict__ volT) {
  const int per_band = P.dims.n_views * P.n_col_tiles;
  const int band = blockIdx.x / per_band;
  const int rem = blockIdx.x - band * per_band;
  const int v = rem / P.n_col_tiles;
  const int ct = rem - v * P.n_col_tiles;
  const int c = ct * kFwdCols + threadIdx.x;
  const int r = band * kFwdRows + threadIdx.y;
  const bool valid = c < P.dims.n_cols && r < P.dims.n_rows;
  const float y = valid ? __ldg(sino + ((size_t)v * P.dims.n_rows + r) * P.dims.n_cols + c) : 0.f;
  const ViewRec& V = views[v];
  Ray R;
  make_ray(V, P.vol, trig, P.dims, v, valid ? r : 0, valid ? c : 0, R);
  const int lo[3] = {0, 0, 0};
  const int hi[3] = {P.vol.n[0], P.vol.n[1], P.vol.n[2]};
  setup_t t_in = 0, t_out = 0;
  const bool hit = valid && y != 0.f && clip(R, lo, hi, t_in, t_out);
  Walk W = {};
  __shared__ double s_anc[7 * kAncStride];
  double* const anc = s_anc + threadIdx.y * kFwdCols + threadIdx.x;
  if (hit) entry(R, t_in, t_out, lo, hi, W, anc, kAncStride);
  const Off nx = P.vol.n[0], ny = P.vol.n[1];
  const bool yfast = V.layout != 0;
  float* const base = yfast ? volT : vol;
  const Off sx = yfast ? ny : (Off)1;
  const Off sy = yfast ? (Off)1 : nx;
  const Off sz = nx * ny;
  const Off off = (Off)W.i[2] * sz + (Off)W.i[1] * sy + (Off)W.i[0] * sx;
  [[maybe_unused]] const size_t n_vox = (size_t)P.vol.n[0] * P.vol.n[1] * P.vol.n[2];
  walk<true, false, kWalkAnchor, Off>(hit, W, lo, hi, off, W.step[0] * sx, W.step[1] * sy, W.step[2] * sz, anc,
                                      [&](Off o, float len, bool) {
                           if (len > 0.f && CTP_IN_BOUNDS(o, n_vox, 10)) atomicAdd(base + o, coef<kPower>(len) * y);
                         });
}

// vol[z][y][x] += volT[z][x][y] (the scatter adjoint's y-fastest accumulator).
__global__ void __launch_bounds__(256) transpose_add_kernel(const float* __restrict__ in, float* __restrict__ out,
                                                            int nx, int ny) {
  __shared__ float tile[32][33];
  const size_t slice = (size_t)blockIdx.z * nx * ny;
  const int x0 = blockIdx.x * 32, y0 = blockIdx.y * 32;
  for (int j = threadIdx.y; j < 32; j += 8) {
    const int y = y0 + threadIdx.x, x = x0 + j;
    if (x < nx && y < ny) tile[j][threadIdx.x] = in[slice + (size_t)x * ny + y];
  }
  __syncthreads();
  for (int j = threadIdx.y; j < 32; j += 8) {
    const int x = x0 + threadIdx.x, y = y0 + j;
    if (x < nx && y < ny) out[slice + (size_t)y * nx + x] += tile[threadIdx.x][j];
  }
}

// ------------------------------------------ parallel slices: shared (x, y) walks --
//
// When every ray lies in a plane of constant z (a parallel beam whose
// direction has no z component) and detector rows step along z only, the rays
// of one detector column in one view all follow the same (x, y) path, each in
// the slice of its own row (the slices decouple; MBIRJAX "Sharding overview",
// section "Why cone beam").  A thread then sets up and walks that path once
// for kR consecutive rows and applies every segment to the kR slices.  Each
// row's FP64 set-up equals that of its own ray in the x and y components (the
// pixel centres differ in z only), so every row sees exactly the segments,
// in the same order, that a walk of its own ray would give.

#ifndef CTP_ROWS_MIN_BLOCKS
#define CTP_ROWS_MIN_BLOCKS 4
#endif

template <typename Off, int kR>
__global__ void __launch_bounds__(kFwdCols* kFwdRows, CTP_ROWS_MIN_BLOCKS)
    forward_rows_kernel(FwdLaunch P, const ViewRec* __restrict__ views, const float* __restrict__ vol,
                        const float* __restrict__ volT, float* __restrict__ sino) {
  int v, c, r0;
  rows_block_position<kR>(P, v, c, r0);
  const bool cvalid = c < P.dims.n_cols;
  const ViewRec& V = views[v];
  const Off nx = P.vol.n[0], ny = P.vol.n[1];
  const Off sz = nx * ny;
  Off zoff[kR];
  const unsigned rows = cvalid ? row_slices<kR, Off>(V, P.vol, r0, c, P.dims.n_rows, sz, zoff) : 0u;
  Ray R;
  setup_t t_in = 0, t_out = 0;
  const bool hit = slice_ray(V, P.vol, P.dims, v, cvalid ? c : 0, R, t_in, t_out) && rows != 0u;
  const int lo[3] = {0, 0, 0};
  const int hi[3] = {P.vol.n[0], P.vol.n[1], P.vol.n[2]};
  Walk W = {};
  if (hit) entry(R, t_in, t_out, lo, hi, W);
  const bool yfast = V.layout != 0;
  const float* __restrict__ base = yfast ? volT : vol;
  const Off sx = yfast ? ny : (Off)1;
  const Off sy = yfast ? (Off)1 : nx;
  const Off off = (Off)W.i[1] * sy + (Off)W.i[0] * sx;
  [[maybe_unused]] const size_t n_vox = (size_t)P.vol.n[0] * P.vol.n[1] * P.vol.n[2];
  float acc[kR];
#pragma unroll
  for (int j = 0; j < kR; ++j) acc[j] = 0.f;
  // every row of the group inside the volume (the common case) takes the
  // walk without per-row tests; the warp decides together
  if (__all_sync(0xffffffffu, rows == (1u << kR) - 1u || !hit)) {
    walk<true, false, 0, Off>(hit, W, lo, hi, off, W.step[0] * sx, W.step[1] * sy, (Off)0, nullptr,
                              [&](Off o, float len, bool) {
#pragma unroll
                                for (int j = 0; j < kR; ++j)
                                  if (CTP_IN_BOUNDS(o + zoff[j], n_vox, 3))
                                    acc[j] = fmaf(len, __ldg(base + o + zoff[j]), acc[j]);
                              });
  } else {
    walk<true, false, 0, Off>(hit, W, lo, hi, off, W.step[0] * sx, W.step[1] * sy, (Off)0, nullptr,
                              [&](Off o, float len, bool) {
#pragma unroll
                                for (int j = 0; j < kR; ++j)
                                  if ((rows & (1u << j)) && CTP_IN_BOUNDS(o + zoff[j], n_vox, 3))
                                    acc[j] = fmaf(len, __ldg(base + o + zoff[j]), acc[j]);
                              });
  }
  if (cvalid) {
#pragma unroll
    for (int j = 0; j < kR; ++j) {
      const int r = r0 + j;
      const size_t i = ((size_t)v * P.dims.n_rows + r) * P.dims.n_cols + c;
      if (r < P.dims.n_rows && CTP_IN_BOUNDS(i, (size_t)P.dims.n_views * P.dims.n_rows * P.dims.n_cols, 4))
        sino[i] = acc[j];
    }
  }
}

template <int kPower, typename Off, int kR>
__global__ void __launch_bounds__(kFwdCols* kFwdRows, CTP_ROWS_MIN_BLOCKS)
    back_scatter_rows_kernel(FwdLaunch P, const ViewRec* __restrict__ views, const float* __restrict__ sino,
                             float* __restrict__ vol, float* __restrict__ volT) {
  int v, c, r0;
  rows_block_position<kR>(P, v, c, r0);
  const bool cvalid = c < P.dims.n_cols;
  const ViewRec& V = views[v];
  const Off nx = P.vol.n[0], ny = P.vol.n[1];
  const Off sz = nx * ny;
  Off zoff[kR];
  unsigned rows = cvalid ? row_slices<kR, Off>(V, P.vol, r0, c, P.dims.n_rows, sz, zoff) : 0u;
  float y[kR];
#pragma unroll
  for (int j = 0; j < kR; ++j) {
    y[j] = (rows & (1u << j)) ? __ldg(sino + ((size_t)v * P.dims.n_rows + r0 + j) * P.dims.n_cols + c) : 0.f;
    if (!(y[j] != 0.f)) rows &= ~(1u << j);  // zero rows add nothing (NaN stays)
  }
  Ray R;
  setup_t t_in = 0, t_out = 0;
  const bool hit = slice_ray(V, P.vol, P.dims, v, cvalid ? c : 0, R, t_in, t_out) && rows != 0u;
  const int lo[3] = {0, 0, 0};
  const int hi[3] = {P.vol.n[0], P.vol.n[1], P.vol.n[2]};
  Walk W = {};
  __shared__ double s_anc[7 * kAncStride];
  double* const anc = s_anc + threadIdx.y * kFwdCols + threadIdx.x;
  if (hit) entry(R, t_in, t_out, lo, hi, W, anc, kAncStride);
  const bool yfast = V.layout != 0;
  float* const base = yfast ? volT : vol;
  const Off sx = yfast ? ny : (Off)1;
  const Off sy = yfast ? (Off)1 : nx;
  const Off off = (Off)W.i[1] * sy + (Off)W.i[0] * sx;
  [[maybe_unused]] const size_t n_vox = (size_t)P.vol.n[0] * P.vol.n[1] * P.vol.n[2];
  // every row of the group inside the volume with a non-zero value (the
  // common case) takes the walk without per-row tests; the warp decides together
  if (__all_sync(0xffffffffu, rows == (1u << kR) - 1u || !hit)) {
    walk<true, false, kWalkAnchor, Off>(hit, W, lo, hi, off, W.step[0] * sx, W.step[1] * sy, (Off)0, anc,
                                        [&](Off o, float len, bool) {
                                          if (len > 0.f) {
                                            const float w = coef<kPower>(len);
#pragma unroll
                                            for (int j = 0; j < kR; ++j)
                                              if (CTP_IN_BOUNDS(o + zoff[j], n_vox, 11))
                                                atomicAdd(base + o + zoff[j], w * y[j]);
                                          }
                                        });
  } else {
    walk<true, false, kWalkAnchor, Off>(hit, W, lo, hi, off, W.step[0] * sx, W.step[1] * sy, (Off)0, anc,
                                        [&](Off o, float len, bool) {
                                          if (len > 0.f) {
                                            const float w = coef<kPower>(len);
#pragma unroll
                                            for (int j = 0; j < kR; ++j)
                                              if ((rows & (1u << j)) && CTP_IN_BOUNDS(o + zoff[j], n_vox, 11))
                                                atomicAdd(base + o + zoff[j], w * y[j]);
                                          }
                                        });
  }
}

// ------------------------------- parallel slices: volumes interleaved by 4 --
//
// Slices taken in groups of four and interleaved: element [g][y][x][s] holds
// slice 4g + s ([g][x][y][s] for the copy whose fastest axes are swapped),
// with ng = ceil(nz / 4) groups and the slices past nz zero.  A thread of a
// shared (x, y) walk over 4 rows whose heights fall in the 4 slices of one
// group (the common case, rows and slices of equal pitch) then reads its 4
// values with one 16-byte load, or adds its 4 contributions with one 16-byte
// reduction; any other row group addresses single elements.  Each row still
// sees exactly its own segments, in the same order.

template <typename Off>
__global__ void __launch_bounds__(kFwdCols* kFwdRows, CTP_ROWS_MIN_BLOCKS)
    forward_rows4_kernel(FwdLaunch P, const ViewRec* __restrict__ views, const float4* __restrict__ vol4,
                         const float4* __restrict__ vol4T, float* __restrict__ sino) {
  int v, c, r0;
  rows_block_position<4>(P, v, c, r0);
  const bool cvalid = c < P.dims.n_cols;
  const ViewRec& V = views[v];
  const Off nx = P.vol.n[0], ny = P.vol.n[1];
  const Off plane = nx * ny;
  [[maybe_unused]] const Off n4 = (Off)((P.vol.n[2] + 3) >> 2) * plane;  // float4 elements of one copy
  int ks[4];
  const unsigned rows = cvalid ? row_slice_index<4>(V, P.vol, r0, c, P.dims.n_rows, ks) : 0u;
  Ray R;
  setup_t t_in = 0, t_out = 0;
  const bool hit = slice_ray(V, P.vol, P.dims, v, cvalid ? c : 0, R, t_in, t_out) && rows != 0u;
  const int lo[3] = {0, 0, 0};
  const int hi[3] = {P.vol.n[0], P.vol.n[1], P.vol.n[2]};
  Walk W = {};
  if (hit) entry(R, t_in, t_out, lo, hi, W);
  const bool yfast = V.layout != 0;
  const float4* __restrict__ base4 = yfast ? vol4T : vol4;
  const float* __restrict__ base1 = reinterpret_cast<const float*>(base4);
  const Off sx = yfast ? ny : (Off)1;
  const Off sy = yfast ? (Off)1 : nx;
  const Off off = (Off)W.i[1] * sy + (Off)W.i[0] * sx;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  if (__all_sync(0xffffffffu, one_group(rows, ks) || !hit)) {
    const Off g = (Off)(ks[0] >> 2) * plane;
    walk<true, false, 0, Off>(hit, W, lo, hi, off, W.step[0] * sx, W.step[1] * sy, (Off)0, nullptr,
                              [&](Off o, float len, bool) {
                                if (CTP_IN_BOUNDS(g + o, n4, 15)) {
                                  const float4 q = __ldg(base4 + g + o);
                                  acc[0] = fmaf(len, q.x, acc[0]);
                                  acc[1] = fmaf(len, q.y, acc[1]);
                                  acc[2] = fmaf(len, q.z, acc[2]);
                                  acc[3] = fmaf(len, q.w, acc[3]);
                                }
                              });
  } else {
    Off e[4];  // float index of row j's slice at (x, y) = (0, 0)
#pragma unroll
    for (int j = 0; j < 4; ++j) e[j] = ((Off)(ks[j] >> 2) * plane) * 4 + (ks[j] & 3);
    walk<true, false, 0, Off>(hit, W, lo, hi, off, W.step[0] * sx, W.step[1] * sy, (Off)0, nullptr,
                              [&](Off o, float len, bool) {
#pragma unroll
                                for (int j = 0; j < 4; ++j)
                                  if ((rows & (1u << j)) && CTP_IN_BOUNDS(e[j] + 4 * o, 4 * n4, 16))
                                    acc[j] = fmaf(len, __ldg(base1 + e[j] + 4 * o), acc[j]);
                              });
  }
  if (cvalid) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int r = r0 + j;
      const size_t i = ((size_t)v * P.dims.n_rows + r) * P.dims.n_cols + c;
      if (r < P.dims.n_rows && CTP_IN_BOUNDS(i, (size_t)P.dims.n_views * P.dims.n_rows * P.dims.n_cols, 4))
        sino[i] = acc[j];
    }
  }
}

template <int kPower, typename Off>
__global__ void __launch_bounds__(kFwdCols* kFwdRows, CTP_ROWS_MIN_BLOCKS)
    back_scatter_rows4_kernel(FwdLaunch P, const ViewRec* __restrict__ views, const float* __restrict__ sino,
                              float4* __restrict__ acc4, float4* __restrict__ acc4T) {
  int v, c, r0;
  rows_block_position<4>(P, v, c, r0);
  const bool cvalid = c < P.dims.n_cols;
  const ViewRec& V = views[v];
  const Off nx = P.vol.n[0], ny = P.vol.n[1];
  const Off plane = nx * ny;
  [[maybe_unused]] const Off n4 = (Off)((P.vol.n[2] + 3) >> 2) * plane;
  int ks[4];
  const unsigned inside = cvalid ? row_slice_index<4>(V, P.vol, r0, c, P.dims.n_rows, ks) : 0u;
  float y[4];
  unsigned rows = inside;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    y[j] = (inside & (1u << j)) ? __ldg(sino + ((size_t)v * P.dims.n_rows + r0 + j) * P.dims.n_cols + c) : 0.f;
    if (!(y[j] != 0.f)) rows &= ~(1u << j);  // zero rows add nothing (NaN stays)
  }
  Ray R;
  setup_t t_in = 0, t_out = 0;
  const bool hit = slice_ray(V, P.vol, P.dims, v, cvalid ? c : 0, R, t_in, t_out) && rows != 0u;
  const int lo[3] = {0, 0, 0};
  const int hi[3] = {P.vol.n[0], P.vol.n[1], P.vol.n[2]};
  Walk W = {};
  __shared__ double s_anc[7 * kAncStride];
  double* const anc = s_anc + threadIdx.y * kFwdCols + threadIdx.x;
  if (hit) entry(R, t_in, t_out, lo, hi, W, anc, kAncStride);
  const bool yfast = V.layout != 0;
  float4* const base4 = yfast ? acc4T : acc4;
  float* const base1 = reinterpret_cast<float*>(base4);
  const Off sx = yfast ? ny : (Off)1;
  const Off sy = yfast ? (Off)1 : nx;
  const Off off = (Off)W.i[1] * sy + (Off)W.i[0] * sx;
  // a group of 4 rows in the 4 slices of one group adds the 4 contributions
  // of a segment with one 16-byte reduction (a zero row adds zeros)
  if (__all_sync(0xffffffffu, one_group(inside, ks) || !hit)) {
    const Off g = (Off)(ks[0] >> 2) * plane;
    walk<true, false, kWalkAnchor, Off>(hit, W, lo, hi, off, W.step[0] * sx, W.step[1] * sy, (Off)0, anc,
                                        [&](Off o, float len, bool) {
                                          if (len > 0.f && CTP_IN_BOUNDS(g + o, n4, 17)) {
                                            const float w = coef<kPower>(len);
                                            atomicAdd(base4 + g + o, make_float4(w * y[0], w * y[1], w * y[2], w * y[3]));
                                          }
                                        });
  } else {
    Off e[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) e[j] = ((Off)(ks[j] >> 2) * plane) * 4 + (ks[j] & 3);
    walk<true, false, kWalkAnchor, Off>(hit, W, lo, hi, off, W.step[0] * sx, W.step[1] * sy, (Off)0, anc,
                                        [&](Off o, float len, bool) {
                                          if (len > 0.f) {
                                            const float w = coef<kPower>(len);
#pragma unroll
                                            for (int j = 0; j < 4; ++j)
                                              if ((rows & (1u << j)) && CTP_IN_BOUNDS(e[j] + 4 * o, 4 * n4, 18))
                                                atomicAdd(base1 + e[j] + 4 * o, w * y[j]);
                                          }
                                        });
  }
}

// Slices of vol [nz][ny][nx] interleaved by 4 into out4 [ng][ny][nx] and, if
// given, out4T [ng][nx][ny].  One block: a 32 x 32 (x, y) tile of one group.
__global__ void __launch_bounds__(256) interleave_kernel(const float* __restrict__ in, float4* __restrict__ out4,
                                                         float4* __restrict__ out4T, int nx, int ny, int nz) {
  __shared__ float tile[4][32][33];
  const int g = blockIdx.z, x0 = blockIdx.x * 32, y0 = blockIdx.y * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const int z = 4 * g + s;
    for (int j = ty; j < 32; j += 8) {
      const int x = x0 + tx, y = y0 + j;
      tile[s][j][tx] = (x < nx && y < ny && z < nz) ? in[((size_t)z * ny + y) * nx + x] : 0.f;
    }
  }
  __syncthreads();
  for (int j = ty; j < 32; j += 8) {
    const int x = x0 + tx, y = y0 + j;
    if (x < nx && y < ny)
      out4[((size_t)g * ny + y) * nx + x] = make_float4(tile[0][j][tx], tile[1][j][tx], tile[2][j][tx], tile[3][j][tx]);
  }
  if (out4T) {
    for (int j = ty; j < 32; j += 8) {
      const int y = y0 + tx, x = x0 + j;
      if (x < nx && y < ny)
        out4T[((size_t)g * nx + x) * ny + y] =
            make_float4(tile[0][tx][j], tile[1][tx][j], tile[2][tx][j], tile[3][tx][j]);
    }
  }
}

// out [nz][ny][nx] = acc4 [ng][ny][nx] (+ acc4T [ng][nx][ny]), slice by slice.
__global__ void __launch_bounds__(256) deinterleave_kernel(const float4* __restrict__ acc4,
                                                           const float4* __restrict__ acc4T, float* __restrict__ out,
                                                           int nx, int ny, int nz) {
  __shared__ float tile[4][32][33];
  const int g = blockIdx.z, x0 = blockIdx.x * 32, y0 = blockIdx.y * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;
  for (int j = ty; j < 32; j += 8) {
    const int x = x0 + tx, y = y0 + j;
    const float4 a = (x < nx && y < ny) ? acc4[((size_t)g * ny + y) * nx + x] : make_float4(0.f, 0.f, 0.f, 0.f);
    tile[0][j][tx] = a.x;
    tile[1][j][tx] = a.y;
    tile[2][j][tx] = a.z;
    tile[3][j][tx] = a.w;
  }
  if (acc4T) {
    __syncthreads();
    for (int j = ty; j < 32; j += 8) {
      const int y = y0 + tx, x = x0 + j;
      const float4 b =
          (x < nx && y < ny) ? acc4T[((size_t)g * nx + x) * ny + y] : make_float4(0.f, 0.f, 0.f, 0.f);
      tile[0][tx][j] += b.x;
      tile[1][tx][j] += b.y;
      tile[2][tx][j] += b.z;
      tile[3][tx][j] += b.w;
    }
  }
  __syncthreads();
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const int z = 4 * g + s;
    if (z >= nz) break;
    for (int j = ty; j < 32; j += 8) {
      const int x = x0 + tx, y = y0 + j;
      if (x < nx && y < ny) out[((size_t)z * ny + y) * nx + x] = tile[s][j][tx];
    }
  }
}

}  // namespace

// ---------------------------------------------------------------- launchers --

cudaError_t launch_interleave(const FwdLaunch& p, const float* vol, float4* vol4, float4* vol4T,
                              cudaStream_t stream) {
  const int ng = (p.vol.n[2] + 3) / 4;
  dim3 tgrid((p.vol.n[0] + 31) / 32, (p.vol.n[1] + 31) / 32, ng);
  interleave_kernel<<<tgrid, dim3(32, 8), 0, stream>>>(vol, vol4, p.any_transposed ? vol4T : nullptr, p.vol.n[0],
                                                      p.vol.n[1], p.vol.n[2]);
  return cudaGetLastError();
}

cudaError_t launch_forward_rows4(const FwdLaunch& p, const ViewRec* views, const float* vol, float4* vol4,
                                 float4* vol4T, float* sino, bool wide_index, cudaStream_t stream) {
  cudaError_t e = launch_interleave(p, vol, vol4, vol4T, stream);
  if (e != cudaSuccess) return e;
  const long long blocks = (long long)rows_bands(p.dims.n_rows, 4) * p.dims.n_views * rows_col_tiles(p.dims.n_cols);
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  if (wide_index)
    forward_rows4_kernel<long long><<<(unsigned)blocks, dim3(kFwdCols, kFwdRows), 0, stream>>>(p, views, vol4, vol4T,
                                                                                                sino);
  else
    forward_rows4_kernel<int><<<(unsigned)blocks, dim3(kFwdCols, kFwdRows), 0, stream>>>(p, views, vol4, vol4T, sino);
  return cudaGetLastError();
}

cudaError_t launch_back_scatter_rows4(const FwdLaunch& p, const ViewRec* views, const float* sino, float* vol,
                                      float4* acc4, float4* acc4T, int power, bool wide_index, cudaStream_t stream) {
  const long long blocks = (long long)rows_bands(p.dims.n_rows, 4) * p.dims.n_views * rows_col_tiles(p.dims.n_cols);
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  if (blocks > 0) {
    const unsigned nb = (unsigned)blocks;
    const dim3 block(kFwdCols, kFwdRows);
    if (power == 2) {
      if (wide_index) back_scatter_rows4_kernel<2, long long><<<nb, block, 0, stream>>>(p, views, sino, acc4, acc4T);
      else back_scatter_rows4_kernel<2, int><<<nb, block, 0, stream>>>(p, views, sino, acc4, acc4T);
    } else {
      if (wide_index) back_scatter_rows4_kernel<1, long long><<<nb, block, 0, stream>>>(p, views, sino, acc4, acc4T);
      else back_scatter_rows4_kernel<1, int><<<nb, block, 0, stream>>>(p, views, sino, acc4, acc4T);
    }
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int ng = (p.vol.n[2] + 3) / 4;
  dim3 tgrid((p.vol.n[0] + 31) / 32, (p.vol.n[1] + 31) / 32, ng);
  deinterleave_kernel<<<tgrid, dim3(32, 8), 0, stream>>>(acc4, p.any_transposed ? acc4T : nullptr, vol, p.vol.n[0],
                                                        p.vol.n[1], p.vol.n[2]);
  return cudaGetLastError();
}

// The bounds-check word of this file's kernels (CTP_DEBUG builds; 0 elsewhere),
// read and cleared.  Synchronous.
unsigned long long debug_take_word_kernels() {
#ifdef CTP_DEBUG
  unsigned long long w = 0, z = 0;
  if (cudaMemcpyFromSymbol(&w, g_debug_word, sizeof(w)) != cudaSuccess) return ~0ull;
  cudaMemcpyToSymbol(g_debug_word, &z, sizeof(z));
  return w;
#else
  return 0;
#endif
}

cudaError_t launch_forward_rows(const FwdLaunch& p, const ViewRec* views, const float* vol, const float* volT,
                                float* sino, bool wide_index, cudaStream_t stream) {
  const long long blocks =
      (long long)rows_bands(p.dims.n_rows, p.row_group) * p.dims.n_views * rows_col_tiles(p.dims.n_cols);
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  dim3 block(kFwdCols, kFwdRows);
  const unsigned nb = (unsigned)blocks;
#define CTP_ROWS_LAUNCH(OFF, R) forward_rows_kernel<OFF, R><<<nb, block, 0, stream>>>(p, views, vol, volT, sino)
  switch (p.row_group) {
    case 2:
      if (wide_index) CTP_ROWS_LAUNCH(long long, 2); else CTP_ROWS_LAUNCH(int, 2);
      break;
    case 4:
      if (wide_index) CTP_ROWS_LAUNCH(long long, 4); else CTP_ROWS_LAUNCH(int, 4);
      break;
    case 8:
      if (wide_index) CTP_ROWS_LAUNCH(long long, 8); else CTP_ROWS_LAUNCH(int, 8);
      break;
    default:
      return cudaErrorInvalidValue;
  }
#undef CTP_ROWS_LAUNCH
  return cudaGetLastError();
}

cudaError_t launch_back_scatter(const FwdLaunch& p, const ViewRec* views, const double* trig, const float* sino,
                                float* vol, float* volT, int power, bool wide_index, cudaStream_t stream) {
  const long long blocks = (long long)p.n_row_bands * p.dims.n_views * p.n_col_tiles;
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  dim3 block(kFwdCols, kFwdRows);
  const unsigned nb = (unsigned)blocks;
  if (p.row_group > 1) {
    const long long rb =
        (long long)rows_bands(p.dims.n_rows, p.row_group) * p.dims.n_views * rows_col_tiles(p.dims.n_cols);
    if (rb > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    const unsigned nr = (unsigned)rb;
#define CTP_SROWS(KP, OFF, R) back_scatter_rows_kernel<KP, OFF, R><<<nr, block, 0, stream>>>(p, views, sino, vol, volT)
    if (p.row_group == 8) {
      if (power == 2) {
        if (wide_index) CTP_SROWS(2, long long, 8); else CTP_SROWS(2, int, 8);
      } else {
        if (wide_index) CTP_SROWS(1, long long, 8); else CTP_SROWS(1, int, 8);
      }
    } else if (p.row_group == 4) {
      if (power == 2) {
        if (wide_index) CTP_SROWS(2, long long, 4); else CTP_SROWS(2, int, 4);
      } else {
        if (wide_index) CTP_SROWS(1, long long, 4); else CTP_SROWS(1, int, 4);
      }
    } else if (p.row_group == 2) {
      if (power == 2) {
        if (wide_index) CTP_SROWS(2, long long, 2); else CTP_SROWS(2, int, 2);
      } else {
        if (wide_index) CTP_SROWS(1, long long, 2); else CTP_SROWS(1, int, 2);
      }
    } else {
      return cudaErrorInvalidValue;
    }
#undef CTP_SROWS
  } else if (power == 2) {
    if (wide_index) back_scatter_kernel<2, long long><<<nb, block, 0, stream>>>(p, views, trig, sino, vol, volT);
    else back_scatter_kernel<2, int><<<nb, block, 0, stream>>>(p, views, trig, sino, vol, volT);
  } else {
    if (wide_index) back_scatter_kernel<1, long long><<<nb, block, 0, stream>>>(p, views, trig, sino, vol, volT);
    else back_scatter_kernel<1, int><<<nb, block, 0, stream>>>(p, views, trig, sino, vol, volT);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || !p.any_transposed) return e;
  dim3 grid((p.vol.n[0] + 31) / 32, (p.vol.n[1] + 31) / 32, p.vol.n[2]);
  transpose_add_kernel<<<grid, dim3(32, 8), 0, stream>>>(volT, vol, p.vol.n[0], p.vol.n[1]);
  return cudaGetLastError();
}

cudaError_t launch_transpose_xy(const float* vol, float* volT, const VolDesc& vd, cudaStream_t stream) {
  dim3 grid((vd.n[0] + 31) / 32, (vd.n[1] + 31) / 32, vd.n[2]);
  transpose_xy_kernel<<<grid, dim3(32, 8), 0, stream>>>(vol, volT, vd.n[0], vd.n[1]);
  return cudaGetLastError();
}

cudaError_t launch_forward(const FwdLaunch& p, const ViewRec* views, const double* trig, const float* vol,
                           const float* volT, float* sino, int kb, bool wide_index, cudaStream_t stream) {
  const long long blocks = (long long)p.n_row_bands * p.dims.n_views * p.n_col_tiles;
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  dim3 block(kFwdCols, kFwdRows);
  const unsigned nb = (unsigned)blocks;
#define CTP_FWD_LAUNCH(OFF, KB) forward_kernel<OFF, KB><<<nb, block, 0, stream>>>(p, views, trig, vol, volT, sino)
  switch (kb) {
    case 1:
      if (wide_index) CTP_FWD_LAUNCH(long long, 1); else CTP_FWD_LAUNCH(int, 1);
      break;
    case 2:
      if (wide_index) CTP_FWD_LAUNCH(long long, 2); else CTP_FWD_LAUNCH(int, 2);
      break;
    case 4:
      if (wide_index) CTP_FWD_LAUNCH(long long, 4); else CTP_FWD_LAUNCH(int, 4);
      break;
    default:
      return cudaErrorInvalidValue;
  }
#undef CTP_FWD_LAUNCH
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

cudaError_t launch_back_sort(const FwdLaunch& p, const ViewRec* views, const double* trig, const float* sino,
                             float* vol, int power, bool wide_index, cudaStream_t stream) {
  const long long blocks = (long long)p.n_row_bands * p.dims.n_views * p.n_col_tiles;
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  dim3 block(kFwdCols, kFwdRows);
  const unsigned nb = (unsigned)blocks;
  if (power == 2) {
    if (wide_index) back_sort_kernel<false, 2, long long><<<nb, block, 0, stream>>>(p, views, trig, sino, vol, nullptr);
    else back_sort_kernel<false, 2, int><<<nb, block, 0, stream>>>(p, views, trig, sino, vol, nullptr);
  } else {
    if (wide_index) back_sort_kernel<false, 1, long long><<<nb, block, 0, stream>>>(p, views, trig, sino, vol, nullptr);
    else back_sort_kernel<false, 1, int><<<nb, block, 0, stream>>>(p, views, trig, sino, vol, nullptr);
  }
  return cudaGetLastError();
}

cudaError_t launch_collision_count(const FwdLaunch& p, const ViewRec* views, const double* trig,
                                   unsigned long long* counters, bool wide_index, cudaStream_t stream) {
  const long long blocks = (long long)p.n_row_bands * p.dims.n_views * p.n_col_tiles;
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  dim3 block(kFwdCols, kFwdRows);
  if (wide_index)
    back_sort_kernel<true, 1, long long><<<(unsigned)blocks, block, 0, stream>>>(p, views, trig, nullptr, nullptr,
                                                                                counters);
  else
    back_sort_kernel<true, 1, int><<<(unsigned)blocks, block, 0, stream>>>(p, views, trig, nullptr, nullptr, counters);
  return cudaGetLastError();
}

size_t back_brick_smem_bytes(const int32_t brick[3], int kb) {
  return sizeof(int) * (size_t)kb * (size_t)(brick[0] + 1) * brick[1] * brick[2];
}

namespace {
template <int kB>
cudaError_t set_back_smem(int bytes) {
  const void* kernels[] = {
      (const void*)back_brick_kernel<1, int, true, kB>,  (const void*)back_brick_kernel<1, long long, true, kB>,
      (const void*)back_brick_kernel<2, int, true, kB>,  (const void*)back_brick_kernel<2, long long, true, kB>,
      (const void*)back_brick_kernel<1, int, false, kB>, (const void*)back_brick_kernel<1, long long, false, kB>,
      (const void*)back_brick_kernel<2, int, false, kB>, (const void*)back_brick_kernel<2, long long, false, kB>};
  for (const void* k : kernels) {
    const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <int kB>
void launch_back_brick_kb(const BackLaunch& p, const ViewRec* views, const double* trig, const float* sino,
                          float* vol, int power, bool wide_index, unsigned nb, size_t smem, cudaStream_t stream) {
  const bool par = p.dims.beam == CTP_BEAM_PARALLEL;
#define CTP_BACK_LAUNCH(KP, OFF, PAR) \
  back_brick_kernel<KP, OFF, PAR, kB><<<nb, kBackThreads, smem, stream>>>(p, views, trig, sino, vol)
  if (power == 2) {
    if (wide_index) {
      if (par) CTP_BACK_LAUNCH(2, long long, true); else CTP_BACK_LAUNCH(2, long long, false);
    } else {
      if (par) CTP_BACK_LAUNCH(2, int, true); else CTP_BACK_LAUNCH(2, int, false);
    }
  } else {
    if (wide_index) {
      if (par) CTP_BACK_LAUNCH(1, long long, true); else CTP_BACK_LAUNCH(1, long long, false);
    } else {
      if (par) CTP_BACK_LAUNCH(1, int, true); else CTP_BACK_LAUNCH(1, int, false);
    }
  }
#undef CTP_BACK_LAUNCH
}
}  // namespace

cudaError_t prepare_back_brick(size_t smem_bytes, int kb) {
  // the limit set so far, per device and member count (one lock: create is rare)
  static std::mutex mu;
  static std::map<std::pair<int, int>, size_t> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  size_t& have = done[{dev, kb}];
  if (smem_bytes <= have) return cudaSuccess;
  e = kb == 2 ? set_back_smem<2>((int)smem_bytes) : set_back_smem<1>((int)smem_bytes);
  if (e == cudaSuccess) have = smem_bytes;
  return e;
}

cudaError_t launch_back_brick(const BackLaunch& p, const ViewRec* views, const double* trig, const float* sino,
                              float* vol, int power, int kb, bool wide_index, cudaStream_t stream) {
  if (kb != 1 && kb != 2) return cudaErrorInvalidValue;
  const long long blocks = (long long)p.nbrick[0] * p.nbrick[1] * p.nbrick[2] * p.view_groups;
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const size_t smem = back_brick_smem_bytes(p.brick, kb);
  if (kb == 2) launch_back_brick_kb<2>(p, views, trig, sino, vol, power, wide_index, (unsigned)blocks, smem, stream);
  else launch_back_brick_kb<1>(p, views, trig, sino, vol, power, wide_index, (unsigned)blocks, smem, stream);
  return cudaGetLastError();
}

}  // namespace ctp
