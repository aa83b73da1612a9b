// Work partition of the output projection's split mode (projection.cuh),
// shared by the projection kernel, its reduce kernel and a host-side test.
//
// Tile t owns units [t*upt, (t+1)*upt) of U units in all; C CTAs; CTA c owns
// the contiguous range [begin(c), begin(c+1)) with begin(c) = floor(c U / C).
// With C <= U every CTA owns at least one unit, and with C > U / upt (more
// CTAs than tiles) a range holds units of at most two tiles, its segments
// 0 and 1.  Plain integer arithmetic, instantiated for 32- and 64-bit types.
#pragma once

#if defined(__CUDACC__)
#define MLA_PLAN_FN __host__ __device__ __forceinline__
#else
#define MLA_PLAN_FN inline
#endif

namespace mla {

// First unit of CTA c.
template <typename I>
MLA_PLAN_FN I proj_unit_begin(I c, I U, I C) {
  return c * U / C;
}

// The CTA whose range holds unit x: the largest c with begin(c) <= x, i.e.
// ceil((x + 1) C / U) - 1.
template <typename I>
MLA_PLAN_FN I proj_cta_of_unit(I x, I U, I C) {
  return ((x + 1) * C - 1) / U;
}

// The CTAs holding units of tile t: [*lo, *hi] (each owns at least one unit
// when C <= U).
template <typename I>
MLA_PLAN_FN void proj_tile_ctas(I t, I upt, I U, I C, I* lo, I* hi) {
  *lo = proj_cta_of_unit(t * upt, U, C);
  *hi = proj_cta_of_unit(t * upt + upt - 1, U, C);
}

// Which segment of CTA c tile t is: 0 when c's range starts in tile t, 1 when
// it starts in the tile before.
template <typename I>
MLA_PLAN_FN int proj_segment_of(I c, I t, I upt, I U, I C) {
  return proj_unit_begin(c, U, C) / upt == t ? 0 : 1;
}

}  // namespace mla
