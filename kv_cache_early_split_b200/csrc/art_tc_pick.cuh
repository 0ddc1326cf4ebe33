// art_tc_pick.cuh -- instantiations of the tensor-core decode kernel, one translation unit per
// head count (art_tc_gp{1,2,4,8}.cu) so that they compile in parallel.
#pragma once

#include "art_tc.cuh"

namespace artk {
namespace tc {

using TcFn = void (*)(TcParams);

// The kernel for GP heads per kv head: mode MODE_FULL / MODE_ART, probe capacity pc (16 or 32, ART),
// a traversal sequence (ord, ART only), a paged cache (paged), the ART controller ncw (0: sequential,
// single-CTA cluster; 1 or 2: scan controller warps).
template <int GP, int MODE, int PC, bool ORD, bool PAGED>
TcFn pick_ncw(int ncw) {
  if (ncw == 0) return &art_decode_tc_kernel<GP, MODE, PC, ORD, PAGED, 0>;
  return ncw == 2 ? &art_decode_tc_kernel<GP, MODE, PC, ORD, PAGED, 2> : &art_decode_tc_kernel<GP, MODE, PC, ORD, PAGED, 1>;
}

template <int GP, int PC>
TcFn pick_art(bool ord, bool paged, int ncw) {
  if (ord) return paged ? pick_ncw<GP, MODE_ART, PC, true, true>(ncw) : pick_ncw<GP, MODE_ART, PC, true, false>(ncw);
  return paged ? pick_ncw<GP, MODE_ART, PC, false, true>(ncw) : pick_ncw<GP, MODE_ART, PC, false, false>(ncw);
}

template <int GP>
TcFn pick_gp(int mode, int pc, bool ord, bool paged, int ncw) {
  if (mode != MODE_ART)
    return paged ? &art_decode_tc_kernel<GP, MODE_FULL, 16, false, true, 1>
                 : &art_decode_tc_kernel<GP, MODE_FULL, 16, false, false, 1>;
  return pc <= 16 ? pick_art<GP, 16>(ord, paged, ncw) : pick_art<GP, 32>(ord, paged, ncw);
}

// defined in art_tc_gp1.cu, art_tc_gp2.cu, art_tc_gp4.cu, art_tc_gp8.cu
TcFn kernel_gp1(int mode, int pc, bool ord, bool paged, int ncw);
TcFn kernel_gp2(int mode, int pc, bool ord, bool paged, int ncw);
TcFn kernel_gp4(int mode, int pc, bool ord, bool paged, int ncw);
TcFn kernel_gp8(int mode, int pc, bool ord, bool paged, int ncw);
// q8 cache, 4 query heads per kv head, natural order, contiguous (defined in art_tc_q8.cu)
TcFn kernel_q8(int mode, int pc, int ncw);

}  // namespace tc
}  // namespace artk
