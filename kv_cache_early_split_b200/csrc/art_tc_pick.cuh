// art_tc_pick.cuh -- instantiations of the tensor-core decode kernel, one translation unit per
// head count (art_tc_gp{1,2,4,8}.cu) so that they compile in parallel.
#pragma once

#include "art_tc.cuh"

namespace artk {
namespace tc {

using TcFn = void (*)(TcParams);

// The kernel for GP heads per kv head: mode MODE_FULL / MODE_ART, probe capacity pc (16 or 32, ART),
// general addressing (traversal sequence or paged cache), ncw ART controller warps (1 or 2).
template <int GP>
TcFn pick_gp(int mode, int pc, bool gen, int ncw) {
  if (mode != MODE_ART)
    return gen ? &art_decode_tc_kernel<GP, MODE_FULL, 16, true, 1> : &art_decode_tc_kernel<GP, MODE_FULL, 16, false, 1>;
  if (pc <= 16) {
    if (gen) return ncw == 2 ? &art_decode_tc_kernel<GP, MODE_ART, 16, true, 2> : &art_decode_tc_kernel<GP, MODE_ART, 16, true, 1>;
    return ncw == 2 ? &art_decode_tc_kernel<GP, MODE_ART, 16, false, 2> : &art_decode_tc_kernel<GP, MODE_ART, 16, false, 1>;
  }
  if (gen) return ncw == 2 ? &art_decode_tc_kernel<GP, MODE_ART, 32, true, 2> : &art_decode_tc_kernel<GP, MODE_ART, 32, true, 1>;
  return ncw == 2 ? &art_decode_tc_kernel<GP, MODE_ART, 32, false, 2> : &art_decode_tc_kernel<GP, MODE_ART, 32, false, 1>;
}

// defined in art_tc_gp1.cu, art_tc_gp2.cu, art_tc_gp4.cu, art_tc_gp8.cu
TcFn kernel_gp1(int mode, int pc, bool gen, int ncw);
TcFn kernel_gp2(int mode, int pc, bool gen, int ncw);
TcFn kernel_gp4(int mode, int pc, bool gen, int ncw);
TcFn kernel_gp8(int mode, int pc, bool gen, int ncw);

}  // namespace tc
}  // namespace artk
