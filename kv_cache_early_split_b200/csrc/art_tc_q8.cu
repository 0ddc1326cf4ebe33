// Tensor-core decode kernel instantiations for a q8 cache (4 query heads per kv head).
#include "art_tc_pick.cuh"

namespace artk {
namespace tc {
template <int PC>
TcFn pick_q8_art(int ncw) {
  if (ncw == 0) return &art_decode_tc_kernel<4, MODE_ART, PC, false, false, 0, true>;
  return ncw == 2 ? &art_decode_tc_kernel<4, MODE_ART, PC, false, false, 2, true>
                  : &art_decode_tc_kernel<4, MODE_ART, PC, false, false, 1, true>;
}
TcFn kernel_q8(int mode, int pc, int ncw) {
  if (mode != MODE_ART) return &art_decode_tc_kernel<4, MODE_FULL, 16, false, false, 1, true>;
  return pc <= 16 ? pick_q8_art<16>(ncw) : pick_q8_art<32>(ncw);
}
}  // namespace tc
}  // namespace artk
