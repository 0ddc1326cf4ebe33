// Tensor-core decode kernel instantiations for 8 query head(s) per kv head.
#include "art_tc_pick.cuh"

namespace artk {
namespace tc {
TcFn kernel_gp8(int mode, int pc, bool ord, bool paged, int ncw) {
  return pick_gp<8>(mode, pc, ord, paged, ncw);
}
}  // namespace tc
}  // namespace artk
