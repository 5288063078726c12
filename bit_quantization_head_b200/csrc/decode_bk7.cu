// Instantiations of the decode split kernel for b_K = 7 (all b_V).
#include "decode_kernel.cuh"

namespace kvtc {
namespace dec {
template <>
SplitFn split_fn_bk<7>(int bV) {
  switch (bV) {
    case 2: return decode_split_kernel<7, 2>;
    case 3: return decode_split_kernel<7, 3>;
    case 4: return decode_split_kernel<7, 4>;
    case 5: return decode_split_kernel<7, 5>;
    case 6: return decode_split_kernel<7, 6>;
    case 7: return decode_split_kernel<7, 7>;
    default: return decode_split_kernel<7, 8>;
  }
}
}  // namespace dec
}  // namespace kvtc
