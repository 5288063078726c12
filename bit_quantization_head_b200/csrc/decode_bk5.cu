// Instantiations of the decode split kernel for b_K = 5 (all b_V).
#include "decode_kernel.cuh"

namespace kvtc {
namespace dec {
template <>
SplitFn split_fn_bk<5>(int bV) {
  switch (bV) {
    case 2: return decode_split_kernel<5, 2>;
    case 3: return decode_split_kernel<5, 3>;
    case 4: return decode_split_kernel<5, 4>;
    case 5: return decode_split_kernel<5, 5>;
    case 6: return decode_split_kernel<5, 6>;
    case 7: return decode_split_kernel<5, 7>;
    default: return decode_split_kernel<5, 8>;
  }
}
}  // namespace dec
}  // namespace kvtc
