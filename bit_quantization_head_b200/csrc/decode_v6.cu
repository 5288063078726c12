// Instantiations of the decode split kernel for 6-bit key codes; value widths 2..8,
// or 16 = uncompressed values.
#include "decode_kernel.cuh"

namespace kvtc {
namespace dec {
template <>
SplitFn split_fn_bk<6>(int bV, bool pack) {
  switch (bV) {
    case 2: return pack ? decode_split_kernel<6, 2, true> : decode_split_kernel<6, 2, false>;
    case 3: return pack ? decode_split_kernel<6, 3, true> : decode_split_kernel<6, 3, false>;
    case 4: return pack ? decode_split_kernel<6, 4, true> : decode_split_kernel<6, 4, false>;
    case 5: return pack ? decode_split_kernel<6, 5, true> : decode_split_kernel<6, 5, false>;
    case 6: return pack ? decode_split_kernel<6, 6, true> : decode_split_kernel<6, 6, false>;
    case 7: return pack ? decode_split_kernel<6, 7, true> : decode_split_kernel<6, 7, false>;
    case 8: return pack ? decode_split_kernel<6, 8, true> : decode_split_kernel<6, 8, false>;
    case 16: return pack ? decode_split_kernel<6, 16, true> : decode_split_kernel<6, 16, false>;
    default: return nullptr;
  }
}
}  // namespace dec
}  // namespace kvtc
