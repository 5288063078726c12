// Instantiations of the decode split kernel for key code width class 4 (0 = any width);
// value width 16 = uncompressed values.
#include "decode_kernel.cuh"

namespace kvtc {
namespace dec {
template <>
SplitFn split_fn_bk<4>(int bV, bool pack) {
  if (bV == 2 && pack == true) return decode_split_kernel<4, 2, true>;
  if (bV == 2 && pack == false) return decode_split_kernel<4, 2, false>;
  if (bV == 4 && pack == true) return decode_split_kernel<4, 4, true>;
  if (bV == 4 && pack == false) return decode_split_kernel<4, 4, false>;
  if (bV == 8 && pack == true) return decode_split_kernel<4, 8, true>;
  if (bV == 8 && pack == false) return decode_split_kernel<4, 8, false>;
  if (bV == 0 && pack == true) return decode_split_kernel<4, 0, true>;
  if (bV == 0 && pack == false) return decode_split_kernel<4, 0, false>;
  if (bV == 16 && pack == true) return decode_split_kernel<4, 16, true>;
  if (bV == 16 && pack == false) return decode_split_kernel<4, 16, false>;
  return nullptr;
}
}  // namespace dec
}  // namespace kvtc
