// Instantiations of the decode split kernel for key code width class 0 (0 = any width);
// value width 16 = uncompressed values.
#include "decode_kernel.cuh"

namespace kvtc {
namespace dec {
template <>
SplitFn split_fn_bk<0>(int bV, bool pack) {
  if (bV == 2 && pack == true) return decode_split_kernel<0, 2, true>;
  if (bV == 2 && pack == false) return decode_split_kernel<0, 2, false>;
  if (bV == 4 && pack == true) return decode_split_kernel<0, 4, true>;
  if (bV == 4 && pack == false) return decode_split_kernel<0, 4, false>;
  if (bV == 8 && pack == true) return decode_split_kernel<0, 8, true>;
  if (bV == 8 && pack == false) return decode_split_kernel<0, 8, false>;
  if (bV == 0 && pack == true) return decode_split_kernel<0, 0, true>;
  if (bV == 0 && pack == false) return decode_split_kernel<0, 0, false>;
  if (bV == 16 && pack == true) return decode_split_kernel<0, 16, true>;
  if (bV == 16 && pack == false) return decode_split_kernel<0, 16, false>;
  return nullptr;
}
}  // namespace dec
}  // namespace kvtc
