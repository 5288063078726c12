// Instantiations of the decode split kernel for key code width class 8 (0 = any width).
#include "decode_kernel.cuh"

namespace kvtc {
namespace dec {
template <>
SplitFn split_fn_bk<8>(int bV, bool pack, bool small) {
    if (bV == 2 && pack == true && small == true) return decode_split_kernel<8, 2, true, 4>;
    if (bV == 2 && pack == true && small == false) return decode_split_kernel<8, 2, true, 8>;
    if (bV == 2 && pack == false && small == true) return decode_split_kernel<8, 2, false, 4>;
    if (bV == 2 && pack == false && small == false) return decode_split_kernel<8, 2, false, 8>;
    if (bV == 4 && pack == true && small == true) return decode_split_kernel<8, 4, true, 4>;
    if (bV == 4 && pack == true && small == false) return decode_split_kernel<8, 4, true, 8>;
    if (bV == 4 && pack == false && small == true) return decode_split_kernel<8, 4, false, 4>;
    if (bV == 4 && pack == false && small == false) return decode_split_kernel<8, 4, false, 8>;
    if (bV == 8 && pack == true && small == true) return decode_split_kernel<8, 8, true, 4>;
    if (bV == 8 && pack == true && small == false) return decode_split_kernel<8, 8, true, 8>;
    if (bV == 8 && pack == false && small == true) return decode_split_kernel<8, 8, false, 4>;
    if (bV == 8 && pack == false && small == false) return decode_split_kernel<8, 8, false, 8>;
    if (bV == 0 && pack == true && small == true) return decode_split_kernel<8, 0, true, 4>;
    if (bV == 0 && pack == true && small == false) return decode_split_kernel<8, 0, true, 8>;
    if (bV == 0 && pack == false && small == true) return decode_split_kernel<8, 0, false, 4>;
    if (bV == 0 && pack == false && small == false) return decode_split_kernel<8, 0, false, 8>;
    return nullptr;
}
}  // namespace dec
}  // namespace kvtc
