// Page layout of the packed code cache (device helpers).
//
// A page holds 128 tokens of one unit and is 16*r*b bytes.  A b-bit code is split into
// parts of width 8, 4, 2 or 1 (binary expansion of b, lowest code bits first); part p
// of width w and low bit lo lives in a plane starting at byte 16*r*lo.  Planes are rows
// of 32-bit little-endian words.  Token t has pair index pi = 2*(t/16) + (t/8)%2.
//   K unit: row rho = j/2 (8w words) holds coordinates 2rho, 2rho+1 of every token;
//     owner o = t%8 owns words [o*w, (o+1)*w); the field sits in word o*w + pi/(16/w) at
//     bit (pi%(16/w))*w + 16*(j%2).
//   V unit: row j (4w words); owner o = (t%8)/2 owns words [o*w, (o+1)*w); the field sits
//     in word o*w + pi/(16/w) at bit (pi%(16/w))*w + 16*(t%2).
// The decode kernel's m16n8k16 A fragments read these words directly: for K, lane
// (g, t') takes owner g's words of rows 8ks+t' and 8ks+4+t'; for V, owner t''s words of
// rows 16mt+g and 16mt+g+8.
#pragma once
#include <cstdint>

namespace kvtc {

struct FieldPos {
  uint32_t word;  // word index within the page
  uint32_t bit;   // bit offset within the word
};

// Part list of a b-bit code: number of parts, and (lo, width) of part i.
__host__ __device__ inline int code_nparts(int b) { return (b & 8 ? 1 : 0) + (b & 4 ? 1 : 0) + (b & 2 ? 1 : 0) + (b & 1); }
__host__ __device__ inline void code_part(int b, int i, int& lo, int& w) {
  lo = 0;
  int k = 0;
  for (int ww = 8; ww >= 1; ww >>= 1) {
    if (b & ww) {
      if (k == i) {
        w = ww;
        return;
      }
      lo += ww;
      ++k;
    }
  }
  w = 0;
}

// Position of the width-w part (low bit lo) of code (t, j) of a unit with r coordinates.
__host__ __device__ inline FieldPos field_pos(int kind, int r, int lo, int w, int t, int j) {
  const uint32_t plane_word = static_cast<uint32_t>(4 * r * lo);  // 16*r*lo bytes
  const int pi = 2 * (t >> 4) + ((t >> 3) & 1);
  const int per_word = 16 / w;
  FieldPos f;
  if (kind == 0) {
    const int o = t & 7;
    f.word = plane_word + static_cast<uint32_t>((j >> 1) * 8 * w + o * w + pi / per_word);
    f.bit = static_cast<uint32_t>((pi % per_word) * w + 16 * (j & 1));
  } else {
    const int o = (t & 7) >> 1;
    f.word = plane_word + static_cast<uint32_t>(j * 4 * w + o * w + pi / per_word);
    f.bit = static_cast<uint32_t>((pi % per_word) * w + 16 * (t & 1));
  }
  return f;
}

}  // namespace kvtc
