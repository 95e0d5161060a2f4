// Host-side check of the fragment-major record layout helpers that the
// encoders' word-parallel merge relies on.  Prints "ok" or the first failure.
//   sign_chunk_bit: for m = 64 and 128 the (sign j, token half h) pairs map
//     one to one onto the chunk's m/2 bits; for m = 128 half h is word h
//     with the h = 0 positions; for m = 64 both halves share word 0, half h
//     at the h = 0 positions + 4 h, inside the nibble mask 0x0f0f0f0f << 4h.
//   lane_word_offset: word w < nw of tile lane l < 32 lands on distinct,
//     4-byte-aligned offsets inside the plane's 128 nw bytes.
//   Codes: 2 PT codes of bw bits fill words_for_bits(2 PT bw) words, and the
//     two halves share a word exactly when PT bw is not a multiple of 32.
#include <cstdio>
#include <vector>

#include "tq_internal.cuh"

int main() {
  using namespace tq;
  long checked = 0;
  for (int m : {64, 128}) {
    const int qb = m / 4;
    const int sw = words_for_bits(2 * qb);
    std::vector<int> seen(32 * sw, 0);
    for (int h = 0; h < 2; ++h)
      for (int j = 0; j < qb; ++j) {
        const int b = sign_chunk_bit(j, h, m), b0 = sign_chunk_bit(j, 0, m);
        if (b < 0 || b >= 32 * sw || seen[b]++) {
          printf("sign bits: m=%d h=%d j=%d -> %d (not one to one)\n", m, h, j, b);
          return 1;
        }
        if (m == 128 && (b0 >= 32 || b != 32 * h + b0)) {
          printf("sign words: m=128 h=%d j=%d -> %d, h=0 gives %d\n", h, j, b, b0);
          return 1;
        }
        if (m == 64 && (b != 4 * h + b0 || !(((0x0f0f0f0fu << (4 * h)) >> b) & 1u))) {
          printf("sign nibbles: m=64 h=%d j=%d -> %d, h=0 gives %d\n", h, j, b, b0);
          return 1;
        }
        ++checked;
      }
    int used = 0;
    for (int v : seen) used += v;
    if (used != 2 * qb) {
      printf("sign bits: m=%d covers %d of %d\n", m, used, 2 * qb);
      return 1;
    }
  }
  for (int nw = 1; nw <= 8; ++nw) {
    std::vector<int> seen(128 * nw / 4, 0);
    for (int w = 0; w < nw; ++w)
      for (int l = 0; l < 32; ++l) {
        const int off = lane_word_offset(w, l, nw);
        if (off < 0 || off % 4 || off >= 128 * nw || seen[off / 4]++) {
          printf("word offsets: nw=%d w=%d l=%d -> %d\n", nw, w, l, off);
          return 1;
        }
        ++checked;
      }
  }
  for (int pt : {8, 16, 32})
    for (int bw = 2; bw <= 8; ++bw) {
      const int bits = 2 * pt * bw, nw = words_for_bits(bits);
      const bool shared = ((pt * bw) & 31) != 0;          // the merge's test
      const bool one_word = ((pt * bw - 1) >> 5) == ((pt * bw) >> 5);   // h = 0's last bit, h = 1's first
      if (nw * 32 < bits || (nw - 1) * 32 >= bits || shared != one_word) {
        printf("code words: pt=%d bw=%d\n", pt, bw);
        return 1;
      }
      ++checked;
    }
  printf("ok %ld\n", checked);
  return 0;
}
