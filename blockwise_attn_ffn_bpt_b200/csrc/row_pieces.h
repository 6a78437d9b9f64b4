// Rows of several sequences split into the rectangles one attention launch
// covers (host code). The flat rows are sequence-major: row r is position
// r % s of sequence r / s. A launch covers either whole sequences or one
// sequence's run of positions, so a run of flat rows becomes, in row order,
// a partial sequence, whole sequences (one piece), and a partial sequence.
#pragma once

#include <algorithm>

namespace bpt {

struct RowPiece {
  int beta;     // first sequence
  int n_seq;    // sequences (whole ones when more than one)
  int t_start;  // first position within the sequence
  int t_len;    // positions per sequence
};

// Calls f(piece) for the pieces of the flat rows [r0, r0 + m) of b sequences
// of s rows (0 <= r0, r0 + m <= b * s, s > 0), in row order; returns the first
// nonzero value f returns, else 0.
template <class F>
int for_each_row_piece(long long r0, long long m, int b, int s, F&& f) {
  for (long long r = r0, end = r0 + m; r < end;) {
    const int beta = (int)(r / s), t = (int)(r - (long long)beta * s);
    const bool whole = t == 0 && end - r >= s;
    const int nb = whole ? (int)std::min<long long>((end - r) / s, (long long)b - beta) : 1;
    const int tl = whole ? s : (int)std::min<long long>((long long)s - t, end - r);
    const int st = f(RowPiece{beta, nb, t, tl});
    if (st != 0) return st;
    r += (long long)nb * tl;
  }
  return 0;
}

}  // namespace bpt
