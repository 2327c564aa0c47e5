// RoPE positions of the joint sequence [text | image | references] (the
// 2-D positions of the prologue and of the rope table): text tokens at
// (0, 0); image token u at (u / img_w, u % img_w); token u of reference
// grid g at (grid_row[g] + u / grid_w[g], grid_col[g] + u % grid_w[g]).
#pragma once

#include "jattn_internal.h"

namespace jattn {

__device__ __forceinline__ void token_pos(const PrologueArgs& a, int t, int& row, int& col) {
  if (t < a.n_txt) {
    row = 0;
    col = 0;
    return;
  }
  int u = t - a.n_txt;
  if (u < a.n_img) {
    row = u / a.img_w;
    col = u - row * a.img_w;
    return;
  }
  u -= a.n_img;
  // The grid holding u, by a fixed-trip scan with constant indices (a
  // data-dependent loop over the parameter arrays measured 8% slower in the
  // FP8 prologue).
  int start = 0, w = a.grid_w[0], row0 = a.grid_row[0], col0 = a.grid_col[0];
#pragma unroll
  for (int g = 1; g < kMaxRefGrids; ++g) {
    if (g < a.n_grids && u >= a.grid_end[g - 1]) {
      start = a.grid_end[g - 1];
      w = a.grid_w[g];
      row0 = a.grid_row[g];
      col0 = a.grid_col[g];
    }
  }
  const int v = u - start;
  const int r = v / w;
  row = row0 + r;
  col = col0 + (v - r * w);
}

}  // namespace jattn
