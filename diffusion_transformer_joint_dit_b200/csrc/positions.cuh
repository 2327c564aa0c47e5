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
  int g = 0;
  while (g + 1 < a.n_grids && u >= a.grid_end[g]) ++g;
  const int v = u - (g > 0 ? a.grid_end[g - 1] : 0);
  const int r = v / a.grid_w[g];
  row = a.grid_row[g] + r;
  col = a.grid_col[g] + (v - r * a.grid_w[g]);
}

}  // namespace jattn
