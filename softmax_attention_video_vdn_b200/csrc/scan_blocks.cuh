// scan_blocks.cuh - which block states each step of the bidirectional scan
// stores (shared by the forward scan and its adjoint).
//
// sd114.wiki, bidirectional linear branch: the forward state of block b
// covers the frames before b's window, the backward state the frames after
// it; anchor frames take no part.
#pragma once

namespace vdn {

__device__ __forceinline__ bool is_anchor(int f, int T, int anchors) {
  return anchors && (f == 0 || f == T - 1);
}

// Blocks whose forward state is the state before frame f (window start == f).
__device__ __forceinline__ void fwd_blocks(int f, int bf, int W, int nb, int* lo, int* hi) {
  if (f == 0) {
    *lo = 0;
    *hi = min(W, nb - 1);
  } else if (f % bf == 0 && f / bf + W < nb) {
    *lo = *hi = f / bf + W;
  } else {
    *lo = 1;
    *hi = 0;
  }
}
// Blocks whose backward state is the state before frame f in decreasing order
// (window end == f + 1).
__device__ __forceinline__ void bwd_blocks(int f, int T, int bf, int W, int nb, int* lo, int* hi) {
  const int e = f + 1;
  if (e == T) {
    // every block whose window reaches the end: (b + W + 1) * bf >= T
    int first = (T + bf - 1) / bf - W - 1;
    *lo = max(first, 0);
    *hi = nb - 1;
  } else if (e % bf == 0 && e / bf - W - 1 >= 0) {
    *lo = *hi = e / bf - W - 1;
  } else {
    *lo = 1;
    *hi = 0;
  }
}

}  // namespace vdn
