// reshard.cu - the layout copy of the head-sharded layer's input exchange.
//
// "Performance Results" (branch-specific Ulysses sequence parallelism on 8
// B200): each rank holds a token shard of q, k, v, [B, Ls, H, d] token-major,
// and sends every other rank that rank's heads. For the all-to-alls to send
// contiguous runs, head h_local of group g (global head g * Hs + h_local)
// goes to
//   out [B, Hs, G, Ls, d]:  out[b][h_local][g][l] = x[b][l][g * Hs + h_local].
// Each 256-byte row (d = 128 bf16) moves as 16 vectors of 16 bytes; both
// sides stay coalesced.
#include "kernels.h"

namespace vdn {

// 16 lanes per 256-byte row (d = 128 bf16): lane c moves bytes [16 c, 16 c
// + 16) of one row; a warp moves two rows per step. rows = B * H * Ls < 2^31.
__global__ void pack_head_groups_kernel(const uint4* __restrict__ x, uint4* __restrict__ out,
                                        int rows, int Ls, int H, int Hs, int G) {
  const int c = threadIdx.x & 15;
  const int stride = (gridDim.x * blockDim.x) >> 4;
  for (int orow = (blockIdx.x * blockDim.x + threadIdx.x) >> 4; orow < rows; orow += stride) {
    // output row ((b * Hs + h) * G + g) * Ls + l
    const int l = orow % Ls;
    int r = orow / Ls;
    const int g = r % G;
    r /= G;
    const int h = r % Hs;
    const int b = r / Hs;
    const long long irow = ((long long)b * Ls + l) * H + g * Hs + h;
    out[(long long)orow * 16 + c] = __ldg(x + irow * 16 + c);
  }
}

}  // namespace vdn
