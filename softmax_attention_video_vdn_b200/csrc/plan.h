// plan.h - the softmax branch's window plan (frame mask, query segments and
// key ranges) built from block arithmetic, and its token-level form passed to
// the softmax kernel as a launch parameter.
//
// sd114.wiki, bidirectional sliding-window softmax branch: latent frames are
// packed into blocks of `bf` frames; a block attends itself and the `W`
// blocks on each side; with anchors every frame also attends the first and
// last frames, and those two frames attend every frame.
#pragma once

#include <stdint.h>

#include <vector>

namespace vdn {

struct FrameSegment {
  int q0, q1;         // query frames [q0, q1), one block, equal mask rows
  int nr;             // number of key ranges (1..3)
  int k0[3], k1[3];   // key frame ranges [k0, k1), ascending, disjoint
};

// Key ranges of query frame i (maximal runs of ones of its mask row).
#if defined(__CUDACC__)
#define VDN_HD __host__ __device__
#else
#define VDN_HD
#endif

VDN_HD inline int frame_row_ranges(int T, int bf, int W, int anchors, int i, int* k0, int* k1) {
  if (anchors && (i == 0 || i == T - 1)) {
    k0[0] = 0;
    k1[0] = T;
    return 1;
  }
  const int b = i / bf;
  const int ws = (b - W) * bf > 0 ? (b - W) * bf : 0;
  const long we_l = (long)(b + W + 1) * bf;
  const int we = we_l < T ? (int)we_l : T;
  int n = 0;
  int s[3], e[3];
  if (anchors && ws > 0) { s[n] = 0; e[n] = 1; ++n; }
  s[n] = ws; e[n] = we; ++n;
  if (anchors && we < T) { s[n] = T - 1; e[n] = T; ++n; }
  // merge touching runs (an anchor next to the window)
  int m = 0;
  for (int r = 0; r < n; ++r) {
    if (m > 0 && s[r] <= k1[m - 1]) {
      if (e[r] > k1[m - 1]) k1[m - 1] = e[r];
    } else {
      k0[m] = s[r];
      k1[m] = e[r];
      ++m;
    }
  }
  return m;
}

inline bool same_row(const FrameSegment& a, int nr, const int* k0, const int* k1) {
  if (a.nr != nr) return false;
  for (int r = 0; r < nr; ++r)
    if (a.k0[r] != k0[r] || a.k1[r] != k1[r]) return false;
  return true;
}

// Query segments: maximal runs of consecutive frames of one block whose mask
// rows are equal.
inline std::vector<FrameSegment> build_segments(int T, int bf, int W, int anchors) {
  std::vector<FrameSegment> segs;
  for (int i = 0; i < T; ++i) {
    int k0[3], k1[3];
    const int nr = frame_row_ranges(T, bf, W, anchors, i, k0, k1);
    if (!segs.empty() && (segs.back().q0 / bf) == (i / bf) && same_row(segs.back(), nr, k0, k1)) {
      segs.back().q1 = i + 1;
      continue;
    }
    FrameSegment s{};
    s.q0 = i;
    s.q1 = i + 1;
    s.nr = nr;
    for (int r = 0; r < nr; ++r) {
      s.k0[r] = k0[r];
      s.k1[r] = k1[r];
    }
    segs.push_back(s);
  }
  return segs;
}

// Token-level plan for one softmax launch (fits the 4 KB parameter space with
// the tensor maps). Segments are sorted by key tokens per query tile,
// heaviest first; a work item is a pair of 128-row q tiles of one segment and
// one (b, h); the forward numbers items (b, h) by (b, h), then segment by
// segment, then pair; the backward segment by segment, then (b, h), then tile.
constexpr int kMaxLaunchSegments = 40;
constexpr int kMaxRanges = 4;   // up to 3 frame ranges, plus the context tokens
constexpr int kQTile = 128;
constexpr int kKvTile = 128;

struct SoftmaxPlan {
  int n_seg;
  int total_tiles;                     // work items (pairs of 128-row q tiles) per (b, h)
  int q0[kMaxLaunchSegments];          // token range of the segment
  int q1[kMaxLaunchSegments];
  int tile_begin[kMaxLaunchSegments];  // first work item (pair of q tiles) of the segment
  int nr[kMaxLaunchSegments];
  int k0[kMaxLaunchSegments][kMaxRanges];  // token ranges of the keys
  int k1[kMaxLaunchSegments][kMaxRanges];
};

}  // namespace vdn
