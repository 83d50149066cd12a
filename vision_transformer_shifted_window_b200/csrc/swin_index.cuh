// Index arithmetic of the shifted-window partition, shared by every kernel
// and by the host code of libswinattn.
//
// Swin's cyclic shift by s followed by an MxM window partition and a region
// mask ("Swin Transformer V2" wiki card, Method: window partitioning as in
// Swin V1; Pitfalls: shift offsets for even and odd window sizes) attends
// token pairs that lie in the same segment on both axes, where an axis of
// length L is cut at s + kM and clipped to [0, L).  The kernels work directly
// on these segments ("rectangles" = one segment per axis): each rectangle is
// an independent dense attention problem, so no rolled copy, no padding and
// no per-element mask is needed.
#pragma once

#include <cstdint>

#define SWIN_HD __host__ __device__ __forceinline__

// Number of segments of an axis of length L.
SWIN_HD int swin_nseg(int L, int M, int s) {
  if (s == 0) return (L + M - 1) / M;
  if (L <= s) return 1;
  return 1 + (L - s + M - 1) / M;
}

// First coordinate of segment k.
SWIN_HD int swin_seg_start(int k, int M, int s) {
  if (s == 0) return k * M;
  return k == 0 ? 0 : s + (k - 1) * M;
}

// Length of segment k (the last one is clipped at L).
SWIN_HD int swin_seg_len(int k, int L, int M, int s) {
  int a = swin_seg_start(k, M, s);
  int b = (s == 0) ? (k + 1) * M : s + k * M;
  return (b < L ? b : L) - a;
}

// Window-local coordinate used for RoPE: the position inside the MxM window
// of the rolled frame, (y - s) mod M.
SWIN_HD int swin_local_coord(int y, int M, int s) {
  int r = (y - s) % M;
  return r < 0 ? r + M : r;
}

// Row of the (2M-1)^2 relative-position table for offset (dy, dx) = query - key.
SWIN_HD int swin_rel_row(int dy, int dx, int M) {
  return (dy + M - 1) * (2 * M - 1) + (dx + M - 1);
}

// Rolled-frame bookkeeping (Swin's own labels) for one token.
struct SwinRolled {
  int window, band, local;
};

SWIN_HD SwinRolled swin_rolled(int y, int x, int H, int W, int M, int s) {
  int Hp = ((H + M - 1) / M) * M, Wp = ((W + M - 1) / M) * M;
  int u = (y - s) % Hp;
  if (u < 0) u += Hp;
  int v = (x - s) % Wp;
  if (v < 0) v += Wp;
  int by = 0, bx = 0;
  if (s > 0) {
    by = u < Hp - M ? 0 : (u < Hp - s ? 1 : 2);
    bx = v < Wp - M ? 0 : (v < Wp - s ? 1 : 2);
  }
  SwinRolled r;
  r.window = (u / M) * (Wp / M) + v / M;
  r.band = by * 3 + bx;
  r.local = (u % M) * M + (v % M);
  return r;
}

// Partitions an axis can be cut into (see include/swin_attn.h).
enum SwinPartition : int { kPartShifted = 0, kPartInterleaved = 1 };

// One window along an axis: its tokens are start + stride * i for i < len,
// and the window-local coordinate of token i is base + i.  Shifted windows
// are the segments above (stride 1; base = (start - s) mod M, so the local
// coordinates of a segment run without a wrap up to M - 1).  Interleaved
// windows ("Iwin Transformer", abstract: interleaved window attention) take
// G = ceil(L / M) windows per axis; window k holds k + G i inside the axis
// (len = ceil((L - k) / G) <= M) and its local coordinate is i.  Offsets of
// two tokens of one window are differences of their i in either partition.
struct SwinAxis {
  int start, stride, len, base;
};

SWIN_HD int swin_nwin(int part, int L, int M, int s) {
  return part == kPartInterleaved ? (L + M - 1) / M : swin_nseg(L, M, s);
}

SWIN_HD SwinAxis swin_axis(int part, int k, int L, int M, int s) {
  SwinAxis a;
  if (part == kPartInterleaved) {
    const int G = (L + M - 1) / M;
    a.start = k;
    a.stride = G;
    a.len = (L - k + G - 1) / G;
    a.base = 0;
  } else {
    a.start = swin_seg_start(k, M, s);
    a.stride = 1;
    a.len = swin_seg_len(k, L, M, s);
    a.base = swin_local_coord(a.start, M, s);
  }
  return a;
}
