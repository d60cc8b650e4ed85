// Window geometry and index arithmetic of the (shifted-)window layer, shared by
// every kernel of the CUDA library (host and device).
//
// Conventions ("Video Swin Transformer" summary page, Method steps 4-6 and the
// window_msa pseudocode; the code walk-through page, section 1.2):
//   * the token grid (T, H, W) is zero-padded at the high end of every axis to
//     Lp = ceil(L / w) * w, then rolled by -s: rolled coordinate r holds
//     original coordinate o = (r + s) mod Lp;
//   * windows are numbered (b, wt, wh, ww) row-major, slots (pt, ph, pw)
//     row-major inside a window, r = window_index * w + slot_position;
//   * on a shifted axis, rolled coordinate r is in region 0 (r < Lp - w),
//     1 (r < Lp - s) or 2 (otherwise); two slots of one window may attend to
//     each other only when their regions agree on every axis;
//   * relative bias row (dt+P-1)(2Mh-1)(2Mw-1) + (dh+Mh-1)(2Mw-1) + (dw+Mw-1),
//     d = slot position of the query minus that of the key.
#pragma once

#include <cstdint>

namespace vswin {

struct Geom {
  int B, T, H, W, C, heads, d;
  int win[3];   // window (P, Mh, Mw)
  int sh[3];    // shift
  int L[3];     // (T, H, W)
  int Lp[3];    // padded extents
  int nw[3];    // windows per axis
  int nW;       // windows per clip
  int N;        // slots per window
  int Npad;     // N rounded up to 16
  int table_rows;
  long long windows;  // B * nW
  long long tokens;   // B * T * H * W
};

__host__ __device__ inline int ceil_to(int v, int m) { return ((v + m - 1) / m) * m; }

__host__ __device__ inline void slot_position(const Geom& g, int n, int* p) {
  p[2] = n % g.win[2];
  p[1] = (n / g.win[2]) % g.win[1];
  p[0] = n / (g.win[2] * g.win[1]);
}

__host__ __device__ inline void window_position(const Geom& g, int w_in_clip, int* wp) {
  wp[2] = w_in_clip % g.nw[2];
  wp[1] = (w_in_clip / g.nw[2]) % g.nw[1];
  wp[0] = w_in_clip / (g.nw[2] * g.nw[1]);
}

// Flat source token of slot n of global window `win` (b * nW + w), or -1 when
// the slot holds zero padding.
__host__ __device__ inline long long slot_source(const Geom& g, long long win, int n) {
  const int b = (int)(win / g.nW);
  const int w = (int)(win % g.nW);
  int wp[3], p[3];
  window_position(g, w, wp);
  slot_position(g, n, p);
  int o[3];
  for (int a = 0; a < 3; ++a) {
    int r = wp[a] * g.win[a] + p[a] + g.sh[a];
    if (r >= g.Lp[a]) r -= g.Lp[a];
    if (r >= g.L[a]) return -1;
    o[a] = r;
  }
  return (((long long)b * g.T + o[0]) * g.H + o[1]) * g.W + o[2];
}

// slot_source in 32-bit arithmetic, for layers whose window slots (and hence
// tokens) number below 2^31: window `gw` = b * nW + w, slot n.
__host__ __device__ inline int slot_source32(const Geom& g, int gw, int n) {
  const int b = gw / g.nW;
  const int w = gw - b * g.nW;
  int wp[3], p[3];
  window_position(g, w, wp);
  slot_position(g, n, p);
  int o[3];
  for (int a = 0; a < 3; ++a) {
    int r = wp[a] * g.win[a] + p[a] + g.sh[a];
    if (r >= g.Lp[a]) r -= g.Lp[a];
    if (r >= g.L[a]) return -1;
    o[a] = r;
  }
  return ((b * g.T + o[0]) * g.H + o[1]) * g.W + o[2];
}

__host__ __device__ inline int axis_region(int r, int Lp, int w, int s) {
  if (s == 0 || r < Lp - w) return 0;
  return r < Lp - s ? 1 : 2;
}

__host__ __device__ inline int slot_region(const Geom& g, int w_in_clip, int n) {
  int wp[3], p[3];
  window_position(g, w_in_clip, wp);
  slot_position(g, n, p);
  int reg = 0;
  for (int a = 0; a < 3; ++a) reg = reg * 3 + axis_region(wp[a] * g.win[a] + p[a], g.Lp[a], g.win[a], g.sh[a]);
  return reg;
}

__host__ __device__ inline int bias_row(const Geom& g, int i, int j) {
  int pi[3], pj[3];
  slot_position(g, i, pi);
  slot_position(g, j, pj);
  const int nh = 2 * g.win[1] - 1, nww = 2 * g.win[2] - 1;
  return (pi[0] - pj[0] + g.win[0] - 1) * nh * nww + (pi[1] - pj[1] + g.win[1] - 1) * nww +
         (pi[2] - pj[2] + g.win[2] - 1);
}

// Window split flags: on axis a the window sits in the last window column and
// the axis is shifted, so its slots fall in two regions (cut at w - s).
__host__ __device__ inline int window_split_bits(const Geom& g, int w_in_clip) {
  int wp[3];
  window_position(g, w_in_clip, wp);
  int bits = 0;
  for (int a = 0; a < 3; ++a)
    if (g.sh[a] > 0 && wp[a] == g.nw[a] - 1) bits |= 1 << a;
  return bits;
}

}  // namespace vswin
