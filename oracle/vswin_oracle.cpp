// Plain double-precision CPU oracle for 3D (shifted-)window multi-head
// self-attention (Video Swin W-MSA / SW-MSA).
//
// TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the
// benchmark's CPU-baseline leg may load this library. It shares no code,
// header, table or constant with the CUDA library; it is written from the
// method's definitions, step by step, with explicit copies:
//
//   pad -> roll by -shift -> partition -> QKV -> masked softmax(QK^T/sqrt(d)+B)V
//   -> output projection -> reverse partition -> roll by +shift -> un-pad
//
// Sources (by page title and section):
//   [VST]  "Video Swin Transformer" (paper summary page): Method steps 3-6,
//          the window_msa pseudocode, eq. 2, "Paper vs code", "Pitfalls".
//   [CODE] Video Swin code walk-through page (section 1.2): block order
//          LayerNorm, F.pad, torch.roll, window_partition, WindowAttention3D
//          (qkv Linear, q*scale, q@k^T, + relative bias, + mask, softmax, @v,
//          proj Linear), then window reverse, roll back, un-pad.
//   [SWIN] "Swin Transformer" tutorial page: sections 2.2/2.3 (W-MSA,
//          SW-MSA, shift back) and 3.2 (mask built from per-region ids).
//
// Readings taken where the pages are silent or disagree (each is a switch in
// `flags` so that tests can show the alternative changes the answer):
//   * roll direction: content moves toward index 0, out[r] = in[(r+s) mod Lp]
//     ([VST] roll by negate(shift); undone by roll by +shift).
//   * order: pad to window multiples first, then roll over the padded extent
//     ([CODE] lists F.pad before torch.roll; the mask is built on the padded
//     extents); undo as un-roll then un-pad.
//   * masked pairs are excluded from the softmax (p = 0); the code's additive
//     -100 is available as flag VSWIN_ORACLE_MASK_ADD100.
//   * regions: on each shifted axis the rolled coordinate r in [0, Lp) is in
//     region 0 if r < Lp-w, 1 if r < Lp-s, else 2 (the three slices whose
//     tokens were not neighbours before the roll, [VST] Method step 5).
//   * padded tokens are real keys with zero input (not masked).
//   * relative bias index: (dt+P-1)(2Mh-1)(2Mw-1) + (dh+Mh-1)(2Mw-1) + (dw+Mw-1)
//     with d = position(query) - position(key) inside the window; temporal
//     offset outermost ([VST] Method step 8 tiles the 2D table along axis 0).
//   * window order (b, wt, wh, ww) and slot order (pt, ph, pw) row-major;
//     head h owns columns [h*d, (h+1)*d) of each of the q | k | v blocks.
//
// Build: g++ -O2 -fopenmp -shared -fPIC -o liboracle.so vswin_oracle.cpp

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

extern "C" {
enum {
  VSWIN_ORACLE_NO_MASK = 1,        // drop the shifted-window mask
  VSWIN_ORACLE_POS_ROLL = 2,       // roll by +shift instead of -shift
  VSWIN_ORACLE_NO_BIAS = 4,        // drop the relative position bias
  VSWIN_ORACLE_ROLL_THEN_PAD = 8,  // roll the unpadded grid, then pad
  VSWIN_ORACLE_MASK_ADD100 = 16,   // masked pairs get -100 instead of exclusion
};
}

namespace {

struct Geom {
  int B, L[3], C, heads, d;
  int w[3], s[3];
  int Lp[3], nw[3];
  long nW;  // windows per clip
  int N;    // tokens per window
};

int ceil_to(int v, int m) { return ((v + m - 1) / m) * m; }

bool make_geom(int B, int T, int H, int W, int C, int heads, const int* window,
               const int* shift, Geom* g) {
  if (B <= 0 || T <= 0 || H <= 0 || W <= 0 || C <= 0 || heads <= 0) return false;
  if (C % heads != 0) return false;
  g->B = B;
  g->L[0] = T; g->L[1] = H; g->L[2] = W;
  g->C = C; g->heads = heads; g->d = C / heads;
  g->nW = 1;
  g->N = 1;
  for (int a = 0; a < 3; ++a) {
    g->w[a] = window[a];
    g->s[a] = shift[a];
    if (g->w[a] < 1 || g->s[a] < 0 || g->s[a] >= g->w[a]) return false;
    g->Lp[a] = ceil_to(g->L[a], g->w[a]);
    g->nw[a] = g->Lp[a] / g->w[a];
    g->nW *= g->nw[a];
    g->N *= g->w[a];
  }
  return true;
}

// A (B, e0, e1, e2, C) grid stored contiguously, channels last.
struct Grid {
  int B, e[3], C;
  std::vector<double> v;
  Grid(int B_, const int* e_, int C_) : B(B_), C(C_) {
    e[0] = e_[0]; e[1] = e_[1]; e[2] = e_[2];
    v.assign((size_t)B * e[0] * e[1] * e[2] * C, 0.0);
  }
  double* at(int b, int t, int h, int w) {
    return &v[((((size_t)b * e[0] + t) * e[1] + h) * e[2] + w) * C];
  }
};

int mod(int a, int m) { return ((a % m) + m) % m; }

// Zero padding at the high end of every axis up to `ext`.
Grid pad_grid(const Grid& in, const int* ext) {
  Grid out(in.B, ext, in.C);
  for (int b = 0; b < in.B; ++b)
    for (int t = 0; t < in.e[0]; ++t)
      for (int h = 0; h < in.e[1]; ++h)
        for (int w = 0; w < in.e[2]; ++w)
          std::memcpy(out.at(b, t, h, w), const_cast<Grid&>(in).at(b, t, h, w),
                      sizeof(double) * in.C);
  return out;
}

// Keep the first `ext` entries of every axis (inverse of pad_grid).
Grid crop_grid(const Grid& in, const int* ext) {
  Grid out(in.B, ext, in.C);
  for (int b = 0; b < in.B; ++b)
    for (int t = 0; t < ext[0]; ++t)
      for (int h = 0; h < ext[1]; ++h)
        for (int w = 0; w < ext[2]; ++w)
          std::memcpy(out.at(b, t, h, w), const_cast<Grid&>(in).at(b, t, h, w),
                      sizeof(double) * in.C);
  return out;
}

// torch.roll semantics: element at index i moves to index (i + by) mod e.
Grid roll_grid(const Grid& in, const int* by) {
  Grid out(in.B, in.e, in.C);
  for (int b = 0; b < in.B; ++b)
    for (int t = 0; t < in.e[0]; ++t)
      for (int h = 0; h < in.e[1]; ++h)
        for (int w = 0; w < in.e[2]; ++w)
          std::memcpy(out.at(b, mod(t + by[0], in.e[0]), mod(h + by[1], in.e[1]),
                             mod(w + by[2], in.e[2])),
                      const_cast<Grid&>(in).at(b, t, h, w), sizeof(double) * in.C);
  return out;
}

// Region label of a rolled coordinate r on one axis of padded extent Lp.
int axis_region(int r, int Lp, int w, int s) {
  if (s == 0) return 0;
  if (r < Lp - w) return 0;
  if (r < Lp - s) return 1;
  return 2;
}

int bias_index(const Geom& g, const int* pi, const int* pj) {
  const int dt = pi[0] - pj[0], dh = pi[1] - pj[1], dw = pi[2] - pj[2];
  const int nh = 2 * g.w[1] - 1, nwd = 2 * g.w[2] - 1;
  return (dt + g.w[0] - 1) * nh * nwd + (dh + g.w[1] - 1) * nwd + (dw + g.w[2] - 1);
}

void slot_pos(const Geom& g, int n, int* p) {
  p[2] = n % g.w[2];
  p[1] = (n / g.w[2]) % g.w[1];
  p[0] = n / (g.w[2] * g.w[1]);
}

void window_pos(const Geom& g, long win, int* wp) {
  wp[2] = (int)(win % g.nw[2]);
  wp[1] = (int)((win / g.nw[2]) % g.nw[1]);
  wp[0] = (int)(win / ((long)g.nw[2] * g.nw[1]));
}

int slot_region(const Geom& g, long win, int n) {
  int wp[3], p[3];
  window_pos(g, win, wp);
  slot_pos(g, n, p);
  int reg[3];
  for (int a = 0; a < 3; ++a) reg[a] = axis_region(wp[a] * g.w[a] + p[a], g.Lp[a], g.w[a], g.s[a]);
  return 9 * reg[0] + 3 * reg[1] + reg[2];
}

// One window: X (N x C) -> y (N x C). Optionally records the attention
// probabilities of one head into probs (N x N).
void window_layer(const Geom& g, const std::vector<double>& X, long win,
                  const double* Wqkv, const double* bqkv, const double* Wproj,
                  const double* bproj, const double* table, int flags,
                  std::vector<double>& y, int probe_head, double* probs) {
  const int N = g.N, C = g.C, d = g.d, C3 = 3 * C;
  // QKV projection: qkv = X Wqkv + bqkv, Wqkv stored [C][3C].
  std::vector<double> qkv((size_t)N * C3);
  for (int n = 0; n < N; ++n)
    for (int j = 0; j < C3; ++j) {
      double acc = bqkv[j];
      for (int c = 0; c < C; ++c) acc += X[(size_t)n * C + c] * Wqkv[(size_t)c * C3 + j];
      qkv[(size_t)n * C3 + j] = acc;
    }
  const bool shifted = (g.s[0] | g.s[1] | g.s[2]) != 0;
  std::vector<int> region(N);
  for (int n = 0; n < N; ++n) region[n] = slot_region(g, win, n);
  std::vector<int> pos((size_t)N * 3);
  for (int n = 0; n < N; ++n) slot_pos(g, n, &pos[(size_t)n * 3]);

  const double inv_sqrt_d = 1.0 / std::sqrt((double)d);
  std::vector<double> o((size_t)N * C, 0.0);
  std::vector<double> e(N);
  std::vector<char> inc(N);
  for (int h = 0; h < g.heads; ++h) {
    for (int i = 0; i < N; ++i) {
      const double* q = &qkv[(size_t)i * C3 + h * d];
      double m = -INFINITY;
      for (int j = 0; j < N; ++j) {
        const double* k = &qkv[(size_t)j * C3 + C + h * d];
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += q[c] * k[c];
        double v = dot * inv_sqrt_d;
        if (!(flags & VSWIN_ORACLE_NO_BIAS))
          v += table[(size_t)bias_index(g, &pos[(size_t)i * 3], &pos[(size_t)j * 3]) * g.heads + h];
        bool same = !shifted || (flags & VSWIN_ORACLE_NO_MASK) || region[i] == region[j];
        if (!same && (flags & VSWIN_ORACLE_MASK_ADD100)) {
          v += -100.0;
          same = true;
        }
        inc[j] = same;
        e[j] = v;
        if (same && v > m) m = v;
      }
      double sum = 0.0;
      for (int j = 0; j < N; ++j) {
        e[j] = inc[j] ? std::exp(e[j] - m) : 0.0;
        sum += e[j];
      }
      for (int j = 0; j < N; ++j) e[j] /= sum;
      if (probs && h == probe_head)
        for (int j = 0; j < N; ++j) probs[(size_t)i * N + j] = e[j];
      double* oi = &o[(size_t)i * C + h * d];
      for (int j = 0; j < N; ++j) {
        if (e[j] == 0.0) continue;
        const double* v = &qkv[(size_t)j * C3 + 2 * C + h * d];
        for (int c = 0; c < d; ++c) oi[c] += e[j] * v[c];
      }
    }
  }
  // Output projection: y = o Wproj + bproj, Wproj stored [C][C].
  y.assign((size_t)N * C, 0.0);
  for (int n = 0; n < N; ++n)
    for (int j = 0; j < C; ++j) {
      double acc = bproj[j];
      for (int c = 0; c < C; ++c) acc += o[(size_t)n * C + c] * Wproj[(size_t)c * C + j];
      y[(size_t)n * C + j] = acc;
    }
}

void set_threads(int nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
}

}  // namespace

extern "C" {

// Number of OpenMP threads a parallel region started now would use.
int vswin_oracle_max_threads(int nthreads) {
  set_threads(nthreads);
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

// Full layer forward. All tensors are host double arrays:
//   x (B,T,H,W,C), Wqkv [C][3C], bqkv [3C], Wproj [C][C], bproj [C],
//   table [(2P-1)(2Mh-1)(2Mw-1)][heads], out (B,T,H,W,C).
// window/shift are taken literally (no clamping). Returns 0 on success,
// 1 on invalid arguments.
// If probe_* select a window and head, that head's attention probabilities
// (N x N, row = query slot) are written to probs.
int vswin_oracle_forward_ex(const double* x, int B, int T, int H, int W, int C, int heads,
                            const int* window, const int* shift, const double* Wqkv,
                            const double* bqkv, const double* Wproj, const double* bproj,
                            const double* table, double* out, int flags, int nthreads,
                            int probe_b, long probe_window, int probe_head, double* probs) {
  Geom g;
  if (!make_geom(B, T, H, W, C, heads, window, shift, &g)) return 1;
  set_threads(nthreads);
  const int L[3] = {T, H, W};
  Grid xin(B, L, C);
  std::memcpy(xin.v.data(), x, sizeof(double) * xin.v.size());

  const int sneg[3] = {-g.s[0], -g.s[1], -g.s[2]};
  const int spos[3] = {g.s[0], g.s[1], g.s[2]};
  const bool pos_roll = (flags & VSWIN_ORACLE_POS_ROLL) != 0;
  const int* fwd = pos_roll ? spos : sneg;
  const int* bwd = pos_roll ? sneg : spos;

  // Step 1-2: pad to window multiples, then cyclic roll over the padded grid.
  Grid xr = (flags & VSWIN_ORACLE_ROLL_THEN_PAD) ? pad_grid(roll_grid(xin, fwd), g.Lp)
                                                 : roll_grid(pad_grid(xin, g.Lp), fwd);
  Grid yr(B, g.Lp, C);

  const long total = (long)B * g.nW;
#pragma omp parallel for schedule(dynamic, 1)
  for (long bw = 0; bw < total; ++bw) {
    const int b = (int)(bw / g.nW);
    const long win = bw % g.nW;
    int wp[3];
    window_pos(g, win, wp);
    // Step 3: partition -- gather the window's slots from the rolled grid.
    std::vector<double> X((size_t)g.N * C);
    for (int n = 0; n < g.N; ++n) {
      int p[3];
      slot_pos(g, n, p);
      std::memcpy(&X[(size_t)n * C],
                  xr.at(b, wp[0] * g.w[0] + p[0], wp[1] * g.w[1] + p[1], wp[2] * g.w[2] + p[2]),
                  sizeof(double) * C);
    }
    std::vector<double> y;
    const bool probe = probs && b == probe_b && win == probe_window;
    window_layer(g, X, win, Wqkv, bqkv, Wproj, bproj, table, flags, y,
                 probe ? probe_head : -1, probe ? probs : nullptr);
    // Reverse partition into the rolled grid.
    for (int n = 0; n < g.N; ++n) {
      int p[3];
      slot_pos(g, n, p);
      std::memcpy(yr.at(b, wp[0] * g.w[0] + p[0], wp[1] * g.w[1] + p[1], wp[2] * g.w[2] + p[2]),
                  &y[(size_t)n * C], sizeof(double) * C);
    }
  }

  // Undo: roll back, then remove the padding (or the mutant's reverse order).
  Grid yo = (flags & VSWIN_ORACLE_ROLL_THEN_PAD) ? roll_grid(crop_grid(yr, L), bwd)
                                                 : crop_grid(roll_grid(yr, bwd), L);
  std::memcpy(out, yo.v.data(), sizeof(double) * yo.v.size());
  return 0;
}

int vswin_oracle_forward(const double* x, int B, int T, int H, int W, int C, int heads,
                         const int* window, const int* shift, const double* Wqkv,
                         const double* bqkv, const double* Wproj, const double* bproj,
                         const double* table, double* out, int flags, int nthreads) {
  return vswin_oracle_forward_ex(x, B, T, H, W, C, heads, window, shift, Wqkv, bqkv, Wproj,
                                 bproj, table, out, flags, nthreads, -1, -1, -1, nullptr);
}

// Outputs of selected windows only, for spot checks of large layers. For each
// global window index win_list[k] = b * nW + w, writes that window's N x C
// projection output y (slot order, before the reverse partition) to
// y_out + k * N * C. Same arithmetic and readings as vswin_oracle_forward.
int vswin_oracle_forward_windows(const double* x, int B, int T, int H, int W, int C, int heads,
                                 const int* window, const int* shift, const double* Wqkv,
                                 const double* bqkv, const double* Wproj, const double* bproj,
                                 const double* table, const long* win_list, int nlist,
                                 double* y_out, int nthreads) {
  Geom g;
  if (!make_geom(B, T, H, W, C, heads, window, shift, &g)) return 1;
  for (int k = 0; k < nlist; ++k)
    if (win_list[k] < 0 || win_list[k] >= (long)B * g.nW) return 1;
  set_threads(nthreads);
  const int L[3] = {T, H, W};
  Grid xin(B, L, C);
  std::memcpy(xin.v.data(), x, sizeof(double) * xin.v.size());
  const int sneg[3] = {-g.s[0], -g.s[1], -g.s[2]};
  Grid xr = roll_grid(pad_grid(xin, g.Lp), sneg);
#pragma omp parallel for schedule(dynamic, 1)
  for (int k = 0; k < nlist; ++k) {
    const int b = (int)(win_list[k] / g.nW);
    const long win = win_list[k] % g.nW;
    int wp[3];
    window_pos(g, win, wp);
    std::vector<double> X((size_t)g.N * C);
    for (int n = 0; n < g.N; ++n) {
      int p[3];
      slot_pos(g, n, p);
      std::memcpy(&X[(size_t)n * C],
                  xr.at(b, wp[0] * g.w[0] + p[0], wp[1] * g.w[1] + p[1], wp[2] * g.w[2] + p[2]),
                  sizeof(double) * C);
    }
    std::vector<double> y;
    window_layer(g, X, win, Wqkv, bqkv, Wproj, bproj, table, 0, y, -1, nullptr);
    std::memcpy(y_out + (size_t)k * g.N * C, y.data(), sizeof(double) * y.size());
  }
  return 0;
}

// Index maps, built by rolling and partitioning an index tensor exactly as the
// layer moves data:
//   win_src[B*nW*N]: flat source token b*T*H*W + (t*H + h)*W + w, or -1 for a
//                    padding slot;
//   region[nW*N]:    9*rt + 3*rh + rw of each slot (all 0 without shift);
//   bias_idx[N*N]:   relative-position table row used by query slot i, key slot j.
int vswin_oracle_index_maps(int B, int T, int H, int W, const int* window, const int* shift,
                            int* win_src, int* region, int* bias_idx) {
  Geom g;
  if (!make_geom(B, T, H, W, 1, 1, window, shift, &g)) return 1;
  const int L[3] = {T, H, W};
  // The index tensor: one double channel carrying the flat token id (+1 so
  // that zero padding reads back as -1 after the shift by one).
  Grid idx(B, L, 1);
  for (int b = 0; b < B; ++b)
    for (int t = 0; t < T; ++t)
      for (int h = 0; h < H; ++h)
        for (int w = 0; w < W; ++w)
          *idx.at(b, t, h, w) = 1.0 + (double)((((long)b * T + t) * H + h) * W + w);
  const int sneg[3] = {-g.s[0], -g.s[1], -g.s[2]};
  Grid r = roll_grid(pad_grid(idx, g.Lp), sneg);
  for (int b = 0; b < B; ++b)
    for (long win = 0; win < g.nW; ++win) {
      int wp[3];
      window_pos(g, win, wp);
      for (int n = 0; n < g.N; ++n) {
        int p[3];
        slot_pos(g, n, p);
        const double v = *r.at(b, wp[0] * g.w[0] + p[0], wp[1] * g.w[1] + p[1], wp[2] * g.w[2] + p[2]);
        win_src[((size_t)b * g.nW + win) * g.N + n] = (int)v - 1;
      }
    }
  for (long win = 0; win < g.nW; ++win)
    for (int n = 0; n < g.N; ++n) region[(size_t)win * g.N + n] = slot_region(g, win, n);
  for (int i = 0; i < g.N; ++i)
    for (int j = 0; j < g.N; ++j) {
      int pi[3], pj[3];
      slot_pos(g, i, pi);
      slot_pos(g, j, pj);
      bias_idx[(size_t)i * g.N + j] = bias_index(g, pi, pj);
    }
  return 0;
}

}  // extern "C"
