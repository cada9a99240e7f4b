// Host-side Gilbert (generalised Hilbert) order of a T x Hg x W token grid.
//
// Video-BLADE, "Preprocessing: Locality-preserving token rearrangement": tokens are
// reordered along a Gilbert space-filling curve before blocking.  The pages do not
// define the curve; this is our own construction, walked with an explicit stack:
//   box = origin o, major direction a (length P), minor directions b (Q), c (R);
//   the walk enters at o and leaves at o + (P-1) a.
//   Q == R == 1          -> straight run along a;
//   2P > 3 max(Q, R)     -> two halves along a, cut at P/2 (made even when P/2 is
//                           odd and Q or R is even);
//   otherwise            -> with b the longer minor: up along b over [0,P/2) x
//                           [0,Q1), across along a over [0,P) x [Q1,Q), back down
//                           along -b over [P/2,P) x [0,Q1); Q1 = Q/2 rounded up to
//                           even.
//   Top level: major = the longest even side (ties x, y, t), else the longest side.
#include <algorithm>
#include <cstdint>
#include <vector>

namespace asa {

namespace {
struct Box {
  int o[3];
  int a[3];
  int P;
  int b[3];
  int Q;
  int c[3];
  int R;
};

inline void set3(int* dst, int x, int y, int z) {
  dst[0] = x;
  dst[1] = y;
  dst[2] = z;
}
}  // namespace

// out[i] = raster index ((t*Hg + y)*W + x) of the cell at curve position i.
// Returns false if the construction ever meets a box it cannot walk (never for
// sides >= 1; kept as a guard).
bool gilbert_order_host(int T, int Hg, int W, int32_t* out) {
  const int sides[3] = {W, Hg, T};
  int major = -1;
  for (int i = 0; i < 3; ++i)
    if (sides[i] % 2 == 0 && (major < 0 || sides[i] > sides[major])) major = i;
  if (major < 0) {
    major = 0;
    for (int i = 1; i < 3; ++i)
      if (sides[i] > sides[major]) major = i;
  }
  int minor[2], nm = 0;
  for (int i = 0; i < 3; ++i)
    if (i != major) minor[nm++] = i;

  Box top;
  set3(top.o, 0, 0, 0);
  set3(top.a, 0, 0, 0);
  set3(top.b, 0, 0, 0);
  set3(top.c, 0, 0, 0);
  top.a[major] = 1;
  top.P = sides[major];
  top.b[minor[0]] = 1;
  top.Q = sides[minor[0]];
  top.c[minor[1]] = 1;
  top.R = sides[minor[1]];

  std::vector<Box> stack;
  stack.push_back(top);
  int64_t pos = 0;
  while (!stack.empty()) {
    Box x = stack.back();
    stack.pop_back();
    if (x.Q == 1 && x.R == 1) {
      for (int i = 0; i < x.P; ++i) {
        const int cx = x.o[0] + i * x.a[0], cy = x.o[1] + i * x.a[1], ct = x.o[2] + i * x.a[2];
        out[pos++] = (ct * Hg + cy) * W + cx;
      }
      continue;
    }
    if (x.P < 2) return false;
    if (2 * x.P > 3 * std::max(x.Q, x.R)) {
      int P1 = x.P / 2;
      if ((P1 & 1) && ((x.Q & 1) == 0 || (x.R & 1) == 0)) ++P1;
      Box h1 = x, h2 = x;
      h1.P = P1;
      for (int k = 0; k < 3; ++k) h2.o[k] = x.o[k] + P1 * x.a[k];
      h2.P = x.P - P1;
      stack.push_back(h2);  // walked second
      stack.push_back(h1);  // walked first
      continue;
    }
    if (x.R > x.Q) {
      int t[3] = {x.b[0], x.b[1], x.b[2]};
      for (int k = 0; k < 3; ++k) {
        x.b[k] = x.c[k];
        x.c[k] = t[k];
      }
      std::swap(x.Q, x.R);
    }
    int Q1 = x.Q / 2;
    if (Q1 & 1) ++Q1;
    const int P1 = x.P / 2;
    Box up, across, down;
    // up: major b (Q1), minors a (P1), c (R)
    for (int k = 0; k < 3; ++k) {
      up.o[k] = x.o[k];
      up.a[k] = x.b[k];
      up.b[k] = x.a[k];
      up.c[k] = x.c[k];
    }
    up.P = Q1;
    up.Q = P1;
    up.R = x.R;
    // down: starts at o + (P-1) a + (Q1-1) b; major -b (Q1), minors -a (P-P1), c (R)
    for (int k = 0; k < 3; ++k) {
      down.o[k] = x.o[k] + (x.P - 1) * x.a[k] + (Q1 - 1) * x.b[k];
      down.a[k] = -x.b[k];
      down.b[k] = -x.a[k];
      down.c[k] = x.c[k];
    }
    down.P = Q1;
    down.Q = x.P - P1;
    down.R = x.R;
    stack.push_back(down);
    if (Q1 < x.Q) {
      // across: starts at o + Q1 b; major a (P), minors b (Q-Q1), c (R)
      for (int k = 0; k < 3; ++k) {
        across.o[k] = x.o[k] + Q1 * x.b[k];
        across.a[k] = x.a[k];
        across.b[k] = x.b[k];
        across.c[k] = x.c[k];
      }
      across.P = x.P;
      across.Q = x.Q - Q1;
      across.R = x.R;
      stack.push_back(across);
    }
    stack.push_back(up);
  }
  return pos == static_cast<int64_t>(T) * Hg * W;
}

}  // namespace asa
