// 3D window partition of the visual token grid (Seaweed-7B report, section
// 3.2: attention restricted to w_t x w_h x w_w windows of the latent grid).
//
// parts[a] windows along axis a of extent X: window k of that axis starts at
// k * (X / parts) + min(k, X % parts), and the first X % parts windows are one
// position longer than the others.
//
// Window-major token order (the layout the window attention reads): windows
// follow one another with the T part slowest and the W part fastest; inside a
// window its tokens keep raster order.  Window (kt, kh, kw) therefore starts at
//   Ts * Hg * Wg + Te * (Hs * Wg + He * Ws)
// where (Ts, Hs, Ws) is its origin and (Te, He, We) its extent.
#pragma once

namespace mmdit {

constexpr int kMaxWindows = 64;

struct WindowGeom {
    int start;         // first window-major token index of the window
    int t0, h0, w0;    // origin in the grid
    int te, he, we;    // extent
};

struct WindowTable {
    int count;         // number of windows (product of the parts)
    int Hg, Wg;        // grid extents of the H and W axes
    WindowGeom w[kMaxWindows];
};

__host__ __device__ inline void axis_part(int k, int extent, int parts, int& start, int& size) {
    const int q = extent / parts, r = extent % parts;
    start = k * q + (k < r ? k : r);
    size = q + (k < r ? 1 : 0);
}

// Requires 1 <= parts[a] <= extent and a product of at most kMaxWindows
// (checked by the C-ABI layer).
inline WindowTable make_window_table(int T, int H, int W, const int parts[3]) {
    WindowTable tab{};
    tab.Hg = H;
    tab.Wg = W;
    int n = 0;
    for (int kt = 0; kt < parts[0]; ++kt) {
        int ts, te;
        axis_part(kt, T, parts[0], ts, te);
        for (int kh = 0; kh < parts[1]; ++kh) {
            int hs, he;
            axis_part(kh, H, parts[1], hs, he);
            for (int kw = 0; kw < parts[2]; ++kw) {
                int ws, we;
                axis_part(kw, W, parts[2], ws, we);
                WindowGeom& g = tab.w[n++];
                g.start = ts * H * W + te * (hs * W + he * ws);
                g.t0 = ts;
                g.h0 = hs;
                g.w0 = ws;
                g.te = te;
                g.he = he;
                g.we = we;
            }
        }
    }
    tab.count = n;
    return tab;
}

// Raster index of the token at window-local index r of window g.
__host__ __device__ inline int window_to_raster(const WindowGeom& g, int r, int Hg, int Wg) {
    const int hw = g.he * g.we;
    const int lt = r / hw;
    const int rem = r - lt * hw;
    const int lh = rem / g.we;
    const int lw = rem - lh * g.we;
    return ((g.t0 + lt) * Hg + g.h0 + lh) * Wg + g.w0 + lw;
}

}  // namespace mmdit
