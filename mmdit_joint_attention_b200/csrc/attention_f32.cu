// Joint (concatenated) non-causal attention in fp32 on the CUDA cores.
//
// Same operation as the tensor-core kernel ("Vimoo 1.0" research page, section
// 2.2: the two streams' Q/K/V are concatenated for joint attention and the
// output is split back; non-causal per the Wan 2.1 report, section 4.3.1), for
// fp32 inputs where the result must stay within 1e-4 of the exact value.
// One warp per query row: each lane holds 4 of the 128 head dims, a score is a
// warp-shuffle sum, and the softmax runs online (running max, rescaled sum and
// accumulator) over the valid keys of the visual stream, then of the
// conditioning stream.
//
// Window mode (Seaweed-7B report, section 3.2, 3D window attention): the
// visual q/k/v are in window-major order (window.h); a visual query row takes
// the visual keys of its own window only (a contiguous range in that order)
// plus the conditioning keys, a conditioning row takes every key, and the
// visual output row is written back at its raster position.
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"

namespace mmdit {
namespace {

__global__ void __launch_bounds__(256)
joint_attn_f32_kernel(const float* __restrict__ qv, const float* __restrict__ kv,
                      const float* __restrict__ vv, const float* __restrict__ qc,
                      const float* __restrict__ kc, const float* __restrict__ vc,
                      const int32_t* __restrict__ ctx_len, float* ov, float* oc,
                      float* __restrict__ lse, int Nv, int Nc, int H, float scale, bool windowed,
                      const __grid_constant__ WindowTable win) {
    const int lane = threadIdx.x & 31;
    const int i = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);  // joint query row
    const int h = blockIdx.y;
    const int b = blockIdx.z;
    if (i >= Nv + Nc) return;
    int L = Nc;
    if (ctx_len) {
        L = ctx_len[b];
        L = L < 0 ? 0 : (L > Nc ? Nc : L);
    }
    const bool vis = i < Nv;
    const size_t qrow = vis ? ((size_t)b * Nv + i) * H + h : ((size_t)b * Nc + (i - Nv)) * H + h;
    int k0 = 0, k1 = Nv;   // visual keys [k0, k1)
    size_t orow = qrow;    // output row
    int jrow = i;          // joint row index of the output (raster order)
    if (windowed && vis) {
        int w = 0;
        while (w + 1 < win.count && win.w[w + 1].start <= i) ++w;
        const WindowGeom& g = win.w[w];
        k0 = g.start;
        k1 = g.start + g.te * g.he * g.we;
        jrow = window_to_raster(g, i - g.start, win.Hg, win.Wg);
        orow = ((size_t)b * Nv + jrow) * H + h;
    }
    float4* dst = reinterpret_cast<float4*>((vis ? ov : oc) + orow * kHeadDim) + lane;
    // lse rows in the order of the inputs (window-major in window mode)
    float* lse_row = lse ? lse + ((size_t)b * H + h) * (size_t)(Nv + Nc) + i : nullptr;
    if (!vis && i - Nv >= L) {  // padded conditioning query: zero output
        *dst = make_float4(0.f, 0.f, 0.f, 0.f);
        if (lse_row && lane == 0) *lse_row = INFINITY;
        return;
    }
    const float4 q = reinterpret_cast<const float4*>((vis ? qv : qc) + qrow * kHeadDim)[lane];
    float m = -INFINITY, l = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int seg = 0; seg < 2; ++seg) {
        const int j0 = seg == 0 ? k0 : 0;
        const int nk = seg == 0 ? k1 : L;
        const float* K = seg == 0 ? kv : kc;
        const float* V = seg == 0 ? vv : vc;
        const int Ns = seg == 0 ? Nv : Nc;
        for (int j = j0; j < nk; ++j) {
            const size_t krow = ((size_t)b * Ns + j) * H + h;
            const float4 k = reinterpret_cast<const float4*>(K + krow * kHeadDim)[lane];
            float d = q.x * k.x + q.y * k.y + q.z * k.z + q.w * k.w;
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
            const float s = d * scale;
            const float mn = fmaxf(m, s);
            const float corr = expf(m - mn);
            const float pj = expf(s - mn);
            const float4 v = reinterpret_cast<const float4*>(V + krow * kHeadDim)[lane];
            l = l * corr + pj;
            acc.x = acc.x * corr + pj * v.x;
            acc.y = acc.y * corr + pj * v.y;
            acc.z = acc.z * corr + pj * v.z;
            acc.w = acc.w * corr + pj * v.w;
            m = mn;
        }
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    *dst = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    if (lse_row && lane == 0) *lse_row = l > 0.f ? m + logf(l) : INFINITY;
}

}  // namespace

cudaError_t launch_joint_attention_f32(const float* qv, const float* kv, const float* vv,
                                       const float* qc, const float* kc, const float* vc,
                                       const int32_t* ctx_len, float* ov, float* oc, float* lse,
                                       int B, int Nv, int Nc, int H, float softmax_scale,
                                       const WindowTable* win, cudaStream_t s) {
    const int rows = Nv + Nc;
    if (rows == 0 || B == 0) return cudaSuccess;
    dim3 grid((rows + 7) / 8, H, B);
    WindowTable tab{};
    if (win) tab = *win;
    joint_attn_f32_kernel<<<grid, 256, 0, s>>>(qv, kv, vv, qc, kc, vc, ctx_len, ov, oc, lse, Nv,
                                               Nc, H, softmax_scale, win != nullptr, tab);
    return cudaGetLastError();
}

}  // namespace mmdit
