// Bandwidth-bound kernels of the block:
//   * fused QK-RMSNorm + 3D RoPE (one read and one write of q and k),
//   * adaLN modulate  y = LN(x) * (1 + scale) + shift,
//   * gated residual  out = x + gate * branch.
// What they compute: "Vimoo 1.0" research page, section 2.2 (QK-RMSNorm within
// each head with distinct learned scales; 3D RoPE over T/H/W with the 128 head
// dims split 16/56/56, visual stream only; LayerNorm with timestep shift and
// scale; gated residual).  The fusion of normalisation and RoPE into one pass
// over memory follows the Seaweed-7B report, section 3.4 "Fused Kernel".
//
// Every kernel moves 16 bytes per thread per access (8 bf16 or 4 fp32) so a
// warp touches whole 128-byte lines, and keeps all arithmetic in fp32.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "internal.h"

namespace mmdit {
namespace {

constexpr unsigned kFull = 0xffffffffu;

template <typename T>
struct Elems;
template <>
struct Elems<__nv_bfloat16> {
    static constexpr int E = 8;  // elements per 16-byte vector
};
template <>
struct Elems<float> {
    static constexpr int E = 4;
};

__device__ __forceinline__ void unpack(const uint4& u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
__device__ __forceinline__ void unpack(const uint4& u, float (&f)[4]) {
    f[0] = __uint_as_float(u.x);
    f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z);
    f[3] = __uint_as_float(u.w);
}
__device__ __forceinline__ uint32_t bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ uint4 pack(const float (&f)[8]) {
    return make_uint4(bf16x2(f[0], f[1]), bf16x2(f[2], f[3]), bf16x2(f[4], f[5]),
                      bf16x2(f[6], f[7]));
}
__device__ __forceinline__ uint4 pack(const float (&f)[4]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
}

// Plain (coherent) 16-byte accesses: outputs may alias inputs.
template <typename T>
__device__ __forceinline__ uint4 ld16(const T* p) {
    return __ldcs(reinterpret_cast<const uint4*>(p));
}
template <typename T>
__device__ __forceinline__ void st16(T* p, const uint4& v) {
    __stcs(reinterpret_cast<uint4*>(p), v);
}

int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    if (!cached[dev]) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        cached[dev] = n > 0 ? n : 148;
    }
    return cached[dev];
}

// ======================================================================
// QK-RMSNorm + 3D RoPE
// ======================================================================

// Unsigned 32-bit division by a run-time constant d >= 1, exact for n < 2^31:
// with l = ceil(log2 d) and m = floor(2^32 (2^l - d) / d) + 1 (computed on the
// host), n / d = (umulhi(n, m) + n) >> l.  (Multiply-high division by an
// invariant integer, Granlund & Montgomery, PLDI 1994.)
struct FastDiv {
    uint32_t d, m, l;
};
FastDiv make_fastdiv(uint32_t d) {
    uint32_t l = 0;
    while ((1ull << l) < d) ++l;
    const uint64_t m = ((1ull << 32) * ((1ull << l) - d)) / d + 1;
    return FastDiv{d, (uint32_t)m, l};
}
__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) {
    return (__umulhi(n, f.m) + n) >> f.l;
}

// One axis of a 3D window partition (see window.h): the first r windows have
// q + 1 positions and cover [0, big), big = r (q + 1); the others have q.
struct AxisSplit {
    uint32_t q, big;
    FastDiv dq1, dq;
};
AxisSplit make_axis_split(int extent, int parts) {
    AxisSplit s;
    s.q = (uint32_t)(extent / parts);
    s.big = (uint32_t)(extent % parts) * (s.q + 1);
    s.dq1 = make_fastdiv(s.q + 1);
    s.dq = make_fastdiv(s.q);
    return s;
}
__device__ __forceinline__ void axis_window(uint32_t x, const AxisSplit& s, uint32_t& start,
                                            uint32_t& ext) {
    if (x < s.big) {
        start = fdiv(x, s.dq1) * (s.q + 1);
        ext = s.q + 1;
    } else {
        start = s.big + fdiv(x - s.big, s.dq) * s.q;
        ext = s.q;
    }
}
// Window-major index of the visual token at grid cell (t, h, w); HW = Hg * Wg.
struct WinMap {
    AxisSplit ax[3];
};
__device__ __forceinline__ uint32_t raster_to_window(uint32_t t, uint32_t h, uint32_t w,
                                                     uint32_t Wg, uint32_t HW, const WinMap& m) {
    uint32_t ts, te, hs, he, ws, we;
    axis_window(t, m.ax[0], ts, te);
    axis_window(h, m.ax[1], hs, he);
    axis_window(w, m.ax[2], ws, we);
    return ts * HW + te * (hs * Wg + he * ws) + ((t - ts) * he + (h - hs)) * we + (w - ws);
}

struct RopeParams {
    FastDiv H, N, HW, W;   // heads, tokens per sample, Hg*Wg, Wg
    WinMap win;            // output order when the kernel permutes to window-major
    int Hg;
    int split[3];
    int off[3];        // first head dim of each axis chunk
    int stride[3];     // table row length of each axis (pairs, rounded up to even)
    int tab_off[3];    // first table entry of each axis
    int tab_entries;
    double pos_scale[3];
    double pos_offset; // text mode: token n sits at pos_offset + n on every axis
    double freq[64];   // frequency of pair j of axis a at index off[a]/2 + j
};

// RoPE modes of the norm kernel
constexpr int kRopeNone = 0;   // conditioning stream without positions
constexpr int kRopeGrid = 1;   // visual stream: (t, h, w) from the token's grid cell
constexpr int kRopeText = 2;   // text tokens, MM-RoPE: one position shared by the three axes

// One group of 128/E lanes owns one (token, head): its q row and its k row.
// Lane g of the group holds head dims [g*E, g*E + E), which lie inside a single
// RoPE axis chunk (the host checks that every chunk boundary is a multiple of
// E), so each lane needs the (cos, sin) of E/2 consecutive pairs of one axis.
// Each warp handles UNR groups of consecutive units per iteration and issues
// all of their loads before any arithmetic, to keep enough bytes in flight.
// 8 units in flight per warp and 2 CTAs of 256 threads per SM measured best at
// 480p (5.5 TB/s, vs 3.6 TB/s with one unit per group and 64-bit index math).
constexpr int kQkUnroll = 8;

// PERM (grid mode only): rows are stored in window-major order instead of in
// place of the input rows.  KONLY: k alone (q is normalised inside the
// attention kernel); q_in / q_out are not touched.
template <typename T, int ROPE, bool TABLE, bool PERM, int UNR, bool KONLY = false>
__global__ void __launch_bounds__(256, 2)
qk_norm_rope_kernel(const T* q_in, const T* k_in, T* q_out, T* k_out,
                    const float* __restrict__ gq, const float* __restrict__ gk, uint32_t units,
                    float eps, const RopeParams rp) {
    constexpr int E = Elems<T>::E;
    constexpr int LPR = kHeadDim / E;  // lanes per row
    constexpr int GPW = 32 / LPR;      // (token, head) units per warp per round
    extern __shared__ float4 rope_tab4[];
    const float2* tab = reinterpret_cast<const float2*>(rope_tab4);

    if (ROPE == kRopeGrid && TABLE) {
        float2* wtab = reinterpret_cast<float2*>(rope_tab4);
        for (int e = threadIdx.x; e < rp.tab_entries; e += blockDim.x) {
            const int a = e < rp.tab_off[1] ? 0 : (e < rp.tab_off[2] ? 1 : 2);
            const int local = e - rp.tab_off[a];
            const int pos = local / rp.stride[a];
            const int j = local - pos * rp.stride[a];
            float c = 1.f, s = 0.f;
            if (j < rp.split[a] / 2) {
                const float ang =
                    (float)((double)pos * rp.pos_scale[a] * rp.freq[rp.off[a] / 2 + j]);
                sincosf(ang, &s, &c);
            }
            wtab[e] = make_float2(c, s);
        }
        __syncthreads();
    }

    const int lane = threadIdx.x & 31;
    const int g = lane % LPR;
    const int grp = lane / LPR;
    const int d0 = g * E;
    float wq[E], wk[E];
#pragma unroll
    for (int i = 0; i < E; ++i) {
        wq[i] = gq[d0 + i];
        wk[i] = gk[d0 + i];
    }
    const int axis = d0 < rp.off[1] ? 0 : (d0 < rp.off[2] ? 1 : 2);
    const int jb = (d0 - rp.off[axis]) >> 1;

    const uint32_t warp0 = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
    for (uint32_t uw = warp0 * (GPW * UNR); uw < units; uw += nwarps * (GPW * UNR)) {
        uint4 rq[UNR], rk[UNR];
#pragma unroll
        for (int r = 0; r < UNR; ++r) {
            const uint32_t u = uw + r * GPW + grp;
            if (u < units) {
                const size_t base = (size_t)u * kHeadDim + d0;
                rq[r] = KONLY ? make_uint4(0, 0, 0, 0) : ld16(q_in + base);
                rk[r] = ld16(k_in + base);
            } else {
                rq[r] = make_uint4(0, 0, 0, 0);
                rk[r] = make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int r = 0; r < UNR; ++r) {
            const uint32_t u = uw + r * GPW + grp;
            float xq[E], xk[E];
            unpack(rq[r], xq);
            unpack(rk[r], xk);
            float sq = 0.f, sk = 0.f;
#pragma unroll
            for (int i = 0; i < E; ++i) {
                sq = fmaf(xq[i], xq[i], sq);
                sk = fmaf(xk[i], xk[i], sk);
            }
#pragma unroll
            for (int o = LPR / 2; o >= 1; o >>= 1) {
                sq += __shfl_xor_sync(kFull, sq, o);
                sk += __shfl_xor_sync(kFull, sk, o);
            }
            const float iq = rsqrtf(sq * (1.0f / kHeadDim) + eps);
            const float ik = rsqrtf(sk * (1.0f / kHeadDim) + eps);
#pragma unroll
            for (int i = 0; i < E; ++i) {
                xq[i] *= iq * wq[i];
                xk[i] *= ik * wk[i];
            }
            uint32_t delta = 0;  // output unit - input unit
            if (ROPE != kRopeNone) {
                const uint32_t uu = u < units ? u : 0;
                const uint32_t bn = fdiv(uu, rp.H);
                const uint32_t n = bn - fdiv(bn, rp.N) * rp.N.d;
                float cs[E];  // (cos, sin) of the lane's E/2 pairs
                if (ROPE == kRopeGrid) {
                    const uint32_t t = fdiv(n, rp.HW);
                    const uint32_t rem = n - t * rp.HW.d;
                    const uint32_t hh = fdiv(rem, rp.W);
                    const uint32_t pos = axis == 0 ? t : (axis == 1 ? hh : rem - hh * rp.W.d);
                    if (PERM)
                        delta = (raster_to_window(t, hh, rem - hh * rp.W.d, rp.W.d, rp.HW.d,
                                                  rp.win) -
                                 n) *
                                rp.H.d;
                    if (TABLE) {
                        const float4* p4 = reinterpret_cast<const float4*>(
                            tab + rp.tab_off[axis] + pos * rp.stride[axis] + jb);
#pragma unroll
                        for (int i = 0; i < E / 4; ++i) {
                            const float4 v = p4[i];
                            cs[4 * i] = v.x;
                            cs[4 * i + 1] = v.y;
                            cs[4 * i + 2] = v.z;
                            cs[4 * i + 3] = v.w;
                        }
                    } else {
#pragma unroll
                        for (int p = 0; p < E / 2; ++p) {
                            const float ang = (float)((double)pos * rp.pos_scale[axis] *
                                                      rp.freq[rp.off[axis] / 2 + jb + p]);
                            sincosf(ang, &cs[2 * p + 1], &cs[2 * p]);
                        }
                    }
                } else {
                    const double pos = rp.pos_offset + (double)n;
#pragma unroll
                    for (int p = 0; p < E / 2; ++p) {
                        const float ang = (float)(pos * rp.freq[rp.off[axis] / 2 + jb + p]);
                        sincosf(ang, &cs[2 * p + 1], &cs[2 * p]);
                    }
                }
#pragma unroll
                for (int p = 0; p < E / 2; ++p) {
                    const float c = cs[2 * p], s = cs[2 * p + 1];
                    const float q0 = xq[2 * p], q1 = xq[2 * p + 1];
                    const float k0 = xk[2 * p], k1 = xk[2 * p + 1];
                    xq[2 * p] = q0 * c - q1 * s;
                    xq[2 * p + 1] = q0 * s + q1 * c;
                    xk[2 * p] = k0 * c - k1 * s;
                    xk[2 * p + 1] = k0 * s + k1 * c;
                }
            }
            if (u < units) {
                const size_t base = (size_t)(u + delta) * kHeadDim + d0;
                if (!KONLY) st16(q_out + base, pack(xq));
                st16(k_out + base, pack(xk));
            }
        }
    }
}

template <typename T, int ROPE, bool TABLE, bool PERM = false, bool KONLY = false>
cudaError_t run_qk(const void* q_in, const void* k_in, void* q_out, void* k_out, const float* gq,
                   const float* gk, uint32_t units, float eps, const RopeParams& rp, size_t smem,
                   cudaStream_t s) {
    // the permuted store next to in-register sin/cos needs more registers
    constexpr int UNR = (PERM && !TABLE) ? kQkUnroll / 2 : kQkUnroll;
    auto kern = qk_norm_rope_kernel<T, ROPE, TABLE, PERM, UNR, KONLY>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
    }
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    constexpr int GPW = 32 / (kHeadDim / Elems<T>::E);
    const long long need = ((long long)units + 8LL * GPW * UNR - 1) / (8LL * GPW * UNR);
    long long blocks = (long long)sm_count() * per_sm;
    if (need < blocks) blocks = need;
    if (blocks < 1) blocks = 1;
    kern<<<(unsigned)blocks, 256, smem, s>>>(
        static_cast<const T*>(q_in), static_cast<const T*>(k_in), static_cast<T*>(q_out),
        static_cast<T*>(k_out), gq, gk, units, eps, rp);
    return cudaGetLastError();
}

// ----------------------------------------------------------------------
// Backward of QK-RMSNorm + RoPE.  For a row x with r = sqrt(mean(x^2) + eps),
// forward y = R (g * x / r), and the upstream gradient dy:
//   u  = R^T dy                      (each pair turned by the opposite angle)
//   dx = g * u / r - x * sum(g * u * x) / (D r^3)
//   dg = sum over rows of u * x / r
// Same lane mapping, angle table and rows-in-flight structure as the forward
// kernel.  Each lane keeps the dg partial sums of its E head dims in registers
// for the whole grid-stride loop; at the end they are summed over the block in
// shared memory and added to dg with one atomic per dim per block (dg is
// zeroed on the stream before the launch).
// ----------------------------------------------------------------------
constexpr int kQkBwdUnroll = 2;   // rows in flight per lane group (x and dy of q and k each)

template <typename T, int ROPE, bool TABLE, int UNR>
__global__ void __launch_bounds__(256, 2)
qk_norm_rope_bwd_kernel(const T* __restrict__ q_in, const T* __restrict__ k_in,
                        const T* __restrict__ dq_out, const T* __restrict__ dk_out,
                        T* __restrict__ dq_in, T* __restrict__ dk_in,
                        const float* __restrict__ gq, const float* __restrict__ gk,
                        float* __restrict__ dgq, float* __restrict__ dgk, uint32_t units,
                        float eps, const RopeParams rp) {
    constexpr int E = Elems<T>::E;
    constexpr int LPR = kHeadDim / E;
    constexpr int GPW = 32 / LPR;
    extern __shared__ float4 rope_tab4[];
    const float2* tab = reinterpret_cast<const float2*>(rope_tab4);
    __shared__ float dg_block[2 * kHeadDim];

    for (int i = threadIdx.x; i < 2 * kHeadDim; i += blockDim.x) dg_block[i] = 0.f;
    if (ROPE == kRopeGrid && TABLE) {
        float2* wtab = reinterpret_cast<float2*>(rope_tab4);
        for (int e = threadIdx.x; e < rp.tab_entries; e += blockDim.x) {
            const int a = e < rp.tab_off[1] ? 0 : (e < rp.tab_off[2] ? 1 : 2);
            const int local = e - rp.tab_off[a];
            const int pos = local / rp.stride[a];
            const int j = local - pos * rp.stride[a];
            float c = 1.f, sn = 0.f;
            if (j < rp.split[a] / 2) {
                const float ang =
                    (float)((double)pos * rp.pos_scale[a] * rp.freq[rp.off[a] / 2 + j]);
                sincosf(ang, &sn, &c);
            }
            wtab[e] = make_float2(c, sn);
        }
    }
    __syncthreads();

    const int lane = threadIdx.x & 31;
    const int g = lane % LPR;
    const int grp = lane / LPR;
    const int d0 = g * E;
    float wq[E], wk[E], aq[E], ak[E];
#pragma unroll
    for (int i = 0; i < E; ++i) {
        wq[i] = gq[d0 + i];
        wk[i] = gk[d0 + i];
        aq[i] = 0.f;
        ak[i] = 0.f;
    }
    const int axis = d0 < rp.off[1] ? 0 : (d0 < rp.off[2] ? 1 : 2);
    const int jb = (d0 - rp.off[axis]) >> 1;

    const uint32_t warp0 = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
    for (uint32_t uw = warp0 * (GPW * UNR); uw < units; uw += nwarps * (GPW * UNR)) {
        uint4 rq[UNR], rk[UNR], rdq[UNR], rdk[UNR];
#pragma unroll
        for (int r = 0; r < UNR; ++r) {
            const uint32_t u = uw + r * GPW + grp;
            const bool live = u < units;
            const size_t base = (size_t)(live ? u : 0) * kHeadDim + d0;
            const uint4 z = make_uint4(0, 0, 0, 0);
            rq[r] = live ? ld16(q_in + base) : z;
            rk[r] = live ? ld16(k_in + base) : z;
            rdq[r] = live ? ld16(dq_out + base) : z;
            rdk[r] = live ? ld16(dk_out + base) : z;
        }
#pragma unroll
        for (int r = 0; r < UNR; ++r) {
            const uint32_t u = uw + r * GPW + grp;
            float xq[E], xk[E], uq[E], uk[E];
            unpack(rq[r], xq);
            unpack(rk[r], xk);
            unpack(rdq[r], uq);
            unpack(rdk[r], uk);
            if (ROPE != kRopeNone) {
                const uint32_t uu = u < units ? u : 0;
                const uint32_t bn = fdiv(uu, rp.H);
                const uint32_t n = bn - fdiv(bn, rp.N) * rp.N.d;
                float cs[E];
                if (ROPE == kRopeText) {
                    // MM-RoPE text position: pos_offset + n on every axis chunk
                    const double tpos = rp.pos_offset + (double)n;
#pragma unroll
                    for (int pp = 0; pp < E / 2; ++pp) {
                        const float ang = (float)(tpos * rp.freq[rp.off[axis] / 2 + jb + pp]);
                        sincosf(ang, &cs[2 * pp + 1], &cs[2 * pp]);
                    }
                } else {
                const uint32_t t = fdiv(n, rp.HW);
                const uint32_t rem = n - t * rp.HW.d;
                const uint32_t hh = fdiv(rem, rp.W);
                const uint32_t pos = axis == 0 ? t : (axis == 1 ? hh : rem - hh * rp.W.d);
                if (TABLE) {
                    const float4* p4 = reinterpret_cast<const float4*>(
                        tab + rp.tab_off[axis] + pos * rp.stride[axis] + jb);
#pragma unroll
                    for (int i = 0; i < E / 4; ++i) {
                        const float4 v = p4[i];
                        cs[4 * i] = v.x;
                        cs[4 * i + 1] = v.y;
                        cs[4 * i + 2] = v.z;
                        cs[4 * i + 3] = v.w;
                    }
                } else {
#pragma unroll
                    for (int pp = 0; pp < E / 2; ++pp) {
                        const float ang = (float)((double)pos * rp.pos_scale[axis] *
                                                  rp.freq[rp.off[axis] / 2 + jb + pp]);
                        sincosf(ang, &cs[2 * pp + 1], &cs[2 * pp]);
                    }
                }
                }
#pragma unroll
                for (int pp = 0; pp < E / 2; ++pp) {
                    const float c = cs[2 * pp], sn = cs[2 * pp + 1];
                    const float q0 = uq[2 * pp], q1 = uq[2 * pp + 1];
                    const float k0 = uk[2 * pp], k1 = uk[2 * pp + 1];
                    uq[2 * pp] = q0 * c + q1 * sn;
                    uq[2 * pp + 1] = q1 * c - q0 * sn;
                    uk[2 * pp] = k0 * c + k1 * sn;
                    uk[2 * pp + 1] = k1 * c - k0 * sn;
                }
            }
            // row sums: mean square of x and sum(g * u * x), for q and k
            float sq = 0.f, sk = 0.f, tq = 0.f, tk = 0.f;
#pragma unroll
            for (int i = 0; i < E; ++i) {
                sq = fmaf(xq[i], xq[i], sq);
                sk = fmaf(xk[i], xk[i], sk);
                tq = fmaf(wq[i] * uq[i], xq[i], tq);
                tk = fmaf(wk[i] * uk[i], xk[i], tk);
            }
#pragma unroll
            for (int o = LPR / 2; o >= 1; o >>= 1) {
                sq += __shfl_xor_sync(kFull, sq, o);
                sk += __shfl_xor_sync(kFull, sk, o);
                tq += __shfl_xor_sync(kFull, tq, o);
                tk += __shfl_xor_sync(kFull, tk, o);
            }
            const float iq = rsqrtf(sq * (1.0f / kHeadDim) + eps);   // 1 / r
            const float ik = rsqrtf(sk * (1.0f / kHeadDim) + eps);
            const float cq = tq * iq * iq * iq * (1.0f / kHeadDim);    // sum(g u x) / (D r^3)
            const float ck = tk * ik * ik * ik * (1.0f / kHeadDim);
            const bool live = u < units;
            float oq[E], ok[E];
#pragma unroll
            for (int i = 0; i < E; ++i) {
                oq[i] = wq[i] * uq[i] * iq - xq[i] * cq;
                ok[i] = wk[i] * uk[i] * ik - xk[i] * ck;
                if (live) {
                    aq[i] = fmaf(uq[i] * xq[i], iq, aq[i]);
                    ak[i] = fmaf(uk[i] * xk[i], ik, ak[i]);
                }
            }
            if (live) {
                const size_t base = (size_t)u * kHeadDim + d0;
                st16(dq_in + base, pack(oq));
                st16(dk_in + base, pack(ok));
            }
        }
    }
    // dg: lanes with the same head dims (g, g + LPR, ...) first, then the block
#pragma unroll
    for (int i = 0; i < E; ++i) {
#pragma unroll
        for (int o = LPR; o < 32; o <<= 1) {
            aq[i] += __shfl_xor_sync(kFull, aq[i], o);
            ak[i] += __shfl_xor_sync(kFull, ak[i], o);
        }
    }
    if (grp == 0) {
#pragma unroll
        for (int i = 0; i < E; ++i) {
            atomicAdd(&dg_block[d0 + i], aq[i]);
            atomicAdd(&dg_block[kHeadDim + d0 + i], ak[i]);
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 2 * kHeadDim; i += blockDim.x)
        atomicAdd(i < kHeadDim ? &dgq[i] : &dgk[i - kHeadDim], dg_block[i]);
}

// ======================================================================
// Row permutation between raster and window-major order
// ======================================================================

// One warp per row of `chunks` 16-byte pieces: forward, row n of sample b
// moves to window-major position perm(n); inverse, position perm(n) moves back
// to n.  Each lane issues all its loads of a row before its stores.
constexpr int kPermUnroll = 4;

__global__ void __launch_bounds__(256)
window_permute_kernel(const uint4* __restrict__ x, uint4* __restrict__ y, uint32_t rows,
                      uint32_t chunks, FastDiv N, FastDiv HW, FastDiv W, WinMap wm, bool inverse) {
    const uint32_t lane = threadIdx.x & 31;
    const uint32_t warp0 = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
    for (uint32_t row = warp0; row < rows; row += nwarps) {
        const uint32_t b = fdiv(row, N);
        const uint32_t n = row - b * N.d;
        const uint32_t t = fdiv(n, HW);
        const uint32_t rem = n - t * HW.d;
        const uint32_t h = fdiv(rem, W);
        const uint32_t other = b * N.d + raster_to_window(t, h, rem - h * W.d, W.d, HW.d, wm);
        const uint4* src = x + (size_t)(inverse ? other : row) * chunks;
        uint4* dst = y + (size_t)(inverse ? row : other) * chunks;
        for (uint32_t c0 = lane; c0 < chunks; c0 += 32 * kPermUnroll) {
            uint4 v[kPermUnroll];
#pragma unroll
            for (int k = 0; k < kPermUnroll; ++k) {
                const uint32_t c = c0 + 32 * k;
                if (c < chunks) v[k] = __ldcs(src + c);
            }
#pragma unroll
            for (int k = 0; k < kPermUnroll; ++k) {
                const uint32_t c = c0 + 32 * k;
                if (c < chunks) __stcs(dst + c, v[k]);
            }
        }
    }
}

// ======================================================================
// adaLN modulate
// ======================================================================

// Pieces of 16 bytes holding (1 + scale) and shift for one 16-byte chunk of x.
template <typename T>
struct ModLayout {
    static constexpr int E = Elems<T>::E;
    static constexpr int PIECES = 2 * E / 4;  // bf16: 4, f32: 2
    // XOR swizzle so the 8 lanes of a quarter-warp, which read the same piece
    // of 8 consecutive chunks, hit 8 different 16-byte bank groups.
    __device__ static __forceinline__ int slot(int c, int k) {
        constexpr int chunks_per_128B = 128 / (PIECES * 16);
        return c * PIECES + (k ^ ((c / chunks_per_128B) & (PIECES - 1)));
    }
};

// One warp per row of C elements.  The row stays in registers (packed), so x
// is read from HBM once; both moments come from one pass over the registers
// and one warp-shuffle reduction.
template <typename T, int CPL>
__device__ __forceinline__ void mod_load(uint4 (&raw)[CPL], const T* x, size_t row, int nch,
                                         int lane) {
    constexpr int E = Elems<T>::E;
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        const int c = lane + 32 * i;
        raw[i] = c < nch ? ld16(x + row + (size_t)c * E) : make_uint4(0, 0, 0, 0);
    }
}

template <typename T, int CPL>
__device__ __forceinline__ void mod_row(const uint4 (&raw)[CPL], T* y, size_t row, int nch,
                                        int lane, float invC, float eps, const float4* mod) {
    using L = ModLayout<T>;
    constexpr int E = L::E;
    constexpr int P = L::PIECES;
    // One pass over the row for both moments, shifted by a pivot (the row's
    // first element) so that E[(x-p)^2] - E[x-p]^2 does not cancel when the
    // row mean is large compared to its spread.
    float pivot;
    {
        float f[E];
        unpack(raw[0], f);
        pivot = __shfl_sync(kFull, f[0], 0);
    }
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        if (lane + 32 * i < nch) {
            float f[E];
            unpack(raw[i], f);
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const float d = f[e] - pivot;
                s1 += d;
                s2 = fmaf(d, d, s2);
            }
        }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        s1 += __shfl_xor_sync(kFull, s1, o);
        s2 += __shfl_xor_sync(kFull, s2, o);
    }
    const float dm = s1 * invC;
    const float var = fmaxf(s2 * invC - dm * dm, 0.f);
    const float mean = pivot + dm;
    const float rstd = rsqrtf(var + eps);
    const float nmr = -mean * rstd;
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        const int c = lane + 32 * i;
        if (c < nch) {
            float f[E];
            unpack(raw[i], f);
            float m[2 * E];
#pragma unroll
            for (int k = 0; k < P; ++k) {
                const float4 v = mod[L::slot(c, k)];
                m[4 * k] = v.x;
                m[4 * k + 1] = v.y;
                m[4 * k + 2] = v.z;
                m[4 * k + 3] = v.w;
            }
#pragma unroll
            for (int e = 0; e < E; ++e) f[e] = fmaf(fmaf(f[e], rstd, nmr), m[e], m[E + e]);
            st16(y + row + (size_t)c * E, pack(f));
        }
    }
}

// The rows of up to two streams (the visual and the conditioning stream of a
// block) in one launch: each CTA works on one (stream, sample) and stages that
// pair's (1 + scale, shift) in shared memory.  A short stream (512 cond rows)
// then rides along with the long one instead of paying a launch of its own.
template <typename T>
struct ModStreams {
    const T* x[2];
    T* y[2];
    const float* shift[2];
    const float* scale[2];
    int N[2];    // rows per sample of each stream (0: stream absent)
    int bx[2];   // CTAs per sample of each stream
    int B;
};

// Two CTAs of 256 threads per SM (about 127 registers, 16 warps): measured
// best at 480p among 1-3 CTAs per SM with and without double-buffered rows.
template <typename T, int CPL>
__global__ void __launch_bounds__(256, 2)
adaln_modulate_kernel(const __grid_constant__ ModStreams<T> a, int C, float eps) {
    using L = ModLayout<T>;
    constexpr int E = L::E;
    constexpr int P = L::PIECES;
    extern __shared__ float4 mod[];
    int id = blockIdx.x;
    int sidx = 0;
    if (id >= a.B * a.bx[0]) {
        id -= a.B * a.bx[0];
        sidx = 1;
    }
    const int b = id / a.bx[sidx];
    const int cx = id - b * a.bx[sidx];
    const float* shift = a.shift[sidx];
    const float* scale = a.scale[sidx];
    const T* x = a.x[sidx];
    T* y = a.y[sidx];
    const int N = a.N[sidx];
    const int nch = C / E;
    for (int idx = threadIdx.x; idx < nch * P; idx += blockDim.x) {
        const int c = idx / P, k = idx - (idx / P) * P;
        float4 v;
        if (k < P / 2) {
            v = *reinterpret_cast<const float4*>(scale + (size_t)b * C + c * E + 4 * k);
            v.x += 1.f;
            v.y += 1.f;
            v.z += 1.f;
            v.w += 1.f;
        } else {
            v = *reinterpret_cast<const float4*>(shift + (size_t)b * C + c * E + 4 * (k - P / 2));
        }
        mod[L::slot(c, k)] = v;
    }
    __syncthreads();

    const int lane = threadIdx.x & 31;
    const int warps = blockDim.x >> 5;
    const float invC = 1.0f / (float)C;
    const int stride = a.bx[sidx] * warps;
    const size_t base = (size_t)b * N * (size_t)C;
    int n = cx * warps + (threadIdx.x >> 5);
    for (; n < N; n += stride) {
        uint4 buf[CPL];
        mod_load<T, CPL>(buf, x, base + (size_t)n * C, nch, lane);
        mod_row<T, CPL>(buf, y, base + (size_t)n * C, nch, lane, invC, eps, mod);
    }
}

// Gated residual followed by the next adaLN modulate, one pass over memory:
//   x' = x + gate[b] * branch   (stored, rounded to T)
//   y  = LN(x') * (1 + scale[b]) + shift[b]
// The statistics use x' as stored (rounded to T), so the result equals the
// two separate kernels run back to back.  One warp per row, as above; gate is
// read through L1, (1 + scale, shift) are staged in shared memory.
template <typename T, int CPL>
__global__ void __launch_bounds__(256, 2)
residual_modulate_kernel(const T* x, const T* br, const float* __restrict__ gate,
                         const float* __restrict__ shift, const float* __restrict__ scale,
                         T* x_out, T* y, int N, int C, float eps) {
    using L = ModLayout<T>;
    constexpr int E = L::E;
    constexpr int P = L::PIECES;
    extern __shared__ float4 mod[];
    const int b = blockIdx.y;
    const int nch = C / E;
    for (int idx = threadIdx.x; idx < nch * P; idx += blockDim.x) {
        const int c = idx / P, k = idx - (idx / P) * P;
        float4 v;
        if (k < P / 2) {
            v = *reinterpret_cast<const float4*>(scale + (size_t)b * C + c * E + 4 * k);
            v.x += 1.f;
            v.y += 1.f;
            v.z += 1.f;
            v.w += 1.f;
        } else {
            v = *reinterpret_cast<const float4*>(shift + (size_t)b * C + c * E + 4 * (k - P / 2));
        }
        mod[L::slot(c, k)] = v;
    }
    __syncthreads();

    const int lane = threadIdx.x & 31;
    const int warps = blockDim.x >> 5;
    const float invC = 1.0f / (float)C;
    const size_t base = (size_t)b * N * (size_t)C;
    const float* g = gate + (size_t)b * C;
    for (int n = blockIdx.x * warps + (threadIdx.x >> 5); n < N; n += gridDim.x * warps) {
        const size_t row = base + (size_t)n * C;
        uint4 raw[CPL], rb[CPL];
        mod_load<T, CPL>(raw, x, row, nch, lane);
        mod_load<T, CPL>(rb, br, row, nch, lane);
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const int c = lane + 32 * i;
            if (c < nch) {
                float fx[E], fb[E];
                unpack(raw[i], fx);
                unpack(rb[i], fb);
#pragma unroll
                for (int k = 0; k < E / 4; ++k) {
                    const float4 gv = __ldg(reinterpret_cast<const float4*>(g + c * E) + k);
                    fx[4 * k] = fmaf(gv.x, fb[4 * k], fx[4 * k]);
                    fx[4 * k + 1] = fmaf(gv.y, fb[4 * k + 1], fx[4 * k + 1]);
                    fx[4 * k + 2] = fmaf(gv.z, fb[4 * k + 2], fx[4 * k + 2]);
                    fx[4 * k + 3] = fmaf(gv.w, fb[4 * k + 3], fx[4 * k + 3]);
                }
                raw[i] = pack(fx);
                st16(x_out + row + (size_t)c * E, raw[i]);
            }
        }
        mod_row<T, CPL>(raw, y, row, nch, lane, invC, eps, mod);
    }
}

template <typename T, int CPL>
cudaError_t run_residual_modulate(const void* x, const void* br, const float* gate,
                                  const float* shift, const float* scale, void* x_out, void* y,
                                  int B, int N, int C, float eps, cudaStream_t s) {
    auto kern = residual_modulate_kernel<T, CPL>;
    const size_t smem = (size_t)C * 8;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
    }
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    long long bx = ((long long)sm_count() * per_sm + B - 1) / B;
    const long long need = (N + 7) / 8;
    if (need < bx) bx = need;
    if (bx < 1) bx = 1;
    dim3 grid((unsigned)bx, (unsigned)B);
    kern<<<grid, 256, smem, s>>>(static_cast<const T*>(x), static_cast<const T*>(br), gate, shift,
                                 scale, static_cast<T*>(x_out), static_cast<T*>(y), N, C, eps);
    return cudaGetLastError();
}

template <typename T, int CPL>
cudaError_t run_modulate(const ModStreamsHost& h, int B, int C, float eps, cudaStream_t s) {
    auto kern = adaln_modulate_kernel<T, CPL>;
    const size_t smem = (size_t)C * 8;  // (1 + scale, shift) per column, fp32
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
    }
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    ModStreams<T> a;
    a.B = B;
    // CTAs of one sample's share of a full wave, split between the streams in
    // proportion to their rows; at least one CTA per present stream and at
    // most one per 8 rows (a row per warp).
    const long long per_sample = std::max<long long>(1, (long long)sm_count() * per_sm / B);
    const long long rows = (long long)h.N[0] + h.N[1];
    for (int k = 0; k < 2; ++k) {
        a.x[k] = static_cast<const T*>(h.x[k]);
        a.y[k] = static_cast<T*>(h.y[k]);
        a.shift[k] = h.shift[k];
        a.scale[k] = h.scale[k];
        a.N[k] = h.N[k];
        long long bx = 0;
        if (h.N[k] > 0) {
            bx = (long long)((double)per_sample * h.N[k] / (double)rows + 0.5);
            bx = std::min<long long>(std::max<long long>(bx, 1), (h.N[k] + 7) / 8);
        }
        a.bx[k] = (int)bx;
    }
    const long long ctas = (long long)B * (a.bx[0] + a.bx[1]);
    if (ctas == 0) return cudaSuccess;
    kern<<<(unsigned)ctas, 256, smem, s>>>(a, C, eps);
    return cudaGetLastError();
}

// ======================================================================
// gated residual
// ======================================================================

template <typename T>
__global__ void __launch_bounds__(256)
gated_residual_kernel(const T* x, const T* br, const float* __restrict__ gate, T* out,
                      long long total, int nch_row, long long nch_sample, int C) {
    constexpr int E = Elems<T>::E;
    const long long stride = (long long)gridDim.x * blockDim.x;
    long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    // two independent chunks per iteration keep more loads in flight
    for (; i + stride < total; i += 2 * stride) {
        const long long i2 = i + stride;
        const uint4 xa = ld16(x + i * E), ba = ld16(br + i * E);
        const uint4 xb = ld16(x + i2 * E), bb = ld16(br + i2 * E);
        const float* ga = gate + (i / nch_sample) * C + (int)(i % nch_row) * E;
        const float* gb = gate + (i2 / nch_sample) * C + (int)(i2 % nch_row) * E;
        float fx[E], fb[E], gx[E], gy[E], fy[E], fz[E];
        unpack(xa, fx);
        unpack(ba, fb);
        unpack(xb, fy);
        unpack(bb, fz);
#pragma unroll
        for (int k = 0; k < E / 4; ++k) {
            const float4 u = __ldg(reinterpret_cast<const float4*>(ga) + k);
            const float4 v = __ldg(reinterpret_cast<const float4*>(gb) + k);
            gx[4 * k] = u.x; gx[4 * k + 1] = u.y; gx[4 * k + 2] = u.z; gx[4 * k + 3] = u.w;
            gy[4 * k] = v.x; gy[4 * k + 1] = v.y; gy[4 * k + 2] = v.z; gy[4 * k + 3] = v.w;
        }
#pragma unroll
        for (int e = 0; e < E; ++e) {
            fx[e] = fmaf(gx[e], fb[e], fx[e]);
            fy[e] = fmaf(gy[e], fz[e], fy[e]);
        }
        st16(out + i * E, pack(fx));
        st16(out + i2 * E, pack(fy));
    }
    if (i < total) {
        const uint4 xa = ld16(x + i * E), ba = ld16(br + i * E);
        const float* ga = gate + (i / nch_sample) * C + (int)(i % nch_row) * E;
        float fx[E], fb[E];
        unpack(xa, fx);
        unpack(ba, fb);
#pragma unroll
        for (int e = 0; e < E; ++e) fx[e] = fmaf(__ldg(ga + e), fb[e], fx[e]);
        st16(out + i * E, pack(fx));
    }
}

template <typename T>
cudaError_t run_residual(const void* x, const void* br, const float* gate, void* out, int B,
                         int N, int C, cudaStream_t s) {
    constexpr int E = Elems<T>::E;
    const int nch_row = C / E;
    const long long nch_sample = (long long)N * nch_row;
    const long long total = (long long)B * nch_sample;
    if (total == 0) return cudaSuccess;
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm,
                                                                  gated_residual_kernel<T>, 256, 0);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    long long blocks = (long long)sm_count() * per_sm;
    const long long need = (total + 255) / 256;
    if (need < blocks) blocks = need;
    gated_residual_kernel<T><<<(unsigned)blocks, 256, 0, s>>>(
        static_cast<const T*>(x), static_cast<const T*>(br), gate, static_cast<T*>(out), total,
        nch_row, nch_sample, C);
    return cudaGetLastError();
}

}  // namespace

// ----------------------------------------------------------------------
cudaError_t launch_qk_norm_rope(const void* q_in, const void* k_in, void* q_out, void* k_out,
                                const float* gq, const float* gk, int B, int N, int H,
                                const RopeGrid* grid, const RopeText* text, const int* win_parts,
                                float eps, bool bf16, cudaStream_t s) {
    const long long units_ll = (long long)B * N * H;
    if (units_ll == 0) return cudaSuccess;
    if (units_ll >= (1LL << 31)) return cudaErrorInvalidValue;  // rejected by the C-ABI layer
    const uint32_t units = (uint32_t)units_ll;
    RopeParams rp{};
    rp.H = make_fastdiv((uint32_t)H);
    rp.N = make_fastdiv((uint32_t)N);
    size_t smem = 0;
    bool table = false;
    if (grid) {
        rp.Hg = grid->H;
        rp.HW = make_fastdiv((uint32_t)grid->H * (uint32_t)grid->W);
        rp.W = make_fastdiv((uint32_t)grid->W);
        const int extent[3] = {grid->T, grid->H, grid->W};
        int off = 0, toff = 0;
        for (int a = 0; a < 3; ++a) {
            rp.split[a] = grid->split[a];
            rp.off[a] = off;
            rp.pos_scale[a] = grid->pos_scale[a];
            const int half = grid->split[a] / 2;
            for (int j = 0; j < half; ++j)
                rp.freq[off / 2 + j] = std::pow(grid->base, -2.0 * j / (double)grid->split[a]);
            rp.stride[a] = (half + 1) & ~1;
            rp.tab_off[a] = toff;
            toff += extent[a] * rp.stride[a];
            off += grid->split[a];
        }
        rp.tab_entries = toff;
        if (win_parts)
            for (int a = 0; a < 3; ++a) rp.win.ax[a] = make_axis_split(extent[a], win_parts[a]);
        smem = (size_t)toff * sizeof(float2);
        table = smem <= 64 * 1024;
        if (!table) smem = 0;
    } else if (text) {
        int off = 0;
        for (int a = 0; a < 3; ++a) {
            rp.split[a] = text->split[a];
            rp.off[a] = off;
            for (int j = 0; j < text->split[a] / 2; ++j)
                rp.freq[off / 2 + j] = std::pow(text->base, -2.0 * j / (double)text->split[a]);
            off += text->split[a];
        }
        rp.pos_offset = text->pos_offset;
        rp.Hg = 1;
        rp.HW = rp.W = make_fastdiv(1);
    } else {
        rp.off[1] = rp.off[2] = kHeadDim;  // every lane on "axis 0", unused
        rp.Hg = 1;
        rp.HW = rp.W = make_fastdiv(1);
    }
#define MMDIT_QK_DISPATCH(T)                                                                   \
    if (!q_in && !grid)                                                                        \
        return run_qk<T, kRopeNone, false, false, true>(q_in, k_in, q_out, k_out, gq, gk, units,  \
                                                       eps, rp, 0, s);                          \
    if (!q_in && table)                                                                        \
        return run_qk<T, kRopeGrid, true, false, true>(q_in, k_in, q_out, k_out, gq, gk, units,   \
                                                      eps, rp, smem, s);                        \
    if (!q_in)                                                                                 \
        return run_qk<T, kRopeGrid, false, false, true>(q_in, k_in, q_out, k_out, gq, gk, units,  \
                                                       eps, rp, 0, s);                          \
    if (text)                                                                                  \
        return run_qk<T, kRopeText, false>(q_in, k_in, q_out, k_out, gq, gk, units, eps, rp, 0, \
                                           s);                                                  \
    if (!grid)                                                                                 \
        return run_qk<T, kRopeNone, false>(q_in, k_in, q_out, k_out, gq, gk, units, eps, rp, 0, \
                                           s);                                                  \
    if (win_parts && table)                                                                    \
        return run_qk<T, kRopeGrid, true, true>(q_in, k_in, q_out, k_out, gq, gk, units, eps, rp, \
                                                smem, s);                                       \
    if (win_parts)                                                                             \
        return run_qk<T, kRopeGrid, false, true>(q_in, k_in, q_out, k_out, gq, gk, units, eps,   \
                                                 rp, 0, s);                                     \
    if (table)                                                                                 \
        return run_qk<T, kRopeGrid, true>(q_in, k_in, q_out, k_out, gq, gk, units, eps, rp,     \
                                          smem, s);                                             \
    return run_qk<T, kRopeGrid, false>(q_in, k_in, q_out, k_out, gq, gk, units, eps, rp, 0, s);
    if (bf16) {
        MMDIT_QK_DISPATCH(__nv_bfloat16)
    }
    MMDIT_QK_DISPATCH(float)
#undef MMDIT_QK_DISPATCH
}

template <typename T, int ROPE, bool TABLE>
cudaError_t run_qk_bwd(const void* q_in, const void* k_in, const void* dq_out, const void* dk_out,
                       const float* gq, const float* gk, void* dq_in, void* dk_in, float* dgq,
                       float* dgk, uint32_t units, float eps, const RopeParams& rp, size_t smem,
                       cudaStream_t s) {
    constexpr int UNR = kQkBwdUnroll;
    auto kern = qk_norm_rope_bwd_kernel<T, ROPE, TABLE, UNR>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
    }
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    constexpr int GPW = 32 / (kHeadDim / Elems<T>::E);
    const long long need = ((long long)units + 8LL * GPW * UNR - 1) / (8LL * GPW * UNR);
    long long blocks = (long long)sm_count() * per_sm;
    if (need < blocks) blocks = need;
    if (blocks < 1) blocks = 1;
    kern<<<(unsigned)blocks, 256, smem, s>>>(
        static_cast<const T*>(q_in), static_cast<const T*>(k_in), static_cast<const T*>(dq_out),
        static_cast<const T*>(dk_out), static_cast<T*>(dq_in), static_cast<T*>(dk_in), gq, gk, dgq,
        dgk, units, eps, rp);
    return cudaGetLastError();
}

cudaError_t launch_qk_norm_rope_bwd(const void* q_in, const void* k_in, const void* dq_out,
                                    const void* dk_out, const float* gq, const float* gk,
                                    void* dq_in, void* dk_in, float* dgq, float* dgk, int B, int N,
                                    int H, const RopeGrid* grid, const RopeText* text, float eps,
                                    bool bf16, cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(dgq, 0, kHeadDim * sizeof(float), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dgk, 0, kHeadDim * sizeof(float), s);
    if (e != cudaSuccess) return e;
    const long long units_ll = (long long)B * N * H;
    if (units_ll == 0) return cudaSuccess;
    const uint32_t units = (uint32_t)units_ll;
    RopeParams rp{};
    rp.H = make_fastdiv((uint32_t)H);
    rp.N = make_fastdiv((uint32_t)N);
    size_t smem = 0;
    bool table = false;
    if (grid) {
        rp.Hg = grid->H;
        rp.HW = make_fastdiv((uint32_t)grid->H * (uint32_t)grid->W);
        rp.W = make_fastdiv((uint32_t)grid->W);
        const int extent[3] = {grid->T, grid->H, grid->W};
        int off = 0, toff = 0;
        for (int a = 0; a < 3; ++a) {
            rp.split[a] = grid->split[a];
            rp.off[a] = off;
            rp.pos_scale[a] = grid->pos_scale[a];
            const int half = grid->split[a] / 2;
            for (int j = 0; j < half; ++j)
                rp.freq[off / 2 + j] = std::pow(grid->base, -2.0 * j / (double)grid->split[a]);
            rp.stride[a] = (half + 1) & ~1;
            rp.tab_off[a] = toff;
            toff += extent[a] * rp.stride[a];
            off += grid->split[a];
        }
        rp.tab_entries = toff;
        smem = (size_t)toff * sizeof(float2);
        table = smem <= 64 * 1024;
        if (!table) smem = 0;
    } else if (text) {
        int off = 0;
        for (int a = 0; a < 3; ++a) {
            rp.split[a] = text->split[a];
            rp.off[a] = off;
            for (int j = 0; j < text->split[a] / 2; ++j)
                rp.freq[off / 2 + j] = std::pow(text->base, -2.0 * j / (double)text->split[a]);
            off += text->split[a];
        }
        rp.pos_offset = text->pos_offset;
        rp.Hg = 1;
        rp.HW = rp.W = make_fastdiv(1);
    } else {
        rp.off[1] = rp.off[2] = kHeadDim;
        rp.Hg = 1;
        rp.HW = rp.W = make_fastdiv(1);
    }
#define MMDIT_QK_BWD(T)                                                                       \
    if (text)                                                                                \
        return run_qk_bwd<T, kRopeText, false>(q_in, k_in, dq_out, dk_out, gq, gk, dq_in, dk_in, \
                                               dgq, dgk, units, eps, rp, 0, s);               \
    if (!grid)                                                                               \
        return run_qk_bwd<T, kRopeNone, false>(q_in, k_in, dq_out, dk_out, gq, gk, dq_in, dk_in, \
                                               dgq, dgk, units, eps, rp, 0, s);               \
    if (table)                                                                               \
        return run_qk_bwd<T, kRopeGrid, true>(q_in, k_in, dq_out, dk_out, gq, gk, dq_in, dk_in,  \
                                              dgq, dgk, units, eps, rp, smem, s);             \
    return run_qk_bwd<T, kRopeGrid, false>(q_in, k_in, dq_out, dk_out, gq, gk, dq_in, dk_in,     \
                                           dgq, dgk, units, eps, rp, 0, s);
    if (bf16) {
        MMDIT_QK_BWD(__nv_bfloat16)
    }
    MMDIT_QK_BWD(float)
#undef MMDIT_QK_BWD
}

cudaError_t launch_adaln_modulate_pair(const ModStreamsHost& h, int B, int C, float eps,
                                       bool bf16, cudaStream_t s) {
    if ((long long)B * ((long long)h.N[0] + h.N[1]) == 0) return cudaSuccess;
    const int E = bf16 ? 8 : 4;
    const int cpl = (C / E + 31) / 32;
#define MMDIT_MOD_CASE(V)                                                          \
    if (cpl <= V)                                                                  \
        return bf16 ? run_modulate<__nv_bfloat16, V>(h, B, C, eps, s)              \
                    : run_modulate<float, V>(h, B, C, eps, s);
    MMDIT_MOD_CASE(1)
    MMDIT_MOD_CASE(2)
    MMDIT_MOD_CASE(4)
    MMDIT_MOD_CASE(8)
    MMDIT_MOD_CASE(12)
    MMDIT_MOD_CASE(16)
#undef MMDIT_MOD_CASE
    return cudaErrorInvalidValue;  // the C-ABI layer rejects such C before this point
}

cudaError_t launch_adaln_modulate(const void* x, const float* shift, const float* scale,
                                  void* y, int B, int N, int C, float eps, bool bf16,
                                  cudaStream_t s) {
    ModStreamsHost h{};
    h.x[0] = x;
    h.y[0] = y;
    h.shift[0] = shift;
    h.scale[0] = scale;
    h.N[0] = N;
    return launch_adaln_modulate_pair(h, B, C, eps, bf16, s);
}

cudaError_t launch_residual_modulate(const void* x, const void* branch, const float* gate,
                                     const float* shift, const float* scale, void* x_out, void* y,
                                     int B, int N, int C, float eps, bool bf16, cudaStream_t s) {
    if ((long long)B * N == 0) return cudaSuccess;
    const int E = bf16 ? 8 : 4;
    const int cpl = (C / E + 31) / 32;
#define MMDIT_RM_CASE(V)                                                                        \
    if (cpl <= V)                                                                               \
        return bf16 ? run_residual_modulate<__nv_bfloat16, V>(x, branch, gate, shift, scale,     \
                                                              x_out, y, B, N, C, eps, s)        \
                    : run_residual_modulate<float, V>(x, branch, gate, shift, scale, x_out, y,  \
                                                      B, N, C, eps, s);
    MMDIT_RM_CASE(1)
    MMDIT_RM_CASE(2)
    MMDIT_RM_CASE(4)
    MMDIT_RM_CASE(8)
    MMDIT_RM_CASE(12)
#undef MMDIT_RM_CASE
    return cudaErrorInvalidValue;  // the C-ABI layer rejects such C before this point
}

cudaError_t launch_gated_residual(const void* x, const void* branch, const float* gate,
                                  void* out, int B, int N, int C, bool bf16, cudaStream_t s) {
    return bf16 ? run_residual<__nv_bfloat16>(x, branch, gate, out, B, N, C, s)
                : run_residual<float>(x, branch, gate, out, B, N, C, s);
}

cudaError_t launch_window_permute(const void* x, void* y, int B, int N, int row_bytes,
                                  const RopeGrid& grid, const int* parts, bool inverse,
                                  cudaStream_t s) {
    const long long rows_ll = (long long)B * N;
    if (rows_ll == 0) return cudaSuccess;
    WinMap wm;
    const int extent[3] = {grid.T, grid.H, grid.W};
    for (int a = 0; a < 3; ++a) wm.ax[a] = make_axis_split(extent[a], parts[a]);
    const uint32_t rows = (uint32_t)rows_ll;
    long long blocks = ((long long)rows + 7) / 8;  // 8 warps per block, one row each
    const long long cap = (long long)sm_count() * 8;
    if (blocks > cap) blocks = cap;
    window_permute_kernel<<<(unsigned)blocks, 256, 0, s>>>(
        static_cast<const uint4*>(x), static_cast<uint4*>(y), rows, (uint32_t)(row_bytes / 16),
        make_fastdiv((uint32_t)N), make_fastdiv((uint32_t)(grid.H * grid.W)),
        make_fastdiv((uint32_t)grid.W), wm, inverse);
    return cudaGetLastError();
}

}  // namespace mmdit
