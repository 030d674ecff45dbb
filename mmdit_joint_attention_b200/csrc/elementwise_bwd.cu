// Backward of the adaLN modulate and of the gated residual (the block's
// elementwise steps, "Vimoo 1.0", section 2.2: shift and scale modulate the
// normalised features, a gate weighs each branch before it is added back).
//
// adaLN modulate, y = xh * (1 + scale[b]) + shift[b] with xh = (x - mean) * rstd
// over the C values of a row, for the upstream gradient dy:
//   g  = dy * (1 + scale[b])
//   dx = rstd * (g - mean_c(g) - xh * mean_c(g * xh))
//   dshift[b, c] = sum_n dy,   dscale[b, c] = sum_n dy * xh
// gated residual, out = x + gate[b] * branch, for the upstream gradient dout:
//   dx = dout,  dbranch = gate[b] * dout,  dgate[b, c] = sum_n dout * branch
//
// A CTA works on one sample; each thread owns one 16-byte column chunk of all
// the CTA's rows, so the per-(b, c) sums stay in registers and are added to
// the [B, C] outputs with one global atomic per column and CTA at the end: the
// outputs are zeroed first, and their last bits depend on the order of those
// atomics.  The LayerNorm statistics of a row are CTA-wide sums, taken for
// several rows at once.  HBM-bound: modulate reads x and dy and writes dx;
// residual reads branch and dout and writes dbranch (and dx when asked for:
// it equals dout).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "../../include/mmdit.h"
#include "internal.h"

namespace mmdit {
namespace {

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8], __nv_bfloat16) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        f[2 * e] = __uint_as_float(w[e] << 16);
        f[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
    }
}

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8], float) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8], __nv_bfloat16) {
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
        w[e] = *reinterpret_cast<const uint32_t*>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8], float) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Elements of T in one 16-byte chunk.
template <typename T>
__host__ __device__ constexpr int chunk_elems() {
    return 16 / (int)sizeof(T);
}

// Layout of both kernels: a CTA works on one sample and owns a set of rows,
// kRows at a time; thread t owns the 16-byte column chunk t of every one of
// those rows (blockDim = the chunks of a row rounded up to a warp).  The
// per-column sums (dshift / dscale, dgate) therefore stay in the owning
// thread's registers over all of the CTA's rows, and reach the [B, C] output
// with one global atomic per column and CTA at the end.  kRows rows are loaded
// before any is used, so a CTA keeps kRows rows of loads in flight.
constexpr int kRows = 4;

// Sum over the CTA of V values per thread; every thread gets the totals.
// red: shared scratch of (warps * V) floats, one array per call site so that
// consecutive reductions never overwrite values still being read.
template <int V>
__device__ __forceinline__ void cta_sum(float (&v)[V], float* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, warps = blockDim.x >> 5;
#pragma unroll
    for (int k = 0; k < V; ++k) v[k] = warp_sum(v[k]);
    if (lane == 0)
#pragma unroll
        for (int k = 0; k < V; ++k) red[warp * V + k] = v[k];
    __syncthreads();
#pragma unroll
    for (int k = 0; k < V; ++k) v[k] = 0.f;
    for (int w = 0; w < warps; ++w)
#pragma unroll
        for (int k = 0; k < V; ++k) v[k] += red[w * V + k];
}

// ---------------------------------------------------------------- modulate bwd
// Per row: both moments in one pass, shifted by the row's first element (so a
// large common offset does not cancel), one CTA reduction for the kRows rows
// of an iteration; then mean_c(g) and mean_c(g * xh), a second reduction.
// MAXT: the largest block the instantiation serves (384 threads leave room
// for 168 registers a thread, which C <= 3072 bf16 needs without spilling).
template <typename T, int MAXT>
__global__ void __launch_bounds__(MAXT)
adaln_modulate_bwd_kernel(const T* x, const float* __restrict__ scale, const T* dy, T* dx,
                          float* dshift, float* dscale, int N, int C, float eps) {
    constexpr int E = chunk_elems<T>();
    __shared__ float red0[16 * 2 * kRows], red1[16 * 2 * kRows];
    const int b = blockIdx.y;
    const int c = threadIdx.x;               // this thread's chunk
    const bool own = c < C / E;
    const float invC = 1.f / (float)C;
    float sc1[E], ash[E], asc[E];            // 1 + scale, dshift and dscale partials
#pragma unroll
    for (int e = 0; e < E; ++e) {
        sc1[e] = own ? 1.f + __ldg(scale + (size_t)b * C + c * E + e) : 0.f;
        ash[e] = 0.f;
        asc[e] = 0.f;
    }
    const size_t sample = (size_t)b * N * (size_t)C;
    for (int n0 = blockIdx.x * kRows; n0 < N; n0 += gridDim.x * kRows) {
        uint4 rx[kRows], rd[kRows];
        float pivot[kRows];
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
            const bool row_ok = n0 + r < N;
            const size_t row = sample + (size_t)(row_ok ? n0 + r : n0) * C;
            rx[r] = make_uint4(0, 0, 0, 0);
            rd[r] = make_uint4(0, 0, 0, 0);
            if (own && row_ok) {
                rx[r] = *reinterpret_cast<const uint4*>(x + row + (size_t)c * E);
                rd[r] = *reinterpret_cast<const uint4*>(dy + row + (size_t)c * E);
            }
            pivot[r] = row_ok ? (float)x[row] : 0.f;
        }
        float st[2 * kRows];                 // per row: sum(x - p), sum((x - p)^2)
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
            float f[8];
            unpack8(rx[r], f, T());
            float s1 = 0.f, s2 = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const float d = own ? f[e] - pivot[r] : 0.f;
                s1 += d;
                s2 = fmaf(d, d, s2);
            }
            st[2 * r] = s1;
            st[2 * r + 1] = s2;
        }
        cta_sum(st, red0);
        float mean[kRows], rstd[kRows], gm[2 * kRows];   // gm: per row sum(g), sum(g * xh)
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
            const float dm = st[2 * r] * invC;
            mean[r] = pivot[r] + dm;
            rstd[r] = rsqrtf(fmaxf(st[2 * r + 1] * invC - dm * dm, 0.f) + eps);
            float fx[8], fd[8];
            unpack8(rx[r], fx, T());
            unpack8(rd[r], fd, T());
            float a = 0.f, bgx = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const float xh = (fx[e] - mean[r]) * rstd[r];
                const float g = fd[e] * sc1[e];
                a += g;
                bgx = fmaf(g, xh, bgx);
            }
            gm[2 * r] = a;
            gm[2 * r + 1] = bgx;
        }
        cta_sum(gm, red1);
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
            if (!own || n0 + r >= N) continue;
            const float mg = gm[2 * r] * invC, mgx = gm[2 * r + 1] * invC;
            float fx[8], fd[8], o[8];
            unpack8(rx[r], fx, T());
            unpack8(rd[r], fd, T());
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const float xh = (fx[e] - mean[r]) * rstd[r];
                o[e] = rstd[r] * (fd[e] * sc1[e] - mg - xh * mgx);
                ash[e] += fd[e];
                asc[e] = fmaf(fd[e], xh, asc[e]);
            }
            *reinterpret_cast<uint4*>(dx + sample + (size_t)(n0 + r) * C + (size_t)c * E) =
                pack8(o, T());
        }
    }
    if (own) {
#pragma unroll
        for (int e = 0; e < E; ++e) {
            atomicAdd(dshift + (size_t)b * C + c * E + e, ash[e]);
            atomicAdd(dscale + (size_t)b * C + c * E + e, asc[e]);
        }
    }
}

// ---------------------------------------------------------------- residual bwd
template <typename T>
__global__ void __launch_bounds__(512)
gated_residual_bwd_kernel(const T* branch, const float* __restrict__ gate, const T* dout,
                          T* dx, T* dbranch, float* dgate, int N, int C) {
    constexpr int E = chunk_elems<T>();
    const int b = blockIdx.y;
    const int c = threadIdx.x;
    if (c >= C / E) return;                 // no barrier below: idle threads may leave
    float g[E], acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        g[e] = __ldg(gate + (size_t)b * C + c * E + e);
        acc[e] = 0.f;
    }
    const size_t sample = (size_t)b * N * (size_t)C;
    for (int n0 = blockIdx.x * kRows; n0 < N; n0 += gridDim.x * kRows) {
        uint4 rb[kRows], rd[kRows];
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
            if (n0 + r < N) {
                const size_t at = sample + (size_t)(n0 + r) * C + (size_t)c * E;
                rb[r] = *reinterpret_cast<const uint4*>(branch + at);
                rd[r] = *reinterpret_cast<const uint4*>(dout + at);
            }
        }
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
            if (n0 + r >= N) continue;
            const size_t at = sample + (size_t)(n0 + r) * C + (size_t)c * E;
            float fb[8], fd[8], o[8];
            unpack8(rb[r], fb, T());
            unpack8(rd[r], fd, T());
#pragma unroll
            for (int e = 0; e < E; ++e) {
                o[e] = g[e] * fd[e];
                acc[e] = fmaf(fd[e], fb[e], acc[e]);
            }
            *reinterpret_cast<uint4*>(dbranch + at) = pack8(o, T());
            if (dx) *reinterpret_cast<uint4*>(dx + at) = rd[r];
        }
    }
#pragma unroll
    for (int e = 0; e < E; ++e) atomicAdd(dgate + (size_t)b * C + c * E + e, acc[e]);
}

int num_sms() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
    if (!cached[dev]) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        cached[dev] = n > 0 ? n : 148;
    }
    return cached[dev];
}

// Threads of a CTA: one per 16-byte chunk of a row, rounded up to a warp.
int threads_for(int C, int E) { return ((C / E + 31) / 32) * 32; }

// CTAs per sample: as many as the SMs hold at once (occupancy of the kernel at
// this block size), but at least 4 * kRows rows per CTA so that the final
// atomics stay few against the rows.
template <typename K>
cudaError_t grid_for(K kern, int threads, int B, int N, dim3& grid) {
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, 0);
    if (e != cudaSuccess) return e;
    long long bx = ((long long)num_sms() * (per_sm > 0 ? per_sm : 1) + B - 1) / B;
    const long long need = ((long long)N + 4 * kRows - 1) / (4 * kRows);
    if (need < bx) bx = need;
    if (bx < 1) bx = 1;
    grid = dim3((unsigned)bx, (unsigned)B);
    return cudaSuccess;
}

template <typename T>
cudaError_t dispatch_modulate_bwd(const void* x, const float* scale, const void* dy, void* dx,
                                  float* dshift, float* dscale, int B, int N, int C, float eps,
                                  cudaStream_t s) {
    const int threads = threads_for(C, chunk_elems<T>());
    auto kern = threads <= 384 ? adaln_modulate_bwd_kernel<T, 384>
                               : adaln_modulate_bwd_kernel<T, 512>;
    dim3 grid;
    cudaError_t e = grid_for(kern, threads, B, N, grid);
    if (e != cudaSuccess) return e;
    kern<<<grid, threads, 0, s>>>(static_cast<const T*>(x), scale, static_cast<const T*>(dy),
                                  static_cast<T*>(dx), dshift, dscale, N, C, eps);
    return cudaGetLastError();
}

template <typename T>
cudaError_t dispatch_residual_bwd(const void* br, const float* gate, const void* dout, void* dx,
                                  void* dbr, float* dgate, int B, int N, int C, cudaStream_t s) {
    const int threads = threads_for(C, chunk_elems<T>());
    dim3 grid;
    cudaError_t e = grid_for(gated_residual_bwd_kernel<T>, threads, B, N, grid);
    if (e != cudaSuccess) return e;
    gated_residual_bwd_kernel<T><<<grid, threads, 0, s>>>(
        static_cast<const T*>(br), gate, static_cast<const T*>(dout), static_cast<T*>(dx),
        static_cast<T*>(dbr), dgate, N, C);
    return cudaGetLastError();
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, const void* b, size_t n) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + n && y < x + n;
}

int status_of(cudaError_t e, const char* where) {
    if (e == cudaSuccess) return MMDIT_OK;
    set_last_error(where, (int)e);
    return MMDIT_ERR_CUDA;
}

// Shared checks of both entry points: MMDIT_OK, or the error to return.
int check_sizes(int B, int N, int C, mmdit_dtype dt) {
    if ((dt != MMDIT_F32 && dt != MMDIT_BF16) || B < 0 || N < 0 || C < 0) return MMDIT_ERR_ARG;
    if (C == 0 || C % 8 != 0 || C / (dt == MMDIT_BF16 ? 8 : 4) > 512) return MMDIT_ERR_UNSUPPORTED;
    if (B > 65535 || (long long)B * N * C >= (1LL << 40)) return MMDIT_ERR_UNSUPPORTED;
    return MMDIT_OK;
}

}  // namespace
}  // namespace mmdit

using namespace mmdit;

extern "C" int mmdit_adaln_modulate_bwd(const void* x, const float* scale, const void* dy,
                                        void* dx, float* dshift, float* dscale, int B, int N,
                                        int C, float eps, mmdit_dtype dt, void* stream) {
    int r = check_sizes(B, N, C, dt);
    if (r != MMDIT_OK) return r;
    if (!(eps >= 0.f) || !std::isfinite(eps)) return MMDIT_ERR_ARG;
    if (B == 0) return MMDIT_OK;
    if (!scale || !dshift || !dscale) return MMDIT_ERR_ARG;
    if (!al16(scale) || !al16(dshift) || !al16(dscale)) return MMDIT_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t vec = (size_t)B * C * sizeof(float);
    if (N > 0) {
        if (!x || !dy || !dx) return MMDIT_ERR_ARG;
        if (!al16(x) || !al16(dy) || !al16(dx)) return MMDIT_ERR_ALIGN;
        const size_t bytes = (size_t)B * N * C * (dt == MMDIT_BF16 ? 2 : 4);
        // dx may replace dy exactly (a thread reads its chunks of a row before
        // writing them), but must not overlap x or be shifted against dy
        if (overlaps(dx, x, bytes) || (dx != dy && overlaps(dx, dy, bytes)))
            return MMDIT_ERR_ARG;
    }
    cudaError_t e = cudaMemsetAsync(dshift, 0, vec, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dscale, 0, vec, s);
    if (e == cudaSuccess && N > 0)
        e = dt == MMDIT_BF16
                ? dispatch_modulate_bwd<__nv_bfloat16>(x, scale, dy, dx, dshift, dscale, B, N, C,
                                                      eps, s)
                : dispatch_modulate_bwd<float>(x, scale, dy, dx, dshift, dscale, B, N, C, eps, s);
    return status_of(e, "adaln_modulate_bwd");
}

extern "C" int mmdit_gated_residual_bwd(const void* branch, const float* gate, const void* dout,
                                        void* dx, void* dbranch, float* dgate, int B, int N,
                                        int C, mmdit_dtype dt, void* stream) {
    int r = check_sizes(B, N, C, dt);
    if (r != MMDIT_OK) return r;
    if (B == 0) return MMDIT_OK;
    if (!gate || !dgate) return MMDIT_ERR_ARG;
    if (!al16(gate) || !al16(dgate)) return MMDIT_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (N > 0) {
        if (!branch || !dout || !dbranch) return MMDIT_ERR_ARG;
        if (!al16(branch) || !al16(dout) || !al16(dbranch) || (dx && !al16(dx)))
            return MMDIT_ERR_ALIGN;
        const size_t bytes = (size_t)B * N * C * (dt == MMDIT_BF16 ? 2 : 4);
        // outputs: not over branch, not over each other, and over dout only
        // exactly (a thread reads its chunk of dout before writing there)
        if (overlaps(dbranch, branch, bytes) || (dx && overlaps(dx, branch, bytes)) ||
            (dx && overlaps(dx, dbranch, bytes)) ||
            (dbranch != dout && overlaps(dbranch, dout, bytes)) ||
            (dx && dx != dout && overlaps(dx, dout, bytes)))
            return MMDIT_ERR_ARG;
    }
    cudaError_t e = cudaMemsetAsync(dgate, 0, (size_t)B * C * sizeof(float), s);
    if (e == cudaSuccess && N > 0)
        e = dt == MMDIT_BF16
                ? dispatch_residual_bwd<__nv_bfloat16>(branch, gate, dout, dx, dbranch, dgate, B,
                                                      N, C, s)
                : dispatch_residual_bwd<float>(branch, gate, dout, dx, dbranch, dgate, B, N, C, s);
    return status_of(e, "gated_residual_bwd");
}
