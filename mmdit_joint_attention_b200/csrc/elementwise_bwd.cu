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
// One warp per row (the row's 16-byte chunks spread over the lanes and held
// in registers between the passes), CTAs of one sample per grid row.  The
// per-(b, c) sums are gathered per CTA in shared memory, then added to the
// [B, C] outputs with one global atomic per column and CTA: the outputs are
// zeroed first, and their last bits depend on the order of those atomics.
// HBM-bound: modulate reads x and dy and writes dx; residual reads branch
// and dout and writes dbranch (and dx when asked for: it equals dout).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "../../include/mmdit.h"
#include "internal.h"

namespace mmdit {
namespace {

constexpr int kThreads = 256;   // 8 warps, one row each at a time

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

// ---------------------------------------------------------------- modulate bwd
template <typename T, int CPL>
__global__ void __launch_bounds__(kThreads)
adaln_modulate_bwd_kernel(const T* x, const float* __restrict__ scale, const T* dy, T* dx,
                          float* dshift, float* dscale, int N, int C, float eps) {
    constexpr int E = chunk_elems<T>();
    extern __shared__ float acc[];          // [0, C): dshift part, [C, 2C): dscale part
    const int b = blockIdx.y;
    for (int i = threadIdx.x; i < 2 * C; i += kThreads) acc[i] = 0.f;
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int nch = C / E;
    const float invC = 1.f / (float)C;
    const float* sc = scale + (size_t)b * C;
    for (int n = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); n < N;
         n += gridDim.x * (kThreads / 32)) {
        const size_t row = ((size_t)b * N + n) * (size_t)C;
        uint4 rx[CPL], rd[CPL];
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const int c = lane + 32 * i;
            if (c < nch) {
                rx[i] = *reinterpret_cast<const uint4*>(x + row + (size_t)c * E);
                rd[i] = *reinterpret_cast<const uint4*>(dy + row + (size_t)c * E);
            }
        }
        // mean, then the centred sum of squares (two passes over the registers)
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            if (lane + 32 * i < nch) {
                float f[8];
                unpack8(rx[i], f, T());
#pragma unroll
                for (int e = 0; e < E; ++e) s += f[e];
            }
        }
        const float mean = warp_sum(s) * invC;
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            if (lane + 32 * i < nch) {
                float f[8];
                unpack8(rx[i], f, T());
#pragma unroll
                for (int e = 0; e < E; ++e) ss += (f[e] - mean) * (f[e] - mean);
            }
        }
        const float rstd = rsqrtf(warp_sum(ss) * invC + eps);
        // mean_c(g), mean_c(g * xh), and this row's share of dshift / dscale
        float mg = 0.f, mgx = 0.f;
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const int c = lane + 32 * i;
            if (c < nch) {
                float fx[8], fd[8];
                unpack8(rx[i], fx, T());
                unpack8(rd[i], fd, T());
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const float xh = (fx[e] - mean) * rstd;
                    const float g = fd[e] * (1.f + __ldg(sc + c * E + e));
                    mg += g;
                    mgx += g * xh;
                    atomicAdd(&acc[c * E + e], fd[e]);
                    atomicAdd(&acc[C + c * E + e], fd[e] * xh);
                }
            }
        }
        mg = warp_sum(mg) * invC;
        mgx = warp_sum(mgx) * invC;
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const int c = lane + 32 * i;
            if (c < nch) {
                float fx[8], fd[8], o[8];
                unpack8(rx[i], fx, T());
                unpack8(rd[i], fd, T());
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const float xh = (fx[e] - mean) * rstd;
                    const float g = fd[e] * (1.f + __ldg(sc + c * E + e));
                    o[e] = rstd * (g - mg - xh * mgx);
                }
                *reinterpret_cast<uint4*>(dx + row + (size_t)c * E) = pack8(o, T());
            }
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < C; i += kThreads) {
        atomicAdd(dshift + (size_t)b * C + i, acc[i]);
        atomicAdd(dscale + (size_t)b * C + i, acc[C + i]);
    }
}

// ---------------------------------------------------------------- residual bwd
template <typename T, int CPL>
__global__ void __launch_bounds__(kThreads)
gated_residual_bwd_kernel(const T* branch, const float* __restrict__ gate, const T* dout,
                          T* dx, T* dbranch, float* dgate, int N, int C) {
    constexpr int E = chunk_elems<T>();
    extern __shared__ float acc[];          // [0, C): dgate part
    const int b = blockIdx.y;
    for (int i = threadIdx.x; i < C; i += kThreads) acc[i] = 0.f;
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int nch = C / E;
    const float* gt = gate + (size_t)b * C;
    for (int n = blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); n < N;
         n += gridDim.x * (kThreads / 32)) {
        const size_t row = ((size_t)b * N + n) * (size_t)C;
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const int c = lane + 32 * i;
            if (c < nch) {
                const uint4 rb = *reinterpret_cast<const uint4*>(branch + row + (size_t)c * E);
                const uint4 rd = *reinterpret_cast<const uint4*>(dout + row + (size_t)c * E);
                float fb[8], fd[8], o[8];
                unpack8(rb, fb, T());
                unpack8(rd, fd, T());
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    o[e] = __ldg(gt + c * E + e) * fd[e];
                    atomicAdd(&acc[c * E + e], fd[e] * fb[e]);
                }
                *reinterpret_cast<uint4*>(dbranch + row + (size_t)c * E) = pack8(o, T());
                if (dx) *reinterpret_cast<uint4*>(dx + row + (size_t)c * E) = rd;
            }
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < C; i += kThreads) atomicAdd(dgate + (size_t)b * C + i, acc[i]);
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

// CTAs per sample: two per SM over the whole grid, no more than the rows need.
dim3 grid_for(int B, int N) {
    long long bx = ((long long)num_sms() * 2 + B - 1) / B;
    const long long need = ((long long)N + 7) / 8;
    if (need < bx) bx = need;
    if (bx < 1) bx = 1;
    return dim3((unsigned)bx, (unsigned)B);
}

template <typename T, int CPL>
cudaError_t run_modulate_bwd(const void* x, const float* scale, const void* dy, void* dx,
                             float* dshift, float* dscale, int B, int N, int C, float eps,
                             cudaStream_t s) {
    const size_t smem = (size_t)C * 8;
    adaln_modulate_bwd_kernel<T, CPL><<<grid_for(B, N), kThreads, smem, s>>>(
        static_cast<const T*>(x), scale, static_cast<const T*>(dy), static_cast<T*>(dx),
        dshift, dscale, N, C, eps);
    return cudaGetLastError();
}

template <typename T, int CPL>
cudaError_t run_residual_bwd(const void* br, const float* gate, const void* dout, void* dx,
                             void* dbr, float* dgate, int B, int N, int C, cudaStream_t s) {
    const size_t smem = (size_t)C * 4;
    gated_residual_bwd_kernel<T, CPL><<<grid_for(B, N), kThreads, smem, s>>>(
        static_cast<const T*>(br), gate, static_cast<const T*>(dout), static_cast<T*>(dx),
        static_cast<T*>(dbr), dgate, N, C);
    return cudaGetLastError();
}

// Chunks of 16 bytes per lane, rounded up to a compiled width.
int cpl_for(int nch) {
    const int need = (nch + 31) / 32;
    return need <= 4 ? 4 : need <= 8 ? 8 : need <= 12 ? 12 : 16;
}

template <typename T>
cudaError_t dispatch_modulate_bwd(const void* x, const float* scale, const void* dy, void* dx,
                                  float* dshift, float* dscale, int B, int N, int C, float eps,
                                  cudaStream_t s) {
    switch (cpl_for(C / chunk_elems<T>())) {
        case 4: return run_modulate_bwd<T, 4>(x, scale, dy, dx, dshift, dscale, B, N, C, eps, s);
        case 8: return run_modulate_bwd<T, 8>(x, scale, dy, dx, dshift, dscale, B, N, C, eps, s);
        case 12: return run_modulate_bwd<T, 12>(x, scale, dy, dx, dshift, dscale, B, N, C, eps, s);
        default: return run_modulate_bwd<T, 16>(x, scale, dy, dx, dshift, dscale, B, N, C, eps, s);
    }
}

template <typename T>
cudaError_t dispatch_residual_bwd(const void* br, const float* gate, const void* dout, void* dx,
                                  void* dbr, float* dgate, int B, int N, int C, cudaStream_t s) {
    switch (cpl_for(C / chunk_elems<T>())) {
        case 4: return run_residual_bwd<T, 4>(br, gate, dout, dx, dbr, dgate, B, N, C, s);
        case 8: return run_residual_bwd<T, 8>(br, gate, dout, dx, dbr, dgate, B, N, C, s);
        case 12: return run_residual_bwd<T, 12>(br, gate, dout, dx, dbr, dgate, B, N, C, s);
        default: return run_residual_bwd<T, 16>(br, gate, dout, dx, dbr, dgate, B, N, C, s);
    }
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
        if (overlaps(dx, x, bytes)) return MMDIT_ERR_ARG;   // dx may replace dy, not x
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
        if (overlaps(dbranch, branch, bytes) || (dx && overlaps(dx, branch, bytes)))
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
