// Quantisation of the attention operands for the 8-bit joint attention (the
// Wan 2.1 report, section 4.4.3: Int8 for S = Q K^T, FP8 E4M3 for O = P V).
//
//   q: int8 per (sample, token, head) row, k: int8 per block of 128
//      consecutive tokens of one (sample, head); symmetric,
//      scale = max|x| / 127 and code = round-half-even(x / scale), both in
//      fp32, clamped to [-127, 127] (scale 0: codes 0).
//   v: E4M3 per (sample, head, channel) over the valid tokens of both
//      streams, scale = max|v| / 448 (fp32), code = E4M3(v / scale) rounded
//      half-even with saturation (cvt.rn.satfinite).
// Scales are laid out [B, H, blocks] (q: one block per token), so a CTA of
// the attention kernel reads its 128 query scales contiguously.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"

namespace mmdit {
namespace {

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ uint32_t i8_code(float x, float s) {
    float q = s > 0.f ? rintf(x / s) : 0.f;
    q = fminf(fmaxf(q, -127.f), 127.f);
    return (uint32_t)((int)q) & 0xffu;
}

// 8 bf16 -> 8 int8 codes (little-endian bytes in a uint2)
__device__ __forceinline__ uint2 i8_pack(const uint4& v, float s) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t out[2];
#pragma unroll
    for (int h = 0; h < 2; ++h)
        out[h] = i8_code(bf_lo(w[2 * h]), s) | (i8_code(bf_hi(w[2 * h]), s) << 8) |
                 (i8_code(bf_lo(w[2 * h + 1]), s) << 16) | (i8_code(bf_hi(w[2 * h + 1]), s) << 24);
    return make_uint2(out[0], out[1]);
}

__device__ __forceinline__ float absmax8(const uint4& v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) m = fmaxf(m, fmaxf(fabsf(bf_lo(w[i])), fabsf(bf_hi(w[i]))));
    return m;
}

// Per-token int8: 16 lanes per (sample, token, head) row of 128 bf16.
__global__ void __launch_bounds__(256)
quant_rows_kernel(const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ codes,
                  float* __restrict__ scales, int N, int H, uint32_t units) {
    const int lane = threadIdx.x & 31;
    const int g = lane & 15;
    const uint32_t warp0 = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
    for (uint32_t uw = warp0 * 2; uw < units; uw += nwarps * 2) {   // two rows per warp
        const uint32_t u = uw + (lane >> 4);
        const bool live = u < units;
        const uint4 v = live ? __ldcs(reinterpret_cast<const uint4*>(x + (size_t)u * 128) + g)
                             : make_uint4(0, 0, 0, 0);
        float m = absmax8(v);
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const float s = m / 127.0f;
        if (live) {
            reinterpret_cast<uint2*>(codes + (size_t)u * 128)[g] = i8_pack(v, s);
            if (g == 0) {
                const uint32_t h = u % H, bn = u / H, n = bn % N, b = bn / N;
                scales[((size_t)b * H + h) * N + n] = s;
            }
        }
    }
}

// Per-block int8: one CTA per (sample, head, block of 128 tokens); thread t
// covers head dims [8 (t % 16), +8) of rows t / 16 + 16 k, k < 8.
__global__ void __launch_bounds__(256)
quant_blocks_kernel(const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ codes,
                    float* __restrict__ scales, int N, int H) {
    __shared__ float wmax[8];
    const int blk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int nblk = gridDim.x;
    const int g = threadIdx.x & 15, r0 = threadIdx.x >> 4;
    uint4 v[8];
    float m = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int n = blk * 128 + r0 + 16 * k;
        v[k] = n < N ? __ldcs(reinterpret_cast<const uint4*>(
                           x + (((size_t)b * N + n) * H + h) * 128) + g)
                     : make_uint4(0, 0, 0, 0);
        m = fmaxf(m, absmax8(v[k]));
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
    __syncthreads();
    m = wmax[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) m = fmaxf(m, wmax[i]);
    const float s = m / 127.0f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int n = blk * 128 + r0 + 16 * k;
        if (n < N)
            reinterpret_cast<uint2*>(codes + (((size_t)b * N + n) * H + h) * 128)[g] =
                i8_pack(v[k], s);
    }
    if (threadIdx.x == 0) scales[((size_t)b * H + h) * nblk + blk] = s;
}

// max|v| per (sample, head, channel) over the valid tokens of a stream, as
// float bits into amax (non-negative floats order like unsigned integers).
// One CTA per (sample, head, chunk of kVChunk tokens): each thread keeps the
// maxima of its 8 channels in registers, the CTA reduces them in shared
// memory, and 128 atomics per CTA update amax.
constexpr int kVChunk = 1024;

__global__ void __launch_bounds__(256)
v_absmax_kernel(const __nv_bfloat16* __restrict__ v, const int32_t* __restrict__ ctx_len,
                unsigned int* __restrict__ amax, int N, int H) {
    __shared__ float red[16][128];
    const int chunk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    int L = N;
    if (ctx_len) {
        L = ctx_len[b];
        L = L < 0 ? 0 : (L > N ? N : L);
    }
    const int g = threadIdx.x & 15, r0 = threadIdx.x >> 4;
    float m[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const int n_end = min(L, (chunk + 1) * kVChunk);
    for (int n = chunk * kVChunk + r0; n < n_end; n += 16) {
        const uint4 x =
            __ldcs(reinterpret_cast<const uint4*>(v + (((size_t)b * N + n) * H + h) * 128) + g);
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            m[2 * i] = fmaxf(m[2 * i], fabsf(bf_lo(w[i])));
            m[2 * i + 1] = fmaxf(m[2 * i + 1], fabsf(bf_hi(w[i])));
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) red[r0][g * 8 + i] = m[i];
    __syncthreads();
    if (threadIdx.x < 128) {
        float t = red[0][threadIdx.x];
#pragma unroll
        for (int k = 1; k < 16; ++k) t = fmaxf(t, red[k][threadIdx.x]);
        atomicMax(amax + ((size_t)b * H + h) * 128 + threadIdx.x, __float_as_uint(t));
    }
}

__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// E4M3 codes of v with the per-channel scale max|v| / 448 from amax.
__global__ void __launch_bounds__(256)
v_quant_kernel(const __nv_bfloat16* __restrict__ v, const unsigned int* __restrict__ amax,
               uint8_t* __restrict__ codes, int N, int H, uint32_t units) {
    const int lane = threadIdx.x & 31;
    const int g = lane & 15;
    const uint32_t first = ((blockIdx.x * blockDim.x + threadIdx.x) >> 4);
    const uint32_t stride = (gridDim.x * blockDim.x) >> 4;
    for (uint32_t u = first; u < units; u += stride) {
        const uint32_t h = u % H, b = (u / H) / N;
        const uint4 x = __ldcs(reinterpret_cast<const uint4*>(v + (size_t)u * 128) + g);
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
        const unsigned int* am = amax + ((size_t)b * H + h) * 128 + g * 8;
        uint32_t out[2];
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            float f[4];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int i = 2 * p + e;
                const float s0 = __uint_as_float(am[2 * i]) / 448.0f;
                const float s1 = __uint_as_float(am[2 * i + 1]) / 448.0f;
                f[2 * e] = s0 > 0.f ? bf_lo(w[i]) / s0 : 0.f;
                f[2 * e + 1] = s1 > 0.f ? bf_hi(w[i]) / s1 : 0.f;
            }
            out[p] = e4m3x2(f[0], f[1]) | (e4m3x2(f[2], f[3]) << 16);
        }
        reinterpret_cast<uint2*>(codes + (size_t)u * 128)[g] = make_uint2(out[0], out[1]);
    }
}

__global__ void v_scales_kernel(const unsigned int* __restrict__ amax, float* __restrict__ scales,
                                int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) scales[i] = __uint_as_float(amax[i]) / 448.0f;
}

int grid_for(uint32_t units) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    long long blocks = ((long long)units + 15) / 16;   // 16 row units per 256 threads
    if (blocks > 8LL * sms) blocks = 8LL * sms;
    return (int)(blocks < 1 ? 1 : blocks);
}

}  // namespace

cudaError_t launch_quant_int8(const void* x, void* codes, float* scales, int B, int N, int H,
                              int block, cudaStream_t s) {
    const long long units = (long long)B * N * H;
    if (units == 0) return cudaSuccess;
    if (block == 1) {
        quant_rows_kernel<<<grid_for((uint32_t)units), 256, 0, s>>>(
            static_cast<const __nv_bfloat16*>(x), static_cast<uint8_t*>(codes), scales, N, H,
            (uint32_t)units);
    } else {
        const dim3 grid((N + 127) / 128, H, B);
        quant_blocks_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x),
                                                 static_cast<uint8_t*>(codes), scales, N, H);
    }
    return cudaGetLastError();
}

cudaError_t launch_quant_v_e4m3(const void* vv, const void* vc, const int32_t* ctx_len, void* cv,
                                void* cc, float* scales, int B, int Nv, int Nc, int H,
                                cudaStream_t s) {
    // scales first holds max|v| as float bits
    unsigned int* amax = reinterpret_cast<unsigned int*>(scales);
    cudaError_t e = cudaMemsetAsync(amax, 0, (size_t)B * H * 128 * sizeof(float), s);
    if (e != cudaSuccess) return e;
    const uint32_t uv = (uint32_t)((long long)B * Nv * H), uc = (uint32_t)((long long)B * Nc * H);
    if (uv)
        v_absmax_kernel<<<dim3((Nv + kVChunk - 1) / kVChunk, H, B), 256, 0, s>>>(
            static_cast<const __nv_bfloat16*>(vv), nullptr, amax, Nv, H);
    if (uc)
        v_absmax_kernel<<<dim3((Nc + kVChunk - 1) / kVChunk, H, B), 256, 0, s>>>(
            static_cast<const __nv_bfloat16*>(vc), ctx_len, amax, Nc, H);
    if (uv) v_quant_kernel<<<grid_for(uv), 256, 0, s>>>(static_cast<const __nv_bfloat16*>(vv),
                                                        amax, static_cast<uint8_t*>(cv), Nv, H, uv);
    if (uc) v_quant_kernel<<<grid_for(uc), 256, 0, s>>>(static_cast<const __nv_bfloat16*>(vc),
                                                        amax, static_cast<uint8_t*>(cc), Nc, H, uc);
    const int n = B * H * 128;
    v_scales_kernel<<<(n + 255) / 256, 256, 0, s>>>(amax, scales, n);
    return cudaGetLastError();
}

}  // namespace mmdit
