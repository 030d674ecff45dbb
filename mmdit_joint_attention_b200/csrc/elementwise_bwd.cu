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
// several rows at once; the modulate backward stages its rows in shared
// memory with bulk copies, so that loads stay in flight across those sums.
// HBM-bound: modulate reads x and dy and writes dx; residual reads branch and
// dout and writes dbranch (and dx when asked for: it equals dout).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "../../include/mmdit.h"
#include "internal.h"
#include "ptx.cuh"

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

// Elements of T in one 16-byte chunk.
template <typename T>
__host__ __device__ constexpr int chunk_elems() {
    return 16 / (int)sizeof(T);
}

// Layout of both kernels: a CTA works on one sample and owns a set of rows,
// a few at a time; thread t owns the 16-byte column chunk t of every one of
// those rows (blockDim = the chunks of a row rounded up to a warp).  The
// per-column sums (dshift / dscale, dgate) therefore stay in the owning
// thread's registers over all of the CTA's rows, and reach the [B, C] output
// with one global atomic per column and CTA at the end.  The residual
// backward loads kRows rows into registers before using any, so a CTA keeps
// kRows rows of loads in flight; the modulate backward stages its rows in
// shared memory (below).
constexpr int kRows = 4;

// ---------------------------------------------------------------- modulate bwd
// Rows reach shared memory through bulk copies (one per row of x and of dy)
// into a ring of kStages stages of kRows rows each, issued by thread 0, and
// stay there: both passes over a row read their chunk from shared memory, so
// that no row data is held in registers across the CTA barrier and the
// per-element arithmetic runs on the paired fp32 pipe (two elements per
// instruction).  Pass 1 takes, per row, four moments with the row's first
// element p as a pivot (d = x - p, so that a large common offset does not
// cancel): sum d, sum d^2, sum g and sum g d, g = dy * (1 + scale); one
// CTA-wide sum gives mean = p + sum d / C, the variance, mean_c(g) and
// mean_c(g xh) = rstd (sum g d - (mean - p) sum g) / C.  Pass 2 writes
//   dx = rstd g - rstd mean_c(g) - rstd mean_c(g xh) xh
// and adds dy and dy xh to the column sums.  A stage is refilled at the
// barrier of the next iteration, when no thread reads it any more; two CTAs
// share an SM (C <= 3072 bf16 / 1536 fp32), so one CTA's waits are the
// other's compute time.
// Measured at 480p (C = 3072 bf16): 4 rows x 2 stages 0.140 ms, 2 rows x 3 or
// 4 stages 0.153 ms, rows held in registers across the barrier 0.149 ms.
constexpr int kModRows = 4;                  // rows per iteration (one CTA barrier each)
constexpr int kStages = 2;
constexpr int kMods = 4 * kModRows;          // moments summed per iteration
constexpr int kModBits = kMods == 16 ? 4 : (kMods == 8 ? 3 : 2);
static_assert((1 << kModBits) == kMods, "moments per iteration: 4, 8 or 16");

// Bit 0: a bounded wait expired in an elementwise backward kernel.
__device__ unsigned int g_elem_status = 0;

// Sum of kMods values over the warp: each of the first kModBits steps swaps
// half of the remaining values with the partner lane (xor 16, 8, ...), the
// last steps add the partners' single values, so that lane l ends with the
// warp total of value mod_of_lane(l); the lanes whose low 5 - kModBits bits
// are zero hold one copy of each.
__device__ __forceinline__ int mod_of_lane(int l) {
    int k = 0;
#pragma unroll
    for (int s = 0; s < kModBits; ++s) k |= ((l >> (4 - s)) & 1) << (kModBits - 1 - s);
    return k;
}
__device__ __forceinline__ int lane_of_mod(int k) {
    int l = 0;
#pragma unroll
    for (int s = 0; s < kModBits; ++s) l |= ((k >> (kModBits - 1 - s)) & 1) << (4 - s);
    return l;
}
__device__ __forceinline__ float warp_reduce_scatter(float (&v)[kMods], int lane) {
#pragma unroll
    for (int step = 0; step < kModBits; ++step) {
        const int h = (kMods / 2) >> step, o = 16 >> step;
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int k = 0; k < h; ++k) {
            const float send = up ? v[k] : v[k + h];
            const float keep = up ? v[k + h] : v[k];
            v[k] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    float t = v[0];
#pragma unroll
    for (int o = 16 >> kModBits; o >= 1; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    return t;
}

// The 16-byte chunk of a row as packed fp32 pairs.
template <typename T>
struct Pairs {
    static constexpr int N = chunk_elems<T>() / 2;
};
__device__ __forceinline__ void to_pairs(const uint4& v, uint64_t (&f)[4], __nv_bfloat16) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e)
        f[e] = f2_pack(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xffff0000u));
}
__device__ __forceinline__ void to_pairs(const uint4& v, uint64_t (&f)[2], float) {
    f[0] = f2_pack(__uint_as_float(v.x), __uint_as_float(v.y));
    f[1] = f2_pack(__uint_as_float(v.z), __uint_as_float(v.w));
}
__device__ __forceinline__ uint4 from_pairs(const uint64_t (&f)[4], __nv_bfloat16) {
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        float lo, hi;
        f2_unpack(f[e], lo, hi);
        w[e] = pack_bf16x2(lo, hi);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}
__device__ __forceinline__ uint4 from_pairs(const uint64_t (&f)[2], float) {
    float a, b, c, d;
    f2_unpack(f[0], a, b);
    f2_unpack(f[1], c, d);
    return make_uint4(__float_as_uint(a), __float_as_uint(b), __float_as_uint(c),
                      __float_as_uint(d));
}
__device__ __forceinline__ float pair_sum(uint64_t v) {
    float lo, hi;
    f2_unpack(v, lo, hi);
    return lo + hi;
}
__device__ __forceinline__ uint64_t splat(float v) { return f2_pack(v, v); }

template <typename T, int MAXT>
__global__ void __launch_bounds__(MAXT, MAXT <= 384 ? 2 : 1)
adaln_modulate_bwd_kernel(const T* x, const float* __restrict__ scale, const T* dy, T* dx,
                          float* dshift, float* dscale, int N, int C, float eps,
                          uint64_t wait_ns) {
    constexpr int E = chunk_elems<T>();
    constexpr int NP = Pairs<T>::N;
    extern __shared__ __align__(128) uint8_t ring[];      // [stage][row][x | dy]
    __shared__ float red[2][16 * kMods];
    __shared__ __align__(8) uint64_t full[kStages];
    __shared__ uint32_t abort_flag;
    const int b = blockIdx.y;
    const int c = threadIdx.x;               // this thread's chunk
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, warps = blockDim.x >> 5;
    const bool own = c < C / E;
    const float invC = 1.f / (float)C;
    const uint32_t row_bytes = (uint32_t)C * sizeof(T);
    const size_t sample = (size_t)b * N * (size_t)C;
    // groups of kModRows rows handled by this CTA: n0 = (blockIdx.x + g gridDim.x) kModRows
    const int groups_all = (N + kModRows - 1) / kModRows;
    const int G = groups_all > (int)blockIdx.x
                      ? (groups_all - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x
                      : 0;
    auto stage_row = [&](int st, int r, int which) -> const T* {
        return reinterpret_cast<const T*>(ring +
                                          ((size_t)(st * kModRows + r) * 2 + which) * row_bytes);
    };
    auto issue = [&](int g) {
        const int st = g % kStages;
        const int n0 = (blockIdx.x + g * gridDim.x) * kModRows;
        const int nr = min(kModRows, N - n0);
        mbar_arrive_expect_tx(&full[st], (uint32_t)nr * 2u * row_bytes);
        for (int r = 0; r < nr; ++r) {
            const size_t row = sample + (size_t)(n0 + r) * C;
            bulk_load(const_cast<T*>(stage_row(st, r, 0)), x + row, row_bytes, &full[st]);
            bulk_load(const_cast<T*>(stage_row(st, r, 1)), dy + row, row_bytes, &full[st]);
        }
    };
    if (threadIdx.x == 0) {
        for (int st = 0; st < kStages; ++st) mbar_init(&full[st], 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    int issued = 0;                          // thread 0: groups whose copies were issued
    if (threadIdx.x == 0)
        for (; issued < G && issued < kStages; ++issued) issue(issued);

    uint64_t sc1[NP], ash[NP], asc[NP];      // 1 + scale, dshift and dscale partials (pairs)
#pragma unroll
    for (int k = 0; k < NP; ++k) {
        const float* sp = scale + (size_t)b * C + c * E + 2 * k;
        sc1[k] = own ? f2_pack(1.f + __ldg(sp), 1.f + __ldg(sp + 1)) : 0ull;
        ash[k] = 0ull;
        asc[k] = 0ull;
    }
    for (int g = 0; g < G; ++g) {
        const int st = g % kStages;
        const int n0 = (blockIdx.x + g * gridDim.x) * kModRows;
        if (!mbar_wait_bounded(&full[st], (uint32_t)(g / kStages) & 1u, &abort_flag, wait_ns)) {
            abort_flag = 1;                   // the rows are garbage from here on; no hang
            atomicOr(&g_elem_status, 1u);
        }
        float v[kMods];                      // per row: sum d, sum d^2, sum g, sum g d
#pragma unroll
        for (int r = 0; r < kModRows; ++r) {
            uint64_t a1 = 0ull, a2 = 0ull, ag = 0ull, agd = 0ull;
            if (own && n0 + r < N) {
                const T* sx = stage_row(st, r, 0);
                const uint64_t p2 = splat((float)sx[0]);
                uint64_t fx[NP], fd[NP];
                to_pairs(reinterpret_cast<const uint4*>(sx)[c], fx, T());
                to_pairs(reinterpret_cast<const uint4*>(stage_row(st, r, 1))[c], fd, T());
#pragma unroll
                for (int k = 0; k < NP; ++k) {
                    const uint64_t d = f2_sub(fx[k], p2);
                    const uint64_t gg = f2_mul(fd[k], sc1[k]);
                    a1 = f2_add(a1, d);
                    a2 = f2_fma(d, d, a2);
                    ag = f2_add(ag, gg);
                    agd = f2_fma(gg, d, agd);
                }
            }
            v[4 * r] = pair_sum(a1);
            v[4 * r + 1] = pair_sum(a2);
            v[4 * r + 2] = pair_sum(ag);
            v[4 * r + 3] = pair_sum(agd);
        }
        const float wsum = warp_reduce_scatter(v, lane);
        float* rb = red[g & 1];              // alternate: no warp can still be reading it
        if ((lane & ((32 >> kModBits) - 1)) == 0) rb[warp * kMods + mod_of_lane(lane)] = wsum;
        __syncthreads();                     // also: no thread reads group g - 1's stage any more
        if (threadIdx.x == 0 && g >= 1 && g + kStages - 1 < G && !abort_flag) {
            fence_proxy_async_smem();
            issue(g + kStages - 1);          // into the stage of group g - 1
            ++issued;
        }
        float tot = 0.f;
        for (int w = 0; w < warps; ++w) tot += rb[w * kMods + mod_of_lane(lane)];
#pragma unroll
        for (int r = 0; r < kModRows; ++r) {
            const float s1 = __shfl_sync(0xffffffffu, tot, lane_of_mod(4 * r));
            const float s2 = __shfl_sync(0xffffffffu, tot, lane_of_mod(4 * r + 1));
            const float sg = __shfl_sync(0xffffffffu, tot, lane_of_mod(4 * r + 2));
            const float sgd = __shfl_sync(0xffffffffu, tot, lane_of_mod(4 * r + 3));
            if (!own || n0 + r >= N) continue;
            const float dm = s1 * invC;
            const float rstd = rsqrtf(fmaxf(s2 * invC - dm * dm, 0.f) + eps);
            const float mg = sg * invC;
            const float mgx = rstd * (sgd - dm * sg) * invC;
            const T* sx = stage_row(st, r, 0);
            const uint64_t p2 = splat((float)sx[0]);
            const uint64_t rs2 = splat(rstd);
            const uint64_t nb2 = splat(-dm * rstd);         // xh = d rstd + nb
            const uint64_t k0 = splat(-rstd * mg), k1 = splat(-rstd * mgx);
            uint64_t fx[NP], fd[NP], o[NP];
            to_pairs(reinterpret_cast<const uint4*>(sx)[c], fx, T());
            to_pairs(reinterpret_cast<const uint4*>(stage_row(st, r, 1))[c], fd, T());
#pragma unroll
            for (int k = 0; k < NP; ++k) {
                const uint64_t xh = f2_fma(f2_sub(fx[k], p2), rs2, nb2);
                o[k] = f2_fma(f2_mul(fd[k], sc1[k]), rs2, f2_fma(xh, k1, k0));
                ash[k] = f2_add(ash[k], fd[k]);
                asc[k] = f2_fma(fd[k], xh, asc[k]);
            }
            *reinterpret_cast<uint4*>(dx + sample + (size_t)(n0 + r) * C + (size_t)c * E) =
                from_pairs(o, T());
        }
    }
    if (own) {
#pragma unroll
        for (int k = 0; k < NP; ++k) {
            float lo, hi;
            f2_unpack(ash[k], lo, hi);
            atomicAdd(dshift + (size_t)b * C + c * E + 2 * k, lo);
            atomicAdd(dshift + (size_t)b * C + c * E + 2 * k + 1, hi);
            f2_unpack(asc[k], lo, hi);
            atomicAdd(dscale + (size_t)b * C + c * E + 2 * k, lo);
            atomicAdd(dscale + (size_t)b * C + c * E + 2 * k + 1, hi);
        }
    }
    // after an expired wait, copies may still be landing in this CTA's shared
    // memory: wait for them (bounded) before the CTA exits
    if (threadIdx.x == 0 && abort_flag)
        for (int g = issued > kStages ? issued - kStages : 0; g < issued; ++g)
            mbar_wait_bounded(&full[g % kStages], (uint32_t)(g / kStages) & 1u, nullptr,
                              200000000ull);
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
// Zeroes the fp32 column-sum outputs (a, and b when not null; n floats each)
// before the row kernels add their partial sums into them.
__global__ void __launch_bounds__(256) zero_sums_kernel(float* __restrict__ a,
                                                        float* __restrict__ b, int n) {
    for (int i = blockIdx.x * 256 + threadIdx.x; i < n; i += gridDim.x * 256) {
        a[i] = 0.f;
        if (b) b[i] = 0.f;
    }
}

cudaError_t zero_sums(float* a, float* b, size_t n, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    const unsigned blocks = (unsigned)((n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024);
    zero_sums_kernel<<<blocks, 256, 0, s>>>(a, b, (int)n);
    return cudaGetLastError();
}

template <typename K>
cudaError_t grid_for(K kern, int threads, size_t smem, int B, int N, dim3& grid) {
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem);
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
    // the ring: kStages stages of kModRows rows of x and dy (at most 128 KB:
    // C <= 4096 bf16 or 2048 fp32)
    const size_t smem = (size_t)kStages * kModRows * 2 * C * sizeof(T);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid;
    e = grid_for(kern, threads, smem, B, N, grid);
    if (e != cudaSuccess) return e;
    kern<<<grid, threads, smem, s>>>(static_cast<const T*>(x), scale, static_cast<const T*>(dy),
                                     static_cast<T*>(dx), dshift, dscale, N, C, eps,
                                     wait_timeout_ns());
    return cudaGetLastError();
}

template <typename T>
cudaError_t dispatch_residual_bwd(const void* br, const float* gate, const void* dout, void* dx,
                                  void* dbr, float* dgate, int B, int N, int C, cudaStream_t s) {
    const int threads = threads_for(C, chunk_elems<T>());
    dim3 grid;
    cudaError_t e = grid_for(gated_residual_bwd_kernel<T>, threads, 0, B, N, grid);
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

cudaError_t read_and_clear_elem_status(unsigned int* out) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_elem_status, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_elem_status, &zero, sizeof(unsigned int));
}

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
    cudaError_t e = zero_sums(dshift, dscale, vec / sizeof(float), s);
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
    cudaError_t e = zero_sums(dgate, nullptr, (size_t)B * C, s);
    if (e == cudaSuccess && N > 0)
        e = dt == MMDIT_BF16
                ? dispatch_residual_bwd<__nv_bfloat16>(branch, gate, dout, dx, dbranch, dgate, B,
                                                      N, C, s)
                : dispatch_residual_bwd<float>(branch, gate, dout, dx, dbranch, dgate, B, N, C, s);
    return status_of(e, "gated_residual_bwd");
}
