// Backward of the joint (concatenated) attention: bf16 in / bf16 out on the
// sm_100a tensor cores, and an fp32 version on the CUDA cores.
//
// What it computes: the reverse-mode derivative of the joint attention of the
// "Vimoo 1.0" research page, section 2.2 (the Seaweed-7B report, section 3.4,
// trains forward and backward of this attention).  With s_ij = scale q_i.k_j
// over valid keys, P = softmax_j(s), O = P V, the upstream gradient dO and
// D_i = dO_i . O_i:
//   dV_j = sum_i P_ij dO_i,   dP_ij = dO_i . v_j,   dS_ij = P_ij (dP_ij - D_i),
//   dQ_i = scale sum_j dS_ij k_j,   dK_j = scale sum_i dS_ij q_i.
// P is recomputed from the forward's row log-sum-exp, P_ij = exp(s_ij - lse_i).
// Rows without an output (padded conditioning rows) carry lse = +inf, so all
// their P are 0 and they contribute nothing; padded keys get zero dK and dV.
//
// Two forms, three launches each.  Two-kernel form (deterministic):
//   1. delta_kernel: D_i into the caller's fp32 workspace (one read of O, dO).
//   2. dq_kernel, query-stationary: a CTA owns 128 query rows of one (b, h)
//      and streams the 128-key K/V tiles.  S = Q K^T and dP = dO V^T go to
//      tensor memory, dS goes back over S in bf16, and dQ += dS K.  S is
//      double-buffered, so the tensor core computes the next tile's S while
//      the softmax warps turn this tile's S and dP into dS.
//   3. dkdv_kernel, key-stationary: a CTA owns 128 keys of one (b, h) and
//      streams 64-row query tiles.  S^T = K Q^T and dP^T = V dO^T (both
//      double-buffered), P^T and dS^T in bf16 back over them, dV += P^T dO and
//      dK += dS^T Q.  Query tiles of 64 keep the four accumulators inside the
//      512 tensor-memory columns.
// Splitting dQ from dK/dV computes S and dP twice but needs no atomics and no
// fp32 dQ accumulator in global memory.
// One-pass form (a caller workspace holds an fp32 dQ accumulator):
//   1. delta_kernel, which also zeroes the accumulator;
//   2. dkdvq_kernel: dkdv_kernel's pipeline that also forms each query tile's
//      dQ^T = K^T dS^T and reduces it into the accumulator (section 3b);
//   3. dq_convert_kernel: dQ = scale * accumulator, in bf16.
// S and dP are formed once (10 N^2 D executed FLOPs per (sample, head)
// instead of 14); the order of the dQ sums varies from run to run.
//
// Every wait is bounded as in the forward kernel: a wait that runs out sets an
// abort flag and the backward status word, every role leaves its loop, copies
// and MMAs in flight are drained (bounded), and tensor memory is freed.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "internal.h"
#include "ptx.cuh"
#include "tensor_map.h"

namespace mmdit {

// Bit 0: a bounded wait expired in a backward kernel.
__device__ unsigned int g_bwd_status = 0;

namespace bwd {

constexpr int kThreads = 384;
// Register split: launched with 168 per thread; the producer warpgroup (TMA,
// MMA issue, the lse / D loader) takes 88, the softmax warpgroups 208.
constexpr int kRegsLaunch = 168;
constexpr int kRegsProducer = 88;
constexpr int kRegsSoftmax = 208;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsProducer == kThreads * kRegsLaunch,
              "register split must add up to the launch allocation");
constexpr uint64_t kDrainLimitNs = 200000000ull;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kTileBytes = 128 * 128 * 2;   // 128 rows x 128 bf16
constexpr int kHalf128 = kTileBytes / 2;    // one 64-column box of a 128-row tile
constexpr int kQ64Bytes = 64 * 128 * 2;     // 64 rows x 128 bf16
constexpr int kHalf64 = kQ64Bytes / 2;

// Abort flag, wait limit and tensor-memory base shared by a CTA's roles.
struct Ctl {
    uint64_t wait_ns;
    uint32_t abort;
    uint32_t tmem_base;
};

__device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity, Ctl* c) {
    if (mbar_wait_bounded(bar, parity, &c->abort, c->wait_ns)) return true;
    c->abort = 1;
    atomicOr(&g_bwd_status, 1u);
    return false;
}
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, Ctl* c) {
    const bool ok = wait(bar, parity, c);
    return __all_sync(0xffffffffu, ok);
}

// K-major operand: k-step s (16 columns of the 128-wide head dim) lies in the
// 64-column half s / 4, 32 bytes * (s % 4) into each 128-byte row.
__device__ __forceinline__ uint64_t kdesc(uint32_t addr) { return smem_desc_sw128(addr, 16, 1024); }
__host__ __device__ constexpr uint64_t koff(int s, int half_bytes) {
    return (uint64_t)((s >> 2) * (half_bytes >> 4) + (s & 3) * 2);
}
// MN-major B operand of `rows` x 128 (rows along K): k-step s = rows
// [16 s, 16 s + 16) = 2048 bytes further; the two 64-wide halves of N are one
// box apart (leading byte offset), 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t mndesc(uint32_t addr, int half_bytes) {
    return smem_desc_sw128(addr, half_bytes, 1024);
}
constexpr uint64_t kMnStep = 2048 >> 4;

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// ======================================================================
// 1. D_i = dO_i . O_i
// ======================================================================

// 128 / E lanes own one (sample, joint row, head) unit; E elements per 16 bytes.
// acc (null when unused): the fused backward's fp32 dQ accumulator
// [B, Nv + Nc, H, 128], whose unit rows are zeroed here.
template <typename T>
__global__ void __launch_bounds__(256)
delta_kernel(const T* __restrict__ ov, const T* __restrict__ dov, const T* __restrict__ oc,
             const T* __restrict__ doc, const int32_t* __restrict__ ctx_len,
             float* __restrict__ delta, float* __restrict__ acc, int Nv, int Nc, int H,
             uint32_t units) {
    constexpr int E = 16 / sizeof(T);
    constexpr int LPR = 128 / E;
    constexpr int GPW = 32 / LPR;
    constexpr int UNR = 4;
    const int Nt = Nv + Nc;
    const int lane = threadIdx.x & 31;
    const int g = lane % LPR;
    const int grp = lane / LPR;
    const uint32_t warp0 = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
    for (uint32_t uw = warp0 * (GPW * UNR); uw < units; uw += nwarps * (GPW * UNR)) {
        uint4 a[UNR], d[UNR];
        uint32_t jr[UNR], bb[UNR], hh[UNR];
        bool live[UNR];
#pragma unroll
        for (int r = 0; r < UNR; ++r) {
            const uint32_t u = uw + r * GPW + grp;
            live[r] = u < units;
            const uint32_t uu = live[r] ? u : 0;
            hh[r] = uu % H;
            const uint32_t bj = uu / H;
            jr[r] = bj % Nt;
            bb[r] = bj / Nt;
            const bool vis = (int)jr[r] < Nv;
            const size_t row = vis ? ((size_t)bb[r] * Nv + jr[r]) * H + hh[r]
                                   : ((size_t)bb[r] * Nc + (jr[r] - Nv)) * H + hh[r];
            const T* o = (vis ? ov : oc) + row * 128 + g * E;
            const T* dO = (vis ? dov : doc) + row * 128 + g * E;
            a[r] = live[r] ? __ldcs(reinterpret_cast<const uint4*>(o)) : make_uint4(0, 0, 0, 0);
            d[r] = live[r] ? __ldcs(reinterpret_cast<const uint4*>(dO)) : make_uint4(0, 0, 0, 0);
            if (acc && live[r]) {
                float4* z = reinterpret_cast<float4*>(
                    acc + (((size_t)bb[r] * Nt + jr[r]) * H + hh[r]) * 128 + g * E);
#pragma unroll
                for (int e = 0; e < E / 4; ++e) z[e] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
#pragma unroll
        for (int r = 0; r < UNR; ++r) {
            const uint32_t aw[4] = {a[r].x, a[r].y, a[r].z, a[r].w};
            const uint32_t dw[4] = {d[r].x, d[r].y, d[r].z, d[r].w};
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (sizeof(T) == 2) {
                    acc = fmaf(bf_lo(aw[i]), bf_lo(dw[i]), acc);
                    acc = fmaf(bf_hi(aw[i]), bf_hi(dw[i]), acc);
                } else {
                    acc = fmaf(__uint_as_float(aw[i]), __uint_as_float(dw[i]), acc);
                }
            }
#pragma unroll
            for (int o = LPR / 2; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (live[r] && g == 0) {
                int L = Nc;
                if (ctx_len) {
                    L = ctx_len[bb[r]];
                    L = L < 0 ? 0 : (L > Nc ? Nc : L);
                }
                const bool out = (int)jr[r] < Nv + L;
                delta[((size_t)bb[r] * H + hh[r]) * Nt + jr[r]] = out ? acc : 0.f;
            }
        }
    }
}

// ======================================================================
// 2. dQ (query-stationary)
// ======================================================================
namespace dq {

// K is read twice per tile (S = Q K^T, then dQ += dS K one tile later), so its
// ring has a third stage: with two, the next K's load could only start just
// before the product that needs it.  V is read once (dP = dO V^T).  K(j) and
// V(j) arrive under one barrier (that of K's stage), so the MMA issuer waits
// once per key tile for both.
constexpr int kKStages = 3;
constexpr int kVStages = 2;

struct Smem {
    static constexpr int q_off = 0;
    static constexpr int do_off = kTileBytes;
    static constexpr int k_off = 2 * kTileBytes;                        // kKStages tiles
    static constexpr int v_off = k_off + kKStages * kTileBytes;         // kVStages tiles
    static constexpr int bar_off = v_off + kVStages * kTileBytes;
    static constexpr int total = bar_off + 256;
};

struct Params {
    CUtensorMap tm_q[2];   // [0] visual, [1] conditioning; 128-row boxes
    CUtensorMap tm_k[2];
    CUtensorMap tm_v[2];
    CUtensorMap tm_do[2];
    __nv_bfloat16* dq[2];
    const float* lse;
    const float* delta;
    const int32_t* ctx_len;
    int N[2];
    int H;
    int q_tiles_vis;
    float sl2;      // softmax_scale * log2(e)
    float scale;
    uint64_t wait_ns;
    // 3D window mode (visual rows in window-major order): the grid holds the
    // conditioning query tiles first, then the query tiles of each window;
    // a visual tile streams its window's keys, a conditioning tile every key
    int windowed;
    int cond_tiles;
    int tile_start[kMaxWindows + 1];   // first tile of each window after the cond tiles
    WindowTable win;
};
static_assert(sizeof(Params) <= 4096, "kernel parameters must fit the 4 KB parameter space");

struct Bars {
    uint64_t q_full;
    uint64_t kv_full[kKStages];   // K(j) in K stage j % 3 and V(j) in V stage j % 2 landed
    uint64_t k_empty[kKStages];
    uint64_t v_empty[kVStages];
    uint64_t s_full[2];    // S and dP of the tile with this S buffer are in tensor memory
    uint64_t dp_free;      // every softmax warp has read dP
    uint64_t ds_full[2];   // [buf]: all of dS of that buffer is in tensor memory
    uint64_t o_done;
    uint64_t drain;
    Ctl ctl;
};
static_assert(sizeof(Bars) <= 256, "barrier block must fit its shared-memory slot");

// dS = exp2(S * scale log2 e - lse log2 e) * (dP - D) for 64 keys of one row,
// packed in bf16 pairs; keys at or past `valid` get dS = 0.  (A variant that
// masks only tail tiles duplicated this loop and made the softmax spill.)
__device__ __forceinline__ void ds_half(const uint32_t (&sr)[2][32], const uint32_t (&dr)[2][32],
                                        uint32_t (&pk)[32], uint64_t sl2x2, uint64_t nl2,
                                        uint64_t ndl, int valid) {
#pragma unroll
    for (int c = 0; c < 32; ++c) {
        const int k = 2 * c;
        const uint64_t x = f2_fma(f2_pack(__uint_as_float(sr[k >> 5][k & 31]),
                                          __uint_as_float(sr[k >> 5][(k & 31) + 1])),
                                  sl2x2, nl2);
        float x0, x1;
        f2_unpack(x, x0, x1);
        if (valid < 64) {
            if (k >= valid) x0 = -INFINITY;
            if (k + 1 >= valid) x1 = -INFINITY;
        }
        const uint64_t pp = f2_pack(ex2_approx(x0), ex2_approx(x1));
        const uint64_t dd = f2_add(f2_pack(__uint_as_float(dr[k >> 5][k & 31]),
                                           __uint_as_float(dr[k >> 5][(k & 31) + 1])),
                                   ndl);
        float d0, d1;
        f2_unpack(f2_mul(pp, dd), d0, d1);
        pk[c] = pack_bf16x2(d0, d1);
    }
}

// Tensor memory: S0 [0,128) S1 [128,256) dP [256,384) dQ [384,512).  dS of
// key half w is written over S at columns [64 w, 64 w + 32).
__global__ void __launch_bounds__(kThreads, 1) dq_kernel(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars* bars = reinterpret_cast<Bars*>(smem + Smem::bar_off);
    Ctl* ctl = &bars->ctl;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x;
    const int h = blockIdx.y;
    const int b = blockIdx.z;
    // query tile: stream seg, first row row0, rows stored below rend; visual
    // keys [vs, vs + vl) (all of them, or the query's window)
    int seg, row0, rend, vs = 0, vl = p.N[0];
    if (!p.windowed) {
        seg = t < p.q_tiles_vis ? 0 : 1;
        row0 = (seg ? t - p.q_tiles_vis : t) * 128;
        rend = p.N[seg];
    } else if (t < p.cond_tiles) {
        seg = 1;
        row0 = 128 * t;
        rend = p.N[1];
    } else {
        const int tt = t - p.cond_tiles;
        int w = 0;
        while (w + 1 < p.win.count && p.tile_start[w + 1] <= tt) ++w;
        const WindowGeom& g = p.win.w[w];
        seg = 0;
        vs = g.start;
        vl = g.te * g.he * g.we;
        row0 = vs + 128 * (tt - p.tile_start[w]);
        rend = vs + vl;
    }
    int L = p.N[1];
    if (p.ctx_len) {
        L = p.ctx_len[b];
        L = L < 0 ? 0 : (L > p.N[1] ? p.N[1] : L);
    }
    const int kv_vis = (vl + 127) / 128;
    const int n_kv = kv_vis + (L + 127) / 128;
    const bool idle = n_kv == 0 || (seg == 1 && row0 >= L);   // no row of this tile has an output

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        for (int i = 0; i < kKStages; ++i) {
            mbar_init(&bars->kv_full[i], 1);
            mbar_init(&bars->k_empty[i], 1);
        }
        for (int i = 0; i < kVStages; ++i) mbar_init(&bars->v_empty[i], 1);
        for (int i = 0; i < 2; ++i) mbar_init(&bars->s_full[i], 1);
        mbar_init(&bars->dp_free, 8);
        for (int i = 0; i < 2; ++i) mbar_init(&bars->ds_full[i], 8);   // one lane per softmax warp
        mbar_init(&bars->o_done, 1);
        mbar_init(&bars->drain, 1);
        ctl->abort = 0;
        ctl->wait_ns = p.wait_ns;
        fence_barrier_init();
    }
    if (warp == 8 && !idle) {
        tmem_alloc(&ctl->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (idle) {
        for (int r = threadIdx.x; r < 128 * 16; r += kThreads) {
            const int row = row0 + r / 16;
            if (row < rend)
                reinterpret_cast<uint4*>(
                    p.dq[seg] + ((size_t)((size_t)b * p.N[seg] + row) * p.H + h) * 128)[r % 16] =
                    make_uint4(0, 0, 0, 0);
        }
        return;
    }
    const uint32_t tmem = ctl->tmem_base;
    const uint32_t sQ = smem_u32(smem + Smem::q_off);
    const uint32_t sDO = smem_u32(smem + Smem::do_off);
    const uint32_t sK = smem_u32(smem + Smem::k_off);
    const uint32_t sV = smem_u32(smem + Smem::v_off);

    if (warp >= 8) {
        regs_dec<kRegsProducer>();
        if (warp == 8 && lane == 0) {
            // ---------------------------------------------- TMA: Q, dO, then K and V
            mbar_arrive_expect_tx(&bars->q_full, 2 * kTileBytes);
            tma_load_4d(smem + Smem::q_off, &p.tm_q[seg], &bars->q_full, 0, h, row0, b);
            tma_load_4d(smem + Smem::q_off + kHalf128, &p.tm_q[seg], &bars->q_full, 64, h, row0, b);
            tma_load_4d(smem + Smem::do_off, &p.tm_do[seg], &bars->q_full, 0, h, row0, b);
            tma_load_4d(smem + Smem::do_off + kHalf128, &p.tm_do[seg], &bars->q_full, 64, h, row0,
                        b);
            int issued = 0;
            for (int j = 0; j < n_kv; ++j) {
                const int kst = j % kKStages, vst = j % kVStages;
                const int ks = j < kv_vis ? 0 : 1;
                const int row = ks ? (j - kv_vis) * 128 : vs + j * 128;
                if (!wait(&bars->k_empty[kst], ((j / kKStages) & 1) ^ 1, ctl)) break;
                if (!wait(&bars->v_empty[vst], ((j / kVStages) & 1) ^ 1, ctl)) break;
                uint8_t* dk = smem + Smem::k_off + kst * kTileBytes;
                uint8_t* dv = smem + Smem::v_off + vst * kTileBytes;
                mbar_arrive_expect_tx(&bars->kv_full[kst], 2 * kTileBytes);
                tma_load_4d(dk, &p.tm_k[ks], &bars->kv_full[kst], 0, h, row, b);
                tma_load_4d(dk + kHalf128, &p.tm_k[ks], &bars->kv_full[kst], 64, h, row, b);
                tma_load_4d(dv, &p.tm_v[ks], &bars->kv_full[kst], 0, h, row, b);
                tma_load_4d(dv + kHalf128, &p.tm_v[ks], &bars->kv_full[kst], 64, h, row, b);
                ++issued;
            }
            if (ctl->abort) {
                for (int j = (issued > kKStages ? issued - kKStages : 0); j < issued; ++j)
                    mbar_wait_bounded(&bars->kv_full[j % kKStages], (j / kKStages) & 1, nullptr,
                                      kDrainLimitNs);
                mbar_wait_bounded(&bars->q_full, 0, nullptr, kDrainLimitNs);
            }
        } else if (warp == 9 && lane == 0) {
            // ---------------------------------------------- MMA issuer
            constexpr uint32_t id_kk = idesc_bf16_f32(128, 128, 0, 0);
            constexpr uint32_t id_mn = idesc_bf16_f32(128, 128, 0, 1);
            bool ok = wait(&bars->q_full, 0, ctl);
            const uint64_t dq_d = kdesc(sQ), ddo_d = kdesc(sDO);
            const uint64_t dv0 = kdesc(sV), dv1 = kdesc(sV + kTileBytes);
            // K stage st: K-major for S, MN-major for dQ (descriptor start
            // addresses differ by whole tiles)
            const uint64_t dk0 = kdesc(sK);
            const uint64_t km0 = mndesc(sK, kHalf128);
            constexpr uint64_t kTileStep = kTileBytes >> 4;
            // dQ += dS(jj) K(jj) once the softmax has written all of dS(jj)
            // (two releases, one per key half, measured slower: one more
            // wait per tile for the issuing thread)
            auto dq_mma = [&](int jj, int kst_jj) -> bool {
                const int pb = jj & 1;
                const uint64_t km = km0 + (uint64_t)kst_jj * kTileStep;
                const uint32_t sb = tmem + 128 * pb;
                if (!wait(&bars->ds_full[pb], (jj >> 1) & 1, ctl)) return false;
                tc_fence_after();
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_ts(tmem + 384, sb + 64 * (s >> 2) + 8 * (s & 3), km + (uint64_t)s * kMnStep,
                           id_mn, (jj > 0 || s > 0) ? 1u : 0u);
                return true;
            };
            int kst = 0, kph = 0, kst_prev = 0;      // K stage of tile j, its phase, and of j - 1
            for (int j = 0; ok && j < n_kv; ++j) {
                const int st = j & 1;                // S buffer and V stage
                if (!(ok = wait(&bars->kv_full[kst], kph, ctl))) break;   // K(j) and V(j)
                tc_fence_after();
                const uint64_t dk = dk0 + (uint64_t)kst * kTileStep;
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    const uint64_t off = koff(s, kHalf128);
                    mma_ss(tmem + 128 * st, dq_d + off, dk + off, id_kk, s > 0 ? 1u : 0u);
                }
                if (j > 0 && !(ok = wait(&bars->dp_free, (j - 1) & 1, ctl))) break;
                tc_fence_after();
                const uint64_t dv = st ? dv1 : dv0;
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    const uint64_t off = koff(s, kHalf128);
                    mma_ss(tmem + 256, ddo_d + off, dv + off, id_kk, s > 0 ? 1u : 0u);
                }
                mma_commit(&bars->s_full[st]);
                mma_commit(&bars->v_empty[st]);
                if (j > 0) {
                    if (!(ok = dq_mma(j - 1, kst_prev))) break;
                    mma_commit(&bars->k_empty[kst_prev]);
                }
                kst_prev = kst;
                if (++kst == kKStages) {
                    kst = 0;
                    kph ^= 1;
                }
            }
            if (ok && (ok = dq_mma(n_kv - 1, kst_prev))) {
                mma_commit(&bars->k_empty[kst_prev]);
                mma_commit(&bars->o_done);
            }
            mma_commit(&bars->drain);
            if (!mbar_wait_bounded(&bars->drain, 0, nullptr, kDrainLimitNs))
                atomicOr(&g_bwd_status, 1u);
        }
    } else {
        regs_inc<kRegsSoftmax>();
        // -------------------------------------------------- dS = P (dP - D)
        const int wg = warp >> 2;        // key columns [64 wg, 64 wg + 64) of every tile
        const int quarter = warp & 3;    // tensor-memory lanes (query rows) of this warp
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const int row = row0 + quarter * 32 + lane;
        const bool has_out = row < rend && (seg == 0 || row < L);
        const size_t lrow =
            ((size_t)b * p.H + h) * (size_t)(p.N[0] + p.N[1]) + (seg ? p.N[0] + row : row);
        const float lse2 = has_out ? p.lse[lrow] * kLog2e : INFINITY;
        const float dl = has_out ? p.delta[lrow] : 0.f;
        const uint64_t sl2x2 = f2_pack(p.sl2, p.sl2);
        const uint64_t nl2 = f2_pack(-lse2, -lse2);
        const uint64_t ndl = f2_pack(-dl, -dl);
        bool ok = true;
        for (int j = 0; j < n_kv; ++j) {
            const int buf = j & 1;
            if (!(ok = wait_warp(&bars->s_full[buf], (j >> 1) & 1, ctl))) break;
            tc_fence_after();
            uint32_t sr[2][32], dr[2][32];
            const uint32_t tS = tmem + 128 * buf + 64 * wg + lane_off;
            const uint32_t tP = tmem + 256 + 64 * wg + lane_off;
            tmem_ld32(tS, sr[0]);
            tmem_ld32(tS + 32, sr[1]);
            tmem_ld32(tP, dr[0]);
            tmem_ld32(tP + 32, dr[1]);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->dp_free);
            const int valid =
                (j < kv_vis ? vl - j * 128 : L - (j - kv_vis) * 128) - 64 * wg;
            uint32_t pk[32];
            ds_half(sr, dr, pk, sl2x2, nl2, ndl, valid);
            tmem_st32(tS, pk);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->ds_full[buf]);
        }
        if (ok) ok = wait_warp(&bars->o_done, 0, ctl);
        tc_fence_after();
        const bool store = row < rend;
        const bool zero = !ok || !has_out;
        uint4* dst = reinterpret_cast<uint4*>(
            p.dq[seg] + ((size_t)((size_t)b * p.N[seg] + (store ? row : 0)) * p.H + h) * 128 +
            64 * wg);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            uint32_t o[32];
            tmem_ld32(tmem + 384 + 64 * wg + 32 * c + lane_off, o);
            tmem_wait_ld();
            if (store) {
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    float f[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        f[e] = zero ? 0.f : __uint_as_float(o[8 * v + e]) * p.scale;
                    dst[4 * c + v] = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                                pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace dq

// ======================================================================
// 3. dK, dV (key-stationary)
// ======================================================================
namespace dkv {

constexpr int kStages = 4;   // Q / dO / (lse, D) ring depth; Q and dO of a tile share a barrier

struct Smem {
    static constexpr int k_off = 0;
    static constexpr int v_off = kTileBytes;
    static constexpr int q_off = 2 * kTileBytes;                  // kStages x 64 rows
    static constexpr int do_off = q_off + kStages * kQ64Bytes;    // kStages x 64 rows
    static constexpr int l_off = do_off + kStages * kQ64Bytes;    // kStages x 64 float2
    static constexpr int bar_off = l_off + kStages * 512;
    static constexpr int total = bar_off + 512;
};

struct Params {
    CUtensorMap tm_k[2];   // 128-row boxes
    CUtensorMap tm_v[2];
    CUtensorMap tm_q[2];   // 64-row boxes
    CUtensorMap tm_do[2];
    CUtensorMap tm_acc;    // fp32 dQ accumulator [B, Nv + Nc, H, 128] (dkdvq_kernel only)
    __nv_bfloat16* dk[2];
    __nv_bfloat16* dv[2];
    const float* lse;
    const float* delta;
    const int32_t* ctx_len;
    int N[2];
    int H;
    int k_tiles_vis;
    float sl2;
    float scale;
    uint64_t wait_ns;
    // 3D window mode (visual rows in window-major order): the grid holds the
    // conditioning key tiles first (every query sees them), then the key
    // tiles of each window (seen by that window's queries and the cond ones)
    int windowed;
    int cond_tiles;
    int tile_start[kMaxWindows + 1];
    WindowTable win;
};
static_assert(sizeof(Params) <= 4096, "kernel parameters must fit the 4 KB parameter space");

struct Bars {
    uint64_t kv_full;
    uint64_t qd_full[kStages], qd_empty[kStages];   // Q and dO of query tile i in stage i % 4
    uint64_t l_full[kStages], l_empty[kStages];
    uint64_t s_full[2];   // S^T and dP^T of the tile with this buffer are in tensor memory
    uint64_t p_full[2];   // every softmax warp has written its P^T and dS^T
    uint64_t o_done;
    uint64_t drain;
    Ctl ctl;
};
static_assert(sizeof(Bars) <= 512, "barrier block must fit its shared-memory slot");

// The key tile a CTA owns and the query tiles that stream past it.
struct KeyTile {
    int seg;      // stream of the keys
    int krow0;    // first key
    int kend;     // keys stored below this row
    int qvs;      // visual query rows [qvs, qvs + qvl) see these keys
    int qvl;
    int L;        // valid conditioning tokens of the sample
    int nq_vis;   // 64-row visual query tiles, then the conditioning ones
    int nq;
    bool idle;    // no valid key or no query
};

__device__ __forceinline__ KeyTile key_tile(const Params& p, int t, int b) {
    KeyTile k;
    k.qvs = 0;
    k.qvl = p.N[0];
    if (!p.windowed) {
        k.seg = t < p.k_tiles_vis ? 0 : 1;
        k.krow0 = (k.seg ? t - p.k_tiles_vis : t) * 128;
        k.kend = p.N[k.seg];
    } else if (t < p.cond_tiles) {
        k.seg = 1;
        k.krow0 = 128 * t;
        k.kend = p.N[1];
    } else {
        const int tt = t - p.cond_tiles;
        int w = 0;
        while (w + 1 < p.win.count && p.tile_start[w + 1] <= tt) ++w;
        const WindowGeom& g = p.win.w[w];
        k.seg = 0;
        k.qvs = g.start;
        k.qvl = g.te * g.he * g.we;
        k.krow0 = k.qvs + 128 * (tt - p.tile_start[w]);
        k.kend = k.qvs + k.qvl;
    }
    k.L = p.N[1];
    if (p.ctx_len) {
        k.L = p.ctx_len[b];
        k.L = k.L < 0 ? 0 : (k.L > p.N[1] ? p.N[1] : k.L);
    }
    k.nq_vis = (k.qvl + 63) / 64;
    k.nq = k.nq_vis + (k.L + 63) / 64;
    k.idle = k.nq == 0 || (k.seg == 1 && k.krow0 >= k.L);
    return k;
}

// First row of query tile i in its stream (qs: 0 visual, 1 conditioning).
__device__ __forceinline__ int query_row(const KeyTile& k, int i, int& qs) {
    qs = i < k.nq_vis ? 0 : 1;
    return qs ? (i - k.nq_vis) * 64 : k.qvs + i * 64;
}

// Zero dK and dV of a key tile that no query sees.
__device__ __forceinline__ void zero_key_tile(const Params& p, const KeyTile& k, int h, int b) {
    for (int r = threadIdx.x; r < 128 * 16; r += kThreads) {
        const int key = k.krow0 + r / 16;
        if (key < k.kend) {
            const size_t off = ((size_t)((size_t)b * p.N[k.seg] + key) * p.H + h) * 128;
            reinterpret_cast<uint4*>(p.dk[k.seg] + off)[r % 16] = make_uint4(0, 0, 0, 0);
            reinterpret_cast<uint4*>(p.dv[k.seg] + off)[r % 16] = make_uint4(0, 0, 0, 0);
        }
    }
}

// TMA producer (one thread): K and V of the key tile under kv_full, then Q
// and dO of each 64-row query tile under qd_full of its ring stage.
template <int S>
__device__ __forceinline__ void stream_key_tile(const Params& p, const KeyTile& k, uint8_t* smem,
                                                int q_off, int do_off, uint64_t* kv_full,
                                                uint64_t* qd_full, uint64_t* qd_empty, Ctl* ctl,
                                                int h, int b) {
    mbar_arrive_expect_tx(kv_full, 2 * kTileBytes);
    tma_load_4d(smem, &p.tm_k[k.seg], kv_full, 0, h, k.krow0, b);
    tma_load_4d(smem + kHalf128, &p.tm_k[k.seg], kv_full, 64, h, k.krow0, b);
    tma_load_4d(smem + kTileBytes, &p.tm_v[k.seg], kv_full, 0, h, k.krow0, b);
    tma_load_4d(smem + kTileBytes + kHalf128, &p.tm_v[k.seg], kv_full, 64, h, k.krow0, b);
    int issued = 0;
    for (int i = 0; i < k.nq; ++i) {
        const int st = i % S;
        int qs;
        const int row = query_row(k, i, qs);
        if (!wait(&qd_empty[st], ((i / S) & 1) ^ 1, ctl)) break;
        uint8_t* dq_ = smem + q_off + st * kQ64Bytes;
        uint8_t* ddo = smem + do_off + st * kQ64Bytes;
        mbar_arrive_expect_tx(&qd_full[st], 2 * kQ64Bytes);
        tma_load_4d(dq_, &p.tm_q[qs], &qd_full[st], 0, h, row, b);
        tma_load_4d(dq_ + kHalf64, &p.tm_q[qs], &qd_full[st], 64, h, row, b);
        tma_load_4d(ddo, &p.tm_do[qs], &qd_full[st], 0, h, row, b);
        tma_load_4d(ddo + kHalf64, &p.tm_do[qs], &qd_full[st], 64, h, row, b);
        ++issued;
    }
    if (ctl->abort) {
        for (int i = (issued > S ? issued - S : 0); i < issued; ++i)
            mbar_wait_bounded(&qd_full[i % S], (i / S) & 1, nullptr, kDrainLimitNs);
        mbar_wait_bounded(kv_full, 0, nullptr, kDrainLimitNs);
    }
}

// (lse * log2 e, D) of each query tile (one warp); rows outside the range
// that sees these keys (past the stream, past the window, or padding) get
// lse = +inf, so their P is 0.
template <int S>
__device__ __forceinline__ void load_lse_delta(const Params& p, const KeyTile& k, float2* lbuf,
                                               uint64_t* l_full, uint64_t* l_empty, Ctl* ctl,
                                               int lane, int h, int b) {
    const size_t base = ((size_t)b * p.H + h) * (size_t)(p.N[0] + p.N[1]);
    for (int i = 0; i < k.nq; ++i) {
        const int st = i % S;
        if (!wait_warp(&l_empty[st], ((i / S) & 1) ^ 1, ctl)) break;
        int qs;
        const int row0q = query_row(k, i, qs);
        const int rlim = qs ? k.L : k.qvs + k.qvl;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int q = lane + 32 * r;
            const int row = row0q + q;
            const bool has = row < rlim && row < p.N[qs];
            const size_t jr = base + (qs ? p.N[0] + row : row);
            lbuf[st * 64 + q] =
                has ? make_float2(p.lse[jr] * kLog2e, p.delta[jr]) : make_float2(INFINITY, 0.f);
        }
        mbar_arrive(&l_full[st]);
    }
}

// P^T and dS^T = P^T (dP^T - D) of 32 queries of one key row, packed in bf16
// pairs, from S^T and dP^T as read from tensor memory.
__device__ __forceinline__ void p_ds(const uint32_t (&sr)[32], const uint32_t (&dr)[32],
                                     const float2* lq, uint64_t sl2x2, uint32_t (&pp)[16],
                                     uint32_t (&pd)[16]) {
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        const float2 l0 = lq[2 * c], l1 = lq[2 * c + 1];
        const uint64_t x = f2_fma(f2_pack(__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1])),
                                  sl2x2, f2_pack(-l0.x, -l1.x));
        float x0, x1;
        f2_unpack(x, x0, x1);
        const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
        const uint64_t dd = f2_sub(
            f2_pack(__uint_as_float(dr[2 * c]), __uint_as_float(dr[2 * c + 1])), f2_pack(l0.y, l1.y));
        float d0, d1;
        f2_unpack(f2_mul(f2_pack(p0, p1), dd), d0, d1);
        pp[c] = pack_bf16x2(p0, p1);
        pd[c] = pack_bf16x2(d0, d1);
    }
}

// dV and dK (times scale) of the key rows of this warp's tensor-memory lanes
// and 64 head-dim columns of warpgroup wg, to bf16 (zero when !ok or for
// padded conditioning keys).
__device__ __forceinline__ void store_dkdv(const Params& p, const KeyTile& k, uint32_t tmem,
                                           int quarter, int wg, int lane, bool ok, int h, int b) {
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int key = k.krow0 + quarter * 32 + lane;
    const bool store = key < k.kend;
    const bool zero = !ok || (k.seg == 1 && key >= k.L);
    const size_t off =
        ((size_t)((size_t)b * p.N[k.seg] + (store ? key : 0)) * p.H + h) * 128 + 64 * wg;
#pragma unroll
    for (int which = 0; which < 2; ++which) {   // 0: dV, 1: dK (times scale)
        uint4* dst = reinterpret_cast<uint4*>((which ? p.dk[k.seg] : p.dv[k.seg]) + off);
        const float mul = which ? p.scale : 1.f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            uint32_t o[32];
            tmem_ld32(tmem + 256 + 128 * which + 64 * wg + 32 * c + lane_off, o);
            tmem_wait_ld();
            if (store) {
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    float f[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        f[e] = zero ? 0.f : __uint_as_float(o[8 * v + e]) * mul;
                    dst[4 * c + v] = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                                pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
                }
            }
        }
    }
}

// Tensor memory: S^T buffers [0,64) [64,128), dP^T buffers [128,192)
// [192,256), dV [256,384), dK [384,512).  Warpgroup w handles query columns
// [32 w, 32 w + 32) of a tile and writes its packed P^T / dS^T at columns
// [32 w, 32 w + 16) of the same buffer.
__host__ __device__ constexpr int packed_col(int s) { return s < 2 ? 8 * s : 32 + 8 * (s - 2); }

__global__ void __launch_bounds__(kThreads, 1) dkdv_kernel(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars* bars = reinterpret_cast<Bars*>(smem + Smem::bar_off);
    Ctl* ctl = &bars->ctl;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int h = blockIdx.y;
    const int b = blockIdx.z;
    const KeyTile kt = key_tile(p, blockIdx.x, b);

    if (threadIdx.x == 0) {
        mbar_init(&bars->kv_full, 1);
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&bars->qd_full[i], 1);
            mbar_init(&bars->qd_empty[i], 1);
            mbar_init(&bars->l_full[i], 32);   // every lane of the loader warp
            mbar_init(&bars->l_empty[i], 8);   // one elected lane per softmax warp
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->s_full[i], 1);
            mbar_init(&bars->p_full[i], 8);
        }
        mbar_init(&bars->o_done, 1);
        mbar_init(&bars->drain, 1);
        ctl->abort = 0;
        ctl->wait_ns = p.wait_ns;
        fence_barrier_init();
    }
    if (warp == 8 && !kt.idle) {
        tmem_alloc(&ctl->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (kt.idle) {
        zero_key_tile(p, kt, h, b);
        return;
    }
    const uint32_t tmem = ctl->tmem_base;
    const uint32_t sK = smem_u32(smem + Smem::k_off);
    const uint32_t sV = smem_u32(smem + Smem::v_off);
    const uint32_t sQ = smem_u32(smem + Smem::q_off);
    const uint32_t sDO = smem_u32(smem + Smem::do_off);
    float2* lbuf = reinterpret_cast<float2*>(smem + Smem::l_off);   // (lse * log2 e, D)

    if (warp >= 8) {
        regs_dec<kRegsProducer>();
        if (warp == 8 && lane == 0) {
            stream_key_tile<kStages>(p, kt, smem, Smem::q_off, Smem::do_off, &bars->kv_full,
                                     bars->qd_full, bars->qd_empty, ctl, h, b);
        } else if (warp == 11) {
            load_lse_delta<kStages>(p, kt, lbuf, bars->l_full, bars->l_empty, ctl, lane, h, b);
        } else if (warp == 9 && lane == 0) {
            // ---------------------------------------------- MMA issuer
            constexpr uint32_t id_n64 = idesc_bf16_f32(128, 64, 0, 0);
            constexpr uint32_t id_mn = idesc_bf16_f32(128, 128, 0, 1);
            bool ok = wait(&bars->kv_full, 0, ctl);
            const uint64_t kd = kdesc(sK), vd = kdesc(sV);
            // dV += P^T dO and dK += dS^T Q of query tile ii
            auto grad_mma = [&](int ii) -> bool {
                const int pb = ii & 1;
                const int pst = ii % kStages;
                if (!wait(&bars->p_full[pb], (ii >> 1) & 1, ctl)) return false;
                tc_fence_after();
                const uint64_t dom = mndesc(sDO + pst * kQ64Bytes, kHalf64);
                const uint64_t qm = mndesc(sQ + pst * kQ64Bytes, kHalf64);
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_ts(tmem + 256, tmem + 64 * pb + packed_col(s), dom + (uint64_t)s * kMnStep,
                           id_mn, (ii > 0 || s > 0) ? 1u : 0u);
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_ts(tmem + 384, tmem + 128 + 64 * pb + packed_col(s),
                           qm + (uint64_t)s * kMnStep, id_mn, (ii > 0 || s > 0) ? 1u : 0u);
                mma_commit(&bars->qd_empty[pst]);
                return true;
            };
            for (int i = 0; ok && i < kt.nq; ++i) {
                const int st = i % kStages;
                const uint32_t ph = (i / kStages) & 1;
                const int buf = i & 1;
                if (!(ok = wait(&bars->qd_full[st], ph, ctl))) break;   // Q and dO of tile i
                tc_fence_after();
                const uint64_t qd = kdesc(sQ + st * kQ64Bytes);
                const uint64_t dod = kdesc(sDO + st * kQ64Bytes);
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_ss(tmem + 64 * buf, kd + koff(s, kHalf128), qd + koff(s, kHalf64), id_n64,
                           s > 0 ? 1u : 0u);
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_ss(tmem + 128 + 64 * buf, vd + koff(s, kHalf128), dod + koff(s, kHalf64),
                           id_n64, s > 0 ? 1u : 0u);
                mma_commit(&bars->s_full[buf]);
                if (i > 0 && !(ok = grad_mma(i - 1))) break;
            }
            if (ok && (ok = grad_mma(kt.nq - 1))) mma_commit(&bars->o_done);
            mma_commit(&bars->drain);
            if (!mbar_wait_bounded(&bars->drain, 0, nullptr, kDrainLimitNs))
                atomicOr(&g_bwd_status, 1u);
        }
    } else {
        regs_inc<kRegsSoftmax>();
        // -------------------------------------------------- P^T, dS^T = P^T (dP^T - D)
        const int wg = warp >> 2;        // query columns [32 wg, 32 wg + 32) of every tile
        const int quarter = warp & 3;    // tensor-memory lanes (keys) of this warp
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const uint64_t sl2x2 = f2_pack(p.sl2, p.sl2);
        bool ok = true;
        for (int i = 0; i < kt.nq; ++i) {
            const int buf = i & 1;
            const int st = i % kStages;
            if (!(ok = wait_warp(&bars->s_full[buf], (i >> 1) & 1, ctl))) break;
            if (!(ok = wait_warp(&bars->l_full[st], (i / kStages) & 1, ctl))) break;
            tc_fence_after();
            uint32_t sr[32], dr[32];
            const uint32_t tS = tmem + 64 * buf + 32 * wg + lane_off;
            const uint32_t tD = tmem + 128 + 64 * buf + 32 * wg + lane_off;
            tmem_ld32(tS, sr);
            tmem_ld32(tD, dr);
            tmem_wait_ld();
            uint32_t pp[16], pd[16];
            p_ds(sr, dr, lbuf + st * 64 + 32 * wg, sl2x2, pp, pd);
            tmem_st16(tS, pp);
            tmem_st16(tD, pd);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars->p_full[buf]);
                mbar_arrive(&bars->l_empty[st]);
            }
        }
        if (ok) ok = wait_warp(&bars->o_done, 0, ctl);
        tc_fence_after();
        store_dkdv(p, kt, tmem, quarter, wg, lane, ok, h, b);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ----------------------------------------------------------------------
// 3b. dK, dV and dQ in one key-stationary pass
// ----------------------------------------------------------------------
// dkdv_kernel's pipeline extended with dQ.  The softmax warps write dS^T to
// shared memory (P^T still goes to tensor memory), where it is the A operand
// of dK += dS^T Q and the B operand of this tile's dQ^T = K^T dS^T (head dim
// x 64 queries; K^T is the stationary K tile read as an MN-major operand).
// Each softmax warp then reads its 32 x 32 block of dQ^T and adds it into an
// fp32 accumulator [B, Nv + Nc, H, 128] in global memory with one bulk tensor
// reduce-add; dq_convert_kernel scales the sums into bf16 dQ.  S and dP are
// formed once, so the backward executes 10 N^2 D FLOPs per (sample, head)
// instead of the 14 of dq_kernel + dkdv_kernel.  The costs: the accumulator
// (zeroed by delta_kernel; a head's rows are reduced into by all its key tiles
// at about the same time, so they stay in L2), dP^T single-buffered (it is
// only read, so the next tile's dP^T waits for the loads, not the softmax),
// and an order of the dQ sums that changes from run to run.
namespace fused {

constexpr int kQdStages = 3;                // Q / dO / (lse, D) ring depth
constexpr int kBlockBytes = 32 * 32 * 4;    // one warp's 32 x 32 fp32 block of dQ^T

struct Smem {
    static constexpr int k_off = 0;
    static constexpr int v_off = kTileBytes;
    static constexpr int q_off = 2 * kTileBytes;
    static constexpr int do_off = q_off + kQdStages * kQ64Bytes;
    static constexpr int ds_off = do_off + kQdStages * kQ64Bytes;   // dS^T: 128 keys x 64 queries
    static constexpr int dq_off = ds_off + kQ64Bytes;               // 8 softmax warps' blocks
    static constexpr int l_off = dq_off + 8 * kBlockBytes;
    static constexpr int bar_off = l_off + kQdStages * 512;
    static constexpr int total = bar_off + 512;
};

struct Bars {
    uint64_t kv_full;
    uint64_t qd_full[kQdStages], qd_empty[kQdStages];
    uint64_t l_full[kQdStages], l_empty[kQdStages];
    uint64_t s_full[2];   // S^T (buffer i % 2) and dP^T of query tile i are in tensor memory
    uint64_t dp_free;     // every softmax warp has read dP^T
    // p_full[i % 2]: every softmax warp has written P^T(i) to tensor memory and
    // dS^T(i) to shared memory, and has read dQ^T(i - 1) (so the MMA issuer
    // needs no other wait before overwriting dQ^T)
    uint64_t p_full[2];
    uint64_t dq_full;     // dQ^T formed; dS^T's shared memory free again
    uint64_t o_done;
    uint64_t drain;
    Ctl ctl;
};
static_assert(sizeof(Bars) <= 512, "barrier block must fit its shared-memory slot");

// Tensor memory: S^T buffers [0,64) [64,128) (P^T packed over them as in
// dkdv_kernel), dP^T [128,192), dQ^T [192,256), dV [256,384), dK [384,512).
constexpr uint32_t kColDP = 128;
constexpr uint32_t kColDQ = 192;

__global__ void __launch_bounds__(kThreads, 1) dkdvq_kernel(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars* bars = reinterpret_cast<Bars*>(smem + Smem::bar_off);
    Ctl* ctl = &bars->ctl;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int h = blockIdx.y;
    const int b = blockIdx.z;
    const KeyTile kt = key_tile(p, blockIdx.x, b);

    if (threadIdx.x == 0) {
        mbar_init(&bars->kv_full, 1);
        for (int i = 0; i < kQdStages; ++i) {
            mbar_init(&bars->qd_full[i], 1);
            mbar_init(&bars->qd_empty[i], 1);
            mbar_init(&bars->l_full[i], 32);   // every lane of the loader warp
            mbar_init(&bars->l_empty[i], 8);   // one elected lane per softmax warp
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->s_full[i], 1);
            mbar_init(&bars->p_full[i], 8);
        }
        mbar_init(&bars->dp_free, 8);
        mbar_init(&bars->dq_full, 1);
        mbar_init(&bars->o_done, 1);
        mbar_init(&bars->drain, 1);
        ctl->abort = 0;
        ctl->wait_ns = p.wait_ns;
        fence_barrier_init();
    }
    if (warp == 8 && !kt.idle) {
        tmem_alloc(&ctl->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (kt.idle) {   // no query sees these keys: they add nothing to dQ
        zero_key_tile(p, kt, h, b);
        return;
    }
    const uint32_t tmem = ctl->tmem_base;
    const uint32_t sK = smem_u32(smem + Smem::k_off);
    const uint32_t sV = smem_u32(smem + Smem::v_off);
    const uint32_t sQ = smem_u32(smem + Smem::q_off);
    const uint32_t sDO = smem_u32(smem + Smem::do_off);
    const uint32_t sDS = smem_u32(smem + Smem::ds_off);
    float2* lbuf = reinterpret_cast<float2*>(smem + Smem::l_off);   // (lse * log2 e, D)

    if (warp >= 8) {
        regs_dec<kRegsProducer>();
        if (warp == 8 && lane == 0) {
            stream_key_tile<kQdStages>(p, kt, smem, Smem::q_off, Smem::do_off, &bars->kv_full,
                                       bars->qd_full, bars->qd_empty, ctl, h, b);
        } else if (warp == 11) {
            load_lse_delta<kQdStages>(p, kt, lbuf, bars->l_full, bars->l_empty, ctl, lane, h, b);
        } else if (warp == 9 && lane == 0) {
            // ---------------------------------------------- MMA issuer
            constexpr uint32_t id_n64 = idesc_bf16_f32(128, 64, 0, 0);   // S^T, dP^T
            constexpr uint32_t id_mn = idesc_bf16_f32(128, 128, 0, 1);   // dV, dK
            constexpr uint32_t id_dq = idesc_bf16_f32(128, 64, 1, 1);    // dQ^T
            bool ok = wait(&bars->kv_full, 0, ctl);
            const uint64_t kd = kdesc(sK), vd = kdesc(sV);
            const uint64_t dsa = kdesc(sDS);   // dS^T as A: M = keys, K = queries
            // dV += P^T dO, dK += dS^T Q, then dQ^T = K^T dS^T of query tile ii
            // (issued once p_full of tile ii has been seen)
            auto grad_mma = [&](int ii) {
                const int pb = ii & 1;
                const int pst = ii % kQdStages;
                tc_fence_after();
                const uint64_t dom = mndesc(sDO + pst * kQ64Bytes, kHalf64);
                const uint64_t qm = mndesc(sQ + pst * kQ64Bytes, kHalf64);
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_ts(tmem + 256, tmem + 64 * pb + packed_col(s), dom + (uint64_t)s * kMnStep,
                           id_mn, (ii > 0 || s > 0) ? 1u : 0u);
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_ss(tmem + 384, dsa + koff(s, 0), qm + (uint64_t)s * kMnStep, id_mn,
                           (ii > 0 || s > 0) ? 1u : 0u);
                mma_commit(&bars->qd_empty[pst]);
                // A = K^T (M = head dim over K's two boxes), B = dS^T (N = 64
                // queries, one swizzle atom); k-step s = keys [16 s, 16 s + 16)
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_ss(tmem + kColDQ, mndesc(sK + 2048 * s, kHalf128),
                           mndesc(sDS + 2048 * s, kQ64Bytes), id_dq, s > 0 ? 1u : 0u);
                mma_commit(&bars->dq_full);
            };
            // iteration i: S^T(i); once the softmax has read dP^T(i - 1),
            // dP^T(i); once it is done with tile i - 1, the gradient products
            // of tile i - 1
            for (int i = 0; ok && i < kt.nq; ++i) {
                const int st = i % kQdStages;
                const int buf = i & 1;
                if (!(ok = wait(&bars->qd_full[st], (i / kQdStages) & 1, ctl))) break;
                tc_fence_after();
                const uint64_t qd = kdesc(sQ + st * kQ64Bytes);
                const uint64_t dod = kdesc(sDO + st * kQ64Bytes);
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_ss(tmem + 64 * buf, kd + koff(s, kHalf128), qd + koff(s, kHalf64), id_n64,
                           s > 0 ? 1u : 0u);
                if (i > 0) {
                    if (!(ok = wait(&bars->dp_free, (i - 1) & 1, ctl))) break;
                    tc_fence_after();
                }
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_ss(tmem + kColDP, vd + koff(s, kHalf128), dod + koff(s, kHalf64), id_n64,
                           s > 0 ? 1u : 0u);
                mma_commit(&bars->s_full[buf]);
                if (i > 0) {
                    if (!(ok = wait(&bars->p_full[(i - 1) & 1], ((i - 1) >> 1) & 1, ctl))) break;
                    grad_mma(i - 1);
                }
            }
            if (ok && (ok = wait(&bars->p_full[(kt.nq - 1) & 1], ((kt.nq - 1) >> 1) & 1, ctl))) {
                grad_mma(kt.nq - 1);
                mma_commit(&bars->o_done);
            }
            mma_commit(&bars->drain);
            if (!mbar_wait_bounded(&bars->drain, 0, nullptr, kDrainLimitNs))
                atomicOr(&g_bwd_status, 1u);
        }
    } else {
        regs_inc<kRegsSoftmax>();
        // -------------------------------------------------- P^T, dS^T, and the dQ reduction
        const int wg = warp >> 2;        // query columns [32 wg, 32 wg + 32) of every tile
        const int quarter = warp & 3;    // tensor-memory lanes (keys; head dim for dQ^T)
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const uint64_t sl2x2 = f2_pack(p.sl2, p.sl2);
        // this thread's key row of dS^T: 128 bytes (64 queries), 16-byte chunk
        // c stored at c ^ (row % 8) (the 128-byte swizzle of the operands)
        const int krow = quarter * 32 + lane;
        uint8_t* ds_row = smem + Smem::ds_off + (krow >> 3) * 1024 + (krow & 7) * 128;
        // keys past the tile's end (the next window's, or padding) and padded
        // conditioning keys are real rows of K: their dS^T must not reach dQ
        const int key = kt.krow0 + krow;
        const bool key_ok = key < kt.kend && !(kt.seg == 1 && key >= kt.L);
        float* blk = reinterpret_cast<float*>(smem + Smem::dq_off + warp * kBlockBytes);
        // Adds this warp's block of dQ^T of query tile j (head dim [32 quarter,
        // +32) x queries [32 wg, +32), read from tensor memory into r) into
        // the accumulator, staged in shared memory as 32 query rows x 32 floats.
        auto reduce_dq = [&](int j, const uint32_t (&r)[32]) {
            if (lane == 0) bulk_wait_group_read<0>();   // the previous block has left
            __syncwarp();
#pragma unroll
            for (int q = 0; q < 32; ++q) blk[q * 32 + lane] = __uint_as_float(r[q]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                int qs;
                const int row = query_row(kt, j, qs);
                tma_reduce_add_4d(&p.tm_acc, blk, 32 * quarter, h,
                                  (qs ? p.N[0] : 0) + row + 32 * wg, b);
                bulk_commit_group();
            }
        };
        const uint32_t tDQ = tmem + kColDQ + 32 * wg + lane_off;
        bool ok = true;
        for (int i = 0; i < kt.nq; ++i) {
            const int buf = i & 1;
            const int st = i % kQdStages;
            if (!(ok = wait_warp(&bars->s_full[buf], (i >> 1) & 1, ctl))) break;
            if (!(ok = wait_warp(&bars->l_full[st], (i / kQdStages) & 1, ctl))) break;
            tc_fence_after();
            uint32_t pp[16], pd[16];
            const uint32_t tS = tmem + 64 * buf + 32 * wg + lane_off;
            {
                uint32_t sr[32], dr[32];
                tmem_ld32(tS, sr);
                tmem_ld32(tmem + kColDP + 32 * wg + lane_off, dr);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->dp_free);
                p_ds(sr, dr, lbuf + st * 64 + 32 * wg, sl2x2, pp, pd);
            }
            if (!key_ok) {
#pragma unroll
                for (int c = 0; c < 16; ++c) pd[c] = 0u;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->l_empty[st]);
            uint32_t r[32];
            if (i > 0) {   // dQ^T of tile i - 1 formed; dS^T's buffer is free
                if (!(ok = wait_warp(&bars->dq_full, (i - 1) & 1, ctl))) break;
                tc_fence_after();
            }
            tmem_ld32(tDQ, r);   // dQ^T of tile i - 1 (not used at i = 0)
            tmem_st16(tS, pp);
#pragma unroll
            for (int c = 0; c < 4; ++c)
                *reinterpret_cast<uint4*>(ds_row + 16 * ((4 * wg + c) ^ (krow & 7))) =
                    make_uint4(pd[4 * c], pd[4 * c + 1], pd[4 * c + 2], pd[4 * c + 3]);
            fence_proxy_async_smem();
            tmem_wait_ld();
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->p_full[buf]);
            if (i > 0) reduce_dq(i - 1, r);
        }
        if (ok && (ok = wait_warp(&bars->dq_full, (kt.nq - 1) & 1, ctl))) {
            tc_fence_after();
            uint32_t r[32];
            tmem_ld32(tDQ, r);
            tmem_wait_ld();
            reduce_dq(kt.nq - 1, r);
        }
        if (ok) ok = wait_warp(&bars->o_done, 0, ctl);
        tc_fence_after();
        store_dkdv(p, kt, tmem, quarter, wg, lane, ok, h, b);
        if (lane == 0) bulk_wait_group<0>();   // reduce-adds complete before the CTA ends
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace fused

}  // namespace dkv

// ======================================================================
// fp32 CUDA-core backward (fp32 inputs, 1e-4 accuracy)
// ======================================================================

// One warp per query row: dQ_i = scale sum_j P_ij (dO_i.v_j - D_i) k_j.
__global__ void __launch_bounds__(256)
dq_f32_kernel(const float* __restrict__ qv, const float* __restrict__ kv,
              const float* __restrict__ vv, const float* __restrict__ qc,
              const float* __restrict__ kc, const float* __restrict__ vc,
              const int32_t* __restrict__ ctx_len, const float* __restrict__ dov,
              const float* __restrict__ doc, const float* __restrict__ lse,
              const float* __restrict__ delta, float* dqv, float* dqc, int Nv, int Nc, int H,
              float scale, bool windowed, const __grid_constant__ WindowTable win) {
    const int lane = threadIdx.x & 31;
    const int i = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
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
    float4* dst = reinterpret_cast<float4*>((vis ? dqv : dqc) + qrow * 128) + lane;
    if (!vis && i - Nv >= L) {
        *dst = make_float4(0.f, 0.f, 0.f, 0.f);
        return;
    }
    const size_t lr = ((size_t)b * H + h) * (size_t)(Nv + Nc) + i;
    const float li = lse[lr], di = delta[lr];
    const float4 q = reinterpret_cast<const float4*>((vis ? qv : qc) + qrow * 128)[lane];
    const float4 g = reinterpret_cast<const float4*>((vis ? dov : doc) + qrow * 128)[lane];
    int k0 = 0, k1 = Nv;   // visual keys [k0, k1): all, or the query's window (window-major)
    if (windowed && vis) {
        int w = 0;
        while (w + 1 < win.count && win.w[w + 1].start <= i) ++w;
        k0 = win.w[w].start;
        k1 = k0 + win.w[w].te * win.w[w].he * win.w[w].we;
    }
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int seg = 0; seg < 2; ++seg) {
        const int nk = seg == 0 ? k1 : L;
        const int Ns = seg == 0 ? Nv : Nc;
        const float* K = seg == 0 ? kv : kc;
        const float* V = seg == 0 ? vv : vc;
        for (int j = seg == 0 ? k0 : 0; j < nk; ++j) {
            const size_t kr = ((size_t)b * Ns + j) * H + h;
            const float4 k = reinterpret_cast<const float4*>(K + kr * 128)[lane];
            const float4 v = reinterpret_cast<const float4*>(V + kr * 128)[lane];
            float s = q.x * k.x + q.y * k.y + q.z * k.z + q.w * k.w;
            float dp = g.x * v.x + g.y * v.y + g.z * v.z + g.w * v.w;
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) {
                s += __shfl_xor_sync(0xffffffffu, s, o);
                dp += __shfl_xor_sync(0xffffffffu, dp, o);
            }
            const float ds = expf(s * scale - li) * (dp - di);
            acc.x += ds * k.x;
            acc.y += ds * k.y;
            acc.z += ds * k.z;
            acc.w += ds * k.w;
        }
    }
    *dst = make_float4(acc.x * scale, acc.y * scale, acc.z * scale, acc.w * scale);
}

// One warp per key row: dV_j = sum_i P_ij dO_i, dK_j = scale sum_i dS_ij q_i.
__global__ void __launch_bounds__(256)
dkdv_f32_kernel(const float* __restrict__ qv, const float* __restrict__ kv,
                const float* __restrict__ vv, const float* __restrict__ qc,
                const float* __restrict__ kc, const float* __restrict__ vc,
                const int32_t* __restrict__ ctx_len, const float* __restrict__ dov,
                const float* __restrict__ doc, const float* __restrict__ lse,
                const float* __restrict__ delta, float* dkv, float* dvv, float* dkc, float* dvc,
                int Nv, int Nc, int H, float scale, bool windowed,
                const __grid_constant__ WindowTable win) {
    const int lane = threadIdx.x & 31;
    const int j = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int h = blockIdx.y;
    const int b = blockIdx.z;
    if (j >= Nv + Nc) return;
    int L = Nc;
    if (ctx_len) {
        L = ctx_len[b];
        L = L < 0 ? 0 : (L > Nc ? Nc : L);
    }
    const bool vis = j < Nv;
    const size_t kr = vis ? ((size_t)b * Nv + j) * H + h : ((size_t)b * Nc + (j - Nv)) * H + h;
    float4* dk_dst = reinterpret_cast<float4*>((vis ? dkv : dkc) + kr * 128) + lane;
    float4* dv_dst = reinterpret_cast<float4*>((vis ? dvv : dvc) + kr * 128) + lane;
    if (!vis && j - Nv >= L) {
        *dk_dst = make_float4(0.f, 0.f, 0.f, 0.f);
        *dv_dst = make_float4(0.f, 0.f, 0.f, 0.f);
        return;
    }
    const float4 k = reinterpret_cast<const float4*>((vis ? kv : kc) + kr * 128)[lane];
    const float4 v = reinterpret_cast<const float4*>((vis ? vv : vc) + kr * 128)[lane];
    float4 ak = make_float4(0.f, 0.f, 0.f, 0.f), av = ak;
    const size_t lb = ((size_t)b * H + h) * (size_t)(Nv + Nc);
    int q0 = 0, q1 = Nv;   // visual queries [q0, q1) that see this key
    if (windowed && vis) {
        int w = 0;
        while (w + 1 < win.count && win.w[w + 1].start <= j) ++w;
        q0 = win.w[w].start;
        q1 = q0 + win.w[w].te * win.w[w].he * win.w[w].we;
    }
    for (int seg = 0; seg < 2; ++seg) {
        const int nq = seg == 0 ? q1 : L;
        const int Ns = seg == 0 ? Nv : Nc;
        const float* Q = seg == 0 ? qv : qc;
        const float* G = seg == 0 ? dov : doc;
        for (int i = seg == 0 ? q0 : 0; i < nq; ++i) {
            const size_t qr = ((size_t)b * Ns + i) * H + h;
            const float4 q = reinterpret_cast<const float4*>(Q + qr * 128)[lane];
            const float4 g = reinterpret_cast<const float4*>(G + qr * 128)[lane];
            float s = q.x * k.x + q.y * k.y + q.z * k.z + q.w * k.w;
            float dp = g.x * v.x + g.y * v.y + g.z * v.z + g.w * v.w;
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) {
                s += __shfl_xor_sync(0xffffffffu, s, o);
                dp += __shfl_xor_sync(0xffffffffu, dp, o);
            }
            const size_t li = lb + (seg ? Nv + i : i);
            const float pij = expf(s * scale - lse[li]);
            const float ds = pij * (dp - delta[li]);
            av.x += pij * g.x;
            av.y += pij * g.y;
            av.z += pij * g.z;
            av.w += pij * g.w;
            ak.x += ds * q.x;
            ak.y += ds * q.y;
            ak.z += ds * q.z;
            ak.w += ds * q.w;
        }
    }
    *dk_dst = make_float4(ak.x * scale, ak.y * scale, ak.z * scale, ak.w * scale);
    *dv_dst = av;
}

template <typename T>
cudaError_t run_delta(const void* ov, const void* dov, const void* oc, const void* doc,
                      const int32_t* ctx_len, float* delta, int B, int Nv, int Nc, int H,
                      cudaStream_t s, float* acc = nullptr) {
    const long long units = (long long)B * (Nv + Nc) * H;
    if (units == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    constexpr int GPW = 32 / (128 / (16 / sizeof(T)));
    long long blocks = (units + 8LL * GPW * 4 - 1) / (8LL * GPW * 4);
    if (blocks > 8LL * sms) blocks = 8LL * sms;
    delta_kernel<T><<<(unsigned)blocks, 256, 0, s>>>(
        static_cast<const T*>(ov), static_cast<const T*>(dov), static_cast<const T*>(oc),
        static_cast<const T*>(doc), ctx_len, delta, acc, Nv, Nc, H, (uint32_t)units);
    return cudaGetLastError();
}

// dQ = softmax_scale * accumulator: fp32 [B, Nv + Nc, H, 128] -> bf16 dq_vis
// [B, Nv, H, 128] and dq_ctx [B, Nc, H, 128].  16 lanes per (sample, joint
// row, head) row, 8 elements each.
__global__ void __launch_bounds__(256)
dq_convert_kernel(const float* __restrict__ acc, __nv_bfloat16* __restrict__ dqv,
                  __nv_bfloat16* __restrict__ dqc, int Nv, int Nc, int H, float scale,
                  uint32_t rows) {
    const uint32_t Nt = (uint32_t)(Nv + Nc);
    const int e = (threadIdx.x & 15) * 8;
    const uint32_t step = gridDim.x * (blockDim.x / 16);
    for (uint32_t r = blockIdx.x * (blockDim.x / 16) + threadIdx.x / 16; r < rows; r += step) {
        const uint32_t hh = r % (uint32_t)H;
        const uint32_t bj = r / (uint32_t)H;
        const uint32_t jr = bj % Nt;
        const uint32_t bb = bj / Nt;
        const float4* src = reinterpret_cast<const float4*>(acc + (size_t)r * 128 + e);
        const float4 x = __ldcs(src), y = __ldcs(src + 1);
        __nv_bfloat16* dst =
            (int)jr < Nv ? dqv + (((size_t)bb * Nv + jr) * H + hh) * 128 + e
                         : dqc + (((size_t)bb * Nc + (jr - Nv)) * H + hh) * 128 + e;
        *reinterpret_cast<uint4*>(dst) =
            make_uint4(pack_bf16x2(x.x * scale, x.y * scale), pack_bf16x2(x.z * scale, x.w * scale),
                       pack_bf16x2(y.x * scale, y.y * scale), pack_bf16x2(y.z * scale, y.w * scale));
    }
}

// Refuses to launch unless the compiled kernel uses exactly kRegsLaunch
// registers per thread (the register split would otherwise wait for ever),
// and raises its shared-memory limit once per device.
template <typename K>
cudaError_t prepare(K kernel, int smem, bool* done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (done[dev]) return cudaSuccess;
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kernel);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != kRegsLaunch) return cudaErrorInvalidKernelImage;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    done[dev] = true;
    return cudaSuccess;
}

}  // namespace bwd

int launch_joint_attention_bwd_bf16(const void* qv, const void* kv, const void* vv,
                                    const void* qc, const void* kc, const void* vc,
                                    const int32_t* ctx_len, const void* ov, const void* oc,
                                    const void* dov, const void* doc, const float* lse,
                                    float* delta, void* dqv, void* dkv, void* dvv, void* dqc,
                                    void* dkc, void* dvc, int B, int Nv, int Nc, int H,
                                    float softmax_scale, cudaStream_t s, const WindowTable* win,
                                    float* dq_acc) {
    using namespace bwd;
    if (!encode_fn()) return -1;
    if (B == 0 || Nv + Nc == 0) return 0;
    cudaError_t e =
        run_delta<__nv_bfloat16>(ov, dov, oc, doc, ctx_len, delta, B, Nv, Nc, H, s, dq_acc);
    if (e != cudaSuccess) return (int)e;

    dq::Params pq;
    dkv::Params pk;
    std::memset(&pq, 0, sizeof(pq));
    std::memset(&pk, 0, sizeof(pk));
    const void* src[2][4] = {{qv, kv, vv, dov}, {qc, kc, vc, doc}};
    const int N[2] = {Nv, Nc};
    for (int sg = 0; sg < 2; ++sg) {
        if (N[sg] == 0) continue;
        bool good = encode_tokens(&pq.tm_q[sg], src[sg][0], B, N[sg], H, 128) &&
                    encode_tokens(&pq.tm_k[sg], src[sg][1], B, N[sg], H, 128) &&
                    encode_tokens(&pq.tm_v[sg], src[sg][2], B, N[sg], H, 128) &&
                    encode_tokens(&pq.tm_do[sg], src[sg][3], B, N[sg], H, 128) &&
                    encode_tokens(&pk.tm_k[sg], src[sg][1], B, N[sg], H, 128) &&
                    encode_tokens(&pk.tm_v[sg], src[sg][2], B, N[sg], H, 128) &&
                    encode_tokens(&pk.tm_q[sg], src[sg][0], B, N[sg], H, 64) &&
                    encode_tokens(&pk.tm_do[sg], src[sg][3], B, N[sg], H, 64);
        if (!good) return 1000 + (int)cudaErrorInvalidValue;
    }
    const float sl2 = softmax_scale * kLog2e;
    pq.dq[0] = static_cast<__nv_bfloat16*>(dqv);
    pq.dq[1] = static_cast<__nv_bfloat16*>(dqc);
    pk.dk[0] = static_cast<__nv_bfloat16*>(dkv);
    pk.dk[1] = static_cast<__nv_bfloat16*>(dkc);
    pk.dv[0] = static_cast<__nv_bfloat16*>(dvv);
    pk.dv[1] = static_cast<__nv_bfloat16*>(dvc);
    pq.lse = pk.lse = lse;
    pq.delta = pk.delta = delta;
    pq.ctx_len = pk.ctx_len = ctx_len;
    pq.N[0] = pk.N[0] = Nv;
    pq.N[1] = pk.N[1] = Nc;
    pq.H = pk.H = H;
    pq.q_tiles_vis = pk.k_tiles_vis = (Nv + 127) / 128;
    pq.sl2 = pk.sl2 = sl2;
    pq.scale = pk.scale = softmax_scale;
    pq.wait_ns = pk.wait_ns = wait_timeout_ns();

    static bool dq_ready[64] = {false}, dkv_ready[64] = {false}, fused_ready[64] = {false};
    const int smem_q = dq::Smem::total + 1024;
    const int smem_k = dkv::Smem::total + 1024;
    const int smem_f = dkv::fused::Smem::total + 1024;
    if (dq_acc) {
        if (!encode_acc_f32(&pk.tm_acc, dq_acc, B, Nv + Nc, H)) return 1000 + (int)cudaErrorInvalidValue;
        if ((e = prepare(dkv::fused::dkdvq_kernel, smem_f, fused_ready)) != cudaSuccess)
            return (int)e;
    } else {
        if ((e = prepare(dq::dq_kernel, smem_q, dq_ready)) != cudaSuccess) return (int)e;
        if ((e = prepare(dkv::dkdv_kernel, smem_k, dkv_ready)) != cudaSuccess) return (int)e;
    }
    dim3 grid((Nv + 127) / 128 + (Nc + 127) / 128, H, B);
    if (win) {
        // window mode: the conditioning tiles first, then each window's tiles
        // of 128 rows (queries for dq_kernel, keys for dkdv_kernel)
        pq.windowed = pk.windowed = 1;
        pq.win = pk.win = *win;
        pq.cond_tiles = pk.cond_tiles = (Nc + 127) / 128;
        int tiles = 0;
        for (int w = 0; w < win->count; ++w) {
            pq.tile_start[w] = pk.tile_start[w] = tiles;
            tiles += (win->w[w].te * win->w[w].he * win->w[w].we + 127) / 128;
        }
        pq.tile_start[win->count] = pk.tile_start[win->count] = tiles;
        grid.x = (unsigned)(pq.cond_tiles + tiles);
    }
    if (dq_acc) {
        dkv::fused::dkdvq_kernel<<<grid, kThreads, smem_f, s>>>(pk);
        if ((e = cudaGetLastError()) != cudaSuccess) return (int)e;
        const long long rows = (long long)B * (Nv + Nc) * H;
        int dev = 0, sms = 148;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        long long blocks = (rows + 15) / 16;
        if (blocks > 8LL * sms) blocks = 8LL * sms;
        dq_convert_kernel<<<(unsigned)blocks, 256, 0, s>>>(
            dq_acc, static_cast<__nv_bfloat16*>(dqv), static_cast<__nv_bfloat16*>(dqc), Nv, Nc, H,
            softmax_scale, (uint32_t)rows);
        return (int)cudaGetLastError();
    }
    dq::dq_kernel<<<grid, kThreads, smem_q, s>>>(pq);
    if ((e = cudaGetLastError()) != cudaSuccess) return (int)e;
    dkv::dkdv_kernel<<<grid, kThreads, smem_k, s>>>(pk);
    return (int)cudaGetLastError();
}

cudaError_t launch_joint_attention_bwd_f32(const float* qv, const float* kv, const float* vv,
                                           const float* qc, const float* kc, const float* vc,
                                           const int32_t* ctx_len, const float* ov,
                                           const float* oc, const float* dov, const float* doc,
                                           const float* lse, float* delta, float* dqv, float* dkv,
                                           float* dvv, float* dqc, float* dkc, float* dvc, int B,
                                           int Nv, int Nc, int H, float softmax_scale,
                                           cudaStream_t s, const WindowTable* win) {
    using namespace bwd;
    const int rows = Nv + Nc;
    if (rows == 0 || B == 0) return cudaSuccess;
    cudaError_t e = run_delta<float>(ov, dov, oc, doc, ctx_len, delta, B, Nv, Nc, H, s);
    if (e != cudaSuccess) return e;
    WindowTable tab{};
    if (win) tab = *win;
    const dim3 grid((rows + 7) / 8, H, B);
    dq_f32_kernel<<<grid, 256, 0, s>>>(qv, kv, vv, qc, kc, vc, ctx_len, dov, doc, lse, delta, dqv,
                                       dqc, Nv, Nc, H, softmax_scale, win != nullptr, tab);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    dkdv_f32_kernel<<<grid, 256, 0, s>>>(qv, kv, vv, qc, kc, vc, ctx_len, dov, doc, lse, delta,
                                         dkv, dvv, dkc, dvc, Nv, Nc, H, softmax_scale,
                                         win != nullptr, tab);
    return cudaGetLastError();
}

cudaError_t read_and_clear_bwd_status(unsigned int* out) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_bwd_status, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_bwd_status, &zero, sizeof(unsigned int));
}

}  // namespace mmdit
