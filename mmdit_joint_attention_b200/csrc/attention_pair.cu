// Joint attention forward on CTA pairs (tcgen05 cta_group::2): the two CTAs
// of a cluster share one MMA-issuing thread, and every product covers 256
// query rows, 128 in each CTA.  What it computes is joint_attn_bf16_kernel's
// plain form (the joint attention of the "Vimoo 1.0" research page, section
// 2.2, over the concatenated visual and conditioning tokens, padded
// conditioning keys masked, bf16 in and out): same tiles, same per-row
// softmax, same order of every sum, so the outputs are bit for bit those of
// that kernel.  What changes:
//   * each CTA holds half of every K tile (keys 64 r .. 64 r + 63 of the
//     128-key tile, r the CTA's rank in the pair) and half of every V tile
//     (head dims 64 r .. 64 r + 63); a product reads the B operand from both
//     CTAs, so each SM's shared memory takes half the K/V fills and serves
//     half the B-operand reads;
//   * one thread (rank 0, warp 9) issues the pair's products; an instruction
//     costs it about what an M = 128 one costs the one-SM kernel's issuer, so
//     the products reach each SM at about the same rate, each with less
//     shared-memory traffic behind it;
//   * both CTAs' copies complete on the leader's barriers (the cta_group::2
//     form of the TMA load, no multicast); the leader's commits arrive on the
//     barrier at the same offset in both CTAs; the softmax warps of both CTAs
//     release P on the leader's barrier through its cluster address.
// Plain form only (no 3D windows, no in-kernel Q normalisation, no row
// log-sum-exp output, no split tail); the one-SM kernel covers the rest.
// Every mbarrier wait is bounded; a wait that runs out sets this kernel's
// status word, and each CTA leaves through the closing cluster barrier, which
// both CTAs reach on every path.
#include <cstdint>
#include <cstring>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"
#include "tensor_map.h"

namespace mmdit {
namespace pair {

// Bit 0: a bounded wait expired in the pair kernel.
__device__ unsigned int g_pair_status = 0;

constexpr int kBlockM = 128, kBlockN = 128, kHeadDim = 128;
constexpr int kStages = 2;
constexpr int kTileBytes = 128 * 128 * 2;   // a Q tile: 128 rows x 128 bf16
constexpr int kQBox = kTileBytes / 2;       // 128 rows x 64 cols
constexpr int kKHalf = 64 * 128 * 2;        // 64 keys x 128 dims (two 8 KB boxes)
constexpr int kKBox = kKHalf / 2;
constexpr int kVHalf = 128 * 64 * 2;        // 128 keys x 64 dims (one box)
constexpr int kThreads = 384;
constexpr int kRegsProducer = 72, kRegsSoftmax = 216;
constexpr uint64_t kDrainLimitNs = 200000000ull;

struct Smem {
    static constexpr int q_off = 0;                               // 2 tiles
    static constexpr int k_off = q_off + 2 * kTileBytes;          // kStages K halves
    static constexpr int v_off = k_off + kStages * kKHalf;        // kStages V halves
    static constexpr int bar_off = v_off + kStages * kVHalf;
    static constexpr int total = bar_off + 256;
};

struct Params {
    CUtensorMap tm_q[2];   // 128-row boxes
    CUtensorMap tm_k[2];   // 64-row boxes
    CUtensorMap tm_v[2];   // 128-row boxes
    __nv_bfloat16* out[2];
    const int32_t* ctx_len;
    int N[2];
    int H;
    int q_tiles_vis, q_tiles;
    float scale_log2;
    uint64_t wait_ns;
};

struct Bars {
    uint64_t q_full;
    uint64_t k_full[kStages], k_empty[kStages];
    uint64_t s_full[2], o_done[2];
    uint64_t p_full[2];
    uint64_t drain;
    uint64_t wait_ns;
    uint32_t tmem_base;
    uint32_t abort;
};

// ------------------------------------------------------------ cluster helpers
__device__ __forceinline__ uint32_t cta_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
                 ::: "memory");
}
// shared::cluster address of `p` (a shared::cta address here) in CTA `rank`
__device__ __forceinline__ uint32_t mapa(const void* p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}
__device__ __forceinline__ void arrive_remote(uint32_t bar_cluster) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster)
                 : "memory");
}
// 4-D tiled load into this CTA's shared memory completing on a barrier of
// either CTA of the pair
__device__ __forceinline__ void tma_load_4d_pair(void* dst, const void* tmap, uint32_t bar_cluster,
                                                 int c0, int c1, int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
        "l"(tmap), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}
__device__ __forceinline__ void mma2_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                        uint32_t acc) {
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
                 "l"(a), "l"(b), "r"(idesc), "r"(acc)
                 : "memory");
}
__device__ __forceinline__ void mma2_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc,
                                        uint32_t acc) {
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
                 "r"(a), "l"(b), "r"(idesc), "r"(acc)
                 : "memory");
}
// commit of this thread's cta_group::2 MMAs to the barrier at the same
// offset in both CTAs of the pair
__device__ __forceinline__ void commit2_both(uint64_t* bar) {
    asm volatile("{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
                 "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}"
                 ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void commit2_local(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void alloc2(uint32_t* dst, uint32_t n) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst)), "r"(n) : "memory");
}
__device__ __forceinline__ void relinquish2() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void dealloc2(uint32_t t, uint32_t n) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(t), "r"(n)
                 : "memory");
}

__device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity, Bars* bars) {
    if (mbar_wait_bounded(bar, parity, &bars->abort, bars->wait_ns)) return true;
    bars->abort = 1;
    atomicOr(&g_pair_status, 1u);
    return false;
}
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, Bars* bars) {
    const bool ok = wait(bar, parity, bars);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void tile_of(const Params& p, int t, int& s, int& row0) {
    if (t < p.q_tiles_vis) { s = 0; row0 = t * kBlockM; }
    else { s = 1; row0 = (t - p.q_tiles_vis) * kBlockM; }
}

// The per-row softmax steps below are those of joint_attn_bf16_kernel
// (attention_tc.cu), kept identical so that both kernels give the same bits
// (tests/test_gpu_pair.py compares them on every run).
// O row of this thread *= f, 32 tensor-memory columns at a time.
__device__ __forceinline__ void rescale_o(uint32_t tO, float f) {
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * c, o);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
        tmem_st32(tO + 32 * c, o);
    }
}
// P = 2^(s * scale_log2 - m) for keys [64 h, 64 h + 64) of one score row,
// packed two bf16 keys per column into rh; returns their sum.
__device__ __forceinline__ float exp_half(const float (&sv)[128], uint32_t (&rh)[32], int h,
                                          uint64_t sl2x2, uint64_t negm2) {
    uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
    for (int c = 0; c < 32; ++c) {
        const int k = 64 * h + 2 * c;
        const uint64_t x2 = f2_fma(f2_pack(sv[k], sv[k + 1]), sl2x2, negm2);
        float x0, x1;
        f2_unpack(x2, x0, x1);
        const uint64_t e2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
        acc[c & 3] = f2_add(acc[c & 3], e2);
        float a0, a1;
        f2_unpack(e2, a0, a1);
        rh[c] = pack_bf16x2(a0, a1);
    }
    const uint64_t s2 = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
    float lo, hi;
    f2_unpack(s2, lo, hi);
    return lo + hi;
}

__global__ void __launch_bounds__(kThreads, 1) pair_kernel(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars* bars = reinterpret_cast<Bars*>(smem + Smem::bar_off);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cta_rank();
    const int cl = blockIdx.x >> 1;
    const int h = blockIdx.y;
    const int b = blockIdx.z;
    // slot i of this CTA: query tile 4 cl + 2 i + rank (the pair's MMA for
    // slot i covers the slot-i tiles of both CTAs); false if past the end
    auto slot = [&](int i, int& sg, int& r0) -> bool {
        const int t = 4 * cl + 2 * i + (int)rank;
        sg = 0;
        r0 = 0;
        if (t >= p.q_tiles) return false;
        tile_of(p, t, sg, r0);
        return true;
    };
    int L = p.N[1];
    if (p.ctx_len) {
        L = p.ctx_len[b];
        L = L < 0 ? 0 : (L > p.N[1] ? p.N[1] : L);
    }
    const int kv_vis = (p.N[0] + kBlockN - 1) / kBlockN;
    const int n_kv = kv_vis + (L + kBlockN - 1) / kBlockN;

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&bars->k_full[i], 1);
            mbar_init(&bars->k_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->s_full[i], 1);
            mbar_init(&bars->o_done[i], 1);
            mbar_init(&bars->p_full[i], 8);   // 4 softmax warps in each CTA of the pair
        }
        mbar_init(&bars->drain, 1);
        bars->abort = 0;
        bars->wait_ns = p.wait_ns;
        fence_barrier_init();
    }
    if (warp == 8) {
        alloc2(&bars->tmem_base, 512);
        relinquish2();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const uint32_t sQ = smem_u32(smem + Smem::q_off);
    const uint32_t sK = smem_u32(smem + Smem::k_off);
    const uint32_t sV = smem_u32(smem + Smem::v_off);

    if (warp >= 8) {
        regs_dec<kRegsProducer>();
        if (warp == 8 && lane == 0) {
            // ------------------------------------------------ TMA: this CTA's Q tiles and K / V halves
            const uint32_t bq = mapa(&bars->q_full, 0);
            const uint32_t bk0 = mapa(&bars->k_full[0], 0), bk1 = mapa(&bars->k_full[1], 0);
            int nq_pair = 0;
            for (int t = 4 * cl; t < 4 * cl + 4; ++t) nq_pair += t < p.q_tiles ? 1 : 0;
            if (rank == 0) mbar_arrive_expect_tx(&bars->q_full, nq_pair * kTileBytes);
            for (int i = 0; i < 2; ++i) {
                int sg, r0;
                if (!slot(i, sg, r0)) continue;
                uint8_t* d = smem + Smem::q_off + i * kTileBytes;
                tma_load_4d_pair(d, &p.tm_q[sg], bq, 0, h, r0, b);
                tma_load_4d_pair(d + kQBox, &p.tm_q[sg], bq, 64, h, r0, b);
            }
            for (int j = 0; j <= n_kv; ++j) {
                const int st = j & 1;
                if (!wait(&bars->k_empty[st], ((j >> 1) & 1) ^ 1, bars)) break;
                const uint32_t bk = st ? bk1 : bk0;
                if (rank == 0)
                    mbar_arrive_expect_tx(&bars->k_full[st],
                                          2 * ((j < n_kv ? kKHalf : 0) + (j > 0 ? kVHalf : 0)));
                if (j < n_kv) {   // K(j): keys [64 rank, 64 rank + 64) of the tile
                    const int sg = j < kv_vis ? 0 : 1;
                    const int row = (sg ? j - kv_vis : j) * kBlockN + 64 * (int)rank;
                    uint8_t* d = smem + Smem::k_off + st * kKHalf;
                    tma_load_4d_pair(d, &p.tm_k[sg], bk, 0, h, row, b);
                    tma_load_4d_pair(d + kKBox, &p.tm_k[sg], bk, 64, h, row, b);
                }
                if (j > 0) {      // V(j - 1): head dims [64 rank, 64 rank + 64)
                    const int jj = j - 1;
                    const int sg = jj < kv_vis ? 0 : 1;
                    const int row = (sg ? jj - kv_vis : jj) * kBlockN;
                    tma_load_4d_pair(smem + Smem::v_off + st * kVHalf, &p.tm_v[sg], bk,
                                     64 * (int)rank, h, row, b);
                }
            }
        } else if (warp == 9 && lane == 0 && rank == 0) {
            // ------------------------------------------------ MMA issuer of the pair
            constexpr uint32_t idesc_qk = idesc_bf16_f32(256, 128, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(256, 128, 0, 1);
            bool ok = wait(&bars->q_full, 0, bars);
            const uint64_t dq0 = smem_desc_sw128(sQ, 16, 1024);
            const uint64_t dq1 = smem_desc_sw128(sQ + kTileBytes, 16, 1024);
            const uint64_t dk0 = smem_desc_sw128(sK, 16, 1024);
            const uint64_t dk1 = smem_desc_sw128(sK + kKHalf, 16, 1024);
            const uint64_t dv0 = smem_desc_sw128(sV, 16, 1024);
            const uint64_t dv1 = smem_desc_sw128(sV + kVHalf, 16, 1024);
            auto qk = [&](int i, int st) {
                const uint64_t dq = i == 0 ? dq0 : dq1;
                const uint64_t dk = st == 0 ? dk0 : dk1;
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    const uint64_t oq = (uint64_t)((s >> 2) * (kQBox >> 4) + (s & 3) * 2);
                    const uint64_t ok_ = (uint64_t)((s >> 2) * (kKBox >> 4) + (s & 3) * 2);
                    mma2_ss(tmem + 128 * i, dq + oq, dk + ok_, idesc_qk, s > 0 ? 1u : 0u);
                }
            };
            auto pv = [&](int i, int st, bool acc, uint32_t par) -> bool {
                const uint64_t dv = st == 0 ? dv0 : dv1;
                if (!wait(&bars->p_full[i], par, bars)) return false;
                tc_fence_after();
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma2_ts(tmem + 256 + 128 * i, tmem + 128 * i + s * 8,
                            dv + (uint64_t)(s * (2048 >> 4)), idesc_pv, (acc || s > 0) ? 1u : 0u);
                return true;
            };
            for (int j = 0; ok && j <= n_kv; ++j) {
                const int st = j & 1;
                if (!(ok = wait(&bars->k_full[st], (j >> 1) & 1, bars))) break;
                for (int i = 0; i < 2; ++i) {
                    if (j > 0 && !(ok = pv(i, st, j > 1, (j - 1) & 1))) break;
                    if (j < n_kv) {
                        if (j == 0) tc_fence_after();
                        qk(i, st);
                        commit2_both(&bars->s_full[i]);
                    } else {
                        commit2_both(&bars->o_done[i]);
                    }
                }
                if (!ok) break;
                commit2_both(&bars->k_empty[st]);
            }
            commit2_local(&bars->drain);
            if (!mbar_wait_bounded(&bars->drain, 0, nullptr, kDrainLimitNs))
                atomicOr(&g_pair_status, 1u);
        }
    } else {
        regs_inc<kRegsSoftmax>();
        const int i = warp >> 2;
        const int quarter = warp & 3;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const uint32_t tS = tmem + i * 128 + lane_off;
        const uint32_t tO = tmem + 256 + i * 128 + lane_off;
        const uint32_t pbar = mapa(&bars->p_full[i], 0);
        const float sl2 = p.scale_log2;
        const uint64_t sl2x2 = f2_pack(sl2, sl2);
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        for (int it = 0; it < n_kv; ++it) {
            if (!(ok = wait_warp(&bars->s_full[i], it & 1, bars))) break;
            tc_fence_after();
            uint32_t r[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, r[c]);
            tmem_wait_ld();
            const int valid = it < kv_vis ? p.N[0] - it * kBlockN : L - (it - kv_vis) * kBlockN;
            float sv[128];
#pragma unroll
            for (int c = 0; c < 128; ++c) sv[c] = __uint_as_float(r[c >> 5][c & 31]);
            if (valid < kBlockN) {
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (c >= valid) sv[c] = -INFINITY;
            }
            float mk[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) mk[k] = fmaxf(sv[k], sv[k + 8]);
#pragma unroll
            for (int c = 16; c < 128; c += 16)
#pragma unroll
                for (int k = 0; k < 8; k += 2)
                    mk[k] = fmax3(mk[k], sv[c + k], sv[c + k + 1]),
                    mk[k + 1] = fmax3(mk[k + 1], sv[c + k + 8], sv[c + k + 9]);
            const float m_tile = fmaxf(fmax3(mk[0], mk[1], mk[2]),
                                       fmaxf(fmax3(mk[3], mk[4], mk[5]), fmaxf(mk[6], mk[7]))) *
                                 sl2;
            if (it == 0) {
                m_run = m_tile;
            } else if (__any_sync(0xffffffffu, m_tile > m_run + 8.0f)) {
                const float m_new = fmaxf(m_run, m_tile);
                const float f = ex2_approx(m_run - m_new);
                m_run = m_new;
                l_run *= f;
                rescale_o(tO, f);
            }
            const uint64_t negm2 = f2_pack(-m_run, -m_run);
            float sum = 0.f;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                sum += exp_half(sv, r[hh], hh, sl2x2, negm2);
                tmem_st32(tS + 32 * hh, r[hh]);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) arrive_remote(pbar);
            l_run += sum;
        }
        if (ok) ok = wait_warp(&bars->o_done[i], 0, bars);
        tc_fence_after();
        int s, r0;
        const bool has = slot(i, s, r0);
        const int row = r0 + quarter * 32 + lane;
        const bool store = has && row < p.N[s];
        const bool zero = !ok || (s == 1 && row >= L);
        const float inv = (l_run > 0.f) ? 1.0f / l_run : 0.f;
        uint4* dst = reinterpret_cast<uint4*>(
            p.out[s] + ((size_t)((size_t)b * p.N[s] + (store ? row : 0)) * p.H + h) * kHeadDim);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + 32 * c, o);
            tmem_wait_ld();
            if (store) {
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    float f[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        f[e] = zero ? 0.f : __uint_as_float(o[8 * v + e]) * inv;
                    dst[4 * c + v] = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                                pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
                }
            }
        }
    }

    // an aborted CTA lets copies it may still have in flight land (its pair's
    // leader counts them, not this CTA), within a bounded time
    if (bars->abort) {
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 2000000ull) {
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 8) {
        tc_fence_after();
        dealloc2(tmem, 512);
    }
}

}  // namespace pair

int launch_joint_attention_pair(const void* qv, const void* kv, const void* vv, const void* qc,
                                const void* kc, const void* vc, const int32_t* ctx_len, void* ov,
                                void* oc, int B, int Nv, int Nc, int H, float softmax_scale,
                                cudaStream_t s) {
    using namespace pair;
    if (!encode_fn()) return -1;
    if (B == 0) return 0;
    Params p;
    std::memset(&p, 0, sizeof(p));
    const void* src[2][3] = {{qv, kv, vv}, {qc, kc, vc}};
    const int N[2] = {Nv, Nc};
    for (int sg = 0; sg < 2; ++sg) {
        if (N[sg] == 0) continue;
        if (!encode_tokens(&p.tm_q[sg], src[sg][0], B, N[sg], H, 128) ||
            !encode_tokens(&p.tm_k[sg], src[sg][1], B, N[sg], H, 64) ||
            !encode_tokens(&p.tm_v[sg], src[sg][2], B, N[sg], H, 128))
            return 1000 + (int)cudaErrorInvalidValue;
    }
    p.out[0] = static_cast<__nv_bfloat16*>(ov);
    p.out[1] = static_cast<__nv_bfloat16*>(oc);
    p.ctx_len = ctx_len;
    p.N[0] = Nv;
    p.N[1] = Nc;
    p.H = H;
    p.q_tiles_vis = (Nv + kBlockM - 1) / kBlockM;
    p.q_tiles = p.q_tiles_vis + (Nc + kBlockM - 1) / kBlockM;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    p.wait_ns = wait_timeout_ns();
    const int smem = Smem::total + 1024;
    static bool ready[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return (int)e;
    if (dev < 0 || dev >= 64) return (int)cudaErrorInvalidDevice;
    if (!ready[dev]) {
        // the register split (72 + 2 x 216 per thread) needs exactly 168 at launch
        cudaFuncAttributes fa;
        if ((e = cudaFuncGetAttributes(&fa, pair_kernel)) != cudaSuccess) return (int)e;
        if (fa.numRegs != 168) return (int)cudaErrorInvalidKernelImage;
        if ((e = cudaFuncSetAttribute(pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      smem)) != cudaSuccess)
            return (int)e;
        ready[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * ((p.q_tiles + 3) / 4), H, B);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, pair_kernel, p);
    return (int)e;
}

cudaError_t read_and_clear_pair_status(unsigned int* out) {
    cudaError_t e = cudaMemcpyFromSymbol(out, pair::g_pair_status, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(pair::g_pair_status, &zero, sizeof(unsigned int));
}

}  // namespace mmdit
