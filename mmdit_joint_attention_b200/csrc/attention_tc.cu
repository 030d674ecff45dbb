// Joint (concatenated) non-causal attention, bf16 in / bf16 out, on the sm_100a
// tensor cores.
//
// What it computes ("Vimoo 1.0" research page, section 2.2): per (sample, head)
// the visual and conditioning streams' Q, K, V are concatenated, attended
// jointly without a causal mask (Wan 2.1 report, section 4.3.1: DiT attention
// is non-causal), and the output rows are split back into the two streams.
// Conditioning keys at index >= ctx_len[b] are padding and are excluded.
//
// Design (flash-style, one pass over K/V, no score matrix in memory):
//   * The concatenation is never materialised.  Each stream has its own TMA
//     descriptors; key tile j < ceil(Nv/128) comes from the visual stream, the
//     remaining ones from the conditioning stream, and query tiles never
//     straddle the two streams, so the "split back" is just the store target.
//   * A CTA owns two 128-row query tiles of one (b, h) and streams 128-key K/V
//     tiles through a 2-stage shared-memory ring filled by TMA (128-byte
//     swizzle).  Both query tiles reuse every K/V tile.
//   * One thread issues tcgen05.mma: S_i = Q_i K^T into tensor memory (fp32),
//     and O_i += P_i V with P_i read straight from tensor memory.
//   * Two softmax warpgroups (one per query tile, one thread per query row)
//     read S_i from tensor memory, run the online softmax in fp32 in the
//     exp2 domain, and write P_i (bf16) back over S_i.  While one warpgroup
//     does its softmax the tensor core works on the other tile (ping-pong).
//   * The running maximum is only raised (and O rescaled in tensor memory)
//     when it grows by more than 2^8; otherwise exponents use the stale
//     maximum, which is exact after the final division by the row sum and
//     keeps every P below 256.
// Tensor memory: S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512) columns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "internal.h"
#include "ptx.cuh"

namespace mmdit {

// Bit 0: a bounded wait expired in the joint-attention kernel.
__device__ unsigned int g_device_status = 0;

namespace attn {

constexpr int kBlockM = 128;         // query rows per tile
constexpr int kBlockN = 128;         // keys per tile
constexpr int kStages = 2;           // K and V ring depth
constexpr int kTileBytes = 128 * 128 * 2;
constexpr int kHalfBytes = kTileBytes / 2;  // one 64-column TMA box (128 B per row)
constexpr int kThreads = 320;        // warps 0-3 softmax tile 0, 4-7 softmax tile 1, 8 TMA, 9 MMA
constexpr int kWarpLoad = 8;
constexpr int kWarpMma = 9;
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s per pipeline wait
constexpr uint64_t kDrainLimitNs = 200000000ull;   // 0.2 s per drain wait after an abort

struct Smem {
    // tiles are placed first, at 1024-byte aligned offsets (128-byte swizzle atoms)
    static constexpr int q_off = 0;                               // 2 tiles
    static constexpr int k_off = q_off + 2 * kTileBytes;          // kStages tiles
    static constexpr int v_off = k_off + kStages * kTileBytes;    // kStages tiles
    static constexpr int bar_off = v_off + kStages * kTileBytes;
    static constexpr int total = bar_off + 256;
};

struct Params {
    CUtensorMap tm_q[2];  // [0] visual, [1] conditioning
    CUtensorMap tm_k[2];
    CUtensorMap tm_v[2];
    __nv_bfloat16* out[2];
    const int32_t* ctx_len;
    int N[2];           // Nv, Nc
    int H;
    int q_tiles_vis;    // ceil(Nv / 128)
    int q_tiles;        // ceil(Nv / 128) + ceil(Nc / 128)
    float scale_log2;   // softmax_scale * log2(e)
};

struct Bars {
    uint64_t q_full;
    uint64_t k_full[kStages], k_empty[kStages];
    uint64_t v_full[kStages], v_empty[kStages];
    uint64_t s_full[2], p_full[2], o_done[2];
    uint64_t drain;
    uint32_t tmem_base;
    uint32_t abort;
};

__device__ __forceinline__ void tile_of(const Params& p, int t, int& s, int& row0) {
    if (t < p.q_tiles_vis) {
        s = 0;
        row0 = t * kBlockM;
    } else {
        s = 1;
        row0 = (t - p.q_tiles_vis) * kBlockM;
    }
}

__device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity, Bars* bars) {
    if (mbar_wait_bounded(bar, parity, &bars->abort, kWaitLimitNs)) return true;
    bars->abort = 1;
    atomicOr(&g_device_status, 1u);
    return false;
}

// Same, but every lane of the warp gets the same answer (the caller then runs
// warp-collective tcgen05 loads / stores).
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, Bars* bars) {
    const bool ok = wait(bar, parity, bars);
    return __all_sync(0xffffffffu, ok);
}

// K-major operand tile (rows x 128 columns bf16) stored as two 64-column halves
// of 128-byte rows with the 128-byte swizzle; k-step s covers columns
// [16 s, 16 s + 16): half s/4, byte offset 32 (s % 4) inside the row.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile, int s) {
    return smem_desc_sw128(tile + (s >> 2) * kHalfBytes + (s & 3) * 32, 16, 1024);
}
// V tile as an MN-major B operand (keys x head-dim, head-dim contiguous):
// k-step s covers keys [16 s, 16 s + 16) = 2048 bytes; the two 64-wide halves
// of the head dim are kHalfBytes apart (leading byte offset), 8-key groups are
// 1024 bytes apart (stride byte offset).
__device__ __forceinline__ uint64_t desc_v(uint32_t tile, int s) {
    return smem_desc_sw128(tile + s * 2048, kHalfBytes, 1024);
}

__global__ void __launch_bounds__(kThreads, 1) joint_attn_bf16_kernel(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars* bars = reinterpret_cast<Bars*>(smem + Smem::bar_off);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int h = blockIdx.y;
    const int b = blockIdx.z;
    const int t0 = 2 * blockIdx.x;
    const bool has1 = t0 + 1 < p.q_tiles;
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
            mbar_init(&bars->v_full[i], 1);
            mbar_init(&bars->v_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->s_full[i], 1);
            mbar_init(&bars->p_full[i], 128);
            mbar_init(&bars->o_done[i], 1);
        }
        mbar_init(&bars->drain, 1);
        bars->abort = 0;
        fence_barrier_init();
    }
    if (warp == kWarpLoad && n_kv > 0) {
        tmem_alloc(&bars->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    const uint32_t sQ = smem_u32(smem + Smem::q_off);
    const uint32_t sK = smem_u32(smem + Smem::k_off);
    const uint32_t sV = smem_u32(smem + Smem::v_off);

    if (n_kv == 0) {
        // no valid key at all: every output row of this CTA is zero
        for (int tt = 0; tt < 2; ++tt) {
            if (tt == 1 && !has1) break;
            int s, row0;
            tile_of(p, t0 + tt, s, row0);
            for (int r = threadIdx.x; r < kBlockM * 16; r += kThreads) {
                const int row = row0 + r / 16;
                if (row < p.N[s]) {
                    uint4* dst = reinterpret_cast<uint4*>(
                        p.out[s] + ((size_t)(b * (size_t)p.N[s] + row) * p.H + h) * kHeadDim);
                    dst[r % 16] = make_uint4(0, 0, 0, 0);
                }
            }
        }
        return;
    }

    if (warp == kWarpLoad) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            for (int seg = 0; seg < 2; ++seg) {
                if (p.N[seg] > 0) {
                    tma_prefetch_desc(&p.tm_q[seg]);
                    tma_prefetch_desc(&p.tm_k[seg]);
                    tma_prefetch_desc(&p.tm_v[seg]);
                }
            }
            int jk = 0, jv = 0;  // K / V tile loads issued
            int s0, r0, s1 = 0, r1 = 0;
            tile_of(p, t0, s0, r0);
            if (has1) tile_of(p, t0 + 1, s1, r1);
            mbar_arrive_expect_tx(&bars->q_full, (has1 ? 2 : 1) * kTileBytes);
            tma_load_4d(smem + Smem::q_off, &p.tm_q[s0], &bars->q_full, 0, h, r0, b);
            tma_load_4d(smem + Smem::q_off + kHalfBytes, &p.tm_q[s0], &bars->q_full, 64, h, r0, b);
            if (has1) {
                tma_load_4d(smem + Smem::q_off + kTileBytes, &p.tm_q[s1], &bars->q_full, 0, h, r1, b);
                tma_load_4d(smem + Smem::q_off + kTileBytes + kHalfBytes, &p.tm_q[s1], &bars->q_full,
                            64, h, r1, b);
            }
            for (int j = 0; j < n_kv; ++j) {
                const int st = j % kStages;
                const uint32_t ph = (j / kStages) & 1;
                const int seg = j < kv_vis ? 0 : 1;
                const int row = (seg == 0 ? j : j - kv_vis) * kBlockN;
                if (!wait(&bars->k_empty[st], ph ^ 1, bars)) break;
                uint8_t* kt = smem + Smem::k_off + st * kTileBytes;
                mbar_arrive_expect_tx(&bars->k_full[st], kTileBytes);
                tma_load_4d(kt, &p.tm_k[seg], &bars->k_full[st], 0, h, row, b);
                tma_load_4d(kt + kHalfBytes, &p.tm_k[seg], &bars->k_full[st], 64, h, row, b);
                ++jk;
                if (!wait(&bars->v_empty[st], ph ^ 1, bars)) break;
                uint8_t* vt = smem + Smem::v_off + st * kTileBytes;
                mbar_arrive_expect_tx(&bars->v_full[st], kTileBytes);
                tma_load_4d(vt, &p.tm_v[seg], &bars->v_full[st], 0, h, row, b);
                tma_load_4d(vt + kHalfBytes, &p.tm_v[seg], &bars->v_full[st], 64, h, row, b);
                ++jv;
            }
            if (bars->abort) {
                // let every copy already issued land before the CTA exits
                volatile uint32_t never = 0;
                mbar_wait_bounded(&bars->q_full, 0, &never, kDrainLimitNs);
                for (int j = (jk > kStages ? jk - kStages : 0); j < jk; ++j)
                    mbar_wait_bounded(&bars->k_full[j % kStages], (j / kStages) & 1, &never,
                                      kDrainLimitNs);
                for (int j = (jv > kStages ? jv - kStages : 0); j < jv; ++j)
                    mbar_wait_bounded(&bars->v_full[j % kStages], (j / kStages) & 1, &never,
                                      kDrainLimitNs);
            }
        }
    } else if (warp == kWarpMma) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 128, 0, 1);
            const uint32_t tS[2] = {tmem + 0, tmem + 128};
            const uint32_t tO[2] = {tmem + 256, tmem + 384};
            const int ntile = has1 ? 2 : 1;
            bool ok = wait(&bars->q_full, 0, bars);
            auto qk = [&](int i, int st) {
                const uint32_t q = sQ + i * kTileBytes;
                const uint32_t k = sK + st * kTileBytes;
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_ss(tS[i], desc_kmajor(q, s), desc_kmajor(k, s), idesc_qk, s > 0 ? 1u : 0u);
            };
            auto pv = [&](int i, int st, bool acc) {
                const uint32_t v = sV + st * kTileBytes;
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_ts(tO[i], tS[i] + s * 8, desc_v(v, s), idesc_pv, (acc || s > 0) ? 1u : 0u);
            };
            for (int j = 0; ok && j < n_kv; ++j) {
                const int st = j % kStages;
                const uint32_t ph = (j / kStages) & 1;
                const int pst = (j + kStages - 1) % kStages;
                const uint32_t pph = ((j - 1) / kStages) & 1;
                if (!(ok = wait(&bars->k_full[st], ph, bars))) break;
                if (j > 0 && !(ok = wait(&bars->v_full[pst], pph, bars))) break;
                for (int i = 0; i < ntile; ++i) {
                    if (j > 0) {
                        if (!(ok = wait(&bars->p_full[i], (j - 1) & 1, bars))) break;
                        tc_fence_after();
                        pv(i, pst, j > 1);
                    }
                    tc_fence_after();
                    qk(i, st);
                    mma_commit(&bars->s_full[i]);
                }
                if (!ok) break;
                if (j > 0) mma_commit(&bars->v_empty[pst]);
                mma_commit(&bars->k_empty[st]);
            }
            if (ok) {
                const int j = n_kv;
                const int pst = (j - 1) % kStages;
                const uint32_t pph = ((j - 1) / kStages) & 1;
                ok = wait(&bars->v_full[pst], pph, bars);
                for (int i = 0; ok && i < ntile; ++i) {
                    if (!(ok = wait(&bars->p_full[i], (j - 1) & 1, bars))) break;
                    tc_fence_after();
                    pv(i, pst, j > 1);
                    mma_commit(&bars->o_done[i]);
                }
                if (ok) mma_commit(&bars->v_empty[pst]);
            }
            // make sure nothing this thread issued is still running before TMEM is freed
            mma_commit(&bars->drain);
            volatile uint32_t never = 0;
            if (!mbar_wait_bounded(&bars->drain, 0, &never, kDrainLimitNs))
                atomicOr(&g_device_status, 1u);
        }
    } else {
        // ------------------------------------------------------------ softmax warpgroups
        const int i = warp >> 2;        // query tile of this warpgroup
        const int quarter = warp & 3;   // TMEM lanes [32 quarter, 32 quarter + 32)
        if (i == 0 || has1) {
            const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
            const uint32_t tS = tmem + i * 128 + lane_off;
            const uint32_t tO = tmem + 256 + i * 128 + lane_off;
            const float sl2 = p.scale_log2;
            float m_run = -INFINITY, l_run = 0.f;
            bool ok = true;
            for (int j = 0; j < n_kv; ++j) {
                if (!(ok = wait_warp(&bars->s_full[i], j & 1, bars))) break;
                tc_fence_after();
                uint32_t r[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, r[c]);
                tmem_wait_ld();
                const int valid = j < kv_vis ? p.N[0] - j * kBlockN : L - (j - kv_vis) * kBlockN;
                float sv[128];
#pragma unroll
                for (int c = 0; c < 128; ++c) sv[c] = __uint_as_float(r[c >> 5][c & 31]);
                if (valid < kBlockN) {
#pragma unroll
                    for (int c = 0; c < 128; ++c)
                        if (c >= valid) sv[c] = -INFINITY;
                }
                float mx = sv[0];
#pragma unroll
                for (int c = 1; c < 128; ++c) mx = fmaxf(mx, sv[c]);
                const float m_tile = mx * sl2;
                // Raise the running maximum only when some row of this warp grew
                // by more than 8 (log2 units); O is then rescaled after P is out
                // of the registers (the two steps are independent).
                bool rescale = false;
                float f = 1.f;
                if (j == 0) {
                    m_run = m_tile;
                } else if (__any_sync(0xffffffffu, m_tile > m_run + 8.0f)) {
                    const float m_new = fmaxf(m_run, m_tile);
                    f = ex2_approx(m_run - m_new);
                    m_run = m_new;
                    l_run *= f;
                    rescale = true;
                }
                const float neg_m = -m_run;
                float sum = 0.f;
                // P packs two keys per 32-bit column; column c only overwrites
                // register slot c, whose score (slot c <= 2c) is already consumed.
#pragma unroll
                for (int c = 0; c < 64; ++c) {
                    const float a0 = ex2_approx(fmaf(sv[2 * c], sl2, neg_m));
                    const float a1 = ex2_approx(fmaf(sv[2 * c + 1], sl2, neg_m));
                    sum += a0 + a1;
                    r[c >> 5][c & 31] = pack_bf16x2(a0, a1);
                }
                l_run += sum;
                tmem_st32(tS, r[0]);
                tmem_st32(tS + 32, r[1]);
                if (rescale) {
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {
                        uint32_t o[32];
                        tmem_ld32(tO + 32 * c, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
                        tmem_st32(tO + 32 * c, o);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bars->p_full[i]);
            }
            // epilogue: O / l  ->  bf16 row of the owning stream
            if (ok) ok = wait_warp(&bars->o_done[i], 0, bars);
            tc_fence_after();
            int s, row0;
            tile_of(p, t0 + i, s, row0);
            const int row = row0 + quarter * 32 + lane;
            const bool store = row < p.N[s];
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
                        uint4 w;
                        float f[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            f[e] = zero ? 0.f : __uint_as_float(o[8 * v + e]) * inv;
                        w.x = pack_bf16x2(f[0], f[1]);
                        w.y = pack_bf16x2(f[2], f[3]);
                        w.z = pack_bf16x2(f[4], f[5]);
                        w.w = pack_bf16x2(f[6], f[7]);
                        dst[4 * c + v] = w;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kWarpLoad) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace attn

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// [B, N, H, 128] bf16 tensor, boxes of 128 tokens x 64 head-dim elements
// (128 bytes, 128-byte swizzle).  Tokens past N read as zero.
bool encode_tokens(CUtensorMap* m, const void* base, int B, int N, int H) {
    const cuuint64_t dims[4] = {(cuuint64_t)kHeadDim, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)H * kHeadDim * 2,
                                   (cuuint64_t)N * H * kHeadDim * 2};
    const cuuint32_t box[4] = {64, 1, 128, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                             strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

int launch_joint_attention_bf16(const void* qv, const void* kv, const void* vv, const void* qc,
                                const void* kc, const void* vc, const int32_t* ctx_len, void* ov,
                                void* oc, int B, int Nv, int Nc, int H, float softmax_scale,
                                cudaStream_t s) {
    using namespace attn;
    if (!encode_fn()) return -1;
    const int q_tiles = (Nv + kBlockM - 1) / kBlockM + (Nc + kBlockM - 1) / kBlockM;
    if (B == 0 || q_tiles == 0) return 0;
    Params p;
    std::memset(&p, 0, sizeof(p));
    if (Nv > 0) {
        if (!encode_tokens(&p.tm_q[0], qv, B, Nv, H) || !encode_tokens(&p.tm_k[0], kv, B, Nv, H) ||
            !encode_tokens(&p.tm_v[0], vv, B, Nv, H))
            return 1000 + (int)cudaErrorInvalidValue;
    }
    if (Nc > 0) {
        if (!encode_tokens(&p.tm_q[1], qc, B, Nc, H) || !encode_tokens(&p.tm_k[1], kc, B, Nc, H) ||
            !encode_tokens(&p.tm_v[1], vc, B, Nc, H))
            return 1000 + (int)cudaErrorInvalidValue;
    }
    p.out[0] = static_cast<__nv_bfloat16*>(ov);
    p.out[1] = static_cast<__nv_bfloat16*>(oc);
    p.ctx_len = ctx_len;
    p.N[0] = Nv;
    p.N[1] = Nc;
    p.H = H;
    p.q_tiles_vis = (Nv + kBlockM - 1) / kBlockM;
    p.q_tiles = q_tiles;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    const int smem = Smem::total + 1024;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(joint_attn_bf16_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return (int)e;
        attr_set = true;
    }
    dim3 grid((q_tiles + 1) / 2, H, B);
    joint_attn_bf16_kernel<<<grid, kThreads, smem, s>>>(p);
    return (int)cudaGetLastError();
}

cudaError_t read_and_clear_device_status(unsigned int* out, cudaStream_t s) {
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(out, g_device_status, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_device_status, &zero, sizeof(unsigned int));
}

}  // namespace mmdit
