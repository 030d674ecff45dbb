// 8-bit joint attention on the sm_100a tensor cores: Int8 for S = Q K^T and
// FP8 E4M3 for O = P V, with fp32 accumulation across key tiles (the Wan 2.1
// report, section 4.4.3, "8-bit FlashAttention"), over the concatenated
// visual and conditioning streams of the "Vimoo 1.0" research page, section
// 2.2, output split back per stream.
//
// Inputs come from quant.cu: q int8 with one scale per row, k int8 with one
// scale per 128-token block (the kernel's key tile), v E4M3 with one scale per
// channel.  The structure is that of the bf16 kernel (attention_tc.cu): one
// CTA per pair of 128-row query tiles, K / V tiles streamed by TMA, one thread
// issuing tcgen05.mma, two softmax warpgroups, P written back over S.  What
// changes:
//   * S_i = Q_i K^T runs as kind::i8 into s32 tensor memory: 4 k-steps of 32
//     bytes instead of 8 of 16 bf16, at twice the bf16 rate;
//   * the softmax turns an s32 score into fp32 exactly (|S| < 2^22: add the
//     magic 1.5 * 2^23 as an integer; the FMA that scales S by
//     s_q s_k scale log2 e takes the magic's share back out of its addend),
//     so x = S * (s_q s_k scale log2 e) in log2 units costs one integer add
//     per score and one FMA per score pair;
//   * the running maximum is an integer, raised to the ceiling of a tile
//     maximum when that exceeds it by more than 2, so every O rescale is by an
//     exact power of two; P' = 2^(x - m + 6) <= 2^8 is rounded to E4M3 (four
//     keys per 32-bit tensor-memory column) while the row sum takes P'
//     unrounded;
//   * O_i += P'_i V runs as kind::f8f6f4 with P' from tensor memory and V as an
//     MN-major E4M3 operand; the epilogue multiplies by the channel scale of v
//     and divides by the row sum.
// The 8-bit tiles take half the shared memory of the bf16 ones.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "internal.h"
#include "ptx.cuh"
#include "tensor_map.h"

namespace mmdit {

// Bit 0: a bounded wait expired in the 8-bit attention kernel.
__device__ unsigned int g_q8_status = 0;

namespace q8 {

constexpr int kBlock = 128;
constexpr int kStages = 2;
constexpr int kTileBytes = 128 * 128;   // 128 rows x 128 one-byte elements
constexpr int kThreads = 384;
constexpr int kWarpLoad = 8;
constexpr int kWarpMma = 9;
constexpr int kRegsLaunch = 168;
constexpr int kRegsProducer = 72;
constexpr int kRegsSoftmax = 216;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsProducer == kThreads * kRegsLaunch,
              "register split must add up to the launch allocation");
constexpr uint64_t kDrainLimitNs = 200000000ull;

struct Smem {
    static constexpr int q_off = 0;
    static constexpr int k_off = q_off + 2 * kTileBytes;
    static constexpr int v_off = k_off + kStages * kTileBytes;
    static constexpr int bar_off = v_off + kStages * kTileBytes;
    static constexpr int total = bar_off + 256;
};

struct Params {
    CUtensorMap tm_q[2];   // [0] visual, [1] conditioning; uint8 [B, N, H, 128]
    CUtensorMap tm_k[2];
    CUtensorMap tm_v[2];
    __nv_bfloat16* out[2];
    const float* sq[2];    // [B, H, N_s]
    const float* sk[2];    // [B, H, ceil(N_s / 128)]
    const float* sv;       // [B, H, 128]
    const int32_t* ctx_len;
    int N[2];
    int H;
    int q_tiles_vis;
    int q_tiles;
    float sl2;             // softmax_scale * log2(e)
    uint64_t wait_ns;
};

struct Bars {
    uint64_t q_full;
    uint64_t k_full[kStages], k_empty[kStages];   // stage j % 2: K(j) and V(j - 1)
    uint64_t s_full[2], o_done[2];
    uint64_t p_full[2];    // [i]: all of P_i is in tensor memory
    uint64_t drain;
    uint64_t wait_ns;
    uint32_t tmem_base;
    uint32_t abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block must fit its shared-memory slot");

__device__ __forceinline__ void tile_of(const Params& p, int t, int& s, int& row0) {
    if (t < p.q_tiles_vis) {
        s = 0;
        row0 = t * kBlock;
    } else {
        s = 1;
        row0 = (t - p.q_tiles_vis) * kBlock;
    }
}

__device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity, Bars* bars) {
    if (mbar_wait_bounded(bar, parity, &bars->abort, bars->wait_ns)) return true;
    bars->abort = 1;
    atomicOr(&g_q8_status, 1u);
    return false;
}
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, Bars* bars) {
    const bool ok = wait(bar, parity, bars);
    return __all_sync(0xffffffffu, ok);
}

// 8-bit K-major operand (rows x 128 bytes, 128-byte swizzle): k-step s (32
// elements) starts 32 s bytes into each row.
__device__ __forceinline__ uint64_t kdesc(uint32_t addr) { return smem_desc_sw128(addr, 16, 1024); }
// V as an MN-major operand (keys x 128 channels, one 128-byte swizzle span
// along N): k-step s (32 keys) starts 32 rows = 4096 bytes further.
__device__ __forceinline__ uint64_t vdesc(uint32_t addr) {
    return smem_desc_sw128(addr, kTileBytes, 1024);
}

// Streams the key tiles through the K/V ring: stage j % 2 receives K(j) and
// V(j - 1), the operands of the MMA issuer's iteration j, under one barrier
// (only K(0) at j = 0, only V(n_kv - 1) at j = n_kv), as in the bf16 kernel.
// On an abort, waits (bounded) for the copies it issued before returning.
__device__ __forceinline__ void stream_kv(const Params& p, uint8_t* smem, Bars* bars, int n_kv,
                                          int kv_vis, int h, int b) {
    int issued = 0;
    for (int j = 0; j <= n_kv; ++j) {
        const int st = j & 1;
        if (!wait(&bars->k_empty[st], ((j >> 1) & 1) ^ 1, bars)) break;
        const int bytes = (j < n_kv ? kTileBytes : 0) + (j > 0 ? kTileBytes : 0);
        mbar_arrive_expect_tx(&bars->k_full[st], bytes);
        for (int w = 0; w < 2; ++w) {    // w = 0: K(j), w = 1: V(j - 1)
            if ((w == 0 && j == n_kv) || (w == 1 && j == 0)) continue;
            const int jj = j - w;
            const int seg = jj < kv_vis ? 0 : 1;
            const int row = (seg == 0 ? jj : jj - kv_vis) * kBlock;
            uint8_t* t = smem + (w == 0 ? Smem::k_off : Smem::v_off) + st * kTileBytes;
            tma_load_4d(t, w == 0 ? &p.tm_k[seg] : &p.tm_v[seg], &bars->k_full[st], 0, h, row, b);
        }
        ++issued;
    }
    if (bars->abort) {
        for (int j = (issued > kStages ? issued - kStages : 0); j < issued; ++j)
            mbar_wait_bounded(&bars->k_full[j & 1], (j >> 1) & 1, nullptr, kDrainLimitNs);
    }
}

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

__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// 2^k for an integer k <= 0, exactly (0 below the normal range).
__device__ __forceinline__ float exp2_int(int k) {
    return k < -126 ? 0.f : __int_as_float((127 + k) << 23);
}

constexpr int kMagic = 0x4B400000;           // bits of 1.5 * 2^23
constexpr float kMagicF = 12582912.0f;

// P' for keys [64 h, 64 h + 64) of one S row (s32 columns in sr), rounded to
// E4M3 four keys per column into pk; returns the sum of the unrounded P'.
// MASK: keys at or past `valid` (counted from 64 h) get P' = 0.
template <bool MASK>
__device__ __forceinline__ float p_half(const uint32_t (&sr)[4][32], uint32_t (&pk)[16], int h,
                                        uint64_t c2, uint64_t b2, int valid) {
    uint64_t acc[2] = {0, 0};
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        float p[4];
#pragma unroll
        for (int pr = 0; pr < 2; ++pr) {
            const int k = 64 * h + 4 * c + 2 * pr;
            const uint32_t s0 = sr[k >> 5][k & 31], s1 = sr[k >> 5][(k & 31) + 1];
            // 1.5 * 2^23 + S exactly in fp32 (|S| < 2^22); b2 takes the offset
            // back out, so the FMA gives x - m + 6 in log2 units
            const uint64_t sf = f2_pack(__uint_as_float(s0 + kMagic), __uint_as_float(s1 + kMagic));
            float x0, x1;
            f2_unpack(f2_fma(sf, c2, b2), x0, x1);
            if (MASK) {
                if (k - 64 * h >= valid) x0 = -INFINITY;
                if (k + 1 - 64 * h >= valid) x1 = -INFINITY;
            }
            const uint64_t e2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
            acc[pr] = f2_add(acc[pr], e2);
            f2_unpack(e2, p[2 * pr], p[2 * pr + 1]);
        }
        pk[c] = e4m3x2(p[0], p[1]) | (e4m3x2(p[2], p[3]) << 16);
    }
    float a0, a1, b0, b1;
    f2_unpack(acc[0], a0, a1);
    f2_unpack(acc[1], b0, b1);
    return (a0 + a1) + (b0 + b1);
}

__global__ void __launch_bounds__(kThreads, 1) joint_attn_q8_kernel(const __grid_constant__ Params p) {
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
    const int kv_vis = (p.N[0] + kBlock - 1) / kBlock;
    const int n_kv = kv_vis + (L + kBlock - 1) / kBlock;

    if (threadIdx.x == 0) {
        mbar_init(&bars->q_full, 1);
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&bars->k_full[i], 1);
            mbar_init(&bars->k_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->s_full[i], 1);
            mbar_init(&bars->p_full[i], 4);   // one elected lane per softmax warp
            mbar_init(&bars->o_done[i], 1);
        }
        mbar_init(&bars->drain, 1);
        bars->abort = 0;
        bars->wait_ns = p.wait_ns;
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
        for (int tt = 0; tt < 2; ++tt) {
            if (tt == 1 && !has1) break;
            int s, row0;
            tile_of(p, t0 + tt, s, row0);
            for (int r = threadIdx.x; r < kBlock * 16; r += kThreads) {
                const int row = row0 + r / 16;
                if (row < p.N[s])
                    reinterpret_cast<uint4*>(
                        p.out[s] + ((size_t)(b * (size_t)p.N[s] + row) * p.H + h) * 128)[r % 16] =
                        make_uint4(0, 0, 0, 0);
            }
        }
        return;
    }

    if (warp >= 8) {
        regs_dec<kRegsProducer>();
    if (warp == kWarpLoad) {
        if (lane == 0) {
            int s0, r0, s1 = 0, r1 = 0;
            tile_of(p, t0, s0, r0);
            if (has1) tile_of(p, t0 + 1, s1, r1);
            mbar_arrive_expect_tx(&bars->q_full, (has1 ? 2 : 1) * kTileBytes);
            tma_load_4d(smem + Smem::q_off, &p.tm_q[s0], &bars->q_full, 0, h, r0, b);
            if (has1)
                tma_load_4d(smem + Smem::q_off + kTileBytes, &p.tm_q[s1], &bars->q_full, 0, h, r1,
                            b);
            stream_kv(p, smem, bars, n_kv, kv_vis, h, b);
            if (bars->abort) mbar_wait_bounded(&bars->q_full, 0, nullptr, kDrainLimitNs);
        }
    } else if (warp == kWarpMma && lane == 0) {
        // one thread issues every MMA: PV_0(j-1), QK_0(j), PV_1(j-1), QK_1(j)
        constexpr uint32_t idesc_qk = idesc_s8_s32(128, 128);
        constexpr uint32_t idesc_pv = idesc_e4m3_f32(128, 128, 1);
        const int ntile = has1 ? 2 : 1;
        bool ok = wait(&bars->q_full, 0, bars);
        const uint64_t dq0 = kdesc(sQ), dq1 = kdesc(sQ + kTileBytes);
        const uint64_t dk0 = kdesc(sK), dk1 = kdesc(sK + kTileBytes);
        const uint64_t dv0 = vdesc(sV), dv1 = vdesc(sV + kTileBytes);
        auto qk = [&](int i, int st) {
            const uint64_t dq = i == 0 ? dq0 : dq1;
            const uint64_t dk = st == 0 ? dk0 : dk1;
#pragma unroll
            for (int s = 0; s < 4; ++s)
                mma_ss_i8(tmem + 128 * i, dq + 2 * s, dk + 2 * s, idesc_qk, s > 0 ? 1u : 0u);
        };
        // O_i += P'_i V (four k-steps of 32 keys) once the softmax has written
        // all of P'_i
        auto pv = [&](int i, int st, bool acc, uint32_t par) -> bool {
            const uint64_t dv = st == 0 ? dv0 : dv1;
            if (!wait(&bars->p_full[i], par, bars)) return false;
            tc_fence_after();
#pragma unroll
            for (int s = 0; s < 4; ++s)
                mma_ts_f8(tmem + 256 + 128 * i, tmem + 128 * i + 8 * s,
                          dv + (uint64_t)s * (4096 >> 4), idesc_pv, (acc || s > 0) ? 1u : 0u);
            return true;
        };
        // iteration j: PV_i(j - 1) then QK_i(j) per tile from stage j % 2
        for (int j = 0; ok && j <= n_kv; ++j) {
            const int st = j & 1;
            if (!(ok = wait(&bars->k_full[st], (j >> 1) & 1, bars))) break;   // K(j), V(j - 1)
            for (int i = 0; i < ntile; ++i) {
                if (j > 0 && !(ok = pv(i, st, j > 1, (j - 1) & 1))) break;
                if (j < n_kv) {
                    if (j == 0) tc_fence_after();
                    qk(i, st);
                    mma_commit(&bars->s_full[i]);
                } else {
                    mma_commit(&bars->o_done[i]);
                }
            }
            if (!ok) break;
            mma_commit(&bars->k_empty[st]);
        }
        mma_commit(&bars->drain);
        if (!mbar_wait_bounded(&bars->drain, 0, nullptr, kDrainLimitNs))
            atomicOr(&g_q8_status, 1u);
    }
    } else {
        regs_inc<kRegsSoftmax>();
        const int i = warp >> 2;
        const int quarter = warp & 3;
        if (i == 0 || has1) {
            const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
            const uint32_t tS = tmem + i * 128 + lane_off;
            const uint32_t tO = tmem + 256 + i * 128 + lane_off;
            int s, row0;
            tile_of(p, t0 + i, s, row0);
            const int row = row0 + quarter * 32 + lane;
            const float sq =
                row < p.N[s] ? p.sq[s][((size_t)b * p.H + h) * (size_t)p.N[s] + row] : 0.f;
            const int nblk_v = kv_vis, nblk_c = (p.N[1] + kBlock - 1) / kBlock;
            float m_run = 0.f, l_run = 0.f;
            bool ok = true;
            for (int j = 0; j < n_kv; ++j) {
                if (!(ok = wait_warp(&bars->s_full[i], j & 1, bars))) break;
                tc_fence_after();
                uint32_t r[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, r[c]);
                tmem_wait_ld();
                const bool vis = j < kv_vis;
                const int tj = vis ? j : j - kv_vis;
                const int valid = vis ? p.N[0] - j * kBlock : L - tj * kBlock;
                const float sk =
                    vis ? p.sk[0][((size_t)b * p.H + h) * nblk_v + tj]
                        : p.sk[1][((size_t)b * p.H + h) * nblk_c + tj];
                const float c = sq * sk * p.sl2;   // log2 units per unit of S
                // tile maximum of the valid s32 scores (c >= 0 keeps the order);
                // only a tail tile pays for masking
                // (8 independent chains of 3-way maxima, so the latency of one
                // dependent chain of 64 does not sit on every row's path)
                int mk[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) mk[k] = INT32_MIN;
                if (valid < kBlock) {
#pragma unroll
                    for (int k = 0; k < 128; k += 2) {
                        const int a0 = k < valid ? (int)r[k >> 5][k & 31] : INT32_MIN;
                        const int a1 = k + 1 < valid ? (int)r[k >> 5][(k & 31) + 1] : INT32_MIN;
                        mk[(k >> 1) & 7] = __vimax3_s32(mk[(k >> 1) & 7], a0, a1);
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < 128; k += 2)
                        mk[(k >> 1) & 7] = __vimax3_s32(mk[(k >> 1) & 7], (int)r[k >> 5][k & 31],
                                                        (int)r[k >> 5][(k & 31) + 1]);
                }
                const int mi = max(__vimax3_s32(mk[0], mk[1], mk[2]),
                                   max(__vimax3_s32(mk[3], mk[4], mk[5]), max(mk[6], mk[7])));
                const float m_tile = ceilf((float)mi * c);
                if (j == 0) {
                    m_run = m_tile;
                } else if (__any_sync(0xffffffffu, m_tile > m_run + 2.0f)) {
                    const float m_new = fmaxf(m_run, m_tile);
                    const float f = exp2_int((int)(m_run - m_new));
                    l_run *= f;
                    rescale_o(tO, f);
                    m_run = m_new;
                }
                const uint64_t c2 = f2_pack(c, c);
                // (1.5 * 2^23 + S) c + b = S c + 6 - m: one FMA per score pair
                // instead of a subtraction and an FMA (b's own rounding is
                // 2^-24 of 1.5 * 2^23 c, far below the E4M3 step of P')
                const float bm = fmaf(-kMagicF, c, 6.0f - m_run);
                const uint64_t b2 = f2_pack(bm, bm);
                float sum = 0.f;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t pk[16];
                    sum += valid >= 128 ? p_half<false>(r, pk, hh, c2, b2, 64)
                                        : p_half<true>(r, pk, hh, c2, b2, valid - 64 * hh);
                    tmem_st16(tS + 16 * hh, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->p_full[i]);
                l_run += sum;
            }
            if (ok) ok = wait_warp(&bars->o_done[i], 0, bars);
            tc_fence_after();
            const bool store = row < p.N[s];
            const bool zero = !ok || (s == 1 && row >= L);
            const float inv = (l_run > 0.f) ? 1.0f / l_run : 0.f;
            const float* sv = p.sv + ((size_t)b * p.H + h) * 128;
            uint4* dst = reinterpret_cast<uint4*>(
                p.out[s] + ((size_t)((size_t)b * p.N[s] + (store ? row : 0)) * p.H + h) * 128);
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                uint32_t o[32];
                tmem_ld32(tO + 32 * cc, o);
                tmem_wait_ld();
                if (store) {
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        float f[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            f[e] = zero ? 0.f
                                        : __uint_as_float(o[8 * v + e]) *
                                              __ldg(sv + 32 * cc + 8 * v + e) * inv;
                        dst[4 * cc + v] =
                            make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                       pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
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

// [B, N, H, 128] one-byte tensor in boxes of 128 tokens x 128 elements
// (128 bytes, 128-byte swizzle).  Tokens past N read as zero.
bool encode_tokens8(CUtensorMap* m, const void* base, int B, int N, int H) {
    const cuuint64_t dims[4] = {128, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
    const cuuint64_t strides[3] = {128, (cuuint64_t)H * 128, (cuuint64_t)N * H * 128};
    const cuuint32_t box[4] = {128, 1, 128, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims,
                       strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                       CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace q8

int launch_joint_attention_q8(const void* qv, const void* kv, const void* vv, const void* qc,
                              const void* kc, const void* vc, const float* sqv, const float* sqc,
                              const float* skv, const float* skc, const float* sv,
                              const int32_t* ctx_len, void* ov, void* oc, int B, int Nv, int Nc,
                              int H, float softmax_scale, cudaStream_t s) {
    using namespace q8;
    if (!encode_fn()) return -1;
    const int q_tiles = (Nv + kBlock - 1) / kBlock + (Nc + kBlock - 1) / kBlock;
    if (B == 0 || q_tiles == 0) return 0;
    Params p;
    std::memset(&p, 0, sizeof(p));
    if (Nv > 0 && !(encode_tokens8(&p.tm_q[0], qv, B, Nv, H) &&
                    encode_tokens8(&p.tm_k[0], kv, B, Nv, H) &&
                    encode_tokens8(&p.tm_v[0], vv, B, Nv, H)))
        return 1000 + (int)cudaErrorInvalidValue;
    if (Nc > 0 && !(encode_tokens8(&p.tm_q[1], qc, B, Nc, H) &&
                    encode_tokens8(&p.tm_k[1], kc, B, Nc, H) &&
                    encode_tokens8(&p.tm_v[1], vc, B, Nc, H)))
        return 1000 + (int)cudaErrorInvalidValue;
    p.out[0] = static_cast<__nv_bfloat16*>(ov);
    p.out[1] = static_cast<__nv_bfloat16*>(oc);
    p.sq[0] = sqv;
    p.sq[1] = sqc;
    p.sk[0] = skv;
    p.sk[1] = skc;
    p.sv = sv;
    p.ctx_len = ctx_len;
    p.N[0] = Nv;
    p.N[1] = Nc;
    p.H = H;
    p.q_tiles_vis = (Nv + kBlock - 1) / kBlock;
    p.q_tiles = q_tiles;
    p.sl2 = softmax_scale * 1.4426950408889634f;
    p.wait_ns = wait_timeout_ns();
    const int smem = Smem::total + 1024;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return (int)e;
    static bool attr_set[64] = {false};
    if (dev < 0 || dev >= 64) return (int)cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
        cudaFuncAttributes fa;
        e = cudaFuncGetAttributes(&fa, joint_attn_q8_kernel);
        if (e != cudaSuccess) return (int)e;
        if (fa.numRegs != kRegsLaunch) return (int)cudaErrorInvalidKernelImage;
        e = cudaFuncSetAttribute(joint_attn_q8_kernel,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return (int)e;
        attr_set[dev] = true;
    }
    const dim3 grid((q_tiles + 1) / 2, H, B);
    joint_attn_q8_kernel<<<grid, kThreads, smem, s>>>(p);
    return (int)cudaGetLastError();
}

cudaError_t read_and_clear_q8_status(unsigned int* out) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_q8_status, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_q8_status, &zero, sizeof(unsigned int));
}

}  // namespace mmdit
