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
//
// Window mode (Seaweed-7B report, section 3.2, 3D window attention): the
// visual q/k/v arrive in window-major order (window.h), so each window is a
// contiguous key range.  A CTA then owns two query tiles of one window and
// streams that window's visual keys followed by the conditioning keys; the
// conditioning query tiles stream every key.  The grid is one-dimensional with
// the conditioning tiles first (they run longest), and the epilogue writes
// each visual row back at its raster position.
//
// Q-norm mode (the fusion of the Seaweed-7B report, section 3.4, of the
// attention preprocessing into the attention): q arrives raw, and the softmax
// warpgroups, idle until the first S tile, RMS-normalise and rotate (3D RoPE
// on visual rows) their own query row in the swizzled shared-memory Q tile
// before the first MMA reads it.  The cos/sin of every (axis position, pair)
// sit in a shared-memory table built by the same warps while the Q tile is in
// flight.  This saves the write and the re-read of the normalised q.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "internal.h"
#include "ptx.cuh"
#include "tensor_map.h"

namespace mmdit {

// Bit 0: a bounded wait expired in the joint-attention kernel.
__device__ unsigned int g_device_status = 0;

namespace attn {

constexpr int kBlockM = 128;         // query rows per tile
constexpr int kBlockN = 128;         // keys per tile
constexpr int kStages = 2;           // K/V ring: stage j % 2 holds K(j) and V(j - 1)
constexpr int kTileBytes = 128 * 128 * 2;
constexpr int kHalfBytes = kTileBytes / 2;  // one 64-column TMA box (128 B per row)
// Warpgroups: 0 = softmax of query tile 0 (warps 0-3), 1 = softmax of tile 1
// (warps 4-7), 2 = warp 8 TMA of Q, K and V, warp 9 MMA issuer, warps 10-11
// idle (they give the producer warpgroup its 128 threads of the register split).
// K(j) and V(j - 1), the operands of one iteration of the MMA issuer, travel
// together under one barrier, so the issuer waits once per key tile: its
// waits, not the tensor core, set the pace of this kernel on B200 (a separate
// V ring with its own barrier measured 2-3 % slower).
constexpr int kThreads = 384;
constexpr int kWarpLoad = 8;
constexpr int kWarpMma = 9;
// Register split: launched with kRegsLaunch per thread (64512 in total); the
// producer warpgroup drops to kRegsProducer, the softmax warpgroups rise to
// kRegsSoftmax: 2*128*216 + 128*72 = 64512, the launch total.
constexpr int kRegsLaunch = 168;
constexpr int kRegsProducer = 72;
constexpr int kRegsSoftmax = 216;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsProducer == kThreads * kRegsLaunch,
              "register split must add up to the launch allocation");
// Split tail: at most kMaxSplitPieces pieces (the workspace bound of the
// public header), each at least kMinSplitTiles key tiles long.
constexpr int kMaxSplitPieces = MMDIT_ATTENTION_SPLIT_MAX_PIECES;
constexpr int kMinSplitTiles = 2;
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // default: 2 s per pipeline wait
constexpr uint64_t kDrainLimitNs = 200000000ull;   // 0.2 s per drain wait after an abort

struct Smem {
    // tiles are placed first, at 1024-byte aligned offsets (128-byte swizzle atoms)
    static constexpr int q_off = 0;                               // 2 tiles
    static constexpr int k_off = q_off + 2 * kTileBytes;          // kStages tiles
    static constexpr int v_off = k_off + kStages * kTileBytes;    // kStages tiles
    static constexpr int bar_off = v_off + kStages * kTileBytes;
    static constexpr int tab_off = bar_off + 256;                 // Q-norm mode: RoPE table
    static constexpr int total = tab_off;                         // + the table's bytes
};
// Largest RoPE table (float2 entries) that fits beside the tiles in the
// 227 KB a CTA may use (alignment slack included); larger grids compute
// sin / cos per element.
constexpr int kMaxTabEntries = (232448 - Smem::total - 1024) / 8;

struct Params {
    CUtensorMap tm_q[2];  // [0] visual, [1] conditioning
    CUtensorMap tm_k[2];
    CUtensorMap tm_v[2];
    __nv_bfloat16* out[2];
    float* lse;         // [B, H, Nv + Nc] row log-sum-exp, or null
    const int32_t* ctx_len;
    int N[2];           // Nv, Nc
    int H;
    int q_tiles_vis;    // ceil(Nv / 128)
    int q_tiles;        // ceil(Nv / 128) + ceil(Nc / 128)
    float scale_log2;   // softmax_scale * log2(e)
    uint64_t wait_ns;   // limit of one pipeline wait
    // window mode only
    int windowed;
    int B;
    int cond_pairs;     // query-tile pairs of the conditioning stream per (b, h)
    int vis_pairs;      // query-tile pairs of all windows per (b, h)
    int pair_start[kMaxWindows + 1];  // first pair of each window
    WindowTable win;
    // Q-norm mode only
    int qnorm;
    float eps;
    const float* gq[2];        // RMSNorm scale of q per stream [128]
    int rope;                  // visual rows get 3D RoPE
    int gT, gH, gW;            // visual grid
    int off[3], split[3];      // first head dim and width of each axis chunk
    int tab_off[3], tab_stride[3], tab_entries;   // table layout; 0 entries: no table
    double pos_scale[3];
    double freq[64];           // frequency of pair j of axis a at off[a] / 2 + j
    // split tail (full mode only; split_parts == 0: off).  The grid is then
    // one-dimensional: items (b, h, query-tile pair) in the order of the
    // three-dimensional grid, the first split_first of them whole, each later
    // one as split_parts pieces of split_per key tiles.  A piece writes its
    // rows' unnormalised O and (m, l) to part_o / part_ml at index
    // piece * 256 + row; attn_combine_kernel then finishes those rows.
    int split_first, split_parts, split_per, pairs;
    float* part_o;             // [pieces][256][128]
    float2* part_ml;           // [pieces][256]: running max (log2 units), sum
};


// What one CTA works on: query tiles (seg, row) of stream seg (0 visual,
// 1 conditioning), the visual key range [vis_start, vis_start + vis_len), and
// the window of its visual rows (-1: rows are stored in place).
struct Work {
    int b, h;
    int seg0, row0, seg1, row1;
    bool has1;
    int vis_start, vis_len;
    int wi;
    int kv_lo, kv_hi;   // key tiles [kv_lo, kv_hi) of the joint sequence (valid ones only)
    int piece;          // split-tail piece index, or -1 (the CTA stores finished rows)
};

struct Bars {
    uint64_t q_full;
    uint64_t k_full[kStages], k_empty[kStages];   // the K/V ring
    uint64_t s_full[2], o_done[2];
    uint64_t p_full[2];  // [i]: all of P_i is in tensor memory
    uint64_t drain;
    uint64_t q_ready;   // Q-norm mode: every softmax warp has rewritten its Q rows
    uint64_t wait_ns;   // limit of one pipeline wait (copied from the parameters)
    uint32_t tmem_base;
    uint32_t abort;
    Work work;          // this CTA's work item, decoded once by thread 0
};

static_assert(sizeof(Params) <= 4096, "kernel parameters must fit the 4 KB parameter space");
static_assert(sizeof(Bars) <= 256, "barrier block must fit its shared-memory slot");

__device__ __forceinline__ void tile_of(const Params& p, int t, int& s, int& row0) {
    if (t < p.q_tiles_vis) {
        s = 0;
        row0 = t * kBlockM;
    } else {
        s = 1;
        row0 = (t - p.q_tiles_vis) * kBlockM;
    }
}

__device__ __forceinline__ Work decode_work(const Params& p) {
    Work w;
    w.vis_start = 0;
    w.vis_len = p.N[0];
    w.wi = -1;
    w.kv_lo = 0;
    w.kv_hi = 1 << 30;
    w.piece = -1;
    if (!p.windowed) {
        int pair = blockIdx.x;
        w.h = blockIdx.y;
        w.b = blockIdx.z;
        if (p.split_parts > 0) {
            int item = blockIdx.x;
            if (item >= p.split_first) {
                const int q = item - p.split_first;
                const int t = q / p.split_parts;
                w.piece = q;
                w.kv_lo = (q - t * p.split_parts) * p.split_per;
                w.kv_hi = w.kv_lo + p.split_per;
                item = p.split_first + t;
            }
            pair = item % p.pairs;
            const int bh = item / p.pairs;
            w.h = bh % p.H;
            w.b = bh / p.H;
        }
        const int t0 = 2 * pair;
        w.has1 = t0 + 1 < p.q_tiles;
        tile_of(p, t0, w.seg0, w.row0);
        w.seg1 = w.seg0;
        w.row1 = w.row0;
        if (w.has1) tile_of(p, t0 + 1, w.seg1, w.row1);
        return w;
    }
    int idx = blockIdx.x;
    const int cond_items = p.B * p.H * p.cond_pairs;
    int bh;
    if (idx < cond_items) {
        bh = idx / p.cond_pairs;
        const int pr = idx - bh * p.cond_pairs;
        w.seg0 = w.seg1 = 1;
        w.row0 = 2 * kBlockM * pr;
        w.row1 = w.row0 + kBlockM;
        w.has1 = w.row1 < p.N[1];
    } else {
        idx -= cond_items;
        bh = idx / p.vis_pairs;
        const int q = idx - bh * p.vis_pairs;
        int wi = 0;
        while (wi + 1 < p.win.count && p.pair_start[wi + 1] <= q) ++wi;
        const int pr = q - p.pair_start[wi];
        const WindowGeom& g = p.win.w[wi];
        w.vis_start = g.start;
        w.vis_len = g.te * g.he * g.we;
        w.wi = wi;
        w.seg0 = w.seg1 = 0;
        w.row0 = g.start + 2 * kBlockM * pr;
        w.row1 = w.row0 + kBlockM;
        w.has1 = 2 * kBlockM * pr + kBlockM < w.vis_len;
    }
    w.h = bh % p.H;
    w.b = bh / p.H;
    return w;
}

// Output row of query row `row` of stream seg, or -1 if the row is not stored
// (past the end of the stream, or of window wi's rows [vis_start,
// vis_start + vis_len) in window mode).
__device__ __forceinline__ int out_row(const Params& p, int seg, int row, int wi, int vis_start,
                                       int vis_len) {
    if (seg == 1 || wi < 0) return row < p.N[seg] ? row : -1;
    const int local = row - vis_start;
    if (local >= vis_len) return -1;
    return window_to_raster(p.win.w[wi], local, p.win.Hg, p.win.Wg);
}

__device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity, Bars* bars) {
    if (mbar_wait_bounded(bar, parity, &bars->abort, bars->wait_ns)) return true;
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

// Streams key tiles [j_lo, j_lo + n_it) of the joint key sequence (kv_vis
// visual tiles from row vis_start on, then conditioning tiles) through the
// K/V ring: stage j % 2 receives K(j) and V(j - 1) under one barrier (only
// K(0) at j = 0, only V(n_it - 1) at j = n_it).  On an abort, waits (bounded)
// for the copies it issued before returning.
__device__ __forceinline__ void stream_kv(const Params& p, uint8_t* smem, Bars* bars, int j_lo,
                                          int n_it, int kv_vis, int vis_start, int h, int b) {
    int issued = 0;
    for (int j = 0; j <= n_it; ++j) {
        const int st = j & 1;
        if (!wait(&bars->k_empty[st], ((j >> 1) & 1) ^ 1, bars)) break;
        const int bytes = (j < n_it ? kTileBytes : 0) + (j > 0 ? kTileBytes : 0);
        mbar_arrive_expect_tx(&bars->k_full[st], bytes);
        for (int w = 0; w < 2; ++w) {    // w = 0: K(j), w = 1: V(j - 1)
            if ((w == 0 && j == n_it) || (w == 1 && j == 0)) continue;
            const int jj = j_lo + j - w;
            const int seg = jj < kv_vis ? 0 : 1;
            const int row = seg == 0 ? vis_start + jj * kBlockN : (jj - kv_vis) * kBlockN;
            const CUtensorMap* tm = w == 0 ? &p.tm_k[seg] : &p.tm_v[seg];
            uint8_t* t = smem + (w == 0 ? Smem::k_off : Smem::v_off) + st * kTileBytes;
            tma_load_4d(t, tm, &bars->k_full[st], 0, h, row, b);
            tma_load_4d(t + kHalfBytes, tm, &bars->k_full[st], 64, h, row, b);
        }
        ++issued;
    }
    if (bars->abort) {
        for (int j = (issued > kStages ? issued - kStages : 0); j < issued; ++j)
            mbar_wait_bounded(&bars->k_full[j & 1], (j >> 1) & 1, nullptr, kDrainLimitNs);
    }
}

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
// packed two bf16 keys per 32-bit column into rh (column c holds keys
// 64 h + 2c, 64 h + 2c + 1); returns their sum.  Products and sums use the
// packed fp32x2 pipe, the partial sums run in four independent chains.
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

// Q-norm mode: RMS-normalise (and, on visual rows, rotate) query row r of
// tile i in place in shared memory, then release it to the MMA issuer.  Run by
// all 256 softmax threads (thread = row of its warpgroup's tile).
// Kept out of line: inlined, it measured slower (the main loop's schedule
// changed).
__device__ __noinline__ void q_prologue(const Params& p, uint8_t* smem, Bars* bars,
                                        const volatile Work* vwk, int i, int r) {
    float2* tab = reinterpret_cast<float2*>(smem + Smem::tab_off);
    const bool use_tab = p.rope && p.tab_entries > 0;
    if (use_tab) {
        for (int e = threadIdx.x; e < p.tab_entries; e += 256) {
            const int a = e < p.tab_off[1] ? 0 : (e < p.tab_off[2] ? 1 : 2);
            const int local = e - p.tab_off[a];
            const int pos = local / p.tab_stride[a];
            const int j = local - pos * p.tab_stride[a];
            float c = 1.f, sn = 0.f;
            if (j < p.split[a] / 2) {
                const float ang = (float)((double)pos * p.pos_scale[a] * p.freq[p.off[a] / 2 + j]);
                sincosf(ang, &sn, &c);
            }
            tab[e] = make_float2(c, sn);
        }
        named_barrier_sync(1, 256);
    }
    const bool has_tile = i == 0 || vwk->has1;
    if (has_tile && wait(&bars->q_full, 0, bars)) {
        const int seg = i ? vwk->seg1 : vwk->seg0;
        const int qrow = (i ? vwk->row1 : vwk->row0) + r;
        uint8_t* row = smem + Smem::q_off + i * kTileBytes + r * 128;
        const float* g = p.gq[seg];
        // mean square: 16 partial sums of 8 dims, then a butterfly over them
        float part[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            const uint4 v = *reinterpret_cast<const uint4*>(row + (c >> 3) * kHalfBytes +
                                                            (((c & 7) ^ (r & 7)) << 4));
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            float acc = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float lo = __uint_as_float(w[e] << 16), hi = __uint_as_float(w[e] & 0xffff0000u);
                acc = fmaf(lo, lo, acc);
                acc = fmaf(hi, hi, acc);
            }
            part[c] = acc;
        }
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1)
#pragma unroll
            for (int c = 0; c < 16; ++c)
                if (!(c & o)) part[c] += part[c | o];
        const float inv = rsqrtf(part[0] * (1.0f / kHeadDim) + p.eps);
        // position of the row (visual rows with RoPE only)
        bool rot = seg == 0 && p.rope;
        int pt = 0, ph = 0, pw = 0;   // grid position (t, h, w)
        if (rot) {
            int n = qrow;
            if (vwk->wi >= 0) {
                const int local = qrow - vwk->vis_start;
                rot = local < vwk->vis_len;
                n = rot ? window_to_raster(p.win.w[vwk->wi], local, p.win.Hg, p.win.Wg) : 0;
            } else {
                rot = qrow < p.N[0];
            }
            const int hw = p.gH * p.gW;
            pt = n / hw;
            ph = (n / p.gW) % p.gH;
            pw = n % p.gW;
        }
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            uint4* addr = reinterpret_cast<uint4*>(row + (c >> 3) * kHalfBytes +
                                                   (((c & 7) ^ (r & 7)) << 4));
            const uint4 v = *addr;
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            float x[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                x[2 * e] = __uint_as_float(w[e] << 16);
                x[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
            }
            const int d0 = 8 * c;
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] *= inv * __ldg(g + d0 + e);
            if (rot) {
                const int a = d0 < p.off[1] ? 0 : (d0 < p.off[2] ? 1 : 2);
                const int pa = a == 0 ? pt : (a == 1 ? ph : pw);
                const int jb = (d0 - p.off[a]) >> 1;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float cs, sn;
                    if (use_tab) {
                        const float2 t = tab[p.tab_off[a] + pa * p.tab_stride[a] + jb + q];
                        cs = t.x;
                        sn = t.y;
                    } else {
                        const float ang = (float)((double)pa * p.pos_scale[a] *
                                                  p.freq[p.off[a] / 2 + jb + q]);
                        sincosf(ang, &sn, &cs);
                    }
                    const float x0 = x[2 * q], x1 = x[2 * q + 1];
                    x[2 * q] = x0 * cs - x1 * sn;
                    x[2 * q + 1] = x0 * sn + x1 * cs;
                }
            }
            *addr = make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                               pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
        }
        fence_proxy_async_smem();
    }
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(&bars->q_ready);
}

__global__ void __launch_bounds__(kThreads, 1) joint_attn_bf16_kernel(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Bars* bars = reinterpret_cast<Bars*>(smem + Smem::bar_off);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        bars->work = decode_work(p);
        mbar_init(&bars->q_full, 1);
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&bars->k_full[i], 1);
            mbar_init(&bars->k_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->s_full[i], 1);
            mbar_init(&bars->p_full[i], 4);          // one elected lane per softmax warp
            mbar_init(&bars->o_done[i], 1);
        }
        mbar_init(&bars->drain, 1);
        mbar_init(&bars->q_ready, 8);
        bars->abort = 0;
        bars->wait_ns = p.wait_ns;
        fence_barrier_init();
    }
    __syncthreads();
    // The work item is read back from shared memory where it is needed, so
    // that it holds no registers through the main loop.
    const volatile Work* vwk = &bars->work;
    const int h = vwk->h;
    const int b = vwk->b;
    const bool has1 = vwk->has1;
    int L = p.N[1];
    if (p.ctx_len) {
        L = p.ctx_len[b];
        L = L < 0 ? 0 : (L > p.N[1] ? p.N[1] : L);
    }
    const int kv_vis = (vwk->vis_len + kBlockN - 1) / kBlockN;
    const int n_kv = kv_vis + (L + kBlockN - 1) / kBlockN;
    // this CTA's key tiles: all of them, or a split-tail piece's range
    const int j_lo = vwk->kv_lo < n_kv ? vwk->kv_lo : n_kv;
    const int n_it = (vwk->kv_hi < n_kv ? vwk->kv_hi : n_kv) - j_lo;
    if (warp == kWarpLoad && n_it > 0) {
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

    if (n_it == 0 && vwk->piece >= 0) {
        // a split-tail piece whose key range holds no valid key: an empty
        // partial (the combine skips it)
        for (int r = threadIdx.x; r < 2 * kBlockM; r += kThreads)
            p.part_ml[(size_t)vwk->piece * (2 * kBlockM) + r] = make_float2(-INFINITY, 0.f);
        return;
    }
    if (n_it == 0) {
        // no valid key at all: every output row of this CTA is zero
        for (int tt = 0; tt < 2; ++tt) {
            if (tt == 1 && !has1) break;
            const int s = tt ? vwk->seg1 : vwk->seg0;
            const int row0 = tt ? vwk->row1 : vwk->row0;
            for (int r = threadIdx.x; r < kBlockM * 16; r += kThreads) {
                const int orow = out_row(p, s, row0 + r / 16, vwk->wi, vwk->vis_start, vwk->vis_len);
                if (orow >= 0) {
                    uint4* dst = reinterpret_cast<uint4*>(
                        p.out[s] + ((size_t)(b * (size_t)p.N[s] + orow) * p.H + h) * kHeadDim);
                    dst[r % 16] = make_uint4(0, 0, 0, 0);
                    // lse rows in the order of the inputs (window-major in window mode)
                    if (p.lse && r % 16 == 0)
                        p.lse[((size_t)b * p.H + h) * (size_t)(p.N[0] + p.N[1]) +
                              (s ? p.N[0] : 0) + row0 + r / 16] = INFINITY;
                }
            }
        }
        return;
    }

    // Each role's whole body sits inside the branch that set its register
    // budget, so the compiler allocates each region with its own limit.
    if (warp >= 8) {
        regs_dec<kRegsProducer>();
    if (warp == kWarpLoad) {
        // ------------------------------------------------------------ TMA: Q, K and V
        if (lane == 0) {
            for (int seg = 0; seg < 2; ++seg) {
                if (p.N[seg] > 0) {
                    tma_prefetch_desc(&p.tm_q[seg]);
                    tma_prefetch_desc(&p.tm_k[seg]);
                    tma_prefetch_desc(&p.tm_v[seg]);
                }
            }
            const int s0 = vwk->seg0, r0 = vwk->row0, s1 = vwk->seg1, r1 = vwk->row1;
            mbar_arrive_expect_tx(&bars->q_full, (has1 ? 2 : 1) * kTileBytes);
            tma_load_4d(smem + Smem::q_off, &p.tm_q[s0], &bars->q_full, 0, h, r0, b);
            tma_load_4d(smem + Smem::q_off + kHalfBytes, &p.tm_q[s0], &bars->q_full, 64, h, r0, b);
            if (has1) {
                tma_load_4d(smem + Smem::q_off + kTileBytes, &p.tm_q[s1], &bars->q_full, 0, h, r1, b);
                tma_load_4d(smem + Smem::q_off + kTileBytes + kHalfBytes, &p.tm_q[s1], &bars->q_full,
                            64, h, r1, b);
            }
            stream_kv(p, smem, bars, j_lo, n_it, kv_vis, vwk->vis_start, h, b);
            if (bars->abort) mbar_wait_bounded(&bars->q_full, 0, nullptr, kDrainLimitNs);
        }
    } else if (warp == kWarpMma && lane == 0) {
        // ------------------------------------------------------------ MMA issuer
        // One thread issues every MMA, in the order PV_0(j-1), QK_0(j),
        // PV_1(j-1), QK_1(j): QK_i(j) overwrites the tensor memory PV_i(j-1)
        // reads, and one thread's MMAs execute in issue order.  (Two issuing
        // threads, one per tile, measured 14 % slower: the tensor core then
        // interleaves the two tiles' batches and both S tiles arrive later.)
        constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 128, 0, 1);
        const int ntile = has1 ? 2 : 1;
        bool ok = wait(p.qnorm ? &bars->q_ready : &bars->q_full, 0, bars);
        // Descriptor bases are computed once; a k-step only adds a constant to
        // the start-address field (shared addresses stay below 256 KB, so the
        // 14-bit field never carries).  This keeps the issuing thread, which
        // shares its SM sub-partition with softmax warps, to a few
        // instructions per MMA.
        const uint64_t dq0 = desc_kmajor(sQ, 0), dq1 = desc_kmajor(sQ + kTileBytes, 0);
        const uint64_t dk0 = desc_kmajor(sK, 0), dk1 = desc_kmajor(sK + kTileBytes, 0);
        const uint64_t dv0 = desc_v(sV, 0), dv1 = desc_v(sV + kTileBytes, 0);
        // tile i: S_i (and P_i over its first 64 columns) at column 128 i, O_i at 256 + 128 i
        auto qk = [&](int i, int st) {
            const uint64_t dq = i == 0 ? dq0 : dq1;
            const uint64_t dk = st == 0 ? dk0 : dk1;
            const uint32_t d = tmem + 128 * i;
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const uint64_t off = (uint64_t)((s >> 2) * (kHalfBytes >> 4) + (s & 3) * 2);
                mma_ss(d, dq + off, dk + off, idesc_qk, s > 0 ? 1u : 0u);
            }
        };
        // O_i += P_i V once the softmax has written all of P_i; false if the
        // wait gave up.  (Releasing P in halves, so that the first half's MMAs
        // start early, measured 1-3 % slower: one more wait per tile for the
        // issuing thread.)
        auto pv = [&](int i, int st, bool acc, uint32_t par) -> bool {
            const uint64_t dv = st == 0 ? dv0 : dv1;
            const uint32_t d = tmem + 256 + 128 * i;
            const uint32_t a = tmem + 128 * i;
            if (!wait(&bars->p_full[i], par, bars)) return false;
            tc_fence_after();
#pragma unroll
            for (int s = 0; s < 8; ++s)
                mma_ts(d, a + s * 8, dv + (uint64_t)(s * (2048 >> 4)), idesc_pv,
                       (acc || s > 0) ? 1u : 0u);
            return true;
        };
        // Iteration j: stage j % 2 holds K(j) and V(j - 1); PV_i(j - 1) then
        // QK_i(j) per tile, and the stage is released when both have run.
        for (int j = 0; ok && j <= n_it; ++j) {
            const int st = j & 1;
            if (!(ok = wait(&bars->k_full[st], (j >> 1) & 1, bars))) break;
            for (int i = 0; i < ntile; ++i) {
                if (j > 0 && !(ok = pv(i, st, j > 1, (j - 1) & 1))) break;
                if (j < n_it) {
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
        // make sure nothing this thread issued is still running before TMEM is freed
        mma_commit(&bars->drain);
        if (!mbar_wait_bounded(&bars->drain, 0, nullptr, kDrainLimitNs))
            atomicOr(&g_device_status, 1u);
    }
    } else {
        regs_inc<kRegsSoftmax>();
        // ------------------------------------------------------------ softmax warpgroups
        const int i = warp >> 2;        // query tile of this warpgroup
        const int quarter = warp & 3;   // TMEM lanes [32 quarter, 32 quarter + 32)
        if (p.qnorm) q_prologue(p, smem, bars, vwk, i, quarter * 32 + lane);
        if (i == 0 || vwk->has1) {
            const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
            const uint32_t tS = tmem + i * 128 + lane_off;
            const uint32_t tO = tmem + 256 + i * 128 + lane_off;
            const float sl2 = p.scale_log2;
            const uint64_t sl2x2 = f2_pack(sl2, sl2);
            float m_run = -INFINITY, l_run = 0.f;
            bool ok = true;
            for (int it = 0; it < n_it; ++it) {
                if (!(ok = wait_warp(&bars->s_full[i], it & 1, bars))) break;
                tc_fence_after();
                uint32_t r[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, r[c]);
                tmem_wait_ld();
                // key tile of this iteration (j_lo equals kv_lo whenever the loop runs)
                const int j = it + vwk->kv_lo;
                const int valid =
                    j < kv_vis ? vwk->vis_len - j * kBlockN : L - (j - kv_vis) * kBlockN;
                float sv[128];
#pragma unroll
                for (int c = 0; c < 128; ++c) sv[c] = __uint_as_float(r[c >> 5][c & 31]);
                if (valid < kBlockN) {
#pragma unroll
                    for (int c = 0; c < 128; ++c)
                        if (c >= valid) sv[c] = -INFINITY;
                }
                // row maximum in 8 independent chains
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
                // Raise the running maximum only when some row of this warp grew
                // by more than 8 (log2 units); O (which holds PV up to the
                // previous tile: S(j) ready implies it completed) is rescaled
                // before this tile's P is released to the MMA.
                if (it == 0) {
                    m_run = m_tile;
                } else if (__any_sync(0xffffffffu, m_tile > m_run + 8.0f)) {
                    const float m_new = fmaxf(m_run, m_tile);
                    const float f = ex2_approx(m_run - m_new);
                    m_run = m_new;
                    l_run *= f;
                    rescale_o(tO, f);
                }
                // P (bf16 pairs) over the first 64 columns of S, released to
                // the MMA issuer in one piece
                const uint64_t negm2 = f2_pack(-m_run, -m_run);
                float sum = 0.f;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    sum += exp_half(sv, r[h], h, sl2x2, negm2);
                    tmem_st32(tS + 32 * h, r[h]);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->p_full[i]);
                l_run += sum;
            }
            // epilogue: O / l  ->  bf16 row of the owning stream (or, for a
            // split-tail piece, the partial row for the combine)
            if (ok) ok = wait_warp(&bars->o_done[i], 0, bars);
            tc_fence_after();
            if (vwk->piece >= 0) {
                // split-tail piece: this row's unnormalised O and (m, l) for
                // the combine
                const size_t prow = (size_t)vwk->piece * (2 * kBlockM) + i * kBlockM +
                                    quarter * 32 + lane;
                float4* dst = reinterpret_cast<float4*>(p.part_o + prow * kHeadDim);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tO + 32 * c, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int v = 0; v < 8; ++v)
                        dst[8 * c + v] = make_float4(
                            __uint_as_float(o[4 * v]), __uint_as_float(o[4 * v + 1]),
                            __uint_as_float(o[4 * v + 2]), __uint_as_float(o[4 * v + 3]));
                }
                p.part_ml[prow] = ok ? make_float2(m_run, l_run) : make_float2(-INFINITY, 0.f);
            } else {
                const int s = i ? vwk->seg1 : vwk->seg0;
                const int row = (i ? vwk->row1 : vwk->row0) + quarter * 32 + lane;
                const int orow = out_row(p, s, row, vwk->wi, vwk->vis_start, vwk->vis_len);
                const bool store = orow >= 0;
                const bool zero = !ok || (s == 1 && row >= L);
                const float inv = (l_run > 0.f) ? 1.0f / l_run : 0.f;
                if (p.lse && store) {
                    // natural-log row log-sum-exp of the scaled scores; m_run and
                    // the exponents are in log2 units.  Rows in the order of the
                    // inputs (window-major in window mode)
                    const int jrow = s == 0 ? row : p.N[0] + row;
                    p.lse[((size_t)vwk->b * p.H + vwk->h) * (size_t)(p.N[0] + p.N[1]) + jrow] =
                        (zero || !(l_run > 0.f)) ? INFINITY
                                                 : (m_run + log2f(l_run)) * 0.6931471805599453f;
                }
                uint4* dst = reinterpret_cast<uint4*>(
                    p.out[s] + ((size_t)((size_t)vwk->b * p.N[s] + (store ? orow : 0)) * p.H +
                                vwk->h) * kHeadDim);
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
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kWarpLoad) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// Finishes the rows of the split-tail items.  Piece p of a row holds
// O_p = sum over its keys of 2^(x - m_p) v and l_p = sum of the same weights
// (x: scaled score in log2 units, m_p the piece's running maximum); the row is
//   M = max_p m_p,  l = sum_p 2^(m_p - M) l_p,  O = sum_p 2^(m_p - M) O_p / l,
// the rescaling the main loop applies between key tiles.  Pieces without a
// valid key (m_p = -inf) drop out.  One warp per row, four head dims a lane.
__global__ void __launch_bounds__(256) attn_combine_kernel(const __grid_constant__ Params p,
                                                           int tail_items) {
    const int row_id = blockIdx.x * 8 + (threadIdx.x >> 5);   // tail item * 256 + row
    const int lane = threadIdx.x & 31;
    const int t = row_id / (2 * kBlockM);
    const int r = row_id - t * (2 * kBlockM);
    if (t >= tail_items) return;
    const int item = p.split_first + t;
    const int pair = item % p.pairs;
    const int bh = item / p.pairs;
    const int h = bh % p.H, b = bh / p.H;
    const int tt = 2 * pair + r / kBlockM;
    if (tt >= p.q_tiles) return;          // the last pair has one tile
    int s, row0;
    tile_of(p, tt, s, row0);
    const int row = row0 + r % kBlockM;
    if (row >= p.N[s]) return;            // past the end of the stream: not stored
    int L = p.N[1];
    if (p.ctx_len) {
        L = p.ctx_len[b];
        L = L < 0 ? 0 : (L > p.N[1] ? p.N[1] : L);
    }
    const bool zero = s == 1 && row >= L;
    const size_t first = (size_t)t * p.split_parts * (2 * kBlockM) + r;   // piece 0's row
    float M = -INFINITY;
    for (int q = 0; q < p.split_parts; ++q)
        M = fmaxf(M, p.part_ml[first + (size_t)q * (2 * kBlockM)].x);
    float l = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (!zero && M > -INFINITY) {
        for (int q = 0; q < p.split_parts; ++q) {
            const size_t pr = first + (size_t)q * (2 * kBlockM);
            const float2 ml = p.part_ml[pr];
            if (!(ml.x > -INFINITY)) continue;
            const float w = exp2f(ml.x - M);
            l += w * ml.y;
            const float4 o = reinterpret_cast<const float4*>(p.part_o + pr * kHeadDim)[lane];
            acc.x += w * o.x;
            acc.y += w * o.y;
            acc.z += w * o.z;
            acc.w += w * o.w;
        }
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    reinterpret_cast<uint2*>(p.out[s] + ((size_t)((size_t)b * p.N[s] + row) * p.H + h) *
                                            kHeadDim)[lane] =
        make_uint2(pack_bf16x2(acc.x * inv, acc.y * inv), pack_bf16x2(acc.z * inv, acc.w * inv));
    if (p.lse && lane == 0)
        p.lse[((size_t)b * p.H + h) * (size_t)(p.N[0] + p.N[1]) + (s ? p.N[0] + row : row)] =
            (zero || !(l > 0.f)) ? INFINITY : (M + log2f(l)) * 0.6931471805599453f;
}

}  // namespace attn

namespace {

std::atomic<unsigned long long> g_wait_timeout_ns{0};  // 0: default


}  // namespace

uint64_t wait_timeout_ns() {
    const unsigned long long v = g_wait_timeout_ns.load(std::memory_order_relaxed);
    return v ? v : attn::kWaitLimitNs;
}

SplitPlan split_plan(int B, int Nv, int Nc, int H, int num_sms, long long ws_bytes) {
    using namespace attn;
    SplitPlan sp{};
    const long long q_tiles = (Nv + kBlockM - 1) / kBlockM + (Nc + kBlockM - 1) / kBlockM;
    const long long total = (long long)B * H * ((q_tiles + 1) / 2);
    const int kv_max = (int)((Nv + (long long)kBlockN - 1) / kBlockN +
                             (Nc + (long long)kBlockN - 1) / kBlockN);
    sp.ctas = total;
    if (num_sms < 1 || total == 0 || total >= (1LL << 31)) return sp;
    const int t = (int)(total % num_sms);
    if (t == 0) return sp;
    int parts = std::min(num_sms / t, std::min(kv_max / kMinSplitTiles, kMaxSplitPieces / t));
    if (parts < 2) return sp;
    const int per = (kv_max + parts - 1) / parts;
    parts = (kv_max + per - 1) / per;
    if ((long long)t * parts * 2 * kBlockM * (kHeadDim + 2) * 4 > ws_bytes) return sp;
    sp.tail = t;
    sp.parts = parts;
    sp.per = per;
    sp.first = (int)(total - t);
    sp.ctas = total - t + (long long)t * parts;
    return sp;
}

int launch_joint_attention_bf16(const void* qv, const void* kv, const void* vv, const void* qc,
                                const void* kc, const void* vc, const int32_t* ctx_len, void* ov,
                                void* oc, float* lse, int B, int Nv, int Nc, int H,
                                float softmax_scale, const WindowTable* win, cudaStream_t s,
                                const QNormArgs* qn, float* split_ws, long long split_ws_bytes) {
    using namespace attn;
    if (!encode_fn()) return -1;
    const int q_tiles = (Nv + kBlockM - 1) / kBlockM + (Nc + kBlockM - 1) / kBlockM;
    if (B == 0 || q_tiles == 0) return 0;
    // the plain form runs on CTA pairs (attention_pair.cu): same outputs, half
    // the issued products per SM; the split tail's workspace is then unused
    if (!win && !qn && !lse && Nv > 0)
        return launch_joint_attention_pair(qv, kv, vv, qc, kc, vc, ctx_len, ov, oc, B, Nv, Nc, H,
                                           softmax_scale, s);
    Params p;
    std::memset(&p, 0, sizeof(p));
    long long items = 0;  // window mode: CTAs of the one-dimensional grid
    if (win) {
        p.windowed = 1;
        p.B = B;
        p.win = *win;
        p.cond_pairs = ((Nc + kBlockM - 1) / kBlockM + 1) / 2;
        int pairs = 0;
        for (int w = 0; w < win->count; ++w) {
            p.pair_start[w] = pairs;
            const int len = win->w[w].te * win->w[w].he * win->w[w].we;
            pairs += ((len + kBlockM - 1) / kBlockM + 1) / 2;
        }
        p.pair_start[win->count] = pairs;
        p.vis_pairs = pairs;
        items = (long long)B * H * (p.cond_pairs + p.vis_pairs);
        if (items >= (1LL << 31)) return (int)cudaErrorInvalidConfiguration;
    }
    if (Nv > 0) {
        if (!encode_tokens(&p.tm_q[0], qv, B, Nv, H, kBlockM) ||
            !encode_tokens(&p.tm_k[0], kv, B, Nv, H, kBlockN) ||
            !encode_tokens(&p.tm_v[0], vv, B, Nv, H, kBlockN))
            return 1000 + (int)cudaErrorInvalidValue;
    }
    if (Nc > 0) {
        if (!encode_tokens(&p.tm_q[1], qc, B, Nc, H, kBlockM) ||
            !encode_tokens(&p.tm_k[1], kc, B, Nc, H, kBlockN) ||
            !encode_tokens(&p.tm_v[1], vc, B, Nc, H, kBlockN))
            return 1000 + (int)cudaErrorInvalidValue;
    }
    p.out[0] = static_cast<__nv_bfloat16*>(ov);
    p.out[1] = static_cast<__nv_bfloat16*>(oc);
    p.lse = lse;
    p.ctx_len = ctx_len;
    p.N[0] = Nv;
    p.N[1] = Nc;
    p.H = H;
    p.q_tiles_vis = (Nv + kBlockM - 1) / kBlockM;
    p.q_tiles = q_tiles;
    p.scale_log2 = softmax_scale * 1.4426950408889634f;
    p.wait_ns = wait_timeout_ns();
    int tab_bytes = 0;
    if (qn) {
        p.qnorm = 1;
        p.eps = qn->eps;
        p.gq[0] = qn->gq[0];
        p.gq[1] = qn->gq[1];
        if (qn->grid) {
            const RopeGrid& g = *qn->grid;
            p.rope = 1;
            p.gT = g.T;
            p.gH = g.H;
            p.gW = g.W;
            const int extent[3] = {g.T, g.H, g.W};
            int off = 0, toff = 0;
            for (int a = 0; a < 3; ++a) {
                p.off[a] = off;
                p.split[a] = g.split[a];
                p.pos_scale[a] = g.pos_scale[a];
                const int half = g.split[a] / 2;
                for (int j = 0; j < half; ++j)
                    p.freq[off / 2 + j] = std::pow(g.base, -2.0 * j / (double)g.split[a]);
                p.tab_stride[a] = (half + 1) & ~1;
                p.tab_off[a] = toff;
                toff += extent[a] * p.tab_stride[a];
                off += g.split[a];
            }
            p.tab_entries = toff <= kMaxTabEntries ? toff : 0;
            tab_bytes = p.tab_entries * 8;
        }
    }
    const int smem = Smem::total + tab_bytes + 1024;
    const int smem_max = Smem::total + kMaxTabEntries * 8 + 1024;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return (int)e;
    static bool attr_set[64] = {false};
    static int sm_count[64] = {0};
    if (dev < 0 || dev >= 64) return (int)cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
        e = cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return (int)e;
        // The register split inside the kernel assumes the launch allocation
        // is exactly kRegsLaunch per thread; refuse to launch otherwise (a
        // smaller allocation would leave the increase waiting for ever).
        cudaFuncAttributes fa;
        e = cudaFuncGetAttributes(&fa, joint_attn_bf16_kernel);
        if (e != cudaSuccess) return (int)e;
        if (fa.numRegs != kRegsLaunch) return (int)cudaErrorInvalidKernelImage;
        e = cudaFuncSetAttribute(joint_attn_bf16_kernel,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, smem_max);
        if (e != cudaSuccess) return (int)e;
        attr_set[dev] = true;
    }
    dim3 grid = win ? dim3((unsigned)items, 1, 1) : dim3((q_tiles + 1) / 2, H, B);
    // Split tail.  One CTA runs per SM, and every item of a full launch costs
    // the same, so the items beyond the last whole wave (total mod #SMs) would
    // run as a wave of their own on a few SMs.  With a workspace, each of them
    // is split over its key tiles into as many pieces as fill the SMs (at
    // least kMinSplitTiles tiles a piece, kMaxSplitPieces pieces in all), and
    // attn_combine_kernel merges the pieces.
    int tail = 0;
    if (!win && split_ws) {
        SplitPlan sp = split_plan(B, Nv, Nc, H, sm_count[dev], split_ws_bytes);
        if (sp.parts >= 2) {
            tail = sp.tail;
            p.split_first = sp.first;
            p.split_parts = sp.parts;
            p.split_per = sp.per;
            p.pairs = (q_tiles + 1) / 2;
            p.part_o = split_ws;
            const size_t o_floats = (size_t)sp.tail * sp.parts * 2 * kBlockM * kHeadDim;
            p.part_ml = reinterpret_cast<float2*>(split_ws + o_floats);
            grid = dim3((unsigned)sp.ctas, 1, 1);
        }
    }
    joint_attn_bf16_kernel<<<grid, kThreads, smem, s>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess || tail == 0) return (int)e;
    attn_combine_kernel<<<tail * 2 * kBlockM / 8, 256, 0, s>>>(p, tail);
    return (int)cudaGetLastError();
}

void set_wait_timeout_ns(unsigned long long ns) {
    g_wait_timeout_ns.store(ns, std::memory_order_relaxed);
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
