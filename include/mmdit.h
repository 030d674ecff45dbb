/*
 * mmdit.h — C ABI of libmmdit.so: one dual-stream MMDiT block's joint-attention
 * core on NVIDIA B200 (sm_100a).
 *
 * What the block computes is stated in "Vimoo 1.0: Video Generation for
 * Compact, Lightweight, and High-Speed", section 2.2 "Dual-Stream MMDiT
 * Backbone" (cited below as [Vimoo §2.2]); the token order of the visual
 * stream follows the patchify-and-flatten step of the Wan 2.1 report, section
 * 4.2.1, and the attention is non-causal (Wan 2.1 report, section 4.3.1).
 *
 * Conventions shared by every entry point (the host-buffer executor at the
 * end, mmdit_block_forward_host, differs where its comment says so):
 *   - All tensor pointers are DEVICE pointers to contiguous row-major arrays,
 *     16-byte aligned.  The caller owns all memory; the library allocates no
 *     device memory and keeps no state between calls.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously on it; the return value reports
 *     argument validation and launch errors only.  A kernel that gives up on a
 *     bounded device-side wait records MMDIT_ERR_TIMEOUT in a device status
 *     word, read back (and cleared) by mmdit_device_status().
 *   - Element type of q/k/v/x/branch/outputs is given by `dt`; every scale,
 *     shift, gate and RMSNorm weight is fp32.  Arithmetic is fp32 (tensor-core
 *     products of bf16 operands accumulate in fp32).
 *   - Head dim D must be 128.  Tokens are laid out [B, N, H, D] for q/k/v/o
 *     and [B, N, C] with C = H*D for x/branch/y.
 *   - On any error nothing is enqueued and no output is touched.
 */
#ifndef MMDIT_H
#define MMDIT_H

#include <stdint.h>

#if defined(__GNUC__)
#define MMDIT_API __attribute__((visibility("default")))
#else
#define MMDIT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { MMDIT_F32 = 0, MMDIT_BF16 = 1 } mmdit_dtype;

enum {
    MMDIT_OK = 0,
    MMDIT_ERR_ARG = -1,          /* null pointer, negative size, bad dtype/eps/scale */
    MMDIT_ERR_SHAPE = -2,        /* sizes inconsistent (e.g. N != T*H*W, split sum != D) */
    MMDIT_ERR_ALIGN = -3,        /* a pointer is not 16-byte aligned */
    MMDIT_ERR_UNSUPPORTED = -4,  /* valid but not implemented (D != 128, C % 8 != 0, ...) */
    MMDIT_ERR_CUDA = -5,         /* a CUDA runtime / driver call failed */
    MMDIT_ERR_TIMEOUT = -6       /* a device-side bounded wait expired */
};

/* Visual token grid and RoPE parameters [Vimoo §2.2]: the visual stream holds
 * T*H*W tokens in raster order n = (t*H + h)*W + w.  Axis a in (T, H, W) owns
 * split[a] consecutive head dims (16, 56, 56 in the paper), pair j of that
 * chunk (dims 2j, 2j+1) turns by pos_a * pos_scale[a] * rope_base^(-2j/split[a]).
 * pos_scale is a per-axis position multiplier (1 = integer grid positions). */
typedef struct {
    int T, H, W;
    float pos_scale[3];
    float rope_base;
    int split[3];
} mmdit_grid;

/* QK-RMSNorm, then 3D RoPE [Vimoo §2.2: Q and K are RMS-normalised per head,
 * Q and K each with its own learned scale; the rotary embedding touches the
 * visual stream's Q and K and leaves the conditioning stream unrotated].
 *
 * For every (b, n, h) row of D values of q_in and of k_in:
 *   y = x / sqrt(mean(x^2) + eps) * scale[d]   (q_scale for q, k_scale for k)
 * and, when grid != NULL, y is then rotated by the RoPE of token n's (t, h, w).
 * grid == NULL is the conditioning stream (no rotation).
 *   q_in, k_in   [B, N, H, D] dt, read
 *   q_out, k_out [B, N, H, D] dt, written; may equal q_in / k_in (in place)
 *   q_scale, k_scale  [D] fp32
 *   grid: host pointer, read during the call only; requires N == T*H*W,
 *         split[] even and summing to D, positions (T-1,H-1,W-1) * pos_scale
 *         finite.
 * Errors: MMDIT_ERR_ARG / _SHAPE / _ALIGN / _UNSUPPORTED / _CUDA. */
MMDIT_API int mmdit_qk_norm_rope(const void* q_in, const void* k_in, void* q_out, void* k_out,
                       const float* q_scale, const float* k_scale,
                       int B, int N, int H, int D, const mmdit_grid* grid, float eps,
                       mmdit_dtype dt, void* stream);

/* Backward of mmdit_qk_norm_rope [the reverse-mode derivative of the QK-RMSNorm
 * + RoPE of Vimoo §2.2; the Seaweed-7B report, section 3.4, fuses the norm and
 * RoPE of both passes]: for each row x of q_in / k_in with r = sqrt(mean(x^2)
 * + eps), scale g and upstream gradient dy of the row of q_out / k_out:
 *   u  = R^T dy      (the RoPE rotation of the row, reversed; u = dy if grid is NULL)
 *   dx = g * u / r - x * sum_d(g * u * x) / (D r^3)
 *   dg = sum over all rows of u * x / r
 *   q_in, k_in       [B, N, H, D] dt, the forward's inputs
 *   dq_out, dk_out   [B, N, H, D] dt, gradients of the forward's outputs
 *   dq_in, dk_in     [B, N, H, D] dt, written (may equal dq_out / dk_out)
 *   q_scale, k_scale [D] fp32;  dq_scale, dk_scale [D] fp32, written
 *   grid, eps: as mmdit_qk_norm_rope (text positions: mmdit_qk_norm_rope_text_bwd).
 * dq_scale / dk_scale are summed with floating-point atomics, so their last
 * bits may differ from run to run.
 * Errors: MMDIT_ERR_ARG / _SHAPE / _ALIGN / _UNSUPPORTED / _CUDA. */
MMDIT_API int mmdit_qk_norm_rope_bwd(const void* q_in, const void* k_in, const void* dq_out,
                                     const void* dk_out, const float* q_scale,
                                     const float* k_scale, void* dq_in, void* dk_in,
                                     float* dq_scale, float* dk_scale, int B, int N, int H, int D,
                                     const mmdit_grid* grid, float eps, mmdit_dtype dt,
                                     void* stream);

/* Text-token positions of MM-RoPE ["Seaweed-7B: Cost-Effective Training of
 * Video Generation Foundation Model", section 3.2: text tokens get a 1D
 * position compatible with the video's 3D one, shared by its three
 * components]: conditioning token n sits at pos_offset + n on each of the T,
 * H and W axis chunks (split[] head dims each, frequencies rope_base^(-2j/d)
 * as for mmdit_grid).  Where the 1D positions start is the caller's choice. */
typedef struct {
    float pos_offset;
    float rope_base;
    int split[3];
} mmdit_text_rope;

/* QK-RMSNorm, then the MM-RoPE rotation of text tokens (see mmdit_text_rope):
 * the same normalisation and rotation as mmdit_qk_norm_rope, with every axis
 * chunk of token n rotated by the shared position pos_offset + n.  An
 * alternative to leaving the conditioning stream unrotated.
 *   q_in, k_in, q_out, k_out, q_scale, k_scale, eps, dt: as mmdit_qk_norm_rope
 *   rope: host pointer, read during the call only; split[] even, summing to D
 * Errors: MMDIT_ERR_ARG / _SHAPE / _ALIGN / _UNSUPPORTED / _CUDA. */
MMDIT_API int mmdit_qk_norm_rope_text(const void* q_in, const void* k_in, void* q_out,
                                      void* k_out, const float* q_scale, const float* k_scale,
                                      int B, int N, int H, int D, const mmdit_text_rope* rope,
                                      float eps, mmdit_dtype dt, void* stream);

/* Backward of mmdit_qk_norm_rope_text [the reverse-mode derivative of the
 * QK-RMSNorm and of the MM-RoPE text rotation, Seaweed-7B, section 3.2; the
 * same report's section 3.4 trains forward and backward]: as
 * mmdit_qk_norm_rope_bwd, with R the rotation of token n by the shared text
 * position pos_offset + n on every axis chunk.
 *   Arguments as mmdit_qk_norm_rope_bwd, with rope (host pointer, read during
 *   the call only; as mmdit_qk_norm_rope_text) in place of grid.
 * Errors: MMDIT_ERR_ARG / _SHAPE / _ALIGN / _UNSUPPORTED / _CUDA. */
MMDIT_API int mmdit_qk_norm_rope_text_bwd(const void* q_in, const void* k_in,
                                          const void* dq_out, const void* dk_out,
                                          const float* q_scale, const float* k_scale,
                                          void* dq_in, void* dk_in, float* dq_scale,
                                          float* dk_scale, int B, int N, int H, int D,
                                          const mmdit_text_rope* rope, float eps, mmdit_dtype dt,
                                          void* stream);

/* Joint non-causal attention over the concatenated streams, output split back
 * [Vimoo §2.2: each stream projects its own Q/K/V, one attention runs over the
 * two sequences joined end to end, and its output rows return to the stream
 * they came from].
 *
 * Per (b, h), with joint sequences Q = [q_vis; q_ctx], K = [k_vis; k_ctx],
 * V = [v_vis; v_ctx] (visual first; never materialised) and key j valid when
 * j < Nv or j - Nv < ctx_len[b]:
 *   O_i = sum_j softmax_j(Q_i . K_j * softmax_scale) V_j   over valid keys j,
 * rows i < Nv written to o_vis, the rest to o_ctx.  Cond query rows at index
 * >= ctx_len[b] (padding) are written as zeros.  A row with no valid key is 0.
 *   q_vis, k_vis, v_vis  [B, Nv, H, D] dt      q_ctx, k_ctx, v_ctx [B, Nc, H, D] dt
 *   ctx_len  DEVICE int32 [B], each clamped to [0, Nc]; NULL = all Nc valid
 *   o_vis [B, Nv, H, D] dt, o_ctx [B, Nc, H, D] dt  (written; must not alias inputs)
 *   softmax_scale > 0 (1/sqrt(D) in the usual form)
 * bf16 runs on the tcgen05 tensor cores (fp32 accumulation in tensor memory):
 * with Nv > 0 on clusters of two SMs that share one MMA-issuing thread
 * (cta_group::2 products of 256 query rows), else on one SM per work item; the
 * two give the same bits.  f32 runs an fp32 CUDA-core kernel.  Nv or Nc may be
 * 0 (the ctx pointers may then be NULL).
 * Errors: MMDIT_ERR_ARG / _SHAPE / _ALIGN / _UNSUPPORTED / _CUDA. */
MMDIT_API int mmdit_joint_attention(const void* q_vis, const void* k_vis, const void* v_vis,
                          const void* q_ctx, const void* k_ctx, const void* v_ctx,
                          const int32_t* ctx_len, void* o_vis, void* o_ctx,
                          int B, int Nv, int Nc, int H, int D, float softmax_scale,
                          mmdit_dtype dt, void* stream);

/* mmdit_qk_norm_rope for k alone: the RMSNorm (scale k_scale) and, with a
 * grid, the 3D RoPE of every row of k_in into k_out (may equal k_in).  Pairs
 * with mmdit_joint_attention_qnorm, which normalises q itself.
 * Errors: MMDIT_ERR_ARG / _SHAPE / _ALIGN / _UNSUPPORTED / _CUDA. */
MMDIT_API int mmdit_k_norm_rope(const void* k_in, void* k_out, const float* k_scale, int B, int N,
                                int H, int D, const mmdit_grid* grid, float eps, mmdit_dtype dt,
                                void* stream);

/* mmdit_joint_attention with the QK-RMSNorm and 3D RoPE of q done inside the
 * attention kernel [Vimoo §2.2 QK-norm and RoPE; the Seaweed-7B report,
 * section 3.4, fuses the attention preprocessing]: q_vis / q_ctx are the RAW
 * queries; each query tile is normalised (q_scale_vis / q_scale_ctx, [D] fp32,
 * eps) and, for visual rows when grid is not NULL, rotated by its grid
 * position, right after it is loaded and before any product reads it.  k_vis /
 * k_ctx must already be normalised and rotated (mmdit_k_norm_rope).  Saves
 * one write and one read of q against mmdit_qk_norm_rope + the attention.
 *   grid: host pointer as for mmdit_qk_norm_rope (Nv == T*H*W), or NULL for
 *   no rotation.  bf16 only (MMDIT_ERR_UNSUPPORTED otherwise).
 *   Other arguments as mmdit_joint_attention.
 * Errors: MMDIT_ERR_ARG / _SHAPE / _ALIGN / _UNSUPPORTED / _CUDA. */
MMDIT_API int mmdit_joint_attention_qnorm(const void* q_vis, const void* k_vis,
                                          const void* v_vis, const void* q_ctx,
                                          const void* k_ctx, const void* v_ctx,
                                          const int32_t* ctx_len, void* o_vis, void* o_ctx,
                                          const float* q_scale_vis, const float* q_scale_ctx,
                                          const mmdit_grid* grid, float eps, int B, int Nv,
                                          int Nc, int H, int D, float softmax_scale,
                                          mmdit_dtype dt, void* stream);

/* mmdit_joint_attention_qnorm with the split tail of mmdit_joint_attention_ws:
 * workspace (device, 256-byte aligned, workspace_bytes long, or NULL) lets the
 * items past the last whole wave of CTAs be split over their key tiles and
 * merged by a second kernel (each piece normalises its own copy of the query
 * tiles).  A NULL or too small workspace gives the unsplit launch.
 * Other arguments as mmdit_joint_attention_qnorm.
 * Errors: MMDIT_ERR_ARG (also workspace_bytes < 0) / _SHAPE / _ALIGN /
 * _UNSUPPORTED / _CUDA. */
MMDIT_API int mmdit_joint_attention_qnorm_ws(const void* q_vis, const void* k_vis,
                                             const void* v_vis, const void* q_ctx,
                                             const void* k_ctx, const void* v_ctx,
                                             const int32_t* ctx_len, void* o_vis, void* o_ctx,
                                             const float* q_scale_vis, const float* q_scale_ctx,
                                             const mmdit_grid* grid, float eps, void* workspace,
                                             long long workspace_bytes, int B, int Nv, int Nc,
                                             int H, int D, float softmax_scale, mmdit_dtype dt,
                                             void* stream);

/* Symmetric int8 quantisation for the 8-bit attention ["Wan 2.1" report,
 * section 4.4.3: Int8 for S = Q K^T]: x [B, N, H, D] bf16 -> codes [B, N, H, D]
 * int8 and one fp32 scale per `block` consecutive tokens of a (sample, head):
 * block = 1 (q: per token) or 128 (k: the attention's key tile).
 *   scale = max|x| / 127, code = round-half-even(x / scale) clamped to
 *   [-127, 127], both in fp32 (scale 0: codes 0); scales [B, H, ceil(N / block)].
 * Errors: MMDIT_ERR_ARG / _ALIGN / _UNSUPPORTED / _CUDA. */
MMDIT_API int mmdit_quantize_int8(const void* x, void* codes, float* scales, int B, int N, int H,
                                  int D, int block, void* stream);

/* FP8 E4M3 quantisation of v for the 8-bit attention [Wan 2.1, section 4.4.3:
 * FP8 for O = P V]: one fp32 scale per (sample, head, channel) over the valid
 * tokens of both streams (visual, and conditioning below ctx_len[b]):
 *   scale = max|v| / 448, code = E4M3(v / scale), half-even with saturation.
 *   v_vis [B, Nv, H, D], v_ctx [B, Nc, H, D] bf16 -> c_vis, c_ctx one byte per
 *   element (padded conditioning rows are encoded too); scales [B, H, D]
 *   (16-byte aligned; used as scratch during the call).
 * Errors: MMDIT_ERR_ARG / _ALIGN / _UNSUPPORTED / _CUDA. */
MMDIT_API int mmdit_quantize_v_e4m3(const void* v_vis, const void* v_ctx, const int32_t* ctx_len,
                                    void* c_vis, void* c_ctx, float* scales, int B, int Nv,
                                    int Nc, int H, int D, void* stream);

/* 8-bit joint attention [Wan 2.1, section 4.4.3: Int8 S = Q K^T, FP8 O = P V,
 * fp32 accumulation across key blocks; the joint streams of Vimoo §2.2]:
 *   S_ij = s_q[i] s_k[block(j)] (q8_i . k8_j), exactly in integers;
 *   online softmax over 128-key tiles with an integer running maximum m (log2
 *   units, raised to the ceiling of a tile maximum once that exceeds it by more
 *   than 2); P' = 2^(S_ij softmax_scale log2(e) - m + 6) rounded to E4M3 for
 *   the P V product, unrounded in the row sum;
 *   O_i = s_v * sum_j E4M3(P'_ij) v8_j / sum_j P'_ij over valid keys.
 *   q/k/v_vis [B, Nv, H, D], q/k/v_ctx [B, Nc, H, D]: codes from
 *   mmdit_quantize_int8 (q block 1, k block 128) and mmdit_quantize_v_e4m3;
 *   sq_vis / sq_ctx, sk_vis / sk_ctx, sv: their scales.
 *   o_vis, o_ctx: bf16 outputs as mmdit_joint_attention (padded rows zero).
 * Errors: MMDIT_ERR_ARG / _ALIGN / _UNSUPPORTED / _CUDA. */
MMDIT_API int mmdit_joint_attention_q8(const void* q_vis, const void* k_vis, const void* v_vis,
                                       const void* q_ctx, const void* k_ctx, const void* v_ctx,
                                       const float* sq_vis, const float* sq_ctx,
                                       const float* sk_vis, const float* sk_ctx, const float* sv,
                                       const int32_t* ctx_len, void* o_vis, void* o_ctx, int B,
                                       int Nv, int Nc, int H, int D, float softmax_scale,
                                       void* stream);

/* mmdit_joint_attention that also writes, for training, the row log-sum-exp
 * the backward pass needs [Vimoo §2.2 joint attention; the Seaweed-7B report,
 * section 3.4, trains its forward and backward]:
 *   lse[b, h, i] = log sum_j exp(Q_i . K_j * softmax_scale) over valid keys j
 * (natural log) for every joint row i (i < Nv visual, then conditioning), and
 * +infinity for rows without an output (padded conditioning rows, or no
 * valid key at all).
 *   lse: DEVICE fp32 [B, H, Nv + Nc], written; 4-byte aligned, not NULL
 *   everything else as mmdit_joint_attention.
 * Errors: MMDIT_ERR_ARG / _SHAPE / _ALIGN / _UNSUPPORTED / _CUDA. */
MMDIT_API int mmdit_joint_attention_fwd(const void* q_vis, const void* k_vis, const void* v_vis,
                                        const void* q_ctx, const void* k_ctx, const void* v_ctx,
                                        const int32_t* ctx_len, void* o_vis, void* o_ctx,
                                        float* lse, int B, int Nv, int Nc, int H, int D,
                                        float softmax_scale, mmdit_dtype dt, void* stream);

/* Joint attention with a device workspace for the split tail (a scheduling
 * choice of this library, not a step of the method): the same results as
 * mmdit_joint_attention / mmdit_joint_attention_fwd up to the order of the
 * floating-point sums [Vimoo §2.2 joint attention].
 *
 * The split applies to the one-SM bf16 kernel, which runs one CTA per SM,
 * one item (b, h, pair of 128-row query tiles) each, and every item costs the
 * same.  The items beyond the last whole wave would run as a short wave on a
 * few SMs; with a workspace, each of them is split over its keys into pieces
 * that run side by side, and a second kernel merges the pieces' partial rows
 * (rescaling them to a common maximum, as between key tiles).  Problems with
 * fewer items than SMs split every item.  Without lse and with Nv > 0 the call
 * runs the paired kernel of mmdit_joint_attention instead (faster whole than
 * the one-SM kernel split), and the workspace is unused.
 *   lse: DEVICE fp32 [B, H, Nv + Nc] as mmdit_joint_attention_fwd, or NULL
 *   workspace: DEVICE memory, 256-byte aligned, of workspace_bytes bytes, or
 *     NULL; MMDIT_ATTENTION_WORKSPACE_BYTES suffice for every problem.  The
 *     tail is split only when the workspace holds the plan's partials; else
 *     the call equals mmdit_joint_attention(_fwd).  Contents need no
 *     initialisation; calls overlapping on the GPU need separate workspaces.
 *   dt == MMDIT_F32 ignores the workspace.
 *   everything else as mmdit_joint_attention.
 * Errors: MMDIT_ERR_ARG / _SHAPE / _ALIGN / _UNSUPPORTED / _CUDA. */
#define MMDIT_ATTENTION_SPLIT_MAX_PIECES 160
#define MMDIT_ATTENTION_WORKSPACE_BYTES (MMDIT_ATTENTION_SPLIT_MAX_PIECES * 256LL * 130 * 4)
MMDIT_API int mmdit_joint_attention_ws(const void* q_vis, const void* k_vis, const void* v_vis,
                                       const void* q_ctx, const void* k_ctx, const void* v_ctx,
                                       const int32_t* ctx_len, void* o_vis, void* o_ctx,
                                       float* lse, void* workspace, long long workspace_bytes,
                                       int B, int Nv, int Nc, int H, int D, float softmax_scale,
                                       mmdit_dtype dt, void* stream);

/* The split-tail plan mmdit_joint_attention_ws follows for bf16 on a GPU of
 * num_sms SMs with a workspace of workspace_bytes (host arithmetic, no CUDA
 * call):
 *   plan[0]  items split (the last ones of the launch), 0: no split
 *   plan[1]  pieces per split item (0 when nothing is split)
 *   plan[2]  key tiles of 128 keys per piece (the last may hold fewer)
 *   plan[3]  CTAs of the attention launch
 * A split launch is followed by one merging launch.
 * Errors: MMDIT_ERR_ARG (negative size, num_sms < 1, plan NULL). */
MMDIT_API int mmdit_joint_attention_split_plan(int B, int Nv, int Nc, int H, int num_sms,
                                               long long workspace_bytes, long long* plan);

/* Backward of the joint attention [the reverse-mode derivative of the joint
 * attention of Vimoo §2.2; Seaweed-7B, section 3.4]: for the upstream
 * gradients do_vis / do_ctx of o_vis / o_ctx, with P the softmax of the
 * forward recomputed from lse and D_i = dO_i . O_i:
 *   dV_j = sum_i P_ij dO_i
 *   dS_ij = P_ij (dO_i . V_j - D_i)
 *   dQ_i = softmax_scale sum_j dS_ij K_j,   dK_j = softmax_scale sum_i dS_ij Q_i
 * over valid keys and over the query rows that have an output; padded
 * conditioning rows get zero dQ, dK and dV.
 *   q/k/v/o_vis, do_vis, dq/dk/dv_vis [B, Nv, H, D] dt (the d* written)
 *   q/k/v/o_ctx, do_ctx, dq/dk/dv_ctx [B, Nc, H, D] dt
 *   lse    DEVICE fp32 [B, H, Nv + Nc] from mmdit_joint_attention_fwd
 *   delta  DEVICE fp32 [B, H, Nv + Nc] caller-owned workspace, overwritten
 *          with D_i (contents on entry ignored)
 *   ctx_len, softmax_scale, dt: as mmdit_joint_attention (3D windows are
 *   not supported here).  Gradients must not alias any input.
 * bf16 runs three kernels: D, then dQ (query-stationary) and dK/dV
 * (key-stationary) on the tcgen05 tensor cores; f32 runs CUDA-core kernels.
 * Errors: MMDIT_ERR_ARG / _ALIGN / _UNSUPPORTED / _CUDA. */
MMDIT_API int mmdit_joint_attention_bwd(const void* q_vis, const void* k_vis, const void* v_vis,
                                        const void* q_ctx, const void* k_ctx, const void* v_ctx,
                                        const int32_t* ctx_len, const void* o_vis,
                                        const void* o_ctx, const void* do_vis, const void* do_ctx,
                                        const float* lse, float* delta, void* dq_vis,
                                        void* dk_vis, void* dv_vis, void* dq_ctx, void* dk_ctx,
                                        void* dv_ctx, int B, int Nv, int Nc, int H, int D,
                                        float softmax_scale, mmdit_dtype dt, void* stream);

/* Bytes of the workspace with which mmdit_joint_attention_bwd_ws (and
 * mmdit_joint_window_attention_bwd_ws) runs the one-pass backward: an fp32
 * dQ accumulator [B, Nv + Nc, H, 128]. */
#define MMDIT_BWD_WORKSPACE_BYTES(B, Nv, Nc, H) \
    ((long long)(B) * ((long long)(Nv) + (long long)(Nc)) * (long long)(H) * 512LL)

/* mmdit_joint_attention_bwd with a workspace for a one-pass backward [same
 * derivative as mmdit_joint_attention_bwd].  With bf16 and workspace_bytes >=
 * MMDIT_BWD_WORKSPACE_BYTES(B, Nv, Nc, H), one key-stationary kernel forms
 * dK, dV and dQ: S and dP are computed once per (key tile, query tile)
 * instead of once in a dQ kernel and again in a dK/dV kernel (10 N^2 D
 * executed FLOPs per sample and head instead of 14); each key tile adds its
 * share of dQ into the workspace with bulk reduce-adds, and a last kernel
 * scales the sums into bf16 dQ.  The order of those additions varies from
 * run to run, so dQ is not bit-reproducible (dK and dV are; the gradients of
 * mmdit_joint_attention_bwd are).  With f32, a NULL workspace or a smaller
 * one, the call is mmdit_joint_attention_bwd.
 *   workspace  DEVICE, 256-byte aligned, caller-owned, contents on entry
 *              ignored and overwritten; must not overlap any other argument
 *   workspace_bytes  its size
 *   everything else as mmdit_joint_attention_bwd.
 * Errors: as mmdit_joint_attention_bwd; MMDIT_ERR_ARG for workspace_bytes < 0,
 * MMDIT_ERR_ALIGN for a workspace not 256-byte aligned. */
MMDIT_API int mmdit_joint_attention_bwd_ws(const void* q_vis, const void* k_vis, const void* v_vis,
                                           const void* q_ctx, const void* k_ctx, const void* v_ctx,
                                           const int32_t* ctx_len, const void* o_vis,
                                           const void* o_ctx, const void* do_vis,
                                           const void* do_ctx, const float* lse, float* delta,
                                           void* workspace, long long workspace_bytes,
                                           void* dq_vis, void* dk_vis, void* dv_vis, void* dq_ctx,
                                           void* dk_ctx, void* dv_ctx, int B, int Nv, int Nc,
                                           int H, int D, float softmax_scale, mmdit_dtype dt,
                                           void* stream);

/* Largest B * H * (Nv + Nc) that mmdit_joint_attention_bwd_noalloc accepts:
 * 4,194,304 rows (its built-in workspace is 16 MiB of fp32 per GPU). */
#define MMDIT_NOALLOC_MAX_ROWS (1 << 22)

/* mmdit_joint_attention_bwd for callers that cannot allocate device memory.
 * No passage of the papers corresponds to this entry point: it exists for
 * callers that must not call cudaMalloc at the point where they run the
 * backward, for example because another allocator owns the device memory, an
 * engine forbids allocation once it runs, or a stream is being captured.
 * Instead of the caller's `delta` workspace it uses a fixed array built into
 * the library (MMDIT_NOALLOC_MAX_ROWS floats, held on every GPU that loads the
 * library until the process exits), so the call allocates nothing.
 *   Arguments, results and errors: as mmdit_joint_attention_bwd without
 *   `delta`.  B * H * (Nv + Nc) above MMDIT_NOALLOC_MAX_ROWS returns
 *   MMDIT_ERR_UNSUPPORTED.
 *   All calls on one GPU share the array: calls whose kernels can overlap on
 *   the GPU (different streams) race and must be ordered by the caller.
 *   The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.  The address is kept for the life of the
 *   process, so resetting a device (cudaDeviceReset) after that first call is
 *   not supported: the kept address would then point into a released module. */
MMDIT_API int mmdit_joint_attention_bwd_noalloc(
    const void* q_vis, const void* k_vis, const void* v_vis, const void* q_ctx, const void* k_ctx,
    const void* v_ctx, const int32_t* ctx_len, const void* o_vis, const void* o_ctx,
    const void* do_vis, const void* do_ctx, const float* lse, void* dq_vis, void* dk_vis,
    void* dv_vis, void* dq_ctx, void* dk_ctx, void* dv_ctx, int B, int Nv, int Nc, int H, int D,
    float softmax_scale, mmdit_dtype dt, void* stream);

/* 3D window partition of the visual grid ["Seaweed-7B", section 3.2: attention
 * restricted to w_t x w_h x w_w windows, e.g. 1x2x2 and 4x1x1 in alternating
 * layers].  parts[a] is the number of windows along axis a (T, H, W), each in
 * [1, extent of the axis], product at most 64.  An axis of extent X split into
 * p windows: window k starts at k*(X/p) + min(k, X%p); the first X%p windows
 * are one position longer.
 * Window-major token order: windows one after another, T part slowest, W part
 * fastest; inside a window its tokens keep raster order. */
typedef struct {
    int parts[3];
} mmdit_window;

/* mmdit_qk_norm_rope for the visual stream, storing the rows in window-major
 * order for mmdit_joint_window_attention: row (b, n, h) of q_in / k_in
 * (raster order, RoPE at its grid position) is written to row
 * (b, window_major(n), h) of q_out / k_out.
 *   Arguments as mmdit_qk_norm_rope (grid required); win: host pointer.
 *   q_out, k_out must not overlap q_in or k_in.
 * Errors: MMDIT_ERR_ARG / _SHAPE / _ALIGN / _UNSUPPORTED / _CUDA. */
MMDIT_API int mmdit_qk_norm_rope_window(const void* q_in, const void* k_in, void* q_out,
                                        void* k_out, const float* q_scale, const float* k_scale,
                                        int B, int N, int H, int D, const mmdit_grid* grid,
                                        const mmdit_window* win, float eps, mmdit_dtype dt,
                                        void* stream);

/* Reorders rows of C elements between raster and window-major order:
 * inverse == 0: y[b, window_major(n)] = x[b, n]; otherwise
 * y[b, n] = x[b, window_major(n)].  Used for v (C = H*D) before
 * mmdit_joint_window_attention; a pure copy.
 *   x, y [B, N, C] dt, N == T*H*W of grid, C*sizeof(dt) a multiple of 16;
 *   y must not overlap x.  grid, win: host pointers (only T, H, W are read).
 * Errors: MMDIT_ERR_ARG / _SHAPE / _ALIGN / _UNSUPPORTED / _CUDA. */
MMDIT_API int mmdit_window_permute(const void* x, void* y, int B, int N, int C,
                                   const mmdit_grid* grid, const mmdit_window* win, int inverse,
                                   mmdit_dtype dt, void* stream);

/* Joint attention restricted to 3D windows ["Seaweed-7B", section 3.2, with
 * the joint streams of Vimoo §2.2]: a visual query row attends to the visual
 * keys of its own window and to every valid conditioning key; a conditioning
 * query row attends to every valid key, as in mmdit_joint_attention.
 *   q_vis, k_vis, v_vis  [B, Nv, H, D] dt in WINDOW-MAJOR order (as written
 *                        by mmdit_qk_norm_rope_window / mmdit_window_permute)
 *   o_vis [B, Nv, H, D] dt written in RASTER order
 *   grid, win: host pointers; Nv == T*H*W (only T, H, W are read)
 *   everything else as mmdit_joint_attention.
 * Errors: MMDIT_ERR_ARG / _SHAPE / _ALIGN / _UNSUPPORTED / _CUDA. */
MMDIT_API int mmdit_joint_window_attention(const void* q_vis, const void* k_vis,
                                           const void* v_vis, const void* q_ctx,
                                           const void* k_ctx, const void* v_ctx,
                                           const int32_t* ctx_len, void* o_vis, void* o_ctx,
                                           int B, int Nv, int Nc, int H, int D,
                                           const mmdit_grid* grid, const mmdit_window* win,
                                           float softmax_scale, mmdit_dtype dt, void* stream);

/* mmdit_joint_window_attention that also writes, for training, the row
 * log-sum-exp the window backward needs [Seaweed-7B, section 3.2 windows;
 * section 3.4 trains forward and backward]:
 *   lse[b, h, r] = log sum_j exp(Q_r . K_j * softmax_scale) over the keys row r
 *   sees (natural log), +infinity for rows without an output.  Rows are in
 *   the order of the INPUTS: r < Nv is the window-major visual row (as q_vis),
 *   then the conditioning rows.
 *   lse: DEVICE fp32 [B, H, Nv + Nc], written; 4-byte aligned, not NULL
 *   everything else as mmdit_joint_window_attention (o_vis in raster order).
 * Errors: MMDIT_ERR_ARG / _SHAPE / _ALIGN / _UNSUPPORTED / _CUDA. */
MMDIT_API int mmdit_joint_window_attention_fwd(const void* q_vis, const void* k_vis,
                                               const void* v_vis, const void* q_ctx,
                                               const void* k_ctx, const void* v_ctx,
                                               const int32_t* ctx_len, void* o_vis, void* o_ctx,
                                               float* lse, int B, int Nv, int Nc, int H, int D,
                                               const mmdit_grid* grid, const mmdit_window* win,
                                               float softmax_scale, mmdit_dtype dt,
                                               void* stream);

/* Backward of the 3D window joint attention [the reverse-mode derivative of
 * mmdit_joint_window_attention; Seaweed-7B, section 3.2 windows, section 3.4
 * forward and backward]: the gradients of mmdit_joint_attention_bwd with each
 * row's key set restricted as the window forward restricts it (a visual row
 * sees its own window's visual keys and the valid conditioning keys; a
 * conditioning row sees every valid key).
 *   Every VISUAL tensor is in window-major order (the order of q_vis): q_vis,
 *   k_vis, v_vis, o_vis, do_vis (permute the raster o and its gradient with
 *   mmdit_window_permute), the outputs dq_vis, dk_vis, dv_vis (the inverse
 *   mmdit_window_permute returns them to raster order), and the visual rows
 *   of lse (from mmdit_joint_window_attention_fwd) and of delta.
 *   grid, win: as mmdit_joint_window_attention; everything else as
 *   mmdit_joint_attention_bwd.
 * Errors: MMDIT_ERR_ARG / _SHAPE / _ALIGN / _UNSUPPORTED / _CUDA. */
MMDIT_API int mmdit_joint_window_attention_bwd(
    const void* q_vis, const void* k_vis, const void* v_vis, const void* q_ctx, const void* k_ctx,
    const void* v_ctx, const int32_t* ctx_len, const void* o_vis, const void* o_ctx,
    const void* do_vis, const void* do_ctx, const float* lse, float* delta, void* dq_vis,
    void* dk_vis, void* dv_vis, void* dq_ctx, void* dk_ctx, void* dv_ctx, int B, int Nv, int Nc,
    int H, int D, const mmdit_grid* grid, const mmdit_window* win, float softmax_scale,
    mmdit_dtype dt, void* stream);

/* mmdit_joint_window_attention_bwd with the workspace of
 * mmdit_joint_attention_bwd_ws: the one-pass backward (dQ reduced into the
 * workspace, not bit-reproducible) when bf16 and workspace_bytes >=
 * MMDIT_BWD_WORKSPACE_BYTES(B, Nv, Nc, H), else mmdit_joint_window_attention_bwd.
 * The accumulator's visual rows are in window-major order like dq_vis.
 *   workspace, workspace_bytes: as mmdit_joint_attention_bwd_ws; everything
 *   else as mmdit_joint_window_attention_bwd.
 * Errors: as mmdit_joint_window_attention_bwd and mmdit_joint_attention_bwd_ws. */
MMDIT_API int mmdit_joint_window_attention_bwd_ws(
    const void* q_vis, const void* k_vis, const void* v_vis, const void* q_ctx, const void* k_ctx,
    const void* v_ctx, const int32_t* ctx_len, const void* o_vis, const void* o_ctx,
    const void* do_vis, const void* do_ctx, const float* lse, float* delta, void* workspace,
    long long workspace_bytes, void* dq_vis, void* dk_vis, void* dv_vis, void* dq_ctx,
    void* dk_ctx, void* dv_ctx, int B, int Nv, int Nc, int H, int D, const mmdit_grid* grid,
    const mmdit_window* win, float softmax_scale, mmdit_dtype dt, void* stream);

/* adaLN modulate [Vimoo §2.2: a LayerNorm sits before attention and the FFN,
 * and the timestep embedding supplies a shift and a scale for its output]:
 *   y = LN(x) * (1 + scale[b]) + shift[b], LN over C without an affine,
 *   biased variance.
 *   x [B, N, C] dt read;  y [B, N, C] dt written (may equal x)
 *   shift, scale [B, C] fp32;  C % 8 == 0 and C <= 4096 (bf16) / 2048 (f32)
 * Errors: MMDIT_ERR_ARG / _ALIGN / _UNSUPPORTED / _CUDA. */
MMDIT_API int mmdit_adaln_modulate(const void* x, const float* shift, const float* scale, void* y,
                         int B, int N, int C, float eps, mmdit_dtype dt, void* stream);

/* mmdit_adaln_modulate of both streams of a block in ONE launch [Vimoo §2.2:
 * each stream has its own LayerNorm and its own shift and scale]: rows of the
 * visual stream use (shift_vis, scale_vis), rows of the conditioning stream
 * (shift_ctx, scale_ctx).  The results equal two mmdit_adaln_modulate calls
 * bit for bit; one launch keeps the short conditioning stream from costing a
 * launch of its own.
 *   x_vis, y_vis [B, N_vis, C] dt;  x_ctx, y_ctx [B, N_ctx, C] dt (y may
 *   equal its own x); shift_*, scale_* [B, C] fp32.  N_vis or N_ctx may be 0
 *   (that stream's pointers are then not read).  C, eps, dt as
 *   mmdit_adaln_modulate.
 * Errors: MMDIT_ERR_ARG / _ALIGN / _UNSUPPORTED / _CUDA. */
MMDIT_API int mmdit_adaln_modulate_pair(const void* x_vis, const float* shift_vis,
                                        const float* scale_vis, void* y_vis, int N_vis,
                                        const void* x_ctx, const float* shift_ctx,
                                        const float* scale_ctx, void* y_ctx, int N_ctx, int B,
                                        int C, float eps, mmdit_dtype dt, void* stream);

/* Gated residual [Vimoo §2.2: a per-channel gate from the timestep embedding
 * weighs each branch before it is added back to the residual stream]:
 *   out = x + gate[b] * branch.
 *   x, branch [B, N, C] dt read;  out [B, N, C] dt written (may equal x)
 *   gate [B, C] fp32;  C % 8 == 0
 * Errors: MMDIT_ERR_ARG / _ALIGN / _UNSUPPORTED / _CUDA. */
MMDIT_API int mmdit_gated_residual(const void* x, const void* branch, const float* gate, void* out,
                         int B, int N, int C, mmdit_dtype dt, void* stream);

/* Backward of mmdit_adaln_modulate [the reverse-mode derivative of the adaLN
 * modulate of Vimoo §2.2]: for the upstream gradient dy of y, with
 * xh = (x - mean) / sqrt(var + eps) per row of C values,
 *   g  = dy * (1 + scale[b])
 *   dx = (g - mean_c(g) - xh * mean_c(g * xh)) / sqrt(var + eps)
 *   dshift[b, c] = sum over the rows of sample b of dy
 *   dscale[b, c] = sum over the rows of sample b of dy * xh
 *   x, dy [B, N, C] dt read;  dx [B, N, C] dt written (may equal dy, not x)
 *   scale [B, C] fp32;  dshift, dscale [B, C] fp32 written (zeroed, then summed
 *   with floating-point atomics: their last bits may differ from run to run)
 *   C % 8 == 0 and C <= 4096 (bf16) / 2048 (f32)
 * Errors: MMDIT_ERR_ARG / _ALIGN / _UNSUPPORTED / _CUDA. */
MMDIT_API int mmdit_adaln_modulate_bwd(const void* x, const float* scale, const void* dy,
                                       void* dx, float* dshift, float* dscale, int B, int N,
                                       int C, float eps, mmdit_dtype dt, void* stream);

/* Backward of mmdit_gated_residual [the reverse-mode derivative of the gated
 * residual of Vimoo §2.2]: for the upstream gradient dout of out,
 *   dx = dout,  dbranch = gate[b] * dout,
 *   dgate[b, c] = sum over the rows of sample b of dout * branch
 *   branch, dout [B, N, C] dt read;  dbranch [B, N, C] dt written (may equal
 *   dout, not branch);  dx [B, N, C] dt written, or NULL (it equals dout)
 *   gate [B, C] fp32;  dgate [B, C] fp32 written (zeroed, then summed with
 *   floating-point atomics);  C % 8 == 0 and C <= 4096 (bf16) / 2048 (f32)
 * Errors: MMDIT_ERR_ARG / _ALIGN / _UNSUPPORTED / _CUDA. */
MMDIT_API int mmdit_gated_residual_bwd(const void* branch, const float* gate, const void* dout,
                                       void* dx, void* dbranch, float* dgate, int B, int N,
                                       int C, mmdit_dtype dt, void* stream);

/* Gated residual fused with the adaLN modulate that follows it, in one pass
 * over memory [Vimoo §2.2: a branch's gated contribution is added to the
 * residual stream, and the next branch starts from a LayerNorm of that stream
 * modulated by its own shift and scale]:
 *   x_out = x + gate[b] * branch                      (stored in dt)
 *   y     = LN(x_out) * (1 + scale[b]) + shift[b]     (LN of x_out as stored)
 * Equal to mmdit_gated_residual followed by mmdit_adaln_modulate, with one
 * read of x fewer.
 *   x, branch [B, N, C] dt read;  x_out [B, N, C] written (may equal x);
 *   y [B, N, C] written (must not alias x, branch or x_out)
 *   gate [B, C] fp32 (this branch);  shift, scale [B, C] fp32 (next branch)
 *   C % 8 == 0 and C <= 3072 (bf16) / 1536 (f32)
 * Errors: MMDIT_ERR_ARG / _ALIGN / _UNSUPPORTED / _CUDA. */
MMDIT_API int mmdit_residual_modulate(const void* x, const void* branch, const float* gate,
                                      const float* shift, const float* scale, void* x_out,
                                      void* y, int B, int N, int C, float eps, mmdit_dtype dt,
                                      void* stream);

/* ---- Host-buffer executor -------------------------------------------------
 *
 * Runs the whole path of one block, step after step, from HOST buffers
 * [Vimoo §2.2, the dual-stream block]:
 *   y   = adaLN modulate of x                    (mmdit_adaln_modulate_pair)
 *   q,k = QK-RMSNorm (+ 3D RoPE on the visual stream)   (mmdit_qk_norm_rope)
 *   o   = joint attention over both streams      (mmdit_joint_attention_ws)
 *   x'  = x + gate * o                           (mmdit_gated_residual, both streams)
 * The projections of a full block (QKV, output, MLP) are outside this library:
 * q, k, v arrive as inputs and the attention output is the gated branch.  Each
 * step is the same computation, with the same kernels and results, as these
 * six calls made one after the other on device buffers (the attention with a
 * workspace of MMDIT_ATTENTION_WORKSPACE_BYTES, which each slot holds).
 *
 * Unlike the rest of this header, the executor moves data between host and
 * device itself: it copies a step's inputs in, runs the kernels and copies the
 * outputs back.  It pipelines the steps over three CUDA streams of its own, so
 * that one step's input copy, another step's kernels and a third step's output
 * copy run at the same time.  Device memory comes from a caller-provided
 * workspace cut into slots of mmdit_block_slot_bytes() bytes; each step takes a
 * slot, and a slot is reused only once the step that held it has copied its
 * outputs out.  Three slots keep the copies and the kernels all busy; one slot
 * runs the steps one after the other. */

/* Sizes and constants shared by every step. */
typedef struct {
    int B, Nv, Nc, H, D;      /* batch, visual tokens, cond tokens, heads, head dim (128);
                                 C = H * D */
    mmdit_grid grid;          /* visual token grid (T*H*W == Nv) and its RoPE */
    const float* gq_vis;      /* DEVICE [D] fp32 RMSNorm scales of q and k per stream */
    const float* gk_vis;
    const float* gq_ctx;      /* may be NULL when Nc == 0 */
    const float* gk_ctx;
    float norm_eps;           /* QK-RMSNorm eps */
    float ln_eps;             /* adaLN LayerNorm eps */
    float softmax_scale;      /* > 0 (1/sqrt(D) in the usual form) */
    mmdit_dtype dt;
} mmdit_block_config;

/* HOST buffers of one step, laid out as in the device entry points above.
 * Page-locked (pinned) memory lets the copies run asynchronously and overlap
 * the kernels; pageable memory gives the same results without the overlap. */
typedef struct {
    const void* q_vis;         /* [B, Nv, H, D] dt */
    const void* k_vis;
    const void* v_vis;
    const void* q_ctx;         /* [B, Nc, H, D] dt (unused when Nc == 0) */
    const void* k_ctx;
    const void* v_ctx;
    const void* x_vis;         /* [B, Nv, C] dt residual stream */
    const void* x_ctx;         /* [B, Nc, C] dt */
    const float* shift_vis;    /* [B, C] fp32 adaLN shift, scale and gate per stream */
    const float* scale_vis;
    const float* gate_vis;
    const float* shift_ctx;
    const float* scale_ctx;
    const float* gate_ctx;
    const int32_t* ctx_len;    /* [B], or NULL: all Nc cond tokens valid */
    void* y_vis;               /* out [B, Nv, C] dt: modulated x, or NULL: not copied back */
    void* y_ctx;
    void* o_vis;               /* out [B, Nv, H, D] dt: attention output, or NULL */
    void* o_ctx;
    void* x_out_vis;           /* out [B, Nv, C] dt: x + gate * o (required) */
    void* x_out_ctx;           /* required when Nc > 0 */
} mmdit_block_step;

/* Device bytes one step's slot needs, or a negative MMDIT_ERR_* code if the
 * configuration is invalid.  Makes no CUDA call. */
MMDIT_API long long mmdit_block_slot_bytes(const mmdit_block_config* cfg);

/* Runs steps[0..n_steps) in order, each from and to its own host buffers.
 *   workspace: DEVICE memory, 256-byte aligned, workspace_bytes long; the
 *     executor uses floor(workspace_bytes / slot bytes) slots (at most 4, at
 *     most n_steps) and must not be given less than one slot.
 *   stream: the work starts after what is already queued on `stream`, and
 *     everything queued on `stream` afterwards waits for the last output copy.
 *     The call returns once the work is enqueued; synchronise `stream` before
 *     reading the host outputs or reusing the host inputs.
 * Host input buffers may be shared between steps; output buffers of different
 * steps may also coincide (the output copies run in step order, so the last
 * step's values remain).  The workspace must not be used by anything else
 * until the work has finished.
 * Errors: MMDIT_ERR_ARG / _SHAPE / _ALIGN / _UNSUPPORTED before anything is
 * enqueued; MMDIT_ERR_CUDA if a CUDA call fails while enqueueing (work already
 * enqueued still completes before later work on `stream`). */
MMDIT_API int mmdit_block_forward_host(const mmdit_block_config* cfg,
                                       const mmdit_block_step* steps, int n_steps,
                                       void* workspace, long long workspace_bytes, void* stream);

/* Synchronises `stream`, then returns and clears the device status word of the
 * current device: MMDIT_OK, or MMDIT_ERR_TIMEOUT if a kernel gave up on a
 * bounded wait since the last call (its outputs are then undefined), or
 * MMDIT_ERR_CUDA if the synchronisation failed. */
MMDIT_API int mmdit_device_status(void* stream);

/* Sets the limit of one bounded wait inside the attention kernels (forward and
 * backward) and the modulate backward for launches made after the call,
 * process-wide: 0 restores the default (2 s).  A wait that
 * runs out makes every role of the kernel stop (outputs undefined), drain the
 * copies and tensor-core work it issued, free its tensor memory and return;
 * the next mmdit_device_status() then reports MMDIT_ERR_TIMEOUT.  No fault or
 * trap is involved, so the CUDA context stays usable.  Meant for diagnostics
 * and for testing that path; the default never expires on a healthy GPU. */
MMDIT_API void mmdit_set_wait_timeout_ns(unsigned long long ns);

/* Text of the CUDA error behind the calling thread's most recent
 * MMDIT_ERR_CUDA return (which call failed and the CUDA error name), or "" if
 * none.  Thread-local storage owned by the library, valid until the thread's
 * next call into the library. */
MMDIT_API const char* mmdit_last_error(void);

/* Human-readable text of a status code (static storage). */
MMDIT_API const char* mmdit_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* MMDIT_H */
