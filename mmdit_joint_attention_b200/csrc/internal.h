// Launchers shared between the C-ABI layer (abi.cu) and the kernel files.
// Arguments arrive already validated by abi.cu.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/mmdit.h"
#include "window.h"

namespace mmdit {

struct RopeGrid {
    int T, H, W;
    double pos_scale[3];
    double base;
    int split[3];
};

// MM-RoPE positions of text tokens: token n at pos_offset + n on all three axes.
struct RopeText {
    double pos_offset;
    double base;
    int split[3];
};

// Validates a RoPE grid for N tokens of head dim D and converts it: MMDIT_OK
// or the MMDIT_ERR_* code the entry points return for it.
int check_grid(const mmdit_grid* grid, long long N, int D, mmdit_dtype dt, RopeGrid& g);

// 0 or a cudaError_t value.  At most one of grid / text is non-null.
// q_in == null: k alone (no text positions, no permutation).
// win_parts (grid mode only, else null): store the rows in the window-major
// order of that 3D window partition (window.h) instead of in place.
cudaError_t launch_qk_norm_rope(const void* q_in, const void* k_in, void* q_out, void* k_out,
                                const float* gq, const float* gk, int B, int N, int H,
                                const RopeGrid* grid, const RopeText* text, const int* win_parts,
                                float eps, bool bf16, cudaStream_t s);

// Backward of launch_qk_norm_rope (grid, text positions or none, at most one
// of them; no permutation): dq_in / dk_in written, dgq / dgk [128] zeroed
// then summed.
cudaError_t launch_qk_norm_rope_bwd(const void* q_in, const void* k_in, const void* dq_out,
                                    const void* dk_out, const float* gq, const float* gk,
                                    void* dq_in, void* dk_in, float* dgq, float* dgk, int B, int N,
                                    int H, const RopeGrid* grid, const RopeText* text, float eps,
                                    bool bf16, cudaStream_t s);

// Rows of row_bytes (a multiple of 16) of [B, N] between raster order and the
// window-major order of `parts` (window.h); inverse: window-major -> raster.
cudaError_t launch_window_permute(const void* x, void* y, int B, int N, int row_bytes,
                                  const RopeGrid& grid, const int* parts, bool inverse,
                                  cudaStream_t s);

cudaError_t launch_adaln_modulate(const void* x, const float* shift, const float* scale,
                                  void* y, int B, int N, int C, float eps, bool bf16,
                                  cudaStream_t s);

// The adaLN modulate of two streams (index 0 visual, 1 conditioning) with the
// same B and C in one launch; a stream with N == 0 is absent.
struct ModStreamsHost {
    const void* x[2];
    void* y[2];
    const float* shift[2];
    const float* scale[2];
    int N[2];
};
cudaError_t launch_adaln_modulate_pair(const ModStreamsHost& h, int B, int C, float eps,
                                       bool bf16, cudaStream_t s);

cudaError_t launch_residual_modulate(const void* x, const void* branch, const float* gate,
                                     const float* shift, const float* scale, void* x_out, void* y,
                                     int B, int N, int C, float eps, bool bf16, cudaStream_t s);

cudaError_t launch_gated_residual(const void* x, const void* branch, const float* gate,
                                  void* out, int B, int N, int C, bool bf16, cudaStream_t s);

// Returns 0 on success, a cudaError_t value on CUDA failure, or -1 if the
// driver entry point for tensor-map encoding is unavailable.
// win (null: full joint attention): 3D window attention; the visual inputs
// are then in the table's window-major order and o_vis is written in raster
// order.
// Q-norm mode of the attention kernel: q arrives raw and is RMS-normalised
// (scale gq[stream]) and, on visual rows when grid is set, rotated in the
// kernel.
struct QNormArgs {
    const float* gq[2];
    const RopeGrid* grid;
    float eps;
};

// Split-tail plan of a full bf16 launch on num_sms SMs with a workspace of
// ws_bytes: `tail` items (the last ones) in `parts` pieces of `per` key tiles
// each, the first `first` items whole, `ctas` CTAs in all (the plain
// launch's count when parts == 0: no split).  Host arithmetic only.
struct SplitPlan {
    int tail, parts, per, first;
    long long ctas;
};
SplitPlan split_plan(int B, int Nv, int Nc, int H, int num_sms, long long ws_bytes);

// lse (null: not written): [B, H, Nv + Nc] natural-log row log-sum-exp of
// the scaled scores, +infinity for rows without an output.  qn (null: q is
// already normalised).  split_ws (null: off; full mode only): workspace of
// split_ws_bytes for the split tail, used when the plan's partials fit.
int launch_joint_attention_bf16(const void* qv, const void* kv, const void* vv,
                                const void* qc, const void* kc, const void* vc,
                                const int32_t* ctx_len, void* ov, void* oc, float* lse, int B,
                                int Nv, int Nc, int H, float softmax_scale,
                                const WindowTable* win, cudaStream_t s,
                                const QNormArgs* qn = nullptr, float* split_ws = nullptr,
                                long long split_ws_bytes = 0);

cudaError_t launch_joint_attention_f32(const float* qv, const float* kv, const float* vv,
                                       const float* qc, const float* kc, const float* vc,
                                       const int32_t* ctx_len, float* ov, float* oc, float* lse,
                                       int B, int Nv, int Nc, int H, float softmax_scale,
                                       const WindowTable* win, cudaStream_t s);

// Joint-attention backward.  delta: caller workspace [B, H, Nv + Nc] fp32
// (row sums of dO * O, written here); lse from the forward.  win (null: full
// joint attention): 3D window attention, with every visual tensor
// (q, k, v, o, dO, the d* outputs, and the visual rows of lse and delta) in
// the table's window-major order.  dq_acc (null: the two-kernel form, dQ and
// dK/dV apart): caller workspace [B, Nv + Nc, H, 128] fp32 for the one-pass
// form, which reduces dQ into it (contents on entry ignored).  Return
// convention of launch_joint_attention_bf16.
int launch_joint_attention_bwd_bf16(const void* qv, const void* kv, const void* vv,
                                    const void* qc, const void* kc, const void* vc,
                                    const int32_t* ctx_len, const void* ov, const void* oc,
                                    const void* dov, const void* doc, const float* lse,
                                    float* delta, void* dqv, void* dkv, void* dvv, void* dqc,
                                    void* dkc, void* dvc, int B, int Nv, int Nc, int H,
                                    float softmax_scale, cudaStream_t s,
                                    const WindowTable* win = nullptr, float* dq_acc = nullptr);
cudaError_t launch_joint_attention_bwd_f32(const float* qv, const float* kv, const float* vv,
                                           const float* qc, const float* kc, const float* vc,
                                           const int32_t* ctx_len, const float* ov,
                                           const float* oc, const float* dov, const float* doc,
                                           const float* lse, float* delta, float* dqv, float* dkv,
                                           float* dvv, float* dqc, float* dkc, float* dvc, int B,
                                           int Nv, int Nc, int H, float softmax_scale,
                                           cudaStream_t s, const WindowTable* win = nullptr);

// 8-bit joint attention: int8 q / k codes with q row scales [B, H, N_s] and k
// block scales [B, H, ceil(N_s / 128)], E4M3 v codes with channel scales
// [B, H, 128]; bf16 outputs.  Return convention of the bf16 launcher.
int launch_joint_attention_q8(const void* qv, const void* kv, const void* vv, const void* qc,
                              const void* kc, const void* vc, const float* sqv, const float* sqc,
                              const float* skv, const float* skc, const float* sv,
                              const int32_t* ctx_len, void* ov, void* oc, int B, int Nv, int Nc,
                              int H, float softmax_scale, cudaStream_t s);
// int8 codes of bf16 x [B, N, H, 128] with one scale per `block` (1 or 128)
// consecutive tokens of a (sample, head): scales [B, H, ceil(N / block)].
cudaError_t launch_quant_int8(const void* x, void* codes, float* scales, int B, int N, int H,
                              int block, cudaStream_t s);
// E4M3 codes of bf16 v of both streams with one scale per (sample, head,
// channel) over the valid tokens: scales [B, H, 128].
cudaError_t launch_quant_v_e4m3(const void* vv, const void* vc, const int32_t* ctx_len, void* cv,
                                void* cc, float* scales, int B, int Nv, int Nc, int H,
                                cudaStream_t s);
cudaError_t read_and_clear_q8_status(unsigned int* out);
// The same for the pair kernel (attention_pair.cu).
cudaError_t read_and_clear_pair_status(unsigned int* out);
// Plain bf16 joint attention (no windows, no Q normalisation, no lse) on CTA
// pairs with one MMA-issuing thread per pair; outputs bit for bit those of
// launch_joint_attention_bf16's kernel.  Return convention of
// launch_joint_attention_bf16.
int launch_joint_attention_pair(const void* qv, const void* kv, const void* vv, const void* qc,
                                const void* kc, const void* vc, const int32_t* ctx_len, void* ov,
                                void* oc, int B, int Nv, int Nc, int H, float softmax_scale,
                                cudaStream_t s);

// Limit of one bounded pipeline wait (set_wait_timeout_ns, else the default).
uint64_t wait_timeout_ns();

// Limit of one bounded pipeline wait in the attention kernel (0 = default).
void set_wait_timeout_ns(unsigned long long ns);

// Device status word (bit set = a bounded wait expired): read-and-clear.
cudaError_t read_and_clear_device_status(unsigned int* out, cudaStream_t s);
// The same for the backward kernels' own status word.
cudaError_t read_and_clear_bwd_status(unsigned int* out);
// The same for the elementwise backward kernels.
cudaError_t read_and_clear_elem_status(unsigned int* out);

constexpr int kHeadDim = 128;

// Records the CUDA error behind an MMDIT_ERR_CUDA return for mmdit_last_error().
void set_last_error(const char* where, int code);

}  // namespace mmdit
