// C ABI of libmmdit.so (declared in include/mmdit.h): argument validation, then
// one launch per call on the caller's stream.  No device memory is allocated.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>

#include "../../include/mmdit.h"
#include "internal.h"

using namespace mmdit;

namespace {

thread_local char g_last_error[256] = "";

}  // namespace

void mmdit::set_last_error(const char* where, int code) {
    const char* name = code >= 1000 ? "cuTensorMapEncodeTiled rejected a tensor map"
                       : code > 0   ? cudaGetErrorName(static_cast<cudaError_t>(code))
                                    : "driver entry point cuTensorMapEncodeTiled unavailable";
    std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%d)", where, name, code);
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int cuda_status(cudaError_t e, const char* where) {
    if (e == cudaSuccess) return MMDIT_OK;
    set_last_error(where, (int)e);
    return MMDIT_ERR_CUDA;
}

bool dtype_ok(mmdit_dtype dt) { return dt == MMDIT_F32 || dt == MMDIT_BF16; }

// Elements per 16-byte vector.
int vec_elems(mmdit_dtype dt) { return dt == MMDIT_BF16 ? 8 : 4; }

int elem_bytes(mmdit_dtype dt) { return dt == MMDIT_BF16 ? 2 : 4; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

}  // namespace

// Validates a RoPE grid for N tokens of head dim D and converts it.
int mmdit::check_grid(const mmdit_grid* grid, long long N, int D, mmdit_dtype dt, RopeGrid& g) {
    if (grid->T < 1 || grid->H < 1 || grid->W < 1) return MMDIT_ERR_SHAPE;
    if ((long long)grid->T * grid->H * grid->W != N) return MMDIT_ERR_SHAPE;
    int sum = 0;
    for (int a = 0; a < 3; ++a) {
        if (grid->split[a] < 0 || (grid->split[a] & 1)) return MMDIT_ERR_SHAPE;
        sum += grid->split[a];
        if (!std::isfinite(grid->pos_scale[a])) return MMDIT_ERR_ARG;
    }
    if (sum != D) return MMDIT_ERR_SHAPE;
    if (!(grid->rope_base > 0.f) || !std::isfinite(grid->rope_base)) return MMDIT_ERR_ARG;
    // every 16-byte vector of head dims must sit inside one axis chunk
    const int E = vec_elems(dt);
    if (grid->split[0] % E || (grid->split[0] + grid->split[1]) % E) return MMDIT_ERR_UNSUPPORTED;
    g.T = grid->T;
    g.H = grid->H;
    g.W = grid->W;
    for (int a = 0; a < 3; ++a) {
        g.pos_scale[a] = grid->pos_scale[a];
        g.split[a] = grid->split[a];
    }
    g.base = grid->rope_base;
    return MMDIT_OK;
}

namespace {

// Validates a window partition of the grid's T, H, W extents.
int check_window(const mmdit_grid* grid, const mmdit_window* win) {
    const int extent[3] = {grid->T, grid->H, grid->W};
    long long count = 1;
    for (int a = 0; a < 3; ++a) {
        if (extent[a] < 1) return MMDIT_ERR_SHAPE;
        if (win->parts[a] < 1 || win->parts[a] > extent[a]) return MMDIT_ERR_SHAPE;
        count *= win->parts[a];
    }
    return count <= kMaxWindows ? MMDIT_OK : MMDIT_ERR_UNSUPPORTED;
}

}  // namespace

extern "C" {

int mmdit_qk_norm_rope(const void* q_in, const void* k_in, void* q_out, void* k_out,
                       const float* q_scale, const float* k_scale, int B, int N, int H, int D,
                       const mmdit_grid* grid, float eps, mmdit_dtype dt, void* stream) {
    if (!dtype_ok(dt) || B < 0 || N < 0 || H < 0 || !(eps >= 0.f) || !std::isfinite(eps))
        return MMDIT_ERR_ARG;
    if (D != kHeadDim) return MMDIT_ERR_UNSUPPORTED;
    if ((long long)B * N * H == 0) return MMDIT_OK;
    if (!q_in || !k_in || !q_out || !k_out || !q_scale || !k_scale) return MMDIT_ERR_ARG;
    if (!aligned16(q_in) || !aligned16(k_in) || !aligned16(q_out) || !aligned16(k_out) ||
        !aligned16(q_scale) || !aligned16(k_scale))
        return MMDIT_ERR_ALIGN;
    if ((long long)B * N * H >= (1LL << 31)) return MMDIT_ERR_UNSUPPORTED;
    RopeGrid g{};
    if (grid) {
        const int r = check_grid(grid, N, D, dt, g);
        if (r != MMDIT_OK) return r;
    }
    return cuda_status(launch_qk_norm_rope(q_in, k_in, q_out, k_out, q_scale, k_scale, B, N, H,
                                           grid ? &g : nullptr, nullptr, nullptr, eps,
                                           dt == MMDIT_BF16, static_cast<cudaStream_t>(stream)),
                       "qk_norm_rope");
}

int mmdit_k_norm_rope(const void* k_in, void* k_out, const float* k_scale, int B, int N, int H,
                      int D, const mmdit_grid* grid, float eps, mmdit_dtype dt, void* stream) {
    if (!dtype_ok(dt) || B < 0 || N < 0 || H < 0 || !(eps >= 0.f) || !std::isfinite(eps))
        return MMDIT_ERR_ARG;
    if (D != kHeadDim) return MMDIT_ERR_UNSUPPORTED;
    if ((long long)B * N * H == 0) return MMDIT_OK;
    if (!k_in || !k_out || !k_scale) return MMDIT_ERR_ARG;
    if (!aligned16(k_in) || !aligned16(k_out) || !aligned16(k_scale)) return MMDIT_ERR_ALIGN;
    if ((long long)B * N * H >= (1LL << 31)) return MMDIT_ERR_UNSUPPORTED;
    RopeGrid g{};
    if (grid) {
        const int r = check_grid(grid, N, D, dt, g);
        if (r != MMDIT_OK) return r;
    }
    return cuda_status(launch_qk_norm_rope(nullptr, k_in, nullptr, k_out, k_scale, k_scale, B, N,
                                           H, grid ? &g : nullptr, nullptr, nullptr, eps,
                                           dt == MMDIT_BF16, static_cast<cudaStream_t>(stream)),
                       "k_norm_rope");
}

int mmdit_qk_norm_rope_bwd(const void* q_in, const void* k_in, const void* dq_out,
                           const void* dk_out, const float* q_scale, const float* k_scale,
                           void* dq_in, void* dk_in, float* dq_scale, float* dk_scale, int B,
                           int N, int H, int D, const mmdit_grid* grid, float eps, mmdit_dtype dt,
                           void* stream) {
    if (!dtype_ok(dt) || B < 0 || N < 0 || H < 0 || !(eps >= 0.f) || !std::isfinite(eps))
        return MMDIT_ERR_ARG;
    if (D != kHeadDim) return MMDIT_ERR_UNSUPPORTED;
    if (!dq_scale || !dk_scale) return MMDIT_ERR_ARG;
    if (!aligned16(dq_scale) || !aligned16(dk_scale)) return MMDIT_ERR_ALIGN;
    const bool empty = (long long)B * N * H == 0;
    if (!empty) {
        if (!q_in || !k_in || !dq_out || !dk_out || !q_scale || !k_scale || !dq_in || !dk_in)
            return MMDIT_ERR_ARG;
        if (!aligned16(q_in) || !aligned16(k_in) || !aligned16(dq_out) || !aligned16(dk_out) ||
            !aligned16(q_scale) || !aligned16(k_scale) || !aligned16(dq_in) || !aligned16(dk_in))
            return MMDIT_ERR_ALIGN;
        if ((long long)B * N * H >= (1LL << 31)) return MMDIT_ERR_UNSUPPORTED;
    }
    RopeGrid g{};
    if (grid) {
        const int r = check_grid(grid, N, D, dt, g);
        if (r != MMDIT_OK) return r;
    }
    return cuda_status(launch_qk_norm_rope_bwd(q_in, k_in, dq_out, dk_out, q_scale, k_scale, dq_in,
                                               dk_in, dq_scale, dk_scale, B, N, H,
                                               grid ? &g : nullptr, nullptr, eps,
                                               dt == MMDIT_BF16,
                                               static_cast<cudaStream_t>(stream)),
                       "qk_norm_rope_bwd");
}

int mmdit_qk_norm_rope_text_bwd(const void* q_in, const void* k_in, const void* dq_out,
                                const void* dk_out, const float* q_scale, const float* k_scale,
                                void* dq_in, void* dk_in, float* dq_scale, float* dk_scale, int B,
                                int N, int H, int D, const mmdit_text_rope* rope, float eps,
                                mmdit_dtype dt, void* stream) {
    if (!dtype_ok(dt) || B < 0 || N < 0 || H < 0 || !(eps >= 0.f) || !std::isfinite(eps) || !rope)
        return MMDIT_ERR_ARG;
    if (D != kHeadDim) return MMDIT_ERR_UNSUPPORTED;
    if (!dq_scale || !dk_scale) return MMDIT_ERR_ARG;
    if (!aligned16(dq_scale) || !aligned16(dk_scale)) return MMDIT_ERR_ALIGN;
    if (!std::isfinite(rope->pos_offset)) return MMDIT_ERR_ARG;
    if (!(rope->rope_base > 0.f) || !std::isfinite(rope->rope_base)) return MMDIT_ERR_ARG;
    int sum = 0;
    for (int a = 0; a < 3; ++a) {
        if (rope->split[a] < 0 || (rope->split[a] & 1)) return MMDIT_ERR_SHAPE;
        sum += rope->split[a];
    }
    if (sum != D) return MMDIT_ERR_SHAPE;
    const int E = vec_elems(dt);
    if (rope->split[0] % E || (rope->split[0] + rope->split[1]) % E) return MMDIT_ERR_UNSUPPORTED;
    if ((long long)B * N * H != 0) {
        if (!q_in || !k_in || !dq_out || !dk_out || !q_scale || !k_scale || !dq_in || !dk_in)
            return MMDIT_ERR_ARG;
        if (!aligned16(q_in) || !aligned16(k_in) || !aligned16(dq_out) || !aligned16(dk_out) ||
            !aligned16(q_scale) || !aligned16(k_scale) || !aligned16(dq_in) || !aligned16(dk_in))
            return MMDIT_ERR_ALIGN;
        if ((long long)B * N * H >= (1LL << 31)) return MMDIT_ERR_UNSUPPORTED;
    }
    RopeText t{};
    t.pos_offset = rope->pos_offset;
    t.base = rope->rope_base;
    for (int a = 0; a < 3; ++a) t.split[a] = rope->split[a];
    return cuda_status(launch_qk_norm_rope_bwd(q_in, k_in, dq_out, dk_out, q_scale, k_scale, dq_in,
                                               dk_in, dq_scale, dk_scale, B, N, H, nullptr, &t,
                                               eps, dt == MMDIT_BF16,
                                               static_cast<cudaStream_t>(stream)),
                       "qk_norm_rope_text_bwd");
}

int mmdit_qk_norm_rope_window(const void* q_in, const void* k_in, void* q_out, void* k_out,
                              const float* q_scale, const float* k_scale, int B, int N, int H,
                              int D, const mmdit_grid* grid, const mmdit_window* win, float eps,
                              mmdit_dtype dt, void* stream) {
    if (!dtype_ok(dt) || B < 0 || N < 0 || H < 0 || !(eps >= 0.f) || !std::isfinite(eps) ||
        !grid || !win)
        return MMDIT_ERR_ARG;
    if (D != kHeadDim) return MMDIT_ERR_UNSUPPORTED;
    RopeGrid g{};
    int r = check_grid(grid, N, D, dt, g);
    if (r != MMDIT_OK) return r;
    if ((r = check_window(grid, win)) != MMDIT_OK) return r;
    if ((long long)B * N * H == 0) return MMDIT_OK;
    if (!q_in || !k_in || !q_out || !k_out || !q_scale || !k_scale) return MMDIT_ERR_ARG;
    if (!aligned16(q_in) || !aligned16(k_in) || !aligned16(q_out) || !aligned16(k_out) ||
        !aligned16(q_scale) || !aligned16(k_scale))
        return MMDIT_ERR_ALIGN;
    if ((long long)B * N * H >= (1LL << 31)) return MMDIT_ERR_UNSUPPORTED;
    const size_t bytes = (size_t)B * N * H * D * elem_bytes(dt);
    if (overlap(q_out, bytes, q_in, bytes) || overlap(q_out, bytes, k_in, bytes) ||
        overlap(k_out, bytes, q_in, bytes) || overlap(k_out, bytes, k_in, bytes) ||
        overlap(q_out, bytes, k_out, bytes))
        return MMDIT_ERR_ARG;
    return cuda_status(launch_qk_norm_rope(q_in, k_in, q_out, k_out, q_scale, k_scale, B, N, H,
                                           &g, nullptr, win->parts, eps, dt == MMDIT_BF16,
                                           static_cast<cudaStream_t>(stream)),
                       "qk_norm_rope_window");
}

int mmdit_window_permute(const void* x, void* y, int B, int N, int C, const mmdit_grid* grid,
                         const mmdit_window* win, int inverse, mmdit_dtype dt, void* stream) {
    if (!dtype_ok(dt) || B < 0 || N < 0 || C < 0 || !grid || !win) return MMDIT_ERR_ARG;
    if (grid->T < 1 || grid->H < 1 || grid->W < 1) return MMDIT_ERR_SHAPE;
    if ((long long)grid->T * grid->H * grid->W != (long long)N) return MMDIT_ERR_SHAPE;
    int r = check_window(grid, win);
    if (r != MMDIT_OK) return r;
    const long long row_bytes = (long long)C * elem_bytes(dt);
    if (C == 0 || row_bytes % 16 != 0) return MMDIT_ERR_UNSUPPORTED;
    if ((long long)B * N == 0) return MMDIT_OK;
    if ((long long)B * N >= (1LL << 31) || row_bytes >= (1LL << 31)) return MMDIT_ERR_UNSUPPORTED;
    if (!x || !y) return MMDIT_ERR_ARG;
    if (!aligned16(x) || !aligned16(y)) return MMDIT_ERR_ALIGN;
    const size_t bytes = (size_t)B * N * row_bytes;
    if (overlap(x, bytes, y, bytes)) return MMDIT_ERR_ARG;
    RopeGrid g{};
    g.T = grid->T;
    g.H = grid->H;
    g.W = grid->W;
    return cuda_status(launch_window_permute(x, y, B, N, (int)row_bytes, g, win->parts,
                                             inverse != 0, static_cast<cudaStream_t>(stream)),
                       "window_permute");
}

int mmdit_qk_norm_rope_text(const void* q_in, const void* k_in, void* q_out, void* k_out,
                            const float* q_scale, const float* k_scale, int B, int N, int H, int D,
                            const mmdit_text_rope* rope, float eps, mmdit_dtype dt, void* stream) {
    if (!dtype_ok(dt) || B < 0 || N < 0 || H < 0 || !(eps >= 0.f) || !std::isfinite(eps) || !rope)
        return MMDIT_ERR_ARG;
    if (D != kHeadDim) return MMDIT_ERR_UNSUPPORTED;
    if ((long long)B * N * H == 0) return MMDIT_OK;
    if (!q_in || !k_in || !q_out || !k_out || !q_scale || !k_scale) return MMDIT_ERR_ARG;
    if (!aligned16(q_in) || !aligned16(k_in) || !aligned16(q_out) || !aligned16(k_out) ||
        !aligned16(q_scale) || !aligned16(k_scale))
        return MMDIT_ERR_ALIGN;
    if ((long long)B * N * H >= (1LL << 31)) return MMDIT_ERR_UNSUPPORTED;
    if (!std::isfinite(rope->pos_offset)) return MMDIT_ERR_ARG;
    if (!(rope->rope_base > 0.f) || !std::isfinite(rope->rope_base)) return MMDIT_ERR_ARG;
    int sum = 0;
    for (int a = 0; a < 3; ++a) {
        if (rope->split[a] < 0 || (rope->split[a] & 1)) return MMDIT_ERR_SHAPE;
        sum += rope->split[a];
    }
    if (sum != D) return MMDIT_ERR_SHAPE;
    const int E = vec_elems(dt);
    if (rope->split[0] % E || (rope->split[0] + rope->split[1]) % E) return MMDIT_ERR_UNSUPPORTED;
    RopeText t{};
    t.pos_offset = rope->pos_offset;
    t.base = rope->rope_base;
    for (int a = 0; a < 3; ++a) t.split[a] = rope->split[a];
    return cuda_status(launch_qk_norm_rope(q_in, k_in, q_out, k_out, q_scale, k_scale, B, N, H,
                                           nullptr, &t, nullptr, eps, dt == MMDIT_BF16,
                                           static_cast<cudaStream_t>(stream)),
                       "qk_norm_rope_text");
}

}  // extern "C"

namespace {

int joint_attention_impl(const void* q_vis, const void* k_vis, const void* v_vis,
                         const void* q_ctx, const void* k_ctx, const void* v_ctx,
                         const int32_t* ctx_len, void* o_vis, void* o_ctx, float* lse, int B,
                         int Nv, int Nc, int H, int D, float softmax_scale, const WindowTable* win,
                         mmdit_dtype dt, void* stream, void* ws = nullptr,
                         long long ws_bytes = 0) {
    if (!dtype_ok(dt) || B < 0 || Nv < 0 || Nc < 0 || H < 0) return MMDIT_ERR_ARG;
    if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale)) return MMDIT_ERR_ARG;
    if (D != kHeadDim) return MMDIT_ERR_UNSUPPORTED;
    if ((long long)B * H * (Nv + (long long)Nc) == 0) return MMDIT_OK;
    if (B > 65535 || H > 65535) return MMDIT_ERR_UNSUPPORTED;
    if (Nv > 0) {
        if (!q_vis || !k_vis || !v_vis || !o_vis) return MMDIT_ERR_ARG;
        if (!aligned16(q_vis) || !aligned16(k_vis) || !aligned16(v_vis) || !aligned16(o_vis))
            return MMDIT_ERR_ALIGN;
    }
    if (Nc > 0) {
        if (!q_ctx || !k_ctx || !v_ctx || !o_ctx) return MMDIT_ERR_ARG;
        if (!aligned16(q_ctx) || !aligned16(k_ctx) || !aligned16(v_ctx) || !aligned16(o_ctx))
            return MMDIT_ERR_ALIGN;
    }
    if (ctx_len && (reinterpret_cast<uintptr_t>(ctx_len) & 3u)) return MMDIT_ERR_ALIGN;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return MMDIT_ERR_ALIGN;
    if ((long long)Nv + Nc > (1LL << 30)) return MMDIT_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dt == MMDIT_F32)
        return cuda_status(launch_joint_attention_f32(
            static_cast<const float*>(q_vis), static_cast<const float*>(k_vis),
            static_cast<const float*>(v_vis), static_cast<const float*>(q_ctx),
            static_cast<const float*>(k_ctx), static_cast<const float*>(v_ctx), ctx_len,
            static_cast<float*>(o_vis), static_cast<float*>(o_ctx), lse, B, Nv, Nc, H,
            softmax_scale, win, s), "joint_attention_f32");
    const int r = launch_joint_attention_bf16(q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, ctx_len,
                                              o_vis, o_ctx, lse, B, Nv, Nc, H, softmax_scale, win,
                                              s, nullptr, static_cast<float*>(ws), ws_bytes);
    if (r == 0) return MMDIT_OK;
    set_last_error("joint_attention_bf16", r);
    return MMDIT_ERR_CUDA;
}

// The attention backward of both entry points (win: null, or the 3D window
// partition of the window-major visual inputs).
int joint_attention_bwd_impl(const void* q_vis, const void* k_vis, const void* v_vis,
                             const void* q_ctx, const void* k_ctx, const void* v_ctx,
                             const int32_t* ctx_len, const void* o_vis, const void* o_ctx,
                             const void* do_vis, const void* do_ctx, const float* lse,
                             float* delta, void* dq_vis, void* dk_vis, void* dv_vis,
                             void* dq_ctx, void* dk_ctx, void* dv_ctx, int B, int Nv, int Nc,
                             int H, int D, float softmax_scale, mmdit_dtype dt, void* stream,
                             const WindowTable* win, void* workspace = nullptr,
                             long long workspace_bytes = 0) {
    if (workspace_bytes < 0) return MMDIT_ERR_ARG;
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return MMDIT_ERR_ALIGN;
    if (!dtype_ok(dt) || B < 0 || Nv < 0 || Nc < 0 || H < 0) return MMDIT_ERR_ARG;
    if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale)) return MMDIT_ERR_ARG;
    if (D != kHeadDim) return MMDIT_ERR_UNSUPPORTED;
    if ((long long)B * H * (Nv + (long long)Nc) == 0) return MMDIT_OK;
    if (B > 65535 || H > 65535) return MMDIT_ERR_UNSUPPORTED;
    if ((long long)B * H * (Nv + (long long)Nc) >= (1LL << 31)) return MMDIT_ERR_UNSUPPORTED;
    const void* vis[] = {q_vis, k_vis, v_vis, o_vis, do_vis, dq_vis, dk_vis, dv_vis};
    const void* ctx[] = {q_ctx, k_ctx, v_ctx, o_ctx, do_ctx, dq_ctx, dk_ctx, dv_ctx};
    for (int i = 0; i < 8; ++i) {
        if (Nv > 0 && !vis[i]) return MMDIT_ERR_ARG;
        if (Nc > 0 && !ctx[i]) return MMDIT_ERR_ARG;
        if (Nv > 0 && !aligned16(vis[i])) return MMDIT_ERR_ALIGN;
        if (Nc > 0 && !aligned16(ctx[i])) return MMDIT_ERR_ALIGN;
    }
    if (!lse || !delta) return MMDIT_ERR_ARG;
    if ((reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(delta) & 3u) ||
        (ctx_len && (reinterpret_cast<uintptr_t>(ctx_len) & 3u)))
        return MMDIT_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dt == MMDIT_F32)
        return cuda_status(
            launch_joint_attention_bwd_f32(
                static_cast<const float*>(q_vis), static_cast<const float*>(k_vis),
                static_cast<const float*>(v_vis), static_cast<const float*>(q_ctx),
                static_cast<const float*>(k_ctx), static_cast<const float*>(v_ctx), ctx_len,
                static_cast<const float*>(o_vis), static_cast<const float*>(o_ctx),
                static_cast<const float*>(do_vis), static_cast<const float*>(do_ctx), lse, delta,
                static_cast<float*>(dq_vis), static_cast<float*>(dk_vis),
                static_cast<float*>(dv_vis), static_cast<float*>(dq_ctx),
                static_cast<float*>(dk_ctx), static_cast<float*>(dv_ctx), B, Nv, Nc, H,
                softmax_scale, s, win),
            "joint_attention_bwd_f32");
    // the one-pass form when the workspace holds the fp32 dQ accumulator
    const bool one_pass =
        workspace && workspace_bytes >= MMDIT_BWD_WORKSPACE_BYTES(B, Nv, Nc, H);
    const int r = launch_joint_attention_bwd_bf16(
        q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, ctx_len, o_vis, o_ctx, do_vis, do_ctx, lse, delta,
        dq_vis, dk_vis, dv_vis, dq_ctx, dk_ctx, dv_ctx, B, Nv, Nc, H, softmax_scale, s, win,
        one_pass ? static_cast<float*>(workspace) : nullptr);
    if (r == 0) return MMDIT_OK;
    set_last_error("joint_attention_bwd_bf16", r);
    return MMDIT_ERR_CUDA;
}

}  // namespace

extern "C" {

int mmdit_joint_attention(const void* q_vis, const void* k_vis, const void* v_vis,
                          const void* q_ctx, const void* k_ctx, const void* v_ctx,
                          const int32_t* ctx_len, void* o_vis, void* o_ctx, int B, int Nv, int Nc,
                          int H, int D, float softmax_scale, mmdit_dtype dt, void* stream) {
    return joint_attention_impl(q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, ctx_len, o_vis, o_ctx,
                                nullptr, B, Nv, Nc, H, D, softmax_scale, nullptr, dt, stream);
}

namespace {

int joint_attention_qnorm_impl(const void* q_vis, const void* k_vis, const void* v_vis,
                               const void* q_ctx, const void* k_ctx, const void* v_ctx,
                               const int32_t* ctx_len, void* o_vis, void* o_ctx,
                               const float* q_scale_vis, const float* q_scale_ctx,
                               const mmdit_grid* grid, float eps, int B, int Nv, int Nc, int H,
                               int D, float softmax_scale, mmdit_dtype dt, void* stream,
                               void* workspace, long long workspace_bytes) {
    if (workspace_bytes < 0) return MMDIT_ERR_ARG;
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return MMDIT_ERR_ALIGN;
    if (!dtype_ok(dt) || B < 0 || Nv < 0 || Nc < 0 || H < 0) return MMDIT_ERR_ARG;
    if (!(eps >= 0.f) || !std::isfinite(eps)) return MMDIT_ERR_ARG;
    if (dt != MMDIT_BF16) return MMDIT_ERR_UNSUPPORTED;
    if ((Nv > 0 && !q_scale_vis) || (Nc > 0 && !q_scale_ctx)) return MMDIT_ERR_ARG;
    if ((q_scale_vis && !aligned16(q_scale_vis)) || (q_scale_ctx && !aligned16(q_scale_ctx)))
        return MMDIT_ERR_ALIGN;
    RopeGrid g{};
    if (grid) {
        const int r = check_grid(grid, Nv, D, dt, g);
        if (r != MMDIT_OK) return r;
    }
    const QNormArgs qn{{q_scale_vis, q_scale_ctx}, grid ? &g : nullptr, eps};
    // the remaining checks and the launch are those of the joint attention
    if (D != kHeadDim) return MMDIT_ERR_UNSUPPORTED;
    if ((long long)B * H * (Nv + (long long)Nc) == 0) return MMDIT_OK;
    if (B > 65535 || H > 65535) return MMDIT_ERR_UNSUPPORTED;
    if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale)) return MMDIT_ERR_ARG;
    if (Nv > 0) {
        if (!q_vis || !k_vis || !v_vis || !o_vis) return MMDIT_ERR_ARG;
        if (!aligned16(q_vis) || !aligned16(k_vis) || !aligned16(v_vis) || !aligned16(o_vis))
            return MMDIT_ERR_ALIGN;
    }
    if (Nc > 0) {
        if (!q_ctx || !k_ctx || !v_ctx || !o_ctx) return MMDIT_ERR_ARG;
        if (!aligned16(q_ctx) || !aligned16(k_ctx) || !aligned16(v_ctx) || !aligned16(o_ctx))
            return MMDIT_ERR_ALIGN;
    }
    if (ctx_len && (reinterpret_cast<uintptr_t>(ctx_len) & 3u)) return MMDIT_ERR_ALIGN;
    if ((long long)Nv + Nc > (1LL << 30)) return MMDIT_ERR_UNSUPPORTED;
    const int r = launch_joint_attention_bf16(
        q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, ctx_len, o_vis, o_ctx, nullptr, B, Nv, Nc, H,
        softmax_scale, nullptr, static_cast<cudaStream_t>(stream), &qn,
        static_cast<float*>(workspace), workspace ? workspace_bytes : 0);
    if (r == 0) return MMDIT_OK;
    set_last_error("joint_attention_qnorm", r);
    return MMDIT_ERR_CUDA;
}

}  // namespace

int mmdit_joint_attention_qnorm(const void* q_vis, const void* k_vis, const void* v_vis,
                                const void* q_ctx, const void* k_ctx, const void* v_ctx,
                                const int32_t* ctx_len, void* o_vis, void* o_ctx,
                                const float* q_scale_vis, const float* q_scale_ctx,
                                const mmdit_grid* grid, float eps, int B, int Nv, int Nc, int H,
                                int D, float softmax_scale, mmdit_dtype dt, void* stream) {
    return joint_attention_qnorm_impl(q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, ctx_len, o_vis,
                                      o_ctx, q_scale_vis, q_scale_ctx, grid, eps, B, Nv, Nc, H, D,
                                      softmax_scale, dt, stream, nullptr, 0);
}

int mmdit_joint_attention_qnorm_ws(const void* q_vis, const void* k_vis, const void* v_vis,
                                   const void* q_ctx, const void* k_ctx, const void* v_ctx,
                                   const int32_t* ctx_len, void* o_vis, void* o_ctx,
                                   const float* q_scale_vis, const float* q_scale_ctx,
                                   const mmdit_grid* grid, float eps, void* workspace,
                                   long long workspace_bytes, int B, int Nv, int Nc, int H, int D,
                                   float softmax_scale, mmdit_dtype dt, void* stream) {
    return joint_attention_qnorm_impl(q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, ctx_len, o_vis,
                                      o_ctx, q_scale_vis, q_scale_ctx, grid, eps, B, Nv, Nc, H, D,
                                      softmax_scale, dt, stream, workspace, workspace_bytes);
}

int mmdit_quantize_int8(const void* x, void* codes, float* scales, int B, int N, int H, int D,
                        int block, void* stream) {
    if (B < 0 || N < 0 || H < 0) return MMDIT_ERR_ARG;
    if (D != kHeadDim || (block != 1 && block != 128)) return MMDIT_ERR_UNSUPPORTED;
    if ((long long)B * N * H == 0) return MMDIT_OK;
    if (!x || !codes || !scales) return MMDIT_ERR_ARG;
    if (!aligned16(x) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 3u))
        return MMDIT_ERR_ALIGN;
    if ((long long)B * N * H >= (1LL << 31) || B > 65535 || H > 65535) return MMDIT_ERR_UNSUPPORTED;
    return cuda_status(launch_quant_int8(x, codes, scales, B, N, H, block,
                                         static_cast<cudaStream_t>(stream)),
                       "quantize_int8");
}

int mmdit_quantize_v_e4m3(const void* v_vis, const void* v_ctx, const int32_t* ctx_len,
                          void* c_vis, void* c_ctx, float* scales, int B, int Nv, int Nc, int H,
                          int D, void* stream) {
    if (B < 0 || Nv < 0 || Nc < 0 || H < 0) return MMDIT_ERR_ARG;
    if (D != kHeadDim) return MMDIT_ERR_UNSUPPORTED;
    if ((long long)B * H == 0) return MMDIT_OK;
    if (!scales) return MMDIT_ERR_ARG;
    if (!aligned16(scales)) return MMDIT_ERR_ALIGN;
    if (Nv > 0 && (!v_vis || !c_vis)) return MMDIT_ERR_ARG;
    if (Nc > 0 && (!v_ctx || !c_ctx)) return MMDIT_ERR_ARG;
    if ((Nv > 0 && (!aligned16(v_vis) || !aligned16(c_vis))) ||
        (Nc > 0 && (!aligned16(v_ctx) || !aligned16(c_ctx))) ||
        (ctx_len && (reinterpret_cast<uintptr_t>(ctx_len) & 3u)))
        return MMDIT_ERR_ALIGN;
    if ((long long)B * (Nv + (long long)Nc) * H >= (1LL << 31) || B > 65535 || H > 65535)
        return MMDIT_ERR_UNSUPPORTED;
    return cuda_status(launch_quant_v_e4m3(v_vis, v_ctx, ctx_len, c_vis, c_ctx, scales, B, Nv, Nc,
                                           H, static_cast<cudaStream_t>(stream)),
                       "quantize_v_e4m3");
}

int mmdit_joint_attention_q8(const void* q_vis, const void* k_vis, const void* v_vis,
                             const void* q_ctx, const void* k_ctx, const void* v_ctx,
                             const float* sq_vis, const float* sq_ctx, const float* sk_vis,
                             const float* sk_ctx, const float* sv, const int32_t* ctx_len,
                             void* o_vis, void* o_ctx, int B, int Nv, int Nc, int H, int D,
                             float softmax_scale, void* stream) {
    if (B < 0 || Nv < 0 || Nc < 0 || H < 0) return MMDIT_ERR_ARG;
    if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale)) return MMDIT_ERR_ARG;
    if (D != kHeadDim) return MMDIT_ERR_UNSUPPORTED;
    if ((long long)B * H * (Nv + (long long)Nc) == 0) return MMDIT_OK;
    if (B > 65535 || H > 65535 || (long long)Nv + Nc > (1LL << 30)) return MMDIT_ERR_UNSUPPORTED;
    if (!sv) return MMDIT_ERR_ARG;
    if (Nv > 0) {
        if (!q_vis || !k_vis || !v_vis || !o_vis || !sq_vis || !sk_vis) return MMDIT_ERR_ARG;
        if (!aligned16(q_vis) || !aligned16(k_vis) || !aligned16(v_vis) || !aligned16(o_vis))
            return MMDIT_ERR_ALIGN;
    }
    if (Nc > 0) {
        if (!q_ctx || !k_ctx || !v_ctx || !o_ctx || !sq_ctx || !sk_ctx) return MMDIT_ERR_ARG;
        if (!aligned16(q_ctx) || !aligned16(k_ctx) || !aligned16(v_ctx) || !aligned16(o_ctx))
            return MMDIT_ERR_ALIGN;
    }
    for (const void* f : {(const void*)sq_vis, (const void*)sq_ctx, (const void*)sk_vis,
                          (const void*)sk_ctx, (const void*)sv, (const void*)ctx_len})
        if (f && (reinterpret_cast<uintptr_t>(f) & 3u)) return MMDIT_ERR_ALIGN;
    const int r = launch_joint_attention_q8(q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, sq_vis, sq_ctx,
                                            sk_vis, sk_ctx, sv, ctx_len, o_vis, o_ctx, B, Nv, Nc,
                                            H, softmax_scale, static_cast<cudaStream_t>(stream));
    if (r == 0) return MMDIT_OK;
    set_last_error("joint_attention_q8", r);
    return MMDIT_ERR_CUDA;
}

int mmdit_joint_attention_fwd(const void* q_vis, const void* k_vis, const void* v_vis,
                              const void* q_ctx, const void* k_ctx, const void* v_ctx,
                              const int32_t* ctx_len, void* o_vis, void* o_ctx, float* lse, int B,
                              int Nv, int Nc, int H, int D, float softmax_scale, mmdit_dtype dt,
                              void* stream) {
    if (!lse && (long long)B * H * (Nv + (long long)Nc) > 0) return MMDIT_ERR_ARG;
    return joint_attention_impl(q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, ctx_len, o_vis, o_ctx,
                                lse, B, Nv, Nc, H, D, softmax_scale, nullptr, dt, stream);
}

int mmdit_joint_attention_ws(const void* q_vis, const void* k_vis, const void* v_vis,
                             const void* q_ctx, const void* k_ctx, const void* v_ctx,
                             const int32_t* ctx_len, void* o_vis, void* o_ctx, float* lse,
                             void* workspace, long long workspace_bytes, int B, int Nv, int Nc,
                             int H, int D, float softmax_scale, mmdit_dtype dt, void* stream) {
    if (workspace_bytes < 0) return MMDIT_ERR_ARG;
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return MMDIT_ERR_ALIGN;
    return joint_attention_impl(q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, ctx_len, o_vis, o_ctx,
                                lse, B, Nv, Nc, H, D, softmax_scale, nullptr, dt, stream,
                                workspace, workspace ? workspace_bytes : 0);
}

int mmdit_joint_attention_split_plan(int B, int Nv, int Nc, int H, int num_sms,
                                     long long workspace_bytes, long long* plan) {
    if (B < 0 || Nv < 0 || Nc < 0 || H < 0 || num_sms < 1 || workspace_bytes < 0 || !plan)
        return MMDIT_ERR_ARG;
    const SplitPlan sp = split_plan(B, Nv, Nc, H, num_sms, workspace_bytes);
    plan[0] = sp.tail;
    plan[1] = sp.parts;
    plan[2] = sp.per;
    plan[3] = sp.ctas;
    return MMDIT_OK;
}

int mmdit_joint_attention_bwd(const void* q_vis, const void* k_vis, const void* v_vis,
                              const void* q_ctx, const void* k_ctx, const void* v_ctx,
                              const int32_t* ctx_len, const void* o_vis, const void* o_ctx,
                              const void* do_vis, const void* do_ctx, const float* lse,
                              float* delta, void* dq_vis, void* dk_vis, void* dv_vis,
                              void* dq_ctx, void* dk_ctx, void* dv_ctx, int B, int Nv, int Nc,
                              int H, int D, float softmax_scale, mmdit_dtype dt, void* stream) {
    return joint_attention_bwd_impl(q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, ctx_len, o_vis,
                                    o_ctx, do_vis, do_ctx, lse, delta, dq_vis, dk_vis, dv_vis,
                                    dq_ctx, dk_ctx, dv_ctx, B, Nv, Nc, H, D, softmax_scale, dt,
                                    stream, nullptr);
}

int mmdit_joint_attention_bwd_ws(const void* q_vis, const void* k_vis, const void* v_vis,
                                 const void* q_ctx, const void* k_ctx, const void* v_ctx,
                                 const int32_t* ctx_len, const void* o_vis, const void* o_ctx,
                                 const void* do_vis, const void* do_ctx, const float* lse,
                                 float* delta, void* workspace, long long workspace_bytes,
                                 void* dq_vis, void* dk_vis, void* dv_vis, void* dq_ctx,
                                 void* dk_ctx, void* dv_ctx, int B, int Nv, int Nc, int H, int D,
                                 float softmax_scale, mmdit_dtype dt, void* stream) {
    return joint_attention_bwd_impl(q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, ctx_len, o_vis,
                                    o_ctx, do_vis, do_ctx, lse, delta, dq_vis, dk_vis, dv_vis,
                                    dq_ctx, dk_ctx, dv_ctx, B, Nv, Nc, H, D, softmax_scale, dt,
                                    stream, nullptr, workspace, workspace_bytes);
}

int mmdit_joint_window_attention(const void* q_vis, const void* k_vis, const void* v_vis,
                                 const void* q_ctx, const void* k_ctx, const void* v_ctx,
                                 const int32_t* ctx_len, void* o_vis, void* o_ctx, int B, int Nv,
                                 int Nc, int H, int D, const mmdit_grid* grid,
                                 const mmdit_window* win, float softmax_scale, mmdit_dtype dt,
                                 void* stream) {
    if (!grid || !win || Nv < 0) return MMDIT_ERR_ARG;
    if (grid->T < 1 || grid->H < 1 || grid->W < 1) return MMDIT_ERR_SHAPE;
    if ((long long)grid->T * grid->H * grid->W != (long long)Nv) return MMDIT_ERR_SHAPE;
    const int r = check_window(grid, win);
    if (r != MMDIT_OK) return r;
    const WindowTable tab = make_window_table(grid->T, grid->H, grid->W, win->parts);
    return joint_attention_impl(q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, ctx_len, o_vis, o_ctx,
                                nullptr, B, Nv, Nc, H, D, softmax_scale, &tab, dt, stream);
}

int mmdit_joint_window_attention_fwd(const void* q_vis, const void* k_vis, const void* v_vis,
                                     const void* q_ctx, const void* k_ctx, const void* v_ctx,
                                     const int32_t* ctx_len, void* o_vis, void* o_ctx, float* lse,
                                     int B, int Nv, int Nc, int H, int D,
                                     const mmdit_grid* grid, const mmdit_window* win,
                                     float softmax_scale, mmdit_dtype dt, void* stream) {
    if (!grid || !win || !lse || Nv < 0) return MMDIT_ERR_ARG;
    if (grid->T < 1 || grid->H < 1 || grid->W < 1) return MMDIT_ERR_SHAPE;
    if ((long long)grid->T * grid->H * grid->W != (long long)Nv) return MMDIT_ERR_SHAPE;
    const int r = check_window(grid, win);
    if (r != MMDIT_OK) return r;
    const WindowTable tab = make_window_table(grid->T, grid->H, grid->W, win->parts);
    return joint_attention_impl(q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, ctx_len, o_vis, o_ctx,
                                lse, B, Nv, Nc, H, D, softmax_scale, &tab, dt, stream);
}

int mmdit_joint_window_attention_bwd(const void* q_vis, const void* k_vis, const void* v_vis,
                                     const void* q_ctx, const void* k_ctx, const void* v_ctx,
                                     const int32_t* ctx_len, const void* o_vis,
                                     const void* o_ctx, const void* do_vis, const void* do_ctx,
                                     const float* lse, float* delta, void* dq_vis, void* dk_vis,
                                     void* dv_vis, void* dq_ctx, void* dk_ctx, void* dv_ctx,
                                     int B, int Nv, int Nc, int H, int D, const mmdit_grid* grid,
                                     const mmdit_window* win, float softmax_scale, mmdit_dtype dt,
                                     void* stream) {
    if (!grid || !win || Nv < 0) return MMDIT_ERR_ARG;
    if (grid->T < 1 || grid->H < 1 || grid->W < 1) return MMDIT_ERR_SHAPE;
    if ((long long)grid->T * grid->H * grid->W != (long long)Nv) return MMDIT_ERR_SHAPE;
    const int r = check_window(grid, win);
    if (r != MMDIT_OK) return r;
    const WindowTable tab = make_window_table(grid->T, grid->H, grid->W, win->parts);
    return joint_attention_bwd_impl(q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, ctx_len, o_vis,
                                    o_ctx, do_vis, do_ctx, lse, delta, dq_vis, dk_vis, dv_vis,
                                    dq_ctx, dk_ctx, dv_ctx, B, Nv, Nc, H, D, softmax_scale, dt,
                                    stream, &tab);
}

int mmdit_joint_window_attention_bwd_ws(
    const void* q_vis, const void* k_vis, const void* v_vis, const void* q_ctx, const void* k_ctx,
    const void* v_ctx, const int32_t* ctx_len, const void* o_vis, const void* o_ctx,
    const void* do_vis, const void* do_ctx, const float* lse, float* delta, void* workspace,
    long long workspace_bytes, void* dq_vis, void* dk_vis, void* dv_vis, void* dq_ctx,
    void* dk_ctx, void* dv_ctx, int B, int Nv, int Nc, int H, int D, const mmdit_grid* grid,
    const mmdit_window* win, float softmax_scale, mmdit_dtype dt, void* stream) {
    if (!grid || !win || Nv < 0) return MMDIT_ERR_ARG;
    if (grid->T < 1 || grid->H < 1 || grid->W < 1) return MMDIT_ERR_SHAPE;
    if ((long long)grid->T * grid->H * grid->W != (long long)Nv) return MMDIT_ERR_SHAPE;
    const int r = check_window(grid, win);
    if (r != MMDIT_OK) return r;
    const WindowTable tab = make_window_table(grid->T, grid->H, grid->W, win->parts);
    return joint_attention_bwd_impl(q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, ctx_len, o_vis,
                                    o_ctx, do_vis, do_ctx, lse, delta, dq_vis, dk_vis, dv_vis,
                                    dq_ctx, dk_ctx, dv_ctx, B, Nv, Nc, H, D, softmax_scale, dt,
                                    stream, &tab, workspace, workspace_bytes);
}

int mmdit_adaln_modulate(const void* x, const float* shift, const float* scale, void* y, int B,
                         int N, int C, float eps, mmdit_dtype dt, void* stream) {
    if (!dtype_ok(dt) || B < 0 || N < 0 || C < 0 || !(eps >= 0.f) || !std::isfinite(eps))
        return MMDIT_ERR_ARG;
    const int E = vec_elems(dt);
    if (C == 0 || C % 8 != 0 || C / E > 512) return MMDIT_ERR_UNSUPPORTED;
    if ((long long)B * N == 0) return MMDIT_OK;
    if (B > 65535) return MMDIT_ERR_UNSUPPORTED;
    if (!x || !shift || !scale || !y) return MMDIT_ERR_ARG;
    if (!aligned16(x) || !aligned16(shift) || !aligned16(scale) || !aligned16(y))
        return MMDIT_ERR_ALIGN;
    return cuda_status(launch_adaln_modulate(x, shift, scale, y, B, N, C, eps, dt == MMDIT_BF16,
                                             static_cast<cudaStream_t>(stream)),
                       "adaln_modulate");
}

int mmdit_adaln_modulate_pair(const void* x_vis, const float* shift_vis, const float* scale_vis,
                              void* y_vis, int N_vis, const void* x_ctx, const float* shift_ctx,
                              const float* scale_ctx, void* y_ctx, int N_ctx, int B, int C,
                              float eps, mmdit_dtype dt, void* stream) {
    if (!dtype_ok(dt) || B < 0 || N_vis < 0 || N_ctx < 0 || C < 0 || !(eps >= 0.f) ||
        !std::isfinite(eps))
        return MMDIT_ERR_ARG;
    const int E = vec_elems(dt);
    if (C == 0 || C % 8 != 0 || C / E > 512) return MMDIT_ERR_UNSUPPORTED;
    if (B > 65535) return MMDIT_ERR_UNSUPPORTED;
    ModStreamsHost h{};
    const void* xs[2] = {x_vis, x_ctx};
    void* ys[2] = {y_vis, y_ctx};
    const float* shifts[2] = {shift_vis, shift_ctx};
    const float* scales[2] = {scale_vis, scale_ctx};
    const int Ns[2] = {N_vis, N_ctx};
    for (int k = 0; k < 2; ++k) {
        if ((long long)B * Ns[k] == 0) continue;
        if (!xs[k] || !shifts[k] || !scales[k] || !ys[k]) return MMDIT_ERR_ARG;
        if (!aligned16(xs[k]) || !aligned16(shifts[k]) || !aligned16(scales[k]) ||
            !aligned16(ys[k]))
            return MMDIT_ERR_ALIGN;
        h.x[k] = xs[k];
        h.y[k] = ys[k];
        h.shift[k] = shifts[k];
        h.scale[k] = scales[k];
        h.N[k] = Ns[k];
    }
    // one launch holds at most 2^31 - 1 CTAs: far above B * (2 * #SMs)
    return cuda_status(launch_adaln_modulate_pair(h, B, C, eps, dt == MMDIT_BF16,
                                                  static_cast<cudaStream_t>(stream)),
                       "adaln_modulate_pair");
}

int mmdit_gated_residual(const void* x, const void* branch, const float* gate, void* out, int B,
                         int N, int C, mmdit_dtype dt, void* stream) {
    if (!dtype_ok(dt) || B < 0 || N < 0 || C < 0) return MMDIT_ERR_ARG;
    if (C == 0 || C % 8 != 0) return MMDIT_ERR_UNSUPPORTED;
    if ((long long)B * N == 0) return MMDIT_OK;
    if (!x || !branch || !gate || !out) return MMDIT_ERR_ARG;
    if (!aligned16(x) || !aligned16(branch) || !aligned16(gate) || !aligned16(out))
        return MMDIT_ERR_ALIGN;
    return cuda_status(launch_gated_residual(x, branch, gate, out, B, N, C, dt == MMDIT_BF16,
                                             static_cast<cudaStream_t>(stream)),
                       "gated_residual");
}

int mmdit_residual_modulate(const void* x, const void* branch, const float* gate,
                            const float* shift, const float* scale, void* x_out, void* y, int B,
                            int N, int C, float eps, mmdit_dtype dt, void* stream) {
    if (!dtype_ok(dt) || B < 0 || N < 0 || C < 0 || !(eps >= 0.f) || !std::isfinite(eps))
        return MMDIT_ERR_ARG;
    const int E = vec_elems(dt);
    if (C == 0 || C % 8 != 0 || C / E > 384) return MMDIT_ERR_UNSUPPORTED;
    if ((long long)B * N == 0) return MMDIT_OK;
    if (B > 65535) return MMDIT_ERR_UNSUPPORTED;
    if (!x || !branch || !gate || !shift || !scale || !x_out || !y) return MMDIT_ERR_ARG;
    if (y == x || y == branch || y == x_out) return MMDIT_ERR_ARG;
    if (!aligned16(x) || !aligned16(branch) || !aligned16(gate) || !aligned16(shift) ||
        !aligned16(scale) || !aligned16(x_out) || !aligned16(y))
        return MMDIT_ERR_ALIGN;
    return cuda_status(launch_residual_modulate(x, branch, gate, shift, scale, x_out, y, B, N, C,
                                                eps, dt == MMDIT_BF16,
                                                static_cast<cudaStream_t>(stream)),
                       "residual_modulate");
}

int mmdit_device_status(void* stream) {
    unsigned int w = 0, wb = 0;
    cudaError_t e = read_and_clear_device_status(&w, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_status(e, "device_status");
    if ((e = read_and_clear_bwd_status(&wb)) != cudaSuccess) return cuda_status(e, "device_status");
    unsigned int wq = 0, we = 0, wp = 0;
    if ((e = read_and_clear_q8_status(&wq)) != cudaSuccess) return cuda_status(e, "device_status");
    if ((e = read_and_clear_elem_status(&we)) != cudaSuccess) return cuda_status(e, "device_status");
    if ((e = read_and_clear_pair_status(&wp)) != cudaSuccess) return cuda_status(e, "device_status");
    return (w | wb | wq | we | wp) ? MMDIT_ERR_TIMEOUT : MMDIT_OK;
}

void mmdit_set_wait_timeout_ns(unsigned long long ns) { set_wait_timeout_ns(ns); }

const char* mmdit_last_error(void) { return g_last_error; }

const char* mmdit_status_string(int status) {
    switch (status) {
        case MMDIT_OK: return "ok";
        case MMDIT_ERR_ARG: return "invalid argument";
        case MMDIT_ERR_SHAPE: return "inconsistent shapes";
        case MMDIT_ERR_ALIGN: return "pointer not 16-byte aligned";
        case MMDIT_ERR_UNSUPPORTED: return "unsupported size or layout";
        case MMDIT_ERR_CUDA: return "CUDA error";
        case MMDIT_ERR_TIMEOUT: return "device-side wait timed out";
        default: return "unknown status";
    }
}

}  // extern "C"
