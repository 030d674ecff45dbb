// mmdit_joint_attention_bwd_noalloc: the attention backward without a
// caller-provided workspace.
//
// mmdit_joint_attention_bwd needs a float workspace of B * H * (Nv + Nc)
// entries for the row sums D_i = dO_i . O_i.  Some callers cannot hand one
// over: code that must not call cudaMalloc at that point (a host whose
// device memory is owned by another allocator, a plugin inside an engine that
// forbids allocation once it runs, code that would otherwise allocate while a
// stream is being captured).  This entry point takes the workspace from a
// fixed array that lives in the library itself, so the call allocates
// nothing.
//
// The array holds kNoAllocRows floats (16 MiB) on every GPU that loads the
// library, until the process exits; larger problems are rejected.  Every
// call on a device shares it, so calls whose kernels overlap on the GPU (on
// different streams, say) race on it; calls in one stream are ordered.  The
// kernels overwrite every entry they read before reading it, so nothing has
// to start at zero and a call leaves no state that matters to the next.
//
// Host code cannot use the array's name as a device address: the device
// address comes from cudaGetSymbolAddress, done once per device by the first
// call made with that device current.  That first call should therefore come
// before any stream capture.  The address is kept until the process exits: a
// device reset after the first call is not supported.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/mmdit.h"
#include "internal.h"

namespace mmdit {
namespace {

constexpr long long kNoAllocRows = MMDIT_NOALLOC_MAX_ROWS;

static __device__ __align__(256) float g_noalloc_delta[kNoAllocRows];

std::mutex g_setup_mutex;
float* g_scratch[64] = {nullptr};   // device address of g_noalloc_delta, per device

// 0 on success, else a cudaError_t value.
int scratch_for_current_device(float** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return (int)e;
    if (dev < 0 || dev >= 64) return (int)cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_delta);
        if (e != cudaSuccess) return (int)e;
        g_scratch[dev] = static_cast<float*>(p);
    }
    *out = g_scratch[dev];
    return 0;
}

}  // namespace
}  // namespace mmdit

extern "C" int mmdit_joint_attention_bwd_noalloc(
    const void* q_vis, const void* k_vis, const void* v_vis, const void* q_ctx, const void* k_ctx,
    const void* v_ctx, const int32_t* ctx_len, const void* o_vis, const void* o_ctx,
    const void* do_vis, const void* do_ctx, const float* lse, void* dq_vis, void* dk_vis,
    void* dv_vis, void* dq_ctx, void* dk_ctx, void* dv_ctx, int B, int Nv, int Nc, int H, int D,
    float softmax_scale, mmdit_dtype dt, void* stream) {
    if (B < 0 || Nv < 0 || Nc < 0 || H < 0) return MMDIT_ERR_ARG;
    const long long rows = (long long)B * H * ((long long)Nv + Nc);
    if (rows > mmdit::kNoAllocRows) return MMDIT_ERR_UNSUPPORTED;
    if (rows == 0) return MMDIT_OK;
    float* delta = nullptr;
    const int r = mmdit::scratch_for_current_device(&delta);
    if (r != 0) {
        mmdit::set_last_error("joint_attention_bwd_noalloc: workspace set-up", r);
        return MMDIT_ERR_CUDA;
    }
    return mmdit_joint_attention_bwd(q_vis, k_vis, v_vis, q_ctx, k_ctx, v_ctx, ctx_len, o_vis,
                                     o_ctx, do_vis, do_ctx, lse, delta, dq_vis, dk_vis, dv_vis,
                                     dq_ctx, dk_ctx, dv_ctx, B, Nv, Nc, H, D, softmax_scale, dt,
                                     stream);
}
