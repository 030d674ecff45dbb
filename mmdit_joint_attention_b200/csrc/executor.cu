// mmdit_block_forward_host: the block's path run step after step from host
// buffers, with the copies in, the kernels and the copies out of different
// steps overlapped on three streams.
//
// A step is six calls of the device entry points, in this order: adaLN
// modulate of both streams (one launch), QK-RMSNorm + RoPE of both streams (in place), the
// joint attention (with its split-tail workspace), and the gated residual of
// both streams (in place on x).  Every buffer a step touches on the device
// lives in its slot of the workspace:
//
//   per stream s in (vis, ctx), N_s tokens:  q, k, v, x, y, o   [B, N_s, C] dt
//   per stream:                              shift, scale, gate [B, C] fp32
//   ctx_len                                  [B] int32
//   attention workspace                      MMDIT_ATTENTION_WORKSPACE_BYTES
//
// each region starting on a 256-byte boundary.
//
// Ordering, for step i in slot k = i mod S (S slots):
//   in stream   waits free[k] (step i - S has copied its outputs out), copies
//               the inputs, records ready[k];
//   compute     waits ready[k], runs the kernels, recording y_done[k] after
//               the modulate, o_done[k] after the attention, x_done[k] at the
//               end;
//   out stream  waits each of those before copying that output, then records
//               free[k].
// The out stream copies x last, after waiting x_done[k], so free[k] also
// orders the next writer of the slot after this step's kernels.  Events are
// reused across the steps of a slot: a wait binds to the record that precedes
// it on the host, and every wait of step i is enqueued before step i + S
// records the same event again.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <initializer_list>

#include "../../include/mmdit.h"
#include "internal.h"

namespace mmdit {
namespace {

constexpr int kMaxSlots = 4;

struct SlotLayout {
    // byte offsets inside a slot
    long long q[2], k[2], v[2], x[2], y[2], o[2];
    long long shift[2], scale[2], gate[2];
    long long ctx_len;
    long long attn_ws;      // split-tail workspace of the attention
    long long bytes;        // slot size (a multiple of 256)
    long long tok_bytes[2]; // bytes of one [B, N_s, C] tensor
    long long vec_bytes;    // bytes of one [B, C] fp32 vector
};

long long round256(long long n) { return (n + 255) & ~255LL; }

bool aligned(const void* p, unsigned a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// MMDIT_OK and the layout, or the MMDIT_ERR_* code of an invalid configuration.
// Covers every check the six entry points make on sizes and constants, so
// that a step cannot fail validation half-way through the enqueue.
int check_config(const mmdit_block_config* c, SlotLayout& L) {
    if (!c) return MMDIT_ERR_ARG;
    if (c->dt != MMDIT_F32 && c->dt != MMDIT_BF16) return MMDIT_ERR_ARG;
    if (c->B < 0 || c->Nv < 0 || c->Nc < 0 || c->H < 0) return MMDIT_ERR_ARG;
    if (!(c->norm_eps >= 0.f) || !std::isfinite(c->norm_eps) || !(c->ln_eps >= 0.f) ||
        !std::isfinite(c->ln_eps))
        return MMDIT_ERR_ARG;
    if (!(c->softmax_scale > 0.f) || !std::isfinite(c->softmax_scale)) return MMDIT_ERR_ARG;
    if (c->D != kHeadDim) return MMDIT_ERR_UNSUPPORTED;
    if (c->B < 1 || c->H < 1 || c->Nv < 1) return MMDIT_ERR_SHAPE;
    RopeGrid g{};
    const int r = check_grid(&c->grid, c->Nv, c->D, c->dt, g);
    if (r != MMDIT_OK) return r;
    const int esz = c->dt == MMDIT_BF16 ? 2 : 4;
    const long long C = (long long)c->H * c->D;
    // adaLN modulate: one CTA row holds C elements, 512 16-byte vectors at most
    if (C * esz / 16 > 512) return MMDIT_ERR_UNSUPPORTED;
    if (c->B > 65535 || c->H > 65535) return MMDIT_ERR_UNSUPPORTED;
    if ((long long)c->B * ((long long)c->Nv + c->Nc) * c->H >= (1LL << 31))
        return MMDIT_ERR_UNSUPPORTED;
    if (!c->gq_vis || !c->gk_vis) return MMDIT_ERR_ARG;
    if (!aligned(c->gq_vis, 16) || !aligned(c->gk_vis, 16)) return MMDIT_ERR_ALIGN;
    if (c->Nc > 0) {
        if (!c->gq_ctx || !c->gk_ctx) return MMDIT_ERR_ARG;
        if (!aligned(c->gq_ctx, 16) || !aligned(c->gk_ctx, 16)) return MMDIT_ERR_ALIGN;
    }
    const int N[2] = {c->Nv, c->Nc};
    long long off = 0;
    L.vec_bytes = (long long)c->B * C * 4;
    for (int s = 0; s < 2; ++s) {
        L.tok_bytes[s] = (long long)c->B * N[s] * C * esz;
        long long* fields[6] = {&L.q[s], &L.k[s], &L.v[s], &L.x[s], &L.y[s], &L.o[s]};
        for (long long* f : fields) {
            *f = off;
            off += round256(L.tok_bytes[s]);
        }
        for (long long* f : {&L.shift[s], &L.scale[s], &L.gate[s]}) {
            *f = off;
            off += round256(L.vec_bytes);
        }
    }
    L.ctx_len = off;
    off += round256((long long)c->B * 4);
    L.attn_ws = off;
    off += round256(MMDIT_ATTENTION_WORKSPACE_BYTES);
    L.bytes = off;
    return MMDIT_OK;
}

int check_step(const mmdit_block_config* c, const mmdit_block_step* s) {
    if (!s->q_vis || !s->k_vis || !s->v_vis || !s->x_vis || !s->shift_vis || !s->scale_vis ||
        !s->gate_vis || !s->x_out_vis)
        return MMDIT_ERR_ARG;
    if (c->Nc > 0 && (!s->q_ctx || !s->k_ctx || !s->v_ctx || !s->x_ctx || !s->shift_ctx ||
                      !s->scale_ctx || !s->gate_ctx || !s->x_out_ctx))
        return MMDIT_ERR_ARG;
    return MMDIT_OK;
}

struct Handles {
    cudaStream_t in = nullptr, cmp = nullptr, out = nullptr;
    cudaEvent_t start = nullptr;
    cudaEvent_t ready[kMaxSlots] = {}, y_done[kMaxSlots] = {}, o_done[kMaxSlots] = {},
                x_done[kMaxSlots] = {}, free_[kMaxSlots] = {};
    cudaEvent_t end[3] = {};
};

cudaError_t create(Handles& h, int slots) {
    cudaError_t e;
    for (cudaStream_t* s : {&h.in, &h.cmp, &h.out})
        if ((e = cudaStreamCreateWithFlags(s, cudaStreamNonBlocking)) != cudaSuccess) return e;
    auto ev = [](cudaEvent_t* x) { return cudaEventCreateWithFlags(x, cudaEventDisableTiming); };
    if ((e = ev(&h.start)) != cudaSuccess) return e;
    for (int k = 0; k < slots; ++k)
        for (cudaEvent_t* x : {&h.ready[k], &h.y_done[k], &h.o_done[k], &h.x_done[k], &h.free_[k]})
            if ((e = ev(x)) != cudaSuccess) return e;
    for (cudaEvent_t& x : h.end)
        if ((e = ev(&x)) != cudaSuccess) return e;
    return cudaSuccess;
}

// Destroying a stream or an event with work still pending is allowed: the
// resources are released once that work completes.
void destroy(Handles& h) {
    for (cudaStream_t s : {h.in, h.cmp, h.out})
        if (s) cudaStreamDestroy(s);
    if (h.start) cudaEventDestroy(h.start);
    for (int k = 0; k < kMaxSlots; ++k)
        for (cudaEvent_t x : {h.ready[k], h.y_done[k], h.o_done[k], h.x_done[k], h.free_[k]})
            if (x) cudaEventDestroy(x);
    for (cudaEvent_t x : h.end)
        if (x) cudaEventDestroy(x);
}

}  // namespace
}  // namespace mmdit

using namespace mmdit;

extern "C" long long mmdit_block_slot_bytes(const mmdit_block_config* cfg) {
    SlotLayout L{};
    const int r = check_config(cfg, L);
    return r != MMDIT_OK ? (long long)r : L.bytes;
}

extern "C" int mmdit_block_forward_host(const mmdit_block_config* cfg,
                                        const mmdit_block_step* steps, int n_steps,
                                        void* workspace, long long workspace_bytes,
                                        void* stream) {
    SlotLayout L{};
    int r = check_config(cfg, L);
    if (r != MMDIT_OK) return r;
    if (n_steps < 0) return MMDIT_ERR_ARG;
    if (n_steps == 0) return MMDIT_OK;
    if (!steps || !workspace) return MMDIT_ERR_ARG;
    if (!aligned(workspace, 256)) return MMDIT_ERR_ALIGN;
    if (workspace_bytes < L.bytes) return MMDIT_ERR_ARG;
    for (int i = 0; i < n_steps; ++i)
        if ((r = check_step(cfg, &steps[i])) != MMDIT_OK) return r;
    long long slots = workspace_bytes / L.bytes;
    if (slots > kMaxSlots) slots = kMaxSlots;
    if (slots > n_steps) slots = n_steps;

    const mmdit_block_config& c = *cfg;
    const int B = c.B, H = c.H, D = c.D, C = H * D;
    const int N[2] = {c.Nv, c.Nc};
    const bool has_ctx = c.Nc > 0;
    const cudaMemcpyKind h2d = cudaMemcpyHostToDevice, d2h = cudaMemcpyDeviceToHost;
    cudaStream_t user = static_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);

    Handles h;
    cudaError_t e = create(h, (int)slots);
    const char* where = "block_forward_host: stream / event set-up";
    int status = MMDIT_OK;
    bool started = false;
    if (e == cudaSuccess) {
        where = "block_forward_host: enqueue";
        e = cudaEventRecord(h.start, user);
        for (cudaStream_t s : {h.in, h.cmp, h.out})
            if (e == cudaSuccess) e = cudaStreamWaitEvent(s, h.start, 0);
        started = e == cudaSuccess;
    }
    for (int i = 0; e == cudaSuccess && status == MMDIT_OK && i < n_steps; ++i) {
        const mmdit_block_step& st = steps[i];
        const int k = i % (int)slots;
        uint8_t* base = ws + (long long)k * L.bytes;
        auto dev = [&](long long off) { return static_cast<void*>(base + off); };
        auto devf = [&](long long off) { return reinterpret_cast<float*>(base + off); };
        const void* in_q[2] = {st.q_vis, st.q_ctx};
        const void* in_k[2] = {st.k_vis, st.k_ctx};
        const void* in_v[2] = {st.v_vis, st.v_ctx};
        const void* in_x[2] = {st.x_vis, st.x_ctx};
        const float* in_shift[2] = {st.shift_vis, st.shift_ctx};
        const float* in_scale[2] = {st.scale_vis, st.scale_ctx};
        const float* in_gate[2] = {st.gate_vis, st.gate_ctx};
        void* out_y[2] = {st.y_vis, st.y_ctx};
        void* out_o[2] = {st.o_vis, st.o_ctx};
        void* out_x[2] = {st.x_out_vis, st.x_out_ctx};

        // ---- copies in
        if (i >= slots) e = cudaStreamWaitEvent(h.in, h.free_[k], 0);
        for (int s = 0; s < 2 && e == cudaSuccess; ++s) {
            if (N[s] == 0) continue;
            const long long tb = L.tok_bytes[s], vb = L.vec_bytes;
            const struct { long long off; const void* src; long long n; } cp[7] = {
                {L.q[s], in_q[s], tb},          {L.k[s], in_k[s], tb},
                {L.v[s], in_v[s], tb},          {L.x[s], in_x[s], tb},
                {L.shift[s], in_shift[s], vb},  {L.scale[s], in_scale[s], vb},
                {L.gate[s], in_gate[s], vb}};
            for (int j = 0; j < 7 && e == cudaSuccess; ++j)
                e = cudaMemcpyAsync(dev(cp[j].off), cp[j].src, (size_t)cp[j].n, h2d, h.in);
        }
        if (e == cudaSuccess && st.ctx_len)
            e = cudaMemcpyAsync(dev(L.ctx_len), st.ctx_len, (size_t)B * 4, h2d, h.in);
        if (e == cudaSuccess) e = cudaEventRecord(h.ready[k], h.in);
        if (e != cudaSuccess) break;

        // ---- kernels
        if ((e = cudaStreamWaitEvent(h.cmp, h.ready[k], 0)) != cudaSuccess) break;
        void* cs = static_cast<void*>(h.cmp);
        status = mmdit_adaln_modulate_pair(
            dev(L.x[0]), devf(L.shift[0]), devf(L.scale[0]), dev(L.y[0]), N[0],
            has_ctx ? dev(L.x[1]) : nullptr, has_ctx ? devf(L.shift[1]) : nullptr,
            has_ctx ? devf(L.scale[1]) : nullptr, has_ctx ? dev(L.y[1]) : nullptr, N[1], B, C,
            c.ln_eps, c.dt, cs);
        if (status != MMDIT_OK) break;
        if ((e = cudaEventRecord(h.y_done[k], h.cmp)) != cudaSuccess) break;
        status = mmdit_qk_norm_rope(dev(L.q[0]), dev(L.k[0]), dev(L.q[0]), dev(L.k[0]), c.gq_vis,
                                    c.gk_vis, B, N[0], H, D, &c.grid, c.norm_eps, c.dt, cs);
        if (status == MMDIT_OK && has_ctx)
            status = mmdit_qk_norm_rope(dev(L.q[1]), dev(L.k[1]), dev(L.q[1]), dev(L.k[1]),
                                        c.gq_ctx, c.gk_ctx, B, N[1], H, D, nullptr, c.norm_eps,
                                        c.dt, cs);
        if (status == MMDIT_OK)
            status = mmdit_joint_attention_ws(
                dev(L.q[0]), dev(L.k[0]), dev(L.v[0]), has_ctx ? dev(L.q[1]) : nullptr,
                has_ctx ? dev(L.k[1]) : nullptr, has_ctx ? dev(L.v[1]) : nullptr,
                st.ctx_len ? reinterpret_cast<const int32_t*>(dev(L.ctx_len)) : nullptr,
                dev(L.o[0]), has_ctx ? dev(L.o[1]) : nullptr, nullptr, dev(L.attn_ws),
                MMDIT_ATTENTION_WORKSPACE_BYTES, B, N[0], N[1], H, D, c.softmax_scale, c.dt, cs);
        if (status != MMDIT_OK) break;
        if ((e = cudaEventRecord(h.o_done[k], h.cmp)) != cudaSuccess) break;
        for (int s = 0; s < 2 && status == MMDIT_OK; ++s)
            if (N[s] > 0)
                status = mmdit_gated_residual(dev(L.x[s]), dev(L.o[s]), devf(L.gate[s]),
                                              dev(L.x[s]), B, N[s], C, c.dt, cs);
        if (status != MMDIT_OK) break;
        if ((e = cudaEventRecord(h.x_done[k], h.cmp)) != cudaSuccess) break;

        // ---- copies out (x last: free[k] must follow every kernel of the step)
        const struct { cudaEvent_t ev; const long long* off; void* const* dst; } outs[3] = {
            {h.y_done[k], L.y, out_y}, {h.o_done[k], L.o, out_o}, {h.x_done[k], L.x, out_x}};
        for (int j = 0; j < 3 && e == cudaSuccess; ++j) {
            const bool last = j == 2;
            if (!last && !outs[j].dst[0] && !outs[j].dst[1]) continue;
            e = cudaStreamWaitEvent(h.out, outs[j].ev, 0);
            for (int s = 0; s < 2 && e == cudaSuccess; ++s)
                if (N[s] > 0 && outs[j].dst[s])
                    e = cudaMemcpyAsync(outs[j].dst[s], dev(outs[j].off[s]),
                                        (size_t)L.tok_bytes[s], d2h, h.out);
        }
        if (e == cudaSuccess) e = cudaEventRecord(h.free_[k], h.out);
    }
    if (status == MMDIT_ERR_CUDA) where = nullptr;   // the failing entry point set the text
    // Whatever was enqueued, later work on the caller's stream waits for it.
    if (started) {
        cudaStream_t ss[3] = {h.in, h.cmp, h.out};
        for (int j = 0; j < 3; ++j) {
            cudaError_t e2 = cudaEventRecord(h.end[j], ss[j]);
            if (e2 == cudaSuccess) e2 = cudaStreamWaitEvent(user, h.end[j], 0);
            if (e == cudaSuccess) e = e2;
        }
    }
    destroy(h);
    if (status != MMDIT_OK) return status;
    if (e != cudaSuccess) {
        if (where) set_last_error(where, (int)e);
        return MMDIT_ERR_CUDA;
    }
    return MMDIT_OK;
}
