/*
 * Float64 CPU oracle for one MMDiT block's joint-attention core.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA library, and the CUDA library never
 * calls it.
 *
 * Every function is the plain definition written out with loops in double
 * precision, parallelised over independent rows with OpenMP and nothing else
 * (no blocking, no fusion, no reordering of a row's arithmetic beyond the
 * definition).  Sources, cited by page title and section:
 *
 *   [V]  "Vimoo 1.0: Video Generation for Compact, Lightweight, and High-Speed",
 *        section 2.2 "Dual-Stream MMDiT Backbone":
 *          - each stream projects its own Q/K/V; the sequences are concatenated
 *            for joint attention and the outputs are split back per stream;
 *          - 3D RoPE over temporal / vertical / horizontal positions, the 128
 *            head dims split 16 / 56 / 56, applied to the visual Q and K only;
 *          - Q and K RMS-normalised within each head with distinct learned
 *            scales;
 *          - LayerNorm before attention with timestep shift / scale, and gates
 *            that control each branch's residual contribution.
 *   [S]  "Seaweed-7B: Cost-Effective Training of Video Generation Foundation
 *        Model", section 3.2: MM-RoPE gives text tokens a 1D position that the
 *        three RoPE components (T, H, W) share; 3D window attention restricts
 *        attention to w_t x w_h x w_w windows of the visual grid.
 *   [W4] "Wan 2.1" technical report (Chinese translation), section 4.2.1
 *        (patchify + flatten of the (T, H, W) latent into a token sequence) and
 *        section 4.3.1 (DiT attention is non-causal).
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - RoPE pairs are adjacent (2j, 2j+1) inside each axis chunk, chunk order
 *     T, H, W; frequency of pair j on an axis of width d is base^(-2j/d);
 *     rotation (x, y) -> (x cos a - y sin a, x sin a + y cos a).
 *   - token n of the visual stream sits at t = n / (Hp*Wp), h = (n / Wp) % Hp,
 *     w = n % Wp (raster flatten); the rotation angle uses pos * pos_scale.
 *   - joint key order is [visual ; conditioning]; cond keys at index
 *     >= ctx_len[b] are excluded; cond query rows >= ctx_len[b] output zero.
 *   - LayerNorm has no affine, biased variance; modulate is
 *     LN(x) * (1 + scale) + shift.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include "oracle.h"

/* ---- QK-RMSNorm [V] -------------------------------------------------------
 * For each row r of D values: y = x / sqrt(mean(x^2) + eps) * g.             */
void oracle_rmsnorm(const double* x, double* y, const double* g,
                    long rows, int D, double eps)
{
    #pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; ++r) {
        const double* xr = x + r * (long)D;
        double* yr = y + r * (long)D;
        double ss = 0.0;
        for (int d = 0; d < D; ++d) ss += xr[d] * xr[d];
        double rms = sqrt(ss / (double)D + eps);
        for (int d = 0; d < D; ++d) yr[d] = xr[d] / rms * g[d];
    }
}

/* ---- 3D RoPE [V], flatten order [W4] ---------------------------------------
 * x: [B, N, H, D] visual rows, rotated in place.  N must equal T*Hp*Wp.      */
void oracle_rope3d(double* x, int B, int N, int H, int D, const oracle_grid* grid)
{
    const int HW = grid->H * grid->W;
    #pragma omp parallel for schedule(static)
    for (long bn = 0; bn < (long)B * N; ++bn) {
        int n = (int)(bn % N);
        int pos[3];
        pos[0] = n / HW;                 /* t */
        pos[1] = (n / grid->W) % grid->H; /* h */
        pos[2] = n % grid->W;            /* w */
        for (int hd = 0; hd < H; ++hd) {
            double* row = x + (bn * H + hd) * (long)D;
            int offset = 0;
            for (int a = 0; a < 3; ++a) {
                int d_a = grid->split[a];
                double p = (double)pos[a] * grid->pos_scale[a];
                for (int j = 0; j < d_a / 2; ++j) {
                    double freq = pow(grid->rope_base, -2.0 * (double)j / (double)d_a);
                    double ang = p * freq;
                    double c = cos(ang), s = sin(ang);
                    double u = row[offset + 2 * j];
                    double v = row[offset + 2 * j + 1];
                    row[offset + 2 * j]     = u * c - v * s;
                    row[offset + 2 * j + 1] = u * s + v * c;
                }
                offset += d_a;
            }
        }
    }
}

/* ---- RoPE at explicit positions ----------------------------------------------
 * Same rotation as oracle_rope3d, but token n of x [B, N, H, D] sits at the
 * per-axis positions pos[3n + a] given by the caller (already scaled).  With
 * pos = (p, p, p) this is the text-token case of the Seaweed-7B report's
 * MM-RoPE (section 3.2): a 1D position shared by the three components.        */
void oracle_rope_positions(double* x, int B, int N, int H, int D, const double* pos,
                           double rope_base, const int* split)
{
    #pragma omp parallel for schedule(static)
    for (long bn = 0; bn < (long)B * N; ++bn) {
        int n = (int)(bn % N);
        for (int hd = 0; hd < H; ++hd) {
            double* row = x + (bn * H + hd) * (long)D;
            int offset = 0;
            for (int a = 0; a < 3; ++a) {
                int d_a = split[a];
                double p = pos[3 * (long)n + a];
                for (int j = 0; j < d_a / 2; ++j) {
                    double ang = p * pow(rope_base, -2.0 * (double)j / (double)d_a);
                    double c = cos(ang), sn = sin(ang);
                    double u = row[offset + 2 * j];
                    double v = row[offset + 2 * j + 1];
                    row[offset + 2 * j]     = u * c - v * sn;
                    row[offset + 2 * j + 1] = u * sn + v * c;
                }
                offset += d_a;
            }
        }
    }
}

/* ---- joint attention [V], non-causal [W4] ----------------------------------
 * Per (b, h): Q = [Qv; Qc], K = [Kv; Kc], V = [Vv; Vc] (joint index i < Nv is
 * visual row i, otherwise cond row i - Nv).  For each requested query row:
 *   s_j = q . k_j * scale over valid keys j, m = max s_j, p_j = exp(s_j - m),
 *   o = sum_j p_j v_j / sum_j p_j.
 * Requested rows are triplets (b, h, i); out is [nrows, D].                   */
void oracle_joint_attention_rows(const double* qv, const double* kv, const double* vv,
                                 const double* qc, const double* kc, const double* vc,
                                 const int* ctx_len, int B, int Nv, int Nc, int H, int D,
                                 double scale, const long* rows, long nrows, double* out)
{
    (void)B;
    #pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)(Nv + Nc + 1));
        #pragma omp for schedule(dynamic, 4)
        for (long r = 0; r < nrows; ++r) {
            long b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
            int L = ctx_len ? ctx_len[b] : Nc;
            double* o = out + r * (long)D;
            for (int d = 0; d < D; ++d) o[d] = 0.0;
            const double* q;
            if (i < Nv) {
                q = qv + ((b * Nv + i) * H + h) * (long)D;
            } else {
                if (i - Nv >= L) continue;        /* padded cond query: zero */
                q = qc + ((b * Nc + (i - Nv)) * H + h) * (long)D;
            }
            int nk = Nv + L;
            double m = -INFINITY;
            for (int j = 0; j < nk; ++j) {
                const double* k = (j < Nv) ? kv + ((b * Nv + j) * H + h) * (long)D
                                           : kc + ((b * Nc + (j - Nv)) * H + h) * (long)D;
                double acc = 0.0;
                for (int d = 0; d < D; ++d) acc += q[d] * k[d];
                s[j] = acc * scale;
                if (s[j] > m) m = s[j];
            }
            if (nk == 0) continue;
            double den = 0.0;
            for (int j = 0; j < nk; ++j) {
                double p = exp(s[j] - m);
                den += p;
                const double* v = (j < Nv) ? vv + ((b * Nv + j) * H + h) * (long)D
                                           : vc + ((b * Nc + (j - Nv)) * H + h) * (long)D;
                for (int d = 0; d < D; ++d) o[d] += p * v[d];
            }
            for (int d = 0; d < D; ++d) o[d] /= den;
        }
        free(s);
    }
}

/* ---- adaLN modulate [V] ------------------------------------------------------
 * Per row of C values of sample b: mu = mean, var = mean((x - mu)^2),
 * y = (x - mu) / sqrt(var + eps) * (1 + scale[b, c]) + shift[b, c].          */
void oracle_adaln_modulate(const double* x, const double* shift, const double* scale,
                           double* y, int B, int N, int C, double eps)
{
    #pragma omp parallel for schedule(static)
    for (long bn = 0; bn < (long)B * N; ++bn) {
        long b = bn / N;
        const double* xr = x + bn * (long)C;
        double* yr = y + bn * (long)C;
        double mu = 0.0;
        for (int c = 0; c < C; ++c) mu += xr[c];
        mu /= (double)C;
        double var = 0.0;
        for (int c = 0; c < C; ++c) var += (xr[c] - mu) * (xr[c] - mu);
        var /= (double)C;
        double rstd = 1.0 / sqrt(var + eps);
        for (int c = 0; c < C; ++c)
            yr[c] = (xr[c] - mu) * rstd * (1.0 + scale[b * C + c]) + shift[b * C + c];
    }
}

/* ---- gated residual [V] -------------------------------------------------------
 * out[b, n, c] = x[b, n, c] + gate[b, c] * branch[b, n, c].                   */
void oracle_gated_residual(const double* x, const double* branch, const double* gate,
                           double* out, int B, int N, int C)
{
    #pragma omp parallel for schedule(static)
    for (long bn = 0; bn < (long)B * N; ++bn) {
        long b = bn / N;
        for (int c = 0; c < C; ++c)
            out[bn * C + c] = x[bn * C + c] + gate[b * C + c] * branch[bn * C + c];
    }
}

/* ---- backward of adaLN modulate [V] -------------------------------------------
 * Reverse-mode derivative of y = xh * (1 + scale[b, c]) + shift[b, c], with
 * xh = (x - mu) * rstd and rstd = 1 / sqrt(var + eps) over the C values of a
 * row (biased variance).  For the upstream gradient dy of a row:
 *   g  = dy * (1 + scale[b, c])
 *   dx = rstd * (g - mean_c(g) - xh * mean_c(g * xh))
 *   dshift[b, c] = sum over the rows of sample b of dy
 *   dscale[b, c] = sum over the rows of sample b of dy * xh
 * dshift and dscale [B, C] are written, not accumulated.                      */
void oracle_adaln_modulate_bwd(const double* x, const double* scale, const double* dy,
                               int B, int N, int C, double eps, double* dx, double* dshift,
                               double* dscale)
{
    for (long i = 0; i < (long)B * C; ++i) {
        dshift[i] = 0.0;
        dscale[i] = 0.0;
    }
    double* xh = (double*)malloc(sizeof(double) * (size_t)C);
    for (int b = 0; b < B; ++b) {
        for (int n = 0; n < N; ++n) {
            const long row = ((long)b * N + n) * C;
            const double* xr = x + row;
            const double* dr = dy + row;
            double sum = 0.0;
            for (int c = 0; c < C; ++c) sum += xr[c];
            const double mean = sum / (double)C;
            double ss = 0.0;
            for (int c = 0; c < C; ++c) ss += (xr[c] - mean) * (xr[c] - mean);
            const double rstd = 1.0 / sqrt(ss / (double)C + eps);
            double mg = 0.0, mgx = 0.0;
            for (int c = 0; c < C; ++c) {
                xh[c] = (xr[c] - mean) * rstd;
                const double g = dr[c] * (1.0 + scale[(long)b * C + c]);
                mg += g;
                mgx += g * xh[c];
                dshift[(long)b * C + c] += dr[c];
                dscale[(long)b * C + c] += dr[c] * xh[c];
            }
            mg /= (double)C;
            mgx /= (double)C;
            for (int c = 0; c < C; ++c) {
                const double g = dr[c] * (1.0 + scale[(long)b * C + c]);
                dx[row + c] = rstd * (g - mg - xh[c] * mgx);
            }
        }
    }
    free(xh);
}

/* ---- backward of the gated residual [V] ------------------------------------
 * out = x + gate[b, c] * branch:  dx = dout,  dbranch = gate[b, c] * dout,
 * dgate[b, c] = sum over the rows of sample b of dout * branch (written).      */
void oracle_gated_residual_bwd(const double* branch, const double* gate, const double* dout,
                               int B, int N, int C, double* dx, double* dbranch, double* dgate)
{
    for (long i = 0; i < (long)B * C; ++i) dgate[i] = 0.0;
    for (int b = 0; b < B; ++b) {
        for (int n = 0; n < N; ++n) {
            const long row = ((long)b * N + n) * C;
            for (int c = 0; c < C; ++c) {
                dx[row + c] = dout[row + c];
                dbranch[row + c] = gate[(long)b * C + c] * dout[row + c];
                dgate[(long)b * C + c] += dout[row + c] * branch[row + c];
            }
        }
    }
}

/* ---- 3D window attention [S] ----------------------------------------------
 * Seaweed-7B report, section 3.2: the visual tokens are partitioned into
 * w_t x w_h x w_w windows and attention is computed only within a window
 * (even layers 1 x 2 x 2, odd layers 4 x 1 x 1).  Readings where the report is
 * silent:
 *   - parts[a] is the number of windows along axis a; an axis of extent X
 *     split into p parts gives the first X % p parts X / p + 1 positions and
 *     the others X / p (part k starts at k * (X / p) + min(k, X % p));
 *   - a visual query attends to the visual keys of its own window and to every
 *     valid conditioning key; a conditioning query attends to every valid key
 *     (the joint attention above, unchanged).
 * Inputs are in raster order; rows are (b, h, i) triplets as above.           */
static int oracle_part_of(int x, int extent, int parts)
{
    const int q = extent / parts, r = extent % parts;
    for (int k = 0; k < parts; ++k) {
        const int start = k * q + (k < r ? k : r);
        const int size = q + (k < r ? 1 : 0);
        if (x >= start && x < start + size) return k;
    }
    return -1;
}

void oracle_window_of_tokens(const oracle_grid* grid, const int* parts, int* win)
{
    for (int t = 0; t < grid->T; ++t)
        for (int h = 0; h < grid->H; ++h)
            for (int w = 0; w < grid->W; ++w) {
                const int kt = oracle_part_of(t, grid->T, parts[0]);
                const int kh = oracle_part_of(h, grid->H, parts[1]);
                const int kw = oracle_part_of(w, grid->W, parts[2]);
                win[(t * grid->H + h) * grid->W + w] = (kt * parts[1] + kh) * parts[2] + kw;
            }
}

void oracle_window_attention_rows(const double* qv, const double* kv, const double* vv,
                                  const double* qc, const double* kc, const double* vc,
                                  const int* ctx_len, int B, int Nv, int Nc, int H, int D,
                                  const oracle_grid* grid, const int* parts, double scale,
                                  const long* rows, long nrows, double* out)
{
    (void)B;
    int* win = (int*)malloc(sizeof(int) * (size_t)(Nv > 0 ? Nv : 1));
    oracle_window_of_tokens(grid, parts, win);
    #pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)(Nv + Nc + 1));
        int* key = (int*)malloc(sizeof(int) * (size_t)(Nv + Nc + 1));
        #pragma omp for schedule(dynamic, 4)
        for (long r = 0; r < nrows; ++r) {
            long b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
            int L = ctx_len ? ctx_len[b] : Nc;
            double* o = out + r * (long)D;
            for (int d = 0; d < D; ++d) o[d] = 0.0;
            const double* q;
            if (i < Nv) {
                q = qv + ((b * Nv + i) * H + h) * (long)D;
            } else {
                if (i >= Nv + L) continue;        /* padded conditioning query: zero */
                q = qc + ((b * Nc + (i - Nv)) * H + h) * (long)D;
            }
            /* the keys this query sees, as joint indices */
            int nk = 0;
            for (int j = 0; j < Nv; ++j)
                if (i >= Nv || win[j] == win[i]) key[nk++] = j;
            for (int j = 0; j < L; ++j) key[nk++] = Nv + j;
            if (nk == 0) continue;
            double m = -INFINITY;
            for (int e = 0; e < nk; ++e) {
                const int j = key[e];
                const double* k = (j < Nv) ? kv + ((b * Nv + j) * H + h) * (long)D
                                           : kc + ((b * Nc + (j - Nv)) * H + h) * (long)D;
                double acc = 0.0;
                for (int d = 0; d < D; ++d) acc += q[d] * k[d];
                s[e] = acc * scale;
                if (s[e] > m) m = s[e];
            }
            double den = 0.0;
            for (int e = 0; e < nk; ++e) {
                const int j = key[e];
                double p = exp(s[e] - m);
                den += p;
                const double* v = (j < Nv) ? vv + ((b * Nv + j) * H + h) * (long)D
                                           : vc + ((b * Nc + (j - Nv)) * H + h) * (long)D;
                for (int d = 0; d < D; ++d) o[d] += p * v[d];
            }
            for (int d = 0; d < D; ++d) o[d] /= den;
        }
        free(key);
        free(s);
    }
    free(win);
}

/* ---- joint attention backward [V], non-causal [W4] -------------------------
 * Gradients of the joint attention above for an upstream gradient dO on every
 * output row (the reverse-mode derivative of the definition; the Seaweed-7B
 * report, section 3.4, trains forward and backward of this attention).  With
 * s_ij = scale q_i . k_j over valid keys, p_ij = softmax_j(s_ij),
 * o_i = sum_j p_ij v_j and D_i = dO_i . o_i:
 *   dv_j += p_ij dO_i
 *   dP_ij = dO_i . v_j,   dS_ij = p_ij (dP_ij - D_i)
 *   dq_i  = scale sum_j dS_ij k_j,   dk_j += scale dS_ij q_i
 * Padded conditioning query rows have a constant (zero) output: they add
 * nothing, and their dq is zero; padded keys get zero dk and dv.
 * lse (if not NULL) [B, H, Nv + Nc] receives log sum_j exp(s_ij) per joint row,
 * +infinity for rows without an output.                                      */
static const double* oracle_row(const double* vis, const double* ctx, long b, long j, int Nv,
                                int Nc, int H, long h, int D)
{
    return (j < Nv) ? vis + ((b * Nv + j) * H + h) * (long)D
                    : ctx + ((b * Nc + (j - Nv)) * H + h) * (long)D;
}

void oracle_joint_attention_bwd(const double* qv, const double* kv, const double* vv,
                                const double* qc, const double* kc, const double* vc,
                                const int* ctx_len, const double* dov, const double* doc,
                                int B, int Nv, int Nc, int H, int D, double scale,
                                double* dqv, double* dkv, double* dvv,
                                double* dqc, double* dkc, double* dvc, double* lse)
{
    const long nv = (long)B * Nv * H * D, nc = (long)B * Nc * H * D;
    memset(dqv, 0, sizeof(double) * (size_t)nv);
    memset(dkv, 0, sizeof(double) * (size_t)nv);
    memset(dvv, 0, sizeof(double) * (size_t)nv);
    memset(dqc, 0, sizeof(double) * (size_t)nc);
    memset(dkc, 0, sizeof(double) * (size_t)nc);
    memset(dvc, 0, sizeof(double) * (size_t)nc);
    #pragma omp parallel
    {
        double* p = (double*)malloc(sizeof(double) * (size_t)(Nv + Nc + 1));
        double* o = (double*)malloc(sizeof(double) * (size_t)D);
        /* each (b, h) owns its rows of every gradient: no two threads write
         * the same element */
        #pragma omp for schedule(dynamic, 1)
        for (long bh = 0; bh < (long)B * H; ++bh) {
            const long b = bh / H, h = bh % H;
            const int L = ctx_len ? ctx_len[b] : Nc;
            const int nk = L + Nv;  /* valid keys */
            for (long i = 0; i < Nv + Nc; ++i) {
                if (lse) lse[bh * (long)(Nv + Nc) + i] = INFINITY;
                if (i >= nk || nk == 0) continue;    /* padded query row */
                const double* q = oracle_row(qv, qc, b, i, Nv, Nc, H, h, D);
                const double* dO = oracle_row(dov, doc, b, i, Nv, Nc, H, h, D);
                double m = -INFINITY;
                for (int j = 0; j < nk; ++j) {
                    const double* k = oracle_row(kv, kc, b, j, Nv, Nc, H, h, D);
                    double acc = 0.0;
                    for (int d = 0; d < D; ++d) acc += q[d] * k[d];
                    p[j] = acc * scale;
                    if (p[j] > m) m = p[j];
                }
                double den = 0.0;
                for (int j = 0; j < nk; ++j) den += exp(p[j] - m);
                if (lse) lse[bh * (long)(Nv + Nc) + i] = m + log(den);
                for (int d = 0; d < D; ++d) o[d] = 0.0;
                for (int j = 0; j < nk; ++j) {
                    p[j] = exp(p[j] - m) / den;
                    const double* v = oracle_row(vv, vc, b, j, Nv, Nc, H, h, D);
                    for (int d = 0; d < D; ++d) o[d] += p[j] * v[d];
                }
                double Di = 0.0;
                for (int d = 0; d < D; ++d) Di += dO[d] * o[d];
                double* dq = (double*)oracle_row(dqv, dqc, b, i, Nv, Nc, H, h, D);
                for (int j = 0; j < nk; ++j) {
                    const double* k = oracle_row(kv, kc, b, j, Nv, Nc, H, h, D);
                    const double* v = oracle_row(vv, vc, b, j, Nv, Nc, H, h, D);
                    double* dk = (double*)oracle_row(dkv, dkc, b, j, Nv, Nc, H, h, D);
                    double* dv = (double*)oracle_row(dvv, dvc, b, j, Nv, Nc, H, h, D);
                    double dP = 0.0;
                    for (int d = 0; d < D; ++d) dP += dO[d] * v[d];
                    const double dS = p[j] * (dP - Di);
                    for (int d = 0; d < D; ++d) {
                        dv[d] += p[j] * dO[d];
                        dq[d] += scale * dS * k[d];
                        dk[d] += scale * dS * q[d];
                    }
                }
            }
        }
        free(o);
        free(p);
    }
}

/* ---- 3D window attention backward [S] --------------------------------------
 * The reverse-mode derivative of oracle_window_attention_rows (the Seaweed-7B
 * report, section 3.2, restricts the attention to windows; its section 3.4
 * trains forward and backward): the joint backward above with the key set of
 * each query row restricted as the window forward restricts it (a visual query
 * sees its own window's visual keys and every valid conditioning key; a
 * conditioning query sees every valid key).  Inputs and outputs in raster
 * order; lse as in oracle_joint_attention_bwd.                                */
void oracle_window_attention_bwd(const double* qv, const double* kv, const double* vv,
                                 const double* qc, const double* kc, const double* vc,
                                 const int* ctx_len, const double* dov, const double* doc,
                                 int B, int Nv, int Nc, int H, int D, const oracle_grid* grid,
                                 const int* parts, double scale, double* dqv, double* dkv,
                                 double* dvv, double* dqc, double* dkc, double* dvc, double* lse)
{
    const long nv = (long)B * Nv * H * D, nc = (long)B * Nc * H * D;
    memset(dqv, 0, sizeof(double) * (size_t)nv);
    memset(dkv, 0, sizeof(double) * (size_t)nv);
    memset(dvv, 0, sizeof(double) * (size_t)nv);
    memset(dqc, 0, sizeof(double) * (size_t)nc);
    memset(dkc, 0, sizeof(double) * (size_t)nc);
    memset(dvc, 0, sizeof(double) * (size_t)nc);
    int* win = (int*)malloc(sizeof(int) * (size_t)(Nv > 0 ? Nv : 1));
    oracle_window_of_tokens(grid, parts, win);
    #pragma omp parallel
    {
        double* p = (double*)malloc(sizeof(double) * (size_t)(Nv + Nc + 1));
        int* key = (int*)malloc(sizeof(int) * (size_t)(Nv + Nc + 1));
        double* o = (double*)malloc(sizeof(double) * (size_t)D);
        /* each (b, h) owns its rows of every gradient */
        #pragma omp for schedule(dynamic, 1)
        for (long bh = 0; bh < (long)B * H; ++bh) {
            const long b = bh / H, h = bh % H;
            const int L = ctx_len ? ctx_len[b] : Nc;
            for (long i = 0; i < Nv + Nc; ++i) {
                if (lse != NULL) lse[bh * (long)(Nv + Nc) + i] = INFINITY;
                if (i >= (long)Nv + L) continue;       /* padded query row */
                int nkeys = 0;                         /* the keys this query sees */
                for (int j = 0; j < Nv; ++j)
                    if (i >= Nv || win[j] == win[i]) key[nkeys++] = j;
                for (int j = 0; j < L; ++j) key[nkeys++] = Nv + j;
                if (nkeys == 0) continue;
                const double* q = oracle_row(qv, qc, b, i, Nv, Nc, H, h, D);
                const double* dO = oracle_row(dov, doc, b, i, Nv, Nc, H, h, D);
                double m = -INFINITY;
                for (int e = 0; e < nkeys; ++e) {
                    const double* k = oracle_row(kv, kc, b, key[e], Nv, Nc, H, h, D);
                    double acc = 0.0;
                    for (int d = 0; d < D; ++d) acc += q[d] * k[d];
                    p[e] = acc * scale;
                    if (p[e] > m) m = p[e];
                }
                double den = 0.0;
                for (int e = 0; e < nkeys; ++e) den += exp(p[e] - m);
                if (lse != NULL) lse[bh * (long)(Nv + Nc) + i] = m + log(den);
                for (int d = 0; d < D; ++d) o[d] = 0.0;
                for (int e = 0; e < nkeys; ++e) {
                    p[e] = exp(p[e] - m) / den;
                    const double* v = oracle_row(vv, vc, b, key[e], Nv, Nc, H, h, D);
                    for (int d = 0; d < D; ++d) o[d] += p[e] * v[d];
                }
                double Di = 0.0;
                for (int d = 0; d < D; ++d) Di += dO[d] * o[d];
                double* dq = (double*)oracle_row(dqv, dqc, b, i, Nv, Nc, H, h, D);
                for (int e = 0; e < nkeys; ++e) {
                    const int j = key[e];
                    const double* k = oracle_row(kv, kc, b, j, Nv, Nc, H, h, D);
                    const double* v = oracle_row(vv, vc, b, j, Nv, Nc, H, h, D);
                    double* dk = (double*)oracle_row(dkv, dkc, b, j, Nv, Nc, H, h, D);
                    double* dv = (double*)oracle_row(dvv, dvc, b, j, Nv, Nc, H, h, D);
                    double dPw = 0.0;
                    for (int d = 0; d < D; ++d) dPw += dO[d] * v[d];
                    const double dSw = p[e] * (dPw - Di);
                    for (int d = 0; d < D; ++d) {
                        dv[d] += p[e] * dO[d];
                        dq[d] += scale * dSw * k[d];
                        dk[d] += scale * dSw * q[d];
                    }
                }
            }
        }
        free(o);
        free(key);
        free(p);
    }
    free(win);
}

/* dq and lse of selected query rows (b, h, i) only, for sizes where the full
 * backward is out of reach: the same definitions, row by row.  dq_out is
 * [nrows, D]; lse_out [nrows].                                                */
void oracle_joint_attention_dq_rows(const double* qv, const double* kv, const double* vv,
                                    const double* qc, const double* kc, const double* vc,
                                    const int* ctx_len, const double* dov, const double* doc,
                                    int B, int Nv, int Nc, int H, int D, double scale,
                                    const long* rows, long nrows, double* dq_out, double* lse_out)
{
    (void)B;
    #pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)(Nv + Nc + 1));
        double* o = (double*)malloc(sizeof(double) * (size_t)D);
        #pragma omp for schedule(dynamic, 4)
        for (long r = 0; r < nrows; ++r) {
            const long b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
            const int L = ctx_len ? ctx_len[b] : Nc;
            const int nk = L + Nv;  /* valid keys */
            double* dq = dq_out + r * (long)D;
            for (int d = 0; d < D; ++d) dq[d] = 0.0;
            lse_out[r] = INFINITY;
            if (i >= nk || nk == 0) continue;
            const double* q = oracle_row(qv, qc, b, i, Nv, Nc, H, h, D);
            const double* dO = oracle_row(dov, doc, b, i, Nv, Nc, H, h, D);
            double mx = -INFINITY;
            for (int j = 0; j < nk; ++j) {
                const double* k = oracle_row(kv, kc, b, j, Nv, Nc, H, h, D);
                double acc = 0.0;
                for (int d = 0; d < D; ++d) acc += q[d] * k[d];
                s[j] = scale * acc;
                mx = s[j] > mx ? s[j] : mx;
            }
            double sum = 0.0;
            for (int j = 0; j < nk; ++j) sum += exp(s[j] - mx);
            lse_out[r] = mx + log(sum);
            for (int d = 0; d < D; ++d) o[d] = 0.0;
            for (int j = 0; j < nk; ++j) {
                s[j] = exp(s[j] - mx) / sum;             /* now p_ij */
                const double* v = oracle_row(vv, vc, b, j, Nv, Nc, H, h, D);
                for (int d = 0; d < D; ++d) o[d] += s[j] * v[d];
            }
            double Dsum = 0.0;
            for (int d = 0; d < D; ++d) Dsum += dO[d] * o[d];
            for (int j = 0; j < nk; ++j) {
                const double* k = oracle_row(kv, kc, b, j, Nv, Nc, H, h, D);
                const double* v = oracle_row(vv, vc, b, j, Nv, Nc, H, h, D);
                double g = 0.0;
                for (int d = 0; d < D; ++d) g += dO[d] * v[d];
                const double w = scale * s[j] * (g - Dsum);
                for (int d = 0; d < D; ++d) dq[d] += w * k[d];
            }
        }
        free(o);
        free(s);
    }
}

/* dK and dV of selected keys (b, h, joint key index j), for the checks at
 * sizes where the whole backward is too slow [the reverse-mode derivative of
 * the joint attention, as oracle_joint_attention_bwd]:
 *   dV_j = sum_i P_ij dO_i,   dK_j = scale * sum_i P_ij (dO_i . V_j - D_i) Q_i
 * over the query rows i that have an output (i < Nv + ctx_len[b]), with
 * P_ij = exp(s_ij - lse_i), s_ij = scale Q_i . K_j and D_i = dO_i . O_i.
 * For every (b, h) that holds a selected key, lse_i and D_i of all its query
 * rows come first, each row computed as the forward defines it; then the sums
 * over i for each selected key.  Padded keys (j >= Nv + ctx_len[b]) get 0. */
void oracle_joint_attention_dkdv_rows(const double* qv, const double* kv, const double* vv,
                                      const double* qc, const double* kc, const double* vc,
                                      const int* ctx_len, const double* dov, const double* doc,
                                      int B, int Nv, int Nc, int H, int D, double scale,
                                      const long* keys, long nkeys, double* dk_out,
                                      double* dv_out)
{
    double* lse = (double*)malloc(sizeof(double) * (size_t)(Nv + Nc + 1));
    double* Dr = (double*)malloc(sizeof(double) * (size_t)(Nv + Nc + 1));
    for (long bh = 0; bh < (long)B * H; ++bh) {
        const long b = bh / H, h = bh % H;
        int any = 0;
        for (long r = 0; r < nkeys; ++r)
            if (keys[3 * r] == b && keys[3 * r + 1] == h) { any = 1; break; }
        if (!any) continue;
        const int L = ctx_len ? ctx_len[b] : Nc;
        const int nval = Nv + L;    /* valid keys, and the query rows with an output */
        #pragma omp parallel
        {
            double* s = (double*)malloc(sizeof(double) * (size_t)(nval + 1));
            double* o = (double*)malloc(sizeof(double) * (size_t)D);
            #pragma omp for schedule(dynamic, 16)
            for (int i = 0; i < nval; ++i) {
                const double* q = oracle_row(qv, qc, b, i, Nv, Nc, H, h, D);
                const double* dO = oracle_row(dov, doc, b, i, Nv, Nc, H, h, D);
                double mx = -INFINITY;
                for (int j = 0; j < nval; ++j) {
                    const double* k = oracle_row(kv, kc, b, j, Nv, Nc, H, h, D);
                    double acc = 0.0;
                    for (int d = 0; d < D; ++d) acc += q[d] * k[d];
                    s[j] = scale * acc;
                    mx = s[j] > mx ? s[j] : mx;
                }
                double sum = 0.0;
                for (int j = 0; j < nval; ++j) sum += exp(s[j] - mx);
                lse[i] = mx + log(sum);
                for (int d = 0; d < D; ++d) o[d] = 0.0;
                for (int j = 0; j < nval; ++j) {
                    const double p = exp(s[j] - mx) / sum;
                    const double* v = oracle_row(vv, vc, b, j, Nv, Nc, H, h, D);
                    for (int d = 0; d < D; ++d) o[d] += p * v[d];
                }
                double Di = 0.0;
                for (int d = 0; d < D; ++d) Di += dO[d] * o[d];
                Dr[i] = Di;
            }
            free(o);
            free(s);
        }
        #pragma omp parallel for schedule(dynamic, 1)
        for (long r = 0; r < nkeys; ++r) {
            if (keys[3 * r] != b || keys[3 * r + 1] != h) continue;
            const long j = keys[3 * r + 2];
            double* dk = dk_out + r * (long)D;
            double* dv = dv_out + r * (long)D;
            for (int d = 0; d < D; ++d) { dk[d] = 0.0; dv[d] = 0.0; }
            if (j >= nval) continue;                          /* padded key */
            const double* k = oracle_row(kv, kc, b, j, Nv, Nc, H, h, D);
            const double* v = oracle_row(vv, vc, b, j, Nv, Nc, H, h, D);
            for (int i = 0; i < nval; ++i) {
                const double* qi = oracle_row(qv, qc, b, i, Nv, Nc, H, h, D);
                const double* dOi = oracle_row(dov, doc, b, i, Nv, Nc, H, h, D);
                double sij = 0.0, dP = 0.0;
                for (int d = 0; d < D; ++d) {
                    sij += qi[d] * k[d];
                    dP += dOi[d] * v[d];
                }
                const double p = exp(scale * sij - lse[i]);
                const double dS = p * (dP - Dr[i]);
                for (int d = 0; d < D; ++d) {
                    dv[d] += p * dOi[d];
                    dk[d] += scale * dS * qi[d];
                }
            }
        }
    }
    free(Dr);
    free(lse);
}

/* ---- QK-RMSNorm + RoPE backward [V], [S] ----------------------------------
 * Reverse-mode derivative of y = R(pos) (x / r * g), r = sqrt(mean(x^2) + eps),
 * for rows x [rows, D] whose RoPE positions are pos [rows, 3] (already scaled;
 * pos == NULL: no rotation, the conditioning stream), given dy [rows, D]:
 *   u  = R(pos)^T dy                         (rotation by the opposite angle)
 *   dg += u * x / r                          (summed over rows)
 *   dx = g * u / r - x * sum_d(g * u * x) / (D r^3)
 * dg [D] is accumulated into (caller zeroes it).                             */
void oracle_rmsnorm_rope_bwd(const double* x, const double* g, const double* dy,
                             const double* pos, double rope_base, const int* split,
                             long rows, int D, double eps, double* dx, double* dg)
{
    double* part = (double*)calloc((size_t)D, sizeof(double));
    #pragma omp parallel
    {
        double* u = (double*)malloc(sizeof(double) * (size_t)D);
        double* acc = (double*)calloc((size_t)D, sizeof(double));
        #pragma omp for schedule(static)
        for (long r = 0; r < rows; ++r) {
            const double* xr = x + r * (long)D;
            const double* dr = dy + r * (long)D;
            for (int d = 0; d < D; ++d) u[d] = dr[d];
            if (pos) {
                int off = 0;
                for (int a = 0; a < 3; ++a) {
                    const int d_a = split[a];
                    for (int j = 0; j < d_a / 2; ++j) {
                        const double ang = pos[3 * r + a] * pow(rope_base, -2.0 * (double)j / (double)d_a);
                        const double c = cos(ang), s = sin(ang);
                        const double a0 = dr[off + 2 * j], a1 = dr[off + 2 * j + 1];
                        u[off + 2 * j] = a0 * c + a1 * s;        /* transpose of the rotation */
                        u[off + 2 * j + 1] = -a0 * s + a1 * c;
                    }
                    off += d_a;
                }
            }
            double ms = 0.0;
            for (int d = 0; d < D; ++d) ms += xr[d] * xr[d];
            const double rr = sqrt(ms / (double)D + eps);
            double dot = 0.0;
            for (int d = 0; d < D; ++d) dot += g[d] * u[d] * xr[d];
            double* dxr = dx + r * (long)D;
            for (int d = 0; d < D; ++d) {
                dxr[d] = g[d] * u[d] / rr - xr[d] * dot / ((double)D * rr * rr * rr);
                acc[d] += u[d] * xr[d] / rr;
            }
        }
        #pragma omp critical
        for (int d = 0; d < D; ++d) part[d] += acc[d];
        free(acc);
        free(u);
    }
    for (int d = 0; d < D; ++d) dg[d] += part[d];
    free(part);
}

/* ---- 8-bit joint attention [W4] ---------------------------------------------
 * Wan 2.1 report, section 4.4.3: Int8 for S = Q K^T, FP8 (E4M3) for O = P V,
 * accumulation across key blocks in fp32.  Readings where the report is
 * silent (each also listed in the design notes):
 *   - q is quantised per (sample, token, head) row, k per block of 128
 *     consecutive tokens of one (sample, head, stream), symmetric:
 *     scale = max|x| / 127 (fp32), code = round-half-even(x / scale) (fp32),
 *     clamped to [-127, 127]; scale 0 gives codes 0;
 *   - v is quantised to E4M3 per (sample, head, channel) over the valid
 *     tokens of both streams: scale = max|v| / 448 (fp32), code = E4M3
 *     rounding (half-even, saturating at 448) of v / scale (fp32);
 *   - the softmax of a row, written plainly: x_j is the score of valid key j
 *     in log2 units (the exact integer dot product of the codes times both
 *     scales, the softmax scale and log2 e), m = ceil(max_j x_j) an integer,
 *     P'_j = 2^(x_j - m + 6) <= 2^6, rounded to E4M3 for the P V product and
 *     unrounded in the row sum:  o = scale_v * sum_j E4M3(P'_j) v8_j / sum_j P'_j.
 * A tiled schedule that keeps an integer running maximum and rescales by
 * 2^(old - new) computes the same values: every P' it rounds differs from the
 * one here by an exact power of two, which E4M3 rounding commutes with, except
 * for keys whose P' here falls in E4M3's subnormal range (x_j < m - 12, a
 * weight below 2^-12 of the largest).
 * The report does not fix the precision in which P' is formed before its E4M3
 * rounding.  An implementation whose P' differs from this one's by a relative
 * amount up to rel can round a P' that lies that close to a rounding midpoint
 * the other way.  With amb non-NULL, amb[r][d] bounds what those choices can
 * move o: sum_j w_j |v8_jd| scale_v,d / sum_j P'_j, where w_j is the larger
 * distance from E4M3(P'_j) to E4M3(P'_j (1 - rel)) and to E4M3(P'_j (1 + rel))
 * (0 unless P'_j is within rel of a midpoint). */

/* E4M3: 1 sign, 4 exponent bits (bias 7), 3 mantissa bits; no infinity; the
 * largest finite magnitude is 1.75 * 2^8 = 448; subnormals step 2^-9.       */
double oracle_e4m3_round(double x)
{
    const double a = fabs(x);
    if (!(a == a)) return x;
    if (a >= 448.0) return copysign(448.0, x);                  /* saturate */
    double quantum;
    if (a < ldexp(1.0, -6)) {
        quantum = ldexp(1.0, -9);                               /* subnormal range */
    } else {
        int e;
        frexp(a, &e);                                           /* a = f 2^e, f in [0.5, 1) */
        quantum = ldexp(1.0, e - 1 - 3);                        /* 3 mantissa bits */
    }
    double r = nearbyint(a / quantum) * quantum;                /* half-even */
    if (r > 448.0) r = 448.0;
    return copysign(r, x);                                      /* keeps the sign of zero */
}

unsigned char oracle_e4m3_encode(double x)
{
    const double r = oracle_e4m3_round(x);
    const unsigned char sign = signbit(r) ? 0x80 : 0;
    const double a = fabs(r);
    if (a == 0.0) return sign;
    if (a < ldexp(1.0, -6)) return sign | (unsigned char)nearbyint(a / ldexp(1.0, -9));
    int e;
    const double f = frexp(a, &e);                              /* a = (2f) 2^(e-1) */
    const int exp_field = e - 1 + 7;
    const int mant = (int)nearbyint((2.0 * f - 1.0) * 8.0);
    return sign | (unsigned char)(exp_field << 3) | (unsigned char)mant;
}

double oracle_e4m3_decode(unsigned char c)
{
    const int exp_field = (c >> 3) & 15, mant = c & 7;
    const double a = exp_field == 0 ? ldexp((double)mant, -9)
                                    : ldexp(1.0 + mant / 8.0, exp_field - 7);
    return (c & 0x80) ? -a : a;
}

/* x [B, N, H, D] -> codes [B, N, H, D], scales [B, H, ceil(N / block)]       */
void oracle_quant_int8(const double* x, int B, int N, int H, int D, int block,
                       signed char* codes, float* scales)
{
    const int nblk = (N + block - 1) / block;
    #pragma omp parallel for schedule(static)
    for (long bh = 0; bh < (long)B * H; ++bh) {
        const long b = bh / H, h = bh % H;
        for (int k = 0; k < nblk; ++k) {
            const int n0 = k * block, n1 = (n0 + block < N) ? n0 + block : N;
            float amax = 0.0f;
            for (int n = n0; n < n1; ++n)
                for (int d = 0; d < D; ++d) {
                    const float v = fabsf((float)x[((b * N + n) * H + h) * (long)D + d]);
                    if (v > amax) amax = v;
                }
            const float s = amax / 127.0f;
            scales[bh * nblk + k] = s;
            for (int n = n0; n < n1; ++n)
                for (int d = 0; d < D; ++d) {
                    const long idx = ((b * N + n) * H + h) * (long)D + d;
                    float q = s > 0.0f ? rintf((float)x[idx] / s) : 0.0f;
                    q = q > 127.0f ? 127.0f : (q < -127.0f ? -127.0f : q);
                    codes[idx] = (signed char)q;
                }
        }
    }
}

/* v [B, N_s, H, D] of both streams -> E4M3 codes, scales [B, H, D]           */
void oracle_quant_v_e4m3(const double* vv, const double* vc, const int* ctx_len, int B, int Nv,
                         int Nc, int H, int D, unsigned char* cv, unsigned char* cc,
                         float* scales)
{
    #pragma omp parallel for schedule(static)
    for (long bh = 0; bh < (long)B * H; ++bh) {
        const long b = bh / H, h = bh % H;
        const int L = ctx_len ? ctx_len[b] : Nc;
        for (int d = 0; d < D; ++d) {
            float amax = 0.0f;
            for (int n = 0; n < Nv; ++n) {
                const float v = fabsf((float)vv[((b * Nv + n) * H + h) * (long)D + d]);
                if (v > amax) amax = v;
            }
            for (int n = 0; n < L; ++n) {
                const float v = fabsf((float)vc[((b * Nc + n) * H + h) * (long)D + d]);
                if (v > amax) amax = v;
            }
            const float s = amax / 448.0f;
            scales[bh * D + d] = s;
            for (int n = 0; n < Nv; ++n) {
                const long idx = ((b * Nv + n) * H + h) * (long)D + d;
                cv[idx] = s > 0.0f ? oracle_e4m3_encode((double)((float)vv[idx] / s)) : 0;
            }
            for (int n = 0; n < Nc; ++n) {
                const long idx = ((b * Nc + n) * H + h) * (long)D + d;
                cc[idx] = s > 0.0f ? oracle_e4m3_encode((double)((float)vc[idx] / s)) : 0;
            }
        }
    }
}

/* Attention output rows (b, h, i) of the 8-bit method from the quantised
 * operands: q codes / scales [B, H, N_s] per stream, k codes / block scales
 * [B, H, ceil(N_s / 128)] per stream, v codes and channel scales [B, H, D]. */
void oracle_attention_q8_rows(const signed char* qv, const signed char* qc, const float* sqv,
                              const float* sqc, const signed char* kv, const signed char* kc,
                              const float* skv, const float* skc, const unsigned char* vv,
                              const unsigned char* vc, const float* sv, const int* ctx_len,
                              int B, int Nv, int Nc, int H, int D, double scale,
                              const long* rows, long nrows, double* out, double rel, double* amb)
{
    (void)B;
    const double log2e = 1.4426950408889634;
    const int tv = (Nv + 127) / 128, tc = (Nc + 127) / 128;
    #pragma omp parallel
    {
        double* x = (double*)malloc(sizeof(double) * (size_t)(Nv + Nc + 1));
        double* acc = (double*)malloc(sizeof(double) * (size_t)D);
        double* wacc = (double*)malloc(sizeof(double) * (size_t)D);
        #pragma omp for schedule(dynamic, 4)
        for (long r = 0; r < nrows; ++r) {
            const long b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
            const int L = ctx_len ? ctx_len[b] : Nc;
            const int nval = Nv + L;                /* valid keys: visual, then cond */
            double* o = out + r * (long)D;
            for (int d = 0; d < D; ++d) { o[d] = 0.0; acc[d] = 0.0; wacc[d] = 0.0; }
            if (amb)
                for (int d = 0; d < D; ++d) amb[r * (long)D + d] = 0.0;
            if (i >= nval || nval == 0) continue;   /* no output */
            const signed char* q = (i < Nv) ? qv + ((b * Nv + i) * H + h) * (long)D
                                            : qc + ((b * Nc + (i - Nv)) * H + h) * (long)D;
            const double sq = (i < Nv) ? sqv[(b * H + h) * (long)Nv + i]
                                       : sqc[(b * H + h) * (long)Nc + (i - Nv)];
            /* scores in log2 units */
            double mx = -INFINITY;
            for (int j = 0; j < nval; ++j) {
                const int seg = j >= Nv, jj = seg ? j - Nv : j, Ns = seg ? Nc : Nv;
                const signed char* k = (seg ? kc : kv) + ((b * Ns + jj) * H + h) * (long)D;
                const double skb = (seg ? skc : skv)[(b * H + h) * (long)(seg ? tc : tv) + jj / 128];
                long dot = 0;
                for (int d = 0; d < D; ++d) dot += (long)q[d] * (long)k[d];
                x[j] = (double)dot * sq * skb * scale * log2e;
                if (x[j] > mx) mx = x[j];
            }
            const double m = ceil(mx);
            double l = 0.0;
            for (int j = 0; j < nval; ++j) {
                const int seg = j >= Nv, jj = seg ? j - Nv : j, Ns = seg ? Nc : Nv;
                const double p = exp2(x[j] - m + 6.0);
                l += p;
                const double pq = oracle_e4m3_round(p);
                const unsigned char* v = (seg ? vc : vv) + ((b * Ns + jj) * H + h) * (long)D;
                for (int d = 0; d < D; ++d) acc[d] += pq * oracle_e4m3_decode(v[d]);
                if (amb) {   /* the other rounding a P' this close to a midpoint can take */
                    const double wl = fabs(pq - oracle_e4m3_round(p * (1.0 - rel)));
                    const double wh = fabs(oracle_e4m3_round(p * (1.0 + rel)) - pq);
                    const double w = wl > wh ? wl : wh;
                    if (w > 0.0)
                        for (int d = 0; d < D; ++d) wacc[d] += w * fabs(oracle_e4m3_decode(v[d]));
                }
            }
            for (int d = 0; d < D; ++d) o[d] = acc[d] * sv[(b * H + h) * (long)D + d] / l;
            if (amb)
                for (int d = 0; d < D; ++d)
                    amb[r * (long)D + d] = wacc[d] * sv[(b * H + h) * (long)D + d] / l;
        }
        free(wacc);
        free(acc);
        free(x);
    }
}
