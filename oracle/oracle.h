/* Float64 CPU oracle (test infrastructure only): declarations.
 * Argument meaning mirrors the CUDA library's entry points, but every array is
 * a host float64 array and every result is written to a separate output. */
#ifndef MMDIT_ORACLE_H
#define MMDIT_ORACLE_H

typedef struct {
    int T, H, W;            /* visual token grid */
    double pos_scale[3];    /* per-axis position multiplier (T, H, W) */
    double rope_base;       /* RoPE frequency base */
    int split[3];           /* head dims per axis; sums to D */
} oracle_grid;

void oracle_rmsnorm(const double* x, double* y, const double* g, long rows, int D, double eps);
void oracle_rope3d(double* x, int B, int N, int H, int D, const oracle_grid* grid);
void oracle_rope_positions(double* x, int B, int N, int H, int D, const double* pos,
                           double rope_base, const int* split);
void oracle_joint_attention_rows(const double* qv, const double* kv, const double* vv,
                                 const double* qc, const double* kc, const double* vc,
                                 const int* ctx_len, int B, int Nv, int Nc, int H, int D,
                                 double scale, const long* rows, long nrows, double* out);
/* Window index (window-major: T part slowest, W part fastest) of every visual
 * token of the grid, in raster order; parts = windows along T, H, W. */
void oracle_window_of_tokens(const oracle_grid* grid, const int* parts, int* win);
void oracle_window_attention_rows(const double* qv, const double* kv, const double* vv,
                                  const double* qc, const double* kc, const double* vc,
                                  const int* ctx_len, int B, int Nv, int Nc, int H, int D,
                                  const oracle_grid* grid, const int* parts, double scale,
                                  const long* rows, long nrows, double* out);
void oracle_joint_attention_bwd(const double* qv, const double* kv, const double* vv,
                                const double* qc, const double* kc, const double* vc,
                                const int* ctx_len, const double* dov, const double* doc,
                                int B, int Nv, int Nc, int H, int D, double scale,
                                double* dqv, double* dkv, double* dvv,
                                double* dqc, double* dkc, double* dvc, double* lse);
void oracle_window_attention_bwd(const double* qv, const double* kv, const double* vv,
                                 const double* qc, const double* kc, const double* vc,
                                 const int* ctx_len, const double* dov, const double* doc,
                                 int B, int Nv, int Nc, int H, int D, const oracle_grid* grid,
                                 const int* parts, double scale, double* dqv, double* dkv,
                                 double* dvv, double* dqc, double* dkc, double* dvc, double* lse);
void oracle_joint_attention_dq_rows(const double* qv, const double* kv, const double* vv,
                                    const double* qc, const double* kc, const double* vc,
                                    const int* ctx_len, const double* dov, const double* doc,
                                    int B, int Nv, int Nc, int H, int D, double scale,
                                    const long* rows, long nrows, double* dq_out, double* lse_out);
void oracle_joint_attention_dkdv_rows(const double* qv, const double* kv, const double* vv,
                                      const double* qc, const double* kc, const double* vc,
                                      const int* ctx_len, const double* dov, const double* doc,
                                      int B, int Nv, int Nc, int H, int D, double scale,
                                      const long* keys, long nkeys, double* dk_out,
                                      double* dv_out);
void oracle_rmsnorm_rope_bwd(const double* x, const double* g, const double* dy,
                             const double* pos, double rope_base, const int* split,
                             long rows, int D, double eps, double* dx, double* dg);
double oracle_e4m3_round(double x);
unsigned char oracle_e4m3_encode(double x);
double oracle_e4m3_decode(unsigned char c);
void oracle_quant_int8(const double* x, int B, int N, int H, int D, int block,
                       signed char* codes, float* scales);
void oracle_quant_v_e4m3(const double* vv, const double* vc, const int* ctx_len, int B, int Nv,
                         int Nc, int H, int D, unsigned char* cv, unsigned char* cc,
                         float* scales);
void oracle_attention_q8_rows(const signed char* qv, const signed char* qc, const float* sqv,
                              const float* sqc, const signed char* kv, const signed char* kc,
                              const float* skv, const float* skc, const unsigned char* vv,
                              const unsigned char* vc, const float* sv, const int* ctx_len,
                              int B, int Nv, int Nc, int H, int D, double scale,
                              const long* rows, long nrows, double* out, double rel,
                              double* amb);
void oracle_adaln_modulate(const double* x, const double* shift, const double* scale,
                           double* y, int B, int N, int C, double eps);
void oracle_gated_residual(const double* x, const double* branch, const double* gate,
                           double* out, int B, int N, int C);
void oracle_adaln_modulate_bwd(const double* x, const double* scale, const double* dy,
                               int B, int N, int C, double eps, double* dx, double* dshift,
                               double* dscale);
void oracle_gated_residual_bwd(const double* branch, const double* gate, const double* dout,
                               int B, int N, int C, double* dx, double* dbranch, double* dgate);

#endif
