/*
 * qsa_oracle.h -- CPU oracle for the QSA forward pass (TEST INFRASTRUCTURE).
 *
 * Only the tests, __graft_entry__.smoke() and bench.py's cpu_baseline /
 * reference leg may use this header or the library built from it.  It is not
 * part of the product and shares nothing with the CUDA library.
 *
 * Limits: idx_dim <= 1024, rope_dims <= idx_dim and even, n_heads divisible by
 * n_groups, budget_tokens divisible by r.  Inputs are finite.
 */
#ifndef QSA_ORACLE_H
#define QSA_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
  int32_t r;              /* tokens per micro-block (4 on the pages)          */
  int32_t budget_tokens;  /* kept tokens per query (2048 on the pages)        */
  int32_t n_heads;        /* attention query heads (24)                       */
  int32_t n_groups;       /* KV groups (2)                                    */
  int32_t head_dim;       /* 256                                               */
  int32_t idx_heads;      /* indexer query heads (4)                           */
  int32_t idx_dim;        /* indexer head dim                                  */
  int32_t rope_dims;      /* rotated dims of the indexer vectors (even)        */
  double rope_base;       /* 1e7                                               */
  double softmax_scale;   /* 1/sqrt(head_dim)                                  */
  int32_t round_bf16;     /* 1: k^ and q~ are held in bf16 (RNE); 0: fp32      */
} qsa_ref_config;

double qsa_ref_round_bf16(double x);
double qsa_ref_rope_theta(const qsa_ref_config* c, int i);
void qsa_ref_rope_cos_sin(const qsa_ref_config* c, int64_t pos, float* cos_out, float* sin_out);
void qsa_ref_rope_vec(const qsa_ref_config* c, const float* x, int64_t pos, float* out);
void qsa_ref_compress_keys(const qsa_ref_config* c, const float* k_idx, int64_t b0, int64_t b1,
                           float* khat);
void qsa_ref_index_scores(const qsa_ref_config* c, const float* q_idx, const float* w, int64_t t,
                          const float* khat, double* s);
int qsa_ref_select(const qsa_ref_config* c, const double* s, int64_t t, int32_t* sel);
void qsa_ref_attend(const qsa_ref_config* c, const float* q, const float* k, const float* v,
                    int64_t ld, int64_t t, const int32_t* sel, int nsel, double* o, double* lse);
void qsa_ref_attend_bwd(const qsa_ref_config* c, const float* q, const float* k, const float* v,
                        int64_t ld, int64_t t, const int32_t* sel, int nsel, const float* dout,
                        double* dq, double* dk, double* dv);
void qsa_ref_forward(const qsa_ref_config* c, const float* q, const float* q_idx, const float* w,
                     const int64_t* pos, int64_t nq, const float* k_idx, const float* k,
                     const float* v, int64_t ld, int32_t* sel, int32_t* nsel, double* o,
                     double* lse, int n_threads);
int qsa_ref_acc_bits(void);

#ifdef __cplusplus
}
#endif
#endif
