/*
 * oracle.h -- fp64 CPU oracle of the routed sparse-MoE block.
 *
 * TEST INFRASTRUCTURE.  Only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference leg may load this code.  It shares no source, header,
 * table or helper with the CUDA library; it reads the packed expert bytes with
 * its own reader, written from the layout description alone.
 *
 * What it computes (the pages give the structure, not formulas):
 *   - per token and layer a router scores all experts and picks 10 of 512,
 *     plus one always-on shared expert, and the GPU adds the results up
 *     ("Strata open-source runtime" page, section on the model itself;
 *      "Why Strata is fast on low-VRAM GPUs", sections "the problem" and
 *      "one token, three workers");
 *   - experts are feed-forward sub-networks (same pages); their form here is
 *     the SwiGLU FFN with 2/3-bit group-32 weights and fp16 scales, the
 *     plainest reading of the quantised "Q2_0"/"IQ3" expert files the pages
 *     name ("Why Strata is fast...", section "the cost").
 *
 * Arithmetic is fp64 throughout; bf16/fp16/fp32 inputs convert exactly.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ORC_PRENORM 1   /* block input is bf16(RMSNorm(x)), eps 1e-6, no weight */
#define ORC_RESIDUAL 2  /* block output is x + MoE(.) */

typedef struct {
  int32_t d, E, F, Fs, k, bits;      /* Fs = 0: no shared expert */
  const float* Wr;                   /* [E][d] */
  const float* bias;                 /* [E] or NULL */
  const int32_t* expert_slot;        /* [E] expert -> slot */
  const uint8_t* codes;              /* [E slots][codes bytes per expert] */
  const uint16_t* scales;            /* [E slots][scales per expert] fp16 bits */
  const uint8_t* shared_codes;
  const uint16_t* shared_scales;
} orc_layer;

/* number formats */
double orc_half_to_double(uint16_t h);
double orc_bf16_to_double(uint16_t b);
uint16_t orc_double_to_bf16(double v);      /* round to nearest even */

/* packed-format reader */
int64_t orc_codes_bytes(int32_t R, int32_t K, int32_t bits);
int32_t orc_read_code(const uint8_t* mat_codes, int32_t R, int32_t K, int32_t bits, int32_t row,
                      int32_t col);
double orc_dequant(const uint8_t* mat_codes, const uint16_t* mat_scales, int32_t R, int32_t K,
                   int32_t bits, int32_t row, int32_t col);
void orc_dequant_matrix(const uint8_t* mat_codes, const uint16_t* mat_scales, int32_t R, int32_t K,
                        int32_t bits, double* W);

/* steps */
void orc_router_logits(const orc_layer* L, const double* x, int32_t T, double* logits);
void orc_select_topk_f32(const float* logits, int32_t T, int32_t E, int32_t k, int32_t* ids);
void orc_select_topk_f64(const double* logits, int32_t T, int32_t E, int32_t k, int32_t* ids);
void orc_renorm_weights(const double* logits, const int32_t* ids, int32_t T, int32_t E, int32_t k,
                        double* w);
void orc_bucket(const int32_t* ids, int32_t T, int32_t k, int32_t E, int32_t* counts,
                int32_t* offsets, int32_t* entries);
double orc_silu(double z);
void orc_expert_ffn(const uint8_t* codes, const uint16_t* scales, int32_t d, int32_t F,
                    int32_t bits, const double* x, double* y);
void orc_rmsnorm_bf16(const uint16_t* x, int32_t T, int32_t d, double eps, uint16_t* xn);

/* whole block for the tokens listed in rows[0..n_rows) (rows == NULL: all T).
 * sel_logits: fp32 logits [T][E] to select on (the device's, in parity mode) or
 * NULL to select on the oracle's own logits rounded to fp32.
 * Outputs per listed token: y [n][d], logits [n][E] (fp64, may be NULL),
 * ids [n][k], w [n][k] (may be NULL).  Returns 0 on success. */
int orc_block_forward(const orc_layer* L, const uint16_t* x_bf16, int32_t T, const int32_t* rows,
                      int32_t n_rows, const float* sel_logits, int32_t flags, double* y,
                      double* logits, int32_t* ids, double* w);

int orc_num_threads(void);
void orc_set_num_threads(int32_t n);

#ifdef __cplusplus
}
#endif
#endif
