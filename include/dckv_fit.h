/* dckv_fit.h -- closed-form fit of the conditional entropy models to a trained codec.
 *
 * Passage: "DCKV: Learned Transform Coding of the Prompt KV Cache in Hybrid Language
 * Models" (trove.briskstack.com summary), section "Evidence": fitting the conditional
 * models in closed form to an already-trained codec gives a saving similar to that of
 * the trained models, without retraining.  The models are those of "How it works",
 * bullet "Conditional entropy models" (even means from the token embedding, odd means
 * from the embedding and both decoded neighbours).
 *
 * The fit, as this library reads it (the pages name it but give no formulas):
 *   mean models   least squares of the codes on each model's own inputs,
 *                   even rows: X = e(tok)                              [rows][2048]
 *                   odd rows:  X = [e(tok), bf16(q_left), bf16(q_right)] [rows][6144]
 *                 (right neighbour 0 where the prompt has none; targets Y = codes
 *                 clipped to +-32767), from the normal equations with a ridge term
 *                   W = (G + ridge * (diag(G) + 1))^-1 C,  G = X^T X,  C = X^T Y;
 *   scales        Laplace maximum likelihood at the table centres:
 *                   b_c = Delta_c * max(sum |q - centre| / rows, 0.05)  (kept c; the
 *                 fp32 value is raised by one ulp if it fell below 0.05 steps); dropped
 *                 components keep their scale, so the component set is unchanged.
 * The transform (basis, correction, steps) stays as trained.
 *
 * Use: zero a stats buffer (DCKV_FIT_STATS_DOUBLES doubles); call dckv_fit_accumulate
 * on calibration batches with the trained codec; dckv_fit_solve; dckv_fit_to_bf16 gives
 * the w_even / w_odd parameters of a codec.  Create that codec (trained scales), zero
 * an int64 [2049] buffer, call dckv_fit_scales_accumulate with it, then
 * dckv_fit_scales_finish gives the fitted laplace_b; a codec created with both is the
 * refit codec.  Run the scale pass on calibration prompts that the mean fit did not
 * see: a least-squares fit's in-sample residuals are biased low, and scales fitted to
 * them are too narrow for new prompts.  With 6,144 regressors per odd-row mean, a ridge
 * of about 0.1 and tens of thousands of calibration rows per parity keep the fitted
 * means from costing more on new prompts than they save.
 *
 * All pointers are device pointers unless stated; the caller owns every buffer.  Calls
 * are asynchronous on `stream` (a cudaStream_t, NULL = legacy default stream) and
 * return DCKV_OK or a host-detected error (dckv.h); device-detected errors go to the
 * int32 status word.  Token ids are clamped to [0, vocab - 1] like the codec does.
 * Alignment: fp64 and int64 buffers 8 bytes, fp32 and int32 4, bf16 2, workspaces 256
 * (DCKV_EINVAL otherwise).
 */
#ifndef DCKV_FIT_H
#define DCKV_FIT_H

#include <stddef.h>
#include <stdint.h>

#include "dckv.h"

#ifdef __cplusplus
extern "C" {
#endif

/* fp64 layout of the normal-equation sums (row-major blocks, in this order):
 *   G_e [2048][2048], C_e [2048][2048] (C_e[k][c] = sum_rows e_k q_c),
 *   G_o [6144][6144], C_o [6144][2048], then n_even, n_odd (row counts) and 6 spare. */
#define DCKV_FIT_STATS_DOUBLES (2ull * 2048 * 2048 + 6144ull * 6144 + 6144ull * 2048 + 8)
#define DCKV_FIT_OFF_GE 0ull
#define DCKV_FIT_OFF_CE (2048ull * 2048)
#define DCKV_FIT_OFF_GO (2ull * 2048 * 2048)
#define DCKV_FIT_OFF_CO (2ull * 2048 * 2048 + 6144ull * 6144)
#define DCKV_FIT_OFF_N (2ull * 2048 * 2048 + 6144ull * 6144 + 6144ull * 2048)

/* Workspace bytes for dckv_fit_accumulate / dckv_fit_scales_accumulate on this batch
 * shape (the encoder's workspace plus the transposed regressors); 0 on bad arguments. */
size_t dckv_fit_workspace_bytes(const dckv_codec *codec, const int64_t *seq_offsets, int batch);

/* Adds one calibration batch to the sums: runs the encoder of `codec` up to its final
 * codes (transform, quantiser, drop, exact recomputation), builds the regressors and
 * targets above, and adds X^T X and X^T Y of both parities (bf16 tensor-core GEMMs over
 * slices of at most 4,096 rows, fp32 in TMEM, each slice added in fp64).
 *   embed      bf16 [vocab][2048], the token embedding the mean models read
 *   rows, token_ids, seq_offsets, batch   as dckv_encode (seq_offsets on the host)
 *   stats      fp64 [DCKV_FIT_STATS_DOUBLES], accumulated into (zero it first)
 *   status     int32 [1], overwritten (DCKV_OK, DCKV_ERANGE, DCKV_ETIMEOUT)
 *   workspace  >= dckv_fit_workspace_bytes, 256-byte aligned */
int dckv_fit_accumulate(const dckv_codec *codec, const uint16_t *embed, int32_t vocab, const void *rows,
                        const int32_t *token_ids, const int64_t *seq_offsets, int batch, double *stats,
                        int32_t *status, void *workspace, size_t ws_bytes, void *stream);

/* Workspace bytes for dckv_fit_solve (one 6,144 x 6,144 fp64 matrix). */
size_t dckv_fit_solve_workspace_bytes(void);

/* Solves both normal equations with a fp64 blocked Cholesky factorisation and two
 * triangular solves (ridge > 0; see above for its size).
 *   w_even  fp64 [2048][2048] out, w_odd fp64 [6144][2048] out (row k, column c: the
 *           weight of input k in the mean of component c, the codec's layout)
 *   status  int32 [1], overwritten; DCKV_ESINGULAR on a non-positive pivot */
int dckv_fit_solve(const double *stats, double ridge, double *w_even, double *w_odd, int32_t *status,
                   void *workspace, size_t ws_bytes, void *stream);

/* bf16 bits of fp64 values, round to nearest even in one step (codec parameter format). */
int dckv_fit_to_bf16(const double *w, int64_t count, uint16_t *out, void *stream);

/* Adds one calibration batch to the scale sums under `codec` (whose mean models give the
 * centres): abs_sum int64 [2049], abs_sum[c] += sum over coded rows of |q - centre| for
 * kept components, abs_sum[2048] += coded rows.  Other arguments as dckv_fit_accumulate. */
int dckv_fit_scales_accumulate(const dckv_codec *codec, const void *rows, const int32_t *token_ids,
                               const int64_t *seq_offsets, int batch, int64_t *abs_sum, int32_t *status,
                               void *workspace, size_t ws_bytes, void *stream);

/* laplace_b fp32 [2048] out: fitted scales for kept components, `codec`'s own scales for
 * dropped ones (formula above). */
int dckv_fit_scales_finish(const dckv_codec *codec, const int64_t *abs_sum, float *laplace_b, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* DCKV_FIT_H */
