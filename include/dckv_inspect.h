/*
 * dckv_inspect.h -- inspection and self-test entry points of the DCKV library.
 *
 * These calls expose intermediates (workspace layout, derived tables, per-stage device
 * times) and the raw tcgen05 GEMM, so that tests can compare each stage with an
 * independent reference and benchmarks can attribute time to kernels.  They are not
 * needed to encode or decode.  Same conventions as dckv.h: device pointers are
 * caller-owned, calls are ordered on the given stream.
 */
#ifndef DCKV_INSPECT_H_
#define DCKV_INSPECT_H_

#include "dckv.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Byte offsets (from the workspace base) of the intermediates of one call shape.
 * which = 0: encode layout, 1: decode layout.  Code arrays have rows of 2048 entries that
 * hold the kept components only, in ascending component order (column m is the m-th kept
 * component); code_width columns are in use (K_eff rounded up to 64, zero past K_eff) and
 * dropped components have code 0.  After dckv_encode on a stream:
 *   q32  int32 [n_rows][2048] codes q = round(y / Delta), rows in prompt order, coded rows
 *        only (positions 4 .. N-129 of each prompt);
 *   qe   bf16 [ne_pad][2048] even-row codes, one extra zero row after each prompt;
 *   cen8 int8 [n_rows][K_eff] centres in slot order: slot row row_slot[r] of coded row r
 *        (chunk order: every even row of every prompt, then every odd row), kept
 *        components in ascending order;
 *   sym16 uint16 [n_rows][K_eff] symbols in the same order;
 *   row_slot int32 [n_rows].
 * After dckv_decode: q16 fp16 [n_rows][2048] decoded codes (exact below 2048), qe.
 * Encode recomputes in fp64 every code whose fp32 ratio y / Delta lies in a guard band
 * around a half-step boundary (whole rows when the row's norm is large). */
typedef struct {
  uint64_t q32, qe, cen8, row_slot, sym16, q16, x16, g16;
  uint64_t counters; /* uint32[64]; encode: [0] codes recomputed exactly, [1] rows recomputed whole;
                        decode: [0] rows holding codes beyond +-2047 */
  int64_t n_rows, ne_pad;
  int32_t n_chunks;
  uint64_t total;
  int32_t code_width;
} dckv_ws_view;

int dckv_ws_offsets(const dckv_codec *codec, const int64_t *seq_offsets, int batch, int which, dckv_ws_view *out);

/* Copy the derived tables to host memory (any pointer may be NULL):
 *   cdf   uint16 [64][510] cumulative frequencies per scale index (cdf[510] = 65536);
 *   scale uint8 [2048] scale index s_c;  keep uint8 [2048] 1 = coded;
 *   exps  int32 [3] power-of-two operand scales (transform, correction, inverse).
 * Synchronises the device. */
int dckv_codec_export(const dckv_codec *codec, uint16_t *cdf, uint8_t *scale, uint8_t *keep, int32_t *exps);

/* Device pointers of the per-vocabulary mean tables, kept components only (column kc is
 * compact index kc, row stride kw from dckv_codec_gemm_shape), built at creation:
 * t_even: int8 [vocab][kw], the even rows' centres clamp(round(embed @ w_even), +-127);
 * t_odd:  fp32 [vocab][kw], embed @ w_odd[0:2048].  NULL without mean models. */
int dckv_codec_tables(const dckv_codec *codec, const void **t_even, const void **t_odd);

/* Chunk rows G in use (chosen at creation when 0 was passed) and the entropy of the kept
 * components' tables in bits per coded row (the rate the codec's own model expects). */
int dckv_codec_info(const dckv_codec *codec, int32_t *chunk_rows, double *model_bits_per_row);

/* Shapes of the codec's compacted GEMMs (kept components only), int32 [4]:
 *   [0] K_eff, kept components;
 *   [1] kw, K_eff rounded up to 64: the K extent of the GEMMs that read codes, and the
 *       code arrays' columns in use;
 *   [2] mp, K_eff rounded up to 256: the M extent of the GEMMs that produce one value per
 *       kept component (transform, odd mean model);
 *   [3] the inverse's lo-half cut: its split operand's lo half is added for the first this
 *       many compact components only (the rest carry less than 2^-15 of the reconstruction's
 *       rms under the codec's Laplace model); equal to kw for a codec with decoder-side
 *       synthesis. */
int dckv_codec_gemm_shape(const dckv_codec *codec, int32_t *shape);

/* Self-test hook: when ratio_dev (device fp32 [n_rows][2048]) is not NULL, later encodes
 * also write the fp32 transform ratios y / Delta there, before any exact recomputation.
 * Pass NULL to stop.  The buffer must cover the largest call's coded rows. */
int dckv_debug_ratio(dckv_codec *codec, void *ratio_dev);

/* Per-stage device times of the last encode / decode that the calling host thread issued
 * on this codec with timing enabled (each thread keeps its own events, so threads do not
 * share them).  Events are recorded on the call's stream; read after synchronising it.
 * Returns the number of stages written to ms / names (at most max). */
int dckv_set_timing(dckv_codec *codec, int enable);
int dckv_get_timing(const dckv_codec *codec, float *ms, const char **names, int max);

/* Kernels this library has launched in this process so far (every codec and device;
 * codec creation included).  Benchmarks read it before and after a timed region. */
long long dckv_launch_count(void);

/* Self-test of the tcgen05 GEMM core: D[n][m] = sum_s sum_k A[s][m][k] * B[n][k]
 * (fp32 accumulate).  A: device fp16/bf16 [slabs][M][K]; B: device [N][K]; D: device
 * fp32 [N][M].  M % 128 == 0, K % 64 == 0, slabs in {1, 2}, bn (N tile) in 16..256 step 16.
 * pair = 1 runs the CTA-pair kernel (cta_group::2, 256 x bn tiles; M % 256 == 0). */
int dckv_debug_gemm(int bf16, const void *A, int slabs, const void *B, int M, int N, int K, float *D, int bn,
                    int pair, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* DCKV_INSPECT_H_ */
