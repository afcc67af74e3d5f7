/*
 * dckv.h -- C ABI of the B200 (sm_100a) DCKV per-token codec.
 *
 * The codec compresses the stored prompt KV cache of a hybrid language model, as
 * described in "DCKV: Learned Transform Coding of the Prompt KV Cache in Hybrid
 * Language Models" (trove.briskstack.com summary, section "How it works"):
 *   - rows: per token, pre-RoPE keys and values of the 6 full-attention layers
 *     (2 KV heads x 256 dims each) stacked into one 6,144-dim bf16 row (12,288 bytes);
 *     the first 4 and last 128 positions of a prompt are stored verbatim in bf16;
 *   - transform: one shared basis maps a row to 2,048 coefficients, plus one hidden
 *     layer of 256 GELU units; components whose Laplace scale is below 0.05
 *     quantisation steps are dropped; per-component quantisation steps;
 *   - coding: rANS under discretised Laplace distributions, codes beyond +-127 escaped
 *     with 64 raw bits each;
 *   - conditional entropy models: even positions take their code means from the
 *     prompt token's embedding, odd positions also from both decoded neighbours
 *     (1-D checkerboard: decoding is exactly two parallel passes);
 *   - decoding inverts the transform and reapplies RoPE to the keys.
 *
 * Memory and streams.  Every pointer argument marked "device" is CUDA device memory
 * owned by the caller; the library never frees it.  dckv_encode and dckv_decode
 * allocate nothing: their scratch is the caller's workspace.  Only dckv_codec_create
 * allocates (derived codec tensors, released by dckv_codec_destroy).  Calls are
 * asynchronous and ordered on the given stream; the return value reports argument
 * errors found on the host, and errors found on the device are written to
 * *status_dev (an int32 the caller reads after synchronising the stream).
 *
 * Determinism.  No floating-point atomics and no split reductions: the same inputs
 * give bit-identical blobs and rows, and a decoder computes exactly the predictions
 * its encoder used (the pages' stated requirement for table selection, "Limits").
 *
 * Threads and devices.  dckv_encode and dckv_decode only read the codec, so one codec
 * may be used from several host threads at once, on different streams, each call with
 * its own workspace and outputs.  Creating, destroying and reconfiguring a codec
 * (dckv_set_timing, dckv_debug_ratio) must not overlap other calls on it.  Every entry
 * point makes the codec's device current while it runs and gives the caller's current
 * device back before it returns.
 */
#ifndef DCKV_H_
#define DCKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- shapes (fixed by the pages' model: 6 layers x {K,V} x 2 heads x 256 dims) ---- */
#define DCKV_ROW_DIM 6144     /* elements per KV row                                */
#define DCKV_N_COEF 2048      /* transform coefficients per row                     */
#define DCKV_N_HIDDEN 256     /* GELU units of the correction                       */
#define DCKV_N_LAYERS 6
#define DCKV_N_KV_HEADS 2
#define DCKV_HEAD_DIM 256
#define DCKV_HEAD_KEPT 4      /* leading positions stored in bf16                   */
#define DCKV_TAIL_KEPT 128    /* trailing positions stored in bf16                  */
#define DCKV_MAX_ROWS 2097152 /* coded rows per call (all prompts together)         */
#define DCKV_MAX_PROMPTS 65536

/* ---- status codes (return values and *status_dev) ---- */
#define DCKV_OK 0
#define DCKV_EINVAL 1      /* bad argument (null pointer, size, shape, alignment)     */
#define DCKV_ECAPACITY 2   /* blob_cap or ws_bytes too small                          */
#define DCKV_ECUDA 3       /* a CUDA runtime call failed                              */
#define DCKV_ECORRUPT 4    /* blob header/tables/streams inconsistent (decode)        */
#define DCKV_ETIMEOUT 5    /* a bounded device wait gave up                           */
#define DCKV_ERANGE 6      /* encode: an input element beyond +-65504 was clamped     */
#define DCKV_ESINGULAR 7   /* fit: a non-positive pivot in the Cholesky factorisation */

typedef struct dckv_codec dckv_codec; /* opaque */

/* Codec weights, as trained (here: seeded synthetics).  All DEVICE pointers, read only,
 * caller-owned; they are read during dckv_codec_create and may be freed afterwards.
 * The linear codec the pages compare DCKV with ("Evidence": no correction, unconditional
 * zero-mean Laplace tables) is w1 = w2 = NULL and embed = w_even = w_odd = NULL (vocab
 * ignored); either pair may be absent on its own.  Without mean models every centre is 0
 * and token_ids may be NULL in encode and decode. */
typedef struct {
  const float *mu;          /* [6144]        codec mean subtracted before the transform   */
  const float *basis;       /* [6144][2048]  shared basis, row-major (basis[d*2048 + c])  */
  const float *w1;          /* [6144][256]   correction layer 1 (row-major, input-major)  */
  const float *w2;          /* [256][2048]   correction layer 2                           */
  const float *delta;       /* [2048]        quantisation step per component (> 0)       */
  const float *laplace_b;   /* [2048]        Laplace scale per component, data units      */
  const uint16_t *embed;    /* bf16 [vocab][2048] prompt-token input embeddings          */
  const uint16_t *w_even;   /* bf16 [2048][2048] even mean model: mu = e @ w_even         */
  const uint16_t *w_odd;    /* bf16 [6144][2048] odd mean model: mu = [e, bf16(q_left),
                               bf16(q_right)] @ w_odd; the neighbour blocks carry Delta_c */
  int32_t vocab;            /* rows of embed (1 .. 2^20; ignored without mean models)    */
  const float *v1;          /* [2048][256]   decoder-side synthesis, first layer, or NULL   */
  const float *v2;          /* [256][6144]   decoder-side synthesis, second layer, or NULL:
                               decode adds GELU((q * Delta) @ v1) @ v2 to mu + (q * Delta) B^T
                               before RoPE (no counterpart on the pages beyond the weight
                               count they report; zero-initialise to leave it out)        */
} dckv_params;

/* Per-blob byte accounting (host-side parse of a blob header and tables). */
typedef struct {
  uint64_t total;          /* whole blob                                               */
  uint64_t header_tables;  /* header + prompt table + chunk table + pad                */
  uint64_t kept_rows;      /* bf16 rows stored verbatim (first 4 / last 128)          */
  uint64_t states;         /* 128 bytes of final rANS states per chunk                 */
  uint64_t esc_counts;     /* 4 bytes per chunk                                        */
  uint64_t esc_values;     /* 8 bytes per escaped code                                 */
  uint64_t words;          /* 16-bit renormalisation words                             */
  uint64_t padding;        /* section padding to 4 bytes                               */
  uint64_t payload;        /* total - kept_rows: what the compression ratio counts     */
  uint32_t n_prompts, n_chunks, n_coded_rows, n_escapes, chunk_rows, k_eff;
} dckv_byte_report;

/* Build a codec on `device` from trained weights.  Derives, on the device: the drop mask
 * and scale indices (Laplace scale in steps beta = b/Delta; dropped if beta < 0.05;
 * s = clamp(round(8 log2(beta/0.05)), 0, 63)), the 64 integer Laplace tables (16-bit
 * precision, 509 residuals + ESC), the split fp16 operands of the transform, correction
 * and inverse GEMMs, and the per-vocabulary mean tables of the kept components: the even
 * centres clamp(round(embed @ w_even), +-127) (int8) and embed @ w_odd[0:2048] (fp32).
 * chunk_rows (1..256) is the number of same-parity rows
 * per rANS chunk; 0 selects 16; -1 selects the smallest count whose fixed per-chunk bytes
 * (states, escape count, offset) stay within 3.5% of the tables' own entropy per row.
 * Fewer rows per chunk give more independent streams (faster decode) and more bytes.
 * Allocates device memory: vocab * kw * 5 bytes for the two tables (kw = kept components
 * rounded up to 64) and about 177 MiB for the split GEMM operands, the fp32 weight copies
 * for the exact recomputation of near-boundary codes and the coder's tables (16 MiB more
 * with decoder-side synthesis weights); 16 MiB more during creation only.
 * Synchronises the device.  Returns DCKV_OK or an error; *out is NULL on error. */
int dckv_codec_create(const dckv_params *params, int device, int chunk_rows, dckv_codec **out);
void dckv_codec_destroy(dckv_codec *codec);

/* Number of kept (coded) components, K_eff in [0, 2048]. */
int dckv_codec_k_eff(const dckv_codec *codec);

/* Workspace bytes needed by dckv_encode / dckv_decode for this batch shape
 * (seq_offsets: HOST int64 [batch+1], seq_offsets[0] = 0, non-decreasing).
 * Returns 0 on a bad shape. */
size_t dckv_workspace_bytes(const dckv_codec *codec, const int64_t *seq_offsets, int batch);

/* Largest blob dckv_encode can produce for this batch shape (every code escaped). */
size_t dckv_blob_bound(const dckv_codec *codec, const int64_t *seq_offsets, int batch);

/* Encode a batch of prompts into one blob.
 *   rows        device bf16 [sum N][6144], pre-RoPE rows (prompt-major, position order)
 *   token_ids   device int32 [sum N], prompt token ids (side information, not stored)
 *   seq_offsets HOST int64 [batch+1], prompt b holds rows seq_offsets[b]..[b+1]-1
 *   blob        device, blob_cap bytes, 16-byte aligned; receives the blob
 *   blob_size_dev  device uint64: the blob's size in bytes on success
 *   status_dev  device int32: DCKV_OK, DCKV_ECAPACITY (blob_cap too small; the blob is
 *               then incomplete), DCKV_ERANGE (input clamped to fp16 range), DCKV_ETIMEOUT
 *   workspace   device, ws_bytes >= dckv_workspace_bytes(...), 256-byte aligned
 * Blob layout: see dckv_bytes.  Returns DCKV_OK or DCKV_EINVAL / DCKV_ECAPACITY (workspace)
 * / DCKV_ECUDA. */
int dckv_encode(const dckv_codec *codec, const void *rows, const int32_t *token_ids,
                const int64_t *seq_offsets, int batch, void *blob, size_t blob_cap,
                uint64_t *blob_size_dev, int32_t *status_dev, void *workspace, size_t ws_bytes,
                void *stream /* cudaStream_t */);

/* Decode a blob into a RoPE'd bf16 KV cache.
 *   blob        device, blob_bytes bytes (16-byte aligned), as written by dckv_encode
 *   token_ids   device int32 [sum N], the same ids the encoder saw
 *   seq_offsets HOST int64 [batch+1], the same prompt lengths
 *   k_out/v_out device bf16 [6][sum N][2][256] each: layer, token, KV head, dim
 *               (RoPE, rotate-half pairs (d, d+128), base 1e7, position = index within
 *               the prompt, applied to keys only)
 *   status_dev  device int32: DCKV_OK or DCKV_ECORRUPT / DCKV_ETIMEOUT
 * Returns DCKV_OK or DCKV_EINVAL / DCKV_ECAPACITY (workspace) / DCKV_ECUDA. */
int dckv_decode(const dckv_codec *codec, const void *blob, size_t blob_bytes,
                const int32_t *token_ids, const int64_t *seq_offsets, int batch, void *k_out,
                void *v_out, int32_t *status_dev, void *workspace, size_t ws_bytes,
                void *stream /* cudaStream_t */);

/* dckv_decode without a caller workspace.  The DCKV method has no counterpart to this call;
 * it serves callers that cannot hand over device memory (a serving engine whose KV-cache
 * pool already holds all free device memory, a host program with no device allocator).
 * Its scratch is one static device array of DCKV_STATIC_SCRATCH_BYTES per GPU that loads
 * the library, held until the process exits; the call allocates nothing.
 *   Limit: batches whose decode scratch (dckv_ws_offsets(..., 1, ...).total) exceeds
 *   DCKV_STATIC_SCRATCH_BYTES -- about 800 coded rows at K_eff = 2048 -- are rejected with
 *   DCKV_ECAPACITY before any device work.
 *   Set-up: the first call on a device looks the array's device address up once (host-side
 *   symbol lookup, under a lock); make that first call before any stream capture.
 *   Sharing: every call on a device uses the same array, which keeps the last call's
 *   contents; each call initialises (clears or overwrites) everything it reads before it
 *   reads it.  Calls that overlap in time on one device -- different streams or host
 *   threads without ordering between them -- race on the array; order them on one stream.
 * Arguments, layouts, status and return values as dckv_decode. */
#define DCKV_STATIC_SCRATCH_BYTES (16u << 20)
int dckv_decode_static(const dckv_codec *codec, const void *blob, size_t blob_bytes,
                       const int32_t *token_ids, const int64_t *seq_offsets, int batch, void *k_out,
                       void *v_out, int32_t *status_dev, void *stream /* cudaStream_t */);

/* Byte breakdown of a blob held in HOST memory (len bytes).  Blob layout, little endian:
 *   64-byte header {u32 magic 0x564B4344 "DCKV", u16 version 1, u16 chunk rows G,
 *     u32 prompts, u32 coefficients (2048), u32 K_eff, u32 even chunks, u32 odd chunks,
 *     u32 kept rows, u64 total bytes, u64 stream offset, u64 kept-row offset, u64 0};
 *   u32 prompt lengths; u32 chunk-section offsets relative to the stream offset
 *   (chunks + 1 entries: every even chunk in prompt order, then every odd chunk);
 *   zero pad to 16; kept rows (bf16 [kept][6144]); chunk sections, each
 *   {u32 final rANS states[32], u32 escape count, i64 escaped codes in symbol order,
 *    u16 words in decoder order, zero pad to 4}.
 * A chunk holds G consecutive same-parity coded rows of one prompt; its symbols run
 * row-major over the kept components and symbol i uses state i mod 32.
 * Returns DCKV_OK, DCKV_EINVAL or DCKV_ECORRUPT. */
int dckv_bytes(const void *blob_host, size_t len, dckv_byte_report *out);

/* Text of the last host-side error on this thread (static storage). */
const char *dckv_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* DCKV_H_ */
