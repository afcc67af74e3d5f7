// dckv_internal.cuh -- shared definitions of the DCKV library (host + device).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <vector>

#include "../../include/dckv.h"

namespace dckv {

constexpr int ROW_DIM = DCKV_ROW_DIM;     // 6144
constexpr int N_COEF = DCKV_N_COEF;       // 2048
constexpr int N_HIDDEN = DCKV_N_HIDDEN;   // 256
constexpr int HEAD_DIM = DCKV_HEAD_DIM;   // 256
constexpr int HEAD_KEPT = DCKV_HEAD_KEPT;
constexpr int TAIL_KEPT = DCKV_TAIL_KEPT;
constexpr int ESC_LIMIT = 127;            // codes beyond +-127 are escaped
constexpr int R_MAX = 2 * ESC_LIMIT;      // residual q - centre in [-254, 254]
constexpr int N_SYM = 2 * R_MAX + 2;      // 509 residual symbols + ESC
constexpr int ESC_SYM = N_SYM - 1;        // 509
constexpr int N_SCALES = 64;
constexpr uint32_t PREC_TOTAL = 1u << 16; // 16-bit frequency precision
constexpr uint32_t RANS_L = 1u << 16;     // lower bound of a 32-bit state
constexpr int LANES = 32;                 // interleaved states per chunk
constexpr double B0_STEPS = 0.05;         // drop threshold and scale-index origin (steps)
constexpr double ROPE_BASE = 1.0e7;
constexpr uint32_t MAGIC = 0x564B4344u;   // "DCKV"
constexpr int VERSION = 1;
constexpr int HEADER_BYTES = 64;
constexpr int CHUNK_FIXED_BYTES = 4 * LANES + 4;  // states + escape count
constexpr int BIG_CODE = 2048;
// Row stride (elements) of the per-call code arrays (q32, qe, q16, qbig).  Their columns
// hold the kept components in compact order (the codec's kw of them are read); the stride
// stays 2,048 so that the fused epilogues address them with a compile-time constant.
constexpr int CODE_LD = N_COEF;
// Lo-half cut of the inverse GEMM's split operand (see dckv_codec::inv_lo_k): the lo halves
// of the components past the cut carry at most this fraction of the reconstruction's rms in
// expectation (about 3e-5; the hi half alone leaves ~2.4e-4 of each term, and bf16 output
// rounding ~2e-3).
constexpr double INV_LO_THETA = 1.0 / 32768.0;            // |q| >= 2048 is not exact in the fp16 code operand
// Guard band of the transform: a code is recomputed in fp64 when its fp32 ratio y / Delta
// lies within REFINE_KAPPA * |x|_2 / Delta + REFINE_W0 of a half-step boundary (the fp32
// path's error grows with the row's norm); rows with |x|_2 > REFINE_NORM_FULL are
// recomputed whole, correction layer included.
constexpr float REFINE_KAPPA = 5.0e-7f;  // measured fp32 error on B200: <= 1.7e-7 * |x|_2
constexpr float REFINE_W0 = 2.0e-5f;
constexpr float REFINE_NORM_FULL = 32.0f;
// GEMM tile widths (tokens per CTA-pair tile): 256, the widest an M = 256 pair MMA takes;
// a wider B tile carries more MMA work per byte moved into shared memory, which is what
// keeps the tensor pipe fed (measured against 224: transform -8%, inverse and odd mean
// model -12% on 64 x 4,096 tokens).
// (The transform and the inverse take 192-token tiles instead where these fill the last
// wave of pairs better: pick_pair_bn.)
constexpr int TRANSFORM_BN = 256;
constexpr int MEAN_ODD_BN = 256;
// Hidden layers (256 rows of M, one pair tile): the decoder's synthesis layer runs narrow
// 64-token tiles (62 pairs for a 4K-token prompt); the encoder's correction layer, K = 6,144,
// runs 256-token tiles with K cut into HIDDEN_SPLIT parts.  A batch with fewer token tiles
// than SMs runs every part as its own tile (64 pairs for a 4K-token prompt: each tile reads
// its A slice once per 256 tokens instead of once per 64) and sums the parts afterwards; a
// larger batch runs each tile's parts as consecutive TMEM partials summed in registers, in
// the same order, so the hidden units are bit-identical on both paths.
constexpr int HIDDEN_BN = 64;
constexpr int HIDDEN_SPLIT_BN = 256;
constexpr int HIDDEN_SPLIT = 4;
// K steps (of 64) per TMEM partial of the transform before it is added into the fp32
// totals: bounds the growth of the tensor core's accumulation error over K = 6,144.
constexpr int TRANSFORM_CHUNK_STEPS = 4;

struct PromptInfo {
  int64_t tok_base;  // first row (token) of the prompt in the batch
  int32_t N;         // tokens
  int32_t n;         // coded rows = max(0, N - 132)
  int32_t n_e, n_o;  // even / odd coded rows
  int32_t row_base;  // first coded row, natural order over the batch
  int32_t ebase;     // first padded even row (each prompt owns n_e + 1 rows, last one zero)
  int32_t kept_base; // first kept row in the blob's kept section
  int32_t n_kept;
  int32_t chunk_e0, chunk_o0;  // first even / odd chunk (global chunk index)
  int32_t slot_e0, slot_o0;    // slot row of the first even / odd row (chunk order)
};

struct ChunkDesc {
  int32_t prompt, parity, j0, nrows;
  int64_t sym_base;  // first symbol slot in the word scratch (rows before * K_eff)
};

// Host-side batch layout, derived from seq_offsets only.
struct Layout {
  int batch = 0;
  int64_t n_tokens = 0;
  int64_t n_rows = 0;     // coded rows
  int64_t ne_pad = 0;     // padded even rows (sum of n_e + 1)
  int64_t n_kept = 0;
  int64_t max_len = 0;    // longest prompt (RoPE table positions)
  int n_chunks = 0, n_chunks_e = 0, n_chunks_o = 0;
  int64_t n_symbols = 0;  // n_rows * K_eff
  int kw = 64;            // columns of the code arrays in use (the codec's kw)
  std::vector<PromptInfo> prompts;
  std::vector<ChunkDesc> chunks;
  uint64_t off_kept = 0, off_streams = 0;  // blob offsets
};

// Workspace carving (byte offsets from the workspace base, each 256-aligned).
struct WsPlan {
  size_t prompts, chunks, row_tok, row_pos, row_edst, e_tok, row_slot, e_slot, slot_chunk;  // tables
  size_t e_row;    // natural coded row of the odd row after each padded even row (-1: none)
  size_t escflag;  // decode: per chunk, 1 if an ESC symbol was seen while writing codes
  size_t qe, cen8;                                                               // both
  size_t x16, g16, q32, sym16, cf32, words, states, nwords, nesc, offs;           // encode
  size_t hpart;    // encode: split-K parts of the correction hidden layer, fp32
  size_t slots16;  // decode: decoded symbols (slot order)
  size_t rope;     // decode: float2 [max_len][128] RoPE (cos, sin)
  size_t row_norm, rowflag, el_bins, bin_count, full_list, g64;        // encode refinement
  uint32_t bin_cap;
  size_t q16, qbig, bigflag, biglist, counters, valid;                  // decode
  size_t total;
};

}  // namespace dckv

// the opaque codec
struct dckv_codec {
  int device = 0;
  int num_sms = 0;
  int chunk_rows = 32;
  int vocab = 0;
  int k_eff = 0;
  // Only kept components are computed: the GEMMs run on compacted operands.  kw = K_eff
  // rounded up to 64 (the width of every code array and the K extent of the GEMMs that read
  // codes), mp = K_eff rounded up to 256 (the M extent of the CTA-pair GEMMs that produce one
  // value per kept component).  Compact index m is component kept_list[m].
  int kw = 64, mp = 256;
  bool has_mlp = true;    // correction layer present (false: linear codec)
  bool has_means = true;  // mean models present (false: unconditional zero-mean tables)
  bool has_synth = false; // decoder-side synthesis correction present
  // caller-owned parameter pointers (read at create)
  dckv_params p{};
  // derived, library-owned device buffers
  void *blk = nullptr;  // one allocation holding everything below but the vocabulary tables
  void *tab_blk = nullptr;  // the vocabulary tables (sized by kw, known after the keep mask)
  __half *a_y = nullptr;     // [2][mp][6144]  basis^T * 2^p_y, split hi/lo, kept components (zero rows after)
  __half *a_w2 = nullptr;    // [2][mp][256]   w2^T * 2^p_y, split, kept components
  __half *a_h = nullptr;     // [2][256][6144] w1^T * 2^p_h, split
  __half *a_inv = nullptr;   // [2][6144][kw]  (Delta_c basis[d][c]) * 2^p_inv, dims permuted, kept c
  __nv_bfloat16 *a_on = nullptr;  // [mp][2 kw]  odd mean model, neighbour blocks, kept in and out
  int8_t *t_even8 = nullptr;  // [vocab][kw]  clamp(round(embed @ w_even), +-127), kept components
  float *t_odd = nullptr;     // [vocab][kw]  embed @ w_odd[0:2048], kept components
  float *mub = nullptr;      // [2048]  mu @ basis
  float *mub_k = nullptr;    // [mp]    mu @ basis of kept components (0 after)
  float *delta_k = nullptr;  // [mp]    Delta of kept components (1 after)
  float *muw1 = nullptr;     // [256]   mu @ w1
  float *mu_perm = nullptr;  // [6144]  mu in the inverse GEMM's row order
  float *delta = nullptr;    // [2048]
  float *lapb = nullptr;     // [2048]  Laplace scales as given (the fit keeps dropped ones)
  uint8_t *keep = nullptr;   // [2048]
  uint8_t *scale = nullptr;  // [2048]
  int16_t *kept_list = nullptr;   // [2048] kept component indices (first k_eff valid)
  uint8_t *kept_scale = nullptr;  // [2048]
  uint16_t *cdf = nullptr;   // [64][510]  cumulative frequencies (cdf[510] = 65536 implied)
  uint16_t *lut = nullptr;   // [64][1024] decoder lookup (symbol holding slot b * 64)
  uint32_t *tail = nullptr;  // [64] lengths of the frequency-1 runs at both ends
  uint16_t *dcdf = nullptr;  // [64][512] cdf, padded with two zero entries (decoder)
  uint2 *cfm_tab = nullptr;  // [64][510] {cdf | (freq - 1) << 16, division multiplier} (encoder)
  int16_t *kidx = nullptr;   // [2048] kept index of a component, -1 if dropped
  double model_bits_per_row = 0.0;  // entropy of the kept components' tables
  float *dbg_ratio = nullptr;       // optional [rows][2048] export of the fp32 ratios y / Delta
  double *theta = nullptr;   // [128] RoPE frequencies
  // exact (fp64) refinement of codes near a half-step boundary: fp32 copies, c-major
  float *bt32 = nullptr;     // [2048][6144] basis^T
  float *w1t32 = nullptr;    // [256][6144]  w1^T
  float *w2t32 = nullptr;    // [2048][256]  w2^T
  double *mub64 = nullptr;   // [2048]  mu @ basis, fp64
  double *muw1_64 = nullptr; // [256]   mu @ w1, fp64
  // decoder-side synthesis (optional): split operands and fp32 copies for the exact fix-up
  __half *a_v1 = nullptr;    // [2][256][kw]  (Delta_c V1[c][h]) * 2^p_v1, split, kept c
  __half *a_v2 = nullptr;    // [2][6144][256]  V2[h][d] * 2^p_inv, split, dims permuted like a_inv
  float *v1t32 = nullptr;    // [256][2048]  V1^T
  float *v2_32 = nullptr;    // [256][6144]  V2
  float *zero256 = nullptr;  // [256] zeros (the synthesis hidden layer has no offset)
  int p_y = 0, p_h = 0, p_inv = 0, p_v1 = 0;  // power-of-two operand scales
  CUtensorMap map_ay2, map_aw2_2, map_aw2_1, map_ah2, map_ainv2, map_ainv1, map_aon1, map_av1, map_av2;
  // The inverse GEMM adds the lo half of its split operand for the first inv_lo_k compact
  // components only (a multiple of 64, at most kw): past them the lo half carries less than
  // INV_LO_THETA of the signal's rms under the codec's own Laplace model.
  int inv_lo_k = 0;
  // stage timing (optional; the events live in a per-thread log of the calling thread)
  int timing = 0;
};
