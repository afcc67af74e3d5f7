// dckv_epilogues.cuh -- fused epilogues of the codec's tcgen05 GEMMs.
//
// An epilogue runs on groups of 128 epilogue threads (EpiCtx); thread (ew, lane) owns
// output feature m = mt*128 + ew*32 + lane and walks its group's token-column chunks
// with tcgen05.ld.
#pragma once
#include "dckv_gemm.cuh"
#include "dckv_internal.cuh"

namespace dckv {

__device__ __forceinline__ float u2f(uint32_t u) { return __uint_as_float(u); }

// RoPE rotation for frequency index i at position pos: angle = pos * 1e7^(-2i/256),
// reduced modulo 2 pi in fp64, then CUDA's sincosf on the reduced fp32 angle.
__device__ __forceinline__ void rope_cs(int pos, int i, const double *theta, float &c, float &s) {
  const double ang = (double)pos * theta[i];
  const double k = rint(ang * 0.15915494309189535);  // 1 / (2 pi)
  double r = fma(-k, 6.283185307179586, ang);
  r = fma(-k, 2.4492935982947064e-16, r);
  sincosf((float)r, &s, &c);
}

// ------------------------------------------------------------------ plain fp32 store
// out[(n0 + n) * ld + m] = D  (per-vocabulary mean tables, GEMM self-test)
struct EpiStoreF32 {
  struct Params {
    float *out;
    int64_t ld;
    float scale;
    int m_valid = 1 << 30;  // features m >= m_valid are not stored
  };
  static constexpr int SMEM_BYTES = 0;
  __device__ __forceinline__ static void tile(const Params &p, const EpiCtx &cx) {
    const int m = cx.mt * GEMM_BM + cx.ew * 32 + cx.lane;
    for (int c0 = cx.grp * 32; c0 < cx.n_valid; c0 += 32 * cx.n_grp) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(cx.tacc + (uint32_t)c0, r);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (c0 + j < cx.n_valid && m < p.m_valid) p.out[(int64_t)(cx.n0 + c0 + j) * p.ld + m] = u2f(r[j]) * p.scale;
    }
  }
};

// ------------------------------------------------------------------ fp64 accumulation
// out[n][m] += D[m][n] in fp64 (the closed-form fit's normal-equation sums: the GEMM runs
// over a slice of calibration rows, fp32 in TMEM, and every slice is added in fp64).
// Lanes hold consecutive m, so the transposed store is coalesced; for a symmetric product
// (G = X^T X) the transpose is the same matrix.
struct EpiAccF64 {
  struct Params {
    double *out;
    int64_t ld;
  };
  static constexpr int SMEM_BYTES = 0;
  __device__ __forceinline__ static void tile(const Params &p, const EpiCtx &cx) {
    const int m = cx.mt * GEMM_BM + cx.ew * 32 + cx.lane;
    for (int c0 = cx.grp * 32; c0 < cx.n_valid; c0 += 32 * cx.n_grp) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(cx.tacc + (uint32_t)c0, r);
      double *o = p.out + (int64_t)(cx.n0 + c0) * p.ld + m;
      const int nv = min(32, cx.n_valid - c0);
      tmem_ld_wait();
#pragma unroll
      for (int h = 0; h < 32; h += 16) {
        double v[16];  // 16 loads before their stores: the compiler cannot tell that they do not alias
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = h + j < nv ? o[(int64_t)(h + j) * p.ld] : 0.0;
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (h + j < nv) o[(int64_t)(h + j) * p.ld] = v[j] + (double)u2f(r[h + j]);
      }
    }
  }
};

// ------------------------------------------------------------------ split-K part
// part[ks][n][m] = D[m][n] (fp32): one K part of a split-K product, summed afterwards in a
// fixed order by the consumer.  Lanes hold consecutive m, so the store is coalesced.
struct EpiPartF32 {
  struct Params {
    float *part;
    int64_t ld;         // M
    int64_t ks_stride;  // rows * M
  };
  static constexpr int SMEM_BYTES = 0;
  __device__ __forceinline__ static void tile(const Params &p, const EpiCtx &cx) {
    const int m = cx.mt * GEMM_BM + cx.ew * 32 + cx.lane;
    float *o = p.part + cx.ks * p.ks_stride + (int64_t)cx.n0 * p.ld + m;
    for (int c0 = cx.grp * 32; c0 < cx.n_valid; c0 += 32 * cx.n_grp) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(cx.tacc + (uint32_t)c0, r);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (c0 + j < cx.n_valid) o[(int64_t)(c0 + j) * p.ld] = u2f(r[j]);
    }
  }
};

// ------------------------------------------------------------------ correction layer 1
// h = D * 2^-p_h - (mu @ w1)[m];  g = GELU(h) (erf form);  G[row][m] = fp16(g),
// G[row][256 + m] = fp16(g - fp16(g))  (the hi/lo pair feeds the second layer's GEMM)
struct EpiGelu {
  struct Params {
    const float *muw1;
    float scale;
    __half *g;  // [rows][512]
  };
  static constexpr int SMEM_BYTES = 0;
  __device__ __forceinline__ static void tile(const Params &p, const EpiCtx &cx) {
    const int m = cx.mt * GEMM_BM + cx.ew * 32 + cx.lane;
    const float mw = p.muw1[m];
    for (int c0 = cx.grp * 32; c0 < cx.n_valid; c0 += 32 * cx.n_grp) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(cx.tacc + (uint32_t)c0, r);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (c0 + j < cx.n_valid) {
          const float h = u2f(r[j]) * p.scale - mw;
          const float g = 0.5f * h * (1.0f + erff(h * 0.70710678118654752f));
          const __half hi = __float2half_rn(g);
          const __half lo = __float2half_rn(g - __half2float(hi));
          __half *row = p.g + (int64_t)(cx.n0 + c0 + j) * (2 * N_HIDDEN);
          row[m] = hi;
          row[N_HIDDEN + m] = lo;
        }
      }
    }
  }
};

// The same layer on the chunk-accumulated CTA-pair kernel: the totals it hands over are the
// fp32 sums, in order, of the TMEM partials of consecutive K parts, the very sums that
// k_gelu_parts forms from the split-K kernel's parts, so G is bit-identical either way.
struct EpiGeluRegs {
  using Params = EpiGelu::Params;
  static constexpr int SMEM_BYTES = 16;
  __device__ __forceinline__ static void stage(const Params &, char *, int, int, int, int) {}
  template <int NC>
  __device__ __forceinline__ static void finish(const Params &p, const char *, const float (&tot)[NC], int mt, int n0,
                                                int n_valid, int col0, int ew, int lane) {
    const int m = mt * GEMM_BM + ew * 32 + lane;
    const float mw = p.muw1[m];
#pragma unroll
    for (int j = 0; j < NC; ++j) {
      const int col = col0 + j;
      if (col < n_valid) {
        const float h = tot[j] * p.scale - mw;
        const float g = 0.5f * h * (1.0f + erff(h * 0.70710678118654752f));
        const __half hi = __float2half_rn(g);
        const __half lo = __float2half_rn(g - __half2float(hi));
        __half *row = p.g + (int64_t)(n0 + col) * (2 * N_HIDDEN);
        row[m] = hi;
        row[N_HIDDEN + m] = lo;
      }
    }
  }
};

// ------------------------------------------------------------------ transform + quantiser
// y = D * 2^-p_y - (mu @ basis)[c];  q = round_half_even(y / Delta_c), 0 if dropped;
// q32[row][c] = q; even rows also write bf16(q) to their padded even row (the odd mean
// model's input).
struct EpiQuant {
  struct Params {
    const float *mub;         // [mp] (mu @ basis) of the kept components, compact order
    const float *delta;       // [mp] Delta of the kept components
    int k_eff;                // features m < k_eff are kept components; the rest give 0
    float scale;
    int32_t *q32;             // [rows][CODE_LD], compact columns
    __nv_bfloat16 *qe;        // [ne_pad][CODE_LD], compact columns
    const int32_t *row_edst;  // [rows]: padded even row or -1
  };
};

// Chunk-accumulated transform + quantiser: takes this thread's totals (NC columns from
// col0) from registers; codes whose fp32 ratio lies in the guard band around a half step
// are listed for exact fp64 recomputation (whole rows when the row is large).
struct EpiQuantRegs {
  struct Params {
    EpiQuant::Params q;
    const float *row_norm;   // [rows] |x|_2 of the coded row
    uint32_t *rowflag;       // [rows] 1 once the row is listed for full refinement
    uint32_t *el_bins;       // codes to refine, binned by component: el_bins[c * bin_cap + i] = row
    uint32_t *bin_count;     // [2048] codes listed per component
    uint32_t *full_list;     // rows to refine whole
    uint32_t *counters;      // [0] listed codes, [1] listed rows
    uint32_t bin_cap;
    float *dbg_ratio;        // optional export of the fp32 ratios (self-test), [rows][2048] by component
    const int16_t *kept_list;  // compact index -> component (for dbg_ratio)
  };
  __device__ static void list_row(const Params &p, int row) {
    if (atomicExch(&p.rowflag[row], 1u) == 0u) p.full_list[atomicAdd(&p.counters[1], 1u)] = (uint32_t)row;
  }
  __device__ static void flag(const Params &pp, int row, int c) {
    if (pp.row_norm[row] > REFINE_NORM_FULL) {
      list_row(pp, row);
    } else {
      const uint32_t idx = atomicAdd(&pp.bin_count[c], 1u);
      if (idx < pp.bin_cap) {
        pp.el_bins[(int64_t)c * pp.bin_cap + idx] = (uint32_t)row;
        atomicAdd(&pp.counters[0], 1u);
      } else {
        list_row(pp, row);  // a full bin: the whole row is recomputed instead
      }
    }
  }
  // per tile column: padded even row (or -1) and the guard-band width's row term
  static constexpr int SMEM_BYTES = GEMM_MAX_BN * 8;
  __device__ __forceinline__ static void stage(const Params &pp, char *buf, int n0, int n_valid, int tid,
                                               int nthreads) {
    int32_t *s_e = reinterpret_cast<int32_t *>(buf);
    float *s_w = reinterpret_cast<float *>(buf + GEMM_MAX_BN * 4);
    for (int j = tid; j < n_valid; j += nthreads) {
      s_e[j] = __ldg(pp.q.row_edst + n0 + j);
      s_w[j] = __ldg(pp.row_norm + n0 + j);
    }
  }
  template <int NC>
  __device__ __forceinline__ static void finish(const Params &pp, const char *buf, const float (&tot)[NC], int mt,
                                                int n0, int n_valid, int col0, int ew, int lane) {
    const EpiQuant::Params &p = pp.q;
    const int32_t *s_e = reinterpret_cast<const int32_t *>(buf);
    const float *s_w = reinterpret_cast<const float *>(buf + GEMM_MAX_BN * 4);
    // compact component index; features past k_eff (zero operands) store code 0 into columns
    // the readers ignore (mp <= CODE_LD)
    const int c = mt * GEMM_BM + ew * 32 + lane;
    const float mb = p.mub[c];
    const float dl = p.delta[c];
    const bool kp = c < p.k_eff;
    const float wk = REFINE_KAPPA / dl;
    uint32_t fm[(NC + 31) / 32];  // columns whose code goes to the exact recomputation
#pragma unroll
    for (int w = 0; w < (NC + 31) / 32; ++w) fm[w] = 0u;
#pragma unroll
    for (int j = 0; j < NC; ++j) {
      const int col = col0 + j;
      if (col < n_valid) {
        const int row = n0 + col;
        const float y = tot[j] * p.scale - mb;
        const float ratio = __fdiv_rn(y, dl);
        const int q = kp ? __float2int_rn(ratio) : 0;
        p.q32[(int64_t)row * CODE_LD + c] = q;
        const int e = s_e[col];
        if (e >= 0) p.qe[(int64_t)e * CODE_LD + c] = __float2bfloat16_rn((float)q);
        if (pp.dbg_ratio && kp) pp.dbg_ratio[(int64_t)row * N_COEF + pp.kept_list[c]] = ratio;
        const float w = wk * s_w[col] + REFINE_W0;
        if (kp && (0.5f - fabsf(ratio - rintf(ratio)) < w || !(fabsf(ratio) < 1.0e6f))) fm[j >> 5] |= 1u << (j & 31);
      }
    }
#pragma unroll
    for (int w = 0; w < (NC + 31) / 32; ++w) {
      uint32_t m = fm[w];
      while (m) {
        const int b = __ffs(m) - 1;
        m &= m - 1u;
        flag(pp, n0 + col0 + w * 32 + b, c);
      }
    }
  }
};

// ------------------------------------------------------------------ odd mean model
// mu = D + (embed @ w_odd[0:2048])[token][c]  (code units);  centre = clamp(round(mu), +-127);
// the table holds kept components only, compact index kc at column kc
// Tile columns are padded even rows e; column e is the odd row whose left neighbour is
// even row e (e_tok[e] = its token's row in the batch, or -1 where there is no odd row).
template <bool DEC>  // false: the encoder's centres; true: the decoder's odd codes
struct EpiMeanOdd {
  struct Params {
    const float *t_odd;      // [vocab][t_ld], kept components (compact)
    const int32_t *tok_ids;  // [tokens]
    const int32_t *e_tok;    // [ne_pad] token row of the odd row, -1 if none
    const int32_t *e_slot;   // [ne_pad] slot row of that odd row
    int t_ld;                // row stride of t_odd (kw)
    int8_t *cen8;            // [slots][k_eff]  (encoder: the odd centres)
    int k_eff;
    int vocab;
    // decoder: the odd codes themselves, code = centre + symbol - 254 (q16 != NULL); an
    // ESC symbol leaves its code to the escape patch and flags its chunk
    const uint16_t *syms;    // [slots][k_eff] decoded symbols
    __half *q16;             // [rows][CODE_LD], compact columns
    const int32_t *e_row;    // [ne_pad] natural coded row of that odd row
    const int32_t *slot_chunk;
    uint32_t *escflag;       // [chunks]
  };
  // per tile column: t_odd row offset (or -1), slot row and natural row (each group its own)
  static constexpr int SMEM_BYTES = 256 * 16;
  // columns per accumulator load: groups take 16-column chunks in turn (four groups of four
  // warps at 256-column tiles: four chunks per warp and tile)
  static constexpr int CW = 16;
  __device__ __forceinline__ static void tile(const Params &p, const EpiCtx &cx) {
    int64_t *s_row = reinterpret_cast<int64_t *>(cx.scratch);
    int32_t *s_slot = reinterpret_cast<int32_t *>(cx.scratch + 256 * 8);
    int32_t *s_nat = reinterpret_cast<int32_t *>(cx.scratch + 256 * 12);
    const int n_valid = cx.n_valid;
    constexpr bool dec = DEC;
    for (int j = cx.et; j < n_valid; j += 128) {
      const int ti = __ldg(p.e_tok + cx.n0 + j);
      int64_t off = -1;
      if (ti >= 0) {
        const int tok = min(max(__ldg(p.tok_ids + ti), 0), p.vocab - 1);
        off = (int64_t)tok * p.t_ld;
      }
      s_row[j] = off;
      s_slot[j] = __ldg(p.e_slot + cx.n0 + j);
      if (dec) s_nat[j] = __ldg(p.e_row + cx.n0 + j);
    }
    named_bar_sync(cx.bar, 128);
    const int kc0 = cx.mt * GEMM_BM + cx.ew * 32 + cx.lane;  // compact index of this thread's feature
    const int kc = kc0 < p.k_eff ? kc0 : -1;
    for (int c0 = cx.grp * CW; c0 < n_valid; c0 += CW * cx.n_grp) {
      uint32_t r[CW];
      tmem_ld_32x32b_x16(cx.tacc + (uint32_t)c0, r);
      float tv[CW];
      uint16_t sv[DEC ? CW : 1];
#pragma unroll
      for (int j = 0; j < CW; ++j) {  // independent loads, issued together
        const int64_t off = (kc >= 0 && c0 + j < n_valid) ? s_row[c0 + j] : -1;
        tv[j] = off >= 0 ? __ldg(p.t_odd + off + kc) : 0.f;
        if constexpr (DEC) sv[j] = off >= 0 ? __ldg(p.syms + (int64_t)s_slot[c0 + j] * p.k_eff + kc) : (uint16_t)0;
      }
      tmem_ld_wait();
      if (kc < 0) continue;
#pragma unroll
      for (int j = 0; j < CW; ++j) {
        if (c0 + j < n_valid && s_row[c0 + j] >= 0) {
          const float mu = u2f(r[j]) + tv[j];
          const float cen = fminf(fmaxf(rintf(mu), -(float)ESC_LIMIT), (float)ESC_LIMIT);
          if constexpr (!DEC) {
            p.cen8[(int64_t)s_slot[c0 + j] * p.k_eff + kc] = (int8_t)cen;
          } else if (sv[j] == ESC_SYM) {
            p.escflag[__ldg(p.slot_chunk + s_slot[c0 + j])] = 1u;
          } else {
            p.q16[(int64_t)s_nat[c0 + j] * CODE_LD + kc] = __float2half_rn((float)((int)sv[j] - R_MAX + (int)cen));
          }
        }
      }
    }
    named_bar_sync(cx.bar, 128);  // the metadata is rewritten by the next tile
  }
};

// Output feature order of the inverse GEMM: M tile mt covers head vector hv = mt / 2
// (hv = (layer*2 + kv)*2 + head) and the 64-dim quarter `half` = mt % 2 of both RoPE
// halves: rows 0..63 are dims half*64 + r, rows 64..127 are dims 128 + half*64 + r - 64,
// so every rotate-half pair (d, d + 128) sits in one tile, 64 rows apart.
__host__ __device__ __forceinline__ int inv_row_to_dim(int p) {
  const int mt = p >> 7, r = p & 127;
  const int hv = mt >> 1, half = mt & 1;
  return hv * HEAD_DIM + (r < 64 ? half * 64 + r : 128 + half * 64 + (r - 64));
}

// ------------------------------------------------------------------ inverse + RoPE + scatter
// x = D * 2^-p_inv + mu[d]; keys get RoPE (rotate-half, base 1e7, position in prompt) with
// cos / sin from a per-call table; bf16 round-to-nearest-even; coalesced 16-byte stores
// into [6][tokens][2][256].  Chunks of 16 columns; the RoPE partner (row +-64) is read
// through shared memory.
struct EpiInverse {
  struct Params {
    const float *mu_perm;
    float scale;
    const float2 *rope;      // [positions][128] (cos, sin) of position * theta_i
    const int32_t *row_tok;  // [rows] token index in the batch
    const int32_t *row_pos;  // [rows] position within the prompt
    __nv_bfloat16 *k_out, *v_out;
    int64_t n_tokens;
  };
  static constexpr int CW = 16;
  static constexpr int XCH_LD = CW + 1;
  static constexpr int SMEM_BYTES = 128 * XCH_LD * 4 + CW * 128 * 2;
  __device__ __forceinline__ static void tile(const Params &p, const EpiCtx &cx) {
    float *xch = reinterpret_cast<float *>(cx.scratch);
    __nv_bfloat16 *ob = reinterpret_cast<__nv_bfloat16 *>(cx.scratch + 128 * XCH_LD * 4);
    const int mt = cx.mt, n0 = cx.n0, n_valid = cx.n_valid, et = cx.et;
    const int ml = cx.ew * 32 + cx.lane;
    const int hv = mt >> 1, half = mt & 1;
    const int layer = hv >> 2, kv = (hv >> 1) & 1, head = hv & 1;
    const bool first = ml < 64;
    const int partner = first ? ml + 64 : ml - 64;
    const int fi = half * 64 + (ml & 63);  // frequency index of this row's pair
    const float mu = p.mu_perm[mt * GEMM_BM + ml];
    __nv_bfloat16 *dst_base = kv == 0 ? p.k_out : p.v_out;
    for (int c0 = cx.grp * CW; c0 < n_valid; c0 += CW * cx.n_grp) {
      uint32_t r[CW];
      tmem_ld_32x32b_x16(cx.tacc + (uint32_t)c0, r);
      tmem_ld_wait();
      float v[CW];
#pragma unroll
      for (int j = 0; j < CW; ++j) v[j] = u2f(r[j]) * p.scale + mu;
      if (kv == 0) {
        float2 cs[CW];
#pragma unroll
        for (int j = 0; j < CW; ++j) {
          const int row = min(n0 + c0 + j, n0 + n_valid - 1);
          cs[j] = __ldg(p.rope + (int64_t)__ldg(p.row_pos + row) * 128 + fi);
          xch[ml * XCH_LD + j] = v[j];
        }
        named_bar_sync(cx.bar, 128);
#pragma unroll
        for (int j = 0; j < CW; ++j) {
          const float pv = xch[partner * XCH_LD + j];
          v[j] = first ? (v[j] * cs[j].x - pv * cs[j].y) : (v[j] * cs[j].x + pv * cs[j].y);
        }
      }
#pragma unroll
      for (int j = 0; j < CW; ++j) ob[j * 128 + ml] = __float2bfloat16_rn(v[j]);
      named_bar_sync(cx.bar, 128);
      // CW tokens x 2 segments x 8 sixteen-byte pieces over 128 threads
#pragma unroll
      for (int it = 0; it < CW / 8; ++it) {
        const int qid = et + 128 * it;
        const int j = qid >> 4, sub = qid & 15, seg = sub >> 3, w = sub & 7;
        if (c0 + j < n_valid) {
          const int row = n0 + c0 + j;
          const int64_t tok = __ldg(p.row_tok + row);
          const int64_t off = ((layer * p.n_tokens + tok) * 2 + head) * HEAD_DIM + seg * 128 + half * 64 + w * 8;
          *reinterpret_cast<uint4 *>(dst_base + off) = *reinterpret_cast<const uint4 *>(ob + j * 128 + seg * 64 + w * 8);
        }
      }
      named_bar_sync(cx.bar, 128);
    }
  }
};

}  // namespace dckv
