// dckv_epilogues.cuh -- fused epilogues of the codec's tcgen05 GEMMs.
//
// Each epilogue runs on the 128 epilogue threads of gemm_kernel; thread (ew, lane) owns
// output feature m = mt*128 + ew*32 + lane and walks the tile's token columns 32 at a
// time with tcgen05.ld.
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
  };
  static constexpr int SMEM_BYTES = 0;
  __device__ static void tile(const Params &p, char *, int mt, int n0, int n_valid, int bn, uint32_t tacc, int ew,
                              int lane, int) {
    const int m = mt * GEMM_BM + ew * 32 + lane;
    for (int c0 = 0; c0 < n_valid; c0 += 32) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(tacc + (uint32_t)c0, r);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (c0 + j < n_valid) p.out[(int64_t)(n0 + c0 + j) * p.ld + m] = u2f(r[j]) * p.scale;
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
  __device__ static void tile(const Params &p, char *, int mt, int n0, int n_valid, int bn, uint32_t tacc, int ew,
                              int lane, int) {
    const int m = mt * GEMM_BM + ew * 32 + lane;
    const float mw = p.muw1[m];
    for (int c0 = 0; c0 < n_valid; c0 += 32) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(tacc + (uint32_t)c0, r);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (c0 + j < n_valid) {
          const float h = u2f(r[j]) * p.scale - mw;
          const float g = 0.5f * h * (1.0f + erff(h * 0.70710678118654752f));
          const __half hi = __float2half_rn(g);
          const __half lo = __float2half_rn(g - __half2float(hi));
          __half *row = p.g + (int64_t)(n0 + c0 + j) * (2 * N_HIDDEN);
          row[m] = hi;
          row[N_HIDDEN + m] = lo;
        }
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
    const float *mub;
    const float *delta;
    const uint8_t *keep;
    float scale;
    int32_t *q32;             // [rows][2048]
    __nv_bfloat16 *qe;        // [ne_pad][2048]
    const int32_t *row_edst;  // [rows]: padded even row or -1
  };
  static constexpr int SMEM_BYTES = 0;
  __device__ static void tile(const Params &p, char *, int mt, int n0, int n_valid, int bn, uint32_t tacc, int ew,
                              int lane, int) {
    const int c = mt * GEMM_BM + ew * 32 + lane;
    const float mb = p.mub[c];
    const float dl = p.delta[c];
    const bool kp = p.keep[c] != 0;
    for (int c0 = 0; c0 < n_valid; c0 += 32) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(tacc + (uint32_t)c0, r);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (c0 + j < n_valid) {
          const int row = n0 + c0 + j;
          const float y = u2f(r[j]) * p.scale - mb;
          const int q = kp ? __float2int_rn(__fdiv_rn(y, dl)) : 0;
          p.q32[(int64_t)row * N_COEF + c] = q;
          const int e = p.row_edst[row];
          if (e >= 0) p.qe[(int64_t)e * N_COEF + c] = __float2bfloat16_rn((float)q);
        }
      }
    }
  }
};

// Chunk-accumulated form of the same epilogue: the thread's 128 totals (columns
// c_begin .. c_begin + 127 of the tile) are already summed in fp32 registers.
struct EpiQuantTotals {
  using Params = EpiQuant::Params;
  __device__ static void finish(const Params &p, int mt, int n0, int n_valid, int c_begin, const float (&tot)[128],
                                int ew, int lane) {
    const int c = mt * GEMM_BM + ew * 32 + lane;
    const float mb = p.mub[c];
    const float dl = p.delta[c];
    const bool kp = p.keep[c] != 0;
#pragma unroll
    for (int j = 0; j < 128; ++j) {
      const int col = c_begin + j;
      if (col < n_valid) {
        const int row = n0 + col;
        const float y = tot[j] * p.scale - mb;
        const int q = kp ? __float2int_rn(__fdiv_rn(y, dl)) : 0;
        p.q32[(int64_t)row * N_COEF + c] = q;
        const int e = p.row_edst[row];
        if (e >= 0) p.qe[(int64_t)e * N_COEF + c] = __float2bfloat16_rn((float)q);
      }
    }
  }
};

// ------------------------------------------------------------------ odd mean model
// mu = D + (embed @ w_odd[0:2048])[token][c]  (code units);  centre = clamp(round(mu), +-127)
// Tile columns are padded even rows e; column e is the odd row whose left neighbour is
// even row e (e_tok[e] = its token's row in the batch, or -1 where there is no odd row).
struct EpiMeanOdd {
  struct Params {
    const float *t_odd;      // [vocab][2048]
    const int32_t *tok_ids;  // [tokens]
    const int32_t *e_tok;    // [ne_pad]
    int8_t *c_odd;           // [ne_pad][2048]
    int vocab;
  };
  static constexpr int SMEM_BYTES = 0;
  __device__ static void tile(const Params &p, char *, int mt, int n0, int n_valid, int bn, uint32_t tacc, int ew,
                              int lane, int) {
    const int c = mt * GEMM_BM + ew * 32 + lane;
    for (int c0 = 0; c0 < n_valid; c0 += 32) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(tacc + (uint32_t)c0, r);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (c0 + j < n_valid) {
          const int e = n0 + c0 + j;
          const int ti = p.e_tok[e];
          if (ti >= 0) {
            int tok = p.tok_ids[ti];
            tok = min(max(tok, 0), p.vocab - 1);
            const float mu = u2f(r[j]) + p.t_odd[(int64_t)tok * N_COEF + c];
            const float cen = fminf(fmaxf(rintf(mu), -(float)ESC_LIMIT), (float)ESC_LIMIT);
            p.c_odd[(int64_t)e * N_COEF + c] = (int8_t)cen;
          }
        }
      }
    }
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
// x = D * 2^-p_inv + mu[d]; keys get RoPE (rotate-half, base 1e7, position in prompt);
// bf16 round-to-nearest-even; coalesced 16-byte stores into [6][tokens][2][256].
struct EpiInverse {
  struct Params {
    const float *mu_perm;
    float scale;
    const double *theta;
    const int32_t *row_tok;  // [rows] token index in the batch
    const int32_t *row_pos;  // [rows] position within the prompt
    __nv_bfloat16 *k_out, *v_out;
    int64_t n_tokens;
  };
  static constexpr int XCH_LD = 33;
  static constexpr int SMEM_BYTES = 128 * XCH_LD * 4 + 32 * 128 * 2;
  __device__ static void tile(const Params &p, char *scratch, int mt, int n0, int n_valid, int bn, uint32_t tacc,
                              int ew, int lane, int et) {
    float *xch = reinterpret_cast<float *>(scratch);
    __nv_bfloat16 *ob = reinterpret_cast<__nv_bfloat16 *>(scratch + 128 * XCH_LD * 4);
    const int ml = ew * 32 + lane;
    const int hv = mt >> 1, half = mt & 1;
    const int layer = hv >> 2, kv = (hv >> 1) & 1, head = hv & 1;
    const bool first = ml < 64;
    const int partner = first ? ml + 64 : ml - 64;
    const int fi = half * 64 + (ml & 63);  // frequency index of this row's pair
    const float mu = p.mu_perm[mt * GEMM_BM + ml];
    __nv_bfloat16 *dst_base = kv == 0 ? p.k_out : p.v_out;
    for (int c0 = 0; c0 < n_valid; c0 += 32) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(tacc + (uint32_t)c0, r);
      tmem_ld_wait();
      float v[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = u2f(r[j]) * p.scale + mu;
      if (kv == 0) {
#pragma unroll
        for (int j = 0; j < 32; ++j) xch[ml * XCH_LD + j] = v[j];
        named_bar_sync(1, 128);
#pragma unroll 4
        for (int j = 0; j < 32; ++j) {
          const float pv = xch[partner * XCH_LD + j];
          const int row = min(n0 + c0 + j, n0 + n_valid - 1);
          float cs, sn;
          rope_cs(p.row_pos[row], fi, p.theta, cs, sn);
          v[j] = first ? (v[j] * cs - pv * sn) : (v[j] * cs + pv * sn);
        }
      }
#pragma unroll
      for (int j = 0; j < 32; ++j) ob[j * 128 + ml] = __float2bfloat16_rn(v[j]);
      named_bar_sync(1, 128);
      // 32 tokens x 2 segments x 8 sixteen-byte chunks = 512 stores over 128 threads
#pragma unroll
      for (int it = 0; it < 4; ++it) {
        const int qid = et + 128 * it;
        const int j = qid >> 4, sub = qid & 15, seg = sub >> 3, w = sub & 7;
        if (c0 + j < n_valid) {
          const int row = n0 + c0 + j;
          const int64_t tok = p.row_tok[row];
          const int64_t off = ((layer * p.n_tokens + tok) * 2 + head) * HEAD_DIM + seg * 128 + half * 64 + w * 8;
          *reinterpret_cast<uint4 *>(dst_base + off) = *reinterpret_cast<const uint4 *>(ob + j * 128 + seg * 64 + w * 8);
        }
      }
      named_bar_sync(1, 128);
    }
  }
};

}  // namespace dckv
