// dckv_rans.cuh -- warp-interleaved rANS encode / decode, escape handling, scan and
// compaction kernels of the DCKV codec.
//
// Coder (per chunk, one warp): 32 interleaved 32-bit states (lane j codes symbols
// i = 32 t + j), 16-bit frequency precision, 16-bit renormalisation words, states in
// [2^16, 2^32).  Symbols of a chunk run row-major over its rows and the kept components;
// symbol = ESC (509) if |q| > 127, else q - centre + 254.  The encoder walks steps
// t = T-1..0; at each step the lanes that must renormalise emit one word each, placed
// with a ballot / popcount so that the decoder, walking t = 0..T-1 and reading words in
// lane order, consumes exactly what was emitted.
#pragma once
#include "dckv_internal.cuh"
#include "dckv_ptx.cuh"

namespace dckv {

constexpr int RANS_WARPS = 8;  // chunks per block
constexpr int CDF_SMEM_BYTES = N_SCALES * (N_SYM) * 2;

__device__ __forceinline__ void load_cdf_smem(uint16_t *s_cdf, const uint16_t *g_cdf) {
  const uint4 *src = reinterpret_cast<const uint4 *>(g_cdf);
  uint4 *dst = reinterpret_cast<uint4 *>(s_cdf);
  for (int i = threadIdx.x; i < CDF_SMEM_BYTES / 16; i += blockDim.x) dst[i] = src[i];
  __syncthreads();
}

__device__ __forceinline__ uint32_t cdf_at(const uint16_t *tab, int k) { return k < N_SYM ? tab[k] : PREC_TOTAL; }

// centre of an even row: clamp(round(T_even[token][c]), +-127)
__device__ __forceinline__ int even_centre(const float *t_even, int tok, int c) {
  const float mu = t_even[(int64_t)tok * N_COEF + c];
  return (int)fminf(fmaxf(rintf(mu), -(float)ESC_LIMIT), (float)ESC_LIMIT);
}

struct RansEncArgs {
  const ChunkDesc *chunks;
  const PromptInfo *prompts;
  int n_chunks;
  int k_eff;
  const int16_t *kept_list;
  const uint8_t *kept_scale;
  const uint16_t *cdf;
  const int32_t *q32;       // [rows][2048]
  const float *t_even;      // [vocab][2048]
  const int32_t *tok_ids;   // [tokens]
  const int8_t *c_odd;      // [ne_pad][2048]
  int vocab;
  uint16_t *words;          // word scratch: chunk c owns [sym_base, sym_base + S)
  uint32_t *states;         // [chunks][32]
  uint32_t *nwords;         // [chunks] words emitted
  uint32_t *nesc;           // [chunks] escapes
};

__global__ void __launch_bounds__(RANS_WARPS * 32) rans_encode_kernel(RansEncArgs a) {
  extern __shared__ __align__(16) uint8_t sm[];
  uint16_t *s_cdf = reinterpret_cast<uint16_t *>(sm);
  load_cdf_smem(s_cdf, a.cdf);
  const int lane = threadIdx.x & 31;
  const int ci = blockIdx.x * RANS_WARPS + (threadIdx.x >> 5);
  if (ci >= a.n_chunks) return;
  const ChunkDesc cd = a.chunks[ci];
  const PromptInfo pi = a.prompts[cd.prompt];
  const int K = a.k_eff;
  const int64_t S = (int64_t)cd.nrows * K;
  const int64_t T = (S + 31) / 32;
  uint16_t *wslot = a.words + cd.sym_base;
  int64_t pos = S;  // words are placed downwards from the end of the slot
  uint32_t x = RANS_L;
  uint32_t n_esc = 0;
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int64_t t = T - 1; t >= 0; --t) {
    const int64_t i = t * 32 + lane;
    const bool valid = i < S;
    uint32_t f = 1, c = 0;
    bool is_esc = false;
    if (valid) {
      const int rl = (int)(i / K);
      const int k = (int)(i - (int64_t)rl * K);
      const int comp = a.kept_list[k];
      const int s = a.kept_scale[k];
      const int j = cd.j0 + rl;
      const int64_t row = (int64_t)pi.row_base + 2 * j + cd.parity;
      const int q = a.q32[row * N_COEF + comp];
      int sym;
      if (q > ESC_LIMIT || q < -ESC_LIMIT) {
        sym = ESC_SYM;
        is_esc = true;
      } else {
        int cen;
        if (cd.parity == 0) {
          int tok = a.tok_ids[pi.tok_base + HEAD_KEPT + 2 * j];
          tok = min(max(tok, 0), a.vocab - 1);
          cen = even_centre(a.t_even, tok, comp);
        } else {
          cen = a.c_odd[(int64_t)(pi.ebase + j) * N_COEF + comp];
        }
        sym = q - cen + R_MAX;
      }
      const uint16_t *tab = s_cdf + s * N_SYM;
      c = tab[sym];
      f = cdf_at(tab, sym + 1) - c;
    }
    const bool emit = valid && x >= (f << 16);
    const uint32_t m = __ballot_sync(0xffffffffu, emit);
    const int nm = __popc(m);
    if (emit) {
      wslot[pos - nm + __popc(m & lt_mask)] = (uint16_t)(x & 0xFFFFu);
      x >>= 16;
    }
    pos -= nm;
    if (valid) x = ((x / f) << 16) + (x % f) + c;
    n_esc += __popc(__ballot_sync(0xffffffffu, is_esc));
  }
  a.states[(int64_t)ci * 32 + lane] = x;
  if (lane == 0) {
    a.nwords[ci] = (uint32_t)(S - pos);
    a.nesc[ci] = n_esc;
  }
}

// Exclusive scan of chunk section sizes (one block); writes the chunk table and header.
struct ScanArgs {
  int n_chunks;
  const uint32_t *nwords, *nesc;
  uint32_t *offs;  // [n_chunks + 1] workspace copy
  uint8_t *blob;
  uint64_t blob_cap;
  uint64_t off_kept, off_streams;
  const PromptInfo *prompts;
  int batch;
  int chunk_rows, k_eff, n_chunks_e, n_chunks_o;
  int64_t n_kept;
  uint64_t *blob_size_dev;
  int32_t *status;
};

__global__ void __launch_bounds__(1024) scan_kernel(ScanArgs a) {
  __shared__ uint64_t warp_sums[32];
  __shared__ uint64_t carry;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < a.n_chunks; base += 1024) {
    const int c = base + tid;
    uint64_t sz = 0;
    if (c < a.n_chunks) sz = ((uint64_t)CHUNK_FIXED_BYTES + 8ull * a.nesc[c] + 2ull * a.nwords[c] + 3ull) & ~3ull;
    uint64_t v = sz;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint64_t u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    if (lane == 31) warp_sums[wid] = v;
    __syncthreads();
    if (wid == 0) {
      uint64_t w = warp_sums[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint64_t u = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += u;
      }
      warp_sums[lane] = w;  // inclusive
    }
    __syncthreads();
    const uint64_t excl = carry + (wid ? warp_sums[wid - 1] : 0) + v - sz;
    if (c < a.n_chunks) a.offs[c] = (uint32_t)excl;
    __syncthreads();
    if (tid == 1023) carry = excl + sz;
    __syncthreads();
  }
  const uint64_t streams = carry;
  const uint64_t total = a.off_streams + streams;
  if (tid == 0) {
    a.offs[a.n_chunks] = (uint32_t)streams;
    if (streams >= (1ull << 32)) atomicExch(a.status, DCKV_ECAPACITY);
    if (total > a.blob_cap) atomicExch(a.status, DCKV_ECAPACITY);
    *a.blob_size_dev = total;
  }
  __syncthreads();
  if (a.off_kept > a.blob_cap) return;
  // header
  if (tid == 0) {
    uint8_t *h = a.blob;
    uint32_t *h32 = reinterpret_cast<uint32_t *>(h);
    h32[0] = MAGIC;
    reinterpret_cast<uint16_t *>(h)[2] = (uint16_t)VERSION;
    reinterpret_cast<uint16_t *>(h)[3] = (uint16_t)a.chunk_rows;
    h32[2] = (uint32_t)a.batch;
    h32[3] = (uint32_t)N_COEF;
    h32[4] = (uint32_t)a.k_eff;
    h32[5] = (uint32_t)a.n_chunks_e;
    h32[6] = (uint32_t)a.n_chunks_o;
    h32[7] = (uint32_t)a.n_kept;
    uint64_t *h64 = reinterpret_cast<uint64_t *>(h + 32);
    h64[0] = total;
    h64[1] = a.off_streams;
    h64[2] = a.off_kept;
    h64[3] = 0;
  }
  uint32_t *pt = reinterpret_cast<uint32_t *>(a.blob + HEADER_BYTES);
  for (int b = tid; b < a.batch; b += 1024) pt[b] = (uint32_t)a.prompts[b].N;
  uint32_t *ct = pt + a.batch;
  for (int c = tid; c <= a.n_chunks; c += 1024) ct[c] = a.offs[c];
  // zero pad up to the kept rows
  const uint64_t tab_end = HEADER_BYTES + 4ull * (a.batch + a.n_chunks + 1);
  for (uint64_t o = tab_end + tid; o < a.off_kept; o += 1024) a.blob[o] = 0;
}

// Writes each chunk section: states, escape count, escaped codes (symbol order), words.
struct CompactArgs {
  const ChunkDesc *chunks;
  const PromptInfo *prompts;
  int n_chunks;
  int k_eff;
  const int16_t *kept_list;
  const int32_t *q32;
  const uint16_t *words;
  const uint32_t *states, *nwords, *nesc, *offs;
  uint8_t *blob;
  uint64_t blob_cap, off_streams;
};

__global__ void __launch_bounds__(RANS_WARPS * 32) compact_kernel(CompactArgs a) {
  const int lane = threadIdx.x & 31;
  const int ci = blockIdx.x * RANS_WARPS + (threadIdx.x >> 5);
  if (ci >= a.n_chunks) return;
  const uint64_t beg = a.off_streams + a.offs[ci];
  const uint64_t end = a.off_streams + a.offs[ci + 1];
  if (end > a.blob_cap) return;  // capacity error already reported by the scan
  uint8_t *sec = a.blob + beg;
  const uint32_t ne = a.nesc[ci], nw = a.nwords[ci];
  reinterpret_cast<uint32_t *>(sec)[lane] = a.states[(int64_t)ci * 32 + lane];
  if (lane == 0) reinterpret_cast<uint32_t *>(sec)[32] = ne;
  const ChunkDesc cd = a.chunks[ci];
  const PromptInfo pi = a.prompts[cd.prompt];
  const int K = a.k_eff;
  const int64_t S = (int64_t)cd.nrows * K;
  // escaped codes in symbol order, 64 raw bits each (sections are 4-byte aligned)
  if (ne) {
    uint32_t *ev = reinterpret_cast<uint32_t *>(sec + CHUNK_FIXED_BYTES);
    uint32_t ep = 0;
    const uint32_t lt_mask = (1u << lane) - 1u;
    for (int64_t i0 = 0; i0 < S && ep < ne; i0 += 32) {
      const int64_t i = i0 + lane;
      int q = 0;
      bool esc = false;
      if (i < S) {
        const int rl = (int)(i / K);
        const int k = (int)(i - (int64_t)rl * K);
        const int64_t row = (int64_t)pi.row_base + 2 * (cd.j0 + rl) + cd.parity;
        q = a.q32[row * N_COEF + a.kept_list[k]];
        esc = q > ESC_LIMIT || q < -ESC_LIMIT;
      }
      const uint32_t m = __ballot_sync(0xffffffffu, esc);
      if (esc) {
        const uint32_t slot = ep + __popc(m & lt_mask);
        const int64_t v = (int64_t)q;
        ev[2 * slot] = (uint32_t)(uint64_t)v;
        ev[2 * slot + 1] = (uint32_t)((uint64_t)v >> 32);
      }
      ep += __popc(m);
    }
  }
  // words (decoder order) follow the escapes; then zero padding to 4 bytes
  uint16_t *wd = reinterpret_cast<uint16_t *>(sec + CHUNK_FIXED_BYTES + 8ull * ne);
  const uint16_t *ws = a.words + cd.sym_base + (S - nw);
  for (uint32_t w = lane; w < nw; w += 32) wd[w] = ws[w];
  const uint64_t used = CHUNK_FIXED_BYTES + 8ull * ne + 2ull * nw;
  if (lane == 0 && (end - beg) > used) wd[nw] = 0;
}

// Decodes one pass (parity) of chunks: one warp per chunk.  Writes q as fp16 (exact for
// |q| < 2048) for the inverse GEMM, bf16(q) into padded even rows for the odd mean model,
// and exact int32 values of codes with |q| >= 2048 (their rows are listed for a fix-up).
struct RansDecArgs {
  const ChunkDesc *chunks;
  const PromptInfo *prompts;
  int chunk0, n_chunks;  // this pass: chunks [chunk0, chunk0 + n_chunks)
  int k_eff;
  const int16_t *kept_list;
  const uint8_t *kept_scale;
  const uint16_t *cdf;
  const float *t_even;
  const int32_t *tok_ids;
  const int8_t *c_odd;
  int vocab;
  const uint8_t *blob;
  uint64_t off_streams;
  const uint32_t *offs;  // chunk table inside the blob
  __half *q16;           // [rows][2048]
  __nv_bfloat16 *qe;     // [ne_pad][2048]
  int32_t *qbig;         // [rows][2048], written only where |q| >= 2048
  uint32_t *bigflag;     // [rows]
  int32_t *biglist;      // [rows]
  uint32_t *bigcount;
  const int32_t *valid;  // header check result (1 = ok)
  int32_t *status;
};

__global__ void __launch_bounds__(RANS_WARPS * 32) rans_decode_kernel(RansDecArgs a) {
  extern __shared__ __align__(16) uint8_t sm[];
  uint16_t *s_cdf = reinterpret_cast<uint16_t *>(sm);
  if (*a.valid != 1) return;
  load_cdf_smem(s_cdf, a.cdf);
  const int lane = threadIdx.x & 31;
  const int wi = blockIdx.x * RANS_WARPS + (threadIdx.x >> 5);
  if (wi >= a.n_chunks) return;
  const int ci = a.chunk0 + wi;
  const ChunkDesc cd = a.chunks[ci];
  const PromptInfo pi = a.prompts[cd.prompt];
  const int K = a.k_eff;
  const int64_t S = (int64_t)cd.nrows * K;
  const int64_t T = (S + 31) / 32;
  const uint64_t beg = a.off_streams + a.offs[ci];
  const uint64_t end = a.off_streams + a.offs[ci + 1];
  const uint8_t *sec = a.blob + beg;
  const uint32_t ne = reinterpret_cast<const uint32_t *>(sec)[32];
  bool bad = (end - beg) < CHUNK_FIXED_BYTES || (uint64_t)CHUNK_FIXED_BYTES + 8ull * ne > (end - beg);
  if (__any_sync(0xffffffffu, bad)) {
    if (lane == 0) atomicExch(a.status, DCKV_ECORRUPT);
    return;
  }
  uint32_t x = reinterpret_cast<const uint32_t *>(sec)[lane];
  const uint32_t *ev = reinterpret_cast<const uint32_t *>(sec + CHUNK_FIXED_BYTES);
  const uint16_t *wd = reinterpret_cast<const uint16_t *>(sec + CHUNK_FIXED_BYTES + 8ull * ne);
  const int64_t n_wd = (int64_t)((end - beg) - CHUNK_FIXED_BYTES - 8ull * ne) / 2;
  int64_t wp = 0;
  uint32_t ep = 0;
  const uint32_t lt_mask = (1u << lane) - 1u;
  if (x < RANS_L) bad = true;
  for (int64_t t = 0; t < T; ++t) {
    const int64_t i = t * 32 + lane;
    const bool valid = i < S;
    int q = 0, comp = 0;
    int64_t row = 0;
    bool need = false, is_esc = false;
    if (valid) {
      const int rl = (int)(i / K);
      const int k = (int)(i - (int64_t)rl * K);
      comp = a.kept_list[k];
      const int s = a.kept_scale[k];
      const int j = cd.j0 + rl;
      row = (int64_t)pi.row_base + 2 * j + cd.parity;
      const uint16_t *tab = s_cdf + s * N_SYM;
      const uint32_t slot = x & 0xFFFFu;
      int lo = 0, hi = N_SYM;  // invariant: tab[lo] <= slot < cdf(hi); 9 halvings
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (tab[mid] <= slot) lo = mid; else hi = mid;
      }
      const uint32_t c = tab[lo];
      const uint32_t f = cdf_at(tab, lo + 1) - c;
      x = f * (x >> 16) + slot - c;
      need = x < RANS_L;
      if (lo == ESC_SYM) {
        is_esc = true;
      } else {
        int cen;
        if (cd.parity == 0) {
          int tok = a.tok_ids[pi.tok_base + HEAD_KEPT + 2 * j];
          tok = min(max(tok, 0), a.vocab - 1);
          cen = even_centre(a.t_even, tok, comp);
        } else {
          cen = a.c_odd[(int64_t)(pi.ebase + j) * N_COEF + comp];
        }
        q = lo - R_MAX + cen;
      }
    }
    const uint32_t m = __ballot_sync(0xffffffffu, need);
    if (need) {
      const int64_t w = wp + __popc(m & lt_mask);
      if (w < n_wd) x = (x << 16) | wd[w]; else bad = true;
    }
    wp += __popc(m);
    const uint32_t me = __ballot_sync(0xffffffffu, is_esc);
    if (is_esc) {
      const uint32_t e = ep + __popc(me & lt_mask);
      if (e < ne) {
        const uint64_t v = (uint64_t)ev[2 * e] | ((uint64_t)ev[2 * e + 1] << 32);
        const int64_t sv = (int64_t)v;
        q = (int)max(min(sv, (int64_t)INT32_MAX), (int64_t)INT32_MIN);
        if (sv >= -ESC_LIMIT && sv <= ESC_LIMIT) bad = true;  // not an escape value
      } else {
        bad = true;
      }
    }
    ep += __popc(me);
    if (__any_sync(0xffffffffu, bad)) break;
    if (valid) {
      a.q16[row * N_COEF + comp] = __float2half_rn((float)q);
      if (cd.parity == 0) {
        const int j = (int)((row - pi.row_base) >> 1);
        a.qe[(int64_t)(pi.ebase + j) * N_COEF + comp] = __float2bfloat16_rn((float)q);
      }
      if (q >= BIG_CODE || q <= -BIG_CODE) {
        a.qbig[row * N_COEF + comp] = q;
        if (atomicExch(&a.bigflag[row], 1u) == 0u) a.biglist[atomicAdd(a.bigcount, 1u)] = (int32_t)row;
      }
    }
  }
  // the stream must be consumed exactly: every state back at L, all escapes used, at
  // most one zero pad word left
  if (!bad) {
    if (x != RANS_L) bad = true;
    if (ep != ne) bad = true;
    if (!(wp == n_wd || (wp == n_wd - 1 && wd[n_wd - 1] == 0))) bad = true;
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicExch(a.status, DCKV_ECORRUPT);
}

}  // namespace dckv
