// dckv_rans.cuh -- warp-interleaved rANS encode / decode, parameter-to-symbol kernels,
// scan and compaction of the DCKV codec.
//
// Coder (per chunk, one warp): 32 interleaved 32-bit states (lane j codes symbols
// i = 32 t + j), 16-bit frequency precision, 16-bit renormalisation words, states in
// [2^16, 2^32).  Symbols of a chunk run row-major over its rows and the kept components;
// symbol = ESC (509) if |q| > 127, else q - centre + 254.  The encoder walks steps
// t = T-1..0; at each step the lanes that must renormalise emit one word each, placed
// with a ballot / popcount so that the decoder, walking t = 0..T-1 and reading words in
// lane order, consumes exactly what was emitted.
//
// Everything a sequential step needs that does not depend on the state (symbols for the
// encoder, centres for the decoder) is computed beforehand by fully parallel kernels and
// laid out in "slot" order -- chunk by chunk, row by row, kept component by kept
// component -- so the sequential loops read contiguous data one step ahead.
#pragma once
#include "dckv_internal.cuh"
#include "dckv_ptx.cuh"

namespace dckv {

constexpr int RANS_WARPS = 4;                            // chunks per block (encoder)
// Decoder: one block per SM (its tables fill the SM's shared memory), DEC_WARPS warps each
// decoding one chunk at a time; a lane's step is a latency-bound dependency chain, so many
// warps per SM keep the schedulers busy.
constexpr int DEC_WARPS = 32;
constexpr int PF = 16;                                   // steps of look-ahead for state-free data
// Decoder tables in shared memory.  Rows are padded by 4 bytes so that the same entry of
// different scales falls in different banks: most lanes of a step decode the central
// symbol, each under its own component's scale, and unpadded 1 KiB / 2 KiB rows would put
// all of them in one bank.
constexpr int DEC_CDF_STRIDE = 514;                      // 510 entries, then zeros
constexpr int CDF_SMEM_BYTES = N_SCALES * DEC_CDF_STRIDE * 2;  // 65,792
constexpr int LUT_BITS = 10;                             // decoder lookup on slot >> 6
constexpr int LUT_SIZE = 1 << LUT_BITS;
constexpr int LUT_STRIDE = LUT_SIZE + 2;
constexpr int LUT_SMEM_BYTES = N_SCALES * LUT_STRIDE * 2;  // 131,328
constexpr int TAIL_SMEM_BYTES = N_SCALES * 4;
constexpr int RANS_DEC_SMEM = CDF_SMEM_BYTES + LUT_SMEM_BYTES + TAIL_SMEM_BYTES + N_COEF;
constexpr uint32_t CF_INVALID = 0xFFFFFFFFu;  // no table entry has cdf 65535 and freq 65536
constexpr uint16_t LUT_SINGLE = 0x4000;       // the bucket lies inside one symbol's range
constexpr uint16_t LUT_MULTI = 0x8000;        // two or more symbol boundaries in the bucket
constexpr uint16_t LUT_SYM = 0x03FF;

__device__ __forceinline__ uint32_t cdf_at(const uint16_t *tab, int k) { return k < N_SYM ? tab[k] : PREC_TOTAL; }

// ------------------------------------------------------------------------------ symbols
// Encoder inputs in slot order: the symbol (ESC if |q| > 127 else q - centre + 254), its
// table entry {cdf | (freq - 1) << 16, division multiplier of freq} (from the codec's
// packed per-(scale, symbol) table), and the escape count of each chunk.  Four positions
// per thread are in flight at a time.
constexpr int SYM_THREADS = 256;
constexpr int SYM_UNROLL = 4;

// Even rows take their centres straight from the even-centre table (and store them in
// cen8 too, where the odd rows' centres already are); with no table (no mean models) every
// centre is 0.

__global__ void __launch_bounds__(SYM_THREADS) k_symbols(int64_t n_rows, const int32_t *row_slot,
                                                         const int32_t *slot_chunk, const int32_t *q32,
                                                         int8_t *cen8, const uint8_t *kept_scale, const uint2 *cfm_tab, int k_eff,
                                                         const int8_t *t_even8, int t_ld, const int32_t *tok_ids,
                                                         const int32_t *row_tok, const int32_t *row_edst, int vocab,
                                                         uint16_t *sym16, uint2 *cfm, uint32_t *nesc) {
  __shared__ int esc_count;
  __shared__ uint8_t s_ks[N_COEF];
  for (int k = threadIdx.x; k < k_eff; k += SYM_THREADS) s_ks[k] = kept_scale[k];
  for (int64_t row = blockIdx.x; row < n_rows; row += gridDim.x) {
    if (threadIdx.x == 0) esc_count = 0;
    __syncthreads();
    const int slot = row_slot[row];
    const int64_t base = (int64_t)slot * k_eff;
    const int32_t *q = q32 + row * CODE_LD;  // compact: kept component k at column k
    const bool even = row_edst[row] >= 0;
    const int8_t *t_row = nullptr;
    if (even && t_even8) t_row = t_even8 + (int64_t)min(max(tok_ids[row_tok[row]], 0), vocab - 1) * t_ld;
    int esc = 0;
    for (int k0 = threadIdx.x; k0 < k_eff; k0 += SYM_UNROLL * SYM_THREADS) {
      int v[SYM_UNROLL], ce[SYM_UNROLL];
#pragma unroll
      for (int u = 0; u < SYM_UNROLL; ++u) {
        const int k = k0 + u * SYM_THREADS;
        v[u] = k < k_eff ? __ldg(q + k) : 0;
        ce[u] = k >= k_eff ? 0 : even ? (t_row ? (int)__ldg(t_row + k) : 0) : (int)__ldg(cen8 + base + k);
      }
#pragma unroll
      for (int u = 0; u < SYM_UNROLL; ++u) {
        const int k = k0 + u * SYM_THREADS;
        if (k < k_eff) {
          const bool is_esc = v[u] > ESC_LIMIT || v[u] < -ESC_LIMIT;
          const int sym = is_esc ? ESC_SYM : v[u] - ce[u] + R_MAX;
          esc += is_esc;
          if (even) cen8[base + k] = (int8_t)ce[u];
          sym16[base + k] = (uint16_t)sym;
          cfm[base + k] = __ldg(cfm_tab + s_ks[k] * N_SYM + sym);
        }
      }
    }
    if (esc) atomicAdd(&esc_count, esc);
    __syncthreads();
    if (threadIdx.x == 0 && esc_count) atomicAdd(&nesc[slot_chunk[slot]], (uint32_t)esc_count);
    __syncthreads();
  }
}

// ------------------------------------------------------------------------------ encode
// Division of the state by a symbol's frequency f uses the multiplier of Granlund and
// Montgomery, "Division by invariant integers using multiplication" (1994), unsigned
// case: with l = ceil(log2 f) and m = floor(2^32 (2^l - f) / f) + 1, every 32-bit x has
// floor(x / f) = (t + ((x - t) >> 1)) >> (l - 1), t = high word of m x.  f = 1 is x itself.
__host__ __device__ inline uint32_t div_multiplier(uint32_t f) {
  if (f < 2) return 0;
  uint32_t l = 0;
  while ((1u << l) < f) ++l;
  return (uint32_t)((((uint64_t)1 << 32) * (((uint64_t)1 << l) - f)) / f + 1);
}

// 16-bit store under a predicate, without a branch.
__device__ __forceinline__ void st_u16_if(uint16_t *p, uint32_t v, bool pred) {
  asm volatile("{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %2, 0;\n\t@q st.global.u16 [%0], %1;\n\t}" ::"l"(p),
               "h"((unsigned short)(v & 0xFFFFu)), "r"((int)pred)
               : "memory");
}

struct RansEncArgs {
  const ChunkDesc *chunks;
  int n_chunks;
  int k_eff;
  const uint2 *cfm;    // slot order: {cdf | (freq - 1) << 16, division multiplier}
  uint16_t *words;     // word scratch: chunk c owns [sym_base, sym_base + S)
  uint32_t *states;    // [chunks][32]
  uint32_t *nwords;    // [chunks] words emitted
};

__global__ void __launch_bounds__(RANS_WARPS * 32) rans_encode_kernel(RansEncArgs a) {
  const int lane = threadIdx.x & 31;
  const int ci = blockIdx.x * RANS_WARPS + (threadIdx.x >> 5);
  if (ci >= a.n_chunks) return;
  const ChunkDesc cd = a.chunks[ci];
  const uint32_t S = (uint32_t)cd.nrows * (uint32_t)a.k_eff;  // < 2^20
  const int T = (int)((S + 31) / 32);
  const uint2 *cfs = a.cfm + cd.sym_base;
  uint16_t *wslot = a.words + cd.sym_base;
  uint32_t pos = S;  // words are placed downwards from the end of the slot
  uint32_t x = RANS_L;
  const uint32_t lt_mask = (1u << lane) - 1u;
  // steps run in groups of 16 from t = T-1 down; the next group's table entries are
  // loaded while the current group is coded (they do not depend on the state)
  uint2 cur[16], nxt[16];
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const int t = T - 1 - u;
    const uint32_t i = (uint32_t)t * 32u + lane;
    cur[u] = (t >= 0 && i < S) ? cfs[i] : make_uint2(CF_INVALID, 0u);
  }
  for (int t0 = T - 1; t0 >= 0; t0 -= 16) {
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int t = t0 - 16 - u;
      const uint32_t i = (uint32_t)t * 32u + lane;
      nxt[u] = (t >= 0 && i < S) ? cfs[i] : make_uint2(CF_INVALID, 0u);
    }
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const uint32_t cf = cur[u].x;
      const bool valid = cf != CF_INVALID;
      const uint32_t c = cf & 0xFFFFu;
      const uint32_t f = valid ? (cf >> 16) + 1u : 1u;
      const bool emit = valid && x >= (f << 16);
      const uint32_t m = __ballot_sync(0xffffffffu, emit);
      const uint32_t nm = __popc(m);
      st_u16_if(wslot + (pos - nm + __popc(m & lt_mask)), x, emit);
      pos -= nm;
      const uint32_t xr = emit ? x >> 16 : x;
      const uint32_t th = __umulhi(cur[u].y, xr);
      const int sh = max(31 - __clz((int)(f - 1u)), 0);
      const uint32_t qf = f == 1u ? xr : (th + ((xr - th) >> 1)) >> sh;
      const uint32_t xn = xr + c + qf * (PREC_TOTAL - f);  // = (qf << 16) + xr mod f + c
      x = valid ? xn : x;
    }
#pragma unroll
    for (int u = 0; u < 16; ++u) cur[u] = nxt[u];
  }
  a.states[(int64_t)ci * 32 + lane] = x;
  if (lane == 0) a.nwords[ci] = S - pos;
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
  const uint64_t tab_end = HEADER_BYTES + 4ull * (a.batch + a.n_chunks + 1);
  for (uint64_t o = tab_end + tid; o < a.off_kept; o += 1024) a.blob[o] = 0;
}

// Writes each chunk section: states, escape count, escaped codes (symbol order), words.
struct CompactArgs {
  const ChunkDesc *chunks;
  const PromptInfo *prompts;
  int n_chunks;
  int k_eff;
  const int32_t *q32;     // [rows][CODE_LD]: kept components in compact order
  const uint16_t *sym16;
  const uint16_t *words;
  const uint32_t *states, *nwords, *nesc, *offs;
  uint8_t *blob;
  uint64_t blob_cap, off_streams;
};

constexpr int COMPACT_THREADS = 128;

// One block per chunk.  Escape values are found in two passes over the chunk's symbols
// (count per warp, then write at the warp's prefix), only in chunks that have escapes.
__global__ void __launch_bounds__(COMPACT_THREADS) compact_kernel(CompactArgs a) {
  __shared__ uint32_t s_cnt[COMPACT_THREADS / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int NW = COMPACT_THREADS / 32;
  const int ci = blockIdx.x;
  if (ci >= a.n_chunks) return;
  const uint64_t beg = a.off_streams + a.offs[ci];
  const uint64_t end = a.off_streams + a.offs[ci + 1];
  if (end > a.blob_cap) return;  // capacity error already reported by the scan
  uint8_t *sec = a.blob + beg;
  const uint32_t ne = a.nesc[ci], nw = a.nwords[ci];
  if (threadIdx.x < 32) reinterpret_cast<uint32_t *>(sec)[lane] = a.states[(int64_t)ci * 32 + lane];
  if (threadIdx.x == 0) reinterpret_cast<uint32_t *>(sec)[32] = ne;
  const ChunkDesc cd = a.chunks[ci];
  const int K = a.k_eff;
  const int64_t S = (int64_t)cd.nrows * K;
  // escaped codes in symbol order, 64 raw bits each (sections are 4-byte aligned)
  if (ne) {
    const PromptInfo pi = a.prompts[cd.prompt];
    uint32_t *ev = reinterpret_cast<uint32_t *>(sec + CHUNK_FIXED_BYTES);
    const uint32_t lt_mask = (1u << lane) - 1u;
    const uint16_t *syms = a.sym16 + cd.sym_base;
    const int64_t per = ((S + NW - 1) / NW + 31) & ~int64_t(31);  // warp w scans [w per, (w+1) per)
    const int64_t i_beg = warp * per, i_end = min(S, i_beg + per);
    uint32_t n = 0;
    for (int64_t i = i_beg + lane; i < i_end; i += 32) n += syms[i] == ESC_SYM;
    for (int o = 16; o; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
    if (lane == 0) s_cnt[warp] = n;
    __syncthreads();
    uint32_t ep = 0;
    for (int w = 0; w < warp; ++w) ep += s_cnt[w];
    for (int64_t i0 = i_beg; i0 < i_end; i0 += 32) {
      const int64_t i = i0 + lane;
      const bool esc = i < i_end && syms[i] == ESC_SYM;
      const uint32_t m = __ballot_sync(0xffffffffu, esc);
      if (esc) {
        const int rl = (int)(i / K);
        const int k = (int)(i - (int64_t)rl * K);
        const int64_t row = (int64_t)pi.row_base + 2 * (cd.j0 + rl) + cd.parity;
        const int64_t v = (int64_t)a.q32[row * CODE_LD + k];
        const uint32_t slot = ep + __popc(m & lt_mask);
        if (slot < ne) {
          ev[2 * slot] = (uint32_t)(uint64_t)v;
          ev[2 * slot + 1] = (uint32_t)((uint64_t)v >> 32);
        }
      }
      ep += __popc(m);
    }
  }
  // words (decoder order) follow the escapes; then zero padding to 4 bytes
  uint16_t *wd = reinterpret_cast<uint16_t *>(sec + CHUNK_FIXED_BYTES + 8ull * ne);
  const uint16_t *ws = a.words + cd.sym_base + (S - nw);
  for (uint32_t w0 = threadIdx.x; w0 < nw; w0 += 4 * COMPACT_THREADS) {
    uint16_t v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t w = w0 + u * COMPACT_THREADS;
      v[u] = w < nw ? ws[w] : (uint16_t)0;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t w = w0 + u * COMPACT_THREADS;
      if (w < nw) wd[w] = v[u];
    }
  }
  const uint64_t used = CHUNK_FIXED_BYTES + 8ull * ne + 2ull * nw;
  if (threadIdx.x == 0 && (end - beg) > used) wd[nw] = 0;
}

// ------------------------------------------------------------------------------ decode
// Decoder tables, per scale s:
//   dcdf[s][0..509] = cdf, dcdf[s][510..513] = 0 (65536 mod 2^16, so that
//     freq = (dcdf[sym + 1] - dcdf[sym]) mod 2^16 for every symbol);
//   lut[s][b] for the 64 slots b * 64 .. b * 64 + 63: bits 0-9 the symbol holding the
//     first of them, LUT_SINGLE if one symbol holds all of them, LUT_MULTI if two or more
//     symbol ranges start inside the bucket (else exactly one does);
//   tail[s] = length of the leading run of frequency-1 symbols (cdf[sym] = sym) in bits
//     0-15 and length n of the trailing run (cdf[sym] = 65536 - 510 + sym, ESC last;
//     slots 65536 - n .. 65535) in bits 16-31; slots in a run decode by arithmetic;
//   cfm_tab[s][sym] = {cdf | (freq - 1) << 16, division multiplier of freq} (encoder).
__global__ void k_build_lut(const uint16_t *cdf, uint16_t *dcdf, uint16_t *lut, uint32_t *tail, uint2 *cfm_tab) {
  const int s = blockIdx.x;
  const uint16_t *tab = cdf + s * N_SYM;
  __shared__ uint32_t runs[2];
  if (threadIdx.x == 0) {
    int lead = 0;  // symbols 0 .. lead-1 have frequency 1
    while (lead < N_SYM && cdf_at(tab, lead + 1) - tab[lead] == 1u) ++lead;
    int trail = N_SYM;  // symbols trail .. 509 have frequency 1
    while (trail > lead && cdf_at(tab, trail) - tab[trail - 1] == 1u) --trail;
    tail[s] = (uint32_t)lead | ((uint32_t)(N_SYM - trail) << 16);
    runs[0] = (uint32_t)lead;                     // slots below this decode by arithmetic
    runs[1] = PREC_TOTAL - (uint32_t)(N_SYM - trail);  // slots from this one on likewise
  }
  __syncthreads();
  auto holder = [&](uint32_t slot) {
    int lo = 0, hi = N_SYM;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (tab[mid] <= slot) lo = mid; else hi = mid;
    }
    return lo;
  };
  for (int b = threadIdx.x; b < LUT_SIZE; b += blockDim.x) {
    // classify the bucket by its slots outside the frequency-1 runs (those are resolved
    // by arithmetic); a bucket wholly inside a run is marked as one symbol
    const uint32_t first = max((uint32_t)b << (16 - LUT_BITS), runs[0]);
    const uint32_t last = min(((uint32_t)(b + 1) << (16 - LUT_BITS)) - 1u, runs[1] - 1u);
    uint16_t e;
    if (first > last) {
      e = (uint16_t)(holder((uint32_t)b << (16 - LUT_BITS)) | LUT_SINGLE);
    } else {
      const int lo = holder(first), hi = holder(last);
      e = (uint16_t)(lo | (hi == lo ? LUT_SINGLE : 0) | (hi >= lo + 2 ? LUT_MULTI : 0));
    }
    lut[s * LUT_STRIDE + b] = e;
  }
  if (threadIdx.x < LUT_STRIDE - LUT_SIZE) lut[s * LUT_STRIDE + LUT_SIZE + threadIdx.x] = 0;
  for (int k = threadIdx.x; k < DEC_CDF_STRIDE; k += blockDim.x) {
    dcdf[s * DEC_CDF_STRIDE + k] = k < N_SYM ? tab[k] : (uint16_t)0;
    if (k < N_SYM) {
      const uint32_t f = cdf_at(tab, k + 1) - tab[k];
      cfm_tab[s * N_SYM + k] = make_uint2((uint32_t)tab[k] | ((f - 1u) << 16), div_multiplier(f));
    }
  }
}

// Several symbol ranges start inside the slot's bucket (outside the tail runs): binary
// search between the bucket's first symbol and the next bucket's.
__device__ __noinline__ int search_symbol(uint32_t slot, int s, uint32_t b, const uint16_t *tab,
                                          const uint16_t *s_lut, uint32_t &c, uint32_t &f) {
  int sym = (int)(s_lut[s * LUT_STRIDE + b] & LUT_SYM);
  int hi = b + 1 < (uint32_t)LUT_SIZE ? (int)(s_lut[s * LUT_STRIDE + b + 1] & LUT_SYM) : N_SYM - 1;  // in [sym, hi]
  while (hi > sym) {
    const int mid = (sym + hi + 1) >> 1;
    if (tab[mid] <= slot) sym = mid; else hi = mid - 1;
  }
  c = tab[sym];
  f = ((uint32_t)tab[sym + 1] - c) & 0xFFFFu;
  return sym;
}

// Symbol holding `slot` under scale s, with its cumulative frequency c and frequency f.
// The bucket entry settles any bucket with at most one boundary outside the tail runs by
// one comparison; slots inside the frequency-1 runs at both tails decode by arithmetic
// (selects, no branch); only a bucket with several boundaries outside the runs (central
// symbols of frequency below 64) takes the search.
__device__ __forceinline__ int find_symbol(uint32_t slot, int s, const uint16_t *s_cdf, const uint16_t *s_lut,
                                           const uint32_t *s_tail, uint32_t &c, uint32_t &f) {
  const uint16_t *tab = s_cdf + s * DEC_CDF_STRIDE;
  const uint32_t b = slot >> (16 - LUT_BITS);
  const uint32_t e = s_lut[s * LUT_STRIDE + b];
  const uint32_t tl = s_tail[s];
  int sym = (int)(e & LUT_SYM);
  const uint32_t c0 = tab[sym], c1 = tab[sym + 1], c2 = tab[sym + 2];
  const bool up = !(e & LUT_SINGLE) && slot >= c1;
  sym += up;
  c = up ? c1 : c0;
  f = ((up ? c2 : c1) - c) & 0xFFFFu;
  const bool lo_run = slot < (tl & 0xFFFFu);
  const bool hi_run = slot + (tl >> 16) >= PREC_TOTAL;
  const bool run = lo_run || hi_run;
  sym = run ? (lo_run ? (int)slot : (int)(slot - (PREC_TOTAL - (uint32_t)N_SYM))) : sym;
  c = run ? slot : c;
  f = run ? 1u : f;
  if ((e & LUT_MULTI) && !run) sym = search_symbol(slot, s, b, tab, s_lut, c, f);
  return sym;
}

struct RansDecArgs {
  const ChunkDesc *chunks;
  int chunk0, n_chunks;  // chunks [chunk0, chunk0 + n_chunks)
  int k_eff;
  const uint8_t *kept_scale;
  const uint16_t *dcdf;
  const uint16_t *lut;
  const uint32_t *tail;
  const uint8_t *blob;
  uint64_t off_streams;
  const uint32_t *offs;  // chunk table inside the blob
  uint16_t *syms;        // slot order: the decoded symbol of every position
  const int32_t *valid;  // header check result (1 = ok)
  int32_t *status;
};

// The decoder's tables (cdf rows, bucket lookup, tail runs, component scales) into shared
// memory with bulk copies issued by one thread, in pieces of at most 32 KiB; every thread
// waits (bounded) for their completion.  Returns false on timeout.
__device__ __forceinline__ bool bulk_load_tables(uint8_t *sm, const uint16_t *dcdf, const uint16_t *lut,
                                                 const uint32_t *tail, const uint8_t *scale, uint64_t *bar,
                                                 volatile int *abort_flag) {
  const uint8_t *src[4] = {reinterpret_cast<const uint8_t *>(dcdf), reinterpret_cast<const uint8_t *>(lut),
                           reinterpret_cast<const uint8_t *>(tail), scale};
  constexpr uint32_t len[4] = {CDF_SMEM_BYTES, LUT_SMEM_BYTES, TAIL_SMEM_BYTES, N_COEF};
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bar, len[0] + len[1] + len[2] + len[3]);
    uint32_t off = 0;
    for (int t = 0; t < 4; ++t) {
      for (uint32_t o = 0; o < len[t]; o += 32768u) {
        const uint32_t n = min(32768u, len[t] - o);
        bulk_load(sm + off + o, src[t] + o, n, bar);
      }
      off += len[t];
    }
  }
  return mbar_wait(bar, 0, abort_flag);
}

// State of one warp decoding one chunk.
struct DecLane {
  uint32_t x;           // rANS state
  uint32_t w0, w1, w2;  // word ring: lane j holds words wb + j, wb + 32 + j, wb + 64 + j
  uint32_t wb, wp;      // ring base, words consumed
  int k;                // kept component of this lane's next symbol
  int s;                // its scale, loaded a step ahead (off the state's dependency chain)
};

// One decode step of all 32 lanes: symbol i = 32 t + lane.  CHECK: some lanes may lie
// beyond the chunk's last symbol.  BIG_K: K >= 32 (the component advances by at most one
// wrap per step).
template <bool CHECK, bool BIG_K>
__device__ __forceinline__ void dec_step(DecLane &d, uint32_t i, uint32_t S, int K, uint32_t lt_mask,
                                         const uint8_t *s_scale, const uint16_t *s_cdf, const uint16_t *s_lut,
                                         const uint32_t *s_tail, const uint16_t *wd, uint32_t n_wd, uint16_t *out) {
  const bool valid = !CHECK || i < S;
  bool need = false;
  if (valid) {
    const uint32_t slot = d.x & 0xFFFFu;
    uint32_t c, f;
    const int sym = find_symbol(slot, d.s, s_cdf, s_lut, s_tail, c, f);
    d.x = f * (d.x >> 16) + slot - c;
    need = d.x < RANS_L;
    out[i] = (uint16_t)sym;
  }
  const uint32_t m = __ballot_sync(0xffffffffu, need);
  const uint32_t p = (d.wp - d.wb) + __popc(m & lt_mask);  // < 64: wp - wb < 32 before the step
  const uint32_t v0 = __shfl_sync(0xffffffffu, d.w0, p & 31);
  const uint32_t v1 = __shfl_sync(0xffffffffu, d.w1, p & 31);
  d.x = need ? (d.x << 16) | (p < 32 ? v0 : v1) : d.x;
  d.wp += __popc(m);
  if (d.wp - d.wb >= 32) {  // warp-uniform: slide the ring by 32 words
    d.w0 = d.w1;
    d.w1 = d.w2;
    d.wb += 32;
    const uint32_t wi = d.wb + 64 + __popc(lt_mask);  // lane index
    d.w2 = wi < n_wd ? wd[wi] : 0u;
  }
  if (BIG_K) {
    d.k += 32;
    d.k = d.k >= K ? d.k - K : d.k;
  } else {
    d.k += 32;
    while (d.k >= K) d.k -= K;
  }
  d.s = s_scale[d.k];
}

// One warp decodes chunk ci: states, escape count and word stream from its section.
template <bool BIG_K>
__device__ __forceinline__ void decode_chunk(const RansDecArgs &a, int ci, int lane, const uint8_t *s_scale,
                                             const uint16_t *s_cdf, const uint16_t *s_lut, const uint32_t *s_tail) {
  const ChunkDesc cd = a.chunks[ci];
  const int K = a.k_eff;
  const uint32_t S = (uint32_t)cd.nrows * (uint32_t)K;  // < 2^20
  const int T = (int)((S + 31) / 32);
  const int T_full = (int)(S / 32);  // steps where every lane holds a symbol
  const uint64_t beg = a.off_streams + a.offs[ci];
  const uint64_t end = a.off_streams + a.offs[ci + 1];
  const uint8_t *sec = a.blob + beg;
  const uint32_t ne = reinterpret_cast<const uint32_t *>(sec)[32];
  if ((end - beg) < CHUNK_FIXED_BYTES || (uint64_t)CHUNK_FIXED_BYTES + 8ull * ne > (end - beg)) {
    if (lane == 0) atomicExch(a.status, DCKV_ECORRUPT);
    return;
  }
  const uint16_t *wd = reinterpret_cast<const uint16_t *>(sec + CHUNK_FIXED_BYTES + 8ull * ne);
  const uint32_t n_wd = (uint32_t)(((end - beg) - CHUNK_FIXED_BYTES - 8ull * ne) / 2);
  uint16_t *out = a.syms + cd.sym_base;
  const uint32_t lt_mask = (1u << lane) - 1u;
  DecLane d;
  d.x = reinterpret_cast<const uint32_t *>(sec)[lane];
  d.wb = 0;
  d.wp = 0;
  d.w0 = (uint32_t)lane < n_wd ? wd[lane] : 0u;
  d.w1 = 32u + lane < n_wd ? wd[32 + lane] : 0u;
  d.w2 = 64u + lane < n_wd ? wd[64 + lane] : 0u;
  d.k = K > 0 ? lane % K : 0;
  d.s = s_scale[d.k];
  bool bad = d.x < RANS_L;
  int t = 0;
  for (; t + 16 <= T_full && !bad; t += 16) {
#pragma unroll
    for (int u = 0; u < 16; ++u)
      dec_step<false, BIG_K>(d, (uint32_t)(t + u) * 32u + lane, S, K, lt_mask, s_scale, s_cdf, s_lut, s_tail, wd,
                             n_wd, out);
    bad = __any_sync(0xffffffffu, bad || d.wp > n_wd);
  }
  for (; t < T && !bad; ++t)
    dec_step<true, BIG_K>(d, (uint32_t)t * 32u + lane, S, K, lt_mask, s_scale, s_cdf, s_lut, s_tail, wd, n_wd, out);
  bad = __any_sync(0xffffffffu, bad || d.wp > n_wd);
  // the stream must be consumed exactly: every state back at L, at most one zero pad
  // word left (escape values are checked by the finishing kernel)
  if (!bad) {
    if (d.x != RANS_L) bad = true;
    if (!(d.wp == n_wd || (d.wp + 1 == n_wd && wd[n_wd - 1] == 0))) bad = true;
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicExch(a.status, DCKV_ECORRUPT);
}

// The rANS arithmetic needs only the table (scale) of each component, never the code
// means, so every chunk of both parities decodes in one launch; centres are applied
// afterwards by the finishing kernel, pass by pass.
template <bool BIG_K>
__global__ void __launch_bounds__(DEC_WARPS * 32, 1) rans_decode_kernel(RansDecArgs a) {
  extern __shared__ __align__(16) uint8_t sm[];
  const uint16_t *s_cdf = reinterpret_cast<const uint16_t *>(sm);
  const uint16_t *s_lut = reinterpret_cast<const uint16_t *>(sm + CDF_SMEM_BYTES);
  const uint32_t *s_tail = reinterpret_cast<const uint32_t *>(sm + CDF_SMEM_BYTES + LUT_SMEM_BYTES);
  uint8_t *s_scale = sm + CDF_SMEM_BYTES + LUT_SMEM_BYTES + TAIL_SMEM_BYTES;
  __shared__ uint64_t tab_bar;
  __shared__ int tab_abort;
  if (*a.valid != 1) return;
  static_assert(CDF_SMEM_BYTES % 16 == 0 && LUT_SMEM_BYTES % 16 == 0 && TAIL_SMEM_BYTES % 16 == 0, "bulk sizes");
  if (!bulk_load_tables(sm, a.dcdf, a.lut, a.tail, a.kept_scale, &tab_bar, &tab_abort)) {
    if (threadIdx.x == 0) {
      atomicExch(a.status, DCKV_ETIMEOUT);
      mbar_drain(&tab_bar, 0);  // the CTA's shared memory stays allocated until its copies land
    }
    return;
  }
  const int lane = threadIdx.x & 31;
  // chunk wi goes to block wi % gridDim.x: consecutive chunks land on different SMs
  for (int wi = (threadIdx.x >> 5) * gridDim.x + blockIdx.x; wi < a.n_chunks; wi += gridDim.x * DEC_WARPS)
    decode_chunk<BIG_K>(a, a.chunk0 + wi, lane, s_scale, s_cdf, s_lut, s_tail);
}

// Finishing a decoded pass in two steps.  k_codes_elem writes code = centre + symbol - 254
// for every symbol of the pass's rows, fully parallel (fp16 to q16; even rows also bf16 to
// qe, the odd mean model's input); an ESC symbol only flags its chunk.  An even row's
// centres are its token's row of the even-centre table (kept components, read in place);
// without mean models every centre is 0.  (The odd pass of a
// codec with mean models gets the same from the odd mean GEMM's epilogue.)  k_escape_patch
// then visits the chunks that store escape values or hold a flagged ESC, ranks the ESC
// symbols in symbol order (escape values are stored in that order), writes those codes,
// lists codes of 2048 or more for the exact fix-up (only escapes reach them: any other code
// lies within 127 + 254), and checks that every escape value is used exactly once.
__global__ void __launch_bounds__(256) k_codes_elem(int parity, int64_t n_rows, const int32_t *row_edst,
                                                    const int32_t *row_slot, const int32_t *slot_chunk,
                                                    const uint16_t *syms, const int8_t *t_even8, int t_ld,
                                                    const int32_t *tok_ids, const int32_t *row_tok, int vocab,
                                                    int k_eff, __half *q16,
                                                    __nv_bfloat16 *qe, uint32_t *escflag, const int32_t *valid) {
  if (*valid != 1) return;
  constexpr int PER = N_COEF / 256;  // blockDim.x == 256
  // a block's rows are r, r + grid, ...: the next row's metadata (its even index, slot and,
  // for an even row, its token's table row) is fetched while this row's symbols load
  auto tab_row = [&](int64_t r, int e) -> const int8_t * {
    return (e >= 0 && t_even8) ? t_even8 + (int64_t)min(max(tok_ids[row_tok[r]], 0), vocab - 1) * t_ld : nullptr;
  };
  int64_t r = blockIdx.x;
  int e = r < n_rows ? row_edst[r] : -1;
  int64_t slot = r < n_rows ? row_slot[r] : 0;
  const int8_t *ce = r < n_rows ? tab_row(r, e) : nullptr;
  while (r < n_rows) {
    const int64_t rn = r + gridDim.x;
    const bool has_next = rn < n_rows;
    const int e_n = has_next ? row_edst[rn] : -1;
    const int64_t slot_n = has_next ? row_slot[rn] : 0;
    const bool mine = (e >= 0) == (parity == 0);  // block-uniform
    int sv[PER], cv[PER];
    if (mine) {
      const uint16_t *sy = syms + slot * k_eff;
#pragma unroll
      for (int u = 0; u < PER; ++u) {  // every load before the stores
        const int k = threadIdx.x + 256 * u;
        sv[u] = k < k_eff ? (int)__ldg(sy + k) : 0;
        cv[u] = (k < k_eff && ce) ? (int)__ldg(ce + k) : 0;
      }
    }
    const int8_t *ce_n = has_next && (e_n >= 0) == (parity == 0) ? tab_row(rn, e_n) : nullptr;
    if (mine) {
      bool esc = false;
#pragma unroll
      for (int u = 0; u < PER; ++u) {
        const int k = threadIdx.x + 256 * u;
        if (k >= k_eff) continue;
        if (sv[u] == ESC_SYM) {
          esc = true;
          continue;
        }
        const int q = sv[u] - R_MAX + cv[u];
        q16[r * CODE_LD + k] = __float2half_rn((float)q);
        if (e >= 0) qe[(int64_t)e * CODE_LD + k] = __float2bfloat16_rn((float)q);
      }
      if (__syncthreads_or(esc) && threadIdx.x == 0) escflag[slot_chunk[slot]] = 1u;
    }
    r = rn;
    e = e_n;
    slot = slot_n;
    ce = ce_n;
  }
}

struct DecCodesArgs {
  const ChunkDesc *chunks;
  const PromptInfo *prompts;
  int chunk0, n_chunks;
  int k_eff;
  const uint16_t *syms;     // slot order (q16, qe, qbig: [rows][CODE_LD], kept components in compact order)
  const uint8_t *blob;
  uint64_t off_streams;
  const uint32_t *offs;
  __half *q16;
  __nv_bfloat16 *qe;
  int32_t *qbig;
  uint32_t *bigflag;
  int32_t *biglist;
  uint32_t *bigcount;
  const uint32_t *escflag;
  const int32_t *valid;
  int32_t *status;
};

constexpr int PATCH_THREADS = 256;

__global__ void __launch_bounds__(PATCH_THREADS) k_escape_patch(DecCodesArgs a) {
  __shared__ uint32_t s_cnt[PATCH_THREADS / 32];
  if (*a.valid != 1) return;
  const int ci = a.chunk0 + blockIdx.x;
  if ((int)blockIdx.x >= a.n_chunks) return;
  const uint8_t *sec = a.blob + a.off_streams + a.offs[ci];
  const uint32_t ne = reinterpret_cast<const uint32_t *>(sec)[32];
  if (ne == 0 && a.escflag[ci] == 0) return;  // block-uniform: no escapes here
  const uint32_t *ev = reinterpret_cast<const uint32_t *>(sec + CHUNK_FIXED_BYTES);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int NW = PATCH_THREADS / 32;
  const uint32_t lt_mask = (1u << lane) - 1u;
  const ChunkDesc cd = a.chunks[ci];
  const PromptInfo pi = a.prompts[cd.prompt];
  const int K = a.k_eff;
  const int64_t S = (int64_t)cd.nrows * K;
  const uint16_t *sy = a.syms + cd.sym_base;
  const int64_t per = ((S + NW - 1) / NW + 31) & ~int64_t(31);  // warp w scans [w per, (w+1) per)
  const int64_t i_beg = warp * per, i_end = min(S, i_beg + per);
  uint32_t n = 0;
  for (int64_t i = i_beg + lane; i < i_end; i += 32) n += sy[i] == ESC_SYM;
  for (int o = 16; o; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
  if (lane == 0) s_cnt[warp] = n;
  __syncthreads();
  uint32_t ep = 0, total = 0;
  for (int w = 0; w < NW; ++w) {
    if (w < warp) ep += s_cnt[w];
    total += s_cnt[w];
  }
  bool bad = threadIdx.x == 0 && total != ne;  // every escape value used exactly once
  for (int64_t i0 = i_beg; i0 < i_end; i0 += 32) {
    const int64_t i = i0 + lane;
    const bool esc = i < i_end && sy[i] == ESC_SYM;
    const uint32_t m = __ballot_sync(0xffffffffu, esc);
    if (esc) {
      const uint32_t e = ep + __popc(m & lt_mask);
      int q = 0;
      if (e < ne) {
        const int64_t sval = (int64_t)((uint64_t)ev[2 * e] | ((uint64_t)ev[2 * e + 1] << 32));
        q = (int)max(min(sval, (int64_t)INT32_MAX), (int64_t)INT32_MIN);
        if (sval >= -ESC_LIMIT && sval <= ESC_LIMIT) bad = true;  // not an escape value
      } else {
        bad = true;
      }
      const int rl = (int)(i / K);
      const int k = (int)(i - (int64_t)rl * K);
      const int64_t row = (int64_t)pi.row_base + 2 * (cd.j0 + rl) + cd.parity;
      a.q16[row * CODE_LD + k] = __float2half_rn((float)q);
      if (cd.parity == 0) a.qe[(int64_t)(pi.ebase + cd.j0 + rl) * CODE_LD + k] = __float2bfloat16_rn((float)q);
      if (q >= BIG_CODE || q <= -BIG_CODE) {
        a.qbig[row * CODE_LD + k] = q;
        if (atomicExch(&a.bigflag[row], 1u) == 0u) a.biglist[atomicAdd(a.bigcount, 1u)] = (int32_t)row;
      }
    }
    ep += __popc(m);
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicExch(a.status, DCKV_ECORRUPT);
}

}  // namespace dckv
