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

constexpr int RANS_WARPS = 4;                            // chunks per block
constexpr int PF = 16;                                   // steps of look-ahead for state-free data
constexpr int CDF_SMEM_BYTES = N_SCALES * N_SYM * 2;     // 65,280
constexpr int LUT_BITS = 10;                             // decoder lookup on slot >> 6
constexpr int LUT_SIZE = 1 << LUT_BITS;
constexpr int LUT_SMEM_BYTES = N_SCALES * LUT_SIZE * 2;  // 131,072
constexpr int RANS_DEC_SMEM = CDF_SMEM_BYTES + LUT_SMEM_BYTES + N_COEF;
constexpr int DEC_FINISH_SMEM = CDF_SMEM_BYTES + LUT_SMEM_BYTES;

__device__ __forceinline__ void copy_smem16(void *dst, const void *src, int bytes) {
  const uint4 *s = reinterpret_cast<const uint4 *>(src);
  uint4 *d = reinterpret_cast<uint4 *>(dst);
  for (int i = threadIdx.x; i < bytes / 16; i += blockDim.x) d[i] = s[i];
}

__device__ __forceinline__ uint32_t cdf_at(const uint16_t *tab, int k) { return k < N_SYM ? tab[k] : PREC_TOTAL; }

// ------------------------------------------------------------------------------ symbols
// Centres of even rows, clamp(round(T_even[token][c]), +-127), in slot order.
__global__ void __launch_bounds__(256) k_centres_even(int64_t n_rows, const int32_t *row_slot,
                                                      const int32_t *row_edst, const int32_t *row_tok,
                                                      const int32_t *tok_ids, const float *t_even, int vocab,
                                                      const int16_t *kept_list, int k_eff, int8_t *cen8,
                                                      const int32_t *valid) {
  if (valid && *valid != 1) return;
  for (int64_t row = blockIdx.x; row < n_rows; row += gridDim.x) {
    if (row_edst[row] < 0) continue;
    int tok = tok_ids[row_tok[row]];
    tok = min(max(tok, 0), vocab - 1);
    const float *te = t_even + (int64_t)tok * N_COEF;
    int8_t *dst = cen8 + (int64_t)row_slot[row] * k_eff;
    for (int k = threadIdx.x; k < k_eff; k += blockDim.x) {
      const float mu = te[kept_list[k]];
      dst[k] = (int8_t)fminf(fmaxf(rintf(mu), -(float)ESC_LIMIT), (float)ESC_LIMIT);
    }
  }
}

// Encoder inputs in slot order: the symbol (ESC if |q| > 127 else q - centre + 254), its
// table entry packed as cdf | (freq - 1) << 16, and the escape count of each chunk.
__global__ void __launch_bounds__(256) k_symbols(int64_t n_rows, const int32_t *row_slot, const int32_t *slot_chunk,
                                                 const int32_t *q32, const int8_t *cen8, const int16_t *kept_list,
                                                 const uint8_t *kept_scale, const uint16_t *cdf, int k_eff,
                                                 uint16_t *sym16, uint32_t *cf32, uint32_t *nesc) {
  __shared__ int esc_count;
  for (int64_t row = blockIdx.x; row < n_rows; row += gridDim.x) {
    if (threadIdx.x == 0) esc_count = 0;
    __syncthreads();
    const int slot = row_slot[row];
    const int64_t base = (int64_t)slot * k_eff;
    const int32_t *q = q32 + row * N_COEF;
    int esc = 0;
    for (int k = threadIdx.x; k < k_eff; k += blockDim.x) {
      const int v = q[kept_list[k]];
      const bool is_esc = v > ESC_LIMIT || v < -ESC_LIMIT;
      const int sym = is_esc ? ESC_SYM : v - cen8[base + k] + R_MAX;
      esc += is_esc;
      const uint16_t *tab = cdf + kept_scale[k] * N_SYM;
      const uint32_t c = tab[sym];
      const uint32_t f = cdf_at(tab, sym + 1) - c;
      sym16[base + k] = (uint16_t)sym;
      cf32[base + k] = c | ((f - 1u) << 16);
    }
    if (esc) atomicAdd(&esc_count, esc);
    __syncthreads();
    if (threadIdx.x == 0 && esc_count) atomicAdd(&nesc[slot_chunk[slot]], (uint32_t)esc_count);
    __syncthreads();
  }
}

// ------------------------------------------------------------------------------ encode
struct RansEncArgs {
  const ChunkDesc *chunks;
  int n_chunks;
  int k_eff;
  const uint32_t *cf32;  // slot order: cdf | (freq - 1) << 16
  uint16_t *words;       // word scratch: chunk c owns [sym_base, sym_base + S)
  uint32_t *states;      // [chunks][32]
  uint32_t *nwords;      // [chunks] words emitted
};

__global__ void __launch_bounds__(RANS_WARPS * 32) rans_encode_kernel(RansEncArgs a) {
  const int lane = threadIdx.x & 31;
  const int ci = blockIdx.x * RANS_WARPS + (threadIdx.x >> 5);
  if (ci >= a.n_chunks) return;
  const ChunkDesc cd = a.chunks[ci];
  const uint32_t S = (uint32_t)cd.nrows * (uint32_t)a.k_eff;  // < 2^20
  const int T = (int)((S + 31) / 32);
  const uint32_t *cfs = a.cf32 + cd.sym_base;
  uint16_t *wslot = a.words + cd.sym_base;
  uint32_t pos = S;  // words are placed downwards from the end of the slot
  uint32_t x = RANS_L;
  const uint32_t lt_mask = (1u << lane) - 1u;
  // table entries are fetched PF steps ahead through a register ring (independent of x)
  uint32_t ring[PF];
#pragma unroll
  for (int u = 0; u < PF; ++u) {
    const int t = T - 1 - u;
    const uint32_t iu = (uint32_t)t * 32u + lane;
    ring[u] = (t >= 0 && iu < S) ? cfs[iu] : 0u;
  }
  for (int t0 = T - 1; t0 >= 0; t0 -= PF) {
#pragma unroll
    for (int u = 0; u < PF; ++u) {
      const int t = t0 - u;
      if (t < 0) break;
      const uint32_t i = (uint32_t)t * 32u + lane;
      const bool valid = i < S;
      const uint32_t cf = ring[u];
      const int tn = t - PF;
      const uint32_t in = (uint32_t)tn * 32u + lane;
      ring[u] = (tn >= 0 && in < S) ? cfs[in] : 0u;
      const uint32_t c = cf & 0xFFFFu;
      const uint32_t f = valid ? (cf >> 16) + 1u : 1u;
      const bool emit = valid && x >= (f << 16);
      const uint32_t m = __ballot_sync(0xffffffffu, emit);
      if (emit) {
        wslot[pos - __popc(m) + __popc(m & lt_mask)] = (uint16_t)(x & 0xFFFFu);
        x >>= 16;
      }
      pos -= __popc(m);
      if (valid) {
        const uint32_t qf = x / f;
        x = (qf << 16) + (x - qf * f) + c;
      }
    }
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
  const int16_t *kept_list;
  const int32_t *q32;
  const uint16_t *sym16;
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
    const uint16_t *syms = a.sym16 + cd.sym_base;
    for (int64_t i0 = 0; i0 < S && ep < ne; i0 += 32) {
      const int64_t i = i0 + lane;
      const bool esc = i < S && syms[i] == ESC_SYM;
      const uint32_t m = __ballot_sync(0xffffffffu, esc);
      if (esc) {
        const int rl = (int)(i / K);
        const int k = (int)(i - (int64_t)rl * K);
        const int64_t row = (int64_t)pi.row_base + 2 * (cd.j0 + rl) + cd.parity;
        const int64_t v = (int64_t)a.q32[row * N_COEF + a.kept_list[k]];
        const uint32_t slot = ep + __popc(m & lt_mask);
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

// ------------------------------------------------------------------------------ decode
// Decoder lookup: lut[s][b] = the symbol whose slot range holds slot b * 64.
__global__ void k_build_lut(const uint16_t *cdf, uint16_t *lut) {
  const int s = blockIdx.x;
  const uint16_t *tab = cdf + s * N_SYM;
  for (int b = threadIdx.x; b < LUT_SIZE; b += blockDim.x) {
    const uint32_t slot = (uint32_t)b << (16 - LUT_BITS);
    int lo = 0, hi = N_SYM;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (tab[mid] <= slot) lo = mid; else hi = mid;
    }
    lut[s * LUT_SIZE + b] = (uint16_t)lo;
  }
}

// Decodes one pass (parity) of chunks, one warp per chunk.  The loop carries only the
// rANS states: for each symbol it finds the table entry holding the state's slot, updates
// the state, renormalises, and writes the slot (slot order) for the finishing kernel.
struct RansDecArgs {
  const ChunkDesc *chunks;
  int chunk0, n_chunks;  // this pass: chunks [chunk0, chunk0 + n_chunks)
  int k_eff;
  const uint8_t *kept_scale;
  const uint16_t *cdf;
  const uint16_t *lut;
  const uint8_t *blob;
  uint64_t off_streams;
  const uint32_t *offs;  // chunk table inside the blob
  uint16_t *slots;       // slot order: the decoded slot of every symbol
  const int32_t *valid;  // header check result (1 = ok)
  int32_t *status;
};

__global__ void __launch_bounds__(RANS_WARPS * 32) rans_decode_kernel(RansDecArgs a) {
  extern __shared__ __align__(16) uint8_t sm[];
  uint16_t *s_cdf = reinterpret_cast<uint16_t *>(sm);
  uint16_t *s_lut = reinterpret_cast<uint16_t *>(sm + CDF_SMEM_BYTES);
  uint8_t *s_scale = sm + CDF_SMEM_BYTES + LUT_SMEM_BYTES;
  if (*a.valid != 1) return;
  copy_smem16(s_cdf, a.cdf, CDF_SMEM_BYTES);
  copy_smem16(s_lut, a.lut, LUT_SMEM_BYTES);
  copy_smem16(s_scale, a.kept_scale, N_COEF);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int wi = blockIdx.x * RANS_WARPS + (threadIdx.x >> 5);
  if (wi >= a.n_chunks) return;
  const int ci = a.chunk0 + wi;
  const ChunkDesc cd = a.chunks[ci];
  const int K = a.k_eff;
  const uint32_t S = (uint32_t)cd.nrows * (uint32_t)K;  // < 2^20
  const int T = (int)((S + 31) / 32);
  const uint64_t beg = a.off_streams + a.offs[ci];
  const uint64_t end = a.off_streams + a.offs[ci + 1];
  const uint8_t *sec = a.blob + beg;
  const uint32_t ne = reinterpret_cast<const uint32_t *>(sec)[32];
  if ((end - beg) < CHUNK_FIXED_BYTES || (uint64_t)CHUNK_FIXED_BYTES + 8ull * ne > (end - beg)) {
    if (lane == 0) atomicExch(a.status, DCKV_ECORRUPT);
    return;
  }
  uint32_t x = reinterpret_cast<const uint32_t *>(sec)[lane];
  const uint16_t *wd = reinterpret_cast<const uint16_t *>(sec + CHUNK_FIXED_BYTES + 8ull * ne);
  const uint32_t n_wd = (uint32_t)(((end - beg) - CHUNK_FIXED_BYTES - 8ull * ne) / 2);
  uint16_t *out = a.slots + cd.sym_base;
  // words pass through a 96-word register ring: lane j holds words wb + j, wb + 32 + j and
  // (prefetched) wb + 64 + j
  uint32_t wb = 0, wp = 0;
  uint32_t w0 = lane < n_wd ? wd[lane] : 0u;
  uint32_t w1 = 32 + lane < n_wd ? wd[32 + lane] : 0u;
  uint32_t w2 = 64 + lane < n_wd ? wd[64 + lane] : 0u;
  const uint32_t lt_mask = (1u << lane) - 1u;
  bool bad = x < RANS_L;
  int k = K > 0 ? lane % K : 0;
  for (int t0 = 0; t0 < T && !bad; t0 += 16) {
#pragma unroll 4
    for (int u = 0; u < 16; ++u) {
      const int t = t0 + u;
      if (t >= T) break;
      const uint32_t i = (uint32_t)t * 32u + lane;
      const bool valid = i < S;
      bool need = false;
      if (valid) {
        const int s = s_scale[k];
        const uint16_t *tab = s_cdf + s * N_SYM;
        const uint32_t slot = x & 0xFFFFu;
        const int b = (int)(slot >> (16 - LUT_BITS));
        int lo = s_lut[s * LUT_SIZE + b];
        int hi = b + 1 < LUT_SIZE ? s_lut[s * LUT_SIZE + b + 1] : N_SYM - 1;  // answer in [lo, hi]
        while (hi > lo) {
          const int mid = (lo + hi + 1) >> 1;
          if (tab[mid] <= slot) lo = mid; else hi = mid - 1;
        }
        const uint32_t c = tab[lo];
        const uint32_t f = cdf_at(tab, lo + 1) - c;
        x = f * (x >> 16) + slot - c;
        need = x < RANS_L;
        out[i] = (uint16_t)slot;
      }
      const uint32_t m = __ballot_sync(0xffffffffu, need);
      const uint32_t p = (wp - wb) + __popc(m & lt_mask);  // < 64 by construction
      const uint32_t v0 = __shfl_sync(0xffffffffu, w0, p & 31);
      const uint32_t v1 = __shfl_sync(0xffffffffu, w1, p & 31);
      if (need) x = (x << 16) | (p < 32 ? v0 : v1);
      wp += __popc(m);
      if (wp - wb >= 32) {  // slide the ring by 32 words
        w0 = w1;
        w1 = w2;
        wb += 32;
        w2 = wb + 64 + lane < n_wd ? wd[wb + 64 + lane] : 0u;
      }
      k += 32;
      if (K > 0)
        while (k >= K) k -= K;
    }
    bad = __any_sync(0xffffffffu, bad || wp > n_wd);
  }
  // the stream must be consumed exactly: every state back at L, at most one zero pad
  // word left (escape values are checked by the finishing kernel)
  if (!bad) {
    if (x != RANS_L) bad = true;
    if (!(wp == n_wd || (wp + 1 == n_wd && wd[n_wd - 1] == 0))) bad = true;
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicExch(a.status, DCKV_ECORRUPT);
}

// Finishing a decoded pass, parallel over rows.  Step 1 (one block per row): symbol from
// (scale, slot) through the lookup table, written back over the slot; escapes counted per
// row.  Step 2 (one warp per row): the row's first escape index is the escape count of
// the chunk's earlier rows; escapes are matched in symbol order to the chunk's 64-bit
// values; q = symbol - 254 + centre is written as fp16 (exact below 2048) for the inverse
// GEMM, bf16(q) into padded even rows for the odd mean model, and exact int32 values of
// codes with |q| >= 2048 (their rows are listed for a fix-up).
__global__ void __launch_bounds__(256) k_decode_symbols(int64_t slot0, int64_t n_slots, int k_eff,
                                                        const uint8_t *kept_scale, const uint16_t *cdf,
                                                        const uint16_t *lut, uint16_t *slots, uint32_t *row_esc,
                                                        const int32_t *valid) {
  extern __shared__ __align__(16) uint8_t sm[];
  uint16_t *s_cdf = reinterpret_cast<uint16_t *>(sm);
  uint16_t *s_lut = reinterpret_cast<uint16_t *>(sm + CDF_SMEM_BYTES);
  __shared__ uint32_t cnt;
  if (*valid != 1) return;
  copy_smem16(s_cdf, cdf, CDF_SMEM_BYTES);
  copy_smem16(s_lut, lut, LUT_SMEM_BYTES);
  __syncthreads();
  for (int64_t r = blockIdx.x; r < n_slots; r += gridDim.x) {
    if (threadIdx.x == 0) cnt = 0;
    __syncthreads();
    uint16_t *sl = slots + (slot0 + r) * k_eff;
    uint32_t esc = 0;
    for (int k = threadIdx.x; k < k_eff; k += blockDim.x) {
      const int s = kept_scale[k];
      const uint16_t *tab = s_cdf + s * N_SYM;
      const uint32_t slot = sl[k];
      const int b = (int)(slot >> (16 - LUT_BITS));
      int lo = s_lut[s * LUT_SIZE + b];
      int hi = b + 1 < LUT_SIZE ? s_lut[s * LUT_SIZE + b + 1] : N_SYM - 1;
      while (hi > lo) {
        const int mid = (lo + hi + 1) >> 1;
        if (tab[mid] <= slot) lo = mid; else hi = mid - 1;
      }
      sl[k] = (uint16_t)lo;
      esc += (lo == ESC_SYM);
    }
    for (int o = 16; o; o >>= 1) esc += __shfl_xor_sync(0xffffffffu, esc, o);
    if ((threadIdx.x & 31) == 0 && esc) atomicAdd(&cnt, esc);
    __syncthreads();
    if (threadIdx.x == 0) row_esc[slot0 + r] = cnt;
    __syncthreads();
  }
}

struct DecCodesArgs {
  const ChunkDesc *chunks;
  const PromptInfo *prompts;
  int chunk0, n_chunks;
  int chunk_rows;
  int k_eff;
  const int16_t *kept_list;
  const int8_t *cen8;
  const uint16_t *syms;     // slot order
  const uint32_t *row_esc;  // per slot row
  const uint8_t *blob;
  uint64_t off_streams;
  const uint32_t *offs;
  __half *q16;
  __nv_bfloat16 *qe;
  int32_t *qbig;
  uint32_t *bigflag;
  int32_t *biglist;
  uint32_t *bigcount;
  const int32_t *valid;
  int32_t *status;
};

__global__ void __launch_bounds__(256) k_decode_codes(DecCodesArgs a) {
  if (*a.valid != 1) return;
  const int lane = threadIdx.x & 31;
  const int nw = blockDim.x >> 5;
  const uint32_t lt_mask = (1u << lane) - 1u;
  const int total_rows = a.n_chunks * a.chunk_rows;  // rows of the pass, chunk-major (some absent)
  for (int wr = blockIdx.x * nw + (threadIdx.x >> 5); wr < total_rows; wr += gridDim.x * nw) {
    const int ci = a.chunk0 + wr / a.chunk_rows;
    const int rl = wr % a.chunk_rows;
    const ChunkDesc cd = a.chunks[ci];
    if (rl >= cd.nrows) continue;
    const PromptInfo pi = a.prompts[cd.prompt];
    const int K = a.k_eff;
    const int64_t slot_row = cd.sym_base / (K > 0 ? K : 1) + rl;
    const uint8_t *sec = a.blob + a.off_streams + a.offs[ci];
    const uint32_t ne = reinterpret_cast<const uint32_t *>(sec)[32];
    const uint32_t *ev = reinterpret_cast<const uint32_t *>(sec + CHUNK_FIXED_BYTES);
    uint32_t ep = 0;
    for (int r = 0; r < rl; ++r) ep += a.row_esc[slot_row - rl + r];
    const uint16_t *sy = a.syms + slot_row * K;
    const int8_t *ce = a.cen8 + slot_row * K;
    const int j = cd.j0 + rl;
    const int64_t row = (int64_t)pi.row_base + 2 * j + cd.parity;
    __half *q16 = a.q16 + row * N_COEF;
    __nv_bfloat16 *qe = cd.parity == 0 ? a.qe + (int64_t)(pi.ebase + j) * N_COEF : nullptr;
    bool bad = false;
    for (int k0 = 0; k0 < K; k0 += 32) {
      const int k = k0 + lane;
      const bool valid = k < K;
      const int sym = valid ? sy[k] : 0;
      const bool is_esc = valid && sym == ESC_SYM;
      const uint32_t me = __ballot_sync(0xffffffffu, is_esc);
      int q = valid ? sym - R_MAX + ce[k] : 0;
      if (is_esc) {
        const uint32_t e = ep + __popc(me & lt_mask);
        if (e < ne) {
          const int64_t sv = (int64_t)((uint64_t)ev[2 * e] | ((uint64_t)ev[2 * e + 1] << 32));
          q = (int)max(min(sv, (int64_t)INT32_MAX), (int64_t)INT32_MIN);
          if (sv >= -ESC_LIMIT && sv <= ESC_LIMIT) bad = true;  // not an escape value
        } else {
          bad = true;
        }
      }
      ep += __popc(me);
      if (valid) {
        const int comp = a.kept_list[k];
        q16[comp] = __float2half_rn((float)q);
        if (qe) qe[comp] = __float2bfloat16_rn((float)q);
        if (q >= BIG_CODE || q <= -BIG_CODE) {
          a.qbig[row * N_COEF + comp] = q;
          if (atomicExch(&a.bigflag[row], 1u) == 0u) a.biglist[atomicAdd(a.bigcount, 1u)] = (int32_t)row;
        }
      }
    }
    // the chunk's last row checks that every escape value was used
    if (rl == cd.nrows - 1 && ep != ne) bad = true;
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicExch(a.status, DCKV_ECORRUPT);
  }
}

}  // namespace dckv
