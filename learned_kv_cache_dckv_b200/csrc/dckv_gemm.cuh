// dckv_gemm.cuh -- persistent tcgen05 GEMM for sm_100a with fused epilogues.
//
// D[m][n] = sum over segments, slabs and k of A[slab][m][k] * B[n][k]
//   m: output features (128 per tile, one TMEM lane each)
//   n: tokens / rows (bn per tile, one TMEM column each; bn <= 256, multiple of 16)
// Every operand is K-major in global memory and moved by TMA (no multicast) into
// 128-byte-swizzled shared memory, 64 elements of K per pipeline stage.  One A stage
// holds one or two "slabs" (the hi/lo parts of a split operand) that multiply the same
// B tile, so a split costs tensor-pipe time but no extra B traffic.
//
// Roles (192 threads): warp 0 issues TMA, warp 1 allocates TMEM and issues tcgen05.mma
// from one thread, warps 2..5 are the epilogue (warp w reads TMEM lanes 32*(w%4)..+31).
// Two 256-column fp32 accumulators in TMEM let the epilogue of one tile overlap the
// main loop of the next.  All waits are bounded (see dckv_ptx.cuh).
#pragma once
#include <cuda.h>

#include "dckv_ptx.cuh"

namespace dckv {

constexpr int GEMM_BM = 128;
constexpr int GEMM_BK = 64;
constexpr int GEMM_MAX_BN = 256;
constexpr int GEMM_THREADS = 192;
constexpr int GEMM_SLAB_BYTES = GEMM_BM * GEMM_BK * 2;         // 16 KiB
constexpr int GEMM_B_BYTES = GEMM_MAX_BN * GEMM_BK * 2;        // 32 KiB
constexpr int GEMM_MAX_SEG = 3;

struct GemmSeg {
  int a_map;        // 0 or 1: which A tensor map
  int a_slab0;      // first slab (3rd coordinate of the A map)
  int n_slab;       // slabs loaded per stage (must equal that map's box depth)
  int a_k0;         // K offset into A (elements)
  int b_map;        // 0 or 1: which B tensor map
  int b_row_shift;  // added to the tile's first row in B
  int b_k0;         // K offset into B (elements)
  int k_steps;      // 64-wide K steps
};

struct GemmProblem {
  int m_tiles;  // M / 128
  int n_rows;   // rows of B covered by the output (tile rows beyond are ignored)
  int bn;       // N tile
  int n_tiles;  // ceil(n_rows / bn)
  int n_seg;
  GemmSeg seg[GEMM_MAX_SEG];
  uint32_t idesc;
  int *status;  // device int32; DCKV_ETIMEOUT (5) is written on a timed-out wait
};

template <int MAX_SLABS, int BN_MAX = GEMM_MAX_BN>
struct GemmSmem {
  static constexpr int STAGE_BYTES = MAX_SLABS * GEMM_SLAB_BYTES + BN_MAX * GEMM_BK * 2;
};

// Epi must provide:
//   struct Params;   static constexpr int SMEM_BYTES;
//   __device__ static void tile(const Params&, char* scratch, int mt, int n0, int n_valid,
//                               uint32_t tmem_acc, int ew, int lane, int et)
// `tile` is called by all 128 epilogue threads (et = 0..127, ew = TMEM lane quarter) and
// reads the accumulator for its rows with tcgen05.ld; it may use named barrier 1.
template <class Epi, int STAGES, int MAX_SLABS>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1,
                const GemmProblem prob, const typename Epi::Params ep) {
  extern __shared__ __align__(1024) uint8_t dyn_smem[];
  constexpr int STAGE_BYTES = GemmSmem<MAX_SLABS>::STAGE_BYTES;
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
  uint8_t *stages = base;
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(base + STAGES * STAGE_BYTES);
  uint64_t *empty_bar = full_bar + STAGES;
  uint64_t *acc_full = empty_bar + STAGES;
  uint64_t *acc_empty = acc_full + 2;
  uint32_t *tmem_base_smem = reinterpret_cast<uint32_t *>(acc_empty + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_base_smem + 1);
  char *epi_scratch = reinterpret_cast<char *>(base + STAGES * STAGE_BYTES + 1024);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int total_tiles = prob.m_tiles * prob.n_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 128);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA0);
    prefetch_tmap(&tmA1);
    prefetch_tmap(&tmB0);
    prefetch_tmap(&tmB1);
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_smem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_base_smem;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
        const int mt = t % prob.m_tiles;
        const int nt = t / prob.m_tiles;
        const int n0 = nt * prob.bn;
        for (int si = 0; si < prob.n_seg; ++si) {
          const GemmSeg sg = prob.seg[si];
          const void *ta = sg.a_map ? (const void *)&tmA1 : (const void *)&tmA0;
          const void *tb = sg.b_map ? (const void *)&tmB1 : (const void *)&tmB0;
          const uint32_t bytes = (uint32_t)(sg.n_slab * GEMM_SLAB_BYTES + prob.bn * GEMM_BK * 2);
          for (int ks = 0; ks < sg.k_steps; ++ks) {
            if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag)) goto producer_done;
            uint8_t *sa = stages + stage * STAGE_BYTES;
            uint8_t *sb = sa + MAX_SLABS * GEMM_SLAB_BYTES;
            mbar_arrive_expect_tx(&full_bar[stage], bytes);
            tma_load_3d(sa, ta, &full_bar[stage], sg.a_k0 + ks * GEMM_BK, mt * GEMM_BM, sg.a_slab0);
            tma_load_2d(sb, tb, &full_bar[stage], sg.b_k0 + ks * GEMM_BK, n0 + sg.b_row_shift);
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
    producer_done:;
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * GEMM_MAX_BN);
        uint32_t accumulate = 0;
        bool ok = true;
        for (int si = 0; si < prob.n_seg && ok; ++si) {
          const GemmSeg sg = prob.seg[si];
          for (int ks = 0; ks < sg.k_steps; ++ks) {
            if (!mbar_wait(&full_bar[stage], phase, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sa = smem_u32(stages + stage * STAGE_BYTES);
            const uint32_t sb = sa + MAX_SLABS * GEMM_SLAB_BYTES;
            for (int sl = 0; sl < sg.n_slab; ++sl) {
#pragma unroll
              for (int kk = 0; kk < GEMM_BK / 16; ++kk) {
                umma_f16(d_tmem, sw128_desc(sa + sl * GEMM_SLAB_BYTES + kk * 32), sw128_desc(sb + kk * 32),
                         prob.idesc, accumulate);
                accumulate = 1;
              }
            }
            umma_commit(&empty_bar[stage]);
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
        if (!ok) break;
        umma_commit(&acc_full[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int et = threadIdx.x - 64;  // 0..127
    const int ew = warp & 3;          // TMEM lane quarter this warp may access
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
      if (et == 0) mbar_wait(&acc_full[acc], acc_phase, abort_flag);
      named_bar_sync(1, 128);
      if (*abort_flag) break;
      tc_fence_after();
      const int mt = t % prob.m_tiles;
      const int nt = t / prob.m_tiles;
      const int n0 = nt * prob.bn;
      const int n_valid = min(prob.bn, prob.n_rows - n0);
      const uint32_t tacc = tmem_base + ((uint32_t)(ew * 32) << 16) + (uint32_t)(acc * GEMM_MAX_BN);
      Epi::tile(ep, epi_scratch, mt, n0, n_valid, prob.bn, tacc, ew, lane, et);
      tc_fence_before();
      mbar_arrive(&acc_empty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  __syncthreads();
  if (*abort_flag && threadIdx.x == 0 && prob.status) atomicExch(prob.status, 5);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

template <class Epi, int STAGES, int MAX_SLABS>
constexpr int gemm_smem_bytes() {
  return 1024 /*align slack*/ + STAGES * GemmSmem<MAX_SLABS>::STAGE_BYTES + 1024 /*barriers*/ + Epi::SMEM_BYTES;
}

// ------------------------------------------------------------------------------------------
// Chunk-accumulated variant (bn = 128).  The tensor core sums each MMA's products into the
// fp32 accumulator with truncation, so over a long K the error grows with the number of
// MMA steps times the accumulator's ulp.  Here every CHUNK_STEPS * 64 elements of K go into
// a fresh TMEM partial P (two alternate, columns 0-127 and 128-255), and the epilogue warps
// add each partial into a TMEM running total T (two alternate per tile, columns 256-383
// and 384-511) with fp32 round-to-nearest adds.  After a tile's last chunk, Epi::tile reads
// its totals from T.  Eight epilogue warps: warp w >= 2 owns TMEM lane quarter w % 4 and
// column half (w - 2) / 4 (64 columns).
constexpr int GEMMC_THREADS = 320;
constexpr int GEMMC_BN = 128;

template <class Epi, int STAGES, int MAX_SLABS, int CHUNK_STEPS>
__global__ void __launch_bounds__(GEMMC_THREADS, 1)
    gemm_chunked_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                        const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1,
                        const GemmProblem prob, const typename Epi::Params ep) {
  extern __shared__ __align__(1024) uint8_t dyn_smem[];
  constexpr int STAGE_BYTES = GemmSmem<MAX_SLABS, GEMMC_BN>::STAGE_BYTES;
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
  uint8_t *stages = base;
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(base + STAGES * STAGE_BYTES);
  uint64_t *empty_bar = full_bar + STAGES;
  uint64_t *part_full = empty_bar + STAGES;
  uint64_t *part_empty = part_full + 2;
  uint32_t *tmem_base_smem = reinterpret_cast<uint32_t *>(part_empty + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_base_smem + 1);
  char *epi_scratch = reinterpret_cast<char *>(base + STAGES * STAGE_BYTES + 1024);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int total_tiles = prob.m_tiles * prob.n_tiles;
  int ksteps = 0;
  for (int si = 0; si < prob.n_seg; ++si) ksteps += prob.seg[si].k_steps;
  const int n_chunks = (ksteps + CHUNK_STEPS - 1) / CHUNK_STEPS;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&part_full[a], 1);
      mbar_init(&part_empty[a], 256);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA0);
    prefetch_tmap(&tmA1);
    prefetch_tmap(&tmB0);
    prefetch_tmap(&tmB1);
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_smem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_base_smem;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
        const int mt = t % prob.m_tiles;
        const int n0 = (t / prob.m_tiles) * prob.bn;
        for (int si = 0; si < prob.n_seg; ++si) {
          const GemmSeg sg = prob.seg[si];
          const void *ta = sg.a_map ? (const void *)&tmA1 : (const void *)&tmA0;
          const void *tb = sg.b_map ? (const void *)&tmB1 : (const void *)&tmB0;
          const uint32_t bytes = (uint32_t)(sg.n_slab * GEMM_SLAB_BYTES + prob.bn * GEMM_BK * 2);
          for (int ks = 0; ks < sg.k_steps; ++ks) {
            if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag)) goto producer_done;
            uint8_t *sa = stages + stage * STAGE_BYTES;
            uint8_t *sb = sa + MAX_SLABS * GEMM_SLAB_BYTES;
            mbar_arrive_expect_tx(&full_bar[stage], bytes);
            tma_load_3d(sa, ta, &full_bar[stage], sg.a_k0 + ks * GEMM_BK, mt * GEMM_BM, sg.a_slab0);
            tma_load_2d(sb, tb, &full_bar[stage], sg.b_k0 + ks * GEMM_BK, n0 + sg.b_row_shift);
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
    producer_done:;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int pb = 0;
      uint32_t pph = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
        int in_chunk = 0, done = 0;
        uint32_t d_tmem = 0, accumulate = 0;
        for (int si = 0; si < prob.n_seg && ok; ++si) {
          const GemmSeg sg = prob.seg[si];
          for (int ks = 0; ks < sg.k_steps; ++ks) {
            if (in_chunk == 0) {
              if (!mbar_wait(&part_empty[pb], pph ^ 1u, abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
              d_tmem = tmem_base + (uint32_t)(pb * GEMMC_BN);
              accumulate = 0;
            }
            if (!mbar_wait(&full_bar[stage], phase, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sa = smem_u32(stages + stage * STAGE_BYTES);
            const uint32_t sb = sa + MAX_SLABS * GEMM_SLAB_BYTES;
            for (int sl = 0; sl < sg.n_slab; ++sl) {
#pragma unroll
              for (int kk = 0; kk < GEMM_BK / 16; ++kk) {
                umma_f16(d_tmem, sw128_desc(sa + sl * GEMM_SLAB_BYTES + kk * 32), sw128_desc(sb + kk * 32),
                         prob.idesc, accumulate);
                accumulate = 1;
              }
            }
            umma_commit(&empty_bar[stage]);
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
            ++done;
            if (++in_chunk == CHUNK_STEPS || done == ksteps) {
              umma_commit(&part_full[pb]);
              in_chunk = 0;
              if (++pb == 2) {
                pb = 0;
                pph ^= 1u;
              }
            }
          }
        }
      }
    }
  } else {
    const int et = threadIdx.x - 64;  // 0..255
    const int ew = warp & 3;
    const int half = (warp - 2) >> 2;
    const uint32_t lane_base = (uint32_t)(ew * 32) << 16;
    int pb = 0, tbuf = 0;
    uint32_t pph = 0;
    bool stop = false;
    for (int t = blockIdx.x; t < total_tiles && !stop; t += gridDim.x) {
      const int mt = t % prob.m_tiles;
      const int n0 = (t / prob.m_tiles) * prob.bn;
      const int n_valid = min(prob.bn, prob.n_rows - n0);
      const uint32_t tot = tmem_base + lane_base + (uint32_t)(2 * GEMMC_BN + tbuf * GEMMC_BN + half * 64);
      for (int ch = 0; ch < n_chunks; ++ch) {
        if (!mbar_wait(&part_full[pb], pph, abort_flag)) {
          stop = true;
          break;
        }
        tc_fence_after();
        const uint32_t part = tmem_base + lane_base + (uint32_t)(pb * GEMMC_BN + half * 64);
#pragma unroll 1
        for (int g = 0; g < 2; ++g) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(part + g * 32, r);
          if (ch > 0) {
            uint32_t s[32];
            tmem_ld_32x32b_x32(tot + g * 32, s);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) + __uint_as_float(s[j]));
          } else {
            tmem_ld_wait();
          }
          tmem_st_32x32b_x32(tot + g * 32, r);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&part_empty[pb]);
        if (++pb == 2) {
          pb = 0;
          pph ^= 1u;
        }
      }
      if (stop) break;
      tc_fence_after();
      Epi::tile(ep, epi_scratch, mt, n0, n_valid, half * 64, tot, ew, lane, et);
      tbuf ^= 1;
    }
  }

  __syncthreads();
  if (*abort_flag && threadIdx.x == 0 && prob.status) atomicExch(prob.status, 5);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

template <class Epi, int STAGES, int MAX_SLABS>
constexpr int gemm_chunked_smem_bytes() {
  return 1024 + STAGES * GemmSmem<MAX_SLABS, GEMMC_BN>::STAGE_BYTES + 1024 + Epi::SMEM_BYTES;
}

}  // namespace dckv
