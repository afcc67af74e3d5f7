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
  int k_split;  // CTA-pair kernel, one segment: K cut into k_split parts, each its own tile
                // (the epilogue writes part ks of the sum; 0 or 1: no split)
  int first_chunk;  // chunk-accumulated kernel: K steps of a tile's first TMEM partial (0: the
                    // kernel's CHUNK_STEPS, like every later partial)
};

// What an epilogue sees of one output tile.  The epilogue threads form groups of 128 (four
// warps, one per TMEM lane quarter); group grp of n_grp takes the tile's column chunks k
// with k % n_grp == grp (each epilogue fixes its chunk width), synchronises on named
// barrier `bar` and owns `scratch` (Epi::SMEM_BYTES of shared memory).
struct EpiCtx {
  int mt;            // 128-row output-feature tile
  int n0, n_valid;   // first token row of the tile, valid columns
  int bn;            // tile width
  uint32_t tacc;     // TMEM address of column 0 for this warp's lane quarter
  int ew, lane;      // lane quarter (warp % 4), lane
  int et;            // thread index in the group, 0..127
  int grp, n_grp;
  int bar;
  char *scratch;
  int ks = 0;        // split-K part of this tile (CTA-pair kernel with prob.k_split > 1)
};

template <int MAX_SLABS, int BN_MAX = GEMM_MAX_BN>
struct GemmSmem {
  static constexpr int STAGE_BYTES = MAX_SLABS * GEMM_SLAB_BYTES + BN_MAX * GEMM_BK * 2;
};

// Teardown state, in the barrier area after the stage and accumulator barriers.  A wait that
// gives up (a timeout) makes the CTA leave its role loop early, possibly with TMA copies into
// its shared memory and MMAs on its TMEM still in flight; before it leaves, the CTA waits
// (bounded) for all of them:
//   - copies: the producer counts the items (K steps) it issued and remembers each stage's
//     last transaction bytes; every item's copies are counted on a full barrier, so waiting
//     for the phases of the last STAGES items (earlier ones were consumed, hence complete)
//     covers every copy still in flight;
//   - MMAs: the issuer commits once more, to drain_bar, which completes when every MMA it
//     issued has.
// In the CTA pair each producer loads its own half of an item into its own shared memory,
// counted on the leader's full barrier, and either producer may stop first.  The peer
// therefore hands the leader its item count and bytes; for the items that only one of them
// issued the leader settles the barrier's count (complete_tx for a half that will not come,
// arrive with the peer's bytes for an item it never armed), drains the phases, and a last
// cluster barrier holds the peer until then.  Without a timeout none of this runs.
template <int STAGES>
struct GemmTail {
  uint64_t drain_bar;
  uint32_t tmem_base;
  int abort;                   // this CTA's abort flag
  int peer_abort;              // the other CTA's flag, stored here by it (CTA pair)
  uint32_t peer_issued;        // the peer producer's item count (leader's copy)
  uint32_t ring[STAGES];       // transaction bytes of the last item issued into each stage
  uint32_t peer_ring[STAGES];  // the peer's ring (leader's copy)
};

// Waits for the copies of the last min(n, STAGES) of n issued items (one thread).
template <int STAGES>
__device__ __forceinline__ void drain_issued(uint64_t *full_bar, uint32_t n) {
  for (uint32_t i = n > (uint32_t)STAGES ? n - STAGES : 0u; i < n; ++i)
    mbar_drain(&full_bar[i % STAGES], (i / STAGES) & 1u);
}

// Leader of a CTA pair after an abort: settles the full barriers of the items only one
// producer issued (l: the leader's count, p: the peer's), then drains them (one thread).
// Both producers wait on releases of the same items, so |l - p| <= STAGES and each of those
// items is the last one its producer put into its stage.
template <int STAGES>
__device__ __forceinline__ void pair_drain_issued(uint64_t *full_bar, uint32_t l, uint32_t p,
                                                  const uint32_t *ring, const volatile uint32_t *peer_ring) {
  for (uint32_t i = l < p ? l : p; i < (l < p ? p : l); ++i) {
    const int s = (int)(i % STAGES);
    if (l > p)
      mbar_complete_tx(&full_bar[s], ring[s]);  // armed for both halves; the peer's never comes
    else
      mbar_arrive_expect_tx(&full_bar[s], peer_ring[s]);  // never armed: count the peer's half
  }
  drain_issued<STAGES>(full_bar, l < p ? p : l);
}

// Epi must provide:
//   struct Params;   static constexpr int SMEM_BYTES;
//   __device__ static void tile(const Params&, const EpiCtx&)
// `tile` is called by every thread of an epilogue group and reads the accumulator for its
// rows with tcgen05.ld; here there is one group (named barrier 1).
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
  GemmTail<STAGES> *tail = reinterpret_cast<GemmTail<STAGES> *>(acc_empty + 2);
  static_assert(sizeof(uint64_t) * (2 * STAGES + 4) + sizeof(GemmTail<STAGES>) <= 1024, "barrier area");
  uint32_t *tmem_base_smem = &tail->tmem_base;
  volatile int *abort_flag = &tail->abort;
  char *epi_scratch = reinterpret_cast<char *>(base + STAGES * STAGE_BYTES + 1024);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int total_tiles = prob.m_tiles * prob.n_tiles;
  uint32_t n_issued = 0;  // items the producer (thread 0) issued

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 128);
    }
    mbar_init(&tail->drain_bar, 1);
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
            ++n_issued;
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
      const EpiCtx cx{mt, n0, n_valid, prob.bn, tacc, ew, lane, et, 0, 1, 1, epi_scratch};
      Epi::tile(ep, cx);
      tc_fence_before();
      mbar_arrive(&acc_empty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  __syncthreads();
  if (*abort_flag) {  // a wait gave up: the copies and MMAs this CTA issued finish first
    if (threadIdx.x == 0) drain_issued<STAGES>(full_bar, n_issued);
    if (warp == 1 && lane == 0) {
      umma_commit(&tail->drain_bar);
      mbar_drain(&tail->drain_bar, 0);
    }
    __syncthreads();
    if (threadIdx.x == 0 && prob.status) atomicExch(prob.status, 5);
  }
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
// CTA-pair variant (cta_group::2).  A cluster of two CTAs owns a 256 x bn output tile: CTA
// r holds A rows 128 r .. 128 r + 127 of the tile and B rows r bn/2 .. r bn/2 + bn/2 - 1, so
// each SM stages half the B tile that a 1-CTA tile of the same width needs, and the pair
// runs one M = 256 MMA per K step.  The leader (rank 0) waits for both halves on its own
// full barrier, issues every MMA and commits to the barriers of both CTAs; each CTA drains
// its own TMEM rows (feature tile 2 * pair_tile + r) with the same epilogue as above.
// prob.m_tiles counts 128-row tiles and must be even; prob.bn <= 256, bn / 2 a multiple of 8.
constexpr int GEMM_B_HALF_BYTES = (GEMM_MAX_BN / 2) * GEMM_BK * 2;  // 16 KiB

// End of a CTA-pair kernel, after every role loop of this CTA has left (__syncthreads):
// the CTAs exchange their abort flags (and the peer its item count and ring) and pass a
// cluster barrier, so that neither leaves while the other may still signal its barriers or
// read its TMEM; after an abort in either CTA the drain described at GemmTail follows.
template <int STAGES>
__device__ __forceinline__ void pair_teardown(GemmTail<STAGES> *tail, uint64_t *full_bar, uint32_t n_issued,
                                              uint32_t rank, int warp, int lane, int *status) {
  const volatile GemmTail<STAGES> *vt = tail;
  if (threadIdx.x == 0) {
    st_shared_cluster_u32(mapa_shared(smem_u32(&tail->peer_abort), rank ^ 1u), (uint32_t)vt->abort);
    if (rank == 1) {
      st_shared_cluster_u32(mapa_shared(smem_u32(&tail->peer_issued), 0), n_issued);
      for (int s = 0; s < STAGES; ++s)
        st_shared_cluster_u32(mapa_shared(smem_u32(&tail->peer_ring[s]), 0), tail->ring[s]);
    }
  }
  cluster_sync();
  if (vt->abort || vt->peer_abort) {
    if (rank == 0 && warp == 1 && lane == 0) umma_commit_pair(&tail->drain_bar);
    if (rank == 0 && threadIdx.x == 0)
      pair_drain_issued<STAGES>(full_bar, n_issued, vt->peer_issued, tail->ring, vt->peer_ring);
    if (warp == 1 && lane == 0) mbar_drain(&tail->drain_bar, 0);
    __syncthreads();
    cluster_sync();
    if (vt->abort && threadIdx.x == 0 && status) atomicExch(status, 5);
  }
}

template <int MAX_SLABS, int BN = GEMM_MAX_BN>
struct Gemm2Smem {  // one stage: the A slabs, then this CTA's half of the B tile (a multiple of 1 KiB)
  static_assert((BN / 2) % 8 == 0, "half tile must hold whole 8-row swizzle atoms");
  static constexpr int STAGE_BYTES = MAX_SLABS * GEMM_SLAB_BYTES + (BN / 2) * GEMM_BK * 2;
};

template <class Epi, int STAGES, int MAX_SLABS, int EPI_WARPS, int BN_MAX = GEMM_MAX_BN>
__global__ void __launch_bounds__(64 + 32 * EPI_WARPS, 1)
    gemm2_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                 const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1,
                 const GemmProblem prob, const typename Epi::Params ep) {
  extern __shared__ __align__(1024) uint8_t dyn_smem[];
  constexpr int STAGE_BYTES = Gemm2Smem<MAX_SLABS, BN_MAX>::STAGE_BYTES;  // stages sized for tiles up to BN_MAX
  constexpr int N_GRP = EPI_WARPS / 4;
  constexpr int EPI_SCRATCH = (Epi::SMEM_BYTES + 15) & ~15;
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
  uint8_t *stages = base;
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(base + STAGES * STAGE_BYTES);  // leader's counts both halves
  uint64_t *empty_bar = full_bar + STAGES;
  uint64_t *acc_full = empty_bar + STAGES;
  uint64_t *acc_empty = acc_full + 2;  // leader's: one arrival per epilogue warp of either CTA
  GemmTail<STAGES> *tail = reinterpret_cast<GemmTail<STAGES> *>(acc_empty + 2);
  static_assert(sizeof(uint64_t) * (2 * STAGES + 4) + sizeof(GemmTail<STAGES>) <= 1024, "barrier area");
  uint32_t *tmem_base_smem = &tail->tmem_base;
  volatile int *abort_flag = &tail->abort;
  char *epi_scratch = reinterpret_cast<char *>(base + STAGES * STAGE_BYTES + 1024);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;
  const int m_pairs = prob.m_tiles >> 1;
  const int n_split = prob.k_split > 1 ? prob.k_split : 1;
  const int mn_tiles = m_pairs * prob.n_tiles;
  const int total_tiles = mn_tiles * n_split;
  const int half_bn = prob.bn >> 1;
  uint32_t n_issued = 0;  // items this CTA's producer (thread 0) issued

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 2 * EPI_WARPS);
    }
    mbar_init(&tail->drain_bar, 1);
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
    tmem_alloc_pair(tmem_base_smem, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers are initialised before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_base_smem;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = pair; t < total_tiles && ok; t += n_pairs) {
        const int mp = (t % mn_tiles) % m_pairs;
        const int n0 = ((t % mn_tiles) / m_pairs) * prob.bn;
        const int part = t / mn_tiles;
        for (int si = 0; si < prob.n_seg && ok; ++si) {
          const GemmSeg sg = prob.seg[si];
          const void *ta = sg.a_map ? (const void *)&tmA1 : (const void *)&tmA0;
          const void *tb = sg.b_map ? (const void *)&tmB1 : (const void *)&tmB0;
          const uint32_t bytes = (uint32_t)(sg.n_slab * GEMM_SLAB_BYTES + half_bn * GEMM_BK * 2);
          const int per = (sg.k_steps + n_split - 1) / n_split;
          const int k_beg = part * per, k_end = min(sg.k_steps, k_beg + per);
          for (int ks = k_beg; ks < k_end; ++ks) {
            if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag)) {
              ok = false;
              break;
            }
            uint8_t *sa = stages + stage * STAGE_BYTES;
            uint8_t *sb = sa + MAX_SLABS * GEMM_SLAB_BYTES;
            const uint32_t fb = mapa_shared(smem_u32(&full_bar[stage]), 0);
            if (rank == 0) mbar_arrive_expect_tx(&full_bar[stage], 2 * bytes);
            tma_load_3d_pair(sa, ta, fb, sg.a_k0 + ks * GEMM_BK, (2 * mp + (int)rank) * GEMM_BM, sg.a_slab0);
            tma_load_2d_pair(sb, tb, fb, sg.b_k0 + ks * GEMM_BK, n0 + (int)rank * half_bn + sg.b_row_shift);
            tail->ring[stage] = bytes;
            ++n_issued;
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
      // wait until the leader has released every stage, so that no commit from it is
      // still in flight towards this CTA's barriers when the CTA exits
      for (int i = 0; i < STAGES && ok; ++i) {
        if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag)) break;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (leader only)
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int t = pair; t < total_tiles; t += n_pairs) {
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * GEMM_MAX_BN);
        uint32_t accumulate = 0;
        bool ok = true;
        const int part = t / mn_tiles;
        for (int si = 0; si < prob.n_seg && ok; ++si) {
          const GemmSeg sg = prob.seg[si];
          const int per = (sg.k_steps + n_split - 1) / n_split;
          const int k_beg = part * per, k_end = min(sg.k_steps, k_beg + per);
          for (int ks = k_beg; ks < k_end; ++ks) {
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
                umma_f16_pair(d_tmem, sw128_desc(sa + sl * GEMM_SLAB_BYTES + kk * 32), sw128_desc(sb + kk * 32),
                              prob.idesc, accumulate);
                accumulate = 1;
              }
            }
            umma_commit_pair(&empty_bar[stage]);
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
        if (!ok) break;
        umma_commit_pair(&acc_full[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    const int grp = (warp - 2) >> 2;
    const int et = threadIdx.x - 64 - 128 * grp;  // 0..127 within the group
    const int ew = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = pair; t < total_tiles; t += n_pairs) {
      if (et == 0) mbar_wait(&acc_full[acc], acc_phase, abort_flag);
      named_bar_sync(1 + grp, 128);
      if (*abort_flag) break;
      tc_fence_after();
      const int mp = (t % mn_tiles) % m_pairs;
      const int n0 = ((t % mn_tiles) / m_pairs) * prob.bn;
      const int n_valid = min(prob.bn, prob.n_rows - n0);
      const uint32_t tacc = tmem_base + ((uint32_t)(ew * 32) << 16) + (uint32_t)(acc * GEMM_MAX_BN);
      const EpiCtx cx{2 * mp + (int)rank, n0, n_valid, prob.bn, tacc, ew, lane, et, grp, N_GRP, 1 + grp,
                      epi_scratch + grp * EPI_SCRATCH, t / mn_tiles};
      Epi::tile(ep, cx);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&acc_empty[acc]), 0));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  __syncthreads();
  pair_teardown<STAGES>(tail, full_bar, n_issued, rank, warp, lane, prob.status);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

template <class Epi, int STAGES, int MAX_SLABS, int EPI_WARPS, int BN_MAX = GEMM_MAX_BN>
constexpr int gemm2_smem_bytes() {
  return 1024 + STAGES * Gemm2Smem<MAX_SLABS, BN_MAX>::STAGE_BYTES + 1024 +
         (EPI_WARPS / 4) * ((Epi::SMEM_BYTES + 15) & ~15);
}

// ------------------------------------------------------------------------------------------
// CTA-pair, chunk-accumulated variant (transform + quantiser).  Every CHUNK_STEPS * 64
// elements of K go into a fresh TMEM partial P (two alternate, columns 0 and 256); the
// eight epilogue warps of each CTA add each partial into running totals held in registers
// (fp32 round-to-nearest adds, in chunk order) -- warp w >= 2 owns lane quarter w % 4 and
// column half (w - 2) / 4, BN / 2 columns -- and after a tile's last chunk hand their totals
// to Epi::finish.  Both P buffers stay free for the MMA while totals are finished.  Per-column
// metadata of a tile is staged into shared memory (Epi::stage, two buffers by tile parity)
// before its chunks are drained, so that finish reads it without global-memory latency.
// Epilogue: GEMM2C_COL_GROUPS groups of four warps, each group BN / GEMM2C_COL_GROUPS
// columns of the tile (four groups: 56 columns and totals per thread at BN = 224, so that
// the quantiser after a tile's last chunk is spread over sixteen warps and finishes within
// the two chunks the MMA runs ahead).
constexpr int GEMM2C_COL_GROUPS = 4;
constexpr int GEMM2C_THREADS = 64 + 128 * GEMM2C_COL_GROUPS;

template <class Epi, int STAGES, int MAX_SLABS, int CHUNK_STEPS, int BN>
__global__ void __launch_bounds__(GEMM2C_THREADS, 1)
    gemm2_chunked_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                         const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1,
                         const GemmProblem prob, const typename Epi::Params ep) {
  static_assert(BN % 32 == 0 && BN <= GEMM_MAX_BN, "BN / 2 must be a multiple of 16");
  static_assert(BN % (8 * GEMM2C_COL_GROUPS) == 0, "column groups of whole 8-column loads");
  constexpr int NC = BN / GEMM2C_COL_GROUPS;  // columns per epilogue thread
  extern __shared__ __align__(1024) uint8_t dyn_smem[];
  constexpr int STAGE_BYTES = Gemm2Smem<MAX_SLABS, BN>::STAGE_BYTES;
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dyn_smem) + 1023) & ~uintptr_t(1023));
  uint8_t *stages = base;
  uint64_t *full_bar = reinterpret_cast<uint64_t *>(base + STAGES * STAGE_BYTES);
  uint64_t *empty_bar = full_bar + STAGES;
  uint64_t *part_full = empty_bar + STAGES;
  uint64_t *part_empty = part_full + 2;  // leader's: one arrival per epilogue warp of either CTA
  GemmTail<STAGES> *tail = reinterpret_cast<GemmTail<STAGES> *>(part_empty + 2);
  static_assert(sizeof(uint64_t) * (2 * STAGES + 4) + sizeof(GemmTail<STAGES>) <= 1024, "barrier area");
  uint32_t *tmem_base_smem = &tail->tmem_base;
  volatile int *abort_flag = &tail->abort;
  constexpr int EPI_BUF = (Epi::SMEM_BYTES + 15) & ~15;
  char *epi_buf = reinterpret_cast<char *>(base + STAGES * STAGE_BYTES + 1024);  // two buffers

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;
  const int m_pairs = prob.m_tiles >> 1;
  const int total_tiles = m_pairs * prob.n_tiles;
  constexpr int half_bn = BN / 2;
  uint32_t n_issued = 0;  // items this CTA's producer (thread 0) issued
  int ksteps = 0;
  for (int si = 0; si < prob.n_seg; ++si) ksteps += prob.seg[si].k_steps;
  // a tile's partials: the first takes first_steps K steps, every later one CHUNK_STEPS.  The
  // MMA can run as far ahead of the epilogue as the first two partials reach, so a longer
  // first partial hides more of the previous tile's finishing epilogue.
  const int first_steps = min(ksteps, prob.first_chunk > 0 ? prob.first_chunk : CHUNK_STEPS);
  const int n_chunks = ksteps > 0 ? 1 + (ksteps - first_steps + CHUNK_STEPS - 1) / CHUNK_STEPS : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&part_full[a], 1);
      mbar_init(&part_empty[a], 2 * 4 * GEMM2C_COL_GROUPS);  // every epilogue warp of both CTAs
    }
    mbar_init(&tail->drain_bar, 1);
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
    tmem_alloc_pair(tmem_base_smem, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_base_smem;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = pair; t < total_tiles && ok; t += n_pairs) {
        const int mp = t % m_pairs;
        const int n0 = (t / m_pairs) * BN;
        for (int si = 0; si < prob.n_seg && ok; ++si) {
          const GemmSeg sg = prob.seg[si];
          const void *ta = sg.a_map ? (const void *)&tmA1 : (const void *)&tmA0;
          const void *tb = sg.b_map ? (const void *)&tmB1 : (const void *)&tmB0;
          const uint32_t bytes = (uint32_t)(sg.n_slab * GEMM_SLAB_BYTES + half_bn * GEMM_BK * 2);
          for (int ks = 0; ks < sg.k_steps; ++ks) {
            if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag)) {
              ok = false;
              break;
            }
            uint8_t *sa = stages + stage * STAGE_BYTES;
            uint8_t *sb = sa + MAX_SLABS * GEMM_SLAB_BYTES;
            const uint32_t fb = mapa_shared(smem_u32(&full_bar[stage]), 0);
            if (rank == 0) mbar_arrive_expect_tx(&full_bar[stage], 2 * bytes);
            tma_load_3d_pair(sa, ta, fb, sg.a_k0 + ks * GEMM_BK, (2 * mp + (int)rank) * GEMM_BM, sg.a_slab0);
            tma_load_2d_pair(sb, tb, fb, sg.b_k0 + ks * GEMM_BK, n0 + (int)rank * half_bn + sg.b_row_shift);
            tail->ring[stage] = bytes;
            ++n_issued;
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
      for (int i = 0; i < STAGES && ok; ++i) {
        if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag)) break;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int pb = 0;
      uint32_t pph = 0;
      bool ok = true;
      for (int t = pair; t < total_tiles && ok; t += n_pairs) {
        int in_chunk = 0, done = 0, chunk_len = first_steps;
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
              d_tmem = tmem_base + (uint32_t)(pb * 256);
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
                umma_f16_pair(d_tmem, sw128_desc(sa + sl * GEMM_SLAB_BYTES + kk * 32), sw128_desc(sb + kk * 32),
                              prob.idesc, accumulate);
                accumulate = 1;
              }
            }
            umma_commit_pair(&empty_bar[stage]);
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
            ++done;
            if (++in_chunk == chunk_len || done == ksteps) {
              umma_commit_pair(&part_full[pb]);
              in_chunk = 0;
              chunk_len = CHUNK_STEPS;
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
    const int ew = warp & 3;
    const int col0 = ((warp - 2) >> 2) * NC;
    const uint32_t lane_base = (uint32_t)(ew * 32) << 16;
    int pb = 0;
    uint32_t pph = 0;
    bool stop = false;
    int tp = 0;
    for (int t = pair; t < total_tiles && !stop; t += n_pairs, tp ^= 1) {
      const int mp = t % m_pairs;
      const int n0 = (t / m_pairs) * BN;
      const int n_valid = min(BN, prob.n_rows - n0);
      char *buf = epi_buf + tp * EPI_BUF;
      Epi::stage(ep, buf, n0, n_valid, threadIdx.x - 64, GEMM2C_THREADS - 64);
      float tot[NC];
#pragma unroll
      for (int j = 0; j < NC; ++j) tot[j] = 0.f;
      for (int ch = 0; ch < n_chunks; ++ch) {
        if (!mbar_wait(&part_full[pb], pph, abort_flag)) {
          stop = true;
          break;
        }
        tc_fence_after();
        const uint32_t part = tmem_base + lane_base + (uint32_t)(pb * 256 + col0);
        constexpr int N32 = NC / 32, REM = NC % 32;  // REM is 0, 8, 16 or 24
#pragma unroll
        for (int g = 0; g < N32; ++g) {
          uint32_t r[32];
          tmem_ld_32x32b_x16(part + (uint32_t)(g * 32), r);
          tmem_ld_32x32b_x16(part + (uint32_t)(g * 32 + 16), r + 16);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) tot[g * 32 + j] += __uint_as_float(r[j]);
        }
        if constexpr (REM > 0) {
          uint32_t r[24];
          if constexpr (REM >= 16) tmem_ld_32x32b_x16(part + (uint32_t)(N32 * 32), r);
          if constexpr (REM % 16 != 0) tmem_ld_32x32b_x8(part + (uint32_t)(N32 * 32 + (REM & 16)), r + (REM & 16));
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < REM; ++j) tot[N32 * 32 + j] += __uint_as_float(r[j]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&part_empty[pb]), 0));
        if (++pb == 2) {
          pb = 0;
          pph ^= 1u;
        }
      }
      if (stop) break;
      named_bar_sync(1, GEMM2C_THREADS - 64);  // the tile's staged metadata is visible
      Epi::template finish<NC>(ep, buf, tot, 2 * mp + (int)rank, n0, n_valid, col0, ew, lane);
    }
  }

  __syncthreads();
  pair_teardown<STAGES>(tail, full_bar, n_issued, rank, warp, lane, prob.status);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

template <class Epi, int STAGES, int MAX_SLABS, int BN>
constexpr int gemm2_chunked_smem_bytes() {
  return 1024 + STAGES * Gemm2Smem<MAX_SLABS, BN>::STAGE_BYTES + 1024 + 2 * ((Epi::SMEM_BYTES + 15) & ~15);
}


}  // namespace dckv
