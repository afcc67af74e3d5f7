// dckv.cu -- the DCKV codec library for B200 (sm_100a): codec setup, encode, decode,
// byte accounting, behind the C ABI declared in include/dckv.h.
//
// Method: "DCKV: Learned Transform Coding of the Prompt KV Cache in Hybrid Language
// Models" (trove.briskstack.com summary), section "How it works" -- row assembly and
// kept rows (first paragraph), transform / drop rule ("Transform"), rANS under Laplace
// with 64-bit escapes ("Coding"), checkerboard conditional means ("Conditional entropy
// models"), RoPE reapplied after decoding (first paragraph).
//
// Encode:  rows --convert--> fp16 coded rows (+ kept rows into the blob)
//          --GEMM H (tcgen05, GELU epilogue)--> correction hidden units (fp16 hi/lo)
//          --GEMM Y (tcgen05, quantise epilogue)--> int32 codes, bf16 even codes
//          --GEMM odd mean (tcgen05, centre epilogue)--> odd centres
//          --rANS encode (one warp per chunk)--> words --scan--> chunk table, header
//          --compaction--> chunk sections
// Decode:  header check --rANS even--> even codes --GEMM odd mean--> odd centres
//          --rANS odd--> odd codes --GEMM inverse (RoPE + scatter epilogue)--> K, V
//          (+ kept rows with RoPE, + exact fix-up of rows holding codes beyond +-2047)
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/dckv_fit.h"
#include "../../include/dckv_inspect.h"
#include "dckv_epilogues.cuh"
#include "dckv_gemm.cuh"
#include "dckv_internal.cuh"
#include "dckv_rans.cuh"

// Kernels launched by this library in this process (all codecs, all devices).
static std::atomic<long long> g_launches{0};

using namespace dckv;

// ============================================================================ errors
static thread_local char g_err[512] = "";

static int fail(int code, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

#define CK(x)                                                                           \
  do {                                                                                  \
    cudaError_t e_ = (x);                                                               \
    if (e_ != cudaSuccess) return fail(DCKV_ECUDA, "%s: %s", #x, cudaGetErrorString(e_)); \
  } while (0)

#define RET(x)                   \
  do {                           \
    int r_ = (x);                \
    if (r_ != DCKV_OK) return r_; \
  } while (0)

extern "C" const char *dckv_last_error(void) { return g_err; }

// Makes a codec's device current for the duration of an entry point and gives the
// caller's current device back on return.
struct DeviceScope {
  int prev = -1;
  cudaError_t err = cudaSuccess;
  explicit DeviceScope(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
    if (prev != dev) err = cudaSetDevice(dev);
    if (prev == dev) prev = -1;  // nothing to restore
  }
  ~DeviceScope() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};
#define DEVICE_SCOPE(dev)  \
  DeviceScope dev_scope_(dev); \
  CK(dev_scope_.err)

// ============================================================================ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// A operand: [slabs][M][K] (K contiguous), box {64, 128, box_slabs}, 128-byte swizzle.
static int map_a(CUtensorMap *m, const void *ptr, bool bf16, uint64_t K, uint64_t M, uint64_t slabs, int box_slabs) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(DCKV_ECUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[3] = {K, M, slabs};
  cuuint64_t strides[2] = {K * 2, K * M * 2};
  cuuint32_t box[3] = {(cuuint32_t)GEMM_BK, (cuuint32_t)GEMM_BM, (cuuint32_t)box_slabs};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                  const_cast<void *>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DCKV_ECUDA, "tensor map (A) encode failed: %d", (int)r);
  return DCKV_OK;
}

// B operand: [rows][K] (K contiguous), box {64, bn}, 128-byte swizzle, zero fill past the end.
// B operand [rows][K] of 16-bit values, rows ld elements apart (ld = K when 0)
static int map_b(CUtensorMap *m, const void *ptr, bool bf16, uint64_t K, uint64_t rows, int bn, uint64_t ld = 0) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(DCKV_ECUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {K, rows};
  cuuint64_t strides[1] = {(ld ? ld : K) * 2};
  cuuint32_t box[2] = {(cuuint32_t)GEMM_BK, (cuuint32_t)bn};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                  const_cast<void *>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DCKV_ECUDA, "tensor map (B) encode failed: %d", (int)r);
  return DCKV_OK;
}

// ============================================================================ GEMM launch
template <class Epi, int STAGES, int MAX_SLABS>
static int run_gemm(const CUtensorMap &a0, const CUtensorMap &a1, const CUtensorMap &b0, const CUtensorMap &b1,
                    const GemmProblem &prob, const typename Epi::Params &ep, int num_sms, cudaStream_t st) {
  constexpr int smem = gemm_smem_bytes<Epi, STAGES, MAX_SLABS>();
  static_assert(smem <= 232448, "GEMM shared memory above the sm_100 limit");
  auto kern = gemm_kernel<Epi, STAGES, MAX_SLABS>;
  CK(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  const int tiles = prob.m_tiles * prob.n_tiles;
  if (tiles <= 0) return DCKV_OK;
  for (int i = 0; i < prob.n_seg; ++i)
    if (prob.seg[i].n_slab < 1 || prob.seg[i].n_slab > MAX_SLABS) return fail(DCKV_EINVAL, "bad slab count");
  const int grid = std::min(tiles, num_sms);
  { kern<<<grid, GEMM_THREADS, smem, st>>>(a0, a1, b0, b1, prob, ep); ++g_launches; }
  CK(cudaGetLastError());
  return DCKV_OK;
}

// CTA-pair launches: clusters of two, one pair per two SMs at most.
static int launch_pairs(const void *kern, int tiles, int num_sms, int threads, int smem, cudaStream_t st,
                        void **args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * std::min(tiles, num_sms / 2)));
  cfg.blockDim = dim3((unsigned)threads);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  CK(cudaLaunchKernelExC(&cfg, kern, args));
  ++g_launches;
  return DCKV_OK;
}

template <class Epi, int STAGES, int MAX_SLABS, int EPI_WARPS, int BN_MAX = GEMM_MAX_BN>
static int run_gemm2(const CUtensorMap &a0, const CUtensorMap &a1, const CUtensorMap &b0, const CUtensorMap &b1,
                     GemmProblem prob, const typename Epi::Params &ep, int num_sms, bool bf16, cudaStream_t st) {
  constexpr int smem = gemm2_smem_bytes<Epi, STAGES, MAX_SLABS, EPI_WARPS, BN_MAX>();
  static_assert(smem <= 232448, "GEMM shared memory above the sm_100 limit");
  auto kern = gemm2_kernel<Epi, STAGES, MAX_SLABS, EPI_WARPS, BN_MAX>;
  CK(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  if (prob.m_tiles % 2 || prob.bn % 16 || prob.bn > BN_MAX) return fail(DCKV_EINVAL, "bad CTA-pair GEMM shape");
  int tiles = (prob.m_tiles / 2) * prob.n_tiles;
  if (prob.k_split > 1) {  // one segment, every part non-empty
    const int per = prob.n_seg == 1 ? (prob.seg[0].k_steps + prob.k_split - 1) / prob.k_split : 0;
    if (prob.n_seg != 1 || per * (prob.k_split - 1) >= prob.seg[0].k_steps) return fail(DCKV_EINVAL, "bad split-K");
    tiles *= prob.k_split;
  }
  if (tiles <= 0) return DCKV_OK;
  for (int i = 0; i < prob.n_seg; ++i)
    if (prob.seg[i].n_slab < 1 || prob.seg[i].n_slab > MAX_SLABS) return fail(DCKV_EINVAL, "bad slab count");
  prob.idesc = idesc_f16(bf16 ? 1 : 0, 2 * GEMM_BM, prob.bn);
  typename Epi::Params epc = ep;
  void *args[] = {(void *)&a0, (void *)&a1, (void *)&b0, (void *)&b1, (void *)&prob, (void *)&epc};
  return launch_pairs((const void *)kern, tiles, num_sms, 64 + 32 * EPI_WARPS, smem, st, args);
}

template <class Epi, int STAGES, int MAX_SLABS, int CHUNK_STEPS, int BN>
static int run_gemm2_chunked(const CUtensorMap &a0, const CUtensorMap &a1, const CUtensorMap &b0,
                             const CUtensorMap &b1, GemmProblem prob, const typename Epi::Params &ep, int num_sms,
                             bool bf16, cudaStream_t st) {
  constexpr int smem = gemm2_chunked_smem_bytes<Epi, STAGES, MAX_SLABS, BN>();
  static_assert(smem <= 232448, "GEMM shared memory above the sm_100 limit");
  auto kern = gemm2_chunked_kernel<Epi, STAGES, MAX_SLABS, CHUNK_STEPS, BN>;
  CK(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  if (prob.m_tiles % 2 || prob.bn != BN) return fail(DCKV_EINVAL, "bad chunked CTA-pair GEMM shape");
  const int tiles = (prob.m_tiles / 2) * prob.n_tiles;
  if (tiles <= 0) return DCKV_OK;
  for (int i = 0; i < prob.n_seg; ++i)
    if (prob.seg[i].n_slab < 1 || prob.seg[i].n_slab > MAX_SLABS) return fail(DCKV_EINVAL, "bad slab count");
  prob.idesc = idesc_f16(bf16 ? 1 : 0, 2 * GEMM_BM, BN);
  typename Epi::Params epc = ep;
  void *args[] = {(void *)&a0, (void *)&a1, (void *)&b0, (void *)&b1, (void *)&prob, (void *)&epc};
  return launch_pairs((const void *)kern, tiles, num_sms, GEMM2C_THREADS, smem, st, args);
}


// Token-tile width of a CTA-pair GEMM with m_pairs feature tiles of 256: 256 tokens, unless
// 192-token tiles fill the last wave of pairs so much better that it pays for their smaller
// MMA work per staged byte (measured: 25-30% more time per token than 256-token tiles).
// The transform of a single 4,096-token prompt (16 token tiles x 7 feature tiles = 112
// tiles on 74 pairs, against 21 x 7 = 147) takes 192: 193 -> 183 us.
static int pick_pair_bn(int64_t n_rows, int m_pairs, int num_sms) {
  const int64_t pairs = std::max(1, num_sms / 2);
  auto cost = [&](int64_t bn, double per_token) {
    const int64_t tiles = (n_rows + bn - 1) / bn * m_pairs;
    return (double)((tiles + pairs - 1) / pairs) * (double)bn * per_token;
  };
  return cost(192, 1.28) < cost(256, 1.0) ? 192 : 256;
}

static GemmProblem make_problem(int m_tiles, int64_t n_rows, int bn, bool bf16, int32_t *status) {
  GemmProblem p;
  memset(&p, 0, sizeof(p));
  p.m_tiles = m_tiles;
  p.n_rows = (int)n_rows;
  p.bn = bn;
  p.n_tiles = (int)((n_rows + bn - 1) / bn);
  p.idesc = idesc_f16(bf16 ? 1 : 0, GEMM_BM, bn);
  p.status = status;
  return p;
}

static void add_seg(GemmProblem &p, int a_map, int a_slab0, int n_slab, int a_k0, int b_map, int b_row_shift, int b_k0,
                    int k_steps) {
  GemmSeg &s = p.seg[p.n_seg++];
  s.a_map = a_map;
  s.a_slab0 = a_slab0;
  s.n_slab = n_slab;
  s.a_k0 = a_k0;
  s.b_map = b_map;
  s.b_row_shift = b_row_shift;
  s.b_k0 = b_k0;
  s.k_steps = k_steps;
}

// Hidden layer from split-K parts: h = (sum of the parts, in part order) * 2^-p - offset[m],
// g = GELU(h) (erf form), G[row][m] = fp16(g), G[row][256 + m] = fp16(g - fp16(g)).
__global__ void __launch_bounds__(256) k_gelu_parts(const float *part, int n_part, int64_t n_rows, const float *offset,
                                                    float scale, __half *g) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n_rows * N_HIDDEN) return;
  const int m = (int)(e % N_HIDDEN);
  float acc = part[e];
  for (int k = 1; k < n_part; ++k) acc += part[(int64_t)k * n_rows * N_HIDDEN + e];
  const float h = acc * scale - offset[m];
  const float v = 0.5f * h * (1.0f + erff(h * 0.70710678118654752f));
  const __half hi = __float2half_rn(v);
  const __half lo = __float2half_rn(v - __half2float(hi));
  __half *row = g + (e / N_HIDDEN) * (2 * N_HIDDEN);
  row[m] = hi;
  row[N_HIDDEN + m] = lo;
}

// ============================================================================ setup kernels
// Drop mask and scale index per component: beta = b / Delta (steps); kept iff beta >= 0.05;
// s = clamp(round(8 log2(beta / 0.05)), 0, 63)  ("Transform": drop below 0.05 steps).
__global__ void k_scale_keep(const float *b, const float *delta, uint8_t *scale, uint8_t *keep, int32_t *bad) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= N_COEF) return;
  const double d = (double)delta[c];
  const double beta = (double)b[c] / d;
  if (!(d > 0.0) || !isfinite(d) || !isfinite(beta) || beta < 0.0) atomicExch(bad, 1);
  const bool kp = beta >= B0_STEPS;
  int s = 0;
  if (kp) {
    const double v = rint(8.0 * log2(beta / B0_STEPS));
    s = (int)fmin(fmax(v, 0.0), (double)(N_SCALES - 1));
  }
  keep[c] = kp ? 1 : 0;
  scale[c] = (uint8_t)s;
}

// Integer Laplace tables ("Coding"): beta_s = 0.05 * 2^(s/8) steps; p(r) = Laplace(0, beta)
// mass of [r - 1/2, r + 1/2] for r in [-254, 254], ESC = mass beyond +-254.5;
// freq = 1 + floor(p * (2^16 - 510)), the remainder of 2^16 to r = 0; cdf in symbol order.
__global__ void k_tables(uint16_t *cdf_out) {
  __shared__ int64_t fr[N_SYM];
  const int s = blockIdx.x;
  const double beta = B0_STEPS * pow(2.0, (double)s / 8.0);
  for (int k = threadIdx.x; k < N_SYM; k += blockDim.x) {
    double p;
    if (k == ESC_SYM) {
      p = exp(-(R_MAX + 0.5) / beta);
    } else {
      const double ar = fabs((double)(k - R_MAX));
      p = ar == 0.0 ? -expm1(-0.5 / beta) : 0.5 * exp(-(ar - 0.5) / beta) * -expm1(-1.0 / beta);
    }
    fr[k] = 1 + (int64_t)floor(p * (double)(PREC_TOTAL - N_SYM));
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int64_t sum = 0;
    for (int k = 0; k < N_SYM; ++k) sum += fr[k];
    fr[R_MAX] += (int64_t)PREC_TOTAL - sum;
    int64_t c = 0;
    for (int k = 0; k < N_SYM; ++k) {
      cdf_out[s * N_SYM + k] = (uint16_t)c;
      c += fr[k];
    }
  }
}

// out[c] = sum_r v[r] * mat[r][c] in fp64, one thread per column, sequential in r.
__global__ void k_vec_mat(const float *v, const float *mat, int rows, int cols, float *out, double *out64) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= cols) return;
  double acc = 0.0;
  for (int r = 0; r < rows; ++r) acc += (double)v[r] * (double)mat[(int64_t)r * cols + c];
  out[c] = (float)acc;
  out64[c] = acc;
}

// max |mat| (optionally times delta[column]) via integer atomicMax on non-negative floats.
__global__ void k_absmax(const float *mat, int64_t n, int cols, const float *delta, int *out) {
  float m = 0.f;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    float v = fabsf(mat[i]);
    if (delta) v *= fabsf(delta[i % cols]);
    m = fmaxf(m, v);
  }
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(out, __float_as_int(m));
}

// Split operand: out[0][m][k] = fp16(v), out[1][m][k] = fp16(v - fp16(v)), v = in(m, k) * 2^p.
//   mode 0: in(m, k) = src[k * M + m]   (transpose of a row-major [K][M] matrix)
//   mode 1: in(m, k) = src[dim(m) * K + k] * delta[k]   (inverse operand, permuted rows)
__global__ void k_split(const float *src, int M, int K, int mode, const float *delta, double scale, __half *out) {
  __shared__ float tile[32][33];
  const int k0 = blockIdx.x * 32, m0 = blockIdx.y * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
  if (mode == 0) {
    for (int y = ty; y < 32; y += 8) {
      const int k = k0 + y, m = m0 + tx;
      tile[y][tx] = (k < K && m < M) ? src[(int64_t)k * M + m] : 0.f;
    }
    __syncthreads();
    for (int y = ty; y < 32; y += 8) {
      const int m = m0 + y, k = k0 + tx;
      if (m < M && k < K) {
        const double v = (double)tile[tx][y] * (delta ? (double)delta[k] : 1.0) * scale;
        const __half hi = __double2half(v);
        const __half lo = __double2half(v - (double)__half2float(hi));
        out[(int64_t)m * K + k] = hi;
        out[(int64_t)M * K + (int64_t)m * K + k] = lo;
      }
    }
  } else if (mode == 2) {  // src [K][dims]: out[p][k] = src[k][dim(p)] (inverse GEMM row order)
    for (int y = ty; y < 32; y += 8) {
      const int m = m0 + y, k = k0 + tx;
      if (m < M && k < K) {
        const double v = (double)src[(int64_t)k * M + inv_row_to_dim(m)] * scale;
        const __half hi = __double2half(v);
        const __half lo = __double2half(v - (double)__half2float(hi));
        out[(int64_t)m * K + k] = hi;
        out[(int64_t)M * K + (int64_t)m * K + k] = lo;
      }
    }
  } else {
    for (int y = ty; y < 32; y += 8) {
      const int m = m0 + y, k = k0 + tx;
      if (m < M && k < K) {
        const double v = (double)src[(int64_t)inv_row_to_dim(m) * K + k] * (double)delta[k] * scale;
        const __half hi = __double2half(v);
        const __half lo = __double2half(v - (double)__half2float(hi));
        out[(int64_t)m * K + k] = hi;
        out[(int64_t)M * K + (int64_t)m * K + k] = lo;
      }
    }
  }
}

// out[o][k] = src[(k + k_off) * ld + o], o < O, k < K  (bf16 bits)
// Split operands restricted to the kept components (the GEMMs compute and read kept
// components only; compact index m is component kept[m], entries past k_eff are zero).
// Rows: out[s][m][k] = split(src[k][kept[m]] * scale), m < M, src [K][2048] row-major
// (basis, w2), through a shared-memory tile so that both sides are coalesced.
__global__ void k_split_kept_rows(const float *src, int K, const int16_t *kept, int k_eff, int M, double scale,
                                  __half *out) {
  __shared__ float tile[32][33];
  const int k0 = blockIdx.x * 32, m0 = blockIdx.y * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
  for (int y = ty; y < 32; y += 8) {
    const int k = k0 + y, m = m0 + tx;
    tile[y][tx] = (k < K && m < k_eff) ? src[(int64_t)k * N_COEF + kept[m]] : 0.f;
  }
  __syncthreads();
  for (int y = ty; y < 32; y += 8) {
    const int m = m0 + y, k = k0 + tx;
    if (m < M && k < K) {
      const double v = (double)tile[tx][y] * scale;
      const __half hi = __double2half(v);
      out[(int64_t)m * K + k] = hi;
      out[(int64_t)M * K + (int64_t)m * K + k] = __double2half(v - (double)__half2float(hi));
    }
  }
}

// Columns: out[s][r][j] = split(src[row(r)][kept[j]] * delta[kept[j]] * scale) for j < kw,
// src [R][2048] row-major; row(r) = the inverse GEMM's row order (inv = 1) or r itself.
// (a_inv: src = basis, R = 6,144.)
__global__ void k_split_kept_cols(const float *src, int R, bool inv, const int16_t *kept, int k_eff, int kw,
                                  const float *delta, double scale, __half *out) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)R * kw) return;
  const int r = (int)(i / kw), j = (int)(i % kw);
  double v = 0.0;
  if (j < k_eff) {
    const int c = kept[j];
    v = (double)src[(int64_t)(inv ? inv_row_to_dim(r) : r) * N_COEF + c] * (double)delta[c] * scale;
  }
  const __half hi = __double2half(v);
  out[i] = hi;
  out[(int64_t)R * kw + i] = __double2half(v - (double)__half2float(hi));
}

// a_v1[s][h][j] = split(v1[kept[j]][h] * delta[kept[j]] * scale), v1 [2048][256].
__global__ void k_split_v1_kept(const float *v1, const int16_t *kept, int k_eff, int kw, const float *delta,
                                double scale, __half *out) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)N_HIDDEN * kw) return;
  const int h = (int)(i / kw), j = (int)(i % kw);
  double v = 0.0;
  if (j < k_eff) {
    const int c = kept[j];
    v = (double)v1[(int64_t)c * N_HIDDEN + h] * (double)delta[c] * scale;
  }
  const __half hi = __double2half(v);
  out[i] = hi;
  out[(int64_t)N_HIDDEN * kw + i] = __double2half(v - (double)__half2float(hi));
}

// The odd mean model's neighbour blocks, K-major over kept inputs and kept outputs:
// a_on[m][j] = w_odd[2048 + b * 2048 + kept[j - b kw]][kept[m]] for block b = j / kw (left,
// right neighbour), zero past k_eff on either side; bf16 bits, tiled through shared memory.
__global__ void k_gather_on(const uint16_t *w_odd, const int16_t *kept, int k_eff, int kw, int mp, uint16_t *out) {
  __shared__ uint16_t tile[32][33];
  const int j0 = blockIdx.x * 32, m0 = blockIdx.y * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;
  for (int y = ty; y < 32; y += 8) {
    const int j = j0 + y, m = m0 + tx;
    uint16_t v = 0;
    if (j < 2 * kw && m < k_eff) {
      const int b = j / kw, jj = j % kw;
      if (jj < k_eff) v = w_odd[(int64_t)(N_COEF + b * N_COEF + kept[jj]) * N_COEF + kept[m]];
    }
    tile[y][tx] = v;
  }
  __syncthreads();
  for (int y = ty; y < 32; y += 8) {
    const int m = m0 + y, j = j0 + tx;
    if (m < mp && j < 2 * kw) out[(int64_t)m * (2 * kw) + j] = tile[tx][y];
  }
}

// Squared column norms of the inverse GEMM's split operand a_inv [2][6144][kw]: per compact
// component m, sum over rows of lo^2 (out[m]) and of (hi + lo)^2 (out[kw + m]), fp64.
__global__ void k_inv_colnorms(const __half *a_inv, int kw, double *out) {
  __shared__ double s_lo[256], s_all[256];
  const int m = blockIdx.x;
  const __half *lo = a_inv + (int64_t)ROW_DIM * kw;
  double l2 = 0.0, a2 = 0.0;
  for (int p = threadIdx.x; p < ROW_DIM; p += blockDim.x) {
    const double h = (double)__half2float(a_inv[(int64_t)p * kw + m]), l = (double)__half2float(lo[(int64_t)p * kw + m]);
    l2 += l * l;
    a2 += (h + l) * (h + l);
  }
  s_lo[threadIdx.x] = l2;
  s_all[threadIdx.x] = a2;
  __syncthreads();
  for (int s = blockDim.x / 2; s > 0; s >>= 1) {
    if ((int)threadIdx.x < s) {
      s_lo[threadIdx.x] += s_lo[threadIdx.x + s];
      s_all[threadIdx.x] += s_all[threadIdx.x + s];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    out[m] = s_lo[0];
    out[kw + m] = s_all[0];
  }
}

// Even centres from the fp32 even table: out[i] = clamp(round-half-even(t[i]), +-127), the rule
// the odd centres follow in their epilogue.
__global__ void k_round_centres(const float *t, int64_t n, int8_t *out) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = (int8_t)fminf(fmaxf(rintf(t[i]), -(float)ESC_LIMIT), (float)ESC_LIMIT);
}

// Per-component constants of the kept components in compact order (pads: Delta 1, mean 0).
__global__ void k_compact_meta(const float *delta, const float *mub, const int16_t *kept, int k_eff, int mp,
                               float *delta_k, float *mub_k) {
  const int m = blockIdx.x * blockDim.x + threadIdx.x;
  if (m >= mp) return;
  delta_k[m] = m < k_eff ? delta[kept[m]] : 1.f;
  mub_k[m] = m < k_eff ? mub[kept[m]] : 0.f;
}

// out[o][k] = src[k + k_off][col(o)] (16-bit), o < O; col(o) = kept[o] for o < o_valid with
// a kept list (rows o_valid .. O - 1 zero), else o.
__global__ void k_transpose16(const uint16_t *src, int ld, int k_off, int O, int K, uint16_t *out,
                              const int16_t *kept = nullptr, int o_valid = 0) {
  __shared__ uint16_t tile[32][33];
  const int k0 = blockIdx.x * 32, o0 = blockIdx.y * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;
  for (int y = ty; y < 32; y += 8) {
    const int k = k0 + y, o = o0 + tx;
    const int col = kept ? (o < o_valid ? kept[o] : -1) : o;
    tile[y][tx] = (k < K && o < O && col >= 0) ? src[(int64_t)(k + k_off) * ld + col] : 0;
  }
  __syncthreads();
  for (int y = ty; y < 32; y += 8) {
    const int o = o0 + y, k = k0 + tx;
    if (o < O && k < K) out[(int64_t)o * K + k] = tile[tx][y];
  }
}

__global__ void k_permute_mu(const float *mu, float *mu_perm) {
  const int p = blockIdx.x * blockDim.x + threadIdx.x;
  if (p < ROW_DIM) mu_perm[p] = mu[inv_row_to_dim(p)];
}

// ============================================================================ per-call kernels
// Row tables of one prompt per block: coded row r = row_base + i holds position 4 + i.
// Grid (prompts, LAYOUT_SPLIT): the blocks of one prompt share its rows.
constexpr int LAYOUT_SPLIT = 8;

__global__ void k_layout(const PromptInfo *prompts, int32_t *row_tok, int32_t *row_pos, int32_t *row_edst,
                         int32_t *row_slot, int32_t *e_tok, int32_t *e_slot, int32_t *e_row, int32_t *slot_chunk,
                         int chunk_rows, __nv_bfloat16 *qe_zero_pad, int kw) {
  const PromptInfo pi = prompts[blockIdx.x];
  const int t0 = blockIdx.y * blockDim.x + threadIdx.x, ts = gridDim.y * blockDim.x;
  for (int j = t0; j < pi.n_e; j += ts) slot_chunk[pi.slot_e0 + j] = pi.chunk_e0 + j / chunk_rows;
  for (int j = t0; j < pi.n_o; j += ts) slot_chunk[pi.slot_o0 + j] = pi.chunk_o0 + j / chunk_rows;
  for (int i = t0; i < pi.n; i += ts) {
    const int r = pi.row_base + i;
    row_tok[r] = (int32_t)(pi.tok_base + HEAD_KEPT + i);
    row_pos[r] = HEAD_KEPT + i;
    row_edst[r] = (i & 1) ? -1 : pi.ebase + (i >> 1);
    row_slot[r] = (i & 1) ? pi.slot_o0 + (i >> 1) : pi.slot_e0 + (i >> 1);
  }
  for (int e = t0; e <= pi.n_e; e += ts) {
    const bool odd = e < pi.n_o;
    e_tok[pi.ebase + e] = odd ? (int32_t)(pi.tok_base + HEAD_KEPT + 2 * e + 1) : -1;
    e_slot[pi.ebase + e] = odd ? pi.slot_o0 + e : 0;
    e_row[pi.ebase + e] = odd ? pi.row_base + 2 * e + 1 : -1;
  }
  if (qe_zero_pad)  // the row after a prompt's last even row is its odd rows' zero right neighbour
    for (int k = t0; k < kw; k += ts)
      qe_zero_pad[(int64_t)(pi.ebase + pi.n_e) * CODE_LD + k] = __float2bfloat16_rn(0.f);
}

__device__ __forceinline__ int find_prompt(const PromptInfo *p, int batch, int64_t tok) {
  int lo = 0, hi = batch;  // last prompt with tok_base <= tok
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (p[mid].tok_base <= tok) lo = mid; else hi = mid;
  }
  return lo;
}

// One block per token row: coded rows -> fp16 copy (clamped to +-65504, reported as
// DCKV_ERANGE), kept rows -> the blob's kept section verbatim.
__global__ void __launch_bounds__(192) k_convert(const __nv_bfloat16 *rows, const PromptInfo *prompts, int batch,
                                                 __half *x16, uint8_t *blob, uint64_t blob_cap, uint64_t off_kept,
                                                 float *row_norm, int32_t *status) {
  __shared__ float red[6];
  const int64_t t = blockIdx.x;
  const int b = find_prompt(prompts, batch, t);
  const PromptInfo pi = prompts[b];
  const int p = (int)(t - pi.tok_base);
  const uint4 *src = reinterpret_cast<const uint4 *>(rows + t * ROW_DIM);
  const bool coded = pi.n > 0 && p >= HEAD_KEPT && p < pi.N - TAIL_KEPT;
  if (coded) {
    uint4 *dst = reinterpret_cast<uint4 *>(x16 + (int64_t)(pi.row_base + p - HEAD_KEPT) * ROW_DIM);
    bool clamped = false;
    float ss = 0.f;
    constexpr int PER = ROW_DIM / 8 / 192;  // 4 sixteen-byte pieces per thread, loaded together
    uint4 inb[PER];
#pragma unroll
    for (int u = 0; u < PER; ++u) inb[u] = __ldg(src + threadIdx.x + u * 192);
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const int v = threadIdx.x + u * 192;
      const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&inb[u]);
      uint4 o;
      __half2 *oh = reinterpret_cast<__half2 *>(&o);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float2 f = __bfloat1622float2(h[q]);
        ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
        const float lim = 65504.f;
        if (!(fabsf(f.x) <= lim) || !(fabsf(f.y) <= lim)) clamped = true;
        f.x = fminf(fmaxf(f.x, -lim), lim);
        f.y = fminf(fmaxf(f.y, -lim), lim);
        oh[q] = __floats2half2_rn(f.x, f.y);
      }
      dst[v] = o;
    }
    if (clamped) atomicExch(status, DCKV_ERANGE);
    for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x == 0) {
      float t = 0.f;
      for (int w = 0; w < 6; ++w) t += red[w];
      row_norm[pi.row_base + p - HEAD_KEPT] = isfinite(t) ? sqrtf(t) : 3.0e38f;
    }
  } else {
    const int kidx = (pi.n == 0 || p < HEAD_KEPT) ? p : HEAD_KEPT + (p - (pi.N - TAIL_KEPT));
    const uint64_t off = off_kept + (uint64_t)(pi.kept_base + kidx) * (ROW_DIM * 2);
    if (off + ROW_DIM * 2 > blob_cap) return;
    uint4 *dst = reinterpret_cast<uint4 *>(blob + off);
    uint4 inb[ROW_DIM / 8 / 192];
#pragma unroll
    for (int u = 0; u < ROW_DIM / 8 / 192; ++u) inb[u] = __ldg(src + threadIdx.x + u * 192);
#pragma unroll
    for (int u = 0; u < ROW_DIM / 8 / 192; ++u) dst[threadIdx.x + u * 192] = inb[u];
  }
}

// Decode-side check of the blob header and tables against the expected batch shape.
struct HeaderCheck {
  const uint8_t *blob;
  uint64_t blob_bytes;
  const PromptInfo *prompts;
  int batch, chunk_rows, k_eff, n_chunks_e, n_chunks_o;
  int64_t n_kept;
  uint64_t off_kept, off_streams;
  int32_t *valid;
  int32_t *status;
};

__global__ void k_check_header(HeaderCheck h) {
  __shared__ int bad;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  const int n_ch = h.n_chunks_e + h.n_chunks_o;
  const uint64_t tab_end = HEADER_BYTES + 4ull * (h.batch + n_ch + 1);
  if (h.blob_bytes < tab_end || h.blob_bytes < h.off_streams) {
    if (threadIdx.x == 0) bad = 1;
  } else {
    if (threadIdx.x == 0) {
      const uint32_t *h32 = reinterpret_cast<const uint32_t *>(h.blob);
      const uint16_t *h16 = reinterpret_cast<const uint16_t *>(h.blob);
      const uint64_t *h64 = reinterpret_cast<const uint64_t *>(h.blob + 32);
      if (h32[0] != MAGIC || h16[2] != VERSION || h16[3] != (uint16_t)h.chunk_rows || h32[2] != (uint32_t)h.batch ||
          h32[3] != (uint32_t)N_COEF || h32[4] != (uint32_t)h.k_eff || h32[5] != (uint32_t)h.n_chunks_e ||
          h32[6] != (uint32_t)h.n_chunks_o || h32[7] != (uint32_t)h.n_kept || h64[1] != h.off_streams ||
          h64[2] != h.off_kept || h64[0] > h.blob_bytes)
        bad = 1;
      const uint32_t *ct = h32 + HEADER_BYTES / 4 + h.batch;
      if (ct[0] != 0 || h.off_streams + ct[n_ch] != h64[0]) bad = 1;
    }
    __syncthreads();
    const uint32_t *pt = reinterpret_cast<const uint32_t *>(h.blob + HEADER_BYTES);
    for (int b = threadIdx.x; b < h.batch; b += blockDim.x)
      if (pt[b] != (uint32_t)h.prompts[b].N) bad = 1;
    const uint32_t *ct = pt + h.batch;
    for (int c = threadIdx.x; c < n_ch; c += blockDim.x)
      if (ct[c + 1] < ct[c] || ct[c + 1] - ct[c] < (uint32_t)CHUNK_FIXED_BYTES || (ct[c] & 3u)) bad = 1;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    *h.valid = bad ? 0 : 1;
    if (bad) atomicExch(h.status, DCKV_ECORRUPT);
  }
}

// Kept rows: bf16 from the blob, RoPE on keys (same rotation as the inverse epilogue), bf16.
__global__ void __launch_bounds__(256) k_kept(const uint8_t *blob, uint64_t off_kept, const PromptInfo *prompts,
                                              int batch, const float2 *rope, __nv_bfloat16 *k_out,
                                              __nv_bfloat16 *v_out, int64_t n_tokens, const int32_t *valid) {
  if (*valid != 1) return;
  const int64_t kr = blockIdx.x;  // kept row index in the blob
  int lo = 0, hi = batch;         // last prompt with kept_base <= kr
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prompts[mid].kept_base <= kr) lo = mid; else hi = mid;
  }
  const PromptInfo pi = prompts[lo];
  const int kidx = (int)(kr - pi.kept_base);
  const int pos = (pi.n == 0 || kidx < HEAD_KEPT) ? kidx : pi.N - TAIL_KEPT + (kidx - HEAD_KEPT);
  const int64_t tok = pi.tok_base + pos;
  const __nv_bfloat16 *row = reinterpret_cast<const __nv_bfloat16 *>(blob + off_kept + (uint64_t)kr * ROW_DIM * 2);
  // 24 head vectors x 128 pairs
  for (int idx = threadIdx.x; idx < 24 * 128; idx += blockDim.x) {
    const int hv = idx >> 7, i = idx & 127;
    const int layer = hv >> 2, kv = (hv >> 1) & 1, head = hv & 1;
    float a = __bfloat162float(row[hv * HEAD_DIM + i]);
    float b = __bfloat162float(row[hv * HEAD_DIM + 128 + i]);
    if (kv == 0) {
      const float2 cs = __ldg(rope + (int64_t)pos * 128 + i);
      const float a2 = a * cs.x - b * cs.y, b2 = b * cs.x + a * cs.y;
      a = a2;
      b = b2;
    }
    __nv_bfloat16 *dst = (kv == 0 ? k_out : v_out) + ((layer * n_tokens + tok) * 2 + head) * HEAD_DIM;
    dst[i] = __float2bfloat16_rn(a);
    dst[128 + i] = __float2bfloat16_rn(b);
  }
}

// RoPE table of a decode call: rope[pos][i] = (cos, sin) of pos * theta_i, the same values
// rope_cs gives the fix-up kernel.
__global__ void __launch_bounds__(128) k_rope_table(float2 *rope, int64_t n_pos, const double *theta,
                                                   const int32_t *valid) {
  if (*valid != 1) return;
  for (int64_t pos = blockIdx.x; pos < n_pos; pos += gridDim.x) {
    float cs, sn;
    rope_cs((int)pos, threadIdx.x, theta, cs, sn);
    rope[pos * 128 + threadIdx.x] = make_float2(cs, sn);
  }
}

__host__ __device__ __forceinline__ int dim_to_inv_row(int d) {
  const int hv = d / HEAD_DIM, dd = d % HEAD_DIM;
  const int half = dd < 128 ? dd / 64 : (dd - 128) / 64;
  const int r = dd < 128 ? dd % 64 : 64 + (dd - 128) % 64;
  return (2 * hv + half) * GEMM_BM + r;
}

// Rows holding a code with |q| >= 2048 (not exact in the fp16 operand) are recomputed
// here in fp32 from the exact codes, after the inverse GEMM wrote them.
__global__ void __launch_bounds__(256) k_fixup(const int32_t *biglist, const uint32_t *bigcount, const __half *q16,
                                               const int32_t *qbig, const __half *a_inv, float inv_scale,
                                               const float *mu_perm, const double *theta, const int32_t *row_tok,
                                               const int32_t *row_pos, __nv_bfloat16 *k_out, __nv_bfloat16 *v_out,
                                               int64_t n_tokens, const float *v1t32, const float *v2_32,
                                               const float *delta, const int16_t *kept_list, int k_eff, int kw) {
  __shared__ float qs[N_COEF];
  __shared__ float xs[ROW_DIM];
  __shared__ float gs[N_HIDDEN];
  const uint32_t n = *bigcount;
  for (uint32_t li = blockIdx.x; li < n; li += gridDim.x) {
    const int64_t r = biglist[li];
    for (int m = threadIdx.x; m < kw; m += blockDim.x) {  // codes of the kept components, compact order
      float v = __half2float(q16[r * CODE_LD + m]);
      if (fabsf(v) >= (float)BIG_CODE) v = (float)qbig[r * CODE_LD + m];
      qs[m] = v;
    }
    __syncthreads();
    const __half *lo = a_inv + (int64_t)ROW_DIM * kw;
    for (int d = threadIdx.x; d < ROW_DIM; d += blockDim.x) {
      const int64_t p = dim_to_inv_row(d);
      float acc = 0.f;
      for (int m = 0; m < k_eff; ++m)
        acc = fmaf(qs[m], __half2float(a_inv[p * kw + m]) + __half2float(lo[p * kw + m]), acc);
      xs[d] = acc * inv_scale + mu_perm[p];
    }
    if (v1t32) {  // decoder-side synthesis: + GELU((q Delta) V1) V2, fp32
      for (int h = threadIdx.x; h < N_HIDDEN; h += blockDim.x) {
        const float *w = v1t32 + (int64_t)h * N_COEF;
        float acc = 0.f;
        for (int m = 0; m < k_eff; ++m) {
          const int c = kept_list[m];
          acc = fmaf(qs[m] * delta[c], w[c], acc);
        }
        gs[h] = 0.5f * acc * (1.0f + erff(acc * 0.70710678118654752f));
      }
      __syncthreads();
      for (int d = threadIdx.x; d < ROW_DIM; d += blockDim.x) {
        float acc = 0.f;
        for (int h = 0; h < N_HIDDEN; ++h) acc = fmaf(gs[h], v2_32[(int64_t)h * ROW_DIM + d], acc);
        xs[d] += acc;
      }
    }
    __syncthreads();
    const int pos = row_pos[r];
    const int64_t tok = row_tok[r];
    for (int idx = threadIdx.x; idx < 24 * 128; idx += blockDim.x) {
      const int hv = idx >> 7, i = idx & 127;
      const int layer = hv >> 2, kv = (hv >> 1) & 1, head = hv & 1;
      float a = xs[hv * HEAD_DIM + i], b = xs[hv * HEAD_DIM + 128 + i];
      if (kv == 0) {
        float cs, sn;
        rope_cs(pos, i, theta, cs, sn);
        const float a2 = a * cs - b * sn, b2 = b * cs + a * sn;
        a = a2;
        b = b2;
      }
      __nv_bfloat16 *dst = (kv == 0 ? k_out : v_out) + ((layer * n_tokens + tok) * 2 + head) * HEAD_DIM;
      dst[i] = __float2bfloat16_rn(a);
      dst[128 + i] = __float2bfloat16_rn(b);
    }
    __syncthreads();
  }
}

// out[o][k] = src[k * O + o] (fp32 transpose of a row-major [K][O] matrix)
__global__ void k_transpose32(const float *src, int K, int O, float *out) {
  __shared__ float tile[32][33];
  const int k0 = blockIdx.x * 32, o0 = blockIdx.y * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;
  for (int y = ty; y < 32; y += 8) {
    const int k = k0 + y, o = o0 + tx;
    tile[y][tx] = (k < K && o < O) ? src[(int64_t)k * O + o] : 0.f;
  }
  __syncthreads();
  for (int y = ty; y < 32; y += 8) {
    const int o = o0 + y, k = k0 + tx;
    if (o < O && k < K) out[(int64_t)o * K + k] = tile[tx][y];
  }
}

__device__ __forceinline__ double warp_sum(double v) {
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// code of compact component m of a row
__device__ __forceinline__ void store_code(int64_t row, int m, double ratio, int32_t *q32, __nv_bfloat16 *qe,
                                           const int32_t *row_edst) {
  const double qd = fmin(fmax(rint(ratio), -2147483648.0), 2147483647.0);
  const int q = (int)qd;
  q32[row * CODE_LD + m] = q;
  const int e = row_edst[row];
  if (e >= 0) qe[(int64_t)e * CODE_LD + m] = __float2bfloat16_rn((float)q);
}

// bf16 bits to fp64, exactly: the sign, exponent and mantissa fields move into place
// (normal numbers; zero, subnormal and non-finite values take the conversion instruction)
__device__ __forceinline__ double bf16_bits_to_f64(uint32_t w) {
  const uint32_t t = w & 0x7FFFu;
  const uint32_t e = t >> 7;
  if (e == 0u || e == 0xFFu) return (double)__uint_as_float(w << 16);
  return __hiloint2double((int)(((w & 0x8000u) << 16) | ((t + 0x1C000u) << 13)), 0);
}

// x . b over a 6,144-dim row in fp64 by one warp: lane l takes the 8-element groups
// v = l, l + 32, ... of the bf16 row (16-byte loads, twelve in flight per lane), eight
// independent partial sums added in a fixed order (the caller reduces across lanes).
// b sits in shared memory as fp64, element 8 v + j at b[j * 768 + v], so that the lanes of
// a warp read consecutive words (no bank conflicts).  Products of a bf16 and an fp32 value
// are exact in fp64.
// x . w over a 6,144-dim row in fp64 by one warp, x (fp64) in shared memory and w fp32 in
// global memory, lanes strided.
__device__ __forceinline__ double smem_dot_lane(const double *xs, const float *w, int lane) {
  double part[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll 4
  for (int i = lane; i < ROW_DIM; i += 128) {
    part[0] = fma(xs[i], (double)__ldg(w + i), part[0]);
    part[1] = fma(xs[i + 32], (double)__ldg(w + i + 32), part[1]);
    part[2] = fma(xs[i + 64], (double)__ldg(w + i + 64), part[2]);
    part[3] = fma(xs[i + 96], (double)__ldg(w + i + 96), part[3]);
  }
  return (part[0] + part[1]) + (part[2] + part[3]);
}

// x . b over a 6,144-dim row in fp64 by one warp, x the caller's bf16 row and b an fp32
// column, both read from global memory: lane l takes the 16-byte groups l, l + 32, ... of x
// (8 elements) and the two float4 of b under each; the products are exact in fp64 and go
// into eight partial sums (one per element of a group), added in a fixed order.
__device__ __forceinline__ double row_dot_glb(const uint4 *xr, const float4 *b, int lane) {
  constexpr int R = ROW_DIM / 8 / 32;  // 24 groups per lane
  constexpr int Q = 6;                 // groups loaded together
  double part[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) part[u] = 0.0;
#pragma unroll
  for (int q0 = 0; q0 < R; q0 += Q) {
    uint4 xv[Q];
    float4 b0[Q], b1[Q];
#pragma unroll
    for (int r = 0; r < Q; ++r) {
      const int g = (q0 + r) * 32 + lane;
      xv[r] = __ldg(xr + g);
      b0[r] = __ldg(b + 2 * g);
      b1[r] = __ldg(b + 2 * g + 1);
    }
#pragma unroll
    for (int r = 0; r < Q; ++r) {
      part[0] = fma(bf16_bits_to_f64(xv[r].x & 0xFFFFu), (double)b0[r].x, part[0]);
      part[1] = fma(bf16_bits_to_f64(xv[r].x >> 16), (double)b0[r].y, part[1]);
      part[2] = fma(bf16_bits_to_f64(xv[r].y & 0xFFFFu), (double)b0[r].z, part[2]);
      part[3] = fma(bf16_bits_to_f64(xv[r].y >> 16), (double)b0[r].w, part[3]);
      part[4] = fma(bf16_bits_to_f64(xv[r].z & 0xFFFFu), (double)b1[r].x, part[4]);
      part[5] = fma(bf16_bits_to_f64(xv[r].z >> 16), (double)b1[r].y, part[5]);
      part[6] = fma(bf16_bits_to_f64(xv[r].w & 0xFFFFu), (double)b1[r].z, part[6]);
      part[7] = fma(bf16_bits_to_f64(xv[r].w >> 16), (double)b1[r].w, part[7]);
    }
  }
  return ((part[0] + part[1]) + (part[2] + part[3])) + ((part[4] + part[5]) + (part[6] + part[7]));
}

// Exact recomputation of codes near a half-step boundary.  The transform's epilogue bins
// them by component; codes are numbered by a prefix sum over the bins (each block computes
// it for itself) and every warp takes one code at a time:
// y = x . basis[:, c] - (mu basis)[c] + g . w2[:, c] in fp64 (x the caller's bf16 row, the
// basis column fp32, the mean term fp64-accumulated at codec creation, g the correction's
// hidden units as their fp16 hi/lo pair), q = round(y / Delta_c).  Consecutive codes share
// their component, so the warps of a block read the same basis column, mostly from L1.
// Lane partial sums are added by a butterfly in a fixed order, so the result is
// deterministic.
constexpr int REFINE_THREADS = 512;
constexpr int REFINE_SMEM = ROW_DIM * 8 + (N_COEF + 1) * 4;  // the whole-row kernels' shared memory

__global__ void __launch_bounds__(REFINE_THREADS) k_refine_codes(
    const uint32_t *el_bins, const uint32_t *bin_count, uint32_t bin_cap, const __nv_bfloat16 *rows,
    const int32_t *row_tok, const double *mub64, const float *bt32, const float *w2t32, const __half *g16,
    const float *delta, const uint32_t *rowflag, const int16_t *kept_list, int32_t *q32, __nv_bfloat16 *qe,
    const int32_t *row_edst) {
  __shared__ uint32_t code0[N_COEF + 1];  // first code of each bin
  __shared__ uint32_t warp_tot[REFINE_THREADS / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // codes per bin, exclusive prefix sum: thread t owns bins PER t .. PER t + PER - 1
  {
    constexpr int PER = N_COEF / REFINE_THREADS;
    uint32_t cnt[PER], run = 0;
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      cnt[u] = min(bin_count[threadIdx.x * PER + u], bin_cap);
      run += cnt[u];
    }
    uint32_t incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    uint32_t base = incl - run;
    for (int w = 0; w < warp; ++w) base += warp_tot[w];
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      code0[threadIdx.x * PER + u] = base;
      base += cnt[u];
    }
    if (threadIdx.x == REFINE_THREADS - 1) code0[N_COEF] = base;
    __syncthreads();
  }
  const uint32_t n_codes = code0[N_COEF];
  const uint32_t n_warps = gridDim.x * (REFINE_THREADS / 32);
  for (uint32_t t = blockIdx.x * (REFINE_THREADS / 32) + warp; t < n_codes; t += n_warps) {
    int lo = 0, hi = N_COEF;  // the bin holding this code: code0[lo] <= t < code0[lo + 1]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (code0[mid] <= t) lo = mid; else hi = mid;
    }
    const int m = lo;  // compact component index of the bin
    const int64_t row = el_bins[(int64_t)m * bin_cap + (t - code0[m])];
    if (rowflag[row]) continue;  // rows listed for whole-row recomputation are left to k_refine_rows
    const int c = kept_list[m];
    double acc = row_dot_glb(reinterpret_cast<const uint4 *>(rows + (int64_t)row_tok[row] * ROW_DIM),
                             reinterpret_cast<const float4 *>(bt32 + (int64_t)c * ROW_DIM), lane);
    if (w2t32) {  // the correction (absent in a linear codec): eight hidden units per lane
      const __half *g = g16 + row * (2 * N_HIDDEN);
      const float *w = w2t32 + (int64_t)c * N_HIDDEN;
      double h = 0.0;
#pragma unroll
      for (int u = 0; u < N_HIDDEN / 32; ++u) {
        const int j = u * 32 + lane;
        h += ((double)__half2float(g[j]) + (double)__half2float(g[N_HIDDEN + j])) * (double)w[j];
      }
      acc += h;
    }
    acc = warp_sum(acc) - mub64[c];
    if (lane == 0) store_code(row, m, acc / (double)delta[c], q32, qe, row_edst);
  }
}

// Whole-row exact recomputation (rows with a large norm), in two launches whose work items
// spread over the grid.  Each block first puts the listed row x (fp64) into shared memory.
// k_refine_hidden: an item is (row, 8 hidden units), one unit per warp:
// h = x . w1[:, u] - (mu w1)[u], g = GELU(h) (erf), fp64, into g64[list index][256].
// k_refine_rows: an item is (row, 8 kept components), one component per warp:
// y = x . basis[:, c] - (mu basis)[c] + g . w2[:, c], then the code (dropped components stay 0).
constexpr int REFINE_GROUP = 8;

__device__ __forceinline__ void load_row_f64(double *xs, const __nv_bfloat16 *xr) {
  const uint16_t *xb = reinterpret_cast<const uint16_t *>(xr);
  for (int i = threadIdx.x; i < ROW_DIM; i += blockDim.x) xs[i] = bf16_bits_to_f64(xb[i]);
}

__global__ void __launch_bounds__(256) k_refine_hidden(const uint32_t *full_list, const uint32_t *counters,
                                                       const __nv_bfloat16 *rows, const int32_t *row_tok,
                                                       const double *muw1_64, const float *w1t32, double *g64) {
  extern __shared__ __align__(16) double xs[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr uint32_t PER_ROW = N_HIDDEN / REFINE_GROUP;
  const uint32_t n_items = counters[1] * PER_ROW;
  for (uint32_t item = blockIdx.x; item < n_items; item += gridDim.x) {
    const uint32_t li = item / PER_ROW;
    const int h = (int)(item % PER_ROW) * REFINE_GROUP + warp;
    load_row_f64(xs, rows + (int64_t)row_tok[full_list[li]] * ROW_DIM);
    __syncthreads();
    const double a = warp_sum(smem_dot_lane(xs, w1t32 + (int64_t)h * ROW_DIM, lane)) - muw1_64[h];
    if (lane == 0) g64[(int64_t)li * N_HIDDEN + h] = 0.5 * a * (1.0 + erf(a * 0.70710678118654752440));
    __syncthreads();
  }
}

__global__ void __launch_bounds__(256) k_refine_rows(const uint32_t *full_list, const uint32_t *counters,
                                                     const __nv_bfloat16 *rows, const int32_t *row_tok,
                                                     const double *mub64, const float *bt32, const float *w2t32,
                                                     const double *g64, const float *delta, const int16_t *kept_list,
                                                     int k_eff, int32_t *q32, __nv_bfloat16 *qe,
                                                     const int32_t *row_edst) {
  extern __shared__ __align__(16) double xs[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t per_row = (uint32_t)(k_eff + REFINE_GROUP - 1) / REFINE_GROUP;
  const uint32_t n_items = counters[1] * per_row;
  for (uint32_t item = blockIdx.x; item < n_items; item += gridDim.x) {
    const uint32_t li = item / per_row;
    const int64_t row = full_list[li];
    const int m = (int)(item % per_row) * REFINE_GROUP + warp;
    load_row_f64(xs, rows + (int64_t)row_tok[row] * ROW_DIM);
    __syncthreads();
    if (m < k_eff) {  // warp-uniform
      const int c = kept_list[m];
      double acc = smem_dot_lane(xs, bt32 + (int64_t)c * ROW_DIM, lane);
      if (w2t32) {
        const double *g = g64 + (int64_t)li * N_HIDDEN;
        for (int h = lane; h < N_HIDDEN; h += 32) acc = fma(g[h], (double)w2t32[c * N_HIDDEN + h], acc);
      }
      acc = warp_sum(acc) - mub64[c];
      if (lane == 0) store_code(row, m, acc / (double)delta[c], q32, qe, row_edst);
    }
    __syncthreads();
  }
}

// ============================================================================ host layout
static inline uint64_t align_up(uint64_t v, uint64_t a) { return (v + a - 1) / a * a; }

static int build_layout(const dckv_codec *c, const int64_t *offs, int batch, Layout &L) {
  if (!offs) return fail(DCKV_EINVAL, "seq_offsets is NULL");
  if (batch < 1 || batch > DCKV_MAX_PROMPTS) return fail(DCKV_EINVAL, "batch %d out of range", batch);
  if (offs[0] != 0) return fail(DCKV_EINVAL, "seq_offsets[0] must be 0");
  L = Layout();
  L.batch = batch;
  const int G = c->chunk_rows;
  int64_t rows = 0, ne = 0, kept = 0;
  int ce = 0, co = 0;
  L.prompts.resize(batch);
  for (int b = 0; b < batch; ++b) {
    const int64_t N = offs[b + 1] - offs[b];
    if (N < 0 || N > (int64_t)1 << 30) return fail(DCKV_EINVAL, "prompt %d has a bad length", b);
    PromptInfo &p = L.prompts[b];
    p.tok_base = offs[b];
    p.N = (int32_t)N;
    p.n = (int32_t)std::max<int64_t>(0, N - HEAD_KEPT - TAIL_KEPT);
    p.n_e = (p.n + 1) / 2;
    p.n_o = p.n / 2;
    p.row_base = (int32_t)rows;
    p.ebase = (int32_t)ne;
    p.kept_base = (int32_t)kept;
    p.n_kept = (int32_t)(N - p.n);
    p.chunk_e0 = ce;
    L.max_len = std::max<int64_t>(L.max_len, N);
    ce += (p.n_e + G - 1) / G;
    rows += p.n;
    ne += p.n_e + 1;
    kept += p.n_kept;
  }
  int64_t se = 0, so = 0;
  for (int b = 0; b < batch; ++b) {
    L.prompts[b].chunk_o0 = ce + co;
    co += (L.prompts[b].n_o + G - 1) / G;
    L.prompts[b].slot_e0 = (int32_t)se;
    se += L.prompts[b].n_e;
  }
  for (int b = 0; b < batch; ++b) {
    L.prompts[b].slot_o0 = (int32_t)(se + so);
    so += L.prompts[b].n_o;
  }
  L.n_tokens = offs[batch];
  if (L.n_tokens >= ((int64_t)1 << 31)) return fail(DCKV_EINVAL, "too many tokens");
  if (rows > DCKV_MAX_ROWS) return fail(DCKV_EINVAL, "too many coded rows (%lld)", (long long)rows);
  L.n_rows = rows;
  L.ne_pad = ne;
  L.n_kept = kept;
  L.n_chunks_e = ce;
  L.n_chunks_o = co;
  L.n_chunks = ce + co;
  L.chunks.resize(L.n_chunks);
  int64_t slot = 0;
  int ci = 0;
  for (int par = 0; par < 2; ++par)
    for (int b = 0; b < batch; ++b) {
      const PromptInfo &p = L.prompts[b];
      const int nr = par ? p.n_o : p.n_e;
      for (int j0 = 0; j0 < nr; j0 += G) {
        ChunkDesc &d = L.chunks[ci++];
        d.prompt = b;
        d.parity = par;
        d.j0 = j0;
        d.nrows = std::min(G, nr - j0);
        d.sym_base = slot * c->k_eff;
        slot += d.nrows;
      }
    }
  L.n_symbols = rows * (int64_t)c->k_eff;
  L.kw = c->kw;
  L.off_kept = align_up(HEADER_BYTES + 4ull * (batch + L.n_chunks + 1), 16);
  L.off_streams = L.off_kept + (uint64_t)kept * ROW_DIM * 2;
  return DCKV_OK;
}

static WsPlan plan_ws(const Layout &L, int which /*0 encode, 1 decode*/) {
  WsPlan w;
  memset(&w, 0, sizeof(w));
  uint64_t o = 0;
  auto take = [&](uint64_t bytes) {
    const uint64_t at = o;
    o = align_up(o + std::max<uint64_t>(bytes, 1), 256);
    return (size_t)at;
  };
  w.prompts = take(sizeof(PromptInfo) * L.batch);
  w.chunks = take(sizeof(ChunkDesc) * std::max(L.n_chunks, 1));
  w.row_tok = take(4ull * L.n_rows);
  w.row_pos = take(4ull * L.n_rows);
  w.row_edst = take(4ull * L.n_rows);
  w.e_tok = take(4ull * L.ne_pad);
  w.row_slot = take(4ull * L.n_rows);
  w.e_slot = take(4ull * L.ne_pad);
  w.e_row = take(4ull * L.ne_pad);
  w.escflag = take(4ull * std::max(L.n_chunks, 1));
  w.slot_chunk = take(4ull * L.n_rows);
  w.qe = take(2ull * L.ne_pad * CODE_LD);
  w.cen8 = take(1ull * L.n_symbols);
  w.counters = take(256);
  if (which == 0) {
    w.x16 = take(2ull * L.n_rows * ROW_DIM);
    w.g16 = take(2ull * L.n_rows * 2 * N_HIDDEN);
    w.hpart = take(4ull * HIDDEN_SPLIT * L.n_rows * N_HIDDEN);
    w.q32 = take(4ull * L.n_rows * CODE_LD);
    w.sym16 = take(2ull * L.n_symbols);
    w.cf32 = take(8ull * L.n_symbols);
    w.words = take(2ull * L.n_symbols);
    w.states = take(128ull * L.n_chunks);
    w.nwords = take(4ull * L.n_chunks);
    w.nesc = take(4ull * L.n_chunks);
    w.offs = take(4ull * (L.n_chunks + 1));
    w.row_norm = take(4ull * L.n_rows);
    w.rowflag = take(4ull * L.n_rows);
    // codes to recompute exactly, binned by component; a code that finds its bin full
    // sends its whole row to the whole-row recomputation instead
    w.bin_cap = (uint32_t)std::min<int64_t>(L.n_rows / 32 + 64, (int64_t)1 << 30);
    w.el_bins = take(4ull * N_COEF * w.bin_cap);
    w.bin_count = take(4ull * N_COEF);
    w.full_list = take(4ull * L.n_rows);
    w.g64 = take(8ull * N_HIDDEN * L.n_rows);  // hidden units of rows recomputed whole, by list index
  } else {
    w.slots16 = take(2ull * L.n_symbols);
    w.g16 = take(2ull * L.n_rows * 2 * N_HIDDEN);  // synthesis hidden units (hi/lo)
    w.rope = take(8ull * 128 * std::max<int64_t>(L.max_len, 1));
    w.q16 = take(2ull * L.n_rows * CODE_LD);
    w.qbig = take(4ull * L.n_rows * CODE_LD);
    w.bigflag = take(4ull * L.n_rows);
    w.biglist = take(4ull * L.n_rows);
  }
  w.total = o;
  return w;
}

// Stage timing (diagnostics): each host thread keeps the events of its own last call on a
// codec with timing enabled, so concurrent calls from several threads never share them.
struct StageLog {
  const dckv_codec *codec = nullptr;
  int device = -1;
  int n = 0;
  const char *names[32];
  cudaEvent_t ev[32] = {};
};
static thread_local StageLog t_stages;

static void stage_begin(const dckv_codec *c) {
  if (!c->timing) return;
  StageLog &g = t_stages;
  if (g.device != c->device) {  // events belong to a device: (re)create them on this one
    for (auto &e : g.ev)
      if (e) cudaEventDestroy(e), e = nullptr;
    for (auto &e : g.ev)
      if (cudaEventCreate(&e) != cudaSuccess) e = nullptr;
    g.device = c->device;
  }
  g.codec = c;
  g.n = 0;
}

static void stage_mark(const dckv_codec *c, cudaStream_t st, const char *name) {
  StageLog &g = t_stages;
  if (!c->timing || g.codec != c || g.n >= 32 || !g.ev[g.n]) return;
  g.names[g.n] = name;
  cudaEventRecord(g.ev[g.n++], st);
}

// ============================================================================ codec create
extern "C" int dckv_codec_create(const dckv_params *prm, int device, int chunk_rows, dckv_codec **out) {
  if (!out) return fail(DCKV_EINVAL, "out is NULL");
  *out = nullptr;
  if (!prm || !prm->mu || !prm->basis || !prm->delta || !prm->laplace_b)
    return fail(DCKV_EINVAL, "a parameter pointer is NULL");
  if (!prm->w1 != !prm->w2) return fail(DCKV_EINVAL, "w1 and w2 must both be given or both be NULL");
  if (!prm->embed != !prm->w_even || !prm->embed != !prm->w_odd)
    return fail(DCKV_EINVAL, "embed, w_even and w_odd must all be given or all be NULL");
  if (!prm->v1 != !prm->v2) return fail(DCKV_EINVAL, "v1 and v2 must both be given or both be NULL");
  const bool has_mlp = prm->w1 != nullptr, has_means = prm->embed != nullptr, has_synth = prm->v1 != nullptr;
  if (has_means && (prm->vocab < 1 || prm->vocab > (1 << 20))) return fail(DCKV_EINVAL, "vocab out of range");
  if (chunk_rows < -1 || chunk_rows > 256) return fail(DCKV_EINVAL, "chunk_rows out of range");
  if (((uintptr_t)prm->embed | (uintptr_t)prm->w_even | (uintptr_t)prm->w_odd) & 15)
    return fail(DCKV_EINVAL, "bf16 parameters must be 16-byte aligned");
  static_assert(RANS_DEC_SMEM <= 232448, "decoder tables exceed shared memory");
  DEVICE_SCOPE(device);
  cudaDeviceProp prop;
  CK(cudaGetDeviceProperties(&prop, device));
  if (prop.major != 10) return fail(DCKV_EINVAL, "needs an sm_100 device (found sm_%d%d)", prop.major, prop.minor);
  if (!encode_fn()) return fail(DCKV_ECUDA, "cuTensorMapEncodeTiled unavailable");

  dckv_codec *c = new dckv_codec();
  c->device = device;
  c->num_sms = prop.multiProcessorCount;
  c->chunk_rows = chunk_rows;
  c->vocab = has_means ? prm->vocab : 0;
  c->has_mlp = has_mlp;
  c->has_means = has_means;
  c->has_synth = has_synth;
  c->p = *prm;

  auto cleanup = [&](int code) {
    dckv_codec_destroy(c);
    return code;
  };

  // one device block for every derived tensor
  const uint64_t V = has_means ? (uint64_t)prm->vocab : 0;
  uint64_t o = 0;
  auto take = [&](uint64_t bytes) {
    const uint64_t at = o;
    o = align_up(o + bytes, 1024);
    return at;
  };
  const uint64_t o_ay = take(2ull * 2 * N_COEF * ROW_DIM);
  const uint64_t o_aw2 = take(2ull * 2 * N_COEF * N_HIDDEN);
  const uint64_t o_ah = take(2ull * 2 * N_HIDDEN * ROW_DIM);
  const uint64_t o_ainv = take(2ull * 2 * ROW_DIM * N_COEF);
  const uint64_t o_aon = take(2ull * N_COEF * 2 * N_COEF);
  const uint64_t o_mub = take(4ull * N_COEF);
  const uint64_t o_mubk = take(4ull * N_COEF);
  const uint64_t o_deltak = take(4ull * N_COEF);
  const uint64_t o_muw1 = take(4ull * N_HIDDEN);
  const uint64_t o_mup = take(4ull * ROW_DIM);
  const uint64_t o_delta = take(4ull * N_COEF);
  const uint64_t o_lapb = take(4ull * N_COEF);
  const uint64_t o_keep = take(N_COEF);
  const uint64_t o_scale = take(N_COEF);
  const uint64_t o_kl = take(2ull * N_COEF);
  const uint64_t o_ks = take(N_COEF);
  const uint64_t o_cdf = take(2ull * N_SCALES * N_SYM);
  const uint64_t o_lut = take(2ull * N_SCALES * LUT_STRIDE);
  const uint64_t o_tail = take(4ull * N_SCALES);
  const uint64_t o_dcdf = take(2ull * N_SCALES * DEC_CDF_STRIDE);
  const uint64_t o_cfm = take(8ull * N_SCALES * N_SYM);
  const uint64_t o_kidx = take(2ull * N_COEF);
  const uint64_t o_theta = take(8ull * 128);
  const uint64_t o_bt32 = take(4ull * N_COEF * ROW_DIM);
  const uint64_t o_w1t32 = take(4ull * N_HIDDEN * ROW_DIM);
  const uint64_t o_w2t32 = take(4ull * N_COEF * N_HIDDEN);
  const uint64_t o_mub64 = take(8ull * N_COEF);
  const uint64_t o_muw164 = take(8ull * N_HIDDEN);
  const uint64_t o_av1 = take(has_synth ? 2ull * 2 * N_HIDDEN * N_COEF : 0);
  const uint64_t o_av2 = take(has_synth ? 2ull * 2 * ROW_DIM * N_HIDDEN : 0);
  const uint64_t o_v1t32 = take(has_synth ? 4ull * N_HIDDEN * N_COEF : 0);
  const uint64_t o_v2_32 = take(has_synth ? 4ull * N_HIDDEN * ROW_DIM : 0);
  const uint64_t o_zero = take(4ull * N_HIDDEN);
  const uint64_t o_scr = take(64);
  if (cudaMalloc(&c->blk, o) != cudaSuccess) return cleanup(fail(DCKV_ECUDA, "cudaMalloc(%llu) failed", (unsigned long long)o));
  uint8_t *B = (uint8_t *)c->blk;
  // setup-only scratch, freed when creation ends: the gathered, K-major W_e^T and W_oE^T,
  // and the inverse operand's column norms
  struct SetupScratch {
    void *p = nullptr;
    ~SetupScratch() {
      if (p) cudaFree(p);
    }
  } setup;
  const uint64_t s_norms = 2ull * 2 * N_COEF * N_COEF;
  if (cudaMalloc(&setup.p, s_norms + 8ull * 2 * N_COEF) != cudaSuccess)
    return cleanup(fail(DCKV_ECUDA, "cudaMalloc of the setup scratch failed"));
  c->a_y = (__half *)(B + o_ay);
  c->a_w2 = (__half *)(B + o_aw2);
  c->a_h = (__half *)(B + o_ah);
  c->a_inv = (__half *)(B + o_ainv);
  c->a_on = (__nv_bfloat16 *)(B + o_aon);
  c->mub = (float *)(B + o_mub);
  c->mub_k = (float *)(B + o_mubk);
  c->delta_k = (float *)(B + o_deltak);
  c->muw1 = (float *)(B + o_muw1);
  c->mu_perm = (float *)(B + o_mup);
  c->delta = (float *)(B + o_delta);
  c->lapb = (float *)(B + o_lapb);
  c->keep = B + o_keep;
  c->scale = B + o_scale;
  c->kept_list = (int16_t *)(B + o_kl);
  c->kept_scale = B + o_ks;
  c->cdf = (uint16_t *)(B + o_cdf);
  c->lut = (uint16_t *)(B + o_lut);
  c->tail = (uint32_t *)(B + o_tail);
  c->dcdf = (uint16_t *)(B + o_dcdf);
  c->cfm_tab = (uint2 *)(B + o_cfm);
  c->kidx = (int16_t *)(B + o_kidx);
  c->theta = (double *)(B + o_theta);
  c->bt32 = (float *)(B + o_bt32);
  c->w1t32 = (float *)(B + o_w1t32);
  c->w2t32 = (float *)(B + o_w2t32);
  c->mub64 = (double *)(B + o_mub64);
  c->muw1_64 = (double *)(B + o_muw164);
  c->a_v1 = (__half *)(B + o_av1);
  c->a_v2 = (__half *)(B + o_av2);
  c->v1t32 = (float *)(B + o_v1t32);
  c->v2_32 = (float *)(B + o_v2_32);
  c->zero256 = (float *)(B + o_zero);
  uint16_t *tmp_e = (uint16_t *)setup.p;  // [mp][2048] each, kept components
  uint16_t *tmp_oe = tmp_e + (size_t)N_COEF * N_COEF;
  int32_t *scr = (int32_t *)(B + o_scr);
  cudaStream_t st = 0;

  if (cudaMemset(scr, 0, 64) != cudaSuccess || cudaMemset(c->zero256, 0, 4ull * N_HIDDEN) != cudaSuccess)
    return cleanup(fail(DCKV_ECUDA, "memset"));
  // drop mask, scale index, tables
  { k_scale_keep<<<(N_COEF + 255) / 256, 256, 0, st>>>(prm->laplace_b, prm->delta, c->scale, c->keep, scr); ++g_launches; }
  { k_tables<<<N_SCALES, 512, 0, st>>>(c->cdf); ++g_launches; }
  { k_build_lut<<<N_SCALES, 256, 0, st>>>(c->cdf, c->dcdf, c->lut, c->tail, c->cfm_tab); ++g_launches; }
  cudaMemcpyAsync(c->delta, prm->delta, 4ull * N_COEF, cudaMemcpyDeviceToDevice, st);
  cudaMemcpyAsync(c->lapb, prm->laplace_b, 4ull * N_COEF, cudaMemcpyDeviceToDevice, st);
  // scale exponents: largest |value| of each split operand brought to about 2^12
  { k_absmax<<<256, 256, 0, st>>>(prm->basis, (int64_t)ROW_DIM * N_COEF, N_COEF, nullptr, scr + 1); ++g_launches; }
  if (has_mlp) {
    { k_absmax<<<64, 256, 0, st>>>(prm->w2, (int64_t)N_HIDDEN * N_COEF, N_COEF, nullptr, scr + 2); ++g_launches; }
    { k_absmax<<<256, 256, 0, st>>>(prm->w1, (int64_t)ROW_DIM * N_HIDDEN, N_HIDDEN, nullptr, scr + 3); ++g_launches; }
  }
  { k_absmax<<<256, 256, 0, st>>>(prm->basis, (int64_t)ROW_DIM * N_COEF, N_COEF, prm->delta, scr + 4); ++g_launches; }
  if (has_synth) {  // synthesis operands: |V1| and |Delta| bound Delta * V1; |V2| joins the inverse's scale
    { k_absmax<<<128, 256, 0, st>>>(prm->v1, (int64_t)N_COEF * N_HIDDEN, N_HIDDEN, nullptr, scr + 6); ++g_launches; }
    { k_absmax<<<8, 256, 0, st>>>(prm->delta, (int64_t)N_COEF, N_COEF, nullptr, scr + 7); ++g_launches; }
    { k_absmax<<<256, 256, 0, st>>>(prm->v2, (int64_t)N_HIDDEN * ROW_DIM, ROW_DIM, nullptr, scr + 8); ++g_launches; }
  }
  int32_t host_scr[16];
  uint8_t keep_h[N_COEF], scale_h[N_COEF];
  if (cudaMemcpy(host_scr, scr, 64, cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemcpy(keep_h, c->keep, N_COEF, cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemcpy(scale_h, c->scale, N_COEF, cudaMemcpyDeviceToHost) != cudaSuccess)
    return cleanup(fail(DCKV_ECUDA, "setup readback failed: %s", cudaGetErrorString(cudaGetLastError())));
  if (host_scr[0]) return cleanup(fail(DCKV_EINVAL, "delta must be positive and laplace_b finite"));
  auto exp_for = [](int32_t bits) {
    float m;
    memcpy(&m, &bits, 4);
    if (!(m > 0.f) || !std::isfinite(m)) return 0;
    int e = (int)std::floor(std::log2(4096.0 / (double)m));
    return std::min(40, std::max(-40, e));
  };
  float mb, mw2;
  memcpy(&mb, &host_scr[1], 4);
  memcpy(&mw2, &host_scr[2], 4);
  int32_t mboth;
  const float mmax = std::max(mb, mw2);
  memcpy(&mboth, &mmax, 4);
  c->p_y = exp_for(mboth);
  c->p_h = exp_for(host_scr[3]);
  {
    float mi, mv2;
    memcpy(&mi, &host_scr[4], 4);
    memcpy(&mv2, &host_scr[8], 4);
    const float m = std::max(mi, has_synth ? mv2 : 0.f);  // the inverse GEMM's A: Delta B and V2
    int32_t bits;
    memcpy(&bits, &m, 4);
    c->p_inv = exp_for(bits);
    float mv1, md;
    memcpy(&mv1, &host_scr[6], 4);
    memcpy(&md, &host_scr[7], 4);
    const float mvd = mv1 * md;
    memcpy(&bits, &mvd, 4);
    c->p_v1 = has_synth ? exp_for(bits) : 0;
  }
  // kept components
  std::vector<int16_t> kl;
  std::vector<uint8_t> ks;
  for (int i = 0; i < N_COEF; ++i)
    if (keep_h[i]) {
      kl.push_back((int16_t)i);
      ks.push_back(scale_h[i]);
    }
  c->k_eff = (int)kl.size();
  c->kw = std::max(64, (c->k_eff + 63) / 64 * 64);
  c->mp = std::max(256, (c->k_eff + 255) / 256 * 256);
  std::vector<int16_t> kx(N_COEF, -1);
  for (int i = 0; i < c->k_eff; ++i) kx[kl[i]] = (int16_t)i;
  kl.resize(N_COEF, 0);
  ks.resize(N_COEF, 0);
  // entropy of the kept components' tables (bits per coded row): the chunk size is the
  // smallest one whose fixed cost (states, escape count, offset, pad: ~137 B) stays
  // within 3.5% of it, unless the caller fixed it
  {
    std::vector<uint16_t> cdf_h((size_t)N_SCALES * N_SYM);
    if (cudaMemcpy(cdf_h.data(), c->cdf, 2ull * N_SCALES * N_SYM, cudaMemcpyDeviceToHost) != cudaSuccess)
      return cleanup(fail(DCKV_ECUDA, "table readback failed"));
    double hs[N_SCALES];
    for (int s = 0; s < N_SCALES; ++s) {
      double h = 0.0;
      for (int k = 0; k < N_SYM; ++k) {
        const double f = (double)((k + 1 < N_SYM ? cdf_h[s * N_SYM + k + 1] : PREC_TOTAL) - cdf_h[s * N_SYM + k]);
        if (f > 0) h -= f / PREC_TOTAL * std::log2(f / PREC_TOTAL);
      }
      hs[s] = h;
    }
    double bits = 0.0;
    for (int i = 0; i < c->k_eff; ++i) bits += hs[ks[i]];
    c->model_bits_per_row = bits;
    if (c->chunk_rows == 0) c->chunk_rows = 16;
    if (c->chunk_rows < 0) {
      const double per_row = 0.035 * bits / 8.0;
      int g = per_row > 0 ? (int)std::ceil((CHUNK_FIXED_BYTES + 5) / per_row) : 256;
      c->chunk_rows = std::min(256, std::max(8, g));
    }
  }
  double theta_h[128];
  for (int i = 0; i < 128; ++i) theta_h[i] = std::pow(ROPE_BASE, -2.0 * i / HEAD_DIM);
  if (cudaMemcpy(c->kept_list, kl.data(), 2 * N_COEF, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(c->kept_scale, ks.data(), N_COEF, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(c->kidx, kx.data(), 2 * N_COEF, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(c->theta, theta_h, sizeof(theta_h), cudaMemcpyHostToDevice) != cudaSuccess)
    return cleanup(fail(DCKV_ECUDA, "setup upload failed"));
  // mean projections in fp64
  { k_vec_mat<<<(N_COEF + 255) / 256, 256, 0, st>>>(prm->mu, prm->basis, ROW_DIM, N_COEF, c->mub, c->mub64); ++g_launches; }
  if (has_mlp) { k_vec_mat<<<1, 256, 0, st>>>(prm->mu, prm->w1, ROW_DIM, N_HIDDEN, c->muw1, c->muw1_64); ++g_launches; }
  { k_permute_mu<<<(ROW_DIM + 255) / 256, 256, 0, st>>>(prm->mu, c->mu_perm); ++g_launches; }
  { k_compact_meta<<<(c->mp + 255) / 256, 256, 0, st>>>(prm->delta, c->mub, c->kept_list, c->k_eff, c->mp,
                                                       c->delta_k, c->mub_k); ++g_launches; }
  // split operands (hi/lo fp16, power-of-two scaled), kept components only where the
  // component is an index of the GEMM
  dim3 tb(32, 8);
  { k_split_kept_rows<<<dim3(ROW_DIM / 32, c->mp / 32), tb, 0, st>>>(prm->basis, ROW_DIM, c->kept_list, c->k_eff,
                                                                      c->mp, std::ldexp(1.0, c->p_y), c->a_y); ++g_launches; }
  if (has_mlp) {
    { k_split_kept_rows<<<dim3(N_HIDDEN / 32, c->mp / 32), tb, 0, st>>>(prm->w2, N_HIDDEN, c->kept_list, c->k_eff,
                                                                         c->mp, std::ldexp(1.0, c->p_y), c->a_w2); ++g_launches; }
    { k_split<<<dim3(ROW_DIM / 32, N_HIDDEN / 32), tb, 0, st>>>(prm->w1, N_HIDDEN, ROW_DIM, 0, nullptr, std::ldexp(1.0, c->p_h), c->a_h); ++g_launches; }
  }
  { k_split_kept_cols<<<(unsigned)((ROW_DIM * (int64_t)c->kw + 255) / 256), 256, 0, st>>>(
        prm->basis, ROW_DIM, true, c->kept_list, c->k_eff, c->kw, prm->delta, std::ldexp(1.0, c->p_inv), c->a_inv); ++g_launches; }
  // fp32 copies for the exact refinement
  { k_transpose32<<<dim3(ROW_DIM / 32, N_COEF / 32), tb, 0, st>>>(prm->basis, ROW_DIM, N_COEF, c->bt32); ++g_launches; }
  if (has_mlp) {
    { k_transpose32<<<dim3(ROW_DIM / 32, N_HIDDEN / 32), tb, 0, st>>>(prm->w1, ROW_DIM, N_HIDDEN, c->w1t32); ++g_launches; }
    { k_transpose32<<<dim3(N_HIDDEN / 32, N_COEF / 32), tb, 0, st>>>(prm->w2, N_HIDDEN, N_COEF, c->w2t32); ++g_launches; }
  }
  if (has_synth) {
    // a_v1[slab][h][c] = split(Delta_c V1[c][h] 2^p_v1); a_v2[slab][p][h] = split(V2[h][dim(p)] 2^p_inv)
    { k_split_v1_kept<<<(unsigned)((N_HIDDEN * (int64_t)c->kw + 255) / 256), 256, 0, st>>>(
          prm->v1, c->kept_list, c->k_eff, c->kw, prm->delta, std::ldexp(1.0, c->p_v1), c->a_v1); ++g_launches; }
    { k_split<<<dim3(N_HIDDEN / 32, ROW_DIM / 32), tb, 0, st>>>(prm->v2, ROW_DIM, N_HIDDEN, 2, nullptr, std::ldexp(1.0, c->p_inv), c->a_v2); ++g_launches; }
    { k_transpose32<<<dim3(N_COEF / 32, N_HIDDEN / 32), tb, 0, st>>>(prm->v1, N_COEF, N_HIDDEN, c->v1t32); ++g_launches; }
    cudaMemcpyAsync(c->v2_32, prm->v2, 4ull * N_HIDDEN * ROW_DIM, cudaMemcpyDeviceToDevice, st);
  }
  // mean-model weights, K-major
  if (has_means) {
    { k_gather_on<<<dim3(2 * c->kw / 32, c->mp / 32), tb, 0, st>>>(prm->w_odd, c->kept_list, c->k_eff, c->kw, c->mp,
                                                                  (uint16_t *)c->a_on); ++g_launches; }
    { k_transpose16<<<dim3(N_COEF / 32, c->mp / 32), tb, 0, st>>>(prm->w_even, N_COEF, 0, c->mp, N_COEF, tmp_e,
                                                                 c->kept_list, c->k_eff); ++g_launches; }
    { k_transpose16<<<dim3(N_COEF / 32, c->mp / 32), tb, 0, st>>>(prm->w_odd, N_COEF, 0, c->mp, N_COEF, tmp_oe,
                                                                 c->kept_list, c->k_eff); ++g_launches; }
  }
  if (cudaGetLastError() != cudaSuccess) return cleanup(fail(DCKV_ECUDA, "setup kernels failed to launch"));
  // tensor maps of the static operands
  int r = DCKV_OK;
  if ((r = map_a(&c->map_ay2, c->a_y, false, ROW_DIM, c->mp, 2, 2)) ||
      (r = map_a(&c->map_aw2_2, c->a_w2, false, N_HIDDEN, c->mp, 2, 2)) ||
      (r = map_a(&c->map_aw2_1, c->a_w2, false, N_HIDDEN, c->mp, 2, 1)) ||
      (r = map_a(&c->map_ah2, c->a_h, false, ROW_DIM, N_HIDDEN, 2, 2)) ||
      (r = map_a(&c->map_ainv2, c->a_inv, false, c->kw, ROW_DIM, 2, 2)) ||
      (r = map_a(&c->map_ainv1, c->a_inv, false, c->kw, ROW_DIM, 2, 1)) ||
      (r = map_a(&c->map_aon1, c->a_on, true, 2 * c->kw, c->mp, 1, 1)) ||
      (has_synth && (r = map_a(&c->map_av1, c->a_v1, false, c->kw, N_HIDDEN, 2, 2))) ||
      (has_synth && (r = map_a(&c->map_av2, c->a_v2, false, N_HIDDEN, ROW_DIM, 2, 2))))
    return cleanup(r);
  // the inverse's lo-half cut: the smallest multiple of 64 such that the lo halves of the
  // components past it carry at most INV_LO_THETA^2 of the expected signal energy,
  // E[q_m^2] |A_m|^2 summed over m, with E[q^2] = 2 beta^2 + 1/12 under the component's own
  // Laplace scale beta (in steps) and A_m = Delta_m basis[:, m].  The decoder-side synthesis
  // variant keeps the whole split (its extra operand takes the second tensor map).
  c->inv_lo_k = c->kw;
  if (!has_synth && c->k_eff > 0) {
    double *norms = (double *)((uint8_t *)setup.p + s_norms);
    { k_inv_colnorms<<<c->kw, 256, 0, st>>>(c->a_inv, c->kw, norms); ++g_launches; }
    std::vector<double> nh(2 * (size_t)c->kw);
    std::vector<float> bh(N_COEF), dh(N_COEF);
    if (cudaMemcpy(nh.data(), norms, 8ull * 2 * c->kw, cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemcpy(bh.data(), prm->laplace_b, 4ull * N_COEF, cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemcpy(dh.data(), prm->delta, 4ull * N_COEF, cudaMemcpyDeviceToHost) != cudaSuccess)
      return cleanup(fail(DCKV_ECUDA, "setup readback failed"));
    std::vector<double> lo_e(c->k_eff);
    double total = 0.0;
    for (int m = 0; m < c->k_eff; ++m) {
      const double beta = (double)bh[kl[m]] / (double)dh[kl[m]];
      const double eq2 = 2.0 * beta * beta + 1.0 / 12.0;
      lo_e[m] = eq2 * nh[m];
      total += eq2 * nh[c->kw + m];
    }
    double tail = 0.0;
    int cut = c->k_eff;  // smallest m with sum over m' >= m of lo_e[m'] within the bound
    for (int m = c->k_eff - 1; m >= 0; --m) {
      tail += lo_e[m];
      if (tail > INV_LO_THETA * INV_LO_THETA * total) break;
      cut = m;
    }
    c->inv_lo_k = std::min(c->kw, (cut + 63) / 64 * 64);
  }
  // per-vocabulary mean tables of the kept components (column kc = compact index), row
  // stride kw: t_odd = embed @ w_odd[0:2048] in fp32 and, since an even row's centre is the
  // table value itself, the even centres clamp(round(embed @ w_even), +-127) as int8 (the
  // fp32 even table passes through the odd table's buffer first)
  if (has_means) {
    if (cudaMalloc(&c->tab_blk, (size_t)V * c->kw * 5) != cudaSuccess)
      return cleanup(fail(DCKV_ECUDA, "cudaMalloc of the vocabulary tables failed"));
    c->t_odd = (float *)c->tab_blk;
    c->t_even8 = (int8_t *)c->tab_blk + (size_t)V * c->kw * 4;
    CUtensorMap ma_e, ma_o, mb_emb;
    if ((r = map_a(&ma_e, tmp_e, true, N_COEF, c->mp, 1, 1)) || (r = map_a(&ma_o, tmp_oe, true, N_COEF, c->mp, 1, 1)) ||
        (r = map_b(&mb_emb, prm->embed, true, N_COEF, V, 256)))
      return cleanup(r);
    for (int which = 0; which < 2; ++which) {
      GemmProblem pr = make_problem(c->mp / GEMM_BM, (int64_t)V, 256, true, scr + 5);
      add_seg(pr, 0, 0, 1, 0, 0, 0, 0, N_COEF / GEMM_BK);
      EpiStoreF32::Params ep{c->t_odd, c->kw, 1.0f, c->kw};
      if ((r = run_gemm<EpiStoreF32, 4, 1>(which ? ma_o : ma_e, ma_e, mb_emb, mb_emb, pr, ep, c->num_sms, st)))
        return cleanup(r);
      if (which == 0) {
        const int64_t n = (int64_t)V * c->kw;
        { k_round_centres<<<(unsigned)std::min<int64_t>((n + 255) / 256, 65535), 256, 0, st>>>(c->t_odd, n, c->t_even8); ++g_launches; }
      }
    }
  }
  if (cudaDeviceSynchronize() != cudaSuccess)
    return cleanup(fail(DCKV_ECUDA, "codec setup failed: %s", cudaGetErrorString(cudaGetLastError())));
  int32_t tmo = 0;
  cudaMemcpy(&tmo, scr + 5, 4, cudaMemcpyDeviceToHost);
  if (tmo) return cleanup(fail(DCKV_ETIMEOUT, "setup GEMM timed out"));
  *out = c;
  return DCKV_OK;
}

extern "C" void dckv_codec_destroy(dckv_codec *c) {
  if (!c) return;
  DeviceScope dev_scope(c->device);
  if (c->blk) cudaFree(c->blk);
  if (c->tab_blk) cudaFree(c->tab_blk);
  if (t_stages.codec == c) t_stages.codec = nullptr;
  delete c;
}

extern "C" int dckv_codec_k_eff(const dckv_codec *c) { return c ? c->k_eff : -1; }

extern "C" size_t dckv_workspace_bytes(const dckv_codec *c, const int64_t *offs, int batch) {
  if (!c) return 0;
  Layout L;
  if (build_layout(c, offs, batch, L) != DCKV_OK) return 0;
  return std::max(plan_ws(L, 0).total, plan_ws(L, 1).total);
}

extern "C" size_t dckv_blob_bound(const dckv_codec *c, const int64_t *offs, int batch) {
  if (!c) return 0;
  Layout L;
  if (build_layout(c, offs, batch, L) != DCKV_OK) return 0;
  // every symbol escaped: 8 bytes of escape value + one word each, plus fixed parts
  return L.off_streams + (uint64_t)L.n_chunks * (CHUNK_FIXED_BYTES + 4) + 10ull * L.n_symbols;
}

// The call's prompt table reaches the device as a kernel parameter (up to
// PROMPT_PARAM_MAX prompts; beyond that one host-to-device copy), and the chunk table is
// built from it on the device: no pageable copy on the launch path of ordinary batches.
constexpr int PROMPT_PARAM_MAX = 400;  // 400 x 56 B of kernel parameters
struct PromptPack {
  PromptInfo p[PROMPT_PARAM_MAX];
};

__global__ void k_build_tables(const __grid_constant__ PromptPack pk, const PromptInfo *src, int batch,
                               int n_chunks_e, int n_chunks, int G, int K, PromptInfo *prompts, ChunkDesc *chunks) {
  const PromptInfo *P = src ? src : pk.p;
  const int tid = blockIdx.x * blockDim.x + threadIdx.x, nth = gridDim.x * blockDim.x;
  if (!src)
    for (int b = tid; b < batch; b += nth) prompts[b] = pk.p[b];
  for (int ci = tid; ci < n_chunks; ci += nth) {
    const int par = ci >= n_chunks_e;
    int lo = 0, hi = batch;  // last prompt whose first chunk of this parity is <= ci
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if ((par ? P[mid].chunk_o0 : P[mid].chunk_e0) <= ci) lo = mid; else hi = mid;
    }
    const PromptInfo pi = P[lo];
    const int j0 = (ci - (par ? pi.chunk_o0 : pi.chunk_e0)) * G;
    const int nr = par ? pi.n_o : pi.n_e;
    ChunkDesc d;
    d.prompt = lo;
    d.parity = par;
    d.j0 = j0;
    d.nrows = min(G, nr - j0);
    d.sym_base = (int64_t)((par ? pi.slot_o0 : pi.slot_e0) + j0) * K;
    chunks[ci] = d;
  }
}

static int upload_tables(const dckv_codec *c, const Layout &L, uint8_t *ws, const WsPlan &w, cudaStream_t st) {
  static thread_local PromptPack pk;
  PromptInfo *dp = (PromptInfo *)(ws + w.prompts);
  const PromptInfo *src = nullptr;
  if (L.batch <= PROMPT_PARAM_MAX) {
    memcpy(pk.p, L.prompts.data(), sizeof(PromptInfo) * L.batch);
  } else {
    CK(cudaMemcpyAsync(dp, L.prompts.data(), sizeof(PromptInfo) * L.batch, cudaMemcpyHostToDevice, st));
    src = dp;
  }
  const int work = std::max(L.batch, L.n_chunks);
  const unsigned blocks = (unsigned)std::max(1, std::min((work + 255) / 256, 1024));
  k_build_tables<<<blocks, 256, 0, st>>>(pk, src, L.batch, L.n_chunks_e, L.n_chunks, c->chunk_rows, c->k_eff, dp,
                                         (ChunkDesc *)(ws + w.chunks));
  ++g_launches;
  CK(cudaGetLastError());
  return DCKV_OK;
}

// ============================================================================ encode
// The encoder.  stop = 0: the whole path; 1: stop once every code is final (after the
// exact recomputation; the closed-form fit reads the codes); 2: stop after the symbol
// kernel (centres final too).  With stop != 0 the blob may be NULL (kept rows are skipped).
static int encode_impl(const dckv_codec *c, const void *rows, const int32_t *token_ids, const int64_t *seq_offsets,
                       int batch, void *blob, size_t blob_cap, uint64_t *blob_size_dev, int32_t *status_dev,
                       void *workspace, size_t ws_bytes, void *stream, int stop) {
  if (!c || !rows || (!stop && (!blob || !blob_size_dev)) || !status_dev || !workspace ||
      (c->has_means && !token_ids))
    return fail(DCKV_EINVAL, "a pointer argument is NULL");
  if (!blob) blob_cap = 0;
  if (((uintptr_t)rows & 15) || ((uintptr_t)blob & 15) || ((uintptr_t)workspace & 255))
    return fail(DCKV_EINVAL, "rows/blob must be 16-byte and workspace 256-byte aligned");
  Layout L;
  RET(build_layout(c, seq_offsets, batch, L));
  const WsPlan w = plan_ws(L, 0);
  if (ws_bytes < w.total) return fail(DCKV_ECAPACITY, "workspace too small (%zu < %zu)", ws_bytes, w.total);
  cudaStream_t st = (cudaStream_t)stream;
  DEVICE_SCOPE(c->device);
  stage_begin(c);
  uint8_t *ws = (uint8_t *)workspace;
  uint8_t *bl = (uint8_t *)blob;
  PromptInfo *d_prompts = (PromptInfo *)(ws + w.prompts);
  ChunkDesc *d_chunks = (ChunkDesc *)(ws + w.chunks);
  int32_t *row_tok = (int32_t *)(ws + w.row_tok), *row_pos = (int32_t *)(ws + w.row_pos);
  int32_t *row_edst = (int32_t *)(ws + w.row_edst), *e_tok = (int32_t *)(ws + w.e_tok);
  int32_t *e_row = (int32_t *)(ws + w.e_row);
  __half *x16 = (__half *)(ws + w.x16);
  __half *g16 = (__half *)(ws + w.g16);
  int32_t *q32 = (int32_t *)(ws + w.q32);
  __nv_bfloat16 *qe = (__nv_bfloat16 *)(ws + w.qe);
  int32_t *row_slot = (int32_t *)(ws + w.row_slot), *e_slot = (int32_t *)(ws + w.e_slot);
  int8_t *cen8 = (int8_t *)(ws + w.cen8);
  uint16_t *sym16 = (uint16_t *)(ws + w.sym16);
  uint2 *cfm = (uint2 *)(ws + w.cf32);
  int32_t *slot_chunk = (int32_t *)(ws + w.slot_chunk);
  uint32_t *nesc_w = (uint32_t *)(ws + w.nesc);

  float *row_norm = (float *)(ws + w.row_norm);
  uint32_t *rowflag = (uint32_t *)(ws + w.rowflag);
  uint32_t *el_bins = (uint32_t *)(ws + w.el_bins), *full_list = (uint32_t *)(ws + w.full_list);
  uint32_t *bin_count = (uint32_t *)(ws + w.bin_count);
  uint32_t *counters = (uint32_t *)(ws + w.counters);  // [0] codes to refine, [1] rows to refine

  stage_mark(c, st, "start");
  CK(cudaMemsetAsync(status_dev, 0, 4, st));
  CK(cudaMemsetAsync(counters, 0, 256, st));
  if (L.n_rows) CK(cudaMemsetAsync(rowflag, 0, 4ull * L.n_rows, st));
  CK(cudaMemsetAsync(bin_count, 0, 4ull * N_COEF, st));
  if (L.n_chunks) CK(cudaMemsetAsync(nesc_w, 0, 4ull * L.n_chunks, st));
  RET(upload_tables(c, L, ws, w, st));
  { k_layout<<<dim3(L.batch, LAYOUT_SPLIT), 256, 0, st>>>(d_prompts, row_tok, row_pos, row_edst, row_slot, e_tok, e_slot, e_row, slot_chunk,
                                    c->chunk_rows, qe, c->kw); ++g_launches; }
  if (L.n_tokens > 0)
    { k_convert<<<(unsigned)L.n_tokens, 192, 0, st>>>((const __nv_bfloat16 *)rows, d_prompts, L.batch, x16, bl, blob_cap,
                                                    L.off_kept, row_norm, status_dev); ++g_launches; }
  CK(cudaGetLastError());
  stage_mark(c, st, "layout+convert");
  if (L.n_rows > 0) {
    CUtensorMap mb_xh, mb_xt, mb_gt, mb_qe;
    RET(map_b(&mb_xh, x16, false, ROW_DIM, L.n_rows, HIDDEN_SPLIT_BN / 2));
    const int bn_t = pick_pair_bn(L.n_rows, c->mp / 256, c->num_sms);  // transform token tile
    RET(map_b(&mb_xt, x16, false, ROW_DIM, L.n_rows, bn_t / 2));
    RET(map_b(&mb_gt, g16, false, 2 * N_HIDDEN, L.n_rows, bn_t / 2));
    RET(map_b(&mb_qe, qe, true, c->kw, L.ne_pad, MEAN_ODD_BN / 2, CODE_LD));
    // correction hidden layer: h = x @ w1 - mu @ w1, GELU, fp16 hi/lo
    if (c->has_mlp && (L.n_rows + HIDDEN_SPLIT_BN - 1) / HIDDEN_SPLIT_BN >= c->num_sms) {
      // enough token tiles for two per CTA pair: the K parts are summed in registers by the
      // chunk-accumulated kernel, whose epilogue applies GELU (no fp32 parts in memory)
      GemmProblem pr = make_problem(N_HIDDEN / GEMM_BM, L.n_rows, HIDDEN_SPLIT_BN, false, status_dev);
      add_seg(pr, 0, 0, 2, 0, 0, 0, 0, ROW_DIM / GEMM_BK);
      EpiGeluRegs::Params ep{c->muw1, (float)std::ldexp(1.0, -c->p_h), g16};
      RET((run_gemm2_chunked<EpiGeluRegs, 4, 2, ROW_DIM / GEMM_BK / HIDDEN_SPLIT, HIDDEN_SPLIT_BN>(
          c->map_ah2, c->map_ah2, mb_xh, mb_xh, pr, ep, c->num_sms, false, st)));
    } else if (c->has_mlp) {
      GemmProblem pr = make_problem(N_HIDDEN / GEMM_BM, L.n_rows, HIDDEN_SPLIT_BN, false, status_dev);
      add_seg(pr, 0, 0, 2, 0, 0, 0, 0, ROW_DIM / GEMM_BK);
      pr.k_split = HIDDEN_SPLIT;
      float *hpart = (float *)(ws + w.hpart);
      EpiPartF32::Params ep{hpart, N_HIDDEN, (int64_t)L.n_rows * N_HIDDEN};
      RET((run_gemm2<EpiPartF32, 4, 2, 8>(c->map_ah2, c->map_ah2, mb_xh, mb_xh, pr, ep, c->num_sms, false, st)));
      { k_gelu_parts<<<(unsigned)((L.n_rows * N_HIDDEN + 255) / 256), 256, 0, st>>>(
            hpart, HIDDEN_SPLIT, L.n_rows, c->muw1, (float)std::ldexp(1.0, -c->p_h), g16); ++g_launches; }
    }
    stage_mark(c, st, "gemm_hidden");
    // transform + quantiser: y = x @ B + g @ w2 - mu @ B
    {
      GemmProblem pr = make_problem(c->mp / GEMM_BM, L.n_rows, bn_t, false, status_dev);
      if (c->has_mlp) {  // g @ w2 (hi/lo on both sides) first, then x @ B
        add_seg(pr, 1, 0, 2, 0, 1, 0, 0, N_HIDDEN / GEMM_BK);
        add_seg(pr, 1, 0, 2, 0, 1, 0, N_HIDDEN, N_HIDDEN / GEMM_BK);
        // the first partial holds the small correction term and the first 256 elements of x @ B
        // (12 K steps instead of 4): the MMA then runs 16 K steps ahead of the epilogue while
        // the previous tile's codes are finished, about as long as that finishing takes
        pr.first_chunk = 2 * N_HIDDEN / GEMM_BK + TRANSFORM_CHUNK_STEPS;
      }
      add_seg(pr, 0, 0, 2, 0, 0, 0, 0, ROW_DIM / GEMM_BK);
      EpiQuantRegs::Params ep{{c->mub_k, c->delta_k, c->k_eff, (float)std::ldexp(1.0, -c->p_y), q32, qe,
                               row_edst},
                              row_norm, rowflag, el_bins, bin_count, full_list, counters, w.bin_cap,
                              c->dbg_ratio, c->kept_list};
      if (bn_t == TRANSFORM_BN)
        RET((run_gemm2_chunked<EpiQuantRegs, 4, 2, TRANSFORM_CHUNK_STEPS, TRANSFORM_BN>(
            c->map_ay2, c->map_aw2_2, mb_xt, mb_gt, pr, ep, c->num_sms, false, st)));
      else
        RET((run_gemm2_chunked<EpiQuantRegs, 4, 2, TRANSFORM_CHUNK_STEPS, 192>(
            c->map_ay2, c->map_aw2_2, mb_xt, mb_gt, pr, ep, c->num_sms, false, st)));
    }
    stage_mark(c, st, "gemm_transform");
    // codes whose fp32 ratio lies in the guard band around a half step: exact fp64 values
    CK(cudaFuncSetAttribute(k_refine_hidden, cudaFuncAttributeMaxDynamicSharedMemorySize, REFINE_SMEM));
    CK(cudaFuncSetAttribute(k_refine_rows, cudaFuncAttributeMaxDynamicSharedMemorySize, REFINE_SMEM));
    { k_refine_codes<<<c->num_sms * 2, REFINE_THREADS, 0, st>>>(
          el_bins, bin_count, w.bin_cap, (const __nv_bfloat16 *)rows, row_tok, c->mub64, c->bt32,
          c->has_mlp ? c->w2t32 : nullptr, g16, c->delta, rowflag, c->kept_list, q32, qe, row_edst);
      ++g_launches; }
    stage_mark(c, st, "refine_codes");
    double *g64 = (double *)(ws + w.g64);
    if (c->has_mlp)
      { k_refine_hidden<<<c->num_sms * 4, 256, REFINE_SMEM, st>>>(full_list, counters, (const __nv_bfloat16 *)rows,
                                                                  row_tok, c->muw1_64, c->w1t32, g64); ++g_launches; }
    { k_refine_rows<<<c->num_sms * 4, 256, REFINE_SMEM, st>>>(full_list, counters, (const __nv_bfloat16 *)rows,
                                                            row_tok, c->mub64, c->bt32,
                                                            c->has_mlp ? c->w2t32 : nullptr, g64, c->delta,
                                                            c->kept_list, c->k_eff, q32, qe, row_edst);
      ++g_launches; }
    CK(cudaGetLastError());
    stage_mark(c, st, "refine_rows");
    if (stop == 1) return DCKV_OK;
    // odd mean model: [e, bf16(q_left), bf16(q_right)] @ w_odd -> centres
    if (c->has_means) {
      GemmProblem pr = make_problem(c->mp / GEMM_BM, L.ne_pad, MEAN_ODD_BN, true, status_dev);
      add_seg(pr, 0, 0, 1, 0, 0, 0, 0, c->kw / GEMM_BK);
      add_seg(pr, 0, 0, 1, c->kw, 0, 1, 0, c->kw / GEMM_BK);
      EpiMeanOdd<false>::Params ep{c->t_odd, token_ids, e_tok, e_slot, c->kw, cen8, c->k_eff, c->vocab};
      RET((run_gemm2<EpiMeanOdd<false>, 6, 1, 16, MEAN_ODD_BN>(c->map_aon1, c->map_aon1, mb_qe, mb_qe, pr, ep, c->num_sms, true, st)));
    }
    stage_mark(c, st, "gemm_mean_odd");
    // even centres from the vocabulary table, then every symbol, in slot order
    const unsigned rg = (unsigned)std::min<int64_t>(L.n_rows, 65535);
    if (!c->has_means && L.n_symbols > 0)
      CK(cudaMemsetAsync(cen8, 0, (size_t)L.n_symbols, st));  // unconditional tables: every centre 0
    { k_symbols<<<rg, SYM_THREADS, 0, st>>>(L.n_rows, row_slot, slot_chunk, q32, cen8, c->kept_scale, c->cfm_tab,
                                          c->k_eff, c->has_means ? c->t_even8 : nullptr, c->kw, token_ids,
                                          row_tok, row_edst, c->vocab, sym16, cfm, nesc_w); ++g_launches; }
    CK(cudaGetLastError());
    stage_mark(c, st, "symbols");
  }
  if (stop) return DCKV_OK;
  uint32_t *states = (uint32_t *)(ws + w.states), *nwords = (uint32_t *)(ws + w.nwords);
  uint32_t *nesc = (uint32_t *)(ws + w.nesc), *offs = (uint32_t *)(ws + w.offs);
  if (L.n_chunks > 0) {
    RansEncArgs a{d_chunks, L.n_chunks, c->k_eff, cfm, (uint16_t *)(ws + w.words), states, nwords};
    { rans_encode_kernel<<<(L.n_chunks + RANS_WARPS - 1) / RANS_WARPS, RANS_WARPS * 32, 0, st>>>(a); ++g_launches; }
    CK(cudaGetLastError());
  }
  stage_mark(c, st, "rans_encode");
  {
    ScanArgs a{L.n_chunks, nwords, nesc, offs, bl, blob_cap, L.off_kept, L.off_streams, d_prompts, L.batch,
               c->chunk_rows, c->k_eff, L.n_chunks_e, L.n_chunks_o, L.n_kept, blob_size_dev, status_dev};
    { scan_kernel<<<1, 1024, 0, st>>>(a); ++g_launches; }
    CK(cudaGetLastError());
  }
  if (L.n_chunks > 0) {
    CompactArgs a{d_chunks, d_prompts, L.n_chunks, c->k_eff, q32, sym16,
                  (const uint16_t *)(ws + w.words), states, nwords, nesc, offs, bl, blob_cap, L.off_streams};
    { compact_kernel<<<L.n_chunks, COMPACT_THREADS, 0, st>>>(a); ++g_launches; }
    CK(cudaGetLastError());
  }
  stage_mark(c, st, "scan+compact");
  return DCKV_OK;
}

extern "C" int dckv_encode(const dckv_codec *c, const void *rows, const int32_t *token_ids, const int64_t *seq_offsets,
                           int batch, void *blob, size_t blob_cap, uint64_t *blob_size_dev, int32_t *status_dev,
                           void *workspace, size_t ws_bytes, void *stream) {
  return encode_impl(c, rows, token_ids, seq_offsets, batch, blob, blob_cap, blob_size_dev, status_dev, workspace,
                     ws_bytes, stream, 0);
}

// ============================================================================ decode
extern "C" int dckv_decode(const dckv_codec *c, const void *blob, size_t blob_bytes, const int32_t *token_ids,
                           const int64_t *seq_offsets, int batch, void *k_out, void *v_out, int32_t *status_dev,
                           void *workspace, size_t ws_bytes, void *stream) {
  if (!c || !blob || !k_out || !v_out || !status_dev || !workspace || (c->has_means && !token_ids))
    return fail(DCKV_EINVAL, "a pointer argument is NULL");
  if (((uintptr_t)blob & 15) || ((uintptr_t)k_out & 15) || ((uintptr_t)v_out & 15) || ((uintptr_t)workspace & 255))
    return fail(DCKV_EINVAL, "blob/k_out/v_out must be 16-byte and workspace 256-byte aligned");
  Layout L;
  RET(build_layout(c, seq_offsets, batch, L));
  const WsPlan w = plan_ws(L, 1);
  if (ws_bytes < w.total) return fail(DCKV_ECAPACITY, "workspace too small (%zu < %zu)", ws_bytes, w.total);
  cudaStream_t st = (cudaStream_t)stream;
  DEVICE_SCOPE(c->device);
  stage_begin(c);
  uint8_t *ws = (uint8_t *)workspace;
  const uint8_t *bl = (const uint8_t *)blob;
  PromptInfo *d_prompts = (PromptInfo *)(ws + w.prompts);
  ChunkDesc *d_chunks = (ChunkDesc *)(ws + w.chunks);
  int32_t *row_tok = (int32_t *)(ws + w.row_tok), *row_pos = (int32_t *)(ws + w.row_pos);
  int32_t *row_edst = (int32_t *)(ws + w.row_edst), *e_tok = (int32_t *)(ws + w.e_tok);
  int32_t *e_row = (int32_t *)(ws + w.e_row);
  __nv_bfloat16 *qe = (__nv_bfloat16 *)(ws + w.qe);
  int32_t *row_slot = (int32_t *)(ws + w.row_slot), *e_slot = (int32_t *)(ws + w.e_slot);
  int8_t *cen8 = (int8_t *)(ws + w.cen8);
  int32_t *slot_chunk = (int32_t *)(ws + w.slot_chunk);
  uint16_t *syms16 = (uint16_t *)(ws + w.slots16);
  float2 *rope = (float2 *)(ws + w.rope);
  __half *q16 = (__half *)(ws + w.q16);
  int32_t *qbig = (int32_t *)(ws + w.qbig);
  uint32_t *bigflag = (uint32_t *)(ws + w.bigflag);
  int32_t *biglist = (int32_t *)(ws + w.biglist);
  uint32_t *counters = (uint32_t *)(ws + w.counters);  // [0] big-row count, [1] header valid
  int32_t *valid = (int32_t *)(counters + 1);

  stage_mark(c, st, "start");
  CK(cudaMemsetAsync(status_dev, 0, 4, st));
  CK(cudaMemsetAsync(counters, 0, 256, st));
  RET(upload_tables(c, L, ws, w, st));
  // every kept code of every row is written below (escapes by the patch); only the pad
  // columns K_eff .. kw - 1, which the GEMMs read against zero operands, and each prompt's
  // zero right-neighbour row (by k_layout) are cleared here
  if (c->kw > c->k_eff) {
    CK(cudaMemset2DAsync(qe + c->k_eff, 2ull * CODE_LD, 0, 2ull * (c->kw - c->k_eff), (size_t)L.ne_pad, st));
    if (L.n_rows)
      CK(cudaMemset2DAsync(q16 + c->k_eff, 2ull * CODE_LD, 0, 2ull * (c->kw - c->k_eff), (size_t)L.n_rows, st));
  }
  if (L.n_rows) CK(cudaMemsetAsync(bigflag, 0, 4ull * L.n_rows, st));
  if (L.n_chunks) CK(cudaMemsetAsync(ws + w.escflag, 0, 4ull * L.n_chunks, st));
  { k_layout<<<dim3(L.batch, LAYOUT_SPLIT), 256, 0, st>>>(d_prompts, row_tok, row_pos, row_edst, row_slot, e_tok, e_slot, e_row, slot_chunk,
                                    c->chunk_rows, qe, c->kw); ++g_launches; }
  HeaderCheck hc{bl, blob_bytes, d_prompts, L.batch, c->chunk_rows, c->k_eff, L.n_chunks_e, L.n_chunks_o,
                 L.n_kept, L.off_kept, L.off_streams, valid, status_dev};
  { k_check_header<<<1, 256, 0, st>>>(hc); ++g_launches; }
  if (L.max_len > 0)
    { k_rope_table<<<(unsigned)std::min<int64_t>(L.max_len, 4096), 128, 0, st>>>(rope, L.max_len, c->theta, valid); ++g_launches; }
  CK(cudaGetLastError());
  stage_mark(c, st, "layout+check");
  const uint32_t *offs = (const uint32_t *)(bl + HEADER_BYTES + 4ull * L.batch);
  CK(cudaFuncSetAttribute(rans_decode_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, RANS_DEC_SMEM));
  CK(cudaFuncSetAttribute(rans_decode_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, RANS_DEC_SMEM));
  RansDecArgs da{d_chunks, 0, L.n_chunks, c->k_eff, c->kept_scale, c->dcdf, c->lut, c->tail, bl, L.off_streams,
                 offs, syms16, valid, status_dev};
  uint32_t *escflag = (uint32_t *)(ws + w.escflag);
  DecCodesArgs fa{d_chunks, d_prompts, 0, L.n_chunks_e, c->k_eff, syms16, bl, L.off_streams,
                  offs, q16, qe, qbig, bigflag, biglist, counters, escflag, valid, status_dev};
  const unsigned rg = (unsigned)std::max<int64_t>(1, std::min<int64_t>(L.n_rows, 65535));
  if (L.n_chunks > 0) {
    // one block per SM at most (each holds the tables), chunks spread over the blocks
    const unsigned g = (unsigned)std::max(1, std::min(c->num_sms, L.n_chunks));
    if (c->k_eff >= 32)
      { rans_decode_kernel<true><<<g, DEC_WARPS * 32, RANS_DEC_SMEM, st>>>(da); ++g_launches; }
    else
      { rans_decode_kernel<false><<<g, DEC_WARPS * 32, RANS_DEC_SMEM, st>>>(da); ++g_launches; }
  }
  CK(cudaGetLastError());
  stage_mark(c, st, "rans_loop");
  if (L.n_chunks_e > 0) {
    { k_codes_elem<<<rg, 256, 0, st>>>(0, L.n_rows, row_edst, row_slot, slot_chunk, syms16,
                                       c->has_means ? c->t_even8 : nullptr, c->kw, token_ids, row_tok, c->vocab,
                                       c->k_eff, q16, qe, escflag, valid); ++g_launches; }
    { k_escape_patch<<<(unsigned)L.n_chunks_e, PATCH_THREADS, 0, st>>>(fa); ++g_launches; }
  }
  CK(cudaGetLastError());
  stage_mark(c, st, "codes_even");
  if (L.n_rows > 0 && c->has_means) {
    CUtensorMap mb_qe;
    RET(map_b(&mb_qe, qe, true, c->kw, L.ne_pad, MEAN_ODD_BN / 2, CODE_LD));
    GemmProblem pr = make_problem(c->mp / GEMM_BM, L.ne_pad, MEAN_ODD_BN, true, status_dev);
    add_seg(pr, 0, 0, 1, 0, 0, 0, 0, c->kw / GEMM_BK);
    add_seg(pr, 0, 0, 1, c->kw, 0, 1, 0, c->kw / GEMM_BK);
    // odd centres, and with them the odd codes (ESC symbols are left to the patch)
    EpiMeanOdd<true>::Params ep{c->t_odd, token_ids, e_tok, e_slot, c->kw, cen8, c->k_eff, c->vocab,
                                syms16, q16, e_row, slot_chunk, escflag};
    RET((run_gemm2<EpiMeanOdd<true>, 6, 1, 16, MEAN_ODD_BN>(c->map_aon1, c->map_aon1, mb_qe, mb_qe, pr, ep, c->num_sms, true, st)));
  }
  stage_mark(c, st, "gemm_mean_odd");
  if (L.n_chunks_o > 0) {
    if (!c->has_means)  // unconditional tables: every odd centre is 0
      { k_codes_elem<<<rg, 256, 0, st>>>(1, L.n_rows, row_edst, row_slot, slot_chunk, syms16, nullptr, c->kw,
                                         token_ids, row_tok, c->vocab,
                                         c->k_eff, q16, qe, escflag, valid); ++g_launches; }
    fa.chunk0 = L.n_chunks_e;
    fa.n_chunks = L.n_chunks_o;
    { k_escape_patch<<<(unsigned)L.n_chunks_o, PATCH_THREADS, 0, st>>>(fa); ++g_launches; }
    CK(cudaGetLastError());
  }
  stage_mark(c, st, "codes_odd");
  __half *g16d = (__half *)(ws + w.g16);
  if (L.n_rows > 0 && c->has_synth) {  // decoder-side synthesis, hidden layer: GELU((q Delta) V1)
    CUtensorMap mb_qh;
    RET(map_b(&mb_qh, q16, false, c->kw, L.n_rows, HIDDEN_BN / 2, CODE_LD));
    GemmProblem pr = make_problem(N_HIDDEN / GEMM_BM, L.n_rows, HIDDEN_BN, false, status_dev);
    add_seg(pr, 0, 0, 2, 0, 0, 0, 0, c->kw / GEMM_BK);
    EpiGelu::Params ep{c->zero256, (float)std::ldexp(1.0, -c->p_v1), g16d};
    RET((run_gemm2<EpiGelu, 4, 2, 4, HIDDEN_BN>(c->map_av1, c->map_av1, mb_qh, mb_qh, pr, ep, c->num_sms, false, st)));
    stage_mark(c, st, "gemm_synth_hidden");
  }
  if (L.n_rows > 0) {
    CUtensorMap mb_q, mb_g;
    const int bn_i = pick_pair_bn(L.n_rows, ROW_DIM / 256, c->num_sms);  // inverse token tile
    RET(map_b(&mb_q, q16, false, c->kw, L.n_rows, bn_i / 2, CODE_LD));
    GemmProblem pr = make_problem(ROW_DIM / GEMM_BM, L.n_rows, bn_i, false, status_dev);
    // hi and lo halves up to the cut, the hi half alone after it (second A map, one slab)
    if (c->inv_lo_k > 0) add_seg(pr, 0, 0, 2, 0, 0, 0, 0, c->inv_lo_k / GEMM_BK);
    if (c->inv_lo_k < c->kw) add_seg(pr, 1, 0, 1, c->inv_lo_k, 0, 0, c->inv_lo_k, (c->kw - c->inv_lo_k) / GEMM_BK);
    if (c->has_synth) {  // + g V2 (hi/lo on both sides)
      RET(map_b(&mb_g, g16d, false, 2 * N_HIDDEN, L.n_rows, bn_i / 2));
      add_seg(pr, 1, 0, 2, 0, 1, 0, 0, N_HIDDEN / GEMM_BK);
      add_seg(pr, 1, 0, 2, 0, 1, 0, N_HIDDEN, N_HIDDEN / GEMM_BK);
    } else {
      mb_g = mb_q;
    }
    EpiInverse::Params ep{c->mu_perm, (float)std::ldexp(1.0, -c->p_inv), rope, row_tok, row_pos,
                          (__nv_bfloat16 *)k_out, (__nv_bfloat16 *)v_out, L.n_tokens};
    RET((run_gemm2<EpiInverse, 4, 2, 8>(c->map_ainv2, c->has_synth ? c->map_av2 : c->map_ainv1, mb_q, mb_g, pr, ep,
                                        c->num_sms, false, st)));
  }
  stage_mark(c, st, "gemm_inverse");
  if (L.n_kept > 0)
    { k_kept<<<(unsigned)L.n_kept, 256, 0, st>>>(bl, L.off_kept, d_prompts, L.batch, rope, (__nv_bfloat16 *)k_out,
                                              (__nv_bfloat16 *)v_out, L.n_tokens, valid); ++g_launches; }
  if (L.n_rows > 0)
    { k_fixup<<<c->num_sms, 256, 0, st>>>(biglist, counters, q16, qbig, c->a_inv, (float)std::ldexp(1.0, -c->p_inv),
                                       c->mu_perm, c->theta, row_tok, row_pos, (__nv_bfloat16 *)k_out,
                                       (__nv_bfloat16 *)v_out, L.n_tokens, c->has_synth ? c->v1t32 : nullptr,
                                       c->v2_32, c->delta, c->kept_list, c->k_eff, c->kw); ++g_launches; }
  CK(cudaGetLastError());
  stage_mark(c, st, "kept+fixup");
  return DCKV_OK;
}

// ============================================================================ bytes
extern "C" int dckv_bytes(const void *blob_host, size_t len, dckv_byte_report *out) {
  if (!blob_host || !out) return fail(DCKV_EINVAL, "NULL argument");
  memset(out, 0, sizeof(*out));
  const uint8_t *b = (const uint8_t *)blob_host;
  if (len < (size_t)HEADER_BYTES) return fail(DCKV_ECORRUPT, "blob shorter than its header");
  uint32_t h32[8];
  uint16_t h16[4];
  uint64_t h64[4];
  memcpy(h32, b, 32);
  memcpy(h16, b, 8);
  memcpy(h64, b + 32, 32);
  if (h32[0] != MAGIC || h16[2] != VERSION || h32[3] != (uint32_t)N_COEF || h16[3] == 0)
    return fail(DCKV_ECORRUPT, "bad header");
  const uint64_t total = h64[0], off_s = h64[1], off_k = h64[2];
  const uint32_t nb = h32[2], n_ch = h32[5] + h32[6], n_kept = h32[7];
  if (total > len) return fail(DCKV_ECORRUPT, "blob truncated");
  const uint64_t tab_end = HEADER_BYTES + 4ull * (nb + (uint64_t)n_ch + 1);
  if (tab_end > total || off_k != align_up(tab_end, 16) || off_s != off_k + (uint64_t)n_kept * ROW_DIM * 2 ||
      off_s > total)
    return fail(DCKV_ECORRUPT, "bad offsets");
  std::vector<uint32_t> lens(nb), offs(n_ch + 1);
  memcpy(lens.data(), b + HEADER_BYTES, 4ull * nb);
  memcpy(offs.data(), b + HEADER_BYTES + 4ull * nb, 4ull * (n_ch + 1));
  if (off_s + offs[n_ch] != total) return fail(DCKV_ECORRUPT, "chunk table does not reach the end");
  uint64_t rows = 0;
  for (uint32_t n : lens) rows += n > (uint32_t)(HEAD_KEPT + TAIL_KEPT) ? n - HEAD_KEPT - TAIL_KEPT : 0;
  for (uint32_t ci = 0; ci < n_ch; ++ci) {
    if (offs[ci + 1] < offs[ci] || offs[ci + 1] - offs[ci] < (uint32_t)CHUNK_FIXED_BYTES)
      return fail(DCKV_ECORRUPT, "bad chunk %u", ci);
    uint32_t ne;
    memcpy(&ne, b + off_s + offs[ci] + 4 * LANES, 4);
    const uint64_t sz = offs[ci + 1] - offs[ci];
    if (CHUNK_FIXED_BYTES + 8ull * ne > sz) return fail(DCKV_ECORRUPT, "bad escape count in chunk %u", ci);
    out->states += 4 * LANES;
    out->esc_counts += 4;
    out->esc_values += 8ull * ne;
    out->n_escapes += ne;
    // words cannot be told from a trailing zero pad word without decoding; count both
    out->words += sz - CHUNK_FIXED_BYTES - 8ull * ne;
  }
  out->total = total;
  out->header_tables = off_k;
  out->kept_rows = off_s - off_k;
  out->payload = total - out->kept_rows;
  out->padding = 0;
  out->n_prompts = nb;
  out->n_chunks = n_ch;
  out->n_coded_rows = (uint32_t)rows;
  out->chunk_rows = h16[3];
  out->k_eff = h32[4];
  return DCKV_OK;
}

// ============================================================================ inspection
extern "C" int dckv_set_timing(dckv_codec *c, int enable) {
  if (!c) return DCKV_EINVAL;
  c->timing = enable ? 1 : 0;
  if (t_stages.codec == c) t_stages.n = 0;
  return DCKV_OK;
}
extern "C" int dckv_get_timing(const dckv_codec *c, float *ms, const char **names, int max) {
  if (!c || !ms) return -1;
  const StageLog &g = t_stages;
  if (g.codec != c) return 0;
  int n = 0;
  for (int i = 1; i < g.n && n < max; ++i, ++n) {
    float t = 0.f;
    cudaEventElapsedTime(&t, g.ev[i - 1], g.ev[i]);
    ms[n] = t;
    if (names) names[n] = g.names[i];
  }
  return n;
}

extern "C" int dckv_codec_export(const dckv_codec *c, uint16_t *cdf_host, uint8_t *scale_host, uint8_t *keep_host,
                                 int32_t *exps_host) {
  if (!c) return fail(DCKV_EINVAL, "NULL codec");
  DEVICE_SCOPE(c->device);
  if (cdf_host) CK(cudaMemcpy(cdf_host, c->cdf, 2ull * N_SCALES * N_SYM, cudaMemcpyDeviceToHost));
  if (scale_host) CK(cudaMemcpy(scale_host, c->scale, N_COEF, cudaMemcpyDeviceToHost));
  if (keep_host) CK(cudaMemcpy(keep_host, c->keep, N_COEF, cudaMemcpyDeviceToHost));
  if (exps_host) {
    exps_host[0] = c->p_y;
    exps_host[1] = c->p_h;
    exps_host[2] = c->p_inv;
  }
  return DCKV_OK;
}

extern "C" int dckv_debug_ratio(dckv_codec *c, void *ratio_dev) {
  if (!c) return fail(DCKV_EINVAL, "NULL codec");
  c->dbg_ratio = (float *)ratio_dev;
  return DCKV_OK;
}

extern "C" long long dckv_launch_count(void) { return g_launches.load(); }

extern "C" int dckv_codec_info(const dckv_codec *c, int32_t *chunk_rows, double *model_bits_per_row) {
  if (!c) return fail(DCKV_EINVAL, "NULL codec");
  if (chunk_rows) *chunk_rows = c->chunk_rows;
  if (model_bits_per_row) *model_bits_per_row = c->model_bits_per_row;
  return DCKV_OK;
}

extern "C" int dckv_codec_gemm_shape(const dckv_codec *c, int32_t *shape) {
  if (!c || !shape) return fail(DCKV_EINVAL, "NULL argument");
  shape[0] = c->k_eff;
  shape[1] = c->kw;
  shape[2] = c->mp;
  shape[3] = c->inv_lo_k;
  return DCKV_OK;
}

extern "C" int dckv_codec_tables(const dckv_codec *c, const void **t_even, const void **t_odd) {
  if (!c) return fail(DCKV_EINVAL, "NULL codec");
  if (t_even) *t_even = c->t_even8;
  if (t_odd) *t_odd = c->t_odd;
  return DCKV_OK;
}

extern "C" int dckv_ws_offsets(const dckv_codec *c, const int64_t *offs, int batch, int which, dckv_ws_view *out) {
  if (!c || !out) return fail(DCKV_EINVAL, "NULL argument");
  Layout L;
  RET(build_layout(c, offs, batch, L));
  const WsPlan w = plan_ws(L, which);
  out->q32 = w.q32;
  out->qe = w.qe;
  out->cen8 = w.cen8;
  out->row_slot = w.row_slot;
  out->sym16 = w.sym16;
  out->q16 = w.q16;
  out->x16 = w.x16;
  out->g16 = w.g16;
  out->counters = w.counters;
  out->n_rows = L.n_rows;
  out->ne_pad = L.ne_pad;
  out->n_chunks = L.n_chunks;
  out->total = w.total;
  out->code_width = c->kw;
  return DCKV_OK;
}

// D[n][m] = sum_s sum_k A[s][m][k] * B[n][k] through the tcgen05 GEMM (self-test).
extern "C" int dckv_debug_gemm(int bf16, const void *A, int slabs, const void *Bm, int M, int N, int K, float *D,
                               int bn, int pair, void *stream) {
  if (!A || !Bm || !D || M % GEMM_BM || K % GEMM_BK || N < 1 || slabs < 1 || slabs > 2 || bn < 16 || bn > 256 ||
      bn % 16 || (pair && M % (2 * GEMM_BM)))
    return fail(DCKV_EINVAL, "bad GEMM shape");
  int dev;
  CK(cudaGetDevice(&dev));
  int sms;
  CK(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  CUtensorMap ma, mb;
  RET(map_a(&ma, A, bf16 != 0, K, M, slabs, slabs));
  RET(map_b(&mb, Bm, bf16 != 0, K, N, pair ? bn / 2 : bn));
  GemmProblem pr = make_problem(M / GEMM_BM, N, bn, bf16 != 0, nullptr);
  add_seg(pr, 0, 0, slabs, 0, 0, 0, 0, K / GEMM_BK);
  EpiStoreF32::Params ep{D, M, 1.0f};
  if (pair) return run_gemm2<EpiStoreF32, 4, 2, 4>(ma, ma, mb, mb, pr, ep, sms, bf16 != 0, (cudaStream_t)stream);
  return run_gemm<EpiStoreF32, 3, 2>(ma, ma, mb, mb, pr, ep, sms, (cudaStream_t)stream);
}

// ============================================================================ decode, static scratch
// Scratch of dckv_decode_static: one file-scope device array per GPU that loads this
// library, held until the process exits.  Callers that cannot hand over a workspace use it:
// a serving engine that has reserved all free device memory for its KV-cache pool before
// it restores cached prompts, or a host program without a device allocator of its own --
// they have no spare device memory to offer, and allocating inside the call would
// synchronise the device and could fail under memory pressure.
static __device__ __align__(256) uint8_t g_static_scratch[DCKV_STATIC_SCRATCH_BYTES];

namespace {
constexpr int MAX_DEVICES = 64;
std::mutex g_static_mu;
void *g_static_ptr[MAX_DEVICES] = {};  // device address of g_static_scratch, per device
}  // namespace

extern "C" int dckv_decode_static(const dckv_codec *c, const void *blob, size_t blob_bytes,
                                  const int32_t *token_ids, const int64_t *seq_offsets, int batch, void *k_out,
                                  void *v_out, int32_t *status_dev, void *stream) {
  if (!c) return fail(DCKV_EINVAL, "codec is NULL");
  Layout L;
  RET(build_layout(c, seq_offsets, batch, L));
  const size_t need = plan_ws(L, 1).total;
  if (need > (size_t)DCKV_STATIC_SCRATCH_BYTES)
    return fail(DCKV_ECAPACITY, "batch needs %zu bytes of decode scratch; the static scratch holds %zu", need,
                (size_t)DCKV_STATIC_SCRATCH_BYTES);
  if (c->device < 0 || c->device >= MAX_DEVICES) return fail(DCKV_EINVAL, "device %d out of range", c->device);
  DEVICE_SCOPE(c->device);
  void *scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (!g_static_ptr[c->device]) {  // first call on this device: look the array up once
      void *p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
      if (e != cudaSuccess || !p)
        return fail(DCKV_ECUDA, "cudaGetSymbolAddress(static scratch) failed: %s", cudaGetErrorString(e));
      g_static_ptr[c->device] = p;
    }
    scratch = g_static_ptr[c->device];
  }
  return dckv_decode(c, blob, blob_bytes, token_ids, seq_offsets, batch, k_out, v_out, status_dev, scratch,
                     (size_t)DCKV_STATIC_SCRATCH_BYTES, stream);
}

// closed-form fit of the conditional models (calibration; not on the encode/decode path)
#include "dckv_fit.cuh"
