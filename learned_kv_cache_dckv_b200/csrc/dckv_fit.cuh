// dckv_fit.cuh -- closed-form fit of the conditional entropy models (included by dckv.cu).
//
// "DCKV: Learned Transform Coding of the Prompt KV Cache in Hybrid Language Models"
// (trove.briskstack.com summary), section "Evidence": the conditional models fitted in
// closed form to a trained codec.  The formulas this library reads into that sentence
// are stated in include/dckv_fit.h.
//
// Data path: the encoder (up to its final codes) -> transposed bf16 regressors and hi/lo
// targets in the workspace -> CTA-pair tcgen05 GEMMs X^T X and Y^T X over row slices,
// fp64 accumulation in the epilogue -> fp64 blocked Cholesky and triangular solves.
#pragma once

namespace dckv {

constexpr int FIT_SLICE = 4096;  // calibration rows per GEMM launch (fp32 TMEM accumulation)
constexpr int FIT_BN = 256;
constexpr int FB = 64;           // fp64 block size of the factorisation
constexpr int CODE_CLIP = 32767;

struct FitPlan {
  WsPlan enc;
  size_t inv, et, yet, xot, yot, total;
  int64_t n_e, n_o, ke, ko;  // rows of each parity and their padded counts (columns)
};

static FitPlan plan_fit(const Layout &L) {
  FitPlan f;
  f.enc = plan_ws(L, 0);
  f.n_e = 0;
  for (const PromptInfo &p : L.prompts) f.n_e += p.n_e;
  f.n_o = L.n_rows - f.n_e;
  f.ke = (f.n_e + 63) / 64 * 64;
  f.ko = (f.n_o + 63) / 64 * 64;
  uint64_t o = (f.enc.total + 255) / 256 * 256;
  auto take = [&](uint64_t bytes) {
    const uint64_t at = o;
    o = (o + std::max<uint64_t>(bytes, 1) + 255) / 256 * 256;
    return (size_t)at;
  };
  f.inv = take(4ull * L.n_rows);
  f.et = take(2ull * N_COEF * f.ke);
  f.yet = take(2ull * 2 * N_COEF * f.ke);
  f.xot = take(2ull * 3 * N_COEF * f.ko);
  f.yot = take(2ull * 2 * N_COEF * f.ko);
  f.total = o;
  return f;
}

__global__ void k_fit_inv(int64_t n_rows, const int32_t *row_slot, int32_t *inv) {
  const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (r < n_rows) inv[row_slot[r]] = (int32_t)r;
}

struct FitRegArgs {
  const PromptInfo *prompts;
  int batch;
  const int32_t *inv;        // slot row -> coded row (natural order)
  const int32_t *row_tok;    // coded row -> token index in the batch
  const int32_t *token_ids;
  const uint16_t *embed;     // bf16 [vocab][2048]
  int vocab;
  const int32_t *q32;        // [n_rows][CODE_LD] final codes of the kept components (compact order)
  const int16_t *kidx;       // [2048] compact index of a component, -1 if dropped (code 0)
  int64_t slot0, n, kpad;    // first slot row of the parity, its rows, padded columns
  int n_x;                   // regressors: 2048 (even) or 6144 (odd)
  uint16_t *x_t;             // [n_x][kpad]        bf16 regressors, transposed
  uint16_t *y_t;             // [2][2048][kpad]    bf16 hi / lo of the clipped codes
};

// code of component c of coded row r (0 for a dropped component)
__device__ __forceinline__ int32_t code_of(const FitRegArgs &a, int64_t r, int c) {
  const int m = __ldg(a.kidx + c);
  return m >= 0 ? __ldg(a.q32 + r * CODE_LD + m) : 0;
}

__device__ __forceinline__ uint16_t bf16_bits_of_code(int32_t q) {
  return __bfloat16_as_ushort(__double2bfloat16((double)q));  // one RNE step, as the mean model reads q
}

// One block: 64 columns (calibration rows of one parity) x 64 features of the combined
// index [regressors | targets]; values staged in shared memory, stored transposed.
__global__ void __launch_bounds__(256) k_fit_regress(FitRegArgs a) {
  __shared__ __align__(16) uint16_t hi[64][66];
  __shared__ __align__(16) uint16_t lo[64][66];
  const int64_t col0 = (int64_t)blockIdx.x * 64;
  const int f0 = blockIdx.y * 64;
  const bool target = f0 >= a.n_x;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int cc = ty; cc < 64; cc += 8) {
    const int64_t col = col0 + cc;
    uint16_t vh[2] = {0, 0}, vl[2] = {0, 0};
    if (col < a.n) {
      const int64_t r = a.inv[a.slot0 + col];
      const int64_t t = a.row_tok[r];
      if (target) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int c = f0 - a.n_x + tx + 32 * h;
          const int32_t q = min(max(code_of(a, r, c), -CODE_CLIP), CODE_CLIP);
          const __nv_bfloat16 bh = __float2bfloat16_rn((float)q);  // exact below 2^8, else the hi part
          vh[h] = __bfloat16_as_ushort(bh);
          vl[h] = __bfloat16_as_ushort(__float2bfloat16_rn((float)q - __bfloat162float(bh)));  // exact
        }
      } else {
        const int tok = min(max(__ldg(a.token_ids + t), 0), a.vocab - 1);
        bool right_ok = true;
        if (f0 >= 2 * N_COEF) {
          const PromptInfo pi = a.prompts[find_prompt(a.prompts, a.batch, t)];
          right_ok = (r - pi.row_base) + 1 < pi.n;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int f = f0 + tx + 32 * h;
          if (f < N_COEF)
            vh[h] = __ldg(a.embed + (int64_t)tok * N_COEF + f);
          else if (f < 2 * N_COEF)
            vh[h] = bf16_bits_of_code(code_of(a, r - 1, f - N_COEF));
          else
            vh[h] = right_ok ? bf16_bits_of_code(code_of(a, r + 1, f - 2 * N_COEF)) : 0;
        }
      }
    }
    hi[tx][cc] = vh[0];
    hi[tx + 32][cc] = vh[1];
    lo[tx][cc] = vl[0];
    lo[tx + 32][cc] = vl[1];
  }
  __syncthreads();
  for (int ff = ty; ff < 64; ff += 8) {
    const int f = f0 + ff;
    const uint32_t vh = *reinterpret_cast<const uint32_t *>(&hi[ff][2 * tx]);
    if (target) {
      const int c = f - a.n_x;
      const uint32_t vl = *reinterpret_cast<const uint32_t *>(&lo[ff][2 * tx]);
      *reinterpret_cast<uint32_t *>(a.y_t + (int64_t)c * a.kpad + col0 + 2 * tx) = vh;
      *reinterpret_cast<uint32_t *>(a.y_t + ((int64_t)N_COEF + c) * a.kpad + col0 + 2 * tx) = vl;
    } else {
      *reinterpret_cast<uint32_t *>(a.x_t + (int64_t)f * a.kpad + col0 + 2 * tx) = vh;
    }
  }
}

__global__ void k_fit_count(double *n_out, int64_t n_e, int64_t n_o) {
  n_out[0] += (double)n_e;
  n_out[1] += (double)n_o;
}

// out [N][M] fp64 += sum over the K columns of A (M rows, `slabs` slabs) times B (N rows),
// one launch per slice of FIT_SLICE columns.
static int fit_gram(const CUtensorMap &ma, int slabs, const CUtensorMap &mb, int M, int N, int64_t kpad, double *out,
                    int32_t *status, int num_sms, cudaStream_t st) {
  for (int64_t k0 = 0; k0 < kpad; k0 += FIT_SLICE) {
    const int steps = (int)(std::min<int64_t>(FIT_SLICE, kpad - k0) / GEMM_BK);
    GemmProblem pr = make_problem(M / GEMM_BM, N, FIT_BN, true, status);
    add_seg(pr, 0, 0, slabs, (int)k0, 0, 0, (int)k0, steps);
    EpiAccF64::Params ep{out, (int64_t)M};
    RET((run_gemm2<EpiAccF64, 4, 2, 8>(ma, ma, mb, mb, pr, ep, num_sms, true, st)));
  }
  return DCKV_OK;
}

// ------------------------------------------------------------------ fp64 factorisation
// Blocked right-looking Cholesky A = L L^T (lower triangle, row-major, n a multiple of
// 64), then L L^T W = C for a row-major right-hand side C [n][r].  Only lower-triangle
// blocks are read; the strictly upper part of A is left as scratch.
__global__ void __launch_bounds__(256) k_fit_prep(const double *G, int n, double ridge, double *A) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (int64_t)n * n) return;
  const int64_t i = e / n, j = e % n;
  const double g = G[e];
  A[e] = (i == j) ? g + ridge * (g + 1.0) : g;
}

__global__ void __launch_bounds__(256) k_chol_diag(double *A, int n, int k, int32_t *status) {
  __shared__ double s[FB][FB + 1];
  const int k0 = k * FB;
  {  // loads into registers first: a shared-memory store between two global loads serialises them
    double v[FB * FB / 256];
#pragma unroll
    for (int u = 0; u < FB * FB / 256; ++u) {
      const int e = threadIdx.x + 256 * u;
      v[u] = A[(int64_t)(k0 + e / FB) * n + k0 + e % FB];
    }
#pragma unroll
    for (int u = 0; u < FB * FB / 256; ++u) {
      const int e = threadIdx.x + 256 * u;
      s[e / FB][e % FB] = v[u];
    }
  }
  __syncthreads();
  for (int j = 0; j < FB; ++j) {
    if (threadIdx.x == 0) {
      double d = s[j][j];
      if (!(d > 0.0)) {
        atomicExch(status, DCKV_ESINGULAR);
        d = 1.0;
      }
      s[j][j] = sqrt(d);
    }
    __syncthreads();
    const double djj = s[j][j];
    for (int i = j + 1 + threadIdx.x; i < FB; i += blockDim.x) s[i][j] /= djj;
    __syncthreads();
    for (int e = threadIdx.x; e < FB * FB; e += blockDim.x) {
      const int i = e / FB, l = e % FB;
      if (l > j && l <= i) s[i][l] -= s[i][j] * s[l][j];
    }
    __syncthreads();
  }
  for (int e = threadIdx.x; e < FB * FB; e += blockDim.x) {
    const int i = e / FB, l = e % FB;
    if (l <= i) A[(int64_t)(k0 + i) * n + k0 + l] = s[i][l];
  }
}

// Panel below the diagonal block k: A_ik <- A_ik L_kk^-T (one thread per row).
__global__ void __launch_bounds__(FB) k_chol_panel(double *A, int n, int k) {
  extern __shared__ double dsm[];
  double(*Lk)[FB + 1] = reinterpret_cast<double(*)[FB + 1]>(dsm);
  double(*P)[FB + 1] = reinterpret_cast<double(*)[FB + 1]>(dsm + FB * (FB + 1));
  const int k0 = k * FB;
  const int64_t r0 = k0 + FB + (int64_t)blockIdx.x * FB;
  const int t = threadIdx.x;
#pragma unroll
  for (int i0 = 0; i0 < FB; i0 += 16) {  // 32 loads in flight, then their shared-memory stores
    double lv[16], pv[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      lv[u] = A[(int64_t)(k0 + i0 + u) * n + k0 + t];
      pv[u] = A[(r0 + i0 + u) * n + k0 + t];
    }
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      Lk[i0 + u][t] = lv[u];
      P[i0 + u][t] = pv[u];
    }
  }
  __syncthreads();
  for (int j = 0; j < FB; ++j) {
    double x = P[t][j];
    for (int p = 0; p < j; ++p) x -= P[t][p] * Lk[j][p];
    P[t][j] = x / Lk[j][j];
  }
  __syncthreads();
  for (int i = 0; i < FB; ++i) A[(r0 + i) * n + k0 + t] = P[i][t];
}

// O[M][N] -= P[M][64] Q[64][N] over 64 x 64 output blocks; P(i, p) = TP ? P[p ldp + i] :
// P[i ldp + p]; Q(p, j) = TQ ? Q[j ldq + p] : Q[p ldq + j]; LOWER skips blocks above the
// block diagonal.
template <bool TP, bool TQ, bool LOWER>
__global__ void __launch_bounds__(256) k_dgemm64(int M, int N, const double *P, int64_t ldp, const double *Q,
                                                 int64_t ldq, double *O, int64_t ldo) {
  extern __shared__ double dsm[];
  double(*Ps)[FB + 1] = reinterpret_cast<double(*)[FB + 1]>(dsm);
  double(*Qs)[FB + 1] = reinterpret_cast<double(*)[FB + 1]>(dsm + FB * (FB + 1));
  const int bi = blockIdx.y, bj = blockIdx.x;
  if (LOWER && bj > bi) return;
  const int i0 = bi * FB, j0 = bj * FB;
  const int t = threadIdx.x;
  {  // 32 loads in flight, then their shared-memory stores
    double pv[FB * FB / 256], qv[FB * FB / 256];
#pragma unroll
    for (int u = 0; u < FB * FB / 256; ++u) {
      const int e = t + 256 * u;
      const int a = e / FB, b = e % FB;  // b runs along memory
      if (TP) pv[u] = (i0 + b < M) ? P[(int64_t)a * ldp + i0 + b] : 0.0;
      else pv[u] = (i0 + a < M) ? P[(int64_t)(i0 + a) * ldp + b] : 0.0;
      if (TQ) qv[u] = (j0 + a < N) ? Q[(int64_t)(j0 + a) * ldq + b] : 0.0;
      else qv[u] = (j0 + b < N) ? Q[(int64_t)a * ldq + j0 + b] : 0.0;
    }
#pragma unroll
    for (int u = 0; u < FB * FB / 256; ++u) {
      const int e = t + 256 * u;
      const int a = e / FB, b = e % FB;
      if (TP) Ps[b][a] = pv[u];
      else Ps[a][b] = pv[u];
      if (TQ) Qs[b][a] = qv[u];
      else Qs[a][b] = qv[u];
    }
  }
  __syncthreads();
  const int tx = t & 15, ty = t >> 4;
  double acc[4][4];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[r][c] = 0.0;
#pragma unroll 4
  for (int p = 0; p < FB; ++p) {
    double av[4], bv[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) av[r] = Ps[ty + 16 * r][p];
#pragma unroll
    for (int c = 0; c < 4; ++c) bv[c] = Qs[p][tx + 16 * c];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[r][c] = fma(av[r], bv[c], acc[r][c]);
  }
  // all sixteen loads before the stores (O may alias P or Q as far as the compiler knows)
  double cur[4][4];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int i = i0 + ty + 16 * r, j = j0 + tx + 16 * c;
      cur[r][c] = (i < M && j < N) ? O[(int64_t)i * ldo + j] : 0.0;
    }
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int i = i0 + ty + 16 * r, j = j0 + tx + 16 * c;
      if (i < M && j < N) O[(int64_t)i * ldo + j] = cur[r][c] - acc[r][c];
    }
}

// Right-hand-side block k: Y_k <- L_kk^-1 Y_k (FWD) or L_kk^-T Y_k (backward), one thread
// per column.
template <bool FWD>
__global__ void __launch_bounds__(128) k_trsm_rhs(const double *A, int n, int k, double *Y, int r) {
  extern __shared__ double dsm[];
  double(*Lk)[FB + 1] = reinterpret_cast<double(*)[FB + 1]>(dsm);
  double(*Ys)[129] = reinterpret_cast<double(*)[129]>(dsm + FB * (FB + 1));
  const int k0 = k * FB, c0 = blockIdx.x * 128, t = threadIdx.x;
  const bool ok = c0 + t < r;
#pragma unroll
  for (int g = 0; g < FB * FB / 128; g += 16) {  // 16 loads in flight, then their stores
    double v[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int e = t + 128 * (g + u);
      v[u] = A[(int64_t)(k0 + e / FB) * n + k0 + e % FB];
    }
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int e = t + 128 * (g + u);
      Lk[e / FB][e % FB] = v[u];
    }
  }
#pragma unroll
  for (int i0 = 0; i0 < FB; i0 += 16) {
    double v[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) v[u] = ok ? Y[(int64_t)(k0 + i0 + u) * r + c0 + t] : 0.0;
#pragma unroll
    for (int u = 0; u < 16; ++u) Ys[i0 + u][t] = v[u];
  }
  __syncthreads();
  if (FWD) {
    for (int i = 0; i < FB; ++i) {
      double y = Ys[i][t];
      for (int p = 0; p < i; ++p) y -= Lk[i][p] * Ys[p][t];
      Ys[i][t] = y / Lk[i][i];
    }
  } else {
    for (int i = FB - 1; i >= 0; --i) {
      double y = Ys[i][t];
      for (int p = i + 1; p < FB; ++p) y -= Lk[p][i] * Ys[p][t];
      Ys[i][t] = y / Lk[i][i];
    }
  }
  if (ok)
    for (int i = 0; i < FB; ++i) Y[(int64_t)(k0 + i) * r + c0 + t] = Ys[i][t];
}

static int chol_solve(double *A, int n, double *Y, int r, int32_t *status, cudaStream_t st) {
  const int nb = n / FB;
  const int dg_smem = 2 * FB * (FB + 1) * 8;
  const int tr_smem = (FB * (FB + 1) + FB * 129) * 8;
  CK(cudaFuncSetAttribute(k_chol_panel, cudaFuncAttributeMaxDynamicSharedMemorySize, dg_smem));
  CK(cudaFuncSetAttribute(k_dgemm64<false, true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, dg_smem));
  CK(cudaFuncSetAttribute(k_dgemm64<false, false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, dg_smem));
  CK(cudaFuncSetAttribute(k_dgemm64<true, false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, dg_smem));
  CK(cudaFuncSetAttribute(k_trsm_rhs<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, tr_smem));
  CK(cudaFuncSetAttribute(k_trsm_rhs<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, tr_smem));
  for (int k = 0; k < nb; ++k) {
    const int k0 = k * FB, rest = n - k0 - FB;
    { k_chol_diag<<<1, 256, 0, st>>>(A, n, k, status); ++g_launches; }
    if (rest > 0) {
      { k_chol_panel<<<rest / FB, FB, dg_smem, st>>>(A, n, k); ++g_launches; }
      const double *pan = A + (int64_t)(k0 + FB) * n + k0;
      { k_dgemm64<false, true, true><<<dim3(rest / FB, rest / FB), 256, dg_smem, st>>>(
            rest, rest, pan, n, pan, n, A + (int64_t)(k0 + FB) * n + k0 + FB, n); ++g_launches; }
    }
  }
  const unsigned cb = (unsigned)((r + 127) / 128);
  for (int k = 0; k < nb; ++k) {  // L Z = C
    const int k0 = k * FB, rest = n - k0 - FB;
    { k_trsm_rhs<true><<<cb, 128, tr_smem, st>>>(A, n, k, Y, r); ++g_launches; }
    if (rest > 0)
      { k_dgemm64<false, false, false><<<dim3((r + FB - 1) / FB, rest / FB), 256, dg_smem, st>>>(
            rest, r, A + (int64_t)(k0 + FB) * n + k0, n, Y + (int64_t)k0 * r, r, Y + (int64_t)(k0 + FB) * r, r); ++g_launches; }
  }
  for (int k = nb - 1; k >= 0; --k) {  // L^T W = Z
    const int k0 = k * FB;
    { k_trsm_rhs<false><<<cb, 128, tr_smem, st>>>(A, n, k, Y, r); ++g_launches; }
    if (k0 > 0)
      { k_dgemm64<true, false, false><<<dim3((r + FB - 1) / FB, k0 / FB), 256, dg_smem, st>>>(
            k0, r, A + (int64_t)k0 * n, n, Y + (int64_t)k0 * r, r, Y, r); ++g_launches; }
  }
  CK(cudaGetLastError());
  return DCKV_OK;
}

__global__ void k_fit_bf16(const double *w, int64_t count, uint16_t *out) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < count; e += (int64_t)gridDim.x * blockDim.x)
    out[e] = __bfloat16_as_ushort(__double2bfloat16(w[e]));
}

// Scale sums: thread k of a block keeps the sum of |q - centre| of kept components
// k, k + 256, ... over the block's rows; integer sums, so the result is exact.
__global__ void __launch_bounds__(256) k_fit_absres(int64_t n_rows, const int32_t *row_slot, const int32_t *q32,
                                                    const int8_t *cen8, const int16_t *kept_list, int k_eff,
                                                    unsigned long long *abs_sum) {
  constexpr int PER = N_COEF / 256;
  long long acc[PER];
#pragma unroll
  for (int u = 0; u < PER; ++u) acc[u] = 0;
  for (int64_t r = blockIdx.x; r < n_rows; r += gridDim.x) {
    const int64_t base = (int64_t)row_slot[r] * k_eff;
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const int k = threadIdx.x + 256 * u;
      if (k < k_eff) {
        const long long d = (long long)__ldg(q32 + r * CODE_LD + k) - (long long)cen8[base + k];
        acc[u] += d < 0 ? -d : d;
      }
    }
  }
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int k = threadIdx.x + 256 * u;
    if (k < k_eff && acc[u]) atomicAdd(abs_sum + kept_list[k], (unsigned long long)acc[u]);
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) atomicAdd(abs_sum + N_COEF, (unsigned long long)n_rows);
}

__global__ void k_fit_scales_finish(const int64_t *abs_sum, const float *b_old, const float *delta,
                                    const uint8_t *keep, float *b_out) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= N_COEF) return;
  const int64_t rows = abs_sum[N_COEF];
  float b = b_old[c];
  if (keep[c] && rows > 0) {
    const double d = (double)delta[c];
    const double beta = fmax((double)abs_sum[c] / (double)rows, B0_STEPS);
    b = __double2float_rn(d * beta);
    if ((double)b / d < B0_STEPS) b = nextafterf(b, INFINITY);
  }
  b_out[c] = b;
}

}  // namespace dckv

// ============================================================================ C ABI
extern "C" size_t dckv_fit_workspace_bytes(const dckv_codec *c, const int64_t *offs, int batch) {
  Layout L;
  if (!c || build_layout(c, offs, batch, L) != DCKV_OK) return 0;
  return plan_fit(L).total;
}

extern "C" size_t dckv_fit_solve_workspace_bytes(void) { return 8ull * 3 * N_COEF * 3 * N_COEF; }

extern "C" int dckv_fit_accumulate(const dckv_codec *c, const uint16_t *embed, int32_t vocab, const void *rows,
                                   const int32_t *token_ids, const int64_t *seq_offsets, int batch, double *stats,
                                   int32_t *status_dev, void *workspace, size_t ws_bytes, void *stream) {
  if (!c || !embed || !token_ids || !stats) return fail(DCKV_EINVAL, "a pointer argument is NULL");
  if (vocab < 1) return fail(DCKV_EINVAL, "vocab must be positive");
  if (((uintptr_t)stats & 7) || ((uintptr_t)embed & 1) || ((uintptr_t)token_ids & 3))
    return fail(DCKV_EINVAL, "stats must be 8-byte, embed 2-byte and token ids 4-byte aligned");
  Layout L;
  RET(build_layout(c, seq_offsets, batch, L));
  const FitPlan f = plan_fit(L);
  if (ws_bytes < f.total) return fail(DCKV_ECAPACITY, "workspace too small (%zu < %zu)", ws_bytes, f.total);
  RET(encode_impl(c, rows, token_ids, seq_offsets, batch, nullptr, 0, nullptr, status_dev, workspace, ws_bytes,
                  stream, 1));
  cudaStream_t st = (cudaStream_t)stream;
  uint8_t *ws = (uint8_t *)workspace;
  if (L.n_rows > 0) {
    int32_t *inv = (int32_t *)(ws + f.inv);
    { k_fit_inv<<<(unsigned)((L.n_rows + 255) / 256), 256, 0, st>>>(L.n_rows, (const int32_t *)(ws + f.enc.row_slot), inv); ++g_launches; }
    FitRegArgs a[2];
    for (int par = 0; par < 2; ++par) {
      a[par] = FitRegArgs{(const PromptInfo *)(ws + f.enc.prompts), L.batch, inv,
                          (const int32_t *)(ws + f.enc.row_tok), token_ids, embed, vocab,
                          (const int32_t *)(ws + f.enc.q32), c->kidx, par ? f.n_e : 0, par ? f.n_o : f.n_e,
                          par ? f.ko : f.ke, par ? 3 * N_COEF : N_COEF,
                          (uint16_t *)(ws + (par ? f.xot : f.et)), (uint16_t *)(ws + (par ? f.yot : f.yet))};
      if (a[par].n == 0) continue;
      { k_fit_regress<<<dim3((unsigned)(a[par].kpad / 64), (unsigned)((a[par].n_x + N_COEF) / 64)), 256, 0, st>>>(a[par]); ++g_launches; }
      CK(cudaGetLastError());
    }
    stage_mark(c, st, "fit_regress");
    for (int par = 0; par < 2; ++par) {
      if (a[par].n == 0) continue;
      CUtensorMap ma_x, ma_y, mb_x;
      RET(map_a(&ma_x, a[par].x_t, true, (uint64_t)a[par].kpad, (uint64_t)a[par].n_x, 1, 1));
      RET(map_a(&ma_y, a[par].y_t, true, (uint64_t)a[par].kpad, (uint64_t)N_COEF, 2, 2));
      RET(map_b(&mb_x, a[par].x_t, true, (uint64_t)a[par].kpad, (uint64_t)a[par].n_x, FIT_BN / 2));
      double *g_out = stats + (par ? DCKV_FIT_OFF_GO : DCKV_FIT_OFF_GE);
      double *c_out = stats + (par ? DCKV_FIT_OFF_CO : DCKV_FIT_OFF_CE);
      RET(fit_gram(ma_x, 1, mb_x, a[par].n_x, a[par].n_x, a[par].kpad, g_out, status_dev, c->num_sms, st));  // X^T X
      RET(fit_gram(ma_y, 2, mb_x, N_COEF, a[par].n_x, a[par].kpad, c_out, status_dev, c->num_sms, st));    // (Y^T X)^T
    }
    stage_mark(c, st, "fit_gram");
  }
  { k_fit_count<<<1, 1, 0, st>>>(stats + DCKV_FIT_OFF_N, f.n_e, f.n_o); ++g_launches; }
  CK(cudaGetLastError());
  return DCKV_OK;
}

extern "C" int dckv_fit_solve(const double *stats, double ridge, double *w_even, double *w_odd, int32_t *status_dev,
                              void *workspace, size_t ws_bytes, void *stream) {
  if (!stats || !w_even || !w_odd || !status_dev || !workspace) return fail(DCKV_EINVAL, "a pointer argument is NULL");
  if (((uintptr_t)stats | (uintptr_t)w_even | (uintptr_t)w_odd | (uintptr_t)workspace) & 7)
    return fail(DCKV_EINVAL, "fp64 buffers must be 8-byte aligned");
  if (!(ridge > 0.0) || !std::isfinite(ridge)) return fail(DCKV_EINVAL, "ridge must be positive and finite");
  if (ws_bytes < dckv_fit_solve_workspace_bytes()) return fail(DCKV_ECAPACITY, "solve workspace too small");
  cudaStream_t st = (cudaStream_t)stream;
  double *A = (double *)workspace;
  CK(cudaMemsetAsync(status_dev, 0, 4, st));
  for (int par = 0; par < 2; ++par) {
    const int n = par ? 3 * N_COEF : N_COEF;
    const double *G = stats + (par ? DCKV_FIT_OFF_GO : DCKV_FIT_OFF_GE);
    const double *C = stats + (par ? DCKV_FIT_OFF_CO : DCKV_FIT_OFF_CE);
    double *W = par ? w_odd : w_even;
    { k_fit_prep<<<(unsigned)(((int64_t)n * n + 255) / 256), 256, 0, st>>>(G, n, ridge, A); ++g_launches; }
    CK(cudaMemcpyAsync(W, C, 8ull * n * N_COEF, cudaMemcpyDeviceToDevice, st));
    RET(chol_solve(A, n, W, N_COEF, status_dev, st));
  }
  return DCKV_OK;
}

extern "C" int dckv_fit_to_bf16(const double *w, int64_t count, uint16_t *out, void *stream) {
  if (!w || !out || count < 0 || ((uintptr_t)w & 7) || ((uintptr_t)out & 1)) return fail(DCKV_EINVAL, "bad arguments");
  if (count == 0) return DCKV_OK;
  cudaStream_t st = (cudaStream_t)stream;
  { k_fit_bf16<<<(unsigned)std::min<int64_t>((count + 255) / 256, 4096), 256, 0, st>>>(w, count, out); ++g_launches; }
  CK(cudaGetLastError());
  return DCKV_OK;
}

extern "C" int dckv_fit_scales_accumulate(const dckv_codec *c, const void *rows, const int32_t *token_ids,
                                          const int64_t *seq_offsets, int batch, int64_t *abs_sum,
                                          int32_t *status_dev, void *workspace, size_t ws_bytes, void *stream) {
  if (!c || !abs_sum) return fail(DCKV_EINVAL, "a pointer argument is NULL");
  if ((uintptr_t)abs_sum & 7) return fail(DCKV_EINVAL, "abs_sum must be 8-byte aligned");
  Layout L;
  RET(build_layout(c, seq_offsets, batch, L));
  const WsPlan w = plan_ws(L, 0);
  RET(encode_impl(c, rows, token_ids, seq_offsets, batch, nullptr, 0, nullptr, status_dev, workspace, ws_bytes,
                  stream, 2));
  cudaStream_t st = (cudaStream_t)stream;
  uint8_t *ws = (uint8_t *)workspace;
  const unsigned grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>(L.n_rows, (int64_t)c->num_sms * 4));
  { k_fit_absres<<<grid, 256, 0, st>>>(L.n_rows, (const int32_t *)(ws + w.row_slot), (const int32_t *)(ws + w.q32),
                                     (const int8_t *)(ws + w.cen8), c->kept_list, c->k_eff,
                                     (unsigned long long *)abs_sum); ++g_launches; }
  CK(cudaGetLastError());
  return DCKV_OK;
}

extern "C" int dckv_fit_scales_finish(const dckv_codec *c, const int64_t *abs_sum, float *laplace_b, void *stream) {
  if (!c || !abs_sum || !laplace_b) return fail(DCKV_EINVAL, "a pointer argument is NULL");
  if (((uintptr_t)abs_sum & 7) || ((uintptr_t)laplace_b & 3)) return fail(DCKV_EINVAL, "misaligned buffer");
  cudaStream_t st = (cudaStream_t)stream;
  { k_fit_scales_finish<<<(N_COEF + 255) / 256, 256, 0, st>>>(abs_sum, c->lapb, c->delta, c->keep, laplace_b); ++g_launches; }
  CK(cudaGetLastError());
  return DCKV_OK;
}
