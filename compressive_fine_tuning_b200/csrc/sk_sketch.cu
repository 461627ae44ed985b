// Sketching stage: from a dense weight Theta [n][d] and calibration
// activations X [s][d] to the frozen index map and the first LUTs
// ("SpaLLM: Unified Compressive Adaptation of LLMs with Sketching", section
// 2.2: weighted Lloyd's algorithm for learning sketched parameters, learning
// the sketching matrix, groups per row; "Sketch to Adapt" OpenReview
// discussion, concern 1: the mapping is fixed one column at a time, each
// step followed by an update of the parameters not yet mapped).
//
//   1. H = X^T X: a tcgen05 GEMM over the calibration tokens, both operands
//      MN-major straight from TMA, fp32 accumulators in TMEM; only the tiles
//      that touch the upper triangle run, and they also write the mirror;
//   2. damping and the inverse factor U (H^-1 = U^T U, U upper), in float64:
//      the index-reversed H is factored by a blocked Cholesky (diagonal
//      block in one CTA, panel solve one thread per row, trailing updates as
//      GEMMs of rank 64 inside and 128 across super-blocks of two blocks),
//      the lower factor is inverted by blocked forward substitution in the
//      same super-blocks, and reversing the indices of that inverse gives U;
//      diag(H^-1) is the column sums of squares of U;
//   3. weighted Lloyd per (row, group), one CTA each: the group's values are
//      sorted once in shared memory, so a cluster is a contiguous range and
//      an assignment is k - 1 binary searches against float32 midpoints;
//      each warp sums one cluster in float64;
//   4. the mapping in blocks of 128 columns: one warp per row walks the
//      block's columns in order (nearest fp16 centroid by float32 midpoints,
//      then the compensation of the block's later columns), and a float64
//      GEMM applies the block's compensation to every later column.
//
// After the Gram matrix all sums and carried values are float64 and every
// integer decision (a cluster, a chosen centroid) compares a value with a
// float32 midpoint, so the decisions agree with a float64 evaluation except
// for values within rounding distance of a midpoint.
#include <cfloat>
#include <cmath>

#include "sk_tc.cuh"

namespace sk {
namespace {

__host__ __device__ constexpr int cdiv(int64_t a, int64_t b) { return (int)((a + b - 1) / b); }

// ============================================================================
// 1. Gram matrix on the tensor cores
// ============================================================================

namespace gr {
constexpr int M = 128, N = 256;
constexpr int KS = 64;              // tokens per pipeline step
constexpr int S = 4;                // stages
constexpr int A_BYTES = 2 * 8192;   // X[:, i0:i0+128]: two 64-column MN atoms x 8 K-groups
constexpr int B_BYTES = 4 * 8192;   // X[:, j0:j0+256]: four 64-column MN atoms
constexpr int STAGE = A_BYTES + B_BYTES;
constexpr int BAR_OFF = S * STAGE;
constexpr int SMEM = 1024 + BAR_OFF + 256;
constexpr int THREADS = 192;        // warps 0-3 epilogue, 4 TMA, 5 MMA
constexpr int TMA_WARP = 4, MMA_WARP = 5;
constexpr uint32_t IDESC = tc::idesc_bf16(M, N, 1, 1);
constexpr int TMEM_COLS = 256;
}  // namespace gr

// H[i0:i0+128][j0:j0+256] (+)= sum_t X[t][i] X[t][j].  H is symmetric, so
// only tiles that touch the upper triangle (j >= i) run; their epilogue
// writes each upper element H[i][j] and its mirror H[j][i] (for a fixed
// column the warp's 32 rows make one coalesced 128-byte store).
__global__ void __launch_bounds__(gr::THREADS, 1)
gram_tc_kernel(const __grid_constant__ CUtensorMap tm_x, int64_t s, int64_t d, float* __restrict__ H, int accumulate,
               unsigned int* check) {
  using namespace gr;
  if ((int64_t)blockIdx.x * N + N - 1 < (int64_t)blockIdx.y * M) return;   // entirely below the diagonal
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* empty = full + S;
  uint64_t* d_full = empty + S;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(d_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = tc::warp_id(), lane = tc::lane_id();
  const int64_t j0 = (int64_t)blockIdx.x * N;
  const int64_t i0 = (int64_t)blockIdx.y * M;
  const int nsteps = cdiv(s, KS);

  if (threadIdx.x == 0) {
    for (int st = 0; st < S; ++st) {
      tc::mbar_init(&full[st], 1);
      tc::mbar_init(&empty[st], 1);
    }
    tc::mbar_init(d_full, 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == MMA_WARP) tc::tmem_alloc(tmem_slot, TMEM_COLS);
  if (warp == TMA_WARP && lane == 0) tc::tma_prefetch(&tm_x);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == TMA_WARP) {
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nsteps && !*abort_flag; ++i) {
        const int st = i % S;
        if (!tc::mbar_wait(&empty[st], ((i / S) & 1) ^ 1, check)) { *abort_flag = 1; break; }
        uint8_t* buf = smem + st * STAGE;
        tc::mbar_arrive_expect_tx(&full[st], STAGE);
        const int tk = i * KS;
        tc::tma_load_2d(buf, &tm_x, &full[st], (int)i0, tk);
        tc::tma_load_2d(buf + 8192, &tm_x, &full[st], (int)i0 + 64, tk);
#pragma unroll
        for (int q = 0; q < 4; ++q) tc::tma_load_2d(buf + A_BYTES + q * 8192, &tm_x, &full[st], (int)j0 + 64 * q, tk);
        ++issued;
      }
      for (int j = issued > S ? issued - S : 0; j < issued; ++j) tc::mbar_wait(&full[j % S], (j / S) & 1, check);
    }
  } else if (warp == MMA_WARP) {
    if (lane == 0) {
      bool ok = true;
      for (int i = 0; i < nsteps; ++i) {
        const int st = i % S;
        if (*abort_flag || !tc::mbar_wait(&full[st], (i / S) & 1, check)) { *abort_flag = 1; ok = false; break; }
        tc::tc_fence_after();
        const uint32_t ab = tc::smem_u32(smem + st * STAGE), bb = ab + A_BYTES;
#pragma unroll
        for (int kk = 0; kk < KS / 16; ++kk) {
          const uint64_t ad = tc::sdesc(ab + kk * 2048, 8192, 1024, tc::kSwizzle128);
          const uint64_t bd = tc::sdesc(bb + kk * 2048, 8192, 1024, tc::kSwizzle128);
          tc::mma_ss(tmem, ad, bd, IDESC, (i > 0 || kk > 0) ? 1u : 0u);
        }
        tc::mma_commit(&empty[st]);
      }
      if (ok) tc::mma_commit(d_full);
    }
  } else {
    // epilogue warps 0-3: thread = row i (TMEM lane), 32 columns per load
    const int64_t i = i0 + threadIdx.x;
    bool have = !*abort_flag && tc::mbar_wait(d_full, 0, check) && nsteps > 0;
    have = __all_sync(0xffffffffu, have);   // tcgen05.ld is warp-collective
    if (have) tc::tc_fence_after();
#pragma unroll 1
    for (int q = 0; q < N / 32; ++q) {
      const int64_t jc = j0 + 32 * q;
      if (jc >= d) break;
      uint32_t v[32];
      if (have) {
        tc::tmem_ld32(tc::tmem_addr(tmem, warp * 32, 32 * q), v);
        tc::tmem_ld_wait();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0u;
      }
      if (i < d && (have || nsteps == 0)) {
        const int cnt = (int)(d - jc < 32 ? d - jc : 32);
        // the upper part of the row (j >= i) and the mirrors of j > i
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int64_t j = jc + e;
          if (e < cnt && j >= i) {
            const float val = __uint_as_float(v[e]);
            float* up = H + i * d + j;
            *up = (accumulate ? *up : 0.f) + val;
            if (j > i) {
              float* lo = H + j * d + i;
              *lo = (accumulate ? *lo : 0.f) + val;
            }
          }
        }
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ============================================================================
// 2. float64 linear algebra: damping, blocked Cholesky, triangular inverse
// ============================================================================

constexpr int NB = 64;   // block size of the factorizations (two of them form a super-block)

// lambda = damp * mean(diag H), a zero diagonal entry counted as 1; one CTA,
// fixed summation order
__global__ void damp_kernel(const float* __restrict__ H, int64_t d, double damp, double* __restrict__ lam) {
  __shared__ double part[1024];
  double acc = 0.0;
  for (int64_t j = threadIdx.x; j < d; j += blockDim.x) {
    const double h = (double)H[j * d + j];
    acc += h == 0.0 ? 1.0 : h;
  }
  part[threadIdx.x] = acc;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if ((int)threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) *lam = damp * (part[0] / (double)d);
}

// A[r][c] = H[d-1-r][d-1-c] for r >= c (the upper triangle of H, index-
// reversed, damped on the diagonal); zero above the diagonal
__global__ void reverse_damp_kernel(const float* __restrict__ H, int64_t d, const double* __restrict__ lam,
                                    double* __restrict__ A) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= d * d) return;
  const int64_t r = e / d, c = e - r * d;
  double v = 0.0;
  if (r >= c) {
    v = (double)H[(d - 1 - r) * d + (d - 1 - c)];
    if (r == c) v = (v == 0.0 ? 1.0 : v) + *lam;
  }
  A[e] = v;
}

// Unblocked Cholesky of the diagonal block A[k0:k0+kb][k0:k0+kb] (lower) in
// shared memory; a pivot that is not positive flags the check word (the
// factor then holds NaNs)
__global__ void __launch_bounds__(1024) potrf_diag_kernel(double* __restrict__ A, int64_t d, int64_t k0, int kb,
                                                         unsigned int* check) {
  __shared__ double a[NB][NB + 1];
  __shared__ double diag[NB];
  for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) {
    const int r = e / NB, c = e % NB;
    a[r][c] = (r < kb && c <= r) ? A[(k0 + r) * d + k0 + c] : 0.0;
  }
  __syncthreads();
  for (int c = 0; c < kb; ++c) {
    // every thread derives the pivot from a[c][c], which nothing writes during
    // this step (the factor's diagonal goes to diag[] and back at the end);
    // the column below is scaled by the pivot's reciprocal
    const double p = a[c][c];
    const double piv = sqrt(p), rp = 1.0 / piv;
    if (threadIdx.x == 0) {
      if (!(p > 0.0)) atomicOr(check, SK_CHECK_NOT_SPD);
      diag[c] = piv;
    }
    for (int r = c + 1 + (int)threadIdx.x; r < kb; r += blockDim.x) a[r][c] *= rp;
    __syncthreads();
    for (int r = c + 1 + (int)(threadIdx.x >> 5); r < kb; r += 32)
      for (int q = c + 1 + (int)(threadIdx.x & 31); q <= r; q += 32) a[r][q] -= a[r][c] * a[q][c];
    __syncthreads();
  }
  for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) {
    const int r = e / NB, c = e % NB;
    if (r < kb && c <= r) A[(k0 + r) * d + k0 + c] = r == c ? diag[r] : a[r][c];
  }
}

// Panel below a factored diagonal block: row r of A[k0+NB:, k0:k0+NB] becomes
// x with x L_kk^T = a (forward substitution), one thread per row
__global__ void __launch_bounds__(64) trsm_panel_kernel(double* __restrict__ A, int64_t d, int64_t k0) {
  __shared__ double l[NB][NB + 1];
  __shared__ double rdiag[NB];
  for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) {
    const int r = e / NB, c = e % NB;
    l[r][c] = c <= r ? A[(k0 + r) * d + k0 + c] : 0.0;
  }
  for (int c = threadIdx.x; c < NB; c += blockDim.x) rdiag[c] = 1.0 / A[(k0 + c) * d + k0 + c];
  __syncthreads();
  const int64_t r = k0 + NB + (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= d) return;
  double* row = A + r * d + k0;
  double x[NB];
#pragma unroll
  for (int c = 0; c < NB; ++c) x[c] = row[c];
  // right-looking: once x_c is final it is removed from every later entry,
  // so each step's updates are independent and only one multiply per column
  // sits on the critical path
#pragma unroll
  for (int c = 0; c < NB; ++c) {
    x[c] *= rdiag[c];
#pragma unroll
    for (int q = c + 1; q < NB; ++q) x[q] = fma(-x[c], l[q][c], x[q]);
  }
#pragma unroll
  for (int c = 0; c < NB; ++c) row[c] = x[c];
}

// C[m][n] -= A[m][K] * B, with B(k, c) = B[c][k] (BT) or B[k][c], K a multiple
// of 16 (64 or 128: the rank of one blocked update).  128 x 128
// output tiles, 8 x 8 per thread (rows ty*4 + {0..3} and 64 + ty*4 + {0..3},
// likewise the columns), K in chunks of 16 staged k-major in shared memory:
// per k a thread loads 8 + 8 doubles for 64 FMAs, which keeps the float64
// FMA pipe, not shared memory, the limit.  LOWER skips the tiles above the
// diagonal.
constexpr int GT = 128, GK = 16, GP = GT + 2;   // tile, K chunk, padded row of a staged chunk

template <bool BT, bool LOWER>
__global__ void __launch_bounds__(256, 1) gemm_sub_f64_kernel(const double* __restrict__ Ap, int64_t lda,
                                                              const double* __restrict__ Bp, int64_t ldb,
                                                              double* __restrict__ C, int64_t ldc, int64_t m,
                                                              int64_t n, int K, int vec_a, int vec_b) {
  if (LOWER && blockIdx.x > blockIdx.y) return;
  // two buffers of [A: GK][GP] + [B: GK][GP]; the next K chunk is loaded into
  // registers while the current one is multiplied, then stored to the other
  // buffer, so global latency hides behind the FMAs (one barrier per chunk)
  extern __shared__ __align__(16) double gsm[];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int64_t r0 = (int64_t)blockIdx.y * GT, c0 = (int64_t)blockIdx.x * GT;
  double acc[8][8];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b) acc[a][b] = 0.0;
  double2 pa[4], pb[4];
  // staging: a k-major operand ([row][k] in memory) is read as 16-byte k pairs,
  // eight threads per row; a row-major one ([k][col]) as 16-byte column pairs
  auto fetch = [&](int k0) {
#pragma unroll
    for (int rep = 0; rep < 4; ++rep) {
      const int e = rep * 256 + tid, rr = e >> 3, kp = (e & 7) * 2;
      const int64_t r = r0 + rr;
      pa[rep] = make_double2(0.0, 0.0);
      if (r < m) {
        const double* src = Ap + r * lda + k0 + kp;
        pa[rep] = vec_a ? *reinterpret_cast<const double2*>(src) : make_double2(src[0], src[1]);
      }
    }
#pragma unroll
    for (int rep = 0; rep < 4; ++rep) {
      const int e = rep * 256 + tid;
      if (BT) {
        const int cc = e >> 3, kp = (e & 7) * 2;
        const int64_t c = c0 + cc;
        pb[rep] = make_double2(0.0, 0.0);
        if (c < n) {
          const double* src = Bp + c * ldb + k0 + kp;
          pb[rep] = vec_b ? *reinterpret_cast<const double2*>(src) : make_double2(src[0], src[1]);
        }
      } else {
        const int kk = e >> 6, cp = (e & 63) * 2;
        const int64_t c = c0 + cp;
        const double* src = Bp + (int64_t)(k0 + kk) * ldb + c;
        pb[rep].x = c < n ? src[0] : 0.0;
        pb[rep].y = c + 1 < n ? src[1] : 0.0;
      }
    }
  };
  auto stash = [&](int buf) {
    double* As = gsm + buf * 2 * GK * GP;   // [k][row]
    double* Bs = As + GK * GP;              // [k][col]
#pragma unroll
    for (int rep = 0; rep < 4; ++rep) {
      const int e = rep * 256 + tid, rr = e >> 3, kp = (e & 7) * 2;
      As[kp * GP + rr] = pa[rep].x;
      As[(kp + 1) * GP + rr] = pa[rep].y;
    }
#pragma unroll
    for (int rep = 0; rep < 4; ++rep) {
      const int e = rep * 256 + tid;
      if (BT) {
        const int cc = e >> 3, kp = (e & 7) * 2;
        Bs[kp * GP + cc] = pb[rep].x;
        Bs[(kp + 1) * GP + cc] = pb[rep].y;
      } else {
        const int kk = e >> 6, cp = (e & 63) * 2;
        *reinterpret_cast<double2*>(&Bs[kk * GP + cp]) = pb[rep];
      }
    }
  };
  fetch(0);
  stash(0);
  __syncthreads();
  int buf = 0;
  for (int k0 = 0; k0 < K; k0 += GK) {
    const bool more = k0 + GK < K;
    if (more) fetch(k0 + GK);
    const double* As = gsm + buf * 2 * GK * GP;
    const double* Bs = As + GK * GP;
#pragma unroll
    for (int kk = 0; kk < GK; ++kk) {
      double av[8], bv[8];
      const double2 a0 = *reinterpret_cast<const double2*>(&As[kk * GP + ty * 4]);
      const double2 a1 = *reinterpret_cast<const double2*>(&As[kk * GP + ty * 4 + 2]);
      const double2 a2 = *reinterpret_cast<const double2*>(&As[kk * GP + 64 + ty * 4]);
      const double2 a3 = *reinterpret_cast<const double2*>(&As[kk * GP + 64 + ty * 4 + 2]);
      const double2 b0 = *reinterpret_cast<const double2*>(&Bs[kk * GP + tx * 4]);
      const double2 b1 = *reinterpret_cast<const double2*>(&Bs[kk * GP + tx * 4 + 2]);
      const double2 b2 = *reinterpret_cast<const double2*>(&Bs[kk * GP + 64 + tx * 4]);
      const double2 b3 = *reinterpret_cast<const double2*>(&Bs[kk * GP + 64 + tx * 4 + 2]);
      av[0] = a0.x; av[1] = a0.y; av[2] = a1.x; av[3] = a1.y; av[4] = a2.x; av[5] = a2.y; av[6] = a3.x; av[7] = a3.y;
      bv[0] = b0.x; bv[1] = b0.y; bv[2] = b1.x; bv[3] = b1.y; bv[4] = b2.x; bv[5] = b2.y; bv[6] = b3.x; bv[7] = b3.y;
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = fma(av[a], bv[b], acc[a][b]);
    }
    if (more) stash(buf ^ 1);
    __syncthreads();
    buf ^= 1;
  }
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const int64_t r = r0 + (a < 4 ? ty * 4 + a : 64 + ty * 4 + a - 4);
    if (r >= m) continue;
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      const int64_t c = c0 + (b < 4 ? tx * 4 + b : 64 + tx * 4 + b - 4);
      if (c < n) C[r * ldc + c] -= acc[a][b];
    }
  }
}

constexpr int kGemmSmem = 2 * 2 * GK * GP * (int)sizeof(double);

__global__ void identity_kernel(double* __restrict__ Mx, int64_t d) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e < d * d) Mx[e] = (e / d == e % d) ? 1.0 : 0.0;
}

// Block row r0 of the inverse of the lower factor L: Mx[r0:r0+kb][c] =
// L_rr^-1 Mx[r0:r0+kb][c] (forward substitution), one thread per column
template <bool FULL>
__global__ void __launch_bounds__(64) trtri_rows_kernel(const double* __restrict__ L, double* __restrict__ Mx,
                                                        int64_t d, int64_t r0, int kb) {
  if (FULL) kb = NB;
  __shared__ double l[NB][NB + 1];
  __shared__ double rdiag[NB];
  for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) {
    const int r = e / NB, c = e % NB;
    l[r][c] = (r < kb && c <= r) ? L[(r0 + r) * d + r0 + c] : (r == c ? 1.0 : 0.0);
  }
  __syncthreads();
  for (int r = threadIdx.x; r < NB; r += blockDim.x) rdiag[r] = 1.0 / l[r][r];
  __syncthreads();
  const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= r0 + kb) return;
  double x[NB];
  const double* src = Mx + r0 * d + c;
#pragma unroll
  for (int r = 0; r < NB; ++r) {
    x[r] = r < kb ? *src : 0.0;
    src += d;
  }
  // right-looking, as in the panel solve
#pragma unroll
  for (int r = 0; r < NB; ++r) {
    x[r] *= rdiag[r];
#pragma unroll
    for (int q = r + 1; q < NB; ++q) x[q] = fma(-l[q][r], x[r], x[q]);
  }
  double* dst = Mx + r0 * d + c;
#pragma unroll
  for (int r = 0; r < NB; ++r) {
    if (r < kb) *dst = x[r];
    dst += d;
  }
}

// U[j][k] = Mx[d-1-j][d-1-k]: element e swaps with element d*d - 1 - e
__global__ void reverse_kernel(double* __restrict__ Mx, int64_t d) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t f = d * d - 1 - e;
  if (e < f) {
    const double t = Mx[e];
    Mx[e] = Mx[f];
    Mx[f] = t;
  }
}

// diag(H^-1)[j] = sum_{k <= j} U[k][j]^2: a CTA takes 32 columns, its eight
// row phases sum rows k = phase mod 8 in order, then the phases are added in
// order (deterministic)
__global__ void __launch_bounds__(256) colnorm_kernel(const double* __restrict__ U, int64_t d,
                                                      double* __restrict__ out) {
  __shared__ double part[8][33];
  const int tx = threadIdx.x & 31, ph = threadIdx.x >> 5;
  const int64_t j = (int64_t)blockIdx.x * 32 + tx;
  double s = 0.0;
  if (j < d)
    for (int64_t k = ph; k <= j; k += 8) {
      const double u = U[k * d + j];
      s = fma(u, u, s);
    }
  part[ph][tx] = s;
  __syncthreads();
  if (ph == 0 && j < d) {
    double t = 0.0;
#pragma unroll
    for (int q = 0; q < 8; ++q) t += part[q][tx];
    out[j] = t;
  }
}

// ============================================================================
// 3. weighted Lloyd's algorithm, one CTA per (row, group)
// ============================================================================

constexpr int kLloydThreads = 512;     // 16 warps: one per cluster

__device__ __forceinline__ float midpoint(float a, float b) { return __fmul_rn(__fadd_rn(a, b), 0.5f); }

// number of the n sorted keys that are <= m
__device__ __forceinline__ int upper_bound(const float* key, int n, float m) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (key[mid] <= m) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

// Shared memory: w (float64, the weight of each sorted value), key (float32,
// sorted values), col (uint16, the value's column in the group): 14 bytes per
// slot of the power-of-two sort length p2.
__global__ void __launch_bounds__(kLloydThreads, 1)
lloyd_kernel(const float* __restrict__ theta, const double* __restrict__ hinv, int64_t d, int64_t gs, int gpr, int k,
             int p2, int max_iter, uint16_t* __restrict__ lut, int32_t* __restrict__ iters_out) {
  extern __shared__ __align__(16) uint8_t lsm[];
  double* w = reinterpret_cast<double*>(lsm);
  float* key = reinterpret_cast<float*>(w + p2);
  uint16_t* col = reinterpret_cast<uint16_t*>(key + p2);
  __shared__ float cent[16];
  __shared__ int bnd[16];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t row = blockIdx.x / gpr;
  const int g = (int)(blockIdx.x % gpr);
  const int n = (int)gs;
  const float* src = theta + row * d + (int64_t)g * gs;
  for (int t = tid; t < p2; t += blockDim.x) {
    key[t] = t < n ? src[t] : INFINITY;
    col[t] = (uint16_t)t;
  }
  __syncthreads();
  // bitonic sort of (value, column), ascending
  for (int size = 2; size <= p2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = tid; t < p2 / 2; t += blockDim.x) {
        const int lo = 2 * t - (t & (stride - 1)), hi = lo + stride;
        const float a = key[lo], b = key[hi];
        const uint16_t ca = col[lo], cb = col[hi];
        const bool greater = a > b || (a == b && ca > cb);
        if (greater == ((lo & size) == 0)) {
          key[lo] = b; key[hi] = a;
          col[lo] = cb; col[hi] = ca;
        }
      }
      __syncthreads();
    }
  }
  // weights 1 / [H^-1]_jj of the sorted values
  // (a padding slot sorts below a finite value only if theta holds NaN; it weighs nothing)
  for (int t = tid; t < n; t += blockDim.x) {
    const int cj = col[t];
    w[t] = cj < n ? __ddiv_rn(1.0, hinv[(int64_t)g * gs + cj]) : 0.0;
  }
  // start: k centroids evenly spaced over [min, max]
  if (tid < k) {
    const double mn = (double)key[0], mx = (double)key[n - 1];
    cent[tid] = __double2float_rn(
        __dadd_rn(mn, __ddiv_rn(__dmul_rn(__dsub_rn(mx, mn), (double)(2 * tid + 1)), (double)(2 * k))));
  }
  __syncthreads();
  // a cluster is a range of the sorted values: cluster c holds [bnd[c-1], bnd[c])
  if (tid < k - 1) bnd[tid] = upper_bound(key, n, midpoint(cent[tid], cent[tid + 1]));
  __syncthreads();
  int it = 0;
  while (it < max_iter) {
    if (warp < k) {
      const int b0 = warp == 0 ? 0 : bnd[warp - 1], b1 = warp == k - 1 ? n : bnd[warp];
      double s1 = 0.0, s0 = 0.0;
      for (int t = b0 + lane; t < b1; t += 32) {
        s1 = __dadd_rn(s1, __dmul_rn(w[t], (double)key[t]));
        s0 = __dadd_rn(s0, w[t]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        s1 = __dadd_rn(s1, __shfl_xor_sync(0xffffffffu, s1, o));
        s0 = __dadd_rn(s0, __shfl_xor_sync(0xffffffffu, s0, o));
      }
      if (lane == 0 && b1 > b0) cent[warp] = __double2float_rn(__ddiv_rn(s1, s0));   // empty: keep
    }
    __syncthreads();
    ++it;
    int nb = 0, moved = 0;
    if (tid < k - 1) {
      nb = upper_bound(key, n, midpoint(cent[tid], cent[tid + 1]));
      moved = nb != bnd[tid];
    }
    __syncthreads();
    if (tid < k - 1) bnd[tid] = nb;
    if (!__syncthreads_or(moved)) break;
  }
  if (tid < k) {
    const __half h = __float2half_rn(cent[tid]);
    lut[((int64_t)row * gpr + g) * k + tid] = __half_as_ushort(h);
  }
  if (tid == 0 && iters_out != nullptr) iters_out[(int64_t)row * gpr + g] = it;
}

// ============================================================================
// 4. column-by-column mapping with error compensation
// ============================================================================

constexpr int kRoundWarps = 32;   // rows per CTA, one warp each
constexpr int RB = 128;           // columns per mapping block (the rank of its lazy update)
constexpr int RQ = RB / 32;       // columns per lane

__global__ void round_init_kernel(const float* __restrict__ theta, int64_t count, double* __restrict__ W) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < count; e += (int64_t)gridDim.x * blockDim.x)
    W[e] = (double)theta[e];
}

// Columns [j0, j0 + kb) of every row, in order: the nearest fp16 centroid of
// the current value (float32 midpoints, ties to the lower centroid), the
// error e = (w_j - q_j) / U_jj, and w_c -= e U_jc for the block's later
// columns c.  A lane holds columns j0 + 32 q + lane (q < 4) of its row; the
// block of U sits in shared memory ([RB][RB] doubles, dynamic).  The errors
// go to E [n][RB] for the GEMM that updates the later blocks.
__global__ void __launch_bounds__(kRoundWarps * 32)
round_block_kernel(double* __restrict__ W, const double* __restrict__ U, const uint16_t* __restrict__ lut, int64_t n,
                   int64_t d, int64_t gs, int gpr, int k, int64_t j0, int kb, double* __restrict__ E,
                   uint8_t* __restrict__ idx, unsigned int* check) {
  extern __shared__ __align__(16) double ub[];   // U[j0 + a][j0 + b] at a * RB + b
  for (int e = threadIdx.x; e < RB * RB; e += blockDim.x) {
    const int a = e / RB, b = e % RB;
    ub[e] = (a < kb && b < kb) ? U[(j0 + a) * d + j0 + b] : 0.0;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t i = (int64_t)blockIdx.x * kRoundWarps + warp;
  if (i >= n) return;
  double* wrow = W + i * d + j0;
  double w[RQ], e_own[RQ];
  int c_own[RQ];
#pragma unroll
  for (int q = 0; q < RQ; ++q) {
    w[q] = 32 * q + lane < kb ? wrow[32 * q + lane] : 0.0;
    e_own[q] = 0.0;
    c_own[q] = 0;
  }
  int cur_g = -1;
  float cent = 0.f, mid = 0.f;
  for (int jj = 0; jj < kb; ++jj) {
    const int g = (int)((j0 + jj) / gs);
    if (g != cur_g) {
      cur_g = g;
      const uint16_t* row_lut = lut + (i * gpr + g) * k;
      cent = lane < k ? __half2float(__ushort_as_half(row_lut[lane])) : 0.f;
      const float next = __shfl_down_sync(0xffffffffu, cent, 1);
      mid = midpoint(cent, next);
      if (lane < k - 1 && next < cent) atomicOr(check, SK_CHECK_LUT_ORDER);
    }
    const int qj = jj >> 5;
    double mine = w[0];
#pragma unroll
    for (int q = 1; q < RQ; ++q)
      if (q == qj) mine = w[q];
    const double th = __shfl_sync(0xffffffffu, mine, jj & 31);
    const int c = __popc(__ballot_sync(0xffffffffu, lane < k - 1 && th > (double)mid));
    const double qv = (double)__shfl_sync(0xffffffffu, cent, c);
    const double e = __ddiv_rn(__dsub_rn(th, qv), ub[jj * RB + jj]);
    const double* urow = ub + jj * RB;
#pragma unroll
    for (int q = 0; q < RQ; ++q) {
      const int col = 32 * q + lane;
      if (col > jj && col < kb) w[q] = __dsub_rn(w[q], __dmul_rn(e, urow[col]));
    }
    if (lane == (jj & 31)) {
#pragma unroll
      for (int q = 0; q < RQ; ++q)
        if (q == qj) { e_own[q] = e; c_own[q] = c; }
    }
  }
  double* erow = E + i * RB;
#pragma unroll
  for (int q = 0; q < RQ; ++q) {
    const int col = 32 * q + lane;
    erow[col] = col < kb ? e_own[q] : 0.0;
    if (col < kb) idx[i * d + j0 + col] = (uint8_t)c_own[q];
  }
}

}  // namespace

// ============================================================================
// host launchers
// ============================================================================

cudaError_t launch_gram(const uint16_t* X, int64_t s, int64_t d, float* H, int accumulate, unsigned int* check,
                        cudaStream_t st) {
  CUtensorMap tm;
  cudaError_t e = make_tmap_2d(&tm, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)d, (uint64_t)s, (uint64_t)d * 2,
                               64, gr::KS, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(gram_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, gr::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)cdiv(d, gr::N), (unsigned)cdiv(d, gr::M));
  gram_tc_kernel<<<grid, gr::THREADS, gr::SMEM, st>>>(tm, s, d, H, accumulate, check);
  return cudaGetLastError();
}

// the GEMM's double-buffered staging needs more than the default 48 KB of
// dynamic shared memory
cudaError_t gemm_smem_setup() {
  cudaError_t e = cudaFuncSetAttribute(gemm_sub_f64_kernel<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kGemmSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gemm_sub_f64_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gemm_sub_f64_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem);
  return e;
}

// 16-byte loads of a k-major operand need an even leading dimension and an
// aligned base
int vec16(const double* p, int64_t ld) { return (ld % 2 == 0 && (reinterpret_cast<uintptr_t>(p) & 15u) == 0) ? 1 : 0; }

size_t inverse_factor_workspace(int64_t d) { return (size_t)d * (size_t)d * sizeof(double) + 256; }

cudaError_t launch_inverse_factor(const float* H, int64_t d, double damp, double* U, double* hinv_diag,
                                  void* workspace, unsigned int* check, cudaStream_t st) {
  double* A = static_cast<double*>(workspace);             // the reversed, damped H, then its lower factor
  double* lam = A + d * d;
  const int64_t dd = d * d;
  const unsigned eg = (unsigned)((dd + 255) / 256);
  cudaError_t e = gemm_smem_setup();
  if (e != cudaSuccess) return e;
  damp_kernel<<<1, 1024, 0, st>>>(H, d, damp, lam);
  reverse_damp_kernel<<<eg, 256, 0, st>>>(H, d, lam, A);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // blocked Cholesky (lower) of A in super-blocks of two 64-column blocks:
  // inside a super-block the first block's panel updates only the second
  // block's columns; the rest of the trailing matrix takes one rank-128 update
  for (int64_t k0 = 0; k0 < d; k0 += 2 * NB) {
    for (int h = 0; h < 2; ++h) {
      const int64_t kk = k0 + h * NB;
      if (kk >= d) break;
      const int kb = (int)(d - kk < NB ? d - kk : NB);
      potrf_diag_kernel<<<1, 1024, 0, st>>>(A, d, kk, kb, check);
      const int64_t rest = d - kk - kb;
      if (rest > 0) trsm_panel_kernel<<<(unsigned)cdiv(rest, 64), 64, 0, st>>>(A, d, kk);
      if (h == 0 && rest > 0) {
        const int64_t n2 = rest < NB ? rest : NB;      // columns of the second block
        const double* panel = A + (kk + NB) * d + kk;
        dim3 grid((unsigned)cdiv(n2, GT), (unsigned)cdiv(rest, GT));
        gemm_sub_f64_kernel<true, false><<<grid, 256, kGemmSmem, st>>>(panel, d, panel, d, A + (kk + NB) * d + kk + NB, d,
                                                               rest, n2, NB, vec16(panel, d), vec16(panel, d));
      }
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
    const int64_t kw = d - k0 < 2 * NB ? d - k0 : 2 * NB;
    const int64_t rest = d - k0 - kw;
    if (rest > 0) {
      const double* panel = A + (k0 + kw) * d + k0;
      dim3 grid((unsigned)cdiv(rest, GT), (unsigned)cdiv(rest, GT));
      gemm_sub_f64_kernel<true, true><<<grid, 256, kGemmSmem, st>>>(panel, d, panel, d, A + (k0 + kw) * d + k0 + kw, d, rest,
                                                            rest, (int)kw, vec16(panel, d), vec16(panel, d));
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // U buffer: inverse of the lower factor by blocked forward substitution,
  // in the same super-blocks
  identity_kernel<<<eg, 256, 0, st>>>(U, d);
  for (int64_t r0 = 0; r0 < d; r0 += 2 * NB) {
    for (int h = 0; h < 2; ++h) {
      const int64_t rr = r0 + h * NB;
      if (rr >= d) break;
      const int kb = (int)(d - rr < NB ? d - rr : NB);
      if (kb == NB) trtri_rows_kernel<true><<<(unsigned)cdiv(rr + kb, 64), 64, 0, st>>>(A, U, d, rr, kb);
      else trtri_rows_kernel<false><<<(unsigned)cdiv(rr + kb, 64), 64, 0, st>>>(A, U, d, rr, kb);
      const int64_t rows2 = d - rr - kb < NB ? d - rr - kb : NB;   // rows of the second block
      if (h == 0 && rows2 > 0) {
        const double* Ab = A + (rr + NB) * d + rr;
        dim3 grid((unsigned)cdiv(rr + kb, GT), (unsigned)cdiv(rows2, GT));
        gemm_sub_f64_kernel<false, false><<<grid, 256, kGemmSmem, st>>>(Ab, d, U + rr * d, d, U + (rr + NB) * d, d, rows2,
                                                                rr + kb, NB, vec16(Ab, d), 0);
      }
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
    const int64_t kw = d - r0 < 2 * NB ? d - r0 : 2 * NB;
    const int64_t rest = d - r0 - kw;
    if (rest > 0) {
      const double* Ab = A + (r0 + kw) * d + r0;
      dim3 grid((unsigned)cdiv(r0 + kw, GT), (unsigned)cdiv(rest, GT));
      gemm_sub_f64_kernel<false, false><<<grid, 256, kGemmSmem, st>>>(Ab, d, U + r0 * d, d, U + (r0 + kw) * d, d, rest,
                                                              r0 + kw, (int)kw, vec16(Ab, d), 0);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  reverse_kernel<<<(unsigned)((dd / 2 + 255) / 256 > 0 ? (dd / 2 + 255) / 256 : 1), 256, 0, st>>>(U, d);
  colnorm_kernel<<<(unsigned)cdiv(d, 32), 256, 0, st>>>(U, d, hinv_diag);
  return cudaGetLastError();
}

cudaError_t launch_lloyd(const float* theta, const double* hinv_diag, int bits, int gpr, int64_t n, int64_t d,
                         int max_iter, uint16_t* lut, int32_t* iters, cudaStream_t st) {
  const int64_t gs = d / gpr;
  int p2 = 32;
  while (p2 < gs) p2 <<= 1;
  const size_t smem = (size_t)p2 * (sizeof(double) + sizeof(float) + sizeof(uint16_t));
  cudaError_t e = cudaFuncSetAttribute(lloyd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  lloyd_kernel<<<(unsigned)(n * gpr), kLloydThreads, smem, st>>>(theta, hinv_diag, d, gs, gpr, 1 << bits, p2, max_iter,
                                                                lut, iters);
  return cudaGetLastError();
}

size_t sketch_round_workspace(int64_t n, int64_t d) {
  return (((size_t)n * (size_t)d + 1) / 2 * 2 + (size_t)n * RB) * sizeof(double) + 256;
}

cudaError_t launch_sketch_round(const float* theta, const double* U, const uint16_t* lut, int bits, int gpr, int64_t n,
                                int64_t d, uint8_t* idx, void* workspace, unsigned int* check, cudaStream_t st) {
  double* W = static_cast<double*>(workspace);   // [n][d] values being mapped
  double* E = W + (n * d + 1) / 2 * 2;           // [n][RB] errors of the current block (16-byte aligned)
  const int64_t gs = d / gpr;
  const int k = 1 << bits;
  round_init_kernel<<<(unsigned)(num_sms() * 8), 256, 0, st>>>(theta, n * d, W);
  cudaError_t e = cudaFuncSetAttribute(round_block_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       RB * RB * (int)sizeof(double));
  if (e == cudaSuccess) e = gemm_smem_setup();
  if (e != cudaSuccess) return e;
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const unsigned rgrid = (unsigned)cdiv(n, kRoundWarps);
  for (int64_t j0 = 0; j0 < d; j0 += RB) {
    const int kb = (int)(d - j0 < RB ? d - j0 : RB);
    round_block_kernel<<<rgrid, kRoundWarps * 32, RB * RB * sizeof(double), st>>>(W, U, lut, n, d, gs, gpr, k, j0, kb,
                                                                                  E, idx, check);
    const int64_t rest = d - j0 - kb;
    if (rest > 0) {
      dim3 grid((unsigned)cdiv(rest, GT), (unsigned)cdiv(n, GT));
      gemm_sub_f64_kernel<false, false><<<grid, 256, kGemmSmem, st>>>(E, RB, U + j0 * d + j0 + RB, d, W + j0 + RB, d, n, rest,
                                                              RB, vec16(E, RB), 0);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace sk
