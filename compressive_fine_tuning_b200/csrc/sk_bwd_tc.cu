// Backward of the sketched linear layer on the 5th-generation tensor cores.
//
// Input gradient (chain rule through the frozen sketch):
//   dX[t][j] = sum_i dY[t][i] * Theta_hat[i][j]
// computed as the transposed tile dX^T[128 columns j x 256 tokens]:
//   * operand A = Theta_hat^T (M = j, K = i) lives in shared memory in the
//     MN-major 128-byte-swizzled layout; eight producer warps dequantise it,
//     each thread owning one weight row i of the step (so the row's LUT is a
//     register table) and one 32-column chunk, writing 16-byte swizzled stores;
//   * operand B = dY (N = t, K = i) arrives by TMA (K-major, 128B swizzle);
//   * one thread issues tcgen05.mma, the fp32 accumulator lives in TMEM, and
//     the epilogue writes bf16 dX.
//
// LUT gradient (the corrected Eq. 6 of the "Sketch to Adapt" OpenReview
// discussion, reply Q1): dlut[i][g][c] = sum_{j in g, idx[i][j] = c} (dY^T X)[i][j].
//   * G tile [128 rows i x 256 columns j] = dY^T X over K = tokens, both
//     operands MN-major straight from TMA;
//   * the epilogue never writes G: each thread takes its row's accumulator
//     32 columns at a time (tcgen05.ld), looks the indices up and adds every
//     value into the (group, centroid) bin it selects.  Bins live in shared
//     memory as [k][thread] (the dynamic bin index never causes a bank
//     conflict); on a group change the thread writes its k sums as one
//     partial for (column tile, row, group slot);
//   * a second small kernel adds the partials of every group over the column
//     tiles in a fixed order, so the result is deterministic, and writes or
//     accumulates dlut.
#include "sk_tc.cuh"

namespace sk {
namespace {

constexpr int kThreads = 320;
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;

__host__ __device__ constexpr int ceil_div(int64_t a, int64_t b) { return (int)((a + b - 1) / b); }

// ============================================================================
// dX
// ============================================================================

namespace dx {
constexpr int N = 256;          // tokens per tile
constexpr int KS = 64;          // weight rows (K) per pipeline step
// two stages, so that two CTAs share an SM (the dequantising warps of one
// overlap the other's MMAs and epilogue): measured 21 % faster than one CTA
// with four stages on the 7B gate_proj at 8192 tokens
constexpr int S = 2;
constexpr int B_BYTES = N * 128;             // dY tile: N rows x 64 bf16
constexpr int A_BYTES = 2 * 8 * 1024;        // two 64-column MN atoms x 8 K-groups
constexpr int STAGE = B_BYTES + A_BYTES;
constexpr int BAR_OFF = S * STAGE;
constexpr int SMEM = 1024 + BAR_OFF + 256;
constexpr uint32_t IDESC = tc::idesc_bf16(128, N, /*a MN-major*/ 1, /*b K-major*/ 0);
constexpr int TMEM_COLS = 256;
}  // namespace dx

// dX on CTA pairs (cta_group::2): the two CTAs of a cluster own 128 columns
// each of a 256-column block and share one 256-token tile.  Each dequantises
// its own columns' A tile into its own shared memory and loads only half of
// the dY tile (128 tokens); the even CTA issues M = 256, N = 256 MMAs.  Half
// the dY bytes per CTA and step let three stages fit beside two CTAs per SM.
namespace dxp {
constexpr int N = 256;                       // tokens per pair tile
constexpr int KS = dx::KS;
constexpr int S = 3;
constexpr int B_BYTES = (N / 2) * 128;       // this CTA's 128 dY rows x 64 bf16
constexpr int A_BYTES = dx::A_BYTES;
constexpr int STAGE = B_BYTES + A_BYTES;
constexpr int BAR_OFF = S * STAGE;
constexpr int SMEM = 1024 + BAR_OFF + 256;
constexpr uint32_t IDESC = tc::idesc_bf16(256, N, /*a MN-major*/ 1, /*b K-major*/ 0);
constexpr int TMEM_COLS = 256;
static_assert(N * 128 * 2 <= BAR_OFF, "the epilogue stages the output tile in the stage memory");
}  // namespace dxp

struct DxArgs {
  const uint8_t* packed;
  int64_t row_bytes;
  const uint16_t* lut;
  int64_t n, d, gs, T;
  int gpr;
  uint16_t* dX;
  unsigned int* check;
  // task-routed batches: dY rows are in task order, tile y covers positions
  // [tiles[3y + 1], + tiles[3y + 2]) of task tiles[3y] and perm maps a
  // position back to its token; nullptr for single-LUT-set batches
  const int* tiles;
  const int* perm;
  int64_t lut_task_stride;
  // 1: the epilogue writes whole token rows of dX from shared memory with bulk
  // copies (16-byte aligned dX); 0: each thread stores its own column
  int y_bulk;
};

// The dequantising producers of dX (both dX kernels): warp w (of 8) fills
// K-group w (8 rows) of every step's 128-column x 64-row A tile (MN-major,
// 128-byte swizzle); lane = (chunk h, row r8).  wait_slot(i) waits until step
// i's A slot may be overwritten, slot(i) is its shared-memory base and
// ready(i) tells the MMA issuer that it is written.
template <int BITS, class WaitSlot, class Slot, class Ready>
__device__ __forceinline__ void dx_produce_a(const DxArgs& a, const uint16_t* lut, int64_t j0, int nsteps, int warp,
                                             int lane, volatile int* abort_flag, WaitSlot wait_slot, Slot slot,
                                             Ready ready) {
  using dx::KS;
  const int r8 = lane & 7, h = lane >> 3;
  const int lr = 8 * warp + r8;                    // row within the step
  const int64_t j = j0 + 32 * h;                   // first column of this thread's chunk
  const bool col_ok = j < a.d;
  const int64_t cchunk = j >> 5;
  const int64_t g = col_ok ? j / a.gs : 0;
  const int m_atom = h >> 1;
  // swizzled 16-byte slots of this thread's four chunks within the K-row
  uint32_t slot_off[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) slot_off[q] = m_atom * 8192 + warp * 1024 + r8 * 128 + (((4 * (h & 1) + q) ^ r8) << 4);
  // software pipeline: this step's index chunk and raw LUT entries are loaded one step ahead
  Chunk<BITS> ch_next{};
  uint4 lraw_next[2] = {};
  auto fetch = [&](int i) {
    const int64_t row = (int64_t)i * KS + lr;
    if (col_ok && row < a.n) {
      ch_next = load_chunk<BITS>(a.packed + row * a.row_bytes, cchunk);
      const uint16_t* lp = lut + (row * a.gpr + g) * (1 << BITS);
      if constexpr (BITS == 4) {
        lraw_next[0] = __ldg(reinterpret_cast<const uint4*>(lp));
        lraw_next[1] = __ldg(reinterpret_cast<const uint4*>(lp) + 1);
      } else if constexpr (BITS == 3) {
        lraw_next[0] = __ldg(reinterpret_cast<const uint4*>(lp));
      } else {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(lp));
        lraw_next[0] = make_uint4(v.x, v.y, 0u, 0u);
      }
    }
  };
  fetch(0);
  for (int i = 0; i < nsteps; ++i) {
    const Chunk<BITS> ch = ch_next;
    const uint4 l0 = lraw_next[0], l1 = lraw_next[1];
    const bool ok = col_ok && (int64_t)i * KS + lr < a.n;
    if (i + 1 < nsteps) fetch(i + 1);
    uint32_t o[16];
    if (ok) {
      LutRegs<BITS> L;
      if constexpr (BITS == 4) {
        uint32_t w[8] = {h2_to_bf2(l0.x), h2_to_bf2(l0.y), h2_to_bf2(l0.z), h2_to_bf2(l0.w),
                         h2_to_bf2(l1.x), h2_to_bf2(l1.y), h2_to_bf2(l1.z), h2_to_bf2(l1.w)};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          L.lo[q] = prmt(w[2 * q], w[2 * q + 1], 0x6420);
          L.hi[q] = prmt(w[2 * q], w[2 * q + 1], 0x7531);
        }
      } else if constexpr (BITS == 3) {
        uint32_t w[4] = {h2_to_bf2(l0.x), h2_to_bf2(l0.y), h2_to_bf2(l0.z), h2_to_bf2(l0.w)};
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          L.lo[q] = prmt(w[2 * q], w[2 * q + 1], 0x6420);
          L.hi[q] = prmt(w[2 * q], w[2 * q + 1], 0x7531);
        }
      } else {
        const uint32_t w0 = h2_to_bf2(l0.x), w1 = h2_to_bf2(l0.y);
        L.lo[0] = prmt(w0, w1, 0x6420);
        L.hi[0] = prmt(w0, w1, 0x7531);
      }
      dequant_chunk<BITS>(ch, L, o);
    } else {
#pragma unroll
      for (int e = 0; e < 16; ++e) o[e] = 0u;
    }
    if (*abort_flag || !wait_slot(i)) { *abort_flag = 1; break; }
    uint8_t* at = slot(i);
#pragma unroll
    for (int q = 0; q < 4; ++q)
      *reinterpret_cast<uint4*>(at + slot_off[q]) = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
    tc::fence_async_smem();
    __syncwarp();
    if (lane == 0) ready(i);
  }
}

template <int BITS>
__global__ void __launch_bounds__(kThreads, 2)
dx_tc_kernel(const __grid_constant__ CUtensorMap tm_dy, DxArgs a) {
  using namespace dx;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_b = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* full_a = full_b + S;
  uint64_t* empty = full_a + S;
  uint64_t* d_full = empty + S;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(d_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = tc::warp_id(), lane = tc::lane_id();
  const int64_t j0 = (int64_t)blockIdx.x * 128;
  int t0 = blockIdx.y * N;            // first dY row of the tile
  int64_t tlen = a.T - t0;            // tokens of the tile (bounded by N below)
  const uint16_t* lut = a.lut;
  if (a.tiles != nullptr) {
    const int tau = a.tiles[3 * blockIdx.y];
    t0 = a.tiles[3 * blockIdx.y + 1];
    tlen = a.tiles[3 * blockIdx.y + 2];
    if (tlen == 0) return;            // an unused tile: the whole CTA leaves before any setup
    lut += (int64_t)tau * a.lut_task_stride;
  }
  if (tlen > N) tlen = N;
  // output row of tile token t (positions map back to tokens when routed)
  auto out_row = [&](int t) -> int64_t { return a.tiles != nullptr ? (int64_t)a.perm[t0 + t] : (int64_t)(t0 + t); };
  const int nsteps = ceil_div(a.n, KS);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      tc::mbar_init(&full_b[s], 1);
      tc::mbar_init(&full_a[s], 8);
      tc::mbar_init(&empty[s], 1);
    }
    tc::mbar_init(d_full, 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == kMmaWarp) tc::tmem_alloc(tmem_slot, TMEM_COLS);
  if (warp == kTmaWarp && lane == 0) tc::tma_prefetch(&tm_dy);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kTmaWarp) {
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nsteps && !*abort_flag; ++i) {
        const int s = i % S;
        if (!tc::mbar_wait(&empty[s], ((i / S) & 1) ^ 1, a.check)) { *abort_flag = 1; break; }
        tc::mbar_arrive_expect_tx(&full_b[s], B_BYTES);
        tc::tma_load_2d(smem + s * STAGE, &tm_dy, &full_b[s], i * KS, t0);
        ++issued;
      }
      for (int j = issued > S ? issued - S : 0; j < issued; ++j) tc::mbar_wait(&full_b[j % S], (j / S) & 1, a.check);
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      bool ok = true;
      for (int i = 0; i < nsteps; ++i) {
        const int s = i % S;
        if (*abort_flag || !tc::mbar_wait(&full_b[s], (i / S) & 1, a.check) ||
            !tc::mbar_wait(&full_a[s], (i / S) & 1, a.check)) {
          *abort_flag = 1; ok = false; break;
        }
        tc::tc_fence_after();
        const uint32_t bb = tc::smem_u32(smem + s * STAGE);
        const uint32_t ab = bb + B_BYTES;
#pragma unroll
        for (int kk = 0; kk < KS / 16; ++kk) {
          const uint64_t ad = tc::sdesc(ab + kk * 2048, 8192, 1024, tc::kSwizzle128);
          const uint64_t bd = tc::sdesc(bb + kk * 32, 16, 1024, tc::kSwizzle128);
          tc::mma_ss(tmem, ad, bd, IDESC, (i > 0 || kk > 0) ? 1u : 0u);
        }
        tc::mma_commit(&empty[s]);
      }
      if (ok) tc::mma_commit(d_full);
    }
  } else {
    // producers: dequantise Θ̂ᵀ into this step's A slot
    dx_produce_a<BITS>(a, lut, j0, nsteps, warp, lane, abort_flag,
                       [&](int i) { return tc::mbar_wait(&empty[i % S], ((i / S) & 1) ^ 1, a.check); },
                       [&](int i) { return smem + (i % S) * STAGE + B_BYTES; },
                       [&](int i) { tc::mbar_arrive(&full_a[i % S]); });
  }

  // epilogue: thread = column j (TMEM lane), warps w and w + 4 split the tokens
  __syncthreads();
  if (warp < 8) {
    const int quad = warp & 3;
    const int64_t j = j0 + quad * 32 + lane;
    bool have = !*abort_flag && tc::mbar_wait(d_full, 0, a.check);
    have = __all_sync(0xffffffffu, have);  // tcgen05.ld is warp-collective
    if (have) tc::tc_fence_after();
    if (a.y_bulk) {
      // the stage memory is free: every MMA has completed (d_full)
      tc::store_tile_bulk<N, 8>(reinterpret_cast<uint16_t*>(smem), tmem, have, warp, lane, j0, a.d, t0, (int)tlen,
                                a.tiles != nullptr ? a.perm : nullptr, a.dX);
    } else if (have) {
      for (int gi = (warp >> 2); gi < N / 16; gi += 2) {
        uint32_t v[16];
        tc::tmem_ld16(tc::tmem_addr(tmem, quad * 32, gi * 16), v);
        tc::tmem_ld_wait();
        if (j < a.d) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int t = gi * 16 + e;
            if (t < tlen) {
              __nv_bfloat16 b = __float2bfloat16_rn(__uint_as_float(v[e]));
              a.dX[out_row(t) * a.d + j] = *reinterpret_cast<uint16_t*>(&b);
            }
          }
        }
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <int BITS>
__global__ void __launch_bounds__(kThreads, 2)
dx_tc_pair_kernel(const __grid_constant__ CUtensorMap tm_dy, DxArgs a) {
  using namespace dxp;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_b = reinterpret_cast<uint64_t*>(smem + BAR_OFF);  // even CTA: both dY halves landed
  uint64_t* full_a = full_b + S;                                    // even CTA: both A tiles written
  uint64_t* empty = full_a + S;                                     // both CTAs: the pair MMAs read the stage
  uint64_t* d_full = empty + S;                                     // both CTAs: accumulator final
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(d_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = tc::warp_id(), lane = tc::lane_id();
  const uint32_t rank = tc::cluster_ctarank();                      // 0: issues the MMAs
  const int64_t j0 = (int64_t)(blockIdx.x >> 1) * 256 + 128 * rank;
  int t0 = blockIdx.y * N;
  int64_t tlen = a.T - t0;
  const uint16_t* lut = a.lut;
  if (a.tiles != nullptr) {
    const int tau = a.tiles[3 * blockIdx.y];
    t0 = a.tiles[3 * blockIdx.y + 1];
    tlen = a.tiles[3 * blockIdx.y + 2];
    if (tlen == 0) return;            // both CTAs of the pair read the same entry and leave together
    lut += (int64_t)tau * a.lut_task_stride;
  }
  if (tlen > N) tlen = N;
  auto out_row = [&](int t) -> int64_t { return a.tiles != nullptr ? (int64_t)a.perm[t0 + t] : (int64_t)(t0 + t); };
  const int nsteps = ceil_div(a.n, KS);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      tc::mbar_init(&full_b[s], 1);
      tc::mbar_init(&full_a[s], 16);
      tc::mbar_init(&empty[s], 1);
    }
    tc::mbar_init(d_full, 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == kMmaWarp) tc::tmem_alloc_pair(tmem_slot, TMEM_COLS);
  if (warp == kTmaWarp && lane == 0) tc::tma_prefetch(&tm_dy);
  tc::tc_fence_before();
  // both CTAs' barriers are initialised before either CTA signals the other
  tc::cluster_sync_all();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kTmaWarp) {
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nsteps && !*abort_flag; ++i) {
        const int s = i % S;
        if (!tc::mbar_wait(&empty[s], ((i / S) & 1) ^ 1, a.check)) { *abort_flag = 1; break; }
        // the even CTA's full_b counts the dY bytes of both CTAs
        if (rank == 0) tc::mbar_arrive_expect_tx(&full_b[s], 2 * B_BYTES);
        tc::tma_load_2d_pair(smem + s * STAGE, &tm_dy, tc::mapa(&full_b[s], 0), i * KS, t0 + 128 * (int)rank);
        ++issued;
      }
      // never leave with a copy still landing in shared memory: the pair MMAs
      // read every landed half before they free its stage
      bool ok = true;
      for (int k = issued > S ? issued - S : 0; k < issued && ok; ++k)
        ok = tc::mbar_wait(&empty[k % S], (k / S) & 1, a.check);
    }
  } else if (warp == kMmaWarp) {
    if (rank == 0 && lane == 0) {
      bool ok = true;
      for (int i = 0; i < nsteps; ++i) {
        const int s = i % S;
        if (*abort_flag || !tc::mbar_wait(&full_b[s], (i / S) & 1, a.check) ||
            !tc::mbar_wait(&full_a[s], (i / S) & 1, a.check)) {
          *abort_flag = 1; ok = false; break;
        }
        tc::tc_fence_after();
        const uint32_t bb = tc::smem_u32(smem + s * STAGE);
        const uint32_t ab = bb + B_BYTES;
#pragma unroll
        for (int kk = 0; kk < KS / 16; ++kk) {
          const uint64_t ad = tc::sdesc(ab + kk * 2048, 8192, 1024, tc::kSwizzle128);
          const uint64_t bd = tc::sdesc(bb + kk * 32, 16, 1024, tc::kSwizzle128);
          tc::mma_ss_pair(tmem, ad, bd, IDESC, (i > 0 || kk > 0) ? 1u : 0u);
        }
        tc::mma_commit_pair(&empty[s]);
      }
      if (ok) tc::mma_commit_pair(d_full);
    }
  } else {
    // producers: dequantise this CTA's 128 columns of Θ̂ᵀ; the even CTA's full_a counts both CTAs' warps
    const uint32_t full_a_even = tc::mapa(&full_a[0], 0);
    dx_produce_a<BITS>(a, lut, j0, nsteps, warp, lane, abort_flag,
                       [&](int i) { return tc::mbar_wait(&empty[i % S], ((i / S) & 1) ^ 1, a.check); },
                       [&](int i) { return smem + (i % S) * STAGE + B_BYTES; },
                       [&](int i) { tc::mbar_arrive_cluster(full_a_even + 8 * (i % S)); });
  }

  // epilogue: each CTA writes its own 128 columns of dX for the pair's tokens
  __syncthreads();
  if (warp < 8) {
    const int quad = warp & 3;
    const int64_t j = j0 + quad * 32 + lane;
    bool have = !*abort_flag && tc::mbar_wait(d_full, 0, a.check);
    have = __all_sync(0xffffffffu, have);  // tcgen05.ld is warp-collective
    if (have) tc::tc_fence_after();
    if (a.y_bulk) {
      tc::store_tile_bulk<N, 8>(reinterpret_cast<uint16_t*>(smem), tmem, have, warp, lane, j0, a.d, t0, (int)tlen,
                                a.tiles != nullptr ? a.perm : nullptr, a.dX);
    } else if (have) {
      for (int gi = (warp >> 2); gi < N / 16; gi += 2) {
        uint32_t v[16];
        tc::tmem_ld16(tc::tmem_addr(tmem, quad * 32, gi * 16), v);
        tc::tmem_ld_wait();
        if (j < a.d) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int t = gi * 16 + e;
            if (t < tlen) {
              __nv_bfloat16 bv = __float2bfloat16_rn(__uint_as_float(v[e]));
              a.dX[out_row(t) * a.d + j] = *reinterpret_cast<uint16_t*>(&bv);
            }
          }
        }
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  // neither CTA leaves (or frees tensor memory) while the other may still
  // signal its barriers or the pair MMAs may still use its memory
  tc::cluster_sync_all();
  if (warp == kMmaWarp) {
    tc::tc_fence_after();
    tc::tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

// ============================================================================
// dlut
// ============================================================================

namespace dl {
constexpr int M = 128, N = 256;
constexpr int KS = 64;          // tokens per pipeline step
constexpr int A_BYTES = 2 * 8192;   // dY^T: two 64-row MN atoms x 8 K-groups
constexpr int B_BYTES = 4 * 8192;   // X: four 64-column MN atoms x 8 K-groups
constexpr int STAGE = A_BYTES + B_BYTES;
// two stages, so that two CTAs share an SM: while one bins its finished tile
// in the epilogue, the other's MMAs keep the tensor pipe busy (measured: 12 %
// faster than one CTA with four stages at 8192 tokens, 30 % per LUT set of a
// routed batch)
constexpr int S = 2;
constexpr int BAR_OFF = S * STAGE;
constexpr int SMEM = 1024 + BAR_OFF + 256;
constexpr int THREADS = 192;        // warps 0-3 epilogue, 4 TMA, 5 MMA
constexpr int TMA_WARP = 4, MMA_WARP = 5;
constexpr uint32_t IDESC = tc::idesc_bf16(M, N, 1, 1);
constexpr int TMEM_COLS = 256;
}  // namespace dl

// The LUT gradient on CTA pairs (cta_group::2): the two CTAs of a cluster own
// 128 rows each of a 256-row block and share one 256-column tile; each loads
// its own dY rows and half of the X tile (128 columns), the even CTA issues
// M = 256, N = 256 MMAs, and each CTA bins its own rows' accumulator as
// above.  Half the X bytes per CTA and step let three stages fit beside two
// CTAs per SM.
namespace dlp {
constexpr int N = 256;
constexpr int KS = dl::KS;
constexpr int A_BYTES = dl::A_BYTES;        // this CTA's 128 rows of dY^T
constexpr int B_BYTES = 2 * 8192;           // this CTA's 128 columns of X
constexpr int STAGE = A_BYTES + B_BYTES;
constexpr int S = 3;
constexpr int BAR_OFF = S * STAGE;
constexpr int SMEM = 1024 + BAR_OFF + 256;
constexpr uint32_t IDESC = tc::idesc_bf16(256, N, 1, 1);
constexpr int TMEM_COLS = 256;
}  // namespace dlp

// Group slots of one 256-column tile: groups [tile*256 / gs, (tile*256 + 255) / gs].
__host__ __device__ inline int dlut_slots(int64_t gs, int gpr) {
  const int64_t s = 255 / gs + 2;
  return (int)(s < gpr ? s : gpr);
}

struct DlutArgs {
  const uint8_t* packed;
  int64_t row_bytes;
  int64_t n, d, gs, T;
  int gpr, slots;
  float* part;          // [jtiles][n][slots][k] partial bins (per LUT set when routed)
  unsigned int* check;
  // several LUT sets: X and dY rows in task order, task z's tokens at
  // positions [segs[2z], segs[2z] + segs[2z + 1]) (64-aligned, zero-padded);
  // nullptr for one LUT set
  const int* segs;
  int64_t part_task_stride;  // floats between the partial bins of consecutive LUT sets
  int row_pairs;             // CTA-pair kernel: 256-row blocks per LUT set
};

template <int BITS>
__global__ void __launch_bounds__(dl::THREADS, 2)
dlut_tc_kernel(const __grid_constant__ CUtensorMap tm_dy, const __grid_constant__ CUtensorMap tm_x, DlutArgs a) {
  using namespace dl;
  constexpr int K = 1 << BITS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* empty = full + S;
  uint64_t* d_full = empty + S;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(d_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = tc::warp_id(), lane = tc::lane_id();
  const int jt = blockIdx.x;
  const int64_t j0 = (int64_t)jt * N;
  const int64_t i0 = (int64_t)blockIdx.y * M;
  int k_first = 0;                    // first token position of this LUT set
  int nsteps = ceil_div(a.T, KS);
  float* part = a.part;
  if (a.segs != nullptr) {
    k_first = a.segs[2 * blockIdx.z];
    nsteps = ceil_div(a.segs[2 * blockIdx.z + 1], KS);   // a set with no tokens writes zero partials
    part += (int64_t)blockIdx.z * a.part_task_stride;
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    tc::mbar_init(d_full, 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == MMA_WARP) tc::tmem_alloc(tmem_slot, TMEM_COLS);
  if (warp == TMA_WARP && lane == 0) {
    tc::tma_prefetch(&tm_dy);
    tc::tma_prefetch(&tm_x);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == TMA_WARP) {
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nsteps && !*abort_flag; ++i) {
        const int s = i % S;
        if (!tc::mbar_wait(&empty[s], ((i / S) & 1) ^ 1, a.check)) { *abort_flag = 1; break; }
        uint8_t* st = smem + s * STAGE;
        tc::mbar_arrive_expect_tx(&full[s], STAGE);
        const int tk = k_first + i * KS;
        tc::tma_load_2d(st, &tm_dy, &full[s], (int)i0, tk);
        tc::tma_load_2d(st + 8192, &tm_dy, &full[s], (int)i0 + 64, tk);
#pragma unroll
        for (int q = 0; q < 4; ++q) tc::tma_load_2d(st + A_BYTES + q * 8192, &tm_x, &full[s], (int)j0 + 64 * q, tk);
        ++issued;
      }
      for (int j = issued > S ? issued - S : 0; j < issued; ++j) tc::mbar_wait(&full[j % S], (j / S) & 1, a.check);
    }
  } else if (warp == MMA_WARP) {
    if (lane == 0) {
      bool ok = true;
      for (int i = 0; i < nsteps; ++i) {
        const int s = i % S;
        if (*abort_flag || !tc::mbar_wait(&full[s], (i / S) & 1, a.check)) { *abort_flag = 1; ok = false; break; }
        tc::tc_fence_after();
        const uint32_t ab = tc::smem_u32(smem + s * STAGE), bb = ab + A_BYTES;
#pragma unroll
        for (int kk = 0; kk < KS / 16; ++kk) {
          const uint64_t ad = tc::sdesc(ab + kk * 2048, 8192, 1024, tc::kSwizzle128);
          const uint64_t bd = tc::sdesc(bb + kk * 2048, 8192, 1024, tc::kSwizzle128);
          tc::mma_ss(tmem, ad, bd, IDESC, (i > 0 || kk > 0) ? 1u : 0u);
        }
        tc::mma_commit(&empty[s]);
      }
      if (ok) tc::mma_commit(d_full);
    }
  } else {
    // epilogue warps 0-3: thread = row i (TMEM lane); bin the row's 256 columns
    float* bins = reinterpret_cast<float*>(smem + BAR_OFF - K * 128 * 4);  // [K][128], tail of stage memory
    const int tid = threadIdx.x;                                         // 0..127
    const int64_t i = i0 + tid;
    // the row's index chunks of this column tile, loaded while the MMAs run so
    // their memory latency is off the binning loop
    Chunk<BITS> chunks[N / 32];
#pragma unroll
    for (int q = 0; q < N / 32; ++q) {
      const int64_t jc = j0 + 32 * q;
      if (i < a.n && jc < a.d) chunks[q] = load_chunk<BITS>(a.packed + i * a.row_bytes, jc >> 5);
    }
    bool have = !*abort_flag && tc::mbar_wait(d_full, 0, a.check) && nsteps > 0;   // no steps: nothing accumulated
    have = __all_sync(0xffffffffu, have);  // tcgen05.ld is warp-collective
    if (have) tc::tc_fence_after();
    // the bins reuse the last stage's memory: wait until every MMA has read it (d_full)
#pragma unroll
    for (int c = 0; c < K; ++c) bins[c * 128 + tid] = 0.f;
    const int first_g = (int)(j0 / a.gs);
    const int gs32 = (int)a.gs;
    int g = first_g, g_end = (first_g + 1) * gs32;
    bool dirty = false;
    auto flush = [&](int gg) {
      if (i < a.n) {
        float* dst = part + (((int64_t)jt * a.n + i) * a.slots + (gg - first_g)) * K;
#pragma unroll
        for (int c = 0; c < K; ++c) dst[c] = bins[c * 128 + tid];
      }
#pragma unroll
      for (int c = 0; c < K; ++c) bins[c * 128 + tid] = 0.f;
    };
#pragma unroll
    for (int q = 0; q < N / 32; ++q) {
      const int64_t jc = j0 + 32 * q;
      if (jc >= a.d) break;
      uint32_t v[32];
      if (have) {
        tc::tmem_ld32(tc::tmem_addr(tmem, warp * 32, 32 * q), v);
        tc::tmem_ld_wait();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0u;
      }
      if ((int)jc >= g_end) {       // chunk in a later group: hand the finished group's sums on
        if (dirty) flush(g);
        do { ++g; g_end += gs32; } while ((int)jc >= g_end);
        dirty = false;
      }
      if (i < a.n) {
#pragma unroll
        for (int e = 0; e < 32; ++e) bins[chunk_index<BITS>(chunks[q], e) * 128 + tid] += __uint_as_float(v[e]);
      }
      dirty = true;
    }
    if (dirty) flush(g);
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <int BITS>
__global__ void __launch_bounds__(dl::THREADS, 2)
dlut_tc_pair_kernel(const __grid_constant__ CUtensorMap tm_dy, const __grid_constant__ CUtensorMap tm_x, DlutArgs a) {
  using namespace dlp;
  constexpr int K = 1 << BITS, TMA_WARP = dl::TMA_WARP, MMA_WARP = dl::MMA_WARP;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + BAR_OFF);   // even CTA: both CTAs' operands landed
  uint64_t* empty = full + S;                                      // both CTAs: the pair MMAs read the stage
  uint64_t* d_full = empty + S;                                    // both CTAs: accumulator final
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(d_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = tc::warp_id(), lane = tc::lane_id();
  const uint32_t rank = tc::cluster_ctarank();                     // 0: issues the MMAs
  // grid: (pair, column tile, row block + row_pairs * LUT set), column tiles
  // fastest after the pair, so the clusters in flight cover all column tiles
  // of a few row blocks
  const int jt = blockIdx.y;
  const int64_t j0 = (int64_t)jt * N;
  const int set = (int)blockIdx.z / a.row_pairs;
  const int64_t i0 = (int64_t)((int)blockIdx.z - set * a.row_pairs) * 256 + 128 * rank;
  int k_first = 0;
  int nsteps = ceil_div(a.T, KS);
  float* part = a.part;
  if (a.segs != nullptr) {
    k_first = a.segs[2 * set];
    nsteps = ceil_div(a.segs[2 * set + 1], KS);   // a set with no tokens writes zero partials
    part += (int64_t)set * a.part_task_stride;
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    tc::mbar_init(d_full, 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == MMA_WARP) tc::tmem_alloc_pair(tmem_slot, TMEM_COLS);
  if (warp == TMA_WARP && lane == 0) {
    tc::tma_prefetch(&tm_dy);
    tc::tma_prefetch(&tm_x);
  }
  tc::tc_fence_before();
  // both CTAs' barriers are initialised before either CTA signals the other
  tc::cluster_sync_all();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == TMA_WARP) {
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nsteps && !*abort_flag; ++i) {
        const int s = i % S;
        if (!tc::mbar_wait(&empty[s], ((i / S) & 1) ^ 1, a.check)) { *abort_flag = 1; break; }
        uint8_t* st = smem + s * STAGE;
        // the even CTA's full counts the operand bytes of both CTAs
        if (rank == 0) tc::mbar_arrive_expect_tx(&full[s], 2 * STAGE);
        const uint32_t bar = tc::mapa(&full[s], 0);
        const int tk = k_first + i * KS;
        tc::tma_load_2d_pair(st, &tm_dy, bar, (int)i0, tk);
        tc::tma_load_2d_pair(st + 8192, &tm_dy, bar, (int)i0 + 64, tk);
        const int jx = (int)j0 + 128 * (int)rank;
        tc::tma_load_2d_pair(st + A_BYTES, &tm_x, bar, jx, tk);
        tc::tma_load_2d_pair(st + A_BYTES + 8192, &tm_x, bar, jx + 64, tk);
        ++issued;
      }
      // never leave with a copy still landing in shared memory: the pair MMAs
      // read every landed stage before they free it
      bool ok = true;
      for (int k = issued > S ? issued - S : 0; k < issued && ok; ++k)
        ok = tc::mbar_wait(&empty[k % S], (k / S) & 1, a.check);
    }
  } else if (warp == MMA_WARP) {
    if (rank == 0 && lane == 0) {
      bool ok = true;
      for (int i = 0; i < nsteps; ++i) {
        const int s = i % S;
        if (*abort_flag || !tc::mbar_wait(&full[s], (i / S) & 1, a.check)) { *abort_flag = 1; ok = false; break; }
        tc::tc_fence_after();
        const uint32_t ab = tc::smem_u32(smem + s * STAGE), bb = ab + A_BYTES;
#pragma unroll
        for (int kk = 0; kk < KS / 16; ++kk) {
          const uint64_t ad = tc::sdesc(ab + kk * 2048, 8192, 1024, tc::kSwizzle128);
          const uint64_t bd = tc::sdesc(bb + kk * 2048, 8192, 1024, tc::kSwizzle128);
          tc::mma_ss_pair(tmem, ad, bd, IDESC, (i > 0 || kk > 0) ? 1u : 0u);
        }
        tc::mma_commit_pair(&empty[s]);
      }
      if (ok) tc::mma_commit_pair(d_full);
    }
  } else {
    // epilogue warps 0-3: thread = row i (TMEM lane); bin the row's 256 columns
    float* bins = reinterpret_cast<float*>(smem + BAR_OFF - K * 128 * 4);  // [K][128], tail of stage memory
    const int tid = threadIdx.x;                                         // 0..127
    const int64_t i = i0 + tid;
    Chunk<BITS> chunks[N / 32];
#pragma unroll
    for (int q = 0; q < N / 32; ++q) {
      const int64_t jc = j0 + 32 * q;
      if (i < a.n && jc < a.d) chunks[q] = load_chunk<BITS>(a.packed + i * a.row_bytes, jc >> 5);
    }
    bool have = !*abort_flag && tc::mbar_wait(d_full, 0, a.check) && nsteps > 0;   // no steps: nothing accumulated
    have = __all_sync(0xffffffffu, have);  // tcgen05.ld is warp-collective
    if (have) tc::tc_fence_after();
    // the bins reuse the last stage's memory: every MMA has read it (d_full)
#pragma unroll
    for (int c = 0; c < K; ++c) bins[c * 128 + tid] = 0.f;
    const int first_g = (int)(j0 / a.gs);
    const int gs32 = (int)a.gs;
    int g = first_g, g_end = (first_g + 1) * gs32;
    bool dirty = false;
    auto flush = [&](int gg) {
      if (i < a.n) {
        float* dst = part + (((int64_t)jt * a.n + i) * a.slots + (gg - first_g)) * K;
#pragma unroll
        for (int c = 0; c < K; ++c) dst[c] = bins[c * 128 + tid];
      }
#pragma unroll
      for (int c = 0; c < K; ++c) bins[c * 128 + tid] = 0.f;
    };
#pragma unroll
    for (int q = 0; q < N / 32; ++q) {
      const int64_t jc = j0 + 32 * q;
      if (jc >= a.d) break;
      uint32_t v[32];
      if (have) {
        tc::tmem_ld32(tc::tmem_addr(tmem, warp * 32, 32 * q), v);
        tc::tmem_ld_wait();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0u;
      }
      if ((int)jc >= g_end) {
        if (dirty) flush(g);
        do { ++g; g_end += gs32; } while ((int)jc >= g_end);
        dirty = false;
      }
      if (i < a.n) {
#pragma unroll
        for (int e = 0; e < 32; ++e) bins[chunk_index<BITS>(chunks[q], e) * 128 + tid] += __uint_as_float(v[e]);
      }
      dirty = true;
    }
    if (dirty) flush(g);
  }

  tc::tc_fence_before();
  __syncthreads();
  // neither CTA leaves (or frees tensor memory) while the other may still
  // signal its barriers or the pair MMAs may still use its memory
  tc::cluster_sync_all();
  if (warp == MMA_WARP) {
    tc::tc_fence_after();
    tc::tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

// Sum the partial bins of every (row, group) over the column tiles that touch
// the group, in tile order, and write (or add to) dlut.
template <int BITS>
__global__ void dlut_reduce_kernel(const float* __restrict__ part, int64_t n, int gpr, int64_t gs, int jtiles,
                                   int slots, float* __restrict__ dlut, int accumulate, int ntask,
                                   int64_t part_task_stride) {
  constexpr int K = 1 << BITS;
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t per_set = n * gpr * K;
  if (e >= per_set * ntask) return;
  const int64_t tau = e / per_set;
  part += tau * part_task_stride;
  const int64_t es = e - tau * per_set;
  const int c = (int)(es % K);
  const int64_t ig = es / K;
  const int g = (int)(ig % gpr);
  const int64_t i = ig / gpr;
  const int t_first = (int)(((int64_t)g * gs) / dl::N);
  int t_last = (int)(((int64_t)(g + 1) * gs - 1) / dl::N);
  if (t_last > jtiles - 1) t_last = jtiles - 1;
  float sum = 0.f;
  for (int t = t_first; t <= t_last; ++t) {
    const int fg = (int)(((int64_t)t * dl::N) / gs);
    sum += part[(((int64_t)t * n + i) * slots + (g - fg)) * K + c];
  }
  dlut[e] = accumulate ? dlut[e] + sum : sum;
}

}  // namespace

size_t dlut_tc_workspace(int64_t n, int64_t d, int bits, int gpr) {
  const int64_t gs = d / gpr;
  const int64_t jtiles = (d + dl::N - 1) / dl::N;
  return (size_t)jtiles * n * dlut_slots(gs, gpr) * (1 << bits) * sizeof(float);
}

namespace {
cudaError_t dx_launch(const Problem& p, const uint16_t* dY, uint16_t* dX, const Routed* rt, cudaStream_t s) {
  CUtensorMap tm;
  cudaError_t e = make_tmap_2d(&tm, rt != nullptr ? rt->Xp : dY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)p.n,
                               (uint64_t)p.T, (uint64_t)p.n * 2, 64, dx::N, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  const int y_bulk = p.d % 8 == 0 && (reinterpret_cast<uintptr_t>(dX) & 15) == 0 && env_int("SK_TC_YBULK", 1) != 0;
  DxArgs args{p.packed, p.row_bytes, p.lut, p.n, p.d, p.gs, p.T, p.gpr, dX, p.check,
              rt != nullptr ? rt->tiles : nullptr, rt != nullptr ? rt->perm : nullptr,
              p.n * p.gpr * (1 << p.bits), y_bulk ? 1 : 0};
  const unsigned tiles = rt != nullptr ? (unsigned)rt->max_tiles : (unsigned)ceil_div(p.T, dx::N);
  if (env_int("SK_DX_PAIR", 1) != 0) {
    // CTA pairs over 256-column blocks (SK_DX_PAIR=0: one CTA per 128 columns)
    CUtensorMap tmp;
    e = make_tmap_2d(&tmp, rt != nullptr ? rt->Xp : dY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)p.n,
                     (uint64_t)p.T, (uint64_t)p.n * 2, 64, dxp::N / 2, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    auto run_pair = [&](auto kern) {
      cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, dxp::SMEM);
      if (err != cudaSuccess) return err;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2u * (unsigned)ceil_div(p.d, 256), tiles, 1u);
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = dxp::SMEM;
      cfg.stream = s;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      err = cudaLaunchKernelEx(&cfg, kern, tmp, args);
      if (err != cudaSuccess) return err;
      return cudaGetLastError();
    };
    switch (p.bits) {
      case 2: return run_pair(dx_tc_pair_kernel<2>);
      case 3: return run_pair(dx_tc_pair_kernel<3>);
      default: return run_pair(dx_tc_pair_kernel<4>);
    }
  }
  dim3 grid((unsigned)ceil_div(p.d, 128), tiles);
  auto run = [&](auto kern) {
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, dx::SMEM);
    if (err != cudaSuccess) return err;
    kern<<<grid, kThreads, dx::SMEM, s>>>(tm, args);
    return cudaGetLastError();
  };
  switch (p.bits) {
    case 2: return run(dx_tc_kernel<2>);
    case 3: return run(dx_tc_kernel<3>);
    default: return run(dx_tc_kernel<4>);
  }
}
}  // namespace

cudaError_t launch_dx_tc(const Problem& p, const uint16_t* dY, uint16_t* dX, cudaStream_t s) {
  return dx_launch(p, dY, dX, nullptr, s);
}

size_t dx_tc_workspace(int64_t T, int64_t n, int ntask) { return route_workspace_bytes(T, n, ntask, dx::N); }

cudaError_t launch_dx_tc_routed(const Problem& p, const uint16_t* dY, uint16_t* dX, void* workspace, cudaStream_t s) {
  Routed rt;
  cudaError_t e = launch_route(p, dY, p.n, dX, p.d, dx::N, workspace, &rt, s);
  if (e != cudaSuccess) return e;
  return dx_launch(p, dY, dX, &rt, s);
}

namespace {
// part: partial bins; rp: the padded task routing (nullptr for one LUT set)
cudaError_t dlut_launch(const Problem& p, const uint16_t* X, const uint16_t* dY, float* dlut, int accumulate,
                        float* part, const RoutedPad* rp, cudaStream_t s) {
  const uint64_t rows = rp != nullptr ? (uint64_t)rp->positions : (uint64_t)p.T;
  CUtensorMap tm_dy, tm_x;
  cudaError_t e = make_tmap_2d(&tm_dy, rp != nullptr ? rp->b : dY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)p.n,
                               rows, (uint64_t)p.n * 2, 64, dl::KS, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  e = make_tmap_2d(&tm_x, rp != nullptr ? rp->a : X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)p.d, rows,
                   (uint64_t)p.d * 2, 64, dl::KS, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  const int slots = dlut_slots(p.gs, p.gpr);
  const int jtiles = ceil_div(p.d, dl::N);
  const int sets = rp != nullptr ? p.ntask : 1;
  const int64_t stride = (int64_t)jtiles * p.n * slots * (1 << p.bits);
  DlutArgs args{p.packed, p.row_bytes, p.n, p.d, p.gs, p.T, p.gpr, slots, part, p.check,
                rp != nullptr ? rp->segs : nullptr, stride, ceil_div(p.n, 256)};
  const int64_t outs = (int64_t)sets * p.n * p.gpr * (1 << p.bits);
  const unsigned rgrid = (unsigned)((outs + 255) / 256);
  // 256-row blocks on CTA pairs unless SK_DLUT_PAIR=0
  const bool pair = env_int("SK_DLUT_PAIR", 1) != 0;
  auto run = [&](auto kern, auto kern_pair, auto red) {
    cudaError_t err;
    if (pair) {
      err = cudaFuncSetAttribute(kern_pair, cudaFuncAttributeMaxDynamicSharedMemorySize, dlp::SMEM);
      if (err != cudaSuccess) return err;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2u, (unsigned)jtiles, (unsigned)(ceil_div(p.n, 256) * sets));
      cfg.blockDim = dim3(dl::THREADS, 1, 1);
      cfg.dynamicSmemBytes = dlp::SMEM;
      cfg.stream = s;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      err = cudaLaunchKernelEx(&cfg, kern_pair, tm_dy, tm_x, args);
    } else {
      err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, dl::SMEM);
      if (err != cudaSuccess) return err;
      dim3 grid((unsigned)jtiles, (unsigned)ceil_div(p.n, dl::M), (unsigned)sets);
      kern<<<grid, dl::THREADS, dl::SMEM, s>>>(tm_dy, tm_x, args);
    }
    if (err != cudaSuccess) return err;
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    red<<<rgrid, 256, 0, s>>>(part, p.n, p.gpr, p.gs, jtiles, slots, dlut, accumulate, sets, stride);
    return cudaGetLastError();
  };
  switch (p.bits) {
    case 2: return run(dlut_tc_kernel<2>, dlut_tc_pair_kernel<2>, dlut_reduce_kernel<2>);
    case 3: return run(dlut_tc_kernel<3>, dlut_tc_pair_kernel<3>, dlut_reduce_kernel<3>);
    default: return run(dlut_tc_kernel<4>, dlut_tc_pair_kernel<4>, dlut_reduce_kernel<4>);
  }
}
}  // namespace

cudaError_t launch_dlut_tc(const Problem& p, const uint16_t* X, const uint16_t* dY, float* dlut, int accumulate,
                           void* workspace, cudaStream_t s) {
  return dlut_launch(p, X, dY, dlut, accumulate, static_cast<float*>(workspace), nullptr, s);
}

// workspace: the padded routing (positions, segments, X and dY in task order),
// then the partial bins of every LUT set
size_t dlut_tc_routed_workspace(int64_t n, int64_t d, int bits, int gpr, int64_t T, int ntask) {
  const size_t route = route_pad_workspace_bytes(T, d, n, ntask, dl::KS);
  return (route + 255) / 256 * 256 + (size_t)ntask * dlut_tc_workspace(n, d, bits, gpr);
}

cudaError_t launch_dlut_tc_routed(const Problem& p, const uint16_t* X, const uint16_t* dY, float* dlut, int accumulate,
                                  void* workspace, cudaStream_t s) {
  RoutedPad rp;
  cudaError_t e = launch_route_padded(p, X, p.d, dY, p.n, dl::KS, workspace, &rp, s);
  if (e != cudaSuccess) return e;
  const size_t route = route_pad_workspace_bytes(p.T, p.d, p.n, p.ntask, dl::KS);
  float* part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + (route + 255) / 256 * 256);
  return dlut_launch(p, X, dY, dlut, accumulate, part, &rp, s);
}

}  // namespace sk

// ============================================================================
// Allocation-free LUT gradient: the same kernels with a fixed scratch array
// ============================================================================
//
// Some callers cannot allocate device memory at the point where they need the
// LUT gradient: a plugin running inside another framework's executor that owns
// every device allocation, a serving or training loop that has reserved all of
// its memory up front and treats any new allocation as an error, or code that
// must not call cudaMalloc because it synchronises the device.  For them the
// partial bins live in one file-scope device array instead of a caller
// workspace.  The array belongs to this file's device module, so it is
// reserved on a device as soon as that module is loaded there -- on the first
// use of any kernel of this file (the tensor-core input and LUT gradients) or
// of the allocation-free call, or when the context is created if modules load
// eagerly -- and it is held until the process exits, whether or not the
// allocation-free call is ever made.
#include <mutex>

namespace sk {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 64;
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
std::mutex g_noalloc_mutex;
std::once_flag g_ctx_once;
CtxGetCurrentFn g_ctx_get_current = nullptr;
// per device: the context the address was looked up in, and the address
CUcontext g_noalloc_ctx[kNoAllocMaxDevices] = {};
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};

void load_ctx_get_current() {
  cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
  void* fn = nullptr;
  if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(fn);
}

}  // namespace

size_t dlut_noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

// Device address of the scratch array on the current device.  In host code the
// array's name only stands for the host-side shadow symbol, so the device
// address is looked up with the device current.  The lookup is cached per
// device together with the context it was made in: if that context has been
// torn down and replaced (a device reset), the module is loaded again at a
// possibly different address and the lookup is repeated.
cudaError_t dlut_noalloc_scratch(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return cudaErrorInvalidDevice;
  std::call_once(g_ctx_once, load_ctx_get_current);
  CUcontext ctx = nullptr;
  if (g_ctx_get_current == nullptr || g_ctx_get_current(&ctx) != CUDA_SUCCESS) ctx = nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_ptr[dev] == nullptr || ctx == nullptr || ctx != g_noalloc_ctx[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev] = p;
    g_noalloc_ctx[dev] = ctx;
  }
  *ptr = g_noalloc_ptr[dev];
  return cudaSuccess;
}

}  // namespace sk
