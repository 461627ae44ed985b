// Forward of the sketched linear layer on the 5th-generation tensor cores:
//   Y[t][i] = sum_j X[t][j] * Theta_hat[i][j]
// ("SpaLLM: Unified Compressive Adaptation of LLMs with Sketching", section
// 2.3: one compressed matmul per layer; Eq. 1 with groups per row gives
// Theta_hat).
//
// The MMA computes the transposed tile Y^T[128 rows x N tokens] =
// Theta_hat[128 x K] * X[N x K]^T with the dequantised weights as operand A in
// tensor memory and the activations as operand B in shared memory:
//   * TMA brings, per 128-column step, the packed index tile (128 rows) and
//     the X tile (N tokens, two 64-column swizzled boxes) into shared memory;
//   * eight dequantisation warps each own 32 weight rows (one per thread, the
//     thread's row is its TMEM lane) and half of the step's columns; a thread
//     looks its own row's indices up in register byte-plane LUTs and writes
//     the bf16 weights straight into tensor memory (tcgen05.st), so the
//     dequantised tile never touches shared memory;
//   * one thread issues tcgen05.mma (kind::f16, A from TMEM, B from SMEM,
//     fp32 accumulator in TMEM) and tcgen05.commit hands stages back;
//   * the epilogue reads the accumulator with tcgen05.ld (thread = row) and
//     writes bf16 Y.
// Decode batches (N <= 64) are split along K over a thread-block cluster; the
// partial accumulators are summed in a fixed order through distributed shared
// memory, so the result is deterministic and needs no workspace.
#include <cooperative_groups.h>

#include "sk_tc.cuh"

namespace cg = cooperative_groups;

namespace sk {
namespace {


__host__ __device__ constexpr int align1k(int x) { return (x + 1023) / 1024 * 1024; }
__host__ __device__ constexpr int pow2ceil(int x) { int p = 32; while (p < x) p *= 2; return p; }

template <int BITS, int N>
struct Cfg {
  // Decode tiles (N <= 64) carry little MMA work per weight element, so the
  // MMA -> commit -> barrier round trip (about 1.5k cycles) must be hidden by
  // running the dequantisation many steps ahead: one CTA per SM owns all 512
  // TMEM columns (7 A stages) and 16 dequantisation warps.  Prefill tiles are
  // MMA-bound and keep 8 warps, 2 A stages and their deeper shared-memory ring.
  static constexpr bool DECODE = N <= 64;
  static constexpr int KSTEP = DECODE ? 256 : 128;            // weight columns per pipeline step
  static constexpr int A_COLS = KSTEP / 2;                    // 32-bit TMEM columns per A stage (bf16 pairs)
  static constexpr int DQW = DECODE ? 16 : 8;                 // dequantisation warps
  static constexpr int TMA_WARP = DQW, MMA_WARP = DQW + 1;
  static constexpr int THREADS = (DQW + 2) * 32;
  static constexpr int CH = KSTEP / 32 / (DQW / 4);           // 32-column chunks per thread per step
  static constexpr int S = N >= 256 ? 3 : N >= 128 ? 5 : N >= 64 ? 4 : N >= 32 ? 5 : 6;  // shared-memory stages
  static constexpr int SA = DECODE ? 3 : 2;                   // tensor-memory stages of operand A
  static constexpr int XBOXES = KSTEP / 64;                   // 64-column X boxes per step
  static constexpr int KB = KSTEP * BITS / 8;                 // index bytes per row per step
  static constexpr int X_BOX = N * 128;                       // one 64-column box of X
  static constexpr int X_BYTES = XBOXES * X_BOX;
  static constexpr int IDX_OFF = align1k(X_BYTES);
  static constexpr int IDX_BYTES = 128 * KB;
  static constexpr int STAGE = IDX_OFF + align1k(IDX_BYTES);
  static constexpr int BAR_OFF = S * STAGE;
  static constexpr int SMEM = 1024 + BAR_OFF + 512;           // + alignment slack + barriers
  static constexpr int D_COL = SA * A_COLS;
  static constexpr int TMEM_COLS = 512;
  static constexpr uint32_t IDESC = tc::idesc_bf16(128, N, 0, 0);
  static_assert(N % 16 == 0 && N >= 16 && N <= 256, "UMMA N for M = 128");
  static_assert(N * (128 + 8) * 4 <= BAR_OFF, "split-K partials reuse the stage memory");
  static_assert(D_COL + N <= TMEM_COLS, "tensor memory budget");
  static_assert(SMEM <= 232448, "shared memory budget");
};

struct FwdArgs {
  const uint16_t* lut;
  int64_t n, d, gs, T;
  int gpr;
  int steps_total;  // ceil(d / C::KSTEP)
  uint16_t* Y;
  unsigned int* check;
  // task-routed batches: X rows are in task order, tile z covers positions
  // [tiles[3z + 1], + tiles[3z + 2]) of task tiles[3z] and perm maps a position
  // back to its token; nullptr for single-LUT-set batches
  const int* tiles;
  const int* perm;
  int64_t lut_task_stride;  // elements between consecutive LUT sets
  // grid order: 0 = (split, row block, token tile), token tiles slowest, so the
  // CTAs in flight share X columns and every token tile sweeps the index map
  // (kept in L2 when it is the smaller operand); 1 = (1, token tile, row block),
  // token tiles fastest, so the CTAs in flight share their row blocks' index
  // rows and X (the smaller operand) stays in L2
  int tiles_fast;
  // 1: the epilogue stages each tile in shared memory and writes every token
  // row of it with one bulk copy (needs 16-byte aligned rows of Y: n % 8 == 0,
  // which the API requires, and a 16-byte aligned Y); 0: each thread stores
  // its own row's outputs
  int y_bulk;
};

// The thread's CH consecutive 32-column chunks of the step, starting at chunk
// c0, read from the TMA-swizzled index tile whose rows are KB bytes (the TMA
// swizzle span equals KB when KB is 32, 64 or 128 bytes: the 16-byte piece p
// of row r sits at p ^ ((r * KB / 128) % (KB / 16))).
template <int BITS, int KB, int CH>
__device__ __forceinline__ void read_idx(const uint8_t* tile, int r, int c0, Chunk<BITS> (&ch)[CH]) {
#pragma unroll
  for (int c = 0; c < CH; ++c) {
    const int q = c0 + c;
    if constexpr (BITS == 4 || BITS == 2) {
      constexpr int PIECES = KB / 16;                       // 16-byte pieces per row
      const int sw = ((r * KB) >> 7) & (PIECES - 1);
      if constexpr (BITS == 4) {                            // one chunk per piece
        const uint4 v = *reinterpret_cast<const uint4*>(tile + r * KB + 16 * (q ^ sw));
        ch[c].w[0] = v.x; ch[c].w[1] = v.y; ch[c].w[2] = v.z; ch[c].w[3] = v.w;
      } else {                                              // two chunks per piece
        const uint2 v = *reinterpret_cast<const uint2*>(tile + r * KB + 16 * ((q >> 1) ^ sw) + 8 * (q & 1));
        ch[c].w[0] = v.x; ch[c].w[1] = v.y;
      }
    } else {                                                // 3-bit: unswizzled rows, 12 bytes per chunk
      const uint32_t* p = reinterpret_cast<const uint32_t*>(tile + r * KB + 12 * q);
      ch[c].w[0] = p[0]; ch[c].w[1] = p[1]; ch[c].w[2] = p[2];
    }
  }
}

template <int BITS, int N>
__global__ void __launch_bounds__(Cfg<BITS, N>::THREADS, 1)
fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_idx, FwdArgs a) {
  using C = Cfg<BITS, N>;
  constexpr int kDequantWarps = C::DQW, kTmaWarp = C::TMA_WARP, kMmaWarp = C::MMA_WARP, kThreads = C::THREADS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* empty = full + C::S;
  uint64_t* a_full = empty + C::S;
  // let the next launch in the stream start its prologue while this one runs
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  constexpr int SA = C::SA;
  uint64_t* a_empty = a_full + SA;
  uint64_t* d_full = a_empty + SA;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(d_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = tc::warp_id(), lane = tc::lane_id();
  const int ks = blockIdx.x, ksplit = gridDim.x;
  const int mb = a.tiles_fast ? blockIdx.z : blockIdx.y, tt = a.tiles_fast ? blockIdx.y : blockIdx.z;
  const int64_t m0 = (int64_t)mb * 128;
  int t0 = tt * N;               // first X row of the tile
  int tlen = N;                  // tokens of the tile (bounded by T below)
  const uint16_t* lut = a.lut;
  if (a.tiles != nullptr) {
    // the routing kernel wrote the tile list: wait for it before the setup
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int tau = a.tiles[3 * tt];
    t0 = a.tiles[3 * tt + 1];
    tlen = a.tiles[3 * tt + 2];
    if (tlen == 0) return;       // the whole cluster shares the tile and leaves together
    lut += (int64_t)tau * a.lut_task_stride;
  } else if (t0 + tlen > a.T) {
    tlen = (int)(a.T - t0);
  }
  // output row of tile token t (positions map back to tokens when routed)
  auto out_row = [&](int t) -> int64_t { return a.tiles != nullptr ? (int64_t)a.perm[t0 + t] : (int64_t)(t0 + t); };
  const int s0 = (int)((int64_t)ks * a.steps_total / ksplit);
  const int s1 = (int)((int64_t)(ks + 1) * a.steps_total / ksplit);
  const int nsteps = s1 - s0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::S; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], kDequantWarps + 1);
    }
    for (int i = 0; i < SA; ++i) {
      tc::mbar_init(&a_full[i], kDequantWarps);
      tc::mbar_init(&a_empty[i], 1);
    }
    tc::mbar_init(d_full, 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == kMmaWarp) tc::tmem_alloc(tmem_slot, C::TMEM_COLS);
  if (warp == kTmaWarp && lane == 0) {
    tc::tma_prefetch(&tm_x);
    tc::tma_prefetch(&tm_idx);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // inputs may come from the previous launch: wait for it before reading any
  if (a.tiles == nullptr) asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == kTmaWarp) {
    // ---------------- producer: TMA loads ----------------
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nsteps && !*abort_flag; ++i) {
        const int s = i % C::S;
        if (!tc::mbar_wait(&empty[s], ((i / C::S) & 1) ^ 1, a.check)) { *abort_flag = 1; break; }
        uint8_t* st = smem + s * C::STAGE;
        tc::mbar_arrive_expect_tx(&full[s], C::X_BYTES + C::IDX_BYTES);
        const int k0 = (s0 + i) * C::KSTEP;
#pragma unroll
        for (int b = 0; b < C::XBOXES; ++b) tc::tma_load_2d(st + b * C::X_BOX, &tm_x, &full[s], k0 + 64 * b, t0);
        tc::tma_load_2d(st + C::IDX_OFF, &tm_idx, &full[s], (s0 + i) * C::KB, (int)m0);
        ++issued;
      }
      // never leave with a copy still landing in shared memory
      for (int j = issued > C::S ? issued - C::S : 0; j < issued; ++j)
        tc::mbar_wait(&full[j % C::S], (j / C::S) & 1, a.check);
    }
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issue ----------------
    if (lane == 0) {
      bool ok = true;
      const uint64_t desc0 = tc::sdesc(tc::smem_u32(smem), 16, 1024, tc::kSwizzle128);
      for (int i = 0; i < nsteps; ++i) {
        const int s = i % C::S, ai = i % SA;
        if (*abort_flag || !tc::mbar_wait(&full[s], (i / C::S) & 1, a.check) ||
            !tc::mbar_wait(&a_full[ai], (i / SA) & 1, a.check)) {
          *abort_flag = 1; ok = false; break;
        }
        tc::tc_fence_after();
        // descriptor of this stage's X tile; the start-address field (bits 0..13,
        // 16-byte units) absorbs the per-MMA offsets without carrying out
        const uint64_t bd0 = desc0 + (uint64_t)((s * C::STAGE) >> 4);
        const uint32_t a0 = tmem + ai * C::A_COLS;
#pragma unroll
        for (int kk = 0; kk < C::KSTEP / 16; ++kk) {
          const uint64_t bd = bd0 + (uint64_t)(((kk >> 2) * C::X_BOX + (kk & 3) * 32) >> 4);
          tc::mma_ts(tmem + C::D_COL, a0 + kk * 8, bd, C::IDESC, (i > 0 || kk > 0) ? 1u : 0u);
        }
        tc::mma_commit(&empty[s]);
        tc::mma_commit(&a_empty[ai]);
      }
      if (ok) tc::mma_commit(d_full);
    }
  } else {
    // ---------------- dequantisation into tensor memory ----------------
    // warp w owns TMEM lanes 32 (w % 4) .. + 31 (its 32 rows) and chunks
    // [part * CH, part * CH + CH) of every 128-column step
    constexpr int CH = C::CH;
    const int quad = warp & 3, part = warp >> 2;
    const int r = quad * 32 + lane;
    const int64_t row = m0 + r;
    const bool row_ok = row < a.n;
    const uint16_t* lut_row = lut + (row_ok ? row : 0) * a.gpr * (1 << BITS);
    // group bookkeeping in 32-bit arithmetic, advanced incrementally (no divisions in the loop)
    const int d32 = (int)a.d, gs32 = (int)a.gs;
    int col = s0 * C::KSTEP + part * CH * 32;  // first column of this thread's chunks in the step
    int g = col / gs32;
    if (g >= a.gpr) g = a.gpr - 1;
    int g_end = (g + 1) * gs32;             // first column past group g
    // fetch the first group's table now, overlapping the first TMA round trip,
    // and always keep the next group's raw table in flight
    LutRegs<BITS> L;
    LutRaw<BITS> nxt;
    load_lut<BITS>(lut_row + g * (1 << BITS), L);
    fetch_lut<BITS>(lut_row + (g + 1 < a.gpr ? g + 1 : g) * (1 << BITS), nxt);
    for (int i = 0; i < nsteps; ++i, col += C::KSTEP) {
      const int s = i % C::S, ai = i % SA;
      if (*abort_flag || !tc::mbar_wait(&full[s], (i / C::S) & 1, a.check) ||
          !tc::mbar_wait(&a_empty[ai], ((i / SA) & 1) ^ 1, a.check)) {
        *abort_flag = 1; break;
      }
      tc::tc_fence_after();
      Chunk<BITS> ch[CH];
      read_idx<BITS, C::KB, CH>(smem + s * C::STAGE + C::IDX_OFF, r, part * CH, ch);
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&empty[s]);
      uint32_t v[16 * CH];
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        const int cc = col + 32 * c;
        if (row_ok && cc < d32) {
          if (cc >= g_end) {             // a chunk never straddles groups (gs % 32 == 0)
            ++g; g_end += gs32;
            if (cc >= g_end) {             // skipped a whole group: fetch directly
              do { ++g; g_end += gs32; } while (cc >= g_end);
              load_lut<BITS>(lut_row + g * (1 << BITS), L);
            } else {
              to_lut<BITS>(nxt, L);
            }
            fetch_lut<BITS>(lut_row + (g + 1 < a.gpr ? g + 1 : g) * (1 << BITS), nxt);
          }
          uint32_t o[16];
          dequant_chunk<BITS>(ch[c], L, o);
#pragma unroll
          for (int e = 0; e < 16; ++e) v[16 * c + e] = o[e];
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) v[16 * c + e] = 0u;
        }
      }
      const uint32_t taddr = tc::tmem_addr(tmem, quad * 32, ai * C::A_COLS + part * CH * 16);
      if constexpr (CH == 2) {
        tc::tmem_st32(taddr, v);
      } else {
        tc::tmem_st16(taddr, v);
      }
      tc::tmem_st_wait();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&a_full[ai]);
    }
  }

  // ---------------- epilogue ----------------
  __syncthreads();
  const bool aborted = *abort_flag != 0;
  // split-K: cluster rank q owns rows [q * 128 / ksplit, (q + 1) * 128 / ksplit)
  // of the tile; every CTA pushes those rows of its partial into rank q's
  // inbox at slot = its own rank.  Inbox layout [slot][N][RP], RP = ceil(128 / ksplit).
  const int RP = (128 + ksplit - 1) / ksplit;
  float* inbox = reinterpret_cast<float*>(smem);
  cg::cluster_group cluster = cg::this_cluster();
  // the accumulator is final once d_full fires; the tensor cores have then also
  // finished reading this CTA's stage memory, which becomes the split-K inbox
  bool have = warp < kDequantWarps && !aborted && tc::mbar_wait(d_full, 0, a.check);
  have = __all_sync(0xffffffffu, have);  // tcgen05.ld is warp-collective
  if (have) tc::tc_fence_after();
  if (ksplit > 1) cluster.sync();  // every peer's stage memory is free now
  if (ksplit == 1 && a.y_bulk) {
    if (warp < kDequantWarps)
      tc::store_tile_bulk<N, kDequantWarps>(reinterpret_cast<uint16_t*>(smem), tmem + C::D_COL, have, warp, lane, m0,
                                        a.n, t0, tlen, a.tiles != nullptr ? a.perm : nullptr, a.Y);
  } else if (warp < kDequantWarps) {
    constexpr int PARTS = kDequantWarps / 4;
    const int quad = warp & 3, part = warp >> 2;
    const int r = quad * 32 + lane;
    const int64_t row = m0 + r;
    int q = (r * ksplit) / 128;              // owner rank of row r
    while ((q + 1) * 128 / ksplit <= r) ++q;
    while (q * 128 / ksplit > r) --q;
    const int rr = r - q * 128 / ksplit;
    constexpr int GROUPS = N / 16;
    for (int gi = part; gi < GROUPS; gi += PARTS) {
      uint32_t v[16];
      if (have) {
        tc::tmem_ld16(tc::tmem_addr(tmem, quad * 32, C::D_COL + gi * 16), v);
        tc::tmem_ld_wait();
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = 0u;
      }
      if (ksplit == 1) {
        if (row < a.n) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int t = gi * 16 + j;
            if (t < tlen) {
              __nv_bfloat16 b = __float2bfloat16_rn(__uint_as_float(v[j]));
              a.Y[out_row(t) * a.n + row] = *reinterpret_cast<uint16_t*>(&b);
            }
          }
        }
      } else {
        float* dst = cluster.map_shared_rank(inbox, q) + (ks * N + gi * 16) * RP + rr;
#pragma unroll
        for (int j = 0; j < 16; ++j) dst[j * RP] = __uint_as_float(v[j]);
      }
    }
  }
  if (ksplit > 1) {
    cluster.sync();  // all pushes landed
    const int lo = ks * 128 / ksplit, rows_mine = (ks + 1) * 128 / ksplit - lo;
    for (int e = threadIdx.x; e < N * rows_mine; e += kThreads) {
      const int t = e / rows_mine, rr = e % rows_mine;
      float sum = 0.f;
      for (int qq = 0; qq < ksplit; ++qq) sum += inbox[(qq * N + t) * RP + rr];
      const int64_t row = m0 + lo + rr;
      if (t < tlen && row < a.n) {
        __nv_bfloat16 b = __float2bfloat16_rn(sum);
        a.Y[out_row(t) * a.n + row] = *reinterpret_cast<uint16_t*>(&b);
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// the shared-memory epilogue needs 16-byte aligned token rows of Y
inline int y_bulk_ok(const Problem& p, const uint16_t* Y) {
  return p.n % 8 == 0 && (reinterpret_cast<uintptr_t>(Y) & 15) == 0 && env_int("SK_TC_YBULK", 1) != 0 ? 1 : 0;
}

// ----------------------------------------------------------------------------
// Prefill tiles on a CTA pair (cta_group::2): the two CTAs of a cluster own
// 128 weight rows each of one 256-row block and share one 256-token tile.
// Each CTA dequantises its own rows into its own tensor memory (as above) but
// loads only half of the X tile (128 tokens); the even CTA issues M = 256,
// N = 256 MMAs that read the A halves from both tensor memories and the X
// halves from both shared memories, and each tensor memory receives the
// accumulator of its own rows.  Per SM this halves the X bytes streamed
// through shared memory per MMA, so the same shared memory holds a ring about
// twice as deep in time (five stages of 128 columns instead of three).
// ----------------------------------------------------------------------------

template <int BITS, int SA_, int DQW_>
struct PairCfg {
  static constexpr int N = 256;                               // tokens per pair tile
  static constexpr int KSTEP = 128;                           // weight columns per pipeline step
  static constexpr int A_COLS = KSTEP / 2;                    // TMEM columns per A stage
  static constexpr int DQW = DQW_;                            // dequantisation warps (8 or 16)
  static constexpr int TMA_WARP = DQW, MMA_WARP = DQW + 1;
  static constexpr int THREADS = (DQW + 2) * 32;
  static constexpr int CH = KSTEP / 32 / (DQW / 4);           // chunks per thread per step
  static constexpr int SA = SA_;                              // tensor-memory stages of operand A
  static constexpr int XBOXES = KSTEP / 64;
  static constexpr int KB = KSTEP * BITS / 8;
  static constexpr int X_BOX = (N / 2) * 128;                 // one 64-column box of this CTA's 128 tokens
  static constexpr int X_BYTES = XBOXES * X_BOX;
  static constexpr int IDX_OFF = align1k(X_BYTES);
  static constexpr int IDX_BYTES = 128 * KB;
  static constexpr int STAGE = IDX_OFF + align1k(IDX_BYTES);
  static constexpr int S = 5;
  static constexpr int BAR_OFF = S * STAGE;
  static constexpr int SMEM = 1024 + BAR_OFF + 512;
  static constexpr int D_COL = SA * A_COLS;
  static constexpr int TMEM_COLS = 512;
  static constexpr uint32_t IDESC = tc::idesc_bf16(256, N, 0, 0);
  static_assert(D_COL + N <= TMEM_COLS, "tensor memory budget");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert((3 * S + 2 * SA + 1) * 8 + 8 <= 512, "barrier area");
};

template <int BITS, int SA_, int DQW_>
__global__ void __launch_bounds__(PairCfg<BITS, SA_, DQW_>::THREADS, 1)
fwd_tc_pair_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_idx, FwdArgs a) {
  using C = PairCfg<BITS, SA_, DQW_>;
  constexpr int kDequantWarps = C::DQW, kTmaWarp = C::TMA_WARP, kMmaWarp = C::MMA_WARP, S = C::S, SA = C::SA;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // x_full: X halves of both CTAs (used in the even CTA only); i_full: this
  // CTA's index tile; empty: stage free again (this CTA's dequantisation warps
  // have read the index tile and the pair MMAs have read the X halves)
  uint64_t* x_full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* i_full = x_full + S;
  uint64_t* empty = i_full + S;
  uint64_t* a_full = empty + S;    // even CTA: both CTAs' A stages written
  uint64_t* a_empty = a_full + SA; // both CTAs: the pair MMAs have read A stage
  uint64_t* d_full = a_empty + SA; // both CTAs: accumulator final
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(d_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const int warp = tc::warp_id(), lane = tc::lane_id();
  const uint32_t rank = tc::cluster_ctarank();      // 0: issues the MMAs
  const int mb = a.tiles_fast ? blockIdx.z : blockIdx.y, tt = a.tiles_fast ? blockIdx.y : blockIdx.z;
  const int64_t m0 = (int64_t)mb * 256 + 128 * rank;  // this CTA's first weight row
  int t0 = tt * C::N;
  int tlen = C::N;
  const uint16_t* lut = a.lut;
  if (a.tiles != nullptr) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int tau = a.tiles[3 * tt];
    t0 = a.tiles[3 * tt + 1];
    tlen = a.tiles[3 * tt + 2];
    if (tlen == 0) return;       // both CTAs of the pair read the same entry and leave together
    lut += (int64_t)tau * a.lut_task_stride;
  } else if (t0 + tlen > a.T) {
    tlen = (int)(a.T - t0);
  }
  auto out_row = [&](int t) -> int64_t { return a.tiles != nullptr ? (int64_t)a.perm[t0 + t] : (int64_t)(t0 + t); };
  const int nsteps = a.steps_total;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      tc::mbar_init(&x_full[s], 1);
      tc::mbar_init(&i_full[s], 1);
      tc::mbar_init(&empty[s], kDequantWarps + 1);
    }
    for (int i = 0; i < SA; ++i) {
      tc::mbar_init(&a_full[i], 2 * kDequantWarps);
      tc::mbar_init(&a_empty[i], 1);
    }
    tc::mbar_init(d_full, 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == kMmaWarp) tc::tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
  if (warp == kTmaWarp && lane == 0) {
    tc::tma_prefetch(&tm_x);
    tc::tma_prefetch(&tm_idx);
  }
  tc::tc_fence_before();
  // both CTAs' barriers are initialised before either CTA signals the other
  tc::cluster_sync_all();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (a.tiles == nullptr) asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == kTmaWarp) {
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nsteps && !*abort_flag; ++i) {
        const int s = i % S;
        if (!tc::mbar_wait(&empty[s], ((i / S) & 1) ^ 1, a.check)) { *abort_flag = 1; break; }
        uint8_t* st = smem + s * C::STAGE;
        // the even CTA's x_full counts the X bytes of both CTAs
        if (rank == 0) tc::mbar_arrive_expect_tx(&x_full[s], 2 * C::X_BYTES);
        const uint32_t xbar = tc::mapa(&x_full[s], 0);
        const int k0 = i * C::KSTEP;
#pragma unroll
        for (int b = 0; b < C::XBOXES; ++b)
          tc::tma_load_2d_pair(st + b * C::X_BOX, &tm_x, xbar, k0 + 64 * b, t0 + 128 * (int)rank);
        tc::mbar_arrive_expect_tx(&i_full[s], C::IDX_BYTES);
        tc::tma_load_2d(st + C::IDX_OFF, &tm_idx, &i_full[s], i * C::KB, (int)m0);
        ++issued;
      }
      // never leave with a copy still landing in shared memory: the index
      // tiles complete on this CTA's i_full; the X halves are read by the pair
      // MMAs, whose completion frees the stage (empty)
      bool ok = true;
      for (int j = issued > S ? issued - S : 0; j < issued && ok; ++j)
        ok = tc::mbar_wait(&i_full[j % S], (j / S) & 1, a.check) && tc::mbar_wait(&empty[j % S], (j / S) & 1, a.check);
    }
  } else if (warp == kMmaWarp) {
    if (rank == 0 && lane == 0) {
      bool ok = true;
      const uint64_t desc0 = tc::sdesc(tc::smem_u32(smem), 16, 1024, tc::kSwizzle128);
      for (int i = 0; i < nsteps; ++i) {
        const int s = i % S, ai = i % SA;
        if (*abort_flag || !tc::mbar_wait(&x_full[s], (i / S) & 1, a.check) ||
            !tc::mbar_wait(&a_full[ai], (i / SA) & 1, a.check)) {
          *abort_flag = 1; ok = false; break;
        }
        tc::tc_fence_after();
        const uint64_t bd0 = desc0 + (uint64_t)((s * C::STAGE) >> 4);
        const uint32_t a0 = tmem + ai * C::A_COLS;
#pragma unroll
        for (int kk = 0; kk < C::KSTEP / 16; ++kk) {
          const uint64_t bd = bd0 + (uint64_t)(((kk >> 2) * C::X_BOX + (kk & 3) * 32) >> 4);
          tc::mma_ts_pair(tmem + C::D_COL, a0 + kk * 8, bd, C::IDESC, (i > 0 || kk > 0) ? 1u : 0u);
        }
        tc::mma_commit_pair(&empty[s]);
        tc::mma_commit_pair(&a_empty[ai]);
      }
      if (ok) tc::mma_commit_pair(d_full);
    }
  } else {
    // dequantisation into this CTA's tensor memory, as in fwd_tc_kernel
    constexpr int CH = C::CH;
    const int quad = warp & 3, part = warp >> 2;
    const int r = quad * 32 + lane;
    const int64_t row = m0 + r;
    const bool row_ok = row < a.n;
    const uint16_t* lut_row = lut + (row_ok ? row : 0) * a.gpr * (1 << BITS);
    const int d32 = (int)a.d, gs32 = (int)a.gs;
    int col = part * CH * 32;
    int g = col / gs32;
    if (g >= a.gpr) g = a.gpr - 1;
    int g_end = (g + 1) * gs32;
    LutRegs<BITS> L;
    LutRaw<BITS> nxt;
    load_lut<BITS>(lut_row + g * (1 << BITS), L);
    fetch_lut<BITS>(lut_row + (g + 1 < a.gpr ? g + 1 : g) * (1 << BITS), nxt);
    const uint32_t afull_even = tc::mapa(&a_full[0], 0);
    for (int i = 0; i < nsteps; ++i, col += C::KSTEP) {
      const int s = i % S, ai = i % SA;
      if (*abort_flag || !tc::mbar_wait(&i_full[s], (i / S) & 1, a.check) ||
          !tc::mbar_wait(&a_empty[ai], ((i / SA) & 1) ^ 1, a.check)) {
        *abort_flag = 1; break;
      }
      tc::tc_fence_after();
      Chunk<BITS> ch[CH];
      read_idx<BITS, C::KB, CH>(smem + s * C::STAGE + C::IDX_OFF, r, part * CH, ch);
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&empty[s]);
      uint32_t v[16 * CH];
#pragma unroll
      for (int c = 0; c < CH; ++c) {
        const int cc = col + 32 * c;
        if (row_ok && cc < d32) {
          if (cc >= g_end) {
            ++g; g_end += gs32;
            if (cc >= g_end) {
              do { ++g; g_end += gs32; } while (cc >= g_end);
              load_lut<BITS>(lut_row + g * (1 << BITS), L);
            } else {
              to_lut<BITS>(nxt, L);
            }
            fetch_lut<BITS>(lut_row + (g + 1 < a.gpr ? g + 1 : g) * (1 << BITS), nxt);
          }
          uint32_t o[16];
          dequant_chunk<BITS>(ch[c], L, o);
#pragma unroll
          for (int e = 0; e < 16; ++e) v[16 * c + e] = o[e];
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) v[16 * c + e] = 0u;
        }
      }
      const uint32_t taddr = tc::tmem_addr(tmem, quad * 32, ai * C::A_COLS + part * CH * 16);
      if constexpr (CH == 2) {
        tc::tmem_st32(taddr, v);
      } else {
        tc::tmem_st16(taddr, v);
      }
      tc::tmem_st_wait();
      tc::tc_fence_before();
      __syncwarp();
      // the even CTA's a_full[ai] (barriers are 8 bytes apart)
      if (lane == 0) tc::mbar_arrive_cluster(afull_even + 8 * ai);
    }
  }

  // ---------------- epilogue: each CTA writes its own 128 rows ----------------
  __syncthreads();
  const bool aborted = *abort_flag != 0;
  bool have = warp < kDequantWarps && !aborted && tc::mbar_wait(d_full, 0, a.check);
  have = __all_sync(0xffffffffu, have);
  if (have) tc::tc_fence_after();
  if (warp < kDequantWarps) {
    if (a.y_bulk) {
      tc::store_tile_bulk<C::N, kDequantWarps>(reinterpret_cast<uint16_t*>(smem), tmem + C::D_COL, have, warp, lane, m0,
                                           a.n, t0, tlen, a.tiles != nullptr ? a.perm : nullptr, a.Y);
    } else {
      constexpr int PARTS = kDequantWarps / 4;
      const int quad = warp & 3, part = warp >> 2;
      const int64_t row = m0 + quad * 32 + lane;
      for (int gi = part; gi < C::N / 16; gi += PARTS) {
        uint32_t v[16];
        if (have) {
          tc::tmem_ld16(tc::tmem_addr(tmem, quad * 32, C::D_COL + gi * 16), v);
          tc::tmem_ld_wait();
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = 0u;
        }
        if (row < a.n) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int t = gi * 16 + j;
            if (t < tlen) {
              __nv_bfloat16 b = __float2bfloat16_rn(__uint_as_float(v[j]));
              a.Y[out_row(t) * a.n + row] = *reinterpret_cast<uint16_t*>(&b);
            }
          }
        }
      }
    }
  }
  tc::tc_fence_before();
  // neither CTA leaves (or frees tensor memory) while the other may still
  // signal its barriers or the pair MMAs may still use its memory
  tc::cluster_sync_all();
  if (warp == kMmaWarp) {
    tc::tc_fence_after();
    tc::tmem_dealloc_pair(tmem, C::TMEM_COLS);
  }
}

template <int BITS, int SA, int DQW>
cudaError_t launch_pair_cfg(const Problem& p, const uint16_t* X, uint16_t* Y, cudaStream_t s, const Routed* rt) {
  using C = PairCfg<BITS, SA, DQW>;
  cudaError_t e = cudaFuncSetAttribute(fwd_tc_pair_kernel<BITS, SA, DQW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM);
  if (e != cudaSuccess) return e;
  CUtensorMap tm_x, tm_idx;
  e = make_tmap_2d(&tm_x, rt != nullptr ? rt->Xp : X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)p.d, (uint64_t)p.T,
                   (uint64_t)p.d * 2, 64, C::N / 2, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  const CUtensorMapSwizzle isw = BITS == 3 ? CU_TENSOR_MAP_SWIZZLE_NONE
                                 : C::KB == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                 : C::KB == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  e = make_tmap_2d(&tm_idx, p.packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)p.row_bytes, (uint64_t)p.n,
                   (uint64_t)p.row_bytes, C::KB, 128, isw);
  if (e != cudaSuccess) return e;
  const int steps = (int)((p.d + C::KSTEP - 1) / C::KSTEP);
  const int64_t m_pairs = (p.n + 255) / 256;
  const int64_t t_tiles = rt != nullptr ? rt->max_tiles : (p.T + C::N - 1) / C::N;
  const int64_t idx_bytes = p.n * p.row_bytes, x_bytes = p.T * p.d * 2;
  int tiles_fast = t_tiles > 1 && idx_bytes > x_bytes ? 1 : 0;
  const int forced_order = env_int("SK_TC_ORDER", -1);
  if (forced_order == 0 || forced_order == 1) tiles_fast = forced_order;
  FwdArgs args{p.lut, p.n, p.d, p.gs, p.T, p.gpr, steps, Y, p.check,
               rt != nullptr ? rt->tiles : nullptr, rt != nullptr ? rt->perm : nullptr,
               p.n * p.gpr * (1 << BITS), tiles_fast, y_bulk_ok(p, Y)};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = tiles_fast ? dim3(2u, (unsigned)t_tiles, (unsigned)m_pairs) : dim3(2u, (unsigned)m_pairs, (unsigned)t_tiles);
  cfg.blockDim = dim3(C::THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, fwd_tc_pair_kernel<BITS, SA, DQW>, tm_x, tm_idx, args);
}

template <int BITS>
cudaError_t launch_pair(const Problem& p, const uint16_t* X, uint16_t* Y, cudaStream_t s, const Routed* rt) {
  const int sa = env_int("SK_TC_PAIR_SA", 4), dqw = env_int("SK_TC_PAIR_DQW", 8);
  if (dqw == 16) {
    if (sa == 2) return launch_pair_cfg<BITS, 2, 16>(p, X, Y, s, rt);
    if (sa == 3) return launch_pair_cfg<BITS, 3, 16>(p, X, Y, s, rt);
    return launch_pair_cfg<BITS, 4, 16>(p, X, Y, s, rt);
  }
  if (sa == 2) return launch_pair_cfg<BITS, 2, 8>(p, X, Y, s, rt);
  if (sa == 3) return launch_pair_cfg<BITS, 3, 8>(p, X, Y, s, rt);
  return launch_pair_cfg<BITS, 4, 8>(p, X, Y, s, rt);
}

// 256-token tiles go to the CTA pair unless SK_TC_PAIR=0
inline bool use_pair() { return env_int("SK_TC_PAIR", 1) != 0; }

template <int BITS, int N>
cudaError_t launch_n(const Problem& p, const uint16_t* X, uint16_t* Y, cudaStream_t s, const Routed* rt = nullptr) {
  using C = Cfg<BITS, N>;
  cudaError_t e = cudaFuncSetAttribute(fwd_tc_kernel<BITS, N>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  CUtensorMap tm_x, tm_idx;
  e = make_tmap_2d(&tm_x, rt != nullptr ? rt->Xp : X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)p.d, (uint64_t)p.T,
                               (uint64_t)p.d * 2, 64, N, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  const CUtensorMapSwizzle isw = BITS == 3 ? CU_TENSOR_MAP_SWIZZLE_NONE
                                 : C::KB == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                 : C::KB == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  e = make_tmap_2d(&tm_idx, p.packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)p.row_bytes, (uint64_t)p.n,
                   (uint64_t)p.row_bytes, C::KB, 128, isw);
  if (e != cudaSuccess) return e;

  const int steps = (int)((p.d + C::KSTEP - 1) / C::KSTEP);
  const int64_t m_blocks = (p.n + 127) / 128;
  const int64_t t_tiles = rt != nullptr ? rt->max_tiles : (p.T + N - 1) / N;
  int ksplit = 1;
  if (C::DECODE) {
    // the largest split (<= 8 CTAs per cluster, >= 2 steps each) that keeps the
    // grid within one wave of one CTA per SM
    const int64_t sms = num_sms();
    for (int k = 8; k >= 1; --k) {
      if (m_blocks * t_tiles * k <= sms && 2 * k <= steps) { ksplit = k; break; }
    }
    const int forced = env_int("SK_TC_KSPLIT", 0);
    if (forced >= 1 && forced <= 8) ksplit = forced <= steps ? forced : 1;
  }
  // keep the smaller of the index map and X in L2: sweep the token tiles
  // fastest when the index map is the larger (only without a K split)
  const int64_t idx_bytes = p.n * p.row_bytes, x_bytes = p.T * p.d * 2;
  int tiles_fast = ksplit == 1 && t_tiles > 1 && idx_bytes > x_bytes ? 1 : 0;
  const int forced_order = env_int("SK_TC_ORDER", -1);
  if (ksplit == 1 && (forced_order == 0 || forced_order == 1)) tiles_fast = forced_order;
  FwdArgs args{p.lut, p.n, p.d, p.gs, p.T, p.gpr, steps, Y, p.check,
               rt != nullptr ? rt->tiles : nullptr, rt != nullptr ? rt->perm : nullptr,
               p.n * p.gpr * (1 << BITS), tiles_fast, y_bulk_ok(p, Y)};

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = tiles_fast ? dim3(1u, (unsigned)t_tiles, (unsigned)m_blocks)
                           : dim3((unsigned)ksplit, (unsigned)m_blocks, (unsigned)t_tiles);
  cfg.blockDim = dim3(C::THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = ksplit;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, fwd_tc_kernel<BITS, N>, tm_x, tm_idx, args);
}

template <int BITS>
cudaError_t launch_bits_routed(const Problem& p, const uint16_t* X, uint16_t* Y, void* ws, cudaStream_t s) {
  const int N = fwd_tc_tile_n(p.T, p.ntask);
  Routed rt;
  cudaError_t e = launch_route(p, X, p.d, Y, p.n, N, ws, &rt, s);
  if (e != cudaSuccess) return e;
  switch (N) {
    case 16: return launch_n<BITS, 16>(p, X, Y, s, &rt);
    case 32: return launch_n<BITS, 32>(p, X, Y, s, &rt);
    case 64: return launch_n<BITS, 64>(p, X, Y, s, &rt);
    case 128: return launch_n<BITS, 128>(p, X, Y, s, &rt);
    default: return use_pair() ? launch_pair<BITS>(p, X, Y, s, &rt) : launch_n<BITS, 256>(p, X, Y, s, &rt);
  }
}

template <int BITS>
cudaError_t launch_bits(const Problem& p, const uint16_t* X, uint16_t* Y, cudaStream_t s) {
  if (p.T <= 16) return launch_n<BITS, 16>(p, X, Y, s);
  if (p.T <= 32) return launch_n<BITS, 32>(p, X, Y, s);
  if (p.T <= 64) return launch_n<BITS, 64>(p, X, Y, s);
  if (p.T <= 128) return launch_n<BITS, 128>(p, X, Y, s);
  return use_pair() ? launch_pair<BITS>(p, X, Y, s, nullptr) : launch_n<BITS, 256>(p, X, Y, s);
}

}  // namespace

int fwd_tc_tile_n(int64_t T, int ntask) {
  const int64_t per = (T + ntask - 1) / ntask;   // tokens per task on average
  return per <= 16 ? 16 : per <= 32 ? 32 : per <= 64 ? 64 : per <= 128 ? 128 : 256;
}

size_t fwd_tc_workspace(int64_t T, int64_t d, int ntask) {
  return route_workspace_bytes(T, d, ntask, fwd_tc_tile_n(T, ntask));
}

cudaError_t launch_fwd_tc_routed(const Problem& p, const uint16_t* X, uint16_t* Y, void* ws, cudaStream_t s) {
  cudaError_t e;
  switch (p.bits) {
    case 2: e = launch_bits_routed<2>(p, X, Y, ws, s); break;
    case 3: e = launch_bits_routed<3>(p, X, Y, ws, s); break;
    default: e = launch_bits_routed<4>(p, X, Y, ws, s); break;
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_fwd_tc(const Problem& p, const uint16_t* X, uint16_t* Y, cudaStream_t s) {
  cudaError_t e;
  switch (p.bits) {
    case 2: e = launch_bits<2>(p, X, Y, s); break;
    case 3: e = launch_bits<3>(p, X, Y, s); break;
    default: e = launch_bits<4>(p, X, Y, s); break;
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace sk
