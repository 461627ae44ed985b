// Decode forward for a few tokens (T <= 16) with 4-bit indices, for one layer
// or a group of layers in one launch:
//   Y_l[t][i] = sum_j X_l[t][j] * Theta_hat_l[i][j]
// ("SpaLLM: Unified Compressive Adaptation of LLMs with Sketching", section
// 2.3: one compressed matmul per layer; Eq. 1 with groups per row gives
// Theta_hat).
//
// At decode batch sizes every weight is used by at most 16 tokens, so a layer
// is bound by streaming the packed indices and by the integer work of the LUT
// lookups, not by multiply-adds.  A decoder block's layers are also small
// (a few microseconds each on this GPU), so per-launch costs -- the DRAM
// latency before the first stage lands, and the wait for the slowest CTA of
// the previous layer -- are a large share of a per-layer launch.  The kernel
// is shaped for that:
//   * one persistent CTA per SM walks a contiguous share of the group's 16-row
//     tiles, cost-weighted by layer width, so the share is even to within one
//     tile whatever the layer shapes; no partial sums leave a CTA;
//   * a share is cut into passes of at most rt_max tiles of one layer; a pass
//     covers its tiles over the layer's whole K;
//   * one producer thread streams every pass's index tiles (one 3-D TMA box
//     per tile and stage, 128-byte swizzle) and the matching X columns
//     through a ring of shared-memory stages that runs on across passes and
//     layers, so DRAM never waits for a pass boundary; the index loads of the
//     first stages are issued before the grid-dependency wait, so with
//     programmatic dependent launch they overlap the end of the previous
//     kernel in the stream;
//   * the LUTs of the next pass are copied into shared memory with cp.async
//     while the current pass computes, and turned into bf16 byte planes at the
//     pass boundary;
//   * the consumer warps split each stage's (row tile, 32-column chunk) items
//     evenly; a lane loads one index word of two rows with ldmatrix, turns it
//     into bf16 weights with byte-permute lookups in register LUT planes, and
//     feeds them as the A operand of mma.sync (m16n8k16, fp32 accumulate)
//     with X as the B operand;
//   * the K order inside each 16-column MMA step is permuted so that a lane's
//     eight consecutive indices (one 32-bit word) fill exactly its A fragment:
//     MMA k-positions {2q, 2q+1, 2q+8, 2q+9} of step s hold columns
//     8q + 4s + {0, 1, 2, 3}; X is read with the same permutation, which is a
//     plain 16-byte load per lane;
//   * the per-warp partial sums of a row tile meet in shared memory and are
//     added in warp order at the end of the pass, so results are
//     deterministic.
//
// The index maps and the LUTs are read before the grid-dependency wait.  That
// is safe because they are layer weights: no kernel of this library that lets
// its dependents start early writes them, and a kernel that does not (the
// packing kernel, an optimizer step) has finished before this one can start.
// X is read, and Y written, only after the wait.
#include "sk_tc.cuh"

namespace sk {
namespace {

constexpr int kMaxDqWarps = 16;                  // consumer warps of the largest configuration
constexpr int kBoxCols = 256;                     // weight columns of one index / X box block
constexpr int kTileRows = 16;                     // rows per MMA tile
constexpr int kIdxBox = kTileRows * 128;          // one 256-column block of one row tile: 2 KB
constexpr int kRtMax = 6;                         // row tiles per pass at most
constexpr int kSmemBudget = 225 * 1024;
constexpr int kMaxLutPitch = 4096;                // byte planes of one row, all its groups

struct DqLayer {
  // packed rows: dims (128 bytes, n rows, row_bytes / 128 blocks), box (128, 16, NB), 128-byte swizzle
  CUtensorMap tm_idx;
  // X: dims (256 columns, T, d / 256 blocks), box (256, T, NB)
  CUtensorMap tm_x;
  const uint16_t* lut;     // fp16 [ntask][n][gpr][16]
  uint16_t* Y;             // bf16 [T][n]
  int64_t n;
  int d, gs, gpr, tiles, segs;
  int64_t cost0;           // cost units (one 16-row tile x 256 columns) of the layers before this one
};

struct DqGroup {
  DqLayer L[kMaxDecodeGroup];
  int nlayers, T;
  int64_t cost;            // cost units of the whole group
  // a single token with a task id (several LUT sets): the LUT set is read on
  // the device; nullptr when the batch has one LUT set
  const int32_t* task;
  int ntask;
  int stages, rt_max;
  int stage_bytes;         // idx (rt_max tiles) + X (T rows) of one stage
  int x_off;               // X offset inside a stage
  int lut_off, lut_pitch, raw_off, red_off, bar_off;
  unsigned int* check;
};

// One pass: rows [16 t0, 16 (t0 + rt)) of layer l over its whole K.
struct Pass {
  int l, t0, rt, te;       // te: the end of this CTA's tiles in layer l
  bool valid;
};

// The tiles of layer l that this CTA owns: tile k of layer l starts at cost
// cost0 + k w (w = d / 256); the CTA owns the tiles whose start lies in its
// cost range [cb, ce).
__device__ __forceinline__ void cta_tiles(const DqGroup& g, int l, int64_t cb, int64_t ce, int& tb, int& te) {
  const DqLayer& L = g.L[l];
  const int64_t w = L.d / kBoxCols;
  auto at = [&](int64_t B) -> int {
    const int64_t r = B - L.cost0;
    if (r <= 0) return 0;
    const int64_t t = (r + w - 1) / w;
    return t > L.tiles ? L.tiles : (int)t;
  };
  tb = at(cb);
  te = at(ce);
}

__device__ __forceinline__ Pass pass_from_layer(const DqGroup& g, int l, int64_t cb, int64_t ce) {
  for (; l < g.nlayers; ++l) {
    int tb, te;
    cta_tiles(g, l, cb, ce, tb, te);
    if (tb < te) return Pass{l, tb, min(g.rt_max, te - tb), te, true};
  }
  return Pass{0, 0, 0, 0, false};
}

__device__ __forceinline__ Pass next_pass(const DqGroup& g, const Pass& p, int64_t cb, int64_t ce) {
  const int t = p.t0 + p.rt;
  if (t < p.te) return Pass{p.l, t, min(g.rt_max, p.te - t), p.te, true};
  return pass_from_layer(g, p.l + 1, cb, ce);
}

// the LUT set of the batch's token (several LUT sets, one token), or of set 0
__device__ __forceinline__ const uint16_t* layer_lut(const DqGroup& g, int l, int tau) {
  if (tau < 0) return nullptr;
  return g.L[l].lut + (int64_t)tau * g.L[l].n * g.L[l].gpr * 16;
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Four 4-bit indices (selector nibbles of `s`, merge selector `m`) looked up in
// the byte planes of one row: low bytes in lo[0..3], high bytes in hi[0..3]
// (entries 4q .. 4q+3 in word q).  Returns the bf16 pairs (col 0, 1) in *p01
// and (col 2, 3) in *p23.
__device__ __forceinline__ void lookup4(uint32_t s, uint32_t m, const uint32_t (&lo)[4], const uint32_t (&hi)[4],
                                        uint32_t& p01, uint32_t& p23) {
  const uint32_t l = prmt(prmt(lo[0], lo[1], s), prmt(lo[2], lo[3], s), m);
  const uint32_t h = prmt(prmt(hi[0], hi[1], s), prmt(hi[2], hi[3], s), m);
  p01 = prmt(l, h, 0x5140);
  p23 = prmt(l, h, 0x7362);
}

// Index words of rows g and g + 8 -> A fragments of the two MMA k-steps of a
// 32-column chunk (step s takes the word's nibbles 4s .. 4s+3).  The byte
// permutes and masks run on the integer ALU, which issues at half rate on
// this GPU; the shifts are written as multiply-highs so they go to the
// multiply-add pipe instead.
__device__ __forceinline__ uint32_t shr16(uint32_t x) { return __umulhi(x, 1u << 16); }
__device__ __forceinline__ uint32_t shr1(uint32_t x) { return __umulhi(x, 1u << 31); }

__device__ __forceinline__ void dequant_frags(uint32_t w0, uint32_t w1, const uint32_t (&lo0)[4],
                                              const uint32_t (&hi0)[4], const uint32_t (&lo1)[4],
                                              const uint32_t (&hi1)[4], uint32_t (&a)[2][4]) {
  const uint32_t s0 = w0 & 0x77777777u, m0 = (shr1(w0) & 0x44444444u) | 0x32103210u;
  const uint32_t s1 = w1 & 0x77777777u, m1 = (shr1(w1) & 0x44444444u) | 0x32103210u;
  lookup4(s0, m0, lo0, hi0, a[0][0], a[0][2]);
  lookup4(s1, m1, lo1, hi1, a[0][1], a[0][3]);
  lookup4(shr16(s0), shr16(m0), lo0, hi0, a[1][0], a[1][2]);
  lookup4(shr16(s1), shr16(m1), lo1, hi1, a[1][1], a[1][3]);
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// the consumer warps' own barrier (the producer warp never joins it)
template <int W>
__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(W * 32) : "memory");
}

// SEG: weight columns per pipeline stage (a multiple of 256).  W: consumer
// warps (plus one producer warp).  NT: 8-token MMA tiles (T <= 8: one).
template <int NT, int SEG, int W>
__global__ void __launch_bounds__((W + 1) * 32, 1) __maxnreg__(W == 8 ? (NT == 1 ? 112 : 224) : 112)
decode_group_kernel(const __grid_constant__ DqGroup g) {
  constexpr int kDqWarps = W, kDqThreads = W * 32;
  constexpr bool PIPE = W == 8;
  constexpr int NB = SEG / kBoxCols;                // index / X box blocks per stage
  constexpr int SEGC = SEG / 32;                    // 32-column chunks per stage
  constexpr uint32_t kTileStage = NB * kIdxBox;     // one row tile of a stage
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + g.bar_off);
  uint64_t* empty = full + g.stages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + g.stages);
  volatile int* task_slot = abort_flag + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int64_t cb = (int64_t)blockIdx.x * g.cost / G, ce = (int64_t)(blockIdx.x + 1) * g.cost / G;
  const int S = g.stages, T = g.T;
  const uint32_t x_off = (uint32_t)g.x_off, x_box = (uint32_t)T * kBoxCols * 2;
  const uint32_t stage_bytes = (uint32_t)g.stage_bytes;
  const uint32_t smem0 = tc::smem_u32(smem);
  const Pass first = pass_from_layer(g, 0, cb, ce);

  if (warp == kDqWarps) {
    if (lane == 0) {
      // ---------------- producer: the first stages ----------------
      // the index rows of the first stages go out before anything else: they are
      // weights, so they need neither the LUT planes nor the previous launch
      for (int st = 0; st < S; ++st) {
        tc::mbar_init(&full[st], 1);
        tc::mbar_init(&empty[st], kDqWarps);
      }
      *abort_flag = 0;
      tc::fence_mbar_init();
      for (int l = 0; l < g.nlayers; ++l) {
        tc::tma_prefetch(&g.L[l].tm_idx);
        tc::tma_prefetch(&g.L[l].tm_x);
      }
      int pl[8], pseg[8], pre = 0;
      Pass P = first;
      int seg = 0;
      while (P.valid && pre < S) {
        uint8_t* st = smem + pre * stage_bytes;
        tc::mbar_arrive_expect_tx(&full[pre], (uint32_t)NB * ((uint32_t)P.rt * kIdxBox + x_box));
        for (int r = 0; r < P.rt; ++r)
          tc::tma_load_3d(st + r * kTileStage, &g.L[P.l].tm_idx, &full[pre], 0, (P.t0 + r) * kTileRows, seg * NB);
        pl[pre] = P.l;
        pseg[pre] = seg;
        ++pre;
        if (++seg == g.L[P.l].segs) { seg = 0; P = next_pass(g, P, cb, ce); }
      }
      asm volatile("griddepcontrol.wait;" ::: "memory");
      for (int i = 0; i < pre; ++i)
        tc::tma_load_3d(smem + i * stage_bytes + x_off, &g.L[pl[i]].tm_x, &full[i], 0, 0, pseg[i] * NB);
    }
  } else {
    // ---------------- consumers: the first pass's LUT planes ----------------
    // planes: [row][group] 16 low bytes then 16 high bytes of the bf16 (RNE)
    // roundings of the fp16 entries; the partial-sum buffer starts at zero
    const int tid = threadIdx.x;
    int tau = 0;
    if (g.task != nullptr) {
      // the token's LUT set: task ids are inputs, so read them after the wait;
      // an id outside [0, ntask) gets all-zero LUTs (a zero output row) and a flag
      asm volatile("griddepcontrol.wait;" ::: "memory");
      tau = __ldg(g.task);
      if (tau < 0 || tau >= g.ntask) {
        tau = -1;
        if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(g.check, SK_CHECK_TASK_RANGE);
      }
    }
    if (tid == 0) *task_slot = tau;
    if (first.valid) {
      const DqLayer& L = g.L[first.l];
      const uint16_t* lut = layer_lut(g, first.l, tau);
      const int64_t row0 = (int64_t)first.t0 * kTileRows;
      uint8_t* planes = smem + g.lut_off;
      for (int e = tid; e < first.rt * kTileRows * L.gpr; e += kDqThreads) {
        const int r = e / L.gpr, gg = e - r * L.gpr;
        uint4 lo = make_uint4(0u, 0u, 0u, 0u), hi = lo;
        if (row0 + r < L.n && lut != nullptr) {
          LutRegs<4> R;
          load_lut<4>(lut + ((row0 + r) * L.gpr + gg) * 16, R);
          lo = make_uint4(R.lo[0], R.lo[1], R.lo[2], R.lo[3]);
          hi = make_uint4(R.hi[0], R.hi[1], R.hi[2], R.hi[3]);
        }
        uint4* dst = reinterpret_cast<uint4*>(planes + r * g.lut_pitch + gg * 32);
        dst[0] = lo;
        dst[1] = hi;
      }
    }
    float* red = reinterpret_cast<float*>(smem + g.red_off);
    for (int e = tid; e < kDqWarps * 2 * kTileRows * T; e += kDqThreads) red[e] = 0.f;
  }
  __syncthreads();

  if (warp == kDqWarps) {
    // ---------------- producer: the rest of the ring ----------------
    if (lane == 0) {
      int j = 0, issued = 0;
      uint32_t st_i = 0, ph = 0;        // ring slot and its empty-phase parity
      int seg = 0;
      for (Pass P = first; P.valid && !*abort_flag;) {
        if (j >= S) {
          if (!tc::mbar_wait(&empty[st_i], ph ^ 1u, g.check)) { *abort_flag = 1; break; }
          uint8_t* st = smem + st_i * stage_bytes;
          tc::mbar_arrive_expect_tx(&full[st_i], (uint32_t)NB * ((uint32_t)P.rt * kIdxBox + x_box));
          for (int r = 0; r < P.rt; ++r)
            tc::tma_load_3d(st + r * kTileStage, &g.L[P.l].tm_idx, &full[st_i], 0, (P.t0 + r) * kTileRows, seg * NB);
          tc::tma_load_3d(st + x_off, &g.L[P.l].tm_x, &full[st_i], 0, 0, seg * NB);
        }
        ++j;
        issued = j;
        if (++st_i == (uint32_t)S) { st_i = 0; ph ^= 1u; }
        if (++seg == g.L[P.l].segs) { seg = 0; P = next_pass(g, P, cb, ce); }
      }
      // never leave with a copy still landing in shared memory
      for (int k = issued > S ? issued - S : 0; k < issued; ++k) tc::mbar_wait(&full[k % S], (k / S) & 1, g.check);
    }
    return;
  }

  // ---------------- consumers ----------------
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int tid = threadIdx.x;
  const int tau = *task_slot;
  const int g8 = lane >> 2, q = lane & 3;
  const int lut_pitch = g.lut_pitch;
  const uint32_t planes0 = smem0 + (uint32_t)g.lut_off + (uint32_t)(g8 * lut_pitch);
  const uint32_t red0 = smem0 + (uint32_t)g.red_off + (uint32_t)(warp * 2 * kTileRows * T) * 4u;
  float* red = reinterpret_cast<float*>(smem + g.red_off);
  uint8_t* raw = smem + g.raw_off;
  // ldmatrix.x4 matrices: (rows 0-7, chunk c), (rows 8-15, c), (rows 0-7, c+1), (rows 8-15, c+1)
  const int lm_row = (lane & 7) + ((lane >> 3) & 1) * 8, lm_chunk = lane >> 4;
  const uint32_t lm_x = (uint32_t)(lm_row & 7);
  uint32_t x_lane[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) x_lane[nt] = (uint32_t)((g8 + 8 * nt < T ? g8 + 8 * nt : T - 1) * kBoxCols * 2 + 16 * q);

  uint32_t slot = 0, phase = 0;
  for (Pass P = first; P.valid;) {
    const Pass Pn = next_pass(g, P, cb, ce);
    const DqLayer& L = g.L[P.l];
    // the next pass's raw fp16 LUT rows go to shared memory while this pass runs
    if (Pn.valid) {
      const DqLayer& Ln = g.L[Pn.l];
      const uint16_t* lutn = layer_lut(g, Pn.l, tau);
      if (lutn != nullptr) {
        const int64_t r0 = (int64_t)Pn.t0 * kTileRows;
        const int64_t nrows = min((int64_t)Pn.rt * kTileRows, Ln.n - r0);
        const int chunks = (int)(nrows * Ln.gpr * 2);        // 16-byte pieces
        const uint8_t* src = reinterpret_cast<const uint8_t*>(lutn + r0 * Ln.gpr * 16);
        for (int e = tid; e < chunks; e += kDqThreads) cp_async16(tc::smem_u32(raw + e * 16), src + (int64_t)e * 16);
      }
      cp_async_commit();
    }

    const int RT = P.rt, segs = L.segs;
    const int d32 = L.d, gs32 = L.gs;
    const uint32_t box_stride = kIdxBox;             // one 256-column block inside a tile's stage slice
    // items of a stage: (row tile, chunk) in row-tile-major order; the warp takes
    // 2 RT consecutive items, an even number starting at an even item, so its
    // items form at most two runs of chunk pairs (c, c + 1) in two row tiles
    const int E = RT * SEGC;
    const int e0 = warp * E / kDqWarps, e1 = (warp + 1) * E / kDqWarps;
    const int rtA = e0 / SEGC, rtB = (e1 - 1) / SEGC;
    const bool hasB = rtB != rtA;
    const int cA0 = e0 % SEGC, cA1 = hasB ? SEGC : (e1 - 1) % SEGC + 1;
    const int cB1 = hasB ? (e1 - 1) % SEGC + 1 : 0;
    // independent accumulator chains keep several MMAs in flight: chunk parity
    // always, and the two k-steps of a chunk when there is one token tile
    constexpr int CH = NT == 1 ? 2 : 1;
    float acc[2][CH][NT][4];
#pragma unroll
    for (int p = 0; p < 2; ++p)
#pragma unroll
      for (int k = 0; k < CH; ++k)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) acc[p][k][nt][jj] = 0.f;
    uint32_t lo0[4], hi0[4], lo1[4], hi1[4];
    int cur_rt = -1, cur_g = -1;
    // group of each run's current column, advanced monotonically (no divisions in the loop)
    int grA = (32 * cA0) / gs32, grA_end = (grA + 1) * gs32, grB = 0, grB_end = gs32;

    for (int i = 0; i < segs; ++i) {
      if (*abort_flag || !tc::mbar_wait(&full[slot], phase, g.check)) {
        *abort_flag = 1;
      } else {
        const uint32_t st = smem0 + slot * stage_bytes;
        const int k0 = i * SEG;
        const int avail = (d32 - k0) >> 5;                  // chunks of this stage inside the layer
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          if (r == 1 && !hasB) break;
          const int rt = r ? rtB : rtA;
          const int cbg = r ? 0 : cA0;
          int cen = r ? cB1 : cA1;
          if (cen > avail) cen = avail;
          if (cbg < cen) {
            int gi = r ? grB : grA, gend = r ? grB_end : grA_end;
            const int col0 = k0 + 32 * cbg;
            while (col0 >= gend) { ++gi; gend += gs32; }
            auto planes_for = [&](int gg) {
              const uint32_t pl = planes0 + (uint32_t)(rt * kTileRows * lut_pitch + gg * 32);
              const uint4 l0 = lds128(pl), h0 = lds128(pl + 16);
              const uint4 l1 = lds128(pl + 8 * lut_pitch), h1 = lds128(pl + 8 * lut_pitch + 16);
              lo0[0] = l0.x; lo0[1] = l0.y; lo0[2] = l0.z; lo0[3] = l0.w;
              hi0[0] = h0.x; hi0[1] = h0.y; hi0[2] = h0.z; hi0[3] = h0.w;
              lo1[0] = l1.x; lo1[1] = l1.y; lo1[2] = l1.z; lo1[3] = l1.w;
              hi1[0] = h1.x; hi1[1] = h1.y; hi1[2] = h1.z; hi1[3] = h1.w;
              cur_rt = rt; cur_g = gg;
            };
            if (rt != cur_rt || gi != cur_g) planes_for(gi);
            const bool one_group = k0 + 32 * cen <= gend;
            const uint32_t idx_row = st + (uint32_t)rt * kTileStage + (uint32_t)lm_row * 128u;
            const uint32_t xs = st + x_off;
            // shared-memory operands of chunk pair c: index words of rows g8 and
            // g8 + 8 for chunks c and c + 1, and the X fragments of both chunks
            auto fetch = [&](int c, uint32_t (&w)[4], uint4 (&x0)[NT], uint4 (&x1)[NT]) {
              const uint32_t addr = idx_row + (uint32_t)(c >> 3) * box_stride +
                                    ((((uint32_t)(c & 7) + (uint32_t)lm_chunk) ^ lm_x) << 4);
              asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                           : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "r"(addr));
              const uint32_t xc = xs + (uint32_t)(c >> 3) * x_box + ((uint32_t)(c & 7) << 6);
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                x0[nt] = lds128(xc + x_lane[nt]);
                x1[nt] = lds128(xc + x_lane[nt] + 64);
              }
            };
            // lookups and MMAs of one chunk pair from its fetched operands
            auto pair_body = [&](const uint32_t (&w)[4], const uint4 (&x0)[NT], const uint4 (&x1)[NT],
                                 bool planes_change, int col) {
              uint32_t af0[2][4];
              dequant_frags(w[0], w[1], lo0, hi0, lo1, hi1, af0);
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                mma_bf16_16816(acc[0][0][nt], af0[0], x0[nt].x, x0[nt].y);
                mma_bf16_16816(acc[0][CH - 1][nt], af0[1], x0[nt].z, x0[nt].w);
              }
              if (planes_change && col + 32 >= gend) { ++gi; gend += gs32; planes_for(gi); }  // boundary inside the pair
              uint32_t af1[2][4];
              dequant_frags(w[2], w[3], lo0, hi0, lo1, hi1, af1);
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                mma_bf16_16816(acc[1][0][nt], af1[0], x1[nt].x, x1[nt].y);
                mma_bf16_16816(acc[1][CH - 1][nt], af1[1], x1[nt].z, x1[nt].w);
              }
            };
            // without the software pipeline: the X fragments of the pair's second
            // chunk are loaded after the first chunk's MMAs (fewer live registers)
            auto x_addr = [&](int c) { return xs + (uint32_t)(c >> 3) * x_box + ((uint32_t)(c & 7) << 6); };
            auto fetch_lazy = [&](int c, uint32_t (&w)[4], uint4 (&x0)[NT]) {
              const uint32_t addr = idx_row + (uint32_t)(c >> 3) * box_stride +
                                    ((((uint32_t)(c & 7) + (uint32_t)lm_chunk) ^ lm_x) << 4);
              asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                           : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "r"(addr));
              const uint32_t xc = x_addr(c);
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) x0[nt] = lds128(xc + x_lane[nt]);
            };
            auto pair_body_lazy = [&](int c, const uint32_t (&w)[4], const uint4 (&x0)[NT], bool planes_change = false,
                                      int col = 0) {
              uint32_t af0[2][4];
              dequant_frags(w[0], w[1], lo0, hi0, lo1, hi1, af0);
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                mma_bf16_16816(acc[0][0][nt], af0[0], x0[nt].x, x0[nt].y);
                mma_bf16_16816(acc[0][CH - 1][nt], af0[1], x0[nt].z, x0[nt].w);
              }
              if (planes_change && col + 32 >= gend) { ++gi; gend += gs32; planes_for(gi); }
              uint4 x1[NT];
              const uint32_t xc = x_addr(c) + 64;
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) x1[nt] = lds128(xc + x_lane[nt]);
              uint32_t af1[2][4];
              dequant_frags(w[2], w[3], lo0, hi0, lo1, hi1, af1);
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                mma_bf16_16816(acc[1][0][nt], af1[0], x1[nt].x, x1[nt].y);
                mma_bf16_16816(acc[1][CH - 1][nt], af1[1], x1[nt].z, x1[nt].w);
              }
            };
            // d % 256 == 0, so every run is whole chunk pairs.  A run inside one
            // group (the usual case) has no checks in its loop.  With 8 consumer
            // warps the next pair's operands are loaded before this pair's
            // lookups, so their shared-memory latency hides behind the permutes;
            // 16 warps hide it by switching warps and keep the registers.
            uint32_t wc[4];
            uint4 xc0[NT], xc1[NT];
            if (one_group) {
              if constexpr (PIPE) {
                fetch(cbg, wc, xc0, xc1);
#pragma unroll 2
                for (int c = cbg; c < cen; c += 2) {
                  uint32_t wn[4];
                  uint4 xn0[NT], xn1[NT];
                  fetch(c + 2 < cen ? c + 2 : c, wn, xn0, xn1);
                  pair_body(wc, xc0, xc1, false, 0);
#pragma unroll
                  for (int k = 0; k < 4; ++k) wc[k] = wn[k];
#pragma unroll
                  for (int nt = 0; nt < NT; ++nt) { xc0[nt] = xn0[nt]; xc1[nt] = xn1[nt]; }
                }
              } else {
#pragma unroll 2
                for (int c = cbg; c < cen; c += 2) {
                  fetch_lazy(c, wc, xc0);
                  pair_body_lazy(c, wc, xc0);
                }
              }
            } else {
#pragma unroll 1
              for (int c = cbg; c < cen; c += 2) {
                const int col = k0 + 32 * c;
                if (col >= gend) { do { ++gi; gend += gs32; } while (col >= gend); planes_for(gi); }
                if constexpr (PIPE) {
                  fetch(c, wc, xc0, xc1);
                  pair_body(wc, xc0, xc1, true, col);
                } else {
                  fetch_lazy(c, wc, xc0);
                  pair_body_lazy(c, wc, xc0, true, col);
                }
              }
            }
            if (r) { grB = gi; grB_end = gend; } else { grA = gi; grA_end = gend; }
          }
          if (hasB) {
            // this run's partial sums into red[warp][r][row][t], chains restarted
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
              for (int jj = 0; jj < 4; ++jj) {
                float v = 0.f;
#pragma unroll
                for (int p = 0; p < 2; ++p)
#pragma unroll
                  for (int k = 0; k < CH; ++k) { v += acc[p][k][nt][jj]; acc[p][k][nt][jj] = 0.f; }
                const int t = 2 * q + (jj & 1) + 8 * nt, rr = g8 + 8 * (jj >> 1);
                if (t < T) {
                  const uint32_t ra = red0 + (uint32_t)((r * kTileRows + rr) * T + t) * 4u;
                  float old;
                  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(old) : "r"(ra));
                  asm volatile("st.shared.f32 [%0], %1;" ::"r"(ra), "f"(old + v));
                }
              }
          }
        }
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&empty[slot]);
      if (++slot == (uint32_t)S) { slot = 0; phase ^= 1u; }
    }
    if (!hasB) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          float v = 0.f;
#pragma unroll
          for (int p = 0; p < 2; ++p)
#pragma unroll
            for (int k = 0; k < CH; ++k) v += acc[p][k][nt][jj];
          const int t = 2 * q + (jj & 1) + 8 * nt, rr = g8 + 8 * (jj >> 1);
          if (t < T) {
            const uint32_t ra = red0 + (uint32_t)(rr * T + t) * 4u;
            asm volatile("st.shared.f32 [%0], %1;" ::"r"(ra), "f"(v));
          }
        }
    }
    cp_async_wait_all();
    consumer_sync<W>();

    // Y[t][row0 + r]: the partials of the warps whose items touch the row tile,
    // in warp order; each entry read is cleared for the next pass
    if (!*abort_flag) {
      const int rows = RT * kTileRows;
      const int ipw = RT * SEGC / kDqWarps;                 // items per warp and stage
      const int64_t row0 = (int64_t)P.t0 * kTileRows;
      for (int idx = tid; idx < rows * T; idx += kDqThreads) {
        const int t = idx / rows, rr = idx - t * rows;
        const int rt = rr / kTileRows, r = rr - rt * kTileRows;
        const int wf = rt * SEGC / ipw, wl = ((rt + 1) * SEGC - 1) / ipw;
        float sum = 0.f;
        for (int w = wf; w <= wl; ++w) {
          const int sl = rt - (w * ipw) / SEGC;
          float* e = &red[((w * 2 + sl) * kTileRows + r) * T + t];
          sum += *e;
          *e = 0.f;
        }
        const int64_t row = row0 + rr;
        if (row < L.n) {
          __nv_bfloat16 b = __float2bfloat16_rn(sum);
          L.Y[(int64_t)t * L.n + row] = *reinterpret_cast<uint16_t*>(&b);
        }
      }
    }
    // the next pass's byte planes from the raw rows copied during this pass
    if (Pn.valid) {
      const DqLayer& Ln = g.L[Pn.l];
      const bool have = layer_lut(g, Pn.l, tau) != nullptr;
      const int64_t r0 = (int64_t)Pn.t0 * kTileRows;
      uint8_t* planes = smem + g.lut_off;
      for (int e = tid; e < Pn.rt * kTileRows * Ln.gpr; e += kDqThreads) {
        const int r = e / Ln.gpr, gg = e - r * Ln.gpr;
        uint4 lo = make_uint4(0u, 0u, 0u, 0u), hi = lo;
        if (have && r0 + r < Ln.n) {
          const uint4* src = reinterpret_cast<const uint4*>(raw + (r * Ln.gpr + gg) * 32);
          LutRaw<4> rw;
          rw.a = src[0];
          rw.b = src[1];
          LutRegs<4> R;
          to_lut<4>(rw, R);
          lo = make_uint4(R.lo[0], R.lo[1], R.lo[2], R.lo[3]);
          hi = make_uint4(R.hi[0], R.hi[1], R.hi[2], R.hi[3]);
        }
        uint4* dst = reinterpret_cast<uint4*>(planes + r * lut_pitch + gg * 32);
        dst[0] = lo;
        dst[1] = hi;
      }
    }
    consumer_sync<W>();
    P = Pn;
  }
}

__host__ __device__ constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }

struct GroupPlan {
  int seg, warps, nt, grid, smem;
};

// Shared-memory plan of one launch over `nl` layers; false when a layer does
// not suit the kernel.
bool plan(const DecodeLayer* layers, int nl, int T, const int32_t* task, int ntask, DqGroup* g, GroupPlan* gp) {
  if (nl < 1 || nl > kMaxDecodeGroup || T < 1 || T > 16) return false;
  if (task != nullptr && ntask != 1 && T != 1) return false;   // several LUT sets: one token only
  int64_t dmax = 0;
  int gpr_max = 0;
  for (int l = 0; l < nl; ++l) {
    const DecodeLayer& L = layers[l];
    // d % 256 == 0: index rows are whole 128-byte blocks (the 3-D box never
    // reaches past a row), X rows whole 256-column blocks
    if (L.d % kBoxCols != 0 || L.gpr < 1 || L.d % L.gpr != 0 || (L.d / L.gpr) % 32 != 0) return false;
    if (L.gpr * 32 + 16 > kMaxLutPitch) return false;
    dmax = L.d > dmax ? L.d : dmax;
    gpr_max = L.gpr > gpr_max ? L.gpr : gpr_max;
  }
  const int lut_pitch = gpr_max * 32 + 16;
  const int red_bytes = align_up(kMaxDqWarps * 2 * kTileRows * T * 4, 16);
  const int bar_bytes = 2 * 8 * 8 + 16;
  // the longest stage (2048 or 1024 columns at most, no longer than the widest
  // layer needs, 512 for narrow layers) with the most tiles per pass whose
  // double buffer fits beside the LUT planes
  int SEG = T <= 8 ? 2048 : 1024;
  while (SEG > 512 && SEG / 2 >= dmax) SEG /= 2;
  int rt = kRtMax, S = 0, stage = 0, lut_bytes = 0, raw_bytes = 0, total = 0;
  for (;; --rt) {
    if (rt < 1) {
      if (SEG == 512) return false;
      SEG /= 2;
      rt = kRtMax;
    }
    const int idx_region = rt * (SEG / kBoxCols) * kIdxBox;
    stage = align_up(idx_region + T * SEG * 2, 1024);
    lut_bytes = align_up(rt * kTileRows * lut_pitch, 16);
    raw_bytes = align_up(rt * kTileRows * gpr_max * 32, 16);
    const int fixed = 1024 + lut_bytes + raw_bytes + red_bytes + bar_bytes;
    S = (kSmemBudget - fixed) / stage;
    if (S > 4) S = 4;
    if (S < 2) continue;
    total = fixed + S * stage;
    break;
  }
  const int idx_region = rt * (SEG / kBoxCols) * kIdxBox;
  int64_t cost = 0;
  for (int l = 0; l < nl; ++l) {
    const DecodeLayer& L = layers[l];
    DqLayer& D = g->L[l];
    D.lut = L.lut;
    D.Y = L.Y;
    D.n = L.n;
    D.d = (int)L.d;
    D.gpr = L.gpr;
    D.gs = (int)(L.d / L.gpr);
    D.tiles = (int)((L.n + kTileRows - 1) / kTileRows);
    D.segs = (int)((L.d + SEG - 1) / SEG);
    D.cost0 = cost;
    cost += (int64_t)D.tiles * (L.d / kBoxCols);
  }
  g->nlayers = nl;
  g->T = T;
  g->cost = cost;
  g->task = (task != nullptr && ntask != 1) ? task : nullptr;
  g->ntask = ntask;
  g->stages = S;
  g->rt_max = rt;
  g->stage_bytes = stage;
  g->x_off = idx_region;
  g->lut_off = S * stage;
  g->lut_pitch = lut_pitch;
  g->raw_off = g->lut_off + lut_bytes;
  g->red_off = g->raw_off + raw_bytes;
  g->bar_off = g->red_off + red_bytes;
  gp->seg = SEG;
  gp->warps = SEG == 512 ? 8 : 16;
  gp->nt = T <= 8 ? 1 : 2;
  gp->smem = total;
  // one CTA per SM, fewer when the group has fewer tiles than SMs
  int64_t tiles = 0;
  for (int l = 0; l < nl; ++l) tiles += g->L[l].tiles;
  const int sms = num_sms();
  gp->grid = (int)(tiles < sms ? tiles : sms);
  return true;
}

template <int NT, int SEG, int W>
cudaError_t launch_k(const DecodeLayer* layers, DqGroup& g, const GroupPlan& gp, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(decode_group_kernel<NT, SEG, W>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       gp.smem);
  if (e != cudaSuccess) return e;
  constexpr int NB = SEG / kBoxCols;
  for (int l = 0; l < g.nlayers; ++l) {
    const DecodeLayer& L = layers[l];
    // one row tile of a stage: dims (128 bytes, rows, 256-column blocks) at
    // strides (row_bytes, 128), box (128, 16, NB)
    const uint64_t nblk = (uint64_t)L.row_bytes / 128;
    e = make_tmap_3d(&g.L[l].tm_idx, L.packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128, (uint64_t)L.n, nblk,
                     (uint64_t)L.row_bytes, 128, 128, kTileRows, NB, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    // X tile: dims (256 columns, tokens, 256-column blocks) at strides (2 d, 512)
    e = make_tmap_3d(&g.L[l].tm_x, L.X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kBoxCols, (uint64_t)g.T,
                     (uint64_t)L.d / kBoxCols, (uint64_t)L.d * 2, kBoxCols * 2, kBoxCols, (uint32_t)g.T, NB,
                     CU_TENSOR_MAP_SWIZZLE_NONE);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)gp.grid, 1, 1);
  cfg.blockDim = dim3((W + 1) * 32, 1, 1);
  cfg.dynamicSmemBytes = (size_t)gp.smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, decode_group_kernel<NT, SEG, W>, g);
  return e != cudaSuccess ? e : cudaGetLastError();
}

DecodeLayer layer_of(const Problem& p, const uint16_t* X, uint16_t* Y) {
  DecodeLayer L;
  L.packed = p.packed;
  L.row_bytes = p.row_bytes;
  L.lut = p.lut;
  L.gpr = p.gpr;
  L.n = p.n;
  L.d = p.d;
  L.X = X;
  L.Y = Y;
  return L;
}

}  // namespace

bool decode_group_supported(const DecodeLayer* layers, int nl, int T, const int32_t* task, int ntask) {
  DqGroup g;
  GroupPlan gp;
  return plan(layers, nl, T, task, ntask, &g, &gp);
}

cudaError_t launch_decode_group(const DecodeLayer* layers, int nl, int T, const int32_t* task, int ntask,
                                unsigned int* check, cudaStream_t s) {
  DqGroup g;
  GroupPlan gp;
  if (!plan(layers, nl, T, task, ntask, &g, &gp)) return cudaErrorInvalidValue;
  g.check = check;
  if (gp.nt == 1) {
    if (gp.seg == 2048) return launch_k<1, 2048, 16>(layers, g, gp, s);
    if (gp.seg == 1024) return launch_k<1, 1024, 16>(layers, g, gp, s);
    return launch_k<1, 512, 8>(layers, g, gp, s);
  }
  if (gp.seg == 1024) return launch_k<2, 1024, 16>(layers, g, gp, s);
  return launch_k<2, 512, 8>(layers, g, gp, s);
}

bool decode_fwd_supported(const Problem& p) {
  if (p.bits != 4) return false;
  const DecodeLayer L = layer_of(p, nullptr, nullptr);
  return decode_group_supported(&L, 1, (int)p.T, p.task, p.ntask);
}

cudaError_t launch_decode_fwd(const Problem& p, const uint16_t* X, uint16_t* Y, cudaStream_t s) {
  if (p.bits != 4) return cudaErrorInvalidValue;
  const DecodeLayer L = layer_of(p, X, Y);
  return launch_decode_group(&L, 1, (int)p.T, p.task, p.ntask, p.check, s);
}

}  // namespace sk
