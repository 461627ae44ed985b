// Decode forward for a few tokens (T <= 16) with 4-bit indices:
//   Y[t][i] = sum_j X[t][j] * Theta_hat[i][j]
// ("SpaLLM: Unified Compressive Adaptation of LLMs with Sketching", section
// 2.3: one compressed matmul per layer; Eq. 1 with groups per row gives
// Theta_hat).
//
// At decode batch sizes every weight is used by at most 16 tokens, so the
// layer is bound by streaming the packed indices and by the integer work of
// the LUT lookups, not by multiply-adds.  The kernel is shaped for that:
//   * every CTA owns a contiguous range of 16-row tiles over the whole K, so
//     no partial sums leave the CTA; the grid is one CTA per SM;
//   * one producer thread streams the CTA's index rows (one 3-D TMA box per
//     stage, 128-byte swizzle) and the matching X columns (one 3-D box)
//     through a ring of shared-memory stages of 512 to 2048 columns; the index
//     loads of the first stages are issued before the grid-dependency wait, so
//     with programmatic dependent launch they overlap the end of the previous
//     kernel in the stream;
//   * the consumer warps split each stage's (row tile, 32-column chunk)
//     items evenly; a lane loads one index word of two rows with ldmatrix,
//     turns it into bf16 weights with byte-permute lookups in register LUT
//     planes, and feeds them as the A operand of mma.sync (m16n8k16, fp32
//     accumulate) with X as the B operand;
//   * the K order inside each 16-column MMA step is permuted so that a lane's
//     eight consecutive indices (one 32-bit word) fill exactly its A fragment:
//     MMA k-positions {2q, 2q+1, 2q+8, 2q+9} of step s hold columns
//     8q + 4s + {0, 1, 2, 3}; X is read with the same permutation, which is a
//     plain 16-byte load per lane;
//   * the per-warp partial sums of a row tile meet in shared memory and are
//     added in warp order, so results are deterministic.
//
// The index map and the LUTs are read before the grid-dependency wait.  That
// is safe because they are layer weights: no kernel of this library that lets
// its dependents start early writes them, and a kernel that does not (the
// packing kernel, an optimizer step) has finished before this one can start.
// X is read, and Y written, only after the wait.
#include "sk_tc.cuh"

namespace sk {
namespace {

constexpr int kMaxDqWarps = 16;                  // consumer warps of the largest configuration
constexpr int kBoxCols = 256;                     // weight columns of one index / X box
constexpr int kTileRows = 16;                     // rows per MMA tile
constexpr int kIdxBox = kTileRows * 128;          // one 128-byte-wide index box of a row tile
constexpr int kRtMax = 6;                         // row tiles per CTA at most
constexpr int kSmemBudget = 110 * 1024;           // leaves room for a CTA of the next launch (T <= 8)
constexpr int kSmemBudget2 = 200 * 1024;          // two token tiles: one CTA per SM

struct DqArgs {
  const uint16_t* lut;
  // a single token with a task id (several LUT sets): the LUT set is read on
  // the device; nullptr when the batch has one LUT set
  const int32_t* task;
  int ntask;
  int64_t n, d, gs;
  int gpr, T;
  int tiles;          // ceil(n / 16)
  int segs;           // ceil(d / 512)
  int stages;         // ring depth
  int rt_max;         // row tiles of the largest CTA
  int stage_bytes;    // idx (rt_max tiles) + X (T rows) of one stage
  int x_off;          // X offset inside a stage
  int lut_off, lut_pitch, red_off, bar_off;
  uint16_t* Y;
  unsigned int* check;
};

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
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

// One token tile (T <= 8) fits two CTAs per SM (this launch and the next one
// in the stream); two token tiles need more registers.
// SEG: weight columns per pipeline stage (a multiple of 256).  Long stages
// give every warp long runs of chunk pairs, which spreads the per-stage and
// per-run bookkeeping over more lookups.
// W: consumer warps (plus one producer warp).
template <int NT, int SEG, int W>
__global__ void __launch_bounds__((W + 1) * 32, 1) __maxnreg__(W == 8 ? (NT == 1 ? 112 : 224) : 96)
decode_kernel(const __grid_constant__ CUtensorMap tm_hi, const __grid_constant__ CUtensorMap tm_lo,
              const __grid_constant__ CUtensorMap tm_x, DqArgs a) {
  constexpr int kDqWarps = W, kDqThreads = (W + 1) * 32;
  constexpr bool PIPE = W == 8;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + a.bar_off);
  uint64_t* empty = full + a.stages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + a.stages);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int rt0 = (int)((int64_t)blockIdx.x * a.tiles / G), rt1 = (int)((int64_t)(blockIdx.x + 1) * a.tiles / G);
  const int RT = rt1 - rt0;                         // rt_max or rt_max - 1
  const int64_t row0 = (int64_t)rt0 * kTileRows;
  const int S = a.stages, T = a.T, gpr = a.gpr, segs = a.segs;
  const int pre = segs < S ? segs : S;
  // stage layout: the index tile as NB blocks of 256 columns (128 bytes) x all
  // the CTA's rows, one 3-D TMA box [block][row][128 B] with the 128-byte
  // swizzle, then the X tile as [block][token][256 columns], one 3-D box
  constexpr int NB = SEG / kBoxCols;                // index / X boxes per stage
  constexpr int SEGC = SEG / 32;                    // 32-column chunks per stage
  const uint32_t box_stride = (uint32_t)RT * kIdxBox;     // one 256-column block of the index tile
  const uint32_t x_off = (uint32_t)a.x_off, x_box = (uint32_t)T * kBoxCols * 2;
  const uint32_t stage_bytes = (uint32_t)a.stage_bytes;
  const uint32_t tx_bytes = (uint32_t)NB * ((uint32_t)RT * kIdxBox + x_box);
  const CUtensorMap* tm_idx = RT == a.rt_max ? &tm_hi : &tm_lo;
  const uint32_t smem0 = tc::smem_u32(smem);

  if (warp == kDqWarps && lane == 0) {
    // ---------------- producer ----------------
    // the index rows of the first stages go out before anything else: they are
    // weights, so they need neither the LUT planes nor the previous launch
    for (int st = 0; st < S; ++st) {
      tc::mbar_init(&full[st], 1);
      tc::mbar_init(&empty[st], kDqWarps);
    }
    *abort_flag = 0;
    tc::fence_mbar_init();
    tc::tma_prefetch(tm_idx);
    tc::tma_prefetch(&tm_x);
    for (int i = 0; i < pre; ++i) {
      uint8_t* st = smem + i * stage_bytes;
      tc::mbar_arrive_expect_tx(&full[i], tx_bytes);
      tc::tma_load_3d(st, tm_idx, &full[i], 0, (int)row0, i * NB);
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    for (int i = 0; i < pre; ++i) {
      uint8_t* st = smem + i * stage_bytes + x_off;
      tc::tma_load_3d(st, &tm_x, &full[i], 0, 0, i * NB);
    }
  } else {
    // LUT byte planes of the CTA's rows: [row][group] 16 low bytes then 16 high
    // bytes of the bf16 (RNE) roundings of the fp16 entries; the partial-sum
    // buffer starts at zero
    uint8_t* planes = smem + a.lut_off;
    const int tid = threadIdx.x < kDqWarps * 32 ? threadIdx.x : threadIdx.x - 1;   // skip the producer thread
    const int nthr = kDqThreads - 1;
    const uint16_t* lut = a.lut;
    if (a.task != nullptr) {
      // the token's LUT set: task ids are inputs, so read them after the wait;
      // an id outside [0, ntask) gets all-zero LUTs (a zero output row) and a flag
      asm volatile("griddepcontrol.wait;" ::: "memory");
      const int tau = __ldg(a.task);
      if (tau < 0 || tau >= a.ntask) {
        lut = nullptr;
        if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(a.check, SK_CHECK_TASK_RANGE);
      } else {
        lut += (int64_t)tau * a.n * gpr * 16;
      }
    }
    for (int e = tid; e < RT * kTileRows * gpr; e += nthr) {
      const int r = e / gpr, g = e - r * gpr;
      uint4 lo = make_uint4(0u, 0u, 0u, 0u), hi = lo;
      if (row0 + r < a.n && lut != nullptr) {
        LutRegs<4> L;
        load_lut<4>(lut + ((row0 + r) * gpr + g) * 16, L);
        lo = make_uint4(L.lo[0], L.lo[1], L.lo[2], L.lo[3]);
        hi = make_uint4(L.hi[0], L.hi[1], L.hi[2], L.hi[3]);
      }
      uint4* dst = reinterpret_cast<uint4*>(planes + r * a.lut_pitch + g * 32);
      dst[0] = lo;
      dst[1] = hi;
    }
    float* red = reinterpret_cast<float*>(smem + a.red_off);
    for (int e = tid; e < kDqWarps * 2 * kTileRows * T; e += nthr) red[e] = 0.f;
  }
  __syncthreads();

  if (warp == kDqWarps) {
    // ---------------- producer: the rest of the ring ----------------
    if (lane == 0) {
      int issued = pre;
      uint32_t st_i = (uint32_t)(pre % S), ph = pre >= S ? 1u : 0u;   // ring slot and its empty-phase parity
      for (int i = pre; i < segs && !*abort_flag; ++i) {
        if (!tc::mbar_wait(&empty[st_i], ph ^ 1u, a.check)) { *abort_flag = 1; break; }
        uint8_t* st = smem + st_i * stage_bytes;
        tc::mbar_arrive_expect_tx(&full[st_i], tx_bytes);
        tc::tma_load_3d(st, tm_idx, &full[st_i], 0, (int)row0, i * NB);
        tc::tma_load_3d(st + x_off, &tm_x, &full[st_i], 0, 0, i * NB);
        ++issued;
        if (++st_i == (uint32_t)S) { st_i = 0; ph ^= 1u; }
      }
      // never leave with a copy still landing in shared memory
      for (int j = issued > S ? issued - S : 0; j < issued; ++j) tc::mbar_wait(&full[j % S], (j / S) & 1, a.check);
    }
  } else {
    // ---------------- consumers ----------------
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int g8 = lane >> 2, q = lane & 3;
    const int d32 = (int)a.d, gs32 = (int)a.gs, lut_pitch = a.lut_pitch;
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
          for (int j = 0; j < 4; ++j) acc[p][k][nt][j] = 0.f;
    const uint32_t planes0 = tc::smem_u32(smem + a.lut_off) + (uint32_t)(g8 * lut_pitch);
    const uint32_t red0 = tc::smem_u32(smem + a.red_off) + (uint32_t)(warp * 2 * kTileRows * T) * 4u;
    uint32_t lo0[4], hi0[4], lo1[4], hi1[4];
    int cur_rt = -1, cur_g = -1;
    // ldmatrix.x4 matrices: (rows 0-7, chunk c), (rows 8-15, c), (rows 0-7, c+1), (rows 8-15, c+1)
    const int lm_row = (lane & 7) + ((lane >> 3) & 1) * 8, lm_chunk = lane >> 4;
    const uint32_t lm_x = (uint32_t)(lm_row & 7);
    uint32_t x_lane[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) x_lane[nt] = (uint32_t)((g8 + 8 * nt < T ? g8 + 8 * nt : T - 1) * kBoxCols * 2 + 16 * q);
    // group of each run's current column, advanced monotonically (no divisions in the loop)
    int grA = (32 * cA0) / gs32, grA_end = (grA + 1) * gs32, grB = 0, grB_end = gs32;

    uint32_t slot = 0, phase = 0;
    for (int i = 0; i < segs; ++i) {
      if (*abort_flag || !tc::mbar_wait(&full[slot], phase, a.check)) { *abort_flag = 1; break; }
      const uint32_t st = smem0 + slot * stage_bytes;
      const int k0 = i * SEG;
      const int avail = (d32 - k0) >> 5;                  // chunks of this stage inside the layer
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        if (r == 1 && !hasB) break;
        const int rt = r ? rtB : rtA;
        const int cb = r ? 0 : cA0;
        int ce = r ? cB1 : cA1;
        if (ce > avail) ce = avail;
        if (cb < ce) {
          int g = r ? grB : grA, gend = r ? grB_end : grA_end;
          const int col0 = k0 + 32 * cb;
          while (col0 >= gend) { ++g; gend += gs32; }
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
          if (rt != cur_rt || g != cur_g) planes_for(g);
          const bool one_group = k0 + 32 * ce <= gend;
          const uint32_t idx_row = st + (uint32_t)(rt * kTileRows + lm_row) * 128u;
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
          auto pair_body = [&](const uint32_t (&w)[4], const uint4 (&x0)[NT], const uint4 (&x1)[NT], bool planes_change,
                               int col) {
            uint32_t af0[2][4];
            dequant_frags(w[0], w[1], lo0, hi0, lo1, hi1, af0);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              mma_bf16_16816(acc[0][0][nt], af0[0], x0[nt].x, x0[nt].y);
              mma_bf16_16816(acc[0][CH - 1][nt], af0[1], x0[nt].z, x0[nt].w);
            }
            if (planes_change && col + 32 >= gend) { ++g; gend += gs32; planes_for(g); }  // boundary inside the pair
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
            if (planes_change && col + 32 >= gend) { ++g; gend += gs32; planes_for(g); }
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
              fetch(cb, wc, xc0, xc1);
#pragma unroll 2
              for (int c = cb; c < ce; c += 2) {
                uint32_t wn[4];
                uint4 xn0[NT], xn1[NT];
                fetch(c + 2 < ce ? c + 2 : c, wn, xn0, xn1);
                pair_body(wc, xc0, xc1, false, 0);
#pragma unroll
                for (int k = 0; k < 4; ++k) wc[k] = wn[k];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) { xc0[nt] = xn0[nt]; xc1[nt] = xn1[nt]; }
              }
            } else {
#pragma unroll 2
              for (int c = cb; c < ce; c += 2) {
                fetch_lazy(c, wc, xc0);
                pair_body_lazy(c, wc, xc0);
              }
            }
          } else {
#pragma unroll 1
            for (int c = cb; c < ce; c += 2) {
              const int col = k0 + 32 * c;
              if (col >= gend) { do { ++g; gend += gs32; } while (col >= gend); planes_for(g); }
              if constexpr (PIPE) {
                fetch(c, wc, xc0, xc1);
                pair_body(wc, xc0, xc1, true, col);
              } else {
                fetch_lazy(c, wc, xc0);
                pair_body_lazy(c, wc, xc0, true, col);
              }
            }
          }
          if (r) { grB = g; grB_end = gend; } else { grA = g; grA_end = gend; }
        }
        if (hasB) {
          // this run's partial sums into red[warp][r][row][t], chains restarted
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              float v = 0.f;
#pragma unroll
              for (int p = 0; p < 2; ++p)
#pragma unroll
                for (int k = 0; k < CH; ++k) { v += acc[p][k][nt][j]; acc[p][k][nt][j] = 0.f; }
              const int t = 2 * q + (j & 1) + 8 * nt, rr = g8 + 8 * (j >> 1);
              if (t < T) {
                const uint32_t ra = red0 + (uint32_t)((r * kTileRows + rr) * T + t) * 4u;
                float old;
                asm volatile("ld.shared.f32 %0, [%1];" : "=f"(old) : "r"(ra));
                asm volatile("st.shared.f32 [%0], %1;" ::"r"(ra), "f"(old + v));
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
        for (int j = 0; j < 4; ++j) {
          float v = 0.f;
#pragma unroll
          for (int p = 0; p < 2; ++p)
#pragma unroll
            for (int k = 0; k < CH; ++k) v += acc[p][k][nt][j];
          const int t = 2 * q + (j & 1) + 8 * nt, rr = g8 + 8 * (j >> 1);
          if (t < T) {
            const uint32_t ra = red0 + (uint32_t)(rr * T + t) * 4u;
            asm volatile("st.shared.f32 [%0], %1;" ::"r"(ra), "f"(v));
          }
        }
    }
  }
  __syncthreads();
  if (*abort_flag) return;
  // Y[t][row0 + r]: the partials of the warps whose items touch the row tile, in warp order
  const float* red = reinterpret_cast<const float*>(smem + a.red_off);
  const int rows = RT * kTileRows;
  const int ipw = RT * SEGC / kDqWarps;                 // items per warp and stage
  for (int idx = threadIdx.x; idx < rows * T; idx += kDqThreads) {
    const int t = idx / rows, rr = idx - t * rows;
    const int rt = rr / kTileRows, r = rr - rt * kTileRows;
    const int wf = rt * SEGC / ipw, wl = ((rt + 1) * SEGC - 1) / ipw;
    float sum = 0.f;
    for (int w = wf; w <= wl; ++w) {
      const int slot = rt - (w * ipw) / SEGC;
      sum += red[((w * 2 + slot) * kTileRows + r) * T + t];
    }
    const int64_t row = row0 + rr;
    if (row < a.n) {
      __nv_bfloat16 b = __float2bfloat16_rn(sum);
      a.Y[(int64_t)t * a.n + row] = *reinterpret_cast<uint16_t*>(&b);
    }
  }
}

__host__ __device__ constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }

// Shared-memory plan of one launch; false when the layer does not suit the kernel.
bool plan(const Problem& p, DqArgs* a, int* grid, int* smem, int* seg) {
  // d % 256 == 0: index rows are whole 128-byte blocks (the 3-D box never
  // reaches past a row), X rows whole 256-column blocks
  if (p.bits != 4 || p.T < 1 || p.T > 16 || p.d % kBoxCols != 0) return false;
  if (p.task != nullptr && p.ntask != 1 && p.T != 1) return false;   // several LUT sets: one token only
  const int tiles = (int)((p.n + kTileRows - 1) / kTileRows);
  const int sms = num_sms();
  int G = tiles < sms ? tiles : sms;
  if ((tiles + G - 1) / G > kRtMax) G = (tiles + kRtMax - 1) / kRtMax;
  const int rt_max = (tiles + G - 1) / G;
  const int T = (int)p.T;
  const int lut_pitch = p.gpr * 32 + 16;
  const int lut_bytes = align_up(rt_max * kTileRows * lut_pitch, 16);
  if (lut_bytes > 48 * 1024) return false;
  const int red_bytes = align_up(kMaxDqWarps * 2 * kTileRows * T * 4, 16);
  const int bar_bytes = 2 * 8 * 8 + 16;
  // the longest stage (2048, 1024 or 512 columns, no longer than the layer
  // needs) whose double buffer fits beside the LUT planes
  const int budget = p.T <= 8 ? kSmemBudget : kSmemBudget2;
  int SEG = p.T <= 8 ? 2048 : 1024;
  while (SEG > 512 && SEG / 2 >= p.d) SEG /= 2;
  for (;; SEG /= 2) {
    const int idx_region = (SEG / kBoxCols) * rt_max * kIdxBox;
    const int stage = align_up(idx_region + T * SEG * 2, 1024);
    const int segs = (int)((p.d + SEG - 1) / SEG);
    int S = (budget - 1024 - lut_bytes - red_bytes - bar_bytes) / stage;
    if (S > 8) S = 8;
    if (S > segs) S = segs;
    if (S < 2) S = 2;
    const int total = 1024 + S * stage + lut_bytes + red_bytes + bar_bytes;
    if (total > budget && SEG > 512) continue;
    if (total > 227 * 1024) return false;
    a->lut = p.lut; a->task = (p.task != nullptr && p.ntask != 1) ? p.task : nullptr; a->ntask = p.ntask;
    a->n = p.n; a->d = p.d; a->gs = p.gs; a->gpr = p.gpr; a->T = T;
    a->tiles = tiles; a->segs = segs; a->stages = S; a->rt_max = rt_max;
    a->stage_bytes = stage; a->x_off = idx_region;
    a->lut_off = S * stage; a->lut_pitch = lut_pitch;
    a->red_off = a->lut_off + lut_bytes;
    a->bar_off = a->red_off + red_bytes;
    a->check = p.check;
    *grid = G;
    *smem = total;
    *seg = SEG;
    return true;
  }
}

template <int NT, int SEG, int W>
cudaError_t launch_nt(const Problem& p, const uint16_t* X, uint16_t* Y, const DqArgs& args0, int grid, int smem,
                      cudaStream_t s) {
  DqArgs args = args0;
  args.Y = Y;
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<NT, SEG, W>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // index tile of all the rows of a CTA (rt_max or rt_max - 1 row tiles):
  // dims (128 bytes, rows, 256-column blocks) at strides (row_bytes, 128)
  CUtensorMap tm_hi, tm_lo, tm_x;
  constexpr int NB = SEG / kBoxCols;
  const int rt_lo = args.rt_max > 1 ? args.rt_max - 1 : 1;
  const uint64_t nblk = (uint64_t)p.row_bytes / 128;
  e = make_tmap_3d(&tm_hi, p.packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128, (uint64_t)p.n, nblk, (uint64_t)p.row_bytes,
                   128, 128, (uint32_t)(args.rt_max * kTileRows), NB, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  e = make_tmap_3d(&tm_lo, p.packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128, (uint64_t)p.n, nblk, (uint64_t)p.row_bytes,
                   128, 128, (uint32_t)(rt_lo * kTileRows), NB, CU_TENSOR_MAP_SWIZZLE_128B);
  if (e != cudaSuccess) return e;
  // X tile: dims (256 columns, tokens, 256-column blocks) at strides (2 d, 512)
  e = make_tmap_3d(&tm_x, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kBoxCols, (uint64_t)p.T, (uint64_t)p.d / kBoxCols,
                   (uint64_t)p.d * 2, kBoxCols * 2, kBoxCols, (uint32_t)p.T, NB, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3((W + 1) * 32, 1, 1);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, decode_kernel<NT, SEG, W>, tm_hi, tm_lo, tm_x, args);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int W>
cudaError_t launch_w(const Problem& p, const uint16_t* X, uint16_t* Y, const DqArgs& a, int grid, int smem, int seg,
                     cudaStream_t s) {
  if (p.T <= 8) {
    if (seg == 2048) return launch_nt<1, 2048, W>(p, X, Y, a, grid, smem, s);
    if (seg == 1024) return launch_nt<1, 1024, W>(p, X, Y, a, grid, smem, s);
    return launch_nt<1, 512, W>(p, X, Y, a, grid, smem, s);
  }
  if (seg == 1024) return launch_nt<2, 1024, W>(p, X, Y, a, grid, smem, s);
  return launch_nt<2, 512, W>(p, X, Y, a, grid, smem, s);
}

}  // namespace

bool decode_fwd_supported(const Problem& p) {
  DqArgs a;
  int g, sm, seg;
  return plan(p, &a, &g, &sm, &seg);
}

// Consumer warps per CTA: 16 by default (four per scheduler hide the
// shared-memory and MMA latencies); SK_DQ_WARPS=8 selects the variant with
// software-pipelined operand loads, for measurements.
cudaError_t launch_decode_fwd(const Problem& p, const uint16_t* X, uint16_t* Y, cudaStream_t s) {
  DqArgs a;
  int grid = 0, smem = 0, seg = 0;
  if (!plan(p, &a, &grid, &smem, &seg)) return cudaErrorInvalidValue;
  // 16 warps need an even number of 32-column chunks per warp and stage: RT x SEG / 512 even
  const int w = env_int("SK_DQ_WARPS", 16);
  return (w == 8 || seg == 512) ? launch_w<8>(p, X, Y, a, grid, smem, seg, s)
                                         : launch_w<16>(p, X, Y, a, grid, smem, seg, s);
}

}  // namespace sk
