// Internal device helpers shared by the sketched-linear kernels.
//
// Dequantisation ("SpaLLM: Unified Compressive Adaptation of LLMs with
// Sketching", section 2.2, Eq. 1 with groups per row): the weight at
// (row i, column j) is the LUT entry of row i, group j / gs, selected by the
// index idx[i][j].  Every kernel works on 32-column chunks; because
// gs % 32 == 0 a chunk never crosses a group boundary, so one set of LUT
// registers serves the whole chunk.
//
// LUT lookups run on the integer ALUs with byte permutes instead of shared
// memory gathers: the k bf16 entries of one (row, group) table are split into
// a plane of low bytes and a plane of high bytes held in registers, and
// `prmt` selects four bytes per instruction with the packed indices as its
// selector nibbles.  The output is bf16x2 words holding adjacent columns
// (even column in the low half), which is the operand layout the tensor cores
// and the packed stores want.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "sk.h"

namespace sk {

// ----------------------------------------------------------------------------
// small PTX wrappers
// ----------------------------------------------------------------------------

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// acc += w * x with bf16 inputs and an fp32 accumulator (one rounding).
__device__ __forceinline__ float fma_bf16_lo(uint32_t w2, uint32_t x2, float acc) {
  asm("{\n\t.reg .b16 wl, wh, xl, xh;\n\t"
      "mov.b32 {wl, wh}, %1;\n\t"
      "mov.b32 {xl, xh}, %2;\n\t"
      "fma.rn.f32.bf16 %0, wl, xl, %0;\n\t}"
      : "+f"(acc) : "r"(w2), "r"(x2));
  return acc;
}

// acc += w.lo * x.lo + w.hi * x.hi (two fp32 roundings).
__device__ __forceinline__ float fma_bf16x2(uint32_t w2, uint32_t x2, float acc) {
  asm("{\n\t.reg .b16 wl, wh, xl, xh;\n\t"
      "mov.b32 {wl, wh}, %1;\n\t"
      "mov.b32 {xl, xh}, %2;\n\t"
      "fma.rn.f32.bf16 %0, wl, xl, %0;\n\t"
      "fma.rn.f32.bf16 %0, wh, xh, %0;\n\t}"
      : "+f"(acc) : "r"(w2), "r"(x2));
  return acc;
}

// acc_lo += w.lo * s and acc_hi += w.hi * s, with s the bf16 in the low half of s2.
__device__ __forceinline__ void fma_bf16x2_scalar(uint32_t w2, uint32_t s2, float& acc_lo, float& acc_hi) {
  asm("{\n\t.reg .b16 wl, wh, sl, sh;\n\t"
      "mov.b32 {wl, wh}, %2;\n\t"
      "mov.b32 {sl, sh}, %3;\n\t"
      "fma.rn.f32.bf16 %0, wl, sl, %0;\n\t"
      "fma.rn.f32.bf16 %1, wh, sl, %1;\n\t}"
      : "+f"(acc_lo), "+f"(acc_hi) : "r"(w2), "r"(s2));
}

__device__ __forceinline__ float bf16_lo_to_f32(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi_to_f32(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t f32x2_to_bf16x2(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&b);
}

// two fp16 values (one 32-bit word) -> the RNE bf16 of each, same positions
__device__ __forceinline__ uint32_t h2_to_bf2(uint32_t h2) {
  __half2 h = *reinterpret_cast<__half2*>(&h2);
  float2 f = __half22float2(h);
  return f32x2_to_bf16x2(f.x, f.y);
}

// ----------------------------------------------------------------------------
// LUT byte planes
// ----------------------------------------------------------------------------

template <int BITS>
struct LutRegs {
  static constexpr int K = 1 << BITS;
  static constexpr int W = (K + 3) / 4;  // words per plane
  uint32_t lo[W], hi[W];
};

// Load the k fp16 entries at `p` (16-byte aligned for k >= 8, 8-byte for k = 4)
// and build the low/high byte planes of their bf16 roundings.
template <int BITS>
__device__ __forceinline__ void load_lut(const uint16_t* __restrict__ p, LutRegs<BITS>& L) {
  if constexpr (BITS == 4) {
    uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
    uint4 b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
    uint32_t w[8] = {h2_to_bf2(a.x), h2_to_bf2(a.y), h2_to_bf2(a.z), h2_to_bf2(a.w),
                     h2_to_bf2(b.x), h2_to_bf2(b.y), h2_to_bf2(b.z), h2_to_bf2(b.w)};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      L.lo[q] = prmt(w[2 * q], w[2 * q + 1], 0x6420);
      L.hi[q] = prmt(w[2 * q], w[2 * q + 1], 0x7531);
    }
  } else if constexpr (BITS == 3) {
    uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
    uint32_t w[4] = {h2_to_bf2(a.x), h2_to_bf2(a.y), h2_to_bf2(a.z), h2_to_bf2(a.w)};
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      L.lo[q] = prmt(w[2 * q], w[2 * q + 1], 0x6420);
      L.hi[q] = prmt(w[2 * q], w[2 * q + 1], 0x7531);
    }
  } else {
    uint2 a = __ldg(reinterpret_cast<const uint2*>(p));
    uint32_t w0 = h2_to_bf2(a.x), w1 = h2_to_bf2(a.y);
    L.lo[0] = prmt(w0, w1, 0x6420);
    L.hi[0] = prmt(w0, w1, 0x7531);
  }
}

// Raw fp16 words of one table, fetched ahead of time; `to_lut` converts them.
template <int BITS>
struct LutRaw {
  uint4 a, b;
};

template <int BITS>
__device__ __forceinline__ void fetch_lut(const uint16_t* __restrict__ p, LutRaw<BITS>& r) {
  if constexpr (BITS == 4) {
    r.a = __ldg(reinterpret_cast<const uint4*>(p));
    r.b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
  } else if constexpr (BITS == 3) {
    r.a = __ldg(reinterpret_cast<const uint4*>(p));
  } else {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
    r.a = make_uint4(v.x, v.y, 0u, 0u);
  }
}

template <int BITS>
__device__ __forceinline__ void to_lut(const LutRaw<BITS>& r, LutRegs<BITS>& L) {
  if constexpr (BITS == 4) {
    uint32_t w[8] = {h2_to_bf2(r.a.x), h2_to_bf2(r.a.y), h2_to_bf2(r.a.z), h2_to_bf2(r.a.w),
                     h2_to_bf2(r.b.x), h2_to_bf2(r.b.y), h2_to_bf2(r.b.z), h2_to_bf2(r.b.w)};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      L.lo[q] = prmt(w[2 * q], w[2 * q + 1], 0x6420);
      L.hi[q] = prmt(w[2 * q], w[2 * q + 1], 0x7531);
    }
  } else if constexpr (BITS == 3) {
    uint32_t w[4] = {h2_to_bf2(r.a.x), h2_to_bf2(r.a.y), h2_to_bf2(r.a.z), h2_to_bf2(r.a.w)};
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      L.lo[q] = prmt(w[2 * q], w[2 * q + 1], 0x6420);
      L.hi[q] = prmt(w[2 * q], w[2 * q + 1], 0x7531);
    }
  } else {
    const uint32_t w0 = h2_to_bf2(r.a.x), w1 = h2_to_bf2(r.a.y);
    L.lo[0] = prmt(w0, w1, 0x6420);
    L.hi[0] = prmt(w0, w1, 0x7531);
  }
}

// ----------------------------------------------------------------------------
// packed chunks of 32 indices
// ----------------------------------------------------------------------------

template <int BITS>
struct ChunkBytes { static constexpr int value = 4 * BITS; };  // 16 / 12 / 8 bytes

template <int BITS>
struct Chunk { uint32_t w[BITS]; };  // 4, 3 or 2 little-endian words

template <int BITS>
__device__ __forceinline__ Chunk<BITS> load_chunk(const uint8_t* __restrict__ row, int64_t c) {
  Chunk<BITS> ch;
  const uint8_t* p = row + c * ChunkBytes<BITS>::value;
  if constexpr (BITS == 4) {
    uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
    ch.w[0] = v.x; ch.w[1] = v.y; ch.w[2] = v.z; ch.w[3] = v.w;
  } else if constexpr (BITS == 2) {
    uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
    ch.w[0] = v.x; ch.w[1] = v.y;
  } else {
    const uint32_t* q = reinterpret_cast<const uint32_t*>(p);
    ch.w[0] = __ldg(q); ch.w[1] = __ldg(q + 1); ch.w[2] = __ldg(q + 2);
  }
  return ch;
}

// 32 indices -> 16 bf16x2 words (word p = columns 2p, 2p+1).
template <int BITS>
__device__ __forceinline__ void dequant_chunk(const Chunk<BITS>& ch, const LutRegs<BITS>& L, uint32_t out[16]);

template <>
__device__ __forceinline__ void dequant_chunk<4>(const Chunk<4>& ch, const LutRegs<4>& L, uint32_t out[16]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t w = ch.w[q];                       // columns 8q .. 8q+7, one nibble each
    uint32_t sel = w & 0x77777777u;                   // low three bits pick a byte in a half table
    uint32_t mrg = ((w >> 1) & 0x44444444u) | 0x32103210u;  // bit 3 picks the half table
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t s = h ? (sel >> 16) : sel;
      const uint32_t m = h ? (mrg >> 16) : mrg;
      uint32_t lo = prmt(prmt(L.lo[0], L.lo[1], s), prmt(L.lo[2], L.lo[3], s), m);
      uint32_t hi = prmt(prmt(L.hi[0], L.hi[1], s), prmt(L.hi[2], L.hi[3], s), m);
      out[4 * q + 2 * h + 0] = prmt(lo, hi, 0x5140);
      out[4 * q + 2 * h + 1] = prmt(lo, hi, 0x7362);
    }
  }
}

template <>
__device__ __forceinline__ void dequant_chunk<2>(const Chunk<2>& ch, const LutRegs<2>& L, uint32_t out[16]) {
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const uint32_t w = ch.w[q];                       // columns 16q .. 16q+15, two bits each
    const uint32_t sa = w & 0x33333333u;              // columns 4m and 4m+2 of byte m, as nibbles
    const uint32_t sb = (w >> 2) & 0x33333333u;       // columns 4m+1 and 4m+3
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t a = h ? (sa >> 16) : sa;
      const uint32_t b = h ? (sb >> 16) : sb;
      uint32_t lo_e = prmt(L.lo[0], L.lo[0], a), hi_e = prmt(L.hi[0], L.hi[0], a);
      uint32_t lo_o = prmt(L.lo[0], L.lo[0], b), hi_o = prmt(L.hi[0], L.hi[0], b);
      uint32_t e0 = prmt(lo_e, hi_e, 0x5140), e1 = prmt(lo_e, hi_e, 0x7362);  // (c0,c2), (c4,c6)
      uint32_t o0 = prmt(lo_o, hi_o, 0x5140), o1 = prmt(lo_o, hi_o, 0x7362);  // (c1,c3), (c5,c7)
      uint32_t* o = out + 8 * q + 4 * h;
      o[0] = prmt(e0, o0, 0x5410);
      o[1] = prmt(e0, o0, 0x7632);
      o[2] = prmt(e1, o1, 0x5410);
      o[3] = prmt(e1, o1, 0x7632);
    }
  }
}

// Eight 3-bit fields (bits 0..23) -> eight nibbles.
__device__ __forceinline__ uint32_t spread3(uint32_t g) {
  uint32_t y = (g & 0xFFFu) | ((g << 4) & 0x0FFF0000u);
  uint32_t z = (y & 0x003F003Fu) | ((y << 2) & 0x3F003F00u);
  return (z & 0x07070707u) | ((z << 1) & 0x70707070u);
}

template <>
__device__ __forceinline__ void dequant_chunk<3>(const Chunk<3>& ch, const LutRegs<3>& L, uint32_t out[16]) {
  uint32_t g[4];
  g[0] = ch.w[0];
  g[1] = __funnelshift_r(ch.w[0], ch.w[1], 24);
  g[2] = __funnelshift_r(ch.w[1], ch.w[2], 16);
  g[3] = ch.w[2] >> 8;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t r = spread3(g[q]);                 // columns 8q .. 8q+7 as nibbles 0..7
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t s = h ? (r >> 16) : r;
      uint32_t lo = prmt(L.lo[0], L.lo[1], s);
      uint32_t hi = prmt(L.hi[0], L.hi[1], s);
      out[4 * q + 2 * h + 0] = prmt(lo, hi, 0x5140);
      out[4 * q + 2 * h + 1] = prmt(lo, hi, 0x7362);
    }
  }
}

// Index of column e (0..31) of a chunk, as an integer.
template <int BITS>
__device__ __forceinline__ uint32_t chunk_index(const Chunk<BITS>& ch, int e) {
  const int bit = e * BITS;
  const int w = bit >> 5, s = bit & 31;
  uint32_t v = ch.w[w] >> s;
  if (BITS == 3 && s > 29) v |= ch.w[w + 1] << (32 - s);
  return v & ((1u << BITS) - 1u);
}

// ----------------------------------------------------------------------------
// launch plumbing shared by the kernel files
// ----------------------------------------------------------------------------

struct Problem {
  const uint8_t* packed;   // [n][row_bytes]
  int64_t row_bytes;
  const uint16_t* lut;     // fp16 [ntask][n][gpr][k]
  int bits, gpr;
  int64_t n, d, gs;        // gs = d / gpr, a multiple of 32
  int64_t T;
  const int32_t* task;     // [T] or nullptr
  int ntask;
  unsigned int* check;     // device check word
};

__device__ __forceinline__ int token_task(const int32_t* task, int64_t t, int ntask, unsigned int* check) {
  if (task == nullptr) return 0;
  int tau = __ldg(task + t);
  if (tau < 0 || tau >= ntask) {
    atomicOr(check, SK_CHECK_TASK_RANGE);
    return -1;
  }
  return tau;
}

__device__ __forceinline__ const uint16_t* lut_ptr(const Problem& p, int tau, int64_t i, int64_t g) {
  return p.lut + (((int64_t)tau * p.n + i) * p.gpr + g) * (1 << p.bits);
}

// Task routing for the tensor-core forward (sk_route.cu).
constexpr int kMaxRouteTasks = 256;
struct Routed {
  const int* perm;   // [T] position in task order -> token
  const int* tiles;  // [max_tiles][3] (task, first position, length); length 0 = empty
  int max_tiles;
  const uint16_t* Xp;  // [T][d] X rows in task order
};
int route_max_tiles(int64_t T, int ntask, int N);
size_t route_workspace_bytes(int64_t T, int64_t d, int ntask, int N);
// Routes the tokens by task (tiles of at most N tokens) and gathers the rows
// of `src` (src_width bf16 each) into task order; out_rows (out_width each)
// gets zero rows for tokens with an out-of-range task id.
cudaError_t launch_route(const Problem& p, const uint16_t* src, int64_t src_width, uint16_t* out_rows,
                         int64_t out_width, int N, void* workspace, Routed* out, cudaStream_t s);
// Padded routing for the LUT gradient: task segments start at multiples of
// `pad` positions (empty positions hold zero rows); two inputs gathered.
struct RoutedPad {
  const int* segs;     // [ntask][2]: first position, token count
  int positions;       // rows of the gathered inputs
  const uint16_t* a;   // [positions][width_a]
  const uint16_t* b;   // [positions][width_b]
};
int route_pad_positions(int64_t T, int ntask, int pad);
size_t route_pad_workspace_bytes(int64_t T, int64_t width_a, int64_t width_b, int ntask, int pad);
cudaError_t launch_route_padded(const Problem& p, const uint16_t* a, int64_t width_a, const uint16_t* b,
                                int64_t width_b, int pad, void* workspace, RoutedPad* out, cudaStream_t s);
// Token tile of the tensor-core forward for a batch of T tokens spread over
// ntask LUT sets (16 ... 256).
int fwd_tc_tile_n(int64_t T, int ntask);
size_t fwd_tc_workspace(int64_t T, int64_t d, int ntask);
cudaError_t launch_fwd_tc_routed(const Problem& p, const uint16_t* X, uint16_t* Y, void* workspace, cudaStream_t s);

// Host-side knobs read from the environment (experiments and tests).
int env_int(const char* name, int dflt);
// Programmatic dependent launch for the forward kernels (SK_PDL=0 turns it off).
bool pdl_enabled();

// Host-side launchers (one per kernel file).  They return cudaGetLastError().
cudaError_t launch_pack(const uint8_t* idx, int64_t n, int64_t d, int bits, uint8_t* packed,
                        int64_t row_bytes, unsigned int* check, cudaStream_t s);
cudaError_t launch_unpack(const uint8_t* packed, int64_t n, int64_t d, int bits, int64_t row_bytes,
                          uint8_t* idx, cudaStream_t s);
cudaError_t launch_dequant(const Problem& p, int task, uint16_t* theta, cudaStream_t s);
cudaError_t launch_gemv_fwd(const Problem& p, const uint16_t* X, uint16_t* Y, cudaStream_t s);
// Decode forward (4-bit, single LUT set, 1 <= T <= 16, d >= 256) on mma.sync.
bool decode_fwd_supported(const Problem& p);
cudaError_t launch_decode_fwd(const Problem& p, const uint16_t* X, uint16_t* Y, cudaStream_t s);
// The same for a group of layers with one token batch size, in one launch.
constexpr int kMaxDecodeGroup = 8;
struct DecodeLayer {
  const uint8_t* packed;   // [n][row_bytes], 4-bit
  int64_t row_bytes;
  const uint16_t* lut;     // fp16 [ntask][n][gpr][16]
  int gpr;
  int64_t n, d;
  const uint16_t* X;       // bf16 [T][d]
  uint16_t* Y;             // bf16 [T][n]
};
bool decode_group_supported(const DecodeLayer* layers, int nl, int T, const int32_t* task, int ntask);
cudaError_t launch_decode_group(const DecodeLayer* layers, int nl, int T, const int32_t* task, int ntask,
                                unsigned int* check, cudaStream_t s);
cudaError_t launch_fwd_tc(const Problem& p, const uint16_t* X, uint16_t* Y, cudaStream_t s);
cudaError_t launch_dx_tc(const Problem& p, const uint16_t* dY, uint16_t* dX, cudaStream_t s);
// dX for a batch with several LUT sets: tokens routed by task (workspace of
// dx_tc_workspace bytes), one LUT set per 256-token tile.
size_t dx_tc_workspace(int64_t T, int64_t n, int ntask);
cudaError_t launch_dx_tc_routed(const Problem& p, const uint16_t* dY, uint16_t* dX, void* workspace, cudaStream_t s);
cudaError_t launch_dlut_tc(const Problem& p, const uint16_t* X, const uint16_t* dY, float* dlut, int accumulate,
                           void* workspace, cudaStream_t s);
size_t dlut_tc_workspace(int64_t n, int64_t d, int bits, int gpr);
// LUT gradient for a batch with several LUT sets: tokens routed by task into
// 64-token-aligned segments, one K range per task.
size_t dlut_tc_routed_workspace(int64_t n, int64_t d, int bits, int gpr, int64_t T, int ntask);
cudaError_t launch_dlut_tc_routed(const Problem& p, const uint16_t* X, const uint16_t* dY, float* dlut, int accumulate,
                                  void* workspace, cudaStream_t s);
size_t dlut_noalloc_scratch_bytes();
cudaError_t dlut_noalloc_scratch(void** ptr);
cudaError_t launch_bin_counts(const uint8_t* packed, int64_t row_bytes, int bits, int64_t n, int gpr, int64_t gs,
                              int32_t* counts, cudaStream_t s);
cudaError_t launch_adamw(float* master, float* m, float* v, const float* grad, const int32_t* counts, int64_t total,
                         int64_t per_set, float lr, float beta1, float beta2, float eps, float weight_decay, int step,
                         uint16_t* lut, cudaStream_t s);
cudaError_t launch_sgd(float* master, const float* grad, const int32_t* counts, int64_t total, int64_t per_set,
                       float lr, uint16_t* lut, cudaStream_t s);
cudaError_t launch_simt_bwd_input(const Problem& p, const uint16_t* dY, uint16_t* dX, cudaStream_t s);
cudaError_t launch_simt_bwd_lut(const Problem& p, const uint16_t* X, const uint16_t* dY, float* dlut,
                                int accumulate, cudaStream_t s);

}  // namespace sk
