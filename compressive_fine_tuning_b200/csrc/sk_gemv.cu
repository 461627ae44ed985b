// Decode forward on the CUDA cores: Y[t][i] = sum_j X[t][j] * Theta_hat[i][j]
// for a handful of tokens ("SpaLLM: Unified Compressive Adaptation of LLMs
// with Sketching", section 2.3: one compressed matmul per layer; section 3.2,
// Table 5: decode is where the single-tower layer pays off).
//
// Work split: a warp owns R weight rows and splits their columns across its
// lanes; each lane walks 32-column chunks (one 16/8/12-byte index load per
// chunk, consecutive lanes on consecutive chunks so a warp-wide load is one
// contiguous span of the row), dequantises them through register LUTs
// and accumulates R x TT fp32 dot products with bf16 x fp32 fused multiply-adds.
// A warp-shuffle tree then reduces the lane partial sums.  Tokens are taken TT
// at a time; tokens with different LUT sets re-dequantise the chunk.
#include "sk_internal.cuh"

namespace sk {
namespace {

constexpr int kWarps = 4;

template <int BITS, int R, int TT>
__global__ void __launch_bounds__(kWarps * 32) gemv_fwd_kernel(Problem p, const uint16_t* __restrict__ X,
                                                               uint16_t* __restrict__ Y) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");  // inputs may come from the previous launch
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row0 = ((int64_t)blockIdx.x * kWarps + warp) * R;
  if (row0 >= p.n) return;
  const int64_t chunks = p.d / 32;
  const int64_t cpg = p.gs / 32;
  const uint8_t* rows[R];
#pragma unroll
  for (int r = 0; r < R; ++r) rows[r] = p.packed + (row0 + r < p.n ? row0 + r : p.n - 1) * p.row_bytes;

  for (int64_t t0 = 0; t0 < p.T; t0 += TT) {
    const int nt = (int)(p.T - t0 < TT ? p.T - t0 : TT);
    int taus[TT];
#pragma unroll
    for (int u = 0; u < TT; ++u) taus[u] = (u < nt) ? token_task(p.task, t0 + u, p.ntask, p.check) : -1;

    float acc[R][TT];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int u = 0; u < TT; ++u) acc[r][u] = 0.f;

    const int cpg32 = (int)cpg;
    int g = lane / cpg32, g_next = (g + 1) * cpg32;   // chunk group, advanced without divisions
    for (int c = lane; c < (int)chunks; c += 32) {
      while (c >= g_next) { ++g; g_next += cpg32; }
      Chunk<BITS> ch[R];
#pragma unroll
      for (int r = 0; r < R; ++r) ch[r] = load_chunk<BITS>(rows[r], c);
      uint32_t w[R][16];
      int cur = -2;
#pragma unroll
      for (int u = 0; u < TT; ++u) {
        if (taus[u] < 0) continue;
        if (taus[u] != cur) {
          cur = taus[u];
#pragma unroll
          for (int r = 0; r < R; ++r) {
            LutRegs<BITS> L;
            load_lut<BITS>(lut_ptr(p, cur, (row0 + r < p.n ? row0 + r : p.n - 1), g), L);
            dequant_chunk<BITS>(ch[r], L, w[r]);
          }
        }
        const uint4* xp = reinterpret_cast<const uint4*>(X + (t0 + u) * p.d + c * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 xv = __ldg(xp + q);
#pragma unroll
          for (int r = 0; r < R; ++r) {
            float a = acc[r][u];
            a = fma_bf16x2(w[r][4 * q + 0], xv.x, a);
            a = fma_bf16x2(w[r][4 * q + 1], xv.y, a);
            a = fma_bf16x2(w[r][4 * q + 2], xv.z, a);
            a = fma_bf16x2(w[r][4 * q + 3], xv.w, a);
            acc[r][u] = a;
          }
        }
      }
    }

#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
      for (int u = 0; u < TT; ++u) {
        float v = acc[r][u];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        acc[r][u] = v;
      }
    }
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if (row0 + r >= p.n) continue;
#pragma unroll
        for (int u = 0; u < TT; ++u) {
          if (u >= nt) continue;
          __nv_bfloat16 b = __float2bfloat16_rn(acc[r][u]);
          Y[(t0 + u) * p.n + row0 + r] = *reinterpret_cast<uint16_t*>(&b);
        }
      }
    }
  }
}

// Single-LUT-set decode (T <= 4): each lane takes a contiguous run of chunks
// of its warp's rows, so a lane loads its rows' group tables once and keeps
// four chunks per row in flight; the lane partial sums meet in a warp-shuffle
// tree.  Nothing in the loop divides.
// X staged in shared memory (XS): 16-byte unit u of token t's row is stored at
// u ^ ((u >> 4) & 7), so the lanes of a warp, which read X 256 bytes apart
// (4 chunks each), hit eight different bank groups.  The XOR only changes the
// low three bits, so rows are padded to a multiple of 8 units.
__device__ __forceinline__ uint32_t xs_unit(uint32_t u) { return u ^ ((u >> 4) & 7u); }

template <int BITS, int R, int TT, bool XS>
__global__ void __launch_bounds__(kWarps * 32) gemv_fwd_single_kernel(Problem p, const uint16_t* __restrict__ X,
                                                                      uint16_t* __restrict__ Y) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");  // inputs may come from the previous launch
  extern __shared__ uint4 xs[];                       // [T][units_pad] 16-byte units (XS only)
  const uint32_t units = (uint32_t)(p.d / 8), units_pad = (units + 7u) & ~7u;
  if constexpr (XS) {
    for (uint32_t e = threadIdx.x; e < (uint32_t)p.T * units; e += kWarps * 32) {
      const uint32_t t = e / units, u = e % units;
      xs[t * units_pad + xs_unit(u)] = __ldg(reinterpret_cast<const uint4*>(X) + e);
    }
    __syncthreads();
  }
  constexpr int PF = 4;                               // chunks per row loaded per batch
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row0 = ((int64_t)blockIdx.x * kWarps + warp) * R;
  if (row0 >= p.n) return;
  const int C = (int)(p.d / 32), cpg = (int)(p.gs / 32);
  const int c_begin = (int)(((int64_t)lane * C) / 32), c_end = (int)(((int64_t)(lane + 1) * C) / 32);
  const int T = (int)p.T;
  const uint8_t* rows[R];
  const uint16_t* luts[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int64_t row = row0 + r < p.n ? row0 + r : p.n - 1;
    rows[r] = p.packed + row * p.row_bytes;
    luts[r] = p.lut + row * p.gpr * (1 << BITS);
  }
  int g = c_begin / cpg, g_end = (g + 1) * cpg;
  LutRegs<BITS> L[R];
  LutRaw<BITS> lraw[R];
#pragma unroll
  for (int r = 0; r < R; ++r) fetch_lut<BITS>(luts[r] + (g < p.gpr ? g : p.gpr - 1) * (1 << BITS), lraw[r]);
  float acc[R][TT];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int u = 0; u < TT; ++u) acc[r][u] = 0.f;

  // two batches of PF chunks per row: the next batch's loads are in flight
  // while the current one is dequantised and multiplied
  Chunk<BITS> ch0[PF][R], ch1[PF][R];
  auto load_batch = [&](Chunk<BITS> (&ch)[PF][R], int cb) {
#pragma unroll
    for (int k = 0; k < PF; ++k)
#pragma unroll
      for (int r = 0; r < R; ++r)
        if (cb + k < c_end) ch[k][r] = load_chunk<BITS>(rows[r], cb + k);
  };
  auto process = [&](const Chunk<BITS> (&ch)[PF][R], int cb) {
#pragma unroll
    for (int k = 0; k < PF; ++k) {
      const int c = cb + k;
      if (c >= c_end) break;
      if (c >= g_end) {
        do { ++g; g_end += cpg; } while (c >= g_end);
#pragma unroll
        for (int r = 0; r < R; ++r) load_lut<BITS>(luts[r] + g * (1 << BITS), L[r]);
      }
      uint32_t w[R][16];
#pragma unroll
      for (int r = 0; r < R; ++r) dequant_chunk<BITS>(ch[k][r], L[r], w[r]);
#pragma unroll
      for (int u = 0; u < TT; ++u) {
        if (u >= T) break;
        const uint4* xp = reinterpret_cast<const uint4*>(X + (int64_t)u * p.d + (int64_t)c * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 xv;
          if constexpr (XS) {
            xv = xs[(uint32_t)u * units_pad + xs_unit(4u * (uint32_t)c + q)];
          } else {
            xv = __ldg(xp + q);
          }
#pragma unroll
          for (int r = 0; r < R; ++r) {
            float a = acc[r][u];
            a = fma_bf16x2(w[r][4 * q + 0], xv.x, a);
            a = fma_bf16x2(w[r][4 * q + 1], xv.y, a);
            a = fma_bf16x2(w[r][4 * q + 2], xv.z, a);
            a = fma_bf16x2(w[r][4 * q + 3], xv.w, a);
            acc[r][u] = a;
          }
        }
      }
    }
  };
  // every global load of the first batch is in flight before anything waits on one
  load_batch(ch0, c_begin);
#pragma unroll
  for (int r = 0; r < R; ++r) to_lut<BITS>(lraw[r], L[r]);
  for (int cb = c_begin; cb < c_end; cb += 2 * PF) {
    if (cb + PF < c_end) load_batch(ch1, cb + PF);
    process(ch0, cb);
    if (cb + 2 * PF < c_end) load_batch(ch0, cb + 2 * PF);
    if (cb + PF < c_end) process(ch1, cb + PF);
  }
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int u = 0; u < TT; ++u) {
      float v = acc[r][u];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      acc[r][u] = v;
    }
  if (lane == 0) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (row0 + r >= p.n) continue;
#pragma unroll
      for (int u = 0; u < TT; ++u) {
        if (u >= T) continue;
        __nv_bfloat16 b = __float2bfloat16_rn(acc[r][u]);
        Y[(int64_t)u * p.n + row0 + r] = *reinterpret_cast<uint16_t*>(&b);
      }
    }
  }
}

template <int BITS, int R, int TT>
cudaError_t launch_single(const Problem& p, const uint16_t* X, uint16_t* Y, cudaStream_t s) {
  const int64_t rows_per_cta = (int64_t)kWarps * R;
  const int64_t xs_bytes = p.T * (((p.d / 8) + 7) / 8 * 8) * 16;
  const bool xs = xs_bytes <= 48 * 1024;
  cudaLaunchConfig_t cfg = {};
  cfg.dynamicSmemBytes = xs ? (size_t)xs_bytes : 0;
  cfg.gridDim = dim3((unsigned)((p.n + rows_per_cta - 1) / rows_per_cta), 1, 1);
  cfg.blockDim = dim3(kWarps * 32, 1, 1);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  cudaError_t e = xs ? cudaLaunchKernelEx(&cfg, gemv_fwd_single_kernel<BITS, R, TT, true>, p, X, Y)
                     : cudaLaunchKernelEx(&cfg, gemv_fwd_single_kernel<BITS, R, TT, false>, p, X, Y);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int BITS, int R, int TT>
cudaError_t launch(const Problem& p, const uint16_t* X, uint16_t* Y, cudaStream_t s) {
  const int64_t rows_per_cta = (int64_t)kWarps * R;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((p.n + rows_per_cta - 1) / rows_per_cta), 1, 1);
  cfg.blockDim = dim3(kWarps * 32, 1, 1);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, gemv_fwd_kernel<BITS, R, TT>, p, X, Y);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int BITS>
cudaError_t launch_bits(const Problem& p, const uint16_t* X, uint16_t* Y, cudaStream_t s) {
  const bool single = p.task == nullptr || p.ntask == 1;
  if (single && p.T == 1) return launch_single<BITS, 2, 1>(p, X, Y, s);
  if (single && p.T == 2) return launch_single<BITS, 2, 2>(p, X, Y, s);
  if (single && p.T <= 4) return launch_single<BITS, 2, 4>(p, X, Y, s);
  if (p.T == 1) return launch<BITS, 2, 1>(p, X, Y, s);
  return launch<BITS, 2, 4>(p, X, Y, s);
}

}  // namespace

cudaError_t launch_gemv_fwd(const Problem& p, const uint16_t* X, uint16_t* Y, cudaStream_t s) {
  switch (p.bits) {
    case 2: return launch_bits<2>(p, X, Y, s);
    case 3: return launch_bits<3>(p, X, Y, s);
    default: return launch_bits<4>(p, X, Y, s);
  }
}

}  // namespace sk
