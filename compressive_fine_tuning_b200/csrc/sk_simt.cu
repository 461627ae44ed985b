// Backward products on the CUDA cores, for small token counts (decode-sized
// batches) where a tensor-core tile would be mostly padding.
//
//   dX = dY Theta_hat           (chain rule through the frozen sketch)
//   dlut[i][g][c] = sum_{j in g, idx[i][j] = c} sum_t dY[t][i] X[t][j]
//                               (the corrected Eq. 6 of the "Sketch to Adapt"
//                                OpenReview discussion, reply Q1)
//
// dX: one thread per (32-column chunk, token); it walks all n rows, dequantises
// its chunk of each row and accumulates 32 fp32 sums.  dlut: one warp per
// (row, group); each lane takes chunks of the group, forms their 32 dense
// gradient values dY[:, i]^T X[:, chunk] in fp32 and adds each into the bin
// its index selects, then a shuffle tree sums the lanes' bins.  Bins live in
// shared memory as [k][blockDim] so that the dynamic bin index never causes a
// bank conflict.  No float atomics, fixed reduction order: deterministic.
#include "sk_internal.cuh"

namespace sk {
namespace {

constexpr int kBlock = 128;

template <int BITS>
__global__ void __launch_bounds__(kBlock) simt_bwd_input_kernel(Problem p, const uint16_t* __restrict__ dY,
                                                                uint16_t* __restrict__ dX) {
  const int64_t chunks = p.d / 32;
  const int64_t c = (int64_t)blockIdx.x * kBlock + threadIdx.x;
  if (c >= chunks) return;
  const int64_t g = (c * 32) / p.gs;
  for (int64_t t = blockIdx.y; t < p.T; t += gridDim.y) {
    const int tau = token_task(p.task, t, p.ntask, p.check);
    float acc[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) acc[e] = 0.f;
    if (tau >= 0) {
      for (int64_t i = 0; i < p.n; ++i) {
        LutRegs<BITS> L;
        load_lut<BITS>(lut_ptr(p, tau, i, g), L);
        Chunk<BITS> ch = load_chunk<BITS>(p.packed + i * p.row_bytes, c);
        uint32_t w[16];
        dequant_chunk<BITS>(ch, L, w);
        const uint32_t s2 = __ldg(dY + t * p.n + i);
#pragma unroll
        for (int e2 = 0; e2 < 16; ++e2) fma_bf16x2_scalar(w[e2], s2, acc[2 * e2], acc[2 * e2 + 1]);
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(dX + t * p.d + c * 32);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      dst[q] = make_uint4(f32x2_to_bf16x2(acc[8 * q + 0], acc[8 * q + 1]), f32x2_to_bf16x2(acc[8 * q + 2], acc[8 * q + 3]),
                          f32x2_to_bf16x2(acc[8 * q + 4], acc[8 * q + 5]), f32x2_to_bf16x2(acc[8 * q + 6], acc[8 * q + 7]));
    }
  }
}

template <int BITS>
__global__ void __launch_bounds__(kBlock) simt_bwd_lut_kernel(Problem p, const uint16_t* __restrict__ X,
                                                              const uint16_t* __restrict__ dY,
                                                              float* __restrict__ dlut, int accumulate) {
  constexpr int K = 1 << BITS;
  __shared__ float bins[K][kBlock];
  const int tid = threadIdx.x, lane = tid & 31;
  const int64_t wid = (int64_t)blockIdx.x * (kBlock / 32) + (tid >> 5);   // one warp per (row, group)
  if (wid >= p.n * p.gpr) return;
  const int64_t i = wid / p.gpr, g = wid % p.gpr;
  const int64_t cpg = p.gs / 32;
  for (int tau = 0; tau < p.ntask; ++tau) {
#pragma unroll
    for (int c = 0; c < K; ++c) bins[c][tid] = 0.f;
    // without task ids every token belongs to LUT set 0; the other sets get zeros
    if (p.task != nullptr || tau == 0) {
      for (int64_t cc = lane; cc < cpg; cc += 32) {
        const int64_t chunk = g * cpg + cc;
        Chunk<BITS> ch = load_chunk<BITS>(p.packed + i * p.row_bytes, chunk);
        float G[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) G[e] = 0.f;
        for (int64_t t = 0; t < p.T; ++t) {
          if (p.task != nullptr && token_task(p.task, t, p.ntask, p.check) != tau) continue;
          const uint32_t s2 = __ldg(dY + t * p.n + i);
          const uint4* xp = reinterpret_cast<const uint4*>(X + t * p.d + chunk * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 xv = __ldg(xp + q);
            fma_bf16x2_scalar(xv.x, s2, G[8 * q + 0], G[8 * q + 1]);
            fma_bf16x2_scalar(xv.y, s2, G[8 * q + 2], G[8 * q + 3]);
            fma_bf16x2_scalar(xv.z, s2, G[8 * q + 4], G[8 * q + 5]);
            fma_bf16x2_scalar(xv.w, s2, G[8 * q + 6], G[8 * q + 7]);
          }
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) bins[chunk_index<BITS>(ch, e)][tid] += G[e];
      }
    }
    // lane partial bins -> the warp's sums (fixed shuffle tree: deterministic)
    float mine = 0.f;
#pragma unroll
    for (int c = 0; c < K; ++c) {
      float v = bins[c][tid];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      if (lane == c) mine = v;
    }
    if (lane < K) {
      float* out = dlut + (((int64_t)tau * p.n + i) * p.gpr + g) * K + lane;
      *out = accumulate ? *out + mine : mine;
    }
  }
}

}  // namespace

cudaError_t launch_simt_bwd_input(const Problem& p, const uint16_t* dY, uint16_t* dX, cudaStream_t s) {
  const int64_t chunks = p.d / 32;
  dim3 grid((unsigned)((chunks + kBlock - 1) / kBlock), (unsigned)(p.T < 65535 ? p.T : 65535));
  switch (p.bits) {
    case 2: simt_bwd_input_kernel<2><<<grid, kBlock, 0, s>>>(p, dY, dX); break;
    case 3: simt_bwd_input_kernel<3><<<grid, kBlock, 0, s>>>(p, dY, dX); break;
    default: simt_bwd_input_kernel<4><<<grid, kBlock, 0, s>>>(p, dY, dX); break;
  }
  return cudaGetLastError();
}

cudaError_t launch_simt_bwd_lut(const Problem& p, const uint16_t* X, const uint16_t* dY, float* dlut,
                                int accumulate, cudaStream_t s) {
  const int64_t warps = p.n * p.gpr;
  const unsigned grid = (unsigned)((warps + kBlock / 32 - 1) / (kBlock / 32));
  switch (p.bits) {
    case 2: simt_bwd_lut_kernel<2><<<grid, kBlock, 0, s>>>(p, X, dY, dlut, accumulate); break;
    case 3: simt_bwd_lut_kernel<3><<<grid, kBlock, 0, s>>>(p, X, dY, dlut, accumulate); break;
    default: simt_bwd_lut_kernel<4><<<grid, kBlock, 0, s>>>(p, X, dY, dlut, accumulate); break;
  }
  return cudaGetLastError();
}

}  // namespace sk
