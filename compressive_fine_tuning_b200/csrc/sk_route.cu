// Task routing for the tensor-core kernels ("SpaLLM: Unified Compressive
// Adaptation of LLMs with Sketching", section 2.3: several LUT sets share one
// index map; every token uses its own task's set).
//
// The tensor-core tiles need one LUT set per tile, so the tokens are bucketed
// by task first:
//   * route_kernel (one CTA) counts the tokens of every task, lays the tasks'
//     segments out back to back, writes the permutation perm[position] = token
//     and the tile list (task, first position, length) with at most N tokens
//     per tile; tokens with an out-of-range task id are left out, flagged in
//     the check word and get a zero output row;
//   * gather_kernel copies the input rows (X for the forward, dY for the input
//     gradient) into segment order.
// The product kernel then runs over the tiles and scatters each output row
// back to its token.  A token's output does not depend on which other tokens
// share its tile, so the order inside a segment does not matter.
#include "sk_internal.cuh"

namespace sk {
namespace {

constexpr int kRouteThreads = 1024;

// workspace layout (4-byte words): perm[T] | tiles[max_tiles * 3] | valid[1], then X_perm (16-byte aligned)
__global__ void __launch_bounds__(kRouteThreads) route_kernel(const int32_t* __restrict__ task, int T, int ntask, int N,
                                                              int* __restrict__ perm, int* __restrict__ tiles,
                                                              int max_tiles, int* __restrict__ valid,
                                                              uint16_t* __restrict__ Y, int64_t n, unsigned int* check) {
  __shared__ int cnt[kMaxRouteTasks], off[kMaxRouteTasks + 1], cur[kMaxRouteTasks];
  for (int i = threadIdx.x; i < ntask; i += kRouteThreads) {
    cnt[i] = 0;
    cur[i] = 0;
  }
  __syncthreads();
  for (int t = threadIdx.x; t < T; t += kRouteThreads) {
    const int tau = task[t];
    if (tau >= 0 && tau < ntask) {
      atomicAdd(&cnt[tau], 1);
    } else {
      atomicOr(check, SK_CHECK_TASK_RANGE);
      for (int64_t i = 0; i < n; ++i) Y[(int64_t)t * n + i] = 0;  // rare: flagged tokens get zeros
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0, nt = 0;
    for (int tau = 0; tau < ntask; ++tau) {
      off[tau] = acc;
      for (int k = 0; k < cnt[tau]; k += N) {
        tiles[3 * nt + 0] = tau;
        tiles[3 * nt + 1] = acc + k;
        tiles[3 * nt + 2] = cnt[tau] - k < N ? cnt[tau] - k : N;
        ++nt;
      }
      acc += cnt[tau];
    }
    off[ntask] = acc;
    *valid = acc;
    for (; nt < max_tiles; ++nt) {
      tiles[3 * nt + 0] = 0;
      tiles[3 * nt + 1] = 0;
      tiles[3 * nt + 2] = 0;  // empty tile: its CTAs exit at once
    }
  }
  __syncthreads();
  for (int t = threadIdx.x; t < T; t += kRouteThreads) {
    const int tau = task[t];
    if (tau >= 0 && tau < ntask) perm[off[tau] + atomicAdd(&cur[tau], 1)] = t;
  }
}

__global__ void gather_kernel(const uint4* __restrict__ X, const int* __restrict__ perm, const int* __restrict__ valid,
                              int T, int64_t units, uint4* __restrict__ Xp) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (int64_t)T * units) return;
  const int64_t p = e / units, u = e % units;
  if (p >= *valid) return;
  Xp[e] = __ldg(X + (int64_t)perm[p] * units + u);
}

// Padded routing for the LUT gradient, whose K dimension is the tokens: the
// segment of task tau starts at a multiple of `pad` positions and is padded
// with empty positions (perm = -1, zero rows after the gather) up to the next
// multiple, so a K step of `pad` tokens never mixes two tasks.  segs[2 tau] =
// first position, segs[2 tau + 1] = token count.
__global__ void __launch_bounds__(kRouteThreads) route_pad_kernel(const int32_t* __restrict__ task, int T, int ntask,
                                                                  int pad, int T_pad, int* __restrict__ perm,
                                                                  int* __restrict__ segs, unsigned int* check) {
  __shared__ int cnt[kMaxRouteTasks], off[kMaxRouteTasks], cur[kMaxRouteTasks];
  for (int i = threadIdx.x; i < ntask; i += kRouteThreads) {
    cnt[i] = 0;
    cur[i] = 0;
  }
  for (int p = threadIdx.x; p < T_pad; p += kRouteThreads) perm[p] = -1;
  __syncthreads();
  for (int t = threadIdx.x; t < T; t += kRouteThreads) {
    const int tau = task[t];
    if (tau >= 0 && tau < ntask) atomicAdd(&cnt[tau], 1);
    else atomicOr(check, SK_CHECK_TASK_RANGE);   // left out of every LUT set's gradient
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int tau = 0; tau < ntask; ++tau) {
      off[tau] = acc;
      segs[2 * tau] = acc;
      segs[2 * tau + 1] = cnt[tau];
      acc += (cnt[tau] + pad - 1) / pad * pad;
    }
  }
  __syncthreads();
  for (int t = threadIdx.x; t < T; t += kRouteThreads) {
    const int tau = task[t];
    if (tau >= 0 && tau < ntask) perm[off[tau] + atomicAdd(&cur[tau], 1)] = t;
  }
}

__global__ void gather_pad_kernel(const uint4* __restrict__ src, const int* __restrict__ perm, int T_pad, int64_t units,
                                  uint4* __restrict__ dst) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (int64_t)T_pad * units) return;
  const int64_t p = e / units, u = e % units;
  const int t = perm[p];
  dst[e] = t >= 0 ? __ldg(src + (int64_t)t * units + u) : make_uint4(0u, 0u, 0u, 0u);
}

}  // namespace

int route_pad_positions(int64_t T, int ntask, int pad) { return (int)(T + (int64_t)ntask * (pad - 1)); }

size_t route_pad_workspace_bytes(int64_t T, int64_t width_a, int64_t width_b, int ntask, int pad) {
  const int64_t tp = route_pad_positions(T, ntask, pad);
  const size_t head = ((size_t)tp + 2 * (size_t)ntask) * 4;
  return (head + 255) / 256 * 256 + (size_t)tp * (width_a + width_b) * 2;
}

cudaError_t launch_route_padded(const Problem& p, const uint16_t* a, int64_t width_a, const uint16_t* b,
                                int64_t width_b, int pad, void* workspace, RoutedPad* out, cudaStream_t s) {
  const int tp = route_pad_positions(p.T, p.ntask, pad);
  int* perm = static_cast<int*>(workspace);
  int* segs = perm + tp;
  const size_t head = (((size_t)tp + 2 * (size_t)p.ntask) * 4 + 255) / 256 * 256;
  uint16_t* ap = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(workspace) + head);
  uint16_t* bp = ap + (size_t)tp * width_a;
  route_pad_kernel<<<1, kRouteThreads, 0, s>>>(p.task, (int)p.T, p.ntask, pad, tp, perm, segs, p.check);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  for (int k = 0; k < 2; ++k) {
    const int64_t units = (k ? width_b : width_a) / 8, total = (int64_t)tp * units;
    gather_pad_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(
        reinterpret_cast<const uint4*>(k ? b : a), perm, tp, units, reinterpret_cast<uint4*>(k ? bp : ap));
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  out->segs = segs;
  out->positions = tp;
  out->a = ap;
  out->b = bp;
  return cudaSuccess;
}

int route_max_tiles(int64_t T, int ntask, int N) { return (int)((T + N - 1) / N) + ntask; }

size_t route_workspace_bytes(int64_t T, int64_t d, int ntask, int N) {
  const size_t words = (size_t)T + 3 * (size_t)route_max_tiles(T, ntask, N) + 1;
  const size_t head = (words * 4 + 255) / 256 * 256;
  return head + (size_t)T * d * 2;
}

cudaError_t launch_route(const Problem& p, const uint16_t* src, int64_t src_width, uint16_t* out_rows,
                         int64_t out_width, int N, void* workspace, Routed* out, cudaStream_t s) {
  const int max_tiles = route_max_tiles(p.T, p.ntask, N);
  int* perm = static_cast<int*>(workspace);
  int* tiles = perm + p.T;
  int* valid = tiles + 3 * max_tiles;
  const size_t words = (size_t)p.T + 3 * (size_t)max_tiles + 1;
  uint16_t* Xp = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(workspace) + (words * 4 + 255) / 256 * 256);
  route_kernel<<<1, kRouteThreads, 0, s>>>(p.task, (int)p.T, p.ntask, N, perm, tiles, max_tiles, valid, out_rows,
                                           out_width, p.check);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t units = src_width / 8;
  const int64_t total = p.T * units;
  gather_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(reinterpret_cast<const uint4*>(src), perm, valid,
                                                                (int)p.T, units, reinterpret_cast<uint4*>(Xp));
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  out->perm = perm;
  out->tiles = tiles;
  out->max_tiles = max_tiles;
  out->Xp = Xp;
  return cudaSuccess;
}

}  // namespace sk
