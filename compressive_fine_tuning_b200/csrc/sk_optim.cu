// LUT update of the sketched linear layer: the static bin counts of the index
// map and one optimizer step on the LUT values.
//
// The pages ("SpaLLM: Unified Compressive Adaptation of LLMs with Sketching",
// section 2.1) train only the LUT values and say that the gradients of the
// virtual parameters sharing one value are averaged; the corrected Eq. 6 of
// the "Sketch to Adapt" discussion gives their sum.  The LUT gradient kernels
// return the sum; the averaging variant divides it by the bin size here.  The
// pages name no optimizer: this is plain AdamW (decoupled weight decay) and
// SGD on fp32 master LUTs, which also refresh the fp16 LUTs the layer reads.
//
// These kernels are elementwise and memory-bound (a few bytes per LUT entry,
// ~1.4 M entries for a 7-layer 7B block at 2 bits): grid-stride loops over
// the entries, one thread per entry.
#include <cmath>

#include "sk_tc.cuh"

namespace sk {
namespace {

// counts[i][g][c]: columns of group g in row i whose index is c.  One thread
// per (row, group) walks the group's 32-column chunks.
template <int BITS>
__global__ void bin_counts_kernel(const uint8_t* __restrict__ packed, int64_t row_bytes, int64_t n, int gpr,
                                  int64_t gs, int32_t* __restrict__ counts) {
  constexpr int K = 1 << BITS;
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n * gpr) return;
  const int64_t i = e / gpr, g = e - i * gpr;
  int cnt[K];
#pragma unroll
  for (int c = 0; c < K; ++c) cnt[c] = 0;
  const uint8_t* row = packed + i * row_bytes;
  const int64_t c0 = g * gs / 32, c1 = (g + 1) * gs / 32;
  for (int64_t ch = c0; ch < c1; ++ch) {
    const Chunk<BITS> chunk = load_chunk<BITS>(row, ch);
    for (int j = 0; j < 32; ++j) {
      const uint32_t v = chunk_index<BITS>(chunk, j);
#pragma unroll
      for (int c = 0; c < K; ++c) cnt[c] += (v == (uint32_t)c) ? 1 : 0;
    }
  }
  int32_t* out = counts + e * K;
#pragma unroll
  for (int c = 0; c < K; ++c) out[c] = cnt[c];
}

__device__ __forceinline__ float shared_grad(const float* grad, const int32_t* counts, int64_t e, int64_t per_set) {
  float gv = grad[e];
  if (counts != nullptr) {
    const int32_t c = counts[e % per_set];
    gv = gv / (float)(c > 1 ? c : 1);
  }
  return gv;
}

__global__ void adamw_kernel(float* __restrict__ master, float* __restrict__ m, float* __restrict__ v,
                             const float* __restrict__ grad, const int32_t* __restrict__ counts, int64_t total,
                             int64_t per_set, float lr, float beta1, float beta2, float eps, float decay,
                             float bc1, float bc2, uint16_t* __restrict__ lut) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const float g = shared_grad(grad, counts, e, per_set);
    float p = master[e] * decay;
    const float mm = beta1 * m[e] + (1.f - beta1) * g;
    const float vv = beta2 * v[e] + (1.f - beta2) * g * g;
    p -= lr * (mm / bc1) / (sqrtf(vv / bc2) + eps);
    master[e] = p;
    m[e] = mm;
    v[e] = vv;
    if (lut != nullptr) {
      const __half h = __float2half_rn(p);
      lut[e] = *reinterpret_cast<const uint16_t*>(&h);
    }
  }
}

__global__ void sgd_kernel(float* __restrict__ master, const float* __restrict__ grad,
                           const int32_t* __restrict__ counts, int64_t total, int64_t per_set, float lr,
                           uint16_t* __restrict__ lut) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const float p = master[e] - lr * shared_grad(grad, counts, e, per_set);
    master[e] = p;
    if (lut != nullptr) {
      const __half h = __float2half_rn(p);
      lut[e] = *reinterpret_cast<const uint16_t*>(&h);
    }
  }
}

unsigned elementwise_grid(int64_t total) {
  const int64_t blocks = (total + 255) / 256;
  const int64_t cap = (int64_t)num_sms() * 8;
  return (unsigned)(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

}  // namespace

cudaError_t launch_bin_counts(const uint8_t* packed, int64_t row_bytes, int bits, int64_t n, int gpr, int64_t gs,
                              int32_t* counts, cudaStream_t s) {
  const unsigned grid = (unsigned)((n * gpr + 127) / 128);
  switch (bits) {
    case 2: bin_counts_kernel<2><<<grid, 128, 0, s>>>(packed, row_bytes, n, gpr, gs, counts); break;
    case 3: bin_counts_kernel<3><<<grid, 128, 0, s>>>(packed, row_bytes, n, gpr, gs, counts); break;
    default: bin_counts_kernel<4><<<grid, 128, 0, s>>>(packed, row_bytes, n, gpr, gs, counts); break;
  }
  return cudaGetLastError();
}

cudaError_t launch_adamw(float* master, float* m, float* v, const float* grad, const int32_t* counts, int64_t total,
                         int64_t per_set, float lr, float beta1, float beta2, float eps, float weight_decay, int step,
                         uint16_t* lut, cudaStream_t s) {
  // bias corrections 1 - beta^t, formed in double on the host
  const float bc1 = (float)(1.0 - std::pow((double)beta1, (double)step));
  const float bc2 = (float)(1.0 - std::pow((double)beta2, (double)step));
  adamw_kernel<<<elementwise_grid(total), 256, 0, s>>>(master, m, v, grad, counts, total, per_set, lr, beta1, beta2,
                                                       eps, 1.f - lr * weight_decay, bc1, bc2, lut);
  return cudaGetLastError();
}

cudaError_t launch_sgd(float* master, const float* grad, const int32_t* counts, int64_t total, int64_t per_set,
                       float lr, uint16_t* lut, cudaStream_t s) {
  sgd_kernel<<<elementwise_grid(total), 256, 0, s>>>(master, grad, counts, total, per_set, lr, lut);
  return cudaGetLastError();
}

}  // namespace sk
