// Index packing (step a0) and dense dequantisation (test / comparison aid).
//
// The packed format stores the one-hot sketching matrix of Eq. 1 ("SpaLLM:
// Unified Compressive Adaptation of LLMs with Sketching", section 2.2) as its
// column indices: 4-bit two per byte (low nibble first), 2-bit four per byte
// (index j at bits 2*(j & 3)), 3-bit 32 per three little-endian words (index j
// at bit 3*(j mod 32)).  Rows are zero-padded to 16 bytes.
//
// One thread handles one 32-index chunk: 32 bytes in, 4*bits bytes out.  These
// kernels run once per model load, far from the hot path; they only need to be
// coalesced and exact.
#include "sk_internal.cuh"

namespace sk {
namespace {

template <int BITS>
__global__ void pack_kernel(const uint8_t* __restrict__ idx, int64_t n, int64_t d,
                            uint8_t* __restrict__ packed, int64_t row_bytes, unsigned int* check) {
  const int64_t chunks = d / 32;
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= n * chunks) return;
  const int64_t i = gid / chunks, c = gid % chunks;
  const uint4* src = reinterpret_cast<const uint4*>(idx + i * d + c * 32);
  uint4 a = __ldg(src), b = __ldg(src + 1);
  uint32_t v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};  // byte e of v[q] = index 4q + e
  const uint32_t kmask = (1u << BITS) - 1u;
  const uint32_t rep = kmask * 0x01010101u;
  bool bad = false;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    bad |= (v[q] & ~rep) != 0u;
    v[q] &= rep;
  }
  if (bad) atomicOr(check, SK_CHECK_INDEX_RANGE);
  uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    const uint32_t x = (v[e >> 2] >> (8 * (e & 3))) & kmask;
    const int bit = e * BITS, wi = bit >> 5, s = bit & 31;
    w[wi] |= x << s;
    if (BITS == 3 && s > 29) w[wi + 1] |= x >> (32 - s);
  }
  uint8_t* row = packed + i * row_bytes;
  uint32_t* dst = reinterpret_cast<uint32_t*>(row + c * ChunkBytes<BITS>::value);
#pragma unroll
  for (int q = 0; q < BITS; ++q) dst[q] = w[q];
  if (c == chunks - 1) {  // zero the row's padding
    for (int64_t b2 = (c + 1) * ChunkBytes<BITS>::value; b2 < row_bytes; ++b2) row[b2] = 0;
  }
}

template <int BITS>
__global__ void unpack_kernel(const uint8_t* __restrict__ packed, int64_t n, int64_t d, int64_t row_bytes,
                              uint8_t* __restrict__ idx) {
  const int64_t chunks = d / 32;
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= n * chunks) return;
  const int64_t i = gid / chunks, c = gid % chunks;
  Chunk<BITS> ch = load_chunk<BITS>(packed + i * row_bytes, c);
  uint32_t v[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    v[q] = chunk_index<BITS>(ch, 4 * q) | (chunk_index<BITS>(ch, 4 * q + 1) << 8) |
           (chunk_index<BITS>(ch, 4 * q + 2) << 16) | (chunk_index<BITS>(ch, 4 * q + 3) << 24);
  }
  uint4* dst = reinterpret_cast<uint4*>(idx + i * d + c * 32);
  dst[0] = make_uint4(v[0], v[1], v[2], v[3]);
  dst[1] = make_uint4(v[4], v[5], v[6], v[7]);
}

template <int BITS>
__global__ void dequant_kernel(Problem p, int task, uint16_t* __restrict__ theta) {
  const int64_t chunks = p.d / 32;
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= p.n * chunks) return;
  const int64_t i = gid / chunks, c = gid % chunks;
  const int64_t g = (c * 32) / p.gs;
  LutRegs<BITS> L;
  load_lut<BITS>(lut_ptr(p, task, i, g), L);
  Chunk<BITS> ch = load_chunk<BITS>(p.packed + i * p.row_bytes, c);
  uint32_t o[16];
  dequant_chunk<BITS>(ch, L, o);
  uint4* dst = reinterpret_cast<uint4*>(theta + i * p.d + c * 32);
#pragma unroll
  for (int q = 0; q < 4; ++q) dst[q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
}

inline unsigned grid_for(int64_t threads, int block) { return (unsigned)((threads + block - 1) / block); }

}  // namespace

cudaError_t launch_pack(const uint8_t* idx, int64_t n, int64_t d, int bits, uint8_t* packed,
                        int64_t row_bytes, unsigned int* check, cudaStream_t s) {
  const int64_t work = n * (d / 32);
  const unsigned g = grid_for(work, 256);
  switch (bits) {
    case 2: pack_kernel<2><<<g, 256, 0, s>>>(idx, n, d, packed, row_bytes, check); break;
    case 3: pack_kernel<3><<<g, 256, 0, s>>>(idx, n, d, packed, row_bytes, check); break;
    default: pack_kernel<4><<<g, 256, 0, s>>>(idx, n, d, packed, row_bytes, check); break;
  }
  return cudaGetLastError();
}

cudaError_t launch_unpack(const uint8_t* packed, int64_t n, int64_t d, int bits, int64_t row_bytes,
                          uint8_t* idx, cudaStream_t s) {
  const unsigned g = grid_for(n * (d / 32), 256);
  switch (bits) {
    case 2: unpack_kernel<2><<<g, 256, 0, s>>>(packed, n, d, row_bytes, idx); break;
    case 3: unpack_kernel<3><<<g, 256, 0, s>>>(packed, n, d, row_bytes, idx); break;
    default: unpack_kernel<4><<<g, 256, 0, s>>>(packed, n, d, row_bytes, idx); break;
  }
  return cudaGetLastError();
}

cudaError_t launch_dequant(const Problem& p, int task, uint16_t* theta, cudaStream_t s) {
  const unsigned g = grid_for(p.n * (p.d / 32), 256);
  switch (p.bits) {
    case 2: dequant_kernel<2><<<g, 256, 0, s>>>(p, task, theta); break;
    case 3: dequant_kernel<3><<<g, 256, 0, s>>>(p, task, theta); break;
    default: dequant_kernel<4><<<g, 256, 0, s>>>(p, task, theta); break;
  }
  return cudaGetLastError();
}

}  // namespace sk
