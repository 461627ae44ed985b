// C ABI of the sketched linear layer: argument validation and dispatch.
//
// Every entry point validates its arguments on the host before touching the
// device, so a bad call returns a status without launching anything.  The
// library allocates no device memory; the only device state is the check word
// below, which kernels set when they meet data they cannot use (a task id out
// of range, an index too large for its bit width).
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cmath>
#include <cstring>
#include <string>

#include "sk_internal.cuh"
#include "sk_sketch.cuh"

namespace {

__device__ unsigned int g_sk_check_word;

thread_local std::string g_last_error;

sk_status fail(sk_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
sk_status fail(sk_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

sk_status ok() { return SK_OK; }

sk_status cuda_fail(cudaError_t e, const char* what) {
  return fail(SK_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

constexpr int kMaxDevices = 64;
std::atomic<unsigned int*> g_check_ptr[kMaxDevices];
std::atomic<int> g_device_ok[kMaxDevices];  // 0 unknown, 1 sm_100, -1 other

// Current device's check word and capability (cached per device).
sk_status device_state(unsigned int** check) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(SK_ERR_UNSUPPORTED, "device ordinal %d too large", dev);
  int okv = g_device_ok[dev].load(std::memory_order_acquire);
  if (okv == 0) {
    int major = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    okv = (major == 10) ? 1 : -1;
    g_device_ok[dev].store(okv, std::memory_order_release);
  }
  if (okv != 1) return fail(SK_ERR_UNSUPPORTED, "device %d is not sm_100 (B200); kernels are built for sm_100a only", dev);
  unsigned int* p = g_check_ptr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    e = cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_sk_check_word);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(check word)");
    g_check_ptr[dev].store(p, std::memory_order_release);
  }
  *check = p;
  return SK_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, size_t an, const void* b, size_t bn) {
  if (a == nullptr || b == nullptr || an == 0 || bn == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + bn && b0 < a0 + an;
}

size_t row_bytes(int64_t d, int bits) {
  if (bits < 2 || bits > 4 || d <= 0) return 0;
  const int64_t raw = (d * bits + 7) / 8;
  return (size_t)((raw + 15) / 16 * 16);
}

constexpr int64_t kMaxDim = int64_t(1) << 31;

// Kernel choice for the forward.  SK_FWD_PATH=gemv|tc|dq forces one path (for
// measurements and tests).  By default a single-LUT-set batch runs on the
// decode kernel when it applies (4-bit, T <= 16), else on the tensor-core
// kernel from kFwdTcMinT tokens on layers at least 128 columns wide, else on
// the CUDA-core kernel.
constexpr int64_t kFwdTcMinT = 2;

int env_path(const char* name) {
  const char* v = getenv(name);
  if (v == nullptr) return 0;
  if (strcmp(v, "gemv") == 0 || strcmp(v, "simt") == 0) return 1;
  if (strcmp(v, "tc") == 0) return 2;
  if (strcmp(v, "dq") == 0) return 3;
  return 0;
}

// Backward kernel choice: the tensor-core kernels take single-LUT-set batches
// of at least kBwdTcMinT tokens on layers with n, d >= 64; SK_BWD_PATH=simt|tc
// forces a path.  sk_workspace_bytes uses the same rule.
constexpr int64_t kBwdTcMinT = 64;

bool use_tensor_cores_bwd(int64_t n, int64_t d, int64_t T, int ntask) {
  const bool tc_ok = ntask == 1 && n >= 64 && d >= 64;
  const int forced = env_path("SK_BWD_PATH");
  if (forced == 1) return false;
  if (forced == 2) return tc_ok;
  return tc_ok && T >= kBwdTcMinT;
}

bool use_tensor_cores_fwd(const sk::Problem& p) {
  const bool tc_ok = (p.task == nullptr || p.ntask == 1) && p.d >= 128;
  const int forced = env_path("SK_FWD_PATH");
  if (forced == 1) return false;
  if (forced == 2) return tc_ok;
  return tc_ok && p.T >= kFwdTcMinT;
}

bool use_decode_fwd(const sk::Problem& p) {
  const int forced = env_path("SK_FWD_PATH");
  if (forced == 1 || forced == 2) return false;
  return sk::decode_fwd_supported(p);
}

// Several LUT sets: the tensor-core forward needs the routing workspace.
bool routed_fwd_possible(int64_t d, int ntask) { return ntask > 1 && ntask <= sk::kMaxRouteTasks && d >= 128; }

// Several LUT sets in the input gradient: routed tensor-core dX under the same
// rules as the single-set tensor-core backward (SK_BWD_PATH=simt|tc forces).
bool routed_dx_possible(int64_t n, int64_t d, int64_t T, int ntask) {
  if (ntask <= 1 || ntask > sk::kMaxRouteTasks || n < 64 || d < 64) return false;
  const int forced = env_path("SK_BWD_PATH");
  if (forced == 1) return false;
  return forced == 2 || T >= kBwdTcMinT;
}

// Shape rules shared by the layer calls.
sk_status check_shape(int bits, int gpr, int64_t n, int64_t d, int64_t T, int ntask) {
  if (bits < 2 || bits > 4) return fail(SK_ERR_INVALID_ARG, "bits must be 2, 3 or 4 (got %d)", bits);
  if (n < 1 || n % 8 != 0 || n >= kMaxDim) return fail(SK_ERR_INVALID_ARG, "n must be a positive multiple of 8 below 2^31 (got %lld)", (long long)n);
  if (d < 32 || d % 32 != 0 || d >= kMaxDim) return fail(SK_ERR_INVALID_ARG, "d must be a positive multiple of 32 below 2^31 (got %lld)", (long long)d);
  if (gpr < 1 || d % gpr != 0 || (d / gpr) % 32 != 0)
    return fail(SK_ERR_INVALID_ARG, "gpr must divide d into groups whose size is a multiple of 32 (d=%lld, gpr=%d)", (long long)d, gpr);
  if (T < 0 || T >= kMaxDim) return fail(SK_ERR_INVALID_ARG, "T must be in [0, 2^31) (got %lld)", (long long)T);
  if (ntask < 1 || ntask > 65535) return fail(SK_ERR_INVALID_ARG, "ntask must be in [1, 65535] (got %d)", ntask);
  return SK_OK;
}

sk::Problem make_problem(const void* packed, const uint16_t* lut, int bits, int gpr, int64_t n, int64_t d,
                         int64_t T, const int32_t* task, int ntask, unsigned int* check) {
  sk::Problem p;
  p.packed = static_cast<const uint8_t*>(packed);
  p.row_bytes = (int64_t)row_bytes(d, bits);
  p.lut = lut;
  p.bits = bits;
  p.gpr = gpr;
  p.n = n;
  p.d = d;
  p.gs = d / gpr;
  p.T = T;
  p.task = task;
  p.ntask = ntask;
  p.check = check;
  return p;
}

}  // namespace

extern "C" {

int sk_abi_version(void) { return SK_ABI_VERSION; }

const char* sk_status_string(sk_status s) {
  switch (s) {
    case SK_OK: return "SK_OK";
    case SK_ERR_INVALID_ARG: return "SK_ERR_INVALID_ARG";
    case SK_ERR_UNSUPPORTED: return "SK_ERR_UNSUPPORTED";
    case SK_ERR_CUDA: return "SK_ERR_CUDA";
    case SK_ERR_DEVICE_CHECK: return "SK_ERR_DEVICE_CHECK";
  }
  return "SK_ERR_UNKNOWN";
}

const char* sk_last_error(void) { return g_last_error.c_str(); }

size_t sk_packed_row_bytes(int64_t d, int bits) {
  if (d % 32 != 0) return 0;
  return row_bytes(d, bits);
}

size_t sk_packed_bytes(int64_t n, int64_t d, int bits) {
  if (n < 0) return 0;
  return (size_t)n * sk_packed_row_bytes(d, bits);
}

sk_status sk_pack(const uint8_t* idx, int64_t n, int64_t d, int bits, void* packed, size_t packed_bytes,
                  sk_stream_t stream) {
  g_last_error.clear();
  if (bits < 2 || bits > 4) return fail(SK_ERR_INVALID_ARG, "bits must be 2, 3 or 4 (got %d)", bits);
  if (n < 0 || d < 32 || d % 32 != 0 || n >= kMaxDim || d >= kMaxDim)
    return fail(SK_ERR_INVALID_ARG, "need n >= 0 and d a positive multiple of 32 (n=%lld, d=%lld)", (long long)n, (long long)d);
  const size_t need = sk_packed_bytes(n, d, bits);
  if (packed_bytes < need) return fail(SK_ERR_INVALID_ARG, "packed buffer holds %zu bytes, need %zu", packed_bytes, need);
  if (n == 0) return ok();
  if (!idx || !packed) return fail(SK_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(idx) || !aligned16(packed)) return fail(SK_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (overlaps(idx, (size_t)(n * d), packed, need)) return fail(SK_ERR_INVALID_ARG, "idx and packed overlap");
  unsigned int* check = nullptr;
  sk_status st = device_state(&check);
  if (st != SK_OK) return st;
  cudaError_t e = sk::launch_pack(idx, n, d, bits, static_cast<uint8_t*>(packed), (int64_t)row_bytes(d, bits), check,
                                  reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ok() : cuda_fail(e, "pack kernel launch");
}

sk_status sk_unpack(const void* packed, int64_t n, int64_t d, int bits, uint8_t* idx, sk_stream_t stream) {
  g_last_error.clear();
  if (bits < 2 || bits > 4) return fail(SK_ERR_INVALID_ARG, "bits must be 2, 3 or 4 (got %d)", bits);
  if (n < 0 || d < 32 || d % 32 != 0 || n >= kMaxDim || d >= kMaxDim)
    return fail(SK_ERR_INVALID_ARG, "need n >= 0 and d a positive multiple of 32 (n=%lld, d=%lld)", (long long)n, (long long)d);
  if (n == 0) return ok();
  if (!idx || !packed) return fail(SK_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(idx) || !aligned16(packed)) return fail(SK_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (overlaps(idx, (size_t)(n * d), packed, sk_packed_bytes(n, d, bits))) return fail(SK_ERR_INVALID_ARG, "idx and packed overlap");
  unsigned int* check = nullptr;
  sk_status st = device_state(&check);
  if (st != SK_OK) return st;
  cudaError_t e = sk::launch_unpack(static_cast<const uint8_t*>(packed), n, d, bits, (int64_t)row_bytes(d, bits), idx,
                                    reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ok() : cuda_fail(e, "unpack kernel launch");
}

sk_status sk_dequant(const void* packed, const uint16_t* lut, int bits, int gpr, int64_t n, int64_t d, int task,
                     int ntask, uint16_t* theta, sk_stream_t stream) {
  g_last_error.clear();
  sk_status st = check_shape(bits, gpr, n, d, 0, ntask);
  if (st != SK_OK) return st;
  if (task < 0 || task >= ntask) return fail(SK_ERR_INVALID_ARG, "task %d outside [0, %d)", task, ntask);
  if (!packed || !lut || !theta) return fail(SK_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(packed) || !aligned16(lut) || !aligned16(theta)) return fail(SK_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  const size_t lut_bytes = (size_t)ntask * n * gpr * (1u << bits) * 2;
  if (overlaps(theta, (size_t)(n * d * 2), packed, sk_packed_bytes(n, d, bits)) || overlaps(theta, (size_t)(n * d * 2), lut, lut_bytes))
    return fail(SK_ERR_INVALID_ARG, "theta overlaps an input");
  unsigned int* check = nullptr;
  st = device_state(&check);
  if (st != SK_OK) return st;
  sk::Problem p = make_problem(packed, lut, bits, gpr, n, d, 0, nullptr, ntask, check);
  cudaError_t e = sk::launch_dequant(p, task, theta, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ok() : cuda_fail(e, "dequant kernel launch");
}

size_t sk_workspace_bytes(int op, int64_t n, int64_t d, int bits, int gpr, int64_t T, int ntask) {
  if (op < SK_OP_FWD || op > SK_OP_BWD_LUT) return 0;
  if (bits < 2 || bits > 4 || n < 1 || d < 32 || gpr < 1 || d % gpr != 0 || T < 1) return 0;
  if (op == SK_OP_BWD_LUT && use_tensor_cores_bwd(n, d, T, ntask))
    return sk::dlut_tc_workspace(n, d, bits, gpr);
  if (op == SK_OP_FWD && routed_fwd_possible(d, ntask)) return sk::fwd_tc_workspace(T, d, ntask);
  if (op == SK_OP_BWD_INPUT && routed_dx_possible(n, d, T, ntask)) return sk::dx_tc_workspace(T, n, ntask);
  if (op == SK_OP_BWD_LUT && routed_dx_possible(n, d, T, ntask))
    return sk::dlut_tc_routed_workspace(n, d, bits, gpr, T, ntask);
  return 0;
}

static sk_status check_layer_buffers(const void* packed, const uint16_t* lut, bool need_lut, int bits, int gpr,
                                     int64_t n, int64_t d, int64_t T, const int32_t* task, int ntask,
                                     const void* in, size_t in_bytes, const void* in2, size_t in2_bytes,
                                     const void* out, size_t out_bytes) {
  if (!packed || (need_lut && !lut) || !in || !out || (in2_bytes && !in2))
    return fail(SK_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(packed) || (need_lut && !aligned16(lut)) || !aligned16(in) || !aligned16(out) || (in2 && !aligned16(in2)))
    return fail(SK_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  const size_t pk = sk_packed_bytes(n, d, bits);
  const size_t lb = need_lut ? (size_t)ntask * n * gpr * (1u << bits) * 2 : 0;
  const size_t tb = task ? (size_t)T * 4 : 0;
  if (overlaps(out, out_bytes, packed, pk) || overlaps(out, out_bytes, lut, lb) || overlaps(out, out_bytes, in, in_bytes) ||
      overlaps(out, out_bytes, in2, in2_bytes) || overlaps(out, out_bytes, task, tb))
    return fail(SK_ERR_INVALID_ARG, "output overlaps an input");
  return SK_OK;
}

sk_status sk_linear_fwd(const void* packed, const uint16_t* lut, int bits, int gpr, int64_t n, int64_t d,
                        const uint16_t* X, int64_t T, const int32_t* task, int ntask, uint16_t* Y,
                        void* workspace, size_t workspace_bytes, sk_stream_t stream) {
  g_last_error.clear();
  (void)workspace;
  sk_status st = check_shape(bits, gpr, n, d, T, ntask);
  if (st != SK_OK) return st;
  if (T == 0) return ok();
  st = check_layer_buffers(packed, lut, true, bits, gpr, n, d, T, task, ntask, X, (size_t)(T * d * 2), nullptr, 0, Y,
                           (size_t)(T * n * 2));
  if (st != SK_OK) return st;
  unsigned int* check = nullptr;
  st = device_state(&check);
  if (st != SK_OK) return st;
  sk::Problem p = make_problem(packed, lut, bits, gpr, n, d, T, task, ntask, check);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (task != nullptr && ntask > 1 && use_decode_fwd(p)) {
    // a single token: one LUT set, chosen on the device by the decode kernel
    e = sk::launch_decode_fwd(p, X, Y, s);
  } else if (task != nullptr && routed_fwd_possible(d, ntask)) {
    // several LUT sets: bucket the tokens by task and run the tensor-core
    // forward per task tile when the caller gave the routing workspace; without
    // it (or with SK_FWD_PATH=gemv) the CUDA-core kernel serves the batch
    const size_t need = sk::fwd_tc_workspace(T, d, ntask);
    const bool ws_ok = workspace != nullptr && workspace_bytes >= need && aligned16(workspace) &&
                       !overlaps(workspace, need, X, (size_t)(T * d * 2)) && !overlaps(workspace, need, Y, (size_t)(T * n * 2));
    if (ws_ok && env_path("SK_FWD_PATH") != 1) {
      e = sk::launch_fwd_tc_routed(p, X, Y, workspace, s);
    } else {
      e = sk::launch_gemv_fwd(p, X, Y, s);
    }
  } else {
    e = use_decode_fwd(p)         ? sk::launch_decode_fwd(p, X, Y, s)
        : use_tensor_cores_fwd(p) ? sk::launch_fwd_tc(p, X, Y, s)
                                  : sk::launch_gemv_fwd(p, X, Y, s);
  }
  return e == cudaSuccess ? ok() : cuda_fail(e, "forward kernel launch");
}

sk_status sk_linear_fwd_group(const sk_layer* layers, int nlayers, int bits, int64_t T, const int32_t* task,
                              int ntask, sk_stream_t stream) {
  g_last_error.clear();
  if (nlayers < 1 || nlayers > SK_MAX_GROUP_LAYERS)
    return fail(SK_ERR_INVALID_ARG, "nlayers must be in [1, %d] (got %d)", SK_MAX_GROUP_LAYERS, nlayers);
  if (layers == nullptr) return fail(SK_ERR_INVALID_ARG, "null pointer");
  for (int l = 0; l < nlayers; ++l) {
    const sk_layer& L = layers[l];
    sk_status st = check_shape(bits, L.gpr, L.n, L.d, T, ntask);
    if (st != SK_OK) return fail(st, "layer %d: %s", l, g_last_error.c_str());
    if (T == 0) continue;
    st = check_layer_buffers(L.packed, L.lut, true, bits, L.gpr, L.n, L.d, T, task, ntask, L.X, (size_t)(T * L.d * 2),
                             nullptr, 0, L.Y, (size_t)(T * L.n * 2));
    if (st != SK_OK) return fail(st, "layer %d: %s", l, g_last_error.c_str());
  }
  if (T == 0) return ok();
  // the layers run side by side: no output may overlap another layer's buffers
  for (int a = 0; a < nlayers; ++a) {
    const sk_layer& A = layers[a];
    const size_t ya = (size_t)(T * A.n * 2);
    for (int b = 0; b < nlayers; ++b) {
      if (a == b) continue;
      const sk_layer& B = layers[b];
      const size_t lb = (size_t)ntask * B.n * B.gpr * (1u << bits) * 2;
      if (overlaps(A.Y, ya, B.Y, (size_t)(T * B.n * 2)) || overlaps(A.Y, ya, B.X, (size_t)(T * B.d * 2)) ||
          overlaps(A.Y, ya, B.packed, sk_packed_bytes(B.n, B.d, bits)) || overlaps(A.Y, ya, B.lut, lb))
        return fail(SK_ERR_INVALID_ARG, "the output of layer %d overlaps a buffer of layer %d", a, b);
    }
  }
  unsigned int* check = nullptr;
  sk_status st = device_state(&check);
  if (st != SK_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  sk::DecodeLayer D[SK_MAX_GROUP_LAYERS];
  for (int l = 0; l < nlayers; ++l) {
    const sk_layer& L = layers[l];
    D[l].packed = static_cast<const uint8_t*>(L.packed);
    D[l].row_bytes = (int64_t)row_bytes(L.d, bits);
    D[l].lut = L.lut;
    D[l].gpr = L.gpr;
    D[l].n = L.n;
    D[l].d = L.d;
    D[l].X = L.X;
    D[l].Y = L.Y;
  }
  const int forced = env_path("SK_FWD_PATH");
  if (bits == 4 && forced != 1 && forced != 2 && sk::decode_group_supported(D, nlayers, (int)T, task, ntask)) {
    cudaError_t e = sk::launch_decode_group(D, nlayers, (int)T, task, ntask, check, s);
    return e == cudaSuccess ? ok() : cuda_fail(e, "grouped decode kernel launch");
  }
  // otherwise one forward per layer, in order (no workspace: a batch with
  // several LUT sets runs on the CUDA-core kernel)
  for (int l = 0; l < nlayers; ++l) {
    const sk_layer& L = layers[l];
    st = sk_linear_fwd(L.packed, L.lut, bits, L.gpr, L.n, L.d, L.X, T, task, ntask, L.Y, nullptr, 0, stream);
    if (st != SK_OK) return st;
  }
  return ok();
}

sk_status sk_linear_bwd_input(const void* packed, const uint16_t* lut, int bits, int gpr, int64_t n, int64_t d,
                              const uint16_t* dY, int64_t T, const int32_t* task, int ntask, uint16_t* dX,
                              void* workspace, size_t workspace_bytes, sk_stream_t stream) {
  g_last_error.clear();
  (void)workspace;
  sk_status st = check_shape(bits, gpr, n, d, T, ntask);
  if (st != SK_OK) return st;
  if (T == 0) return ok();
  st = check_layer_buffers(packed, lut, true, bits, gpr, n, d, T, task, ntask, dY, (size_t)(T * n * 2), nullptr, 0, dX,
                           (size_t)(T * d * 2));
  if (st != SK_OK) return st;
  unsigned int* check = nullptr;
  st = device_state(&check);
  if (st != SK_OK) return st;
  sk::Problem p = make_problem(packed, lut, bits, gpr, n, d, T, task, ntask, check);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (task != nullptr && ntask > 1) {
    // several LUT sets: tokens bucketed by task for the tensor cores when the
    // caller gave the routing workspace, else the CUDA-core kernel
    const size_t need = sk::dx_tc_workspace(T, n, ntask);
    const bool ws_ok = workspace != nullptr && workspace_bytes >= need && aligned16(workspace) &&
                       !overlaps(workspace, need, dY, (size_t)(T * n * 2)) && !overlaps(workspace, need, dX, (size_t)(T * d * 2));
    e = (ws_ok && routed_dx_possible(n, d, T, ntask)) ? sk::launch_dx_tc_routed(p, dY, dX, workspace, s)
                                                      : sk::launch_simt_bwd_input(p, dY, dX, s);
  } else {
    e = use_tensor_cores_bwd(n, d, T, ntask) ? sk::launch_dx_tc(p, dY, dX, s) : sk::launch_simt_bwd_input(p, dY, dX, s);
  }
  return e == cudaSuccess ? ok() : cuda_fail(e, "input-gradient kernel launch");
}

sk_status sk_linear_bwd_lut(const void* packed, int bits, int gpr, int64_t n, int64_t d, const uint16_t* X,
                            const uint16_t* dY, int64_t T, const int32_t* task, int ntask, float* dlut,
                            int accumulate, void* workspace, size_t workspace_bytes, sk_stream_t stream) {
  g_last_error.clear();
  (void)workspace;
  sk_status st = check_shape(bits, gpr, n, d, T, ntask);
  if (st != SK_OK) return st;
  if (accumulate != 0 && accumulate != 1) return fail(SK_ERR_INVALID_ARG, "accumulate must be 0 or 1");
  const size_t dlut_bytes = (size_t)ntask * n * gpr * (1u << bits) * 4;
  if (!dlut) return fail(SK_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(dlut)) return fail(SK_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  if (T == 0) {
    if (accumulate) return ok();
    cudaError_t e = cudaMemsetAsync(dlut, 0, dlut_bytes, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, "cudaMemsetAsync(dlut)");
  }
  st = check_layer_buffers(packed, nullptr, false, bits, gpr, n, d, T, task, ntask, X, (size_t)(T * d * 2), dY,
                           (size_t)(T * n * 2), dlut, dlut_bytes);
  if (st != SK_OK) return st;
  const bool routed = task != nullptr && ntask > 1;
  if (!routed && workspace_bytes < sk_workspace_bytes(SK_OP_BWD_LUT, n, d, bits, gpr, T, ntask))
    return fail(SK_ERR_INVALID_ARG, "workspace too small");
  unsigned int* check = nullptr;
  st = device_state(&check);
  if (st != SK_OK) return st;
  sk::Problem p = make_problem(packed, nullptr, bits, gpr, n, d, T, task, ntask, check);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (routed) {
    // several LUT sets: the tokens of every set form their own K range of the
    // tensor-core product when the caller gave the routing workspace, else
    // the CUDA-core kernel
    const size_t need = sk::dlut_tc_routed_workspace(n, d, bits, gpr, T, ntask);
    const bool ws_ok = workspace != nullptr && workspace_bytes >= need && aligned16(workspace) &&
                       !overlaps(workspace, need, X, (size_t)(T * d * 2)) && !overlaps(workspace, need, dY, (size_t)(T * n * 2)) &&
                       !overlaps(workspace, need, dlut, dlut_bytes);
    e = (ws_ok && routed_dx_possible(n, d, T, ntask)) ? sk::launch_dlut_tc_routed(p, X, dY, dlut, accumulate, workspace, s)
                                                      : sk::launch_simt_bwd_lut(p, X, dY, dlut, accumulate, s);
  } else if (use_tensor_cores_bwd(n, d, T, ntask)) {
    const size_t need = sk::dlut_tc_workspace(n, d, bits, gpr);
    if (workspace == nullptr || workspace_bytes < need || !aligned16(workspace))
      return fail(SK_ERR_INVALID_ARG, "workspace of %zu bytes (16-byte aligned) required", need);
    e = sk::launch_dlut_tc(p, X, dY, dlut, accumulate, workspace, s);
  } else {
    e = sk::launch_simt_bwd_lut(p, X, dY, dlut, accumulate, s);
  }
  return e == cudaSuccess ? ok() : cuda_fail(e, "LUT-gradient kernel launch");
}

sk_status sk_linear_bwd_lut_noalloc(const void* packed, int bits, int gpr, int64_t n, int64_t d, const uint16_t* X,
                                    const uint16_t* dY, int64_t T, const int32_t* task, int ntask, float* dlut,
                                    int accumulate, sk_stream_t stream) {
  g_last_error.clear();
  sk_status st = check_shape(bits, gpr, n, d, T, ntask);
  if (st != SK_OK) return st;
  if (accumulate != 0 && accumulate != 1) return fail(SK_ERR_INVALID_ARG, "accumulate must be 0 or 1");
  const size_t dlut_bytes = (size_t)ntask * n * gpr * (1u << bits) * 4;
  if (!dlut) return fail(SK_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(dlut)) return fail(SK_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  if (T == 0) {
    if (accumulate) return ok();
    cudaError_t e = cudaMemsetAsync(dlut, 0, dlut_bytes, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, "cudaMemsetAsync(dlut)");
  }
  st = check_layer_buffers(packed, nullptr, false, bits, gpr, n, d, T, task, ntask, X, (size_t)(T * d * 2), dY,
                           (size_t)(T * n * 2), dlut, dlut_bytes);
  if (st != SK_OK) return st;
  const bool tc = use_tensor_cores_bwd(n, d, T, ntask);
  if (tc) {
    const size_t need = sk::dlut_tc_workspace(n, d, bits, gpr);
    if (need > sk::dlut_noalloc_scratch_bytes())
      return fail(SK_ERR_INVALID_ARG,
                  "this layer needs %zu bytes of scratch but the allocation-free call holds %zu; "
                  "use sk_linear_bwd_lut with a caller workspace", need, sk::dlut_noalloc_scratch_bytes());
  }
  unsigned int* check = nullptr;
  st = device_state(&check);
  if (st != SK_OK) return st;
  sk::Problem p = make_problem(packed, nullptr, bits, gpr, n, d, T, task, ntask, check);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (tc) {
    void* scratch = nullptr;
    e = sk::dlut_noalloc_scratch(&scratch);
    if (e != cudaSuccess) return cuda_fail(e, "looking up the scratch array's device address");
    e = sk::launch_dlut_tc(p, X, dY, dlut, accumulate, scratch, s);
  } else {
    e = sk::launch_simt_bwd_lut(p, X, dY, dlut, accumulate, s);
  }
  return e == cudaSuccess ? ok() : cuda_fail(e, "LUT-gradient kernel launch");
}

sk_status sk_bin_counts(const void* packed, int bits, int gpr, int64_t n, int64_t d, int32_t* counts,
                        sk_stream_t stream) {
  g_last_error.clear();
  sk_status st = check_shape(bits, gpr, n, d, 0, 1);
  if (st != SK_OK) return st;
  if (!packed || !counts) return fail(SK_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(packed) || !aligned16(counts)) return fail(SK_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  const size_t cb = (size_t)n * gpr * (1u << bits) * 4;
  if (overlaps(counts, cb, packed, sk_packed_bytes(n, d, bits))) return fail(SK_ERR_INVALID_ARG, "output overlaps an input");
  unsigned int* check = nullptr;
  st = device_state(&check);
  if (st != SK_OK) return st;
  cudaError_t e = sk::launch_bin_counts(static_cast<const uint8_t*>(packed), (int64_t)sk_packed_row_bytes(d, bits), bits,
                                        n, gpr, d / gpr, counts, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ok() : cuda_fail(e, "bin-count kernel launch");
}

// Checks shared by the LUT updates: sizes, pointers, and that no output
// overlaps another buffer.
static sk_status check_update(const void* const* outs, int nout, const float* grad, const int32_t* counts, int ntask,
                              int64_t n, int gpr, int bits, int64_t* total, int64_t* per_set) {
  if (bits < 2 || bits > 4) return fail(SK_ERR_INVALID_ARG, "bits must be 2, 3 or 4 (got %d)", bits);
  if (ntask < 1 || n < 1 || gpr < 1 || n >= kMaxDim || gpr >= (1 << 24))
    return fail(SK_ERR_INVALID_ARG, "ntask, n and gpr must be positive");
  *per_set = n * gpr * (1 << bits);
  *total = *per_set * ntask;
  const size_t fb = (size_t)*total * 4, hb = (size_t)*total * 2, cb = (size_t)*per_set * 4;
  if (!grad) return fail(SK_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(grad) || (counts && !aligned16(counts))) return fail(SK_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  for (int a = 0; a < nout; ++a) {
    const bool half = a == nout - 1;            // the last output is the fp16 LUT (may be NULL)
    if (!outs[a] && !half) return fail(SK_ERR_INVALID_ARG, "null pointer");
    if (!outs[a]) continue;
    if (!aligned16(outs[a])) return fail(SK_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
    const size_t ab = half ? hb : fb;
    if (overlaps(outs[a], ab, grad, fb) || (counts && overlaps(outs[a], ab, counts, cb)))
      return fail(SK_ERR_INVALID_ARG, "output overlaps an input");
    for (int b = 0; b < a; ++b)
      if (outs[b] && overlaps(outs[a], ab, outs[b], fb)) return fail(SK_ERR_INVALID_ARG, "outputs overlap");
  }
  return SK_OK;
}

sk_status sk_lut_adamw(float* master, float* m, float* v, const float* grad, const int32_t* counts, int ntask,
                       int64_t n, int gpr, int bits, float lr, float beta1, float beta2, float eps,
                       float weight_decay, int step, uint16_t* lut, sk_stream_t stream) {
  g_last_error.clear();
  const void* outs[4] = {master, m, v, lut};
  int64_t total = 0, per_set = 0;
  sk_status st = check_update(outs, 4, grad, counts, ntask, n, gpr, bits, &total, &per_set);
  if (st != SK_OK) return st;
  if (!(std::isfinite(lr) && beta1 >= 0.f && beta1 < 1.f && beta2 >= 0.f && beta2 < 1.f && eps > 0.f &&
        std::isfinite(eps) && std::isfinite(weight_decay) && step >= 1))
    return fail(SK_ERR_INVALID_ARG, "AdamW needs finite lr and weight_decay, 0 <= beta < 1, eps > 0, step >= 1");
  unsigned int* check = nullptr;
  st = device_state(&check);
  if (st != SK_OK) return st;
  cudaError_t e = sk::launch_adamw(master, m, v, grad, counts, total, per_set, lr, beta1, beta2, eps, weight_decay,
                                   step, lut, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ok() : cuda_fail(e, "AdamW kernel launch");
}

sk_status sk_lut_sgd(float* master, const float* grad, const int32_t* counts, int ntask, int64_t n, int gpr,
                     int bits, float lr, uint16_t* lut, sk_stream_t stream) {
  g_last_error.clear();
  const void* outs[2] = {master, lut};
  int64_t total = 0, per_set = 0;
  sk_status st = check_update(outs, 2, grad, counts, ntask, n, gpr, bits, &total, &per_set);
  if (st != SK_OK) return st;
  if (!std::isfinite(lr)) return fail(SK_ERR_INVALID_ARG, "lr must be finite");
  unsigned int* check = nullptr;
  st = device_state(&check);
  if (st != SK_OK) return st;
  cudaError_t e = sk::launch_sgd(master, grad, counts, total, per_set, lr, lut, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ok() : cuda_fail(e, "SGD kernel launch");
}

// ---------------------------------------------------------------------------
// Sketching stage
// ---------------------------------------------------------------------------

constexpr int64_t kMaxSketchDim = int64_t(1) << 16;

size_t sk_inverse_factor_workspace_bytes(int64_t d) {
  if (d < 1 || d > kMaxSketchDim) return 0;
  return sk::inverse_factor_workspace(d);
}

size_t sk_sketch_round_workspace_bytes(int64_t n, int64_t d) {
  if (n < 1 || d < 1 || n >= kMaxDim || d > kMaxSketchDim) return 0;
  return sk::sketch_round_workspace(n, d);
}

sk_status sk_gram(const uint16_t* X, int64_t s, int64_t d, float* H, int accumulate, sk_stream_t stream) {
  g_last_error.clear();
  if (s < 0 || s >= kMaxDim || d < 64 || d > kMaxSketchDim || d % 8)
    return fail(SK_ERR_INVALID_ARG, "need 0 <= s < 2^31 and 64 <= d <= 65536 with d %% 8 == 0 (s=%lld, d=%lld)",
                (long long)s, (long long)d);
  if (!H || (s > 0 && !X)) return fail(SK_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(H) || (X && !aligned16(X))) return fail(SK_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  if (overlaps(H, (size_t)d * d * 4, X, (size_t)s * d * 2)) return fail(SK_ERR_INVALID_ARG, "output overlaps an input");
  unsigned int* check = nullptr;
  sk_status st = device_state(&check);
  if (st != SK_OK) return st;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  if (s == 0) {
    if (!accumulate) e = cudaMemsetAsync(H, 0, (size_t)d * d * 4, cs);
  } else {
    e = sk::launch_gram(X, s, d, H, accumulate, check, cs);
  }
  return e == cudaSuccess ? ok() : cuda_fail(e, "Gram kernel launch");
}

sk_status sk_inverse_factor(const float* H, int64_t d, double damp, double* U, double* hinv_diag, void* workspace,
                            size_t workspace_bytes, sk_stream_t stream) {
  g_last_error.clear();
  if (d < 1 || d > kMaxSketchDim) return fail(SK_ERR_INVALID_ARG, "need 1 <= d <= 65536 (d=%lld)", (long long)d);
  if (!(damp >= 0.0) || !std::isfinite(damp)) return fail(SK_ERR_INVALID_ARG, "damp must be finite and >= 0");
  if (!H || !U || !hinv_diag || !workspace) return fail(SK_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(H) || !aligned16(U) || !aligned16(hinv_diag) || !aligned16(workspace))
    return fail(SK_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  const size_t need = sk::inverse_factor_workspace(d);
  if (workspace_bytes < need)
    return fail(SK_ERR_INVALID_ARG, "workspace too small: %zu bytes, need %zu", workspace_bytes, need);
  const size_t hb = (size_t)d * d * 4, ub = (size_t)d * d * 8, db = (size_t)d * 8;
  if (overlaps(U, ub, H, hb) || overlaps(hinv_diag, db, H, hb) || overlaps(workspace, need, H, hb) ||
      overlaps(U, ub, hinv_diag, db) || overlaps(U, ub, workspace, need) || overlaps(hinv_diag, db, workspace, need))
    return fail(SK_ERR_INVALID_ARG, "buffers overlap");
  unsigned int* check = nullptr;
  sk_status st = device_state(&check);
  if (st != SK_OK) return st;
  cudaError_t e = sk::launch_inverse_factor(H, d, damp, U, hinv_diag, workspace, check,
                                            reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ok() : cuda_fail(e, "inverse-factor kernel launch");
}

static sk_status check_sketch_shape(int bits, int gpr, int64_t n, int64_t d) {
  if (bits < 2 || bits > 4) return fail(SK_ERR_INVALID_ARG, "bits must be 2, 3 or 4 (got %d)", bits);
  if (n < 1 || d < 1 || gpr < 1 || n >= kMaxDim || d > kMaxSketchDim || d % gpr)
    return fail(SK_ERR_INVALID_ARG, "need n, d, gpr >= 1, d <= 65536 and d %% gpr == 0 (n=%lld, d=%lld, gpr=%d)",
                (long long)n, (long long)d, gpr);
  return SK_OK;
}

sk_status sk_lloyd(const float* theta, const double* hinv_diag, int bits, int gpr, int64_t n, int64_t d, int max_iter,
                   uint16_t* lut, int32_t* iters, sk_stream_t stream) {
  g_last_error.clear();
  sk_status st = check_sketch_shape(bits, gpr, n, d);
  if (st != SK_OK) return st;
  if (d / gpr > sk::kSketchMaxGroup)
    return fail(SK_ERR_UNSUPPORTED, "groups of %lld columns; at most %lld", (long long)(d / gpr),
                (long long)sk::kSketchMaxGroup);
  if (n * gpr >= kMaxDim) return fail(SK_ERR_INVALID_ARG, "n * gpr must be below 2^31");
  if (max_iter < 0) return fail(SK_ERR_INVALID_ARG, "max_iter must be >= 0");
  if (!theta || !hinv_diag || !lut) return fail(SK_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(theta) || !aligned16(hinv_diag) || !aligned16(lut) || (iters && !aligned16(iters)))
    return fail(SK_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  const size_t lb = (size_t)n * gpr * (1u << bits) * 2, ib = (size_t)n * gpr * 4;
  const size_t tb = (size_t)n * d * 4, hb = (size_t)d * 8;
  if (overlaps(lut, lb, theta, tb) || overlaps(lut, lb, hinv_diag, hb) ||
      (iters && (overlaps(iters, ib, theta, tb) || overlaps(iters, ib, hinv_diag, hb) || overlaps(iters, ib, lut, lb))))
    return fail(SK_ERR_INVALID_ARG, "buffers overlap");
  unsigned int* check = nullptr;
  st = device_state(&check);
  if (st != SK_OK) return st;
  cudaError_t e = sk::launch_lloyd(theta, hinv_diag, bits, gpr, n, d, max_iter, lut, iters,
                                   reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ok() : cuda_fail(e, "Lloyd kernel launch");
}

sk_status sk_sketch_round(const float* theta, const double* U, const uint16_t* lut, int bits, int gpr, int64_t n,
                          int64_t d, uint8_t* idx, void* workspace, size_t workspace_bytes, sk_stream_t stream) {
  g_last_error.clear();
  sk_status st = check_sketch_shape(bits, gpr, n, d);
  if (st != SK_OK) return st;
  if (n > (int64_t)65535 * 64) return fail(SK_ERR_UNSUPPORTED, "at most 4194240 rows");
  if (!theta || !U || !lut || !idx || !workspace) return fail(SK_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(theta) || !aligned16(U) || !aligned16(lut) || !aligned16(idx) || !aligned16(workspace))
    return fail(SK_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  const size_t need = sk::sketch_round_workspace(n, d);
  if (workspace_bytes < need)
    return fail(SK_ERR_INVALID_ARG, "workspace too small: %zu bytes, need %zu", workspace_bytes, need);
  const size_t xb = (size_t)n * d, tb = xb * 4, ub = (size_t)d * d * 8, lb = (size_t)n * gpr * (1u << bits) * 2;
  if (overlaps(idx, xb, theta, tb) || overlaps(idx, xb, U, ub) || overlaps(idx, xb, lut, lb) ||
      overlaps(idx, xb, workspace, need) || overlaps(workspace, need, theta, tb) || overlaps(workspace, need, U, ub) ||
      overlaps(workspace, need, lut, lb))
    return fail(SK_ERR_INVALID_ARG, "buffers overlap");
  unsigned int* check = nullptr;
  st = device_state(&check);
  if (st != SK_OK) return st;
  cudaError_t e = sk::launch_sketch_round(theta, U, lut, bits, gpr, n, d, idx, workspace, check,
                                          reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ok() : cuda_fail(e, "mapping kernel launch");
}

sk_status sk_device_check(uint32_t* flags, int clear, sk_stream_t stream) {
  g_last_error.clear();
  if (!flags) return fail(SK_ERR_INVALID_ARG, "null pointer");
  unsigned int* check = nullptr;
  sk_status st = device_state(&check);
  if (st != SK_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned int host = 0;
  cudaError_t e = cudaMemcpyAsync(&host, check, sizeof host, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess && clear) e = cudaMemsetAsync(check, 0, sizeof host, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device check word");
  *flags = host;
  if (host) return fail(SK_ERR_DEVICE_CHECK, "device check word 0x%x", host);
  return SK_OK;
}

}  // extern "C"
