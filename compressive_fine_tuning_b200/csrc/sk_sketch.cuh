// Host launchers of the sketching stage (sk_sketch.cu): the calibration Gram
// matrix, its damped inverse factor, weighted Lloyd per (row, group) and the
// column-by-column mapping with error compensation ("SpaLLM: Unified
// Compressive Adaptation of LLMs with Sketching", section 2.2).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace sk {

// longest group (columns per (row, group)) that weighted Lloyd handles
constexpr int64_t kSketchMaxGroup = 16384;

// H [d][d] (+)= X^T X for bf16 X [s][d] (s >= 1, d % 8 == 0)
cudaError_t launch_gram(const uint16_t* X, int64_t s, int64_t d, float* H, int accumulate, unsigned int* check,
                        cudaStream_t st);
// bytes of scratch sk_inverse_factor needs for a d x d Gram matrix
size_t inverse_factor_workspace(int64_t d);
cudaError_t launch_inverse_factor(const float* H, int64_t d, double damp, double* U, double* hinv_diag,
                                  void* workspace, unsigned int* check, cudaStream_t st);
cudaError_t launch_lloyd(const float* theta, const double* hinv_diag, int bits, int gpr, int64_t n, int64_t d,
                         int max_iter, uint16_t* lut, int32_t* iters, cudaStream_t st);
size_t sketch_round_workspace(int64_t n, int64_t d);
cudaError_t launch_sketch_round(const float* theta, const double* U, const uint16_t* lut, int bits, int gpr, int64_t n,
                                int64_t d, uint8_t* idx, void* workspace, unsigned int* check, cudaStream_t st);

}  // namespace sk
