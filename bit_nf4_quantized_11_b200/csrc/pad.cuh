// pad.cuh -- copies between compact and rank-padded LoRA tensors.
//
// The layer's kernels take the LoRA rank in multiples of 8 (16-byte rows of
// the [tokens, r] and [out, r] bf16 tensors, which their TMA loads and
// vector accesses need).  For any other rank 1 <= r <= 256 the library runs
// them at rp = r rounded up to 8 on zero-padded copies: the extra rank
// columns of A, B and us are zero, so they add exactly nothing to h, dx, du,
// and the extra rows and columns of the padded dA and dB are discarded.
#pragma once

#include "common.cuh"

namespace qnf4 {

// dst[i][j] = src[i][j] where i < src_rows and j < src_cols, else 0, for
// i < dst_rows, j < dst_cols (both row-major).  T is 2- or 4-byte.
template <typename T>
__global__ void __launch_bounds__(256) copy_pad_kernel(const T* __restrict__ src, int64_t src_rows,
                                                       int64_t src_cols, T* __restrict__ dst, int64_t dst_rows,
                                                       int64_t dst_cols) {
  const int64_t n = dst_rows * dst_cols;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t i = e / dst_cols, j = e % dst_cols;
    dst[e] = (i < src_rows && j < src_cols) ? src[i * src_cols + j] : T(0);
  }
}

}  // namespace qnf4
