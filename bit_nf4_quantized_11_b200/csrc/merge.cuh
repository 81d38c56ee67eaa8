// merge.cuh -- the adapter merged into a bf16 copy of the dequantized base:
//   W'[o][i] = bf16_rne(fp32(w_hat[o][i] + fp32(s * acc[o][i]))),
//   acc[o][i] = fp32 sum over j = 0 .. r-1, in that order, of B[o][j] A[j][i],
// with w_hat = bf16_rne(fp32(level[code] * c_hat)) the dequantized base and
// s = fp32(alpha / r).  Merging needs the base dequantized first and is done
// into a higher-precision copy, since merging straight back into 4 bit is
// lossy ("QLoRA", llm-compass, 调参与实践经验; "QLoRA: Fine-Tuning on One
// Consumer GPU", skillbyai, Merging the adapter for serving).
//
// Each product of two bf16 numbers is exact in fp32, so every fused
// multiply-add below rounds exactly once, like the in-order fp32 sum it
// implements.  A thread takes 4 rows x 8 consecutive columns: per rank index
// j it converts the 8 A values once and reuses them for the 4 rows.
#pragma once

#include "common.cuh"

namespace qnf4 {

constexpr int kMergeRows = 4;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__global__ void __launch_bounds__(256) merge_adapter_kernel(
    const uint8_t* __restrict__ codes, const int8_t* __restrict__ q8, const float* __restrict__ step2,
    const float* __restrict__ mean_ptr, const uint16_t* __restrict__ A, const uint16_t* __restrict__ B, int r,
    float s, int64_t rows, int64_t cols, uint16_t* __restrict__ out, Levels L) {
  __shared__ float s_lv[16];                                         // levels, indexed by code
#pragma unroll
  for (int k = 0; k < 16; ++k)
    if (threadIdx.x == k) s_lv[k] = L.v[k];
  __syncthreads();
  const float mu = *mean_ptr;
  const int64_t cgroups = cols / 8;
  const int64_t n_units = (rows / kMergeRows) * cgroups;
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; u < n_units;
       u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t o0 = (u / cgroups) * kMergeRows;
    const int64_t i0 = (u % cgroups) * 8;
    float acc[kMergeRows][8];
#pragma unroll
    for (int k = 0; k < kMergeRows; ++k)
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[k][c] = 0.f;
    for (int j = 0; j < r; ++j) {
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(A + static_cast<int64_t>(j) * cols + i0));
      const float af[8] = {bf16_lo(a.x), bf16_hi(a.x), bf16_lo(a.y), bf16_hi(a.y),
                           bf16_lo(a.z), bf16_hi(a.z), bf16_lo(a.w), bf16_hi(a.w)};
#pragma unroll
      for (int k = 0; k < kMergeRows; ++k) {
        const float bk = __uint_as_float(static_cast<uint32_t>(__ldg(B + (o0 + k) * r + j)) << 16);
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[k][c] = __fmaf_rn(bk, af[c], acc[k][c]);
      }
    }
#pragma unroll
    for (int k = 0; k < kMergeRows; ++k) {
      const int64_t o = o0 + k;
      const int64_t blk = o * (cols / 64) + i0 / 64;
      const float c_hat = block_scale(__ldg(q8 + blk), __ldg(step2 + blk / 256), mu);
      const uint32_t cw = __ldg(reinterpret_cast<const uint32_t*>(codes + o * (cols / 2) + i0 / 2));
      uint32_t packed[4];
#pragma unroll
      for (int c = 0; c < 8; c += 2) {
        float v[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const uint32_t code = (cw >> (4 * (c + e))) & 0xFu;
          const float w_hat = __bfloat162float(__float2bfloat16_rn(__fmul_rn(s_lv[code], c_hat)));
          v[e] = __fadd_rn(w_hat, __fmul_rn(s, acc[k][c + e]));
        }
        packed[c / 2] = pack_bf16x2_rn(v[0], v[1]);
      }
      *reinterpret_cast<uint4*>(out + o * cols + i0) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
  }
}

}  // namespace qnf4
