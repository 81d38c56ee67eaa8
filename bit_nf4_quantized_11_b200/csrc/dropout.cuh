// dropout.cuh -- LoRA dropout on the adapter input (inverted scaling, keep
// mask given by the caller as bits: bit i%8 of byte i/8 of a row keeps
// column i).  The layer becomes
//   h  = x W0^T + s ((x * k) / (1 - p)) A^T B^T
//   dx = dh W0 + s ((dh B) A) * k / (1 - p)
// (dropout 0.05 in every configuration on the pages: "QLoRA", aigrafen.se,
// llm-compass 实现要点, skillbyai, learn-interview-questions section 3; the
// placement on the adapter input is this library's reading).
//
// The masked input x * k (exact in bf16: kept or zero) is never stored: the
// rank-r kernels apply the keep bits to the activation tiles they stage
// (lora_sm100.cuh).
// dropout_dx_kernel    dx = bf16(fp32(dx_base) + (k / (1 - p)) * sum_j du[m][j] A[j][i])
//                      after the dx GEMM ran without its rank-r tail; the sum
//                      is an in-order fp32 fused multiply-add chain
#pragma once

#include "common.cuh"

namespace qnf4 {

constexpr int kDxRows = 4;

// A thread takes kDxRows rows x 8 consecutive columns of dx.
__global__ void __launch_bounds__(256) dropout_dx_kernel(
    uint16_t* __restrict__ dx, const uint16_t* __restrict__ du, const uint16_t* __restrict__ A,
    const uint8_t* __restrict__ keep_bits, int64_t M, int64_t n, int r, float inv_keep) {
  const int64_t cgroups = n / 8;
  const int64_t n_units = ((M + kDxRows - 1) / kDxRows) * cgroups;
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; u < n_units;
       u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m0 = (u / cgroups) * kDxRows;
    const int64_t i0 = (u % cgroups) * 8;
    float acc[kDxRows][8];
#pragma unroll
    for (int k = 0; k < kDxRows; ++k)
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[k][c] = 0.f;
    for (int j = 0; j < r; ++j) {
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(A + static_cast<int64_t>(j) * n + i0));
      const float af[8] = {__uint_as_float(a.x << 16), __uint_as_float(a.x & 0xFFFF0000u),
                           __uint_as_float(a.y << 16), __uint_as_float(a.y & 0xFFFF0000u),
                           __uint_as_float(a.z << 16), __uint_as_float(a.z & 0xFFFF0000u),
                           __uint_as_float(a.w << 16), __uint_as_float(a.w & 0xFFFF0000u)};
#pragma unroll
      for (int k = 0; k < kDxRows; ++k) {
        const int64_t m = min(m0 + k, M - 1);                        // rows past M: computed, not stored
        const float dk = __uint_as_float(static_cast<uint32_t>(__ldg(du + m * r + j)) << 16);
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[k][c] = __fmaf_rn(dk, af[c], acc[k][c]);
      }
    }
#pragma unroll
    for (int k = 0; k < kDxRows; ++k) {
      const int64_t m = m0 + k;
      if (m >= M) break;
      const uint32_t kb = __ldg(keep_bits + m * cgroups + i0 / 8);
      uint16_t* p = dx + m * n + i0;
      const uint4 d = *reinterpret_cast<const uint4*>(p);
      const uint32_t dw[4] = {d.x, d.y, d.z, d.w};
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float k0 = (kb >> (2 * e)) & 1u ? inv_keep : 0.f;
        const float k1 = (kb >> (2 * e + 1)) & 1u ? inv_keep : 0.f;
        const float v0 = __fadd_rn(__uint_as_float(dw[e] << 16), __fmul_rn(k0, acc[k][2 * e]));
        const float v1 = __fadd_rn(__uint_as_float(dw[e] & 0xFFFF0000u), __fmul_rn(k1, acc[k][2 * e + 1]));
        o[e] = pack_bf16x2_rn(v0, v1);
      }
      *reinterpret_cast<uint4*>(p) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

}  // namespace qnf4
