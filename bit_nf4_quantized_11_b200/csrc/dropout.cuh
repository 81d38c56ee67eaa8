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
#pragma once

#include "common.cuh"

namespace qnf4 {

// dropout_dx_kernel    dx = bf16(fp32(dx_base) + fp32((k / (1 - p)) * P)),
//                      P = du . A (fp32 accumulation), after the dx GEMM
//                      ran without its rank-r tail.
// A CTA takes a tile of 64 rows x 128 columns of dx: it stages du[rows, :r]
// and A[:r, columns] in shared memory, its four warps compute P for 16 rows
// each with warp-level bf16 MMAs (m16n8k16, the rank in 16-wide steps, rows
// of du and A past r are zero), leave P in shared memory, and then every
// thread applies 8 consecutive columns of one row: one 16-byte read and
// write of dx, one keep byte, two 16-byte reads of P.
constexpr int kDxTileRows = 64;
constexpr int kDxTileCols = 128;
constexpr int kDxThreads = 128;

__host__ __device__ constexpr int dx_rank_pad(int r) { return (r + 15) / 16 * 16; }
__host__ __device__ constexpr int dx_du_pitch(int r) { return dx_rank_pad(r) * 2 + 16; }   // bytes per du row
constexpr int kDxAPitch = kDxTileCols * 2 + 16;                                           // bytes per A row
constexpr int kDxPPitch = kDxTileCols * 4 + 16;                                           // bytes per P row
__host__ __device__ constexpr int dx_smem_bytes(int r) {
  const int stage = kDxTileRows * dx_du_pitch(r) + dx_rank_pad(r) * kDxAPitch;
  const int p = kDxTileRows * kDxPPitch;
  return stage > p ? stage : p;
}

__global__ void __launch_bounds__(kDxThreads) dropout_dx_kernel(
    uint16_t* __restrict__ dx, const uint16_t* __restrict__ du, const uint16_t* __restrict__ A,
    const uint8_t* __restrict__ keep_bits, int64_t M, int64_t n, int r, float inv_keep) {
  extern __shared__ __align__(16) uint8_t s_dx[];
  const int rk = dx_rank_pad(r);
  const int du_pitch = dx_du_pitch(r);
  uint8_t* s_du = s_dx;
  uint8_t* s_a = s_dx + kDxTileRows * du_pitch;
  const int64_t tiles_n = (n + kDxTileCols - 1) / kDxTileCols;     // n % 64 == 0: the last tile may be half
  const int64_t m0 = (static_cast<int64_t>(blockIdx.x) / tiles_n) * kDxTileRows;
  const int64_t i0 = (static_cast<int64_t>(blockIdx.x) % tiles_n) * kDxTileCols;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // stage du[m0 .. m0+63][0 .. rk) and A[0 .. rk)[i0 .. i0+127] (zero past M and r)
  for (int e = threadIdx.x; e < kDxTileRows * (rk / 8); e += kDxThreads) {
    const int row = e / (rk / 8), ch = e % (rk / 8);
    const bool ok = m0 + row < M && ch * 8 < r;
    cp_async_16(smem_u32(s_du + row * du_pitch + ch * 16), du + (ok ? (m0 + row) * r + ch * 8 : 0), ok);
  }
  for (int e = threadIdx.x; e < rk * (kDxTileCols / 8); e += kDxThreads) {
    const int row = e / (kDxTileCols / 8), ch = e % (kDxTileCols / 8);
    const bool ok = row < r && i0 + ch * 8 < n;
    cp_async_16(smem_u32(s_a + row * kDxAPitch + ch * 16), A + (ok ? static_cast<int64_t>(row) * n + i0 + ch * 8 : 0),
                ok);
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();

  // P[16 rows of this warp][128 columns] = du . A
  float acc[16][4];
#pragma unroll
  for (int t = 0; t < 16; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
  const uint32_t du_base = smem_u32(s_du), a_base = smem_u32(s_a);
  for (int k0 = 0; k0 < rk; k0 += 16) {
    uint32_t a0, a1, a2, a3;
    {
      const int row = warp * 16 + (lane & 15);
      ldsm_x4(du_base + row * du_pitch + (k0 + 8 * (lane >> 4)) * 2, a0, a1, a2, a3);
    }
#pragma unroll
    for (int tp = 0; tp < 16; tp += 2) {
      // matrices: (k lo, n 8 tp..), (k hi, n 8 tp..), (k lo, n 8 tp+8..), (k hi, n 8 tp+8..)
      const int mi = lane >> 3;
      const int krow = k0 + ((mi & 1) << 3) + (lane & 7);
      const int ncol = tp * 8 + ((mi >> 1) << 3);
      uint32_t b0, b1, b2, b3;
      ldsm_x4_trans(a_base + krow * kDxAPitch + ncol * 2, b0, b1, b2, b3);
      mma_bf16_16816(acc[tp], a0, a1, a2, a3, b0, b1);
      mma_bf16_16816(acc[tp + 1], a0, a1, a2, a3, b2, b3);
    }
  }
  __syncthreads();                                                   // the staged operands are read
  {
    const int g = lane >> 2, q = lane & 3;
#pragma unroll
    for (int t = 0; t < 16; ++t) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = warp * 16 + g + 8 * h;
        const uint32_t addr = smem_u32(s_dx + row * kDxPPitch + (t * 8 + 2 * q) * 4);
        asm volatile("st.shared.v2.f32 [%0], {%1, %2};" :: "r"(addr), "f"(acc[t][2 * h]), "f"(acc[t][2 * h + 1])
                     : "memory");
      }
    }
  }
  __syncthreads();

  // dx += (k / (1 - p)) * P, 8 columns of one row per thread and unit; all
  // of a thread's dx and keep loads are issued before any store
  constexpr int kUnits = kDxTileRows * (kDxTileCols / 8) / kDxThreads;   // 8
  uint4 dv[kUnits];
  uint32_t kv[kUnits];
#pragma unroll
  for (int u = 0; u < kUnits; ++u) {
    const int e = threadIdx.x + u * kDxThreads;
    const int row = e / (kDxTileCols / 8), c8 = e % (kDxTileCols / 8);
    const int64_t m = m0 + row, i = i0 + c8 * 8;
    dv[u] = make_uint4(0, 0, 0, 0);
    kv[u] = 0;
    if (m < M && i < n) {
      dv[u] = *reinterpret_cast<const uint4*>(dx + m * n + i);
      kv[u] = __ldg(keep_bits + m * (n / 8) + i / 8);
    }
  }
#pragma unroll
  for (int u = 0; u < kUnits; ++u) {
    const int e = threadIdx.x + u * kDxThreads;
    const int row = e / (kDxTileCols / 8), c8 = e % (kDxTileCols / 8);
    const int64_t m = m0 + row, i = i0 + c8 * 8;
    if (m >= M || i >= n) continue;
    float pv[8];
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(pv[0]), "=f"(pv[1]), "=f"(pv[2]), "=f"(pv[3])
                 : "r"(smem_u32(s_dx + row * kDxPPitch + c8 * 32)) : "memory");
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(pv[4]), "=f"(pv[5]), "=f"(pv[6]), "=f"(pv[7])
                 : "r"(smem_u32(s_dx + row * kDxPPitch + c8 * 32 + 16)) : "memory");
    const uint32_t dw[4] = {dv[u].x, dv[u].y, dv[u].z, dv[u].w};
    const uint32_t kb = kv[u];
    uint32_t o[4];
#pragma unroll
    for (int e2 = 0; e2 < 4; ++e2) {
      const float k0 = (kb >> (2 * e2)) & 1u ? inv_keep : 0.f;
      const float k1 = (kb >> (2 * e2 + 1)) & 1u ? inv_keep : 0.f;
      const float v0 = __fadd_rn(__uint_as_float(dw[e2] << 16), __fmul_rn(k0, pv[2 * e2]));
      const float v1 = __fadd_rn(__uint_as_float(dw[e2] & 0xFFFF0000u), __fmul_rn(k1, pv[2 * e2 + 1]));
      o[e2] = pack_bf16x2_rn(v0, v1);
    }
    *reinterpret_cast<uint4*>(dx + m * n + i) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace qnf4
