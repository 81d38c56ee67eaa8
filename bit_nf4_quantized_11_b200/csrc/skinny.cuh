// skinny.cuh -- the rank-r contractions of the QLoRA layer (sm_100a).
//
// All of them have one dimension equal to the LoRA rank r (8..256), stream a
// token-sized operand from HBM once and are bound by that read, so they run
// on warp-level bf16 MMA (fp32 accumulation) with coalesced 16-byte loads:
//
//   row-wise  out[m][n] = bf16(scale * sum_k act[m][k] * Wt[n][k])
//       forward   us = bf16(s x A^T)      act = x  [M, in],  Wt = A  [r, in]
//       backward  du = bf16(s dh B)       act = dh [M, out], Wt = B^T [r, out]
//   col-wise  part[c][p][n] = sum_{m in chunk c} act[m][p] * u[m][n]
//       backward  dB   = dh^T us          act = dh [M, out], u = us [M, r]
//       backward  dA^T = x^T du           act = x  [M, in],  u = du [M, r]
//   followed by a fixed-order sum over the token chunks (deterministic).
//
// ("QLoRA", llm-compass, 方法与公式: h = dequant(W0) x + (alpha/r) B A x with
// gradients only for A and B.)
#pragma once

#include "common.cuh"

namespace qnf4 {

// ---------------------------------------------------------------------------
// row-wise skinny GEMM.  CTA = 8 warps on 16 token rows; the K range is cut
// into 32-wide chunks dealt round-robin to the warps; partial 16 x 64 tiles
// are reduced through shared memory in a fixed order.  The MMA's K order is
// permuted consistently for both operands (thread q of a quad owns physical
// k = 8q..8q+7 of every 32-chunk), so each operand fragment is one 16-byte
// load.  Output columns are processed 64 at a time.
// ---------------------------------------------------------------------------
constexpr int kRowThreads = 256;

__global__ void __launch_bounds__(kRowThreads) rowwise_skinny_kernel(
    const uint16_t* __restrict__ act, const uint16_t* __restrict__ Wt,
    uint16_t* __restrict__ out, int M, int K, int R, float scale) {
  __shared__ float s_red[8][16][65];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
  const int m0 = blockIdx.x * 16;
  const int n_chunks = K / 32;
  const bool row0 = (m0 + g) < M, row1 = (m0 + g + 8) < M;
  const uint16_t* a_row0 = act + static_cast<int64_t>(row0 ? m0 + g : 0) * K + 8 * q;
  const uint16_t* a_row1 = act + static_cast<int64_t>(row1 ? m0 + g + 8 : 0) * K + 8 * q;

  for (int nb = 0; nb < R; nb += 64) {
    const int nt = min(8, (R - nb) / 8);
    float acc[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;

    for (int c = warp; c < n_chunks; c += 8) {
      const int k0 = c * 32;
      const uint4 z = make_uint4(0, 0, 0, 0);
      const uint4 u0 = row0 ? ld_nc_v4(a_row0 + k0) : z;
      const uint4 u1 = row1 ? ld_nc_v4(a_row1 + k0) : z;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < nt) {
          const uint4 b = ld_nc_v4(Wt + static_cast<int64_t>(nb + 8 * j + g) * K + k0 + 8 * q);
          mma_bf16_16816(acc[j], u0.x, u1.x, u0.y, u1.y, b.x, b.y);
          mma_bf16_16816(acc[j], u0.z, u1.z, u0.w, u1.w, b.z, b.w);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      s_red[warp][g][8 * j + 2 * q] = acc[j][0];
      s_red[warp][g][8 * j + 2 * q + 1] = acc[j][1];
      s_red[warp][g + 8][8 * j + 2 * q] = acc[j][2];
      s_red[warp][g + 8][8 * j + 2 * q + 1] = acc[j][3];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < 16 * 64; e += kRowThreads) {
      const int rr = e >> 6, cc = e & 63;
      if (cc < nt * 8 && m0 + rr < M) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) v += s_red[w][rr][cc];
        out[static_cast<int64_t>(m0 + rr) * R + nb + cc] =
            __bfloat16_as_ushort(__float2bfloat16_rn(v * scale));
      }
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// col-wise skinny GEMM (reduction over tokens).  CTA = 4 warps on a 128-wide
// p tile and a chunk of kColChunk tokens; 32-token steps are staged in shared
// memory with cp.async (double buffered, rows padded to an odd number of
// 16-byte units so ldmatrix.trans is conflict free) and consumed with
// ldmatrix.trans + mma.  Each warp owns 32 p rows x 64 n columns.
// ---------------------------------------------------------------------------
constexpr int kColChunk = 256;
constexpr int kColThreads = 128;
constexpr int kActStride = 128 * 2 + 16;   // bytes per staged act row (17 x 16 B)
constexpr int kUStride = 64 * 2 + 16;      // bytes per staged u row   (9 x 16 B)

__global__ void __launch_bounds__(kColThreads) colwise_skinny_kernel(
    const uint16_t* __restrict__ act, const uint16_t* __restrict__ u,
    float* __restrict__ part, int M, int P, int R) {
  __shared__ __align__(128) uint8_t s_act[2][32 * kActStride];
  __shared__ __align__(128) uint8_t s_u[2][32 * kUStride];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int p0 = blockIdx.x * 128;
  const int chunk = blockIdx.y;
  const int mb = chunk * kColChunk;
  const int m_end = min(M, mb + kColChunk);
  const int n_steps = (m_end - mb + 31) / 32;

  for (int nb = 0; nb < R; nb += 64) {
    const int nt = min(8, (R - nb) / 8);
    float acc[2][8][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j][0] = acc[i][j][1] = acc[i][j][2] = acc[i][j][3] = 0.f;

    auto stage = [&](int st, int buf) {
      const int ms = mb + st * 32;
      // act tile: 32 rows x 128 p = 512 16-byte pieces
      for (int e = threadIdx.x; e < 512; e += kColThreads) {
        const int row = e >> 4, pc = e & 15;
        const int m = ms + row, p = p0 + pc * 8;
        const bool ok = (m < m_end) && (p < P);
        const uint16_t* src = act + static_cast<int64_t>(ok ? m : 0) * P + (ok ? p : 0);
        cp_async_16(smem_u32(&s_act[buf][row * kActStride + pc * 16]), src, ok);
      }
      // u tile: 32 rows x 64 n = 256 pieces
      for (int e = threadIdx.x; e < 256; e += kColThreads) {
        const int row = e >> 3, nc = e & 7;
        const int m = ms + row, n = nb + nc * 8;
        const bool ok = (m < m_end) && (n < R);
        const uint16_t* src = u + static_cast<int64_t>(ok ? m : 0) * R + (ok ? n : 0);
        cp_async_16(smem_u32(&s_u[buf][row * kUStride + nc * 16]), src, ok);
      }
      cp_async_commit();
    };

    if (n_steps > 0) stage(0, 0);
    for (int st = 0; st < n_steps; ++st) {
      const int buf = st & 1;
      if (st + 1 < n_steps) { stage(st + 1, buf ^ 1); cp_async_wait<1>(); }
      else { cp_async_wait<0>(); }
      __syncthreads();
      const uint32_t a_base = smem_u32(s_act[buf]);
      const uint32_t u_base = smem_u32(s_u[buf]);
      const int mi = lane >> 3, ri = lane & 7;
#pragma unroll
      for (int ks = 0; ks < 2; ++ks) {           // two 16-token MMA steps
        uint32_t a[2][4];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int mrow = ks * 16 + ((mi >> 1) << 3) + ri;
          const int pcol = warp * 32 + i * 16 + ((mi & 1) << 3);
          ldsm_x4_trans(a_base + mrow * kActStride + pcol * 2, a[i][0], a[i][1], a[i][2], a[i][3]);
        }
#pragma unroll
        for (int jp = 0; jp < 4; ++jp) {          // pairs of n tiles
          if (2 * jp < nt) {
            const int mrow = ks * 16 + ((mi & 1) << 3) + ri;
            const int ncol = jp * 16 + ((mi >> 1) << 3);
            uint32_t b0, b1, b2, b3;
            ldsm_x4_trans(u_base + mrow * kUStride + ncol * 2, b0, b1, b2, b3);
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              mma_bf16_16816(acc[i][2 * jp], a[i][0], a[i][1], a[i][2], a[i][3], b0, b1);
              if (2 * jp + 1 < nt)
                mma_bf16_16816(acc[i][2 * jp + 1], a[i][0], a[i][1], a[i][2], a[i][3], b2, b3);
            }
          }
        }
      }
      __syncthreads();
    }
    // write the partial tile: part[chunk][p][n]
    const int g = lane >> 2, q = lane & 3;
    float* dst = part + static_cast<int64_t>(chunk) * P * R;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int pr = p0 + warp * 32 + i * 16 + g;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < nt) {
          const int n = nb + 8 * j + 2 * q;
          if (pr < P) {
            dst[static_cast<int64_t>(pr) * R + n] = acc[i][j][0];
            dst[static_cast<int64_t>(pr) * R + n + 1] = acc[i][j][1];
          }
          if (pr + 8 < P) {
            dst[static_cast<int64_t>(pr + 8) * R + n] = acc[i][j][2];
            dst[static_cast<int64_t>(pr + 8) * R + n + 1] = acc[i][j][3];
          }
        }
      }
    }
  }
}

// out[p][n] (or out[n][p] when transpose) = sum over chunks c = 0..C-1 of
// part[c][p][n], added in chunk order.
__global__ void __launch_bounds__(256) sum_chunks_kernel(
    const float* __restrict__ part, int C, int P, int R, float* __restrict__ out, int transpose) {
  const int64_t n_el = static_cast<int64_t>(P) * R;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n_el;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float v = 0.f;
    for (int c = 0; c < C; ++c) v += part[static_cast<int64_t>(c) * n_el + e];
    if (transpose) {
      const int64_t p = e / R, n = e % R;
      out[n * P + p] = v;
    } else {
      out[e] = v;
    }
  }
}

// Bt[j][o] = B[o][j]  (B [out, r] -> B^T [r, out]), 32x32 tiles via shared memory.
__global__ void __launch_bounds__(256) transpose_bf16_kernel(
    const uint16_t* __restrict__ src, int rows, int cols, uint16_t* __restrict__ dst) {
  __shared__ uint16_t tile[32][33];
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  for (int i = threadIdx.x; i < 1024; i += 256) {
    const int rr = i >> 5, cc = i & 31;
    if (r0 + rr < rows && c0 + cc < cols) tile[rr][cc] = src[static_cast<int64_t>(r0 + rr) * cols + c0 + cc];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 1024; i += 256) {
    const int cc = i >> 5, rr = i & 31;
    if (r0 + rr < rows && c0 + cc < cols) dst[static_cast<int64_t>(c0 + cc) * rows + r0 + rr] = tile[rr][cc];
  }
}

}  // namespace qnf4
