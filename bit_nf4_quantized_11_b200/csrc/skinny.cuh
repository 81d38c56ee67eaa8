// skinny.cuh -- the rank-r contractions of the QLoRA layer (sm_100a).
//
// All of them have one dimension equal to the LoRA rank r (8..256), stream a
// token-sized operand from HBM once and are bound by that read, so they run
// on warp-level bf16 MMA (fp32 accumulation) with coalesced 16-byte loads:
//
//   row-wise  out[m][n] = bf16(scale * sum_k act[m][k] * Wt[n][k])
//       forward   us = bf16(s x A^T)      act = x  [M, in],  Wt = A  [r, in]
//       backward  du = bf16(s dh B)       act = dh [M, out], W  = B   [out, r]
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
// row-wise skinny GEMM.  CTA = 8 warps on 16 token rows and one K range
// (blockIdx.y splits K when there are few rows); the K range is cut into
// 32-wide chunks dealt round-robin to the warps, which load a batch of chunks
// before issuing its MMAs so that several loads are in flight per thread.
// The MMA's K order is permuted consistently for both operands (thread q of a
// quad owns physical k = 8q..8q+7 of every 32-chunk), so each activation
// fragment is one 16-byte load.  The second operand is either Wt [R][K]
// (k contiguous: one 16-byte load per n-tile) or W [K][R] (n contiguous:
// element loads that stay in L1, so no transposed copy is needed).
// Warp partials are reduced through shared memory in a fixed order; with
// one K range the result is scaled and rounded to bf16, otherwise fp32
// partials go to part[split][row][n] for rowwise_finalize_kernel.
// Output columns are processed 8*NT at a time.
// ---------------------------------------------------------------------------
constexpr int kRowThreads = 256;

template <int NT, bool kKR>
__device__ __forceinline__ void rowwise_b_frag(const uint16_t* __restrict__ W, int K, int R, int nb, int j,
                                               int g, int q, int k0, uint4& b) {
  if (!kKR) {
    b = ld_nc_v4(W + static_cast<int64_t>(nb + 8 * j + g) * K + k0 + 8 * q);
  } else {
    const uint16_t* p = W + static_cast<int64_t>(k0 + 8 * q) * R + nb + 8 * j + g;
    uint32_t e[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) e[i] = __ldg(p + static_cast<int64_t>(i) * R);
    b = make_uint4(e[0] | (e[1] << 16), e[2] | (e[3] << 16), e[4] | (e[5] << 16), e[6] | (e[7] << 16));
  }
}

template <int NT, bool kKR>
__global__ void __launch_bounds__(kRowThreads) rowwise_skinny_kernel(
    const uint16_t* __restrict__ act, const uint16_t* __restrict__ W,
    uint16_t* __restrict__ out, float* __restrict__ part, int M, int K, int R, float scale,
    int chunks_per_split) {
  constexpr int kBatch = NT <= 2 ? 4 : (NT == 4 ? 2 : 1);
  __shared__ float s_red[8][16][8 * NT + 1];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
  const int m0 = blockIdx.x * 16;
  const int c_begin = blockIdx.y * chunks_per_split;
  const int c_end = min(K / 32, c_begin + chunks_per_split);
  const bool row0 = (m0 + g) < M, row1 = (m0 + g + 8) < M;
  const uint16_t* a_row0 = act + static_cast<int64_t>(row0 ? m0 + g : 0) * K + 8 * q;
  const uint16_t* a_row1 = act + static_cast<int64_t>(row1 ? m0 + g + 8 : 0) * K + 8 * q;
  const uint4 z = make_uint4(0, 0, 0, 0);

  for (int nb = 0; nb < R; nb += 8 * NT) {
    const int nt = min(NT, (R - nb) / 8);
    float acc[NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;

    for (int c = c_begin + warp; c < c_end; c += 8 * kBatch) {
      uint4 u0[kBatch], u1[kBatch], b[kBatch][NT];
#pragma unroll
      for (int bi = 0; bi < kBatch; ++bi) {
        const int cc = c + 8 * bi;
        const bool ok = cc < c_end;
        const int k0 = cc * 32;
        u0[bi] = (ok && row0) ? ld_nc_v4(a_row0 + k0) : z;
        u1[bi] = (ok && row1) ? ld_nc_v4(a_row1 + k0) : z;
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          b[bi][j] = z;
          if (ok && j < nt) rowwise_b_frag<NT, kKR>(W, K, R, nb, j, g, q, k0, b[bi][j]);
        }
      }
#pragma unroll
      for (int bi = 0; bi < kBatch; ++bi) {
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          if (j < nt) {
            mma_bf16_16816(acc[j], u0[bi].x, u1[bi].x, u0[bi].y, u1[bi].y, b[bi][j].x, b[bi][j].y);
            mma_bf16_16816(acc[j], u0[bi].z, u1[bi].z, u0[bi].w, u1[bi].w, b[bi][j].z, b[bi][j].w);
          }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      s_red[warp][g][8 * j + 2 * q] = acc[j][0];
      s_red[warp][g][8 * j + 2 * q + 1] = acc[j][1];
      s_red[warp][g + 8][8 * j + 2 * q] = acc[j][2];
      s_red[warp][g + 8][8 * j + 2 * q + 1] = acc[j][3];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < 16 * 8 * NT; e += kRowThreads) {
      const int rr = e / (8 * NT), cc = e % (8 * NT);
      if (cc < nt * 8 && m0 + rr < M) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) v += s_red[w][rr][cc];
        if (part == nullptr) {
          out[static_cast<int64_t>(m0 + rr) * R + nb + cc] = __bfloat16_as_ushort(__float2bfloat16_rn(v * scale));
        } else {
          part[(static_cast<int64_t>(blockIdx.y) * M + m0 + rr) * R + nb + cc] = v;
        }
      }
    }
    __syncthreads();
  }
}

// out[m][n] = bf16(scale * sum_{s < splits} part[s][m][n]), splits added in order.
__global__ void __launch_bounds__(256) rowwise_finalize_kernel(
    const float* __restrict__ part, int splits, int M, int R, float scale, uint16_t* __restrict__ out) {
  const int64_t n_el = static_cast<int64_t>(M) * R;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n_el;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float v = 0.f;
    for (int s = 0; s < splits; ++s) v += part[static_cast<int64_t>(s) * n_el + e];
    out[e] = __bfloat16_as_ushort(__float2bfloat16_rn(v * scale));
  }
}

// ---------------------------------------------------------------------------
// col-wise skinny GEMM (reduction over tokens), both backward problems in one
// launch (blockIdx.z): dB = dh^T us and dA^T = x^T du.  CTA = 4 warps on a
// 128-wide p tile and a chunk of kColChunk tokens; 32-token steps are staged
// in shared memory with cp.async in a kColStages-deep ring (rows padded to an
// odd number of 16-byte units so ldmatrix.trans is conflict free) and consumed
// with ldmatrix.trans + mma.  Each warp owns 32 p rows x 64 n columns.
// Partials are written in the orientation of the final output: [c][p][n] for
// dB (out, r) and [c][n][p] for dA (r, in), so the chunk sum is elementwise.
// ---------------------------------------------------------------------------
constexpr int kColChunk = 512;
constexpr int kColThreads = 128;
constexpr int kColStages = 4;
constexpr int kActStride = 128 * 2 + 16;   // bytes per staged act row (17 x 16 B)
constexpr int kUStride = 64 * 2 + 16;      // bytes per staged u row   (9 x 16 B)
constexpr int kColStageBytes = 32 * kActStride + 32 * kUStride;

struct ColProblem {
  const uint16_t* act;   // [M, P]
  const uint16_t* u;     // [M, R]
  float* part;           // [chunks][P][R] or [chunks][R][P]
  int P;
  int n_major;           // 1: partial layout [c][n][p]
};

__global__ void __launch_bounds__(kColThreads) colwise_skinny_kernel(ColProblem prob0, ColProblem prob1,
                                                                     int M, int R) {
  extern __shared__ __align__(128) uint8_t s_col[];
  const ColProblem pr = blockIdx.z == 0 ? prob0 : prob1;
  const int P = pr.P;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int p0 = blockIdx.x * 128;
  if (p0 >= P) return;                                   // CTA-uniform
  const int chunk = blockIdx.y;
  const int mb = chunk * kColChunk;
  const int m_end = min(M, mb + kColChunk);
  const int n_steps = (m_end - mb + 31) / 32;
  const int mi = lane >> 3, ri = lane & 7;

  for (int nb = 0; nb < R; nb += 64) {
    const int nt = min(8, (R - nb) / 8);
    float acc[2][8][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j][0] = acc[i][j][1] = acc[i][j][2] = acc[i][j][3] = 0.f;

    auto stage = [&](int st) {
      uint8_t* s_act = s_col + (st % kColStages) * kColStageBytes;
      uint8_t* s_u = s_act + 32 * kActStride;
      const int ms = mb + st * 32;
      for (int e = threadIdx.x; e < 512; e += kColThreads) {      // 32 rows x 128 p
        const int row = e >> 4, pc = e & 15;
        const int m = ms + row, p = p0 + pc * 8;
        const bool ok = (m < m_end) && (p < P);
        const uint16_t* src = pr.act + static_cast<int64_t>(ok ? m : 0) * P + (ok ? p : 0);
        cp_async_16(smem_u32(s_act + row * kActStride + pc * 16), src, ok);
      }
      for (int e = threadIdx.x; e < 256; e += kColThreads) {      // 32 rows x 64 n
        const int row = e >> 3, nc = e & 7;
        const int m = ms + row, n = nb + nc * 8;
        const bool ok = (m < m_end) && (n < R);
        const uint16_t* src = pr.u + static_cast<int64_t>(ok ? m : 0) * R + (ok ? n : 0);
        cp_async_16(smem_u32(s_u + row * kUStride + nc * 16), src, ok);
      }
    };

#pragma unroll
    for (int st = 0; st < kColStages - 1; ++st) {
      if (st < n_steps) stage(st);
      cp_async_commit();                                   // empty groups keep the count uniform
    }
    for (int st = 0; st < n_steps; ++st) {
      cp_async_wait<kColStages - 2>();
      __syncthreads();
      if (st + kColStages - 1 < n_steps) stage(st + kColStages - 1);
      cp_async_commit();
      const uint8_t* s_act = s_col + (st % kColStages) * kColStageBytes;
      const uint32_t a_base = smem_u32(s_act);
      const uint32_t u_base = a_base + 32 * kActStride;
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
    }
    cp_async_wait<0>();
    __syncthreads();
    // write the partial tile
    const int g = lane >> 2, q = lane & 3;
    float* dst = pr.part + static_cast<int64_t>(chunk) * P * R;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int pa = p0 + warp * 32 + i * 16 + g;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < nt) {
          const int n = nb + 8 * j + 2 * q;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int pp = pa + 8 * h;
            if (pp < P) {
              if (pr.n_major) {
                dst[static_cast<int64_t>(n) * P + pp] = acc[i][j][2 * h];
                dst[static_cast<int64_t>(n + 1) * P + pp] = acc[i][j][2 * h + 1];
              } else {
                *reinterpret_cast<float2*>(dst + static_cast<int64_t>(pp) * R + n) =
                    make_float2(acc[i][j][2 * h], acc[i][j][2 * h + 1]);
              }
            }
          }
        }
      }
    }
  }
}

// out_z[e] = sum over chunks c = 0..C-1 of part_z[c][e], in chunk order, for
// the two problems z = blockIdx.y (float4-vectorised; n_el % 4 == 0).
__global__ void __launch_bounds__(256) sum_chunks_kernel(
    const float* __restrict__ part0, float* __restrict__ out0, int64_t n_el0,
    const float* __restrict__ part1, float* __restrict__ out1, int64_t n_el1, int C) {
  const float* part = blockIdx.y == 0 ? part0 : part1;
  float* out = blockIdx.y == 0 ? out0 : out1;
  const int64_t n4 = (blockIdx.y == 0 ? n_el0 : n_el1) / 4;
  const int64_t stride = n4;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n4;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = 0; c < C; ++c) {
      const float4 t = __ldg(reinterpret_cast<const float4*>(part) + c * stride + e);
      v.x += t.x; v.y += t.y; v.z += t.z; v.w += t.w;
    }
    reinterpret_cast<float4*>(out)[e] = v;
  }
}

}  // namespace qnf4
