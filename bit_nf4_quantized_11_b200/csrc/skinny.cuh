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
// row-wise skinny GEMM: out[m][n] = scale * sum_k act[m][k] * W[n][k] for n in
// one 64-wide chunk of the rank (grid.z), over one K range (grid.y).
// CTA = 4 warps on 64 token rows; K is streamed in 64-wide stages through a
// kRowStages-deep cp.async ring (the activation tile and the matching W tile),
// consumed with ldmatrix + mma.sync (each warp owns 16 rows x 8*NT columns).
// W is either [R][K] (k contiguous, ldmatrix) or [K][R] (n contiguous,
// ldmatrix.trans), so neither orientation needs a transposed copy.
// Activation rows are 128 B in shared memory with the 16-byte chunk index
// XOR-ed by (row & 7), so every ldmatrix phase hits 8 different bank groups.
// With one K range the result is scaled and rounded to bf16 in place;
// otherwise fp32 partials go to part[split][row][n] for the finalize kernel.
// ---------------------------------------------------------------------------
constexpr int kRowThreads = 128;
constexpr int kRowStages = 4;
constexpr int kRowActBytes = 64 * 128;                  // 64 rows x 64 k bf16

template <int NT, bool kKR>
struct RowCfg {
  static constexpr int RC = 8 * NT;                     // rank columns per CTA
  // The tile always spans at least 16 rank columns (an x4 ldmatrix reads two
  // 8-column tiles); columns past the rank are zero-filled.
  static constexpr int RCA = RC < 16 ? 16 : RC;
  static constexpr int NTA = RCA / 8;
  // W tile: [RCA rows x 64 k] (128 B rows, swizzled) or [64 k rows x RCA n] (padded rows)
  static constexpr int W_PITCH = kKR ? (RCA * 2 + ((RCA * 2 / 16) % 2 == 0 ? 16 : 0)) : 128;
  static constexpr int W_BYTES = kKR ? 64 * W_PITCH : RCA * 128;
  static constexpr int STAGE = kRowActBytes + ((W_BYTES + 127) / 128) * 128;
  static constexpr int SMEM = kRowStages * STAGE;
};

template <int NT, bool kKR>
__global__ void __launch_bounds__(kRowThreads) rowwise_skinny_kernel(
    const uint16_t* __restrict__ act, const uint16_t* __restrict__ W,
    uint16_t* __restrict__ out, float* __restrict__ part, int M, int K, int R, float scale,
    int stages_per_split) {
  using C = RowCfg<NT, kKR>;
  extern __shared__ __align__(128) uint8_t s_row[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 64;
  const int nb = blockIdx.z * C::RC;
  const int nt = min(NT, (R - nb) / 8);
  const int kst_begin = blockIdx.y * stages_per_split;
  const int kst_end = min(K / 64, kst_begin + stages_per_split);
  const int n_st = kst_end - kst_begin;

  auto stage = [&](int i) {
    uint8_t* sa = s_row + (i % kRowStages) * C::STAGE;
    uint8_t* sw = sa + kRowActBytes;
    const int k0 = (kst_begin + i) * 64;
    for (int e = threadIdx.x; e < 64 * 8; e += kRowThreads) {       // activation 64 x 64
      const int row = e >> 3, ch = e & 7;
      const bool ok = m0 + row < M;
      const uint16_t* src = act + static_cast<int64_t>(ok ? m0 + row : 0) * K + k0 + ch * 8;
      cp_async_16(smem_u32(sa + row * 128 + ((ch ^ (row & 7)) << 4)), src, ok);
    }
    if (!kKR) {
      for (int e = threadIdx.x; e < C::RCA * 8; e += kRowThreads) {  // W rows n, 64 k
        const int row = e >> 3, ch = e & 7;
        const bool ok = row < C::RC && nb + row < R;
        const uint16_t* src = W + static_cast<int64_t>(ok ? nb + row : 0) * K + k0 + ch * 8;
        cp_async_16(smem_u32(sw + row * 128 + ((ch ^ (row & 7)) << 4)), src, ok);
      }
    } else {
      for (int e = threadIdx.x; e < 64 * C::NTA; e += kRowThreads) { // W rows k, RCA n
        const int row = e / C::NTA, ch = e % C::NTA;
        const bool ok = ch < NT && nb + ch * 8 < R;
        const uint16_t* src = W + static_cast<int64_t>(k0 + row) * R + (ok ? nb + ch * 8 : 0);
        cp_async_16(smem_u32(sw + row * C::W_PITCH + ch * 16), src, ok);
      }
    }
  };

  float acc[NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;

#pragma unroll
  for (int i = 0; i < kRowStages - 1; ++i) {
    if (i < n_st) stage(i);
    cp_async_commit();
  }
  for (int i = 0; i < n_st; ++i) {
    cp_async_wait<kRowStages - 2>();
    __syncthreads();
    if (i + kRowStages - 1 < n_st) stage(i + kRowStages - 1);
    cp_async_commit();
    const uint32_t sa = smem_u32(s_row + (i % kRowStages) * C::STAGE);
    const uint32_t sw = sa + kRowActBytes;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t a0, a1, a2, a3;
      {
        const int row = warp * 16 + (lane & 15);
        const int ch = 2 * kk + (lane >> 4);
        ldsm_x4(sa + row * 128 + ((ch ^ (row & 7)) << 4), a0, a1, a2, a3);
      }
#pragma unroll
      for (int jp = 0; jp < NT; jp += 2) {
        if (jp < nt) {
          uint32_t b0, b1, b2, b3;
          if (!kKR) {
            // matrices: (n jp*8.., k lo), (n jp*8.., k hi), (n jp*8+8.., k lo), (n jp*8+8.., k hi)
            const int mi = lane >> 3;
            const int row = jp * 8 + ((mi >> 1) << 3) + (lane & 7);
            const int ch = 2 * kk + (mi & 1);
            ldsm_x4(sw + row * 128 + ((ch ^ (row & 7)) << 4), b0, b1, b2, b3);
          } else {
            // matrices: (k lo, n jp*8..), (k hi, n jp*8..), (k lo, n jp*8+8..), (k hi, n jp*8+8..)
            const int mi = lane >> 3;
            const int krow = kk * 16 + ((mi & 1) << 3) + (lane & 7);
            const int ncol = jp * 8 + ((mi >> 1) << 3);
            ldsm_x4_trans(sw + krow * C::W_PITCH + ncol * 2, b0, b1, b2, b3);
          }
          mma_bf16_16816(acc[jp], a0, a1, a2, a3, b0, b1);
          if (jp + 1 < nt) mma_bf16_16816(acc[jp + 1], a0, a1, a2, a3, b2, b3);
        }
      }
    }
  }
  cp_async_wait<0>();

  const int g = lane >> 2, q = lane & 3;
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    if (j < nt) {
      const int n = nb + 8 * j + 2 * q;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int m = m0 + warp * 16 + g + 8 * h;
        if (m < M) {
          const float v0 = acc[j][2 * h], v1 = acc[j][2 * h + 1];
          if (part == nullptr) {
            *reinterpret_cast<uint32_t*>(out + static_cast<int64_t>(m) * R + n) =
                pack_bf16x2_rn(v0 * scale, v1 * scale);
          } else {
            *reinterpret_cast<float2*>(part + (static_cast<int64_t>(blockIdx.y) * M + m) * R + n) =
                make_float2(v0, v1);
          }
        }
      }
    }
  }
}

// out[m][n] = bf16(scale * sum_{s < splits} part[s][m][n]), splits added in
// order; four outputs per thread (M*R is a multiple of 8).
__global__ void __launch_bounds__(256) rowwise_finalize_kernel(
    const float* __restrict__ part, int splits, int M, int R, float scale, uint16_t* __restrict__ out) {
  const int64_t n4 = static_cast<int64_t>(M) * R / 4;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n4;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    const float4* p = reinterpret_cast<const float4*>(part) + e;
#pragma unroll 4
    for (int s = 0; s < splits; ++s) {
      const float4 t = __ldg(p + static_cast<int64_t>(s) * n4);
      v.x += t.x; v.y += t.y; v.z += t.z; v.w += t.w;
    }
    reinterpret_cast<uint2*>(out)[e] =
        make_uint2(pack_bf16x2_rn(v.x * scale, v.y * scale), pack_bf16x2_rn(v.z * scale, v.w * scale));
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
#pragma unroll 4
    for (int c = 0; c < C; ++c) {
      const float4 t = __ldg(reinterpret_cast<const float4*>(part) + c * stride + e);
      v.x += t.x; v.y += t.y; v.z += t.z; v.w += t.w;
    }
    reinterpret_cast<float4*>(out)[e] = v;
  }
}

}  // namespace qnf4
