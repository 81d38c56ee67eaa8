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
// With one K range the result is scaled and rounded to bf16 in place.  With
// several, the K ranges of a row tile form one thread-block cluster along y:
// each CTA leaves its fp32 partial tile in its own shared memory, then every
// CTA adds up its share of the tile over distributed shared memory, partials
// in rank order (deterministic), and scales, rounds and stores it.
// ---------------------------------------------------------------------------
// Sum over the CTAs of this cluster, in rank order, of the float4 at local
// shared address `addr` of each (all loads issued before the first add).
__device__ __forceinline__ float4 cluster_sum_f4(uint32_t addr, int ranks) {
  float4 t[8];
#pragma unroll
  for (int rk = 0; rk < 8; ++rk) {
    t[rk] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (rk < ranks)
      asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                   : "=f"(t[rk].x), "=f"(t[rk].y), "=f"(t[rk].z), "=f"(t[rk].w)
                   : "r"(mapa_shared(addr, rk)) : "memory");
  }
  float4 v = t[0];
#pragma unroll
  for (int rk = 1; rk < 8; ++rk) {
    if (rk < ranks) {
      v.x += t[rk].x; v.y += t[rk].y; v.z += t[rk].z; v.w += t[rk].w;
    }
  }
  return v;
}

// 4-byte asynchronous copy (a row's keep bits for 32 columns), zero-filled when invalid.
__device__ __forceinline__ void cp_async_4(uint32_t smem_dst, const void* src, bool valid) {
  const int n = valid ? 4 : 0;
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" :: "r"(smem_dst), "l"(src), "r"(n) : "memory");
}

// Zero the bf16 values of a 16-byte chunk (8 columns) whose keep bit is 0
// (bit e of `bits` keeps column e): exact, a value is kept or becomes +0.
__device__ __forceinline__ void mask_chunk(uint32_t addr, uint32_t bits) {
  uint32_t w[4];
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "r"(addr)
               : "memory");
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const uint32_t lo = (bits >> (2 * e)) & 1u ? 0x0000FFFFu : 0u;
    const uint32_t hi = (bits >> (2 * e + 1)) & 1u ? 0xFFFF0000u : 0u;
    w[e] &= lo | hi;
  }
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" :: "r"(addr), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3])
               : "memory");
}

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
  static constexpr int MASK_BYTES = 64 * 8;            // keep bits of the 64 x 64 activation tile
  static constexpr int STAGE = kRowActBytes + ((W_BYTES + 127) / 128) * 128 + MASK_BYTES;
  static constexpr int SMEM = kRowStages * STAGE;
  static_assert(64 * RC * 4 <= SMEM, "partial tile must fit the stage ring");
};

template <int NT, bool kKR, bool kMask>
__global__ void __launch_bounds__(kRowThreads) rowwise_skinny_kernel(
    const uint16_t* __restrict__ act, const uint16_t* __restrict__ W,
    uint16_t* __restrict__ out, int M, int K, int R, float scale, int stages_per_split,
    const uint8_t* __restrict__ keep) {
  using C = RowCfg<NT, kKR>;
  extern __shared__ __align__(128) uint8_t s_row[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 64;
  const int nb = blockIdx.z * C::RC;
  const int nt = min(NT, (R - nb) / 8);
  const int kst_begin = blockIdx.y * stages_per_split;
  const int kst_end = min(K / 64, kst_begin + stages_per_split);
  const int n_st = kst_end - kst_begin;

  // activation tile.  With a keep mask (LoRA dropout, kMask) thread t loads
  // chunks 4 (t & 1) .. +3 of row t >> 1 and the matching 4 mask bytes;
  // without, consecutive threads take consecutive chunks.
  const int a_row = threadIdx.x >> 1, a_ch0 = 4 * (threadIdx.x & 1);
  auto stage = [&](int i) {
    uint8_t* sa = s_row + (i % kRowStages) * C::STAGE;
    uint8_t* sw = sa + kRowActBytes;
    const int k0 = (kst_begin + i) * 64;
    if (kMask) {
      const bool ok = m0 + a_row < M;
      const int64_t m = ok ? m0 + a_row : 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int ch = a_ch0 + j;
        cp_async_16(smem_u32(sa + a_row * 128 + ((ch ^ (a_row & 7)) << 4)), act + m * K + k0 + ch * 8, ok);
      }
      cp_async_4(smem_u32(sa + C::STAGE - C::MASK_BYTES + a_row * 8 + a_ch0), keep + (m * K + k0) / 8 + a_ch0, ok);
    } else {
      for (int e = threadIdx.x; e < 64 * 8; e += kRowThreads) {     // activation 64 x 64
        const int row = e >> 3, ch = e & 7;
        const bool ok = m0 + row < M;
        const uint16_t* src = act + static_cast<int64_t>(ok ? m0 + row : 0) * K + k0 + ch * 8;
        cp_async_16(smem_u32(sa + row * 128 + ((ch ^ (row & 7)) << 4)), src, ok);
      }
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
    if (kMask) {                                                     // this thread's own chunks, now landed
      const uint32_t sa = smem_u32(s_row + (i % kRowStages) * C::STAGE);
      uint32_t bits;
      asm volatile("ld.shared.u32 %0, [%1];" : "=r"(bits) : "r"(sa + C::STAGE - C::MASK_BYTES + a_row * 8 + a_ch0)
                   : "memory");
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int ch = a_ch0 + j;
        mask_chunk(sa + a_row * 128 + ((ch ^ (a_row & 7)) << 4), (bits >> (8 * j)) & 0xFFu);
      }
    }
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
  if (gridDim.y == 1) {
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      if (j < nt) {
        const int n = nb + 8 * j + 2 * q;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int m = m0 + warp * 16 + g + 8 * h;
          if (m < M)
            *reinterpret_cast<uint32_t*>(out + static_cast<int64_t>(m) * R + n) =
                pack_bf16x2_rn(acc[j][2 * h] * scale, acc[j][2 * h + 1] * scale);
        }
      }
    }
    return;
  }

  // cluster of the row tile's K ranges: partial tile [64 rows][RC] in shared memory
  __syncthreads();                                                   // every warp is done with the stages
  float* red = reinterpret_cast<float*>(s_row);
#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int h = 0; h < 2; ++h)
      *reinterpret_cast<float2*>(red + (warp * 16 + g + 8 * h) * C::RC + 8 * j + 2 * q) =
          make_float2(acc[j][2 * h], acc[j][2 * h + 1]);
  cluster_sync_all();
  {
    // every CTA of the cluster reduces and stores its share of the tile
    const int ks = static_cast<int>(gridDim.y), rank = static_cast<int>(cluster_ctarank());
    constexpr int n4 = 64 * C::RC / 4;
    const uint32_t red_addr = smem_u32(red);
    for (int e = rank * n4 / ks + threadIdx.x; e < (rank + 1) * n4 / ks; e += kRowThreads) {
      const int row = e / (C::RC / 4), c4 = e % (C::RC / 4);
      const float4 v = cluster_sum_f4(red_addr + e * 16, ks);
      const int m = m0 + row, n = nb + 4 * c4;
      if (m < M && n < R)
        *reinterpret_cast<uint2*>(out + static_cast<int64_t>(m) * R + n) =
            make_uint2(pack_bf16x2_rn(v.x * scale, v.y * scale), pack_bf16x2_rn(v.z * scale, v.w * scale));
    }
  }
  cluster_sync_all();                                                // partials stay until all are read
}

// ---------------------------------------------------------------------------
// col-wise skinny GEMM (reduction over tokens), both backward problems in one
// launch (blockIdx.z): dB = dh^T us and dA = du^T x.  CTA = 4 warps on a
// 128-wide p tile and one token chunk; 32-token steps are staged in shared
// memory with cp.async in a kColStages-deep ring (rows padded to an odd number
// of 16-byte units so ldmatrix.trans is conflict free) and consumed with
// ldmatrix.trans + mma.  Each warp owns 32 p rows x 64 n columns.  The token
// chunks of a p tile form one thread-block cluster along y (at most 8): each
// CTA leaves its fp32 partial tile in shared memory, in the orientation of the
// output ([p][n] for dB [out, r], [n][p] for dA [r, in]), then every CTA adds
// up its share of the tile over distributed shared memory, partials in rank
// order (deterministic), and stores it.
// ---------------------------------------------------------------------------
constexpr int kColMaxChunks = 8;
constexpr int kColThreads = 128;
constexpr int kColStages = 4;
constexpr int kActStride = 128 * 2 + 16;   // bytes per staged act row (17 x 16 B)
constexpr int kUStride = 64 * 2 + 16;      // bytes per staged u row   (9 x 16 B)
constexpr int kColMaskBytes = 32 * 16;      // keep bits of the 32 x 128 activation tile
constexpr int kColStageBytes = 32 * kActStride + 32 * kUStride + kColMaskBytes;
static_assert(128 * 64 * 4 <= kColStages * kColStageBytes, "partial tile must fit the stage ring");

struct ColProblem {
  const uint16_t* act;   // [M, P]
  const uint16_t* u;     // [M, R]
  float* out;            // [P][R] (dB) or [R][P] (dA)
  int P;
  int n_major;           // 1: output layout [n][p]
  float scale;           // applied to the reduced sum before it is stored
  const uint8_t* keep;   // keep bits of act ([M][P/8], bit i % 8 of byte i / 8), or null
};

template <bool kMask>
__global__ void __launch_bounds__(kColThreads, kMask ? 4 : 1) colwise_skinny_kernel(ColProblem prob0, ColProblem prob1,
                                                                        int M, int R, int chunk_tokens) {
  extern __shared__ __align__(128) uint8_t s_col[];
  const ColProblem pr = blockIdx.z == 0 ? prob0 : prob1;
  const int P = pr.P;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int p0 = blockIdx.x * 128;
  // a p tile past P still takes part in its cluster's barriers (with no work)
  const bool p_live = p0 < P;
  const int chunk = blockIdx.y;
  const int mb = chunk * chunk_tokens;
  const int m_end = min(M, mb + chunk_tokens);
  const int n_steps = p_live && m_end > mb ? (m_end - mb + 31) / 32 : 0;
  const int mi = lane >> 3, ri = lane & 7;

  for (int nb = 0; nb < R; nb += 64) {
    const int nt = min(8, (R - nb) / 8);
    float acc[2][8][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j][0] = acc[i][j][1] = acc[i][j][2] = acc[i][j][3] = 0.f;

    // activation tile.  With keep masks (LoRA dropout, kMask) thread t loads
    // chunks 4 (t & 3) .. +3 of row t >> 2 and the matching 4 mask bytes;
    // without, consecutive threads take consecutive chunks.
    const int a_row = threadIdx.x >> 2, a_pc0 = 4 * (threadIdx.x & 3);
    auto stage = [&](int st) {
      uint8_t* s_act = s_col + (st % kColStages) * kColStageBytes;
      uint8_t* s_u = s_act + 32 * kActStride;
      const int ms = mb + st * 32;
      if (!kMask) {
        for (int e = threadIdx.x; e < 512; e += kColThreads) {    // 32 rows x 128 p
          const int row = e >> 4, pc = e & 15;
          const int m = ms + row, p = p0 + pc * 8;
          const bool ok = (m < m_end) && (p < P);
          const uint16_t* src = pr.act + static_cast<int64_t>(ok ? m : 0) * P + (ok ? p : 0);
          cp_async_16(smem_u32(s_act + row * kActStride + pc * 16), src, ok);
        }
      } else {
        const int m = ms + a_row;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int pc = a_pc0 + j, p = p0 + pc * 8;
          const bool ok = (m < m_end) && (p < P);
          const uint16_t* src = pr.act + static_cast<int64_t>(ok ? m : 0) * P + (ok ? p : 0);
          cp_async_16(smem_u32(s_act + a_row * kActStride + pc * 16), src, ok);
        }
        if (pr.keep != nullptr) {
          const bool ok = (m < m_end) && (p0 + a_pc0 * 8 < P);
          const uint8_t* src = pr.keep + (static_cast<int64_t>(ok ? m : 0) * P + (ok ? p0 : 0)) / 8 + (ok ? a_pc0 : 0);
          cp_async_4(smem_u32(s_act + kColStageBytes - kColMaskBytes + a_row * 16 + a_pc0), src, ok);
        }
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
      if (kMask && pr.keep != nullptr) {                           // this thread's own chunks, now landed
        const uint32_t sa = smem_u32(s_col + (st % kColStages) * kColStageBytes);
        uint32_t bits;
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(bits)
                     : "r"(sa + kColStageBytes - kColMaskBytes + a_row * 16 + a_pc0) : "memory");
#pragma unroll
        for (int j = 0; j < 4; ++j) mask_chunk(sa + a_row * kActStride + (a_pc0 + j) * 16, (bits >> (8 * j)) & 0xFFu);
      }
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
    // partial tile [128 p][64 n] (dB) or [64 n][128 p] (dA) in shared memory
    const int g = lane >> 2, q = lane & 3;
    float* red = reinterpret_cast<float*>(s_col);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int pl = warp * 32 + i * 16 + g;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int nl = 8 * j + 2 * q;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (pr.n_major) {
            red[nl * 128 + pl + 8 * h] = acc[i][j][2 * h];
            red[(nl + 1) * 128 + pl + 8 * h] = acc[i][j][2 * h + 1];
          } else {
            *reinterpret_cast<float2*>(red + (pl + 8 * h) * 64 + nl) = make_float2(acc[i][j][2 * h], acc[i][j][2 * h + 1]);
          }
        }
      }
    }
    cluster_sync_all();
    if (p_live) {
      // every CTA of the cluster reduces (chunks in rank order) and stores its share of the tile
      const int ks = static_cast<int>(gridDim.y), rank = static_cast<int>(cluster_ctarank());
      constexpr int n4 = 128 * 64 / 4;
      const uint32_t red_addr = smem_u32(red);
      for (int e = rank * n4 / ks + threadIdx.x; e < (rank + 1) * n4 / ks; e += kColThreads) {
        float4 v = cluster_sum_f4(red_addr + e * 16, ks);
        if (pr.scale != 1.f) {
          v.x = __fmul_rn(v.x, pr.scale); v.y = __fmul_rn(v.y, pr.scale);
          v.z = __fmul_rn(v.z, pr.scale); v.w = __fmul_rn(v.w, pr.scale);
        }
        if (pr.n_major) {                                            // red [n][p]: 4 consecutive p
          const int nl = e / 32, pl = (e % 32) * 4;
          if (nl < 8 * nt && p0 + pl < P)
            *reinterpret_cast<float4*>(pr.out + static_cast<int64_t>(nb + nl) * P + p0 + pl) = v;
        } else {                                                     // red [p][n]: 4 consecutive n
          const int pl = e / 16, nl = (e % 16) * 4;
          if (nl < 8 * nt && p0 + pl < P)
            *reinterpret_cast<float4*>(pr.out + static_cast<int64_t>(p0 + pl) * R + nb + nl) = v;
        }
      }
    }
    cluster_sync_all();                                              // partials stay until all are read
  }
}

}  // namespace qnf4
