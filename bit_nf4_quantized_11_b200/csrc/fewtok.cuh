// fewtok.cuh -- the rank-r product of the few-token forward (M <= 16):
//   us[m][j] = bf16( s * sum_k (x[m][k] * keep[m][k]) A[j][k] )
// ("QLoRA", llm-compass, 方法与公式: the B A x branch; keep = 1 without LoRA
// dropout).  With a handful of tokens this is a tiny contraction (M x r
// outputs) over a long K, so it is split over many CTAs rather than tiled:
// CTA c takes the 256 K columns [256 c, 256 c + 256), stages that slice of x
// (masked, as fp32) in shared memory, and each warp forms the partial dot
// products of its rows of A with every token; the partials go to the
// workspace, and the CTA that finishes last (a ticket the host zeroes before
// the launch) adds them in chunk order, so the result does not depend on
// which CTA ran when.
#pragma once

#include "common.cuh"

namespace qnf4 {

constexpr int kFtChunk = 256;       // K columns per CTA
constexpr int kFtThreads = 256;
constexpr int kFtMaxTok = 16;

// Workspace of the partials: [chunks][16][r] fp32.
__host__ __device__ constexpr int64_t fewtok_part_floats(int64_t K, int r) {
  return (K + kFtChunk - 1) / kFtChunk * kFtMaxTok * r;
}

__device__ __forceinline__ float fewtok_bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float fewtok_bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// kTok: token rows processed (8 or 16, >= M).  r % 8 == 0, K % 64 == 0.
template <int kTok>
__global__ void __launch_bounds__(kFtThreads) fewtok_us_kernel(
    const uint16_t* __restrict__ x, const uint8_t* __restrict__ keep, const uint16_t* __restrict__ A, int M,
    int64_t K, int r, float s, float* __restrict__ part, unsigned int* __restrict__ ticket,
    uint16_t* __restrict__ us) {
  __shared__ __align__(16) float xs[kTok][kFtChunk];
  __shared__ bool is_last;
  const int c = blockIdx.x;
  const int64_t k0 = static_cast<int64_t>(c) * kFtChunk;
  const int kc = K - k0 < kFtChunk ? static_cast<int>(K - k0) : kFtChunk;   // a multiple of 64
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // x[m][k0 .. k0 + kc) * keep as fp32, zero past M and past kc
  for (int e = threadIdx.x; e < kTok * (kFtChunk / 8); e += kFtThreads) {
    const int m = e / (kFtChunk / 8), c8 = e % (kFtChunk / 8);
    uint4 v = make_uint4(0, 0, 0, 0);
    if (m < M && 8 * c8 < kc) {
      v = __ldg(reinterpret_cast<const uint4*>(x + m * K + k0 + 8 * c8));
      if (keep != nullptr) {
        const uint32_t kb = __ldg(keep + m * (K / 8) + k0 / 8 + c8);
        v.x &= ((kb & 1u) ? 0x0000FFFFu : 0u) | ((kb & 2u) ? 0xFFFF0000u : 0u);
        v.y &= ((kb & 4u) ? 0x0000FFFFu : 0u) | ((kb & 8u) ? 0xFFFF0000u : 0u);
        v.z &= ((kb & 16u) ? 0x0000FFFFu : 0u) | ((kb & 32u) ? 0xFFFF0000u : 0u);
        v.w &= ((kb & 64u) ? 0x0000FFFFu : 0u) | ((kb & 128u) ? 0xFFFF0000u : 0u);
      }
    }
    float* d = &xs[m][8 * c8];
    *reinterpret_cast<float4*>(d) = make_float4(fewtok_bf16_lo(v.x), fewtok_bf16_hi(v.x), fewtok_bf16_lo(v.y),
                                                fewtok_bf16_hi(v.y));
    *reinterpret_cast<float4*>(d + 4) = make_float4(fewtok_bf16_lo(v.z), fewtok_bf16_hi(v.z), fewtok_bf16_lo(v.w),
                                                    fewtok_bf16_hi(v.w));
  }
  __syncthreads();

  // warp w: rows j = w, w + 8, ... of A; lane l: columns 8 l .. 8 l + 7 of the chunk
  const bool col_ok = 8 * lane < kc;
  for (int j = warp; j < r; j += kFtThreads / 32) {
    float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (col_ok) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(A + j * K + k0 + 8 * lane));
      a[0] = fewtok_bf16_lo(v.x); a[1] = fewtok_bf16_hi(v.x);
      a[2] = fewtok_bf16_lo(v.y); a[3] = fewtok_bf16_hi(v.y);
      a[4] = fewtok_bf16_lo(v.z); a[5] = fewtok_bf16_hi(v.z);
      a[6] = fewtok_bf16_lo(v.w); a[7] = fewtok_bf16_hi(v.w);
    }
    float p[kTok];
#pragma unroll
    for (int m = 0; m < kTok; ++m) {
      const float4 x0 = *reinterpret_cast<const float4*>(&xs[m][8 * lane]);
      const float4 x1 = *reinterpret_cast<const float4*>(&xs[m][8 * lane + 4]);
      float v = a[0] * x0.x;
      v = fmaf(a[1], x0.y, v);
      v = fmaf(a[2], x0.z, v);
      v = fmaf(a[3], x0.w, v);
      v = fmaf(a[4], x1.x, v);
      v = fmaf(a[5], x1.y, v);
      v = fmaf(a[6], x1.z, v);
      v = fmaf(a[7], x1.w, v);
      p[m] = v;
    }
    // Sum each token's value over the 32 lanes with the xor butterfly
    // (offsets 16, 8, 4, 2, 1), halving the values a lane carries at each of
    // the first steps: a lane keeps the tokens whose bit matches its own lane
    // bit and adds its partner's copy of them.  The pairs added are those of
    // a per-token butterfly, so every sum is the same.
    int width = kTok;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      if (width > 1) {
        const bool upper = (lane & off) != 0;
        width >>= 1;
#pragma unroll
        for (int i = 0; i < kTok / 2; ++i) {
          if (i < width) {
            const float send = upper ? p[i] : p[i + width];
            const float keep = upper ? p[i + width] : p[i];
            p[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, off);
          }
        }
      } else {
        p[0] += __shfl_xor_sync(0xFFFFFFFFu, p[0], off);
      }
    }
    // lane bits 4, 3, ... (one per halving) name the token whose sum it holds
    int m = 0;
#pragma unroll
    for (int off = 16, w = kTok / 2; w > 0; off >>= 1, w >>= 1)
      if (lane & off) m += w;
    constexpr int kLowMask = 32 / kTok - 1;                        // lanes with these bits 0 write
    if ((lane & kLowMask) == 0 && m < M) part[(static_cast<int64_t>(c) * kFtMaxTok + m) * r + j] = p[0];
  }

  // the last CTA to finish adds the chunks' partials in chunk order
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = atomicAdd(ticket, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  const int chunks = static_cast<int>(gridDim.x);
  for (int e = threadIdx.x; e < M * r; e += kFtThreads) {
    const int m = e / r, j = e % r;
    const float* pe = part + static_cast<int64_t>(m) * r + j;
    const int64_t stride = static_cast<int64_t>(kFtMaxTok) * r;
    float v = 0.f;
    for (int cc = 0; cc < chunks; cc += 16) {       // sixteen loads in flight, added in chunk order
      float t[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) t[i] = cc + i < chunks ? __ldcg(pe + (cc + i) * stride) : 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) v += t[i];
    }
    us[e] = __bfloat16_as_ushort(__float2bfloat16_rn(s * v));
  }
  if (threadIdx.x == 0) *ticket = 0u;
}

}  // namespace qnf4
