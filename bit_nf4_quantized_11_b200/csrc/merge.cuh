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
// implements.  The rank-r product is the expensive part (r multiply-adds per
// weight against 2.5 bytes of traffic), so the kernel is organised around the
// fp32 FMA pipe: a CTA of 256 threads takes a tile of 64 rows x 256 columns
// and stages up to 64 rank indices of A (as fp32, [j][column]) and of B
// (transposed, [j][row]) in shared memory; a CTA walks a column-major run of
// tiles, so for r <= 64 it stages A once per column tile.  Each thread accumulates an 8 x 8
// block in registers; a warp covers 32 rows x 64 columns, so per rank index
// its lanes read 256 distinct bytes of A and 128 of B (the rest broadcast)
// for 64 FMAs each, which keeps the shared-memory pipe well below the FMA
// pipe.
#pragma once

#include "common.cuh"

namespace qnf4 {

constexpr int kMergeTileRows = 64;
constexpr int kMergeTileCols = 256;
constexpr int kMergeChunk = 64;                                      // rank indices staged at a time

// shared memory for a rank of r (chunks of at most kMergeChunk rank indices)
__host__ __device__ constexpr int merge_smem_bytes(int r) {
  return (r < kMergeChunk ? r : kMergeChunk) * (kMergeTileCols + kMergeTileRows) * 4;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// acc[c] = fp32(acc[c] + b * a[c]) for the 8 columns, in order of the rank index.
__device__ __forceinline__ void merge_fma_row(float (&acc)[8], float b, float4 a0, float4 a1) {
  acc[0] = __fmaf_rn(b, a0.x, acc[0]);
  acc[1] = __fmaf_rn(b, a0.y, acc[1]);
  acc[2] = __fmaf_rn(b, a0.z, acc[2]);
  acc[3] = __fmaf_rn(b, a0.w, acc[3]);
  acc[4] = __fmaf_rn(b, a1.x, acc[4]);
  acc[5] = __fmaf_rn(b, a1.y, acc[5]);
  acc[6] = __fmaf_rn(b, a1.z, acc[6]);
  acc[7] = __fmaf_rn(b, a1.w, acc[7]);
}

__global__ void __launch_bounds__(256, 2) merge_adapter_kernel(
    const uint8_t* __restrict__ codes, const int8_t* __restrict__ q8, const float* __restrict__ step2,
    const float* __restrict__ mean_ptr, const uint16_t* __restrict__ A, const uint16_t* __restrict__ B, int r,
    float s, int64_t rows, int64_t cols, uint16_t* __restrict__ out, Levels L) {
  extern __shared__ __align__(16) float s_merge[];
  const int chunk = min(r, kMergeChunk);
  float* As = s_merge;                                               // [chunk][kMergeTileCols]
  float* Bs = s_merge + chunk * kMergeTileCols;                      // [chunk][kMergeTileRows]
  __shared__ float s_lv[16];                                         // levels, indexed by code
#pragma unroll
  for (int k = 0; k < 16; ++k)                                       // constant indices keep L in registers
    if (threadIdx.x == k) s_lv[k] = L.v[k];
  const float mu = *mean_ptr;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tr = 32 * (warp >> 2) + 8 * (lane >> 3);                 // first of this thread's 8 rows in the tile
  const int tc = 64 * (warp & 3) + 8 * (lane & 7);                   // first of its 8 columns
  const int64_t col_tiles = (cols + kMergeTileCols - 1) / kMergeTileCols;
  const int64_t row_tiles = rows / kMergeTileRows;
  const int64_t n_tiles = row_tiles * col_tiles;
  // Tiles column-major, a contiguous run of them per CTA: consecutive tiles
  // share their columns, so with r <= kMergeChunk the staged A is reused
  // until the run moves to the next column tile.
  const int64_t t_begin = static_cast<int64_t>(blockIdx.x) * n_tiles / gridDim.x;
  const int64_t t_end = static_cast<int64_t>(blockIdx.x + 1) * n_tiles / gridDim.x;
  int64_t staged_i0 = -1;                                            // columns whose A is in shared memory

  for (int64_t tile = t_begin; tile < t_end; ++tile) {
    const int64_t o0 = (tile % row_tiles) * kMergeTileRows;
    const int64_t i0 = (tile / row_tiles) * kMergeTileCols;
    const int64_t i = i0 + tc;
    const bool col_ok = i < cols;                                    // cols % 64 == 0: 8-column groups are whole
    float acc[8][8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[k][c] = 0.f;

    for (int j0 = 0; j0 < r; j0 += chunk) {
      const int jc = min(chunk, r - j0);
      __syncthreads();                                               // previous chunk (or tile) fully read
      // A[j0 + jj][i0 .. i0 + 256) as fp32, zero past the last column (kept
      // from the previous tile when it is the same single chunk)
      const bool stage_a = !(r <= kMergeChunk && staged_i0 == i0);
      staged_i0 = r <= kMergeChunk ? i0 : -1;
      for (int e = threadIdx.x; stage_a && e < jc * (kMergeTileCols / 8); e += 256) {
        const int jj = e / (kMergeTileCols / 8), c8 = e % (kMergeTileCols / 8);
        const int64_t ia = i0 + 8 * c8;
        uint4 a = make_uint4(0, 0, 0, 0);
        if (ia < cols) a = __ldg(reinterpret_cast<const uint4*>(A + static_cast<int64_t>(j0 + jj) * cols + ia));
        float* d = As + jj * kMergeTileCols + 8 * c8;
        *reinterpret_cast<float4*>(d) = make_float4(bf16_lo(a.x), bf16_hi(a.x), bf16_lo(a.y), bf16_hi(a.y));
        *reinterpret_cast<float4*>(d + 4) = make_float4(bf16_lo(a.z), bf16_hi(a.z), bf16_lo(a.w), bf16_hi(a.w));
      }
      // B[o0 + row][j0 + jj] as fp32, transposed to [jj][row]: eight rank
      // indices of one row per 16-byte load when r % 8 == 0, else one by one
      for (int e = threadIdx.x; r % 8 != 0 && e < jc * kMergeTileRows; e += 256) {
        const int row = e / jc, jj = e % jc;
        Bs[jj * kMergeTileRows + row] =
            __uint_as_float(static_cast<uint32_t>(__ldg(B + (o0 + row) * r + j0 + jj)) << 16);
      }
      for (int e = threadIdx.x; r % 8 == 0 && e < (jc / 8) * kMergeTileRows; e += 256) {
        const int row = e / (jc / 8), j8 = 8 * (e % (jc / 8));
        const uint4 b = __ldg(reinterpret_cast<const uint4*>(B + (o0 + row) * r + j0 + j8));
        float* d = Bs + j8 * kMergeTileRows + row;
        d[0 * kMergeTileRows] = bf16_lo(b.x);
        d[1 * kMergeTileRows] = bf16_hi(b.x);
        d[2 * kMergeTileRows] = bf16_lo(b.y);
        d[3 * kMergeTileRows] = bf16_hi(b.y);
        d[4 * kMergeTileRows] = bf16_lo(b.z);
        d[5 * kMergeTileRows] = bf16_hi(b.z);
        d[6 * kMergeTileRows] = bf16_lo(b.w);
        d[7 * kMergeTileRows] = bf16_hi(b.w);
      }
      __syncthreads();
      for (int jj = 0; jj < jc; ++jj) {
        const float4 b0 = *reinterpret_cast<const float4*>(Bs + jj * kMergeTileRows + tr);
        const float4 b1 = *reinterpret_cast<const float4*>(Bs + jj * kMergeTileRows + tr + 4);
        const float4 a0 = *reinterpret_cast<const float4*>(As + jj * kMergeTileCols + tc);
        const float4 a1 = *reinterpret_cast<const float4*>(As + jj * kMergeTileCols + tc + 4);
        merge_fma_row(acc[0], b0.x, a0, a1);
        merge_fma_row(acc[1], b0.y, a0, a1);
        merge_fma_row(acc[2], b0.z, a0, a1);
        merge_fma_row(acc[3], b0.w, a0, a1);
        merge_fma_row(acc[4], b1.x, a0, a1);
        merge_fma_row(acc[5], b1.y, a0, a1);
        merge_fma_row(acc[6], b1.z, a0, a1);
        merge_fma_row(acc[7], b1.w, a0, a1);
      }
    }

    if (col_ok) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int64_t o = o0 + tr + k;
        const int64_t blk = o * (cols / 64) + i / 64;
        const float c_hat = block_scale(__ldg(q8 + blk), __ldg(step2 + blk / 256), mu);
        const uint32_t cwk = __ldg(reinterpret_cast<const uint32_t*>(codes + o * (cols / 2) + i / 2));
        uint32_t packed[4];
#pragma unroll
        for (int c = 0; c < 8; c += 2) {
          float v[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const uint32_t code = (cwk >> (4 * (c + e))) & 0xFu;
            const float w_hat = __bfloat162float(__float2bfloat16_rn(__fmul_rn(s_lv[code], c_hat)));
            v[e] = __fadd_rn(w_hat, __fmul_rn(s, acc[k][c + e]));
          }
          packed[c / 2] = pack_bf16x2_rn(v[0], v[1]);
        }
        *reinterpret_cast<uint4*>(out + o * cols + i) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      }
    }
  }
}

}  // namespace qnf4
