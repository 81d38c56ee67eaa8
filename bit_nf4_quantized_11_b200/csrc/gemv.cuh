// gemv.cuh -- few-token (M <= 16) QLoRA forward: split-K streaming NF4 GEMV.
//
// With 1..16 tokens the layer is bound by streaming the packed weight from
// HBM (0.52 byte per weight), so the kernel is organised around that stream:
// each warp walks 32 weight rows along a K range, one 64-weight block per
// step, decodes nibble pairs through a 256-entry table of bf16 level pairs in
// shared memory (one copy per lane, so lookups never conflict), scales them
// by the block's double-quantized scale with one packed bf16 multiply, and
// feeds warp-level bf16 MMAs with the weights as the 16-row operand and the
// tokens as the 8-column operand.  Per-split fp32 partials are summed in a
// fixed order by the finalize kernel, which also adds the LoRA branch
// us . B^T ("QLoRA", llm-compass, 方法与公式: h = dequant(W0) x + (alpha/r) B A x).
//
// The weight operand here is bf16(bf16(level) * bf16(c_hat)) rather than the
// exactly rounded bf16(level * c_hat) of the GEMM path: a relative difference
// of a few 2^-9 per weight, far inside the output tolerance, bought to keep
// the decode at ~2 instructions per weight.
#pragma once

#include "common.cuh"

namespace qnf4 {

constexpr int kGemvThreads = 256;        // 8 warps x 32 rows = 256 rows per CTA
constexpr int kGemvRowsPerCta = 256;

struct GemvArgs {
  const uint8_t* codes;
  const int8_t* q8;
  const float* step2;
  const float* mean;
  const uint16_t* x;       // [M, in]
  float* part;             // [splits, 16, out]
  int M, in, out;
  int blocks_per_split;    // 64-weight blocks of K per split
  Levels L;
};

__global__ void __launch_bounds__(kGemvThreads) nf4_gemv_splitk_kernel(const GemvArgs a) {
  extern __shared__ uint32_t s_lut[];      // [256][32]: entry b, copy per lane
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int e = threadIdx.x; e < 256 * 32; e += kGemvThreads) {
    const int b = e >> 5;
    const float lo = a.L.v[b & 15], hi = a.L.v[b >> 4];
    s_lut[e] = pack_bf16x2_rn(lo, hi);
  }
  __syncthreads();

  const int g = lane >> 2, q = lane & 3;
  const int row_base = blockIdx.x * kGemvRowsPerCta + warp * 32;
  const int split = blockIdx.y;
  const int n_blocks_row = a.in / 64;
  const int blk_begin = split * a.blocks_per_split;
  const int blk_end = min(n_blocks_row, blk_begin + a.blocks_per_split);
  const float mu = __ldg(a.mean);
  const uint32_t lut_lane = smem_u32(s_lut) + lane * 4;
  const int n_tok_tiles = (a.M + 7) / 8;      // 1 or 2

  // rows handled by this thread: t = 0..3 -> row_base + 16*(t>>1) + g + 8*(t&1)
  int rows[4];
  bool rvalid[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    rows[t] = row_base + 16 * (t >> 1) + g + 8 * (t & 1);
    rvalid[t] = rows[t] < a.out;
  }
  const int tok0 = g, tok1 = g + 8;
  const bool tv0 = tok0 < a.M, tv1 = tok1 < a.M;

  float acc[2][2][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 2; ++j) acc[i][j][0] = acc[i][j][1] = acc[i][j][2] = acc[i][j][3] = 0.f;

#pragma unroll 2
  for (int blk = blk_begin; blk < blk_end; ++blk) {
    uint2 cw[4];
    __nv_bfloat162 sc[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      cw[t] = make_uint2(0, 0);
      float c_hat = 0.f;
      if (rvalid[t]) {
        const int64_t r = rows[t];
        cw[t] = __ldg(reinterpret_cast<const uint2*>(a.codes + r * (a.in / 2) + blk * 32 + q * 8));
        const int64_t bi = r * n_blocks_row + blk;
        c_hat = block_scale(__ldg(a.q8 + bi), __ldg(a.step2 + bi / 256), mu);
      }
      sc[t] = __float2bfloat162_rn(c_hat);
    }
    // token fragments: x[tok][blk*64 + 16q .. +15]
    uint4 xa0 = make_uint4(0, 0, 0, 0), xa1 = xa0, xb0 = xa0, xb1 = xa0;
    const int64_t kx = static_cast<int64_t>(blk) * 64 + q * 16;
    if (tv0) { xa0 = __ldg(reinterpret_cast<const uint4*>(a.x + tok0 * static_cast<int64_t>(a.in) + kx));
               xa1 = __ldg(reinterpret_cast<const uint4*>(a.x + tok0 * static_cast<int64_t>(a.in) + kx + 8)); }
    if (tv1) { xb0 = __ldg(reinterpret_cast<const uint4*>(a.x + tok1 * static_cast<int64_t>(a.in) + kx));
               xb1 = __ldg(reinterpret_cast<const uint4*>(a.x + tok1 * static_cast<int64_t>(a.in) + kx + 8)); }
    const uint32_t xw0[8] = {xa0.x, xa0.y, xa0.z, xa0.w, xa1.x, xa1.y, xa1.z, xa1.w};
    const uint32_t xw1[8] = {xb0.x, xb0.y, xb0.z, xb0.w, xb1.x, xb1.y, xb1.z, xb1.w};

#pragma unroll
    for (int i = 0; i < 4; ++i) {          // MMA k-steps: physical k = 16q + 4i .. +3
      uint32_t af[4][2];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const uint32_t word = (i < 2) ? cw[t].x : cw[t].y;
        const int sh = (i & 1) * 16;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t byte = (word >> (sh + 8 * h)) & 0xFFu;
          uint32_t v;
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(lut_lane + byte * 128));
          __nv_bfloat162 p = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&v), sc[t]);
          af[t][h] = *reinterpret_cast<uint32_t*>(&p);
        }
      }
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        // rows g (t = 2mt) and g+8 (t = 2mt+1): a0 = row g pair 0, a1 = row g+8 pair 0,
        // a2 = row g pair 1, a3 = row g+8 pair 1
        mma_bf16_16816(acc[mt][0], af[2 * mt][0], af[2 * mt + 1][0], af[2 * mt][1], af[2 * mt + 1][1],
                       xw0[2 * i], xw0[2 * i + 1]);
        if (n_tok_tiles > 1)
          mma_bf16_16816(acc[mt][1], af[2 * mt][0], af[2 * mt + 1][0], af[2 * mt][1], af[2 * mt + 1][1],
                         xw1[2 * i], xw1[2 * i + 1]);
      }
    }
  }

  // partials: part[split][token][row]; D fragment (row g / g+8, tokens 2q, 2q+1)
  float* dst = a.part + static_cast<int64_t>(split) * 16 * a.out;
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int t0 = 8 * j + 2 * q;
      const int ra = rows[2 * mt], rb = rows[2 * mt + 1];
      if (rvalid[2 * mt]) {
        dst[static_cast<int64_t>(t0) * a.out + ra] = acc[mt][j][0];
        dst[static_cast<int64_t>(t0 + 1) * a.out + ra] = acc[mt][j][1];
      }
      if (rvalid[2 * mt + 1]) {
        dst[static_cast<int64_t>(t0) * a.out + rb] = acc[mt][j][2];
        dst[static_cast<int64_t>(t0 + 1) * a.out + rb] = acc[mt][j][3];
      }
    }
  }
}

// h[m][o] = bf16( sum_s part[s][m][o] + sum_j us[m][j] * B[o][j] ), m < M.
__global__ void __launch_bounds__(256) gemv_finalize_kernel(
    const float* __restrict__ part, int splits, int M, int out,
    const uint16_t* __restrict__ us, const uint16_t* __restrict__ B, int r,
    uint16_t* __restrict__ h) {
  const int64_t n_el = static_cast<int64_t>(M) * out;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n_el;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int m = static_cast<int>(e / out), o = static_cast<int>(e % out);
    float v = 0.f;
    for (int s = 0; s < splits; ++s) v += part[(static_cast<int64_t>(s) * 16 + m) * out + o];
    const uint16_t* ur = us + static_cast<int64_t>(m) * r;
    const uint16_t* br = B + static_cast<int64_t>(o) * r;
    float l = 0.f;
    for (int j = 0; j < r; ++j)
      l = fmaf(__bfloat162float(__ushort_as_bfloat16(ur[j])), __bfloat162float(__ushort_as_bfloat16(br[j])), l);
    h[e] = __bfloat16_as_ushort(__float2bfloat16_rn(v + l));
  }
}

}  // namespace qnf4
