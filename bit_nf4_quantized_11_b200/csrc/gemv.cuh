// gemv.cuh -- few-token (M <= 16) QLoRA forward: streaming NF4 GEMV.
//
// With 1..16 tokens the layer is bound by streaming the packed weight from
// HBM (0.52 byte per weight), so the kernel is organised around that stream.
// The work is (row tile of 128 weight rows) x (stage of 128 K columns)
// units, ordered tile-major; a persistent grid sized to the resident capacity
// splits the unit sequence evenly, so every CTA streams the same number of
// bytes whatever the shape.  Each warp owns 16 rows of the current tile (the
// 16-row operand of a warp-level bf16 MMA); per unit a thread holds, for rows
// g and g+8, 32 consecutive codes (16 bytes, always inside one 64-weight
// block) and keeps kGvPF units in flight in registers, across tile
// boundaries.  Nibble pairs are decoded through a 256-entry table of bf16
// level pairs in shared memory (one copy per lane, so lookups never conflict)
// and scaled by the block's double-quantized scale with one packed bf16
// multiply; activations are read through L1.  The MMA's K order is permuted
// consistently for both operands: step i of a unit takes physical columns
// 32q + 4i .. 32q + 4i + 3 for quad lane q.  Where a CTA's range starts or
// ends inside a tile it writes an fp32 partial of that tile; the finalize
// kernel adds a tile's partials in CTA order and the LoRA branch us . B^T
// ("QLoRA", llm-compass, 方法与公式: h = dequant(W0) x + (alpha/r) B A x).
//
// The weight operand here is bf16(bf16(level) * bf16(c_hat)) rather than the
// exactly rounded bf16(level * c_hat) of the GEMM path: a relative difference
// of a few 2^-9 per weight, far inside the output tolerance, bought to keep
// the decode at ~2 instructions per weight.
#pragma once

#include "common.cuh"

namespace qnf4 {

constexpr int kGvThreads = 256;          // 8 warps x 16 rows
constexpr int kGvRows = 128;             // weight rows per tile
constexpr int kGvStageK = 128;           // K columns per unit
constexpr int kGvPF = 4;                 // units of codes in flight per thread
constexpr int kGvSmem = 256 * 32 * 4;    // level-pair table, one copy per lane

struct GemvArgs {
  const uint8_t* codes;
  const int8_t* q8;
  const float* step2;
  const float* mean;
  const uint16_t* x;       // [M, in]
  float* part;             // [ctas][local_tiles][M][kGvRows]
  int M, in, out;
  int n_st;                // units per tile = ceil(in / 128)
  int64_t n_units;         // tiles * n_st
  int local_tiles;         // partial tiles reserved per CTA
  Levels L;
};

// First unit of CTA c when n units are split over p CTAs.
__host__ __device__ __forceinline__ int64_t gemv_unit_begin(int64_t c, int64_t n, int64_t p) {
  return c * n / p;
}

struct GvStage {
  uint4 c[2];        // codes of rows g and g+8
  int q[2];          // second-level codes of their blocks
  float st[2];       // steps of their groups
};

__global__ void __launch_bounds__(kGvThreads) nf4_gemv_kernel(const GemvArgs a) {
  extern __shared__ __align__(16) uint32_t s_lut[];                 // [256][32]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, q = lane & 3;
  const int n_tok_tiles = (a.M + 7) / 8;                            // 1 or 2
  const int64_t u_begin = gemv_unit_begin(blockIdx.x, a.n_units, gridDim.x);
  const int64_t u_end = gemv_unit_begin(blockIdx.x + 1, a.n_units, gridDim.x);
  if (u_begin >= u_end) return;                                     // CTA-uniform
  const int t_first = static_cast<int>(u_begin / a.n_st);

  for (int e = threadIdx.x; e < 256 * 32; e += kGvThreads) {
    const int b = e >> 5;
    s_lut[e] = pack_bf16x2_rn(a.L.v[b & 15], a.L.v[b >> 4]);
  }
  __syncthreads();

  const int64_t row_bytes = a.in / 2;
  const int64_t row_blocks = a.in / 64;
  const float mu = __ldg(a.mean);
  const int row_in_tile0 = warp * 16 + g;

  // (tile, unit-in-tile) of the next unit to load, advanced one unit per load
  int64_t u_ld = u_begin;
  int t_ld = t_first;
  int st_ld = static_cast<int>(u_begin - static_cast<int64_t>(t_first) * a.n_st);
  auto load = [&](GvStage& d) {
    d.c[0] = d.c[1] = make_uint4(0, 0, 0, 0);
    d.q[0] = d.q[1] = 0;
    d.st[0] = d.st[1] = 0.f;
    const bool live = u_ld < u_end;
    const int t = t_ld, st = st_ld;
    ++u_ld;
    if (++st_ld == a.n_st) { st_ld = 0; ++t_ld; }
    if (!live) return;
    const int col = st * kGvStageK + 32 * q;
    if (col >= a.in) return;                                         // half unit (in % 128 == 64)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = t * kGvRows + row_in_tile0 + 8 * h;
      if (r < a.out) {
        d.c[h] = ld_stream_v4(a.codes + static_cast<int64_t>(r) * row_bytes + col / 2);
        const int64_t b = static_cast<int64_t>(r) * row_blocks + col / 64;
        d.q[h] = __ldg(a.q8 + b);
        d.st[h] = __ldg(a.step2 + b / 256);
      }
    }
  };

  GvStage ring[kGvPF];
#pragma unroll
  for (int i = 0; i < kGvPF; ++i) load(ring[i]);

  float acc[2][4];
#pragma unroll
  for (int j = 0; j < 2; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
  const uint32_t lut_lane = smem_u32(s_lut) + lane * 4;
  const bool tok0 = g < a.M, tok1 = g + 8 < a.M;
  const uint16_t* x0 = a.x + static_cast<int64_t>(tok0 ? g : 0) * a.in + 32 * q;
  const uint16_t* x1 = a.x + static_cast<int64_t>(tok1 ? g + 8 : 0) * a.in + 32 * q;

  int t = t_first;                                                  // tile / unit of the unit computed
  int st = static_cast<int>(u_begin - static_cast<int64_t>(t_first) * a.n_st);
  for (int64_t u0 = u_begin; u0 < u_end; u0 += kGvPF) {
#pragma unroll
    for (int k = 0; k < kGvPF; ++k) {
      const int64_t u = u0 + k;
      if (u < u_end) {
        const GvStage cur = ring[k];
        load(ring[k]);
        const int col = st * kGvStageK;
        const __nv_bfloat162 s0 = __float2bfloat162_rn(block_scale(cur.q[0], cur.st[0], mu));
        const __nv_bfloat162 s1 = __float2bfloat162_rn(block_scale(cur.q[1], cur.st[1], mu));
        const bool colv = col + 32 * q < a.in;
        const uint32_t w0[4] = {cur.c[0].x, cur.c[0].y, cur.c[0].z, cur.c[0].w};
        const uint32_t w1[4] = {cur.c[1].x, cur.c[1].y, cur.c[1].z, cur.c[1].w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {          // k16 steps: physical columns 32q + 4i .. +3
          // activations of this step: 4 consecutive columns per token row (L1 hits)
          uint2 xa = make_uint2(0, 0), xb = make_uint2(0, 0);
          if (tok0 && colv) xa = __ldg(reinterpret_cast<const uint2*>(x0 + col + 4 * i));
          if (tok1 && colv) xb = __ldg(reinterpret_cast<const uint2*>(x1 + col + 4 * i));
          const int word = i >> 1, sh = (i & 1) * 16;
          uint32_t e0, e1, e2, e3;
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(e0) : "r"(lut_lane + ((w0[word] >> sh) & 0xFFu) * 128));
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(e1) : "r"(lut_lane + ((w0[word] >> (sh + 8)) & 0xFFu) * 128));
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(e2) : "r"(lut_lane + ((w1[word] >> sh) & 0xFFu) * 128));
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(e3) : "r"(lut_lane + ((w1[word] >> (sh + 8)) & 0xFFu) * 128));
          __nv_bfloat162 p0 = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&e0), s0);
          __nv_bfloat162 p1 = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&e2), s1);
          __nv_bfloat162 p2 = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&e1), s0);
          __nv_bfloat162 p3 = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&e3), s1);
          const uint32_t a0 = *reinterpret_cast<uint32_t*>(&p0);   // row g,   columns 4i, 4i+1
          const uint32_t a1 = *reinterpret_cast<uint32_t*>(&p1);   // row g+8, columns 4i, 4i+1
          const uint32_t a2 = *reinterpret_cast<uint32_t*>(&p2);   // row g,   columns 4i+2, 4i+3
          const uint32_t a3 = *reinterpret_cast<uint32_t*>(&p3);   // row g+8, columns 4i+2, 4i+3
          mma_bf16_16816(acc[0], a0, a1, a2, a3, xa.x, xa.y);
          if (n_tok_tiles > 1) mma_bf16_16816(acc[1], a0, a1, a2, a3, xb.x, xb.y);
        }
        // end of this CTA's part of tile t: write the partial and restart
        if (st == a.n_st - 1 || u == u_end - 1) {
          float* dst = a.part + ((static_cast<int64_t>(blockIdx.x) * a.local_tiles + (t - t_first)) * a.M) * kGvRows;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const int tk = 8 * j + 2 * q + hh;
              if (tk < a.M) {
                dst[static_cast<int64_t>(tk) * kGvRows + row_in_tile0] = acc[j][hh];
                dst[static_cast<int64_t>(tk) * kGvRows + row_in_tile0 + 8] = acc[j][2 + hh];
              }
            }
            acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
          }
        }
        if (++st == a.n_st) { st = 0; ++t; }
      }
    }
  }
}

// h[m][o] = bf16( sum of the partials of o's tile, in CTA order
//                 + sum_j us[m][j] * B[o][j] ),  m < M.
__global__ void __launch_bounds__(256) gemv_finalize_kernel(
    const float* __restrict__ part, int ctas, int local_tiles, int64_t n_units, int n_st, int M, int out,
    const uint16_t* __restrict__ us, const uint16_t* __restrict__ B, int r, uint16_t* __restrict__ h) {
  const int64_t n_el = static_cast<int64_t>(M) * out;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n_el;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int m = static_cast<int>(e / out), o = static_cast<int>(e % out);
    const int t = o / kGvRows, row = o % kGvRows;
    // CTA holding the tile's first unit: the largest c with begin(c) <= t * n_st
    const int64_t u = static_cast<int64_t>(t) * n_st;
    int64_t c = u * ctas / n_units;
    while (c + 1 < ctas && gemv_unit_begin(c + 1, n_units, ctas) <= u) ++c;
    while (c > 0 && gemv_unit_begin(c, n_units, ctas) > u) --c;
    float v = 0.f;
    for (; c < ctas; ++c) {
      const int64_t b = gemv_unit_begin(c, n_units, ctas);
      if (b >= u + n_st) break;                                     // past this tile
      if (gemv_unit_begin(c + 1, n_units, ctas) <= b) continue;     // empty CTA
      const int lt = t - static_cast<int>(b / n_st);
      v += __ldg(part + ((c * local_tiles + lt) * M + m) * static_cast<int64_t>(kGvRows) + row);
    }
    const uint16_t* ur = us + static_cast<int64_t>(m) * r;
    const uint16_t* br = B + static_cast<int64_t>(o) * r;
    float l = 0.f;
    for (int j = 0; j < r; j += 8) {
      const uint4 ua = __ldg(reinterpret_cast<const uint4*>(ur + j));
      const uint4 ba = __ldg(reinterpret_cast<const uint4*>(br + j));
      const uint32_t uw[4] = {ua.x, ua.y, ua.z, ua.w}, bw[4] = {ba.x, ba.y, ba.z, ba.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 uf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&uw[i]));
        const float2 bf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bw[i]));
        l = fmaf(uf.x, bf.x, l);
        l = fmaf(uf.y, bf.y, l);
      }
    }
    h[e] = __bfloat16_as_ushort(__float2bfloat16_rn(v + l));
  }
}

}  // namespace qnf4
