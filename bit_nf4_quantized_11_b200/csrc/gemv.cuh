// gemv.cuh -- few-token (M <= 16) QLoRA forward: split-K streaming NF4 GEMV.
//
// With 1..16 tokens the layer is bound by streaming the packed weight from
// HBM (0.52 byte per weight), so the kernel is organised around that stream.
// A CTA owns 128 weight rows and a range of K; each warp owns 16 rows (the
// 16-row operand of a warp-level bf16 MMA) and walks the range in stages of
// 128 columns.  Per stage a thread holds, for rows g and g+8 of its warp
// tile, 32 consecutive codes (16 bytes, always inside one 64-weight block)
// and keeps kGvPF stages of them in flight in registers.  Nibble pairs are
// decoded through a 256-entry table of bf16 level pairs in shared memory (one
// copy per lane, so lookups never conflict) and scaled by the block's
// double-quantized scale with one packed bf16 multiply.  The MMA's K order is
// permuted consistently for both operands: step i of a stage takes physical
// columns 32q + 4i .. 32q + 4i + 3 for quad lane q.  The activations of the
// CTA's K range sit in shared memory.  Per-split fp32 partials are summed in
// a fixed order by the finalize kernel, which also adds the LoRA branch
// us . B^T ("QLoRA", llm-compass, 方法与公式: h = dequant(W0) x + (alpha/r) B A x).
//
// The weight operand here is bf16(bf16(level) * bf16(c_hat)) rather than the
// exactly rounded bf16(level * c_hat) of the GEMM path: a relative difference
// of a few 2^-9 per weight, far inside the output tolerance, bought to keep
// the decode at ~2 instructions per weight.
#pragma once

#include "common.cuh"

namespace qnf4 {

constexpr int kGvThreads = 256;          // 8 warps x 16 rows
constexpr int kGvRows = 128;             // weight rows per CTA
constexpr int kGvStageK = 128;           // K columns per stage
constexpr int kGvMaxStages = 16;         // stages per split (activation tile <= 2048 columns)
constexpr int kGvPF = 4;                 // stages of codes in flight per thread

struct GemvArgs {
  const uint8_t* codes;
  const int8_t* q8;
  const float* step2;
  const float* mean;
  const uint16_t* x;       // [M, in]
  float* part;             // [splits, M, out]
  int M, in, out;
  int stages_per_split;
  int x_pitch;             // shared-memory row pitch of the activation tile, in bf16
  Levels L;
};

__host__ __device__ constexpr int gemv_x_pitch(int stages_per_split) {
  return stages_per_split * kGvStageK + 8;          // +16 B: rows start in different banks
}

__host__ __device__ constexpr int gemv_smem_bytes(int M, int stages_per_split) {
  return 256 * 32 * 4 + (M <= 8 ? 8 : 16) * gemv_x_pitch(stages_per_split) * 2;
}

struct GvStage {
  uint4 c[2];        // codes of rows g and g+8
  int q[2];          // second-level codes of their blocks
  float st[2];       // steps of their groups
};

__global__ void __launch_bounds__(kGvThreads) nf4_gemv_splitk_kernel(const GemvArgs a) {
  extern __shared__ __align__(16) uint32_t s_gv[];
  uint32_t* s_lut = s_gv;                                           // [256][32]
  uint16_t* s_x = reinterpret_cast<uint16_t*>(s_gv + 256 * 32);     // [tokens][x_pitch]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, q = lane & 3;
  const int n_tok_tiles = (a.M + 7) / 8;                            // 1 or 2
  const int n_st = (a.in + kGvStageK - 1) / kGvStageK;     // last stage may be half (in % 128 == 64)
  const int st_begin = blockIdx.y * a.stages_per_split;
  const int st_end = min(n_st, st_begin + a.stages_per_split);
  const int k_begin = st_begin * kGvStageK;
  const int k_len = (st_end - st_begin) * kGvStageK;

  for (int e = threadIdx.x; e < 256 * 32; e += kGvThreads) {
    const int b = e >> 5;
    s_lut[e] = pack_bf16x2_rn(a.L.v[b & 15], a.L.v[b >> 4]);
  }
  const int n_tok = n_tok_tiles * 8;
  for (int e = threadIdx.x; e < n_tok * (k_len / 8); e += kGvThreads) {
    const int tok = e / (k_len / 8), c8 = e % (k_len / 8);
    uint4 v = make_uint4(0, 0, 0, 0);
    if (tok < a.M && k_begin + 8 * c8 < a.in) v = ld_nc_v4(a.x + static_cast<int64_t>(tok) * a.in + k_begin + 8 * c8);
    *reinterpret_cast<uint4*>(s_x + tok * a.x_pitch + 8 * c8) = v;
  }
  __syncthreads();

  const int r0 = blockIdx.x * kGvRows + warp * 16 + g;
  const int r1 = r0 + 8;
  const bool v0 = r0 < a.out, v1 = r1 < a.out;
  const int64_t row_bytes = a.in / 2;
  const int64_t row_blocks = a.in / 64;
  const float mu = __ldg(a.mean);
  const uint8_t* cp0 = a.codes + static_cast<int64_t>(v0 ? r0 : 0) * row_bytes + 16 * q;
  const uint8_t* cp1 = a.codes + static_cast<int64_t>(v1 ? r1 : 0) * row_bytes + 16 * q;
  const int64_t bq0 = static_cast<int64_t>(v0 ? r0 : 0) * row_blocks + (q >> 1);
  const int64_t bq1 = static_cast<int64_t>(v1 ? r1 : 0) * row_blocks + (q >> 1);

  auto load = [&](int st, GvStage& d) {
    d.c[0] = d.c[1] = make_uint4(0, 0, 0, 0);
    d.q[0] = d.q[1] = 0;
    d.st[0] = d.st[1] = 0.f;
    if (st < st_end && st * kGvStageK + 32 * q < a.in) {     // columns past `in` stay zero
      if (v0) {
        d.c[0] = ld_stream_v4(cp0 + static_cast<int64_t>(st) * 64);
        const int64_t b = bq0 + 2 * st;
        d.q[0] = __ldg(a.q8 + b);
        d.st[0] = __ldg(a.step2 + b / 256);
      }
      if (v1) {
        d.c[1] = ld_stream_v4(cp1 + static_cast<int64_t>(st) * 64);
        const int64_t b = bq1 + 2 * st;
        d.q[1] = __ldg(a.q8 + b);
        d.st[1] = __ldg(a.step2 + b / 256);
      }
    }
  };

  GvStage ring[kGvPF];
#pragma unroll
  for (int i = 0; i < kGvPF; ++i) load(st_begin + i, ring[i]);

  float acc[2][4];
#pragma unroll
  for (int j = 0; j < 2; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
  const uint32_t lut_lane = smem_u32(s_lut) + lane * 4;
  const uint32_t x_base0 = smem_u32(s_x) + (g * a.x_pitch + 32 * q) * 2;
  const uint32_t x_base1 = x_base0 + 8 * a.x_pitch * 2;

  for (int st0 = st_begin; st0 < st_end; st0 += kGvPF) {
#pragma unroll
    for (int u = 0; u < kGvPF; ++u) {
      const int st = st0 + u;
      if (st < st_end) {
        const GvStage cur = ring[u];
        load(st + kGvPF, ring[u]);
        const __nv_bfloat162 s0 = __float2bfloat162_rn(block_scale(cur.q[0], cur.st[0], mu));
        const __nv_bfloat162 s1 = __float2bfloat162_rn(block_scale(cur.q[1], cur.st[1], mu));
        // activations of this stage: 32 consecutive columns per token row
        const uint32_t xo = (st - st_begin) * kGvStageK * 2;
        uint4 xa[4], xb[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(xa[i].x), "=r"(xa[i].y), "=r"(xa[i].z), "=r"(xa[i].w) : "r"(x_base0 + xo + 16 * i));
          if (n_tok_tiles > 1)
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(xb[i].x), "=r"(xb[i].y), "=r"(xb[i].z), "=r"(xb[i].w) : "r"(x_base1 + xo + 16 * i));
        }
        const uint32_t w0[4] = {cur.c[0].x, cur.c[0].y, cur.c[0].z, cur.c[0].w};
        const uint32_t w1[4] = {cur.c[1].x, cur.c[1].y, cur.c[1].z, cur.c[1].w};
        const uint32_t xw0[16] = {xa[0].x, xa[0].y, xa[0].z, xa[0].w, xa[1].x, xa[1].y, xa[1].z, xa[1].w,
                                  xa[2].x, xa[2].y, xa[2].z, xa[2].w, xa[3].x, xa[3].y, xa[3].z, xa[3].w};
        const uint32_t xw1[16] = {xb[0].x, xb[0].y, xb[0].z, xb[0].w, xb[1].x, xb[1].y, xb[1].z, xb[1].w,
                                  xb[2].x, xb[2].y, xb[2].z, xb[2].w, xb[3].x, xb[3].y, xb[3].z, xb[3].w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {          // k16 steps: physical columns 32q + 4i .. +3
          const int word = i >> 1, sh = (i & 1) * 16;
          uint32_t a0, a1, a2, a3;
          {
            uint32_t e0, e1, e2, e3;
            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(e0) : "r"(lut_lane + ((w0[word] >> sh) & 0xFFu) * 128));
            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(e1) : "r"(lut_lane + ((w0[word] >> (sh + 8)) & 0xFFu) * 128));
            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(e2) : "r"(lut_lane + ((w1[word] >> sh) & 0xFFu) * 128));
            asm volatile("ld.shared.u32 %0, [%1];" : "=r"(e3) : "r"(lut_lane + ((w1[word] >> (sh + 8)) & 0xFFu) * 128));
            __nv_bfloat162 p0 = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&e0), s0);
            __nv_bfloat162 p1 = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&e2), s1);
            __nv_bfloat162 p2 = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&e1), s0);
            __nv_bfloat162 p3 = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&e3), s1);
            a0 = *reinterpret_cast<uint32_t*>(&p0);   // row g,   columns 4i, 4i+1
            a1 = *reinterpret_cast<uint32_t*>(&p1);   // row g+8, columns 4i, 4i+1
            a2 = *reinterpret_cast<uint32_t*>(&p2);   // row g,   columns 4i+2, 4i+3
            a3 = *reinterpret_cast<uint32_t*>(&p3);   // row g+8, columns 4i+2, 4i+3
          }
          mma_bf16_16816(acc[0], a0, a1, a2, a3, xw0[2 * i], xw0[2 * i + 1]);
          if (n_tok_tiles > 1) mma_bf16_16816(acc[1], a0, a1, a2, a3, xw1[2 * i], xw1[2 * i + 1]);
        }
      }
    }
  }

  // partials: part[split][token][row]; D fragment rows g / g+8, tokens 8j + 2q, +1
  float* dst = a.part + static_cast<int64_t>(blockIdx.y) * a.M * a.out;
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int t0 = 8 * j + 2 * q;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int t = t0 + h;
      if (t < a.M) {
        if (v0) dst[static_cast<int64_t>(t) * a.out + r0] = acc[j][h];
        if (v1) dst[static_cast<int64_t>(t) * a.out + r1] = acc[j][2 + h];
      }
    }
  }
}

// h[m][o] = bf16( sum_s part[s][m][o] + sum_j us[m][j] * B[o][j] ), m < M,
// splits added in order.
__global__ void __launch_bounds__(256) gemv_finalize_kernel(
    const float* __restrict__ part, int splits, int M, int out,
    const uint16_t* __restrict__ us, const uint16_t* __restrict__ B, int r,
    uint16_t* __restrict__ h) {
  const int64_t n_el = static_cast<int64_t>(M) * out;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n_el;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int m = static_cast<int>(e / out), o = static_cast<int>(e % out);
    float v = 0.f;
#pragma unroll 4
    for (int s = 0; s < splits; ++s) v += __ldg(part + static_cast<int64_t>(s) * n_el + e);
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
