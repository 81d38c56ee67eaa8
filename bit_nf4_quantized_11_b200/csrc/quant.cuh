// quant.cuh -- NF4 blockwise quantizer with double quantization, and the
// standalone dequantizer (sm_100a, CUDA cores; all HBM-streaming kernels).
//
// Method ("QLoRA", llm-compass, 方法与公式 items 1-2; learn-interview-questions
// QLoRA page, section 2): 64-weight blocks, one absmax per block, nearest of
// 16 normal-quantile levels; the fp32 block absmaxes are quantized again to
// 8 bit around their mean, one fp32 step per group of 256 blocks.
//
// Every fp32 operation below is a separately rounded IEEE operation
// (__fmul_rn/__fadd_rn/__fsub_rn/__fdiv_rn/__frcp_rn, fp64 __dadd_rn/__ddiv_rn),
// so the packed codes, the int8 scale codes, the steps, the mean and the
// dequantized bf16 weights are bit-reproducible.
#pragma once

#include "common.cuh"

namespace qnf4 {

constexpr int kBlock = 64;        // weights per first-level block
constexpr int kGroup = 256;       // blocks per second-level group
constexpr int kTreeChunk = 4096;  // leaves summed by one CTA of the scale-mean tree
constexpr int kTreeTop = 1024;    // most partial sums the last CTA of a pass finishes

// ---------------------------------------------------------------------------
// K1 and its code table
// ---------------------------------------------------------------------------
constexpr int kQRounds = 2;

// Exact nearest level without a search.  [-1, 1] (slightly widened: a block's
// normalised values can exceed 1 by an ulp) is cut into 33 cells by
// n = round(16 v) + 16; every cell contains at most one threshold and every
// threshold lies more than 4e-3 from a cell edge, so for any fp32 v
//   #{j : v > thr_j} = below[n] + (v > inside[n])
// where below[n] counts the thresholds under the cell and inside[n] is the
// threshold inside it (+inf if none).  The host builds the table from the
// fp32 thresholds; n comes from one fused multiply-add whose single rounding
// to an integer (magnitude 1.5 * 2^23) yields round(16 v) in the low bits.
constexpr int kCodeCells = 33;
constexpr float kCellMagic = 12582928.0f;          // 1.5 * 2^23 + 16
struct CodeTable { uint32_t below[kCodeCells]; float inside[kCodeCells]; };

__device__ __forceinline__ uint32_t nearest_code(float v, uint32_t tab_lane) {
  const float y = __fmaf_rn(v, 16.0f, kCellMagic);
  // finite |v| <= 1 + 2^-22 gives n in 0..32; the clamp keeps any input in the table
  const uint32_t n = min(static_cast<uint32_t>(__float_as_int(y) - __float_as_int(kCellMagic) + 16),
                         static_cast<uint32_t>(kCodeCells - 1));
  uint32_t below, inside_bits;
  // not volatile: the table is written before the barrier that precedes every
  // weight load, and each lookup depends on a loaded weight
  asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(below), "=r"(inside_bits) : "r"(tab_lane + n * 256));
  return below + (v > __uint_as_float(inside_bits) ? 1u : 0u);
}

// K1: per-block absmax, nearest-level code, nibble packing (fp32 or bf16
// weights; a bf16 weight is quantized as its exact fp32 value).
// Four lanes per 64-weight block: lane q takes the 4-weight chunks q, q+4,
// q+8, q+12, so each load instruction reads every block's 64 consecutive
// bytes (fp32) in one piece; the absmax is reduced over the 4 lanes with two
// shuffles, and lane q writes the 2 code bytes of each of its chunks.  A warp
// takes 8 * kQRounds consecutive blocks per iteration and issues all their
// loads before any arithmetic (64 B per lane per round in flight).
// The cell table sits in shared memory with one copy per lane (entry n of
// lane l at (n*32 + l)*8), so lookups never conflict.
// Four consecutive weights as fp32: 16 bytes of fp32, or 8 bytes of bf16
// widened exactly (a bf16 number is the top half of its fp32 pattern).
__device__ __forceinline__ float4 load_w4(const float* W, int64_t i) {
  const uint4 u = ld_stream_v4(W + i);
  return make_float4(__uint_as_float(u.x), __uint_as_float(u.y), __uint_as_float(u.z), __uint_as_float(u.w));
}
__device__ __forceinline__ float4 load_w4(const uint16_t* W, int64_t i) {
  uint32_t a, b;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(a), "=r"(b) : "l"(W + i));
  return make_float4(__uint_as_float(a << 16), __uint_as_float(a & 0xFFFF0000u), __uint_as_float(b << 16),
                     __uint_as_float(b & 0xFFFF0000u));
}

template <typename Tin>
__global__ void __launch_bounds__(256, 4) nf4_quantize_blocks_kernel(
    const Tin* __restrict__ W, int64_t n_blocks, uint8_t* __restrict__ codes,
    float* __restrict__ absmax, CodeTable tab, unsigned int* __restrict__ ticket) {
  __shared__ __align__(16) uint2 s_tab[kCodeCells * 32];
  if (blockIdx.x == 0 && threadIdx.x == 0) *ticket = 0u;            // for the tree pass after this kernel
  for (int e = threadIdx.x; e < kCodeCells * 32; e += blockDim.x)
    s_tab[e] = make_uint2(tab.below[e >> 5], __float_as_uint(tab.inside[e >> 5]));
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int bl = lane >> 2;            // block of this lane among the warp's 8
  const int q = lane & 3;              // chunks q + 4k, k = 0..3
  const uint32_t tab_lane = smem_u32(s_tab) + lane * 8;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;

  for (int64_t base = warp * 8 * kQRounds; base < n_blocks; base += n_warps * 8 * kQRounds) {
    float4 w[kQRounds][4];
#pragma unroll
    for (int rd = 0; rd < kQRounds; ++rd) {
      const int64_t b = base + 8 * rd + bl;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        w[rd][k] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (b < n_blocks) w[rd][k] = load_w4(W, b * kBlock + (q + 4 * k) * 4);
      }
    }
#pragma unroll
    for (int rd = 0; rd < kQRounds; ++rd) {
      const int64_t b = base + 8 * rd + bl;
      float m = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        m = fmaxf(m, fmaxf(fmaxf(fabsf(w[rd][k].x), fabsf(w[rd][k].y)), fmaxf(fabsf(w[rd][k].z), fabsf(w[rd][k].w))));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
      // m is now the exact absmax of this lane's block
      const float r = __frcp_rn(m);
      uint32_t packed[4];
      if (m > 0.f && isinf(r)) {
        // absmax so small (subnormal) that 1/absmax overflows: normalise by
        // one correctly rounded division instead (rare, block-uniform path)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t c0 = nearest_code(__fdiv_rn(w[rd][k].x, m), tab_lane);
          const uint32_t c1 = nearest_code(__fdiv_rn(w[rd][k].y, m), tab_lane);
          const uint32_t c2 = nearest_code(__fdiv_rn(w[rd][k].z, m), tab_lane);
          const uint32_t c3 = nearest_code(__fdiv_rn(w[rd][k].w, m), tab_lane);
          packed[k] = c0 | (c1 << 4) | (c2 << 8) | (c3 << 12);
        }
      } else if (m > 0.f) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t c0 = nearest_code(__fmul_rn(w[rd][k].x, r), tab_lane);
          const uint32_t c1 = nearest_code(__fmul_rn(w[rd][k].y, r), tab_lane);
          const uint32_t c2 = nearest_code(__fmul_rn(w[rd][k].z, r), tab_lane);
          const uint32_t c3 = nearest_code(__fmul_rn(w[rd][k].w, r), tab_lane);
          packed[k] = c0 | (c1 << 4) | (c2 << 8) | (c3 << 12);
        }
      } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) packed[k] = 0x7777u;
      }
      if (b < n_blocks) {
        uint16_t* dst = reinterpret_cast<uint16_t*>(codes + b * (kBlock / 2));
#pragma unroll
        for (int k = 0; k < 4; ++k) dst[q + 4 * k] = static_cast<uint16_t>(packed[k]);
        if (q == 0) absmax[b] = m;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// K2: fixed fp64 summation tree over the block absmaxes.
// The tree is defined on the whole array zero-padded to a power of two, with
// adjacent pairs added level by level.  One CTA (256 threads) sums an aligned
// chunk of 4096 leaves: 16 consecutive leaves per thread (in-register tree),
// then a xor-butterfly across the warp (offset 1, 2, 4, ... adds adjacent
// pairs), then the 8 warp sums pairwise.  Chunks are aligned subtrees, so
// summing the chunk sums the same way reproduces the full tree exactly;
// missing leaves are exact zeros.  With `finish` (at most kTreeTop chunks),
// the CTA that completes last (a ticket counter, reset to 0 by the kernel
// before) sums the chunk sums -- 4 per thread, butterfly, warp sums -- and
// writes mean = fp32(T / n_leaves) with the division in fp64.  Otherwise the
// host runs another pass over the chunk sums.
// ---------------------------------------------------------------------------
template <int kPer>
__device__ __forceinline__ double tree_256(const double (&v0)[kPer], double* s_warp) {
  double v[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) v[i] = v0[i];
#pragma unroll
  for (int width = kPer / 2; width >= 1; width >>= 1) {
#pragma unroll
    for (int i = 0; i < width; ++i) v[i] = __dadd_rn(v[2 * i], v[2 * i + 1]);
  }
  double s = v[0];
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) s = __dadd_rn(s, __shfl_xor_sync(0xffffffffu, s, off));
  if ((threadIdx.x & 31) == 0) s_warp[threadIdx.x >> 5] = s;
  __syncthreads();
  const double a = __dadd_rn(__dadd_rn(s_warp[0], s_warp[1]), __dadd_rn(s_warp[2], s_warp[3]));
  const double b = __dadd_rn(__dadd_rn(s_warp[4], s_warp[5]), __dadd_rn(s_warp[6], s_warp[7]));
  return __dadd_rn(a, b);                                            // same value in every thread
}

template <typename T>
__global__ void __launch_bounds__(256) pairwise_tree_kernel(
    const T* __restrict__ in, int64_t n, double* __restrict__ out, int finish,
    unsigned int* __restrict__ ticket, int64_t n_leaves_total, float* __restrict__ mean_out,
    unsigned int* __restrict__ next_ticket) {
  __shared__ double s_warp[8];
  __shared__ int s_last;
  if (blockIdx.x == 0 && threadIdx.x == 0 && next_ticket != nullptr) *next_ticket = 0u;
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kTreeChunk + threadIdx.x * 16;
  double v[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = (base + i < n) ? static_cast<double>(in[base + i]) : 0.0;
  const double t = tree_256<16>(v, s_warp);
  if (threadIdx.x == 0) {
    out[blockIdx.x] = t;
    if (finish) {
      __threadfence();
      s_last = atomicAdd(ticket, 1u) == gridDim.x - 1;
    }
  }
  __syncthreads();
  if (!finish || !s_last) return;                                    // CTA-uniform
  __threadfence();
  double w[kTreeTop / 256];
#pragma unroll
  for (int i = 0; i < kTreeTop / 256; ++i) {
    const int idx = threadIdx.x * (kTreeTop / 256) + i;
    w[i] = idx < static_cast<int>(gridDim.x) ? __ldcg(out + idx) : 0.0;
  }
  __syncthreads();                                                   // s_warp is reused
  const double total = tree_256<kTreeTop / 256>(w, s_warp);
  if (threadIdx.x == 0) *mean_out = __double2float_rn(__ddiv_rn(total, static_cast<double>(n_leaves_total)));
}

// ---------------------------------------------------------------------------
// K3: second-level codes.  One warp per group of 256 block scales:
// d = fp32(c - mean), step2 = fp32(max|d| / 127),
// q8 = clamp(rne(fp32(d * fp32(1/step2))), -127, 127), with fp32(d / step2)
// in place of the product when fp32(1/step2) overflows; 0 when step2 == 0.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) dq_scales_kernel(
    const float* __restrict__ absmax, int64_t n_blocks, const float* __restrict__ mean_ptr,
    int8_t* __restrict__ q8, float* __restrict__ step2) {
  const int lane = threadIdx.x & 31;
  const int64_t g = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_groups = (n_blocks + kGroup - 1) / kGroup;
  if (g >= n_groups) return;                       // warp-uniform
  const float mu = *mean_ptr;
  float d[8];
  float S = 0.f;
  const int64_t base = g * kGroup + lane * 8;
  if (base + 8 <= n_blocks) {                                        // two 16-byte loads
    const float4 a = __ldg(reinterpret_cast<const float4*>(absmax + base));
    const float4 b = __ldg(reinterpret_cast<const float4*>(absmax + base + 4));
    const float c[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) d[i] = __fsub_rn(c[i], mu);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) d[i] = (base + i < n_blocks) ? __fsub_rn(absmax[base + i], mu) : 0.f;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) S = fmaxf(S, fabsf(d[i]));
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) S = fmaxf(S, __shfl_xor_sync(0xffffffffu, S, off));
  const float st = __fdiv_rn(S, 127.0f);
  if (lane == 0) step2[g] = st;
  const float inv = (st != 0.f) ? __frcp_rn(st) : 0.f;
  const bool by_div = isinf(inv);                  // subnormal step: divide instead (warp-uniform)
  uint32_t packed[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int q = 0;
    if (st != 0.f) {
      const float p = by_div ? __fdiv_rn(d[i], st) : __fmul_rn(d[i], inv);
      q = min(127, max(-127, __float2int_rn(p)));
    }
    packed[i >> 2] |= (static_cast<uint32_t>(q) & 0xFFu) << (8 * (i & 3));
  }
  if (base + 8 <= n_blocks) {
    *reinterpret_cast<uint2*>(q8 + base) = make_uint2(packed[0], packed[1]);   // one 8-byte store
  } else {
    for (int i = 0; i < 8 && base + i < n_blocks; ++i)
      q8[base + i] = static_cast<int8_t>((packed[i >> 2] >> (8 * (i & 3))) & 0xFFu);
  }
}

// ---------------------------------------------------------------------------
// K4: dequantize to bf16.  A warp takes 128 consecutive 32-bit code words
// (8 codes each, 1024 weights) per round; lane l decodes words l, l + 32,
// l + 64, l + 96, so each of its four 16-byte output stores is part of one
// 512-byte contiguous warp store, and each code load one 128-byte warp load.
// A word's block scale and 16-entry bf16 table are built by its lane (the
// eight lanes of a block share the scale code through a broadcast load).
// kDqRounds rounds are loaded before any is decoded.
// ---------------------------------------------------------------------------
constexpr int kDqRounds = 2;

__global__ void __launch_bounds__(256) nf4_dequantize_kernel(
    const uint8_t* __restrict__ codes, const int8_t* __restrict__ q8,
    const float* __restrict__ step2, const float* __restrict__ mean_ptr,
    int64_t n_words, uint16_t* __restrict__ out, Levels L) {
  const float mu = *mean_ptr;
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const uint32_t* cw = reinterpret_cast<const uint32_t*>(codes);
  for (int64_t base = warp * 128 * kDqRounds; base < n_words; base += n_warps * 128 * kDqRounds) {
    uint32_t w[kDqRounds][4];
    float ch[kDqRounds][4];
#pragma unroll
    for (int rd = 0; rd < kDqRounds; ++rd) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int64_t i = base + rd * 128 + k * 32 + lane;           // word index
        if (i < n_words) {
          const int64_t b = i >> 3;                                  // 8 words per 64-weight block
          w[rd][k] = __ldcs(cw + i);
          ch[rd][k] = block_scale(__ldg(q8 + b), __ldg(step2 + (b >> 8)), mu);
        }
      }
    }
#pragma unroll
    for (int rd = 0; rd < kDqRounds; ++rd) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int64_t i = base + rd * 128 + k * 32 + lane;
        if (i < n_words) {
          const Nf4Table t = make_table(L, ch[rd][k]);
          uint32_t o[4];
          decode8(t, w[rd][k], o);
          st_v4(out + i * 8, make_uint4(o[0], o[1], o[2], o[3]));
        }
      }
    }
  }
}

}  // namespace qnf4
