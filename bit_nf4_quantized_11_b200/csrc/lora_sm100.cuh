// lora_sm100.cuh -- the rank-r contractions of the QLoRA layer on tcgen05.
//
// ("QLoRA", llm-compass, 方法与公式: h = dequant(W0) x + (alpha/r) B A x, with
// gradients for A and B only; aigrafen.se, opening paragraph.)
//
// All four products have one dimension equal to the LoRA rank r and stream a
// token-sized operand from HBM once, so they are bound by that read.  Each is
// one tcgen05 tile product D[128 x N] (+)= A . B^T with N = r rounded up to a
// multiple of 16 (at most 256), fp32 accumulation in tensor memory, both
// operands staged by TMA (128-byte swizzle) in a ring of shared-memory stages:
//
//   row form  out[m][j] = bf16(scale * sum_k act[m][k] * w(j, k))
//     us = bf16(s x A^T)   act = x  [M, in]  (K-major), w = A [r, in]  (K-major)
//     du = bf16(s dh B)    act = dh [M, out] (K-major), w = B [out, r] (N-major)
//   col form  D[f][j] = scale * sum_m act[m][f] * u[m][j]
//     dB   = dh^T us       act = dh [M, out] (MN-major), u = us [M, r] (N-major)
//     dA^T = x^T du        act = x  [M, in]  (MN-major), u = du [M, r] (N-major)
//
// The tile rows are tokens (row form) or features (col form); the
// contraction (K of the row form, the tokens of the col form) is split over
// the CTAs of a thread-block cluster (at most 8).  Each CTA moves its fp32
// partial tile from tensor memory to its own shared memory; then every CTA
// adds up its share of the tile's rows over distributed shared memory,
// partials in rank order (deterministic), and stores it.
//
// Roles (128 threads, 320 with a keep mask): warp 0 lane 0 issues the TMA
// loads, warp 1 allocates tensor memory and its lane 0 issues the MMAs, and
// with a LoRA-dropout keep mask warps 2-9 zero the dropped activations of
// each landed stage in shared memory (bit c % 8 of byte c / 8 of a token's
// row keeps column c) before the MMAs read it; afterwards warps 0-3 read the
// accumulator (warp w owns rows 32 w .. 32 w + 31, its TMEM lanes) and all
// warps take part in the cluster reduction.
// Every wait is bounded: on timeout the CTA sets the device error flag,
// issues nothing more, waits (bounded) for what it issued and exits.
// No TMA multicast is used.
#pragma once

#include "common.cuh"

namespace qnf4 {

constexpr int kLrThreads = 128;
constexpr int kLrMaskThreads = 320;                        // with a keep mask: eight masking warps
constexpr int kLrMaxStages = 8;
constexpr int kLrTileRows = 128;
constexpr int kLrAStage = kLrTileRows * 64 * 2;           // 16 KB: 128 rows x 64 k (or two 64-wide MN atoms)

// Instruction descriptor, kind::f16 with bf16 A and B, fp32 D; either
// operand K-major or MN-major.
__host__ __device__ constexpr uint32_t umma_idesc_bf16_ab(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

struct LrProblem {
  void* out;             // row form: bf16 [rows, r]; col form: fp32 [rows, r] or, transposed, [r, rows]
  int rows;              // tokens (row form) or features (col form)
  int tiles;             // ceil(rows / 128)
  int transpose_out;     // col form: write D^T (dA [r, in])
  float scale;
  const uint8_t* keep;   // LoRA dropout keep bits of the token operand [tokens, features / 8], or null
  int features;          // columns of the token operand (row form: K; col form: rows)
};

struct LrArgs {
  LrProblem p[2];        // blockIdx.x < p[0].tiles: problem 0, else problem 1
  int K;                 // contraction length (row form: features; col form: tokens)
  int r;                 // rank
  int N;                 // r rounded up to 16
  int n_alloc;           // TMEM columns (power of two >= 32, >= N)
  int stages_per_split;  // 64-wide contraction stages per CTA of the cluster
  int ring;              // shared-memory stages in flight (<= kLrMaxStages)
  uint64_t timeout_ns;
};

// Shared bytes of one stage of the B operand (N rows x 64 k K-major, or
// ceil(N / 64) atoms of 64 n x 64 k) and of the fp32 partial tile (padded rows).
__host__ __device__ constexpr int lr_b_stage(int N, bool b_mn_major) {
  return b_mn_major ? ((N + 63) / 64) * 8192 : ((N * 128 + 1023) / 1024) * 1024;
}
__host__ __device__ constexpr int lr_partial_pitch(int N) { return N * 4 + 16; }
__host__ __device__ constexpr int lr_smem_bytes(int N, bool b_mn_major, int stages) {
  const int ring = stages * (kLrAStage + lr_b_stage(N, b_mn_major));
  const int part = kLrTileRows * lr_partial_pitch(N);
  return (ring > part ? ring : part) + 512 + 1024;
}

// kCol: col form (A MN-major, output fp32); otherwise row form (A K-major,
// output bf16).  kBMN: B operand N-major.
template <bool kCol, bool kBMN>
__global__ void __launch_bounds__(kLrMaskThreads) lora_umma_kernel(
    const __grid_constant__ CUtensorMap tm_a0, const __grid_constant__ CUtensorMap tm_b0,
    const __grid_constant__ CUtensorMap tm_a1, const __grid_constant__ CUtensorMap tm_b1, const LrArgs args) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const int N = args.N;
  const int b_stage = lr_b_stage(N, kBMN);
  const int S = args.ring;                                           // stages of the ring
  const int ring_bytes = S * (kLrAStage + b_stage);
  const int part_bytes = kLrTileRows * lr_partial_pitch(N);
  uint8_t* a_ring = smem;
  uint8_t* b_ring = smem + S * kLrAStage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (ring_bytes > part_bytes ? ring_bytes : part_bytes));
  uint64_t* full = bars;
  uint64_t* empty = bars + kLrMaxStages;
  uint64_t* masked = bars + 2 * kLrMaxStages;                        // (keep mask) the stage is masked
  uint64_t* acc_full = bars + 3 * kLrMaxStages;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int prob = static_cast<int>(blockIdx.x) < args.p[0].tiles ? 0 : 1;
  // fields of this CTA's problem (selected, not indexed: no local-memory copy)
  void* const p_out = prob == 0 ? args.p[0].out : args.p[1].out;
  const int p_rows = prob == 0 ? args.p[0].rows : args.p[1].rows;
  const bool p_transpose = (prob == 0 ? args.p[0].transpose_out : args.p[1].transpose_out) != 0;
  const float p_scale = prob == 0 ? args.p[0].scale : args.p[1].scale;
  const uint8_t* const p_keep = prob == 0 ? args.p[0].keep : args.p[1].keep;
  const int p_features = prob == 0 ? args.p[0].features : args.p[1].features;
  const bool do_mask = p_keep != nullptr;                            // CTA-uniform
  const int tile = prob == 0 ? static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.x) - args.p[0].tiles;
  const CUtensorMap* tm_a = prob == 0 ? &tm_a0 : &tm_a1;
  const CUtensorMap* tm_b = prob == 0 ? &tm_b0 : &tm_b1;
  const int row0 = tile * kLrTileRows;
  const int ks = static_cast<int>(gridDim.y);
  const int split = static_cast<int>(blockIdx.y);
  const int n_stages_total = (args.K + 63) / 64;
  const int st_begin = split * args.stages_per_split;
  const int st_end = min(n_stages_total, st_begin + args.stages_per_split);
  const int n_iter = max(0, st_end - st_begin);
  const uint64_t tmo = args.timeout_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
      mbar_init(masked + s, (blockDim.x - 64) / 32);                 // one arrive per masking warp
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, static_cast<uint32_t>(args.n_alloc));
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_holder;

  auto wait = [&](uint64_t* bar, uint32_t parity) {
    if (*abort_flag) return;
    if (!mbar_wait_bounded(bar, parity, tmo)) {
      *abort_flag = 1;
      raise_device_error(1);
    }
  };

  const uint32_t stage_tx = static_cast<uint32_t>(kLrAStage + b_stage);
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(tm_a);
      tma_prefetch_desc(tm_b);
      int issued = 0;
      for (int it = 0; it < n_iter; ++it) {
        const int s = it % S;
        wait(empty + s, ((it / S) & 1u) ^ 1u);
        if (*abort_flag) break;
        mbar_arrive_expect_tx(full + s, stage_tx);
        const uint32_t a_dst = smem_u32(a_ring + s * kLrAStage);
        const uint32_t b_dst = smem_u32(b_ring + s * b_stage);
        const int k0 = (st_begin + it) * 64;
        if (!kCol) {
          tma_load_2d(a_dst, tm_a, full + s, k0, row0);                      // [128 rows x 64 k]
        } else {
          tma_load_2d(a_dst, tm_a, full + s, row0, k0);                      // two atoms of 64 features x 64 tokens
          tma_load_2d(a_dst + 8192, tm_a, full + s, row0 + 64, k0);
        }
        if (!kBMN) {
          tma_load_2d(b_dst, tm_b, full + s, k0, 0);                         // [N rows x 64 k]
        } else {
          for (int a = 0; a * 64 < N; ++a) tma_load_2d(b_dst + a * 8192, tm_b, full + s, a * 64, k0);
        }
        ++issued;
      }
      // only the last S issued stages can still be in flight
      for (int it = issued > S ? issued - S : 0; it < issued; ++it)
        mbar_wait_bounded(full + (it % S), (it / S) & 1u, tmo);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      const uint32_t idesc = umma_idesc_bf16_ab(kLrTileRows, N, kCol, kBMN);
      for (int it = 0; it < n_iter; ++it) {
        const int s = it % S;
        wait(full + s, (it / S) & 1u);
        if (do_mask) wait(masked + s, (it / S) & 1u);
        if (*abort_flag) break;
        tc_fence_after_sync();
        const uint32_t a_base = smem_u32(a_ring + s * kLrAStage);
        const uint32_t b_base = smem_u32(b_ring + s * b_stage);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t adesc = kCol ? umma_desc_sw128(a_base + kk * 2048, 8192, 1024)
                                      : umma_desc_sw128(a_base + kk * 32, 16, 1024);
          const uint64_t bdesc = kBMN ? umma_desc_sw128(b_base + kk * 2048, 8192, 1024)
                                      : umma_desc_sw128(b_base + kk * 32, 16, 1024);
          umma_bf16_ss(tmem_base, adesc, bdesc, idesc, (it > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(empty + s);
      }
      umma_commit(acc_full);
      mbar_wait_bounded(acc_full, 0, tmo);
    }
  } else if (do_mask) {
    // ------------------------------------------------------------ keep mask
    // The MT = blockDim - 64 masking threads split a stage into 256 items,
    // (row i, half q) = (j % 128, j / 128) for j = t + MT h: row form, token
    // row0 + i; col form, token k0 + i % 64 of the 64-feature atom i / 64;
    // half q is 16-byte chunks 4q .. 4q + 3 of the row (32 values, one
    // 32-bit word of keep bits).  In each landed stage the thread zeroes the
    // values of its items whose keep bit is 0.
    const int t = threadIdx.x - 64;
    const int MT = static_cast<int>(blockDim.x) - 64;
    const int n_items = 2 * kLrTileRows / MT;                        // 1, 2 or 4 per thread
    const int64_t kb_row = p_features / 8;                           // keep bytes per token
    auto mask_chunk16 = [](uint32_t addr, uint32_t bits) {           // 8 bf16 at addr, bit e keeps value e
      uint32_t v[4];
      asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
                   : "r"(addr) : "memory");
#pragma unroll
      for (int e = 0; e < 4; ++e)
        v[e] &= ((bits >> (2 * e)) & 1u ? 0x0000FFFFu : 0u) | ((bits >> (2 * e + 1)) & 1u ? 0xFFFF0000u : 0u);
      sts_v4(addr, v[0], v[1], v[2], v[3]);
    };
    // keep-bit address of item h of stage `it`, or null past the token or feature end
    auto keep_ptr = [&](int it, int h) -> const uint32_t* {
      if (it >= n_iter || h >= n_items) return nullptr;
      const int j = t + MT * h, i = j & (kLrTileRows - 1), q = j >> 7;
      const int k0 = (st_begin + it) * 64;
      int64_t tok, f0;
      if (!kCol) { tok = row0 + i; f0 = k0; }
      else { tok = k0 + (i & 63); f0 = row0 + 64 * (i >> 6); }
      const int64_t n_tok = kCol ? args.K : p_rows;
      if (tok >= n_tok || f0 >= p_features) return nullptr;
      return reinterpret_cast<const uint32_t*>(p_keep + tok * kb_row + f0 / 8) + q;   // 4-byte aligned
    };
    auto load_keep = [&](int it, uint32_t (&kb)[4]) {
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const uint32_t* src = keep_ptr(it, h);
        kb[h] = src != nullptr ? __ldg(src) : 0u;
      }
    };
    // loaded into registers two stages ahead and brought into L2 six stages
    // ahead, so their latency overlaps the stream
    auto prefetch_keep = [&](int it) {
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const uint32_t* src = keep_ptr(it, h);
        if (src != nullptr) asm volatile("prefetch.global.L2 [%0];" :: "l"(src));
      }
    };
    for (int i = 2; i < 6; ++i) prefetch_keep(i);
    uint32_t kb_n1[4], kb_n2[4];
    load_keep(0, kb_n1);
    load_keep(1, kb_n2);
    for (int it = 0; it < n_iter; ++it) {
      const int s = it % S;
      uint32_t kb[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        kb[h] = kb_n1[h];
        kb_n1[h] = kb_n2[h];
      }
      load_keep(it + 2, kb_n2);
      prefetch_keep(it + 6);
      wait(full + s, (it / S) & 1u);
      if (*abort_flag) break;
      const uint32_t a_base = smem_u32(a_ring + s * kLrAStage);
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        if (h >= n_items) continue;
        const int j = t + MT * h, i = j & (kLrTileRows - 1), q = j >> 7;
        // row form: row i of the 128-row tile; col form: row i % 64 of atom i / 64
        const int r = kCol ? (i & 63) : i;
        const uint32_t rbase = a_base + (kCol ? (i >> 6) * 8192 : 0) + r * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t bits = (kb[h] >> (8 * c)) & 0xFFu;
          if (bits != 0xFFu) mask_chunk16(rbase + ((((4 * q + c) ^ r) & 7) << 4), bits);
        }
      }
      fence_proxy_async_smem();                                     // generic writes before the MMAs read
      __syncwarp();
      if (lane == 0) mbar_arrive(masked + s);
    }
  }

  // ---------------------------------------------------------------- epilogue
  // Wait for the accumulator (the commit arrives even when no stage was
  // issued; an empty split leaves zeros).
  __syncwarp();
  wait(acc_full, 0);
  tc_fence_after_sync();
  const int row = warp * 32 + lane;                                  // this thread's TMEM lane / tile row
  const int pitch = lr_partial_pitch(N);
  uint8_t* part = smem;                                              // the ring is free once acc_full completed
  __syncthreads();                                                   // every stage read by the tensor cores
  for (int c0 = 0; warp < 4 && c0 < N; c0 += 32) {
    uint32_t v[32];
    tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(warp * 32) << 16) + c0, v);
    tmem_ld_wait();
    if (n_iter == 0) {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = 0u;                        // nothing accumulated
    }
    const uint32_t dst = smem_u32(part + row * pitch + c0 * 4);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (c0 + 4 * i < N) sts_v4(dst + 16 * i, v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  }
  tc_fence_before_sync();
  __syncthreads();
  if (ks > 1) cluster_sync_all();                                    // every CTA's partial is in place

  // this CTA's share of the tile's rows, summed over the cluster in rank order
  const int share = kLrTileRows / ks;
  const int r_lo = split * share;
  const int n4 = args.r / 4;                                         // float4 groups of the rank
  for (int e = threadIdx.x; e < share * n4; e += static_cast<int>(blockDim.x)) {
    int rr, c4;
    if (kCol && p_transpose) {                                   // rows fastest: coalesced dA^T stores
      rr = r_lo + e % share;
      c4 = e / share;
    } else {
      rr = r_lo + e / n4;
      c4 = e % n4;
    }
    const int grow = row0 + rr;
    const uint32_t addr = smem_u32(part + rr * pitch + c4 * 16);
    float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int rk = 0; rk < ks; ++rk) {
      float4 u;
      if (ks == 1) {
        asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(u.x), "=f"(u.y), "=f"(u.z), "=f"(u.w)
                     : "r"(addr) : "memory");
      } else {
        asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                     : "=f"(u.x), "=f"(u.y), "=f"(u.z), "=f"(u.w) : "r"(mapa_shared(addr, rk)) : "memory");
      }
      t.x += u.x; t.y += u.y; t.z += u.z; t.w += u.w;
    }
    if (grow >= p_rows) continue;
    const float sc = p_scale;
    if (!kCol) {
      uint16_t* o = static_cast<uint16_t*>(p_out) + static_cast<int64_t>(grow) * args.r + c4 * 4;
      *reinterpret_cast<uint2*>(o) = make_uint2(pack_bf16x2_rn(t.x * sc, t.y * sc), pack_bf16x2_rn(t.z * sc, t.w * sc));
    } else if (!p_transpose) {
      float* o = static_cast<float*>(p_out) + static_cast<int64_t>(grow) * args.r + c4 * 4;
      *reinterpret_cast<float4*>(o) = make_float4(t.x * sc, t.y * sc, t.z * sc, t.w * sc);
    } else {
      float* o = static_cast<float*>(p_out);
      const int64_t ld = p_rows;
      o[static_cast<int64_t>(c4 * 4 + 0) * ld + grow] = t.x * sc;
      o[static_cast<int64_t>(c4 * 4 + 1) * ld + grow] = t.y * sc;
      o[static_cast<int64_t>(c4 * 4 + 2) * ld + grow] = t.z * sc;
      o[static_cast<int64_t>(c4 * 4 + 3) * ld + grow] = t.w * sc;
    }
  }
  if (ks > 1) cluster_sync_all();                                    // no CTA leaves while others read it
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, static_cast<uint32_t>(args.n_alloc));
  }
}

}  // namespace qnf4
