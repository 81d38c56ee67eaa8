// gemm_sm100.cuh -- fused dequant-in-mainloop QLoRA GEMM on tcgen05/TMEM.
//
// One kernel computes both large-M products of the QLoRA linear layer
// ("QLoRA", llm-compass, 方法与公式: h = dequant(W0) x + (alpha/r) B A x; the
// gradient flows through the frozen quantized base):
//
//   forward  h [M, out] = [x | us] . [W0 | B]^T       K = in  + r
//   backward dx[M, in ] = [dh | du] . [W0 ; A]        K = out + r
//
// with W0 dequantized on the fly ("Hoe het werkt" diagram of the auryth
// glossary page: NF4 -> 16-bit per layer, on the fly).  The LoRA branch is the
// extra rank-r K-slice appended after the main K loop.
//
// Tiling (per CTA, one output tile, 576 threads):
//   BM = 128*MS token rows (A operand: x or dh, TMA-loaded, 128B swizzle)
//   BN = 256 output columns (B operand: dequantized W0 written to shared
//        memory by 8 dequant warps, in the UMMA 128B-swizzled layout;
//        K-major for the forward, MN-major for dx)
//   BK = 64 (one NF4 block along K per stage for the forward; for dx each
//        stage spans 64 rows of W0, and every thread's 64 columns are one
//        block)
//   fp32 accumulators in TMEM (MS x 256 columns), UMMA 128x256x16 issued by
//   one thread, kStages-deep shared-memory ring with mbarriers.
// Warp roles: warp 0 TMA producer, warp 1 TMEM allocator + UMMA issuer,
// warps 2..17 dequant producers in two groups of 8 that take alternate
// stages (so each thread has two stages of time to hide its global loads),
// then all 16 run the epilogue (TMEM -> bf16 -> HBM).
//
// Every mbarrier wait is bounded: after the timeout the CTA sets the device
// error flag, stops waiting, lets every role run to the end of its fixed trip
// count, waits (bounded) for its own TMA loads and MMAs, frees TMEM and exits.
#pragma once

#include "common.cuh"

namespace qnf4 {

struct GemmArgs {
  const uint8_t* codes;   // [w_rows, w_cols/2]
  const int8_t* q8;       // [w_rows*w_cols/64]
  const float* step2;
  const float* mean;
  const uint16_t* lora_w; // forward: B [out, r]; dx: A [r, in]
  uint16_t* out;          // forward: h [M, out]; dx: dx [M, in]
  int M;                  // token rows
  int N;                  // output columns (forward: out, dx: in)
  int K;                  // main contraction length (forward: in, dx: out)
  int r;                  // LoRA rank (multiple of 8)
  int w_cols;             // columns of W0 (= in)
  int codes_32b;          // codes 32-byte aligned: a thread's 32 code bytes in one load
  Levels L;
  uint64_t timeout_ns;
};

template <int MS, int kStages>
struct GemmCfg {
  static constexpr int BM = 128 * MS;
  static constexpr int BN = 256;
  static constexpr int BK = 64;
  static constexpr int A_SUB = 128 * 64 * 2;                 // one 128-row A tile, bytes
  static constexpr int A_STAGE = MS * A_SUB;
  static constexpr int B_STAGE = BN * BK * 2;                // 32 KB
  static constexpr int RING = kStages * (A_STAGE + B_STAGE);
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM = RING + BAR_BYTES + 1024;       // + alignment slack
  static constexpr uint32_t TMEM_COLS = MS * 256;            // 256 or 512
  static constexpr int THREADS = 576;                         // 2 + 16 warps
};

// Bounded wait shared by all roles of a CTA; after the first timeout every
// later wait returns immediately.
__device__ __forceinline__ void pipe_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns,
                                          volatile int* abort_flag) {
  if (*abort_flag) return;
  if (!mbar_wait_bounded(bar, parity, timeout_ns)) {
    *abort_flag = 1;
    raise_device_error(1);
  }
}

template <int MS, bool kDx, int kStages>
__global__ void __launch_bounds__(576, 1)
qlora_gemm_kernel(const __grid_constant__ CUtensorMap tm_act,
                  const __grid_constant__ CUtensorMap tm_lora,
                  const GemmArgs args) {
  using Cfg = GemmCfg<MS, kStages>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment of the ring (required by the 128B swizzle atoms)
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* a_ring = smem;
  uint8_t* b_ring = smem + kStages * Cfg::A_STAGE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::RING);
  uint64_t* full_a = bars;
  uint64_t* full_b = bars + kStages;
  uint64_t* empty = bars + 2 * kStages;
  uint64_t* acc_full = bars + 3 * kStages;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tiles_m = (args.M + Cfg::BM - 1) / Cfg::BM;
  const int tile_m = blockIdx.x % tiles_m;
  const int tile_n = blockIdx.x / tiles_m;
  const int m0 = tile_m * Cfg::BM;
  const int n0 = tile_n * Cfg::BN;
  const int n_main = args.K / Cfg::BK;
  const int n_lora = (args.r + 63) / 64;
  const int n_iter = n_main + n_lora;
  const uint64_t tmo = args.timeout_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_a + s, 1);
      mbar_init(full_b + s, 256);
      mbar_init(empty + s, 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_act);
      tma_prefetch_desc(&tm_lora);
      int issued = 0;
      for (int it = 0; it < n_iter; ++it) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1u;
        pipe_wait(empty + s, ph ^ 1u, tmo, abort_flag);
        if (*abort_flag) break;                           // a wait timed out: issue nothing more
        mbar_arrive_expect_tx(full_a + s, Cfg::A_STAGE);
        const uint32_t dst = smem_u32(a_ring + s * Cfg::A_STAGE);
#pragma unroll
        for (int sub = 0; sub < MS; ++sub) {
          if (it < n_main)
            tma_load_2d(dst + sub * Cfg::A_SUB, &tm_act, full_a + s, it * 64, m0 + sub * 128);
          else
            tma_load_2d(dst + sub * Cfg::A_SUB, &tm_lora, full_a + s, (it - n_main) * 64, m0 + sub * 128);
        }
        ++issued;
      }
      // make sure no copy is still in flight when the CTA exits: only the
      // last kStages issued stages can be unconsumed
      for (int it = issued > kStages ? issued - kStages : 0; it < issued; ++it)
        mbar_wait_bounded(full_a + (it % kStages), (it / kStages) & 1u, tmo);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16(128, 256, kDx);
      for (int it = 0; it < n_iter; ++it) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1u;
        pipe_wait(full_a + s, ph, tmo, abort_flag);
        pipe_wait(full_b + s, ph, tmo, abort_flag);
        if (*abort_flag) break;                           // commit what was issued, then finish
        tc_fence_after_sync();
        const uint32_t a_base = smem_u32(a_ring + s * Cfg::A_STAGE);
        const uint32_t b_base = smem_u32(b_ring + s * Cfg::B_STAGE);
        int ksteps = 4;
        if (it >= n_main) ksteps = min(4, (args.r - (it - n_main) * 64 + 15) / 16);
        for (int kk = 0; kk < ksteps; ++kk) {
          const uint64_t bdesc = kDx ? umma_desc_sw128(b_base + kk * 2048, 8192, 1024)
                                     : umma_desc_sw128(b_base + kk * 32, 16, 1024);
#pragma unroll
          for (int sub = 0; sub < MS; ++sub) {
            const uint64_t adesc = umma_desc_sw128(a_base + sub * Cfg::A_SUB + kk * 32, 16, 1024);
            umma_bf16_ss(tmem_base + sub * 256, adesc, bdesc, idesc, (it > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(empty + s);     // frees the stage when these MMAs finish
      }
      umma_commit(acc_full);        // accumulators complete
      mbar_wait_bounded(acc_full, 0, tmo);
    }
  } else {
    // -------------------------------------------------- dequant producers
    const int group = (warp - 2) >> 3;                    // stages it = group, group+2, ...
    const int t = (threadIdx.x - 64) & 255;               // 0..255 within the group
    const int64_t w_row_bytes = args.w_cols / 2;
    const int64_t w_row_blocks = args.w_cols / 64;
    const float mu = __ldg(args.mean);

    // Per-thread walk over the packed weight: stage `it` reads 32 code bytes
    // at code_ptr + it*code_step and one scale code at q8_idx + it*q8_step.
    const uint8_t* code_ptr;
    int64_t code_step, q8_idx, q8_step;
    uint32_t row_off;     // byte offset of this thread's 128-byte row in a B stage
    uint32_t key;         // 128B-swizzle key (row index mod 8)
    bool col_valid;
    int lora_row;         // row of the LoRA matrix copied in the LoRA stages
    if (!kDx) {
      const int n = t;                                    // output column = W0 row
      col_valid = (n0 + n) < args.N;
      const int64_t wr = col_valid ? (n0 + n) : 0;
      code_ptr = args.codes + wr * w_row_bytes;
      code_step = 32;
      q8_idx = wr * w_row_blocks;
      q8_step = 1;
      row_off = n * 128;
      key = n & 7;
      lora_row = n0 + n;
    } else {
      const int k = t & 63, a = t >> 6;                   // W0 row in stage, 64-col atom
      col_valid = (n0 + 64 * a) < args.N;
      const int64_t wc = col_valid ? (n0 + 64 * a) : 0;
      code_ptr = args.codes + static_cast<int64_t>(k) * w_row_bytes + wc / 2;
      code_step = 64 * w_row_bytes;
      q8_idx = static_cast<int64_t>(k) * w_row_blocks + wc / 64;
      q8_step = 64 * w_row_blocks;
      row_off = a * 8192 + k * 128;
      key = k & 7;
      lora_row = k;
    }

    // everything one stage needs from global memory, loaded ahead of use
    struct StageIn {
      uint4 c0, c1;
      int q;
      float st;
    };
    auto load_stage = [&](int it, StageIn& d) {
      if (col_valid && it < n_main) {
        const uint8_t* p = code_ptr + it * code_step;
        const int64_t blk = q8_idx + it * q8_step;
        if (args.codes_32b) {
          ld_nc_v8(p, d.c0, d.c1);
        } else {
          d.c0 = ld_nc_v4(p);
          d.c1 = ld_nc_v4(p + 16);
        }
        d.q = __ldg(args.q8 + blk);
        d.st = __ldg(args.step2 + blk / 256);
      }
    };

    StageIn na{}, nb{};
    load_stage(group, na);
    load_stage(group + 2, nb);

    for (int it = group; it < n_iter; it += 2) {
      const StageIn cur = na;
      na = nb;
      load_stage(it + 4, nb);

      const int s = it % kStages;
      const uint32_t ph = (it / kStages) & 1u;
      const uint32_t dst = smem_u32(b_ring + s * Cfg::B_STAGE) + row_off;
      pipe_wait(empty + s, ph ^ 1u, tmo, abort_flag);

      if (it < n_main) {
        if (col_valid) {
          const float c_hat = block_scale(cur.q, cur.st, mu);
          const Nf4Table tb = make_table(args.L, c_hat);
          const uint32_t w[8] = {cur.c0.x, cur.c0.y, cur.c0.z, cur.c0.w, cur.c1.x, cur.c1.y, cur.c1.z, cur.c1.w};
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint32_t o[4];
            decode8(tb, w[c], o);
            sts_v4(dst + ((c ^ key) << 4), o[0], o[1], o[2], o[3]);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 8; ++c) sts_v4(dst + (c << 4), 0u, 0u, 0u, 0u);
        }
      } else {
        // LoRA K-slice: copy 64 bf16 of B (forward) or A (dx), zero-padded
        const int j = it - n_main;
        const uint16_t* src = nullptr;
        int count = 0;
        if (!kDx) {
          if (col_valid) {
            src = args.lora_w + static_cast<int64_t>(lora_row) * args.r + j * 64;
            count = min(64, args.r - j * 64);
          }
        } else {
          const int kr = j * 64 + lora_row;
          if (col_valid && kr < args.r) {
            src = args.lora_w + static_cast<int64_t>(kr) * args.w_cols + n0 + 64 * (t >> 6);
            count = 64;
          }
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4 v = make_uint4(0, 0, 0, 0);
          if (c * 8 < count) v = ld_nc_v4(src + c * 8);
          sts_v4(dst + ((c ^ key) << 4), v.x, v.y, v.z, v.w);
        }
      }
      fence_proxy_async_smem();      // generic-proxy writes -> tensor-core reads
      mbar_arrive(full_b + s);
    }

    // ------------------------------------------------------------ epilogue
    // 16 warps: 4 per TMEM lane quadrant, each takes a quarter of the
    // quadrant's accumulator columns.
    pipe_wait(acc_full, 0, tmo, abort_flag);
    tc_fence_after_sync();
    const int q = warp & 3;                       // TMEM lane quadrant of this warp
    const int part = (warp - 2) >> 2;             // 0..3
    const int sub = (MS == 2) ? (part >> 1) : 0;
    const int c_count = (MS == 2) ? 128 : 64;
    const int c_begin = (MS == 2) ? (part & 1) * 128 : part * 64;
    const int m = m0 + sub * 128 + q * 32 + lane;
    for (int cc = 0; cc < c_count; cc += 32) {
      const int col = c_begin + cc;
      uint32_t v[32];
      tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + sub * 256 + col, v);
      tmem_ld_wait();
      if (m < args.M && n0 + col < args.N) {
        uint16_t* dstp = args.out + static_cast<int64_t>(m) * args.N + n0 + col;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 o = make_uint4(
              pack_bf16x2_rn(__uint_as_float(v[8 * i + 0]), __uint_as_float(v[8 * i + 1])),
              pack_bf16x2_rn(__uint_as_float(v[8 * i + 2]), __uint_as_float(v[8 * i + 3])),
              pack_bf16x2_rn(__uint_as_float(v[8 * i + 4]), __uint_as_float(v[8 * i + 5])),
              pack_bf16x2_rn(__uint_as_float(v[8 * i + 6]), __uint_as_float(v[8 * i + 7])));
          st_v4(dstp + 8 * i, o);
        }
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

// Diagnostic: one thread waits on a barrier phase that nothing completes,
// bounded by timeout_ns; the timeout path sets the device error flag and the
// kernel returns normally.
__global__ void wait_timeout_selftest_kernel(uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait_bounded(&bar, 0, timeout_ns)) raise_device_error(2);
}

}  // namespace qnf4
