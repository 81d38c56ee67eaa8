// gemm_pair_sm100.cuh -- fused dequant-in-mainloop QLoRA GEMM on a CTA pair
// (tcgen05 cta_group::2).
//
// Same products as gemm_sm100.cuh ("QLoRA", llm-compass, 方法与公式):
//   forward  h [M, out] = [x | us] . [W0 | B]^T       K = in  + r
//   backward dx[M, in ] = [dh | du] . [W0 ; A]        K = out + r
// with W0 dequantized on the fly, but one output tile of 512 token rows x 256
// columns is computed by a pair of CTAs on two SMs.  Each UMMA is
// 256 x 256 x 16 (cta_group::2): its A rows come half from each CTA and its B
// columns half from each CTA, so each SM dequantizes only its 128-column half
// of the weight tile and its tensor core reads that half once per UMMA.
// Compared with one CTA on a 256 x 256 tile this halves both the dequant work
// per tensor-core FLOP and the shared-memory traffic for the weight operand.
//
// Per CTA (576 threads, 4-stage ring of 32 KB activation + 16 KB weight):
//   warp 0     TMA producer for this CTA's two 128-row activation tiles; the
//              copies of both CTAs complete on the even CTA's "full" barrier
//   warp 1     TMEM allocation (both CTAs); UMMA issue for the pair (even CTA)
//   warps 2-17 dequant producers in four groups of 4, each group taking every
//              fourth stage:
//              a thread decodes its next stage into registers before it
//              waits for the buffer, then stores, fences and (one lane per
//              warp) arrives on the even CTA's "full" barrier; afterwards
//              the epilogue of this CTA's 256 accumulator rows
// TMEM: two 256-column fp32 accumulators per CTA (token sub-tiles 0 and 1).
// The even CTA's "full" barrier counts its TMA arrive (with the byte count of
// both CTAs' copies) and the 8 dequant warps of both CTAs.  The even CTA
// commits each stage with a multicast arrive on both CTAs' "empty" barriers,
// and the end of the accumulation on both "acc_full".
// Every wait is bounded (see gemm_sm100.cuh); no TMA multicast is used.
#pragma once

#include "common.cuh"
#include "gemm_sm100.cuh"

namespace qnf4 {

struct PairCfg {
  static constexpr int kStages = 4;
  static constexpr int BM = 512;                       // token rows per pair
  static constexpr int BN = 256;                       // output columns per pair
  static constexpr int A_SUB = 128 * 64 * 2;           // one 128-row activation tile
  static constexpr int A_STAGE = 2 * A_SUB;            // two token sub-tiles per CTA
  static constexpr int B_STAGE = 128 * 64 * 2;         // this CTA's half of the weight tile
  static constexpr int RING = kStages * (A_STAGE + B_STAGE);
  static constexpr int SMEM = RING + 256 + 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int kGroups = 4;                    // dequant groups, one stage each in turn
  static constexpr int THREADS = 64 + kGroups * 128;   // 2 + 16 warps
};

template <bool kDx>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg::THREADS, 1)
qlora_gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_act,
                       const __grid_constant__ CUtensorMap tm_lora,
                       const GemmArgs args) {
  using Cfg = PairCfg;
  constexpr int kStages = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* a_ring = smem;
  uint8_t* b_ring = smem + kStages * Cfg::A_STAGE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::RING);
  uint64_t* full = bars;                       // (even CTA) both CTAs' stage is complete
  uint64_t* empty = bars + kStages;            // the pair's UMMAs on the stage finished
  uint64_t* acc_full = bars + 2 * kStages;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  // (even CTA) the number of stages whose copies each CTA of the pair issued
  volatile int* issued_by = reinterpret_cast<volatile int*>(tmem_holder + 2);

  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int pair = blockIdx.x >> 1;
  const int tiles_m = (args.M + Cfg::BM - 1) / Cfg::BM;
  const int tile_m = pair % tiles_m;
  const int tile_n = pair / tiles_m;
  const int m0 = tile_m * Cfg::BM;
  const int n0 = tile_n * Cfg::BN;
  const int n0_half = n0 + 128 * static_cast<int>(rank);
  const int n_main = args.K / 64;
  const int n_lora = (args.r + 63) / 64;
  const int n_iter = n_main + n_lora;
  const uint64_t tmo = args.timeout_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full + s, 1 + 8);     // TMA arrive + 4 dequant warps (one group) per CTA
      mbar_init(empty + s, 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, Cfg::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before_sync();
  __syncthreads();
  cluster_sync_all();                 // both CTAs' barriers exist before any remote arrive
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_holder;

  // bounded waits (cluster-scope acquire: other CTAs and the pair's tensor
  // cores arrive on these barriers)
  auto wait = [&](uint64_t* bar, uint32_t parity) {
    if (*abort_flag) return;
    if (!mbar_wait_cluster_bounded(bar, parity, tmo)) {
      *abort_flag = 1;
      raise_device_error(1);
    }
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_act);
      tma_prefetch_desc(&tm_lora);
      int issued = 0;
      for (int it = 0; it < n_iter; ++it) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1u;
        wait(empty + s, ph ^ 1u);
        if (*abort_flag) break;                           // a wait timed out: issue nothing more
        if (leader) mbar_arrive_expect_tx(full + s, 2 * Cfg::A_STAGE);    // both CTAs' bytes
        const uint32_t bar = mapa_shared(smem_u32(full + s), 0);
        const uint32_t dst = smem_u32(a_ring + s * Cfg::A_STAGE);
        if (it + kStages < n_main) {                      // warm L2 for a later stage
#pragma unroll
          for (int sub = 0; sub < 2; ++sub)
            tma_prefetch_l2_2d(&tm_act, (it + kStages) * 64, m0 + sub * 256 + static_cast<int>(rank) * 128);
        }
#pragma unroll
        for (int sub = 0; sub < 2; ++sub) {
          const int row = m0 + sub * 256 + static_cast<int>(rank) * 128;
          if (it < n_main)
            tma_load_2d_pair(dst + sub * Cfg::A_SUB, &tm_act, bar, it * 64, row);
          else
            tma_load_2d_pair(dst + sub * Cfg::A_SUB, &tm_lora, bar, (it - n_main) * 64, row);
        }
        ++issued;
      }
      // Copies of both CTAs complete on the even CTA's barriers, which drains
      // them after the cluster barrier below; it needs both issued counts.
      asm volatile("st.shared::cluster.u32 [%0], %1;"
                   :: "r"(mapa_shared(smem_u32(const_cast<int*>(issued_by + rank)), 0)), "r"(issued) : "memory");
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------------------------------------------------- UMMA issuer
      constexpr uint32_t idesc = umma_idesc_bf16(256, 256, kDx);
      for (int it = 0; it < n_iter; ++it) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1u;
        wait(full + s, ph);
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
          for (int sub = 0; sub < 2; ++sub) {
            const uint64_t adesc = umma_desc_sw128(a_base + sub * Cfg::A_SUB + kk * 32, 16, 1024);
            umma_bf16_ss_pair(tmem_base + sub * 256, adesc, bdesc, idesc, (it > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit_pair_multicast(empty + s, 0x3);
      }
      umma_commit_pair_multicast(acc_full, 0x3);
      mbar_wait_cluster_bounded(acc_full, 0, tmo);
    }
  } else {
    // -------------------------------------------------- dequant producers
    constexpr int G = Cfg::kGroups;
    const int group = (warp - 2) >> 2;                    // stages it = group, group+G, ...
    const int t = (threadIdx.x - 64) & 127;               // 0..127 within the group
    const int64_t w_row_bytes = args.w_cols / 2;
    const int64_t w_row_blocks = args.w_cols / 64;
    const float mu = __ldg(args.mean);

    const uint8_t* code_ptr;
    int64_t code_step, q8_idx, q8_step;
    uint32_t row_off, key;
    bool col_valid;
    int lora_row;
    if (!kDx) {
      col_valid = (n0_half + t) < args.N;
      const int64_t wr = col_valid ? (n0_half + t) : 0;
      code_ptr = args.codes + wr * w_row_bytes;
      code_step = 32;
      q8_idx = wr * w_row_blocks;
      q8_step = 1;
      row_off = t * 128;
      key = t & 7;
      lora_row = n0_half + t;
    } else {
      const int k = t & 63, a = t >> 6;
      col_valid = (n0_half + 64 * a) < args.N;
      const int64_t wc = col_valid ? (n0_half + 64 * a) : 0;
      code_ptr = args.codes + static_cast<int64_t>(k) * w_row_bytes + wc / 2;
      code_step = 64 * w_row_bytes;
      q8_idx = static_cast<int64_t>(k) * w_row_blocks + wc / 64;
      q8_step = 64 * w_row_blocks;
      row_off = a * 8192 + k * 128;
      key = k & 7;
      lora_row = k;
    }

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

    // Decode (or fetch the LoRA rows of) stage `it` into 8 x 16 B of registers.
    auto produce = [&](int it, const StageIn& in, uint4 (&v)[8]) {
      if (it < n_main) {
        if (col_valid) {
          const float c_hat = block_scale(in.q, in.st, mu);
          const Nf4Table tb = make_table(args.L, c_hat);
          const uint32_t w[8] = {in.c0.x, in.c0.y, in.c0.z, in.c0.w, in.c1.x, in.c1.y, in.c1.z, in.c1.w};
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint32_t o[4];
            decode8(tb, w[c], o);
            v[c] = make_uint4(o[0], o[1], o[2], o[3]);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 8; ++c) v[c] = make_uint4(0, 0, 0, 0);
        }
      } else {
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
            src = args.lora_w + static_cast<int64_t>(kr) * args.w_cols + n0_half + 64 * (t >> 6);
            count = 64;
          }
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) v[c] = (c * 8 < count) ? ld_nc_v4(src + c * 8) : make_uint4(0, 0, 0, 0);
      }
    };

    // codes and scale codes are loaded two of this group's turns ahead (eight
    // stages), so their global-load latency overlaps two turns of MMAs
    StageIn na{}, nb{};
    load_stage(group, na);
    load_stage(group + G, nb);
    const bool warp_lead = lane == 0;

    for (int it = group; it < n_iter; it += G) {
      const StageIn cur = na;
      na = nb;
      load_stage(it + 2 * G, nb);
      uint4 v[8];
      produce(it, cur, v);                          // before waiting for the buffer

      const int s = it % kStages;
      const uint32_t ph = (it / kStages) & 1u;
      const uint32_t dst = smem_u32(b_ring + s * Cfg::B_STAGE) + row_off;
      wait(empty + s, ph ^ 1u);
#pragma unroll
      for (int c = 0; c < 8; ++c) sts_v4(dst + ((c ^ key) << 4), v[c].x, v[c].y, v[c].z, v[c].w);
      fence_proxy_async_smem();
      __syncwarp();
      if (warp_lead) mbar_arrive_remote(mapa_shared(smem_u32(full + s), 0));
    }

    // ------------------------------------------------------------ epilogue
    // This CTA's TMEM holds 128 rows (lanes) x 256 columns for each token
    // sub-tile; each of the 16 warps writes 128 columns of one sub-tile for
    // the 32 lanes of its quadrant.
    wait(acc_full, 0);
    tc_fence_after_sync();
    const int q = warp & 3;
    const int part = (warp - 2) >> 2;                     // 0..3
    const int sub = part >> 1;
    const int m = m0 + sub * 256 + static_cast<int>(rank) * 128 + q * 32 + lane;
    for (int col = (part & 1) * 128; col < (part & 1) * 128 + 128; col += 32) {
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
  cluster_sync_all();                 // both issued counts are visible to the even CTA
  if (leader && warp == 0 && lane == 0) {
    // Wait (bounded) for the stages whose copies may still be in flight: a
    // stage more than kStages behind the last one issued was consumed, so
    // its copies have landed.  Without a timeout every phase has completed
    // and these waits return at once.
    const int n = max(issued_by[0], issued_by[1]);
    for (int it = n > kStages ? n - kStages : 0; it < n; ++it)
      mbar_wait_cluster_bounded(full + (it % kStages), (it / kStages) & 1u, tmo);
  }
  cluster_sync_all();                 // no CTA leaves while its pair may still use its memory
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
  }
}

}  // namespace qnf4
