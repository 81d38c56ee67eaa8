// gemv.cuh -- few-token (M <= 16) QLoRA forward: streaming NF4 GEMV.
//
// With 1..16 tokens the layer is bound by streaming the packed weight from
// HBM (0.52 byte per weight), so the kernel is organised around that stream
// and around the issue and load/store-unit budget per weight it leaves
// ("QLoRA", llm-compass, 方法与公式: h = dequant(W0) x + (alpha/r) B A x; the
// auryth glossary's "Hoe het werkt" diagram: W0 is dequantized on the fly per
// layer).
//
// Work decomposition.  Every warp of a CTA owns one 256-column K slice (four
// 64-weight blocks); the WARPS slices of a CTA form a K group.  An item is
// (K group, 16-row tile); items are ordered group-major and a persistent grid
// of one CTA per SM splits them evenly by work, so each CTA mostly stays in
// one group and each warp keeps the activations of its slice in registers
// for the whole run (loaded once per group, never re-read per tile).
//
// Stream.  Each warp runs its own TMA pipeline: lane 0 loads the 16 x 128-byte
// code tile of its slice (128-byte swizzle) into a private ring of stages and
// refills a stage as soon as the warp has read it; no barrier couples the
// warps while they stream.
//
// Decode and MMA.  A warp computes its slice of a tile with warp-level bf16
// MMAs (m16n8k16: the 16 weight rows x 8 tokens); each MMA covers 16 columns
// of ONE block (quad lane q takes columns 16q + 4s .. +3 of the block in step
// s, the same permuted K order for weights and activations), so a block's
// four MMAs accumulate into a fresh fp32 tile that is added to the running
// sum times the block's exact fp32 scale c_hat.  The weight operand is
// bf16(level), exactly rounded; the GEMM path's bf16(level * c_hat) differs
// from it by at most 2^-9 relative per weight, far inside the tolerance.
// Rows g (g = lane / 4) are decoded through a shared-memory table of bf16
// level pairs (one prmt and one load per code byte); rows g + 8 through a
// register-resident 16-entry table selected with prmt (no memory access), so
// the decode splits its work between the load/store unit and the ALUs.
// A block's scale is computed once per quad lane and passed to the other
// three lanes by shuffles.
//
// Reduction.  Each warp leaves its partial tile (16 rows x tokens) in the
// free upper halves of the table's rows; every few items the CTA sums the
// warps' partials in warp order.  With one K group that sum, plus the LoRA
// term us . B^T, is the output; otherwise it is the group's fp32 partial,
// and gemv_finalize_kernel adds the groups' partials in group order and the
// LoRA term.  Every summation order is fixed, so h is deterministic.
#pragma once

#include "common.cuh"

namespace qnf4 {

constexpr int kGvSlice = 256;                             // K columns per warp (four blocks)
constexpr int kGvTile = 16;                               // weight rows per tile
constexpr int kGvTileBytes = kGvTile * kGvSlice / 2;      // 2 KB of packed codes
constexpr int kGvStages = 4;                              // per-warp ring of code tiles
constexpr int kGvLutBytes = 256 * 256;                    // 256 rows of 256 B on a 64 KB boundary
constexpr int kGvMaxTok = 16;

template <int NT>
struct GvCfg {
  static constexpr int WARPS = NT == 8 ? 16 : 12;         // K slices per CTA (register budget)
  static constexpr int THREADS = 32 * WARPS;
  static constexpr int GROUP = WARPS * kGvSlice;          // K columns per group
  static constexpr int SLOTS = WARPS * kGvStages;
  static constexpr int CHUNKS_PER_WARP = NT / 2;          // 128-byte pieces of one warp's partial tile
  static constexpr int RED_ITEMS = 256 / (WARPS * CHUNKS_PER_WARP);   // items per reduction round
  // the table's 64 KB, the stages (2 KB slots below and above the table; less
  // than one slot of the gap below it stays unused) and the barriers, plus
  // alignment slack
  static constexpr int SMEM = kGvLutBytes + SLOTS * kGvTileBytes + 4096;
  static_assert(RED_ITEMS >= 1, "reduction round");
};

struct GemvArgs {
  const int8_t* q8;
  const float* step2;
  const float* mean;
  const uint16_t* x;       // [M, in] bf16
  const uint16_t* us;      // [M, r] bf16, s x A^T (written before this kernel)
  const uint16_t* B;       // [out, r] bf16
  uint16_t* h;             // [M, out] bf16
  float* part;             // [groups, out, M] fp32 group partials (groups > 1)
  int M, in, out, r;
  int n_slices;            // ceil(in / 256)
  int groups;              // ceil(n_slices / WARPS)
  int tiles;               // out / 16
  int64_t n_items;         // groups * tiles
  uint64_t timeout_ns;
  Levels L;
};

// Work of the items before item i (group-major; every group but the last has
// WARPS slices), and the first item whose preceding work reaches w.
__device__ __forceinline__ int64_t gv_work_before(int64_t i, int64_t tiles, int warps, int last_slices,
                                                  int groups) {
  const int64_t full = static_cast<int64_t>(groups - 1) * tiles;
  return i <= full ? i * warps : full * warps + (i - full) * last_slices;
}
__device__ __forceinline__ int64_t gv_item_at(int64_t w, int64_t tiles, int warps, int last_slices, int groups) {
  const int64_t full = static_cast<int64_t>(groups - 1) * tiles;
  const int64_t wf = full * warps;
  if (w <= wf) return (w + warps - 1) / warps;
  return full + (w - wf + last_slices - 1) / last_slices;
}

__device__ __forceinline__ void gv_mma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Table lookups: not volatile, so the compiler may interleave them with the
// MMAs; every table address derives from a value loaded after the barrier
// that publishes the table.
__device__ __forceinline__ uint32_t gv_lds(uint32_t addr) {
  uint32_t v;
  asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

// Stage reads: volatile, so they stay after the pipeline wait.
__device__ __forceinline__ uint2 gv_lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr) : "memory");
  return v;
}

// Bounded wait on the mbarrier at shared address `bar` for the phase of the
// given parity; false on timeout.
__device__ __forceinline__ bool gv_wait(uint32_t bar, uint32_t parity, uint64_t timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 > timeout_ns) return false;
  }
}

__device__ __forceinline__ uint4 gv_ldg128(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// Sum over j < r of us[m][j] * B[o][j] (bf16 inputs, fp32 FMAs in j order).
__device__ __forceinline__ float gv_lora(const uint16_t* __restrict__ us, const uint16_t* __restrict__ B, int m,
                                         int o, int r) {
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
  return l;
}

// kRegSteps: of the four MMA steps of a block, how many decode the rows g + 8
// with the register table (ALU) instead of the shared table (load/store unit).
template <int NT, int kRegSteps>
__global__ void __launch_bounds__(GvCfg<NT>::THREADS, 1)
    nf4_gemv_kernel(const __grid_constant__ CUtensorMap tm_codes, const GemvArgs a) {
  using C = GvCfg<NT>;
  constexpr int W = C::WARPS;
  constexpr int kTok2 = NT == 16;                          // a second 8-token MMA tile
  extern __shared__ __align__(1024) uint8_t s_raw[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, q = lane & 3;

  // ---- work range of this CTA (split by work: slices x tiles)
  const int last_slices = a.n_slices - (a.groups - 1) * W;
  const int64_t total = gv_work_before(a.n_items, a.tiles, W, last_slices, a.groups);
  const int64_t i_begin = gv_item_at(total * blockIdx.x / gridDim.x, a.tiles, W, last_slices, a.groups);
  const int64_t i_end = gv_item_at(total * (blockIdx.x + 1) / gridDim.x, a.tiles, W, last_slices, a.groups);
  if (i_begin >= i_end) return;                                      // CTA-uniform
  const int n_local = static_cast<int>(i_end - i_begin);

  // ---- shared-memory layout: the table on the first 64 KB boundary of the
  // window, code stages in 2 KB slots below and above it, barriers last
  const uint32_t raw = smem_u32(s_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t lut = (base + 0xFFFFu) & ~0xFFFFu;
  const int below = static_cast<int>((lut - base) / kGvTileBytes);  // slots that fit under the table
  auto slot_addr = [&](int k) -> uint32_t {
    return k < below ? base + k * kGvTileBytes : lut + kGvLutBytes + (k - below) * kGvTileBytes;
  };
  const uint32_t bar_base = slot_addr(C::SLOTS);
  const uint32_t end = max(bar_base + C::SLOTS * 8, lut + kGvLutBytes);
  if (end > raw + C::SMEM || lut >= (1u << 24)) {                    // cannot place them (CTA-uniform)
    if (threadIdx.x == 0) raise_device_error(3);
    return;
  }
  auto full_bar = [&](int s) -> uint32_t { return bar_base + (warp * kGvStages + s) * 8; };

  if (lane == 0) {
    for (int s = 0; s < kGvStages; ++s)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" :: "r"(full_bar(s)) : "memory");
    fence_mbar_init();
  }
  // level-pair table: row b (a code byte) holds bf16(level[b & 15]) | bf16(level[b >> 4]) << 16, one copy per lane
  for (int e = threadIdx.x; e < 256 * 32; e += C::THREADS) {
    const int b = e >> 5, l = e & 31;
    const uint32_t v = pack_bf16x2_rn(a.L.v[b & 15], a.L.v[b >> 4]);
    asm volatile("st.shared.u32 [%0], %1;" :: "r"(lut + b * 256 + l * 4), "r"(v) : "memory");
  }
  __syncthreads();

  // register table of the rows g + 8: bf16(level[j] * 1)
  const Nf4Table rt = make_table(a.L, 1.0f);
  uint32_t lane_key;                                                 // bytes 0 and 2 of every table address
  asm volatile("mov.b32 %0, %1;" : "=r"(lane_key) : "r"(lut | static_cast<uint32_t>(lane * 4)) : "memory");

  const int row_blocks = a.in / 64;
  const float mu = __ldg(a.mean);

  // (group, tile) of an item, advanced item by item (no division in the loop)
  struct ItemPos { int grp, tile; };
  const ItemPos first{static_cast<int>(i_begin / a.tiles), static_cast<int>(i_begin % a.tiles)};
  auto advance = [&](ItemPos p) -> ItemPos {
    if (++p.tile == a.tiles) { p.tile = 0; ++p.grp; }
    return p;
  };
  auto active_in = [&](int grp) { return grp * W + warp < a.n_slices; };

  // ---- TMA issue of item `it` (at position p) into stage it % kGvStages (lane 0)
  auto issue = [&](int it, ItemPos p) -> bool {
    if (it >= n_local || !active_in(p.grp)) return false;
    const int s = it % kGvStages;
    const uint32_t dst = slot_addr(warp * kGvStages + s);
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 :: "r"(full_bar(s)), "r"(kGvTileBytes) : "memory");
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        :: "r"(dst), "l"(&tm_codes), "r"((p.grp * W + warp) * (kGvSlice / 2)), "r"(p.tile * kGvTile),
           "r"(full_bar(s)) : "memory");
    return true;
  };
  // lane 0: the next item to issue, its position, and how many loads were
  // issued (the warp's active items are a prefix of the CTA's range)
  int next_issue = 0, n_issued = 0;
  ItemPos issue_pos = first;
  if (lane == 0) {
    asm volatile("prefetch.tensormap [%0];" :: "l"(&tm_codes) : "memory");
    for (; next_issue < kGvStages; ++next_issue) {
      n_issued += issue(next_issue, issue_pos) ? 1 : 0;
      issue_pos = advance(issue_pos);
    }
  }

  // stage-relative read offsets (128-byte swizzle): codes of row g (row g+8: + 1024)
  // for block j: 8 bytes at byte 32 j + 8 q of the row's 128
  uint32_t coff[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int c = 2 * j + (q >> 1);
    coff[j] = static_cast<uint32_t>(g * 128 + (((c ^ g) & 7) << 4) + (q & 1) * 8);
  }

  // activations of this warp's slice (per block j: 16 consecutive columns
  // 64 j + 16 q .. +15 of tokens g and g + 8), loaded when the group changes
  uint32_t xa[4][8], xc[4][8];
  int cur_grp = -1;
  auto load_x = [&](int grp) {
    const int c0 = (grp * W + warp) * kGvSlice;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int col = c0 + 64 * j + 16 * q;
      const bool cok = col < a.in;
#pragma unroll
      for (int t2 = 0; t2 < (kTok2 ? 2 : 1); ++t2) {
        const int tok = g + 8 * t2;
        uint4 v0 = make_uint4(0, 0, 0, 0), v1 = v0;
        if (cok && tok < a.M) {
          const uint16_t* p = a.x + static_cast<int64_t>(tok) * a.in + col;
          v0 = gv_ldg128(p);
          v1 = gv_ldg128(p + 8);
        }
        if (t2 == 0) {
          xa[j][0] = v0.x; xa[j][1] = v0.y; xa[j][2] = v0.z; xa[j][3] = v0.w;
          xa[j][4] = v1.x; xa[j][5] = v1.y; xa[j][6] = v1.z; xa[j][7] = v1.w;
        } else {
          xc[j][0] = v0.x; xc[j][1] = v0.y; xc[j][2] = v0.z; xc[j][3] = v0.w;
          xc[j][4] = v1.x; xc[j][5] = v1.y; xc[j][6] = v1.z; xc[j][7] = v1.w;
        }
      }
    }
  };

  // scale codes of this quad lane's block in rows g and g + 8 of an item's
  // tile (code 0 and step 0 past the K end), fetched one item ahead
  struct ScaleIn { int q0, q1; float st0, st1; };
  auto fetch_scales = [&](int it, ItemPos p, ScaleIn& f) {
    f.q0 = f.q1 = 0;
    f.st0 = f.st1 = 0.f;
    if (it >= n_local) return;
    const int blk = (p.grp * W + warp) * 4 + q;
    if (blk >= row_blocks) return;
    const int64_t b0 = static_cast<int64_t>(p.tile * kGvTile + g) * row_blocks + blk;
    const int64_t b1 = b0 + 8ll * row_blocks;
    f.q0 = __ldg(a.q8 + b0);
    f.q1 = __ldg(a.q8 + b1);
    f.st0 = __ldg(a.step2 + (b0 >> 8));
    f.st1 = __ldg(a.step2 + (b1 >> 8));
  };
  ScaleIn nxt;
  fetch_scales(0, first, nxt);

  const uint32_t red_base = lut + 128;                               // upper half of every table row
  bool ok_all = true;
  int stuck = n_local;                                               // first item not consumed
  ItemPos pos = first;
  ItemPos round_first = first;                                       // position of the round's first item
  for (int it = 0; it < n_local; ++it, pos = advance(pos)) {
    const int grp = pos.grp;
    const bool act = active_in(grp);
    if (it % C::RED_ITEMS == 0) round_first = pos;
    float d[2][4];
#pragma unroll
    for (int t2 = 0; t2 < 2; ++t2) d[t2][0] = d[t2][1] = d[t2][2] = d[t2][3] = 0.f;
    if (act && ok_all) {
      if (grp != cur_grp) {
        load_x(grp);
        cur_grp = grp;
      }
      // this lane's two block scales (exchanged with its quad below); the
      // next item's codes are fetched now
      const ScaleIn cur = nxt;
      fetch_scales(it + 1, advance(pos), nxt);
      const float s0 = block_scale(cur.q0, cur.st0, mu);
      const float s1 = block_scale(cur.q1, cur.st1, mu);
      const int s = it % kGvStages;
      const bool landed = gv_wait(full_bar(s), static_cast<uint32_t>((it / kGvStages) & 1), a.timeout_ns);
      if (!__all_sync(0xFFFFFFFFu, landed)) {                        // warp-uniform give-up
        if (lane == 0) raise_device_error(1);
        ok_all = false;
        stuck = it;
      } else {
        const uint32_t sb = slot_addr(warp * kGvStages + s);
        uint2 cg[4], ch[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          cg[j] = gv_lds64(sb + coff[j]);
          ch[j] = gv_lds64(sb + coff[j] + 1024);
        }
        // the stage is read: hand it back to the copy engine for item it + kGvStages
        __syncwarp();
        if (lane == 0) {
          fence_proxy_async_smem();
          n_issued += issue(next_issue, issue_pos) ? 1 : 0;          // item it + kGvStages
          ++next_issue;
          issue_pos = advance(issue_pos);
        }
        float sc0[4], sc1[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          sc0[j] = __shfl_sync(0xFFFFFFFFu, s0, (lane & ~3) | j);
          sc1[j] = __shfl_sync(0xFFFFFFFFu, s1, (lane & ~3) | j);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float pb[2][4];
#pragma unroll
          for (int st = 0; st < 4; ++st) {
            const uint32_t wg = st < 2 ? cg[j].x : cg[j].y;
            const uint32_t wh = st < 2 ? ch[j].x : ch[j].y;
            const int bi = (2 * st) & 3;                             // byte of the column pair 4 st, 4 st + 1
            const uint32_t a0 = gv_lds(prmt(wg, lane_key, 0x7604u | (bi << 4)));
            const uint32_t a2 = gv_lds(prmt(wg, lane_key, 0x7604u | ((bi + 1) << 4)));
            uint32_t a1, a3;
            if (st < kRegSteps) {
              decode4(rt, wh >> (8 * bi), a1, a3);                   // ALU: register table
            } else {
              a1 = gv_lds(prmt(wh, lane_key, 0x7604u | (bi << 4)));  // load/store unit: shared table
              a3 = gv_lds(prmt(wh, lane_key, 0x7604u | ((bi + 1) << 4)));
            }
            if (st == 0) {
              pb[0][0] = pb[0][1] = pb[0][2] = pb[0][3] = 0.f;
              pb[1][0] = pb[1][1] = pb[1][2] = pb[1][3] = 0.f;
            }
            gv_mma(pb[0], a0, a1, a2, a3, xa[j][2 * st], xa[j][2 * st + 1]);
            if (kTok2) gv_mma(pb[1], a0, a1, a2, a3, xc[j][2 * st], xc[j][2 * st + 1]);
          }
#pragma unroll
          for (int t2 = 0; t2 < (kTok2 ? 2 : 1); ++t2) {
            d[t2][0] = fmaf(pb[t2][0], sc0[j], d[t2][0]);
            d[t2][1] = fmaf(pb[t2][1], sc0[j], d[t2][1]);
            d[t2][2] = fmaf(pb[t2][2], sc1[j], d[t2][2]);
            d[t2][3] = fmaf(pb[t2][3], sc1[j], d[t2][3]);
          }
        }
      }
    }
    // ---- this warp's partial tile into its reduction piece: value (row, tok)
    // at byte 4 (row NT + tok) of the warp's NT/2 chunks of 128 B
    const int k = it % C::RED_ITEMS;
    {
      const int chunk0 = (k * W + warp) * C::CHUNKS_PER_WARP;
#pragma unroll
      for (int t2 = 0; t2 < (kTok2 ? 2 : 1); ++t2) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int off = ((g + 8 * hh) * NT + 8 * t2 + 2 * q) * 4;
          const uint32_t addr = red_base + (chunk0 + (off >> 7)) * 256 + (off & 127);
          asm volatile("st.shared.v2.f32 [%0], {%1, %2};" :: "r"(addr), "f"(d[t2][2 * hh]), "f"(d[t2][2 * hh + 1])
                       : "memory");
        }
      }
    }
    if (k != C::RED_ITEMS - 1 && it != n_local - 1) continue;

    // ---- reduction round over items it0 .. it (CTA-uniform)
    __syncthreads();
    const int n_round = k + 1;
    for (int u = threadIdx.x; u < n_round * kGvTile * NT; u += C::THREADS) {
      const int kk = u / (kGvTile * NT), v = u % (kGvTile * NT);
      const int row = v / NT, tok = v % NT;
      float sum = 0.f;
#pragma unroll 4
      for (int w = 0; w < W; ++w) {
        const int off = v * 4;
        float t;
        asm volatile("ld.shared.f32 %0, [%1];" : "=f"(t)
                     : "r"(red_base + ((kk * W + w) * C::CHUNKS_PER_WARP + (off >> 7)) * 256 + (off & 127))
                     : "memory");
        sum += t;
      }
      if (tok < a.M) {
        ItemPos ip = round_first;
        for (int j = 0; j < kk; ++j) ip = advance(ip);
        const int gi = ip.grp, ti = ip.tile;
        const int o = ti * kGvTile + row;
        if (a.groups == 1)
          a.h[static_cast<int64_t>(tok) * a.out + o] =
              __bfloat16_as_ushort(__float2bfloat16_rn(sum + gv_lora(a.us, a.B, tok, o, a.r)));
        else
          a.part[(static_cast<int64_t>(gi) * a.out + o) * a.M + tok] = sum;
      }
    }
    __syncthreads();                                                 // the pieces are reused
  }

  // leave no copy in flight when the CTA exits: after a give-up at item
  // `stuck`, the stages of items stuck .. stuck + kGvStages - 1 may have been
  // issued and not consumed; wait for them, bounded
  if (lane == 0 && stuck < n_local) {
    for (int it = stuck; it < n_issued; ++it)                        // the issued loads are items 0 .. n_issued - 1
      gv_wait(full_bar(it % kGvStages), static_cast<uint32_t>((it / kGvStages) & 1), a.timeout_ns);
  }
}

// h[m][o] = bf16( sum over the K groups, in group order, of part[g][o][m]
//                 + sum_j us[m][j] * B[o][j] ),  m < M (K split over groups).
__global__ void __launch_bounds__(256) gemv_finalize_kernel(const float* __restrict__ part, int groups, int M,
                                                            int out, const uint16_t* __restrict__ us,
                                                            const uint16_t* __restrict__ B, int r,
                                                            uint16_t* __restrict__ h) {
  const int64_t n_el = static_cast<int64_t>(M) * out;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n_el;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int o = static_cast<int>(e / M), m = static_cast<int>(e % M);
    float v = 0.f;
    for (int gg = 0; gg < groups; ++gg) v += __ldg(part + static_cast<int64_t>(gg) * n_el + e);
    h[static_cast<int64_t>(m) * out + o] = __bfloat16_as_ushort(__float2bfloat16_rn(v + gv_lora(us, B, m, o, r)));
  }
}

}  // namespace qnf4
