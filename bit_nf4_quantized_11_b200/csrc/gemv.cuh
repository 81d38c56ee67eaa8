// gemv.cuh -- few-token (M <= 16) QLoRA forward: streaming NF4 GEMV.
//
// With 1..16 tokens the layer is bound by streaming the packed weight from
// HBM (0.52 byte per weight), so the kernel is organised around that stream
// and around the issue and load/store-unit budget per weight it leaves.  The
// work is (row tile of 256 weight rows) x (unit of 256 K columns = four
// 64-weight blocks) units, ordered tile-major; a persistent grid of one CTA
// per SM splits the unit sequence evenly, so every CTA streams the same
// number of bytes whatever the shape.
//
// Per unit, one thread issues two TMA loads into a ring of shared-memory
// stages: the 256 x 128-byte code tile and the 8- (or 16-) token x 256-column
// activation tile, both with 128-byte swizzle so that the reads below are
// bank-conflict free.  16 warps own 16 rows each (the 16-row operand of a
// warp-level bf16 MMA); per unit a thread reads, for rows g and g+8, 16
// consecutive codes of each of the four blocks, and its warp releases the
// code part of the stage as soon as they are in registers.  Second-level
// scale codes (four per row and unit) and group steps are fetched two units
// ahead (one unit ahead, with cached steps, in the 16-token kernel).
//
// Each MMA step covers 16 columns of ONE block for all four quad lanes: step
// s of block j takes columns 64j + 16q + 4s .. +3 for quad lane q, in the
// same permuted K order for weights and activations.  A block's four steps
// accumulate into a fresh fp32 tile that is then added to the running sum
// times the block's exact fp32 scale c_hat (rows g and g+8 each with their
// own), so the MMA's weight operand is bf16(level) -- the exactly rounded
// level -- and the scale costs nothing per weight.  (The GEMM path instead
// rounds bf16(level * c_hat) per weight; the two differ by at most 2^-9
// relative per weight, far inside the output tolerance.)
//
// Decoding is one byte permute and one shared load per nibble pair: the
// 256-entry table of bf16 level pairs has one 256-byte row per byte value,
// with one 4-byte copy per lane in its first 128 bytes (so lookups never
// conflict), and sits on a 64 KB boundary of the shared window, so that a
// single prmt assembles (window bits 16-17 | byte << 8 | lane * 4), the
// complete shared address.  Where a CTA's range starts or ends inside a tile
// it writes an fp32 partial of that tile; the finalize kernel adds a tile's
// partials in CTA order and the LoRA branch us . B^T ("QLoRA", llm-compass,
// 方法与公式: h = dequant(W0) x + (alpha/r) B A x).
#pragma once

#include "common.cuh"

namespace qnf4 {

constexpr int kGvWarps = 16;
constexpr int kGvThreads = 32 * kGvWarps;
constexpr int kGvRows = 16 * kGvWarps;                    // weight rows per tile (256)
constexpr int kGvStageK = 256;                            // K columns per unit (four blocks)
constexpr int kGvStages = 3;                              // ring of unit tiles (2 in flight)
constexpr int kGvCodeBytes = kGvRows * kGvStageK / 2;     // 32 KB
constexpr int kGvXBox = 64;                               // activation box: 64 columns x tokens
constexpr int kGvStageBytes = kGvCodeBytes + 16 * kGvStageK * 2;   // + up to 16 tokens x 256 columns
constexpr int kGvLutBytes = 256 * 256;                    // 256 rows of 256 bytes
constexpr int kGvSmem = 192 * 1024;                       // stages, then the table on the next 64 KB boundary

struct GemvArgs {
  const int8_t* q8;
  const float* step2;
  const float* mean;
  float* part;             // [ctas][local_tiles][M][kGvRows]
  int M, in, out;
  int n_st;                // units per tile = ceil(in / 256)
  int64_t n_units;         // tiles * n_st
  int local_tiles;         // partial tiles reserved per CTA
  uint64_t timeout_ns;     // bound of every pipeline wait
  Levels L;
};

// First unit of CTA c when n units are split over p CTAs.
__host__ __device__ __forceinline__ int64_t gemv_unit_begin(int64_t c, int64_t n, int64_t p) {
  return c * n / p;
}

// Register-only MMAs and table loads without `volatile`, so that the
// compiler may interleave the lookups of one step with the MMA of the
// previous one.  Every table address derives from a value produced after the
// barrier that publishes the table (a volatile move).
__device__ __forceinline__ void gv_mma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// d = A B with a zero accumulator input.
__device__ __forceinline__ void gv_mma_z(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%10, %10, %10, %10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.f));
}

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

__device__ __forceinline__ uint4 gv_lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr) : "memory");
  return v;
}

// Byte offset, in a tile of 128-byte rows written with 128-byte swizzle, of
// the 16-byte chunk c of row `row` (chunk index XOR row % 8) plus `half` * 8.
__device__ __forceinline__ uint32_t gv_swz128(int row, int c, int half) {
  return static_cast<uint32_t>(row * 128 + (((c ^ row) & 7) << 4) + half * 8);
}

// kPaired: in % 256 == 0, so every unit holds four whole blocks whose index
// run starts at a multiple of 4 (one aligned 32-bit load of their q8 codes,
// one group step for all four).  kTwoTok: 9..16 tokens, a second 8-token MMA
// tile.
template <bool kPaired, bool kTwoTok>
__global__ void __launch_bounds__(kGvThreads, 1)
    nf4_gemv_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_x,
                    const GemvArgs a) {
  constexpr int XR = kTwoTok ? 16 : 8;                               // token rows of the activation box
  constexpr uint32_t kTxBytes = kGvCodeBytes + 4 * kGvXBox * 2 * XR;
  extern __shared__ __align__(1024) uint8_t s_raw[];
  __shared__ __align__(8) uint64_t full_bar[kGvStages], empty_bar[kGvStages];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t u_begin = gemv_unit_begin(blockIdx.x, a.n_units, gridDim.x);
  const int64_t u_end = gemv_unit_begin(blockIdx.x + 1, a.n_units, gridDim.x);
  if (u_begin >= u_end) return;                                     // CTA-uniform
  const int n_local = static_cast<int>(u_end - u_begin);
  const int t_first = static_cast<int>(u_begin / a.n_st);
  const int st_first = static_cast<int>(u_begin - static_cast<int64_t>(t_first) * a.n_st);

  // contiguous 1024-aligned stages at the start of s_raw, the table on the
  // next 64 KB boundary of the window after them
  const uint32_t raw = smem_u32(s_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  const uint32_t lut = (sbase + kGvStages * kGvStageBytes + 0xFFFFu) & ~0xFFFFu;
  if (lut + kGvLutBytes > raw + kGvSmem || lut >= (1u << 24)) {     // cannot place them (CTA-uniform)
    if (threadIdx.x == 0) raise_device_error(3);
    return;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kGvStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kGvWarps);
    }
    fence_mbar_init();
  }
  for (int e = threadIdx.x; e < 256 * 32; e += kGvThreads) {
    const int b = e >> 5, l = e & 31;
    const uint32_t v = pack_bf16x2_rn(a.L.v[b & 15], a.L.v[b >> 4]);
    asm volatile("st.shared.u32 [%0], %1;" :: "r"(lut + b * 256 + l * 4), "r"(v) : "memory");
  }
  __syncthreads();

  // Unit tiles: thread 0 issues unit i's loads into stage i % kGvStages once
  // every warp has released the unit that used that stage before.
  const bool producer = threadIdx.x == 0;
  int p_issued = 0, p_st = st_first, p_t = t_first;
  bool p_ok = true;
  auto produce_until = [&](int limit) {                            // issue loads of units < limit
    for (; p_ok && p_issued < limit && p_issued < n_local; ++p_issued) {
      const int s = p_issued % kGvStages;
      if (p_issued >= kGvStages &&
          !mbar_wait_bounded(&empty_bar[s], ((p_issued / kGvStages) + 1) & 1, a.timeout_ns)) {
        raise_device_error(1);
        p_ok = false;
        break;
      }
      const uint32_t dst = sbase + s * kGvStageBytes;
      mbar_arrive_expect_tx(&full_bar[s], kTxBytes);
      tma_load_2d(dst, &tm_codes, &full_bar[s], p_st * (kGvStageK / 2), p_t * kGvRows);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        tma_load_2d(dst + kGvCodeBytes + j * (kGvXBox * 2 * XR), &tm_x, &full_bar[s],
                    p_st * kGvStageK + j * kGvXBox, 0);
      if (++p_st == a.n_st) { p_st = 0; ++p_t; }
    }
  };
  if (producer) {
    tma_prefetch_desc(&tm_codes);
    tma_prefetch_desc(&tm_x);
    produce_until(kGvStages - 1);
  }

  const int g = lane >> 2, q = lane & 3;
  uint32_t lane_key;                                                 // bytes 0 and 2 of every table address
  asm volatile("mov.b32 %0, %1;" : "=r"(lane_key) : "r"(lut | static_cast<uint32_t>(lane * 4)) : "memory");
  const int row_in_tile0 = warp * 16 + g;
  const bool tok0 = g < a.M, tok1 = kTwoTok && g + 8 < a.M;
  // stage-relative read offsets: codes of row g, block j (row g+8: + 1024);
  // activation chunks 2q, 2q+1 of token g (token g+8: + 1024)
  uint32_t coff[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) coff[j] = gv_swz128(row_in_tile0, 2 * j + (q >> 1), q & 1);
  const uint32_t xoff0 = kGvCodeBytes + gv_swz128(g, 2 * q, 0);
  const uint32_t xoff1 = kGvCodeBytes + gv_swz128(g, 2 * q + 1, 0);
  constexpr uint32_t kXBlk = kGvXBox * 2 * XR;                       // bytes per activation box

  const int64_t row_blocks = a.in / 64;
  const float mu = __ldg(a.mean);

  // Block scales are computed once per (row, block) and shared through the
  // free upper half of the table's rows: lane l of a warp handles row
  // (l % 16) of the warp's 16 and blocks 2 (l / 16), 2 (l / 16) + 1 of the
  // unit, writes them to its warp's 256-byte slot (rows 0-7 in table row
  // 2 warp, rows 8-15 in 2 warp + 1, 16 bytes per row) and reads back the
  // four scales of rows g and g+8.
  const int srow = lane & 15, spair = lane >> 4;
  const uint32_t s_st = lut + (2 * warp + (srow >> 3)) * 256 + 128 + (srow & 7) * 16 + spair * 8;
  const uint32_t s_ld = lut + 2 * warp * 256 + 128 + g * 16;         // row g; row g+8: + 256
  int rs = t_first * kGvRows + warp * 16 + srow;                    // this lane's scale row
  const int8_t* qp = a.q8 + static_cast<int64_t>(rs) * row_blocks + 4 * st_first + 2 * spair;
  const int64_t b_wrap = kGvRows * row_blocks - 4 * static_cast<int64_t>(a.n_st);
  // Paired, 9..16 tokens: the two q8 codes of the next unit (each byte XOR
  // 0x80) and a cached group step.  Paired, 1..8 tokens: the q8 codes and
  // group steps of units i + 1 and i + 2, read by a cursor that walks this
  // lane's (row, block pair) sequence two units ahead, so that no scale
  // waits on a load issued one unit earlier while the stream holds HBM busy
  // (the two-token kernel has no registers to spare for it).
  constexpr bool kAhead = kPaired && !kTwoTok;
  uint32_t qn = 0x8080u;
  float sv = 0.f;
  if (kPaired && !kAhead && rs < a.out)
    qn = static_cast<uint32_t>(__ldg(reinterpret_cast<const uint16_t*>(qp))) ^ 0x8080u;
  uint32_t qa = 0x8080u, qb = 0x8080u;
  float sa = 0.f, sb2 = 0.f;
  const int8_t* qpf = qp;
  int rpf = rs, spf = st_first;
  auto pf_load = [&](uint32_t& qd, float& sd) {
    if (rpf < a.out) {
      qd = static_cast<uint32_t>(__ldg(reinterpret_cast<const uint16_t*>(qpf))) ^ 0x8080u;
      sd = __ldg(a.step2 + (((qpf - a.q8) - 2 * spair) >> 8));
    }
    qpf += 4;
    if (++spf == a.n_st) { spf = 0; rpf += kGvRows; qpf += b_wrap; }
  };
  if (kAhead) {
    pf_load(qa, sa);
    if (n_local > 1) pf_load(qb, sb2);
  }

  float acc[2][4];
#pragma unroll
  for (int j = 0; j < 2; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;

  int t = t_first, st = st_first;
  int s = 0;
  uint32_t phase = 0, sb = sbase;
  bool new_row = true;                                               // group steps to (re)load
  for (int i = 0; i < n_local; ++i) {
    const bool ok = mbar_wait_bounded(&full_bar[s], phase, a.timeout_ns);
    if (!__all_sync(0xFFFFFFFFu, ok)) {                              // warp-uniform give-up
      if (lane == 0) raise_device_error(1);
      break;
    }
    uint2 cg[4], ch[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      cg[j] = gv_lds64(sb + coff[j]);
      ch[j] = gv_lds64(sb + coff[j] + 1024);
    }

    const int col0 = st * kGvStageK;
    const bool last_in_tile = st == a.n_st - 1;

    // this lane's two block scales, then the eight of rows g and g+8
    {
      const bool row_ok = rs < a.out;
      float s0, s1;
      if (kPaired) {
        uint32_t qc;
        float svc;
        if constexpr (kAhead) {
          qc = qa;
          svc = sa;
          qa = qb;
          sa = sb2;
          if (i + 2 < n_local) pf_load(qb, sb2);
        } else {
          qc = qn;
          const int8_t* q_next = last_in_tile ? qp + b_wrap + 4 : qp + 4;
          const bool next_ok = last_in_tile ? rs + kGvRows < a.out : row_ok;
          if (next_ok && i + 1 < n_local)
            qn = static_cast<uint32_t>(__ldg(reinterpret_cast<const uint16_t*>(q_next))) ^ 0x8080u;
          // a unit's four blocks share one group; a group starts at a multiple of 256 blocks
          const int64_t b_unit = (qp - a.q8) - 2 * spair;
          if (row_ok && (new_row || (static_cast<uint32_t>(b_unit) & 255u) == 0)) sv = __ldg(a.step2 + (b_unit >> 8));
          svc = sv;
        }
        // exact floats of the signed codes: 2^23 + (q + 128) - (2^23 + 128)
        const float q0 = __fadd_rn(__uint_as_float(prmt(qc, 0x4B000000u, 0x7650u)), -8388736.0f);
        const float q1 = __fadd_rn(__uint_as_float(prmt(qc, 0x4B000000u, 0x7651u)), -8388736.0f);
        s0 = __fadd_rn(__fmul_rn(q0, svc), mu);
        s1 = __fadd_rn(__fmul_rn(q1, svc), mu);
      } else {
        const int c0 = col0 + 128 * spair;
        const bool l0 = row_ok && c0 < a.in, l1 = row_ok && c0 + 64 < a.in;
        const int64_t b = qp - a.q8;
        s0 = block_scale(l0 ? __ldg(qp) : 0, l0 ? __ldg(a.step2 + (b >> 8)) : 0.f, mu);
        s1 = block_scale(l1 ? __ldg(qp + 1) : 0, l1 ? __ldg(a.step2 + ((b + 1) >> 8)) : 0.f, mu);
      }
      asm volatile("st.shared.v2.f32 [%0], {%1, %2};" :: "r"(s_st), "f"(s0), "f"(s1) : "memory");
    }
    __syncwarp();
    float sc[2][4];
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(sc[0][0]), "=f"(sc[0][1]), "=f"(sc[0][2]), "=f"(sc[0][3]) : "r"(s_ld) : "memory");
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(sc[1][0]), "=f"(sc[1][1]), "=f"(sc[1][2]), "=f"(sc[1][3]) : "r"(s_ld + 256) : "memory");
    new_row = false;

#pragma unroll
    for (int blk = 0; blk < 4; ++blk) {
      if (kPaired || blk == 0 || col0 + 64 * blk < a.in) {
        // activations: 16 consecutive columns 64 blk + 16q .. +15 of token rows g, g+8
        uint4 xa0 = make_uint4(0, 0, 0, 0), xa1 = xa0, xc0 = xa0, xc1 = xa0;
        if (tok0) {
          xa0 = gv_lds128(sb + xoff0 + blk * kXBlk);
          xa1 = gv_lds128(sb + xoff1 + blk * kXBlk);
        }
        if (tok1) {
          xc0 = gv_lds128(sb + xoff0 + blk * kXBlk + 1024);
          xc1 = gv_lds128(sb + xoff1 + blk * kXBlk + 1024);
        }
        const uint32_t xa[8] = {xa0.x, xa0.y, xa0.z, xa0.w, xa1.x, xa1.y, xa1.z, xa1.w};
        const uint32_t xc[8] = {xc0.x, xc0.y, xc0.z, xc0.w, xc1.x, xc1.y, xc1.z, xc1.w};
        const uint32_t wg[2] = {cg[blk].x, cg[blk].y}, wh[2] = {ch[blk].x, ch[blk].y};
        float pb[2][4];
#pragma unroll
        for (int s4 = 0; s4 < 4; ++s4) {     // columns 64 blk + 16q + 4 s4 .. +3: bytes 2 s4, 2 s4 + 1
          const uint32_t sel_lo = 0x7604u | ((2 * (s4 & 1)) << 4);
          const uint32_t sel_hi = 0x7604u | ((2 * (s4 & 1) + 1) << 4);
          const uint32_t e0 = gv_lds(prmt(wg[s4 >> 1], lane_key, sel_lo));
          const uint32_t e1 = gv_lds(prmt(wh[s4 >> 1], lane_key, sel_lo));
          const uint32_t e2 = gv_lds(prmt(wg[s4 >> 1], lane_key, sel_hi));
          const uint32_t e3 = gv_lds(prmt(wh[s4 >> 1], lane_key, sel_hi));
          // a0: row g columns +0,+1; a1: row g+8 same; a2, a3: columns +2,+3
          if (s4 == 0) {
            gv_mma_z(pb[0], e0, e1, e2, e3, xa[0], xa[1]);
            if (kTwoTok) gv_mma_z(pb[1], e0, e1, e2, e3, xc[0], xc[1]);
          } else {
            gv_mma(pb[0], e0, e1, e2, e3, xa[2 * s4], xa[2 * s4 + 1]);
            if (kTwoTok) gv_mma(pb[1], e0, e1, e2, e3, xc[2 * s4], xc[2 * s4 + 1]);
          }
        }
#pragma unroll
        for (int j = 0; j < (kTwoTok ? 2 : 1); ++j) {
          acc[j][0] = fmaf(pb[j][0], sc[0][blk], acc[j][0]);
          acc[j][1] = fmaf(pb[j][1], sc[0][blk], acc[j][1]);
          acc[j][2] = fmaf(pb[j][2], sc[1][blk], acc[j][2]);
          acc[j][3] = fmaf(pb[j][3], sc[1][blk], acc[j][3]);
        }
      }
    }
    // the stage (codes and activations) is no longer read by this warp
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[s]);
    if (producer) produce_until(i + kGvStages);                     // refill the stage of unit i - 1

    // end of this CTA's part of tile t: write the partial and restart
    if (last_in_tile || i == n_local - 1) {
      float* dst = a.part + ((static_cast<int64_t>(blockIdx.x) * a.local_tiles + (t - t_first)) * a.M) * kGvRows;
#pragma unroll
      for (int j = 0; j < (kTwoTok ? 2 : 1); ++j) {
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
    qp += 4;
    if (++st == a.n_st) { st = 0; ++t; rs += kGvRows; qp += b_wrap; new_row = true; }
    sb += kGvStageBytes;
    if (++s == kGvStages) { s = 0; phase ^= 1u; sb = sbase; }
  }
  // leave no copy in flight when the CTA exits (only on a give-up path can
  // issued loads still be unconsumed): wait, bounded, for the last ones
  if (producer)
    for (int j = p_issued > kGvStages ? p_issued - kGvStages : 0; j < p_issued; ++j)
      if (!mbar_wait_bounded(&full_bar[j % kGvStages], (j / kGvStages) & 1, a.timeout_ns)) raise_device_error(1);
}

// h[m][o] = bf16( sum of the partials of o's tile, in CTA order
//                 + sum_j us[m][j] * B[o][j] ),  m < M.
// One CTA per (256-row tile, token), one thread per row.  Thread 0 lists the
// CTAs whose unit ranges touch the tile (with the tile's slot in each CTA's
// partials); longer lists than kGvFinMax are walked by every thread.
constexpr int kGvFinMax = 32;

__global__ void __launch_bounds__(kGvRows) gemv_finalize_kernel(
    const float* __restrict__ part, int ctas, int local_tiles, int64_t n_units, int n_st, int M, int out,
    const uint16_t* __restrict__ us, const uint16_t* __restrict__ B, int r, uint16_t* __restrict__ h) {
  __shared__ int s_c[kGvFinMax], s_lt[kGvFinMax];
  __shared__ int s_n, s_c0;
  const int t = blockIdx.x, m = blockIdx.y, row = threadIdx.x;
  const int o = t * kGvRows + row;
  const int64_t u = static_cast<int64_t>(t) * n_st;
  if (threadIdx.x == 0) {
    // unit ranges in 32-bit arithmetic when the products fit (the same floors)
    const bool small = static_cast<uint64_t>(n_units) * static_cast<uint64_t>(ctas) < (1ull << 32);
    auto begin = [&](int c) -> int64_t {
      return small ? static_cast<int64_t>(static_cast<uint32_t>(c) * static_cast<uint32_t>(n_units) /
                                          static_cast<uint32_t>(ctas))
                   : gemv_unit_begin(c, n_units, ctas);
    };
    // CTA holding the tile's first unit: the largest c with begin(c) <= t * n_st
    int c0 = static_cast<int>(u * ctas / n_units);
    while (c0 + 1 < ctas && begin(c0 + 1) <= u) ++c0;
    while (c0 > 0 && begin(c0) > u) --c0;
    int n = 0;
    int64_t b = begin(c0);
    for (int c = c0; c < ctas && b < u + n_st; ++c) {
      const int64_t b_next = begin(c + 1);
      if (b_next > b) {                                             // a CTA with units
        if (n < kGvFinMax) {
          s_c[n] = c;
          s_lt[n] = t - static_cast<int>(b / n_st);
        }
        ++n;
      }
      b = b_next;
    }
    s_n = n;
    s_c0 = c0;
  }
  __syncthreads();
  if (o >= out) return;
  float v = 0.f;
  const int n = s_n;
  if (n <= kGvFinMax) {
    for (int i = 0; i < n; ++i)
      v += __ldg(part + ((static_cast<int64_t>(s_c[i]) * local_tiles + s_lt[i]) * M + m) * kGvRows + row);
  } else {
    int64_t b = gemv_unit_begin(s_c0, n_units, ctas);
    for (int c = s_c0; c < ctas && b < u + n_st; ++c) {
      const int64_t b_next = gemv_unit_begin(c + 1, n_units, ctas);
      if (b_next > b)
        v += __ldg(part + ((static_cast<int64_t>(c) * local_tiles + (t - static_cast<int>(b / n_st))) * M + m) *
                              kGvRows + row);
      b = b_next;
    }
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
  h[static_cast<int64_t>(m) * out + o] = __bfloat16_as_ushort(__float2bfloat16_rn(v + l));
}

}  // namespace qnf4
