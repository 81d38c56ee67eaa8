// api.cu -- the C ABI of libqlora_nf4.so: argument validation, workspace
// layout, tensor-map encoding and kernel launches.  Declarations and the
// contract of every entry point are in include/qlora_nf4.h.
#include "qlora_nf4.h"

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "gemm_sm100.cuh"
#include "gemm_pair_sm100.cuh"
#include "gemv.cuh"
#include "merge.cuh"
#include "dropout.cuh"
#include "quant.cuh"
#include "lora_sm100.cuh"
#include "pad.cuh"
#include "fewtok.cuh"

namespace qnf4_host {
void build_codebook(float levels[16], float thresholds[15]);
void build_int4_codebook(float levels[16], float thresholds[15]);
}

namespace {

using qnf4::Levels;
using qnf4::Thresholds;

std::atomic<uint64_t> g_timeout_ns{2000000000ull};

struct Tables {
  Levels L;
  Thresholds T;
  qnf4::CodeTable C;
  bool ok;      // the cell table is valid for these thresholds
};

// Cell table of nearest_code: cell n covers 16 v in [n - 16.5, n - 15.5);
// below[n] = thresholds under the cell, inside[n] = the (at most one)
// threshold in it or +inf.  Returns false when a cell would hold two
// thresholds or a threshold sits on a cell edge (where the rounding of 16 v
// to the cell index could go either way).
bool build_code_table(const Thresholds& T, qnf4::CodeTable* c) {
  bool ok = true;
  for (int n = 0; n < qnf4::kCodeCells; ++n) {
    const double lo = (n - 16.5) / 16.0, hi = (n - 15.5) / 16.0;
    uint32_t below = 0;
    int n_inside = 0;
    float inside = INFINITY;
    for (int j = 0; j < 15; ++j) {
      const double t = T.v[j];
      if (t == lo) ok = false;
      if (t < lo) ++below;
      else if (t < hi) {
        inside = T.v[j];
        ++n_inside;
      }
    }
    if (n_inside > 1) ok = false;
    c->below[n] = below;
    c->inside[n] = inside;
  }
  return ok;
}

// Levels, thresholds and cell table of a codebook kind (QLORA_CODEBOOK_*).
const Tables* tables_for(int kind) {
  static Tables t[2];
  static std::once_flag once;
  std::call_once(once, [] {
    qnf4_host::build_codebook(t[0].L.v, t[0].T.v);
    t[0].ok = build_code_table(t[0].T, &t[0].C);
    qnf4_host::build_int4_codebook(t[1].L.v, t[1].T.v);
    t[1].ok = build_code_table(t[1].T, &t[1].C);
  });
  if (kind < 0 || kind > 1 || !t[kind].ok) return nullptr;
  return &t[kind];
}

const Tables& tables() { return *tables_for(QLORA_CODEBOOK_NF4); }

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
constexpr int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
constexpr size_t round256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

// ------------------------------------------------------------------ timing
struct TimedLaunch {
  const char* name;
  cudaEvent_t start, stop;
};
std::mutex g_timing_mu;
std::atomic<int> g_timing_on{0};
std::vector<TimedLaunch> g_timed;       // recorded launches since the last reset
std::vector<cudaEvent_t> g_event_pool;  // events free for reuse

cudaEvent_t pool_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// Brackets the kernel launches made during its lifetime with two events.
class LaunchTimer {
 public:
  LaunchTimer(const char* name, cudaStream_t st) : name_(name), st_(st) {
    if (!g_timing_on.load()) return;
    std::lock_guard<std::mutex> lk(g_timing_mu);
    start_ = pool_event();
    stop_ = pool_event();
    if (start_ && stop_) cudaEventRecord(start_, st_);
  }
  ~LaunchTimer() {
    if (!start_ || !stop_) return;
    cudaEventRecord(stop_, st_);
    std::lock_guard<std::mutex> lk(g_timing_mu);
    g_timed.push_back({name_, start_, stop_});
  }
  LaunchTimer(const LaunchTimer&) = delete;
  LaunchTimer& operator=(const LaunchTimer&) = delete;

 private:
  const char* name_;
  cudaStream_t st_;
  cudaEvent_t start_ = nullptr, stop_ = nullptr;
};

#define QLORA_CUDA_TRY(expr)                          \
  do {                                                \
    if ((expr) != cudaSuccess) return QLORA_ERR_CUDA; \
  } while (0)

// ------------------------------------------------------------------ tensor maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D bf16 row-major [rows, cols] tensor, box {64 cols, 128 rows}, 128B swizzle,
// out-of-range elements read as zero.
bool make_tmap_bf16(CUtensorMap* map, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows = 128) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D byte tensor [rows, cols] (packed NF4 codes, cols = in / 2), box
// {128 bytes, 256 rows}, 128B swizzle, out-of-range bytes read as zero.
bool make_tmap_codes(CUtensorMap* map, const void* ptr, uint64_t rows, uint64_t cols) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(qnf4::kGvStageK / 2), static_cast<cuuint32_t>(qnf4::kGvRows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Per-device facts the launch planning needs on every call, looked up once
// per device (a failed lookup, e.g. with no device, is not cached).
constexpr int kMaxDevices = 64;

int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) d = 0;
  return d;
}

int device_sm_count() {
  static std::atomic<int> cache[kMaxDevices];
  const int dev = current_device();
  const int c = cache[dev].load(std::memory_order_relaxed);
  if (c > 0) return c;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) return 148;
  cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

// The dynamic shared-memory limit of a kernel, raised to at least `bytes`
// on the current device.  The attribute persists for the process, so the
// largest value set so far is remembered per kernel and device and only a
// larger request calls cudaFuncSetAttribute again (a launch may use any
// size up to the limit).
cudaError_t set_max_smem(const void* kern, int bytes) {
  struct Entry { const void* kern; int dev; int bytes; };
  static std::mutex mu;
  static std::vector<Entry> done;
  const int dev = current_device();
  std::lock_guard<std::mutex> lk(mu);
  Entry* e = nullptr;
  for (Entry& x : done)
    if (x.kern == kern && x.dev == dev) e = &x;
  if (e != nullptr && e->bytes >= bytes) return cudaSuccess;
  const cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (err != cudaSuccess) return err;
  if (e != nullptr) e->bytes = bytes;
  else done.push_back(Entry{kern, dev, bytes});
  return cudaSuccess;
}

// ------------------------------------------------------------------ workspace
struct QuantWs {
  size_t absmax_off, tree_off, ticket_off, total;
  int64_t tree_count;  // doubles reserved for all tree passes
};

constexpr QuantWs quant_ws(int64_t rows, int64_t cols) {
  QuantWs w{};
  const int64_t n_blocks = rows * cols / 64;
  w.absmax_off = 0;
  w.tree_off = round256(static_cast<size_t>(n_blocks) * 4);
  // chunk sums of every pass down to the one the last CTA finishes, then two
  // ticket counters (one per pass parity)
  int64_t count = 0, n = n_blocks;
  do {
    n = cdiv(n, qnf4::kTreeChunk);
    count += n;
  } while (n > qnf4::kTreeTop);
  w.tree_count = count;
  w.ticket_off = w.tree_off + round256(static_cast<size_t>(count) * 8);
  w.total = w.ticket_off + 256;
  return w;
}

struct GemvPlan {
  int ctas, local_tiles, n_st;
  int64_t n_units;
};

int gemv_ctas_per_sm() {
  static std::atomic<int> cache[kMaxDevices];
  const int dev = current_device();
  const int c = cache[dev].load(std::memory_order_relaxed);
  if (c > 0) return c;
  int n = 0;
  const void* kern = reinterpret_cast<const void*>(qnf4::nf4_gemv_kernel<true, true>);
  if (set_max_smem(kern, qnf4::kGvSmem) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, qnf4::nf4_gemv_kernel<true, true>, qnf4::kGvThreads,
                                                    qnf4::kGvSmem) != cudaSuccess ||
      n < 1)
    return 1;
  cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

// Persistent grid (every CTA resident at once) splitting the (256-row tile x
// 256-column unit) sequence evenly; local_tiles bounds the tiles one CTA's
// range touches.
GemvPlan gemv_plan(int64_t in, int64_t out) {
  GemvPlan p{};
  p.n_st = static_cast<int>(cdiv(in, qnf4::kGvStageK));
  p.n_units = cdiv(out, qnf4::kGvRows) * p.n_st;
  const int64_t resident = static_cast<int64_t>(gemv_ctas_per_sm()) * device_sm_count();
  p.ctas = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(resident, p.n_units)));
  const int64_t per_cta = cdiv(p.n_units, p.ctas);
  p.local_tiles = static_cast<int>(cdiv(per_cta, p.n_st) + 1);
  return p;
}

size_t gemv_ws(int64_t M, int64_t in, int64_t out) {
  const GemvPlan p = gemv_plan(in, out);
  return round256(static_cast<size_t>(p.ctas) * p.local_tiles * M * qnf4::kGvRows * 4);
}

// LoRA rank as the kernels take it: a multiple of 8 (16-byte rows).
constexpr int padded_rank(int r) { return (r + 7) / 8 * 8; }

// Zero-padded copies used when r % 8 != 0 (pad.cuh): A [rp, in], B [out, rp],
// us [M, rp], and in the backward dA [rp, in], dB [out, rp] (fp32).
struct PadWs {
  size_t a_off, b_off, us_off, da_off, db_off, total;
};

PadWs pad_ws(int64_t M, int64_t in, int64_t out, int r, bool backward, size_t base) {
  PadWs w{};
  if (r % 8 == 0) {
    w.total = base;
    return w;
  }
  const size_t rp = static_cast<size_t>(padded_rank(r));
  w.a_off = base;
  w.b_off = w.a_off + round256(rp * in * 2);
  w.us_off = w.b_off + round256(out * rp * 2);
  w.da_off = w.us_off + round256(M * rp * 2);
  w.db_off = w.da_off + (backward ? round256(rp * in * 4) : 0);
  w.total = w.db_off + (backward ? round256(out * rp * 4) : 0);
  return w;
}

// Few-token rank-r product (fewtok.cuh): its partials, then its ticket.
size_t fewtok_ws(int64_t in, int r) {
  return round256(static_cast<size_t>(qnf4::fewtok_part_floats(in, padded_rank(r))) * 4) + 256;
}

// Forward workspace: for M <= 16 the GEMV partials, then the few-token
// rank-r partials and ticket; then the padded copies (r % 8 != 0).
size_t fwd_base_ws(int64_t M, int64_t in, int64_t out, int r) {
  return M <= 16 ? gemv_ws(M, in, out) + fewtok_ws(in, r) : 0;
}

size_t fwd_ws(int64_t M, int64_t in, int64_t out, int r) {
  return pad_ws(M, in, out, r, false, fwd_base_ws(M, in, out, r)).total;
}

size_t fwd_dropout_ws(int64_t M, int64_t in, int64_t out, int r) { return fwd_ws(M, in, out, r); }

struct BwdWs {
  size_t du_off;
  PadWs pad;
  size_t total;
};

BwdWs bwd_ws(int64_t M, int64_t in, int64_t out, int r) {
  BwdWs w{};
  w.du_off = 0;
  w.pad = pad_ws(M, in, out, r, true, round256(static_cast<size_t>(M) * padded_rank(r) * 2));
  w.total = w.pad.total;
  return w;
}

template <typename T>
int launch_copy_pad(const T* src, int64_t src_rows, int64_t src_cols, T* dst, int64_t dst_rows, int64_t dst_cols,
                    cudaStream_t st) {
  const int64_t n = dst_rows * dst_cols;
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(cdiv(n, 256), device_sm_count() * 8)));
  {
    LaunchTimer lt_("lora_pad", st);
    qnf4::copy_pad_kernel<T><<<grid, 256, 0, st>>>(src, src_rows, src_cols, dst, dst_rows, dst_cols);
  }
  QLORA_CUDA_TRY(cudaGetLastError());
  return QLORA_OK;
}

// ------------------------------------------------------------------ launches
// K1: codes and block absmaxes.  Also resets tickets[0] for the tree pass after it.
template <typename Tin>
int launch_blocks(const Tin* W, int64_t n_blocks, uint8_t* codes, float* absmax, unsigned int* tickets,
                  const Tables& tb, cudaStream_t st) {
  const int sms = device_sm_count();
  const int64_t want = cdiv(n_blocks, 64 * qnf4::kQRounds);       // 8 warps x 8 blocks x rounds per CTA
  // one wave: 4 CTAs of 256 threads fit an SM at the kernel's register count
  const int grid1 = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(want, static_cast<int64_t>(sms) * 4)));
  {
    LaunchTimer lt_("quantize_blocks", st);
    qnf4::nf4_quantize_blocks_kernel<Tin><<<grid1, 256, 0, st>>>(W, n_blocks, codes, absmax, tb.C, tickets);
  }
  QLORA_CUDA_TRY(cudaGetLastError());
  return QLORA_OK;
}

// Fixed summation tree from `n` leaves (block absmaxes, or the fp64 sums of
// 4096-leaf subtrees): 4096x reductions; the pass that leaves at most
// kTreeTop sums is finished (and mean = fp32(total / n_leaves_total) written)
// by its last CTA.  tickets[0] must be 0 on entry; each pass resets the
// ticket of the pass after it (they alternate).  `tree` holds the sums of
// every pass.
template <typename T>
int launch_mean_tree(const T* leaves, int64_t n, double* tree, unsigned int* tickets, int64_t n_leaves_total,
                     float* mean, cudaStream_t st) {
  int64_t parts = cdiv(n, qnf4::kTreeChunk);
  int pass = 0;
  {
    LaunchTimer lt_("scale_mean_tree", st);
    qnf4::pairwise_tree_kernel<T><<<static_cast<unsigned>(parts), 256, 0, st>>>(
        leaves, n, tree, parts <= qnf4::kTreeTop, tickets, n_leaves_total, mean, tickets + 1);
  }
  QLORA_CUDA_TRY(cudaGetLastError());
  double* prev = tree;
  while (parts > qnf4::kTreeTop) {
    n = parts;
    parts = cdiv(n, qnf4::kTreeChunk);
    double* next = prev + n;
    ++pass;
    {
      LaunchTimer lt_("scale_mean_tree", st);
      qnf4::pairwise_tree_kernel<double><<<static_cast<unsigned>(parts), 256, 0, st>>>(
          prev, n, next, parts <= qnf4::kTreeTop, tickets + (pass & 1), n_leaves_total, mean,
          tickets + ((pass + 1) & 1));
    }
    QLORA_CUDA_TRY(cudaGetLastError());
    prev = next;
  }
  return QLORA_OK;
}

// K3: second-level codes of n_blocks scales against a finished mean.
int launch_dq(const float* absmax, int64_t n_blocks, const float* mean, int8_t* q8, float* step2, cudaStream_t st) {
  const int64_t n_groups = cdiv(n_blocks, qnf4::kGroup);
  {
    LaunchTimer lt_("dq_scales", st);
    qnf4::dq_scales_kernel<<<static_cast<unsigned>(cdiv(n_groups * 32, 256)), 256, 0, st>>>(absmax, n_blocks, mean,
                                                                                          q8, step2);
  }
  QLORA_CUDA_TRY(cudaGetLastError());
  return QLORA_OK;
}

template <typename Tin>
int launch_quantize(const Tin* W, int64_t rows, int64_t cols, uint8_t* codes, int8_t* q8, float* step2,
                    float* mean, void* ws, cudaStream_t st, const Tables& tb = tables()) {
  const int64_t n_blocks = rows * cols / 64;
  const QuantWs w = quant_ws(rows, cols);
  float* absmax = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + w.absmax_off);
  double* tree = reinterpret_cast<double*>(static_cast<uint8_t*>(ws) + w.tree_off);
  unsigned int* tickets = reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(ws) + w.ticket_off);
  int rc = launch_blocks(W, n_blocks, codes, absmax, tickets, tb, st);
  if (rc != QLORA_OK) return rc;
  rc = launch_mean_tree(static_cast<const float*>(absmax), n_blocks, tree, tickets, n_blocks, mean, st);
  if (rc != QLORA_OK) return rc;
  return launch_dq(absmax, n_blocks, mean, q8, step2, st);
}

// Sharded quantization: rank k of `world` takes the 4096-block chunks
// [k cpr, (k+1) cpr) of the flattened weight, cpr = ceil(chunks / world), so
// every shard starts on a chunk (hence on a 256-block group) boundary and
// its chunk sums are exactly the first-pass sums of the unsharded tree.
struct ShardWs {
  size_t absmax_off, tree_off, ticket_off, total;
};

ShardWs shard_ws(int64_t n_blocks_shard, int64_t n_roots_total) {
  ShardWs w{};
  w.absmax_off = 0;
  w.tree_off = round256(static_cast<size_t>(std::max<int64_t>(n_blocks_shard, 1)) * 4);
  int64_t count = 0, n = n_roots_total;
  do {
    n = cdiv(n, qnf4::kTreeChunk);
    count += n;
  } while (n > qnf4::kTreeTop);
  w.ticket_off = w.tree_off + round256(static_cast<size_t>(count) * 8);
  w.total = w.ticket_off + 256;
  return w;
}

int gemm_tile_m(int64_t M) {
  static int forced = [] {
    const char* e = std::getenv("QLORA_NF4_GEMM_TILE_M");
    return e ? std::atoi(e) : 0;
  }();
  if (forced == 128 || forced == 256 || forced == 512) return forced;
  if (M > 384) return 512;       // CTA-pair tile (cta_group::2)
  return M > 128 ? 256 : 128;
}

template <int MS, bool kDx, int kStages>
int launch_gemm_t(const qnf4::GemmArgs& args, const CUtensorMap& tm_act, const CUtensorMap& tm_lora,
                  cudaStream_t st) {
  using Cfg = qnf4::GemmCfg<MS, kStages>;
  auto kern = qnf4::qlora_gemm_kernel<MS, kDx, kStages>;
  QLORA_CUDA_TRY(set_max_smem(reinterpret_cast<const void*>(kern), Cfg::SMEM));
  const int64_t tiles = cdiv(args.M, Cfg::BM) * cdiv(args.N, Cfg::BN);
  {
    LaunchTimer lt_(kDx ? "gemm_dx" : "gemm_fwd", st);
    kern<<<static_cast<unsigned>(tiles), Cfg::THREADS, Cfg::SMEM, st>>>(tm_act, tm_lora, args);
  }
  QLORA_CUDA_TRY(cudaGetLastError());
  return QLORA_OK;
}

template <bool kDx>
int launch_gemm_pair(const qnf4::GemmArgs& args, const CUtensorMap& tm_act, const CUtensorMap& tm_lora,
                     cudaStream_t st) {
  using Cfg = qnf4::PairCfg;
  auto kern = qnf4::qlora_gemm_pair_kernel<kDx>;
  QLORA_CUDA_TRY(set_max_smem(reinterpret_cast<const void*>(kern), Cfg::SMEM));
  const int64_t pairs = cdiv(args.M, Cfg::BM) * cdiv(args.N, Cfg::BN);
  {
    LaunchTimer lt_(kDx ? "gemm_dx" : "gemm_fwd", st);
    kern<<<static_cast<unsigned>(2 * pairs), Cfg::THREADS, Cfg::SMEM, st>>>(tm_act, tm_lora, args);
  }
  QLORA_CUDA_TRY(cudaGetLastError());
  return QLORA_OK;
}

// act [M, K] and lora_act [M, r] are the A operands; the output has N columns.
int launch_gemm(bool dx, const qlora_nf4_weight* w, const uint16_t* act, int64_t M, int64_t K,
                const uint16_t* lora_act, const uint16_t* lora_w, int r, uint16_t* out, int64_t N,
                cudaStream_t st) {
  CUtensorMap tm_act, tm_lora;
  if (!make_tmap_bf16(&tm_act, act, M, K)) return QLORA_ERR_CUDA;
  if (r == 0) tm_lora = tm_act;                  // no rank-r tail: the map is never used
  else if (!make_tmap_bf16(&tm_lora, lora_act, M, r)) return QLORA_ERR_CUDA;
  qnf4::GemmArgs a{};
  a.codes = w->codes;
  a.q8 = w->q8;
  a.step2 = w->step2;
  a.mean = w->mean;
  a.lora_w = lora_w;
  a.out = out;
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  a.r = r;
  a.w_cols = static_cast<int>(w->cols);
  a.codes_32b = aligned(w->codes, 32) ? 1 : 0;
  a.L = tables().L;
  a.timeout_ns = g_timeout_ns.load();
  const int tm = gemm_tile_m(M);
  if (tm == 512) return dx ? launch_gemm_pair<true>(a, tm_act, tm_lora, st) : launch_gemm_pair<false>(a, tm_act, tm_lora, st);
  if (!dx) {
    return tm == 256 ? launch_gemm_t<2, false, 3>(a, tm_act, tm_lora, st)
                     : launch_gemm_t<1, false, 4>(a, tm_act, tm_lora, st);
  }
  return tm == 256 ? launch_gemm_t<2, true, 3>(a, tm_act, tm_lora, st)
                   : launch_gemm_t<1, true, 4>(a, tm_act, tm_lora, st);
}

// ------------------------------------------------------------------ tcgen05 rank-r products
int lr_n_alloc(int N) {
  int a = 32;
  while (a < N) a *= 2;
  return a;
}

// Launch shape of a rank-r product: a ring of 4 stages (measured best: deeper
// rings in one CTA per SM streamed slower), two CTAs per SM where the
// shared memory allows it; the contraction is split over a cluster (a power
// of two <= 8) as far as the CTAs still fit about one per SM, keeping at
// least 2 stages per split.
struct LrShape {
  int ks, ring;
};

// Split count ks (a power of two <= 8, the cluster size): doubled while the
// grid stays within the CTAs that fit at once (one or two per SM, by the
// kernel's shared memory for this rank) and every split keeps at least two
// 64-wide stages.
LrShape lr_shape(int64_t tiles, int64_t stages, int N, bool b_mn_major) {
  const int sms = device_sm_count();
  LrShape sh{1, 4};
  const int per_sm = 2 * (qnf4::lr_smem_bytes(N, b_mn_major, sh.ring) + 1024) <= 228 * 1024 ? 2 : 1;
  while (sh.ks < 8 && tiles * sh.ks * 2 <= per_sm * sms && stages / (2 * sh.ks) >= 2) sh.ks *= 2;
  return sh;
}

template <bool kCol, bool kBMN>
int launch_lora_umma(const CUtensorMap (&tm)[4], const qnf4::LrArgs& a, int ks, unsigned grid_x, const char* name,
                     cudaStream_t st) {
  auto kern = qnf4::lora_umma_kernel<kCol, kBMN>;
  const int smem = qnf4::lr_smem_bytes(a.N, kBMN, a.ring);
  QLORA_CUDA_TRY(set_max_smem(reinterpret_cast<const void*>(kern), smem));
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid_x, static_cast<unsigned>(ks), 1);
  const bool masked = a.p[0].keep != nullptr || a.p[1].keep != nullptr;
  cfg.blockDim = dim3(masked ? qnf4::kLrMaskThreads : qnf4::kLrThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = static_cast<unsigned>(ks);
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = ks > 1 ? 1 : 0;
  {
    LaunchTimer lt_(name, st);
    QLORA_CUDA_TRY(cudaLaunchKernelEx(&cfg, kern, tm[0], tm[1], tm[2], tm[3], a));
  }
  QLORA_CUDA_TRY(cudaGetLastError());
  return QLORA_OK;
}

// Row form: out[M, r] = bf16(scale * act[M, K] . w^T), w given as [r, K]
// (w_n_major = false: A of the forward) or as [K, r] (true: B of du).
int launch_lora_row(const uint16_t* act, const uint16_t* w, uint16_t* out, int64_t M, int64_t K, int r, float scale,
                    bool w_n_major, const char* name, cudaStream_t st, const uint8_t* keep = nullptr) {
  qnf4::LrArgs a{};
  a.r = r;
  a.N = (r + 15) / 16 * 16;
  a.n_alloc = lr_n_alloc(a.N);
  a.K = static_cast<int>(K);
  a.p[0] = qnf4::LrProblem{out, static_cast<int>(M), static_cast<int>(cdiv(M, 128)), 0, scale, keep,
                           static_cast<int>(K)};
  a.p[1] = a.p[0];
  a.timeout_ns = g_timeout_ns.load();
  const int64_t stages = cdiv(K, 64);
  const LrShape sh = lr_shape(a.p[0].tiles, stages, a.N, w_n_major);
  // with a keep mask the 320-thread CTAs ran slower in clusters of 8 (7B
  // attention: 25.2 us against 23.1 us in clusters of 4)
  const int ks = keep != nullptr ? std::min(sh.ks, 4) : sh.ks;
  a.ring = sh.ring;
  a.stages_per_split = static_cast<int>(cdiv(stages, ks));
  CUtensorMap tm[4];
  if (!make_tmap_bf16(&tm[0], act, M, K, 128)) return QLORA_ERR_CUDA;
  const bool ok = w_n_major ? make_tmap_bf16(&tm[1], w, K, r, 64) : make_tmap_bf16(&tm[1], w, r, K, a.N);
  if (!ok) return QLORA_ERR_CUDA;
  tm[2] = tm[0];
  tm[3] = tm[1];
  const unsigned gx = static_cast<unsigned>(a.p[0].tiles);
  return w_n_major ? launch_lora_umma<false, true>(tm, a, ks, gx, name, st)
                   : launch_lora_umma<false, false>(tm, a, ks, gx, name, st);
}

// Col form, both adapter gradients in one launch: dB [out, r] = dh^T us and
// dA [r, in] = (x^T du)^T * dA_scale.
int launch_lora_col(const uint16_t* dh, const uint16_t* us, const uint16_t* x, const uint16_t* du, int64_t M,
                    int64_t in, int64_t out, int r, float* dB, float* dA, float dA_scale, cudaStream_t st,
                    const uint8_t* keep = nullptr) {
  qnf4::LrArgs a{};
  a.r = r;
  a.N = (r + 15) / 16 * 16;
  a.n_alloc = lr_n_alloc(a.N);
  a.K = static_cast<int>(M);
  a.p[0] = qnf4::LrProblem{dB, static_cast<int>(out), static_cast<int>(cdiv(out, 128)), 0, 1.f, nullptr,
                           static_cast<int>(out)};
  a.p[1] = qnf4::LrProblem{dA, static_cast<int>(in), static_cast<int>(cdiv(in, 128)), 1, dA_scale, keep,
                           static_cast<int>(in)};
  a.timeout_ns = g_timeout_ns.load();
  const int64_t stages = cdiv(M, 64);
  const LrShape sh = lr_shape(a.p[0].tiles + a.p[1].tiles, stages, a.N, true);
  const int ks = sh.ks;
  a.ring = sh.ring;
  a.stages_per_split = static_cast<int>(cdiv(stages, ks));
  CUtensorMap tm[4];
  if (!make_tmap_bf16(&tm[0], dh, M, out, 64) || !make_tmap_bf16(&tm[1], us, M, r, 64) ||
      !make_tmap_bf16(&tm[2], x, M, in, 64) || !make_tmap_bf16(&tm[3], du, M, r, 64))
    return QLORA_ERR_CUDA;
  return launch_lora_umma<true, true>(tm, a, ks, static_cast<unsigned>(a.p[0].tiles + a.p[1].tiles), "lora_colwise",
                                      st);
}

// out[M, R] = bf16(scale * (act[M, K] * k) . W^T) with W given as [R, K] (kKR =
// false) or as [K, R] (kKR = true); k the keep mask of LoRA dropout, or all
// ones when keep is null.
template <bool kKR>
int launch_rowwise(const uint16_t* act, const uint16_t* W, uint16_t* out, int64_t M, int64_t K, int R, float scale,
                   cudaStream_t st, const uint8_t* keep = nullptr) {
  return launch_lora_row(act, W, out, M, K, R, scale, kKR, kKR ? "lora_rowwise_du" : "lora_rowwise", st, keep);
}

// dB = dh^T us -> [out, r] and dA = du^T (x * k) * dA_scale -> [r, in] in one launch.
int launch_lora_grads(const uint16_t* dh, const uint16_t* us, const uint16_t* x, const uint16_t* du, int64_t M,
                      int64_t in, int64_t out, int R, float* dB, float* dA, cudaStream_t st, float dA_scale = 1.f,
                      const uint8_t* keep = nullptr) {
  return launch_lora_col(dh, us, x, du, M, in, out, R, dB, dA, dA_scale, st, keep);
}

// ------------------------------------------------------------------ validation
bool weight_ok(const qlora_nf4_weight* w) {
  return w != nullptr && w->codes && w->q8 && w->step2 && w->mean && aligned(w->codes, 16) &&
         aligned(w->q8, 16) && aligned(w->step2, 16) && aligned(w->mean, 16);
}

int check_linear_shapes(int64_t M, const qlora_nf4_weight* w, int r) {
  if (M < 1 || w->rows < 64 || w->cols < 64) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (w->cols % 64 != 0 || w->rows % 64 != 0) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (r < 1 || r > 256) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (M > (1ll << 31) - 1024 || w->rows > (1ll << 30) || w->cols > (1ll << 30))
    return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (w->rows * w->cols > (1ll << 40)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  return QLORA_OK;
}

// ------------------------------------------------------------------ internal streams
// Two internal streams per device (highest and lowest priority), created on
// first use and kept for the process, and a pool of events.  The mutex
// covers one call's issue (the streams and events are shared).
struct GroupStreams {
  std::mutex mu;
  cudaStream_t hi = nullptr, lo = nullptr;
  std::vector<cudaEvent_t> ev;
};

GroupStreams& group_streams() {
  static GroupStreams g[kMaxDevices];
  return g[current_device()];
}

// With g.mu held: the streams exist and the pool has at least n events.
int ensure_group_streams(GroupStreams& g, int n) {
  if (g.hi == nullptr) {
    int least = 0, greatest = 0;
    QLORA_CUDA_TRY(cudaDeviceGetStreamPriorityRange(&least, &greatest));
    QLORA_CUDA_TRY(cudaStreamCreateWithPriority(&g.hi, cudaStreamNonBlocking, greatest));
    QLORA_CUDA_TRY(cudaStreamCreateWithPriority(&g.lo, cudaStreamNonBlocking, least));
  }
  while (static_cast<int>(g.ev.size()) < n) {
    cudaEvent_t e;
    QLORA_CUDA_TRY(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
    g.ev.push_back(e);
  }
  return QLORA_OK;
}

// Forward after validation: us = bf16(s_lora * (x * k) A^T) (k all ones, or
// the keep mask of LoRA dropout with s_lora = s / (1 - p)), then
// h = [x | us] [W0 | B]^T; `workspace` is the GEMV part (M <= 16).
int linear_fwd_impl(const uint16_t* x, const uint8_t* keep, int64_t M, const qlora_nf4_weight* w,
                    const uint16_t* A, const uint16_t* B, int r, float s_lora, uint16_t* h, uint16_t* us_out,
                    void* workspace, cudaStream_t st) {
  const int64_t in = w->cols, out = w->rows;
  int rc = QLORA_OK;
  if (M <= 16) {                                                            // us = bf16(s (x k) A^T)
    uint8_t* ft = static_cast<uint8_t*>(workspace) + gemv_ws(M, in, out);
    float* ft_part = reinterpret_cast<float*>(ft);
    unsigned int* ticket = reinterpret_cast<unsigned int*>(ft + fewtok_ws(in, r) - 256);
    QLORA_CUDA_TRY(cudaMemsetAsync(ticket, 0, sizeof(unsigned int), st));
    const unsigned chunks = static_cast<unsigned>(cdiv(in, qnf4::kFtChunk));
    LaunchTimer lt_("lora_fewtok", st);
    if (M > 8)
      qnf4::fewtok_us_kernel<16><<<chunks, qnf4::kFtThreads, 0, st>>>(x, keep, A, static_cast<int>(M), in, r, s_lora,
                                                                      ft_part, ticket, us_out);
    else
      qnf4::fewtok_us_kernel<8><<<chunks, qnf4::kFtThreads, 0, st>>>(x, keep, A, static_cast<int>(M), in, r, s_lora,
                                                                     ft_part, ticket, us_out);
  } else {
    rc = launch_rowwise<false>(x, A, us_out, M, in, r, s_lora, st, keep);    // us = bf16(s (x k) A^T)
  }
  if (rc != QLORA_OK) return rc;
  QLORA_CUDA_TRY(cudaGetLastError());
  if (M <= 16) {
    const GemvPlan p = gemv_plan(in, out);
    qnf4::GemvArgs g{};
    g.q8 = w->q8;
    g.step2 = w->step2;
    g.mean = w->mean;
    g.part = static_cast<float*>(workspace);
    g.M = static_cast<int>(M);
    g.in = static_cast<int>(in);
    g.out = static_cast<int>(out);
    g.n_st = p.n_st;
    g.n_units = p.n_units;
    g.local_tiles = p.local_tiles;
    g.timeout_ns = g_timeout_ns.load();
    g.L = tables().L;
    CUtensorMap tm_codes, tm_x;
    if (!make_tmap_codes(&tm_codes, w->codes, static_cast<uint64_t>(out), static_cast<uint64_t>(in / 2)) ||
        !make_tmap_bf16(&tm_x, x, static_cast<uint64_t>(M), static_cast<uint64_t>(in), M > 8 ? 16 : 8))
      return QLORA_ERR_CUDA;
    {
      LaunchTimer lt_("gemv", st);
      const bool paired = in % qnf4::kGvStageK == 0, two_tok = M > 8;   // four whole blocks per unit
      auto kern = paired ? (two_tok ? qnf4::nf4_gemv_kernel<true, true> : qnf4::nf4_gemv_kernel<true, false>)
                         : (two_tok ? qnf4::nf4_gemv_kernel<false, true> : qnf4::nf4_gemv_kernel<false, false>);
      QLORA_CUDA_TRY(set_max_smem(reinterpret_cast<const void*>(kern), qnf4::kGvSmem));
      kern<<<p.ctas, qnf4::kGvThreads, qnf4::kGvSmem, st>>>(tm_codes, tm_x, g);
    }
    QLORA_CUDA_TRY(cudaGetLastError());
    {
      LaunchTimer lt_("gemv_finalize", st);
      const dim3 grid(static_cast<unsigned>(cdiv(out, qnf4::kGvRows)), static_cast<unsigned>(M));
      qnf4::gemv_finalize_kernel<<<grid, qnf4::kGvRows, 0, st>>>(
          g.part, p.ctas, p.local_tiles, p.n_units, p.n_st, static_cast<int>(M), static_cast<int>(out), us_out, B, r, h);
    }
    QLORA_CUDA_TRY(cudaGetLastError());
    return QLORA_OK;
  }
  return launch_gemm(false, w, x, M, in, us_out, B, r, h, out, st);  // h = [x|us] [W0|B]^T
}

// Forward at any rank: r % 8 == 0 runs linear_fwd_impl directly; otherwise
// on zero-padded copies of A and B at rp = r rounded up to 8, with us
// computed at rp in the workspace and copied back to [M, r].
int linear_fwd_any_rank(const uint16_t* x, const uint8_t* keep, int64_t M, const qlora_nf4_weight* w,
                        const uint16_t* A, const uint16_t* B, int r, float s_lora, uint16_t* h, uint16_t* us_out,
                        void* workspace, cudaStream_t st) {
  if (r % 8 == 0) return linear_fwd_impl(x, keep, M, w, A, B, r, s_lora, h, us_out, workspace, st);
  const int64_t in = w->cols, out = w->rows;
  const int rp = padded_rank(r);
  const PadWs pw = pad_ws(M, in, out, r, false, fwd_base_ws(M, in, out, r));
  uint8_t* base = static_cast<uint8_t*>(workspace);
  uint16_t* A_p = reinterpret_cast<uint16_t*>(base + pw.a_off);
  uint16_t* B_p = reinterpret_cast<uint16_t*>(base + pw.b_off);
  uint16_t* us_p = reinterpret_cast<uint16_t*>(base + pw.us_off);
  int rc = launch_copy_pad(A, r, in, A_p, rp, in, st);
  if (rc == QLORA_OK) rc = launch_copy_pad(B, out, r, B_p, out, rp, st);
  if (rc == QLORA_OK) rc = linear_fwd_impl(x, keep, M, w, A_p, B_p, rp, s_lora, h, us_p, workspace, st);
  if (rc == QLORA_OK) rc = launch_copy_pad(us_p, M, rp, us_out, M, r, st);
  return rc;
}

// Backward after validation, rank a multiple of 8: du = bf16(s dh B) into
// `du`, then dx (with its rank-r tail, or without it plus the masked term
// when keep is given) and dB, dA.
int linear_bwd_impl(const uint16_t* dh, const uint16_t* x, const uint16_t* us, int64_t M,
                    const qlora_nf4_weight* w, const uint16_t* A, const uint16_t* B, int r, float s,
                    const uint8_t* keep, float inv_keep, uint16_t* dx, float* dA, float* dB, uint16_t* du,
                    cudaStream_t st) {
  const int64_t in = w->cols, out = w->rows;
  if (keep == nullptr) {
    int rc = launch_rowwise<true>(dh, B, du, M, out, r, s, st);                         // du = bf16(s dh B)
    if (rc != QLORA_OK) return rc;
    rc = launch_gemm(true, w, dh, M, out, du, A, r, dx, in, st);                         // dx = [dh|du][W0;A]
    if (rc != QLORA_OK) return rc;
    return launch_lora_grads(dh, us, x, du, M, in, out, r, dB, dA, st);                  // dB, dA
  }
  // LoRA dropout: the dx GEMM runs without its rank-r tail, so du and the
  // adapter gradients do not wait for it.  The GEMM goes first on the internal
  // high-priority stream; du, dB and dA run on the low-priority one, on the
  // SMs the GEMM's last wave leaves free; the masked dx term waits for the
  // GEMM and for du.  Both streams are forked from and joined back into `st`.
  GroupStreams& g = group_streams();
  std::lock_guard<std::mutex> lock(g.mu);
  const int rc0 = ensure_group_streams(g, 4);
  if (rc0 != QLORA_OK) return rc0;
  QLORA_CUDA_TRY(cudaEventRecord(g.ev[0], st));
  QLORA_CUDA_TRY(cudaStreamWaitEvent(g.hi, g.ev[0], 0));
  QLORA_CUDA_TRY(cudaStreamWaitEvent(g.lo, g.ev[0], 0));
  int rc = launch_gemm(true, w, dh, M, out, nullptr, nullptr, 0, dx, in, g.hi);          // dx = dh W0
  if (rc == QLORA_OK) rc = launch_rowwise<true>(dh, B, du, M, out, r, s, g.lo);         // du = bf16(s dh B)
  if (rc == QLORA_OK && cudaEventRecord(g.ev[1], g.lo) != cudaSuccess) rc = QLORA_ERR_CUDA;
  if (rc == QLORA_OK)
    rc = launch_lora_grads(dh, us, x, du, M, in, out, r, dB, dA, g.lo, inv_keep, keep);  // dB, dA
  if (rc == QLORA_OK && cudaStreamWaitEvent(g.hi, g.ev[1], 0) != cudaSuccess) rc = QLORA_ERR_CUDA;
  if (rc == QLORA_OK) {
    const int64_t tiles = cdiv(M, qnf4::kDxTileRows) * cdiv(in, qnf4::kDxTileCols);
    const int smem = qnf4::dx_smem_bytes(r);
    if (set_max_smem(reinterpret_cast<const void*>(qnf4::dropout_dx_kernel), smem) != cudaSuccess) {
      rc = QLORA_ERR_CUDA;
    } else {
      LaunchTimer lt_("dropout_dx", g.hi);
      qnf4::dropout_dx_kernel<<<static_cast<unsigned>(tiles), qnf4::kDxThreads, smem, g.hi>>>(
          dx, du, A, keep, M, in, r, inv_keep);                                           // + (du A) k/(1-p)
      if (cudaGetLastError() != cudaSuccess) rc = QLORA_ERR_CUDA;
    }
  }
  // join both streams back into `st` (after an error too)
  QLORA_CUDA_TRY(cudaEventRecord(g.ev[2], g.hi));
  QLORA_CUDA_TRY(cudaEventRecord(g.ev[3], g.lo));
  QLORA_CUDA_TRY(cudaStreamWaitEvent(st, g.ev[2], 0));
  QLORA_CUDA_TRY(cudaStreamWaitEvent(st, g.ev[3], 0));
  return rc;
}

// Backward at any rank (the padded copies as in linear_fwd_any_rank; dA and
// dB are computed at rp and copied back to [r, in] and [out, r]).
int linear_bwd_any_rank(const uint16_t* dh, const uint16_t* x, const uint16_t* us, int64_t M,
                        const qlora_nf4_weight* w, const uint16_t* A, const uint16_t* B, int r, float s,
                        const uint8_t* keep, float inv_keep, uint16_t* dx, float* dA, float* dB, void* workspace,
                        cudaStream_t st) {
  const int64_t in = w->cols, out = w->rows;
  const BwdWs ws = bwd_ws(M, in, out, r);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  uint16_t* du = reinterpret_cast<uint16_t*>(base + ws.du_off);
  if (r % 8 == 0) return linear_bwd_impl(dh, x, us, M, w, A, B, r, s, keep, inv_keep, dx, dA, dB, du, st);
  const int rp = padded_rank(r);
  uint16_t* A_p = reinterpret_cast<uint16_t*>(base + ws.pad.a_off);
  uint16_t* B_p = reinterpret_cast<uint16_t*>(base + ws.pad.b_off);
  uint16_t* us_p = reinterpret_cast<uint16_t*>(base + ws.pad.us_off);
  float* dA_p = reinterpret_cast<float*>(base + ws.pad.da_off);
  float* dB_p = reinterpret_cast<float*>(base + ws.pad.db_off);
  int rc = launch_copy_pad(A, r, in, A_p, rp, in, st);
  if (rc == QLORA_OK) rc = launch_copy_pad(B, out, r, B_p, out, rp, st);
  if (rc == QLORA_OK) rc = launch_copy_pad(us, M, r, us_p, M, rp, st);
  if (rc == QLORA_OK) rc = linear_bwd_impl(dh, x, us_p, M, w, A_p, B_p, rp, s, keep, inv_keep, dx, dA_p, dB_p, du, st);
  if (rc == QLORA_OK) rc = launch_copy_pad(dA_p, rp, in, dA, r, in, st);
  if (rc == QLORA_OK) rc = launch_copy_pad(dB_p, out, rp, dB, out, r, st);
  return rc;
}

int check_fwd_args(const uint16_t* x, int64_t M, const qlora_nf4_weight* w, const uint16_t* A, const uint16_t* B,
                   int r, float alpha, const uint16_t* h, const uint16_t* us_out) {
  if (!x || !weight_ok(w) || !A || !B || !h || !us_out) return QLORA_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(A, 16) || !aligned(B, 16) || !aligned(h, 16) || !aligned(us_out, 16))
    return QLORA_ERR_INVALID_ARG;
  if (!std::isfinite(alpha)) return QLORA_ERR_INVALID_ARG;
  return check_linear_shapes(M, w, r);
}

int check_dropout_args(const uint8_t* keep_bits, float p) {
  if (keep_bits == nullptr || !aligned(keep_bits, 4) || !(p >= 0.f && p < 1.f)) return QLORA_ERR_INVALID_ARG;
  return QLORA_OK;
}

int check_bwd_args(const uint16_t* dh, const uint16_t* x, const uint16_t* us, int64_t M, const qlora_nf4_weight* w,
                   const uint16_t* A, const uint16_t* B, int r, float alpha, const uint16_t* dx, const float* dA,
                   const float* dB) {
  if (!dh || !x || !us || !weight_ok(w) || !A || !B || !dx || !dA || !dB) return QLORA_ERR_INVALID_ARG;
  if (!aligned(dh, 16) || !aligned(x, 16) || !aligned(us, 16) || !aligned(A, 16) || !aligned(B, 16) ||
      !aligned(dx, 16) || !aligned(dA, 16) || !aligned(dB, 16))
    return QLORA_ERR_INVALID_ARG;
  if (!std::isfinite(alpha)) return QLORA_ERR_INVALID_ARG;
  return check_linear_shapes(M, w, r);
}

// The rank-r work of a projection moves to the low-priority stream only on
// the path where it is separate from the GEMM (M > 16, r % 8 == 0).
bool group_split(const qlora_linear_problem& p) { return p.M > 16 && p.r % 8 == 0; }

size_t group_ws_each(bool backward, const qlora_linear_problem& p) {
  const size_t n = backward ? bwd_ws(p.M, p.w->cols, p.w->rows, p.r).total : fwd_ws(p.M, p.w->cols, p.w->rows, p.r);
  return round256(n);
}

// Issue a group: fork both internal streams from `st`, run `body`, join
// both back into `st` (also after an error, so that `st` stays ordered
// after everything that was issued).
template <typename Body>
int group_issue(int n_events, cudaStream_t st, Body body) {
  GroupStreams& g = group_streams();
  std::lock_guard<std::mutex> lock(g.mu);
  const int rc0 = ensure_group_streams(g, n_events + 3);
  if (rc0 != QLORA_OK) return rc0;
  cudaEvent_t fork = g.ev[0], j_hi = g.ev[1], j_lo = g.ev[2];
  QLORA_CUDA_TRY(cudaEventRecord(fork, st));
  QLORA_CUDA_TRY(cudaStreamWaitEvent(g.hi, fork, 0));
  QLORA_CUDA_TRY(cudaStreamWaitEvent(g.lo, fork, 0));
  const int rc = body(g.hi, g.lo, g.ev.data() + 3);
  QLORA_CUDA_TRY(cudaEventRecord(j_hi, g.hi));
  QLORA_CUDA_TRY(cudaEventRecord(j_lo, g.lo));
  QLORA_CUDA_TRY(cudaStreamWaitEvent(st, j_hi, 0));
  QLORA_CUDA_TRY(cudaStreamWaitEvent(st, j_lo, 0));
  return rc;
}


}  // namespace

// ============================================================================ C ABI
extern "C" {

int qlora_nf4_codebook(float levels[16], float thresholds[15]) {
  if (levels == nullptr) return QLORA_ERR_INVALID_ARG;
  const Tables& t = tables();
  std::memcpy(levels, t.L.v, sizeof(t.L.v));
  if (thresholds != nullptr) std::memcpy(thresholds, t.T.v, sizeof(t.T.v));
  return QLORA_OK;
}

size_t qlora_workspace_size(int op, int64_t M, int64_t in_features, int64_t out_features, int r) {
  if (M < 0 || in_features < 0 || out_features < 0 || r < 0) return static_cast<size_t>(-1);
  switch (op) {
    case QLORA_OP_QUANTIZE:
      if (in_features < 64 || out_features < 1) return 0;
      return quant_ws(out_features, in_features).total;
    case QLORA_OP_DEQUANTIZE:
      return 0;
    case QLORA_OP_LINEAR_FWD:
      if (M < 1) return 0;
      return fwd_ws(M, in_features, out_features, r);
    case QLORA_OP_LINEAR_BWD:
      if (M < 1 || r < 1) return 0;
      return bwd_ws(M, in_features, out_features, r).total;
    case QLORA_OP_LINEAR_FWD_DROPOUT:
      if (M < 1) return 0;
      return fwd_dropout_ws(M, in_features, out_features, r);
    case QLORA_OP_LINEAR_BWD_DROPOUT:
      if (M < 1 || r < 1) return 0;
      return bwd_ws(M, in_features, out_features, r).total;
    default:
      return static_cast<size_t>(-1);
  }
}

int qlora_quantize_nf4(const float* W, int64_t rows, int64_t cols, uint8_t* codes, int8_t* q8, float* step2,
                       float* mean, void* workspace, size_t workspace_bytes, void* stream) {
  if (!W || !codes || !q8 || !step2 || !mean) return QLORA_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(codes, 16) || !aligned(q8, 16) || !aligned(step2, 16) || !aligned(mean, 16))
    return QLORA_ERR_INVALID_ARG;
  if (rows < 1 || cols < 64 || cols % 64 != 0 || rows * cols > (1ll << 40)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  const QuantWs w = quant_ws(rows, cols);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < w.total) return QLORA_ERR_WORKSPACE;
  return launch_quantize(W, rows, cols, codes, q8, step2, mean, workspace, static_cast<cudaStream_t>(stream));
}

int qlora_quantize_nf4_bf16(const uint16_t* W, int64_t rows, int64_t cols, uint8_t* codes, int8_t* q8, float* step2,
                            float* mean, void* workspace, size_t workspace_bytes, void* stream) {
  if (!W || !codes || !q8 || !step2 || !mean) return QLORA_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(codes, 16) || !aligned(q8, 16) || !aligned(step2, 16) || !aligned(mean, 16))
    return QLORA_ERR_INVALID_ARG;
  if (rows < 1 || cols < 64 || cols % 64 != 0 || rows * cols > (1ll << 40)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  const QuantWs w = quant_ws(rows, cols);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < w.total) return QLORA_ERR_WORKSPACE;
  return launch_quantize(W, rows, cols, codes, q8, step2, mean, workspace, static_cast<cudaStream_t>(stream));
}

int qlora_quantize_shard_plan(int64_t n_blocks_total, int world, int rank, int64_t* block_begin,
                              int64_t* block_end, int64_t* roots_per_rank) {
  if (!block_begin || !block_end || !roots_per_rank) return QLORA_ERR_INVALID_ARG;
  if (n_blocks_total < 1 || n_blocks_total > (1ll << 34) || world < 1 || rank < 0 || rank >= world)
    return QLORA_ERR_INVALID_ARG;
  const int64_t chunks = cdiv(n_blocks_total, qnf4::kTreeChunk);
  const int64_t cpr = cdiv(chunks, world);
  *block_begin = std::min(n_blocks_total, static_cast<int64_t>(rank) * cpr * qnf4::kTreeChunk);
  *block_end = std::min(n_blocks_total, static_cast<int64_t>(rank + 1) * cpr * qnf4::kTreeChunk);
  *roots_per_rank = cpr;
  return QLORA_OK;
}

size_t qlora_quantize_shard_workspace_size(int64_t n_blocks_shard, int64_t n_roots_total) {
  if (n_blocks_shard < 0 || n_roots_total < 1) return static_cast<size_t>(-1);
  return shard_ws(n_blocks_shard, n_roots_total).total;
}

int qlora_quantize_nf4_shard_local(const float* W_shard, int64_t n_blocks_shard, uint8_t* codes_shard,
                                   double* roots, int64_t roots_per_rank, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  if (!roots || roots_per_rank < 1 || n_blocks_shard < 0) return QLORA_ERR_INVALID_ARG;
  if (n_blocks_shard > roots_per_rank * qnf4::kTreeChunk) return QLORA_ERR_INVALID_ARG;
  if (n_blocks_shard > 0 && (!W_shard || !codes_shard || !aligned(W_shard, 16) || !aligned(codes_shard, 16)))
    return QLORA_ERR_INVALID_ARG;
  if (!aligned(roots, 16)) return QLORA_ERR_INVALID_ARG;
  const ShardWs w = shard_ws(n_blocks_shard, roots_per_rank);
  // the block absmaxes and one ticket word (the rest of the workspace is the finishing call's)
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < w.tree_off + 256)
    return QLORA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  float* absmax = reinterpret_cast<float*>(base + w.absmax_off);
  const int64_t parts = cdiv(n_blocks_shard, qnf4::kTreeChunk);
  if (parts < roots_per_rank)                                       // chunks past the weight sum to zero
    QLORA_CUDA_TRY(cudaMemsetAsync(roots + parts, 0, static_cast<size_t>(roots_per_rank - parts) * 8, st));
  if (n_blocks_shard == 0) return QLORA_OK;
  // K1 resets its ticket word; the single first tree pass below does not
  // finish, so it neither reads nor moves a ticket.  Both live in the tree
  // area of the workspace, which the finishing call reuses.
  unsigned int* scratch_ticket = reinterpret_cast<unsigned int*>(base + w.tree_off);
  int rc = launch_blocks(W_shard, n_blocks_shard, codes_shard, absmax, scratch_ticket, tables(), st);
  if (rc != QLORA_OK) return rc;
  {
    LaunchTimer lt_("scale_mean_tree", st);
    qnf4::pairwise_tree_kernel<float><<<static_cast<unsigned>(parts), 256, 0, st>>>(
        absmax, n_blocks_shard, roots, 0, scratch_ticket, n_blocks_shard, nullptr, nullptr);
  }
  QLORA_CUDA_TRY(cudaGetLastError());
  return QLORA_OK;
}

int qlora_quantize_nf4_shard_finish(const double* roots_all, int64_t n_roots_total, int64_t n_blocks_total,
                                    int64_t n_blocks_shard, int8_t* q8_shard, float* step2_shard, float* mean,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  if (!roots_all || !mean || n_roots_total < 1 || n_blocks_total < 1 || n_blocks_shard < 0 ||
      n_blocks_shard > n_blocks_total || n_blocks_total > n_roots_total * qnf4::kTreeChunk)
    return QLORA_ERR_INVALID_ARG;
  if (!aligned(roots_all, 16) || !aligned(mean, 16)) return QLORA_ERR_INVALID_ARG;
  if (n_blocks_shard > 0 && (!q8_shard || !step2_shard || !aligned(q8_shard, 16) || !aligned(step2_shard, 16)))
    return QLORA_ERR_INVALID_ARG;
  const ShardWs w = shard_ws(n_blocks_shard, n_roots_total);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < w.total) return QLORA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  const float* absmax = reinterpret_cast<const float*>(base + w.absmax_off);
  double* tree = reinterpret_cast<double*>(base + w.tree_off);
  unsigned int* tickets = reinterpret_cast<unsigned int*>(base + w.ticket_off);
  QLORA_CUDA_TRY(cudaMemsetAsync(tickets, 0, 2 * sizeof(unsigned int), st));
  int rc = launch_mean_tree(roots_all, n_roots_total, tree, tickets, n_blocks_total, mean, st);
  if (rc != QLORA_OK || n_blocks_shard == 0) return rc;
  return launch_dq(absmax, n_blocks_shard, mean, q8_shard, step2_shard, st);
}

int qlora_merge_adapter(const qlora_nf4_weight* w, const uint16_t* A, const uint16_t* B, int r, float alpha,
                        uint16_t* W_out, void* stream) {
  if (!weight_ok(w) || !A || !B || !W_out || !aligned(A, 16) || !aligned(B, 16) || !aligned(W_out, 16))
    return QLORA_ERR_INVALID_ARG;
  if (!std::isfinite(alpha)) return QLORA_ERR_INVALID_ARG;
  if (r < 1 || r > 256 || w->rows < 64 || w->cols < 64 || w->rows % 64 != 0 || w->cols % 64 != 0 ||
      w->rows * w->cols > (1ll << 40))
    return QLORA_ERR_UNSUPPORTED_SHAPE;
  const float s = alpha / static_cast<float>(r);
  const int64_t tiles = (w->rows / qnf4::kMergeTileRows) * cdiv(w->cols, qnf4::kMergeTileCols);
  // a few CTAs per SM slot: each walks a run of tiles, long enough to reuse its staged A
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(tiles, device_sm_count() * 8)));
  const int smem = qnf4::merge_smem_bytes(r);
  QLORA_CUDA_TRY(set_max_smem(reinterpret_cast<const void*>(qnf4::merge_adapter_kernel), smem));
  {
    LaunchTimer lt_("merge_adapter", static_cast<cudaStream_t>(stream));
    qnf4::merge_adapter_kernel<<<grid, 256, smem, static_cast<cudaStream_t>(stream)>>>(
        w->codes, w->q8, w->step2, w->mean, A, B, r, s, w->rows, w->cols, W_out, tables().L);
  }
  QLORA_CUDA_TRY(cudaGetLastError());
  return QLORA_OK;
}

int qlora_dequantize_nf4(const qlora_nf4_weight* w, uint16_t* W_out, void* stream) {
  return qlora_dequantize_codebook(QLORA_CODEBOOK_NF4, w, W_out, stream);
}

int qlora_codebook(int kind, float levels[16], float thresholds[15]) {
  const Tables* t = tables_for(kind);
  if (t == nullptr || levels == nullptr) return QLORA_ERR_INVALID_ARG;
  std::memcpy(levels, t->L.v, sizeof(t->L.v));
  if (thresholds != nullptr) std::memcpy(thresholds, t->T.v, sizeof(t->T.v));
  return QLORA_OK;
}

int qlora_quantize_codebook(int kind, const float* W, int64_t rows, int64_t cols, uint8_t* codes, int8_t* q8,
                            float* step2, float* mean, void* workspace, size_t workspace_bytes, void* stream) {
  const Tables* tb = tables_for(kind);
  if (tb == nullptr) return QLORA_ERR_INVALID_ARG;
  if (!W || !codes || !q8 || !step2 || !mean) return QLORA_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(codes, 16) || !aligned(q8, 16) || !aligned(step2, 16) || !aligned(mean, 16))
    return QLORA_ERR_INVALID_ARG;
  if (rows < 1 || cols < 64 || cols % 64 != 0 || rows * cols > (1ll << 40)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  const QuantWs w = quant_ws(rows, cols);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < w.total) return QLORA_ERR_WORKSPACE;
  return launch_quantize(W, rows, cols, codes, q8, step2, mean, workspace, static_cast<cudaStream_t>(stream), *tb);
}

int qlora_dequantize_codebook(int kind, const qlora_nf4_weight* w, uint16_t* W_out, void* stream) {
  const Tables* tb = tables_for(kind);
  if (tb == nullptr) return QLORA_ERR_INVALID_ARG;
  if (!weight_ok(w) || !W_out || !aligned(W_out, 16)) return QLORA_ERR_INVALID_ARG;
  if (w->rows < 1 || w->cols < 64 || w->cols % 64 != 0 || w->rows * w->cols > (1ll << 40))
    return QLORA_ERR_UNSUPPORTED_SHAPE;
  const int64_t words = w->rows * w->cols / 8;
  const int64_t want = cdiv(words, 8 * 128 * qnf4::kDqRounds);        // 8 warps x 128 words x rounds per CTA
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(want, device_sm_count() * 8)));
  {
    LaunchTimer lt_("dequantize", static_cast<cudaStream_t>(stream));
    qnf4::nf4_dequantize_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      w->codes, w->q8, w->step2, w->mean, words, W_out, tb->L);
  }
  QLORA_CUDA_TRY(cudaGetLastError());
  return QLORA_OK;
}

int qlora_linear_fwd(const uint16_t* x, int64_t M, const qlora_nf4_weight* w, const uint16_t* A,
                     const uint16_t* B, int r, float alpha, uint16_t* h, uint16_t* us_out, void* workspace,
                     size_t workspace_bytes, void* stream) {
  const int sc = check_fwd_args(x, M, w, A, B, r, alpha, h, us_out);
  if (sc != QLORA_OK) return sc;
  const size_t need = fwd_ws(M, w->cols, w->rows, r);
  if (need > 0 && (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < need))
    return QLORA_ERR_WORKSPACE;
  return linear_fwd_any_rank(x, nullptr, M, w, A, B, r, alpha / static_cast<float>(r), h, us_out, workspace,
                             static_cast<cudaStream_t>(stream));
}

int qlora_linear_fwd_dropout(const uint16_t* x, int64_t M, const qlora_nf4_weight* w, const uint16_t* A,
                             const uint16_t* B, int r, float alpha, const uint8_t* keep_bits, float p, uint16_t* h,
                             uint16_t* us_out, void* workspace, size_t workspace_bytes, void* stream) {
  int sc = check_fwd_args(x, M, w, A, B, r, alpha, h, us_out);
  if (sc != QLORA_OK) return sc;
  if ((sc = check_dropout_args(keep_bits, p)) != QLORA_OK) return sc;
  const int64_t in = w->cols;
  const size_t need = fwd_dropout_ws(M, in, w->rows, r);
  if (need > 0 && (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < need))
    return QLORA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const float s_lora = (alpha / static_cast<float>(r)) / (1.f - p);
  return linear_fwd_any_rank(x, keep_bits, M, w, A, B, r, s_lora, h, us_out, workspace, st);
}

int qlora_linear_bwd(const uint16_t* dh, const uint16_t* x, const uint16_t* us, int64_t M,
                     const qlora_nf4_weight* w, const uint16_t* A, const uint16_t* B, int r, float alpha,
                     uint16_t* dx, float* dA, float* dB, void* workspace, size_t workspace_bytes, void* stream) {
  const int sc = check_bwd_args(dh, x, us, M, w, A, B, r, alpha, dx, dA, dB);
  if (sc != QLORA_OK) return sc;
  const BwdWs ws = bwd_ws(M, w->cols, w->rows, r);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < ws.total) return QLORA_ERR_WORKSPACE;
  return linear_bwd_any_rank(dh, x, us, M, w, A, B, r, alpha / static_cast<float>(r), nullptr, 1.f, dx, dA, dB,
                             workspace, static_cast<cudaStream_t>(stream));
}

int qlora_linear_bwd_dropout(const uint16_t* dh, const uint16_t* x, const uint16_t* us, int64_t M,
                             const qlora_nf4_weight* w, const uint16_t* A, const uint16_t* B, int r, float alpha,
                             const uint8_t* keep_bits, float p, uint16_t* dx, float* dA, float* dB, void* workspace,
                             size_t workspace_bytes, void* stream) {
  int sc = check_bwd_args(dh, x, us, M, w, A, B, r, alpha, dx, dA, dB);
  if (sc != QLORA_OK) return sc;
  if ((sc = check_dropout_args(keep_bits, p)) != QLORA_OK) return sc;
  const BwdWs ws = bwd_ws(M, w->cols, w->rows, r);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < ws.total) return QLORA_ERR_WORKSPACE;
  return linear_bwd_any_rank(dh, x, us, M, w, A, B, r, alpha / static_cast<float>(r), keep_bits, 1.f / (1.f - p), dx,
                             dA, dB, workspace, static_cast<cudaStream_t>(stream));
}

size_t qlora_linear_group_workspace_size(int backward, int n, const qlora_linear_problem* problems) {
  if (n < 0 || (n > 0 && problems == nullptr)) return static_cast<size_t>(-1);
  size_t total = 0;
  for (int i = 0; i < n; ++i) {
    const qlora_linear_problem& p = problems[i];
    if (!weight_ok(p.w) || p.M < 1 || p.r < 1) return static_cast<size_t>(-1);
    total += group_ws_each(backward != 0, p);
  }
  return total;
}

int qlora_linear_fwd_group(int n, const qlora_linear_problem* problems, void* workspace, size_t workspace_bytes,
                           void* stream) {
  if (n < 0 || (n > 0 && problems == nullptr)) return QLORA_ERR_INVALID_ARG;
  size_t need = 0;
  for (int i = 0; i < n; ++i) {
    const qlora_linear_problem& p = problems[i];
    const int sc = check_fwd_args(p.x, p.M, p.w, p.A, p.B, p.r, p.alpha, p.h, p.us);
    if (sc != QLORA_OK) return sc;
    need += group_ws_each(false, p);
  }
  if (n == 0) return QLORA_OK;
  if (need > 0 && (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < need))
    return QLORA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return group_issue(n, st, [&](cudaStream_t hi, cudaStream_t lo, cudaEvent_t* ev) -> int {
    // us_i = bf16(s x_i A_i^T) on the low-priority stream, then ev[i]
    auto rank_r = [&](int i) -> int {
      const qlora_linear_problem& p = problems[i];
      if (!group_split(p)) return QLORA_OK;
      const int rc = launch_rowwise<false>(p.x, p.A, p.us, p.M, p.w->cols, p.r, p.alpha / static_cast<float>(p.r), lo);
      if (rc != QLORA_OK) return rc;
      QLORA_CUDA_TRY(cudaEventRecord(ev[i], lo));
      return QLORA_OK;
    };
    int rc = rank_r(0);
    uint8_t* base = static_cast<uint8_t*>(workspace);
    for (int i = 0; i < n && rc == QLORA_OK; ++i) {
      const qlora_linear_problem& p = problems[i];
      const int64_t in = p.w->cols, out = p.w->rows;
      if (group_split(p)) {
        QLORA_CUDA_TRY(cudaStreamWaitEvent(hi, ev[i], 0));
        rc = launch_gemm(false, p.w, p.x, p.M, in, p.us, p.B, p.r, p.h, out, hi);   // h = [x|us] [W0|B]^T
      } else {
        rc = linear_fwd_any_rank(p.x, nullptr, p.M, p.w, p.A, p.B, p.r, p.alpha / static_cast<float>(p.r), p.h,
                                 p.us, base, hi);
      }
      base += group_ws_each(false, p);
      if (rc == QLORA_OK && i + 1 < n) rc = rank_r(i + 1);
    }
    return rc;
  });
}

int qlora_linear_bwd_group(int n, const qlora_linear_problem* problems, void* workspace, size_t workspace_bytes,
                           void* stream) {
  if (n < 0 || (n > 0 && problems == nullptr)) return QLORA_ERR_INVALID_ARG;
  size_t need = 0;
  for (int i = 0; i < n; ++i) {
    const qlora_linear_problem& p = problems[i];
    const int sc = check_bwd_args(p.dh, p.x, p.us, p.M, p.w, p.A, p.B, p.r, p.alpha, p.dx, p.dA, p.dB);
    if (sc != QLORA_OK) return sc;
    need += group_ws_each(true, p);
  }
  if (n == 0) return QLORA_OK;
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < need) return QLORA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  std::vector<uint8_t*> ws(n);
  {
    uint8_t* base = static_cast<uint8_t*>(workspace);
    for (int i = 0; i < n; ++i) {
      ws[i] = base;
      base += group_ws_each(true, problems[i]);
    }
  }
  return group_issue(n, st, [&](cudaStream_t hi, cudaStream_t lo, cudaEvent_t* ev) -> int {
    // du_i = bf16(s dh_i B_i) into projection i's workspace, then ev[i]
    auto du_of = [&](int i) { return reinterpret_cast<uint16_t*>(ws[i] + bwd_ws(problems[i].M, problems[i].w->cols,
                                                                                  problems[i].w->rows,
                                                                                  problems[i].r).du_off); };
    auto rank_r = [&](int i) -> int {
      const qlora_linear_problem& p = problems[i];
      if (!group_split(p)) return QLORA_OK;
      const int rc = launch_rowwise<true>(p.dh, p.B, du_of(i), p.M, p.w->rows, p.r, p.alpha / static_cast<float>(p.r),
                                          lo);
      if (rc != QLORA_OK) return rc;
      QLORA_CUDA_TRY(cudaEventRecord(ev[i], lo));
      return QLORA_OK;
    };
    int rc = rank_r(0);
    for (int i = 0; i < n && rc == QLORA_OK; ++i) {
      const qlora_linear_problem& p = problems[i];
      const int64_t in = p.w->cols, out = p.w->rows;
      if (group_split(p)) {
        QLORA_CUDA_TRY(cudaStreamWaitEvent(hi, ev[i], 0));
        rc = launch_gemm(true, p.w, p.dh, p.M, out, du_of(i), p.A, p.r, p.dx, in, hi);   // dx = [dh|du][W0;A]
        if (rc == QLORA_OK && i + 1 < n) rc = rank_r(i + 1);                             // next du first
        if (rc == QLORA_OK)
          rc = launch_lora_grads(p.dh, p.us, p.x, du_of(i), p.M, in, out, p.r, p.dB, p.dA, lo);   // dB, dA
      } else {
        rc = linear_bwd_any_rank(p.dh, p.x, p.us, p.M, p.w, p.A, p.B, p.r, p.alpha / static_cast<float>(p.r), nullptr,
                                 1.f, p.dx, p.dA, p.dB, ws[i], hi);
        if (rc == QLORA_OK && i + 1 < n) rc = rank_r(i + 1);
      }
    }
    return rc;
  });
}

int qlora_last_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return QLORA_ERR_CUDA;
  int flag = 0;
  if (cudaMemcpyFromSymbol(&flag, qnf4::g_device_error, sizeof(int)) != cudaSuccess) return QLORA_ERR_CUDA;
  if (flag != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(qnf4::g_device_error, &zero, sizeof(int)) != cudaSuccess) return QLORA_ERR_CUDA;
    return QLORA_ERR_TIMEOUT;
  }
  return QLORA_OK;
}

uint64_t qlora_set_wait_timeout_ns(uint64_t ns) {
  if (ns < 1000) ns = 1000;
  return g_timeout_ns.exchange(ns);
}

int qlora_selftest_wait_timeout(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  qnf4::wait_timeout_selftest_kernel<<<1, 32, 0, st>>>(g_timeout_ns.load());
  if (cudaGetLastError() != cudaSuccess) return QLORA_ERR_CUDA;
  return qlora_last_device_status(stream);
}

int qlora_timing_enable(int on) { return g_timing_on.exchange(on != 0 ? 1 : 0); }

void qlora_timing_reset(void) {
  std::lock_guard<std::mutex> lk(g_timing_mu);
  for (auto& t : g_timed) {
    g_event_pool.push_back(t.start);
    g_event_pool.push_back(t.stop);
  }
  g_timed.clear();
}

int qlora_timing_collect(const char* kernel, double* total_ms, int64_t* launches) {
  if (kernel == nullptr) return QLORA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_timing_mu);
  double sum = 0.0;
  int64_t n = 0;
  for (auto& t : g_timed) {
    if (std::strcmp(t.name, kernel) != 0) continue;
    if (cudaEventSynchronize(t.stop) != cudaSuccess) return QLORA_ERR_CUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, t.start, t.stop) != cudaSuccess) return QLORA_ERR_CUDA;
    sum += ms;
    ++n;
  }
  if (total_ms) *total_ms = sum;
  if (launches) *launches = n;
  return QLORA_OK;
}

const char* qlora_status_string(int status) {
  switch (status) {
    case QLORA_OK: return "ok";
    case QLORA_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, bad scalar)";
    case QLORA_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case QLORA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case QLORA_ERR_CUDA: return "CUDA error";
    case QLORA_ERR_TIMEOUT: return "a device-side wait timed out";
    case QLORA_ERR_SCRATCH_LIMIT: return "size exceeds the fixed scratch of the no-allocation entry point";
    default: return "unknown status";
  }
}

}  // extern "C"

// ============================================================================
// No-allocation quantizer: the scratch of qlora_quantize_nf4 in a fixed
// device array of this library instead of a caller workspace.
namespace {

constexpr int64_t kNoAllocMaxBlocks = QLORA_NOALLOC_MAX_BLOCKS;
constexpr size_t kNoAllocScratchBytes =
    ((static_cast<size_t>(kNoAllocMaxBlocks) * 4 + 255) & ~static_cast<size_t>(255)) +
    ((static_cast<size_t>(kNoAllocMaxBlocks / qnf4::kTreeChunk + 1) * 8 + 255) & ~static_cast<size_t>(255)) + 256;

// The largest tensor the array accepts fits the quantizer's scratch layout
// (block absmaxes, every tree pass's sums, the ticket words).
static_assert(quant_ws(1, kNoAllocMaxBlocks * 64).total <= kNoAllocScratchBytes,
              "the no-allocation scratch is smaller than the quantizer's workspace at its maximum size");
static_assert(quant_ws(kNoAllocMaxBlocks / 4096, 4096 * 64).total <= kNoAllocScratchBytes,
              "the no-allocation scratch is smaller than the quantizer's workspace at its maximum size");

// One copy per device that loads the library.  In host code this name is a
// host-side stand-in, never a device address: the address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Identifier of the calling thread's current CUDA context (0 if unknown).
unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(p);
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

std::mutex g_noalloc_mu;
struct NoAllocAddr {
  void* ptr;
  unsigned long long ctx;   // context the address belongs to
};
NoAllocAddr g_noalloc_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (with that device current) and again only if the device's
// context was replaced since (a reset destroys the module and its array).
void* noalloc_scratch_for_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  const unsigned long long ctx = current_context_id();      // 0 before the runtime made a context current
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  NoAllocAddr& e = g_noalloc_addr[dev];
  if (e.ptr == nullptr || ctx == 0 || e.ctx != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    e.ptr = p;
    e.ctx = current_context_id();                           // the lookup made the context current
  }
  return e.ptr;
}

}  // namespace

extern "C" int qlora_quantize_nf4_noalloc(const float* W, int64_t rows, int64_t cols, uint8_t* codes,
                                          int8_t* q8, float* step2, float* mean, void* stream) {
  if (!W || !codes || !q8 || !step2 || !mean) return QLORA_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(codes, 16) || !aligned(q8, 16) || !aligned(step2, 16) || !aligned(mean, 16))
    return QLORA_ERR_INVALID_ARG;
  if (rows < 1 || cols < 64 || cols % 64 != 0 || rows * cols > (1ll << 40)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (rows * cols / 64 > kNoAllocMaxBlocks) return QLORA_ERR_SCRATCH_LIMIT;
  if (quant_ws(rows, cols).total > kNoAllocScratchBytes) return QLORA_ERR_SCRATCH_LIMIT;
  void* scratch = noalloc_scratch_for_current_device();
  if (scratch == nullptr) return QLORA_ERR_CUDA;
  return launch_quantize(W, rows, cols, codes, q8, step2, mean, scratch, static_cast<cudaStream_t>(stream));
}

