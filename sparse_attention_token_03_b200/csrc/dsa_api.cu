// C ABI of libdsa_index.so: argument validation, workspace layout, TMA
// descriptor encoding and kernel launches.  Declarations and the contract of
// every entry point live in include/dsa_index.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/dsa_index.h"
#include "dsa_dosa.cuh"
#include "dsa_kernels.cuh"
#include "dsa_ptx.cuh"

using namespace dsa;

namespace {

thread_local std::string g_last_error = "no error";

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(DSA_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// bf16 matrix [rows][128] read as tiles of box_rows x 64 columns, 128B swizzle.
int make_tmap(CUtensorMap* m, const void* base, int64_t rows, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(DSA_ECUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(kD) * 2};
  cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DSA_ECUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return DSA_OK;
}

// FP8 matrix [rows][128] of E4M3 codes read as tiles of box_rows x 128
// codes (one 128-byte row each), 128B swizzle.
int make_tmap_u8(CUtensorMap* m, const void* base, int64_t rows, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(DSA_ECUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(kD)};
  cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DSA_ECUDA, "cuTensorMapEncodeTiled (u8) failed (%d)", static_cast<int>(r));
  return DSA_OK;
}

// Workspace of dsa_index_seeds_from_history: status word, control words,
// count histogram and counts (one memset clears all four), tile prefixes.
struct HistoryPlan {
  size_t off_ctl, off_hist, off_counts, off_tile_gt, off_tile_eq, zero_bytes, bytes;
};

HistoryPlan plan_history(int64_t n_keys) {
  HistoryPlan P{};
  const size_t n_tiles = static_cast<size_t>((n_keys + 1023) / 1024);
  P.off_ctl = 64;
  P.off_hist = 256;
  P.off_counts = P.off_hist + 65536 * 4;
  size_t off = P.off_counts + static_cast<size_t>(n_keys) * 4;
  P.zero_bytes = off;
  off = (off + 255) / 256 * 256;
  P.off_tile_gt = off;
  off = (off + n_tiles * 4 + 255) / 256 * 256;
  P.off_tile_eq = off;
  P.bytes = (off + n_tiles * 4 + 255) / 256 * 256;
  return P;
}

int sm_count() {
  // per-device cache; host threads may race on it harmlessly (atomic, and
  // every writer stores the same value)
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64) {
    const int c = cached[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 148;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (dev >= 0 && dev < 64) cached[dev].store(n, std::memory_order_relaxed);
  return n;
}

// Optional per-kernel timing: when enabled, every entry point records a CUDA
// event on its stream before its first launch and after each launch.
constexpr int kProfileEvents = 32;
struct Profile {
  bool enabled = false;
  int n = 0;
  cudaEvent_t ev[kProfileEvents] = {};
  const char* name[kProfileEvents] = {};
};
thread_local Profile g_prof;

void prof_begin(cudaStream_t st) {
  if (!g_prof.enabled) return;
  g_prof.n = 0;
  if (!g_prof.ev[0]) cudaEventCreate(&g_prof.ev[0]);
  cudaEventRecord(g_prof.ev[0], st);
  g_prof.name[0] = "begin";
  g_prof.n = 1;
}

void prof_mark(cudaStream_t st, const char* kernel) {
  if (!g_prof.enabled || g_prof.n >= kProfileEvents) return;
  cudaEvent_t& e = g_prof.ev[g_prof.n];
  if (!e) cudaEventCreate(&e);
  cudaEventRecord(e, st);
  g_prof.name[g_prof.n] = kernel;
  ++g_prof.n;
}

// One-shot failure injection armed by dsa_test_inject_wait_timeout (per
// host thread): the next fused-kernel launch withholds its loads and limits
// its pipeline waits, so that a wait runs out on the device.
struct WaitInjection {
  bool armed = false;
  uint64_t limit_ns = 0;
};
thread_local WaitInjection g_inject;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_shape(int H, int d, int topk) {
  if (d != kD) return fail(DSA_EUNSUPPORTED, "d = %d: only d = 128 is supported", d);
  if (H != 32 && H != 64) return fail(DSA_EUNSUPPORTED, "H = %d: only H = 32 or 64 is supported", H);
  if (topk < 1 || topk > kMaxTopk) return fail(DSA_EUNSUPPORTED, "topk = %d outside [1, %d]", topk, kMaxTopk);
  return DSA_OK;
}


// ----------------------------------------------------------------- prefill
struct PrefillPlan {
  int G, n_groups, S, n_units, grid;
  int eg;  // epilogue warpgroups of the fused kernel (2 or 4)
  CandLayout lay;
  size_t off_meta, off_cand, bytes;
};

PrefillPlan plan_prefill(int64_t T_q, int64_t T_k, int64_t q_offset_hint, int H, int topk, int G = 0,
                         int max_s = 64) {
  PrefillPlan P{};
  P.G = G > 0 ? G : 256 / H;
  P.n_groups = static_cast<int>((T_q + P.G - 1) / P.G);
  const int sms = sm_count();
  P.S = 1;
  if (P.n_groups > 0 && P.n_groups < sms) {
    // few long rows: split each group's keys so that every SM has work
    const int64_t min_keys = std::max<int64_t>(q_offset_hint + 1, 1);
    const int64_t tiles = (min_keys + kTileKeys - 1) / kTileKeys;
    const int want = (sms + P.n_groups - 1) / P.n_groups;
    P.S = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(want, tiles / 16)));
    P.S = std::min(P.S, std::max(max_s, 1));
  }
  P.n_units = P.n_groups * P.S;
  // Epilogue width: four warpgroups (one query each at H = 64) hide the
  // admission work and keep 16 weights per thread in registers; only for
  // units of very many keys per selected record, where admissions are rare
  // and the head sums dominate, two warpgroups with all head weights in
  // registers are used.
  const double unit_keys = (static_cast<double>(std::max<int64_t>(q_offset_hint, 0)) +
                            0.5 * static_cast<double>(T_q + 1)) / P.S;
  P.eg = unit_keys >= static_cast<double>(kWideKeysPerRecord) * topk ? 2 : 4;
  P.lay = cand_layout(topk);
  P.grid = std::max(1, std::min(sms, P.n_units));
  size_t off = 256;  // device status word
  P.off_meta = off;
  off = align_up(off + static_cast<size_t>(P.n_units) * P.G * kMetaInts * sizeof(int32_t), 256);
  P.off_cand = off;
  off = align_up(off + static_cast<size_t>(P.n_units) * P.G * P.lay.query_recs() * sizeof(uint64_t), 256);
  P.bytes = off;
  (void)T_k;
  return P;
}

// ----------------------------------------------------------------- decode
struct DecodePlan {
  int grid, units_max;
  CandLayout lay;
  size_t off_seq_start, off_unit_tab, off_cta_ubeg, off_seq_ubeg, off_seq_ucnt, off_meta, off_cand,
      bytes;
};

constexpr size_t align_c(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace layout of a batched decode of B sequences run on `grid` CTAs.
// (g_rows > 1: each unit scores g_rows consecutive rows, the shared refine
// stream's groups)
constexpr DecodePlan plan_decode_layout(int B, int topk, int grid, int g_rows = 1) {
  DecodePlan P{};
  P.grid = grid;
  P.units_max = P.grid + B;
  P.lay = cand_layout(topk);
  size_t off = 256;
  P.off_seq_start = off;
  off = align_c(off + static_cast<size_t>(B + 1) * sizeof(int64_t), 256);
  P.off_unit_tab = off;
  off = align_c(off + static_cast<size_t>(P.units_max) * 3 * sizeof(int32_t), 256);
  P.off_cta_ubeg = off;
  off = align_c(off + static_cast<size_t>(P.grid + 1) * sizeof(int32_t), 256);
  P.off_seq_ubeg = off;
  off = align_c(off + static_cast<size_t>(B) * sizeof(int32_t), 256);
  P.off_seq_ucnt = off;
  off = align_c(off + static_cast<size_t>(B) * sizeof(int32_t), 256);
  P.off_meta = off;
  off = align_c(off + static_cast<size_t>(P.units_max) * g_rows * kMetaInts * sizeof(int32_t), 256);
  P.off_cand = off;
  off = align_c(off + static_cast<size_t>(P.units_max) * g_rows * P.lay.query_recs() * sizeof(uint64_t), 256);
  P.bytes = off;
  return P;
}

DecodePlan plan_decode(int B, int topk) { return plan_decode_layout(B, topk, std::min(sm_count(), 1024)); }

int check_decode_args(const uint16_t* q, const float* w, const uint16_t* k_cache,
                      const int32_t* seq_len, int B, int64_t t_cap, int H, int d, int topk,
                      int32_t* out_idx, float* out_score) {
  int rc = check_shape(H, d, topk);
  if (rc != DSA_OK) return rc;
  if (B < 1 || B > 65536 || t_cap < 0) return fail(DSA_EINVAL, "need 1 <= B <= 65536 and t_cap >= 0");
  if (static_cast<int64_t>(B) * std::max<int64_t>(t_cap, 1) >= (int64_t(1) << 31))
    return fail(DSA_EINVAL, "B * t_cap must be below 2^31");
  if (!q || !w || !k_cache || !seq_len || !out_idx || !out_score)
    return fail(DSA_EINVAL, "null pointer argument");
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(w, 4) || !aligned(seq_len, 4) ||
      !aligned(out_idx, 4) || !aligned(out_score, 4))
    return fail(DSA_EINVAL, "misaligned pointer (q and k_cache need 16 bytes)");
  return DSA_OK;
}

// The decode path proper (arguments already validated): planner, fused score
// kernel and final selection, all on `st`, scratch in `ws` laid out by P.
// A paged key cache: the page pool [n_pages][page_size][128] and the
// sequences' block tables [B][max_blocks].
struct PagedKeys {
  const int32_t* block_table;
  int max_blocks;
  int page_size;
  int64_t n_pages;
};

int decode_run(const uint16_t* q, const float* w, const uint16_t* k_cache, const int32_t* seq_len,
               int B, int64_t t_cap, int H, int topk, int32_t* out_idx, float* out_score,
               uint8_t* ws, const DecodePlan& P, bool profile, cudaStream_t st, const PagedKeys* paged = nullptr) {
  int rc;
  CUtensorMap tq, tk;
  if ((rc = make_tmap(&tq, q, static_cast<int64_t>(B) * H, H)) != DSA_OK) return rc;
  if (paged) {
    // pages of a multiple of 128 keys hold whole key tiles (128-row boxes);
    // 64-key pages split a tile's halves over two pages (64-row boxes)
    const int box = paged->page_size % kTileKeys == 0 ? kTileKeys : 64;
    if ((rc = make_tmap(&tk, k_cache, paged->n_pages * paged->page_size, box)) != DSA_OK) return rc;
  } else if ((rc = make_tmap(&tk, k_cache, std::max<int64_t>(static_cast<int64_t>(B) * t_cap, 1), kTileKeys)) !=
             DSA_OK) {
    return rc;
  }
  cudaError_t e = cudaMemsetAsync(ws, 0, 4, st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  if (profile) prof_begin(st);

  DecodePlanParams dp{};
  dp.B = B;
  dp.grid = P.grid;
  dp.t_cap = t_cap;
  dp.seq_len = seq_len;
  dp.seq_start = reinterpret_cast<int64_t*>(ws + P.off_seq_start);
  dp.unit_tab = reinterpret_cast<int32_t*>(ws + P.off_unit_tab);
  dp.cta_ubeg = reinterpret_cast<int32_t*>(ws + P.off_cta_ubeg);
  dp.seq_ubeg = reinterpret_cast<int32_t*>(ws + P.off_seq_ubeg);
  dp.seq_ucnt = reinterpret_cast<int32_t*>(ws + P.off_seq_ucnt);
  dp.err = reinterpret_cast<uint32_t*>(ws);
  if ((e = launch_decode_plan(dp, st)) != cudaSuccess) return cuda_fail(e, "decode plan launch");
  if (profile) prof_mark(st, "decode_plan");

  ScoreParams sp{};
  sp.mode = kModeDecode;
  sp.topk = topk;
  sp.lay = P.lay;
  sp.S = 1;
  sp.t_cap = t_cap;
  sp.w = w;
  sp.seq_len = seq_len;
  sp.unit_tab = dp.unit_tab;
  sp.cta_ubeg = dp.cta_ubeg;
  sp.cand = reinterpret_cast<uint64_t*>(ws + P.off_cand);
  sp.meta = reinterpret_cast<int32_t*>(ws + P.off_meta);
  sp.err = dp.err;
  if (paged) {
    sp.block_table = paged->block_table;
    sp.max_blocks = paged->max_blocks;
    sp.page_size = paged->page_size;
    sp.n_pages = paged->n_pages;
  }
  if ((e = launch_score(H, 1, 1, tq, tk, sp, P.grid, st)) != cudaSuccess) return cuda_fail(e, "score kernel launch");
  if (profile) prof_mark(st, "score_topk");

  SelectParams se{};
  se.mode = kModeDecode;
  se.G = 1;
  se.S = 1;
  se.topk = topk;
  se.lay = P.lay;
  se.n_rows = B;
  se.cand = sp.cand;
  se.meta = sp.meta;
  se.seq_ubeg = dp.seq_ubeg;
  se.seq_ucnt = dp.seq_ucnt;
  se.out_idx = out_idx;
  se.out_score = out_score;
  se.err = dp.err;
  if ((e = launch_select(se, st)) != cudaSuccess) return cuda_fail(e, "select kernel launch");
  if (profile) prof_mark(st, "select_topk");
  return DSA_OK;
}

// ---------------------------------------------------------------------------
// Workspace of the pruned (DoSA) prefill.
//
// The chunk's first probe rows always take the pruned path; from their
// survivor counts a device-side decision (decide_kernel) either lets the
// remaining rows take it too or marks them for the dense pass, so that the
// call never costs much more than the dense one on inputs where the bound
// filters little.  Nothing synchronises with the host.
// ---------------------------------------------------------------------------
constexpr int64_t kProbeRows = 64;  // a multiple of every query group size (4, 8)

struct PrunedPlan {
  int64_t probe;          // rows of the probe (all rows of a short chunk)
  PrefillPlan seed[2];    // seed scoring of the probe rows / the remaining rows
  PrefillPlan screen[2];  // screening geometry (16 plan rows per query), same split
  PrefillPlan dense;      // exact dense pass over flagged rows
  DecodePlan refine;      // refine: one "sequence" of survivors per row
  DecodePlan refine2;     // shared refine stream: one "sequence" per group of four rows
  int64_t n_groups;
  int cap_row;            // survivor ids kept per row
  int rec_stride;         // seed records per row (topk rounded up to even)
  int64_t mask_words;
  size_t off_stats, off_ctl, off_seed_bits, off_k_seed, off_cand, off_seed_rec, off_tau, off_plan_q, off_plan_s,
      off_knorm, off_bitmask, off_surv_count, off_surv_ids, off_refine_len, off_row_flags, off_init_thr,
      off_refine, off_group_mask, off_group_ids, off_group_len, off_refine2, bytes;
};

int pruned_cap_row(int64_t T_k, int topk) {
  // survivor lists hold up to a sixteenth of the keys: a row with more
  // survivors is cheaper to recompute densely than to refine key by key
  const int64_t c = std::max<int64_t>(T_k / 16, 4 * static_cast<int64_t>(topk));
  return static_cast<int>(std::min<int64_t>(std::min<int64_t>(c, T_k), int64_t(1) << 30));
}

PrunedPlan plan_pruned(int64_t T_q, int64_t T_k, int64_t q_offset, int H, int topk, int n_seed) {
  PrunedPlan P{};
  P.probe = T_q > 2 * kProbeRows ? kProbeRows : T_q;
  const int64_t rows[2] = {P.probe, T_q - P.probe};
  for (int i = 0; i < 2; ++i) {
    // a seed-scoring split needs a few times topk keys, or its streaming
    // threshold never rises and the seed select merges every seed record
    P.seed[i] = plan_prefill(rows[i], n_seed, n_seed - 1, H, topk, 0, n_seed / (2 * topk));
    P.screen[i] = plan_prefill(rows[i], T_k, q_offset + (i ? P.probe : 0), kPlanRows, topk, kScreenQueries);
  }
  P.dense = plan_prefill(T_q, T_k, q_offset, H, topk);
  P.refine = plan_decode(static_cast<int>(T_q), topk);
  P.n_groups = (T_q + 3) / 4;
  P.refine2 = plan_decode_layout(static_cast<int>(P.n_groups), topk, std::min(sm_count(), 1024), 4);
  P.cap_row = pruned_cap_row(T_k, topk);
  P.rec_stride = (topk + 1) & ~1;
  P.mask_words = (T_k + 31) / 32;
  size_t off = 256;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  P.off_stats = take(8 * sizeof(unsigned long long));
  P.off_ctl = take(8 * sizeof(uint32_t));
  P.off_seed_bits = take(static_cast<size_t>(P.mask_words) * 4);
  P.off_k_seed = take(static_cast<size_t>(n_seed) * kD * 2);
  // seed scoring and the dense pass run at different times and share one area
  P.off_cand = take(std::max({P.seed[0].bytes, P.seed[1].bytes, P.dense.bytes}));
  P.off_seed_rec = take(static_cast<size_t>(T_q) * P.rec_stride * 8);
  P.off_tau = take(static_cast<size_t>(T_q) * 4);
  P.off_plan_q = take(static_cast<size_t>(T_q) * kPlanRows * kD * 2);
  P.off_plan_s = take(static_cast<size_t>(T_q) * kPlanScalars * 4);
  P.off_knorm = take(static_cast<size_t>(T_k) * 4);
  P.off_bitmask = take(static_cast<size_t>(T_q) * P.mask_words * 4);
  P.off_surv_count = take(static_cast<size_t>(T_q) * 4);
  P.off_surv_ids = take(static_cast<size_t>(T_q) * P.cap_row * 4);
  P.off_refine_len = take(static_cast<size_t>(T_q) * 4);
  P.off_row_flags = take(static_cast<size_t>(T_q) * 4);
  P.off_init_thr = take(static_cast<size_t>(T_q) * 8);
  P.off_refine = take(P.refine.bytes);
  P.off_group_mask = take(static_cast<size_t>(P.n_groups) * P.mask_words * 4);
  P.off_group_ids = take(static_cast<size_t>(P.n_groups) * P.cap_row * 4);
  P.off_group_len = take(static_cast<size_t>(P.n_groups) * 4);
  P.off_refine2 = take(P.refine2.bytes);
  P.bytes = off;
  return P;
}

// Seed scoring, plan, screen and compaction of the n rows starting at r0 of
// a pruned call (i = 0: the probe rows, i = 1: the rest of the chunk).
// skip (device, may be null): every launch does nothing while the word is set.
int pruned_rows(const PrunedPlan& P, int i, int64_t r0, int64_t n, const uint16_t* q, const float* w,
                int64_t q_offset, int64_t T_k, int H, int topk, const int32_t* seed_idx, int n_seed,
                const CUtensorMap& tk, uint8_t* ws, const uint32_t* skip, cudaStream_t st) {
  if (n <= 0) return DSA_OK;
  int rc;
  cudaError_t e;
  uint32_t* err = reinterpret_cast<uint32_t*>(ws);
  auto at = [&](size_t off) { return ws + off; };
  const uint16_t* qr = q + static_cast<size_t>(r0) * H * kD;
  const float* wr = w + static_cast<size_t>(r0) * H;
  const PrefillPlan& SP = P.seed[i];
  const PrefillPlan& CP = P.screen[i];
  float* tau = reinterpret_cast<float*>(at(P.off_tau)) + r0;
  uint64_t* seed_rec = reinterpret_cast<uint64_t*>(at(P.off_seed_rec)) + r0 * P.rec_stride;
  uint16_t* plan_q = reinterpret_cast<uint16_t*>(at(P.off_plan_q)) + r0 * kPlanRows * kD;
  float* plan_s = reinterpret_cast<float*>(at(P.off_plan_s)) + r0 * kPlanScalars;
  uint32_t* bitmask = reinterpret_cast<uint32_t*>(at(P.off_bitmask)) + r0 * P.mask_words;
  int32_t* surv_count = reinterpret_cast<int32_t*>(at(P.off_surv_count)) + r0;
  CUtensorMap tq, tks, tplan;
  if ((rc = make_tmap(&tq, qr, n * H, SP.G * H)) != DSA_OK) return rc;
  if ((rc = make_tmap(&tks, at(P.off_k_seed), n_seed, kTileKeys)) != DSA_OK) return rc;
  if ((rc = make_tmap(&tplan, plan_q, n * kPlanRows, CP.G * kPlanRows)) != DSA_OK) return rc;
  // seed scores with all heads; per row: sorted seed Top-k records and tau
  ScoreParams s1{};
  s1.mode = kModeGathered;
  s1.topk = topk;
  s1.lay = SP.lay;
  s1.S = SP.S;
  s1.n_groups = SP.n_groups;
  s1.n_units = SP.n_units;
  s1.T_q = n;
  s1.T_k = n_seed;
  s1.w = wr;
  s1.key_ids = seed_idx;
  s1.cand = reinterpret_cast<uint64_t*>(at(P.off_cand + SP.off_cand));
  s1.meta = reinterpret_cast<int32_t*>(at(P.off_cand + SP.off_meta));
  s1.err = err;
  s1.skip = skip;
  if ((e = launch_score(H, SP.G, SP.eg, tq, tks, s1, SP.grid, st)) != cudaSuccess)
    return cuda_fail(e, "seed score launch");
  prof_mark(st, "seed_score");
  SelectParams s2{};
  s2.mode = kModePrefill;
  s2.G = SP.G;
  s2.S = SP.S;
  s2.topk = topk;
  s2.lay = SP.lay;
  s2.n_rows = n;
  s2.cand = s1.cand;
  s2.meta = s1.meta;
  s2.out_rec = seed_rec;
  s2.rec_stride = P.rec_stride;
  s2.out_kth = tau;
  s2.err = err;
  s2.skip = skip;
  if ((e = launch_select(s2, st)) != cudaSuccess) return cuda_fail(e, "seed select launch");
  prof_mark(st, "seed_select");
  // screening plan per row
  PlanParams pp{qr, wr, reinterpret_cast<const uint16_t*>(at(P.off_k_seed)), n_seed, n, tau, plan_q, plan_s, skip};
  if ((e = launch_plan(H, pp, st)) != cudaSuccess) return cuda_fail(e, "plan launch");
  prof_mark(st, "plan");
  // screen every visible non-seed key: bound -> survivor bitmask
  ScoreParams s3{};
  s3.mode = kModePrefill;
  s3.topk = topk;
  s3.lay = CP.lay;
  s3.S = CP.S;
  s3.n_groups = CP.n_groups;
  s3.n_units = CP.n_units;
  s3.q_offset = q_offset + r0;
  s3.T_q = n;
  s3.T_k = T_k;
  s3.err = err;
  s3.plan_s = plan_s;
  s3.knorm = reinterpret_cast<const float*>(at(P.off_knorm));
  s3.seed_bits = reinterpret_cast<const uint32_t*>(at(P.off_seed_bits));
  s3.bitmask = bitmask;
  s3.mask_words = P.mask_words;
  s3.surv_count = surv_count;
  s3.skip = skip;
  if ((e = launch_screen(tplan, tk, s3, CP.grid, st)) != cudaSuccess) return cuda_fail(e, "screen launch");
  prof_mark(st, "screen");
  // the shared refine stream of every full group of four rows (r0 is a
  // multiple of four), then the rows' own id lists without those keys; rows
  // whose survivors overflow are flagged
  uint32_t* gmask = reinterpret_cast<uint32_t*>(at(P.off_group_mask)) + (r0 / 4) * P.mask_words;
  int32_t* glen = reinterpret_cast<int32_t*>(at(P.off_group_len)) + r0 / 4;
  ShareParams sh{n, q_offset + r0, bitmask, P.mask_words, surv_count, P.cap_row, gmask,
                 reinterpret_cast<int32_t*>(at(P.off_group_ids)) + (r0 / 4) * P.cap_row, glen, err, skip};
  if ((e = launch_share(sh, st)) != cudaSuccess) return cuda_fail(e, "share launch");
  prof_mark(st, "share");
  CompactParams cp{n, q_offset + r0, topk, bitmask, P.mask_words, surv_count, P.cap_row,
                   reinterpret_cast<int32_t*>(at(P.off_surv_ids)) + r0 * P.cap_row,
                   reinterpret_cast<int32_t*>(at(P.off_refine_len)) + r0,
                   reinterpret_cast<int32_t*>(at(P.off_row_flags)) + r0, seed_rec, P.rec_stride,
                   reinterpret_cast<uint64_t*>(at(P.off_init_thr)) + r0, err, skip, gmask, glen};
  if ((e = launch_compact(cp, st)) != cudaSuccess) return cuda_fail(e, "compact launch");
  prof_mark(st, "compact");
  return DSA_OK;
}

// ---------------------------------------------------------------------------
// Scratch for dsa_index_decode_noalloc.  The array lives in the library's
// device image, so every GPU on which the library's kernels are loaded holds
// it (36,827,136 bytes, about 37 MB) until the process exits.  Host code must
// not hand the symbol itself to a kernel: on the host it only names a
// stand-in; the device address comes from cudaGetSymbolAddress, looked up on
// every call with the caller's device current (cheap, not a stream
// operation), so that a context that was torn down and re-created never
// leaves a stale address behind.
// ---------------------------------------------------------------------------
constexpr int kNoAllocMaxB = 64;      // largest batch served from the static scratch
constexpr int kNoAllocMaxGrid = 160;  // persistent CTAs used by that path (<= SMs)
constexpr size_t kNoAllocScratchBytes = plan_decode_layout(kNoAllocMaxB, kMaxTopk, kNoAllocMaxGrid).bytes;
// the header states this size; keep the two in step
static_assert(kNoAllocScratchBytes == 36827136, "static decode scratch size changed: update dsa_index.h");

__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the static scratch on the current device.
int noalloc_scratch(void** out) {
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || p == nullptr) return cuda_fail(e, "cudaGetSymbolAddress(static decode scratch)");
  *out = p;
  return DSA_OK;
}

// Paged prefill: the caller's workspace holds, in order, the workspace of
// the contiguous call, the page gather's status word (256 bytes) and the
// gathered keys [T_k][128] bf16.  The contiguous call's status word stays at
// byte 0, where dsa_index_device_status reads it.
size_t paged_tail_bytes(int64_t T_k) { return 256 + align_up(static_cast<size_t>(T_k) * kD * 2, 256); }

int check_paged_pool(const uint16_t* k_pages, int64_t n_pages, int page_size, const int32_t* block_table) {
  if (!k_pages || !block_table) return fail(DSA_EINVAL, "null pointer argument");
  if (n_pages < 1 || page_size < 1) return fail(DSA_EINVAL, "need n_pages >= 1 and page_size >= 1");
  if (n_pages * page_size >= (int64_t(1) << 31)) return fail(DSA_EINVAL, "n_pages * page_size must be below 2^31");
  if (!aligned(k_pages, 16) || !aligned(block_table, 4))
    return fail(DSA_EINVAL, "misaligned pointer (k_pages needs 16 bytes)");
  return DSA_OK;
}

// Gathers the sequence's first T_k keys behind the contiguous workspace of
// inner_bytes; returns the key matrix through *keys.
int gather_paged_keys(const uint16_t* k_pages, int64_t n_pages, int page_size, const int32_t* block_table,
                      int64_t T_k, uint8_t* ws, size_t inner_bytes, uint16_t** keys, cudaStream_t st) {
  uint32_t* gst = reinterpret_cast<uint32_t*>(ws + inner_bytes);
  *keys = reinterpret_cast<uint16_t*>(ws + inner_bytes + 256);
  cudaError_t e = cudaMemsetAsync(gst, 0, 4, st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  PageGatherParams gp{};
  gp.k_pages = k_pages;
  gp.n_pages = n_pages;
  gp.page_size = page_size;
  gp.block_table = block_table;
  gp.T_k = T_k;
  gp.k_out = *keys;
  gp.status = gst;
  if ((e = launch_page_gather(gp, sm_count(), st)) != cudaSuccess) return cuda_fail(e, "page gather launch");
  return DSA_OK;
}

int check_prefill_args(int64_t q_offset, int64_t T_q, int64_t T_k, int H, int d, int topk) {
  int rc = check_shape(H, d, topk);
  if (rc != DSA_OK) return rc;
  if (T_q < 0 || T_k < 1 || q_offset < 0 || q_offset + T_q > T_k)
    return fail(DSA_EINVAL, "need T_q >= 0, T_k >= 1, 0 <= q_offset, q_offset + T_q <= T_k");
  if (T_k >= (int64_t(1) << 31) || T_q * H >= (int64_t(1) << 31))
    return fail(DSA_EINVAL, "T_k and T_q*H must be below 2^31");
  return DSA_OK;
}

// Fused score + streaming Top-k over the chunk's rows, then the final
// selection, on device buffers (arguments already checked).  reset_status
// clears the workspace's device status word first; begin_profile starts the
// per-kernel events, profile records them.
// FP8 inputs of a prefill: the E4M3 codes and their per-row scales (q and k
// of prefill_run then point at the codes).
struct Fp8Scales {
  const float* q_scale;  // [T_q][H]
  const float* k_scale;  // [T_k]
};

int prefill_run(const void* q, const float* w, const void* k, int64_t q_offset, int64_t T_q,
                int64_t T_k, int H, int topk, int32_t* out_idx, float* out_score, uint8_t* ws,
                const PrefillPlan& P, bool reset_status, bool begin_profile, bool profile, cudaStream_t st,
                const Fp8Scales* f8 = nullptr) {
  int rc;
  CUtensorMap tq, tk;
  if (f8) {
    if ((rc = make_tmap_u8(&tq, q, T_q * H, P.G * H)) != DSA_OK) return rc;
    if ((rc = make_tmap_u8(&tk, k, T_k, kTileKeys)) != DSA_OK) return rc;
  } else {
    if ((rc = make_tmap(&tq, q, T_q * H, P.G * H)) != DSA_OK) return rc;
    if ((rc = make_tmap(&tk, k, T_k, kTileKeys)) != DSA_OK) return rc;
  }
  cudaError_t e;
  if (reset_status && (e = cudaMemsetAsync(ws, 0, 4, st)) != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  if (begin_profile) prof_begin(st);

  ScoreParams sp{};
  sp.mode = kModePrefill;
  sp.topk = topk;
  sp.lay = P.lay;
  sp.S = P.S;
  sp.n_groups = P.n_groups;
  sp.n_units = P.n_units;
  sp.q_offset = q_offset;
  sp.T_q = T_q;
  sp.T_k = T_k;
  sp.w = w;
  sp.cand = reinterpret_cast<uint64_t*>(ws + P.off_cand);
  sp.meta = reinterpret_cast<int32_t*>(ws + P.off_meta);
  sp.err = reinterpret_cast<uint32_t*>(ws);
  if (f8) {
    sp.q_scale = f8->q_scale;
    sp.k_scale = f8->k_scale;
    if ((e = launch_score_fp8(H, P.G, P.eg, tq, tk, sp, P.grid, st)) != cudaSuccess)
      return cuda_fail(e, "FP8 score kernel launch");
  } else if ((e = launch_score(H, P.G, P.eg, tq, tk, sp, P.grid, st)) != cudaSuccess) {
    return cuda_fail(e, "score kernel launch");
  }
  if (profile) prof_mark(st, "score_topk");

  SelectParams se{};
  se.mode = kModePrefill;
  se.G = P.G;
  se.S = P.S;
  se.topk = topk;
  se.lay = P.lay;
  se.n_rows = T_q;
  se.cand = sp.cand;
  se.meta = sp.meta;
  se.out_idx = out_idx;
  se.out_score = out_score;
  se.err = sp.err;
  if ((e = launch_select(se, st)) != cudaSuccess) return cuda_fail(e, "select kernel launch");
  if (profile) prof_mark(st, "select_topk");
  return DSA_OK;
}

// Row blocks of a large prefill.  A chunk whose candidate buffers would not
// fit the caller's workspace runs as consecutive launches over row blocks
// (rows are independent, so the result is the same bit for bit); the
// workspace size query caps its answer at kPrefillWorkspaceCap.
constexpr size_t kPrefillWorkspaceCap = size_t(4) << 30;

// Workspace of a launch over `rows` rows, sized for the most key splits any
// offset can give them (q_offset = T_k - rows).
size_t block_bytes(int64_t rows, int64_t T_k, int H, int topk) {
  return plan_prefill(rows, T_k, std::max<int64_t>(T_k - rows, 0), H, topk).bytes;
}

// Largest row count (all rows, or a multiple of the query group) whose launch
// fits `bytes`; 0 when not even one group fits.
int64_t prefill_block_rows(int64_t T_q, int64_t T_k, int H, int topk, size_t bytes) {
  if (block_bytes(T_q, T_k, H, topk) <= bytes) return T_q;
  const int64_t G = 256 / H;
  int64_t lo = 0, hi = (T_q - 1) / G;  // in groups
  while (lo < hi) {
    const int64_t mid = (lo + hi + 1) / 2;
    if (block_bytes(mid * G, T_k, H, topk) <= bytes) lo = mid; else hi = mid - 1;
  }
  return lo * G;
}

// ------------------------------------------------------- host-buffer prefill
// Row blocks of a chunk stream through two device slots: while block b is
// scored on the caller's stream, the inputs of block b+1 cross PCIe on one
// library stream and the outputs of block b-1 come back on another (the two
// copy directions run at once).  Keys go to the device once per call.
struct HostPlan {
  int64_t block_rows;
  int nb;
  size_t off_k, off_q[2], off_w[2], off_idx[2], off_score[2], off_ws, ws_bytes, bytes;
};

HostPlan plan_host(int64_t T_q, int64_t T_k, int H, int d, int topk) {
  HostPlan P{};
  const int64_t nb = std::min<int64_t>(std::max<int64_t>((T_q + 2047) / 2048, 1), 16);
  P.block_rows = std::max<int64_t>(((T_q + nb - 1) / nb + 7) / 8 * 8, 1);
  P.nb = static_cast<int>((T_q + P.block_rows - 1) / P.block_rows);
  const int64_t br = P.block_rows, last = T_q - (P.nb - 1) * br;
  // one prefill workspace first (its device status word at offset 0, where
  // dsa_index_device_status reads it), reused block after block on the
  // caller's stream; then the keys and two slots of block buffers
  P.ws_bytes = std::max(plan_prefill(br, T_k, T_k - br, H, topk).bytes,
                        plan_prefill(last, T_k, T_k - last, H, topk).bytes);
  P.off_ws = 0;
  size_t off = align_up(P.ws_bytes, 256);
  auto take = [&](size_t n) {
    const size_t o = off;
    off = align_up(off + n, 256);
    return o;
  };
  P.off_k = take(static_cast<size_t>(T_k) * d * 2);
  for (int s = 0; s < 2; ++s) {
    P.off_q[s] = take(static_cast<size_t>(br) * H * d * 2);
    P.off_w[s] = take(static_cast<size_t>(br) * H * 4);
    P.off_idx[s] = take(static_cast<size_t>(br) * topk * 4);
    P.off_score[s] = take(static_cast<size_t>(br) * topk * 4);
  }
  P.bytes = off;
  return P;
}

struct HostStreams {
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, keys = nullptr;
  cudaEvent_t in[16] = {}, comp[16] = {}, out[16] = {};
};

std::mutex g_host_mu;

int host_streams(HostStreams** out) {
  static HostStreams per_dev[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(DSA_EDEVICE, "device ordinal %d out of range", dev);
  HostStreams& H = per_dev[dev];
  if (!H.h2d) {
    auto ev = [&](cudaEvent_t* x) { return cudaEventCreateWithFlags(x, cudaEventDisableTiming); };
    if ((e = cudaStreamCreateWithFlags(&H.h2d, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaStreamCreateWithFlags(&H.d2h, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = ev(&H.start)) != cudaSuccess || (e = ev(&H.keys)) != cudaSuccess)
      return cuda_fail(e, "library stream/event creation");
    for (int i = 0; i < 16; ++i)
      if ((e = ev(&H.in[i])) != cudaSuccess || (e = ev(&H.comp[i])) != cudaSuccess ||
          (e = ev(&H.out[i])) != cudaSuccess)
        return cuda_fail(e, "library event creation");
  }
  *out = &H;
  return DSA_OK;
}

}  // namespace

namespace dsa {
void take_wait_injection(ScoreParams& p) {
  if (!g_inject.armed) return;
  g_inject.armed = false;
  p.stall_loads = 1;
  p.wait_ns = g_inject.limit_ns;
}
}  // namespace dsa

extern "C" {

int dsa_test_inject_wait_timeout(int64_t limit_ns) {
  if (limit_ns < 1000000 || limit_ns > 2000000000)
    return fail(DSA_EINVAL, "limit_ns = %lld outside [1 ms, 2 s]", static_cast<long long>(limit_ns));
  g_inject.armed = true;
  g_inject.limit_ns = static_cast<uint64_t>(limit_ns);
  return DSA_OK;
}


const char* dsa_last_error_string(void) { return g_last_error.c_str(); }

size_t dsa_index_prefill_workspace_bytes(int64_t T_q, int64_t T_k, int H, int d, int topk) {
  if (check_shape(H, d, topk) != DSA_OK || T_q < 0 || T_k < 1) return 0;
  const size_t full = block_bytes(T_q, T_k, H, topk);
  if (full <= kPrefillWorkspaceCap) return full;
  // larger chunks run in row blocks whose workspace fits the cap
  return block_bytes(prefill_block_rows(T_q, T_k, H, topk, kPrefillWorkspaceCap), T_k, H, topk);
}

int dsa_index_prefill(const uint16_t* q, const float* w, const uint16_t* k, int64_t q_offset,
                      int64_t T_q, int64_t T_k, int H, int d, int topk, int32_t* out_idx,
                      float* out_score, void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_prefill_args(q_offset, T_q, T_k, H, d, topk);
  if (rc != DSA_OK || T_q == 0) return rc;
  if (!q || !w || !k || !out_idx || !out_score || !workspace)
    return fail(DSA_EINVAL, "null pointer argument");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(workspace, 16) || !aligned(w, 4) ||
      !aligned(out_idx, 4) || !aligned(out_score, 4))
    return fail(DSA_EINVAL, "misaligned pointer (q, k, workspace need 16 bytes)");
  // as many rows per launch as the workspace holds (all of them when it can)
  const int64_t br = prefill_block_rows(T_q, T_k, H, topk, ws_bytes);
  if (br < 1)
    return fail(DSA_EWORKSPACE, "workspace of %zu bytes, %zu needed", ws_bytes,
                block_bytes(std::min<int64_t>(T_q, 256 / H), T_k, H, topk));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  for (int64_t r0 = 0; r0 < T_q; r0 += br) {
    const int64_t n = std::min(br, T_q - r0);
    const PrefillPlan P = plan_prefill(n, T_k, q_offset + r0, H, topk);
    if (P.bytes > ws_bytes) return fail(DSA_EWORKSPACE, "internal: row block workspace too small");
    rc = prefill_run(q + static_cast<size_t>(r0) * H * kD, w + static_cast<size_t>(r0) * H, k, q_offset + r0, n,
                     T_k, H, topk, out_idx + static_cast<size_t>(r0) * topk, out_score + static_cast<size_t>(r0) * topk,
                     ws, P, r0 == 0, r0 == 0, true, st);
    if (rc != DSA_OK) return rc;
  }
  return DSA_OK;
}

int dsa_index_prefill_fp8(const uint8_t* q, const float* q_scale, const float* w, const uint8_t* k,
                          const float* k_scale, int64_t q_offset, int64_t T_q, int64_t T_k, int H, int d, int topk,
                          int32_t* out_idx, float* out_score, void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_prefill_args(q_offset, T_q, T_k, H, d, topk);
  if (rc != DSA_OK || T_q == 0) return rc;
  if (!q || !q_scale || !w || !k || !k_scale || !out_idx || !out_score || !workspace)
    return fail(DSA_EINVAL, "null pointer argument");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(workspace, 16) || !aligned(w, 4) || !aligned(q_scale, 4) ||
      !aligned(k_scale, 4) || !aligned(out_idx, 4) || !aligned(out_score, 4))
    return fail(DSA_EINVAL, "misaligned pointer (q, k, workspace need 16 bytes)");
  const int64_t br = prefill_block_rows(T_q, T_k, H, topk, ws_bytes);
  if (br < 1)
    return fail(DSA_EWORKSPACE, "workspace of %zu bytes, %zu needed", ws_bytes,
                block_bytes(std::min<int64_t>(T_q, 256 / H), T_k, H, topk));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  for (int64_t r0 = 0; r0 < T_q; r0 += br) {
    const int64_t n = std::min(br, T_q - r0);
    const PrefillPlan P = plan_prefill(n, T_k, q_offset + r0, H, topk);
    if (P.bytes > ws_bytes) return fail(DSA_EWORKSPACE, "internal: row block workspace too small");
    const Fp8Scales f8{q_scale + static_cast<size_t>(r0) * H, k_scale};
    rc = prefill_run(q + static_cast<size_t>(r0) * H * kD, w + static_cast<size_t>(r0) * H, k, q_offset + r0, n,
                     T_k, H, topk, out_idx + static_cast<size_t>(r0) * topk, out_score + static_cast<size_t>(r0) * topk,
                     ws, P, r0 == 0, r0 == 0, true, st, &f8);
    if (rc != DSA_OK) return rc;
  }
  return DSA_OK;
}

size_t dsa_index_prefill_host_workspace_bytes(int64_t T_q, int64_t T_k, int H, int d, int topk) {
  if (check_shape(H, d, topk) != DSA_OK || T_q < 1 || T_k < 1) return 0;
  return plan_host(T_q, T_k, H, d, topk).bytes;
}

int dsa_index_prefill_host(const uint16_t* q, const float* w, const uint16_t* k, int64_t q_offset,
                           int64_t T_q, int64_t T_k, int H, int d, int topk, int32_t* out_idx,
                           float* out_score, void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_prefill_args(q_offset, T_q, T_k, H, d, topk);
  if (rc != DSA_OK || T_q == 0) return rc;
  if (!q || !w || !k || !out_idx || !out_score || !workspace)
    return fail(DSA_EINVAL, "null pointer argument");
  if (!aligned(workspace, 256)) return fail(DSA_EINVAL, "misaligned workspace (needs 256 bytes)");
  const HostPlan P = plan_host(T_q, T_k, H, d, topk);
  if (ws_bytes < P.bytes) return fail(DSA_EWORKSPACE, "workspace of %zu bytes, %zu needed", ws_bytes, P.bytes);
  std::lock_guard<std::mutex> lock(g_host_mu);
  HostStreams* S = nullptr;
  if ((rc = host_streams(&S)) != DSA_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* pws = ws + P.off_ws;
  auto ck = [&](cudaError_t x, const char* what) { return x == cudaSuccess ? DSA_OK : cuda_fail(x, what); };
  // the copy streams start after everything already queued on the caller's stream
  if ((rc = ck(cudaEventRecord(S->start, st), "cudaEventRecord")) != DSA_OK) return rc;
  if ((rc = ck(cudaStreamWaitEvent(S->h2d, S->start, 0), "cudaStreamWaitEvent")) != DSA_OK) return rc;
  if ((rc = ck(cudaStreamWaitEvent(S->d2h, S->start, 0), "cudaStreamWaitEvent")) != DSA_OK) return rc;
  if ((rc = ck(cudaMemsetAsync(pws, 0, 4, st), "cudaMemsetAsync")) != DSA_OK) return rc;
  uint16_t* dk = reinterpret_cast<uint16_t*>(ws + P.off_k);
  if ((rc = ck(cudaMemcpyAsync(dk, k, static_cast<size_t>(T_k) * d * 2, cudaMemcpyHostToDevice, S->h2d),
               "key copy")) != DSA_OK) return rc;
  if ((rc = ck(cudaEventRecord(S->keys, S->h2d), "cudaEventRecord")) != DSA_OK) return rc;
  if ((rc = ck(cudaStreamWaitEvent(st, S->keys, 0), "cudaStreamWaitEvent")) != DSA_OK) return rc;
  // last block first: under a causal mask later rows see more keys, so the
  // longest scoring overlaps the copies and the exposed tail is short
  for (int i = 0; i < P.nb; ++i) {
    const int b = P.nb - 1 - i, s = i & 1;
    const int64_t r0 = b * P.block_rows, rows = std::min(P.block_rows, T_q - r0);
    uint16_t* dq = reinterpret_cast<uint16_t*>(ws + P.off_q[s]);
    float* dw = reinterpret_cast<float*>(ws + P.off_w[s]);
    int32_t* di = reinterpret_cast<int32_t*>(ws + P.off_idx[s]);
    float* dsc = reinterpret_cast<float*>(ws + P.off_score[s]);
    // inputs of block b, once slot s is free (the outputs of the block two
    // steps earlier copied out)
    if (i >= 2 && (rc = ck(cudaStreamWaitEvent(S->h2d, S->out[i - 2], 0), "cudaStreamWaitEvent")) != DSA_OK)
      return rc;
    if ((rc = ck(cudaMemcpyAsync(dq, q + r0 * H * d, static_cast<size_t>(rows) * H * d * 2,
                                 cudaMemcpyHostToDevice, S->h2d), "query copy")) != DSA_OK) return rc;
    if ((rc = ck(cudaMemcpyAsync(dw, w + r0 * H, static_cast<size_t>(rows) * H * 4, cudaMemcpyHostToDevice,
                                 S->h2d), "weight copy")) != DSA_OK) return rc;
    if ((rc = ck(cudaEventRecord(S->in[i], S->h2d), "cudaEventRecord")) != DSA_OK) return rc;
    // score block b on the caller's stream
    if ((rc = ck(cudaStreamWaitEvent(st, S->in[i], 0), "cudaStreamWaitEvent")) != DSA_OK) return rc;
    const PrefillPlan PB = plan_prefill(rows, T_k, q_offset + r0, H, topk);
    if (PB.bytes > P.ws_bytes) return fail(DSA_EWORKSPACE, "internal: block workspace too small");
    if ((rc = prefill_run(dq, dw, dk, q_offset + r0, rows, T_k, H, topk, di, dsc, pws, PB, false, false, false, st)) !=
        DSA_OK)
      return rc;
    if ((rc = ck(cudaEventRecord(S->comp[i], st), "cudaEventRecord")) != DSA_OK) return rc;
    // its outputs back to the host
    if ((rc = ck(cudaStreamWaitEvent(S->d2h, S->comp[i], 0), "cudaStreamWaitEvent")) != DSA_OK) return rc;
    if ((rc = ck(cudaMemcpyAsync(out_idx + r0 * topk, di, static_cast<size_t>(rows) * topk * 4,
                                 cudaMemcpyDeviceToHost, S->d2h), "index copy")) != DSA_OK) return rc;
    if ((rc = ck(cudaMemcpyAsync(out_score + r0 * topk, dsc, static_cast<size_t>(rows) * topk * 4,
                                 cudaMemcpyDeviceToHost, S->d2h), "score copy")) != DSA_OK) return rc;
    if ((rc = ck(cudaEventRecord(S->out[i], S->d2h), "cudaEventRecord")) != DSA_OK) return rc;
  }
  // the caller's stream completes when the last outputs are on the host
  return ck(cudaStreamWaitEvent(st, S->out[P.nb - 1], 0), "cudaStreamWaitEvent");
}

size_t dsa_index_decode_workspace_bytes(int B, int64_t t_cap, int H, int d, int topk) {
  if (check_shape(H, d, topk) != DSA_OK || B < 1 || t_cap < 0) return 0;
  return plan_decode(B, topk).bytes;
}

int dsa_index_decode(const uint16_t* q, const float* w, const uint16_t* k_cache,
                     const int32_t* seq_len, int B, int64_t t_cap, int H, int d, int topk,
                     int32_t* out_idx, float* out_score, void* workspace, size_t ws_bytes,
                     void* stream) {
  int rc = check_decode_args(q, w, k_cache, seq_len, B, t_cap, H, d, topk, out_idx, out_score);
  if (rc != DSA_OK) return rc;
  if (!workspace) return fail(DSA_EINVAL, "null workspace");
  if (!aligned(workspace, 16)) return fail(DSA_EINVAL, "misaligned workspace (needs 16 bytes)");
  const DecodePlan P = plan_decode(B, topk);
  if (ws_bytes < P.bytes) return fail(DSA_EWORKSPACE, "workspace of %zu bytes, %zu needed", ws_bytes, P.bytes);
  return decode_run(q, w, k_cache, seq_len, B, t_cap, H, topk, out_idx, out_score,
                    static_cast<uint8_t*>(workspace), P, true, static_cast<cudaStream_t>(stream));
}

int dsa_index_decode_paged(const uint16_t* q, const float* w, const uint16_t* k_pages, int64_t n_pages,
                           int page_size, const int32_t* block_table, int max_blocks, const int32_t* seq_len, int B,
                           int H, int d, int topk, int32_t* out_idx, float* out_score, void* workspace,
                           size_t ws_bytes, void* stream) {
  if (page_size < 64 || page_size % 64 != 0 || max_blocks < 1 || n_pages < 1)
    return fail(DSA_EINVAL, "need page_size a positive multiple of 64, max_blocks >= 1, n_pages >= 1");
  if (n_pages * page_size >= (int64_t(1) << 31)) return fail(DSA_EINVAL, "n_pages * page_size must be below 2^31");
  const int64_t t_cap = static_cast<int64_t>(max_blocks) * page_size;
  int rc = check_shape(H, d, topk);
  if (rc != DSA_OK) return rc;
  if (B < 1 || B > 65536) return fail(DSA_EINVAL, "need 1 <= B <= 65536");
  if (t_cap >= (int64_t(1) << 31)) return fail(DSA_EINVAL, "max_blocks * page_size must be below 2^31");
  if (!q || !w || !k_pages || !block_table || !seq_len || !out_idx || !out_score || !workspace)
    return fail(DSA_EINVAL, "null pointer argument");
  if (!aligned(q, 16) || !aligned(k_pages, 16) || !aligned(workspace, 16) || !aligned(w, 4) ||
      !aligned(block_table, 4) || !aligned(seq_len, 4) || !aligned(out_idx, 4) || !aligned(out_score, 4))
    return fail(DSA_EINVAL, "misaligned pointer (q, k_pages and workspace need 16 bytes)");
  const DecodePlan P = plan_decode(B, topk);
  if (ws_bytes < P.bytes) return fail(DSA_EWORKSPACE, "workspace of %zu bytes, %zu needed", ws_bytes, P.bytes);
  const PagedKeys pk{block_table, max_blocks, page_size, n_pages};
  return decode_run(q, w, k_pages, seq_len, B, t_cap, H, topk, out_idx, out_score, static_cast<uint8_t*>(workspace),
                    P, true, static_cast<cudaStream_t>(stream), &pk);
}

int dsa_index_prefill_pruned(const uint16_t* q, const float* w, const uint16_t* k, int64_t q_offset,
                             int64_t T_q, int64_t T_k, int H, int d, int topk, const int32_t* seed_idx,
                             int n_seed, int32_t* out_idx, float* out_score, dsa_stats* stats,
                             void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_shape(H, d, topk);
  if (rc != DSA_OK) return rc;
  if (T_q < 0 || T_k < 1 || q_offset < 0 || q_offset + T_q > T_k)
    return fail(DSA_EINVAL, "need T_q >= 0, T_k >= 1, 0 <= q_offset, q_offset + T_q <= T_k");
  if (T_k >= (int64_t(1) << 31) || T_q * H >= (int64_t(1) << 31) || T_q * kPlanRows >= (int64_t(1) << 31))
    return fail(DSA_EINVAL, "T_k and T_q*H must be below 2^31");
  if (T_q > 65536) return fail(DSA_EINVAL, "the pruned path takes at most 65536 query rows per call");
  if (n_seed < topk || n_seed > q_offset)
    return fail(DSA_ESEED, "need topk <= n_seed <= q_offset (seeds are keys visible to every row), got n_seed = %d",
                n_seed);
  if (stats) std::memset(stats, 0, sizeof(dsa_stats));
  if (T_q == 0) return DSA_OK;
  if (!q || !w || !k || !seed_idx || !out_idx || !out_score || !workspace)
    return fail(DSA_EINVAL, "null pointer argument");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(workspace, 16) || !aligned(w, 4) ||
      !aligned(seed_idx, 4) || !aligned(out_idx, 4) || !aligned(out_score, 4))
    return fail(DSA_EINVAL, "misaligned pointer (q, k, workspace need 16 bytes)");
  const PrunedPlan P = plan_pruned(T_q, T_k, q_offset, H, topk, n_seed);
  if (ws_bytes < P.bytes) return fail(DSA_EWORKSPACE, "workspace of %zu bytes, %zu needed", ws_bytes, P.bytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* err = reinterpret_cast<uint32_t*>(ws);
  auto at = [&](size_t off) { return ws + off; };
  uint32_t* bypass = reinterpret_cast<uint32_t*>(at(P.off_ctl));
  int32_t* row_flags = reinterpret_cast<int32_t*>(at(P.off_row_flags));
  int32_t* refine_len = reinterpret_cast<int32_t*>(at(P.off_refine_len));
  int32_t* surv_count = reinterpret_cast<int32_t*>(at(P.off_surv_count));
  cudaError_t e;
  // zeroed state: status word, counters, control words, seed bitmap, survivor counts
  if ((e = cudaMemsetAsync(ws, 0, 4, st)) != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  if ((e = cudaMemsetAsync(at(P.off_stats), 0, 8 * sizeof(unsigned long long), st)) != cudaSuccess ||
      (e = cudaMemsetAsync(bypass, 0, 8 * sizeof(uint32_t), st)) != cudaSuccess ||
      (e = cudaMemsetAsync(at(P.off_seed_bits), 0, P.mask_words * 4, st)) != cudaSuccess ||
      (e = cudaMemsetAsync(surv_count, 0, T_q * 4, st)) != cudaSuccess ||
      (e = cudaMemsetAsync(at(P.off_group_len), 0, P.n_groups * 4, st)) != cudaSuccess)
    return cuda_fail(e, "cudaMemsetAsync");
  prof_begin(st);

  // 1. seeds: validate, mark, gather; key norms for the screen
  SeedPrepParams sp0{seed_idx, n_seed, q_offset, k, reinterpret_cast<uint32_t*>(at(P.off_seed_bits)),
                     reinterpret_cast<uint16_t*>(at(P.off_k_seed)), err};
  if ((e = launch_seed_prep(sp0, st)) != cudaSuccess) return cuda_fail(e, "seed prep launch");
  prof_mark(st, "seed_prep");
  if ((e = launch_keynorm(k, T_k, reinterpret_cast<float*>(at(P.off_knorm)), st)) != cudaSuccess)
    return cuda_fail(e, "keynorm launch");
  prof_mark(st, "keynorm");
  CUtensorMap tk, tqrow;
  if ((rc = make_tmap(&tk, k, T_k, kTileKeys)) != DSA_OK) return rc;
  if ((rc = make_tmap(&tqrow, q, T_q * H, H)) != DSA_OK) return rc;
  // 2. the probe rows: seed scoring, plan, screen, compaction
  if ((rc = pruned_rows(P, 0, 0, P.probe, q, w, q_offset, T_k, H, topk, seed_idx, n_seed, tk, ws, nullptr, st)) !=
      DSA_OK)
    return rc;
  // 3. keep pruning the rest of the chunk, or mark it for the dense pass
  if (P.probe < T_q) {
    DecideParams dp{P.probe, T_q, q_offset, n_seed, surv_count, row_flags, refine_len, bypass};
    if ((e = launch_decide(dp, st)) != cudaSuccess) return cuda_fail(e, "decide launch");
    prof_mark(st, "decide");
    if ((rc = pruned_rows(P, 1, P.probe, T_q - P.probe, q, w, q_offset, T_k, H, topk, seed_idx, n_seed, tk, ws,
                          bypass, st)) != DSA_OK)
      return rc;
  }
  // 4. refine survivors exactly (all heads), keeping records at or above the
  //    row's topk-th seed record, then the final exact Top-k over seed records
  //    and refined candidates of the rows that came out of the screen exact
  uint8_t* rws = at(P.off_refine);
  const DecodePlan& R = P.refine;
  DecodePlanParams dq{};
  dq.B = static_cast<int>(T_q);
  dq.grid = R.grid;
  dq.t_cap = P.cap_row;
  dq.seq_len = refine_len;
  dq.seq_start = reinterpret_cast<int64_t*>(rws + R.off_seq_start);
  dq.unit_tab = reinterpret_cast<int32_t*>(rws + R.off_unit_tab);
  dq.cta_ubeg = reinterpret_cast<int32_t*>(rws + R.off_cta_ubeg);
  dq.seq_ubeg = reinterpret_cast<int32_t*>(rws + R.off_seq_ubeg);
  dq.seq_ucnt = reinterpret_cast<int32_t*>(rws + R.off_seq_ucnt);
  dq.err = err;
  if ((e = launch_decode_plan(dq, st)) != cudaSuccess) return cuda_fail(e, "refine plan launch");
  ScoreParams s4{};
  s4.mode = kModeRefine;
  s4.topk = topk;
  s4.lay = R.lay;
  s4.S = 1;
  s4.T_k = T_k;
  s4.w = w;
  s4.seq_len = dq.seq_len;
  s4.unit_tab = dq.unit_tab;
  s4.cta_ubeg = dq.cta_ubeg;
  s4.cand = reinterpret_cast<uint64_t*>(rws + R.off_cand);
  s4.meta = reinterpret_cast<int32_t*>(rws + R.off_meta);
  s4.err = err;
  s4.surv_ids = reinterpret_cast<const int32_t*>(at(P.off_surv_ids));
  s4.surv_stride = P.cap_row;
  s4.k_gather = k;
  s4.init_thr = reinterpret_cast<const uint64_t*>(at(P.off_init_thr));
  if ((e = launch_score(H, 1, 1, tqrow, tk, s4, R.grid, st)) != cudaSuccess) return cuda_fail(e, "refine launch");
  prof_mark(st, "refine");
  // the shared stream: each group's shared keys scored once for its four rows
  uint8_t* rws2 = at(P.off_refine2);
  const DecodePlan& R2 = P.refine2;
  DecodePlanParams dq2{};
  dq2.B = static_cast<int>(P.n_groups);
  dq2.grid = R2.grid;
  dq2.t_cap = P.cap_row;
  dq2.seq_len = reinterpret_cast<const int32_t*>(at(P.off_group_len));
  dq2.seq_start = reinterpret_cast<int64_t*>(rws2 + R2.off_seq_start);
  dq2.unit_tab = reinterpret_cast<int32_t*>(rws2 + R2.off_unit_tab);
  dq2.cta_ubeg = reinterpret_cast<int32_t*>(rws2 + R2.off_cta_ubeg);
  dq2.seq_ubeg = reinterpret_cast<int32_t*>(rws2 + R2.off_seq_ubeg);
  dq2.seq_ucnt = reinterpret_cast<int32_t*>(rws2 + R2.off_seq_ucnt);
  dq2.err = err;
  if ((e = launch_decode_plan(dq2, st)) != cudaSuccess) return cuda_fail(e, "shared refine plan launch");
  CUtensorMap tq4;
  if ((rc = make_tmap(&tq4, q, T_q * H, 4 * H)) != DSA_OK) return rc;
  ScoreParams s4b = s4;
  s4b.mode = kModeRefineShared;
  s4b.T_q = T_q;
  s4b.seq_len = dq2.seq_len;
  s4b.unit_tab = dq2.unit_tab;
  s4b.cta_ubeg = dq2.cta_ubeg;
  s4b.cand = reinterpret_cast<uint64_t*>(rws2 + R2.off_cand);
  s4b.meta = reinterpret_cast<int32_t*>(rws2 + R2.off_meta);
  s4b.surv_ids = reinterpret_cast<const int32_t*>(at(P.off_group_ids));
  if ((e = launch_refine_shared(H, tq4, tk, s4b, R2.grid, st)) != cudaSuccess)
    return cuda_fail(e, "shared refine launch");
  prof_mark(st, "refine_shared");
  SelectParams s5{};
  s5.mode = kModeDecode;
  s5.G = 1;
  s5.S = 1;
  s5.topk = topk;
  s5.lay = R.lay;
  s5.n_rows = T_q;
  s5.cand = s4.cand;
  s5.meta = s4.meta;
  s5.seq_ubeg = dq.seq_ubeg;
  s5.seq_ucnt = dq.seq_ucnt;
  s5.cand2 = s4b.cand;
  s5.meta2 = s4b.meta;
  s5.ubeg2 = dq2.seq_ubeg;
  s5.ucnt2 = dq2.seq_ucnt;
  s5.G2 = 4;
  s5.extra_rec = reinterpret_cast<const uint64_t*>(at(P.off_seed_rec));
  s5.rec_stride = P.rec_stride;
  s5.row_flags = row_flags;
  s5.skip_flagged = 1;
  s5.out_idx = out_idx;
  s5.out_score = out_score;
  s5.err = err;
  if ((e = launch_select(s5, st)) != cudaSuccess) return cuda_fail(e, "final select launch");
  prof_mark(st, "final_select");
  // 5. exact dense pass over every flagged row (overflow, bad seeds, bypass)
  {
    ScoreParams s6{};
    s6.mode = kModePrefill;
    s6.topk = topk;
    s6.lay = P.dense.lay;
    s6.S = P.dense.S;
    s6.n_groups = P.dense.n_groups;
    s6.n_units = P.dense.n_units;
    s6.q_offset = q_offset;
    s6.T_q = T_q;
    s6.T_k = T_k;
    s6.w = w;
    s6.cand = reinterpret_cast<uint64_t*>(at(P.off_cand + P.dense.off_cand));
    s6.meta = reinterpret_cast<int32_t*>(at(P.off_cand + P.dense.off_meta));
    s6.err = err;
    s6.row_flags = row_flags;
    CUtensorMap tqd;
    if ((rc = make_tmap(&tqd, q, T_q * H, P.dense.G * H)) != DSA_OK) return rc;
    if ((e = launch_score(H, P.dense.G, P.dense.eg, tqd, tk, s6, P.dense.grid, st)) != cudaSuccess)
      return cuda_fail(e, "recovery launch");
    prof_mark(st, "dense_pass");
    SelectParams s7{};
    s7.mode = kModePrefill;
    s7.G = P.dense.G;
    s7.S = P.dense.S;
    s7.topk = topk;
    s7.lay = P.dense.lay;
    s7.n_rows = T_q;
    s7.cand = s6.cand;
    s7.meta = s6.meta;
    s7.out_idx = out_idx;
    s7.out_score = out_score;
    s7.row_flags = row_flags;
    s7.err = err;
    if ((e = launch_select(s7, st)) != cudaSuccess) return cuda_fail(e, "recovery select launch");
    prof_mark(st, "dense_select");
  }
  if (stats) {
    unsigned long long* cnt = reinterpret_cast<unsigned long long*>(at(P.off_stats));
    StatsParams sp{T_q, q_offset, n_seed, topk, R.lay, surv_count, refine_len, row_flags, s4.meta,
                   dq.seq_ubeg, dq.seq_ucnt, dq2.seq_len, s4b.meta, dq2.seq_ubeg, dq2.seq_ucnt, cnt};
    if ((e = launch_stats(sp, st)) != cudaSuccess) return cuda_fail(e, "stats launch");
    unsigned long long h[8] = {};
    uint32_t status = 0;
    if ((e = cudaMemcpyAsync(h, cnt, sizeof(h), cudaMemcpyDeviceToHost, st)) != cudaSuccess ||
        (e = cudaMemcpyAsync(&status, err, 4, cudaMemcpyDeviceToHost, st)) != cudaSuccess ||
        (e = cudaStreamSynchronize(st)) != cudaSuccess)
      return cuda_fail(e, "reading the pruned-path counters");
    stats->survivor_pairs = static_cast<int64_t>(h[0]);
    stats->refined_pairs = static_cast<int64_t>(h[1]);
    stats->recovered_rows = static_cast<int64_t>(h[2]);
    stats->bypassed_rows = static_cast<int64_t>(h[3]);
    stats->screened_pairs = static_cast<int64_t>(h[4]);
    stats->records = static_cast<int64_t>(h[5]);
    stats->shared_keys = static_cast<int64_t>(h[6]);
    if (status & kErrSeed) return fail(DSA_ESEED, "a seed was out of range or repeated; the rows were recomputed densely");
    if (status & kErrTimeout) return fail(DSA_EDEVICE, "a device-side wait gave up (status 0x%x)", status);
    if (status & kErrNonFinite) return fail(DSA_EDEVICE, "a visible pair scored inf or NaN (non-finite input)");
  }
  return DSA_OK;
}

int dsa_index_prefill_pruned_survivors(const void* workspace, int64_t T_q, int64_t T_k, int64_t q_offset, int H,
                                       int d, int topk, int n_seed, uint32_t* mask, float* tau, int32_t* row_state,
                                       void* stream) {
  int rc = check_shape(H, d, topk);
  if (rc != DSA_OK) return rc;
  if (T_q < 1 || T_k < 1 || q_offset < 0 || q_offset + T_q > T_k || n_seed < 1)
    return fail(DSA_EINVAL, "need T_q >= 1, T_k >= 1, 0 <= q_offset, q_offset + T_q <= T_k, n_seed >= 1");
  if (!workspace || !mask || !tau || !row_state) return fail(DSA_EINVAL, "null pointer argument");
  const PrunedPlan P = plan_pruned(T_q, T_k, q_offset, H, topk, n_seed);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const uint8_t* ws = static_cast<const uint8_t*>(workspace);
  cudaError_t e;
  if ((e = cudaMemcpyAsync(mask, ws + P.off_bitmask, static_cast<size_t>(T_q) * P.mask_words * 4,
                           cudaMemcpyDeviceToDevice, st)) != cudaSuccess ||
      (e = cudaMemcpyAsync(tau, ws + P.off_tau, static_cast<size_t>(T_q) * 4, cudaMemcpyDeviceToDevice, st)) !=
          cudaSuccess ||
      (e = cudaMemcpyAsync(row_state, ws + P.off_row_flags, static_cast<size_t>(T_q) * 4, cudaMemcpyDeviceToDevice,
                           st)) != cudaSuccess)
    return cuda_fail(e, "copying the screen's survivor mask");
  return DSA_OK;
}

size_t dsa_index_prefill_paged_workspace_bytes(int64_t T_q, int64_t T_k, int H, int d, int topk) {
  const size_t inner = dsa_index_prefill_workspace_bytes(T_q, T_k, H, d, topk);
  return inner ? align_up(inner, 256) + paged_tail_bytes(T_k) : 0;
}

int dsa_index_prefill_paged(const uint16_t* q, const float* w, const uint16_t* k_pages, int64_t n_pages,
                            int page_size, const int32_t* block_table, int64_t q_offset, int64_t T_q, int64_t T_k,
                            int H, int d, int topk, int32_t* out_idx, float* out_score, void* workspace,
                            size_t ws_bytes, void* stream) {
  int rc = check_prefill_args(q_offset, T_q, T_k, H, d, topk);
  if (rc != DSA_OK || T_q == 0) return rc;
  if ((rc = check_paged_pool(k_pages, n_pages, page_size, block_table)) != DSA_OK) return rc;
  if (!workspace || !aligned(workspace, 256)) return fail(DSA_EINVAL, "workspace must be 256-byte aligned");
  const size_t tail = paged_tail_bytes(T_k);
  if (ws_bytes < tail + 256) return fail(DSA_EWORKSPACE, "workspace of %zu bytes, %zu needed for the keys alone",
                                         ws_bytes, tail + 256);
  const size_t inner = (ws_bytes - tail) & ~static_cast<size_t>(255);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint16_t* keys = nullptr;
  if ((rc = gather_paged_keys(k_pages, n_pages, page_size, block_table, T_k, ws, inner, &keys, st)) != DSA_OK)
    return rc;
  if ((rc = dsa_index_prefill(q, w, keys, q_offset, T_q, T_k, H, d, topk, out_idx, out_score, ws, inner, stream)) !=
      DSA_OK)
    return rc;
  cudaError_t e = launch_status_or(reinterpret_cast<const uint32_t*>(ws + inner), reinterpret_cast<uint32_t*>(ws), st);
  return e == cudaSuccess ? DSA_OK : cuda_fail(e, "status merge launch");
}

size_t dsa_index_prefill_pruned_paged_workspace_bytes(int64_t T_q, int64_t T_k, int H, int d, int topk,
                                                      int n_seed) {
  const size_t inner = dsa_index_prefill_pruned_workspace_bytes(T_q, T_k, H, d, topk, n_seed);
  return inner ? align_up(inner, 256) + paged_tail_bytes(T_k) : 0;
}

int dsa_index_prefill_pruned_paged(const uint16_t* q, const float* w, const uint16_t* k_pages, int64_t n_pages,
                                   int page_size, const int32_t* block_table, int64_t q_offset, int64_t T_q,
                                   int64_t T_k, int H, int d, int topk, const int32_t* seed_idx, int n_seed,
                                   int32_t* out_idx, float* out_score, dsa_stats* stats, void* workspace,
                                   size_t ws_bytes, void* stream) {
  int rc = check_prefill_args(q_offset, T_q, T_k, H, d, topk);
  if (rc != DSA_OK) return rc;
  if ((rc = check_paged_pool(k_pages, n_pages, page_size, block_table)) != DSA_OK) return rc;
  if (!workspace || !aligned(workspace, 256)) return fail(DSA_EINVAL, "workspace must be 256-byte aligned");
  const size_t tail = paged_tail_bytes(T_k);
  const size_t need = dsa_index_prefill_pruned_paged_workspace_bytes(T_q, T_k, H, d, topk, n_seed);
  if (need == 0) return fail(DSA_EINVAL, "bad sizes");
  if (ws_bytes < need) return fail(DSA_EWORKSPACE, "workspace of %zu bytes, %zu needed", ws_bytes, need);
  const size_t inner = need - tail;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint16_t* keys = nullptr;
  if (T_q > 0 &&
      (rc = gather_paged_keys(k_pages, n_pages, page_size, block_table, T_k, ws, inner, &keys, st)) != DSA_OK)
    return rc;
  if ((rc = dsa_index_prefill_pruned(q, w, keys ? keys : k_pages, q_offset, T_q, T_k, H, d, topk, seed_idx, n_seed,
                                     out_idx, out_score, stats, ws, inner, stream)) != DSA_OK)
    return rc;
  if (T_q == 0) return DSA_OK;
  cudaError_t e = launch_status_or(reinterpret_cast<const uint32_t*>(ws + inner), reinterpret_cast<uint32_t*>(ws), st);
  if (e != cudaSuccess) return cuda_fail(e, "status merge launch");
  if (stats) {  // the pruned call synchronised before the merge: read the gather's bit as well
    uint32_t s = 0;
    if ((e = cudaMemcpyAsync(&s, ws + inner, 4, cudaMemcpyDeviceToHost, st)) != cudaSuccess ||
        (e = cudaStreamSynchronize(st)) != cudaSuccess)
      return cuda_fail(e, "reading the page gather status");
    if (s) return fail(DSA_EDEVICE, "a block-table entry lies outside the page pool (status 0x%x)", s);
  }
  return DSA_OK;
}

size_t dsa_index_seeds_from_history_workspace_bytes(int64_t n_keys) {
  if (n_keys < 1 || n_keys > INT32_MAX) return 0;
  return plan_history(n_keys).bytes;
}

int dsa_index_seeds_from_history(const int32_t* prev_idx, int64_t n_rows, int topk, int64_t n_keys, int n_seed,
                                 int32_t* seeds_out, void* workspace, size_t ws_bytes, void* stream) {
  if (!seeds_out || !workspace || (n_rows > 0 && !prev_idx)) return fail(DSA_EINVAL, "null pointer argument");
  if (n_rows < 0 || topk < 1 || n_keys < 1 || n_keys > INT32_MAX)
    return fail(DSA_EINVAL, "n_rows = %lld, topk = %d, n_keys = %lld: need n_rows >= 0, topk >= 1, 1 <= n_keys < 2^31",
                static_cast<long long>(n_rows), topk, static_cast<long long>(n_keys));
  if (n_seed < 1 || n_seed > n_keys)
    return fail(DSA_EINVAL, "n_seed = %d outside [1, n_keys = %lld]", n_seed, static_cast<long long>(n_keys));
  if (n_rows > 0 && n_rows > static_cast<int64_t>(UINT32_MAX) / topk)
    return fail(DSA_EINVAL, "n_rows * topk = %lld * %d exceeds 2^32 - 1 list entries",
                static_cast<long long>(n_rows), topk);
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return fail(DSA_EINVAL, "workspace not 256-byte aligned");
  const HistoryPlan P = plan_history(n_keys);
  if (ws_bytes < P.bytes) return fail(DSA_EWORKSPACE, "workspace of %zu bytes, %zu needed", ws_bytes, P.bytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaError_t e = cudaMemsetAsync(ws, 0, P.zero_bytes, st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  HistoryParams hp{};
  hp.prev = prev_idx;
  hp.n_rows = n_rows;
  hp.topk = topk;
  hp.n_keys = n_keys;
  hp.n_seed = n_seed;
  hp.num_sms = sm_count();
  hp.counts = reinterpret_cast<uint32_t*>(ws + P.off_counts);
  hp.hist = reinterpret_cast<uint32_t*>(ws + P.off_hist);
  hp.ctl = reinterpret_cast<uint32_t*>(ws + P.off_ctl);
  hp.tile_gt = reinterpret_cast<uint32_t*>(ws + P.off_tile_gt);
  hp.tile_eq = reinterpret_cast<uint32_t*>(ws + P.off_tile_eq);
  hp.seeds = seeds_out;
  if ((e = launch_history_seeds(hp, st)) != cudaSuccess) return cuda_fail(e, "history seed kernels");
  return DSA_OK;
}

size_t dsa_index_prefill_pruned_workspace_bytes(int64_t T_q, int64_t T_k, int H, int d, int topk, int n_seed) {
  if (check_shape(H, d, topk) != DSA_OK || T_q < 0 || T_k < 1 || n_seed < 1) return 0;
  return plan_pruned(T_q, T_k, T_k - T_q, H, topk, n_seed).bytes;
}

int dsa_index_decode_noalloc(const uint16_t* q, const float* w, const uint16_t* k_cache,
                             const int32_t* seq_len, int B, int64_t t_cap, int H, int d, int topk,
                             int32_t* out_idx, float* out_score, void* stream) {
  int rc = check_decode_args(q, w, k_cache, seq_len, B, t_cap, H, d, topk, out_idx, out_score);
  if (rc != DSA_OK) return rc;
  if (B > kNoAllocMaxB)
    return fail(DSA_EINVAL,
                "dsa_index_decode_noalloc: B = %d sequences exceeds the static scratch limit of %d; "
                "use dsa_index_decode with a caller workspace",
                B, kNoAllocMaxB);
  const DecodePlan P = plan_decode_layout(B, topk, std::min(sm_count(), kNoAllocMaxGrid));
  if (P.bytes > kNoAllocScratchBytes)
    return fail(DSA_EWORKSPACE, "static decode scratch of %zu bytes, %zu needed", kNoAllocScratchBytes, P.bytes);
  void* ws = nullptr;
  if ((rc = noalloc_scratch(&ws)) != DSA_OK) return rc;
  return decode_run(q, w, k_cache, seq_len, B, t_cap, H, topk, out_idx, out_score,
                    static_cast<uint8_t*>(ws), P, false, static_cast<cudaStream_t>(stream));
}

int dsa_index_decode_noalloc_status(uint32_t* status, void* stream) {
  if (!status) return fail(DSA_EINVAL, "null pointer argument");
  void* ws = nullptr;
  int rc = noalloc_scratch(&ws);
  if (rc != DSA_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(status, ws, 4, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "reading the static scratch's device status word");
  return DSA_OK;
}

int dsa_profile_enable(int on) {
  g_prof.enabled = on != 0;
  g_prof.n = 0;
  return DSA_OK;
}

int dsa_profile_read(float* ms, const char** names, int max_n, int* n_out) {
  if (!ms || !n_out) return fail(DSA_EINVAL, "null pointer argument");
  const int n = g_prof.n > 1 ? g_prof.n - 1 : 0;
  *n_out = n;
  if (n == 0) return DSA_OK;
  cudaError_t e = cudaEventSynchronize(g_prof.ev[g_prof.n - 1]);
  if (e != cudaSuccess) return cuda_fail(e, "cudaEventSynchronize");
  for (int i = 0; i < n && i < max_n; ++i) {
    e = cudaEventElapsedTime(&ms[i], g_prof.ev[i], g_prof.ev[i + 1]);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventElapsedTime");
    if (names) names[i] = g_prof.name[i + 1];
  }
  return DSA_OK;
}

int dsa_index_device_status(const void* workspace, uint32_t* status, void* stream) {
  if (!workspace || !status) return fail(DSA_EINVAL, "null pointer argument");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(status, workspace, 4, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
  return DSA_OK;
}

}  // extern "C"
