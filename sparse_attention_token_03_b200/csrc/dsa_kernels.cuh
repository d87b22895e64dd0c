// Shared declarations of the indexer kernels: launch parameters, shared
// memory layout and the candidate-buffer conventions.
//
// Candidate buffers.  A "slot" is one work unit (a query group and a range of
// key tiles).  Every (slot, query) pair owns two halves (ping-pong for
// compaction); a half holds a base region of keep_cap records (what the last
// compaction kept) and four append regions of app_cap records, one per
// epilogue warp (TMEM lane quarter), so that admissions need no atomics.
// Meta per (slot, query): kMetaInts ints = {active half, base count, four
// append counts, admission threshold record (low word, high word)}.  Records are 64-bit (score code << 32 | ~key): unsigned
// order is the selection order, and 0 is never a record.
#pragma once

#include <cuda.h>
#include <cstdint>

namespace dsa {

constexpr int kD = 128;          // index head width d^I (only 128 is supported)
constexpr int kTileKeys = 128;   // keys per MMA tile (M)
constexpr int kMaxTopk = 2048;   // largest supported k
constexpr int kEpiThreads = 128; // threads of one epilogue warpgroup
// Score kernel block: one epilogue warpgroup runs after a producer warp and an
// MMA warp (6 warps); two or four epilogue warpgroups run after a whole
// control warpgroup (producer, MMA, two idle warps) so that registers can be
// moved between warpgroups with setmaxnreg (12 or 20 warps).
__host__ __device__ constexpr int score_epi_warp0(int eg) { return eg == 1 ? 2 : 4; }
__host__ __device__ constexpr int score_threads(int eg) { return 32 * score_epi_warp0(eg) + kEpiThreads * eg; }
// Register split with eg = 2 or 4 epilogue warpgroups: registers per thread
// at launch (65536 / threads, rounded down to 8), then the control
// warpgroup's and each epilogue thread's after setmaxnreg.  The split may
// not ask for more than the block launched with: 128 x 56 + 256 x 224 =
// 384 x 168 and 128 x 56 + 512 x 104 <= 640 x 96.
__host__ __device__ constexpr uint32_t regs_launch(int eg) { return eg == 2 ? 168u : 96u; }
__host__ __device__ constexpr uint32_t regs_ctl(int) { return 56u; }
__host__ __device__ constexpr uint32_t regs_epi(int eg) { return eg == 2 ? 224u : 104u; }
static_assert(128 * regs_ctl(2) + 256 * regs_epi(2) <= 384 * regs_launch(2), "register split (12 warps)");
static_assert(128 * regs_ctl(4) + 512 * regs_epi(4) <= 640 * regs_launch(4), "register split (20 warps)");
static_assert(regs_launch(2) * 384 <= 65536 && regs_launch(4) * 640 <= 65536, "launch registers");
constexpr int kSelectThreads = 256;
// A grouped prefill unit whose keys number at least this many times topk
// runs the two-warpgroup epilogue, shorter ones the four-warpgroup one
// (measured: four warpgroups are faster up to 1M keys at topk = 2048).
constexpr int kWideKeysPerRecord = 2048;

constexpr int kMetaInts = 8;
// Score-code histogram of a query's buffered records, 1024 bins: 1/8-octave
// bins (a score's exponent and top three mantissa bits) over positive scores
// in [2^-32, 2^32) are bins 512 .. 1023, the mirror image over negative scores
// in (-2^32, -2^-32] bins 0 .. 511; smaller magnitudes go to bin 511 or 512
// and larger ones to bins 0 and 1023.  The bin never decreases along the
// score order, and hist_edge(b) is the smallest score code in bin b.  Signed
// bins keep the admissions of a row's first keys (threshold still at its
// minimum, scores of both signs) spread over many bins.
constexpr int kHistBins = 1024;
constexpr uint32_t kHistFine0 = 768u;  // (exponent << 3 | 3 mantissa bits) of 2^-32
__host__ __device__ constexpr uint32_t hist_clamp511(uint32_t fine) {
  return fine < kHistFine0 ? 0u : (fine - kHistFine0 > 511u ? 511u : fine - kHistFine0);
}
__host__ __device__ constexpr uint32_t hist_bin(uint32_t code) {
  return (code & 0x80000000u) ? 512u + hist_clamp511((code & 0x7FFFFFFFu) >> 20)
                              : 511u - hist_clamp511((~code & 0x7FFFFFFFu) >> 20);
}
__host__ __device__ constexpr uint32_t hist_edge(uint32_t bin) {
  return bin >= 513u ? (0x80000000u | ((bin - 512u + kHistFine0) << 20))
         : bin == 512u ? 0x80000000u
         : bin == 0u   ? 0u
                       : 0x7FFFFFFFu - (((kHistFine0 + 511u - bin) << 20) | 0xFFFFFu);
}
static_assert(hist_bin(hist_edge(1)) == 1 && hist_bin(hist_edge(1) - 1) == 0 &&
              hist_bin(hist_edge(511)) == 511 && hist_bin(hist_edge(511) - 1) == 510 &&
              hist_bin(hist_edge(512)) == 512 && hist_bin(hist_edge(512) - 1) == 511 &&
              hist_bin(hist_edge(513)) == 513 && hist_bin(hist_edge(513) - 1) == 512 &&
              hist_bin(hist_edge(1023)) == 1023 && hist_bin(hist_edge(1023) - 1) == 1022,
              "histogram bins");
// The epilogue publishes append counts and checks for overflow every
// kCheckTiles tiles; a warp appends at most 32 records per query per tile.
constexpr int kCheckTiles = 16;
static_assert((kCheckTiles & (kCheckTiles - 1)) == 0, "the check cadence is a power of two");

struct CandLayout {
  int keep_cap;  // records kept by a compaction (>= topk), multiple of 32
  int app_cap;   // records per warp append region, multiple of 32
  __host__ __device__ constexpr int half_recs() const { return keep_cap + 4 * app_cap + 32; }
  __host__ __device__ constexpr int region_off(int r) const { return r == 0 ? 0 : keep_cap + (r - 1) * app_cap; }
  __host__ __device__ constexpr size_t query_recs() const { return 2 * static_cast<size_t>(half_recs()); }
};

__host__ __device__ constexpr CandLayout cand_layout(int topk) {
  CandLayout L{0, 0};
  L.keep_cap = ((2 * topk + 31) / 32) * 32;
  // a warp's region takes a quarter of topk plus kCheckTiles tiles of appends
  // past the overflow check
  L.app_cap = (((topk / 4 + 64 * kCheckTiles) + 31) / 32) * 32;
  return L;
}

// Work decomposition of one fused score launch.
enum ScoreMode : int {
  kModePrefill = 0,  // query groups of a causal chunk; keys 0..q_offset+t
  kModeDecode = 1,   // one query per sequence; keys 0..seq_len[b]-1 of its own cache
  kModeGathered = 2, // query groups; keys are a gathered list (all visible), ids remapped
  kModeRefine = 3,   // one query row per unit (table like decode); keys gathered by id
  kModeRefineShared = 4,  // G consecutive rows per unit (table over row groups); keys gathered by id
};

// Epilogue variants of the fused kernel.
enum ScoreEpilogue : int {
  kEpiScore = 0,   // weighted ReLU head sum + streaming Top-k admission
  kEpiScreen = 1,  // DoSA upper bound from the screening plan + survivor ballot bitmask
};

// DoSA screening plan: rows per query in the screening MMA and the per-row
// scalars (floats): [0, 14) retained head weights, [14, 28) half of the
// retained heads' residual coefficients, [28] key-norm coefficient, [29] tau.
constexpr int kPlanRows = 16;
constexpr int kRetained = kPlanRows - 2;
constexpr int kPlanScalars = 32;
constexpr int kScreenQueries = 8;  // queries per screening MMA (N = 8 x 16 plan rows)

struct ScoreParams {
  int mode;
  int topk;
  CandLayout lay;
  int S;          // key splits per query group (prefill / gathered)
  int n_groups;   // query groups (prefill / gathered)
  int n_units;    // total work units
  int64_t q_offset;
  int64_t T_q;
  int64_t T_k;       // keys in the key tensor (gathered: number of gathered keys)
  int64_t t_cap;     // decode: keys per sequence cache
  const float* w;    // [rows][H]
  const int32_t* seq_len;   // decode
  const int32_t* unit_tab;  // decode: [unit][3] = {b, tile_lo, tile_hi}
  const int32_t* cta_ubeg;  // decode: [grid + 1]
  const int32_t* key_ids;   // gathered: real key id of each gathered key
  uint64_t* cand;
  int32_t* meta;
  uint32_t* err;
  const int32_t* row_flags; // prefill: when set, groups without a flagged row do nothing
  const uint32_t* skip;     // optional: when *skip != 0 the launch does nothing
  // failure injection for tests (dsa_test_inject_wait_timeout): when set, the
  // producer issues no loads, so the MMA warp's first wait runs out after
  // wait_ns and the launch unwinds with the timeout bit
  int stall_loads;
  uint64_t wait_ns;         // limit of the pipeline waits (0: kWaitTimeoutNs)
  // FP8 inputs: one positive fp32 scale per query head row [T_q][H] and per
  // key [T_k] (the bf16 kernels ignore them)
  const float* q_scale;
  const float* k_scale;
  // paged decode: sequence b's key i sits at row block_table[b][i / page_size]
  // * page_size + i % page_size of the page pool (null: contiguous caches)
  const int32_t* block_table;
  int max_blocks;
  int page_size;    // a multiple of 64
  int64_t n_pages;
  // refine: survivor key ids per row (stride surv_stride), the key matrix they
  // index, and an initial admission threshold record per row
  const int32_t* surv_ids;
  int64_t surv_stride;
  const uint16_t* k_gather;
  const uint64_t* init_thr;
  // screen: plan scalars [T_q][kPlanScalars], key norms [T_k], seed bitmap,
  // survivor bitmask [T_q][mask_words] and per-row survivor counts
  const float* plan_s;
  const float* knorm;
  const uint32_t* seed_bits;
  uint32_t* bitmask;
  int64_t mask_words;
  int32_t* surv_count;
};

struct SelectParams {
  int mode;       // kModePrefill / kModeGathered: slots of row t are [(t/G)*S, +S); decode: table
  int G;
  int S;
  int topk;
  CandLayout lay;
  int64_t n_rows;
  const uint64_t* cand;
  const int32_t* meta;
  const int32_t* seq_ubeg;  // decode / refine
  const int32_t* seq_ucnt;  // decode / refine
  // optional second candidate source (the DoSA shared refine stream): units
  // of G2 consecutive rows; row r reads units ubeg2[r / G2] .. + ucnt2[r / G2]
  // as query r % G2
  const uint64_t* cand2;
  const int32_t* meta2;
  const int32_t* ubeg2;
  const int32_t* ucnt2;
  int G2;
  const uint64_t* extra_rec;  // optional [n_rows][rec_stride] extra records (0 = none) merged per row
  int rec_stride;             // row stride of extra_rec / out_rec (>= topk, even)
  const int32_t* row_flags;   // optional: only rows with a non-zero flag are written
  int skip_flagged;           // with row_flags: write only the rows whose flag is zero instead
  const uint32_t* skip;       // optional: when *skip != 0 the launch does nothing
  int32_t* out_idx;         // [n_rows][topk] (may be null when out_rec is set)
  float* out_score;         // [n_rows][topk]
  uint64_t* out_rec;        // optional [n_rows][rec_stride] records (sorted, 0-padded)
  float* out_kth;           // optional [n_rows] score of the last selected record
  uint32_t* err;
};

struct DecodePlanParams {
  int B;
  int grid;
  int64_t t_cap;
  const int32_t* seq_len;
  int64_t* seq_start;  // [B + 1] tile prefix
  int32_t* unit_tab;   // [grid + B][3]
  int32_t* cta_ubeg;   // [grid + 1]
  int32_t* seq_ubeg;   // [B]
  int32_t* seq_ucnt;   // [B]
  uint32_t* err;
};

// Shared-memory footprint of the fused score kernel for N = G*H MMA columns
// and NS key stages (host and device agree on this layout).
struct ScoreSmem {
  int n_cols;
  int ns;
  int eg;    // epilogue warpgroups
  int nqh;   // per-query score-code histograms (kHistBins bins each); 0 for the screen
  int subs;  // 128-byte swizzled column blocks per row: 2 for bf16 (d = 128), 1 for FP8
  __host__ __device__ constexpr uint32_t q_sub() const { return static_cast<uint32_t>(n_cols) * 128u; }
  __host__ __device__ constexpr uint32_t q_bytes() const { return static_cast<uint32_t>(subs) * q_sub(); }
  __host__ __device__ constexpr uint32_t k_sub() const { return 128u * 128u; }
  __host__ __device__ constexpr uint32_t k_stage() const { return static_cast<uint32_t>(subs) * k_sub(); }
  __host__ __device__ constexpr uint32_t off_k() const { return q_bytes(); }
  __host__ __device__ constexpr uint32_t off_w() const { return off_k() + ns * k_stage(); }
  // screening-plan scalars (screen) or the head weights of the tile's queries
  // (score epilogue with four warpgroups): 2 KB
  __host__ __device__ constexpr uint32_t off_hist() const { return off_w() + 512u * 4u; }
  __host__ __device__ constexpr uint32_t off_thr() const { return off_hist() + nqh * kHistBins * 4u; }
  // per query: base count, count at the last threshold update; per (query,
  // warp quarter): published append count
  __host__ __device__ constexpr uint32_t off_count() const { return off_thr() + 8u * 8u; }
  __host__ __device__ constexpr uint32_t off_upd() const { return off_count() + 8u * 4u; }
  __host__ __device__ constexpr uint32_t off_wcnt() const { return off_upd() + 8u * 4u; }
  __host__ __device__ constexpr uint32_t off_half() const { return off_wcnt() + 32u * 4u; }
  __host__ __device__ constexpr uint32_t off_misc() const { return off_half() + 8u * 4u; }
  __host__ __device__ constexpr uint32_t off_bars() const { return off_misc() + eg * 32u * 4u; }
  __host__ __device__ constexpr uint32_t n_bars() const { return 2u + 2u * ns + 4u; }
  __host__ __device__ constexpr uint32_t off_tmem() const { return off_bars() + n_bars() * 8u; }
  __host__ __device__ constexpr uint32_t off_abort() const { return off_tmem() + 4u; }
  __host__ __device__ constexpr uint32_t bytes() const { return off_abort() + 4u; }
  // dynamic smem request: layout + slack to align the base to 1024 bytes
  __host__ __device__ constexpr uint32_t request() const { return bytes() + 1024u; }
};

// Host side of the failure injection: moves a pending one-shot injection of
// the calling thread into the launch's parameters (dsa_api.cu).
void take_wait_injection(ScoreParams& p);

// Launchers (defined in the .cu files).
cudaError_t launch_score(int H, int G, int eg, const CUtensorMap& tmap_q, const CUtensorMap& tmap_k,
                         const ScoreParams& p, int grid, cudaStream_t stream);
// The same fused kernel on FP8 (E4M3) query and key tiles (prefill only).
cudaError_t launch_score_fp8(int H, int G, int eg, const CUtensorMap& tmap_q, const CUtensorMap& tmap_k,
                             const ScoreParams& p, int grid, cudaStream_t stream);
cudaError_t launch_refine_shared(int H, const CUtensorMap& tmap_q, const CUtensorMap& tmap_k, const ScoreParams& p,
                                 int grid, cudaStream_t stream);
cudaError_t launch_screen(const CUtensorMap& tmap_plan, const CUtensorMap& tmap_k, const ScoreParams& p,
                          int grid, cudaStream_t stream);
cudaError_t launch_select(const SelectParams& p, cudaStream_t stream);

// Paged key cache -> contiguous keys (dsa_pages.cu).
struct PageGatherParams {
  const uint16_t* k_pages;      // [n_pages][page_size][128]
  int64_t n_pages;
  int page_size;
  const int32_t* block_table;   // [ceil(T_k / page_size)] page ids of the sequence
  int64_t T_k;
  uint16_t* k_out;              // [T_k][128]
  uint32_t* status;             // status word (overflow bit on a bad page id)
};
cudaError_t launch_page_gather(const PageGatherParams& p, int sms, cudaStream_t st);
cudaError_t launch_status_or(const uint32_t* src, uint32_t* dst, cudaStream_t st);
cudaError_t launch_decode_plan(const DecodePlanParams& p, cudaStream_t stream);

}  // namespace dsa
