// Fused lightning-indexer scoring with streaming Top-k admission (sm_100a).
//
// Computes, for every query row t of a work unit and every visible key s,
//     I(t,s) = sum_j w(t,j) * ReLU(q(t,j) . k(s))
// ("DeepSeek DSA FLOPs", Lightning Indexer, eq. index score) and keeps a
// superset of each row's Top-k in a candidate buffer, so that the T_q x T_k
// score matrix never reaches HBM (the fused score + Top-k idea that the DoSA
// write-up, section 04, credits to LiteTopK).
//
// Layout of one CTA (one per SM, persistent over work units):
//   warp 0  TMA producer: the unit's query tile once (B operand, N = G*H rows
//           of 128 bf16), then key tiles of 128 keys (A operand) through an
//           NS-stage ring (refine units gather survivor keys with cp.async).
//   warp 1  TMEM owner and MMA issuer: per key tile, 8 tcgen05.mma (K = 16
//           each) into one of two TMEM accumulators of N fp32 columns; keys
//           sit on the 128 TMEM lanes, (query, head) on the columns.
//   epilogue  EG warpgroups (after warps 0-1 when EG = 1, after a whole
//           control warpgroup when EG = 2 or 4, with setmaxnreg moving
//           registers to the epilogue); they split the tile's queries.  Each
//           thread owns one key (TMEM lane), reads its dot products in
//           16-column chunks with tcgen05.ld, forms the weighted ReLU head sum
//           on the FMA pipe (head_acc16: eight fp32 chains in a fixed order)
//           and appends (score, key) records that pass the row's running
//           threshold to its warp's region of the candidate buffer.
//   Every kCheckTiles tiles a warpgroup raises each row's threshold from the
//   row's score histogram in shared memory and compacts a buffer that could
//   overflow (one copy pass, or an exact radix select when too many records
//   share the threshold's bin).  The screen variant (EPI = kEpiScreen)
//   evaluates the DoSA bound instead and writes a survivor bitmask.
//
// The admission rule keeps the selection exact: a threshold is only raised
// to a value with at least k buffered records at or above it, so any later
// key below it (records order by score, then smaller key first) can never
// enter the Top-k.
#include <atomic>

#include "dsa_kernels.cuh"
#include "dsa_ptx.cuh"

namespace dsa {

namespace {

// ---------------------------------------------------------------------------
// Helpers for the 128 threads of one epilogue warpgroup (named barrier 1 + e).
// ---------------------------------------------------------------------------
// Each epilogue warpgroup e synchronises on named barrier 1 + e.
__device__ __forceinline__ void epi_sync(int bar) { named_bar_sync(bar, kEpiThreads); }

// Shared-memory histogram increment.
__device__ __forceinline__ void hist_add(uint32_t* hist, bool valid, uint32_t digit) {
  if (valid) atomicAdd(&hist[digit], 1u);
}

// Find the digit bucket B holding the need-th largest record:
// the largest B with above + sum_{d >= B} hist[d] >= need.
// Writes {B, above + sum_{d > B} hist[d], hist[B]} to res[0..3).
// tid in [0, 128); nb in {512, 2048}; scratch >= 4 ints.
__device__ void epi_find_bucket(const uint32_t* hist, int nb, int above, int need, int tid,
                                int* scratch, int* res, int bar) {
  const int bpt = (nb + kEpiThreads - 1) / kEpiThreads;
  const int lo = tid * bpt;
  int local = 0;
  for (int b = 0; b < bpt; ++b)
    if (lo + b < nb) local += hist[lo + b];
  // exclusive suffix sum over threads (higher tid = higher digits)
  const int lane = tid & 31, wid = tid >> 5;
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int v = __shfl_down_sync(0xFFFFFFFFu, incl, o);
    if (lane + o < 32) incl += v;
  }
  if (lane == 0) scratch[wid] = incl;  // warp total
  epi_sync(bar);
  int higher_warps = 0;
  for (int w2 = wid + 1; w2 < kEpiThreads / 32; ++w2) higher_warps += scratch[w2];
  const int excl = incl - local + higher_warps;  // sum over threads > tid
  if (above + excl < need && above + excl + local >= need) {
    int acc = above + excl;
    for (int b = bpt - 1; b >= 0; --b) {
      if (lo + b >= nb) continue;
      const int h = hist[lo + b];
      if (acc + h >= need) {
        res[0] = lo + b;
        res[1] = acc;
        res[2] = h;
        break;
      }
      acc += h;
    }
  }
  epi_sync(bar);
}

// Threshold update with two barriers: the thread holding the topk-th record's
// bin raises the threshold itself.
__device__ void epi_raise(const uint32_t* hist, int need, int tid, int* scratch, int* res, uint64_t* thr,
                          int* upd, int total, int bar) {
  constexpr int bpt = kHistBins / kEpiThreads;
  const int lo = tid * bpt;
  int local = 0;
#pragma unroll
  for (int b = 0; b < bpt; ++b) local += hist[lo + b];
  const int lane = tid & 31, wid = tid >> 5;
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int v = __shfl_down_sync(0xFFFFFFFFu, incl, o);
    if (lane + o < 32) incl += v;
  }
  if (lane == 0) scratch[wid] = incl;
  epi_sync(bar);
  int higher_warps = 0;
  for (int w2 = wid + 1; w2 < kEpiThreads / 32; ++w2) higher_warps += scratch[w2];
  const int excl = incl - local + higher_warps;
  if (excl < need && excl + local >= need) {
    int acc = excl;
    for (int b = bpt - 1; b >= 0; --b) {
      const int h = hist[lo + b];
      if (acc + h >= need) {
        res[0] = lo + b;
        res[1] = acc;
        res[2] = h;
        const uint64_t t_new = static_cast<uint64_t>(hist_edge(static_cast<uint32_t>(lo + b))) << 32;
        if (t_new > *thr) *thr = t_new;
        *upd = total;
        break;
      }
      acc += h;
    }
  }
  epi_sync(bar);
}

// Exact fallback compaction of one (slot, query), run by its epilogue
// warpgroup when the histogram threshold would keep too many records.  The records of the active half (base region + four append
// regions) are reduced to a superset of the `need` largest ones holding at
// most lay.keep_cap records, written to the base region of the other half.
// Radix digits start at the highest bit in which the smallest and largest
// buffered records [lo, hi] differ, so one histogram pass usually decides.
// Returns the new admission threshold (the smallest kept record prefix).
__device__ uint64_t epi_compact(uint64_t* qbuf, const CandLayout lay, int q, int need, int tid,
                                uint32_t* s_hist, uint64_t* s_thr, int* s_count, int* s_wcnt,
                                int* s_half, int* s_misc, uint64_t lo, uint64_t hi, int bar) {
  const int half = s_half[q];
  const uint64_t* src = qbuf + static_cast<size_t>(half) * lay.half_recs();
  uint64_t* dst = qbuf + static_cast<size_t>(half ^ 1) * lay.half_recs();
  int seg_n[5];
  seg_n[0] = s_count[q];
#pragma unroll
  for (int r = 1; r < 5; ++r) seg_n[r] = s_wcnt[q * 4 + r - 1];

  uint64_t prefix = 0;
  int pbits = 0, above = 0;
  const uint64_t diff = lo ^ hi;
  if (diff != 0) {
    pbits = __clzll(static_cast<long long>(diff));
    prefix = pbits > 0 ? (hi >> (64 - pbits)) : 0ull;
  }
  uint64_t thr = lo;
  for (int pass = 0; pass < 7 && diff != 0; ++pass) {
    const int shift = max(64 - pbits - 10, 0);
    const int width = 64 - pbits - shift;
    const int nb = 1 << width;
    for (int i = tid; i < nb; i += kEpiThreads) s_hist[i] = 0;
    epi_sync(bar);
#pragma unroll 1
    for (int r = 0; r < 5; ++r) {
      const uint64_t* sp = src + lay.region_off(r);
      const int n = seg_n[r];
      for (int base = 0; base < n; base += 8 * kEpiThreads) {
        uint64_t v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int i = base + j * kEpiThreads + tid;
          v[j] = i < n ? sp[i] : 0ull;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int i = base + j * kEpiThreads + tid;
          bool ok = i < n;
          if (pbits > 0) ok = ok && ((v[j] >> (64 - pbits)) == prefix);
          hist_add(s_hist, ok, static_cast<uint32_t>(v[j] >> shift) & static_cast<uint32_t>(nb - 1));
        }
      }
    }
    epi_sync(bar);
    epi_find_bucket(s_hist, nb, above, need, tid, s_misc + 4, s_misc + 1, bar);
    const int B = s_misc[1], new_above = s_misc[2], cnt = s_misc[3];
    prefix = (prefix << width) | static_cast<uint64_t>(B);
    pbits += width;
    if (new_above + cnt <= lay.keep_cap || pbits == 64) {
      thr = (pbits == 64) ? prefix : (prefix << (64 - pbits));
      break;
    }
    above = new_above;
  }
  if (tid == 0) s_misc[0] = 0;
  epi_sync(bar);
#pragma unroll 1
  for (int r = 0; r < 5; ++r) {
    const uint64_t* sp = src + lay.region_off(r);
    const int n = seg_n[r];
    for (int base = 0; base < n; base += 8 * kEpiThreads) {
      uint64_t v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int i = base + j * kEpiThreads + tid;
        v[j] = i < n ? sp[i] : 0ull;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int i = base + j * kEpiThreads + tid;
        const bool keep = (i < n) && (v[j] >= thr);
        const uint32_t bal = __ballot_sync(0xFFFFFFFFu, keep);
        if (bal) {
          int pos = 0;
          if ((tid & 31) == 0) pos = atomicAdd(&s_misc[0], __popc(bal));
          pos = __shfl_sync(0xFFFFFFFFu, pos, 0);
          const int at = pos + __popc(bal & lanemask_lt());
          if (keep && at < lay.keep_cap) dst[at] = v[j];
        }
      }
    }
  }
  epi_sync(bar);
  if (tid == 0) {
    s_count[q] = min(s_misc[0], lay.keep_cap);
#pragma unroll
    for (int r = 0; r < 4; ++r) s_wcnt[q * 4 + r] = 0;
    s_half[q] = half ^ 1;
    if (thr > s_thr[q]) s_thr[q] = thr;
  }
  epi_sync(bar);
  return s_thr[q];
}

// Geometry of one work unit, computed identically by every role.
struct Unit {
  int slot;         // candidate-buffer slot
  int64_t row0;     // first query row (prefill / gathered) or sequence (decode)
  int rows;         // valid query rows in the group
  int64_t q_row;    // first row of the query tensor map
  int64_t k_row;    // key tensor-map row of local key 0
  int64_t tile_lo, tile_hi;
  int64_t vis_base; // visible keys: local key < vis_base + row offset (prefill) or < vis_base
};

template <int G>
__device__ __forceinline__ Unit unit_geometry(const ScoreParams& p, int u, int H) {
  Unit U;
  if (p.mode == kModeDecode || p.mode == kModeRefine || p.mode == kModeRefineShared) {
    // b: the sequence / row, or (shared refine) the group of G rows
    const int b = p.unit_tab[3 * u + 0];
    U.slot = u;
    if (p.mode == kModeRefineShared) {
      U.row0 = static_cast<int64_t>(b) * G;
      U.rows = static_cast<int>(p.T_q - U.row0 < G ? p.T_q - U.row0 : G);
    } else {
      U.row0 = b;
      U.rows = 1;
    }
    U.q_row = U.row0 * H;
    U.k_row = (p.mode == kModeDecode) ? static_cast<int64_t>(b) * p.t_cap : 0;
    U.tile_lo = p.unit_tab[3 * u + 1];
    U.tile_hi = p.unit_tab[3 * u + 2];
    U.vis_base = p.seq_len[b];
  } else {
    const int g = p.n_groups - 1 - u / p.S;  // longest groups first
    const int s = u % p.S;
    U.slot = g * p.S + s;
    U.row0 = static_cast<int64_t>(g) * G;
    U.rows = static_cast<int>(p.T_q - U.row0 < G ? p.T_q - U.row0 : G);
    U.q_row = U.row0 * H;
    U.k_row = 0;
    int64_t nkeys;
    if (p.mode == kModePrefill) {
      nkeys = p.q_offset + U.row0 + U.rows;  // keys visible to the group's last row
      U.vis_base = p.q_offset + U.row0 + 1;  // row i of the group sees local keys < vis_base + i
    } else {
      nkeys = p.T_k;
      U.vis_base = p.T_k;
    }
    const int64_t nt = (nkeys + kTileKeys - 1) / kTileKeys;
    U.tile_lo = s * nt / p.S;
    U.tile_hi = (s + 1) * nt / p.S;
    if (p.row_flags) {  // recovery pass: skip groups whose rows all came out exact
      bool any = false;
      for (int i = 0; i < U.rows; ++i) any = any || (p.row_flags[U.row0 + i] != 0);
      if (!any) U.tile_hi = U.tile_lo;
    }
  }
  return U;
}

__device__ __forceinline__ bool gathered_ids(const ScoreParams& p) {
  return p.mode == kModeRefine || p.mode == kModeRefineShared;
}
__device__ __forceinline__ bool tabled(const ScoreParams& p) {
  return p.mode == kModeDecode || gathered_ids(p);
}
// Row of the key-id table a refine unit reads (its row, or its row group).
template <int G>
__device__ __forceinline__ int64_t id_row(const ScoreParams& p, const Unit& U) {
  return p.mode == kModeRefineShared ? U.row0 / G : U.row0;
}
__device__ __forceinline__ int cta_unit_begin(const ScoreParams& p) {
  return tabled(p) ? p.cta_ubeg[blockIdx.x] : static_cast<int>(blockIdx.x);
}
__device__ __forceinline__ int cta_unit_end(const ScoreParams& p) {
  return tabled(p) ? p.cta_ubeg[blockIdx.x + 1] : p.n_units;
}
__device__ __forceinline__ int cta_unit_step(const ScoreParams& p) {
  return tabled(p) ? 1 : static_cast<int>(gridDim.x);
}

// Head weight j of a query row as the epilogue uses it (before halving):
// w for bf16 inputs; w times the row's scale for FP8 inputs (the query
// scale is a positive factor of the head's ReLU term).
template <bool F8>
__device__ __forceinline__ float head_weight(const ScoreParams& p, int64_t i) {
  if constexpr (F8) return __ldg(p.w + i) * __ldg(p.q_scale + i);
  return __ldg(p.w + i);
}

}  // namespace

template <int H, int G, int NS, int EG, int EPI, bool F8 = false>
__global__ void __launch_bounds__(score_threads(EG), 1)
    score_topk_kernel(const __grid_constant__ CUtensorMap tmap_q,
                      const __grid_constant__ CUtensorMap tmap_k, const ScoreParams p) {
  constexpr int N = G * H;
  constexpr int GQ = G / EG;  // queries of a tile handled by one epilogue warpgroup
  constexpr bool kWSmem = EG >= 4;  // head weights read from shared memory (register budget)
  constexpr ScoreSmem L{N, NS, EG, EPI == kEpiScore ? G : 0, F8 ? 1 : 2};
  constexpr int ACC_COLS = N;
  constexpr uint32_t TMEM_COLS = (2 * ACC_COLS <= 32) ? 32u : (2 * ACC_COLS <= 64) ? 64u
                                 : (2 * ACC_COLS <= 128) ? 128u : (2 * ACC_COLS <= 256) ? 256u : 512u;
  constexpr uint32_t IDESC = F8 ? idesc_e4m3_f32(128, N) : idesc_bf16_f32(128, N);
  static_assert(!F8 || EPI == kEpiScore, "FP8 tiles feed the score epilogue only");
  static_assert(N % 16 == 0 && N >= 16 && N <= 256, "MMA N must be a multiple of 16 in [16, 256]");
  static_assert(G % EG == 0, "queries must split evenly over the epilogue warpgroups");

  if (p.skip && *p.skip) return;  // whole launch disabled by an earlier kernel (uniform)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase;
  const uint32_t sK = sbase + L.off_k();
  float* s_w = reinterpret_cast<float*>(smem + L.off_w());
  uint64_t* s_thr = reinterpret_cast<uint64_t*>(smem + L.off_thr());
  int* s_count = reinterpret_cast<int*>(smem + L.off_count());
  int* s_upd = reinterpret_cast<int*>(smem + L.off_upd());
  int* s_half = reinterpret_cast<int*>(smem + L.off_half());
  const uint32_t bar0 = sbase + L.off_bars();
  const uint32_t bar_q_full = bar0, bar_q_empty = bar0 + 8;
  auto bar_k_full = [&](int s) { return bar0 + 16 + 8 * s; };
  auto bar_k_empty = [&](int s) { return bar0 + 16 + 8 * NS + 8 * s; };
  auto bar_acc_full = [&](int a) { return bar0 + 16 + 16 * NS + 8 * a; };
  auto bar_acc_empty = [&](int a) { return bar0 + 16 + 16 * NS + 16 + 8 * a; };
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + L.off_tmem());
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + L.off_abort());

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bar_q_full, 1);
    mbar_init(bar_q_empty, 1);
    for (int s = 0; s < NS; ++s) {
      // gathered key tiles are signalled by all 32 producer lanes, TMA tiles by one
      mbar_init(bar_k_full(s), gathered_ids(p) ? 32 : 1);
      mbar_init(bar_k_empty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar_acc_full(a), 1);
      mbar_init(bar_acc_empty(a), EG * kEpiThreads / 32);
    }
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(s_tmem), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;

  const int u_begin = cta_unit_begin(p), u_end = cta_unit_end(p), u_step = cta_unit_step(p);
  const uint64_t wlim = p.wait_ns ? p.wait_ns : kWaitTimeoutNs;  // pipeline waits

  if (warp < score_epi_warp0(EG)) {
   // one setmaxnreg for the whole control warpgroup
   if constexpr (EG >= 2) regs_dec<regs_ctl(EG)>();
   if (!F8 && warp == 0 && gathered_ids(p) && !p.stall_loads) {
    // ------------------------------------------------ producer (gathered keys)
    // Survivor keys are gathered row by row with 16-byte cp.async into the
    // 128B-swizzled layout the MMA reads.  A stage is signalled LAG tiles
    // later, once its copies are complete and fenced for the async proxy.
    constexpr int LAG = NS / 2;
    uint32_t kt = 0, qi = 0, pending = 0;
    bool ok = true;
    auto signal_oldest = [&]() {
      fence_proxy_async_smem();
      __syncwarp();
      mbar_arrive(bar_k_full((kt - pending) % NS));
      --pending;
    };
    auto drain = [&]() {
      cp_async_wait<0>();
      while (pending > 0) signal_oldest();
    };
    for (int u = u_begin; ok && u < u_end; u += u_step) {
      const Unit U = unit_geometry<G>(p, u, H);
      if (U.tile_hi <= U.tile_lo) continue;
      drain();  // the MMA must see this unit's predecessor complete before the query tile changes
      if (lane == 0) {
        ok = mbar_wait(bar_q_empty, (qi & 1) ^ 1, s_abort, p.err, wlim);
        if (ok) {
          mbar_arrive_expect_tx(bar_q_full, L.q_bytes());
          tma_load_2d(sQ, &tmap_q, 0, static_cast<int32_t>(U.q_row), bar_q_full);
          tma_load_2d(sQ + L.q_sub(), &tmap_q, 64, static_cast<int32_t>(U.q_row), bar_q_full);
        }
      }
      ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      ++qi;
      const int32_t* ids = p.surv_ids + id_row<G>(p, U) * p.surv_stride;
      const int64_t n = U.vis_base;
      for (int64_t t = U.tile_lo; t < U.tile_hi; ++t) {
        const int s = kt % NS;
        if (!(ok = mbar_wait(bar_k_empty(s), ((kt / NS) & 1) ^ 1, s_abort, p.err, wlim))) break;
        const uint32_t stage = sK + s * L.k_stage();
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int j = lane + 32 * jj;
          const int64_t local = t * kTileKeys + j;
          const int32_t id = ids[local < n ? local : 0];
          const uint16_t* src = p.k_gather + static_cast<size_t>(id) * kD;
#pragma unroll
          for (int c = 0; c < 16; ++c)
            cp_async16(stage + (c >> 3) * L.k_sub() + j * 128 + (((c & 7) ^ (j & 7)) << 4), src + c * 8);
        }
        cp_async_commit();
        ++kt;
        ++pending;
        if (pending > LAG) {
          cp_async_wait<LAG>();
          signal_oldest();
        }
      }
    }
    drain();
   } else if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && !p.stall_loads) {
      tma_prefetch_desc(&tmap_q);
      tma_prefetch_desc(&tmap_k);
      uint32_t kt = 0, qi = 0;
      bool ok = true;
      for (int u = u_begin; ok && u < u_end; u += u_step) {
        const Unit U = unit_geometry<G>(p, u, H);
        if (U.tile_hi <= U.tile_lo) continue;
        if (!(ok = mbar_wait(bar_q_empty, (qi & 1) ^ 1, s_abort, p.err, wlim))) break;
        mbar_arrive_expect_tx(bar_q_full, L.q_bytes());
        // bf16: two 64-column boxes per row; FP8: one box of the 128 codes
        tma_load_2d(sQ, &tmap_q, 0, static_cast<int32_t>(U.q_row), bar_q_full);
        if constexpr (!F8) tma_load_2d(sQ + L.q_sub(), &tmap_q, 64, static_cast<int32_t>(U.q_row), bar_q_full);
        ++qi;
        if (u + u_step < u_end) {  // warm L2 with the next unit's query tile
          const Unit V = unit_geometry<G>(p, u + u_step, H);
          tma_prefetch_l2_2d(&tmap_q, 0, static_cast<int32_t>(V.q_row));
          if constexpr (!F8) tma_prefetch_l2_2d(&tmap_q, 64, static_cast<int32_t>(V.q_row));
        }
        // paged key cache: each 64-key half of a tile lies in one page (page
        // sizes are multiples of 64); the block-table entries of tile t + 1
        // are read while tile t's stage is awaited.  Keys past the sequence's
        // length read page 0 and are masked by the epilogue.
        int32_t pg[2] = {0, 0}, pn[2] = {0, 0};
        auto lookup = [&](int64_t t, int32_t (&o)[2]) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int64_t key0 = t * kTileKeys + 64 * h;
            o[h] = key0 < U.vis_base ? p.block_table[U.row0 * p.max_blocks + key0 / p.page_size] : 0;
          }
        };
        if (!F8 && p.block_table) lookup(U.tile_lo, pg);
        for (int64_t t = U.tile_lo; t < U.tile_hi; ++t) {
          const int s = kt % NS;
          if (!F8 && p.block_table && t + 1 < U.tile_hi) lookup(t + 1, pn);
          if (!(ok = mbar_wait(bar_k_empty(s), ((kt / NS) & 1) ^ 1, s_abort, p.err, wlim))) break;
          mbar_arrive_expect_tx(bar_k_full(s), L.k_stage());
          if (!F8 && p.block_table) {
            // pages of a multiple of 128 keys hold whole tiles: one box of 128
            // rows per column half (the key map's box is 128 rows then);
            // 64-key pages take one box of 64 rows per half tile
            const int nh = (p.page_size % kTileKeys == 0) ? 1 : 2;
            for (int h = 0; h < nh; ++h) {
              const int64_t key0 = t * kTileKeys + 64 * h;
              int32_t page = pg[h];
              if (page < 0 || page >= p.n_pages) {
                atomicOr(p.err, kErrOverflow);
                page = 0;
              }
              const int32_t prow = static_cast<int32_t>(static_cast<int64_t>(page) * p.page_size + key0 % p.page_size);
              const uint32_t half = static_cast<uint32_t>(h) * 64u * 128u;
              tma_load_2d(sK + s * L.k_stage() + half, &tmap_k, 0, prow, bar_k_full(s));
              tma_load_2d(sK + s * L.k_stage() + L.k_sub() + half, &tmap_k, 64, prow, bar_k_full(s));
            }
            pg[0] = pn[0];
            pg[1] = pn[1];
          } else {
            const int32_t krow = static_cast<int32_t>(U.k_row + t * kTileKeys);
            tma_load_2d(sK + s * L.k_stage(), &tmap_k, 0, krow, bar_k_full(s));
            if constexpr (!F8) tma_load_2d(sK + s * L.k_stage() + L.k_sub(), &tmap_k, 64, krow, bar_k_full(s));
          }
          ++kt;
        }
      }
      if (!ok) {
        // let the copies already issued land before the CTA's memory is released
        volatile int never = 0;
        const uint32_t first = kt > NS ? kt - NS : 0;
        for (uint32_t i = first; i < kt; ++i)
          mbar_wait(bar_k_full(i % NS), (i / NS) & 1, &never, p.err);
        if (qi > 0) mbar_wait(bar_q_full, (qi - 1) & 1, &never, p.err);
      }
    }
   } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t kt = 0, at = 0, qi = 0, nq = 0;
      bool ok = true;
      for (int u = u_begin; ok && u < u_end; u += u_step) {
        const Unit U = unit_geometry<G>(p, u, H);
        if (U.tile_hi <= U.tile_lo) continue;
        if (!(ok = mbar_wait(bar_q_full, qi & 1, s_abort, p.err, wlim))) break;
        ++qi;
        for (int64_t t = U.tile_lo; t < U.tile_hi; ++t) {
          const int s = kt % NS;
          const int a = at & 1;
          if (!(ok = mbar_wait(bar_k_full(s), (kt / NS) & 1, s_abort, p.err, wlim))) break;
          if (!(ok = mbar_wait(bar_acc_empty(a), ((at >> 1) & 1) ^ 1, s_abort, p.err, wlim))) break;
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + a * ACC_COLS;
          const uint32_t a_base = sK + s * L.k_stage();
#pragma unroll
          // K steps of 32 bytes: 8 x (K = 16 bf16) or 4 x (K = 32 E4M3)
          for (int kk = 0; kk < (F8 ? kD / 32 : kD / 16); ++kk) {
            const uint32_t sub = F8 ? 0u : kk >> 2, off = (F8 ? kk : (kk & 3)) * 32;
            const uint64_t adesc = smem_desc_sw128(a_base + sub * L.k_sub() + off);
            const uint64_t bdesc = smem_desc_sw128(sQ + sub * L.q_sub() + off);
            if constexpr (F8) {
              mma_e4m3(d_tmem, adesc, bdesc, IDESC, kk > 0 ? 1u : 0u);
            } else {
              mma_bf16(d_tmem, adesc, bdesc, IDESC, kk > 0 ? 1u : 0u);
            }
          }
          mma_commit(bar_k_empty(s));
          mma_commit(bar_acc_full(a));
          ++kt;
          ++at;
        }
        if (ok) {
          mma_commit(bar_q_empty);
          ++nq;
        }
      }
      // drain: make sure no MMA still writes TMEM when it is released
      mma_commit(bar_q_empty);
      ++nq;
      volatile int never = 0;
      mbar_wait(bar_q_empty, (nq - 1) & 1, &never, p.err);
    }
   }
  } else if constexpr (EPI == kEpiScreen) {
    // ------------------------------------------------------------ screen epilogue
    // DoSA upper bound per (key, query) from the plan's 16 dot products:
    //   U = sum_i [w_i max(d_i, 0) + (alpha_i / 2) |d_i|] + d_pos / 2
    //       - max(d_neg, 0) + C ||k||
    // (retained heads i < 14, folded positive row d_pos, folded negative row
    // d_neg; C carries the residual, bf16-rounding and fp32 slack terms).  A
    // visible non-seed key survives unless U < tau ("DoSA", step 2: prune only
    // when the bound is strictly below the threshold, keep when unsure).
    // Since w max(d, 0) = (w d + w |d|) / 2, the linear parts of every term
    // are one plan row L (its dot d_L comes from the MMA) and the rest is
    // U = d_L + sum_i c_i |d_i| - max(d_neg, 0) + C ||k||, one FMA with an
    // absolute-value operand per retained head; the fp32 rounding of the
    // coefficients and of the sum lies far inside the 2^-10 S ||k|| part of
    // C.  The coefficients of this thread's queries stay in registers for the
    // whole unit.
    if constexpr (EG >= 2) regs_inc<regs_epi(EG)>();
    const int e = (warp - score_epi_warp0(EG)) >> 2;
    const int quarter = warp & 3;
    const int row_in_tile = quarter * 32 + lane;
    const int q_lo = e * GQ;
    uint32_t at = 0;
    bool ok = true;
    for (int u = u_begin; ok && u < u_end; u += u_step) {
      const Unit U = unit_geometry<G>(p, u, H);
      float c2[GQ][kRetained], cc[GQ], tau[GQ];
#pragma unroll
      for (int i = 0; i < GQ; ++i) {
        const int qq = q_lo + i;
        const bool on = qq < U.rows;
        const float* ps = p.plan_s + (U.row0 + (on ? qq : 0)) * kPlanScalars;
#pragma unroll
        for (int r = 0; r < kRetained; ++r) c2[i][r] = on ? __ldg(ps + r) : 0.0f;
        cc[i] = on ? __ldg(ps + 28) : 0.0f;
        tau[i] = on ? __ldg(ps + 29) : 0.0f;
      }
      int surv[GQ];
#pragma unroll
      for (int i = 0; i < GQ; ++i) surv[i] = 0;
      for (int64_t t = U.tile_lo; ok && t < U.tile_hi; ++t) {
        const int a = at & 1;
        if (!(ok = mbar_wait(bar_acc_full(a), (at >> 1) & 1, s_abort, p.err, wlim))) break;
        tc_fence_after();
        const int64_t key_local = t * kTileKeys + row_in_tile;
        const bool in_range = key_local < p.T_k;
        const bool is_seed = in_range && ((p.seed_bits[key_local >> 5] >> lane) & 1u);
        const float kn = in_range ? p.knorm[key_local] : 0.0f;
        const uint32_t trow = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                              static_cast<uint32_t>(a * ACC_COLS + q_lo * H);
        uint32_t xb[2][16];
        tmem_ld16(trow, xb[0]);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < GQ; ++i) {
          if (i + 1 < GQ) tmem_ld16(trow + (i + 1) * H, xb[(i + 1) & 1]);
          const uint32_t* d = xb[i & 1];
          // two chains over the retained heads, then the linear row, the
          // negative fold and the slack
          float u0 = __uint_as_float(d[kRetained]), u1 = 0.0f;
#pragma unroll
          for (int r = 0; r < kRetained; r += 2) {
            u0 = fmaf(c2[i][r], fabsf(__uint_as_float(d[r])), u0);
            u1 = fmaf(c2[i][r + 1], fabsf(__uint_as_float(d[r + 1])), u1);
          }
          float ub = u0 + u1;
          ub -= fmaxf(__uint_as_float(d[kRetained + 1]), 0.0f);
          ub = fmaf(cc[i], kn, ub);
          const int qq = q_lo + i;
          const bool vis = qq < U.rows && key_local < U.vis_base + qq && !is_seed;
          const bool keep = vis && !(ub < tau[i]);
          const uint32_t word = __ballot_sync(0xFFFFFFFFu, keep);
          if (lane == 0 && qq < U.rows && (key_local >> 5) < p.mask_words)
            p.bitmask[(U.row0 + qq) * p.mask_words + (key_local >> 5)] = word;
          surv[i] += __popc(word);
          if (i + 1 < GQ) tmem_wait_ld();
          if (i + 2 == GQ || GQ == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_acc_empty(a));
          }
        }
        ++at;
      }
      if (!ok) break;
      if (lane == 0) {
#pragma unroll
        for (int i = 0; i < GQ; ++i)
          if (q_lo + i < U.rows && surv[i] > 0) atomicAdd(&p.surv_count[U.row0 + q_lo + i], surv[i]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    if constexpr (EG >= 2) regs_inc<regs_epi(EG)>();
    const int e = (warp - score_epi_warp0(EG)) >> 2;  // epilogue warpgroup
    const int bar = 1 + e;
    const int etid = (threadIdx.x - 32 * score_epi_warp0(EG)) & (kEpiThreads - 1);
    const int quarter = warp & 3;  // TMEM lane quarter this warp may access = its append region
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t lt_mask = (1u << lane) - 1u;
    const int q_lo = e * GQ;
    uint32_t* s_qh = reinterpret_cast<uint32_t*>(smem + L.off_hist());  // [G][kHistBins]
    int* s_misc = reinterpret_cast<int*>(smem + L.off_misc()) + e * 32;
    uint64_t* s_wred = reinterpret_cast<uint64_t*>(s_misc + 8);  // [4] lo, [4] hi per warp
    int* s_wcnt = reinterpret_cast<int*>(smem + L.off_wcnt());
    const CandLayout lay = p.lay;
    uint32_t at = 0;
    bool ok = true;
    for (int u = u_begin; ok && u < u_end; u += u_step) {
      const Unit U = unit_geometry<G>(p, u, H);
      epi_sync(bar);
      for (int i = etid; i < GQ * kHistBins; i += kEpiThreads) s_qh[q_lo * kHistBins + i] = 0u;
      if (etid < GQ) {
        const int qq = q_lo + etid;
        s_upd[qq] = 0;
        s_count[qq] = 0;
        s_thr[qq] = (p.init_thr && qq < U.rows) ? p.init_thr[U.row0 + qq] : 0ull;
        s_half[qq] = 0;
#pragma unroll
        for (int r = 0; r < 4; ++r) s_wcnt[qq * 4 + r] = 0;
      }
      if constexpr (kWSmem) {
        // this warpgroup's halved head weights, in shared memory for the whole unit
        for (int i = etid; i < GQ * H; i += kEpiThreads) {
          const int qq = q_lo + i / H;
          s_w[q_lo * H + i] = qq < U.rows ? half_weight(head_weight<F8>(p, (U.row0 + qq) * H + i % H)) : 0.0f;
        }
      }
      epi_sync(bar);
      // with one or two warpgroups, the halved head weights stay in registers
      // for the whole unit
      // with four warpgroups the first 16 weights of the warpgroup's first
      // query stay in registers too: a quarter (H = 64) or an eighth (H = 32)
      // fewer shared-memory broadcasts per tile
      constexpr int kWReg = kWSmem ? 16 : 0;
      float wq[kWReg > 0 ? kWReg : 1];
      if constexpr (kWReg > 0) {
        const bool on = q_lo < U.rows;
        const int64_t wrow0 = (U.row0 + (on ? q_lo : 0)) * H;
#pragma unroll
        for (int j = 0; j < kWReg; ++j) wq[j] = on ? half_weight(head_weight<F8>(p, wrow0 + j)) : 0.0f;
      }
      float wr[kWSmem ? 1 : GQ][kWSmem ? 1 : H];
      if constexpr (!kWSmem) {
#pragma unroll
        for (int i = 0; i < GQ; ++i) {
          const int qq = q_lo + i;
          const int64_t wrow = (U.row0 + (qq < U.rows ? qq : 0)) * H;
          const bool on = qq < U.rows;
#pragma unroll
          for (int j = 0; j < H; ++j) wr[i][j] = on ? half_weight(head_weight<F8>(p, wrow + j)) : 0.0f;
        }
      }
      uint64_t* cand_unit = p.cand + static_cast<size_t>(U.slot) * G * lay.query_recs();
      // per warp and query: append count (warp-uniform); per lane: smallest
      // and largest record it admitted (reduced only when compacting)
      int cnt[GQ];
      uint32_t rlo[GQ], rhi[GQ];  // score codes: records lie in [rlo << 32, (rhi << 32) | ~0]
#pragma unroll
      for (int i = 0; i < GQ; ++i) {
        cnt[i] = 0;
        rlo[i] = 0xFFFFFFFFu;
        rhi[i] = 0u;
      }
      // per query: the admission threshold (record, and the lowest fp32 score
      // that can reach it) and this warp's append region in the active half.
      // They change only in the periodic check below, which reloads them.
      uint64_t thr[GQ];
      float thr_f[GQ];
      uint64_t* app[GQ];
      auto reload = [&]() {
#pragma unroll
        for (int i = 0; i < GQ; ++i) {
          const int qq = q_lo + i;
          thr[i] = s_thr[qq];
          thr_f[i] = threshold_floor(thr[i]);
          app[i] = cand_unit + static_cast<size_t>(qq) * lay.query_recs() +
                   static_cast<size_t>(s_half[qq]) * lay.half_recs() + lay.region_off(1 + quarter);
        }
      };
      reload();
      bool nonfinite = false;  // a visible pair scored inf or NaN (reported at the unit's end)
      // per query: local keys below visq are visible (none for missing rows).
      // Keys, tiles and these bounds fit 32 bits (T_k < 2^31).
      int visq[GQ];
#pragma unroll
      for (int i = 0; i < GQ; ++i)
        visq[i] = (q_lo + i < U.rows)
                      ? static_cast<int>(p.mode == kModePrefill ? U.vis_base + q_lo + i : U.vis_base)
                      : 0;
      const int t_lo = static_cast<int>(U.tile_lo), t_hi = static_cast<int>(U.tile_hi);
      for (int t = t_lo; ok && t < t_hi; ++t) {
        const int a = at & 1;
        if (!(ok = mbar_wait(bar_acc_full(a), (at >> 1) & 1, s_abort, p.err, wlim))) break;
        tc_fence_after();
        const int key_local = t * kTileKeys + row_in_tile;
        uint32_t key_id = static_cast<uint32_t>(key_local);
        if (p.mode == kModeGathered && key_local < p.T_k) key_id = static_cast<uint32_t>(p.key_ids[key_local]);
        if (gathered_ids(p) && key_local < U.vis_base)
          key_id = static_cast<uint32_t>(p.surv_ids[id_row<G>(p, U) * p.surv_stride + key_local]);
        // this warpgroup's GQ x H dot products, read in 16-column chunks: the
        // next chunk's TMEM load overlaps the current chunk's head sums
        constexpr int CPQ = H / 16, NC = GQ * CPQ;
        const uint32_t trow = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                              static_cast<uint32_t>(a * ACC_COLS + q_lo * H);
        // loads run RING - 1 chunks ahead of the math (one ahead in the
        // one-query four-warpgroup epilogue, whose registers are tightest)
        constexpr int RING = (kWSmem && GQ == 1) ? 2 : 3;
        uint32_t xb[RING][16];
        float score[GQ];
        float2 acc[4];
#pragma unroll
        for (int r = 0; r < RING - 1 && r < NC; ++r) tmem_ld16(trow + r * 16, xb[r]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          if (c + RING - 1 < NC) tmem_ld16(trow + (c + RING - 1) * 16, xb[(c + RING - 1) % RING]);
          if (c % CPQ == 0) {
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[j] = make_float2(0.0f, 0.0f);
          }
          if constexpr (kWSmem) {
            if (c * 16 < kWReg)
              head_acc16(acc, xb[c % RING], &wq[(c * 16) % (kWReg > 0 ? kWReg : 16)]);
            else
              head_acc16_smem(acc, xb[c % RING], s_w + (q_lo + c / CPQ) * H + (c % CPQ) * 16);
          } else {
            head_acc16(acc, xb[c % RING], &wr[c / CPQ][(c % CPQ) * 16]);
          }
          if (c % CPQ == CPQ - 1) score[c / CPQ] = head_finish(acc);
          if (c + RING - 1 < NC) tmem_wait_ld();
          // after the last load has landed, release the accumulator
          if (c == (NC > RING - 1 ? NC - RING : 0)) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_acc_empty(a));
          }
        }
        ++at;
        if constexpr (F8) {
          // FP8: the key's scale multiplies its whole score (positive factor)
          const float ks = key_local < p.T_k ? __ldg(p.k_scale + key_local) : 0.0f;
          nonfinite = nonfinite || !(ks >= 0.0f && ks <= 3.402823466e38f);
#pragma unroll
          for (int i = 0; i < GQ; ++i) score[i] *= ks;
        }
#pragma unroll
        for (int i = 0; i < GQ; ++i) {
          const int qq = q_lo + i;
          // one float compare rules out keys that cannot reach the threshold;
          // the exact record test runs only in warps where some lane passes
          const bool vis = key_local < visq[i];
          nonfinite = nonfinite || (vis && !(fabsf(score[i]) <= 3.402823466e38f));
          const bool pre = vis && score[i] >= thr_f[i];
          if (__any_sync(0xFFFFFFFFu, pre)) {
            const uint64_t rec = make_record(score[i], key_id);
            const bool admit = pre && rec >= thr[i];
            const uint32_t bal = __ballot_sync(0xFFFFFFFFu, admit);
            if (admit) {
              app[i][cnt[i] + __popc(bal & lt_mask)] = rec;
              const uint32_t code = static_cast<uint32_t>(rec >> 32);
              atomicAdd(&s_qh[qq * kHistBins + hist_bin(code)], 1u);
              rlo[i] = min(rlo[i], code);
              rhi[i] = max(rhi[i], code);
            }
            cnt[i] += __popc(bal);
          }
        }
        // every kCheckTiles-th tile (and at the unit's end) the warpgroup
        // publishes its append counts, raises each row's admission threshold
        // from the row's score-code histogram, and compacts buffers that
        // could overflow before the next check
        if (((t - t_lo) & (kCheckTiles - 1)) != kCheckTiles - 1 && t + 1 != t_hi) continue;
        if (lane == 0) {
#pragma unroll
          for (int i = 0; i < GQ; ++i) s_wcnt[(q_lo + i) * 4 + quarter] = cnt[i];
        }
        epi_sync(bar);
#pragma unroll
        for (int i = 0; i < GQ; ++i) {
          const int qq = q_lo + i;
          uint32_t* qh = s_qh + qq * kHistBins;
          bool full = false;
          int total = s_count[qq];
#pragma unroll
          for (int w2 = 0; w2 < 4; ++w2) {
            full = full || (s_wcnt[qq * 4 + w2] > lay.app_cap - kCheckTiles * 32);
            total += s_wcnt[qq * 4 + w2];
          }
          // The histogram counts exactly the buffered records.  With at least
          // topk of them in bins >= B, a later key whose score code lies below
          // bin B is beaten by topk records and can never be selected.
          int kept_above = 0;
          if (total >= p.topk && (full || total - s_upd[qq] >= 256)) {
            epi_raise(qh, p.topk, etid, s_misc + 4, s_misc + 1, &s_thr[qq], &s_upd[qq], total, bar);
            kept_above = s_misc[2] + s_misc[3];
          }
          if (!full) continue;
          const int half_q = s_half[qq];
          uint64_t* qbuf = cand_unit + static_cast<size_t>(qq) * lay.query_recs();
          const uint64_t thr_q = s_thr[qq];
          if (kept_above <= lay.keep_cap) {
            // one copy pass: keep the records at or above the threshold
            const uint64_t* src = qbuf + static_cast<size_t>(half_q) * lay.half_recs();
            uint64_t* dst = qbuf + static_cast<size_t>(half_q ^ 1) * lay.half_recs();
            if (etid == 0) s_misc[0] = 0;
            epi_sync(bar);
#pragma unroll 1
            for (int r = 0; r < 5; ++r) {
              const uint64_t* sp = src + lay.region_off(r);
              const int n = (r == 0) ? s_count[qq] : s_wcnt[qq * 4 + r - 1];
              for (int base = 0; base < n; base += 8 * kEpiThreads) {
                uint64_t v[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                  const int idx = base + j * kEpiThreads + etid;
                  v[j] = idx < n ? sp[idx] : 0ull;
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                  const int idx = base + j * kEpiThreads + etid;
                  const bool keep = (idx < n) && (v[j] >= thr_q);
                  const uint32_t kb = __ballot_sync(0xFFFFFFFFu, keep);
                  if (kb) {
                    int pos = 0;
                    if (lane == 0) pos = atomicAdd(&s_misc[0], __popc(kb));
                    pos = __shfl_sync(0xFFFFFFFFu, pos, 0);
                    const int at2 = pos + __popc(kb & lt_mask);
                    if (keep && at2 < lay.keep_cap) dst[at2] = v[j];
                  }
                }
              }
            }
            epi_sync(bar);
            // records below the threshold are gone: clear their bins
            const uint32_t b_thr = hist_bin(static_cast<uint32_t>(thr_q >> 32));
            for (int bb = etid; bb < kHistBins; bb += kEpiThreads)
              if (static_cast<uint32_t>(bb) < b_thr) qh[bb] = 0u;
            if (etid == 0) {
              s_count[qq] = min(s_misc[0], lay.keep_cap);
#pragma unroll
              for (int r = 0; r < 4; ++r) s_wcnt[qq * 4 + r] = 0;
              s_half[qq] = half_q ^ 1;
            }
            epi_sync(bar);
          } else {
            // too many records share the threshold's bin: exact radix fallback
            // (10-bit digits in the histogram array), then rebuild the histogram
            uint64_t lo = static_cast<uint64_t>(__reduce_min_sync(0xFFFFFFFFu, rlo[i])) << 32;
            uint64_t hi = (static_cast<uint64_t>(__reduce_max_sync(0xFFFFFFFFu, rhi[i])) << 32) | 0xFFFFFFFFull;
            if (lane == 0) {
              s_wred[quarter] = lo;
              s_wred[4 + quarter] = hi;
            }
            epi_sync(bar);
#pragma unroll
            for (int w2 = 0; w2 < 4; ++w2) {
              lo = s_wred[w2] < lo ? s_wred[w2] : lo;
              hi = s_wred[4 + w2] > hi ? s_wred[4 + w2] : hi;
            }
            if (thr_q > lo) lo = thr_q;  // every buffered record is >= the threshold
            epi_sync(bar);
            epi_compact(qbuf, lay, qq, p.topk, etid, qh, s_thr, s_count, s_wcnt, s_half, s_misc, lo, hi, bar);
            for (int bb = etid; bb < kHistBins; bb += kEpiThreads) qh[bb] = 0u;
            epi_sync(bar);
            const uint64_t* kept = qbuf + static_cast<size_t>(s_half[qq]) * lay.half_recs();
            const int nk = s_count[qq];
            for (int idx = etid; idx < nk; idx += kEpiThreads)
              atomicAdd(&qh[hist_bin(static_cast<uint32_t>(kept[idx] >> 32))], 1u);
            epi_sync(bar);
            rhi[i] = static_cast<uint32_t>(hi >> 32);
          }
          if (etid == 0) s_upd[qq] = s_count[qq];
          cnt[i] = 0;
          rlo[i] = 0xFFFFFFFFu;
          epi_sync(bar);
        }
        reload();
      }
      if (__any_sync(0xFFFFFFFFu, nonfinite) && lane == 0) atomicOr(p.err, kErrNonFinite);
      if (!ok) break;
      epi_sync(bar);
      if (etid < GQ) {
        const int qq = q_lo + etid;
        int32_t* m = p.meta + (static_cast<size_t>(U.slot) * G + qq) * kMetaInts;
        m[0] = s_half[qq];
        m[1] = s_count[qq];
#pragma unroll
        for (int w2 = 0; w2 < 4; ++w2) m[2 + w2] = s_wcnt[qq * 4 + w2];
        // the unit's admission threshold: at least topk of its buffered
        // records are >= it once it is above the initial one
        m[6] = static_cast<int32_t>(static_cast<uint32_t>(s_thr[qq]));
        m[7] = static_cast<int32_t>(static_cast<uint32_t>(s_thr[qq] >> 32));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Host launcher
// ---------------------------------------------------------------------------
template <int H, int G, int NS, int EG, int EPI = kEpiScore, bool F8 = false>
static cudaError_t launch_score_t(const CUtensorMap& tq, const CUtensorMap& tk,
                                  const ScoreParams& p, int grid, cudaStream_t stream) {
  constexpr ScoreSmem L{G * H, NS, EG, EPI == kEpiScore ? G : 0, F8 ? 1 : 2};
  static_assert(L.request() <= 227u * 1024u, "shared memory budget");
  auto kern = score_topk_kernel<H, G, NS, EG, EPI, F8>;
  int dev = 0;
  cudaGetDevice(&dev);
  // per (kernel instance, device); racing host threads only repeat the
  // idempotent attribute calls
  static std::atomic<bool> configured[64];
  if (dev < 0 || dev >= 64 || !configured[dev].load(std::memory_order_acquire)) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(L.request()));
    if (e != cudaSuccess) return e;
    if constexpr (EG >= 2) {
      // the setmaxnreg split only balances if every thread launches with exactly
      // regs_launch(EG) registers; refuse to launch otherwise (it would never finish)
      cudaFuncAttributes fa{};
      e = cudaFuncGetAttributes(&fa, kern);
      if (e != cudaSuccess) return e;
      if (fa.numRegs != static_cast<int>(regs_launch(EG))) return cudaErrorInvalidConfiguration;
    }
    if (dev >= 0 && dev < 64) configured[dev].store(true, std::memory_order_release);
  }
  kern<<<grid, score_threads(EG), L.request(), stream>>>(tq, tk, p);
  return cudaGetLastError();
}

cudaError_t launch_score(int H, int G, int eg, const CUtensorMap& tq, const CUtensorMap& tk,
                         const ScoreParams& p0, int grid, cudaStream_t stream) {
  ScoreParams p = p0;
  take_wait_injection(p);
  if (H == 64 && G == 4 && eg == 4) return launch_score_t<64, 4, 4, 4>(tq, tk, p, grid, stream);
  if (H == 64 && G == 4 && eg == 2) return launch_score_t<64, 4, 4, 2>(tq, tk, p, grid, stream);
  if (H == 32 && G == 8 && eg == 4) return launch_score_t<32, 8, 3, 4>(tq, tk, p, grid, stream);
  if (H == 32 && G == 8 && eg == 2) return launch_score_t<32, 8, 3, 2>(tq, tk, p, grid, stream);
  if (H == 64 && G == 1) return launch_score_t<64, 1, 6, 1>(tq, tk, p, grid, stream);
  if (H == 32 && G == 1) return launch_score_t<32, 1, 6, 1>(tq, tk, p, grid, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_score_fp8(int H, int G, int eg, const CUtensorMap& tq, const CUtensorMap& tk,
                             const ScoreParams& p0, int grid, cudaStream_t stream) {
  ScoreParams p = p0;
  take_wait_injection(p);
  if (p.mode != kModePrefill) return cudaErrorInvalidValue;
  // FP8 stages are half the size: twice as many fit
  if (H == 64 && G == 4 && eg == 4) return launch_score_t<64, 4, 8, 4, kEpiScore, true>(tq, tk, p, grid, stream);
  if (H == 64 && G == 4 && eg == 2) return launch_score_t<64, 4, 8, 2, kEpiScore, true>(tq, tk, p, grid, stream);
  if (H == 32 && G == 8 && eg == 4) return launch_score_t<32, 8, 6, 4, kEpiScore, true>(tq, tk, p, grid, stream);
  if (H == 32 && G == 8 && eg == 2) return launch_score_t<32, 8, 6, 2, kEpiScore, true>(tq, tk, p, grid, stream);
  return cudaErrorInvalidValue;
}

// The DoSA shared refine stream: four consecutive rows per unit (N = 4 H),
// survivor keys gathered by id.
cudaError_t launch_refine_shared(int H, const CUtensorMap& tq, const CUtensorMap& tk, const ScoreParams& p0,
                                 int grid, cudaStream_t stream) {
  ScoreParams p = p0;
  take_wait_injection(p);
  if (p.mode != kModeRefineShared) return cudaErrorInvalidValue;
  if (H == 64) return launch_score_t<64, 4, 4, 4>(tq, tk, p, grid, stream);
  if (H == 32) return launch_score_t<32, 4, 5, 2>(tq, tk, p, grid, stream);
  return cudaErrorInvalidValue;
}

// Screening: 16 plan rows per query, kScreenQueries = 8 queries per MMA
// (N = 128), four per epilogue thread so that their bound coefficients fit in
// registers.
cudaError_t launch_screen(const CUtensorMap& tplan, const CUtensorMap& tk, const ScoreParams& p0,
                          int grid, cudaStream_t stream) {
  ScoreParams p = p0;
  take_wait_injection(p);
  return launch_score_t<kPlanRows, kScreenQueries, 5, 2, kEpiScreen>(tplan, tk, p, grid, stream);
}

}  // namespace dsa
