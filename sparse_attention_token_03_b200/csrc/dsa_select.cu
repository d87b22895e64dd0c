// Final exact Top-k over candidate records, and the decode work planner.
//
// select_topk_kernel: one CTA of 256 threads per output row.  It merges the
// row's candidate buffers (one per key split, plus an optional segment of
// extra records) into the row's m = min(k, candidates) largest records,
// sorted by score descending, then key ascending (the order of the records
// as unsigned integers), and pads the row with key -1 / score -inf past m
// ("DeepSeek DSA FLOPs", selected pair count: a row keeps min(k, visible)).
//
// Every candidate buffer carries its unit's final admission threshold: at
// least k of the unit's records are at or above it, so no record below the
// largest of these thresholds can be selected.  One coalesced pass over the
// row's buffers stages only the records at or above it (usually a little
// more than k) in shared memory; a counting pass over a digit that is linear
// in the score (1024 buckets between the staged minimum and maximum) finds
// the bucket holding the m-th record, the records from that bucket up are
// scattered into bucket order, and a rank count inside each bucket places
// every winner; the row is written in order.  Rows with more records than the
// staging buffer holds, or whose winners crowd one bucket, take an exact
// radix select (10-bit digits) and a bitonic sort instead.  Shared memory
// stays at about 50 KB so that four rows run on each SM at once.
//
// decode_plan_kernel: splits the flattened (sequence, key tile) space of a
// batched decode evenly over the persistent score CTAs and emits the unit
// table (one unit per CTA x sequence overlap).
#include <atomic>
#include <cfloat>

#include "dsa_kernels.cuh"
#include "dsa_ptx.cuh"

namespace dsa {

namespace {

constexpr int kSelBins = 1024;   // buckets of the counting select and radix digits (10 bits)
constexpr int kSelStage = 3072;  // records at or above the row threshold staged in shared memory
constexpr int kSelSegs = 320;    // candidate segments of a row tabulated in shared memory
constexpr int kRankMax = 256;    // largest bucket ranked by counting
constexpr int kBatch = 4;        // records per thread per step of a pass
constexpr size_t kSelectSmem = (kSelStage + kMaxTopk) * sizeof(uint64_t);  // staging + output (dynamic)
static_assert(kSelStage >= kMaxTopk, "the sort exchange reuses the staging buffer");

// Block-wide: largest bucket B with above + sum_{d >= B} hist[d] >= need.
// Writes {B, above + sum_{d > B} hist[d], hist[B]} to res.
template <int NT>
__device__ void find_bucket_blk(const uint32_t* hist, int nb, int above, int need, int* scratch,
                                int* res) {
  const int tid = threadIdx.x;
  const int bpt = (nb + NT - 1) / NT;
  const int lo = tid * bpt;
  int local = 0;
  for (int b = 0; b < bpt; ++b)
    if (lo + b < nb) local += hist[lo + b];
  const int lane = tid & 31, wid = tid >> 5;
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int v = __shfl_down_sync(0xFFFFFFFFu, incl, o);
    if (lane + o < 32) incl += v;
  }
  if (lane == 0) scratch[wid] = incl;
  __syncthreads();
  int higher = 0;
  for (int w2 = wid + 1; w2 < NT / 32; ++w2) higher += scratch[w2];
  const int excl = incl - local + higher;
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
  __syncthreads();
}

struct RowUnits {
  int slot_lo;
  int n_u;
  int q;
};

__device__ __forceinline__ RowUnits row_units(const SelectParams& p, int64_t row) {
  RowUnits r;
  if (p.mode == kModeDecode) {
    r.slot_lo = p.seq_ubeg[row];
    r.n_u = p.seq_ucnt[row];
    r.q = 0;
  } else {
    r.slot_lo = static_cast<int>(row / p.G) * p.S;
    r.n_u = p.S;
    r.q = static_cast<int>(row % p.G);
  }
  return r;
}

// Descending bitonic sort of 2048 records held 8 per thread (thread t owns
// positions 8t..8t+7) by 256 threads.  Compare-exchange partners at distance
// j < 8 sit in the same thread, 8 <= j < 256 in the same warp (register
// shuffles), and only j >= 256 goes through shared memory.
__device__ __forceinline__ void sort2048_desc(uint64_t (&v)[8], uint64_t* s_x) {
  const int t = threadIdx.x;
#pragma unroll
  for (int k = 2; k <= 2048; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j < 8) {
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          if ((s & j) == 0) {
            const int o = s | j;
            const bool desc = (((8 * t + s) & k) == 0);
            const uint64_t a = v[s], b = v[o];
            const bool sw = desc ? (a < b) : (a > b);
            v[s] = sw ? b : a;
            v[o] = sw ? a : b;
          }
        }
      } else {
        const int m = j >> 3;
        const bool lower = (t & m) == 0;
        const bool desc = ((8 * t) & k) == 0;
        const bool take_max = (lower == desc);
        if (j < 256) {
#pragma unroll
          for (int s = 0; s < 8; ++s) {
            const uint64_t o = __shfl_xor_sync(0xFFFFFFFFu, v[s], m);
            v[s] = take_max ? (v[s] > o ? v[s] : o) : (v[s] < o ? v[s] : o);
          }
        } else {
#pragma unroll
          for (int s = 0; s < 8; ++s) s_x[8 * t + s] = v[s];
          __syncthreads();
          const int pt = t ^ m;
#pragma unroll
          for (int s = 0; s < 8; ++s) {
            const uint64_t o = s_x[8 * pt + s];
            v[s] = take_max ? (v[s] > o ? v[s] : o) : (v[s] < o ? v[s] : o);
          }
          __syncthreads();
        }
      }
    }
  }
}

// Warp-aggregated append of the kept records of one step into s_rec
// (positions past cap are counted but not written).
__device__ __forceinline__ void stage_append(bool keep, uint64_t r, uint64_t* s_rec, int cap, int* s_n, int lane) {
  const uint32_t bal = __ballot_sync(0xFFFFFFFFu, keep);
  if (bal == 0u) return;
  int pos = 0;
  if (lane == 0) pos = atomicAdd(s_n, __popc(bal));
  pos = __shfl_sync(0xFFFFFFFFu, pos, 0);
  const int at = pos + __popc(bal & lanemask_lt());
  if (keep && at < cap) s_rec[at] = r;
}

}  // namespace

template <int NT>
__global__ void __launch_bounds__(NT, 4) select_topk_kernel(const SelectParams p) {
  static_assert(NT == 256, "the sort layout assumes 256 threads x 8 records");
  extern __shared__ __align__(16) uint64_t s_dyn[];
  uint64_t* s_rec = s_dyn;              // [kSelStage] staged records, then winners in bucket order
  uint64_t* s_out = s_dyn + kSelStage;  // [kMaxTopk] the row's output in order / radix winners
  __shared__ __align__(16) uint32_t s_hist[kSelBins];
  __shared__ __align__(16) uint32_t s_cur[kSelBins];
  __shared__ int s_segoff[kSelSegs + 1];
  __shared__ const uint64_t* s_segptr[kSelSegs];
  __shared__ int s_scratch[NT / 32];
  __shared__ int s_res[4];
  __shared__ int s_total, s_n, s_pos, s_maxc;
  __shared__ unsigned long long s_thr, s_lo, s_hi;

  const int64_t row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  if (p.skip && *p.skip) return;
  // with row flags, write either the flagged rows (recovery) or the others
  if (p.row_flags && ((p.row_flags[row] != 0) == (p.skip_flagged != 0))) return;
  const RowUnits R = row_units(p, row);
  const int G = (p.mode == kModeDecode) ? 1 : p.G;
  const CandLayout lay = p.lay;

  // segment sg = 5 * unit + region of the row's candidate buffers (its own
  // units, then the units of the second source); one more segment holds the
  // row's extra records when given
  int n_u2 = 0, slot2 = 0, q2 = 0;
  if (p.cand2) {
    const int64_t g2 = row / p.G2;
    slot2 = p.ubeg2[g2];
    n_u2 = p.ucnt2[g2];
    q2 = static_cast<int>(row % p.G2);
  }
  const int n_own = 5 * R.n_u;
  auto unit_meta = [&](int u) -> const int32_t* {
    if (u >= R.n_u) return p.meta2 + (static_cast<size_t>(slot2 + u - R.n_u) * p.G2 + q2) * kMetaInts;
    return p.meta + (static_cast<size_t>(R.slot_lo + u) * G + R.q) * kMetaInts;
  };
  auto segment = [&](int sg, int& cnt) -> const uint64_t* {
    if (sg == 5 * (R.n_u + n_u2)) {
      cnt = p.topk;
      return p.extra_rec + static_cast<size_t>(row) * p.rec_stride;
    }
    const int u = sg / 5, r = sg % 5;
    const bool second = sg >= n_own;
    const size_t qi = second ? static_cast<size_t>(slot2 + u - R.n_u) * p.G2 + q2
                             : static_cast<size_t>(R.slot_lo + u) * G + R.q;
    const int32_t* mt = (second ? p.meta2 : p.meta) + qi * kMetaInts;
    const int cap = (r == 0) ? lay.keep_cap : lay.app_cap;
    cnt = min(max(mt[1 + r], 0), cap);  // counts are always in range; clamp defensively
    return (second ? p.cand2 : p.cand) + qi * lay.query_recs() + static_cast<size_t>(mt[0] & 1) * lay.half_recs() +
           lay.region_off(r);
  };
  const int n_seg = 5 * (R.n_u + n_u2) + (p.extra_rec ? 1 : 0);
  const bool table = n_seg <= kSelSegs;

  // 1. warp 0: segment table (offsets of a flattened index), total count and
  //    the row threshold (largest unit threshold; the extra segment, sorted,
  //    holds k records >= its k-th)
  if (wid == 0) {
    uint64_t thr = 0;
    int off = 0;
    for (int base = 0; base < n_seg; base += 32) {
      const int sg = base + lane;
      int c = 0;
      const uint64_t* ptr = nullptr;
      if (sg < n_seg) {
        ptr = segment(sg, c);
        if (sg == 5 * (R.n_u + n_u2)) {
          const uint64_t kth = ptr[p.topk - 1];
          thr = kth > thr ? kth : thr;
        } else if (sg % 5 == 0) {
          const int32_t* mt = unit_meta(sg / 5);
          const uint64_t ut = (static_cast<uint64_t>(static_cast<uint32_t>(mt[7])) << 32) |
                              static_cast<uint64_t>(static_cast<uint32_t>(mt[6]));
          thr = ut > thr ? ut : thr;
        }
      }
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += v;
      }
      if (sg < n_seg && table) {
        s_segoff[sg] = off + incl - c;
        s_segptr[sg] = ptr;
      }
      off += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const uint64_t v = __shfl_xor_sync(0xFFFFFFFFu, thr, o);
      thr = v > thr ? v : thr;
    }
    if (lane == 0) {
      s_total = off;
      if (table) s_segoff[n_seg] = off;
      s_thr = thr;
      s_n = 0;
      s_pos = 0;
      s_maxc = 0;
      s_lo = ~0ull;
      s_hi = 0ull;
    }
  }
  __syncthreads();
  const int total = s_total;
  const uint64_t thr = s_thr;

  // 2. one coalesced pass: count and stage the records at or above the row
  //    threshold, tracking their score-code range
  {
    uint32_t clo = 0xFFFFFFFFu, chi = 0u;
    auto take = [&](bool in, uint64_t r) {
      const bool keep = in && r != 0ull && r >= thr;
      stage_append(keep, r, s_rec, kSelStage, &s_n, lane);
      if (keep) {
        const uint32_t c = static_cast<uint32_t>(r >> 32);
        clo = min(clo, c);
        chi = max(chi, c);
      }
    };
    if (table) {
      // thread tid reads the flattened indices tid, tid + NT, ...: its
      // segment only moves forward; 8 streaming loads are in flight per step
      constexpr int kLoads = 8;
      int sg = 0;
      for (int base = 0; base < total; base += kLoads * NT) {
        uint64_t r[kLoads];
#pragma unroll
        for (int j = 0; j < kLoads; ++j) {
          const int i = base + j * NT + tid;
          r[j] = 0ull;
          if (i < total) {
            while (s_segoff[sg + 1] <= i) ++sg;
            r[j] = __ldcs(reinterpret_cast<const unsigned long long*>(s_segptr[sg]) + (i - s_segoff[sg]));
          }
        }
        // one shared-memory atomic per warp and step for the staging slots
        uint32_t bal[kLoads];
        int tot = 0;
#pragma unroll
        for (int j = 0; j < kLoads; ++j) {
          bal[j] = __ballot_sync(0xFFFFFFFFu, base + j * NT + tid < total && r[j] != 0ull && r[j] >= thr);
          tot += __popc(bal[j]);
        }
        if (tot == 0) continue;
        int at = 0;
        if (lane == 0) at = atomicAdd(&s_n, tot);
        at = __shfl_sync(0xFFFFFFFFu, at, 0);
#pragma unroll
        for (int j = 0; j < kLoads; ++j) {
          if ((bal[j] >> lane) & 1u) {
            const int pos = at + __popc(bal[j] & lanemask_lt());
            if (pos < kSelStage) s_rec[pos] = r[j];
            const uint32_t c = static_cast<uint32_t>(r[j] >> 32);
            clo = min(clo, c);
            chi = max(chi, c);
          }
          at += __popc(bal[j]);
        }
      }
    } else {
      for (int sg = 0; sg < n_seg; ++sg) {
        int cnt;
        const uint64_t* buf = segment(sg, cnt);
        for (int base = 0; base < cnt; base += NT) {
          const int i = base + tid;
          take(i < cnt, i < cnt ? buf[i] : 0ull);
        }
      }
    }
    clo = __reduce_min_sync(0xFFFFFFFFu, clo);
    chi = __reduce_max_sync(0xFFFFFFFFu, chi);
    if (lane == 0 && chi != 0u) {
      atomicMin(&s_lo, static_cast<unsigned long long>(clo) << 32);
      atomicMax(&s_hi, (static_cast<unsigned long long>(chi) << 32) | 0xFFFFFFFFull);
    }
  }
  __syncthreads();
  int n = s_n;  // records at or above the row threshold
  const int m = min(p.topk, n);
  bool staged = n <= kSelStage;

  // 2b. more records than the staging buffer holds: count all of them over
  //     the linear score digit of the counting path (range [s_lo, s_hi]),
  //     find the bucket B of the m-th, and stage again only the records in
  //     buckets >= B (every one of the m winners, usually a few more); the
  //     counting path then runs on them unchanged
  if (!staged && m > 0 && table) {
    const float smin = record_score(s_lo), srange = record_score(s_hi) - smin;
    const float scale = static_cast<float>(kSelBins - 1) / srange;
    if (srange >= 1e-30f && srange <= 3.0e38f && scale <= 3.0e38f) {
      auto digit = [&](uint64_t r) {
        return min(static_cast<uint32_t>(kSelBins - 1), static_cast<uint32_t>((record_score(r) - smin) * scale));
      };
      for (int i = tid; i < kSelBins; i += NT) s_hist[i] = 0u;
      __syncthreads();
      // one pass over the row's records: f(valid, record) for index tid, tid + NT, ...
      auto for_records = [&](auto&& f) {
        int sg = 0;
        for (int base = 0; base < total; base += NT) {
          const int i = base + tid;
          uint64_t r = 0ull;
          if (i < total) {
            while (s_segoff[sg + 1] <= i) ++sg;
            r = s_segptr[sg][i - s_segoff[sg]];
          }
          f(i < total && r != 0ull && r >= thr, r);
        }
      };
      for_records([&](bool in, uint64_t r) {
        if (in) atomicAdd(&s_hist[digit(r)], 1u);
      });
      __syncthreads();
      find_bucket_blk<NT>(s_hist, kSelBins, 0, m, s_scratch, s_res);
      const uint32_t B = static_cast<uint32_t>(s_res[0]);
      if (tid == 0) s_n = 0;
      __syncthreads();
      for_records([&](bool in, uint64_t r) { stage_append(in && digit(r) >= B, r, s_rec, kSelStage, &s_n, lane); });
      __syncthreads();
      n = s_n;
      staged = n <= kSelStage;
    }
  }

  const size_t o = static_cast<size_t>(row) * p.topk;
  const size_t orec = static_cast<size_t>(row) * p.rec_stride;
  auto put = [&](int i, uint64_t r) {  // position i of the row's output; r = 0 pads
    const bool ok = r != 0ull;
    if (p.out_idx) p.out_idx[o + i] = ok ? static_cast<int32_t>(record_key(r)) : -1;
    if (p.out_score) p.out_score[o + i] = ok ? record_score(r) : -INFINITY;
    if (p.out_rec) p.out_rec[orec + i] = r;
    if (p.out_kth && i == m - 1) p.out_kth[row] = record_score(r);
  };
  if (p.out_kth && m == 0 && tid == 0) p.out_kth[row] = -INFINITY;

  // 3. counting path over the staged records
  bool done = false;
  if (staged && m > 0) {
    for (int i = tid; i < kSelBins; i += NT) s_hist[i] = 0u;
    // bucket of a record: linear in its score between the staged minimum and
    // maximum (any digit that never decreases along the record order keeps
    // the selection exact; a linear one spreads the winners evenly, where the
    // score code would crowd scores of both signs near zero), or, when that
    // range is zero or not finite, the top 10 bits of (record - smallest)
    const float smin = record_score(s_lo), srange = record_score(s_hi) - smin;
    const float scale = static_cast<float>(kSelBins - 1) / srange;
    const bool lin = srange >= 1e-30f && srange <= 3.0e38f && scale <= 3.0e38f;
    __syncthreads();
    if (!lin) {
      uint64_t lo = ~0ull, hi = 0ull;
      for (int i = tid; i < n; i += NT) {
        const uint64_t r = s_rec[i];
        lo = r < lo ? r : lo;
        hi = r > hi ? r : hi;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const uint64_t l2 = __shfl_xor_sync(0xFFFFFFFFu, lo, off), h2 = __shfl_xor_sync(0xFFFFFFFFu, hi, off);
        lo = l2 < lo ? l2 : lo;
        hi = h2 > hi ? h2 : hi;
      }
      if (tid == 0) {
        s_lo = ~0ull;
        s_hi = 0ull;
      }
      __syncthreads();
      if (lane == 0) {
        atomicMin(&s_lo, static_cast<unsigned long long>(lo));
        atomicMax(&s_hi, static_cast<unsigned long long>(hi));
      }
      __syncthreads();
    }
    const uint64_t rlo = s_lo;
    const uint64_t span = s_hi - rlo;
    const int shift = max(0, 64 - __clzll(static_cast<long long>(span)) - 10);  // span >> shift < 1024
    auto digit = [&](uint64_t r) {
      if (lin) return min(static_cast<uint32_t>(kSelBins - 1), static_cast<uint32_t>((record_score(r) - smin) * scale));
      return static_cast<uint32_t>((r - rlo) >> shift);
    };
    for (int base = tid; base < n; base += kBatch * NT) {
      uint64_t r[kBatch];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) r[j] = base + j * NT < n ? s_rec[base + j * NT] : 0ull;
#pragma unroll
      for (int j = 0; j < kBatch; ++j)
        if (r[j] != 0ull) atomicAdd(&s_hist[digit(r[j])], 1u);
    }
    __syncthreads();
    // descending exclusive scan: thread t owns buckets 1023-4t down to 1020-4t
    const uint4 h4 = reinterpret_cast<const uint4*>(s_hist)[(kSelBins - 4 - 4 * tid) >> 2];
    const uint32_t c[4] = {h4.w, h4.z, h4.y, h4.x};
    const uint32_t sum = c[0] + c[1] + c[2] + c[3];
    uint32_t incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, off);
      if (lane >= off) incl += v;
    }
    if (lane == 31) s_scratch[wid] = static_cast<int>(incl);
    __syncthreads();
    uint32_t run = incl - sum;
    for (int w2 = 0; w2 < wid; ++w2) run += static_cast<uint32_t>(s_scratch[w2]);
    uint32_t ex[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      ex[j] = run;
      const int d = kSelBins - 1 - 4 * tid - j;
      if (c[j] > 0u && run <= static_cast<uint32_t>(m - 1) && static_cast<uint32_t>(m - 1) < run + c[j]) {
        s_res[0] = d;
        s_res[1] = static_cast<int>(run);
        s_res[2] = static_cast<int>(c[j]);
      }
      run += c[j];
    }
    reinterpret_cast<uint4*>(s_cur)[(kSelBins - 4 - 4 * tid) >> 2] = make_uint4(ex[3], ex[2], ex[1], ex[0]);
    __syncthreads();
    const int B = s_res[0], above = s_res[1], cntB = s_res[2];
    uint32_t mc = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (kSelBins - 1 - 4 * tid - j >= B) mc = c[j] > mc ? c[j] : mc;
    mc = __reduce_max_sync(0xFFFFFFFFu, mc);
    if (lane == 0) atomicMax(&s_maxc, static_cast<int>(mc));
    __syncthreads();
    const int nw = above + cntB;  // records in bucket B and above
    if (s_maxc <= kRankMax) {
      // scatter the winners into bucket order, in place: every thread holds
      // its records in registers across the barrier
      constexpr int kPer = kSelStage / NT;
      uint64_t v[kPer];
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int i = j * NT + tid;
        v[j] = i < n ? s_rec[i] : 0ull;
      }
      __syncthreads();
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        if (j * NT >= n) break;
        if (v[j] == 0ull) continue;
        const uint32_t d = digit(v[j]);
        if (static_cast<int>(d) >= B) s_rec[atomicAdd(&s_cur[d], 1u)] = v[j];
      }
      __syncthreads();
      // s_cur[d] is now the end of bucket d; each thread ranks one winner at
      // a time inside its own bucket (consecutive threads hold consecutive
      // winners, so a warp scans about one bucket's length) and writes it
      // straight to its final position of the output
      for (int i = tid; i < nw; i += NT) {
        const uint64_t r = s_rec[i];
        const uint32_t d = digit(r);
        const int end = static_cast<int>(s_cur[d]);
        const int beg = end - static_cast<int>(s_hist[d]);
        int rank = 0;
        for (int x = beg; x < end; x += 2) {
          const uint64_t a0 = s_rec[x];
          const uint64_t a1 = x + 1 < end ? s_rec[x + 1] : 0ull;
          rank += (a0 > r ? 1 : 0) + (a1 > r ? 1 : 0);
        }
        if (beg + rank < m) put(beg + rank, r);
      }
      for (int i = m + tid; i < p.topk; i += NT) put(i, 0ull);
      done = true;
    }
    __syncthreads();
  }
  if (done) return;

  // 4. radix-select + bitonic-sort path (rows with more records than the
  //    staging buffer, or with crowded buckets): over the staged records or
  //    the buffers themselves, records below the row threshold skipped
  uint64_t rthr = thr > 1ull ? thr : 1ull;  // records are >= 1
  if (m > 0 && m < n) {
    uint64_t prefix = 0;
    int pbits = 0, above = 0;
    for (int pass = 0; pass < 8; ++pass) {
      const int shift = max(64 - pbits - 10, 0);
      const int width = 64 - pbits - shift;
      const int nb = 1 << width;
      for (int i = tid; i < nb; i += NT) s_hist[i] = 0;
      __syncthreads();
      auto hist_pass = [&](const uint64_t* buf, int cnt) {
        for (int base = 0; base < cnt; base += 4 * NT) {
          uint64_t v[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int i = base + j * NT + tid;
            v[j] = i < cnt ? buf[i] : 0ull;
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            bool ok = v[j] != 0ull && v[j] >= thr;
            if (pbits > 0) ok = ok && ((v[j] >> (64 - pbits)) == prefix);
            if (ok) atomicAdd(&s_hist[static_cast<uint32_t>(v[j] >> shift) & static_cast<uint32_t>(nb - 1)], 1u);
          }
        }
      };
      if (staged) {
        hist_pass(s_rec, n);
      } else {
        for (int sg = 0; sg < n_seg; ++sg) {
          int cnt;
          const uint64_t* buf = segment(sg, cnt);
          hist_pass(buf, cnt);
        }
      }
      __syncthreads();
      find_bucket_blk<NT>(s_hist, nb, above, m, s_scratch, s_res);
      const int B = s_res[0], new_above = s_res[1], cnt = s_res[2];
      prefix = (prefix << width) | static_cast<uint64_t>(B);
      pbits += width;
      if (new_above + cnt == m || pbits == 64) {
        rthr = (pbits == 64) ? prefix : (prefix << (64 - pbits));
        break;
      }
      above = new_above;
      __syncthreads();
    }
  }

  // gather the m winners (in any order) into s_out
  auto gather = [&](const uint64_t* buf, int cnt) {
    for (int base = 0; base < cnt; base += NT) {
      const int i = base + tid;
      const uint64_t r = (i < cnt) ? buf[i] : 0ull;
      const bool keep = (i < cnt) && (r >= rthr) && (r >= thr) && (r != 0ull);
      const uint32_t bal = __ballot_sync(0xFFFFFFFFu, keep);
      if (bal) {
        int pos = 0;
        if (lane == 0) pos = atomicAdd(&s_pos, __popc(bal));
        pos = __shfl_sync(0xFFFFFFFFu, pos, 0);
        const int at = pos + __popc(bal & lanemask_lt());
        if (keep && at < kMaxTopk) s_out[at] = r;
      }
    }
  };
  if (staged) {
    gather(s_rec, n);
  } else {
    for (int sg = 0; sg < n_seg; ++sg) {
      int cnt;
      const uint64_t* buf = segment(sg, cnt);
      gather(buf, cnt);
    }
  }
  __syncthreads();
  if (tid == 0 && s_pos != m) atomicOr(p.err, kErrOverflow);  // never expected
  uint64_t v[8];
#pragma unroll
  for (int s2 = 0; s2 < 8; ++s2) {
    const int i = 8 * tid + s2;
    v[s2] = (i < m) ? s_out[i] : 0ull;
  }
  __syncthreads();
  sort2048_desc(v, s_rec);
#pragma unroll
  for (int s2 = 0; s2 < 8; ++s2) {
    const int i = 8 * tid + s2;
    if (i < p.topk) put(i, i < m ? v[s2] : 0ull);
  }
}

cudaError_t launch_select(const SelectParams& p, cudaStream_t stream) {
  if (p.n_rows <= 0) return cudaSuccess;
  constexpr int NT = kSelectThreads;
  static std::atomic<bool> configured[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || !configured[dev].load(std::memory_order_acquire)) {
    cudaError_t e = cudaFuncSetAttribute(select_topk_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSelectSmem));
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) configured[dev].store(true, std::memory_order_release);
  }
  select_topk_kernel<NT><<<static_cast<unsigned>(p.n_rows), NT, kSelectSmem, stream>>>(p);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Decode planner (one CTA of 1024 threads).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) decode_plan_kernel(const DecodePlanParams p) {
  __shared__ int64_t s_part[1024];
  __shared__ int s_cnt[1024];
  const int tid = threadIdx.x;
  const int B = p.B;
  // 1) tile counts and their exclusive prefix (chunks of 1024 sequences)
  int64_t carry = 0;
  for (int base = 0; base < B; base += 1024) {
    const int b = base + tid;
    int64_t nt = 0;
    if (b < B) {
      int len = p.seq_len[b];
      if (len < 0 || len > p.t_cap) {
        atomicOr(p.err, kErrOverflow);
        len = 0;
      }
      nt = (static_cast<int64_t>(len) + kTileKeys - 1) / kTileKeys;
    }
    s_part[tid] = nt;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {
      const int64_t v = (tid >= o) ? s_part[tid - o] : 0;
      __syncthreads();
      s_part[tid] += v;
      __syncthreads();
    }
    if (b < B) p.seq_start[b] = carry + s_part[tid] - nt;
    carry += s_part[1023];
    __syncthreads();
  }
  if (tid == 0) p.seq_start[B] = carry;
  for (int b = tid; b < B; b += 1024) {
    p.seq_ubeg[b] = 0;
    p.seq_ucnt[b] = 0;
  }
  __syncthreads();
  const int64_t total = carry;
  // 2) per CTA: its tile range and the sequences it touches
  const int grid = p.grid;
  auto seq_of = [&](int64_t x) {  // last b with seq_start[b] <= x
    int lo = 0, hi = B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.seq_start[mid] <= x) lo = mid; else hi = mid - 1;
    }
    return lo;
  };
  for (int base = 0; base < grid; base += 1024) {
    const int c = base + tid;
    int cnt = 0;
    int64_t lo = 0, hi = 0;
    if (c < grid) {
      lo = total * c / grid;
      hi = total * (c + 1) / grid;
      if (hi > lo) {
        const int b0 = seq_of(lo), b1 = seq_of(hi - 1);
        for (int b = b0; b <= b1; ++b)
          if (p.seq_start[b + 1] > p.seq_start[b]) ++cnt;
      }
    }
    s_cnt[tid] = cnt;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {
      const int v = (tid >= o) ? s_cnt[tid - o] : 0;
      __syncthreads();
      s_cnt[tid] += v;
      __syncthreads();
    }
    const int carry_u = (base == 0) ? 0 : p.cta_ubeg[base];
    int u = carry_u + s_cnt[tid] - cnt;
    if (c < grid) {
      p.cta_ubeg[c] = u;
      if (hi > lo) {
        const int b0 = seq_of(lo), b1 = seq_of(hi - 1);
        for (int b = b0; b <= b1; ++b) {
          const int64_t s0 = p.seq_start[b], s1 = p.seq_start[b + 1];
          if (s1 <= s0) continue;
          const int64_t a = max(lo, s0), e = min(hi, s1);
          p.unit_tab[3 * u + 0] = b;
          p.unit_tab[3 * u + 1] = static_cast<int32_t>(a - s0);
          p.unit_tab[3 * u + 2] = static_cast<int32_t>(e - s0);
          ++u;
        }
      }
      if (c == grid - 1) p.cta_ubeg[grid] = u;
    }
    __syncthreads();
    if (c == min(grid, base + 1024) - 1 && base + 1024 < grid) p.cta_ubeg[base + 1024] = u;
    __syncthreads();
  }
  __syncthreads();
  // 3) per sequence: its first unit and unit count (units of a sequence are contiguous)
  const int n_units = p.cta_ubeg[grid];
  for (int u = tid; u < n_units; u += 1024) {
    const int b = p.unit_tab[3 * u];
    if (p.unit_tab[3 * u + 1] == 0) p.seq_ubeg[b] = u;
    atomicAdd(&p.seq_ucnt[b], 1);
  }
}

cudaError_t launch_decode_plan(const DecodePlanParams& p, cudaStream_t stream) {
  decode_plan_kernel<<<1, 1024, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace dsa
