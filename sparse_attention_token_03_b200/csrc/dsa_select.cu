// Final exact Top-k over candidate records, and the decode work planner.
//
// select_topk_kernel: one CTA per output row.  It merges the row's candidate
// buffers (one per key split), finds the m-th largest record exactly
// (m = min(k, candidates); 11-bit radix passes over the 64-bit records,
// top digits first, stopping as soon as the selected prefix holds exactly
// the records still needed), gathers the m winners into shared memory and
// bitonic-sorts them (score descending, then key ascending: the order of the
// records as unsigned integers).  Rows are padded with key -1 / score -inf
// past m ("DeepSeek DSA FLOPs", selected pair count: a row keeps min(k, visible)).
//
// decode_plan_kernel: splits the flattened (sequence, key tile) space of a
// batched decode evenly over the persistent score CTAs and emits the unit
// table (one unit per CTA x sequence overlap).
#include <cfloat>

#include "dsa_kernels.cuh"
#include "dsa_ptx.cuh"

namespace dsa {

namespace {

constexpr int kStageRecs = 7680;  // candidates of a row staged in shared memory (60 KB)
constexpr int kWinCap = 4096;     // records in the boundary bucket and above it (32 KB)
constexpr int kRankMax = 256;     // largest bucket ranked by counting
constexpr int kBatch = 4;         // staged records per thread per step of a pass

__device__ __forceinline__ void hist_add_blk(uint32_t* hist, bool valid, uint32_t digit) {
  if (valid) atomicAdd(&hist[digit], 1u);
}

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

}  // namespace

// One CTA of 256 threads per output row.
//
// Staged rows (the usual case) take one counting pass: a 2048-bucket digit
// of each record that never decreases along the record order (linear in the
// score over the row's score range), a descending prefix scan of the bucket
// counts, which also finds the bucket holding the m-th record, a scatter of
// every record in that bucket or above it into bucket order, and a rank
// count inside each bucket that gives each winner its final position (the
// row's output is then written in order).  Rows whose candidates do not fit the staging buffer, or whose
// records crowd more than kRankMax into one bucket, take the radix-select +
// bitonic-sort path instead.
template <int NT>
__global__ void __launch_bounds__(NT) select_topk_kernel(const SelectParams p) {
  static_assert(NT == 256, "the sort layout assumes 256 threads x 8 records");
  extern __shared__ __align__(16) uint64_t s_dyn[];
  uint64_t* s_rec = s_dyn;               // [kStageRecs] staged candidates (0 = empty slot)
  uint64_t* s_win = s_dyn + kStageRecs;  // [kWinCap] winners in bucket order / sort exchange
  __shared__ __align__(16) uint32_t s_hist[2048];
  __shared__ __align__(16) uint32_t s_cur[2048];
  __shared__ int s_scratch[NT / 32];
  __shared__ int s_res[4];
  __shared__ int s_n, s_staged, s_pos, s_maxc;
  __shared__ unsigned long long s_lo, s_hi;
  __shared__ __align__(8) uint64_t s_bar;

  const int64_t row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  if (p.row_flags && p.row_flags[row] == 0) return;  // row already exact
  const RowUnits R = row_units(p, row);
  const int G = (p.mode == kModeDecode) ? 1 : p.G;
  const CandLayout lay = p.lay;

  // segment sg = 5 * unit + region of the row's candidate buffers; one more
  // segment holds the row's extra records when given
  auto segment = [&](int sg, int& cnt) -> const uint64_t* {
    if (sg == 5 * R.n_u) {
      cnt = p.topk;
      return p.extra_rec + static_cast<size_t>(row) * p.rec_stride;
    }
    const int u = sg / 5, r = sg % 5;
    const size_t qi = static_cast<size_t>(R.slot_lo + u) * G + R.q;
    const int32_t* mt = p.meta + qi * kMetaInts;
    const int cap = (r == 0) ? lay.keep_cap : lay.app_cap;
    cnt = min(max(mt[1 + r], 0), cap);  // counts are always in range; clamp defensively
    return p.cand + qi * lay.query_recs() + static_cast<size_t>(mt[0] & 1) * lay.half_recs() +
           lay.region_off(r);
  };
  const int n_seg = 5 * R.n_u + (p.extra_rec ? 1 : 0);

  // warp 0 sizes the segments (one lane per segment, a warp scan for the
  // staging offsets) and, when they fit, issues one bulk copy per segment
  // into consecutive 16-byte aligned slots
  if (wid == 0) {
    int n = 0, staged = 0;
    for (int base = 0; base < n_seg; base += 32) {
      int c = 0;
      if (base + lane < n_seg) segment(base + lane, c);
      int c2 = (c + 1) & ~1;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        c += __shfl_xor_sync(0xFFFFFFFFu, c, o);
        c2 += __shfl_xor_sync(0xFFFFFFFFu, c2, o);
      }
      n += c;
      staged += c2;
    }
    if (lane == 0) {
      s_n = n;
      s_staged = staged;
      s_pos = 0;
      s_maxc = 0;
      s_lo = ~0ull;
      s_hi = 0ull;
    }
    if (staged <= kStageRecs && n > 0) {
      const uint32_t bar = smem_u32(&s_bar);
      if (lane == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(bar, static_cast<uint32_t>(staged) * 8u);
      }
      __syncwarp();
      int off = 0;
      for (int base = 0; base < n_seg; base += 32) {
        int c = 0;
        const uint64_t* src = nullptr;
        if (base + lane < n_seg) src = segment(base + lane, c);
        const int c2 = (c + 1) & ~1;
        int incl = c2;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
          if (lane >= o) incl += v;
        }
        if (c2 > 0) bulk_load(smem_u32(s_rec + off + incl - c2), src, static_cast<uint32_t>(c2) * 8u, bar);
        off += __shfl_sync(0xFFFFFFFFu, incl, 31);
      }
    }
  }
  __syncthreads();
  const int n = s_n;
  const int m = min(p.topk, n);
  const bool staged = s_staged <= kStageRecs;
  const int n_st = staged ? s_staged : 0;

  if (staged && n > 0) {
    // warp 0 alone waits for the copies (the other warps park at the barrier
    // below instead of spinning on the mbarrier) and blanks the padding slot
    // after each odd-sized segment
    if (wid == 0) {
      volatile int never = 0;
      mbar_wait(smem_u32(&s_bar), 0, &never, p.err);
      __syncwarp();
      int off = 0;
      for (int base = 0; base < n_seg; base += 32) {
        int c = 0;
        if (base + lane < n_seg) segment(base + lane, c);
        const int c2 = (c + 1) & ~1;
        int incl = c2;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
          if (lane >= o) incl += v;
        }
        if (c & 1) s_rec[off + incl - 1] = 0ull;
        off += __shfl_sync(0xFFFFFFFFu, incl, 31);
      }
    }
    __syncthreads();
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

  // ---- counting path
  bool done = false;
  if (staged && m > 0) {
    // every pass over the staged records takes kBatch of them per thread at a
    // time, loads first, so that their shared-memory latencies overlap.
    // First the row's smallest and largest score code (the high words;
    // padding slots are 0 and wrap to the top under c - 1)
    const uint32_t* s_code = reinterpret_cast<const uint32_t*>(s_rec);
    uint32_t clo = 0xFFFFFFFFu, chi = 0u;
    for (int base = tid; base < n_st; base += kBatch * NT) {
      uint32_t c[kBatch];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) c[j] = base + j * NT < n_st ? s_code[2 * (base + j * NT) + 1] : 0u;
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        clo = min(clo, c[j] - 1u);
        chi = max(chi, c[j]);
      }
    }
    clo = __reduce_min_sync(0xFFFFFFFFu, clo);
    chi = __reduce_max_sync(0xFFFFFFFFu, chi);
    for (int i = tid; i < 2048; i += NT) s_hist[i] = 0u;
    if (lane == 0) {
      atomicMin(&s_lo, static_cast<unsigned long long>(clo + 1u) << 32);
      atomicMax(&s_hi, (static_cast<unsigned long long>(chi) << 32) | 0xFFFFFFFFull);
    }
    __syncthreads();
    // bucket of a record: linear in its score between the row's smallest and
    // largest score (any digit that never decreases along the record order
    // works; a linear one spreads the winners evenly), or, when that range is
    // zero or not finite, the top 11 bits of (record - smallest record)
    const float smin = record_score(s_lo), srange = record_score(s_hi) - smin;
    const float scale = 2047.0f / srange;
    const bool lin = srange >= 1e-30f && srange <= 3.0e38f && scale <= 3.0e38f;
    if (!lin) {
      // equal (or non-finite) extreme scores: the exact record range instead
      uint64_t lo = ~0ull, hi = 0ull;
      for (int i = tid; i < n_st; i += NT) {
        const uint64_t r = s_rec[i];
        if (r != 0ull) {
          lo = r < lo ? r : lo;
          hi = r > hi ? r : hi;
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const uint64_t l2 = __shfl_xor_sync(0xFFFFFFFFu, lo, off), h2 = __shfl_xor_sync(0xFFFFFFFFu, hi, off);
        lo = l2 < lo ? l2 : lo;
        hi = h2 > hi ? h2 : hi;
      }
      __syncthreads();
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
    const int shift = max(0, 64 - __clzll(static_cast<long long>(span)) - 11);  // span >> shift < 2048
    auto digit = [&](uint64_t r) {
      if (lin) return min(2047u, static_cast<uint32_t>((record_score(r) - smin) * scale));
      return static_cast<uint32_t>((r - rlo) >> shift);
    };
    for (int base = tid; base < n_st; base += kBatch * NT) {
      uint64_t r[kBatch];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) r[j] = base + j * NT < n_st ? s_rec[base + j * NT] : 0ull;
#pragma unroll
      for (int j = 0; j < kBatch; ++j)
        if (r[j] != 0ull) atomicAdd(&s_hist[digit(r[j])], 1u);
    }
    __syncthreads();
    // descending exclusive scan: thread t owns buckets 2047-8t down to 2040-8t
    const uint4 ha = reinterpret_cast<const uint4*>(s_hist)[(2040 - 8 * tid) >> 2];
    const uint4 hb = reinterpret_cast<const uint4*>(s_hist)[(2044 - 8 * tid) >> 2];
    const uint32_t c[8] = {hb.w, hb.z, hb.y, hb.x, ha.w, ha.z, ha.y, ha.x};
    uint32_t sum = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) sum += c[j];
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
    uint32_t ex[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      ex[j] = run;
      const int d = 2047 - 8 * tid - j;
      if (c[j] > 0u && run <= static_cast<uint32_t>(m - 1) && static_cast<uint32_t>(m - 1) < run + c[j]) {
        s_res[0] = d;
        s_res[1] = static_cast<int>(run);
        s_res[2] = static_cast<int>(c[j]);
      }
      run += c[j];
    }
    reinterpret_cast<uint4*>(s_cur)[(2040 - 8 * tid) >> 2] = make_uint4(ex[7], ex[6], ex[5], ex[4]);
    reinterpret_cast<uint4*>(s_cur)[(2044 - 8 * tid) >> 2] = make_uint4(ex[3], ex[2], ex[1], ex[0]);
    __syncthreads();
    const int B = s_res[0], above = s_res[1], cntB = s_res[2];
    uint32_t mc = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (2047 - 8 * tid - j >= B) mc = c[j] > mc ? c[j] : mc;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const uint32_t v = __shfl_xor_sync(0xFFFFFFFFu, mc, off);
      mc = v > mc ? v : mc;
    }
    if (lane == 0) atomicMax(&s_maxc, static_cast<int>(mc));
    __syncthreads();
    const int nw = above + cntB;  // records in bucket B and above
    if (nw <= kWinCap && s_maxc <= kRankMax) {
      for (int base = tid; base < n_st; base += kBatch * NT) {
        uint64_t r[kBatch];
        uint32_t pos[kBatch];
#pragma unroll
        for (int j = 0; j < kBatch; ++j) r[j] = base + j * NT < n_st ? s_rec[base + j * NT] : 0ull;
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
          const uint32_t d = r[j] != 0ull ? digit(r[j]) : 0u;
          pos[j] = (r[j] != 0ull && static_cast<int>(d) >= B) ? atomicAdd(&s_cur[d], 1u) : 0xFFFFFFFFu;
        }
#pragma unroll
        for (int j = 0; j < kBatch; ++j)
          if (pos[j] != 0xFFFFFFFFu) s_win[pos[j]] = r[j];
      }
      __syncthreads();
      // s_cur[d] is now the end of bucket d; rank each record inside its
      // bucket and place the winners in order in the (now free) staging buffer
      for (int base = tid; base < nw; base += kBatch * NT) {
        uint64_t r[kBatch];
        int beg[kBatch], end[kBatch];
#pragma unroll
        for (int j = 0; j < kBatch; ++j) r[j] = base + j * NT < nw ? s_win[base + j * NT] : 0ull;
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
          const uint32_t d = r[j] != 0ull ? digit(r[j]) : 0u;
          end[j] = static_cast<int>(s_cur[d]);
          beg[j] = r[j] != 0ull ? end[j] - static_cast<int>(s_hist[d]) : end[j];
        }
        // the batch's bucket scans advance together (independent loads)
        int rank[kBatch], len = 0;
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
          rank[j] = 0;
          len = max(len, end[j] - beg[j]);
        }
        for (int x = 0; x < len; x += 2) {
#pragma unroll
          for (int j = 0; j < kBatch; ++j) {
            const uint64_t a0 = beg[j] + x < end[j] ? s_win[beg[j] + x] : 0ull;
            const uint64_t a1 = beg[j] + x + 1 < end[j] ? s_win[beg[j] + x + 1] : 0ull;
            rank[j] += (a0 > r[j] ? 1 : 0) + (a1 > r[j] ? 1 : 0);
          }
        }
#pragma unroll
        for (int j = 0; j < kBatch; ++j)
          if (r[j] != 0ull && beg[j] + rank[j] < m) s_rec[beg[j] + rank[j]] = r[j];
      }
      __syncthreads();
      for (int i = tid; i < p.topk; i += NT) put(i, i < m ? s_rec[i] : 0ull);
      done = true;
    }
    __syncthreads();
  }
  if (done) return;

  // ---- radix-select + bitonic-sort path
  uint64_t thr = 1;  // records are >= 1: keeps all
  if (m > 0 && m < n) {
    uint64_t prefix = 0;
    int pbits = 0, above = 0;
    if (staged) {
      // start the digits at the highest bit in which the records differ
      // (s_lo / s_hi bracket the records; the counting path reduced them)
      const uint64_t diff = s_lo ^ s_hi;  // non-zero: records are distinct
      pbits = __clzll(static_cast<long long>(diff));
      prefix = pbits > 0 ? (s_hi >> (64 - pbits)) : 0ull;
    }
    for (int pass = 0; pass < 7; ++pass) {
      const int shift = max(64 - pbits - 11, 0);
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
            bool ok = v[j] != 0ull;
            if (pbits > 0) ok = ok && ((v[j] >> (64 - pbits)) == prefix);
            hist_add_blk(s_hist, ok, static_cast<uint32_t>(v[j] >> shift) & static_cast<uint32_t>(nb - 1));
          }
        }
      };
      if (staged) {
        hist_pass(s_rec, n_st);
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
        thr = (pbits == 64) ? prefix : (prefix << (64 - pbits));
        break;
      }
      above = new_above;
      __syncthreads();
    }
  }

  // gather the m winners (in any order) into s_win
  auto gather = [&](const uint64_t* buf, int cnt) {
    for (int base = 0; base < cnt; base += NT) {
      const int i = base + tid;
      const uint64_t r = (i < cnt) ? buf[i] : 0ull;
      const bool keep = (i < cnt) && (r >= thr) && (r != 0ull);
      const uint32_t bal = __ballot_sync(0xFFFFFFFFu, keep);
      if (bal) {
        int pos = 0;
        if (lane == 0) pos = atomicAdd(&s_pos, __popc(bal));
        pos = __shfl_sync(0xFFFFFFFFu, pos, 0);
        const int at = pos + __popc(bal & lanemask_lt());
        if (keep && at < kMaxTopk) s_win[at] = r;
      }
    }
  };
  if (staged) {
    gather(s_rec, n_st);
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
  for (int s = 0; s < 8; ++s) {
    const int i = 8 * tid + s;
    v[s] = (i < m) ? s_win[i] : 0ull;
  }
  __syncthreads();
  sort2048_desc(v, s_win);
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const int i = 8 * tid + s;
    if (i < p.topk) put(i, i < m ? v[s] : 0ull);
  }
}

cudaError_t launch_select(const SelectParams& p, cudaStream_t stream) {
  if (p.n_rows <= 0) return cudaSuccess;
  constexpr int NT = kSelectThreads;
  const size_t smem = (kStageRecs + kWinCap) * sizeof(uint64_t);
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(select_topk_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  select_topk_kernel<NT><<<static_cast<unsigned>(p.n_rows), NT, smem, stream>>>(p);
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
