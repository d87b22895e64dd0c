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

template <int NT>
__device__ __forceinline__ void hist_add_blk(uint32_t* hist, bool valid, uint32_t digit) {
  const uint32_t key = valid ? digit : 0xFFFFFFFFu;
  const uint32_t peers = __match_any_sync(0xFFFFFFFFu, key);
  if (valid && (threadIdx.x & 31) == (__ffs(peers) - 1)) atomicAdd(&hist[digit], __popc(peers));
}

// Block-wide: largest bucket B with above + sum_{d >= B} hist[d] >= need.
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

}  // namespace

template <int NT>
__global__ void __launch_bounds__(NT) select_topk_kernel(const SelectParams p) {
  __shared__ uint32_t s_hist[2048];
  __shared__ uint64_t s_sort[kMaxTopk];
  __shared__ int s_scratch[NT / 32];
  __shared__ int s_res[4];
  __shared__ int s_n;
  __shared__ int s_pos;

  const int64_t row = blockIdx.x;
  const int tid = threadIdx.x;
  const RowUnits R = row_units(p, row);
  const int G = (p.mode == kModeDecode) ? 1 : p.G;

  if (tid == 0) {
    int n = 0;
    for (int u = 0; u < R.n_u; ++u) {
      const int c = p.meta[(static_cast<size_t>(R.slot_lo + u) * G + R.q) * 2];
      n += min(max(c, 0), p.cap);
    }
    s_n = n;
    s_pos = 0;
  }
  __syncthreads();
  const int n = s_n;
  const int m = min(p.topk, n);

  auto unit_buf = [&](int u, int& cnt) -> const uint64_t* {
    const int32_t* mt = p.meta + (static_cast<size_t>(R.slot_lo + u) * G + R.q) * 2;
    cnt = min(max(mt[0], 0), p.cap);  // counts are always in range; clamp defensively
    return p.cand + ((static_cast<size_t>(R.slot_lo + u) * G + R.q) * 2 + (mt[1] & 1)) *
                        static_cast<size_t>(p.cap);
  };

  uint64_t thr = 0;  // every record is > 0, so thr = 0 keeps all
  if (m > 0 && m < n) {
    uint64_t prefix = 0;
    int pbits = 0, above = 0;
    for (int pass = 0; pass < 6; ++pass) {
      const int shift = max(64 - 11 * (pass + 1), 0);
      const int width = 64 - pbits - shift;
      const int nb = 1 << width;
      for (int i = tid; i < nb; i += NT) s_hist[i] = 0;
      __syncthreads();
      for (int u = 0; u < R.n_u; ++u) {
        int cnt;
        const uint64_t* buf = unit_buf(u, cnt);
        for (int base = 0; base < cnt; base += NT) {
          const int i = base + tid;
          bool ok = i < cnt;
          const uint64_t r = ok ? buf[i] : 0ull;
          if (pbits > 0) ok = ok && ((r >> (64 - pbits)) == prefix);
          hist_add_blk<NT>(s_hist, ok, static_cast<uint32_t>(r >> shift) & static_cast<uint32_t>(nb - 1));
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

  // gather the winners
  for (int u = 0; u < R.n_u; ++u) {
    int cnt;
    const uint64_t* buf = unit_buf(u, cnt);
    for (int base = 0; base < cnt; base += NT) {
      const int i = base + tid;
      const uint64_t r = (i < cnt) ? buf[i] : 0ull;
      const bool keep = (i < cnt) && (r >= thr) && (r != 0ull);
      const uint32_t bal = __ballot_sync(0xFFFFFFFFu, keep);
      if (bal) {
        int pos = 0;
        if ((tid & 31) == 0) pos = atomicAdd(&s_pos, __popc(bal));
        pos = __shfl_sync(0xFFFFFFFFu, pos, 0);
        const int at = pos + __popc(bal & lanemask_lt());
        if (keep && at < kMaxTopk) s_sort[at] = r;
      }
    }
  }
  __syncthreads();
  const int got = s_pos;
  if (got != m && tid == 0) atomicOr(p.err, kErrOverflow);  // never expected
  int P2 = 1;
  while (P2 < m) P2 <<= 1;
  for (int i = m + tid; i < P2; i += NT) s_sort[i] = 0ull;
  __syncthreads();
  // bitonic sort, descending
  for (int k = 2; k <= P2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < P2; i += NT) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const uint64_t a = s_sort[i], b = s_sort[ixj];
          const bool desc = (i & k) == 0;
          if (desc ? (a < b) : (a > b)) {
            s_sort[i] = b;
            s_sort[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  const size_t o = static_cast<size_t>(row) * p.topk;
  for (int i = tid; i < p.topk; i += NT) {
    const bool v = i < m;
    const uint64_t r = v ? s_sort[i] : 0ull;
    if (p.out_idx) p.out_idx[o + i] = v ? static_cast<int32_t>(record_key(r)) : -1;
    if (p.out_score) p.out_score[o + i] = v ? record_score(r) : -INFINITY;
    if (p.out_rec) p.out_rec[o + i] = r;
  }
  if (p.out_kth && tid == 0) p.out_kth[row] = (m > 0) ? record_score(s_sort[m - 1]) : -INFINITY;
}

cudaError_t launch_select(const SelectParams& p, cudaStream_t stream) {
  if (p.n_rows <= 0) return cudaSuccess;
  select_topk_kernel<kSelectThreads><<<static_cast<unsigned>(p.n_rows), kSelectThreads, 0, stream>>>(p);
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
