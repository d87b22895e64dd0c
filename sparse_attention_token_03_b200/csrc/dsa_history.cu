// Seed keys from historical selection frequency (163.com DoSA write-up,
// section 03: the seed set of a chunk may be taken from the keys that earlier
// rows selected most often).
//
// Given the Top-k index lists of earlier rows, the seeds are the n_seed keys
// below n_keys with the largest selection counts, ties going to the smaller
// key, written in ascending key order.  An exact top-n_seed by
// (count desc, key asc) over a count array:
//
//   count_kernel      counts[s] += 1 for every list entry s in [0, n_keys)
//   hist_kernel x2    radix histogram of the counts, high then low 16 bits
//   pick_kernel x2    one block: the bin holding the n_seed-th largest count
//                     -> the cut-off count c* and how many keys at c* to take
//   tile_kernel       per tile of 1024 keys: keys above c*, keys at c*
//   scan_kernel       one block: exclusive prefix of both over the tiles
//   scatter_kernel    keys above c*, and the first keys at c* in key order,
//                     to their ascending-order slot
//
// Nothing here is floating point: the result is unique and exact.
#include <algorithm>

#include "dsa_dosa.cuh"

namespace dsa {

namespace {

constexpr int kBins = 65536;
constexpr int kPickThreads = 1024;
constexpr int kBinsPerThread = kBins / kPickThreads;
constexpr int kHistTile = 1024;

// Control words (in the workspace, zeroed with the counts).
struct HistCtl {
  uint32_t hi;       // high 16 bits of c*
  uint32_t need;     // keys still to take at the start of a pass
  uint32_t cstar;    // the cut-off count
  uint32_t take_eq;  // keys with count == c* to take (the smallest ones)
};

__global__ void count_kernel(const int32_t* __restrict__ prev, int64_t n, int64_t n_keys,
                             uint32_t* __restrict__ counts) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
    const int32_t s = __ldcs(prev + i);
    if (s >= 0 && s < n_keys) atomicAdd(counts + s, 1u);
  }
}

// Pass 0 bins every count by its high 16 bits; pass 1 bins, by the low 16
// bits, the counts whose high bits equal ctl->hi.  Lanes of a warp that hit
// the same bin add once (most counts share a few small values).
__global__ void hist_kernel(const uint32_t* __restrict__ counts, int64_t n_keys, int pass,
                            const HistCtl* __restrict__ ctl, uint32_t* __restrict__ hist) {
  const int lane = threadIdx.x & 31;
  const uint32_t hi = pass ? ctl->hi : 0u;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * blockDim.x + (threadIdx.x & ~31); base < n_keys;
       base += stride) {
    const int64_t i = base + lane;
    bool ok = i < n_keys;
    const uint32_t c = ok ? counts[i] : 0u;
    if (pass) ok = ok && (c >> 16) == hi;
    const uint32_t bin = pass ? (c & 0xFFFFu) : (c >> 16);
    const uint32_t act = __ballot_sync(0xFFFFFFFFu, ok);
    if (ok) {
      const uint32_t peers = __match_any_sync(act, bin);
      if (lane == __ffs(peers) - 1) atomicAdd(hist + bin, static_cast<uint32_t>(__popc(peers)));
    }
  }
}

// Inclusive prefix sum over the block's threads (blockDim.x == 1024).
__device__ uint32_t block_inclusive_scan(uint32_t v, uint32_t* s_warp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t u = __shfl_up_sync(0xFFFFFFFFu, v, o);
    if (lane >= o) v += u;
  }
  if (lane == 31) s_warp[warp] = v;
  __syncthreads();
  if (warp == 0) {
    uint32_t t = s_warp[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_up_sync(0xFFFFFFFFu, t, o);
      if (lane >= o) t += u;
    }
    s_warp[lane] = t;
  }
  __syncthreads();
  const uint32_t r = v + (warp > 0 ? s_warp[warp - 1] : 0u);
  __syncthreads();
  return r;
}

// One block of 1024 threads.  Thread j owns bins [64 (1023 - j), 64 (1024 - j)),
// so the inclusive scan runs from the top bin down: `above` = keys in
// higher bins.  The owner of the bin holding the need-th largest count walks
// its bins downwards to find it.  The histogram is left zeroed.
__global__ void __launch_bounds__(kPickThreads) pick_kernel(uint32_t* __restrict__ hist, int pass, int n_seed,
                                                           HistCtl* __restrict__ ctl) {
  __shared__ uint32_t s_warp[32];
  const int j = threadIdx.x;
  const int lo = (kPickThreads - 1 - j) * kBinsPerThread;
  uint32_t sum = 0;
#pragma unroll 4
  for (int b = 0; b < kBinsPerThread; ++b) sum += hist[lo + b];
  const uint32_t need = pass ? ctl->need : static_cast<uint32_t>(n_seed);
  const uint32_t incl = block_inclusive_scan(sum, s_warp);
  uint32_t above = incl - sum;
  if (sum > 0 && above < need && need <= incl) {
#pragma unroll 1
    for (int b = kBinsPerThread - 1; b >= 0; --b) {
      const uint32_t h = hist[lo + b];
      if (above + h >= need) {
        const uint32_t bin = static_cast<uint32_t>(lo + b);
        if (pass == 0) {
          ctl->hi = bin;
          ctl->need = need - above;
        } else {
          ctl->cstar = (ctl->hi << 16) | bin;
          ctl->take_eq = need - above;
        }
        break;
      }
      above += h;
    }
  }
  __syncthreads();
#pragma unroll 4
  for (int b = 0; b < kBinsPerThread; ++b) hist[lo + b] = 0u;
}

__global__ void __launch_bounds__(kHistTile) tile_kernel(const uint32_t* __restrict__ counts, int64_t n_keys,
                                                        const HistCtl* __restrict__ ctl,
                                                        uint32_t* __restrict__ tile_gt,
                                                        uint32_t* __restrict__ tile_eq) {
  __shared__ uint32_t s_gt[32], s_eq[32];
  const int64_t i = static_cast<int64_t>(blockIdx.x) * kHistTile + threadIdx.x;
  const uint32_t cstar = ctl->cstar;
  const uint32_t c = i < n_keys ? counts[i] : 0u;
  const bool valid = i < n_keys;
  const uint32_t gt = __popc(__ballot_sync(0xFFFFFFFFu, valid && c > cstar));
  const uint32_t eq = __popc(__ballot_sync(0xFFFFFFFFu, valid && c == cstar));
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) {
    s_gt[warp] = gt;
    s_eq[warp] = eq;
  }
  __syncthreads();
  if (warp == 0) {
    uint32_t a = s_gt[lane], e = s_eq[lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      a += __shfl_xor_sync(0xFFFFFFFFu, a, o);
      e += __shfl_xor_sync(0xFFFFFFFFu, e, o);
    }
    if (lane == 0) {
      tile_gt[blockIdx.x] = a;
      tile_eq[blockIdx.x] = e;
    }
  }
}

// Exclusive prefix over the tiles, in place, 1024 tiles per round.
__global__ void __launch_bounds__(kPickThreads) scan_kernel(uint32_t* __restrict__ tile_gt,
                                                           uint32_t* __restrict__ tile_eq, int64_t n_tiles) {
  __shared__ uint32_t s_warp[32];
  uint32_t carry_gt = 0, carry_eq = 0;
  for (int64_t base = 0; base < n_tiles; base += kPickThreads) {
    const int64_t t = base + threadIdx.x;
    const uint32_t g = t < n_tiles ? tile_gt[t] : 0u;
    const uint32_t e = t < n_tiles ? tile_eq[t] : 0u;
    const uint32_t ig = block_inclusive_scan(g, s_warp);
    const uint32_t ie = block_inclusive_scan(e, s_warp);
    if (t < n_tiles) {
      tile_gt[t] = carry_gt + ig - g;
      tile_eq[t] = carry_eq + ie - e;
    }
    // the last thread's inclusive sums are the round's totals
    if (threadIdx.x == kPickThreads - 1) {
      s_warp[0] = ig;
      s_warp[1] = ie;
    }
    __syncthreads();
    carry_gt += s_warp[0];
    carry_eq += s_warp[1];
    __syncthreads();
  }
}

__global__ void __launch_bounds__(kHistTile) scatter_kernel(const uint32_t* __restrict__ counts, int64_t n_keys,
                                                           const HistCtl* __restrict__ ctl,
                                                           const uint32_t* __restrict__ pre_gt,
                                                           const uint32_t* __restrict__ pre_eq,
                                                           int32_t* __restrict__ seeds) {
  __shared__ uint32_t s_warp[32];
  const int64_t i = static_cast<int64_t>(blockIdx.x) * kHistTile + threadIdx.x;
  const uint32_t cstar = ctl->cstar, take_eq = ctl->take_eq;
  const bool valid = i < n_keys;
  const uint32_t c = valid ? counts[i] : 0u;
  const bool gt = valid && c > cstar, eq = valid && c == cstar;
  // both flags in one scan: keys above c* in the high half, at c* in the low
  const uint32_t v = (gt ? 0x10000u : 0u) | (eq ? 1u : 0u);
  const uint32_t ex = block_inclusive_scan(v, s_warp) - v;
  const uint32_t gt_before = pre_gt[blockIdx.x] + (ex >> 16);
  const uint32_t eq_before = pre_eq[blockIdx.x] + (ex & 0xFFFFu);
  if (gt || (eq && eq_before < take_eq)) seeds[gt_before + min(eq_before, take_eq)] = static_cast<int32_t>(i);
}

}  // namespace

cudaError_t launch_history_seeds(const HistoryParams& p, cudaStream_t st) {
  HistCtl* ctl = reinterpret_cast<HistCtl*>(p.ctl);
  const int64_t n = p.n_rows * p.topk;
  const int64_t n_tiles = (p.n_keys + kHistTile - 1) / kHistTile;
  const int cap = p.num_sms * 8;
  if (n > 0) {
    const int grid = static_cast<int>(std::min<int64_t>((n + 255) / 256, cap));
    count_kernel<<<grid, 256, 0, st>>>(p.prev, n, p.n_keys, p.counts);
  }
  const int hgrid = static_cast<int>(std::min<int64_t>((p.n_keys + 255) / 256, cap));
  for (int pass = 0; pass < 2; ++pass) {
    hist_kernel<<<hgrid, 256, 0, st>>>(p.counts, p.n_keys, pass, ctl, p.hist);
    pick_kernel<<<1, kPickThreads, 0, st>>>(p.hist, pass, p.n_seed, ctl);
  }
  tile_kernel<<<static_cast<unsigned>(n_tiles), kHistTile, 0, st>>>(p.counts, p.n_keys, ctl, p.tile_gt, p.tile_eq);
  scan_kernel<<<1, kPickThreads, 0, st>>>(p.tile_gt, p.tile_eq, n_tiles);
  scatter_kernel<<<static_cast<unsigned>(n_tiles), kHistTile, 0, st>>>(p.counts, p.n_keys, ctl, p.tile_gt,
                                                                      p.tile_eq, p.seeds);
  return cudaGetLastError();
}

}  // namespace dsa
