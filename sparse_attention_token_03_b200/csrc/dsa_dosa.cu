// Support kernels of the DoSA certified-pruning path ("DoSA: Dots Sparse
// Attention", steps 1-3; 163.com write-up, sections 03-04).
//
//   seed_prep_kernel    validate the seed list, mark it in a key bitmap and
//                       gather the seed keys into a contiguous matrix
//   keynorm_kernel      ||k_s|| for every key, rounded up
//   plan_kernel         per query row: retained heads, least-squares residual
//                       bound, folded positive / negative auxiliary rows and
//                       the scalars of the screening bound
//   compact_kernel      survivor bitmask -> ascending survivor id list per row
//   decide_kernel       after the probe rows: keep pruning or send the rest of
//                       the chunk to the dense path
//   stats_kernel        counters for the dsa_stats struct
//
// The screening MMA and the exact refine are variants of the fused score
// kernel (dsa_score.cu); the final merge is the shared select kernel.
#include <cfloat>

#include "dsa_dosa.cuh"
#include "dsa_ptx.cuh"

namespace dsa {

namespace {

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

// Round an fp32 value to bf16 (nearest, ties to even); finite inputs.
__device__ __forceinline__ uint16_t f32_to_bf16(float f) {
  uint32_t u = __float_as_uint(f);
  const uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return static_cast<uint16_t>(u >> 16);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

}  // namespace

// ---------------------------------------------------------------------------
// Seeds: every seed must be a distinct key visible to every row of the chunk
// (0 <= seed < q_offset), so that the topk-th largest seed score is a lower
// bound on every row's true topk-th score ("DoSA", step 1).
// ---------------------------------------------------------------------------
__global__ void seed_prep_kernel(const SeedPrepParams p) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;  // one thread per (seed, 16-byte chunk)
  const int seed = i >> 4, chunk = i & 15;
  if (seed >= p.n_seed) return;
  int32_t id = p.seed_idx[seed];
  if (id < 0 || id >= p.q_offset) {
    if (chunk == 0) atomicOr(p.err, kErrSeed);
    id = 0;  // gather something in bounds; the call recovers densely
  } else if (chunk == 0) {
    const uint32_t bit = 1u << (id & 31);
    const uint32_t old = atomicOr(&p.seed_bits[id >> 5], bit);
    if (old & bit) atomicOr(p.err, kErrSeed);  // duplicate
  }
  const uint4* src = reinterpret_cast<const uint4*>(p.k + static_cast<size_t>(id) * kD);
  uint4* dst = reinterpret_cast<uint4*>(p.k_seed + static_cast<size_t>(seed) * kD);
  dst[chunk] = src[chunk];
}

// ||k_s|| in fp32, rounded up by a relative 2^-12 so that it bounds the exact
// norm despite the fp32 sum of squares.
__global__ void keynorm_kernel(const uint16_t* __restrict__ k, int64_t T_k, float* __restrict__ knorm) {
  const int64_t key = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 4;
  const int part = threadIdx.x & 15;  // 16 lanes per key, 8 values each
  float acc = 0.0f;
  if (key < T_k) {
    const uint4 v = reinterpret_cast<const uint4*>(k + key * kD)[part];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float lo = __uint_as_float(w[j] << 16), hi = __uint_as_float(w[j] & 0xFFFF0000u);
      acc = fmaf(lo, lo, acc);
      acc = fmaf(hi, hi, acc);
    }
  }
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
  if (key < T_k && part == 0) knorm[key] = sqrtf(acc) * (1.0f + 1.0f / 4096.0f);
}

// ---------------------------------------------------------------------------
// Screening plan of one query row (one CTA of 128 threads per row).
//
//  importance_j = |w_j| * sum over sampled seeds s of max(q_j . k_s, 0)
//  R            = the kRetained heads of largest importance (ties: smaller j)
//  P / N        = omitted heads with w_j > 0 / w_j < 0
//  for j in P   c_j = least-squares coefficients of q_j on {q_i, i in R}
//               (zero if the Gram matrix is not positive definite: any
//               coefficients keep the bound valid), rho_j = ||q_j - sum c q_i||
//  alpha_i = sum_P w_j |c_ji|,  beta = sum_P w_j rho_j
//  q_pos = sum_P w_j q_j, q_neg = sum_N |w_j| q_j (rounded to bf16 for the MMA)
// With d = q . k, the screening bound is
//  U = sum_R [w_i max(d_i,0) + alpha_i |d_i| / 2] + d_pos/2 - max(d_neg,0) + C ||k||,
// evaluated (w max(d,0) = w d/2 + w |d|/2) as
//  U = L . k + sum_R c_i |d_i| - max(d_neg,0) + C ||k||,
//  L = q_pos/2 + sum_R (w_i/2) q_i,   c_i = (w_i + alpha_i)/2,
//  C = beta/2 + ||L - bf16(L)|| + ||q_neg - bf16(q_neg)|| + 2^-10 S,
//  S = sum_j |w_j| ||q_j|| + ||q_pos|| + ||q_neg|| + sum_R alpha_i ||q_i||,
// where the last term absorbs the fp32 tensor-core accumulation and the fp32
// arithmetic of the bound and of the exact score (each far below 2^-10 S ||k||).
// Plan rows: the retained q_i, then L, then q_neg (bf16).
// ---------------------------------------------------------------------------
template <int H>
__global__ void __launch_bounds__(128) plan_kernel(const PlanParams p) {
  constexpr int NT = 128, NSAMP = 64, R = kRetained;
  __shared__ uint16_t qf[H][kD + 2];  // bf16 bits (padded rows: no bank conflicts)
  __shared__ uint16_t kf[NSAMP][kD];  // bf16 bits
  __shared__ float part[NT];
  __shared__ float imp[H];
  __shared__ float qn[H];      // ||q_j||
  __shared__ int sel[R];
  __shared__ double Lc[R][R];  // Cholesky factor of the retained Gram matrix
  __shared__ int chol_ok;
  __shared__ float coef[4][R];  // per-warp least-squares coefficients
  __shared__ float wal[4][R];   // per-warp alpha partials
  __shared__ float wbe[4];      // per-warp beta partials

  if (p.skip && *p.skip) return;
  const int t = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const uint16_t* qrow = p.q + static_cast<size_t>(t) * H * kD;
  const float* wrow = p.w + static_cast<size_t>(t) * H;

  for (int i = tid; i < H * kD; i += NT) qf[i / kD][i % kD] = qrow[i];
  const int nsamp = p.n_seed < NSAMP ? p.n_seed : NSAMP;
  for (int i = tid; i < nsamp * kD; i += NT) {
    const int s = i / kD;
    const int pos = static_cast<int>(((2LL * s + 1) * p.n_seed) / (2LL * nsamp));
    kf[s][i % kD] = p.k_seed[static_cast<size_t>(pos) * kD + (i % kD)];
  }
  __syncthreads();

  // importance: NT / H threads per head, each over a fixed slice of samples,
  // four samples at a time (four independent FMA chains, each over e in
  // ascending order) reading bf16 pairs
  {
    constexpr int TPH = NT / H;
    const int j = tid % H, slice = tid / H;
    const uint32_t* qj = reinterpret_cast<const uint32_t*>(&qf[j][0]);
    float acc = 0.0f;
    for (int s0 = slice; s0 < nsamp; s0 += 4 * TPH) {
      const uint32_t* ks[4];
      float d[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int sm = s0 + m * TPH;
        ks[m] = reinterpret_cast<const uint32_t*>(&kf[sm < nsamp ? sm : 0][0]);
        d[m] = 0.0f;
      }
#pragma unroll 4
      for (int e2 = 0; e2 < kD / 2; ++e2) {
        const uint32_t qp = qj[e2];
        const float q0 = __uint_as_float(qp << 16), q1 = __uint_as_float(qp & 0xFFFF0000u);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const uint32_t kp = ks[m][e2];
          d[m] = fmaf(q0, __uint_as_float(kp << 16), d[m]);
          d[m] = fmaf(q1, __uint_as_float(kp & 0xFFFF0000u), d[m]);
        }
      }
#pragma unroll
      for (int m = 0; m < 4; ++m)
        if (s0 + m * TPH < nsamp) acc += fmaxf(d[m], 0.0f);
    }
    part[tid] = acc;
    __syncthreads();
    if (tid < H) {
      float v = 0.0f;
      for (int sl = 0; sl < TPH; ++sl) v += part[sl * H + tid];
      imp[tid] = fabsf(wrow[tid]) * v;
    }
    // ||q_j||
    if (tid < H) {
      float n2 = 0.0f;
      for (int e = 0; e < kD; ++e) n2 = fmaf(bf16_to_f32(qf[tid][e]), bf16_to_f32(qf[tid][e]), n2);
      qn[tid] = sqrtf(n2) * (1.0f + 1.0f / 4096.0f);
    }
    __syncthreads();
  }
  // retained heads: largest importance first, smaller index on ties (warp 0:
  // lane l holds heads l and l + 32; importances are >= 0, -1 marks taken)
  if (wid == 0) {
    float v0 = lane < H ? imp[lane] : -1.0f, v1 = lane + 32 < H ? imp[lane + 32] : -1.0f;
    for (int a = 0; a < R; ++a) {
      float bv = v0;
      int bi = lane;
      if (v1 > v0) {
        bv = v1;
        bi = lane + 32;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, o);
        const int oi = __shfl_xor_sync(0xFFFFFFFFu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) {
          bv = ov;
          bi = oi;
        }
      }
      if (lane == 0) sel[a] = bi;
      if (bi == lane) v0 = -1.0f;
      if (bi == lane + 32) v1 = -1.0f;
    }
  }
  __syncthreads();
  // Gram matrix of the retained rows (fp32 dots, fp64 factorisation)
  for (int ab = wid; ab < R * R; ab += 4) {
    const int a = ab / R, b = ab % R;
    if (b > a) continue;
    float v = 0.0f;
    for (int e = lane; e < kD; e += 32) v = fmaf(bf16_to_f32(qf[sel[a]][e]), bf16_to_f32(qf[sel[b]][e]), v);
    v = warp_sum(v);
    if (lane == 0) Lc[a][b] = v;
  }
  __syncthreads();
  if (wid == 0) {
    // Cholesky, one column per step: the diagonal from a warp sum, then lane i
    // (j < i < R) finishes L[i][j]
    bool ok = true;
    for (int j = 0; j < R; ++j) {
      double sq = lane < j ? Lc[j][lane] * Lc[j][lane] : 0.0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xFFFFFFFFu, sq, o);
      const double s = Lc[j][j] - sq;
      if (!(s > 1e-9 * (1.0 + fabs(Lc[j][j])))) {
        ok = false;
        break;
      }
      const double ljj = sqrt(s);
      if (lane > j && lane < R) {
        double v = Lc[lane][j];
        for (int k2 = 0; k2 < j; ++k2) v -= Lc[lane][k2] * Lc[j][k2];
        Lc[lane][j] = v / ljj;
      }
      __syncwarp();
      if (lane == 0) Lc[j][j] = ljj;
      __syncwarp();
    }
    if (lane == 0) chol_ok = ok ? 1 : 0;
  }
  for (int i = tid; i < 4 * R; i += NT) (&wal[0][0])[i] = 0.0f;
  if (tid < 4) wbe[tid] = 0.0f;
  __syncthreads();

  // positive omitted heads: one warp per head, warps take heads in turn
  for (int j = wid; j < H; j += 4) {
    bool retained = false;
    for (int a = 0; a < R; ++a) retained = retained || (sel[a] == j);
    const float wj = wrow[j];
    if (retained || !(wj > 0.0f)) continue;
    float b[R];
#pragma unroll
    for (int a = 0; a < R; ++a) {
      float v = 0.0f;
      for (int e = lane; e < kD; e += 32) v = fmaf(bf16_to_f32(qf[sel[a]][e]), bf16_to_f32(qf[j][e]), v);
      b[a] = warp_sum(v);
    }
    // G c = b by the two triangular solves, lane a holding entry a: after
    // entry i is final, the lanes below (forward) / above (backward) update
    double x = 0.0;
#pragma unroll
    for (int a = 0; a < R; ++a)
      if (lane == a && chol_ok) x = static_cast<double>(b[a]);
    if (chol_ok) {
      for (int i = 0; i < R; ++i) {
        const double xi = __shfl_sync(0xFFFFFFFFu, x, i) / Lc[i][i];
        if (lane == i) x = xi;
        if (lane > i && lane < R) x -= Lc[lane][i] * xi;
      }
      for (int i = R - 1; i >= 0; --i) {
        const double xi = __shfl_sync(0xFFFFFFFFu, x, i) / Lc[i][i];
        if (lane == i) x = xi;
        if (lane < i) x -= Lc[i][lane] * xi;
      }
    }
    if (lane < R) coef[wid][lane] = static_cast<float>(x);
    __syncwarp();
    float r2 = 0.0f;
    for (int e = lane; e < kD; e += 32) {
      float r = bf16_to_f32(qf[j][e]);
      for (int a = 0; a < R; ++a) r = fmaf(-coef[wid][a], bf16_to_f32(qf[sel[a]][e]), r);
      r2 = fmaf(r, r, r2);
    }
    r2 = warp_sum(r2);
    if (lane == 0) {
      const float rho = sqrtf(r2) * (1.0f + 1.0f / 4096.0f);
      wbe[wid] += wj * rho;
      for (int a = 0; a < R; ++a) wal[wid][a] += wj * fabsf(coef[wid][a]);
    }
    __syncwarp();
  }
  __syncthreads();

  // folded auxiliary rows (thread e owns element e), in ascending head
  // order: the positive omitted heads' q_pos, the negative ones' q_neg, and
  // the linear row L = q_pos / 2 + sum_R (w_i / 2) q_i, which carries the
  // linear half of the bound (w max(d, 0) = w d / 2 + w |d| / 2) into the MMA
  {
    const int e = tid;
    float pos = 0.0f, neg = 0.0f;
    for (int j = 0; j < H; ++j) {
      bool retained = false;
      for (int a = 0; a < R; ++a) retained = retained || (sel[a] == j);
      if (retained) continue;
      const float wj = wrow[j];
      if (wj > 0.0f) pos = fmaf(wj, bf16_to_f32(qf[j][e]), pos);
      else if (wj < 0.0f) neg = fmaf(-wj, bf16_to_f32(qf[j][e]), neg);
    }
    float lin = 0.5f * pos;
    for (int a = 0; a < R; ++a) lin = fmaf(0.5f * wrow[sel[a]], bf16_to_f32(qf[sel[a]][e]), lin);
    const uint16_t bl = f32_to_bf16(lin), bn = f32_to_bf16(neg);
    uint16_t* prow = p.plan_q + static_cast<size_t>(t) * kPlanRows * kD;
    prow[kRetained * kD + e] = bl;
    prow[(kRetained + 1) * kD + e] = bn;
    for (int a = 0; a < R; ++a) prow[a * kD + e] = qrow[sel[a] * kD + e];
    const float dl = lin - bf16_to_f32(bl), dn = neg - bf16_to_f32(bn);
    // reduce: ||pos||^2, ||neg||^2, ||dl||^2, ||dn||^2
    float v[4] = {pos * pos, neg * neg, dl * dl, dn * dn};
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = warp_sum(v[i]);
    __shared__ float r4[4][4];
    if (lane == 0)
      for (int i = 0; i < 4; ++i) r4[wid][i] = v[i];
    __syncthreads();
    if (tid == 0) {
      float n[4];
      for (int i = 0; i < 4; ++i) n[i] = sqrtf(((r4[0][i] + r4[1][i]) + r4[2][i]) + r4[3][i]) * (1.0f + 1.0f / 4096.0f);
      float alpha[R];
      float beta = ((wbe[0] + wbe[1]) + wbe[2]) + wbe[3];
      float S = 0.0f;
      for (int j = 0; j < H; ++j) S += fabsf(wrow[j]) * qn[j];
      S += n[0] + n[1];
      for (int a = 0; a < R; ++a) {
        alpha[a] = ((wal[0][a] + wal[1][a]) + wal[2][a]) + wal[3][a];
        S += alpha[a] * qn[sel[a]];
      }
      float* ps = p.plan_s + static_cast<size_t>(t) * kPlanScalars;
      for (int a = 0; a < R; ++a) {
        ps[a] = 0.5f * wrow[sel[a]] + 0.5f * alpha[a];  // coefficient of |d_a|
        ps[kRetained + a] = 0.0f;
      }
      // C: the residual term, the bf16 rounding of L and q_neg, and 2^-10 S
      // for the fp32 arithmetic (S bounds every product the bound sums)
      const float C = 0.5f * beta + n[2] + n[3] + S * (1.0f / 1024.0f);
      ps[28] = C * (1.0f + 1.0f / 1024.0f);
      ps[29] = p.tau[t];
      ps[30] = 0.0f;
      ps[31] = 0.0f;
    }
  }
}

// ---------------------------------------------------------------------------
// Survivor bitmask of one row -> ascending list of survivor key ids (one CTA
// of 256 threads per row).  Rows whose survivors exceed the list capacity, or
// all rows when the seed list was invalid, are flagged for the exact dense
// recovery pass and get an empty refine list.  Also sets the row's refine
// admission threshold: its topk-th seed record.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) compact_kernel(const CompactParams p) {
  __shared__ int s_scan[256 / 32];
  __shared__ int s_base;
  if (p.skip && *p.skip) return;
  const int t = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int count = p.surv_count[t];
  const bool bad_seed = (*p.err & kErrSeed) != 0;
  if (tid == 0) p.init_thr[t] = p.seed_rec[static_cast<size_t>(t) * p.rec_stride + p.topk - 1];
  if (bad_seed || count > p.cap_row) {
    if (tid == 0) {
      p.row_flags[t] = bad_seed ? kRowBadSeed : kRowOverflow;
      p.refine_len[t] = 0;
    }
    return;
  }
  if (tid == 0) {
    p.row_flags[t] = kRowRefined;
    s_base = 0;
  }
  __syncthreads();
  const int64_t pos = p.q_offset + t;
  const int64_t words = pos / 32 + 1;
  const uint32_t* bm = p.bitmask + static_cast<size_t>(t) * p.mask_words;
  int32_t* ids = p.surv_ids + static_cast<size_t>(t) * p.cap_row;
  // keys of the row's group's shared stream (in the words of the group's
  // common range) are refined there, not here
  const int g = t >> 2;
  const uint32_t* gm = (p.group_mask && p.group_len[g] > 0) ? p.group_mask + static_cast<size_t>(g) * p.mask_words
                                                            : nullptr;
  const int64_t gwords = (p.q_offset + 4 * static_cast<int64_t>(g)) / 32 + 1;
  for (int64_t base = 0; base < words; base += 256) {
    const int64_t wi = base + tid;
    uint32_t word = wi < words ? bm[wi] : 0u;
    if (gm && wi < gwords) word &= ~gm[wi];
    if (wi == words - 1 && (pos & 31) != 31) word &= (2u << (pos & 31)) - 1u;  // keys beyond pos
    const int c = __popc(word);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) s_scan[wid] = incl;
    __syncthreads();
    int before = s_base;
    for (int w2 = 0; w2 < wid; ++w2) before += s_scan[w2];
    int at = before + incl - c;
    while (word) {
      const int b = __ffs(word) - 1;
      word &= word - 1;
      if (at < p.cap_row) ids[at] = static_cast<int32_t>(wi * 32 + b);
      ++at;
    }
    __syncthreads();
    if (tid == 255) s_base = before + incl;
    __syncthreads();
  }
  if (tid == 0) p.refine_len[t] = min(s_base, p.cap_row);  // the row's own list
}

// ---------------------------------------------------------------------------
// Shared refine stream of one group of four consecutive rows (one CTA of 256
// threads per group; "DoSA" notes, annotation WFZZA9CL, step 3).  Only full
// groups whose four rows keep their survivor lists take part.  A key in the
// group's common range (keys 0 .. position of the group's first row) kept by
// at least two of the rows goes to the group's list: it is gathered once and
// scored exactly for all four rows; each row's own list leaves it out.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) share_kernel(const ShareParams p) {
  __shared__ int s_scan[256 / 32];
  __shared__ int s_base;
  if (p.skip && *p.skip) return;
  const int g = blockIdx.x;
  const int64_t t0 = 4 * static_cast<int64_t>(g);
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  bool share = t0 + 4 <= p.T_q && (*p.err & kErrSeed) == 0;
  for (int r = 0; r < 4 && share; ++r) share = p.surv_count[t0 + r] <= p.cap_row;
  if (!share) {
    if (tid == 0) p.group_len[g] = 0;
    return;
  }
  if (tid == 0) s_base = 0;
  __syncthreads();
  const int64_t pos = p.q_offset + t0;  // the group's first row sees keys 0..pos
  const int64_t words = pos / 32 + 1;
  const uint32_t* bm = p.bitmask + static_cast<size_t>(t0) * p.mask_words;
  uint32_t* gm = p.group_mask + static_cast<size_t>(g) * p.mask_words;
  int32_t* ids = p.group_ids + static_cast<size_t>(g) * p.cap_row;
  for (int64_t base = 0; base < words; base += 256) {
    const int64_t wi = base + tid;
    uint32_t word = 0u;
    if (wi < words) {
      const uint32_t a = bm[wi], b = bm[p.mask_words + wi], c = bm[2 * p.mask_words + wi],
                     d = bm[3 * p.mask_words + wi];
      word = (a & b) | (a & c) | (a & d) | (b & c) | (b & d) | (c & d);  // at least two of four
      if (wi == words - 1 && (pos & 31) != 31) word &= (2u << (pos & 31)) - 1u;
      gm[wi] = word;
    }
    const int cnt = __popc(word);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) s_scan[wid] = incl;
    __syncthreads();
    int before = s_base;
    for (int w2 = 0; w2 < wid; ++w2) before += s_scan[w2];
    int at = before + incl - cnt;
    while (word) {
      const int bit = __ffs(word) - 1;
      word &= word - 1;
      if (at < p.cap_row) ids[at] = static_cast<int32_t>(wi * 32 + bit);
      ++at;
    }
    __syncthreads();
    if (tid == 255) s_base = before + incl;
    __syncthreads();
  }
  if (tid == 0) p.group_len[g] = min(s_base, p.cap_row);
}

// ---------------------------------------------------------------------------
// Probe decision (one CTA of 256 threads).  The probe rows went through the
// whole pruned path; from them, estimate the pruned cost of a row relative to
// its dense cost:
//   kScreenCost                       screening every visible key
//   + kSeedCost * n_seed / v          scoring the seeds with all heads
//   + kPlanPairs / v                  the per-row plan
//   + overflow fraction               rows recomputed densely
//   + kRefineCost * refined / pairs   exact refine of the survivors
// (v = mean visible keys of a probe row).  The constants are the measured
// per-pair costs of these kernels on B200 relative to the dense kernel's
// (128K and 1M chunks).  When the estimate reaches 1 the remaining rows skip
// the pruned path and are marked for the dense pass.
// ---------------------------------------------------------------------------
constexpr float kScreenCost = 0.6f;
constexpr float kSeedCost = 1.6f;
constexpr float kPlanPairs = 15000.0f;
constexpr float kRefineCost = 10.0f;

__global__ void __launch_bounds__(256) decide_kernel(const DecideParams p) {
  __shared__ float s_red[3][8];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  float over = 0.0f, refined = 0.0f, vis = 0.0f;
  for (int64_t t = tid; t < p.probe_rows; t += 256) {
    const bool ok = p.row_flags[t] == kRowRefined;
    over += ok ? 0.0f : 1.0f;
    refined += ok ? static_cast<float>(p.surv_count[t]) : 0.0f;
    vis += static_cast<float>(p.q_offset + t + 1);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    over += __shfl_xor_sync(0xFFFFFFFFu, over, o);
    refined += __shfl_xor_sync(0xFFFFFFFFu, refined, o);
    vis += __shfl_xor_sync(0xFFFFFFFFu, vis, o);
  }
  if (lane == 0) {
    s_red[0][wid] = over;
    s_red[1][wid] = refined;
    s_red[2][wid] = vis;
  }
  __syncthreads();
  __shared__ int s_bypass;
  if (tid == 0) {
    float o = 0.0f, r = 0.0f, v = 0.0f;
    for (int i = 0; i < 8; ++i) {
      o += s_red[0][i];
      r += s_red[1][i];
      v += s_red[2][i];
    }
    const float n = static_cast<float>(p.probe_rows);
    const float vbar = v / n;
    const float est = kScreenCost + kSeedCost * static_cast<float>(p.n_seed) / vbar + kPlanPairs / vbar + o / n +
                      kRefineCost * r / v;
    s_bypass = est >= 1.0f ? 1 : 0;
    *p.bypass = static_cast<uint32_t>(s_bypass);
  }
  __syncthreads();
  if (!s_bypass) return;
  for (int64_t t = p.probe_rows + tid; t < p.T_q; t += 256) {
    p.row_flags[t] = kRowBypassed;
    p.refine_len[t] = 0;
  }
}

// Sums for dsa_stats (one CTA): out[0] survivor pairs, [1] refined pairs
// (exact scores computed: own lists, plus four per shared key), [2] rows
// recovered after screening, [3] bypassed rows, [4] screened pairs, [5]
// records the final selection read (seed Top-k + refined candidates of the
// rows it finished), [6] shared keys.
__global__ void __launch_bounds__(256) stats_kernel(const StatsParams p) {
  unsigned long long a = 0, b = 0, c = 0, by = 0, sc = 0, rec = 0;
  for (int64_t t = threadIdx.x; t < p.T_q; t += blockDim.x) {
    const int32_t f = p.row_flags[t];
    if (f == kRowBypassed) {
      ++by;
      continue;
    }
    a += static_cast<unsigned long long>(p.surv_count[t]);
    b += static_cast<unsigned long long>(p.refine_len[t]);
    sc += static_cast<unsigned long long>(p.q_offset + t + 1 - p.n_seed);
    if (f != kRowRefined) {
      ++c;
      continue;
    }
    rec += static_cast<unsigned long long>(p.topk);
    auto unit_recs = [&](const int32_t* m) {
      unsigned long long r = static_cast<unsigned long long>(min(max(m[1], 0), p.lay.keep_cap));
      for (int q = 0; q < 4; ++q) r += static_cast<unsigned long long>(min(max(m[2 + q], 0), p.lay.app_cap));
      return r;
    };
    const int u0 = p.seq_ubeg[t], nu = p.seq_ucnt[t];
    for (int u = u0; u < u0 + nu; ++u) rec += unit_recs(p.meta + static_cast<size_t>(u) * kMetaInts);
    if (p.group_len) {
      const int64_t g = t >> 2;
      const int g0 = p.gs_ubeg[g], gn = p.gs_ucnt[g];
      for (int u = g0; u < g0 + gn; ++u) rec += unit_recs(p.meta2 + (static_cast<size_t>(u) * 4 + (t & 3)) * kMetaInts);
    }
  }
  unsigned long long shared = 0;
  if (p.group_len)
    for (int64_t g = threadIdx.x; g < (p.T_q + 3) / 4; g += blockDim.x) {
      const unsigned long long n = static_cast<unsigned long long>(p.group_len[g]);
      shared += n;
      b += 4 * n;
    }
  atomicAdd(&p.out[0], a);
  atomicAdd(&p.out[1], b);
  atomicAdd(&p.out[2], c);
  atomicAdd(&p.out[3], by);
  atomicAdd(&p.out[4], sc);
  atomicAdd(&p.out[5], rec);
  atomicAdd(&p.out[6], shared);
}

cudaError_t launch_seed_prep(const SeedPrepParams& p, cudaStream_t st) {
  const int threads = 256;
  const int64_t n = static_cast<int64_t>(p.n_seed) * 16;
  seed_prep_kernel<<<static_cast<unsigned>((n + threads - 1) / threads), threads, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_keynorm(const uint16_t* k, int64_t T_k, float* knorm, cudaStream_t st) {
  const int threads = 256;
  const int64_t n = T_k * 16;
  keynorm_kernel<<<static_cast<unsigned>((n + threads - 1) / threads), threads, 0, st>>>(k, T_k, knorm);
  return cudaGetLastError();
}

cudaError_t launch_plan(int H, const PlanParams& p, cudaStream_t st) {
  if (H == 64) plan_kernel<64><<<static_cast<unsigned>(p.T_q), 128, 0, st>>>(p);
  else if (H == 32) plan_kernel<32><<<static_cast<unsigned>(p.T_q), 128, 0, st>>>(p);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_share(const ShareParams& p, cudaStream_t st) {
  const int64_t groups = (p.T_q + 3) / 4;
  if (groups > 0) share_kernel<<<static_cast<unsigned>(groups), 256, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_compact(const CompactParams& p, cudaStream_t st) {
  compact_kernel<<<static_cast<unsigned>(p.T_q), 256, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_decide(const DecideParams& p, cudaStream_t st) {
  decide_kernel<<<1, 256, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_stats(const StatsParams& p, cudaStream_t st) {
  stats_kernel<<<1, 256, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace dsa
