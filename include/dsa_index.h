/*
 * dsa_index.h - C ABI of the B200 lightning-indexer library (libdsa_index.so).
 *
 * The library computes, for query rows t and keys s, the DeepSeek Sparse
 * Attention lightning-indexer score
 *
 *     I(t,s) = sum_{j<H} w(t,j) * ReLU(q(t,j) . k(s))
 *
 * ("DeepSeek DSA FLOPs", Lightning Indexer, eq. index score: H index heads of
 * width d share one key vector per position) and returns, per query row, the
 * exact Top-k keys among the causally visible ones.  A query at absolute
 * position p sees keys 0..p ("DeepSeek DSA FLOPs", causal token-pair count,
 * N_dense = T(T+1)/2) and keeps m = min(k, p+1) of them (N_sel).
 *
 * Conventions shared by every entry point
 *  - Pointers marked "device" are CUDA device pointers on the current device;
 *    the caller owns all of them.  Inputs are read-only; outputs are fully
 *    overwritten.  The library allocates no memory: scratch comes from the
 *    caller's workspace, sized by the matching *_workspace_bytes() call.
 *  - Layouts are row-major and contiguous.  q/k hold bf16 values as raw
 *    16-bit patterns; w is fp32.  q, k and the workspace must be 16-byte
 *    aligned (TMA), w/out_* 4-byte aligned.
 *  - Outputs per row: out_idx[row][0..topk) int32 key indices and
 *    out_score[row][0..topk) fp32 scores, sorted by score descending, ties by
 *    smaller key index; entries past m are idx = -1, score = -inf.
 *  - Scores are fp32: dot products accumulate in fp32 on the tensor cores
 *    from the exact bf16 inputs.  The head sum runs as eight fp32 chains,
 *    chain c = j mod 8 holding a_c = fmaf(w_j, max(dot_j, 0), a_c) over its
 *    heads in ascending j from a_c = +0, combined as
 *    ((a0 + a1) + (a2 + a3)) + ((a4 + a5) + (a6 + a7)).  Every entry point
 *    (dense, decode, pruned) uses this one order, so their scores agree bit
 *    for bit.
 *  - Supported: d == 128, H in {32, 64}, 1 <= topk <= 2048, key counts
 *    below 2^31.  Inputs must be finite: a pair that scores NaN is never
 *    selected, and a row with any non-finite pair (NaN or +-inf) has
 *    unspecified contents; non-finite inputs never fault or hang.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *    legacy default stream) unless stated otherwise, and returns a status:
 */
#ifndef DSA_INDEX_H
#define DSA_INDEX_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DSA_API __attribute__((visibility("default")))
#else
#define DSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define DSA_OK 0
#define DSA_EINVAL (-1)       /* null pointer, negative/inconsistent sizes, misalignment */
#define DSA_EUNSUPPORTED (-2) /* d != 128, H not in {32, 64}, topk outside [1, 2048] */
#define DSA_EWORKSPACE (-3)   /* ws_bytes below the *_workspace_bytes() requirement */
#define DSA_ESEED (-4)        /* (pruned) bad seed list: see dsa_index_prefill_pruned */
#define DSA_ECUDA (-5)        /* a CUDA runtime call failed: see dsa_last_error_string() */
#define DSA_EDEVICE (-6)      /* a device-side check failed (reported by synchronous calls) */

/* Counters of the pruned (DoSA) path; all are sums over the call's rows. */
typedef struct dsa_stats {
  int64_t screened_pairs; /* non-seed visible (row, key) pairs given an upper bound */
  int64_t survivor_pairs; /* screened pairs whose bound reached the threshold */
  int64_t refined_pairs;  /* survivor pairs scored exactly with all heads */
  int64_t records;        /* records written for the final selection (seed + refined) */
  int64_t recovered_rows; /* screened rows recomputed by the dense path (survivor overflow, bad seeds) */
  int64_t bypassed_rows;  /* rows the probe sent to the dense path without screening */
  int64_t shared_keys;    /* keys of the groups' shared refine streams (each scored for 4 rows) */
} dsa_stats;

/* Text of the last error seen by this library in the calling thread. */
DSA_API const char* dsa_last_error_string(void);

/*
 * Chunked causal prefill ("DeepSeek DSA FLOPs", Full-prefix index scoring and
 * Prefill / training): query row t (0 <= t < T_q) sits at absolute position
 * q_offset + t and scores keys 0..q_offset+t of k.
 *   q          device, [T_q][H][d] bf16
 *   w          device, [T_q][H] fp32 head weights, used as given
 *   k          device, [T_k][d] bf16 keys; requires 0 <= q_offset,
 *              q_offset + T_q <= T_k
 *   out_idx    device, [T_q][topk] int32
 *   out_score  device, [T_q][topk] fp32
 *   workspace  device, ws_bytes bytes.  dsa_index_prefill_workspace_bytes()
 *              gives what one launch over all rows needs, capped at 4 GiB;
 *              with less (at least one query group's worth, else
 *              DSA_EWORKSPACE) the call runs consecutive launches over row
 *              blocks that fit, with the same result bit for bit (rows are
 *              independent).
 * T_q == 0 is a no-op.
 */
DSA_API size_t dsa_index_prefill_workspace_bytes(int64_t T_q, int64_t T_k, int H, int d, int topk);
DSA_API int dsa_index_prefill(const uint16_t* q, const float* w, const uint16_t* k, int64_t q_offset,
                      int64_t T_q, int64_t T_k, int H, int d, int topk, int32_t* out_idx,
                      float* out_score, void* workspace, size_t ws_bytes, void* stream);

/*
 * The chunked causal prefill on FP8 inputs ("DeepSeek DSA FLOPs", Lightning
 * Indexer: the indexer runs in FP8).  q and k are OCP FP8 E4M3 codes with one
 * fp32 scale per stored row, so the vectors scored are
 *     q(t,j) = q_scale[t][j] * e4m3(q[t][j]),   k(s) = k_scale[s] * e4m3(k[s]),
 * and I(t,s) = sum_j w(t,j) * ReLU(q(t,j) . k(s)) as above.  Scales must be
 * positive (or zero) and finite: they are applied as positive factors,
 *     I(t,s) = k_scale[s] * sum_j (w(t,j) * q_scale[t][j]) * ReLU(e4m3 dot),
 * the E4M3 dot products accumulating in fp32 on the tensor cores
 * (tcgen05 kind::f8f6f4, products exact) and the head sum in the fp32 order
 * stated above with halved weights w * q_scale / 2; a negative or non-finite
 * key scale sets status bit 3.
 *   q          device, [T_q][H][d] E4M3 codes (uint8), 16-byte aligned
 *   q_scale    device, [T_q][H] fp32
 *   w          device, [T_q][H] fp32
 *   k          device, [T_k][d] E4M3 codes (uint8), 16-byte aligned
 *   k_scale    device, [T_k] fp32
 * Other arguments, outputs and the workspace (dsa_index_prefill_workspace_bytes)
 * as for dsa_index_prefill; the same row-block rule applies.
 */
DSA_API int dsa_index_prefill_fp8(const uint8_t* q, const float* q_scale, const float* w, const uint8_t* k,
                                  const float* k_scale, int64_t q_offset, int64_t T_q, int64_t T_k, int H,
                                  int d, int topk, int32_t* out_idx, float* out_score, void* workspace,
                                  size_t ws_bytes, void* stream);

/*
 * The same chunked causal prefill from HOST buffers: q, w and k are host
 * arrays with the layouts above, out_idx / out_score host arrays
 * [T_q][topk].  The call copies the keys to the device once and streams the
 * query rows through in up to 16 row blocks (rows are independent, "DeepSeek
 * DSA FLOPs", index score): while one block is scored on `stream`, the next
 * block's inputs and the previous block's outputs cross PCIe on two library
 * streams, so the copies in both directions overlap the kernels.  Results
 * equal dsa_index_prefill's bit for bit.  The call is asynchronous: the host
 * outputs are complete once `stream` has been synchronised.  Host buffers
 * should be page-locked (cudaHostAlloc / pinned) for the copies to overlap;
 * pageable buffers work but serialise.  The workspace (device, 256-byte
 * aligned, dsa_index_prefill_host_workspace_bytes()) holds the prefill
 * workspace at offset 0 (dsa_index_device_status reads it there), the keys
 * and two slots of row-block buffers.  Calls are serialised by a library
 * mutex; the library's two copy streams per device live until the process
 * exits.  The pages have no counterpart: this is the boundary's host-buffer
 * form of dsa_index_prefill.
 */
DSA_API size_t dsa_index_prefill_host_workspace_bytes(int64_t T_q, int64_t T_k, int H, int d, int topk);
DSA_API int dsa_index_prefill_host(const uint16_t* q, const float* w, const uint16_t* k, int64_t q_offset,
                                   int64_t T_q, int64_t T_k, int H, int d, int topk, int32_t* out_idx,
                                   float* out_score, void* workspace, size_t ws_bytes, void* stream);

/*
 * Batched decode ("DeepSeek DSA FLOPs", Decode): sequence b has one new query
 * q[b] (H rows) and its own key cache k_cache[b] of capacity t_cap, of which
 * the first seq_len[b] keys are visible (the new token's key included).
 *   q          device, [B][H][d] bf16
 *   w          device, [B][H] fp32
 *   k_cache    device, [B][t_cap][d] bf16
 *   seq_len    device, [B] int32, 0 <= seq_len[b] <= t_cap (a length outside
 *              that range is treated as 0 and sets the device status word)
 *   out_idx    device, [B][topk] int32 key positions within the sequence
 *   out_score  device, [B][topk] fp32
 * Requires 1 <= B <= 65536 and B * t_cap < 2^31.
 */
DSA_API size_t dsa_index_decode_workspace_bytes(int B, int64_t t_cap, int H, int d, int topk);
DSA_API int dsa_index_decode(const uint16_t* q, const float* w, const uint16_t* k_cache,
                     const int32_t* seq_len, int B, int64_t t_cap, int H, int d, int topk,
                     int32_t* out_idx, float* out_score, void* workspace, size_t ws_bytes,
                     void* stream);

/*
 * Batched decode over a PAGED key cache (the DoSA notes' port reads keys
 * through pages, annotation LJZ23SXM; the layout here is this library's):
 * sequence b's key i (0 <= i < seq_len[b]) is row
 *     block_table[b][i / page_size] * page_size + i % page_size
 * of the page pool.  Same computation and outputs as dsa_index_decode (key
 * indices are positions within the sequence).
 *   k_pages      device, [n_pages][page_size][d] bf16, 16-byte aligned
 *   page_size    a positive multiple of 64
 *   block_table  device, [B][max_blocks] int32 page ids; entries covering
 *                keys below seq_len[b] must lie in [0, n_pages) (an entry
 *                outside is read as page 0 and sets status bit 1)
 *   seq_len      device, [B] int32, 0 <= seq_len[b] <= max_blocks * page_size
 *                (a length outside is treated as 0 and sets status bit 1)
 * The workspace is dsa_index_decode_workspace_bytes(B, max_blocks * page_size,
 * ...).  Requires n_pages * page_size < 2^31.
 */
DSA_API int dsa_index_decode_paged(const uint16_t* q, const float* w, const uint16_t* k_pages, int64_t n_pages,
                                   int page_size, const int32_t* block_table, int max_blocks,
                                   const int32_t* seq_len, int B, int H, int d, int topk, int32_t* out_idx,
                                   float* out_score, void* workspace, size_t ws_bytes, void* stream);

/*
 * Chunked causal prefill with DoSA certified pruning ("DoSA: Dots Sparse
 * Attention", steps 1-3; 163.com write-up, section 03).  Same inputs and the
 * same outputs, bit for bit, as dsa_index_prefill: the seed set only changes
 * how much work is skipped, never the result.
 *   1. The n_seed seed keys are scored with all heads; per row, tau is the
 *      topk-th largest seed score (a lower bound on the row's true topk-th).
 *   2. Every other visible key gets an upper bound U from 14 retained heads,
 *      a residual bound for the omitted positive-weight heads and a folded
 *      lower bound on the omitted negative-weight heads' penalty; keys with
 *      U < tau are pruned (strictly; a key whose bound is uncertain is kept).
 *   3. Survivors are scored exactly with all heads; records at or above the
 *      row's topk-th seed record enter the final exact Top-k with the seeds'.
 *      Within each group of four consecutive rows whose survivor lists all
 *      fit, a key kept by at least two rows and visible to all four is
 *      gathered once and scored for the four ("DoSA" notes, annotation
 *      WFZZA9CL, step 3: the shared stream); the others are scored per row.
 * The first 64 rows of a chunk longer than 128 rows are a probe: they
 * always take steps 1-3, and from their survivor counts the device estimates
 * whether pruning pays for this chunk (screen, seed and refine costs against
 * a dense pass).  If it does not, the remaining rows skip steps 1-3 and go
 * straight to the dense kernel, so the call costs little more than
 * dsa_index_prefill on inputs the bound cannot filter.  Rows whose survivors
 * exceed a list of max(T_k / 16, 4 topk) keys are also recomputed densely.
 * The decision is taken on the device: the call never waits for the host.
 *   seed_idx   device, [n_seed] int32: distinct keys with 0 <= seed < q_offset
 *              (visible to every row); topk <= n_seed <= q_offset, else
 *              DSA_ESEED before any launch.  Out-of-range or repeated seeds
 *              found on the device make every row fall back to the exact
 *              dense computation (reported as DSA_ESEED when stats is given).
 *   stats      host, may be NULL: when given, the call synchronises `stream`
 *              and fills the counters, over the rows that were screened
 *              (screened_pairs: their visible non-seed pairs; survivor_pairs:
 *              pairs with U >= tau; refined_pairs: survivors scored exactly;
 *              records: seed Top-k + refined candidates read by the final
 *              selection of the rows it finished; recovered_rows: screened
 *              rows recomputed densely after a survivor overflow or a bad
 *              seed list), bypassed_rows (rows sent to the dense kernel
 *              without screening) and shared_keys (keys of the shared
 *              streams; refined_pairs counts four scores for each).
 * Requires T_q <= 65536.  The workspace is sized by
 * dsa_index_prefill_pruned_workspace_bytes().
 */
DSA_API size_t dsa_index_prefill_pruned_workspace_bytes(int64_t T_q, int64_t T_k, int H, int d, int topk,
                                                        int n_seed);
DSA_API int dsa_index_prefill_pruned(const uint16_t* q, const float* w, const uint16_t* k, int64_t q_offset,
                                     int64_t T_q, int64_t T_k, int H, int d, int topk,
                                     const int32_t* seed_idx, int n_seed, int32_t* out_idx,
                                     float* out_score, dsa_stats* stats, void* workspace,
                                     size_t ws_bytes, void* stream);

/*
 * Diagnostics of the most recent dsa_index_prefill_pruned call that used
 * `workspace` with the same sizes ("DoSA", step 2: the screen's survivor
 * decisions).  Copies, on `stream`:
 *   mask       device, [T_q][ceil(T_k / 32)] uint32: bit s % 32 of word s / 32
 *              of row t is 1 when the screen kept key s (U >= tau), 0 when it
 *              pruned it.  Defined for screened rows, keys 0..q_offset+t;
 *              seed keys read 0 (they are scored exactly, never screened).
 *   tau        device, [T_q] fp32: the row's topk-th seed score.
 *   row_state  device, [T_q] int32: 0 screened and refined, 1 screened and
 *              recomputed densely (survivor overflow), 2 not screened
 *              (the probe's bypass), 3 bad seed list.
 * For tests of the bound's safety: a pruned key must score below tau.
 */
DSA_API int dsa_index_prefill_pruned_survivors(const void* workspace, int64_t T_q, int64_t T_k,
                                               int64_t q_offset, int H, int d, int topk, int n_seed,
                                               uint32_t* mask, float* tau, int32_t* row_state,
                                               void* stream);

/*
 * Chunked prefill, dense and DoSA-pruned, over a paged key cache (the pages'
 * port keeps keys in pages and reads them through page tables: "DoSA" notes,
 * annotation LJZ23SXM).  Same computation, outputs and status bits as
 * dsa_index_prefill / dsa_index_prefill_pruned on the keys
 *     k(s) = k_pages[block_table[s / page_size]][s % page_size],  0 <= s < T_k.
 * One bandwidth-bound pass first gathers those T_k keys into the workspace
 * (2 x 256 bytes per key moved, against the O(T_q x T_k) scoring that
 * follows); the scoring kernels then stream them as contiguous TMA tiles.
 *   k_pages      device, [n_pages][page_size][128] bf16, 16-byte aligned;
 *                page_size >= 1, n_pages * page_size < 2^31
 *   block_table  device, [ceil(T_k / page_size)] int32 page ids of this
 *                sequence; an id outside [0, n_pages) reads zeros and sets
 *                status bit 1 (the pruned call with stats returns
 *                DSA_EDEVICE for it)
 *   workspace    256-byte aligned, of the *_paged_workspace_bytes() size:
 *                the contiguous call's workspace (its status word at byte 0,
 *                read with dsa_index_device_status; for the pruned call also
 *                dsa_index_prefill_pruned_survivors), then the gathered keys.
 *                The dense call accepts less and runs row blocks.
 */
DSA_API size_t dsa_index_prefill_paged_workspace_bytes(int64_t T_q, int64_t T_k, int H, int d, int topk);
DSA_API int dsa_index_prefill_paged(const uint16_t* q, const float* w, const uint16_t* k_pages, int64_t n_pages,
                                    int page_size, const int32_t* block_table, int64_t q_offset, int64_t T_q,
                                    int64_t T_k, int H, int d, int topk, int32_t* out_idx, float* out_score,
                                    void* workspace, size_t ws_bytes, void* stream);
DSA_API size_t dsa_index_prefill_pruned_paged_workspace_bytes(int64_t T_q, int64_t T_k, int H, int d, int topk,
                                                              int n_seed);
DSA_API int dsa_index_prefill_pruned_paged(const uint16_t* q, const float* w, const uint16_t* k_pages,
                                           int64_t n_pages, int page_size, const int32_t* block_table,
                                           int64_t q_offset, int64_t T_q, int64_t T_k, int H, int d, int topk,
                                           const int32_t* seed_idx, int n_seed, int32_t* out_idx, float* out_score,
                                           dsa_stats* stats, void* workspace, size_t ws_bytes, void* stream);

/*
 * Seed keys from historical selection frequency (163.com write-up, section
 * 03: a chunk's seed set may be the keys that earlier rows selected most).
 * Counts how often each key 0..n_keys-1 occurs in the Top-k lists of earlier
 * rows and writes the n_seed keys with the largest counts, ties going to the
 * smaller key (keys never selected fill up from key 0), in ascending key
 * order.  With n_keys = the next chunk's q_offset and n_seed >= topk the
 * output is a valid seed_idx for dsa_index_prefill_pruned.  Exact integer
 * work; no host synchronisation.
 *   prev_idx   device, [n_rows][topk] int32: earlier rows' out_idx; entries
 *              outside [0, n_keys) (the -1 padding) are not counted.  May be
 *              NULL when n_rows == 0 (then the seeds are keys 0..n_seed-1).
 *   n_keys     1 <= n_keys < 2^31;  1 <= n_seed <= n_keys;
 *              n_rows * topk < 2^32, else DSA_EINVAL.
 *   seeds_out  device, [n_seed] int32, ascending.
 *   workspace  device, 256-byte aligned, of
 *              dsa_index_seeds_from_history_workspace_bytes(n_keys) bytes
 *              (about 4 n_keys + 256 KB); after the call it holds the
 *              per-key counts as uint32 at byte offset 256 + 262144.
 */
DSA_API size_t dsa_index_seeds_from_history_workspace_bytes(int64_t n_keys);
DSA_API int dsa_index_seeds_from_history(const int32_t* prev_idx, int64_t n_rows, int topk, int64_t n_keys,
                                         int n_seed, int32_t* seeds_out, void* workspace, size_t ws_bytes,
                                         void* stream);

/*
 * Batched decode that allocates nothing (no counterpart in the paper; a
 * library convenience).  Same computation, arguments and outputs as
 * dsa_index_decode, without the workspace: for callers that cannot hand the
 * library device memory of their own, such as hosts whose device memory is
 * entirely carved up by an allocator they do not control, or code that must
 * not call cudaMalloc on a latency-critical path because it can synchronise
 * the device.
 *  - Scratch is a fixed array in the library's device image, sized for at
 *    most 64 sequences at topk <= 2048 (36,827,136 bytes, about 37 MB).
 *    Every GPU on which the library is loaded holds that memory until the
 *    process exits.  B > 64 returns DSA_EINVAL with an explanatory message;
 *    nothing is launched.
 *  - The call itself allocates no device memory: no cudaMalloc/cudaFree, no
 *    allocating library routine.  Each call looks up the scratch's device
 *    address on the current device (cudaGetSymbolAddress; the first lookup
 *    on a device loads the library's kernels there), so make the first call
 *    on each device before any stream capture.
 *  - All calls share the one scratch array, which keeps the last call's
 *    contents; each call initialises what it reads.  Calls whose executions
 *    overlap on the GPU (different streams, or host threads racing on the
 *    same device) race on the scratch and give undefined results: serialise
 *    them.
 *  - Device-side checks (a length outside [0, t_cap], a bounded wait that
 *    gave up, a non-finite pair) set the status word at the start of the
 *    static scratch, not in a caller workspace: read it with
 *    dsa_index_decode_noalloc_status().
 */
DSA_API int dsa_index_decode_noalloc(const uint16_t* q, const float* w, const uint16_t* k_cache,
                                     const int32_t* seq_len, int B, int64_t t_cap, int H, int d,
                                     int topk, int32_t* out_idx, float* out_score, void* stream);

/*
 * Device status word of the most recent dsa_index_decode_noalloc call on the
 * current device (the word at the start of the library's static scratch;
 * bits as for dsa_index_device_status below).  Synchronises `stream`; it
 * allocates nothing.  No counterpart in the paper: the status reader of the
 * allocation-free decode.
 */
DSA_API int dsa_index_decode_noalloc_status(uint32_t* status, void* stream);

/*
 * Device status word of the most recent call that used `workspace`: 0 when
 * every device-side check passed.  Synchronises `stream`.
 * Bit 0: a bounded wait inside a kernel gave up (the kernel unwound).
 * Bit 1: a capacity or length check failed.  Bit 2: the seed list was invalid.
 * Bit 3: a causally visible (query, key) pair scored inf or NaN, i.e. q, k or
 * w holds a non-finite value; NaN pairs are never selected and the rows with
 * a non-finite pair are unspecified.
 */
DSA_API int dsa_index_device_status(const void* workspace, uint32_t* status, void* stream);

/*
 * Failure injection for tests of the bounded device waits (no counterpart on
 * the pages).  Arms a one-shot fault for the calling host thread: the next
 * fused scoring launch of any entry point issues no loads, so its MMA warp
 * waits for data that never arrives; that wait gives up after limit_ns
 * (1 ms .. 2 s), the kernel unwinds (in-flight copies and tensor-core work
 * drained, tensor memory released), sets bit 0 of the device status word and
 * returns.  The call's outputs are then unspecified; later calls are
 * unaffected.  Nothing faults or hangs: every wait in the library is bounded.
 */
DSA_API int dsa_test_inject_wait_timeout(int64_t limit_ns);

/*
 * Per-kernel timing of the calling thread's entry-point calls (for
 * benchmarks; no counterpart on the pages).  With profiling enabled, each
 * entry point records a CUDA event on its stream before its first kernel and
 * after each kernel launch.  dsa_profile_read() waits for the last call's
 * final event and returns the device time of each of its kernels in
 * milliseconds (ms[i], names[i] may be NULL; at most max_n entries written;
 * *n_out = number of kernels of that call).
 */
DSA_API int dsa_profile_enable(int on);
DSA_API int dsa_profile_read(float* ms, const char** names, int max_n, int* n_out);

#ifdef __cplusplus
}
#endif

#endif /* DSA_INDEX_H */
