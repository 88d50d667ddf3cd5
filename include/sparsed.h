/*
 * sparsed.h -- C ABI of the block-sparse bidirectional attention library
 * (libsparsed.so, built for NVIDIA B200 / sm_100a only).
 *
 * What it computes. Multi-head bidirectional (non-causal) attention of a
 * diffusion language model across its denoising steps, in three parts:
 *   - dense attention for the early steps
 *     (SparseD: Sparse Attention for Diffusion Language Models, abstract:
 *      full attention in the early steps, which are critical for generation);
 *   - a head-specific block-sparse pattern selected from one full-attention
 *     pass and reused at later steps
 *     (SparseD abstract: patterns differ across heads and stay similar across
 *      steps, so they are pre-computed once and reused; Step-dLLM: Adaptive
 *      Step-aware Sparse Attention for Efficient Diffusion LLM Inference,
 *      abstract: the block-sparse mask is refreshed at anchor steps and the
 *      sparsity budget may be head-adaptive);
 *   - block-sparse attention that visits only the kept key blocks
 *     (Step-dLLM abstract: block-sparse attention kernel; PulseCol abstract:
 *      block-sparse computation in the later iterations).
 * Beside these: a column-sparse pattern (PulseCol abstract), a head-sharded
 * entropy selection and step driver, and block-wise generation over a prefix
 * cache with active-token reuse (LoSA: Locality Aware Sparse Attention for
 * Block-Wise Diffusion Language Models); each section below says which.
 *
 * Conventions shared by every entry point
 *   Layout    Q, K, V, O are [H, L, d] bf16 (raw 16-bit patterns), row-major,
 *             d contiguous, one contiguous buffer each. LSE is [H, L] fp32,
 *             natural log of the softmax denominator of each query row.
 *             Query block i covers rows [i*bq, min((i+1)*bq, L)); key block j
 *             covers keys [j*bk, min((j+1)*bk, L)); nqb = ceil(L/bq),
 *             nkb = ceil(L/bk). L need not be a multiple of the block sizes.
 *   Pattern   kv_idx is [H, nqb, kv_stride] int32, kv_count is [H, nqb] int32:
 *             the kept key blocks of (head h, query block i) are
 *             kv_idx[(h*nqb+i)*kv_stride + 0 .. kv_count[h*nqb+i]-1], strictly
 *             ascending, each in [0, nkb). Slots past kv_count are never read
 *             or written.
 *   Sizes     d in {64, 128}; bq, bk in {64, 128}; H >= 0, L >= 0 (H*L == 0 is
 *             a no-op returning SPARSED_OK); H*L*d < 2^31.
 *   Memory    Every array argument is DEVICE memory owned by the caller; the
 *             library never allocates, frees or retains user memory. Q, K, V,
 *             O must be 16-byte aligned. Scratch space comes only from a
 *             caller-supplied workspace of the size sparsed_workspace_bytes
 *             reports.
 *   Streams   `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *             stream). Calls are asynchronous on that stream unless stated.
 *   Errors    Every call returns an int status: SPARSED_OK (0) or a negative
 *             SPARSED_ERR_* code; arguments are validated on the host before
 *             anything is launched, and a failed validation launches nothing.
 *             Faults found on the device (a bad pattern entry, a bounded wait
 *             that expired) are recorded in a device error word and returned
 *             by the next sparsed_check(). No kernel traps or hangs on bad
 *             input: every device-side wait is bounded.
 */
#ifndef SPARSED_H
#define SPARSED_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SPARSED_VERSION 100 /* major*10000 + minor*100 + patch: 0.1.0 */

enum {
  SPARSED_OK = 0,
  SPARSED_ERR_INVALID_ARG = -1,    /* null pointer, negative size, misaligned buffer */
  SPARSED_ERR_UNSUPPORTED = -2,    /* d, bq or bk outside the supported set, size limits */
  SPARSED_ERR_WORKSPACE = -3,      /* workspace missing or smaller than required */
  SPARSED_ERR_BAD_PATTERN = -4,    /* a pattern entry out of range / not ascending (device) */
  SPARSED_ERR_CUDA = -5,           /* a CUDA runtime call failed; see sparsed_last_cuda_error */
  SPARSED_ERR_DEVICE_TIMEOUT = -6, /* a bounded device-side wait expired */
  SPARSED_ERR_NO_DEVICE = -7,      /* no sm_100 device is current */
  SPARSED_ERR_EXCHANGE = -8        /* the caller's exchange callback returned nonzero */
};

enum { SPARSED_BUDGET_UNIFORM = 0, SPARSED_BUDGET_ENTROPY = 1 };
enum { SPARSED_STEP_DENSE = 0, SPARSED_STEP_SELECT = 1, SPARSED_STEP_SPARSE = 2 };

/* Library version (the SPARSED_VERSION it was compiled with). Never fails. */
int sparsed_version(void);

/* Static message for a status code; never NULL. */
const char* sparsed_strerror(int status);

/* The cudaError_t of the last runtime failure mapped to SPARSED_ERR_CUDA
 * (0 if none). Host-side, thread-shared, not reset by successful calls. */
int sparsed_last_cuda_error(void);

/* Synchronises `stream`, then returns and clears the device error word: the
 * first device-side fault recorded since the previous check
 * (SPARSED_ERR_BAD_PATTERN or SPARSED_ERR_DEVICE_TIMEOUT), else SPARSED_OK. */
int sparsed_check(void* stream);

/* Self-test of the bounded device waits (not part of the method): launches one
 * thread that waits on an mbarrier nothing arrives on; after timeout_ns
 * (1 .. 1e9) it gives up, records SPARSED_ERR_DEVICE_TIMEOUT and returns, so
 * the next sparsed_check reports that status and clears it. No copy or MMA is
 * in flight, and the context stays usable. */
int sparsed_selftest_wait_timeout(unsigned long long timeout_ns, void* stream);

/* Host-only. Kept key blocks per query block under the uniform budget:
 * k = clamp(ceil(keep_ratio * nkb - 1e-6), 1, nkb), nkb = ceil(L/bk)
 * (Step-dLLM abstract: a uniform budget across heads; "90% sparsity" keeps
 * 0.10). keep_ratio must be in (0, 1]. */
int sparsed_uniform_keep(int L, int bk, float keep_ratio, int* k_out);

/* Host-only. Step kinds of a T-step denoising run, written to kinds[0..T-1]
 * (host memory) as SPARSED_STEP_*: with n_dense = clamp(ceil(w*T - 1e-6), 1, T),
 * steps t < n_dense-1 are DENSE, t = n_dense-1 is SELECT, and a later step is
 * SELECT when refresh_every > 0 and (t - (n_dense-1)) % refresh_every == 0,
 * else SPARSE; if n_dense == T every step is DENSE (SparseD abstract: full
 * attention early, pattern computed once and reused; Step-dLLM abstract:
 * refresh at anchor steps). warmup_frac in [0, 1], refresh_every >= 0. */
int sparsed_schedule(int T, float warmup_frac, int refresh_every, int8_t* kinds);

/* Host-only. Bytes of workspace sparsed_select_pattern and sparsed_run_steps
 * need for these sizes (0 < result; layout is private to the library). */
int sparsed_workspace_bytes(int H, int L, int bq, int bk, size_t* bytes);

/* Dense bidirectional attention (SparseD abstract: attention over all
 * query-key pairs; Step-dLLM abstract: the full map is recomputed at every
 * step since bidirectional attention has no KV cache).
 *   O[h,r,:]  = sum_c softmax_c(scale * <Q[h,r,:], K[h,c,:]>) * V[h,c,:]   (bf16)
 *   LSE[h,r]  = ln sum_c exp(scale * <Q[h,r,:], K[h,c,:]>)                  (fp32)
 * Products and the softmax run in fp32 on bf16 tensor cores; P is rounded to
 * bf16 before the PV product. bq/bk are the tile sizes (results agree across
 * tile sizes to rounding; sparsed_block_sparse_attn with every block kept and
 * the same bk is bitwise equal). */
int sparsed_dense_attn(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                       int H, int L, int d, float scale, int bq, int bk,
                       uint16_t* O, float* LSE, void* stream);

/* One full-attention pass that also selects the block-sparse pattern
 * (SparseD abstract: head-specific patterns from full attention; Step-dLLM
 * abstract: block-sparse mask, uniform or head-adaptive budget).
 *   1. O, LSE as sparsed_dense_attn (this pass's output is the step's output).
 *   2. block mass M[h,i,j] = sum over rows r of query block i and keys c of key
 *      block j of exp(scale*<q_r,k_c> - LSE[h,r]), from fp32 scores
 *      (written to block_mass [H,nqb,nkb] fp32 when non-NULL).
 *   3. per-head budget k_h: UNIFORM: sparsed_uniform_keep for every head.
 *      ENTROPY: E_h = mean over i of the entropy of M[h,i,:]/sum_j M[h,i,j];
 *      B = clamp(ceil(keep_ratio*H*nkb - 1e-6), H, H*nkb); each head keeps one
 *      block and the extra B-H is split in proportion to E_h (evenly if the
 *      split heads' entropies sum to 0), capping a head at nkb and re-splitting
 *      its overflow, then rounded by largest remainder (ties to the lower head);
 *      sum_h k_h = B. Written to head_k [H] int32 when non-NULL.
 *   4. per (h, i): the k_h blocks of largest M[h,i,:] (ties to the lower block
 *      index), written ascending to kv_idx, and kv_count[h*nqb+i] = k_h.
 * kv_stride >= k (UNIFORM) or >= nkb (ENTROPY). workspace: device memory of at
 * least sparsed_workspace_bytes(H, L, bq, bk) bytes, 256-byte aligned, owned by
 * the caller; contents on entry are ignored. The full pass takes its pairs of
 * query blocks from counters kept in the workspace (cleared by the call), so
 * one workspace must not serve two calls at the same time. */
int sparsed_select_pattern(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                           int H, int L, int d, float scale, int bq, int bk,
                           float keep_ratio, int budget_mode,
                           uint16_t* O, float* LSE,
                           int32_t* kv_idx, int32_t* kv_count, int kv_stride,
                           float* block_mass, int32_t* head_k,
                           void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes with which sparsed_run_steps fuses the block mass into
 * the full pass of its SELECT steps: sparsed_workspace_bytes plus the
 * per-warp mass partials [H, nqb, nkb, 4] fp32 and one [H, L] fp32 LSE copy,
 * every part 256-byte aligned. */
int sparsed_run_steps_workspace_bytes(int H, int L, int bq, int bk, size_t* bytes);

/* Block-sparse attention over a cached pattern (Step-dLLM abstract: the mask
 * is reused within each interval; SparseD abstract: the precomputed pattern is
 * reused at all later steps). For each row r of query block i of head h, the
 * softmax runs over the keys of blocks kv_idx[h,i,0..kv_count[h,i]-1] only:
 *   O[h,r,:] = sum over kept keys c of softmax(scale*<q_r,k_c>) v_c  (bf16)
 *   LSE[h,r] = ln sum over kept keys of exp(scale*<q_r,k_c>)          (fp32)
 * kv_count 0 gives O = 0 and LSE = -inf for that block's rows. A pattern entry
 * out of range or out of order is clamped (no out-of-bounds access) and
 * reported as SPARSED_ERR_BAD_PATTERN by the next sparsed_check. */
int sparsed_block_sparse_attn(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                              int H, int L, int d, float scale, int bq, int bk,
                              const int32_t* kv_idx, const int32_t* kv_count, int kv_stride,
                              uint16_t* O, float* LSE, void* stream);

/* The denoising loop for one attention layer with fixed inputs: steps
 * t = start_step .. T-1 run the kind sparsed_schedule(T, warmup_frac,
 * refresh_every) gives -- DENSE: sparsed_dense_attn; SELECT:
 * sparsed_select_pattern into kv_idx/kv_count (the pattern cache, caller
 * memory); SPARSE: sparsed_block_sparse_attn with the cached pattern.
 * O and LSE hold the last step's output. have_pattern != 0 means kv_idx/
 * kv_count already hold a pattern (resume after the switch); a SPARSE step
 * with no pattern yet is SPARSED_ERR_INVALID_ARG (checked before launching).
 * step_kind (nullable, HOST [T] int8) receives the kinds of all T steps.
 * step_ms (nullable, HOST [T] fp32) receives each executed step's device time
 * in ms from CUDA events (0 for skipped steps); when given, the call
 * synchronises the stream before returning. workspace: at least
 * sparsed_workspace_bytes(H, L, bq, bk) bytes as in sparsed_select_pattern.
 * With sparsed_run_steps_workspace_bytes(H, L, bq, bk) bytes, a SELECT step
 * that follows an earlier full pass of this call (a DENSE step just before
 * it, or an earlier SELECT) takes the block mass from its own full pass: the
 * attention kernel sums each tile's probabilities with the LSE of that earlier
 * pass, which equals this pass's LSE because the loop's inputs are fixed
 * (Step-dLLM abstract: selection cost matters at every anchor). A SELECT step
 * with no earlier full pass in the call, or a smaller workspace, runs the
 * separate block-mass pass of sparsed_select_pattern. With a workspace of at
 * least sparsed_workspace_bytes, the loop's full passes take their pairs of
 * query blocks from counters kept in it (cleared by one memset per call), so
 * the CTAs in flight stay on neighbouring query blocks and share K/V in L2.
 * The results are the same bits as with the static order of a call without
 * a workspace. The workspace must not be in use by another call at the same
 * time. */
int sparsed_run_steps(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                      int H, int L, int d, float scale, int bq, int bk,
                      float keep_ratio, int budget_mode,
                      int T, float warmup_frac, int refresh_every,
                      int start_step, int have_pattern,
                      int32_t* kv_idx, int32_t* kv_count, int kv_stride,
                      uint16_t* O, float* LSE,
                      int8_t* step_kind, float* step_ms,
                      void* workspace, size_t workspace_bytes, void* stream);

/* Steps start_step .. end_step-1 of the same loop (0 <= start_step <=
 * end_step <= T): the schedule is still that of T steps, so a run can be cut
 * into spans and continued -- e.g. around SELECT steps that the caller runs
 * itself (the head-sharded entropy selection below). Arguments and outputs
 * as sparsed_run_steps; step_ms receives the span's steps (0 elsewhere); a
 * SELECT step inside the span uses the fused block mass only when a full pass
 * of the same span comes before it. */
int sparsed_run_steps_span(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                           int H, int L, int d, float scale, int bq, int bk,
                           float keep_ratio, int budget_mode,
                           int T, float warmup_frac, int refresh_every,
                           int start_step, int end_step, int have_pattern,
                           int32_t* kv_idx, int32_t* kv_count, int kv_stride,
                           uint16_t* O, float* LSE,
                           int8_t* step_kind, float* step_ms,
                           void* workspace, size_t workspace_bytes, void* stream);

/* The exchange of the head-sharded loop, supplied by the caller (an
 * all-gather over the ranks that hold the heads of one layer). It is called on
 * the host at every selecting step with this rank's h_local per-head
 * entropies (host memory, fp64) and must fill all_entropy with the h_total
 * entropies of the layer in head order (host memory), then return 0. Any
 * other return value stops the loop with SPARSED_ERR_EXCHANGE. */
typedef int (*sparsed_exchange_fn)(const double* local_entropy, int h_local, double* all_entropy, int h_total,
                                   void* user);

/* The denoising loop for this rank's heads of a layer whose h_total heads are
 * split over ranks (Step-dLLM abstract: a head-adaptive global budget spans
 * the heads of a layer). This rank holds heads [head_offset, head_offset + H)
 * of Q, K, V ([H, L, d], as sparsed_run_steps).
 *   - budget_mode SPARSED_BUDGET_UNIFORM: every head's budget is its own, so
 *     the loop is sparsed_run_steps on the local heads; exchange is not
 *     called and may be null.
 *   - SPARSED_BUDGET_ENTROPY: the loop is cut at its SELECT steps. Steps
 *     between them run as sparsed_run_steps_span. Each SELECT step runs as
 *     follows:
 *       1. the full pass, the block mass and the mean row entropy of each
 *          local head (sparsed_select_head_entropy);
 *       2. the entropies are copied to the host (a stream synchronisation);
 *       3. exchange(...) gathers all h_total entropies;
 *       4. the allocation of sparsed_entropy_budget over all heads;
 *       5. top-k with this rank's k_h (sparsed_select_with_head_k).
 *     Every rank reaches the same allocation from the same gathered
 *     entropies.
 * kv_idx / kv_count: the pattern cache, [H, nqb, kv_stride] / [H, nqb] int32,
 * kv_stride >= nkb for the entropy budget. step_kind: nullable [T]. The
 * workspace: sparsed_workspace_bytes(H, L, bq, bk) bytes, 256-byte aligned,
 * for the entropy budget. Returns the first failing call's status,
 * SPARSED_ERR_INVALID_ARG for inconsistent head counts or a null exchange with
 * the entropy budget, SPARSED_ERR_EXCHANGE when the callback fails. */
int sparsed_run_steps_sharded(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                              int H, int L, int d, float scale, int bq, int bk,
                              float keep_ratio, int budget_mode, int h_total, int head_offset,
                              int T, float warmup_frac, int refresh_every,
                              int32_t* kv_idx, int32_t* kv_count, int kv_stride,
                              uint16_t* O, float* LSE, int8_t* step_kind,
                              sparsed_exchange_fn exchange, void* user,
                              void* workspace, size_t workspace_bytes, void* stream);

/* ---- Queries that change across the denoising steps.
 *
 * The pages give no per-step activations; attention patterns stay similar
 * across steps (SparseD abstract) and are only locally consistent, shifting at
 * some transitions (Step-dLLM abstract). These entry points give every step t
 * its own queries, a seeded perturbation of Q with the same bits on any
 * machine:
 *   Q_t = bf16(fp32(Q) + fp32(amplitude * u)), elementwise (nearest even),
 *   u   = (fmix32(i ^ key) >> 8) * 2^-23 - 1, in [-1, 1) on a 2^-23 grid,
 *   key = fmix32(fmix32(seed) ^ t),
 * where i is the element's row-major index in [H, L, d] and fmix32 is the
 * MurmurHash3 32-bit finalizer (h ^= h>>16; h *= 0x85ebca6b; h ^= h>>13;
 * h *= 0xc2b2ae35; h ^= h>>16). The product and the sum are rounded once
 * each. */

/* Q_out = Q_t for step t (device pointers, [H, L, d] bf16, 16-byte aligned;
 * Q_out may not overlap Q). Returns SPARSED_ERR_INVALID_ARG for null or
 * misaligned pointers, t < 0 or a non-finite amplitude,
 * SPARSED_ERR_UNSUPPORTED for d not in {64, 128} or H*L*d >= 2^31. Asynchronous
 * on `stream`. */
int sparsed_drift_queries(const uint16_t* Q, int H, int L, int d, unsigned int seed, int t,
                          float amplitude, uint16_t* Q_out, void* stream);

/* sparsed_run_steps_span with per-step queries: before step t the driver
 * writes Q_t (sparsed_drift_queries with drift_seed, drift_amplitude) into
 * Q_step (caller memory, [H, L, d] bf16, 16-byte aligned, not overlapping the
 * other arrays) and runs the step on Q_step, K and V. A SELECT step that uses
 * the fused block mass (the workspace of sparsed_run_steps_workspace_bytes,
 * an earlier full pass in the span) weights each row's probabilities with the
 * LSE of that earlier pass, computed on earlier queries: each row's masses
 * are then scaled by exp(lse_now - lse_then), so the selection equals the
 * separate pass's wherever the relative gap between the k-th and (k+1)-th
 * block mass exceeds 1 - exp(-2 * max |lse_now - lse_then|). Errors as
 * sparsed_run_steps_span, and SPARSED_ERR_INVALID_ARG for a null or misaligned
 * Q_step or a non-finite amplitude. */
int sparsed_run_steps_drift(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                            int H, int L, int d, float scale, int bq, int bk,
                            float keep_ratio, int budget_mode,
                            int T, float warmup_frac, int refresh_every,
                            int start_step, int end_step, int have_pattern,
                            unsigned int drift_seed, float drift_amplitude, uint16_t* Q_step,
                            int32_t* kv_idx, int32_t* kv_count, int kv_stride,
                            uint16_t* O, float* LSE,
                            int8_t* step_kind, float* step_ms,
                            void* workspace, size_t workspace_bytes, void* stream);

/* ---- Head-sharded selection with the entropy budget (the heads of one
 * layer split over several GPUs: only the per-head entropies cross ranks, one
 * all-gather of H doubles per selection; Step-dLLM abstract: head-adaptive
 * global budget). The three calls below, with the entropies of all heads
 * gathered in head order between the first and the second, give every head
 * the same k_h, kv_idx and kv_count as sparsed_select_pattern with
 * SPARSED_BUDGET_ENTROPY on the whole layer. */

/* Steps 1-2 of sparsed_select_pattern for this rank's H heads, then the mean
 * row entropy E_h of every head (as in the ENTROPY budget) into head_entropy
 * (DEVICE [H] fp64). The block mass stays in the workspace (at least
 * sparsed_workspace_bytes(H, L, bq, bk) bytes) for sparsed_select_with_head_k.
 * The full pass takes its pairs from counters in the workspace, as in
 * sparsed_select_pattern. */
int sparsed_select_head_entropy(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                                int H, int L, int d, float scale, int bq, int bk,
                                uint16_t* O, float* LSE, double* head_entropy,
                                void* workspace, size_t workspace_bytes, void* stream);

/* The ENTROPY budget allocation of sparsed_select_pattern on the HOST: from
 * the entropies of all H heads of the layer (HOST [H] fp64) to k_h (HOST [H]
 * int32). Runs without a GPU; identical to the device allocation. */
int sparsed_entropy_budget(const double* head_entropy, int H, int nkb, float keep_ratio, int32_t* head_k);

/* Step 4 of sparsed_select_pattern for this rank's H heads with given k_h
 * (DEVICE [H] int32), over the block mass a preceding
 * sparsed_select_head_entropy left in the same workspace (stream-ordered).
 * kv_stride >= nkb. */
int sparsed_select_with_head_k(int H, int L, int bq, int bk, const int32_t* head_k,
                               int32_t* kv_idx, int32_t* kv_count, int kv_stride,
                               void* workspace, size_t workspace_bytes, void* stream);

/* ---- Column-sparse path (PulseCol: Periodically Refreshed Column-Sparse
 * Attention for Accelerating Diffusion Language Models, abstract: the sparse
 * pattern is a set of key columns of the attention map instead of blocks,
 * identified at an early denoising step, reused, and refreshed at a few
 * intermediate steps). A column pattern keeps, per head h, kc key positions
 * cols[h*col_stride + 0..kc-1] (strictly ascending) shared by every query of
 * that head; kc = clamp(ceil(keep_ratio*L - 1e-6), 1, L). The block size
 * arguments bq, bk only choose the tiles of the attention kernel. */

/* kc for a sequence of L keys (as sparsed_uniform_keep with nkb = L). */
int sparsed_column_keep(int L, float keep_ratio, int* kc);

/* Workspace bytes of the column path for H heads, L tokens, head dim d and kc
 * kept columns: the column-mass array [H, L] fp32, the gathered K and V
 * columns [H, kc, d] bf16 each and the full passes' pair counters, every part
 * 256-byte aligned. */
int sparsed_column_workspace_bytes(int H, int L, int d, int kc, size_t* bytes);

/* One full-attention pass that also selects the column pattern:
 *   1. O, LSE as sparsed_dense_attn (this pass's output is the step's output).
 *   2. column mass A[h,c] = sum over every row r of exp(scale*<q_r,k_c> - LSE[h,r])
 *      from fp32 scores (written to col_mass [H, L] fp32 when non-NULL).
 *   3. per head: the kc columns of largest A (ties to the lower column),
 *      written ascending to cols [H, col_stride], col_stride >= kc.
 * workspace: device memory of at least sparsed_column_workspace_bytes(H, L, d,
 * kc) bytes, 256-byte aligned, owned by the caller; contents on entry are
 * ignored. The full pass takes its pairs from counters in the workspace, as in
 * sparsed_select_pattern. */
int sparsed_select_columns(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                           int H, int L, int d, float scale, int bq, int bk, float keep_ratio,
                           uint16_t* O, float* LSE, int32_t* cols, int col_stride,
                           float* col_mass, void* workspace, size_t workspace_bytes, void* stream);

/* Attention of every query over its head's kc kept columns:
 *   O[h,r,:] = sum over c in cols[h] of softmax(scale*<q_r,k_c>) v_c  (bf16)
 *   LSE[h,r] = ln sum over c in cols[h] of exp(scale*<q_r,k_c>)       (fp32)
 * The kept K and V rows are first gathered into the workspace (as in
 * sparsed_select_columns). An entry outside [0, L) or not above its predecessor
 * reads row 0 and is reported as SPARSED_ERR_BAD_PATTERN by the next
 * sparsed_check. */
int sparsed_column_sparse_attn(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                               int H, int L, int d, float scale, int bq, int bk,
                               const int32_t* cols, int kc, int col_stride,
                               uint16_t* O, float* LSE, void* workspace, size_t workspace_bytes,
                               void* stream);

/* The denoising loop with the column pattern: the step kinds of
 * sparsed_schedule(T, warmup_frac, refresh_every); DENSE: sparsed_dense_attn;
 * SELECT: sparsed_select_columns into cols (the pattern cache, caller memory);
 * SPARSE: sparsed_column_sparse_attn with the cached columns. Arguments and
 * outputs otherwise as sparsed_run_steps; the full passes take their pairs of
 * query blocks from counters in the workspace as there. */
int sparsed_run_steps_columns(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                              int H, int L, int d, float scale, int bq, int bk, float keep_ratio,
                              int T, float warmup_frac, int refresh_every,
                              int start_step, int have_pattern, int32_t* cols, int col_stride,
                              uint16_t* O, float* LSE, int8_t* step_kind, float* step_ms,
                              void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of the library's built-in scratch array used by
 * sparsed_select_pattern_noalloc (16 MiB, held by every GPU that loads the
 * library until the process exits). */
#define SPARSED_NOALLOC_SCRATCH_BYTES (16u << 20)

/* sparsed_select_pattern without a workspace, for callers that may not
 * allocate device memory -- for example code running inside a host framework
 * that owns the whole device-memory budget through its own pool, or
 * latency-critical loops where cudaMalloc/cudaFree would implicitly
 * synchronise the device. The pages describe no such entry point; it has no
 * counterpart there. Arguments, outputs and results are those of
 * sparsed_select_pattern (the caller still passes every input and output);
 * the scratch comes from a fixed array inside the library instead of a
 * workspace, and no cudaMalloc, cudaFree or other allocating routine is called.
 *   - Returns SPARSED_ERR_WORKSPACE, launching nothing, when these sizes need
 *     more than SPARSED_NOALLOC_SCRATCH_BYTES of scratch
 *     (sparsed_workspace_bytes(H, L, bq, bk) > SPARSED_NOALLOC_SCRATCH_BYTES;
 *     e.g. H=32, L=32768, bq=bk=128 fits, L=65536 does not).
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current and caches it under the
 *     device's CUDA context (a context created after cudaDeviceReset gets a
 *     fresh lookup on its first call); make that first call before any stream
 *     capture.
 *   - Every call on a device shares the one array, which keeps the previous
 *     call's contents; each call overwrites all scratch it reads, so nothing
 *     needs clearing. Calls that overlap on the GPU race on the array: issue
 *     them on one stream (or otherwise order them). */
int sparsed_select_pattern_noalloc(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                                   int H, int L, int d, float scale, int bq, int bk,
                                   float keep_ratio, int budget_mode,
                                   uint16_t* O, float* LSE,
                                   int32_t* kv_idx, int32_t* kv_count, int kv_stride,
                                   float* block_mass, int32_t* head_k, void* stream);

/* ---- Block-wise generation with active-token reuse
 *
 * LoSA: Locality Aware Sparse Attention for Block-Wise Diffusion Language
 * Models (section 1: a block's queries load the union of the prefix positions
 * they select; section 2: between consecutive steps only a few tokens' queries
 * change much; section 3: active tokens -- large query change, measured by
 * MSE -- get sparse prefix attention over the union of their selections,
 * stable tokens reuse their cached prefix output, and prefix and in-block
 * ("suffix") parts are merged by online softmax; the first step of a block is
 * dense and fills the cache).
 *
 * Setting. A block of B tokens is denoised over T steps on top of a prefix of
 * P cached tokens.
 *   Q, K, V          [H, B, d] bf16: the block's queries, keys, values at this step
 *   K_prefix, V_prefix  [H, P, d] bf16: the prefix cache (fixed during the block)
 *   Prefix key block j covers prefix positions [j*bk, min((j+1)*bk, P));
 *   nkb = ceil(P / bk).
 * State carried across the block's steps (caller memory, written by
 * sparsed_losa_init, read and updated by sparsed_losa_step):
 *   o_cache   [H, B, d] bf16: every token's prefix attention output
 *   lse_cache [H, B] fp32: its natural-log LSE over the prefix keys it attended
 *   sel       [H, B, n_sel] int32: each token's n_sel prefix blocks (ascending)
 * Every step's output O [H, B, d] bf16 and LSE [H, B] fp32 is attention over
 * the token's prefix part (from the cache) together with all B block keys.
 *
 * Selector. The pages name the selector only (QUEST, a separate method); the
 * method works with any. This library uses the SparseD selector at token
 * granularity: in the block's first (dense) step each token's prefix blocks
 * are scored by their post-softmax probability mass
 *   M[h,b,j] = sum over c in block j of exp(scale*<q_b,k_c> - lse_cache[h,b])
 * and the n_sel largest (ties to the lower block) are kept for the block.
 * An active token attends to every key of its head's union.
 *
 * Work is split: a head's union is cut into `splits` chunks processed as
 * separate work items of the block-sparse kernel and merged by LSE, so that a
 * step keeps the SMs busy although a block holds few query rows.
 *
 * Sizes: 1 <= B <= 1024; P >= 1; nkb <= 32768; d in {64, 128}; bq, bk in
 * {64, 128}; n_sel >= 1 (values above nkb act as nkb); splits >= 1 (values
 * above min(32, ceil(nkb/4)) act as that bound); H*P*d < 2^31.
 * Pointers: device memory, Q/K/V/prefix/o_cache/O 16-byte aligned, the rest
 * 4-byte aligned; the workspace 256-byte aligned. Returns as every entry
 * point; the union-building kernel reports a selection entry outside [0, nkb)
 * as SPARSED_ERR_BAD_PATTERN (skipping it).
 *
 * Streams: the block's own attention of a step runs on a second stream that
 * the library creates once per device (non-blocking), forked from `stream`
 * with an event before it and joined back into `stream` with an event before
 * the merge; to the caller the step is ordered on `stream` alone, and a graph
 * capture of `stream` records both branches. Make the first call on a device
 * outside a graph capture (it creates that stream and its two events). */

/* Splits for a step of these sizes on a GPU with sm_count SMs: as many as
 * keep one split's H*ceil(B/bq) work items per SM at most
 * (floor(sm_count / (H*ceil(B/bq))), at least 1, at most min(32, ceil(nkb/4))). */
int sparsed_losa_splits(int H, int B, int bq, int P, int bk, int sm_count, int* splits);

/* Workspace bytes of sparsed_losa_init / _step / _block for these sizes:
 * the active flags and union (B + H*nkb + H int32), the split lists, the
 * replicated queries and partial outputs ([H, splits*ceil(B/bq)*bq, d] bf16
 * each, plus their LSE), the per-token block mass [H, B, nkb] fp32 and its
 * counts, every part 256-byte aligned. */
int sparsed_losa_workspace_bytes(int H, int B, int P, int d, int bq, int bk, int splits,
                                 size_t* bytes);

/* First step of a block: dense prefix attention of every token (the cache),
 * each token's n_sel blocks (sel, row stride n_sel), the suffix attention and
 * the merged output O, LSE. token_mass (nullable, [H, B, nkb] fp32) receives
 * the per-token block mass. */
int sparsed_losa_init(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                      const uint16_t* K_prefix, const uint16_t* V_prefix,
                      int H, int B, int P, int d, float scale, int bq, int bk, int n_sel, int splits,
                      uint16_t* o_cache, float* lse_cache, int32_t* sel,
                      uint16_t* O, float* LSE, float* token_mass,
                      void* workspace, size_t workspace_bytes, void* stream);

/* A later step of the block, in the page's order:
 *   1. mse_b = mean over heads and dimensions of (Q - Q_prev)^2 (fp64), and
 *      active[b] = (mse_b > tau) as int32 0/1 (active: nullable [B]);
 *   2. per head, the ascending union of the active tokens' sel blocks
 *      (union_idx: nullable [H, nkb], first union_count[h] entries;
 *      union_count: nullable [H]);
 *   3. prefix attention of the active tokens over every key of the union:
 *      their o_cache / lse_cache entries are replaced; stable tokens keep
 *      theirs;
 *   4. suffix attention over the block, merged with the prefix part into O, LSE.
 * Q_prev is the block's queries at the previous step ([H, B, d] bf16); tau is
 * finite and >= 0. */
int sparsed_losa_step(const uint16_t* Q, const uint16_t* K, const uint16_t* V, const uint16_t* Q_prev,
                      const uint16_t* K_prefix, const uint16_t* V_prefix,
                      int H, int B, int P, int d, float scale, int bq, int bk, int n_sel, float tau,
                      int splits, uint16_t* o_cache, float* lse_cache, const int32_t* sel,
                      uint16_t* O, float* LSE, int32_t* active, int32_t* union_idx,
                      int32_t* union_count, void* workspace, size_t workspace_bytes, void* stream);

/* All T >= 1 steps of a block: sparsed_losa_init on step 0, then
 * sparsed_losa_step with the previous step's queries. Qs, Ks, Vs, Os are
 * [T, H, B, d], LSEs [T, H, B]. actives (nullable, [T, B]) and union_counts
 * (nullable, [T, H]) record each step's active flags and union sizes; step 0
 * records every token active and nkb blocks per head. o_cache, lse_cache and
 * sel hold the state after the last step. */
int sparsed_losa_block(const uint16_t* Qs, const uint16_t* Ks, const uint16_t* Vs,
                       const uint16_t* K_prefix, const uint16_t* V_prefix, int T,
                       int H, int B, int P, int d, float scale, int bq, int bk, int n_sel, float tau,
                       int splits, uint16_t* o_cache, float* lse_cache, int32_t* sel,
                       uint16_t* Os, float* LSEs, int32_t* actives, int32_t* union_counts,
                       void* workspace, size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SPARSED_H */
