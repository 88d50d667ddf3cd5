// Block-wise generation with active-token reuse (LoSA: Locality Aware Sparse
// Attention for Block-Wise Diffusion Language Models, sections 1-3).
//
// A block of B tokens is denoised over several steps on top of a prefix of P
// cached tokens. Per head, the state carried across the block's steps is the
// prefix attention output and LSE of every block token (the cache) and each
// token's selected prefix key blocks. The first step of a block runs dense
// prefix attention for every token and selects each token's blocks from that
// pass; every later step
//
//   query_mse_kernel      mse_b = mean over (h, c) of (Q_t - Q_{t-1})^2 in fp64;
//                         active_b = mse_b > tau
//   losa_lists_kernel     per head: the union of the active tokens' blocks
//                         (ascending), cut into S chunks ("splits"), one
//                         block list per (split, query tile), and the active
//                         tokens' queries copied once per split
//   attn_fwd_kernel       sparse mode over those lists: each split's partial
//                         prefix attention (O, LSE) of every active token
//   attn_fwd_kernel       dense over the block itself: the suffix part
//   losa_merge_kernel     active tokens: the splits' partials merged by LSE
//                         into a new cache entry; stable tokens: the cache
//                         as it is; then prefix and suffix merged by LSE
//
// and the first step also runs
//
//   token_block_mass_kernel  M[h,b,j] = sum over prefix keys c of block j of
//                            exp(scale*<q_b,k_c> - LSE_b), S = Q K^T on tcgen05
//   topk_kernel              (select_kernels.cuh) each token's n_sel blocks
//
// Splitting a head's list over several work items is what keeps the SMs busy:
// a block holds one or a few query tiles per head, so without splits a step
// would have H to a few H work items for 148 SMs.
#pragma once

#include "ptx_sm100.cuh"

namespace sparsed {

constexpr int kLosaMaxB = 1024;        // block tokens (the active list lives in shared memory)
constexpr int kLosaMaxWords = 1024;    // union bitmask words: at most 32768 prefix blocks
constexpr int kLosaMinChunk = 4;       // fewest blocks a non-empty split holds
constexpr int kLosaMaxSplits = 32;     // splits of a head's list (one per lane in the merge)

// PER (2 or 4) consecutive bf16 from an address aligned to 2*PER bytes, widened to fp32.
template <int PER>
__device__ __forceinline__ void load_bf16(const uint16_t* p, float (&f)[PER]) {
  static_assert(PER == 2 || PER == 4, "2 or 4 elements");
  if constexpr (PER == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    f[0] = __uint_as_float(u.x << 16);
    f[1] = __uint_as_float(u.x & 0xffff0000u);
    f[2] = __uint_as_float(u.y << 16);
    f[3] = __uint_as_float(u.y & 0xffff0000u);
  } else {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
    f[0] = __uint_as_float(u << 16);
    f[1] = __uint_as_float(u & 0xffff0000u);
  }
}

// p[0..n) = value (the step-0 rows of the per-step records).
__global__ void __launch_bounds__(256) fill_i32_kernel(int32_t* __restrict__ p, int n, int32_t value) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) p[i] = value;
}

// ---------------------------------------------------------------- locality score

// One CTA of 256 threads per block token b: the squared query change summed
// over every head and dimension in fp64 (each thread takes 16-byte pieces of
// the token's rows, 8 elements each, then a fixed shuffle tree and the 8
// warps in order), divided by H*d. d is a multiple of 8.
__global__ void __launch_bounds__(256)
    query_mse_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ q_prev, int H, int B, int d,
                     double tau, int32_t* __restrict__ active) {
  __shared__ double s_part[8];
  ptx::grid_dep_launch();  // the union-and-lists kernel may launch; it waits for this grid to complete
  const int b = blockIdx.x;
  const int row_u4 = d / 8;
  const int n_u4 = H * row_u4;
  const uint4* q4 = reinterpret_cast<const uint4*>(q);
  const uint4* p4 = reinterpret_cast<const uint4*>(q_prev);
  double acc = 0.0;
#pragma unroll 4
  for (int e = threadIdx.x; e < n_u4; e += blockDim.x) {
    const int h = e / row_u4;
    const long idx = (static_cast<long>(h) * B + b) * row_u4 + (e - h * row_u4);
    const uint4 x = q4[idx], y = p4[idx];
    const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const double d0 = static_cast<double>(__uint_as_float(xs[i] << 16)) - __uint_as_float(ys[i] << 16);
      const double d1 = static_cast<double>(__uint_as_float(xs[i] & 0xffff0000u)) -
                        __uint_as_float(ys[i] & 0xffff0000u);
      acc += d0 * d0 + d1 * d1;
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if ((threadIdx.x & 31) == 0) s_part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < 8; ++w) t += s_part[w];
    active[b] = (t / static_cast<double>(H * d)) > tau ? 1 : 0;
  }
}

// ---------------------------------------------------------------- union and split lists

struct LosaListArgs {
  int H, B, d;
  int nkb;         // prefix key blocks
  int n_sel;       // blocks selected per token (already clamped to nkb)
  int sel_stride;  // row stride of sel
  int bq;          // query tile rows of the prefix pass
  int tiles;       // query tiles per split: ceil(B / bq)
  int R;           // rows per split: tiles * bq
  int S;           // splits
  int kv_stride;   // row stride of kv_idx
  const int32_t* active;  // [B]; nullptr: first step (every token, every block)
  const int32_t* sel;     // [H, B, sel_stride]
  const uint16_t* q;      // [H, B, d]
  int32_t* pos;           // [B]: index in the active list, or -1
  int32_t* union_idx;     // [H, nkb]: ascending union, first union_count[h] entries
  int32_t* union_count;   // [H]
  int32_t* kv_idx;        // [H, S * tiles, kv_stride]
  int32_t* kv_count;      // [H, S * tiles]
  uint16_t* q_rep;        // [H, S * R, d]
};

// One CTA of 256 threads per head h.
//   1. the active tokens in ascending order (warp ballots), and pos[] (head 0)
//   2. the union as a bitmask over prefix blocks (shared-memory atomics)
//   3. the ascending union list: each thread expands a contiguous run of words
//      at the offset of an exclusive scan of the runs' bit counts, and writes
//      each entry straight into the split lists as well
//   4. split s holds union entries [s*chunk, (s+1)*chunk), chunk =
//      max(kLosaMinChunk, ceil(u / S)); work item (s, t) of query tile t gets
//      that chunk when the tile holds an active token, else nothing (counts)
//   5. row s*R + a of q_rep is the a-th active token's query (zero past the
//      active count) for every split and tile that have work
__global__ void __launch_bounds__(256) losa_lists_kernel(const LosaListArgs a) {
  __shared__ int s_act[kLosaMaxB];
  __shared__ uint32_t s_bits[kLosaMaxWords];
  __shared__ int s_scan[8];
  __shared__ int s_warp[8];
  __shared__ int s_u;
  // a programmatic dependent of the locality score: active[] is complete
  // past this point (a no-op after an ordinary launch)
  ptx::grid_dep_wait();
  ptx::grid_dep_launch();
  const int h = blockIdx.x;
  const int tid = threadIdx.x;
  const int lane = tid & 31, wid = tid >> 5;
  const unsigned lt_mask = (1u << lane) - 1u;

  // 1. active list
  int na = 0;
  for (int c0 = 0; c0 < a.B; c0 += 256) {
    const int b = c0 + tid;
    const bool act = b < a.B && (a.active == nullptr || a.active[b] != 0);
    const unsigned ball = __ballot_sync(0xffffffffu, act);
    if (lane == 0) s_warp[wid] = __popc(ball);
    __syncthreads();
    int before = 0, total = 0;
    for (int w = 0; w < 8; ++w) {
      if (w < wid) before += s_warp[w];
      total += s_warp[w];
    }
    const int p = na + before + __popc(ball & lt_mask);
    if (act) s_act[p] = b;
    if (h == 0 && b < a.B) a.pos[b] = act ? p : -1;
    na += total;
    __syncthreads();
  }

  // 2. union bitmask
  const int words = (a.nkb + 31) >> 5;
  for (int w = tid; w < words; w += 256) {
    uint32_t m = 0u;
    if (a.active == nullptr) {
      const int left = a.nkb - (w << 5);
      m = left >= 32 ? 0xffffffffu : ((1u << left) - 1u);
    }
    s_bits[w] = m;
  }
  __syncthreads();
  if (a.active != nullptr) {
    for (int e = tid; e < na * a.n_sel; e += 256) {
      const int ai = e / a.n_sel;
      const int s = e - ai * a.n_sel;
      const int j = a.sel[(static_cast<long>(h) * a.B + s_act[ai]) * a.sel_stride + s];
      if (j < 0 || j >= a.nkb) {
        ptx::record_error(kErrBadPattern);
        continue;
      }
      atomicOr(&s_bits[j >> 5], 1u << (j & 31));
    }
  }
  __syncthreads();

  // 3. ascending union list
  const int wpt = (words + 255) / 256;
  const int w0 = tid * wpt < words ? tid * wpt : words;
  const int w1 = w0 + wpt < words ? w0 + wpt : words;
  int cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(s_bits[w]);
  // exclusive scan of the 256 counts: within each warp by shuffles, then
  // over the 8 warp totals
  int incl = cnt;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) s_scan[wid] = incl;
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int w = 0; w < 8; ++w) {
      const int c = s_scan[w];
      s_scan[w] = run;
      run += c;
    }
    s_u = run;
  }
  __syncthreads();
  int32_t* ulist = a.union_idx + static_cast<long>(h) * a.nkb;
  const int u = s_u;
  const int items = a.S * a.tiles;
  int chunk = (u + a.S - 1) / a.S;
  if (chunk < kLosaMinChunk) chunk = kLosaMinChunk;
  const long item0 = static_cast<long>(h) * items;
  int outp = s_scan[wid] + incl - cnt;
  for (int w = w0; w < w1; ++w) {
    uint32_t m = s_bits[w];
    while (m) {
      const int j = (w << 5) + (__ffs(m) - 1);
      ulist[outp] = j;
      // entry outp of the union is entry jj of split s, for every tile with work
      const int s = outp / chunk, jj = outp - s * chunk;
      for (int t = 0; t < a.tiles && t * a.bq < na; ++t) a.kv_idx[(item0 + s * a.tiles + t) * a.kv_stride + jj] = j;
      ++outp;
      m &= m - 1u;
    }
  }
  if (tid == 0) a.union_count[h] = u;

  // 4. split list lengths
  auto split_len = [&](int s) -> int {
    if (na == 0) return 0;
    const int left = u - s * chunk;
    return left <= 0 ? 0 : (left < chunk ? left : chunk);
  };
  for (int it = tid; it < items; it += 256) {
    const int s = it / a.tiles;
    const int t = it - s * a.tiles;
    a.kv_count[item0 + it] = (t * a.bq < na) ? split_len(s) : 0;
  }

  // 5. replicated queries of the tiles that have work: each 16-byte piece of
  // an active token's query is read once and stored into every split
  const int row_u4 = a.d / 8;
  const uint4* qsrc = reinterpret_cast<const uint4*>(a.q) + static_cast<long>(h) * a.B * row_u4;
  uint4* qdst = reinterpret_cast<uint4*>(a.q_rep) + static_cast<long>(h) * a.S * a.R * row_u4;
  const int rows = ((na + a.bq - 1) / a.bq) * a.bq;  // rows of the tiles with work (<= R)
  const int total = rows * row_u4;
  for (int e0 = tid; e0 < total; e0 += 4 * 256) {
    uint4 val[4];  // four pieces' loads in flight before their stores
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int e = e0 + k * 256;
      const int r = e / row_u4;
      val[k] = (e < total && r < na) ? qsrc[static_cast<long>(s_act[r]) * row_u4 + (e - r * row_u4)]
                                     : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int e = e0 + k * 256;
      if (e >= total) break;
      const int r = e / row_u4;
      for (int s = 0; s < a.S; ++s)
        if (split_len(s) > 0) qdst[(static_cast<long>(s) * a.R + r) * row_u4 + (e - r * row_u4)] = val[k];
    }
  }
}

// ---------------------------------------------------------------- merge and cache

struct LosaMergeArgs {
  int H, B, d, S, R, tiles, bq;  // d == D of the kernel
  const int32_t* pos;       // [B]; nullptr: every token active, pos[b] = b
  const int32_t* kv_count;  // [H, S * tiles] of the prefix pass
  const uint16_t* o_rep;    // [H, S * R, d]
  const float* lse_rep;     // [H, S * R]
  uint16_t* o_cache;        // [H, B, d]  prefix output of every token
  float* lse_cache;         // [H, B]
  uint16_t* o;              // [H, B, d]  in: suffix output; out: the step's output
  float* lse;               // [H, B]
};

// One warp per (h, b). An active token's prefix part is the LSE-weighted sum
// of its splits' partial outputs (lane s holds split s's LSE and weight; an
// empty split weighs 0), written back to the cache in bf16; a stable token's
// is the cache entry. The output merges that prefix part with the suffix part
// the same way (fp32 arithmetic, fixed reduction order). At most 32 splits.
template <int D>
__global__ void __launch_bounds__(256) losa_merge_kernel(const LosaMergeArgs a) {
  constexpr int PER = D / 32;  // contiguous elements per lane
  ptx::grid_dep_wait();        // a programmatic dependent of the prefix pass
  const int lane = threadIdx.x & 31;
  const long row = static_cast<long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= static_cast<long>(a.H) * a.B) return;
  const int h = static_cast<int>(row / a.B);
  const int b = static_cast<int>(row - static_cast<long>(h) * a.B);
  const int c0 = lane * PER;
  const float kNegInf = -__int_as_float(0x7f800000);
  const long crow = (static_cast<long>(h) * a.B + b) * a.d;
  const long lrow = static_cast<long>(h) * a.B + b;
  const int ap = a.pos ? a.pos[b] : b;
  // the suffix part, read before any branch
  float osuf[PER];
  load_bf16<PER>(a.o + crow + c0, osuf);
  const float ls = a.lse[lrow];
  float op[PER];
  float lp;
  if (ap >= 0) {
    const int t = ap / a.bq;
    const long rep0 = static_cast<long>(h) * a.S * a.R + ap;
    // both loads at once: every split's rows are written by the prefix pass
    // (LSE -inf for a split without work), so the LSE read never waits on the count
    const int kc = lane < a.S ? a.kv_count[static_cast<long>(h) * a.S * a.tiles + lane * a.tiles + t] : 0;
    const float lr = lane < a.S ? a.lse_rep[rep0 + static_cast<long>(lane) * a.R] : kNegInf;
    const float l_s = kc > 0 ? lr : kNegInf;
    float m = l_s;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    const float w = (m == kNegInf || l_s == kNegInf) ? 0.f : expf(l_s - m);
    float z = w;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
#pragma unroll
    for (int e = 0; e < PER; ++e) op[e] = 0.f;
    // every split's rows are written by the prefix pass (zeros for an empty one)
#pragma unroll 4
    for (int s = 0; s < a.S; ++s) {
      const float ws = __shfl_sync(0xffffffffu, w, s);
      float part[PER];
      load_bf16<PER>(a.o_rep + (rep0 + static_cast<long>(s) * a.R) * a.d + c0, part);
#pragma unroll
      for (int e = 0; e < PER; ++e) op[e] += ws * part[e];
    }
    if (z > 0.f) {
      const float inv = 1.f / z;
#pragma unroll
      for (int e = 0; e < PER; ++e) op[e] *= inv;
      lp = m + logf(z);
    } else {
      lp = kNegInf;
    }
#pragma unroll
    for (int e = 0; e < PER; e += 2)
      *reinterpret_cast<uint32_t*>(a.o_cache + crow + c0 + e) = ptx::pack_bf16x2(op[e], op[e + 1]);
    if (lane == 0) a.lse_cache[lrow] = lp;
  } else {
    load_bf16<PER>(a.o_cache + crow + c0, op);
    lp = a.lse_cache[lrow];
  }
  const float m2 = fmaxf(lp, ls);
  const float wp = lp == kNegInf ? 0.f : expf(lp - m2);
  const float ws2 = ls == kNegInf ? 0.f : expf(ls - m2);
  const float z2 = wp + ws2;
  const float inv2 = z2 > 0.f ? 1.f / z2 : 0.f;
  float out[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) out[e] = (wp * op[e] + ws2 * osuf[e]) * inv2;
  __syncwarp();  // every lane has read its suffix inputs before any lane overwrites them
#pragma unroll
  for (int e = 0; e < PER; e += 2)
    *reinterpret_cast<uint32_t*>(a.o + crow + c0 + e) = ptx::pack_bf16x2(out[e], out[e + 1]);
  if (lane == 0) a.lse[lrow] = z2 > 0.f ? m2 + logf(z2) : kNegInf;
}

// ---------------------------------------------------------------- per-token top-k

// One warp per row of mass[rows, n]: the k <= 32 largest entries (ties to the
// lower index), written in ascending index order to idx[row * stride ..]. In
// the order "mass descending, index ascending", round r takes the best entry
// after the pick of round r-1: each lane scans its strided share of the row,
// a shuffle reduction gives the warp's best, and lane r keeps it. Each lane's
// rank among the k picks by index is its output slot. The kept set is the one
// of topk_kernel (rank(j) < k in the same order).
__global__ void __launch_bounds__(256)
    topk_small_kernel(const float* __restrict__ mass, int rows, int n, int k, int32_t* __restrict__ idx,
                      int stride) {
  const int lane = threadIdx.x & 31;
  const long row = static_cast<long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const float* m = mass + row * n;
  const float kInf = __int_as_float(0x7f800000);
  float pv = kInf;  // the previous pick; every finite entry comes after (+inf, -1)
  int pj = -1;
  int mine = 0;     // lane r: the pick of round r
  for (int r = 0; r < k; ++r) {
    float bv = -kInf;
    int bj = 0x7fffffff;
    for (int j = lane; j < n; j += 32) {
      const float v = m[j];
      const bool after = v < pv || (v == pv && j > pj);
      if (after && (v > bv || (v == bv && j < bj))) {
        bv = v;
        bj = j;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oj = __shfl_xor_sync(0xffffffffu, bj, off);
      if (ov > bv || (ov == bv && oj < bj)) {
        bv = ov;
        bj = oj;
      }
    }
    pv = bv;
    pj = bj;
    if (lane == r) mine = bj;
  }
  int rank = 0;
  for (int s = 0; s < k; ++s) rank += __shfl_sync(0xffffffffu, mine, s) < mine;
  if (lane < k) idx[row * stride + rank] = mine;
}

// ---------------------------------------------------------------- per-token block mass

struct TokMassArgs {
  int H, B, P, nkb;
  int tiles_per_cta;  // 128-key tiles of the prefix per CTA
  float scale_log2;
  const float* lse;   // [H, B] natural-log prefix LSE of every block token
  float* mass;        // [H, B, nkb]
  uint64_t timeout_ns;
};

template <int D>
struct TokMassCfg {
  static constexpr int M = 128;  // block tokens per CTA (TMEM lanes)
  static constexpr int N = 128;  // prefix keys per tile
  static constexpr int STAGES = 3;
  static constexpr int DCH = D / 64;
  static constexpr int CHUNK = 128 * 128;  // bytes of one 64-column chunk of a 128-row tile
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = TILE_BYTES;
  static constexpr int OFF_BAR = OFF_K + STAGES * TILE_BYTES;
  static constexpr int B_QFULL = 0;
  static constexpr int B_KFULL = 1;
  static constexpr int B_KEMPTY = B_KFULL + STAGES;
  static constexpr int B_SFULL = B_KEMPTY + STAGES;  // [2]
  static constexpr int B_SFREE = B_SFULL + 2;        // [2] one arrival per reducer thread
  static constexpr int B_DRAIN = B_SFREE + 2;
  static constexpr int NUM_BARS = B_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;  // tmem slot, abort flag
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int TM_S0 = 0;
  static constexpr int TM_S1 = N;
  static constexpr int TM_ALLOC = 256;
  static constexpr uint32_t IDESC = ptx::idesc_bf16_f32(M, N, 0, 0);
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// Grid (ceil(ceil(P/128) / tiles_per_cta), H, ceil(B/128)), 128 + 128 * 128/BK
// threads. CTA (x, h, z) holds the query tile z (block tokens z*128 ..) and
// streams the prefix key tiles x*tiles_per_cta .. through a 3-deep ring: warp 0
// issues the copies, warp 1 owns TMEM and issues S = Q K^T per tile
// (double-buffered in TMEM), warps 4 .. reduce in 128/BK groups of four, group
// g taking key block g of every tile (two warps per SM sub-partition at
// BK = 64). Thread r of a group is token z*128 + r (TMEM lane r, warp % 4 the
// lane quarter): per tile it sums 2^(s*scale*log2e - LSE*log2e) over its key
// block's keys below P in a fixed order (packed fp32x2 accumulators) and
// writes M[h, b, j].
template <int D, int BK>
__global__ void __launch_bounds__(384, 1)
    token_block_mass_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                            const TokMassArgs a) {
  using C = TokMassCfg<D>;
  static_assert(BK == 64 || BK == 128, "key block of 64 or 128");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sb = ptx::smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int qt = blockIdx.z;
  const int ntiles = (a.P + C::N - 1) / C::N;
  const int t0 = blockIdx.x * a.tiles_per_cta;
  const int t1 = t0 + a.tiles_per_cta < ntiles ? t0 + a.tiles_per_cta : ntiles;
  const int n = t1 > t0 ? t1 - t0 : 0;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  auto bar = [&](int idx) -> uint32_t { return sb + C::OFF_BAR + 8 * idx; };

  if (threadIdx.x == 0) {
    ptx::mbar_init(bar(C::B_QFULL), 1);
    for (int s = 0; s < C::STAGES; ++s) {
      ptx::mbar_init(bar(C::B_KFULL + s), 1);
      ptx::mbar_init(bar(C::B_KEMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(bar(C::B_SFULL + b), 1);
      ptx::mbar_init(bar(C::B_SFREE + b), 128 * (C::N / BK));
    }
    ptx::mbar_init(bar(C::B_DRAIN), 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), C::TM_ALLOC);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (n > 0 && warp == 0 && lane == 0) {
    // ================================================================ producer
    ptx::mbar_arrive_expect_tx(bar(C::B_QFULL), C::TILE_BYTES);
#pragma unroll
    for (int c = 0; c < C::DCH; ++c)
      ptx::tma_load_3d(sb + C::OFF_Q + c * C::CHUNK, &tm_q, bar(C::B_QFULL), c * 64, qt * C::M, h);
    int issued = 0;
    for (int i = 0; i < n; ++i) {
      const int s = i % C::STAGES;
      if (i >= C::STAGES &&
          !ptx::mbar_wait(bar(C::B_KEMPTY + s), (i / C::STAGES - 1) & 1, abort_flag, a.timeout_ns, kErrTimeout))
        break;
      ptx::mbar_arrive_expect_tx(bar(C::B_KFULL + s), C::TILE_BYTES);
#pragma unroll
      for (int c = 0; c < C::DCH; ++c)
        ptx::tma_load_3d(sb + C::OFF_K + s * C::TILE_BYTES + c * C::CHUNK, &tm_k, bar(C::B_KFULL + s), c * 64,
                         (t0 + i) * C::N, h);
      ++issued;
    }
    if (*abort_flag) {
      // let the copies in flight land before the CTA's shared memory goes away
      const uint64_t short_ns = a.timeout_ns / 4;
      volatile int dummy = 0;
      ptx::mbar_wait(bar(C::B_QFULL), 0, &dummy, short_ns, 0);
      for (int t = (issued > C::STAGES ? issued - C::STAGES : 0); t < issued; ++t)
        ptx::mbar_wait(bar(C::B_KFULL + t % C::STAGES), (t / C::STAGES) & 1, &dummy, short_ns, 0);
    }
  } else if (n > 0 && warp == 1 && lane == 0) {
    // ================================================================ MMA issuer
    constexpr uint32_t HI = ptx::sdesc_sw128_hi(1024);
    const uint32_t qlo = ptx::sdesc_sw128_lo(sb + C::OFF_Q, 16);
    const uint32_t klo = ptx::sdesc_sw128_lo(sb + C::OFF_K, 16);
    bool ok = ptx::mbar_wait(bar(C::B_QFULL), 0, abort_flag, a.timeout_ns, kErrTimeout);
    for (int i = 0; ok && i < n; ++i) {
      const int s = i % C::STAGES;
      const int b = i & 1;
      if (!ptx::mbar_wait(bar(C::B_KFULL + s), (i / C::STAGES) & 1, abort_flag, a.timeout_ns, kErrTimeout) ||
          (i >= 2 &&
           !ptx::mbar_wait(bar(C::B_SFREE + b), ((i - 2) >> 1) & 1, abort_flag, a.timeout_ns, kErrTimeout))) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const uint32_t k0 = klo + static_cast<uint32_t>(s * C::TILE_BYTES >> 4);
      const uint32_t s_tmem = tmem + (b ? C::TM_S1 : C::TM_S0);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * (C::CHUNK >> 4) + (kk & 3) * 2;
        ptx::umma_ss_lohi(s_tmem, qlo + off, k0 + off, HI, C::IDESC, kk > 0 ? 1u : 0u);
      }
      ptx::umma_commit(bar(C::B_SFULL + b));
      ptx::umma_commit(bar(C::B_KEMPTY + s));
    }
    if (!ok) {
      ptx::umma_commit(bar(C::B_DRAIN));
      volatile int dummy = 0;
      ptx::mbar_wait(bar(C::B_DRAIN), 0, &dummy, a.timeout_ns / 4, 0);
    }
  } else if (n > 0 && warp >= 4) {
    // ================================================================ reducers
    constexpr int G = C::N / BK;     // key blocks per tile, one reducer group each
    const int g = (warp - 4) >> 2;   // my key block within the tile
    const int wq = warp & 3;
    const int r = wq * 32 + lane;    // token of this CTA == TMEM lane
    const int tok = qt * C::M + r;
    const bool valid = tok < a.B;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const uint64_t sl2 = ptx::f32x2(a.scale_log2, a.scale_log2);
    const float nl = valid ? a.lse[static_cast<long>(h) * a.B + tok] * -1.44269504088896340736f : 0.f;
    const uint64_t nl2 = ptx::f32x2(nl, nl);
    float* out = a.mass + (static_cast<long>(h) * a.B + (valid ? tok : 0)) * a.nkb;
    for (int i = 0; i < n; ++i) {
      const int b = i & 1;
      if (!ptx::mbar_wait_warp(bar(C::B_SFULL + b), (i >> 1) & 1, abort_flag, a.timeout_ns, kErrTimeout)) break;
      ptx::tc_fence_after();
      uint32_t raw[BK / 32][32];
#pragma unroll
      for (int c = 0; c < BK / 32; ++c)
        ptx::tmem_ld32(lane_base + (b ? C::TM_S1 : C::TM_S0) + g * BK + c * 32, raw[c]);
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
      ptx::mbar_arrive(bar(C::B_SFREE + b));  // S_b is in registers: the MMA may overwrite it
      const int blk = (t0 + i) * G + g;
      const int nvalid = a.P - blk * BK;      // keys of my block below P
      uint64_t acc0 = ptx::f32x2(0.f, 0.f), acc1 = acc0;
#pragma unroll
      for (int c = 0; c < BK / 32; ++c) {
        ptx::reg_fence32(raw[c]);
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float x0, x1;
          ptx::f32x2_split(ptx::fma_f32x2(ptx::f32x2(__uint_as_float(raw[c][e]), __uint_as_float(raw[c][e + 1])), sl2,
                                          nl2),
                           x0, x1);
          float p0 = ptx::ex2(x0), p1 = ptx::ex2(x1);
          if (nvalid < BK) {  // the ragged end of the prefix
            p0 = c * 32 + e < nvalid ? p0 : 0.f;
            p1 = c * 32 + e + 1 < nvalid ? p1 : 0.f;
          }
          if (e & 2)
            acc1 = ptx::add_f32x2(acc1, ptx::f32x2(p0, p1));
          else
            acc0 = ptx::add_f32x2(acc0, ptx::f32x2(p0, p1));
        }
      }
      float a0, a1, b0, b1;
      ptx::f32x2_split(acc0, a0, a1);
      ptx::f32x2_split(acc1, b0, b1);
      if (valid && blk < a.nkb) out[blk] = (a0 + b0) + (a1 + b1);
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::TM_ALLOC);
  }
}

}  // namespace sparsed
