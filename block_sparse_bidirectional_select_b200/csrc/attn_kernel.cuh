// Dense bidirectional attention for sm_100a, two query tiles per CTA.
//
// Work item (h, i): one head h and one query block i of up to 128 rows,
//   O = softmax(scale * Q_i K^T) V over every key block 0..nkb-1, and the
//   fp32 natural-log LSE of every row (SparseD abstract: full attention in the
//   early denoising steps; Step-dLLM abstract: the full map is recomputed at
//   every step). Block-sparse passes, whose query tiles each walk their own
//   list, run in the one-tile kernel of attn_list_kernel.cuh.
//
// A CTA works on pairs of work items, (h, 2p) in slot 0 and (h, 2p+1) in
// slot 1. Each slot has its own Q tile, S/P and O in TMEM, its own softmax
// warpgroup and its own MMA-issuing warp. Both slots read the same K_t / V_t
// tiles, so a tile is loaded once for two query tiles. Per slot the chain is
// S(t) = Q K_t^T -> softmax -> O += P(t) V_t -> S(t+1). The two slots run it
// independently, so the tensor core works on one slot's MMAs while the other
// slot's softmax runs. O += P V is issued in NPV parts, each as soon as the
// softmax has stored that part of P, so it overlaps the rest of the
// exponentials.
//
// Persistent CTAs: the grid holds one CTA per SM and CTA b starts with pair b
// of the flattened (h, p) order. Its later pairs are b + G, b + 2G, ... (G =
// grid size) or, given a counter, the next unclaimed pair, so the CTAs
// resident at any moment cover consecutive query blocks of at most two heads
// and share their K/V tiles in L2. The producer takes each pair index and
// publishes it to the other warps through shared memory (B_WFULL / B_WEMPTY).
// The pipelines run on across pair boundaries.
//
// Warp roles (384 threads):
//   warps 0-3   softmax of slot 0: warp w holds rows 32w..32w+31 of the tile,
//               one full row per thread (row max and sum need no exchange)
//   warps 4-7   softmax of slot 1, likewise
//   warp 8      TMA producer: Q of each slot, K_t and V_t into one NST-deep ring
//   warp 9      TMEM owner; MMA issuer of slot 0
//   warp 10     MMA issuer of slot 1
//   warp 11     idle (donates its registers)
// The producer and issuers run warp-uniform code and one elected lane issues
// each copy, MMA and commit.
// TMEM (128 lanes): [S0 | S1 | O0 | O1] = 2*BK + 2*D fp32 columns. P_s is
// written as bf16 pairs over the first BK/2 columns of S_s, which PV_s reads
// before S_s(t+1) overwrites them (MMAs of one thread execute in order).
// Ordering facts the roles rely on (a slot's MMAs all come from one thread,
// and a commit tracks every MMA that thread issued before it):
//   * S_s(t) is issued after PV_s(t-1), so when S_s(t) completes (SFULL_s),
//     O_s holds every tile before t: the softmax may rescale O_s right away;
//   * the first part of PV_s(t) waits for the softmax's first PFULL_s(t)
//     arrival, which follows its rescale of O_s and its epilogue reads of O_s
//     (the first PV of an item overwrites O_s);
//   * a ring stage is released by two commits after the MMAs reading it, one
//     from each slot (two from slot 0 when the pair has no second query block).
// The lazy rescale keeps O and the running sum on a stale row max until some
// row of the warp sees its max grow by more than 2^8 (warp-uniform decision).
// MASS variant: the pass also yields the block mass of pattern selection.
// Each tile's probabilities of a row sum to ps = sum_c 2^(s_c*sl2 - m) in the
// exp pass; times 2^(m - lse2), with lse2 the row's LSE from an earlier full
// pass of the same inputs, that is the row's mass in the tile, and the warp
// writes its 32 rows' sum as one of kMassParts partials per tile.
// Every wait is bounded (mbarriers only, no named barriers), so a timed-out
// warp cannot strand the others.
#pragma once

#include "ptx_sm100.cuh"

namespace sparsed {

// Partial block-mass sums per (head, query block, key block) written by the
// MASS variant: one per softmax warp of a slot.
constexpr int kMassParts = 4;

struct AttnArgs {
  int H, L, bq, nqb, nkb;
  int Lk;                    // keys (== L, except over the gathered columns of a column pattern)
  float scale_log2;          // scale * log2(e)
  const int32_t* kv_idx;     // block-sparse passes (attn_list_kernel) only
  const int32_t* kv_count;   // block-sparse passes only
  int kv_stride;
  float* lse;                // [H, L]
  uint16_t* o;               // [H, L, D]
  // block mass from this pass (MASS variant): the LSE of an earlier full pass
  // of the same inputs, and per (head, query block, key block) one partial sum
  // per softmax warp, [H, nqb, nkb, kMassParts]
  const float* lse_prev;
  float* mass_part;
  uint64_t timeout_ns;       // bound of every device-side wait
  // Pair scheduling (two-tile kernel). sched == nullptr: CTA b takes pairs b,
  // b + G, b + 2G, ... (G = grid size). Otherwise CTA b takes pair b first and
  // then claims pair G + atomicAdd(sched, 1) until the pairs run out, so the
  // pairs in flight stay a window of about G consecutive pairs however
  // unevenly the CTAs progress. *sched must be 0 at launch; the kernel sets
  // *sched_reset (nullable) to 0 for the next launch.
  int* sched;
  int* sched_reset;
};

__device__ __forceinline__ void setmaxnreg_inc_224() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 224;" ::: "memory");
}
__device__ __forceinline__ void setmaxnreg_dec_56() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 56;" ::: "memory");
}

template <int D, int BK>
struct AttnCfg {
  static constexpr int M = 128;
  static constexpr int DCH = D / 64;
  static constexpr int Q_CHUNK = M * 128;    // bytes of one 64-column chunk of a Q tile
  static constexpr int KV_CHUNK = BK * 128;  // ... of a K or V tile
  static constexpr int Q_BYTES = M * D * 2;
  static constexpr int KV_BYTES = BK * D * 2;
  static constexpr int SMEM_LIMIT = 232448;
  static constexpr int NST_FIT = (SMEM_LIMIT - 1024 - 2 * Q_BYTES - 512) / KV_BYTES;
  static constexpr int NST = NST_FIT > 8 ? 8 : NST_FIT;  // ring stages (K and V tiles)
  static constexpr int OFF_Q0 = 0;
  static constexpr int OFF_Q1 = Q_BYTES;
  static constexpr int OFF_RING = 2 * Q_BYTES;
  static constexpr int OFF_BAR = OFF_RING + NST * KV_BYTES;
  static constexpr int B_QFULL = 0;             // [2]
  static constexpr int B_QEMPTY = 2;            // [2]
  static constexpr int B_FULL = 4;              // [NST]
  static constexpr int B_EMPTY = B_FULL + NST;  // [NST]
  static constexpr int NPV = 2;                 // parts of P / of the PV MMAs of a tile
  static constexpr int B_SFULL = B_EMPTY + NST; // [2]
  static constexpr int B_PFULL = B_SFULL + 2;   // [2][NPV] 4 warp arrivals
  static constexpr int B_PVDONE = B_PFULL + 2 * NPV;  // [2]
  static constexpr int B_DRAIN = B_PVDONE + 2;  // [2]
  static constexpr int B_WFULL = B_DRAIN + 2;   // [2] pair index published
  static constexpr int B_WEMPTY = B_WFULL + 2;  // [2] pair index read by every consumer warp
  static constexpr int N_WTAKERS = 10;          // softmax warps 0-7, MMA issuers 9-10
  static constexpr int NUM_BARS = B_WEMPTY + 2;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;  // tmem slot, abort flag, pair index [2]
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int TM_S0 = 0;
  static constexpr int TM_S1 = BK;
  static constexpr int TM_O0 = 2 * BK;
  static constexpr int TM_O1 = 2 * BK + D;
  static constexpr int TM_USED = 2 * BK + 2 * D;
  static constexpr int TM_ALLOC = TM_USED <= 256 ? 256 : 512;
  static constexpr uint32_t IDESC_S = ptx::idesc_bf16_f32(128, BK, 0, 0);
  static constexpr uint32_t IDESC_PV = ptx::idesc_bf16_f32(128, D, 0, 1);
  static constexpr int THREADS = 384;
  static constexpr int REGS_SOFTMAX = 224;  // warps 0-7
  static constexpr int REGS_OTHER = 56;     // warps 8-11
  static_assert(NST >= 4, "ring too shallow");
  static_assert(TM_USED <= 512, "TMEM budget");
  static_assert(SMEM_BYTES <= SMEM_LIMIT, "shared memory budget");
};

// The exp pass over 32 columns of a row: P = bf16(2^(s*sl2 - m)) packed in
// pairs (even column in the low half), the fp32 sums into acc0 / acc1.
__device__ __forceinline__ void exp_chunk32(const float* s, uint64_t scale2, uint64_t negm2, uint32_t (&pk)[16],
                                            uint64_t& acc0, uint64_t& acc1) {
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    float x0, x1;
    ptx::f32x2_split(ptx::fma_f32x2(ptx::f32x2(s[2 * e], s[2 * e + 1]), scale2, negm2), x0, x1);
    const float p0 = ptx::ex2(x0);
    const float p1 = ptx::ex2(x1);
    if (e & 1)
      acc1 = ptx::add_f32x2(acc1, ptx::f32x2(p0, p1));
    else
      acc0 = ptx::add_f32x2(acc0, ptx::f32x2(p0, p1));
    pk[e] = ptx::pack_bf16x2(p0, p1);
  }
}

// Query blocks of pair w: (h, 2p) and (h, 2p+1), the second absent when nqb
// is odd and p is the head's last pair.
struct Pair {
  int h, q0;
  bool has1;
};

__device__ __forceinline__ Pair pair_of(const AttnArgs& a, int w, int npairs_h) {
  Pair r;
  r.h = w / npairs_h;
  const int p = w - r.h * npairs_h;
  r.q0 = 2 * p;
  r.has1 = r.q0 + 1 < a.nqb;
  return r;
}

template <int D, int BK, bool MASS = false>
__global__ void __launch_bounds__(384, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const AttnArgs a) {
  using C = AttnCfg<D, BK>;
  constexpr int NST = C::NST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sb = ptx::smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int npairs_h = (a.nqb + 1) >> 1;
  const int n_pairs = a.H * npairs_h;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  // the producer publishes each pair index it takes here, double-buffered
  volatile int* pair_w = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  auto bar = [&](int idx) -> uint32_t { return sb + C::OFF_BAR + 8 * idx; };

  // ---- setup
  if (threadIdx.x == 0) {
    if (a.sched_reset && blockIdx.x == 0) *a.sched_reset = 0;
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(bar(C::B_WFULL + s), 1);
      ptx::mbar_init(bar(C::B_WEMPTY + s), C::N_WTAKERS);
      ptx::mbar_init(bar(C::B_QFULL + s), 1);
      ptx::mbar_init(bar(C::B_QEMPTY + s), 1);
      ptx::mbar_init(bar(C::B_SFULL + s), 1);
      for (int q = 0; q < C::NPV; ++q)
        ptx::mbar_init(bar(C::B_PFULL + s * C::NPV + q), 4);  // one arrival per softmax warp of the slot
      ptx::mbar_init(bar(C::B_PVDONE + s), 1);
      ptx::mbar_init(bar(C::B_DRAIN + s), 1);
    }
    for (int s = 0; s < NST; ++s) {
      ptx::mbar_init(bar(C::B_FULL + s), 1);
      ptx::mbar_init(bar(C::B_EMPTY + s), 2);  // two commits per tile
    }
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 9) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), C::TM_ALLOC);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8) {
    setmaxnreg_dec_56();
    const uint32_t leader = ptx::elect_one();
    auto wait = [&](int idx, int parity) -> bool {
      return ptx::mbar_wait_warp(bar(idx), parity & 1, abort_flag, a.timeout_ns, kErrTimeout);
    };
    if (warp == 8) {
      // ============================================================ producer
      // warp-uniform; one elected lane issues the copies
      if (leader) {
        ptx::tma_prefetch_desc(&tm_q);
        ptx::tma_prefetch_desc(&tm_k);
        ptx::tma_prefetch_desc(&tm_v);
      }
      int seq = 0;               // ring tiles issued
      int qn0 = 0, qn1 = 0;      // Q tiles issued per slot
      bool ok = true;
      int h = 0;
      // one K or V tile of key block blk into the next ring stage
      auto load_tile = [&](const CUtensorMap* tm, int blk) -> bool {
        const int st = seq % NST;
        if (seq >= NST && !wait(C::B_EMPTY + st, (seq / NST) - 1)) return false;
        ptx::mbar_arrive_expect_tx_if(leader, bar(C::B_FULL + st), C::KV_BYTES);
#pragma unroll
        for (int c = 0; c < C::DCH; ++c)
          ptx::tma_load_3d_if(leader, sb + C::OFF_RING + st * C::KV_BYTES + c * C::KV_CHUNK, tm, bar(C::B_FULL + st),
                              c * 64, blk * BK, h);
        ++seq;
        return true;
      };
      auto load_q = [&](int s, int qi) -> bool {
        const int qn = s ? qn1 : qn0;
        if (qn > 0 && !wait(C::B_QEMPTY + s, qn - 1)) return false;
        ptx::mbar_arrive_expect_tx_if(leader, bar(C::B_QFULL + s), C::Q_BYTES);
#pragma unroll
        for (int c = 0; c < C::DCH; ++c)
          ptx::tma_load_3d_if(leader, sb + (s ? C::OFF_Q1 : C::OFF_Q0) + c * C::Q_CHUNK, &tm_q, bar(C::B_QFULL + s),
                              c * 64, qi * a.bq, h);
        if (s) ++qn1;
        else ++qn0;
        return true;
      };
      int np = 0;  // pair indices published
      // publish pair index w (n_pairs: no more pairs) once every consumer
      // warp has read the index published two before it
      auto publish = [&](int w) -> bool {
        const int b = np & 1;
        if (np >= 2 && !wait(C::B_WEMPTY + b, (np >> 1) - 1)) return false;
        if (leader) {
          pair_w[b] = w;
          ptx::mbar_arrive(bar(C::B_WFULL + b));
        }
        __syncwarp();
        ++np;
        return true;
      };
      int w = blockIdx.x;
      while (ok) {
        ok = publish(w < n_pairs ? w : n_pairs);
        if (!ok || w >= n_pairs) break;
        const Pair pr = pair_of(a, w, npairs_h);
        h = pr.h;
        // the CTA's next pair: the static stride, or a claim on the counter
        int w_next = w + static_cast<int>(gridDim.x);
        if (a.sched) {
          int claim = 0;
          if (leader) claim = atomicAdd(a.sched, 1);
          w_next = static_cast<int>(gridDim.x) + __reduce_max_sync(0xffffffffu, claim);
        }
        // the next pair's Q rows into L2 while this pair runs
        if (leader && w_next < n_pairs) {
          const Pair pn = pair_of(a, w_next, npairs_h);
#pragma unroll
          for (int c = 0; c < C::DCH; ++c) {
            ptx::tma_prefetch_3d(&tm_q, c * 64, pn.q0 * a.bq, pn.h);
            if (pn.has1) ptx::tma_prefetch_3d(&tm_q, c * 64, (pn.q0 + 1) * a.bq, pn.h);
          }
        }
        // in the order the slots consume them: Q0, K_0, Q1, V_0, K_1, V_1, ...
        for (int j = 0; ok && j < a.nkb; ++j) {
          if (j == 0) ok = load_q(0, pr.q0);
          if (ok) ok = load_tile(&tm_k, j);
          if (ok && pr.has1 && j == 0) ok = load_q(1, pr.q0 + 1);
          if (ok) ok = load_tile(&tm_v, j);
        }
        w = w_next;
      }
      if (!ok) {
        // let the copies in flight land before the CTA's shared memory goes
        // away: the last Q of each slot and the last NST tiles
        const uint64_t short_ns = a.timeout_ns / 4;
        volatile int dummy = 0;
        if (qn0 > 0) ptx::mbar_wait(bar(C::B_QFULL + 0), (qn0 - 1) & 1, &dummy, short_ns, 0);
        if (qn1 > 0) ptx::mbar_wait(bar(C::B_QFULL + 1), (qn1 - 1) & 1, &dummy, short_ns, 0);
        for (int u = (seq > NST ? seq - NST : 0); u < seq; ++u)
          ptx::mbar_wait(bar(C::B_FULL + u % NST), (u / NST) & 1, &dummy, short_ns, 0);
        __syncwarp();
      }
    } else if (warp == 9 || warp == 10) {
      // ============================================================ MMA issuers
      // Warp 9 issues slot 0's MMAs, warp 10 slot 1's, so neither slot's chain
      // (S(t) -> softmax -> PV(t) -> S(t+1)) waits on the other's softmax. The
      // whole warp runs the loop (warp-uniform control flow, descriptors in
      // uniform registers); one elected lane issues the MMAs and commits. A
      // ring stage gets two commits (EMPTY counts two): one from each slot, or
      // both from slot 0 when the pair has no second query block.
      const int s = warp - 9;
      constexpr uint32_t HI = ptx::sdesc_sw128_hi(1024);
      const uint32_t q_lo = ptx::sdesc_sw128_lo(sb + (s ? C::OFF_Q1 : C::OFF_Q0), 16);
      const uint32_t k_lo = ptx::sdesc_sw128_lo(sb + C::OFF_RING, 16);
      const uint32_t v_lo = ptx::sdesc_sw128_lo(sb + C::OFF_RING, C::KV_CHUNK);
      const uint32_t s_tmem = tmem + (s ? C::TM_S1 : C::TM_S0);
      const uint32_t o_tmem = tmem + (s ? C::TM_O1 : C::TM_O0);
      constexpr int KPP = BK / 16 / C::NPV;  // PV MMAs per part of P
      int seq = 0;      // ring tiles (same numbering as the producer)
      int qn = 0;       // Q tiles consumed
      int tcnt = 0;     // tiles of this slot (PFULL phases)
      bool ok = true;
      auto commit = [&](int idx) { ptx::umma_commit_if(leader, bar(idx)); };
      for (int np = 0; ok; ++np) {
        if (!wait(C::B_WFULL + (np & 1), np >> 1)) {
          ok = false;
          break;
        }
        const int w = pair_w[np & 1];
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(C::B_WEMPTY + (np & 1)));
        if (w >= n_pairs) break;
        const Pair pr = pair_of(a, w, npairs_h);
        const bool mine = s == 0 || pr.has1;   // slot 1 idles on a pair without a second block
        const bool sole = !pr.has1;             // slot 0 then gives both commits of each tile
        for (int j = 0; j < a.nkb; ++j) {
          const int sk = seq, sv = seq + 1;     // K_j and V_j
          seq += 2;
          if (!mine) continue;
          if ((j == 0 && !wait(C::B_QFULL + s, qn++)) || !wait(C::B_FULL + sk % NST, sk / NST)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            constexpr uint32_t QC = C::Q_CHUNK >> 4, KC = C::KV_CHUNK >> 4;
            const uint32_t ao = (kk >> 2) * QC + (kk & 3) * 2;
            const uint32_t bo = (kk >> 2) * KC + (kk & 3) * 2;
            ptx::umma_ss_lohi_if(leader, s_tmem, q_lo + ao,
                                 k_lo + static_cast<uint32_t>((sk % NST) * C::KV_BYTES >> 4) + bo, HI, C::IDESC_S,
                                 kk > 0 ? 1u : 0u);
          }
          commit(C::B_SFULL + s);
          commit(C::B_EMPTY + sk % NST);
          if (sole) commit(C::B_EMPTY + sk % NST);
          if (j == a.nkb - 1) commit(C::B_QEMPTY + s);
          // O += P V in NPV parts, each issued as soon as the softmax has
          // stored that part of P
          if (!wait(C::B_FULL + sv % NST, sv / NST)) {
            ok = false;
            break;
          }
          const uint32_t vb = v_lo + static_cast<uint32_t>((sv % NST) * C::KV_BYTES >> 4);
#pragma unroll
          for (int q = 0; q < C::NPV; ++q) {
            if (!wait(C::B_PFULL + s * C::NPV + q, tcnt)) {
              ok = false;
              break;
            }
            ptx::tc_fence_after();
#pragma unroll
            for (int u = 0; u < KPP; ++u) {
              const int kk = q * KPP + u;
              ptx::umma_ts_lohi_if(leader, o_tmem, s_tmem + kk * 8, vb + kk * (2048 >> 4), HI, C::IDESC_PV,
                                   (j > 0 || kk > 0) ? 1u : 0u);
            }
          }
          if (!ok) break;
          commit(C::B_PVDONE + s);
          commit(C::B_EMPTY + sv % NST);
          if (sole) commit(C::B_EMPTY + sv % NST);
          ++tcnt;
        }
        if (!ok) break;
      }
      if (!ok) {
        commit(C::B_DRAIN + s);
        volatile int dummy = 0;
        ptx::mbar_wait(bar(C::B_DRAIN + s), 0, &dummy, a.timeout_ns / 4, 0);
        __syncwarp();
      }
    }
  } else {
    // ================================================================ softmax
    setmaxnreg_inc_224();
    const int slot = warp >> 2;
    const int wq = warp & 3;
    const int r = wq * 32 + lane;  // row == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t s_col = slot ? C::TM_S1 : C::TM_S0;
    const uint32_t o_col = slot ? C::TM_O1 : C::TM_O0;
    const float sl2 = a.scale_log2;
    const uint64_t scale2 = ptx::f32x2(sl2, sl2);
    int tcount = 0;  // tiles of this slot so far (SFULL / PVDONE phases)
    bool ok = true;
    for (int np = 0; ok; ++np) {
      if (!ptx::mbar_wait_warp(bar(C::B_WFULL + (np & 1)), (np >> 1) & 1, abort_flag, a.timeout_ns, kErrTimeout)) {
        ok = false;
        break;
      }
      const int w = pair_w[np & 1];
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar(C::B_WEMPTY + (np & 1)));
      if (w >= n_pairs) break;
      const Pair pr = pair_of(a, w, npairs_h);
      const int h = pr.h;
      const int qi = pr.q0 + slot;
      if (slot == 1 && !pr.has1) continue;
      const int grow = qi * a.bq + r;
      const bool row_valid = (r < a.bq) && (grow < a.L);
      uint4* o_dst = reinterpret_cast<uint4*>(a.o + (static_cast<long>(h) * a.L + grow) * D);
      float m = -__int_as_float(0x7f800000);  // running row max, log2 units (scaled)
      float l = 0.f;                          // running row sum
      // MASS: my row's LSE (log2 units) from the earlier full pass
      float lse2_prev = 0.f;
      if constexpr (MASS)
        lse2_prev = row_valid ? a.lse_prev[static_cast<long>(h) * a.L + grow] * 1.44269504088896340736f : 0.f;
      for (int jj = 0; jj < a.nkb; ++jj, ++tcount) {
        const int blk = jj;
        if (!ptx::mbar_wait_warp(bar(C::B_SFULL + slot), tcount & 1, abort_flag, a.timeout_ns, kErrTimeout)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        float s[BK];
        {
          uint32_t raw[BK / 32][32];
#pragma unroll
          for (int c = 0; c < BK / 32; ++c) ptx::tmem_ld32(lane_base + s_col + c * 32, raw[c]);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < BK / 32; ++c) {
            ptx::reg_fence32(raw[c]);
#pragma unroll
            for (int e = 0; e < 32; ++e) s[c * 32 + e] = __uint_as_float(raw[c][e]);
          }
        }
        // ragged last key block: keys past Lk do not exist
        const int valid = a.Lk - blk * BK;
        if (valid < BK) {
#pragma unroll
          for (int c = 0; c < BK; ++c)
            if (c >= valid) s[c] = -__int_as_float(0x7f800000);
        }
        float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
        for (int c = 4; c < BK; c += 8) {
          mx0 = ptx::max3(mx0, s[c], s[c + 1]);
          mx1 = ptx::max3(mx1, s[c + 2], s[c + 3]);
          if (c + 4 < BK) {
            mx2 = ptx::max3(mx2, s[c + 4], s[c + 5]);
            mx3 = ptx::max3(mx3, s[c + 6], s[c + 7]);
          }
        }
        const float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
        const float m_new = fmaxf(m, mx * sl2);
        if (jj == 0) {
          m = m_new;
        } else if (__any_sync(0xffffffffu, m_new > m + 8.0f)) {
          // O_s holds every earlier tile of this item (S_s(t) was issued after
          // PV_s(t-1)): rescale my row
          const float alpha = ptx::ex2(m - m_new);
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t raw[32];
            ptx::tmem_ld32(lane_base + o_col + c * 32, raw);
            ptx::tmem_wait_ld();
            ptx::reg_fence32(raw);
#pragma unroll
            for (int e = 0; e < 32; ++e) raw[e] = __float_as_uint(__uint_as_float(raw[e]) * alpha);
            ptx::tmem_st32(lane_base + o_col + c * 32, raw);
          }
          l *= alpha;
          m = m_new;
        }
        // P_s over the first BK/2 columns of S_s (read out above)
        const uint64_t negm2 = ptx::f32x2(-m, -m);
        uint64_t acc0 = ptx::f32x2(0.f, 0.f), acc1 = acc0;
        constexpr int CPP = BK / 32 / C::NPV;  // 32-column chunks per part of P
#pragma unroll
        for (int c = 0; c < BK / 32; ++c) {
          uint32_t pk[16];
          exp_chunk32(s + 32 * c, scale2, negm2, pk, acc0, acc1);
          ptx::tmem_st32_16(lane_base + s_col + c * 16, pk);
          if ((c + 1) % CPP == 0 && c + 1 < BK / 32) {
            // this part of P is in TMEM: its PV MMAs may start
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(C::B_PFULL + slot * C::NPV + c / CPP));
          }
        }
        float a0, a1, b0, b1;
        ptx::f32x2_split(acc0, a0, a1);
        ptx::f32x2_split(acc1, b0, b1);
        const float ps = (a0 + b0) + (a1 + b1);
        l += ps;
        if constexpr (MASS) {
          // this tile's probability mass of my row is ps * 2^(m - lse2); the
          // warp's 32 rows summed by a fixed shuffle tree
          float cm = row_valid ? ps * ptx::ex2(m - lse2_prev) : 0.f;
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) cm += __shfl_xor_sync(0xffffffffu, cm, off);
          if (lane == 0) a.mass_part[((static_cast<long>(h) * a.nqb + qi) * a.nkb + jj) * kMassParts + wq] = cm;
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(C::B_PFULL + slot * C::NPV + C::NPV - 1));
      }
      if (!ok) break;
      // ---- epilogue: every PV of the item is done -> O / l -> bf16 -> global; LSE
      if (!ptx::mbar_wait_warp(bar(C::B_PVDONE + slot), (tcount - 1) & 1, abort_flag, a.timeout_ns, kErrTimeout)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const float inv_l = 1.0f / l;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t raw[32];
        ptx::tmem_ld32(lane_base + o_col + c * 32, raw);
        ptx::tmem_wait_ld();
        ptx::reg_fence32(raw);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = ptx::pack_bf16x2(__uint_as_float(raw[2 * e]) * inv_l, __uint_as_float(raw[2 * e + 1]) * inv_l);
        if (row_valid) {
#pragma unroll
          for (int u = 0; u < 4; ++u)
            o_dst[c * 4 + u] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
        }
      }
      if (row_valid) a.lse[static_cast<long>(h) * a.L + grow] = (m + ptx::lg2(l)) * 0.69314718055994530942f;
      // the next item's first PV overwrites O_s only after this warp's next
      // PFULL arrival, which follows the loads above (tcgen05.wait::ld)
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::TM_ALLOC);
  }
}

}  // namespace sparsed
