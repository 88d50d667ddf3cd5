// Block-sparse attention for sm_100a, one query tile per CTA (the kernel of
// the block-sparse steps).
//
// Work item (h, i): one head h and one query block i of up to 128 rows,
//   O = softmax(scale * Q_i K^T) V over the key blocks kv_idx[h,i,0..kv_count)
//   (Step-dLLM abstract: block-sparse attention over a reused mask), and the
//   fp32 natural-log LSE of every row.
// Each work item walks its own list, so no K/V tile is shared between the
// query tiles of a CTA; the one-tile layout keeps Q to 32 KB of shared memory
// and gives K and V three ring stages each (6 tiles = 192 KB), enough to
// cover the copy latency of a list walked at full speed, with S
// double-buffered in TMEM so that S(g+1) is computed while the softmax works
// on S(g). (Dense passes, whose K/V tiles two query tiles can share, run in
// the two-tile kernel of attn_kernel.cuh.)
//
// Persistent CTAs: the grid holds one CTA per SM and CTA b takes the work
// items b, b + G, b + 2G, ... of the flattened (h, i) order (G = grid size), so
// the CTAs resident at any moment cover consecutive query blocks of one head
// and share its K/V tiles in L2. Every pipeline below runs on across item
// boundaries (the tile counter g counts tiles over all of the CTA's items).
//
// Warp roles (384 threads):
//   warps 0-7   softmax. Warp w covers the 16 rows 32*(w%4) + 16*(w/4) + 0..15
//               of the tile with the "16x32bx2" TMEM access: thread t holds row
//               t%16 and the column half t/16 of every S tile, so the two
//               halves of a row meet in one warp (row max / sum by shuffle).
//   warp 8      TMA producer: Q of each item, K_g / V_g into KS- / VS-deep rings
//   warp 9      TMEM owner; issues the S = Q K^T MMAs
//   warp 10     issues the O += P V MMAs
// (warps 8-10 run warp-uniform code; one elected lane issues each copy, MMA
// and commit)
//   warp 11     idle (donates its registers)
// TMEM (128 lanes): [S0 | S1 | O | Q0 | Q1] = 2*BK + 2*D fp32 columns. S is
// double-buffered, so S(g+1) is computed while the softmax works on S(g); P(g)
// is written over the first BK/2 columns of S_b(g) once the softmax has read
// them. Q sits in TMEM (two buffers, one per item in flight) so that
// S = Q K^T is a TS MMA: only K comes from shared memory, which leaves shared
// memory bandwidth for the K/V copies. The two issuers run independently (a
// commit from one thread tracks only its own MMAs):
//   S issuer : S_b(g) once PV(g-2) is done (the softmax has read S_b(g-2) and
//              PV has read the P_b(g-2) written over it)       (PVDONE)
//              and the item's Q is in TMEM                      (QTFULL)
//   softmax  : reads S_b(g), writes P_b(g) over it              (SFULL -> PFULL)
//              copies each item's Q from shared memory into TMEM Q_c, after
//              every S MMA that read Q_c two items earlier      (QFULL, QTEMPTY
//                                                                -> QTFULL, QEMPTY)
//   PV issuer: O += P_b(g) V_g; the first tile of an item overwrites O, which
//              the softmax warps have read out before they wrote that P
//                                                               (PFULL -> PVDONE)
//   producer : Q of the next item once the softmax has copied the current
//              one into TMEM                                    (QEMPTY)
// The lazy rescale keeps O and the running sum on a stale row max until a
// row's max grows by more than 2^8; both halves of a row see the same max, so
// they take the same decision, and each rescales its half of O.
// The epilogue writes O straight from registers to global memory (each thread
// one contiguous half row), so no shared memory is held across items.
// Every wait is bounded (mbarriers only, no named barriers), so a timed-out
// warp cannot strand the others.
#pragma once

#include "attn_kernel.cuh"

namespace sparsed {

template <int D, int BK>
struct ListCfg {
  static constexpr int M = 128;
  static constexpr int HALF = BK / 2;  // S columns per softmax thread
  static constexpr int DCH = D / 64;
  static constexpr int Q_CHUNK = M * 128;
  static constexpr int KV_CHUNK = BK * 128;
  static constexpr int Q_BYTES = M * D * 2;
  static constexpr int KV_BYTES = BK * D * 2;
  static constexpr int KS = 3;
  // a third V stage when it fits next to Q, three K stages and the barriers
  static constexpr int VS = (Q_BYTES + 6 * KV_BYTES + 2048) <= 232448 ? 3 : 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = Q_BYTES;
  static constexpr int OFF_V = OFF_K + KS * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + VS * KV_BYTES;
  static constexpr int B_QFULL = 0;
  static constexpr int B_QEMPTY = 1;             // 8 softmax-warp arrivals: Q copied into TMEM
  static constexpr int B_KFULL = 2;
  static constexpr int B_KEMPTY = B_KFULL + KS;
  static constexpr int B_VFULL = B_KEMPTY + KS;
  static constexpr int B_VEMPTY = B_VFULL + VS;
  static constexpr int B_SFULL = B_VEMPTY + VS;  // [2]
  static constexpr int B_PFULL = B_SFULL + 2;    // [2] 8 warp arrivals
  static constexpr int B_PVDONE = B_PFULL + 2;   // [2]
  static constexpr int B_DRAIN = B_PVDONE + 2;   // [2] per issuer
  static constexpr int B_QTFULL = B_DRAIN + 2;   // [2] Q_c in TMEM: 8 softmax-warp arrivals
  static constexpr int B_QTEMPTY = B_QTFULL + 2; // [2] every S MMA that read Q_c is complete
  static constexpr int NUM_BARS = B_QTEMPTY + 2;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;  // tmem slot, abort flag
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int TM_S0 = 0;
  static constexpr int TM_S1 = BK;
  static constexpr int TM_O = 2 * BK;
  static constexpr int TM_Q0 = 2 * BK + D;       // Q as the A operand: D/2 columns of bf16 pairs
  static constexpr int TM_Q1 = TM_Q0 + D / 2;
  static constexpr int TM_USED = TM_Q1 + D / 2;
  static constexpr int TM_ALLOC = TM_USED <= 256 ? 256 : 512;
  static constexpr uint32_t IDESC_S = ptx::idesc_bf16_f32(128, BK, 0, 0);
  static constexpr uint32_t IDESC_PV = ptx::idesc_bf16_f32(128, D, 0, 1);
  static constexpr int THREADS = 384;
  static constexpr int REGS_SOFTMAX = 224;
  static constexpr int REGS_OTHER = 56;
  static_assert(TM_USED <= 512, "TMEM budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// The exp pass of one half row: P = bf16(2^(s*sl2 - m)) for HALF columns into
// TMEM at p_taddr through the 16x32bx2 access (two columns per 32-bit cell,
// even column in the low half; the other half row's cells HALF/2 further on),
// returning the fp32 sum. Column pairs go through packed fp32x2 FMA/ADD.
template <int HALF>
__device__ __forceinline__ float softmax_half_exp(const float (&s)[HALF], float sl2, float m, uint32_t p_taddr) {
  static_assert(HALF == 32 || HALF == 64, "half row of 32 or 64 columns");
  const uint64_t scale2 = ptx::f32x2(sl2, sl2);
  const uint64_t negm2 = ptx::f32x2(-m, -m);
  uint64_t acc0 = ptx::f32x2(0.f, 0.f), acc1 = acc0;
  constexpr int W = HALF / 2;  // packed cells
  uint32_t pk[32];
#pragma unroll
  for (int e = 0; e < W; ++e) {
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
  // thread t's cells go to column half t/16 of the tile's P cells
  if constexpr (W == 32) {
    ptx::tmem_st16x2_32<HALF / 2>(p_taddr, pk);
  } else {
    ptx::tmem_st16x2_16<HALF / 2>(p_taddr, pk);
  }
  float a0, a1, b0, b1;
  ptx::f32x2_split(acc0, a0, a1);
  ptx::f32x2_split(acc1, b0, b1);
  return (a0 + b0) + (a1 + b1);
}

// One work item's key-block list.
template <bool SPARSE>
struct ItemList {
  int n = 0;
  const int32_t* list = nullptr;
  int nkb = 0;
  __device__ __forceinline__ int raw(int jj) const {
    if constexpr (SPARSE) return list[jj];
    else return jj;
  }
  // clamped for addressing: a bad entry (reported by the producer) reads block 0
  __device__ __forceinline__ int block(int jj) const {
    const int j = raw(jj);
    return (j >= 0 && j < nkb) ? j : 0;
  }
};

// kv_count of work item w (row h*nqb + i of the [H, nqb] count array); every
// role reads the next item's count one item ahead, off its critical path
template <bool SPARSE>
__device__ __forceinline__ int raw_count(const AttnArgs& a, int w) {
  if constexpr (SPARSE) return w < a.H * a.nqb ? a.kv_count[w] : 0;
  else return a.nkb;
}

template <bool SPARSE>
__device__ __forceinline__ ItemList<SPARSE> item_list(const AttnArgs& a, int w, int n_raw) {
  ItemList<SPARSE> it;
  it.nkb = a.nkb;
  it.n = a.nkb;
  if constexpr (SPARSE) {
    const int cap = a.kv_stride < a.nkb ? a.kv_stride : a.nkb;
    it.n = n_raw < 0 ? 0 : (n_raw > cap ? cap : n_raw);  // a bad count is reported by the producer
    it.list = a.kv_idx + static_cast<long>(w) * a.kv_stride;
  }
  return it;
}

template <int D, int BK>
__global__ void __launch_bounds__(384, 1)
    attn_list_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const AttnArgs a) {
  using C = ListCfg<D, BK>;
  constexpr int HALF = C::HALF;
  constexpr bool SPARSE = true;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sb = ptx::smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_items = a.H * a.nqb;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  auto bar = [&](int idx) -> uint32_t { return sb + C::OFF_BAR + 8 * idx; };

  // ---- setup
  if (threadIdx.x == 0) {
    ptx::mbar_init(bar(C::B_QFULL), 1);
    ptx::mbar_init(bar(C::B_QEMPTY), 8);  // one arrival per softmax warp
    for (int c = 0; c < 2; ++c) {
      ptx::mbar_init(bar(C::B_QTFULL + c), 8);
      ptx::mbar_init(bar(C::B_QTEMPTY + c), 1);
    }
    for (int s = 0; s < C::KS; ++s) {
      ptx::mbar_init(bar(C::B_KFULL + s), 1);
      ptx::mbar_init(bar(C::B_KEMPTY + s), 1);
    }
    for (int s = 0; s < C::VS; ++s) {
      ptx::mbar_init(bar(C::B_VFULL + s), 1);
      ptx::mbar_init(bar(C::B_VEMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(bar(C::B_SFULL + b), 1);
      ptx::mbar_init(bar(C::B_PFULL + b), 8);  // one arrival per softmax warp
      ptx::mbar_init(bar(C::B_PVDONE + b), 1);
      ptx::mbar_init(bar(C::B_DRAIN + b), 1);
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
  // As a programmatic dependent (the block-wise steps) the setup above ran
  // while the previous kernel finished; nothing global is read before here.
  ptx::grid_dep_wait();
  ptx::grid_dep_launch();

  if (warp >= 8) {
    setmaxnreg_dec_56();
    // The producer and the issuers run warp-uniform code (descriptors and
    // counters stay in uniform registers); one elected lane issues each copy,
    // MMA and commit.
    const uint32_t leader = ptx::elect_one();
    auto wait = [&](int idx, int parity) -> bool {
      return ptx::mbar_wait_warp(bar(idx), parity & 1, abort_flag, a.timeout_ns, kErrTimeout);
    };
    if (warp == 8) {
      // ============================================================ producer
      if (leader) {
        ptx::tma_prefetch_desc(&tm_q);
        ptx::tma_prefetch_desc(&tm_k);
        ptx::tma_prefetch_desc(&tm_v);
      }
      int g = 0, iq = 0;  // tile counter, Q tiles loaded so far
      int issued_k = 0, issued_v = 0;
      bool ok = true;
      int n_raw = raw_count<SPARSE>(a, blockIdx.x), n_raw_next = 0;
      for (int w = blockIdx.x; ok && w < n_items; w += gridDim.x, n_raw = n_raw_next) {
        n_raw_next = raw_count<SPARSE>(a, w + gridDim.x);
        const int h = w / a.nqb, qi = w - h * a.nqb;
        const ItemList<SPARSE> it = item_list<SPARSE>(a, w, n_raw);
        if (SPARSE && leader && n_raw != it.n) ptx::record_error(kErrBadPattern);
        if (it.n == 0) continue;
        // Q of this item once the softmax has copied the previous one into TMEM
        if (iq > 0 && !wait(C::B_QEMPTY, iq - 1)) {
          ok = false;
          break;
        }
        ptx::mbar_arrive_expect_tx_if(leader, bar(C::B_QFULL), C::Q_BYTES);
#pragma unroll
        for (int c = 0; c < C::DCH; ++c)
          ptx::tma_load_3d_if(leader, sb + C::OFF_Q + c * C::Q_CHUNK, &tm_q, bar(C::B_QFULL), c * 64, qi * a.bq, h);
        ++iq;
        // list entries are read one tile ahead, off the copy-issue path
        int prev = -1, raw_next = it.raw(0);
        for (int jj = 0; jj < it.n; ++jj, ++g) {
          const int raw = raw_next;
          if (jj + 1 < it.n) raw_next = it.raw(jj + 1);
          if constexpr (SPARSE) {
            if (leader && (raw < 0 || raw >= a.nkb || raw <= prev)) ptx::record_error(kErrBadPattern);
            prev = raw;
          }
          const int j = (raw >= 0 && raw < a.nkb) ? raw : 0;
          const int ks = g % C::KS;
          if (g >= C::KS && !wait(C::B_KEMPTY + ks, g / C::KS - 1)) {
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx_if(leader, bar(C::B_KFULL + ks), C::KV_BYTES);
#pragma unroll
          for (int c = 0; c < C::DCH; ++c)
            ptx::tma_load_3d_if(leader, sb + C::OFF_K + ks * C::KV_BYTES + c * C::KV_CHUNK, &tm_k,
                                bar(C::B_KFULL + ks), c * 64, j * BK, h);
          issued_k = g + 1;
          const int vs = g % C::VS;
          if (g >= C::VS && !wait(C::B_VEMPTY + vs, g / C::VS - 1)) {
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx_if(leader, bar(C::B_VFULL + vs), C::KV_BYTES);
#pragma unroll
          for (int c = 0; c < C::DCH; ++c)
            ptx::tma_load_3d_if(leader, sb + C::OFF_V + vs * C::KV_BYTES + c * C::KV_CHUNK, &tm_v,
                                bar(C::B_VFULL + vs), c * 64, j * BK, h);
          issued_v = g + 1;
        }
      }
      if (!ok) {
        // let the copies in flight land before the CTA's shared memory goes
        // away: the last Q and the last KS / VS tiles
        const uint64_t short_ns = a.timeout_ns / 4;
        volatile int dummy = 0;
        if (iq > 0) ptx::mbar_wait(bar(C::B_QFULL), (iq - 1) & 1, &dummy, short_ns, 0);
        for (int u = (issued_k > C::KS ? issued_k - C::KS : 0); u < issued_k; ++u)
          ptx::mbar_wait(bar(C::B_KFULL + u % C::KS), (u / C::KS) & 1, &dummy, short_ns, 0);
        for (int u = (issued_v > C::VS ? issued_v - C::VS : 0); u < issued_v; ++u)
          ptx::mbar_wait(bar(C::B_VFULL + u % C::VS), (u / C::VS) & 1, &dummy, short_ns, 0);
        __syncwarp();
      }
    } else if (warp == 9) {
      // ============================================================ S issuer
      constexpr uint32_t HI = ptx::sdesc_sw128_hi(1024);
      const uint32_t klo = ptx::sdesc_sw128_lo(sb + C::OFF_K, 16);
      int g = 0, iq = 0;
      bool ok = true;
      int n_raw = raw_count<SPARSE>(a, blockIdx.x), n_raw_next = 0;
      for (int w = blockIdx.x; ok && w < n_items; w += gridDim.x, n_raw = n_raw_next) {
        n_raw_next = raw_count<SPARSE>(a, w + gridDim.x);
        const ItemList<SPARSE> it = item_list<SPARSE>(a, w, n_raw);
        if (it.n == 0) continue;
        const int qc = iq & 1;
        if (!wait(C::B_QTFULL + qc, iq >> 1)) {
          ok = false;
          break;
        }
        const uint32_t q_tmem = tmem + (qc ? C::TM_Q1 : C::TM_Q0);
        for (int jj = 0; jj < it.n; ++jj, ++g) {
          const int b = g & 1;
          const int ks = g % C::KS;
          if (!wait(C::B_KFULL + ks, g / C::KS) || (g >= 2 && !wait(C::B_PVDONE + b, (g - 2) >> 1))) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t b0 = klo + static_cast<uint32_t>(ks * C::KV_BYTES >> 4);
          const uint32_t s_tmem = tmem + (b ? C::TM_S1 : C::TM_S0);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t bo = (kk >> 2) * (C::KV_CHUNK >> 4) + (kk & 3) * 2;
            ptx::umma_ts_lohi_if(leader, s_tmem, q_tmem + kk * 8, b0 + bo, HI, C::IDESC_S, kk > 0 ? 1u : 0u);
          }
          ptx::umma_commit_if(leader, bar(C::B_SFULL + b));
          ptx::umma_commit_if(leader, bar(C::B_KEMPTY + ks));
        }
        if (!ok) break;
        // every S MMA of this item read Q_qc: the softmax may copy a later item's Q there
        ptx::umma_commit_if(leader, bar(C::B_QTEMPTY + qc));
        ++iq;
      }
      if (!ok) {
        ptx::umma_commit_if(leader, bar(C::B_DRAIN));
        volatile int dummy = 0;
        ptx::mbar_wait(bar(C::B_DRAIN), 0, &dummy, a.timeout_ns / 4, 0);
        __syncwarp();
      }
    } else if (warp == 10) {
      // ============================================================ PV issuer
      constexpr uint32_t HI = ptx::sdesc_sw128_hi(1024);
      const uint32_t vlo = ptx::sdesc_sw128_lo(sb + C::OFF_V, C::KV_CHUNK);
      int g = 0;
      bool ok = true;
      int n_raw = raw_count<SPARSE>(a, blockIdx.x), n_raw_next = 0;
      for (int w = blockIdx.x; ok && w < n_items; w += gridDim.x, n_raw = n_raw_next) {
        n_raw_next = raw_count<SPARSE>(a, w + gridDim.x);
        const ItemList<SPARSE> it = item_list<SPARSE>(a, w, n_raw);
        for (int jj = 0; jj < it.n; ++jj, ++g) {
          const int b = g & 1;
          const int vs = g % C::VS;
          if (!wait(C::B_PFULL + b, g >> 1) || !wait(C::B_VFULL + vs, g / C::VS)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t b0 = vlo + static_cast<uint32_t>(vs * C::KV_BYTES >> 4);
          const uint32_t p_tmem = tmem + (b ? C::TM_S1 : C::TM_S0);  // P_b over S_b
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            ptx::umma_ts_lohi_if(leader, tmem + C::TM_O, p_tmem + kk * 8, b0 + kk * (2048 >> 4), HI, C::IDESC_PV,
                                 (jj > 0 || kk > 0) ? 1u : 0u);
          ptx::umma_commit_if(leader, bar(C::B_VEMPTY + vs));
          ptx::umma_commit_if(leader, bar(C::B_PVDONE + b));
        }
      }
      if (!ok) {
        ptx::umma_commit_if(leader, bar(C::B_DRAIN + 1));
        volatile int dummy = 0;
        ptx::mbar_wait(bar(C::B_DRAIN + 1), 0, &dummy, a.timeout_ns / 4, 0);
        __syncwarp();
      }
    }
  } else {
    // ================================================================ softmax
    setmaxnreg_inc_224();
    const int half = lane >> 4;                                        // column half of my row
    const int r = (warp & 3) * 32 + (warp >> 2) * 16 + (lane & 15);  // row == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32 + (warp >> 2) * 16) << 16);
    const float sl2 = a.scale_log2;
    const int s_off = half * HALF;  // first S column of my half row
    int g = 0;
    int iq = 0;  // items with work so far; their Q copies are numbered alike
    int cq = 0;  // Q copies into TMEM so far
    // Copy the Q tile in shared memory (that of item cq) into TMEM Q_{cq&1}, as
    // the A operand of the S MMAs: row r in lane r, elements 2j, 2j+1 in
    // column j. Warp w copies the 64-element chunk w/4 of rows 32*(w%4) ..
    // +31 (the 32x32b access); the tile is in the 128-byte swizzle of its
    // TMA copy (16-byte unit u of row r at unit u ^ (r % 8)).
    auto copy_q = [&]() -> bool {
      const int c = cq & 1;
      if (!ptx::mbar_wait_warp(bar(C::B_QFULL), cq & 1, abort_flag, a.timeout_ns, kErrTimeout)) return false;
      if (cq >= 2 &&
          !ptx::mbar_wait_warp(bar(C::B_QTEMPTY + c), ((cq >> 1) - 1) & 1, abort_flag, a.timeout_ns, kErrTimeout))
        return false;
      ptx::tc_fence_after();
      const int chunk = warp >> 2;
      if (chunk < C::DCH) {
        const int qr = (warp & 3) * 32 + lane;
        const uint8_t* src = smem + C::OFF_Q + chunk * C::Q_CHUNK + qr * 128;
        uint32_t v[32];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint4 x = *reinterpret_cast<const uint4*>(src + ((u ^ (qr & 7)) << 4));
          v[4 * u] = x.x;
          v[4 * u + 1] = x.y;
          v[4 * u + 2] = x.z;
          v[4 * u + 3] = x.w;
        }
        ptx::tmem_st32(tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + (c ? C::TM_Q1 : C::TM_Q0) +
                           chunk * 32,
                       v);
        ptx::tmem_wait_st();
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        ptx::mbar_arrive(bar(C::B_QTFULL + c));
        ptx::mbar_arrive(bar(C::B_QEMPTY));
      }
      ++cq;
      return true;
    };
    bool ok = true;
    int n_raw = raw_count<SPARSE>(a, blockIdx.x), n_raw_next = 0;
    for (int w = blockIdx.x; ok && w < n_items; w += gridDim.x, n_raw = n_raw_next) {
      n_raw_next = raw_count<SPARSE>(a, w + gridDim.x);
      const int h = w / a.nqb, qi = w - h * a.nqb;
      const ItemList<SPARSE> it = item_list<SPARSE>(a, w, n_raw);
      const int grow = qi * a.bq + r;
      const bool row_valid = (r < a.bq) && (grow < a.L);
      // my contiguous half row of O: D/2 bf16 = D bytes
      uint4* o_dst = reinterpret_cast<uint4*>(a.o + (static_cast<long>(h) * a.L + grow) * D) + half * (D / 16);
      if (it.n == 0) {
        if (row_valid) {
#pragma unroll
          for (int c = 0; c < D / 16; ++c) o_dst[c] = make_uint4(0, 0, 0, 0);
          if (half == 0) a.lse[static_cast<long>(h) * a.L + grow] = -__int_as_float(0x7f800000);
        }
        continue;
      }
      // this item's Q, unless it was copied ahead at the end of the previous one
      if (cq == iq && !copy_q()) {
        ok = false;
        break;
      }
      float m = -__int_as_float(0x7f800000);  // running row max, log2 units (scaled)
      float l = 0.f;                          // running sum of my half row
      // only a list that can hold the ragged last key block needs its entries
      // here; they are read one tile ahead, off the critical path
      const bool ragged = SPARSE && (a.Lk % BK) != 0;
      int blk_next = ragged ? it.block(0) : 0;
      for (int jj = 0; jj < it.n; ++jj, ++g) {
        int blk = jj;
        if (ragged) {
          blk = blk_next;
          if (jj + 1 < it.n) blk_next = it.block(jj + 1);
        }
        const int b = g & 1;
        if (!ptx::mbar_wait_warp(bar(C::B_SFULL + b), (g >> 1) & 1, abort_flag, a.timeout_ns, kErrTimeout)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        float s[HALF];
        {
          uint32_t raw[HALF / 32][32];
#pragma unroll
          for (int c = 0; c < HALF / 32; ++c)
            ptx::tmem_ld16x2_32<HALF>(lane_base + (b ? C::TM_S1 : C::TM_S0) + c * 32, raw[c]);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < HALF / 32; ++c) {
            ptx::reg_fence32(raw[c]);
#pragma unroll
            for (int e = 0; e < 32; ++e) s[c * 32 + e] = __uint_as_float(raw[c][e]);
          }
        }
        // ragged last key block: keys past L do not exist
        const int valid = a.Lk - blk * BK - s_off;
        if (valid < HALF) {
#pragma unroll
          for (int c = 0; c < HALF; ++c)
            if (c >= valid) s[c] = -__int_as_float(0x7f800000);
        }
        float mx0 = s[0], mx1 = s[1];
#pragma unroll
        for (int c = 2; c < HALF; c += 4) {
          mx0 = ptx::max3(mx0, s[c], s[c + 1]);
          if (c + 3 < HALF) mx1 = ptx::max3(mx1, s[c + 2], s[c + 3]);
        }
        float mx = fmaxf(mx0, mx1);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));  // the other half of my row
        const float m_new = fmaxf(m, mx * sl2);
        if (jj == 0) {
          m = m_new;
        } else if (__any_sync(0xffffffffu, m_new > m + 8.0f)) {
          // O holds this item's tiles before g-1 plus PV(g-1): wait for it,
          // rescale my half
          if (!ptx::mbar_wait_warp(bar(C::B_PVDONE + ((g - 1) & 1)), ((g - 1) >> 1) & 1, abort_flag,
                                   a.timeout_ns, kErrTimeout)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const float alpha = ptx::ex2(m - m_new);
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            uint32_t raw[32];
            ptx::tmem_ld16x2_32<D / 2>(lane_base + C::TM_O + c * 32, raw);
            ptx::tmem_wait_ld();
            ptx::reg_fence32(raw);
#pragma unroll
            for (int e = 0; e < 32; ++e) raw[e] = __float_as_uint(__uint_as_float(raw[e]) * alpha);
            ptx::tmem_st16x2_32<D / 2>(lane_base + C::TM_O + c * 32, raw);
          }
          ptx::tmem_wait_st();
          l *= alpha;
          m = m_new;
        }
        // P_b(g) over S_b(g), read out above; PV(g-2), the last reader of
        // P_b(g-2), completed before S_b(g) was issued
        const float ps = softmax_half_exp<HALF>(s, sl2, m, lane_base + (b ? C::TM_S1 : C::TM_S0));
        l += ps;
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar(C::B_PFULL + b));
      }
      if (!ok) break;
      ++iq;
      // the next item's Q into TMEM now, so its S MMAs can start during this
      // item's epilogue (the next item with work, if it is the next one)
      const int w_next = w + static_cast<int>(gridDim.x);
      if (w_next < n_items && item_list<SPARSE>(a, w_next, n_raw_next).n > 0 && !copy_q()) {
        ok = false;
        break;
      }
      // ---- epilogue: every PV of the item is done -> O / l -> bf16 -> global; LSE
      if (!ptx::mbar_wait_warp(bar(C::B_PVDONE + ((g - 1) & 1)), ((g - 1) >> 1) & 1, abort_flag, a.timeout_ns,
                               kErrTimeout)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const float lt = l + __shfl_xor_sync(0xffffffffu, l, 16);
      const float inv_l = 1.0f / lt;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t raw[32];
        ptx::tmem_ld16x2_32<D / 2>(lane_base + C::TM_O + c * 32, raw);
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
      if (row_valid && half == 0)
        a.lse[static_cast<long>(h) * a.L + grow] = (m + ptx::lg2(lt)) * 0.69314718055994530942f;
      // the next item's first PV overwrites O only after this warp's next
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
