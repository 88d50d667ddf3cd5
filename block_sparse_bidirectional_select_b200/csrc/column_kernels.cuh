// Column-sparse attention (PulseCol abstract: column-level instead of
// block-level sparsity; the pattern is identified at an early denoising step
// and reused, refreshed at a few intermediate steps).
//
// A column pattern keeps, per head h, the kc key positions ("columns" of the
// attention map) that receive the most full-attention probability mass; every
// query of the head attends to exactly those keys. The path is
//
//   column_mass_kernel    A[h,c] = sum over all rows r of exp(scale*<q_r,k_c> - LSE_r)
//                         recomputes S^T = K Q^T on tcgen05 (keys as the M
//                         dimension, so each TMEM lane is one key and its sum
//                         over queries is a per-thread accumulation in a fixed
//                         order: bit-reproducible)
//   topk_columns_kernel   per head: the kc largest masses, ties to the lower
//                         column, emitted in ascending column order (radix
//                         select on the fp32 bit patterns, then an in-order
//                         compaction)
//   gather_rows_kernel    K_sel[h,t,:] = K[h,cols[h,t],:] and the same for V
//
// after which the attention over the kept columns is the dense attention
// kernel with kc keys (all query blocks share the head's columns).
#pragma once

#include "ptx_sm100.cuh"

namespace sparsed {

struct ColMassArgs {
  int H, L, Lk;
  float scale_log2;
  const float* lse;  // [H, L]
  float* mass;       // [H, Lk]
  uint64_t timeout_ns;
};

template <int D>
struct ColMassCfg {
  static constexpr int M = 128;  // keys per CTA (TMEM lanes)
  static constexpr int N = 128;  // queries per tile
  static constexpr int STAGES = 3;
  static constexpr int DCH = D / 64;
  static constexpr int CHUNK = 128 * 128;  // one 64-column chunk of a 128-row tile
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_Q = TILE_BYTES;
  static constexpr int G = 4;             // column groups of reducer warps
  static constexpr int CW = N / G;        // query columns per group and tile
  static constexpr int RWARPS = 4 * G;    // reducer warps (4 + w)
  static constexpr int REDUCERS = 32 * RWARPS;
  static constexpr int OFF_LSE = OFF_Q + STAGES * TILE_BYTES;  // float2 [RWARPS][2][CW/2]: -LSE (log2 units)
  static constexpr int OFF_TOT = OFF_LSE + RWARPS * CW * 8;    // float [G-1][128]: groups 1.. sums
  static constexpr int OFF_BAR = OFF_TOT + (G - 1) * 128 * 4;
  static constexpr int B_KFULL = 0;
  static constexpr int B_QFULL = 1;
  static constexpr int B_QEMPTY = B_QFULL + STAGES;
  static constexpr int B_SFULL = B_QEMPTY + STAGES;  // [2]
  static constexpr int B_SFREE = B_SFULL + 2;        // [2] one arrival per reducer thread
  static constexpr int B_DRAIN = B_SFREE + 2;
  static constexpr int NUM_BARS = B_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;  // tmem slot, abort flag
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int TM_S0 = 0;
  static constexpr int TM_S1 = N;
  static constexpr int TM_ALLOC = 256;
  static constexpr uint32_t IDESC = ptx::idesc_bf16_f32(M, N, 0, 0);
  static constexpr int THREADS = 128 + REDUCERS;
  static_assert(CW % 32 == 0, "whole 32-column TMEM loads per group");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// Grid (ceil(Lk/128), H), 128 + 32 * 4G threads: warp 0 loads K once and streams the
// query tiles, warp 1 owns TMEM and issues S^T_i = K_j Q_i^T (double-buffered),
// warps 4 .. 4 + 4G - 1 reduce. A reducer thread is a key row (its TMEM lane,
// warp % 4 the lane quarter); group g (warps 4 + 4g .. 4 + 4g + 3) takes query
// columns g*CW .. g*CW + CW - 1 of every tile, so G warps per SM
// sub-partition keep the exponentials coming. Each thread sums its columns in
// a fixed order (two packed fp32x2 accumulators, then one running total per
// group), and the groups' totals are added in a fixed order at the end:
// bit-reproducible. Each reducer warp stages the -LSE of its CW query columns
// in its own
// double-buffered shared-memory slice, loaded one tile ahead, so the warps
// synchronise only through the S buffers' mbarriers.
template <int D>
__global__ void __launch_bounds__(ColMassCfg<D>::THREADS, 1)
    column_mass_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const ColMassArgs a) {
  using C = ColMassCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sb = ptx::smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int kj = blockIdx.x;
  const int h = blockIdx.y;
  const int n = (a.L + C::N - 1) / C::N;  // query tiles
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  auto bar = [&](int idx) -> uint32_t { return sb + C::OFF_BAR + 8 * idx; };

  if (threadIdx.x == 0) {
    ptx::mbar_init(bar(C::B_KFULL), 1);
    for (int s = 0; s < C::STAGES; ++s) {
      ptx::mbar_init(bar(C::B_QFULL + s), 1);
      ptx::mbar_init(bar(C::B_QEMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(bar(C::B_SFULL + b), 1);
      ptx::mbar_init(bar(C::B_SFREE + b), C::REDUCERS);
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

  if (warp == 0 && lane == 0) {
    // ================================================================ producer
    ptx::mbar_arrive_expect_tx(bar(C::B_KFULL), C::TILE_BYTES);
#pragma unroll
    for (int c = 0; c < C::DCH; ++c)
      ptx::tma_load_3d(sb + C::OFF_K + c * C::CHUNK, &tm_k, bar(C::B_KFULL), c * 64, kj * C::M, h);
    int issued = 0;
    for (int i = 0; i < n; ++i) {
      const int s = i % C::STAGES;
      if (i >= C::STAGES &&
          !ptx::mbar_wait(bar(C::B_QEMPTY + s), (i / C::STAGES - 1) & 1, abort_flag, a.timeout_ns, kErrTimeout))
        break;
      ptx::mbar_arrive_expect_tx(bar(C::B_QFULL + s), C::TILE_BYTES);
#pragma unroll
      for (int c = 0; c < C::DCH; ++c)
        ptx::tma_load_3d(sb + C::OFF_Q + s * C::TILE_BYTES + c * C::CHUNK, &tm_q, bar(C::B_QFULL + s), c * 64,
                         i * C::N, h);
      ++issued;
    }
    if (*abort_flag) {
      // let the copies in flight land before the CTA's shared memory goes away
      const uint64_t short_ns = a.timeout_ns / 4;
      volatile int dummy = 0;
      ptx::mbar_wait(bar(C::B_KFULL), 0, &dummy, short_ns, 0);
      for (int t = (issued > C::STAGES ? issued - C::STAGES : 0); t < issued; ++t)
        ptx::mbar_wait(bar(C::B_QFULL + t % C::STAGES), (t / C::STAGES) & 1, &dummy, short_ns, 0);
    }
  } else if (warp == 1 && lane == 0) {
    // ================================================================ MMA issuer
    constexpr uint32_t HI = ptx::sdesc_sw128_hi(1024);
    const uint32_t klo = ptx::sdesc_sw128_lo(sb + C::OFF_K, 16);
    const uint32_t qlo = ptx::sdesc_sw128_lo(sb + C::OFF_Q, 16);
    bool ok = ptx::mbar_wait(bar(C::B_KFULL), 0, abort_flag, a.timeout_ns, kErrTimeout);
    for (int i = 0; ok && i < n; ++i) {
      const int s = i % C::STAGES;
      const int b = i & 1;
      if (!ptx::mbar_wait(bar(C::B_QFULL + s), (i / C::STAGES) & 1, abort_flag, a.timeout_ns, kErrTimeout) ||
          (i >= 2 &&
           !ptx::mbar_wait(bar(C::B_SFREE + b), ((i - 2) >> 1) & 1, abort_flag, a.timeout_ns, kErrTimeout))) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const uint32_t b0 = qlo + static_cast<uint32_t>(s * C::TILE_BYTES >> 4);
      const uint32_t s_tmem = tmem + (b ? C::TM_S1 : C::TM_S0);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * (C::CHUNK >> 4) + (kk & 3) * 2;
        ptx::umma_ss_lohi(s_tmem, klo + off, b0 + off, HI, C::IDESC, kk > 0 ? 1u : 0u);
      }
      ptx::umma_commit(bar(C::B_SFULL + b));
      ptx::umma_commit(bar(C::B_QEMPTY + s));
    }
    if (!ok) {
      ptx::umma_commit(bar(C::B_DRAIN));
      volatile int dummy = 0;
      ptx::mbar_wait(bar(C::B_DRAIN), 0, &dummy, a.timeout_ns / 4, 0);
    }
  } else if (warp >= 4) {
    // ================================================================ reducers
    const int g = (warp - 4) >> 2;  // column group
    const int wq = warp & 3;
    const int r = wq * 32 + lane;   // key row of this CTA == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const uint64_t sl2 = ptx::f32x2(a.scale_log2, a.scale_log2);
    const float* lse_h = a.lse + static_cast<long>(h) * a.L;
    float* tot = reinterpret_cast<float*>(smem + C::OFF_TOT);
    const float kNegInf = -__int_as_float(0x7f800000);
    // -LSE (log2 units) of this warp's query columns 2*lane, 2*lane + 1 of
    // tile i (lanes below CW/2); queries past L weigh nothing
    auto neg_lse2_of = [&](int i) -> float2 {
      const int q = i * C::N + g * C::CW + 2 * lane;
      float2 v;
      v.x = q < a.L ? lse_h[q] * -1.44269504088896340736f : kNegInf;
      v.y = q + 1 < a.L ? lse_h[q + 1] * -1.44269504088896340736f : kNegInf;
      return v;
    };
    float2* wl = reinterpret_cast<float2*>(smem + C::OFF_LSE) + (warp - 4) * C::CW;  // [2][CW/2] float2
    constexpr int HW = C::CW / 2;
    float2 nxt = lane < HW ? neg_lse2_of(0) : float2{};
    float total = 0.f;
    for (int i = 0; i < n; ++i) {
      const int b = i & 1;
      // buffer b was last read at tile i - 2, before the __syncwarp of tile i - 1
      if (lane < HW) wl[b * HW + lane] = nxt;
      __syncwarp();
      if (i + 1 < n && lane < HW) nxt = neg_lse2_of(i + 1);
      const bool ok =
          ptx::mbar_wait_warp(bar(C::B_SFULL + b), (i >> 1) & 1, abort_flag, a.timeout_ns, kErrTimeout);
      if (!ok) continue;
      ptx::tc_fence_after();
      constexpr int NC = C::CW / 32;
      uint32_t raw[NC][32];
      const uint32_t col0 = (b ? C::TM_S1 : C::TM_S0) + g * C::CW;
#pragma unroll
      for (int c = 0; c < NC; ++c) ptx::tmem_ld32(lane_base + col0 + c * 32, raw[c]);
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
      ptx::mbar_arrive(bar(C::B_SFREE + b));  // S_b is in registers: the MMA may overwrite it
      const float2* nl = wl + b * HW;
      uint64_t acc0 = ptx::f32x2(0.f, 0.f), acc1 = acc0;
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        ptx::reg_fence32(raw[c]);
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float2 l2 = nl[(c * 32 + e) >> 1];
          float x0, x1;
          ptx::f32x2_split(ptx::fma_f32x2(ptx::f32x2(__uint_as_float(raw[c][e]), __uint_as_float(raw[c][e + 1])),
                                          sl2, ptx::f32x2(l2.x, l2.y)),
                           x0, x1);
          const uint64_t p2 = ptx::f32x2(ptx::ex2(x0), ptx::ex2(x1));
          if (e & 2)
            acc1 = ptx::add_f32x2(acc1, p2);
          else
            acc0 = ptx::add_f32x2(acc0, p2);
        }
      }
      float a0, a1, b0, b1;
      ptx::f32x2_split(acc0, a0, a1);
      ptx::f32x2_split(acc1, b0, b1);
      total += (a0 + b0) + (a1 + b1);
    }
    // the groups' sums of every key row, added in a fixed order
    if (g > 0) tot[(g - 1) * 128 + r] = total;
    ptx::named_bar_sync(2, C::REDUCERS);
    const int key = kj * C::M + r;
    if (g == 0 && key < a.Lk && !*abort_flag) {
#pragma unroll
      for (int q = 1; q < C::G; ++q) total += tot[(q - 1) * 128 + r];
      a.mass[static_cast<long>(h) * a.Lk + key] = total;
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::TM_ALLOC);
  }
}

// ---------------------------------------------------------------- top-k columns

// One CTA of 1024 threads per head. Masses are >= 0, so their fp32 bit
// patterns order like their values: four 8-bit radix passes (most significant
// first) find T, the bit pattern of the kc-th largest mass, and how many of the
// masses equal to T are kept (the lowest columns first). A pass in column
// order then writes every column above T and those first ties, ascending.
__global__ void __launch_bounds__(1024)
    topk_columns_kernel(const float* __restrict__ mass, int Lk, int kc, int32_t* __restrict__ cols,
                        int col_stride) {
  __shared__ unsigned hist[256];
  __shared__ unsigned s_prefix, s_need;
  __shared__ int w_gt[32], w_eq[32], w_take[32];
  const int h = blockIdx.x;
  const int tid = threadIdx.x;
  const int lane = tid & 31, wid = tid >> 5;
  const uint32_t* m = reinterpret_cast<const uint32_t*>(mass + static_cast<long>(h) * Lk);
  int32_t* out = cols + static_cast<long>(h) * col_stride;
  uint32_t prefix = 0, pmask = 0;
  unsigned need = static_cast<unsigned>(kc);
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int t = tid; t < 256; t += blockDim.x) hist[t] = 0;
    __syncthreads();
    for (int i = tid; i < Lk; i += blockDim.x) {
      const uint32_t u = m[i];
      if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid == 0) {
      unsigned acc = 0;
      int sel = 0;
      for (int bkt = 255; bkt >= 0; --bkt) {
        if (acc + hist[bkt] >= need) {
          sel = bkt;
          break;
        }
        acc += hist[bkt];
      }
      s_prefix = prefix | (static_cast<uint32_t>(sel) << shift);
      s_need = need - acc;
    }
    __syncthreads();
    prefix = s_prefix;
    need = s_need;
    pmask |= 0xFFu << shift;
  }
  const uint32_t T = prefix;
  const unsigned lt_mask = (1u << lane) - 1u;
  int base = 0, eq_seen = 0;
  for (int c0 = 0; c0 < Lk; c0 += blockDim.x) {
    const int i = c0 + tid;
    const bool valid = i < Lk;
    const uint32_t u = valid ? m[i] : 0u;
    const bool gt = valid && u > T;
    const bool eq = valid && u == T;
    const unsigned b_gt = __ballot_sync(0xffffffffu, gt);
    const unsigned b_eq = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) {
      w_gt[wid] = __popc(b_gt);
      w_eq[wid] = __popc(b_eq);
    }
    __syncthreads();
    int gt_before = 0, eq_before = 0, gt_all = 0, eq_all = 0;
    for (int w = 0; w < 32; ++w) {
      if (w < wid) {
        gt_before += w_gt[w];
        eq_before += w_eq[w];
      }
      gt_all += w_gt[w];
      eq_all += w_eq[w];
    }
    // ties are taken in column order: my rank among the ties seen so far
    const int eq_rank = eq_seen + eq_before + __popc(b_eq & lt_mask);
    const bool take_eq = eq && eq_rank < static_cast<int>(need);
    const unsigned b_take = __ballot_sync(0xffffffffu, take_eq);
    // columns kept before mine in this chunk: all gt ones and the taken ties
    // of the lower warps, plus those of my warp below me
    if (lane == 0) w_take[wid] = __popc(b_take);
    __syncthreads();
    int take_before = 0, take_all = 0;
    for (int w = 0; w < 32; ++w) {
      if (w < wid) take_before += w_take[w];
      take_all += w_take[w];
    }
    if (gt || take_eq)
      out[base + gt_before + take_before + __popc((b_gt | b_take) & lt_mask)] = i;
    base += gt_all + take_all;
    eq_seen += eq_all;
    __syncthreads();
  }
}

// ---------------------------------------------------------------- gather

// K_sel[h,t,:] = K[h,cols[h,t],:] and V_sel likewise, 16 bytes per thread.
// The column list must be strictly ascending and inside [0, L): a bad entry is
// reported (kErrBadPattern) and reads row 0 instead.
__global__ void __launch_bounds__(256)
    gather_rows_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v, const int32_t* __restrict__ cols,
                       int L, int kc, int col_stride, int row_u4, uint4* __restrict__ k_sel,
                       uint4* __restrict__ v_sel) {
  const int h = blockIdx.y;
  const long e = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;  // element within the head
  if (e >= static_cast<long>(kc) * row_u4) return;
  const int t = static_cast<int>(e / row_u4);
  const int u = static_cast<int>(e - static_cast<long>(t) * row_u4);
  const int32_t* lst = cols + static_cast<long>(h) * col_stride;
  int c = lst[t];
  if (u == 0 && (c < 0 || c >= L || (t > 0 && c <= lst[t - 1]))) ptx::record_error(kErrBadPattern);
  if (c < 0 || c >= L) c = 0;
  const long src = (static_cast<long>(h) * L + c) * row_u4 + u;
  const long dst = (static_cast<long>(h) * kc + t) * row_u4 + u;
  k_sel[dst] = k[src];
  v_sel[dst] = v[src];
}

}  // namespace sparsed
