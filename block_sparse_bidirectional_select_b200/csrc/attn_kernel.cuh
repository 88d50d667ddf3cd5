// Flash-style bidirectional attention for sm_100a, dense or block-sparse.
//
// One CTA computes one (head h, query block i) output tile of up to 128 rows:
//   O = softmax(scale * Q_i K^T) V  over the key blocks of its list, plus the
//   fp32 natural-log LSE of every row.
// Dense mode walks key blocks 0..nkb-1 (SparseD abstract: full attention in
// the early denoising steps; Step-dLLM abstract: the full map is recomputed at
// every step). Sparse mode walks kv_idx[h,i,0..kv_count) (Step-dLLM abstract:
// block-sparse attention over a reused mask). Both modes share every line of
// the arithmetic, so a sparse call that keeps every block in ascending order is
// bitwise equal to the dense call.
//
// Warp roles (256 threads):
//   warp 0       TMA producer: Q tile once, then K_j and V_j tiles into a
//                STAGES-deep ring (128B-swizzled boxes of 64 columns).
//   warp 1       tcgen05 issuer (one thread) and TMEM owner:
//                  S_b = Q K_j^T   (SS MMA, M=128, N=BK, K=D, fp32 in TMEM)
//                  O  += P_b V_j   (TS MMA, P from TMEM, V MN-major, N=D)
//   warps 4..7   softmax warpgroup, thread r owns row r (TMEM lane r):
//                reads S_b, running max (log2 domain), exp2, row sum, writes
//                P_b = bf16(exp2(s*scale*log2e - m)) back into TMEM, rescales
//                O in TMEM only when the running max grew by more than 2^8
//                (the stale max is exact: O and l share it), epilogue O/l ->
//                bf16 -> swizzled smem -> TMA store, LSE = (m + log2 l) ln 2.
// S and P are double-buffered in TMEM so the MMA of tile j+1 runs while the
// softmax of tile j does, and PV of tile j overlaps the softmax of tile j+1.
#pragma once

#include "ptx_sm100.cuh"

namespace sparsed {

struct AttnArgs {
  int H, L, bq, nqb, nkb;
  float scale_log2;          // scale * log2(e)
  const int32_t* kv_idx;     // sparse mode only
  const int32_t* kv_count;   // sparse mode only
  int kv_stride;
  float* lse;                // [H, L]
  uint16_t* o;               // [H, L, D] (used only for kv_count == 0 rows)
  uint64_t timeout_ns;       // bound of every device-side wait
};

template <int D, int BK>
struct AttnCfg {
  static constexpr int M = 128;
  static constexpr int STAGES = 2;
  static constexpr int DCH = D / 64;             // 64-column chunks of the head dim
  static constexpr int Q_CHUNK = M * 128;        // bytes of one chunk of the Q tile
  static constexpr int KV_CHUNK = BK * 128;      // bytes of one chunk of a K/V tile
  static constexpr int Q_BYTES = M * D * 2;
  static constexpr int KV_BYTES = BK * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + STAGES * KV_BYTES;
  // barrier indices
  static constexpr int B_QFULL = 0;
  static constexpr int B_KFULL = 1;
  static constexpr int B_KEMPTY = B_KFULL + STAGES;
  static constexpr int B_VFULL = B_KEMPTY + STAGES;
  static constexpr int B_VEMPTY = B_VFULL + STAGES;
  static constexpr int B_SFULL = B_VEMPTY + STAGES;
  static constexpr int B_SFREE = B_SFULL + 2;
  static constexpr int B_PFULL = B_SFREE + 2;
  static constexpr int B_PVDONE = B_PFULL + 2;
  static constexpr int B_DRAIN = B_PVDONE + 2;
  static constexpr int NUM_BARS = B_DRAIN + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;  // tmem slot, abort flag
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
  // TMEM columns
  static constexpr int TM_S0 = 0;
  static constexpr int TM_S1 = BK;
  static constexpr int TM_O = 2 * BK;
  static constexpr int TM_P0 = 2 * BK + D;
  static constexpr int TM_P1 = TM_P0 + BK / 2;
  static constexpr int TM_USED = TM_P1 + BK / 2;
  static constexpr int TM_ALLOC = TM_USED <= 256 ? 256 : 512;
  static constexpr uint32_t IDESC_S = ptx::idesc_bf16_f32(128, BK, 0, 0);
  static constexpr uint32_t IDESC_PV = ptx::idesc_bf16_f32(128, D, 0, 1);
  static_assert(TM_USED <= 512, "TMEM budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

constexpr int kErrBadPattern = -4;
constexpr int kErrTimeout = -6;

template <int D, int BK, bool SPARSE>
__global__ void __launch_bounds__(256, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                    const AttnArgs a) {
  using C = AttnCfg<D, BK>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sb = ptx::smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qi = blockIdx.x;
  const int h = blockIdx.y;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  auto bar = [&](int idx) -> uint32_t { return sb + C::OFF_BAR + 8 * idx; };

  // ---- work list of this tile
  int n = a.nkb;
  const int32_t* list = nullptr;
  if constexpr (SPARSE) {
    const long row = static_cast<long>(h) * a.nqb + qi;
    n = a.kv_count[row];
    const int cap = a.kv_stride < a.nkb ? a.kv_stride : a.nkb;
    if (n < 0 || n > cap) {
      if (threadIdx.x == 0) ptx::record_error(kErrBadPattern);
      n = n < 0 ? 0 : cap;
    }
    list = a.kv_idx + row * a.kv_stride;
  }
  auto kv_block = [&](int jj) -> int {
    if constexpr (SPARSE) {
      const int j = list[jj];
      return (j >= 0 && j < a.nkb) ? j : 0;
    } else {
      return jj;
    }
  };

  // ---- setup
  if (threadIdx.x == 0) {
    ptx::mbar_init(bar(C::B_QFULL), 1);
    for (int s = 0; s < C::STAGES; ++s) {
      ptx::mbar_init(bar(C::B_KFULL + s), 1);
      ptx::mbar_init(bar(C::B_KEMPTY + s), 1);
      ptx::mbar_init(bar(C::B_VFULL + s), 1);
      ptx::mbar_init(bar(C::B_VEMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(bar(C::B_SFULL + b), 1);
      ptx::mbar_init(bar(C::B_SFREE + b), 128);
      ptx::mbar_init(bar(C::B_PFULL + b), 128);
      ptx::mbar_init(bar(C::B_PVDONE + b), 1);
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

  if (warp == 0 && lane == 0 && n > 0) {
    // ================================================================ producer
    ptx::tma_prefetch_desc(&tm_q);
    ptx::tma_prefetch_desc(&tm_k);
    ptx::tma_prefetch_desc(&tm_v);
    ptx::mbar_arrive_expect_tx(bar(C::B_QFULL), C::Q_BYTES);
#pragma unroll
    for (int c = 0; c < C::DCH; ++c)
      ptx::tma_load_3d(sb + C::OFF_Q + c * C::Q_CHUNK, &tm_q, bar(C::B_QFULL), c * 64, qi * a.bq, h);
    int prev = -1;
    int issued_k = 0, issued_v = 0;
    for (int jj = 0; jj < n; ++jj) {
      const int s = jj % C::STAGES;
      const uint32_t use = static_cast<uint32_t>(jj / C::STAGES);
      if (jj >= C::STAGES &&
          !ptx::mbar_wait(bar(C::B_KEMPTY + s), (use - 1) & 1, abort_flag, a.timeout_ns, kErrTimeout))
        break;
      int j = jj;
      if constexpr (SPARSE) {
        j = list[jj];
        if (j < 0 || j >= a.nkb || j <= prev) ptx::record_error(kErrBadPattern);
        prev = j;
        j = kv_block(jj);
      }
      ptx::mbar_arrive_expect_tx(bar(C::B_KFULL + s), C::KV_BYTES);
#pragma unroll
      for (int c = 0; c < C::DCH; ++c)
        ptx::tma_load_3d(sb + C::OFF_K + s * C::KV_BYTES + c * C::KV_CHUNK, &tm_k, bar(C::B_KFULL + s),
                         c * 64, j * BK, h);
      ++issued_k;
      if (jj >= C::STAGES &&
          !ptx::mbar_wait(bar(C::B_VEMPTY + s), (use - 1) & 1, abort_flag, a.timeout_ns, kErrTimeout))
        break;
      ptx::mbar_arrive_expect_tx(bar(C::B_VFULL + s), C::KV_BYTES);
#pragma unroll
      for (int c = 0; c < C::DCH; ++c)
        ptx::tma_load_3d(sb + C::OFF_V + s * C::KV_BYTES + c * C::KV_CHUNK, &tm_v, bar(C::B_VFULL + s),
                         c * 64, j * BK, h);
      ++issued_v;
    }
    if (*abort_flag) {
      // let every copy already in flight land before the CTA's smem goes away
      const uint64_t short_ns = a.timeout_ns / 4;
      for (int t = (issued_k > C::STAGES ? issued_k - C::STAGES : 0); t < issued_k; ++t) {
        volatile int dummy = 0;
        ptx::mbar_wait(bar(C::B_KFULL + t % C::STAGES), (t / C::STAGES) & 1, &dummy, short_ns, 0);
      }
      for (int t = (issued_v > C::STAGES ? issued_v - C::STAGES : 0); t < issued_v; ++t) {
        volatile int dummy = 0;
        ptx::mbar_wait(bar(C::B_VFULL + t % C::STAGES), (t / C::STAGES) & 1, &dummy, short_ns, 0);
      }
    }
  } else if (warp == 1 && lane == 0 && n > 0) {
    // ================================================================ MMA issuer
    bool ok = ptx::mbar_wait(bar(C::B_QFULL), 0, abort_flag, a.timeout_ns, kErrTimeout);
    ptx::tc_fence_after();
    auto issue_pv = [&](int t) -> bool {
      const int b = t & 1;
      const int s = t % C::STAGES;
      if (!ptx::mbar_wait(bar(C::B_PFULL + b), (t >> 1) & 1, abort_flag, a.timeout_ns, kErrTimeout))
        return false;
      if (!ptx::mbar_wait(bar(C::B_VFULL + s), (t / C::STAGES) & 1, abort_flag, a.timeout_ns,
                          kErrTimeout))
        return false;
      ptx::tc_fence_after();
      const uint32_t p_tmem = tmem + (b ? C::TM_P1 : C::TM_P0);
      const uint32_t v_base = sb + C::OFF_V + s * C::KV_BYTES;
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk) {
        const uint64_t bdesc = ptx::sdesc_sw128(v_base + kk * 2048, C::KV_CHUNK, 1024);
        ptx::umma_ts(tmem + C::TM_O, p_tmem + kk * 8, bdesc, C::IDESC_PV, (t > 0 || kk > 0) ? 1u : 0u);
      }
      ptx::umma_commit(bar(C::B_VEMPTY + s));
      ptx::umma_commit(bar(C::B_PVDONE + b));
      return true;
    };
    for (int jj = 0; ok && jj < n; ++jj) {
      const int s = jj % C::STAGES;
      const int b = jj & 1;
      if (!ptx::mbar_wait(bar(C::B_KFULL + s), (jj / C::STAGES) & 1, abort_flag, a.timeout_ns,
                          kErrTimeout)) {
        ok = false;
        break;
      }
      if (jj >= 2 &&
          !ptx::mbar_wait(bar(C::B_SFREE + b), ((jj - 2) >> 1) & 1, abort_flag, a.timeout_ns,
                          kErrTimeout)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const uint32_t s_tmem = tmem + (b ? C::TM_S1 : C::TM_S0);
      const uint32_t k_base = sb + C::OFF_K + s * C::KV_BYTES;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk & 3) * 32;  // 16 bf16 = 32 bytes inside the swizzle atom
        const uint64_t adesc = ptx::sdesc_sw128(sb + C::OFF_Q + (kk >> 2) * C::Q_CHUNK + off, 16, 1024);
        const uint64_t bdesc = ptx::sdesc_sw128(k_base + (kk >> 2) * C::KV_CHUNK + off, 16, 1024);
        ptx::umma_ss(s_tmem, adesc, bdesc, C::IDESC_S, kk > 0 ? 1u : 0u);
      }
      ptx::umma_commit(bar(C::B_SFULL + b));
      ptx::umma_commit(bar(C::B_KEMPTY + s));
      if (jj >= 1 && !issue_pv(jj - 1)) {
        ok = false;
        break;
      }
    }
    if (ok) ok = issue_pv(n - 1);
    if (!ok) {
      // drain: wait until every MMA this thread issued has completed
      ptx::umma_commit(bar(C::B_DRAIN));
      volatile int dummy = 0;
      ptx::mbar_wait(bar(C::B_DRAIN), 0, &dummy, a.timeout_ns / 4, 0);
    }
  } else if (warp >= 4) {
    // ================================================================ softmax
    const int wq = warp & 3;
    const int r = wq * 32 + lane;  // row within the tile == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const int grow = qi * a.bq + r;  // row within the head
    const bool row_valid = (r < a.bq) && (grow < a.L);
    const float sl2 = a.scale_log2;
    if (n == 0) {
      if (row_valid) {
        uint4* dst = reinterpret_cast<uint4*>(a.o + (static_cast<long>(h) * a.L + grow) * D);
#pragma unroll
        for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
        a.lse[static_cast<long>(h) * a.L + grow] = -__int_as_float(0x7f800000);
      }
    } else {
      float m = -__int_as_float(0x7f800000);  // running max, log2 units (scaled)
      float l = 0.f;
      bool ok = true;
      for (int jj = 0; jj < n; ++jj) {
        const int b = jj & 1;
        if (!ptx::mbar_wait_warp(bar(C::B_SFULL + b), (jj >> 1) & 1, abort_flag, a.timeout_ns,
                                 kErrTimeout)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        float s[BK];
#pragma unroll
        for (int c = 0; c < BK / 32; ++c) {
          uint32_t raw[32];
          ptx::tmem_ld32(lane_base + (b ? C::TM_S1 : C::TM_S0) + c * 32, raw);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) s[c * 32 + e] = __uint_as_float(raw[e]);
        }
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar(C::B_SFREE + b));
        // ragged last key block: keys past L do not exist
        const int j = kv_block(jj);
        const int valid = a.L - j * BK;
        if (valid < BK) {
#pragma unroll
          for (int c = 0; c < BK; ++c)
            if (c >= valid) s[c] = -__int_as_float(0x7f800000);
        }
        float mx = s[0];
#pragma unroll
        for (int c = 1; c < BK; ++c) mx = fmaxf(mx, s[c]);
        const float m_new = fmaxf(m, mx * sl2);
        if (jj == 0) {
          m = m_new;
        } else {
          const bool need = m_new > m + 8.0f;
          if (__any_sync(0xffffffffu, need)) {
            // O holds tiles < jj-1 plus PV(jj-1): wait for it, then rescale in place
            if (!ptx::mbar_wait_warp(bar(C::B_PVDONE + ((jj - 1) & 1)), ((jj - 1) >> 1) & 1,
                                     abort_flag, a.timeout_ns, kErrTimeout)) {
              ok = false;
              break;
            }
            ptx::tc_fence_after();
            const float alpha = ptx::ex2(m - m_new);
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t raw[32];
              ptx::tmem_ld32(lane_base + C::TM_O + c * 32, raw);
              ptx::tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) raw[e] = __float_as_uint(__uint_as_float(raw[e]) * alpha);
              ptx::tmem_st32(lane_base + C::TM_O + c * 32, raw);
            }
            ptx::tmem_wait_st();
            l *= alpha;
            m = m_new;
          }
        }
        // P_b is free once PV(jj-2) has consumed it
        if (jj >= 2 && !ptx::mbar_wait_warp(bar(C::B_PVDONE + b), ((jj - 2) >> 1) & 1, abort_flag,
                                            a.timeout_ns, kErrTimeout)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
        for (int c = 0; c < BK / 64; ++c) {
          uint32_t pk[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float p0 = ptx::ex2(fmaf(s[c * 64 + 2 * e], sl2, -m));
            const float p1 = ptx::ex2(fmaf(s[c * 64 + 2 * e + 1], sl2, -m));
            acc0 += p0;
            acc1 += p1;
            pk[e] = ptx::pack_bf16x2(p0, p1);
          }
          ptx::tmem_st32(lane_base + (b ? C::TM_P1 : C::TM_P0) + c * 32, pk);
        }
        ptx::tmem_wait_st();
        l += acc0 + acc1;
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar(C::B_PFULL + b));
      }
      if (ok) ok = ptx::mbar_wait_warp(bar(C::B_PVDONE + ((n - 1) & 1)), ((n - 1) >> 1) & 1,
                                       abort_flag, a.timeout_ns, kErrTimeout);
      if (ok) {
        ptx::tc_fence_after();
        // ---- epilogue: O / l -> bf16 -> swizzled smem (the Q tile's bytes,
        // no longer read by any MMA) -> TMA store; LSE straight to global.
        const float inv_l = 1.0f / l;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t raw[32];
          ptx::tmem_ld32(lane_base + C::TM_O + c * 32, raw);
          ptx::tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = ptx::pack_bf16x2(__uint_as_float(raw[2 * e]) * inv_l,
                                     __uint_as_float(raw[2 * e + 1]) * inv_l);
          uint8_t* chunk = smem + C::OFF_Q + (c >> 1) * C::Q_CHUNK + r * 128;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int unit = ((c & 1) * 4 + u) ^ (r & 7);
            *reinterpret_cast<uint4*>(chunk + unit * 16) =
                make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
          }
        }
        if (row_valid)
          a.lse[static_cast<long>(h) * a.L + grow] = (m + ptx::lg2(l)) * 0.69314718055994530942f;
        ptx::fence_proxy_async_smem();
      }
      // all 128 softmax threads take this barrier on every path
      ptx::named_bar_sync(1, 128);
      if (ok && r == 0 && !*abort_flag) {
#pragma unroll
        for (int c = 0; c < C::DCH; ++c)
          ptx::tma_store_3d(&tm_o, sb + C::OFF_Q + c * C::Q_CHUNK, c * 64, qi * a.bq, h);
        ptx::bulk_commit();
        ptx::bulk_wait0();
      }
    }
  }

  // ---- teardown
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::TM_ALLOC);
  }
}

}  // namespace sparsed
