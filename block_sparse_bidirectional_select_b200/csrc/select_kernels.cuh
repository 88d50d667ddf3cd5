// Pattern selection after the full-attention pass (SparseD abstract: the
// head-specific sparse pattern is computed once from full attention; Step-dLLM
// abstract: a block-sparse mask under a uniform or head-adaptive budget).
//
//   mass_from_parts_kernel  the same M from per-warp partial sums the
//                       attention kernel's fused variant wrote in its pass
//   block_mass_kernel   M[h,i,j] = sum_{r in qblk i, c in kblk j}
//                                  exp(scale*<q_r,k_c> - LSE_r)
//                       recomputes S = Q K^T on tcgen05 (fp32 in TMEM) and
//                       reduces every 128 x BK tile to one fp32 scalar in a
//                       fixed order (bit-reproducible): BK/32 groups of four
//                       reducer warps, each warp 32 columns of every tile, its
//                       partial handed to one combining warp through shared
//                       memory (mbarriers, no barrier across the reducers).
//   row_entropy_kernel  entropy of each row M[h,i,:] / sum_j M[h,i,j] (fp64)
//   budget_kernel       per-head k_h from the mean row entropy (fp64, one thread)
//   topk_kernel         per (h,i): the k_h largest masses, ties to the lower
//                       block index, written in ascending block order.
#pragma once

#include "ptx_sm100.cuh"

namespace sparsed {

struct MassArgs {
  int H, L, bq, nqb, nkb;
  float scale_log2;
  const float* lse;   // [H, L]
  float* mass;        // [H, nqb, nkb]
  uint64_t timeout_ns;
};

template <int D, int BK>
struct MassCfg {
  static constexpr int M = 128;
  static constexpr int STAGES = 3;
  static constexpr int DCH = D / 64;
  static constexpr int Q_CHUNK = M * 128;
  static constexpr int KV_CHUNK = BK * 128;
  static constexpr int Q_BYTES = M * D * 2;
  static constexpr int K_BYTES = BK * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = Q_BYTES;
  static constexpr int OFF_BAR = OFF_K + STAGES * K_BYTES;
  static constexpr int B_QFULL = 0;
  static constexpr int B_KFULL = 1;
  static constexpr int B_KEMPTY = B_KFULL + STAGES;
  static constexpr int B_SFULL = B_KEMPTY + STAGES;
  static constexpr int B_SFREE = B_SFULL + 2;
  static constexpr int B_DRAIN = B_SFREE + 2;
  static constexpr int B_REDFULL = B_DRAIN + 1;    // [2] one arrival per reducer warp
  static constexpr int B_REDEMPTY = B_REDFULL + 2; // [2] the combining warp has read red[b]
  static constexpr int NUM_BARS = B_REDEMPTY + 2;
  static constexpr int G = BK / 32;                // reducer groups: 32 columns of every tile each
  static constexpr int RWARPS = 4 * G;             // reducer warps (warps 4 ..)
  static constexpr int THREADS = 128 + 32 * RWARPS;
  static constexpr int OFF_RED = OFF_BAR + NUM_BARS * 8;     // float red[2][RWARPS]
  static constexpr int OFF_MISC = OFF_RED + 2 * RWARPS * 4;  // tmem slot, abort flag
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int TM_S0 = 0;
  static constexpr int TM_S1 = BK;
  static constexpr int TM_ALLOC = 2 * BK <= 128 ? 128 : 256;
  static constexpr uint32_t IDESC_S = ptx::idesc_bf16_f32(128, BK, 0, 0);
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

template <int D, int BK>
__global__ void __launch_bounds__(MassCfg<D, BK>::THREADS, 1)
    block_mass_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const MassArgs a) {
  using C = MassCfg<D, BK>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sb = ptx::smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qi = blockIdx.x;
  const int h = blockIdx.y;
  const int n = a.nkb;
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);
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
      ptx::mbar_init(bar(C::B_SFREE + b), 32 * C::RWARPS);
      ptx::mbar_init(bar(C::B_REDFULL + b), C::RWARPS);
      ptx::mbar_init(bar(C::B_REDEMPTY + b), 1);
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
    ptx::mbar_arrive_expect_tx(bar(C::B_QFULL), C::Q_BYTES);
#pragma unroll
    for (int c = 0; c < C::DCH; ++c)
      ptx::tma_load_3d(sb + C::OFF_Q + c * C::Q_CHUNK, &tm_q, bar(C::B_QFULL), c * 64, qi * a.bq, h);
    int issued = 0;
    for (int j = 0; j < n; ++j) {
      const int s = j % C::STAGES;
      const uint32_t use = static_cast<uint32_t>(j / C::STAGES);
      if (j >= C::STAGES &&
          !ptx::mbar_wait(bar(C::B_KEMPTY + s), (use - 1) & 1, abort_flag, a.timeout_ns, kErrTimeout))
        break;
      ptx::mbar_arrive_expect_tx(bar(C::B_KFULL + s), C::K_BYTES);
#pragma unroll
      for (int c = 0; c < C::DCH; ++c)
        ptx::tma_load_3d(sb + C::OFF_K + s * C::K_BYTES + c * C::KV_CHUNK, &tm_k, bar(C::B_KFULL + s),
                         c * 64, j * BK, h);
      ++issued;
    }
    if (*abort_flag) {
      const uint64_t short_ns = a.timeout_ns / 4;
      for (int t = (issued > C::STAGES ? issued - C::STAGES : 0); t < issued; ++t) {
        volatile int dummy = 0;
        ptx::mbar_wait(bar(C::B_KFULL + t % C::STAGES), (t / C::STAGES) & 1, &dummy, short_ns, 0);
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ================================================================ MMA issuer
    bool ok = ptx::mbar_wait(bar(C::B_QFULL), 0, abort_flag, a.timeout_ns, kErrTimeout);
    ptx::tc_fence_after();
    for (int j = 0; ok && j < n; ++j) {
      const int s = j % C::STAGES;
      const int b = j & 1;
      if (!ptx::mbar_wait(bar(C::B_KFULL + s), (j / C::STAGES) & 1, abort_flag, a.timeout_ns,
                          kErrTimeout)) {
        ok = false;
        break;
      }
      if (j >= 2 && !ptx::mbar_wait(bar(C::B_SFREE + b), ((j - 2) >> 1) & 1, abort_flag, a.timeout_ns,
                                    kErrTimeout)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const uint32_t s_tmem = tmem + (b ? C::TM_S1 : C::TM_S0);
      const uint32_t k_base = sb + C::OFF_K + s * C::K_BYTES;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk & 3) * 32;
        const uint64_t adesc = ptx::sdesc_sw128(sb + C::OFF_Q + (kk >> 2) * C::Q_CHUNK + off, 16, 1024);
        const uint64_t bdesc = ptx::sdesc_sw128(k_base + (kk >> 2) * C::KV_CHUNK + off, 16, 1024);
        ptx::umma_ss(s_tmem, adesc, bdesc, C::IDESC_S, kk > 0 ? 1u : 0u);
      }
      ptx::umma_commit(bar(C::B_SFULL + b));
      ptx::umma_commit(bar(C::B_KEMPTY + s));
    }
    if (!ok) {
      ptx::umma_commit(bar(C::B_DRAIN));
      volatile int dummy = 0;
      ptx::mbar_wait(bar(C::B_DRAIN), 0, &dummy, a.timeout_ns / 4, 0);
    }
  } else if (warp == 2) {
    // ================================================================ combiner
    // tile j's mass: the reducer warps' partials in warp order
    float* out = a.mass + (static_cast<long>(h) * a.nqb + qi) * a.nkb;
    for (int j = 0; j < n; ++j) {
      const int b = j & 1;
      if (!ptx::mbar_wait_warp(bar(C::B_REDFULL + b), (j >> 1) & 1, abort_flag, a.timeout_ns, kErrTimeout)) break;
      if (lane == 0) {
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < C::RWARPS; ++w) t += red[b * C::RWARPS + w];
        if (!*abort_flag) out[j] = t;
        ptx::mbar_arrive(bar(C::B_REDEMPTY + b));
      }
      __syncwarp();
    }
  } else if (warp >= 4) {
    // ================================================================ reducers
    const int rw = warp - 4;    // reducer warp
    const int g = rw >> 2;      // columns 32g .. 32g + 31 of every tile
    const int wq = warp & 3;    // TMEM lane quarter
    const int r = wq * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const int grow = qi * a.bq + r;
    const bool row_valid = (r < a.bq) && (grow < a.L);
    const float nl = row_valid ? a.lse[static_cast<long>(h) * a.L + grow] * -1.44269504088896340736f : 0.f;
    const uint64_t nl2 = ptx::f32x2(nl, nl);
    const uint64_t sl2 = ptx::f32x2(a.scale_log2, a.scale_log2);
    for (int j = 0; j < n; ++j) {
      const int b = j & 1;
      if (!ptx::mbar_wait_warp(bar(C::B_SFULL + b), (j >> 1) & 1, abort_flag, a.timeout_ns, kErrTimeout)) break;
      ptx::tc_fence_after();
      uint32_t raw[32];
      ptx::tmem_ld32(lane_base + (b ? C::TM_S1 : C::TM_S0) + g * 32, raw);
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
      ptx::mbar_arrive(bar(C::B_SFREE + b));  // S_b is in registers: the MMA may overwrite it
      ptx::reg_fence32(raw);
      const int valid = (a.L - j * BK < BK ? a.L - j * BK : BK) - g * 32;  // key columns of mine below L
      uint64_t acc0 = ptx::f32x2(0.f, 0.f), acc1 = acc0;
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        float x0, x1;
        ptx::f32x2_split(ptx::fma_f32x2(ptx::f32x2(__uint_as_float(raw[e]), __uint_as_float(raw[e + 1])), sl2, nl2),
                         x0, x1);
        float p0 = ptx::ex2(x0), p1 = ptx::ex2(x1);
        if (valid < 32) {  // the ragged last key block
          p0 = e < valid ? p0 : 0.f;
          p1 = e + 1 < valid ? p1 : 0.f;
        }
        if (e & 2)
          acc1 = ptx::add_f32x2(acc1, ptx::f32x2(p0, p1));
        else
          acc0 = ptx::add_f32x2(acc0, ptx::f32x2(p0, p1));
      }
      float a0, a1, b0, b1;
      ptx::f32x2_split(acc0, a0, a1);
      ptx::f32x2_split(acc1, b0, b1);
      float acc = row_valid ? (a0 + b0) + (a1 + b1) : 0.f;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      // red[b] was last read for tile j - 2
      if (j >= 2 && !ptx::mbar_wait_warp(bar(C::B_REDEMPTY + b), ((j >> 1) - 1) & 1, abort_flag, a.timeout_ns,
                                         kErrTimeout))
        break;
      if (lane == 0) {
        red[b * C::RWARPS + rw] = acc;
        ptx::mbar_arrive(bar(C::B_REDFULL + b));
      }
      __syncwarp();
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::TM_ALLOC);
  }
}

// ---------------------------------------------------------------- fused mass

// Block mass from the partial sums the attention kernel's MASS variant wrote
// during its full pass: mass[e] = sum of the 4 softmax warps' partials of tile
// e = (h, i, j), in a fixed order.
__global__ void __launch_bounds__(256)
    mass_from_parts_kernel(const float4* __restrict__ part, long n, float* __restrict__ mass) {
  const long e = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= n) return;
  const float4 a = part[e];
  mass[e] = (a.x + a.y) + (a.z + a.w);
}

// ---------------------------------------------------------------- top-k

// One warp per (h, i) row (head_k: per-head k from the entropy budget, else
// k_uniform for every head). rank(j) = #{j' : M[j'] > M[j] or (M[j'] == M[j] and
// j' < j)}; block j is kept iff rank(j) < k_h. Kept blocks are written in
// ascending j by warp-ballot compaction.
__global__ void __launch_bounds__(256)
    topk_kernel(const float* __restrict__ mass, int rows, int nqb, int nkb, int k_uniform,
                const int32_t* __restrict__ head_k, int32_t* __restrict__ head_k_out,
                int32_t* __restrict__ kv_idx, int32_t* __restrict__ kv_count, int kv_stride) {
  constexpr int CH = 1024;
  __shared__ float buf[8][CH];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long row = static_cast<long>(blockIdx.x) * 8 + warp;
  if (row >= rows) return;
  const int h = static_cast<int>(row / nqb);
  int k = head_k ? head_k[h] : k_uniform;
  k = k < 0 ? 0 : (k > nkb ? nkb : k);
  if (k > kv_stride) k = kv_stride;
  const float* m = mass + row * nkb;
  int32_t* dst = kv_idx + row * kv_stride;
  int written = 0;
  for (int base = 0; base < nkb; base += 32) {
    const int j = base + lane;
    const float mj = j < nkb ? m[j] : 0.f;
    int rank = 0;
    for (int c0 = 0; c0 < nkb; c0 += CH) {
      const int len = nkb - c0 < CH ? nkb - c0 : CH;
      __syncwarp();
      for (int t = lane; t < len; t += 32) buf[warp][t] = m[c0 + t];
      __syncwarp();
      for (int t = 0; t < len; ++t) {
        const float x = buf[warp][t];
        rank += (x > mj) || (x == mj && c0 + t < j);
      }
    }
    const bool keep = j < nkb && rank < k;
    const unsigned ball = __ballot_sync(0xffffffffu, keep);
    if (keep) dst[written + __popc(ball & ((1u << lane) - 1u))] = j;
    written += __popc(ball);
  }
  if (lane == 0) {
    kv_count[row] = k;
    if (head_k_out && row % nqb == 0) head_k_out[h] = k;  // uniform budget: export k per head
  }
}

// ---------------------------------------------------------------- entropy budget

// One warp per (h, i): z = sum_j M, entropy = -sum_j (M/z) ln(M/z) over M > 0 (fp64).
__global__ void __launch_bounds__(256)
    row_entropy_kernel(const float* __restrict__ mass, int rows, int nkb, double* __restrict__ ent) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long row = static_cast<long>(blockIdx.x) * 8 + warp;
  if (row >= rows) return;
  const float* m = mass + row * nkb;
  double z = 0.0;
  for (int j = lane; j < nkb; j += 32) z += static_cast<double>(m[j]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
  double e = 0.0;
  if (z > 0.0) {
    for (int j = lane; j < nkb; j += 32) {
      const double x = static_cast<double>(m[j]);
      if (x > 0.0) {
        const double p = x / z;
        e -= p * log(p);
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) e += __shfl_xor_sync(0xffffffffu, e, off);
  if (lane == 0) ent[row] = e;
}

// The head-adaptive allocation (one thread, fp64): B = clamp(ceil(rho*H*nkb -
// 1e-6), H, H*nkb); one block per head, the extra B-H split in proportion to
// E_h (evenly if the split heads' E sum to 0), shares above nkb-1 capped and
// the rest re-split, then largest-remainder rounding with ties to the lower
// head. Writes k_h = 1 + extra_h. Shared by the device budget kernel and the
// host entry point for head-sharded selection; the budget product is formed
// without fused multiply-add so both sides take identical steps.
// scratch: extra, quota, mark (3*H doubles).
__host__ __device__ inline void allocate_budget(const double* E, int H, int nkb, float keep_ratio,
                                                double* extra, double* quota, double* mark, int32_t* head_k) {
  for (int h = 0; h < H; ++h) {
    extra[h] = -1.0;  // < 0: not yet decided
    mark[h] = 0.0;
  }
  const double rho = static_cast<double>(keep_ratio);
#ifdef __CUDA_ARCH__
  const double prod = __dmul_rn(__dmul_rn(rho, static_cast<double>(H)), static_cast<double>(nkb));
  long B = static_cast<long>(ceil(__dsub_rn(prod, 1e-6)));
#else
  volatile double prod = rho * static_cast<double>(H);
  prod = prod * static_cast<double>(nkb);
  long B = static_cast<long>(ceil(prod - 1e-6));
#endif
  if (B < H) B = H;
  if (B > static_cast<long>(H) * nkb) B = static_cast<long>(H) * nkb;
  const double cap = nkb - 1;
  while (true) {
    int nfree = 0;
    long fixed = 0;
    double sE = 0.0;
    for (int h = 0; h < H; ++h) {
      if (extra[h] < 0.0) {
        ++nfree;
        sE += E[h];
      } else {
        fixed += static_cast<long>(extra[h]);
      }
    }
    if (nfree == 0) break;
    const long Xf = (B - H) - fixed;
    const bool prop = sE > 0.0;
    const double sw = prop ? sE : static_cast<double>(nfree);
    bool over = false;
    for (int h = 0; h < H; ++h) {
      if (extra[h] >= 0.0) continue;
      const double w = prop ? E[h] : 1.0;
      if (static_cast<double>(Xf) * w / sw > cap) {
        extra[h] = cap;
        over = true;
      }
    }
    if (over) continue;
    long assigned = 0;
    for (int h = 0; h < H; ++h) {
      if (extra[h] >= 0.0) {
        quota[h] = -1.0;
        continue;
      }
      const double w = prop ? E[h] : 1.0;
      quota[h] = static_cast<double>(Xf) * w / sw;
      extra[h] = floor(quota[h]);
      assigned += static_cast<long>(extra[h]);
    }
    long rem = Xf - assigned;
    while (rem > 0) {  // one more unit to the largest fractions, ties to the lower head
      int best = -1;
      double bf = -1.0;
      for (int h = 0; h < H; ++h) {
        if (quota[h] < 0.0 || mark[h] != 0.0) continue;
        const double f = quota[h] - floor(quota[h]);
        if (f > bf) { bf = f; best = h; }
      }
      if (best < 0) break;
      extra[best] += 1.0;
      mark[best] = 1.0;
      --rem;
    }
    // (the floors never sum above Xf: quotas that sum to Xf up to a few ulps
    // can cross an integer from below only with fractional parts within an
    // ulp of 1, and one crossing more than the fractional parts add up to is
    // impossible, so rem >= 0)
    break;
  }
  for (int h = 0; h < H; ++h) head_k[h] = 1 + static_cast<int32_t>(extra[h]);
}

// Per-head mean of the row entropies: E_h = (sum_i ent[h,i]) / nqb, the sum
// sequential in i.
__device__ __forceinline__ double head_mean_entropy(const double* ent, int h, int nqb) {
  double s = 0.0;
  for (int i = 0; i < nqb; ++i) s += ent[static_cast<long>(h) * nqb + i];
  return s / nqb;
}

__global__ void head_entropy_kernel(const double* __restrict__ ent, int H, int nqb, double* __restrict__ E) {
  for (int h = threadIdx.x + blockIdx.x * blockDim.x; h < H; h += blockDim.x * gridDim.x)
    E[h] = head_mean_entropy(ent, h, nqb);
}

// One block: the head means, then the allocation on one thread.
// scratch: 4*H doubles (entropy, extra, quota, mark).
__global__ void budget_kernel(const double* __restrict__ ent, int H, int nqb, int nkb, float keep_ratio,
                              int32_t* __restrict__ head_k, double* __restrict__ scratch) {
  double* E = scratch;
  for (int h = threadIdx.x; h < H; h += blockDim.x) E[h] = head_mean_entropy(ent, h, nqb);
  __syncthreads();
  if (threadIdx.x != 0) return;
  allocate_budget(E, H, nkb, keep_ratio, scratch + H, scratch + 2 * H, scratch + 3 * H, head_k);
}

}  // namespace sparsed
