// Host side of the C ABI declared in include/sparsed.h: argument validation,
// workspace layout, TMA descriptor encoding, kernel launches and the
// denoising-step drivers. Every step of the computation runs in the kernels of
// attn_kernel.cuh, select_kernels.cuh, column_kernels.cuh and
// losa_kernels.cuh; nothing here computes attention.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "sparsed.h"
#include "attn_kernel.cuh"
#include "attn_list_kernel.cuh"
#include "select_kernels.cuh"
#include "column_kernels.cuh"
#include "losa_kernels.cuh"

using namespace sparsed;

namespace {

constexpr uint64_t kWaitTimeoutNs = 2000000000ull;  // 2 s bound on every device wait
constexpr double kRoundEps = 1e-6;

std::atomic<int> g_last_cuda{0};

int fail_cuda(cudaError_t e) {
  g_last_cuda.store(static_cast<int>(e));
  return SPARSED_ERR_CUDA;
}

#define SP_CUDA(x)                                   \
  do {                                               \
    cudaError_t e_ = (x);                            \
    if (e_ != cudaSuccess) return fail_cuda(e_);     \
  } while (0)

#define SP_TRY(x)                \
  do {                           \
    int rc_ = (x);               \
    if (rc_ != SPARSED_OK) return rc_; \
  } while (0)

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
cudaError_t g_encode_err = cudaSuccess;

int get_encoder() {
  std::call_once(g_encode_once, [] {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    g_encode_err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (g_encode_err == cudaSuccess && q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    else if (g_encode_err == cudaSuccess)
      g_encode_err = cudaErrorSymbolNotFound;
  });
  if (!g_encode) return fail_cuda(g_encode_err);
  return SPARSED_OK;
}

// Process-unique id of the CUDA context current on this thread (0 when none
// is current yet). Device-side addresses and library-owned streams belong to
// a context: caches of them are keyed on this id, so that a context created
// after cudaDeviceReset never sees the handles of the one before.
PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_id = nullptr;
std::once_flag g_ctx_once;

int context_id(unsigned long long* id) {
  std::call_once(g_ctx_once, [] {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(fn);
  });
  if (!g_ctx_current || !g_ctx_id) return fail_cuda(cudaErrorSymbolNotFound);
  CUcontext ctx = nullptr;
  if (g_ctx_current(&ctx) != CUDA_SUCCESS) return fail_cuda(cudaErrorContextIsDestroyed);
  *id = 0;
  if (ctx && g_ctx_id(ctx, id) != CUDA_SUCCESS) return fail_cuda(cudaErrorContextIsDestroyed);
  return SPARSED_OK;
}

int require_sm100() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaErrorNoDevice || e == cudaErrorInsufficientDriver) {
    g_last_cuda.store(static_cast<int>(e));
    return SPARSED_ERR_NO_DEVICE;
  }
  SP_CUDA(e);
  int major = 0, minor = 0;
  SP_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
  SP_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
  if (major != 10 || minor != 0) return SPARSED_ERR_NO_DEVICE;
  return SPARSED_OK;
}

// Number of SMs of the current device (the persistent grid size).
int sm_count(int* out) {
  int dev = 0;
  SP_CUDA(cudaGetDevice(&dev));
  SP_CUDA(cudaDeviceGetAttribute(out, cudaDevAttrMultiProcessorCount, dev));
  return SPARSED_OK;
}

inline long cdiv(long a, long b) { return (a + b - 1) / b; }
inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_shapes(int H, int L, int d, float scale, int bq, int bk) {
  if (H < 0 || L < 0) return SPARSED_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return SPARSED_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SPARSED_ERR_UNSUPPORTED;
  if ((bq != 64 && bq != 128) || (bk != 64 && bk != 128)) return SPARSED_ERR_UNSUPPORTED;
  if (H > 65535) return SPARSED_ERR_UNSUPPORTED;
  if (static_cast<long long>(H) * L * d >= (1ll << 31)) return SPARSED_ERR_UNSUPPORTED;
  return SPARSED_OK;
}

int check_qkvo(const void* Q, const void* K, const void* V, const void* O, const void* LSE) {
  if (!Q || !K || !V || !O || !LSE) return SPARSED_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return SPARSED_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(LSE) & 3u) != 0) return SPARSED_ERR_INVALID_ARG;
  return SPARSED_OK;
}

int uniform_k(int nkb, float keep) {
  const double k = std::ceil(static_cast<double>(keep) * nkb - kRoundEps);
  long kk = static_cast<long>(k);
  if (kk < 1) kk = 1;
  if (kk > nkb) kk = nkb;
  return static_cast<int>(kk);
}

// [H, L, d] bf16 viewed as a 3-D tensor (d innermost), boxes of 64 columns x rows.
int make_map(CUtensorMap* m, const void* ptr, int H, int L, int d, int box_rows) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(L),
                        static_cast<cuuint64_t>(H)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(L) * d * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
                        es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail_cuda(cudaErrorInvalidValue);
  return SPARSED_OK;
}

// One thread waits on an mbarrier that nothing arrives on: the bounded wait
// gives up after timeout_ns, records SPARSED_ERR_DEVICE_TIMEOUT in the device
// error word and returns. No copy or MMA is in flight.
__global__ void wait_timeout_selftest_kernel(unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ptx::mbar_init(ptx::smem_u32(&bar), 1);
    abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    volatile int* ab = &abort_flag;
    ptx::mbar_wait(ptx::smem_u32(&bar), 0, ab, timeout_ns, kErrTimeout);
  }
}

// ---- queries that change across the denoising steps
// Q_t = bf16(fp32(Q) + fp32(amplitude * u)) elementwise, with the counter-based
// uniform u = (fmix32(i ^ key) >> 8) * 2^-23 - 1 of element i (row-major over
// [H, L, d]) and key = fmix32(fmix32(seed) ^ t); fmix32 is the MurmurHash3
// 32-bit finalizer. The product and the sum are rounded once each (no fused
// multiply-add), so the bits are those of any other implementation of the
// same definition.
__host__ __device__ inline uint32_t fmix32(uint32_t h) {
  h ^= h >> 16;
  h *= 0x85EBCA6Bu;
  h ^= h >> 13;
  h *= 0xC2B2AE35u;
  h ^= h >> 16;
  return h;
}

inline uint32_t drift_key(uint32_t seed, int t) { return fmix32(fmix32(seed) ^ static_cast<uint32_t>(t)); }

__device__ __forceinline__ uint16_t bf16_rne(float x) {
  const uint32_t b = __float_as_uint(x);
  return static_cast<uint16_t>((b + 0x7FFFu + ((b >> 16) & 1u)) >> 16);
}

// Eight elements (16 bytes) per thread; n is a multiple of 8 (d is).
__global__ void __launch_bounds__(256)
    drift_queries_kernel(const uint4* __restrict__ q, long n8, uint32_t key, float amplitude,
                         uint4* __restrict__ q_out) {
  const long v = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (v >= n8) return;
  const uint4 in = q[v];
  const uint32_t w[4] = {in.x, in.y, in.z, in.w};
  uint32_t o[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    uint16_t r[2];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const uint32_t i = static_cast<uint32_t>(v * 8 + e * 2 + half);
      const float u = __fsub_rn(__fmul_rn(static_cast<float>(fmix32(i ^ key) >> 8), 0x1p-23f), 1.0f);
      const float qv = __uint_as_float((half ? (w[e] >> 16) : (w[e] & 0xFFFFu)) << 16);
      r[half] = bf16_rne(__fadd_rn(qv, __fmul_rn(u, amplitude)));
    }
    o[e] = static_cast<uint32_t>(r[0]) | (static_cast<uint32_t>(r[1]) << 16);
  }
  q_out[v] = make_uint4(o[0], o[1], o[2], o[3]);
}

struct Problem {
  const uint16_t *Q, *K, *V;
  uint16_t* O;
  float* LSE;
  int H, L, d, bq, bk, nqb, nkb;
  int Lk;  // rows of K and V: L, or the kept columns of a column pattern
  float scale;
};

// Counter slots of the two-tile kernel's pair scheduler, in a caller's
// workspace. Launch k of a sequence on one stream claims pairs from slot k % 2
// and clears slot (k + 1) % 2 for launch k + 1; stream order has finished
// launch k - 1, that slot's last user, by then. One memset clears the first
// slot when the sequence starts. Without slots (base == nullptr) the kernel
// takes its pairs by the static stride.
struct PairSched {
  int* base = nullptr;
  int k = 0;
};

int begin_pair_sched(PairSched* ps, void* slots, cudaStream_t st) {
  ps->base = static_cast<int*>(slots);
  ps->k = 0;
  if (ps->base) SP_CUDA(cudaMemsetAsync(ps->base, 0, 2 * sizeof(int), st));
  return SPARSED_OK;
}

// The register split of the kernel (setmaxnreg) must be funded by its launch
// register count; checked once per kernel before the first launch, so a raise
// can never wait forever.
template <int D, int BK, bool MASS>
int launch_attn_t(const Problem& p, const float* lse_prev, float* mass_part, PairSched* ps, cudaStream_t st) {
  using C = AttnCfg<D, BK>;
  auto kern = attn_fwd_kernel<D, BK, MASS>;
  static int regs = -1;
  if (regs < 0) {
    cudaFuncAttributes fa;
    SP_CUDA(cudaFuncGetAttributes(&fa, kern));
    regs = fa.numRegs;
  }
  if (regs * C::THREADS < C::REGS_SOFTMAX * 256 + C::REGS_OTHER * (C::THREADS - 256)) return SPARSED_ERR_UNSUPPORTED;
  CUtensorMap tq, tk, tv;
  SP_TRY(make_map(&tq, p.Q, p.H, p.L, D, 128));
  SP_TRY(make_map(&tk, p.K, p.H, p.Lk, D, BK));
  SP_TRY(make_map(&tv, p.V, p.H, p.Lk, D, BK));
  AttnArgs a;
  a.H = p.H;
  a.L = p.L;
  a.Lk = p.Lk;
  a.bq = p.bq;
  a.nqb = p.nqb;
  a.nkb = p.nkb;
  a.scale_log2 = p.scale * 1.44269504088896340736f;
  a.kv_idx = nullptr;
  a.kv_count = nullptr;
  a.kv_stride = 0;
  a.lse = p.LSE;
  a.o = p.O;
  a.lse_prev = lse_prev;
  a.mass_part = mass_part;
  a.timeout_ns = kWaitTimeoutNs;
  const bool dyn = ps && ps->base;
  a.sched = dyn ? ps->base + (ps->k & 1) : nullptr;
  a.sched_reset = dyn ? ps->base + ((ps->k + 1) & 1) : nullptr;
  int sms = 0;
  SP_TRY(sm_count(&sms));
  SP_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES));
  // persistent: one CTA per SM (its registers admit one); CTA b starts with
  // pair b, then takes pairs by the static stride or from the counter
  const long pairs = static_cast<long>(p.H) * ((p.nqb + 1) / 2);
  const int grid = static_cast<int>(pairs < sms ? pairs : sms);
  kern<<<grid, C::THREADS, C::SMEM_BYTES, st>>>(tq, tk, tv, a);
  SP_CUDA(cudaGetLastError());
  if (dyn) ++ps->k;
  return SPARSED_OK;
}

// A kernel launch that may start as a programmatic dependent of the previous
// kernel on the stream (pdl): its CTAs are scheduled while that kernel
// finishes and wait in the kernel (griddepcontrol.wait) before they read its
// results. Only kernels that wait before any global access are launched so.
template <typename... KArgs, typename... Args>
int launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  SP_CUDA(cudaLaunchKernelEx(&cfg, kern, args...));
  return SPARSED_OK;
}

// Block-sparse passes: the one-tile kernel (each query tile walks its own
// list), with the same register-split check.
template <int D, int BK>
int launch_list_t(const Problem& p, const int32_t* kv_idx, const int32_t* kv_count, int kv_stride,
                  cudaStream_t st, bool pdl = false) {
  using C = ListCfg<D, BK>;
  auto kern = attn_list_kernel<D, BK>;
  static int regs = -1;
  if (regs < 0) {
    cudaFuncAttributes fa;
    SP_CUDA(cudaFuncGetAttributes(&fa, kern));
    regs = fa.numRegs;
  }
  if (regs * C::THREADS < C::REGS_SOFTMAX * 256 + C::REGS_OTHER * 128) return SPARSED_ERR_UNSUPPORTED;
  CUtensorMap tq, tk, tv;
  SP_TRY(make_map(&tq, p.Q, p.H, p.L, D, 128));
  SP_TRY(make_map(&tk, p.K, p.H, p.Lk, D, BK));
  SP_TRY(make_map(&tv, p.V, p.H, p.Lk, D, BK));
  AttnArgs a;
  a.H = p.H;
  a.L = p.L;
  a.Lk = p.Lk;
  a.bq = p.bq;
  a.nqb = p.nqb;
  a.nkb = p.nkb;
  a.scale_log2 = p.scale * 1.44269504088896340736f;
  a.kv_idx = kv_idx;
  a.kv_count = kv_count;
  a.kv_stride = kv_stride;
  a.lse = p.LSE;
  a.o = p.O;
  a.lse_prev = nullptr;
  a.mass_part = nullptr;
  a.timeout_ns = kWaitTimeoutNs;
  a.sched = nullptr;
  a.sched_reset = nullptr;
  int sms = 0;
  SP_TRY(sm_count(&sms));
  SP_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES));
  // persistent: one CTA per SM, each walking items blockIdx.x, blockIdx.x + gridDim.x, ...
  const long items = static_cast<long>(p.H) * p.nqb;
  const int grid = static_cast<int>(items < sms ? items : sms);
  if (pdl) return launch_k(kern, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, st, true, tq, tk, tv, a);
  kern<<<grid, C::THREADS, C::SMEM_BYTES, st>>>(tq, tk, tv, a);
  SP_CUDA(cudaGetLastError());
  return SPARSED_OK;
}

// Dense passes (and the fused selecting pass) run in the two-tile kernel,
// block-sparse passes in the one-tile kernel. mass_part != nullptr selects the
// fused variant (dense only): the pass also writes the block-mass partials,
// using lse_prev as every row's LSE. ps (nullable) gives the dense passes the
// counter slots of their pair scheduler; pdl launches a block-sparse pass as a
// programmatic dependent of the previous kernel on the stream.
int launch_attn(const Problem& p, bool sparse, const int32_t* kv_idx, const int32_t* kv_count,
                int kv_stride, cudaStream_t st, const float* lse_prev = nullptr, float* mass_part = nullptr,
                PairSched* ps = nullptr, bool pdl = false) {
#define SP_ATTN(D_, BK_)                                                                                  \
  if (p.d == D_ && p.bk == BK_) {                                                                         \
    if (sparse) return launch_list_t<D_, BK_>(p, kv_idx, kv_count, kv_stride, st, pdl);                   \
    if (mass_part) return launch_attn_t<D_, BK_, true>(p, lse_prev, mass_part, ps, st);                 \
    return launch_attn_t<D_, BK_, false>(p, nullptr, nullptr, ps, st);                                    \
  }
  SP_ATTN(64, 64)
  SP_ATTN(64, 128)
  SP_ATTN(128, 64)
  SP_ATTN(128, 128)
#undef SP_ATTN
  return SPARSED_ERR_UNSUPPORTED;
}

// One dense pass whose pairs come from the counter slots in a call's workspace.
int dense_pass_counted(const Problem& p, void* slots, cudaStream_t st) {
  PairSched ps;
  SP_TRY(begin_pair_sched(&ps, slots, st));
  return launch_attn(p, false, nullptr, nullptr, 0, st, nullptr, nullptr, &ps);
}

template <int D, int BK>
int launch_mass_t(const Problem& p, float* mass, cudaStream_t st) {
  using C = MassCfg<D, BK>;
  CUtensorMap tq, tk;
  SP_TRY(make_map(&tq, p.Q, p.H, p.L, D, 128));
  SP_TRY(make_map(&tk, p.K, p.H, p.L, D, BK));
  MassArgs a;
  a.H = p.H;
  a.L = p.L;
  a.bq = p.bq;
  a.nqb = p.nqb;
  a.nkb = p.nkb;
  a.scale_log2 = p.scale * 1.44269504088896340736f;
  a.lse = p.LSE;
  a.mass = mass;
  a.timeout_ns = kWaitTimeoutNs;
  auto kern = block_mass_kernel<D, BK>;
  SP_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES));
  kern<<<dim3(p.nqb, p.H), C::THREADS, C::SMEM_BYTES, st>>>(tq, tk, a);
  SP_CUDA(cudaGetLastError());
  return SPARSED_OK;
}

int launch_mass(const Problem& p, float* mass, cudaStream_t st) {
  if (p.d == 64 && p.bk == 64) return launch_mass_t<64, 64>(p, mass, st);
  if (p.d == 64 && p.bk == 128) return launch_mass_t<64, 128>(p, mass, st);
  if (p.d == 128 && p.bk == 64) return launch_mass_t<128, 64>(p, mass, st);
  if (p.d == 128 && p.bk == 128) return launch_mass_t<128, 128>(p, mass, st);
  return SPARSED_ERR_UNSUPPORTED;
}

// ---- column path (PulseCol abstract): column mass, top-k columns, gather,
// then the dense attention kernel over the gathered keys

template <int D>
int launch_col_mass_t(const Problem& p, float* mass, cudaStream_t st) {
  using C = ColMassCfg<D>;
  CUtensorMap tq, tk;
  SP_TRY(make_map(&tq, p.Q, p.H, p.L, D, C::N));
  SP_TRY(make_map(&tk, p.K, p.H, p.L, D, C::M));
  ColMassArgs a;
  a.H = p.H;
  a.L = p.L;
  a.Lk = p.L;
  a.scale_log2 = p.scale * 1.44269504088896340736f;
  a.lse = p.LSE;
  a.mass = mass;
  a.timeout_ns = kWaitTimeoutNs;
  auto kern = column_mass_kernel<D>;
  SP_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES));
  kern<<<dim3(static_cast<unsigned>(cdiv(p.L, C::M)), p.H), C::THREADS, C::SMEM_BYTES, st>>>(tq, tk, a);
  SP_CUDA(cudaGetLastError());
  return SPARSED_OK;
}

int launch_col_mass(const Problem& p, float* mass, cudaStream_t st) {
  if (p.d == 64) return launch_col_mass_t<64>(p, mass, st);
  if (p.d == 128) return launch_col_mass_t<128>(p, mass, st);
  return SPARSED_ERR_UNSUPPORTED;
}

struct ColWorkspace {
  size_t mass, ksel, vsel, sched, total;
};

ColWorkspace col_ws_layout(int H, int L, int d, int kc) {
  ColWorkspace w;
  w.mass = 0;
  w.ksel = align256(static_cast<size_t>(H) * L * sizeof(float));
  w.vsel = w.ksel + align256(static_cast<size_t>(H) * kc * d * 2);
  w.sched = w.vsel + align256(static_cast<size_t>(H) * kc * d * 2);
  w.total = w.sched + align256(2 * sizeof(int32_t));  // the pair scheduler's counter slots
  return w;
}

int check_column_args(const Problem& p, int kc, const int32_t* cols, int col_stride, const void* workspace,
                      size_t ws_bytes) {
  if (!cols || kc < 1 || kc > p.L || col_stride < kc) return SPARSED_ERR_INVALID_ARG;
  if (static_cast<long long>(p.H) * col_stride >= (1ll << 31)) return SPARSED_ERR_UNSUPPORTED;
  if (!workspace || ws_bytes < col_ws_layout(p.H, p.L, p.d, kc).total) return SPARSED_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return SPARSED_ERR_INVALID_ARG;
  return SPARSED_OK;
}

// After the dense pass wrote O and LSE: column mass -> the kc columns per head.
int select_columns_after_dense(const Problem& p, int kc, int32_t* cols, int col_stride, float* mass_out,
                               void* workspace, cudaStream_t st) {
  float* mass = mass_out ? mass_out
                         : reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                                    col_ws_layout(p.H, p.L, p.d, kc).mass);
  SP_TRY(launch_col_mass(p, mass, st));
  topk_columns_kernel<<<p.H, 1024, 0, st>>>(mass, p.L, kc, cols, col_stride);
  SP_CUDA(cudaGetLastError());
  return SPARSED_OK;
}

// Attention of every query over the head's kc kept columns: gather them, then
// run the dense kernel with kc keys.
int column_attn(const Problem& p, const int32_t* cols, int kc, int col_stride, void* workspace, cudaStream_t st) {
  const ColWorkspace w = col_ws_layout(p.H, p.L, p.d, kc);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint16_t* ksel = reinterpret_cast<uint16_t*>(ws + w.ksel);
  uint16_t* vsel = reinterpret_cast<uint16_t*>(ws + w.vsel);
  const int row_u4 = p.d * 2 / 16;
  const long per_head = static_cast<long>(kc) * row_u4;
  gather_rows_kernel<<<dim3(static_cast<unsigned>(cdiv(per_head, 256)), p.H), 256, 0, st>>>(
      reinterpret_cast<const uint4*>(p.K), reinterpret_cast<const uint4*>(p.V), cols, p.L, kc, col_stride, row_u4,
      reinterpret_cast<uint4*>(ksel), reinterpret_cast<uint4*>(vsel));
  SP_CUDA(cudaGetLastError());
  Problem g = p;
  g.K = ksel;
  g.V = vsel;
  g.Lk = kc;
  g.nkb = static_cast<int>(cdiv(kc, p.bk));
  return launch_attn(g, false, nullptr, nullptr, 0, st);
}

struct Workspace {
  size_t grid, ent, scratch, headk, sched, total;
};

Workspace ws_layout(int H, int nqb, int nkb) {
  Workspace w;
  w.grid = 0;
  w.ent = w.grid + align256(static_cast<size_t>(H) * nqb * nkb * sizeof(float));
  w.scratch = w.ent + align256(static_cast<size_t>(H) * nqb * sizeof(double));
  w.headk = w.scratch + align256(static_cast<size_t>(H) * 4 * sizeof(double));
  w.sched = w.headk + align256(static_cast<size_t>(H) * sizeof(int32_t));
  w.total = w.sched + align256(2 * sizeof(int32_t));  // the pair scheduler's counter slots
  return w;
}

// Steps 3-4 of pattern selection from a block-mass grid: budget and top-k.
int select_from_mass(const Problem& p, const float* mass, float keep_ratio, int budget_mode, int32_t* kv_idx,
                     int32_t* kv_count, int kv_stride, int32_t* head_k, void* workspace, cudaStream_t st) {
  const Workspace w = ws_layout(p.H, p.nqb, p.nkb);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int rows = p.H * p.nqb;
  const int kblocks = (rows + 7) / 8;
  int32_t* hk = nullptr;
  int k_uniform = uniform_k(p.nkb, keep_ratio);
  if (budget_mode == SPARSED_BUDGET_ENTROPY) {
    double* ent = reinterpret_cast<double*>(ws + w.ent);
    double* scratch = reinterpret_cast<double*>(ws + w.scratch);
    hk = head_k ? head_k : reinterpret_cast<int32_t*>(ws + w.headk);
    row_entropy_kernel<<<kblocks, 256, 0, st>>>(mass, rows, p.nkb, ent);
    SP_CUDA(cudaGetLastError());
    budget_kernel<<<1, 256, 0, st>>>(ent, p.H, p.nqb, p.nkb, keep_ratio, hk, scratch);
    SP_CUDA(cudaGetLastError());
  }
  int32_t* hk_out = (budget_mode == SPARSED_BUDGET_UNIFORM) ? head_k : nullptr;
  topk_kernel<<<kblocks, 256, 0, st>>>(mass, rows, p.nqb, p.nkb, k_uniform, hk, hk_out, kv_idx,
                                       kv_count, kv_stride);
  SP_CUDA(cudaGetLastError());
  return SPARSED_OK;
}

// Steps 2-4 of pattern selection, after the dense pass wrote O and LSE.
int select_after_dense(const Problem& p, float keep_ratio, int budget_mode, int32_t* kv_idx,
                       int32_t* kv_count, int kv_stride, float* block_mass, int32_t* head_k,
                       void* workspace, cudaStream_t st) {
  const Workspace w = ws_layout(p.H, p.nqb, p.nkb);
  float* mass = block_mass ? block_mass : reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + w.grid);
  SP_TRY(launch_mass(p, mass, st));
  return select_from_mass(p, mass, keep_ratio, budget_mode, kv_idx, kv_count, kv_stride, head_k, workspace, st);
}

// Fused selection of the step loop: the scratch after the selection workspace
// holds the block-mass partials of the fused pass and a copy of the LSE of
// the run's last full pass.
struct FusedWorkspace {
  size_t part, lse_prev, total;
};

FusedWorkspace fused_ws_layout(int H, int L, int nqb, int nkb) {
  FusedWorkspace f;
  f.part = ws_layout(H, nqb, nkb).total;
  f.lse_prev = f.part + align256(static_cast<size_t>(H) * nqb * nkb * kMassParts * sizeof(float));
  f.total = f.lse_prev + align256(static_cast<size_t>(H) * L * sizeof(float));
  return f;
}

// A selecting step whose block mass comes from its own full pass: every row's
// LSE is taken from lse_prev, the LSE of an earlier full pass of the same
// inputs (so it equals the LSE this pass computes).
int fused_select(const Problem& p, float keep_ratio, int budget_mode, int32_t* kv_idx, int32_t* kv_count,
                 int kv_stride, void* workspace, PairSched* ps, cudaStream_t st) {
  const FusedWorkspace f = fused_ws_layout(p.H, p.L, p.nqb, p.nkb);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* part = reinterpret_cast<float*>(ws + f.part);
  const float* lse_prev = reinterpret_cast<const float*>(ws + f.lse_prev);
  SP_TRY(launch_attn(p, false, nullptr, nullptr, 0, st, lse_prev, part, ps));
  float* mass = reinterpret_cast<float*>(ws + ws_layout(p.H, p.nqb, p.nkb).grid);
  const long n = static_cast<long>(p.H) * p.nqb * p.nkb;
  mass_from_parts_kernel<<<static_cast<unsigned>(cdiv(n, 256)), 256, 0, st>>>(reinterpret_cast<const float4*>(part),
                                                                               n, mass);
  SP_CUDA(cudaGetLastError());
  return select_from_mass(p, mass, keep_ratio, budget_mode, kv_idx, kv_count, kv_stride, nullptr, workspace, st);
}

int save_lse(const Problem& p, void* workspace, cudaStream_t st) {
  const FusedWorkspace f = fused_ws_layout(p.H, p.L, p.nqb, p.nkb);
  SP_CUDA(cudaMemcpyAsync(static_cast<uint8_t*>(workspace) + f.lse_prev, p.LSE,
                          static_cast<size_t>(p.H) * p.L * sizeof(float), cudaMemcpyDeviceToDevice, st));
  return SPARSED_OK;
}

int prepare(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int H, int L, int d, float scale,
            int bq, int bk, uint16_t* O, float* LSE, Problem* p, bool* empty) {
  SP_TRY(check_shapes(H, L, d, scale, bq, bk));
  *empty = (static_cast<long>(H) * L == 0);
  if (*empty) return SPARSED_OK;
  SP_TRY(check_qkvo(Q, K, V, O, LSE));
  p->Q = Q;
  p->K = K;
  p->V = V;
  p->O = O;
  p->LSE = LSE;
  p->H = H;
  p->L = L;
  p->d = d;
  p->bq = bq;
  p->bk = bk;
  p->nqb = static_cast<int>(cdiv(L, bq));
  p->nkb = static_cast<int>(cdiv(L, bk));
  p->Lk = L;
  p->scale = scale;
  return SPARSED_OK;
}

int check_select_args(const Problem& p, float keep_ratio, int budget_mode, int32_t* kv_idx,
                      int32_t* kv_count, int kv_stride, void* workspace, size_t ws_bytes) {
  if (!(keep_ratio > 0.f && keep_ratio <= 1.f)) return SPARSED_ERR_INVALID_ARG;
  if (budget_mode != SPARSED_BUDGET_UNIFORM && budget_mode != SPARSED_BUDGET_ENTROPY)
    return SPARSED_ERR_INVALID_ARG;
  if (!kv_idx || !kv_count) return SPARSED_ERR_INVALID_ARG;
  const int need = budget_mode == SPARSED_BUDGET_UNIFORM ? uniform_k(p.nkb, keep_ratio) : p.nkb;
  if (kv_stride < need) return SPARSED_ERR_INVALID_ARG;
  if (static_cast<long long>(p.H) * p.nqb * kv_stride >= (1ll << 31)) return SPARSED_ERR_UNSUPPORTED;
  if (static_cast<long long>(p.H) * p.nqb * p.nkb >= (1ll << 31)) return SPARSED_ERR_UNSUPPORTED;
  const Workspace w = ws_layout(p.H, p.nqb, p.nkb);
  if (!workspace || ws_bytes < w.total) return SPARSED_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SPARSED_ERR_WORKSPACE;
  return SPARSED_OK;
}

// Per-step queries of the step driver: seed and amplitude of the drift, and
// the caller's buffer that receives each step's queries.
struct Drift {
  uint32_t seed;
  float amplitude;
  uint16_t* q_step;
};

int launch_drift(const uint16_t* Q, long n, uint32_t seed, int t, float amplitude, uint16_t* Q_out,
                 cudaStream_t st) {
  const long n8 = n / 8;
  drift_queries_kernel<<<static_cast<unsigned>(cdiv(n8, 256)), 256, 0, st>>>(
      reinterpret_cast<const uint4*>(Q), n8, drift_key(seed, t), amplitude, reinterpret_cast<uint4*>(Q_out));
  SP_CUDA(cudaGetLastError());
  return SPARSED_OK;
}

int run_steps_impl(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int H, int L, int d,
                   float scale, int bq, int bk, float keep_ratio, int budget_mode, int T,
                   float warmup_frac, int refresh_every, int start_step, int end_step,
                   int have_pattern, int32_t* kv_idx, int32_t* kv_count, int kv_stride, uint16_t* O,
                   float* LSE, int8_t* step_kind, float* step_ms, void* workspace,
                   size_t workspace_bytes, void* stream, const Drift* drift);

}  // namespace

extern "C" {

int sparsed_version(void) { return SPARSED_VERSION; }

const char* sparsed_strerror(int status) {
  switch (status) {
    case SPARSED_OK: return "ok";
    case SPARSED_ERR_INVALID_ARG: return "invalid argument (null pointer, negative size, bad value or misaligned buffer)";
    case SPARSED_ERR_UNSUPPORTED: return "unsupported configuration (d, block size or size limit)";
    case SPARSED_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case SPARSED_ERR_BAD_PATTERN: return "block pattern entry out of range or not strictly ascending";
    case SPARSED_ERR_CUDA: return "CUDA runtime error (see sparsed_last_cuda_error)";
    case SPARSED_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait expired";
    case SPARSED_ERR_NO_DEVICE: return "no sm_100 (B200) device is current";
    case SPARSED_ERR_EXCHANGE: return "the exchange callback of the head-sharded loop failed";
    default: return "unknown status";
  }
}

int sparsed_last_cuda_error(void) { return g_last_cuda.load(); }

int sparsed_check(void* stream) {
  SP_TRY(require_sm100());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SP_CUDA(cudaStreamSynchronize(st));
  int code = 0;
  SP_CUDA(cudaMemcpyFromSymbol(&code, ptx::g_device_error, sizeof(int)));
  if (code != 0) {
    const int zero = 0;
    SP_CUDA(cudaMemcpyToSymbol(ptx::g_device_error, &zero, sizeof(int)));
  }
  return code;
}

int sparsed_selftest_wait_timeout(unsigned long long timeout_ns, void* stream) {
  if (timeout_ns == 0 || timeout_ns > 1000000000ull) return SPARSED_ERR_INVALID_ARG;
  SP_TRY(require_sm100());
  wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(timeout_ns);
  SP_CUDA(cudaGetLastError());
  return SPARSED_OK;
}

int sparsed_uniform_keep(int L, int bk, float keep_ratio, int* k_out) {
  if (!k_out || L <= 0 || bk <= 0) return SPARSED_ERR_INVALID_ARG;
  if (!(keep_ratio > 0.f && keep_ratio <= 1.f)) return SPARSED_ERR_INVALID_ARG;
  *k_out = uniform_k(static_cast<int>(cdiv(L, bk)), keep_ratio);
  return SPARSED_OK;
}

int sparsed_schedule(int T, float warmup_frac, int refresh_every, int8_t* kinds) {
  if (T < 0 || refresh_every < 0) return SPARSED_ERR_INVALID_ARG;
  if (!(warmup_frac >= 0.f && warmup_frac <= 1.f)) return SPARSED_ERR_INVALID_ARG;
  if (T == 0) return SPARSED_OK;
  if (!kinds) return SPARSED_ERR_INVALID_ARG;
  long n_dense = static_cast<long>(std::ceil(static_cast<double>(warmup_frac) * T - kRoundEps));
  if (n_dense < 1) n_dense = 1;
  if (n_dense > T) n_dense = T;
  for (int t = 0; t < T; ++t) {
    int8_t k;
    if (n_dense == T || t < n_dense - 1)
      k = SPARSED_STEP_DENSE;
    else if (t == n_dense - 1)
      k = SPARSED_STEP_SELECT;
    else if (refresh_every > 0 && (t - (n_dense - 1)) % refresh_every == 0)
      k = SPARSED_STEP_SELECT;
    else
      k = SPARSED_STEP_SPARSE;
    kinds[t] = k;
  }
  return SPARSED_OK;
}

int sparsed_workspace_bytes(int H, int L, int bq, int bk, size_t* bytes) {
  if (!bytes || H < 0 || L < 0) return SPARSED_ERR_INVALID_ARG;
  if ((bq != 64 && bq != 128) || (bk != 64 && bk != 128)) return SPARSED_ERR_UNSUPPORTED;
  *bytes = ws_layout(H, static_cast<int>(cdiv(L, bq)), static_cast<int>(cdiv(L, bk))).total;
  return SPARSED_OK;
}

int sparsed_run_steps_workspace_bytes(int H, int L, int bq, int bk, size_t* bytes) {
  if (!bytes || H < 0 || L < 0) return SPARSED_ERR_INVALID_ARG;
  if ((bq != 64 && bq != 128) || (bk != 64 && bk != 128)) return SPARSED_ERR_UNSUPPORTED;
  *bytes = fused_ws_layout(H, L, static_cast<int>(cdiv(L, bq)), static_cast<int>(cdiv(L, bk))).total;
  return SPARSED_OK;
}

int sparsed_dense_attn(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int H, int L, int d,
                       float scale, int bq, int bk, uint16_t* O, float* LSE, void* stream) {
  Problem p;
  bool empty = false;
  SP_TRY(prepare(Q, K, V, H, L, d, scale, bq, bk, O, LSE, &p, &empty));
  if (empty) return SPARSED_OK;
  SP_TRY(require_sm100());
  SP_TRY(get_encoder());
  return launch_attn(p, false, nullptr, nullptr, 0, static_cast<cudaStream_t>(stream));
}

int sparsed_select_pattern(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int H, int L, int d,
                           float scale, int bq, int bk, float keep_ratio, int budget_mode, uint16_t* O,
                           float* LSE, int32_t* kv_idx, int32_t* kv_count, int kv_stride,
                           float* block_mass, int32_t* head_k, void* workspace, size_t workspace_bytes,
                           void* stream) {
  Problem p;
  bool empty = false;
  SP_TRY(prepare(Q, K, V, H, L, d, scale, bq, bk, O, LSE, &p, &empty));
  if (empty) return SPARSED_OK;
  SP_TRY(check_select_args(p, keep_ratio, budget_mode, kv_idx, kv_count, kv_stride, workspace,
                           workspace_bytes));
  SP_TRY(require_sm100());
  SP_TRY(get_encoder());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SP_TRY(dense_pass_counted(p, static_cast<uint8_t*>(workspace) + ws_layout(p.H, p.nqb, p.nkb).sched, st));
  return select_after_dense(p, keep_ratio, budget_mode, kv_idx, kv_count, kv_stride, block_mass, head_k,
                            workspace, st);
}

int sparsed_block_sparse_attn(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int H, int L, int d,
                              float scale, int bq, int bk, const int32_t* kv_idx, const int32_t* kv_count,
                              int kv_stride, uint16_t* O, float* LSE, void* stream) {
  Problem p;
  bool empty = false;
  SP_TRY(prepare(Q, K, V, H, L, d, scale, bq, bk, O, LSE, &p, &empty));
  if (empty) return SPARSED_OK;
  if (!kv_idx || !kv_count || kv_stride < 1) return SPARSED_ERR_INVALID_ARG;
  if (static_cast<long long>(p.H) * p.nqb * kv_stride >= (1ll << 31)) return SPARSED_ERR_UNSUPPORTED;
  SP_TRY(require_sm100());
  SP_TRY(get_encoder());
  return launch_attn(p, true, kv_idx, kv_count, kv_stride, static_cast<cudaStream_t>(stream));
}

int sparsed_run_steps(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int H, int L, int d,
                      float scale, int bq, int bk, float keep_ratio, int budget_mode, int T,
                      float warmup_frac, int refresh_every, int start_step, int have_pattern,
                      int32_t* kv_idx, int32_t* kv_count, int kv_stride, uint16_t* O, float* LSE,
                      int8_t* step_kind, float* step_ms, void* workspace, size_t workspace_bytes,
                      void* stream) {
  return sparsed_run_steps_span(Q, K, V, H, L, d, scale, bq, bk, keep_ratio, budget_mode, T, warmup_frac,
                                refresh_every, start_step, T, have_pattern, kv_idx, kv_count, kv_stride, O, LSE,
                                step_kind, step_ms, workspace, workspace_bytes, stream);
}

int sparsed_run_steps_span(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int H, int L, int d,
                           float scale, int bq, int bk, float keep_ratio, int budget_mode, int T,
                           float warmup_frac, int refresh_every, int start_step, int end_step,
                           int have_pattern, int32_t* kv_idx, int32_t* kv_count, int kv_stride, uint16_t* O,
                           float* LSE, int8_t* step_kind, float* step_ms, void* workspace,
                           size_t workspace_bytes, void* stream) {
  return run_steps_impl(Q, K, V, H, L, d, scale, bq, bk, keep_ratio, budget_mode, T, warmup_frac, refresh_every,
                        start_step, end_step, have_pattern, kv_idx, kv_count, kv_stride, O, LSE, step_kind, step_ms,
                        workspace, workspace_bytes, stream, nullptr);
}

int sparsed_run_steps_drift(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int H, int L, int d,
                            float scale, int bq, int bk, float keep_ratio, int budget_mode, int T,
                            float warmup_frac, int refresh_every, int start_step, int end_step,
                            int have_pattern, unsigned int drift_seed, float drift_amplitude, uint16_t* Q_step,
                            int32_t* kv_idx, int32_t* kv_count, int kv_stride, uint16_t* O, float* LSE,
                            int8_t* step_kind, float* step_ms, void* workspace, size_t workspace_bytes,
                            void* stream) {
  if (!Q_step || !aligned16(Q_step) || !std::isfinite(drift_amplitude)) return SPARSED_ERR_INVALID_ARG;
  const Drift drift{drift_seed, drift_amplitude, Q_step};
  return run_steps_impl(Q, K, V, H, L, d, scale, bq, bk, keep_ratio, budget_mode, T, warmup_frac, refresh_every,
                        start_step, end_step, have_pattern, kv_idx, kv_count, kv_stride, O, LSE, step_kind, step_ms,
                        workspace, workspace_bytes, stream, &drift);
}

int sparsed_drift_queries(const uint16_t* Q, int H, int L, int d, unsigned int seed, int t, float amplitude,
                          uint16_t* Q_out, void* stream) {
  if (H < 0 || L < 0 || t < 0) return SPARSED_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SPARSED_ERR_UNSUPPORTED;
  if (!Q || !Q_out || !aligned16(Q) || !aligned16(Q_out) || !std::isfinite(amplitude))
    return SPARSED_ERR_INVALID_ARG;
  if (static_cast<long long>(H) * L * d >= (1ll << 31)) return SPARSED_ERR_UNSUPPORTED;
  if (static_cast<long>(H) * L == 0) return SPARSED_OK;
  SP_TRY(require_sm100());
  return launch_drift(Q, static_cast<long>(H) * L * d, seed, t, amplitude, Q_out, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {

int run_steps_impl(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int H, int L, int d,
                   float scale, int bq, int bk, float keep_ratio, int budget_mode, int T,
                   float warmup_frac, int refresh_every, int start_step, int end_step,
                   int have_pattern, int32_t* kv_idx, int32_t* kv_count, int kv_stride, uint16_t* O,
                   float* LSE, int8_t* step_kind, float* step_ms, void* workspace,
                   size_t workspace_bytes, void* stream, const Drift* drift) {
  if (T < 0 || start_step < 0 || start_step > end_step || end_step > T) return SPARSED_ERR_INVALID_ARG;
  std::vector<int8_t> kinds(static_cast<size_t>(T) + 1);
  SP_TRY(sparsed_schedule(T, warmup_frac, refresh_every, kinds.data()));
  if (step_kind && T > 0) std::memcpy(step_kind, kinds.data(), static_cast<size_t>(T));
  if (step_ms)
    for (int t = 0; t < T; ++t) step_ms[t] = 0.f;
  Problem p;
  bool empty = false;
  SP_TRY(prepare(Q, K, V, H, L, d, scale, bq, bk, O, LSE, &p, &empty));
  if (empty) return SPARSED_OK;
  bool any_select = false, pattern_ready = have_pattern != 0;
  for (int t = start_step; t < end_step; ++t) {
    if (kinds[t] == SPARSED_STEP_SELECT) pattern_ready = any_select = true;
    if (kinds[t] == SPARSED_STEP_SPARSE && !pattern_ready) return SPARSED_ERR_INVALID_ARG;
  }
  if (any_select)
    SP_TRY(check_select_args(p, keep_ratio, budget_mode, kv_idx, kv_count, kv_stride, workspace,
                             workspace_bytes));
  else if (start_step < end_step && pattern_ready && (!kv_idx || !kv_count || kv_stride < 1))
    return SPARSED_ERR_INVALID_ARG;
  SP_TRY(require_sm100());
  SP_TRY(get_encoder());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // fused selection when the workspace has room for it (see the header)
  const bool fused = any_select && workspace &&
                     workspace_bytes >= fused_ws_layout(p.H, p.L, p.nqb, p.nkb).total &&
                     static_cast<long long>(p.H) * p.nqb * p.nkb * kMassParts < (1ll << 31);
  bool have_lse = false;  // a full pass of this call left its LSE in the workspace
  // the dense passes take their pairs from counters in the workspace when it
  // has the room
  const Workspace wl = ws_layout(p.H, p.nqb, p.nkb);
  PairSched ps;
  SP_TRY(begin_pair_sched(&ps, workspace && workspace_bytes >= wl.total ? static_cast<uint8_t*>(workspace) + wl.sched
                                                                        : nullptr,
                          st));
  std::vector<cudaEvent_t> ev;
  if (step_ms && start_step < end_step) {
    ev.resize(static_cast<size_t>(end_step - start_step) + 1, nullptr);
    for (auto& e : ev) SP_CUDA(cudaEventCreate(&e));
    SP_CUDA(cudaEventRecord(ev[0], st));
  }
  int rc = SPARSED_OK;
  if (drift) p.Q = drift->q_step;  // every step attends with its own queries
  for (int t = start_step; t < end_step && rc == SPARSED_OK; ++t) {
    if (drift) rc = launch_drift(Q, static_cast<long>(p.H) * p.L * p.d, drift->seed, t, drift->amplitude,
                                 drift->q_step, st);
    if (rc != SPARSED_OK) break;
    switch (kinds[t]) {
      case SPARSED_STEP_DENSE:
        rc = launch_attn(p, false, nullptr, nullptr, 0, st, nullptr, nullptr, &ps);
        if (rc == SPARSED_OK && fused && t + 1 < end_step && kinds[t + 1] == SPARSED_STEP_SELECT) {
          rc = save_lse(p, workspace, st);
          have_lse = true;
        }
        break;
      case SPARSED_STEP_SELECT:
        if (fused && have_lse) {
          rc = fused_select(p, keep_ratio, budget_mode, kv_idx, kv_count, kv_stride, workspace, &ps, st);
        } else {
          rc = launch_attn(p, false, nullptr, nullptr, 0, st, nullptr, nullptr, &ps);
          if (rc == SPARSED_OK)
            rc = select_after_dense(p, keep_ratio, budget_mode, kv_idx, kv_count, kv_stride, nullptr,
                                    nullptr, workspace, st);
        }
        if (rc == SPARSED_OK && fused) {
          rc = save_lse(p, workspace, st);
          have_lse = true;
        }
        break;
      default:
        rc = launch_attn(p, true, kv_idx, kv_count, kv_stride, st);
        break;
    }
    if (!ev.empty() && rc == SPARSED_OK) {
      cudaError_t e = cudaEventRecord(ev[t - start_step + 1], st);
      if (e != cudaSuccess) rc = fail_cuda(e);
    }
  }
  if (!ev.empty()) {
    if (rc == SPARSED_OK) {
      cudaError_t e = cudaEventSynchronize(ev.back());
      if (e != cudaSuccess) rc = fail_cuda(e);
      for (int t = start_step; t < end_step && rc == SPARSED_OK; ++t) {
        float ms = 0.f;
        e = cudaEventElapsedTime(&ms, ev[t - start_step], ev[t - start_step + 1]);
        if (e != cudaSuccess) rc = fail_cuda(e);
        step_ms[t] = ms;
      }
    }
    for (auto& e : ev)
      if (e) cudaEventDestroy(e);
  }
  return rc;
}

}  // namespace

extern "C" {

// ---- head-sharded entropy budget (the heads of one layer split over ranks)

int sparsed_entropy_budget(const double* head_entropy, int H, int nkb, float keep_ratio, int32_t* head_k) {
  if (!head_entropy || !head_k || H < 1 || nkb < 1 || !(keep_ratio > 0.f && keep_ratio <= 1.f))
    return SPARSED_ERR_INVALID_ARG;
  std::vector<double> scratch(static_cast<size_t>(H) * 3);
  allocate_budget(head_entropy, H, nkb, keep_ratio, scratch.data(), scratch.data() + H, scratch.data() + 2 * H,
                  head_k);
  return SPARSED_OK;
}

int sparsed_select_head_entropy(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int H, int L, int d,
                                float scale, int bq, int bk, uint16_t* O, float* LSE, double* head_entropy,
                                void* workspace, size_t workspace_bytes, void* stream) {
  Problem p;
  bool empty = false;
  SP_TRY(prepare(Q, K, V, H, L, d, scale, bq, bk, O, LSE, &p, &empty));
  if (empty) return SPARSED_OK;
  if (!head_entropy) return SPARSED_ERR_INVALID_ARG;
  if (static_cast<long long>(p.H) * p.nqb * p.nkb >= (1ll << 31)) return SPARSED_ERR_UNSUPPORTED;
  const Workspace w = ws_layout(p.H, p.nqb, p.nkb);
  if (!workspace || workspace_bytes < w.total) return SPARSED_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SPARSED_ERR_WORKSPACE;
  SP_TRY(require_sm100());
  SP_TRY(get_encoder());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* mass = reinterpret_cast<float*>(ws + w.grid);
  double* ent = reinterpret_cast<double*>(ws + w.ent);
  SP_TRY(dense_pass_counted(p, ws + w.sched, st));
  SP_TRY(launch_mass(p, mass, st));
  const int rows = p.H * p.nqb;
  row_entropy_kernel<<<(rows + 7) / 8, 256, 0, st>>>(mass, rows, p.nkb, ent);
  SP_CUDA(cudaGetLastError());
  head_entropy_kernel<<<(p.H + 255) / 256, 256, 0, st>>>(ent, p.H, p.nqb, head_entropy);
  SP_CUDA(cudaGetLastError());
  return SPARSED_OK;
}

int sparsed_select_with_head_k(int H, int L, int bq, int bk, const int32_t* head_k, int32_t* kv_idx,
                               int32_t* kv_count, int kv_stride, void* workspace, size_t workspace_bytes,
                               void* stream) {
  if (H < 0 || L < 0) return SPARSED_ERR_INVALID_ARG;
  if ((bq != 64 && bq != 128) || (bk != 64 && bk != 128)) return SPARSED_ERR_UNSUPPORTED;
  if (static_cast<long>(H) * L == 0) return SPARSED_OK;
  const int nqb = static_cast<int>(cdiv(L, bq)), nkb = static_cast<int>(cdiv(L, bk));
  if (!head_k || !kv_idx || !kv_count || kv_stride < nkb) return SPARSED_ERR_INVALID_ARG;
  if (static_cast<long long>(H) * nqb * kv_stride >= (1ll << 31)) return SPARSED_ERR_UNSUPPORTED;
  const Workspace w = ws_layout(H, nqb, nkb);
  if (!workspace || workspace_bytes < w.total) return SPARSED_ERR_WORKSPACE;
  SP_TRY(require_sm100());
  const float* mass = reinterpret_cast<const float*>(static_cast<uint8_t*>(workspace) + w.grid);
  const int rows = H * nqb;
  topk_kernel<<<(rows + 7) / 8, 256, 0, static_cast<cudaStream_t>(stream)>>>(mass, rows, nqb, nkb, 0, head_k,
                                                                              nullptr, kv_idx, kv_count, kv_stride);
  SP_CUDA(cudaGetLastError());
  return SPARSED_OK;
}

int sparsed_run_steps_sharded(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int H, int L, int d,
                              float scale, int bq, int bk, float keep_ratio, int budget_mode, int h_total,
                              int head_offset, int T, float warmup_frac, int refresh_every, int32_t* kv_idx,
                              int32_t* kv_count, int kv_stride, uint16_t* O, float* LSE, int8_t* step_kind,
                              sparsed_exchange_fn exchange, void* user, void* workspace, size_t workspace_bytes,
                              void* stream) {
  if (h_total < H || head_offset < 0 || head_offset > h_total - H || T < 0) return SPARSED_ERR_INVALID_ARG;
  if (budget_mode == SPARSED_BUDGET_UNIFORM)
    return run_steps_impl(Q, K, V, H, L, d, scale, bq, bk, keep_ratio, budget_mode, T, warmup_frac, refresh_every,
                          0, T, 0, kv_idx, kv_count, kv_stride, O, LSE, step_kind, nullptr, workspace,
                          workspace_bytes, stream, nullptr);
  if (budget_mode != SPARSED_BUDGET_ENTROPY || !exchange) return SPARSED_ERR_INVALID_ARG;
  if (!(keep_ratio > 0.f && keep_ratio <= 1.f)) return SPARSED_ERR_INVALID_ARG;
  std::vector<int8_t> kinds(static_cast<size_t>(T) + 1);
  SP_TRY(sparsed_schedule(T, warmup_frac, refresh_every, kinds.data()));
  if (step_kind && T > 0) std::memcpy(step_kind, kinds.data(), static_cast<size_t>(T));
  Problem p;
  bool empty = false;
  SP_TRY(prepare(Q, K, V, H, L, d, scale, bq, bk, O, LSE, &p, &empty));
  if (empty) return SPARSED_OK;
  SP_TRY(check_select_args(p, keep_ratio, budget_mode, kv_idx, kv_count, kv_stride, workspace, workspace_bytes));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Workspace w = ws_layout(p.H, p.nqb, p.nkb);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  double* ent_dev = reinterpret_cast<double*>(ws + w.scratch);  // H doubles of the budget scratch
  int32_t* k_dev = reinterpret_cast<int32_t*>(ws + w.headk);
  std::vector<double> ent_local(static_cast<size_t>(H)), ent_all(static_cast<size_t>(h_total));
  std::vector<double> scratch(static_cast<size_t>(h_total) * 3);
  std::vector<int32_t> k_all(static_cast<size_t>(h_total));
  bool have_pattern = false;
  int t0 = 0;
  for (int t = 0; t <= T; ++t) {
    if (t < T && kinds[t] != SPARSED_STEP_SELECT) continue;
    if (t > t0)  // the steps before this SELECT (or the end): no selection among them
      SP_TRY(run_steps_impl(Q, K, V, H, L, d, scale, bq, bk, keep_ratio, budget_mode, T, warmup_frac,
                            refresh_every, t0, t, have_pattern ? 1 : 0, kv_idx, kv_count, kv_stride, O, LSE,
                            nullptr, nullptr, workspace, workspace_bytes, stream, nullptr));
    if (t == T) break;
    SP_TRY(sparsed_select_head_entropy(Q, K, V, H, L, d, scale, bq, bk, O, LSE, ent_dev, workspace,
                                       workspace_bytes, stream));
    SP_CUDA(cudaMemcpyAsync(ent_local.data(), ent_dev, static_cast<size_t>(H) * sizeof(double),
                            cudaMemcpyDeviceToHost, st));
    SP_CUDA(cudaStreamSynchronize(st));
    if (exchange(ent_local.data(), H, ent_all.data(), h_total, user) != 0) return SPARSED_ERR_EXCHANGE;
    allocate_budget(ent_all.data(), h_total, p.nkb, keep_ratio, scratch.data(), scratch.data() + h_total,
                    scratch.data() + 2 * h_total, k_all.data());
    SP_CUDA(cudaMemcpyAsync(k_dev, k_all.data() + head_offset, static_cast<size_t>(H) * sizeof(int32_t),
                            cudaMemcpyHostToDevice, st));
    SP_TRY(sparsed_select_with_head_k(H, L, bq, bk, k_dev, kv_idx, kv_count, kv_stride, workspace, workspace_bytes,
                                      stream));
    // k_all is reused at the next selection only after this one's copy has run
    SP_CUDA(cudaStreamSynchronize(st));
    have_pattern = true;
    t0 = t + 1;
  }
  return SPARSED_OK;
}

int sparsed_column_keep(int L, float keep_ratio, int* kc) {
  if (!kc || L < 1 || !(keep_ratio > 0.f && keep_ratio <= 1.f)) return SPARSED_ERR_INVALID_ARG;
  *kc = uniform_k(L, keep_ratio);
  return SPARSED_OK;
}

int sparsed_column_workspace_bytes(int H, int L, int d, int kc, size_t* bytes) {
  if (!bytes || H < 0 || L < 0 || kc < 0 || kc > L) return SPARSED_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SPARSED_ERR_UNSUPPORTED;
  *bytes = col_ws_layout(H, L, d, kc).total;
  return SPARSED_OK;
}

int sparsed_select_columns(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int H, int L, int d,
                           float scale, int bq, int bk, float keep_ratio, uint16_t* O, float* LSE, int32_t* cols,
                           int col_stride, float* col_mass, void* workspace, size_t workspace_bytes, void* stream) {
  Problem p;
  bool empty = false;
  SP_TRY(prepare(Q, K, V, H, L, d, scale, bq, bk, O, LSE, &p, &empty));
  if (empty) return SPARSED_OK;
  if (!(keep_ratio > 0.f && keep_ratio <= 1.f)) return SPARSED_ERR_INVALID_ARG;
  const int kc = uniform_k(L, keep_ratio);
  SP_TRY(check_column_args(p, kc, cols, col_stride, workspace, workspace_bytes));
  SP_TRY(require_sm100());
  SP_TRY(get_encoder());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SP_TRY(dense_pass_counted(p, static_cast<uint8_t*>(workspace) + col_ws_layout(p.H, p.L, p.d, kc).sched, st));
  return select_columns_after_dense(p, kc, cols, col_stride, col_mass, workspace, st);
}

int sparsed_column_sparse_attn(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int H, int L, int d,
                               float scale, int bq, int bk, const int32_t* cols, int kc, int col_stride,
                               uint16_t* O, float* LSE, void* workspace, size_t workspace_bytes, void* stream) {
  Problem p;
  bool empty = false;
  SP_TRY(prepare(Q, K, V, H, L, d, scale, bq, bk, O, LSE, &p, &empty));
  if (empty) return SPARSED_OK;
  SP_TRY(check_column_args(p, kc, cols, col_stride, workspace, workspace_bytes));
  SP_TRY(require_sm100());
  SP_TRY(get_encoder());
  return column_attn(p, cols, kc, col_stride, workspace, static_cast<cudaStream_t>(stream));
}

int sparsed_run_steps_columns(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int H, int L, int d,
                              float scale, int bq, int bk, float keep_ratio, int T, float warmup_frac,
                              int refresh_every, int start_step, int have_pattern, int32_t* cols, int col_stride,
                              uint16_t* O, float* LSE, int8_t* step_kind, float* step_ms, void* workspace,
                              size_t workspace_bytes, void* stream) {
  if (T < 0 || start_step < 0 || start_step > T) return SPARSED_ERR_INVALID_ARG;
  if (!(keep_ratio > 0.f && keep_ratio <= 1.f)) return SPARSED_ERR_INVALID_ARG;
  std::vector<int8_t> kinds(static_cast<size_t>(T) + 1);
  SP_TRY(sparsed_schedule(T, warmup_frac, refresh_every, kinds.data()));
  if (step_kind && T > 0) std::memcpy(step_kind, kinds.data(), static_cast<size_t>(T));
  if (step_ms)
    for (int t = 0; t < T; ++t) step_ms[t] = 0.f;
  Problem p;
  bool empty = false;
  SP_TRY(prepare(Q, K, V, H, L, d, scale, bq, bk, O, LSE, &p, &empty));
  if (empty) return SPARSED_OK;
  bool pattern_ready = have_pattern != 0;
  for (int t = start_step; t < T; ++t) {
    if (kinds[t] == SPARSED_STEP_SELECT) pattern_ready = true;
    if (kinds[t] == SPARSED_STEP_SPARSE && !pattern_ready) return SPARSED_ERR_INVALID_ARG;
  }
  const int kc = uniform_k(L, keep_ratio);
  if (start_step < T) SP_TRY(check_column_args(p, kc, cols, col_stride, workspace, workspace_bytes));
  SP_TRY(require_sm100());
  SP_TRY(get_encoder());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the full passes take their pairs from counters in the workspace
  PairSched ps;
  if (start_step < T)
    SP_TRY(begin_pair_sched(&ps, static_cast<uint8_t*>(workspace) + col_ws_layout(p.H, p.L, p.d, kc).sched, st));
  std::vector<cudaEvent_t> ev;
  if (step_ms && start_step < T) {
    ev.resize(static_cast<size_t>(T - start_step) + 1, nullptr);
    for (auto& e : ev) SP_CUDA(cudaEventCreate(&e));
    SP_CUDA(cudaEventRecord(ev[0], st));
  }
  int rc = SPARSED_OK;
  for (int t = start_step; t < T && rc == SPARSED_OK; ++t) {
    switch (kinds[t]) {
      case SPARSED_STEP_DENSE:
        rc = launch_attn(p, false, nullptr, nullptr, 0, st, nullptr, nullptr, &ps);
        break;
      case SPARSED_STEP_SELECT:
        rc = launch_attn(p, false, nullptr, nullptr, 0, st, nullptr, nullptr, &ps);
        if (rc == SPARSED_OK) rc = select_columns_after_dense(p, kc, cols, col_stride, nullptr, workspace, st);
        break;
      default:
        rc = column_attn(p, cols, kc, col_stride, workspace, st);
        break;
    }
    if (!ev.empty() && rc == SPARSED_OK) {
      cudaError_t e = cudaEventRecord(ev[t - start_step + 1], st);
      if (e != cudaSuccess) rc = fail_cuda(e);
    }
  }
  if (!ev.empty()) {
    if (rc == SPARSED_OK) {
      cudaError_t e = cudaEventSynchronize(ev.back());
      if (e != cudaSuccess) rc = fail_cuda(e);
      for (int t = start_step; t < T && rc == SPARSED_OK; ++t) {
        float ms = 0.f;
        e = cudaEventElapsedTime(&ms, ev[t - start_step], ev[t - start_step + 1]);
        if (e != cudaSuccess) rc = fail_cuda(e);
        step_ms[t] = ms;
      }
    }
    for (auto& e : ev)
      if (e) cudaEventDestroy(e);
  }
  return rc;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free pattern selection.
//
// Some callers may not allocate device memory at all: code that runs inside a
// host framework which owns the whole device-memory budget through its own pool
// (a foreign cudaMalloc would bypass its accounting), or latency-critical loops
// where cudaMalloc/cudaFree would implicitly synchronise the device. For them,
// sparsed_select_pattern_noalloc takes no workspace: its scratch (block-mass
// grid, row entropies, budget scratch, per-head k) lives in the fixed-size
// array below, which every GPU that loads this library holds until exit.
//
// The array is shared by every call on a device and keeps the previous call's
// contents. Each call writes every scratch byte it later reads before reading
// it, so nothing has to be cleared between calls. Calls that overlap on the
// GPU (different streams, or several host threads) race on the array.
// ---------------------------------------------------------------------------

static __device__ __align__(256) unsigned char g_noalloc_scratch[SPARSED_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kNoAllocMaxDevices = 64;
struct NoAllocAddr {
  unsigned long long ctx = 0;  // context id (0: slot unused)
  void* addr = nullptr;
};
std::mutex g_noalloc_mu;
NoAllocAddr g_noalloc_addr[kNoAllocMaxDevices];

// Device address of g_noalloc_scratch in the current device's context. In
// host code the array's name is only a host-side stand-in, so the address is
// looked up with cudaGetSymbolAddress, once per context (the first call on a
// device, with that device current), and cached under the context's id: a
// context created after cudaDeviceReset gets its own lookup.
int noalloc_scratch_address(void** out) {
  int dev = 0;
  SP_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kNoAllocMaxDevices) return SPARSED_ERR_UNSUPPORTED;
  unsigned long long ctx = 0;
  SP_TRY(context_id(&ctx));
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoAllocAddr& slot = g_noalloc_addr[dev];
  if (ctx == 0 || slot.ctx != ctx) {
    void* addr = nullptr;
    SP_CUDA(cudaGetSymbolAddress(&addr, g_noalloc_scratch));  // makes the primary context current if none was
    SP_TRY(context_id(&ctx));
    slot.ctx = ctx;
    slot.addr = addr;
  }
  *out = slot.addr;
  return SPARSED_OK;
}

}  // namespace

extern "C" int sparsed_select_pattern_noalloc(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                                              int H, int L, int d, float scale, int bq, int bk,
                                              float keep_ratio, int budget_mode, uint16_t* O, float* LSE,
                                              int32_t* kv_idx, int32_t* kv_count, int kv_stride,
                                              float* block_mass, int32_t* head_k, void* stream) {
  Problem p;
  bool empty = false;
  SP_TRY(prepare(Q, K, V, H, L, d, scale, bq, bk, O, LSE, &p, &empty));
  if (empty) return SPARSED_OK;
  // The whole scratch layout of these sizes must fit in the built-in array.
  if (ws_layout(p.H, p.nqb, p.nkb).total > static_cast<size_t>(SPARSED_NOALLOC_SCRATCH_BYTES))
    return SPARSED_ERR_WORKSPACE;
  SP_TRY(require_sm100());
  void* scratch = nullptr;
  SP_TRY(noalloc_scratch_address(&scratch));
  SP_TRY(check_select_args(p, keep_ratio, budget_mode, kv_idx, kv_count, kv_stride, scratch,
                           static_cast<size_t>(SPARSED_NOALLOC_SCRATCH_BYTES)));
  SP_TRY(get_encoder());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SP_TRY(launch_attn(p, false, nullptr, nullptr, 0, st));
  return select_after_dense(p, keep_ratio, budget_mode, kv_idx, kv_count, kv_stride, block_mass, head_k,
                            scratch, st);
}

// ---- block-wise generation with active-token reuse (LoSA: Locality Aware
// Sparse Attention for Block-Wise Diffusion Language Models, section 3)

namespace {

struct LosaDims {
  int H, B, P, d, bq, bk;
  int nkb;     // prefix key blocks
  int n_sel;   // blocks selected per token, clamped to nkb
  int S;       // splits of a head's block list
  int tiles;   // query tiles of the block: ceil(B / bq)
  int R;       // rows per split: tiles * bq
  int stride;  // kv list row stride: the longest split
};

int losa_dims(int H, int B, int P, int d, int bq, int bk, int n_sel, int splits, LosaDims* g) {
  if (H < 1 || B < 1 || P < 1 || n_sel < 1 || splits < 1) return SPARSED_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SPARSED_ERR_UNSUPPORTED;
  if ((bq != 64 && bq != 128) || (bk != 64 && bk != 128)) return SPARSED_ERR_UNSUPPORTED;
  if (H > 65535 || B > kLosaMaxB) return SPARSED_ERR_UNSUPPORTED;
  const long nkb = cdiv(P, bk);
  if (nkb > static_cast<long>(kLosaMaxWords) * 32) return SPARSED_ERR_UNSUPPORTED;
  if (static_cast<long long>(H) * P * d >= (1ll << 31)) return SPARSED_ERR_UNSUPPORTED;
  g->H = H;
  g->B = B;
  g->P = P;
  g->d = d;
  g->bq = bq;
  g->bk = bk;
  g->nkb = static_cast<int>(nkb);
  g->n_sel = n_sel < g->nkb ? n_sel : g->nkb;
  // a split past ceil(nkb / kLosaMinChunk) could never hold a block; the merge
  // holds one split per lane
  int s_max = static_cast<int>(cdiv(nkb, kLosaMinChunk));
  if (s_max > kLosaMaxSplits) s_max = kLosaMaxSplits;
  g->S = splits < s_max ? splits : s_max;
  g->tiles = static_cast<int>(cdiv(B, bq));
  g->R = g->tiles * bq;
  long stride = cdiv(nkb, g->S);
  if (stride < kLosaMinChunk) stride = kLosaMinChunk;
  if (stride > nkb) stride = nkb;
  g->stride = static_cast<int>(stride);
  if (static_cast<long long>(H) * g->S * g->R * d >= (1ll << 31)) return SPARSED_ERR_UNSUPPORTED;
  if (static_cast<long long>(H) * g->S * g->tiles * g->stride >= (1ll << 31)) return SPARSED_ERR_UNSUPPORTED;
  if (static_cast<long long>(H) * B * nkb >= (1ll << 31)) return SPARSED_ERR_UNSUPPORTED;
  return SPARSED_OK;
}

struct LosaWorkspace {
  size_t active, pos, ucount, uidx, kvc, kvi, qrep, orep, lserep, mass, selcnt, total;
};

LosaWorkspace losa_ws_layout(const LosaDims& g) {
  LosaWorkspace w;
  const size_t items = static_cast<size_t>(g.H) * g.S * g.tiles;
  const size_t rep_rows = static_cast<size_t>(g.H) * g.S * g.R;
  w.active = 0;
  w.pos = w.active + align256(static_cast<size_t>(g.B) * 4);
  w.ucount = w.pos + align256(static_cast<size_t>(g.B) * 4);
  w.uidx = w.ucount + align256(static_cast<size_t>(g.H) * 4);
  w.kvc = w.uidx + align256(static_cast<size_t>(g.H) * g.nkb * 4);
  w.kvi = w.kvc + align256(items * 4);
  w.qrep = w.kvi + align256(items * g.stride * 4);
  w.orep = w.qrep + align256(rep_rows * g.d * 2);
  w.lserep = w.orep + align256(rep_rows * g.d * 2);
  w.mass = w.lserep + align256(rep_rows * 4);
  w.selcnt = w.mass + align256(static_cast<size_t>(g.H) * g.B * g.nkb * 4);
  w.total = w.selcnt + align256(static_cast<size_t>(g.H) * g.B * 4);
  return w;
}

// A second stream per device on which a step's suffix attention (the block
// over its own keys) runs beside the union building and the prefix pass of
// the caller's stream: forked from and joined back to the caller's stream by
// events, so the caller sees one ordered stream (and a graph capture of it
// takes both branches). Created at the first use on a device; the lock keeps
// the fork / join of concurrent callers apart.
struct SideStream {
  unsigned long long ctx = 0;  // id of the context the handles belong to
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  std::mutex mu;
};
constexpr int kSideMaxDevices = 64;
SideStream g_side[kSideMaxDevices];
std::mutex g_side_init_mu;

int side_stream(SideStream** out) {
  int dev = 0;
  SP_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kSideMaxDevices) return SPARSED_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_side_init_mu);
  SideStream& ss = g_side[dev];
  unsigned long long ctx = 0;
  SP_TRY(context_id(&ctx));
  // handles created in a context that has since gone (cudaDeviceReset) are
  // not valid any more: make new ones in the current context
  if (ss.s != nullptr && (ctx == 0 || ss.ctx != ctx)) ss.s = nullptr;
  if (ss.s == nullptr) {
    // all three or none: a failed creation leaves the slot empty for a retry
    cudaStream_t s = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
    cudaError_t e = cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&join, cudaEventDisableTiming);
    if (e != cudaSuccess) {
      if (join) cudaEventDestroy(join);
      if (fork) cudaEventDestroy(fork);
      if (s) cudaStreamDestroy(s);
      return fail_cuda(e);
    }
    SP_TRY(context_id(&ctx));
    ss.ctx = ctx;
    ss.fork = fork;
    ss.join = join;
    ss.s = s;
  }
  *out = &ss;
  return SPARSED_OK;
}

// Fork: the side stream waits for everything issued on st so far. Nothing is
// forked when this fails.
int fork_side(SideStream* side, cudaStream_t st) {
  SP_CUDA(cudaEventRecord(side->fork, st));
  SP_CUDA(cudaStreamWaitEvent(side->s, side->fork, 0));
  return SPARSED_OK;
}

int record_join(SideStream* side) {
  SP_CUDA(cudaEventRecord(side->join, side->s));
  return SPARSED_OK;
}

// Any failure after a fork: record the join on the side stream (best effort;
// it may already be recorded) and make st wait for it, so the caller's stream
// stays ordered after the side work and a stream capture of st never ends
// with the side stream left unjoined. Returns rc.
int rejoin_after_error(SideStream* side, cudaStream_t st, int rc) {
  cudaEventRecord(side->join, side->s);
  cudaStreamWaitEvent(st, side->join, 0);
  return rc;
}

int losa_check_ws(const LosaDims& g, const void* workspace, size_t ws_bytes) {
  if (!workspace || ws_bytes < losa_ws_layout(g).total) return SPARSED_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SPARSED_ERR_WORKSPACE;
  return SPARSED_OK;
}

// The block's own tensors, the prefix cache and the carried state.
int losa_check_ptrs(const void* Q, const void* K, const void* V, const void* Kp, const void* Vp,
                    const void* o_cache, const float* lse_cache, const int32_t* sel, const void* O,
                    const float* LSE) {
  if (!Q || !K || !V || !Kp || !Vp || !o_cache || !lse_cache || !sel || !O || !LSE) return SPARSED_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(Kp) || !aligned16(Vp) || !aligned16(o_cache) ||
      !aligned16(O))
    return SPARSED_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(lse_cache) & 3u) || (reinterpret_cast<uintptr_t>(LSE) & 3u) ||
      (reinterpret_cast<uintptr_t>(sel) & 3u))
    return SPARSED_ERR_INVALID_ARG;
  return SPARSED_OK;
}

// Suffix part: dense attention of the block over its own keys, into O / LSE.
int losa_suffix(const LosaDims& g, const uint16_t* Q, const uint16_t* K, const uint16_t* V, float scale, uint16_t* O,
                float* LSE, cudaStream_t st) {
  Problem p;
  p.Q = Q;
  p.K = K;
  p.V = V;
  p.O = O;
  p.LSE = LSE;
  p.H = g.H;
  p.L = g.B;
  p.d = g.d;
  p.bq = g.bq;
  p.bk = g.bk;
  p.nqb = g.tiles;
  p.nkb = static_cast<int>(cdiv(g.B, g.bk));
  p.Lk = g.B;
  p.scale = scale;
  return launch_attn(p, false, nullptr, nullptr, 0, st);
}

// The union, the split lists and the replicated queries; active == nullptr
// for the first step of a block (every token, every prefix block).
int losa_lists(const LosaDims& g, const int32_t* active, const int32_t* sel, int sel_stride, const uint16_t* Q,
               int32_t* union_idx, int32_t* union_count, uint8_t* ws, cudaStream_t st) {
  const LosaWorkspace w = losa_ws_layout(g);
  LosaListArgs a;
  a.H = g.H;
  a.B = g.B;
  a.d = g.d;
  a.nkb = g.nkb;
  a.n_sel = g.n_sel;
  a.sel_stride = sel_stride;
  a.bq = g.bq;
  a.tiles = g.tiles;
  a.R = g.R;
  a.S = g.S;
  a.kv_stride = g.stride;
  a.active = active;
  a.sel = sel;
  a.q = Q;
  a.pos = reinterpret_cast<int32_t*>(ws + w.pos);
  a.union_idx = union_idx ? union_idx : reinterpret_cast<int32_t*>(ws + w.uidx);
  a.union_count = union_count ? union_count : reinterpret_cast<int32_t*>(ws + w.ucount);
  a.kv_idx = reinterpret_cast<int32_t*>(ws + w.kvi);
  a.kv_count = reinterpret_cast<int32_t*>(ws + w.kvc);
  a.q_rep = reinterpret_cast<uint16_t*>(ws + w.qrep);
  return launch_k(losa_lists_kernel, dim3(g.H), dim3(256), 0, st, true, a);
}

// Prefix pass over the split lists (block-sparse kernel, the replicated
// queries against the prefix cache), then the merge into cache and output.
int losa_prefix_and_merge(const LosaDims& g, const uint16_t* Kp, const uint16_t* Vp, float scale, bool all_active,
                          uint16_t* o_cache, float* lse_cache, uint16_t* O, float* LSE, uint8_t* ws,
                          cudaStream_t st, cudaEvent_t suffix_done = nullptr) {
  const LosaWorkspace w = losa_ws_layout(g);
  Problem p;
  p.Q = reinterpret_cast<const uint16_t*>(ws + w.qrep);
  p.K = Kp;
  p.V = Vp;
  p.O = reinterpret_cast<uint16_t*>(ws + w.orep);
  p.LSE = reinterpret_cast<float*>(ws + w.lserep);
  p.H = g.H;
  p.L = g.S * g.R;
  p.d = g.d;
  p.bq = g.bq;
  p.bk = g.bk;
  p.nqb = g.S * g.tiles;
  p.nkb = g.nkb;
  p.Lk = g.P;
  p.scale = scale;
  const int32_t* kvc = reinterpret_cast<const int32_t*>(ws + w.kvc);
  SP_TRY(launch_attn(p, true, reinterpret_cast<const int32_t*>(ws + w.kvi), kvc, g.stride, st, nullptr, nullptr,
                     nullptr, true));
  if (suffix_done) SP_CUDA(cudaStreamWaitEvent(st, suffix_done, 0));  // the merge reads the suffix part
  LosaMergeArgs m;
  m.H = g.H;
  m.B = g.B;
  m.d = g.d;
  m.S = g.S;
  m.R = g.R;
  m.tiles = g.tiles;
  m.bq = g.bq;
  m.pos = all_active ? nullptr : reinterpret_cast<const int32_t*>(ws + w.pos);
  m.kv_count = kvc;
  m.o_rep = p.O;
  m.lse_rep = p.LSE;
  m.o_cache = o_cache;
  m.lse_cache = lse_cache;
  m.o = O;
  m.lse = LSE;
  const unsigned grid = static_cast<unsigned>(cdiv(static_cast<long>(g.H) * g.B, 8));
  return launch_k(g.d == 64 ? losa_merge_kernel<64> : losa_merge_kernel<128>, dim3(grid), dim3(256), 0, st, true, m);
}

template <int D, int BK>
int launch_tok_mass_t(const LosaDims& g, const uint16_t* Q, const uint16_t* Kp, float scale, const float* lse,
                      float* mass, cudaStream_t st) {
  using C = TokMassCfg<D>;
  CUtensorMap tq, tk;
  SP_TRY(make_map(&tq, Q, g.H, g.B, D, C::M));
  SP_TRY(make_map(&tk, Kp, g.H, g.P, D, C::N));
  TokMassArgs a;
  a.H = g.H;
  a.B = g.B;
  a.P = g.P;
  a.nkb = g.nkb;
  a.tiles_per_cta = 8;
  a.scale_log2 = scale * 1.44269504088896340736f;
  a.lse = lse;
  a.mass = mass;
  a.timeout_ns = kWaitTimeoutNs;
  auto kern = token_block_mass_kernel<D, BK>;
  SP_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES));
  const long ntiles = cdiv(g.P, C::N);
  const dim3 grid(static_cast<unsigned>(cdiv(ntiles, a.tiles_per_cta)), static_cast<unsigned>(g.H),
                  static_cast<unsigned>(cdiv(g.B, C::M)));
  kern<<<grid, 128 + 128 * (C::N / BK), C::SMEM_BYTES, st>>>(tq, tk, a);
  SP_CUDA(cudaGetLastError());
  return SPARSED_OK;
}

int launch_tok_mass(const LosaDims& g, const uint16_t* Q, const uint16_t* Kp, float scale, const float* lse,
                    float* mass, cudaStream_t st) {
  if (g.d == 64 && g.bk == 64) return launch_tok_mass_t<64, 64>(g, Q, Kp, scale, lse, mass, st);
  if (g.d == 64 && g.bk == 128) return launch_tok_mass_t<64, 128>(g, Q, Kp, scale, lse, mass, st);
  if (g.d == 128 && g.bk == 64) return launch_tok_mass_t<128, 64>(g, Q, Kp, scale, lse, mass, st);
  if (g.d == 128 && g.bk == 128) return launch_tok_mass_t<128, 128>(g, Q, Kp, scale, lse, mass, st);
  return SPARSED_ERR_UNSUPPORTED;
}

int losa_init_impl(const LosaDims& g, const uint16_t* Q, const uint16_t* K, const uint16_t* V, const uint16_t* Kp,
                   const uint16_t* Vp, float scale, int sel_stride, uint16_t* o_cache, float* lse_cache,
                   int32_t* sel, uint16_t* O, float* LSE, float* token_mass, uint8_t* ws, cudaStream_t st) {
  const LosaWorkspace w = losa_ws_layout(g);
  SideStream* side = nullptr;
  SP_TRY(side_stream(&side));
  {
    std::lock_guard<std::mutex> lock(side->mu);
    SP_TRY(fork_side(side, st));
    int rc = losa_suffix(g, Q, K, V, scale, O, LSE, side->s);
    if (rc == SPARSED_OK) rc = record_join(side);
    if (rc == SPARSED_OK) rc = losa_lists(g, nullptr, nullptr, sel_stride, Q, nullptr, nullptr, ws, st);
    if (rc == SPARSED_OK)
      rc = losa_prefix_and_merge(g, Kp, Vp, scale, true, o_cache, lse_cache, O, LSE, ws, st, side->join);
    if (rc != SPARSED_OK) return rejoin_after_error(side, st, rc);
  }
  float* mass = token_mass ? token_mass : reinterpret_cast<float*>(ws + w.mass);
  SP_TRY(launch_tok_mass(g, Q, Kp, scale, lse_cache, mass, st));
  const int rows = g.H * g.B;
  if (g.n_sel <= 32)
    topk_small_kernel<<<(rows + 7) / 8, 256, 0, st>>>(mass, rows, g.nkb, g.n_sel, sel, sel_stride);
  else
    topk_kernel<<<(rows + 7) / 8, 256, 0, st>>>(mass, rows, g.B, g.nkb, g.n_sel, nullptr, nullptr, sel,
                                               reinterpret_cast<int32_t*>(ws + w.selcnt), sel_stride);
  SP_CUDA(cudaGetLastError());
  return SPARSED_OK;
}

int losa_step_impl(const LosaDims& g, const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                   const uint16_t* Q_prev, const uint16_t* Kp, const uint16_t* Vp, float scale, float tau,
                   int sel_stride, uint16_t* o_cache, float* lse_cache, const int32_t* sel, uint16_t* O,
                   float* LSE, int32_t* active, int32_t* union_idx, int32_t* union_count, uint8_t* ws,
                   cudaStream_t st) {
  const LosaWorkspace w = losa_ws_layout(g);
  int32_t* act = active ? active : reinterpret_cast<int32_t*>(ws + w.active);
  SideStream* side = nullptr;
  SP_TRY(side_stream(&side));
  std::lock_guard<std::mutex> lock(side->mu);
  SP_TRY(fork_side(side, st));
  int rc = losa_suffix(g, Q, K, V, scale, O, LSE, side->s);
  if (rc == SPARSED_OK) rc = record_join(side);
  if (rc == SPARSED_OK) {
    query_mse_kernel<<<g.B, 256, 0, st>>>(Q, Q_prev, g.H, g.B, g.d, static_cast<double>(tau), act);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) rc = fail_cuda(e);
  }
  if (rc == SPARSED_OK) rc = losa_lists(g, act, sel, sel_stride, Q, union_idx, union_count, ws, st);
  if (rc == SPARSED_OK)
    rc = losa_prefix_and_merge(g, Kp, Vp, scale, false, o_cache, lse_cache, O, LSE, ws, st, side->join);
  if (rc != SPARSED_OK) return rejoin_after_error(side, st, rc);
  return rc;
}

int losa_prepare(int H, int B, int P, int d, int bq, int bk, int n_sel, int splits, float scale, LosaDims* g) {
  SP_TRY(losa_dims(H, B, P, d, bq, bk, n_sel, splits, g));
  if (!std::isfinite(scale)) return SPARSED_ERR_INVALID_ARG;
  return SPARSED_OK;
}

}  // namespace

extern "C" {

int sparsed_losa_splits(int H, int B, int bq, int P, int bk, int sm_count, int* splits) {
  if (!splits || H < 1 || B < 1 || P < 1 || sm_count < 1) return SPARSED_ERR_INVALID_ARG;
  if ((bq != 64 && bq != 128) || (bk != 64 && bk != 128)) return SPARSED_ERR_UNSUPPORTED;
  const long per_split = static_cast<long>(H) * cdiv(B, bq);  // work items of one split
  long s = sm_count / per_split;
  if (s < 1) s = 1;
  long s_max = cdiv(cdiv(P, bk), kLosaMinChunk);
  if (s_max > kLosaMaxSplits) s_max = kLosaMaxSplits;
  if (s > s_max) s = s_max;
  *splits = static_cast<int>(s);
  return SPARSED_OK;
}

int sparsed_losa_workspace_bytes(int H, int B, int P, int d, int bq, int bk, int splits, size_t* bytes) {
  if (!bytes) return SPARSED_ERR_INVALID_ARG;
  LosaDims g;
  SP_TRY(losa_dims(H, B, P, d, bq, bk, 1, splits, &g));
  *bytes = losa_ws_layout(g).total;
  return SPARSED_OK;
}

int sparsed_losa_init(const uint16_t* Q, const uint16_t* K, const uint16_t* V, const uint16_t* K_prefix,
                      const uint16_t* V_prefix, int H, int B, int P, int d, float scale, int bq, int bk,
                      int n_sel, int splits, uint16_t* o_cache, float* lse_cache, int32_t* sel, uint16_t* O,
                      float* LSE, float* token_mass, void* workspace, size_t workspace_bytes, void* stream) {
  LosaDims g;
  SP_TRY(losa_prepare(H, B, P, d, bq, bk, n_sel, splits, scale, &g));
  SP_TRY(losa_check_ptrs(Q, K, V, K_prefix, V_prefix, o_cache, lse_cache, sel, O, LSE));
  if (token_mass && (reinterpret_cast<uintptr_t>(token_mass) & 3u)) return SPARSED_ERR_INVALID_ARG;
  SP_TRY(losa_check_ws(g, workspace, workspace_bytes));
  SP_TRY(require_sm100());
  SP_TRY(get_encoder());
  return losa_init_impl(g, Q, K, V, K_prefix, V_prefix, scale, n_sel, o_cache, lse_cache, sel, O, LSE, token_mass,
                        static_cast<uint8_t*>(workspace), static_cast<cudaStream_t>(stream));
}

int sparsed_losa_step(const uint16_t* Q, const uint16_t* K, const uint16_t* V, const uint16_t* Q_prev,
                      const uint16_t* K_prefix, const uint16_t* V_prefix, int H, int B, int P, int d, float scale,
                      int bq, int bk, int n_sel, float tau, int splits, uint16_t* o_cache, float* lse_cache,
                      const int32_t* sel, uint16_t* O, float* LSE, int32_t* active, int32_t* union_idx,
                      int32_t* union_count, void* workspace, size_t workspace_bytes, void* stream) {
  LosaDims g;
  SP_TRY(losa_prepare(H, B, P, d, bq, bk, n_sel, splits, scale, &g));
  SP_TRY(losa_check_ptrs(Q, K, V, K_prefix, V_prefix, o_cache, lse_cache, sel, O, LSE));
  if (!Q_prev || !aligned16(Q_prev)) return SPARSED_ERR_INVALID_ARG;
  if (!std::isfinite(tau) || tau < 0.f) return SPARSED_ERR_INVALID_ARG;
  // the optional int32 outputs are stored by the kernels as int32
  for (const int32_t* ptr : {static_cast<const int32_t*>(active), static_cast<const int32_t*>(union_idx),
                             static_cast<const int32_t*>(union_count)})
    if (ptr && (reinterpret_cast<uintptr_t>(ptr) & 3u)) return SPARSED_ERR_INVALID_ARG;
  SP_TRY(losa_check_ws(g, workspace, workspace_bytes));
  SP_TRY(require_sm100());
  SP_TRY(get_encoder());
  return losa_step_impl(g, Q, K, V, Q_prev, K_prefix, V_prefix, scale, tau, n_sel, o_cache, lse_cache, sel, O, LSE,
                        active, union_idx, union_count, static_cast<uint8_t*>(workspace),
                        static_cast<cudaStream_t>(stream));
}

int sparsed_losa_block(const uint16_t* Qs, const uint16_t* Ks, const uint16_t* Vs, const uint16_t* K_prefix,
                       const uint16_t* V_prefix, int T, int H, int B, int P, int d, float scale, int bq, int bk,
                       int n_sel, float tau, int splits, uint16_t* o_cache, float* lse_cache, int32_t* sel,
                       uint16_t* Os, float* LSEs, int32_t* actives, int32_t* union_counts, void* workspace,
                       size_t workspace_bytes, void* stream) {
  if (T < 1) return SPARSED_ERR_INVALID_ARG;
  LosaDims g;
  SP_TRY(losa_prepare(H, B, P, d, bq, bk, n_sel, splits, scale, &g));
  SP_TRY(losa_check_ptrs(Qs, Ks, Vs, K_prefix, V_prefix, o_cache, lse_cache, sel, Os, LSEs));
  if (!std::isfinite(tau) || tau < 0.f) return SPARSED_ERR_INVALID_ARG;
  if ((actives && (reinterpret_cast<uintptr_t>(actives) & 3u)) ||
      (union_counts && (reinterpret_cast<uintptr_t>(union_counts) & 3u)))
    return SPARSED_ERR_INVALID_ARG;
  SP_TRY(losa_check_ws(g, workspace, workspace_bytes));
  SP_TRY(require_sm100());
  SP_TRY(get_encoder());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t blk = static_cast<size_t>(H) * B * d;  // elements of one step's Q, K, V or O
  const size_t rows = static_cast<size_t>(H) * B;
  SP_TRY(losa_init_impl(g, Qs, Ks, Vs, K_prefix, V_prefix, scale, n_sel, o_cache, lse_cache, sel, Os, LSEs, nullptr,
                        ws, st));
  // step 0: every token active, every prefix block read
  if (actives) {
    fill_i32_kernel<<<static_cast<unsigned>(cdiv(B, 256)), 256, 0, st>>>(actives, B, 1);
    SP_CUDA(cudaGetLastError());
  }
  if (union_counts) {
    fill_i32_kernel<<<static_cast<unsigned>(cdiv(H, 256)), 256, 0, st>>>(union_counts, H, g.nkb);
    SP_CUDA(cudaGetLastError());
  }
  for (int t = 1; t < T; ++t) {
    SP_TRY(losa_step_impl(g, Qs + t * blk, Ks + t * blk, Vs + t * blk, Qs + (t - 1) * blk, K_prefix, V_prefix, scale,
                          tau, n_sel, o_cache, lse_cache, sel, Os + t * blk, LSEs + t * rows,
                          actives ? actives + static_cast<size_t>(t) * B : nullptr, nullptr,
                          union_counts ? union_counts + static_cast<size_t>(t) * H : nullptr, ws, st));
  }
  return SPARSED_OK;
}

}  // extern "C"
