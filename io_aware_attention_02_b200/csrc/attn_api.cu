// C ABI of libattn_sm100.so (declared in include/attn.h): argument
// validation, TMA descriptor construction, kernel selection and launch.
// Host code only marshals; every step of the attention runs in the kernels.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cuda.h>
#include <cuda_runtime.h>
#include <mutex>

#include "../../include/attn.h"
#include "bwd_fused_sm100.cuh"
#include "bwd_sm100.cuh"
#include "fwd256_sm100.cuh"
#include "fwd_sm100.cuh"
#include "quant_fp8.cuh"
#include "splitkv_sm100.cuh"

namespace {

constexpr int kMaxDevices = 64;

struct DeviceState {
  int* status = nullptr;  // 4 ints, see ptx.cuh
  int sm_count = 0;
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
int g_fault_mode = 0;
int g_fault_limit_ms = 0;
int g_ablation = 0;   // attn_debug_set_ablation: 1 = serialised tiles in the bf16 d = 128 forward

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Per-device lazily created state: status word and SM count.
attn_status_t device_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState& st = g_dev[dev];
  if (st.status == nullptr) {
    if (cudaDeviceGetAttribute(&st.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return ATTN_ERR_CUDA;
    int* p = nullptr;
    if (cudaMalloc(&p, 4 * sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
    if (cudaMemset(p, 0, 4 * sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
    st.status = p;
  }
  *out = &st;
  return ATTN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Kernel attributes (the dynamic shared-memory opt-in) are set per device:
// each launch helper keeps one flag per device in `done`.  The flags are
// atomic so that calls from several host threads may race on them; the worst
// case is setting the same attribute twice.
using AttrFlags = std::atomic<bool>[kMaxDevices];
bool attr_needed(AttrFlags& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return true;
  return !done[dev].load(std::memory_order_acquire);
}
void attr_mark(AttrFlags& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < kMaxDevices)
    done[dev].store(true, std::memory_order_release);
}

// Element strides of a [B][H][N][d] view over (batch, head, row); the head
// dim is contiguous.
struct Strides {
  long long b, h, n;
};
Strides contiguous(int H, int N, int d) {
  return {static_cast<long long>(H) * N * d, static_cast<long long>(N) * d, d};
}

// Strides TMA can use: positive multiples of 16 bytes, rows not overlapping
// (n >= d).
bool strides_ok(const Strides& s, int d, int esize) {
  const long long a[3] = {s.b, s.h, s.n};
  for (long long x : a)
    if (x <= 0 || (x * esize) % 16 != 0) return false;
  return s.n >= d;
}

// 4-D tiled map over (d, N, H, B) with the given strides: box = (box_cols,
// 128, 1, 1), 128-byte swizzle (64-byte when the box row is 64 bytes);
// out-of-range rows and columns read as zero.
attn_status_t make_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int esize,
                       int B, int H, int N, int D, const Strides& st, int box_cols) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return ATTN_ERR_CUDA;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(st.n) * esize, static_cast<cuuint64_t>(st.h) * esize,
                           static_cast<cuuint64_t>(st.b) * esize};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(box_cols), 128u, 1u, 1u};
  cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  const CUtensorMapSwizzle swz = box_cols * esize == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  CUresult r = enc(map, dt, 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

// 3-D fp32 map over the backward's dQ accumulator [BH][N][d]: box 32 x 32
// rows, 128-byte swizzle (reduce-add target; rows past N are not written).
attn_status_t make_map_dq(CUtensorMap* map, float* base, int BH, int N, int d) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return ATTN_ERR_CUDA;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 4, static_cast<cuuint64_t>(N) * d * 4};
  cuuint32_t box[3] = {32u, 32u, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

unsigned long long wait_limit_ns() {
  static unsigned long long ns = [] {
    const char* e = std::getenv("ATTN_WAIT_LIMIT_MS");
    long ms = e ? std::strtol(e, nullptr, 10) : 0;
    if (ms <= 0) ms = 1000;
    return static_cast<unsigned long long>(ms) * 1000000ull;
  }();
  return ns;
}

attn_status_t common_checks(int B, int H, int N, float scale, int causal) {
  if (B < 1 || H < 1 || N < 1) return ATTN_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H * N >= (1ll << 31)) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

// Work distribution (see sched_unit / decode_unit in fwd_sm100.cuh):
// `n_blocks` row blocks per head, `grid` persistent CTAs, `kv_bytes` the K
// and V of all heads.  Longest first across heads (order 1) puts every head
// in flight at once; that pays while their K and V stay near L2 size (about
// 300 MB: 126 MB of L2 plus the reuse within a round), measured at 2K-8K
// tokens, and loses to longest first within each head beyond it (32K).
void set_schedule(attn::FwdParams* p, int causal, int n_blocks, int grid, double kv_bytes) {
  p->snake = causal ? 1 : 0;
  p->order = (causal && n_blocks < grid && kv_bytes <= 300e6) ? 1 : 0;
}

double kv_bytes_of(int BH, int N, int d, int esize) { return 2.0 * BH * N * d * esize; }

template <typename E, int D, bool CAUSAL, bool VT = false, bool SERIAL = false>
attn_status_t launch_fwd(const attn::FwdParams& p, int grid, cudaStream_t stream) {
  using Cfg = attn::FwdCfg<E, D>;
  auto kern = attn::attn_fwd_sm100_kernel<E, D, CAUSAL, VT, SERIAL>;
  static AttrFlags attr_done;  // per instance and device
  if (attr_needed(attr_done)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes) !=
        cudaSuccess)
      return ATTN_ERR_CUDA;
    attr_mark(attr_done);
  }
  kern<<<grid, Cfg::kThreads, Cfg::kSmemBytes, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <typename E, int D>
attn_status_t launch_fwd_c(const attn::FwdParams& p, int grid, int causal, cudaStream_t s) {
  return causal ? launch_fwd<E, D, true>(p, grid, s) : launch_fwd<E, D, false>(p, grid, s);
}

// Head dim 256: one 128-row Q tile per work unit (n_qpairs then counts
// 128-row tiles).
template <typename E, bool CAUSAL>
attn_status_t launch_fwd256(attn::FwdParams p, int sm_count, cudaStream_t stream) {
  using Cfg = attn::Fwd256Cfg<E>;
  auto kern = attn::attn_fwd_sm100_d256_kernel<E, CAUSAL>;
  static AttrFlags attr_done;
  if (attr_needed(attr_done)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes) !=
        cudaSuccess)
      return ATTN_ERR_CUDA;
    attr_mark(attr_done);
  }
  p.n_qpairs = (p.N + 127) / 128;
  p.n_units = p.BH * p.n_qpairs;
  const int grid = p.n_units < sm_count ? p.n_units : sm_count;
  set_schedule(&p, CAUSAL ? 1 : 0, p.n_qpairs, grid, kv_bytes_of(p.BH, p.N, 256, Cfg::kBytes));
  kern<<<grid, Cfg::kThreads, Cfg::kSmemBytes, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

// Hands the one-shot test hook (attn_debug_set_fault) to a launch and
// resets it.
void take_fault_hook(attn::FwdParams* p) {
  std::lock_guard<std::mutex> lock(g_mu);
  p->fault = g_fault_mode;
  if (g_fault_mode != 0 && g_fault_limit_ms > 0)
    p->wait_limit_ns = static_cast<unsigned long long>(g_fault_limit_ms) * 1000000ull;
  g_fault_mode = 0;
  g_fault_limit_ms = 0;
}

// Fills the fields shared by the 16-bit and FP8 launches.
attn_status_t fill_common(attn::FwdParams* p, DeviceState* st, float* lse, void* o, int BH, int H,
                          int N, float scale) {
  p->o = o;
  p->lse = lse;
  p->status = st->status;
  p->BH = BH;
  p->N = N;
  p->H = H;
  p->o_sb = p->o_sh = p->o_sn = 0;   // O strides: set by each caller
  p->n_kv = (N + 127) / 128;
  p->n_qpairs = (N + 255) / 256;
  p->n_units = BH * p->n_qpairs;
  p->scale_log2 = scale * 1.4426950408889634f;
  p->wait_limit_ns = wait_limit_ns();
  take_fault_hook(p);
  return ATTN_OK;
}

bool ablation_on() {
  std::lock_guard<std::mutex> lock(g_mu);
  return g_ablation != 0;
}

// 16-bit forward over strided [B][H][N][d] views (head dim contiguous).
attn_status_t fwd16(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                    int N, int d, const Strides& sq, const Strides& sk, const Strides& sv,
                    const Strides& so, float scale, int causal, int dtype, void* stream) {
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return ATTN_ERR_INVALID_ARG;
  attn_status_t r = common_checks(B, H, N, scale, causal);
  if (r != ATTN_OK) return r;
  if (d < 1) return ATTN_ERR_INVALID_ARG;
  // any multiple of 8 up to 256 (16-byte rows for TMA); run as 64, 128 or 256
  if (d > 256 || (d % 8) != 0) return ATTN_ERR_UNSUPPORTED;
  const int dk = d <= 64 ? 64 : (d <= 128 ? 128 : 256);
  if (dtype != ATTN_BF16 && dtype != ATTN_FP16) return ATTN_ERR_UNSUPPORTED;
  if (!strides_ok(sq, d, 2) || !strides_ok(sk, d, 2) || !strides_ok(sv, d, 2) || !strides_ok(so, d, 2))
    return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_MISALIGNED;
  if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return ATTN_ERR_MISALIGNED;

  DeviceState* st = nullptr;
  if ((r = device_state(&st)) != ATTN_OK) return r;

  const int BH = B * H;
  const CUtensorMapDataType dt =
      dtype == ATTN_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  attn::FwdParams p{};
  if ((r = make_map(&p.tm_q, q, dt, 2, B, H, N, d, sq, 64)) != ATTN_OK) return r;
  if ((r = make_map(&p.tm_k, k, dt, 2, B, H, N, d, sk, 64)) != ATTN_OK) return r;
  if ((r = make_map(&p.tm_v, v, dt, 2, B, H, N, d, sv, 64)) != ATTN_OK) return r;
  fill_common(&p, st, lse, o, BH, H, N, scale);
  p.d_out = d;
  p.o_sb = so.b;
  p.o_sh = so.h;
  p.o_sn = so.n;
  const int grid = p.n_units < st->sm_count ? p.n_units : st->sm_count;
  set_schedule(&p, causal, p.n_qpairs, grid, kv_bytes_of(BH, N, d, 2));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dk == 256) {
    if (dtype == ATTN_BF16)
      return causal ? launch_fwd256<__nv_bfloat16, true>(p, st->sm_count, s)
                    : launch_fwd256<__nv_bfloat16, false>(p, st->sm_count, s);
    return causal ? launch_fwd256<__half, true>(p, st->sm_count, s)
                  : launch_fwd256<__half, false>(p, st->sm_count, s);
  }
  if (ablation_on()) {   // bench hook: serialised query tiles, bf16 d = 128 only
    if (dtype != ATTN_BF16 || dk != 128) return ATTN_ERR_UNSUPPORTED;
    return causal ? launch_fwd<__nv_bfloat16, 128, true, false, true>(p, grid, s)
                  : launch_fwd<__nv_bfloat16, 128, false, false, true>(p, grid, s);
  }
  if (dtype == ATTN_BF16)
    return dk == 64 ? launch_fwd_c<__nv_bfloat16, 64>(p, grid, causal, s)
                    : launch_fwd_c<__nv_bfloat16, 128>(p, grid, causal, s);
  return dk == 64 ? launch_fwd_c<__half, 64>(p, grid, causal, s)
                  : launch_fwd_c<__half, 128>(p, grid, causal, s);
}

// Backward: the dQ kernel (which also writes the row statistics) then the
// dK/dV kernel, on the same stream and the same persistent grid shape.
template <typename E, int D, bool CAUSAL>
attn_status_t launch_bwd(attn::BwdParams p, int sm_count, cudaStream_t stream) {
  using Cfg = attn::BwdCfg<D>;
  auto kq = attn::attn_bwd_dq_kernel<E, D, CAUSAL>;
  auto kkv = attn::attn_bwd_dkdv_kernel<E, D, CAUSAL>;
  static AttrFlags attr_done;
  if (attr_needed(attr_done)) {
    if (cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kDqSmem) != cudaSuccess ||
        cudaFuncSetAttribute(kkv, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kKvSmem) != cudaSuccess)
      return ATTN_ERR_CUDA;
    attr_mark(attr_done);
  }
  p.n_units = p.BH * p.n_t;
  const int grid = p.n_units < sm_count ? p.n_units : sm_count;
  p.snake = CAUSAL ? 1 : 0;
  p.order = (CAUSAL && p.n_t < grid) ? 1 : 0;
  kq<<<grid, Cfg::kThreads, Cfg::kDqSmem, stream>>>(p);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  kkv<<<grid, Cfg::kThreads, Cfg::kKvSmem, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <typename E, int D>
attn_status_t launch_bwd_c(const attn::BwdParams& p, int sm_count, int causal, cudaStream_t s) {
  return causal ? launch_bwd<E, D, true>(p, sm_count, s) : launch_bwd<E, D, false>(p, sm_count, s);
}

// Fused path: row statistics, then the fused kernel, then the dQ conversion.
template <typename E, int D, bool CAUSAL>
attn_status_t launch_bwd_fused(attn::BwdParams p, int sm_count, const void* o, const void* d_o,
                               cudaStream_t stream) {
  using Cfg = attn::FusedCfg<D>;
  auto kf = attn::attn_bwd_fused_kernel<E, D, CAUSAL>;
  static AttrFlags attr_done;
  if (attr_needed(attr_done)) {
    if (cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem) != cudaSuccess)
      return ATTN_ERR_CUDA;
    attr_mark(attr_done);
  }
  attn::attn_bwd_prep_kernel<E><<<p.BH * p.n_t, 256, 0, stream>>>(
      static_cast<const E*>(o), static_cast<const E*>(d_o), p.lse, p.rows, p.dq_acc, p.N, p.n_t, p.d_out);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  p.n_units = p.BH * p.n_t;
  const int grid = p.n_units < sm_count ? p.n_units : sm_count;
  // causal: longest first within each head (snake rounds), which keeps the
  // Q and dO tiles of the two or three heads in flight in L2 (measured +10 %
  // over longest first across heads at 8K tokens)
  p.snake = CAUSAL ? 1 : 0;
  p.order = 0;
  kf<<<grid, Cfg::kThreads, Cfg::kSmem, stream>>>(p);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  const size_t n8 = static_cast<size_t>(p.BH) * p.N * p.d_out / 8;
  attn::attn_bwd_dq_convert_kernel<E><<<sm_count * 4, 256, 0, stream>>>(p.dq_acc, static_cast<E*>(p.dq), n8,
                                                                        p.scale);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <typename E, int D>
attn_status_t launch_bwd_fused_c(const attn::BwdParams& p, int sm_count, int causal, const void* o,
                                 const void* d_o, cudaStream_t s) {
  return causal ? launch_bwd_fused<E, D, true>(p, sm_count, o, d_o, s)
                : launch_bwd_fused<E, D, false>(p, sm_count, o, d_o, s);
}

// Split-KV forward: split kernel, then the merge.
template <typename E, int D, bool CAUSAL>
attn_status_t launch_splitkv(const attn::SplitParams& p, int grid, void* o, float* lse, cudaStream_t stream) {
  using Cfg = attn::SplitCfg<D>;
  auto kern = attn::attn_splitkv_kernel<E, D, CAUSAL>;
  static AttrFlags attr_done;
  if (attr_needed(attr_done)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem) != cudaSuccess)
      return ATTN_ERR_CUDA;
    attr_mark(attr_done);
  }
  kern<<<grid, Cfg::kThreads, Cfg::kSmem, stream>>>(p);
  if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
  const long long warps = static_cast<long long>(p.BH) * p.Nq;
  attn::attn_splitkv_combine_kernel<E, CAUSAL><<<static_cast<unsigned>((warps + 7) / 8), 256, 0, stream>>>(
      p.o_part, p.lse_part, static_cast<E*>(o), lse, p.BH, p.Nq, p.n_kv, p.n_splits, p.q_off, p.d_out);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <typename E, int D>
attn_status_t launch_splitkv_c(const attn::SplitParams& p, int grid, int causal, void* o, float* lse,
                               cudaStream_t s) {
  return causal ? launch_splitkv<E, D, true>(p, grid, o, lse, s) : launch_splitkv<E, D, false>(p, grid, o, lse, s);
}

size_t splitkv_workspace_bytes(int B, int H, int Nq, int d, int n_splits) {
  const size_t rows = static_cast<size_t>(n_splits) * B * H * Nq;
  return rows * d * sizeof(float) + ((rows * sizeof(float) + 15) / 16) * 16;
}

// Split count when the caller passes 0: the fewest splits (from enough to
// cover the SMs) whose work units fill their last round of CTAs to at least
// 90 %, each split keeping at least two key tiles.
int splitkv_auto_splits(int BH, int n_qt, int n_kv, int sm_count) {
  const long long base = static_cast<long long>(BH) * n_qt;
  const int cap = n_kv / 2 > 1 ? n_kv / 2 : 1;
  int first = static_cast<int>((sm_count + base - 1) / base);
  if (first < 1) first = 1;
  if (first > cap) return cap;
  for (int n = first; n <= cap && n <= 256; ++n) {
    const long long units = base * n;
    const long long rounds = (units + sm_count - 1) / sm_count;
    if (units * 10 >= rounds * sm_count * 9) return n;
  }
  return first;
}

size_t bwd_rows_bytes(int B, int H, int N) {
  return static_cast<size_t>(B) * H * ((N + 127) / 128) * 256 * sizeof(float);
}

size_t bwd_workspace_bytes(int B, int H, int N, int d, int deterministic) {
  size_t b = bwd_rows_bytes(B, H, N);
  if (!deterministic) b += static_cast<size_t>(B) * H * N * d * sizeof(float);
  return b;
}

// Persistent quantiser: kMinBlocks CTAs of 128 threads per SM, each with its
// ring of TMA block loads in dynamic shared memory.
template <int D>
attn_status_t launch_quant(const attn::QuantParams& p, int sm_count, cudaStream_t stream) {
  using C = attn::QuantCfg<D>;
  static AttrFlags attr_done;
  if (attr_needed(attr_done)) {
    if (cudaFuncSetAttribute(attn::attn_quant_fp8_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmem) != cudaSuccess)
      return ATTN_ERR_CUDA;
    attr_mark(attr_done);
  }
  const int grid = p.total < C::kMinBlocks * sm_count ? p.total : C::kMinBlocks * sm_count;
  attn::attn_quant_fp8_kernel<D><<<grid, C::kThreads, C::kSmem, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace

extern "C" {

const char* attn_status_string(attn_status_t s) {
  switch (s) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported head dim or dtype";
    case ATTN_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case ATTN_ERR_CUDA: return "CUDA error";
    case ATTN_ERR_TIMEOUT: return "kernel wait timed out";
    case ATTN_ERR_BOUNDS: return "debug bounds check failed";
  }
  return "unknown status";
}

attn_status_t attn_debug_set_fault(int mode, int wait_limit_ms) {
  if (mode < 0 || mode > 2 || wait_limit_ms < 0) return ATTN_ERR_INVALID_ARG;
  if (mode == 2 && !ATTN_DEBUG_BOUNDS) return ATTN_ERR_UNSUPPORTED;   // the range checks exist in the debug build only
  std::lock_guard<std::mutex> lock(g_mu);
  g_fault_mode = mode;
  g_fault_limit_ms = wait_limit_ms;
  return ATTN_OK;
}

attn_status_t attn_debug_set_ablation(int mode) {
  if (mode < 0 || mode > 1) return ATTN_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_mu);
  g_ablation = mode;
  return ATTN_OK;
}

attn_status_t attn_last_status(void* stream, int* where) {
  DeviceState* st = nullptr;
  attn_status_t r = device_state(&st);
  if (r != ATTN_OK) return r;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_CUDA;
  int h[4] = {0, 0, 0, 0};
  if (cudaMemcpy(h, st->status, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaMemset(st->status, 0, sizeof(h)) != cudaSuccess) return ATTN_ERR_CUDA;
  if (where != nullptr) {
    where[0] = h[1];
    where[1] = h[2];
  }
  if (h[0] == 0) return ATTN_OK;
  if (h[0] == ATTN_ERR_TIMEOUT || h[0] == ATTN_ERR_BOUNDS) return static_cast<attn_status_t>(h[0]);
  return ATTN_ERR_CUDA;
}

attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                       int H, int N, int d, float scale, int causal, int dtype, void* stream) {
  const Strides c = contiguous(H, N, d);
  return fwd16(q, k, v, o, lse, B, H, N, d, c, c, c, c, scale, causal, dtype, stream);
}

attn_status_t attn_fwd_strided(const void* q, const void* k, const void* v, void* o, float* lse,
                               int B, int H, int N, int d, const long long* q_strides,
                               const long long* k_strides, const long long* v_strides,
                               const long long* o_strides, float scale, int causal, int dtype,
                               void* stream) {
  if (q_strides == nullptr || k_strides == nullptr || v_strides == nullptr || o_strides == nullptr)
    return ATTN_ERR_INVALID_ARG;
  const Strides sq{q_strides[0], q_strides[1], q_strides[2]};
  const Strides sk{k_strides[0], k_strides[1], k_strides[2]};
  const Strides sv{v_strides[0], v_strides[1], v_strides[2]};
  const Strides so{o_strides[0], o_strides[1], o_strides[2]};
  return fwd16(q, k, v, o, lse, B, H, N, d, sq, sk, sv, so, scale, causal, dtype, stream);
}

attn_status_t attn_quant_fp8(const void* x, void* x8, float* descale, int B, int H, int N, int d,
                             int hadamard, const float* signs, void* stream) {
  if (x == nullptr || x8 == nullptr || descale == nullptr) return ATTN_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1 || static_cast<long long>(B) * H * N >= (1ll << 31))
    return ATTN_ERR_INVALID_ARG;
  if (hadamard != 0 && hadamard != 1) return ATTN_ERR_INVALID_ARG;
  if (d < 1) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(x8) || (reinterpret_cast<uintptr_t>(descale) & 3u) != 0 ||
      (signs != nullptr && (reinterpret_cast<uintptr_t>(signs) & 3u) != 0))
    return ATTN_ERR_MISALIGNED;
  DeviceState* st = nullptr;
  attn_status_t r = device_state(&st);
  if (r != ATTN_OK) return r;
  attn::QuantParams p{};
  if ((r = make_map(&p.tm_x, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, B, H, N, d, contiguous(H, N, d), 64)) !=
      ATTN_OK)
    return r;
  // codes: one box spans a row of d bytes (64-byte swizzle at d = 64), or
  // half a row at d = 256
  const int box8 = d < 128 ? d : 128;
  if ((r = make_map(&p.tm_x8, x8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, B, H, N, d, contiguous(H, N, d), box8)) !=
      ATTN_OK)
    return r;
  p.descale = descale;
  p.signs = signs;
  p.status = st->status;
  p.wait_limit_ns = wait_limit_ns();
  p.H = H;
  p.N = N;
  p.n_blocks = (N + 127) / 128;
  p.total = p.n_blocks * B * H;
  p.hadamard = hadamard;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 256) return launch_quant<256>(p, st->sm_count, s);
  return d == 64 ? launch_quant<64>(p, st->sm_count, s) : launch_quant<128>(p, st->sm_count, s);
}

attn_status_t attn_fwd_fp8(const void* q8, const void* k8, const void* v8, const float* q_descale,
                           const float* k_descale, const float* v_descale, void* o, float* lse,
                           int B, int H, int N, int d, float scale, int causal, int v_transpose,
                           void* stream) {
  if (q8 == nullptr || k8 == nullptr || v8 == nullptr || o == nullptr || q_descale == nullptr ||
      k_descale == nullptr || v_descale == nullptr)
    return ATTN_ERR_INVALID_ARG;
  attn_status_t r = common_checks(B, H, N, scale, causal);
  if (r != ATTN_OK) return r;
  if (v_transpose != 0 && v_transpose != 1) return ATTN_ERR_INVALID_ARG;
  if (d < 1) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128 && d != 256) return ATTN_ERR_UNSUPPORTED;
  if (v_transpose && d != 128) return ATTN_ERR_UNSUPPORTED;   // the transposer handles 128-byte rows
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8) || !aligned16(o)) return ATTN_ERR_MISALIGNED;
  const uintptr_t a4 = reinterpret_cast<uintptr_t>(q_descale) | reinterpret_cast<uintptr_t>(k_descale) |
                       reinterpret_cast<uintptr_t>(v_descale) |
                       (lse ? reinterpret_cast<uintptr_t>(lse) : 0);
  if ((a4 & 3u) != 0) return ATTN_ERR_MISALIGNED;

  DeviceState* st = nullptr;
  if ((r = device_state(&st)) != ATTN_OK) return r;
  const int BH = B * H;
  attn::FwdParams p{};
  const CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const Strides c8 = contiguous(H, N, d);
  // one box spans a whole e4m3 row of 128 bytes (64-byte swizzle at d = 64),
  // or half a row at d = 256
  const int box = d < 128 ? d : 128;
  if ((r = make_map(&p.tm_q, q8, dt, 1, B, H, N, d, c8, box)) != ATTN_OK) return r;
  if ((r = make_map(&p.tm_k, k8, dt, 1, B, H, N, d, c8, box)) != ATTN_OK) return r;
  if ((r = make_map(&p.tm_v, v8, dt, 1, B, H, N, d, c8, box)) != ATTN_OK) return r;
  p.q_desc = q_descale;
  p.k_desc = k_descale;
  p.v_desc = v_descale;
  fill_common(&p, st, lse, o, BH, H, N, scale);
  p.d_out = d;
  p.o_sb = c8.b;
  p.o_sh = c8.h;
  p.o_sn = c8.n;
  const int grid = p.n_units < st->sm_count ? p.n_units : st->sm_count;
  set_schedule(&p, causal, p.n_qpairs, grid, kv_bytes_of(BH, N, d, 1));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 256)
    return causal ? launch_fwd256<__nv_fp8_e4m3, true>(p, st->sm_count, s)
                  : launch_fwd256<__nv_fp8_e4m3, false>(p, st->sm_count, s);
  if (v_transpose)
    return causal ? launch_fwd<__nv_fp8_e4m3, 128, true, true>(p, grid, s)
                  : launch_fwd<__nv_fp8_e4m3, 128, false, true>(p, grid, s);
  return d == 64 ? launch_fwd_c<__nv_fp8_e4m3, 64>(p, grid, causal, s)
                 : launch_fwd_c<__nv_fp8_e4m3, 128>(p, grid, causal, s);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free variant of attn_fwd (see include/attn.h).  Its scratch, the
// kernel's 16-byte status record, lives in this file-scope device array; host
// code uses the array's device address from cudaGetSymbolAddress, never the
// host-side name.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = 256;
constexpr size_t kNoAllocStatusBytes = 4 * sizeof(int);
static_assert(kNoAllocStatusBytes <= kNoAllocScratchBytes, "status record must fit the scratch array");
static __device__ __align__(256) int g_noalloc_scratch[kNoAllocScratchBytes / sizeof(int)];

struct NoAllocDevice {
  int* scratch = nullptr;  // device address of g_noalloc_scratch on this device
  int sm_count = 0;
};
NoAllocDevice g_noalloc_dev[kMaxDevices];

// Once per device, with that device current: look up the array's address.
attn_status_t noalloc_device(NoAllocDevice** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  NoAllocDevice& st = g_noalloc_dev[dev];
  if (st.scratch == nullptr) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return ATTN_ERR_CUDA;
    int* ptr = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&ptr), g_noalloc_scratch) != cudaSuccess ||
        ptr == nullptr)
      return ATTN_ERR_CUDA;
    st.sm_count = sms;
    st.scratch = ptr;
  }
  *out = &st;
  return ATTN_OK;
}

}  // namespace

extern "C" attn_status_t attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o,
                                          float* lse, int B, int H, int N, int d, float scale,
                                          int causal, int dtype, void* stream) {
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return ATTN_ERR_INVALID_ARG;
  attn_status_t r = common_checks(B, H, N, scale, causal);
  if (r != ATTN_OK) return r;
  if (d < 1) return ATTN_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (dtype != ATTN_BF16 && dtype != ATTN_FP16) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_MISALIGNED;
  if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return ATTN_ERR_MISALIGNED;

  NoAllocDevice* st = nullptr;
  if ((r = noalloc_device(&st)) != ATTN_OK) return r;

  const int BH = B * H;
  const CUtensorMapDataType dt =
      dtype == ATTN_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  attn::FwdParams p{};
  const Strides cs = contiguous(H, N, d);
  if ((r = make_map(&p.tm_q, q, dt, 2, B, H, N, d, cs, 64)) != ATTN_OK) return r;
  if ((r = make_map(&p.tm_k, k, dt, 2, B, H, N, d, cs, 64)) != ATTN_OK) return r;
  if ((r = make_map(&p.tm_v, v, dt, 2, B, H, N, d, cs, 64)) != ATTN_OK) return r;
  p.o = o;
  p.lse = lse;
  p.status = st->scratch;
  p.BH = BH;
  p.H = H;
  p.N = N;
  p.o_sb = cs.b;
  p.o_sh = cs.h;
  p.o_sn = cs.n;
  p.n_kv = (N + 127) / 128;
  p.n_qpairs = (N + 255) / 256;
  p.n_units = BH * p.n_qpairs;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.wait_limit_ns = wait_limit_ns();
  take_fault_hook(&p);
  p.d_out = d;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the record keeps the previous call's contents: it must start at zero
  if (cudaMemsetAsync(st->scratch, 0, kNoAllocStatusBytes, s) != cudaSuccess) return ATTN_ERR_CUDA;
  const int grid = p.n_units < st->sm_count ? p.n_units : st->sm_count;
  set_schedule(&p, causal, p.n_qpairs, grid, kv_bytes_of(BH, N, d, 2));
  if (dtype == ATTN_BF16)
    return d == 64 ? launch_fwd_c<__nv_bfloat16, 64>(p, grid, causal, s)
                   : launch_fwd_c<__nv_bfloat16, 128>(p, grid, causal, s);
  return d == 64 ? launch_fwd_c<__half, 64>(p, grid, causal, s)
                 : launch_fwd_c<__half, 128>(p, grid, causal, s);
}

extern "C" attn_status_t attn_noalloc_last_status(void* stream, int* where) {
  NoAllocDevice* st = nullptr;
  attn_status_t r = noalloc_device(&st);
  if (r != ATTN_OK) return r;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_CUDA;
  int h[4] = {0, 0, 0, 0};   // host copy of the record: no device memory involved
  if (cudaMemcpy(h, st->scratch, kNoAllocStatusBytes, cudaMemcpyDeviceToHost) != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaMemset(st->scratch, 0, kNoAllocStatusBytes) != cudaSuccess) return ATTN_ERR_CUDA;
  if (where != nullptr) {
    where[0] = h[1];
    where[1] = h[2];
  }
  if (h[0] == 0) return ATTN_OK;
  if (h[0] == ATTN_ERR_TIMEOUT || h[0] == ATTN_ERR_BOUNDS) return static_cast<attn_status_t>(h[0]);
  return ATTN_ERR_CUDA;
}

extern "C" int attn_debug_status_allocated(void) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  std::lock_guard<std::mutex> lock(g_mu);
  return g_dev[dev].status != nullptr ? 1 : 0;
}

extern "C" size_t attn_bwd_workspace_bytes(int B, int H, int N, int d, int deterministic) {
  if (B < 1 || H < 1 || N < 1 || d < 1 || (deterministic != 0 && deterministic != 1)) return 0;
  return bwd_workspace_bytes(B, H, N, d, deterministic);
}

extern "C" attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* o,
                                  const void* d_o, const float* lse, void* dq, void* dk, void* dv,
                                  void* workspace, size_t workspace_bytes, int B, int H, int N, int d,
                                  float scale, int causal, int deterministic, int dtype, void* stream) {
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || d_o == nullptr || lse == nullptr ||
      dq == nullptr || dk == nullptr || dv == nullptr || workspace == nullptr)
    return ATTN_ERR_INVALID_ARG;
  attn_status_t r = common_checks(B, H, N, scale, causal);
  if (r != ATTN_OK) return r;
  if (deterministic != 0 && deterministic != 1) return ATTN_ERR_INVALID_ARG;
  if (d < 1) return ATTN_ERR_INVALID_ARG;
  if (d > 128 || (d % 8) != 0) return ATTN_ERR_UNSUPPORTED;
  if (dtype != ATTN_BF16 && dtype != ATTN_FP16) return ATTN_ERR_UNSUPPORTED;
  if (workspace_bytes < bwd_workspace_bytes(B, H, N, d, deterministic)) return ATTN_ERR_INVALID_ARG;
  const void* p16[] = {q, k, v, o, d_o, dq, dk, dv, workspace};
  for (const void* x : p16)
    if (!aligned16(x)) return ATTN_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return ATTN_ERR_MISALIGNED;

  DeviceState* st = nullptr;
  if ((r = device_state(&st)) != ATTN_OK) return r;
  const CUtensorMapDataType dt =
      dtype == ATTN_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const Strides cs = contiguous(H, N, d);
  attn::BwdParams p{};
  if ((r = make_map(&p.tm_q, q, dt, 2, B, H, N, d, cs, 64)) != ATTN_OK) return r;
  if ((r = make_map(&p.tm_k, k, dt, 2, B, H, N, d, cs, 64)) != ATTN_OK) return r;
  if ((r = make_map(&p.tm_v, v, dt, 2, B, H, N, d, cs, 64)) != ATTN_OK) return r;
  if ((r = make_map(&p.tm_o, o, dt, 2, B, H, N, d, cs, 64)) != ATTN_OK) return r;
  if ((r = make_map(&p.tm_do, d_o, dt, 2, B, H, N, d, cs, 64)) != ATTN_OK) return r;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.lse = lse;
  p.rows = static_cast<float*>(workspace);
  p.dq_acc = deterministic ? nullptr
                           : reinterpret_cast<float*>(static_cast<char*>(workspace) + bwd_rows_bytes(B, H, N));
  if (!deterministic && (r = make_map_dq(&p.tm_dq, p.dq_acc, B * H, N, d)) != ATTN_OK) return r;
  p.status = st->status;
  p.BH = B * H;
  p.H = H;
  p.N = N;
  p.n_t = (N + 127) / 128;
  p.d_out = d;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.wait_limit_ns = wait_limit_ns();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool bf = dtype == ATTN_BF16;
  const bool d64 = d <= 64;
  if (deterministic) {
    if (bf)
      return d64 ? launch_bwd_c<__nv_bfloat16, 64>(p, st->sm_count, causal, s)
                 : launch_bwd_c<__nv_bfloat16, 128>(p, st->sm_count, causal, s);
    return d64 ? launch_bwd_c<__half, 64>(p, st->sm_count, causal, s)
               : launch_bwd_c<__half, 128>(p, st->sm_count, causal, s);
  }
  if (bf)
    return d64 ? launch_bwd_fused_c<__nv_bfloat16, 64>(p, st->sm_count, causal, o, d_o, s)
               : launch_bwd_fused_c<__nv_bfloat16, 128>(p, st->sm_count, causal, o, d_o, s);
  return d64 ? launch_bwd_fused_c<__half, 64>(p, st->sm_count, causal, o, d_o, s)
             : launch_bwd_fused_c<__half, 128>(p, st->sm_count, causal, o, d_o, s);
}

extern "C" size_t attn_fwd_splitkv_workspace_bytes(int B, int H, int Nq, int d, int n_splits) {
  if (B < 1 || H < 1 || Nq < 1 || d < 1 || n_splits < 1) return 0;
  return splitkv_workspace_bytes(B, H, Nq, d, n_splits);
}

extern "C" int attn_fwd_splitkv_auto_splits(int B, int H, int Nq, int Nk) {
  if (B < 1 || H < 1 || Nq < 1 || Nk < 1) return 0;
  DeviceState* st = nullptr;
  if (device_state(&st) != ATTN_OK) return 0;
  return splitkv_auto_splits(B * H, (Nq + 127) / 128, (Nk + 127) / 128, st->sm_count);
}

extern "C" attn_status_t attn_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse,
                                          int B, int H, int Nq, int Nk, int d, float scale, int causal,
                                          int n_splits, int dtype, void* workspace, size_t workspace_bytes,
                                          void* stream) {
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || workspace == nullptr)
    return ATTN_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || Nq < 1 || Nk < 1) return ATTN_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H * Nk >= (1ll << 31) || static_cast<long long>(B) * H * Nq >= (1ll << 31))
    return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (causal && Nq > Nk) return ATTN_ERR_INVALID_ARG;   // every query must see at least one key
  if (n_splits < 0) return ATTN_ERR_INVALID_ARG;
  if (d < 1) return ATTN_ERR_INVALID_ARG;
  if (d > 256 || (d % 8) != 0) return ATTN_ERR_UNSUPPORTED;
  if (dtype != ATTN_BF16 && dtype != ATTN_FP16) return ATTN_ERR_UNSUPPORTED;
  const void* p16[] = {q, k, v, o, workspace};
  for (const void* x : p16)
    if (!aligned16(x)) return ATTN_ERR_MISALIGNED;
  if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return ATTN_ERR_MISALIGNED;
  attn_status_t r;
  DeviceState* st = nullptr;
  if ((r = device_state(&st)) != ATTN_OK) return r;
  const int BH = B * H;
  const int n_qt = (Nq + 127) / 128, n_kv = (Nk + 127) / 128;
  if (n_splits == 0) n_splits = splitkv_auto_splits(BH, n_qt, n_kv, st->sm_count);
  if (n_splits > n_kv) n_splits = n_kv;
  if (static_cast<long long>(BH) * n_qt * n_splits >= (1ll << 31)) return ATTN_ERR_INVALID_ARG;
  if (workspace_bytes < splitkv_workspace_bytes(B, H, Nq, d, n_splits)) return ATTN_ERR_INVALID_ARG;
  const CUtensorMapDataType dt =
      dtype == ATTN_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  attn::SplitParams p{};
  if ((r = make_map(&p.tm_q, q, dt, 2, B, H, Nq, d, contiguous(H, Nq, d), 64)) != ATTN_OK) return r;
  if ((r = make_map(&p.tm_k, k, dt, 2, B, H, Nk, d, contiguous(H, Nk, d), 64)) != ATTN_OK) return r;
  if ((r = make_map(&p.tm_v, v, dt, 2, B, H, Nk, d, contiguous(H, Nk, d), 64)) != ATTN_OK) return r;
  p.o_part = static_cast<float*>(workspace);
  p.lse_part = p.o_part + static_cast<size_t>(n_splits) * BH * Nq * d;
  p.status = st->status;
  p.BH = BH;
  p.H = H;
  p.Nq = Nq;
  p.Nk = Nk;
  p.n_qt = n_qt;
  p.n_kv = n_kv;
  p.n_splits = n_splits;
  p.n_units = BH * n_qt * n_splits;
  p.q_off = Nk - Nq;
  p.d_out = d;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.wait_limit_ns = wait_limit_ns();
  const int grid = p.n_units < st->sm_count ? p.n_units : st->sm_count;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int dk = d <= 64 ? 64 : (d <= 128 ? 128 : 256);
  if (dtype == ATTN_BF16)
    return dk == 64    ? launch_splitkv_c<__nv_bfloat16, 64>(p, grid, causal, o, lse, s)
           : dk == 128 ? launch_splitkv_c<__nv_bfloat16, 128>(p, grid, causal, o, lse, s)
                       : launch_splitkv_c<__nv_bfloat16, 256>(p, grid, causal, o, lse, s);
  return dk == 64    ? launch_splitkv_c<__half, 64>(p, grid, causal, o, lse, s)
         : dk == 128 ? launch_splitkv_c<__half, 128>(p, grid, causal, o, lse, s)
                     : launch_splitkv_c<__half, 256>(p, grid, causal, o, lse, s);
}

// ---------------------------------------------------------------------------
// Host-buffer forward with transfers overlapped with compute (see
// include/attn.h).  Heads are processed in chunks through two device slots:
// H2D copies of chunk c+1 on one internal stream and D2H copies of chunk c-1
// on another run while chunk c computes on the caller's stream.
// ---------------------------------------------------------------------------
namespace {

struct HostPipe {
  std::mutex mu;  // held while a call enqueues on the shared streams and events
  bool ready = false;
  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaEvent_t start = nullptr, in_done[2] = {nullptr, nullptr}, comp_done[2] = {nullptr, nullptr},
              out_done[2] = {nullptr, nullptr};
};
HostPipe g_pipe[kMaxDevices];

attn_status_t host_pipe(HostPipe** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  HostPipe& hp = g_pipe[dev];
  if (!hp.ready) {
    if (cudaStreamCreateWithFlags(&hp.s_in, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&hp.s_out, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&hp.start, cudaEventDisableTiming) != cudaSuccess)
      return ATTN_ERR_CUDA;
    for (int i = 0; i < 2; ++i)
      if (cudaEventCreateWithFlags(&hp.in_done[i], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&hp.comp_done[i], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&hp.out_done[i], cudaEventDisableTiming) != cudaSuccess)
        return ATTN_ERR_CUDA;
    hp.ready = true;
  }
  *out = &hp;
  return ATTN_OK;
}

// Heads per chunk: about a sixteenth of the heads (at least one).  The
// first chunk's copy-in and the last chunk's compute and copy-out are not
// overlapped, so smaller chunks shorten that fill and drain (eighths: 8.3 ms
// per step at B=4, H=16, N=8K, d=128, where the copy-in alone takes ~7.2 ms).
int host_chunk_heads(int BH) { return BH >= 16 ? (BH + 15) / 16 : 1; }

size_t host_slot_bytes(int chunk, int N, int d) {
  const size_t t = static_cast<size_t>(chunk) * N * d * 2;   // one 16-bit [chunk][N][d] tensor
  const size_t l = ((static_cast<size_t>(chunk) * N * 4 + 255) / 256) * 256;
  return ((4 * t + 255) / 256) * 256 + l;                    // q, k, v, o, then lse
}

}  // namespace

extern "C" size_t attn_fwd_host_workspace_bytes(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || d < 1) return 0;
  return 2 * host_slot_bytes(host_chunk_heads(B * H), N, d);
}

extern "C" attn_status_t attn_fwd_host(const void* q_host, const void* k_host, const void* v_host, void* o_host,
                                       float* lse_host, int B, int H, int N, int d, float scale, int causal,
                                       int dtype, void* workspace, size_t workspace_bytes, void* stream) {
  if (q_host == nullptr || k_host == nullptr || v_host == nullptr || o_host == nullptr || workspace == nullptr)
    return ATTN_ERR_INVALID_ARG;
  attn_status_t r = common_checks(B, H, N, scale, causal);
  if (r != ATTN_OK) return r;
  if (d < 1) return ATTN_ERR_INVALID_ARG;
  if (d > 256 || (d % 8) != 0) return ATTN_ERR_UNSUPPORTED;
  if (dtype != ATTN_BF16 && dtype != ATTN_FP16) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(workspace)) return ATTN_ERR_MISALIGNED;
  const int BH = B * H;
  const int chunk = host_chunk_heads(BH);
  const size_t slot = host_slot_bytes(chunk, N, d);
  if (workspace_bytes < 2 * slot) return ATTN_ERR_INVALID_ARG;
  HostPipe* hp = nullptr;
  if ((r = host_pipe(&hp)) != ATTN_OK) return r;
  // Calls from several host threads take turns enqueueing: each event wait
  // below must see the record made by the same call.
  std::lock_guard<std::mutex> pipe_lock(hp->mu);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t row_bytes = static_cast<size_t>(N) * d * 2;    // one head of one tensor
  const size_t t_bytes = static_cast<size_t>(chunk) * row_bytes;
  const size_t t_pad = ((4 * t_bytes + 255) / 256) * 256;
  // copies of this call start after the work already queued on `stream`
  if (cudaEventRecord(hp->start, s) != cudaSuccess || cudaStreamWaitEvent(hp->s_in, hp->start, 0) != cudaSuccess)
    return ATTN_ERR_CUDA;
  const int n_chunks = (BH + chunk - 1) / chunk;
  for (int c = 0; c < n_chunks; ++c) {
    const int i = c & 1;
    const int h0 = c * chunk;
    const int nh = BH - h0 < chunk ? BH - h0 : chunk;
    char* base = static_cast<char*>(workspace) + i * slot;
    char* dq = base;
    char* dk = base + t_bytes;
    char* dv = base + 2 * t_bytes;
    char* dout = base + 3 * t_bytes;
    float* dlse = reinterpret_cast<float*>(base + t_pad);
    const size_t off = static_cast<size_t>(h0) * row_bytes;
    const size_t bytes = static_cast<size_t>(nh) * row_bytes;
    // the slot is free once its previous results have been copied out (the
    // wait is a no-op for an event never recorded)
    if (cudaStreamWaitEvent(hp->s_in, hp->out_done[i], 0) != cudaSuccess) return ATTN_ERR_CUDA;
    if (cudaMemcpyAsync(dq, static_cast<const char*>(q_host) + off, bytes, cudaMemcpyHostToDevice, hp->s_in) !=
            cudaSuccess ||
        cudaMemcpyAsync(dk, static_cast<const char*>(k_host) + off, bytes, cudaMemcpyHostToDevice, hp->s_in) !=
            cudaSuccess ||
        cudaMemcpyAsync(dv, static_cast<const char*>(v_host) + off, bytes, cudaMemcpyHostToDevice, hp->s_in) !=
            cudaSuccess)
      return ATTN_ERR_CUDA;
    if (cudaEventRecord(hp->in_done[i], hp->s_in) != cudaSuccess ||
        cudaStreamWaitEvent(s, hp->in_done[i], 0) != cudaSuccess)
      return ATTN_ERR_CUDA;
    const Strides cs = contiguous(nh, N, d);
    if ((r = fwd16(dq, dk, dv, dout, lse_host ? dlse : nullptr, 1, nh, N, d, cs, cs, cs, cs, scale, causal, dtype,
                   stream)) != ATTN_OK)
      return r;
    if (cudaEventRecord(hp->comp_done[i], s) != cudaSuccess ||
        cudaStreamWaitEvent(hp->s_out, hp->comp_done[i], 0) != cudaSuccess)
      return ATTN_ERR_CUDA;
    if (cudaMemcpyAsync(static_cast<char*>(o_host) + off, dout, bytes, cudaMemcpyDeviceToHost, hp->s_out) !=
        cudaSuccess)
      return ATTN_ERR_CUDA;
    if (lse_host != nullptr &&
        cudaMemcpyAsync(lse_host + static_cast<size_t>(h0) * N, dlse, static_cast<size_t>(nh) * N * 4,
                        cudaMemcpyDeviceToHost, hp->s_out) != cudaSuccess)
      return ATTN_ERR_CUDA;
    if (cudaEventRecord(hp->out_done[i], hp->s_out) != cudaSuccess) return ATTN_ERR_CUDA;
  }
  // the call completes on `stream` once every result has reached the host
  for (int i = 0; i < 2 && i < n_chunks; ++i)
    if (cudaStreamWaitEvent(s, hp->out_done[i], 0) != cudaSuccess) return ATTN_ERR_CUDA;
  return ATTN_OK;
}
