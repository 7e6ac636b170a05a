// Split-KV attention forward for sm_100a (bf16 / fp16, head dim 64, 128 or
// 256):
// short query blocks against long key/value sequences, the keys of each
// (head, query tile) divided among CTAs and the partial results merged.
//
// The pages contrast FlashAttention-3 with FlashDecoding, which parallelises
// the decode phase over the key/value sequence length ("FlashAttention-3"
// explainer, droidorbit.com, FAQ "How does FlashAttention-3 compare to
// FlashDecoding?").  Each split s computes, for its keys J_s, the exact
// partial softmax statistics of the forward (same page, "Mathematical
// Formulation: The Online Softmax Rescaling Trick"):
//
//   O_s = sum_{j in J_s} exp(s_j - LSE_s) v_j,   LSE_s = ln sum_{j in J_s} exp(s_j)
//
// and the merge is the same rescaling applied across splits:
//
//   LSE = ln sum_s exp(LSE_s),   O = sum_s exp(LSE_s - LSE) O_s.
//
// Queries may be fewer than keys (Nq <= Nk when causal): query i sits at
// position Nk - Nq + i, so causal masking keeps keys j <= Nk - Nq + i (the
// decode alignment; with Nq = Nk it is the forward's mask).
//
// attn_splitkv_kernel: persistent, one CTA of 256 threads per SM; a work unit
// is (b*h, 128-row query tile, split).  Warp 0 issues TMA loads (Q once per
// unit, then K and V tiles in the order the MMA consumes them), warp 1 issues
// tcgen05 products, warps 4-7 run the online softmax (thread = query row).
// S is double-buffered in TMEM (S_a | S_b | O: 128 + 128 + d <= 512
// columns), so the product S(j+1) runs
// while the softmax works on S(j); P is written over its S buffer and
// O += P V_j reads it from TMEM.  Warps whose 32 rows are all past Nq skip the
// arithmetic (decode tiles are mostly padding rows).  Each unit writes its
// fp32 O_s and LSE_s to a workspace; attn_splitkv_combine_kernel merges them.
#pragma once
#include "fwd_sm100.cuh"

namespace attn {

struct SplitParams {
  CUtensorMap tm_q;   // 4-D maps (d, rows, H, B): q over Nq rows, k and v over Nk rows
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  float* o_part;      // [n_splits][BH][Nq][d_out] fp32, O_s normalised by its own l
  float* lse_part;    // [n_splits][BH][Nq] natural-log LSE_s (-inf: no visible key)
  int* status;
  int BH, H, Nq, Nk, n_qt, n_kv, n_splits, n_units, q_off, d_out;
  float scale_log2;
  unsigned long long wait_limit_ns;
};

template <int D>
struct SplitCfg {
  static constexpr int kChunkBytes = 128 * 128;
  static constexpr int kChunks = D / 64;
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  // K/V ring (deep where it fits: the decode shapes stream from HBM); at
  // d = 256 a tile is 64 KiB and only two fit beside Q
  static constexpr int kStages = (D == 64) ? 10 : (D == 128 ? 6 : 2);
  static constexpr int kOffKV = kTileBytes;             // [Q | ring | barriers]
  static constexpr int kOffBar = kOffKV + kStages * kTileBytes;
  static constexpr int kSmem = kOffBar + 512 + 1024;
  static constexpr int kThreads = 256;
  static constexpr int kTmemCols = 512;                 // S_a 0-127 | S_b 128-255 | O 256-
  static constexpr int kColO = 256;
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
};

// Key tiles a (query tile, split) unit covers: [j0, j1), empty when the
// split index is at or past the tile's split count.  Used by the kernel and
// (with the same arithmetic) by the combine kernel.
__host__ __device__ __forceinline__ int splitkv_needed_tiles(int qt, int Nq, int n_kv, int q_off, bool causal) {
  if (!causal) return n_kv;
  const int last_row = min(qt * 128 + 127, Nq - 1);
  return min(n_kv, (last_row + q_off) / 128 + 1);
}
__host__ __device__ __forceinline__ int splitkv_count(int needed, int n_splits) {
  return min(n_splits, needed);
}

template <bool CAUSAL>
__device__ __forceinline__ bool splitkv_unit(const SplitParams& p, int unit, int& bh, int& qt, int& j0, int& j1) {
  const int sp = unit % p.n_splits;
  const int rest = unit / p.n_splits;
  qt = rest % p.n_qt;
  bh = rest / p.n_qt;
  const int need = splitkv_needed_tiles(qt, p.Nq, p.n_kv, p.q_off, CAUSAL);
  const int ns = splitkv_count(need, p.n_splits);
  if (sp >= ns) return false;
  j0 = static_cast<int>(static_cast<long long>(sp) * need / ns);
  j1 = static_cast<int>(static_cast<long long>(sp + 1) * need / ns);
  return true;
}

template <typename E, int D, bool CAUSAL>
__global__ void __launch_bounds__(256, 1) attn_splitkv_kernel(const __grid_constant__ SplitParams p) {
  using Cfg = SplitCfg<D>;
  using T = E;
  constexpr int S = Cfg::kStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + Cfg::kOffKV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kOffBar);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* s_full = bars + 2;     // [2] S buffer b holds a finished S
  uint64_t* p_full = bars + 4;     // [2] P written over S buffer b (128 arrivals)
  uint64_t* o_ready = bars + 6;    // one O += P V product complete
  uint64_t* o_full = bars + 7;     // O of the unit complete
  uint64_t* drain = bars + 8;
  uint64_t* kv_full = bars + 9;    // [S]
  uint64_t* kv_empty = bars + 9 + S;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 9 + 2 * S);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(s_full + 1, 1);
    mbar_init(p_full, 128);
    mbar_init(p_full + 1, 128);
    mbar_init(o_ready, 1);
    mbar_init(o_full, 1);
    mbar_init(drain, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const unsigned long long lim = p.wait_limit_ns;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA
    if (lane == 0) {
      uint32_t kv_iter = 0, unit_iter = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int unit = k * static_cast<int>(gridDim.x) + static_cast<int>(blockIdx.x);
        if (unit >= p.n_units) break;
        int bh, qt, j0, j1;
        if (!splitkv_unit<CAUSAL>(p, unit, bh, qt, j0, j1)) continue;
        const int h = bh % p.H, b = bh / p.H;
        const int n = j1 - j0;
        ok = mbar_wait(q_empty, (unit_iter & 1) ^ 1, p.status, abort_flag, kWhereQEmpty, lim);
        if (!ok) break;
        mbar_arrive_expect_tx(q_full, Cfg::kTileBytes);
        for (int c = 0; c < Cfg::kChunks; ++c)
          if (smem_range_ok(sQ + c * Cfg::kChunkBytes, Cfg::kChunkBytes, smem, 0, Cfg::kOffKV, p.status, kChkQLoad))
            tma_load_4d(sQ + c * Cfg::kChunkBytes, &p.tm_q, q_full, c * 64, qt * 128, h, b);
        ++unit_iter;
        // consumption order: K0, K1, then V(jj), K(jj + 2) for jj = 0, 1, ...
        auto load = [&](const CUtensorMap* map, int j) -> bool {
          const uint32_t s = kv_iter % S;
          if (!mbar_wait(kv_empty + s, ((kv_iter / S) & 1) ^ 1, p.status, abort_flag, kWhereKvEmpty, lim))
            return false;
          mbar_arrive_expect_tx(kv_full + s, Cfg::kTileBytes);
          for (int c = 0; c < Cfg::kChunks; ++c)
            if (smem_range_ok(sKV + s * Cfg::kTileBytes + c * Cfg::kChunkBytes, Cfg::kChunkBytes, smem, Cfg::kOffKV,
                              Cfg::kOffBar, p.status, kChkKvLoad))
              tma_load_4d(sKV + s * Cfg::kTileBytes + c * Cfg::kChunkBytes, map, kv_full + s, c * 64, j * 128, h, b);
          ++kv_iter;
          return true;
        };
        ok = load(&p.tm_k, j0);
        if (ok && n > 1) ok = load(&p.tm_k, j0 + 1);
        for (int jj = 0; jj < n && ok; ++jj) {
          ok = load(&p.tm_v, j0 + jj);
          if (ok && jj + 2 < n) ok = load(&p.tm_k, j0 + jj + 2);
        }
      }
      if (!ok) {
        volatile int never = 0;
        for (uint32_t i = (kv_iter > S ? kv_iter - S : 0); i < kv_iter; ++i)
          mbar_wait(kv_full + (i % S), (i / S) & 1, nullptr, &never, kWhereDrain, 100000000ull);
        if (unit_iter > 0) mbar_wait(q_full, (unit_iter - 1) & 1, nullptr, &never, kWhereDrain, 100000000ull);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t fmt = Elem<E>::kFmt;
      constexpr uint32_t idesc_s = make_idesc(fmt, fmt, 0, 0, 128, 128);
      constexpr uint32_t idesc_o = make_idesc(fmt, fmt, 0, 1, 128, D);
      const uint64_t dQ = smem_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dK = smem_desc_sw128(smem_u32(sKV), 16, 1024);
      const uint64_t dV = smem_desc_sw128(smem_u32(sKV), Cfg::kChunkBytes, 1024);
      uint32_t kv_iter = 0, unit_iter = 0, p_cnt[2] = {0, 0};
      bool ok = true;
      auto wait_kv = [&]() -> uint32_t {
        const uint32_t s = kv_iter % S;
        ok = mbar_wait(kv_full + s, (kv_iter / S) & 1, p.status, abort_flag, kWhereKvFull, lim);
        tc_fence_after();
        ++kv_iter;
        return s;
      };
      // S(buffer b) = Q K^T from ring stage s
      auto issue_s = [&](int b, uint32_t s) {
        const uint64_t b0 = dK + static_cast<uint64_t>((s * Cfg::kTileBytes) >> 4);
        const bool in_range =
            tmem_range_ok(tmem + b * 128, tmem, 128, b * 128, b * 128 + 128, p.status, kChkSOut) &&
            smem_range_ok(sKV + s * Cfg::kTileBytes, Cfg::kTileBytes, smem, Cfg::kOffKV, Cfg::kOffBar, p.status,
                          kChkSK);
#pragma unroll
        for (int kk = 0; kk < D / 16 && in_range; ++kk) {
          const uint32_t off = ((kk >> 2) * Cfg::kChunkBytes + (kk & 3) * 32) >> 4;
          mma_ss(tmem + b * 128, dQ + off, b0 + off, idesc_s, kk > 0, false);
        }
        mma_commit(s_full + b);
        mma_commit(kv_empty + s);
      };
      for (int k = 0; ok; ++k) {
        const int unit = k * static_cast<int>(gridDim.x) + static_cast<int>(blockIdx.x);
        if (unit >= p.n_units) break;
        int bh_, qt_, j0, j1;
        if (!splitkv_unit<CAUSAL>(p, unit, bh_, qt_, j0, j1)) continue;
        (void)bh_;
        (void)qt_;
        const int n = j1 - j0;
        ok = mbar_wait(q_full, unit_iter & 1, p.status, abort_flag, kWhereQFull, lim);
        tc_fence_after();
        ++unit_iter;
        if (!ok) break;
        uint32_t s = wait_kv();
        if (!ok) break;
        issue_s(0, s);
        if (n > 1) {
          s = wait_kv();
          if (!ok) break;
          issue_s(1, s);
        }
        for (int jj = 0; jj < n && ok; ++jj) {
          const int b = jj & 1;
          if (!(ok = mbar_wait(p_full + b, p_cnt[b] & 1, p.status, abort_flag, kWherePFull, lim))) break;
          ++p_cnt[b];
          tc_fence_after();
          const uint32_t sv = wait_kv();
          if (!ok) break;
          // O += P V: P packed over S buffer b (8 columns per 16 keys), V MN-major
          const uint64_t b0 = dV + static_cast<uint64_t>((sv * Cfg::kTileBytes) >> 4);
          const bool pv_in_range =
              tmem_range_ok(tmem + Cfg::kColO, tmem, D, Cfg::kColO, Cfg::kColO + D, p.status, kChkOOut) &&
              tmem_range_ok(tmem + b * 128, tmem, 64, b * 128, b * 128 + 64, p.status, kChkPIn) &&
              smem_range_ok(sKV + sv * Cfg::kTileBytes, Cfg::kTileBytes, smem, Cfg::kOffKV, Cfg::kOffBar, p.status,
                            kChkVIn);
#pragma unroll
          for (int kk = 0; kk < 8 && pv_in_range; ++kk)
            mma_ts(tmem + Cfg::kColO, tmem + b * 128 + kk * 8, b0 + ((kk * 16 * 128) >> 4), idesc_o,
                   (jj > 0 || kk > 0) ? 1u : 0u, false);
          mma_commit(kv_empty + sv);
          mma_commit(o_ready);
          if (jj + 2 < n) {
            // S(jj + 2) over P(jj), which the product just issued consumes first
            const uint32_t sk = wait_kv();
            if (!ok) break;
            issue_s(b, sk);
          }
        }
        if (!ok) break;
        mma_commit(o_full);
        mma_commit(q_empty);
      }
      if (!ok) {
        mma_commit(drain);
        volatile int never = 0;
        mbar_wait(drain, 0, nullptr, &never, kWhereDrain, 100000000ull);
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // -------------------------------------------------------------- softmax
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tO = tmem + lane_off + Cfg::kColO;
    uint32_t s_cnt[2] = {0, 0}, g = 0, o_cnt = 0;
    bool ok = true;
    constexpr float kLazy = 8.0f;
    for (int k = 0; ok; ++k) {
      const int unit = k * static_cast<int>(gridDim.x) + static_cast<int>(blockIdx.x);
      if (unit >= p.n_units) break;
      int bh, qt, j0, j1;
      if (!splitkv_unit<CAUSAL>(p, unit, bh, qt, j0, j1)) continue;
      const int sp = unit % p.n_splits;
      const int n = j1 - j0;
      const int row = qt * 128 + r;
      // this warp's 32 rows hold no query: it only keeps the barrier protocol
      const bool warp_active = qt * 128 + quarter * 32 < p.Nq;
      const int lim_key = CAUSAL ? min(row + p.q_off, p.Nk - 1) : (p.Nk - 1);
      const float c = p.scale_log2;
      float m = -INFINITY, l = 0.f;
      for (int jj = 0; jj < n; ++jj, ++g) {
        const int b = jj & 1;
        bool w = mbar_wait(s_full + b, s_cnt[b] & 1, p.status, abort_flag, kWhereSFull, lim);
        ++s_cnt[b];
        if (!__all_sync(0xffffffffu, w)) { ok = false; *abort_flag = 1; break; }
        tc_fence_after();
        if (warp_active) {
          const uint32_t tS = tmem + lane_off + b * 128;
          float s[128];
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t rr[32];
            if (tmem_range_ok(tS + cc * 32, tmem, 32, b * 128, b * 128 + 128, p.status, kChkSLoad))
              tmem_ld32(tS + cc * 32, rr);
#pragma unroll
            for (int i = 0; i < 32; ++i) s[cc * 32 + i] = __uint_as_float(rr[i]);
          }
          tmem_wait_ld();
          tmem_reg_fence(s);
          const int key0 = (j0 + jj) * 128;
          const bool need_mask = (CAUSAL && key0 + 127 > qt * 128 + p.q_off) || (key0 + 128 > p.Nk);
          if (need_mask) {
#pragma unroll
            for (int i = 0; i < 128; ++i)
              if (key0 + i > lim_key) s[i] = -INFINITY;
          }
          const float mx = row_max128(s) * c;
          float alpha = 1.0f;
          if (mx > m + kLazy) {
            alpha = ex2_approx(m - mx);
            m = mx;
          }
          // Rescale O when some row of this warp raised its max: wait for the
          // previous O += P V product first (S(jj) completing guarantees only
          // the one before it).
          if (jj > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
            w = mbar_wait(o_ready, (g - 1) & 1, p.status, abort_flag, kWhereOFull, lim);
            if (!__all_sync(0xffffffffu, w)) { ok = false; *abort_flag = 1; break; }
            tc_fence_after();
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
              uint32_t rr[32];
              if (!tmem_range_ok(tO + cc * 32, tmem, 32, Cfg::kColO, Cfg::kColO + D, p.status, kChkORescale))
                continue;
              tmem_ld32(tO + cc * 32, rr);
              tmem_wait_ld();
              tmem_reg_fence(rr);
#pragma unroll
              for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * alpha);
              tmem_st32(tO + cc * 32, rr);
              tmem_wait_st();     // the store reads rr asynchronously
              tmem_reg_fence(rr);
            }
          }
          // a row that has seen no visible key yet keeps m = -inf: its P is 0
          const float neg_m = (m == -INFINITY) ? 0.f : -m;
          float sum = 0.f;
#pragma unroll
          for (int h = 0; h < 2; ++h)
            if (tmem_range_ok(tS + 32 * h, tmem, 32, b * 128, b * 128 + 64, p.status, kChkPStore))
              sum += need_mask ? exp_pack_half<false, T, false>(s, h, c, neg_m, 1.0f, tS)
                               : exp_pack_half<false, T, true>(s, h, c, neg_m, 1.0f, tS);
          l = l * alpha + sum;
          tmem_wait_st();
        }
        tc_fence_before();
        mbar_arrive(p_full + b);
      }
      if (!ok) break;
      // every warp counts the unit's o_full phase; only active warps wait on it
      const uint32_t o_phase = o_cnt++;
      if (!warp_active) continue;
      // -------------------------------------------------------- epilogue
      bool w = mbar_wait(o_full, o_phase & 1, p.status, abort_flag, kWhereOFull, lim);
      if (!__all_sync(0xffffffffu, w)) { ok = false; *abort_flag = 1; break; }
      tc_fence_after();
      const bool any = l > 0.f;
      const float inv_l = any ? 1.0f / l : 0.f;
      const size_t prow = (static_cast<size_t>(sp) * p.BH + bh) * p.Nq + row;
      float* orow = p.o_part + prow * p.d_out;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t rr[32];
        if (tmem_range_ok(tO + cc * 32, tmem, 32, Cfg::kColO, Cfg::kColO + D, p.status, kChkOLoad))
          tmem_ld32(tO + cc * 32, rr);
        tmem_wait_ld();
        tmem_reg_fence(rr);
        if (row < p.Nq) {
#pragma unroll
          for (int g4 = 0; g4 < 8; ++g4)
            if (cc * 32 + 4 * g4 < p.d_out)
              *reinterpret_cast<float4*>(orow + cc * 32 + 4 * g4) =
                  make_float4(__uint_as_float(rr[4 * g4]) * inv_l, __uint_as_float(rr[4 * g4 + 1]) * inv_l,
                              __uint_as_float(rr[4 * g4 + 2]) * inv_l, __uint_as_float(rr[4 * g4 + 3]) * inv_l);
        }
      }
      if (row < p.Nq) p.lse_part[prow] = any ? (m + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, Cfg::kTmemCols);
}

// Merge of the splits: one warp per (b*h, query row), lanes over the head
// dim (4 columns each, d <= 128).
template <typename T, bool CAUSAL>
__global__ void __launch_bounds__(256) attn_splitkv_combine_kernel(const float* __restrict__ o_part,
                                                                   const float* __restrict__ lse_part, T* o,
                                                                   float* lse, int BH, int Nq, int n_kv, int n_splits,
                                                                   int q_off, int d_out) {
  const int gw = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= BH * Nq) return;   // whole warps exit together
  const int bh = gw / Nq, row = gw % Nq;
  const int ns = splitkv_count(splitkv_needed_tiles(row / 128, Nq, n_kv, q_off, CAUSAL), n_splits);
  float mx = -INFINITY;
  for (int s = lane; s < ns; s += 32) mx = fmaxf(mx, lse_part[(static_cast<size_t>(s) * BH + bh) * Nq + row]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  // each lane owns 4 columns of every 128-column group (d_out <= 256)
  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  float wsum = 0.f;
  if (mx != -INFINITY) {
    for (int s = 0; s < ns; ++s) {
      const size_t prow = (static_cast<size_t>(s) * BH + bh) * Nq + row;
      const float ls = lse_part[prow];
      if (ls == -INFINITY) continue;
      const float wgt = __expf(ls - mx);
      wsum += wgt;
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        const int col = 128 * g + 4 * lane;
        if (col < d_out) {
          const float4 x = *reinterpret_cast<const float4*>(o_part + prow * d_out + col);
          acc[g][0] = fmaf(wgt, x.x, acc[g][0]);
          acc[g][1] = fmaf(wgt, x.y, acc[g][1]);
          acc[g][2] = fmaf(wgt, x.z, acc[g][2]);
          acc[g][3] = fmaf(wgt, x.w, acc[g][3]);
        }
      }
    }
  }
  const float inv = wsum > 0.f ? 1.0f / wsum : 0.f;
  const size_t orow = static_cast<size_t>(bh) * Nq + row;
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    const int col = 128 * g + 4 * lane;
    if (col < d_out) {
      uint2 v;
      v.x = pack2<T>(acc[g][0] * inv, acc[g][1] * inv);
      v.y = pack2<T>(acc[g][2] * inv, acc[g][3] * inv);
      *reinterpret_cast<uint2*>(o + orow * d_out + col) = v;
    }
  }
  if (lse != nullptr && lane == 0) lse[orow] = wsum > 0.f ? mx + __logf(wsum) : -INFINITY;
}

}  // namespace attn
