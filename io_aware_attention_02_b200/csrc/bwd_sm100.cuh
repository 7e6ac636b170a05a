// Attention backward for sm_100a (bf16 / fp16, head dim up to 128).
//
// The chain rule of the forward definition (Softmax(Q K^T / sqrt(d)) V,
// "FlashAttention-3" explainer, droidorbit.com), tiled like the forward:
//
//   P  = exp(scale * Q K^T - LSE)         (LSE saved by the forward pass)
//   dV = P^T dO,   dP = dO V^T,   D = rowsum(dO * O),   dS = P * (dP - D)
//   dQ = scale * dS K,   dK = scale * dS^T Q
//
// The pages benchmark the backward next to the forward (quantum-bit repost
// "H100 utilisation 75% ... FlashAttention-3", attention benchmark) without
// spelling it out.  Two kernels, neither needing atomics, so results are
// deterministic:
//
//   * attn_bwd_dq_kernel, one 128-row Q tile per work unit: for each key tile
//     S = Q K^T and dP = dO V^T into TMEM, the row warps turn them into dS
//     (16-bit, written over S) and dQ += dS K accumulates in TMEM.  It also
//     writes, per 128-row tile, the row statistics the second kernel needs:
//     LSE * log2(e) and D = rowsum(dO * O) (from the shared-memory tiles).
//   * attn_bwd_dkdv_kernel, one 128-key tile per work unit: for each Q tile
//     S^T = K Q^T and dP^T = V dO^T into TMEM (rows = keys), the row warps
//     turn them into P^T and dS^T (16-bit, over S^T and dP^T), and
//     dV += P^T dO, dK += dS^T Q accumulate in TMEM.
//
// The same TMA tiles serve as K-major or MN-major operands through different
// shared-memory descriptors.  Roles: warp 0 TMA, warp 1 MMA issuer (one
// thread) and TMEM allocator, warps 4-7 one thread per TMEM lane (row).
// Every wait is bounded, as in the forward kernels; no named barriers, so a
// warp that gives up cannot strand the others.
#pragma once
#include "fwd_sm100.cuh"

namespace attn {

struct BwdParams {
  CUtensorMap tm_q, tm_k, tm_v, tm_o, tm_do;   // 4-D maps (d, N, H, B), 64-column boxes
  CUtensorMap tm_dq;                           // fp32 accumulator (d, N, BH), 32 x 32 boxes (fused path)
  void* dq;                                    // [BH][N][d_out] 16-bit outputs
  void* dk;
  void* dv;
  const float* lse;                            // [BH][N] natural-log LSE of the forward
  float* rows;                                 // [BH][n_t][2][128]: LSE*log2(e) | D per Q tile
  float* dq_acc;                               // [BH][N][d_out] fp32 dQ / scale (fused path)
  int* status;
  int BH, H, N, n_t, n_units, d_out;
  float scale, scale_log2;
  unsigned long long wait_limit_ns;
  int snake, order;
};

template <int D>
struct BwdCfg {
  static constexpr int kChunkBytes = 128 * 128;
  static constexpr int kChunks = D / 64;
  static constexpr int kTileBytes = kChunks * kChunkBytes;   // 128 rows x D (16-bit)
  static constexpr int kRowBytes = 2 * 128 * 4;              // LSE2 and D of one Q tile
  static constexpr int kThreads = 256;
  static constexpr int kTmemCols = 512;
  // dQ kernel: [Q | dO | O | ring of K/V tiles | barriers]
  static constexpr int kDqStages = (D == 64) ? 6 : 3;
  static constexpr int kDqOffRing = 3 * kTileBytes;
  static constexpr int kDqOffBar = kDqOffRing + kDqStages * kTileBytes;
  static constexpr int kDqSmem = kDqOffBar + 512 + 1024;
  // dK/dV kernel: [K | V | ring of (Q, dO) | ring of row statistics | barriers]
  static constexpr int kKvStages = (D == 64) ? 4 : 2;
  static constexpr int kKvOffRing = 2 * kTileBytes;
  static constexpr int kKvOffRow = kKvOffRing + kKvStages * 2 * kTileBytes;
  static constexpr int kKvOffBar = kKvOffRow + kKvStages * kRowBytes;
  static constexpr int kKvSmem = kKvOffBar + 512 + 1024;
  static_assert(kDqSmem <= 227 * 1024 && kKvSmem <= 227 * 1024, "shared memory budget");
};

// Stores 32 fp32 accumulator columns of one row as 16-bit values times `mul`,
// the columns below `d_out` only (d_out a multiple of 8).
template <typename T>
__device__ __forceinline__ void store_row32(T* row, int col0, int d_out, const uint32_t (&r)[32], float mul) {
  uint32_t pk[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) pk[i] = pack2<T>(__uint_as_float(r[2 * i]) * mul, __uint_as_float(r[2 * i + 1]) * mul);
#pragma unroll
  for (int g = 0; g < 4; ++g)
    if (col0 + 8 * g < d_out)
      *reinterpret_cast<uint4*>(row + col0 + 8 * g) = make_uint4(pk[4 * g], pk[4 * g + 1], pk[4 * g + 2], pk[4 * g + 3]);
}

// ---------------------------------------------------------------------------
// dQ, and the per-row statistics
// ---------------------------------------------------------------------------
template <typename E, int D, bool CAUSAL>
__global__ void __launch_bounds__(256, 1) attn_bwd_dq_kernel(const __grid_constant__ BwdParams p) {
  using Cfg = BwdCfg<D>;
  using T = E;
  constexpr int S = Cfg::kDqStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sdO = smem + Cfg::kTileBytes;
  uint8_t* sO = smem + 2 * Cfg::kTileBytes;
  uint8_t* sKV = smem + Cfg::kDqOffRing;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kDqOffBar);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* sd_full = bars + 2;      // S and dP of the current key tile in TMEM
  uint64_t* ds_ready = bars + 3;     // dS written over S
  uint64_t* dq_full = bars + 4;      // dQ of the unit accumulated
  uint64_t* drain = bars + 5;
  uint64_t* kv_full = bars + 6;      // [S]
  uint64_t* kv_empty = bars + 6 + S; // [S]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 6 + 2 * S);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  constexpr int kColS = 0, kColDP = 128, kColDQ = 256;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(sd_full, 1);
    mbar_init(ds_ready, 128);
    mbar_init(dq_full, 1);
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
  const int n_t = p.n_t;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA
    if (lane == 0) {
      uint32_t kv_iter = 0, unit_iter = 0;
      bool ok = true;
      for (int k = 0; ok; ++k, ++unit_iter) {
        const int unit = sched_unit(k, p.snake);
        if (unit >= p.n_units) break;
        int bh, qt;
        decode_unit<CAUSAL>(unit, n_t, p.BH, p.order, bh, qt);
        const int n = CAUSAL ? qt + 1 : n_t;
        const int h = bh % p.H, b = bh / p.H;
        ok = mbar_wait(q_empty, (unit_iter & 1) ^ 1, p.status, abort_flag, kWhereQEmpty, lim);
        if (!ok) break;
        mbar_arrive_expect_tx(q_full, 3 * Cfg::kTileBytes);
        for (int c = 0; c < Cfg::kChunks; ++c) {
          tma_load_4d(sQ + c * Cfg::kChunkBytes, &p.tm_q, q_full, c * 64, qt * 128, h, b);
          tma_load_4d(sdO + c * Cfg::kChunkBytes, &p.tm_do, q_full, c * 64, qt * 128, h, b);
          tma_load_4d(sO + c * Cfg::kChunkBytes, &p.tm_o, q_full, c * 64, qt * 128, h, b);
        }
        // K_j at ring index base + 2j, V_j at base + 2j + 1
        for (int j = 0; j < n && ok; ++j) {
          for (int which = 0; which < 2; ++which, ++kv_iter) {
            const uint32_t s = kv_iter % S;
            ok = mbar_wait(kv_empty + s, ((kv_iter / S) & 1) ^ 1, p.status, abort_flag, kWhereKvEmpty, lim);
            if (!ok) break;
            mbar_arrive_expect_tx(kv_full + s, Cfg::kTileBytes);
            const CUtensorMap* map = which == 0 ? &p.tm_k : &p.tm_v;
            for (int c = 0; c < Cfg::kChunks; ++c)
              tma_load_4d(sKV + s * Cfg::kTileBytes + c * Cfg::kChunkBytes, map, kv_full + s, c * 64,
                          j * 128, h, b);
          }
        }
      }
      if (!ok) {
        // let the copies already issued land before the CTA exits
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
      constexpr uint32_t idesc_kk = make_idesc(fmt, fmt, 0, 0, 128, 128);   // S, dP: both K-major
      constexpr uint32_t idesc_dq = make_idesc(fmt, fmt, 0, 1, 128, D);     // dQ: B = K_j MN-major
      const uint64_t dQd = smem_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t ddO = smem_desc_sw128(smem_u32(sdO), 16, 1024);
      const uint64_t dRingK = smem_desc_sw128(smem_u32(sKV), 16, 1024);
      const uint64_t dRingMN = smem_desc_sw128(smem_u32(sKV), Cfg::kChunkBytes, 1024);
      uint32_t kv_iter = 0, unit_iter = 0, ds_cnt = 0;
      bool ok = true;
      // D[128 x 128] = A[128 x D] B[128 x D]^T, both K-major 128-byte swizzled
      auto kmajor = [&](uint32_t d_col, uint64_t a0, uint64_t b0) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * Cfg::kChunkBytes + (kk & 3) * 32) >> 4;
          mma_ss(tmem + d_col, a0 + off, b0 + off, idesc_kk, kk > 0, false);
        }
      };
      auto wait_kv = [&](uint32_t idx) -> bool {
        bool r = mbar_wait(kv_full + (idx % S), (idx / S) & 1, p.status, abort_flag, kWhereKvFull, lim);
        tc_fence_after();
        return r;
      };
      for (int k = 0; ok; ++k, ++unit_iter) {
        const int unit = sched_unit(k, p.snake);
        if (unit >= p.n_units) break;
        int bh_, qt;
        decode_unit<CAUSAL>(unit, n_t, p.BH, p.order, bh_, qt);
        (void)bh_;
        const int n = CAUSAL ? qt + 1 : n_t;
        const uint32_t base = kv_iter;
        ok = mbar_wait(q_full, unit_iter & 1, p.status, abort_flag, kWhereQFull, lim);
        tc_fence_after();
        if (!ok) break;
        for (int j = 0; j < n && ok; ++j) {
          const uint32_t ik = base + 2 * j, iv = ik + 1;
          if (!(ok = wait_kv(ik) && wait_kv(iv))) break;
          // S = Q K_j^T and dP = dO V_j^T.  They overwrite dS of the previous
          // tile, which the dQ products issued before them have consumed
          // (tcgen05 operations of one thread run in issue order).
          kmajor(kColS, dQd, dRingK + (((ik % S) * Cfg::kTileBytes) >> 4));
          kmajor(kColDP, ddO, dRingK + (((iv % S) * Cfg::kTileBytes) >> 4));
          mma_commit(sd_full);
          mma_commit(kv_empty + (iv % S));
          if (!(ok = mbar_wait(ds_ready, ds_cnt & 1, p.status, abort_flag, kWherePFull, lim))) break;
          ++ds_cnt;
          tc_fence_after();
          // dQ += dS K_j: A = dS (TMEM, 16-bit packed over S), B = K_j MN-major;
          // 16 keys (8 packed columns, 16 rows of 128 bytes) per product
          const uint64_t b0 = dRingMN + (((ik % S) * Cfg::kTileBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tmem + kColDQ, tmem + kColS + kk * 8, b0 + ((kk * 16 * 128) >> 4), idesc_dq,
                   (j > 0 || kk > 0) ? 1u : 0u, false);
          mma_commit(kv_empty + (ik % S));
        }
        if (!ok) break;
        mma_commit(dq_full);
        mma_commit(q_empty);
        kv_iter += 2 * n;
      }
      if (!ok) {
        mma_commit(drain);
        volatile int never = 0;
        mbar_wait(drain, 0, nullptr, &never, kWhereDrain, 100000000ull);
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------- row warps
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + kColS;
    const uint32_t tDP = tmem + lane_off + kColDP;
    const uint32_t tDQ = tmem + lane_off + kColDQ;
    const float c2 = p.scale_log2;
    uint32_t q_cnt = 0, sd_cnt = 0;
    bool ok = true;
    for (int k = 0; ok; ++k, ++q_cnt) {
      const int unit = sched_unit(k, p.snake);
      if (unit >= p.n_units) break;
      int bh, qt;
      decode_unit<CAUSAL>(unit, n_t, p.BH, p.order, bh, qt);
      const int n = CAUSAL ? qt + 1 : n_t;
      const int row = qt * 128 + r;
      const bool valid_row = row < p.N;
      const size_t rbase = static_cast<size_t>(bh) * p.N;

      // D = rowsum(dO * O) from the 128-byte-swizzled shared-memory tiles
      // (16-byte group g of row r sits at group g ^ (r % 8))
      bool w = mbar_wait(q_full, q_cnt & 1, p.status, abort_flag, kWhereQFull, lim);
      if (!__all_sync(0xffffffffu, w)) { ok = false; *abort_flag = 1; break; }
      float dsum = 0.f;
#pragma unroll
      for (int c = 0; c < Cfg::kChunks; ++c) {
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const int off = c * Cfg::kChunkBytes + r * 128 + ((g ^ (r & 7)) << 4);
          const uint4 a = *reinterpret_cast<const uint4*>(sdO + off);
          const uint4 b = *reinterpret_cast<const uint4*>(sO + off);
          const T* ta = reinterpret_cast<const T*>(&a);
          const T* tb = reinterpret_cast<const T*>(&b);
#pragma unroll
          for (int e = 0; e < 8; ++e) dsum = fmaf(static_cast<float>(ta[e]), static_cast<float>(tb[e]), dsum);
        }
      }
      const float lse2 = valid_row ? p.lse[rbase + row] * 1.4426950408889634f : 0.f;
      float* rows = p.rows + (static_cast<size_t>(bh) * n_t + qt) * 256;
      rows[r] = lse2;
      rows[128 + r] = dsum;

      const int lim_key = CAUSAL ? min(row, p.N - 1) : (p.N - 1);
      for (int j = 0; j < n; ++j) {
        w = mbar_wait(sd_full, sd_cnt & 1, p.status, abort_flag, kWhereSFull, lim);
        ++sd_cnt;
        if (!__all_sync(0xffffffffu, w)) { ok = false; *abort_flag = 1; break; }
        tc_fence_after();
        const int key0 = j * 128;
        // 32 keys at a time; dS of chunk cc goes to S columns 16cc..16cc+15,
        // which chunks 0..cc have already read
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t sr[32], dr[32];
          tmem_ld32(tS + cc * 32, sr);
          tmem_ld32(tDP + cc * 32, dr);
          tmem_wait_ld();
          tmem_reg_fence(sr);
          tmem_reg_fence(dr);
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float ds2[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int kk = 2 * i + e;
              const float pr = (key0 + cc * 32 + kk <= lim_key)
                                   ? ex2_approx(fmaf(__uint_as_float(sr[kk]), c2, -lse2)) : 0.f;
              ds2[e] = pr * (__uint_as_float(dr[kk]) - dsum);
            }
            pk[i] = pack2<T>(ds2[0], ds2[1]);
          }
          tmem_st16(tS + cc * 16, pk);
          tmem_wait_st();   // the store reads pk asynchronously; the next chunk reuses it
          tmem_reg_fence(pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(ds_ready);
      }
      if (!ok) break;
      w = mbar_wait(dq_full, q_cnt & 1, p.status, abort_flag, kWhereOFull, lim);
      if (!__all_sync(0xffffffffu, w)) { ok = false; *abort_flag = 1; break; }
      tc_fence_after();
      T* drow = reinterpret_cast<T*>(p.dq) + (rbase + (valid_row ? row : 0)) * p.d_out;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t rr[32];
        tmem_ld32(tDQ + cc * 32, rr);   // every lane loads (warp-wide); rows past N do not store
        tmem_wait_ld();
        tmem_reg_fence(rr);
        if (valid_row) store_row32<T>(drow, cc * 32, p.d_out, rr, p.scale);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, Cfg::kTmemCols);
}

// ---------------------------------------------------------------------------
// dK, dV
// ---------------------------------------------------------------------------
template <typename E, int D, bool CAUSAL>
__global__ void __launch_bounds__(256, 1) attn_bwd_dkdv_kernel(const __grid_constant__ BwdParams p) {
  using Cfg = BwdCfg<D>;
  using T = E;
  constexpr int S = Cfg::kKvStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem;
  uint8_t* sV = smem + Cfg::kTileBytes;
  uint8_t* sRing = smem + Cfg::kKvOffRing;   // stage s: Q tile at 2s, dO tile at 2s + 1
  const float* sRows = reinterpret_cast<const float*>(smem + Cfg::kKvOffRow);   // stage s: 256 floats
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kKvOffBar);
  uint64_t* kv_full = bars + 0;
  uint64_t* kv_empty = bars + 1;
  uint64_t* st_full = bars + 2;      // S^T and dP^T in TMEM
  uint64_t* p_ready = bars + 3;      // P^T and dS^T written
  uint64_t* acc_full = bars + 4;     // dV, dK of the unit accumulated
  uint64_t* drain = bars + 5;
  uint64_t* q_full = bars + 6;       // [S]
  uint64_t* q_empty = bars + 6 + S;  // [S]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 6 + 2 * S);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  constexpr int kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + D;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    mbar_init(st_full, 1);
    mbar_init(p_ready, 128);
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(q_full + s, 1);
      mbar_init(q_empty + s, 1);
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
  const int n_t = p.n_t;
  // Key tile of a unit.  Causal work shrinks as the key tile grows (tile j
  // meets Q tiles j..n_t-1), so the longest-first block order of
  // decode_unit maps to key tiles in rising order.
  auto key_tile = [&](int blk) { return CAUSAL ? n_t - 1 - blk : blk; };

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA
    if (lane == 0) {
      uint32_t q_iter = 0, unit_iter = 0;
      bool ok = true;
      for (int k = 0; ok; ++k, ++unit_iter) {
        const int unit = sched_unit(k, p.snake);
        if (unit >= p.n_units) break;
        int bh, blk;
        decode_unit<CAUSAL>(unit, n_t, p.BH, p.order, bh, blk);
        const int j = key_tile(blk);
        const int i0 = CAUSAL ? j : 0;
        const int h = bh % p.H, b = bh / p.H;
        ok = mbar_wait(kv_empty, (unit_iter & 1) ^ 1, p.status, abort_flag, kWhereQEmpty, lim);
        if (!ok) break;
        mbar_arrive_expect_tx(kv_full, 2 * Cfg::kTileBytes);
        for (int c = 0; c < Cfg::kChunks; ++c) {
          tma_load_4d(sK + c * Cfg::kChunkBytes, &p.tm_k, kv_full, c * 64, j * 128, h, b);
          tma_load_4d(sV + c * Cfg::kChunkBytes, &p.tm_v, kv_full, c * 64, j * 128, h, b);
        }
        for (int i = i0; i < n_t && ok; ++i, ++q_iter) {
          const uint32_t s = q_iter % S;
          ok = mbar_wait(q_empty + s, ((q_iter / S) & 1) ^ 1, p.status, abort_flag, kWhereKvEmpty, lim);
          if (!ok) break;
          mbar_arrive_expect_tx(q_full + s, 2 * Cfg::kTileBytes + Cfg::kRowBytes);
          uint8_t* st = sRing + s * 2 * Cfg::kTileBytes;
          for (int c = 0; c < Cfg::kChunks; ++c) {
            tma_load_4d(st + c * Cfg::kChunkBytes, &p.tm_q, q_full + s, c * 64, i * 128, h, b);
            tma_load_4d(st + Cfg::kTileBytes + c * Cfg::kChunkBytes, &p.tm_do, q_full + s, c * 64, i * 128, h, b);
          }
          bulk_load(smem + Cfg::kKvOffRow + s * Cfg::kRowBytes,
                    p.rows + (static_cast<size_t>(bh) * n_t + i) * 256, Cfg::kRowBytes, q_full + s);
        }
      }
      if (!ok) {
        volatile int never = 0;
        for (uint32_t i = (q_iter > S ? q_iter - S : 0); i < q_iter; ++i)
          mbar_wait(q_full + (i % S), (i / S) & 1, nullptr, &never, kWhereDrain, 100000000ull);
        if (unit_iter > 0) mbar_wait(kv_full, (unit_iter - 1) & 1, nullptr, &never, kWhereDrain, 100000000ull);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t fmt = Elem<E>::kFmt;
      constexpr uint32_t idesc_kk = make_idesc(fmt, fmt, 0, 0, 128, 128);   // S^T, dP^T
      constexpr uint32_t idesc_acc = make_idesc(fmt, fmt, 0, 1, 128, D);    // dV, dK: B MN-major
      const uint64_t dKd = smem_desc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dVd = smem_desc_sw128(smem_u32(sV), 16, 1024);
      const uint64_t dRingK = smem_desc_sw128(smem_u32(sRing), 16, 1024);
      const uint64_t dRingMN = smem_desc_sw128(smem_u32(sRing), Cfg::kChunkBytes, 1024);
      uint32_t q_iter = 0, unit_iter = 0, p_cnt = 0;
      bool ok = true;
      auto kmajor = [&](uint32_t d_col, uint64_t a0, uint64_t b0) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * Cfg::kChunkBytes + (kk & 3) * 32) >> 4;
          mma_ss(tmem + d_col, a0 + off, b0 + off, idesc_kk, kk > 0, false);
        }
      };
      // D[128 x D] (+)= A[128 x 128] (TMEM, 16-bit packed) B[128 x D] (MN-major)
      auto accum = [&](uint32_t d_col, uint32_t a_col, uint64_t b0, bool acc) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + d_col, tmem + a_col + kk * 8, b0 + ((kk * 16 * 128) >> 4), idesc_acc,
                 (acc || kk > 0) ? 1u : 0u, false);
      };
      for (int k = 0; ok; ++k, ++unit_iter) {
        const int unit = sched_unit(k, p.snake);
        if (unit >= p.n_units) break;
        int bh_, blk;
        decode_unit<CAUSAL>(unit, n_t, p.BH, p.order, bh_, blk);
        (void)bh_;
        const int j = key_tile(blk);
        const int i0 = CAUSAL ? j : 0;
        ok = mbar_wait(kv_full, unit_iter & 1, p.status, abort_flag, kWhereQFull, lim);
        tc_fence_after();
        if (!ok) break;
        for (int i = i0; i < n_t && ok; ++i, ++q_iter) {
          const uint32_t s = q_iter % S;
          if (!(ok = mbar_wait(q_full + s, (q_iter / S) & 1, p.status, abort_flag, kWhereKvFull, lim))) break;
          tc_fence_after();
          const uint32_t qoff = (s * 2 * Cfg::kTileBytes) >> 4, dooff = ((s * 2 + 1) * Cfg::kTileBytes) >> 4;
          // S^T = K Q_i^T, dP^T = V dO_i^T, over P^T / dS^T of the previous Q
          // tile, which the products issued before these have consumed
          kmajor(kColS, dKd, dRingK + qoff);
          kmajor(kColDP, dVd, dRingK + dooff);
          mma_commit(st_full);
          if (!(ok = mbar_wait(p_ready, p_cnt & 1, p.status, abort_flag, kWherePFull, lim))) break;
          ++p_cnt;
          tc_fence_after();
          accum(kColDV, kColS, dRingMN + dooff, i > i0);    // dV += P^T dO_i
          accum(kColDK, kColDP, dRingMN + qoff, i > i0);    // dK += dS^T Q_i
          mma_commit(q_empty + s);
        }
        if (!ok) break;
        mma_commit(acc_full);
        mma_commit(kv_empty);
      }
      if (!ok) {
        mma_commit(drain);
        volatile int never = 0;
        mbar_wait(drain, 0, nullptr, &never, kWhereDrain, 100000000ull);
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------- row warps
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;             // key row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + kColS;
    const uint32_t tDP = tmem + lane_off + kColDP;
    const float c2 = p.scale_log2;
    uint32_t st_cnt = 0, acc_cnt = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int unit = sched_unit(k, p.snake);
      if (unit >= p.n_units) break;
      int bh, blk;
      decode_unit<CAUSAL>(unit, n_t, p.BH, p.order, bh, blk);
      const int j = key_tile(blk);
      const int i0 = CAUSAL ? j : 0;
      const int key = j * 128 + r;
      const size_t rbase = static_cast<size_t>(bh) * p.N;
      for (int i = i0; i < n_t; ++i, ++st_cnt) {
        const uint32_t s = st_cnt % S;
        // the stage's row statistics (TMA) and S^T, dP^T (MMA)
        bool w = mbar_wait(q_full + s, (st_cnt / S) & 1, p.status, abort_flag, kWhereKvFull, lim);
        w = w && mbar_wait(st_full, st_cnt & 1, p.status, abort_flag, kWhereSFull, lim);
        if (!__all_sync(0xffffffffu, w)) { ok = false; *abort_flag = 1; break; }
        tc_fence_after();
        const float* lse2 = sRows + s * 256;
        const float* dvec = lse2 + 128;
        const int q0 = i * 128;
        // 32 queries at a time: P^T of chunk cc goes to S^T columns
        // 16cc..16cc+15 and dS^T to dP^T columns 16cc..16cc+15, which chunks
        // 0..cc have already read
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t sr[32], dr[32];
          tmem_ld32(tS + cc * 32, sr);
          tmem_ld32(tDP + cc * 32, dr);
          tmem_wait_ld();
          tmem_reg_fence(sr);
          tmem_reg_fence(dr);
          uint32_t pp[16], pd[16];
#pragma unroll
          for (int ii = 0; ii < 16; ++ii) {
            float pv[2], dv[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int qq = cc * 32 + 2 * ii + e;
              const int qg = q0 + qq;
              const bool vis = qg < p.N && (!CAUSAL || key <= qg);
              const float pr = vis ? ex2_approx(fmaf(__uint_as_float(sr[2 * ii + e]), c2, -lse2[qq])) : 0.f;
              pv[e] = pr;
              dv[e] = pr * (__uint_as_float(dr[2 * ii + e]) - dvec[qq]);
            }
            pp[ii] = pack2<T>(pv[0], pv[1]);
            pd[ii] = pack2<T>(dv[0], dv[1]);
          }
          tmem_st16(tS + cc * 16, pp);
          tmem_st16(tDP + cc * 16, pd);
          tmem_wait_st();   // the stores read pp, pd asynchronously; the next chunk reuses them
          tmem_reg_fence(pp);
          tmem_reg_fence(pd);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_ready);
      }
      if (!ok) break;
      bool w = mbar_wait(acc_full, acc_cnt & 1, p.status, abort_flag, kWhereOFull, lim);
      ++acc_cnt;
      if (!__all_sync(0xffffffffu, w)) { ok = false; *abort_flag = 1; break; }
      tc_fence_after();
      const bool valid = key < p.N;
      const size_t orow = (rbase + (valid ? key : 0)) * p.d_out;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t tA = tmem + lane_off + (which == 0 ? kColDV : kColDK);
        T* dst = reinterpret_cast<T*>(which == 0 ? p.dv : p.dk) + orow;
        const float mul = which == 0 ? 1.0f : p.scale;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t rr[32];
          tmem_ld32(tA + cc * 32, rr);   // every lane loads (warp-wide); rows past N do not store
          tmem_wait_ld();
          tmem_reg_fence(rr);
          if (valid) store_row32<T>(dst, cc * 32, p.d_out, rr, mul);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, Cfg::kTmemCols);
}

}  // namespace attn
