// Fused attention backward for sm_100a: one pass over the key tiles that
// produces dK, dV and dQ together (five N x N x d products instead of the
// seven of the two-kernel path), with dQ summed across key tiles by fp32
// TMA reduce-adds (atomic in L2).  Same gradients as bwd_sm100.cuh ("FlashAttention-3"
// explainer, droidorbit.com, definition Softmax(Q K^T / sqrt(d)) V, chain
// rule):
//
//   P = exp(scale * Q K^T - LSE),  dV = P^T dO,  dS = P * (dO V^T - D),
//   dK = scale * dS^T Q,           dQ = scale * dS K,   D = rowsum(dO * O)
//
// Three launches:
//   attn_bwd_prep_kernel   D and LSE * log2(e) per query row (row-statistics
//                          workspace) and zeroes the fp32 dQ accumulator;
//   attn_bwd_fused_kernel  one 128-key tile per work unit, all Q tiles it
//                          meets;
//   attn_bwd_dq_convert_kernel  dQ = scale * accumulator, rounded to 16 bits.
//
// Fused kernel, per Q tile i of the unit's key tile j (TMEM columns at d=128:
// S^T 0-127 | dP^T 128-255 | dV 256-383 | dK 384-511):
//   MMA   S^T = K Q_i^T, dP^T = V dO_i^T (SS, both K-major)
//   rows  two warpgroups, thread = key, queries 0-63 and 64-127.  Phase 1,
//         as soon as S^T is done: P^T, 16-bit, packed into TMEM columns 32-95
//         of S^T (each warpgroup writes only columns it has already read);
//         dV += P^T dO_i starts then and releases dO_i.  Phase 2, once dP^T
//         is done: dS = P (dP - D) from that 16-bit P, packed into columns
//         32-95 of dP^T, and dS into shared memory (query-contiguous rows,
//         the MN-major A operand of the dQ product)
//   MMA   dV += P^T dO_i, dK += dS^T Q_i (TS), dQ_i = dS K_j (SS, both
//         MN-major) into the dP^T columns, which dK has just consumed
//   dQ    one warpgroup, thread = query: TMEM -> registers (the next dP^T
//         may then start), then 32 x 32 fp32 boxes staged in shared memory
//         and added into the accumulator by TMA reduce-add.
// Shared memory at d=128: K, V, two Q stages, one dO buffer (released right
// after the dV product), dS, two dQ staging buffers: 7 x 32 KiB.
// At d=64 dQ has columns of its own (384-447).  Every wait is bounded.
#pragma once
#include "bwd_sm100.cuh"

namespace attn {

template <int D>
struct FusedCfg {
  static constexpr int kChunkBytes = 128 * 128;
  static constexpr int kChunks = D / 64;
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  static constexpr int kQStages = (D == 64) ? 3 : 2;          // Q ring (with the row statistics)
  static constexpr int kDoStages = (D == 64) ? 2 : 1;         // dO ring: released right after dV
  static constexpr int kRowBytes = 2 * 128 * 4;
  static constexpr int kOffV = kTileBytes;
  static constexpr int kOffQ = 2 * kTileBytes;
  static constexpr int kOffDo = kOffQ + kQStages * kTileBytes;
  static constexpr int kOffDS = kOffDo + kDoStages * kTileBytes;    // dS: 128 keys x 128 queries, 16-bit
  static constexpr int kOffStage = kOffDS + 2 * kChunkBytes;       // dQ staging: two 16 KiB box buffers
  static constexpr int kStageBytes = kChunkBytes;
  static constexpr int kOffRow = kOffStage + 2 * kStageBytes;
  static constexpr int kOffBar = kOffRow + kQStages * kRowBytes;
  static constexpr int kSmem = kOffBar + 256;                  // base must be 1 KiB aligned (checked)
  static constexpr int kThreads = 512;
  static constexpr int kTmemCols = 512;
  static constexpr int kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + D;
  static constexpr bool kDqShared = (D != 64);                 // dQ over the dP^T columns
  static constexpr int kColDQ = kDqShared ? kColDP : 384;
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
};

enum : int { kErrLayout = 4, kWhereLayout = 9 };

// ---------------------------------------------------------------------------
// D = rowsum(dO * O), LSE * log2(e) per row; dQ accumulator rows set to 0.
// One 128-row tile per CTA of 256 threads, 16 threads per row (d <= 128).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) attn_bwd_prep_kernel(const T* __restrict__ o, const T* __restrict__ d_o,
                                                            const float* __restrict__ lse, float* rows,
                                                            float* dq_acc, int N, int n_t, int d) {
  const int tile = blockIdx.x;   // bh * n_t + q tile
  const int bh = tile / n_t, qt = tile % n_t;
  const int seg = threadIdx.x & 15;
  float* out = rows + static_cast<size_t>(tile) * 256;
  for (int rr = threadIdx.x >> 4; rr < 128; rr += 16) {
    const int row = qt * 128 + rr;
    const bool valid = row < N;
    float dsum = 0.f;
    if (valid && seg * 8 < d) {
      const size_t off = (static_cast<size_t>(bh) * N + row) * d + seg * 8;
      const uint4 a = *reinterpret_cast<const uint4*>(d_o + off);
      const uint4 b = *reinterpret_cast<const uint4*>(o + off);
      const T* ta = reinterpret_cast<const T*>(&a);
      const T* tb = reinterpret_cast<const T*>(&b);
#pragma unroll
      for (int e = 0; e < 8; ++e) dsum = fmaf(static_cast<float>(ta[e]), static_cast<float>(tb[e]), dsum);
      float4* z = reinterpret_cast<float4*>(dq_acc + off);
      z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int m = 8; m >= 1; m >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, m);
    if (seg == 0) {
      out[rr] = valid ? lse[static_cast<size_t>(bh) * N + row] * 1.4426950408889634f : 0.f;
      out[128 + rr] = dsum;
    }
  }
}

// dq = scale * acc, eight elements per step.
template <typename T>
__global__ void __launch_bounds__(256) attn_bwd_dq_convert_kernel(const float* __restrict__ acc, T* __restrict__ dq,
                                                                  size_t n8, float scale) {
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float4 a = reinterpret_cast<const float4*>(acc)[2 * i];
    const float4 b = reinterpret_cast<const float4*>(acc)[2 * i + 1];
    reinterpret_cast<uint4*>(dq)[i] = make_uint4(pack2<T>(a.x * scale, a.y * scale), pack2<T>(a.z * scale, a.w * scale),
                                                 pack2<T>(b.x * scale, b.y * scale), pack2<T>(b.z * scale, b.w * scale));
  }
}

// ---------------------------------------------------------------------------
// The fused kernel
// ---------------------------------------------------------------------------
// Register split (setmaxnreg, per warpgroup): 512 threads launch with 128
// registers each.  d=128: the TMA/MMA warpgroup gives 40 to the row
// warpgroups and the dQ warpgroup, which holds a whole 128-column dQ tile
// (88 + 136 + 136 + 152 = 4 * 128).  d=64: the MMA issuer runs the look-ahead
// order (below) and keeps 112, the row warpgroups 128, the dQ warpgroup 144.
template <int D>
struct BwdRegs {
  static constexpr int kLow = D == 64 ? 112 : 88;
  static constexpr int kRows = D == 64 ? 128 : 136;
  static constexpr int kDq = D == 64 ? 144 : 152;
  static_assert(128 * kLow + 256 * kRows + 128 * kDq <= 512 * 128, "register split exceeds the launch pool");
};

template <typename E, int D, bool CAUSAL>
__global__ void __launch_bounds__(512, 1) attn_bwd_fused_kernel(const __grid_constant__ BwdParams p) {
  using Cfg = FusedCfg<D>;
  using T = E;
  constexpr int SQ = Cfg::kQStages, SD = Cfg::kDoStages;
  extern __shared__ __align__(1024) uint8_t smem[];
  // The layout fills the 227 KiB budget at d=128 with no room to realign.
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) report_error(p.status, kErrLayout, kWhereLayout);
    return;
  }
  uint8_t* sK = smem;
  uint8_t* sV = smem + Cfg::kOffV;
  uint8_t* sQ = smem + Cfg::kOffQ;
  uint8_t* sDo = smem + Cfg::kOffDo;
  uint8_t* sDS = smem + Cfg::kOffDS;       // dS, the A operand of the dQ product
  uint8_t* sStage = smem + Cfg::kOffStage;
  const float* sRows = reinterpret_cast<const float*>(smem + Cfg::kOffRow);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kOffBar);
  uint64_t* kv_full = bars + 0;
  uint64_t* kv_empty = bars + 1;
  uint64_t* s_full = bars + 2;       // S^T in TMEM
  uint64_t* p_ready = bars + 3;      // P^T, dS^T in TMEM and dS in shared memory
  uint64_t* dq_full = bars + 4;      // dQ_i in TMEM
  uint64_t* dq_empty = bars + 5;     // dQ_i loaded out of TMEM
  uint64_t* acc_full = bars + 6;     // dV, dK of the unit complete
  uint64_t* drain = bars + 7;
  uint64_t* q_full = bars + 8;                 // [SQ] Q tile and its row statistics
  uint64_t* q_empty = bars + 8 + SQ;           // [SQ]
  uint64_t* do_full = bars + 8 + 2 * SQ;       // [SD]
  uint64_t* do_empty = bars + 8 + 2 * SQ + SD; // [SD]
  uint64_t* dp_full = bars + 8 + 2 * SQ + 2 * SD;   // dP^T in TMEM
  uint64_t* pt_ready = bars + 9 + 2 * SQ + 2 * SD;  // packed P^T in TMEM (both row warpgroups)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 10 + 2 * SQ + 2 * SD);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  constexpr int kColS = Cfg::kColS, kColDP = Cfg::kColDP, kColDV = Cfg::kColDV, kColDK = Cfg::kColDK;
  constexpr int kColDQ = Cfg::kColDQ;
  constexpr int kPk = 32;            // packed P^T / dS^T start 32 columns into S^T / dP^T
  // Look-ahead order (d=64, where dQ has columns of its own): S^T of the next
  // tile is issued right after dV of this one, into the columns dV has just
  // read, so the row warpgroups find it done when they finish dS.  At d=128,
  // S^T of the next tile follows dQ instead, where it covers the load of dQ
  // out of the columns the next dP^T takes (measured: look-ahead -10 % at
  // d=128, +12-17 % at d=64).
  constexpr bool kAhead = !Cfg::kDqShared;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(pt_ready, 256);
    mbar_init(p_ready, 256);
    mbar_init(dq_full, 1);
    mbar_init(dq_empty, 128);
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    for (int s = 0; s < SQ; ++s) {
      mbar_init(q_full + s, 1);
      mbar_init(q_empty + s, 1);
    }
    for (int s = 0; s < SD; ++s) {
      mbar_init(do_full + s, 1);
      mbar_init(do_empty + s, 1);
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
  auto key_tile = [&](int blk) { return CAUSAL ? n_t - 1 - blk : blk; };

  if (warp < 4) {
  reg_dealloc<BwdRegs<D>::kLow>();
  if (warp == 0) {
    // ------------------------------------------------------------------ TMA
    if (lane == 0) {
      uint32_t nq = 0, nd = 0, unit_iter = 0;   // Q and dO tiles issued, units started
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
        for (int i = i0; i < n_t && ok; ++i) {
          const uint32_t sq = nq % SQ;
          ok = mbar_wait(q_empty + sq, ((nq / SQ) & 1) ^ 1, p.status, abort_flag, kWhereKvEmpty, lim);
          if (!ok) break;
          mbar_arrive_expect_tx(q_full + sq, Cfg::kTileBytes + Cfg::kRowBytes);
          for (int c = 0; c < Cfg::kChunks; ++c)
            tma_load_4d(sQ + sq * Cfg::kTileBytes + c * Cfg::kChunkBytes, &p.tm_q, q_full + sq, c * 64, i * 128, h, b);
          bulk_load(smem + Cfg::kOffRow + sq * Cfg::kRowBytes, p.rows + (static_cast<size_t>(bh) * n_t + i) * 256,
                    Cfg::kRowBytes, q_full + sq);
          ++nq;
          const uint32_t sd = nd % SD;
          ok = mbar_wait(do_empty + sd, ((nd / SD) & 1) ^ 1, p.status, abort_flag, kWhereKvEmpty, lim);
          if (!ok) break;
          mbar_arrive_expect_tx(do_full + sd, Cfg::kTileBytes);
          for (int c = 0; c < Cfg::kChunks; ++c)
            tma_load_4d(sDo + sd * Cfg::kTileBytes + c * Cfg::kChunkBytes, &p.tm_do, do_full + sd, c * 64, i * 128, h, b);
          ++nd;
        }
      }
      if (!ok) {
        // let the copies already issued land before the CTA exits
        volatile int never = 0;
        for (uint32_t i = (nq > SQ ? nq - SQ : 0); i < nq; ++i)
          mbar_wait(q_full + (i % SQ), (i / SQ) & 1, nullptr, &never, kWhereDrain, 100000000ull);
        for (uint32_t i = (nd > SD ? nd - SD : 0); i < nd; ++i)
          mbar_wait(do_full + (i % SD), (i / SD) & 1, nullptr, &never, kWhereDrain, 100000000ull);
        if (unit_iter > 0) mbar_wait(kv_full, (unit_iter - 1) & 1, nullptr, &never, kWhereDrain, 100000000ull);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t fmt = Elem<E>::kFmt;
      constexpr uint32_t idesc_kk = make_idesc(fmt, fmt, 0, 0, 128, 128);   // S^T, dP^T
      constexpr uint32_t idesc_acc = make_idesc(fmt, fmt, 0, 1, 128, D);    // dV, dK: A in TMEM, B MN-major
      constexpr uint32_t idesc_dq = make_idesc(fmt, fmt, 1, 1, 128, D);     // dQ: A, B MN-major
      const uint64_t dKd = smem_desc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dVd = smem_desc_sw128(smem_u32(sV), 16, 1024);
      const uint64_t dKmn = smem_desc_sw128(smem_u32(sK), Cfg::kChunkBytes, 1024);
      const uint64_t dDS = smem_desc_sw128(smem_u32(sDS), Cfg::kChunkBytes, 1024);
      const uint64_t dQk = smem_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dQmn = smem_desc_sw128(smem_u32(sQ), Cfg::kChunkBytes, 1024);
      const uint64_t dDok = smem_desc_sw128(smem_u32(sDo), 16, 1024);
      const uint64_t dDomn = smem_desc_sw128(smem_u32(sDo), Cfg::kChunkBytes, 1024);
      uint32_t q_iter = 0, unit_iter = 0;
      bool ok = true;
      auto kmajor = [&](uint32_t d_col, uint64_t a0, uint64_t b0) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * Cfg::kChunkBytes + (kk & 3) * 32) >> 4;
          mma_ss(tmem + d_col, a0 + off, b0 + off, idesc_kk, kk > 0, false);
        }
      };
      // A = 128 keys x 128 queries, 16-bit packed from column a_col (8 columns per 16 queries)
      auto accum = [&](uint32_t d_col, uint32_t a_col, uint64_t b0, bool acc) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + d_col, tmem + a_col + kk * 8, b0 + ((kk * 16 * 128) >> 4), idesc_acc,
                 (acc || kk > 0) ? 1u : 0u, false);
      };
      // dQ may be overwritten once the previous tile's dQ has been loaded out
      auto wait_dq_free = [&]() -> bool {
        if (q_iter == 0) return true;
        bool r = mbar_wait(dq_empty, (q_iter - 1) & 1, p.status, abort_flag, kWhereOFull, lim);
        tc_fence_after();
        return r;
      };
      // look-ahead order only: S^T and dP^T of tile t
      auto issue_st = [&](uint32_t t) -> bool {
        const uint32_t sq = t % SQ;
        if (!mbar_wait(q_full + sq, (t / SQ) & 1, p.status, abort_flag, kWhereKvFull, lim)) return false;
        tc_fence_after();
        kmajor(kColS, dKd, dQk + ((sq * Cfg::kTileBytes) >> 4));
        mma_commit(s_full);
        return true;
      };
      auto issue_dpt = [&](uint32_t t) -> bool {
        const uint32_t sd = t % SD;
        if (!mbar_wait(do_full + sd, (t / SD) & 1, p.status, abort_flag, kWhereKvFull, lim)) return false;
        tc_fence_after();
        kmajor(kColDP, dVd, dDok + ((sd * Cfg::kTileBytes) >> 4));
        mma_commit(dp_full);
        return true;
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
        if constexpr (kAhead) {
          // dV(t); S^T(t+1) into the columns dV(t) has just read; dK(t), dQ(t)
          // (dQ in columns of its own, once dQ(t-1) is out); dP^T(t+1)
          if (!(ok = issue_st(q_iter) && issue_dpt(q_iter))) break;
          for (int i = i0; i < n_t && ok; ++i, ++q_iter) {
            const uint32_t sq = q_iter % SQ, sd = q_iter % SD;
            const uint32_t qoff = (sq * Cfg::kTileBytes) >> 4, dooff = (sd * Cfg::kTileBytes) >> 4;
            if (!(ok = mbar_wait(pt_ready, q_iter & 1, p.status, abort_flag, kWherePFull, lim))) break;
            tc_fence_after();
            accum(kColDV, kColS + kPk, dDomn + dooff, i > i0);   // dV += P^T dO_i
            mma_commit(do_empty + sd);
            if (i + 1 < n_t && !(ok = issue_st(q_iter + 1))) break;
            if (!(ok = mbar_wait(p_ready, q_iter & 1, p.status, abort_flag, kWherePFull, lim))) break;
            tc_fence_after();
            accum(kColDK, kColDP + kPk, dQmn + qoff, i > i0);    // dK += dS^T Q_i
            mma_commit(q_empty + sq);
            if (!(ok = wait_dq_free())) break;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ss(tmem + kColDQ, dDS + ((kk * 16 * 128) >> 4), dKmn + ((kk * 16 * 128) >> 4), idesc_dq,
                     kk > 0 ? 1u : 0u, false);
            mma_commit(dq_full);
            if (i + 1 < n_t && !(ok = issue_dpt(q_iter + 1))) break;
          }
          if (!ok) break;
          mma_commit(acc_full);
          mma_commit(kv_empty);
          continue;
        }
        for (int i = i0; i < n_t && ok; ++i, ++q_iter) {
          const uint32_t sq = q_iter % SQ, sd = q_iter % SD;
          if (!(ok = mbar_wait(q_full + sq, (q_iter / SQ) & 1, p.status, abort_flag, kWhereKvFull, lim))) break;
          tc_fence_after();
          const uint32_t qoff = (sq * Cfg::kTileBytes) >> 4, dooff = (sd * Cfg::kTileBytes) >> 4;
          // S^T over P^T of the previous tile (consumed by the dV product
          // issued before); dP^T over dS^T (consumed by dK) and, at d=128,
          // over the previous dQ once it has been loaded out
          kmajor(kColS, dKd, dQk + qoff);
          mma_commit(s_full);
          if (Cfg::kDqShared && !(ok = wait_dq_free())) break;
          if (!(ok = mbar_wait(do_full + sd, (q_iter / SD) & 1, p.status, abort_flag, kWhereKvFull, lim))) break;
          tc_fence_after();
          kmajor(kColDP, dVd, dDok + dooff);
          mma_commit(dp_full);
          // dV as soon as P^T is packed (phase 1): dO is released while the
          // row warpgroups still compute dS
          if (!(ok = mbar_wait(pt_ready, q_iter & 1, p.status, abort_flag, kWherePFull, lim))) break;
          tc_fence_after();
          accum(kColDV, kColS + kPk, dDomn + dooff, i > i0);   // dV += P^T dO_i
          mma_commit(do_empty + sd);
          if (!(ok = mbar_wait(p_ready, q_iter & 1, p.status, abort_flag, kWherePFull, lim))) break;
          tc_fence_after();
          accum(kColDK, kColDP + kPk, dQmn + qoff, i > i0);    // dK += dS^T Q_i
          mma_commit(q_empty + sq);
          if (!Cfg::kDqShared && !(ok = wait_dq_free())) break;
          // dQ_i = dS K_j: 16 keys (16 rows of 128 bytes in both operands) per product
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tmem + kColDQ, dDS + ((kk * 16 * 128) >> 4), dKmn + ((kk * 16 * 128) >> 4), idesc_dq,
                   kk > 0 ? 1u : 0u, false);
          mma_commit(dq_full);
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
  }
  } else if (warp < 12) {
    if constexpr (BwdRegs<D>::kRows > 128) reg_alloc<BwdRegs<D>::kRows>();
    // ------------------------------------------------------------- key rows
    const int half = (warp - 4) >> 2;          // queries 64*half .. 64*half+63
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + kColS;
    const uint32_t tDP = tmem + lane_off + kColDP;
    const float c2 = p.scale_log2;
    uint8_t* ds_row = sDS + half * Cfg::kChunkBytes + r * 128;
    const int sw = r & 7;
    uint32_t t = 0, acc_cnt = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int unit = sched_unit(k, p.snake);
      if (unit >= p.n_units) break;
      int bh, blk;
      decode_unit<CAUSAL>(unit, n_t, p.BH, p.order, bh, blk);
      const int j = key_tile(blk);
      const int i0 = CAUSAL ? j : 0;
      const int key = j * 128 + r;
      const bool key_ok = key < p.N;
      const size_t rbase = static_cast<size_t>(bh) * p.N;
      for (int i = i0; i < n_t; ++i, ++t) {
        const uint32_t s = t % SQ;
        bool w = mbar_wait(q_full + s, (t / SQ) & 1, p.status, abort_flag, kWhereKvFull, lim);
        w = w && mbar_wait(s_full, t & 1, p.status, abort_flag, kWhereSFull, lim);
        if (!__all_sync(0xffffffffu, w)) { ok = false; *abort_flag = 1; break; }
        tc_fence_after();
        const float* lse2 = sRows + s * 256;
        const float* dvec = lse2 + 128;
        const int q0 = i * 128;
        // every pair of this tile is visible: no per-element mask
        const bool full = !(CAUSAL && i == j) && q0 + 128 <= p.N && j * 128 + 128 <= p.N;
        // Phase 1 (S^T only, while dP^T may still be computed): P for this
        // warpgroup's 64 queries, packed to 16 bits into columns
        // 32 + 32*half .. of S^T (inside the 64 columns it has just read) --
        // the A operand of dV, which starts as soon as both halves are in.
        uint32_t pp[32];   // P of this warpgroup's 64 queries, 16-bit pairs
        {
          uint32_t sr[64];
          tmem_ld32(tS + (2 * half) * 32, *reinterpret_cast<uint32_t(*)[32]>(sr));
          tmem_ld32(tS + (2 * half + 1) * 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
          tmem_wait_ld();
          tmem_reg_fence(sr);
#pragma unroll
          for (int x4 = 0; x4 < 16; ++x4) {
            const float4 lv = reinterpret_cast<const float4*>(lse2 + half * 64)[x4];   // broadcast reads
            const float l4[4] = {lv.x, lv.y, lv.z, lv.w};
            float pv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int x = 4 * x4 + e;
              float pr = ex2_approx(fmaf(__uint_as_float(sr[x]), c2, -l4[e]));
              if (!full) {
                const int qg = q0 + half * 64 + x;
                const bool vis = key_ok && qg < p.N && (!CAUSAL || key <= qg);
                pr = vis ? pr : 0.f;
              }
              pv[e] = pr;
            }
            pp[2 * x4] = pack2<T>(pv[0], pv[1]);
            pp[2 * x4 + 1] = pack2<T>(pv[2], pv[3]);
          }
          tmem_st32(tS + kPk + half * 32, pp);
        }
        tmem_wait_st();
        tmem_reg_fence(pp);
        tc_fence_before();
        mbar_arrive(pt_ready);
        w = mbar_wait(dp_full, t & 1, p.status, abort_flag, kWhereSFull, lim);
        if (!__all_sync(0xffffffffu, w)) { ok = false; *abort_flag = 1; break; }
        tc_fence_after();
        // Phase 2: dS = P (dP - D) with the 16-bit P of phase 1.  Chunks of 32
        // queries, in an order that makes every packed dS^T write land on
        // columns of dP^T this warpgroup has already read: half 0 reads 0-63
        // and writes 32-63 (chunk 1 first), half 1 reads 64-127 and writes
        // 64-95.
#pragma unroll
        for (int n = 0; n < 2; ++n) {
          const int cc = half == 0 ? 1 - n : 2 + n;
          // P of queries 32cc .. 32cc+31: from phase 1's registers under the
          // look-ahead order (S^T of the next tile may already overwrite its
          // columns), else read back from TMEM
          uint32_t pr16[16], dr[32];
          if constexpr (kAhead) {
#pragma unroll
            for (int x = 0; x < 16; ++x) pr16[x] = pp[(cc - 2 * half) * 16 + x];
          } else {
            tmem_ld16(tS + kPk + cc * 16, pr16);
          }
          tmem_ld32(tDP + cc * 32, dr);
          tmem_wait_ld();
          if constexpr (!kAhead) tmem_reg_fence(pr16);
          tmem_reg_fence(dr);
          uint32_t pd[16];
#pragma unroll
          for (int x4 = 0; x4 < 8; ++x4) {
            const float4 dv = reinterpret_cast<const float4*>(dvec + cc * 32)[x4];
            const float2 p01 = unpack2<T>(pr16[2 * x4]);
            const float2 p23 = unpack2<T>(pr16[2 * x4 + 1]);
            pd[2 * x4] = pack2<T>(p01.x * (__uint_as_float(dr[4 * x4]) - dv.x),
                                  p01.y * (__uint_as_float(dr[4 * x4 + 1]) - dv.y));
            pd[2 * x4 + 1] = pack2<T>(p23.x * (__uint_as_float(dr[4 * x4 + 2]) - dv.z),
                                      p23.y * (__uint_as_float(dr[4 * x4 + 3]) - dv.w));
          }
          tmem_st16(tDP + kPk + cc * 16, pd);
          // dS row `key`, queries 32cc..32cc+31: 16-byte groups 4(cc%2)..+3 of
          // this half's chunk, 128-byte swizzled
#pragma unroll
          for (int gg = 0; gg < 4; ++gg) {
            const int g = (cc & 1) * 4 + gg;
            *reinterpret_cast<uint4*>(ds_row + ((g ^ sw) << 4)) =
                make_uint4(pd[4 * gg], pd[4 * gg + 1], pd[4 * gg + 2], pd[4 * gg + 3]);
          }
          tmem_wait_st();   // the TMEM store reads pd asynchronously; the next chunk reuses it
          tmem_reg_fence(pd);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(p_ready);
      }
      if (!ok) break;
      bool w = mbar_wait(acc_full, acc_cnt & 1, p.status, abort_flag, kWhereOFull, lim);
      ++acc_cnt;
      if (!__all_sync(0xffffffffu, w)) { ok = false; *abort_flag = 1; break; }
      tc_fence_after();
      // half 0 stores dV, half 1 stores dK (times scale)
      const uint32_t tA = tmem + lane_off + (half == 0 ? kColDV : kColDK);
      T* dst = reinterpret_cast<T*>(half == 0 ? p.dv : p.dk) + (rbase + (key_ok ? key : 0)) * p.d_out;
      const float mul = half == 0 ? 1.0f : p.scale;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t rr[32];
        tmem_ld32(tA + cc * 32, rr);   // every lane loads (warp-wide); rows past N do not store
        tmem_wait_ld();
        tmem_reg_fence(rr);
        if (key_ok) store_row32<T>(dst, cc * 32, p.d_out, rr, mul);
      }
    }
  } else {
    reg_alloc<BwdRegs<D>::kDq>();
    // ------------------------------------------------------------ dQ rows
    // Thread = query row.  The whole dQ tile goes to registers (then the
    // next dP^T may overwrite the columns), then 32 x 32 fp32 boxes, staged
    // in this warp's 4 KiB slice of two box buffers, are added into the
    // accumulator by TMA reduce-add.
    const int quarter = warp & 3;              // rows 32*quarter .. +31 of the Q tile
    const uint32_t tDQ = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + kColDQ;
    uint8_t* stage = sStage + quarter * 4096 + lane * 128;
    const int sw = lane & 7;
    uint32_t t = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int unit = sched_unit(k, p.snake);
      if (unit >= p.n_units) break;
      int bh, blk;
      decode_unit<CAUSAL>(unit, n_t, p.BH, p.order, bh, blk);
      const int j = key_tile(blk);
      const int i0 = CAUSAL ? j : 0;
      for (int i = i0; i < n_t; ++i, ++t) {
        bool w = mbar_wait(dq_full, t & 1, p.status, abort_flag, kWhereDrain, lim);
        if (!__all_sync(0xffffffffu, w)) { ok = false; *abort_flag = 1; break; }
        tc_fence_after();
        uint32_t rr[D];
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) tmem_ld32(tDQ + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(rr + cc * 32));
        tmem_wait_ld();
        tmem_reg_fence(rr);
        tc_fence_before();
        mbar_arrive(dq_empty);
        const int row0 = i * 128 + quarter * 32;
#pragma unroll
        for (int m = 0; m < D / 32; ++m) {
          // buffer m % 2 is free once at most one (the other buffer's) box is still read
          if (lane == 0) bulk_wait_group_read<1>();
          __syncwarp();
          uint8_t* dst = stage + (m & 1) * Cfg::kStageBytes;
#pragma unroll
          for (int g = 0; g < 8; ++g)
            *reinterpret_cast<uint4*>(dst + ((g ^ sw) << 4)) =
                make_uint4(rr[32 * m + 4 * g], rr[32 * m + 4 * g + 1], rr[32 * m + 4 * g + 2], rr[32 * m + 4 * g + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (row0 < p.N && 32 * m < p.d_out)
              tma_reduce_add_3d(&p.tm_dq, sStage + (m & 1) * Cfg::kStageBytes + quarter * 4096, 32 * m, row0, bh);
            bulk_commit_group();
          }
        }
      }
    }
    if (lane == 0) bulk_wait_group<0>();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, Cfg::kTmemCols);
}

}  // namespace attn
