// Fused attention forward for sm_100a, head dim 256 (bf16 / fp16, and e4m3
// with per-block descale factors as in fwd_sm100.cuh).
//
// Same computation as fwd_sm100.cuh (exact attention with online softmax,
// running max m and sum l, division by l at the end; droidorbit.com,
// "Mathematical Formulation: The Online Softmax Rescaling Trick"), arranged
// for the larger head dim.  One 128-row Q tile per work unit: its O
// accumulator takes 256 TMEM columns, so two Q tiles no longer fit.  S is
// instead double-buffered in TMEM (S_a | S_b | O = 512 columns), which is the
// pages' intra-warpgroup two-stage pipeline (quantum-bit repost, second
// technical upgrade: while the softmax of the current tile runs, the tensor
// core computes the next tile's Q K^T and the previous tile's P V):
//
//   MMA issue order:  S(0), S(1), PV(0), S(2), PV(1), S(3), ...
//   softmax:          P(j) from S(j) while the tensor core runs PV(j-1), S(j+1)
//
// Roles (256 threads): warp 0 TMA, warp 1 MMA issuer (one thread) and TMEM
// allocator, warps 4-7 softmax (one thread per query row).  Shared memory:
// Q (64 KiB) and a two-stage K/V ring of 64 KiB tiles (e4m3: 32 KiB tiles, a
// four-stage ring).  P of key tile j is written over S(j) as 16-bit pairs (or
// e4m3 quads) and published in two 64-key halves.  Before publishing P(j)
// the softmax waits for PV(j-1) (it may rescale O).
#pragma once
#include "fwd_sm100.cuh"

namespace attn {

template <typename E>
struct Fwd256Cfg {
  static constexpr int kBytes = Elem<E>::kBytes;
  static constexpr int kChunkBytes = 128 * 128;   // 128 rows x 128 bytes
  static constexpr int kChunkCols = 128 / kBytes; // columns per chunk
  static constexpr int kChunks = 256 / kChunkCols;
  static constexpr int kTileBytes = kChunks * kChunkBytes;   // 64 KiB (32 KiB e4m3)
  static constexpr int kStages = kBytes == 2 ? 2 : 4;
  static constexpr int kKeysPerMma = 32 / kBytes; // 32 bytes of K per tcgen05.mma
  static constexpr int kThreads = 256;
  static constexpr int kTmemCols = 512;           // S_a | S_b | O
  static constexpr int kColO = 256;
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = kTileBytes;
  static constexpr int kOffBar = kOffKV + kStages * kTileBytes;
  static constexpr int kBarBytes = 256;
  static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;
};

// Position of K_j / V_j in a unit's load sequence, which follows the order
// the tensor core consumes them: K0, K1, V0, K2, V1, ..., K(n-1), V(n-2), V(n-1).
// With a two-stage ring each load then has one MMA block of time to land.
__device__ __forceinline__ uint32_t seq_k(int j) { return j == 0 ? 0u : static_cast<uint32_t>(2 * j - 1); }
__device__ __forceinline__ uint32_t seq_v(int j, int n) {
  return j == n - 1 ? static_cast<uint32_t>(2 * n - 1) : static_cast<uint32_t>(2 * j + 2);
}

template <typename E, bool CAUSAL>
__global__ void __launch_bounds__(256, 1) attn_fwd_sm100_d256_kernel(const __grid_constant__ FwdParams p) {
  using Cfg = Fwd256Cfg<E>;
  using T = typename Elem<E>::Out;
  constexpr bool kF8 = Elem<E>::kF8;
  constexpr int D = 256;
  constexpr int S = Cfg::kStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + Cfg::kOffQ;
  uint8_t* sKV = smem + Cfg::kOffKV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kOffBar);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* s_full = bars + 2;       // [2 S buffers]
  uint64_t* p_full = bars + 4;       // [2 key halves]
  uint64_t* o_ready = bars + 6;      // PV(j) completed
  uint64_t* o_full = bars + 7;       // last PV of the unit completed
  uint64_t* drain = bars + 8;
  uint64_t* kv_full = bars + 9;      // [S]
  uint64_t* kv_empty = bars + 9 + S; // [S]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 9 + 2 * S);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full + b, 1);
      mbar_init(p_full + b, 128);
    }
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
  const int n_kv = p.n_kv;
  const int n_qt = p.n_qpairs;          // 128-row Q tiles per head in this kernel
  const unsigned long long lim = p.wait_limit_ns;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      uint32_t kv_iter = 0, unit_iter = 0;
      int64_t skipped = -1;
      bool ok = true;
      for (int k = 0; ok; ++k, ++unit_iter) {
        const int unit = sched_unit(k, p.snake);
        if (unit >= p.n_units) break;
        int bh, qt;
        decode_unit<CAUSAL>(unit, n_qt, p.BH, p.order, bh, qt);
        const int n = CAUSAL ? min(qt + 1, n_kv) : n_kv;
        ok = mbar_wait(q_empty, (unit_iter & 1) ^ 1, p.status, abort_flag, kWhereQEmpty, lim);
        if (!ok) break;
        mbar_arrive_expect_tx(q_full, Cfg::kTileBytes);
        for (int c = 0; c < Cfg::kChunks; ++c)
          if (smem_range_ok(sQ + c * Cfg::kChunkBytes, Cfg::kChunkBytes, smem, Cfg::kOffQ, Cfg::kOffKV, p.status,
                            kChkQLoad))
            tma_load_4d(sQ + c * Cfg::kChunkBytes, &p.tm_q, q_full, c * Cfg::kChunkCols, qt * 128, bh % p.H,
                        bh / p.H);
        for (int q = 0; q < 2 * n && ok; ++q, ++kv_iter) {
          // q -> (K or V, key tile j), inverse of seq_k / seq_v
          const bool is_v = (q == 2 * n - 1) || (q > 0 && (q & 1) == 0);
          const int j = (q == 2 * n - 1) ? n - 1 : (is_v ? (q - 2) / 2 : (q + 1) / 2);
          const uint32_t s = kv_iter % S;
          ok = mbar_wait(kv_empty + s, ((kv_iter / S) & 1) ^ 1, p.status, abort_flag, kWhereKvEmpty, lim);
          if (!ok) break;
          if (p.fault == 1 && blockIdx.x == 0 && kv_iter == 0) {
            skipped = 0;  // test hook: this stage never completes
            continue;
          }
          mbar_arrive_expect_tx(kv_full + s, Cfg::kTileBytes);
          const CUtensorMap* map = is_v ? &p.tm_v : &p.tm_k;
          for (int c = 0; c < Cfg::kChunks; ++c)
            if (smem_range_ok(sKV + s * Cfg::kTileBytes + c * Cfg::kChunkBytes, Cfg::kChunkBytes, smem, Cfg::kOffKV,
                              Cfg::kOffBar, p.status, kChkKvLoad))
              tma_load_4d(sKV + s * Cfg::kTileBytes + c * Cfg::kChunkBytes, map, kv_full + s,
                          c * Cfg::kChunkCols, j * 128, bh % p.H, bh / p.H);
        }
      }
      if (!ok) {
        volatile int never = 0;
        for (uint32_t i = (kv_iter > S ? kv_iter - S : 0); i < kv_iter; ++i)
          if (static_cast<int64_t>(i) != skipped)
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
      constexpr uint32_t idesc_o = make_idesc(fmt, fmt, 0, 1, 128, 256);
      const uint64_t dQ = smem_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dK = smem_desc_sw128(smem_u32(sKV), 16, 1024);
      const uint64_t dV = smem_desc_sw128(smem_u32(sKV), Cfg::kChunkBytes, 1024);
      uint32_t kv_iter = 0, unit_iter = 0, p_cnt = 0;
      bool ok = true;

      auto issue_s = [&](int buf, uint32_t kstage) {
        const uint64_t b0 = dK + static_cast<uint64_t>((kstage * Cfg::kTileBytes) >> 4);
        if (!tmem_range_ok(tmem + buf * 128, tmem, 128, buf * 128, buf * 128 + 128, p.status, kChkSOut) ||
            !smem_range_ok(sQ, Cfg::kTileBytes, smem, Cfg::kOffQ, Cfg::kOffKV, p.status, kChkSQ) ||
            !smem_range_ok(sKV + kstage * Cfg::kTileBytes, Cfg::kTileBytes, smem, Cfg::kOffKV, Cfg::kOffBar,
                           p.status, kChkSK))
          return;
#pragma unroll
        for (int kk = 0; kk < D / Cfg::kKeysPerMma; ++kk) {
          // 32 bytes of the head dim per product, four per 128-byte chunk row
          const uint32_t off = ((kk >> 2) * Cfg::kChunkBytes + (kk & 3) * 32) >> 4;
          mma_ss(tmem + buf * 128, dQ + off, b0 + off, idesc_s, kk > 0, kF8);
        }
      };
      // O += P(j) V_j, each 64-key half as soon as it is published.  P:
      // kKeysPerMma keys = 8 TMEM columns per product; V: MN-major,
      // kKeysPerMma rows of 128-byte chunks per product.
      auto pv = [&](int buf, uint32_t vstage, bool acc) -> bool {
        const uint64_t b0 = dV + static_cast<uint64_t>((vstage * Cfg::kTileBytes) >> 4);
        constexpr int kSteps = 64 / Cfg::kKeysPerMma;
        const bool in_range =
            tmem_range_ok(tmem + Cfg::kColO, tmem, D, Cfg::kColO, Cfg::kColO + D, p.status, kChkOOut) &&
            tmem_range_ok(tmem + buf * 128, tmem, 64, buf * 128, buf * 128 + 64, p.status, kChkPIn) &&
            smem_range_ok(sKV + vstage * Cfg::kTileBytes, Cfg::kTileBytes, smem, Cfg::kOffKV, Cfg::kOffBar, p.status,
                          kChkVIn);
        for (int h = 0; h < 2; ++h) {
          if (!mbar_wait(p_full + h, p_cnt & 1, p.status, abort_flag, kWherePFull, lim)) return false;
          tc_fence_after();
          if (!in_range) continue;
#pragma unroll
          for (int kk = kSteps * h; kk < kSteps * (h + 1); ++kk)
            mma_ts(tmem + Cfg::kColO, tmem + buf * 128 + kk * 8, b0 + ((kk * Cfg::kKeysPerMma * 128) >> 4),
                   idesc_o, (acc || kk > 0) ? 1u : 0u, kF8);
        }
        ++p_cnt;
        return true;
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
        decode_unit<CAUSAL>(unit, n_qt, p.BH, p.order, bh_, qt);
        (void)bh_;
        const int n = CAUSAL ? min(qt + 1, n_kv) : n_kv;
        const uint32_t base = kv_iter;  // K_j at base + seq_k(j), V_j at base + seq_v(j, n)
        ok = mbar_wait(q_full, unit_iter & 1, p.status, abort_flag, kWhereQFull, lim);
        tc_fence_after();
        if (!ok) break;
        if (!(ok = wait_kv(base))) break;
        issue_s(0, base % S);
        mma_commit(s_full + 0);
        mma_commit(kv_empty + (base % S));
        for (int j = 1; j < n && ok; ++j) {
          // S(j) into buffer j%2: P(j-2) there was consumed by PV(j-2),
          // issued before this point (products run in issue order).
          const uint32_t ik = base + seq_k(j), iv = base + seq_v(j - 1, n);
          if (!(ok = wait_kv(ik))) break;
          issue_s(j & 1, ik % S);
          mma_commit(s_full + (j & 1));
          mma_commit(kv_empty + (ik % S));
          if (!(ok = wait_kv(iv))) break;
          if (!(ok = pv((j - 1) & 1, iv % S, j - 1 > 0))) break;
          mma_commit(o_ready);
          mma_commit(kv_empty + (iv % S));
        }
        if (!ok) break;
        const uint32_t iv = base + seq_v(n - 1, n);
        if (!(ok = wait_kv(iv))) break;
        if (!(ok = pv((n - 1) & 1, iv % S, n - 1 > 0))) break;
        mma_commit(o_ready);
        mma_commit(o_full);
        mma_commit(kv_empty + (iv % S));
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
    // -------------------------------------------------------------- softmax
    const int quarter = warp & 3;
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tO = tmem + lane_off + Cfg::kColO;
    uint32_t s_cnt[2] = {0, 0}, or_cnt = 0, o_cnt = 0;
    bool ok = true;
    // e4m3: P is multiplied by a power-of-two gain times v_descale[j] / max
    // v_descale before rounding, and the max may lag the true max by at most
    // kLazy (log2 units), so that P * gain <= 256 * 2^0.75 < 448 stays finite
    constexpr float kPGain = 256.0f;
    constexpr float kLazy = kF8 ? 0.75f : 8.0f;

    for (int k = 0; ok; ++k) {
      const int unit = sched_unit(k, p.snake);
      if (unit >= p.n_units) break;
      int bh, qt;
      decode_unit<CAUSAL>(unit, n_qt, p.BH, p.order, bh, qt);
      const int n = CAUSAL ? min(qt + 1, n_kv) : n_kv;
      const int row = qt * 128 + row_in_tile;
      float cq = p.scale_log2;   // score -> log2 domain factor (times the q descale for e4m3)
      float vmax = 1.0f;         // e4m3: max v descale of this head
      if constexpr (kF8) {
        const size_t dbase = static_cast<size_t>(bh) * n_kv;
        cq *= p.q_desc[dbase + min(qt, n_kv - 1)];
        float vm = 0.f;
        for (int b = lane; b < n_kv; b += 32) vm = fmaxf(vm, p.v_desc[dbase + b]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) vm = fmaxf(vm, __shfl_xor_sync(0xffffffffu, vm, o));
        vmax = vm;
      }
      float m = -INFINITY, l = 0.f;

      for (int j = 0; j < n; ++j) {
        const int buf = j & 1;
        const uint32_t tS = tmem + lane_off + buf * 128;
        bool w = mbar_wait(s_full + buf, s_cnt[buf] & 1, p.status, abort_flag, kWhereSFull, lim);
        ++s_cnt[buf];
        if (!__all_sync(0xffffffffu, w)) { ok = false; *abort_flag = 1; break; }
        tc_fence_after();
        float c = cq;
        float pgain = 1.0f;
        if constexpr (kF8) {
          const size_t dbase = static_cast<size_t>(bh) * n_kv;
          c = cq * p.k_desc[dbase + j];
          pgain = kPGain * __fdiv_rn(p.v_desc[dbase + j], vmax);
        }

        float s[128];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t r[32];
          if (tmem_range_ok(tS + cc * 32, tmem, 32, buf * 128, buf * 128 + 128, p.status, kChkSLoad))
            tmem_ld32(tS + cc * 32, r);
#pragma unroll
          for (int i = 0; i < 32; ++i) s[cc * 32 + i] = __uint_as_float(r[i]);
        }
        tmem_wait_ld();
        tmem_reg_fence(s);
        const int key0 = j * 128;
        const bool need_mask = (CAUSAL && key0 + 127 > qt * 128) || (key0 + 128 > p.N);
        if (need_mask) {
          const int lim_key = CAUSAL ? min(row, p.N - 1) : (p.N - 1);
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
        // first half of P into registers, then (after PV(j-1) has finished)
        // the optional rescale of O and the publication of both halves
        uint32_t pk0[kF8 ? 16 : 32];
        float sum = exp_half<kF8, T, false>(s, 0, c, -m, pgain, pk0);
        if (j > 0) {
          w = mbar_wait(o_ready, or_cnt & 1, p.status, abort_flag, kWhereOFull, lim);
          ++or_cnt;
          if (!__all_sync(0xffffffffu, w)) { ok = false; *abort_flag = 1; break; }
          tc_fence_after();
          if (__any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
              uint32_t r[32];
              if (!tmem_range_ok(tO + cc * 32, tmem, 32, Cfg::kColO, Cfg::kColO + D, p.status, kChkORescale))
                continue;
              tmem_ld32(tO + cc * 32, r);
              tmem_wait_ld();
              tmem_reg_fence(r);
#pragma unroll
              for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
              tmem_st32(tO + cc * 32, r);
              tmem_wait_st();     // the store reads r asynchronously
              tmem_reg_fence(r);
            }
          }
        }
        const bool p_ok = tmem_range_ok(tS, tmem, 64, buf * 128, buf * 128 + 64, p.status, kChkPStore);
        if (p_ok) store_p_half<kF8>(tS, 0, pk0);
        tc_fence_before();
        mbar_arrive(p_full + 0);
        if (p_ok)
          sum += need_mask ? exp_pack_half<kF8, T, false>(s, 1, c, -m, pgain, tS)
                           : exp_pack_half<kF8, T, true>(s, 1, c, -m, pgain, tS);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_full + 1);
        l = l * alpha + sum;
      }
      if (!ok) break;

      // ------------------------------------------------------------ epilogue
      // o_ready of the unit's last PV is consumed here too, keeping the phase
      // count in step with the MMA side
      bool w = mbar_wait(o_ready, or_cnt & 1, p.status, abort_flag, kWhereOFull, lim);
      ++or_cnt;
      w = w && mbar_wait(o_full, o_cnt & 1, p.status, abort_flag, kWhereOFull, lim);
      ++o_cnt;
      if (!__all_sync(0xffffffffu, w)) { ok = false; *abort_flag = 1; break; }
      tc_fence_after();
      const float inv_l = kF8 ? __fdiv_rn(vmax, kPGain * l) : 1.0f / l;
      // O rows are d_out wide (d_out <= D: smaller head dims run zero-padded
      // to D; the padding columns of O are zero and are not stored); O may be
      // strided over (batch, head, row)
      T* orow = reinterpret_cast<T*>(p.o) + static_cast<int64_t>(bh / p.H) * p.o_sb +
                static_cast<int64_t>(bh % p.H) * p.o_sh + static_cast<int64_t>(row) * p.o_sn;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t r[32];
        if (tmem_range_ok(tO + cc * 32, tmem, 32, Cfg::kColO, Cfg::kColO + D, p.status, kChkOLoad))
          tmem_ld32(tO + cc * 32, r);
        tmem_wait_ld();
        tmem_reg_fence(r);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack2<T>(__uint_as_float(r[2 * i]) * inv_l, __uint_as_float(r[2 * i + 1]) * inv_l);
        if (row < p.N) {
          uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
          const int groups = min(4, (p.d_out - cc * 32) >> 3);   // 8 values per 16-byte store
#pragma unroll
          for (int i = 0; i < 4; ++i)
            if (i < groups) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
      if (p.lse != nullptr && row < p.N)
        p.lse[static_cast<size_t>(bh) * p.N + row] = (m + __log2f(l)) * 0.69314718055994530942f;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, Cfg::kTmemCols);
}

}  // namespace attn
