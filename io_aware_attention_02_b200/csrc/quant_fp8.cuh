// Per-block e4m3 quantisation with optional incoherent processing.
//
// Block-wise quantisation (one scale per block, not per tensor) and
// incoherent processing (rotate Q and K by a random orthogonal matrix, here
// diag(signs) times the Sylvester Hadamard matrix over the head dim, so that
// outliers are spread across coordinates before rounding): quantum-bit repost
// "H100 utilisation 75% ... FlashAttention-3", third technical upgrade;
// "FlashAttention-3 (HE)" (systems-analysis.info), "Technical innovations",
// item 3.  The rotation leaves Q K^T unchanged because it is orthogonal.
//
// Pure streaming kernel: 2 bytes read and 1 byte written per element, bound
// by HBM bandwidth.  Persistent CTAs (two or three per SM) walk the blocks of
// 128 rows of one (batch, head) in a strided order.  A block is one
// contiguous run of 128 * D bf16 values, so one thread copies it into shared
// memory with a single bulk copy; a ring of kStages such copies per CTA keeps
// bytes in flight while the CTA works on the oldest one.  Each row is handled
// by D/8 threads holding 8 consecutive values: the fast Walsh-Hadamard
// transform runs three butterfly stages in registers and the rest across
// lanes with shuffles.  The block's amax needs every row, so the CTA meets at
// one barrier per block; that barrier also tells the copying thread that the
// block's buffer has been read and may be refilled.
#pragma once
#include "ptx.cuh"

namespace attn {

enum : int { kWhereQuantFull = 10 };

struct QuantParams {
  const __nv_bfloat16* x;   // [BH][N][D]
  uint8_t* x8;              // [BH][N][D] e4m3 codes
  float* descale;           // [BH][n_blocks]
  const float* signs;       // [D] or nullptr
  int* status;
  unsigned long long wait_limit_ns;
  int N, n_blocks, total;   // total = BH * n_blocks
  int hadamard;
};

template <int D>
struct QuantCfg {
  static constexpr int kRows = 128;
  static constexpr int kTileBytes = kRows * D * 2;
  // 3 x 32 KiB per CTA and two CTAs per SM at D = 128; 4 x 16 KiB and three
  // CTAs per SM at D = 64 (registers allow it there).
  static constexpr int kStages = D == 64 ? 4 : 3;
  static constexpr int kMinBlocks = D == 64 ? 3 : 2;
  static constexpr int kBarOff = kStages * kTileBytes;
  static constexpr int kAbortOff = kBarOff + 64;
  static constexpr int kRedOff = kBarOff + 128;             // float [2][8]
  static constexpr int kSmem = kBarOff + 256;
  static_assert(kStages * 8 <= 64, "barriers overflow their slot");
};

// e4m3 codes of y[0..3] / s, identical to rounding the IEEE fp32 quotient
// RN(y / s) to e4m3, without a division in the common case.  With r_lo and
// r_hi the reciprocal of s moved down and up by a relative 2^-20, the
// products RN(y r_lo) and RN(y r_hi) bracket RN(y / s): every rounding on the
// way (reciprocal, nudge, product, quotient) moves a value by at most 2^-24
// relative, far less than the nudge.  Rounding to e4m3 is monotone, so when
// both ends of the bracket give the same code the quotient gives it too.
// Otherwise the quotient lies within about 2^-20 of an e4m3 rounding
// midpoint (a few values in ten thousand) and is taken by division.
__device__ __forceinline__ uint32_t quant4_e4m3(const float* y, float s, float r_lo, float r_hi, bool fast) {
  if (fast) {
    const uint32_t a = pack4_e4m3(__fmul_rn(y[0], r_lo), __fmul_rn(y[1], r_lo), __fmul_rn(y[2], r_lo),
                                  __fmul_rn(y[3], r_lo));
    const uint32_t b = pack4_e4m3(__fmul_rn(y[0], r_hi), __fmul_rn(y[1], r_hi), __fmul_rn(y[2], r_hi),
                                  __fmul_rn(y[3], r_hi));
    if (a == b) return a;
  }
  return pack4_e4m3(__fdiv_rn(y[0], s), __fdiv_rn(y[1], s), __fdiv_rn(y[2], s), __fdiv_rn(y[3], s));
}

template <int D>
__global__ void __launch_bounds__(256, QuantCfg<D>::kMinBlocks) attn_quant_fp8_kernel(const QuantParams p) {
  using C = QuantCfg<D>;
  constexpr int TPR = D / 8;              // threads per row
  constexpr int RPP = 256 / TPR;          // rows per pass
  constexpr int PASSES = 128 / RPP;
  extern __shared__ __align__(1024) uint8_t smem[];
  auto* tiles = reinterpret_cast<__nv_bfloat16*>(smem);
  auto* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  auto* abort_flag = reinterpret_cast<volatile int*>(smem + C::kAbortOff);
  auto* red = reinterpret_cast<float*>(smem + C::kRedOff);

  const int tid = threadIdx.x;
  const int rip = tid / TPR;              // row within pass
  const int seg = tid % TPR;              // 8-value segment within the row

  // Block t = bh * n_blocks + blk: rows [128 blk, min(128 blk + 128, N)) of
  // head bh, contiguous in memory.
  auto issue = [&](int t, int stage) {
    const int blk = t % p.n_blocks;
    const int rows = min(C::kRows, p.N - blk * C::kRows);
    const uint32_t bytes = static_cast<uint32_t>(rows) * D * 2;
    const __nv_bfloat16* src = p.x + static_cast<size_t>(t / p.n_blocks) * p.N * D +
                               static_cast<size_t>(blk) * C::kRows * D;
    mbar_arrive_expect_tx(&full[stage], bytes);
    bulk_load(tiles + static_cast<size_t>(stage) * C::kRows * D, src, bytes, &full[stage]);
  };

  if (tid == 0) {
    for (int s = 0; s < C::kStages; ++s) mbar_init(&full[s], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      const int t = blockIdx.x + s * gridDim.x;
      if (t < p.total) issue(t, s);
    }
  }

  float sg[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) sg[i] = (p.hadamard && p.signs != nullptr) ? p.signs[seg * 8 + i] : 1.f;
  const float norm = rsqrtf(static_cast<float>(D));

  int it = 0;
  bool failed = false;
  for (int t = blockIdx.x; t < p.total; t += gridDim.x, ++it) {
    const int stage = it % C::kStages;
    const bool ok = mbar_wait(&full[stage], (it / C::kStages) & 1, p.status, abort_flag,
                              kWhereQuantFull, p.wait_limit_ns);
    const int row0 = (t % p.n_blocks) * C::kRows;
    const __nv_bfloat16* tile = tiles + static_cast<size_t>(stage) * C::kRows * D;

    float y[PASSES][8];
    float amax = 0.f;
#pragma unroll
    for (int ps = 0; ps < PASSES; ++ps) {
      const int r = ps * RPP + rip;
      if (ok && row0 + r < p.N) {
        const uint4 raw = *reinterpret_cast<const uint4*>(tile + r * D + seg * 8);
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __bfloat1622float2(h2[i]);
          y[ps][2 * i] = f.x;
          y[ps][2 * i + 1] = f.y;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) y[ps][i] = 0.f;
      }
      if (p.hadamard) {
#pragma unroll
        for (int i = 0; i < 8; ++i) y[ps][i] *= sg[i];
        // butterflies over the 3 low index bits (inside this thread)
#pragma unroll
        for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            if ((i & h) == 0) {
              const float a = y[ps][i], b = y[ps][i | h];
              y[ps][i] = a + b;
              y[ps][i | h] = a - b;
            }
          }
        }
        // butterflies over the high index bits (across the row's lanes)
#pragma unroll
        for (int m = 1; m < TPR; m <<= 1) {
          // lower lane: y + other; upper lane: other - y (one rounding each)
          const float sgn = (seg & m) != 0 ? -1.f : 1.f;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float other = __shfl_xor_sync(0xffffffffu, y[ps][i], m);
            y[ps][i] = fmaf(sgn, y[ps][i], other);
          }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) y[ps][i] *= norm;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(y[ps][i]));
    }

    // Block amax.  The slots alternate between blocks: a warp writes slot
    // set (it & 1) again only two barriers later, after every warp has read it.
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    float* slots = red + (it & 1) * 8;
    if ((tid & 31) == 0) slots[tid >> 5] = amax;
    // Every thread has read this block's buffer once it passes the barrier;
    // a wait that gave up anywhere ends the loop in every thread.
    if (__syncthreads_or(!ok)) {
      failed = true;
      break;
    }
    if (tid == 0) {
      const int tn = t + C::kStages * gridDim.x;
      if (tn < p.total) {
        fence_proxy_async_smem();
        issue(tn, stage);
      }
    }
    float bmax = slots[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) bmax = fmaxf(bmax, slots[w]);
    const float s = (bmax == 0.f) ? 1.0f : __fdiv_rn(bmax, 448.0f);
    if (tid == 0) p.descale[t] = s;
    // The bracket needs the reciprocal and the products to stay normal and
    // finite: a block scale far outside [2^-100, 2^100] takes the division.
    const bool fast = s >= 0x1p-100f && s <= 0x1p100f;
    const float r = __frcp_rn(s);
    const float r_lo = __fmul_rn(r, 1.f - 0x1p-20f), r_hi = __fmul_rn(r, 1.f + 0x1p-20f);

    uint8_t* out_blk = p.x8 + static_cast<size_t>(t / p.n_blocks) * p.N * D + static_cast<size_t>(row0) * D;
#pragma unroll
    for (int ps = 0; ps < PASSES; ++ps) {
      const int r = ps * RPP + rip;
      if (row0 + r < p.N) {
        uint2 out;
        out.x = quant4_e4m3(&y[ps][0], s, r_lo, r_hi, fast);
        out.y = quant4_e4m3(&y[ps][4], s, r_lo, r_hi, fast);
        *reinterpret_cast<uint2*>(out_blk + static_cast<size_t>(r) * D + seg * 8) = out;
      }
    }
  }

  // After a wait gave up, let the copies still in flight land (bounded)
  // before the CTA's shared memory is released.
  if (failed && tid == 0) {
    volatile int never = 0;
    for (int j = it; j < it + C::kStages; ++j) {
      const int t = blockIdx.x + j * gridDim.x;
      if (t < p.total)
        mbar_wait(&full[j % C::kStages], (j / C::kStages) & 1, nullptr, &never, kWhereQuantFull, 100000000ull);
    }
  }
}

}  // namespace attn
