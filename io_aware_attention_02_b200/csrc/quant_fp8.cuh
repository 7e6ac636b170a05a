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
// Streaming kernel: 2 bytes read and 1 byte written per element, meant to run
// at HBM bandwidth.  Persistent CTAs of 256 threads (three per SM) at D = 64,
// 256 (two per SM) at 128 and 512 (one per SM) at 256 walk the blocks of 128
// rows of one (batch, head) in a strided order.
// Thread 0 keeps a ring of kStages blocks in flight: each block arrives by
// TMA (tile loads of 64 columns x 128 rows, 128-byte swizzle, rows past N
// zero-filled).  A thread owns kVals columns of one row (32 at D = 64, 64
// otherwise; the threads of a row are neighbouring lanes): it reads them from
// shared memory (the swizzle spreads a warp's 16-byte reads over all banks),
// applies the signs (a flip of the bf16 sign bits), runs the butterfly stages
// of the fast Walsh-Hadamard transform that stay inside its values in
// registers and the remaining stages with its neighbours by one lane shuffle
// per value and stage; then it scales by 1/sqrt(D) and takes its amax.  The block's amax
// needs every row, so the CTA meets at one barrier per block; that barrier
// also tells thread 0 that the block's buffer has been read and may be
// refilled.  Each thread then rounds its 64 values to e4m3 into one of two
// shared-memory staging tiles (swizzled like the input, so a warp's 16-byte
// writes spread over all banks), and thread 0 writes the block to global
// memory with one TMA store (rows past N are clipped).
#pragma once
#include "ptx.cuh"

namespace attn {

enum : int { kWhereQuantFull = 10 };

struct QuantParams {
  CUtensorMap tm_x;         // 4-D map over x (D, N, H, B): box 64 x 128, 128-byte swizzle
  CUtensorMap tm_x8;        // 4-D map over the codes (D, N, H, B): box min(D, 128) x 128, same swizzle width
  float* descale;           // [BH][n_blocks]
  const float* signs;       // [D] or nullptr
  int* status;
  unsigned long long wait_limit_ns;
  int H, N, n_blocks, total;   // total = BH * n_blocks
  int hadamard;
};

template <int D>
struct QuantCfg {
  static constexpr int kRows = 128;
  static constexpr int kChunkBytes = kRows * 128;            // 64 bf16 columns x 128 rows
  static constexpr int kChunks = D / 64;
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  // input ring + two output staging tiles: 2 x 32 + 2 x 16 KiB per CTA and
  // two CTAs per SM at D = 128; 3 x 16 + 2 x 8 KiB and three CTAs at D = 64;
  // 2 x 64 + 2 x 32 KiB and one CTA at D = 256
  static constexpr int kStages = D == 64 ? 3 : 2;
  static constexpr int kMinBlocks = D == 64 ? 3 : (D == 128 ? 2 : 1);
  // values of a row per thread: 32 at D = 64 (twice the warps of 64 values,
  // measured 10 % faster there), 64 otherwise (32 measured 6 % slower at
  // D = 128: one more lane-shuffle stage per value)
  static constexpr int kVals = D == 64 ? 32 : 64;
  static constexpr int kOutBytes = kRows * D;                // one block of codes
  // the codes of a block go out in column chunks of at most 128 bytes (the
  // widest swizzled box): one chunk up to D = 128, two at D = 256
  static constexpr int kOutChunkCols = D < 128 ? D : 128;
  static constexpr int kOutChunks = D / kOutChunkCols;
  static constexpr int kTpr = D / kVals;                     // threads per row
  static constexpr int kPieces = kVals / 8;                  // 16-byte input pieces per thread
  static constexpr int kThreads = 128 * kTpr;
  static constexpr int kWarps = kThreads / 32;
  static constexpr int kOutOff = kStages * kTileBytes;     // [2] staging tiles
  static constexpr int kBarOff = kOutOff + 2 * kOutBytes;
  static constexpr int kAbortOff = kBarOff + 64;
  static constexpr int kRedOff = kBarOff + 128;             // float [2][kWarps <= 32]
  static constexpr int kSgnOff = kBarOff + 384;             // uint32 [D / 2]: sign bits per bf16 pair
  static_assert(2 * kWarps * 4 <= 256, "amax slots overflow their region");
  static_assert(D == 64 || D == 128 || D == 256, "head dim 64, 128 or 256");
  static constexpr int kSmem = kSgnOff + 2 * D + 1024;      // + alignment slack for the swizzle
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
// The four values come as two pairs; the products are taken two at a time
// (each lane of a paired multiply rounds like the scalar one).
__device__ __forceinline__ uint32_t quant4_e4m3(float2 y01, float2 y23, float s, float2 r_lo, float2 r_hi,
                                                bool fast) {
  if (fast) {
    const float2 a01 = __fmul2_rn(y01, r_lo), a23 = __fmul2_rn(y23, r_lo);
    const float2 b01 = __fmul2_rn(y01, r_hi), b23 = __fmul2_rn(y23, r_hi);
    const uint32_t a = pack4_e4m3(a01.x, a01.y, a23.x, a23.y);
    const uint32_t b = pack4_e4m3(b01.x, b01.y, b23.x, b23.y);
    if (a == b) return a;
  }
  return pack4_e4m3(__fdiv_rn(y01.x, s), __fdiv_rn(y01.y, s), __fdiv_rn(y23.x, s), __fdiv_rn(y23.y, s));
}

template <int D>
__global__ void __launch_bounds__(QuantCfg<D>::kThreads, QuantCfg<D>::kMinBlocks)
    attn_quant_fp8_kernel(const __grid_constant__ QuantParams p) {
  using C = QuantCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle pattern
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  auto* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  auto* abort_flag = reinterpret_cast<volatile int*>(smem + C::kAbortOff);
  auto* red = reinterpret_cast<float*>(smem + C::kRedOff);
  auto* sgn = reinterpret_cast<uint32_t*>(smem + C::kSgnOff);
  uint8_t* out_tiles = smem + C::kOutOff;

  const int tid = threadIdx.x;
  const int r = tid / C::kTpr;            // row within the block
  const int hc = tid % C::kTpr;           // which kVals columns of that row
  const int warp = tid >> 5;

  // Block t = bh * n_blocks + blk: rows [128 blk, 128 blk + 128) of head bh.
  auto issue = [&](int t, int stage) {
    const int bh = t / p.n_blocks, blk = t % p.n_blocks;
    mbar_arrive_expect_tx(&full[stage], C::kTileBytes);
#pragma unroll
    for (int c = 0; c < C::kChunks; ++c)
      tma_load_4d(smem + stage * C::kTileBytes + c * C::kChunkBytes, &p.tm_x, &full[stage], c * 64,
                  blk * C::kRows, bh % p.H, bh / p.H);
  };

  if (tid == 0) {
    for (int s = 0; s < C::kStages; ++s) mbar_init(&full[s], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  // The signs as bf16 sign bits, one word per pair of elements: multiplying
  // by -1 is flipping that bit of the packed input (exact).
  if (tid < D / 2) {
    uint32_t w = 0;
    if (p.hadamard && p.signs != nullptr) {
      if (p.signs[2 * tid] < 0.f) w |= 0x8000u;
      if (p.signs[2 * tid + 1] < 0.f) w |= 0x80000000u;
    }
    sgn[tid] = w;
  }
  __syncthreads();
  if (tid == 0) {
    tma_prefetch_desc(&p.tm_x);
    tma_prefetch_desc(&p.tm_x8);
    for (int s = 0; s < C::kStages; ++s) {
      const int t = blockIdx.x + s * gridDim.x;
      if (t < p.total) issue(t, s);
    }
  }

  const bool rot = p.hadamard != 0;
  const float norm = rsqrtf(static_cast<float>(D));

  int it = 0;
  bool failed = false;
  for (int t = blockIdx.x; t < p.total; t += gridDim.x, ++it) {
    const int stage = it % C::kStages;
    const bool ok = mbar_wait(&full[stage], (it / C::kStages) & 1, p.status, abort_flag,
                              kWhereQuantFull, p.wait_limit_ns);
    const int row0 = (t % p.n_blocks) * C::kRows;

    // this thread's kVals values, columns kVals*hc .. (16-byte piece q of a
    // 64-column chunk sits at piece q ^ (row % 8) of the row's 128 bytes),
    // held as pairs y[i] = (value 2i, value 2i + 1)
    float2 y[C::kVals / 2];
    const uint8_t* tile = smem + stage * C::kTileBytes + (hc * C::kVals / 64) * C::kChunkBytes + r * 128;
    const int qbase = (hc * C::kVals % 64) / 8;   // first piece of this thread in its chunk row
#pragma unroll
    for (int q = 0; q < C::kPieces; ++q) {
      uint4 raw = make_uint4(0u, 0u, 0u, 0u);
      if (ok) raw = *reinterpret_cast<const uint4*>(tile + (((qbase + q) ^ (r & 7)) << 4));
      if (rot) {   // four words shared by the threads of this column range: a broadcast read
        const uint4 m = reinterpret_cast<const uint4*>(sgn)[hc * C::kPieces + q];
        raw.x ^= m.x; raw.y ^= m.y; raw.z ^= m.z; raw.w ^= m.w;
      }
      y[q * 4 + 0] = unpack2<__nv_bfloat16>(raw.x);
      y[q * 4 + 1] = unpack2<__nv_bfloat16>(raw.y);
      y[q * 4 + 2] = unpack2<__nv_bfloat16>(raw.z);
      y[q * 4 + 3] = unpack2<__nv_bfloat16>(raw.w);
    }
    if (rot) {
      // fast Walsh-Hadamard transform, one rounding per output of each stage
      // (index bit 0 first): bit 0 pairs the two values of a pair ...
#pragma unroll
      for (int i = 0; i < C::kVals / 2; ++i) {
        const float a = y[i].x, b = y[i].y;
        y[i] = make_float2(a + b, a - b);
      }
      // ... the next bits up to log2(kVals) - 1 pair whole pairs: one paired
      // add and one paired multiply-add by -1 (an exact negation, then the
      // one rounding of a - b) per two butterflies ...
      const float2 neg1 = make_float2(-1.f, -1.f);
#pragma unroll
      for (int h = 1; h < C::kVals / 2; h <<= 1) {
#pragma unroll
        for (int i = 0; i < C::kVals / 2; ++i) {
          if ((i & h) == 0) {
            const float2 a = y[i], b = y[i | h];
            y[i] = __fadd2_rn(a, b);
            y[i | h] = __ffma2_rn(b, neg1, a);
          }
        }
      }
      // ... and the index bits above (bit log2(kVals) + s is bit s of hc)
      // with the lane that differs in that bit (lower half: y + other;
      // upper half: other - y)
#pragma unroll
      for (int sb = 1; sb < C::kTpr; sb <<= 1) {
        const float sg = (hc & sb) == 0 ? 1.f : -1.f;
        const float2 sg2 = make_float2(sg, sg);
#pragma unroll
        for (int i = 0; i < C::kVals / 2; ++i) {
          const float2 other = make_float2(__shfl_xor_sync(0xffffffffu, y[i].x, sb),
                                           __shfl_xor_sync(0xffffffffu, y[i].y, sb));
          y[i] = __ffma2_rn(sg2, y[i], other);
        }
      }
      const float2 norm2 = make_float2(norm, norm);
#pragma unroll
      for (int i = 0; i < C::kVals / 2; ++i) y[i] = __fmul2_rn(y[i], norm2);
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < C::kVals / 2; ++i) amax = fmax3(amax, fabsf(y[i].x), fabsf(y[i].y));

    // Block amax.  The slots alternate between blocks: a warp writes slot
    // set (it & 1) again only two barriers later, after every warp has read it.
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    float* slots = red + (it & 1) * C::kWarps;
    if ((tid & 31) == 0) slots[warp] = amax;
    // staging tile (it & 1) was last stored two blocks ago: let that store
    // finish reading it before anyone writes it again (the barrier below)
    if (tid == 0) bulk_wait_group_read<1>();
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
    for (int w = 1; w < C::kWarps; ++w) bmax = fmaxf(bmax, slots[w]);
    const float s = (bmax == 0.f) ? 1.0f : __fdiv_rn(bmax, 448.0f);
    if (tid == 0) p.descale[t] = s;
    // The bracket needs the reciprocal and the products to stay normal and
    // finite: a block scale far outside [2^-100, 2^100] takes the division.
    const bool fast = s >= 0x1p-100f && s <= 0x1p100f;
    const float rc = __frcp_rn(s);
    const float r_lo = __fmul_rn(rc, 1.f - 0x1p-20f), r_hi = __fmul_rn(rc, 1.f + 0x1p-20f);
    const float2 r_lo2 = make_float2(r_lo, r_lo), r_hi2 = make_float2(r_hi, r_hi);

    // this thread's kVals codes: 16-byte pieces kVals*hc/16 + g of the row,
    // in column chunk (kVals*hc) / kOutChunkCols, swizzled the way the TMA
    // store reads them (the swizzle XORs the 16-byte piece index within the
    // chunk row with address bits 7 and up: row % 8 for 128-byte rows,
    // (row / 2) % 4 for 64-byte rows)
    const int xr = D >= 128 ? (r & 7) : ((r >> 1) & 3);
    constexpr int kPiecesPerChunkRow = C::kOutChunkCols / 16;
    const int opiece = hc * C::kVals / 16;
    const int piece0 = opiece % kPiecesPerChunkRow;
    uint8_t* orow = out_tiles + (it & 1) * C::kOutBytes + (opiece / kPiecesPerChunkRow) * (C::kRows * C::kOutChunkCols) +
                    r * C::kOutChunkCols;
#pragma unroll
    for (int g = 0; g < C::kVals / 16; ++g) {
      uint4 v;
      v.x = quant4_e4m3(y[8 * g], y[8 * g + 1], s, r_lo2, r_hi2, fast);
      v.y = quant4_e4m3(y[8 * g + 2], y[8 * g + 3], s, r_lo2, r_hi2, fast);
      v.z = quant4_e4m3(y[8 * g + 4], y[8 * g + 5], s, r_lo2, r_hi2, fast);
      v.w = quant4_e4m3(y[8 * g + 6], y[8 * g + 7], s, r_lo2, r_hi2, fast);
      *reinterpret_cast<uint4*>(orow + (((piece0 + g) ^ xr) << 4)) = v;
    }
    fence_proxy_async_smem();   // generic writes, read next by the TMA store
    __syncthreads();
    if (tid == 0) {
      const int bh = t / p.n_blocks;
#pragma unroll
      for (int c = 0; c < C::kOutChunks; ++c)
        tma_store_4d(&p.tm_x8, out_tiles + (it & 1) * C::kOutBytes + c * (C::kRows * C::kOutChunkCols),
                     c * C::kOutChunkCols, row0, bh % p.H, bh / p.H);
      bulk_commit_group();
    }
  }
  if (tid == 0) bulk_wait_group<0>();   // the last stores have landed

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
