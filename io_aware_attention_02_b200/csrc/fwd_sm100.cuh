// Fused attention forward for sm_100a, 16-bit inputs (bf16 / fp16), head dim
// 64 or 128, optional causal mask.
//
// What it computes (exact attention, the definition Softmax(Q K^T / sqrt(d)) V
// of the "FlashAttention-3" explainer on droidorbit.com, with `scale` in place
// of 1/sqrt(d)), tiled as in "FlashAttention-3: como exprimir H100 al limite
// con atencion IO-aware" (dibro.site), "Arquitectura y metodo": Q in 128-row
// tiles, K/V in 128-row tiles, the running max m and sum l kept per row, the
// output rescaled by exp2(m_old - m_new) ("Mathematical Formulation: The
// Online Softmax Rescaling Trick", droidorbit.com) and divided by l once at
// the end.  The N x N score matrix never leaves the SM: S lives in tensor
// memory, P overwrites it in place as 16-bit values.
//
// Structure (Blackwell-native; the pages' Hopper WGMMA design is prior art):
//   * persistent grid, one CTA per SM, work unit = (batch*head, 256 query rows)
//     = two 128-row Q tiles ("slots"); causal units are taken longest first
//     and dealt to the CTAs in a snake order for balance;
//   * warp 0: TMA producer -- Q tiles once per unit, then K_j, V_j through a
//     multi-stage shared-memory ring guarded by full/empty mbarriers
//     (producer/consumer warp specialisation: dibro.site, "Arquitectura y
//     metodo" item 3; quantum-bit repost, first technical upgrade);
//   * warp 1: one thread issues every tcgen05.mma -- S_t = Q_t K_j^T
//     (SMEM x SMEM -> TMEM) and O_t += P_t V_j (P from TMEM, V from SMEM);
//   * warps 4-7 / 8-11: softmax warpgroups, one per Q tile, one thread per
//     query row (warps 2-3 idle; setmaxnreg moves their registers and those
//     of warps 0-1 to the softmax warpgroups).  While one group turns S into P the tensor core works on the
//     other tile: the ping-pong schedule of the quantum-bit repost
//     ("ping-pong scheduling") carried over to tcgen05;
//   * causal: key tiles entirely above the diagonal are never loaded or
//     multiplied (dibro.site, "Contribuciones clave"); the diagonal tile and a
//     ragged last tile are masked element-wise;
//   * the running max is only raised when it grows by more than 2^8 (lazy
//     rescaling); the final division by l keeps the result exact up to
//     rounding while O is rescaled only on the rare large jumps.
//
// The same pipeline runs the FP8 (e4m3) variant (dibro.site, "Arquitectura
// y metodo": FP8 with in-line per-block quantisation; quantum-bit repost, FP8
// paragraph): tcgen05 kind::f8f6f4 products, scores scaled per (query block,
// key block) by the blocks' descale factors, P rounded to e4m3 after a
// power-of-two gain (256) times v_descale[j] / max v_descale, statistics and
// accumulators in fp32 (vikram-blog.pages.dev, "Production Gotchas": softmax
// accumulators stay fp32 under FP8), O divided by 256 * l / max v_descale at
// the end.
//
// Every mbarrier wait is bounded (timeout -> status word, no trap, no hang).
#pragma once
#include <cuda_fp8.h>

#include <type_traits>

#include "ptx.cuh"

namespace attn {

// Element traits: bytes per value, tcgen05 kind, operand format code.
template <typename E>
struct Elem;
template <>
struct Elem<__nv_bfloat16> {
  static constexpr int kBytes = 2;
  static constexpr bool kF8 = false;
  static constexpr uint32_t kFmt = 1;   // kind::f16 BF16
  using Out = __nv_bfloat16;
};
template <>
struct Elem<__half> {
  static constexpr int kBytes = 2;
  static constexpr bool kF8 = false;
  static constexpr uint32_t kFmt = 0;   // kind::f16 F16
  using Out = __half;
};
template <>
struct Elem<__nv_fp8_e4m3> {
  static constexpr int kBytes = 1;
  static constexpr bool kF8 = true;
  static constexpr uint32_t kFmt = 0;   // kind::f8f6f4 E4M3
  using Out = __nv_bfloat16;
};

struct FwdParams {
  CUtensorMap tm_q;  // 4-D maps over (d, N, H, B) with caller strides, 128-byte boxes, 128-byte swizzle
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  void* o;           // [BH][N][D] 16-bit output
  float* lse;        // [BH][N] natural-log LSE, may be null
  const float* q_desc;  // FP8 only: [BH][n_kv] descale factors per 128-row block
  const float* k_desc;
  const float* v_desc;
  int* status;       // 4-int device status word
  int BH, H, N, n_kv, n_qpairs, n_units;
  long long o_sb, o_sh, o_sn;   // element strides of O over (batch, head, row); head dim contiguous
  int d_out;         // head dim of the tensors (<= the kernel's D; columns beyond it read as zero)
  int snake;         // work distribution: alternate round direction (causal)
  int order;         // 1 = longest-first across heads (causal, short heads)
  float scale_log2;  // scale * log2(e)
  unsigned long long wait_limit_ns;
  int fault;         // test hook: 1 = CTA 0 skips its first K load (waits must run out)
};

template <typename E, int D>
struct FwdCfg {
  static constexpr int kTileRows = 128;
  // A tile is kChunks column chunks of 128 rows x kSwz bytes, each laid out
  // with a kSwz-byte swizzle: 128 bytes, or 64 where a whole row is 64 bytes
  // (e4m3 at head dim 64).
  static constexpr int kRowBytes = D * Elem<E>::kBytes;
  static constexpr int kSwz = kRowBytes >= 128 ? 128 : 64;
  static constexpr int kChunkBytes = 128 * kSwz;
  static constexpr int kChunkCols = kSwz / Elem<E>::kBytes;
  static constexpr int kChunks = kRowBytes / kSwz;
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  static constexpr int kStages = (kTileBytes <= 16384) ? 8 : 4;
  static constexpr int kKeysPerMma = 32 / Elem<E>::kBytes;  // 32 bytes of K per tcgen05.mma
  static constexpr int kThreads = 384;   // 3 warpgroups: TMA+MMA | softmax 0 | softmax 1
  static constexpr int kTmemCols = 512;                   // S0 | S1 | O0 | O1
  static constexpr int kColS = 0;                         // + t * 128
  static constexpr int kColO = 256;                       // + t * D
  // dynamic shared memory: [Q0 | Q1 | ring of kStages tiles | 2 transposed
  // V tiles (FP8 only) | barriers]
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = 2 * kTileBytes;
  static constexpr int kOffVt = kOffKV + kStages * kTileBytes;
  static constexpr int kVtBytes = Elem<E>::kF8 ? 2 * kTileBytes : 0;
  static constexpr int kOffBar = kOffVt + kVtBytes;
  static constexpr int kBarBytes = 512;
  static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;  // + 1 KiB alignment slack
};

// Work distribution.  The persistent CTAs walk the unit list in rounds of
// gridDim.x units.  Non-causal units all cost the same: plain rounds, in
// head-major order, so the CTAs of a round share one head's K/V in L2.
// Causal units get longer with the row block: the rounds alternate direction
// (a snake), which over a longest-first list gives every CTA a near-equal
// share.  Longest first is taken across heads when a head has fewer units
// than there are CTAs, and within each head otherwise (then every running
// CTA streams the same head's K/V).
__device__ __forceinline__ int sched_unit(int k, int snake) {
  const int r = (snake && (k & 1)) ? static_cast<int>(gridDim.x - 1 - blockIdx.x)
                                   : static_cast<int>(blockIdx.x);
  return k * static_cast<int>(gridDim.x) + r;
}

// unit -> (batch*head, block of query rows); order 1 = longest first across
// heads (causal only).
template <bool CAUSAL>
__device__ __forceinline__ void decode_unit(int unit, int n_blocks, int BH, int order, int& bh, int& blk) {
  if (CAUSAL && order == 1) {
    blk = n_blocks - 1 - unit / BH;
    bh = unit % BH;
  } else {
    bh = unit / n_blocks;
    blk = unit % n_blocks;
    if (CAUSAL) blk = n_blocks - 1 - blk;
  }
}

// Barrier ids reported on timeout (status[1]).
enum : int {
  kWhereQEmpty = 1, kWhereKvEmpty = 2, kWhereQFull = 3, kWhereKvFull = 4,
  kWherePFull = 5, kWhereSFull = 6, kWhereOFull = 7, kWhereDrain = 8
};

// Range-check ids reported by the debug build (status[1] with kErrBounds):
// which access of the forward kernel fell outside its region.
enum : int {
  kChkQLoad = 21, kChkKvLoad = 22, kChkSOut = 23, kChkSQ = 24, kChkSK = 25, kChkOOut = 26, kChkPIn = 27,
  kChkVIn = 28, kChkSLoad = 29, kChkPStore = 30, kChkORescale = 31, kChkOLoad = 32, kChkVtSrc = 33,
  kChkVtDst = 34
};

// ---------------------------------------------------------------------------
// Softmax arithmetic helpers
// ---------------------------------------------------------------------------

// max of 128 values with 3-input max instructions, four independent chains:
// s[0..3] start the chains, 15 steps of 8 cover s[4..123], s[124..127] close
// them (every index stays inside the array).
__device__ __forceinline__ float row_max128(const float (&s)[128]) {
  float a[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
  for (int i = 4; i < 124; i += 8) {
#pragma unroll
    for (int k = 0; k < 4; ++k) a[k] = fmax3(a[k], s[i + k], s[i + 4 + k]);
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) a[k] = fmaxf(a[k], s[124 + k]);
  return fmax3(fmaxf(a[0], a[1]), a[2], a[3]);
}

// 2^x for a pair on the FMA pipe (Cody-Waite style split, then a minimax
// polynomial): j = round(x) through the 1.5*2^23 addition, f = x - j in
// [-1/2, 1/2], 2^f ~ p(f), and 2^j added into the exponent field with one
// shift-add.  x is clamped to >= -125 so the exponent arithmetic cannot wrap
// (2^-125 is far below anything that survives the final division by l).
// Coefficients: minimax relative-error fit of degree kDeg (Remez exchange),
// produced by io_aware_attention_02_b200/fit_exp2_poly.py; max relative
// error 7.5e-5 (degree 3) / 1.7e-3 (degree 2).
template <int kDeg>
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  x.x = fmaxf(x.x, -125.0f);
  x.y = fmaxf(x.y, -125.0f);
  const float2 t = __fadd2_rn(x, make_float2(kMagic, kMagic));
  const float2 r = __fadd2_rn(t, make_float2(-kMagic, -kMagic));
  const float2 f = __ffma2_rn(r, make_float2(-1.0f, -1.0f), x);
  float2 p;
  if constexpr (kDeg == 3) {
    p = __ffma2_rn(make_float2(0.0551716685295105f, 0.0551716685295105f), f,
                   make_float2(0.2426111251115799f, 0.2426111251115799f));
    p = __ffma2_rn(p, f, make_float2(0.6932609677314758f, 0.6932609677314758f));
    p = __ffma2_rn(p, f, make_float2(0.9999280571937561f, 0.9999280571937561f));
  } else {
    p = __ffma2_rn(make_float2(0.23842893540859222f, 0.23842893540859222f), f,
                   make_float2(0.7034479975700378f, 0.7034479975700378f));
    p = __ffma2_rn(p, f, make_float2(1.0004431009292603f, 1.0004431009292603f));
  }
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}

__device__ __forceinline__ float2 exp2_mufu2(float2 x) {
  return make_float2(ex2_approx(x.x), ex2_approx(x.y));
}

// Pairs i with (i % 8) < kPolyPairsPer8 take the polynomial path.
constexpr int kPolyPairsPer8 = 1;

// P = 2^(s*c - m) for one half (64 keys, h = 0 or 1) of a 128-key row,
// packed to 16-bit pairs (or e4m3 quads, after the gain) into pk.  Returns the
// fp32 sum of the unrounded P of that half.
template <bool kF8, typename T, bool kPoly>
__device__ __forceinline__ float exp_half(const float (&s)[128], int h, float c, float neg_m, float pgain,
                                          uint32_t (&pk)[kF8 ? 16 : 32]) {
  const float2 c2 = make_float2(c, c);
  const float2 nm2 = make_float2(neg_m, neg_m);
  float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  if constexpr (!kF8) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int e = 64 * h + 2 * i;
      const float2 x = __ffma2_rn(make_float2(s[e], s[e + 1]), c2, nm2);
      const float2 pr = (kPoly && (i % 8) < kPolyPairsPer8) ? exp2_poly2<3>(x) : exp2_mufu2(x);
      acc[i & 1] = __fadd2_rn(acc[i & 1], pr);
      pk[i] = pack2<T>(pr.x, pr.y);
    }
  } else {
    const float2 g2 = make_float2(pgain, pgain);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int e = 64 * h + 4 * i;
      const float2 x0 = __ffma2_rn(make_float2(s[e], s[e + 1]), c2, nm2);
      const float2 x1 = __ffma2_rn(make_float2(s[e + 2], s[e + 3]), c2, nm2);
      const float2 p0 = (kPoly && (i % 4) < 1) ? exp2_poly2<2>(x0) : exp2_mufu2(x0);
      const float2 p1 = (kPoly && (i % 4) < 2) ? exp2_poly2<2>(x1) : exp2_mufu2(x1);
      acc[0] = __fadd2_rn(acc[0], p0);
      acc[1] = __fadd2_rn(acc[1], p1);
      const float2 g0 = __fmul2_rn(p0, g2);
      const float2 g1 = __fmul2_rn(p1, g2);
      pk[i] = pack4_e4m3(g0.x, g0.y, g1.x, g1.y);
    }
  }
  const float2 a = __fadd2_rn(acc[0], acc[1]);
  return a.x + a.y;
}

// Write one half of P over the row's S columns in TMEM (32 columns per half at
// 16 bit, 16 at e4m3).  The store has completed when it returns: tcgen05.st
// reads its source registers asynchronously, so they must not be reused
// before tcgen05.wait::st.
template <bool kF8>
__device__ __forceinline__ void store_p_half(uint32_t tS, int h, uint32_t (&pk)[kF8 ? 16 : 32]) {
  if constexpr (!kF8) {
    tmem_st32(tS + 32 * h, pk);
  } else {
    tmem_st16(tS + 16 * h, pk);
  }
  tmem_wait_st();
  tmem_reg_fence(pk);
}

// exp_half followed by store_p_half; returns the half's sum.
template <bool kF8, typename T, bool kPoly>
__device__ __forceinline__ float exp_pack_half(const float (&s)[128], int h, float c, float neg_m,
                                               float pgain, uint32_t tS) {
  uint32_t pk[kF8 ? 16 : 32];
  const float sum = exp_half<kF8, T, kPoly>(s, h, c, neg_m, pgain, pk);
  store_p_half<kF8>(tS, h, pk);
  return sum;
}

// In-shared-memory transpose of one FP8 V tile (128 keys x 128 head-dim
// bytes), from the TMA layout (MN-major for the P.V product: one 128-byte row
// per key, 16-byte chunks swizzled by key % 8) to the K-major layout (one
// 128-byte row per head-dim column, chunks swizzled by column % 8).  64
// threads each move one 16 x 16 byte block with 16-byte loads and stores and
// a register transpose of 4 x 4 byte blocks (byte permutes); block (kb, cb)
// of thread t is kb = t % 8, cb = (t % 8 + t / 8) % 8, so that the 8 threads
// of a quarter warp touch 8 distinct 16-byte bank groups on both sides.
// This is the pages' V-tile transpose for FP8 (quantum-bit repost, FP8
// paragraph: FP8 tensor cores want the reduction dim contiguous, so blocks of
// V are transposed in place).
__device__ __forceinline__ void transpose_v_tile_e4m3(const uint8_t* src, uint8_t* dst, int t) {
  const int kb = t & 7;
  const int cb = ((t & 7) + (t >> 3)) & 7;
  uint32_t w[16][4];
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    const int key = kb * 16 + r;
    const uint4 v = *reinterpret_cast<const uint4*>(src + key * 128 + ((cb ^ (key & 7)) << 4));
    w[r][0] = v.x; w[r][1] = v.y; w[r][2] = v.z; w[r][3] = v.w;
  }
  // For each 4-column group q: rows c = 4q .. 4q+3 of the output, word g =
  // bytes of column cb*16 + c for keys kb*16 + 4g .. 4g+3; stored at once so
  // only 16 output words are live.
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t o[4][4];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const uint32_t a = w[4 * g][q], b = w[4 * g + 1][q], c = w[4 * g + 2][q], d = w[4 * g + 3][q];
      const uint32_t t0 = __byte_perm(a, b, 0x5140), t1 = __byte_perm(a, b, 0x7362);
      const uint32_t t2 = __byte_perm(c, d, 0x5140), t3 = __byte_perm(c, d, 0x7362);
      o[0][g] = __byte_perm(t0, t2, 0x5410);
      o[1][g] = __byte_perm(t0, t2, 0x7632);
      o[2][g] = __byte_perm(t1, t3, 0x5410);
      o[3][g] = __byte_perm(t1, t3, 0x7632);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int col = cb * 16 + 4 * q + k;
      *reinterpret_cast<uint4*>(dst + col * 128 + ((kb ^ (col & 7)) << 4)) =
          make_uint4(o[k][0], o[k][1], o[k][2], o[k][3]);
    }
  }
}

constexpr int kRegsLow = 104;    // TMA + MMA warpgroup
constexpr int kRegsHigh = 200;  // each softmax warpgroup
static_assert(128 * kRegsLow + 256 * kRegsHigh <= 384 * 168, "register split exceeds the launch pool");

// SERIAL (the ablation of the overlap, 16-bit d = 128 only): the tensor core
// waits for both tiles' P before any product of the next key tile, and both
// tiles' S are published together, so no product overlaps a softmax.
template <typename E, int D, bool CAUSAL, bool VT = false, bool SERIAL = false>
__global__ void __launch_bounds__(384, 1) attn_fwd_sm100_kernel(const __grid_constant__ FwdParams p) {
  static_assert(!VT || (Elem<E>::kF8 && D == 128), "V transpose is the FP8 d=128 path");
  using Cfg = FwdCfg<E, D>;
  using T = typename Elem<E>::Out;
  constexpr bool kF8 = Elem<E>::kF8;
  constexpr int S = Cfg::kStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + Cfg::kOffQ;
  uint8_t* sKV = smem + Cfg::kOffKV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kOffBar);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* s_full = bars + 2;       // [2]
  uint64_t* p_full = bars + 4;       // [2 tiles][2 key halves]
  uint64_t* o_full = bars + 8;       // [2]
  uint64_t* drain = bars + 10;
  uint64_t* kv_full = bars + 11;     // [S]
  uint64_t* kv_empty = bars + 11 + S; // [S]
  uint64_t* vt_full = bars + 11 + 2 * S;   // [2] transposed V tile ready (FP8, VT)
  uint64_t* vt_empty = bars + 13 + 2 * S;  // [2] transposed V tile consumed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 15 + 2 * S);
  uint8_t* sVt = smem + Cfg::kOffVt;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(s_full + t, 1);
      mbar_init(p_full + 2 * t, 128);
      mbar_init(p_full + 2 * t + 1, 128);
      mbar_init(o_full + t, 1);
    }
    mbar_init(drain, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(kv_full + s, 1);
      mbar_init(kv_empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(vt_full + b, 1);
      mbar_init(vt_empty + b, 1);
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
  const unsigned long long lim = p.wait_limit_ns;

  // Register split (setmaxnreg acts per warpgroup): the TMA/MMA warpgroup
  // gives registers to the two softmax warpgroups.  128*104 + 256*200 =
  // 64512 = 384 threads * 168 registers, the launch allocation.  Each
  // setmaxnreg sits inside its role's branch, so no code after a control-flow
  // merge is held to the lower count.
  if (warp < 4) {
  reg_dealloc<kRegsLow>();
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
        int bh, qp;
        decode_unit<CAUSAL>(unit, p.n_qpairs, p.BH, p.order, bh, qp);
        const int n1 = CAUSAL ? min(2 * qp + 2, n_kv) : n_kv;
        ok = mbar_wait(q_empty, (unit_iter & 1) ^ 1, p.status, abort_flag, kWhereQEmpty, lim);
        if (!ok) break;
        mbar_arrive_expect_tx(q_full, 2 * Cfg::kTileBytes);
        for (int t = 0; t < 2; ++t)
          for (int c = 0; c < Cfg::kChunks; ++c) {
            uint8_t* dst = sQ + t * Cfg::kTileBytes + c * Cfg::kChunkBytes;
            if (smem_range_ok(dst, Cfg::kChunkBytes, smem, Cfg::kOffQ, Cfg::kOffKV, p.status, kChkQLoad))
              tma_load_4d(dst, &p.tm_q, q_full, c * Cfg::kChunkCols, qp * 256 + t * 128, bh % p.H, bh / p.H);
          }
        for (int j = 0; j < n1 && ok; ++j) {
          for (int which = 0; which < 2; ++which, ++kv_iter) {
            const uint32_t s = kv_iter % S;
            ok = mbar_wait(kv_empty + s, ((kv_iter / S) & 1) ^ 1, p.status, abort_flag, kWhereKvEmpty, lim);
            if (!ok) break;
            if (p.fault == 1 && blockIdx.x == 0 && kv_iter == 0) {
              skipped = 0;  // test hook: this stage never completes
              continue;
            }
            mbar_arrive_expect_tx(kv_full + s, Cfg::kTileBytes);
            const CUtensorMap* map = which == 0 ? &p.tm_k : &p.tm_v;
            for (int c = 0; c < Cfg::kChunks; ++c) {
              uint8_t* dst = sKV + s * Cfg::kTileBytes + c * Cfg::kChunkBytes;
              if (smem_range_ok(dst, Cfg::kChunkBytes, smem, Cfg::kOffKV, Cfg::kOffVt, p.status, kChkKvLoad))
                tma_load_4d(dst, map, kv_full + s, c * Cfg::kChunkCols, j * 128, bh % p.H, bh / p.H);
            }
          }
        }
      }
      if (!ok) {
        // Let the copies already issued land before the CTA may exit: wait
        // for each ring stage's last armed phase and for the last Q load.
        volatile int never = 0;
        for (uint32_t i = (kv_iter > S ? kv_iter - S : 0); i < kv_iter; ++i)
          if (static_cast<int64_t>(i) != skipped) mbar_wait(kv_full + (i % S), (i / S) & 1, nullptr, &never, kWhereDrain, 100000000ull);
        if (unit_iter > 0) mbar_wait(q_full, (unit_iter - 1) & 1, nullptr, &never, kWhereDrain, 100000000ull);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      constexpr uint32_t fmt = Elem<E>::kFmt;
      constexpr uint32_t idesc_s = make_idesc(fmt, fmt, 0, 0, 128, 128);
      // P.V with V MN-major straight from the TMA tile, or (VT) K-major from
      // the transposed copy
      constexpr uint32_t idesc_o = make_idesc(fmt, fmt, 0, VT ? 0 : 1, 128, D);
      uint32_t kv_iter = 0, unit_iter = 0;
      uint32_t p_cnt[2] = {0, 0};
      bool ok = true;

      // Descriptors are built once and advanced by adding (byte offset >> 4)
      // to their start-address field (addresses stay below 256 KiB, so the
      // 14-bit field never carries).
      constexpr int kSwz = Cfg::kSwz;
      const uint64_t dQ = smem_desc_swz(smem_u32(sQ), 16, 8 * kSwz, kSwz);
      const uint64_t dK = smem_desc_swz(smem_u32(sKV), 16, 8 * kSwz, kSwz);
      const uint64_t dV = VT ? smem_desc_sw128(smem_u32(sVt), 16, 1024)
                             : smem_desc_swz(smem_u32(sKV), Cfg::kChunkBytes, 8 * kSwz, kSwz);
      uint32_t v_cnt = 0;   // V tiles consumed (VT: selects the transposed buffer and phase)

      auto issue_s = [&](int t, uint32_t kstage) {
        const uint64_t a0 = dQ + static_cast<uint64_t>((t * Cfg::kTileBytes) >> 4);
        const uint64_t b0 = dK + static_cast<uint64_t>((kstage * Cfg::kTileBytes) >> 4);
        if (!tmem_range_ok(tmem + Cfg::kColS + t * 128, tmem, 128, Cfg::kColS + t * 128, Cfg::kColS + t * 128 + 128,
                           p.status, kChkSOut) ||
            !smem_range_ok(sQ + t * Cfg::kTileBytes, Cfg::kTileBytes, smem, Cfg::kOffQ, Cfg::kOffKV, p.status,
                           kChkSQ) ||
            !smem_range_ok(sKV + kstage * Cfg::kTileBytes, Cfg::kTileBytes, smem, Cfg::kOffKV, Cfg::kOffVt,
                           p.status, kChkSK))
          return;
#pragma unroll
        for (int kk = 0; kk < D / Cfg::kKeysPerMma; ++kk) {
          // K-major, kSwz-byte swizzle: each product consumes 32 bytes of the
          // head dim; four (128-byte swizzle) or two (64-byte) span one chunk
          // row.
          constexpr int kPerRow = kSwz / 32;   // products per swizzled row
          const uint32_t off = ((kk / kPerRow) * Cfg::kChunkBytes + (kk % kPerRow) * 32) >> 4;
          mma_ss(tmem + Cfg::kColS + t * 128, a0 + off, b0 + off, idesc_s, kk > 0, kF8);
        }
      };
      // One half (64 keys) of O_t += P_t V_j.
      auto issue_pv_half = [&](int t, uint32_t vstage, int h, bool acc) {
        const uint64_t b0 = dV + static_cast<uint64_t>((vstage * Cfg::kTileBytes) >> 4);  // stage or Vt buffer
        constexpr int kSteps = 64 / Cfg::kKeysPerMma;
        if (!tmem_range_ok(tmem + Cfg::kColO + t * D, tmem, D, Cfg::kColO + t * D, Cfg::kColO + (t + 1) * D, p.status,
                           kChkOOut) ||
            !(VT ? smem_range_ok(sVt + vstage * Cfg::kTileBytes, Cfg::kTileBytes, smem, Cfg::kOffVt,
                                 Cfg::kOffVt + Cfg::kVtBytes, p.status, kChkVIn)
                 : smem_range_ok(sKV + vstage * Cfg::kTileBytes, Cfg::kTileBytes, smem, Cfg::kOffKV, Cfg::kOffVt,
                                 p.status, kChkVIn)))
          return;
#pragma unroll
        for (int kk = h * kSteps; kk < (h + 1) * kSteps; ++kk) {
          // P_t: 128 rows x 128 keys packed in TMEM (32 bytes = 8 columns per
          // product).  V_j: MN-major (head dim contiguous), kKeysPerMma keys
          // = kKeysPerMma swizzled rows of kSwz bytes per product.
          const uint32_t voff = VT ? ((kk * 32) >> 4) : ((kk * Cfg::kKeysPerMma * kSwz) >> 4);
          if (!tmem_range_ok(tmem + Cfg::kColS + t * 128 + kk * 8, tmem, 8, Cfg::kColS + t * 128,
                             Cfg::kColS + t * 128 + 64, p.status, kChkPIn))
            continue;
          mma_ts(tmem + Cfg::kColO + t * D, tmem + Cfg::kColS + t * 128 + kk * 8,
                 b0 + voff, idesc_o, (acc || kk > 0) ? 1u : 0u, kF8);
        }
      };
      // O_t += P_t V_j as soon as each half of P_t is in TMEM: the first
      // half's products run while the softmax still computes the second.
      auto pv = [&](int t, uint32_t vstage, bool acc) -> bool {
        for (int h = 0; h < 2; ++h) {
          if (!mbar_wait(p_full + 2 * t + h, p_cnt[t] & 1, p.status, abort_flag, kWherePFull, lim))
            return false;
          tc_fence_after();
          issue_pv_half(t, vstage, h, acc);
        }
        ++p_cnt[t];
        return true;
      };
      // Ablation (serial): wait until both tiles have published P(j-1)
      // before any product of step j, so that the tensor core never runs
      // while a softmax does (pv() then finds those phases complete).
      auto wait_p_both = [&](bool has0) -> bool {
        for (int t = has0 ? 0 : 1; t < 2; ++t)
          for (int h = 0; h < 2; ++h)
            if (!mbar_wait(p_full + 2 * t + h, p_cnt[t] & 1, p.status, abort_flag, kWherePFull, lim)) return false;
        return true;
      };
      auto wait_kv = [&](uint32_t idx) -> bool {
        bool r = mbar_wait(kv_full + (idx % S), (idx / S) & 1, p.status, abort_flag, kWhereKvFull, lim);
        tc_fence_after();
        return r;
      };
      // V_j for the P.V products: the ring stage itself, or (VT) the
      // transposed copy; returns the value pv() takes as its V "stage".
      auto wait_v = [&](uint32_t idx, bool& r) -> uint32_t {
        if constexpr (VT) {
          const uint32_t b = v_cnt & 1;
          r = mbar_wait(vt_full + b, (v_cnt >> 1) & 1, p.status, abort_flag, kWhereKvFull, lim);
          tc_fence_after();
          return b;
        } else {
          r = wait_kv(idx);
          return idx % S;
        }
      };
      // Release V_j after both tiles' products: the ring stage (the
      // transposer already released it under VT) or the transposed buffer.
      auto release_v = [&](uint32_t vstage) {
        if constexpr (VT) {
          mma_commit(vt_empty + vstage);
          ++v_cnt;
        } else {
          mma_commit(kv_empty + vstage);
        }
      };

      for (int k = 0; ok; ++k, ++unit_iter) {
        const int unit = sched_unit(k, p.snake);
        if (unit >= p.n_units) break;
        int bh_, qp;
        decode_unit<CAUSAL>(unit, p.n_qpairs, p.BH, p.order, bh_, qp);
        (void)bh_;
        const int n0 = CAUSAL ? min(2 * qp + 1, n_kv) : n_kv;
        const int n1 = CAUSAL ? min(2 * qp + 2, n_kv) : n_kv;
        const uint32_t base = kv_iter;  // K_j at base + 2j, V_j at base + 2j + 1

        ok = mbar_wait(q_full, unit_iter & 1, p.status, abort_flag, kWhereQFull, lim);
        tc_fence_after();
        if (!ok) break;
        ok = wait_kv(base);
        if (!ok) break;
        issue_s(0, base % S);
        mma_commit(s_full + 0);
        issue_s(1, base % S);
        mma_commit(s_full + 1);
        mma_commit(kv_empty + (base % S));

        for (int j = 1; j < n1 && ok; ++j) {
          const uint32_t ik = base + 2 * j, iv = base + 2 * (j - 1) + 1;
          if (!(ok = wait_kv(ik))) break;
          const uint32_t vs = wait_v(iv, ok);
          if (!ok) break;
          if (SERIAL && !(ok = wait_p_both(j <= n0))) break;
          if (j < n0) {
            if (!(ok = pv(0, vs, j - 1 > 0))) break;
            issue_s(0, ik % S);
            if (!SERIAL) mma_commit(s_full + 0);
          } else if (j == n0) {
            if (!(ok = pv(0, vs, j - 1 > 0))) break;
            mma_commit(o_full + 0);
          }
          if (!(ok = pv(1, vs, j - 1 > 0))) break;
          release_v(vs);
          issue_s(1, ik % S);
          if (SERIAL && j < n0) mma_commit(s_full + 0);   // both S published together
          mma_commit(s_full + 1);
          mma_commit(kv_empty + (ik % S));
        }
        if (!ok) break;
        // the unit's last S products are issued: Q may be replaced by the next
        // unit's once they complete (the P.V products left do not read it)
        mma_commit(q_empty);
        const uint32_t iv = base + 2 * (n1 - 1) + 1;
        const uint32_t vs = wait_v(iv, ok);
        if (!ok) break;
        if (n0 == n1) {
          if (!(ok = pv(0, vs, n1 - 1 > 0))) break;
          mma_commit(o_full + 0);
        }
        if (!(ok = pv(1, vs, n1 - 1 > 0))) break;
        mma_commit(o_full + 1);
        release_v(vs);
        kv_iter += 2 * n1;
      }
      if (!ok) {
        // Wait for the MMAs already issued before TMEM is released.
        mma_commit(drain);
        volatile int never = 0;
        mbar_wait(drain, 0, nullptr, &never, kWhereDrain, 100000000ull);
      }
    }
    __syncwarp();
  } else if (VT) {
    // ---------------------------------------------------------- V transpose
    // Warps 2-3: each V tile of the ring, in the order the MMA consumes
    // them, into one of two K-major buffers; then release the ring stage.
    const int tt = threadIdx.x - 64;              // 0..63
    uint32_t kv_iter = 0, v_cnt = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int unit = sched_unit(k, p.snake);
      if (unit >= p.n_units) break;
      int bh_, qp;
      decode_unit<CAUSAL>(unit, p.n_qpairs, p.BH, p.order, bh_, qp);
      (void)bh_;
      const int n1 = CAUSAL ? min(2 * qp + 2, n_kv) : n_kv;
      for (int j = 0; j < n1; ++j, ++v_cnt) {
        const uint32_t iv = kv_iter + 2 * j + 1;
        const uint32_t b = v_cnt & 1;
        bool w = mbar_wait(kv_full + (iv % S), (iv / S) & 1, p.status, abort_flag, kWhereKvFull, lim);
        w = w && mbar_wait(vt_empty + b, ((v_cnt >> 1) & 1) ^ 1, p.status, abort_flag, kWhereKvEmpty, lim);
        if (!__all_sync(0xffffffffu, w)) *abort_flag = 1;
        named_bar_sync(3, 64);
        if (*abort_flag) { ok = false; break; }
        if (smem_range_ok(sKV + (iv % S) * Cfg::kTileBytes, Cfg::kTileBytes, smem, Cfg::kOffKV, Cfg::kOffVt, p.status,
                          kChkVtSrc) &&
            smem_range_ok(sVt + b * Cfg::kTileBytes, Cfg::kTileBytes, smem, Cfg::kOffVt, Cfg::kOffVt + Cfg::kVtBytes,
                          p.status, kChkVtDst))
          transpose_v_tile_e4m3(sKV + (iv % S) * Cfg::kTileBytes, sVt + b * Cfg::kTileBytes, tt);
        // generic-proxy shared-memory writes, read next by the tensor core
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        named_bar_sync(3, 64);
        if (tt == 0) {
          mbar_arrive(kv_empty + (iv % S));
          mbar_arrive(vt_full + b);
        }
      }
      kv_iter += 2 * n1;
    }
  }
  } else {
    reg_alloc<kRegsHigh>();
    // -------------------------------------------------------------- softmax
    const int t = (warp - 4) >> 2;                 // Q tile (slot) 0 or 1
    const int quarter = warp & 3;                  // TMEM lane quarter this warp may access
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + Cfg::kColS + t * 128;
    const uint32_t tO = tmem + lane_off + Cfg::kColO + t * D;
    uint32_t s_cnt = 0, o_cnt = 0;
    bool ok = true;
    // FP8: P is multiplied by this power of two before rounding to e4m3, and
    // the max may lag the true max by at most kLazy (log2 units) so that
    // P * gain <= 256 * 2^0.75 < 448 stays finite in e4m3.
    constexpr float kPGain = 256.0f;
    constexpr float kLazy = kF8 ? 0.75f : 8.0f;

    for (int k = 0; ok; ++k) {
      const int unit = sched_unit(k, p.snake);
      if (unit >= p.n_units) break;
      int bh, qp;
      decode_unit<CAUSAL>(unit, p.n_qpairs, p.BH, p.order, bh, qp);
      const int nt = CAUSAL ? min(2 * qp + t + 1, n_kv) : n_kv;
      const int row = qp * 256 + t * 128 + row_in_tile;
      float m = -INFINITY, l = 0.f;
      float cq = p.scale_log2;   // score -> log2 domain factor (times q descale for FP8)
      float vmax = 1.0f;         // FP8: max v descale of this head
      if constexpr (kF8) {
        const size_t dbase = static_cast<size_t>(bh) * n_kv;
        const int qblk = qp * 2 + t;
        cq *= p.q_desc[dbase + min(qblk, n_kv - 1)];
        float vm = 0.f;
        for (int b = lane; b < n_kv; b += 32) vm = fmaxf(vm, p.v_desc[dbase + b]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) vm = fmaxf(vm, __shfl_xor_sync(0xffffffffu, vm, o));
        vmax = vm;
      }

      for (int j = 0; j < nt; ++j) {
        bool w = mbar_wait(s_full + t, s_cnt & 1, p.status, abort_flag, kWhereSFull, lim);
        ++s_cnt;
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
#if ATTN_DEBUG_BOUNDS
          // test hook (fault mode 2): CTA 0's first S load is checked as if it
          // were 512 columns further on, so that check fails; the load itself
          // is not shifted, and the failed check skips it
          const uint32_t shift = (p.fault == 2 && blockIdx.x == 0 && k == 0 && j == 0 && cc == 0) ? 512u : 0u;
#else
          constexpr uint32_t shift = 0u;
#endif
          if (tmem_range_ok(tS + cc * 32 + shift, tmem, 32, Cfg::kColS + t * 128, Cfg::kColS + t * 128 + 128,
                            p.status, kChkSLoad))
            tmem_ld32(tS + cc * 32, r);
#pragma unroll
          for (int i = 0; i < 32; ++i) s[cc * 32 + i] = __uint_as_float(r[i]);
        }
        tmem_wait_ld();
        tmem_reg_fence(s);

        const int key0 = j * 128;
        const bool need_mask = (CAUSAL && key0 + 127 > qp * 256 + t * 128) || (key0 + 128 > p.N);
        if (need_mask) {
          const int lim_key = CAUSAL ? min(row, p.N - 1) : (p.N - 1);
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (key0 + i > lim_key) s[i] = -INFINITY;
        }
        const float mx = row_max128(s) * c;
        // Lazy max: raise m only when the tile max exceeds it by more than
        // kLazy (log2 units); then alpha = 2^(m_old - m_new), 0 on the first
        // tile.  The final division by l makes the stale max exact.
        float alpha = 1.0f;
        if (mx > m + kLazy) {
          alpha = ex2_approx(m - mx);
          m = mx;
        }
        // Rescale O_t when some row of this warp raised its max, before the
        // first half of P is published (its PV product accumulates into O_t).
        // The PV product of the previous key tile has completed: S_t(j) was
        // committed after it.
        // (16 columns at a time: with the 128 scores live, wider chunks
        // would spill)
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll 1
          for (int cc = 0; cc < D / 16; ++cc) {
            uint32_t r[16];
            if (!tmem_range_ok(tO + cc * 16, tmem, 16, Cfg::kColO + t * D, Cfg::kColO + (t + 1) * D, p.status,
                               kChkORescale))
              continue;
            tmem_ld16(tO + cc * 16, r);
            tmem_wait_ld();
            tmem_reg_fence(r);
#pragma unroll
            for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st16(tO + cc * 16, r);
            tmem_wait_st();       // the store reads r asynchronously; the next chunk reloads it
            tmem_reg_fence(r);
          }
        }
        // P in two halves of 64 keys, each published as soon as it is in
        // TMEM (exp_pack_half returns with its store complete).  Masked tiles hold -inf scores, which only the MUFU path maps
        // to an exact 0; unmasked tiles may send part of their exp2 work to
        // the FMA pipe.
        float sum = 0.f;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (tmem_range_ok(tS + (kF8 ? 16 : 32) * h, tmem, kF8 ? 16 : 32, Cfg::kColS + t * 128,
                            Cfg::kColS + t * 128 + 64, p.status, kChkPStore))
            sum += need_mask ? exp_pack_half<kF8, T, false>(s, h, c, -m, pgain, tS)
                             : exp_pack_half<kF8, T, true>(s, h, c, -m, pgain, tS);
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(p_full + 2 * t + h);
        }
        l = l * alpha + sum;
      }
      if (!ok) break;

      // ------------------------------------------------------------ epilogue
      bool w = mbar_wait(o_full + t, o_cnt & 1, p.status, abort_flag, kWhereOFull, lim);
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
        if (tmem_range_ok(tO + cc * 32, tmem, 32, Cfg::kColO + t * D, Cfg::kColO + (t + 1) * D, p.status, kChkOLoad))
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
