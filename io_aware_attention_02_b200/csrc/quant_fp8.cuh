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
// One CTA per (block of 128 rows, batch*head); 256 threads; each row is
// handled by D/8 threads holding 8 consecutive values, so the fast
// Walsh-Hadamard transform runs three butterfly stages in registers and the
// rest across lanes with shuffles.  Pure streaming kernel: it reads 2 bytes
// and writes 1 byte per element, bound by HBM bandwidth.
#pragma once
#include "ptx.cuh"

namespace attn {

template <int D>
__global__ void __launch_bounds__(256) attn_quant_fp8_kernel(
    const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ x8, float* __restrict__ descale,
    const float* __restrict__ signs, int N, int n_blocks, int hadamard) {
  constexpr int TPR = D / 8;              // threads per row
  constexpr int RPP = 256 / TPR;          // rows per pass
  constexpr int PASSES = 128 / RPP;
  const int blk = blockIdx.x % n_blocks;
  const int bh = blockIdx.x / n_blocks;
  const int tid = threadIdx.x;
  const int rip = tid / TPR;              // row within pass
  const int seg = tid % TPR;              // 8-value segment within the row
  const size_t head_off = static_cast<size_t>(bh) * N * D;

  float y[PASSES][8];
  float amax = 0.f;
#pragma unroll
  for (int ps = 0; ps < PASSES; ++ps) {
    const int row = blk * 128 + ps * RPP + rip;
    if (row < N) {
      const uint4 raw = *reinterpret_cast<const uint4*>(x + head_off + static_cast<size_t>(row) * D + seg * 8);
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
    if (hadamard) {
      if (signs != nullptr) {
#pragma unroll
        for (int i = 0; i < 8; ++i) y[ps][i] *= signs[seg * 8 + i];
      }
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
        const bool upper = (seg & m) != 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float other = __shfl_xor_sync(0xffffffffu, y[ps][i], m);
          y[ps][i] = upper ? (other - y[ps][i]) : (y[ps][i] + other);
        }
      }
      const float norm = rsqrtf(static_cast<float>(D));
#pragma unroll
      for (int i = 0; i < 8; ++i) y[ps][i] *= norm;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(y[ps][i]));
  }

  // block amax
  __shared__ float red[8];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((tid & 31) == 0) red[tid >> 5] = amax;
  __syncthreads();
  float bmax = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) bmax = fmaxf(bmax, red[w]);
  const float s = (bmax == 0.f) ? 1.0f : __fdiv_rn(bmax, 448.0f);
  if (tid == 0) descale[static_cast<size_t>(bh) * n_blocks + blk] = s;

#pragma unroll
  for (int ps = 0; ps < PASSES; ++ps) {
    const int row = blk * 128 + ps * RPP + rip;
    if (row < N) {
      uint2 out;
      out.x = pack4_e4m3(__fdiv_rn(y[ps][0], s), __fdiv_rn(y[ps][1], s), __fdiv_rn(y[ps][2], s),
                         __fdiv_rn(y[ps][3], s));
      out.y = pack4_e4m3(__fdiv_rn(y[ps][4], s), __fdiv_rn(y[ps][5], s), __fdiv_rn(y[ps][6], s),
                         __fdiv_rn(y[ps][7], s));
      *reinterpret_cast<uint2*>(x8 + head_off + static_cast<size_t>(row) * D + seg * 8) = out;
    }
  }
}

}  // namespace attn
