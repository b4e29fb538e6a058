// quant_kernel.cuh — per-block FP8 e4m3 quantiser.
//
// FP8 with block quantisation keeps accuracy when some features are outliers (page
// "FlashAttention-3: Rekordverdächtige Geschwindigkeit und Präzision bei AI-Modellen",
// section "Analyse").  One CTA per (b, h, block of 128 rows):
//   a = max |x| over the block; scale = a / 448; q = e4m3_rn_satfinite(x * (448 / a)),
// both divisions correctly rounded fp32 (__fdiv_rn), the product rounded once (__fmul_rn).
// A block of zeros stores scale 1.
//
// HBM-bound: the block (128 x D fp32, at most 128 KB) is read once into registers — every
// thread issues all its 16-byte loads before reducing — then written as 4 codes per float4.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace attn {

constexpr int kQuantThreads = 512;

// VEC float4 per thread: 8 covers D <= 128 (two CTAs fit per SM), 16 covers D <= 256.
template <int VEC>
__global__ void __launch_bounds__(kQuantThreads)
quant_e4m3_kernel(const float* __restrict__ x, uint8_t* __restrict__ xq, float* __restrict__ scales,
                  int S, int D, int nsb) {
  __shared__ float warp_max[kQuantThreads / 32];
  const int blk = blockIdx.x;
  const int bh = blk / nsb, sb = blk % nsb;
  const int r0 = sb * 128;
  const int rows = min(128, S - r0);
  const size_t base = (static_cast<size_t>(bh) * S + r0) * D;
  const int n4 = rows * D / 4;   // D is a multiple of 16
  const float4* src = reinterpret_cast<const float4*>(x + base);

  float4 v[VEC];
  float m = 0.f;
#pragma unroll
  for (int u = 0; u < VEC; ++u) {
    const int i = threadIdx.x + u * kQuantThreads;
    v[u] = i < n4 ? __ldcs(src + i) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int u = 0; u < VEC; ++u)
    m = fmaxf(m, fmaxf(fmaxf(fabsf(v[u].x), fabsf(v[u].y)), fmaxf(fabsf(v[u].z), fabsf(v[u].w))));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = m;
  __syncthreads();
  float a = 0.f;
#pragma unroll
  for (int w = 0; w < kQuantThreads / 32; ++w) a = fmaxf(a, warp_max[w]);
  const bool zero = !(a > 0.f);
  const float mult = zero ? 1.f : __fdiv_rn(448.f, a);
  if (threadIdx.x == 0) scales[static_cast<size_t>(bh) * nsb + sb] = zero ? 1.f : __fdiv_rn(a, 448.f);

  uint32_t* dst = reinterpret_cast<uint32_t*>(xq + base);
#pragma unroll
  for (int u = 0; u < VEC; ++u) {
    const int i = threadIdx.x + u * kQuantThreads;
    if (i < n4) {
      const uint32_t lo = pack_e4m3x2(__fmul_rn(v[u].x, mult), __fmul_rn(v[u].y, mult));
      const uint32_t hi = pack_e4m3x2(__fmul_rn(v[u].z, mult), __fmul_rn(v[u].w, mult));
      __stcs(dst + i, lo | (hi << 16));
    }
  }
}

}  // namespace attn
