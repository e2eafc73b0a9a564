// K2: fused smooth + quantise, one CTA per (tensor, head, block of tokens).
//
// "Turbo Diffusion：秒级生成与高清保真的视频扩散技术突破", section 三(一)
// SageAttention2++: item 1 (smooth outliers before quantising -- here K minus
// its per-channel mean over tokens) and item 2 (every sub-block has its own
// quantisation parameters -- here one float32 scale per block of BLK tokens x
// D channels).  Per block: m = max|x|, s = m / 127 (IEEE float32 division),
// code = clamp(round_half_even(float32(x / s)), -127, 127); a block with m = 0
// has s = 0 and zero codes.  Rows past N (up to NB*BLK) get zero codes.  For Q
// the kernel also writes the float64 mean of each block's valid rows (the
// pooled query block of the mask).
//
// The block stays in registers as packed bf16 (the smoothed K value is
// recomputed, one float32 subtraction, when it is quantised).  The quotient
// x / s is taken as y0 = x * (1/s): with y = float32(x / s), |y - y0| < 2e-5
// for |x / s| <= 128 (two float32 roundings of relative size 2^-24 plus half
// an ulp of y), so round_half_even(y) = round_half_even(y0) unless y0 lies
// within 3e-5 of a half-integer; only then is the IEEE division done.
#pragma once
#include <cuda_bf16.h>
#include "sm100.cuh"

namespace sla {

__device__ __forceinline__ int quant_code(float x, float s, float rs) {
  const float y0 = x * rs;
  // round half to even through the 1.5 * 2^23 magic number (|y0| < 2^22)
  const float big = y0 + 12582912.f;
  int q = __float_as_int(big) - 0x4B400000;
  const float frac = fabsf(y0 - (big - 12582912.f));   // distance to the chosen integer
  if (fabsf(frac - 0.5f) < 3e-5f) q = __float2int_rn(__fdiv_rn(x, s));
  return max(-127, min(127, q));
}

template <int D, int BLK>
__global__ void __launch_bounds__(256) k_quant(const __nv_bfloat16* __restrict__ Q,
                                              const __nv_bfloat16* __restrict__ K, const float* __restrict__ mu,
                                              int8_t* __restrict__ qi8, int8_t* __restrict__ ki8,
                                              float* __restrict__ sq, float* __restrict__ sk,
                                              double* __restrict__ qbar, int N, int NB) {
  constexpr int VEC = 8;
  constexpr int GROUPS = D / VEC;
  constexpr int NV = BLK * GROUPS / 256;   // 16-byte vectors per thread
  static_assert(NV >= 1 && (BLK * GROUPS) % 256 == 0, "tile shape");
  constexpr int RSTEP = 256 / GROUPS;
  __shared__ float wmax[8];
  __shared__ double red[8][D];

  const int j = blockIdx.x;
  const long long bh = blockIdx.y;
  const bool isk = blockIdx.z == 1;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int row0 = j * BLK;
  const int rows = min(BLK, N - row0);
  const __nv_bfloat16* src = (isk ? K : Q) + (bh * N + row0) * (long long)D;
  const int g = tid % GROUPS;

  uint4 raw[NV];
#pragma unroll
  for (int t = 0; t < NV; ++t) {
    const int r = tid / GROUPS + t * RSTEP;
    raw[t] = (r < rows) ? *reinterpret_cast<const uint4*>(src + (long long)r * D + g * VEC) : make_uint4(0, 0, 0, 0);
  }
  float muc[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) muc[e] = isk ? mu[bh * D + g * VEC + e] : 0.f;

  float mloc = 0.f;
  double part[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) part[e] = 0.0;
#pragma unroll
  for (int t = 0; t < NV; ++t) {
    const int r = tid / GROUPS + t * RSTEP;
    const uint16_t* hv = reinterpret_cast<const uint16_t*>(&raw[t]);
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      float f = __uint_as_float(uint32_t(hv[e]) << 16);
      if (!isk) part[e] += (double)f;                     // padding rows hold 0
      if (isk && r < rows) f = __fsub_rn(f, muc[e]);
      mloc = fmaxf(mloc, fabsf(f));
    }
  }
  if (!isk && qbar != nullptr) {
    // lanes sharing a channel group combine first (fixed order), then warps
#pragma unroll
    for (int o = GROUPS; o < 32; o <<= 1)
#pragma unroll
      for (int e = 0; e < VEC; ++e) part[e] += __shfl_xor_sync(0xffffffffu, part[e], o);
    if ((tid & 31) < GROUPS)
#pragma unroll
      for (int e = 0; e < VEC; ++e) red[warp][g * VEC + e] = part[e];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, o));
  if ((tid & 31) == 0) wmax[warp] = mloc;
  __syncthreads();
  float m = wmax[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) m = fmaxf(m, wmax[w]);
  const float s = __fdiv_rn(m, 127.0f);
  float* sdst = isk ? sk : sq;
  if (tid == 0 && sdst != nullptr) sdst[bh * NB + j] = s;
  if (!isk && qbar != nullptr && tid < D) {
    double acc = 0.0;
#pragma unroll
    for (int w = 0; w < 8; ++w) acc += red[w][tid];
    qbar[(bh * NB + j) * (long long)D + tid] = acc / (double)rows;
  }
  int8_t* dbase = isk ? ki8 : qi8;
  if (dbase == nullptr) return;
  int8_t* dst = dbase + (bh * (long long)NB * BLK + row0) * (long long)D;
  const float rs = (s > 0.f) ? __frcp_rn(s) : 0.f;
#pragma unroll
  for (int t = 0; t < NV; ++t) {
    const int r = tid / GROUPS + t * RSTEP;
    const uint16_t* hv = reinterpret_cast<const uint16_t*>(&raw[t]);
    uint32_t packed[2] = {0u, 0u};
    if (s > 0.f) {
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        float f = __uint_as_float(uint32_t(hv[e]) << 16);
        if (isk && r < rows) f = __fsub_rn(f, muc[e]);
        const int qv = quant_code(f, s, rs);
        packed[e >> 2] |= (uint32_t(qv) & 0xFFu) << (8 * (e & 3));
      }
    }
    *reinterpret_cast<uint2*>(dst + (long long)r * D + g * VEC) = make_uint2(packed[0], packed[1]);
  }
}

}  // namespace sla
