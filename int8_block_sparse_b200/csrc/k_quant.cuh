// K2: fused smooth + quantise, one CTA per (tensor, head, block of tokens).
//
// "Turbo Diffusion：秒级生成与高清保真的视频扩散技术突破", section 三(一)
// SageAttention2++: item 1 (smooth outliers before quantising -- here K minus
// its per-channel mean over tokens) and item 2 (every sub-block has its own
// quantisation parameters -- here one float32 scale per block of BLK tokens x
// D channels, or, finer, one per group of 2^gshift tokens x D channels
// inside the block: G = BLK >> gshift groups).  Per group: m = max|x|, s = m /
// 127 (IEEE float32 division), code = clamp(round_half_even(float32(x / s)),
// -127, 127) (the clamp never acts: see pack_i8x4); a group with m = 0 has
// s = 0 and zero codes.  Rows past N (up to NB*BLK) get zero codes.  For Q the kernel also writes the
// float64 mean of each block's valid rows (the pooled query block of the mask).
//
// The smoothed K value is recomputed (one float32 subtraction) when it is
// quantised.  The quotient x / s is taken as y0 = x * (1/s): with
// y = float32(x / s), |y - y0| < 2e-5 for |x / s| <= 128 (two float32
// roundings of relative size 2^-24 plus half an ulp of y), so
// round_half_even(y) = round_half_even(y0) unless y0 lies within 3e-5 of a
// half-integer; only then is the IEEE division done.
#pragma once
#include <cuda_bf16.h>
#include "sm100.cuh"

namespace sla {

__device__ __forceinline__ int quant_code(float x, float s, float rs) {
  const float y0 = x * rs;
  // round half to even through the 1.5 * 2^23 magic number (|y0| < 2^22)
  const float big = y0 + 12582912.f;
  const int q = __float_as_int(big) - 0x4B400000;
  const float d = y0 - (big - 12582912.f);   // y0 minus the chosen integer, in [-0.5, 0.5]
  if (fabsf(d) > 0.5f - 3e-5f) return __float2int_rn(__fdiv_rn(x, s));
  return q;
}

// Four codes -> four int8 bytes (code e in byte e), saturating to [-128, 127].
// Codes are in [-127, 127] already: |x| <= m gives |x / s| <= 127 up to one
// float32 rounding, which rounds to at most 127 in magnitude.
__device__ __forceinline__ uint32_t pack_i8x4(int c0, int c1, int c2, int c3) {
  uint32_t hi, r;
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, 0;" : "=r"(hi) : "r"(c3), "r"(c2));
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(c1), "r"(c0), "r"(hi));
  return r;
}

template <int D, int BLK>
struct QuantCfg {
  static constexpr int TILE_BYTES = BLK * D * 2;            // the bf16 block, rows past N zero-filled by the TMA
  static constexpr int RED_BYTES = 8 * D * 8 + 8 * 4 * 4;   // per-warp float64 partials, per-warp group maxima
  static constexpr int SMEM = TILE_BYTES + RED_BYTES + 16 + 1024;
};

// The block arrives in shared memory by one TMA load (several blocks per SM
// are in flight); pass 1 takes the maximum (and, for Q, the float64 sums),
// pass 2 quantises from shared memory.
// FINE: one scale per group of 2^gshift tokens inside the block (G groups);
// otherwise one per block (the default, its own code path).
template <int D, int BLK, bool FINE>
__global__ void __launch_bounds__(256) k_quant(const __grid_constant__ CUtensorMap tm_q,
                                              const __grid_constant__ CUtensorMap tm_k, const float* __restrict__ mu,
                                              int8_t* __restrict__ qi8, int8_t* __restrict__ ki8,
                                              float* __restrict__ sq, float* __restrict__ sk,
                                              double* __restrict__ qbar, int N, int NB, int z0, int gshift) {
  using C = QuantCfg<D, BLK>;
  constexpr int VEC = 8;
  constexpr int GROUPS = D / VEC;
  constexpr int NV = BLK * GROUPS / 256;   // 16-byte vectors per thread
  static_assert(NV >= 1 && (BLK * GROUPS) % 256 == 0, "tile shape");
  constexpr int RSTEP = 256 / GROUPS;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint16_t* tile = reinterpret_cast<const uint16_t*>(base);        // [BLK][D] bf16
  double* red = reinterpret_cast<double*>(base + C::TILE_BYTES);         // [8][D]
  float* wmax = reinterpret_cast<float*>(red + 8 * D);                   // [8 warps][4 groups]
  uint64_t* bar = reinterpret_cast<uint64_t*>(wmax + 32);

  const int j = blockIdx.x;
  const int bh = blockIdx.y;
  const bool isk = blockIdx.z + z0 == 1;   // grid z: {Q, K}, {Q} (z0 0) or {K} (z0 1)
  const int tid = threadIdx.x, warp = tid >> 5;
  const int row0 = j * BLK;
  const int rows = min(BLK, N - row0);
  const int g = tid % GROUPS;

  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    mbar_expect_tx(bar, C::TILE_BYTES);
    tma_load_3d(base, isk ? &tm_k : &tm_q, bar, 0, row0, bh);
  }
  float muc[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) muc[e] = isk ? mu[(long long)bh * D + g * VEC + e] : 0.f;
  __syncthreads();   // barrier initialised before anyone waits on it
  const bool landed = mbar_wait(bar, 0, nullptr);
  if (!__syncthreads_and(landed)) {
    // uniform exit if the load did not land in time; the copy may still be in
    // flight, so one thread waits for it once more (bounded) before the CTA's
    // shared memory is handed on
    if (tid == 0) (void)mbar_wait(bar, 0, nullptr);
    return;
  }

  // pass 1: maximum of |x| per group (K: x - mu on valid rows) and, for Q,
  // float64 channel sums
  constexpr int MG = FINE ? 4 : 1;              // group maxima a thread keeps
  const int G = FINE ? BLK >> gshift : 1;       // groups per block
  float gm[MG];
#pragma unroll
  for (int q = 0; q < MG; ++q) gm[q] = 0.f;
  double part[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) part[e] = 0.0;
#pragma unroll
  for (int t = 0; t < NV; ++t) {
    const int r = tid / GROUPS + t * RSTEP;
    const uint4 raw = *reinterpret_cast<const uint4*>(tile + r * D + g * VEC);
    const uint16_t* hv = reinterpret_cast<const uint16_t*>(&raw);
    float rmax = 0.f;
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      float f = __uint_as_float(uint32_t(hv[e]) << 16);
      if (!isk) part[e] += (double)f;                     // rows past N hold 0
      if (isk && r < rows) f = __fsub_rn(f, muc[e]);
      rmax = fmaxf(rmax, fabsf(f));
    }
    const int gi = FINE ? r >> gshift : 0;
#pragma unroll
    for (int q = 0; q < MG; ++q)
      if (gi == q) gm[q] = fmaxf(gm[q], rmax);
  }
  if (!isk && qbar != nullptr) {
    // lanes sharing a channel group combine first (fixed order), then warps
#pragma unroll
    for (int o = GROUPS; o < 32; o <<= 1)
#pragma unroll
      for (int e = 0; e < VEC; ++e) part[e] += __shfl_xor_sync(0xffffffffu, part[e], o);
    if ((tid & 31) < GROUPS)
#pragma unroll
      for (int e = 0; e < VEC; ++e) red[warp * D + g * VEC + e] = part[e];
  }
#pragma unroll
  for (int q = 0; q < MG; ++q) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) gm[q] = fmaxf(gm[q], __shfl_xor_sync(0xffffffffu, gm[q], o));
  }
  if ((tid & 31) == 0)
#pragma unroll
    for (int q = 0; q < MG; ++q) wmax[warp * 4 + q] = gm[q];
  __syncthreads();
  float gs[MG], grs[MG];   // scale and its reciprocal per group
#pragma unroll
  for (int q = 0; q < MG; ++q) {
    float m = wmax[q];
#pragma unroll
    for (int w = 1; w < 8; ++w) m = fmaxf(m, wmax[w * 4 + q]);
    gs[q] = __fdiv_rn(m, 127.0f);
    grs[q] = (gs[q] > 0.f) ? __frcp_rn(gs[q]) : 0.f;
  }
  float* sdst = isk ? sk : sq;
  if (tid < G && sdst != nullptr) {
    float sv = gs[0];
#pragma unroll
    for (int q = 1; q < MG; ++q)
      if (tid == q) sv = gs[q];
    sdst[((long long)bh * NB + j) * G + tid] = sv;
  }
  if (!isk && qbar != nullptr && tid < D) {
    double acc = 0.0;
#pragma unroll
    for (int w = 0; w < 8; ++w) acc += red[w * D + tid];
    qbar[((long long)bh * NB + j) * D + tid] = acc / (double)rows;
  }
  int8_t* dbase = isk ? ki8 : qi8;
  if (dbase == nullptr) return;
  // pass 2: codes, eight per 8-byte store
  int8_t* dst = dbase + ((long long)bh * NB * BLK + row0) * D;
#pragma unroll
  for (int t = 0; t < NV; ++t) {
    const int r = tid / GROUPS + t * RSTEP;
    const int gi = FINE ? r >> gshift : 0;
    float s = gs[0], rs = grs[0];
#pragma unroll
    for (int q = 1; q < MG; ++q)
      if (gi == q) {
        s = gs[q];
        rs = grs[q];
      }
    const uint4 raw = *reinterpret_cast<const uint4*>(tile + r * D + g * VEC);
    const uint16_t* hv = reinterpret_cast<const uint16_t*>(&raw);
    uint32_t packed[2] = {0u, 0u};
    if (s > 0.f) {
      int qv[VEC];
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        float f = __uint_as_float(uint32_t(hv[e]) << 16);
        if (isk && r < rows) f = __fsub_rn(f, muc[e]);
        qv[e] = quant_code(f, s, rs);
      }
      packed[0] = pack_i8x4(qv[0], qv[1], qv[2], qv[3]);
      packed[1] = pack_i8x4(qv[4], qv[5], qv[6], qv[7]);
    }
    *reinterpret_cast<uint2*>(dst + (long long)r * D + g * VEC) = make_uint2(packed[0], packed[1]);
  }
}

}  // namespace sla
