// K1: per-key-block statistics of K and V.
//
// For key block j of head (b, h) -- rows [j*BLK, min(N, (j+1)*BLK)) -- it
// writes
//   ksum[bh][j][c]   float64 sum of the raw K values of channel c (used for the
//                    pooled block means of the mask and for the channel mean);
//   kexp[bh][j][c]   largest and smallest bf16 exponent field among the nonzero
//                    K values of the channel (checks that the float64 sums are
//                    exact);
//   hstate[bh][j][:] the linear-attention state of the block, bf16:
//                    h_j = sum_n phi(k_n) v_n^T as a D x D row-major matrix
//                    followed by z_j = sum_n phi(k_n) (D values), phi = elu + 1.
// ("Turbo Diffusion：秒级生成与高清保真的视频扩散技术突破", section 三(二) SLA
// item 2: the non-selected blocks go through an O(N) linear branch; section
// 三(一) item 1: K smoothing needs the channel mean.)
#pragma once
#include <cuda_bf16.h>
#include "sm100.cuh"

namespace sla {

// phi = elu + 1: x + 1 for x > 0, exp(x) otherwise.
__device__ __forceinline__ float phi_elu1(float x) { return x > 0.f ? x + 1.f : expf(x); }

// bf16 exponent field of a raw 16-bit pattern.
__device__ __forceinline__ uint32_t bf16_exp_field(uint16_t b) { return (b >> 7) & 0xFFu; }

template <int D, int BLK>
__global__ void __launch_bounds__(256) k_kstats(const __nv_bfloat16* __restrict__ K,
                                               const __nv_bfloat16* __restrict__ V, double* __restrict__ ksum,
                                               uint8_t* __restrict__ kexp, __nv_bfloat16* __restrict__ hstate,
                                               int N, int NB, long long hpitch) {
  constexpr int VEC = 8;             // bf16 per 16-byte load
  constexpr int GROUPS = D / VEC;    // vector columns per row
  constexpr int RSTEP = 256 / GROUPS;
  constexpr int TILE = D / 16;       // each thread owns a TILE x TILE patch of h
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  float* phk = reinterpret_cast<float*>(smem_raw);                 // [BLK][D]
  float* vv = phk + BLK * D;                                       // [BLK][D]
  double* red = reinterpret_cast<double*>(vv + BLK * D);           // [RSTEP][D]
  uint32_t* ered = reinterpret_cast<uint32_t*>(red + RSTEP * D);   // [RSTEP][D] packed max|min

  const int j = blockIdx.x;
  const long long bh = blockIdx.y;
  const int tid = threadIdx.x;
  const int row0 = j * BLK;
  const int rows = min(BLK, N - row0);
  const __nv_bfloat16* kb = K + (bh * N + row0) * (long long)D;
  const __nv_bfloat16* vb = V + (bh * N + row0) * (long long)D;

  const int g = tid % GROUPS;
  double part[VEC];
  uint32_t emax[VEC], emin[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) { part[e] = 0.0; emax[e] = 0u; emin[e] = 255u; }
  for (int r = tid / GROUPS; r < BLK; r += RSTEP) {
    uint4 kr = make_uint4(0, 0, 0, 0), vr = make_uint4(0, 0, 0, 0);
    if (r < rows) {
      kr = *reinterpret_cast<const uint4*>(kb + (long long)r * D + g * VEC);
      if (hstate != nullptr) vr = *reinterpret_cast<const uint4*>(vb + (long long)r * D + g * VEC);
    }
    const uint16_t* kh = reinterpret_cast<const uint16_t*>(&kr);
    const uint16_t* vh = reinterpret_cast<const uint16_t*>(&vr);
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      const float kf = __uint_as_float(uint32_t(kh[e]) << 16);
      const float vf = __uint_as_float(uint32_t(vh[e]) << 16);
      part[e] += (double)kf;
      const uint32_t ef = bf16_exp_field(kh[e]);
      if ((kh[e] & 0x7FFFu) != 0u) { emax[e] = max(emax[e], ef); emin[e] = min(emin[e], ef); }
      phk[r * D + g * VEC + e] = (r < rows) ? phi_elu1(kf) : 0.f;
      vv[r * D + g * VEC + e] = vf;
    }
  }
  const int rg = tid / GROUPS;
#pragma unroll
  for (int e = 0; e < VEC; ++e) {
    red[rg * D + g * VEC + e] = part[e];
    ered[rg * D + g * VEC + e] = (emax[e] << 8) | emin[e];
  }
  __syncthreads();
  if (tid < D) {
    double s = 0.0;
    uint32_t mx = 0u, mn = 255u;
    for (int q = 0; q < RSTEP; ++q) {
      s += red[q * D + tid];
      const uint32_t w = ered[q * D + tid];
      mx = max(mx, w >> 8);
      mn = min(mn, w & 0xFFu);
    }
    const long long o = (bh * NB + j) * (long long)D + tid;
    ksum[o] = s;
    kexp[2 * o] = (uint8_t)mx;
    kexp[2 * o + 1] = (uint8_t)mn;
  }

  if (hstate == nullptr) return;
  // h = phi(K)^T V on the CUDA cores (float32 accumulation), then bf16.
  const int ta = (tid / 16) * TILE, tc = (tid % 16) * TILE;
  float acc[TILE][TILE];
#pragma unroll
  for (int x = 0; x < TILE; ++x)
#pragma unroll
    for (int y = 0; y < TILE; ++y) acc[x][y] = 0.f;
  for (int n = 0; n < rows; ++n) {
    float pa[TILE], pv[TILE];
#pragma unroll
    for (int x = 0; x < TILE; ++x) pa[x] = phk[n * D + ta + x];
#pragma unroll
    for (int y = 0; y < TILE; ++y) pv[y] = vv[n * D + tc + y];
#pragma unroll
    for (int x = 0; x < TILE; ++x)
#pragma unroll
      for (int y = 0; y < TILE; ++y) acc[x][y] = fmaf(pa[x], pv[y], acc[x][y]);
  }
  __nv_bfloat16* hs = hstate + (bh * (long long)NB + j) * hpitch;
#pragma unroll
  for (int x = 0; x < TILE; ++x)
#pragma unroll
    for (int y = 0; y < TILE; ++y) hs[(ta + x) * D + tc + y] = __float2bfloat16_rn(acc[x][y]);
  if (tid < D) {
    float z = 0.f;
    for (int n = 0; n < rows; ++n) z += phk[n * D + tid];
    hs[D * D + tid] = __float2bfloat16_rn(z);
  }
}

template <int D, int BLK>
constexpr size_t kstats_smem() {
  return size_t(2) * BLK * D * sizeof(float) + size_t(256 / (D / 8)) * D * (sizeof(double) + sizeof(uint32_t));
}

// mu[bh][c] = float32 nearest to (sum_j ksum[bh][j][c]) / N.  The block sums
// are exact when every K value of the channel is a multiple of the smallest
// one's unit in the last place and the total stays below 2^53 of those units;
// kexp lets the kernel check that and raise DEV_ERR_INEXACT otherwise.
__global__ void k_channel_mean(const double* __restrict__ ksum, const uint8_t* __restrict__ kexp,
                               float* __restrict__ mu, int NB, int D, int N, long long total) {
  const long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (t >= total) return;
  const long long bh = t / D;
  const int c = int(t % D);
  double s = 0.0;
  uint32_t mx = 0u, mn = 255u;
  for (int j = 0; j < NB; ++j) {
    const long long o = (bh * NB + j) * (long long)D + c;
    s += ksum[o];
    mx = max(mx, (uint32_t)kexp[2 * o]);
    mn = min(mn, (uint32_t)kexp[2 * o + 1]);
  }
  int lgN = 0;
  while ((1LL << lgN) < (long long)N) ++lgN;
  if (mx >= mn && int(mx) - int(mn) + 8 + lgN + 1 > 53) raise_error(DEV_ERR_INEXACT);
  // Correct rounding of s / N to float32: the float64 quotient q is within
  // half a float64 ulp of s/N, so it rounds to the same float32 unless q is a
  // float32 midpoint; then the sign of the exact remainder s - q*N decides.
  const double dn = (double)N;
  const double q = s / dn;
  float f = __double2float_rn(q);
  const double fd = (double)f;
  if (fd != q) {
    // neighbouring float32 on the other side of q
    const float g2 = (q > fd) ? nextafterf(f, INFINITY) : nextafterf(f, -INFINITY);
    const double mid = 0.5 * (fd + (double)g2);
    if (mid == q) {
      const double rem = fma(-q, dn, s);  // exact: s - q*N
      if (rem == 0.0) {
        f = (__float_as_uint(f) & 1u) ? g2 : f;   // exact tie: even mantissa
      } else {
        const bool above = rem > 0.0;             // s/N > q
        const float lo = fminf(f, g2), hi = fmaxf(f, g2);
        f = above ? hi : lo;
      }
    }
  }
  mu[t] = f;
}

}  // namespace sla
