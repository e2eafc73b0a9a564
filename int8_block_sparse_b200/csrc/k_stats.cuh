// K1: per-key-block statistics of K and V.
//
// For key block j of head (b, h) -- rows [j*BLK, min(N, (j+1)*BLK)) -- it
// writes
//   ksum[bh][j][c]   float64 sum of the raw K values of channel c (for the
//                    channel mean);
//   kbar[bh][c][j]   float64 mean of those values (the pooled block of the mask),
//                    channel-major so that the mask reads contiguous channel slabs
//                    (row pitch kbar_pitch(NB), a multiple of 16 bytes);
//   kexp[bh][j][c]   largest and smallest bf16 exponent field among the nonzero
//                    K values of the channel (checks that the float64 sums are
//                    exact);
//   hstate[bh][j][:] (optional) the block's linear-attention state, bf16:
//                    h'_j = sum_n phi(k_n) (v_n W_proj)^T as a D x D row-major
//                    matrix followed by z_j = sum_n phi(k_n) (D values),
//                    phi = elu + 1.
// ("Turbo Diffusion：秒级生成与高清保真的视频扩散技术突破", section 三(二) SLA
// item 2: the non-selected blocks go through an O(N) linear branch with a
// linear projection; section 三(一) item 1: K smoothing needs the channel mean.)
//
// W_proj is folded into the states: O_lin W = phi(q) (sum_j h_j) W / den =
// phi(q) (sum_j phi(K_j)^T (V_j W)) / den, so the query side needs one product
// instead of two.  Both products run on the tensor cores (bf16 operands,
// float32 accumulation): V'_j = V_j W with the TMA-loaded V tile as a K-major A
// operand, then h'_j = phi(K_j)^T V'_j with phi(K_j)^T built in shared memory as
// an MN-major A operand and V'_j written back over V_j as an MN-major B operand.
#pragma once
#include <cuda_bf16.h>
#include "exact_mean.cuh"
#include "sm100.cuh"

namespace sla {

// phi = elu + 1: x + 1 for x > 0, exp(x) otherwise (the fast exponential: phi
// enters h' as bf16 and z as a float32 sum).
__device__ __forceinline__ float phi_elu1(float x) { return x > 0.f ? x + 1.f : __expf(x); }

// A normal or zero bf16 value (raw bits) as a float64, built from its fields
// (exact; subnormal bf16 values are converted by the caller instead).
__device__ __forceinline__ double bf16_normal_to_f64(uint32_t h) {
  const uint64_t sgn = uint64_t(h & 0x8000u) << 48;
  const uint32_t e = (h >> 7) & 0xFFu;
  const uint64_t bits = e ? (sgn | (uint64_t(e + 896u) << 52) | (uint64_t(h & 0x7Fu) << 45)) : sgn;
  return __longlong_as_double((long long)bits);
}

// Row pitch (in doubles) of the channel-major pooled K blocks: NB rounded up
// to an even count, so that rows start on 16-byte boundaries (TMA strides).
__host__ __device__ __forceinline__ long long kbar_pitch(int NB) { return (NB + 1) & ~1; }

template <int D, int BLK>
struct StatsCfg {
  static constexpr int V_BYTES = BLK * D * 2;        // V tile, then V' (MN-major, 64-channel atoms)
  static constexpr int W_BYTES = D * D * 2;          // W_proj (MN-major B)
  static constexpr int P_BYTES = 128 * BLK * 2;      // phi(K)^T (MN-major A, 128 rows of a; D=64 pads)
  static constexpr int THREADS = 256;
  static constexpr int WARPS = THREADS / 32;
  static constexpr int GROUPS = D / 8;               // 16-byte vectors per row
  static constexpr int RG = THREADS / GROUPS;        // row groups (threads per channel group)
  static constexpr int RED_BYTES = WARPS * D * (8 + 4 + 2);  // per-warp partials after a shuffle step
  // two CTAs per SM (228 KB, 1 KB of it reserved per CTA)
  static constexpr int SMEM = V_BYTES + W_BYTES + P_BYTES + RED_BYTES + 1024 + 128;
  static_assert(D != 128 || BLK != 128 || 2 * (SMEM + 1024) <= 233472, "two CTAs per SM");
};

template <int D, int BLK>
__global__ void __launch_bounds__(256, 2) k_kstats(const __grid_constant__ CUtensorMap tm_v,
                                               const __grid_constant__ CUtensorMap tm_w,
                                               const __nv_bfloat16* __restrict__ K, double* __restrict__ ksum,
                                               double* __restrict__ kbar, uint8_t* __restrict__ kexp,
                                               __nv_bfloat16* __restrict__ hstate, int N, int NB,
                                               long long hpitch) {
  using C = StatsCfg<D, BLK>;
  constexpr int GROUPS = C::GROUPS, RG = C::RG;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sV = base;
  unsigned char* sW = sV + C::V_BYTES;
  unsigned char* sP = sW + C::W_BYTES;
  double* red = reinterpret_cast<double*>(sP + C::P_BYTES);        // [WARPS][D]
  float* redz = reinterpret_cast<float*>(red + C::WARPS * D);      // [WARPS][D]
  uint16_t* rede = reinterpret_cast<uint16_t*>(redz + C::WARPS * D);   // [WARPS][D] max<<8 | min
  uint64_t* bars = reinterpret_cast<uint64_t*>(rede + C::WARPS * D);   // 0: TMA, 1: MMA0, 2: MMA1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int j = blockIdx.x;
  const long long bh = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int row0 = j * BLK;
  const int rows = min(BLK, N - row0);
  const bool states = hstate != nullptr;

  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    mbar_init(&bars[2], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (states && warp == 0) {
    tmem_alloc(tmem_slot, D);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = states ? *tmem_slot : 0u;

  if (states && tid == 0) {
    mbar_expect_tx(&bars[0], C::V_BYTES + C::W_BYTES);
#pragma unroll
    for (int hh = 0; hh < D / 64; ++hh) {
      tma_load_3d(sV + hh * BLK * 128, &tm_v, &bars[0], hh * 64, row0, (int)bh);
      tma_load_2d(sW + hh * D * 128, &tm_w, &bars[0], hh * 64, 0);
    }
  }

  // K rows: float64 sums, exponent range, phi (float32 sums for z, bf16 for h').
  // All of the thread's rows are loaded first, so their DRAM latencies overlap.
  const __nv_bfloat16* kb = K + (bh * N + row0) * (long long)D;
  const int g = tid % GROUPS, rg = tid / GROUPS;
  constexpr int NR = BLK / RG;   // rows per thread
  uint4 kr[NR];
#pragma unroll
  for (int t = 0; t < NR; ++t) {
    const int r = rg + t * RG;
    kr[t] = (r < rows) ? *reinterpret_cast<const uint4*>(kb + (long long)r * D + g * 8) : make_uint4(0, 0, 0, 0);
  }
  double part[8];
  float zp[8];
  // magnitudes (sign cleared) of channel pairs, packed 16-bit: largest, and
  // smallest nonzero (0x7FFF = none); their exponent fields bound the channel's
  uint32_t mxp[4], mnp[4];
#pragma unroll
  for (int e = 0; e < 8; ++e) { part[e] = 0.0; zp[e] = 0.f; }
#pragma unroll
  for (int w = 0; w < 4; ++w) { mxp[w] = 0u; mnp[w] = 0x7FFF7FFFu; }
#pragma unroll
  for (int t = 0; t < NR; ++t) {
    const int r = rg + t * RG;
    const uint32_t wv[4] = {kr[t].x, kr[t].y, kr[t].z, kr[t].w};
    bool sub = false;   // a subnormal bf16 among the eight values
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint32_t m = wv[w] & 0x7FFF7FFFu;
      mxp[w] = __vmaxu2(mxp[w], m);
      mnp[w] = __vminu2(mnp[w], m | (__vcmpeq2(m, 0u) & 0x7FFF7FFFu));
      const uint32_t ez = __vcmpeq2(m & 0x7F807F80u, 0u) & ~__vcmpeq2(m, 0u);
      sub = sub || ez != 0u;
    }
    uint32_t pk[4];
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      const uint32_t h0 = wv[e >> 1] & 0xFFFFu, h1 = wv[e >> 1] >> 16;
      const float k0 = __uint_as_float(h0 << 16), k1 = __uint_as_float(h1 << 16);
      if (!sub) {
        part[e] += bf16_normal_to_f64(h0);
        part[e + 1] += bf16_normal_to_f64(h1);
      } else {
        part[e] += (double)k0;
        part[e + 1] += (double)k1;
      }
      const float p0 = (r < rows) ? phi_elu1(k0) : 0.f, p1 = (r < rows) ? phi_elu1(k1) : 0.f;
      zp[e] += p0;
      zp[e + 1] += p1;
      pk[e >> 1] = pack_bf16x2(p0, p1);
    }
    if (states) {
      // phi(K)^T, MN-major: channel a = g*8.. is the M index, row r the K index
      const int atom = (g * 8) / 64, chunk = ((g * 8) % 64) / 8;
      *reinterpret_cast<uint4*>(sP + atom * BLK * 128 + sw128_offset(r, chunk)) =
          make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
  }
  if (states && D == 64) {
    // rows a = 64..127 of the 128-row A operand are zero
    for (int e = tid; e < BLK * 128 / 16; e += C::THREADS)
      reinterpret_cast<uint4*>(sP + BLK * 128)[e] = make_uint4(0, 0, 0, 0);
  }
  // lanes of a warp that share a channel group first combine (fixed order)
#pragma unroll
  for (int o = GROUPS; o < 32; o <<= 1) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      part[e] += __shfl_xor_sync(0xffffffffu, part[e], o);
      zp[e] += __shfl_xor_sync(0xffffffffu, zp[e], o);
    }
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      mxp[w] = __vmaxu2(mxp[w], __shfl_xor_sync(0xffffffffu, mxp[w], o));
      mnp[w] = __vminu2(mnp[w], __shfl_xor_sync(0xffffffffu, mnp[w], o));
    }
  }
  if ((tid & 31) < GROUPS) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      red[warp * D + g * 8 + e] = part[e];
      redz[warp * D + g * 8 + e] = zp[e];
      const uint32_t emx = ((e & 1) ? (mxp[e >> 1] >> 16) : (mxp[e >> 1] & 0xFFFFu)) >> 7;
      const uint32_t emn = ((e & 1) ? (mnp[e >> 1] >> 16) : (mnp[e >> 1] & 0xFFFFu)) >> 7;
      rede[warp * D + g * 8 + e] = uint16_t((emx << 8) | emn);
    }
  }
  fence_async_shared();
  __syncthreads();
  if (tid < D) {
    double s = 0.0;
    float z = 0.f;
    uint32_t mx = 0u, mn = 255u;
    for (int q = 0; q < C::WARPS; ++q) {
      s += red[q * D + tid];
      z += redz[q * D + tid];
      const uint32_t w = rede[q * D + tid];
      mx = max(mx, w >> 8);
      mn = min(mn, w & 0xFFu);
    }
    const long long o = (bh * NB + j) * (long long)D + tid;
    ksum[o] = s;
    kbar[(bh * (long long)D + tid) * kbar_pitch(NB) + j] = s / (double)rows;
    kexp[2 * o] = (uint8_t)mx;
    kexp[2 * o + 1] = (uint8_t)mn;
    if (states) hstate[(bh * (long long)NB + j) * hpitch + D * D + tid] = __float2bfloat16_rn(z);
  }
  if (!states) return;

  // V' = V W_proj: A = V tile (K-major over channels), B = W_proj (MN-major)
  if (tid == 0) {
    bool ok = mbar_wait(&bars[0], 0, abort_flag);
    if (ok) {
      tc_fence_after();
      const uint32_t id0 = idesc_bf16(D, false, true);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t da = smem_desc(smem_u32(sV + (kk >> 2) * BLK * 128) + (kk & 3) * 32, 16, 1024, 2);
        const uint64_t db = smem_desc(smem_u32(sW) + kk * 2048, D * 128, 1024, 2);
        mma_bf16_ss(tmem, da, db, id0, kk > 0 ? 1u : 0u);
      }
    }
    tc_commit(&bars[1]);
  }
  __syncwarp();
  bool ok = mbar_wait(&bars[1], 0, abort_flag);
  tc_fence_after();
  // token row n of V' = TMEM lane (warps w and w + 4 share a lane quarter and
  // take half of the columns each): bf16 back over the V tile (same swizzled layout)
  const int lrow = (warp & 3) * 32 + (tid & 31);
  const int chalf = warp >> 2;
  {
    const uint32_t trow = tmem + (uint32_t((warp & 3) * 32) << 16);
#pragma unroll
    for (int cq = 0; cq < D / 32; ++cq) {
      const int ch = chalf * (D / 32) + cq;
      uint32_t v[16];
      SLA_TMEM_LD16(trow + ch * 16, v);
      tmem_ld_wait();
      if (lrow < BLK) {
        uint32_t pk[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) pk[e >> 1] = pack_bf16x2(__uint_as_float(v[e]), __uint_as_float(v[e + 1]));
        const int c0 = ch * 16, atom = c0 / 64;
        unsigned char* dst = sV + atom * BLK * 128;
        *reinterpret_cast<uint4*>(dst + sw128_offset(lrow, (c0 % 64) / 8)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *reinterpret_cast<uint4*>(dst + sw128_offset(lrow, (c0 % 64) / 8 + 1)) =
            make_uint4(pk[4], pk[5], pk[6], pk[7]);
      }
    }
  }
  fence_async_shared();
  tc_fence_before();
  __syncthreads();
  // h' = phi(K)^T V': A MN-major (a contiguous), B MN-major (channels contiguous)
  if (tid == 0) {
    if (ok) {
      tc_fence_after();
      const uint32_t id1 = idesc_bf16(D, true, true);
#pragma unroll
      for (int kk = 0; kk < BLK / 16; ++kk) {
        const uint64_t da = smem_desc(smem_u32(sP) + kk * 2048, BLK * 128, 1024, 2);
        const uint64_t db = smem_desc(smem_u32(sV) + kk * 2048, BLK * 128, 1024, 2);
        mma_bf16_ss(tmem, da, db, id1, kk > 0 ? 1u : 0u);
      }
    }
    tc_commit(&bars[2]);
  }
  __syncwarp();
  ok = mbar_wait(&bars[2], 0, abort_flag) && ok;
  tc_fence_after();
  {
    const uint32_t trow = tmem + (uint32_t((warp & 3) * 32) << 16);
    __nv_bfloat16* hs = hstate + (bh * (long long)NB + j) * hpitch + (long long)lrow * D;
#pragma unroll
    for (int cq = 0; cq < D / 32; ++cq) {
      const int ch = chalf * (D / 32) + cq;
      uint32_t v[16];
      SLA_TMEM_LD16(trow + ch * 16, v);
      tmem_ld_wait();
      if (ok && lrow < D) {
        uint32_t pk[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) pk[e >> 1] = pack_bf16x2(__uint_as_float(v[e]), __uint_as_float(v[e + 1]));
        uint4* d4 = reinterpret_cast<uint4*>(hs + ch * 16);
        d4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        d4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, D);
}

// mu[bh][c] = float32 nearest to (sum of the N values of K[bh][:][c]) / N.
// One CTA per (batch, head, group of CG channels).
//
// Fast path: thread (gi, c) sums every G-th float64 block sum of channel c,
// then the G partial sums are added in a fixed order.  The block sums are
// exact when every K value of the channel is a multiple of the smallest one's
// unit in the last place and the total stays below 2^53 of those units, so the
// order does not matter; kexp (largest and smallest exponent field per block)
// shows whether that holds.
// Exact path, for a channel where it does not: the CTA re-reads the channel's
// N values and sums them as 320-bit integers (exact_mean.cuh), then rounds the
// exact quotient once.  Either way mu is the correctly rounded exact mean.
constexpr int kMeanCG = 8;   // channels per CTA

template <int D>
__global__ void __launch_bounds__(1024) k_channel_mean(const double* __restrict__ ksum,
                                                      const uint8_t* __restrict__ kexp,
                                                      const __nv_bfloat16* __restrict__ K, float* __restrict__ mu,
                                                      int NB, int N) {
  constexpr int CG = kMeanCG;
  constexpr int G = 1024 / CG;
  __shared__ double rs[G][CG];
  __shared__ uint32_t re[G][CG];
  __shared__ int need_exact[CG];
  __shared__ Wide320 wpart[32][CG][2];   // per warp and channel: positive, negative part
  const long long bh = blockIdx.x;
  const int cc = threadIdx.x % CG, gi = threadIdx.x / CG;
  const int c = blockIdx.y * CG + cc;
  double s = 0.0;
  uint32_t mx = 0u, mn = 255u;
  for (int j = gi; j < NB; j += G) {
    const long long o = (bh * NB + j) * (long long)D + c;
    s += ksum[o];
    mx = max(mx, (uint32_t)kexp[2 * o]);
    mn = min(mn, (uint32_t)kexp[2 * o + 1]);
  }
  rs[gi][cc] = s;
  re[gi][cc] = (mx << 8) | mn;
  __syncthreads();
  if (gi == 0) {
    s = 0.0;
    mx = 0u;
    mn = 255u;
    for (int q = 0; q < G; ++q) {
      s += rs[q][cc];
      mx = max(mx, re[q][cc] >> 8);
      mn = min(mn, re[q][cc] & 0xFFu);
    }
    int lgN = 0;
    while ((1LL << lgN) < (long long)N) ++lgN;
    const bool wide = mx >= mn && int(mx) - int(mn) + 8 + lgN + 1 > 53;
    need_exact[cc] = wide ? 1 : 0;
    if (!wide) {
      // Correct rounding of s / N to float32: the float64 quotient q is within
      // half a float64 ulp of s/N, so it rounds to the same float32 unless q is
      // a float32 midpoint; then the sign of the exact remainder s - q*N decides.
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
      mu[bh * D + c] = f;
    }
  }
  __syncthreads();
  int any = 0;
#pragma unroll
  for (int q = 0; q < CG; ++q) any |= need_exact[q];
  if (!any) return;   // uniform

  // exact path: thread (gi, cc) takes rows gi, gi + G, ... of channel c
  Wide320 pos, neg;
  wide_zero(pos);
  wide_zero(neg);
  if (need_exact[cc]) {
    const uint16_t* kc = reinterpret_cast<const uint16_t*>(K) + bh * (long long)N * D + c;
    for (int n = gi; n < N; n += G) wide_add_bf16(pos, neg, __ldg(kc + (long long)n * D));
  }
  // lanes l, l ^ 8, l ^ 16, l ^ 24 hold the same channel
#pragma unroll
  for (int o = CG; o < 32; o <<= 1) {
    Wide320 a, b;
#pragma unroll
    for (int i = 0; i < kWideLimbs; ++i) {
      a.w[i] = __shfl_xor_sync(0xffffffffu, pos.w[i], o);
      b.w[i] = __shfl_xor_sync(0xffffffffu, neg.w[i], o);
    }
    wide_add(pos, a);
    wide_add(neg, b);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane < CG) {
    wpart[warp][lane][0] = pos;
    wpart[warp][lane][1] = neg;
  }
  __syncthreads();
  if (gi == 0 && need_exact[cc]) {
    wide_zero(pos);
    wide_zero(neg);
    for (int w = 0; w < 32; ++w) {
      wide_add(pos, wpart[w][cc][0]);
      wide_add(neg, wpart[w][cc][1]);
    }
    mu[bh * D + c] = wide_mean_to_f32(pos, neg, (uint32_t)N);
  }
}

}  // namespace sla
