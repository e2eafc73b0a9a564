// K3: pooled block scores and top-k block selection.
//
// "Turbo Diffusion：秒级生成与高清保真的视频扩散技术突破", section 三(二) SLA
// item 1 keeps the top-K (10%) most important regions; "TurboDiffusion技术指南",
// T2V parameter list, reads --sla_topk 0.1 as 10%.  Importance of key block j
// for query block i is the float64 score qbar_i . kbar_j / sqrt(D) of the
// mean-pooled raw blocks (valid rows only).  Softmax over j is monotonic, so
// the kc largest scores are the kc largest probabilities; equal scores go to
// the lower block index.  The kept indices are written in ascending order.
//
// One CTA handles R query blocks of one head (R = 8: a warp per row): it stages
// the pooled query blocks and, 32 at a time, the pooled key blocks in shared
// memory (each lane takes one key block and four independent partial dot
// products), writes the R x NB scores to shared memory, then each warp selects
// the top kc of its row by a bitwise search for the kc-th largest
// order-preserving key.
#pragma once
#include "sm100.cuh"

namespace sla {

__device__ __forceinline__ unsigned long long order_key(double v) {
  const unsigned long long u = (unsigned long long)__double_as_longlong(v);
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

template <int D>
__global__ void __launch_bounds__(256) k_mask(const double* __restrict__ qbar, const double* __restrict__ kbar,
                                             int NB, int kc, int rows_per_cta,
                                             int32_t* __restrict__ idx, uint8_t* __restrict__ bitmap,
                                             __nv_bfloat16* __restrict__ notcrit, int ncpitch) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const int R = rows_per_cta;
  double* qb = reinterpret_cast<double*>(smem_raw);   // [R][D]
  double* kbs = qb + R * D;                           // [32][D+1]
  double* sc = kbs + 32 * (D + 1);                    // [R][NB]

  const long long bh = blockIdx.y;
  const int i0 = blockIdx.x * R;
  const int nrows = min(R, NB - i0);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const double sqd = sqrt((double)D);

  for (int e = tid; e < R * D; e += 256) {
    const int r = e / D;
    qb[e] = (r < nrows) ? qbar[(bh * NB + i0) * (long long)D + e] : 0.0;
  }
  for (int j0 = 0; j0 < NB; j0 += 32) {
    __syncthreads();
    for (int e = tid; e < 32 * D; e += 256) {
      const int r = e / D, c = e % D;
      kbs[r * (D + 1) + c] = (j0 + r < NB) ? kbar[(bh * NB + j0 + r) * (long long)D + c] : 0.0;
    }
    __syncthreads();
    const int j = j0 + lane;
    for (int r = warp; r < nrows; r += 8) {
      double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
#pragma unroll 4
      for (int c = 0; c < D; c += 4) {
        a0 = fma(qb[r * D + c], kbs[lane * (D + 1) + c], a0);
        a1 = fma(qb[r * D + c + 1], kbs[lane * (D + 1) + c + 1], a1);
        a2 = fma(qb[r * D + c + 2], kbs[lane * (D + 1) + c + 2], a2);
        a3 = fma(qb[r * D + c + 3], kbs[lane * (D + 1) + c + 3], a3);
      }
      if (j < NB) sc[r * NB + j] = ((a0 + a1) + (a2 + a3)) / sqd;
    }
  }
  __syncthreads();

  for (int r = warp; r < nrows; r += 8) {
    const int i = i0 + r;
    const double* row = sc + r * NB;
    // kc-th largest key
    unsigned long long T = 0ull;
    for (int bit = 63; bit >= 0; --bit) {
      const unsigned long long cand = T | (1ull << bit);
      int cnt = 0;
      for (int j = lane; j < NB; j += 32) cnt += (order_key(row[j]) >= cand) ? 1 : 0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
      if (cnt >= kc) T = cand;
    }
    int gt = 0;
    for (int j = lane; j < NB; j += 32) gt += (order_key(row[j]) > T) ? 1 : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) gt += __shfl_xor_sync(0xffffffffu, gt, o);
    const int need_eq = kc - gt;
    int eq_seen = 0, out_pos = 0;
    int32_t* dst = idx + (bh * NB + i) * (long long)kc;
    for (int j0 = 0; j0 < NB; j0 += 32) {
      const int j = j0 + lane;
      const unsigned long long key = (j < NB) ? order_key(row[j]) : 0ull;
      const bool inb = j < NB;
      const bool eq = inb && key == T;
      const unsigned eqmask = __ballot_sync(0xffffffffu, eq);
      const int eq_before = eq_seen + __popc(eqmask & ((1u << lane) - 1u));
      const bool sel = inb && (key > T || (eq && eq_before < need_eq));
      const unsigned selmask = __ballot_sync(0xffffffffu, sel);
      if (sel) dst[out_pos + __popc(selmask & ((1u << lane) - 1u))] = j;
      if (bitmap != nullptr && inb) bitmap[(bh * NB + i) * (long long)NB + j] = sel ? 1 : 0;
      if (notcrit != nullptr && j < ncpitch)
        notcrit[(bh * NB + i) * (long long)ncpitch + j] = __float2bfloat16_rn((inb && !sel) ? 1.f : 0.f);
      eq_seen += __popc(eqmask);
      out_pos += __popc(selmask);
    }
    if (notcrit != nullptr) {
      const int jstart = ((NB + 31) / 32) * 32;
      for (int j = jstart + lane; j < ncpitch; j += 32)
        notcrit[(bh * NB + i) * (long long)ncpitch + j] = __float2bfloat16_rn(0.f);
    }
  }
}

template <int D>
size_t mask_smem(int rows, int NB) {
  return (size_t(rows) * D + 32 * (D + 1) + size_t(rows) * NB) * sizeof(double);
}

}  // namespace sla
