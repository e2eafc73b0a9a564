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
// One CTA handles R query blocks of one head (R <= 8: a warp per row in the
// selection; R = 8 unless the scores of a long sequence need a smaller R to fit
// in shared memory).  Scores: thread t takes key blocks t, t + 256, ... and computes
// the R dot products of its key block with the R pooled query blocks (staged
// in shared memory, read as broadcasts), each as four interleaved partial sums
// over the channels (c mod 4) added as (a0 + a1) + (a2 + a3); its pooled key
// block is read once, straight from global memory.  Selection: each warp turns
// its row into order-preserving 64-bit keys and finds the kc-th largest by a
// bitwise search over the high 32 bits (warp reductions with redux.sync), then
// over the low 32 bits of the keys tied at that high half, if they are not all
// kept.
#pragma once
#include "sm100.cuh"

namespace sla {

__device__ __forceinline__ unsigned long long order_key(double v) {
  const unsigned long long u = (unsigned long long)__double_as_longlong(v);
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

template <int D, int R>
__global__ void __launch_bounds__(256) k_mask(const double* __restrict__ qbar, const double* __restrict__ kbar,
                                             int NB, int kc, int32_t* __restrict__ idx, uint8_t* __restrict__ bitmap,
                                             __nv_bfloat16* __restrict__ notcrit, int ncpitch) {
  static_assert(R >= 1 && R <= 8, "one warp per row in the selection");
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  double* qb = reinterpret_cast<double*>(smem_raw);   // [R][D]
  double* sc = qb + R * D;                            // [R][NB]

  const long long bh = blockIdx.y;
  const int i0 = blockIdx.x * R;
  const int nrows = min(R, NB - i0);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const double sqd = sqrt((double)D);

  for (int e = tid; e < R * D; e += 256) {
    const int r = e / D;
    qb[e] = (r < nrows) ? qbar[(bh * NB + i0) * (long long)D + e] : 0.0;
  }
  __syncthreads();
  for (int j = tid; j < NB; j += 256) {
    const double2* kr = reinterpret_cast<const double2*>(kbar + (bh * NB + j) * (long long)D);
    double a[R][4];
#pragma unroll
    for (int r = 0; r < R; ++r) a[r][0] = a[r][1] = a[r][2] = a[r][3] = 0.0;
#pragma unroll 2
    for (int c = 0; c < D; c += 4) {
      const double2 k01 = __ldg(kr + c / 2), k23 = __ldg(kr + c / 2 + 1);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const double2 q01 = *reinterpret_cast<const double2*>(qb + r * D + c);
        const double2 q23 = *reinterpret_cast<const double2*>(qb + r * D + c + 2);
        a[r][0] = fma(q01.x, k01.x, a[r][0]);
        a[r][1] = fma(q01.y, k01.y, a[r][1]);
        a[r][2] = fma(q23.x, k23.x, a[r][2]);
        a[r][3] = fma(q23.y, k23.y, a[r][3]);
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
      if (r < nrows) sc[r * NB + j] = ((a[r][0] + a[r][1]) + (a[r][2] + a[r][3])) / sqd;
  }
  __syncthreads();

  for (int r = warp; r < nrows; r += 8) {
    const int i = i0 + r;
    // scores -> order-preserving 64-bit keys, in place
    unsigned long long* rk = reinterpret_cast<unsigned long long*>(sc + r * NB);
    for (int j = lane; j < NB; j += 32) rk[j] = order_key(sc[r * NB + j]);
    __syncwarp();
    const uint32_t* w32 = reinterpret_cast<const uint32_t*>(rk);   // word 2j: low half, 2j+1: high half
    // T = the kc-th largest key: first the kc-th largest high half Th, then,
    // among the keys whose high half is Th, the (kc - #above)-th largest low half
    uint32_t Th = 0u;
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = Th | (1u << bit);
      uint32_t cnt = 0u;
      for (int j = lane; j < NB; j += 32) cnt += (w32[2 * j + 1] >= cand) ? 1u : 0u;
      if (__reduce_add_sync(0xffffffffu, cnt) >= (uint32_t)kc) Th = cand;
    }
    uint32_t above = 0u, tied = 0u, tied_min = 0xFFFFFFFFu;
    for (int j = lane; j < NB; j += 32) {
      const uint32_t h = w32[2 * j + 1];
      above += (h > Th) ? 1u : 0u;
      if (h == Th) {
        ++tied;
        tied_min = min(tied_min, w32[2 * j]);
      }
    }
    above = __reduce_add_sync(0xffffffffu, above);
    tied = __reduce_add_sync(0xffffffffu, tied);
    tied_min = __reduce_min_sync(0xffffffffu, tied_min);
    const uint32_t need = (uint32_t)kc - above;   // >= 1: at least kc high halves are >= Th
    uint32_t Tl = tied_min;                       // all tied keys are kept
    if (tied != need) {
      Tl = 0u;
      for (int bit = 31; bit >= 0; --bit) {
        const uint32_t cand = Tl | (1u << bit);
        uint32_t cnt = 0u;
        for (int j = lane; j < NB; j += 32) cnt += (w32[2 * j + 1] == Th && w32[2 * j] >= cand) ? 1u : 0u;
        if (__reduce_add_sync(0xffffffffu, cnt) >= need) Tl = cand;
      }
    }
    const unsigned long long T = ((unsigned long long)Th << 32) | Tl;
    int gt = 0;
    for (int j = lane; j < NB; j += 32) gt += (rk[j] > T) ? 1 : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) gt += __shfl_xor_sync(0xffffffffu, gt, o);
    const int need_eq = kc - gt;
    int eq_seen = 0, out_pos = 0;
    int32_t* dst = idx + (bh * NB + i) * (long long)kc;
    for (int j0 = 0; j0 < NB; j0 += 32) {
      const int j = j0 + lane;
      const unsigned long long key = (j < NB) ? rk[j] : 0ull;
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
  return (size_t(rows) * D + size_t(rows) * NB) * sizeof(double);
}

}  // namespace sla
