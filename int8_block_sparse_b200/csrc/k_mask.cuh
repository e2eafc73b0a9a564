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
// in shared memory).  Scores: for each group of 256 key blocks, thread t takes
// key block 256 * group + t and computes the R dot products of it with the R
// pooled query blocks (staged in shared memory, read as broadcasts), each as
// four interleaved partial sums over the channels (c mod 4) added as
// (a0 + a1) + (a2 + a3).  The pooled key blocks are stored channel-major
// (kbar[bh][c][j]); slabs of 16 channels x 256 key blocks come into a
// double-buffered shared ring by TMA, the next slab landing while the
// current one is used.  Selection: each warp turns its
// row into order-preserving 64-bit keys in place (their halves also held in
// registers when the row has at most 256 key blocks) and finds the kc-th
// largest by a bitwise search over the high 32 bits (warp reductions with
// redux.sync), then over the low 32 bits of the keys tied at that high half,
// if they are not all kept.
//
// Per-head counts and a third class (an extension: the pages name two
// classes): head h keeps kc_h blocks and may leave its kn_h lowest-ranked
// blocks out of the linear branch as well (ranking: larger score first, equal
// scores lower index first).  The blocks that are not negligible are then the
// top nblk - kn_h, found by the same search.  The linear indicator row
// (notcrit) marks the blocks of the linear class; the optional byte map holds
// 1 for kept blocks or, in class mode, the class (2 kept, 1 linear, 0 left out).
#pragma once
#include "sm100.cuh"

namespace sla {

__device__ __forceinline__ unsigned long long order_key(double v) {
  const unsigned long long u = (unsigned long long)__double_as_longlong(v);
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

// Number of the warp's keys (KPL per lane, or all NB from shared memory when
// KPL == 0; w32[2j] low, w32[2j + 1] high half of key j) whose high half is
// >= cand (tied: high half == th and low half >= cand).
template <int KPL>
__device__ __forceinline__ uint32_t count_ge(const uint32_t* hi_r, const uint32_t* lo_r, const uint32_t* w32,
                                             int NB, int lane, bool tied, uint32_t th, uint32_t cand) {
  uint32_t cnt = 0u;
  if (KPL > 0) {
#pragma unroll
    for (int e = 0; e < KPL; ++e) {
      const bool in = lane + 32 * e < NB;
      cnt += (in && (tied ? (hi_r[e] == th && lo_r[e] >= cand) : hi_r[e] >= cand)) ? 1u : 0u;
    }
  } else {
    for (int j = lane; j < NB; j += 32)
      cnt += (tied ? (w32[2 * j + 1] == th && w32[2 * j] >= cand) : w32[2 * j + 1] >= cand) ? 1u : 0u;
  }
  return __reduce_add_sync(0xffffffffu, cnt);
}

constexpr int kMaskSlabCh = 16;                               // channels per slab
constexpr int kMaskSlabBytes = kMaskSlabCh * 256 * 8;          // 32 KB
constexpr int kMaxHeadCounts = 512;

// Block counts per head, passed by value: head bh % H keeps kc[.] blocks and
// leaves kn[.] out; kcp is the pitch of the block lists (the largest kc).
struct HeadCounts {
  int H, kcp, classes;            // classes: the byte map holds classes, not 0/1
  uint16_t kc[kMaxHeadCounts];
  uint16_t kn[kMaxHeadCounts];
};

template <int D, int R>
__global__ void __launch_bounds__(256) k_mask(const __grid_constant__ CUtensorMap tm_kbar,
                                             const double* __restrict__ qbar, int NB,
                                             const __grid_constant__ HeadCounts hc, int* __restrict__ kc_bh,
                                             int32_t* __restrict__ idx, uint8_t* __restrict__ bitmap,
                                             __nv_bfloat16* __restrict__ notcrit, int ncpitch) {
  static_assert(R >= 1 && R <= 8, "one warp per row in the selection");
  static_assert(D % kMaskSlabCh == 0, "whole slabs");
  constexpr int SLABS = D / kMaskSlabCh;                      // slabs per group of key blocks
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  double* kbuf = reinterpret_cast<double*>(smem_raw);          // [2][16][256]
  double* qb = kbuf + 2 * kMaskSlabCh * 256;                   // [R][D]
  double* sc = qb + R * D;                                     // [R][NB] scores, then their order keys
  uint64_t* full = reinterpret_cast<uint64_t*>(sc + R * NB);   // [2]

  const long long bh = blockIdx.y;
  const int kc = hc.kc[bh % hc.H], kn = hc.kn[bh % hc.H];
  const int i0 = blockIdx.x * R;
  const int nrows = min(R, NB - i0);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const double sqd = sqrt((double)D);
  const int groups = (NB + 255) / 256;
  const int total = groups * SLABS;

  auto issue = [&](int n) {   // slab n: group n / SLABS, channels 16 * (n % SLABS) ..
    const int b = n & 1;
    mbar_expect_tx(&full[b], kMaskSlabBytes);
    tma_load_2d(kbuf + b * kMaskSlabCh * 256, &tm_kbar, &full[b], (n / SLABS) * 256,
                int(bh * D + (n % SLABS) * kMaskSlabCh));
  };
  int issued = 0;   // slabs requested (thread 0)
  if (kc_bh != nullptr && blockIdx.x == 0 && tid == 0) kc_bh[bh] = kc;
  if (tid == 0) {
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_kbar);
    issue(0);
    issued = 1;
    if (total > 1) issue(issued++);
  }
  for (int e = tid; e < R * D; e += 256) {
    const int r = e / D;
    qb[e] = (r < nrows) ? qbar[(bh * NB + i0) * (long long)D + e] : 0.0;
  }
  __syncthreads();
  double a[R][4];
  bool ok = true;
  for (int n = 0; n < total; ++n) {
    const int grp = n / SLABS, slab = n % SLABS;
    if (slab == 0) {
#pragma unroll
      for (int r = 0; r < R; ++r) a[r][0] = a[r][1] = a[r][2] = a[r][3] = 0.0;
    }
    ok = __syncthreads_and(mbar_wait(&full[n & 1], (n >> 1) & 1, nullptr)) && ok;
    const double* kb = kbuf + (n & 1) * kMaskSlabCh * 256;
    if (ok) {
#pragma unroll
      for (int cc = 0; cc < kMaskSlabCh; cc += 4) {
        const int c = slab * kMaskSlabCh + cc;
        const double k0 = kb[cc * 256 + tid], k1 = kb[(cc + 1) * 256 + tid];
        const double k2 = kb[(cc + 2) * 256 + tid], k3 = kb[(cc + 3) * 256 + tid];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const double2 q01 = *reinterpret_cast<const double2*>(qb + r * D + c);
          const double2 q23 = *reinterpret_cast<const double2*>(qb + r * D + c + 2);
          a[r][0] = fma(q01.x, k0, a[r][0]);
          a[r][1] = fma(q01.y, k1, a[r][1]);
          a[r][2] = fma(q23.x, k2, a[r][2]);
          a[r][3] = fma(q23.y, k3, a[r][3]);
        }
      }
    }
    const int j = grp * 256 + tid;
    if (slab == SLABS - 1 && j < NB) {
#pragma unroll
      for (int r = 0; r < R; ++r)
        if (r < nrows) sc[r * NB + j] = ((a[r][0] + a[r][1]) + (a[r][2] + a[r][3])) / sqd;
    }
    __syncthreads();   // the buffer of slab n is free again
    if (!ok) break;    // uniform: a slab did not land in time (recorded as a timeout)
    if (tid == 0 && n + 2 < total) issue(issued++);
  }
  if (!ok) {
    // slabs still in flight land before the CTA's shared memory is handed on
    if (tid == 0)
      for (int q = issued > 2 ? issued - 2 : 0; q < issued; ++q) (void)mbar_wait(&full[q & 1], (q >> 1) & 1, nullptr);
    return;
  }

  for (int r = warp; r < nrows; r += 8) {
    const int i = i0 + r;
    // scores -> order-preserving 64-bit keys, in place
    unsigned long long* rk = reinterpret_cast<unsigned long long*>(sc + r * NB);
    for (int j = lane; j < NB; j += 32) rk[j] = order_key(sc[r * NB + j]);
    __syncwarp();
    const uint32_t* w32 = reinterpret_cast<const uint32_t*>(rk);   // word 2j: low half, 2j+1: high half
    constexpr int KPL = 8;                       // register keys per lane when NB <= 256
    const bool regs = NB <= 32 * KPL;
    uint32_t hi_r[KPL], lo_r[KPL];
#pragma unroll
    for (int e = 0; e < KPL; ++e) {
      const int j = lane + 32 * e;
      hi_r[e] = (regs && j < NB) ? w32[2 * j + 1] : 0u;
      lo_r[e] = (regs && j < NB) ? w32[2 * j] : 0u;
    }
    // The k-th largest key T and how many keys equal to T rank before the
    // cut (need_eq): first the k-th largest high half Th by a bitwise search,
    // then, among the keys whose high half is Th, the (k - #above)-th largest
    // low half.
    auto kth = [&](int k, unsigned long long& T, int& need_eq) {
      uint32_t Th = 0u;
      for (int bit = 31; bit >= 0; --bit) {
        const uint32_t cand = Th | (1u << bit);
        const uint32_t cnt = regs ? count_ge<KPL>(hi_r, lo_r, w32, NB, lane, false, 0u, cand)
                                  : count_ge<0>(hi_r, lo_r, w32, NB, lane, false, 0u, cand);
        if (cnt >= (uint32_t)k) Th = cand;
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
      const uint32_t need = (uint32_t)k - above;   // >= 1: at least k high halves are >= Th
      uint32_t Tl = tied_min;                      // all tied keys are kept
      if (tied != need) {
        Tl = 0u;
        for (int bit = 31; bit >= 0; --bit) {
          const uint32_t cand = Tl | (1u << bit);
          const uint32_t cnt = regs ? count_ge<KPL>(hi_r, lo_r, w32, NB, lane, true, Th, cand)
                                    : count_ge<0>(hi_r, lo_r, w32, NB, lane, true, Th, cand);
          if (cnt >= need) Tl = cand;
        }
      }
      int gt = 0;
      T = ((unsigned long long)Th << 32) | Tl;
      for (int j = lane; j < NB; j += 32) gt += (rk[j] > T) ? 1 : 0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) gt += __shfl_xor_sync(0xffffffffu, gt, o);
      need_eq = k - gt;
    };
    unsigned long long Tc, Tn = 0ull;
    int need_c, need_n = 0;
    kth(kc, Tc, need_c);
    if (kn > 0) kth(NB - kn, Tn, need_n);   // the blocks ranked before NB - kn are not negligible
    int eqc_seen = 0, eqn_seen = 0, out_pos = 0;
    const unsigned lt = (1u << lane) - 1u;
    int32_t* dst = idx + (bh * NB + i) * (long long)hc.kcp;
    for (int j0 = 0; j0 < NB; j0 += 32) {
      const int j = j0 + lane;
      const bool inb = j < NB;
      const unsigned long long key = inb ? rk[j] : 0ull;
      const bool eqc = inb && key == Tc;
      const unsigned eqcmask = __ballot_sync(0xffffffffu, eqc);
      const bool sel = (inb && key > Tc) || (eqc && eqc_seen + __popc(eqcmask & lt) < need_c);
      bool keep = inb;                        // not negligible
      if (kn > 0) {
        const bool eqn = inb && key == Tn;
        const unsigned eqnmask = __ballot_sync(0xffffffffu, eqn);
        keep = (inb && key > Tn) || (eqn && eqn_seen + __popc(eqnmask & lt) < need_n);
        eqn_seen += __popc(eqnmask);
      }
      const unsigned selmask = __ballot_sync(0xffffffffu, sel);
      if (sel) dst[out_pos + __popc(selmask & lt)] = j;
      if (bitmap != nullptr && inb)
        bitmap[(bh * NB + i) * (long long)NB + j] = hc.classes ? (sel ? 2 : (keep ? 1 : 0)) : (sel ? 1 : 0);
      if (notcrit != nullptr && j < ncpitch)
        notcrit[(bh * NB + i) * (long long)ncpitch + j] = __float2bfloat16_rn((keep && !sel) ? 1.f : 0.f);
      eqc_seen += __popc(eqcmask);
      out_pos += __popc(selmask);
    }
    for (int t = kc + lane; t < hc.kcp; t += 32) dst[t] = -1;   // lists shorter than the pitch
    if (notcrit != nullptr) {
      const int jstart = ((NB + 31) / 32) * 32;
      for (int j = jstart + lane; j < ncpitch; j += 32)
        notcrit[(bh * NB + i) * (long long)ncpitch + j] = __float2bfloat16_rn(0.f);
    }
  }
}

template <int D>
size_t mask_smem(int rows, int NB) {
  return size_t(2) * kMaskSlabBytes + (size_t(rows) * D + size_t(rows) * NB) * sizeof(double) + 2 * 8;
}

}  // namespace sla
