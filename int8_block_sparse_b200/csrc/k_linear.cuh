// K5: the linear-attention branch for the key blocks that were not selected.
//
// "Turbo Diffusion：秒级生成与高清保真的视频扩散技术突破", section 三(二) SLA
// item 2: the rest of the attention goes through an O(N) linear branch with a
// linear projection.  With per-key-block states h_j = sum phi(k) v^T and
// z_j = sum phi(k) (phi = elu + 1), query block i needs the sums over the key
// blocks it did NOT select:
//     G_i = sum_{j not in crit(i)} h_j,   g_i = sum_{j not in crit(i)} z_j.
// For all i at once that is a GEMM with the 0/1 "not selected" matrix:
//     [G | g] (NB x (D*D + D)) = notcrit (NB x NB) . [h | z] (NB x (D*D + D))
// (k_lingemm, tcgen05 bf16 with float32 accumulation; summing the
// non-selected blocks directly avoids the cancellation of total minus
// selected).  The states arrive with W_proj folded in (h'_j = h_j W_proj, see
// k_stats.cuh), so per query row n of block i
//     out_n = O_sparse,n + phi(q_n) G'_i / (phi(q_n) . g_i),   G'_i = G_i W_proj,
// one tensor-core product per query block, done inside k_attn (k_attn.cuh).
#pragma once
#include <cuda_bf16.h>
#include "sm100.cuh"

namespace sla {

// ------------------------------------------------------------------ k_lingemm
// Persistent, warp-specialised: a work unit is (head bh, group of 256 query
// blocks = two 128-row M tiles, a run of consecutive 128-entry N tiles);
// units u = blockIdx.x, +gridDim.x, ...  With RESIDENT (at most 256 key
// blocks: the unit's A tiles fit in shared memory) the unit's A tiles (the
// 0/1 matrix rows of its 256 query blocks) are loaded once and kept for all
// of its N tiles, and only the state tiles stream through the ring; otherwise
// every k-step brings its A and B tiles (one N tile per unit).  K = key blocks
// in steps of 64; the two accumulator sets (2 x 2 x 128 columns of TMEM)
// alternate between N tiles so that one tile's epilogue overlaps the next
// tile's products.
//   warp 0  TMA producer     warp 1  tcgen05.mma issuer
//   warps 2-9  epilogue (TMEM lane quarter = warp % 4; warps 2-5 the first 64
//              columns of an N tile, warps 6-9 the other 64)
struct LinGemmParams {
  __nv_bfloat16* grest;   // [BH][NB][D*D]
  float* zrest;           // [BH][NB][D]
  int NB, D, E;           // E = D*D + D
  int nkt;                // number of 64-wide K steps
  int mgroups, ntiles, units;
  int tpu;                // N tiles per unit
};

constexpr int LG_STAGES = 4;
constexpr int LG_A_BYTES = 128 * 64 * 2;                 // one M tile x 64 key blocks: 16 KB
constexpr int LG_B_BYTES = 64 * 128 * 2;                 // 64 key blocks x 128 entries: 16 KB
constexpr int LG_MAX_RESIDENT_KT = 4;                    // A kept in shared memory up to 256 key blocks
constexpr int LG_BAR_BYTES = (2 * LG_STAGES + 4 + 2) * 8 + 16;
template <bool RESIDENT>
struct LinGemmCfg {
  // ring stage: A (both M tiles) + B, or B alone when A is resident
  static constexpr int STAGE_BYTES = RESIDENT ? LG_B_BYTES : 2 * LG_A_BYTES + LG_B_BYTES;
  static constexpr int A_REGION = RESIDENT ? LG_MAX_RESIDENT_KT * 2 * LG_A_BYTES : 0;
  static constexpr int SMEM_USED = A_REGION + LG_STAGES * STAGE_BYTES + LG_BAR_BYTES;
  static constexpr int SMEM = SMEM_USED + 1024;
};
constexpr int LG_THREADS = 320;

template <bool RESIDENT>
__global__ void __launch_bounds__(LG_THREADS, 1) k_lingemm(const __grid_constant__ CUtensorMap tm_a,
                                                           const __grid_constant__ CUtensorMap tm_b,
                                                           const LinGemmParams p) {
  using C = LinGemmCfg<RESIDENT>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if (uint32_t(base - smem_raw) + C::SMEM_USED > dynamic_smem_bytes()) {
    if (threadIdx.x == 0) raise_error(DEV_ERR_LAYOUT);
    return;   // uniform: every thread sees the same base
  }
  unsigned char* aregion = base;                              // RESIDENT: [nkt][2 M tiles] A tiles
  unsigned char* ring = base + C::A_REGION;
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + LG_STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + LG_STAGES;
  uint64_t* acc_full = empty + LG_STAGES;    // [2] products of an N tile done
  uint64_t* acc_empty = acc_full + 2;        // [2] epilogue has read the accumulators
  uint64_t* a_full = acc_empty + 2;          // RESIDENT: the unit's A tiles have landed
  uint64_t* a_empty = a_full + 1;            // RESIDENT: the unit's products are done with them
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(a_empty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  auto stage = [&](int s) { return ring + s * C::STAGE_BYTES; };
  auto a_tile = [&](int kt, int mt) -> unsigned char* {
    return RESIDENT ? aregion + (kt * 2 + mt) * LG_A_BYTES : nullptr;
  };

  if (tid == 0) {
    for (int q = 0; q < LG_STAGES; ++q) {
      mbar_init(&full[q], 1);
      mbar_init(&empty[q], 1);
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(&acc_full[q], 1);
      mbar_init(&acc_empty[q], 256);
    }
    mbar_init(a_full, 1);
    mbar_init(a_empty, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // unit u: head bh, M group m0 (first query block), N tiles [t0, t1)
  auto unit_coords = [&](int u, int& bh, int& m0, int& t0, int& t1) {
    const int nchunks = (p.ntiles + p.tpu - 1) / p.tpu;
    t0 = (u % nchunks) * p.tpu;
    t1 = min(p.ntiles, t0 + p.tpu);
    m0 = ((u / nchunks) % p.mgroups) * 256;
    bh = u / (nchunks * p.mgroups);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_a);
      tma_prefetch_desc(&tm_b);
      uint32_t n = 0, un = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x, ++un) {
        int bh, m0, t0, t1;
        unit_coords(u, bh, m0, t0, t1);
        if (RESIDENT) {
          // the previous unit's products are done with the A region
          if (!(ok = mbar_wait(a_empty, (un & 1) ^ 1, abort_flag))) break;
          mbar_expect_tx(a_full, p.nkt * 2 * LG_A_BYTES);
          for (int kt = 0; kt < p.nkt; ++kt) {
            tma_load_3d(a_tile(kt, 0), &tm_a, a_full, kt * 64, m0, bh);
            tma_load_3d(a_tile(kt, 1), &tm_a, a_full, kt * 64, m0 + 128, bh);
          }
        }
        for (int tn = t0; tn < t1 && ok; ++tn) {
          const int n0 = tn * 128;
          for (int kt = 0; kt < p.nkt; ++kt, ++n) {
            const int s = n % LG_STAGES;
            if (!(ok = mbar_wait(&empty[s], ((n / LG_STAGES) & 1) ^ 1, abort_flag))) break;
            unsigned char* st = stage(s);
            mbar_expect_tx(&full[s], C::STAGE_BYTES);
            unsigned char* bdst = st;
            if (!RESIDENT) {
              tma_load_3d(st, &tm_a, &full[s], kt * 64, m0, bh);
              tma_load_3d(st + LG_A_BYTES, &tm_a, &full[s], kt * 64, m0 + 128, bh);
              bdst = st + 2 * LG_A_BYTES;
            }
#pragma unroll
            for (int q = 0; q < 2; ++q)
              tma_load_3d(bdst + q * 8192, &tm_b, &full[s], n0 + q * 64, kt * 64, bh);
          }
        }
      }
      // loads still in flight (only after a failed wait) land before the CTA exits
      for (uint32_t q = n > LG_STAGES ? n - LG_STAGES : 0; q < n; ++q)
        (void)mbar_wait(&full[q % LG_STAGES], (q / LG_STAGES) & 1, nullptr);
      if (RESIDENT && un > 0) (void)mbar_wait(a_full, (un - 1) & 1, nullptr);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, false, true);
      uint32_t n = 0, it = 0, un = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x, ++un) {
        int bh, m0, t0, t1;
        unit_coords(u, bh, m0, t0, t1);
        if (RESIDENT && !(ok = mbar_wait(a_full, un & 1, abort_flag))) break;
        for (int tn = t0; tn < t1 && ok; ++tn, ++it) {
          const int a = it & 1;   // accumulator set
          if (!(ok = mbar_wait(&acc_empty[a], ((it >> 1) & 1) ^ 1, abort_flag))) break;
          tc_fence_after();
          const uint32_t d0 = tmem + a * 256, d1 = d0 + 128;   // M tile 0, M tile 1
          for (int kt = 0; kt < p.nkt; ++kt, ++n) {
            const int s = n % LG_STAGES;
            if (!(ok = mbar_wait(&full[s], (n / LG_STAGES) & 1, abort_flag))) break;
            tc_fence_after();
            unsigned char* st = stage(s);
            unsigned char* a0 = RESIDENT ? a_tile(kt, 0) : st;
            unsigned char* a1 = RESIDENT ? a_tile(kt, 1) : st + LG_A_BYTES;
            unsigned char* bsrc = RESIDENT ? st : st + 2 * LG_A_BYTES;
            const uint64_t da0 = smem_desc(smem_u32(a0), 16, 1024, 2);
            const uint64_t da1 = smem_desc(smem_u32(a1), 16, 1024, 2);
            const uint64_t db = smem_desc(smem_u32(bsrc), 8192, 1024, 2);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t acc = (kt > 0 || kk > 0) ? 1u : 0u;
              mma_bf16_ss(d0, da0 + uint64_t(kk * 2), db + uint64_t(kk * (2048 >> 4)), idesc, acc);
              mma_bf16_ss(d1, da1 + uint64_t(kk * 2), db + uint64_t(kk * (2048 >> 4)), idesc, acc);
            }
            tc_commit(&empty[s]);
          }
          tc_commit(&acc_full[a]);
        }
        if (RESIDENT) tc_commit(a_empty);   // the unit's products are done with its A tiles
      }
      // every MMA issued here finishes before the CTA frees TMEM (bounded)
      tc_commit(&acc_full[(it & 1)]);
      (void)mbar_wait(&acc_full[(it & 1)], (it >> 1) & 1, nullptr);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int r = (warp & 3) * 32 + lane;          // accumulator row = TMEM lane
    const int ch = (warp - 2) >> 2;                // column half of the N tile
    const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
    const int DD = p.D * p.D;
    uint32_t it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
      int bh, m0, t0, t1;
      unit_coords(u, bh, m0, t0, t1);
      for (int tn = t0; tn < t1 && ok; ++tn, ++it) {
        const int a = it & 1;
        const int n0 = tn * 128;
        if (!(ok = mbar_wait(&acc_full[a], (it >> 1) & 1, abort_flag))) break;
        tc_fence_after();
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          const int row = m0 + mt * 128 + r;
          const uint32_t taddr = tmem + a * 256 + mt * 128 + lane_off;
          {
            const int c4 = ch;
            uint32_t v[4][16];
#pragma unroll
            for (int q = 0; q < 4; ++q) SLA_TMEM_LD16(taddr + (c4 * 4 + q) * 16, v[q]);   // warp-collective
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int e0 = n0 + (c4 * 4 + q) * 16;
              if (row < p.NB && e0 < p.E) {
                if (e0 < DD) {
                  uint32_t pk[8];
#pragma unroll
                  for (int e = 0; e < 16; e += 2)
                    pk[e >> 1] = pack_bf16x2(__uint_as_float(v[q][e]), __uint_as_float(v[q][e + 1]));
                  uint4* dst = reinterpret_cast<uint4*>(p.grest + ((long long)bh * p.NB + row) * DD + e0);
                  dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                  dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                } else {
                  float* dst = p.zrest + ((long long)bh * p.NB + row) * p.D + (e0 - DD);
#pragma unroll
                  for (int e = 0; e < 16; ++e) dst[e] = __uint_as_float(v[q][e]);
                }
              }
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&acc_empty[a]);
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace sla
