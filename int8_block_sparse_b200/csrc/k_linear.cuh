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
// Tile 128 (query blocks) x 256 (state entries), K = key blocks in steps of 64.
struct LinGemmParams {
  __nv_bfloat16* grest;   // [BH][NB][D*D]
  float* zrest;           // [BH][NB][D]
  int NB, D, E;           // E = D*D + D
  int nkt;                // number of 64-wide K steps
};

constexpr int LG_STAGES = 2;   // two CTAs per SM: one drains its epilogue while the other loads
constexpr int LG_A_BYTES = 128 * 64 * 2;   // 16 KB
constexpr int LG_B_BYTES = 64 * 256 * 2;   // 32 KB
constexpr int LG_SMEM = LG_STAGES * (LG_A_BYTES + LG_B_BYTES) + 1024 + 256;

__global__ void __launch_bounds__(128, 2) k_lingemm(const __grid_constant__ CUtensorMap tm_a,
                                                    const __grid_constant__ CUtensorMap tm_b,
                                                    const LinGemmParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(base + LG_STAGES * (LG_A_BYTES + LG_B_BYTES));
  uint64_t* empty = full + LG_STAGES;
  uint64_t* done = empty + LG_STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.x * 256;   // state entry
  const int m0 = blockIdx.y * 128;   // query block
  const int bh = blockIdx.z;

  if (tid == 0) {
    for (int s = 0; s < LG_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    for (int kt = 0; kt < p.nkt; ++kt) {
      const int s = kt % LG_STAGES;
      if (!mbar_wait(&empty[s], ((kt / LG_STAGES) & 1) ^ 1, abort_flag)) break;
      unsigned char* sa = base + s * (LG_A_BYTES + LG_B_BYTES);
      unsigned char* sb = sa + LG_A_BYTES;
      mbar_expect_tx(&full[s], LG_A_BYTES + LG_B_BYTES);
      tma_load_3d(sa, &tm_a, &full[s], kt * 64, m0, bh);
#pragma unroll
      for (int q = 0; q < 4; ++q) tma_load_3d(sb + q * 8192, &tm_b, &full[s], n0 + q * 64, kt * 64, bh);
    }
  } else if (warp == 1 && lane == 0) {
    const uint32_t idesc = idesc_bf16(256, false, true);
    for (int kt = 0; kt < p.nkt; ++kt) {
      const int s = kt % LG_STAGES;
      if (!mbar_wait(&full[s], (kt / LG_STAGES) & 1, abort_flag)) break;
      tc_fence_after();
      unsigned char* sa = base + s * (LG_A_BYTES + LG_B_BYTES);
      unsigned char* sb = sa + LG_A_BYTES;
      const uint64_t da = smem_desc(smem_u32(sa), 16, 1024, 2);
      const uint64_t db = smem_desc(smem_u32(sb), 8192, 1024, 2);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16_ss(tmem, da + uint64_t(kk * 2), db + uint64_t(kk * (2048 >> 4)), idesc,
                    (kt > 0 || kk > 0) ? 1u : 0u);
      tc_commit(&empty[s]);
    }
    tc_commit(done);
  }
  __syncwarp();
  // epilogue: thread = query block row of the tile
  const bool ok = mbar_wait(done, 0, abort_flag);
  tc_fence_after();
  const int row = m0 + tid;
  const uint32_t taddr = tmem + (uint32_t(warp * 32) << 16);
  const int DD = p.D * p.D;
  // four 16-column TMEM loads in flight per wait (the loads, not the stores,
  // are what the epilogue waits on)
  for (int c4 = 0; c4 < 4; ++c4) {
    uint32_t v[4][16];
#pragma unroll
    for (int q = 0; q < 4; ++q) SLA_TMEM_LD16(taddr + (c4 * 4 + q) * 16, v[q]);   // warp-collective
    tmem_ld_wait();
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e0 = n0 + (c4 * 4 + q) * 16;
      if (ok && row < p.NB && e0 < p.E) {
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

}  // namespace sla
