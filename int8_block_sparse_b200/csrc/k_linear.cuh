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
// k_stats.cuh), so per query row n of block i (k_linout)
//     out_n = O_sparse,n + phi(q_n) G'_i / (phi(q_n) . g_i),   G'_i = G_i W_proj,
// one tensor-core product per query block.
#pragma once
#include <cuda_bf16.h>
#include "sm100.cuh"
#include "k_stats.cuh"

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

// ------------------------------------------------------------------ k_linout
struct LinOutParams {
  const __nv_bfloat16* q;      // [BH][N][D]
  const float* zrest;          // [BH][NB][D]
  int N, NB, BLK;
};

template <int D>
struct LinOutCfg {
  static constexpr int A_BYTES = 128 * D * 2;   // phi(Q) tile (K-major, 64-column atoms of 16 KB)
  static constexpr int G_BYTES = D * D * 2;     // G'_i (MN-major)
  // after the product, A and G are reused for the 128 x D float32 result y,
  // as D/32 column chunks of 32 floats (128-byte rows, 128-byte swizzle)
  static constexpr int Y_BYTES = 128 * D * 4;
  static constexpr int AG_BYTES = (A_BYTES + G_BYTES > Y_BYTES) ? A_BYTES + G_BYTES : Y_BYTES;
  static constexpr int SMEM = AG_BYTES + 1024 + 128 + D * 4;
};

// One CTA (128 threads, thread = query row) per query block.  out holds
// O_sparse on entry; y = phi(q) G' / den is staged in shared memory and added
// to out by TMA reductions (float32 add in L2, one add per element).
template <int D>
__global__ void __launch_bounds__(128) k_linout(const __grid_constant__ CUtensorMap tm_q,
                                               const __grid_constant__ CUtensorMap tm_g,
                                               const __grid_constant__ CUtensorMap tm_out, const LinOutParams p) {
  using C = LinOutCfg<D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sa = base;
  unsigned char* sg = sa + C::A_BYTES;
  float* sz = reinterpret_cast<float*>(sa + C::AG_BYTES);          // z_rest of this query block
  uint64_t* bars = reinterpret_cast<uint64_t*>(sz + D);            // 0: G load, 1: MMA
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int i = blockIdx.x;
  const int bh = blockIdx.y;

  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, D);
    tmem_relinquish();
  }
  if (tid < D) sz[tid] = p.zrest[((long long)bh * p.NB + i) * D + tid];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (tid == 0) {
    // the query tile lands in the A operand's own layout (K-major, 128-byte
    // swizzle, 64-column atoms of 16 KB); rows past N arrive as zeros
    mbar_expect_tx(&bars[0], C::G_BYTES + C::A_BYTES);
#pragma unroll
    for (int hh = 0; hh < D / 64; ++hh) {
      tma_load_2d(sg + hh * D * 128, &tm_g, &bars[0], hh * 64, int(((long long)bh * p.NB + i) * D));
      tma_load_3d(sa + hh * 16384, &tm_q, &bars[0], hh * 64, i * p.BLK, bh);
    }
  }

  const int r = tid;
  const long long n = (long long)i * p.BLK + r;
  const bool valid = r < p.BLK && n < p.N;
  const bool landed = __syncthreads_and(mbar_wait(&bars[0], 0, abort_flag));
  // phi(q) in place: each thread rewrites its own row of the A tile
  float den = 0.f;
  {
#pragma unroll
    for (int c8 = 0; c8 < D / 8; ++c8) {
      const int atom = c8 >> 3, chunk = c8 & 7;
      uint4* slot = reinterpret_cast<uint4*>(sa + atom * 16384 + sw128_offset(r, chunk));
      const uint4 raw = *slot;
      const uint16_t* hv = reinterpret_cast<const uint16_t*>(&raw);
      uint32_t pk[4];
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        const float f0 = valid ? phi_elu1(__uint_as_float(uint32_t(hv[e]) << 16)) : 0.f;
        const float f1 = valid ? phi_elu1(__uint_as_float(uint32_t(hv[e + 1]) << 16)) : 0.f;
        den = fmaf(f0, sz[c8 * 8 + e], den);
        den = fmaf(f1, sz[c8 * 8 + e + 1], den);
        pk[e >> 1] = pack_bf16x2(f0, f1);
      }
      *slot = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
  }
  fence_async_shared();
  __syncthreads();
  if (tid == 0) {
    if (landed) {
      tc_fence_after();
      const uint32_t idesc = idesc_bf16(D, false, true);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t da = smem_desc(smem_u32(sa + (kk >> 2) * 16384) + (kk & 3) * 32, 16, 1024, 2);
        const uint64_t db = smem_desc(smem_u32(sg) + kk * 2048, D * 128, 1024, 2);
        mma_bf16_ss(tmem, da, db, idesc, kk > 0 ? 1u : 0u);
      }
    }
    tc_commit(&bars[1]);
  }
  __syncwarp();
  const bool ok = __syncthreads_and(mbar_wait(&bars[1], 0, abort_flag));
  tc_fence_after();
  // y row r = phi(q_r) G' / den_r -> shared memory over A and G (the product
  // is complete): chunk c holds columns [32c, 32c + 32) as 128-byte rows
  const uint32_t trow = tmem + (uint32_t(warp * 32) << 16);
  const float inv_den = (valid && den > 0.f) ? 1.f / den : 0.f;
#pragma unroll
  for (int ch = 0; ch < D / 16; ++ch) {
    uint32_t v[16];
    SLA_TMEM_LD16(trow + ch * 16, v);
    tmem_ld_wait();
    unsigned char* chunk = base + (ch >> 1) * 16384;
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4)
      *reinterpret_cast<float4*>(chunk + sw128_offset(r, (ch & 1) * 4 + q4)) =
          make_float4(__uint_as_float(v[4 * q4]) * inv_den, __uint_as_float(v[4 * q4 + 1]) * inv_den,
                      __uint_as_float(v[4 * q4 + 2]) * inv_den, __uint_as_float(v[4 * q4 + 3]) * inv_den);
  }
  fence_async_shared();
  tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    if (ok) {
      // rows past N are dropped by the TMA; the box is BLK rows high
#pragma unroll
      for (int c = 0; c < D / 32; ++c) tma_reduce_add_3d(&tm_out, base + c * 16384, c * 32, i * p.BLK, bh);
      bulk_commit_group();
    }
    bulk_wait_group_read0();
  }
  tc_fence_after();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, D);
}

}  // namespace sla
