// K4: critical-block attention on the 5th-generation tensor cores.
//
// "Turbo Diffusion：秒级生成与高清保真的视频扩散技术突破", section 三(一) item 3
// (attention re-tiled to 128x128 tensor-core tiles with a parallel softmax) and
// section 三(二) item 3 (SageSLA: after the block selection, INT8 computation
// on the selected blocks).  For query block i of head (b, h) and each selected
// key block j (ascending):
//     S = int32(Qi8_i . Ki8_j^T) * sq_i * sk_j / sqrt(D)   (tcgen05 kind::i8)
//     online softmax in float32 (exp2 domain), P rounded to bf16
//     O += P . V_j                                        (tcgen05 kind::f16)
// and finally O_sparse = O / l, l being the sum of the unrounded P.
//
// One persistent CTA per SM runs two independent pipelines ("tiles"), each
// working on its own sequence of (head, query block) items:
//   warp 0 / 2   TMA producer of tile 0 / 1 (Q once per item, K/V ring of 2)
//   warp 1 / 3   tcgen05.mma issuer of tile 0 / 1
//   warps 4-7    softmax + epilogue of tile 0 (thread = query row = TMEM lane)
//   warps 8-11   softmax + epilogue of tile 1
// TMEM (512 columns): tile u uses columns [256u, 256u+128) for S (P, bf16,
// is written over the first half of S) and [256u+128, 256u+128+D) for O.
#pragma once
#include <cuda_bf16.h>
#include "sm100.cuh"

namespace sla {

struct AttnParams {
  const int32_t* idx;   // [BH][NB][kc]
  const float* sq;      // [BH][NB]
  const float* sk;      // [BH][NB]
  float* o;             // [BH][N][D] float32: O_sparse
  int N, NB, NP, kc, items;
  float qk_scale;       // log2(e) / sqrt(D)
};

template <int D, int BLK>
struct AttnCfg {
  static constexpr int BQ = 128;                 // query rows per tile (MMA M)
  static constexpr int Q_BYTES = BQ * D;         // int8
  static constexpr int K_BYTES = BLK * D;        // int8
  static constexpr int V_BYTES = BLK * D * 2;    // bf16
  static constexpr int STAGES = 2;
  static constexpr int TILE_BYTES = Q_BYTES + STAGES * (K_BYTES + V_BYTES);
  // at least 120 KB, so that one CTA (holding all 512 TMEM columns) fills an SM
  static constexpr int SMEM_USED = 2 * TILE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
  static constexpr int SMEM = SMEM_USED > 122880 ? SMEM_USED : 122880;
  static constexpr uint32_t KSW = (D == 128) ? 2u : 4u;     // Q/K swizzle: 128B or 64B rows
  static constexpr uint32_t KSBO = (D == 128) ? 1024u : 512u;
};

struct TileBars {
  uint64_t q_full, q_empty, s_full, p_full, o_full, o_free;
  uint64_t kv_full[2], kv_empty[2];
};

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int D, int BLK>
__global__ void __launch_bounds__(384, 1) k_attn(const __grid_constant__ CUtensorMap tm_q,
                                                 const __grid_constant__ CUtensorMap tm_k,
                                                 const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  using C = AttnCfg<D, BLK>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  TileBars* bars = reinterpret_cast<TileBars*>(base + 2 * C::TILE_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int u = 0; u < 2; ++u) {
      TileBars& b = bars[u];
      mbar_init(&b.q_full, 1);
      mbar_init(&b.q_empty, 1);
      mbar_init(&b.s_full, 1);
      mbar_init(&b.p_full, 128);
      mbar_init(&b.o_full, 1);
      mbar_init(&b.o_free, 128);
      for (int s = 0; s < 2; ++s) {
        mbar_init(&b.kv_full[s], 1);
        mbar_init(&b.kv_empty[s], 1);
      }
    }
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
  const uint32_t tmem_base = *tmem_slot;

  const int kc = p.kc;
  const int NB = p.NB;
  const int tiles_total = 2 * gridDim.x;

  if (warp < 4) {
    const int u = warp >> 1;
    TileBars& b = bars[u];
    unsigned char* tq = base + u * C::TILE_BYTES;
    unsigned char* tk[2] = {tq + C::Q_BYTES, tq + C::Q_BYTES + C::K_BYTES + C::V_BYTES};
    unsigned char* tv[2] = {tk[0] + C::K_BYTES, tk[1] + C::K_BYTES};
    if ((warp & 1) == 0) {
      // ------------------------------------------------------------ producer
      if (lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        uint32_t kv_it = 0, item_it = 0;
        bool ok = true;
        for (int item = blockIdx.x * 2 + u; item < p.items && ok; item += tiles_total, ++item_it) {
          const int bh = item / NB, i = item % NB;
          if (!(ok = mbar_wait(&b.q_empty, (item_it & 1) ^ 1, abort_flag))) break;
          mbar_expect_tx(&b.q_full, C::Q_BYTES);
          tma_load_2d(tq, &tm_q, &b.q_full, 0, bh * p.NP + i * BLK);
          const int32_t* lst = p.idx + ((long long)bh * NB + i) * kc;
          for (int t = 0; t < kc; ++t, ++kv_it) {
            const int j = __ldg(lst + t);
            const int s = kv_it & 1;
            if (!(ok = mbar_wait(&b.kv_empty[s], ((kv_it >> 1) & 1) ^ 1, abort_flag))) break;
            mbar_expect_tx(&b.kv_full[s], C::K_BYTES + C::V_BYTES);
            tma_load_2d(tk[s], &tm_k, &b.kv_full[s], 0, bh * p.NP + j * BLK);
#pragma unroll
            for (int hh = 0; hh < D / 64; ++hh)
              tma_load_3d(tv[s] + hh * BLK * 128, &tm_v, &b.kv_full[s], hh * 64, j * BLK, bh);
          }
        }
      }
    } else {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        const uint32_t tS = tmem_base + u * 256;
        const uint32_t tO = tS + 128;
        const uint32_t id_qk = idesc_i8(BLK);
        const uint32_t id_pv = idesc_bf16(D, false, true);
        const uint64_t dq = smem_desc(smem_u32(tq), 16, C::KSBO, C::KSW);
        uint32_t kv_it = 0, item_it = 0, it = 0;
        bool ok = true;
        for (int item = blockIdx.x * 2 + u; item < p.items && ok; item += tiles_total, ++item_it) {
          if (!(ok = mbar_wait(&b.q_full, item_it & 1, abort_flag))) break;
          for (int t = 0; t < kc; ++t, ++kv_it, ++it) {
            const int s = kv_it & 1;
            if (!(ok = mbar_wait(&b.kv_full[s], (kv_it >> 1) & 1, abort_flag))) break;
            tc_fence_after();
            const uint64_t dk = smem_desc(smem_u32(tk[s]), 16, C::KSBO, C::KSW);
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk)
              mma_i8_ss(tS, dq + uint64_t(kk * 2), dk + uint64_t(kk * 2), id_qk, kk > 0 ? 1u : 0u);
            tc_commit(&b.s_full);
            if (t == kc - 1) tc_commit(&b.q_empty);
            if (!(ok = mbar_wait(&b.p_full, it & 1, abort_flag))) break;
            if (t == 0 && !(ok = mbar_wait(&b.o_free, (item_it & 1) ^ 1, abort_flag))) break;
            tc_fence_after();
            const uint64_t dv = smem_desc(smem_u32(tv[s]), BLK * 128, 1024, 2);
#pragma unroll
            for (int kk = 0; kk < BLK / 16; ++kk)
              mma_bf16_ts(tO, tS + kk * 8, dv + uint64_t(kk * (2048 >> 4)), id_pv, (t > 0 || kk > 0) ? 1u : 0u);
            tc_commit(&b.kv_empty[s]);
            if (t == kc - 1) tc_commit(&b.o_full);
          }
        }
      }
    }
  } else {
    // -------------------------------------------------------------- softmax
    const int u = (warp - 4) >> 2;
    TileBars& b = bars[u];
    const int r = tid - 128 * (u + 1);              // query row inside the tile = TMEM lane
    const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
    const uint32_t tS = tmem_base + u * 256 + lane_off;
    const uint32_t tO = tS + 128;
    uint32_t item_it = 0, it = 0;
    bool ok = true;
    for (int item = blockIdx.x * 2 + u; item < p.items && ok; item += tiles_total, ++item_it) {
      const int bh = item / NB, i = item % NB;
      const float sq_i = __ldg(p.sq + (long long)bh * NB + i);
      const int32_t* lst = p.idx + ((long long)bh * NB + i) * kc;
      float m = -INFINITY, l = 0.f;
      for (int t = 0; t < kc; ++t, ++it) {
        const int j = __ldg(lst + t);
        const float c = sq_i * __ldg(p.sk + (long long)bh * NB + j) * p.qk_scale;
        const int nvalid = p.N - j * BLK;
        if (!(ok = mbar_wait(&b.s_full, it & 1, abort_flag))) break;
        tc_fence_after();
        float mx = -INFINITY;
#pragma unroll
        for (int ch = 0; ch < BLK / 16; ++ch) {
          uint32_t v[16];
          SLA_TMEM_LD16(tS + ch * 16, v);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float x = (float)(int)v[e] * c;
            if (ch * 16 + e >= nvalid) x = -INFINITY;
            mx = fmaxf(mx, x);
          }
        }
        const float m_new = fmaxf(m, mx);
        // tcgen05.ld/st are warp-collective: the whole warp rescales when any
        // of its rows has a new maximum (alpha is exactly 1 for the others).
        if (t > 0 && __any_sync(0xffffffffu, m_new > m)) {
          const float alpha = (m_new > m) ? ex2_approx(m - m_new) : 1.f;
          l *= alpha;
#pragma unroll
          for (int ch = 0; ch < D / 16; ++ch) {
            uint32_t v[16];
            SLA_TMEM_LD16(tO + ch * 16, v);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
            SLA_TMEM_ST16(tO + ch * 16, v);
          }
        }
        m = m_new;
#pragma unroll
        for (int ch = 0; ch < BLK / 16; ++ch) {
          uint32_t v[16];
          SLA_TMEM_LD16(tS + ch * 16, v);
          tmem_ld_wait();
          uint32_t pk[8];
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            float x0 = (float)(int)v[e] * c, x1 = (float)(int)v[e + 1] * c;
            float p0 = (ch * 16 + e < nvalid) ? ex2_approx(x0 - m) : 0.f;
            float p1 = (ch * 16 + e + 1 < nvalid) ? ex2_approx(x1 - m) : 0.f;
            l += p0 + p1;
            pk[e >> 1] = pack_bf16x2(p0, p1);
          }
          SLA_TMEM_ST8(tS + ch * 8, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&b.p_full);
      }
      if (!ok) break;
      if (!(ok = mbar_wait(&b.o_full, item_it & 1, abort_flag))) break;
      tc_fence_after();
      const float inv_l = 1.f / l;
      const long long n = (long long)i * BLK + r;
      const bool valid = r < BLK && n < p.N;
      const long long obase = ((long long)bh * p.N + n) * D;
#pragma unroll
      for (int ch = 0; ch < D / 16; ++ch) {
        uint32_t v[16];
        SLA_TMEM_LD16(tO + ch * 16, v);
        tmem_ld_wait();
        if (valid) {
          float4* dst = reinterpret_cast<float4*>(p.o + obase + ch * 16);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_float4(__uint_as_float(v[4 * q]) * inv_l, __uint_as_float(v[4 * q + 1]) * inv_l,
                                 __uint_as_float(v[4 * q + 2]) * inv_l, __uint_as_float(v[4 * q + 3]) * inv_l);
        }
      }
      tc_fence_before();
      mbar_arrive(&b.o_free);
    }
  }

  __syncwarp();   // reconverge the single-lane roles before the CTA barrier
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem_base, 512);
}

}  // namespace sla
