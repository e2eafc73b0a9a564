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
//   warp 0 / 2   TMA producers of tile 0 / 1: lane 0 loads Q and K, lane 1 V
//                (two-stage rings; a K stage is released when its block's QK^T
//                products finish, a V stage when its PV products finish, so
//                the next K tile is not held up by the PV of the previous one)
//   warp 1 / 3   tcgen05.mma issuer of tile 0 / 1
//   warps 4-7    softmax + epilogue of tile 0 (thread = query row = TMEM lane)
//   warps 8-11   softmax + epilogue of tile 1
// A tile walks its key blocks in halves of 64 keys.  TMEM (512 columns): tile
// u owns columns [256u, 256u+256): two S buffers of 64 columns (S for half h
// goes to buffer h % 2; P, bf16, is written over the first 32 columns of its
// S) and O in [256u+128, 256u+128+D).  With two S buffers the QK^T of the next
// half is already queued on the tensor core while the softmax of this half
// runs.  The tensor core executes one CTA's MMAs in issue order, so a QK^T
// issued after a PV may overwrite the S buffer that PV reads P from.
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
  static constexpr int HB = 64;                  // keys per half block (MMA N of QK^T)
  static constexpr int NH = BLK / HB;            // halves per key block
  static constexpr int Q_BYTES = BQ * D;         // int8
  static constexpr int K_BYTES = BLK * D;        // int8
  static constexpr int V_BYTES = BLK * D * 2;    // bf16
  static constexpr int STAGES = 2;
  static constexpr int TILE_BYTES = Q_BYTES + STAGES * (K_BYTES + V_BYTES);
  static constexpr int BAR_BYTES = 2 * 20 * 8 + 16;         // two TileBars, TMEM slot, abort flag
  static constexpr int SMEM_USED = 2 * TILE_BYTES + BAR_BYTES;
  static constexpr int SMEM_LIMIT = 232448;                  // 227 KB per CTA
  static_assert(SMEM_USED <= SMEM_LIMIT, "tile rings do not fit in shared memory");
  // room to round the base up to 1024 bytes where the limit allows (checked at
  // run time), and at least 120 KB, so that one CTA (holding all 512 TMEM
  // columns) fills an SM
  static constexpr int SMEM_ALIGNED = SMEM_USED + 1024 < SMEM_LIMIT ? SMEM_USED + 1024 : SMEM_LIMIT;
  static constexpr int SMEM = SMEM_ALIGNED > 122880 ? SMEM_ALIGNED : 122880;
  static constexpr uint32_t KSW = (D == 128) ? 2u : 4u;     // Q/K swizzle: 128B or 64B rows
  static constexpr uint32_t KSBO = (D == 128) ? 1024u : 512u;
  static constexpr uint32_t K_HALF_BYTES = HB * D;          // 64 rows of K (int8)
  static constexpr uint32_t V_HALF_BYTES = HB * 128;        // 64 rows of one 64-channel V atom
};

struct TileBars {
  uint64_t q_full, q_empty, o_full, o_free;
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t mma_drain, pad;   // end of the MMA issuer: every MMA it issued has finished
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
  constexpr int NH = C::NH;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  static_assert(sizeof(TileBars) == 20 * 8, "barrier block size");
  if (uint32_t(base - smem_raw) + C::SMEM_USED > dynamic_smem_bytes()) {
    if (threadIdx.x == 0) raise_error(DEV_ERR_LAYOUT);
    return;   // uniform: every thread sees the same base
  }
  TileBars* bars = reinterpret_cast<TileBars*>(base + 2 * C::TILE_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int u = 0; u < 2; ++u) {
      TileBars& b = bars[u];
      mbar_init(&b.q_full, 1);
      mbar_init(&b.q_empty, 1);
      mbar_init(&b.o_full, 1);
      mbar_init(&b.o_free, 128);
      mbar_init(&b.mma_drain, 1);
      for (int s = 0; s < 2; ++s) {
        mbar_init(&b.s_full[s], 1);
        mbar_init(&b.p_full[s], 128);
        mbar_init(&b.pv_done[s], 1);
        mbar_init(&b.k_full[s], 1);
        mbar_init(&b.k_empty[s], 1);
        mbar_init(&b.v_full[s], 1);
        mbar_init(&b.v_empty[s], 1);
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
    if ((warp & 1) == 0) {
      // ------------------------------------------------------------ producers
      // Lane 0 loads Q and the K tiles, lane 1 the V tiles; each walks the
      // block list on its own, reading the next entry one block ahead.
      if (lane < 2) {
        if (lane == 0) {
          tma_prefetch_desc(&tm_q);
          tma_prefetch_desc(&tm_k);
        } else {
          tma_prefetch_desc(&tm_v);
        }
        uint32_t blk_it = 0, item_it = 0;
        uint32_t nq = 0, nkv = 0;   // loads issued: Q (lane 0), K or V (lane 0 / lane 1)
        bool ok = true;
        for (int item = blockIdx.x * 2 + u; item < p.items && ok; item += tiles_total, ++item_it) {
          const int bh = item / NB, i = item % NB;
          if (lane == 0) {
            if (!(ok = mbar_wait(&b.q_empty, (item_it & 1) ^ 1, abort_flag))) break;
            mbar_expect_tx(&b.q_full, C::Q_BYTES);
            tma_load_2d(tq, &tm_q, &b.q_full, 0, bh * p.NP + i * BLK);
            ++nq;
          }
          const int32_t* lst = p.idx + ((long long)bh * NB + i) * kc;
          int jn = __ldg(lst);
          for (int t = 0; t < kc; ++t, ++blk_it) {
            const int j = jn;
            if (t + 1 < kc) jn = __ldg(lst + t + 1);
            const int s = blk_it & 1;
            const uint32_t par = ((blk_it >> 1) & 1) ^ 1;
            unsigned char* tk = tq + C::Q_BYTES + s * (C::K_BYTES + C::V_BYTES);
            if (lane == 0) {
              if (!(ok = mbar_wait(&b.k_empty[s], par, abort_flag))) break;
              mbar_expect_tx(&b.k_full[s], C::K_BYTES);
              tma_load_2d(tk, &tm_k, &b.k_full[s], 0, bh * p.NP + j * BLK);
              ++nkv;
            } else {
              if (!(ok = mbar_wait(&b.v_empty[s], par, abort_flag))) break;
              mbar_expect_tx(&b.v_full[s], C::V_BYTES);
#pragma unroll
              for (int hh = 0; hh < D / 64; ++hh)
                tma_load_3d(tk + C::K_BYTES + hh * BLK * 128, &tm_v, &b.v_full[s], hh * 64, j * BLK, bh);
              ++nkv;
            }
          }
        }
        // Loads still in flight (only after a failed wait) land before the CTA
        // exits: wait (bounded) for the last phase armed on each barrier.
        if (lane == 0 && nq > 0) (void)mbar_wait(&b.q_full, (nq - 1) & 1, nullptr);
        for (uint32_t bb = nkv > 2 ? nkv - 2 : 0; bb < nkv; ++bb)
          (void)mbar_wait(lane == 0 ? &b.k_full[bb & 1] : &b.v_full[bb & 1], (bb >> 1) & 1, nullptr);
      }
    } else {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        const uint32_t tS = tmem_base + u * 256;   // S buffers at tS and tS + 64
        const uint32_t tO = tS + 128;
        const uint32_t id_qk = idesc_i8(C::HB);
        const uint32_t id_pv = idesc_bf16(D, false, true);
        const uint64_t dq = smem_desc(smem_u32(tq), 16, C::KSBO, C::KSW);
        uint32_t kv_it = 0, item_it = 0, hg = 0;   // hg: halves of the items before this one
        bool ok = true;
        for (int item = blockIdx.x * 2 + u; item < p.items && ok; item += tiles_total, ++item_it) {
          const int H = kc * NH;
          if (!(ok = mbar_wait(&b.q_full, item_it & 1, abort_flag))) break;
          // S(y) = Q K_half(y)^T into buffer (hg + y) % 2; at the first half of a
          // key block it first waits for that block's K/V stage
          auto issue_qk = [&](int y) -> bool {
            const uint32_t g = hg + y;
            const uint32_t blk_it = kv_it + y / NH;
            const int s = blk_it & 1;
            if (y % NH == 0) {
              if (!mbar_wait(&b.k_full[s], (blk_it >> 1) & 1, abort_flag)) return false;
              tc_fence_after();
            }
            unsigned char* tk = tq + C::Q_BYTES + s * (C::K_BYTES + C::V_BYTES);
            const uint64_t dk = smem_desc(smem_u32(tk) + (y % NH) * C::K_HALF_BYTES, 16, C::KSBO, C::KSW);
            const uint32_t dS = tS + (g & 1) * 64;
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk)
              mma_i8_ss(dS, dq + uint64_t(kk * 2), dk + uint64_t(kk * 2), id_qk, kk > 0 ? 1u : 0u);
            tc_commit(&b.s_full[g & 1]);
            if (y % NH == NH - 1) tc_commit(&b.k_empty[s]);
            if (y == H - 1) tc_commit(&b.q_empty);
            return true;
          };
          ok = issue_qk(0);
          if (ok && H > 1) ok = issue_qk(1);
          for (int x = 0; x < H && ok; ++x) {
            const uint32_t g = hg + x;
            if (!(ok = mbar_wait(&b.p_full[g & 1], (g >> 1) & 1, abort_flag))) break;
            if (x == 0 && !(ok = mbar_wait(&b.o_free, (item_it & 1) ^ 1, abort_flag))) break;
            const uint32_t vblk = kv_it + x / NH;
            const int s = vblk & 1;
            if (x % NH == 0 && !(ok = mbar_wait(&b.v_full[s], (vblk >> 1) & 1, abort_flag))) break;
            tc_fence_after();
            unsigned char* tv = tq + C::Q_BYTES + s * (C::K_BYTES + C::V_BYTES) + C::K_BYTES;
            const uint64_t dv = smem_desc(smem_u32(tv) + (x % NH) * C::V_HALF_BYTES, BLK * 128, 1024, 2);
            const uint32_t aP = tS + (g & 1) * 64;
#pragma unroll
            for (int kk = 0; kk < C::HB / 16; ++kk)
              mma_bf16_ts(tO, aP + kk * 8, dv + uint64_t(kk * (2048 >> 4)), id_pv, (x > 0 || kk > 0) ? 1u : 0u);
            tc_commit(&b.pv_done[g & 1]);
            if (x % NH == NH - 1) tc_commit(&b.v_empty[s]);
            if (x == H - 1) tc_commit(&b.o_full);
            if (x + 2 < H) ok = issue_qk(x + 2);
          }
          hg += H;
          kv_it += kc;
        }
        // every MMA issued here finishes before the CTA frees TMEM (bounded)
        tc_commit(&b.mma_drain);
        (void)mbar_wait(&b.mma_drain, 0, nullptr);
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
    uint32_t item_it = 0, hg = 0;
    bool ok = true;
    const int part_rows = p.N % BLK;                // rows of a partial last block (0: none)
    for (int item = blockIdx.x * 2 + u; item < p.items && ok; item += tiles_total, ++item_it) {
      const int bh = item / NB, i = item % NB;
      const float sq_i = __ldg(p.sq + (long long)bh * NB + i) * p.qk_scale;
      const int32_t* lst = p.idx + ((long long)bh * NB + i) * kc;
      const int H = kc * NH;
      // running maximum m (log2 domain) and normaliser l of this row
      float m = -INFINITY, l = 0.f;
      float cl = 0.f;
      int jl = 0;
      for (int x = 0; x < H; ++x) {
        const int t = x / NH;
        const uint32_t g = hg + x;
        if ((t & 31) == 0 && x % NH == 0) {   // block list and scales, 32 blocks at a time
          jl = (t + lane < kc) ? __ldg(lst + t + lane) : 0;
          cl = sq_i * __ldg(p.sk + (long long)bh * NB + jl);
        }
        const int j = __shfl_sync(0xffffffffu, jl, t & 31);
        const float c = __shfl_sync(0xffffffffu, cl, t & 31);   // sq_i * sk_j * log2(e) / sqrt(D) >= 0
        // valid keys of this half (fewer only in a partial last block)
        const int nvalid = (part_rows != 0 && j == NB - 1)
                               ? min(max(part_rows - (x % NH) * C::HB, 0), C::HB)
                               : C::HB;
        const bool partial = nvalid < C::HB;       // uniform across the CTA
        if (!(ok = mbar_wait(&b.s_full[g & 1], (g >> 1) & 1, abort_flag))) break;
        tc_fence_after();
        const uint32_t sbuf = tS + (g & 1) * 64;
        uint32_t v[64];
        SLA_TMEM_LD32(sbuf, v);
        SLA_TMEM_LD32(sbuf + 32, (v + 32));
        tmem_ld_wait();
        // row maximum of the int32 scores (c >= 0 keeps the order)
        int amax = INT_MIN;
        if (!partial) {
#pragma unroll
          for (int e = 0; e < 64; ++e) amax = max(amax, (int)v[e]);
        } else {
#pragma unroll
          for (int e = 0; e < 64; ++e)
            if (e < nvalid) amax = max(amax, (int)v[e]);
        }
        const float mx = (nvalid > 0) ? (float)amax * c : -INFINITY;
        if (x == 0) {
          m = mx;
        } else if (__any_sync(0xffffffffu, mx > m + 8.f)) {
          // Some row's maximum grew by more than 2^8: once the previous PV has
          // finished, the warp rescales O (tcgen05.ld/st are warp-collective);
          // rows whose maximum did not grow keep alpha = 1.  Otherwise the
          // stale maximum stays (P <= 2^8).
          // PV(g-2) and older are complete (QK(g) was issued after PV(g-2) and
          // its S is ready); PV(g-1) uses buffer (g-1)&1, whose uses before it
          // are complete, so this parity names PV(g-1) without ambiguity.
          if (!(ok = mbar_wait(&b.pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1, abort_flag))) break;
          tc_fence_after();
          const float m_new = fmaxf(m, mx);
          const float alpha = ex2_approx(m - m_new);
          l *= alpha;
          m = m_new;
#pragma unroll
          for (int ch = 0; ch < D / 16; ++ch) {   // 16 columns at a time: v[] is still live
            uint32_t w[16];
            SLA_TMEM_LD16(tO + ch * 16, w);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e) w[e] = __float_as_uint(__uint_as_float(w[e]) * alpha);
            SLA_TMEM_ST16(tO + ch * 16, w);
          }
        }
        // P = 2^(acc * c - m) rounded to bf16 into TMEM.  The float with bits
        // acc + 0x4B400000 is exactly 1.5*2^23 + acc (|acc| <= D*127^2 < 2^22),
        // so acc*c - m = fma(that, c, -(1.5*2^23*c + m)); the one rounding of
        // that constant shifts all exponents of this row and half by the same
        // amount (< 2^-24 relative to 1.5*2^23*c), i.e. scales P and l alike.
        // The packed pair e/2 goes to v[e/2], a slot already consumed.
        const float kk = -fmaf(12582912.f, c, m);
        float l0 = 0.f, l1 = 0.f, l2 = 0.f, l3 = 0.f;
#pragma unroll
        for (int e = 0; e < 64; e += 4) {
          float p0 = ex2_approx(fmaf(__int_as_float((int)v[e] + 0x4B400000), c, kk));
          float p1 = ex2_approx(fmaf(__int_as_float((int)v[e + 1] + 0x4B400000), c, kk));
          float p2 = ex2_approx(fmaf(__int_as_float((int)v[e + 2] + 0x4B400000), c, kk));
          float p3 = ex2_approx(fmaf(__int_as_float((int)v[e + 3] + 0x4B400000), c, kk));
          if (partial) {
            p0 = (e < nvalid) ? p0 : 0.f;
            p1 = (e + 1 < nvalid) ? p1 : 0.f;
            p2 = (e + 2 < nvalid) ? p2 : 0.f;
            p3 = (e + 3 < nvalid) ? p3 : 0.f;
          }
          l0 += p0;
          l1 += p1;
          l2 += p2;
          l3 += p3;
          v[e >> 1] = pack_bf16x2(p0, p1);
          v[(e >> 1) + 1] = pack_bf16x2(p2, p3);
        }
        l += (l0 + l1) + (l2 + l3);
        SLA_TMEM_ST16(sbuf, v);
        SLA_TMEM_ST16(sbuf + 16, (v + 16));
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&b.p_full[g & 1]);
      }
      if (!ok) break;
      hg += H;
      if (!(ok = mbar_wait(&b.o_full, item_it & 1, abort_flag))) break;
      tc_fence_after();
      const float inv_l = 1.f / l;
      const long long n = (long long)i * BLK + r;
      const bool valid = r < BLK && n < p.N;
      const long long obase = ((long long)bh * p.N + n) * D;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t w[32];
        SLA_TMEM_LD32(tO + ch * 32, w);
        tmem_ld_wait();
        if (valid) {
          float4* dst = reinterpret_cast<float4*>(p.o + obase + ch * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q] = make_float4(__uint_as_float(w[4 * q]) * inv_l, __uint_as_float(w[4 * q + 1]) * inv_l,
                                 __uint_as_float(w[4 * q + 2]) * inv_l, __uint_as_float(w[4 * q + 3]) * inv_l);
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
