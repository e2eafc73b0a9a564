// K4: critical-block attention plus the linear part, on the 5th-generation
// tensor cores.
//
// "Turbo Diffusion：秒级生成与高清保真的视频扩散技术突破", section 三(一) item 3
// (attention re-tiled to 128x128 tensor-core tiles with a parallel softmax),
// section 三(二) item 3 (SageSLA: after the block selection, INT8 computation
// on the selected blocks) and item 2 (the rest through a linear branch and a
// linear projection).  For query block i of head (b, h) and each selected key
// block j (ascending):
//     S = int32(Qi8_i . Ki8_j^T) * sq_i * sk_j / sqrt(D)   (tcgen05 kind::i8)
//     online softmax in float32 (exp2 domain), P rounded to bf16
//     O += P . V_j                                        (tcgen05 kind::f16)
// then the linear part of the non-selected blocks, with W_proj folded into the
// states (G'_i = sum_{j not selected} h_j W_proj, g_i = sum z_j):
//     O += A . G'_i,  A = bf16(phi(q) * l / den),  den = phi(q) . g_i
// (one more kind::f16 product, A taken from TMEM like P), so that
//     out = O / l = O_sparse + phi(q) G'_i / den,
// l being the sum of the unrounded P; out is written as bf16 (round to nearest
// even) or float32.  Either part can be switched off (p.sparse, p.lin): with
// the linear part alone l = 1.
//
// One persistent CTA per SM runs two independent pipelines ("tiles"), each
// working on its own sequence of (head, query block) items: tile u of CTA c
// takes items c + u * G, then every 2G further (G CTAs).  In the last, partial
// round the items fall on tile 0 of distinct CTAs, so each runs alone on its
// SM instead of two sharing one while other SMs idle.
//   warp 0 / 2   TMA producers of tile 0 / 1: lane 0 loads Q and K, lane 1 V
//                and G'_i (two-stage rings; G'_i goes through the V ring as
//                one more block; a K stage is released when its block's QK^T
//                products finish, a V stage when its PV products finish)
//   warp 1 / 3   tcgen05.mma issuer of tile 0 / 1
//   warps 4-7    softmax of tile 0 (thread = query row = TMEM lane)
//   warps 8-11   softmax of tile 1
//   warps 12-15  output warpgroup of both tiles (thread = query row): den and
//                A of the linear part, then the epilogue O / l -> out
// The softmax warpgroups hand each row's l over through shared memory, so
// they go on to the next item while the output warpgroup finishes this one.
// Registers are split with setmaxnreg: 80 per thread for warps 0-3, 144 for
// the other three warpgroups (512 threads x 128 at launch = 65536).
// A tile walks its key blocks in halves of 64 keys.  TMEM (512 columns): tile
// u owns columns [256u, 256u+256): two S buffers of 64 columns (S for half h
// goes to buffer h % 2; P, bf16, is written over the first 32 columns of its
// S) and O in [256u+128, 256u+128+D).  With two S buffers the QK^T of the next
// half is already queued on the tensor core while the softmax of this half
// runs.  The tensor core executes one CTA's MMAs in issue order, so a QK^T
// issued after a PV may overwrite the S buffer that PV reads P from.  A (D/2
// columns) goes to the S buffer the next item's first QK^T will use, after the
// PV that last read it has finished.
#pragma once
#include <cuda_bf16.h>
#include "sm100.cuh"

namespace sla {

struct AttnParams {
  const int32_t* idx;          // [BH][NB][kcp] kept blocks, ascending
  const int* kc_bh;            // [BH] list length per head, or nullptr: kc for every head
  const float* sq;             // [BH][NB][G] scale per group of 2^gshift query rows (G = BLK >> gshift)
  const float* sk;             // [BH][NB][G] scale per group of 2^gshift keys
  const __nv_bfloat16* q;      // [BH][N][D] raw queries (phi(q) of the linear part)
  const float* zrest;          // [BH][NB][D] g_i: z sums over the non-selected blocks
  void* out;                   // [BH][N][D], bf16 or float32
  int N, NB, NP, kc, kcp, items, gshift;
  int sparse;                  // the selected blocks (softmax attention) take part
  int lin;                     // the linear part is added
  int out_f32;                 // float32 output (else bf16)
  float qk_scale;              // log2(e) / sqrt(D)
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
  static constexpr int BAR_BYTES = 2 * 22 * 8 + 16;         // two TileBars, TMEM slot, abort flag
  static constexpr int L_BYTES = 2 * 128 * 4;               // l of every row of both tiles
  static constexpr int SMEM_USED = 2 * TILE_BYTES + BAR_BYTES + L_BYTES;
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
  // G'_i (D x D bf16, rows = the K dimension of A . G'_i) passes through the V
  // ring in LC chunks of LROWS rows, laid out like V blocks
  static constexpr int LROWS = D < BLK ? D : BLK;
  static constexpr int LC = D / LROWS;
  static constexpr int G_CHUNK_BYTES = LROWS * D * 2;
  static_assert(G_CHUNK_BYTES <= V_BYTES, "a G' chunk fits in a V stage");
};

struct TileBars {
  uint64_t q_full, q_empty, o_full, o_free;
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t mma_drain;   // end of the MMA issuer: every MMA it issued has finished
  uint64_t a_full;      // A of the linear part is in TMEM
  uint64_t l_full;      // the softmax has finished the item: l is in shared memory
  uint64_t pad;
};

constexpr int kAttnThreads = 512;
constexpr uint32_t kRegsLoad = 80;    // warps 0-3: TMA producers, MMA issuers
constexpr uint32_t kRegsMath = 144;   // warps 4-15: softmax, output
static_assert(128 * (kRegsLoad + 3 * kRegsMath) <= 65536, "register split within the launch's registers");

// The running row maximum is raised (and O, l rescaled) only when a new
// maximum exceeds it by more than this many powers of two; until then P may
// reach 2^kRescaleLog2, far inside the range of bf16 P and float32 sums.
constexpr float kRescaleLog2 = 16.f;

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// phi = elu + 1 of a bf16 value (raw bits): x + 1 for x > 0, else e^x.
__device__ __forceinline__ float phi_bf16(uint16_t bits) {
  const float x = __uint_as_float(uint32_t(bits) << 16);
  return x > 0.f ? x + 1.f : ex2_approx(x * 1.4426950408889634f);
}

// den = phi(q) . g for one query row (zero for a row past the block or N).
template <int D>
__device__ __forceinline__ float linear_den(const __nv_bfloat16* qrow, const float* g, bool valid) {
  float d0 = 0.f, d1 = 0.f;
  if (valid) {
#pragma unroll 4
    for (int c8 = 0; c8 < D / 8; ++c8) {
      const uint4 raw = __ldg(reinterpret_cast<const uint4*>(qrow) + c8);
      const float4 g0 = __ldg(reinterpret_cast<const float4*>(g) + 2 * c8);
      const float4 g1 = __ldg(reinterpret_cast<const float4*>(g) + 2 * c8 + 1);
      d0 = fmaf(phi_bf16(uint16_t(raw.x)), g0.x, d0);
      d1 = fmaf(phi_bf16(uint16_t(raw.x >> 16)), g0.y, d1);
      d0 = fmaf(phi_bf16(uint16_t(raw.y)), g0.z, d0);
      d1 = fmaf(phi_bf16(uint16_t(raw.y >> 16)), g0.w, d1);
      d0 = fmaf(phi_bf16(uint16_t(raw.z)), g1.x, d0);
      d1 = fmaf(phi_bf16(uint16_t(raw.z >> 16)), g1.y, d1);
      d0 = fmaf(phi_bf16(uint16_t(raw.w)), g1.z, d0);
      d1 = fmaf(phi_bf16(uint16_t(raw.w >> 16)), g1.w, d1);
    }
  }
  return d0 + d1;
}

// FINE: one quantisation scale per group of 2^gshift tokens (finer than the
// block); otherwise one per block (the default operator, its own code path).
template <int D, int BLK, bool FINE>
__global__ void __launch_bounds__(kAttnThreads, 1) k_attn(const __grid_constant__ CUtensorMap tm_q,
                                                 const __grid_constant__ CUtensorMap tm_k,
                                                 const __grid_constant__ CUtensorMap tm_v,
                                                 const __grid_constant__ CUtensorMap tm_g, const AttnParams p) {
  using C = AttnCfg<D, BLK>;
  constexpr int NH = C::NH;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  static_assert(sizeof(TileBars) == 22 * 8, "barrier block size");
  if (uint32_t(base - smem_raw) + C::SMEM_USED > dynamic_smem_bytes()) {
    if (threadIdx.x == 0) raise_error(DEV_ERR_LAYOUT);
    return;   // uniform: every thread sees the same base
  }
  TileBars* bars = reinterpret_cast<TileBars*>(base + 2 * C::TILE_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* l_buf = reinterpret_cast<float*>(base + 2 * C::TILE_BYTES + C::BAR_BYTES);   // [2][128]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int u = 0; u < 2; ++u) {
      TileBars& b = bars[u];
      mbar_init(&b.q_full, 1);
      mbar_init(&b.q_empty, 1);
      mbar_init(&b.o_full, 1);
      mbar_init(&b.o_free, 128);
      mbar_init(&b.mma_drain, 1);
      mbar_init(&b.a_full, 128);
      mbar_init(&b.l_full, 128);
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

  const int NB = p.NB;
  const int tiles_total = 2 * gridDim.x;
  const bool sparse = p.sparse != 0, lin = p.lin != 0;
  // kept blocks of the items of head bh, and the halves (64 keys) they make
  auto kc_of = [&](int bh) { return p.kc_bh != nullptr ? __ldg(p.kc_bh + bh) : p.kc; };
  auto halves_of = [&](int bh) { return sparse ? kc_of(bh) * NH : 0; };
  const int G = FINE ? BLK >> p.gshift : 1;   // quantisation scales per block

  if (warp < 4)
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLoad));
  else
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsMath));

  if (warp < 4) {
    const int u = warp >> 1;
    TileBars& b = bars[u];
    unsigned char* tq = base + u * C::TILE_BYTES;
    auto k_stage = [&](int s) { return tq + C::Q_BYTES + s * (C::K_BYTES + C::V_BYTES); };
    auto v_stage = [&](int s) { return tq + C::Q_BYTES + s * (C::K_BYTES + C::V_BYTES) + C::K_BYTES; };
    if ((warp & 1) == 0) {
      // ------------------------------------------------------------ producers
      // Lane 0 loads Q and the K tiles, lane 1 the V tiles and G'_i; each walks
      // the block list on its own, reading the next entry one block ahead.
      if (lane < 2) {
        if (lane == 0) {
          tma_prefetch_desc(&tm_q);
          tma_prefetch_desc(&tm_k);
        } else {
          tma_prefetch_desc(&tm_v);
          if (lin) tma_prefetch_desc(&tm_g);
        }
        uint32_t item_it = 0, nq = 0, nl = 0;   // nl: K loads (lane 0) or V-ring loads (lane 1)
        bool ok = true;
        for (int item = blockIdx.x + u * gridDim.x; item < p.items && ok; item += tiles_total, ++item_it) {
          const int bh = item / NB, i = item % NB;
          if (sparse) {
            const int kc = kc_of(bh);
            if (lane == 0) {
              if (!(ok = mbar_wait(&b.q_empty, (item_it & 1) ^ 1, abort_flag))) break;
              mbar_expect_tx(&b.q_full, C::Q_BYTES);
              tma_load_2d(tq, &tm_q, &b.q_full, 0, bh * p.NP + i * BLK);
              ++nq;
            }
            const int32_t* lst = p.idx + ((long long)bh * NB + i) * p.kcp;
            int jn = __ldg(lst);
            for (int t = 0; t < kc; ++t) {
              const int j = jn;
              if (t + 1 < kc) jn = __ldg(lst + t + 1);
              const int s = nl & 1;
              const uint32_t par = ((nl >> 1) & 1) ^ 1;
              if (lane == 0) {
                if (!(ok = mbar_wait(&b.k_empty[s], par, abort_flag))) break;
                mbar_expect_tx(&b.k_full[s], C::K_BYTES);
                tma_load_2d(k_stage(s), &tm_k, &b.k_full[s], 0, bh * p.NP + j * BLK);
              } else {
                if (!(ok = mbar_wait(&b.v_empty[s], par, abort_flag))) break;
                mbar_expect_tx(&b.v_full[s], C::V_BYTES);
#pragma unroll
                for (int hh = 0; hh < D / 64; ++hh)
                  tma_load_3d(v_stage(s) + hh * BLK * 128, &tm_v, &b.v_full[s], hh * 64, j * BLK, bh);
              }
              ++nl;
            }
          }
          if (lin && lane == 1) {
            for (int ch = 0; ch < C::LC && ok; ++ch) {
              const int s = nl & 1;
              if (!(ok = mbar_wait(&b.v_empty[s], ((nl >> 1) & 1) ^ 1, abort_flag))) break;
              mbar_expect_tx(&b.v_full[s], C::G_CHUNK_BYTES);
#pragma unroll
              for (int hh = 0; hh < D / 64; ++hh)
                tma_load_2d(v_stage(s) + hh * BLK * 128, &tm_g, &b.v_full[s], hh * 64,
                            int(((long long)bh * NB + i) * D + ch * C::LROWS));
              ++nl;
            }
          }
        }
        // Loads still in flight (only after a failed wait) land before the CTA
        // exits: wait (bounded) for the last phase armed on each barrier.
        if (lane == 0 && nq > 0) (void)mbar_wait(&b.q_full, (nq - 1) & 1, nullptr);
        for (uint32_t bb = nl > 2 ? nl - 2 : 0; bb < nl; ++bb)
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
        uint32_t kit = 0, vit = 0, item_it = 0, hg = 0;   // hg: halves of the items before this one
        bool ok = true;
        for (int item = blockIdx.x + u * gridDim.x; item < p.items && ok; item += tiles_total, ++item_it) {
          const int H = halves_of(item / NB);
          if (sparse) {
            if (!(ok = mbar_wait(&b.q_full, item_it & 1, abort_flag))) break;
            // S(y) = Q K_half(y)^T into buffer (hg + y) % 2; at the first half of a
            // key block it first waits for that block's K stage
            auto issue_qk = [&](int y) -> bool {
              const uint32_t g = hg + y;
              const uint32_t blk = kit + y / NH;
              const int s = blk & 1;
              if (y % NH == 0) {
                if (!mbar_wait(&b.k_full[s], (blk >> 1) & 1, abort_flag)) return false;
                tc_fence_after();
              }
              const uint64_t dk = smem_desc(smem_u32(k_stage(s)) + (y % NH) * C::K_HALF_BYTES, 16, C::KSBO, C::KSW);
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
              const uint32_t vb = vit + x / NH;
              const int s = vb & 1;
              if (x % NH == 0 && !(ok = mbar_wait(&b.v_full[s], (vb >> 1) & 1, abort_flag))) break;
              tc_fence_after();
              const uint64_t dv = smem_desc(smem_u32(v_stage(s)) + (x % NH) * C::V_HALF_BYTES, BLK * 128, 1024, 2);
              const uint32_t aP = tS + (g & 1) * 64;
#pragma unroll
              for (int kk = 0; kk < C::HB / 16; ++kk)
                mma_bf16_ts(tO, aP + kk * 8, dv + uint64_t(kk * (2048 >> 4)), id_pv, (x > 0 || kk > 0) ? 1u : 0u);
              tc_commit(&b.pv_done[g & 1]);
              if (x % NH == NH - 1) tc_commit(&b.v_empty[s]);
              if (x + 2 < H) ok = issue_qk(x + 2);
            }
            if (!ok) break;
            kit += H / NH;
            vit += H / NH;
          }
          if (lin) {
            // O += A . G'_i, A (bf16, D/2 columns) in the S buffer of half hg + H
            if (H == 0 && !(ok = mbar_wait(&b.o_free, (item_it & 1) ^ 1, abort_flag))) break;
            if (!(ok = mbar_wait(&b.a_full, item_it & 1, abort_flag))) break;
            const uint32_t aL = tS + ((hg + H) & 1) * 64;
            for (int ch = 0; ch < C::LC && ok; ++ch) {
              const int s = vit & 1;
              if (!(ok = mbar_wait(&b.v_full[s], (vit >> 1) & 1, abort_flag))) break;
              tc_fence_after();
              const uint64_t dv = smem_desc(smem_u32(v_stage(s)), BLK * 128, 1024, 2);
#pragma unroll
              for (int kk = 0; kk < C::LROWS / 16; ++kk)
                mma_bf16_ts(tO, aL + (ch * (C::LROWS / 16) + kk) * 8, dv + uint64_t(kk * (2048 >> 4)), id_pv,
                            (H > 0 || ch > 0 || kk > 0) ? 1u : 0u);
              tc_commit(&b.v_empty[s]);
              ++vit;
            }
            if (!ok) break;
          }
          tc_commit(&b.o_full);
          hg += H;
        }
        // every MMA issued here finishes before the CTA frees TMEM (bounded)
        tc_commit(&b.mma_drain);
        (void)mbar_wait(&b.mma_drain, 0, nullptr);
      }
    }
  } else if (warp < 12) {
    // -------------------------------------------------------------- softmax
    const int u = (warp - 4) >> 2;
    TileBars& b = bars[u];
    const int r = tid - 128 * (u + 1);              // query row inside the tile = TMEM lane
    const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
    const uint32_t tS = tmem_base + u * 256 + lane_off;
    const uint32_t tO = tS + 128;
    uint32_t hg = 0;
    bool ok = true;
    const int part_rows = p.N % BLK;                // rows of a partial last block (0: none)
    for (int item = blockIdx.x + u * gridDim.x; sparse && item < p.items && ok; item += tiles_total) {
      const int bh = item / NB, i = item % NB;
      const int kc = kc_of(bh), H = kc * NH;
      // the scale of this row's group (rows past the block reuse the last one)
      const float sq_i = FINE ? __ldg(p.sq + ((long long)bh * NB + i) * G + (min(r, BLK - 1) >> p.gshift)) * p.qk_scale
                              : __ldg(p.sq + (long long)bh * NB + i) * p.qk_scale;
      const int32_t* lst = p.idx + ((long long)bh * NB + i) * p.kcp;
      // running maximum m (log2 domain) and normaliser l of this row
      float m = -INFINITY, l = 0.f;
      float cl = 0.f;
      int jl = 0;
      for (int x = 0; x < H; ++x) {
        const int t = x / NH;
        const uint32_t g = hg + x;
        if ((t & 31) == 0 && x % NH == 0) {   // block list (and block scales), 32 blocks at a time
          jl = (t + lane < kc) ? __ldg(lst + t + lane) : 0;
          if (!FINE) cl = sq_i * __ldg(p.sk + (long long)bh * NB + jl);
        }
        const int j = __shfl_sync(0xffffffffu, jl, t & 31);
        // c0, c1 = sq * sk * log2(e) / sqrt(D) >= 0 for keys 0-31 and 32-63 of the half
        float c0, c1;
        if (!FINE) {
          c0 = c1 = __shfl_sync(0xffffffffu, cl, t & 31);
        } else {
          const float* skb = p.sk + ((long long)bh * NB + j) * G;
          const int ko = (x % NH) * C::HB;
          c0 = sq_i * __ldg(skb + (ko >> p.gshift));
          c1 = sq_i * __ldg(skb + ((ko + 32) >> p.gshift));
        }
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
        // The float with bits acc + 0x4B400000 is exactly 1.5*2^23 + acc
        // (|acc| <= D*127^2 < 2^22); c >= 0, so its maximum gives the row's.
#pragma unroll
        for (int e = 0; e < 64; ++e) v[e] += 0x4B400000u;
        if (partial) {   // keys past N (a partial last block): out of the maximum
#pragma unroll
          for (int e = 0; e < 64; ++e)
            if (e >= nvalid) v[e] = 0xFF800000u;   // -inf
        }
        float mx;
        if constexpr (!FINE) {
          float xm[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) xm[q] = fmax3(__uint_as_float(v[3 * q]), __uint_as_float(v[3 * q + 1]),
                                                    __uint_as_float(v[3 * q + 2]));
#pragma unroll
          for (int e = 24; e < 64; e += 2)
            xm[(e / 2) & 7] = fmax3(xm[(e / 2) & 7], __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
          const float xmax = fmaxf(fmax3(xm[0], xm[1], xm[2]), fmax3(fmax3(xm[3], xm[4], xm[5]), xm[6], xm[7]));
          mx = (xmax - 12582912.f) * c0;   // exact difference; -inf when no key is valid
        } else {
          // maxima of keys 0-31 and 32-63 (their scales may differ)
          float xa[4], xb[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            xa[q] = fmax3(__uint_as_float(v[3 * q]), __uint_as_float(v[3 * q + 1]), __uint_as_float(v[3 * q + 2]));
            xb[q] = fmax3(__uint_as_float(v[32 + 3 * q]), __uint_as_float(v[33 + 3 * q]),
                          __uint_as_float(v[34 + 3 * q]));
          }
#pragma unroll
          for (int e = 12; e < 32; e += 2) {
            xa[(e / 2) & 3] = fmax3(xa[(e / 2) & 3], __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
            xb[(e / 2) & 3] = fmax3(xb[(e / 2) & 3], __uint_as_float(v[32 + e]), __uint_as_float(v[33 + e]));
          }
          const float xm0 = fmaxf(fmax3(xa[0], xa[1], xa[2]), xa[3]);
          const float xm1 = fmaxf(fmax3(xb[0], xb[1], xb[2]), xb[3]);
          // exact differences; -inf for a group without a valid key (NaN, ignored
          // by the maximum, if that group's scale is 0)
          mx = fmaxf((xm0 - 12582912.f) * c0, (xm1 - 12582912.f) * c1);
        }
        if (x == 0) {
          m = mx;
        } else if (__any_sync(0xffffffffu, mx > m + kRescaleLog2)) {
          // Some row's maximum grew by more than 2^kRescaleLog2: once the
          // previous PV has finished, the warp rescales O (tcgen05.ld/st are
          // warp-collective).  Otherwise the stale maximum stays
          // (P <= 2^kRescaleLog2).
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
        // P = 2^(acc * c - m) = 2^((1.5*2^23 + acc) * c - (1.5*2^23 * c + m)):
        // one FMA per key (two per packed instruction); the one rounding of
        // the constant shifts all exponents of a scale group by the same
        // amount (< 2^-24 relative to 1.5*2^23*c), i.e. scales its P and
        // their share of l alike (with one scale per block, the whole half).
        const float kk0 = -fmaf(12582912.f, c0, m), kk1 = FINE ? -fmaf(12582912.f, c1, m) : kk0;
        const uint64_t c20 = f32x2(c0, c0), k20 = f32x2(kk0, kk0);
        const uint64_t c21 = FINE ? f32x2(c1, c1) : c20, k21 = FINE ? f32x2(kk1, kk1) : k20;
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
          float y0, y1;
          f32x2_split(fma_f32x2(f32x2(__uint_as_float(v[e]), __uint_as_float(v[e + 1])), e < 32 ? c20 : c21,
                                e < 32 ? k20 : k21),
                      y0, y1);
          v[e] = __float_as_uint(ex2_approx(y0));
          v[e + 1] = __float_as_uint(ex2_approx(y1));
        }
        if (partial) {
#pragma unroll
          for (int e = 0; e < 64; ++e)
            if (e >= nvalid) v[e] = 0u;
        }
        // l sums the unrounded P (four packed partial sums); the bf16 pair
        // e/2 goes to v[e/2], a slot already consumed
        uint64_t la = f32x2(0.f, 0.f), lb = la;
#pragma unroll
        for (int e = 0; e < 64; e += 4) {
          la = add_f32x2(la, f32x2(__uint_as_float(v[e]), __uint_as_float(v[e + 1])));
          lb = add_f32x2(lb, f32x2(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3])));
          v[e >> 1] = pack_bf16x2(__uint_as_float(v[e]), __uint_as_float(v[e + 1]));
          v[(e >> 1) + 1] = pack_bf16x2(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
        }
        {
          float a0, a1, b0, b1;
          f32x2_split(la, a0, a1);
          f32x2_split(lb, b0, b1);
          l += (a0 + a1) + (b0 + b1);
        }
        SLA_TMEM_ST16(sbuf, v);
        SLA_TMEM_ST16(sbuf + 16, (v + 16));
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&b.p_full[g & 1]);
      }
      if (!ok) break;
      hg += H;
      // hand l over: the output warpgroup reads it before it releases O
      // (o_free), which the next item's first PV waits for
      l_buf[u * 128 + r] = l;
      mbar_arrive(&b.l_full);
    }
  } else {
    // -------------------------------------------------------------- output
    // Rounds of items, one of each tile.  Per tile u:
    //   A(u): once the softmax has finished the item (l_full), A of the
    //         linear part goes to TMEM (a_full);
    //   E(u): once O is final (o_full), the epilogue O / l -> out (o_free).
    // Order: A(0), A(1) if tile 1 is already done, E(0), A(1) otherwise,
    // E(1), then den of both tiles' next items, which no tile waits for then:
    // tile 0's next first PV (o_free) never waits for tile 1.
    const int r = tid - 384;                        // query row inside a tile = TMEM lane
    const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
    uint32_t hgs[2] = {0u, 0u};
    float den[2] = {0.f, 0.f}, lrow[2] = {1.f, 1.f};
    bool ok = true;
    int it = 0;
    auto row_of = [&](int u, int round, int& bh, int& i, long long& n) {
      const int item = blockIdx.x + u * gridDim.x + round * tiles_total;
      bh = item / NB;
      i = item % NB;
      n = (long long)i * BLK + r;
      return r < BLK && n < p.N;                    // a row of the output
    };
    // tile 1's item of a round lies G items past tile 0's, so it has one only
    // in rounds where tile 0 has one too
    auto has = [&](int u, int round) { return blockIdx.x + u * gridDim.x + round * tiles_total < p.items; };
    auto make_dens = [&](int round) {
#pragma unroll
      for (int u = 0; u < 2; ++u)
        if (has(u, round)) {
          int bh, i;
          long long n;
          const bool valid = row_of(u, round, bh, i, n);
          den[u] = linear_den<D>(p.q + ((long long)bh * p.N + (valid ? n : 0)) * D,
                                 p.zrest + ((long long)bh * NB + i) * D, valid);
        }
    };
    // A of tile u (after its softmax); false if a wait gave up
    auto do_a = [&](int u) -> bool {
      TileBars& b = bars[u];
      const int H = halves_of((blockIdx.x + u * gridDim.x + it * tiles_total) / NB);
      if (sparse) {
        if (!mbar_wait(&b.l_full, it & 1, abort_flag)) return false;
        lrow[u] = l_buf[u * 128 + r];
      }
      if (lin) {
        int bh, i;
        long long n;
        const bool valid = row_of(u, it, bh, i, n);
        // A = bf16(phi(q) * l / den) into the S buffer of half hg + H, once
        // the PV that last read that buffer (half hg + H - 2 of this item) is
        // done; an earlier reader finished before the previous o_full
        const float sc = (valid && den[u] > 0.f) ? lrow[u] / den[u] : 0.f;
        const uint4* qr = reinterpret_cast<const uint4*>(p.q + ((long long)bh * p.N + (valid ? n : 0)) * D);
        uint32_t a[D / 2];
#pragma unroll
        for (int c8 = 0; c8 < D / 8; ++c8) {
          const uint4 raw = valid ? __ldg(qr + c8) : make_uint4(0, 0, 0, 0);
          a[4 * c8] = raw.x;
          a[4 * c8 + 1] = raw.y;
          a[4 * c8 + 2] = raw.z;
          a[4 * c8 + 3] = raw.w;
        }
#pragma unroll
        for (int c = 0; c < D / 2; ++c)
          a[c] = pack_bf16x2(phi_bf16(uint16_t(a[c])) * sc, phi_bf16(uint16_t(a[c] >> 16)) * sc);
        if (H >= 2) {
          const uint32_t gp = hgs[u] + H - 2;
          if (!mbar_wait(&b.pv_done[gp & 1], (gp >> 1) & 1, abort_flag)) return false;
        }
        tc_fence_after();
        const uint32_t abuf = tmem_base + u * 256 + lane_off + ((hgs[u] + H) & 1) * 64;
#pragma unroll
        for (int c = 0; c < D / 2; c += 16) SLA_TMEM_ST16(abuf + c, (a + c));
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&b.a_full);
      }
      hgs[u] += H;
      return true;
    };
    // epilogue of tile u; false if the wait gave up
    auto do_e = [&](int u) -> bool {
      TileBars& b = bars[u];
      if (!mbar_wait(&b.o_full, it & 1, abort_flag)) return false;
      tc_fence_after();
      int bh, i;
      long long n;
      const bool valid = row_of(u, it, bh, i, n);
      const uint32_t tO = tmem_base + u * 256 + lane_off + 128;
      const float inv_l = 1.f / lrow[u];
      const long long obase = ((long long)bh * p.N + n) * D;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t w[32];
        SLA_TMEM_LD32(tO + ch * 32, w);
        tmem_ld_wait();
        if (valid) {
          if (p.out_f32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + obase + ch * 32);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              dst[q] = make_float4(__uint_as_float(w[4 * q]) * inv_l, __uint_as_float(w[4 * q + 1]) * inv_l,
                                   __uint_as_float(w[4 * q + 2]) * inv_l, __uint_as_float(w[4 * q + 3]) * inv_l);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + obase + ch * 32);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dst[q] = make_uint4(
                  pack_bf16x2(__uint_as_float(w[8 * q]) * inv_l, __uint_as_float(w[8 * q + 1]) * inv_l),
                  pack_bf16x2(__uint_as_float(w[8 * q + 2]) * inv_l, __uint_as_float(w[8 * q + 3]) * inv_l),
                  pack_bf16x2(__uint_as_float(w[8 * q + 4]) * inv_l, __uint_as_float(w[8 * q + 5]) * inv_l),
                  pack_bf16x2(__uint_as_float(w[8 * q + 6]) * inv_l, __uint_as_float(w[8 * q + 7]) * inv_l));
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&b.o_free);
      return true;
    };
    if (lin) make_dens(0);
    for (; ok && has(0, it); ++it) {
      const bool t1 = has(1, it);
      ok = do_a(0);
      bool a1 = false;
      if (ok && t1 && (!sparse || __all_sync(0xffffffffu, mbar_test_wait(&bars[1].l_full, it & 1)))) {
        ok = do_a(1);
        a1 = true;
      }
      ok = ok && do_e(0);
      if (ok && t1 && !a1) ok = do_a(1);
      if (ok && t1) ok = do_e(1);
      if (ok && lin) make_dens(it + 1);
    }
  }

  __syncwarp();   // reconverge the single-lane roles before the CTA barrier
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem_base, 512);
}

}  // namespace sla
