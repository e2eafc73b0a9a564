// W8A8 linear layer with 128x128 block quantisation.
//
// "Turbo Diffusion：秒级生成与高清保真的视频扩散技术突破", section 三(四) item 1:
// weights and activations of the linear layers in 8 bits, one set of
// quantisation parameters per 128x128 block, activations quantised at run
// time; the chooseai.net news page (linear-layer acceleration) puts both
// parameters and activations on 128x128 blocks.  Y = X . W^T (+ bias) with
// X [M, K] and W [N, K] (out_features x in_features):
//   scale of a block s = float32(max|x| / 127), code = clamp(rne(x / s), +-127)
//   (the attention quantiser's rule, k_quant.cuh);
//   Y[m, n] = sum over 128-column blocks kb of P_kb[m, n] * (sx[m/128][kb] *
//   sw[n/128][kb]), P_kb the exact int32 sum of the int8 products of block kb,
//   accumulated in float32 in the order of kb, + bias[n], stored as bf16
//   (round to nearest even) or float32.
//
// k_quant2d: one CTA per 128x128 block: the bf16 tile by one TMA load, pass 1
// the maximum, pass 2 the codes.
//
// k_w8a8_gemm: persistent, one CTA per SM, output tiles of 128 rows x 256
// columns (the width is a template parameter; 128 and 192 were slower: more
// operand traffic per product, or register spills).  Per k-block one tcgen05.mma kind::i8 product (M 128, N 256, K
// 128 as four K=32 instructions) goes into one of two 256-column TMEM buffers;
// the promotion warps read it, scale it and add it into float32 accumulators
// in registers while the tensor core fills the other buffer.  The int32 sums
// are read as floats without a conversion instruction: each buffer is
// pre-loaded with the bits of 1.5 * 2^23 (0x4B400000) and the products are
// accumulated onto it, so the int32 result is the bit pattern of the float
// 1.5 * 2^23 + P, exact because |P| <= 128 * 127^2 < 2^22; one subtraction
// recovers P and one fused multiply-add adds P * s: two float32 operations
// per element, the subtraction packed in pairs (packed forms run on one half
// of the FMA pipe only) and the multiply-adds scalar (either half).
//   warp 0  TMA producer (A: 128 x 128 int8, B: 256 x 128 int8 per stage)
//   warp 1  TMEM allocation and the MMA issuer (warps 2-3 idle)
//   warps 4-11 promotion and epilogue: warp w owns TMEM lanes 32 (w % 4) ..
//           (tile rows) and columns 128 ((w - 4) / 4) .. of the tile
// Registers: 168 per thread at launch (384 x 168); setmaxnreg moves the
// first warpgroup to 40 and the two promotion warpgroups to 232 (128 x 40 +
// 256 x 232 = 384 x 168), room for 128 float32 accumulators per thread.
#pragma once
#include <cuda_bf16.h>
#include "k_quant.cuh"
#include "sm100.cuh"

namespace sla {

// ------------------------------------------------------------------ k_quant2d
constexpr int kQ2Tile = 128;
constexpr int kQ2Bytes = kQ2Tile * kQ2Tile * 2;   // the bf16 tile
constexpr int kQ2Smem = kQ2Bytes + 8 * 4 + 16 + 1024;

__global__ void __launch_bounds__(256) k_quant2d(const __grid_constant__ CUtensorMap tm_x, int R, int K,
                                                int8_t* __restrict__ codes, float* __restrict__ scales) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint16_t* tile = reinterpret_cast<const uint16_t*>(base);   // [128][128] bf16, zero past R, K
  float* wmax = reinterpret_cast<float*>(base + kQ2Bytes);
  uint64_t* bar = reinterpret_cast<uint64_t*>(wmax + 8);
  const int kb = blockIdx.x, rb = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int g = tid & 15;                       // 8-column group
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
    mbar_expect_tx(bar, kQ2Bytes);
    tma_load_2d(base, &tm_x, bar, kb * kQ2Tile, rb * kQ2Tile);
  }
  __syncthreads();
  const bool landed = mbar_wait(bar, 0, nullptr);
  if (!__syncthreads_and(landed)) {
    if (tid == 0) (void)mbar_wait(bar, 0, nullptr);   // the copy lands before the CTA exits
    return;
  }
  float mloc = 0.f;
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    const int r = (tid >> 4) + 16 * t;
    const uint4 raw = *reinterpret_cast<const uint4*>(tile + r * kQ2Tile + g * 8);
    const uint16_t* hv = reinterpret_cast<const uint16_t*>(&raw);
#pragma unroll
    for (int e = 0; e < 8; ++e) mloc = fmaxf(mloc, fabsf(__uint_as_float(uint32_t(hv[e]) << 16)));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, o));
  if ((tid & 31) == 0) wmax[warp] = mloc;
  __syncthreads();
  float m = wmax[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) m = fmaxf(m, wmax[w]);
  const float s = __fdiv_rn(m, 127.0f);
  const int KB = (K + kQ2Tile - 1) / kQ2Tile;
  if (tid == 0) scales[(long long)rb * KB + kb] = s;
  const float rs = (s > 0.f) ? __frcp_rn(s) : 0.f;
  const int col = kb * kQ2Tile + g * 8;
  if (col >= K) return;                         // K is a multiple of 16: a group is all in or all out
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    const int r = (tid >> 4) + 16 * t;
    const long long row = (long long)rb * kQ2Tile + r;
    if (row >= R) break;
    const uint4 raw = *reinterpret_cast<const uint4*>(tile + r * kQ2Tile + g * 8);
    const uint16_t* hv = reinterpret_cast<const uint16_t*>(&raw);
    uint32_t packed[2] = {0u, 0u};
    if (s > 0.f) {
      int qv[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) qv[e] = quant_code(__uint_as_float(uint32_t(hv[e]) << 16), s, rs);
      packed[0] = pack_i8x4(qv[0], qv[1], qv[2], qv[3]);
      packed[1] = pack_i8x4(qv[4], qv[5], qv[6], qv[7]);
    }
    *reinterpret_cast<uint2*>(codes + row * K + col) = make_uint2(packed[0], packed[1]);
  }
}

// ------------------------------------------------------------------ k_w8a8_gemm
struct W8A8Params {
  const float* sx;                 // [ceil(M/128)][KB]
  const float* sw;                 // [ceil(N/128)][KB]
  const __nv_bfloat16* bias;       // [N] or nullptr
  void* y;                         // [M][N] bf16 or float32
  int M, N, K, KB;                 // KB = ceil(K / 128) k-blocks
  int tiles_n, tiles;              // tiles of 128 x BN
  int out_f32;
};

constexpr uint32_t kMagicBits = 0x4B400000u;        // 1.5 * 2^23
constexpr int kW8TileN = 256;                        // output tile width BN
constexpr int kW8Buffers = 2;                        // TMEM buffers (k-blocks in flight)

// BN-column tiles, NBUF TMEM buffers of BN columns, 8 promotion warps of
// BN / 2 columns each (32 TMEM lanes x BN / 2 columns) read CW columns at a
// time; threads and register split.
template <int BN, int NBUF>
struct W8Cfg {
  static constexpr int STAGES = BN >= 256 ? 4 : 5;
  static constexpr int A_BYTES = 128 * 128;          // X tile: 128 rows x 128 k (int8)
  static constexpr int B_BYTES = BN * 128;           // W tile: BN rows x 128 k
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int BAR_BYTES = (2 * STAGES + 2 * NBUF + 1) * 8 + 16;
  static constexpr int SMEM_USED = STAGES * STAGE_BYTES + BAR_BYTES;
  static constexpr int SMEM = SMEM_USED + 1024;
  static constexpr int THREADS = 384;                // warpgroup 0: producer, MMA; 1-2: promotion
  static constexpr int COLS = BN / 2;                // columns per promotion warp
  static constexpr int CW = COLS % 32 == 0 ? 32 : 16; // columns per TMEM load
  static constexpr int NCH = COLS / CW;              // TMEM loads per k-block
  static constexpr int REGS_LOAD = 40;
  static constexpr int REGS_MATH = 232;
  static_assert(128 * REGS_LOAD + 256 * REGS_MATH <= THREADS * 168, "register split within the launch's");
  static_assert(BN % 32 == 0 && BN <= 256 && NBUF * BN <= 512, "tile halves of whole chunks; buffers fit TMEM");
  static_assert(SMEM <= 232448, "stages fit in shared memory");
};

// The same 32-bit value into 32 (16) consecutive TMEM columns of the warp's 32 lanes.
__device__ __forceinline__ void tmem_fill32(uint32_t taddr, uint32_t x) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,"
      "%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(taddr),
      "r"(x)
      : "memory");
}
__device__ __forceinline__ void tmem_fill16(uint32_t taddr, uint32_t x) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1,%1};" ::"r"(
                   taddr),
               "r"(x)
               : "memory");
}
template <int CW>
__device__ __forceinline__ void tmem_fill_cols(uint32_t taddr, uint32_t x) {
  if constexpr (CW == 32) tmem_fill32(taddr, x);
  else tmem_fill16(taddr, x);
}
template <int CW>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t* r) {
  if constexpr (CW == 32) {
    SLA_TMEM_LD32(taddr, r);
  } else {
    SLA_TMEM_LD16(taddr, r);
  }
}

template <int BN, int NBUF>
__global__ void __launch_bounds__(W8Cfg<BN, NBUF>::THREADS, 1) k_w8a8_gemm(const __grid_constant__ CUtensorMap tm_a,
                                                                           const __grid_constant__ CUtensorMap tm_b,
                                                                           const W8A8Params p) {
  using C = W8Cfg<BN, NBUF>;
  constexpr int CW = C::CW;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if (uint32_t(base - smem_raw) + C::SMEM_USED > dynamic_smem_bytes()) {
    if (threadIdx.x == 0) raise_error(DEV_ERR_LAYOUT);
    return;   // uniform: every thread sees the same base
  }
  uint64_t* full = reinterpret_cast<uint64_t*>(base + C::STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* t_full = empty + C::STAGES;     // [NBUF] a k-block's product is in TMEM buffer b
  uint64_t* t_empty = t_full + NBUF;        // [NBUF] buffer b was read and re-armed with the magic bits
  uint64_t* drain = t_empty + NBUF;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  auto stage = [&](int s) { return base + s * C::STAGE_BYTES; };

  if (tid == 0) {
    for (int q = 0; q < C::STAGES; ++q) {
      mbar_init(&full[q], 1);
      mbar_init(&empty[q], 1);
    }
    for (int q = 0; q < NBUF; ++q) {
      mbar_init(&t_full[q], 1);
      mbar_init(&t_empty[q], 256);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the register split and the roles in one branch each, so that the
  // promotion code is only reachable with the larger register count
  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::REGS_LOAD));
    if (warp == 0) {
      // ------------------------------------------------------------ TMA producer
      if (lane == 0) {
        tma_prefetch_desc(&tm_a);
        tma_prefetch_desc(&tm_b);
        uint32_t n = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < p.tiles && ok; t += gridDim.x) {
          const int m0 = (t / p.tiles_n) * 128, n0 = (t % p.tiles_n) * BN;
          for (int kb = 0; kb < p.KB; ++kb, ++n) {
            const int s = n % C::STAGES;
            if (!(ok = mbar_wait(&empty[s], ((n / C::STAGES) & 1) ^ 1, abort_flag))) break;
            mbar_expect_tx(&full[s], C::STAGE_BYTES);
            tma_load_2d(stage(s), &tm_a, &full[s], kb * 128, m0);
            tma_load_2d(stage(s) + C::A_BYTES, &tm_b, &full[s], kb * 128, n0);
          }
        }
        // loads still in flight (only after a failed wait) land before the CTA exits
        for (uint32_t q = n > C::STAGES ? n - C::STAGES : 0; q < n; ++q)
          (void)mbar_wait(&full[q % C::STAGES], (q / C::STAGES) & 1, nullptr);
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        const uint32_t idesc = idesc_i8(BN);
        uint32_t n = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < p.tiles && ok; t += gridDim.x) {
          for (int kb = 0; kb < p.KB; ++kb, ++n) {
            const int s = n % C::STAGES;
            const uint32_t b = n % NBUF;
            if (!(ok = mbar_wait(&t_empty[b], (n / NBUF) & 1, abort_flag))) break;
            if (!(ok = mbar_wait(&full[s], (n / C::STAGES) & 1, abort_flag))) break;
            tc_fence_after();
            const uint64_t da = smem_desc(smem_u32(stage(s)), 16, 1024, 2);
            const uint64_t db = smem_desc(smem_u32(stage(s) + C::A_BYTES), 16, 1024, 2);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)   // accumulate onto the magic bits
              mma_i8_ss(tmem + b * BN, da + uint64_t(kk * 2), db + uint64_t(kk * 2), idesc, 1u);
            tc_commit(&empty[s]);
            tc_commit(&t_full[b]);
          }
        }
        // every MMA issued here finishes before the CTA frees TMEM (bounded)
        tc_commit(drain);
        (void)mbar_wait(drain, 0, nullptr);
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::REGS_MATH));
    // ------------------------------------------------------------ promotion + epilogue
    const int q4 = warp & 3;                       // TMEM lane quarter
    const int cbase = ((warp - 4) >> 2) * C::COLS; // first tile column of the warp
    const int r = q4 * 32 + lane;                  // tile row
    const uint32_t lane_off = uint32_t(q4 * 32) << 16;
    // arm every buffer
#pragma unroll
    for (int b = 0; b < NBUF; ++b)
#pragma unroll
      for (int c = 0; c < C::NCH; ++c) tmem_fill_cols<CW>(tmem + lane_off + b * BN + cbase + c * CW, kMagicBits);
    tmem_st_wait();
    tc_fence_before();
#pragma unroll
    for (int b = 0; b < NBUF; ++b) mbar_arrive(&t_empty[b]);
    const uint64_t negc2 = f32x2(-12582912.f, -12582912.f);
    uint32_t n = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.tiles && ok; t += gridDim.x) {
      const int m0 = (t / p.tiles_n) * 128, n0 = (t % p.tiles_n) * BN;
      const float* sxr = p.sx + (long long)(m0 >> 7) * p.KB;
      // W scale rows of the warp's columns: the first chunk's block and, when
      // the warp's columns cross into the next 128-column block, that one (a
      // 32-column chunk never crosses a block boundary)
      const int col0 = n0 + cbase;
      const int split = ((col0 >> 7) + 1) * 128 - col0;   // columns in the first block
      const float* swa = p.sw + (long long)(col0 < p.N ? col0 >> 7 : 0) * p.KB;
      const float* swb = p.sw + (long long)(col0 + split < p.N ? (col0 >> 7) + 1 : 0) * p.KB;
      float acc[C::COLS];
#pragma unroll
      for (int e = 0; e < C::COLS; ++e) acc[e] = 0.f;
      float sxn = __ldg(sxr), swan = __ldg(swa), swbn = __ldg(swb);
      for (int kb = 0; kb < p.KB; ++kb, ++n) {
        // one float32 rounding of each scale product
        const float sca = sxn * swan, scb = sxn * swbn;
        if (kb + 1 < p.KB) {
          sxn = __ldg(sxr + kb + 1);
          swan = __ldg(swa + kb + 1);
          swbn = __ldg(swb + kb + 1);
        }
        const uint32_t b = n % NBUF;
        if (!(ok = mbar_wait(&t_full[b], (n / NBUF) & 1, abort_flag))) break;
        tc_fence_after();
        const uint32_t tb = tmem + lane_off + b * BN + cbase;
        // P of a pair exactly by one packed subtraction (the packed forms run on
        // one half of the FMA pipe), then two scalar fused multiply-adds (either half)
        auto add_chunk = [&](const uint32_t* w, int c) {
          const float scc = c * CW < split ? sca : scb;
#pragma unroll
          for (int e = 0; e < CW; e += 2) {
            float p0, p1;
            f32x2_split(add_f32x2(f32x2(__uint_as_float(w[e]), __uint_as_float(w[e + 1])), negc2), p0, p1);
            acc[c * CW + e] = fmaf(p0, scc, acc[c * CW + e]);
            acc[c * CW + e + 1] = fmaf(p1, scc, acc[c * CW + e + 1]);
          }
        };
        // chunk c + 1 is read from TMEM while chunk c is added up; each chunk
        // is re-armed once read, and the buffer released before the last
        // chunk's arithmetic
        uint32_t v[2][CW];
        tmem_ld_cols<CW>(tb, v[0]);
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) {
          tmem_ld_wait();
          if (c + 1 < C::NCH) tmem_ld_cols<CW>(tb + (c + 1) * CW, v[(c + 1) & 1]);
          tmem_fill_cols<CW>(tb + c * CW, kMagicBits);
          if (c == C::NCH - 1) {
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&t_empty[b]);
          }
          add_chunk(v[c & 1], c);
        }
      }
      if (!ok) break;
      // epilogue: + bias, store the row's columns
      const long long row = (long long)m0 + r;
      const int c0 = n0 + cbase;
      if (row < p.M && c0 < p.N) {
        const int ncols = min(C::COLS, p.N - c0);   // a multiple of 16
#pragma unroll
        for (int c = 0; c < C::COLS; c += 16) {
          if (c >= ncols) break;
          float o[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] = acc[c + e];
          if (p.bias != nullptr) {
            const uint4* bp = reinterpret_cast<const uint4*>(p.bias + c0 + c);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const uint4 raw = __ldg(bp + hh);
              const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                o[hh * 8 + 2 * e] += __uint_as_float(w4[e] << 16);
                o[hh * 8 + 2 * e + 1] += __uint_as_float(w4[e] & 0xFFFF0000u);
              }
            }
          }
          if (p.out_f32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.y) + row * p.N + c0 + c);
#pragma unroll
            for (int e = 0; e < 4; ++e) dst[e] = make_float4(o[4 * e], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.y) + row * p.N + c0 + c);
            dst[0] = make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                                pack_bf16x2(o[6], o[7]));
            dst[1] = make_uint4(pack_bf16x2(o[8], o[9]), pack_bf16x2(o[10], o[11]), pack_bf16x2(o[12], o[13]),
                                pack_bf16x2(o[14], o[15]));
          }
        }
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace sla
