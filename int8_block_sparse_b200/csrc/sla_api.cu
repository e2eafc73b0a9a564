// C interface of the SageSLA attention library: argument checks, temporary
// device memory, TMA descriptors and the launch sequence of the kernels
//   K1 k_kstats        K block sums + linear states          (k_stats.cuh)
//      k_channel_mean  mu                                   (k_stats.cuh)
//   K2 k_quant         smoothing + INT8 codes + Q block sums (k_quant.cuh)
//   K3 k_mask          pooled scores + top-k                 (k_mask.cuh)
//   K5 k_lingemm       sums of the non-selected states       (k_linear.cuh)
//   K4 k_attn          critical-block attention + linear part (k_attn.cuh)
// and of the W8A8 linear layer
//      k_quant2d       128x128 block quantisation               (k_w8a8.cuh)
//      k_w8a8_gemm     block-scaled INT8 GEMM                   (k_w8a8.cuh)
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "sla.h"
#include "k_attn.cuh"
#include "k_linear.cuh"
#include "k_mask.cuh"
#include "k_quant.cuh"
#include "k_stats.cuh"
#include "k_w8a8.cuh"

using namespace sla;

namespace {

// ------------------------------------------------------------------ helpers
struct Shape {
  int B, H, N, d, block;
  long long BH, NB, NP, kc;
  int gshift;   // log2 of the tokens per quantisation scale (the block by default)
  long long G() const { return (long long)block >> gshift; }
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_shape(int B, int H, int N, int d, int block, Shape* s) {
  if (B < 1 || H < 1 || N < 1 || d < 1 || block < 1) return SLA_ERR_INVALID_ARG;
  if (!(d == 64 || d == 128) || !(block == 64 || block == 128)) return SLA_ERR_UNSUPPORTED;
  s->B = B; s->H = H; s->N = N; s->d = d; s->block = block;
  s->gshift = block == 128 ? 7 : 6;
  s->BH = (long long)B * H;
  s->NB = (N + block - 1) / block;
  s->NP = s->NB * block;
  if (s->BH > 65535 || s->NB > 16384) return SLA_ERR_UNSUPPORTED;
  if (s->BH * s->NP >= (1LL << 31)) return SLA_ERR_UNSUPPORTED;
  return SLA_OK;
}

long long topk_count_ll(long long nblk, float frac) {
  const double kc = std::ceil((double)frac * (double)nblk);
  if (kc < 1.0) return 1;
  if (kc > (double)nblk) return nblk;
  return (long long)kc;
}

bool frac_ok(float f) { return f > 0.f && f <= 1.f; }

// Tokens per quantisation scale: 32, 64 or 128, dividing the block.
int set_gran(Shape* s, int gran) {
  if (!(gran == 32 || gran == 64 || gran == 128)) return SLA_ERR_UNSUPPORTED;
  if (gran > s->block) return SLA_ERR_UNSUPPORTED;
  s->gshift = gran == 32 ? 5 : (gran == 64 ? 6 : 7);
  return SLA_OK;
}
bool skip_ok(float f) { return f >= 0.f && f < 1.f; }

long long skip_count_ll(long long nblk, long long kc, float frac) {
  const double kn = std::floor((double)frac * (double)nblk);
  return std::min<long long>((long long)kn, nblk - kc);
}

// Counts of the two-class mask: every head keeps kc blocks.
HeadCounts uniform_counts(long long kc) {
  HeadCounts hc;
  std::memset(&hc, 0, sizeof(hc));
  hc.H = 1;
  hc.kcp = (int)kc;
  hc.kc[0] = (uint16_t)kc;
  return hc;
}

// Per-head counts (topk_frac[h], skip_frac[h] or 0); SLA_OK or an error code.
int head_counts(long long nblk, int H, const float* topk_frac, const float* skip_frac, HeadCounts* hc,
                bool* linear) {
  if (topk_frac == nullptr) return SLA_ERR_INVALID_ARG;
  if (H > kMaxHeadCounts) return SLA_ERR_UNSUPPORTED;
  std::memset(hc, 0, sizeof(*hc));
  hc->H = H;
  hc->classes = 1;
  *linear = false;
  for (int h = 0; h < H; ++h) {
    if (!frac_ok(topk_frac[h])) return SLA_ERR_INVALID_ARG;
    const float sf = skip_frac != nullptr ? skip_frac[h] : 0.f;
    if (!skip_ok(sf)) return SLA_ERR_INVALID_ARG;
    const long long kc = topk_count_ll(nblk, topk_frac[h]);
    const long long kn = skip_count_ll(nblk, kc, sf);
    hc->kc[h] = (uint16_t)kc;
    hc->kn[h] = (uint16_t)kn;
    hc->kcp = std::max(hc->kcp, (int)kc);
    *linear = *linear || kc + kn < nblk;
  }
  return SLA_OK;
}

// ------------------------------------------------------------------ TMA descriptors
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool make_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* ptr, const cuuint64_t* dims,
              const cuuint64_t* strides_bytes, const cuuint32_t* box, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, dt, (cuuint32_t)rank, const_cast<void*>(ptr), dims, strides_bytes, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ temporary memory
// One stream-ordered pool per device that keeps its memory between calls.
cudaMemPool_t pool_for_current_device() {
  static std::mutex mu;
  static cudaMemPool_t pools[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (pools[dev] == nullptr) {
    cudaMemPoolProps props;
    std::memset(&props, 0, sizeof(props));
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t p = nullptr;
    if (cudaMemPoolCreate(&p, &props) != cudaSuccess) return nullptr;
    uint64_t thr = UINT64_MAX;
    cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &thr);
    pools[dev] = p;
  }
  return pools[dev];
}

struct Arena {
  char* base = nullptr;
  size_t off = 0, cap = 0;
  template <class T>
  T* take(size_t count) {
    const size_t bytes = (count * sizeof(T) + 255) & ~size_t(255);
    T* p = reinterpret_cast<T*>(base + off);
    off += bytes;
    return p;
  }
};

template <class T>
size_t rounded(size_t count) { return (count * sizeof(T) + 255) & ~size_t(255); }

struct Workspace {
  double* ksum; double* kbar; uint8_t* kexp; float* mu; double* qbar;
  int8_t* qi8; int8_t* ki8; float* sq; float* sk; int32_t* idx; int* kc_bh;
  __nv_bfloat16* notcrit; __nv_bfloat16* hstate; __nv_bfloat16* grest; float* zrest;
  long long ncpitch, hpitch;
};

// what: bit 0 quant outputs, bit 1 mask, bit 2 attention, bit 3 linear branch
size_t workspace_bytes(const Shape& s, int what) {
  const size_t BH = s.BH, NB = s.NB, NP = s.NP, d = s.d, kc = s.kc;
  const size_t ncpitch = (NB + 63) / 64 * 64, hpitch = d * d + d;
  size_t b = rounded<double>(BH * NB * d) * 2 + rounded<double>(BH * d * (size_t)kbar_pitch((int)NB)) +
             rounded<uint8_t>(BH * NB * d * 2) + rounded<float>(BH * d);
  if (what & 1) b += rounded<int8_t>(BH * NP * d) * 2 + rounded<float>(BH * NB * (size_t)s.G()) * 2;
  if (what & 2) b += rounded<int32_t>(BH * NB * kc) + rounded<int>(BH);
  if (what & 8)
    b += rounded<__nv_bfloat16>(BH * NB * ncpitch) + rounded<__nv_bfloat16>(BH * NB * hpitch) +
         rounded<__nv_bfloat16>(BH * NB * d * d) + rounded<float>(BH * NB * d);
  return b;
}

Workspace carve(const Shape& s, int what, char* base) {
  Arena a;
  a.base = base;
  Workspace w{};
  const size_t BH = s.BH, NB = s.NB, NP = s.NP, d = s.d, kc = s.kc;
  w.ncpitch = (NB + 63) / 64 * 64;
  w.hpitch = d * d + d;
  w.ksum = a.take<double>(BH * NB * d);
  w.kbar = a.take<double>(BH * d * (size_t)kbar_pitch((int)NB));
  w.qbar = a.take<double>(BH * NB * d);
  w.kexp = a.take<uint8_t>(BH * NB * d * 2);
  w.mu = a.take<float>(BH * d);
  if (what & 1) {
    w.qi8 = a.take<int8_t>(BH * NP * d);
    w.ki8 = a.take<int8_t>(BH * NP * d);
    w.sq = a.take<float>(BH * NB * (size_t)s.G());
    w.sk = a.take<float>(BH * NB * (size_t)s.G());
  }
  if (what & 2) {
    w.idx = a.take<int32_t>(BH * NB * kc);
    w.kc_bh = a.take<int>(BH);
  }
  if (what & 8) {
    w.notcrit = a.take<__nv_bfloat16>(BH * NB * w.ncpitch);
    w.hstate = a.take<__nv_bfloat16>(BH * NB * w.hpitch);
    w.grest = a.take<__nv_bfloat16>(BH * NB * d * d);
    w.zrest = a.take<float>(BH * NB * d);
  }
  return w;
}

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return SLA_OK;
  if (e == cudaErrorMemoryAllocation) return SLA_ERR_OOM;
  return SLA_ERR_CUDA;
}

// ------------------------------------------------------------------ optional per-kernel timing
struct ProfRecord {
  int kind;
  cudaEvent_t a, b;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRecord> g_prof;

// Records an event before the launch that follows and one after it (at scope exit).
struct ProfScope {
  int kind;
  cudaStream_t st;
  cudaEvent_t a = nullptr, b = nullptr;
  ProfScope(int k, cudaStream_t s) : kind(k), st(s) {
    if (!g_prof_on) return;
    if (cudaEventCreate(&a) != cudaSuccess || cudaEventCreate(&b) != cudaSuccess) return;
    cudaEventRecord(a, st);
  }
  ~ProfScope() {
    if (a == nullptr || b == nullptr) return;
    cudaEventRecord(b, st);
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof.push_back({kind, a, b});
  }
};

// ------------------------------------------------------------------ launch helpers
int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

// K block sums and (states) the linear states (k_kstats), then mu (k_channel_mean).
template <int D, int BLK>
int launch_kstats(const Shape& s, const __nv_bfloat16* k, const __nv_bfloat16* v, const __nv_bfloat16* proj,
                  Workspace& w, bool states, cudaStream_t st, cudaEvent_t after_stats = nullptr) {
  CUtensorMap mv, mw;
  std::memset(&mv, 0, sizeof(mv));
  std::memset(&mw, 0, sizeof(mw));
  if (states) {
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)s.N, (cuuint64_t)s.BH};
    cuuint64_t str[2] = {(cuuint64_t)D * 2, (cuuint64_t)s.N * D * 2};
    cuuint32_t box[3] = {64u, (cuuint32_t)BLK, 1u};
    if (!make_map(&mv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, v, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return SLA_ERR_CUDA;
    cuuint64_t wd[2] = {(cuuint64_t)D, (cuuint64_t)D};
    cuuint64_t ws[1] = {(cuuint64_t)D * 2};
    cuuint32_t wb[2] = {64u, (cuuint32_t)D};
    if (!make_map(&mw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, proj, wd, ws, wb, CU_TENSOR_MAP_SWIZZLE_128B))
      return SLA_ERR_CUDA;
  }
  const int sm1 = StatsCfg<D, BLK>::SMEM;
  cudaFuncSetAttribute(k_kstats<D, BLK>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm1);
  dim3 g1((unsigned)s.NB, (unsigned)s.BH);
  { ProfScope ps(SLA_K_STATS, st);
  k_kstats<D, BLK><<<g1, StatsCfg<D, BLK>::THREADS, sm1, st>>>(mv, mw, k, w.ksum, w.kbar, w.kexp, states ? w.hstate : nullptr, s.N,
                                         (int)s.NB, w.hpitch); }
  if (after_stats != nullptr && cudaEventRecord(after_stats, st) != cudaSuccess) return SLA_ERR_CUDA;
  { ProfScope ps(SLA_K_MEAN, st);
  k_channel_mean<D><<<dim3((unsigned)s.BH, D / kMeanCG), 1024, 0, st>>>(w.ksum, w.kexp, k, w.mu, (int)s.NB, s.N); }
  return cuda_status(cudaGetLastError());
}

// Codes, scales (and for Q the pooled blocks) of Q (which & 1) and of K - mu
// (which & 2; needs mu) in one launch.
template <int D, int BLK>
int launch_quant(const Shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k, Workspace& w, int which,
                 int8_t* qi8, int8_t* ki8, float* sq, float* sk, cudaStream_t st) {
  CUtensorMap mq, mk;
  {
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)s.N, (cuuint64_t)s.BH};
    cuuint64_t str[2] = {(cuuint64_t)D * 2, (cuuint64_t)s.N * D * 2};
    cuuint32_t box[3] = {(cuuint32_t)D, (cuuint32_t)BLK, 1u};
    if (!make_map(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, q, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE))
      return SLA_ERR_CUDA;
    if (!make_map(&mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, k, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE))
      return SLA_ERR_CUDA;
  }
  const int sm2 = QuantCfg<D, BLK>::SMEM;
  dim3 g2((unsigned)s.NB, (unsigned)s.BH, which == 3 ? 2u : 1u);
  const bool fine = s.G() > 1;
  auto kq = fine ? k_quant<D, BLK, true> : k_quant<D, BLK, false>;
  cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, sm2);
  { ProfScope ps(SLA_K_QUANT, st);
  kq<<<g2, 256, sm2, st>>>(mq, mk, w.mu, qi8, ki8, sq, sk, w.qbar, s.N, (int)s.NB, which == 2 ? 1 : 0, s.gshift); }
  return cuda_status(cudaGetLastError());
}

// Both, in order (the entry points that need no overlap).
template <int D, int BLK>
int launch_stats_quant(const Shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v,
                       const __nv_bfloat16* proj, Workspace& w, bool states, bool kcodes, int8_t* qi8,
                       int8_t* ki8, float* sq, float* sk, cudaStream_t st) {
  const int rc = launch_kstats<D, BLK>(s, k, v, proj, w, states, st);
  if (rc) return rc;
  return launch_quant<D, BLK>(s, q, k, w, kcodes ? 3 : 1, qi8, ki8, sq, sk, st);
}

template <int D, int R>
int launch_mask_rows(const Shape& s, Workspace& w, const HeadCounts& hc, int* kc_bh, int32_t* idx, uint8_t* bitmap,
                     __nv_bfloat16* notcrit, cudaStream_t st) {
  // kbar as a 2-D float64 tensor [BH * D rows][NB key blocks]; slabs of 16 rows x 256
  CUtensorMap mkb;
  {
    cuuint64_t dims[2] = {(cuuint64_t)s.NB, (cuuint64_t)(s.BH * D)};
    cuuint64_t str[1] = {(cuuint64_t)kbar_pitch((int)s.NB) * 8};
    cuuint32_t box[2] = {256u, (cuuint32_t)kMaskSlabCh};
    if (!make_map(&mkb, CU_TENSOR_MAP_DATA_TYPE_FLOAT64, 2, w.kbar, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE))
      return SLA_ERR_CUDA;
  }
  const size_t sm = mask_smem<D>(R, (int)s.NB);
  cudaFuncSetAttribute(k_mask<D, R>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  dim3 g((unsigned)((s.NB + R - 1) / R), (unsigned)s.BH);
  ProfScope ps(SLA_K_MASK, st);
  k_mask<D, R><<<g, 256, sm, st>>>(mkb, w.qbar, (int)s.NB, hc, kc_bh, idx, bitmap, notcrit, (int)w.ncpitch);
  return cuda_status(cudaGetLastError());
}

template <int D>
int launch_mask(const Shape& s, Workspace& w, const HeadCounts& hc, int* kc_bh, int32_t* idx, uint8_t* bitmap,
                __nv_bfloat16* notcrit, cudaStream_t st) {
  // rows per CTA: 8 unless the R x NB float64 scores would not fit
  const size_t lim = 200 * 1024;
  if (mask_smem<D>(8, (int)s.NB) <= lim) return launch_mask_rows<D, 8>(s, w, hc, kc_bh, idx, bitmap, notcrit, st);
  if (mask_smem<D>(4, (int)s.NB) <= lim) return launch_mask_rows<D, 4>(s, w, hc, kc_bh, idx, bitmap, notcrit, st);
  if (mask_smem<D>(2, (int)s.NB) <= lim) return launch_mask_rows<D, 2>(s, w, hc, kc_bh, idx, bitmap, notcrit, st);
  return launch_mask_rows<D, 1>(s, w, hc, kc_bh, idx, bitmap, notcrit, st);
}


// k_attn in one of its modes: sparse (the selected blocks), lin (the linear
// part), out as float32 or bf16.
template <int D, int BLK>
int launch_attn(const Shape& s, Workspace& w, const int* kc_bh, const __nv_bfloat16* q, const __nv_bfloat16* v,
                void* out, bool out_f32, bool sparse, bool lin, cudaStream_t st) {
  using C = AttnCfg<D, BLK>;
  CUtensorMap mq, mk, mv, mg;
  std::memset(&mq, 0, sizeof(mq));
  std::memset(&mk, 0, sizeof(mk));
  std::memset(&mv, 0, sizeof(mv));
  std::memset(&mg, 0, sizeof(mg));
  const CUtensorMapSwizzle ksw = (D == 128) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  if (sparse) {
    cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)(s.BH * s.NP)};
    cuuint64_t str[1] = {(cuuint64_t)D};
    cuuint32_t boxq[2] = {(cuuint32_t)D, 128u};
    cuuint32_t boxk[2] = {(cuuint32_t)D, (cuuint32_t)BLK};
    if (!make_map(&mq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, w.qi8, dims, str, boxq, ksw)) return SLA_ERR_CUDA;
    if (!make_map(&mk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, w.ki8, dims, str, boxk, ksw)) return SLA_ERR_CUDA;
    cuuint64_t vd[3] = {(cuuint64_t)D, (cuuint64_t)s.N, (cuuint64_t)s.BH};
    cuuint64_t vs[2] = {(cuuint64_t)D * 2, (cuuint64_t)s.N * D * 2};
    cuuint32_t vb[3] = {64u, (cuuint32_t)BLK, 1u};
    if (!make_map(&mv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, v, vd, vs, vb, CU_TENSOR_MAP_SWIZZLE_128B))
      return SLA_ERR_CUDA;
  }
  if (lin) {
    cuuint64_t gd[2] = {(cuuint64_t)D, (cuuint64_t)(s.BH * s.NB * D)};
    cuuint64_t gs[1] = {(cuuint64_t)D * 2};
    cuuint32_t gb[2] = {64u, (cuuint32_t)C::LROWS};
    if (!make_map(&mg, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w.grest, gd, gs, gb, CU_TENSOR_MAP_SWIZZLE_128B))
      return SLA_ERR_CUDA;
  }
  AttnParams p;
  p.idx = w.idx; p.sq = w.sq; p.sk = w.sk; p.q = q; p.zrest = w.zrest; p.out = out;
  p.kc_bh = kc_bh;
  p.N = s.N; p.NB = (int)s.NB; p.NP = (int)s.NP; p.kc = (int)s.kc; p.kcp = (int)s.kc; p.items = (int)(s.BH * s.NB);
  p.gshift = s.gshift;
  p.sparse = sparse ? 1 : 0;
  p.lin = lin ? 1 : 0;
  p.out_f32 = out_f32 ? 1 : 0;
  p.qk_scale = (float)(1.4426950408889634 / std::sqrt((double)D));
  auto ka = s.G() > 1 ? k_attn<D, BLK, true> : k_attn<D, BLK, false>;
  cudaFuncSetAttribute(ka, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  const int ctas = (int)std::min<long long>(num_sms(), (p.items + 1) / 2);
  ProfScope ps(SLA_K_ATTN, st);
  ka<<<ctas, kAttnThreads, C::SMEM, st>>>(mq, mk, mv, mg, p);
  return cuda_status(cudaGetLastError());
}

// G'_i and g_i, the sums of the linear states over the blocks query block i
// did not select (k_lingemm), for k_attn's linear part.
template <int D>
int launch_lingemm(const Shape& s, Workspace& w, cudaStream_t st) {
  CUtensorMap ma, mb;
  {
    cuuint64_t dims[3] = {(cuuint64_t)w.ncpitch, (cuuint64_t)s.NB, (cuuint64_t)s.BH};
    cuuint64_t str[2] = {(cuuint64_t)w.ncpitch * 2, (cuuint64_t)(w.ncpitch * s.NB * 2)};
    cuuint32_t box[3] = {64u, 128u, 1u};
    if (!make_map(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, w.notcrit, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return SLA_ERR_CUDA;
  }
  {
    cuuint64_t dims[3] = {(cuuint64_t)w.hpitch, (cuuint64_t)s.NB, (cuuint64_t)s.BH};
    cuuint64_t str[2] = {(cuuint64_t)w.hpitch * 2, (cuuint64_t)(w.hpitch * s.NB * 2)};
    cuuint32_t box[3] = {64u, 64u, 1u};
    if (!make_map(&mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, w.hstate, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return SLA_ERR_CUDA;
  }
  LinGemmParams gp;
  gp.grest = w.grest; gp.zrest = w.zrest; gp.NB = (int)s.NB; gp.D = D; gp.E = D * D + D;
  gp.nkt = (int)((s.NB + 63) / 64);
  gp.mgroups = (int)((s.NB + 255) / 256);
  gp.ntiles = (gp.E + 127) / 128;
  const bool resident = gp.nkt <= LG_MAX_RESIDENT_KT;
  const long long groups = s.BH * gp.mgroups;
  // resident A: the N tiles of a (head, M group) split into runs so that the
  // units number at most one per SM; otherwise one N tile per unit
  const long long runs = resident ? std::max<long long>(1, num_sms() / groups) : gp.ntiles;
  gp.tpu = (int)((gp.ntiles + runs - 1) / runs);
  gp.units = (int)(groups * ((gp.ntiles + gp.tpu - 1) / gp.tpu));
  const int ctas = std::min(num_sms(), gp.units);
  ProfScope ps(SLA_K_LINGEMM, st);
  if (resident) {
    cudaFuncSetAttribute(k_lingemm<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, LinGemmCfg<true>::SMEM);
    k_lingemm<true><<<ctas, LG_THREADS, LinGemmCfg<true>::SMEM, st>>>(ma, mb, gp);
  } else {
    cudaFuncSetAttribute(k_lingemm<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, LinGemmCfg<false>::SMEM);
    k_lingemm<false><<<ctas, LG_THREADS, LinGemmCfg<false>::SMEM, st>>>(ma, mb, gp);
  }
  return cuda_status(cudaGetLastError());
}

// Set by the host-buffer path around its calls: run the operator's kernels
// on the caller's stream only.
thread_local bool t_one_stream = false;

// ------------------------------------------------------------------ second stream of the operator
// The operator's kernels run on two streams of the device: the caller's and
// this one (created at the first call on a device and kept).  Its events
// order the two; the mutex keeps one call's record/wait sequence from
// interleaving with another's.
struct SideStream {
  std::mutex mu;
  cudaStream_t st = nullptr;
  cudaEvent_t fork = nullptr, stats = nullptr, join = nullptr;
};

SideStream* side_stream() {
  static std::mutex mu;
  static SideStream* sets[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (sets[dev] == nullptr) {
    SideStream* x = new SideStream();
    if (cudaStreamCreateWithFlags(&x->st, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&x->fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&x->stats, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&x->join, cudaEventDisableTiming) != cudaSuccess)
      return nullptr;
    sets[dev] = x;
  }
  return sets[dev];
}

// ------------------------------------------------------------------ dispatch
// s.kc is the pitch of the block lists (the largest count of hc); `linear`:
// some query block has blocks in the linear branch.
//
// Two streams: the caller's runs k_kstats, k_channel_mean, the K half of
// k_quant and k_attn; the side stream runs the Q half of k_quant (needs no
// mu: it overlaps k_kstats), then, once k_kstats is done, k_mask and
// k_lingemm (they need the pooled blocks and the states, not mu or the K
// codes: they overlap k_channel_mean and the K quantisation).
template <int D, int BLK>
int run_attn(const Shape& s, const HeadCounts& hc, bool linear, const __nv_bfloat16* q, const __nv_bfloat16* k,
             const __nv_bfloat16* v, const __nv_bfloat16* proj, void* out, bool out_f32, float* o_sparse,
             float* o_lin, Workspace& w, cudaStream_t st) {
  int* kc_bh = hc.H > 1 || hc.kc[0] != s.kc ? w.kc_bh : nullptr;   // per-head list lengths
  int rc = SLA_OK;
  if (t_one_stream) {
    // everything in order on the caller's stream (the host-buffer path
    // overlaps whole chunks of heads on its own streams instead)
    rc = launch_stats_quant<D, BLK>(s, q, k, v, proj, w, linear, true, w.qi8, w.ki8, w.sq, w.sk, st);
    if (rc == SLA_OK) rc = launch_mask<D>(s, w, hc, kc_bh, w.idx, nullptr, linear ? w.notcrit : nullptr, st);
    if (rc == SLA_OK && linear) rc = launch_lingemm<D>(s, w, st);
  } else {
    SideStream* ss = side_stream();
    if (ss == nullptr) return SLA_ERR_CUDA;
    std::lock_guard<std::mutex> lk(ss->mu);
    if (cudaEventRecord(ss->fork, st) != cudaSuccess || cudaStreamWaitEvent(ss->st, ss->fork, 0) != cudaSuccess)
      return SLA_ERR_CUDA;
    rc = launch_quant<D, BLK>(s, q, k, w, 1, w.qi8, w.ki8, w.sq, w.sk, ss->st);
    if (rc == SLA_OK) rc = launch_kstats<D, BLK>(s, k, v, proj, w, linear, st, ss->stats);
    if (rc == SLA_OK && cudaStreamWaitEvent(ss->st, ss->stats, 0) != cudaSuccess) rc = SLA_ERR_CUDA;
    if (rc == SLA_OK) rc = launch_quant<D, BLK>(s, q, k, w, 2, w.qi8, w.ki8, w.sq, w.sk, st);
    if (rc == SLA_OK) rc = launch_mask<D>(s, w, hc, kc_bh, w.idx, nullptr, linear ? w.notcrit : nullptr, ss->st);
    if (rc == SLA_OK && linear) rc = launch_lingemm<D>(s, w, ss->st);
    // the caller's stream waits for the side stream, on every path (its
    // temporary memory is released in the caller's stream order)
    if (cudaEventRecord(ss->join, ss->st) != cudaSuccess || cudaStreamWaitEvent(st, ss->join, 0) != cudaSuccess)
      if (rc == SLA_OK) rc = SLA_ERR_CUDA;
  }
  if (rc) return rc;
  if ((rc = launch_attn<D, BLK>(s, w, kc_bh, q, v, out, out_f32, true, linear, st))) return rc;
  // the two parts on their own, in float32 (inspection and tests)
  if (o_sparse != nullptr && (rc = launch_attn<D, BLK>(s, w, kc_bh, q, v, o_sparse, true, true, false, st)))
    return rc;
  if (o_lin != nullptr) {
    if (linear) return launch_attn<D, BLK>(s, w, kc_bh, q, v, o_lin, true, false, true, st);
    return cuda_status(cudaMemsetAsync(o_lin, 0, (size_t)s.BH * s.N * D * sizeof(float), st));
  }
  return SLA_OK;
}

template <class F>
int with_dims(int d, int block, F&& f) {
  if (d == 128 && block == 128) return f(std::integral_constant<int, 128>(), std::integral_constant<int, 128>());
  if (d == 128 && block == 64) return f(std::integral_constant<int, 128>(), std::integral_constant<int, 64>());
  if (d == 64 && block == 128) return f(std::integral_constant<int, 64>(), std::integral_constant<int, 128>());
  if (d == 64 && block == 64) return f(std::integral_constant<int, 64>(), std::integral_constant<int, 64>());
  return SLA_ERR_UNSUPPORTED;
}

struct Scratch {
  void* ptr = nullptr;
  cudaStream_t st = nullptr;
  int get(size_t bytes, cudaStream_t s) {
    st = s;
    cudaMemPool_t pool = pool_for_current_device();
    if (pool == nullptr) return SLA_ERR_CUDA;
    const cudaError_t e = cudaMallocFromPoolAsync(&ptr, bytes, pool, s);
    if (e != cudaSuccess) { ptr = nullptr; return cuda_status(e); }
    return SLA_OK;
  }
  ~Scratch() {
    if (ptr != nullptr) cudaFreeAsync(ptr, st);
  }
};

// ------------------------------------------------------------------ failure-path self test
// One thread waits, with the library's bounded wait, on an mbarrier that no
// one arrives at; the wait gives up, records DEV_ERR_TIMEOUT and returns.
__global__ void k_selftest_wait_timeout() {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  abort_flag = 0;
  fence_mbar_init();
  (void)mbar_wait(&bar, 0, &abort_flag);
}

// ------------------------------------------------------------------ fixed scratch for sla_mask_noalloc
// For callers that cannot allocate device memory while they run: the block
// sums of sla_mask_noalloc live here instead of in the stream-ordered pool.
// Host code must not use this name as an address; see noalloc_scratch().
static __device__ __align__(256) unsigned char g_noalloc_scratch[SLA_NOALLOC_SCRATCH_BYTES];

// Loads every kernel sla_mask_noalloc can launch onto the current device, so
// that no later call does so (with lazy module loading, a kernel's first use
// would otherwise load its code then, which may allocate device memory).
bool noalloc_load_kernels() {
  cudaFuncAttributes a;
  bool ok = true;
  auto load = [&](const void* f) { ok = ok && cudaFuncGetAttributes(&a, f) == cudaSuccess; };
  load((const void*)k_kstats<64, 64>);
  load((const void*)k_kstats<64, 128>);
  load((const void*)k_kstats<128, 64>);
  load((const void*)k_kstats<128, 128>);
  load((const void*)k_channel_mean<64>);
  load((const void*)k_channel_mean<128>);
  load((const void*)k_quant<64, 64, false>);
  load((const void*)k_quant<64, 128, false>);
  load((const void*)k_quant<128, 64, false>);
  load((const void*)k_quant<128, 128, false>);
  load((const void*)k_mask<64, 1>);
  load((const void*)k_mask<64, 2>);
  load((const void*)k_mask<64, 4>);
  load((const void*)k_mask<64, 8>);
  load((const void*)k_mask<128, 1>);
  load((const void*)k_mask<128, 2>);
  load((const void*)k_mask<128, 4>);
  load((const void*)k_mask<128, 8>);
  return ok;
}

// Device address of g_noalloc_scratch on the current device, looked up once per
// device (cudaGetSymbolAddress, checked) together with the loading of the
// entry point's kernels; nullptr if either failed.
void* noalloc_scratch() {
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    if (!noalloc_load_kernels()) return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
}

// ------------------------------------------------------------------ W8A8 linear layer
int w8a8_check(int M, int N, int K) {
  if (M < 1 || N < 1 || K < 1) return SLA_ERR_INVALID_ARG;
  if (K % 16 != 0 || N % 16 != 0) return SLA_ERR_UNSUPPORTED;
  if ((long long)M * K >= (1LL << 40) || (long long)N * K >= (1LL << 40)) return SLA_ERR_UNSUPPORTED;
  return SLA_OK;
}

// codes and scales of a bf16 [R, K] matrix, 128x128 blocks
int launch_quant2d(const void* x, int R, int K, int8_t* codes, float* scales, cudaStream_t st) {
  CUtensorMap m;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)R};
  cuuint64_t str[1] = {(cuuint64_t)K * 2};
  cuuint32_t box[2] = {128u, 128u};
  if (!make_map(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE))
    return SLA_ERR_CUDA;
  cudaFuncSetAttribute(k_quant2d, cudaFuncAttributeMaxDynamicSharedMemorySize, kQ2Smem);
  dim3 g((unsigned)((K + 127) / 128), (unsigned)((R + 127) / 128));
  ProfScope ps(SLA_K_QUANT2D, st);
  k_quant2d<<<g, 256, kQ2Smem, st>>>(m, R, K, codes, scales);
  return cuda_status(cudaGetLastError());
}

int launch_w8a8_gemm(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw, const void* bias, void* y,
                     bool out_f32, int M, int N, int K, cudaStream_t st) {
  constexpr int BN = kW8TileN, NBUF = kW8Buffers;
  using C = W8Cfg<BN, NBUF>;
  CUtensorMap ma, mb;
  {
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    cuuint64_t str[1] = {(cuuint64_t)K};
    cuuint32_t box[2] = {128u, 128u};
    if (!make_map(&ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, xq, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return SLA_ERR_CUDA;
  }
  {
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)N};
    cuuint64_t str[1] = {(cuuint64_t)K};
    cuuint32_t box[2] = {128u, (cuuint32_t)BN};
    if (!make_map(&mb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, wq, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return SLA_ERR_CUDA;
  }
  W8A8Params p;
  p.sx = sx; p.sw = sw; p.bias = static_cast<const __nv_bfloat16*>(bias); p.y = y;
  p.M = M; p.N = N; p.K = K; p.KB = (K + 127) / 128;
  p.tiles_n = (N + BN - 1) / BN;
  const long long tiles = (long long)((M + 127) / 128) * p.tiles_n;
  if (tiles >= (1LL << 31)) return SLA_ERR_UNSUPPORTED;
  p.tiles = (int)tiles;
  p.out_f32 = out_f32 ? 1 : 0;
  cudaFuncSetAttribute(k_w8a8_gemm<BN, NBUF>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  const int ctas = (int)std::min<long long>(num_sms(), tiles);
  ProfScope ps(SLA_K_W8A8, st);
  k_w8a8_gemm<BN, NBUF><<<ctas, C::THREADS, C::SMEM, st>>>(ma, mb, p);
  return cuda_status(cudaGetLastError());
}

// ------------------------------------------------------------------ host-buffer entry point
// Streams and events of sla_attn_host, created once per device and kept (a
// call holds the device's set for its duration).
constexpr int kHostStreams = 3;
constexpr long long kHostChunks = 6;

struct HostStreams {
  std::mutex mu;
  cudaStream_t st[kHostStreams] = {};
  cudaEvent_t ev[kHostStreams] = {};
};

HostStreams* host_streams() {
  static std::mutex mu;
  static HostStreams* sets[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (sets[dev] == nullptr) {
    HostStreams* h = new HostStreams();
    for (int i = 0; i < kHostStreams; ++i)
      if (cudaStreamCreateWithFlags(&h->st[i], cudaStreamNonBlocking) != cudaSuccess ||
          cudaEventCreateWithFlags(&h->ev[i], cudaEventDisableTiming) != cudaSuccess)
        return nullptr;
    sets[dev] = h;
  }
  return sets[dev];
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

int sla_topk_count(int N, int block, float topk_frac) {
  if (N < 1 || block < 1 || !frac_ok(topk_frac)) return -SLA_ERR_INVALID_ARG;
  const long long nb = ((long long)N + block - 1) / block;
  return (int)topk_count_ll(nb, topk_frac);
}

const char* sla_status_string(int status) {
  switch (status) {
    case SLA_OK: return "ok";
    case SLA_ERR_INVALID_ARG: return "invalid argument";
    case SLA_ERR_UNSUPPORTED: return "unsupported shape or parameter";
    case SLA_ERR_CUDA: return "CUDA error";
    case SLA_ERR_OOM: return "out of device memory";
    case SLA_ERR_TIMEOUT: return "a kernel wait timed out";
    case SLA_ERR_SCRATCH_LIMIT: return "problem larger than the fixed no-allocation scratch buffer";
    case SLA_ERR_SMEM_LAYOUT: return "a kernel could not place its shared-memory tiles";
    default: return "unknown status";
  }
}

int sla_quant(const void* q, const void* k, int8_t* q_i8, int8_t* k_i8, float* q_scale, float* k_scale,
              float* k_mean, int B, int H, int N, int d, int block, void* stream) {
  if (!q || !k || !q_i8 || !k_i8 || !q_scale || !k_scale) return SLA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q_i8) || !aligned16(k_i8)) return SLA_ERR_INVALID_ARG;
  Shape s;
  int rc = check_shape(B, H, N, d, block, &s);
  if (rc) return rc;
  s.kc = 1;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Scratch sc;
  if ((rc = sc.get(workspace_bytes(s, 0), st))) return rc;
  Workspace w = carve(s, 0, static_cast<char*>(sc.ptr));
  if (k_mean != nullptr) w.mu = k_mean;
  return with_dims(d, block, [&](auto D_, auto B_) {
    constexpr int D = decltype(D_)::value, BLK = decltype(B_)::value;
    return launch_stats_quant<D, BLK>(s, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                                      nullptr, nullptr, w, false, true, q_i8, k_i8, q_scale, k_scale, st);
  });
}

int sla_quant_gran(const void* q, const void* k, int8_t* q_i8, int8_t* k_i8, float* q_scale, float* k_scale,
                   float* k_mean, int B, int H, int N, int d, int block, int gran, void* stream) {
  if (!q || !k || !q_i8 || !k_i8 || !q_scale || !k_scale) return SLA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q_i8) || !aligned16(k_i8)) return SLA_ERR_INVALID_ARG;
  Shape s;
  int rc = check_shape(B, H, N, d, block, &s);
  if (rc) return rc;
  if ((rc = set_gran(&s, gran))) return rc;
  s.kc = 1;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Scratch sc;
  if ((rc = sc.get(workspace_bytes(s, 0), st))) return rc;
  Workspace w = carve(s, 0, static_cast<char*>(sc.ptr));
  if (k_mean != nullptr) w.mu = k_mean;
  return with_dims(d, block, [&](auto D_, auto B_) {
    constexpr int D = decltype(D_)::value, BLK = decltype(B_)::value;
    return launch_stats_quant<D, BLK>(s, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                                      nullptr, nullptr, w, false, true, q_i8, k_i8, q_scale, k_scale, st);
  });
}

int sla_mask(const void* q, const void* k, int32_t* blk_idx, uint8_t* bitmap, int B, int H, int N, int d,
             int block, float topk_frac, void* stream) {
  if (!q || !k || !blk_idx) return SLA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k)) return SLA_ERR_INVALID_ARG;
  if (!frac_ok(topk_frac)) return SLA_ERR_INVALID_ARG;
  Shape s;
  int rc = check_shape(B, H, N, d, block, &s);
  if (rc) return rc;
  s.kc = topk_count_ll(s.NB, topk_frac);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Scratch sc;
  if ((rc = sc.get(workspace_bytes(s, 0), st))) return rc;
  Workspace w = carve(s, 0, static_cast<char*>(sc.ptr));
  return with_dims(d, block, [&](auto D_, auto B_) {
    constexpr int D = decltype(D_)::value, BLK = decltype(B_)::value;
    int r = launch_stats_quant<D, BLK>(s, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                                       nullptr, nullptr, w, false, false, nullptr, nullptr, nullptr, nullptr, st);
    if (r) return r;
    return launch_mask<D>(s, w, uniform_counts(s.kc), nullptr, blk_idx, bitmap, nullptr, st);
  });
}

int sla_mask_noalloc(const void* q, const void* k, int32_t* blk_idx, uint8_t* bitmap, int B, int H, int N, int d,
                     int block, float topk_frac, void* stream) {
  if (!q || !k || !blk_idx) return SLA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k)) return SLA_ERR_INVALID_ARG;
  if (!frac_ok(topk_frac)) return SLA_ERR_INVALID_ARG;
  Shape s;
  int rc = check_shape(B, H, N, d, block, &s);
  if (rc) return rc;
  s.kc = topk_count_ll(s.NB, topk_frac);
  if (workspace_bytes(s, 0) > SLA_NOALLOC_SCRATCH_BYTES) return SLA_ERR_SCRATCH_LIMIT;
  void* scratch = noalloc_scratch();
  if (scratch == nullptr) return SLA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Workspace w = carve(s, 0, static_cast<char*>(scratch));
  return with_dims(d, block, [&](auto D_, auto B_) {
    constexpr int D = decltype(D_)::value, BLK = decltype(B_)::value;
    int r = launch_stats_quant<D, BLK>(s, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                                       nullptr, nullptr, w, false, false, nullptr, nullptr, nullptr, nullptr, st);
    if (r) return r;
    return launch_mask<D>(s, w, uniform_counts(s.kc), nullptr, blk_idx, bitmap, nullptr, st);
  });
}

int sla_attn_ex(const void* q, const void* k, const void* v, const void* proj, void* out, int out_dtype,
                float* o_sparse, float* o_lin, int B, int H, int N, int d, int block, float topk_frac,
                void* stream) {
  if (!q || !k || !v || !proj || !out) return SLA_ERR_INVALID_ARG;
  if (out_dtype != SLA_OUT_BF16 && out_dtype != SLA_OUT_F32) return SLA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(proj) || !aligned16(out) ||
      !aligned16(o_sparse) || !aligned16(o_lin))
    return SLA_ERR_INVALID_ARG;
  if (!frac_ok(topk_frac)) return SLA_ERR_INVALID_ARG;
  Shape s;
  int rc = check_shape(B, H, N, d, block, &s);
  if (rc) return rc;
  s.kc = topk_count_ll(s.NB, topk_frac);
  const bool linear = s.kc < s.NB;
  const int what = 1 | 2 | 4 | (linear ? 8 : 0);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Scratch sc;
  if ((rc = sc.get(workspace_bytes(s, what), st))) return rc;
  Workspace w = carve(s, what, static_cast<char*>(sc.ptr));
  return with_dims(d, block, [&](auto D_, auto B_) {
    constexpr int D = decltype(D_)::value, BLK = decltype(B_)::value;
    return run_attn<D, BLK>(s, uniform_counts(s.kc), linear, static_cast<const __nv_bfloat16*>(q),
                            static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v),
                            static_cast<const __nv_bfloat16*>(proj), out, out_dtype == SLA_OUT_F32, o_sparse, o_lin,
                            w, st);
  });
}

int sla_attn_classes(const void* q, const void* k, const void* v, const void* proj, void* out, int out_dtype,
                     float* o_sparse, float* o_lin, int B, int H, int N, int d, int block, const float* topk_frac,
                     const float* skip_frac, void* stream) {
  if (!q || !k || !v || !proj || !out) return SLA_ERR_INVALID_ARG;
  if (out_dtype != SLA_OUT_BF16 && out_dtype != SLA_OUT_F32) return SLA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(proj) || !aligned16(out) ||
      !aligned16(o_sparse) || !aligned16(o_lin))
    return SLA_ERR_INVALID_ARG;
  Shape s;
  int rc = check_shape(B, H, N, d, block, &s);
  if (rc) return rc;
  HeadCounts hc;
  bool linear = false;
  if ((rc = head_counts(s.NB, H, topk_frac, skip_frac, &hc, &linear))) return rc;
  s.kc = hc.kcp;
  const int what = 1 | 2 | 4 | (linear ? 8 : 0);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Scratch sc;
  if ((rc = sc.get(workspace_bytes(s, what), st))) return rc;
  Workspace w = carve(s, what, static_cast<char*>(sc.ptr));
  return with_dims(d, block, [&](auto D_, auto B_) {
    constexpr int D = decltype(D_)::value, BLK = decltype(B_)::value;
    return run_attn<D, BLK>(s, hc, linear, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                            static_cast<const __nv_bfloat16*>(v), static_cast<const __nv_bfloat16*>(proj), out,
                            out_dtype == SLA_OUT_F32, o_sparse, o_lin, w, st);
  });
}

int sla_mask_classes(const void* q, const void* k, int32_t* blk_idx, uint8_t* classes, int B, int H, int N, int d,
                     int block, const float* topk_frac, const float* skip_frac, void* stream) {
  if (!q || !k || !blk_idx) return SLA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k)) return SLA_ERR_INVALID_ARG;
  Shape s;
  int rc = check_shape(B, H, N, d, block, &s);
  if (rc) return rc;
  HeadCounts hc;
  bool linear = false;
  if ((rc = head_counts(s.NB, H, topk_frac, skip_frac, &hc, &linear))) return rc;
  s.kc = hc.kcp;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Scratch sc;
  if ((rc = sc.get(workspace_bytes(s, 0), st))) return rc;
  Workspace w = carve(s, 0, static_cast<char*>(sc.ptr));
  return with_dims(d, block, [&](auto D_, auto B_) {
    constexpr int D = decltype(D_)::value, BLK = decltype(B_)::value;
    int r = launch_stats_quant<D, BLK>(s, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                                       nullptr, nullptr, w, false, false, nullptr, nullptr, nullptr, nullptr, st);
    if (r) return r;
    return launch_mask<D>(s, w, hc, nullptr, blk_idx, classes, nullptr, st);
  });
}

int sla_head_counts(int N, int block, int H, const float* topk_frac, const float* skip_frac, int* kc, int* kn) {
  if (N < 1 || block < 1 || H < 1) return -SLA_ERR_INVALID_ARG;
  HeadCounts hc;
  bool linear = false;
  const long long nb = ((long long)N + block - 1) / block;
  const int rc = head_counts(nb, H, topk_frac, skip_frac, &hc, &linear);
  if (rc) return -rc;
  for (int h = 0; h < H; ++h) {
    if (kc) kc[h] = hc.kc[h];
    if (kn) kn[h] = hc.kn[h];
  }
  return hc.kcp;
}

int sla_attn_gran(const void* q, const void* k, const void* v, const void* proj, void* out, int out_dtype,
                  float* o_sparse, float* o_lin, int B, int H, int N, int d, int block, float topk_frac, int gran,
                  void* stream) {
  if (!q || !k || !v || !proj || !out) return SLA_ERR_INVALID_ARG;
  if (out_dtype != SLA_OUT_BF16 && out_dtype != SLA_OUT_F32) return SLA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(proj) || !aligned16(out) ||
      !aligned16(o_sparse) || !aligned16(o_lin))
    return SLA_ERR_INVALID_ARG;
  if (!frac_ok(topk_frac)) return SLA_ERR_INVALID_ARG;
  Shape s;
  int rc = check_shape(B, H, N, d, block, &s);
  if (rc) return rc;
  if ((rc = set_gran(&s, gran))) return rc;
  s.kc = topk_count_ll(s.NB, topk_frac);
  const bool linear = s.kc < s.NB;
  const int what = 1 | 2 | 4 | (linear ? 8 : 0);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Scratch sc;
  if ((rc = sc.get(workspace_bytes(s, what), st))) return rc;
  Workspace w = carve(s, what, static_cast<char*>(sc.ptr));
  return with_dims(d, block, [&](auto D_, auto B_) {
    constexpr int D = decltype(D_)::value, BLK = decltype(B_)::value;
    return run_attn<D, BLK>(s, uniform_counts(s.kc), linear, static_cast<const __nv_bfloat16*>(q),
                            static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v),
                            static_cast<const __nv_bfloat16*>(proj), out, out_dtype == SLA_OUT_F32, o_sparse, o_lin,
                            w, st);
  });
}

int sla_attn(const void* q, const void* k, const void* v, const void* proj, void* out, int B, int H, int N, int d,
             int block, float topk_frac, void* stream) {
  return sla_attn_ex(q, k, v, proj, out, SLA_OUT_BF16, nullptr, nullptr, B, H, N, d, block, topk_frac, stream);
}

}  // extern "C"

namespace {

// sla_attn_host and sla_attn_classes_host: one fraction for every head, or
// (tf != nullptr) the three-class operator with per-head fractions.
int attn_host(const void* q, const void* k, const void* v, const void* proj, void* out, int B, int H, int N, int d,
              int block, float topk_frac, const float* tf, const float* sf) {
  if (!q || !k || !v || !proj || !out) return SLA_ERR_INVALID_ARG;
  Shape s;
  int rc = check_shape(B, H, N, d, block, &s);
  if (rc) return rc;
  if (tf == nullptr && !frac_ok(topk_frac)) return SLA_ERR_INVALID_ARG;
  if (tf != nullptr) {   // the whole argument check before any copy
    HeadCounts hc;
    bool linear = false;
    if ((rc = head_counts(s.NB, H, tf, sf, &hc, &linear))) return rc;
  }
  HostStreams* hs = host_streams();
  if (hs == nullptr) return SLA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(hs->mu);
  cudaStream_t* st = hs->st;
  const size_t head = (size_t)N * d * 2;                    // bytes of one head of q, k, v or out
  const size_t tb = (size_t)s.BH * head, pb = (size_t)d * d * 2;
  const size_t off = (tb + 255) & ~size_t(255), poff = (pb + 255) & ~size_t(255);
  char* buf = nullptr;
  cudaMemPool_t pool = pool_for_current_device();
  cudaError_t e = pool ? cudaMallocFromPoolAsync(reinterpret_cast<void**>(&buf), 4 * off + poff, pool, st[0])
                       : cudaErrorInitializationError;
  if (e != cudaSuccess) return cuda_status(e);
  char *dq = buf, *dk = buf + off, *dv = buf + 2 * off, *dout = buf + 3 * off, *dp = buf + 4 * off;
  rc = SLA_OK;
  if (cudaMemcpyAsync(dp, proj, pb, cudaMemcpyHostToDevice, st[0]) != cudaSuccess ||
      cudaEventRecord(hs->ev[0], st[0]) != cudaSuccess)
    rc = SLA_ERR_CUDA;
  // heads in chunks over the streams: a chunk's copies in, operator and copy
  // out are ordered on its stream; chunks on different streams overlap (the
  // operator of a chunk then keeps to its chunk's stream)
  struct OneStream {
    OneStream() { t_one_stream = true; }
    ~OneStream() { t_one_stream = false; }
  } one_stream;
  long long chunks = std::min<long long>(s.BH, kHostChunks);
  if (tf != nullptr)   // a chunk's per-head counts must fit the kernels' table
    chunks = std::max<long long>(chunks, (s.BH + kMaxHeadCounts - 1) / kMaxHeadCounts);
  const long long per = (s.BH + chunks - 1) / chunks;
  for (long long c = 0; c < chunks && rc == SLA_OK; ++c) {
    const long long h0 = c * per, nh = std::min<long long>(per, s.BH - h0);
    if (nh <= 0) break;
    cudaStream_t sc = st[c % kHostStreams];
    const size_t o = (size_t)h0 * head, nb = (size_t)nh * head;
    if ((c % kHostStreams != 0 && cudaStreamWaitEvent(sc, hs->ev[0], 0) != cudaSuccess) ||
        cudaMemcpyAsync(dq + o, static_cast<const char*>(q) + o, nb, cudaMemcpyHostToDevice, sc) != cudaSuccess ||
        cudaMemcpyAsync(dk + o, static_cast<const char*>(k) + o, nb, cudaMemcpyHostToDevice, sc) != cudaSuccess ||
        cudaMemcpyAsync(dv + o, static_cast<const char*>(v) + o, nb, cudaMemcpyHostToDevice, sc) != cudaSuccess) {
      rc = SLA_ERR_CUDA;
      break;
    }
    if (tf == nullptr) {
      rc = sla_attn(dq + o, dk + o, dv + o, dp, dout + o, 1, (int)nh, N, d, block, topk_frac, sc);
    } else {   // the chunk's heads h0 .. h0 + nh - 1 of the B*H, head index (h0 + t) % H
      std::vector<float> ctf((size_t)nh), csf((size_t)nh);
      for (long long t = 0; t < nh; ++t) {
        ctf[t] = tf[(h0 + t) % H];
        csf[t] = sf != nullptr ? sf[(h0 + t) % H] : 0.f;
      }
      rc = sla_attn_classes(dq + o, dk + o, dv + o, dp, dout + o, SLA_OUT_BF16, nullptr, nullptr, 1, (int)nh, N, d,
                            block, ctf.data(), csf.data(), sc);
    }
    if (rc == SLA_OK &&
        cudaMemcpyAsync(static_cast<char*>(out) + o, dout + o, nb, cudaMemcpyDeviceToHost, sc) != cudaSuccess)
      rc = SLA_ERR_CUDA;
  }
  // join the streams, release the buffers, wait for the results
  for (int i = 1; i < kHostStreams; ++i)
    if (cudaEventRecord(hs->ev[i], st[i]) != cudaSuccess || cudaStreamWaitEvent(st[0], hs->ev[i], 0) != cudaSuccess)
      if (rc == SLA_OK) rc = SLA_ERR_CUDA;
  cudaFreeAsync(buf, st[0]);
  const cudaError_t se = cudaStreamSynchronize(st[0]);
  if (rc == SLA_OK && se != cudaSuccess) rc = SLA_ERR_CUDA;
  return rc;
}

}  // namespace

extern "C" {

int sla_attn_host(const void* q, const void* k, const void* v, const void* proj, void* out, int B, int H, int N,
                  int d, int block, float topk_frac) {
  return attn_host(q, k, v, proj, out, B, H, N, d, block, topk_frac, nullptr, nullptr);
}

int sla_attn_classes_host(const void* q, const void* k, const void* v, const void* proj, void* out, int B, int H,
                          int N, int d, int block, const float* topk_frac, const float* skip_frac) {
  if (topk_frac == nullptr) return SLA_ERR_INVALID_ARG;
  return attn_host(q, k, v, proj, out, B, H, N, d, block, 0.f, topk_frac, skip_frac);
}

int sla_w8a8_quant(const void* x, int R, int K, int8_t* codes, float* scales, void* stream) {
  if (!x || !codes || !scales) return SLA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes)) return SLA_ERR_INVALID_ARG;
  const int rc = w8a8_check(R, 16, K);
  if (rc) return rc;
  return launch_quant2d(x, R, K, codes, scales, static_cast<cudaStream_t>(stream));
}

int sla_w8a8_gemm(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw, const void* bias, void* y,
                  int out_dtype, int M, int N, int K, void* stream) {
  if (!xq || !sx || !wq || !sw || !y) return SLA_ERR_INVALID_ARG;
  if (out_dtype != SLA_OUT_BF16 && out_dtype != SLA_OUT_F32) return SLA_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(wq) || !aligned16(y) || !aligned16(bias)) return SLA_ERR_INVALID_ARG;
  const int rc = w8a8_check(M, N, K);
  if (rc) return rc;
  return launch_w8a8_gemm(xq, sx, wq, sw, bias, y, out_dtype == SLA_OUT_F32, M, N, K,
                          static_cast<cudaStream_t>(stream));
}

int sla_w8a8_linear(const void* x, const int8_t* wq, const float* sw, const void* bias, void* y, int out_dtype, int M,
                    int N, int K, void* stream) {
  if (!x || !wq || !sw || !y) return SLA_ERR_INVALID_ARG;
  if (out_dtype != SLA_OUT_BF16 && out_dtype != SLA_OUT_F32) return SLA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(wq) || !aligned16(y) || !aligned16(bias)) return SLA_ERR_INVALID_ARG;
  int rc = w8a8_check(M, N, K);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t cb = rounded<int8_t>((size_t)M * K);
  const size_t sb = rounded<float>((size_t)((M + 127) / 128) * ((K + 127) / 128));
  Scratch sc;
  if ((rc = sc.get(cb + sb, st))) return rc;
  int8_t* xq = static_cast<int8_t*>(sc.ptr);
  float* sx = reinterpret_cast<float*>(static_cast<char*>(sc.ptr) + cb);
  if ((rc = launch_quant2d(x, M, K, xq, sx, st))) return rc;
  return launch_w8a8_gemm(xq, sx, wq, sw, bias, y, out_dtype == SLA_OUT_F32, M, N, K, st);
}

int sla_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = on != 0;
  return SLA_OK;
}

int sla_profile_read(double* ms, long long* launches, int n) {
  std::vector<ProfRecord> recs;
  {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    recs.swap(g_prof);
  }
  if (n > SLA_K_COUNT) n = SLA_K_COUNT;
  for (int k = 0; k < n; ++k) {
    if (ms) ms[k] = 0.0;
    if (launches) launches[k] = 0;
  }
  int rc = SLA_OK;
  for (const ProfRecord& r : recs) {
    float t = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess)
      rc = SLA_ERR_CUDA;
    if (r.kind < n) {
      if (ms) ms[r.kind] += t;
      if (launches) launches[r.kind] += 1;
    }
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  return rc;
}

int sla_selftest_wait_timeout(void* stream) {
  k_selftest_wait_timeout<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
  return cuda_status(cudaGetLastError());
}

int sla_get_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SLA_ERR_CUDA;
  unsigned int word = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word)) != cudaSuccess) return SLA_ERR_CUDA;
  if (word != 0 && cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess) return SLA_ERR_CUDA;
  if (word & DEV_ERR_TIMEOUT) return SLA_ERR_TIMEOUT;
  if (word & DEV_ERR_LAYOUT) return SLA_ERR_SMEM_LAYOUT;
  return SLA_OK;
}

}  // extern "C"
