// Plain C++ CPU oracle for the W8A8 block-quantised linear layer.
//
// TEST INFRASTRUCTURE ONLY: built into libsla_oracle.so by oracle/build.py and
// loaded through oracle/w8a8_cpp.py by the tests and the benchmark's CPU
// leg, never by the library; it shares no code with the CUDA sources.
//
// Sources.
//   "Turbo Diffusion：秒级生成与高清保真的视频扩散技术突破" (lanhy.cn),
//   section 三(四) item 1: weights and activations of the linear layers in
//   8 bits, quantisation parameters per independent 128x128 block of the
//   weight matrix, activations quantised dynamically at inference time with
//   clipping of extreme values.
//   chooseai.net news page ("TuroDiffusion：为高质量视频'系统性提速'"), the
//   linear-layer paragraph: parameters and activations in 8 bits with
//   128x128 block granularity.
//
// Readings (the pages give no formula; the same as the numpy statement):
//   Y = X W^T + bias, X [M, K] and W [N, K] bf16, bias [N] bf16 (optional).
//   Both operands are cut into 128 x 128 blocks (partial at the edges); a
//   block's scale is s = float32(max|x| / 127), its codes
//   clamp(round_half_even(float32(x / s)), -127, 127), all 0 when s = 0
//   ("clipping" read as the saturation).  Y[m, n] = sum over column blocks
//   kb, in order, of P_kb * (sx * sw) (+ bias), P_kb the exact integer sum of
//   the block's int8 products, evaluated here in float64.
//
// Build flags: -ffp-contract=off and no -ffast-math, so every operation is
// one IEEE rounding in the order written.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

constexpr int kBlk = 128;

float bf16_value(uint16_t h) {
  const uint32_t u = uint32_t(h) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return f;
}

int nblocks(int n) { return (n + kBlk - 1) / kBlk; }

}  // namespace

extern "C" {

// x: bf16 bits [R, K] row-major -> codes int8 [R, K], scales float32
// [nblocks(R), nblocks(K)].
void ora_w8a8_quantize(const uint16_t* x, int R, int K, int8_t* codes, float* scales) {
  const int nrb = nblocks(R), nkb = nblocks(K);
  for (int rb = 0; rb < nrb; ++rb) {
    for (int kb = 0; kb < nkb; ++kb) {
      const int r0 = rb * kBlk, r1 = std::min(R, r0 + kBlk);
      const int c0 = kb * kBlk, c1 = std::min(K, c0 + kBlk);
      float m = 0.f;
      for (int r = r0; r < r1; ++r)
        for (int c = c0; c < c1; ++c) m = std::max(m, std::fabs(bf16_value(x[(long long)r * K + c])));
      const float s = m / 127.0f;
      scales[(long long)rb * nkb + kb] = s;
      for (int r = r0; r < r1; ++r) {
        for (int c = c0; c < c1; ++c) {
          int8_t q = 0;
          if (s > 0.f) {
            const float t = bf16_value(x[(long long)r * K + c]) / s;
            const float rq = std::nearbyint(t);   // round half to even (default mode)
            q = (int8_t)std::min(127.f, std::max(-127.f, rq));
          }
          codes[(long long)r * K + c] = q;
        }
      }
    }
  }
}

// Rows rows[0..nrows) of X against every row of W:
//   y[t, n] = sum_kb P_kb(rows[t], n) * (sx * sw) (+ bias[n]),
//   a[t, n] = sum_kb |P_kb * (sx * sw)| (+ |bias[n]|),
// float64, [nrows, N] each.  xq [M, K], sx [nblocks(M), nkb], wq [N, K],
// sw [nblocks(N), nkb]; bias may be null.  Work is split over `threads`
// std::thread workers by rows (each output element is one worker's).
void ora_w8a8_gemm(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw, const uint16_t* bias,
                   int N, int K, const long long* rows, int nrows, int threads, double* y, double* a) {
  const int nkb = nblocks(K);
  auto work = [&](int t0, int t1) {
    for (int t = t0; t < t1; ++t) {
      const long long m = rows[t];
      const long long mb = m / kBlk;
      for (int n = 0; n < N; ++n) {
        const int nb = n / kBlk;
        double acc = 0.0, mag = 0.0;
        for (int kb = 0; kb < nkb; ++kb) {
          const int c0 = kb * kBlk, c1 = std::min(K, c0 + kBlk);
          int32_t p = 0;   // |p| <= 128 * 127^2 < 2^31
          for (int c = c0; c < c1; ++c) p += int32_t(xq[m * K + c]) * int32_t(wq[(long long)n * K + c]);
          const double s = (double)sx[mb * nkb + kb] * (double)sw[(long long)nb * nkb + kb];   // exact
          const double term = (double)p * s;
          acc += term;
          mag += std::fabs(term);
        }
        if (bias != nullptr) {
          const double b = (double)bf16_value(bias[n]);
          acc += b;
          mag += std::fabs(b);
        }
        y[(long long)t * N + n] = acc;
        a[(long long)t * N + n] = mag;
      }
    }
  };
  const int nt = std::max(1, std::min(threads, nrows));
  std::vector<std::thread> pool;
  for (int w = 0; w < nt; ++w) {
    const int t0 = (int)((long long)nrows * w / nt), t1 = (int)((long long)nrows * (w + 1) / nt);
    pool.emplace_back(work, t0, t1);
  }
  for (auto& th : pool) th.join();
}

}  // extern "C"
