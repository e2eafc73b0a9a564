// CPU oracle for SageSLA attention, in plain C++ -- TEST INFRASTRUCTURE ONLY.
//
// The slow, direct statement of what the CUDA path computes.  Only the tests,
// the package's smoke check and the benchmark's CPU-baseline leg call it
// (through oracle/cpp_oracle.py); the library never does, and it shares no
// code with the CUDA sources.  Plain loops in float64 (float32 exactly where
// the reading fixes float32), no BLAS; the work over query blocks is spread
// over std::thread workers.
//
// What it follows (the pages describe the method in prose only):
//   "Turbo Diffusion：秒级生成与高清保真的视频扩散技术突破" (lanhy.cn), section
//   三(一) SageAttention2++ items 1-3 (outlier smoothing, per-sub-block
//   quantisation parameters, 128x128 tensor-core tiles with a parallel softmax)
//   and section 三(二) SLA items 1-3 (top-K 10% block selection, an O(N)
//   linear branch with a linear projection, SageSLA = selection followed by
//   INT8 computation on the kept blocks);
//   "TurboDiffusion技术指南：突破视频生成效率瓶颈的实践方案" (blog.gitcode.com),
//   section "SageSLA" and the T2V parameter list (--sla_topk 0.1 keeps 10%);
//   "TurboDiffusion: 即時AI影片生成的重大突破" (bonega.ai), section "SLA:
//   稀疏線性注意力" (cheaper substitutes where full attention is not needed),
//   the basis of the optional third block class (left out entirely) and of
//   per-head fractions, an extension the pages do not spell out.
// The readings where the pages leave a step open are stated at each function;
// they are the same readings as oracle/sla_oracle.py (the numpy statement),
// which this file restates independently.
//
// Inputs are bf16 bit patterns (uint16), tensors [B, H, N, d] row-major; a
// block r covers rows [r*block, min(N, (r+1)*block)).
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

// ---------------------------------------------------------------- number formats

double bf16_value(uint16_t b) {
  uint32_t u = uint32_t(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return double(f);
}

float bf16_value_f(uint16_t b) { return float(bf16_value(b)); }

// Nearest bf16 value (8 significant bits) to x, ties to even, returned as a
// double.  With x = m * 2^e, 0.5 <= |m| < 1, the spacing of bf16 values near x
// is 2^(e-8); below the smallest normal bf16 (2^-126) it stays 2^-133.
double round_bf16(double x) {
  if (x == 0.0 || !std::isfinite(x)) return x;
  int e = 0;
  std::frexp(x, &e);
  if (e < -125) e = -125;
  const double y = std::ldexp(std::nearbyint(std::ldexp(x, 8 - e)), e - 8);
  if (std::fabs(y) > 3.3895313892515355e38) return std::copysign(INFINITY, x);
  return y;
}

// Unsigned integer of up to 12 * 32 = 384 bits, least significant word first.
struct Big {
  uint32_t w[12];
};

Big big_zero() {
  Big b;
  std::memset(b.w, 0, sizeof(b.w));
  return b;
}

// b += v * 2^shift (v < 2^63)
void big_add_shifted(Big& b, uint64_t v, int shift) {
  // spread v << shift over words, then add with carries
  uint32_t add[12] = {0};
  const int wq = shift / 32, bq = shift % 32;
  unsigned __int128 t = (unsigned __int128)v << bq;
  for (int k = 0; k < 4 && wq + k < 12; ++k) add[wq + k] = uint32_t(t >> (32 * k));
  uint64_t carry = 0;
  for (int k = 0; k < 12; ++k) {
    const uint64_t s = uint64_t(b.w[k]) + add[k] + carry;
    b.w[k] = uint32_t(s);
    carry = s >> 32;
  }
}

int big_cmp(const Big& a, const Big& b) {
  for (int k = 11; k >= 0; --k)
    if (a.w[k] != b.w[k]) return a.w[k] < b.w[k] ? -1 : 1;
  return 0;
}

// a - b for a >= b
Big big_sub(const Big& a, const Big& b) {
  Big r;
  int64_t borrow = 0;
  for (int k = 0; k < 12; ++k) {
    int64_t d = int64_t(a.w[k]) - int64_t(b.w[k]) - borrow;
    borrow = d < 0 ? 1 : 0;
    r.w[k] = uint32_t(d + (borrow << 32));
  }
  return r;
}

// a * m (m < 2^32)
Big big_mul_small(const Big& a, uint32_t m) {
  Big r;
  uint64_t carry = 0;
  for (int k = 0; k < 12; ++k) {
    const uint64_t p = uint64_t(a.w[k]) * m + carry;
    r.w[k] = uint32_t(p);
    carry = p >> 32;
  }
  return r;
}

// a * 2^s (s >= 0; the result stays below 2^384 where it is used)
Big big_shl(const Big& a, int s) {
  Big r = big_zero();
  for (int k = 0; k < 12; ++k)
    if (a.w[k]) big_add_shifted(r, a.w[k], 32 * k + s);
  return r;
}

// Approximate value of a as a double (for the first candidate only).
double big_approx(const Big& a) {
  double v = 0.0;
  for (int k = 11; k >= 0; --k) v = v * 4294967296.0 + double(a.w[k]);
  return v;
}

// The exact sum of bf16 values: integer significand sums per exponent field.
// A finite bf16 value is sig * 2^(E - 134), sig < 256, E = max(field, 1); in
// units of 2^-133 it is sig * 2^(E - 1).
struct ExactSum {
  int64_t bins[256];
  ExactSum() { std::memset(bins, 0, sizeof(bins)); }
  void add(uint16_t b) {
    const int field = (b >> 7) & 0xFF;
    const int64_t sig = field ? ((b & 0x7F) | 0x80) : (b & 0x7F);
    bins[field ? field : 1] += (b & 0x8000) ? -sig : sig;
  }
  // magnitude (units of 2^-133) and sign of the total
  Big total(bool& negative) const {
    Big pos = big_zero(), neg = big_zero();
    for (int e = 1; e < 256; ++e) {
      if (bins[e] > 0) big_add_shifted(pos, uint64_t(bins[e]), e - 1);
      if (bins[e] < 0) big_add_shifted(neg, uint64_t(-bins[e]), e - 1);
    }
    negative = big_cmp(pos, neg) < 0;
    return negative ? big_sub(neg, pos) : big_sub(pos, neg);
  }
};

// Compares the exact value X = mag * 2^-133 / den (den >= 1) with the
// non-negative dyadic number (a + b) / 2 for two doubles a, b >= 0: returns
// the sign of X - (a + b) / 2.  Both sides are brought to integers:
// 2 * mag * 2^u  versus  (A + B) * den * 2^(e + 133 + u), with a = A 2^ea,
// b = B 2^eb (integer significands), e = min(ea, eb), u >= 0 making both
// exponents non-negative.
int cmp_half_sum(const Big& mag, uint32_t den, double a, double b) {
  auto split = [](double x, uint64_t& m, int& e) {
    if (x == 0.0) { m = 0; e = 0; return; }
    int ex = 0;
    const double f = std::frexp(x, &ex);       // x = f * 2^ex, 0.5 <= f < 1
    m = uint64_t(std::ldexp(f, 53));
    e = ex - 53;
  };
  uint64_t A, Bm;
  int ea, eb;
  split(a, A, ea);
  split(b, Bm, eb);
  if (A == 0) ea = eb;
  if (Bm == 0) eb = ea;
  const int e = std::min(ea, eb);
  // (a + b) = (A 2^(ea-e) + B 2^(eb-e)) 2^e, an integer S times 2^e
  Big S = big_zero();
  big_add_shifted(S, A, ea - e);
  big_add_shifted(S, Bm, eb - e);
  Big rhs = big_mul_small(S, den);
  Big lhs = big_shl(mag, 1);
  const int k = e + 133;   // X vs mid  <=>  2 mag  vs  S den 2^k
  if (k >= 0)
    rhs = big_shl(rhs, k);
  else
    lhs = big_shl(lhs, -k);
  return big_cmp(lhs, rhs);
}

// The float (T = float or double) nearest to mag * 2^-133 / den, ties to the
// even neighbour, with the given sign.  The double approximation picks a first
// candidate; exact comparisons with the midpoints to its neighbours decide.
template <class T>
T round_exact(const Big& mag, bool negative, uint32_t den) {
  Big zero = big_zero();
  if (big_cmp(mag, zero) == 0) return T(0);
  const double approx = std::ldexp(big_approx(mag), -133) / double(den);
  T c = T(approx);
  auto odd = [](T v) {
    if constexpr (sizeof(T) == 4) {
      uint32_t u;
      std::memcpy(&u, &v, 4);
      return (u & 1u) != 0;
    } else {
      uint64_t u;
      std::memcpy(&u, &v, 8);
      return (u & 1u) != 0;
    }
  };
  for (int it = 0; it < 64; ++it) {
    const T up = std::nextafter(c, T(INFINITY)), dn = std::nextafter(c, T(0));
    const int hi = cmp_half_sum(mag, den, double(c), double(up));
    const int lo = c > T(0) ? cmp_half_sum(mag, den, double(dn), double(c)) : 1;
    if (hi > 0 || (hi == 0 && odd(c))) {
      c = up;
    } else if (lo < 0 || (lo == 0 && odd(c))) {
      c = dn;
    } else {
      break;
    }
  }
  return negative ? -c : c;
}

// ---------------------------------------------------------------- worker pool

template <class F>
void parallel_for(long long n, int threads, F&& f) {
  if (threads < 1) threads = 1;
  std::atomic<long long> next(0);
  auto work = [&]() {
    for (long long i = next++; i < n; i = next++) f(i);
  };
  std::vector<std::thread> pool;
  for (int t = 1; t < threads; ++t) pool.emplace_back(work);
  work();
  for (auto& th : pool) th.join();
}

}  // namespace

extern "C" {

// bf16 rounding of float64 values, for the pins (ties to even).
void ora_round_bf16(const double* x, long long n, double* y) {
  for (long long i = 0; i < n; ++i) y[i] = round_bf16(x[i]);
}

// mu[bh][c] = the float32 nearest to the exact mean of K[bh][:][c] over all N
// tokens (the per-channel mean that smooths K: section 三(一) item 1; reading:
// the sum is exact and rounded once, ties to even).
void ora_channel_mean(const uint16_t* k, int BH, int N, int d, int threads, float* mu) {
  parallel_for((long long)BH * d, threads, [&](long long t) {
    const long long bh = t / d;
    const int c = int(t % d);
    ExactSum s;
    for (int n = 0; n < N; ++n) s.add(k[(bh * N + n) * d + c]);
    bool neg = false;
    const Big m = s.total(neg);
    mu[bh * d + c] = round_exact<float>(m, neg, uint32_t(N));
  });
}

// Symmetric INT8 quantisation with one float32 scale per group of `gran`
// tokens x d channels (section 三(一) item 2, each sub-block has its own
// parameters; gran = block: one scale per block of the mask, gran < block:
// the finer "thread level" groups, gran dividing block).  x: float32
// [BH][N][d]; codes: int8 [BH][nblk*block][d] (rows past N are 0); scales:
// float32 [BH][nblk*block/gran].  Per group: m = max |x| over its valid rows,
// s = float32(m / 127), code = clamp(round_half_even(float32(x / s)), -127,
// 127); a group with m = 0 (or wholly past N) has s = 0 and zero codes.
void ora_quantize_blocks(const float* x, int BH, int N, int d, int block, int gran, int threads, int8_t* codes,
                         float* scales) {
  const int nblk = (N + block - 1) / block;
  const int ng = nblk * (block / gran);
  parallel_for((long long)BH * ng, threads, [&](long long t) {
    const long long bh = t / ng;
    const int r = int(t % ng);
    const int lo = r * gran, hi = std::min(N, lo + gran);
    float m = 0.f;
    for (int n = lo; n < hi; ++n)
      for (int c = 0; c < d; ++c) m = std::max(m, std::fabs(x[(bh * N + n) * d + c]));
    const float s = m / 127.0f;
    scales[bh * ng + r] = s;
    for (int n = lo; n < lo + gran; ++n)
      for (int c = 0; c < d; ++c) {
        int8_t q = 0;
        if (n < hi && s > 0.f) {
          const float y = x[(bh * N + n) * d + c] / s;
          const float rq = std::nearbyint(y);     // half to even (default rounding mode)
          q = int8_t(std::max(-127.f, std::min(127.f, rq)));
        }
        codes[(bh * (long long)nblk * block + n) * d + c] = q;
      }
  });
}

// K_s = float32(K) - mu, one float32 subtraction per element (Q is not smoothed).
void ora_smooth_k(const uint16_t* k, const float* mu, int BH, int N, int d, float* ks) {
  for (long long bh = 0; bh < BH; ++bh)
    for (int n = 0; n < N; ++n)
      for (int c = 0; c < d; ++c) {
        const long long o = (bh * N + n) * d + c;
        ks[o] = bf16_value_f(k[o]) - mu[bh * d + c];
      }
}

// Mean of each block's valid rows per channel, float64: the exact block sum
// rounded once to float64, divided by the number of valid rows (the pooled
// blocks of the mask, section 三(二) item 1; reading: raw values, valid rows
// only).  out: [BH][nblk][d].
void ora_block_means(const uint16_t* x, int BH, int N, int d, int block, int threads, double* out) {
  const int nblk = (N + block - 1) / block;
  parallel_for((long long)BH * nblk, threads, [&](long long t) {
    const long long bh = t / nblk;
    const int r = int(t % nblk);
    const int lo = r * block, hi = std::min(N, lo + block);
    for (int c = 0; c < d; ++c) {
      ExactSum s;
      for (int n = lo; n < hi; ++n) s.add(x[(bh * N + n) * d + c]);
      bool neg = false;
      const Big m = s.total(neg);
      out[(bh * nblk + r) * d + c] = round_exact<double>(m, neg, 1u) / double(hi - lo);
    }
  });
}

// p[bh][i][j] = softmax over j of qbar_i . kbar_j / sqrt(d), float64.
void ora_block_probs(const double* qbar, const double* kbar, int BH, int nblk, int d, int threads, double* p) {
  const double rs = std::sqrt(double(d));
  parallel_for((long long)BH * nblk, threads, [&](long long t) {
    const long long bh = t / nblk;
    const int i = int(t % nblk);
    double* row = p + (bh * nblk + i) * nblk;
    double mx = -INFINITY;
    for (int j = 0; j < nblk; ++j) {
      double s = 0.0;
      for (int c = 0; c < d; ++c) s += qbar[(bh * nblk + i) * d + c] * kbar[(bh * nblk + j) * d + c];
      row[j] = s / rs;
      mx = std::max(mx, row[j]);
    }
    double tot = 0.0;
    for (int j = 0; j < nblk; ++j) {
      row[j] = std::exp(row[j] - mx);
      tot += row[j];
    }
    for (int j = 0; j < nblk; ++j) row[j] /= tot;
  });
}

// The kc largest entries of each of `rows` rows of p (length n); equal values
// go to the lower index; listed ascending.  near_tie[r] = 1 when the kc-th and
// (kc+1)-th largest differ by at most 1e-9 of the kc-th.
void ora_select_topk(const double* p, long long rows, int n, int kc, int threads, int32_t* idx,
                     uint8_t* near_tie) {
  parallel_for(rows, threads, [&](long long r) {
    const double* row = p + r * n;
    std::vector<int> order(n);
    for (int j = 0; j < n; ++j) order[j] = j;
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return row[a] > row[b]; });
    std::vector<int> keep(order.begin(), order.begin() + kc);
    std::sort(keep.begin(), keep.end());
    for (int t = 0; t < kc; ++t) idx[r * kc + t] = keep[t];
    uint8_t tie = 0;
    if (kc < n) {
      const double a = row[order[kc - 1]], b = row[order[kc]];
      tie = (a - b) <= 1e-9 * a ? 1 : 0;
    }
    near_tie[r] = tie;
  });
}

// kc = clamp(ceil(float(topk_frac) * nblk), 1, nblk) (section 三(二) item 1,
// top-K 10%; --sla_topk 0.1 keeps 10%).  -1 if topk_frac is not in (0, 1].
int ora_topk_count(int nblk, float topk_frac) {
  const double f = double(topk_frac);
  if (!(f > 0.0 && f <= 1.0)) return -1;
  const double kc = std::ceil(f * double(nblk));
  return int(std::min(double(nblk), std::max(1.0, kc)));
}

// Negligible blocks per query block: floor(float(skip_frac) * nblk), at most
// nblk - kc (the third class of the three-class mask: left out of the linear
// branch too; none when skip_frac = 0).  -1 if skip_frac is not in [0, 1).
int ora_skip_count(int nblk, int kc, float skip_frac) {
  const double f = double(skip_frac);
  if (!(f >= 0.0 && f < 1.0)) return -1;
  const double kn = std::floor(f * double(nblk));
  return int(std::min(kn, double(nblk - kc)));
}

// Classes of the key blocks in each of `rows` rows of p (length nblk): row r
// belongs to head (r / rows_per_head) % H and uses kc and kn of that head.
// Ranking: larger value first, equal values by the lower index first;
// rank < kc: critical (2); rank >= nblk - kn: negligible (0); otherwise
// linear (1).  A block's rank is the number of blocks ranked before it,
// counted directly.  near_tie[r] = 1 when a class boundary separates values
// within 1e-9 (relative).
void ora_block_classes(const double* p, long long rows, int nblk, long long rows_per_head, int H, const int* kc,
                       const int* kn, int threads, uint8_t* cls, uint8_t* near_tie) {
  parallel_for(rows, threads, [&](long long r) {
    const int h = int((r / rows_per_head) % H);
    const int c = kc[h], z = kn[h];
    const double* row = p + r * nblk;
    std::vector<int> rank(nblk);
    for (int j = 0; j < nblk; ++j) {
      int before = 0;
      for (int m = 0; m < nblk; ++m) before += (row[m] > row[j] || (row[m] == row[j] && m < j)) ? 1 : 0;
      rank[j] = before;
      cls[r * nblk + j] = before < c ? 2 : (before >= nblk - z ? 0 : 1);
    }
    std::vector<int> at(nblk);
    for (int j = 0; j < nblk; ++j) at[rank[j]] = j;
    uint8_t tie = 0;
    for (int cut : {c, nblk - z})
      if (cut > 0 && cut < nblk) {
        const double a = row[at[cut - 1]], b = row[at[cut]];
        if ((a - b) <= 1e-9 * a) tie = 1;
      }
    near_tie[r] = tie;
  });
}

// Output rows of the whole operator for a list of query blocks.
//   q, k, v: bf16 [B][H][N][d]; w: bf16 [d][d] (W_proj, O_lin . W: row vectors)
//   cls: uint8 [B][H][nblk][nblk] the class of every (query block, key
//     block): 2 kept (exact attention), 1 linear branch, 0 left out
//   mu: float32 [B][H][d] (the K channel mean)
//   qi8, ki8, sq, sk: the INT8 codes and scales (quant = 1), else unused;
//     one scale per `gran` tokens ([B][H][nblk*block/gran])
//   items: n_items triples (b, h, i)
//   out, o_sparse, o_lin: float64 [n_items][block][d] (rows past N are 0);
//   o_lin is before the projection.
// Readings (sections 三(一) item 3, 三(二) items 2-3):
//   S = float32(int32(Qi8 . Ki8^T)) * float32(sq_n * sk_m) * float32(1/sqrt(d))
//   in float32 (quant = 0: S = Q . K_s^T / sqrt(d) in float64, K_s = K - mu
//   when smooth = 1, else K); keys at or past N are out; softmax with the row
//   maximum over all kept keys: P = exp(S - max) in float64, l = sum of the
//   unrounded P, P rounded to bf16 when pcast = 1; O_sparse = (P . V) / l.
//   phi(x) = x + 1 for x > 0, else exp(x); per key block j h_j = sum phi(k)
//   v^T, z_j = sum phi(k) over its valid rows (raw K); h_rest, z_rest are
//   summed directly over the blocks of class 1; O_lin = phi(q) h_rest /
//   (phi(q) . z_rest), zero when no block is of class 1; out = O_sparse +
//   O_lin W.
int ora_sla_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* w, int B, int H, int N,
                 int d, int block, const uint8_t* cls, const float* mu, const int8_t* qi8,
                 const int8_t* ki8, const float* sq, const float* sk, int gran, int quant, int pcast, int smooth,
                 const int32_t* items, int n_items, int threads, double* out, double* o_sparse, double* o_lin) {
  const int nblk = (N + block - 1) / block;
  const long long NP = (long long)nblk * block;
  auto phi = [](double x) { return x > 0.0 ? x + 1.0 : std::exp(x); };
  std::vector<double> W((size_t)d * d);
  for (int a = 0; a < d * d; ++a) W[a] = bf16_value(w[a]);

  // linear states of every head that an item needs: h [nblk][d][d], z [nblk][d]
  std::vector<int> head_of((size_t)B * H, -1);
  std::vector<long long> heads;
  for (int t = 0; t < n_items; ++t) {
    const long long bh = (long long)items[3 * t] * H + items[3 * t + 1];
    if (head_of[bh] < 0) {
      head_of[bh] = int(heads.size());
      heads.push_back(bh);
    }
  }
  std::vector<std::vector<double>> hs(heads.size()), zs(heads.size());
  parallel_for((long long)heads.size(), threads, [&](long long x) {
    const long long bh = heads[x];
    std::vector<double>& h = hs[x];
    std::vector<double>& z = zs[x];
    h.assign((size_t)nblk * d * d, 0.0);
    z.assign((size_t)nblk * d, 0.0);
    std::vector<double> pk(d), vv(d);
    for (int n = 0; n < N; ++n) {
      const int j = n / block;
      for (int c = 0; c < d; ++c) {
        pk[c] = phi(bf16_value(k[(bh * N + n) * d + c]));
        vv[c] = bf16_value(v[(bh * N + n) * d + c]);
      }
      for (int a = 0; a < d; ++a) {
        z[(size_t)j * d + a] += pk[a];
        for (int c = 0; c < d; ++c) h[((size_t)j * d + a) * d + c] += pk[a] * vv[c];
      }
    }
  });

  const double rsd = 1.0 / std::sqrt(double(d));
  const float rsd_f = float(rsd);
  parallel_for(n_items, threads, [&](long long t) {
    const int b = items[3 * t], hh = items[3 * t + 1], i = items[3 * t + 2];
    const long long bh = (long long)b * H + hh;
    const uint8_t* row_cls = cls + (bh * nblk + i) * nblk;
    std::vector<int> lst;
    for (int j = 0; j < nblk; ++j)
      if (row_cls[j] == 2) lst.push_back(j);
    const int kc = int(lst.size());
    const int lo = i * block, hi = std::min(N, lo + block);
    const int rows = hi - lo;
    double* po = out + (size_t)t * block * d;
    double* ps = o_sparse + (size_t)t * block * d;
    double* pl = o_lin + (size_t)t * block * d;
    std::fill(po, po + (size_t)block * d, 0.0);
    std::fill(ps, ps + (size_t)block * d, 0.0);
    std::fill(pl, pl + (size_t)block * d, 0.0);
    // the kept keys, in list order
    std::vector<int> keys;
    for (int u = 0; u < kc; ++u)
      for (int m = lst[u] * block; m < std::min(N, (lst[u] + 1) * block); ++m) keys.push_back(m);
    std::vector<double> S(keys.size()), P(keys.size()), Pw(keys.size()), acc_c(d);
    for (int r = 0; r < rows; ++r) {
      const int n = lo + r;
      for (size_t u = 0; u < keys.size(); ++u) {
        const int m = keys[u];
        if (quant) {
          const int8_t* qa = qi8 + (bh * NP + n) * d;
          const int8_t* kb = ki8 + (bh * NP + m) * d;
          int32_t acc = 0;   // exact: |acc| <= d * 127^2
          for (int c = 0; c < d; ++c) acc += int32_t(qa[c]) * int32_t(kb[c]);
          const long long ng = NP / gran;   // scale groups per head
          const float cscale = sq[bh * ng + n / gran] * sk[bh * ng + m / gran];
          const float s32 = (float(acc) * cscale) * rsd_f;
          S[u] = double(s32);
        } else {
          double acc = 0.0;
          for (int c = 0; c < d; ++c) {
            double kv = bf16_value(k[(bh * N + m) * d + c]);
            if (smooth) kv -= double(mu[bh * d + c]);
            acc += bf16_value(q[(bh * N + n) * d + c]) * kv;
          }
          S[u] = acc * rsd;
        }
      }
      double mx = -INFINITY;
      for (double sv : S) mx = std::max(mx, sv);
      double l = 0.0;
      for (size_t u = 0; u < keys.size(); ++u) {
        P[u] = std::exp(S[u] - mx);
        l += P[u];
        Pw[u] = pcast ? round_bf16(P[u]) : P[u];
      }
      // (P . V) per channel, the keys added in list order
      std::fill(acc_c.begin(), acc_c.end(), 0.0);
      for (size_t u = 0; u < keys.size(); ++u) {
        const uint16_t* vr = v + (bh * N + keys[u]) * d;
        for (int c = 0; c < d; ++c) acc_c[c] += Pw[u] * bf16_value(vr[c]);
      }
      for (int c = 0; c < d; ++c) ps[(size_t)r * d + c] = acc_c[c] / l;
    }
    // linear part over the blocks of class 1
    bool any_rest = false;
    for (int j = 0; j < nblk; ++j) any_rest = any_rest || row_cls[j] == 1;
    if (any_rest) {
      const std::vector<double>& h = hs[head_of[bh]];
      const std::vector<double>& z = zs[head_of[bh]];
      std::vector<double> hr((size_t)d * d, 0.0), zr(d, 0.0);
      for (int j = 0; j < nblk; ++j) {
        if (row_cls[j] != 1) continue;
        for (int a = 0; a < d; ++a) {
          zr[a] += z[(size_t)j * d + a];
          for (int c = 0; c < d; ++c) hr[(size_t)a * d + c] += h[((size_t)j * d + a) * d + c];
        }
      }
      std::vector<double> pq(d);
      for (int r = 0; r < rows; ++r) {
        const int n = lo + r;
        double den = 0.0;
        for (int a = 0; a < d; ++a) {
          pq[a] = phi(bf16_value(q[(bh * N + n) * d + a]));
          den += pq[a] * zr[a];
        }
        // phi(q) h_rest, the components a added in order
        std::vector<double> num(d, 0.0);
        for (int a = 0; a < d; ++a)
          for (int c = 0; c < d; ++c) num[c] += pq[a] * hr[(size_t)a * d + c];
        for (int c = 0; c < d; ++c) pl[(size_t)r * d + c] = num[c] / den;
      }
    }
    // out = O_sparse + O_lin W, the components a added in order
    std::vector<double> proj(d);
    for (int r = 0; r < rows; ++r) {
      std::fill(proj.begin(), proj.end(), 0.0);
      for (int a = 0; a < d; ++a)
        for (int c = 0; c < d; ++c) proj[c] += pl[(size_t)r * d + a] * W[(size_t)a * d + c];
      for (int c = 0; c < d; ++c) po[(size_t)r * d + c] = ps[(size_t)r * d + c] + proj[c];
    }
  });
  return 0;
}

}  // extern "C"
