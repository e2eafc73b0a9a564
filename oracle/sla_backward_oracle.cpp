// Plain C++ CPU oracle for the SLA fine-tune path: its forward and gradient.
//
// TEST INFRASTRUCTURE ONLY: built into libsla_oracle.so by oracle/build.py and
// loaded through oracle/sla_backward_cpp.py by the tests, never by the
// library; it shares no code with the CUDA sources.  No CUDA kernel computes
// this yet.
//
// Sources: "Turbo Diffusion：秒级生成与高清保真的视频扩散技术突破" (lanhy.cn),
// section 三(二) SLA items 1-2 (kept blocks through softmax attention, the
// rest through an O(N) linear branch with a linear projection) and section 四
// step 1 (SLA fine-tuning: gradients flow through the SLA operator).
//
// Readings (the same as the numpy statement, sla_backward_oracle.py): the
// training forward has no INT8 step; the kept-block lists are fixed inputs;
// one head, float64, row-major [N, d] tensors, W_proj [d, d] applied on the
// right; the gradient is that of L = sum(out * G).
//   out_n = sum_m p_nm v_m + (phi(q_n)^T H_i / phi(q_n).Z_i) W,
//   p_nm = softmax over the kept keys m of q_n.k_m / sqrt(d),
//   H_i, Z_i = sums of h_j = sum phi(k) v^T, z_j = sum phi(k) over the blocks
//   query block i did not keep; phi = elu + 1.
// Plain loops; each sum in the order written.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <vector>

namespace {

double phi1(double x) { return x > 0 ? x + 1.0 : std::exp(x); }
double dphi1(double x) { return x > 0 ? 1.0 : std::exp(x); }

struct Head {
  int N, d, block, nblk;
  const double *q, *k, *v, *w;
  const uint8_t* kept;   // [nblk][nblk]: 1 where query block i keeps key block j
  std::vector<double> h, z;   // [nblk][d][d], [nblk][d]

  Head(const double* q_, const double* k_, const double* v_, const double* w_, const uint8_t* kept_, int N_, int d_,
       int block_)
      : N(N_), d(d_), block(block_), nblk((N_ + block_ - 1) / block_), q(q_), k(k_), v(v_), w(w_), kept(kept_) {
    h.assign((size_t)nblk * d * d, 0.0);
    z.assign((size_t)nblk * d, 0.0);
    for (int j = 0; j < nblk; ++j)
      for (int m = j * block; m < std::min(N, (j + 1) * block); ++m)
        for (int a = 0; a < d; ++a) {
          const double f = phi1(k[(size_t)m * d + a]);
          z[(size_t)j * d + a] += f;
          for (int c = 0; c < d; ++c) h[((size_t)j * d + a) * d + c] += f * v[(size_t)m * d + c];
        }
  }
  int row_end(int i) const { return std::min(N, (i + 1) * block); }
  std::vector<int> keys(int i) const {
    std::vector<int> ks;
    for (int j = 0; j < nblk; ++j)
      if (kept[(size_t)i * nblk + j])
        for (int m = j * block; m < row_end(j); ++m) ks.push_back(m);
    return ks;
  }
  // H_i, Z_i over the blocks not kept; false when every block is kept
  bool rest(int i, std::vector<double>& H, std::vector<double>& Z) const {
    H.assign((size_t)d * d, 0.0);
    Z.assign(d, 0.0);
    bool any = false;
    for (int j = 0; j < nblk; ++j) {
      if (kept[(size_t)i * nblk + j]) continue;
      any = true;
      for (int x = 0; x < d * d; ++x) H[x] += h[(size_t)j * d * d + x];
      for (int a = 0; a < d; ++a) Z[a] += z[(size_t)j * d + a];
    }
    return any;
  }
  // softmax row of query n over keys ks: p (normalised) and o_s
  void softmax_row(int n, const std::vector<int>& ks, std::vector<double>& p, std::vector<double>& os) const {
    const double sc = 1.0 / std::sqrt((double)d);
    p.assign(ks.size(), 0.0);
    double mx = -INFINITY;
    for (size_t t = 0; t < ks.size(); ++t) {
      double s = 0.0;
      for (int c = 0; c < d; ++c) s += q[(size_t)n * d + c] * k[(size_t)ks[t] * d + c];
      p[t] = s * sc;
      mx = std::max(mx, p[t]);
    }
    double l = 0.0;
    for (double& x : p) {
      x = std::exp(x - mx);
      l += x;
    }
    for (double& x : p) x /= l;
    os.assign(d, 0.0);
    for (size_t t = 0; t < ks.size(); ++t)
      for (int c = 0; c < d; ++c) os[c] += p[t] * v[(size_t)ks[t] * d + c];
  }
  // O_lin row of query n: f = phi(q_n), a = f H, b = f . Z, ol = a / b
  void linear_row(int n, const std::vector<double>& H, const std::vector<double>& Z, std::vector<double>& f,
                  std::vector<double>& ol, double& b) const {
    f.assign(d, 0.0);
    ol.assign(d, 0.0);
    b = 0.0;
    for (int a = 0; a < d; ++a) {
      f[a] = phi1(q[(size_t)n * d + a]);
      b += f[a] * Z[a];
    }
    for (int c = 0; c < d; ++c) {
      double s = 0.0;
      for (int a = 0; a < d; ++a) s += f[a] * H[(size_t)a * d + c];
      ol[c] = s / b;
    }
  }
};

}  // namespace

extern "C" {

// out [N, d] of the fine-tune forward.
void ora_sla_train_forward(const double* q, const double* k, const double* v, const double* w, const uint8_t* kept,
                           int N, int d, int block, double* out) {
  Head hd(q, k, v, w, kept, N, d, block);
  std::vector<double> p, os, H, Z, f, ol;
  for (int i = 0; i < hd.nblk; ++i) {
    const std::vector<int> ks = hd.keys(i);
    const bool lin = hd.rest(i, H, Z);
    for (int n = i * block; n < hd.row_end(i); ++n) {
      hd.softmax_row(n, ks, p, os);
      for (int c = 0; c < d; ++c) out[(size_t)n * d + c] = os[c];
      if (!lin) continue;
      double b;
      hd.linear_row(n, H, Z, f, ol, b);
      for (int c = 0; c < d; ++c) {
        double s = 0.0;
        for (int r = 0; r < d; ++r) s += ol[r] * w[(size_t)r * d + c];
        out[(size_t)n * d + c] += s;
      }
    }
  }
}

// Gradients of sum(out * g): dq, dk, dv [N, d], dw [d, d] (overwritten).
void ora_sla_train_backward(const double* q, const double* k, const double* v, const double* w, const uint8_t* kept,
                            int N, int d, int block, const double* g, double* dq, double* dk, double* dv,
                            double* dw) {
  Head hd(q, k, v, w, kept, N, d, block);
  const int nblk = hd.nblk;
  const double sc = 1.0 / std::sqrt((double)d);
  std::fill(dq, dq + (size_t)N * d, 0.0);
  std::fill(dk, dk + (size_t)N * d, 0.0);
  std::fill(dv, dv + (size_t)N * d, 0.0);
  std::fill(dw, dw + (size_t)d * d, 0.0);
  std::vector<double> dh((size_t)nblk * d * d, 0.0), dz((size_t)nblk * d, 0.0);
  std::vector<double> p, os, H, Z, f, ol, dH, dZ, dol(d), dA(d);
  for (int i = 0; i < nblk; ++i) {
    const std::vector<int> ks = hd.keys(i);
    const bool lin = hd.rest(i, H, Z);
    dH.assign((size_t)d * d, 0.0);
    dZ.assign(d, 0.0);
    for (int n = i * block; n < hd.row_end(i); ++n) {
      const double* gn = g + (size_t)n * d;
      // softmax attention over the kept keys
      hd.softmax_row(n, ks, p, os);
      double D = 0.0;
      for (int c = 0; c < d; ++c) D += gn[c] * os[c];
      for (size_t t = 0; t < ks.size(); ++t) {
        const int m = ks[t];
        double dp = 0.0;
        for (int c = 0; c < d; ++c) {
          dv[(size_t)m * d + c] += p[t] * gn[c];
          dp += gn[c] * v[(size_t)m * d + c];
        }
        const double ds = p[t] * (dp - D);
        for (int c = 0; c < d; ++c) {
          dq[(size_t)n * d + c] += ds * k[(size_t)m * d + c] * sc;
          dk[(size_t)m * d + c] += ds * q[(size_t)n * d + c] * sc;
        }
      }
      if (!lin) continue;
      // linear branch: out += (a / b) W with a = f H, b = f . Z
      double b;
      hd.linear_row(n, H, Z, f, ol, b);
      for (int r = 0; r < d; ++r) {
        double s = 0.0;
        for (int c = 0; c < d; ++c) {
          dw[(size_t)r * d + c] += ol[r] * gn[c];
          s += gn[c] * w[(size_t)r * d + c];
        }
        dol[r] = s;
      }
      double db = 0.0;
      for (int c = 0; c < d; ++c) {
        dA[c] = dol[c] / b;
        db -= dol[c] * ol[c];
      }
      db /= b;
      for (int a = 0; a < d; ++a) {
        double df = db * Z[a];
        for (int c = 0; c < d; ++c) df += dA[c] * H[(size_t)a * d + c];
        dq[(size_t)n * d + a] += df * dphi1(q[(size_t)n * d + a]);
        for (int c = 0; c < d; ++c) dH[(size_t)a * d + c] += f[a] * dA[c];
        dZ[a] += f[a] * db;
      }
    }
    if (!lin) continue;
    for (int j = 0; j < nblk; ++j) {
      if (hd.kept[(size_t)i * nblk + j]) continue;
      for (int x = 0; x < d * d; ++x) dh[(size_t)j * d * d + x] += dH[x];
      for (int a = 0; a < d; ++a) dz[(size_t)j * d + a] += dZ[a];
    }
  }
  // through the states: h_j = sum phi(k_m) v_m^T, z_j = sum phi(k_m)
  for (int j = 0; j < nblk; ++j)
    for (int m = j * block; m < hd.row_end(j); ++m)
      for (int a = 0; a < d; ++a) {
        const double km = k[(size_t)m * d + a];
        double df = dz[(size_t)j * d + a];
        for (int c = 0; c < d; ++c) {
          df += v[(size_t)m * d + c] * dh[((size_t)j * d + a) * d + c];
          dv[(size_t)m * d + c] += phi1(km) * dh[((size_t)j * d + a) * d + c];
        }
        dk[(size_t)m * d + a] += df * dphi1(km);
      }
}

}  // extern "C"
