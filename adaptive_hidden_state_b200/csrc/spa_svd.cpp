// Host-side truncated SVD for the singular proxy W_r = Lambda_r V_r^T.
//
// SPA-Cache takes the top-r right singular vectors and values of the Value
// projection offline (papernotes.org, 关键设计 2).  Only the top r are needed,
// so this runs randomised block subspace iteration on W^T W in double
// precision with a block of b = min(d, 2r + 16) vectors (oversampling makes
// the convergence rate (sigma_{b+1}/sigma_r)^2 per iteration instead of the
// tiny sigma_{r+1}/sigma_r gap), orthonormalises with block classical
// Gram-Schmidt run twice (Gram-Schmidt within each block), and finishes with a
// Rayleigh-Ritz step: a cyclic Jacobi eigensolver on Q^T W^T W Q.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace spa {

namespace {

// C[m x n] = A[m x k] (row-major, lda) * B[k x n] (row-major), or A^T when transA.
void gemm_rm(bool transA, int m, int n, int k, const double* A, int lda, const double* B,
             double* C) {
  const int MB = 32, KB = 256;
#pragma omp parallel for schedule(dynamic, 1)
  for (int i0 = 0; i0 < m; i0 += MB) {
    const int i1 = std::min(m, i0 + MB);
    for (int i = i0; i < i1; ++i) std::memset(C + (size_t)i * n, 0, sizeof(double) * n);
    for (int k0 = 0; k0 < k; k0 += KB) {
      const int k1 = std::min(k, k0 + KB);
      for (int i = i0; i < i1; ++i) {
        double* c = C + (size_t)i * n;
        for (int kk = k0; kk < k1; ++kk) {
          const double a = transA ? A[(size_t)kk * lda + i] : A[(size_t)i * lda + kk];
          const double* b = B + (size_t)kk * n;
#pragma omp simd
          for (int j = 0; j < n; ++j) c[j] += a * b[j];
        }
      }
    }
  }
}

// Z (d x b, row-major) <- orthonormal basis of its column span.
void orthonormalise(std::vector<double>& Z, int d, int b) {
  const int BS = 32;
  std::vector<double> coef;
  for (int j0 = 0; j0 < b; j0 += BS) {
    const int j1 = std::min(b, j0 + BS), w = j1 - j0;
    for (int pass = 0; pass < 2; ++pass) {
      if (j0 > 0) {
        // coef[j0 x w] = Q_prev^T Z_J ; Z_J -= Q_prev coef
        coef.assign((size_t)j0 * w, 0.0);
#pragma omp parallel
        {
          std::vector<double> loc((size_t)j0 * w, 0.0);
#pragma omp for schedule(static)
          for (int i = 0; i < d; ++i) {
            const double* z = &Z[(size_t)i * b];
            for (int p = 0; p < j0; ++p) {
              const double q = z[p];
              double* l = &loc[(size_t)p * w];
              for (int c = 0; c < w; ++c) l[c] += q * z[j0 + c];
            }
          }
#pragma omp critical
          for (size_t t = 0; t < loc.size(); ++t) coef[t] += loc[t];
        }
#pragma omp parallel for schedule(static)
        for (int i = 0; i < d; ++i) {
          double* z = &Z[(size_t)i * b];
          for (int c = 0; c < w; ++c) {
            double s = 0.0;
            for (int p = 0; p < j0; ++p) s += z[p] * coef[(size_t)p * w + c];
            z[j0 + c] -= s;
          }
        }
      }
      // modified Gram-Schmidt inside the block
      for (int c = j0; c < j1; ++c) {
        for (int p = j0; p < c; ++p) {
          double s = 0.0;
          for (int i = 0; i < d; ++i) s += Z[(size_t)i * b + p] * Z[(size_t)i * b + c];
          for (int i = 0; i < d; ++i) Z[(size_t)i * b + c] -= s * Z[(size_t)i * b + p];
        }
        double nn = 0.0;
        for (int i = 0; i < d; ++i) nn += Z[(size_t)i * b + c] * Z[(size_t)i * b + c];
        nn = std::sqrt(nn);
        const double inv = nn > 0.0 ? 1.0 / nn : 0.0;
        for (int i = 0; i < d; ++i) Z[(size_t)i * b + c] *= inv;
      }
    }
  }
}

// Cyclic Jacobi eigendecomposition of the symmetric n x n matrix A (row-major).
// On return A's diagonal holds the eigenvalues and V (row-major) the
// eigenvectors as columns.
void jacobi_eig(std::vector<double>& A, std::vector<double>& V, int n) {
  V.assign((size_t)n * n, 0.0);
  for (int i = 0; i < n; ++i) V[(size_t)i * n + i] = 1.0;
  for (int sweep = 0; sweep < 60; ++sweep) {
    double off = 0.0, diag = 0.0;
    for (int i = 0; i < n; ++i)
      for (int j = 0; j < n; ++j) {
        const double a = A[(size_t)i * n + j];
        if (i != j) off += a * a; else diag += a * a;
      }
    if (off <= 1e-30 * diag || off == 0.0) break;
    for (int p = 0; p < n - 1; ++p)
      for (int q = p + 1; q < n; ++q) {
        const double apq = A[(size_t)p * n + q];
        if (std::fabs(apq) < 1e-300) continue;
        const double app = A[(size_t)p * n + p], aqq = A[(size_t)q * n + q];
        const double theta = (aqq - app) / (2.0 * apq);
        const double t = (theta >= 0 ? 1.0 : -1.0) / (std::fabs(theta) + std::sqrt(theta * theta + 1.0));
        const double c = 1.0 / std::sqrt(t * t + 1.0), s = t * c;
        for (int k = 0; k < n; ++k) {  // columns p, q
          const double akp = A[(size_t)k * n + p], akq = A[(size_t)k * n + q];
          A[(size_t)k * n + p] = c * akp - s * akq;
          A[(size_t)k * n + q] = s * akp + c * akq;
        }
        for (int k = 0; k < n; ++k) {  // rows p, q
          const double apk = A[(size_t)p * n + k], aqk = A[(size_t)q * n + k];
          A[(size_t)p * n + k] = c * apk - s * aqk;
          A[(size_t)q * n + k] = s * apk + c * aqk;
        }
        for (int k = 0; k < n; ++k) {
          const double vkp = V[(size_t)k * n + p], vkq = V[(size_t)k * n + q];
          V[(size_t)k * n + p] = c * vkp - s * vkq;
          V[(size_t)k * n + q] = s * vkp + c * vkq;
        }
      }
  }
}

uint64_t splitmix64(uint64_t& x) {
  uint64_t z = (x += 0x9E3779B97F4A7C15ull);
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

}  // namespace

// w_v: [d, d] float, row-major [out, in].  w_r: [r, d] float output.
int singular_proxy_host(const float* w_v, int d, int r, float* w_r, int iters) {
  if (!w_v || !w_r || d < 1 || r < 1 || r > d) return -1;
  const int b = std::min(d, 2 * r + 16);
  std::vector<double> W((size_t)d * d);
  for (size_t i = 0; i < W.size(); ++i) W[i] = (double)w_v[i];
  // Gaussian start block (Box-Muller on a fixed splitmix64 stream)
  std::vector<double> Q((size_t)d * b), Y((size_t)d * b);
  uint64_t st = 0x5A5A1234ull;
  for (size_t i = 0; i < Q.size(); ++i) {
    const double u1 = ((splitmix64(st) >> 11) + 0.5) * (1.0 / 9007199254740992.0);
    const double u2 = ((splitmix64(st) >> 11) + 0.5) * (1.0 / 9007199254740992.0);
    Q[i] = std::sqrt(-2.0 * std::log(u1)) * std::cos(6.283185307179586 * u2);
  }
  orthonormalise(Q, d, b);
  for (int it = 0; it < iters; ++it) {
    gemm_rm(false, d, b, d, W.data(), d, Q.data(), Y.data());  // Y = W Q
    gemm_rm(true, d, b, d, W.data(), d, Y.data(), Q.data());   // Q = W^T Y
    orthonormalise(Q, d, b);
  }
  // Rayleigh-Ritz on W^T W restricted to span(Q): G = (W Q)^T (W Q)
  gemm_rm(false, d, b, d, W.data(), d, Q.data(), Y.data());
  std::vector<double> G((size_t)b * b, 0.0), E;
  gemm_rm(true, b, b, d, Y.data(), b, Y.data(), G.data());
  jacobi_eig(G, E, b);
  std::vector<int> order(b);
  for (int i = 0; i < b; ++i) order[i] = i;
  std::sort(order.begin(), order.end(), [&](int x, int y) {
    return G[(size_t)x * b + x] > G[(size_t)y * b + y];
  });
  for (int i = 0; i < r; ++i) {
    const int e = order[i];
    const double sigma = std::sqrt(std::max(0.0, G[(size_t)e * b + e]));
    // v = Q E[:, e]
    std::vector<double> v(d, 0.0);
    for (int row = 0; row < d; ++row) {
      double s = 0.0;
      for (int c = 0; c < b; ++c) s += Q[(size_t)row * b + c] * E[(size_t)c * b + e];
      v[row] = s;
    }
    int jmax = 0;
    for (int j = 1; j < d; ++j)
      if (std::fabs(v[j]) > std::fabs(v[jmax])) jmax = j;
    const double sgn = v[jmax] < 0 ? -1.0 : 1.0;
    for (int j = 0; j < d; ++j) w_r[(size_t)i * d + j] = (float)(sgn * sigma * v[j]);
  }
  return 0;
}

}  // namespace spa
