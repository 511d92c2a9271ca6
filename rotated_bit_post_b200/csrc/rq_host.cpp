// Host-side preparation for the rotated W4A4 linear layer: the RPBH rotation
// tables, the Lloyd-Max codebook of the rotated-coordinate marginal, the PCA
// basis of the low-rank branch, and an E4M3 encoder for codebook centroids.
// Everything here runs once per layer (offline); nothing runs per token.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#include "rq_host.h"

namespace rq {

// ---------------------------------------------------------------- SplitMix64
// Steele, Lea & Flood (2014): state advances by the golden-ratio gamma, the
// output is the state passed through the 64-bit finaliser.
struct SplitMix64 {
  uint64_t s;
  explicit SplitMix64(uint64_t seed) : s(seed) {}
  uint64_t next() {
    s += 0x9E3779B97F4A7C15ull;
    uint64_t z = s;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
  }
  // uniform in [0, n): reject draws at or above the largest multiple of n
  uint64_t below(uint64_t n) {
    const uint64_t rem = (0ull - n) % n;  // 2^64 mod n
    while (true) {
      const uint64_t z = next();
      if (rem == 0 || z < 0ull - rem) return z % n;
    }
  }
};

void make_rotation(int K, uint64_t seed, int8_t* sign, int32_t* perm, int32_t* rot) {
  SplitMix64 g(seed);
  std::vector<int8_t> sg(K);
  for (int k = 0; k < K; ++k) sg[k] = (g.next() >> 63) ? -1 : 1;
  std::vector<int32_t> p(K);
  for (int k = 0; k < K; ++k) p[k] = k;
  for (int i = K - 1; i > 0; --i) {
    const int j = (int)g.below((uint64_t)i + 1);
    std::swap(p[i], p[j]);
  }
  if (sign) std::memcpy(sign, sg.data(), K);
  if (perm) std::memcpy(perm, p.data(), (size_t)K * 4);
  if (rot)
    for (int i = 0; i < K; ++i) rot[i] = p[i] | (sg[p[i]] < 0 ? (int32_t)0x80000000u : 0);
}

// ---------------------------------------------------------------- E4M3
// OCP FP8 E4M3: bias 7, 3 mantissa bits, subnormals m/8 * 2^-6, largest finite
// 448 (code 0x7E; 0x7F is NaN).  Round to nearest even, saturate to 448.
uint8_t e4m3_encode(double v) {
  const uint8_t sgn = std::signbit(v) ? 0x80 : 0;
  double a = std::fabs(v);
  if (!(a < 448.0)) return sgn | 0x7E;
  uint32_t code;
  if (a < std::ldexp(1.0, -6)) {
    const double m = std::nearbyint(a * 512.0);  // units of 2^-9, ties to even
    code = (uint32_t)m;                          // m == 8 is the smallest normal, code 0x08
  } else {
    int e;
    std::frexp(a, &e);  // a = f * 2^e, f in [0.5, 1)
    e -= 1;             // a = (1 + t) * 2^e
    const double m = std::nearbyint((std::ldexp(a, -e) - 1.0) * 8.0);
    code = (uint32_t)((e + 7) << 3) + (uint32_t)m;  // m == 8 carries into the exponent
  }
  if (code > 0x7E) code = 0x7E;
  return sgn | (uint8_t)code;
}

// ---------------------------------------------------------------- Lloyd-Max
namespace {

// 20-point Gauss-Legendre nodes on [-1, 1], generated once by Newton iteration
// on the Legendre polynomial.
struct GaussLegendre {
  static constexpr int N = 20;
  double x[N], w[N];
  GaussLegendre() {
    for (int i = 0; i < N; ++i) {
      double z = std::cos(M_PI * (i + 0.75) / (N + 0.5));
      for (int it = 0; it < 100; ++it) {
        double p0 = 1.0, p1 = 0.0;
        for (int j = 1; j <= N; ++j) {
          const double p2 = p1;
          p1 = p0;
          p0 = ((2.0 * j - 1.0) * z * p1 - (j - 1.0) * p2) / j;
        }
        const double dp = N * (z * p0 - p1) / (z * z - 1.0);
        const double dz = p0 / dp;
        z -= dz;
        if (std::fabs(dz) < 1e-16) {
          x[i] = z;
          w[i] = 2.0 / ((1.0 - z * z) * dp * dp);
          break;
        }
        x[i] = z;
        w[i] = 2.0 / ((1.0 - z * z) * dp * dp);
      }
    }
  }
};

// Unnormalised density (1 - u^2/K)^alpha on [0, top); moments over [a, b] by
// composite Gauss-Legendre on panels no wider than 1/32.
struct Marginal {
  double K, alpha, top;
  const GaussLegendre& gl;
  Marginal(int K_, const GaussLegendre& g)
      : K(K_), alpha((K_ - 3) / 2.0), top(std::min(std::sqrt((double)K_), 40.0)), gl(g) {}
  double g(double u) const {
    const double t = u * u / K;
    return t >= 1.0 ? 0.0 : std::exp(alpha * std::log1p(-t));
  }
  void moments(double a, double b, double& m0, double& m1) const {
    b = std::min(b, top);
    m0 = m1 = 0.0;
    if (b <= a) return;
    const int panels = std::max(1, (int)std::ceil((b - a) * 32.0));
    const double h = (b - a) / panels;
    for (int p = 0; p < panels; ++p) {
      const double lo = a + p * h, mid = lo + 0.5 * h;
      for (int i = 0; i < GaussLegendre::N; ++i) {
        const double u = mid + 0.5 * h * gl.x[i];
        const double f = gl.w[i] * g(u) * 0.5 * h;
        m0 += f;
        m1 += f * u;
      }
    }
  }
};

}  // namespace

bool lloyd_max(int K, int levels, std::vector<double>& cent, std::vector<double>& bnd) {
  static const GaussLegendre gl;
  const Marginal mg(K, gl);
  const int h = levels / 2;
  std::vector<double> c(h), nb(h + 1);
  for (int i = 0; i < h; ++i) c[i] = (i + 0.5) * 3.0 / h;
  bool done = false;
  for (int it = 0; it < 200000 && !done; ++it) {
    nb[0] = 0.0;
    for (int i = 0; i + 1 < h; ++i) nb[i + 1] = 0.5 * (c[i] + c[i + 1]);
    nb[h] = mg.top;
    double delta = 0.0;
    for (int i = 0; i < h; ++i) {
      double m0, m1;
      mg.moments(nb[i], nb[i + 1], m0, m1);
      const double v = m1 / m0;
      delta = std::max(delta, std::fabs(v - c[i]));
      c[i] = v;
    }
    done = delta < 1e-13;
  }
  if (!done) return false;
  cent.assign(levels, 0.0);
  bnd.assign(levels - 1, 0.0);
  for (int i = 0; i < h; ++i) {
    cent[h + i] = c[i];
    cent[h - 1 - i] = -c[i];
  }
  bnd[h - 1] = 0.0;
  for (int i = 0; i + 1 < h; ++i) {
    const double b = 0.5 * (c[i] + c[i + 1]);
    bnd[h + i] = b;
    bnd[h - 2 - i] = -b;
  }
  return true;
}

// ---------------------------------------------------------------- PCA
// Cyclic Jacobi eigen-decomposition of a symmetric n x n matrix (row-major);
// eigenvalues on the diagonal of A, eigenvectors in the columns of V.
static void jacobi_eigen(std::vector<double>& A, std::vector<double>& V, int n) {
  V.assign((size_t)n * n, 0.0);
  for (int i = 0; i < n; ++i) V[(size_t)i * n + i] = 1.0;
  for (int sweep = 0; sweep < 100; ++sweep) {
    double off = 0.0, diag = 0.0;
    for (int i = 0; i < n; ++i) {
      diag += A[(size_t)i * n + i] * A[(size_t)i * n + i];
      for (int j = i + 1; j < n; ++j) off += A[(size_t)i * n + j] * A[(size_t)i * n + j];
    }
    if (off <= 1e-30 * diag) break;
    for (int p = 0; p < n - 1; ++p) {
      for (int q = p + 1; q < n; ++q) {
        const double apq = A[(size_t)p * n + q];
        if (std::fabs(apq) < 1e-300) continue;
        const double app = A[(size_t)p * n + p], aqq = A[(size_t)q * n + q];
        const double theta = (aqq - app) / (2.0 * apq);
        const double t = (theta >= 0 ? 1.0 : -1.0) / (std::fabs(theta) + std::sqrt(theta * theta + 1.0));
        const double c = 1.0 / std::sqrt(t * t + 1.0), s = t * c;
        for (int k = 0; k < n; ++k) {  // rows p, q
          const double akp = A[(size_t)p * n + k], akq = A[(size_t)q * n + k];
          A[(size_t)p * n + k] = c * akp - s * akq;
          A[(size_t)q * n + k] = s * akp + c * akq;
        }
        for (int k = 0; k < n; ++k) {  // columns p, q
          const double akp = A[(size_t)k * n + p], akq = A[(size_t)k * n + q];
          A[(size_t)k * n + p] = c * akp - s * akq;
          A[(size_t)k * n + q] = s * akp + c * akq;
        }
        for (int k = 0; k < n; ++k) {
          const double vkp = V[(size_t)k * n + p], vkq = V[(size_t)k * n + q];
          V[(size_t)k * n + p] = c * vkp - s * vkq;
          V[(size_t)k * n + q] = s * vkp + c * vkq;
        }
      }
    }
  }
}

static inline double bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

uint16_t float_to_bf16_rne(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

bool pca_basis(const uint16_t* calib, int n, int K, int r, uint16_t* U, double* evals) {
  // S = X^T X / n shares its non-zero spectrum with G = X X^T / n; for an
  // eigenpair (lambda, v) of G, u = X^T v / sqrt(n lambda) is a unit eigenvector of S.
  std::vector<double> X((size_t)n * K);
  for (size_t i = 0; i < X.size(); ++i) X[i] = bf16_to_double(calib[i]);
  std::vector<double> G((size_t)n * n, 0.0), V;
  for (int i = 0; i < n; ++i)
    for (int j = i; j < n; ++j) {
      double s = 0.0;
      const double* xi = &X[(size_t)i * K];
      const double* xj = &X[(size_t)j * K];
      for (int k = 0; k < K; ++k) s += xi[k] * xj[k];
      G[(size_t)i * n + j] = G[(size_t)j * n + i] = s / n;
    }
  jacobi_eigen(G, V, n);
  std::vector<int> order(n);
  for (int i = 0; i < n; ++i) order[i] = i;
  std::sort(order.begin(), order.end(),
            [&](int a, int b) { return G[(size_t)a * n + a] > G[(size_t)b * n + b]; });
  std::vector<double> u(K);
  for (int j = 0; j < r; ++j) {
    const int e = order[j];
    const double lam = G[(size_t)e * n + e];
    if (!(lam > 0)) return false;
    std::fill(u.begin(), u.end(), 0.0);
    for (int i = 0; i < n; ++i) {
      const double vi = V[(size_t)i * n + e];
      const double* xi = &X[(size_t)i * K];
      for (int k = 0; k < K; ++k) u[k] += vi * xi[k];
    }
    double nrm = 0.0;
    for (int k = 0; k < K; ++k) nrm += u[k] * u[k];
    nrm = std::sqrt(nrm);
    int imax = 0;
    for (int k = 1; k < K; ++k)
      if (std::fabs(u[k]) > std::fabs(u[imax])) imax = k;
    const double sgn = u[imax] < 0 ? -1.0 : 1.0;
    for (int k = 0; k < K; ++k) U[(size_t)k * r + j] = float_to_bf16_rne((float)(sgn * u[k] / nrm));
    if (evals) evals[j] = lam;
  }
  return true;
}

// TR-DQ's zigzag permutation (section 3.2): channels ranked by magnitude,
// largest first (equal magnitudes: lower index first), dealt to the K/block
// blocks back and forth (0 .. nblk-1, then nblk-1 .. 0, ...), keeping inside
// each block the order in which they arrive.  perm[i] is the channel read at
// position i; rot2 is the same table as a signed permutation (no signs).
void make_zigzag(const float* mag, int K, int block, int32_t* perm, int32_t* rot2) {
  std::vector<int> order(K);
  for (int i = 0; i < K; ++i) order[i] = i;
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return mag[a] > mag[b]; });
  const int nblk = K / block;
  std::vector<int32_t> p(K);
  for (int t = 0; t < K; ++t) {
    const int rnd = t / nblk, i = t % nblk;
    const int blk = (rnd % 2 == 0) ? i : nblk - 1 - i;
    p[(size_t)blk * block + rnd] = order[t];
  }
  for (int i = 0; i < K; ++i) {
    if (perm) perm[i] = p[i];
    if (rot2) rot2[i] = p[i];
  }
}

}  // namespace rq
