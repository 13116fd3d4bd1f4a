// Offline calibration of the key and value rotations, on the host in fp64.
//
// Keys: the quantisation error of a key reaches the output through the logits
// q.k, so its weight is the second moment of the queries; values: through the
// attention output, so the value second moment is weighted by the attention
// each key receives.  The eigenbases of those two matrices, followed by the
// normalised Hadamard and the bit-reversal permutation, are the rotations
// (gen-hub.ru, "Together AI открывает OSCAR…", section "Что придумали в
// Together AI"; calibration is offline and once per model, section
// "Открытый код — это серьёзно").
#include <math.h>
#include <omp.h>

#include <algorithm>
#include <vector>

#include "okv.h"
#include "okv_internal.h"

namespace {

constexpr int kDim = 128;

// Cyclic Jacobi eigenvalue iteration for a symmetric n x n matrix (row-major,
// overwritten).  On return w holds the eigenvalues and the columns of v the
// eigenvectors.  Returns false if the off-diagonal mass does not vanish.
bool jacobi_eigen(std::vector<double>& a, int n, std::vector<double>& w, std::vector<double>& v) {
  v.assign((size_t)n * n, 0.0);
  for (int i = 0; i < n; ++i) v[(size_t)i * n + i] = 1.0;
  double norm = 0.0;
  for (double x : a) norm += x * x;
  if (norm == 0.0) {
    w.assign(n, 0.0);
    return true;
  }
  bool converged = false;
  for (int sweep = 0; sweep < 80; ++sweep) {
    double off = 0.0;
    for (int p = 0; p < n; ++p)
      for (int q = p + 1; q < n; ++q) off += a[(size_t)p * n + q] * a[(size_t)p * n + q];
    if (off <= 1e-32 * norm) {
      converged = true;
      break;
    }
    for (int p = 0; p < n - 1; ++p) {
      for (int q = p + 1; q < n; ++q) {
        const double apq = a[(size_t)p * n + q];
        if (apq == 0.0) continue;
        const double app = a[(size_t)p * n + p], aqq = a[(size_t)q * n + q];
        const double theta = (aqq - app) / (2.0 * apq);
        const double t = (theta >= 0 ? 1.0 : -1.0) / (fabs(theta) + sqrt(theta * theta + 1.0));
        const double c = 1.0 / sqrt(t * t + 1.0), s = t * c;
        for (int r = 0; r < n; ++r) {
          const double arp = a[(size_t)r * n + p], arq = a[(size_t)r * n + q];
          a[(size_t)r * n + p] = c * arp - s * arq;
          a[(size_t)r * n + q] = s * arp + c * arq;
        }
        for (int r = 0; r < n; ++r) {
          const double apr = a[(size_t)p * n + r], aqr = a[(size_t)q * n + r];
          a[(size_t)p * n + r] = c * apr - s * aqr;
          a[(size_t)q * n + r] = s * apr + c * aqr;
        }
        for (int r = 0; r < n; ++r) {
          const double vrp = v[(size_t)r * n + p], vrq = v[(size_t)r * n + q];
          v[(size_t)r * n + p] = c * vrp - s * vrq;
          v[(size_t)r * n + q] = s * vrp + c * vrq;
        }
      }
    }
  }
  w.resize(n);
  for (int i = 0; i < n; ++i) w[i] = a[(size_t)i * n + i];
  return converged;
}

// Columns sorted by descending eigenvalue (ties keep the solver's order), and
// each column signed so its largest-magnitude entry (first on ties) is positive.
void order_and_sign(const std::vector<double>& w, const std::vector<double>& v, int n, std::vector<double>& u) {
  std::vector<int> idx(n);
  for (int i = 0; i < n; ++i) idx[i] = i;
  std::stable_sort(idx.begin(), idx.end(), [&](int x, int y) { return w[x] > w[y]; });
  u.assign((size_t)n * n, 0.0);
  for (int j = 0; j < n; ++j) {
    const int src = idx[j];
    int arg = 0;
    double best = -1.0;
    for (int r = 0; r < n; ++r) {
      const double m = fabs(v[(size_t)r * n + src]);
      if (m > best) {
        best = m;
        arg = r;
      }
    }
    const double sgn = v[(size_t)arg * n + src] < 0 ? -1.0 : 1.0;
    for (int r = 0; r < n; ++r) u[(size_t)r * n + j] = sgn * v[(size_t)r * n + src];
  }
}

int bitrev7(int j) {
  int r = 0;
  for (int b = 0; b < 7; ++b) r |= ((j >> b) & 1) << (6 - b);
  return r;
}

// R = U H P_br: R[c][j] = sum_i U[c][i] H[i][br(j)], H_ij = (-1)^popcount(i&j)/sqrt(d)
void compose_rotation(const std::vector<double>& u, std::vector<double>& r) {
  const double inv = 1.0 / sqrt((double)kDim);
  r.assign((size_t)kDim * kDim, 0.0);
  for (int c = 0; c < kDim; ++c) {
    for (int j = 0; j < kDim; ++j) {
      const int col = bitrev7(j);
      double acc = 0.0;
      for (int i = 0; i < kDim; ++i) {
        const double h = (__builtin_popcount((unsigned)(i & col)) & 1) ? -inv : inv;
        acc += u[(size_t)c * kDim + i] * h;
      }
      r[(size_t)c * kDim + j] = acc;
    }
  }
}

void store(float* dst, int h, const std::vector<double>& m) {
  if (dst == nullptr) return;
  float* o = dst + (size_t)h * kDim * kDim;
  for (size_t i = 0; i < m.size(); ++i) o[i] = (float)m[i];
}

}  // namespace

extern "C" okv_status okv_calibrate_rotations(const float* q, int64_t nq, const float* k, const float* v,
                                              int64_t nk, int32_t hq, int32_t hkv, int32_t d, float* r_k,
                                              float* r_v, float* u_k, float* u_v) {
  using okv::fail;
  if (q == nullptr || k == nullptr || v == nullptr) return fail(OKV_ERR_INVALID_ARG, "q, k, v must be non-NULL");
  if (d != kDim) return fail(OKV_ERR_UNSUPPORTED, "head_dim %d: only 128 is built", d);
  if (nq < 1 || nk < 1) return fail(OKV_ERR_INVALID_ARG, "nq and nk must be >= 1");
  if (hkv < 1 || hq < 1 || hq % hkv != 0) return fail(OKV_ERR_INVALID_ARG, "hq must be a multiple of hkv");
  const int g = hq / hkv;
  const double inv_sqrt_d = 1.0 / sqrt((double)kDim);
  for (int h = 0; h < hkv; ++h) {
    // C_Q: uncentred second moment of the group's queries
    std::vector<double> cq((size_t)kDim * kDim, 0.0);
#pragma omp parallel
    {
      std::vector<double> loc((size_t)kDim * kDim, 0.0);
      double x[kDim];
#pragma omp for schedule(static)
      for (int64_t n = 0; n < nq; ++n) {
        for (int gi = 0; gi < g; ++gi) {
          const float* src = q + ((size_t)n * hq + (size_t)h * g + gi) * kDim;
          for (int c = 0; c < kDim; ++c) x[c] = src[c];
          for (int a = 0; a < kDim; ++a)
            for (int b = 0; b < kDim; ++b) loc[(size_t)a * kDim + b] += x[a] * x[b];
        }
      }
#pragma omp critical
      for (size_t i = 0; i < loc.size(); ++i) cq[i] += loc[i];
    }
    const double nqg = (double)nq * g;
    for (double& x : cq) x /= nqg;

    // attention mass each calibration key receives, summed over all queries
    std::vector<double> kd((size_t)nk * kDim), vd((size_t)nk * kDim);
    for (int64_t j = 0; j < nk; ++j)
      for (int c = 0; c < kDim; ++c) {
        kd[(size_t)j * kDim + c] = k[((size_t)j * hkv + h) * kDim + c];
        vd[(size_t)j * kDim + c] = v[((size_t)j * hkv + h) * kDim + c];
      }
    std::vector<double> mass(nk, 0.0);
    double total = 0.0;
#pragma omp parallel
    {
      std::vector<double> lmass(nk, 0.0), s(nk);
      double ltotal = 0.0;
      double x[kDim];
#pragma omp for schedule(static)
      for (int64_t n = 0; n < nq * g; ++n) {
        const int64_t qi = n / g;
        const int gi = (int)(n % g);
        const float* src = q + ((size_t)qi * hq + (size_t)h * g + gi) * kDim;
        for (int c = 0; c < kDim; ++c) x[c] = src[c];
        double mx = -INFINITY;
        for (int64_t j = 0; j < nk; ++j) {
          const double* kr = &kd[(size_t)j * kDim];
          double acc = 0.0;
          for (int c = 0; c < kDim; ++c) acc += x[c] * kr[c];
          s[j] = acc * inv_sqrt_d;
          mx = std::max(mx, s[j]);
        }
        double z = 0.0;
        for (int64_t j = 0; j < nk; ++j) {
          s[j] = exp(s[j] - mx);
          z += s[j];
        }
        for (int64_t j = 0; j < nk; ++j) {
          const double p = s[j] / z;
          lmass[j] += p;
          ltotal += p;
        }
      }
#pragma omp critical
      {
        for (int64_t j = 0; j < nk; ++j) mass[j] += lmass[j];
        total += ltotal;
      }
    }
    std::vector<double> cs((size_t)kDim * kDim, 0.0);
    for (int64_t j = 0; j < nk; ++j) {
      const double* vr = &vd[(size_t)j * kDim];
      for (int a = 0; a < kDim; ++a)
        for (int b = 0; b < kDim; ++b) cs[(size_t)a * kDim + b] += mass[j] * vr[a] * vr[b];
    }
    for (double& x : cs) x /= total;

    for (int which = 0; which < 2; ++which) {
      std::vector<double> a = which == 0 ? cq : cs;
      std::vector<double> w, vecs, u, r;
      if (!jacobi_eigen(a, kDim, w, vecs))
        return fail(OKV_ERR_NUMERIC, "Jacobi eigensolver did not converge (kv head %d, %s)", h,
                    which == 0 ? "keys" : "values");
      order_and_sign(w, vecs, kDim, u);
      compose_rotation(u, r);
      store(which == 0 ? u_k : u_v, h, u);
      store(which == 0 ? r_k : r_v, h, r);
    }
  }
  return OKV_OK;
}
