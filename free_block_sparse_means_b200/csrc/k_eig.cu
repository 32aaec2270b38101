// Leading eigenpairs of the small symmetric d x d matrices of the call: the
// sampled-query response metric M_K [paperlayer App. B.1] and the weighted
// probe-residual Gram matrix [paperlayer App. A.3].
//
// One block per matrix, everything in shared memory, fp32, following the
// textbook route for a few eigenpairs of a dense symmetric matrix (Golub & Van
// Loan, "Matrix Computations": Householder tridiagonalisation §8.3.1,
// bisection on Sturm sequence counts §8.4.1, inverse iteration §7.6.1):
//   1. A = Q T Q^T with T tridiagonal: n-2 Householder reflectors, each applied
//      to the trailing block as a symmetric rank-2 update (3 barriers each;
//      the matrix-vector product and the update go one warp per row).
//   2. The K largest eigenvalues of T by multisection: a group of G lanes of
//      one warp evaluates the Sturm count (number of eigenvalues below x, i.e.
//      negative pivots of T - xI = L D L^T) at G points per step.
//   3. Eigenvectors of T by inverse iteration on (T - lambda I) with partial
//      pivoting, then orthonormalised in descending eigenvalue order by
//      Cholesky QR (Y Y^T = L L^T, Y <- L^-1 Y).
//   4. Back-transformation x = H_0 H_1 ... H_{n-3} y.
// Outputs: evals[m][k] (descending, k < K), evecs[m][row][k] (stride n), and
// the trace of each matrix.
#include <float.h>

#include "spr_internal.cuh"

namespace spr {

constexpr int EIG_THREADS = 512;

template <int NN>
__device__ int sturm_count(const float* a, const float* b2, float pivmin, float x) {
  int c = 0;
  float q = a[0] - x;
  if (fabsf(q) < pivmin) q = -pivmin;
  c += q < 0.f;
  for (int i = 1; i < NN; ++i) {
    q = (a[i] - x) - __fdividef(b2[i - 1], q);
    if (fabsf(q) < pivmin) q = -pivmin;
    c += q < 0.f;
  }
  return c;
}

template <int NN>
__global__ void __launch_bounds__(EIG_THREADS) k_eig_top(const float* Ain, int K, float* evals,
                                                        float* evecs, float* trace_out) {
  constexpr int LD = NN + 1;
  extern __shared__ __align__(16) float esm[];
  float* A = esm;                // NN x LD; later the eigenvectors Y (K x LD)
  float* Vh = A + NN * LD;       // NN x NN reflectors, row j = v_j (entries j+1..)
  float* ta = Vh + NN * NN;      // diag of T
  float* tb = ta + NN;           // off-diagonal of T (tb[i] couples i, i+1)
  float* tb2 = tb + NN;          // tb^2
  float* tau = tb2 + NN;         // reflector scales
  float* lam = tau + NN;         // eigenvalues (K)
  float* pw = lam + NN;          // p = tau A22 v
  float* misc = pw + NN;         // [8], then the Cholesky-QR Gram matrix
  const int m = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* src = Ain + (size_t)m * NN * NN;
  for (int e = tid; e < NN * NN; e += EIG_THREADS) {
    const int i = e / NN, j = e % NN;
    A[i * LD + j] = 0.5f * (src[i * NN + j] + src[j * NN + i]);
  }
  __syncthreads();
  if (warp == 0) {
    float t = 0.f;
    for (int i = lane; i < NN; i += 32) t += A[i * LD + i];
    t = warp_sum(t);
    if (lane == 0 && trace_out) trace_out[m] = t;
  }
  // ---- 1. tridiagonalisation --------------------------------------------
  for (int k = 0; k < NN - 2; ++k) {
    const int r0 = k + 1, mlen = NN - r0;
    if (warp == 0) {
      float sig = 0.f;
      for (int i = r0 + 1 + lane; i < NN; i += 32) {
        const float x = A[i * LD + k];
        sig += x * x;
      }
      sig = warp_sum(sig);
      const float x0 = A[r0 * LD + k];
      float t = 0.f, alpha = x0, v0 = 0.f;
      if (sig > 0.f) {
        const float nrm = sqrtf(x0 * x0 + sig);
        alpha = x0 >= 0.f ? -nrm : nrm;
        v0 = x0 - alpha;
        t = 2.f / (v0 * v0 + sig);
      }
      for (int i = r0 + lane; i < NN; i += 32)
        Vh[k * NN + i] = (t == 0.f) ? 0.f : (i == r0 ? v0 : A[i * LD + k]);
      if (lane == 0) {
        tau[k] = t;
        ta[k] = A[k * LD + k];
        tb[k] = alpha;
      }
    }
    __syncthreads();
    const float t = tau[k];
    if (t != 0.f) {
      const float* v = Vh + k * NN;
      // p = t A22 v, one thread per row; A22 is kept exactly symmetric, so the
      // thread reads its column (consecutive threads, consecutive addresses)
      if (tid >= r0 && tid < NN) {
        float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
        int j = r0;
        for (; j + 3 < NN; j += 4) {
          s0 += A[j * LD + tid] * v[j];
          s1 += A[(j + 1) * LD + tid] * v[j + 1];
          s2 += A[(j + 2) * LD + tid] * v[j + 2];
          s3 += A[(j + 3) * LD + tid] * v[j + 3];
        }
        for (; j < NN; ++j) s0 += A[j * LD + tid] * v[j];
        pw[tid] = t * ((s0 + s1) + (s2 + s3));
      }
      __syncthreads();
      float kk = 0.f;  // (t / 2) p.v, every warp for itself
      for (int j = r0 + lane; j < NN; j += 32) kk += pw[j] * v[j];
      kk = 0.5f * t * warp_sum(kk);
      for (int i = r0 + warp; i < NN; i += EIG_THREADS / 32) {
        const float vi = v[i], wi = pw[i] - kk * vi;
        for (int j = r0 + lane; j < NN; j += 32) {
          const float vj = v[j];
          A[i * LD + j] -= vi * (pw[j] - kk * vj) + wi * vj;
        }
      }
      __syncthreads();
    }
  }
  if (tid == 0) {
    ta[NN - 2] = A[(NN - 2) * LD + NN - 2];
    ta[NN - 1] = A[(NN - 1) * LD + NN - 1];
    tb[NN - 2] = A[(NN - 1) * LD + NN - 2];
    tau[NN - 2] = 0.f;
    tb[NN - 1] = 0.f;
  }
  __syncthreads();
  for (int i = tid; i < NN; i += EIG_THREADS) tb2[i] = tb[i] * tb[i];
  if (warp == 0) {
    float lo = FLT_MAX, hi = -FLT_MAX, bmax = 0.f;
    for (int i = lane; i < NN; i += 32) {
      const float r = (i > 0 ? fabsf(tb[i - 1]) : 0.f) + (i < NN - 1 ? fabsf(tb[i]) : 0.f);
      lo = fminf(lo, ta[i] - r);
      hi = fmaxf(hi, ta[i] + r);
      bmax = fmaxf(bmax, tb[i] * tb[i]);
    }
    for (int o = 16; o > 0; o >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
      bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, o));
    }
    if (lane == 0) {
      const float span = fmaxf(fabsf(lo), fabsf(hi));
      misc[0] = lo - 1e-6f * span - 1e-30f;
      misc[1] = hi + 1e-6f * span + 1e-30f;
      misc[2] = 1e-30f * fmaxf(1.f, bmax);
      misc[3] = fmaxf(span, 1e-30f);
    }
  }
  __syncthreads();
  // ---- 2. K largest eigenvalues by multisection --------------------------
  {
    int G = 32;
    while (G > 1 && G * K > EIG_THREADS) G >>= 1;
    const int groups_per_pass = EIG_THREADS / G;
    const float pivmin = misc[2], span = misc[3];
    for (int e0 = 0; e0 < K; e0 += groups_per_pass) {
      const int e = e0 + tid / G, s = tid % G;
      const unsigned gmask = (G == 32) ? 0xffffffffu : (((1u << G) - 1u) << (lane & ~(G - 1)));
      float lo = misc[0], hi = misc[1];
      const int j = NN - 1 - (e < K ? e : 0);  // ascending index of the e-th largest
      for (int it = 0; it < 64; ++it) {
        if (hi - lo <= 4e-7f * span) break;
        const float x = lo + (hi - lo) * (float)(s + 1) / (float)(G + 1);
        const int c = sturm_count<NN>(ta, tb2, pivmin, x);
        const unsigned below = __ballot_sync(gmask, c <= j) & gmask;  // x at or below target
        const int nb = __popc(below);  // prefix length (monotone in s)
        const float xlo = __shfl_sync(gmask, x, (lane & ~(G - 1)) + max(nb - 1, 0));
        const float xhi = __shfl_sync(gmask, x, (lane & ~(G - 1)) + min(nb, G - 1));
        if (nb > 0) lo = xlo;
        if (nb < G) hi = xhi;
      }
      if (s == 0 && e < K) lam[e] = 0.5f * (lo + hi);
    }
  }
  __syncthreads();
  // ---- 3. inverse iteration (one thread per eigenvector) -----------------
  float* Y = A;  // K x LD, reuses the reduced matrix storage
  for (int e = tid; e < K; e += EIG_THREADS) {
    const float l = lam[e];
    float ud[NN], us[NN], uf[NN], ml[NN], y[NN];
    bool pv[NN];
    // factor T - l I with partial pivoting (rows i, i+1 at step i)
    float g = ta[0] - l, h = tb[0];
    for (int i = 0; i < NN - 1; ++i) {
      const float sdn = tb[i], gn = ta[i + 1] - l, hn = (i + 1 < NN - 1) ? tb[i + 1] : 0.f;
      if (fabsf(g) >= fabsf(sdn)) {
        const float mult = (g != 0.f) ? __fdividef(sdn, g) : 0.f;
        ud[i] = g;
        us[i] = h;
        uf[i] = 0.f;
        ml[i] = mult;
        pv[i] = false;
        g = gn - mult * h;
        h = hn;
      } else {
        const float mult = __fdividef(g, sdn);
        ud[i] = sdn;
        us[i] = gn;
        uf[i] = hn;
        ml[i] = mult;
        pv[i] = true;
        g = h - mult * gn;
        h = -mult * hn;
      }
    }
    ud[NN - 1] = g;
    const float tiny = 1e-7f * misc[3];
    for (int i = 0; i < NN; ++i)
      if (fabsf(ud[i]) < tiny) ud[i] = ud[i] < 0.f ? -tiny : tiny;
    for (int i = 0; i < NN; ++i) y[i] = 0.5f + (float)((i * 2654435761u + e * 40503u) % 1024u) / 1024.f;
    for (int it = 0; it < 3; ++it) {
      for (int i = 0; i < NN - 1; ++i) {  // forward: L^-1 P
        if (pv[i]) {
          const float t = y[i];
          y[i] = y[i + 1];
          y[i + 1] = t;
        }
        y[i + 1] -= ml[i] * y[i];
      }
      y[NN - 1] = __fdividef(y[NN - 1], ud[NN - 1]);  // back: U^-1
      y[NN - 2] = __fdividef(y[NN - 2] - us[NN - 2] * y[NN - 1], ud[NN - 2]);
      for (int i = NN - 3; i >= 0; --i)
        y[i] = __fdividef(y[i] - us[i] * y[i + 1] - uf[i] * y[i + 2], ud[i]);
      float nrm = 0.f;
      for (int i = 0; i < NN; ++i) nrm += y[i] * y[i];
      const float inv = nrm > 0.f ? rsqrtf(nrm) : 0.f;
      for (int i = 0; i < NN; ++i) y[i] *= inv;
    }
    for (int i = 0; i < NN; ++i) Y[e * LD + i] = y[i];
  }
  __syncthreads();
  // Orthonormalise in descending eigenvalue order by Cholesky QR (the same
  // basis as Gram-Schmidt in that order): Gm = Y Y^T = L L^T, Y <- L^-1 Y.
  float* Gm = misc + 8;  // K x (K + 1)
  const int GL = K + 1;
  for (int e = tid; e < K * K; e += EIG_THREADS) {
    const int a = e / K, b = e % K;
    if (b <= a) {
      float s = 0.f;
      for (int i = 0; i < NN; ++i) s += Y[a * LD + i] * Y[b * LD + i];
      Gm[a * GL + b] = s;
    }
  }
  __syncthreads();
  if (warp == 0) {  // Cholesky of Gm, lanes over rows
    for (int kq = 0; kq < K; ++kq) {
      const float dkk = sqrtf(fmaxf(Gm[kq * GL + kq], 1e-30f));
      __syncwarp();
      for (int i = kq + 1 + lane; i < K; i += 32) Gm[i * GL + kq] /= dkk;
      if (lane == 0) Gm[kq * GL + kq] = dkk;
      __syncwarp();
      for (int i = kq + 1 + lane; i < K; i += 32) {
        const float lik = Gm[i * GL + kq];
        for (int j = kq + 1; j <= i; ++j) Gm[i * GL + j] -= lik * Gm[j * GL + kq];
      }
      __syncwarp();
    }
  }
  __syncthreads();
  for (int i = tid; i < NN; i += EIG_THREADS) {  // forward substitution per column of Y
    for (int a = 0; a < K; ++a) {
      float s = Y[a * LD + i];
      for (int b = 0; b < a; ++b) s -= Gm[a * GL + b] * Y[b * LD + i];
      Y[a * LD + i] = s / Gm[a * GL + a];
    }
  }
  __syncthreads();
  // ---- 4. back-transformation, one warp per vector -----------------------
  for (int kq = warp; kq < K; kq += EIG_THREADS / 32) {
    float* y = Y + kq * LD;
    for (int j = NN - 3; j >= 0; --j) {
      const float t = tau[j];
      if (t == 0.f) continue;
      const float* v = Vh + j * NN;
      float d = 0.f;
      for (int i = j + 1 + lane; i < NN; i += 32) d += v[i] * y[i];
      d = warp_sum(d) * t;
      for (int i = j + 1 + lane; i < NN; i += 32) y[i] -= d * v[i];
      __syncwarp();
    }
  }
  __syncthreads();
  for (int e = tid; e < K; e += EIG_THREADS) evals[(size_t)m * NN + e] = lam[e];
  for (int e = tid; e < NN * K; e += EIG_THREADS) {
    const int row = e / K, kq = e % K;
    evecs[(size_t)m * NN * NN + row * NN + kq] = Y[kq * LD + row];
  }
}

template <int NN>
static cudaError_t eig_n(const float* A, int count, int K, float* ev, float* evec, float* trace,
                         cudaStream_t st) {
  // A / Y, reflectors, T and scratch vectors, misc, Cholesky-QR Gram (K <= NN)
  const size_t smem = (size_t)(NN * (NN + 1) + NN * NN + 6 * NN + 8 + NN * (NN + 1)) * 4;
  cudaError_t e = cudaFuncSetAttribute(k_eig_top<NN>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  spr_launch(k_eig_top<NN>, count, EIG_THREADS, smem, st, A, K, ev, evec, trace);
  return cudaGetLastError();
}

cudaError_t launch_eig(const float* A, int count, int n, int K, float* evals, float* evecs,
                       float* trace, cudaStream_t st) {
  if (K < 1 || K > n) return cudaErrorInvalidValue;
  if (n == 64) return eig_n<64>(A, count, K, evals, evecs, trace, st);
  if (n == 128) return eig_n<128>(A, count, K, evals, evecs, trace, st);
  return cudaErrorInvalidValue;
}

}  // namespace spr
