// Symmetric eigensolver for the small d x d matrices of the call: the
// sampled-query response metric M_K [paperlayer App. B.1] and the weighted
// probe-residual Gram matrix [paperlayer App. A.3].
//
// Cyclic two-sided Jacobi (Golub & Van Loan, "Matrix Computations", the
// symmetric Schur decomposition) with the parallel round-robin ordering: each
// round rotates NN/2 disjoint (p, q) index pairs at once, A' = J^T A J.  Every
// thread owns a set of 2 x 2 blocks (rows {p_k, q_k} x columns {p_l, q_l}) and
// applies both the row and the column rotation to them, reading the old matrix
// and writing a second buffer, so one barrier per round suffices; the rotation
// angles are recomputed by each thread from the old matrix.  Sweeps stop when
// the off-diagonal Frobenius norm falls below 1e-6 of the total (the fp32
// floor) or after 16 sweeps.  One block per matrix, all in shared memory.
#include "spr_internal.cuh"

namespace spr {

__device__ __forceinline__ int rr_p(int round, int k, int n) {
  return k == 0 ? n - 1 : (round + k) % (n - 1);
}
__device__ __forceinline__ int rr_q(int round, int k, int n) {
  return k == 0 ? round : (round - k + (n - 1)) % (n - 1);
}

// Rotation (c, s) that zeroes the (p, q) entry of J^T A J.
__device__ __forceinline__ void jacobi_cs(float app, float aqq, float apq, float& c, float& s) {
  c = 1.f;
  s = 0.f;
  if (fabsf(apq) > 1e-30f) {
    const float theta = (aqq - app) / (2.f * apq);
    float t;
    if (fabsf(theta) > 1e15f)
      t = 0.5f / theta;
    else
      t = (theta >= 0.f ? 1.f : -1.f) / (fabsf(theta) + sqrtf(theta * theta + 1.f));
    c = 1.f / sqrtf(t * t + 1.f);
    s = t * c;
  }
}

template <int NN>
__global__ void __launch_bounds__(512) k_eig(const float* Ain, float* evals, float* evecs) {
  constexpr int LD = NN + 1, NP = NN / 2, NT = 512, TPR = NT / NP;  // threads per pair-row
  extern __shared__ __align__(16) float esm[];
  float* Abuf0 = esm;
  float* Abuf1 = Abuf0 + NN * LD;
  float* V = Abuf1 + NN * LD;
  float* red = V + NN * LD;                    // [64]
  int* rank = reinterpret_cast<int*>(red + 64);  // [NN]
  const int m = blockIdx.x, tid = threadIdx.x;
  const float* src = Ain + (size_t)m * NN * NN;
  for (int e = tid; e < NN * NN; e += NT) {
    const int i = e / NN, j = e % NN;
    Abuf0[i * LD + j] = 0.5f * (src[i * NN + j] + src[j * NN + i]);
    V[i * LD + j] = (i == j) ? 1.f : 0.f;
  }
  __syncthreads();
  float* A = Abuf0;
  float* An = Abuf1;
  const int k = tid / TPR, sub = tid % TPR;
  for (int sweep = 0; sweep < 16; ++sweep) {
    float off = 0.f, tot = 0.f;
    for (int e = tid; e < NN * NN; e += NT) {
      const int i = e / NN, j = e % NN;
      const float a = A[i * LD + j];
      tot += a * a;
      if (i != j) off += a * a;
    }
    off = warp_sum(off);
    tot = warp_sum(tot);
    if ((tid & 31) == 0) {
      red[tid >> 5] = off;
      red[32 + (tid >> 5)] = tot;
    }
    __syncthreads();
    float offn = 0.f, totn = 0.f;
    for (int w = 0; w < NT / 32; ++w) {
      offn += red[w];
      totn += red[32 + w];
    }
    __syncthreads();
    if (!(offn > 1e-12f * totn) || !(totn > 0.f)) break;
    for (int round = 0; round < NN - 1; ++round) {
      const int pk = rr_p(round, k, NN), qk = rr_q(round, k, NN);
      float ck, sk;
      jacobi_cs(A[pk * LD + pk], A[qk * LD + qk], A[pk * LD + qk], ck, sk);
      for (int l = sub; l < NP; l += TPR) {
        const int pl = rr_p(round, l, NN), ql = rr_q(round, l, NN);
        float cl, sl;
        jacobi_cs(A[pl * LD + pl], A[ql * LD + ql], A[pl * LD + ql], cl, sl);
        const float app = A[pk * LD + pl], apq = A[pk * LD + ql];
        const float aqp = A[qk * LD + pl], aqq = A[qk * LD + ql];
        // rows: J_k^T
        const float rpp = ck * app - sk * aqp, rpq = ck * apq - sk * aqq;
        const float rqp = sk * app + ck * aqp, rqq = sk * apq + ck * aqq;
        // columns: J_l
        An[pk * LD + pl] = cl * rpp - sl * rpq;
        An[pk * LD + ql] = sl * rpp + cl * rpq;
        An[qk * LD + pl] = cl * rqp - sl * rqq;
        An[qk * LD + ql] = sl * rqp + cl * rqq;
        // eigenvectors: V J_l on the two rows this thread owns
        float vp = V[pk * LD + pl], vq = V[pk * LD + ql];
        V[pk * LD + pl] = cl * vp - sl * vq;
        V[pk * LD + ql] = sl * vp + cl * vq;
        vp = V[qk * LD + pl];
        vq = V[qk * LD + ql];
        V[qk * LD + pl] = cl * vp - sl * vq;
        V[qk * LD + ql] = sl * vp + cl * vq;
      }
      __syncthreads();
      float* t = A;
      A = An;
      An = t;
    }
  }
  for (int i = tid; i < NN; i += NT) {
    const float li = A[i * LD + i];
    int r = 0;
    for (int j = 0; j < NN; ++j) {
      const float lj = A[j * LD + j];
      r += (lj > li) || (lj == li && j < i);
    }
    rank[i] = r;
    evals[(size_t)m * NN + r] = li;
  }
  __syncthreads();
  for (int e = tid; e < NN * NN; e += NT) {
    const int row = e / NN, i = e % NN;
    evecs[(size_t)m * NN * NN + row * NN + rank[i]] = V[row * LD + i];
  }
}

template <int NN>
static cudaError_t eig_n(const float* A, int count, float* ev, float* evec, cudaStream_t st) {
  const size_t smem = (size_t)(3 * NN * (NN + 1) + 64 + NN) * 4;
  cudaError_t e = cudaFuncSetAttribute(k_eig<NN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  spr_launch(k_eig<NN>, count, 512, smem, st, A, ev, evec);
  return cudaGetLastError();
}

cudaError_t launch_eig(const float* A, int count, int n, float* evals, float* evecs,
                       cudaStream_t st) {
  if (n == 64) return eig_n<64>(A, count, evals, evecs, st);
  if (n == 128) return eig_n<128>(A, count, evals, evecs, st);
  return cudaErrorInvalidValue;
}

}  // namespace spr
