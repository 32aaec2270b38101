// Probe-Fitted Residual Reconstruction and output restoration [paperlayer §4,
// App. A, A.3; gist-nl §2B].
//
// Per head, with X = sparse outputs of the probe rows, R = exact dense rows
// minus X and coverage weights w (sum 1):
//   Rbar = sum w R, xbar = sum w X, Rc = R - Rbar, Xc = X - xbar,
//   U_r  = leading eigenvectors of Rc^T W Rc (right singular vectors of the
//          weighted centred residual), directions with sigma <= 1e-3 sigma_max
//          dropped (the fp32 noise floor of the Gram eigenvalues),
//   B    = (Xc^T W Xc + lambda I)^-1 Xc^T W (Rc U_r)      (ridge, Cholesky),
//   O(x) = x + Rbar + (x - xbar) B U_r^T on unprobed rows; probe rows take
//          their exact dense value; rows return to the original query order.
#include <float.h>

#include "spr_internal.cuh"

namespace spr {

// Weighted means and the two d x d second-moment matrices.  Grid BH, 1024 thr.
template <int D>
__global__ void __launch_bounds__(1024) k_fit_moments(const float* osp, const float* odn,
                                                      const int32_t* ppos, const float* pw,
                                                      int N, int M, float lambda, float* gram,
                                                      float* axx, float* rxbar) {
  constexpr int TB = 16;  // probe rows staged per step
  __shared__ float Rs[TB][D], Xs[TB][D], ws[TB];
  __shared__ float rbar[D], xbar[D];
  const int bh = blockIdx.x, tid = threadIdx.x;
  if (tid < D) {
    double sr = 0.0, sx = 0.0;
    for (int t = 0; t < M; ++t) {
      const float w = pw[(size_t)bh * M + t];
      const float x = osp[((size_t)bh * N + ppos[(size_t)bh * M + t]) * D + tid];
      const float dn = odn[((size_t)bh * M + t) * D + tid];
      sr += (double)w * (double)(dn - x);
      sx += (double)w * (double)x;
    }
    rbar[tid] = (float)sr;
    xbar[tid] = (float)sx;
    rxbar[(size_t)bh * 2 * D + tid] = (float)sr;
    rxbar[(size_t)bh * 2 * D + D + tid] = (float)sx;
  }
  __syncthreads();
  constexpr int PER = D * D / 1024;  // entries per thread
  float g[PER], a[PER];
#pragma unroll
  for (int k = 0; k < PER; ++k) g[k] = a[k] = 0.f;
  for (int t0 = 0; t0 < M; t0 += TB) {
    for (int e = tid; e < TB * D; e += 1024) {
      const int tt = e / D, c = e % D, t = t0 + tt;
      float rv = 0.f, xv = 0.f;
      if (t < M) {
        const float x = osp[((size_t)bh * N + ppos[(size_t)bh * M + t]) * D + c];
        rv = odn[((size_t)bh * M + t) * D + c] - x - rbar[c];
        xv = x - xbar[c];
      }
      Rs[tt][c] = rv;
      Xs[tt][c] = xv;
    }
    for (int e = tid; e < TB; e += 1024) ws[e] = (t0 + e < M) ? pw[(size_t)bh * M + t0 + e] : 0.f;
    __syncthreads();
    for (int tt = 0; tt < TB; ++tt) {
      const float w = ws[tt];
#pragma unroll
      for (int k = 0; k < PER; ++k) {
        const int e = tid + k * 1024, i = e / D, j = e % D;
        g[k] += w * Rs[tt][i] * Rs[tt][j];
        a[k] += w * Xs[tt][i] * Xs[tt][j];
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int e = tid + k * 1024, i = e / D, j = e % D;
    gram[(size_t)bh * D * D + e] = g[k];
    axx[(size_t)bh * D * D + e] = a[k] + (i == j ? lambda : 0.f);
  }
}

// Subspace, ridge solve and the full-width map.  Grid BH, 512 threads.
// Dynamic smem: A (D x (D+1)) Cholesky factor, Bm (D x D) right-hand sides.
template <int D>
__global__ void __launch_bounds__(512) k_fit_solve(const float* osp, const float* odn,
                                                   const int32_t* ppos, const float* pw, int N,
                                                   int M, int r, const float* evals,
                                                   const float* evecs, const float* axx,
                                                   const float* rxbar, float* proj, float* fitU,
                                                   float* fitB, float* fitBv,
                                                   spr_head_stats* stats, Header* hdr) {
  extern __shared__ __align__(16) float fsm[];
  constexpr int LD = D + 1;
  float* A = fsm;             // D x LD
  float* Bm = A + D * LD;     // D x D  (rhs, then B)
  __shared__ int reff_s;
  __shared__ float rbar[D], xbar[D];
  const int bh = blockIdx.x, tid = threadIdx.x, nt = blockDim.x;
  const float* U = evecs + (size_t)bh * D * D;
  if (tid == 0) {
    const float l0 = fmaxf(evals[(size_t)bh * D], 0.f);
    int k = 0;
    if (l0 > 0.f)
      while (k < r && k < D && fmaxf(evals[(size_t)bh * D + k], 0.f) > 1e-6f * l0) ++k;
    reff_s = k;
    stats[bh].r_eff = k;
  }
  for (int c = tid; c < D; c += nt) {
    rbar[c] = rxbar[(size_t)bh * 2 * D + c];
    xbar[c] = rxbar[(size_t)bh * 2 * D + D + c];
  }
  for (int e = tid; e < D * D; e += nt) {
    A[(e / D) * LD + (e % D)] = axx[(size_t)bh * D * D + e];
    fitU[(size_t)bh * D * D + e] = U[e];
  }
  __syncthreads();
  const int re = reff_s;
  // proj[t][k] = (R_t - Rbar) . U_k
  for (int e = tid; e < M * re; e += nt) {
    const int t = e / re, k = e % re;
    const float* xr = osp + ((size_t)bh * N + ppos[(size_t)bh * M + t]) * D;
    const float* dr = odn + ((size_t)bh * M + t) * D;
    float s = 0.f;
    for (int c = 0; c < D; ++c) s += (dr[c] - xr[c] - rbar[c]) * U[c * D + k];
    proj[((size_t)bh * M + t) * D + k] = s;
  }
  __syncthreads();
  // rhs[i][k] = sum_t w_t (X_t - xbar)_i proj[t][k]
  for (int e = tid; e < D * re; e += nt) {
    const int i = e / re, k = e % re;
    float s = 0.f;
    for (int t = 0; t < M; ++t) {
      const float x = osp[((size_t)bh * N + ppos[(size_t)bh * M + t]) * D + i] - xbar[i];
      s += pw[(size_t)bh * M + t] * x * proj[((size_t)bh * M + t) * D + k];
    }
    Bm[i * D + k] = s;
  }
  __syncthreads();
  // Cholesky A = L L^T (lower triangle in place), right-looking.
  for (int k = 0; k < D; ++k) {
    if (tid == 0) {
      float v = A[k * LD + k];
      if (!(v > 0.f)) {
        if (!isfinite(v)) set_error(hdr, ERR_NUMERIC, 10, bh, k);
        v = FLT_MIN * 1e10f;
      }
      A[k * LD + k] = sqrtf(v);
    }
    __syncthreads();
    const float dkk = A[k * LD + k];
    for (int i = k + 1 + tid; i < D; i += nt) A[i * LD + k] /= dkk;
    __syncthreads();
    const int m = D - k - 1;
    for (int e = tid; e < m * m; e += nt) {
      const int i = k + 1 + e / m, j = k + 1 + e % m;
      if (j <= i) A[i * LD + j] -= A[i * LD + k] * A[j * LD + k];
    }
    __syncthreads();
  }
  // Solve L L^T B = rhs, one column per thread.
  for (int k = tid; k < re; k += nt) {
    for (int i = 0; i < D; ++i) {
      float s = Bm[i * D + k];
      for (int j = 0; j < i; ++j) s -= A[i * LD + j] * Bm[j * D + k];
      Bm[i * D + k] = s / A[i * LD + i];
    }
    for (int i = D - 1; i >= 0; --i) {
      float s = Bm[i * D + k];
      for (int j = i + 1; j < D; ++j) s -= A[j * LD + i] * Bm[j * D + k];
      Bm[i * D + k] = s / A[i * LD + i];
    }
  }
  __syncthreads();
  // Full map F = B U_r^T (d x d) and intercept b = Rbar - xbar F.
  for (int e = tid; e < D * D; e += nt) {
    const int i = e / D, j = e % D;
    float s = 0.f;
    for (int k = 0; k < re; ++k) s += Bm[i * D + k] * U[j * D + k];
    fitB[(size_t)bh * D * D + e] = s;
  }
  __syncthreads();
  for (int j = tid; j < D; j += nt) {
    float s = 0.f;
    for (int i = 0; i < D; ++i) s += xbar[i] * fitB[(size_t)bh * D * D + i * D + j];
    fitBv[(size_t)bh * D + j] = rbar[j] - s;
  }
}

__global__ void k_fit_zero(float* fitB, float* fitBv, int D, int BH) {
  const size_t n = (size_t)BH * D * D;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (size_t)gridDim.x * blockDim.x) {
    fitB[e] = 0.f;
    if (e < (size_t)BH * D) fitBv[e] = 0.f;
  }
}

// O[orig row] = x + b + x F (unprobed) or the dense probe row; bf16 output in
// the original query order.  Grid (blocks per head, BH), 256 threads, one warp
// per permuted row.  Dynamic smem: F (D x D fp32).
template <int D>
__global__ void __launch_bounds__(256) k_apply(const float* osp, const float* odn,
                                               const int32_t* ppos, const int32_t* permq,
                                               const float* fitB, const float* fitBv, int N, int M,
                                               int B_, int H, int64_t sb, int64_t sh, int64_t sn,
                                               bf16* O, int do_fit, Header* hdr) {
  extern __shared__ __align__(16) float Fs[];
  __shared__ float bv[D];
  constexpr int V = D / 32;  // values per lane
  const int bh = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (do_fit) {
    for (int e = tid; e < D * D; e += 256) Fs[e] = fitB[(size_t)bh * D * D + e];
    for (int e = tid; e < D; e += 256) bv[e] = fitBv[(size_t)bh * D + e];
  }
  __syncthreads();
  const int b = bh / H, h = bh - b * H;
  bf16* ob = O + b * sb + h * sh;
  const int32_t* pp = ppos + (size_t)bh * M;
  for (int pos = blockIdx.x * 8 + warp; pos < N; pos += gridDim.x * 8) {
    const float* xr = osp + ((size_t)bh * N + pos) * D;
    float x[V];
    if (V == 4) {
      const float4 v = reinterpret_cast<const float4*>(xr)[lane];
      x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3 % V] = v.w;
    } else {
      const float2 v = reinterpret_cast<const float2*>(xr)[lane];
      x[0] = v.x; x[1 % V] = v.y;
    }
    // probe slot lookup (ppos ascending)
    int slot = -1;
    if (M > 0) {
      int lo = 0, hi = M - 1;
      while (lo <= hi) {
        const int mid = (lo + hi) >> 1, v = pp[mid];
        if (v == pos) { slot = mid; break; }
        if (v < pos) lo = mid + 1; else hi = mid - 1;
      }
    }
    float y[V];
    if (slot >= 0) {
      const float* dr = odn + ((size_t)bh * M + slot) * D;
#pragma unroll
      for (int k = 0; k < V; ++k) y[k] = dr[lane * V + k];
    } else if (do_fit) {
#pragma unroll
      for (int k = 0; k < V; ++k) y[k] = x[k] + bv[lane * V + k];
      for (int i = 0; i < D; ++i) {
        const float xi = __shfl_sync(0xffffffffu, x[i % V], i / V);
        const float* fr = Fs + i * D + lane * V;
#pragma unroll
        for (int k = 0; k < V; ++k) y[k] += xi * fr[k];
      }
    } else {
#pragma unroll
      for (int k = 0; k < V; ++k) y[k] = x[k];
    }
    const int orig = permq[(size_t)bh * N + pos];
    if (orig < 0 || orig >= N) {
      set_error(hdr, ERR_INDEX, 20, bh, orig);
      continue;
    }
    bf16* dst = ob + (int64_t)orig * sn + lane * V;
    if (V == 4) {
      uint2 u;
      u.x = pack_bf16(y[0], y[1 % V]);
      u.y = pack_bf16(y[2 % V], y[3 % V]);
      *reinterpret_cast<uint2*>(dst) = u;
    } else {
      *reinterpret_cast<uint32_t*>(dst) = pack_bf16(y[0], y[1 % V]);
    }
  }
  (void)B_;
}

// Per-head accounting: probe pairs, rho_exec, k-means objectives.
__global__ void k_stats(spr_head_stats* stats, const double* part, const double* qterm,
                        int nchunk, int Gq, int N, int M, int BH) {
  const int bh = blockIdx.x * blockDim.x + threadIdx.x;
  if (bh >= BH) return;
  double ok = 0.0, un = 0.0, qt = 0.0;
  for (int c = 0; c < nchunk; ++c) {
    ok += part[((size_t)bh * 2 + 0) * (nchunk + 1) + c];
    un += part[((size_t)bh * 2 + 1) * (nchunk + 1) + c];
  }
  for (int g = 0; g < Gq; ++g) qt += qterm[(size_t)bh * Gq + g];
  spr_head_stats& s = stats[bh];
  s.probe_pairs = (int64_t)M * N;
  s.rho_exec = (double)(s.routed_pairs + s.probe_pairs) / ((double)N * (double)N);
  s.obj_k = ok;
  s.obj_q = un - qt;
}

template <int D>
static cudaError_t reconstruct_d(const spr_params& p, const Layout& L, const Ptrs& P, bf16* O,
                                 cudaStream_t st) {
  const int BH = L.BH, N = p.N, M = p.M;
  if (M > 0) {
    spr_launch(k_fit_moments<D>, BH, 1024, 0, st, P.osp, P.odn, P.ppos, P.pw, N, M, (float)p.lambda,
                                          P.gram, P.axx, P.rxbar);
    cudaError_t e = launch_eig(P.gram, BH, D, P.eval, P.evec, st);
    if (e != cudaSuccess) return e;
    const size_t sm = (size_t)(D * (D + 1) + D * D) * 4;
    cudaFuncSetAttribute(k_fit_solve<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    spr_launch(k_fit_solve<D>, BH, 512, sm, st, P.osp, P.odn, P.ppos, P.pw, N, M, p.r, P.eval, P.evec,
                                        P.axx, P.rxbar, P.proj, P.fitU, P.fitB, P.fitBv, P.stats,
                                        P.hdr);
  } else {
    spr_launch(k_fit_zero, num_sms(), 256, 0, st, P.fitB, P.fitBv, D, BH);
  }
  const size_t sm = (size_t)D * D * 4;
  cudaFuncSetAttribute(k_apply<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  const int bph = max(1, min((N + 7) / 8, (num_sms() * 4 + BH - 1) / BH));
  spr_launch(k_apply<D>, dim3(bph, BH), 256, sm, st, P.osp, P.odn, P.ppos, P.permq, P.fitB, P.fitBv, N,
                                             M, p.B, p.H, p.o_strides[0], p.o_strides[1],
                                             p.o_strides[2], O, M > 0, P.hdr);
  spr_launch(k_stats, (BH + 127) / 128, 128, 0, st, P.stats, P.part, P.part + (size_t)BH * 2 * (L.nchunk + 1),
                                            L.nchunk, p.Gq, N, M, BH);
  return cudaGetLastError();
}

cudaError_t launch_reconstruct(const spr_params& p, const Layout& L, const Ptrs& P, bf16* O,
                               cudaStream_t st) {
  if (p.d == 64) return reconstruct_d<64>(p, L, P, O, st);
  return reconstruct_d<128>(p, L, P, O, st);
}

}  // namespace spr
