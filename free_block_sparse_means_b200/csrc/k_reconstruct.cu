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

// Residual directions kept by the fit: the leading r eigenvalues of the Gram
// above 1e-6 of the largest (sigma above 1e-3 sigma_max, the fp32 noise floor).
__device__ __forceinline__ int fit_rank(const float* ev, int D, int r) {
  const float l0 = fmaxf(ev[0], 0.f);
  int k = 0;
  if (l0 > 0.f)
    while (k < r && k < D && fmaxf(ev[k], 0.f) > 1e-6f * l0) ++k;
  return k;
}

constexpr int FIT_TM = 64;  // probes per right-hand-side block

// Partial right-hand sides of the ridge system for one block of FIT_TM probes:
// part[i][k] = sum_t w_t (x_t - xbar)_i ((r_t - Rbar) . u_k), k < r_eff, stride R.
// Grid (BH, ceil(M / FIT_TM)), 256 threads.  Dynamic smem: Rs, Xs (TM x D),
// Us (D x R), Ps (TM x R).
template <int D>
__global__ void __launch_bounds__(256) k_fit_rhs(const float* osp, const float* odn,
                                                 const int32_t* ppos, const float* pw, int N,
                                                 int M, int r, int R, const float* evals,
                                                 const float* evecs, const float* rxbar,
                                                 float* part) {
  extern __shared__ __align__(16) float rsm[];
  float* Rs = rsm;
  float* Xs = Rs + FIT_TM * D;
  float* Us = Xs + FIT_TM * D;
  float* Ps = Us + D * R;
  __shared__ float ws[FIT_TM];
  const int bh = blockIdx.x, c = blockIdx.y, tid = threadIdx.x, t0 = c * FIT_TM;
  const int re = fit_rank(evals + (size_t)bh * D, D, r);
  const float* rbar = rxbar + (size_t)bh * 2 * D;
  const float* xbar = rbar + D;
  for (int e = tid; e < FIT_TM * D; e += 256) {
    const int tt = e / D, col = e % D, t = t0 + tt;
    float rv = 0.f, xv = 0.f;
    if (t < M) {
      const float x = osp[((size_t)bh * N + ppos[(size_t)bh * M + t]) * D + col];
      rv = odn[((size_t)bh * M + t) * D + col] - x - rbar[col];
      xv = x - xbar[col];
    }
    Rs[e] = rv;
    Xs[e] = xv;
  }
  for (int e = tid; e < D * R; e += 256) {
    const int i = e / R, k = e % R;
    Us[e] = k < re ? evecs[((size_t)bh * D + i) * D + k] : 0.f;
  }
  for (int e = tid; e < FIT_TM; e += 256) ws[e] = (t0 + e < M) ? pw[(size_t)bh * M + t0 + e] : 0.f;
  __syncthreads();
  for (int e = tid; e < FIT_TM * R; e += 256) {
    const int tt = e / R, k = e % R;
    float s = 0.f;
    if (k < re)
      for (int col = 0; col < D; ++col) s += Rs[tt * D + col] * Us[col * R + k];
    Ps[e] = ws[tt] * s;
  }
  __syncthreads();
  float* out = part + ((size_t)bh * gridDim.y + c) * D * R;
  for (int e = tid; e < D * R; e += 256) {
    const int i = e / R, k = e % R;
    float s = 0.f;
    if (k < re)
      for (int tt = 0; tt < FIT_TM; ++tt) s += Xs[tt * D + i] * Ps[tt * R + k];
    out[e] = s;
  }
}

// Subspace, ridge solve and the intercept.  Grid BH, 512 threads.
// Dynamic smem: A (D x (D+1)) Cholesky factor, Bm (D x D) right-hand sides.
template <int D>
__global__ void __launch_bounds__(512) k_fit_solve(int r, int R, int nchunk, const float* evals,
                                                   const float* evecs, const float* axx,
                                                   const float* rxbar, const float* part,
                                                   float* fitU, float* fitB, float* fitBv,
                                                   spr_head_stats* stats, Header* hdr) {
  extern __shared__ __align__(16) float fsm[];
  constexpr int LD = D + 1;
  float* A = fsm;             // D x LD
  float* Bm = A + D * LD;     // D x D  (rhs, then B)
  __shared__ float rbar[D], xbar[D];
  const int bh = blockIdx.x, tid = threadIdx.x, nt = blockDim.x;
  const float* U = evecs + (size_t)bh * D * D;
  const int re = fit_rank(evals + (size_t)bh * D, D, r);
  if (tid == 0) stats[bh].r_eff = re;
  for (int c = tid; c < D; c += nt) {
    rbar[c] = rxbar[(size_t)bh * 2 * D + c];
    xbar[c] = rxbar[(size_t)bh * 2 * D + D + c];
  }
  for (int e = tid; e < D * D; e += nt) {
    A[(e / D) * LD + (e % D)] = axx[(size_t)bh * D * D + e];
    fitU[(size_t)bh * D * D + e] = U[e];
  }
  for (int e = tid; e < D * re; e += nt) {  // sum the probe blocks in a fixed order
    const int i = e / re, k = e % re;
    float s = 0.f;
    for (int c = 0; c < nchunk; ++c) s += part[(((size_t)bh * nchunk + c) * D + i) * R + k];
    Bm[i * D + k] = s;
  }
  __syncthreads();
  // Cholesky A = L L^T, right-looking, one barrier per column: step k updates
  // the trailing block from the unscaled column k and scales column k - 1.
  const int warp = tid >> 5, lane = tid & 31, nw = nt >> 5;
  for (int k = 0; k < D; ++k) {
    float akk = A[k * LD + k];
    if (!(akk > 0.f)) {
      if (tid == 0 && !isfinite(akk)) set_error(hdr, ERR_NUMERIC, 10, bh, k);
      akk = FLT_MIN * 1e10f;
    }
    const float inv = 1.f / akk;
    for (int i = k + 1 + warp; i < D; i += nw) {
      const float aik = A[i * LD + k] * inv;
      for (int j = k + 1 + lane; j <= i; j += 32) A[i * LD + j] -= aik * A[j * LD + k];
    }
    if (k > 0) {
      float ap = A[(k - 1) * LD + k - 1];
      if (!(ap > 0.f)) ap = FLT_MIN * 1e10f;
      const float dp = sqrtf(ap);
      for (int i = k + tid; i < D; i += nt) A[i * LD + k - 1] /= dp;
    }
    __syncthreads();
    if (k > 0 && tid == 0) {
      float ap = A[(k - 1) * LD + k - 1];
      A[(k - 1) * LD + k - 1] = sqrtf(ap > 0.f ? ap : FLT_MIN * 1e10f);
    }
  }
  __syncthreads();
  {
    float ap = A[(D - 1) * LD + D - 1];
    if (tid == 0) A[(D - 1) * LD + D - 1] = sqrtf(ap > 0.f ? ap : FLT_MIN * 1e10f);
  }
  __syncthreads();
  // Solve L L^T B = rhs: one warp per column, lanes split each inner product.
  {
    const int warp = tid >> 5, lane = tid & 31;
    for (int k = warp; k < re; k += nt / 32) {
      for (int i = 0; i < D; ++i) {
        float s = 0.f;
        for (int j = lane; j < i; j += 32) s += A[i * LD + j] * Bm[j * D + k];
        s = warp_sum(s);
        if (lane == 0) Bm[i * D + k] = (Bm[i * D + k] - s) / A[i * LD + i];
        __syncwarp();
      }
      for (int i = D - 1; i >= 0; --i) {
        float s = 0.f;
        for (int j = i + 1 + lane; j < D; j += 32) s += A[j * LD + i] * Bm[j * D + k];
        s = warp_sum(s);
        if (lane == 0) Bm[i * D + k] = (Bm[i * D + k] - s) / A[i * LD + i];
        __syncwarp();
      }
    }
  }
  __syncthreads();
  // B (d x r_eff, stride d) and the full-width intercept b = Rbar - (xbar B) U_r^T.
  __shared__ float xb[D];
  for (int e = tid; e < D * D; e += nt) {
    const int i = e / D, k = e % D;
    fitB[(size_t)bh * D * D + e] = k < re ? Bm[i * D + k] : 0.f;
  }
  for (int k = tid; k < D; k += nt) {
    float s = 0.f;
    if (k < re)
      for (int i = 0; i < D; ++i) s += xbar[i] * Bm[i * D + k];
    xb[k] = s;
  }
  __syncthreads();
  for (int j = tid; j < D; j += nt) {
    float s = 0.f;
    for (int k = 0; k < re; ++k) s += xb[k] * U[j * D + k];
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

// O[orig row] = x + b + (x B) U_r^T (unprobed) or the dense probe row; bf16
// output in the original query order.  Grid (blocks per head, BH), 256
// threads; each block takes tiles of APPLY_TR consecutive permuted rows:
// T = X B (tile x r) and Y = X + b + T U_r^T from shared memory.
// Dynamic smem: B as [D][R], U_r as [R][D], the X tile and T.
constexpr int APPLY_TR = 32;

template <int D>
__global__ void __launch_bounds__(256) k_apply(const float* osp, const float* odn,
                                               const int32_t* pslot, const int32_t* permq,
                                               const float* fitB, const float* fitU,
                                               const float* fitBv, const spr_head_stats* stats,
                                               int R, int N, int M, int H, int64_t sb, int64_t sh,
                                               int64_t sn, bf16* O, int do_fit, Header* hdr) {
  extern __shared__ __align__(16) float fsh[];
  constexpr int XL = D + 4;  // padded row of the X tile
  float* Bs = fsh;                    // [D][R]
  float* Us = Bs + D * R;             // [R][D]
  float* Xs = Us + R * D;             // [APPLY_TR][XL]
  float* Ts = Xs + APPLY_TR * XL;     // [APPLY_TR][R]
  __shared__ float bv[D];
  __shared__ int slot_s[APPLY_TR], orig_s[APPLY_TR];
  const int bh = blockIdx.y, tid = threadIdx.x;
  const int re = do_fit ? min(stats[bh].r_eff, R) : 0;
  for (int e = tid; e < D * R; e += 256) {
    const int i = e / R, k = e % R;
    Bs[e] = k < re ? fitB[((size_t)bh * D + i) * D + k] : 0.f;
    Us[k * D + i] = k < re ? fitU[((size_t)bh * D + i) * D + k] : 0.f;
  }
  for (int e = tid; e < D; e += 256) bv[e] = do_fit ? fitBv[(size_t)bh * D + e] : 0.f;
  const int b = bh / H, h = bh - b * H;
  bf16* ob = O + b * sb + h * sh;
  const int ntile = (N + APPLY_TR - 1) / APPLY_TR;
  for (int tile = blockIdx.x; tile < ntile; tile += gridDim.x) {
    const int pos0 = tile * APPLY_TR;
    __syncthreads();  // previous tile fully consumed
    for (int e = tid; e < APPLY_TR * (D / 4); e += 256) {
      const int r = e / (D / 4), c4 = e % (D / 4), pos = pos0 + r;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (pos < N) v = reinterpret_cast<const float4*>(osp + ((size_t)bh * N + pos) * D)[c4];
      *reinterpret_cast<float4*>(Xs + r * XL + c4 * 4) = v;
    }
    if (tid < APPLY_TR) {
      const int pos = pos0 + tid;
      int slot = -1, orig = -1;
      if (pos < N) {
        slot = M > 0 ? pslot[(size_t)bh * N + pos] : -1;
        orig = permq[(size_t)bh * N + pos];
        if (slot >= M || orig < 0 || orig >= N) {
          set_error(hdr, ERR_INDEX, 20, bh, pos);
          orig = -1;
        }
      }
      slot_s[tid] = slot;
      orig_s[tid] = orig;
    }
    __syncthreads();
    if (re > 0) {
      for (int e = tid; e < APPLY_TR * re; e += 256) {
        const int r = e / re, k = e % re;
        float s = 0.f;
#pragma unroll 8
        for (int i = 0; i < D; ++i) s += Xs[r * XL + i] * Bs[i * R + k];
        Ts[r * R + k] = s;
      }
      __syncthreads();
    }
    for (int e = tid; e < APPLY_TR * (D / 2); e += 256) {
      const int r = e / (D / 2), j = 2 * (e % (D / 2));
      const int orig = orig_s[r];
      if (orig < 0) continue;
      float y0, y1;
      if (slot_s[r] >= 0) {
        const float* dr = odn + ((size_t)bh * M + slot_s[r]) * D + j;
        y0 = dr[0];
        y1 = dr[1];
      } else {
        y0 = Xs[r * XL + j] + bv[j];
        y1 = Xs[r * XL + j + 1] + bv[j + 1];
        for (int k = 0; k < re; ++k) {
          const float tk = Ts[r * R + k];
          y0 += tk * Us[k * D + j];
          y1 += tk * Us[k * D + j + 1];
        }
      }
      *reinterpret_cast<uint32_t*>(ob + (int64_t)orig * sn + j) = pack_bf16(y0, y1);
    }
  }
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
    cudaError_t e = launch_eig(P.gram, BH, D, p.r > 0 ? p.r : 1, P.eval, P.evec, nullptr, st);
    if (e != cudaSuccess) return e;
    const int R = p.r > 0 ? p.r : 1, nchunk = (M + FIT_TM - 1) / FIT_TM;
    const size_t smr = (size_t)(2 * FIT_TM * D + D * R + FIT_TM * R) * 4;
    cudaFuncSetAttribute(k_fit_rhs<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smr);
    spr_launch(k_fit_rhs<D>, dim3(BH, nchunk), 256, smr, st, P.osp, P.odn, P.ppos, P.pw, N, M,
               p.r, R, P.eval, P.evec, P.rxbar, P.proj);
    const size_t sm = (size_t)(D * (D + 1) + D * D) * 4;
    cudaFuncSetAttribute(k_fit_solve<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    spr_launch(k_fit_solve<D>, BH, 512, sm, st, p.r, R, nchunk, P.eval, P.evec, P.axx, P.rxbar,
               P.proj, P.fitU, P.fitB, P.fitBv, P.stats, P.hdr);
  } else {
    spr_launch(k_fit_zero, num_sms(), 256, 0, st, P.fitB, P.fitBv, D, BH);
  }
  const int R = p.r > 0 ? p.r : 1;
  const size_t sm = (size_t)(2 * D * R + APPLY_TR * (D + 4) + APPLY_TR * R) * 4;
  cudaFuncSetAttribute(k_apply<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  const int bph = max(1, min((N + APPLY_TR - 1) / APPLY_TR, (num_sms() * 4 + BH - 1) / BH));
  spr_launch(k_apply<D>, dim3(bph, BH), 256, sm, st, P.osp, P.odn, P.pslot, P.permq, P.fitB,
             P.fitU, P.fitBv, P.stats, R, N, M, p.H, p.o_strides[0], p.o_strides[1],
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
