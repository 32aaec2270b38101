// Probe-Fitted Residual Reconstruction and output restoration [paperlayer §4,
// App. A, A.3; gist-nl §2B].
//
// Per head, with X = sparse outputs of the probe rows, R = exact dense rows
// minus X and coverage weights w (sum 1):
//   Rbar = sum w R, xbar = sum w X, Rc = R - Rbar, Xc = X - xbar,
//   U_r  = leading eigenvectors of Rc^T W Rc (right singular vectors of the
//          weighted centred residual), directions with sigma <= 1e-3 sigma_max
//          dropped (the fp32 noise floor of the Gram eigenvalues),
//   B    = (Xc^T W Xc + lambda I)^-1 Xc^T W (Rc U_r)      (ridge, LDL^T),
//   O(x) = x + Rbar + (x - xbar) B U_r^T on unprobed rows; probe rows take
//          their exact dense value; rows return to the original query order.
#include <float.h>

#include "spr_internal.cuh"

namespace spr {

constexpr int FIT_GB = 32;  // probe rows per gather block

// Probe rows into compact buffers: X_t = O_sp[slot t], R_t = O_dense,t - X_t,
// and the block's weighted sums sum w R, sum w X over its FIT_GB rows (warp
// partials added in warp order).  Grid (ceil(M / FIT_GB), BH), 256 threads.
template <int D>
__global__ void __launch_bounds__(256) k_fit_gather(const float* osp, const float* odn,
                                                    const int32_t* ppos, const float* pw, int N,
                                                    int M, float* Xp, float* Rp, float* pmean) {
  constexpr int C4 = D / 4;  // float4 columns per row
  __shared__ float ws[FIT_GB];
  __shared__ int ps[FIT_GB];
  __shared__ float4 sr[8][C4], sx[8][C4];
  const int bh = blockIdx.y, blk = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t0 = blk * FIT_GB;
  if (tid < FIT_GB) {
    const int t = t0 + tid;
    ps[tid] = t < M ? ppos[(size_t)bh * M + t] : -1;
    ws[tid] = t < M ? pw[(size_t)bh * M + t] : 0.f;
  }
  __syncthreads();
  float4 ar = make_float4(0.f, 0.f, 0.f, 0.f), ax = ar;
  if (lane < C4) {
#pragma unroll
    for (int u = 0; u < FIT_GB / 8; ++u) {
      const int tt = warp + 8 * u, pos = ps[tt];
      if (pos < 0) continue;
      const size_t t = (size_t)bh * M + t0 + tt;
      const float4 x = reinterpret_cast<const float4*>(osp + ((size_t)bh * N + pos) * D)[lane];
      const float4 dn = reinterpret_cast<const float4*>(odn + t * D)[lane];
      const float4 r = make_float4(dn.x - x.x, dn.y - x.y, dn.z - x.z, dn.w - x.w);
      reinterpret_cast<float4*>(Xp + t * D)[lane] = x;
      reinterpret_cast<float4*>(Rp + t * D)[lane] = r;
      const float w = ws[tt];
      ar = make_float4(fmaf(w, r.x, ar.x), fmaf(w, r.y, ar.y), fmaf(w, r.z, ar.z), fmaf(w, r.w, ar.w));
      ax = make_float4(fmaf(w, x.x, ax.x), fmaf(w, x.y, ax.y), fmaf(w, x.z, ax.z), fmaf(w, x.w, ax.w));
    }
    sr[warp][lane] = ar;
    sx[warp][lane] = ax;
  }
  __syncthreads();
  if (tid < 2 * D) {
    const int which = tid / D, c = tid % D;
    const float* src = reinterpret_cast<const float*>(which ? &sx[0][0] : &sr[0][0]);
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += src[w * D + c];
    pmean[(((size_t)bh * gridDim.x + blk) * 2 + which) * D + c] = s;
  }
}

// Weighted means (block sums added in block order, fp64) and the slab of
// columns [32 s, 32 s + 32) of the two d x d second moments
//   gram = Rc^T W Rc,   axx = Xc^T W Xc + lambda I.
// Grid (D / 32, BH), 256 threads, each a 4 x 4 block of both matrices.
template <int D>
__global__ void __launch_bounds__(256) k_fit_moments(const float* Xp, const float* Rp,
                                                     const float* pw, const float* pmean,
                                                     int M, int nblk, float lambda, float* gram,
                                                     float* axx, float* rxbar) {
  constexpr int TT = 32;     // probes per staged tile
  constexpr int XL = D + 4;  // padded row
  __shared__ __align__(16) float Rw[TT][XL], Xw[TT][XL];  // weighted, centred
  __shared__ __align__(16) float Rc[TT][36], Xc[TT][36];  // centred, this slab's columns
  __shared__ float rbar[D], xbar[D], ws[TT];
  const int bh = blockIdx.y, slab = blockIdx.x, tid = threadIdx.x;
  const int j0 = slab * 32;
  if (tid < 2 * D) {
    const int which = tid / D, c = tid % D;
    double s = 0.0;
    for (int b = 0; b < nblk; ++b) s += (double)pmean[(((size_t)bh * nblk + b) * 2 + which) * D + c];
    (which ? xbar : rbar)[c] = (float)s;
    if (slab == 0) rxbar[(size_t)bh * 2 * D + which * D + c] = (float)s;
  }
  const int ib = tid >> 3, jb = tid & 7;  // rows 4 ib .., columns j0 + 4 jb ..
  float g[4][4], a[4][4];
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) g[u][v] = a[u][v] = 0.f;
  for (int t0 = 0; t0 < M; t0 += TT) {
    __syncthreads();  // means ready / previous tile consumed
    if (tid < TT) ws[tid] = t0 + tid < M ? pw[(size_t)bh * M + t0 + tid] : 0.f;
    __syncthreads();
    for (int e = tid; e < TT * (D / 4); e += 256) {
      const int tt = e / (D / 4), c = 4 * (e % (D / 4)), t = t0 + tt;
      float4 r = make_float4(0.f, 0.f, 0.f, 0.f), x = r;
      if (t < M) {
        r = reinterpret_cast<const float4*>(Rp + ((size_t)bh * M + t) * D)[c / 4];
        x = reinterpret_cast<const float4*>(Xp + ((size_t)bh * M + t) * D)[c / 4];
        r = make_float4(r.x - rbar[c], r.y - rbar[c + 1], r.z - rbar[c + 2], r.w - rbar[c + 3]);
        x = make_float4(x.x - xbar[c], x.y - xbar[c + 1], x.z - xbar[c + 2], x.w - xbar[c + 3]);
      }
      const float w = ws[tt];
      *reinterpret_cast<float4*>(&Rw[tt][c]) = make_float4(w * r.x, w * r.y, w * r.z, w * r.w);
      *reinterpret_cast<float4*>(&Xw[tt][c]) = make_float4(w * x.x, w * x.y, w * x.z, w * x.w);
      if (c >= j0 && c < j0 + 32) {
        *reinterpret_cast<float4*>(&Rc[tt][c - j0]) = r;
        *reinterpret_cast<float4*>(&Xc[tt][c - j0]) = x;
      }
    }
    __syncthreads();
    if (4 * ib >= D) continue;  // (d = 64: half the threads hold no block)
#pragma unroll 4
    for (int tt = 0; tt < TT; ++tt) {
      const float4 ri = *reinterpret_cast<const float4*>(&Rw[tt][4 * ib]);
      const float4 rj = *reinterpret_cast<const float4*>(&Rc[tt][4 * jb]);
      const float4 xi = *reinterpret_cast<const float4*>(&Xw[tt][4 * ib]);
      const float4 xj = *reinterpret_cast<const float4*>(&Xc[tt][4 * jb]);
      const float rI[4] = {ri.x, ri.y, ri.z, ri.w}, rJ[4] = {rj.x, rj.y, rj.z, rj.w};
      const float xI[4] = {xi.x, xi.y, xi.z, xi.w}, xJ[4] = {xj.x, xj.y, xj.z, xj.w};
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          g[u][v] = fmaf(rI[u], rJ[v], g[u][v]);
          a[u][v] = fmaf(xI[u], xJ[v], a[u][v]);
        }
    }
  }
  if (4 * ib < D) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = 4 * ib + u;
      const int j = j0 + 4 * jb;
      float4 gv = make_float4(g[u][0], g[u][1], g[u][2], g[u][3]);
      float4 av = make_float4(a[u][0], a[u][1], a[u][2], a[u][3]);
      if (i >= j && i < j + 4) (&av.x)[i - j] += lambda;
      *reinterpret_cast<float4*>(gram + ((size_t)bh * D + i) * D + j) = gv;
      *reinterpret_cast<float4*>(axx + ((size_t)bh * D + i) * D + j) = av;
    }
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
__global__ void __launch_bounds__(256) k_fit_rhs(const float* Xp, const float* Rp,
                                                 const float* pw, int M, int r, int R,
                                                 const float* evals, const float* evecs,
                                                 const float* rxbar, float* part) {
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
      rv = Rp[((size_t)bh * M + t) * D + col] - rbar[col];
      xv = Xp[((size_t)bh * M + t) * D + col] - xbar[col];
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

__device__ __forceinline__ float fit_pivot(float a) { return a > 0.f ? a : FLT_MIN * 1e10f; }

// Subspace, ridge solve and the intercept.  Grid BH, 512 threads.
// A = L D L^T (unit lower L, one barrier per column: step k updates the
// trailing block from the unscaled column k), then for each right-hand side
// (one warp each, the vector in registers, lane owning rows lane + 32 m) the
// substitutions L z = b, D y = z, L^T x = y in column order.
// Dynamic smem: A (D x (D+1)), Bt (R x (D+1)) right-hand sides by column.
template <int D>
__global__ void __launch_bounds__(512) k_fit_solve(int r, int R, int nchunk, const float* evals,
                                                   const float* evecs, const float* axx,
                                                   const float* rxbar, const float* part,
                                                   float* fitU, float* fitB, float* fitBv,
                                                   spr_head_stats* stats, Header* hdr) {
  extern __shared__ __align__(16) float fsm[];
  constexpr int LD = D + 1, RM = D / 32;
  float* A = fsm;           // D x LD
  float* Bt = A + D * LD;   // R x LD
  __shared__ float rbar[D], xbar[D], xb[D];
  const int bh = blockIdx.x, tid = threadIdx.x, nt = blockDim.x;
  const int warp = tid >> 5, lane = tid & 31, nw = nt >> 5;
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
    Bt[k * LD + i] = s;
  }
  __syncthreads();
  for (int k = 0; k < D; ++k) {
    const float akk = A[k * LD + k];
    if (tid == 0 && !isfinite(akk)) set_error(hdr, ERR_NUMERIC, 10, bh, k);
    const float rk = 1.f / fit_pivot(akk);
    for (int i = k + 1 + warp; i < D; i += nw) {
      const float lik = A[i * LD + k] * rk;
      for (int j = k + 1 + lane; j <= i; j += 32) A[i * LD + j] = fmaf(-lik, A[j * LD + k], A[i * LD + j]);
    }
    __syncthreads();
  }
  for (int e = tid; e < D * D; e += nt) {  // L_ij = A_ij / d_j below the diagonal
    const int i = e / D, j = e % D;
    if (j < i) A[i * LD + j] *= 1.f / fit_pivot(A[j * LD + j]);
  }
  __syncthreads();
  for (int k = warp; k < re; k += nw) {
    float b[RM];
#pragma unroll
    for (int m = 0; m < RM; ++m) b[m] = Bt[k * LD + lane + 32 * m];
#pragma unroll
    for (int j = 0; j < D; ++j) {  // L z = b
      const float zj = __shfl_sync(0xffffffffu, b[j >> 5], j & 31);
#pragma unroll
      for (int m = j >> 5; m < RM; ++m) {
        const int i = lane + 32 * m;
        if (i > j) b[m] = fmaf(-A[i * LD + j], zj, b[m]);
      }
    }
#pragma unroll
    for (int m = 0; m < RM; ++m) {  // D y = z
      const int i = lane + 32 * m;
      b[m] *= 1.f / fit_pivot(A[i * LD + i]);
    }
#pragma unroll
    for (int j = D - 1; j > 0; --j) {  // L^T x = y
      const float xj = __shfl_sync(0xffffffffu, b[j >> 5], j & 31);
#pragma unroll
      for (int m = 0; m <= (j >> 5); ++m) {
        const int i = lane + 32 * m;
        if (i < j) b[m] = fmaf(-A[j * LD + i], xj, b[m]);
      }
    }
#pragma unroll
    for (int m = 0; m < RM; ++m) Bt[k * LD + lane + 32 * m] = b[m];
  }
  __syncthreads();
  // B (d x r_eff, stride d) and the full-width intercept b = Rbar - (xbar B) U_r^T.
  for (int e = tid; e < D * D; e += nt) {
    const int i = e / D, k = e % D;
    fitB[(size_t)bh * D * D + e] = k < re ? Bt[k * LD + i] : 0.f;
  }
  for (int k = tid; k < D; k += nt) {
    float s = 0.f;
    if (k < re)
      for (int i = 0; i < D; ++i) s += xbar[i] * Bt[k * LD + i];
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
// threads; each block takes tiles of APPLY_TR = 32 consecutive permuted rows,
// held transposed in shared memory (Xt[i][row]).  T = X B: thread (i-quarter
// q, rows 4 rb.., columns 2 kb..) sums its quarter of i, the four quarters
// are added in order.  Y: thread (rows 4 rb.., columns 4 cb..) accumulates
// T U_r^T as outer products of 4-vectors.
// Dynamic smem: B as [D][R], U_r as [R][D], Xt [D][XT], Tp [4][R][XT].
constexpr int APPLY_TR = 32;
constexpr int APPLY_XT = APPLY_TR + 4;  // padded transposed row

template <int D>
__global__ void __launch_bounds__(256) k_apply(const float* osp, const float* odn,
                                               const int32_t* pslot, const int32_t* permq,
                                               const float* fitB, const float* fitU,
                                               const float* fitBv, const spr_head_stats* stats,
                                               int R, int N, int M, int H, int64_t sb, int64_t sh,
                                               int64_t sn, bf16* O, int do_fit, Header* hdr) {
  extern __shared__ __align__(16) float fsh[];
  constexpr int XT = APPLY_XT, CB = D / 4;
  float* Bs = fsh;                  // [D][R]
  float* Us = Bs + D * R;           // [R][D]
  float* Xt = Us + R * D;           // [D][XT]
  float* Tp = Xt + D * XT;          // [4][R][XT]
  __shared__ float bv[D];
  __shared__ int slot_s[APPLY_TR], orig_s[APPLY_TR];
  const int bh = blockIdx.y, tid = threadIdx.x;
  const int re = do_fit ? min(stats[bh].r_eff, R) : 0;
  const int rep = (re + 1) & ~1;  // columns of T computed (even)
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
      const int r = e % APPLY_TR, c4 = e / APPLY_TR, pos = pos0 + r;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (pos < N) v = reinterpret_cast<const float4*>(osp + ((size_t)bh * N + pos) * D)[c4];
      Xt[(4 * c4) * XT + r] = v.x;
      Xt[(4 * c4 + 1) * XT + r] = v.y;
      Xt[(4 * c4 + 2) * XT + r] = v.z;
      Xt[(4 * c4 + 3) * XT + r] = v.w;
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
      const int q = tid >> 6, rb = (tid >> 3) & 7, kb = tid & 7;
      for (int k0 = 2 * kb; k0 < rep; k0 += 16) {
        float t[4][2];
#pragma unroll
        for (int u = 0; u < 4; ++u) t[u][0] = t[u][1] = 0.f;
#pragma unroll 4
        for (int i = q * (D / 4); i < (q + 1) * (D / 4); ++i) {
          const float4 x4 = *reinterpret_cast<const float4*>(Xt + i * XT + 4 * rb);
          const float2 b2 = *reinterpret_cast<const float2*>(Bs + i * R + k0);
          const float xr[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            t[u][0] = fmaf(xr[u], b2.x, t[u][0]);
            t[u][1] = fmaf(xr[u], b2.y, t[u][1]);
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          Tp[(q * R + k0) * XT + 4 * rb + u] = t[u][0];
          Tp[(q * R + k0 + 1) * XT + 4 * rb + u] = t[u][1];
        }
      }
      __syncthreads();
      for (int e = tid; e < rep * APPLY_TR; e += 256) {  // add the quarters in order
        const int k = e / APPLY_TR, rr = e % APPLY_TR;
        float s = Tp[k * XT + rr];
#pragma unroll
        for (int qq = 1; qq < 4; ++qq) s += Tp[(qq * R + k) * XT + rr];
        Tp[k * XT + rr] = s;
      }
      __syncthreads();
    }
    if (tid < 8 * CB) {
      const int rb = tid / CB, cb = tid % CB, j = 4 * cb;
      float y[4][4];
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const float4 x4 = *reinterpret_cast<const float4*>(Xt + (j + v) * XT + 4 * rb);
        y[0][v] = x4.x + bv[j + v];
        y[1][v] = x4.y + bv[j + v];
        y[2][v] = x4.z + bv[j + v];
        y[3][v] = x4.w + bv[j + v];
      }
      for (int k = 0; k < re; ++k) {
        const float4 t4 = *reinterpret_cast<const float4*>(Tp + k * XT + 4 * rb);
        const float4 u4 = *reinterpret_cast<const float4*>(Us + k * D + j);
        const float tr[4] = {t4.x, t4.y, t4.z, t4.w}, uc[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int v = 0; v < 4; ++v) y[u][v] = fmaf(tr[u], uc[v], y[u][v]);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int rr = 4 * rb + u, orig = orig_s[rr];
        if (orig < 0) continue;
        float o0 = y[u][0], o1 = y[u][1], o2 = y[u][2], o3 = y[u][3];
        if (slot_s[rr] >= 0) {
          const float4 d4 = *reinterpret_cast<const float4*>(odn + ((size_t)bh * M + slot_s[rr]) * D + j);
          o0 = d4.x;
          o1 = d4.y;
          o2 = d4.z;
          o3 = d4.w;
        }
        uint2 pk;
        pk.x = pack_bf16(o0, o1);
        pk.y = pack_bf16(o2, o3);
        *reinterpret_cast<uint2*>(ob + (int64_t)orig * sn + j) = pk;
      }
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
  const int R = p.r > 0 ? p.r : 1;
  if (M > 0) {
    const int nblk = (M + FIT_GB - 1) / FIT_GB;
    spr_launch(k_fit_gather<D>, dim3(nblk, BH), 256, 0, st, P.osp, P.odn, P.ppos, P.pw, N, M,
               P.xp, P.rp, P.pmean);
    spr_launch(k_fit_moments<D>, dim3(D / 32, BH), 256, 0, st, P.xp, P.rp, P.pw, P.pmean, M, nblk,
               (float)p.lambda, P.gram, P.axx, P.rxbar);
    cudaError_t e = launch_eig(P.gram, BH, D, R, P.eval, P.evec, nullptr, st);
    if (e != cudaSuccess) return e;
    const int nchunk = (M + FIT_TM - 1) / FIT_TM;
    const size_t smr = (size_t)(2 * FIT_TM * D + D * R + FIT_TM * R) * 4;
    cudaFuncSetAttribute(k_fit_rhs<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smr);
    spr_launch(k_fit_rhs<D>, dim3(BH, nchunk), 256, smr, st, P.xp, P.rp, P.pw, M, p.r, R, P.eval,
               P.evec, P.rxbar, P.proj);
    const size_t sm = (size_t)(D + R) * (D + 1) * 4;
    cudaFuncSetAttribute(k_fit_solve<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    spr_launch(k_fit_solve<D>, BH, 512, sm, st, p.r, R, nchunk, P.eval, P.evec, P.axx, P.rxbar,
               P.proj, P.fitU, P.fitB, P.fitBv, P.stats, P.hdr);
  } else {
    spr_launch(k_fit_zero, num_sms(), 256, 0, st, P.fitB, P.fitBv, D, BH);
  }
  if (D == 128) {  // the tensor-core application
    cudaError_t e = launch_apply_tc(p, L, P, O, R, st);
    if (e != cudaSuccess) return e;
    spr_launch(k_stats, (BH + 127) / 128, 128, 0, st, P.stats, P.part,
               P.part + (size_t)BH * 2 * (L.nchunk + 1), L.nchunk, p.Gq, N, M, BH);
    return cudaGetLastError();
  }
  const int RA = (R + 1) & ~1;
  const size_t sm = (size_t)(2 * D * RA + D * APPLY_XT + 4 * RA * APPLY_XT) * 4;
  cudaFuncSetAttribute(k_apply<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  // one wave: four 256-thread blocks fit on an SM (63 registers, 44 KB of
  // shared memory at d = 128), so at most 4 x SMs blocks in all
  const int bph = max(1, min((N + APPLY_TR - 1) / APPLY_TR, num_sms() * 4 / BH));
  spr_launch(k_apply<D>, dim3(bph, BH), 256, sm, st, P.osp, P.odn, P.pslot, P.permq, P.fitB,
             P.fitU, P.fitBv, P.stats, RA, N, M, p.H, p.o_strides[0], p.o_strides[1],
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
