// Routing, probe selection and the attention work list [paperlayer §4 "Sparse
// Execution", App. A.2].
//
// Route (reading R5 of the oracle): per query group i and nonempty K/V group
// j the logit s * qbar_i . c_j + ln|K_j| (the log of the group's unnormalised
// attention mass when its keys sit at the centroid); cells of one query group
// are ranked by softmax mass (ties to the lower j); a cell's tail mass is the
// mass ranked at or after it (one minus the cumulative mass before it, summed
// from the small end so that the tails of peaked rows stay distinct); all of
// it in fp64.
// Tau mode keeps cells whose mass before them is below tau (tail > 1 - tau);
// budget mode keeps every cell whose tail is at least the smallest threshold
// for which the true pair cost plus the M*N probe pairs fits rho_target*N^2.
// Each group's top cell is always kept.
#include <float.h>

#include "spr_internal.cuh"

namespace spr {

__device__ __forceinline__ long long warp_sum_ll(long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Block-wide reductions for blockDim.x a multiple of 32 (<= 1024).
template <typename T, typename Op>
__device__ T block_reduce(T v, T* sh, Op op) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if (lane == 0) sh[w] = v;
  __syncthreads();
  T r = sh[0];
  for (int i = 1; i < nw; ++i) r = op(r, sh[i]);
  __syncthreads();
  return r;
}

// Block-wide exclusive scan of ints (blockDim.x <= 1024); returns the total.
__device__ int block_exscan(int v, int* sh, int* out) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += t;
  }
  __syncthreads();
  if (lane == 31) sh[w] = x;
  __syncthreads();
  int before = 0, total = 0;
  for (int i = 0; i < nw; ++i) {
    if (i < w) before += sh[i];
    total += sh[i];
  }
  *out = before + x - v;
  __syncthreads();
  return total;
}

// L[i][j] = s qbar_i . C_j + ln|K_j| (-inf for empty K/V groups), fp64 from
// the fp64 group means: the routing decision then agrees with an fp64
// evaluation of the rule up to rounding of the last bits.
// Grid (BH, ceil(Gq/32), ceil(Gk/32)), block 256.
__global__ void __launch_bounds__(256) k_route_logits(const double* qbar, const double* Craw,
                                                      const int32_t* kvoff, int Gq, int Gk, int D,
                                                      double scale, double* L) {
  __shared__ double As[32][33], Bs[32][33];
  const int bh = blockIdx.x, i0 = blockIdx.y * 32, j0 = blockIdx.z * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int c0 = 0; c0 < D; c0 += 32) {
    for (int e = threadIdx.x; e < 1024; e += 256) {
      const int rr = e >> 5, c = e & 31;
      As[rr][c] = (i0 + rr < Gq) ? qbar[((size_t)bh * Gq + i0 + rr) * D + c0 + c] : 0.0;
      Bs[rr][c] = (j0 + rr < Gk) ? Craw[((size_t)bh * Gk + j0 + rr) * D + c0 + c] : 0.0;
    }
    __syncthreads();
    for (int c = 0; c < 32; ++c) {
      const double bv = Bs[tx][c];
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[k] = fma(As[ty * 4 + k][c], bv, acc[k]);
    }
    __syncthreads();
  }
  const int j = j0 + tx;
  if (j >= Gk) return;
  const int nk = kvoff[(size_t)bh * (Gk + 1) + j + 1] - kvoff[(size_t)bh * (Gk + 1) + j];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int i = i0 + ty * 4 + k;
    if (i < Gq)
      L[((size_t)bh * Gq + i) * Gk + j] = nk > 0 ? scale * acc[k] + log((double)nk) : -INFINITY;
  }
}

// Softmax mass, rank and tail mass (mass ranked at or after the cell,
// suffix-summed from the smallest so peaked rows keep distinct tails) of every
// cell of one query group, in fp64.  Grid (BH, Gq), block 256 (>= Gk).  Dead
// cells get tail -1; the top-ranked cell of a live row is flagged in `top`.
__global__ void __launch_bounds__(256) k_route_mass(const double* L, const int32_t* qoff,
                                                    const int32_t* kvoff, int Gq, int Gk,
                                                    int tau_mode, double tau, double* tail,
                                                    uint8_t* top, uint8_t* sel) {
  __shared__ double shf[32];
  __shared__ double pis[MAX_GROUPS];
  __shared__ double sorted[MAX_GROUPS];
  const int bh = blockIdx.x, i = blockIdx.y, j = threadIdx.x;
  const int nq = qoff[(size_t)bh * (Gq + 1) + i + 1] - qoff[(size_t)bh * (Gq + 1) + i];
  const size_t cell = ((size_t)bh * Gq + i) * Gk + j;
  bool live = false;
  double l = -INFINITY;
  if (j < Gk) {
    const int nk = kvoff[(size_t)bh * (Gk + 1) + j + 1] - kvoff[(size_t)bh * (Gk + 1) + j];
    live = nq > 0 && nk > 0;
    if (live) l = L[cell];
  }
  const double mx = block_reduce(l, shf, [](double a, double b) { return fmax(a, b); });
  const double w = live ? exp(l - mx) : 0.0;
  const double sum = block_reduce(w, shf, [](double a, double b) { return a + b; });
  const double pi = (live && sum > 0.0) ? w / sum : 0.0;
  if (j < MAX_GROUPS) pis[j] = j < Gk ? (live ? pi : -1.0) : -2.0;
  __syncthreads();
  int rank = 0;
  if (j < Gk) {
    const double mine = live ? pi : -1.0;
    for (int t = 0; t < Gk; ++t) {
      const double o = pis[t];
      rank += (o > mine) || (o == mine && t < j);
    }
    sorted[rank] = live ? pi : 0.0;
  }
  __syncthreads();
  // suffix (inclusive) sums over sorted masses: reverse index, warp scans
  const int jr = blockDim.x - 1 - j;  // reversed position handled by this thread
  const double v = (jr < Gk) ? sorted[jr] : 0.0;
  double x = v;
  const int lane = j & 31, wi = j >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double t = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += t;
  }
  if (lane == 31) shf[wi] = x;
  __syncthreads();
  double before = 0.0;
  for (int t = 0; t < wi; ++t) before += shf[t];
  __syncthreads();
  if (jr < Gk) pis[jr] = before + x;  // tail at sorted position jr
  __syncthreads();
  if (j < Gk) {
    const double r = live ? pis[rank] : -1.0;
    tail[cell] = r;
    top[cell] = live && rank == 0;
    if (tau_mode) sel[cell] = live && (r > 1.0 - tau || rank == 0);
  }
}

// Budget mode: smallest threshold T on the tail-mass bit pattern (fp64 tails
// are non-negative, so their 64-bit patterns order like the values) with
// cost(bits(tail) >= T) <= rho_target N^2 - M N (exact int64 costs); kept
// cells are those at or above T plus every row's top cell.
__global__ void __launch_bounds__(1024) k_route_budget(const double* tail, const uint8_t* top,
                                                       const int32_t* qoff, const int32_t* kvoff,
                                                       int Gq, int Gk, int N, int M, double rho,
                                                       uint8_t* sel, spr_head_stats* stats) {
  __shared__ long long shl[32];
  __shared__ double shf[32];
  __shared__ int nqs[MAX_GROUPS], nks[MAX_GROUPS];
  const int bh = blockIdx.x, tid = threadIdx.x;
  for (int g = tid; g < Gq; g += 1024)
    nqs[g] = qoff[(size_t)bh * (Gq + 1) + g + 1] - qoff[(size_t)bh * (Gq + 1) + g];
  for (int g = tid; g < Gk; g += 1024)
    nks[g] = kvoff[(size_t)bh * (Gk + 1) + g + 1] - kvoff[(size_t)bh * (Gk + 1) + g];
  __syncthreads();
  const double budget = rho * (double)N * (double)N - (double)M * (double)N;
  const int ncell = Gq * Gk;
  const double* R = tail + (size_t)bh * ncell;
  auto bits = [](double r) -> long long { return r < 0.0 ? -1ll : __double_as_longlong(r); };
  // the first RB_CACHE cells of every thread stay in registers (bit pattern,
  // pair count) for the whole search; more cells are read again each round
  constexpr int RB_CACHE = 8;
  long long cb[RB_CACHE];
  long long cw[RB_CACHE];
  long long tmin = 0x7FF0000000000000ll, tmax = -1;
#pragma unroll
  for (int q = 0; q < RB_CACHE; ++q) {
    const int t = tid + q * 1024;
    cb[q] = -1;
    cw[q] = 0;
    if (t < ncell) {
      const int i = t / Gk, j = t - i * Gk;
      if (nqs[i] > 0 && nks[j] > 0) {
        cb[q] = bits(R[t]);
        cw[q] = (long long)nqs[i] * nks[j];
      }
    }
  }
  auto cost = [&](long long T) {
    long long c = 0;
#pragma unroll
    for (int q = 0; q < RB_CACHE; ++q) c += cb[q] >= T ? cw[q] : 0ll;
    for (int t = tid + RB_CACHE * 1024; t < ncell; t += 1024) {
      const int i = t / Gk, j = t - i * Gk;
      if (nqs[i] > 0 && nks[j] > 0 && bits(R[t]) >= T) c += (long long)nqs[i] * nks[j];
    }
    return block_reduce(c, shl, [](long long a, long long b) { return a + b; });
  };
  // the search runs between the smallest and largest live tail patterns
  for (int t = tid; t < ncell; t += 1024) {
    const int i = t / Gk, j = t - i * Gk;
    if (nqs[i] > 0 && nks[j] > 0) {
      const long long b = bits(R[t]);
      tmin = b < tmin ? b : tmin;
      tmax = b > tmax ? b : tmax;
    }
  }
  tmin = block_reduce(tmin, shl, [](long long a, long long b) { return a < b ? a : b; });
  tmax = block_reduce(tmax, shl, [](long long a, long long b) { return a > b ? a : b; });
  // cost(T) is non-increasing in T; cost(tmax + 1) = 0.
  long long Tstar;
  if (tmax < 0 || (double)cost(tmin) <= budget) {
    Tstar = tmax < 0 ? 0 : tmin;
  } else {
    long long lo = tmin, hi = tmax + 1;  // cost(lo) > budget >= cost(hi)
    while (hi - lo > 1) {
      const long long mid = lo + (hi - lo) / 2;
      if ((double)cost(mid) <= budget)
        hi = mid;
      else
        lo = mid;
    }
    Tstar = hi;
  }
  double kept_min = INFINITY;
  int only_top = 1;
  for (int t = tid; t < ncell; t += 1024) {
    const int i = t / Gk, j = t - i * Gk;
    const bool live = nqs[i] > 0 && nks[j] > 0;
    const bool above = live && bits(R[t]) >= Tstar;
    const bool k = above || (live && top[(size_t)bh * ncell + t]);
    sel[(size_t)bh * ncell + t] = k;
    if (above) {
      kept_min = fmin(kept_min, R[t]);
      if (!top[(size_t)bh * ncell + t]) only_top = 0;
    }
  }
  kept_min = block_reduce(kept_min, shf, [](double a, double b) { return fmin(a, b); });
  const long long nt = block_reduce((long long)(1 - only_top), shl,
                                    [](long long a, long long b) { return a + b; });
  if (tid == 0) {
    stats[bh].route_threshold = kept_min;
    stats[bh].flags |= nt == 0 ? 1 : 0;
  }
}

// CSR of routed cells (ascending K/V group), merged contiguous key ranges,
// routed pair count.  Grid BH, block 256 (threads over query groups).
__global__ void __launch_bounds__(256) k_route_csr(const uint8_t* sel, const int32_t* qoff,
                                                   const int32_t* kvoff, int Gq, int Gk,
                                                   int32_t* rowptr, int32_t* colidx,
                                                   int32_t* runptr, int2* runs,
                                                   spr_head_stats* stats) {
  __shared__ int sh[32];
  __shared__ long long shl[32];
  const int bh = blockIdx.x, i = threadIdx.x;
  const uint8_t* S = sel + (size_t)bh * Gq * Gk;
  const int32_t* ko = kvoff + (size_t)bh * (Gk + 1);
  int cnt = 0, nrun = 0;
  long long keys = 0;
  if (i < Gq) {
    int end = -1;
    for (int j = 0; j < Gk; ++j) {
      if (!S[(size_t)i * Gk + j]) continue;
      ++cnt;
      keys += ko[j + 1] - ko[j];
      if (ko[j] != end) ++nrun;
      end = ko[j + 1];
    }
  }
  int cbase, rbase;
  const int ctot = block_exscan(cnt, sh, &cbase);
  const int rtot = block_exscan(nrun, sh, &rbase);
  if (i < Gq) {
    rowptr[(size_t)bh * (Gq + 1) + i] = cbase;
    runptr[(size_t)bh * (Gq + 1) + i] = rbase;
    if (i == 0) {
      rowptr[(size_t)bh * (Gq + 1) + Gq] = ctot;
      runptr[(size_t)bh * (Gq + 1) + Gq] = rtot;
    }
    int c = cbase, r = rbase - 1, end = -1;
    for (int j = 0; j < Gk; ++j) {
      if (!S[(size_t)i * Gk + j]) continue;
      colidx[(size_t)bh * Gq * Gk + c++] = j;
      if (ko[j] != end) {
        ++r;
        runs[(size_t)bh * Gq * Gk + r] = make_int2(ko[j], ko[j + 1]);
      } else {
        runs[(size_t)bh * Gq * Gk + r].y = ko[j + 1];
      }
      end = ko[j + 1];
    }
  }
  const long long nq =
      i < Gq ? (long long)(qoff[(size_t)bh * (Gq + 1) + i + 1] - qoff[(size_t)bh * (Gq + 1) + i]) : 0;
  const long long pairs = block_reduce(nq * keys, shl, [](long long a, long long b) { return a + b; });
  if (i == 0) {
    stats[bh].routed_pairs = pairs;
    stats[bh].nnz_cells = ctot;
  }
}

// Stratified probes with coverage weights (reading R6), or every probe
// weighing 1 / (probes selected) when `uniform`.  Grid BH, block 256.
// pslot[bh][pos] receives the probe slot of each probed permuted position (the
// caller fills it with -1 first).
__global__ void __launch_bounds__(256) k_probes(const int32_t* qoff, const int32_t* permq, int Gq,
                                                int N, int M, int uniform, int32_t* ppos,
                                                int32_t* pidx, float* pw, int32_t* pslot,
                                                spr_head_stats* stats) {
  __shared__ int sh[32];
  __shared__ long long shl[32];
  __shared__ long long rems[MAX_GROUPS];
  __shared__ int cnts[MAX_GROUPS];
  const int bh = blockIdx.x, g = threadIdx.x;
  const int cnt = g < Gq ? qoff[(size_t)bh * (Gq + 1) + g + 1] - qoff[(size_t)bh * (Gq + 1) + g] : 0;
  if (g < MAX_GROUPS) cnts[g] = cnt;
  int dummy;
  const int ne = block_exscan(cnt > 0 ? 1 : 0, sh, &dummy);
  if (g == 0) stats[bh].gq_nonempty = ne;
  long long m = 0;
  if (M > 0) {
    if (M >= ne) {
      m = cnt > 0 ? 1 : 0;
      const long long R = M - ne, S = (long long)N - ne;
      long long rem = -1;
      if (R > 0 && cnt > 0) {
        const long long num = R * (long long)(cnt - 1);
        m += num / S;
        rem = num % S;
      }
      const long long fl = (R > 0 && cnt > 0) ? m - 1 : 0;
      const long long flsum = block_reduce(fl, shl, [](long long a, long long b) { return a + b; });
      if (g < MAX_GROUPS) rems[g] = rem;
      __syncthreads();
      if (R > 0 && g < Gq && rem > 0) {
        const long long left = R - flsum;
        int rank = 0;
        for (int t = 0; t < Gq; ++t)
          rank += rems[t] > 0 && (rems[t] > rem || (rems[t] == rem && t < g));
        if (rank < left) m += 1;
      }
    } else if (g < Gq && cnt > 0) {
      int rank = 0;
      for (int t = 0; t < Gq; ++t) rank += cnts[t] > 0 && (cnts[t] > cnt || (cnts[t] == cnt && t < g));
      m = rank < M ? 1 : 0;
    }
  }
  __syncthreads();
  const long long covered =
      block_reduce(m > 0 ? (long long)cnt : 0ll, shl, [](long long a, long long b) { return a + b; });
  const long long nsel =
      block_reduce((long long)m, shl, [](long long a, long long b) { return a + b; });
  int base;
  block_exscan((int)m, sh, &base);
  if (g < Gq && m > 0) {
    const int q0 = qoff[(size_t)bh * (Gq + 1) + g];
    const float w = uniform ? (float)(1.0 / (double)min(nsel, (long long)M))
                            : (float)(((double)cnt / (double)m) / (double)covered);
    for (int t = 0; t < (int)m && base + t < M; ++t) {
      const int pos = q0 + (int)(((2ll * t + 1) * cnt) / (2 * m));
      ppos[(size_t)bh * M + base + t] = pos;
      pidx[(size_t)bh * M + base + t] = permq[(size_t)bh * N + pos];
      pw[(size_t)bh * M + base + t] = w;
      pslot[(size_t)bh * N + pos] = base + t;
    }
  }
}

// Attention work list: probe tiles of every head first (they span all keys),
// then the query tiles of every (head, query group) with routed cells.
// Items: {bh, q0, nrows, grp} with grp = -1 for a probe tile (q0 = probe slot).
__global__ void __launch_bounds__(1024) k_worklist(const int32_t* qoff, const int32_t* rowptr,
                                                   int BH, int Gq, int M, int max_items,
                                                   int4* items, Header* hdr) {
  __shared__ int sh[32];
  const int tid = threadIdx.x;
  const int nent = BH + BH * Gq;
  const int per = (nent + 1023) / 1024;
  const int e0 = tid * per, e1 = min(nent, e0 + per);
  auto count = [&](int e) -> int {
    if (e < BH) return (M + ATT_BM - 1) / ATT_BM;
    const int bh = (e - BH) / Gq, i = (e - BH) % Gq;
    const int nq = qoff[(size_t)bh * (Gq + 1) + i + 1] - qoff[(size_t)bh * (Gq + 1) + i];
    const int nc = rowptr[(size_t)bh * (Gq + 1) + i + 1] - rowptr[(size_t)bh * (Gq + 1) + i];
    return (nq > 0 && nc > 0) ? (nq + ATT_BM - 1) / ATT_BM : 0;
  };
  int local = 0;
  for (int e = e0; e < e1; ++e) local += count(e);
  int base;
  const int total = block_exscan(local, sh, &base);
  if (tid == 0) {
    hdr->n_items = total <= max_items ? total : 0;
    hdr->work_next = 0;
    if (total > max_items) set_error(hdr, ERR_WORKLIST, total, max_items, 0);
  }
  if (total > max_items) return;
  int k = base;
  for (int e = e0; e < e1; ++e) {
    const int c = count(e);
    for (int t = 0; t < c; ++t) {
      if (e < BH) {
        const int q0 = t * ATT_BM;
        items[k++] = make_int4(e, q0, min(ATT_BM, M - q0), -1);
      } else {
        const int bh = (e - BH) / Gq, i = (e - BH) % Gq;
        const int s = qoff[(size_t)bh * (Gq + 1) + i], en = qoff[(size_t)bh * (Gq + 1) + i + 1];
        const int q0 = s + t * ATT_BM;
        items[k++] = make_int4(bh, q0, min(ATT_BM, en - q0), i);
      }
    }
  }
}

template <int D>
__global__ void __launch_bounds__(256) k_gather_probe(const bf16* Qp, const int32_t* ppos, int N,
                                                      int M, int BH, bf16* out) {
  constexpr int LANES = D / 8;
  const int64_t total = (int64_t)BH * M * LANES;
  for (int64_t e = (int64_t)blockIdx.x * 256 + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * 256) {
    const int64_t rowi = e / LANES;
    const int c = (int)(e % LANES);
    const int bh = (int)(rowi / M);
    const int pos = ppos[rowi];
    reinterpret_cast<uint4*>(out)[e] =
        reinterpret_cast<const uint4*>(Qp + ((size_t)bh * N + pos) * D)[c];
  }
}

cudaError_t launch_route(const spr_params& p, const Layout& L, const Ptrs& P, cudaStream_t st) {
  const int BH = L.BH, D = p.d;
  const double scale = p.scale > 0.f ? (double)p.scale : 1.0 / sqrt((double)D);
  spr_launch(k_route_logits, dim3(BH, (p.Gq + 31) / 32, (p.Gk + 31) / 32), 256, 0, st,
             P.qbar64, P.craw64, P.kvoff, p.Gq, p.Gk, D, scale, P.logit);
  const int tau_mode = p.route_mode == SPR_ROUTE_TAU;
  spr_launch(k_route_mass, dim3(BH, p.Gq), 256, 0, st, P.logit, P.qoff, P.kvoff, p.Gq, p.Gk,
             tau_mode, p.tau, P.entry, P.top, P.sel);
  if (!tau_mode)
    spr_launch(k_route_budget, BH, 1024, 0, st, P.entry, P.top, P.qoff, P.kvoff, p.Gq, p.Gk,
               p.N, p.M, p.rho_target, P.sel, P.stats);
  spr_launch(k_route_csr, BH, 256, 0, st, P.sel, P.qoff, P.kvoff, p.Gq, p.Gk, P.rowptr, P.colidx,
                                  P.runptr, P.runs, P.stats);
  if (cudaMemsetAsync(P.pslot, 0xFF, (size_t)BH * p.N * sizeof(int32_t), st) != cudaSuccess)
    return cudaGetLastError();
  spr_launch(k_probes, BH, 256, 0, st, P.qoff, P.permq, p.Gq, p.N, p.M,
             p.weights == SPR_WEIGHTS_UNIFORM ? 1 : 0, P.ppos, P.pidx, P.pw,
             P.pslot, P.stats);
  if (p.M > 0) {
    const int grid = num_sms() * 4;
    if (D == 64)
      spr_launch(k_gather_probe<64>, grid, 256, 0, st, P.Qp, P.ppos, p.N, p.M, BH, P.qprobe);
    else
      spr_launch(k_gather_probe<128>, grid, 256, 0, st, P.Qp, P.ppos, p.N, p.M, BH, P.qprobe);
  }
  spr_launch(k_worklist, 1, 1024, 0, st, P.qoff, P.rowptr, BH, p.Gq, p.M, L.max_items, P.items, P.hdr);
  return cudaGetLastError();
}

}  // namespace spr
