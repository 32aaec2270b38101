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
  auto live_cell = [&](int t) {
    const int i = t / Gk, j = t - i * Gk;
    return nqs[i] > 0 && nks[j] > 0;
  };
  auto weight = [&](int t) -> long long {
    const int i = t / Gk, j = t - i * Gk;
    return (long long)nqs[i] * nks[j];
  };
  auto cost = [&](long long T) {  // pairs of the live cells at or above pattern T
    long long c = 0;
    for (int t = tid; t < ncell; t += 1024)
      if (live_cell(t) && bits(R[t]) >= T) c += weight(t);
    return block_reduce(c, shl, [](long long a, long long b) { return a + b; });
  };
  long long tmin = 0x7FF0000000000000ll, tmax = -1;
  for (int t = tid; t < ncell; t += 1024) {
    if (live_cell(t)) {
      const long long b = bits(R[t]);
      tmin = b < tmin ? b : tmin;
      tmax = b > tmax ? b : tmax;
    }
  }
  tmin = block_reduce(tmin, shl, [](long long a, long long b) { return a < b ? a : b; });
  tmax = block_reduce(tmax, shl, [](long long a, long long b) { return a > b ? a : b; });
  // cost(T) is non-increasing in T.  T* = B* + 1 with B* the largest live
  // pattern whose cost exceeds the budget; T* = tmin when every live cell fits.
  // B* is located with 1024 sample patterns (every (ncell / 1024)-th cell,
  // sorted): each live cell's pairs go to the bin of samples around its
  // pattern, suffix sums over the bins give the bin holding B*, and B* is
  // found exactly among that bin's cells (or, past RB_LIST of them, by
  // bisection over the bin's pattern range).
  constexpr int RB_LIST = 1536;
  __shared__ long long samp[1024];
  __shared__ unsigned long long binw[1025];
  __shared__ long long lb[RB_LIST];
  __shared__ long long lw[RB_LIST];
  __shared__ int nl_s;
  {
    const int t = (int)(((long long)tid * ncell) / 1024);
    samp[tid] = (t < ncell && live_cell(t)) ? bits(R[t]) : -1;
  }
  binw[tid] = 0ull;
  if (tid == 0) {
    binw[1024] = 0ull;
    nl_s = 0;
  }
  __syncthreads();
  for (int k = 2; k <= 1024; k <<= 1) {  // bitonic sort of the samples, ascending
    for (int j = k >> 1; j > 0; j >>= 1) {
      const int ixj = tid ^ j;
      if (ixj > tid) {
        const long long a = samp[tid], b = samp[ixj];
        if ((a > b) == ((tid & k) == 0)) {
          samp[tid] = b;
          samp[ixj] = a;
        }
      }
      __syncthreads();
    }
  }
  auto bin_of = [&](long long b) {  // samples <= b: 0 .. 1024
    int lo = 0, hi = 1024;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (samp[mid] <= b) lo = mid + 1; else hi = mid;
    }
    return lo;
  };
  for (int t = tid; t < ncell; t += 1024)
    if (live_cell(t)) atomicAdd(&binw[bin_of(bits(R[t]))], (unsigned long long)weight(t));
  __syncthreads();
  // suffix sums S(k) = sum of bins k .. 1024 (non-increasing in k): thread
  // tid holds S(1023 - tid) from a prefix scan over the bins in reverse order
  const long long s_top = (long long)binw[1024];
  long long mine;
  {
    const int lane = tid & 31, w = tid >> 5;
    long long inc = (long long)binw[1023 - tid];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long u = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += u;
    }
    if (lane == 31) shl[w] = inc;
    __syncthreads();
    long long before = 0;
    for (int i = 0; i < w; ++i) before += shl[i];
    __syncthreads();
    mine = before + inc + s_top;
  }
  // k* = the largest bin with S(k*) > budget: bins 0 .. k* are exactly those
  const int above = (int)block_reduce((long long)((double)mine > budget ? 1 : 0), shl,
                                      [](long long a, long long b) { return a + b; });
  const bool top_over = (double)s_top > budget;
  long long Tstar;
  if (tmax < 0) {
    Tstar = 0;
  } else if (above == 0 && !top_over) {
    Tstar = tmin;  // every live cell fits
  } else {
    const int kst = top_over ? 1024 : above - 1;
    // the cost of the cells in the bins above k*: S(k* + 1)
    long long part = 0;
    for (int k = kst + 1 + tid; k <= 1024; k += 1024) part += (long long)binw[k];
    const long long c_above = block_reduce(part, shl, [](long long a, long long b) { return a + b; });
    for (int t = tid; t < ncell; t += 1024) {
      if (live_cell(t)) {
        const long long b = bits(R[t]);
        if (bin_of(b) == kst) {
          const int at = atomicAdd(&nl_s, 1);
          if (at < RB_LIST) {
            lb[at] = b;
            lw[at] = weight(t);
          }
        }
      }
    }
    __syncthreads();
    const int nl = nl_s;
    long long bstar = -1;
    if (nl <= RB_LIST) {
      // cost(b) for each listed pattern: the cells above the bin plus the
      // listed cells at or above b; B* = the largest with cost > budget
      for (int e = tid; e < nl; e += 1024) {
        long long c = c_above;
        for (int f = 0; f < nl; ++f) c += lb[f] >= lb[e] ? lw[f] : 0ll;
        if ((double)c > budget && lb[e] > bstar) bstar = lb[e];
      }
      bstar = block_reduce(bstar, shl, [](long long a, long long b) { return a > b ? a : b; });
    } else {
      // bisection over the bin's pattern range [lo, hi): cost(lo) > budget >= cost(hi)
      long long lo = kst > 0 ? samp[kst - 1] : tmin, hi = kst < 1024 ? samp[kst] : tmax + 1;
      if (lo < tmin) lo = tmin;
      while (hi - lo > 1) {
        const long long mid = lo + (hi - lo) / 2;
        if ((double)cost(mid) <= budget)
          hi = mid;
        else
          lo = mid;
      }
      bstar = hi - 1;
    }
    Tstar = bstar + 1;
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

// Distance-ranked probes (reading R16): the squared distance of permuted query
// pos (original row n) to its group's centroid in query-response coordinates,
//   ||u_n - c_g||^2 = ||u_n||^2 - 2 (f_n q_n . Bq_g - beta_g),
// with f_n = scale / rms_n, Bq_g = A a_g (bf16 hi + lo rows) and beta_g =
// ||c_g||^2 / 2 from the final query centroids a_g, ||u_n||^2 from the RMS
// pass.  One warp per permuted row: lane l holds D / 32 coordinates.
template <int D>
__global__ void __launch_bounds__(256) k_probe_dist(const bf16* Qp, const int32_t* permq,
                                                    const int32_t* labq, const float* rms,
                                                    const float* un2, const bf16* bq,
                                                    const float* beta, int N, int G,
                                                    int split_rows, float scale, int BH,
                                                    float* dist) {
  constexpr int V = D / 32;
  const int lane = threadIdx.x & 31;
  const long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (w >= (long long)BH * N) return;
  const int bh = (int)(w / N), pos = (int)(w - (long long)bh * N);
  const int n = permq[(size_t)bh * N + pos];
  const int g = labq[(size_t)bh * N + n];
  const bf16* q = Qp + ((size_t)bh * N + pos) * D + lane * V;
  const bf16* bh_row = bq + (((size_t)bh * 2 + 0) * split_rows + g) * D + lane * V;
  const bf16* bl_row = bq + (((size_t)bh * 2 + 1) * split_rows + g) * D + lane * V;
  float acc = 0.f;
#pragma unroll
  for (int v = 0; v < V; ++v)
    acc = fmaf(__bfloat162float(q[v]),
               __bfloat162float(bh_row[v]) + __bfloat162float(bl_row[v]), acc);
  acc = warp_sum(acc);
  if (lane == 0) {
    const float f = scale / rms[(size_t)bh * N + n];
    const float score = fmaf(f, acc, -beta[(size_t)bh * G + g]);
    dist[(size_t)bh * N + pos] = fmaf(-2.f, score, un2[(size_t)bh * N + n]);
  }
}

// Orderable 64-bit key of (distance, original row): smaller distance first,
// ties to the lower row; NaN sorts last.
__device__ __forceinline__ unsigned long long dist_key(float d, int row) {
  uint32_t b = __float_as_uint(d);
  if (d != d) b = 0xffffffffu;
  else b = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  return ((unsigned long long)b << 32) | (uint32_t)row;
}

// Replace each query group's stratified probe rows by its m_g rows nearest
// the centroid (reading R16; counts and weights unchanged).  Grid (Gq, BH),
// 256 threads.  The group's slots are the entries of the ascending probe
// list inside its position range; the m_g smallest keys are found one at a
// time (the k-th smallest is the smallest key above the (k-1)-th), then
// written in ascending position order.
__global__ void __launch_bounds__(256) k_probes_ranked(const int32_t* qoff, const int32_t* permq,
                                                       const float* dist, int Gq, int N, int M,
                                                       int32_t* ppos, int32_t* pidx,
                                                       int32_t* pslot) {
  __shared__ int sel[MAX_PROBES];
  __shared__ unsigned long long shk[8];
  __shared__ int shp[8];
  const int g = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
  const int q0 = qoff[(size_t)bh * (Gq + 1) + g], q1 = qoff[(size_t)bh * (Gq + 1) + g + 1];
  if (q1 <= q0 || M == 0) return;
  int32_t* pp = ppos + (size_t)bh * M;
  auto lower = [&](int x) {  // first probe slot whose position is >= x
    int lo = 0, hi = M;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (pp[mid] < x) lo = mid + 1; else hi = mid;
    }
    return lo;
  };
  const int base = lower(q0), m = lower(q1) - base;
  if (m <= 0) return;
  // the stratified rows lose their slots
  for (int t = tid; t < m; t += 256) pslot[(size_t)bh * N + pp[base + t]] = -1;
  const float* dg = dist + (size_t)bh * N;
  const int32_t* pq = permq + (size_t)bh * N;
  unsigned long long last = 0ull;
  for (int k = 0; k < m; ++k) {
    unsigned long long best = ~0ull;
    int bpos = -1;
    for (int pos = q0 + tid; pos < q1; pos += 256) {
      const unsigned long long key = dist_key(dg[pos], pq[pos]);
      if ((k == 0 || key > last) && key < best) {
        best = key;
        bpos = pos;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long ok = __shfl_xor_sync(0xffffffffu, best, o);
      const int op = __shfl_xor_sync(0xffffffffu, bpos, o);
      if (ok < best) {
        best = ok;
        bpos = op;
      }
    }
    if ((tid & 31) == 0) {
      shk[tid >> 5] = best;
      shp[tid >> 5] = bpos;
    }
    __syncthreads();
    if (tid == 0) {
      for (int i = 1; i < 8; ++i)
        if (shk[i] < shk[0]) {
          shk[0] = shk[i];
          shp[0] = shp[i];
        }
      sel[k] = shp[0];
    }
    __syncthreads();
    last = shk[0];
    __syncthreads();
  }
  // ascending positions: each chosen position's rank among the chosen
  for (int t = tid; t < m; t += 256) {
    const int pos = sel[t];
    int rank = 0;
    for (int u = 0; u < m; ++u) rank += sel[u] < pos;
    pp[base + rank] = pos;
    pidx[(size_t)bh * M + base + rank] = pq[pos];
    pslot[(size_t)bh * N + pos] = base + rank;
  }
}

// Attention work list: probe items of every head first (they span all keys),
// then the query items of every (head, query group) with routed cells; an
// item holds up to ATT_ITEM rows.
// Items: {bh, q0, nrows, grp} with grp = -1 for probe rows (q0 = probe slot).
__global__ void __launch_bounds__(1024) k_worklist(const int32_t* qoff, const int32_t* rowptr,
                                                   int BH, int Gq, int M, int max_items,
                                                   int4* items, Header* hdr) {
  __shared__ int sh[32];
  const int tid = threadIdx.x;
  const int nent = BH + BH * Gq;
  const int per = (nent + 1023) / 1024;
  const int e0 = tid * per, e1 = min(nent, e0 + per);
  auto count = [&](int e) -> int {
    if (e < BH) return (M + ATT_ITEM - 1) / ATT_ITEM;
    const int bh = (e - BH) / Gq, i = (e - BH) % Gq;
    const int nq = qoff[(size_t)bh * (Gq + 1) + i + 1] - qoff[(size_t)bh * (Gq + 1) + i];
    const int nc = rowptr[(size_t)bh * (Gq + 1) + i + 1] - rowptr[(size_t)bh * (Gq + 1) + i];
    return (nq > 0 && nc > 0) ? (nq + ATT_ITEM - 1) / ATT_ITEM : 0;
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
        const int q0 = t * ATT_ITEM;
        items[k++] = make_int4(e, q0, min(ATT_ITEM, M - q0), -1);
      } else {
        const int bh = (e - BH) / Gq, i = (e - BH) % Gq;
        const int s = qoff[(size_t)bh * (Gq + 1) + i], en = qoff[(size_t)bh * (Gq + 1) + i + 1];
        const int q0 = s + t * ATT_ITEM;
        items[k++] = make_int4(bh, q0, min(ATT_ITEM, en - q0), i);
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
  if (p.probes == SPR_PROBES_RANKED && p.M > 0) {
    const int split_rows = bq_rows(p.Gk > p.Gq ? p.Gk : p.Gq, D);
    const float fscale = (float)scale;
    const long long warps = (long long)BH * p.N;
    const int grid = (int)((warps * 32 + 255) / 256);
    if (D == 64)
      spr_launch(k_probe_dist<64>, grid, 256, 0, st, static_cast<const bf16*>(P.Qp), P.permq,
                 P.labq, P.rms, P.un2, static_cast<const bf16*>(P.bq16), P.beta, p.N, p.Gq,
                 split_rows, fscale, BH, P.pdist);
    else
      spr_launch(k_probe_dist<128>, grid, 256, 0, st, static_cast<const bf16*>(P.Qp), P.permq,
                 P.labq, P.rms, P.un2, static_cast<const bf16*>(P.bq16), P.beta, p.N, p.Gq,
                 split_rows, fscale, BH, P.pdist);
    spr_launch(k_probes_ranked, dim3(p.Gq, BH), 256, 0, st, P.qoff, P.permq,
               static_cast<const float*>(P.pdist), p.Gq, p.N, p.M, P.ppos, P.pidx, P.pslot);
  }
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
