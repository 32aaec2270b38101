// Response-Coupled Partitioning on the GPU [paperlayer §4, App. B.1, B.2;
// gist-nl §2A]: sampled-query metric, its eigen-coordinates, key k-means,
// paired K/V groups, centred K/V centroids, RMS-normalised query-response
// coordinates (never materialised: the query k-means works in the head
// dimension through Ctilde^T Ctilde), query k-means and the stable
// group-major permutations of Q, K and V.
#include <float.h>

#include "spr_internal.cuh"

namespace spr {

int padded_p(int) { return 32; }

// ---------------------------------------------------------------------------
// M_K = Q_s^T Q_s / M_s with Q_s the rows floor(i N / M_s), i < M_s.
// Grid (BH, (D/32)^2), one 32x32 output tile per block.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) k_metric(TensorView Q, int N, int Ms, float* MK) {
  constexpr int SB = 128;  // sampled rows staged per step
  const int bh = blockIdx.x;
  const int ti = blockIdx.y / (D / 32), tj = blockIdx.y % (D / 32);
  __shared__ float As[SB][33], Bs[SB][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  // a stage: 128 sampled rows x 32 columns of each operand, as 16-byte
  // pieces (4 per row and operand), every load issued before any is used
  constexpr int NL = SB * 4 * 2 / 256;
  for (int s0 = 0; s0 < Ms; s0 += SB) {
    uint4 v[NL];
#pragma unroll
    for (int q = 0; q < NL; ++q) {
      const int e = q * 256 + threadIdx.x;
      const int mat = e / (SB * 4), rr = (e % (SB * 4)) >> 2, c = e & 3, s = s0 + rr;
      v[q] = make_uint4(0, 0, 0, 0);
      if (s < Ms) {
        const int row = (int)(((int64_t)s * N) / Ms);
        v[q] = *reinterpret_cast<const uint4*>(Q.row(bh, row) + (mat ? tj : ti) * 32 + c * 8);
      }
    }
#pragma unroll
    for (int q = 0; q < NL; ++q) {
      const int e = q * 256 + threadIdx.x;
      const int mat = e / (SB * 4), rr = (e % (SB * 4)) >> 2, c = e & 3;
      float* dst = (mat ? &Bs[rr][0] : &As[rr][0]) + c * 8;
      const uint32_t w[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[k]));
        dst[2 * k] = f.x;
        dst[2 * k + 1] = f.y;
      }
    }
    __syncthreads();
#pragma unroll 8
    for (int rr = 0; rr < SB; ++rr) {
      const float bv = Bs[rr][tx];
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[k] += As[rr][ty * 4 + k] * bv;
    }
    __syncthreads();
  }
#pragma unroll
  for (int k = 0; k < 4; ++k)
    MK[((size_t)bh * D + ti * 32 + ty * 4 + k) * D + tj * 32 + tx] = acc[k] / (float)Ms;
}

// W[:, k] = u_k sqrt(lambda_k / sum_j lambda_j) for k < p; zero for p <= k < pp.
// The eigenvalue sum of the positive semidefinite M_K is its trace.
__global__ void k_keyweights(const float* evals, const float* evecs, const float* trace, int D,
                             int p, int pp, float* W) {
  const int bh = blockIdx.x;
  const float tot = trace[bh];
  for (int e = threadIdx.x; e < D * pp; e += blockDim.x) {
    const int i = e / pp, k = e % pp;
    float w = 0.f;
    if (k < p && tot > 0.f)
      w = evecs[((size_t)bh * D + i) * D + k] * sqrtf(fmaxf(evals[(size_t)bh * D + k], 0.f) / tot);
    W[(size_t)bh * D * pp + e] = w;
  }
}

// ---------------------------------------------------------------------------
// k-means initial rows: partial Fisher-Yates over 0..N-1 driven by splitmix64
// (Steele, Lea & Flood 2014).  Stream state: seed XOR ((2 bh + which + 1) *
// 0xD1B54A32D192ED03).  One block per (bh, which); a small open-addressing map
// stores the displaced entries of the virtual identity array.
// ---------------------------------------------------------------------------
__global__ void k_init_idx(int N, int Gk, int Gq, uint64_t seed, int head0, int32_t* init_k,
                           int32_t* init_q) {
  constexpr int CAP = 2048;
  __shared__ int keys[CAP], vals[CAP];
  const int bh = blockIdx.x, which = blockIdx.y;
  const int G = which ? Gq : Gk;
  int32_t* out = (which ? init_q : init_k) + (size_t)bh * G;
  for (int i = threadIdx.x; i < CAP; i += blockDim.x) keys[i] = -1;
  __syncthreads();
  if (threadIdx.x != 0) return;
  auto slot = [&](int k) {
    uint32_t h = (uint32_t)k * 2654435761u;
    int s = (int)(h & (CAP - 1));
    while (keys[s] != -1 && keys[s] != k) s = (s + 1) & (CAP - 1);
    return s;
  };
  auto get = [&](int k) {
    const int s = slot(k);
    return keys[s] == k ? vals[s] : k;
  };
  auto put = [&](int k, int v) {
    const int s = slot(k);
    keys[s] = k;
    vals[s] = v;
  };
  // the stream of head head0 + bh (heads of one call are numbered from head0)
  uint64_t x = seed ^ ((uint64_t)(2 * ((int64_t)head0 + bh) + which + 1) * 0xD1B54A32D192ED03ull);
  for (int i = 0; i < G; ++i) {
    x += 0x9E3779B97F4A7C15ull;
    uint64_t z = x;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    z ^= z >> 31;
    const int j = i + (int)(z % (uint64_t)(N - i));
    const int ai = get(i), aj = get(j);
    put(i, aj);
    put(j, ai);
    out[i] = aj;
  }
}

__global__ void k_init_centk(const float* Z, int N, int G, int PP, const int32_t* init,
                             float* cent) {
  const int bh = blockIdx.x;
  for (int e = threadIdx.x; e < G * PP; e += blockDim.x) {
    const int g = e / PP, k = e % PP;
    cent[(size_t)bh * G * PP + e] = Z[((size_t)bh * N + init[(size_t)bh * G + g]) * PP + k];
  }
}

// Warm start of the key k-means [paperlayer App. C.1]: the previous call's
// raw-key group means in this call's key-response coordinates,
// c_g = W^T Craw_g (z = W^T k is linear; zero columns of W give zeros).
__global__ void k_warm_centk(const float* Craw, const float* W, int G, int D, int PP, float* cent) {
  const int bh = blockIdx.x;
  for (int e = threadIdx.x; e < G * PP; e += blockDim.x) {
    const int g = e / PP, k = e % PP;
    const float* c = Craw + ((size_t)bh * G + g) * D;
    const float* w = W + (size_t)bh * D * PP + k;
    float s = 0.f;
    for (int i = 0; i < D; ++i) s = fmaf(c[i], w[(size_t)i * PP], s);
    cent[(size_t)bh * G * PP + e] = s;
  }
}

// ---------------------------------------------------------------------------
// ---------------------------------------------------------------------------
// Per (bh, g): base of each chunk within the group (exclusive scan over
// chunks), group sizes, and group offsets (exclusive scan over g).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_chunk_scan(const int32_t* __restrict__ chunk_cnt,
                                                    int nchunk, int G, int N,
                                                    int32_t* __restrict__ cbase,
                                                    int32_t* __restrict__ off,
                                                    int32_t* __restrict__ counts) {
  __shared__ int wsum[8];
  const int bh = blockIdx.x, g = threadIdx.x;
  int tot = 0;
  if (g < G) {
    const int32_t* src = chunk_cnt + (size_t)bh * nchunk * G + g;
    int32_t* dst = cbase + (size_t)bh * nchunk * G + g;
    int c = 0;
    for (; c + 8 <= nchunk; c += 8) {  // eight loads in flight ahead of the running sum
      int v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = src[(size_t)(c + u) * G];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        dst[(size_t)(c + u) * G] = tot;
        tot += v[u];
      }
    }
    for (; c < nchunk; ++c) {
      dst[(size_t)c * G] = tot;
      tot += src[(size_t)c * G];
    }
    counts[(size_t)bh * G + g] = tot;
  }
  // block exclusive scan of tot over g
  int v = tot;
  const int lane = g & 31, w = g >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  if (lane == 31) wsum[w] = v;
  __syncthreads();
  int before = 0;
  for (int i = 0; i < w; ++i) before += wsum[i];
  if (g < G) off[(size_t)bh * (G + 1) + g] = before + v - tot;
  if (g == 0) off[(size_t)bh * (G + 1) + G] = N;
}

// Stable scatter: perm[off[g] + chunk base + rank among equal labels before
// this row in the chunk] = row.
__global__ void __launch_bounds__(CHUNK) k_scatter(const int32_t* lab, int N, int G, int nchunk,
                                                  const int32_t* cbase, const int32_t* off,
                                                  int32_t* perm, Header* hdr) {
  __shared__ int cnt[32][MAX_GROUPS];
  const int bh = blockIdx.y, chunk = blockIdx.x, tid = threadIdx.x;
  const int w = tid >> 5, lane = tid & 31;
  for (int e = tid; e < 32 * G; e += CHUNK) cnt[e / G][e % G] = 0;
  __syncthreads();
  const int n = chunk * CHUNK + tid;
  int g = n < N ? lab[(size_t)bh * N + n] : -1;
  if (g >= G || g < -1) {
    set_error(hdr, ERR_INDEX, 1, bh, n);
    g = -1;
  }
  const unsigned mask = __match_any_sync(0xffffffffu, g);
  const int rank_w = __popc(mask & ((1u << lane) - 1u));
  if (g >= 0 && (__ffs(mask) - 1) == lane) cnt[w][g] = __popc(mask);
  __syncthreads();
  if (g >= 0) {
    int before = 0;
    for (int i = 0; i < w; ++i) before += cnt[i][g];
    const int pos = off[(size_t)bh * (G + 1) + g] + cbase[((size_t)bh * nchunk + chunk) * G + g] +
                    before + rank_w;
    if (pos < 0 || pos >= N)
      set_error(hdr, ERR_INDEX, 2, bh, pos);
    else
      perm[(size_t)bh * N + pos] = n;
  }
}

// Means of the contiguous group-major bf16 rows of each group, balanced over
// groups of very different sizes: each group's range is cut into GM_SLICES
// equal slices, one block per (group, slice) sums its rows (fixed order,
// fp64), and k_gmean_fin adds the slices in order.  Empty groups get zero.
constexpr int GM_SLICES = 8;

template <int D>
__global__ void __launch_bounds__(256) k_gmean_part(const bf16* Xp, const int32_t* off, int N, int G,
                                                    double* part) {
  constexpr int NV = D / 32;  // values per lane (bf16 pairs: NV / 2)
  __shared__ double red[8][D];
  const int g = blockIdx.x, bh = blockIdx.y, sl = blockIdx.z;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int o0 = off[(size_t)bh * (G + 1) + g], cnt = off[(size_t)bh * (G + 1) + g + 1] - o0;
  const int lo = o0 + (int)((int64_t)cnt * sl / GM_SLICES);
  const int hi = o0 + (int)((int64_t)cnt * (sl + 1) / GM_SLICES);
  double acc[NV];
#pragma unroll
  for (int q = 0; q < NV; ++q) acc[q] = 0.0;
  for (int i0 = lo + w; i0 < hi; i0 += 8 * 4) {
    float v[4][NV];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + 8 * u;
#pragma unroll
      for (int q = 0; q < NV / 2; ++q) {
        float2 x = make_float2(0.f, 0.f);
        if (i < hi)
          x = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(Xp + ((size_t)bh * N + i) * D)[lane + 32 * q]);
        v[u][2 * q] = x.x;
        v[u][2 * q + 1] = x.y;
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int q = 0; q < NV; ++q) acc[q] += (double)v[u][q];
  }
#pragma unroll
  for (int q = 0; q < NV / 2; ++q) {
    red[w][2 * (lane + 32 * q)] = acc[2 * q];
    red[w][2 * (lane + 32 * q) + 1] = acc[2 * q + 1];
  }
  __syncthreads();
  for (int k = threadIdx.x; k < D; k += 256) {
    double t = 0.0;
#pragma unroll
    for (int q = 0; q < 8; ++q) t += red[q][k];
    part[(((size_t)bh * G + g) * GM_SLICES + sl) * D + k] = t;
  }
}

// Group means in fp32 (out) and fp64 (out64: the routing logits use them).
template <int D>
__global__ void k_gmean_fin(const double* part, const int32_t* off, int G, float* out,
                            double* out64) {
  const int g = blockIdx.x, bh = blockIdx.y, k = threadIdx.x;
  const int cnt = off[(size_t)bh * (G + 1) + g + 1] - off[(size_t)bh * (G + 1) + g];
  double t = 0.0;
#pragma unroll
  for (int sl = 0; sl < GM_SLICES; ++sl) t += part[(((size_t)bh * G + g) * GM_SLICES + sl) * D + k];
  const double mean = cnt > 0 ? t / cnt : 0.0;
  out[((size_t)bh * G + g) * D + k] = (float)mean;
  out64[((size_t)bh * G + g) * D + k] = mean;
}

// Key objective with the final centroids: sum_n ||z_n - c_{lab_n}||^2 (fp64
// partial per chunk).
template <int PP>
__global__ void __launch_bounds__(256) k_obj_z(const float* Z, int N, int G, const float* cent,
                                               const int32_t* lab, int nchunk, double* part) {
  static_assert(PP == 32, "one lane per coordinate");
  __shared__ double red[8];
  const int bh = blockIdx.y, chunk = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // warp w takes rows w, w + 8, ... of the chunk (128-byte coalesced rows);
  // each lane sums its coordinate's squared differences, then the warp adds
  double acc = 0.0;
  for (int n = chunk * CHUNK + warp; n < min(N, (chunk + 1) * CHUNK); n += 8) {
    const int g = lab[(size_t)bh * N + n];
    const float t = Z[((size_t)bh * N + n) * PP + lane] - cent[((size_t)bh * G + g) * PP + lane];
    acc += (double)(t * t);
  }
  acc = warp_sum(acc);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int i = 0; i < 8; ++i) s += red[i];
    part[((size_t)bh * 2 + 0) * (nchunk + 1) + chunk] = s;
  }
}

// Permuted copy of bf16 rows: dst[bh, i, :] = src.row(bh, perm[bh, i]).
template <int D>
__global__ void __launch_bounds__(256) k_gather_rows(TensorView src, const int32_t* perm, int N,
                                                     int BH, bf16* dst) {
  constexpr int LANES = D / 8;  // uint4 per row
  const int64_t total = (int64_t)BH * N * LANES;
  for (int64_t e = (int64_t)blockIdx.x * 256 + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * 256) {
    const int64_t rowi = e / LANES;
    const int c = (int)(e % LANES);
    const int bh = (int)(rowi / N);
    const int n = perm[rowi];
    reinterpret_cast<uint4*>(dst)[e] = reinterpret_cast<const uint4*>(src.row(bh, n))[c];
  }
}

// Transposed gather: dst[bh][c][n] = src(bh, perm[bh][n])[c] for the values in
// the group-major key order, rows of vt_ld(N) keys (the tail past N is zero).
// One block per 64 keys of one head: the 64 source rows are read whole into
// shared memory, and each of the D output rows gets its 64 keys as eight
// 16-byte stores.  Row stride of the staging tile: D + 8 elements, so that the
// column reads of the transpose spread over the banks.
template <int D>
__global__ void __launch_bounds__(256) k_gather_vt(TensorView src, const int32_t* perm, int N,
                                                   bf16* dst) {
  constexpr int KB = 64, LD = D + 8;
  __shared__ __align__(16) bf16 tile[KB * LD];
  const int bh = blockIdx.y, n0 = blockIdx.x * KB;
  const int64_t ld = vt_ld(N);
  for (int e = threadIdx.x; e < KB * (D / 8); e += 256) {
    const int r = e / (D / 8), c = e % (D / 8);
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (n0 + r < N) {
      const int n = perm[(int64_t)bh * N + n0 + r];
      v = reinterpret_cast<const uint4*>(src.row(bh, n))[c];
    }
    *reinterpret_cast<uint4*>(tile + r * LD + c * 8) = v;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < D * (KB / 8); e += 256) {
    const int c = e / (KB / 8), k8 = e % (KB / 8);
    if (n0 + k8 * 8 >= ld) continue;  // past the padded row
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint16_t lo = reinterpret_cast<const uint16_t*>(tile)[(k8 * 8 + 2 * i) * LD + c];
      const uint16_t hi = reinterpret_cast<const uint16_t*>(tile)[(k8 * 8 + 2 * i + 1) * LD + c];
      w[i] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    *reinterpret_cast<uint4*>(dst + ((int64_t)bh * D + c) * ld + n0 + k8 * 8) =
        make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// The values in the group-major key order, in the layout the attention reads.
template <int D>
void gather_values(TensorView V, const Ptrs& P, int N, int BH, int ggrid, cudaStream_t st) {
  if (P.Vt)
    spr_launch(k_gather_vt<D>, dim3((N + 63) / 64, BH), 256, 0, st, V, P.permk, N, P.Vt);
  else
    spr_launch(k_gather_rows<D>, ggrid, 256, 0, st, V, P.permk, N, BH, P.Vp);
}

// ---------------------------------------------------------------------------
// Centred nonempty K/V centroids [paperlayer App. B.2]: Ctilde rows (compacted,
// ascending group index) = c_j - mean over nonempty j of c_j.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_center(const float* Craw, const int32_t* counts, int G,
                                                int D, float* Ct, spr_head_stats* stats) {
  __shared__ int idx[MAX_GROUPS];
  __shared__ int nne;
  const int bh = blockIdx.x;
  if (threadIdx.x == 0) {
    int k = 0;
    for (int j = 0; j < G; ++j)
      if (counts[(size_t)bh * G + j] > 0) idx[k++] = j;
    nne = k;
    stats[bh].gk_nonempty = k;
  }
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += 256) {
    double s = 0.0;
    for (int t = 0; t < nne; ++t) s += Craw[((size_t)bh * G + idx[t]) * D + c];
    const float mean = nne ? (float)(s / nne) : 0.f;
    for (int t = 0; t < G; ++t)
      Ct[((size_t)bh * G + t) * D + c] =
          t < nne ? Craw[((size_t)bh * G + idx[t]) * D + c] - mean : 0.f;
  }
}

// A = Ctilde^T Ctilde (D x D) and its bf16 hi/lo split for the tensor-core
// quadratic form.  Grid (BH, (D/32)^2).
__global__ void __launch_bounds__(256) k_amat(const float* Ct, int G, int D,
                                              const spr_head_stats* stats, float* A, bf16* split,
                                              int split_rows) {
  __shared__ float As[32][33], Bs[32][33];
  const int bh = blockIdx.x, nt = D / 32;
  const int ti = blockIdx.y / nt, tj = blockIdx.y % nt;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int nne = stats[bh].gk_nonempty;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int t0 = 0; t0 < nne; t0 += 32) {
    for (int e = threadIdx.x; e < 1024; e += 256) {
      const int rr = e >> 5, c = e & 31, t = t0 + rr;
      As[rr][c] = t < nne ? Ct[((size_t)bh * G + t) * D + ti * 32 + c] : 0.f;
      Bs[rr][c] = t < nne ? Ct[((size_t)bh * G + t) * D + tj * 32 + c] : 0.f;
    }
    __syncthreads();
    for (int rr = 0; rr < 32; ++rr) {
      const float bv = Bs[rr][tx];
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[k] += As[rr][ty * 4 + k] * bv;
    }
    __syncthreads();
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int i = ti * 32 + ty * 4 + k, j = tj * 32 + tx;
    const float v = acc[k];
    A[((size_t)bh * D + i) * D + j] = v;
    const bf16 hi = __float2bfloat16_rn(v);
    const bf16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
    // split layout [BH][2][split_rows][D]; row = output column j, k-index = i
    split[(((size_t)bh * 2 + 0) * split_rows + j) * D + i] = hi;
    split[(((size_t)bh * 2 + 1) * split_rows + j) * D + i] = lo;
  }
}

// Initial query centroids: a_g = (s / rms_n) q_n at the seeded rows.
__global__ void k_init_centq(TensorView Q, int N, int G, int D, const int32_t* init,
                             const float* rms, float scale, float* centq) {
  const int bh = blockIdx.x;  // grid (BH, y): blocks of a head share its rows
  for (int e = blockIdx.y * blockDim.x + threadIdx.x; e < G * D; e += blockDim.x * gridDim.y) {
    const int g = e / D, c = e % D;
    const int n = init[(size_t)bh * G + g];
    centq[(size_t)bh * G * D + e] = scale / rms[(size_t)bh * N + n] * bf2f(Q.row(bh, n)[c]);
  }
}

// Bq_g = A a_g, beta_g = a_g . Bq_g / 2 (= ||m_g||^2 / 2), bf16 hi/lo split of Bq.
// Grid (BH, G), D threads.  Also n_g * a_g^T A a_g into part for the objective.
__global__ void k_qprep(const float* A, const float* centq, int G, int D, const int32_t* counts,
                        float* beta, bf16* split, int split_rows, double* qterm) {
  __shared__ float av[128];
  __shared__ float red[4];
  const int bh = blockIdx.x, g = blockIdx.y, i = threadIdx.x;
  av[i] = centq[((size_t)bh * G + g) * D + i];
  __syncthreads();
  float s = 0.f;
  const float* Ab = A + (size_t)bh * D * D;
  for (int j = 0; j < D; ++j) s += Ab[(size_t)j * D + i] * av[j];  // A symmetric
  const bf16 hi = __float2bfloat16_rn(s);
  const bf16 lo = __float2bfloat16_rn(s - __bfloat162float(hi));
  split[(((size_t)bh * 2 + 0) * split_rows + g) * D + i] = hi;
  split[(((size_t)bh * 2 + 1) * split_rows + g) * D + i] = lo;
  float t = warp_sum(s * av[i]);
  if ((i & 31) == 0) red[i >> 5] = t;
  __syncthreads();
  if (i == 0) {
    float q = 0.f;
    for (int w = 0; w < D / 32; ++w) q += red[w];
    beta[(size_t)bh * G + g] = 0.5f * q;
    if (qterm) qterm[(size_t)bh * G + g] = (double)counts[(size_t)bh * G + g] * (double)q;
  }
}

// ---------------------------------------------------------------------------
// Semantic partition (the comparator of [paperlayer §2 "Token Partitioning";
// §3.1 O3]): k-means on the raw key rows and, independently, on the raw query
// rows.  It runs through the query k-means kernels with A = I (so Bq_g = c_g
// and beta_g = ||c_g||^2 / 2) and every row's factor scale / rms = 1 (rms set
// to the scale): the score x . c_g - ||c_g||^2 / 2 ranks groups by distance.
// ---------------------------------------------------------------------------
__global__ void k_semantic_setup(float* A, float* rms, int D, int N, float scale) {
  const int bh = blockIdx.y;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < D * D + N; e += gridDim.x * blockDim.x) {
    if (e < D * D)
      A[(size_t)bh * D * D + e] = (e / D == e % D) ? 1.f : 0.f;
    else
      rms[(size_t)bh * N + (e - D * D)] = scale;
  }
}

// Raw-row k-means objective sum_n ||x_n - c_{lab_n}||^2, fp64 partial per
// chunk into part[bh][which][chunk] (which = 0 keys, 1 queries).
template <int D>
__global__ void __launch_bounds__(256) k_obj_rows(TensorView X, int N, int G, const float* cent,
                                                  const int32_t* lab, int nchunk, int which,
                                                  double* part) {
  __shared__ double red[8];
  const int bh = blockIdx.y, chunk = blockIdx.x;
  double acc = 0.0;
  for (int n = chunk * CHUNK + threadIdx.x; n < min(N, (chunk + 1) * CHUNK); n += 256) {
    const int g = lab[(size_t)bh * N + n];
    const bf16* x = X.row(bh, n);
    const float* c = cent + ((size_t)bh * G + g) * D;
    float s = 0.f;
    for (int k = 0; k < D; ++k) {
      const float t = bf2f(x[k]) - c[k];
      s = fmaf(t, t, s);
    }
    acc += s;
  }
  acc = warp_sum(acc);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int i = 0; i < 8; ++i) s += red[i];
    part[((size_t)bh * 2 + which) * (nchunk + 1) + chunk] = s;
  }
}

template <int D>
static cudaError_t partition_semantic_d(const spr_params& p, const Layout& L, const Ptrs& P,
                                        const TensorView& Q, const TensorView& K,
                                        const TensorView& V, cudaStream_t st) {
  const int BH = L.BH, N = p.N, nchunk = L.nchunk;
  const float scale = p.scale > 0.f ? p.scale : 1.f / sqrtf((float)D);
  const int Gm = p.Gk > p.Gq ? p.Gk : p.Gq;
  const int split_rows = bq_rows(Gm, D);
  const int ggrid = num_sms() * 8;
  cudaError_t e;
  spr_launch(k_semantic_setup, dim3(64, BH), 256, 0, st, P.Amat, P.rms, D, N, scale);
  spr_launch(k_init_idx, dim3(BH, 2), 128, 0, st, N, p.Gk, p.Gq, p.seed, p.head0, P.initk,
             P.initq);
  auto lloyd = [&](const TensorView& X, int G, const int32_t* init, float* cent,
                   int32_t* lab) -> cudaError_t {
    if (p.init != SPR_INIT_WARM)  // warm: cent holds the previous call's raw-row centroids
      spr_launch(k_init_centq, dim3(BH, 32), 256, 0, st, X, N, G, D, init, P.rms, scale, cent);
    if (cudaMemsetAsync(P.gbits, 0, L.bytes[B_GBITS], st) != cudaSuccess) return cudaGetLastError();
    LloydStep ls{};
    ls.mode = KM_QUERY;
    ls.d = D;
    ls.N = N;
    ls.G = G;
    ls.BH = BH;
    ls.split_rows = split_rows;
    ls.X = X;
    ls.bq = P.bq16;
    ls.rms = P.rms;
    ls.scale = scale;
    ls.beta = P.beta;
    ls.cent = cent;
    ls.lab = lab;
    ls.slots = P.csum;
    ls.slot_cnt = P.slotcnt;
    ls.tmask = P.tmask;
    ls.gbits = P.gbits;
    ls.hdr = P.hdr;
    ls.slots_bytes = L.bytes[B_CSUM];
    ls.slot_cnt_bytes = L.bytes[B_SLOTCNT];
    ls.tmask_bytes = L.bytes[B_TMASK];
    ls.gbits_bytes = L.bytes[B_GBITS];
    ls.A = P.Amat;  // each update also prepares the next iteration's operand
    spr_launch(k_qprep, dim3(BH, G), D, 0, st, P.Amat, cent, G, D, P.counts, P.beta, P.bq16,
               split_rows, nullptr);
    for (int it = 0; it < p.iters; ++it) {
      const cudaError_t e2 = lloyd_step(ls, st);
      if (e2 != cudaSuccess) return e2;
    }
    return label_hist(lab, N, G, nchunk, BH, P.chunk, P.hdr, st);
  };
  // K/V groups from the raw keys; the k-means centroids live in Craw until
  // the group means of the permuted keys replace them
  if ((e = lloyd(K, p.Gk, P.initk, P.Craw, P.labk)) != cudaSuccess) return e;
  spr_launch(k_chunk_scan, BH, 256, 0, st, P.chunk, nchunk, p.Gk, N, P.cbase, P.kvoff, P.counts);
  spr_launch(k_scatter, dim3(nchunk, BH), CHUNK, 0, st, P.labk, N, p.Gk, nchunk, P.cbase, P.kvoff,
             P.permk, P.hdr);
  spr_launch(k_obj_rows<D>, dim3(nchunk, BH), 256, 0, st, K, N, p.Gk, P.Craw, P.labk, nchunk, 0,
             P.part);
  spr_launch(k_gather_rows<D>, ggrid, 256, 0, st, K, P.permk, N, BH, P.Kp);
  gather_values<D>(V, P, N, BH, ggrid, st);
  spr_launch(k_gmean_part<D>, dim3(p.Gk, BH, GM_SLICES), 256, 0, st, P.Kp, P.kvoff, N, p.Gk, P.gpart);
  spr_launch(k_gmean_fin<D>, dim3(p.Gk, BH), D, 0, st, P.gpart, P.kvoff, p.Gk, P.Craw, P.craw64);
  spr_launch(k_center, BH, 256, 0, st, P.Craw, P.counts, p.Gk, D, P.Ct, P.stats);
  // query groups from the raw queries
  if ((e = lloyd(Q, p.Gq, P.initq, P.centq, P.labq)) != cudaSuccess) return e;
  spr_launch(k_chunk_scan, BH, 256, 0, st, P.chunk, nchunk, p.Gq, N, P.cbase, P.qoff, P.counts);
  spr_launch(k_scatter, dim3(nchunk, BH), CHUNK, 0, st, P.labq, N, p.Gq, nchunk, P.cbase, P.qoff,
             P.permq, P.hdr);
  spr_launch(k_obj_rows<D>, dim3(nchunk, BH), 256, 0, st, Q, N, p.Gq, P.centq, P.labq, nchunk, 1,
             P.part);
  // the objective is direct here: no n_g a_g^T A a_g term to subtract
  if (cudaMemsetAsync(P.part + (size_t)BH * 2 * (nchunk + 1), 0, (size_t)BH * p.Gq * sizeof(double),
                      st) != cudaSuccess)
    return cudaGetLastError();
  spr_launch(k_gather_rows<D>, ggrid, 256, 0, st, Q, P.permq, N, BH, P.Qp);
  spr_launch(k_gmean_part<D>, dim3(p.Gq, BH, GM_SLICES), 256, 0, st, P.Qp, P.qoff, N, p.Gq, P.gpart);
  spr_launch(k_gmean_fin<D>, dim3(p.Gq, BH), D, 0, st, P.gpart, P.qoff, p.Gq, P.qbar, P.qbar64);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Host orchestration of stage 1.
// ---------------------------------------------------------------------------
template <int D>
static cudaError_t partition_d(const spr_params& p, const Layout& L, const Ptrs& P,
                               const TensorView& Q, const TensorView& K, const TensorView& V,
                               cudaStream_t st) {
  const int BH = L.BH, N = p.N, nchunk = L.nchunk, pp = padded_p(p.p);
  const float scale = p.scale > 0.f ? p.scale : 1.f / sqrtf((float)D);
  const int sms = num_sms();
  cudaError_t e;
  // Key-response coordinates
  spr_launch(k_metric<D>, dim3(BH, (D / 32) * (D / 32)), 256, 0, st, Q, N, p.Ms, P.MK);
  if ((e = launch_eig(P.MK, BH, D, p.p, P.eval, P.evec, P.trace, st)) != cudaSuccess) return e;
  spr_launch(k_keyweights, BH, 256, 0, st, P.eval, P.evec, P.trace, D, p.p, pp, P.W);
  if ((e = launch_project(K, N, D, pp, BH, P.W, P.Z, P.zhl, P.hdr, st)) != cudaSuccess) return e;
  spr_launch(k_init_idx, dim3(BH, 2), 128, 0, st, N, p.Gk, p.Gq, p.seed, p.head0, P.initk,
             P.initq);
  if (p.init == SPR_INIT_WARM)  // the previous call's centroids, mapped (Craw still holds them)
    spr_launch(k_warm_centk, BH, 256, 0, st, P.Craw, P.W, p.Gk, D, pp, P.centk);
  else
    spr_launch(k_init_centk, BH, 256, 0, st, P.Z, N, p.Gk, pp, P.initk, P.centk);
  // Key k-means
  if (cudaMemsetAsync(P.gbits, 0, L.bytes[B_GBITS], st) != cudaSuccess) return cudaGetLastError();
  if ((e = lloyd_key_operand(P.centk, p.Gk, BH, P.bk16, P.beta, st)) != cudaSuccess) return e;
  {
    LloydStep ks{};
    ks.mode = KM_KEY;
    ks.d = D;
    ks.N = N;
    ks.G = p.Gk;
    ks.BH = BH;
    ks.Z = P.Z;
    ks.Zhl = P.zhl;
    ks.bk = P.bk16;
    ks.beta = P.beta;
    ks.cent = P.centk;
    ks.lab = P.labk;
    ks.slots = P.csum;
    ks.slot_cnt = P.slotcnt;
    ks.tmask = P.tmask;
    ks.gbits = P.gbits;
    ks.hdr = P.hdr;
    ks.slots_bytes = L.bytes[B_CSUM];
    ks.slot_cnt_bytes = L.bytes[B_SLOTCNT];
    ks.tmask_bytes = L.bytes[B_TMASK];
    ks.gbits_bytes = L.bytes[B_GBITS];
    for (int it = 0; it < p.iters; ++it)
      if ((e = lloyd_step(ks, st)) != cudaSuccess) return e;
  }
  if ((e = label_hist(P.labk, N, p.Gk, nchunk, BH, P.chunk, P.hdr, st)) != cudaSuccess) return e;
  // group-major key order of the final labels
  spr_launch(k_chunk_scan, BH, 256, 0, st, P.chunk, nchunk, p.Gk, N, P.cbase, P.kvoff, P.counts);
  spr_launch(k_scatter, dim3(nchunk, BH), CHUNK, 0, st, P.labk, N, p.Gk, nchunk, P.cbase, P.kvoff,
             P.permk, P.hdr);
spr_launch(k_obj_z<32>, dim3(nchunk, BH), 256, 0, st, P.Z, N, p.Gk, P.centk, P.labk, nchunk,
             P.part);
  // Paired K/V groups: permuted keys and values, raw-key centroids
  const int ggrid = sms * 8;
  spr_launch(k_gather_rows<D>, ggrid, 256, 0, st, K, P.permk, N, BH, P.Kp);
  gather_values<D>(V, P, N, BH, ggrid, st);
  spr_launch(k_gmean_part<D>, dim3(p.Gk, BH, GM_SLICES), 256, 0, st, P.Kp, P.kvoff, N, p.Gk, P.gpart);
  spr_launch(k_gmean_fin<D>, dim3(p.Gk, BH), D, 0, st, P.gpart, P.kvoff, p.Gk, P.Craw, P.craw64);
  // P.counts holds |K_j| now; keep a copy of key counts in kv_off differences.
  spr_launch(k_center, BH, 256, 0, st, P.Craw, P.counts, p.Gk, D, P.Ct, P.stats);
  const int split_rows = bq_rows(p.Gk > p.Gq ? p.Gk : p.Gq, D);
  spr_launch(k_amat, dim3(BH, (D / 32) * (D / 32)), 256, 0, st, P.Ct, p.Gk, D, P.stats, P.Amat, P.bq16,
                                                         split_rows);
  // Query-response RMS (tensor-core quadratic form)
  // tcgen05; its per-tile sums use the k-means partial-sum area (idle here)
  if ((e = launch_rms_tc(Q, p.B, p.H, N, D, nchunk, split_rows, P.bq16, scale, P.stats, P.rms,
                         P.un2, reinterpret_cast<double*>(P.csum), P.part, P.hdr, st)) !=
      cudaSuccess)
    return e;
  // Query k-means in the head dimension
  if (p.init != SPR_INIT_WARM)  // warm: centq keeps the previous call's head-dim centroids
    spr_launch(k_init_centq, dim3(BH, 32), 256, 0, st, Q, N, p.Gq, D, P.initq, P.rms, scale,
               P.centq);
  if (cudaMemsetAsync(P.gbits, 0, L.bytes[B_GBITS], st) != cudaSuccess) return cudaGetLastError();
  {
    LloydStep qs{};
    qs.mode = KM_QUERY;
    qs.d = D;
    qs.N = N;
    qs.G = p.Gq;
    qs.BH = BH;
    qs.split_rows = split_rows;
    qs.X = Q;
    qs.bq = P.bq16;
    qs.rms = P.rms;
    qs.scale = scale;
    qs.beta = P.beta;
    qs.cent = P.centq;
    qs.lab = P.labq;
    qs.slots = P.csum;
    qs.slot_cnt = P.slotcnt;
    qs.tmask = P.tmask;
    qs.gbits = P.gbits;
    qs.hdr = P.hdr;
    qs.slots_bytes = L.bytes[B_CSUM];
    qs.slot_cnt_bytes = L.bytes[B_SLOTCNT];
    qs.tmask_bytes = L.bytes[B_TMASK];
    qs.gbits_bytes = L.bytes[B_GBITS];
    qs.A = P.Amat;  // each update also prepares the next iteration's operand
    spr_launch(k_qprep, dim3(BH, p.Gq), D, 0, st, P.Amat, P.centq, p.Gq, D, P.counts, P.beta,
               P.bq16, split_rows, nullptr);
    for (int it = 0; it < p.iters; ++it)
      if ((e = lloyd_step(qs, st)) != cudaSuccess) return e;
  }
  if ((e = label_hist(P.labq, N, p.Gq, nchunk, BH, P.chunk, P.hdr, st)) != cudaSuccess) return e;
  // group-major query order of the final labels
  spr_launch(k_chunk_scan, BH, 256, 0, st, P.chunk, nchunk, p.Gq, N, P.cbase, P.qoff, P.counts);
  spr_launch(k_scatter, dim3(nchunk, BH), CHUNK, 0, st, P.labq, N, p.Gq, nchunk, P.cbase, P.qoff,
             P.permq, P.hdr);
  // objective terms n_g a_g^T A a_g with the final centroids (into part's tail)
  spr_launch(k_qprep, dim3(BH, p.Gq), D, 0, st, P.Amat, P.centq, p.Gq, D, P.counts, P.beta, P.bq16,
                                        split_rows, P.part + (size_t)BH * 2 * (nchunk + 1));
  // Group-major queries and raw query means
  spr_launch(k_gather_rows<D>, ggrid, 256, 0, st, Q, P.permq, N, BH, P.Qp);
  spr_launch(k_gmean_part<D>, dim3(p.Gq, BH, GM_SLICES), 256, 0, st, P.Qp, P.qoff, N, p.Gq, P.gpart);
  spr_launch(k_gmean_fin<D>, dim3(p.Gq, BH), D, 0, st, P.gpart, P.qoff, p.Gq, P.qbar, P.qbar64);
  return cudaGetLastError();
}

cudaError_t launch_partition(const spr_params& p, const Layout& L, const Ptrs& P,
                             const TensorView& Q, const TensorView& K, const TensorView& V,
                             cudaStream_t st) {
  if (p.partition == SPR_PARTITION_SEMANTIC) {
    if (p.d == 64) return partition_semantic_d<64>(p, L, P, Q, K, V, st);
    return partition_semantic_d<128>(p, L, P, Q, K, V, st);
  }
  if (p.d == 64) return partition_d<64>(p, L, P, Q, K, V, st);
  return partition_d<128>(p, L, P, Q, K, V, st);
}

}  // namespace spr
