// Leading eigenpairs of the small symmetric d x d matrices of the call: the
// sampled-query response metric M_K [paperlayer App. B.1] and the weighted
// probe-residual Gram matrix [paperlayer App. A.3].
//
// One block per matrix, fp32, following the textbook route for a few
// eigenpairs of a dense symmetric matrix (Golub & Van Loan, "Matrix
// Computations": Householder tridiagonalisation §8.3.1, bisection on Sturm
// sequence counts §8.4.1, inverse iteration §7.6.1):
//   1. A = Q T Q^T with T tridiagonal: n-2 Householder reflectors, each applied
//      to the trailing block as a symmetric rank-2 update, with the matrix held
//      in registers (two barriers per reflector).
//   2. The K largest eigenvalues of T by multisection: a group of G lanes of
//      one warp evaluates the Sturm count (number of eigenvalues below x, i.e.
//      negative pivots of T - xI = L D L^T) at G points per step.
//   3. Eigenvectors of T by inverse iteration on (T - lambda I) with partial
//      pivoting (one thread per eigenvector, factors in shared memory), then
//      orthonormalised in descending eigenvalue order by Gram-Schmidt applied
//      twice (a vector left in the span of the earlier ones, as happens for
//      eigenvalues fp32 cannot separate, is replaced by a unit vector).
//   4. Back-transformation x = H_0 H_1 ... H_{n-3} y, each warp holding its
//      vectors in registers.
// Outputs: evals[m][k] (descending, k < K), evecs[m][row][k] (stride n), and
// the trace of each matrix.
#include <float.h>

#include "spr_internal.cuh"

namespace spr {

constexpr int EIG_THREADS = 512;
constexpr int EIG_WARPS = EIG_THREADS / 32;

template <int NN>
__device__ int sturm_count(const float* a, const float* b2, float pivmin, float x) {
  int c = 0;
  float q = a[0] - x;
  if (fabsf(q) < pivmin) q = -pivmin;
  c += q < 0.f;
#pragma unroll 8
  for (int i = 1; i < NN; ++i) {
    q = (a[i] - x) - __fdividef(b2[i - 1], q);
    if (fabsf(q) < pivmin) q = -pivmin;
    c += q < 0.f;
  }
  return c;
}

// Shared-memory plan (floats), all offsets multiples of 4.
template <int NN>
struct EigSmem {
  static constexpr int LD = NN + 1;
  static constexpr int TR = NN / 32;   // rows per thread block (tridiagonalisation)
  static constexpr int TC = NN / 16;   // columns per thread block
  static constexpr int VPAD = NN + NN / 2;  // a vector with 4 floats of padding after every 8
  static constexpr int VH = 0;                           // NN x NN reflectors
  static constexpr int TV = VH + NN * NN;                // ta, tb, tb2, tau, lam (NN each)
  static constexpr int MISC = TV + 5 * NN;               // [8]
  static constexpr int VS = MISC + 8;                    // [2][VPAD] reflector vectors
  static constexpr int PS = VS + 2 * VPAD;               // [VPAD] p
  static constexpr int PART = PS + VPAD;                 // [EIG_WARPS] partial p.v
  static constexpr int Y = PART + EIG_WARPS;             // K x LD eigenvectors of T
  static constexpr int INV = 5 * NN * 32 + NN * 8;       // inverse-iteration factors of 32 vectors
  __host__ __device__ static int g_off(int K) { return Y + ((K * LD + 3) & ~3); }
  // the inverse-iteration storage is reused by the orthonormalisation (NN + 1 floats)
  __host__ __device__ static int total(int K) { return g_off(K) + INV; }
};

template <int NN>
__global__ void __launch_bounds__(EIG_THREADS, 1) k_eig_top(const float* Ain, int K, float* evals,
                                                        float* evecs, float* trace_out) {
  using S = EigSmem<NN>;
  constexpr int LD = S::LD, TR = S::TR, TC = S::TC, VPAD = S::VPAD;
  static_assert(TR % 2 == 0 && TC % 4 == 0 && 32 * TR == NN, "block shape");
  auto vpad = [](int j) { return j + (j >> 3) * 4; };
  extern __shared__ __align__(16) float esm[];
  float* Vh = esm + S::VH;  // row j = v_j (entries j+1..)
  float* ta = esm + S::TV;  // diag of T
  float* tb = ta + NN;      // off-diagonal of T (tb[i] couples i, i+1)
  float* tb2 = tb + NN;     // tb^2
  float* tau = tb2 + NN;    // reflector scales
  float* lam = tau + NN;    // eigenvalues (K)
  float* misc = esm + S::MISC;
  float* vsb = esm + S::VS;
  float* psb = esm + S::PS;
  float* part = esm + S::PART;
  float* Y = esm + S::Y;           // K x LD
  float* Gr = esm + S::g_off(K);   // inverse-iteration factors, then Gram-Schmidt scratch
  const int m = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* src = Ain + (size_t)m * NN * NN;
  if (warp == 0) {
    float t = 0.f;
    for (int i = lane; i < NN; i += 32) t += src[i * NN + i];
    t = warp_sum(t);
    if (lane == 0 && trace_out) trace_out[m] = t;
  }
  // ---- 1. tridiagonalisation --------------------------------------------
  // The matrix lives in registers: a warp holds 2R consecutive rows, its lane
  // (rb, cb) the R x C block of rows row0.. and columns c0.. (16 column blocks
  // of C).  Step k applies reflector H_k (defined by row k, equal to column k
  // by symmetry) to the trailing rows and columns: p = t A v (row partials
  // reduced over the 16 column-block lanes), K = t/2 p.v, w = p - K v, and
  // A -= v w^T + w v^T, i.e. a_ij -= v_i p_j + (p_i - 2 K v_i) v_j.  Reduced
  // rows and columns need no masking in the update: v and p are zero there.
  // The warp owning row k+1 builds the next reflector right after its own
  // update, so a step takes two barriers.  Vectors live in shared memory with
  // 4 floats of padding after every 8, so that the lanes' 16-byte reads of
  // one vector hit distinct banks.
  {
    const int rb = lane >> 4, cb = lane & 15;
    const int row0 = warp * 2 * TR + rb * TR, c0 = cb * TC;
    float a[TR][TC];
#pragma unroll
    for (int r = 0; r < TR; ++r)
#pragma unroll
      for (int c = 0; c < TC; ++c)
        a[r][c] = 0.5f * (src[(row0 + r) * NN + c0 + c] + src[(c0 + c) * NN + row0 + r]);

    // Row rk of this thread's block (rk in [0, TR); other values give row 0).
    auto select_row = [&](int rk, float* rv) {
#pragma unroll
      for (int c = 0; c < TC; ++c) {
        float x = a[0][c];
#pragma unroll
        for (int r = 1; r < TR; ++r) x = (rk == r) ? a[r][c] : x;
        rv[c] = x;
      }
    };
    // Reflector of step k from the current row k, given as rv by the 16 lanes
    // of the row block that holds it (the whole warp runs this; the other row
    // block's values are ignored).
    auto prepare = [&](int k, float* vs, const float* rv) {
      const int rk = k - row0;
      float sig = 0.f, x0 = 0.f, dg = 0.f;
#pragma unroll
      for (int c = 0; c < TC; ++c) {
        const int col = c0 + c;
        sig = (col > k + 1) ? fmaf(rv[c], rv[c], sig) : sig;
        x0 = (col == k + 1) ? rv[c] : x0;
        dg = (col == k) ? rv[c] : dg;
      }
#pragma unroll
      for (int o = 1; o < 16; o <<= 1) {
        sig += __shfl_xor_sync(0xffffffffu, sig, o);
        x0 += __shfl_xor_sync(0xffffffffu, x0, o);
        dg += __shfl_xor_sync(0xffffffffu, dg, o);
      }
      if (rk >= 0 && rk < TR) {
        float t = 0.f, alpha = x0, v0 = 0.f;
        if (sig > 0.f) {
          const float nrm = sqrtf(fmaf(x0, x0, sig));
          alpha = x0 >= 0.f ? -nrm : nrm;
          v0 = x0 - alpha;
          t = 2.f * __frcp_rn(fmaf(v0, v0, sig));
        }
#pragma unroll
        for (int c = 0; c < TC; c += 4) {
          float4 val;
          float* pv4 = &val.x;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int col = c0 + c + u;
            pv4[u] = (t == 0.f || col <= k) ? 0.f : (col == k + 1 ? v0 : rv[c + u]);
          }
          *reinterpret_cast<float4*>(vs + vpad(c0 + c)) = val;
          *reinterpret_cast<float4*>(Vh + k * NN + c0 + c) = val;
        }
        if (cb == 0) {
          tau[k] = t;
          ta[k] = dg;
          tb[k] = alpha;
        }
      }
    };

    if (warp == 0) {
      float rv[TC];
      select_row(-row0, rv);
      prepare(0, vsb, rv);
    }
    __syncthreads();
    // lane -> the row whose full product it holds after the transposed reduction
    const int rsum = (TR == 4) ? 2 * ((lane >> 3) & 1) + ((lane >> 2) & 1) : ((lane >> 3) & 1);
    const bool rwriter = (TR == 4) ? (lane & 3) == 0 : (lane & 7) == 0;
    for (int k = 0; k < NN - 2; ++k) {
      const float t = tau[k];
      const bool owner = warp == (k + 1) / (2 * TR);
      if (t == 0.f) {  // nothing to apply (uniform: every thread reads the same t)
        if (owner) {
          float rv[TC];
          select_row(k + 1 - row0, rv);
          prepare(k + 1, vsb + ((k + 1) & 1) * VPAD, rv);
        }
        __syncthreads();
        continue;
      }
      const float* vs = vsb + (k & 1) * VPAD;
      // blocks whose rows or columns are all reduced skip the arithmetic
      const bool work = row0 + TR - 1 > k && c0 + TC > k + 1;
      float vc[TC], s[TR];
#pragma unroll
      for (int c = 0; c < TC; c += 4) {
        const float4 v4 = *reinterpret_cast<const float4*>(vs + vpad(c0 + c));
        vc[c] = v4.x;
        vc[c + 1] = v4.y;
        vc[c + 2] = v4.z;
        vc[c + 3] = v4.w;
      }
#pragma unroll
      for (int r = 0; r < TR; ++r) s[r] = 0.f;
      if (work) {
#pragma unroll
        for (int r = 0; r < TR; ++r)
#pragma unroll
          for (int c = 0; c < TC; ++c) s[r] = fmaf(a[r][c], vc[c], s[r]);
      }
      // transposed reduction over the 16 column-block lanes: every lane ends
      // with the full product of row row0 + rsum
      float u;
      if constexpr (TR == 4) {
        const bool hi = lane & 8, mid = lane & 4;
        const float r0 = __shfl_xor_sync(0xffffffffu, hi ? s[0] : s[2], 8);
        const float r1 = __shfl_xor_sync(0xffffffffu, hi ? s[1] : s[3], 8);
        const float t0 = (hi ? s[2] : s[0]) + r0, t1 = (hi ? s[3] : s[1]) + r1;
        u = (mid ? t1 : t0) + __shfl_xor_sync(0xffffffffu, mid ? t0 : t1, 4);
        u += __shfl_xor_sync(0xffffffffu, u, 2);
        u += __shfl_xor_sync(0xffffffffu, u, 1);
      } else {
        const bool hi = lane & 8;
        u = (hi ? s[1] : s[0]) + __shfl_xor_sync(0xffffffffu, hi ? s[0] : s[1], 8);
        u += __shfl_xor_sync(0xffffffffu, u, 4);
        u += __shfl_xor_sync(0xffffffffu, u, 2);
        u += __shfl_xor_sync(0xffffffffu, u, 1);
      }
      {
        const int rw = row0 + rsum;
        const float prow = rw > k ? t * u : 0.f;
        float pv = 0.f;
        if (rwriter) {
          psb[vpad(rw)] = prow;
          pv = prow * vs[vpad(rw)];
        }
#pragma unroll
        for (int o = (TR == 4 ? 4 : 8); o < 32; o <<= 1) pv += __shfl_xor_sync(0xffffffffu, pv, o);
        if (lane == 0) part[warp] = pv;
      }
      __syncthreads();
      float kk = 0.f;
#pragma unroll
      for (int w = 0; w < EIG_WARPS / 4; ++w) {
        const float4 q4 = reinterpret_cast<const float4*>(part)[w];
        kk += (q4.x + q4.y) + (q4.z + q4.w);
      }
      kk *= 0.5f * t;
      float pc[TC], vi[TR], pi[TR];
#pragma unroll
      for (int c = 0; c < TC; c += 4) {
        const float4 p4 = *reinterpret_cast<const float4*>(psb + vpad(c0 + c));
        pc[c] = p4.x;
        pc[c + 1] = p4.y;
        pc[c + 2] = p4.z;
        pc[c + 3] = p4.w;
      }
#pragma unroll
      for (int r = 0; r < TR; ++r) {
        vi[r] = vs[vpad(row0 + r)];
        pi[r] = psb[vpad(row0 + r)];
      }
      if (work) {
#pragma unroll
        for (int r = 0; r < TR; ++r) {
          const float ci = fmaf(-2.f * kk, vi[r], pi[r]);
#pragma unroll
          for (int c = 0; c < TC; ++c) a[r][c] = fmaf(-vi[r], pc[c], fmaf(-ci, vc[c], a[r][c]));
        }
      }
      if (owner) {  // the next reflector from the updated row k+1
        float rv[TC];
        select_row(k + 1 - row0, rv);
        prepare(k + 1, vsb + ((k + 1) & 1) * VPAD, rv);
      }
      __syncthreads();
    }
    if (warp == (NN - 1) / (2 * TR)) {  // last diagonal entry
      float rv[TC];
      select_row(NN - 1 - row0, rv);
      prepare(NN - 1, vsb, rv);
    }
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
  // ---- 3. inverse iteration (warp 0, one lane per eigenvector) ------------
  // Factors of T - lambda I = P L U in shared memory, [i][lane] so that the
  // lanes' accesses fall in distinct banks: U's diagonal (as its reciprocal),
  // first and second superdiagonals, L's multipliers, the iterate, pivots.
  if (warp == 0) {
    float* rud = Gr;
    float* us = rud + NN * 32;
    float* uf = us + NN * 32;
    float* ml = uf + NN * 32;
    float* yv = ml + NN * 32;
    uint8_t* pv = reinterpret_cast<uint8_t*>(yv + NN * 32);
    const float tiny = 1e-7f * misc[3];
    auto clamp_rcp = [&](float u) {
      if (fabsf(u) < tiny) u = u < 0.f ? -tiny : tiny;
      return 1.f / u;
    };
    for (int e0 = 0; e0 < K; e0 += 32) {
      const int e = e0 + lane;
      if (e < K) {
        const float l = lam[e];
        // factor with partial pivoting (rows i, i+1 at step i)
        float g = ta[0] - l, h = tb[0];
        for (int i = 0; i < NN - 1; ++i) {
          const float sdn = tb[i], gn = ta[i + 1] - l, hn = (i + 1 < NN - 1) ? tb[i + 1] : 0.f;
          const int o = i * 32 + lane;
          if (fabsf(g) >= fabsf(sdn)) {
            const float mult = (g != 0.f) ? __fdividef(sdn, g) : 0.f;
            rud[o] = clamp_rcp(g);
            us[o] = h;
            uf[o] = 0.f;
            ml[o] = mult;
            pv[o] = 0;
            g = gn - mult * h;
            h = hn;
          } else {
            const float mult = __fdividef(g, sdn);
            rud[o] = clamp_rcp(sdn);
            us[o] = gn;
            uf[o] = hn;
            ml[o] = mult;
            pv[o] = 1;
            g = h - mult * gn;
            h = -mult * hn;
          }
        }
        rud[(NN - 1) * 32 + lane] = clamp_rcp(g);
        for (int i = 0; i < NN; ++i)
          yv[i * 32 + lane] = 0.5f + (float)((i * 2654435761u + e * 40503u) % 1024u) / 1024.f;
        for (int it = 0; it < 3; ++it) {
          // forward: y <- L^-1 P y, the running entry carried in a register
          float cur = yv[lane];
#pragma unroll 4
          for (int i = 0; i < NN - 1; ++i) {
            float nxt = yv[(i + 1) * 32 + lane];
            if (pv[i * 32 + lane]) {
              const float t = cur;
              cur = nxt;
              nxt = t;
            }
            nxt -= ml[i * 32 + lane] * cur;
            yv[i * 32 + lane] = cur;
            cur = nxt;
          }
          // back: y <- U^-1 y, with y_{i+1}, y_{i+2} carried in registers
          // Near-singular pivots make the solution grow step by step; when an
          // entry passes 1e15 the whole system (solved entries and the
          // right-hand side still to be used) is scaled by 1e-15 -- the
          // direction is all that matters -- so y^2 sums stay finite.
          auto shrink = [&]() {
            for (int j = 0; j < NN; ++j) yv[j * 32 + lane] *= 1e-15f;
          };
          yv[(NN - 1) * 32 + lane] = cur;
          float y2 = cur * rud[(NN - 1) * 32 + lane];
          if (fabsf(y2) > 1e15f) {
            shrink();
            y2 *= 1e-15f;
          }
          yv[(NN - 1) * 32 + lane] = y2;
          float y1 = (yv[(NN - 2) * 32 + lane] - us[(NN - 2) * 32 + lane] * y2) *
                     rud[(NN - 2) * 32 + lane];
          if (fabsf(y1) > 1e15f) {
            shrink();
            y1 *= 1e-15f;
            y2 *= 1e-15f;
          }
          yv[(NN - 2) * 32 + lane] = y1;
#pragma unroll 4
          for (int i = NN - 3; i >= 0; --i) {
            const int o = i * 32 + lane;
            float yi = (yv[o] - us[o] * y1 - uf[o] * y2) * rud[o];
            if (fabsf(yi) > 1e15f) {
              shrink();
              yi *= 1e-15f;
              y1 *= 1e-15f;
              y2 *= 1e-15f;
            }
            yv[o] = yi;
            y2 = y1;
            y1 = yi;
          }
          float nrm = 0.f;
          for (int i = 0; i < NN; ++i) nrm += yv[i * 32 + lane] * yv[i * 32 + lane];
          const float inv = nrm > 0.f ? rsqrtf(nrm) : 0.f;
          for (int i = 0; i < NN; ++i) yv[i * 32 + lane] *= inv;
        }
        for (int i = 0; i < NN; ++i) Y[e * LD + i] = yv[i * 32 + lane];
      }
      __syncwarp();
    }
  }
  __syncthreads();
  // Orthonormalise in descending eigenvalue order by classical Gram-Schmidt
  // applied twice per vector (Giraud, Langou & Rozloznik 2005: two passes
  // give orthogonality to working precision).  Inverse iteration on
  // eigenvalues that fp32 cannot separate (a cluster at the noise floor)
  // returns nearly parallel vectors; a vector that keeps less than 1/8 of
  // its length after the two passes lies in the span of the earlier ones and
  // is replaced by the first unit vector e_j (j = a, a+1, ... mod n) that
  // keeps more, so the basis stays orthonormal and finite.
  {
    float* dots = Gr;  // [NN], reuses the inverse-iteration storage
    float* nrm_s = Gr + NN;
    constexpr int TPE = EIG_THREADS / NN;  // threads per vector entry
    const int ent = tid / TPE, sub = tid % TPE;
    for (int a = 0; a < K; ++a) {
      for (int attempt = 0; attempt <= NN; ++attempt) {
        if (attempt > 0) {  // replacement: e_j for the attempt-th candidate j
          const int j = (a + attempt - 1) % NN;
          for (int i = tid; i < NN; i += EIG_THREADS) Y[a * LD + i] = i == j ? 1.f : 0.f;
          __syncthreads();
        }
        for (int pass = 0; pass < 2; ++pass) {
          for (int bq = warp; bq < a; bq += EIG_WARPS) {  // dots with the earlier vectors
            float d = 0.f;
            for (int i = lane; i < NN; i += 32) d = fmaf(Y[a * LD + i], Y[bq * LD + i], d);
            d = warp_sum(d);
            if (lane == 0) dots[bq] = d;
          }
          __syncthreads();
          float sacc = 0.f;  // sum_b dots[b] Y[b][ent], split over the TPE threads
          for (int bq = sub; bq < a; bq += TPE) sacc = fmaf(dots[bq], Y[bq * LD + ent], sacc);
#pragma unroll
          for (int o = 1; o < TPE; o <<= 1) sacc += __shfl_xor_sync(0xffffffffu, sacc, o);
          __syncthreads();  // every dot read before Y[a] changes
          if (sub == 0) Y[a * LD + ent] -= sacc;
          __syncthreads();
        }
        if (warp == 0) {
          float q = 0.f;
          for (int i = lane; i < NN; i += 32) q = fmaf(Y[a * LD + i], Y[a * LD + i], q);
          q = warp_sum(q);
          if (lane == 0) *nrm_s = q;
        }
        __syncthreads();
        const float q = *nrm_s;
        // the iterate and the replacements enter with unit length
        if (isfinite(q) && q > 1.f / 64.f) {
          const float inv = rsqrtf(q);
          for (int i = tid; i < NN; i += EIG_THREADS) Y[a * LD + i] *= inv;
          __syncthreads();
          break;
        }
        __syncthreads();
      }
    }
  }
  __syncthreads();
  // ---- 4. back-transformation: each warp takes two vectors at a time and
  // keeps them in registers (lane holds rows lane + 32 m) ------------------
  {
    constexpr int RM = NN / 32;
    for (int kq0 = warp; kq0 < K; kq0 += 2 * EIG_WARPS) {
      const int kq1 = kq0 + EIG_WARPS;
      const bool two = kq1 < K;
      float y0[RM], y1[RM];
#pragma unroll
      for (int r = 0; r < RM; ++r) {
        y0[r] = Y[kq0 * LD + lane + 32 * r];
        y1[r] = two ? Y[kq1 * LD + lane + 32 * r] : 0.f;
      }
      for (int j = NN - 3; j >= 0; --j) {
        const float t = tau[j];
        if (t == 0.f) continue;
        const float* v = Vh + j * NN;  // zero at rows <= j
        float vr[RM], d0 = 0.f, d1 = 0.f;
#pragma unroll
        for (int r = 0; r < RM; ++r) {
          vr[r] = v[lane + 32 * r];
          d0 = fmaf(vr[r], y0[r], d0);
          d1 = fmaf(vr[r], y1[r], d1);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          d0 += __shfl_xor_sync(0xffffffffu, d0, o);
          d1 += __shfl_xor_sync(0xffffffffu, d1, o);
        }
        d0 *= t;
        d1 *= t;
#pragma unroll
        for (int r = 0; r < RM; ++r) {
          y0[r] = fmaf(-d0, vr[r], y0[r]);
          y1[r] = fmaf(-d1, vr[r], y1[r]);
        }
      }
#pragma unroll
      for (int r = 0; r < RM; ++r) {
        Y[kq0 * LD + lane + 32 * r] = y0[r];
        if (two) Y[kq1 * LD + lane + 32 * r] = y1[r];
      }
    }
  }
  __syncthreads();
  for (int e = tid; e < K; e += EIG_THREADS) evals[(size_t)m * NN + e] = lam[e];
  for (int e = tid; e < NN * NN; e += EIG_THREADS) {  // columns past K are zero
    const int row = e / NN, kq = e % NN;
    evecs[(size_t)m * NN * NN + e] = kq < K ? Y[kq * LD + row] : 0.f;
  }
}

template <int NN>
static cudaError_t eig_n(const float* A, int count, int K, float* ev, float* evec, float* trace,
                         cudaStream_t st) {
  const size_t smem = (size_t)EigSmem<NN>::total(K) * 4;
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
