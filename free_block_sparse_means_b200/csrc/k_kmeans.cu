// One Lloyd iteration of the partition's two k-means [paperlayer App. B.1,
// B.2] on a chunk of CHUNK rows, fused into one kernel:
//   1. assignment on the tensor cores (tcgen05.mma kind::f16, bf16 operands
//      in K-major 128-byte-swizzled shared memory, fp32 accumulator of 128
//      rows x NC groups in TMEM), tiles of 128 rows double-buffered with
//      cp.async; one thread per row reads its scores back for the argmax;
//        query rows: score_g = (s / rms_n) q . Bq_g - beta_g, q exact in bf16,
//                    Bq_g split into bf16 hi + lo (two products);
//        key rows:   score_g = 2 z . c_g - ||c_g||^2, z and c_g both split
//                    into hi + lo (three products: hh, hl, lh);
//      label = argmax (ties to the lowest g), i.e. the nearest centroid;
//   2. the chunk's label histogram, its exclusive scan, and a stable
//      chunk-local sort of the rows by label;
//   3. segmented partial sums of the update rows ((s / rms_n) q or z) over
//      32-position segments of the sorted order, one slot per (group,
//      segment) at g + segment, for the fixed-order reducer k_chunk_reduce.
// The chunk's labels, histogram and local offsets also serve the final
// stable scatter into group-major order.
#include <float.h>

#include "spr_internal.cuh"
#include "tc_sm100.cuh"

namespace spr {

constexpr int KM_THREADS = 256;
constexpr int KM_TILE = 128;                 // rows per sub-tile (the UMMA M)
constexpr uint32_t KM_BOX = KM_TILE * 128;   // one 64-column SW128 box of a tile: 16 KB
constexpr uint64_t KM_WAIT_NS = 2000000000ull;

// Shared-memory plan (bytes from a 1024-aligned base):
//   Bh, Bl     centroid operand, K-major SW128, nbox boxes of NC rows x 128 B
//   A region   QUERY: two tiles of nbox boxes; KEY: two raw fp32 tiles, then
//              the hi / lo bf16 tiles (one box each); reused afterwards by
//              the sort arrays and the segment staging
//   betas[MAX_GROUPS], labs[CHUNK], mbarrier, TMEM base, abort flag
struct KmPlan {
  int nbox, NC;
  size_t b_off, a_off, a_size, tail_off, total;
};
__host__ __device__ inline KmPlan km_plan(int mode, int DK, int SW, int G) {
  KmPlan p;
  p.nbox = DK > 64 ? DK / 64 : 1;
  p.NC = ((G + 31) / 32) * 32;
  const size_t sb = (size_t)p.nbox * p.NC * 128;
  p.b_off = 0;
  p.a_off = 2 * sb;
  const size_t tiles = mode == KM_KEY ? 2 * (size_t)KM_TILE * SW * 4 + 2 * (size_t)KM_BOX
                                      : 2 * (size_t)p.nbox * KM_BOX;
  const size_t rb = mode == KM_KEY ? (size_t)SW * 4 : (size_t)SW * 2;
  const size_t stg = (size_t)(KM_THREADS / 32) * (mode == KM_KEY ? 32 : 16) * rb;
  const size_t sortb = (32 * (size_t)G + CHUNK + MAX_GROUPS + 32) * 4 + stg;
  p.a_size = ((tiles > sortb ? tiles : sortb) + 1023) & ~(size_t)1023;
  p.tail_off = p.a_off + p.a_size;
  p.total = p.tail_off + (MAX_GROUPS + CHUNK) * 4 + 64;
  return p;
}

// 16-byte chunk c (K-major: K elements 8c .. 8c + 7) of row r in a tile or
// operand of nbox 64-column SW128 boxes of `rows` rows.
__device__ __forceinline__ uint32_t sw_off(int r, int c, int rows) {
  return (uint32_t)((c >> 3) * rows * 128 + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ uint4 split8(const float* v, bool lo) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bf16 h0 = __float2bfloat16_rn(v[2 * i]), h1 = __float2bfloat16_rn(v[2 * i + 1]);
    w[i] = lo ? pack_bf16(v[2 * i] - __bfloat162float(h0), v[2 * i + 1] - __bfloat162float(h1))
              : pack_bf16(__bfloat162float(h0), __bfloat162float(h1));
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

template <int MODE, int DK, int SW>
__global__ void __launch_bounds__(KM_THREADS, 1) k_kmeans_step(KmArgs a) {
  constexpr int KS = DK / 16;  // UMMA k-steps
  constexpr int NCH = DK / 8;  // 16-byte chunks per A / B row
  extern __shared__ uint8_t km_raw[];
  uint8_t* km = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(km_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  const int G = a.G;
  const KmPlan pl = km_plan(MODE, DK, SW, G);
  const int NC = pl.NC;
  uint8_t* Bh = km + pl.b_off;
  uint8_t* Bl = Bh + (size_t)pl.nbox * NC * 128;
  uint8_t* Ab = km + pl.a_off;
  float* betas = reinterpret_cast<float*>(km + pl.tail_off);
  int* labs = reinterpret_cast<int*>(betas + MAX_GROUPS);
  uint64_t* mbar = reinterpret_cast<uint64_t*>(labs + CHUNK);
  uint32_t* tmem_s = reinterpret_cast<uint32_t*>(mbar + 1);
  volatile int* abort_s = reinterpret_cast<volatile int*>(tmem_s + 1);
  const int bh = blockIdx.y, chunk = blockIdx.x, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int N = a.N, n0 = chunk * CHUNK, rows = min(CHUNK, N - n0);
  const uint32_t tcols = NC <= 32 ? 32 : NC <= 64 ? 64 : NC <= 128 ? 128 : 256;

  // ---- centroid operand (K-major SW128, bf16 hi and lo) -------------------
  if (MODE == KM_QUERY) {
    const bf16* bsrc = a.bsplit + (size_t)bh * 2 * a.split_rows * DK;
    for (int e = tid; e < NC * NCH; e += KM_THREADS) {
      const int r = e / NCH, c = e % NCH;
      uint4 hi = make_uint4(0, 0, 0, 0), lo = hi;
      if (r < G) {
        hi = reinterpret_cast<const uint4*>(bsrc + (size_t)r * DK)[c];
        lo = reinterpret_cast<const uint4*>(bsrc + ((size_t)a.split_rows + r) * DK)[c];
      }
      *reinterpret_cast<uint4*>(Bh + sw_off(r, c, NC)) = hi;
      *reinterpret_cast<uint4*>(Bl + sw_off(r, c, NC)) = lo;
    }
    for (int g = tid; g < MAX_GROUPS; g += KM_THREADS)
      betas[g] = g < G ? a.beta[(size_t)bh * G + g] : 0.f;
  } else {
    const float* cs = a.cent + (size_t)bh * G * SW;
    for (int e = tid; e < NC * NCH; e += KM_THREADS) {
      const int r = e / NCH, c = e % NCH;
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = (r < G && 8 * c + i < SW) ? cs[r * SW + 8 * c + i] : 0.f;
      *reinterpret_cast<uint4*>(Bh + sw_off(r, c, NC)) = split8(v, false);
      *reinterpret_cast<uint4*>(Bl + sw_off(r, c, NC)) = split8(v, true);
    }
    for (int g = tid; g < MAX_GROUPS; g += KM_THREADS) {
      float s = 0.f;
      if (g < G)
        for (int c = 0; c < SW; ++c) s = fmaf(cs[g * SW + c], cs[g * SW + c], s);
      betas[g] = s;
    }
  }
  if (tid == 0) {
    tc::mbar_init(mbar, 1);
    *abort_s = 0;
    tc::fence_barrier_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(tmem_s, tcols);
    tc::tmem_relinquish();
  }
  tc::fence_proxy_async_smem();
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = *tmem_s;

  // ---- assignment on the tensor cores ------------------------------------
  // QUERY: A tiles [2][nbox boxes] loaded with cp.async into the SW128 layout.
  // KEY:   raw fp32 tiles [2][KM_TILE][SW] with cp.async, converted into the
  //        hi / lo bf16 tiles (one box each) before each use.
  uint8_t* raw = Ab;
  uint8_t* Akey = Ab + (MODE == KM_KEY ? 2 * (size_t)KM_TILE * SW * 4 : 0);
  auto load_tile = [&](int sub, int buf) {
    const int r0 = n0 + sub * KM_TILE;
    if (MODE == KM_QUERY) {
      uint8_t* dst = Ab + (size_t)buf * pl.nbox * KM_BOX;
      for (int e = tid; e < KM_TILE * NCH; e += KM_THREADS) {
        const int r = e / NCH, c = e % NCH, n = r0 + r;
        cp_async16(dst + sw_off(r, c, KM_TILE), a.Q.row(bh, n < N ? n : 0) + c * 8, n < N ? 16 : 0);
      }
    } else {
      uint8_t* dst = raw + (size_t)buf * KM_TILE * SW * 4;
      for (int e = tid; e < KM_TILE * (SW / 4); e += KM_THREADS) {
        const int r = e / (SW / 4), c = e % (SW / 4), n = r0 + r;
        cp_async16(dst + (r * SW + c * 4) * 4, a.Z + ((size_t)bh * N + (n < N ? n : 0)) * SW + c * 4,
                   n < N ? 16 : 0);
      }
    }
    cp_async_commit();
  };
  const uint32_t idesc = tc::idesc_bf16(KM_TILE, NC, 0);
  const uint32_t bh_addr = smem_u32(Bh), bl_addr = smem_u32(Bl);
  const int nsub = (rows + KM_TILE - 1) / KM_TILE;
  uint32_t phase = 0;
  load_tile(0, 0);
  for (int sub = 0; sub < nsub; ++sub) {
    if (sub + 1 < nsub) {
      load_tile(sub + 1, (sub + 1) & 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    uint32_t ah_addr, al_addr = 0;
    if (MODE == KM_QUERY) {
      ah_addr = smem_u32(Ab + (size_t)(sub & 1) * pl.nbox * KM_BOX);
    } else {
      __syncthreads();  // raw tile complete
      const float* src = reinterpret_cast<const float*>(raw + (size_t)(sub & 1) * KM_TILE * SW * 4);
      for (int e = tid; e < KM_TILE * NCH; e += KM_THREADS) {
        const int r = e / NCH, c = e % NCH;
        float v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = 8 * c + i < SW ? src[r * SW + 8 * c + i] : 0.f;
        *reinterpret_cast<uint4*>(Akey + sw_off(r, c, KM_TILE)) = split8(v, false);
        *reinterpret_cast<uint4*>(Akey + KM_BOX + sw_off(r, c, KM_TILE)) = split8(v, true);
      }
      ah_addr = smem_u32(Akey);
      al_addr = smem_u32(Akey + KM_BOX);
    }
    tc::fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {  // D = A Bh^T + A Bl^T (+ Al Bh^T), fp32 in TMEM
      tc::tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const uint32_t ao = (ks >> 2) * KM_BOX + (ks & 3) * 32;
        const uint32_t bo = (ks >> 2) * NC * 128 + (ks & 3) * 32;
        tc::mma_ss(tbase, tc::smem_desc_sw128(ah_addr + ao, 16, 1024),
                   tc::smem_desc_sw128(bh_addr + bo, 16, 1024), idesc, ks > 0);
        tc::mma_ss(tbase, tc::smem_desc_sw128(ah_addr + ao, 16, 1024),
                   tc::smem_desc_sw128(bl_addr + bo, 16, 1024), idesc, 1);
        if (MODE == KM_KEY)
          tc::mma_ss(tbase, tc::smem_desc_sw128(al_addr + ao, 16, 1024),
                     tc::smem_desc_sw128(bh_addr + bo, 16, 1024), idesc, 1);
      }
      tc::mma_commit(mbar);
    }
    if (warp < 4) {  // one tile row per thread: scores from TMEM, argmax
      bool ok = tc::mbar_wait(mbar, phase, abort_s, KM_WAIT_NS);
      __syncwarp();
      ok = __all_sync(0xffffffffu, ok);
      tc::tc_fence_after();
      const int lr = sub * KM_TILE + warp * 32 + lane, n = n0 + lr;
      int arg = -1;
      if (ok) {
        float alpha = 2.f;
        if (MODE == KM_QUERY) alpha = n < N ? a.scale / a.rms[(size_t)bh * N + n] : 0.f;
        float best = -FLT_MAX;
        arg = 0;
        for (int c0 = 0; c0 < NC; c0 += 32) {
          uint32_t v[32];
          __syncwarp();
          tc::tmem_ld32(tbase + ((uint32_t)(warp * 32) << 16) + c0, v);
          tc::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int g = c0 + j;
            const float sc = alpha * __uint_as_float(v[j]) - betas[g];
            if (g < G && sc > best) {
              best = sc;
              arg = g;
            }
          }
        }
      }
      labs[lr] = n < N ? arg : -1;
      if (n < N && arg >= 0) a.lab[(size_t)bh * N + n] = arg;
    }
    phase ^= 1;
    tc::tc_fence_before();
    __syncthreads();  // TMEM read and tile buffers free
  }
  if (*abort_s) {
    if (tid == 0) {
      set_error(a.hdr, ERR_TIMEOUT, 7, bh, chunk);
      tc::mbar_wait_bounded(mbar, phase ^ 1, KM_WAIT_NS);  // the last commit, if still pending
    }
    __syncthreads();
  }
  tc::tc_fence_after();
  if (warp == 0) {
    __syncwarp();
    tc::tmem_dealloc(tbase, tcols);
  }

  // ---- histogram, scan, stable chunk-local sort (A region reused) --------
  int* cnt = reinterpret_cast<int*>(Ab);  // [32][G]: per 32-row group and label
  int* srt = cnt + 32 * G;                // [CHUNK]: local row | label << 10
  int* lof = srt + CHUNK;                 // [MAX_GROUPS]: histogram, then offsets
  int* wsum = lof + MAX_GROUPS;           // [32]
  for (int e = tid; e < 32 * G; e += KM_THREADS) cnt[e] = 0;
  for (int e = tid; e < CHUNK; e += KM_THREADS) srt[e] = -1;
  for (int e = tid; e < MAX_GROUPS; e += KM_THREADS) lof[e] = 0;
  __syncthreads();
  constexpr int NP = CHUNK / KM_THREADS;  // rows per thread
  int gl[NP], rk[NP];
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int row = p * KM_THREADS + tid;
    int g = row < rows ? labs[row] : -1;
    if (g >= G || g < -1) {
      set_error(a.hdr, ERR_INDEX, 5, bh, n0 + row);
      g = -1;
    }
    gl[p] = g;
    if (g >= 0) atomicAdd(&lof[g], 1);
  }
  __syncthreads();
  {  // exclusive scan of the histogram (G <= 256 = KM_THREADS)
    const int v = tid < G ? lof[tid] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int x = lane < KM_THREADS / 32 ? wsum[lane] : 0;
      int xi = x;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, xi, o);
        if (lane >= o) xi += t;
      }
      if (lane < KM_THREADS / 32) wsum[lane] = xi - x;
    }
    __syncthreads();
    if (tid < G) {
      const int lo = wsum[warp] + incl - v;
      lof[tid] = lo;
      const size_t cidx = ((size_t)bh * a.nchunk + chunk) * G + tid;
      a.loff[cidx] = lo;
      a.chunk_cnt[cidx] = v;
    }
  }
#pragma unroll
  for (int p = 0; p < NP; ++p) {  // ranks within each 32-row group
    const unsigned mask = __match_any_sync(0xffffffffu, gl[p]);
    rk[p] = __popc(mask & ((1u << lane) - 1u));
    if (gl[p] >= 0 && (__ffs(mask) - 1) == lane) cnt[(p * (KM_THREADS / 32) + warp) * G + gl[p]] = __popc(mask);
  }
  __syncthreads();
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int g = gl[p];
    if (g < 0) continue;
    const int grp = p * (KM_THREADS / 32) + warp;
    int before = 0;
    for (int i = 0; i < grp; ++i) before += cnt[i * G + g];
    const int pos = lof[g] + before + rk[p];
    if (pos < 0 || pos >= rows)
      set_error(a.hdr, ERR_INDEX, 6, bh, pos);
    else
      srt[pos] = (p * KM_THREADS + tid) | (g << 10);
  }
  __syncthreads();

  // ---- segmented partial sums over 32-position segments ------------------
  constexpr int NV = (MODE == KM_KEY) ? (SW + 31) / 32 : SW / 32;  // values per lane
  float* slot0 = a.part + ((size_t)bh * a.nchunk + chunk) * (size_t)(G + CSUM_SLOTS) * SW;
  const float* zbase = MODE == KM_KEY ? a.Z + (size_t)bh * N * SW : nullptr;
  const bf16* qbase = MODE == KM_QUERY ? a.Q.row(bh, 0) : nullptr;
  const int64_t qsn = a.Q.sn;
  // rows of a segment are staged in shared memory with cp.async (every row of
  // a batch in flight at once), KM_STAGE rows per batch and warp
  constexpr int RB = (MODE == KM_KEY) ? SW * 4 : SW * 2;  // bytes per update row
  constexpr int KM_STAGE = (MODE == KM_KEY) ? 32 : 16;
  uint8_t* stage = reinterpret_cast<uint8_t*>(wsum + 32) + (size_t)warp * KM_STAGE * RB;
  for (int seg = warp; seg < CHUNK / 32; seg += KM_THREADS / 32) {
    const int p0 = 32 * seg, p1 = min(p0 + 32, rows);
    if (p0 >= p1) break;
    const int e_l = p0 + lane < p1 ? srt[p0 + lane] : -1;
    const int g_l = e_l >= 0 ? e_l >> 10 : -1;
    const int row_l = n0 + (e_l >= 0 ? (e_l & 1023) : 0);
    float f_l = 1.f;
    if (MODE == KM_QUERY && e_l >= 0) f_l = a.scale / a.rms[(size_t)bh * N + row_l];
    float acc[NV];
#pragma unroll
    for (int q = 0; q < NV; ++q) acc[q] = 0.f;
    int cur = __shfl_sync(0xffffffffu, g_l, 0);
    auto flush = [&](int gg) {
      if (gg < 0) return;
      float* dst = slot0 + (size_t)(gg + seg) * SW;
      if (MODE == KM_KEY) {
#pragma unroll
        for (int q = 0; q < NV; ++q)
          if (lane + 32 * q < SW) dst[lane + 32 * q] = acc[q];
      } else {
#pragma unroll
        for (int q = 0; q < NV / 2; ++q)
          reinterpret_cast<float2*>(dst)[lane + 32 * q] = make_float2(acc[2 * q], acc[2 * q + 1]);
      }
    };
    for (int b0 = 0; b0 < 32; b0 += KM_STAGE) {
      // stage: 16-byte pieces, lane-strided over the batch's rows (the trip
      // count is the same for every lane)
      constexpr int PR = RB / 16;  // pieces per row
      static_assert((KM_STAGE * PR) % 32 == 0, "uniform staging loop");
      __syncwarp();  // the previous batch is consumed
#pragma unroll
      for (int e = lane; e < KM_STAGE * PR; e += 32) {
        const int u = e / PR, c = e % PR;
        const int row = __shfl_sync(0xffffffffu, row_l, b0 + u);
        const bool ok = __shfl_sync(0xffffffffu, g_l, b0 + u) >= 0;
        const uint8_t* src = (MODE == KM_KEY)
                                 ? reinterpret_cast<const uint8_t*>(zbase + (size_t)row * SW)
                                 : reinterpret_cast<const uint8_t*>(qbase + row * qsn);
        if (ok) cp_async16(stage + u * RB + c * 16, src + c * 16, 16);
      }
      cp_async_commit();
      cp_async_wait<0>();
      __syncwarp();
#pragma unroll
      for (int u = 0; u < KM_STAGE; ++u) {
        const int gu = __shfl_sync(0xffffffffu, g_l, b0 + u);
        const float fu = __shfl_sync(0xffffffffu, f_l, b0 + u);
        if (gu < 0) continue;
        if (gu != cur) {
          flush(cur);
#pragma unroll
          for (int q = 0; q < NV; ++q) acc[q] = 0.f;
          cur = gu;
        }
        if (MODE == KM_KEY) {
          const float* x = reinterpret_cast<const float*>(stage + u * RB);
#pragma unroll
          for (int q = 0; q < NV; ++q)
            if (lane + 32 * q < SW) acc[q] = fmaf(fu, x[lane + 32 * q], acc[q]);
        } else {
          const __nv_bfloat162* x = reinterpret_cast<const __nv_bfloat162*>(stage + u * RB);
#pragma unroll
          for (int q = 0; q < NV / 2; ++q) {
            const float2 xv = __bfloat1622float2(x[lane + 32 * q]);
            acc[2 * q] = fmaf(fu, xv.x, acc[2 * q]);
            acc[2 * q + 1] = fmaf(fu, xv.y, acc[2 * q + 1]);
          }
        }
      }
    }
    flush(cur);
  }
}

// Key-response coordinates Z = K W on the tensor cores [paperlayer App.
// B.1]: K rows exact in bf16, W (d x pp, fp32) split into bf16 hi + lo (two
// products), fp32 accumulation in TMEM.  One 128-row tile per block:
// A = the tile (K-major SW128, cp.async), B = W^T hi / lo ([n][k] rows, n
// padded to NP >= 32 with zeros), D = 128 x NP in TMEM; four warps write one
// Z row (pp floats) per thread.
template <int D, int PP>
__global__ void __launch_bounds__(KM_THREADS, 1) k_project_tc(TensorView K, int N, const float* W, float* Z,
                                                              Header* hdr) {
  constexpr int NP = PP < 32 ? 32 : PP;  // UMMA N (and TMEM columns)
  constexpr int NCH = D / 8, NBOX = D / 64;
  extern __shared__ uint8_t pr_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(pr_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint8_t* At = sm;                              // NBOX boxes of 128 rows
  uint8_t* Bh = At + NBOX * KM_BOX;              // NBOX boxes of NP rows
  uint8_t* Bl = Bh + (size_t)NBOX * NP * 128;
  uint64_t* mbar = reinterpret_cast<uint64_t*>(Bl + (size_t)NBOX * NP * 128);
  uint32_t* tmem_s = reinterpret_cast<uint32_t*>(mbar + 1);
  volatile int* abort_s = reinterpret_cast<volatile int*>(tmem_s + 1);
  const int bh = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r0 = blockIdx.x * KM_TILE;
  for (int e = tid; e < KM_TILE * NCH; e += KM_THREADS) {
    const int r = e / NCH, c = e % NCH, n = r0 + r;
    cp_async16(At + sw_off(r, c, KM_TILE), K.row(bh, n < N ? n : 0) + c * 8, n < N ? 16 : 0);
  }
  cp_async_commit();
  const float* wb = W + (size_t)bh * D * PP;
  for (int e = tid; e < NP * NCH; e += KM_THREADS) {
    const int r = e / NCH, c = e % NCH;  // r = output column, c = 8 of the d inputs
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = r < PP ? wb[(8 * c + i) * PP + r] : 0.f;
    *reinterpret_cast<uint4*>(Bh + sw_off(r, c, NP)) = split8(v, false);
    *reinterpret_cast<uint4*>(Bl + sw_off(r, c, NP)) = split8(v, true);
  }
  if (tid == 0) {
    tc::mbar_init(mbar, 1);
    *abort_s = 0;
    tc::fence_barrier_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(tmem_s, NP);
    tc::tmem_relinquish();
  }
  cp_async_wait<0>();
  tc::fence_proxy_async_smem();
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = *tmem_s;
  if (tid == 0) {
    const uint32_t idesc = tc::idesc_bf16(KM_TILE, NP, 0);
    const uint32_t a_addr = smem_u32(At), bh_addr = smem_u32(Bh), bl_addr = smem_u32(Bl);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const uint32_t ao = (ks >> 2) * KM_BOX + (ks & 3) * 32;
      const uint32_t bo = (ks >> 2) * NP * 128 + (ks & 3) * 32;
      tc::mma_ss(tbase, tc::smem_desc_sw128(a_addr + ao, 16, 1024),
                 tc::smem_desc_sw128(bh_addr + bo, 16, 1024), idesc, ks > 0);
      tc::mma_ss(tbase, tc::smem_desc_sw128(a_addr + ao, 16, 1024),
                 tc::smem_desc_sw128(bl_addr + bo, 16, 1024), idesc, 1);
    }
    tc::mma_commit(mbar);
  }
  if (warp < 4) {
    bool ok = tc::mbar_wait(mbar, 0, abort_s, KM_WAIT_NS);
    __syncwarp();
    ok = __all_sync(0xffffffffu, ok);
    tc::tc_fence_after();
    const int n = r0 + warp * 32 + lane;
    if (ok) {
#pragma unroll
      for (int c0 = 0; c0 < NP; c0 += 32) {
        uint32_t v[32];
        __syncwarp();
        tc::tmem_ld32(tbase + ((uint32_t)(warp * 32) << 16) + c0, v);
        tc::tmem_wait_ld();
        if (n < N) {
          float4* dst = reinterpret_cast<float4*>(Z + ((size_t)bh * N + n) * PP + c0);
#pragma unroll
          for (int q = 0; q < (PP < 32 ? PP : 32) / 4; ++q)
            dst[q] = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                 __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
        }
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (*abort_s) {
    if (tid == 0) {
      set_error(hdr, ERR_TIMEOUT, 8, bh, blockIdx.x);
      tc::mbar_wait_bounded(mbar, 0, KM_WAIT_NS);
    }
    __syncthreads();
  }
  tc::tc_fence_after();
  if (warp == 0) {
    __syncwarp();
    tc::tmem_dealloc(tbase, NP);
  }
}

template <int D, int PP>
static cudaError_t proj_launch(const TensorView& K, int N, int BH, const float* W, float* Z,
                               Header* hdr, cudaStream_t st) {
  constexpr int NP = PP < 32 ? 32 : PP;
  const size_t sm = 1024 + (size_t)(D / 64) * (KM_BOX + 2 * NP * 128) + 64;
  cudaError_t e = cudaFuncSetAttribute(k_project_tc<D, PP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sm);
  if (e != cudaSuccess) return e;
  spr_launch(k_project_tc<D, PP>, dim3((N + KM_TILE - 1) / KM_TILE, BH), KM_THREADS, sm, st, K, N, W,
             Z, hdr);
  return cudaGetLastError();
}

cudaError_t launch_project(const TensorView& K, int N, int D, int PP, int BH, const float* W,
                           float* Z, Header* hdr, cudaStream_t st) {
#define PJ(DV, PV) return proj_launch<DV, PV>(K, N, BH, W, Z, hdr, st)
  if (D == 128) {
    if (PP == 8) PJ(128, 8);
    if (PP == 16) PJ(128, 16);
    if (PP == 32) PJ(128, 32);
    if (PP == 64) PJ(128, 64);
  } else if (D == 64) {
    if (PP == 8) PJ(64, 8);
    if (PP == 16) PJ(64, 16);
    if (PP == 32) PJ(64, 32);
    if (PP == 64) PJ(64, 64);
  }
#undef PJ
  return cudaErrorInvalidValue;
}

size_t kmeans_step_smem(int mode, int DK, int SW, int G) {
  return km_plan(mode, DK, SW, G).total + 1024;  // + alignment slack
}

template <int MODE, int DK, int SW>
static cudaError_t km_launch(const KmArgs& a, int nchunk, int BH, cudaStream_t st) {
  const size_t sm = kmeans_step_smem(MODE, DK, SW, a.G);
  cudaError_t e = cudaFuncSetAttribute(k_kmeans_step<MODE, DK, SW>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  spr_launch(k_kmeans_step<MODE, DK, SW>, dim3(nchunk, BH), KM_THREADS, sm, st, a);
  return cudaGetLastError();
}

cudaError_t launch_kmeans_step(int mode, int width, const KmArgs& a, int nchunk, int BH,
                               cudaStream_t st) {
  if (mode == KM_QUERY) {
    if (width == 64) return km_launch<KM_QUERY, 64, 64>(a, nchunk, BH, st);
    if (width == 128) return km_launch<KM_QUERY, 128, 128>(a, nchunk, BH, st);
  } else {
    if (width == 8) return km_launch<KM_KEY, 16, 8>(a, nchunk, BH, st);
    if (width == 16) return km_launch<KM_KEY, 16, 16>(a, nchunk, BH, st);
    if (width == 32) return km_launch<KM_KEY, 32, 32>(a, nchunk, BH, st);
    if (width == 64) return km_launch<KM_KEY, 64, 64>(a, nchunk, BH, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace spr
