// One Lloyd iteration of the partition's two k-means [paperlayer App. B.1,
// B.2] on a chunk of CHUNK rows, fused into one kernel:
//   1. assignment on the tensor cores (mma.sync m16n8k16 bf16, fp32
//      accumulation), tiles of 128 rows double-buffered in shared memory;
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

namespace spr {

constexpr int KM_THREADS = 256;
constexpr int KM_TILE = 128;  // rows per sub-tile: 8 warps x 16

__host__ __device__ constexpr int km_rs(int DK) { return DK * 2 + 16; }  // padded bf16 row (bytes)

template <int MODE, int DK, int SW>
__global__ void __launch_bounds__(KM_THREADS) k_kmeans_step(KmArgs a) {
  constexpr int RS = km_rs(DK);
  constexpr int NA = (MODE == KM_KEY) ? 2 : 1;  // A tiles: hi (and lo)
  constexpr int KS = DK / 16;                    // k-steps
  extern __shared__ __align__(128) uint8_t km[];
  const int G = a.G, NC = ((G + 31) / 32) * 32;
  uint8_t* Bh = km;
  uint8_t* Bl = Bh + NC * RS;
  float* betas = reinterpret_cast<float*>(Bl + NC * RS);
  int* labs = reinterpret_cast<int*>(betas + MAX_GROUPS);
  uint8_t* Ab = reinterpret_cast<uint8_t*>(labs + CHUNK);
  const int bh = blockIdx.y, chunk = blockIdx.x, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31, gid = lane >> 2, tig = lane & 3;
  const int N = a.N, n0 = chunk * CHUNK, rows = min(CHUNK, N - n0);

  // ---- centroid operand -------------------------------------------------
  if (MODE == KM_QUERY) {
    const bf16* bsrc = a.bsplit + (size_t)bh * 2 * a.split_rows * DK;
    for (int e = tid; e < NC * (DK / 8); e += KM_THREADS) {
      const int r = e / (DK / 8), c = e % (DK / 8);
      uint4 hi = make_uint4(0, 0, 0, 0), lo = hi;
      if (r < G) {
        hi = reinterpret_cast<const uint4*>(bsrc + (size_t)r * DK)[c];
        lo = reinterpret_cast<const uint4*>(bsrc + ((size_t)a.split_rows + r) * DK)[c];
      }
      *reinterpret_cast<uint4*>(Bh + r * RS + c * 16) = hi;
      *reinterpret_cast<uint4*>(Bl + r * RS + c * 16) = lo;
    }
    for (int g = tid; g < MAX_GROUPS; g += KM_THREADS)
      betas[g] = g < G ? a.beta[(size_t)bh * G + g] : 0.f;
  } else {
    const float* cs = a.cent + (size_t)bh * G * SW;
    for (int e = tid; e < NC * DK; e += KM_THREADS) {
      const int r = e / DK, c = e % DK;
      const float v = (r < G && c < SW) ? cs[r * SW + c] : 0.f;
      const bf16 hi = __float2bfloat16_rn(v);
      reinterpret_cast<bf16*>(Bh + r * RS)[c] = hi;
      reinterpret_cast<bf16*>(Bl + r * RS)[c] = __float2bfloat16_rn(v - __bfloat162float(hi));
    }
    for (int g = tid; g < MAX_GROUPS; g += KM_THREADS) {
      float s = 0.f;
      if (g < G)
        for (int c = 0; c < SW; ++c) s = fmaf(cs[g * SW + c], cs[g * SW + c], s);
      betas[g] = s;
    }
  }

  // ---- assignment -------------------------------------------------------
  // QUERY: A tiles [2][KM_TILE][RS] loaded with cp.async.
  // KEY:   raw fp32 tiles [2][KM_TILE][SW] with cp.async, converted into the
  //        hi / lo bf16 tiles Ah, Al [KM_TILE][RS] before each use.
  uint8_t* raw = Ab;
  uint8_t* Akey = Ab + (MODE == KM_KEY ? 2 * KM_TILE * SW * 4 : 0);
  auto load_tile = [&](int sub, int buf) {
    const int r0 = n0 + sub * KM_TILE;
    if (MODE == KM_QUERY) {
      uint8_t* dst = Ab + (size_t)buf * KM_TILE * RS;
      for (int e = tid; e < KM_TILE * (DK / 8); e += KM_THREADS) {
        const int r = e / (DK / 8), c = e % (DK / 8), n = r0 + r;
        cp_async16(dst + r * RS + c * 16, a.Q.row(bh, n < N ? n : 0) + c * 8, n < N ? 16 : 0);
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
  const int nsub = (rows + KM_TILE - 1) / KM_TILE;
  load_tile(0, 0);
  for (int sub = 0; sub < nsub; ++sub) {
    if (sub + 1 < nsub) {
      load_tile(sub + 1, (sub + 1) & 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint8_t* Ah;
    const uint8_t* Al = nullptr;
    if (MODE == KM_QUERY) {
      Ah = Ab + (size_t)(sub & 1) * KM_TILE * RS;
    } else {
      const float* src = reinterpret_cast<const float*>(raw + (size_t)(sub & 1) * KM_TILE * SW * 4);
      uint8_t* h = Akey;
      uint8_t* l = Akey + KM_TILE * RS;
      for (int e = tid; e < KM_TILE * (DK / 4); e += KM_THREADS) {
        const int r = e / (DK / 4), c4 = e % (DK / 4);
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (4 * c4 < SW) v = reinterpret_cast<const float4*>(src + r * SW)[c4];
        const bf16 hx = __float2bfloat16_rn(v.x), hy = __float2bfloat16_rn(v.y);
        const bf16 hz = __float2bfloat16_rn(v.z), hw = __float2bfloat16_rn(v.w);
        uint2 ph, pl;
        ph.x = pack_bf16(__bfloat162float(hx), __bfloat162float(hy));
        ph.y = pack_bf16(__bfloat162float(hz), __bfloat162float(hw));
        pl.x = pack_bf16(v.x - __bfloat162float(hx), v.y - __bfloat162float(hy));
        pl.y = pack_bf16(v.z - __bfloat162float(hz), v.w - __bfloat162float(hw));
        *reinterpret_cast<uint2*>(h + r * RS + c4 * 8) = ph;
        *reinterpret_cast<uint2*>(l + r * RS + c4 * 8) = pl;
      }
      __syncthreads();
      Ah = h;
      Al = l;
    }
    uint32_t af[KS][4], al[NA == 2 ? KS : 1][4];
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const int r = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
      const int c = ks * 2 + (lane >> 4);
      ldsm_x4(af[ks][0], af[ks][1], af[ks][2], af[ks][3], Ah + r * RS + c * 16);
      if (NA == 2)
        ldsm_x4(al[ks][0], al[ks][1], al[ks][2], al[ks][3], Al + r * RS + c * 16);
    }
    const int lr_lo = sub * KM_TILE + warp * 16 + gid, lr_hi = lr_lo + 8;  // chunk-local rows
    const int r_lo = n0 + lr_lo, r_hi = n0 + lr_hi;
    float alpha_lo = 2.f, alpha_hi = 2.f;
    if (MODE == KM_QUERY) {
      alpha_lo = r_lo < N ? a.scale / a.rms[(size_t)bh * N + r_lo] : 0.f;
      alpha_hi = r_hi < N ? a.scale / a.rms[(size_t)bh * N + r_hi] : 0.f;
    }
    float best_lo = -FLT_MAX, best_hi = -FLT_MAX;
    int arg_lo = 0, arg_hi = 0;
    for (int nc = 0; nc < NC; nc += 32) {
      float acc[4][4];
#pragma unroll
      for (int t = 0; t < 4; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[t][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
        for (int pr = 0; pr < 2; ++pr) {  // two n-tile pairs of 16 columns
          const int brow = nc + pr * 16 + (lane & 7) + (lane >> 4) * 8;
          const int bc = ks * 2 + ((lane >> 3) & 1);
          uint32_t b0, b1, b2, b3;
          ldsm_x4(b0, b1, b2, b3, Bh + brow * RS + bc * 16);
          mma16816(acc[pr * 2], af[ks], b0, b1);
          mma16816(acc[pr * 2 + 1], af[ks], b2, b3);
          if (NA == 2) {
            mma16816(acc[pr * 2], al[ks], b0, b1);
            mma16816(acc[pr * 2 + 1], al[ks], b2, b3);
          }
          ldsm_x4(b0, b1, b2, b3, Bl + brow * RS + bc * 16);
          mma16816(acc[pr * 2], af[ks], b0, b1);
          mma16816(acc[pr * 2 + 1], af[ks], b2, b3);
        }
      }
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int col = nc + t * 8 + 2 * tig;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int g = col + e;
          if (g < G) {
            const float sl = alpha_lo * acc[t][e] - betas[g];
            const float sh = alpha_hi * acc[t][2 + e] - betas[g];
            if (sl > best_lo) { best_lo = sl; arg_lo = g; }
            if (sh > best_hi) { best_hi = sh; arg_hi = g; }
          }
        }
      }
    }
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      const float bl = __shfl_xor_sync(0xffffffffu, best_lo, o);
      const int al_ = __shfl_xor_sync(0xffffffffu, arg_lo, o);
      if (bl > best_lo || (bl == best_lo && al_ < arg_lo)) { best_lo = bl; arg_lo = al_; }
      const float bhv = __shfl_xor_sync(0xffffffffu, best_hi, o);
      const int ah = __shfl_xor_sync(0xffffffffu, arg_hi, o);
      if (bhv > best_hi || (bhv == best_hi && ah < arg_hi)) { best_hi = bhv; arg_hi = ah; }
    }
    if (tig == 0) {
      labs[lr_lo] = r_lo < N ? arg_lo : -1;
      labs[lr_hi] = r_hi < N ? arg_hi : -1;
      if (r_lo < N) a.lab[(size_t)bh * N + r_lo] = arg_lo;
      if (r_hi < N) a.lab[(size_t)bh * N + r_hi] = arg_hi;
    }
    __syncthreads();  // tile buffers free for the next load
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

size_t kmeans_step_smem(int mode, int DK, int SW, int G) {
  const size_t NC = (size_t)((G + 31) / 32) * 32;
  const size_t rs = (size_t)km_rs(DK);
  const size_t b = 2 * NC * rs + MAX_GROUPS * 4 + CHUNK * 4;
  const size_t tiles = mode == KM_KEY ? 2 * (size_t)KM_TILE * SW * 4 + 2 * (size_t)KM_TILE * rs
                                      : 2 * (size_t)KM_TILE * rs;
  const size_t rb = mode == KM_KEY ? (size_t)SW * 4 : (size_t)SW * 2;
  const size_t stg = (size_t)(KM_THREADS / 32) * (mode == KM_KEY ? 32 : 16) * rb;
  const size_t sortb = (32 * (size_t)G + CHUNK + MAX_GROUPS + 32) * 4 + stg;
  return b + (tiles > sortb ? tiles : sortb);
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
