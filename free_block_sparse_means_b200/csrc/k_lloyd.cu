// One Lloyd iteration of the partition's two k-means [paperlayer App. B.1,
// B.2; App. C.1 names a GPU k-means] as a persistent, warp-specialised kernel
// plus a reducer.
//
// Assignment (k_lloyd): each block takes a contiguous range of 128-row tiles
// of the flattened (head, tile) sequence; the tensor cores score every row of
// a tile against every centroid (tcgen05.mma kind::f16, bf16 operands in
// 128-byte-swizzled shared memory, fp32 accumulators in TMEM) and one thread
// per row takes the argmax (ties to the lowest group index):
//   query rows: score_g = (s / rms_n) q . Bq_g - beta_g; q exact in bf16, Bq_g
//               split into bf16 hi + lo (two products);
//   key rows:   score_g = z . c_g - beta_g with beta_g = ||c_g||^2 / 2 in
//               fp32; z and c_g split into hi + lo (three products: hh, hl,
//               lh).
// Roles: warp 0 lane 0 issues TMA loads (data tiles into an NS-stage ring; the
// centroid operand once per head); warp 1 owns TMEM (two score buffers) and
// one of its threads issues the products; warps 4-7 hold one row each (=
// TMEM lane): they convert key tiles to hi / lo, take the argmax of tile t
// while the products of tile t + 1 run, then sort the tile's rows stably by
// label and sum each label's run of update rows ((s / rms) q or z, read from
// the tile in shared memory) in fixed order.  A tile writes one partial sum
// and row count per label present, at the label's rank among the labels
// present; its 256-bit presence mask; and, per label, one bit of a
// group-major tile bitmap (integer OR, so its final value does not depend on
// timing).
//
// Update (k_lloyd_reduce): per (head, group), the tiles holding the group
// (from the bitmap, in tile order), their partial sums added in that order in
// fp64, divided by the count; an empty group keeps its centroid.  Every sum is
// taken in an order fixed by the data alone, so results are deterministic.
// Key centroids are also split into the next iteration's hi / lo operand.
//
// Every mbarrier wait is bounded in time: a wait that runs out sets an abort
// flag that ends every role, the device error word records a timeout, copies
// and products in flight are drained, and TMEM is freed.
#include <float.h>

#include "spr_internal.cuh"
#include "tc_sm100.cuh"

namespace spr {

namespace {

constexpr int LL_THREADS = 256;
constexpr int LL_TILE = 128;                 // rows per tile (the UMMA M)
constexpr uint32_t LL_BOX = LL_TILE * 128;   // one 64-column bf16 SW128 box of a tile: 16 KB
constexpr int LL_KW = 32;                    // key coordinates per row (p padded)
constexpr int LL_KSTEPS_KEY = LL_KW / 16;    // key K = 32 coordinates
constexpr uint32_t LL_MISC = 8192;
constexpr uint32_t LL_SMEM_LIMIT = 227 * 1024;
constexpr uint64_t LL_WAIT_NS = 2000000000ull;
constexpr int LL_ROW0 = 128;                 // first thread of the row role (warps 4-7)
constexpr int LL_SLOTS = LLOYD_SLOTS;        // partial sums per tile: at most one per row

struct LlPlan {
  int NC, NCS, nboxA, nboxB, NS;
  uint32_t tcols, stage_bytes, b_bytes, aset_bytes;
  uint32_t off_bl, off_aset, off_stage, off_misc, total;
};

// Shared memory (from a 1024-aligned base): centroid operand hi, lo (nboxB
// boxes of NC rows x 128 B each); key mode: two hi / lo conversion sets; the
// data stages; the misc area.  TMEM: two score buffers of NCS columns.
template <int MODE, int DK>
__host__ __device__ inline LlPlan ll_plan(int G) {
  LlPlan p;
  p.NC = (G + 31) / 32 * 32;
  p.NCS = 32;
  while (p.NCS < p.NC) p.NCS <<= 1;
  p.tcols = 2u * (uint32_t)p.NCS;
  if (MODE == KM_QUERY) {
    p.nboxA = DK / 64;
    p.nboxB = DK / 64;
    p.stage_bytes = (uint32_t)p.nboxA * LL_BOX;
    p.aset_bytes = 0;
  } else {
    p.nboxA = 1;
    p.nboxB = 1;
    p.stage_bytes = LL_TILE * LL_KW * 4;
    p.aset_bytes = 2 * LL_BOX;  // hi box, lo box (64 of their 128 bytes per row used)
  }
  p.b_bytes = (uint32_t)p.nboxB * (uint32_t)p.NC * 128u;
  p.off_bl = p.b_bytes;
  p.off_aset = 2 * p.b_bytes;
  p.off_stage = p.off_aset + 2 * p.aset_bytes;
  const int avail = (int)LL_SMEM_LIMIT - 1024 - (int)LL_MISC - (int)p.off_stage;
  int ns = avail > 0 ? avail / (int)p.stage_bytes : 0;
  p.NS = ns > 4 ? 4 : ns;
  p.off_misc = p.off_stage + (uint32_t)(p.NS > 0 ? p.NS : 0) * p.stage_bytes;
  p.total = p.off_misc + LL_MISC + 1024;
  return p;
}

struct LlArgs {
  int N, G, BH, H, ntile, nword;
  float scale;
  const float* rms;    // query: row RMS; the factor of row n is scale / rms[n]
  const float* beta;   // [BH][G]: query beta_g; key ||c_g||^2 / 2
  int32_t* lab;        // [BH][N] labels (out)
  float* slots;        // [BH * ntile][LL_SLOTS][W] partial sums (out)
  int32_t* slot_cnt;   // [BH * ntile][LL_SLOTS] rows per partial sum (out)
  uint32_t* tmask;     // [BH * ntile][8] labels present in each tile (out)
  uint32_t* gbits;     // [BH][G][nword] tiles holding each label (OR-ed in)
  Header* hdr;
};

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

// Byte offset of 16-byte chunk c of row r inside a 128-byte-swizzled box.
__device__ __forceinline__ uint32_t swz128(int r, int c) {
  return (uint32_t)(r * 128 + (((c ^ r) & 7) << 4));
}

__device__ __forceinline__ int warp_incl_scan(int x, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += t;
  }
  return x;
}

template <int MODE, int DK>
__global__ void __launch_bounds__(LL_THREADS, 1)
    k_lloyd(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
            LlArgs a) {
  constexpr int W = MODE == KM_QUERY ? DK : LL_KW;  // update-row width
  constexpr int VPL = W / 32;                        // update values per lane
  extern __shared__ uint8_t ll_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ll_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  const int G = a.G;
  const LlPlan pl = ll_plan<MODE, DK>(G);
  const int NC = pl.NC, NCS = pl.NCS, NS = pl.NS;
  uint8_t* Bh = sm;
  uint8_t* Bl = sm + pl.off_bl;
  uint8_t* Aset = sm + pl.off_aset;
  uint8_t* stg = sm + pl.off_stage;
  uint8_t* misc = sm + pl.off_misc;
  float* betas = reinterpret_cast<float*>(misc);           // [256]
  float* rowf = betas + 256;                               // [128]
  int* lof = reinterpret_cast<int*>(rowf + 128);           // [256] run start of each label
  int* lidx = lof + 256;                                   // [256] rank among labels present
  int* srt = lidx + 256;                                   // [128] row | label << 8, sorted
  uint32_t* cntw32 = reinterpret_cast<uint32_t*>(srt + 128);  // [256] words = [4][256] bytes
  uint8_t* cntw = reinterpret_cast<uint8_t*>(cntw32);
  int* scanw = reinterpret_cast<int*>(cntw32 + 256);       // [8]
  int* sbeg = scanw + 8;                                   // [4] first run start per warp
  int* stop_s = sbeg + 4;
  uint64_t* bars = reinterpret_cast<uint64_t*>(misc + 5376);
  uint64_t* d_full = bars;        // [4]
  uint64_t* d_empty = bars + 4;   // [4]
  uint64_t* a_ready = bars + 8;   // [2]
  uint64_t* s_full = bars + 10;   // [2]
  uint64_t* s_free = bars + 12;   // [2]
  uint64_t* b_full = bars + 14;
  uint64_t* b_free = bars + 15;
  uint64_t* drain = bars + 16;
  uint32_t* tmem_s = reinterpret_cast<uint32_t*>(bars + 17);
  volatile int* abort_s = reinterpret_cast<volatile int*>(tmem_s + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = a.BH * a.ntile;
  const int tb = (int)(((int64_t)blockIdx.x * T) / gridDim.x);
  const int te = (int)(((int64_t)(blockIdx.x + 1) * T) / gridDim.x);

  if (tid == 0) {
    for (int s = 0; s < 4; ++s) {
      tc::mbar_init(d_full + s, 1);
      tc::mbar_init(d_empty + s, 4);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(a_ready + s, 4);
      tc::mbar_init(s_full + s, 1);
      tc::mbar_init(s_free + s, 4);
    }
    tc::mbar_init(b_full, 1);
    tc::mbar_init(b_free, 1);
    tc::mbar_init(drain, 1);
    *abort_s = 0;
    *stop_s = 0;
    tc::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tc::prefetch_tmap(&tmX);
    tc::prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_s, pl.tcols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = *tmem_s;
  auto head_of = [&](int t) { return t / a.ntile; };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int k = 0, nb = 0, loads = 0;
      for (int t = tb; t < te; ++t, ++k) {
        const int bh = head_of(t), tl = t - bh * a.ntile;
        if (t == tb || bh != head_of(t - 1)) {  // centroid operand of a new head
          if (nb > 0 && !tc::mbar_wait(b_free, (nb - 1) & 1, abort_s, LL_WAIT_NS)) break;
          tc::mbar_expect_tx(b_full, 2 * pl.b_bytes);
          for (int h = 0; h < 2; ++h)
            for (int j = 0; j < pl.nboxB; ++j)
              tc::tma_load_3d((h ? Bl : Bh) + (uint32_t)j * NC * 128, &tmB, 64 * j, 0, 2 * bh + h,
                              b_full);
          ++nb;
        }
        const int s = k % NS;
        if (k >= NS && !tc::mbar_wait(d_empty + s, ((k / NS) - 1) & 1, abort_s, LL_WAIT_NS)) break;
        tc::mbar_expect_tx(d_full + s, pl.stage_bytes);
        uint8_t* dst = stg + (uint32_t)s * pl.stage_bytes;
        if (MODE == KM_QUERY) {
          // [B, H, N, d] view: coordinates (column, row, head, batch)
          const int bb = bh / a.H, hh = bh - bb * a.H;
          for (int j = 0; j < pl.nboxA; ++j)
            tc::tma_load_4d(dst + (uint32_t)j * LL_BOX, &tmX, 64 * j, tl * LL_TILE, hh, bb,
                            d_full + s);
        } else {
          tc::tma_load_3d(dst, &tmX, 0, tl * LL_TILE, bh, d_full + s);
        }
        ++loads;
      }
      if (*abort_s) {  // let the copies in flight land before the block exits
        for (int q = loads - NS; q < loads; ++q)
          if (q >= 0) tc::mbar_wait_bounded(d_full + (q % NS), (q / NS) & 1, 100000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ products
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16(LL_TILE, NC, 0);
      const uint32_t bh_addr = smem_u32(Bh), bl_addr = smem_u32(Bl);
      int k = 0, nb = 0;
      bool ok = true;
      for (int t = tb; t < te && ok; ++t, ++k) {
        const int bh = head_of(t);
        const bool hstart = t == tb || bh != head_of(t - 1);
        const bool hend = t + 1 == te || head_of(t + 1) != bh;
        if (hstart) {
          if (!tc::mbar_wait(b_full, nb & 1, abort_s, LL_WAIT_NS)) break;
          ++nb;
        }
        const int s = k % NS, b = k & 1;
        if (MODE == KM_QUERY) {
          if (!tc::mbar_wait(d_full + s, (k / NS) & 1, abort_s, LL_WAIT_NS)) break;
        } else {
          if (!tc::mbar_wait(a_ready + b, (k >> 1) & 1, abort_s, LL_WAIT_NS)) break;
        }
        if (k >= 2 && !tc::mbar_wait(s_free + b, ((k >> 1) - 1) & 1, abort_s, LL_WAIT_NS)) break;
        tc::tc_fence_after();
        const uint32_t d = tbase + (uint32_t)(b * NCS);
        if (MODE == KM_QUERY) {
          const uint32_t a_addr = smem_u32(stg + (uint32_t)s * pl.stage_bytes);
#pragma unroll
          for (int ks = 0; ks < DK / 16; ++ks) {
            const uint32_t ao = (ks >> 2) * LL_BOX + (ks & 3) * 32;
            const uint32_t bo = (ks >> 2) * NC * 128 + (ks & 3) * 32;
            tc::mma_ss(d, tc::smem_desc_sw128(a_addr + ao, 16, 1024),
                       tc::smem_desc_sw128(bh_addr + bo, 16, 1024), idesc, ks > 0);
            tc::mma_ss(d, tc::smem_desc_sw128(a_addr + ao, 16, 1024),
                       tc::smem_desc_sw128(bl_addr + bo, 16, 1024), idesc, 1);
          }
        } else {
          const uint32_t ah = smem_u32(Aset + (uint32_t)b * pl.aset_bytes), al = ah + LL_BOX;
#pragma unroll
          for (int ks = 0; ks < LL_KSTEPS_KEY; ++ks) {
            const uint32_t o = ks * 32;
            tc::mma_ss(d, tc::smem_desc_sw128(ah + o, 16, 1024),
                       tc::smem_desc_sw128(bh_addr + o, 16, 1024), idesc, ks > 0);
            tc::mma_ss(d, tc::smem_desc_sw128(ah + o, 16, 1024),
                       tc::smem_desc_sw128(bl_addr + o, 16, 1024), idesc, 1);
            tc::mma_ss(d, tc::smem_desc_sw128(al + o, 16, 1024),
                       tc::smem_desc_sw128(bh_addr + o, 16, 1024), idesc, 1);
          }
        }
        tc::mma_commit(s_full + b);
        if (hend) tc::mma_commit(b_free);
      }
      tc::mma_commit(drain);  // every product issued so far completes before TMEM is freed
      tc::mbar_wait_bounded(drain, 0, LL_WAIT_NS);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ rows
    const int r = tid - LL_ROW0, rw = warp - 4;
    const uint32_t lane_f = (uint32_t)(rw * 32) << 16;
    const unsigned lt_mask = (1u << lane) - 1u;
    int cur_bh = -1;
    bool ok = true;
    // key tiles: fp32 rows -> hi / lo bf16 conversion set (k & 1)
    auto convert = [&](int kk) -> bool {
      const int s = kk % NS;
      bool got = tc::mbar_wait(d_full + s, (kk / NS) & 1, abort_s, LL_WAIT_NS);
      got = __all_sync(0xffffffffu, got);
      if (!got) return false;
      const uint8_t* src = stg + (uint32_t)s * pl.stage_bytes;
      float z[LL_KW];
#pragma unroll
      for (int c = 0; c < LL_KW / 4; ++c) {
        const float4 v = *reinterpret_cast<const float4*>(src + swz128(r, c));
        z[4 * c] = v.x;
        z[4 * c + 1] = v.y;
        z[4 * c + 2] = v.z;
        z[4 * c + 3] = v.w;
      }
      uint8_t* ah = Aset + (uint32_t)(kk & 1) * pl.aset_bytes;
#pragma unroll
      for (int j = 0; j < LL_KW / 8; ++j) {
        *reinterpret_cast<uint4*>(ah + swz128(r, j)) = split8(z + 8 * j, false);
        *reinterpret_cast<uint4*>(ah + LL_BOX + swz128(r, j)) = split8(z + 8 * j, true);
      }
      tc::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(a_ready + (kk & 1));
      return true;
    };
    if (MODE == KM_KEY && te > tb) ok = convert(0);
    int k = 0;
    for (int t = tb; t < te; ++t, ++k) {
      // a uniform stop decision for the four row warps
      tc::named_sync(1, 128);
      if (r == 0) *stop_s = *abort_s;
      tc::named_sync(1, 128);
      if (*stop_s) break;
      const int bh = head_of(t), tl = t - bh * a.ntile;
      const int n0 = tl * LL_TILE, n = n0 + r;
      const bool valid = n < a.N;
      const int nvalid = min(LL_TILE, a.N - n0);
      if (MODE == KM_KEY && t + 1 < te) ok = convert(k + 1) && ok;
      float f = 1.f;
      if (MODE == KM_QUERY) f = valid ? a.scale / a.rms[(size_t)bh * a.N + n] : 0.f;
      if (bh != cur_bh) {  // this head's beta_g (every row warp is past the last argmax)
        for (int g = r; g < NC; g += 128) betas[g] = g < G ? a.beta[(size_t)bh * G + g] : 0.f;
        tc::named_sync(1, 128);
      }
      cur_bh = bh;
      // ---- scores of tile k from TMEM, argmax (ties to the lowest index)
      const int b = k & 1;
      bool got = tc::mbar_wait(s_full + b, (k >> 1) & 1, abort_s, LL_WAIT_NS);
      got = __all_sync(0xffffffffu, got);
      int arg = 0;
      if (got) {
        tc::tc_fence_after();
        float best[4] = {-FLT_MAX, -FLT_MAX, -FLT_MAX, -FLT_MAX};
        int bi[4] = {0, 0, 0, 0};
        for (int c0 = 0; c0 < NC; c0 += 32) {
          uint32_t v[32];
          __syncwarp();
          tc::tmem_ld32(tbase + lane_f + (uint32_t)(b * NCS + c0), v);
          tc::tmem_wait_ld();
          if (c0 + 32 <= G) {
#pragma unroll
            for (int j4 = 0; j4 < 8; ++j4) {
              const float4 be = *reinterpret_cast<const float4*>(betas + c0 + 4 * j4);
              const float bq[4] = {be.x, be.y, be.z, be.w};
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int j = 4 * j4 + q;
                const float sc = MODE == KM_QUERY ? fmaf(f, __uint_as_float(v[j]), -bq[q])
                                                  : __uint_as_float(v[j]) - bq[q];
                if (sc > best[q]) {
                  best[q] = sc;
                  bi[q] = c0 + j;
                }
              }
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int g = c0 + j;
              if (g < G) {
                const float sc = MODE == KM_QUERY ? fmaf(f, __uint_as_float(v[j]), -betas[g])
                                                  : __uint_as_float(v[j]) - betas[g];
                if (sc > best[j & 3]) {
                  best[j & 3] = sc;
                  bi[j & 3] = g;
                }
              }
            }
          }
        }
        float bb = best[0];
        arg = bi[0];
#pragma unroll
        for (int q = 1; q < 4; ++q)
          if (best[q] > bb || (best[q] == bb && bi[q] < arg)) {
            bb = best[q];
            arg = bi[q];
          }
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(s_free + b);
      } else {
        ok = false;
      }
      const int g = valid ? arg : -1;
      if (valid && got) a.lab[(size_t)bh * a.N + n] = g;
      rowf[r] = f;
      // ---- stable sort of the tile's rows by label
      cntw32[r] = 0u;
      cntw32[r + 128] = 0u;
      const unsigned mt = __match_any_sync(0xffffffffu, g);
      const int rank = __popc(mt & lt_mask);
      tc::named_sync(1, 128);
      if (g >= 0 && (__ffs(mt) - 1) == lane) cntw[rw * 256 + g] = (uint8_t)__popc(mt);
      tc::named_sync(1, 128);
      int hcount[2];
#pragma unroll
      for (int q = 0; q < 2; ++q) {  // bins r and r + 128: counts over warps, prefix in place
        const int bin = r + 128 * q;
        const int c0 = cntw[bin], c1 = cntw[256 + bin], c2 = cntw[512 + bin], c3 = cntw[768 + bin];
        cntw[bin] = 0;
        cntw[256 + bin] = (uint8_t)c0;
        cntw[512 + bin] = (uint8_t)(c0 + c1);
        cntw[768 + bin] = (uint8_t)(c0 + c1 + c2);
        hcount[q] = c0 + c1 + c2 + c3;
      }
      // exclusive scans over the 256 bins of (count, present) packed in one int
      const int x0 = hcount[0] | ((hcount[0] > 0) << 16), x1 = hcount[1] | ((hcount[1] > 0) << 16);
      const int i0 = warp_incl_scan(x0, lane), i1 = warp_incl_scan(x1, lane);
      if (lane == 31) {
        scanw[rw] = i0;
        scanw[4 + rw] = i1;
      }
      tc::named_sync(1, 128);
      int b0 = 0, b1 = 0, tot0 = 0;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        tot0 += scanw[w];
        if (w < rw) {
          b0 += scanw[w];
          b1 += scanw[4 + w];
        }
      }
      const int e0 = b0 + i0 - x0, e1 = tot0 + b1 + i1 - x1;
      lof[r] = e0 & 0xFFFF;
      lidx[r] = e0 >> 16;
      lof[r + 128] = e1 & 0xFFFF;
      lidx[r + 128] = e1 >> 16;
      // labels present: the tile's mask and the group-major tile bitmap
      const unsigned m0 = __ballot_sync(0xffffffffu, hcount[0] > 0);
      const unsigned m1 = __ballot_sync(0xffffffffu, hcount[1] > 0);
      if (lane == 0) {
        a.tmask[(size_t)t * 8 + rw] = m0;
        a.tmask[(size_t)t * 8 + 4 + rw] = m1;
      }
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int bin = r + 128 * q;
        if (hcount[q] > 0 && bin < G)
          atomicOr(a.gbits + ((size_t)bh * G + bin) * a.nword + (tl >> 5), 1u << (tl & 31));
      }
      tc::named_sync(1, 128);
      if (g >= 0) {
        const int pos = lof[g] + cntw[rw * 256 + g] + rank;
        if (pos < 0 || pos >= nvalid)
          set_error(a.hdr, ERR_INDEX, 9, bh, n);
        else
          srt[pos] = r | (g << 8);
      }
      tc::named_sync(1, 128);
      {  // first run start in this warp's 32 sorted positions
        const int p = 32 * rw + lane;
        const int lp = p < nvalid ? srt[p] >> 8 : -1;
        const int lq = (p > 0 && p - 1 < nvalid) ? srt[p - 1] >> 8 : -2;
        const unsigned st = __ballot_sync(0xffffffffu, p < nvalid && lp != lq);
        if (lane == 0) sbeg[rw] = st ? 32 * rw + __ffs(st) - 1 : -1;
      }
      tc::named_sync(1, 128);
      // ---- run sums: this warp takes the runs that start in its positions
      const int beg = sbeg[rw];
      if (beg >= 0) {
        int end = nvalid;
        for (int w2 = rw + 1; w2 < 4; ++w2)
          if (sbeg[w2] >= 0) {
            end = sbeg[w2];
            break;
          }
        const uint8_t* tile = stg + (uint32_t)(k % NS) * pl.stage_bytes;
        float acc[VPL];
#pragma unroll
        for (int q = 0; q < VPL; ++q) acc[q] = 0.f;
        int cur = -1, cnt = 0;
        float* sbase = a.slots + (size_t)t * LL_SLOTS * W;
        auto flush = [&]() {
          if (cur < 0) return;
          const int slot = lidx[cur];
          float* dst = sbase + (size_t)slot * W + lane * VPL;
          if (VPL == 4)
            *reinterpret_cast<float4*>(dst) = make_float4(acc[0], acc[1], acc[2], acc[3]);
          else if (VPL == 2)
            *reinterpret_cast<float2*>(dst) = make_float2(acc[0], acc[1]);
          else
            dst[0] = acc[0];
          if (lane == 0) a.slot_cnt[(size_t)t * LL_SLOTS + slot] = cnt;
        };
        for (int pb = beg; pb < end; pb += 32) {
          const int e_l = pb + lane < end ? srt[pb + lane] : -1;
          const int row_l = e_l & 255;
          const int g_l = e_l >= 0 ? e_l >> 8 : -1;
          const float f_l = e_l >= 0 ? rowf[row_l] : 0.f;
          const int nu = min(32, end - pb);
          for (int u = 0; u < nu; ++u) {
            const int gu = __shfl_sync(0xffffffffu, g_l, u);
            const int ru = __shfl_sync(0xffffffffu, row_l, u);
            const float fu = __shfl_sync(0xffffffffu, f_l, u);
            if (gu != cur) {
              flush();
#pragma unroll
              for (int q = 0; q < VPL; ++q) acc[q] = 0.f;
              cur = gu;
              cnt = 0;
            }
            ++cnt;
            if (MODE == KM_QUERY) {
              if (DK == 128) {
                const uint32_t off = (uint32_t)(lane >> 4) * LL_BOX + swz128(ru, (lane & 15) >> 1) +
                                     ((lane & 1) << 3);
                const uint2 x = *reinterpret_cast<const uint2*>(tile + off);
                const float2 xa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&x.x));
                const float2 xb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&x.y));
                acc[0] = fmaf(fu, xa.x, acc[0]);
                acc[1] = fmaf(fu, xa.y, acc[1]);
                acc[2] = fmaf(fu, xb.x, acc[2]);
                acc[3] = fmaf(fu, xb.y, acc[3]);
              } else {
                const uint32_t off = swz128(ru, lane >> 2) + ((lane & 3) << 2);
                const float2 xa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(tile + off));
                acc[0] = fmaf(fu, xa.x, acc[0]);
                acc[1] = fmaf(fu, xa.y, acc[1]);
              }
            } else {
              const uint32_t off = swz128(ru, lane >> 2) + ((lane & 3) << 2);
              acc[0] += *reinterpret_cast<const float*>(tile + off);
            }
          }
        }
        flush();
      }
      // the tile's data stage is free again
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(d_empty + (k % NS));
      tc::named_sync(1, 128);  // sort arrays and row factors are reused by the next tile
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (tid == 0 && *abort_s) set_error(a.hdr, ERR_TIMEOUT, 9, blockIdx.x, 0);
  if (warp == 1) {
    __syncwarp();
    tc::tmem_dealloc(tbase, pl.tcols);
  }
}

// Key operand of the next assignment from centroid c_g (32 coordinates, one
// per lane): hi / lo bf16 rows of 64 columns (coordinates in 0..31, zeros
// after) and beta_g = ||c_g||^2 / 2 in fp32 (lane sums in a fixed order).
__device__ __forceinline__ void key_operand_row(float v, int lane, bf16* hi_row, bf16* lo_row,
                                                float* beta) {
  const float nrm = warp_sum(v * v);
  const bf16 vh = __float2bfloat16_rn(v);
  hi_row[lane] = vh;
  lo_row[lane] = __float2bfloat16_rn(v - __bfloat162float(vh));
  hi_row[32 + lane] = __float2bfloat16_rn(0.f);
  lo_row[32 + lane] = __float2bfloat16_rn(0.f);
  if (lane == 0 && beta) *beta = 0.5f * nrm;
}

// Grid (ncrows, BH), 32 threads: the key operand of rows g < ncrows (rows
// past G are zero) and beta_g of the G groups.
__global__ void __launch_bounds__(32) k_kprep(const float* cent, int G, int ncrows, bf16* bk,
                                              float* beta) {
  const int g = blockIdx.x, bh = blockIdx.y, lane = threadIdx.x;
  const float v = g < G ? cent[((size_t)bh * G + g) * LL_KW + lane] : 0.f;
  bf16* hi = bk + (((size_t)bh * 2 + 0) * ncrows + g) * 64;
  bf16* lo = bk + (((size_t)bh * 2 + 1) * ncrows + g) * 64;
  key_operand_row(v, lane, hi, lo, g < G ? beta + (size_t)bh * G + g : nullptr);
}

// Block-wide exclusive scan (blockDim.x a multiple of 32, at most 1024).
__device__ __forceinline__ int block_exscan_small(int v, int* sh, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int x = warp_incl_scan(v, lane);
  if (lane == 31) sh[w] = x;
  __syncthreads();
  int before = 0, tot = 0;
  for (int i = 0; i < nw; ++i) {
    if (i < w) before += sh[i];
    tot += sh[i];
  }
  __syncthreads();
  *total = tot;
  return before + x - v;
}

// The update of group g of head bh: its partial sums in tile order (the
// group's row of the tile bitmap, cleared here for the next iteration), added
// in fp64, over the rows counted; an empty group keeps its centroid.  Key
// mode also writes the next iteration's operand row.  Grid (G, BH), W threads.
template <int W>
__global__ void __launch_bounds__(W) k_lloyd_reduce(const float* slots, const int32_t* slot_cnt,
                                                    const uint32_t* tmask, uint32_t* gbits, int G,
                                                    int ntile, int nword, float* cent, bf16* bk,
                                                    float* beta, int ncrows) {
  __shared__ int list[32 * W];
  __shared__ int shs[32];
  const int g = blockIdx.x, bh = blockIdx.y, c = threadIdx.x;
  uint32_t* row = gbits + ((size_t)bh * G + g) * nword;
  const float* sb = slots + (size_t)bh * ntile * LL_SLOTS * W;
  const int32_t* cb = slot_cnt + (size_t)bh * ntile * LL_SLOTS;
  const uint32_t* mb = tmask + (size_t)bh * ntile * 8;
  double s0 = 0.0, s1 = 0.0;
  long long cnt = 0;
  for (int w0 = 0; w0 < nword; w0 += W) {
    const int w = w0 + c;
    uint32_t bits = w < nword ? row[w] : 0u;
    if (w < nword) row[w] = 0u;
    int n;
    int o = block_exscan_small(__popc(bits), shs, &n);
    while (bits) {  // the tiles of this word, in increasing order
      list[o++] = w * 32 + __ffs(bits) - 1;
      bits &= bits - 1u;
    }
    __syncthreads();
    for (int i = c; i < n; i += W) {  // slot of g in each listed tile: its rank among the labels
      const int tl = list[i];
      const uint32_t* m = mb + (size_t)tl * 8;
      int rk = __popc(m[g >> 5] & ((1u << (g & 31)) - 1u));
      for (int j = 0; j < (g >> 5); ++j) rk += __popc(m[j]);
      list[i] = tl * LL_SLOTS + rk;
    }
    __syncthreads();
    int i = 0;
    for (; i + 1 < n; i += 2) {  // two interleaved fp64 chains, added in order at the end
      s0 += (double)sb[(size_t)list[i] * W + c];
      s1 += (double)sb[(size_t)list[i + 1] * W + c];
    }
    if (i < n) s0 += (double)sb[(size_t)list[i] * W + c];
    for (int q = 0; q < n; ++q) cnt += cb[list[q]];
    __syncthreads();
  }
  float* cg = cent + ((size_t)bh * G + g) * W;
  float v = cg[c];
  if (cnt > 0) {
    v = (float)((s0 + s1) / (double)cnt);
    cg[c] = v;
  }
  if (bk != nullptr && W == LL_KW) {
    bf16* hi = bk + (((size_t)bh * 2 + 0) * ncrows + g) * 64;
    bf16* lo = bk + (((size_t)bh * 2 + 1) * ncrows + g) * 64;
    key_operand_row(v, c, hi, lo, beta + (size_t)bh * G + g);
  }
}

// Chunk label histograms chunk_cnt[bh][chunk][g] for the stable scatter into
// group-major order.  Grid (nchunk, BH), CHUNK threads.
__global__ void __launch_bounds__(CHUNK) k_label_hist(const int32_t* lab, int N, int G, int nchunk,
                                                      int32_t* chunk_cnt, Header* hdr) {
  __shared__ int h[MAX_GROUPS];
  const int chunk = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
  for (int e = tid; e < G; e += CHUNK) h[e] = 0;
  __syncthreads();
  const int n = chunk * CHUNK + tid;
  if (n < N) {
    const int g = lab[(size_t)bh * N + n];
    if (g >= 0 && g < G)
      atomicAdd(&h[g], 1);
    else
      set_error(hdr, ERR_INDEX, 11, bh, n);
  }
  __syncthreads();
  for (int e = tid; e < G; e += CHUNK) chunk_cnt[((size_t)bh * nchunk + chunk) * G + e] = h[e];
}

template <int MODE, int DK>
cudaError_t lloyd_launch(const CUtensorMap& tmX, const CUtensorMap& tmB, const LlArgs& a,
                         cudaStream_t st) {
  const LlPlan pl = ll_plan<MODE, DK>(a.G);
  if (pl.NS < 2) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(k_lloyd<MODE, DK>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.total);
  if (e != cudaSuccess) return e;
  const int T = a.BH * a.ntile;
  const int grid = T < num_sms() ? T : num_sms();
  spr_launch(k_lloyd<MODE, DK>, grid, LL_THREADS, pl.total, st, tmX, tmB, a);
  return cudaGetLastError();
}

}  // namespace

int lloyd_ncrows(int G) { return (G + 31) / 32 * 32; }

cudaError_t lloyd_step(const LloydStep& s, cudaStream_t st) {
  const int ntile = (s.N + LL_TILE - 1) / LL_TILE;
  const int nword = (ntile + 31) / 32;
  const int NC = lloyd_ncrows(s.G);
  // every buffer the step writes must hold what it writes
  const size_t nt = (size_t)s.BH * ntile;
  if (s.G < 1 || s.G > MAX_GROUPS || s.slots_bytes < lloyd_slot_bytes(s.BH, s.N, s.d) ||
      s.slot_cnt_bytes < nt * LL_SLOTS * 4 || s.tmask_bytes < nt * 8 * 4 ||
      s.gbits_bytes < (size_t)s.BH * s.G * nword * 4)
    return cudaErrorInvalidValue;
  CUtensorMap tmX, tmB;
  if (s.mode == KM_QUERY) {
    if (s.d != 64 && s.d != 128) return cudaErrorInvalidValue;
    // data rows: the [B, H, N, d] view with its element strides
    const int B = s.BH / s.X.H, H = s.X.H;
    const uint64_t dims[4] = {(uint64_t)s.d, (uint64_t)s.N, (uint64_t)H, (uint64_t)B};
    const uint64_t str[3] = {(uint64_t)s.X.sn * 2, (uint64_t)s.X.sh * 2, (uint64_t)s.X.sb * 2};
    const uint32_t box[4] = {64, LL_TILE, 1, 1};
    if (!encode_tmap(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, s.X.base, dims, str, box,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    // centroid operand: [BH][2][split_rows][d] bf16, rows 0 .. NC - 1 read
    const uint64_t bd[3] = {(uint64_t)s.d, (uint64_t)NC, (uint64_t)(2 * s.BH)};
    const uint64_t bs[2] = {(uint64_t)s.d * 2, (uint64_t)s.split_rows * s.d * 2};
    const uint32_t bb[3] = {64, (uint32_t)NC, 1};
    if (NC > s.split_rows ||
        !encode_tmap(&tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, s.bq, bd, bs, bb,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  } else {
    const uint64_t dims[3] = {(uint64_t)LL_KW, (uint64_t)s.N, (uint64_t)s.BH};
    const uint64_t str[2] = {(uint64_t)LL_KW * 4, (uint64_t)s.N * LL_KW * 4};
    const uint32_t box[3] = {LL_KW, LL_TILE, 1};
    if (!encode_tmap(&tmX, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, s.Z, dims, str, box,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    const uint64_t bd[3] = {64, (uint64_t)NC, (uint64_t)(2 * s.BH)};
    const uint64_t bs[2] = {128, (uint64_t)NC * 128};
    const uint32_t bb[3] = {64, (uint32_t)NC, 1};
    if (!encode_tmap(&tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, s.bk, bd, bs, bb,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  LlArgs a{};
  a.N = s.N;
  a.G = s.G;
  a.BH = s.BH;
  a.H = s.X.H > 0 ? s.X.H : 1;
  a.ntile = ntile;
  a.nword = nword;
  a.scale = s.scale;
  a.rms = s.rms;
  a.beta = s.beta;
  a.lab = s.lab;
  a.slots = s.slots;
  a.slot_cnt = s.slot_cnt;
  a.tmask = s.tmask;
  a.gbits = s.gbits;
  a.hdr = s.hdr;
  cudaError_t e;
  if (s.mode == KM_QUERY)
    e = s.d == 64 ? lloyd_launch<KM_QUERY, 64>(tmX, tmB, a, st)
                  : lloyd_launch<KM_QUERY, 128>(tmX, tmB, a, st);
  else
    e = lloyd_launch<KM_KEY, LL_KW>(tmX, tmB, a, st);
  if (e != cudaSuccess) return e;
  // the update
  const dim3 rg(s.G, s.BH);
  if (s.mode == KM_QUERY) {
    if (s.d == 64)
      spr_launch(k_lloyd_reduce<64>, rg, 64, 0, st, static_cast<const float*>(s.slots),
                 static_cast<const int32_t*>(s.slot_cnt), static_cast<const uint32_t*>(s.tmask),
                 s.gbits, s.G, ntile, nword, s.cent, static_cast<bf16*>(nullptr),
                 static_cast<float*>(nullptr), 0);
    else
      spr_launch(k_lloyd_reduce<128>, rg, 128, 0, st, static_cast<const float*>(s.slots),
                 static_cast<const int32_t*>(s.slot_cnt), static_cast<const uint32_t*>(s.tmask),
                 s.gbits, s.G, ntile, nword, s.cent, static_cast<bf16*>(nullptr),
                 static_cast<float*>(nullptr), 0);
  } else {
    spr_launch(k_lloyd_reduce<LL_KW>, rg, LL_KW, 0, st, static_cast<const float*>(s.slots),
               static_cast<const int32_t*>(s.slot_cnt), static_cast<const uint32_t*>(s.tmask),
               s.gbits, s.G, ntile, nword, s.cent, s.bk, const_cast<float*>(s.beta), NC);
  }
  return cudaGetLastError();
}

cudaError_t lloyd_key_operand(const float* cent, int G, int BH, bf16* bk, float* beta,
                              cudaStream_t st) {
  spr_launch(k_kprep, dim3(lloyd_ncrows(G), BH), 32, 0, st, cent, G, lloyd_ncrows(G), bk, beta);
  return cudaGetLastError();
}

cudaError_t label_hist(const int32_t* lab, int N, int G, int nchunk, int BH, int32_t* chunk_cnt,
                       Header* hdr, cudaStream_t st) {
  spr_launch(k_label_hist, dim3(nchunk, BH), CHUNK, 0, st, lab, N, G, nchunk, chunk_cnt, hdr);
  return cudaGetLastError();
}

size_t lloyd_slot_bytes(int BH, int N, int d) {
  const size_t ntile = ((size_t)N + LL_TILE - 1) / LL_TILE;
  const size_t w = d > LL_KW ? d : LL_KW;
  return (size_t)BH * ntile * LL_SLOTS * w * 4;
}

}  // namespace spr
