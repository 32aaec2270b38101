// One Lloyd iteration of the partition's two k-means [paperlayer App. B.1,
// B.2; App. C.1 names a GPU k-means]: a persistent, warp-specialised
// assignment kernel on the tensor cores, an update kernel that sums each
// tile's rows per label, and a reducer.
//
// Assignment (k_lloyd_assign): each block takes a contiguous range of
// 128-row tiles of the flattened (head, tile) sequence; the tensor cores
// score every row of a tile against every centroid (tcgen05.mma kind::f16,
// bf16 operands in 128-byte-swizzled shared memory, fp32 accumulators in
// TMEM) and one thread per row takes the argmax (ties to the lowest group
// index):
//   query rows: score_g = (s / rms_n) q . Bq_g - beta_g; q exact in bf16, Bq_g
//               split into bf16 hi + lo (two products);
//   key rows:   score_g = z . c_g - beta_g with beta_g = ||c_g||^2 / 2 in
//               fp32; z (read as its bf16 hi | lo copy) and c_g split into
//               hi + lo (three products: hh, hl, lh).
// Roles: warp 8 lane 0 issues TMA loads (data tiles into an NS-stage ring, the
// centroid operand once per head); warp 9 owns TMEM (two score buffers) and
// one of its threads issues the products; a data stage is released by the
// commit of its products.  Warps 0-3 and 4-7 are two groups of row threads
// (warp w reads TMEM lanes 32 (w % 4) ..) that take alternate tiles, each with
// its own score buffer, so two row warps share every scheduler.
//
// Update (k_lloyd_update): one warp per tile sorts the tile's 128 (label,
// row) keys in registers (bitonic network, keys unique so the order within a
// label is the row order) and sums the update rows ((s / rms) q or the fp32
// z) of each label in that order, one run per label; run r of the sorted
// order (the rank of its label among the labels present) goes to slot r of
// the tile, with its row count, the tile's 256-bit label mask and, per label,
// one bit of a group-major tile bitmap (integer OR, so its final value does
// not depend on timing).
//
// Reduction (k_lloyd_reduce): per (head, group), the tiles holding the group
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

constexpr int LL_THREADS = 320;              // warps 0-7 rows, 8 producer, 9 TMEM / products
constexpr int LL_PRODUCER = 8;
constexpr int LL_MMA = 9;
constexpr int LL_TILE = 128;                 // rows per tile (the UMMA M)
constexpr uint32_t LL_BOX = LL_TILE * 128;   // one 64-column bf16 SW128 box of a tile: 16 KB
constexpr int LL_KW = 32;                    // key coordinates per row (p padded)
constexpr int LL_KSTEPS_KEY = LL_KW / 16;    // key K = 32 coordinates
constexpr uint32_t LL_MISC = 8 * 1024 + 256; // eight warps' beta rows, barriers
constexpr uint32_t LL_SMEM_LIMIT = 227 * 1024;
constexpr uint64_t LL_WAIT_NS = 2000000000ull;
constexpr int LL_SLOTS = LLOYD_SLOTS;        // partial sums per tile (labels present <= 128)
constexpr int LU_WARPS = 4;                  // update: tiles per block

struct LlPlan {
  int NC, NCS, nboxB, NS;
  uint32_t tcols, stage_bytes, b_bytes;
  uint32_t off_bl, off_stage, off_misc, total;
};

// Shared memory (from a 1024-aligned base): centroid operand hi, lo (nboxB
// boxes of NC rows x 128 B each); the data stages (query: d / 64 boxes of the
// bf16 rows; key: one box of the hi | lo rows); the misc area.  TMEM: two
// score buffers of NCS columns.
template <int MODE, int DK>
__host__ __device__ inline LlPlan ll_plan(int G) {
  LlPlan p;
  p.NC = (G + 31) / 32 * 32;
  p.NCS = 32;
  while (p.NCS < p.NC) p.NCS <<= 1;
  p.tcols = 2u * (uint32_t)p.NCS;
  p.nboxB = MODE == KM_QUERY ? DK / 64 : 1;
  p.stage_bytes = MODE == KM_QUERY ? (uint32_t)(DK / 64) * LL_BOX : LL_BOX;
  p.b_bytes = (uint32_t)p.nboxB * (uint32_t)p.NC * 128u;
  p.off_bl = p.b_bytes;
  p.off_stage = 2 * p.b_bytes;
  const int avail = (int)LL_SMEM_LIMIT - 1024 - (int)LL_MISC - (int)p.off_stage;
  int ns = avail > 0 ? avail / (int)p.stage_bytes : 0;
  p.NS = ns > 4 ? 4 : ns;
  p.off_misc = p.off_stage + (uint32_t)(p.NS > 0 ? p.NS : 0) * p.stage_bytes;
  p.total = p.off_misc + LL_MISC + 1024;
  return p;
}

struct LlArgs {
  int N, G, BH, H, ntile;
  float scale;
  const float* rms;    // query: row RMS; the factor of row n is scale / rms[n]
  const float* beta;   // [BH][G]: query beta_g; key ||c_g||^2 / 2
  int32_t* lab;        // [BH][N] labels (out)
  Header* hdr;
};

__device__ __forceinline__ int warp_incl_scan(int x, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += t;
  }
  return x;
}

// Scores of one row (this thread's TMEM lane) in columns 0 .. NC - 1 of a
// score buffer: argmax over g < G of f * s_g - beta_g (query) or s_g - beta_g
// (key), ties to the lowest g.  Eight chains take the columns in increasing
// order with a strict comparison; the chains are merged by (score, index).
template <int MODE>
__device__ __forceinline__ int row_argmax(uint32_t taddr, int NC, int G, float f,
                                          const float* betas) {
  float best[8];
  int bi[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    best[q] = -FLT_MAX;
    bi[q] = 0;
  }
  for (int c0 = 0; c0 < NC; c0 += 64) {
    uint32_t v[64];
    const bool two = c0 + 32 < NC;
    __syncwarp();
    tc::tmem_ld32(taddr + (uint32_t)c0, v);
    if (two) tc::tmem_ld32(taddr + (uint32_t)c0 + 32u, v + 32);
    tc::tmem_wait_ld();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int cb = c0 + 32 * h;
      if (h == 1 && !two) break;
      if (cb + 32 <= G) {
#pragma unroll
        for (int j4 = 0; j4 < 8; ++j4) {
          const float4 be = *reinterpret_cast<const float4*>(betas + cb + 4 * j4);
          const float bq[4] = {be.x, be.y, be.z, be.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = 4 * j4 + e, q = j & 7;
            const float x = __uint_as_float(v[32 * h + j]);
            const float sc = MODE == KM_QUERY ? fmaf(f, x, -bq[e]) : x - bq[e];
            if (sc > best[q]) {
              best[q] = sc;
              bi[q] = cb + j;
            }
          }
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int g = cb + j, q = j & 7;
          if (g < G) {
            const float x = __uint_as_float(v[32 * h + j]);
            const float sc = MODE == KM_QUERY ? fmaf(f, x, -betas[g]) : x - betas[g];
            if (sc > best[q]) {
              best[q] = sc;
              bi[q] = g;
            }
          }
        }
      }
    }
  }
  float bb = best[0];
  int arg = bi[0];
#pragma unroll
  for (int q = 1; q < 8; ++q)
    if (best[q] > bb || (best[q] == bb && bi[q] < arg)) {
      bb = best[q];
      arg = bi[q];
    }
  return arg;
}

template <int MODE, int DK>
__global__ void __launch_bounds__(LL_THREADS, 1)
    k_lloyd_assign(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
                   LlArgs a) {
  extern __shared__ uint8_t ll_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ll_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  const int G = a.G;
  const LlPlan pl = ll_plan<MODE, DK>(G);
  const int NC = pl.NC, NCS = pl.NCS, NS = pl.NS;
  uint8_t* Bh = sm;
  uint8_t* Bl = sm + pl.off_bl;
  uint8_t* stg = sm + pl.off_stage;
  uint8_t* misc = sm + pl.off_misc;
  float* betas_all = reinterpret_cast<float*>(misc);       // [8 warps][256]
  uint64_t* bars = reinterpret_cast<uint64_t*>(misc + 8 * 1024);
  uint64_t* d_full = bars;        // [4]
  uint64_t* d_empty = bars + 4;   // [4]
  uint64_t* s_full = bars + 8;    // [2]
  uint64_t* s_free = bars + 10;   // [2]
  uint64_t* b_full = bars + 12;
  uint64_t* b_free = bars + 13;
  uint64_t* drain = bars + 14;
  uint32_t* tmem_s = reinterpret_cast<uint32_t*>(bars + 15);
  volatile int* abort_s = reinterpret_cast<volatile int*>(tmem_s + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = a.BH * a.ntile;
  const int tb = (int)(((int64_t)blockIdx.x * T) / gridDim.x);
  const int te = (int)(((int64_t)(blockIdx.x + 1) * T) / gridDim.x);

  if (tid == 0) {
    for (int s = 0; s < 4; ++s) {
      tc::mbar_init(d_full + s, 1);
      tc::mbar_init(d_empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(s_full + s, 1);
      tc::mbar_init(s_free + s, 4);
    }
    tc::mbar_init(b_full, 1);
    tc::mbar_init(b_free, 1);
    tc::mbar_init(drain, 1);
    *abort_s = 0;
    tc::fence_barrier_init();
  }
  if (warp == LL_PRODUCER && lane == 0) {
    tc::prefetch_tmap(&tmX);
    tc::prefetch_tmap(&tmB);
  }
  if (warp == LL_MMA) {
    tc::tmem_alloc(tmem_s, pl.tcols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = *tmem_s;
  auto head_of = [&](int t) { return t / a.ntile; };

  if (warp == LL_PRODUCER) {
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
          for (int j = 0; j < DK / 64; ++j)
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
  } else if (warp == LL_MMA) {
    // ------------------------------------------------------------ products
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16(LL_TILE, NC, 0);
      const uint32_t bh_addr = smem_u32(Bh), bl_addr = smem_u32(Bl);
      int k = 0, nb = 0;
      for (int t = tb; t < te; ++t, ++k) {
        const int bh = head_of(t);
        const bool hstart = t == tb || bh != head_of(t - 1);
        const bool hend = t + 1 == te || head_of(t + 1) != bh;
        if (hstart) {
          if (!tc::mbar_wait(b_full, nb & 1, abort_s, LL_WAIT_NS)) break;
          ++nb;
        }
        const int s = k % NS, b = k & 1;
        if (!tc::mbar_wait(d_full + s, (k / NS) & 1, abort_s, LL_WAIT_NS)) break;
        if (k >= 2 && !tc::mbar_wait(s_free + b, ((k >> 1) - 1) & 1, abort_s, LL_WAIT_NS)) break;
        tc::tc_fence_after();
        const uint32_t d = tbase + (uint32_t)(b * NCS);
        const uint32_t a_addr = smem_u32(stg + (uint32_t)s * pl.stage_bytes);
        if (MODE == KM_QUERY) {
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
          // row = z_hi (columns 0-31) | z_lo (columns 32-63)
#pragma unroll
          for (int ks = 0; ks < LL_KSTEPS_KEY; ++ks) {
            const uint32_t o = ks * 32;
            tc::mma_ss(d, tc::smem_desc_sw128(a_addr + o, 16, 1024),
                       tc::smem_desc_sw128(bh_addr + o, 16, 1024), idesc, ks > 0);
            tc::mma_ss(d, tc::smem_desc_sw128(a_addr + o, 16, 1024),
                       tc::smem_desc_sw128(bl_addr + o, 16, 1024), idesc, 1);
            tc::mma_ss(d, tc::smem_desc_sw128(a_addr + 64 + o, 16, 1024),
                       tc::smem_desc_sw128(bh_addr + o, 16, 1024), idesc, 1);
          }
        }
        tc::mma_commit(d_empty + s);  // the stage is free once these products are done
        tc::mma_commit(s_full + b);
        if (hend) tc::mma_commit(b_free);
      }
      tc::mma_commit(drain);  // every product issued so far completes before TMEM is freed
      tc::mbar_wait_bounded(drain, 0, LL_WAIT_NS);
    }
  } else {
    // ------------------------------------------------------------ rows
    const int grp = warp >> 2, quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_f = (uint32_t)(quarter * 32) << 16;
    float* betas = betas_all + warp * 256;
    int cur_bh = -1;
    for (int k = grp, t = tb + grp; t < te; k += 2, t += 2) {
      const int bh = head_of(t), tl = t - bh * a.ntile;
      const int n = tl * LL_TILE + r;
      const bool valid = n < a.N;
      if (bh != cur_bh) {  // this head's beta_g, in this warp's own copy
        __syncwarp();
        for (int g = lane; g < NC; g += 32) betas[g] = g < G ? a.beta[(size_t)bh * G + g] : 0.f;
        __syncwarp();
        cur_bh = bh;
      }
      float f = 1.f;
      if (MODE == KM_QUERY) f = valid ? a.scale / a.rms[(size_t)bh * a.N + n] : 0.f;
      bool got = tc::mbar_wait(s_full + grp, (k >> 1) & 1, abort_s, LL_WAIT_NS);
      got = __all_sync(0xffffffffu, got);
      if (!got) break;
      tc::tc_fence_after();
      const int arg = row_argmax<MODE>(tbase + lane_f + (uint32_t)(grp * NCS), NC, G, f, betas);
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(s_free + grp);
      if (valid) a.lab[(size_t)bh * a.N + n] = arg;
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (tid == 0 && *abort_s) set_error(a.hdr, ERR_TIMEOUT, 9, blockIdx.x, 0);
  if (warp == LL_MMA) {
    __syncwarp();
    tc::tmem_dealloc(tbase, pl.tcols);
  }
}

struct LuArgs {
  int N, G, BH, ntile, nword;
  float scale;
  TensorView X;        // query mode rows
  const float* Z;      // key mode: [BH][N][32] fp32 coordinates
  const float* rms;    // query mode: row RMS
  const int32_t* lab;  // [BH][N]
  float* slots;        // [BH * ntile][LL_SLOTS][W]
  int32_t* slot_cnt;   // [BH * ntile][LL_SLOTS]
  uint32_t* tmask;     // [BH * ntile][8]
  uint32_t* gbits;     // [BH][G][nword]
  Header* hdr;
};

// Ascending bitonic sort of 128 distinct keys held by one warp, key[q] of
// lane l at position 32 q + l.
__device__ __forceinline__ void warp_sort128(int (&key)[4], int lane) {
#pragma unroll
  for (int k = 2; k <= 128; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j >= 32) {  // partner in this lane, register q ^ (j / 32)
        const int jq = j >> 5;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if ((q & jq) == 0) {
            const int q2 = q | jq;
            const bool asc = ((32 * q) & k) == 0;
            const int lo = min(key[q], key[q2]), hi = max(key[q], key[q2]);
            key[q] = asc ? lo : hi;
            key[q2] = asc ? hi : lo;
          }
        }
      } else {  // partner in lane ^ j, same register
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int o = __shfl_xor_sync(0xffffffffu, key[q], j);
          const bool asc = ((32 * q + lane) & k) == 0;
          const bool lower = (lane & j) == 0;
          key[q] = (asc == lower) ? min(key[q], o) : max(key[q], o);
        }
      }
    }
  }
}

// Grid ceil(BH * ntile / LU_WARPS), LU_WARPS warps: warp w of block b takes
// tile t = LU_WARPS b + w.
template <int MODE, int DK>
__global__ void __launch_bounds__(LU_WARPS * 32) k_lloyd_update(LuArgs a) {
  constexpr int W = MODE == KM_QUERY ? DK : LL_KW;  // update-row width
  constexpr int VPL = W / 32;                        // update values per lane
  constexpr int INVALID = 0x7fffffff;
  __shared__ float rowf_all[LU_WARPS][LL_TILE];
  __shared__ int keys_all[LU_WARPS][LL_TILE];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * LU_WARPS + warp;
  if (t >= a.BH * a.ntile) return;
  float* rowf = rowf_all[warp];
  const int bh = t / a.ntile, tl = t - bh * a.ntile;
  const int n0 = tl * LL_TILE, nvalid = min(LL_TILE, a.N - n0);
  // keys label << 7 | row; rows past N and out-of-range labels sort last
  int key[4];
  uint32_t mword = 0u;  // this lane's share of the label mask word `lane` (lanes 0-7)
  uint32_t bits[8];
#pragma unroll
  for (int w = 0; w < 8; ++w) bits[w] = 0u;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int rr = 32 * q + lane, n = n0 + rr;
    key[q] = INVALID;
    float f = 0.f;
    if (rr < nvalid) {
      const int g = a.lab[(size_t)bh * a.N + n];
      if (g >= 0 && g < a.G) {
        key[q] = (g << 7) | rr;
#pragma unroll
        for (int w = 0; w < 8; ++w)
          if ((g >> 5) == w) bits[w] |= 1u << (g & 31);
      } else {
        set_error(a.hdr, ERR_INDEX, 9, bh, n);
      }
      if (MODE == KM_QUERY) f = a.scale / a.rms[(size_t)bh * a.N + n];
    }
    if (MODE == KM_QUERY) rowf[rr] = f;
  }
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    const uint32_t m = __reduce_or_sync(0xffffffffu, bits[w]);
    if (lane == w) mword = m;
  }
  if (lane < 8) a.tmask[(size_t)t * 8 + lane] = mword;
  // rows with a label in range (all of them, unless the error word is set)
  int nkeys = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) nkeys += __popc(__ballot_sync(0xffffffffu, key[q] != INVALID));
  warp_sort128(key, lane);
  // the sorted keys, position p = 32 q + lane, for the in-order pass below
  int* keys = keys_all[warp];
#pragma unroll
  for (int q = 0; q < 4; ++q) keys[32 * q + lane] = key[q];
  __syncwarp();  // keys and row factors visible to the whole warp
  // row r of the tile: lane's VPL values at xbase + r * xstride
  const char* xbase;
  int64_t xstride;
  if constexpr (MODE == KM_QUERY) {
    xbase = reinterpret_cast<const char*>(a.X.row(bh, n0) + lane * VPL);
    xstride = a.X.sn * 2;
  } else {
    xbase = reinterpret_cast<const char*>(a.Z + ((size_t)bh * a.N + n0) * LL_KW + lane);
    xstride = LL_KW * 4;
  }
  float acc[VPL];
#pragma unroll
  for (int v = 0; v < VPL; ++v) acc[v] = 0.f;
  int run = -1, run_start = 0, cur_g = -1;
  float* sbase = a.slots + (size_t)t * LL_SLOTS * W + lane * VPL;
  auto flush = [&](int count) {
    float* dst = sbase + (size_t)run * W;
    if (VPL == 4)
      *reinterpret_cast<float4*>(dst) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    else if (VPL == 2)
      *reinterpret_cast<float2*>(dst) = make_float2(acc[0], acc[1]);
    else
      dst[0] = acc[0];
    if (lane == 0) {
      a.slot_cnt[(size_t)t * LL_SLOTS + run] = count;
      atomicOr(a.gbits + ((size_t)bh * a.G + cur_g) * a.nword + (tl >> 5), 1u << (tl & 31));
    }
  };
  // sorted positions in order, UB rows loaded ahead of the sums; a label
  // change in the sorted order starts the next run (slot)
  constexpr int UB = 8;
  for (int p0 = 0; p0 < nkeys; p0 += UB) {
    const int pe = min(UB, nkeys - p0);
    int kk[UB];
    float x[UB][VPL];
#pragma unroll
    for (int e = 0; e < UB; ++e) {
      kk[e] = e < pe ? keys[p0 + e] : keys[p0];
      const char* src = xbase + (int64_t)(kk[e] & 127) * xstride;
      if constexpr (MODE == KM_QUERY && VPL == 4) {  // bf16 -> fp32 is a shift
        const uint2 raw = *reinterpret_cast<const uint2*>(src);
        x[e][0] = __uint_as_float(raw.x << 16);
        x[e][1] = __uint_as_float(raw.x & 0xffff0000u);
        x[e][2] = __uint_as_float(raw.y << 16);
        x[e][3] = __uint_as_float(raw.y & 0xffff0000u);
      } else if constexpr (MODE == KM_QUERY) {
        const uint32_t raw = *reinterpret_cast<const uint32_t*>(src);
        x[e][0] = __uint_as_float(raw << 16);
        x[e][1] = __uint_as_float(raw & 0xffff0000u);
      } else {
        x[e][0] = *reinterpret_cast<const float*>(src);
      }
    }
#pragma unroll
    for (int e = 0; e < UB; ++e) {
      if (e < pe) {
        const int g = kk[e] >> 7;
        if (g != cur_g) {
          if (run >= 0) flush(p0 + e - run_start);
          ++run;
          run_start = p0 + e;
          cur_g = g;
#pragma unroll
          for (int v = 0; v < VPL; ++v) acc[v] = 0.f;
        }
        if constexpr (MODE == KM_QUERY) {
          const float f = rowf[kk[e] & 127];
#pragma unroll
          for (int v = 0; v < VPL; ++v) acc[v] = fmaf(f, x[e][v], acc[v]);
        } else {
          acc[0] += x[e][0];
        }
      }
    }
  }
  if (run >= 0) flush(nkeys - run_start);
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
                                                    float* beta, int ncrows, const float* A,
                                                    bf16* bq, int split_rows) {
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
      const uint4* m4 = reinterpret_cast<const uint4*>(mb + (size_t)tl * 8);
      const uint4 ma = m4[0], mc = m4[1];  // the tile's eight mask words, two loads
      const uint32_t mw[8] = {ma.x, ma.y, ma.z, ma.w, mc.x, mc.y, mc.z, mc.w};
      int rk = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t keep = j < (g >> 5) ? 0xffffffffu : j == (g >> 5) ? (1u << (g & 31)) - 1u : 0u;
        rk += __popc(mw[j] & keep);
      }
      list[i] = tl * LL_SLOTS + rk;
    }
    __syncthreads();
    // two interleaved fp64 chains (even entries into s0, odd into s1, added in
    // order at the end), eight loads in flight ahead of the adds
    int i = 0;
    for (; i + 8 <= n; i += 8) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = sb[(size_t)list[i + u] * W + c];
#pragma unroll
      for (int u = 0; u < 8; u += 2) {
        s0 += (double)v[u];
        s1 += (double)v[u + 1];
      }
    }
    for (; i + 1 < n; i += 2) {
      s0 += (double)sb[(size_t)list[i] * W + c];
      s1 += (double)sb[(size_t)list[i + 1] * W + c];
    }
    if (i < n) s0 += (double)sb[(size_t)list[i] * W + c];
    // rows: one count per listed tile, summed over the block
    int cpart = 0;
    for (int q = c; q < n; q += W) cpart += cb[list[q]];
    int ctot;
    block_exscan_small(cpart, shs, &ctot);
    cnt += ctot;
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
  if (A != nullptr) {
    // query mode: the next assignment's operand row Bq_g = A a_g (A symmetric,
    // j ascending) split into bf16 hi + lo, and beta_g = a_g . Bq_g / 2
    __shared__ float av[W];
    __shared__ float red[W / 32];
    av[c] = v;
    __syncthreads();
    const float* Ab = A + (size_t)bh * W * W;
    float sv = 0.f;
#pragma unroll 16
    for (int j = 0; j < W; ++j) sv += Ab[(size_t)j * W + c] * av[j];
    const bf16 hi = __float2bfloat16_rn(sv);
    const bf16 lo = __float2bfloat16_rn(sv - __bfloat162float(hi));
    bq[(((size_t)bh * 2 + 0) * split_rows + g) * W + c] = hi;
    bq[(((size_t)bh * 2 + 1) * split_rows + g) * W + c] = lo;
    const float t = warp_sum(sv * v);
    if ((c & 31) == 0) red[c >> 5] = t;
    __syncthreads();
    if (c == 0) {
      float q = 0.f;
      for (int w = 0; w < W / 32; ++w) q += red[w];
      beta[(size_t)bh * G + g] = 0.5f * q;
    }
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
  cudaError_t e = cudaFuncSetAttribute(k_lloyd_assign<MODE, DK>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.total);
  if (e != cudaSuccess) return e;
  const int T = a.BH * a.ntile;
  const int grid = T < num_sms() ? T : num_sms();
  spr_launch(k_lloyd_assign<MODE, DK>, grid, LL_THREADS, pl.total, st, tmX, tmB, a);
  return cudaGetLastError();
}

template <int MODE, int DK>
void update_launch(const LuArgs& u, cudaStream_t st) {
  const int T = u.BH * u.ntile;
  spr_launch(k_lloyd_update<MODE, DK>, (T + LU_WARPS - 1) / LU_WARPS, LU_WARPS * 32, 0, st, u);
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
    // bf16 rows z_hi | z_lo: [BH][N][64]
    const uint64_t dims[3] = {64, (uint64_t)s.N, (uint64_t)s.BH};
    const uint64_t str[2] = {128, (uint64_t)s.N * 128};
    const uint32_t box[3] = {64, LL_TILE, 1};
    if (s.Zhl == nullptr || s.Z == nullptr ||
        !encode_tmap(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, s.Zhl, dims, str, box,
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
  a.scale = s.scale;
  a.rms = s.rms;
  a.beta = s.beta;
  a.lab = s.lab;
  a.hdr = s.hdr;
  cudaError_t e;
  if (s.mode == KM_QUERY)
    e = s.d == 64 ? lloyd_launch<KM_QUERY, 64>(tmX, tmB, a, st)
                  : lloyd_launch<KM_QUERY, 128>(tmX, tmB, a, st);
  else
    e = lloyd_launch<KM_KEY, LL_KW>(tmX, tmB, a, st);
  if (e != cudaSuccess) return e;
  // per-tile sums of each label's rows
  LuArgs u{};
  u.N = s.N;
  u.G = s.G;
  u.BH = s.BH;
  u.ntile = ntile;
  u.nword = nword;
  u.scale = s.scale;
  u.X = s.X;
  u.Z = s.Z;
  u.rms = s.rms;
  u.lab = s.lab;
  u.slots = s.slots;
  u.slot_cnt = s.slot_cnt;
  u.tmask = s.tmask;
  u.gbits = s.gbits;
  u.hdr = s.hdr;
  if (s.mode == KM_QUERY) {
    if (s.d == 64)
      update_launch<KM_QUERY, 64>(u, st);
    else
      update_launch<KM_QUERY, 128>(u, st);
  } else {
    update_launch<KM_KEY, LL_KW>(u, st);
  }
  // the update
  const dim3 rg(s.G, s.BH);
  if (s.mode == KM_QUERY) {
    if (s.d == 64)
      spr_launch(k_lloyd_reduce<64>, rg, 64, 0, st, static_cast<const float*>(s.slots),
                 static_cast<const int32_t*>(s.slot_cnt), static_cast<const uint32_t*>(s.tmask),
                 s.gbits, s.G, ntile, nword, s.cent, static_cast<bf16*>(nullptr),
                 s.A ? const_cast<float*>(s.beta) : static_cast<float*>(nullptr), 0, s.A,
                 s.A ? const_cast<bf16*>(s.bq) : static_cast<bf16*>(nullptr), s.split_rows);
    else
      spr_launch(k_lloyd_reduce<128>, rg, 128, 0, st, static_cast<const float*>(s.slots),
                 static_cast<const int32_t*>(s.slot_cnt), static_cast<const uint32_t*>(s.tmask),
                 s.gbits, s.G, ntile, nword, s.cent, static_cast<bf16*>(nullptr),
                 s.A ? const_cast<float*>(s.beta) : static_cast<float*>(nullptr), 0, s.A,
                 s.A ? const_cast<bf16*>(s.bq) : static_cast<bf16*>(nullptr), s.split_rows);
  } else {
    spr_launch(k_lloyd_reduce<LL_KW>, rg, LL_KW, 0, st, static_cast<const float*>(s.slots),
               static_cast<const int32_t*>(s.slot_cnt), static_cast<const uint32_t*>(s.tmask),
               s.gbits, s.G, ntile, nword, s.cent, s.bk, const_cast<float*>(s.beta), NC,
               static_cast<const float*>(nullptr), static_cast<bf16*>(nullptr), 0);
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
