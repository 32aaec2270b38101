// Routed attention on the 5th-generation tensor cores (tcgen05, TMEM, TMA) for
// head dimensions 64 and 128 [paperlayer §1, §4 "Sparse Execution"; App. A.2].
//
// Each work item is a tile of up to 128 query rows (one query group's rows in
// the group-major layout, or 128 gathered probe rows) plus its key ranges (the
// merged K/V groups routed to the query group, or [0, N) for probes).  Every
// row's softmax is renormalised over exactly those keys (hard drop).
//
// One persistent CTA per SM, 12 warps:
//   warp 0      producer: takes the next item from the global cursor and
//               publishes it in a 4-slot shared-memory ring for the other
//               roles; TMA-loads the Q tile once per item and K and V tiles of
//               128 keys into a three-stage ring (128-byte-swizzled boxes).  A
//               key range's first tile starts at its first key rounded down
//               to 8 (see TileIter).
//   warp 1      owns TMEM (S0, S1, O, Q and a few exchange columns) and
//               issues every tensor-core operation from one thread.  With VT
//               (the values stored transposed, the attention stage's layout):
//               Q is copied into TMEM once per item (tcgen05.cp), S = Q K^T
//               takes A from TMEM and B = the K tile, O += P V takes A = P
//               from TMEM (the bf16 probabilities the softmax wrote over S)
//               and B = the transposed value tile, so every operand the
//               tensor cores read is K-major.  Without VT (caller-owned
//               [N, d] values) S reads Q from shared memory and PV reads V as
//               an MN-major B.  S of a tile whose key range ends early is
//               computed only up to its last 16-key block; PV always covers
//               the tile's 128 keys (P is zero past the valid ones), so that
//               each group of products issues as straight-line code.
//   warps 2, 3  idle.
//   warps 4..11 the softmax, two warps per scheduler: warps 4 + q and 8 + q
//               hold rows 32q .. 32q + 31 (their TMEM lanes), the first keys
//               0 .. 63 of every tile, the second keys 64 .. 127.  Per tile:
//               masked half-row max, agreed with the partner through TMEM and
//               a pair barrier; exp2, row sums, P back to TMEM; O is rescaled
//               in TMEM only when the running max grows by more than 2^8 (the
//               final normalisation uses the same stale max, so this is
//               exact); per item the pair adds its row sums and each writes
//               its half of O / l to global memory.
// Every mbarrier wait is bounded in time; a wait that runs out sets an abort
// flag that ends every role, the device error word records a timeout, copies
// and MMAs in flight are drained, and TMEM is freed.  TMEM loads and stores
// are warp-collective, so the softmax warps reconverge before each one.
#include <cudaTypedefs.h>
#include <stdlib.h>
#include <string.h>

#include "tc_sm100.cuh"

namespace spr {

namespace {

constexpr int TBM = 128, TBN = 128;  // query rows and keys per tile
constexpr int NST = 3;                         // K/V pipeline stages
constexpr int NITQ = 4;                        // item ring slots
constexpr uint32_t BOX_BYTES = TBN * 64 * 2;   // one 64-column swizzled box: 16 KB
constexpr uint32_t S_COL0 = 0, S_COL1 = 128, O_COL = 256, Q_COL = 384, X_COL = 448, TMEM_COLS = 512;
constexpr int ATT_THREADS = 384;  // producer, MMA issuer, two idle warps, eight softmax warps
constexpr uint64_t WAIT_NS = 2000000000ull;  // 2 s
// one Q, K or V tile of head dimension TD (TD / 64 boxes) and the CTA's shared memory
template <int TD>
__host__ __device__ constexpr uint32_t tile_bytes() { return TBN * TD * 2; }
template <int TD>
__host__ __device__ constexpr size_t smem_bytes() { return 1024 + (1 + 2 * NST) * (size_t)tile_bytes<TD>() + 512; }

struct TcArgs {
  const int4* items;
  const int32_t* runptr;
  const int2* runs;
  int N, M, Gq, Gk;
  float scale_log2;
  float* osp;
  float* odn;
  Header* hdr;
  spr_head_stats* stats;
};

// Key tiles of one item: for each key range [x, y), the first tile starts at x
// rounded down to 8 keys, the next ones 128 keys apart.  The transposed values
// are addressed by key, and a tile's first key must sit on a 16-byte boundary;
// the first lo keys of a range's first tile lie before the range and are
// masked.  Both value layouts use the same tiles, so that they sum in the same
// order.  The range after the current one is loaded when the current one
// starts, so that moving to it waits on no global load.
struct TileIter {
  const int2* runs;
  int r, rend, t0, lo;
  int2 run, nxt;
  bool valid;
  __device__ void start_run() {
    t0 = run.x & ~7;
    lo = run.x - t0;
  }
  __device__ void init(const TcArgs& a, const int4& it) {
    runs = nullptr;
    r = 0;
    rend = 1;
    run = make_int2(0, a.N);
    nxt = make_int2(0, 0);
    if (it.w >= 0) {
      r = a.runptr[(size_t)it.x * (a.Gq + 1) + it.w];
      rend = a.runptr[(size_t)it.x * (a.Gq + 1) + it.w + 1];
      runs = a.runs + (size_t)it.x * a.Gq * a.Gk;
      run = r < rend ? runs[r] : make_int2(0, 0);
      if (r + 1 < rend) nxt = runs[r + 1];
    }
    start_run();
    valid = r < rend && run.x < run.y;
  }
  __device__ int nvalid() const { return min(TBN, run.y - t0); }
  __device__ void next() {
    t0 += TBN;
    lo = 0;
    if (t0 >= run.y) {
      ++r;
      if (r < rend) {
        run = nxt;
        start_run();
        if (r + 1 < rend) nxt = runs[r + 1];
      } else {
        valid = false;
      }
    }
  }
};

__device__ __forceinline__ uint32_t f2u(float f) { return __float_as_uint(f); }

// Packed two-lane fp32 arithmetic (sm_100): one instruction for two scores.
__device__ __forceinline__ void fma2(float& d0, float& d1, float a0, float a1, float b, float c) {
  asm("{\n.reg .b64 ra, rb, rc, rd;\n"
      "mov.b64 ra, {%2, %3};\nmov.b64 rb, {%4, %4};\nmov.b64 rc, {%5, %5};\n"
      "fma.rn.ftz.f32x2 rd, ra, rb, rc;\nmov.b64 {%0, %1}, rd;\n}\n"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b), "f"(c));
}
__device__ __forceinline__ void add2(float& d0, float& d1, float a0, float a1) {
  asm("{\n.reg .b64 ra, rd;\n"
      "mov.b64 ra, {%2, %3};\nmov.b64 rd, {%0, %1};\n"
      "add.rn.ftz.f32x2 rd, rd, ra;\nmov.b64 {%0, %1}, rd;\n}\n"
      : "+f"(d0), "+f"(d1)
      : "f"(a0), "f"(a1));
}
// three-input maximum (sm_100)
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// VT: the values are transposed, [BH][d][vt_ld(N)] (tmV maps them), Q is copied
// into TMEM and both products take their A operand from TMEM and a K-major B
// from shared memory.  Without VT the values are [BH][N][d] and PV reads them
// as an MN-major B: a stream that mixes K-major and MN-major operands runs the
// tensor cores at about half rate.
template <int TD, bool VT>
__global__ void __launch_bounds__(ATT_THREADS, 1)
    k_attend_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQprobe,
                const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                TcArgs a) {
  constexpr uint32_t TILE_BYTES = tile_bytes<TD>();
  constexpr int NBOX = TD / 64;  // 64-column boxes per row
  constexpr uint32_t VBOX = TD * 128;  // VT: one box of 64 keys x TD rows of the transposed values
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = base;
  uint8_t* sKV = base + TILE_BYTES;  // stage s: K at sKV + 2s tiles, V right after
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + (1 + 2 * NST) * TILE_BYTES);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* kv_full = bars + 2;         // [NST]
  uint64_t* kv_empty = bars + 2 + NST;  // [NST]
  uint64_t* s_full = bars + 2 + 2 * NST;   // [2]
  uint64_t* p_full = bars + 4 + 2 * NST;   // [2]
  uint64_t* o_done = bars + 6 + 2 * NST;   // [2]: PV(g) of the g-th tile commits o_done[g & 1]
  uint64_t* o_free = bars + 8 + 2 * NST;
  uint64_t* drain = bars + 9 + 2 * NST;
  uint64_t* it_full = bars + 10 + 2 * NST;           // [NITQ]
  uint64_t* it_empty = bars + 10 + 2 * NST + NITQ;   // [NITQ]
  uint64_t* pair_bar = bars + 10 + 2 * NST + 2 * NITQ;      // [4] softmax pairs, once per tile
  uint64_t* ep_bar = bars + 14 + 2 * NST + 2 * NITQ;        // [4] softmax pairs, once per item
  int* it_ring = reinterpret_cast<int*>(bars + 18 + 2 * NST + 2 * NITQ);  // [NITQ]
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(it_ring + NITQ);
  volatile int* abort_s = reinterpret_cast<volatile int*>(tmem_base_s + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = a.hdr->n_items;
  if (threadIdx.x == 0) {
    tc::mbar_init(q_full, 1);
    tc::mbar_init(q_empty, 1);
    for (int s = 0; s < NST; ++s) {
      tc::mbar_init(kv_full + s, 1);
      tc::mbar_init(kv_empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(s_full + s, 1);
      tc::mbar_init(p_full + s, 256);
    }
    for (int s = 0; s < NITQ; ++s) {
      tc::mbar_init(it_full + s, 1);
      tc::mbar_init(it_empty + s, 1 + 256);  // the MMA thread and every softmax thread
    }
    for (int s = 0; s < 4; ++s) {
      tc::mbar_init(pair_bar + s, 64);
      tc::mbar_init(ep_bar + s, 64);
    }
    tc::mbar_init(o_done, 1);
    tc::mbar_init(o_done + 1, 1);
    tc::mbar_init(o_free, 256);
    tc::mbar_init(drain, 1);
    *abort_s = 0;
    tc::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tc::prefetch_tmap(&tmQ);
    tc::prefetch_tmap(&tmQprobe);
    tc::prefetch_tmap(&tmK);
    tc::prefetch_tmap(&tmV);
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_base_s, TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = *tmem_base_s;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int kv = 0, q_loads = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int slot = k % NITQ;
        if (k >= NITQ && !tc::mbar_wait(it_empty + slot, ((k / NITQ) - 1) & 1, abort_s, WAIT_NS))
          break;
        const int item = (int)atomicAdd(&a.hdr->work_next, 1u);
        it_ring[slot] = item;
        tc::mbar_arrive(it_full + slot);
        if (item >= n_items) break;
        const int4 it = a.items[item];
        TileIter I;
        I.init(a, it);
        if (k > 0 && !tc::mbar_wait(q_empty, (k - 1) & 1, abort_s, WAIT_NS)) break;
        tc::mbar_expect_tx(q_full, TILE_BYTES);
        const CUtensorMap* qm = it.w >= 0 ? &tmQ : &tmQprobe;
        const int qrow = it.w >= 0 ? it.x * a.N + it.y : it.x * a.M + it.y;
        for (int j = 0; j < NBOX; ++j)
          tc::tma_load_2d(sQ + j * BOX_BYTES, qm, 64 * j, qrow, q_full);
        ++q_loads;
        for (; I.valid; I.next(), ++kv) {
          const int s = kv % NST;
          if (kv >= NST &&
              !tc::mbar_wait(kv_empty + s, ((kv / NST) - 1) & 1, abort_s, WAIT_NS)) {
            ok = false;
            break;
          }
          uint8_t* kd = sKV + (size_t)(2 * s) * TILE_BYTES;
          uint8_t* vd = kd + TILE_BYTES;
          tc::mbar_expect_tx(kv_full + s, 2 * TILE_BYTES);
          const int krow = it.x * a.N + I.t0;
          for (int j = 0; j < NBOX; ++j) {
            tc::tma_load_2d(kd + j * BOX_BYTES, &tmK, 64 * j, krow, kv_full + s);
            if (!VT) tc::tma_load_2d(vd + j * BOX_BYTES, &tmV, 64 * j, krow, kv_full + s);
          }
          if (VT)  // keys t0 .. t0 + 127 of the TD rows of this head (t0 is a multiple of 8)
            for (int j = 0; j < 2; ++j)
              tc::tma_load_2d(vd + j * VBOX, &tmV, I.t0 + 64 * j, it.x * TD, kv_full + s);
        }
      }
      if (*abort_s) {  // let our copies in flight land before the block exits
        for (int k = kv - NST; k < kv; ++k)
          if (k >= 0) tc::mbar_wait_bounded(kv_full + (k % NST), (k / NST) & 1, 100000000ull);
        if (q_loads > 0) tc::mbar_wait_bounded(q_full, (q_loads - 1) & 1, 100000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // The issuing thread shares its scheduler with a softmax warp, so its
      // per-tile instruction count bounds the product stream: descriptors are
      // formed once and advanced by constant offsets (the start address field
      // is address >> 4 and never carries), and stages and phases rotate.
      constexpr uint32_t STAGE_D = (2 * TILE_BYTES) >> 4;  // descriptor step between stages
      const uint64_t qdesc = tc::smem_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t kdesc0 = tc::smem_desc_sw128(smem_u32(sKV), 16, 1024);
      const uint64_t vdesc0 = VT ? tc::smem_desc_sw128(smem_u32(sKV + TILE_BYTES), 16, 1024)
                                 : tc::smem_desc_sw128(smem_u32(sKV + TILE_BYTES), BOX_BYTES, 1024);
      const uint32_t idPV = tc::idesc_bf16(TBM, TD, VT ? 0 : 1);
      int ss = 0, ps = 0;          // K/V stage of the next S and the next PV product
      uint32_t sph = 0;            // kv_full phase of stage ss
      uint32_t sb = 0, pb = 0;     // S buffer of the next S and of the next PV product
      uint32_t pbph = 0;           // p_full phase of buffer pb
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int slot = k % NITQ;
        if (!tc::mbar_wait(it_full + slot, (k / NITQ) & 1, abort_s, WAIT_NS)) break;
        const int item = it_ring[slot];
        tc::mbar_arrive(it_empty + slot);
        if (item >= n_items) break;
        const int4 it = a.items[item];
        TileIter Is, Ip;
        Is.init(a, it);
        Ip.init(a, it);
        if (!tc::mbar_wait(q_full, k & 1, abort_s, WAIT_NS)) break;
        if (VT) {  // Q into TMEM; its shared-memory tile is free once copied
          tc::tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < TD / 16; ++ks)
            tc::tmem_cp_128x256b(tbase + Q_COL + ks * 8,
                                 qdesc + (((ks >> 2) * BOX_BYTES + (ks & 3) * 32) >> 4));
          tc::mma_commit(q_empty);
        }
        auto issue_s = [&]() -> bool {
          if (!tc::mbar_wait(kv_full + ss, sph, abort_s, WAIT_NS)) return false;
          tc::tc_fence_after();
          const uint32_t idS = tc::idesc_bf16(TBM, (Is.nvalid() + 15) & ~15, 0);
          const uint32_t d = tbase + sb * S_COL1;
          const uint64_t kd = kdesc0 + (uint64_t)(ss * STAGE_D);
#pragma unroll
          for (int ks = 0; ks < TD / 16; ++ks) {
            const uint32_t off = ((ks >> 2) * BOX_BYTES + (ks & 3) * 32) >> 4;
            if (VT)
              tc::mma_ts(d, tbase + Q_COL + ks * 8, kd + off, idS, ks > 0);
            else
              tc::mma_ss(d, qdesc + off, kd + off, idS, ks > 0);
          }
          tc::mma_commit(s_full + sb);
          if (++ss == NST) {
            ss = 0;
            sph ^= 1u;
          }
          sb ^= 1u;
          return true;
        };
        for (int j = 0; j < 2 && Is.valid && ok; ++j) {
          ok = issue_s();
          Is.next();
        }
        bool first = true;
        for (; Ip.valid && ok; Ip.next()) {
          if (!tc::mbar_wait(p_full + pb, pbph, abort_s, WAIT_NS)) {
            ok = false;
            break;
          }
          if (first && k > 0 && !tc::mbar_wait(o_free, (k - 1) & 1, abort_s, WAIT_NS)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint64_t vd = vdesc0 + (uint64_t)(ps * STAGE_D);
          const uint32_t p_col = tbase + pb * S_COL1;
          // every 16-key block of the tile, as straight-line code (a branch
          // between products slows their issue); P is zero past the valid keys
#pragma unroll
          for (int kk = 0; kk < TBN / 16; ++kk) {
            const uint32_t voff = VT ? ((kk >> 2) * VBOX + (kk & 3) * 32) >> 4 : kk * (2048 >> 4);
            tc::mma_ts(tbase + O_COL, p_col + kk * 8, vd + voff, idPV, !(first && kk == 0));
          }
          tc::mma_commit(kv_empty + ps);
          tc::mma_commit(o_done + pb);
          first = false;
          if (++ps == NST) ps = 0;
          pb ^= 1u;
          if (pb == 0) pbph ^= 1u;
          if (Is.valid) {
            ok = issue_s();
            Is.next();
          }
        }
        if (!VT) tc::mma_commit(q_empty);  // the last S product has read the Q tile
      }
      // drain: every MMA issued so far completes before TMEM is released
      tc::mma_commit(drain);
      tc::mbar_wait_bounded(drain, 0, WAIT_NS);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    // Two warps per quarter of the rows: warps 4 + q and 8 + q both hold rows
    // 32q .. 32q + 31 (their TMEM lanes); the first takes keys 0 .. 63 of
    // every tile, the second keys 64 .. 127, so that each scheduler runs two
    // softmax warps and one's bookkeeping overlaps the other's exponentials.
    // The pair agrees on each tile's row max, and adds its row sums at the
    // end of an item, through TMEM columns X_COL.. and a pair barrier.
    const int q = warp & 3, hh = (warp - 4) >> 2;               // row quarter, key half
    const int row = 32 * q + lane;                              // query row in the tile
    const uint32_t lane_f = (uint32_t)(q * 32) << 16;           // TMEM lane field
    const uint32_t xcol = tbase + lane_f + X_COL;
    constexpr int OH = TD / 2;                                  // O columns of one half
    int pg = 0;  // tiles this CTA has processed: the g of the tile below
    int ng = 0;  // items with tiles this CTA has processed
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int slot = k % NITQ;
      const bool got_it = tc::mbar_wait(it_full + slot, (k / NITQ) & 1, abort_s, WAIT_NS);
      __syncwarp();
      if (!__all_sync(0xffffffffu, got_it)) break;
      const int item = it_ring[slot];
      tc::mbar_arrive(it_empty + slot);
      if (item >= n_items) break;
      const int4 it = a.items[item];
      TileIter I;
      I.init(a, it);
      float m = -INFINITY, l = 0.f;
      bool first = true;
      int ntiles = 0;
      unsigned long long exec_pairs = 0;
      for (; I.valid; I.next(), ++pg, ++ntiles) {
        const int b = pg & 1;
        const uint32_t scol = tbase + lane_f + (b ? S_COL1 : S_COL0);
        const int nvalid = I.nvalid();
        exec_pairs += (unsigned long long)TBM * ((nvalid + 15) & ~15);
        const int nch = (nvalid + 31) >> 5;  // 32-key chunks holding valid keys
        const bool got_s = tc::mbar_wait(s_full + b, (pg >> 1) & 1, abort_s, WAIT_NS);
        __syncwarp();  // TMEM loads and stores below are warp-collective
        if (!__all_sync(0xffffffffu, got_s)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        uint32_t sr[64];  // keys 64 hh .. 64 hh + 63 of the tile
#pragma unroll
        for (int c = 0; c < 2; ++c)
          if (2 * hh + c < nch) tc::tmem_ld32(scol + 64 * hh + 32 * c, sr + 32 * c);
        tc::tmem_wait_ld();
        // keys past the tile's valid count, and keys before the range in its
        // first, 8-aligned tile, are masked to -inf
        if (nvalid < 64 * hh + 64) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (64 * hh + c >= nvalid) sr[c] = f2u(-INFINITY);
        }
        if (hh == 0 && I.lo > 0) {
#pragma unroll
          for (int c = 0; c < 8; ++c)
            if (c < I.lo) sr[c] = f2u(-INFINITY);
        }
        // max of the raw scores of this half (the scale is positive)
        float mx8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          mx8[e] = fmaxf(__uint_as_float(sr[e]), __uint_as_float(sr[e + 8]));
#pragma unroll
        for (int c = 16; c < 64; c += 16)
#pragma unroll
          for (int e = 0; e < 8; ++e)
            mx8[e] = max3(mx8[e], __uint_as_float(sr[c + e]), __uint_as_float(sr[c + 8 + e]));
        const float mxh = fmaxf(max3(mx8[0], mx8[1], mx8[2]),
                                max3(max3(mx8[3], mx8[4], mx8[5]), mx8[6], mx8[7]));
        // exchange with the other half of the row: column X_COL + 2 b + hh
        // holds this half's max of tile g; it is next written at tile g + 2,
        // after the pair barrier of tile g + 1, which needs this thread's
        // read below
        __syncwarp();
        tc::tmem_st1(xcol + 2 * b + hh, f2u(mxh));
        tc::tmem_wait_st();
        tc::tc_fence_before();
        tc::mbar_arrive(pair_bar + q);
        const bool got_x = tc::mbar_wait(pair_bar + q, pg & 1, abort_s, WAIT_NS);
        __syncwarp();
        if (!__all_sync(0xffffffffu, got_x)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        const float mxo = __uint_as_float(tc::tmem_ld1(xcol + 2 * b + (1 - hh)));
        tc::tmem_wait_ld();
        const float mx = fmaxf(mxh, mxo) * a.scale_log2;  // the same value in both halves
        const float mn = fmaxf(m, mx);
        float m_use = m;
        bool rescale = false;
        if (first || mn > m + 8.f) {
          m_use = mn;
          rescale = !first;
        }
        const float corr = rescale ? ex2(m - m_use) : 1.f;
        const float neg = -m_use;
        float sum4[4] = {0.f, 0.f, 0.f, 0.f};
        if (64 * hh < nvalid) {  // uniform across the warp: one tile for all rows
          uint32_t pr[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            float x0, x1;
            fma2(x0, x1, __uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1]),
                 a.scale_log2, neg);
            const float p0 = ex2(x0), p1 = ex2(x1);
            add2(sum4[2 * (c & 1)], sum4[2 * (c & 1) + 1], p0, p1);
            pr[c] = pack_bf16(p0, p1);
          }
          __syncwarp();
          tc::tmem_st32(scol + 32 * hh, pr);
        } else {  // no valid key in this half: P = 0 for the PV product
          uint32_t z[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) z[c] = 0u;
          __syncwarp();
          tc::tmem_st32(scol + 32 * hh, z);
        }
        const float sum = (sum4[0] + sum4[1]) + (sum4[2] + sum4[3]);
        // P(g) is released without waiting for PV(g - 1): only a rescale of O
        // has to wait for it.  Waiting here for PV(g - 2), done long before,
        // keeps at most two phases of o_done[g & 1] in play, so that every
        // parity wait on it (here, the rescale's and the epilogue's) is exact.
        if (pg >= 2) {
          const bool got = tc::mbar_wait(o_done + (pg & 1), ((pg - 2) >> 1) & 1, abort_s, WAIT_NS);
          __syncwarp();
          if (!__all_sync(0xffffffffu, got)) {
            ok = false;
            break;
          }
        }
        // the rescale is per row, the TMEM access per warp: a warp rescales
        // its half of O's columns when any of its rows needs it (the others
        // multiply by 1; both halves of a row decide alike), once PV(g - 1)
        // has finished accumulating into O
        if (__any_sync(0xffffffffu, rescale)) {
          const bool got_o =
              tc::mbar_wait(o_done + ((pg - 1) & 1), ((pg - 1) >> 1) & 1, abort_s, WAIT_NS);
          __syncwarp();
          if (!__all_sync(0xffffffffu, got_o)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
#pragma unroll
          for (int c = 0; c < OH / 32; ++c) {
            uint32_t o[32];
            __syncwarp();
            tc::tmem_ld32(tbase + lane_f + O_COL + OH * hh + 32 * c, o);
            tc::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = f2u(__uint_as_float(o[e]) * corr);
            __syncwarp();
            tc::tmem_st32(tbase + lane_f + O_COL + OH * hh + 32 * c, o);
          }
        }
        l = l * corr + sum;
        m = m_use;
        __syncwarp();
        tc::tmem_wait_st();
        tc::tc_fence_before();
        tc::mbar_arrive(p_full + b);
        first = false;
      }
      if (!ok) break;
      if (ntiles == 0) {  // keep one o_free phase per item
        tc::mbar_arrive(o_free);
        continue;
      }
      const int gl = pg - 1;  // the item's last tile: its PV completes after all others
      const bool got_o = tc::mbar_wait(o_done + (gl & 1), (gl >> 1) & 1, abort_s, WAIT_NS);
      __syncwarp();
      if (!__all_sync(0xffffffffu, got_o)) {
        ok = false;
        break;
      }
      // the row sum of both halves (column X_COL + 4 + hh, next written at the
      // next item's end, after this item's pair barrier has been passed by both)
      __syncwarp();
      tc::tmem_st1(xcol + 4 + hh, f2u(l));
      tc::tmem_wait_st();
      tc::tc_fence_before();
      tc::mbar_arrive(ep_bar + q);
      const bool got_e = tc::mbar_wait(ep_bar + q, ng & 1, abort_s, WAIT_NS);
      __syncwarp();
      if (!__all_sync(0xffffffffu, got_e)) {
        ok = false;
        break;
      }
      ++ng;
      tc::tc_fence_after();
      const float lo_ = __uint_as_float(tc::tmem_ld1(xcol + 4 + (1 - hh)));
      tc::tmem_wait_ld();
      const float lt = hh == 0 ? l + lo_ : lo_ + l;  // the same sum in both halves
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      float* dst = (it.w >= 0 ? a.osp + ((size_t)it.x * a.N + it.y + row) * TD
                              : a.odn + ((size_t)it.x * a.M + it.y + row) * TD) +
                   OH * hh;
#pragma unroll
      for (int c = 0; c < OH / 32; ++c) {
        uint32_t o[32];
        __syncwarp();
        tc::tmem_ld32(tbase + lane_f + O_COL + OH * hh + 32 * c, o);
        tc::tmem_wait_ld();
        if (row < it.z) {
          float4* d4 = reinterpret_cast<float4*>(dst + 32 * c);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            d4[e] = make_float4(__uint_as_float(o[4 * e]) * inv, __uint_as_float(o[4 * e + 1]) * inv,
                                __uint_as_float(o[4 * e + 2]) * inv,
                                __uint_as_float(o[4 * e + 3]) * inv);
        }
      }
      tc::tc_fence_before();
      tc::mbar_arrive(o_free);
      if (row == 0 && hh == 0)
        atomicAdd(reinterpret_cast<unsigned long long*>(&a.stats[it.x].tile_pairs), exec_pairs);
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (threadIdx.x == 0 && *abort_s) set_error(a.hdr, ERR_TIMEOUT, blockIdx.x, 0, 0);
  if (warp == 1) {
    __syncwarp();  // lane 0 comes from the MMA loop, the others from the barrier
    tc::tmem_dealloc(tbase, TMEM_COLS);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// Row-major [rows, 128] bf16 tensor, 64 x 128 boxes, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* ptr, uint64_t rows, int TD) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)TD, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)TD * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)TBN};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Transposed values [BH * TD rows][ld keys] (ld a multiple of 8), boxes of 64
// keys x TD rows, 128-byte swizzle.
bool make_map_vt(CUtensorMap* m, const void* ptr, uint64_t BH, int TD, uint64_t ld) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)ld, (cuuint64_t)(BH * TD)};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)TD};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// The tcgen05 path serves d = 64 and 128 unless SPR_ATTEND=mma selects the
// mma.sync kernel (kept for side-by-side checks).
bool attend_tc_enabled(int d) {
  if (d != 64 && d != 128) return false;
  const char* e = getenv("SPR_ATTEND");
  return !(e && strcmp(e, "mma") == 0);
}

cudaError_t attend_tc_preload() {
  if (!get_encode()) return cudaErrorInvalidValue;
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, k_attend_tc<64, false>);
  if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, k_attend_tc<128, false>);
  if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, k_attend_tc<64, true>);
  return e != cudaSuccess ? e : cudaFuncGetAttributes(&fa, k_attend_tc<128, true>);
}

cudaError_t launch_attend_tc(const spr_params& p, const Layout& L, const Ptrs& P,
                             cudaStream_t st) {
  CUtensorMap mQ, mQp, mK, mV;
  const uint64_t rows = (uint64_t)L.BH * p.N;
  const bool vt = P.Vt != nullptr;
  if (!make_map(&mQ, P.Qp, rows, p.d) || !make_map(&mK, P.Kp, rows, p.d) ||
      !(vt ? make_map_vt(&mV, P.Vt, (uint64_t)L.BH, p.d, (uint64_t)vt_ld(p.N))
           : make_map(&mV, P.Vp, rows, p.d)))
    return cudaErrorInvalidValue;
  if (!make_map(&mQp, P.qprobe, (uint64_t)L.BH * (p.M > 0 ? p.M : 1), p.d))
    return cudaErrorInvalidValue;
  TcArgs a;
  a.items = P.items;
  a.runptr = P.runptr;
  a.runs = P.runs;
  a.N = p.N;
  a.M = p.M;
  a.Gq = p.Gq;
  a.Gk = p.Gk;
  const float scale = p.scale > 0.f ? p.scale : 1.f / sqrtf((float)p.d);
  a.scale_log2 = scale * 1.4426950408889634f;
  a.osp = P.osp;
  a.odn = P.odn;
  a.hdr = P.hdr;
  a.stats = P.stats;
  auto go = [&](auto kern, size_t smem) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    spr_launch(kern, num_sms(), ATT_THREADS, smem, st, mQ, mQp, mK, mV, a);
    return cudaSuccess;
  };
  cudaError_t e;
  if (p.d == 64)
    e = vt ? go(k_attend_tc<64, true>, smem_bytes<64>()) : go(k_attend_tc<64, false>, smem_bytes<64>());
  else
    e = vt ? go(k_attend_tc<128, true>, smem_bytes<128>())
           : go(k_attend_tc<128, false>, smem_bytes<128>());
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace spr
