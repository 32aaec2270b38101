// Query-response RMS on the tensor cores [paperlayer App. B.2, C.1] for head
// dimensions 64 and 128.
//
// u = s C~ q has ||u||^2 = s^2 q^T A q with A = C~^T C~ (d x d, symmetric),
// so every row needs one quadratic form: rms = sqrt(s^2 q^T A q / G'_k +
// 1e-6) (G'_k nonempty K/V groups) and ||u_hat||^2 = s^2 q^T A q / rms^2.
//
// k_rms_tc is persistent, one CTA per SM over a contiguous range of the
// flattened (head, 128-row tile) sequence:
//   warp 0 lane 0   TMA: the head's A as bf16 hi and lo rows (d / 64 boxes of
//                   64 columns each) and the query tiles ([B, H, N, d] view,
//                   strided) into a 4-stage ring;
//   warp 1          owns TMEM (two d-column buffers); one thread issues
//                   T = q A_hi + q A_lo (tcgen05.mma kind::f16, bf16
//                   operands, fp32 accumulation; q is exact in bf16, the
//                   split carries ~16 bits of A);
//   warps 4-7       one thread per row (= TMEM lane): q^T A q = sum_j T_j q_j
//                   in fp32 (j ascending, q from the tile in shared memory),
//                   rms and ||u_hat||^2 to global memory, and per warp the
//                   fp64 sum of ||u_hat||^2 over its 32 rows of the tile.
// k_un2_chunks adds those per-warp sums, in tile then warp order, into the
// 512-row chunk sums of the query objective.
// Every mbarrier wait is bounded; a wait that runs out sets an abort flag
// that ends every role, the error word records a timeout, copies and
// products in flight are drained and TMEM is freed.
#include "spr_internal.cuh"
#include "tc_sm100.cuh"

namespace spr {

namespace {

constexpr int RT_TM = 128;
constexpr uint32_t RT_BOX = RT_TM * 128;      // 128 query rows x 64 bf16: 16 KB
constexpr int RT_NS = 4;
constexpr int RT_THREADS = 256;
constexpr uint64_t RT_WAIT_NS = 2000000000ull;
// per head dimension D: a query tile is D / 64 boxes, A (D x D) is D / 64
// boxes of D rows x 64 columns
template <int D>
__host__ __device__ constexpr uint32_t rt_qtile() { return (D / 64) * RT_BOX; }
template <int D>
__host__ __device__ constexpr uint32_t rt_abox() { return D * 128; }
template <int D>
__host__ __device__ constexpr size_t rt_smem() {
  return 1024 + 2 * (size_t)(D / 64) * rt_abox<D>() + (size_t)RT_NS * rt_qtile<D>() + 256;
}

struct RtArgs {
  int N, BH, H, ntile;
  float scale;
  const spr_head_stats* stats;
  float* rms;
  float* un2;
  double* tpart;   // [BH * ntile][4] per-warp sums of ||u_hat||^2
  Header* hdr;
};

__device__ __forceinline__ uint32_t rt_swz(int r, int q) {  // 16-byte chunk q of row r
  return (uint32_t)(r * 128 + (((q ^ r) & 7) << 4));
}

template <int D>
__global__ void __launch_bounds__(RT_THREADS, 1)
    k_rms_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmA,
             RtArgs a) {
  extern __shared__ uint8_t rt_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(rt_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  constexpr int NB = D / 64;
  constexpr uint32_t QTILE = rt_qtile<D>(), ABOX = rt_abox<D>(), ATILE = NB * ABOX;
  uint8_t* Ah = sm;                    // A hi: NB boxes
  uint8_t* Al = sm + ATILE;            // A lo: NB boxes
  uint8_t* Qs = sm + 2 * ATILE;        // [RT_NS] tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(Qs + RT_NS * QTILE);
  uint64_t* q_full = bars;             // [4]
  uint64_t* q_empty = bars + 4;        // [4]
  uint64_t* t_full = bars + 8;         // [2]
  uint64_t* t_free = bars + 10;        // [2]
  uint64_t* a_full = bars + 12;
  uint64_t* a_free = bars + 13;
  uint64_t* drain = bars + 14;
  uint32_t* tmem_s = reinterpret_cast<uint32_t*>(bars + 15);
  volatile int* abort_s = reinterpret_cast<volatile int*>(tmem_s + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = a.BH * a.ntile;
  const int tb = (int)(((int64_t)blockIdx.x * T) / gridDim.x);
  const int te = (int)(((int64_t)(blockIdx.x + 1) * T) / gridDim.x);
  auto head_of = [&](int t) { return t / a.ntile; };

  if (tid == 0) {
    for (int s = 0; s < RT_NS; ++s) {
      tc::mbar_init(q_full + s, 1);
      tc::mbar_init(q_empty + s, 4);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(t_full + s, 1);
      tc::mbar_init(t_free + s, 4);
    }
    tc::mbar_init(a_full, 1);
    tc::mbar_init(a_free, 1);
    tc::mbar_init(drain, 1);
    *abort_s = 0;
    tc::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tc::prefetch_tmap(&tmQ);
    tc::prefetch_tmap(&tmA);
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_s, 2 * D);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = *tmem_s;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int k = 0, na = 0, loads = 0;
      for (int t = tb; t < te; ++t, ++k) {
        const int bh = head_of(t), tl = t - bh * a.ntile;
        if (t == tb || bh != head_of(t - 1)) {  // this head's A, hi and lo
          if (na > 0 && !tc::mbar_wait(a_free, (na - 1) & 1, abort_s, RT_WAIT_NS)) break;
          tc::mbar_expect_tx(a_full, 2 * ATILE);
          for (int h = 0; h < 2; ++h)
            for (int j = 0; j < NB; ++j)
              tc::tma_load_3d((h ? Al : Ah) + j * ABOX, &tmA, 64 * j, 0, 2 * bh + h, a_full);
          ++na;
        }
        const int s = k % RT_NS;
        if (k >= RT_NS &&
            !tc::mbar_wait(q_empty + s, ((k / RT_NS) - 1) & 1, abort_s, RT_WAIT_NS))
          break;
        tc::mbar_expect_tx(q_full + s, QTILE);
        const int bb = bh / a.H, hh = bh - bb * a.H;
        for (int j = 0; j < NB; ++j)
          tc::tma_load_4d(Qs + s * QTILE + j * RT_BOX, &tmQ, 64 * j, tl * RT_TM, hh, bb,
                          q_full + s);
        ++loads;
      }
      if (*abort_s) {  // let the copies in flight land before the block exits
        for (int q = loads - RT_NS; q < loads; ++q)
          if (q >= 0) tc::mbar_wait_bounded(q_full + (q % RT_NS), (q / RT_NS) & 1, 100000000ull);
        if (na > 0) tc::mbar_wait_bounded(a_full, (na - 1) & 1, 100000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ products
    if (lane == 0) {
      const uint32_t idesc = tc::idesc_bf16(RT_TM, D, 0);
      const uint32_t ah = smem_u32(Ah), al = smem_u32(Al);
      int k = 0, na = 0;
      for (int t = tb; t < te; ++t, ++k) {
        const int bh = head_of(t);
        const bool hstart = t == tb || bh != head_of(t - 1);
        const bool hend = t + 1 == te || head_of(t + 1) != bh;
        if (hstart) {
          if (!tc::mbar_wait(a_full, na & 1, abort_s, RT_WAIT_NS)) break;
          ++na;
        }
        const int s = k % RT_NS, b = k & 1;
        if (!tc::mbar_wait(q_full + s, (k / RT_NS) & 1, abort_s, RT_WAIT_NS)) break;
        if (k >= 2 && !tc::mbar_wait(t_free + b, ((k >> 1) - 1) & 1, abort_s, RT_WAIT_NS)) break;
        tc::tc_fence_after();
        const uint32_t d = tbase + (uint32_t)(b * D);
        const uint32_t q_addr = smem_u32(Qs + s * QTILE);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (ks >> 2) * RT_BOX + (ks & 3) * 32;   // query tile
          const uint32_t offa = (ks >> 2) * ABOX + (ks & 3) * 32;    // A
          tc::mma_ss(d, tc::smem_desc_sw128(q_addr + off, 16, 1024),
                     tc::smem_desc_sw128(ah + offa, 16, 1024), idesc, ks > 0);
          tc::mma_ss(d, tc::smem_desc_sw128(q_addr + off, 16, 1024),
                     tc::smem_desc_sw128(al + offa, 16, 1024), idesc, 1);
        }
        tc::mma_commit(t_full + b);
        if (hend) tc::mma_commit(a_free);
      }
      tc::mma_commit(drain);  // every product issued so far completes before TMEM is freed
      tc::mbar_wait_bounded(drain, 0, RT_WAIT_NS);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ rows
    const int quarter = warp & 3, r = quarter * 32 + lane;
    const uint32_t lane_f = (uint32_t)(quarter * 32) << 16;
    const float s2 = a.scale * a.scale;
    for (int t = tb, k = 0; t < te; ++t, ++k) {
      const int bh = head_of(t), tl = t - bh * a.ntile;
      const int n = tl * RT_TM + r;
      const bool valid = n < a.N;
      const float gk = (float)max(1, a.stats[bh].gk_nonempty);
      const int s = k % RT_NS, b = k & 1;
      bool got = tc::mbar_wait(t_full + b, (k >> 1) & 1, abort_s, RT_WAIT_NS);
      got = __all_sync(0xffffffffu, got);
      if (!got) break;
      tc::tc_fence_after();
      const uint8_t* qt = Qs + s * QTILE;
      float quad = 0.f;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {  // columns 32c .. 32c + 31
        uint32_t v[32];
        __syncwarp();
        tc::tmem_ld32(tbase + lane_f + (uint32_t)(b * D + 32 * c), v);
        tc::tmem_wait_ld();
        const uint8_t* box = qt + (c >> 1) * RT_BOX;
#pragma unroll
        for (int q = 0; q < 4; ++q) {  // 8 bf16 per 16-byte chunk
          const uint4 w = *reinterpret_cast<const uint4*>(box + rt_swz(r, 4 * (c & 1) + q));
          const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            quad = fmaf(__uint_as_float(v[8 * q + 2 * e]), __uint_as_float(ww[e] << 16), quad);
            quad = fmaf(__uint_as_float(v[8 * q + 2 * e + 1]),
                        __uint_as_float(ww[e] & 0xffff0000u), quad);
          }
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        tc::mbar_arrive(t_free + b);
        tc::mbar_arrive(q_empty + s);
      }
      double u2sum = 0.0;
      if (valid) {
        const float ms = s2 * fmaxf(quad, 0.f) / gk;
        const float rr = sqrtf(ms + 1e-6f);
        const float u2 = s2 * fmaxf(quad, 0.f) / (rr * rr);
        a.rms[(size_t)bh * a.N + n] = rr;
        a.un2[(size_t)bh * a.N + n] = u2;
        u2sum = (double)u2;
      }
      u2sum = warp_sum(u2sum);
      if (lane == 0) a.tpart[(size_t)t * 4 + quarter] = u2sum;
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (tid == 0 && *abort_s) set_error(a.hdr, ERR_TIMEOUT, 22, blockIdx.x, 0);
  if (warp == 1) {
    __syncwarp();
    tc::tmem_dealloc(tbase, 2 * D);
  }
}

// Chunk sums of ||u_hat||^2 for the query objective: chunk c of head bh
// (rows 512 c ..) adds its tiles' per-warp sums in tile, then warp order.
// Grid (nchunk, BH), one thread.
__global__ void k_un2_chunks(const double* tpart, int ntile, int nchunk, double* part) {
  const int c = blockIdx.x, bh = blockIdx.y;
  constexpr int TPC = CHUNK / RT_TM;
  double s = 0.0;
  for (int t = c * TPC; t < min(ntile, (c + 1) * TPC); ++t)
    for (int w = 0; w < 4; ++w) s += tpart[((size_t)bh * ntile + t) * 4 + w];
  part[((size_t)bh * 2 + 1) * (nchunk + 1) + c] = s;
}

}  // namespace

template <int D>
cudaError_t launch_rms_tc_d(const TensorView& Q, int B, int H, int N, int nchunk, int split_rows,
                            const bf16* bsplit, float scale, const spr_head_stats* stats,
                            float* rms, float* un2, double* tpart, double* part, Header* hdr,
                            cudaStream_t st) {
  const int BH = B * H;
  CUtensorMap mQ, mA;
  {
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)N, (uint64_t)H, (uint64_t)B};
    const uint64_t str[3] = {(uint64_t)Q.sn * 2, (uint64_t)Q.sh * 2, (uint64_t)Q.sb * 2};
    const uint32_t box[4] = {64, RT_TM, 1, 1};
    if (!encode_tmap(&mQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, Q.base, dims, str, box,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  {
    // [BH][2][split_rows][d] bf16: rows 0 .. d - 1 of A (hi, then lo)
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)split_rows, (uint64_t)(2 * BH)};
    const uint64_t str[2] = {(uint64_t)D * 2, (uint64_t)split_rows * D * 2};
    const uint32_t box[3] = {64, (uint32_t)D, 1};
    if (split_rows < D ||
        !encode_tmap(&mA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, bsplit, dims, str, box,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  RtArgs a{};
  a.N = N;
  a.BH = BH;
  a.H = H;
  a.ntile = (N + RT_TM - 1) / RT_TM;
  a.scale = scale;
  a.stats = stats;
  a.rms = rms;
  a.un2 = un2;
  a.tpart = tpart;
  a.hdr = hdr;
  cudaError_t e = cudaFuncSetAttribute(k_rms_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)rt_smem<D>());
  if (e != cudaSuccess) return e;
  const int T = BH * a.ntile;
  const int grid = T < num_sms() ? T : num_sms();
  spr_launch(k_rms_tc<D>, grid, RT_THREADS, rt_smem<D>(), st, mQ, mA, a);
  spr_launch(k_un2_chunks, dim3(nchunk, BH), 1, 0, st, static_cast<const double*>(tpart),
             a.ntile, nchunk, part);
  return cudaGetLastError();
}

cudaError_t launch_rms_tc(const TensorView& Q, int B, int H, int N, int D, int nchunk,
                          int split_rows, const bf16* bsplit, float scale,
                          const spr_head_stats* stats, float* rms, float* un2, double* tpart,
                          double* part, Header* hdr, cudaStream_t st) {
  if (D == 64)
    return launch_rms_tc_d<64>(Q, B, H, N, nchunk, split_rows, bsplit, scale, stats, rms, un2,
                               tpart, part, hdr, st);
  if (D == 128)
    return launch_rms_tc_d<128>(Q, B, H, N, nchunk, split_rows, bsplit, scale, stats, rms, un2,
                                tpart, part, hdr, st);
  return cudaErrorInvalidValue;
}

}  // namespace spr
