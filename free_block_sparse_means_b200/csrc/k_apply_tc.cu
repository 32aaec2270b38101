// Residual application on the tensor cores [paperlayer App. A.3; gist-nl §2B]
// for head dimension 128.
//
// The fitted correction of an unprobed row is affine in its hard-drop output
// x (a row of O_sp): y = x + b + (x B) U_r^T = x + b + x W with W = B U_r^T
// (d x d per head).  Probe rows take their exact dense rows instead.  The
// output is bf16 in the original query order.
//
// k_fit_w folds W once per head (W^T, the K-major B operand).  k_apply_tc is
// persistent, one CTA per SM over a contiguous range of the flattened
// (head, 128-row tile) sequence of the permuted rows:
//   warp 0 lane 0   TMA: the head's W^T (4 boxes of 32 fp32 columns) and the
//                   tiles of O_sp (4 such boxes each) into a 2-stage ring;
//   warp 1          owns TMEM (two 128-column buffers); one thread issues
//                   x W as tcgen05.mma kind::tf32 (16 products of K = 8,
//                   fp32 accumulation) into the tile's buffer;
//   warps 4-7       one thread per row (= TMEM lane): x W from TMEM, x from
//                   the tile in shared memory, + b (or the probe's dense
//                   row), bf16 to the row's original position.
// The operands enter the products as tf32 (10-bit mantissa): the correction
// x W carries that rounding, x itself and b are added in fp32, and the
// result is stored in bf16 (8-bit mantissa).
// Every mbarrier wait is bounded; a wait that runs out sets an abort flag
// that ends every role, the error word records a timeout, copies and
// products in flight are drained and TMEM is freed.
#include "spr_internal.cuh"
#include "tc_sm100.cuh"

namespace spr {

namespace {

constexpr int AP_D = 128;
constexpr int AP_TM = 128;                     // rows per tile (the UMMA M)
constexpr uint32_t AP_BOX = AP_TM * 128;       // 128 rows x 32 fp32 (128-byte swizzle): 16 KB
constexpr uint32_t AP_TILE = 4 * AP_BOX;       // 128 x 128 fp32
constexpr int AP_NS = 2;
constexpr int AP_THREADS = 256;
constexpr uint64_t AP_WAIT_NS = 2000000000ull;
constexpr size_t AP_SMEM = 1024 + (size_t)(1 + AP_NS) * AP_TILE + 256;

// instruction descriptor, kind::tf32: fp32 accumulator, tf32 A and B, both
// K-major, M x N
constexpr uint32_t idesc_tf32(int M, int N) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

struct ApArgs {
  const float* odn;       // [BH][M][D] exact dense probe rows
  const int32_t* pslot;   // [BH][N] probe slot of each permuted row, -1 if none
  const int32_t* permq;   // [BH][N] original row of each permuted row
  const float* fitBv;     // [BH][D] intercept b
  int N, M, H, BH, ntile;
  int64_t sb, sh, sn;     // output strides (elements)
  bf16* O;
  Header* hdr;
};

// W^T of head bh: Wt[j][i] = sum_{k < r_eff} B[i][k] U[j][k] (zero without a
// fit).  Grid (D, BH), D threads: block j, thread i.
template <int D>
__global__ void __launch_bounds__(D) k_fit_w(const float* fitB, const float* fitU,
                                             const spr_head_stats* stats, int R, int do_fit,
                                             float* Wt) {
  __shared__ float uj[D];
  const int j = blockIdx.x, bh = blockIdx.y, i = threadIdx.x;
  const int re = do_fit ? min(stats[bh].r_eff, R) : 0;
  uj[i] = i < re ? fitU[((size_t)bh * D + j) * D + i] : 0.f;
  __syncthreads();
  float s = 0.f;
  for (int k = 0; k < re; ++k) s = fmaf(fitB[((size_t)bh * D + i) * D + k], uj[k], s);
  Wt[((size_t)bh * D + j) * D + i] = s;
}

// 16-byte chunk q (fp32 columns 4q .. 4q + 3) of row r in a 128-byte-swizzled box
__device__ __forceinline__ uint32_t ap_swz(int r, int q) {
  return (uint32_t)(r * 128 + (((q ^ r) & 7) << 4));
}

__global__ void __launch_bounds__(AP_THREADS, 1)
    k_apply_tc(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
               ApArgs a) {
  extern __shared__ uint8_t ap_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ap_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint8_t* Ws = sm;                  // W^T: 4 boxes
  uint8_t* Xs = sm + AP_TILE;        // [AP_NS] tiles of 4 boxes
  uint64_t* bars = reinterpret_cast<uint64_t*>(Xs + AP_NS * AP_TILE);
  uint64_t* x_full = bars;           // [2]
  uint64_t* x_empty = bars + 2;      // [2]
  uint64_t* y_full = bars + 4;       // [2]
  uint64_t* y_free = bars + 6;       // [2]
  uint64_t* w_full = bars + 8;
  uint64_t* w_free = bars + 9;
  uint64_t* drain = bars + 10;
  uint32_t* tmem_s = reinterpret_cast<uint32_t*>(bars + 11);
  volatile int* abort_s = reinterpret_cast<volatile int*>(tmem_s + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = a.BH * a.ntile;
  const int tb = (int)(((int64_t)blockIdx.x * T) / gridDim.x);
  const int te = (int)(((int64_t)(blockIdx.x + 1) * T) / gridDim.x);
  auto head_of = [&](int t) { return t / a.ntile; };

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(x_full + s, 1);
      tc::mbar_init(x_empty + s, 4);
      tc::mbar_init(y_full + s, 1);
      tc::mbar_init(y_free + s, 4);
    }
    tc::mbar_init(w_full, 1);
    tc::mbar_init(w_free, 1);
    tc::mbar_init(drain, 1);
    *abort_s = 0;
    tc::fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tc::prefetch_tmap(&tmX);
    tc::prefetch_tmap(&tmW);
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_s, 2 * AP_D);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = *tmem_s;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int k = 0, nw = 0, loads = 0;
      for (int t = tb; t < te; ++t, ++k) {
        const int bh = head_of(t), tl = t - bh * a.ntile;
        if (t == tb || bh != head_of(t - 1)) {  // this head's W^T
          if (nw > 0 && !tc::mbar_wait(w_free, (nw - 1) & 1, abort_s, AP_WAIT_NS)) break;
          tc::mbar_expect_tx(w_full, AP_TILE);
          for (int j = 0; j < 4; ++j)
            tc::tma_load_2d(Ws + j * AP_BOX, &tmW, 32 * j, bh * AP_D, w_full);
          ++nw;
        }
        const int s = k % AP_NS;
        if (k >= AP_NS &&
            !tc::mbar_wait(x_empty + s, ((k / AP_NS) - 1) & 1, abort_s, AP_WAIT_NS))
          break;
        tc::mbar_expect_tx(x_full + s, AP_TILE);
        for (int j = 0; j < 4; ++j)
          tc::tma_load_2d(Xs + s * AP_TILE + j * AP_BOX, &tmX, 32 * j, bh * a.N + tl * AP_TM,
                          x_full + s);
        ++loads;
      }
      if (*abort_s) {  // let the copies in flight land before the block exits
        for (int q = loads - AP_NS; q < loads; ++q)
          if (q >= 0) tc::mbar_wait_bounded(x_full + (q % AP_NS), (q / AP_NS) & 1, 100000000ull);
        if (nw > 0) tc::mbar_wait_bounded(w_full, (nw - 1) & 1, 100000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ products
    if (lane == 0) {
      const uint32_t idesc = idesc_tf32(AP_TM, AP_D);
      const uint32_t w_addr = smem_u32(Ws);
      int k = 0, nw = 0;
      for (int t = tb; t < te; ++t, ++k) {
        const int bh = head_of(t);
        const bool hstart = t == tb || bh != head_of(t - 1);
        const bool hend = t + 1 == te || head_of(t + 1) != bh;
        if (hstart) {
          if (!tc::mbar_wait(w_full, nw & 1, abort_s, AP_WAIT_NS)) break;
          ++nw;
        }
        const int s = k % AP_NS, b = k & 1;
        if (!tc::mbar_wait(x_full + s, (k / AP_NS) & 1, abort_s, AP_WAIT_NS)) break;
        if (k >= 2 && !tc::mbar_wait(y_free + b, ((k >> 1) - 1) & 1, abort_s, AP_WAIT_NS)) break;
        tc::tc_fence_after();
        const uint32_t d = tbase + (uint32_t)(b * AP_D);
        const uint32_t x_addr = smem_u32(Xs + s * AP_TILE);
#pragma unroll
        for (int ks = 0; ks < AP_D / 8; ++ks) {
          const uint32_t off = (ks >> 2) * AP_BOX + (ks & 3) * 32;
          mma_tf32(d, tc::smem_desc_sw128(x_addr + off, 16, 1024),
                   tc::smem_desc_sw128(w_addr + off, 16, 1024), idesc, ks > 0);
        }
        tc::mma_commit(y_full + b);
        if (hend) tc::mma_commit(w_free);
      }
      tc::mma_commit(drain);  // every product issued so far completes before TMEM is freed
      tc::mbar_wait_bounded(drain, 0, AP_WAIT_NS);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3, r = quarter * 32 + lane;
    const uint32_t lane_f = (uint32_t)(quarter * 32) << 16;
    for (int t = tb, k = 0; t < te; ++t, ++k) {
      const int bh = head_of(t), tl = t - bh * a.ntile;
      const int pos = tl * AP_TM + r;
      const bool valid = pos < a.N;
      int slot = -1, orig = -1;
      if (valid) {
        slot = a.M > 0 ? a.pslot[(size_t)bh * a.N + pos] : -1;
        orig = a.permq[(size_t)bh * a.N + pos];
        if (slot >= a.M || orig < 0 || orig >= a.N) {
          set_error(a.hdr, ERR_INDEX, 21, bh, pos);
          orig = -1;
        }
      }
      const int s = k % AP_NS, b = k & 1;
      bool got = tc::mbar_wait(y_full + b, (k >> 1) & 1, abort_s, AP_WAIT_NS);
      got = __all_sync(0xffffffffu, got);
      if (!got) break;
      tc::tc_fence_after();
      const uint8_t* xt = Xs + s * AP_TILE;
      const int b_ = bh / a.H, h_ = bh - b_ * a.H;
      bf16* orow = orig >= 0 ? a.O + b_ * a.sb + h_ * a.sh + (int64_t)orig * a.sn : nullptr;
      const float* drow = slot >= 0 ? a.odn + ((size_t)bh * a.M + slot) * AP_D : nullptr;
      const float4* bv = reinterpret_cast<const float4*>(a.fitBv + (size_t)bh * AP_D);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {  // 32 columns per chunk (one swizzle box)
        uint32_t y[32];
        __syncwarp();
        tc::tmem_ld32(tbase + lane_f + (uint32_t)(b * AP_D + 32 * c), y);
        tc::tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float4 v;
          if (drow != nullptr) {
            v = reinterpret_cast<const float4*>(drow)[8 * c + q];
          } else {
            const float4 x = *reinterpret_cast<const float4*>(xt + c * AP_BOX + ap_swz(r, q));
            const float4 bb = __ldg(bv + 8 * c + q);
            v.x = x.x + bb.x + __uint_as_float(y[4 * q]);
            v.y = x.y + bb.y + __uint_as_float(y[4 * q + 1]);
            v.z = x.z + bb.z + __uint_as_float(y[4 * q + 2]);
            v.w = x.w + bb.w + __uint_as_float(y[4 * q + 3]);
          }
          pk[2 * q] = pack_bf16(v.x, v.y);
          pk[2 * q + 1] = pack_bf16(v.z, v.w);
        }
        if (orow != nullptr) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        tc::mbar_arrive(y_free + b);
        tc::mbar_arrive(x_empty + s);
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (tid == 0 && *abort_s) set_error(a.hdr, ERR_TIMEOUT, 21, blockIdx.x, 0);
  if (warp == 1) {
    __syncwarp();
    tc::tmem_dealloc(tbase, 2 * AP_D);
  }
}

// Row-major [rows, 128] fp32 tensor, boxes of 32 columns x 128 rows, 128-byte swizzle.
bool ap_map(CUtensorMap* m, const void* ptr, uint64_t rows) {
  const uint64_t dims[2] = {(uint64_t)AP_D, rows};
  const uint64_t strides[1] = {(uint64_t)AP_D * 4};
  const uint32_t box[2] = {32, (uint32_t)AP_TM};
  return encode_tmap(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, ptr, dims, strides, box,
                     CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

cudaError_t launch_apply_tc(const spr_params& p, const Layout& L, const Ptrs& P, bf16* O,
                            int R, cudaStream_t st) {
  const int BH = L.BH, N = p.N, M = p.M;
  if (p.d != AP_D) return cudaErrorInvalidValue;
  spr_launch(k_fit_w<AP_D>, dim3(AP_D, BH), AP_D, 0, st, static_cast<const float*>(P.fitB),
             static_cast<const float*>(P.fitU), static_cast<const spr_head_stats*>(P.stats), R,
             M > 0 ? 1 : 0, P.fitw);
  CUtensorMap mX, mW;
  if (!ap_map(&mX, P.osp, (uint64_t)BH * N) || !ap_map(&mW, P.fitw, (uint64_t)BH * AP_D))
    return cudaErrorInvalidValue;
  ApArgs a{};
  a.odn = P.odn;
  a.pslot = P.pslot;
  a.permq = P.permq;
  a.fitBv = P.fitBv;
  a.N = N;
  a.M = M;
  a.H = p.H;
  a.BH = BH;
  a.ntile = (N + AP_TM - 1) / AP_TM;
  a.sb = p.o_strides[0];
  a.sh = p.o_strides[1];
  a.sn = p.o_strides[2];
  a.O = O;
  a.hdr = P.hdr;
  cudaError_t e = cudaFuncSetAttribute(k_apply_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)AP_SMEM);
  if (e != cudaSuccess) return e;
  const int T = BH * a.ntile;
  const int grid = T < num_sms() ? T : num_sms();
  spr_launch(k_apply_tc, grid, AP_THREADS, AP_SMEM, st, mX, mW, a);
  return cudaGetLastError();
}

}  // namespace spr
