// Key-response coordinates Z = K W on the tensor cores [paperlayer App. B.1]
// (the input rows of the key k-means), in fp32 and as bf16 hi | lo rows.
#include <float.h>

#include "spr_internal.cuh"
#include "tc_sm100.cuh"

namespace spr {

constexpr int KM_THREADS = 256;
constexpr int KM_TILE = 128;                 // rows per sub-tile (the UMMA M)
constexpr uint32_t KM_BOX = KM_TILE * 128;   // one 64-column SW128 box of a tile: 16 KB
constexpr uint64_t KM_WAIT_NS = 2000000000ull;

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

// Key-response coordinates Z = K W on the tensor cores [paperlayer App.
// B.1]: K rows exact in bf16, W (d x pp, fp32) split into bf16 hi + lo (two
// products), fp32 accumulation in TMEM.  One 128-row tile per block:
// A = the tile (K-major SW128, cp.async), B = W^T hi / lo ([n][k] rows, n
// padded to NP >= 32 with zeros), D = 128 x NP in TMEM; four warps write one
// Z row (pp floats) per thread, and its split z_hi = bf16(z), z_lo =
// bf16(z - z_hi) as one 128-byte row (the k-means assignment's operand).
template <int D, int PP>
__global__ void __launch_bounds__(KM_THREADS, 1) k_project_tc(TensorView K, int N, const float* W, float* Z,
                                                              bf16* Zhl, Header* hdr) {
  static_assert(PP == 32, "the hi | lo rows hold 32 coordinates");
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
          float z[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) z[i] = __uint_as_float(v[i]);
          uint4* hl = reinterpret_cast<uint4*>(Zhl + ((size_t)bh * N + n) * 64);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            hl[j] = split8(z + 8 * j, false);
            hl[4 + j] = split8(z + 8 * j, true);
          }
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
                               bf16* Zhl, Header* hdr, cudaStream_t st) {
  constexpr int NP = PP < 32 ? 32 : PP;
  const size_t sm = 1024 + (size_t)(D / 64) * (KM_BOX + 2 * NP * 128) + 64;
  cudaError_t e = cudaFuncSetAttribute(k_project_tc<D, PP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sm);
  if (e != cudaSuccess) return e;
  spr_launch(k_project_tc<D, PP>, dim3((N + KM_TILE - 1) / KM_TILE, BH), KM_THREADS, sm, st, K, N, W,
             Z, Zhl, hdr);
  return cudaGetLastError();
}

cudaError_t launch_project(const TensorView& K, int N, int D, int PP, int BH, const float* W,
                           float* Z, bf16* Zhl, Header* hdr, cudaStream_t st) {
  if (PP != 32) return cudaErrorInvalidValue;
  if (D == 128) return proj_launch<128, 32>(K, N, BH, W, Z, Zhl, hdr, st);
  if (D == 64) return proj_launch<64, 32>(K, N, BH, W, Z, Zhl, hdr, st);
  return cudaErrorInvalidValue;
}

}  // namespace spr
