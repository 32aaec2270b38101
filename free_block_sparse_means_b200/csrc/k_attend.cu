// Routed attention under renormalized hard drop, fused with the exact dense
// probe rows [paperlayer §1, §4 "Sparse Execution"; App. A.2].
//
// Work items come from the device-built list: up to ATT_ITEM (256) permuted
// query rows of one query group plus the merged key ranges of the K/V groups
// routed to that group, or up to 256 probe rows with the single key range
// [0, N).  This kernel takes an item's rows 128 at a time.  Each row's softmax is taken over exactly the keys of its
// ranges (renormalised hard drop); keys past a range end are masked.
//
// This file holds the mma.sync (m16n8k16 bf16) implementation: 8 warps x 16
// rows, 64-key tiles double-buffered with cp.async, online softmax in
// registers, fp32 accumulation.  Persistent blocks take items from an atomic
// cursor (no inter-block waiting).
#include <float.h>

#include "spr_internal.cuh"

namespace spr {

struct AttArgs {
  const bf16 *Qp, *Kp, *Vp, *qprobe;
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

constexpr int BN = 64;

template <int D>
__global__ void __launch_bounds__(256, 1) k_attend_mma(AttArgs a) {
  constexpr int CH = D / 8;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* Qs = smem;
  uint8_t* Ks = Qs + ATT_BM * D * 2;  // [2][BN][D]
  uint8_t* Vs = Ks + 2 * BN * D * 2;  // [2][BN][D]
  __shared__ int4 item_s;
  __shared__ int idx_s;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gid = lane >> 2, tig = lane & 3;
  const int n_items = a.hdr->n_items;
  for (;;) {
    if (tid == 0) {
      const int idx = (int)atomicAdd(&a.hdr->work_next, 1u);
      idx_s = idx;
      if (idx < n_items) item_s = a.items[idx];
    }
    __syncthreads();
    if (idx_s >= n_items) break;
    const int4 it = item_s;
    const int bh = it.x, grp = it.w;
    // an item holds up to ATT_ITEM rows: they are taken 128 at a time
    for (int h0 = 0; h0 < it.z; h0 += ATT_BM) {
    const int q0 = it.y + h0, nrows = min(ATT_BM, it.z - h0);
    const bf16* qsrc = grp >= 0 ? a.Qp + ((size_t)bh * a.N + q0) * D
                                : a.qprobe + ((size_t)bh * a.M + q0) * D;
    int rbeg = 0, rend = 1;
    const int2* runs = nullptr;
    if (grp >= 0) {
      rbeg = a.runptr[(size_t)bh * (a.Gq + 1) + grp];
      rend = a.runptr[(size_t)bh * (a.Gq + 1) + grp + 1];
      runs = a.runs + (size_t)bh * a.Gq * a.Gk;
    }
    auto run_at = [&](int r) -> int2 { return runs ? runs[r] : make_int2(0, a.N); };
    const bf16* kbase = a.Kp + (size_t)bh * a.N * D;
    const bf16* vbase = a.Vp + (size_t)bh * a.N * D;
    // Q tile
    for (int e = tid; e < ATT_BM * CH; e += 256) {
      const int r = e / CH, c = e % CH;
      cp_async16(Qs + swz<CH>(r, c), qsrc + (size_t)(r < nrows ? r : 0) * D + c * 8,
                 r < nrows ? 16 : 0);
    }
    auto load_tile = [&](int stage, int t0) {
      uint8_t* kd = Ks + stage * BN * D * 2;
      uint8_t* vd = Vs + stage * BN * D * 2;
      for (int e = tid; e < BN * CH; e += 256) {
        const int r = e / CH, c = e % CH, key = t0 + r;
        const bool ok = key < a.N;
        const size_t off = (size_t)(ok ? key : 0) * D + c * 8;
        cp_async16(kd + swz<CH>(r, c), kbase + off, ok ? 16 : 0);
        cp_async16(vd + swz<CH>(r, c), vbase + off, ok ? 16 : 0);
      }
    };
    int r = rbeg;
    int2 run = run_at(r);
    int t0 = run.x;
    load_tile(0, t0);
    cp_async_commit();
    float o[D / 8][4];
#pragma unroll
    for (int t = 0; t < D / 8; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[t][e] = 0.f;
    float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;
    uint32_t qf[D / 16][4];
    int stage = 0, ntiles = 0;
    bool have = run.x < run.y;
    bool qloaded = false;
    while (have) {
      // next tile position
      int r2 = r, t2 = t0 + BN;
      int2 run2 = run;
      if (t2 >= run.y) {
        ++r2;
        if (r2 < rend) {
          run2 = run_at(r2);
          t2 = run2.x;
        }
      }
      const bool more = r2 < rend;
      if (more) load_tile(stage ^ 1, t2);
      cp_async_commit();
      cp_async_wait<1>();
      __syncthreads();
      if (!qloaded) {
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int rr = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
          const int cc = ks * 2 + (lane >> 4);
          ldsm_x4(qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], Qs + swz<CH>(rr, cc));
        }
        qloaded = true;
      }
      const uint8_t* kt = Ks + stage * BN * D * 2;
      const uint8_t* vt = Vs + stage * BN * D * 2;
      float s[BN / 8][4];
#pragma unroll
      for (int t = 0; t < BN / 8; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[t][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
        for (int np = 0; np < BN / 16; ++np) {
          const int kr = np * 16 + (lane & 7) + (lane >> 4) * 8;
          const int kc = ks * 2 + ((lane >> 3) & 1);
          uint32_t b0, b1, b2, b3;
          ldsm_x4(b0, b1, b2, b3, kt + swz<CH>(kr, kc));
          mma16816(s[2 * np], qf[ks], b0, b1);
          mma16816(s[2 * np + 1], qf[ks], b2, b3);
        }
      }
      // mask, scale to log2 domain, running max
      const int kend = run.y;
      float mx_lo = -INFINITY, mx_hi = -INFINITY;
#pragma unroll
      for (int t = 0; t < BN / 8; ++t) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const bool ok = t0 + t * 8 + 2 * tig + e < kend;
          s[t][e] = ok ? s[t][e] * a.scale_log2 : -INFINITY;
          s[t][2 + e] = ok ? s[t][2 + e] * a.scale_log2 : -INFINITY;
          mx_lo = fmaxf(mx_lo, s[t][e]);
          mx_hi = fmaxf(mx_hi, s[t][2 + e]);
        }
      }
      mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 1));
      mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 2));
      mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 1));
      mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 2));
      const float mn_lo = fmaxf(m_lo, mx_lo), mn_hi = fmaxf(m_hi, mx_hi);
      const float c_lo = ex2(m_lo - mn_lo), c_hi = ex2(m_hi - mn_hi);
      m_lo = mn_lo;
      m_hi = mn_hi;
      l_lo *= c_lo;
      l_hi *= c_hi;
#pragma unroll
      for (int t = 0; t < D / 8; ++t) {
        o[t][0] *= c_lo;
        o[t][1] *= c_lo;
        o[t][2] *= c_hi;
        o[t][3] *= c_hi;
      }
      uint32_t pf[BN / 16][4];
#pragma unroll
      for (int t = 0; t < BN / 8; ++t) {
        const float p0 = ex2(s[t][0] - mn_lo), p1 = ex2(s[t][1] - mn_lo);
        const float p2 = ex2(s[t][2] - mn_hi), p3 = ex2(s[t][3] - mn_hi);
        l_lo += p0 + p1;
        l_hi += p2 + p3;
        pf[t >> 1][(t & 1) * 2 + 0] = pack_bf16(p0, p1);
        pf[t >> 1][(t & 1) * 2 + 1] = pack_bf16(p2, p3);
      }
#pragma unroll
      for (int kk = 0; kk < BN / 16; ++kk) {
#pragma unroll
        for (int np = 0; np < D / 16; ++np) {
          const int vr = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
          const int vc = np * 2 + (lane >> 4);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(b0, b1, b2, b3, vt + swz<CH>(vr, vc));
          mma16816(o[2 * np], pf[kk], b0, b1);
          mma16816(o[2 * np + 1], pf[kk], b2, b3);
        }
      }
      ++ntiles;
      __syncthreads();  // stage fully consumed before it is refilled
      stage ^= 1;
      r = r2;
      run = run2;
      t0 = t2;
      have = more;
    }
    cp_async_wait<0>();
    // finalize
    l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 1);
    l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 2);
    l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 1);
    l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 2);
    const float il = l_lo > 0.f ? 1.f / l_lo : 0.f, ih = l_hi > 0.f ? 1.f / l_hi : 0.f;
    float* dst = grp >= 0 ? a.osp + ((size_t)bh * a.N + q0) * D : a.odn + ((size_t)bh * a.M + q0) * D;
    const int rl = warp * 16 + gid, rh = rl + 8;
#pragma unroll
    for (int t = 0; t < D / 8; ++t) {
      const int c = t * 8 + 2 * tig;
      if (rl < nrows)
        *reinterpret_cast<float2*>(dst + (size_t)rl * D + c) = make_float2(o[t][0] * il, o[t][1] * il);
      if (rh < nrows)
        *reinterpret_cast<float2*>(dst + (size_t)rh * D + c) = make_float2(o[t][2] * ih, o[t][3] * ih);
    }
    if (tid == 0)
      atomicAdd(reinterpret_cast<unsigned long long*>(&a.stats[bh].tile_pairs),
                (unsigned long long)ntiles * BN * ATT_BM);
    __syncthreads();
    }
  }
}

// Rewind the work-list cursor and the per-head executed tile-pair counters so
// that the stage can be run again on the same workspace.
__global__ void k_attend_reset(Header* hdr, spr_head_stats* stats, int BH) {
  if (threadIdx.x == 0) hdr->work_next = 0;
  for (int i = threadIdx.x; i < BH; i += blockDim.x) stats[i].tile_pairs = 0;
}

// Load the device code of every attention-stage kernel now (a kernel is
// otherwise loaded at its first launch, which may take device memory).
cudaError_t attend_preload() {
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, k_attend_reset);
  if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, k_attend_mma<64>);
  if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, k_attend_mma<128>);
  if (e == cudaSuccess) e = attend_tc_preload();
  return e;
}

cudaError_t launch_attend(const spr_params& p, const Layout& L, const Ptrs& P, cudaStream_t st) {
  spr_launch(k_attend_reset, 1, 256, 0, st, P.hdr, P.stats, L.BH);
  if (attend_tc_enabled(p.d)) return launch_attend_tc(p, L, P, st);
  AttArgs a;
  a.Qp = P.Qp;
  a.Kp = P.Kp;
  a.Vp = P.Vp;
  a.qprobe = P.qprobe;
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
  const int grid = num_sms();
  if (p.d == 64) {
    const size_t sm = (size_t)(ATT_BM + 4 * BN) * 64 * 2;
    cudaFuncSetAttribute(k_attend_mma<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    spr_launch(k_attend_mma<64>, grid, 256, sm, st, a);
  } else {
    const size_t sm = (size_t)(ATT_BM + 4 * BN) * 128 * 2;
    cudaFuncSetAttribute(k_attend_mma<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    spr_launch(k_attend_mma<128>, grid, 256, sm, st, a);
  }
  return cudaGetLastError();
}

}  // namespace spr
