// Routed attention on caller-owned group-major inputs, with no device memory
// allocation (sparsepr_attend_routed_noalloc in include/sparsepr.h).
//
// Some callers cannot allocate device memory at the point where they run
// attention: a serving loop that replays a fixed sequence of launches, an
// engine whose memory pool is carved up before the first request, or a host
// thread that must not take the allocator's lock.  The regular entry points
// keep their state in a caller-sized workspace; this one needs only a small,
// bounded amount of state (an error word, a work cursor, per-head counters and
// the work list), so that state lives in a fixed area of device memory that is
// part of the library image and is located once per device.
//
// The computation is the routed-attention stage of the call [paperlayer §4
// "Sparse Execution"; App. A.2]: every row of query group i attends, with its
// softmax renormalised over the retained keys, to the key ranges routed to i.
// It runs the same attention kernels as sparsepr_attend.
#include <mutex>

#include "spr_internal.cuh"

namespace spr {
namespace {

constexpr size_t NA_SCRATCH_BYTES = size_t(4) << 20;  // 4 MiB
constexpr size_t NA_HDR_BYTES = 256;
constexpr int NA_MAX_DEVICES = 64;

// Zero at module load; every call re-initialises what it reads.
__device__ __align__(256) uint8_t g_na_scratch[NA_SCRATCH_BYTES];

std::mutex g_na_mu;
void* g_na_base[NA_MAX_DEVICES];

__global__ void k_na_check(const int32_t* qoff, const int32_t* runptr, const int2* runs, int BH,
                           int N, int Gq, int Gk, int32_t* counts, Header* hdr);
__global__ void k_na_plan(const int32_t* qoff, const int32_t* counts, int BH, int Gq,
                          int max_items, int4* items, Header* hdr);
__global__ void k_na_status(const Header* hdr, int32_t* status);

// Address of the scratch area on the current device, with the one-time
// set-up of that device: the symbol's address, and every kernel this entry
// point can launch loaded now (device code is otherwise loaded at a kernel's
// first launch, which may take device memory).
cudaError_t na_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= NA_MAX_DEVICES) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_na_mu);
  if (!g_na_base[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_na_scratch);
    if (e != cudaSuccess) return e;
    cudaFuncAttributes fa;
    if ((e = cudaFuncGetAttributes(&fa, k_na_check)) != cudaSuccess) return e;
    if ((e = cudaFuncGetAttributes(&fa, k_na_plan)) != cudaSuccess) return e;
    if ((e = cudaFuncGetAttributes(&fa, k_na_status)) != cudaSuccess) return e;
    if ((e = attend_preload()) != cudaSuccess) return e;
    g_na_base[dev] = p;
  }
  *out = g_na_base[dev];
  return cudaSuccess;
}

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

// Work-list capacity: a query group of n rows gives ceil(n / 128) items and
// the groups of a head hold at most N rows, so a head gives fewer than
// ceil(N / 128) + Gq items.
int64_t na_max_items(int64_t BH, int64_t N, int64_t Gq) {
  return BH * ((N + ATT_BM - 1) / ATT_BM + Gq) + 1;
}

// Scratch layout: header | per-head stats | per-(head, group) tile counts | work list.
size_t na_counts_off(int64_t BH) { return NA_HDR_BYTES + round256((size_t)BH * sizeof(spr_head_stats)); }
size_t na_items_off(int64_t BH, int64_t Gq) {
  return na_counts_off(BH) + round256((size_t)BH * Gq * sizeof(int32_t));
}
size_t na_bytes_needed(int64_t BH, int64_t N, int64_t Gq) {
  return na_items_off(BH, Gq) + (size_t)na_max_items(BH, N, Gq) * sizeof(int4);
}

// One thread per (head, query group): check the group's offsets and every key
// range the attention kernels will follow, and store the group's tile count
// (ceil(rows / ATT_ITEM) when it has rows and at least one range, else 0).  A bad
// index stores 0 and sets the error word with info = {head, group, 0 query
// offsets | 1 range pointers | 2 a key range}.  Block 0 first resets the
// header's cursor and counts (the error word is reset by the host-side
// memset below, before this kernel).
__global__ void __launch_bounds__(256) k_na_check(const int32_t* qoff, const int32_t* runptr,
                                                  const int2* runs, int BH, int N, int Gq, int Gk,
                                                  int32_t* counts, Header* hdr) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= BH * Gq) return;
  const int bh = e / Gq, i = e - bh * Gq;
  const int64_t run_cap = (int64_t)Gq * Gk;
  const int32_t* qo = qoff + (size_t)bh * (Gq + 1);
  const int32_t* rp = runptr + (size_t)bh * (Gq + 1);
  int c = 0;
  const int q0 = qo[i], q1 = qo[i + 1];
  if (!(0 <= q0 && q0 <= q1 && q1 <= N)) {
    set_error(hdr, ERR_INDEX, bh, i, 0);
  } else {
    const int r0 = rp[i], r1 = rp[i + 1];
    if (!(0 <= r0 && r0 <= r1 && r1 <= run_cap)) {
      set_error(hdr, ERR_INDEX, bh, i, 1);
    } else {
      bool ok = true;
      for (int r = r0; r < r1 && ok; ++r) {
        const int2 kr = runs[(size_t)bh * run_cap + r];
        if (!(0 <= kr.x && kr.x < kr.y && kr.y <= N)) {
          set_error(hdr, ERR_INDEX, bh, i, 2);
          ok = false;
        }
      }
      if (ok && q1 > q0 && r1 > r0) c = (q1 - q0 + ATT_ITEM - 1) / ATT_ITEM;
    }
  }
  counts[e] = c;
}

// One block: unless the check above found a bad index, the exclusive scan of
// the item counts and the work list (items of at most ATT_ITEM rows of each
// group, in head-major, group-major order).
__global__ void __launch_bounds__(1024) k_na_plan(const int32_t* qoff, const int32_t* counts,
                                                  int BH, int Gq, int max_items, int4* items,
                                                  Header* hdr) {
  __shared__ int wsum[32];
  __shared__ int total_s;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (hdr->err != 0) return;  // written by the check kernel before this launch
  const int nent = BH * Gq;
  // contiguous slices of entries per thread keep the list in entry order
  const int per = (nent + (int)blockDim.x - 1) / (int)blockDim.x;
  const int e0 = min(nent, tid * per), e1 = min(nent, e0 + per);
  int local = 0;
  for (int e = e0; e < e1; ++e) local += counts[e];
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = (int)blockDim.x >> 5;
    int w = lane < nw ? wsum[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += v;
    }
    if (lane < nw) wsum[lane] = wi - w;
    if (lane == nw - 1) total_s = wi;
  }
  __syncthreads();
  const int total = total_s;
  if (total > max_items) {
    if (tid == 0) set_error(hdr, ERR_WORKLIST, total, max_items, 0);
    return;
  }
  int k = wsum[warp] + incl - local;
  for (int e = e0; e < e1; ++e) {
    const int c = counts[e];
    if (c == 0) continue;
    const int bh = e / Gq, i = e - bh * Gq;
    const int s = qoff[(size_t)bh * (Gq + 1) + i], en = qoff[(size_t)bh * (Gq + 1) + i + 1];
    for (int t = 0; t < c; ++t) {
      const int q0 = s + t * ATT_ITEM;
      items[k++] = make_int4(bh, q0, min(ATT_ITEM, en - q0), i);
    }
  }
  if (tid == 0) hdr->n_items = total;
}

// Copy the error word and its info words to the caller's status buffer.
__global__ void k_na_status(const Header* hdr, int32_t* status) {
  if (threadIdx.x == 0) {
    status[0] = hdr->err;
    status[1] = hdr->err_info[0];
    status[2] = hdr->err_info[1];
    status[3] = hdr->err_info[2];
  }
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace
}  // namespace spr

using namespace spr;

extern "C" spr_status sparsepr_attend_routed_noalloc(
    const void* Qp, const void* Kp, const void* Vp, const int32_t* q_off, const int32_t* run_ptr,
    const int32_t* runs, int32_t BH, int32_t N, int32_t d, int32_t Gq, int32_t Gk, float scale,
    float* O, int32_t* status, void* stream) {
  if (!Qp || !Kp || !Vp || !q_off || !run_ptr || !runs || !O) return SPR_EINVAL;
  if (BH < 1 || N < 1 || Gq < 1 || Gk < 1 || Gq > MAX_GROUPS || Gk > MAX_GROUPS)
    return SPR_EINVAL;
  if (d != 64 && d != 128) return SPR_EUNSUPPORTED;
  if ((int64_t)BH * N > (int64_t)INT32_MAX) return SPR_EINVAL;
  if (!aligned(Qp, 16) || !aligned(Kp, 16) || !aligned(Vp, 16) || !aligned(O, 16) ||
      !aligned(runs, 8) || !aligned(q_off, 4) || !aligned(run_ptr, 4) ||
      (status && !aligned(status, 4)))
    return SPR_EUNSUPPORTED;
  if (na_bytes_needed(BH, N, Gq) > NA_SCRATCH_BYTES) return SPR_ESCRATCH;

  void* base = nullptr;
  if (na_scratch(&base) != cudaSuccess) return SPR_ECUDA;
  uint8_t* b = static_cast<uint8_t*>(base);
  const size_t stats_off = NA_HDR_BYTES;
  const size_t counts_off = na_counts_off(BH);
  const size_t items_off = na_items_off(BH, Gq);
  const int max_items = (int)na_max_items(BH, N, Gq);

  Ptrs P{};
  P.hdr = reinterpret_cast<Header*>(b);
  P.stats = reinterpret_cast<spr_head_stats*>(b + stats_off);
  P.items = reinterpret_cast<int4*>(b + items_off);
  P.Qp = const_cast<bf16*>(static_cast<const bf16*>(Qp));
  P.Kp = const_cast<bf16*>(static_cast<const bf16*>(Kp));
  P.Vp = const_cast<bf16*>(static_cast<const bf16*>(Vp));
  P.qprobe = P.Qp;  // no probe rows: never read
  P.runptr = const_cast<int32_t*>(run_ptr);
  P.runs = reinterpret_cast<int2*>(const_cast<int32_t*>(runs));
  P.osp = O;
  P.odn = O;  // no probe rows: never written

  spr_params p{};
  p.B = 1;
  p.H = BH;
  p.N = N;
  p.d = d;
  p.scale = scale;
  p.Gq = Gq;
  p.Gk = Gk;
  p.M = 0;
  Layout L{};
  L.BH = BH;
  L.N = N;
  L.d = d;
  L.max_items = max_items;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* counts = reinterpret_cast<int32_t*>(b + counts_off);
  // the header (error word, cursor, item count) starts each call at zero
  if (cudaMemsetAsync(P.hdr, 0, sizeof(Header), st) != cudaSuccess) return SPR_ECUDA;
  const int nent = BH * Gq;
  spr_launch(k_na_check, (nent + 255) / 256, 256, 0, st, q_off, run_ptr,
             static_cast<const int2*>(P.runs), (int)BH, (int)N, (int)Gq, (int)Gk, counts, P.hdr);
  spr_launch(k_na_plan, 1, 1024, 0, st, q_off, static_cast<const int32_t*>(counts), (int)BH,
             (int)Gq, max_items, P.items, P.hdr);
  if (cudaGetLastError() != cudaSuccess) return SPR_ECUDA;
  if (launch_attend(p, L, P, st) != cudaSuccess) return SPR_ECUDA;
  if (status) {
    spr_launch(k_na_status, 1, 32, 0, st, static_cast<const Header*>(P.hdr), status);
    if (cudaGetLastError() != cudaSuccess) return SPR_ECUDA;
  }
  return SPR_OK;
}
