// Internal declarations shared by the SparsePR CUDA sources (not part of the
// public C ABI).  Workspace layout, launch helpers and device utilities.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sparsepr.h"

namespace spr {

typedef __nv_bfloat16 bf16;

constexpr int CHUNK = 512;         // rows per histogram chunk (k-means, permutation)
constexpr int MAX_GROUPS = 256;    // Gk, Gq upper bound
constexpr int MAX_P = 32;          // eigen-coordinate upper bound (coordinates padded to 32)
constexpr int MAX_PROBES = 4096;   // M upper bound
constexpr int ATT_BM = 128;        // query rows per attention tile
constexpr int ATT_ITEM = 128;      // query rows per attention work item (one tile)

// Device error word codes (first error wins; info words carry details).
enum : int32_t {
  ERR_NONE = 0,
  ERR_INDEX = 1,       // an index read from the workspace is out of range
  ERR_WORKLIST = 2,    // attention work list overflow
  ERR_NUMERIC = 3,     // non-finite value where the method needs a finite one
  ERR_TIMEOUT = 4,     // a bounded wait gave up
};

// Workspace buffers.
enum Buf : int {
  B_HDR, B_STATS, B_MK, B_TRACE, B_EVAL, B_EVEC, B_W, B_Z, B_INITK, B_INITQ, B_CENTK,
  B_LABK, B_LABQ, B_CHUNK, B_CBASE, B_COUNTS, B_PERMK, B_KVOFF, B_PERMQ, B_QOFF,
  B_KP, B_VP, B_QP, B_CRAW, B_CT, B_AMAT, B_RMS, B_UN2, B_CENTQ, B_BQ16, B_BETA,
  B_QBAR, B_LOGIT, B_ENTRY, B_TOP, B_SEL, B_ROWPTR, B_COLIDX, B_RUNPTR, B_RUNS, B_PPOS,
  B_PIDX, B_PW, B_PSLOT, B_QPROBE, B_ITEMS, B_OSP, B_ODN, B_FITU, B_FITB, B_FITBV,
  B_GRAM, B_AXX, B_RXBAR, B_PROJ, B_PART, B_CSUM, B_XP, B_RP, B_PMEAN, B_CRAW64, B_QBAR64,
  B_SLOTCNT, B_TMASK, B_GBITS, B_BK16, B_ZHL, B_PDIST, B_FITW, B_COUNT_
};

struct Layout {
  size_t off[B_COUNT_];
  size_t bytes[B_COUNT_];
  size_t total;
  int BH, N, d, nchunk, max_items, part_slots;
};

// Header block at the start of the workspace.
struct Header {
  int32_t err;          // ERR_* of the first fault
  int32_t err_info[3];
  uint32_t work_next;   // attention work-list cursor
  int32_t n_items;      // attention work items
  int32_t pad[10];
};

bool make_layout(const spr_params* p, Layout* L);
// Eigen-coordinate width: 32 (p <= 32; columns past p are zero).
int padded_p(int p);
// Rows per head of the query k-means operand buffer: max(round32(Gmax), d).
inline int bq_rows(int Gmax, int d) {
  const int nc = (Gmax + 31) / 32 * 32;
  return nc > d ? nc : d;
}

// Pointers of one call, resolved from the workspace base.
struct Ptrs {
  Header* hdr;
  spr_head_stats* stats;
  float *MK, *trace, *eval, *evec, *W, *Z, *centk, *Craw, *Ct, *Amat, *rms, *un2, *centq, *beta,
      *qbar, *pw, *osp, *odn, *fitU, *fitB, *fitBv, *gram, *axx, *rxbar,
      *proj, *csum, *xp, *rp, *pmean;
  double* part;
  double *logit, *entry;  // route logits and tail masses [BH][Gq][Gk] (fp64)
  double *craw64, *qbar64;  // raw-key and raw-query group means (fp64)
  double* gpart;          // group-mean slice sums (aliases the k-means partial sums)
  int32_t *initk, *initq, *labk, *labq, *chunk, *cbase, *counts, *permk, *kvoff, *permq,
      *qoff, *rowptr, *colidx, *runptr, *ppos, *pidx, *pslot, *slotcnt;
  uint32_t *tmask, *gbits;  // k-means update bookkeeping
  bf16* bk16;               // key k-means operand [BH][2][round32(Gk)][64]
  bf16* zhl;                // key coordinates as bf16 hi | lo rows [BH][N][64]
  float* pdist;             // ranked probes: distance of each permuted query [BH][N]
  float* fitw;              // W^T = (B U_r^T)^T of the fit [BH][d][d] (d = 128 path)
  int2* runs;
  int4* items;
  uint8_t *sel, *top;
  bf16 *Kp, *Vp, *Qp, *bq16, *qprobe;
  // Vp holds V in the group-major key order, [BH][N][d]; when the tensor-core
  // attention runs (attend_tc_enabled), the partition writes it transposed
  // instead, [BH][d][vt_ld(N)], and Vt points at it (null otherwise).
  bf16* Vt;
};

// Row length of the transposed V: N rounded up to 8 keys (16 bytes), so that
// every row starts 16-byte aligned for the tensor-memory-access unit.
__host__ __device__ inline int64_t vt_ld(int64_t N) { return (N + 7) & ~int64_t(7); }

Ptrs resolve(const Layout& L, void* ws);

// Strided input view of one tensor (elements).
struct TensorView {
  const bf16* base;
  int64_t sb, sh, sn;
  int H;
  __host__ __device__ const bf16* row(int bh, int n) const {
    int b = bh / H, h = bh - b * H;
    return base + b * sb + h * sh + (int64_t)n * sn;
  }
};

// ---- stage launchers (host) ----
cudaError_t launch_partition(const spr_params& p, const Layout& L, const Ptrs& P,
                             const TensorView& Q, const TensorView& K, const TensorView& V,
                             cudaStream_t st);
cudaError_t launch_route(const spr_params& p, const Layout& L, const Ptrs& P, cudaStream_t st);
cudaError_t launch_attend(const spr_params& p, const Layout& L, const Ptrs& P, cudaStream_t st);
// tcgen05 routed attention (head dims 64 and 128); attend_tc_enabled says whether
// launch_attend uses it for this head dim.
cudaError_t launch_attend_tc(const spr_params& p, const Layout& L, const Ptrs& P, cudaStream_t st);
bool attend_tc_enabled(int d);
// Load the attention kernels' device code ahead of their first launch (and
// resolve the tensor-map encoder the tcgen05 kernel needs).
cudaError_t attend_preload();
cudaError_t attend_tc_preload();
cudaError_t launch_reconstruct(const spr_params& p, const Layout& L, const Ptrs& P,
                               bf16* O, cudaStream_t st);
// Query-response RMS and ||u_hat||^2 on the tensor cores (head dimension D =
// 64 or 128), with the chunk sums of ||u_hat||^2 into part (tpart: BH *
// ceil(N / 128) * 4 doubles).
cudaError_t launch_rms_tc(const TensorView& Q, int B, int H, int N, int D, int nchunk,
                          int split_rows, const bf16* bsplit, float scale,
                          const spr_head_stats* stats, float* rms, float* un2, double* tpart,
                          double* part, Header* hdr, cudaStream_t st);
// Residual application on the tensor cores (d = 128): O = x + b + x W per
// unprobed permuted row, the dense row per probe, bf16 in the original order.
cudaError_t launch_apply_tc(const spr_params& p, const Layout& L, const Ptrs& P, bf16* O, int R,
                            cudaStream_t st);
// Leading eigenpairs of `count` symmetric n x n matrices (fp32, row-major):
// evals[m * n + k] for the K largest (descending), evecs[(m * n + row) * n + k]
// the matching unit eigenvectors as columns, trace[m] the trace (may be null).
cudaError_t launch_eig(const float* A, int count, int n, int K, float* evals, float* evecs,
                       float* trace, cudaStream_t st);
int num_sms();

enum { KM_QUERY = 0, KM_KEY = 1 };
// One Lloyd iteration (assignment on the tensor cores, then the update) of
// the query (KM_QUERY: rows of X, width d, operand bq from k_qprep) or key
// (KM_KEY: rows of Z, 32 coordinates, operand bk) k-means; cent receives the
// new centroids (and, key mode, bk the next operand).
constexpr int LLOYD_SLOTS = 128;
struct LloydStep {
  int mode, d, N, G, BH, split_rows;
  TensorView X;        // query mode: the rows ([B, H, N, d] view)
  const float* Z;      // key mode: [BH][N][32] coordinates (fp32, summed by the update)
  const bf16* Zhl;     // key mode: [BH][N][64] the same rows as bf16 hi | lo (scored)
  const bf16* bq;      // query mode: [BH][2][split_rows][d] operand (hi, lo)
  bf16* bk;            // key mode: [BH][2][lloyd_ncrows(G)][64] operand (hi, lo)
  const float* rms;    // query mode: row RMS (factor scale / rms)
  const float* A;      // query mode, optional: A = C~^T C~ [BH][d][d]; the update then also
                       // writes the next iteration's operand bq and beta (as k_qprep does)
  float scale;
  const float* beta;   // [BH][G]: query beta_g (k_qprep); key ||c_g||^2 / 2 (written by the update)
  float* cent;         // [BH][G][width] centroids, updated in place
  int32_t* lab;        // [BH][N] labels (out)
  float* slots;        // lloyd_slot_bytes(BH, N, d): per-tile partial sums
  int32_t* slot_cnt;   // [BH * ceil(N / 128)][LLOYD_SLOTS]
  uint32_t* tmask;     // [BH * ceil(N / 128)][8]
  uint32_t* gbits;     // [BH][G][ceil(ceil(N / 128) / 32)], zero before the first step
  Header* hdr;
  // capacities in bytes of slots, slot_cnt, tmask, gbits (checked before launch)
  size_t slots_bytes, slot_cnt_bytes, tmask_bytes, gbits_bytes;
};
cudaError_t lloyd_step(const LloydStep& s, cudaStream_t st);
// Key operand rows and beta_g = ||c_g||^2 / 2 from centroids (first iteration).
cudaError_t lloyd_key_operand(const float* cent, int G, int BH, bf16* bk, float* beta,
                              cudaStream_t st);
int lloyd_ncrows(int G);
size_t lloyd_slot_bytes(int BH, int N, int d);
// Chunk label histograms [BH][nchunk][G] (for k_chunk_scan / k_scatter).
cudaError_t label_hist(const int32_t* lab, int N, int G, int nchunk, int BH, int32_t* chunk_cnt,
                       Header* hdr, cudaStream_t st);

// Key-response coordinates Z = K W (tensor cores); W is [BH][d][pp] fp32.
cudaError_t launch_project(const TensorView& K, int N, int D, int PP, int BH, const float* W,
                           float* Z, bf16* Zhl, Header* hdr, cudaStream_t st);

// Every kernel launch of the library goes through spr_launch, which counts it
// (sparsepr_launch_count reports the total).
void note_launch();
#ifdef __CUDACC__
template <typename... KArgs, typename... Args>
inline void spr_launch(void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args... args) {
  k<<<grid, block, smem, st>>>(args...);
  note_launch();
}
#endif

}  // namespace spr

// ------------------------------------------------------------------------
// Device helpers
// ------------------------------------------------------------------------
#ifdef __CUDACC__
namespace spr {

__device__ __forceinline__ void set_error(Header* h, int code, int a = 0, int b = 0, int c = 0) {
  if (atomicCAS(&h->err, 0, code) == 0) {
    h->err_info[0] = a;
    h->err_info[1] = b;
    h->err_info[2] = c;
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte asynchronous global->shared copy; src_bytes = 0 zero-fills.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(smem)),
               "l"(gmem), "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

__device__ __forceinline__ void ldsm_x4(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                        const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3,
                                          const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(smem_u32(p)));
}

// D = A(16x16 bf16, row) * B(16x8 bf16, col) + D (fp32)
__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// exp2 through the hardware approximation instruction.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));  // pure: free to schedule
  return y;
}

// Byte offset of 16-byte chunk `c` of row `r` in a row-major bf16 tile with
// `CH` chunks per row, XOR-swizzled so that 8 consecutive rows at the same
// logical chunk hit 8 distinct bank groups.
template <int CH>
__device__ __forceinline__ int swz(int r, int c) {
  return (r * CH + (c ^ (r & 7))) * 16;
}

__device__ __forceinline__ float bf2f(bf16 v) { return __bfloat162float(v); }

}  // namespace spr
#endif
