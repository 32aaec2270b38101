// C-ABI entry points of the SparsePR call: parameter validation, workspace
// layout and the stage sequence.  Every entry point only enqueues work on the
// caller's stream; no memory is allocated here.
#include <math.h>
#include <string.h>

#include <atomic>

#include "spr_internal.cuh"

namespace spr {

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool make_layout(const spr_params* p, Layout* L) {
  if (sparsepr_check_params(p) != SPR_OK) return false;
  const size_t BH = (size_t)p->B * p->H, N = p->N, d = p->d, P = padded_p(p->p);
  const size_t Gk = p->Gk, Gq = p->Gq, Gm = Gk > Gq ? Gk : Gq, M = p->M;
  const size_t nchunk = (N + CHUNK - 1) / CHUNK;
  const size_t tiles = (N + ATT_BM - 1) / ATT_BM;
  const size_t max_items = BH * (tiles + Gq + (M + ATT_BM - 1) / ATT_BM) + 1;
  const size_t part_slots = BH * (nchunk + 1) * 2 + BH * Gq;
  size_t sz[B_COUNT_];
  sz[B_HDR] = sizeof(Header);
  sz[B_STATS] = BH * sizeof(spr_head_stats);
  sz[B_MK] = BH * d * d * 4;
  sz[B_TRACE] = BH * 4;
  sz[B_EVAL] = BH * d * 4;
  sz[B_EVEC] = BH * d * d * 4;
  sz[B_W] = BH * d * P * 4;
  sz[B_Z] = BH * N * P * 4;
  sz[B_INITK] = BH * Gk * 4;
  sz[B_INITQ] = BH * Gq * 4;
  sz[B_CENTK] = BH * Gk * P * 4;
  sz[B_LABK] = BH * N * 4;
  sz[B_LABQ] = BH * N * 4;
  sz[B_CHUNK] = BH * nchunk * Gm * 4;
  sz[B_CBASE] = BH * nchunk * Gm * 4;
  sz[B_COUNTS] = BH * Gm * 4;
  sz[B_PERMK] = BH * N * 4;
  sz[B_KVOFF] = BH * (Gk + 1) * 4;
  sz[B_PERMQ] = BH * N * 4;
  sz[B_QOFF] = BH * (Gq + 1) * 4;
  sz[B_KP] = BH * N * d * 2;
  sz[B_VP] = BH * vt_ld(N) * d * 2;  // [BH][N][d], or transposed [BH][d][vt_ld(N)]
  sz[B_QP] = BH * N * d * 2;
  sz[B_CRAW] = BH * Gk * d * 4;
  sz[B_CT] = BH * Gk * d * 4;
  sz[B_AMAT] = BH * d * d * 4;
  sz[B_RMS] = BH * N * 4;
  sz[B_UN2] = BH * N * 4;
  sz[B_CENTQ] = BH * Gq * d * 4;
  sz[B_BQ16] = BH * 2 * (size_t)bq_rows((int)Gm, (int)d) * d * 2;  // semantic mode: key groups too
  sz[B_BETA] = BH * Gm * 4;
  sz[B_QBAR] = BH * Gq * d * 4;
  sz[B_LOGIT] = BH * Gq * Gk * 8;
  sz[B_ENTRY] = BH * Gq * Gk * 8;
  sz[B_TOP] = BH * Gq * Gk;
  sz[B_SEL] = BH * Gq * Gk;
  sz[B_ROWPTR] = BH * (Gq + 1) * 4;
  sz[B_COLIDX] = BH * Gq * Gk * 4;
  sz[B_RUNPTR] = BH * (Gq + 1) * 4;
  sz[B_RUNS] = BH * Gq * Gk * 8;
  sz[B_PPOS] = BH * (M ? M : 1) * 4;
  sz[B_PIDX] = BH * (M ? M : 1) * 4;
  sz[B_PW] = BH * (M ? M : 1) * 4;
  sz[B_PSLOT] = BH * N * 4;
  sz[B_QPROBE] = BH * (M ? M : 1) * d * 2;
  sz[B_ITEMS] = max_items * 16;
  sz[B_OSP] = BH * N * d * 4;
  sz[B_ODN] = BH * (M ? M : 1) * d * 4;
  sz[B_FITU] = BH * d * d * 4;
  sz[B_FITB] = BH * d * d * 4;
  sz[B_FITBV] = BH * d * 4;
  sz[B_GRAM] = BH * d * d * 4;
  sz[B_AXX] = BH * d * d * 4;
  sz[B_RXBAR] = BH * 2 * d * 4;
  sz[B_PROJ] = BH * (M ? (M + 63) / 64 : 1) * d * (p->r > 0 ? p->r : 1) * 4;  // fit rhs partials
  sz[B_PART] = part_slots * 8;
  // k-means partial sums (one per label present in each 128-row tile), also
  // the group-mean slices (fp64)
  sz[B_CSUM] = lloyd_slot_bytes((int)BH, (int)N, (int)d);
  if (sz[B_CSUM] < BH * Gm * 8 * d * 8) sz[B_CSUM] = BH * Gm * 8 * d * 8;
  // probe rows gathered for the fit: sparse outputs X, residuals R, block means
  sz[B_XP] = BH * (M ? M : 1) * d * 4;
  sz[B_RP] = BH * (M ? M : 1) * d * 4;
  sz[B_PMEAN] = BH * (M ? (M + 31) / 32 : 1) * 2 * d * 4;
  sz[B_CRAW64] = BH * Gk * d * 8;
  sz[B_QBAR64] = BH * Gq * d * 8;
  const size_t ntile = (N + 127) / 128, nword = (ntile + 31) / 32;
  sz[B_SLOTCNT] = BH * ntile * LLOYD_SLOTS * 4;
  sz[B_TMASK] = BH * ntile * 8 * 4;
  sz[B_GBITS] = BH * Gm * nword * 4;
  sz[B_BK16] = BH * 2 * (size_t)lloyd_ncrows((int)Gk) * 64 * 2;
  sz[B_ZHL] = BH * N * 64 * 2;
  sz[B_PDIST] = BH * N * 4;  // written only with ranked probes
  sz[B_FITW] = BH * d * d * 4;
  size_t off = 0;
  for (int i = 0; i < B_COUNT_; ++i) {
    L->off[i] = off;
    L->bytes[i] = sz[i];
    off = align_up(off + sz[i], 256);
  }
  L->total = off;
  L->BH = (int)BH;
  L->N = (int)N;
  L->d = (int)d;
  L->nchunk = (int)nchunk;
  L->max_items = (int)max_items;
  L->part_slots = (int)part_slots;
  return true;
}

Ptrs resolve(const Layout& L, void* ws) {
  char* b = static_cast<char*>(ws);
  Ptrs P;
#define AT(T, i) reinterpret_cast<T>(b + L.off[i])
  P.hdr = AT(Header*, B_HDR);
  P.stats = AT(spr_head_stats*, B_STATS);
  P.MK = AT(float*, B_MK);
  P.trace = AT(float*, B_TRACE);
  P.eval = AT(float*, B_EVAL);
  P.evec = AT(float*, B_EVEC);
  P.W = AT(float*, B_W);
  P.Z = AT(float*, B_Z);
  P.initk = AT(int32_t*, B_INITK);
  P.initq = AT(int32_t*, B_INITQ);
  P.centk = AT(float*, B_CENTK);
  P.labk = AT(int32_t*, B_LABK);
  P.labq = AT(int32_t*, B_LABQ);
  P.chunk = AT(int32_t*, B_CHUNK);
  P.cbase = AT(int32_t*, B_CBASE);
  P.counts = AT(int32_t*, B_COUNTS);
  P.permk = AT(int32_t*, B_PERMK);
  P.kvoff = AT(int32_t*, B_KVOFF);
  P.permq = AT(int32_t*, B_PERMQ);
  P.qoff = AT(int32_t*, B_QOFF);
  P.Kp = AT(bf16*, B_KP);
  P.Vp = AT(bf16*, B_VP);
  P.Vt = attend_tc_enabled(L.d) ? P.Vp : nullptr;
  P.Qp = AT(bf16*, B_QP);
  P.Craw = AT(float*, B_CRAW);
  P.Ct = AT(float*, B_CT);
  P.Amat = AT(float*, B_AMAT);
  P.rms = AT(float*, B_RMS);
  P.un2 = AT(float*, B_UN2);
  P.centq = AT(float*, B_CENTQ);
  P.bq16 = AT(bf16*, B_BQ16);
  P.beta = AT(float*, B_BETA);
  P.qbar = AT(float*, B_QBAR);
  P.logit = AT(double*, B_LOGIT);
  P.entry = AT(double*, B_ENTRY);
  P.sel = AT(uint8_t*, B_SEL);
  P.top = AT(uint8_t*, B_TOP);
  P.rowptr = AT(int32_t*, B_ROWPTR);
  P.colidx = AT(int32_t*, B_COLIDX);
  P.runptr = AT(int32_t*, B_RUNPTR);
  P.runs = AT(int2*, B_RUNS);
  P.ppos = AT(int32_t*, B_PPOS);
  P.pidx = AT(int32_t*, B_PIDX);
  P.pw = AT(float*, B_PW);
  P.pslot = AT(int32_t*, B_PSLOT);
  P.qprobe = AT(bf16*, B_QPROBE);
  P.items = AT(int4*, B_ITEMS);
  P.osp = AT(float*, B_OSP);
  P.odn = AT(float*, B_ODN);
  P.fitU = AT(float*, B_FITU);
  P.fitB = AT(float*, B_FITB);
  P.fitBv = AT(float*, B_FITBV);
  P.gram = AT(float*, B_GRAM);
  P.axx = AT(float*, B_AXX);
  P.rxbar = AT(float*, B_RXBAR);
  P.proj = AT(float*, B_PROJ);
  P.part = AT(double*, B_PART);
  P.csum = AT(float*, B_CSUM);
  P.xp = AT(float*, B_XP);
  P.rp = AT(float*, B_RP);
  P.pmean = AT(float*, B_PMEAN);
  P.craw64 = AT(double*, B_CRAW64);
  P.qbar64 = AT(double*, B_QBAR64);
  P.gpart = AT(double*, B_CSUM);
  P.slotcnt = AT(int32_t*, B_SLOTCNT);
  P.tmask = AT(uint32_t*, B_TMASK);
  P.gbits = AT(uint32_t*, B_GBITS);
  P.bk16 = AT(bf16*, B_BK16);
  P.zhl = AT(bf16*, B_ZHL);
  P.pdist = AT(float*, B_PDIST);
  P.fitw = AT(float*, B_FITW);
#undef AT
  return P;
}

static std::atomic<long long> g_launches{0};
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

static bool strides_ok(const int64_t* s, const void* base) {
  if (s[0] < 0 || s[1] < 0 || s[2] <= 0) return false;
  if ((s[0] % 8) || (s[1] % 8) || (s[2] % 8)) return false;
  if (base && (reinterpret_cast<uintptr_t>(base) & 15)) return false;
  return true;
}

}  // namespace spr

using namespace spr;

extern "C" {

const char* sparsepr_version(void) { return "sparsepr-b200 0.1 (sm_100a)"; }

int64_t sparsepr_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

spr_status sparsepr_check_params(const spr_params* p) {
  if (!p) return SPR_EINVAL;
  if (p->B < 1 || p->H < 1 || p->N < 1) return SPR_EINVAL;
  if (p->d != 64 && p->d != 128) return SPR_EUNSUPPORTED;
  if ((int64_t)p->B * p->H * p->N > (int64_t)1 << 30) return SPR_EUNSUPPORTED;
  if (p->Ms < 1 || p->Ms > p->N) return SPR_EINVAL;
  if (p->p < 1 || p->p > p->d) return SPR_EINVAL;
  if (p->p > MAX_P) return SPR_EUNSUPPORTED;
  if (p->Gk < 1 || p->Gq < 1 || p->Gk > p->N || p->Gq > p->N) return SPR_EINVAL;
  if (p->Gk > MAX_GROUPS || p->Gq > MAX_GROUPS) return SPR_EUNSUPPORTED;
  if (p->iters < 1 || p->iters > 100) return SPR_EINVAL;
  if (p->route_mode != SPR_ROUTE_TAU && p->route_mode != SPR_ROUTE_BUDGET) return SPR_EINVAL;
  if (p->route_mode == SPR_ROUTE_TAU && !(p->tau > 0.0)) return SPR_EINVAL;
  if (p->route_mode == SPR_ROUTE_BUDGET && !(p->rho_target > 0.0 && p->rho_target <= 1e6))
    return SPR_EINVAL;
  if (p->M < 0 || p->M > p->N) return SPR_EINVAL;
  if (p->M > MAX_PROBES) return SPR_EUNSUPPORTED;
  if (p->r < 0 || p->r > p->d) return SPR_EINVAL;
  if (!(p->lambda >= 0.0) || !isfinite(p->lambda)) return SPR_EINVAL;
  if (!isfinite(p->scale)) return SPR_EINVAL;
  if (p->partition != SPR_PARTITION_RESPONSE && p->partition != SPR_PARTITION_SEMANTIC)
    return SPR_EINVAL;
  if (p->init != SPR_INIT_SEEDED && p->init != SPR_INIT_WARM) return SPR_EINVAL;
  if (p->weights != SPR_WEIGHTS_COVERAGE && p->weights != SPR_WEIGHTS_UNIFORM) return SPR_EINVAL;
  if (p->probes != SPR_PROBES_STRATIFIED && p->probes != SPR_PROBES_RANKED) return SPR_EINVAL;
  if (p->probes == SPR_PROBES_RANKED && p->partition != SPR_PARTITION_RESPONSE)
    return SPR_EUNSUPPORTED;  // no query-response coordinates to rank in
  if (p->head0 < 0 || p->head0 > (1 << 30)) return SPR_EINVAL;
  return SPR_OK;
}

size_t sparsepr_workspace_size(const spr_params* prm) {
  Layout L;
  if (!make_layout(prm, &L)) return 0;
  return L.total;
}

static spr_status prologue(const spr_params* prm, void* ws, size_t ws_bytes, Layout* L) {
  spr_status s = sparsepr_check_params(prm);
  if (s != SPR_OK) return s;
  make_layout(prm, L);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255)) return SPR_EWORKSPACE;
  if (ws_bytes < L->total) return SPR_EWORKSPACE;
  return SPR_OK;
}

static TensorView view(const void* base, const int64_t* s, int H) {
  TensorView v;
  v.base = static_cast<const bf16*>(base);
  v.sb = s[0];
  v.sh = s[1];
  v.sn = s[2];
  v.H = H;
  return v;
}

spr_status sparsepr_partition(const spr_params* prm, const void* Q, const void* K,
                              const void* V, void* ws, size_t ws_bytes, void* stream) {
  Layout L;
  spr_status s = prologue(prm, ws, ws_bytes, &L);
  if (s != SPR_OK) return s;
  if (!Q || !K || !V) return SPR_EINVAL;
  if (!strides_ok(prm->q_strides, Q) || !strides_ok(prm->k_strides, K) ||
      !strides_ok(prm->v_strides, V))
    return SPR_EUNSUPPORTED;
  Ptrs P = resolve(L, ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, L.off[B_STATS] + L.bytes[B_STATS], st) != cudaSuccess)
    return SPR_ECUDA;
  cudaError_t e = launch_partition(*prm, L, P, view(Q, prm->q_strides, prm->H),
                                   view(K, prm->k_strides, prm->H),
                                   view(V, prm->v_strides, prm->H), st);
  return e == cudaSuccess ? SPR_OK : SPR_ECUDA;
}

spr_status sparsepr_route(const spr_params* prm, void* ws, size_t ws_bytes, void* stream) {
  Layout L;
  spr_status s = prologue(prm, ws, ws_bytes, &L);
  if (s != SPR_OK) return s;
  cudaError_t e = launch_route(*prm, L, resolve(L, ws), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SPR_OK : SPR_ECUDA;
}

spr_status sparsepr_attend(const spr_params* prm, void* ws, size_t ws_bytes, void* stream) {
  Layout L;
  spr_status s = prologue(prm, ws, ws_bytes, &L);
  if (s != SPR_OK) return s;
  cudaError_t e = launch_attend(*prm, L, resolve(L, ws), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SPR_OK : SPR_ECUDA;
}

spr_status sparsepr_reconstruct(const spr_params* prm, void* ws, size_t ws_bytes, void* O,
                                void* stream) {
  Layout L;
  spr_status s = prologue(prm, ws, ws_bytes, &L);
  if (s != SPR_OK) return s;
  if (!O) return SPR_EINVAL;
  if (!strides_ok(prm->o_strides, O)) return SPR_EUNSUPPORTED;
  cudaError_t e = launch_reconstruct(*prm, L, resolve(L, ws), static_cast<bf16*>(O),
                                     static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SPR_OK : SPR_ECUDA;
}

spr_status sparsepr_call(const spr_params* prm, const void* Q, const void* K, const void* V,
                         void* O, void* ws, size_t ws_bytes, void* stream) {
  if (!O) return SPR_EINVAL;
  if (prm && sparsepr_check_params(prm) == SPR_OK && !strides_ok(prm->o_strides, O))
    return SPR_EUNSUPPORTED;
  spr_status s = sparsepr_partition(prm, Q, K, V, ws, ws_bytes, stream);
  if (s != SPR_OK) return s;
  if ((s = sparsepr_route(prm, ws, ws_bytes, stream)) != SPR_OK) return s;
  if ((s = sparsepr_attend(prm, ws, ws_bytes, stream)) != SPR_OK) return s;
  return sparsepr_reconstruct(prm, ws, ws_bytes, O, stream);
}

spr_status sparsepr_get_stats(const spr_params* prm, const void* ws, size_t ws_bytes,
                              spr_head_stats* host_out, int32_t* device_error, void* stream) {
  Layout L;
  spr_status s = prologue(prm, const_cast<void*>(ws), ws_bytes, &L);
  if (s != SPR_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Header h;
  const char* b = static_cast<const char*>(ws);
  if (cudaMemcpyAsync(&h, b + L.off[B_HDR], sizeof(Header), cudaMemcpyDeviceToHost, st) !=
      cudaSuccess)
    return SPR_ECUDA;
  if (host_out && cudaMemcpyAsync(host_out, b + L.off[B_STATS], L.bytes[B_STATS],
                                  cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return SPR_ECUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return SPR_ECUDA;
  if (device_error) *device_error = h.err;
  return h.err ? SPR_EDEVICE : SPR_OK;
}

spr_status sparsepr_workspace_view(const spr_params* prm, int32_t which, size_t* offset,
                                   size_t* bytes) {
  Layout L;
  if (!make_layout(prm, &L)) return SPR_EINVAL;
  static const int map[SPR_VIEW_COUNT] = {
      B_LABK, B_LABQ, B_PERMK, B_PERMQ, B_KVOFF, B_QOFF, B_ROWPTR, B_COLIDX, B_PPOS,
      B_PIDX, B_PW,   B_OSP,   B_ODN,   B_W,     B_CENTK, B_CENTQ, B_CT,    B_RMS,
      B_ENTRY, B_FITU, B_FITB, B_FITBV, B_PDIST};
  if (which < 0 || which >= SPR_VIEW_COUNT) return SPR_EINVAL;
  if (offset) *offset = L.off[map[which]];
  if (bytes) *bytes = L.bytes[map[which]];
  return SPR_OK;
}

}  // extern "C"
