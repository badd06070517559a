// C ABI of libsla2.so (declared in include/sla2.h): argument checks, the
// workspace layout, TMA descriptors and the launch sequence of the forward
// pass. Nothing here computes on the host; every step runs in the kernels.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "sla2.h"
#include "device.cuh"
#include "kernels.cuh"

using namespace sla2;

namespace {

constexpr unsigned long long DEFAULT_BUDGET_NS = kDefaultWaitBudgetNs;

unsigned long long g_budget_ns = DEFAULT_BUDGET_NS;

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int topk_count(int nk, float frac) {
  if (!(frac > 0.f) || !(frac <= 1.f) || nk < 1) return 0;
  long long k = (long long)std::floor((double)frac * (double)nk + 1e-3);
  if (k < 1) k = 1;
  if (k > nk) k = nk;
  return (int)k;
}

sla2_status check_desc(const sla2_desc* d, float frac, Shape* s) {
  if (!d) return SLA2_ERR_INVALID_ARG;
  if (d->B < 1 || d->H < 1 || d->N < 1 || d->d < 1) return SLA2_ERR_INVALID_ARG;
  if (!(frac > 0.f) || !(frac <= 1.f)) return SLA2_ERR_INVALID_ARG;
  if (d->quantize != 0 && d->quantize != 1) return SLA2_ERR_INVALID_ARG;
  if (d->out_dtype != 0 && d->out_dtype != 1) return SLA2_ERR_INVALID_ARG;
  if (d->N % BQ != 0 || (d->d != 64 && d->d != 128)) return SLA2_ERR_UNSUPPORTED;
  const long long BH = (long long)d->B * d->H;
  if (BH * d->N > 0x7fffffffLL || BH * (d->N / BKB) * d->d > 0x7fffffffLL) return SLA2_ERR_UNSUPPORTED;
  if (d->N / BKB > scores_topk_max_nk()) return SLA2_ERR_UNSUPPORTED;
  s->BH = (int)BH;
  s->N = d->N;
  s->d = d->d;
  s->nq = d->N / BQ;
  s->nk = d->N / BKB;
  s->k = topk_count(s->nk, frac);
  s->G = linear_chunks(s->BH, s->nk);
  return SLA2_OK;
}

// Workspace regions (each 256-byte aligned).
struct Layout {
  size_t qbar, ksum, c64, c32, kbs, A, Bk, scores, mask, idx, mask16, qhat, sq, vamax, csum, khat, sk, vhatT, sv, h, z,
      hpart, zpart, Htot, Ztot, htile, hscale, hi, Zi, z16, os, total;
};

Layout make_layout(const Shape& s, int quant) {
  Layout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  const size_t BH = s.BH, N = s.N, d = s.d, nq = s.nq, nk = s.nk, k = s.k;
  const size_t G = s.G;
  L.qbar = take(BH * nq * d * 4);
  L.ksum = take(BH * nk * d * 8);
  L.c64 = take(BH * d * 8);
  L.c32 = take(BH * d * 4);
  L.kbs = take(BH * nk * d * 4);
  L.A = take(BH * nq * d * 4);
  L.Bk = take(BH * nk * d * 4);
  L.scores = take(BH * nq * nk * 4);
  L.mask = take(BH * nq * nk);
  L.idx = take(BH * nq * k * 4);
  L.mask16 = take(BH * nq * ((nk + 7) & ~size_t(7)) * 2);   // fp16 mask, rows padded to 8
  L.qhat = take(quant ? BH * N * d : 0);
  L.sq = take(BH * nq * 4);
  L.vamax = take(BH * d * 4);
  L.csum = take(BH * d * 8);         // fp64 column sums of K (pool pass, atomic adds)
  L.khat = take(quant ? BH * N * d : 0);
  L.sk = take(BH * nk * 4);
  L.vhatT = take(BH * nk * d * BKB * (quant ? 1 : 2));
  L.sv = take(BH * d * 4);
  L.h = take(BH * nk * d * d * 2);   // fp16 -s h_j^T operand tiles
  L.z = take(BH * nk * d * 4);
  L.z16 = take(BH * nk * d * 2);     // fp16 z_j, the selected-state product's operand
  L.hpart = take(BH * G * d * d * 4);
  L.zpart = take(BH * G * d * 4);
  L.Htot = take(BH * d * d * 4);
  L.Ztot = take(BH * d * 4);
  L.htile = take(BH * d * d * 2);    // fp16 s H_total^T operand tiles
  L.hscale = take(BH * 4);
  L.hi = take(BH * nq * d * d * 2);  // fp16 s H_i^T operand images
  L.Zi = take(BH * nq * d * 4);
  L.os = take(BH * N * d * (quant ? 2 : 4));   // fp16 O_s / s_v, or fp32 O_s
  L.total = off;
  return L;
}

// Workspace of the backward pass: the router's regions, fp32 per-block states,
// and the gradient accumulators.
struct BwdLayout {
  Layout L;          // router and linear-state regions (h: fp32 h_j^T)
  size_t dos, dHacc, dZacc, dHtot, dZtot, total;
};

BwdLayout make_bwd_layout(const Shape& s) {
  BwdLayout B{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  const size_t BH = s.BH, d = s.d, nq = s.nq, nk = s.nk, k = s.k, G = s.G;
  Layout& L = B.L;
  L.qbar = take(BH * nq * d * 4);
  L.ksum = take(BH * nk * d * 8);
  L.c64 = take(BH * d * 8);
  L.c32 = take(BH * d * 4);
  L.kbs = take(BH * nk * d * 4);
  L.A = take(BH * nq * d * 4);
  L.Bk = take(BH * nk * d * 4);
  L.scores = take(BH * nq * nk * 4);
  L.mask = take(BH * nq * nk);
  L.idx = take(BH * nq * k * 4);
  L.sq = take(BH * nq * 4);
  L.vamax = take(BH * d * 4);
  L.csum = take(BH * d * 8);
  L.h = take(BH * nk * d * d * 4);
  L.z = take(BH * nk * d * 4);
  L.hpart = take(BH * G * d * d * 4);
  L.zpart = take(BH * G * d * 4);
  L.Htot = take(BH * d * d * 4);
  L.Ztot = take(BH * d * 4);
  B.dos = take(BH * nq * 4);
  B.dHacc = take(BH * nk * d * d * 4);
  B.dZacc = take(BH * nk * d * 4);
  B.dHtot = take(BH * d * d * 4);
  B.dZtot = take(BH * d * 4);
  B.total = off;
  return B;
}

template <class T>
T* at(const sla2_desc* d, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(d->workspace) + off);
}

// ---- TMA descriptors (driver entry point fetched once through the runtime)
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool get_encode() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}

// 2-D row-major map: `rows` rows of `cols` elements, box = box_cols x box_rows.
bool make_map(CUtensorMap* m, const void* ptr, CUtensorMapDataType dt, int esz, uint64_t cols, uint64_t rows,
              uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw) {
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * (cuuint64_t)esz};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

bool sla2::make_tmap_2d(CUtensorMap* m, const void* ptr, int esz, uint64_t cols, uint64_t rows, uint32_t box_cols,
                        uint32_t box_rows, int swizzle_bytes) {
  if (!get_encode()) return false;
  const CUtensorMapSwizzle sw = swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                      : CU_TENSOR_MAP_SWIZZLE_NONE;
  return make_map(m, ptr, esz == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, esz, cols,
                  rows, box_cols, box_rows, sw);
}

namespace {

sla2_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SLA2_OK : SLA2_ERR_CUDA; }

#define SLA2_TRY(expr)                                   \
  do {                                                   \
    cudaError_t _e = (expr);                             \
    if (_e != cudaSuccess) return SLA2_ERR_CUDA;         \
  } while (0)

// Router, first part: the pass over Q, K (and V) and the column means.
sla2_status router_head(const sla2_desc* d, const Shape& s, const Layout& L, const void* q, const void* k,
                        const void* v, int quant, cudaStream_t st) {
  // the column sums start at zero; with V given, so does its per-channel |V| max (V-hat
  // scales, fp16 scale of the linear state), which sits right before them
  if (v)
    SLA2_TRY(cudaMemsetAsync(at<void>(d, L.vamax), 0, L.csum - L.vamax + (size_t)s.BH * s.d * 8, st));
  else
    SLA2_TRY(cudaMemsetAsync(at<void>(d, L.csum), 0, (size_t)s.BH * s.d * 8, st));
  SLA2_TRY(launch_pool(s, q, k, v, at<float>(d, L.qbar), at<double>(d, L.ksum),
                       quant ? at<int8_t>(d, L.qhat) : nullptr, at<float>(d, L.sq),
                       v ? at<unsigned>(d, L.vamax) : nullptr, d->status, g_budget_ns, st, at<double>(d, L.csum)));
  SLA2_TRY(launch_colmean(s, at<double>(d, L.ksum), at<double>(d, L.c64), at<float>(d, L.c32), at<float>(d, L.kbs),
                           st, at<double>(d, L.csum)));
  return SLA2_OK;
}

// Router, second part: projections, logits and the hard top-k.
sla2_status router_tail(const sla2_desc* d, const Shape& s, const Layout& L, const float* wq, const float* wk,
                        uint8_t* mask, int32_t* idx, cudaStream_t st, uint16_t* mask16 = nullptr) {
  SLA2_TRY(launch_proj(s, d->H, at<float>(d, L.qbar), at<float>(d, L.kbs), wq, wk, at<float>(d, L.A),
                       at<float>(d, L.Bk), st));
  float* scores = d->dbg_scores ? d->dbg_scores : at<float>(d, L.scores);
  SLA2_TRY(launch_scores(s, at<float>(d, L.A), at<float>(d, L.Bk), scores, st));
  SLA2_TRY(launch_topk(s, scores, mask, idx, st, mask16));
  return SLA2_OK;
}

sla2_status run_router(const sla2_desc* d, const Shape& s, const Layout& L, const void* q, const void* k,
                       const void* v, const float* wq, const float* wk, uint8_t* mask, int32_t* idx, int quant,
                       cudaStream_t st) {
  sla2_status r = router_head(d, s, L, q, k, v, quant, st);
  if (r != SLA2_OK) return r;
  return router_tail(d, s, L, wq, wk, mask, idx, st);
}

// One auxiliary stream per device, created on the first forward call on that
// device and kept for the life of the process, on which the router's tail runs
// while the linear-state pass runs on the caller's stream (the two depend only
// on the column means). The fork / join events belong to it too; the mutex
// keeps each call's record / wait pairs together when several host threads
// enqueue forward calls at once.
struct AuxStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
constexpr int kMaxDevices = 64;
AuxStream g_aux[kMaxDevices];
std::mutex g_aux_mu;

cudaError_t aux_stream(AuxStream** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  AuxStream& a = g_aux[dev];
  if (!a.stream) {
    if ((e = cudaStreamCreateWithFlags(&a.stream, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&a.fork, cudaEventDisableTiming)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&a.join, cudaEventDisableTiming)) != cudaSuccess) return e;
  }
  *out = &a;
  return cudaSuccess;
}

// Copy streams and slot events of sla2_forward_host, one set per device,
// created on the first call there and kept for the life of the process. The
// slot events are re-recorded for every group; a wait always refers to the
// latest record, which the enqueue order below makes the right one.
struct HostPipe {
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr;
  cudaEvent_t in_ready[2] = {nullptr, nullptr}, comp_done[2] = {nullptr, nullptr}, out_done[2] = {nullptr, nullptr};
};
HostPipe g_pipe[kMaxDevices];
std::mutex g_pipe_mu;

cudaError_t host_pipe(HostPipe** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  HostPipe& p = g_pipe[dev];
  if (!p.h2d) {
    cudaStream_t a = nullptr, b = nullptr;
    if ((e = cudaStreamCreateWithFlags(&a, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaStreamCreateWithFlags(&b, cudaStreamNonBlocking)) != cudaSuccess) return e;
    cudaEvent_t* evs[7] = {&p.start, &p.in_ready[0], &p.in_ready[1], &p.comp_done[0], &p.comp_done[1],
                           &p.out_done[0], &p.out_done[1]};
    for (cudaEvent_t* ev : evs)
      if ((e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming)) != cudaSuccess) return e;
    p.d2h = b;
    p.h2d = a;   // set last: a set h2d marks a complete set
  }
  *out = &p;
  return cudaSuccess;
}

// Clears the caller's status word (if any) on the call's stream, so that a code
// left there by an earlier call is not read as this call's.
cudaError_t clear_status(const sla2_desc* d, cudaStream_t st) {
  if (!d->status) return cudaSuccess;
  return cudaMemsetAsync(d->status, 0, sizeof(unsigned), st);
}

}  // namespace

namespace {

// The forward pass for the description `desc` and the shape `s` (checked by the
// caller): `H` heads per batch index the projections and alpha.
sla2_status forward_body(const sla2_desc* desc, const Shape& s, int H, const Layout& L, const void* q,
                         const void* k, const void* v, const float* proj_q, const float* proj_k,
                         const float* alpha, void* out, cudaStream_t st) {
  const int quant = desc->quantize;
  if (!get_encode()) return SLA2_ERR_CUDA;
  auto mark = [&](int i) -> cudaError_t {
    if (!desc->stage_events) return cudaSuccess;
    return cudaEventRecord(static_cast<cudaEvent_t>(desc->stage_events[i]), st);
  };
  SLA2_TRY(mark(0));

  uint8_t* mask = at<uint8_t>(desc, L.mask);
  int32_t* idx = at<int32_t>(desc, L.idx);
  sla2_status r = router_head(desc, s, L, q, k, v, quant, st);
  if (r != SLA2_OK) return r;
  SLA2_TRY(mark(1));

  // fork: the linear state on the auxiliary stream, the router's tail on `st`. The
  // projection GEMM, enqueued on the GPU at the same time, takes the SMs first and
  // runs at full width; the logits and the top-k then fit beside the linear-state
  // CTAs and finish while it runs, so the sparse branch follows the linear state.
  std::lock_guard<std::mutex> aux_lock(g_aux_mu);
  AuxStream* aux = nullptr;
  SLA2_TRY(aux_stream(&aux));
  SLA2_TRY(cudaEventRecord(aux->fork, st));
  SLA2_TRY(cudaStreamWaitEvent(aux->stream, aux->fork, 0));

  LinearOut o{};
  o.h = at<void>(desc, L.h);
  o.h_mode = 2;
  o.z = at<float>(desc, L.z);
  o.hpart = at<float>(desc, L.hpart);
  o.zpart = at<float>(desc, L.zpart);
  o.khat = quant ? at<int8_t>(desc, L.khat) : nullptr;
  o.sk = at<float>(desc, L.sk);
  o.vhatT = at<void>(desc, L.vhatT);
  o.sv = at<float>(desc, L.sv);
  o.vamax = at<unsigned>(desc, L.vamax);
  o.quant = quant;
  o.status = desc->status;
  o.budget_ns = g_budget_ns;
  SLA2_TRY(launch_linear_state(s, k, v, at<float>(desc, L.c32), o, aux->stream));
  SLA2_TRY(launch_linear_reduce(s, o.hpart, o.zpart, o.vamax, at<float>(desc, L.Htot), at<float>(desc, L.Ztot),
                                at<uint16_t>(desc, L.htile), at<float>(desc, L.hscale), aux->stream, o.z,
                                at<uint16_t>(desc, L.z16)));
  SLA2_TRY(cudaEventRecord(aux->join, aux->stream));
  uint16_t* mask16 = s.k < s.nk ? at<uint16_t>(desc, L.mask16) : nullptr;
  r = router_tail(desc, s, L, proj_q, proj_k, mask, idx, st, mask16);
  if (r != SLA2_OK) return r;
  SLA2_TRY(cudaStreamWaitEvent(st, aux->join, 0));   // join
  SLA2_TRY(mark(2));

  // sparse branch: tensor maps over the (quantised) operands
  CUtensorMap tq, tk, tv;
  const uint64_t rows = (uint64_t)s.BH * s.N, vrows = (uint64_t)s.BH * s.nk * s.d;
  bool okm;
  if (quant) {
    const CUtensorMapSwizzle sw = s.d == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    okm = make_map(&tq, at<void>(desc, L.qhat), CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, s.d, rows, s.d, BQ, sw) &&
          make_map(&tk, at<void>(desc, L.khat), CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, s.d, rows, s.d, BKB, sw) &&
          make_map(&tv, at<void>(desc, L.vhatT), CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, BKB, vrows, BKB, s.d,
                   CU_TENSOR_MAP_SWIZZLE_64B);
  } else {
    okm = make_map(&tq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, s.d, rows, 64, BQ, CU_TENSOR_MAP_SWIZZLE_128B) &&
          make_map(&tk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, s.d, rows, 64, BKB, CU_TENSOR_MAP_SWIZZLE_128B) &&
          make_map(&tv, at<void>(desc, L.vhatT), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, BKB, vrows, BKB, s.d,
                   CU_TENSOR_MAP_SWIZZLE_128B);
  }
  if (!okm) return SLA2_ERR_CUDA;
  // O_s: fp16 O_s / s_v on the quantised path (the epilogue applies s_v and, when asked,
  // exports fp32 O_s), else fp32 (written straight into the export when there is one)
  void* os = (!quant && desc->dbg_os) ? static_cast<void*>(desc->dbg_os) : at<void>(desc, L.os);
  SparseArgs sa{idx, at<float>(desc, L.sq), at<float>(desc, L.sk), at<float>(desc, L.sv), os, desc->status, g_budget_ns};
  // the selected-state product does not depend on the sparse branch: it goes on the
  // auxiliary stream, enqueued after the sparse kernel, and takes the SMs that the
  // sparse branch's last CTAs leave
  const bool hsel_on = s.k < s.nk;
  if (hsel_on) SLA2_TRY(cudaEventRecord(aux->fork, st));
  SLA2_TRY(launch_sparse(s, quant, tq, tk, tv, sa, st));
  SLA2_TRY(mark(3));

  // the linear branch's s H_i^T and Z_i for every query block (one product with the mask)
  if (hsel_on) {
    SLA2_TRY(cudaStreamWaitEvent(aux->stream, aux->fork, 0));
    CUtensorMap tm, ti, tz;
    const uint64_t nk8 = ((uint64_t)s.nk + 7) & ~uint64_t(7);
    if (!make_map(&tm, mask16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, nk8, (uint64_t)s.BH * s.nq, 64, 128,
                  CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&ti, at<void>(desc, L.h), CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)s.d * s.d,
                  (uint64_t)s.BH * s.nk, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&tz, at<void>(desc, L.z16), CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)s.d,
                  (uint64_t)s.BH * s.nk, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B))
      return SLA2_ERR_CUDA;
    HselArgs ha{};
    ha.htile = at<uint16_t>(desc, L.htile);
    ha.Ztot = at<float>(desc, L.Ztot);
    ha.hi = at<uint16_t>(desc, L.hi);
    ha.Zi = at<float>(desc, L.Zi);
    ha.status = desc->status;
    ha.budget_ns = g_budget_ns;
    SLA2_TRY(launch_hsel(s, tm, ti, tz, ha, aux->stream));
    SLA2_TRY(cudaEventRecord(aux->join, aux->stream));
    SLA2_TRY(cudaStreamWaitEvent(st, aux->join, 0));
  }

  EpilogueArgs ea{};
  ea.q = q;
  ea.hi = at<uint16_t>(desc, L.hi);
  ea.Zi = at<float>(desc, L.Zi);
  ea.hscale = at<float>(desc, L.hscale);
  ea.os = os;
  ea.os_half = quant;
  ea.sv = at<float>(desc, L.sv);
  ea.os_dbg = quant ? desc->dbg_os : nullptr;
  ea.alpha = alpha;
  ea.H = H;
  ea.out = out;
  ea.out_f32 = desc->out_dtype;
  ea.ol_dbg = desc->dbg_ol;
  ea.status = desc->status;
  ea.budget_ns = g_budget_ns;
  CUtensorMap teq, tos, tout;
  if (!make_map(&teq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, s.d, rows, 64, BQ, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tos, quant ? os : q, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, s.d, rows, 64, BQ,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tout, desc->out_dtype ? q : out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, s.d, rows, 64, BQ,
                CU_TENSOR_MAP_SWIZZLE_128B))
    return SLA2_ERR_CUDA;
  SLA2_TRY(launch_epilogue(s, teq, tos, tout, ea, st));
  SLA2_TRY(mark(4));

  // debug exports
  auto cp = [&](void* dst, size_t off, size_t bytes) -> cudaError_t {
    if (!dst) return cudaSuccess;
    return cudaMemcpyAsync(dst, at<uint8_t>(desc, off), bytes, cudaMemcpyDeviceToDevice, st);
  };
  const size_t BH = s.BH;
  SLA2_TRY(cp(desc->dbg_mask, L.mask, BH * s.nq * s.nk));
  SLA2_TRY(cp(desc->dbg_idx, L.idx, BH * s.nq * s.k * 4));
  if (quant) {
    SLA2_TRY(cp(desc->dbg_qhat, L.qhat, BH * s.N * s.d));
    SLA2_TRY(cp(desc->dbg_khat, L.khat, BH * s.N * s.d));
    SLA2_TRY(cp(desc->dbg_vhat, L.vhatT, BH * s.nk * s.d * BKB));
    SLA2_TRY(cp(desc->dbg_qscale, L.sq, BH * s.nq * 4));
    SLA2_TRY(cp(desc->dbg_kscale, L.sk, BH * s.nk * 4));
    SLA2_TRY(cp(desc->dbg_vscale, L.sv, BH * s.d * 4));
  }
  return SLA2_OK;
}

}  // namespace

unsigned long long sla2::wait_budget_ns() { return g_budget_ns; }

extern "C" {

const char* sla2_status_string(sla2_status s) {
  switch (s) {
    case SLA2_OK: return "ok";
    case SLA2_ERR_INVALID_ARG: return "invalid argument";
    case SLA2_ERR_UNSUPPORTED: return "unsupported shape (N % 128 != 0, d not in {64,128}, or too large)";
    case SLA2_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case SLA2_ERR_CUDA: return "CUDA error";
    case SLA2_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait ran out";
  }
  return "unknown status";
}

int sla2_topk_count(int nk, float topk_frac) { return topk_count(nk, topk_frac); }

size_t sla2_workspace_size(const sla2_desc* desc, float topk_frac) {
  Shape s;
  if (check_desc(desc, topk_frac, &s) != SLA2_OK) return 0;
  return make_layout(s, desc->quantize).total;
}

// Test knob: the budget (ns) of every bounded device wait in later launches;
// 0 restores the default (declared in include/sla2_test.h).
void sla2_set_wait_budget_ns(unsigned long long ns) { g_budget_ns = ns ? ns : DEFAULT_BUDGET_NS; }

sla2_status sla2_router(const sla2_desc* desc, const void* q, const void* k, const float* proj_q,
                        const float* proj_k, float topk_frac, uint8_t* mask_out, int32_t* idx_out,
                        float* colmean_out, void* stream) {
  Shape s;
  sla2_status r = check_desc(desc, topk_frac, &s);
  if (r != SLA2_OK) return r;
  if (!q || !k || !proj_q || !proj_k || !mask_out || !idx_out) return SLA2_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(proj_q) || !aligned16(proj_k)) return SLA2_ERR_INVALID_ARG;
  const Layout L = make_layout(s, 0);
  if (!desc->workspace || desc->workspace_bytes < L.total ||
      (reinterpret_cast<uintptr_t>(desc->workspace) & 255u))
    return SLA2_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SLA2_TRY(clear_status(desc, st));
  r = run_router(desc, s, L, q, k, nullptr, proj_q, proj_k, mask_out, idx_out, 0, st);
  if (r != SLA2_OK) return r;
  if (colmean_out)
    SLA2_TRY(cudaMemcpyAsync(colmean_out, at<float>(desc, L.c32), (size_t)s.BH * s.d * 4, cudaMemcpyDeviceToDevice, st));
  return SLA2_OK;
}

sla2_status sla2_router_soft(const sla2_desc* desc, const void* q, const void* k, const float* proj_q,
                             const float* proj_k, float topk_frac, float tau, float* soft_out, float* lambda_out,
                             void* stream) {
  Shape s;
  sla2_status r = check_desc(desc, topk_frac, &s);
  if (r != SLA2_OK) return r;
  if (!q || !k || !proj_q || !proj_k || !soft_out) return SLA2_ERR_INVALID_ARG;
  if (!(tau > 0.f) || !(tau < INFINITY)) return SLA2_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(proj_q) || !aligned16(proj_k)) return SLA2_ERR_INVALID_ARG;
  const Layout L = make_layout(s, 0);
  if (!desc->workspace || desc->workspace_bytes < L.total ||
      (reinterpret_cast<uintptr_t>(desc->workspace) & 255u))
    return SLA2_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SLA2_TRY(clear_status(desc, st));
  r = router_head(desc, s, L, q, k, nullptr, 0, st);
  if (r != SLA2_OK) return r;
  SLA2_TRY(launch_proj(s, desc->H, at<float>(desc, L.qbar), at<float>(desc, L.kbs), proj_q, proj_k,
                       at<float>(desc, L.A), at<float>(desc, L.Bk), st));
  float* scores = desc->dbg_scores ? desc->dbg_scores : at<float>(desc, L.scores);
  SLA2_TRY(launch_scores(s, at<float>(desc, L.A), at<float>(desc, L.Bk), scores, st));
  SLA2_TRY(launch_soft_topk(s, scores, tau, soft_out, lambda_out, st));
  return SLA2_OK;
}

sla2_status sla2_linear_state(const sla2_desc* desc, const void* k, const void* v, const float* colmean,
                              float* h_out, float* z_out, float* Htot_out, float* Ztot_out, void* stream) {
  Shape s;
  sla2_status r = check_desc(desc, 1.f, &s);
  if (r != SLA2_OK) return r;
  if (!k || !v || !colmean || !h_out || !z_out || !Htot_out || !Ztot_out) return SLA2_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(h_out) || !aligned16(Htot_out)) return SLA2_ERR_INVALID_ARG;
  const Layout L = make_layout(s, 0);
  if (!desc->workspace || desc->workspace_bytes < L.total ||
      (reinterpret_cast<uintptr_t>(desc->workspace) & 255u))
    return SLA2_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SLA2_TRY(clear_status(desc, st));
  LinearOut o{};
  o.h = h_out;
  o.h_mode = 0;
  o.z = z_out;
  o.hpart = at<float>(desc, L.hpart);
  o.zpart = at<float>(desc, L.zpart);
  o.quant = 0;
  o.status = desc->status;
  o.budget_ns = g_budget_ns;
  SLA2_TRY(launch_linear_state(s, k, v, colmean, o, st));
  SLA2_TRY(launch_linear_reduce(s, o.hpart, o.zpart, nullptr, Htot_out, Ztot_out, nullptr, nullptr, st));
  return SLA2_OK;
}

sla2_status sla2_forward(const sla2_desc* desc, const void* q, const void* k, const void* v, const float* proj_q,
                         const float* proj_k, const float* alpha, float topk_frac, void* out, void* stream) {
  Shape s;
  sla2_status r = check_desc(desc, topk_frac, &s);
  if (r != SLA2_OK) return r;
  if (!q || !k || !v || !proj_q || !proj_k || !alpha || !out) return SLA2_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(proj_q) || !aligned16(proj_k) ||
      !aligned16(out))
    return SLA2_ERR_INVALID_ARG;
  if (out == q || out == k || out == v) return SLA2_ERR_INVALID_ARG;
  const int quant = desc->quantize;
  const Layout L = make_layout(s, quant);
  if (!desc->workspace || desc->workspace_bytes < L.total ||
      (reinterpret_cast<uintptr_t>(desc->workspace) & 255u))
    return SLA2_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SLA2_TRY(clear_status(desc, st));
  return forward_body(desc, s, desc->H, L, q, k, v, proj_q, proj_k, alpha, out, st);
}

size_t sla2_backward_workspace_size(const sla2_desc* desc, float topk_frac) {
  Shape s;
  if (check_desc(desc, topk_frac, &s) != SLA2_OK) return 0;
  return make_bwd_layout(s).total;
}

sla2_status sla2_backward(const sla2_desc* desc, const void* q, const void* k, const void* v, const float* proj_q,
                          const float* proj_k, const float* alpha, float topk_frac, const float* dout, float* dq,
                          float* dk, float* dv, float* dalpha, void* stream) {
  Shape s;
  sla2_status r = check_desc(desc, topk_frac, &s);
  if (r != SLA2_OK) return r;
  if (!q || !k || !v || !proj_q || !proj_k || !alpha || !dout || !dq || !dk || !dv || !dalpha)
    return SLA2_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(proj_q) || !aligned16(proj_k) ||
      !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return SLA2_ERR_INVALID_ARG;
  const BwdLayout B = make_bwd_layout(s);
  const Layout& L = B.L;
  if (!desc->workspace || desc->workspace_bytes < B.total ||
      (reinterpret_cast<uintptr_t>(desc->workspace) & 255u))
    return SLA2_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SLA2_TRY(clear_status(desc, st));
  // the forward's mask (router) and the per-key-block states (fp32 h_j^T)
  r = run_router(desc, s, L, q, k, nullptr, proj_q, proj_k, at<uint8_t>(desc, L.mask), at<int32_t>(desc, L.idx), 0,
                 st);
  if (r != SLA2_OK) return r;
  LinearOut o{};
  o.h = at<void>(desc, L.h);
  o.h_mode = 0;
  o.z = at<float>(desc, L.z);
  o.hpart = at<float>(desc, L.hpart);
  o.zpart = at<float>(desc, L.zpart);
  o.quant = 0;
  o.status = desc->status;
  o.budget_ns = g_budget_ns;
  SLA2_TRY(launch_linear_state(s, k, v, at<float>(desc, L.c32), o, st));
  SLA2_TRY(launch_linear_reduce(s, o.hpart, o.zpart, nullptr, at<float>(desc, L.Htot), at<float>(desc, L.Ztot),
                                nullptr, nullptr, st));
  const size_t E = (size_t)s.BH * s.N * s.d;
  SLA2_TRY(cudaMemsetAsync(dk, 0, E * 4, st));
  SLA2_TRY(cudaMemsetAsync(dv, 0, E * 4, st));
  SLA2_TRY(cudaMemsetAsync(dalpha, 0, (size_t)desc->H * s.nq * 4, st));
  SLA2_TRY(cudaMemsetAsync(at<uint8_t>(desc, B.dHacc), 0, B.total - B.dHacc, st));   // dHacc .. dZtot
  BackwardArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.c32 = at<float>(desc, L.c32);
  a.alpha = alpha;
  a.dout = dout;
  a.idx = at<int32_t>(desc, L.idx);
  a.hT = at<float>(desc, L.h);
  a.z = at<float>(desc, L.z);
  a.HtotT = at<float>(desc, L.Htot);
  a.Ztot = at<float>(desc, L.Ztot);
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.dalpha = dalpha;
  a.dos_sum = at<float>(desc, B.dos);
  a.dHacc = at<float>(desc, B.dHacc);
  a.dZacc = at<float>(desc, B.dZacc);
  a.dHtot = at<float>(desc, B.dHtot);
  a.dZtot = at<float>(desc, B.dZtot);
  SLA2_TRY(launch_backward(s, desc->H, a, st));
  return SLA2_OK;
}

size_t sla2_workspace_size_heads(const sla2_desc* desc, int h_count, float topk_frac) {
  Shape s;
  if (check_desc(desc, topk_frac, &s) != SLA2_OK) return 0;
  if (h_count < 1 || h_count > desc->H) return 0;
  s.BH = h_count;   // one batch index at a time; the chunking stays the full problem's
  return make_layout(s, desc->quantize).total;
}

sla2_status sla2_forward_heads(const sla2_desc* desc, int h_begin, int h_count, const void* q, const void* k,
                               const void* v, const float* proj_q, const float* proj_k, const float* alpha,
                               float topk_frac, void* out, void* stream) {
  Shape s;
  sla2_status r = check_desc(desc, topk_frac, &s);
  if (r != SLA2_OK) return r;
  if (h_begin < 0 || h_count < 1 || h_begin > desc->H - h_count) return SLA2_ERR_INVALID_ARG;
  if (!q || !k || !v || !proj_q || !proj_k || !alpha || !out) return SLA2_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(proj_q) || !aligned16(proj_k) ||
      !aligned16(out))
    return SLA2_ERR_INVALID_ARG;
  if (out == q || out == k || out == v) return SLA2_ERR_INVALID_ARG;
  if (desc->dbg_scores || desc->dbg_os || desc->dbg_ol || desc->dbg_qhat || desc->dbg_khat || desc->dbg_vhat ||
      desc->dbg_qscale || desc->dbg_kscale || desc->dbg_vscale || desc->dbg_mask || desc->dbg_idx ||
      desc->stage_events)
    return SLA2_ERR_INVALID_ARG;
  Shape sh = s;
  sh.BH = h_count;   // s.G (from all B x H heads) fixes the linear state's summation order
  const Layout L = make_layout(sh, desc->quantize);
  if (!desc->workspace || desc->workspace_bytes < L.total ||
      (reinterpret_cast<uintptr_t>(desc->workspace) & 255u))
    return SLA2_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SLA2_TRY(clear_status(desc, st));
  const size_t nd = (size_t)s.N * s.d, osz = desc->out_dtype ? 4 : 2;
  const float* pq = proj_q + (size_t)h_begin * s.d * s.d;
  const float* pk = proj_k + (size_t)h_begin * s.d * s.d;
  const float* al = alpha + (size_t)h_begin * s.nq;
  for (int b = 0; b < desc->B; ++b) {
    // heads [h_begin, h_begin + h_count) of batch index b are contiguous in [B][H][N][d]
    const size_t e0 = ((size_t)b * desc->H + h_begin) * nd;
    r = forward_body(desc, sh, h_count, L, static_cast<const uint16_t*>(q) + e0, static_cast<const uint16_t*>(k) + e0,
                     static_cast<const uint16_t*>(v) + e0, pq, pk, al, static_cast<uint8_t*>(out) + e0 * osz, st);
    if (r != SLA2_OK) return r;
  }
  return SLA2_OK;
}

}  // extern "C"

namespace {

// Workspace of sla2_forward_host: the forward workspace of one group of heads,
// the projections and alpha of all heads, then two slots of group inputs
// (Q, K, V) and outputs.
struct HostLayout {
  size_t fwd, proj_q, proj_k, alpha, slot[2], in_bytes, out_bytes, total;
};

HostLayout make_host_layout(const Shape& s, const sla2_desc* d, int hpg) {
  HostLayout HL{};
  Shape sh = s;
  sh.BH = hpg;
  size_t off = align256(make_layout(sh, d->quantize).total);
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  const size_t nd = (size_t)s.N * s.d;
  HL.fwd = 0;
  HL.proj_q = take((size_t)d->H * s.d * s.d * 4);
  HL.proj_k = take((size_t)d->H * s.d * s.d * 4);
  HL.alpha = take((size_t)d->H * s.nq * 4);
  HL.in_bytes = align256((size_t)hpg * nd * 2);
  HL.out_bytes = align256((size_t)hpg * nd * (d->out_dtype ? 4 : 2));
  for (int b = 0; b < 2; ++b) HL.slot[b] = take(3 * HL.in_bytes + HL.out_bytes);
  HL.total = off;
  return HL;
}

}  // namespace

extern "C" {

size_t sla2_forward_host_workspace_size(const sla2_desc* desc, int heads_per_group, float topk_frac) {
  Shape s;
  if (check_desc(desc, topk_frac, &s) != SLA2_OK) return 0;
  if (heads_per_group < 1 || heads_per_group > desc->H) return 0;
  return make_host_layout(s, desc, heads_per_group).total;
}

sla2_status sla2_forward_host(const sla2_desc* desc, int heads_per_group, const void* q, const void* k,
                              const void* v, const float* proj_q, const float* proj_k, const float* alpha,
                              float topk_frac, void* out, void* stream) {
  Shape s;
  sla2_status r = check_desc(desc, topk_frac, &s);
  if (r != SLA2_OK) return r;
  if (heads_per_group < 1 || heads_per_group > desc->H) return SLA2_ERR_INVALID_ARG;
  if (!q || !k || !v || !proj_q || !proj_k || !alpha || !out) return SLA2_ERR_INVALID_ARG;
  if (out == q || out == k || out == v) return SLA2_ERR_INVALID_ARG;
  if (desc->dbg_scores || desc->dbg_os || desc->dbg_ol || desc->dbg_qhat || desc->dbg_khat || desc->dbg_vhat ||
      desc->dbg_qscale || desc->dbg_kscale || desc->dbg_vscale || desc->dbg_mask || desc->dbg_idx ||
      desc->stage_events)
    return SLA2_ERR_INVALID_ARG;
  const HostLayout HL = make_host_layout(s, desc, heads_per_group);
  if (!desc->workspace || desc->workspace_bytes < HL.total ||
      (reinterpret_cast<uintptr_t>(desc->workspace) & 255u))
    return SLA2_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> pipe_lock(g_pipe_mu);
  HostPipe* p = nullptr;
  SLA2_TRY(host_pipe(&p));
  SLA2_TRY(clear_status(desc, st));
  // the copy streams start after everything already enqueued on `stream`
  // (an earlier call may still be reading the same workspace)
  SLA2_TRY(cudaEventRecord(p->start, st));
  SLA2_TRY(cudaStreamWaitEvent(p->h2d, p->start, 0));
  SLA2_TRY(cudaStreamWaitEvent(p->d2h, p->start, 0));
  const int H = desc->H;
  const size_t dd = (size_t)s.d * s.d, nd = (size_t)s.N * s.d, osz = desc->out_dtype ? 4 : 2;
  float* pq = at<float>(desc, HL.proj_q);
  float* pk = at<float>(desc, HL.proj_k);
  float* al = at<float>(desc, HL.alpha);
  SLA2_TRY(cudaMemcpyAsync(pq, proj_q, (size_t)H * dd * 4, cudaMemcpyHostToDevice, p->h2d));
  SLA2_TRY(cudaMemcpyAsync(pk, proj_k, (size_t)H * dd * 4, cudaMemcpyHostToDevice, p->h2d));
  SLA2_TRY(cudaMemcpyAsync(al, alpha, (size_t)H * s.nq * 4, cudaMemcpyHostToDevice, p->h2d));
  int g = 0;
  for (int b = 0; b < desc->B; ++b) {
    for (int h0 = 0; h0 < H; h0 += heads_per_group, ++g) {
      const int hc = H - h0 < heads_per_group ? H - h0 : heads_per_group;
      const int sl = g & 1;
      uint8_t* slot = at<uint8_t>(desc, HL.slot[sl]);
      uint8_t* dq = slot;
      uint8_t* dk = slot + HL.in_bytes;
      uint8_t* dv = slot + 2 * HL.in_bytes;
      uint8_t* dout = slot + 3 * HL.in_bytes;
      const size_t e0 = ((size_t)b * H + h0) * nd;   // first element of the group in [B][H][N][d]
      const size_t in_b = (size_t)hc * nd * 2, out_b = (size_t)hc * nd * osz;
      // inputs: the slot was last read by the forward of group g - 2
      if (g >= 2) SLA2_TRY(cudaStreamWaitEvent(p->h2d, p->comp_done[sl], 0));
      SLA2_TRY(cudaMemcpyAsync(dq, static_cast<const uint8_t*>(q) + e0 * 2, in_b, cudaMemcpyHostToDevice, p->h2d));
      SLA2_TRY(cudaMemcpyAsync(dk, static_cast<const uint8_t*>(k) + e0 * 2, in_b, cudaMemcpyHostToDevice, p->h2d));
      SLA2_TRY(cudaMemcpyAsync(dv, static_cast<const uint8_t*>(v) + e0 * 2, in_b, cudaMemcpyHostToDevice, p->h2d));
      SLA2_TRY(cudaEventRecord(p->in_ready[sl], p->h2d));
      // compute: the output slot was last copied out for group g - 2
      SLA2_TRY(cudaStreamWaitEvent(st, p->in_ready[sl], 0));
      if (g >= 2) SLA2_TRY(cudaStreamWaitEvent(st, p->out_done[sl], 0));
      Shape sh = s;
      sh.BH = hc;   // s.G (from all B x H heads) fixes the linear state's summation order
      const Layout L = make_layout(sh, desc->quantize);
      r = forward_body(desc, sh, hc, L, dq, dk, dv, pq + (size_t)h0 * dd, pk + (size_t)h0 * dd,
                       al + (size_t)h0 * s.nq, dout, st);
      if (r != SLA2_OK) return r;
      SLA2_TRY(cudaEventRecord(p->comp_done[sl], st));
      // output
      SLA2_TRY(cudaStreamWaitEvent(p->d2h, p->comp_done[sl], 0));
      SLA2_TRY(cudaMemcpyAsync(static_cast<uint8_t*>(out) + e0 * osz, dout, out_b, cudaMemcpyDeviceToHost, p->d2h));
      SLA2_TRY(cudaEventRecord(p->out_done[sl], p->d2h));
    }
  }
  // `stream` reaches this point once the last output copy (and so every one) is done
  SLA2_TRY(cudaStreamWaitEvent(st, p->out_done[(g - 1) & 1], 0));
  return SLA2_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Self-test of the bounded device wait (declared in include/sla2_test.h): one
// warp waits on an mbarrier that nothing arrives on; after `budget_ns` the
// wait gives up, writes SLA2_ERR_DEVICE_TIMEOUT into *status and the kernel
// returns normally.
namespace {
__global__ void timeout_probe_kernel(unsigned* status, unsigned long long budget_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sla2::mbar_init(&bar, 1);
    abort_flag = 0;
    sla2::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) sla2::mbar_wait(&bar, 0, &abort_flag, status, budget_ns);
}
}  // namespace

extern "C" sla2_status sla2_selftest_timeout(unsigned* status, unsigned long long budget_ns, void* stream) {
  if (!status || budget_ns == 0 || budget_ns > 10000000000ull) return SLA2_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SLA2_TRY(cudaMemsetAsync(status, 0, sizeof(unsigned), st));
  timeout_probe_kernel<<<1, 32, 0, st>>>(status, budget_ns);
  return cuda_status(cudaGetLastError());
}
