// sla2_router_noalloc: the router (K smoothing, pooling, projections, logits,
// hard top-k) with its scratch memory in a fixed device array compiled into
// this library, for callers that cannot allocate device memory. Examples are
// a plugin inside a host framework that owns every device allocation (a
// serving runtime with a pre-sized memory pool), or code on a latency-critical
// path where cudaMalloc is not allowed because it can synchronise the device.
// The caller still passes the inputs and the outputs; nothing here calls
// cudaMalloc, cudaFree or any allocating routine.
//
// The array below is part of the module: every GPU that loads libsla2.so holds
// its 16 MiB until the process exits. All calls share it, so calls whose
// kernels may overlap on the GPU (different streams, or different host
// threads) race on it and must be serialised by the caller. It keeps whatever
// the last call left in it; none of the router's scratch needs to start at
// zero (every region is fully written before it is read), so nothing is
// cleared between calls.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "sla2.h"
#include "kernels.cuh"

namespace {

constexpr size_t kScratchBytes = SLA2_ROUTER_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_router_scratch[kScratchBytes];

// Host code may not use g_router_scratch as a device address (on the host it
// names a stand-in object); the device address is looked up once per device.
constexpr int kMaxDevices = 64;
void* g_scratch_dev[kMaxDevices] = {};
std::mutex g_scratch_mu;

cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_dev[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_router_scratch);   // with `dev` current
    if (e != cudaSuccess) return e;
    g_scratch_dev[dev] = p;
  }
  *out = g_scratch_dev[dev];
  return cudaSuccess;
}

inline size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

struct RouterScratch {
  size_t qbar, ksum, c64, c32, kbs, A, Bk, scores, total;
};

RouterScratch router_layout(const sla2::Shape& s) {
  RouterScratch L{};
  size_t off = 0;
  auto take = [&](size_t b) {
    const size_t o = off;
    off += al256(b);
    return o;
  };
  const size_t BH = s.BH, d = s.d, nq = s.nq, nk = s.nk;
  L.qbar = take(BH * nq * d * 4);
  L.ksum = take(BH * nk * d * 8);
  L.c64 = take(BH * d * 8);
  L.c32 = take(BH * d * 4);
  L.kbs = take(BH * nk * d * 4);
  L.A = take(BH * nq * d * 4);
  L.Bk = take(BH * nk * d * 4);
  L.scores = take(BH * nq * nk * 4);
  L.total = off;
  return L;
}

}  // namespace

extern "C" sla2_status sla2_router_noalloc(const sla2_desc* desc, const void* q, const void* k,
                                           const float* proj_q, const float* proj_k, float topk_frac,
                                           uint8_t* mask_out, int32_t* idx_out, float* colmean_out, void* stream) {
  if (!desc) return SLA2_ERR_INVALID_ARG;
  if (desc->B < 1 || desc->H < 1 || desc->N < 1 || desc->d < 1) return SLA2_ERR_INVALID_ARG;
  if (!(topk_frac > 0.f) || !(topk_frac <= 1.f)) return SLA2_ERR_INVALID_ARG;
  if (desc->N % sla2::BQ != 0 || (desc->d != 64 && desc->d != 128)) return SLA2_ERR_UNSUPPORTED;
  if (!q || !k || !proj_q || !proj_k || !mask_out || !idx_out) return SLA2_ERR_INVALID_ARG;
  auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!a16(q) || !a16(k) || !a16(proj_q) || !a16(proj_k)) return SLA2_ERR_INVALID_ARG;
  const long long BH = (long long)desc->B * desc->H;
  if (BH * desc->N > 0x7fffffffLL || desc->N / sla2::BKB > sla2::scores_topk_max_nk()) return SLA2_ERR_UNSUPPORTED;
  sla2::Shape s{};
  s.BH = (int)BH;
  s.N = desc->N;
  s.d = desc->d;
  s.nq = desc->N / sla2::BQ;
  s.nk = desc->N / sla2::BKB;
  long long kk = (long long)std::floor((double)topk_frac * (double)s.nk + 1e-3);
  s.k = (int)(kk < 1 ? 1 : (kk > s.nk ? s.nk : kk));
  const RouterScratch L = router_layout(s);
  if (L.total > kScratchBytes) return SLA2_ERR_WORKSPACE;   // larger than the fixed array

  void* base = nullptr;
  if (scratch_address(&base) != cudaSuccess) return SLA2_ERR_CUDA;
  unsigned char* p = static_cast<unsigned char*>(base);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (desc->status && cudaMemsetAsync(desc->status, 0, sizeof(unsigned), st) != cudaSuccess) return SLA2_ERR_CUDA;
  auto f32 = [&](size_t off) { return reinterpret_cast<float*>(p + off); };
  auto f64 = [&](size_t off) { return reinterpret_cast<double*>(p + off); };
  if (sla2::launch_pool(s, q, k, nullptr, f32(L.qbar), f64(L.ksum), nullptr, nullptr, nullptr, desc->status,
                        sla2::wait_budget_ns(), st) != cudaSuccess)
    return SLA2_ERR_CUDA;
  if (sla2::launch_colmean(s, f64(L.ksum), f64(L.c64), f32(L.c32), f32(L.kbs), st) != cudaSuccess)
    return SLA2_ERR_CUDA;
  if (sla2::launch_proj(s, desc->H, f32(L.qbar), f32(L.kbs), proj_q, proj_k, f32(L.A), f32(L.Bk), st) !=
      cudaSuccess)
    return SLA2_ERR_CUDA;
  float* scores = desc->dbg_scores ? desc->dbg_scores : f32(L.scores);
  if (sla2::launch_scores(s, f32(L.A), f32(L.Bk), scores, st) != cudaSuccess) return SLA2_ERR_CUDA;
  if (sla2::launch_topk(s, scores, mask_out, idx_out, st) != cudaSuccess) return SLA2_ERR_CUDA;
  if (colmean_out &&
      cudaMemcpyAsync(colmean_out, f32(L.c32), (size_t)s.BH * s.d * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return SLA2_ERR_CUDA;
  return SLA2_OK;
}
