// The linear branch's per-query-block state (SLA2 summary page, step 3:
// H_i = H_total - sum of the selected h_j, Z_i likewise; SLA2 detail page §7
// note 2: the h_j are precomputed per key block and accumulated per query
// block), for every (head, query block) at once.
//
// The selected blocks' share is a product with the router's block mask M
// (nq x nk, 0 / 1): G = M S, where row j of S is the linear-state pass's fp16
// operand image -s h_j^T (d*d values in the epilogue's swizzled K-major
// layout; the product acts on each position of the image alike). On B200 the
// dense product on the tensor cores is cheaper than gathering the k selected
// images of every query block (k * 32 KB per block from L2 at d = 128): it
// reads each image once per 128 query blocks, and its 2 * nq * nk * d^2 flops
// take a few tens of microseconds. Then
//   s H_i^T = s H_total^T + G_i          (fp32 accumulation, rounded once to fp16)
// is written in the same operand layout, and
//   Z_i     = Z_total - sum_{j selected} z_j     (fp32, ascending j, CUDA cores)
// alongside it.
//
// One CTA per (128 query blocks, 256 image positions, head); 128 threads:
// warp 0 lane 0 issues the TMA loads (A = M as fp16 [nq][nk8], K-major; B = the
// images as a [nk][d*d] fp16 matrix, MN-major, 128-byte swizzle) into a
// 2-stage ring, warp 1 lane 0 issues the tcgen05 kind::f16 MMAs (M = 128,
// N = 256, fp32 accumulator in TMEM); then every thread reads one accumulator
// row (a query block) back, adds s H_total^T, rounds and stores. Before that,
// while the MMAs run, each thread forms Z_i for its query block on the
// 256 / d features that belong to this CTA's image positions.
#include <cuda_fp16.h>

#include "device.cuh"
#include "kernels.cuh"

namespace sla2 {

namespace {

constexpr int HS_THREADS = 128;
constexpr int HS_BM = 128;      // query blocks per tile
constexpr int HS_BN = 256;      // image positions per tile
constexpr int HS_BK = 64;       // key blocks per stage
constexpr int HS_NST = 2;       // stages

struct HsCfg {
  static constexpr int A_BYTES = HS_BM * HS_BK * 2;                // 16 KB, K-major, 128-byte rows
  static constexpr int SLAB = HS_BK * 128;                         // 64 key rows x 64 positions (8 KB)
  static constexpr int B_BYTES = (HS_BN / 64) * SLAB;              // 32 KB, MN-major, four slabs
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int OFF_HT = HS_NST * STAGE;                    // s H_total^T positions of the tile (fp32)
  static constexpr int OFF_BAR = OFF_HT + HS_BN * 4;
  static constexpr int SMEM = OFF_BAR + 8 * (2 * HS_NST + 2) + 16 + 1024;
  // fp16 x fp16 -> fp32, M = 128, N = 256, A K-major, B MN-major (bit 16)
  static constexpr uint32_t IDESC = make_idesc(1, 0, 0, HS_BM, HS_BN) | (1u << 16);
  static_assert(2 * (SMEM + 1024) <= 233472, "two CTAs per SM");
};

__device__ __forceinline__ uint32_t h2u(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <int D>
__global__ void __launch_bounds__(HS_THREADS, 2) hsel_kernel(const __grid_constant__ CUtensorMap tmask,
                                                             const __grid_constant__ CUtensorMap timg, Shape s,
                                                             HselArgs a) {
  using C = HsCfg;
  constexpr int FPT = HS_BN / D;                 // Z features per CTA (2 at d = 128, 4 at d = 64)
  extern __shared__ uint8_t hsm_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(hsm_raw) + 1023) & ~uintptr_t(1023));
  float* ht = reinterpret_cast<float*>(base + C::OFF_HT);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + C::OFF_BAR);   // [NST]
  uint64_t* empty = full + HS_NST;                                    // [NST]
  uint64_t* done = empty + HS_NST;
  uint64_t* drain = done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_flag = reinterpret_cast<int*>(drain + 1) + 1;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = blockIdx.x * HS_BM, e0 = blockIdx.y * HS_BN, bh = blockIdx.z;
  const int nkt = (s.nk + HS_BK - 1) / HS_BK;

  if (tid == 0) {
    for (int i = 0; i < HS_NST; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
    }
    mbar_init(done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, HS_BN);
    tmem_relinquish();
  }
  // s H_total^T at this tile's positions, for the epilogue
  for (int c = tid; c < HS_BN; c += HS_THREADS)
    ht[c] = __half2float(__ushort_as_half(a.htile[(size_t)bh * D * D + e0 + c]));
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  bool ok = true;
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int n = 0;
      for (; n < nkt; ++n) {
        const int st = n % HS_NST;
        if (n >= HS_NST && !mbar_wait(empty + st, ((n / HS_NST) - 1) & 1, abort_flag, a.status, a.budget_ns)) {
          ok = false;
          break;
        }
        uint8_t* sa = base + st * C::STAGE;
        mbar_arrive_expect_tx(full + st, (uint32_t)C::STAGE);
        tma_load_2d(sa, &tmask, full + st, n * HS_BK, bh * s.nq + m0);
#pragma unroll
        for (int sl = 0; sl < HS_BN / 64; ++sl)
          tma_load_2d(sa + C::A_BYTES + sl * C::SLAB, &timg, full + st, e0 + sl * 64, bh * s.nk + n * HS_BK);
      }
      if (!ok)   // copies in flight land before the CTA releases its shared memory
        for (int q = n > HS_NST ? n - HS_NST : 0; q < n; ++q)
          mbar_wait_drain(full + q % HS_NST, (q / HS_NST) & 1, 20000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool issued = false;
      for (int n = 0; n < nkt; ++n) {
        const int st = n % HS_NST;
        if (!mbar_wait(full + st, (n / HS_NST) & 1, abort_flag, a.status, a.budget_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_u32(base + st * C::STAGE);
#pragma unroll
        for (int ks = 0; ks < HS_BK / 16; ++ks) {
          const uint64_t ad = make_sdesc(sa + ks * 32, 1024, LAYOUT_SW128);
          const uint64_t bd = make_sdesc(sa + C::A_BYTES + ks * 2048, 1024, LAYOUT_SW128, C::SLAB);
          mma_f16(tmem, ad, bd, C::IDESC, (n > 0 || ks > 0) ? 1u : 0u);
        }
        issued = true;
        tc_commit(empty + st);
      }
      if (ok) {
        tc_commit(done);
      } else if (issued) {   // issued MMAs finish before TMEM and shared memory are released
        tc_commit(drain);
        mbar_wait_drain(drain, 0, 20000000ull);
      }
    }
  }
  __syncwarp();

  // ------------------------------------------------------------ Z_i (overlaps the MMAs)
  const int row = m0 + tid;                      // query block of this thread = TMEM lane
  if (row < s.nq) {
    const int f0 = blockIdx.y * FPT;
    const int32_t* sel = a.idx + ((size_t)bh * s.nq + row) * s.k;
    float zacc[FPT];
#pragma unroll
    for (int f = 0; f < FPT; ++f) zacc[f] = a.Ztot[(size_t)bh * D + f0 + f];
    // eight selected blocks at a time: their indices, then their z slices, all in flight
    // together; subtracted in ascending order
    const float* zh = a.z + (size_t)bh * s.nk * D + f0;
    for (int n0 = 0; n0 < s.k; n0 += 8) {
      int jj[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) jj[u] = n0 + u < s.k ? __ldg(sel + n0 + u) : -1;
      float zz[8][FPT];
#pragma unroll
      for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int f = 0; f < FPT; ++f) zz[u][f] = jj[u] >= 0 ? __ldg(zh + (size_t)jj[u] * D + f) : 0.f;
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (jj[u] >= 0)
#pragma unroll
          for (int f = 0; f < FPT; ++f) zacc[f] -= zz[u][f];
    }
#pragma unroll
    for (int f = 0; f < FPT; ++f) a.Zi[((size_t)bh * s.nq + row) * D + f0 + f] = zacc[f];
  }

  // ------------------------------------------------------------ epilogue: s H_i^T = s H_total^T + G_i
  bool dok = mbar_wait(done, 0, abort_flag, a.status, a.budget_ns);
  dok = __all_sync(0xffffffffu, dok);
  tc_fence_after();
  if (dok) {
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    uint16_t* dst = a.hi + ((size_t)bh * s.nq + row) * D * D + e0;
#pragma unroll 1
    for (int cc = 0; cc < HS_BN / 32; ++cc) {
      uint32_t v[32];
      tmem_ld32(tmem + lane_base + (uint32_t)(cc * 32), v);
      tmem_wait_ld();
      if (row < s.nq) {
#pragma unroll
        for (int q = 0; q < 32; q += 8) {
          const float* h = ht + cc * 32 + q;
          *reinterpret_cast<uint4*>(dst + cc * 32 + q) =
              make_uint4(h2u(h[0] + __uint_as_float(v[q]), h[1] + __uint_as_float(v[q + 1])),
                         h2u(h[2] + __uint_as_float(v[q + 2]), h[3] + __uint_as_float(v[q + 3])),
                         h2u(h[4] + __uint_as_float(v[q + 4]), h[5] + __uint_as_float(v[q + 5])),
                         h2u(h[6] + __uint_as_float(v[q + 6]), h[7] + __uint_as_float(v[q + 7])));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, HS_BN);
  }
}

}  // namespace

size_t hsel_smem_bytes() { return (size_t)HsCfg::SMEM; }

cudaError_t launch_hsel(const Shape& s, const CUtensorMap& tmask, const CUtensorMap& timg, const HselArgs& a,
                        cudaStream_t st) {
  const dim3 grid((s.nq + HS_BM - 1) / HS_BM, (s.d * s.d) / HS_BN, s.BH);
  if (s.d == 128) {
    cudaFuncSetAttribute(hsel_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, HsCfg::SMEM);
    hsel_kernel<128><<<grid, HS_THREADS, HsCfg::SMEM, st>>>(tmask, timg, s, a);
  } else {
    cudaFuncSetAttribute(hsel_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, HsCfg::SMEM);
    hsel_kernel<64><<<grid, HS_THREADS, HsCfg::SMEM, st>>>(tmask, timg, s, a);
  }
  return cudaGetLastError();
}

}  // namespace sla2
