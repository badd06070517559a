// The linear branch's per-query-block state (SLA2 summary page, step 3:
// H_i = H_total - sum of the selected h_j; SLA2 detail page §7 note 2: the h_j
// are precomputed per key block and accumulated per query block), for every
// (head, query block) at once.
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
// is written in the same operand layout, where the epilogue reads it. The same
// product with the fp16 z_j as rows gives Z_i = Z_total - sum of the selected z_j
// (one more tile of N = d per 128 query blocks, written as fp32).
//
// Persistent CTAs (one per SM) walk the tiles (head, 256 image positions, 128
// query blocks; query-block tiles of the same positions on neighbouring CTAs, so
// an image tile is fetched from HBM once and re-read from L2). 192 threads:
//   warp 0    TMA producer: per tile and 64-key-block step, A = M as fp16
//             [nq][nk8] (K-major) and B = the images as a [nk][d*d] fp16 matrix
//             (MN-major, four 64-position slabs), 128-byte swizzle, into a
//             4-stage ring that runs on across tiles;
//   warp 1    MMA issuer: tcgen05 kind::f16, M = 128, N = 256, into one of two
//             TMEM accumulators (the other one is being read out);
//   warps 2-5 per tile: the tile's s H_total^T positions into shared memory,
//             then the accumulator row of their query block (one TMEM lane
//             each) + s H_total^T, rounded and stored through per-warp staging.
#include <cuda_fp16.h>

#include "device.cuh"
#include "kernels.cuh"

namespace sla2 {

namespace {

constexpr int HS_THREADS = 192;
constexpr int HS_BM = 128;        // query blocks per tile
constexpr int HS_BN = 256;        // image positions per tile
constexpr int HS_BK = 64;         // key blocks per stage
constexpr int HS_NST = 4;         // stages

struct HsCfg {
  static constexpr int A_BYTES = HS_BM * HS_BK * 2;                // 16 KB, K-major, 128-byte rows
  static constexpr int SLAB = HS_BK * 128;                         // 64 key rows x 64 positions (8 KB)
  static constexpr int B_BYTES = (HS_BN / 64) * SLAB;              // 32 KB, MN-major, four slabs
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int OFF_STG = HS_NST * STAGE;                  // output staging, 4 warps x 32 rows x 128 B
  static constexpr int OFF_HT = OFF_STG + 4 * 32 * 128;           // s H_total^T at the tile's positions (fp32)
  static constexpr int OFF_BAR = OFF_HT + HS_BN * 4;
  static constexpr int NBAR = 2 * HS_NST + 4 + 1;                  // full, empty [NST]; tfull, tfree [2]; drain
  static constexpr int SMEM = OFF_BAR + 8 * NBAR + 16 + 1024;
  static_assert(SMEM <= 232448, "dynamic shared memory per CTA (227 KB)");
  // fp16 x fp16 -> fp32, M = 128, N = 256 (image tiles) or d (the z tile), A K-major,
  // B MN-major (bit 16)
  static constexpr uint32_t IDESC = make_idesc(1, 0, 0, HS_BM, HS_BN) | (1u << 16);
  static constexpr uint32_t IDESC_Z128 = make_idesc(1, 0, 0, HS_BM, 128) | (1u << 16);
  static constexpr uint32_t IDESC_Z64 = make_idesc(1, 0, 0, HS_BM, 64) | (1u << 16);
};

__device__ __forceinline__ uint32_t h2u(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <int D>
__global__ void __launch_bounds__(HS_THREADS, 1) hsel_kernel(const __grid_constant__ CUtensorMap tmask,
                                                             const __grid_constant__ CUtensorMap timg,
                                                             const __grid_constant__ CUtensorMap tz, Shape s,
                                                             HselArgs a) {
  using C = HsCfg;
  constexpr int NT = D * D / HS_BN + 1;          // position tiles per head, the last one z
  extern __shared__ uint8_t hsm_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(hsm_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(base + C::OFF_BAR);   // [NST]
  uint64_t* empty = full + HS_NST;                                    // [NST]
  uint64_t* tfull = empty + HS_NST;                                   // [2] accumulator complete
  uint64_t* tfree = tfull + 2;                                        // [2] accumulator read out
  uint64_t* drain = tfree + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(full + C::NBAR);
  int* abort_flag = reinterpret_cast<int*>(full + C::NBAR) + 1;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nmt = (s.nq + HS_BM - 1) / HS_BM;    // query-block tiles per head
  const int tiles = s.BH * NT * nmt;
  const int nkt = (s.nk + HS_BK - 1) / HS_BK;
  // tile t: query-block tile fastest, then position tile, then head
  auto tile_of = [&](int t, int& bh, int& m0, int& e0) {
    m0 = (t % nmt) * HS_BM;
    e0 = ((t / nmt) % NT) * HS_BN;
    bh = t / (nmt * NT);
  };

  if (tid == 0) {
    for (int i = 0; i < HS_NST; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(tfull + i, 1);
      mbar_init(tfree + i, 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 2 * HS_BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t g = 0;   // stages filled, over all tiles
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
        int bh, m0, e0;
        tile_of(t, bh, m0, e0);
        for (int n = 0; n < nkt; ++n, ++g) {
          const int st = (int)(g % HS_NST);
          if (g >= (uint32_t)HS_NST &&
              !mbar_wait(empty + st, ((g / HS_NST) - 1) & 1, abort_flag, a.status, a.budget_ns)) {
            ok = false;
            break;
          }
          uint8_t* sa = base + st * C::STAGE;
          const bool zt = e0 == (NT - 1) * HS_BN;   // the z tile: D columns of z_j
          mbar_arrive_expect_tx(full + st, (uint32_t)(C::A_BYTES + (zt ? (D / 64) * C::SLAB : C::B_BYTES)));
          tma_load_2d(sa, &tmask, full + st, n * HS_BK, bh * s.nq + m0);
          if (zt) {
#pragma unroll
            for (int sl = 0; sl < D / 64; ++sl)
              tma_load_2d(sa + C::A_BYTES + sl * C::SLAB, &tz, full + st, sl * 64, bh * s.nk + n * HS_BK);
          } else {
#pragma unroll
            for (int sl = 0; sl < HS_BN / 64; ++sl)
              tma_load_2d(sa + C::A_BYTES + sl * C::SLAB, &timg, full + st, e0 + sl * 64, bh * s.nk + n * HS_BK);
          }
        }
      }
      if (!ok)   // copies in flight land before the CTA releases its shared memory
        for (uint32_t q = g > (uint32_t)HS_NST ? g - HS_NST : 0u; q < g; ++q)
          mbar_wait_drain(full + q % HS_NST, (q / HS_NST) & 1, 20000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t g = 0;
      int i = 0;        // tiles of this CTA
      bool ok = true, issued = false;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++i) {
        const int acc = i & 1;
        const bool zt = (t / nmt) % NT == NT - 1;
        const uint32_t idesc = zt ? (D == 128 ? C::IDESC_Z128 : C::IDESC_Z64) : C::IDESC;
        if (i >= 2 && !mbar_wait(tfree + acc, ((i >> 1) - 1) & 1, abort_flag, a.status, a.budget_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int n = 0; n < nkt; ++n, ++g) {
          const int st = (int)(g % HS_NST);
          if (!mbar_wait(full + st, (g / HS_NST) & 1, abort_flag, a.status, a.budget_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(base + st * C::STAGE);
#pragma unroll
          for (int ks = 0; ks < HS_BK / 16; ++ks) {
            const uint64_t ad = make_sdesc(sa + ks * 32, 1024, LAYOUT_SW128);
            const uint64_t bd = make_sdesc(sa + C::A_BYTES + ks * 2048, 1024, LAYOUT_SW128, C::SLAB);
            mma_f16(tmem + (uint32_t)(acc * HS_BN), ad, bd, idesc, (n > 0 || ks > 0) ? 1u : 0u);
          }
          issued = true;
          tc_commit(empty + st);
        }
        if (ok) tc_commit(tfull + acc);
      }
      if (!ok && issued) {   // issued MMAs finish before TMEM and shared memory are released
        tc_commit(drain);
        mbar_wait_drain(drain, 0, 20000000ull);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue warps
    const int qd = warp & 3;                     // TMEM lane quadrant
    const int lr = qd * 32 + lane;               // accumulator row (query block within the tile)
    const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
    // this thread's two s H_total^T positions of a tile (fp16 pair), loaded one tile ahead
    // so that the L2 latency is not paid at the start of each tile
    auto ht_load = [&](int t2) -> uint32_t {
      if (t2 >= tiles) return 0u;
      int bh2, m2, e2;
      tile_of(t2, bh2, m2, e2);
      if (e2 == (NT - 1) * HS_BN) return 0u;   // the z tile has none
      return __ldg(reinterpret_cast<const uint32_t*>(a.htile + (size_t)bh2 * D * D + e2) + lr);
    };
    uint32_t hw_next = ht_load(blockIdx.x);
    int i = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
      int bh, m0, e0;
      tile_of(t, bh, m0, e0);
      const int acc = i & 1;
      const uint32_t hw = hw_next;
      hw_next = ht_load(t + gridDim.x);
      if (e0 == (NT - 1) * HS_BN) {
        // the z tile: Z_i = Z_total - G_i, fp32, one query block per thread
        bool ok = mbar_wait(tfull + acc, (i >> 1) & 1, abort_flag, a.status, a.budget_ns);
        ok = __all_sync(0xffffffffu, ok);
        tc_fence_after();
        if (!ok) break;
        const int row = m0 + lr;
        const float* zt = a.Ztot + (size_t)bh * D;
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_base + (uint32_t)(acc * HS_BN + cc * 32), v);
          tmem_wait_ld();
          if (row < s.nq) {
            float* dst = a.Zi + ((size_t)bh * s.nq + row) * D + cc * 32;
#pragma unroll
            for (int c = 0; c < 32; c += 4) {
              const float4 zz = __ldg(reinterpret_cast<const float4*>(zt + cc * 32 + c));
              *reinterpret_cast<float4*>(dst + c) =
                  make_float4(zz.x - __uint_as_float(v[c]), zz.y - __uint_as_float(v[c + 1]),
                              zz.z - __uint_as_float(v[c + 2]), zz.w - __uint_as_float(v[c + 3]));
            }
          }
        }
        tc_fence_before();
        mbar_arrive(tfree + acc);
        continue;
      }
      // the tile's s H_total^T positions (fp32) into shared memory, two per thread (loaded
      // during the previous tile); the previous tile's readers are past the barrier that
      // ended it
      float* hts = reinterpret_cast<float*>(base + C::OFF_HT);
      {
        const float2 h = __half22float2(*reinterpret_cast<const __half2*>(&hw));
        asm volatile("bar.sync 1, 128;" ::: "memory");
        hts[2 * lr] = h.x;
        hts[2 * lr + 1] = h.y;
        asm volatile("bar.sync 1, 128;" ::: "memory");
      }
      // s H_i^T = s H_total^T + G_i at the tile's positions
      bool ok = mbar_wait(tfull + acc, (i >> 1) & 1, abort_flag, a.status, a.budget_ns);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      if (!ok) break;
      // kept in L2 for the epilogue, which reads every image once right after this kernel
      const uint64_t keep = l2_policy_evict_last();
      // 64 positions at a time: each lane converts its row's 128 bytes into the warp's
      // staging rows (16-byte chunk k of row r at chunk k ^ (r & 7): conflict-free both
      // ways), then the warp stores 4 whole rows' 128 bytes per instruction
      uint8_t* stg = base + C::OFF_STG + (qd * 32) * 128;
#pragma unroll 1
      for (int c64 = 0; c64 < HS_BN / 64; ++c64) {
        uint32_t v[64];
        tmem_ld32(tmem + lane_base + (uint32_t)(acc * HS_BN + c64 * 64), *reinterpret_cast<uint32_t(*)[32]>(v));
        tmem_ld32(tmem + lane_base + (uint32_t)(acc * HS_BN + c64 * 64 + 32),
                  *reinterpret_cast<uint32_t(*)[32]>(v + 32));
        tmem_wait_ld();
        __syncwarp();   // the previous chunk's staging rows have been read
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float4 h0 = *reinterpret_cast<const float4*>(hts + c64 * 64 + k * 8);       // same for every lane
          const float4 h1 = *reinterpret_cast<const float4*>(hts + c64 * 64 + k * 8 + 4);
          const float h[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
          uint32_t o[4];
#pragma unroll
          for (int u = 0; u < 4; ++u)
            o[u] = h2u(h[2 * u] + __uint_as_float(v[k * 8 + 2 * u]), h[2 * u + 1] + __uint_as_float(v[k * 8 + 2 * u + 1]));
          *reinterpret_cast<uint4*>(stg + lane * 128 + ((k ^ (lane & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int rr = i * 4 + (lane >> 3), k = lane & 7;   // warp row, 16-byte chunk
          const int grow = m0 + qd * 32 + rr;
          const uint4 val = *reinterpret_cast<const uint4*>(stg + rr * 128 + ((k ^ (rr & 7)) << 4));
          if (grow < s.nq)
            stg_u4_policy(a.hi + ((size_t)bh * s.nq + grow) * D * D + e0 + c64 * 64 + k * 8, val, keep);
        }
      }
      tc_fence_before();
      mbar_arrive(tfree + acc);   // the accumulator can take tile i + 2
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * HS_BN);
  }
}

}  // namespace

cudaError_t launch_hsel(const Shape& s, const CUtensorMap& tmask, const CUtensorMap& timg, const CUtensorMap& tz,
                        const HselArgs& a, cudaStream_t st) {
  constexpr int kSMs = 148;   // B200 streaming multiprocessors
  const int tiles = s.BH * ((s.d * s.d) / HS_BN + 1) * ((s.nq + HS_BM - 1) / HS_BM);
  const int grid = tiles < kSMs ? tiles : kSMs;
  if (s.d == 128) {
    cudaFuncSetAttribute(hsel_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, HsCfg::SMEM);
    hsel_kernel<128><<<grid, HS_THREADS, HsCfg::SMEM, st>>>(tmask, timg, tz, s, a);
  } else {
    cudaFuncSetAttribute(hsel_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, HsCfg::SMEM);
    hsel_kernel<64><<<grid, HS_THREADS, HsCfg::SMEM, st>>>(tmask, timg, tz, s, a);
  }
  return cudaGetLastError();
}

}  // namespace sla2
