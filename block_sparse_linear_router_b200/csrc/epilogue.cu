// Linear branch apply + mix (SLA2 summary page, steps 3 and 4; SLA2 detail
// page §7 note 2: per-key-block h_j precomputed, then accumulated):
//   H_i = H_total - sum_{j selected} h_j,   Z_i = Z_total - sum_{j selected} z_j
//   O_l = phi(Q_i) H_i / (phi(Q_i) Z_i)      (phi: softmax over the d features)
//   O   = alpha_i O_s + (1 - alpha_i) O_l
// When every key block is selected there is no unselected block and O_l := 0.
//
// Persistent CTAs (one per SM) walk the (head, query block) items in
// head-major order, so the SMs work on neighbouring query blocks of the same
// head and the head's h_j^T stay in L2. Per CTA:
//   warp 8     producer: per item, the bf16 Q tile by TMA (128-byte swizzle,
//              the K-major operand layout) into one of two tile buffers, then
//              the selected bf16 h_j^T tiles (contiguous d x d blocks) into a
//              ring of shared-memory stages with 1-D bulk copies; it runs
//              ahead of the compute warps across items;
//   warps 0-7  per item: phi(Q_i) computed in place over the Q tile (fp16);
//              H_i^T = H_total^T - sum of the ring tiles in fp32 registers;
//              [H_i | Z_i] scaled by a per-head power of two (fp16 range) and
//              written as the K-major B operand; one tcgen05 kind::f16 MMA
//              chain D = phi(Q_i) [H_i | Z_i] (128 x (d+16) fp32 in TMEM:
//              numerator columns 0..d-1, denominator column d); then
//              O_l = num / den (the scale cancels), the alpha mix with O_s
//              and the store.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "device.cuh"
#include "kernels.cuh"

namespace sla2 {

namespace {

constexpr int EPI_COMPUTE = 256;          // warps 0-7
constexpr int EPI_THREADS = EPI_COMPUTE + 32;

template <int D>
struct EpiCfg {
  static constexpr int NB = D + 16;                  // B rows (MMA N): H_i^T, Z_i, zeros
  static constexpr int SLABS = D / 64;               // K slabs of 64 fp16 (128 bytes)
  static constexpr int QA_SLAB = BQ * 128;
  static constexpr int QA_BYTES = SLABS * QA_SLAB;   // Q tile (bf16) -> phi (fp16), in place
  static constexpr int B_SLAB = NB * 128;
  static constexpr int B_BYTES = SLABS * B_SLAB;
  static constexpr int TILE = D * D * 2;             // one bf16 h_j^T tile
  static constexpr int NS = D == 128 ? 3 : 8;        // ring stages
  static constexpr int OFF_B = 2 * QA_BYTES;
  static constexpr int OFF_RING = OFF_B + B_BYTES;
  static constexpr int OFF_BAR = OFF_RING + NS * TILE;
  static constexpr int NBAR = 2 * NS + 5;
  static constexpr int SMEM = OFF_BAR + 8 * NBAR + 16 + 1024;
  static constexpr uint32_t IDESC = make_idesc(1, 0, 0, 128, NB);   // fp16 x fp16 -> fp32
  static constexpr int KSTEPS = D / 16;              // 16 fp16 (32 bytes) per MMA
  static constexpr uint32_t TMEM_COLS = NB <= 128 ? 128 : 256;
  static constexpr int SLOTS = D * D / 8 / EPI_COMPUTE;   // 8-element slots per compute thread
};

__device__ __forceinline__ void unpack8(const uint4& w, float (&x)[8]) {
  x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x);
  x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
  x[4] = bf16_lo(w.z); x[5] = bf16_hi(w.z);
  x[6] = bf16_lo(w.w); x[7] = bf16_hi(w.w);
}

__device__ __forceinline__ uint32_t h2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Byte offset of the 16-byte chunk holding elements (row, col..col+7) of a
// K-major 16-bit operand stored as 128-byte-swizzled slabs of 64 columns.
__device__ __forceinline__ uint32_t sw128_h(int row, int col, int slab_bytes) {
  return (uint32_t)((col >> 6) * slab_bytes + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4));
}

// Barrier over the 256 compute threads that also returns, to every one of
// them, whether any of them passed `failed` (so all take the same exit).
__device__ __forceinline__ bool compute_sync_any(bool failed) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 256, p;\n\tselp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)failed)
      : "memory");
  return r != 0;
}

template <int D>
__global__ void __launch_bounds__(EPI_THREADS, 1) epilogue_kernel(const __grid_constant__ CUtensorMap tq, Shape s,
                                                                  EpilogueArgs a) {
  using C = EpiCfg<D>;
  extern __shared__ uint8_t esm_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(esm_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sB = base + C::OFF_B;
  uint8_t* ring = base + C::OFF_RING;
  uint64_t* full = reinterpret_cast<uint64_t*>(base + C::OFF_BAR);
  uint64_t* empty = full + C::NS;
  uint64_t* qfull = empty + C::NS;        // [2]
  uint64_t* qfree = qfull + 2;            // [2]
  uint64_t* mma_done = qfree + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  int* abort_flag = reinterpret_cast<int*>(mma_done + 1) + 1;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int total = s.BH * s.nq;
  const bool has_linear = s.k < s.nk;

  if (tid == 0) {
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, EPI_COMPUTE);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(qfull + b, 1);
      mbar_init(qfree + b, 1);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  // rows d+1 .. d+15 of the B operand are zero for every item
  if (tid < EPI_COMPUTE) {
    for (int t = tid; t < 15 * D / 8; t += EPI_COMPUTE)
      *reinterpret_cast<uint4*>(sB + sw128_h(D + 1 + t / (D / 8), (t % (D / 8)) * 8, C::B_SLAB)) =
          make_uint4(0u, 0u, 0u, 0u);
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ---------------------------------------------------------------- producer
    if (lane == 0 && has_linear) {
      tma_prefetch_desc(&tq);
      int g = 0, it = 0;
      bool ok = true;
      for (int w = blockIdx.x; ok && w < total; w += gridDim.x, ++it) {
        const int bh = w / s.nq, qi = w % s.nq;
        const int b = it & 1;
        if (it >= 2 && !mbar_wait(qfree + b, ((it >> 1) - 1) & 1, abort_flag, a.status, a.budget_ns)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(qfull + b, C::QA_BYTES);
#pragma unroll
        for (int sl = 0; sl < C::SLABS; ++sl)
          tma_load_2d(base + b * C::QA_BYTES + sl * C::QA_SLAB, &tq, qfull + b, sl * 64, bh * s.N + qi * BQ);
        const int32_t* sel = a.idx + ((size_t)bh * s.nq + qi) * s.k;
        for (int n = 0; n < s.k; ++n, ++g) {
          const int st = g % C::NS;
          if (g >= C::NS && !mbar_wait(empty + st, ((g / C::NS) - 1) & 1, abort_flag, a.status, a.budget_ns)) {
            ok = false;
            break;
          }
          const int j = __ldg(sel + n);
          mbar_arrive_expect_tx(full + st, C::TILE);
          bulk_load(ring + st * C::TILE, a.hT + ((size_t)bh * s.nk + j) * D * D, C::TILE, full + st);
        }
      }
      if (!ok) {   // let the copies in flight land before the CTA's shared memory is released
        for (int q = (g > C::NS ? g - C::NS : 0); q < g; ++q)
          mbar_wait_drain(full + q % C::NS, (q / C::NS) & 1, 20000000ull);
        for (int q = (it > 2 ? it - 2 : 0); q <= it; ++q) mbar_wait_drain(qfull + (q & 1), (q >> 1) & 1, 20000000ull);
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- compute warps
    constexpr int TPR = D / 8, RPP = EPI_COMPUTE / TPR;
    const int cg = tid % TPR, rg = tid / TPR;
    const int r = (warp & 3) * 32 + lane;        // TMEM lane / query row of the readout
    const int half = warp >> 2;
    constexpr int HC = D / 2;
    const uint32_t taddr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    int g = 0, it = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < total; w += gridDim.x, ++it) {
      const int bh = w / s.nq, qi = w % s.nq;
      const int h = bh % a.H;
      const float alpha = a.alpha[(size_t)h * s.nq + qi];
      const size_t row = (size_t)bh * s.N + (size_t)qi * BQ + r;
      float4 osv[HC / 4];
      if (has_linear) {
        const int32_t* sel = a.idx + ((size_t)bh * s.nq + qi) * s.k;
        uint8_t* qa = base + (it & 1) * C::QA_BYTES;
        // ---- H_total^T (issued first; its loads overlap the phi work)
        float acc[C::SLOTS][8];
        const float4* Ht = reinterpret_cast<const float4*>(a.Htot + (size_t)bh * D * D);
#pragma unroll
        for (int u = 0; u < C::SLOTS; ++u) {
          const int slot = tid + u * EPI_COMPUTE;
          const float4 x0 = __ldg(Ht + 2 * slot), x1 = __ldg(Ht + 2 * slot + 1);
          acc[u][0] = x0.x; acc[u][1] = x0.y; acc[u][2] = x0.z; acc[u][3] = x0.w;
          acc[u][4] = x1.x; acc[u][5] = x1.y; acc[u][6] = x1.z; acc[u][7] = x1.w;
        }
        // ---- phi(Q_i) in place over the TMA-loaded bf16 Q tile -> fp16
        ok = mbar_wait(qfull + (it & 1), (it >> 1) & 1, abort_flag, a.status, a.budget_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
#pragma unroll 2
          for (int rr = rg; rr < BQ; rr += RPP) {
            uint4* p = reinterpret_cast<uint4*>(qa + sw128_h(rr, cg * 8, C::QA_SLAB));
            float x[8];
            unpack8(*p, x);
            float m = x[0];
#pragma unroll
            for (int c = 1; c < 8; ++c) m = fmaxf(m, x[c]);
#pragma unroll
            for (int off = TPR / 2; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
            float sum = 0.f;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              x[c] = expf(x[c] - m);
              sum += x[c];
            }
#pragma unroll
            for (int off = TPR / 2; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
            const float inv = 1.f / sum;
            *p = make_uint4(h2(x[0] * inv, x[1] * inv), h2(x[2] * inv, x[3] * inv), h2(x[4] * inv, x[5] * inv),
                            h2(x[6] * inv, x[7] * inv));
          }
        }
        // ---- H_i^T = H_total^T - sum of the selected h_j^T
        for (int n = 0; ok && n < s.k; ++n, ++g) {
          const int st = g % C::NS;
          ok = mbar_wait(full + st, (g / C::NS) & 1, abort_flag, a.status, a.budget_ns);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          const uint4* tile = reinterpret_cast<const uint4*>(ring + st * C::TILE);
#pragma unroll
          for (int u = 0; u < C::SLOTS; ++u) {
            float x[8];
            unpack8(tile[tid + u * EPI_COMPUTE], x);
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[u][c] -= x[c];
          }
          mbar_arrive(empty + st);
        }
        // ---- [H_i^T ; Z_i] * scale -> fp16 B operand
        const float sc = a.zscale[bh];
#pragma unroll
        for (int u = 0; u < C::SLOTS; ++u) {
          const int slot = tid + u * EPI_COMPUTE;
          const int brow = slot / (D / 8), bcol = (slot % (D / 8)) * 8;
          *reinterpret_cast<uint4*>(sB + sw128_h(brow, bcol, C::B_SLAB)) =
              make_uint4(h2(acc[u][0] * sc, acc[u][1] * sc), h2(acc[u][2] * sc, acc[u][3] * sc),
                         h2(acc[u][4] * sc, acc[u][5] * sc), h2(acc[u][6] * sc, acc[u][7] * sc));
        }
        if (tid < D / 8) {
          float z[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) z[c] = a.Ztot[(size_t)bh * D + tid * 8 + c];
          for (int n = 0; n < s.k; ++n) {
            const float* zj = a.z + ((size_t)bh * s.nk + __ldg(sel + n)) * D + tid * 8;
#pragma unroll
            for (int c = 0; c < 8; ++c) z[c] -= zj[c];
          }
          *reinterpret_cast<uint4*>(sB + sw128_h(D, tid * 8, C::B_SLAB)) =
              make_uint4(h2(z[0] * sc, z[1] * sc), h2(z[2] * sc, z[3] * sc), h2(z[4] * sc, z[5] * sc),
                         h2(z[6] * sc, z[7] * sc));
        }
        fence_proxy_async_smem();
        tc_fence_before();
        if (compute_sync_any(!ok)) break;     // every compute thread takes this exit together
        // ---- D = phi(Q_i) [H_i | Z_i]
        if (tid == 0) {
          tc_fence_after();
          const uint32_t a0 = smem_u32(qa), b0 = smem_u32(sB);
#pragma unroll
          for (int ks = 0; ks < C::KSTEPS; ++ks) {
            const uint32_t off = (ks & 3) * 32;
            const uint64_t ad = make_sdesc(a0 + (ks >> 2) * C::QA_SLAB + off, 1024, LAYOUT_SW128);
            const uint64_t bd = make_sdesc(b0 + (ks >> 2) * C::B_SLAB + off, 1024, LAYOUT_SW128);
            mma_f16(tmem, ad, bd, C::IDESC, ks > 0);
          }
          tc_commit(mma_done);
          tc_commit(qfree + (it & 1));
        }
        // O_s loads overlap the MMA
        const float* osr = a.os + row * D + half * HC;
#pragma unroll
        for (int c = 0; c < HC / 4; ++c) osv[c] = __ldg(reinterpret_cast<const float4*>(osr) + c);
        ok = mbar_wait(mma_done, it & 1, abort_flag, a.status, a.budget_ns);
        ok = __all_sync(0xffffffffu, ok);
        tc_fence_after();
        if (!ok) continue;   // a failed wait: skip the store; the next barrier ends the loop
      } else {
        const float* osr = a.os + row * D + half * HC;
#pragma unroll
        for (int c = 0; c < HC / 4; ++c) osv[c] = __ldg(reinterpret_cast<const float4*>(osr) + c);
      }
      // ---- O_l, mix, store: warp w reads TMEM lanes 32 (w % 4).., column half w / 4
      float inv_den = 0.f;
      if (has_linear) {
        uint32_t dv[32];
        tmem_ld32(taddr + D, dv);
        tmem_wait_ld();
        inv_den = 1.f / __uint_as_float(dv[0]);
      }
#pragma unroll
      for (int cc = 0; cc < HC / 32; ++cc) {
        uint32_t nv[32];
        if (has_linear) {
          tmem_ld32(taddr + half * HC + cc * 32, nv);
          tmem_wait_ld();
        }
        float o[32], ol[32];
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          const float4 v = osv[(cc * 32 + c) / 4];
          const float os4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            ol[c + u] = has_linear ? __uint_as_float(nv[c + u]) * inv_den : 0.f;
            o[c + u] = alpha * os4[u] + (1.f - alpha) * ol[c + u];
          }
        }
        const size_t off = row * D + half * HC + cc * 32;
        if (a.ol_dbg) {
#pragma unroll
          for (int c = 0; c < 32; c += 4)
            *reinterpret_cast<float4*>(a.ol_dbg + off + c) = make_float4(ol[c], ol[c + 1], ol[c + 2], ol[c + 3]);
        }
        if (a.out_f32) {
#pragma unroll
          for (int c = 0; c < 32; c += 4)
            *reinterpret_cast<float4*>(static_cast<float*>(a.out) + off + c) =
                make_float4(o[c], o[c + 1], o[c + 2], o[c + 3]);
        } else {
          __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.out) + off;
#pragma unroll
          for (int c = 0; c < 32; c += 8)
            *reinterpret_cast<uint4*>(dst + c) =
                make_uint4(cvt_bf16x2(o[c], o[c + 1]), cvt_bf16x2(o[c + 2], o[c + 3]),
                           cvt_bf16x2(o[c + 4], o[c + 5]), cvt_bf16x2(o[c + 6], o[c + 7]));
        }
      }
      tc_fence_before();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

constexpr int kSMs = 148;   // B200 streaming multiprocessors

}  // namespace

cudaError_t launch_epilogue(const Shape& s, const EpilogueArgs& a, const CUtensorMap& tq, cudaStream_t st) {
  const int total = s.BH * s.nq;
  const int grid = total < kSMs ? total : kSMs;
  if (s.d == 128) {
    auto k = epilogue_kernel<128>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, EpiCfg<128>::SMEM);
    k<<<grid, EPI_THREADS, EpiCfg<128>::SMEM, st>>>(tq, s, a);
  } else {
    auto k = epilogue_kernel<64>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, EpiCfg<64>::SMEM);
    k<<<grid, EPI_THREADS, EpiCfg<64>::SMEM, st>>>(tq, s, a);
  }
  return cudaGetLastError();
}

}  // namespace sla2
