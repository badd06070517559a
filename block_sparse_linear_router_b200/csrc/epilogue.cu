// Linear branch apply + mix (SLA2 summary page, steps 3 and 4; SLA2 detail
// page §7 note 2: per-key-block h_j precomputed, then accumulated):
//   H_i = H_total - sum_{j selected} h_j,   Z_i = Z_total - sum_{j selected} z_j
//   O_l = phi(Q_i) H_i / (phi(Q_i) Z_i)      (phi: softmax over the d features)
//   O   = alpha_i O_s + (1 - alpha_i) O_l
// When every key block is selected there is no unselected block and O_l := 0.
//
// One CTA (256 threads) per (head, query block), heads outermost:
//   1. gather: [H_i^T | Z_i] (fp32) = totals - selected h_j^T (bf16) / z_j,
//      written as the B operand (N = d + 16 rows: d rows of H_i^T, Z_i, zeros);
//   2. phi(Q_i) (fp32, from bf16 Q) written as the A operand;
//   3. one tcgen05 kind::tf32 MMA chain D = phi(Q_i) [H_i | Z_i] (128 x (d+16)
//      fp32 in TMEM): numerator columns 0..d-1, denominator column d;
//   4. TMEM -> registers, O_l = num / den, mix with O_s, store.
// Operand tiles are K-major, 128-byte swizzled slabs of 32 fp32 columns.
#include <cuda_bf16.h>

#include "device.cuh"
#include "kernels.cuh"

namespace sla2 {

namespace {

constexpr int EPI_THREADS = 256;

template <int D>
struct EpiCfg {
  static constexpr int NB = D + 16;                  // B rows (MMA N)
  static constexpr int SLABS = D / 32;               // K slabs (32 fp32 = 128 bytes)
  static constexpr int A_SLAB = BQ * 128;
  static constexpr int B_SLAB = NB * 128;
  static constexpr int A_BYTES = SLABS * A_SLAB;
  static constexpr int B_BYTES = SLABS * B_SLAB;
  static constexpr int SMEM = A_BYTES + B_BYTES + 64 + 1024;
  static constexpr uint32_t IDESC = make_idesc(1, 2, 2, 128, NB);
  static constexpr int KSTEPS = D / 8;               // 8 tf32 (32 bytes) per MMA
  static constexpr uint32_t TMEM_COLS = NB <= 128 ? 128 : 256;
};

__device__ __forceinline__ void unpack8(const uint4& w, float (&x)[8]) {
  x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x);
  x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
  x[4] = bf16_lo(w.z); x[5] = bf16_hi(w.z);
  x[6] = bf16_lo(w.w); x[7] = bf16_hi(w.w);
}

template <int D>
__global__ void __launch_bounds__(EPI_THREADS, 1) epilogue_kernel(Shape s, EpilogueArgs a) {
  using C = EpiCfg<D>;
  extern __shared__ uint8_t esm_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(esm_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = base;
  uint8_t* sB = base + C::A_BYTES;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sB + C::B_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 1);
  int* abort_flag = reinterpret_cast<int*>(bar + 2);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x / s.nq, qi = blockIdx.x % s.nq;
  const int h = bh % a.H;
  const float alpha = a.alpha[(size_t)h * s.nq + qi];
  const bool has_linear = s.k < s.nk;
  const int32_t* sel = a.idx + ((size_t)bh * s.nq + qi) * s.k;

  if (tid == 0) {
    mbar_init(bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }

  if (has_linear) {
    // ---- 1. B operand: [H_i^T ; Z_i ; 0] (tf32)
    constexpr int SLOTS = D * D / 8 / EPI_THREADS;     // 8-element slots per thread
    float acc[SLOTS][8];
    const float* Ht = a.Htot + (size_t)bh * D * D;
#pragma unroll
    for (int u = 0; u < SLOTS; ++u) {
      const int slot = tid + u * EPI_THREADS;
      const float4 x0 = __ldg(reinterpret_cast<const float4*>(Ht) + 2 * slot);
      const float4 x1 = __ldg(reinterpret_cast<const float4*>(Ht) + 2 * slot + 1);
      acc[u][0] = x0.x; acc[u][1] = x0.y; acc[u][2] = x0.z; acc[u][3] = x0.w;
      acc[u][4] = x1.x; acc[u][5] = x1.y; acc[u][6] = x1.z; acc[u][7] = x1.w;
    }
    for (int n = 0; n < s.k; ++n) {
      const int j = __ldg(sel + n);
      const uint4* hj = reinterpret_cast<const uint4*>(a.hT + ((size_t)bh * s.nk + j) * D * D);
      uint4 w[SLOTS];
#pragma unroll
      for (int u = 0; u < SLOTS; ++u) w[u] = __ldg(hj + tid + u * EPI_THREADS);
#pragma unroll
      for (int u = 0; u < SLOTS; ++u) {
        float x[8];
        unpack8(w[u], x);
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[u][c] -= x[c];
      }
    }
#pragma unroll
    for (int u = 0; u < SLOTS; ++u) {
      const int slot = tid + u * EPI_THREADS;
      const int row = slot / (D / 8), col = (slot % (D / 8)) * 8;
      float4 v0 = make_float4(to_tf32(acc[u][0]), to_tf32(acc[u][1]), to_tf32(acc[u][2]), to_tf32(acc[u][3]));
      float4 v1 = make_float4(to_tf32(acc[u][4]), to_tf32(acc[u][5]), to_tf32(acc[u][6]), to_tf32(acc[u][7]));
      *reinterpret_cast<float4*>(sB + sw128_f32(row, col, C::B_SLAB)) = v0;
      *reinterpret_cast<float4*>(sB + sw128_f32(row, col + 4, C::B_SLAB)) = v1;
    }
    if (tid < D) {
      float z = a.Ztot[(size_t)bh * D + tid];
      for (int n = 0; n < s.k; ++n) z -= a.z[((size_t)bh * s.nk + __ldg(sel + n)) * D + tid];
      *reinterpret_cast<float*>(sB + sw128_f32(D, tid, C::B_SLAB)) = to_tf32(z);
    }
    for (int t = tid; t < 15 * D; t += EPI_THREADS)
      *reinterpret_cast<float*>(sB + sw128_f32(D + 1 + t / D, t % D, C::B_SLAB)) = 0.f;

    // ---- 2. A operand: phi(Q_i) (tf32), TPR threads per query row
    constexpr int TPR = D / 8, RPP = EPI_THREADS / TPR;
    const int cg = tid % TPR, rg = tid / TPR;
    const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q) + ((size_t)bh * s.N + (size_t)qi * BQ) * D;
#pragma unroll 2
    for (int r = rg; r < BQ; r += RPP) {
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(q + (size_t)r * D + cg * 8));
      float x[8];
      unpack8(w, x);
      float m = x[0];
#pragma unroll
      for (int c = 1; c < 8; ++c) m = fmaxf(m, x[c]);
#pragma unroll
      for (int off = TPR / 2; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      float e[8], sum = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        e[c] = expf(x[c] - m);
        sum += e[c];
      }
#pragma unroll
      for (int off = TPR / 2; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      const float inv = 1.f / sum;
      *reinterpret_cast<float4*>(sA + sw128_f32(r, cg * 8, C::A_SLAB)) =
          make_float4(to_tf32(e[0] * inv), to_tf32(e[1] * inv), to_tf32(e[2] * inv), to_tf32(e[3] * inv));
      *reinterpret_cast<float4*>(sA + sw128_f32(r, cg * 8 + 4, C::A_SLAB)) =
          make_float4(to_tf32(e[4] * inv), to_tf32(e[5] * inv), to_tf32(e[6] * inv), to_tf32(e[7] * inv));
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // ---- 3. D = phi(Q_i) [H_i | Z_i]
  if (has_linear && tid == 0) {
    const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
#pragma unroll
    for (int ks = 0; ks < C::KSTEPS; ++ks) {
      const uint32_t off = (ks & 3) * 32;
      const uint64_t ad = make_sdesc(a0 + (ks >> 2) * C::A_SLAB + off, 1024, LAYOUT_SW128);
      const uint64_t bd = make_sdesc(b0 + (ks >> 2) * C::B_SLAB + off, 1024, LAYOUT_SW128);
      mma_tf32(tmem, ad, bd, C::IDESC, ks > 0);
    }
    tc_commit(bar);
  }

  // ---- 4. O_l, mix, store: warp w reaches TMEM lanes 32 (w % 4).., columns half (w / 4)
  bool ok = true;
  if (has_linear) {
    ok = mbar_wait(bar, 0, abort_flag, a.status, a.budget_ns);
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
  }
  if (ok) {
    const int r = (warp & 3) * 32 + lane;
    const int half = warp >> 2;
    constexpr int HC = D / 2;
    const uint32_t taddr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    float inv_den = 0.f;
    if (has_linear) {
      uint32_t dv[32];
      tmem_ld32(taddr + D, dv);
      tmem_wait_ld();
      inv_den = 1.f / __uint_as_float(dv[0]);
    }
    const size_t row = (size_t)bh * s.N + (size_t)qi * BQ + r;
    const float* osr = a.os + row * D + half * HC;
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
        const float4 v = *reinterpret_cast<const float4*>(osr + cc * 32 + c);
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
          *reinterpret_cast<float4*>(static_cast<float*>(a.out) + off + c) = make_float4(o[c], o[c + 1], o[c + 2], o[c + 3]);
      } else {
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.out) + off;
#pragma unroll
        for (int c = 0; c < 32; c += 8)
          *reinterpret_cast<uint4*>(dst + c) = make_uint4(cvt_bf16x2(o[c], o[c + 1]), cvt_bf16x2(o[c + 2], o[c + 3]),
                                                          cvt_bf16x2(o[c + 4], o[c + 5]), cvt_bf16x2(o[c + 6], o[c + 7]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace

cudaError_t launch_epilogue(const Shape& s, const EpilogueArgs& a, cudaStream_t st) {
  if (s.d == 128) {
    auto k = epilogue_kernel<128>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, EpiCfg<128>::SMEM);
    k<<<s.BH * s.nq, EPI_THREADS, EpiCfg<128>::SMEM, st>>>(s, a);
  } else {
    auto k = epilogue_kernel<64>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, EpiCfg<64>::SMEM);
    k<<<s.BH * s.nq, EPI_THREADS, EpiCfg<64>::SMEM, st>>>(s, a);
  }
  return cudaGetLastError();
}

}  // namespace sla2
