// Linear branch apply + mix (SLA2 summary page, steps 3 and 4):
//   H_i = H_total - sum_{j selected} h_j,   Z_i = Z_total - sum_{j selected} z_j
//   O_l = phi(Q_i) H_i / (phi(Q_i) Z_i)      (phi: softmax over the d features)
//   O   = alpha_i O_s + (1 - alpha_i) O_l
// When every key block is selected there is no unselected block and O_l := 0.
// One CTA per (head, query block); the 128 rows are processed in two halves.
#include <cuda_bf16.h>

#include "device.cuh"
#include "kernels.cuh"

namespace sla2 {

namespace {

constexpr int EPI_THREADS = 256;
constexpr int EPI_ROWS = 64;   // rows per half

__device__ __forceinline__ void unpack8(const uint4& w, float (&x)[8]) {
  x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x);
  x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
  x[4] = bf16_lo(w.z); x[5] = bf16_hi(w.z);
  x[6] = bf16_lo(w.w); x[7] = bf16_hi(w.w);
}

template <int D>
__global__ void __launch_bounds__(EPI_THREADS) epilogue_kernel(Shape s, EpilogueArgs a) {
  constexpr int TPR = D / 8;                 // threads per row for phi
  constexpr int RPP = EPI_THREADS / TPR;     // rows per pass
  constexpr int CT = D / 16;                 // output columns per thread
  constexpr int RT = EPI_ROWS / 16;          // output rows per thread
  extern __shared__ float esm[];
  float* Hs = esm;                           // [D][D]
  float* Zs = Hs + D * D;                    // [D]
  float* phq = Zs + D;                       // [EPI_ROWS][D]
  float* den = phq + EPI_ROWS * D;           // [EPI_ROWS]
  const int i = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
  const int h = bh % a.H;
  const float alpha = a.alpha[(size_t)h * s.nq + i];
  const bool has_linear = s.k < s.nk;
  const int32_t* sel = a.idx + ((size_t)bh * s.nq + i) * s.k;

  if (has_linear) {
    const float4* Ht = reinterpret_cast<const float4*>(a.Htot + (size_t)bh * D * D);
    for (int e4 = tid; e4 < D * D / 4; e4 += EPI_THREADS) {
      float4 acc = Ht[e4];
      for (int n = 0; n < s.k; ++n) {
        const int j = __ldg(sel + n);
        const float4 hv = __ldg(reinterpret_cast<const float4*>(a.h + ((size_t)bh * s.nk + j) * D * D) + e4);
        acc.x -= hv.x; acc.y -= hv.y; acc.z -= hv.z; acc.w -= hv.w;
      }
      reinterpret_cast<float4*>(Hs)[e4] = acc;
    }
    if (tid < D) {
      float z = a.Ztot[(size_t)bh * D + tid];
      for (int n = 0; n < s.k; ++n) z -= a.z[((size_t)bh * s.nk + __ldg(sel + n)) * D + tid];
      Zs[tid] = z;
    }
  }
  __syncthreads();

  const int cg = tid % TPR, rg = tid / TPR;
  const int ty = tid / 16, tx = tid % 16;
  for (int half = 0; half < BQ / EPI_ROWS; ++half) {
    const size_t row0 = (size_t)bh * s.N + (size_t)i * BQ + half * EPI_ROWS;
    if (has_linear) {
      for (int r = rg; r < EPI_ROWS; r += RPP) {
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.q) +
                                                             (row0 + r) * D + cg * 8));
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
        float dz = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float p = e[c] * inv;
          phq[r * D + cg * 8 + c] = p;
          dz = fmaf(p, Zs[cg * 8 + c], dz);
        }
#pragma unroll
        for (int off = TPR / 2; off > 0; off >>= 1) dz += __shfl_xor_sync(0xffffffffu, dz, off);
        if (cg == 0) den[r] = dz;
      }
    }
    __syncthreads();
    float acc[RT][CT];
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
      for (int c = 0; c < CT; ++c) acc[r][c] = 0.f;
    if (has_linear) {
      for (int e = 0; e < D; ++e) {
        float pr[RT], hv[CT];
#pragma unroll
        for (int r = 0; r < RT; ++r) pr[r] = phq[(ty * RT + r) * D + e];
#pragma unroll
        for (int c = 0; c < CT; ++c) hv[c] = Hs[e * D + tx * CT + c];
#pragma unroll
        for (int r = 0; r < RT; ++r)
#pragma unroll
          for (int c = 0; c < CT; ++c) acc[r][c] = fmaf(pr[r], hv[c], acc[r][c]);
      }
    }
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      const int rr = ty * RT + r;
      const size_t off = (row0 + rr) * D + tx * CT;
      const float inv_den = has_linear ? 1.f / den[rr] : 0.f;
      float o[CT];
#pragma unroll
      for (int c = 0; c < CT; c += 4) {
        const float4 os = *reinterpret_cast<const float4*>(a.os + off + c);
        const float osv[4] = {os.x, os.y, os.z, os.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float ol = acc[r][c + u] * inv_den;
          acc[r][c + u] = ol;
          o[c + u] = alpha * osv[u] + (1.f - alpha) * ol;
        }
      }
      if (a.ol_dbg) {
#pragma unroll
        for (int c = 0; c < CT; c += 4)
          *reinterpret_cast<float4*>(a.ol_dbg + off + c) = make_float4(acc[r][c], acc[r][c + 1], acc[r][c + 2], acc[r][c + 3]);
      }
      if (a.out_f32) {
#pragma unroll
        for (int c = 0; c < CT; c += 4)
          *reinterpret_cast<float4*>(static_cast<float*>(a.out) + off + c) = make_float4(o[c], o[c + 1], o[c + 2], o[c + 3]);
      } else {
        uint32_t w[CT / 2];
#pragma unroll
        for (int c = 0; c < CT; c += 2) w[c / 2] = cvt_bf16x2(o[c], o[c + 1]);
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.out) + off;
        if constexpr (CT == 8) {
          *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
        } else {
          *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
        }
      }
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_epilogue(const Shape& s, const EpilogueArgs& a, cudaStream_t st) {
  dim3 grid(s.nq, s.BH);
  const size_t smem = (size_t)(s.d * s.d + s.d + EPI_ROWS * s.d + EPI_ROWS) * sizeof(float);
  if (s.d == 128) {
    cudaFuncSetAttribute(epilogue_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    epilogue_kernel<128><<<grid, EPI_THREADS, smem, st>>>(s, a);
  } else {
    cudaFuncSetAttribute(epilogue_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    epilogue_kernel<64><<<grid, EPI_THREADS, smem, st>>>(s, a);
  }
  return cudaGetLastError();
}

}  // namespace sla2
