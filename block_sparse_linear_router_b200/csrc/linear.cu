// Linear-branch state and the K / V quantisation pass (SLA2 summary page,
// step 3: H_j = phi(K_j)^T V_j, Z_j = rowsum(phi(K_j)^T); SLA2 detail page §7
// note 2: h_j precomputed per key block, then accumulated; step 2's low-bit K
// and V).
//
// One CTA walks a contiguous chunk of key blocks of one head. Per key block j:
//   K_s = fp32(K) - fp32(c)                      (K smoothing, detail §7 note 1)
//   K-hat_j = INT8 of K_s over the 64 x d block, s_k = amax / 127
//   V-hat_j^T = e4m3(V * 448 / amax_channel) stored channel-major [d][64]
//   phi(K_s) = softmax over the d features (fp32, accurate expf)
//   z_j = sum_t phi_t, h_j = phi^T V  (fp32)
// and the chunk's partial sums of h_j, z_j, later reduced in a fixed order to
// H_total, Z_total.
#include <cuda_bf16.h>

#include "device.cuh"
#include "kernels.cuh"

namespace sla2 {

namespace {

constexpr int LIN_THREADS = 256;
constexpr int LIN_CHUNKS = 32;

__device__ __forceinline__ void unpack8(const uint4& w, float (&x)[8]) {
  x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x);
  x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
  x[4] = bf16_lo(w.z); x[5] = bf16_hi(w.z);
  x[6] = bf16_lo(w.w); x[7] = bf16_hi(w.w);
}

template <int D>
__global__ void __launch_bounds__(LIN_THREADS) linear_state_kernel(
    const __nv_bfloat16* __restrict__ kin, const __nv_bfloat16* __restrict__ vin, const float* __restrict__ c32,
    int N, int nk, LinearOut o) {
  constexpr int TPR = D / 8;              // threads per token row (8 channels each)
  constexpr int RPP = LIN_THREADS / TPR;  // token rows per pass
  constexpr int NP = BKB / RPP;           // passes over 64 tokens
  constexpr int T = D / 16;               // h tile per thread: T x T
  extern __shared__ float lsm[];
  float* phi = lsm;                  // [64][D]
  float* vs = phi + BKB * D;         // [64][D]
  float* cs = vs + BKB * D;          // [D]
  float* vinv = cs + D;              // [D] 448 / amax
  float* red8 = vinv + D;            // [8]
  const int bh = blockIdx.y, chunk = blockIdx.x, G = gridDim.x, tid = threadIdx.x;
  const int j0 = (int)((long long)chunk * nk / G), j1 = (int)((long long)(chunk + 1) * nk / G);
  const int cg = tid % TPR, rg = tid / TPR;
  const int ty = tid / 16, tx = tid % 16;

  for (int e = tid; e < D; e += LIN_THREADS) {
    cs[e] = c32[(size_t)bh * D + e];
    if (o.quant == 1) {
      const float a = __uint_as_float(o.vamax[(size_t)bh * D + e]);
      vinv[e] = a > 0.f ? __fdiv_rn(448.f, a) : 0.f;
      if (chunk == 0) o.sv[(size_t)bh * D + e] = a > 0.f ? __fdiv_rn(a, 448.f) : 0.f;
    }
  }
  float hp[T][T];
#pragma unroll
  for (int a = 0; a < T; ++a)
#pragma unroll
    for (int b = 0; b < T; ++b) hp[a][b] = 0.f;
  float zp = 0.f;
  __syncthreads();

  for (int j = j0; j < j1; ++j) {
    const size_t rowbase = (size_t)bh * N + (size_t)j * BKB;
    float x[NP][8];
    float amax = 0.f;
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      const int t = p * RPP + rg;
      const uint4 wk = __ldg(reinterpret_cast<const uint4*>(kin + (rowbase + t) * D + cg * 8));
      const uint4 wv = __ldg(reinterpret_cast<const uint4*>(vin + (rowbase + t) * D + cg * 8));
      float kv[8], vv[8];
      unpack8(wk, kv);
      unpack8(wv, vv);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        x[p][c] = __fsub_rn(kv[c], cs[cg * 8 + c]);
        amax = fmaxf(amax, fabsf(x[p][c]));
        vs[t * D + cg * 8 + c] = vv[c];
      }
      // phi: softmax over the D features of token t (TPR consecutive lanes share the row)
      float m = x[p][0];
#pragma unroll
      for (int c = 1; c < 8; ++c) m = fmaxf(m, x[p][c]);
#pragma unroll
      for (int off = TPR / 2; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      float e[8], s = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        e[c] = expf(x[p][c] - m);
        s += e[c];
      }
#pragma unroll
      for (int off = TPR / 2; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
      const float inv = 1.f / s;
#pragma unroll
      for (int c = 0; c < 8; ++c) phi[t * D + cg * 8 + c] = e[c] * inv;
    }
    // K-hat of the smoothed block
    if (o.khat) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      if ((tid & 31) == 0) red8[tid >> 5] = amax;
      __syncthreads();
      float a = red8[0];
#pragma unroll
      for (int w = 1; w < 8; ++w) a = fmaxf(a, red8[w]);
      const float inv = a > 0.f ? __fdiv_rn(127.f, a) : 0.f;
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        const int t = p * RPP + rg;
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int q0 = max(-127, min(127, __float2int_rn(__fmul_rn(x[p][c], inv))));
          const int q1 = max(-127, min(127, __float2int_rn(__fmul_rn(x[p][c + 4], inv))));
          lo |= (uint32_t)(q0 & 0xFF) << (8 * c);
          hi |= (uint32_t)(q1 & 0xFF) << (8 * c);
        }
        *reinterpret_cast<uint2*>(o.khat + (rowbase + t) * D + cg * 8) = make_uint2(lo, hi);
      }
      if (tid == 0) o.sk[(size_t)bh * nk + j] = a > 0.f ? __fdiv_rn(a, 127.f) : 0.f;
    }
    __syncthreads();   // phi, vs complete
    // V-hat^T (or the bf16 V^T copy): channel-major 64 tokens per row
    if (o.vhatT) {
      constexpr int HALVES = LIN_THREADS / D;      // threads per channel row
      constexpr int TOK = BKB / HALVES;            // tokens per thread
      const int c = tid / HALVES, part = tid % HALVES;
      const size_t orow = ((size_t)bh * nk + j) * D + c;
      if (o.quant == 1) {
        uint8_t* dst = static_cast<uint8_t*>(o.vhatT) + orow * BKB + part * TOK;
        const float iv = vinv[c];
#pragma unroll
        for (int t0 = 0; t0 < TOK; t0 += 16) {
          uint32_t w[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int t = part * TOK + t0 + 4 * u;
            const uint16_t lo = cvt_e4m3x2(__fmul_rn(vs[t * D + c], iv), __fmul_rn(vs[(t + 1) * D + c], iv));
            const uint16_t hi = cvt_e4m3x2(__fmul_rn(vs[(t + 2) * D + c], iv), __fmul_rn(vs[(t + 3) * D + c], iv));
            w[u] = (uint32_t)lo | ((uint32_t)hi << 16);
          }
          *reinterpret_cast<uint4*>(dst + t0) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      } else {
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(o.vhatT) + orow * BKB + part * TOK;
#pragma unroll
        for (int t0 = 0; t0 < TOK; t0 += 8) {
          uint32_t w[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int t = part * TOK + t0 + 2 * u;
            w[u] = cvt_bf16x2(vs[t * D + c], vs[(t + 1) * D + c]);
          }
          *reinterpret_cast<uint4*>(dst + t0) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
    // z_j
    if (tid < D) {
      float z = 0.f;
      for (int t = 0; t < BKB; ++t) z += phi[t * D + tid];
      o.z[((size_t)bh * nk + j) * D + tid] = z;
      zp += z;
    }
    // h_j = phi^T V : thread tile rows [ty*T, +T) x cols [tx*T, +T)
    float acc[T][T];
#pragma unroll
    for (int a = 0; a < T; ++a)
#pragma unroll
      for (int b = 0; b < T; ++b) acc[a][b] = 0.f;
    for (int t = 0; t < BKB; ++t) {
      float pa[T], vb[T];
#pragma unroll
      for (int a = 0; a < T; ++a) pa[a] = phi[t * D + ty * T + a];
#pragma unroll
      for (int b = 0; b < T; ++b) vb[b] = vs[t * D + tx * T + b];
#pragma unroll
      for (int a = 0; a < T; ++a)
#pragma unroll
        for (int b = 0; b < T; ++b) acc[a][b] = fmaf(pa[a], vb[b], acc[a][b]);
    }
    float* hdst = o.h + ((size_t)bh * nk + j) * D * D;
#pragma unroll
    for (int a = 0; a < T; ++a) {
#pragma unroll
      for (int b = 0; b < T; b += 4) {
        *reinterpret_cast<float4*>(hdst + (size_t)(ty * T + a) * D + tx * T + b) =
            make_float4(acc[a][b], acc[a][b + 1], acc[a][b + 2], acc[a][b + 3]);
      }
#pragma unroll
      for (int b = 0; b < T; ++b) hp[a][b] += acc[a][b];
    }
    __syncthreads();   // before the next block overwrites phi / vs
  }
  float* pdst = o.hpart + ((size_t)bh * G + chunk) * D * D;
#pragma unroll
  for (int a = 0; a < T; ++a)
#pragma unroll
    for (int b = 0; b < T; b += 4)
      *reinterpret_cast<float4*>(pdst + (size_t)(ty * T + a) * D + tx * T + b) =
          make_float4(hp[a][b], hp[a][b + 1], hp[a][b + 2], hp[a][b + 3]);
  if (tid < D) o.zpart[((size_t)bh * G + chunk) * D + tid] = zp;
}

__global__ void linear_reduce_kernel(const float* __restrict__ hpart, const float* __restrict__ zpart, int G, int D,
                                     float* __restrict__ Htot, float* __restrict__ Ztot) {
  const int bh = blockIdx.y;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  const int DD = D * D;
  if (e < DD) {
    float s = 0.f;
    for (int g = 0; g < G; ++g) s += hpart[((size_t)bh * G + g) * DD + e];
    Htot[(size_t)bh * DD + e] = s;
  }
  if (blockIdx.x == 0 && threadIdx.x < D) {
    float s = 0.f;
    for (int g = 0; g < G; ++g) s += zpart[((size_t)bh * G + g) * D + threadIdx.x];
    Ztot[(size_t)bh * D + threadIdx.x] = s;
  }
}

}  // namespace

int linear_chunks(int nk) { return nk < LIN_CHUNKS ? nk : LIN_CHUNKS; }

cudaError_t launch_linear_state(const Shape& s, const void* k, const void* v, const float* c32, const LinearOut& o,
                                cudaStream_t st) {
  dim3 grid(linear_chunks(s.nk), s.BH);
  const size_t smem = (size_t)(2 * BKB * s.d + 2 * s.d + 8) * sizeof(float);
  auto kb = static_cast<const __nv_bfloat16*>(k);
  auto vb = static_cast<const __nv_bfloat16*>(v);
  if (s.d == 128) {
    cudaFuncSetAttribute(linear_state_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    linear_state_kernel<128><<<grid, LIN_THREADS, smem, st>>>(kb, vb, c32, s.N, s.nk, o);
  } else {
    cudaFuncSetAttribute(linear_state_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    linear_state_kernel<64><<<grid, LIN_THREADS, smem, st>>>(kb, vb, c32, s.N, s.nk, o);
  }
  return cudaGetLastError();
}

cudaError_t launch_linear_reduce(const Shape& s, const float* hpart, const float* zpart, float* Htot, float* Ztot,
                                 cudaStream_t st) {
  const int DD = s.d * s.d;
  dim3 grid((DD + 255) / 256, s.BH);
  linear_reduce_kernel<<<grid, 256, 0, st>>>(hpart, zpart, linear_chunks(s.nk), s.d, Htot, Ztot);
  return cudaGetLastError();
}

}  // namespace sla2
