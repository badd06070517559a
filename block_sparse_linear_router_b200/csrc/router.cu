// The learnable router (SLA2 summary page, step 1; SLA2 detail page §3
// "Learnable Router" and §7 note 1 on K smoothing):
//
//   pool      one pass over Q, K (and V): Qbar (fp32), exact fp64 column sums of
//             every 64-token key block, the INT8 Q-hat of every 128-token query
//             block, and each channel's |V| maximum (for the FP8 V scale).
//   colmean   c = (sum over all key blocks) / N in fp64; fp32 copy for K_s.
//   proj      A = Qbar Wq, Bk = (Kbar - c) Wk  (y = x W, W stored [d_in][d_out]).
//   topk      s_ij = A_i . Bk_j / sqrt(d) in fp32; per row the k largest,
//             ties to the lower block index; mask M_c and ascending index list.
//
// HBM-bound: pool reads Q, K, V once (bf16) and writes Q-hat; the rest touches
// O((nq + nk) d) bytes per head.
#include <cuda_bf16.h>

#include "device.cuh"
#include "kernels.cuh"

namespace sla2 {

namespace {

__device__ __forceinline__ void unpack8(const uint4& w, float (&x)[8]) {
  x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x);
  x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
  x[4] = bf16_lo(w.z); x[5] = bf16_hi(w.z);
  x[6] = bf16_lo(w.w); x[7] = bf16_hi(w.w);
}

__device__ __forceinline__ float block_max_256(float v, float* red8) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red8[w] = v;
  __syncthreads();
  float m = red8[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) m = fmaxf(m, red8[i]);
  return m;
}

// Symmetric INT8 of one value given the block's amax (fp32, RNE, no FMA).
__device__ __forceinline__ int quant_i8(float x, float inv) {
  int qv = __float2int_rn(__fmul_rn(x, inv));
  return max(-127, min(127, qv));
}

template <int D>
__global__ void __launch_bounds__(256) pool_kernel(const __nv_bfloat16* __restrict__ q,
                                                   const __nv_bfloat16* __restrict__ k,
                                                   const __nv_bfloat16* __restrict__ v, int N, int nq, int nk,
                                                   float* __restrict__ qbar, double* __restrict__ ksum,
                                                   int8_t* __restrict__ qhat, float* __restrict__ sq,
                                                   unsigned* __restrict__ vamax) {
  constexpr int TPR = D / 8;       // threads per row, 8 channels each
  constexpr int RPP = 256 / TPR;   // rows per pass
  constexpr int NP = BQ / RPP;     // passes over the 128 rows
  __shared__ double red[RPP * D];
  __shared__ float red8[8];
  const int i = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
  const int cg = tid % TPR, rg = tid / TPR;
  const size_t base = ((size_t)bh * N + (size_t)i * BQ) * D + cg * 8;

  uint4 wq[NP], wk[NP], wv[NP];
#pragma unroll
  for (int p = 0; p < NP; ++p) wq[p] = __ldg(reinterpret_cast<const uint4*>(q + base + (size_t)(p * RPP + rg) * D));
#pragma unroll
  for (int p = 0; p < NP; ++p) wk[p] = __ldg(reinterpret_cast<const uint4*>(k + base + (size_t)(p * RPP + rg) * D));
  if (vamax) {
#pragma unroll
    for (int p = 0; p < NP; ++p) wv[p] = __ldg(reinterpret_cast<const uint4*>(v + base + (size_t)(p * RPP + rg) * D));
  }

  // ---- Q: pooled mean (exact fp64 sum, one rounding to fp32) and INT8 Q-hat
  double cs[8];
  float amax = 0.f;
#pragma unroll
  for (int c = 0; c < 8; ++c) cs[c] = 0.0;
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    float x[8];
    unpack8(wq[p], x);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      cs[c] += (double)x[c];
      amax = fmaxf(amax, fabsf(x[c]));
    }
  }
#pragma unroll
  for (int c = 0; c < 8; ++c) red[rg * D + cg * 8 + c] = cs[c];
  __syncthreads();
  if (tid < D) {
    double s = 0.0;
    for (int r = 0; r < RPP; ++r) s += red[r * D + tid];
    qbar[((size_t)bh * nq + i) * D + tid] = (float)(s / (double)BQ);
  }
  if (qhat) {
    const float a = block_max_256(amax, red8);
    const float inv = a > 0.f ? __fdiv_rn(127.f, a) : 0.f;
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      float x[8];
      unpack8(wq[p], x);
      uint32_t lo = 0, hi = 0;
#pragma unroll
      for (int c = 0; c < 4; ++c) lo |= (uint32_t)(quant_i8(x[c], inv) & 0xFF) << (8 * c);
#pragma unroll
      for (int c = 0; c < 4; ++c) hi |= (uint32_t)(quant_i8(x[c + 4], inv) & 0xFF) << (8 * c);
      *reinterpret_cast<uint2*>(qhat + base + (size_t)(p * RPP + rg) * D) = make_uint2(lo, hi);
    }
    if (tid == 0) sq[(size_t)bh * nq + i] = a > 0.f ? __fdiv_rn(a, 127.f) : 0.f;
  }

  // ---- K: exact fp64 column sums of the two 64-token key blocks
#pragma unroll
  for (int half = 0; half < 2; ++half) {
#pragma unroll
    for (int c = 0; c < 8; ++c) cs[c] = 0.0;
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      if ((p * RPP) / BKB != half) continue;
      float x[8];
      unpack8(wk[p], x);
#pragma unroll
      for (int c = 0; c < 8; ++c) cs[c] += (double)x[c];
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < 8; ++c) red[rg * D + cg * 8 + c] = cs[c];
    __syncthreads();
    if (tid < D) {
      double s = 0.0;
      for (int r = 0; r < RPP; ++r) s += red[r * D + tid];
      ksum[((size_t)bh * nk + 2 * i + half) * D + tid] = s;
    }
  }

  // ---- V: per-channel |V| maximum (non-negative floats order like their bits)
  if (vamax) {
    float vm[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) vm[c] = 0.f;
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      float x[8];
      unpack8(wv[p], x);
#pragma unroll
      for (int c = 0; c < 8; ++c) vm[c] = fmaxf(vm[c], fabsf(x[c]));
    }
    float* fred = reinterpret_cast<float*>(red);
    __syncthreads();
#pragma unroll
    for (int c = 0; c < 8; ++c) fred[rg * D + cg * 8 + c] = vm[c];
    __syncthreads();
    if (tid < D) {
      float m = 0.f;
      for (int r = 0; r < RPP; ++r) m = fmaxf(m, fred[r * D + tid]);
      atomicMax(vamax + (size_t)bh * D + tid, __float_as_uint(m));
    }
  }
}

__global__ void colmean_kernel(const double* __restrict__ ksum, int nk, int N, int D, double* __restrict__ c64,
                               float* __restrict__ c32) {
  const int bh = blockIdx.x;
  for (int e = threadIdx.x; e < D; e += blockDim.x) {
    double s = 0.0;
    for (int j = 0; j < nk; ++j) s += ksum[((size_t)bh * nk + j) * D + e];
    const double m = s / (double)N;
    c64[(size_t)bh * D + e] = m;
    c32[(size_t)bh * D + e] = (float)m;
  }
}

constexpr int PROJ_ROWS = 32;

template <int D>
__global__ void __launch_bounds__(256) proj_kernel(const float* __restrict__ qbar, const double* __restrict__ ksum,
                                                   const double* __restrict__ c64, const float* __restrict__ wq,
                                                   const float* __restrict__ wk, int H, int nq, int nk,
                                                   float* __restrict__ A, float* __restrict__ Bk) {
  extern __shared__ float psm[];
  float* W = psm;              // [D][D]
  float* X = psm + D * D;      // [PROJ_ROWS][D]
  const int bh = blockIdx.y, h = bh % H, tid = threadIdx.x;
  const int nqb = (nq + PROJ_ROWS - 1) / PROJ_ROWS;
  const bool isq = (int)blockIdx.x < nqb;
  const int r0 = (isq ? blockIdx.x : blockIdx.x - nqb) * PROJ_ROWS;
  const int nrows = isq ? nq : nk;
  const float* Wsrc = (isq ? wq : wk) + (size_t)h * D * D;
  for (int t = tid; t < D * D / 4; t += 256)
    reinterpret_cast<float4*>(W)[t] = __ldg(reinterpret_cast<const float4*>(Wsrc) + t);
  for (int t = tid; t < PROJ_ROWS * D; t += 256) {
    const int r = t / D, e = t % D, row = r0 + r;
    float x = 0.f;
    if (row < nrows) {
      if (isq) {
        x = qbar[((size_t)bh * nq + row) * D + e];
      } else {
        x = (float)(ksum[((size_t)bh * nk + row) * D + e] / (double)BKB - c64[(size_t)bh * D + e]);
      }
    }
    X[t] = x;
  }
  __syncthreads();
  constexpr int GROUPS = 256 / D;
  constexpr int RPG = PROJ_ROWS / GROUPS;
  const int col = tid % D, g = tid / D;
  float* out = isq ? A : Bk;
  for (int rr = 0; rr < RPG; ++rr) {
    const int r = g * RPG + rr, row = r0 + r;
    float acc = 0.f;
#pragma unroll 8
    for (int f = 0; f < D; ++f) acc = fmaf(X[r * D + f], W[f * D + col], acc);
    if (row < nrows) out[((size_t)bh * nrows + row) * D + col] = acc;
  }
}

constexpr int TOPK_ROWS = 8;          // one warp per query-block row
constexpr int TOPK_MAX_NK = 6144;     // scores of 8 rows stay in shared memory

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (f == 0.f) u = 0u;                // +0 and -0 tie, as in exact arithmetic
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int D>
__global__ void __launch_bounds__(256) scores_topk_kernel(const float* __restrict__ A, const float* __restrict__ Bk,
                                                          int nq, int nk, int k, uint8_t* __restrict__ mask,
                                                          int32_t* __restrict__ idx, float* __restrict__ scores) {
  extern __shared__ float tsm[];
  float* As = tsm;                          // [TOPK_ROWS][D]
  float* Bt = As + TOPK_ROWS * D;           // [D][33]
  float* sc = Bt + D * 33;                  // [TOPK_ROWS][nk]
  const int bh = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row0 = blockIdx.x * TOPK_ROWS, row = row0 + warp;
  const bool valid = row < nq;
  for (int t = tid; t < TOPK_ROWS * D; t += 256) {
    const int r = t / D;
    As[t] = (row0 + r < nq) ? A[((size_t)bh * nq + row0) * D + t] : 0.f;
  }
  const float sqrt_d = sqrtf((float)D);
  for (int jt = 0; jt < nk; jt += 32) {
    __syncthreads();
    for (int t = tid; t < 32 * D; t += 256) {
      const int jj = t / D, e = t % D;
      Bt[e * 33 + jj] = (jt + jj < nk) ? Bk[((size_t)bh * nk + jt + jj) * D + e] : 0.f;
    }
    __syncthreads();
    if (valid && jt + lane < nk) {
      float acc = 0.f;
#pragma unroll 8
      for (int e = 0; e < D; ++e) acc = fmaf(As[warp * D + e], Bt[e * 33 + lane], acc);
      sc[warp * nk + jt + lane] = __fdiv_rn(acc, sqrt_d);
    }
  }
  __syncwarp();
  if (!valid) return;
  const float* s = sc + warp * nk;
  // k-th largest key by a bitwise search from the top bit down
  uint32_t T = 0u;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    int cnt = 0;
    for (int j = lane; j < nk; j += 32) cnt += order_key(s[j]) >= cand;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (cnt >= k) T = cand;
  }
  int gt = 0;
  for (int j = lane; j < nk; j += 32) gt += order_key(s[j]) > T;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) gt += __shfl_xor_sync(0xffffffffu, gt, o);
  const int need = k - gt;          // how many entries equal to T are kept (lowest indices first)
  const uint32_t lt = (1u << lane) - 1u;
  int eq_seen = 0, pos = 0;
  const size_t rbase = (size_t)bh * nq + row;
  for (int jb = 0; jb < nk; jb += 32) {
    const int j = jb + lane;
    const bool in = j < nk;
    const float sv = in ? s[j] : 0.f;
    const uint32_t key = in ? order_key(sv) : 0u;
    const bool is_gt = in && key > T;
    const bool is_eq = in && key == T;
    const uint32_t eqm = __ballot_sync(0xffffffffu, is_eq);
    const bool sel = is_gt || (is_eq && (eq_seen + __popc(eqm & lt)) < need);
    eq_seen += __popc(eqm);
    const uint32_t selm = __ballot_sync(0xffffffffu, sel);
    if (in) {
      mask[rbase * nk + j] = sel ? 1 : 0;
      if (scores) scores[rbase * nk + j] = sv;
    }
    if (sel) idx[rbase * k + pos + __popc(selm & lt)] = j;
    pos += __popc(selm);
  }
}

}  // namespace

cudaError_t launch_pool(const Shape& s, const void* q, const void* k, const void* v, float* qbar, double* ksum,
                        int8_t* qhat, float* sq, unsigned* vamax, cudaStream_t st) {
  dim3 grid(s.nq, s.BH);
  auto qb = static_cast<const __nv_bfloat16*>(q);
  auto kb = static_cast<const __nv_bfloat16*>(k);
  auto vb = static_cast<const __nv_bfloat16*>(v);
  if (s.d == 128)
    pool_kernel<128><<<grid, 256, 0, st>>>(qb, kb, vb, s.N, s.nq, s.nk, qbar, ksum, qhat, sq, vamax);
  else
    pool_kernel<64><<<grid, 256, 0, st>>>(qb, kb, vb, s.N, s.nq, s.nk, qbar, ksum, qhat, sq, vamax);
  return cudaGetLastError();
}

cudaError_t launch_colmean(const Shape& s, const double* ksum, double* c64, float* c32, cudaStream_t st) {
  colmean_kernel<<<s.BH, 128, 0, st>>>(ksum, s.nk, s.N, s.d, c64, c32);
  return cudaGetLastError();
}

cudaError_t launch_proj(const Shape& s, int H, const float* qbar, const double* ksum, const double* c64,
                          const float* wq, const float* wk, float* A, float* Bk, cudaStream_t st) {
  const int nb = (s.nq + PROJ_ROWS - 1) / PROJ_ROWS + (s.nk + PROJ_ROWS - 1) / PROJ_ROWS;
  dim3 grid(nb, s.BH);
  const size_t smem = (size_t)(s.d * s.d + PROJ_ROWS * s.d) * sizeof(float);
  if (s.d == 128) {
    cudaFuncSetAttribute(proj_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    proj_kernel<128><<<grid, 256, smem, st>>>(qbar, ksum, c64, wq, wk, H, s.nq, s.nk, A, Bk);
  } else {
    cudaFuncSetAttribute(proj_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    proj_kernel<64><<<grid, 256, smem, st>>>(qbar, ksum, c64, wq, wk, H, s.nq, s.nk, A, Bk);
  }
  return cudaGetLastError();
}

int scores_topk_max_nk() { return TOPK_MAX_NK; }

cudaError_t launch_scores_topk(const Shape& s, const float* A, const float* Bk, uint8_t* mask, int32_t* idx,
                               float* scores_opt, cudaStream_t st) {
  dim3 grid((s.nq + TOPK_ROWS - 1) / TOPK_ROWS, s.BH);
  const size_t smem = (size_t)(TOPK_ROWS * s.d + s.d * 33 + TOPK_ROWS * s.nk) * sizeof(float);
  if (s.d == 128) {
    cudaFuncSetAttribute(scores_topk_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    scores_topk_kernel<128><<<grid, 256, smem, st>>>(A, Bk, s.nq, s.nk, s.k, mask, idx, scores_opt);
  } else {
    cudaFuncSetAttribute(scores_topk_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    scores_topk_kernel<64><<<grid, 256, smem, st>>>(A, Bk, s.nq, s.nk, s.k, mask, idx, scores_opt);
  }
  return cudaGetLastError();
}

}  // namespace sla2
