// Backward pass of the SLA2 attention (SLA2 detail page §7 note 3: the
// gradient is derived by hand, and the linear branch's dH_i and dZ_i are
// formed once per query block so that each key block needs one matrix
// addition per selecting query block; §2 table: the low-bit kernels serve the
// forward pass, the backward runs at higher precision). It differentiates the
// unquantised forward O = alpha O_s + (1 - alpha) O_l for the router's hard
// mask, held fixed (piecewise constant in Q, K and the projections), with K
// smoothing K_s = K - colmean(K) included. Arithmetic is fp32 on the CUDA
// cores throughout; the per-key-block states h_j come from the linear-state
// pass (tensor-core products with fp16 operands, fp32 accumulation).
//
// Kernels, in launch order (after the router and the linear-state pass):
//   bwd_sparse_kernel  one CTA per (head, query block): two passes over the
//       selected key blocks. Pass 1 recomputes the softmax statistics and
//       O_s; pass 2 forms P, dP = dO_s V^T, dS = P (dP - rowsum(dO_s O_s)) and
//       dQ_i = dS K_s / sqrt(d) (rows, two threads per row), then per key
//       block dK_s += dS^T Q_i / sqrt(d) and dV += P^T dO_s (tiled products,
//       fp32 atomic adds). It also leaves sum(dO * O_s) of the block for dalpha.
//   bwd_linear_kernel  one CTA per (head, query block): H_i, Z_i (from the
//       totals minus the selected states), phi(Q_i), O_l, the gradients of the
//       numerator and denominator, dQ_i += phi-backward, dalpha, and
//       dH_i = phi(Q_i)^T dnum, dZ_i = phi(Q_i)^T dden, added to a per-head
//       total and subtracted from each selected key block's accumulator.
//   bwd_keys_kernel    one CTA per (head, key block): dh_j = total + its
//       accumulator (the sum over the query blocks that did not select j),
//       dV_j += phi(K_j) dh_j, dphi = V_j dh_j^T + dz_j, dK_s += phi-backward.
//   bwd_colmean_kernel dK = dK_s - colmean(dK_s) per head and channel.
// The library's states are stored transposed (h^T[channel][feature]); the
// gradient accumulators use the same orientation.
#include <cuda_bf16.h>

#include "device.cuh"
#include "kernels.cuh"

namespace sla2 {

namespace {

constexpr int BW_THREADS = 256;

__device__ __forceinline__ float bf16f(const __nv_bfloat16* p, size_t i) { return __bfloat162float(p[i]); }

// Shared layout of bwd_sparse_kernel, in bytes.
template <int D>
struct SpB {
  static constexpr int Q = 0;                       // Q_i  [128][D]  bf16 (exact)
  static constexpr int DO = Q + BQ * D * 2;         // dO_s [128][D]  fp32 (alpha dO)
  static constexpr int KS = DO + BQ * D * 4;        // K_s,j [64][D]  fp32
  static constexpr int V = KS + BKB * D * 4;        // V_j  [64][D]   bf16 (exact)
  static constexpr int P = V + BKB * D * 2;         // P    [128][64] fp32
  static constexpr int DS = P + BQ * BKB * 4;       // dS   [128][64] fp32
  static constexpr size_t BYTES = DS + BQ * BKB * 4;
  static_assert(BYTES <= 232448, "shared memory per CTA");
};

// Loads key block j of head bh: K_s = K - c (fp32) and V (bf16).
template <int D>
__device__ void load_kv_block(const __nv_bfloat16* k, const __nv_bfloat16* v, const float* c32, int bh, int N, int j,
                              float* ks, __nv_bfloat16* vs) {
  const size_t base = ((size_t)bh * N + (size_t)j * BKB) * D;
  for (int e = threadIdx.x; e < BKB * D; e += blockDim.x) {
    ks[e] = bf16f(k, base + e) - c32[(size_t)bh * D + e % D];
    vs[e] = v[base + e];
  }
}

template <int D>
__global__ void __launch_bounds__(BW_THREADS, 1) bwd_sparse_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    const float* __restrict__ c32, const float* __restrict__ alpha, int H, const float* __restrict__ dout,
    const int32_t* __restrict__ idx, Shape s, float* __restrict__ dq, float* __restrict__ dks, float* __restrict__ dv,
    float* __restrict__ dos_sum) {
  using L = SpB<D>;
  extern __shared__ __align__(16) uint8_t smb[];
  __nv_bfloat16* Qs = reinterpret_cast<__nv_bfloat16*>(smb + L::Q);
  float* DOs = reinterpret_cast<float*>(smb + L::DO);
  float* Ks = reinterpret_cast<float*>(smb + L::KS);
  __nv_bfloat16* Vs = reinterpret_cast<__nv_bfloat16*>(smb + L::V);
  float* Ps = reinterpret_cast<float*>(smb + L::P);
  float* DSs = reinterpret_cast<float*>(smb + L::DS);
  const int bh = blockIdx.x / s.nq, qi = blockIdx.x % s.nq;
  const int tid = threadIdx.x;
  const int r = tid >> 1, half = tid & 1;              // two threads per query row
  constexpr int HD = D / 2;                            // features of this thread
  const float al = alpha[(size_t)(bh % H) * s.nq + qi];
  const float rs = rsqrtf((float)D);
  const size_t row0 = (size_t)bh * s.N + (size_t)qi * BQ;
  for (int e = tid; e < BQ * D; e += BW_THREADS) {
    Qs[e] = q[row0 * D + e];
    DOs[e] = al * dout[row0 * D + e];
  }
  const int32_t* sel = idx + ((size_t)bh * s.nq + qi) * s.k;
  // this thread's half row of Q and of dO_s, in registers
  float qr[HD], dor[HD];
#pragma unroll
  for (int f = 0; f < HD; ++f) {
    qr[f] = bf16f(q, (row0 + r) * D + half * HD + f);
    dor[f] = al * dout[(row0 + r) * D + half * HD + f];
  }

  // ---- pass 1: row max, row sum and O_s = P V / l
  float m = -INFINITY, l = 0.f;
  float acc[HD];
#pragma unroll
  for (int f = 0; f < HD; ++f) acc[f] = 0.f;
  for (int n = 0; n < s.k; ++n) {
    const int j = __ldg(sel + n);
    __syncthreads();
    load_kv_block<D>(k, v, c32, bh, s.N, j, Ks, Vs);
    __syncthreads();
    for (int t = 0; t < BKB; ++t) {
      const float* kt = Ks + t * D + half * HD;
      float p = 0.f;
#pragma unroll 16
      for (int f = 0; f < HD; ++f) p = fmaf(qr[f], kt[f], p);
      p += __shfl_xor_sync(0xffffffffu, p, 1);
      const float sc = p * rs;
      const float mn = fmaxf(m, sc);
      const float cr = expf(m - mn), e = expf(sc - mn);
      l = l * cr + e;
      const __nv_bfloat16* vt = Vs + t * D + half * HD;
#pragma unroll 16
      for (int f = 0; f < HD; ++f) acc[f] = fmaf(e, __bfloat162float(vt[f]), acc[f] * cr);
      m = mn;
    }
  }
  // D_r = rowsum(dO_s * O_s); also sum(dO * O_s) over the block for dalpha
  float dr = 0.f;
#pragma unroll 16
  for (int f = 0; f < HD; ++f) dr = fmaf(dor[f], acc[f] / l, dr);
  dr += __shfl_xor_sync(0xffffffffu, dr, 1);
  {
    // sum over the block of dO * O_s (the raw upstream gradient), for dalpha
    const float* gr = dout + (row0 + r) * D + half * HD;
    float blk = 0.f;
#pragma unroll 16
    for (int f = 0; f < HD; ++f) blk = fmaf(gr[f], acc[f] / l, blk);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) blk += __shfl_xor_sync(0xffffffffu, blk, o);
    __shared__ float red[BW_THREADS / 32];
    if ((tid & 31) == 0) red[tid >> 5] = blk;
    __syncthreads();
    if (tid == 0) {
      float tsum = 0.f;
      for (int w = 0; w < BW_THREADS / 32; ++w) tsum += red[w];
      dos_sum[blockIdx.x] = tsum;
    }
  }
  // ---- pass 2: P, dP, dS, dQ (rows); dK_s and dV per key block (tiles)
  float dqa[HD];
#pragma unroll
  for (int f = 0; f < HD; ++f) dqa[f] = 0.f;
  for (int n = 0; n < s.k; ++n) {
    const int j = __ldg(sel + n);
    __syncthreads();
    load_kv_block<D>(k, v, c32, bh, s.N, j, Ks, Vs);
    __syncthreads();
    for (int t = 0; t < BKB; ++t) {
      const float* kt = Ks + t * D + half * HD;
      const __nv_bfloat16* vt = Vs + t * D + half * HD;
      float p = 0.f, dp = 0.f;
#pragma unroll 16
      for (int f = 0; f < HD; ++f) {
        p = fmaf(qr[f], kt[f], p);
        dp = fmaf(dor[f], __bfloat162float(vt[f]), dp);
      }
      p += __shfl_xor_sync(0xffffffffu, p, 1);
      dp += __shfl_xor_sync(0xffffffffu, dp, 1);
      const float pr = expf(p * rs - m) / l;
      const float ds = pr * (dp - dr);
#pragma unroll 16
      for (int f = 0; f < HD; ++f) dqa[f] = fmaf(ds, kt[f], dqa[f]);
      if (half == 0) {
        Ps[r * BKB + t] = pr;
        DSs[r * BKB + t] = ds;
      }
    }
    __syncthreads();
    // dK_s[j] += dS^T Q / sqrt(d), dV[j] += P^T dO_s: 64 x D outputs, D / 4 per thread
    const size_t kbase = ((size_t)bh * s.N + (size_t)j * BKB) * D;
    for (int o = tid; o < BKB * D; o += BW_THREADS) {
      const int t = o / D, f = o % D;
      float gk = 0.f, gv = 0.f;
#pragma unroll 8
      for (int rr = 0; rr < BQ; ++rr) {
        gk = fmaf(DSs[rr * BKB + t], __bfloat162float(Qs[rr * D + f]), gk);
        gv = fmaf(Ps[rr * BKB + t], DOs[rr * D + f], gv);
      }
      atomicAdd(dks + kbase + o, gk * rs);
      atomicAdd(dv + kbase + o, gv);
    }
  }
  float* dqr = dq + (row0 + r) * D + half * HD;
#pragma unroll 16
  for (int f = 0; f < HD; ++f) dqr[f] = dqa[f] * rs;
}

// Shared layout of bwd_linear_kernel (floats).
template <int D>
struct LiB {
  static constexpr int HT = 0;                  // H_i^T [D][D+1] (channel, feature)
  static constexpr int A = HT + D * (D + 1);    // phi(Q_i) [128][D]
  static constexpr int DN = A + BQ * D;         // dnum [128][D]
  static constexpr int Z = DN + BQ * D;         // Z_i [D]
  static constexpr int DD = Z + D;              // dden [128]
  static constexpr int TOTAL = DD + BQ + 32;
  static constexpr size_t BYTES = (size_t)TOTAL * 4;
  static_assert(BYTES <= 232448, "shared memory per CTA");
};

template <int D>
__global__ void __launch_bounds__(BW_THREADS, 1) bwd_linear_kernel(
    const __nv_bfloat16* __restrict__ q, const float* __restrict__ alpha, int H, const float* __restrict__ dout,
    const int32_t* __restrict__ idx, const float* __restrict__ hT, const float* __restrict__ z,
    const float* __restrict__ HtotT, const float* __restrict__ Ztot, const float* __restrict__ dos_sum, Shape s,
    float* __restrict__ dq, float* __restrict__ dHacc, float* __restrict__ dZacc, float* __restrict__ dHtot,
    float* __restrict__ dZtot, float* __restrict__ dalpha) {
  using L = LiB<D>;
  extern __shared__ float sm[];
  float* Ht = sm + L::HT;
  float* As = sm + L::A;
  float* DN = sm + L::DN;
  float* Zs = sm + L::Z;
  float* DDs = sm + L::DD;
  float* red = DDs + BQ;
  const int bh = blockIdx.x / s.nq, qi = blockIdx.x % s.nq;
  const int h = bh % H;
  const int tid = threadIdx.x;
  const int r = tid >> 1, half = tid & 1;
  constexpr int HD = D / 2;
  const float al = alpha[(size_t)h * s.nq + qi];
  const size_t row0 = (size_t)bh * s.N + (size_t)qi * BQ;
  const int32_t* sel = idx + ((size_t)bh * s.nq + qi) * s.k;
  const bool linear = s.k < s.nk;
  // H_i^T = H_total^T - sum of the selected h_j^T;  Z_i likewise
  if (linear) {
    for (int e = tid; e < D * D; e += BW_THREADS) {
      float acc = HtotT[(size_t)bh * D * D + e];
      for (int n = 0; n < s.k; ++n) acc -= hT[((size_t)bh * s.nk + __ldg(sel + n)) * D * D + e];
      Ht[(e / D) * (D + 1) + e % D] = acc;
    }
    for (int f = tid; f < D; f += BW_THREADS) {
      float acc = Ztot[(size_t)bh * D + f];
      for (int n = 0; n < s.k; ++n) acc -= z[((size_t)bh * s.nk + __ldg(sel + n)) * D + f];
      Zs[f] = acc;
    }
  }
  // phi(Q_i) rows (two threads per row)
  float a[HD];
  {
    const size_t qo = (row0 + r) * D + half * HD;
    float mx = -INFINITY;
#pragma unroll 16
    for (int f = 0; f < HD; ++f) {
      a[f] = bf16f(q, qo + f);
      mx = fmaxf(mx, a[f]);
    }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    float sum = 0.f;
#pragma unroll 16
    for (int f = 0; f < HD; ++f) {
      a[f] = expf(a[f] - mx);
      sum += a[f];
    }
    sum += __shfl_xor_sync(0xffffffffu, sum, 1);
    const float inv = 1.f / sum;
#pragma unroll 16
    for (int f = 0; f < HD; ++f) {
      a[f] *= inv;
      As[r * D + half * HD + f] = a[f];
    }
  }
  __syncthreads();
  // O_l = num / den, dnum = dO_l / den, dden = -rowsum(dO_l * O_l) / den (this thread: channels of its half)
  float dol[HD], num[HD];
  const float* dor = dout + (row0 + r) * D + half * HD;
  float den = 0.f, dsl = 0.f;          // den over all features; sum(dO * O_l) over this half
  if (linear) {
    for (int f = 0; f < D; ++f) den = fmaf(As[r * D + f], Zs[f], den);
#pragma unroll 4
    for (int c = 0; c < HD; ++c) {
      const float* hrow = Ht + (half * HD + c) * (D + 1);   // channel half*HD + c, all features
      float acc = 0.f;
      for (int f = 0; f < D; ++f) acc = fmaf(As[r * D + f], hrow[f], acc);
      num[c] = acc;
    }
  }
  float drow = 0.f;                    // sum over channels of dO_l * O_l (this half)
#pragma unroll 16
  for (int c = 0; c < HD; ++c) {
    const float ol = linear ? num[c] / den : 0.f;
    dol[c] = (1.f - al) * dor[c];
    dsl = fmaf(dor[c], ol, dsl);
    drow = fmaf(dol[c], ol, drow);
  }
  drow += __shfl_xor_sync(0xffffffffu, drow, 1);
  // dalpha_i = sum(dO * O_s) - sum(dO * O_l); the sparse kernel left sum(dO * O_s)
  {
    float blk = dsl;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) blk += __shfl_xor_sync(0xffffffffu, blk, o);
    if ((tid & 31) == 0) red[tid >> 5] = blk;
    __syncthreads();
    if (tid == 0) {
      float tsum = 0.f;
      for (int w = 0; w < BW_THREADS / 32; ++w) tsum += red[w];
      atomicAdd(dalpha + (size_t)h * s.nq + qi, dos_sum[blockIdx.x] - tsum);   // summed over the batch
    }
  }
  if (!linear) return;
  const float dden = -drow / den;
#pragma unroll 16
  for (int c = 0; c < HD; ++c) DN[r * D + half * HD + c] = dol[c] / den;
  if (half == 0) DDs[r] = dden;
  __syncthreads();
  // da[f] = sum_ch dnum[ch] H_i[f][ch] + dden Z_i[f] (features of this half), then phi-backward
  float da[HD];
  float dot = 0.f;
#pragma unroll 4
  for (int f = 0; f < HD; ++f) {
    const int ff = half * HD + f;
    float acc = dden * Zs[ff];
    for (int ch = 0; ch < D; ++ch) acc = fmaf(DN[r * D + ch], Ht[ch * (D + 1) + ff], acc);
    da[f] = acc;
    dot = fmaf(acc, a[f], dot);
  }
  dot += __shfl_xor_sync(0xffffffffu, dot, 1);
  float* dqr = dq + (row0 + r) * D + half * HD;
#pragma unroll 16
  for (int f = 0; f < HD; ++f) dqr[f] += a[f] * (da[f] - dot);
  // dH_i^T[ch][f] = sum_r dnum[r][ch] a[r][f]; dZ_i[f] = sum_r dden[r] a[r][f]
  float* dHt = dHtot + (size_t)bh * D * D;
  for (int o = tid; o < D * D; o += BW_THREADS) {
    const int ch = o / D, f = o % D;
    float acc = 0.f;
#pragma unroll 8
    for (int rr = 0; rr < BQ; ++rr) acc = fmaf(DN[rr * D + ch], As[rr * D + f], acc);
    atomicAdd(dHt + o, acc);
    for (int n = 0; n < s.k; ++n) atomicAdd(dHacc + ((size_t)bh * s.nk + __ldg(sel + n)) * D * D + o, -acc);
  }
  for (int f = tid; f < D; f += BW_THREADS) {
    float acc = 0.f;
    for (int rr = 0; rr < BQ; ++rr) acc = fmaf(DDs[rr], As[rr * D + f], acc);
    atomicAdd(dZtot + (size_t)bh * D + f, acc);
    for (int n = 0; n < s.k; ++n) atomicAdd(dZacc + ((size_t)bh * s.nk + __ldg(sel + n)) * D + f, -acc);
  }
}

// Shared layout of bwd_keys_kernel (floats).
template <int D>
struct KeB {
  static constexpr int DHT = 0;                    // dh_j^T [D][D+1] (channel, feature)
  static constexpr int PH = DHT + D * (D + 1);     // phi(K_s,j) [64][D+1]
  static constexpr int V = PH + BKB * (D + 1);     // V_j [64][D+1]
  static constexpr int DZ = V + BKB * (D + 1);     // dz_j [D]
  static constexpr int TOTAL = DZ + D;
  static constexpr size_t BYTES = (size_t)TOTAL * 4;
  static_assert(BYTES <= 232448, "shared memory per CTA");
};

template <int D>
__global__ void __launch_bounds__(BW_THREADS, 1) bwd_keys_kernel(
    const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v, const float* __restrict__ c32,
    const float* __restrict__ dHacc, const float* __restrict__ dZacc, const float* __restrict__ dHtot,
    const float* __restrict__ dZtot, Shape s, float* __restrict__ dks, float* __restrict__ dv) {
  using L = KeB<D>;
  extern __shared__ float sm[];
  float* DHT = sm + L::DHT;
  float* PH = sm + L::PH;
  float* Vs = sm + L::V;
  float* DZ = sm + L::DZ;
  const int bh = blockIdx.x / s.nk, j = blockIdx.x % s.nk;
  const int tid = threadIdx.x;
  for (int o = tid; o < D * D; o += BW_THREADS)
    DHT[(o / D) * (D + 1) + o % D] = dHtot[(size_t)bh * D * D + o] + dHacc[((size_t)bh * s.nk + j) * D * D + o];
  for (int f = tid; f < D; f += BW_THREADS) DZ[f] = dZtot[(size_t)bh * D + f] + dZacc[((size_t)bh * s.nk + j) * D + f];
  {
    const size_t base = ((size_t)bh * s.N + (size_t)j * BKB) * D;
    for (int e = tid; e < BKB * D; e += BW_THREADS) {
      const int t = e / D, f = e % D;
      PH[t * (D + 1) + f] = bf16f(k, base + e) - c32[(size_t)bh * D + f];
      Vs[t * (D + 1) + f] = bf16f(v, base + e);
    }
  }
  __syncthreads();
  // phi over the features of each key row (four threads per row)
  {
    const int t = tid >> 2, part = tid & 3;
    constexpr int QD = D / 4;
    float* row = PH + t * (D + 1) + part * QD;
    float mx = -INFINITY;
    for (int f = 0; f < QD; ++f) mx = fmaxf(mx, row[f]);
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    float sum = 0.f;
    for (int f = 0; f < QD; ++f) {
      row[f] = expf(row[f] - mx);
      sum += row[f];
    }
    sum += __shfl_xor_sync(0xffffffffu, sum, 1);
    sum += __shfl_xor_sync(0xffffffffu, sum, 2);
    const float inv = 1.f / sum;
    for (int f = 0; f < QD; ++f) row[f] *= inv;
  }
  __syncthreads();
  // dV[t][ch] += sum_f phi[t][f] dh[f][ch];  dphi[t][f] = sum_ch V[t][ch] dh[f][ch] + dz[f]
  const size_t kbase = ((size_t)bh * s.N + (size_t)j * BKB) * D;
  for (int o = tid; o < BKB * D; o += BW_THREADS) {
    const int t = o / D, ch = o % D;
    float acc = 0.f;
    for (int f = 0; f < D; ++f) acc = fmaf(PH[t * (D + 1) + f], DHT[ch * (D + 1) + f], acc);
    dv[kbase + o] += acc;
  }
  // phi-backward per key row: dK_s[t][f] += phi[t][f] (dphi[t][f] - sum_g dphi[t][g] phi[t][g])
  {
    const int t = tid >> 2, part = tid & 3;
    constexpr int QD = D / 4;
    float dphi[QD];
    float dot = 0.f;
    for (int f = 0; f < QD; ++f) {
      const int ff = part * QD + f;
      float acc = DZ[ff];
      for (int ch = 0; ch < D; ++ch) acc = fmaf(Vs[t * (D + 1) + ch], DHT[ch * (D + 1) + ff], acc);
      dphi[f] = acc;
      dot = fmaf(acc, PH[t * (D + 1) + ff], dot);
    }
    dot += __shfl_xor_sync(0xffffffffu, dot, 1);
    dot += __shfl_xor_sync(0xffffffffu, dot, 2);
    for (int f = 0; f < QD; ++f) {
      const int ff = part * QD + f;
      dks[kbase + (size_t)t * D + ff] += PH[t * (D + 1) + ff] * (dphi[f] - dot);
    }
  }
}

// dK = dK_s - mean over the tokens of dK_s, per (head, channel): one CTA per head.
__global__ void bwd_colmean_kernel(float* __restrict__ dk, int N, int D) {
  const int bh = blockIdx.x, f = threadIdx.x;
  float* base = dk + (size_t)bh * N * D;
  float acc = 0.f;
  for (int t = 0; t < N; ++t) acc += base[(size_t)t * D + f];
  const float mean = acc / (float)N;
  for (int t = 0; t < N; ++t) base[(size_t)t * D + f] -= mean;
}

template <int D>
cudaError_t launch_bwd_t(const Shape& s, int H, const BackwardArgs& a, cudaStream_t st) {
  const int items = s.BH * s.nq;
  cudaError_t e = cudaFuncSetAttribute(bwd_sparse_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SpB<D>::BYTES);
  if (e != cudaSuccess) return e;
  bwd_sparse_kernel<D><<<items, BW_THREADS, SpB<D>::BYTES, st>>>(
      static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k),
      static_cast<const __nv_bfloat16*>(a.v), a.c32, a.alpha, H, a.dout, a.idx, s, a.dq, a.dk, a.dv, a.dos_sum);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = cudaFuncSetAttribute(bwd_linear_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)LiB<D>::BYTES)) != cudaSuccess)
    return e;
  bwd_linear_kernel<D><<<items, BW_THREADS, LiB<D>::BYTES, st>>>(
      static_cast<const __nv_bfloat16*>(a.q), a.alpha, H, a.dout, a.idx, a.hT, a.z, a.HtotT, a.Ztot, a.dos_sum, s,
      a.dq, a.dHacc, a.dZacc, a.dHtot, a.dZtot, a.dalpha);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (s.k < s.nk) {
    if ((e = cudaFuncSetAttribute(bwd_keys_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)KeB<D>::BYTES)) != cudaSuccess)
      return e;
    bwd_keys_kernel<D><<<s.BH * s.nk, BW_THREADS, KeB<D>::BYTES, st>>>(
        static_cast<const __nv_bfloat16*>(a.k), static_cast<const __nv_bfloat16*>(a.v), a.c32, a.dHacc, a.dZacc,
        a.dHtot, a.dZtot, s, a.dk, a.dv);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  bwd_colmean_kernel<<<s.BH, D, 0, st>>>(a.dk, s.N, D);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_backward(const Shape& s, int H, const BackwardArgs& a, cudaStream_t st) {
  return s.d == 128 ? launch_bwd_t<128>(s, H, a, st) : launch_bwd_t<64>(s, H, a, st);
}

}  // namespace sla2
