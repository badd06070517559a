// The learnable router (SLA2 summary page, step 1; SLA2 detail page §3
// "Learnable Router" and §7 note 1 on K smoothing):
//
//   pool      one pass over Q, K (and V): Qbar (fp32), exact fp64 column sums of
//             every 64-token key block, the INT8 Q-hat of every 128-token query
//             block, and each channel's |V| maximum (for the FP8 V scale).
//   colmean   c = (sum over all key blocks) / N in fp64; fp32 copy for K_s.
//   proj      A = Qbar Wq, Bk = (Kbar - c) Wk  (y = x W, W stored [d_in][d_out]).
//   logits    s_ij = A_i . Bk_j / sqrt(d) in fp32.
//   topk      per row the k largest s_ij, ties to the lower block index; mask
//             M_c and ascending index list (soft_topk: the SoftTop-k weights).
//
// HBM-bound: pool reads Q, K, V once (bf16) and writes Q-hat; the rest touches
// O((nq + nk) d) bytes per head.
#include <cuda_bf16.h>

#include "device.cuh"
#include "kernels.cuh"

namespace sla2 {

namespace {

// Symmetric INT8 of one value given the block's amax (fp32, RNE, no FMA).
__device__ __forceinline__ int quant_i8(float x, float inv) {
  int qv = __float2int_rn(__fmul_rn(x, inv));
  return max(-127, min(127, qv));
}

constexpr int POOL_CONS = 256;                    // consumer threads (8 warps)
constexpr int POOL_THREADS = POOL_CONS + 32;      // + one producer warp

template <int D>
struct PoolCfg {
  static constexpr int TILE = BQ * D * 2;        // the 128 bf16 rows of one tensor for one query block
  static constexpr int STAGE = 3 * TILE;         // Q, K, V
  static constexpr int NS = D == 128 ? 2 : 4;    // pipeline depth (192 KB of stages)
  static constexpr int TPR = D / 4;              // threads per row, 4 channels each
  static constexpr int RPP = POOL_CONS / TPR;    // rows per pass
  static constexpr int NP = BQ / RPP;            // passes over the 128 rows
  static constexpr int RED = 8 * D;              // one per-warp partial table [8 warps][D]
  static constexpr int OFF_RED = NS * STAGE;     // fp64 tables for Q, K rows 0..63, K rows 64..127; fp32 for V
  static constexpr int OFF_A = OFF_RED + 3 * RED * 8 + RED * 4;   // per-warp |Q| maxima
  static constexpr int OFF_BAR = OFF_A + 64;
  static constexpr int SMEM = OFF_BAR + 2 * NS * 8 + 16;
  static_assert(SMEM <= 232448, "dynamic shared memory per CTA (227 KB)");
  static_assert(TILE % 16 == 0 && STAGE % 16 == 0 && OFF_BAR % 8 == 0, "bulk-copy and mbarrier alignment");
};

__device__ __forceinline__ void unpack4(const uint2& w, float (&x)[4]) {
  x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x);
  x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
}

// Barrier over the 256 consumer threads that returns, to every one of them,
// whether any of them passed `failed` (so that all take the same exit).
__device__ __forceinline__ bool pool_sync_any(bool failed) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 256, p;\n\tselp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)failed)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void pool_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// Persistent pass over the query blocks (one CTA per SM). A producer warp
// streams each block's 128 rows of Q, K (and V) into shared memory with three
// bulk copies, two blocks ahead of the 8 consumer warps, which reduce them
// there; the rows are contiguous in [B*H][N][d], so every copy is one piece.
template <int D>
__global__ void __launch_bounds__(POOL_THREADS, 1) pool_kernel(const __nv_bfloat16* __restrict__ q,
                                                               const __nv_bfloat16* __restrict__ k,
                                                               const __nv_bfloat16* __restrict__ v, int BH, int N,
                                                               int nq, int nk, float* __restrict__ qbar,
                                                               double* __restrict__ ksum, int8_t* __restrict__ qhat,
                                                               float* __restrict__ sq, unsigned* __restrict__ vamax,
                                                               unsigned* status, unsigned long long budget_ns,
                                                               double* __restrict__ csum) {
  using C = PoolCfg<D>;
  constexpr int TPR = C::TPR, RPP = C::RPP, NP = C::NP, NS = C::NS;
  extern __shared__ __align__(128) uint8_t pool_smem[];
  uint8_t* base = pool_smem;
  double* redq = reinterpret_cast<double*>(base + C::OFF_RED);
  double* redk0 = redq + C::RED;
  double* redk1 = redk0 + C::RED;
  float* redv = reinterpret_cast<float*>(redk1 + C::RED);
  float* reda = reinterpret_cast<float*>(base + C::OFF_A);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + C::OFF_BAR);
  uint64_t* empty = full + NS;
  int* abort_flag = reinterpret_cast<int*>(empty + NS);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int items = BH * nq;
  const uint32_t bytes = (v ? 3u : 2u) * (uint32_t)C::TILE;

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, POOL_CONS / 32);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == POOL_CONS / 32) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int n = 0;
      for (int it = blockIdx.x; it < items; it += gridDim.x, ++n) {
        const int s = n % NS;
        if (n >= NS && !mbar_wait(empty + s, ((n / NS) & 1) ^ 1, abort_flag, status, budget_ns)) break;
        const int bh = it / nq, i = it % nq;
        const size_t row0 = ((size_t)bh * N + (size_t)i * BQ) * D;
        uint8_t* st = base + s * C::STAGE;
        mbar_arrive_expect_tx(full + s, bytes);
        bulk_load(st, q + row0, C::TILE, full + s);
        bulk_load(st + C::TILE, k + row0, C::TILE, full + s);
        if (v) bulk_load(st + 2 * C::TILE, v + row0, C::TILE, full + s);
      }
      // copies still in flight after an abort land before the CTA exits
      for (int j = n - NS < 0 ? 0 : n - NS; j < n; ++j) mbar_wait_drain(full + j % NS, (j / NS) & 1, budget_ns);
    }
    return;
  }

  // -------------------------------------------------------------------- consumers
  const int cg = tid % TPR, rg = tid / TPR;   // channels cg*4 .. +3; rows rg, rg + RPP, ...
  // the head's column sums (threads tid < D): this CTA's block sums of the current head,
  // added to csum when the head changes (exact fp64 sums, so neither the grouping nor
  // the order of the adds changes the result)
  double run = 0.0;
  int run_bh = -1;
  int n = 0;
  for (int it = blockIdx.x; it < items; it += gridDim.x, ++n) {
    const int s = n % NS;
    const bool ok = mbar_wait(full + s, (n / NS) & 1, abort_flag, status, budget_ns);
    // also: every consumer is done with the previous block's partial tables
    if (pool_sync_any(!ok)) break;
    const int bh = it / nq, i = it % nq;
    const uint8_t* sQ = base + s * C::STAGE;
    const uint8_t* sK = sQ + C::TILE;
    const uint8_t* sV = sK + C::TILE;

    // ---- partial sums (exact in fp64) and maxima over this thread's rows
    double cq[4], ck0[4], ck1[4];
    float vm[4], amax = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      cq[c] = 0.0; ck0[c] = 0.0; ck1[c] = 0.0; vm[c] = 0.f;
    }
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      const int row = p * RPP + rg;
      float x[4], y[4];
      unpack4(*reinterpret_cast<const uint2*>(sQ + row * D * 2 + cg * 8), x);
      unpack4(*reinterpret_cast<const uint2*>(sK + row * D * 2 + cg * 8), y);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        cq[c] += (double)x[c];
        amax = fmaxf(amax, fabsf(x[c]));
        if ((p * RPP) / BKB == 0) ck0[c] += (double)y[c];
        else ck1[c] += (double)y[c];
      }
      if (v) {
        unpack4(*reinterpret_cast<const uint2*>(sV + row * D * 2 + cg * 8), x);
#pragma unroll
        for (int c = 0; c < 4; ++c) vm[c] = fmaxf(vm[c], fabsf(x[c]));
      }
    }
    // ---- combine the row groups of a warp (lanes with the same cg), then one row per warp
#pragma unroll
    for (int o = TPR; o < 32; o <<= 1) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        cq[c] += __shfl_xor_sync(0xffffffffu, cq[c], o);
        ck0[c] += __shfl_xor_sync(0xffffffffu, ck0[c], o);
        ck1[c] += __shfl_xor_sync(0xffffffffu, ck1[c], o);
        vm[c] = fmaxf(vm[c], __shfl_xor_sync(0xffffffffu, vm[c], o));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (lane < TPR) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        redq[warp * D + cg * 4 + c] = cq[c];
        redk0[warp * D + cg * 4 + c] = ck0[c];
        redk1[warp * D + cg * 4 + c] = ck1[c];
        redv[warp * D + cg * 4 + c] = vm[c];
      }
    }
    if (lane == 0) reda[warp] = amax;
    pool_sync();

    // ---- per-channel results (fixed order over the 8 warps; the fp64 sums are exact)
    if (tid < D) {
      double sqs = 0.0, s0 = 0.0, s1 = 0.0;
      float m = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        sqs += redq[w * D + tid];
        s0 += redk0[w * D + tid];
        s1 += redk1[w * D + tid];
        m = fmaxf(m, redv[w * D + tid]);
      }
      qbar[((size_t)bh * nq + i) * D + tid] = (float)(sqs / (double)BQ);
      ksum[((size_t)bh * nk + 2 * i) * D + tid] = s0;
      ksum[((size_t)bh * nk + 2 * i + 1) * D + tid] = s1;
      if (csum) {
        if (bh != run_bh) {
          if (run_bh >= 0) atomicAdd(csum + (size_t)run_bh * D + tid, run);
          run = 0.0;
          run_bh = bh;
        }
        run += s0;
        run += s1;
      }
      if (v) atomicMax(vamax + (size_t)bh * D + tid, __float_as_uint(m));   // non-negative floats order like their bits
    }
    // ---- INT8 Q-hat with the block's |Q| maximum
    if (qhat) {
      float a = reda[0];
#pragma unroll
      for (int w = 1; w < 8; ++w) a = fmaxf(a, reda[w]);
      const float inv = a > 0.f ? __fdiv_rn(127.f, a) : 0.f;
      const size_t base_row = (size_t)bh * N + (size_t)i * BQ;
      const bool magic = __float_as_uint(inv) < 0x7F800000u;   // finite (block-uniform); else the saturating path
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        const int row = p * RPP + rg;
        float x[4];
        unpack4(*reinterpret_cast<const uint2*>(sQ + row * D * 2 + cg * 8), x);
        uint32_t w;
        if (magic) {
          w = pack_low_bytes(q8_magic(x[0], inv), q8_magic(x[1], inv), q8_magic(x[2], inv), q8_magic(x[3], inv));
        } else {
          w = 0;
#pragma unroll
          for (int c = 0; c < 4; ++c) w |= (uint32_t)(quant_i8(x[c], inv) & 0xFF) << (8 * c);
        }
        *reinterpret_cast<uint32_t*>(qhat + (base_row + row) * D + cg * 4) = w;
      }
      if (tid == 0) sq[(size_t)bh * nq + i] = a > 0.f ? __fdiv_rn(a, 127.f) : 0.f;
    }
    // ---- the stage is free for the producer
    __syncwarp();
    if (lane == 0) mbar_arrive(empty + s);
  }
  if (csum && tid < D && run_bh >= 0) atomicAdd(csum + (size_t)run_bh * D + tid, run);
}

// c = (sum of the exact per-block column sums) / N in fp64, then the smoothed
// pooled keys Kbar_j - c (fp32). One CTA per (head, 32 columns); 8 warps split
// the key blocks, partial sums are combined in a fixed order.
__global__ void __launch_bounds__(256) colmean_kbar_kernel(const double* __restrict__ ksum, int nk, int N, int D,
                                                           double* __restrict__ c64, float* __restrict__ c32,
                                                           float* __restrict__ kbar_s) {
  __shared__ double part[8][32];
  __shared__ double cm[32];
  const int bh = blockIdx.x, col = blockIdx.y * 32 + (threadIdx.x & 31), w = threadIdx.x >> 5;
  double acc = 0.0;
  for (int j = w; j < nk; j += 8) acc += ksum[((size_t)bh * nk + j) * D + col];
  part[w][threadIdx.x & 31] = acc;
  __syncthreads();
  if (w == 0) {
    double t = 0.0;
#pragma unroll
    for (int u = 0; u < 8; ++u) t += part[u][threadIdx.x];
    const double m = t / (double)N;
    cm[threadIdx.x] = m;
    c64[(size_t)bh * D + col] = m;
    c32[(size_t)bh * D + col] = (float)m;
  }
  __syncthreads();
  const double m = cm[threadIdx.x & 31];
  for (int j = w; j < nk; j += 8) {
    const size_t o = ((size_t)bh * nk + j) * D + col;
    kbar_s[o] = (float)(ksum[o] / (double)BKB - m);
  }
}

// The same from the head's column sums gathered by the pool pass: one thread per
// (head, key block, column), c = csum / N in fp64 and Kbar_j - c in fp32.
__global__ void __launch_bounds__(256) kbar_kernel(const double* __restrict__ csum, const double* __restrict__ ksum,
                                                   int BH, int nk, int N, int D, double* __restrict__ c64,
                                                   float* __restrict__ c32, float* __restrict__ kbar_s) {
  const size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (size_t)BH * nk * D) return;
  const int col = (int)(e % D);
  const size_t bhj = e / D;
  const int bh = (int)(bhj / nk), j = (int)(bhj % nk);
  const double m = csum[(size_t)bh * D + col] / (double)N;
  if (j == 0) {
    c64[(size_t)bh * D + col] = m;
    c32[(size_t)bh * D + col] = (float)m;
  }
  kbar_s[e] = (float)(ksum[e] / (double)BKB - m);
}

// Batched fp32 SIMT GEMM for the router's projections, both of them in one
// launch (blockIdx.z < p0.batch: p0, else p1):
//   C[b][m][n] = (sum_k X[b][m][k] * Y[yb][k][n]) / div,  Y stored [K][N],
// yb = b % ymod. K is the head dimension (a multiple of 16); each product is
// accumulated sequentially over k in fp32. 32 x 64 tile per CTA of 128 threads,
// 4 x 4 per thread, 16-deep k slabs double-buffered in shared memory with the
// next slab's global loads in flight during the current slab's products.
struct GemmProblem {
  const float* X;
  const float* Y;
  float* C;
  int batch, M, N, K, ymod;
  float div;
};

__global__ void __launch_bounds__(128, 8) gemm_f32_kernel(GemmProblem p0, GemmProblem p1) {
  __shared__ __align__(16) float Xs[2][16][36];
  __shared__ __align__(16) float Ys[2][16][68];
  const bool second = (int)blockIdx.z >= p0.batch;
  const int b = second ? (int)blockIdx.z - p0.batch : (int)blockIdx.z;
  const int M = second ? p1.M : p0.M, N = second ? p1.N : p0.N, K = second ? p1.K : p0.K;
  const int m0 = blockIdx.y * 32, n0 = blockIdx.x * 64;
  if (m0 >= M || n0 >= N) return;
  const int yb = b % (second ? p1.ymod : p0.ymod), tid = threadIdx.x;
  const int ty = tid >> 4, tx = tid & 15;     // rows ty*4 .. +3, columns tx*4 .. +3
  const float* Xb = (second ? p1.X : p0.X) + (size_t)b * M * K;
  const float* Yb = (second ? p1.Y : p0.Y) + (size_t)yb * N * K;
  const int xr = tid >> 2, xk = (tid & 3) * 4;   // this thread's X element group of a slab
  float4 px, py[2];
  auto fetch = [&](int k0) {
    px = m0 + xr < M ? *reinterpret_cast<const float4*>(Xb + (size_t)(m0 + xr) * K + k0 + xk)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int t = tid + u * 128;
      const int kk = t >> 4, nq4 = (t & 15) * 4;
      py[u] = n0 + nq4 < N ? *reinterpret_cast<const float4*>(Yb + (size_t)(k0 + kk) * N + n0 + nq4)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  fetch(0);
  for (int k0 = 0, buf = 0; k0 < K; k0 += 16, buf ^= 1) {
    // X slab -> Xs[k][m], Y slab -> Ys[k][n]
    Xs[buf][xk][xr] = px.x; Xs[buf][xk + 1][xr] = px.y; Xs[buf][xk + 2][xr] = px.z; Xs[buf][xk + 3][xr] = px.w;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int t = tid + u * 128;
      const int kk = t >> 4, nq4 = (t & 15) * 4;
      *reinterpret_cast<float4*>(&Ys[buf][kk][nq4]) = py[u];
    }
    __syncthreads();   // this slab is staged; every thread is done with the slab two steps back
    if (k0 + 16 < K) fetch(k0 + 16);
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      const float4 a = *reinterpret_cast<const float4*>(&Xs[buf][kk][ty * 4]);
      const float4 bq = *reinterpret_cast<const float4*>(&Ys[buf][kk][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {bq.x, bq.y, bq.z, bq.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
  }
  const float div = second ? p1.div : p0.div;
  float* Cb = (second ? p1.C : p0.C) + (size_t)b * M * N;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n < N) Cb[(size_t)m * N + n] = div == 1.f ? acc[i][j] : __fdiv_rn(acc[i][j], div);
    }
  }
}

// Router logits s = A Bk^T / div for one head's 32 query blocks x 64 key blocks
// per CTA, with the whole K = d extent staged once: rows of A and Bk are copied
// 16 bytes at a time (cp.async, no register staging) into rows padded to d + 4
// floats, then one barrier, then d sequential fp32 FMAs per output (the same
// order as gemm_f32_kernel, so the logits are bit-identical). 128 threads, 4 x 4
// outputs each: query rows ty*4 .. +3, key rows tx + 16 j (so that a warp's key
// reads spread over the banks).
template <int D>
__global__ void __launch_bounds__(128) logits_fullk_kernel(const float* __restrict__ A, const float* __restrict__ Bk,
                                                           float* __restrict__ C, int M, int N, float div) {
  constexpr int LD = D + 4;   // padded row length (floats); rows stay 16-byte aligned
  static_assert((LD * 4) % 16 == 0 && 96 * LD * 4 <= 232448, "cp.async row alignment, shared memory");
  extern __shared__ __align__(16) float lg_smem[];
  float* As = lg_smem;             // [32][LD]
  float* Bs = lg_smem + 32 * LD;   // [64][LD]
  const int b = blockIdx.z, m0 = blockIdx.y * 32, n0 = blockIdx.x * 64, tid = threadIdx.x;
  const float* Ab = A + ((size_t)b * M) * D;
  const float* Bb = Bk + ((size_t)b * N) * D;
  constexpr int CPR = D / 4;   // 16-byte pieces per row
  for (int p = tid; p < 32 * CPR; p += 128) {
    const int r = p / CPR, q = p % CPR;
    float* dst = As + r * LD + q * 4;
    if (m0 + r < M)
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)),
                   "l"(Ab + (size_t)(m0 + r) * D + q * 4) : "memory");
    else
      *reinterpret_cast<float4*>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int p = tid; p < 64 * CPR; p += 128) {
    const int r = p / CPR, q = p % CPR;
    float* dst = Bs + r * LD + q * 4;
    if (n0 + r < N)
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)),
                   "l"(Bb + (size_t)(n0 + r) * D + q * 4) : "memory");
    else
      *reinterpret_cast<float4*>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();
  const int ty = tid >> 4, tx = tid & 15;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 4
  for (int k = 0; k < D; k += 4) {
    float4 a[4], bq[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = *reinterpret_cast<const float4*>(As + (ty * 4 + i) * LD + k);
#pragma unroll
    for (int j = 0; j < 4; ++j) bq[j] = *reinterpret_cast<const float4*>(Bs + (tx + 16 * j) * LD + k);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        acc[i][j] = fmaf(a[i].x, bq[j].x, acc[i][j]);
        acc[i][j] = fmaf(a[i].y, bq[j].y, acc[i][j]);
        acc[i][j] = fmaf(a[i].z, bq[j].z, acc[i][j]);
        acc[i][j] = fmaf(a[i].w, bq[j].w, acc[i][j]);
      }
  }
  float* Cb = C + (size_t)b * M * N;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx + 16 * j;
      if (n < N) Cb[(size_t)m * N + n] = __fdiv_rn(acc[i][j], div);
    }
  }
}

constexpr int TOPK_WARPS = 4;         // one warp per query-block row
constexpr int TOPK_MAX_NK = 6144;     // a row's order keys stay in shared memory

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (f == 0.f) u = 0u;                // +0 and -0 tie, as in exact arithmetic
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Hard top-k of one logit row per warp: the k-th largest order key by a
// bitwise search from the top bit down, then an ascending ballot compaction
// that keeps every key above it and the lowest-indexed keys equal to it.
__global__ void __launch_bounds__(TOPK_WARPS * 32) topk_kernel(const float* __restrict__ scores, int rows, int nk,
                                                               int k, uint8_t* __restrict__ mask,
                                                               int32_t* __restrict__ idx, uint16_t* __restrict__ mask16,
                                                               int nk8) {
  extern __shared__ uint32_t keys_all[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * TOPK_WARPS + warp;
  if (row >= rows) return;
  uint32_t* keys = keys_all + (size_t)warp * nk;
  const float* s = scores + (size_t)row * nk;
  for (int j = lane; j < nk; j += 32) keys[j] = order_key(s[j]);
  __syncwarp();
  uint32_t T = 0u;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    int cnt = 0;
    for (int j = lane; j < nk; j += 32) cnt += keys[j] >= cand;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (cnt >= k) T = cand;
  }
  int gt = 0;
  for (int j = lane; j < nk; j += 32) gt += keys[j] > T;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) gt += __shfl_xor_sync(0xffffffffu, gt, o);
  const int need = k - gt;          // entries equal to T that are kept (lowest indices first)
  const uint32_t lt = (1u << lane) - 1u;
  int eq_seen = 0, pos = 0;
  for (int jb = 0; jb < nk; jb += 32) {
    const int j = jb + lane;
    const bool in = j < nk;
    const uint32_t key = in ? keys[j] : 0u;
    const bool is_gt = in && key > T;
    const bool is_eq = in && key == T;
    const uint32_t eqm = __ballot_sync(0xffffffffu, is_eq);
    const bool sel = is_gt || (is_eq && (eq_seen + __popc(eqm & lt)) < need);
    eq_seen += __popc(eqm);
    const uint32_t selm = __ballot_sync(0xffffffffu, sel);
    if (in) mask[(size_t)row * nk + j] = sel ? 1 : 0;
    if (mask16 && j < nk8) mask16[(size_t)row * nk8 + j] = sel ? 0x3C00u : 0u;   // fp16 1 / 0, zero padding
    if (sel) idx[(size_t)row * k + pos + __popc(selm & lt)] = j;
    pos += __popc(selm);
  }
}

// The same hard Top-k with the row held in registers (NPL keys per lane, row
// lengths up to 32 NPL): one compare per key and one warp reduction per bit.
template <int NPL>
__global__ void __launch_bounds__(TOPK_WARPS * 32, 1) topk_reg_kernel(const float* __restrict__ scores, int rows, int nk,
                                                                   int k, uint8_t* __restrict__ mask,
                                                                   int32_t* __restrict__ idx,
                                                                   uint16_t* __restrict__ mask16, int nk8) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * TOPK_WARPS + warp;
  if (row >= rows) return;
  const float* s = scores + (size_t)row * nk;
  uint32_t key[NPL];
#pragma unroll
  for (int u = 0; u < NPL; ++u) {
    const int j = u * 32 + lane;
    key[u] = j < nk ? order_key(s[j]) : 0u;      // padding keys sit below every real key
  }
  uint32_t T = 0u;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    uint32_t c4[4] = {0u, 0u, 0u, 0u};   // four short count chains instead of one long one
#pragma unroll
    for (int u = 0; u < NPL; ++u) c4[u & 3] += key[u] >= cand;
    if ((int)__reduce_add_sync(0xffffffffu, (c4[0] + c4[1]) + (c4[2] + c4[3])) >= k) T = cand;
  }
  uint32_t gtc = 0;
#pragma unroll
  for (int u = 0; u < NPL; ++u) gtc += key[u] > T;
  const int need = k - (int)__reduce_add_sync(0xffffffffu, gtc);   // keys equal to T that are kept
  const uint32_t lt = (1u << lane) - 1u;
  int eq_seen = 0, pos = 0;
#pragma unroll
  for (int u = 0; u < NPL; ++u) {
    const int j = u * 32 + lane;
    const bool in = j < nk;
    const bool is_gt = in && key[u] > T;
    const bool is_eq = in && key[u] == T;
    const uint32_t eqm = __ballot_sync(0xffffffffu, is_eq);
    const bool sel = is_gt || (is_eq && (eq_seen + __popc(eqm & lt)) < need);
    eq_seen += __popc(eqm);
    const uint32_t selm = __ballot_sync(0xffffffffu, sel);
    if (in) mask[(size_t)row * nk + j] = sel ? 1 : 0;
    if (mask16 && j < nk8) mask16[(size_t)row * nk8 + j] = sel ? 0x3C00u : 0u;   // fp16 1 / 0, zero padding
    if (sel) idx[(size_t)row * k + pos + __popc(selm & lt)] = j;
    pos += __popc(selm);
  }
}

// SoftTop-k of one logit row per warp (SLA2 detail page §4, Eq. 17): P_c = row
// softmax of the logits, m_j = sigmoid(P_c[j] / tau + lambda) with lambda found
// by bisection on [logit(k / nk) - 1 / tau, logit(k / nk)] so that the row sums
// to k. x = P_c / tau is kept in shared memory for the bisection passes.
constexpr int SOFT_ITERS = 48;        // halvings of a bracket 1 / tau wide: below fp32 resolution

__global__ void __launch_bounds__(TOPK_WARPS * 32) soft_topk_kernel(const float* __restrict__ scores, int rows,
                                                                    int nk, int k, float tau,
                                                                    float* __restrict__ soft,
                                                                    float* __restrict__ lam_out) {
  extern __shared__ float xs_all[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * TOPK_WARPS + warp;
  if (row >= rows) return;
  float* xs = xs_all + (size_t)warp * nk;
  const float* srow = scores + (size_t)row * nk;
  float* out = soft + (size_t)row * nk;
  if (k >= nk) {                      // every block kept: the relaxation is identically 1
    for (int j = lane; j < nk; j += 32) out[j] = 1.f;
    if (lam_out && lane == 0) lam_out[row] = INFINITY;
    return;
  }
  float m = -INFINITY;
  for (int j = lane; j < nk; j += 32) m = fmaxf(m, srow[j]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float sum = 0.f;
  for (int j = lane; j < nk; j += 32) {
    const float e = expf(srow[j] - m);
    xs[j] = e;
    sum += e;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float scale = 1.f / (sum * tau);          // x = P_c / tau
  for (int j = lane; j < nk; j += 32) xs[j] *= scale;
  __syncwarp();
  const float base = logf((float)k / (float)(nk - k));
  float lo = base - 1.f / tau, hi = base;
  for (int itn = 0; itn < SOFT_ITERS; ++itn) {
    const float mid = 0.5f * (lo + hi);
    float f = 0.f;
    for (int j = lane; j < nk; j += 32) f += 1.f / (1.f + expf(-(xs[j] + mid)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) f += __shfl_xor_sync(0xffffffffu, f, o);
    if (f < (float)k) lo = mid;
    else hi = mid;
  }
  const float lam = 0.5f * (lo + hi);
  for (int j = lane; j < nk; j += 32) out[j] = 1.f / (1.f + expf(-(xs[j] + lam)));
  if (lam_out && lane == 0) lam_out[row] = lam;
}

}  // namespace

cudaError_t launch_soft_topk(const Shape& s, const float* scores, float tau, float* soft, float* lam,
                             cudaStream_t st) {
  const int rows = s.BH * s.nq;
  const size_t smem = (size_t)TOPK_WARPS * s.nk * sizeof(float);
  cudaFuncSetAttribute(soft_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  soft_topk_kernel<<<(rows + TOPK_WARPS - 1) / TOPK_WARPS, TOPK_WARPS * 32, smem, st>>>(scores, rows, s.nk, s.k, tau,
                                                                                         soft, lam);
  return cudaGetLastError();
}

cudaError_t launch_pool(const Shape& s, const void* q, const void* k, const void* v, float* qbar, double* ksum,
                        int8_t* qhat, float* sq, unsigned* vamax, unsigned* status, unsigned long long budget_ns,
                        cudaStream_t st, double* csum) {
  constexpr int kSMs = 148;   // B200 streaming multiprocessors
  const int items = s.BH * s.nq;
  const int grid = items < kSMs ? items : kSMs;
  auto qb = static_cast<const __nv_bfloat16*>(q);
  auto kb = static_cast<const __nv_bfloat16*>(k);
  auto vb = static_cast<const __nv_bfloat16*>(v);
  if (s.d == 128) {
    cudaFuncSetAttribute(pool_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, PoolCfg<128>::SMEM);
    pool_kernel<128><<<grid, POOL_THREADS, PoolCfg<128>::SMEM, st>>>(qb, kb, vb, s.BH, s.N, s.nq, s.nk, qbar, ksum,
                                                                      qhat, sq, vamax, status, budget_ns, csum);
  } else {
    cudaFuncSetAttribute(pool_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, PoolCfg<64>::SMEM);
    pool_kernel<64><<<grid, POOL_THREADS, PoolCfg<64>::SMEM, st>>>(qb, kb, vb, s.BH, s.N, s.nq, s.nk, qbar, ksum,
                                                                    qhat, sq, vamax, status, budget_ns, csum);
  }
  return cudaGetLastError();
}

cudaError_t launch_colmean(const Shape& s, const double* ksum, double* c64, float* c32, float* kbar_s,
                           cudaStream_t st, const double* csum) {
  if (csum) {
    const size_t n = (size_t)s.BH * s.nk * s.d;
    kbar_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(csum, ksum, s.BH, s.nk, s.N, s.d, c64, c32, kbar_s);
  } else {
    colmean_kbar_kernel<<<dim3(s.BH, s.d / 32), 256, 0, st>>>(ksum, s.nk, s.N, s.d, c64, c32, kbar_s);
  }
  return cudaGetLastError();
}

static cudaError_t gemm(const GemmProblem& p0, const GemmProblem& p1, cudaStream_t st) {
  const int N = p0.N > p1.N ? p0.N : p1.N, M = p0.M > p1.M ? p0.M : p1.M;
  dim3 grid((N + 63) / 64, (M + 31) / 32, p0.batch + p1.batch);
  gemm_f32_kernel<<<grid, 128, 0, st>>>(p0, p1);
  return cudaGetLastError();
}

cudaError_t launch_proj(const Shape& s, int H, const float* qbar, const float* kbar_s, const float* wq,
                        const float* wk, float* A, float* Bk, cudaStream_t st) {
  const GemmProblem pq{qbar, wq, A, s.BH, s.nq, s.d, s.d, H, 1.f};
  const GemmProblem pk{kbar_s, wk, Bk, s.BH, s.nk, s.d, s.d, H, 1.f};
  return gemm(pq, pk, st);
}

cudaError_t launch_scores(const Shape& s, const float* A, const float* Bk, float* scores, cudaStream_t st) {
  const dim3 grid((s.nk + 63) / 64, (s.nq + 31) / 32, s.BH);
  const float div = sqrtf((float)s.d);
  if (s.d == 128) {
    const int smem = 96 * (128 + 4) * 4;
    cudaFuncSetAttribute(logits_fullk_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    logits_fullk_kernel<128><<<grid, 128, smem, st>>>(A, Bk, scores, s.nq, s.nk, div);
  } else {
    const int smem = 96 * (64 + 4) * 4;
    logits_fullk_kernel<64><<<grid, 128, smem, st>>>(A, Bk, scores, s.nq, s.nk, div);
  }
  return cudaGetLastError();
}

int scores_topk_max_nk() { return TOPK_MAX_NK; }

cudaError_t launch_topk(const Shape& s, const float* scores, uint8_t* mask, int32_t* idx, cudaStream_t st,
                        uint16_t* mask16) {
  const int nk8 = (s.nk + 7) & ~7;
  const int rows = s.BH * s.nq;
  const dim3 grid((rows + TOPK_WARPS - 1) / TOPK_WARPS), block(TOPK_WARPS * 32);
  if (s.nk <= 128) {
    topk_reg_kernel<4><<<grid, block, 0, st>>>(scores, rows, s.nk, s.k, mask, idx, mask16, nk8);
    return cudaGetLastError();
  }
  if (s.nk <= 256) {
    topk_reg_kernel<8><<<grid, block, 0, st>>>(scores, rows, s.nk, s.k, mask, idx, mask16, nk8);
    return cudaGetLastError();
  }
  if (s.nk <= 512) {
    topk_reg_kernel<16><<<grid, block, 0, st>>>(scores, rows, s.nk, s.k, mask, idx, mask16, nk8);
    return cudaGetLastError();
  }
  if (s.nk <= 1024) {
    topk_reg_kernel<32><<<grid, block, 0, st>>>(scores, rows, s.nk, s.k, mask, idx, mask16, nk8);
    return cudaGetLastError();
  }
  const size_t smem = (size_t)TOPK_WARPS * s.nk * sizeof(uint32_t);
  cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  topk_kernel<<<(rows + TOPK_WARPS - 1) / TOPK_WARPS, TOPK_WARPS * 32, smem, st>>>(scores, rows, s.nk, s.k, mask,
                                                                                   idx, mask16, nk8);
  return cudaGetLastError();
}

}  // namespace sla2
