// Linear-branch state and the K / V quantisation pass (SLA2 summary page,
// step 3: H_j = phi(K_j)^T V_j, Z_j = rowsum(phi(K_j)^T); SLA2 detail page §7
// note 2: h_j precomputed per key block, then accumulated; step 2's low-bit K
// and V).
//
// One CTA walks a contiguous chunk of key blocks of one head (chunks sized so
// that all CTAs run in one wave at two CTAs per SM). Per key block j:
//   K_s   = fp32(K) - fp32(c)                      (K smoothing, detail §7 note 1)
//   K-hat = INT8 of K_s over the 64 x d block, s_k = amax / 127
//   V-hat^T = e4m3(V * 448 / amax_channel), channel-major [d][64]
//   phi   = softmax of each K_s row over the d features (fp32, ex2.approx)
//   z_j   = sum over the block's tokens of phi                   (fp32)
//   h_j^T = V_j^T phi_j  on the tensor core: tcgen05 kind::f16 with fp16
//           operands (V exactly, phi rounded once), fp32 accumulation in TMEM;
//           a second TMEM accumulator sums h_j^T over the chunk (partial H^T).
//           h_j^T is stored as fp32 or bf16 rows, or (forward pass) as the
//           fp16 tile -s h_j^T already in a swizzled K-major operand layout
//           (atom by atom), which the epilogue's tensor-core MMA consumes as
//           it lands.
// The staged tiles are [token][column] with 128-byte swizzle, which is the
// MN-major operand layout: the converters overwrite K with phi (fp16) and V
// with V (fp16) in place, and the MMA reads them as A = V (M = channel) and
// B = phi (N = feature), both MN-major, K = the 64 tokens.
// Roles: warps 0-7 convert (quantised copies, phi, z, fp16 operands) and read
// results back from TMEM (warps w and w + 4 share TMEM lane quadrant w % 4 and
// split the columns); warp 8 lane 0 issues the TMA loads (two stages) and the
// MMAs.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "device.cuh"
#include "kernels.cuh"

namespace sla2 {

namespace {

constexpr int LIN_CONV = 256;        // 8 converter warps
constexpr int LIN_MMA_WARP = 8;      // TMA / MMA warp
constexpr int LIN_THREADS = LIN_CONV + 32;

template <int D>
struct LinCfg {
  static constexpr int SLABS = D / 64;                 // 64-column (128-byte) slabs of a staged tile
  static constexpr int SLAB = BKB * 128;               // one slab: 64 tokens x 128 bytes
  static constexpr int KV_TILE = SLABS * SLAB;         // bytes of one staged bf16 K (or V) tile
  static constexpr int OFF_V = KV_TILE;                // V tile (then a zero slab when D = 64: M is 128)
  static constexpr int STAGE = KV_TILE + 2 * SLAB;
  static constexpr int EG = D / 8;                     // feature groups of 8 per token row
  static constexpr int TG = LIN_CONV / EG;             // token groups
  static constexpr int TPT = BKB / TG;                 // tokens per converter thread
  static constexpr int OFF_RED = 2 * STAGE;            // z partials [TG][D] + amax [2][8]
  static constexpr int OFF_H = ((OFF_RED + (TG * D + 16) * 4) + 1023) / 1024 * 1024;   // staged h_j tile
  static constexpr int H_BYTES = D * D * 2;
  static constexpr int OFF_BAR = OFF_H + H_BYTES;
  static constexpr int SMEM = OFF_BAR + 64 + 1024;
  static_assert(2 * (SMEM + 1024) <= 233472, "two CTAs per SM (228 KB, 1 KB reserved per CTA)");
  static_assert(OFF_H % 1024 == 0 && (32 * D * 2) % 16 == 0, "h staging: atom alignment, 16-byte bulk pieces");
  static constexpr uint32_t IDESC = make_idesc_mn(1, 0, 0, 128, D);   // fp16 x fp16 -> fp32, M = 128, N = D
  static constexpr uint32_t TMEM_COLS = D == 128 ? 256 : 128;
  static constexpr uint32_t COL_TOT = D;                // running partial H^T
};

__device__ __forceinline__ void unpack8(const uint4& w, float (&x)[8]) {
  x[0] = bf16_lo(w.x); x[1] = bf16_hi(w.x);
  x[2] = bf16_lo(w.y); x[3] = bf16_hi(w.y);
  x[4] = bf16_lo(w.z); x[5] = bf16_hi(w.z);
  x[6] = bf16_lo(w.w); x[7] = bf16_hi(w.w);
}

__device__ __forceinline__ uint32_t h2_bits(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// named barrier over the 256 converter threads (warps 0-7)
__device__ __forceinline__ void conv_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// Barrier over the 256 converter threads that returns, to every one of them,
// whether any of them passed `failed`, so that all take the same exit and no
// later barrier waits for a warp that has left.
__device__ __forceinline__ bool conv_sync_any(bool failed) {
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
__global__ void __launch_bounds__(LIN_THREADS, 2) linear_state_kernel(const __grid_constant__ CUtensorMap tk,
                                                                      const __grid_constant__ CUtensorMap tv,
                                                                      const float* __restrict__ c32, int N, int nk,
                                                                      LinearOut o) {
  using C = LinCfg<D>;
  extern __shared__ uint8_t lsm_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(lsm_raw) + 1023) & ~uintptr_t(1023));
  float* zred_all = reinterpret_cast<float*>(base + C::OFF_RED);     // [TG][D]
  float* ared_all = zred_all + C::TG * D;                            // [2][8]
  uint8_t* hst = base + C::OFF_H;                                    // h_j tile (h_mode 2), atom layout
  uint64_t* bar = reinterpret_cast<uint64_t*>(base + C::OFF_BAR);
  uint64_t* tma_full = bar;          // [2]
  uint64_t* conv_done = bar + 2;
  uint64_t* mma_done = bar + 3;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 4);
  int* abort_flag = reinterpret_cast<int*>(bar + 5);        // bar + 6: drain barrier
  uint64_t* rd_done = bar + 7;       // the per-block accumulator has been read

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y, chunk = blockIdx.x, G = gridDim.x;
  const int j0 = (int)((long long)chunk * nk / G), j1 = (int)((long long)(chunk + 1) * nk / G);
  const int cnt = j1 - j0;

  if (tid == 0) {
    mbar_init(tma_full, 1);
    mbar_init(tma_full + 1, 1);
    mbar_init(conv_done, LIN_CONV);
    mbar_init(mma_done, 1);
    mbar_init(bar + 6, 1);
    mbar_init(rd_done, LIN_CONV);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == LIN_MMA_WARP) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == LIN_MMA_WARP) {
    // ---------------------------------------------------------------- TMA + MMA issuer
    if (lane == 0 && cnt > 0) {
      auto load = [&](int n) {
        uint8_t* stg = base + (n & 1) * C::STAGE;
        const int row = bh * N + (j0 + n) * BKB;
        mbar_arrive_expect_tx(tma_full + (n & 1), 2 * C::KV_TILE);
#pragma unroll
        for (int sl = 0; sl < C::SLABS; ++sl) {
          tma_load_2d(stg + sl * C::SLAB, &tk, tma_full + (n & 1), sl * 64, row);
          tma_load_2d(stg + C::OFF_V + sl * C::SLAB, &tv, tma_full + (n & 1), sl * 64, row);
        }
      };
      load(0);
      if (cnt > 1) load(1);
      bool ok = true;
      for (int n = 0; n < cnt; ++n) {
        if (!mbar_wait(conv_done, n & 1, abort_flag, o.status, o.budget_ns)) { ok = false; break; }
        // the per-block accumulator is free once block n - 1 has been read out of it
        if (n >= 1 && !mbar_wait(rd_done, (n - 1) & 1, abort_flag, o.status, o.budget_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t stg = smem_u32(base + (n & 1) * C::STAGE);
#pragma unroll
        for (int ks = 0; ks < BKB / 16; ++ks) {      // 16 tokens = two 8-row groups per MMA
          const uint64_t ad = make_sdesc(stg + C::OFF_V + ks * 2048, 1024, LAYOUT_SW128, C::SLAB);
          const uint64_t bd = make_sdesc(stg + ks * 2048, 1024, LAYOUT_SW128, C::SLAB);
          mma_f16(tmem, ad, bd, C::IDESC, ks > 0);
          mma_f16(tmem + C::COL_TOT, ad, bd, C::IDESC, (n > 0 || ks > 0));
        }
        tc_commit(mma_done);
        if (n + 2 < cnt) {                           // the stage is free once the MMA has read it
          if (!mbar_wait(mma_done, n & 1, abort_flag, o.status, o.budget_ns)) { ok = false; break; }
          load(n + 2);
        }
      }
      if (!ok) {
        // let in-flight copies land and issued MMAs finish before the CTA releases its memory
        for (int n = (cnt > 2 ? cnt - 2 : 0); n < cnt; ++n) mbar_wait_drain(tma_full + (n & 1), (n >> 1) & 1, 20000000ull);
        tc_commit(bar + 6);
        mbar_wait_drain(bar + 6, 0, 20000000ull);
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- converters (256 threads)
    constexpr int EG = C::EG, TG = C::TG, TPT = C::TPT;
    const int tg = tid / EG;          // token group: tokens tg*TPT .. +TPT
    const int eg = tid % EG;          // feature / channel group: 8 columns eg*8 ..
    const int sl = eg >> 3, ch = eg & 7;
    // V is converted with another split: each warp takes 32 / TG whole channel
    // groups over all 64 tokens, so that a warp's V-hat^T stores fill whole rows
    const int tgv = lane % TG, egv = warp * (32 / TG) + lane / TG;
    const int slv = egv >> 3, chv = egv & 7;
    float cs[8], vinv[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      cs[c] = c32[(size_t)bh * D + eg * 8 + c];
      vinv[c] = 0.f;
      if (o.quant == 1) {
        const float a = __uint_as_float(o.vamax[(size_t)bh * D + egv * 8 + c]);
        vinv[c] = a > 0.f ? __fdiv_rn(448.f, a) : 0.f;
      }
    }
    if (o.quant == 1 && chunk == 0 && tid < D) {
      const float a = __uint_as_float(o.vamax[(size_t)bh * D + tid]);
      o.sv[(size_t)bh * D + tid] = a > 0.f ? __fdiv_rn(a, 448.f) : 0.f;
    }
    if (D < 128) {   // channels D..127 of the A operand are a zero slab (the MMA always has M = 128)
      for (int st = 0; st < 2; ++st)
        for (int t = tid; t < C::SLAB / 16; t += LIN_CONV)
          *reinterpret_cast<uint4*>(base + st * C::STAGE + C::OFF_V + C::KV_TILE + t * 16) = make_uint4(0u, 0u, 0u, 0u);
    }
    float hs = 1.f;                  // h_mode 2: the head's fp16 operand scale
    if (o.h_mode == 2) {
      float m = tid < D ? __uint_as_float(o.vamax[(size_t)bh * D + tid]) : 0.f;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      if (lane == 0) zred_all[warp] = m;
      conv_sync();
      float mx = zred_all[0];
#pragma unroll
      for (int w = 1; w < LIN_CONV / 32; ++w) mx = fmaxf(mx, zred_all[w]);
      hs = h_fp16_scale(mx, N);
      conv_sync();
    }
    float zp = 0.f;                  // this thread's feature (tid < D) partial of Z
    const int qd = warp & 3, hh = warp >> 2;    // TMEM lane quadrant, column half of the readouts
    const uint32_t lane_taddr = tmem + ((uint32_t)(qd * 32) << 16);
    constexpr int RC = D / 2;                   // readout columns per warp
    // h_j^T of block nn: TMEM lane c (one channel per thread) -> registers, the
    // accumulator released to the next block's MMA, then fp16 / bf16 / fp32 -> global
    auto readout = [&](int nn) -> bool {
      const int j = j0 + nn;
      const bool rok = mbar_wait(mma_done, nn & 1, abort_flag, o.status, o.budget_ns);
      if (conv_sync_any(!rok)) return false;
      tc_fence_after();
      const int c = qd * 32 + lane;
      if (qd * 32 >= D) {   // no accumulator lanes for this warp (D = 64)
        tc_fence_before();
        mbar_arrive(rd_done);
        return true;
      }
      if (o.h_mode == 2) {
        // -s h_j^T through shared memory, one 32-column chunk at a time: warps qd and qd + 4
        // own rows 32 qd .. 32 qd + 31, which form one contiguous 32 d x 2-byte piece of the
        // atom layout; lane 0 of warp qd writes that piece to global memory with one bulk copy
        const bool issuer = hh == 0 && lane == 0;
        const uint32_t piece = (uint32_t)qd * 32 * D * 2;
        if (issuer) bulk_wait_read0();      // its previous copy has read the staging rows
        named_bar_sync(2 + qd, 64);
        const float ns = -hs;
#pragma unroll
        for (int c2 = 0; c2 < RC / 32; ++c2) {
          const int cc = hh * (RC / 32) + c2;
          uint32_t r[32];
          tmem_ld32(lane_taddr + cc * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 32; q += 8)
            *reinterpret_cast<uint4*>(hst + atom_off(c, cc * 32 + q, D / 64)) = make_uint4(
                h2_bits(ns * __uint_as_float(r[q]), ns * __uint_as_float(r[q + 1])),
                h2_bits(ns * __uint_as_float(r[q + 2]), ns * __uint_as_float(r[q + 3])),
                h2_bits(ns * __uint_as_float(r[q + 4]), ns * __uint_as_float(r[q + 5])),
                h2_bits(ns * __uint_as_float(r[q + 6]), ns * __uint_as_float(r[q + 7])));
        }
        tc_fence_before();
        mbar_arrive(rd_done);               // the accumulator is free for the next block's MMA
        fence_proxy_async_smem();
        named_bar_sync(2 + qd, 64);
        if (issuer) {
          uint8_t* tile = static_cast<uint8_t*>(o.h) + ((size_t)bh * nk + j) * (size_t)(D * D * 2);
          bulk_store(tile + piece, hst + piece, 32 * D * 2);
          bulk_commit();
        }
        return true;
      }
      uint32_t rr[RC / 32][32];
#pragma unroll
      for (int c2 = 0; c2 < RC / 32; ++c2) tmem_ld32(lane_taddr + (hh * (RC / 32) + c2) * 32, rr[c2]);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(rd_done);
#pragma unroll
      for (int c2 = 0; c2 < RC / 32; ++c2) {
        const int cc = hh * (RC / 32) + c2;   // 32-column chunk of this warp's half
        const uint32_t (&r)[32] = rr[c2];
        if (o.h_mode == 1) {
          __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(o.h) + (((size_t)bh * nk + j) * D + c) * D + cc * 32;
#pragma unroll
          for (int q = 0; q < 32; q += 8)
            *reinterpret_cast<uint4*>(dst + q) = make_uint4(
                cvt_bf16x2(__uint_as_float(r[q]), __uint_as_float(r[q + 1])),
                cvt_bf16x2(__uint_as_float(r[q + 2]), __uint_as_float(r[q + 3])),
                cvt_bf16x2(__uint_as_float(r[q + 4]), __uint_as_float(r[q + 5])),
                cvt_bf16x2(__uint_as_float(r[q + 6]), __uint_as_float(r[q + 7])));
        } else {
          float* dst = static_cast<float*>(o.h) + (((size_t)bh * nk + j) * D + c) * D + cc * 32;
#pragma unroll
          for (int q = 0; q < 32; q += 4)
            *reinterpret_cast<float4*>(dst + q) = make_float4(__uint_as_float(r[q]), __uint_as_float(r[q + 1]),
                                                              __uint_as_float(r[q + 2]), __uint_as_float(r[q + 3]));
        }
      }
      return true;
    };

    bool ok = true;
    for (int n = 0; n < cnt; ++n) {
      const int j = j0 + n;
      float* zred = zred_all;
      float* ared = ared_all + (n & 1) * 8;
      ok = mbar_wait(tma_full + (n & 1), (n >> 1) & 1, abort_flag, o.status, o.budget_ns);
      if (conv_sync_any(!ok)) { ok = false; break; }
      uint8_t* sK = base + (n & 1) * C::STAGE;
      uint8_t* sV = sK + C::OFF_V;
      const size_t rowbase = (size_t)bh * N + (size_t)j * BKB;
      // ---- K: smooth, K-hat, phi
      float x[TPT][8];
      float amax = 0.f;
#pragma unroll
      for (int u = 0; u < TPT; ++u) {
        const int t = tg * TPT + u;
        const uint4 w = *reinterpret_cast<const uint4*>(sK + sl * C::SLAB + t * 128 + ((ch ^ (t & 7)) << 4));
        float kv[8];
        unpack8(w, kv);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          x[u][c] = __fsub_rn(kv[c], cs[c]);
          amax = fmaxf(amax, fabsf(x[u][c]));
        }
      }
      float ablk = INFINITY;         // the block's max |K_s| (quantised path)
      if (o.khat) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        if (lane == 0) ared[warp] = amax;
        conv_sync();
        const float a = fmaxf(fmaxf(fmaxf(ared[0], ared[1]), fmaxf(ared[2], ared[3])),
                              fmaxf(fmaxf(ared[4], ared[5]), fmaxf(ared[6], ared[7])));
        ablk = a;
        const float inv = a > 0.f ? __fdiv_rn(127.f, a) : 0.f;
        const bool magic = __float_as_uint(inv) < 0x7F800000u;   // finite (block-uniform); else the saturating path
#pragma unroll
        for (int u = 0; u < TPT; ++u) {
          uint32_t lo = 0, hi = 0;
          if (magic) {
            lo = pack_low_bytes(q8_magic(x[u][0], inv), q8_magic(x[u][1], inv), q8_magic(x[u][2], inv),
                                q8_magic(x[u][3], inv));
            hi = pack_low_bytes(q8_magic(x[u][4], inv), q8_magic(x[u][5], inv), q8_magic(x[u][6], inv),
                                q8_magic(x[u][7], inv));
          } else {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int q0 = max(-127, min(127, __float2int_rn(__fmul_rn(x[u][c], inv))));
              const int q1 = max(-127, min(127, __float2int_rn(__fmul_rn(x[u][c + 4], inv))));
              lo |= (uint32_t)(q0 & 0xFF) << (8 * c);
              hi |= (uint32_t)(q1 & 0xFF) << (8 * c);
            }
          }
          *reinterpret_cast<uint2*>(o.khat + (rowbase + tg * TPT + u) * D + eg * 8) = make_uint2(lo, hi);
        }
        if (tid == 0) o.sk[(size_t)bh * nk + j] = a > 0.f ? __fdiv_rn(a, 127.f) : 0.f;
      }
      float zc[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) zc[c] = 0.f;
      // phi is a softmax over the features, so any shift works: with the block's max |K_s|
      // (a bound on every token's max) known, exp(x - a) >= 2^-116 for a < 40 and the
      // per-token max (four shuffle levels a token) is not needed; else the token's own max
      const bool shift_blk = ablk < 40.f;   // block-uniform
#pragma unroll
      for (int u = 0; u < TPT; ++u) {
        float m = ablk;
        if (!shift_blk) {
          m = x[u][0];
#pragma unroll
          for (int c = 1; c < 8; ++c) m = fmaxf(m, x[u][c]);
#pragma unroll
          for (int off = EG / 2; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        }
        // exp(x - m) as 2^(x log2 e - m log2 e); phi is rounded to fp16 for the MMA
        const float mb = m * 1.4426950408889634f;
        float sum = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          x[u][c] = ex2_approx(fmaf(x[u][c], 1.4426950408889634f, -mb));
          sum += x[u][c];
        }
#pragma unroll
        for (int off = EG / 2; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        const float inv = __frcp_rn(sum);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          x[u][c] *= inv;          // phi
          zc[c] += x[u][c];
        }
      }
      // phi (fp16) in place over the staged K tile: the MMA's B operand
#pragma unroll
      for (int u = 0; u < TPT; ++u) {
        const int t = tg * TPT + u;
        *reinterpret_cast<uint4*>(sK + sl * C::SLAB + t * 128 + ((ch ^ (t & 7)) << 4)) =
            make_uint4(h2_bits(x[u][0], x[u][1]), h2_bits(x[u][2], x[u][3]), h2_bits(x[u][4], x[u][5]),
                       h2_bits(x[u][6], x[u][7]));
      }
      // ---- V: fp16 in place (the MMA's A operand), V-hat^T (e4m3) or the bf16 V^T copy
      float vv[TPT][8];
#pragma unroll
      for (int u = 0; u < TPT; ++u) {
        const int t = tgv * TPT + u;
        uint4* p = reinterpret_cast<uint4*>(sV + slv * C::SLAB + t * 128 + ((chv ^ (t & 7)) << 4));
        unpack8(*p, vv[u]);
        *p = make_uint4(h2_bits(vv[u][0], vv[u][1]), h2_bits(vv[u][2], vv[u][3]), h2_bits(vv[u][4], vv[u][5]),
                        h2_bits(vv[u][6], vv[u][7]));
      }
      if (o.vhatT) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const size_t orow = ((size_t)bh * nk + j) * D + egv * 8 + c;
          if (o.quant == 1) {
            uint16_t pr[TPT / 2];
#pragma unroll
            for (int u = 0; u < TPT; u += 2)
              pr[u / 2] = cvt_e4m3x2(__fmul_rn(vv[u][c], vinv[c]), __fmul_rn(vv[u + 1][c], vinv[c]));
            uint8_t* vd = static_cast<uint8_t*>(o.vhatT) + orow * BKB + tgv * TPT;
            if constexpr (TPT == 4)
              *reinterpret_cast<uint32_t*>(vd) = (uint32_t)pr[0] | ((uint32_t)pr[1] << 16);
            else
              *reinterpret_cast<uint16_t*>(vd) = pr[0];
          } else {
            __nv_bfloat16* vd = static_cast<__nv_bfloat16*>(o.vhatT) + orow * BKB + tgv * TPT;
            if constexpr (TPT == 4)
              *reinterpret_cast<uint2*>(vd) = make_uint2(cvt_bf16x2(vv[0][c], vv[1][c]), cvt_bf16x2(vv[2][c], vv[3][c]));
            else
              *reinterpret_cast<uint32_t*>(vd) = cvt_bf16x2(vv[0][c], vv[1][c]);
          }
        }
      }
      // ---- operands complete: hand them (and the staged tile) to the MMA thread
      if (!o.khat) conv_sync();   // the previous block's z partials have been summed (the quantised path synced above)
      // row tg of the z partials holds channels eg*8 .. +3 at eg*4 and eg*8+4 .. +7 at
      // D/2 + eg*4 (two conflict-free 16-byte stores)
      *reinterpret_cast<float4*>(zred + tg * D + eg * 4) = make_float4(zc[0], zc[1], zc[2], zc[3]);
      *reinterpret_cast<float4*>(zred + tg * D + D / 2 + eg * 4) = make_float4(zc[4], zc[5], zc[6], zc[7]);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(conv_done);
      conv_sync();
      if (tid < D) {
        float z = 0.f;
#pragma unroll
        for (int g = 0; g < TG; ++g) z += zred[g * D + ((tid & 4) ? D / 2 : 0) + (tid >> 3) * 4 + (tid & 3)];
        o.z[((size_t)bh * nk + j) * D + tid] = z;
        zp += z;
      }
      // ---- h_j^T of the previous block (its MMA ran while this block was converted)
      if (n >= 1 && !readout(n - 1)) {
        ok = false;
        break;
      }
    }
    if (ok && cnt >= 1) ok = readout(cnt - 1);
    // ---- chunk partials (H^T from the accumulating TMEM columns, Z)
    if (ok && qd * 32 < D) {
      const int c = qd * 32 + lane;
#pragma unroll
      for (int c2 = 0; c2 < RC / 32; ++c2) {
        const int cc = hh * (RC / 32) + c2;
        uint32_t r[32];
        tmem_ld32(lane_taddr + C::COL_TOT + cc * 32, r);
        tmem_wait_ld();
        float* dst = o.hpart + (((size_t)bh * G + chunk) * D + c) * D + cc * 32;
#pragma unroll
        for (int q = 0; q < 32; q += 4)
          *reinterpret_cast<float4*>(dst + q) = make_float4(__uint_as_float(r[q]), __uint_as_float(r[q + 1]),
                                                            __uint_as_float(r[q + 2]), __uint_as_float(r[q + 3]));
      }
    }
    if (tid < D) o.zpart[((size_t)bh * G + chunk) * D + tid] = zp;
    if (o.h_mode == 2) bulk_wait0();   // the staged tiles have reached global memory
  }
  tc_fence_before();
  __syncthreads();
  if (warp == LIN_MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// H_total^T and Z_total as fixed-order sums of the chunk partials. With vamax
// given, also the head's fp16 scale s (the same value the linear-state pass
// used for its h_j tiles) and s H_total^T as an fp16 operand image in the
// h_mode-2 layout, to which the epilogue adds the selected blocks' images.
__global__ void linear_reduce_kernel(const float* __restrict__ hpart, const float* __restrict__ zpart, int G, int D,
                                     int N, const unsigned* __restrict__ vamax, float* __restrict__ Htot,
                                     float* __restrict__ Ztot, uint16_t* __restrict__ htile,
                                     float* __restrict__ hscale, const float* __restrict__ z,
                                     uint16_t* __restrict__ z16, int nk) {
  __shared__ float red[8];
  const int bh = blockIdx.y;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  const int DD = D * D;
  float hs = 1.f;
  if (vamax) {
    float m = threadIdx.x < D ? __uint_as_float(vamax[(size_t)bh * D + threadIdx.x]) : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    float mx = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) mx = fmaxf(mx, red[w]);
    hs = h_fp16_scale(mx, N);
    if (blockIdx.x == 0 && threadIdx.x == 0 && hscale) hscale[bh] = hs;
  }
  if (e < DD) {
    // fixed summation order; the loads are independent, so batches of them are issued together
    float s = 0.f;
#pragma unroll 8
    for (int g = 0; g < G; ++g) s += __ldg(hpart + ((size_t)bh * G + g) * DD + e);
    Htot[(size_t)bh * DD + e] = s;
    if (vamax && htile) {
      const int row = e / D, col = e % D;
      const __half hv = __float2half_rn(hs * s);
      htile[(size_t)bh * DD + (atom_off(row, col, D / 64) >> 1) + (col & 7)] = *reinterpret_cast<const uint16_t*>(&hv);
    }
  }
  if (blockIdx.x == 0 && threadIdx.x < D) {
    float s = 0.f;
#pragma unroll 8
    for (int g = 0; g < G; ++g) s += __ldg(zpart + ((size_t)bh * G + g) * D + threadIdx.x);
    Ztot[(size_t)bh * D + threadIdx.x] = s;
  }
  if (z16)   // z_j as fp16, the operand of the selected-state product
    for (int x = e; x < nk * D; x += DD)
      z16[(size_t)bh * nk * D + x] = __half_as_ushort(__float2half_rn(__ldg(z + (size_t)bh * nk * D + x)));
}

constexpr int kSMs = 148;   // B200 streaming multiprocessors

}  // namespace

int linear_chunks(int BH, int nk) {
  int G = (2 * kSMs) / BH;   // one wave at two CTAs per SM
  if (G < 1) G = 1;
  if (G > nk) G = nk;
  return G;
}

cudaError_t launch_linear_state(const Shape& s, const void* k, const void* v, const float* c32, const LinearOut& o,
                                cudaStream_t st) {
  CUtensorMap tk, tv;
  const uint64_t rows = (uint64_t)s.BH * s.N;
  if (!make_tmap_2d(&tk, k, 2, s.d, rows, 64, BKB, 128) || !make_tmap_2d(&tv, v, 2, s.d, rows, 64, BKB, 128))
    return cudaErrorInvalidValue;
  dim3 grid(s.G, s.BH);
  if (s.d == 128) {
    auto kern = linear_state_kernel<128>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, LinCfg<128>::SMEM);
    kern<<<grid, LIN_THREADS, LinCfg<128>::SMEM, st>>>(tk, tv, c32, s.N, s.nk, o);
  } else {
    auto kern = linear_state_kernel<64>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, LinCfg<64>::SMEM);
    kern<<<grid, LIN_THREADS, LinCfg<64>::SMEM, st>>>(tk, tv, c32, s.N, s.nk, o);
  }
  return cudaGetLastError();
}

cudaError_t launch_linear_reduce(const Shape& s, const float* hpart, const float* zpart, const unsigned* vamax,
                                 float* Htot, float* Ztot, uint16_t* htile, float* hscale, cudaStream_t st,
                                 const float* z, uint16_t* z16) {
  const int DD = s.d * s.d;
  dim3 grid((DD + 255) / 256, s.BH);
  linear_reduce_kernel<<<grid, 256, 0, st>>>(hpart, zpart, s.G, s.d, s.N, vamax, Htot, Ztot,
                                             htile, hscale, z, z16, s.nk);
  return cudaGetLastError();
}

}  // namespace sla2
