// Block-sparse branch O_s (SLA2 summary page, step 2: FlashAttention over the
// M = 1 positions only, with S = dequant(Q-hat K-hat^T / sqrt(d)), P = softmax
// over the selected entries, O_s = dequant(P-hat V-hat); SLA2 detail page §7
// note 2: only the selected block pairs are computed).
//
// One CTA per (head, query block), heads outermost so a head's key blocks stay
// in L2 while its query blocks run. 192 threads in four roles:
//   warps 0-3  softmax: thread t owns query row t (= TMEM lane t); online
//              softmax with one running-max update per key block, P written
//              to shared memory as e4m3 (x448 fixed scale) or bf16, O rescaled
//              in TMEM when a row max grows, final normalisation and store.
//   warp 4     TMA producer: Q tile once, then (K_j, V_j^T) per selected j
//              into a ring of NS stages (no multicast).
//   warp 5     tcgen05 issuer: S_n = Q K_j^T into one of two TMEM buffers
//              (kind::i8 -> s32, or kind::f16 -> f32), then O += P_n V_j
//              (kind::f8f6f4 e4m3 or kind::f16 bf16 -> f32 TMEM); QK for the
//              next block is issued before PV of the current one.
// TMEM columns: [0,64) S buffer 0, [64,128) S buffer 1, [128,128+D) O.
#include <cuda_bf16.h>

#include "device.cuh"
#include "kernels.cuh"

namespace sla2 {

namespace {

template <int D, bool QUANT>
struct Cfg {
  static constexpr int ESZ = QUANT ? 1 : 2;                 // bytes per element of Q/K/V/P
  static constexpr int NS = QUANT ? 3 : 2;                  // K/V ring depth
  static constexpr int QK_ROW = D * ESZ;                    // bytes of one Q/K row
  static constexpr int QK_SW = QK_ROW >= 128 ? 128 : 64;    // swizzle span of Q/K tiles
  static constexpr int QK_PARTS = QK_ROW / QK_SW;           // 128-byte column slabs of a Q/K tile
  static constexpr int VP_ROW = BKB * ESZ;                  // bytes of one V^T / P row (64 tokens)
  static constexpr int Q_BYTES = BQ * QK_ROW;
  static constexpr int K_BYTES = BKB * QK_ROW;
  static constexpr int V_BYTES = D * VP_ROW;
  static constexpr int P_BYTES = BQ * VP_ROW;
  static constexpr int QK_STEPS = QK_ROW / 32;              // 32 bytes of K per MMA instruction
  static constexpr int PV_STEPS = VP_ROW / 32;
  static constexpr uint32_t QK_LAYOUT = QK_SW == 128 ? LAYOUT_SW128 : LAYOUT_SW64;
  static constexpr uint32_t VP_LAYOUT = VP_ROW == 128 ? LAYOUT_SW128 : LAYOUT_SW64;
  static constexpr int OFF_K = Q_BYTES;
  static constexpr int OFF_V = OFF_K + NS * K_BYTES;
  static constexpr int OFF_P = OFF_V + NS * V_BYTES;
  static constexpr int OFF_BAR = OFF_P + 2 * P_BYTES;
  // barriers: q_full, kv_full[NS], kv_empty[NS], s_full[2], s_empty[2], p_full[2], pv_done
  static constexpr int NBAR = 1 + 2 * NS + 6 + 1;
  static constexpr int OFF_SV = OFF_BAR + 8 * 16;
  static constexpr int OFF_MISC = OFF_SV + 4 * D;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;         // + alignment slack
  static constexpr uint32_t IDESC_QK = QUANT ? make_idesc(2, 1, 1, 128, 64) : make_idesc(1, 1, 1, 128, 64);
  static constexpr uint32_t IDESC_PV = QUANT ? make_idesc(1, 0, 0, 128, D) : make_idesc(1, 1, 1, 128, D);
  static constexpr uint32_t TMEM_COLS = 256;
  static constexpr uint32_t COL_O = 128;
};

// Address of the 32-byte K step `ks` inside a K-major tile made of 128-byte (or
// 64-byte) swizzled column slabs of `rows` rows each.
template <int SW>
__device__ __forceinline__ uint32_t kstep_addr(uint32_t tile, int rows, int ks) {
  const int byte = ks * 32;
  return tile + (uint32_t)((byte / SW) * rows * SW + (byte % SW));
}

constexpr uint64_t DRAIN_NS = 20000000ull;   // 20 ms for in-flight copies / MMAs after an abort

template <int D, bool QUANT>
__global__ void __launch_bounds__(192, QUANT ? 2 : 1) sparse_kernel(const __grid_constant__ CUtensorMap tq,
                                                        const __grid_constant__ CUtensorMap tk,
                                                        const __grid_constant__ CUtensorMap tv, Shape s,
                                                        SparseArgs a) {
  using C = Cfg<D, QUANT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;
  uint8_t* sK = base + C::OFF_K;
  uint8_t* sV = base + C::OFF_V;
  uint8_t* sP = base + C::OFF_P;
  uint64_t* bar = reinterpret_cast<uint64_t*>(base + C::OFF_BAR);
  uint64_t* q_full = bar;
  uint64_t* kv_full = bar + 1;
  uint64_t* kv_empty = bar + 1 + C::NS;
  uint64_t* s_full = bar + 1 + 2 * C::NS;
  uint64_t* s_empty = s_full + 2;
  uint64_t* p_full = s_full + 4;
  uint64_t* pv_done = s_full + 6;
  uint64_t* drain = s_full + 7;
  float* s_sv = reinterpret_cast<float*>(base + C::OFF_SV);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + C::OFF_MISC);
  int* abort_flag = reinterpret_cast<int*>(base + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x / s.nq, qi = blockIdx.x % s.nq;
  const int k = s.k;
  const int32_t* sel = a.idx + ((size_t)bh * s.nq + qi) * k;
  volatile int* abortf = abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int st = 0; st < C::NS; ++st) {
      mbar_init(kv_full + st, 1);
      mbar_init(kv_empty + st, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full + b, 1);
      mbar_init(s_empty + b, 128);
      mbar_init(p_full + b, 128);
    }
    mbar_init(pv_done, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (QUANT && threadIdx.x < 128) {
    for (int e = threadIdx.x; e < D; e += 128) s_sv[e] = a.sv[(size_t)bh * D + e];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tk);
      tma_prefetch_desc(&tv);
      const int qrow = bh * s.N + qi * BQ;
      mbar_arrive_expect_tx(q_full, C::Q_BYTES);
#pragma unroll
      for (int part = 0; part < C::QK_PARTS; ++part)
        tma_load_2d(sQ + part * BQ * C::QK_SW, &tq, q_full, part * (C::QK_SW / C::ESZ), qrow);
      int issued = 0;
      for (int n = 0; n < k; ++n) {
        const int st = n % C::NS;
        if (n >= C::NS && !mbar_wait(kv_empty + st, ((n / C::NS) - 1) & 1, abortf, a.status, a.budget_ns)) break;
        ++issued;
        const int j = __ldg(sel + n);
        mbar_arrive_expect_tx(kv_full + st, C::K_BYTES + C::V_BYTES);
#pragma unroll
        for (int part = 0; part < C::QK_PARTS; ++part)
          tma_load_2d(sK + st * C::K_BYTES + part * BKB * C::QK_SW, &tk, kv_full + st, part * (C::QK_SW / C::ESZ),
                      bh * s.N + j * BKB);
        tma_load_2d(sV + st * C::V_BYTES, &tv, kv_full + st, 0, (bh * s.nk + j) * D);
      }
      if (*abortf) {
        // let the copies still in flight land before the CTA's shared memory is released
        mbar_wait_drain(q_full, 0, DRAIN_NS);
        for (int n = issued > C::NS ? issued - C::NS : 0; n < issued; ++n)
          mbar_wait_drain(kv_full + n % C::NS, (n / C::NS) & 1, DRAIN_NS);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV), p_addr = smem_u32(sP);
      auto issue_qk = [&](int n) -> bool {
        const int st = n % C::NS, b = n & 1;
        if (!mbar_wait(kv_full + st, (n / C::NS) & 1, abortf, a.status, a.budget_ns)) return false;
        if (n >= 2 && !mbar_wait(s_empty + b, ((n - 2) >> 1) & 1, abortf, a.status, a.budget_ns)) return false;
        tc_fence_after();
        const uint32_t kt = k_addr + st * C::K_BYTES;
#pragma unroll
        for (int ks = 0; ks < C::QK_STEPS; ++ks) {
          const uint64_t ad = make_sdesc(kstep_addr<C::QK_SW>(q_addr, BQ, ks), 8 * C::QK_SW, C::QK_LAYOUT);
          const uint64_t bd = make_sdesc(kstep_addr<C::QK_SW>(kt, BKB, ks), 8 * C::QK_SW, C::QK_LAYOUT);
          if (QUANT)
            mma_i8(tmem + b * 64, ad, bd, C::IDESC_QK, ks > 0);
          else
            mma_f16(tmem + b * 64, ad, bd, C::IDESC_QK, ks > 0);
        }
        tc_commit(s_full + b);
        return true;
      };
      auto issue_pv = [&](int n) -> bool {
        const int st = n % C::NS, b = n & 1;
        if (!mbar_wait(p_full + b, (n >> 1) & 1, abortf, a.status, a.budget_ns)) return false;
        tc_fence_after();
        const uint32_t pt = p_addr + b * C::P_BYTES, vt = v_addr + st * C::V_BYTES;
#pragma unroll
        for (int ks = 0; ks < C::PV_STEPS; ++ks) {
          const uint64_t ad = make_sdesc(pt + ks * 32, 8 * C::VP_ROW, C::VP_LAYOUT);
          const uint64_t bd = make_sdesc(vt + ks * 32, 8 * C::VP_ROW, C::VP_LAYOUT);
          if (QUANT)
            mma_f8(tmem + C::COL_O, ad, bd, C::IDESC_PV, (n > 0 || ks > 0));
          else
            mma_f16(tmem + C::COL_O, ad, bd, C::IDESC_PV, (n > 0 || ks > 0));
        }
        tc_commit(kv_empty + st);
        tc_commit(pv_done);
        return true;
      };
      bool ok = mbar_wait(q_full, 0, abortf, a.status, a.budget_ns);
      if (ok) {
        tc_fence_after();
        ok = issue_qk(0);
      }
      for (int n = 1; ok && n < k; ++n) {
        ok = issue_qk(n);
        if (ok) ok = issue_pv(n - 1);
      }
      if (ok) ok = issue_pv(k - 1);
      if (!ok) {
        // wait for every MMA issued so far before the tensor memory is released
        tc_commit(drain);
        mbar_wait_drain(drain, 0, DRAIN_NS);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warps
    const int r = threadIdx.x;                       // query row within the block
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    constexpr float LOG2E = 1.4426950408889634f;
    const float rs_d = rsqrtf((float)D);
    const float sq_i = QUANT ? a.sq[(size_t)bh * s.nq + qi] : 1.f;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int n = 0; n < k; ++n) {
      const int b = n & 1;
      ok = mbar_wait(s_full + b, (n >> 1) & 1, abortf, a.status, a.budget_ns);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[64];
      tmem_ld32(lane_addr + b * 64, *reinterpret_cast<uint32_t(*)[32]>(sr));
      tmem_ld32(lane_addr + b * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(s_empty + b);

      float scale;   // logits in log2 units = raw * scale
      if (QUANT) {
        const int j = __ldg(sel + n);
        scale = sq_i * __ldg(a.sk + (size_t)bh * s.nk + j) * rs_d * LOG2E;
      } else {
        scale = rs_d * LOG2E;
      }
      float x[64];
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        x[c] = QUANT ? (float)(int)sr[c] : __uint_as_float(sr[c]);
        x[c] *= scale;
        mx = fmaxf(mx, x[c]);
      }
      const float m_new = fmaxf(m, mx);
      const float corr = ex2_approx(m - m_new);     // 0 on the first block
      float rowsum = 0.f;
      uint32_t pk[QUANT ? 16 : 32];
#pragma unroll
      for (int c = 0; c < 64; c += 4) {
        const float p0 = ex2_approx(x[c] - m_new), p1 = ex2_approx(x[c + 1] - m_new);
        const float p2 = ex2_approx(x[c + 2] - m_new), p3 = ex2_approx(x[c + 3] - m_new);
        rowsum += (p0 + p1) + (p2 + p3);
        if (QUANT) {
          const uint16_t lo = cvt_e4m3x2(448.f * p0, 448.f * p1);
          const uint16_t hi = cvt_e4m3x2(448.f * p2, 448.f * p3);
          pk[c / 4] = (uint32_t)lo | ((uint32_t)hi << 16);
        } else {
          pk[c / 2] = cvt_bf16x2(p0, p1);
          pk[c / 2 + 1] = cvt_bf16x2(p2, p3);
        }
      }
      l = l * corr + rowsum;
      m = m_new;
      // P buffer b was last read by PV n-2; O must be final for PV n-1 before rescaling
      if (n >= 1) {
        ok = mbar_wait(pv_done, (n - 1) & 1, abortf, a.status, a.budget_ns);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
      }
      uint8_t* prow = sP + b * C::P_BYTES + r * C::VP_ROW;
      if (QUANT) {
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const int pc = ch ^ ((r >> 1) & 3);        // 64-byte swizzle
          *reinterpret_cast<uint4*>(prow + pc * 16) = make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        }
      } else {
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const int pc = ch ^ (r & 7);               // 128-byte swizzle
          *reinterpret_cast<uint4*>(prow + pc * 16) = make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        }
      }
      if (n >= 1 && __any_sync(0xffffffffu, corr != 1.f)) {
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(lane_addr + C::COL_O + cc * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * corr);
          tmem_st32(lane_addr + C::COL_O + cc * 32, o);
        }
        tmem_wait_st();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full + b);
    }
    if (ok) {
      ok = mbar_wait(pv_done, (k - 1) & 1, abortf, a.status, a.budget_ns);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      float* orow = a.os + ((size_t)bh * s.N + (size_t)qi * BQ + r) * D;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        tmem_ld32(lane_addr + C::COL_O + cc * 32, o);
        tmem_wait_ld();
        float v[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float acc = __uint_as_float(o[c]);
          v[c] = QUANT ? acc * s_sv[cc * 32 + c] * (1.f / 448.f) * inv_l : acc * inv_l;
        }
#pragma unroll
        for (int c = 0; c < 32; c += 4)
          *reinterpret_cast<float4*>(orow + cc * 32 + c) = make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int D, bool QUANT>
cudaError_t launch_t(const Shape& s, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     const SparseArgs& a, cudaStream_t st) {
  using C = Cfg<D, QUANT>;
  auto kern = sparse_kernel<D, QUANT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<s.BH * s.nq, 192, C::SMEM, st>>>(tq, tk, tv, s, a);
  return cudaGetLastError();
}

}  // namespace

size_t sparse_smem_bytes(int d, int quant) {
  if (quant) return d == 128 ? Cfg<128, true>::SMEM : Cfg<64, true>::SMEM;
  return d == 128 ? Cfg<128, false>::SMEM : Cfg<64, false>::SMEM;
}

cudaError_t launch_sparse(const Shape& s, int quant, const CUtensorMap& tq, const CUtensorMap& tk,
                          const CUtensorMap& tv, const SparseArgs& a, cudaStream_t st) {
  if (quant) return s.d == 128 ? launch_t<128, true>(s, tq, tk, tv, a, st) : launch_t<64, true>(s, tq, tk, tv, a, st);
  return s.d == 128 ? launch_t<128, false>(s, tq, tk, tv, a, st) : launch_t<64, false>(s, tq, tk, tv, a, st);
}

}  // namespace sla2
