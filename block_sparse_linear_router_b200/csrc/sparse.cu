// Block-sparse branch O_s (SLA2 summary page, step 2: FlashAttention over the
// M = 1 positions only, with S = dequant(Q-hat K-hat^T / sqrt(d)), P = softmax
// over the selected entries, O_s = dequant(P-hat V-hat); SLA2 detail page §7
// note 2: only the selected block pairs are computed).
//
// Persistent CTAs (two per SM) walk the (head, query block) items in
// head-major order, so the SMs work on neighbouring query blocks of the same
// head and the head's K/V blocks stay in L2. Each item is one 128-row query
// block and its k selected 64-token key blocks, visited in ascending order.
// Tensor memory and barriers are set up once; barrier phases run on across
// items (g counts key blocks over all items of the CTA). 192 threads:
//   warps 0-3  softmax: thread t owns query row t (= TMEM lane t); online
//              softmax with one running-max update per key block; P written
//              as e4m3 (x448 fixed scale) into TMEM, over key columns 0-15 of
//              its own S buffer, or as bf16 to shared memory; O rescaled in
//              TMEM when a row max grows; at the end of an item the row is
//              normalised and stored while the next item's S is computed (fp32
//              O_s, or on the quantised path the fp16 row O_s / s_v: a
//              weighted mean of e4m3 V-hat codes, so |.| <= 448 and the
//              epilogue applies s_v).
//   warp 4     TMA producer: per item the Q tile (double-buffered, prefetched
//              one item ahead); K_j and V_j^T of each selected j into separate
//              rings of NS stages (no multicast): a K stage is released when
//              its QK has finished, a V stage when its PV has, and V is loaded
//              one block behind K because PV runs two blocks behind QK.
//   warp 5     tcgen05 issuer, in the order PV(g-2), QK(g): O += P_g V_j
//              (kind::f8f6f4 e4m3 with P from TMEM, or kind::f16 bf16 -> f32),
//              and S_g = Q K_j^T into one of two TMEM buffers (kind::i8 -> s32,
//              or kind::f16 -> f32) as soon as that buffer's previous S has been
//              read. The tensor pipe
//              runs MMAs in issue order, so QK(g) overwrites P(g-2) only after
//              PV(g-2) has read it.
// TMEM columns: [0,64) S buffer 0, [64,128) S buffer 1, [128,128+D) O.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "device.cuh"
#include "kernels.cuh"

namespace sla2 {

namespace {

// D[tmem] (+)= A[tmem] x B[smem]^T for e4m3 operands: A (M = 128 lanes, four 8-bit K
// values per 32-bit column) read from tensor memory, B by descriptor.
__device__ __forceinline__ void mma_f8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

template <int D, bool QUANT>
struct Cfg {
  static constexpr int ESZ = QUANT ? 1 : 2;                 // bytes per element of Q/K/V/P
  static constexpr int NS = 3;                              // depth of the K ring and of the V ring
  // V(g) is loaded after K(g+1) and needs PV(g - NS) done, which the issuer
  // starts before QK(g+1): NS >= 3 keeps the issue orders free of a cycle
  static_assert(NS >= 3, "ring depth");
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
  static constexpr int OFF_K = 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + NS * K_BYTES;
  static constexpr int OFF_P = OFF_V + NS * V_BYTES;
  static constexpr int OFF_BAR = OFF_P + (QUANT ? 0 : 2 * P_BYTES);   // the INT8 path keeps P in TMEM
  // barriers: q_full[2], q_free[2], k_full[NS], k_empty[NS], v_full[NS], v_empty[NS],
  //           s_full[2], s_empty[2], p_full[2], p_free[2], o_full, o_free, drain
  static constexpr int NBAR = 4 + 4 * NS + 8 + 3;
  static_assert(NBAR <= 32, "barrier region");
  static constexpr int OFF_MISC = OFF_BAR + ((8 * NBAR + 15) / 16) * 16;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;         // + alignment slack
  static_assert(SMEM <= 232448, "dynamic shared memory per CTA (227 KB)");
  static_assert(!QUANT || 2 * (SMEM + 1024) <= 233472, "two CTAs per SM (228 KB, 1 KB reserved per CTA)");
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

__device__ __forceinline__ uint32_t h2_bits(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <int D, bool QUANT>
__global__ void __launch_bounds__(192, QUANT ? 2 : 1) sparse_kernel(const __grid_constant__ CUtensorMap tq,
                                                                    const __grid_constant__ CUtensorMap tk,
                                                                    const __grid_constant__ CUtensorMap tv, Shape s,
                                                                    SparseArgs a) {
  using C = Cfg<D, QUANT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = base + C::OFF_K;
  uint8_t* sV = base + C::OFF_V;
  uint8_t* sP = base + C::OFF_P;
  uint64_t* bar = reinterpret_cast<uint64_t*>(base + C::OFF_BAR);
  uint64_t* q_full = bar;                     // [2]
  uint64_t* q_free = bar + 2;                 // [2]
  uint64_t* k_full = bar + 4;                 // [NS]
  uint64_t* k_empty = k_full + C::NS;         // [NS]
  uint64_t* v_full = k_empty + C::NS;         // [NS]
  uint64_t* v_empty = v_full + C::NS;         // [NS]
  uint64_t* s_full = v_empty + C::NS;         // [2]
  uint64_t* s_empty = s_full + 2;             // [2]
  uint64_t* p_full = s_full + 4;              // [2]
  uint64_t* p_free = s_full + 6;              // [2]: the PV reading P buffer b has finished
  uint64_t* o_full = s_full + 8;              // the last PV of an item has finished
  uint64_t* o_free = s_full + 9;              // the softmax warps have read O of the item
  uint64_t* drain = s_full + 10;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + C::OFF_MISC);
  int* abort_flag = reinterpret_cast<int*>(base + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k = s.k;
  const int total = s.BH * s.nq;
  const int nitems = total > (int)blockIdx.x ? (total - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
  const int nblocks = nitems * k;             // key blocks over all of this CTA's items
  volatile int* abortf = abort_flag;
  auto item_of = [&](int it) { return (int)blockIdx.x + it * (int)gridDim.x; };

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(q_full + b, 1);
      mbar_init(q_free + b, 1);
      mbar_init(s_full + b, 1);
      mbar_init(s_empty + b, 4);     // one arrival per softmax warp
      mbar_init(p_full + b, 4);
      mbar_init(p_free + b, 1);
    }
    for (int st = 0; st < C::NS; ++st) {
      mbar_init(k_full + st, 1);
      mbar_init(k_empty + st, 1);
      mbar_init(v_full + st, 1);
      mbar_init(v_empty + st, 1);
    }
    mbar_init(o_full, 1);
    mbar_init(o_free, 4);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && nitems > 0) {
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tk);
      tma_prefetch_desc(&tv);
      int g = 0, qissued = 0;
      bool ok = true;
      auto load_q = [&](int it) -> bool {
        const int b = it & 1;
        if (it >= 2 && !mbar_wait(q_free + b, ((it >> 1) - 1) & 1, abortf, a.status, a.budget_ns)) return false;
        const int w = item_of(it);
        const int bh = w / s.nq, qi = w % s.nq;
        mbar_arrive_expect_tx(q_full + b, C::Q_BYTES);
#pragma unroll
        for (int part = 0; part < C::QK_PARTS; ++part)
          tma_load_2d(base + b * C::Q_BYTES + part * BQ * C::QK_SW, &tq, q_full + b, part * (C::QK_SW / C::ESZ),
                      bh * s.N + qi * BQ);
        ++qissued;
        return true;
      };
      ok = load_q(0);
      int gv = 0;                            // V blocks issued (V trails K by one block)
      int bh_prev = 0, j_prev = 0;
      auto load_v = [&](int bh, int j) -> bool {
        const int st = gv % C::NS;
        if (gv >= C::NS && !mbar_wait(v_empty + st, ((gv / C::NS) - 1) & 1, abortf, a.status, a.budget_ns)) return false;
        mbar_arrive_expect_tx(v_full + st, C::V_BYTES);
        tma_load_2d(sV + st * C::V_BYTES, &tv, v_full + st, 0, (bh * s.nk + j) * D);
        ++gv;
        return true;
      };
      for (int it = 0; ok && it < nitems; ++it) {
        const int w = item_of(it);
        const int bh = w / s.nq, qi = w % s.nq;
        const int32_t* sel = a.idx + ((size_t)bh * s.nq + qi) * k;
        int j_next = __ldg(sel);
        for (int n = 0; n < k; ++n) {
          const int st = g % C::NS;
          const int j = j_next;
          if (n + 1 < k) j_next = __ldg(sel + n + 1);
          if (g >= C::NS && !mbar_wait(k_empty + st, ((g / C::NS) - 1) & 1, abortf, a.status, a.budget_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(k_full + st, C::K_BYTES);
#pragma unroll
          for (int part = 0; part < C::QK_PARTS; ++part)
            tma_load_2d(sK + st * C::K_BYTES + part * BKB * C::QK_SW, &tk, k_full + st,
                        part * (C::QK_SW / C::ESZ), bh * s.N + j * BKB);
          ++g;
          if (g >= 2 && !load_v(bh_prev, j_prev)) {
            ok = false;
            break;
          }
          bh_prev = bh;
          j_prev = j;
          // prefetch the next item's Q once this item's first K block is on its way
          if (n == 0 && it + 1 < nitems && !load_q(it + 1)) {
            ok = false;
            break;
          }
        }
      }
      if (ok && g > 0) ok = load_v(bh_prev, j_prev);
      if (!ok) {   // let the copies still in flight land before shared memory is released
        for (int q = (g > C::NS ? g - C::NS : 0); q < g; ++q)
          mbar_wait_drain(k_full + q % C::NS, (q / C::NS) & 1, DRAIN_NS);
        for (int q = (gv > C::NS ? gv - C::NS : 0); q < gv; ++q)
          mbar_wait_drain(v_full + q % C::NS, (q / C::NS) & 1, DRAIN_NS);
        for (int q = (qissued > 2 ? qissued - 2 : 0); q < qissued; ++q)
          mbar_wait_drain(q_full + (q & 1), (q >> 1) & 1, DRAIN_NS);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && nitems > 0) {
      const uint32_t k_addr = smem_u32(sK), v_addr = smem_u32(sV), p_addr = smem_u32(sP);
      auto issue_qk = [&](int g) -> bool {
        const int it = g / k, n = g - it * k;
        const int st = g % C::NS, b = g & 1, qb = it & 1;
        if (n == 0 && !mbar_wait(q_full + qb, (it >> 1) & 1, abortf, a.status, a.budget_ns)) return false;
        if (!mbar_wait(k_full + st, (g / C::NS) & 1, abortf, a.status, a.budget_ns)) return false;
        if (g >= 2 && !mbar_wait(s_empty + b, ((g >> 1) - 1) & 1, abortf, a.status, a.budget_ns)) return false;
        tc_fence_after();
        const uint32_t qt = smem_u32(base + qb * C::Q_BYTES), kt = k_addr + st * C::K_BYTES;
#pragma unroll
        for (int ks = 0; ks < C::QK_STEPS; ++ks) {
          const uint64_t ad = make_sdesc(kstep_addr<C::QK_SW>(qt, BQ, ks), 8 * C::QK_SW, C::QK_LAYOUT);
          const uint64_t bd = make_sdesc(kstep_addr<C::QK_SW>(kt, BKB, ks), 8 * C::QK_SW, C::QK_LAYOUT);
          if (QUANT)
            mma_i8(tmem + b * 64, ad, bd, C::IDESC_QK, ks > 0);
          else
            mma_f16(tmem + b * 64, ad, bd, C::IDESC_QK, ks > 0);
        }
        tc_commit(s_full + b);
        tc_commit(k_empty + st);
        if (n == k - 1) tc_commit(q_free + qb);      // the item's Q tile has been read
        return true;
      };
      auto issue_pv = [&](int g) -> bool {
        const int it = g / k, n = g - it * k;
        const int st = g % C::NS, b = g & 1;
        if (!mbar_wait(v_full + st, (g / C::NS) & 1, abortf, a.status, a.budget_ns)) return false;
        if (!mbar_wait(p_full + b, (g >> 1) & 1, abortf, a.status, a.budget_ns)) return false;
        // the first PV of an item overwrites O: the previous item's O must have been read
        if (n == 0 && it > 0 && !mbar_wait(o_free, (it - 1) & 1, abortf, a.status, a.budget_ns)) return false;
        tc_fence_after();
        const uint32_t pt = p_addr + b * C::P_BYTES, vt = v_addr + st * C::V_BYTES;
#pragma unroll
        for (int ks = 0; ks < C::PV_STEPS; ++ks) {
          const uint64_t bd = make_sdesc(vt + ks * 32, 8 * C::VP_ROW, C::VP_LAYOUT);
          if (QUANT)   // P(g) in TMEM columns b*64 .. +15, 8 columns per 32-value K step
            mma_f8_ts(tmem + C::COL_O, tmem + b * 64 + ks * 8, bd, C::IDESC_PV, (n > 0 || ks > 0));
          else
            mma_f16(tmem + C::COL_O, make_sdesc(pt + ks * 32, 8 * C::VP_ROW, C::VP_LAYOUT), bd, C::IDESC_PV,
                    (n > 0 || ks > 0));
        }
        tc_commit(v_empty + st);
        tc_commit(p_free + b);
        if (n == k - 1) tc_commit(o_full);
        return true;
      };
      bool ok = true;
      // PV(g - 2) goes into the tensor pipe ahead of QK(g): on the INT8 path QK(g) overwrites
      // the TMEM columns that hold P(g - 2), and the pipe runs MMAs in issue order
      for (int g = 0; ok && g < nblocks + 2; ++g) {
        if (g >= 2) ok = issue_pv(g - 2);
        if (ok && g < nblocks) ok = issue_qk(g);
      }
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
    bool ok = true;
    int g = 0;
    for (int it = 0; ok && it < nitems; ++it) {
      const int w = item_of(it);
      const int bh = w / s.nq, qi = w % s.nq;
      const int32_t* sel = a.idx + ((size_t)bh * s.nq + qi) * k;
      const float sq_i = QUANT ? __ldg(a.sq + (size_t)bh * s.nq + qi) : 1.f;
      float m = -INFINITY, l = 0.f;
      // K-block scales prefetched two blocks ahead (their loads depend on the index list)
      const float* skh = a.sk + (size_t)bh * s.nk;
      float sk_cur = QUANT ? __ldg(skh + __ldg(sel)) : 1.f;
      float sk_nxt = (QUANT && k > 1) ? __ldg(skh + __ldg(sel + 1)) : 1.f;
      for (int n = 0; n < k; ++n, ++g) {
        const int b = g & 1;
        const int j2 = (QUANT && n + 2 < k) ? __ldg(sel + n + 2) : 0;
        ok = mbar_wait(s_full + b, (g >> 1) & 1, abortf, a.status, a.budget_ns);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[64];
        tmem_ld32(lane_addr + b * 64, *reinterpret_cast<uint32_t(*)[32]>(sr));
        tmem_ld32(lane_addr + b * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_empty + b);

        // logits in log2 units = raw * scale
        const float scale = QUANT ? sq_i * sk_cur * rs_d * LOG2E : rs_d * LOG2E;
        if (QUANT) {
          sk_cur = sk_nxt;
          sk_nxt = n + 2 < k ? __ldg(skh + j2) : 1.f;
        }
        // Raw logits as fp32 pairs. For INT8 the s32 accumulator plus 0x4B400000 is
        // the bit pattern of 12582912 + S exactly (|S| < 2^22); subtracting
        // 12582912 is exact too, so S becomes a float without an int->float
        // conversion. (Presetting the accumulator to 0x4B400000 would save the adds,
        // but key columns 0-15 hold P(g - 2) until QK(g) overwrites them.)
        uint64_t f2[32];
        const uint64_t off2 = f2_pack(-12582912.f, -12582912.f);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          if (QUANT)
            f2[c] = f2_add(f2_pack(__uint_as_float(sr[2 * c] + 0x4B400000u), __uint_as_float(sr[2 * c + 1] + 0x4B400000u)),
                           off2);
          else
            f2[c] = f2_pack(__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1]));
        }
        float mx8[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float x0, x1, y0, y1;
          f2_unpack(f2[c], x0, x1);
          f2_unpack(f2[c + 8], y0, y1);
          mx8[c] = fmax3(x0, x1, fmaxf(y0, y1));
        }
#pragma unroll
        for (int c = 16; c < 32; c += 2) {
          float x0, x1, y0, y1;
          f2_unpack(f2[c], x0, x1);
          f2_unpack(f2[c + 1], y0, y1);
          const int q = (c - 16) >> 1;
          mx8[q] = fmax3(mx8[q], x0, fmax3(x1, y0, y1));
        }
        const float mxf = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
        const float m_new = fmaxf(m, mxf * scale);
        const float corr = ex2_approx(m - m_new);     // 0 on the first block
        // exponent of p = fma(S, scale, c2); the quantised path yields 448 p directly
        const float c2 = QUANT ? 8.807354922057604f - m_new : -m_new;
        const uint64_t sc2 = f2_pack(scale, scale), cc2 = f2_pack(c2, c2);
        uint64_t rs2a = f2_pack(0.f, 0.f), rs2b = f2_pack(0.f, 0.f);
        uint32_t pk[QUANT ? 16 : 32];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          float t0, t1, t2, t3;
          f2_unpack(f2_fma(f2[c], sc2, cc2), t0, t1);
          f2_unpack(f2_fma(f2[c + 1], sc2, cc2), t2, t3);
          const float p0 = ex2_approx(t0), p1 = ex2_approx(t1), p2 = ex2_approx(t2), p3 = ex2_approx(t3);
          rs2a = f2_add(rs2a, f2_pack(p0, p1));
          rs2b = f2_add(rs2b, f2_pack(p2, p3));
          if (QUANT) {
            const uint16_t lo = cvt_e4m3x2(p0, p1);
            const uint16_t hi = cvt_e4m3x2(p2, p3);
            pk[c / 2] = (uint32_t)lo | ((uint32_t)hi << 16);
          } else {
            pk[c] = cvt_bf16x2(p0, p1);
            pk[c + 1] = cvt_bf16x2(p2, p3);
          }
        }
        float ra0, ra1;
        f2_unpack(f2_add(rs2a, rs2b), ra0, ra1);
        l = l * corr + (ra0 + ra1);
        m = m_new;
        // P buffer b was last read by PV g-2 (on the INT8 path QK(g) has already followed
        // PV(g-2) in the tensor pipe; the wait keeps this warp's view of the p_free phases
        // in step for the rescale's wait below)
        if (g >= 2) {
          ok = mbar_wait(p_free + b, ((g >> 1) - 1) & 1, abortf, a.status, a.budget_ns);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        }
        if (QUANT) {
          // e4m3 P(g) into key columns 0-15 of its own S buffer (S(g) is in registers), four
          // values per column: the A operand of PV(g)
          tmem_st16(lane_addr + b * 64, *reinterpret_cast<uint32_t(*)[16]>(pk));
        } else {
          uint8_t* prow = sP + b * C::P_BYTES + r * C::VP_ROW;
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const int pc = ch ^ (r & 7);               // 128-byte swizzle
            *reinterpret_cast<uint4*>(prow + pc * 16) =
                make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
          }
        }
        if (!QUANT) fence_proxy_async_smem();
        // O must be rescaled by corr (after PV n-1 has finished) before PV n adds to it;
        // P is already stored, so its write and proxy fence overlap this wait
        if (n >= 1 && __any_sync(0xffffffffu, corr != 1.f)) {
          ok = mbar_wait(p_free + ((g - 1) & 1), ((g - 1) >> 1) & 1, abortf, a.status, a.budget_ns);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          tc_fence_after();
          uint32_t o0[32], o1[32], o2[32], o3[32];
          tmem_ld32(lane_addr + C::COL_O, o0);
          if (D > 32) tmem_ld32(lane_addr + C::COL_O + 32, o1);
          if (D > 64) {
            tmem_ld32(lane_addr + C::COL_O + 64, o2);
            tmem_ld32(lane_addr + C::COL_O + 96, o3);
          }
          tmem_wait_ld();
          const uint64_t corr2 = f2_pack(corr, corr);
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            float x0, x1;
            f2_unpack(f2_mul(f2_pack(__uint_as_float(o0[c]), __uint_as_float(o0[c + 1])), corr2), x0, x1);
            o0[c] = __float_as_uint(x0);
            o0[c + 1] = __float_as_uint(x1);
            if (D > 32) {
              f2_unpack(f2_mul(f2_pack(__uint_as_float(o1[c]), __uint_as_float(o1[c + 1])), corr2), x0, x1);
              o1[c] = __float_as_uint(x0);
              o1[c + 1] = __float_as_uint(x1);
            }
            if (D > 64) {
              f2_unpack(f2_mul(f2_pack(__uint_as_float(o2[c]), __uint_as_float(o2[c + 1])), corr2), x0, x1);
              o2[c] = __float_as_uint(x0);
              o2[c + 1] = __float_as_uint(x1);
              f2_unpack(f2_mul(f2_pack(__uint_as_float(o3[c]), __uint_as_float(o3[c + 1])), corr2), x0, x1);
              o3[c] = __float_as_uint(x0);
              o3[c + 1] = __float_as_uint(x1);
            }
          }
          tmem_st32(lane_addr + C::COL_O, o0);
          if (D > 32) tmem_st32(lane_addr + C::COL_O + 32, o1);
          if (D > 64) {
            tmem_st32(lane_addr + C::COL_O + 64, o2);
            tmem_st32(lane_addr + C::COL_O + 96, o3);
          }
          tmem_wait_st();
        }
        if (QUANT) tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full + b);     // P written and O rescaled
      }
      if (!ok) break;
      // ---- item done: normalise O and store it, then hand O back to the MMA issuer
      ok = mbar_wait(o_full, it & 1, abortf, a.status, a.budget_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const float inv_l = 1.f / l;     // quantised path: l holds 448 x the row sum
      const size_t orow = ((size_t)bh * s.N + (size_t)qi * BQ + r) * D;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        tmem_ld32(lane_addr + C::COL_O + cc * 32, o);
        tmem_wait_ld();
        if constexpr (QUANT) {
          // O_s / s_v = acc / l: a weighted mean of V-hat codes, |.| <= 448, stored as fp16
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__half*>(a.os) + orow + cc * 32);
#pragma unroll
          for (int c = 0; c < 32; c += 8)
            dst[c / 8] = make_uint4(
                h2_bits(__uint_as_float(o[c]) * inv_l, __uint_as_float(o[c + 1]) * inv_l),
                h2_bits(__uint_as_float(o[c + 2]) * inv_l, __uint_as_float(o[c + 3]) * inv_l),
                h2_bits(__uint_as_float(o[c + 4]) * inv_l, __uint_as_float(o[c + 5]) * inv_l),
                h2_bits(__uint_as_float(o[c + 6]) * inv_l, __uint_as_float(o[c + 7]) * inv_l));
        } else {
          float* dst = static_cast<float*>(a.os) + orow + cc * 32;
#pragma unroll
          for (int c = 0; c < 32; c += 4)
            *reinterpret_cast<float4*>(dst + c) =
                make_float4(__uint_as_float(o[c]) * inv_l, __uint_as_float(o[c + 1]) * inv_l,
                            __uint_as_float(o[c + 2]) * inv_l, __uint_as_float(o[c + 3]) * inv_l);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_free);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

constexpr int kSMs = 148;   // B200 streaming multiprocessors

template <int D, bool QUANT>
cudaError_t launch_t(const Shape& s, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     const SparseArgs& a, cudaStream_t st) {
  using C = Cfg<D, QUANT>;
  auto kern = sparse_kernel<D, QUANT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int total = s.BH * s.nq;
  const int per_sm = QUANT ? 2 : 1;
  const int grid = total < per_sm * kSMs ? total : per_sm * kSMs;
  kern<<<grid, 192, C::SMEM, st>>>(tq, tk, tv, s, a);
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
