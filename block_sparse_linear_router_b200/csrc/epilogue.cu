// Linear branch apply + mix (SLA2 summary page, steps 3 and 4; SLA2 detail
// page §7 note 2: per-key-block h_j precomputed, then accumulated):
//   H_i = H_total - sum_{j selected} h_j,   Z_i = Z_total - sum_{j selected} z_j
//   O_l = phi(Q_i) H_i / (phi(Q_i) Z_i)      (phi: softmax over the d features)
//   O   = alpha_i O_s + (1 - alpha_i) O_l
// When every key block is selected there is no unselected block and O_l := 0.
//
// H_i is formed per query block on the CUDA cores: the linear-state pass
// stored each -s h_j^T, and the reduce pass s H_total^T, as fp16 d x d images
// already in the 128-byte-swizzled K-major operand layout, so eight "sum"
// warps add the k + 1 images element by element in fp32 (each thread owns the
// same 16-byte chunks of every image: coalesced L2 reads, no shared-memory
// traffic for the gather) and write s H_i^T, rounded once to fp16, as the B
// operand of ONE tensor-core product D = phi(Q_i) (s H_i) per query block. s is
// a per-head power of two that keeps s H_total inside the fp16 range. The
// sum warps also form Z_i = Z_total - sum_sel z_j. The denominator
// phi(Q_i) Z_i is a d-term fp32 dot product per query row, taken while phi is
// computed; s cancels in O_l = D / (s den), and so does phi's normalisation
// (the operand is exp(q - rowmax) without the row sum).
//
// Persistent CTAs (one per SM, 16 warps) walk the (head, query block) items in
// head-major order, so the SMs work on neighbouring query blocks of the same
// head and the head's h_j images stay in L2. Per CTA:
//   warps 8-15 sum: per item, Z_i and s H_i^T (fp16 image) into one of two
//              shared buffers (the one the MMA of the item before last read);
//   warps 0-7  per item: exp(Q_i - rowmax), one query row per thread and half
//              of the features per warp (the two halves exchange their row
//              max), stored as fp16 into one of two TMEM A buffers, and the
//              denominators; then thread 0 issues the item's d / 16 tcgen05
//              kind::f16 MMAs (A from TMEM, B = the s H_i^T image) into one of
//              two TMEM accumulators and commits; while they run, the warps
//              read out the previous item: 16 accumulator columns at a time,
//              O_l = D / (s den), the alpha mix with O_s and the store.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "device.cuh"
#include "kernels.cuh"

namespace sla2 {

namespace {

constexpr int EPI_COMPUTE = 256;          // warps 0-7
constexpr int EPI_LOAD_WARP = 8;          // warp 8: bulk copies of the s H_i^T images and Z_i, Q and O_s rows
constexpr int EPI_THREADS = EPI_COMPUTE + 32;

template <int D>
struct EpiCfg {
  static constexpr int SLABS = D / 64;               // K slabs of 64 fp16 (128 bytes)
  static constexpr int TILE = D * D * 2;             // one fp16 operand image (atom_off layout)
  static constexpr int SBO = SLABS * 1024;           // bytes between 8-row groups of an image
  static constexpr int HC = D / 2;                   // features (and output columns) per compute thread
  static constexpr int RSLAB = BQ * 128;             // 128 rows x 64 16-bit columns, 128-byte swizzle
  static constexpr int QB = SLABS * RSLAB;           // the item's Q rows (bf16)
  static constexpr int OSB = SLABS * RSLAB;          // the item's O_s / s_v rows (fp16, quantised path)
  static constexpr int ASLOT = TILE + QB;            // ring A: the s H_i^T image and the Q rows of an item
  static constexpr int NA = 2;                       // ring A slots (freed when the item's MMA completes)
  static constexpr int NO = D == 128 ? 2 : 4;        // ring O slots (freed after the item's readout)
  static constexpr int OFF_O = NA * ASLOT;                    // ring O
  static constexpr int OFF_Z = OFF_O + NO * OSB;              // Z_i [NA][D]
  static constexpr int OFF_SV = OFF_Z + NA * D * 4;           // s_v of each ring O item's head [NO][D]
  static constexpr int OFF_XCH = OFF_SV + NO * D * 4;         // row max per half [2][BQ]
  static constexpr int OFF_DEN = OFF_XCH + 2 * BQ * 4;        // denominator halves [2 buffers][2][BQ]
  static constexpr int OFF_BAR = OFF_DEN + 4 * BQ * 4;
  static constexpr int NBAR = 2 * NA + 2 * NO + 3;   // afull, afree [NA]; ofull, ofree [NO]; dfull [2]; drain
  static constexpr int SMEM = OFF_BAR + 8 * NBAR + 16 + 1024;
  static_assert(SMEM <= 232448, "dynamic shared memory per CTA (227 KB)");
  static_assert(TILE % 1024 == 0 && ASLOT % 1024 == 0 && OFF_O % 1024 == 0 && OSB % 1024 == 0 && OFF_Z % 16 == 0,
                "slot alignment (128-byte swizzle)");
  static constexpr int KSTEPS = D / 16;              // 16 fp16 (8 TMEM columns of A) per MMA
  static constexpr uint32_t IDESC = make_idesc(1, 0, 0, 128, D);   // fp16 x fp16 -> fp32, N = D
  static constexpr uint32_t ACOL = 2 * D;            // accumulators: columns b * D; A buffers: ACOL + b * D / 2
  static constexpr uint32_t TMEM_COLS = 512;
};

// Byte offset of logical 16-byte chunk `c` (8 16-bit columns) of row `r` in
// rows staged by TMA as 64-column slabs with 128-byte swizzle.
__device__ __forceinline__ uint32_t swz_chunk(int r, int c) {
  return (uint32_t)((c >> 3) * (BQ * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

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

// Read-only 16-byte load kept where it is written (its latency overlaps the
// work in between instead of being moved down to the first use), with an L2
// cache policy.
__device__ __forceinline__ uint4 ldg_v4_early(const uint4* p, uint64_t pol) {
  uint4 r;
  asm volatile("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(reinterpret_cast<uint64_t>(p)), "l"(pol));
  return r;
}

// Barrier over the 256 compute threads (id 1).
__device__ __forceinline__ void compute_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
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

// 16 consecutive columns of one row of O_s, at element offset `off` of
// [BH][N][d], as loaded: four 16-byte words of fp32, or two of fp16 O_s / s_v.
// The loads are issued here and consumed later by os_convert.
struct OsChunk {
  uint4 w[4];
};

__device__ __forceinline__ void os_issue(const EpilogueArgs& a, size_t off, uint64_t pol, OsChunk& c) {
  if (a.os_half) {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __half*>(a.os) + off);
    c.w[0] = ldg_v4_early(src, pol);
    c.w[1] = ldg_v4_early(src + 1, pol);
  } else {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const float*>(a.os) + off);
#pragma unroll
    for (int i = 0; i < 4; ++i) c.w[i] = ldg_v4_early(src + i, pol);
  }
}

// The chunk as fp32 O_s (fp16 O_s / s_v times s_v of columns col .. col + 15 of
// head bh, read from `svs`, the head's s_v row in shared memory, when given), also
// written to the fp32 export when there is one.
template <int D>
__device__ __forceinline__ void os_convert(const EpilogueArgs& a, int bh, size_t off, int col, const OsChunk& c,
                                           float (&o)[16], const float* svs = nullptr) {
  if (a.os_half) {
    const float4* sv4 = reinterpret_cast<const float4*>(a.sv + (size_t)bh * D + col);
    const float4* svs4 = reinterpret_cast<const float4*>(svs + col);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const uint32_t u[4] = {c.w[i].x, c.w[i].y, c.w[i].z, c.w[i].w};
      const float4 s0 = svs ? svs4[2 * i] : __ldg(sv4 + 2 * i), s1 = svs ? svs4[2 * i + 1] : __ldg(sv4 + 2 * i + 1);
      const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u[j]));
        o[i * 8 + 2 * j] = f.x * sv[2 * j];
        o[i * 8 + 2 * j + 1] = f.y * sv[2 * j + 1];
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      o[4 * i] = __uint_as_float(c.w[i].x);
      o[4 * i + 1] = __uint_as_float(c.w[i].y);
      o[4 * i + 2] = __uint_as_float(c.w[i].z);
      o[4 * i + 3] = __uint_as_float(c.w[i].w);
    }
  }
  if (a.os_dbg) {
#pragma unroll
    for (int k = 0; k < 16; k += 4)
      *reinterpret_cast<float4*>(a.os_dbg + off + k) = make_float4(o[k], o[k + 1], o[k + 2], o[k + 3]);
  }
}

// O = alpha O_s + (1 - alpha) O_l for NC consecutive columns of one row
// (stored with the streaming L2 policy `pol`).
template <int NC>
__device__ __forceinline__ void mix_store(const EpilogueArgs& a, size_t off, float alpha, const float* osv,
                                          const float* ol, uint64_t pol) {
  float o[NC];
#pragma unroll
  for (int c = 0; c < NC; ++c) o[c] = alpha * osv[c] + (1.f - alpha) * ol[c];
  if (a.ol_dbg) {
#pragma unroll
    for (int c = 0; c < NC; c += 4)
      *reinterpret_cast<float4*>(a.ol_dbg + off + c) = make_float4(ol[c], ol[c + 1], ol[c + 2], ol[c + 3]);
  }
  if (a.out_f32) {
#pragma unroll
    for (int c = 0; c < NC; c += 4)
      stg_u4_policy(static_cast<float*>(a.out) + off + c,
                    make_uint4(__float_as_uint(o[c]), __float_as_uint(o[c + 1]), __float_as_uint(o[c + 2]),
                               __float_as_uint(o[c + 3])),
                    pol);
  } else {
    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.out) + off;
#pragma unroll
    for (int c = 0; c < NC; c += 8)
      stg_u4_policy(dst + c,
                    make_uint4(cvt_bf16x2(o[c], o[c + 1]), cvt_bf16x2(o[c + 2], o[c + 3]), cvt_bf16x2(o[c + 4], o[c + 5]),
                               cvt_bf16x2(o[c + 6], o[c + 7])),
                    pol);
  }
}

template <int D>
__global__ void __launch_bounds__(EPI_THREADS, 1) epilogue_kernel(const __grid_constant__ CUtensorMap tq,
                                                                  const __grid_constant__ CUtensorMap tos,
                                                                  const __grid_constant__ CUtensorMap tout, Shape s,
                                                                  EpilogueArgs a) {
  using C = EpiCfg<D>;
  extern __shared__ uint8_t esm_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(esm_raw) + 1023) & ~uintptr_t(1023));
  // ring A slot b: s H_i^T image at b * ASLOT, Q rows at + TILE; ring O slot c at OFF_O + c * OSB
  float* zbuf = reinterpret_cast<float*>(base + C::OFF_Z);
  float* svbuf = reinterpret_cast<float*>(base + C::OFF_SV);
  float* xch = reinterpret_cast<float*>(base + C::OFF_XCH);
  float* den_s = reinterpret_cast<float*>(base + C::OFF_DEN);
  uint64_t* afull = reinterpret_cast<uint64_t*>(base + C::OFF_BAR);   // [NA] image, Q rows and Z_i landed
  uint64_t* afree = afull + C::NA;        // [NA] the item's MMA has completed (phi read Q before it)
  uint64_t* ofull = afree + C::NA;        // [NO] O_s rows landed
  uint64_t* ofree = ofull + C::NO;        // [NO] the item's readout is done
  uint64_t* dfull = ofree + C::NO;        // [2] accumulator complete
  uint64_t* drain = dfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(afull + C::NBAR);
  int* abort_flag = reinterpret_cast<int*>(afull + C::NBAR) + 1;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int total = s.BH * s.nq;
  const bool has_linear = s.k < s.nk;

  if (tid == 0) {
    for (int b = 0; b < C::NA; ++b) {
      mbar_init(afull + b, 1);
      mbar_init(afree + b, 1);
    }
    for (int b = 0; b < C::NO; ++b) {
      mbar_init(ofull + b, 1);
      mbar_init(ofree + b, EPI_COMPUTE);
    }
    mbar_init(dfull, 1);
    mbar_init(dfull + 1, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == EPI_LOAD_WARP) {
    // ---------------------------------------------------------------- loader
    // lane 0, ring A: per item the s H_i^T image and the Z_i row (bulk copies) and the
    //   Q rows (TMA, 64-column slabs), once the MMA of item it - NA has completed;
    // lane 1, ring O: per item the fp16 O_s rows (TMA; quantised path only) and the
    //   head's s_v row (bulk copy), once the readout of item it - NO is done.
    if (lane < 2 && has_linear && (lane == 0 || a.os_half)) {
      const uint64_t once = l2_policy_evict_first();   // each is read once
      const int NR = lane == 0 ? C::NA : C::NO;
      uint64_t* rfull = lane == 0 ? afull : ofull;
      uint64_t* rfree = lane == 0 ? afree : ofree;
      int it = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < total; w += gridDim.x, ++it) {
        const int sb = it % NR;
        if (it >= NR && !mbar_wait(rfree + sb, ((it / NR) - 1) & 1, abort_flag, a.status, a.budget_ns)) {
          ok = false;
          break;
        }
        const int row0 = w * BQ;                   // (head, query block) w starts at row w * 128 of [BH*N]
        if (lane == 0) {
          uint8_t* slot = base + sb * C::ASLOT;
          mbar_arrive_expect_tx(afull + sb, (uint32_t)(C::TILE + C::QB + D * 4));
          bulk_load_hint(slot, a.hi + (size_t)w * D * D, (uint32_t)C::TILE, afull + sb, once);
#pragma unroll
          for (int sl = 0; sl < C::SLABS; ++sl)
            tma_load_2d(slot + C::TILE + sl * C::RSLAB, &tq, afull + sb, sl * 64, row0);
          bulk_load(zbuf + sb * D, a.Zi + (size_t)w * D, (uint32_t)(D * 4), afull + sb);
        } else {
          uint8_t* slot = base + C::OFF_O + sb * C::OSB;
          mbar_arrive_expect_tx(ofull + sb, (uint32_t)(C::OSB + D * 4));
#pragma unroll
          for (int sl = 0; sl < C::SLABS; ++sl) tma_load_2d(slot + sl * C::RSLAB, &tos, ofull + sb, sl * 64, row0);
          // and the head's s_v row beside it (the readout's dequantisation scale, read
          // from shared memory instead of 16 global loads a thread and item)
          bulk_load(svbuf + sb * D, a.sv + (size_t)(w / s.nq) * D, (uint32_t)(D * 4), ofull + sb);
        }
      }
      if (!ok)   // copies in flight land before the CTA releases its shared memory
        for (int q = it > NR ? it - NR : 0; q < it; ++q) mbar_wait_drain(rfull + q % NR, (q / NR) & 1, 20000000ull);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- compute warps
    constexpr int HC = C::HC;
    constexpr float kLog2e = 1.4426950408889634f;
    const int qd = warp & 3, fh = warp >> 2;     // TMEM lane quadrant, feature / column half
    const int r = qd * 32 + lane;                // query row of the block = TMEM lane
    const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
    const uint64_t stream_pol = l2_policy_evict_first();   // Q, O_s and out are touched once here
    auto row_of = [&](int w) { return (size_t)(w / s.nq) * s.N + (size_t)(w % s.nq) * BQ + r; };

    if (!has_linear) {
      float zero[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) zero[c] = 0.f;
      for (int w = blockIdx.x; w < total; w += gridDim.x) {
        const int bh = w / s.nq, qi = w % s.nq;
        const float alpha = a.alpha[(size_t)(bh % a.H) * s.nq + qi];
        const size_t row = row_of(w);
#pragma unroll
        for (int cc = 0; cc < HC / 16; ++cc) {
          const size_t off = row * D + fh * HC + cc * 16;
          OsChunk ch;
          os_issue(a, off, stream_pol, ch);
          float osv[16];
          os_convert<D>(a, bh, off, fh * HC + cc * 16, ch, osv);
          mix_store<16>(a, off, alpha, osv, zero, stream_pol);
        }
      }
    } else {
      // bf16 output on the quantised path: staged in the O_s slot and stored by TMA
      const bool tma_out = a.os_half && !a.out_f32;
      int out_pending = -1;                      // thread 0: ring O slot whose TMA store may still read it
      // readout of item `itp` (work index wp): 16 accumulator columns at a time
      // scaled to O_l, mixed with O_s (from the item's slot on the quantised path)
      // and stored; then the slot is handed back to the loader
      auto readout = [&](int itp, int wp) -> bool {
        const int bh = wp / s.nq, qi = wp % s.nq;
        const float alpha = a.alpha[(size_t)(bh % a.H) * s.nq + qi];
        const float hsc = a.hscale[bh];
        const size_t row = row_of(wp);
        const int bp = itp & 1;
        const int so = itp % C::NO;
        const uint8_t* osl = base + C::OFF_O + so * C::OSB;
        const size_t off0 = row * D + fh * HC;
        OsChunk ch[2];
        if (!a.os_half) os_issue(a, off0, stream_pol, ch[0]);   // fp32 O_s from global, in flight during the wait
        bool ok = mbar_wait(dfull + bp, (itp >> 1) & 1, abort_flag, a.status, a.budget_ns);
        if (a.os_half) ok = ok && mbar_wait(ofull + so, (itp / C::NO) & 1, abort_flag, a.status, a.budget_ns);
        // every compute thread takes the same exit (the output path below has a barrier)
        if (compute_sync_any(!ok)) return false;
        tc_fence_after();
        const float inv = 1.f / (hsc * (den_s[(bp * 2) * BQ + r] + den_s[(bp * 2 + 1) * BQ + r]));
#pragma unroll
        for (int cc = 0; cc < HC / 16; ++cc) {
          const int col = fh * HC + cc * 16;
          if (a.os_half) {
            ch[cc & 1].w[0] = *reinterpret_cast<const uint4*>(osl + swz_chunk(r, col / 8));
            ch[cc & 1].w[1] = *reinterpret_cast<const uint4*>(osl + swz_chunk(r, col / 8 + 1));
          } else if (cc + 1 < HC / 16) {
            os_issue(a, off0 + (cc + 1) * 16, stream_pol, ch[(cc + 1) & 1]);
          }
          uint32_t v[16];
          tmem_ld16(tmem + lane_base + (uint32_t)(bp * D + col), v);
          tmem_wait_ld();
          float osv[16];
          os_convert<D>(a, bh, off0 + cc * 16, col, ch[cc & 1], osv, a.os_half ? svbuf + so * D : nullptr);
          float ol[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) ol[c] = __uint_as_float(v[c]) * inv;
          if (tma_out) {
            float o[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) o[c] = alpha * osv[c] + (1.f - alpha) * ol[c];
            uint8_t* ow = const_cast<uint8_t*>(osl);
            *reinterpret_cast<uint4*>(ow + swz_chunk(r, col / 8)) =
                make_uint4(cvt_bf16x2(o[0], o[1]), cvt_bf16x2(o[2], o[3]), cvt_bf16x2(o[4], o[5]), cvt_bf16x2(o[6], o[7]));
            *reinterpret_cast<uint4*>(ow + swz_chunk(r, col / 8 + 1)) =
                make_uint4(cvt_bf16x2(o[8], o[9]), cvt_bf16x2(o[10], o[11]), cvt_bf16x2(o[12], o[13]),
                           cvt_bf16x2(o[14], o[15]));
            if (a.ol_dbg) {
#pragma unroll
              for (int c = 0; c < 16; c += 4)
                *reinterpret_cast<float4*>(a.ol_dbg + off0 + cc * 16 + c) = make_float4(ol[c], ol[c + 1], ol[c + 2], ol[c + 3]);
            }
          } else {
            mix_store<16>(a, off0 + cc * 16, alpha, osv, ol, stream_pol);
          }
        }
        tc_fence_before();   // the reads are ordered before the next compute barrier (the MMA that reuses it)
        if (tma_out) {
          // the bf16 rows are in the O_s slot (each thread overwrote the chunks it read):
          // thread 0 stores them with TMA and releases the slot once the store has read it
          fence_proxy_async_smem();
          compute_sync();
          if (tid == 0) {
            if (out_pending >= 0) {
              bulk_wait_read0();
              mbar_arrive(ofree + out_pending);
            }
#pragma unroll
            for (int sl = 0; sl < C::SLABS; ++sl) tma_store_2d(&tout, osl + sl * C::RSLAB, sl * 64, wp * BQ);
            bulk_commit();
            out_pending = so;
          } else {
            mbar_arrive(ofree + so);
          }
        } else {
          mbar_arrive(ofree + so);
        }
        return true;
      };

      int it = 0, wprev = -1;
      bool ok = true, rd_ok = true, issued = false;
      for (int w = blockIdx.x; w < total; w += gridDim.x, ++it) {
        const int b = it & 1;                    // TMEM A buffer, accumulator and denominators
        const int sb = it % C::NA;               // the item's ring A slot
        const uint8_t* qs = base + sb * C::ASLOT + C::TILE;
        bool fok = mbar_wait(afull + sb, (it / C::NA) & 1, abort_flag, a.status, a.budget_ns);
        fok = __all_sync(0xffffffffu, fok);
        ok = ok && fok;
        // ---- phi = softmax over the d features. Its normalisation cancels in
        // O_l = phi H_i / (phi Z_i), so the operand is e = exp(q - M) with M
        // the row max (exchanged between the two halves) and no row sum.
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int q = 0; q < HC / 8; ++q) {
          float v8[8];
          unpack8(fok ? *reinterpret_cast<const uint4*>(qs + swz_chunk(r, fh * (HC / 8) + q)) : make_uint4(0u, 0u, 0u, 0u),
                  v8);
#pragma unroll
          for (int c = 0; c < 8; ++c) m4[c & 3] = fmaxf(m4[c & 3], v8[c]);
        }
        const float m = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        xch[fh * BQ + r] = m;
        compute_sync();
        const float mb = fmaxf(m, xch[(fh ^ 1) * BQ + r]) * kLog2e;
        // den = e . Z_i over this half of the features
        const float4* zi4 = reinterpret_cast<const float4*>(zbuf + sb * D + fh * HC);
        float d4[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t pk[HC / 2];
#pragma unroll
        for (int q = 0; q < HC / 8; ++q) {
          float v8[8];
          unpack8(fok ? *reinterpret_cast<const uint4*>(qs + swz_chunk(r, fh * (HC / 8) + q)) : make_uint4(0u, 0u, 0u, 0u),
                  v8);
#pragma unroll
          for (int c = 0; c < 8; c += 4) {
            const float4 zz = fok ? zi4[(q * 8 + c) / 4] : make_float4(0.f, 0.f, 0.f, 0.f);
            const float p0 = ex2_approx(fmaf(v8[c], kLog2e, -mb)), p1 = ex2_approx(fmaf(v8[c + 1], kLog2e, -mb));
            const float p2 = ex2_approx(fmaf(v8[c + 2], kLog2e, -mb)), p3 = ex2_approx(fmaf(v8[c + 3], kLog2e, -mb));
            d4[0] = fmaf(p0, zz.x, d4[0]);
            d4[1] = fmaf(p1, zz.y, d4[1]);
            d4[2] = fmaf(p2, zz.z, d4[2]);
            d4[3] = fmaf(p3, zz.w, d4[3]);
            pk[(q * 8 + c) / 2] = h2(p0, p1);
            pk[(q * 8 + c) / 2 + 1] = h2(p2, p3);
          }
        }
        den_s[(b * 2 + fh) * BQ + r] = (d4[0] + d4[1]) + (d4[2] + d4[3]);
        const uint32_t ta = tmem + lane_base + C::ACOL + (uint32_t)(b * (D / 2) + fh * (HC / 2));
        if constexpr (HC / 2 == 32) {
          tmem_st32(ta, pk);
        } else {
          tmem_st16(ta, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        // every compute thread takes this exit together; past it, the phi operand is in
        // TMEM and the readout of item it - 2 (same accumulator) is complete
        if (compute_sync_any(!ok || !rd_ok)) { ok = false; break; }
        if (tid == 0) {   // MMA issue: D_b = phi(Q_i) (s H_i), the image from the item's slot
          tc_fence_after();
          const uint32_t acol = tmem + C::ACOL + (uint32_t)(b * (D / 2));
          const uint64_t bd = make_sdesc(smem_u32(base + sb * C::ASLOT), C::SBO, LAYOUT_SW128);
#pragma unroll
          for (int ks = 0; ks < C::KSTEPS; ++ks)
            mma_f16_ts(tmem + (uint32_t)(b * D), acol + ks * 8,
                       bd + (uint64_t)(((ks >> 2) * 1024 + (ks & 3) * 32) >> 4), C::IDESC, ks != 0);
          issued = true;
          tc_commit(afree + sb);   // the image and the Q rows (read by phi before this) can be reloaded
          tc_commit(dfull + b);
        }
        // ---- the previous item's readout overlaps this item's MMAs
        if (wprev >= 0) rd_ok = readout(it - 1, wprev);
        wprev = w;
      }
      if (ok && rd_ok && wprev >= 0) rd_ok = readout(it - 1, wprev);
      if (tid == 0 && out_pending >= 0) bulk_wait0();   // the last output rows have reached global memory
      if (tid == 0 && issued && !(ok && rd_ok)) {   // issued MMAs finish before TMEM and shared memory are released
        tc_commit(drain);
        mbar_wait_drain(drain, 0, 20000000ull);
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

constexpr int kSMs = 148;   // B200 streaming multiprocessors

}  // namespace

cudaError_t launch_epilogue(const Shape& s, const CUtensorMap& tq, const CUtensorMap& tos, const CUtensorMap& tout,
                            const EpilogueArgs& a, cudaStream_t st) {
  const int total = s.BH * s.nq;
  const int grid = total < kSMs ? total : kSMs;
  if (s.d == 128) {
    auto k = epilogue_kernel<128>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, EpiCfg<128>::SMEM);
    k<<<grid, EPI_THREADS, EpiCfg<128>::SMEM, st>>>(tq, tos, tout, s, a);
  } else {
    auto k = epilogue_kernel<64>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, EpiCfg<64>::SMEM);
    k<<<grid, EPI_THREADS, EpiCfg<64>::SMEM, st>>>(tq, tos, tout, s, a);
  }
  return cudaGetLastError();
}

}  // namespace sla2
