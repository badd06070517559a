// Linear branch apply + mix (SLA2 summary page, steps 3 and 4; SLA2 detail
// page §7 note 2: per-key-block h_j precomputed, then accumulated):
//   H_i = H_total - sum_{j selected} h_j,   Z_i = Z_total - sum_{j selected} z_j
//   O_l = phi(Q_i) H_i / (phi(Q_i) Z_i)      (phi: softmax over the d features)
//   O   = alpha_i O_s + (1 - alpha_i) O_l
// When every key block is selected there is no unselected block and O_l := 0.
//
// The numerator never forms H_i: by linearity it is one tensor-core
// accumulation over k + 1 operand tiles,
//   D = phi(Q_i) (s H_total) + sum_{j selected} phi(Q_i) (-s h_j)
// where the linear-state pass stored each -s h_j^T, and the reduce pass
// s H_total^T, as fp16 d x d tiles already in the 128-byte-swizzled K-major
// operand layout; s is a per-head power of two that keeps s H_total inside
// the fp16 range. The denominator phi(Q_i) Z_i is a d-term fp32 dot product
// per query row, taken while phi is computed; s cancels in O_l = D / (s den).
//
// The tiles go to the tensor core in groups of G = 256 / d, stacked along N,
// so that every MMA is 128 x 256 x 16: at that size the tensor pipe hides the
// per-group barrier wait and commit, which cost a large share of the time of
// 128 x 128 MMAs. The accumulator then holds G column blocks, one per tile
// slot, which the readout adds up.
//
// Persistent CTAs (one per SM) walk the (head, query block) items in
// head-major order, so the SMs work on neighbouring query blocks of the same
// head and the head's tiles stay in L2. Per CTA:
//   warps 8,10 producers: each group's tiles, one 1-D bulk copy per tile,
//              into a ring of shared-memory stages (a single issuing thread
//              serialises its bulk copies, so two warps share the issue);
//   warp 9     MMA issuer: per group, d/16 tcgen05 kind::f16 MMAs with
//              A = phi(Q_i) in tensor memory and B = the stacked tiles, into
//              the TMEM accumulator, then a commit that frees the stage;
//   warps 0-7  per item: phi(Q_i), one query row
//              per thread and half of the features per warp (the two halves
//              exchange their row max and sum), stored as fp16 into one of two
//              TMEM A buffers; the denominators phi(Q_i) . Z_i (Z_i precomputed
//              per query block, copied in by producer 0); then, while the MMAs of this
//              item run, the readout of the previous item: the accumulator is
//              read into registers and released at once, then O_l = D / (s den),
//              the alpha mix with O_s and the store.
// A lives in tensor memory and Q / O_s go through registers, so shared memory
// holds only the tile ring and its bandwidth goes to the tiles, each written
// once by its copy and read once by the MMAs.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "device.cuh"
#include "kernels.cuh"

namespace sla2 {

namespace {

constexpr int EPI_COMPUTE = 256;          // warps 0-7
constexpr int EPI_PRODUCER_WARP0 = 8;
constexpr int EPI_MMA_WARP = 9;
constexpr int EPI_PRODUCER_WARP1 = 10;
constexpr int EPI_NPROD = 2;
constexpr int EPI_THREADS = EPI_COMPUTE + 96;

template <int D>
struct EpiCfg {
  static constexpr int G = 256 / D;                  // tiles per group (MMA N = 256)
  static constexpr int SLABS = D / 64;               // K slabs of 64 fp16 (128 bytes)
  static constexpr int TILE = D * D * 2;             // one fp16 operand tile (atom_off layout)
  static constexpr int SBO = SLABS * 1024;           // bytes between 8-row groups of a tile / group
  static constexpr int STAGE = G * TILE;             // one ring stage (a group: tiles back to back)
  static constexpr int NS = (192 * 1024) / STAGE;    // ring stages: 3 (d = 128), 6 (d = 64)
  static constexpr int HC = D / 2;                   // features (and output columns) per thread
  static constexpr int OFF_Z = NS * STAGE;                    // Z_i of two items [2][D]
  static constexpr int OFF_XCH = OFF_Z + 2 * D * 4;           // (max, sum) per row and half [2][BQ]
  static constexpr int OFF_DEN = OFF_XCH + 2 * BQ * 8;        // denominator halves [2 buffers][2][BQ]
  static constexpr int OFF_BAR = OFF_DEN + 4 * BQ * 4;
  static constexpr int NBAR = 2 * NS + 9;
  static constexpr int SMEM = OFF_BAR + 8 * NBAR + 16 + 1024;
  static_assert(SMEM <= 232448, "dynamic shared memory per CTA (227 KB)");
  static_assert(STAGE % 1024 == 0 && OFF_Z % 16 == 0, "bulk-copy and swizzle-atom alignment of the ring");
  static constexpr int KSTEPS = D / 16;              // 16 fp16 (8 TMEM columns of A) per MMA
  static constexpr uint32_t ACOL = 256;              // A buffers: columns ACOL + b * D / 2
  static constexpr uint32_t TMEM_COLS = 512;
};

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

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<uint64_t>(p)));
}

// Barrier over the 256 compute threads.
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

// O = alpha O_s + (1 - alpha) O_l for 32 consecutive columns of one row
// (stored with the streaming L2 policy `pol`).
__device__ __forceinline__ void mix_store(const EpilogueArgs& a, size_t off, float alpha, const float4* osv,
                                          const float* ol, uint64_t pol) {
  float o[32];
#pragma unroll
  for (int c = 0; c < 32; c += 4) {
    const float4 v = osv[c / 4];
    o[c] = alpha * v.x + (1.f - alpha) * ol[c];
    o[c + 1] = alpha * v.y + (1.f - alpha) * ol[c + 1];
    o[c + 2] = alpha * v.z + (1.f - alpha) * ol[c + 2];
    o[c + 3] = alpha * v.w + (1.f - alpha) * ol[c + 3];
  }
  if (a.ol_dbg) {
#pragma unroll
    for (int c = 0; c < 32; c += 4)
      *reinterpret_cast<float4*>(a.ol_dbg + off + c) = make_float4(ol[c], ol[c + 1], ol[c + 2], ol[c + 3]);
  }
  if (a.out_f32) {
#pragma unroll
    for (int c = 0; c < 32; c += 4)
      stg_u4_policy(static_cast<float*>(a.out) + off + c,
                    make_uint4(__float_as_uint(o[c]), __float_as_uint(o[c + 1]), __float_as_uint(o[c + 2]),
                               __float_as_uint(o[c + 3])),
                    pol);
  } else {
    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.out) + off;
#pragma unroll
    for (int c = 0; c < 32; c += 8)
      stg_u4_policy(dst + c,
                    make_uint4(cvt_bf16x2(o[c], o[c + 1]), cvt_bf16x2(o[c + 2], o[c + 3]), cvt_bf16x2(o[c + 4], o[c + 5]),
                               cvt_bf16x2(o[c + 6], o[c + 7])),
                    pol);
  }
}

template <int D>
__global__ void __launch_bounds__(EPI_THREADS, 1) epilogue_kernel(Shape s, EpilogueArgs a) {
  using C = EpiCfg<D>;
  extern __shared__ uint8_t esm_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(esm_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = base;
  float* zbuf = reinterpret_cast<float*>(base + C::OFF_Z);
  float2* xch = reinterpret_cast<float2*>(base + C::OFF_XCH);
  float* den_s = reinterpret_cast<float*>(base + C::OFF_DEN);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + C::OFF_BAR);
  uint64_t* empty = full + C::NS;
  uint64_t* aready = empty + C::NS;       // [2] phi(Q) operand written to TMEM
  uint64_t* dfull = aready + 2;           // accumulator complete
  uint64_t* dfree = dfull + 1;            // accumulator read into registers
  uint64_t* zfull = dfree + 1;            // [2] Z_i of an item landed
  uint64_t* zfree = zfull + 2;            // [2] Z_i of an item used
  uint64_t* drain = zfree + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_flag = reinterpret_cast<int*>(drain + 1) + 1;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int total = s.BH * s.nq;
  const bool has_linear = s.k < s.nk;
  const int ntile = s.k + 1;
  const int nblk = ntile < C::G ? ntile : C::G;   // accumulator column blocks in use

  if (tid == 0) {
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(full + i, EPI_NPROD);
      mbar_init(empty + i, 1);
    }
    mbar_init(aready, EPI_COMPUTE);
    mbar_init(aready + 1, EPI_COMPUTE);
    mbar_init(dfull, 1);
    mbar_init(dfree, EPI_COMPUTE);
    for (int b = 0; b < 2; ++b) {
      mbar_init(zfull + b, 1);
      mbar_init(zfree + b, EPI_COMPUTE);
    }
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

  if (warp == EPI_PRODUCER_WARP0 || warp == EPI_PRODUCER_WARP1) {
    // ---------------------------------------------------------------- producers
    const int pr = warp == EPI_PRODUCER_WARP0 ? 0 : 1;   // this producer's tiles: t = pr, pr + 2, ...
    if (lane == 0 && has_linear) {
      const size_t tile_elems = (size_t)D * D;
      const uint64_t keep = l2_policy_evict_last();   // a tile is re-read by ~k query blocks of the head
      int st = 0, ng = 0, it = 0, nz = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int w = blockIdx.x; ok && w < total; w += gridDim.x, ++it) {
        const int bh = w / s.nq, qi = w % s.nq;
        const int32_t* sel = a.idx + ((size_t)bh * s.nq + qi) * s.k;
        if (pr == 0) {   // Z_i of this item (its buffer was last read for item it - 2)
          const int b = it & 1;
          if (it >= 2 && !mbar_wait(zfree + b, ((it >> 1) - 1) & 1, abort_flag, a.status, a.budget_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(zfull + b, D * 4);
          bulk_load(zbuf + b * D, a.Zi + ((size_t)bh * s.nq + qi) * D, D * 4, zfull + b);
          ++nz;
        }
        for (int n0 = 0; n0 < ntile; n0 += C::G) {
          const int cnt = ntile - n0 < C::G ? ntile - n0 : C::G;
          if (ng >= C::NS && !mbar_wait(empty + st, ph ^ 1u, abort_flag, a.status, a.budget_ns)) {
            ok = false;
            break;
          }
          const int mine = cnt > pr ? (cnt - pr + EPI_NPROD - 1) / EPI_NPROD : 0;
          mbar_arrive_expect_tx(full + st, (uint32_t)(mine * C::TILE));
          uint8_t* dst = ring + st * C::STAGE;
          for (int t = pr; t < cnt; t += EPI_NPROD) {
            const int n = n0 + t;
            const uint16_t* src = n == 0 ? a.htile + (size_t)bh * tile_elems
                                         : a.hT + ((size_t)bh * s.nk + __ldg(sel + n - 1)) * tile_elems;
            bulk_load_hint(dst + t * C::TILE, src, C::TILE, full + st, keep);
          }
          ++ng;
          if (++st == C::NS) {
            st = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {   // let the copies in flight land before the CTA's shared memory is released
        for (int q = (ng > C::NS ? ng - C::NS : 0); q < ng; ++q)
          mbar_wait_drain(full + q % C::NS, (q / C::NS) & 1, 20000000ull);
        for (int q = (nz > 2 ? nz - 2 : 0); q < nz; ++q) mbar_wait_drain(zfull + (q & 1), (q >> 1) & 1, 20000000ull);
      }
    }
    __syncwarp();
  } else if (warp == EPI_MMA_WARP) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0 && has_linear) {
      const uint64_t bdesc0 = make_sdesc(smem_u32(ring), C::SBO, LAYOUT_SW128);
      int st = 0, it = 0;
      uint32_t ph = 0;
      bool ok = true, issued = false;
      for (int w = blockIdx.x; ok && w < total; w += gridDim.x, ++it) {
        const int b = it & 1;
        if (!mbar_wait(aready + b, (it >> 1) & 1, abort_flag, a.status, a.budget_ns)) { ok = false; break; }
        if (it >= 1 && !mbar_wait(dfree, (it - 1) & 1, abort_flag, a.status, a.budget_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t acol = tmem + C::ACOL + (uint32_t)(b * (D / 2));
        for (int n0 = 0; n0 < ntile; n0 += C::G) {
          const int cnt = ntile - n0 < C::G ? ntile - n0 : C::G;
          const uint32_t idesc = make_idesc(1, 0, 0, 128, (uint32_t)(cnt * D));   // fp16 x fp16 -> fp32
          if (!mbar_wait(full + st, ph, abort_flag, a.status, a.budget_ns)) { ok = false; break; }
          tc_fence_after();
          // descriptor start addresses advance in 16-byte units
          const uint64_t bd = bdesc0 + (uint64_t)((st * C::STAGE) >> 4);
#pragma unroll
          for (int ks = 0; ks < C::KSTEPS; ++ks)
            mma_f16_ts(tmem, acol + ks * 8, bd + (uint64_t)(((ks >> 2) * 1024 + (ks & 3) * 32) >> 4), idesc,
                       (n0 | ks) != 0);
          issued = true;
          tc_commit(empty + st);
          if (++st == C::NS) {
            st = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(dfull);
      }
      if (!ok && issued) {   // issued MMAs finish before the CTA releases TMEM and shared memory
        tc_commit(drain);
        mbar_wait_drain(drain, 0, 20000000ull);
      }
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
      float zero[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) zero[c] = 0.f;
      for (int w = blockIdx.x; w < total; w += gridDim.x) {
        const int bh = w / s.nq, qi = w % s.nq;
        const float alpha = a.alpha[(size_t)(bh % a.H) * s.nq + qi];
        const size_t row = row_of(w);
#pragma unroll
        for (int cc = 0; cc < HC / 32; ++cc) {
          float4 osv[8];
          const float4* osr = reinterpret_cast<const float4*>(a.os + row * D + fh * HC + cc * 32);
#pragma unroll
          for (int c = 0; c < 8; ++c) osv[c] = __ldg(osr + c);
          mix_store(a, row * D + fh * HC + cc * 32, alpha, osv, zero, stream_pol);
        }
      }
    } else {
      // readout of item `itp` (work index wp): the accumulator's column blocks
      // summed into registers, the accumulator released, then O_l, mix, store
      auto readout = [&](int itp, int wp) -> bool {
        const int bh = wp / s.nq, qi = wp % s.nq;
        const float alpha = a.alpha[(size_t)(bh % a.H) * s.nq + qi];
        const float hsc = a.hscale[bh];
        const size_t row = row_of(wp);
        const int bp = itp & 1;
        const float* osr = a.os + row * D + fh * HC;
        float4 osv[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) osv[c] = ldg_f4_policy(reinterpret_cast<const float4*>(osr) + c, stream_pol);
        bool ok = mbar_wait(dfull, itp & 1, abort_flag, a.status, a.budget_ns);
        ok = __all_sync(0xffffffffu, ok);
        tc_fence_after();
        if (!ok) return false;
        float ol[HC];
#pragma unroll
        for (int cc = 0; cc < HC / 32; ++cc) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_base + (uint32_t)(fh * HC + cc * 32), v);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) ol[cc * 32 + c] = __uint_as_float(v[c]);
          for (int blk = 1; blk < nblk; ++blk) {
            tmem_ld32(tmem + lane_base + (uint32_t)(blk * D + fh * HC + cc * 32), v);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) ol[cc * 32 + c] += __uint_as_float(v[c]);
          }
        }
        tc_fence_before();
        mbar_arrive(dfree);
        const float inv = 1.f / (hsc * (den_s[(bp * 2) * BQ + r] + den_s[(bp * 2 + 1) * BQ + r]));
#pragma unroll
        for (int c = 0; c < HC; ++c) ol[c] *= inv;
#pragma unroll
        for (int cc = 0; cc < HC / 32; ++cc) {
          if (cc > 0) {
#pragma unroll
            for (int c = 0; c < 8; ++c) osv[c] = ldg_f4_policy(reinterpret_cast<const float4*>(osr + cc * 32) + c, stream_pol);
          }
          mix_store(a, row * D + fh * HC + cc * 32, alpha, osv, ol + cc * 32, stream_pol);
        }
        return true;
      };

      uint4 qv[HC / 8];                          // this thread's half row of Q (bf16)
      auto load_q = [&](int w) {               // issued here, consumed one item later
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.q) + row_of(w) * D + fh * HC);
#pragma unroll
        for (int i = 0; i < HC / 8; ++i) qv[i] = ldg_v4_early(src + i, stream_pol);
      };
      load_q(blockIdx.x);
      int it = 0, wprev = -1;
      bool ok = true, rd_ok = true;
      for (int w = blockIdx.x; w < total; w += gridDim.x, ++it) {
        const int bh = w / s.nq, qi = w % s.nq;
        const int b = it & 1;
        if (wprev >= 0) {                        // O_s of the previous item, read out below
          const float* p = a.os + row_of(wprev) * D + fh * HC;
#pragma unroll
          for (int c = 0; c < HC; c += 32) prefetch_l2(p + c);
        }
        (void)bh;
        (void)qi;
        // ---- phi = softmax over the d features: local max / sum, then exchanged between the halves
        float x[HC];
#pragma unroll
        for (int q = 0; q < HC / 8; ++q) {
          float v8[8];
          unpack8(qv[q], v8);
#pragma unroll
          for (int c = 0; c < 8; ++c) x[q * 8 + c] = v8[c];
        }
        {
          const int wn = w + gridDim.x;          // the next item's Q rows, consumed next iteration
          if (wn < total) load_q(wn);
        }
        // four independent partial chains for the max and the sum
        float m4[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
        for (int c = 4; c < HC; ++c) m4[c & 3] = fmaxf(m4[c & 3], x[c]);
        const float m = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        const float mb = m * kLog2e;
        float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < HC; ++c) {
          x[c] = ex2_approx(fmaf(x[c], kLog2e, -mb));
          s4[c & 3] += x[c];
        }
        const float sum = (s4[0] + s4[1]) + (s4[2] + s4[3]);
        xch[fh * BQ + r] = make_float2(m, sum);
        compute_sync();
        const float2 o = xch[(fh ^ 1) * BQ + r];
        const float M = fmaxf(m, o.x);
        const float e_own = ex2_approx((m - M) * kLog2e);
        const float scale = e_own / (sum * e_own + o.y * ex2_approx((o.x - M) * kLog2e));
        // den = phi(Q_i) . Z_i over this half of the features
        bool zok = mbar_wait(zfull + b, (it >> 1) & 1, abort_flag, a.status, a.budget_ns);
        zok = __all_sync(0xffffffffu, zok);
        ok = ok && zok;
        const float4* zi4 = reinterpret_cast<const float4*>(zbuf + b * D + fh * HC);
        float d4[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t pk[HC / 2];
#pragma unroll
        for (int c = 0; c < HC; c += 4) {
          const float4 zz = zok ? zi4[c / 4] : make_float4(0.f, 0.f, 0.f, 0.f);
          const float p0 = x[c] * scale, p1 = x[c + 1] * scale, p2 = x[c + 2] * scale, p3 = x[c + 3] * scale;
          d4[0] = fmaf(p0, zz.x, d4[0]);
          d4[1] = fmaf(p1, zz.y, d4[1]);
          d4[2] = fmaf(p2, zz.z, d4[2]);
          d4[3] = fmaf(p3, zz.w, d4[3]);
          pk[c / 2] = h2(p0, p1);
          pk[c / 2 + 1] = h2(p2, p3);
        }
        mbar_arrive(zfree + b);
        den_s[(b * 2 + fh) * BQ + r] = (d4[0] + d4[1]) + (d4[2] + d4[3]);
        const uint32_t ta = tmem + lane_base + C::ACOL + (uint32_t)(b * (D / 2) + fh * (HC / 2));
        if constexpr (HC / 2 == 32) {
          tmem_st32(ta, pk);
        } else {
          tmem_st16(ta, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(aready + b);
        // every compute thread takes this exit together
        if (compute_sync_any(!ok || !rd_ok)) { ok = false; break; }
        // ---- the previous item's readout overlaps this item's MMAs
        if (wprev >= 0) rd_ok = readout(it - 1, wprev);
        wprev = w;
      }
      if (ok && rd_ok && wprev >= 0) readout(it - 1, wprev);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// Z_i = Z_total - sum of the selected z_j for every (head, query block), one
// feature per thread, the selected blocks in ascending order.
__global__ void zsel_kernel(const float* __restrict__ Ztot, const float* __restrict__ z, const int32_t* __restrict__ idx,
                            int nq, int nk, int k, float* __restrict__ Zi) {
  const int qi = blockIdx.x, bh = blockIdx.y, c = threadIdx.x, D = blockDim.x;
  const int32_t* sel = idx + ((size_t)bh * nq + qi) * k;
  float acc = Ztot[(size_t)bh * D + c];
#pragma unroll 8
  for (int n = 0; n < k; ++n) acc -= z[((size_t)bh * nk + __ldg(sel + n)) * D + c];
  Zi[((size_t)bh * nq + qi) * D + c] = acc;
}

constexpr int kSMs = 148;   // B200 streaming multiprocessors

}  // namespace

cudaError_t launch_zsel(const Shape& s, const float* Ztot, const float* z, const int32_t* idx, float* Zi,
                        cudaStream_t st) {
  zsel_kernel<<<dim3(s.nq, s.BH), s.d, 0, st>>>(Ztot, z, idx, s.nq, s.nk, s.k, Zi);
  return cudaGetLastError();
}

cudaError_t launch_epilogue(const Shape& s, const EpilogueArgs& a, cudaStream_t st) {
  const int total = s.BH * s.nq;
  const int grid = total < kSMs ? total : kSMs;
  if (s.d == 128) {
    auto k = epilogue_kernel<128>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, EpiCfg<128>::SMEM);
    k<<<grid, EPI_THREADS, EpiCfg<128>::SMEM, st>>>(s, a);
  } else {
    auto k = epilogue_kernel<64>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, EpiCfg<64>::SMEM);
    k<<<grid, EPI_THREADS, EpiCfg<64>::SMEM, st>>>(s, a);
  }
  return cudaGetLastError();
}

}  // namespace sla2
