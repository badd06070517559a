// Launch wrappers shared between the kernel files and the C-ABI layer.
// All pointers are device pointers; every launcher enqueues on `st` and
// returns the launch status.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace sla2 {

// 2-D row-major TMA map (rows x cols elements of esz bytes, box box_cols x
// box_rows, swizzle 0/64/128 bytes); implemented in api.cu.
bool make_tmap_2d(CUtensorMap* m, const void* ptr, int esz, uint64_t cols, uint64_t rows, uint32_t box_cols,
                  uint32_t box_rows, int swizzle_bytes);

constexpr int BQ = 128;   // query block (b_q)
constexpr int BKB = 64;   // key block (b_k)

struct Shape {
  int BH, N, d, nq, nk, k;
  int G;   // key-block chunks per head of the linear-state pass (fixes H_total's summation order)
};

// ---- router (router.cu) ----------------------------------------------------
// Pass over Q, K (and V): pooled Q (fp32), exact fp64 column sums per key block,
// optional INT8 Q-hat + s_q, optional per-channel |V| max (atomic, as uint bits).
// Its pipeline waits are bounded by budget_ns (status gets the timeout code).
// csum (optional, zero at launch): the head's fp64 column sums of K, gathered with
// atomic adds (exact sums, so independent of their order).
cudaError_t launch_pool(const Shape& s, const void* q, const void* k, const void* v, float* qbar, double* ksum,
                        int8_t* qhat, float* sq, unsigned* vamax, unsigned* status, unsigned long long budget_ns,
                        cudaStream_t st, double* csum = nullptr);
constexpr unsigned long long kDefaultWaitBudgetNs = 2000000000ull;   // 2 s per device wait
// The budget every bounded device wait of the next launches gets (the default, or the
// value last set by sla2_set_wait_budget_ns); implemented in api.cu.
unsigned long long wait_budget_ns();
// colmean (fp64 and fp32) from the per-block sums (or, given csum, from the column
// sums the pool pass gathered), and the smoothed pooled keys.
cudaError_t launch_colmean(const Shape& s, const double* ksum, double* c64, float* c32, float* kbar_s,
                           cudaStream_t st, const double* csum = nullptr);
// A = Qbar Wq, Bk = (Kbar - c) Wk, fp32.
cudaError_t launch_proj(const Shape& s, int H, const float* qbar, const float* kbar_s, const float* wq,
                        const float* wk, float* A, float* Bk, cudaStream_t st);
// logits s = A Bk^T / sqrt(d), fp32 [BH][nq][nk]
cudaError_t launch_scores(const Shape& s, const float* A, const float* Bk, float* scores, cudaStream_t st);
// hard top-k per logit row (ties -> lower index), mask and ascending index list
// mask16 (optional): the mask also as fp16 1 / 0 rows of nk8 = nk rounded up to 8
// (zero padding), the A operand of the selected-state product (hsel.cu).
cudaError_t launch_topk(const Shape& s, const float* scores, uint8_t* mask, int32_t* idx, cudaStream_t st,
                        uint16_t* mask16 = nullptr);
int scores_topk_max_nk();
// SoftTop-k relaxation of each logit row: sigmoid(P_c / tau + lambda), row sums k
cudaError_t launch_soft_topk(const Shape& s, const float* scores, float tau, float* soft, float* lam,
                             cudaStream_t st);

// ---- linear state (linear.cu) ---------------------------------------------
// Per key block: h_j, z_j (fp32) and per-chunk partial sums; optionally K-hat /
// s_k and V-hat^T / s_v (quant = 1: e4m3; quant = 0: bf16 copy of V^T).
struct LinearOut {
  // h_j^T [BH][nk][d (V channel e)][d (phi feature c)], by h_mode:
  //   0: fp32 row-major;  1: bf16 row-major;
  //   2: fp16 -s h_j^T (s = h_fp16_scale of the head, from vamax) as the image of
  //      a K-major operand tile in the atom_off layout: 8-row x 128-byte atoms,
  //      16-byte chunks swizzled by row & 7 (what the epilogue's MMA reads as B).
  void* h;
  int h_mode;        // partial sums (and so H_total) are always written transposed too
  float* z;          // [BH][nk][d]
  float* hpart;      // [BH][G][d][d]
  float* zpart;      // [BH][G][d]
  int8_t* khat;      // [BH][N][d] or nullptr
  float* sk;         // [BH][nk]
  void* vhatT;       // [BH][nk][d][64] (u8 e4m3 or bf16) or nullptr
  float* sv;         // [BH][d]
  const unsigned* vamax;  // [BH][d] per-channel max |V| as float bits (quant = 1 or h_mode = 2)
  int quant;
  unsigned* status;
  unsigned long long budget_ns;
};
// number of key-block chunks (CTAs) per head of the linear-state pass for BH heads in
// one launch; the launch itself uses Shape::G
int linear_chunks(int BH, int nk);
cudaError_t launch_linear_state(const Shape& s, const void* k, const void* v, const float* c32, const LinearOut& o,
                                cudaStream_t st);
// H_total^T / Z_total (fp32) from the chunk partials; optionally (vamax given)
// the fp16 image of s H_total^T in the h_mode-2 layout and s per head.
cudaError_t launch_linear_reduce(const Shape& s, const float* hpart, const float* zpart, const unsigned* vamax,
                                 float* Htot, float* Ztot, uint16_t* htile, float* hscale, cudaStream_t st,
                                 const float* z = nullptr, uint16_t* z16 = nullptr);

// ---- sparse branch (sparse.cu) --------------------------------------------
struct SparseArgs {
  const int32_t* idx;   // [BH][nq][k]
  const float* sq;      // [BH][nq]   (quant)
  const float* sk;      // [BH][nk]   (quant)
  const float* sv;      // [BH][d]    (quant)
  void* os;             // [BH][N][d] out: fp32 O_s, or (quant) fp16 O_s / s_v (magnitudes <= 448)
  unsigned* status;
  unsigned long long budget_ns;
};
// tensor maps are built by the caller (api.cu) and passed by value
cudaError_t launch_sparse(const Shape& s, int quant, const CUtensorMap& tq, const CUtensorMap& tk,
                          const CUtensorMap& tv, const SparseArgs& a, cudaStream_t st);
size_t sparse_smem_bytes(int d, int quant);

// ---- epilogue (epilogue.cu) -----------------------------------------------
// ---- selected-state product (hsel.cu) -----------------------------------------
struct HselArgs {
  const uint16_t* htile;  // fp16 s H_total^T operand images [BH][d*d]
  const float* Ztot;      // [BH][d] Z_total
  uint16_t* hi;           // out: fp16 s H_i^T operand images [BH][nq][d*d]
  float* Zi;              // out: [BH][nq][d] Z_i
  unsigned* status;
  unsigned long long budget_ns;
};
// tmask: the fp16 mask [BH*nq][nk8], box {64, 128}; timg: the -s h_j^T images as a
// [BH*nk][d*d] fp16 matrix, box {64, 64}; tz: the fp16 z_j as a [BH*nk][d] matrix,
// box {64, 64}; all with 128-byte swizzle.
cudaError_t launch_hsel(const Shape& s, const CUtensorMap& tmask, const CUtensorMap& timg, const CUtensorMap& tz,
                        const HselArgs& a, cudaStream_t st);

struct EpilogueArgs {
  const void* q;          // bf16 [BH][N][d]
  const uint16_t* hi;     // fp16 s H_i^T operand images [BH][nq][d*d]
  const float* Zi;        // [BH][nq][d] Z_i
  const float* hscale;    // [BH] s
  const void* os;         // [BH][N][d] O_s: fp32, or fp16 O_s / s_v when os_half
  int os_half;
  const float* sv;        // [BH][d] s_v (os_half)
  float* os_dbg;          // optional [BH][N][d] fp32 O_s export
  const float* alpha;     // [H][nq]
  int H;
  void* out;              // [BH][N][d]
  int out_f32;
  float* ol_dbg;          // optional [BH][N][d]
  unsigned* status;
  unsigned long long budget_ns;
};
// tq: Q as [BH*N][d] bf16, box {64, 128}; tos: O_s as [BH*N][d] fp16, box {64, 128}
// (used when os_half); tout: out as [BH*N][d] bf16, box {64, 128} (used when os_half
// and the output is bf16); all with 128-byte swizzle.
cudaError_t launch_epilogue(const Shape& s, const CUtensorMap& tq, const CUtensorMap& tos, const CUtensorMap& tout,
                            const EpilogueArgs& a, cudaStream_t st);

// ---- backward pass (backward.cu) ------------------------------------------
struct BackwardArgs {
  const void* q;          // bf16 [BH][N][d]
  const void* k;
  const void* v;
  const float* c32;       // colmean of K, [BH][d]
  const float* alpha;     // [H][nq]
  const float* dout;      // dL/dO, fp32 [BH][N][d]
  const int32_t* idx;     // selected key blocks [BH][nq][k]
  const float* hT;        // h_j^T fp32 [BH][nk][d][d] (channel, feature)
  const float* z;         // z_j [BH][nk][d]
  const float* HtotT;     // H_total^T [BH][d][d]
  const float* Ztot;      // Z_total [BH][d]
  float* dq;              // outputs, fp32 [BH][N][d]
  float* dk;              // zeroed by the caller (accumulates dK_s, then dK)
  float* dv;              // zeroed by the caller
  float* dalpha;          // [H][nq], zeroed by the caller (summed over the batch)
  float* dos_sum;         // [BH][nq] scratch
  float* dHacc;           // [BH][nk][d][d] scratch, zeroed
  float* dZacc;           // [BH][nk][d] scratch, zeroed
  float* dHtot;           // [BH][d][d] scratch, zeroed
  float* dZtot;           // [BH][d] scratch, zeroed
};
cudaError_t launch_backward(const Shape& s, int H, const BackwardArgs& a, cudaStream_t st);

}  // namespace sla2
