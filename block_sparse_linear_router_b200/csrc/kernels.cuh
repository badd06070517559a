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
};

// ---- router (router.cu) ----------------------------------------------------
// Pass over Q, K (and V): pooled Q (fp32), exact fp64 column sums per key block,
// optional INT8 Q-hat + s_q, optional per-channel |V| max (atomic, as uint bits).
cudaError_t launch_pool(const Shape& s, const void* q, const void* k, const void* v, float* qbar, double* ksum,
                        int8_t* qhat, float* sq, unsigned* vamax, cudaStream_t st);
// colmean (fp64 and fp32) from the per-block sums, and the smoothed pooled keys.
cudaError_t launch_colmean(const Shape& s, const double* ksum, double* c64, float* c32, float* kbar_s,
                           cudaStream_t st);
// A = Qbar Wq, Bk = (Kbar - c) Wk, fp32.
cudaError_t launch_proj(const Shape& s, int H, const float* qbar, const float* kbar_s, const float* wq,
                        const float* wk, float* A, float* Bk, cudaStream_t st);
// logits s = A Bk^T / sqrt(d), fp32 [BH][nq][nk]
cudaError_t launch_scores(const Shape& s, const float* A, const float* Bk, float* scores, cudaStream_t st);
// hard top-k per logit row (ties -> lower index), mask and ascending index list
cudaError_t launch_topk(const Shape& s, const float* scores, uint8_t* mask, int32_t* idx, cudaStream_t st);
int scores_topk_max_nk();

// ---- linear state (linear.cu) ---------------------------------------------
// Per key block: h_j, z_j (fp32) and per-chunk partial sums; optionally K-hat /
// s_k and V-hat^T / s_v (quant = 1: e4m3; quant = 0: bf16 copy of V^T).
struct LinearOut {
  void* h;           // h_j^T [BH][nk][d (channel c)][d (feature e)]: h_mode 0 fp32, 1 bf16
  int h_mode;        // partial sums (and so H_total) are always written transposed too
  float* z;          // [BH][nk][d]
  float* hpart;      // [BH][G][d][d]
  float* zpart;      // [BH][G][d]
  int8_t* khat;      // [BH][N][d] or nullptr
  float* sk;         // [BH][nk]
  void* vhatT;       // [BH][nk][d][64] (u8 e4m3 or bf16) or nullptr
  float* sv;         // [BH][d]
  const unsigned* vamax;  // [BH][d] (quant = 1)
  int quant;
  unsigned* status;
  unsigned long long budget_ns;
};
// number of key-block chunks (CTAs) per head of the linear-state pass
int linear_chunks(int BH, int nk);
cudaError_t launch_linear_state(const Shape& s, const void* k, const void* v, const float* c32, const LinearOut& o,
                                cudaStream_t st);
cudaError_t launch_linear_reduce(const Shape& s, const float* hpart, const float* zpart, float* Htot, float* Ztot,
                                 float* zscale, cudaStream_t st);

// ---- sparse branch (sparse.cu) --------------------------------------------
struct SparseArgs {
  const int32_t* idx;   // [BH][nq][k]
  const float* sq;      // [BH][nq]   (quant)
  const float* sk;      // [BH][nk]   (quant)
  const float* sv;      // [BH][d]    (quant)
  float* os;            // [BH][N][d] fp32 out
  unsigned* status;
  unsigned long long budget_ns;
};
// tensor maps are built by the caller (api.cu) and passed by value
cudaError_t launch_sparse(const Shape& s, int quant, const CUtensorMap& tq, const CUtensorMap& tk,
                          const CUtensorMap& tv, const SparseArgs& a, cudaStream_t st);
size_t sparse_smem_bytes(int d, int quant);

// ---- epilogue (epilogue.cu) -----------------------------------------------
struct EpilogueArgs {
  const void* q;        // bf16 [BH][N][d]
  const float* Htot;    // H_total^T [BH][d][d] (fp32)
  const float* Ztot;    // [BH][d]
  const float* zscale;  // [BH] power of two with Z_total * zscale <= 1
  const uint16_t* hT;   // h_j^T bf16 [BH][nk][d][d]
  const float* z;       // [BH][nk][d]
  const int32_t* idx;   // [BH][nq][k]
  const float* os;      // [BH][N][d]
  const float* alpha;   // [H][nq]
  int H;
  void* out;            // [BH][N][d]
  int out_f32;
  float* ol_dbg;        // optional [BH][N][d]
  unsigned* status;
  unsigned long long budget_ns;
};
cudaError_t launch_epilogue(const Shape& s, const EpilogueArgs& a, const CUtensorMap& tq, cudaStream_t st);

}  // namespace sla2
