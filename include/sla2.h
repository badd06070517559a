/*
 * sla2.h -- C ABI of libsla2.so: the SLA2 sparse-linear attention inference
 * forward pass on NVIDIA B200 (sm_100a).
 *
 * The operation (sources: the SLA2 summary page at paper.rainbus.top, first
 * paragraph, steps 1-4; the SLA2 detail page at zhaifeiyue.github.io, §3
 * flowchart, §4 symbol table, §7 implementation notes):
 *
 *   K_s  = K - colmean(K)                                    (detail §7, note 1)
 *   Qbar = mean-pool(Q, 128 tokens), Kbar = mean-pool(K_s, 64 tokens)
 *   s    = (Qbar Wq)(Kbar Wk)^T / sqrt(d); M_c = hard top-k per row      (step 1)
 *   O_s  = softmax attention over the selected blocks, INT8 Q/K, FP8 P/V (step 2)
 *   O_l  = phi(Q_i) H_i / (phi(Q_i) Z_i), H_i, Z_i over unselected blocks (step 3)
 *   O    = alpha * O_s + (1 - alpha) * O_l                               (step 4)
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     never allocates, frees or synchronises. Scratch memory is the caller's
 *     workspace (see sla2_workspace_size).
 *   - Q, K, V, out: contiguous [B][H][N][d]; Q/K/V bf16; out bf16 or fp32.
 *     proj_q, proj_k: fp32 [H][d][d], applied as y = x W (row vector times W,
 *     W stored [d_in][d_out]). alpha: fp32 [H][N/128], shared over the batch,
 *     used as given (expected in [0, 1]).
 *   - Shapes: N % 128 == 0, d in {64, 128}, B, H >= 1. Every base pointer must
 *     be 16-byte aligned. out must not alias an input.
 *   - k (key blocks kept per query block) = clamp(floor(frac * nk + 1e-3), 1, nk)
 *     with nk = N / 64; frac must lie in (0, 1].
 *   - Calls enqueue on `stream` (a cudaStream_t; NULL = legacy default stream)
 *     and return. SLA2_OK means "arguments valid and kernels enqueued".
 *     Arguments are checked before any launch; on an argument error nothing is
 *     written. Launch failures return SLA2_ERR_CUDA.
 *   - A workspace may be reused by back-to-back calls on one stream; calls that
 *     may run concurrently need separate workspaces.
 *   - Device-side waits are bounded; a wait that runs out writes a nonzero code
 *     into the optional status word (desc.status) and the kernel returns.
 *   - The library keeps per-device state for the life of the process (the
 *     auxiliary stream of sla2_forward, the device address of the fixed array
 *     of sla2_router_noalloc). Do not keep using the library on a device after
 *     cudaDeviceReset on it: that state would refer to the destroyed context.
 */
#ifndef SLA2_H
#define SLA2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SLA2_OK = 0,
  SLA2_ERR_INVALID_ARG = 1,    /* NULL pointer, bad size, frac outside (0,1], misalignment */
  SLA2_ERR_UNSUPPORTED = 2,    /* N % 128 != 0 or d not in {64, 128} */
  SLA2_ERR_WORKSPACE = 3,      /* workspace NULL or smaller than sla2_workspace_size() */
  SLA2_ERR_CUDA = 4,           /* a CUDA runtime / driver call failed */
  SLA2_ERR_DEVICE_TIMEOUT = 5  /* reported through the status word, after a sync */
} sla2_status;

/* Problem description shared by all entry points. */
typedef struct {
  int B, H, N, d;
  int quantize;        /* 1: INT8 Q/K + FP8 e4m3 P/V sparse branch (default);
                          0: bf16 tensor-core sparse branch (no quantisation)   */
  int out_dtype;       /* 0: bf16 output, 1: fp32 output                        */
  void* workspace;     /* device scratch, >= sla2_workspace_size() bytes,
                          256-byte aligned                                      */
  size_t workspace_bytes;
  unsigned int* status;/* optional device word; every entry point clears it on
                          `stream` before its first launch, and a bounded
                          device wait that runs out sets it to
                          SLA2_ERR_DEVICE_TIMEOUT                               */
  /* Optional debug exports (NULL = not written), all device pointers:        */
  float* dbg_scores;   /* router logits s, fp32 [B][H][N/128][N/64]            */
  float* dbg_os;       /* sparse branch O_s, fp32 [B][H][N][d]                 */
  float* dbg_ol;       /* linear branch O_l, fp32 [B][H][N][d]                 */
  int8_t* dbg_qhat;    /* INT8 Q-hat [B][H][N][d]  (quantize = 1 only)          */
  int8_t* dbg_khat;    /* INT8 K-hat of K_s [B][H][N][d]                        */
  uint8_t* dbg_vhat;   /* e4m3 V-hat codes in the layout the sparse kernel reads:
                          per key block, channel-major [B][H][N/64][d][64]     */
  float* dbg_qscale;   /* s_q [B][H][N/128]                                     */
  float* dbg_kscale;   /* s_k [B][H][N/64]                                      */
  float* dbg_vscale;   /* s_v [B][H][d]                                         */
  uint8_t* dbg_mask;   /* M_c [B][H][N/128][N/64]                               */
  int32_t* dbg_idx;    /* selected block indices, ascending, [B][H][N/128][k]   */
  /* Optional timing hooks: NULL, or an array of SLA2_STAGE_EVENTS cudaEvent_t
     that sla2_forward records on `stream` at the stage boundaries
     [start, pass over Q/K/V and column means done, linear state and router
     tail (projections, logits, top-k; run concurrently) done, sparse branch
     done, end].                                                             */
  void* const* stage_events;
} sla2_desc;

#define SLA2_STAGE_EVENTS 5

/* Human-readable name of a status code (static string, never NULL). */
const char* sla2_status_string(sla2_status s);

/* k for a given key-block count and fraction (see conventions); 0 if frac is
 * outside (0, 1] or nk < 1. Host-only, no CUDA call. */
int sla2_topk_count(int nk, float topk_frac);

/* Bytes of device workspace sla2_forward needs for this description and
 * fraction; 0 if the description is invalid. Host-only, no CUDA call. */
size_t sla2_workspace_size(const sla2_desc* desc, float topk_frac);

/* Steps 1 (and K smoothing) only: the learnable router.
 *   q, k      : bf16 [B][H][N][d]
 *   proj_q/k  : fp32 [H][d][d]
 *   mask_out  : uint8 [B][H][N/128][N/64], M_c (1 = selected)
 *   idx_out   : int32 [B][H][N/128][k], selected key blocks in ascending order
 *   colmean_out: fp32 [B][H][d] (the K smoothing mean, rounded to fp32) or NULL
 * Uses desc->workspace (sla2_workspace_size bytes suffice); desc->dbg_scores
 * receives the fp32 logits when non-NULL. Top-k ties go to the lower index.
 * (Summary page, step 1; detail page §3 "Learnable Router".) */
sla2_status sla2_router(const sla2_desc* desc, const void* q, const void* k,
                        const float* proj_q, const float* proj_k, float topk_frac,
                        uint8_t* mask_out, int32_t* idx_out, float* colmean_out,
                        void* stream);

/* SoftTop-k relaxation of the router's mask (detail page §4, Eq. 17; the
 * training-time mask of summary step 1):
 *   soft_out[b][h][i][j] = sigmoid(P_c[i][j] / tau + lambda_i),  fp32 [B][H][N/128][N/64]
 *   lambda_out[b][h][i]  = lambda_i (fp32 [B][H][N/128]) or NULL
 * P_c is the row softmax of the router logits of sla2_router; lambda_i is found
 * by bisection so that every row sums to k, the number of blocks the hard
 * Top-k keeps (k = nk gives all ones and lambda = +inf). tau must be positive
 * and finite (the pages use 0.1); otherwise SLA2_ERR_INVALID_ARG. Uses
 * desc->workspace; desc->dbg_scores receives the logits when non-NULL. */
sla2_status sla2_router_soft(const sla2_desc* desc, const void* q, const void* k, const float* proj_q,
                             const float* proj_k, float topk_frac, float tau, float* soft_out,
                             float* lambda_out, void* stream);

/* The router of sla2_router, for callers that cannot allocate device memory
 * (no counterpart on the SLA2 pages; an addition of this library). Some
 * callers may not call cudaMalloc at all: a plugin inside a host framework
 * that owns every device allocation (for instance a serving runtime with a
 * pre-sized memory pool), or code on a latency-critical path where an
 * allocation, which can synchronise the device, is not allowed. This entry
 * point allocates nothing: its scratch is a fixed device array of
 * SLA2_ROUTER_NOALLOC_SCRATCH_BYTES compiled into libsla2.so, which every GPU
 * that loads the library holds until the process exits.
 *   - Arguments and outputs are those of sla2_router; desc->workspace is
 *     ignored (desc->dbg_scores is honoured).
 *   - Shapes whose router scratch exceeds the array are rejected with
 *     SLA2_ERR_WORKSPACE before anything is launched. The scratch is about
 *     (5/16) N d + N^2 / 2048 bytes per (batch, head): 1.84 MB for N = 32768,
 *     d = 128, so up to 9 such heads fit in one call.
 *   - desc->status is honoured as in sla2_router (cleared, then set if a
 *     bounded device wait runs out), and so is sla2_set_wait_budget_ns.
 *   - The first call on each device looks up the array's device address with
 *     cudaGetSymbolAddress while that device is current; make that first call
 *     before any stream capture.
 *   - All calls share the one array and it keeps the last call's contents
 *     (nothing in it has to start at zero). Calls whose kernels may overlap on
 *     the GPU (other streams, other host threads) race on it: serialise them. */
#define SLA2_ROUTER_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
sla2_status sla2_router_noalloc(const sla2_desc* desc, const void* q, const void* k,
                                const float* proj_q, const float* proj_k, float topk_frac,
                                uint8_t* mask_out, int32_t* idx_out, float* colmean_out,
                                void* stream);

/* Step 3's per-key-block linear-attention state (detail page §7, note 2:
 * h_j precomputed per key block, then accumulated):
 *   phi(x) = softmax over the d features; K_s = K - colmean (fp32)
 *   h_out    : fp32 [B][H][N/64][d][d], TRANSPOSED: h_out[..][j][c][e] =
 *              sum over the block's tokens t of V[t][c] * phi(K_s[t])[e]
 *              (= (phi(K_s,j)^T V_j)^T; tensor-core products with fp16
 *              operands, fp32 accumulation)
 *   z_out    : fp32 [B][H][N/64][d],    z_j = column sums of phi(K_s,j)
 *   Htot_out : fp32 [B][H][d][d] = sum_j h_out[j] (same transposed layout)
 *   Ztot_out : fp32 [B][H][d] = sum_j z_j
 *   colmean  : fp32 [B][H][d] as returned by sla2_router.
 * Uses desc->workspace for the per-chunk partial sums. */
sla2_status sla2_linear_state(const sla2_desc* desc, const void* k, const void* v,
                              const float* colmean, float* h_out, float* z_out,
                              float* Htot_out, float* Ztot_out, void* stream);

/* The whole forward pass (steps 1-4): out = alpha O_s + (1 - alpha) O_l.
 *   out : bf16 or fp32 (desc->out_dtype) [B][H][N][d]
 * All intermediates live in desc->workspace; optional debug exports in desc.
 * The linear-state pass runs on a library-owned non-blocking stream, forked
 * from and joined back into `stream` with events, concurrently with the
 * router's projections, logits and top-k on `stream`; the selected-state product
 * (H_i, Z_i of every query block) runs on it too, beside the sparse branch. That
 * stream and its two events are created by the first call on each device and
 * kept until the process exits;
 * make that first call outside any stream capture. Later calls can be captured
 * (the fork and join become graph edges). Calls from several host threads are
 * serialised while they enqueue.
 * Arithmetic: router in fp32; sparse branch INT8 Q K^T (int32 accumulate) and
 * e4m3 P V (fp32 accumulate) with quantize = 1, bf16 operands with quantize = 0;
 * linear branch on fp16 tensor-core operands with fp32 accumulation, h_j and
 * H_total scaled per head by a power of two derived from max|V| (V magnitudes
 * up to about 1e30 stay in range). */
sla2_status sla2_forward(const sla2_desc* desc, const void* q, const void* k, const void* v,
                         const float* proj_q, const float* proj_k, const float* alpha,
                         float topk_frac, void* out, void* stream);

/* Backward pass (detail page §7 note 3: the hand-derived gradient with the
 * linear branch's dH_i and dZ_i formed once per query block; §2 table: the
 * backward runs at higher precision than the INT8/FP8 forward kernels). It is
 * the gradient of the UNQUANTISED forward O = alpha O_s + (1 - alpha) O_l for
 * the mask the router selects for these inputs, held fixed (the hard Top-k is
 * piecewise constant, so proj_q and proj_k receive no gradient on this path),
 * with K smoothing included.
 *   q, k, v     : bf16 [B][H][N][d] (the forward's inputs); proj_q/proj_k,
 *                 alpha, topk_frac as for sla2_forward
 *   dout        : fp32 [B][H][N][d], dL/dO
 *   dq, dk, dv  : fp32 [B][H][N][d], written (not accumulated)
 *   dalpha      : fp32 [H][N/128], dL/dalpha summed over the batch (alpha is
 *                 shared over the batch), written
 * Arithmetic: fp32 on the CUDA cores; the per-key-block states h_j come from
 * the linear-state pass (fp16 tensor-core operands, fp32 accumulation).
 * Workspace: sla2_backward_workspace_size bytes; desc->quantize, out_dtype and
 * the debug exports are ignored. */
size_t sla2_backward_workspace_size(const sla2_desc* desc, float topk_frac);
sla2_status sla2_backward(const sla2_desc* desc, const void* q, const void* k, const void* v, const float* proj_q,
                          const float* proj_k, const float* alpha, float topk_frac, const float* dout, float* dq,
                          float* dk, float* dv, float* dalpha, void* stream);

/* The whole forward pass from HOST memory to HOST memory, with the copies
 * overlapped with the computation. Heads are taken in groups of
 * `heads_per_group` (per batch index, the last group of each batch index may
 * be smaller): group g's Q, K and V are copied in on a library-owned stream
 * while group g - 1 is computed on `stream` and group g - 2's output is copied
 * out on another library-owned stream, through two device slots of the
 * workspace. Each group is computed as sla2_forward_heads computes it, so the
 * output is bit-identical to sla2_forward's for the same description.
 *   q, k, v       : HOST bf16 [B][H][N][d]
 *   proj_q, proj_k: HOST fp32 [H][d][d];  alpha: HOST fp32 [H][N/128]
 *   out           : HOST bf16 or fp32 (desc->out_dtype) [B][H][N][d]
 *   desc->workspace : DEVICE memory of sla2_forward_host_workspace_size bytes
 *                   (the per-group forward workspace, the projections and
 *                   alpha, and the two slots of group inputs and outputs)
 *   1 <= heads_per_group <= H; desc's debug exports and stage_events must be
 *   NULL (else SLA2_ERR_INVALID_ARG).
 * Returns once everything is enqueued; out is complete when `stream` has
 * reached that point (the call makes `stream` wait for the last copy out), and
 * the host buffers must stay valid until then. Page-locked host memory lets
 * the copies run asynchronously and concurrently; with pageable memory the
 * result is the same but the copies serialise with the host. The copy streams
 * and their events are created by the first call on each device and kept until
 * the process exits; calls from several host threads are serialised while they
 * enqueue. */
size_t sla2_forward_host_workspace_size(const sla2_desc* desc, int heads_per_group, float topk_frac);
sla2_status sla2_forward_host(const sla2_desc* desc, int heads_per_group, const void* q, const void* k,
                              const void* v, const float* proj_q, const float* proj_k, const float* alpha,
                              float topk_frac, void* out, void* stream);

/* One rank's share of a head-sharded forward pass (the summary page's
 * future-work paragraph names multi-GPU execution; every step of the pass is
 * independent per (batch, head), so a contiguous range of heads per GPU needs
 * no collective).
 *   desc  : the FULL problem (B, H, N, d, quantize, out_dtype, workspace, status);
 *           its debug exports and stage_events must be NULL (else
 *           SLA2_ERR_INVALID_ARG).
 *   q, k, v, out : the full [B][H][N][d] tensors; proj_q/proj_k: the full
 *           [H][d][d]; alpha: the full [H][N/128].
 *   Computes out[b][h] for every b and every h in [h_begin, h_begin + h_count)
 *   and writes nothing else of out. Those heads are bit-identical to the ones
 *   sla2_forward writes for the same full description (the linear state's
 *   chunking, which fixes its summation order, is taken from all B x H heads).
 *   Workspace: sla2_workspace_size_heads(desc, h_count, frac) bytes, reused for
 *   each batch index in turn (one pass of the forward per batch index, in
 *   order, on `stream`). 0 <= h_begin, 1 <= h_count, h_begin + h_count <= H. */
size_t sla2_workspace_size_heads(const sla2_desc* desc, int h_count, float topk_frac);
sla2_status sla2_forward_heads(const sla2_desc* desc, int h_begin, int h_count, const void* q, const void* k,
                               const void* v, const float* proj_q, const float* proj_k, const float* alpha,
                               float topk_frac, void* out, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* SLA2_H */
