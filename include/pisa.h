/*
 * pisa.h -- C ABI of libpisa: PISA piecewise sparse attention (forward) on
 * NVIDIA B200 (sm_100a).
 *
 * The method ("PISA: Piecewise Sparse Attention Is Wiser for Efficient
 * Diffusion Transformers"; the gist.science "Technical Summary", section 2
 * "Methodology"): every query block i attends exactly to its selected key/value
 * blocks S_i, and every unselected block j in U_i enters the same softmax
 * numerator N_t and denominator D_t through a block-wise zeroth-order Taylor
 * term (block centroid kbar_j, value sum SigmaV_j) plus, in the paper ("hyd")
 * variant, one shared global first-order correction Hbar, the mean of the
 * block first-order matrices.  o_t = N_t / D_t.
 *
 * Conventions shared by every call:
 *  - Tensors are dense row-major.  Q, K, V and the output are [B, H, L, d]
 *    (token rows of d elements, heads and batches outermost).  Statistics are
 *    float32: qbar/kbar/vsum [B, H, N, d], hbar [B, H, d, d], cov [B, H, N].
 *    Selected block indices are int32 [B, H, N, k_sel], ascending per row.
 *    N = ceil(L / block_size); only the last block may be partial.
 *  - Every pointer argument is a DEVICE pointer owned by the caller, except
 *    where stated.  The library keeps no pointer after a call returns.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream) and performs no host synchronisation, except
 *    pisa_device_status.
 *  - Arguments are validated on the host before anything is launched.  A
 *    failed check returns PISA_ERR_INVALID_ARG or PISA_ERR_UNSUPPORTED and
 *    launches nothing.  A failed launch returns PISA_ERR_CUDA.  Errors found
 *    by the kernels themselves (an index out of range, a bounded wait that ran
 *    out) are recorded in a device status word that pisa_device_status reads.
 *  - Supported now: d in {64, 128}; block_size 64 or 128 (the block-wise
 *    first-order mode and the score histogram: 64 only; the authors' README
 *    uses 64, the skill page gives 64-128); dtype bf16 or f32 (f32
 *    inputs are rounded to bf16 for the tensor-core products; statistics are
 *    accumulated in float32 from the inputs as given); all data pointers
 *    16-byte aligned.
 *  - There is no CPU fallback: every step runs in this library's CUDA kernels.
 *
 * Softmax scale: s multiplies every q.k product (exact logits, centroid
 * logits, selection scores and the first-order term s q Hbar); 0 selects the
 * default 1/sqrt(d).
 */
#ifndef PISA_H
#define PISA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *pisa_stream_t; /* identical to cudaStream_t */

typedef enum {
  PISA_OK = 0,
  PISA_ERR_INVALID_ARG = 1, /* bad shape, pointer, alignment or option */
  PISA_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. d = 96) */
  PISA_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
  PISA_ERR_WORKSPACE = 4,   /* caller workspace too small */
  PISA_ERR_TIMEOUT = 5,     /* a kernel's bounded wait ran out (device word) */
  PISA_ERR_DEVICE = 6       /* a kernel's range check failed (device word) */
} pisa_status;

typedef enum {
  PISA_MODE_HYD = 0, /* zeroth-order tail + global first-order term ("_hyd") */
  PISA_MODE_0TH = 1, /* zeroth-order tail only ("_0th") */
  PISA_MODE_1ST = 2  /* block-wise first order: every unselected block j adds
                        alpha_tj (s q_t H_j) with its own H_j (the gist.science
                        summary, "Global First-Order Correction": the per-block
                        alternative to Hbar; atlas.scime.ai "Surprising findings":
                        the "first-order-only" ablation).  Work equals dense
                        attention: every K/V block is read. */
} pisa_mode;

typedef enum { PISA_BF16 = 0, PISA_F32 = 1 } pisa_dtype;

/* sink_idx values: the authors' README, "Attention sink for MMDiT": 0 or -1
 * force the first or the last K/V block into the exact set of every query
 * block; PISA_SINK_NONE forces nothing. */
#define PISA_SINK_NONE INT32_MIN

/* Options of pisa_attention_ex.  Zero-initialise, then set what you need. */
typedef struct {
  float scale;        /* softmax scale s; 0 = 1/sqrt(d) */
  float cov_weight;   /* lambda of covariance-aware scoring; 0 = off */
  pisa_dtype dtype;   /* dtype of q, k, v and out */
  void *workspace;    /* device scratch; NULL = allocate per call (stream-ordered) */
  size_t ws_bytes;    /* size of `workspace` */
  int fuse_select;    /* block_size 128 only (else PISA_ERR_UNSUPPORTED): no
                         separate selection step; each CTA of the fused kernel,
                         which holds one query block, scores that block against
                         every centroid and takes its own top k_sel (the same
                         float32 scores, tie rule and sink as pisa_select, so
                         the same sets) before its exact tiles start */
  int32_t *idx_out;   /* optional (NULL = not wanted): device [B,H,N,k_sel] int32,
                         4-byte aligned, receives the selection the call used */
} pisa_options;

/* ---- sizes ------------------------------------------------------------- */

/* N = ceil(L / block_size); -1 on invalid arguments. */
int pisa_num_blocks(int L, int block_size);

/* Exact blocks per query block: density is the fraction of K/V blocks kept
 * exact (the authors' README `density`; 0.15 is "85% sparsity").
 * k_sel = clamp(floor(density * N + 1e-6), 1, N), computed in double; the sink
 * block counts inside k_sel.  -1 on invalid arguments. */
int pisa_num_selected(int N, double density);

/* Workspace bytes that pisa_attention_ex needs for these arguments (the sum
 * of the three calls' needs below, plus bf16 copies for f32 inputs). */
size_t pisa_workspace_bytes(int B, int H, int L, int d, int block_size,
                            double density, pisa_dtype dtype, int want_cov);
size_t pisa_block_stats_workspace_bytes(int B, int H, int L, int d, int block_size);
size_t pisa_select_workspace_bytes(int B, int H, int N);
size_t pisa_sparse_attention_workspace_bytes(int B, int H, int L, int d, int block_size,
                                             pisa_dtype dtype);

/* ---- the three steps of the path -------------------------------------- */

/* Block statistics (gist.science summary, "Hardware Implementation" step 1,
 * "Core Algorithm", "Global First-Order Correction", "Covariance-Aware
 * Routing"):
 *   qbar_i = mean query of block i            [B,H,N,d]
 *   kbar_j = mean key of block j (centroid)   [B,H,N,d]
 *   vsum_j = sum of the values of block j     [B,H,N,d]
 *   hbar   = (1/N) sum_j H_j, H_j = sum_n (k_{j,n} - kbar_j)^T v_{j,n}  [B,H,d,d]
 *   cov_j  = || H_j - hbar ||_F               [B,H,N]   (only if want_cov;
 *                                                         cov may be NULL otherwise)
 * q, k, v: [B,H,L,d] in `dtype`.  All outputs float32.  `workspace` must
 * hold pisa_block_stats_workspace_bytes(...) bytes (deterministic partial
 * sums; no atomics, so results are bitwise reproducible). */
pisa_status pisa_block_stats(const void *q, const void *k, const void *v, pisa_dtype dtype,
                             int B, int H, int L, int d, int block_size, int want_cov,
                             float *qbar, float *kbar, float *vsum, float *hbar, float *cov,
                             void *workspace, size_t ws_bytes, pisa_stream_t stream);

/* Covariance-aware top-k routing with sink forcing (gist.science summary,
 * "Covariance-Aware Routing"; authors' README "Attention sink for MMDiT"):
 *   score_ij = scale * qbar_i . kbar_j + cov_weight * cov_j   (float32)
 * keeps, per query block i, the k_sel = pisa_num_selected(N, density) highest
 * scores, ties going to the lower block index; with sink_idx 0 / -1 the block
 * 0 / N-1 is always kept and the other k_sel-1 are the best of the rest.
 * idx [B,H,N,k_sel] int32, each row ascending.  cov may be NULL when
 * cov_weight == 0.  `workspace`: pisa_select_workspace_bytes(B,H,N) bytes.
 * The scores are formed to float32 accuracy: with a float32 FMA chain over d
 * for N <= 512, and on the tensor cores from three-part bf16 splits of qbar
 * and kbar (six cross products) for longer rows.  Two blocks whose scores
 * agree to float32 rounding may therefore be ordered differently from an
 * fp64 evaluation; exact float32 ties go to the lower index. */
pisa_status pisa_select(const float *qbar, const float *kbar, const float *cov,
                        float cov_weight, float scale, int B, int H, int N, int d,
                        double density, int sink_idx, int32_t *idx,
                        void *workspace, size_t ws_bytes, pisa_stream_t stream);

/* Fused exact-or-approximate attention (gist.science summary, "Core
 * Algorithm" numerator equation and "Hardware Implementation" phases 1-3): for
 * token t of query block i,
 *   D_t = sum_{j in S_i} sum_n e^{s q_t k_{j,n}} + sum_{j in U_i} n_j alpha_tj
 *   N_t = sum_{j in S_i} sum_n e^{s q_t k_{j,n}} v_{j,n} + sum_{j in U_i} alpha_tj vsum_j
 *         + [hyd] (s q_t hbar) sum_{j in U_i} alpha_tj,     alpha_tj = e^{s q_t kbar_j}
 *         + [1st] sum_{j in U_i} alpha_tj (s q_t H_j)  (computed per token as
 *           sum_n alpha_tj (s q_t k_{j,n} - s q_t kbar_j) v_{j,n}; hbar unused)
 *   out_t = N_t / D_t
 * with S_i = idx row i (k_sel ascending, distinct indices < N) and U_i its
 * complement.  kbar, vsum, hbar as written by pisa_block_stats.  out
 * [B,H,L,d] in `dtype`; it must not overlap any input.  `workspace`:
 * pisa_sparse_attention_workspace_bytes(...) bytes. */
pisa_status pisa_sparse_attention(const void *q, const void *k, const void *v,
                                  pisa_dtype dtype, const float *kbar, const float *vsum,
                                  const float *hbar, const int32_t *idx, int k_sel,
                                  int B, int H, int L, int d, int block_size, float scale,
                                  pisa_mode mode, void *out, void *workspace,
                                  size_t ws_bytes, pisa_stream_t stream);

/* pisa_sparse_attention that also writes lse [B,H,L] float32 (4-byte
 * aligned): lse_t = ln D_t, the natural log of the denominator above (the
 * same in modes hyd and 0th, which differ only in the numerator).  It is what
 * pisa_sparse_attention_bwd needs from the forward.  out_f32 (may be NULL;
 * else 16-byte aligned, [B,H,L,d], overlapping neither out nor an input)
 * receives the output in float32, before its rounding to `dtype`; given to
 * pisa_sparse_attention_bwd it saves the backward one sweep.  With out_f32
 * the denominator D_t (and so out and lse) is the sum of the same
 * bf16-rounded weights the numerator uses: out then differs from the call
 * without out_f32 at the bf16 rounding level, and dout_t . out_t matches the
 * backward's probabilities even when one key holds nearly all the weight. */
pisa_status pisa_sparse_attention_fwd(const void *q, const void *k, const void *v,
                                      pisa_dtype dtype, const float *kbar, const float *vsum,
                                      const float *hbar, const int32_t *idx, int k_sel, int B,
                                      int H, int L, int d, int block_size, float scale,
                                      pisa_mode mode, void *out, float *lse, float *out_f32,
                                      void *workspace, size_t ws_bytes, pisa_stream_t stream);

/* ---- training: gradients of the zeroth-order variant ------------------------ */

/* Workspace bytes of pisa_sparse_attention_bwd for k_sel selected blocks per
 * query block (0 on invalid arguments). */
size_t pisa_sparse_attention_bwd_workspace_bytes(int B, int H, int L, int d, int block_size,
                                                 int k_sel);

/* Gradients of the zeroth-order forward (the authors' README, "Kernel
 * variants": piecewise_sparse_attention_0th is the variant meant for training;
 * the forward is the equation above without the hyd term).  Given dout = dL/d out, writes
 *   dq = dL/dq,  dk = dL/dk,  dv = dL/dv        bf16 [B,H,L,d]
 * with the selection idx held fixed (a discrete step) and the statistics
 * differentiated: kbar_j is the mean key and vsum_j the value sum of block j,
 * so each tail term's gradient reaches every key and value of block j.
 * q, k, v, dout: bf16 [B,H,L,d]; lse from pisa_sparse_attention_fwd on the
 * same q, k, v, kbar, vsum, idx; kbar, vsum: float32 from pisa_block_stats.
 * The row term Delta_t = sum_m P_tm (dout_t . value_m) equals dout_t . out_t.
 * With out_f32 (the forward's float32 output, 16-byte aligned) it is formed
 * that way; with out_f32 NULL it is formed from the recomputed probabilities
 * in an extra sweep over the tiles.  The bf16 output alone is not enough:
 * its rounding, amplified by the cancellation in P (dP - Delta), can move dq
 * by several per cent on short sequences.  dq, dk, dv must not overlap any
 * input or one another.  No atomics: bitwise reproducible.
 * `workspace`: pisa_sparse_attention_bwd_workspace_bytes(...) bytes.
 * With out_f32, part of the work (the centroid gradients and the key-block
 * lists, which need nothing from dq) runs beside dq on a second stream that
 * the library keeps per calling thread and device; it starts after the work
 * already on `stream` and `stream` waits for it before the call's last
 * kernel, so to the caller every effect is ordered on `stream` (also under
 * stream capture), whatever the call returns. */
pisa_status pisa_sparse_attention_bwd(const void *q, const void *k, const void *v,
                                      const void *dout, const float *lse, const float *out_f32,
                                      const float *kbar, const float *vsum, const int32_t *idx,
                                      int k_sel, int B, int H, int L, int d, int block_size,
                                      float scale, void *dq, void *dk, void *dv, void *workspace,
                                      size_t ws_bytes, pisa_stream_t stream);

/* ---- diagnostic ------------------------------------------------------------ */

/* Distributional stability of the non-critical blocks (gist.science summary,
 * section 2 "Key Insights" 1: their pre-softmax scores are bell-shaped and
 * centred at or below zero, which is why their Taylor approximation is
 * accurate).  For every token t of the query blocks i = 0, query_stride,
 * 2 query_stride, ..., every unselected block j in U_i (idx row i gives S_i) and
 * every key n of block j:
 *   x = s q_t k_n               pre-softmax score
 *   y = s q_t (k_n - kbar_j)    the variable of block j's Taylor expansion
 * hist_x / hist_y (nbins + 2 counts each, device, zeroed here): [0] values
 * below lo, [1 .. nbins] the equal bins of [lo, hi), [nbins + 1] values >= hi.
 * moments (5 doubles, device, zeroed here): count, sum x, sum x^2, sum y,
 * sum y^2.  bf16 q, k only; 1 <= nbins <= 4096.  Reads every key of every
 * unselected block of the sampled query blocks (dense-size work when
 * query_stride is 1). */
pisa_status pisa_tail_score_histogram(const void *q, const void *k, pisa_dtype dtype,
                                      const int32_t *idx, int k_sel, int B, int H, int L, int d,
                                      int block_size, float scale, float lo, float hi, int nbins,
                                      int query_stride, unsigned long long *hist_x,
                                      unsigned long long *hist_y, double *moments,
                                      pisa_stream_t stream);

/* ---- the whole path ----------------------------------------------------- */

/* The authors' `piecewise_sparse_attention_{hyd,0th}(q, k, v, density,
 * block_size, sink_idx)`: statistics -> selection -> fused attention, bf16
 * I/O, scale 1/sqrt(d), covariance weight 0.  Scratch memory is allocated and
 * freed stream-ordered (cudaMallocAsync / cudaFreeAsync) on `stream`. */
pisa_status pisa_attention(const void *q, const void *k, const void *v, void *out,
                           int B, int H, int L, int d, int block_size, double density,
                           int sink_idx, pisa_mode mode, pisa_stream_t stream);

/* pisa_attention with options (scale, covariance weight, f32 I/O, caller
 * workspace).  With opts->workspace non-NULL nothing is allocated; it must
 * hold pisa_workspace_bytes(...) bytes, else PISA_ERR_WORKSPACE.  opts may be
 * NULL (defaults). */
pisa_status pisa_attention_ex(const void *q, const void *k, const void *v, void *out,
                              int B, int H, int L, int d, int block_size, double density,
                              int sink_idx, pisa_mode mode, const pisa_options *opts,
                              pisa_stream_t stream);

/* Dense softmax attention out = softmax(s q k^T) v over all L keys, same
 * layout and dtypes: the dense baseline timed beside the sparse path. */
pisa_status pisa_dense_attention(const void *q, const void *k, const void *v, void *out,
                                 pisa_dtype dtype, int B, int H, int L, int d, float scale,
                                 void *workspace, size_t ws_bytes, pisa_stream_t stream);
size_t pisa_dense_attention_workspace_bytes(int B, int H, int L, int d, pisa_dtype dtype);

/* ---- block statistics without any allocation ----------------------------- */

/* Largest scratch, in bytes, that pisa_block_stats_noalloc can use. */
#define PISA_NOALLOC_SCRATCH_BYTES (32u << 20)

/* pisa_block_stats for callers that cannot allocate device memory.  The
 * paper has no counterpart: this is a packaging variant, not part of the
 * method.  Some hosts give a library only the buffers of one call and forbid
 * cudaMalloc (plugin interfaces of inference runtimes, frameworks whose own
 * allocator has reserved the device), and some loops cannot afford the device
 * synchronisation that cudaMalloc / cudaFree may cause.  Such callers cannot
 * provide the workspace that pisa_block_stats needs.
 *
 * This call computes exactly what pisa_block_stats computes (same kernels,
 * same reduction order, bitwise the same results), with the same argument
 * meaning, layout and ownership, but keeps its chunk partial sums in one
 * static device array of PISA_NOALLOC_SCRATCH_BYTES bytes inside libpisa.
 * Every GPU that loads the library holds that array until the process exits.
 *  - It allocates nothing and calls no allocating routine.
 *  - Shapes whose scratch need, pisa_block_stats_workspace_bytes(B, H, L, d,
 *    block_size), exceeds PISA_NOALLOC_SCRATCH_BYTES are rejected with
 *    PISA_ERR_WORKSPACE before anything is launched (pisa_last_error gives the
 *    sizes).  Example: the Wan2.1-like shape (B=1, H=40, L=75600, d=128)
 *    needs 20 MiB.
 *  - The first call on each device looks up that device's address of the
 *    array (cudaGetSymbolAddress) with the device current; make that first
 *    call before any stream capture begins on the device.  A context that
 *    replaces the device's context (after cudaDeviceReset, say) holds a fresh,
 *    zero-filled copy of the array at another address: the first call in it
 *    looks the address up again, so it too belongs before any capture.
 *  - All calls on a device share the one array, which keeps whatever the last
 *    call left there.  Nothing in it needs to start at zero: each call writes
 *    every partial it later reads.  Calls whose kernels may overlap on the GPU
 *    (different streams without ordering, or several host threads) race on
 *    the array and give wrong results; order them on one stream. */
pisa_status pisa_block_stats_noalloc(const void *q, const void *k, const void *v,
                                     pisa_dtype dtype, int B, int H, int L, int d,
                                     int block_size, int want_cov, float *qbar, float *kbar,
                                     float *vsum, float *hbar, float *cov,
                                     pisa_stream_t stream);

/* ---- errors -------------------------------------------------------------- */

/* Synchronises `stream`, then reads and clears the device status word set by
 * the kernels.  Returns PISA_OK, PISA_ERR_TIMEOUT, PISA_ERR_DEVICE, or
 * PISA_ERR_CUDA if the stream itself reported an error. */
pisa_status pisa_device_status(pisa_stream_t stream);

/* Self-test of the failure path (no counterpart in the paper).  Launches one
 * warp that waits, with the same bounded mbarrier wait every kernel of this
 * library uses, on a barrier that nothing ever completes, giving up after
 * limit_ns nanoseconds (1 .. 1e9).  The kernel then records PISA_ERR_TIMEOUT in
 * the device status word and returns, so a following pisa_device_status
 * reports PISA_ERR_TIMEOUT and the CUDA context stays usable.  No fault, trap
 * or unbounded spin is involved. */
pisa_status pisa_selftest_timeout(uint64_t limit_ns, pisa_stream_t stream);

/* Static description of a status code. */
const char *pisa_status_string(pisa_status s);

/* Text of the last CUDA error seen by this library on the calling thread
 * ("" if none). */
const char *pisa_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* PISA_H */
