/*
 * vsa.h -- C ABI of the content-adaptive block-sparse video attention library
 * (libvsa.so, hand-written CUDA for sm_100a).
 *
 * The method (NABLA: Neighborhood Adaptive Block-Level Attention, gist.science
 * summary of arXiv 2507.13546, "Methodology" items 1-3; the same top-p block
 * selection appears in Sparse VideoGen2, arXiv 2505.18875 summary, section 2B,
 * and in DynamicRad's dynamic-threshold mode, arXiv 2604.20470 summary,
 * section 2A) runs in five steps, one entry point each:
 *   1. vsa_fractal_flatten       reorder a T x H x W token grid so each P x P
 *                                spatial patch is a contiguous run of 64 tokens;
 *   2. vsa_pool_qk               mean-pool Q and K over those 64-token blocks;
 *   3.-4. vsa_block_mask         reduced softmax of pooled scores, per-row CDF
 *                                (top-p) selection, optional union with a
 *                                sliding-tile (STA) window, compacted to CSR;
 *   5. vsa_sparse_attn_fwd       attention forward over the kept 64 x 64 tiles,
 *                                returning O and the log-sum-exp;
 *   and vsa_fractal_unflatten    to bring O back to raster order.
 * Steps 1 and 5's unflattening can also be left to the attention's own
 * loads and stores: vsa_pool_qk_raster and vsa_sparse_attn_fwd_raster take
 * raster tensors and give the same results with no permuted copy written;
 * vsa_sparse_attn_fwd_to_raster takes flattened q, k, v and writes o and lse
 * in raster order.
 *
 * Conventions shared by every entry point
 *   - Pointers marked "device" are CUDA device pointers on the current device;
 *     the caller allocates and frees every buffer, the library allocates
 *     nothing.  Tensors are dense and contiguous, bf16 = IEEE bfloat16 stored
 *     as uint16, layout [B, heads, N, d] (d fastest).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call is
 *     asynchronous on that stream and never synchronises the host.
 *   - Arguments are validated on the host before anything is launched; a
 *     non-OK status means nothing was enqueued.  vsa_last_error() returns a
 *     message for the last non-OK status of the calling thread.
 *   - Kernels never trap.  A bounded device-side wait that gives up records a
 *     code in a per-device error word; vsa_device_status() synchronises the
 *     stream, reports and clears it.
 */
#ifndef VSA_H
#define VSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    VSA_OK = 0,
    VSA_ERR_INVALID_ARG = 1,     /* null pointer, negative size, thr outside [0,1) ... */
    VSA_ERR_UNSUPPORTED = 2,     /* valid but not implemented: d not 64/128, P*P != 64,
                                    H or W not a multiple of P, misaligned pointer */
    VSA_ERR_CAPACITY = 3,        /* an output or workspace buffer is too small */
    VSA_ERR_CUDA = 4,            /* a CUDA runtime call failed (message has the reason) */
    VSA_ERR_DEVICE_TIMEOUT = 5   /* a device-side wait gave up (see vsa_device_status) */
} vsa_status;

/* Token grid and head geometry.  N = T*H*W tokens per (batch, head);
 * blocks of P*P = 64 tokens; Nb = N/64 blocks per (batch, head). */
typedef struct {
    int32_t B, heads, T, H, W, d, P;
} vsa_shape;

/* Block-selection parameters.
 * thr     : CDF threshold in [0, 1).  Each row keeps the smallest set of its
 *           highest-probability blocks whose mass reaches 1 - thr (equal
 *           probabilities: lower block index first); thr = 0 keeps all blocks.
 * use_sta : non-zero to union the kept set with the STA window.
 * sta_t, sta_h, sta_w : STA radii in frames, patch rows and patch columns
 *           (Chebyshev window, clipped at the grid edges); >= 0. */
typedef struct {
    float thr;
    int32_t use_sta;
    int32_t sta_t, sta_h, sta_w;
} vsa_mask_params;

/* 1. Fractal flattening (NABLA, Methodology item 1).
 * y[b,h,f(n),:] = x[b,h,n,:] with raster n = (t*H + y)*W + x and
 * f(n) = t*H*W + ((y/P)*(W/P) + x/P)*P*P + (y%P)*P + x%P.
 * x, y : device bf16 [B,heads,N,d], must not overlap.  P must be 8. */
vsa_status vsa_fractal_flatten(const void *x, void *y, vsa_shape s, void *stream);

/* Inverse permutation: x[b,h,n,:] = y[b,h,f(n),:]. */
vsa_status vsa_fractal_unflatten(const void *y, void *x, vsa_shape s, void *stream);

/* 2. Block mean pooling (NABLA, Methodology item 2, "downsampling").
 * qp[b,h,r,:] = (1/64) * sum_{i<64} qf[b,h,64r+i,:], same for k.
 * qf, kf : device bf16 [B,heads,N,d] in flattened order.
 * qp, kp : device fp64 [B,heads,Nb,d].  A bf16 carries 8 significant bits,
 *          so the sum of 64 of them needs at most 14 + (exponent spread) bits:
 *          it is exact in fp64 whenever the block's nonzero magnitudes lie
 *          within a factor 2^39 of each other (data of one scale always do),
 *          and the division by 64 is exact, so each pooled value is then the
 *          exact block mean, independent of summation order.  Outside that
 *          range the result is within a few fp64 roundings of it. */
vsa_status vsa_pool_qk(const void *qf, const void *kf, double *qp, double *kp,
                       vsa_shape s, void *stream);

/* 1.+2. fused: fractal flattening of Q and K and their block means in one
 * pass (NABLA, Methodology items 1-2), so the flattened tensors are not read
 * back for pooling.  Results are bit-identical to
 *   vsa_fractal_flatten(q -> qf), vsa_fractal_flatten(k -> kf),
 *   vsa_pool_qk(qf, kf -> qp, kp).
 * q, k   : device bf16 [B,heads,N,d] in raster order (may alias each other).
 * qf, kf : device bf16 [B,heads,N,d], flattened order (outputs).
 * qp, kp : device fp64 [B,heads,Nb,d] (outputs).
 * No output may overlap an input or another output (VSA_ERR_INVALID_ARG). */
vsa_status vsa_flatten_pool_qk(const void *q, const void *k, void *qf, void *kf, double *qp,
                               double *kp, vsa_shape s, void *stream);

/* 1.+2. without the copies: the block means of the fractal blocks read
 * straight from raster Q and K (NABLA, Methodology items 1-2: block r of a
 * head is the P x P patch (r % (H/P*W/P)) of frame r / (H/P*W/P), patches
 * row-major).  Bit-identical to the qp, kp of vsa_flatten_pool_qk; for use
 * with vsa_sparse_attn_fwd_raster, which needs no flattened tensors.
 * q, k   : device bf16 [B,heads,N,d], raster order (may alias each other).
 * qp, kp : device fp64 [B,heads,Nb,d] (outputs); neither may overlap an input
 *          or the other (VSA_ERR_INVALID_ARG). */
vsa_status vsa_pool_qk_raster(const void *q, const void *k, double *qp, double *kp,
                              vsa_shape s, void *stream);

/* 3.-4. Block mask (NABLA, Methodology items 2-3).
 * For every (b, h) and query block r: A[r,:] = softmax(qp_r . kp_c / sqrt(d))
 * over the Nb key blocks c, CDF selection at thr, union with the STA window
 * when enabled, and the kept blocks listed in ascending order:
 *   row_ptr : device int64 [B*heads*Nb + 1]; row g = (b*heads + h)*Nb + r;
 *             row_ptr[0] = 0, row_ptr[g+1] - row_ptr[g] = kept count of row g.
 *   col_idx : device int32 [col_capacity]; key block indices within the head.
 *             col_capacity must be >= B*heads*Nb*Nb (the worst case), so no
 *             host read-back of the kept count is ever needed.
 *   kept_count : optional device int32 [B*heads*Nb] (may be NULL).
 *   workspace  : device scratch of at least vsa_block_mask_workspace_size(s)
 *                bytes, 256-byte aligned; its contents need no initialisation.
 * Scores come from exact integer tensor-core products of base-2^7 digits of
 * the fp64 means, with a proven bound on the dropped low-order products; a
 * row is decided on them only when that bound cannot change its kept set, and
 * is otherwise recomputed in fp64 (scores, softmax, sorted prefix mass).  The
 * kept sets therefore match an fp64 evaluation except where fp64 rounding
 * order itself decides (a cut mass within rounding of 1 - thr). */
size_t vsa_block_mask_workspace_size(vsa_shape s);
vsa_status vsa_block_mask(const double *qp, const double *kp, vsa_shape s,
                          vsa_mask_params p, int64_t *row_ptr, int32_t *col_idx,
                          int64_t col_capacity, int32_t *kept_count,
                          void *workspace, size_t workspace_bytes, void *stream);

/* Static-ratio block mask (DynamicRad, arXiv 2604.20470 summary, section 2,
 * "Dual-Mode Strategy", Static-Ratio mode: every row keeps a fixed share of
 * its blocks).  The page does not say which blocks; this call keeps each
 * row's k blocks of highest reduced-attention probability, ordered as in
 * vsa_block_mask (probability descending, equal probabilities to the lower
 * block index), then ORs in the STA window when p.use_sta is set (p.thr is
 * ignored).  k >= Nb keeps every block; k < 1 is VSA_ERR_INVALID_ARG.
 * Outputs, capacity, alignment and workspace (vsa_block_mask_workspace_size)
 * are those of vsa_block_mask.  Probabilities are fp32-accurate, so only rows
 * whose k-th and (k+1)-th probabilities lie within a relative 1e-5 (or below
 * 2^-120 of the row maximum) can differ from exact arithmetic. */
vsa_status vsa_block_mask_topk(const double *qp, const double *kp, vsa_shape s, int32_t k,
                               vsa_mask_params p, int64_t *row_ptr, int32_t *col_idx,
                               int64_t col_capacity, int32_t *kept_count, void *workspace,
                               size_t workspace_bytes, void *stream);

/* The STA window as the whole mask (NABLA, Methodology item 3, the sliding-
 * tile component M_STA alone; equally a static local-window mask): query block
 * (t, y, x) keeps the key blocks within Chebyshev radii (sta_t, sta_h, sta_w)
 * in (frame, patch row, patch column), clipped at the grid edges, ascending;
 * the same for every (b, h).  Needs no pooled tensors and no workspace.
 *   row_ptr : device int64 [B*heads*Nb + 1];  kept_count : optional int32.
 *   col_idx : device int32, col_capacity >= the window's total entry count
 *             (B*heads * sum_t w_t * sum_y w_y * sum_x w_x, w the clipped
 *             widths), else VSA_ERR_CAPACITY.  Negative radii are
 *             VSA_ERR_INVALID_ARG. */
vsa_status vsa_sta_mask(vsa_shape s, int32_t sta_t, int32_t sta_h, int32_t sta_w,
                        int64_t *row_ptr, int32_t *col_idx, int64_t col_capacity,
                        int32_t *kept_count, void *stream);

/* 5. Block-sparse attention forward (NABLA, Methodology item 2, "expansion":
 * the block mask decides which 64 x 64 tiles are computed; Sparse VideoGen2
 * section 2C: dense loads of contiguous query blocks, sparse loads of K/V).
 * For each query token of query block r of head (b,h), softmax attention over
 * the keys of blocks col_idx[row_ptr[g] .. row_ptr[g+1]), g = (b*heads+h)*Nb + r:
 *   O = sum_j softmax_j(scale * q . k_j) v_j,  LSE = ln sum_j exp(scale * q . k_j).
 * qf, kf, vf : device bf16 [B,heads,N,d], flattened order.
 * row_ptr, col_idx : as produced by vsa_block_mask (any valid CSR: columns
 *             strictly ascending and < Nb within each row).  An empty row
 *             gives O = 0 and LSE = -inf.
 * scale     : logit scale; <= 0 selects 1/sqrt(d).
 * o         : device bf16 [B,heads,N,d];  lse : device fp32 [B,heads,N].
 * workspace : device scratch of at least vsa_sparse_attn_workspace_size(s)
 *             bytes, 256-byte aligned (work list of the persistent scheduler). */
size_t vsa_sparse_attn_workspace_size(vsa_shape s);
vsa_status vsa_sparse_attn_fwd(const void *qf, const void *kf, const void *vf,
                               const int64_t *row_ptr, const int32_t *col_idx,
                               vsa_shape s, float scale, void *o, float *lse,
                               void *workspace, size_t workspace_bytes,
                               void *stream);

/* 5. with raster tensors: the same computation as vsa_sparse_attn_fwd, with
 * q, k, v, o : device bf16 [B,heads,N,d] and lse : fp32 [B,heads,N] in
 * raster token order n = (t*H + y)*W + x instead of flattened order.  The
 * mask (row_ptr, col_idx) is unchanged: it indexes fractal blocks, block r of
 * a head being the P x P patch (r % (H/P*W/P)) of frame r / (H/P*W/P).  Each
 * block is fetched by one patch-shaped TMA box and each output row is stored
 * at its raster position, so
 *   vsa_sparse_attn_fwd_raster(q, k, v -> o, lse)
 * equals, bit for bit, vsa_fractal_flatten of q, k and v, vsa_sparse_attn_fwd,
 * then vsa_fractal_unflatten of o and the same permutation of lse.  Workspace
 * and errors as vsa_sparse_attn_fwd. */
vsa_status vsa_sparse_attn_fwd_raster(const void *q, const void *k, const void *v,
                                      const int64_t *row_ptr, const int32_t *col_idx,
                                      vsa_shape s, float scale, void *o, float *lse,
                                      void *workspace, size_t workspace_bytes, void *stream);

/* 5. from flattened q, k, v (as vsa_sparse_attn_fwd takes them) to raster o
 * and lse: the output unflattening (vsa_fractal_unflatten) folded into the
 * attention's stores, each output row written at its raster position
 * n = (t*H + y)*W + x.  qf, kf, vf : device bf16 [B,heads,N,d] flattened;
 * o : device bf16 [B,heads,N,d] and lse : fp32 [B,heads,N] in raster order.
 * Equals, bit for bit, vsa_sparse_attn_fwd followed by vsa_fractal_unflatten
 * of o and the same permutation of lse.  Workspace and errors as
 * vsa_sparse_attn_fwd. */
vsa_status vsa_sparse_attn_fwd_to_raster(const void *qf, const void *kf, const void *vf,
                                         const int64_t *row_ptr, const int32_t *col_idx,
                                         vsa_shape s, float scale, void *o, float *lse,
                                         void *workspace, size_t workspace_bytes,
                                         void *stream);

/* Query-subset attention (HSA, arXiv 2605.06892 summary, section 2.2 "KV cache
 * synchronisation": only the active tokens form queries, against the whole
 * cached K and V, so the cost is O(|active| * N) instead of O(N^2)).  At block
 * granularity: only the listed query blocks are computed, each exactly as
 * vsa_sparse_attn_fwd computes it over its CSR key blocks (a CSR that keeps
 * every block gives HSA's full-context attention); O and LSE rows of every
 * other query block are left untouched.  A block with an active token is
 * computed whole (all 64 of its rows).
 * qblocks : device int32 [n_qblocks], global query-block rows
 *           g = (b*heads + h)*Nb + r, strictly ascending.  Listed blocks share
 *           128-row tensor-core tiles two by two in list order within a head.
 *           An entry out of range or out of order is recorded in the device
 *           error word (vsa_device_status reports "bad block index"); the set
 *           of blocks then computed is unspecified, and every access stays in
 *           bounds.
 * Other arguments, layouts and the workspace are those of vsa_sparse_attn_fwd;
 * n_qblocks = 0 does nothing. */
vsa_status vsa_sparse_attn_fwd_rows(const void *qf, const void *kf, const void *vf,
                                    const int64_t *row_ptr, const int32_t *col_idx,
                                    vsa_shape s, float scale, const int32_t *qblocks,
                                    int64_t n_qblocks, void *o, float *lse, void *workspace,
                                    size_t workspace_bytes, void *stream);

/* Block-sparse attention forward without a caller-provided workspace.
 * The paper has no counterpart to this call; it exists for callers that cannot
 * allocate device memory -- plugins whose host framework passes them only
 * inputs and outputs, processes that reserve all device memory at start-up,
 * and latency-critical paths where cudaMalloc/cudaFree would synchronise the
 * device.  Same arguments and results as vsa_sparse_attn_fwd, minus the
 * workspace: the scheduler's scratch lives in a fixed 8 MiB array inside the
 * library (held by every GPU that loads it until the process exits), which
 * fits about two million 128-row query tiles; larger shapes return
 * VSA_ERR_CAPACITY.  All calls share that array and it keeps the last call's
 * contents (each call re-plans and resets it first), so calls that overlap on
 * the GPU race.  The first call on a device looks up the array's address;
 * make it before any stream capture.  Allocates nothing. */
vsa_status vsa_sparse_attn_fwd_noalloc(const void *qf, const void *kf, const void *vf,
                                       const int64_t *row_ptr, const int32_t *col_idx,
                                       vsa_shape s, float scale, void *o, float *lse,
                                       void *stream);

/* Semantic-aware permutation attention (Sparse VideoGen2, arXiv 2505.18875
 * summary, sections 2A-2C).  Per (b, h): k-means on Q into Cq clusters and on
 * K into Ck clusters (Lloyd's iterations from the given centroids -- the
 * centroid cache of section 2C -- or from the tokens at positions
 * floor(j*N/C); squared Euclidean distance with the centroids rounded to bf16,
 * ties to the lower cluster; an empty cluster keeps its centroid), tokens
 * permuted so that each cluster is contiguous (token order inside a cluster),
 * key clusters kept per query cluster by the centroids' estimated attention
 * a_j ~ |K_j| exp(c_q . c_kj / sqrt(d)) until the kept mass reaches p (ties to
 * the lower index; p = 1 keeps every cluster), and attention of every query
 * token over the key tokens of its cluster's kept clusters.
 * q, k, v : device bf16 [B,heads,N,d] in any token order (the result does not
 *           depend on the order beyond the initial centroids).
 * o, lse  : device bf16 [B,heads,N,d], fp32 [B,heads,N], same token order.
 * init_q, init_k : optional device fp32 [B,heads,Cq|Ck,d] initial centroids.
 * state   : optional; each non-null member receives that intermediate.
 * Limits: 1 <= Cq, Ck <= min(1024, N), 0 <= iters <= 64, 0 < p <= 1;
 * the workspace (vsa_cluster_attn_workspace_size, 256-byte aligned) holds the
 * padded permuted tensors, so it is several times the size of Q. */
typedef struct {
    int32_t Cq, Ck;     /* clusters of Q and of K */
    int32_t iters;      /* Lloyd iterations (assign + update) before the final assignment */
    float p;            /* kept estimated-attention mass per query cluster */
} vsa_cluster_params;

typedef struct {
    int32_t *q_labels, *k_labels;       /* [B,heads,N] */
    int32_t *q_counts, *k_counts;       /* [B,heads,Cq|Ck] cluster sizes */
    float *q_centroids, *k_centroids;   /* [B,heads,Cq|Ck,d], the ones labels were assigned with */
    uint8_t *keep;                      /* [B,heads,Cq,Ck] kept key clusters */
} vsa_cluster_state;

size_t vsa_cluster_attn_workspace_size(vsa_shape s, vsa_cluster_params c);
vsa_status vsa_cluster_attn_fwd(const void *q, const void *k, const void *v, vsa_shape s,
                                vsa_cluster_params c, float scale, const float *init_q,
                                const float *init_k, void *o, float *lse,
                                const vsa_cluster_state *state, void *workspace,
                                size_t workspace_bytes, void *stream);

/* Message for the last non-OK status returned to the calling thread. */
const char *vsa_last_error(void);

/* Synchronises `stream`, then reports and clears the device error word of the
 * current device: VSA_OK, or VSA_ERR_DEVICE_TIMEOUT if a kernel gave up a
 * bounded wait since the last call, or VSA_ERR_CUDA if the stream failed. */
vsa_status vsa_device_status(void *stream);

/* Diagnostic of the failure-detection path (no counterpart on the pages): one
 * device thread waits, with a limit of `wait_cycles` SM clock cycles, on an
 * mbarrier that nothing arrives at.  The wait gives up, records code 32 in the
 * device error word and the kernel returns, exactly as a library kernel whose
 * expected arrival never comes does.  The next vsa_device_status() on the
 * stream then returns VSA_ERR_DEVICE_TIMEOUT (and clears the word); later
 * calls are unaffected.  wait_cycles in [1, 2^32] (VSA_ERR_INVALID_ARG
 * otherwise); about 2^21 cycles is a millisecond. */
vsa_status vsa_wait_probe(int64_t wait_cycles, void *stream);

/* Library version, "major.minor.patch". */
const char *vsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* VSA_H */
