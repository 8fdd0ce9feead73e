// vsa_internal.h -- launch functions shared between the C-ABI layer and the
// kernel translation units of libvsa.  Host-side only; not part of the ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/vsa.h"

namespace vsa {

struct Geometry {
  int64_t BH;   // batch * heads
  int64_t N;    // tokens per (batch, head)
  int64_t Nb;   // 64-token blocks per (batch, head)
  int T, H, W, d, P, Hb, Wb;
};

inline Geometry geometry(const vsa_shape &s) {
  Geometry g;
  g.BH = static_cast<int64_t>(s.B) * s.heads;
  g.N = static_cast<int64_t>(s.T) * s.H * s.W;
  g.Nb = g.N / 64;
  g.T = s.T; g.H = s.H; g.W = s.W; g.d = s.d; g.P = s.P;
  g.Hb = s.P ? s.H / s.P : 0;
  g.Wb = s.P ? s.W / s.P : 0;
  return g;
}

int num_sms();   // SM count of the current device (cached per device)

cudaError_t launch_fractal_permute(const void *src, void *dst, const Geometry &g, bool inverse,
                                   cudaStream_t st);
cudaError_t launch_pool_qk(const void *qf, const void *kf, double *qp, double *kp,
                           const Geometry &g, cudaStream_t st);
// qf, kf null: only the block means are written (pooling straight from raster).
cudaError_t launch_flatten_pool_qk(const void *q, const void *k, void *qf, void *kf, double *qp,
                                   double *kp, const Geometry &g, cudaStream_t st);

// Block mask: workspace carve-up and launch.
size_t block_mask_workspace_bytes(const Geometry &g);
// topk > 0 selects the static-ratio rule (k blocks per row), 0 the top-p rule.
cudaError_t launch_block_mask(const double *qp, const double *kp, const Geometry &g,
                              const vsa_mask_params &p, int topk, int64_t *row_ptr,
                              int32_t *col_idx, int32_t *kept_count, void *ws, unsigned *err,
                              cudaStream_t st);

// STA window alone: closed-form CSR, no workspace.
int64_t sta_mask_nnz(const Geometry &g, int rt, int rh, int rw);
cudaError_t launch_sta_mask(const Geometry &g, int rt, int rh, int rw, int64_t *row_ptr,
                            int32_t *col_idx, int32_t *kept_count, cudaStream_t st);

// Sparse attention: workspace carve-up and launch.
size_t sparse_attn_workspace_bytes(const Geometry &g);
cudaError_t launch_sparse_attn(const void *qf, const void *kf, const void *vf,
                               const int64_t *row_ptr, const int32_t *col_idx,
                               const Geometry &g, float scale, void *o, float *lse, void *ws,
                               unsigned *err, cudaStream_t st, const char **why,
                               const int32_t *qblocks = nullptr, int64_t n_qblocks = 0,
                               const int32_t *kvalid = nullptr, int layout = 0);

// Semantic-aware permutation attention: workspace and launch.
size_t cluster_workspace_bytes(const Geometry &g, const vsa_cluster_params &c);
cudaError_t launch_cluster_attn(const void *q, const void *k, const void *v, const Geometry &g,
                                const vsa_cluster_params &c, float scale, const float *init_q,
                                const float *init_k, void *o, float *lse,
                                const vsa_cluster_state *out_state, void *ws, unsigned *err,
                                cudaStream_t st, const char **why);

// Diagnostic: one thread waits, with the given cycle limit, on an mbarrier
// that nothing arrives at; the wait gives up and records kErrWaitProbe.
cudaError_t launch_wait_probe(int64_t wait_cycles, unsigned *err, cudaStream_t st);

}  // namespace vsa
