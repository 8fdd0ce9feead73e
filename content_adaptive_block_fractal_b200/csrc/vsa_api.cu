// vsa_api.cu -- the extern "C" entry points of libvsa (declared in
// include/vsa.h): host-side validation, launch, error reporting.
#include "vsa_internal.h"

#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>

namespace vsa {
size_t block_mask_smem_bytes(const Geometry &g);
}

namespace {

thread_local std::string g_last_error;

// Per-device error word written by bounded device waits (bit flags).
__device__ unsigned g_device_error;

constexpr int kMaxDevices = 64;
constexpr size_t kMaxSmem = 232448;  // opt-in dynamic shared memory per block on sm_100

vsa_status fail(vsa_status st, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

vsa_status cuda_fail(cudaError_t e, const char *what) {
  return fail(VSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

unsigned *device_error_word(cudaError_t *err) {
  static unsigned *addr[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if ((*err = cudaGetDevice(&dev)) != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void *p = nullptr;
    if ((*err = cudaGetSymbolAddress(&p, g_device_error)) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<unsigned *>(p);
  }
  return addr[dev];
}

// Shape checks shared by every entry point.
vsa_status check_shape(const vsa_shape &s) {
  if (s.B < 0 || s.heads < 0 || s.T < 0 || s.H < 0 || s.W < 0 || s.d <= 0 || s.P <= 0)
    return fail(VSA_ERR_INVALID_ARG, "negative or zero size in shape (B=%d heads=%d T=%d H=%d W=%d d=%d P=%d)",
                s.B, s.heads, s.T, s.H, s.W, s.d, s.P);
  if (s.P * s.P != 64)
    return fail(VSA_ERR_UNSUPPORTED, "patch size P=%d: blocks must be P*P = 64 tokens (P = 8)", s.P);
  if (s.H % s.P || s.W % s.P)
    return fail(VSA_ERR_UNSUPPORTED, "grid H=%d W=%d is not a multiple of P=%d", s.H, s.W, s.P);
  if (s.d != 64 && s.d != 128)
    return fail(VSA_ERR_UNSUPPORTED, "head dim d=%d: only 64 and 128 are implemented", s.d);
  const long long n = 1LL * s.B * s.heads * s.T * s.H * s.W;
  if (n > (1LL << 31) - 1)
    return fail(VSA_ERR_UNSUPPORTED, "B*heads*N = %lld exceeds 2^31-1 tokens", n);
  return VSA_OK;
}

bool empty(const vsa_shape &s) { return 1LL * s.B * s.heads * s.T * s.H * s.W == 0; }

}  // namespace

namespace vsa {
void set_last_error(const char *msg) { g_last_error = msg; }

int num_sms() {
  static int cache[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  if (!cache[dev]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = n > 0 ? n : 148;
  }
  return cache[dev];
}
}  // namespace vsa

extern "C" {

const char *vsa_version(void) { return "0.2.0"; }

const char *vsa_last_error(void) { return g_last_error.c_str(); }

static vsa_status check_cluster(const vsa_shape &s, const vsa_cluster_params &c) {
  vsa_status st = check_shape(s);
  if (st != VSA_OK) return st;
  const vsa::Geometry g = vsa::geometry(s);
  if (c.Cq < 1 || c.Ck < 1 || c.Cq > 1024 || c.Ck > 1024 || c.Cq > g.N || c.Ck > g.N)
    return fail(VSA_ERR_INVALID_ARG, "cluster counts (%d, %d) outside [1, min(1024, N)]", c.Cq,
                c.Ck);
  if (c.iters < 0 || c.iters > 64) return fail(VSA_ERR_INVALID_ARG, "iters=%d outside [0, 64]", c.iters);
  if (!(c.p > 0.0f && c.p <= 1.0f))
    return fail(VSA_ERR_INVALID_ARG, "p=%g outside (0, 1]", static_cast<double>(c.p));
  const int64_t Np = g.N + 64LL * (c.Cq > c.Ck ? c.Cq : c.Ck);
  if (g.BH * Np >= (1LL << 31))
    return fail(VSA_ERR_UNSUPPORTED, "padded sequence too long for 32-bit row coordinates");
  return VSA_OK;
}

size_t vsa_cluster_attn_workspace_size(vsa_shape s, vsa_cluster_params c) {
  if (check_cluster(s, c) != VSA_OK) return 0;
  return vsa::cluster_workspace_bytes(vsa::geometry(s), c);
}

vsa_status vsa_cluster_attn_fwd(const void *q, const void *k, const void *v, vsa_shape s,
                                vsa_cluster_params c, float scale, const float *init_q,
                                const float *init_k, void *o, float *lse,
                                const vsa_cluster_state *state, void *workspace,
                                size_t workspace_bytes, void *stream) {
  vsa_status st = check_cluster(s, c);
  if (st != VSA_OK) return st;
  if (empty(s)) return VSA_OK;
  if (!q || !k || !v || !o || !lse || !workspace)
    return fail(VSA_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      (init_q && !aligned16(init_q)) || (init_k && !aligned16(init_k)))
    return fail(VSA_ERR_UNSUPPORTED, "misaligned pointer (tensors 16 B, workspace 256 B)");
  if (!(scale == scale)) return fail(VSA_ERR_INVALID_ARG, "scale is NaN");
  const vsa::Geometry g = vsa::geometry(s);
  const size_t ws = vsa::cluster_workspace_bytes(g, c);
  if (workspace_bytes < ws)
    return fail(VSA_ERR_CAPACITY, "cluster attention workspace %zu < %zu bytes", workspace_bytes, ws);
  if (scale <= 0.0f) scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(s.d)));
  cudaError_t e;
  unsigned *err = device_error_word(&e);
  if (!err) return cuda_fail(e, "device error word");
  const char *why = nullptr;
  e = vsa::launch_cluster_attn(q, k, v, g, c, scale, init_q, init_k, o, lse, state, workspace,
                               err, static_cast<cudaStream_t>(stream), &why);
  if (e != cudaSuccess)
    return why ? fail(e == cudaErrorInvalidValue ? VSA_ERR_UNSUPPORTED : VSA_ERR_CUDA, "%s", why)
               : cuda_fail(e, "cluster attention launch");
  return VSA_OK;
}

static vsa_status permute(const void *src, void *dst, vsa_shape s, void *stream, bool inverse) {
  vsa_status st = check_shape(s);
  if (st != VSA_OK) return st;
  if (empty(s)) return VSA_OK;
  if (!src || !dst) return fail(VSA_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(src) || !aligned16(dst))
    return fail(VSA_ERR_UNSUPPORTED, "tensor pointers must be 16-byte aligned");
  const vsa::Geometry g = vsa::geometry(s);
  const size_t bytes = static_cast<size_t>(g.BH * g.N) * g.d * 2;
  const char *a = static_cast<const char *>(src);
  const char *b = static_cast<const char *>(dst);
  if (a < b + bytes && b < a + bytes)
    return fail(VSA_ERR_INVALID_ARG, "source and destination overlap");
  cudaError_t e = vsa::launch_fractal_permute(src, dst, g, inverse,
                                              static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? VSA_OK : cuda_fail(e, "fractal permute launch");
}

vsa_status vsa_fractal_flatten(const void *x, void *y, vsa_shape s, void *stream) {
  return permute(x, y, s, stream, false);
}

vsa_status vsa_fractal_unflatten(const void *y, void *x, vsa_shape s, void *stream) {
  return permute(y, x, s, stream, true);
}

vsa_status vsa_pool_qk(const void *qf, const void *kf, double *qp, double *kp, vsa_shape s,
                       void *stream) {
  vsa_status st = check_shape(s);
  if (st != VSA_OK) return st;
  if (empty(s)) return VSA_OK;
  if (!qf || !kf || !qp || !kp) return fail(VSA_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(qf) || !aligned16(kf) || !aligned16(qp) || !aligned16(kp))
    return fail(VSA_ERR_UNSUPPORTED, "tensor pointers must be 16-byte aligned");
  cudaError_t e = vsa::launch_pool_qk(qf, kf, qp, kp, vsa::geometry(s),
                                      static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? VSA_OK : cuda_fail(e, "pool launch");
}

static bool overlap(const void *a, size_t abytes, const void *b, size_t bbytes) {
  const char *x = static_cast<const char *>(a);
  const char *y = static_cast<const char *>(b);
  return x < y + bbytes && y < x + abytes;
}

vsa_status vsa_flatten_pool_qk(const void *q, const void *k, void *qf, void *kf, double *qp,
                               double *kp, vsa_shape s, void *stream) {
  vsa_status st = check_shape(s);
  if (st != VSA_OK) return st;
  if (empty(s)) return VSA_OK;
  if (!q || !k || !qf || !kf || !qp || !kp) return fail(VSA_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(qf) || !aligned16(kf) || !aligned16(qp) ||
      !aligned16(kp))
    return fail(VSA_ERR_UNSUPPORTED, "tensor pointers must be 16-byte aligned");
  const vsa::Geometry g = vsa::geometry(s);
  const size_t bytes = static_cast<size_t>(g.BH * g.N) * g.d * 2;
  const size_t pbytes = static_cast<size_t>(g.BH * g.Nb) * g.d * 8;
  // every output against every other buffer (the inputs may alias each other)
  const void *outs[4] = {qf, kf, qp, kp};
  const size_t osz[4] = {bytes, bytes, pbytes, pbytes};
  for (int i = 0; i < 4; ++i) {
    if (overlap(outs[i], osz[i], q, bytes) || overlap(outs[i], osz[i], k, bytes))
      return fail(VSA_ERR_INVALID_ARG, "an output overlaps an input");
    for (int j = i + 1; j < 4; ++j)
      if (overlap(outs[i], osz[i], outs[j], osz[j]))
        return fail(VSA_ERR_INVALID_ARG, "outputs overlap");
  }
  cudaError_t e = vsa::launch_flatten_pool_qk(q, k, qf, kf, qp, kp, g,
                                              static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? VSA_OK : cuda_fail(e, "flatten+pool launch");
}

vsa_status vsa_pool_qk_raster(const void *q, const void *k, double *qp, double *kp, vsa_shape s,
                              void *stream) {
  vsa_status st = check_shape(s);
  if (st != VSA_OK) return st;
  if (empty(s)) return VSA_OK;
  if (!q || !k || !qp || !kp) return fail(VSA_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(qp) || !aligned16(kp))
    return fail(VSA_ERR_UNSUPPORTED, "tensor pointers must be 16-byte aligned");
  const vsa::Geometry g = vsa::geometry(s);
  const size_t bytes = static_cast<size_t>(g.BH * g.N) * g.d * 2;
  const size_t pbytes = static_cast<size_t>(g.BH * g.Nb) * g.d * 8;
  if (overlap(qp, pbytes, q, bytes) || overlap(qp, pbytes, k, bytes) ||
      overlap(kp, pbytes, q, bytes) || overlap(kp, pbytes, k, bytes))
    return fail(VSA_ERR_INVALID_ARG, "an output overlaps an input");
  if (overlap(qp, pbytes, kp, pbytes)) return fail(VSA_ERR_INVALID_ARG, "outputs overlap");
  cudaError_t e = vsa::launch_flatten_pool_qk(q, k, nullptr, nullptr, qp, kp, g,
                                              static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? VSA_OK : cuda_fail(e, "raster pool launch");
}

size_t vsa_block_mask_workspace_size(vsa_shape s) {
  if (check_shape(s) != VSA_OK) return 0;
  return vsa::block_mask_workspace_bytes(vsa::geometry(s));
}

vsa_status vsa_block_mask(const double *qp, const double *kp, vsa_shape s, vsa_mask_params p,
                          int64_t *row_ptr, int32_t *col_idx, int64_t col_capacity,
                          int32_t *kept_count, void *workspace, size_t workspace_bytes,
                          void *stream) {
  vsa_status st = check_shape(s);
  if (st != VSA_OK) return st;
  if (!(p.thr >= 0.0f && p.thr < 1.0f))
    return fail(VSA_ERR_INVALID_ARG, "thr=%g outside [0, 1)", static_cast<double>(p.thr));
  if (p.use_sta && (p.sta_t < 0 || p.sta_h < 0 || p.sta_w < 0))
    return fail(VSA_ERR_INVALID_ARG, "negative STA radius (%d, %d, %d)", p.sta_t, p.sta_h, p.sta_w);
  if (!row_ptr) return fail(VSA_ERR_INVALID_ARG, "null row_ptr");
  const vsa::Geometry g = vsa::geometry(s);
  const int64_t need = g.BH * g.Nb * g.Nb;
  if (col_capacity < need)
    return fail(VSA_ERR_CAPACITY, "col_capacity %lld < B*heads*Nb*Nb = %lld",
                static_cast<long long>(col_capacity), static_cast<long long>(need));
  if (empty(s)) {
    cudaError_t e = cudaMemsetAsync(row_ptr, 0, sizeof(int64_t), static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? VSA_OK : cuda_fail(e, "row_ptr reset");
  }
  if (!qp || !kp || !col_idx || !workspace)
    return fail(VSA_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(qp) || !aligned16(kp) || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      (reinterpret_cast<uintptr_t>(row_ptr) & 7u) || (reinterpret_cast<uintptr_t>(col_idx) & 3u) ||
      (kept_count && (reinterpret_cast<uintptr_t>(kept_count) & 3u)))
    return fail(VSA_ERR_UNSUPPORTED, "misaligned pointer (tensors 16 B, workspace 256 B)");
  const size_t ws = vsa::block_mask_workspace_bytes(g);
  if (workspace_bytes < ws)
    return fail(VSA_ERR_CAPACITY, "block mask workspace %zu < %zu bytes", workspace_bytes, ws);
  if (vsa::block_mask_smem_bytes(g) > kMaxSmem)
    return fail(VSA_ERR_UNSUPPORTED, "Nb=%lld blocks per head exceeds the mask kernel's shared memory",
                static_cast<long long>(g.Nb));
  cudaError_t e;
  unsigned *err = device_error_word(&e);
  if (!err) return cuda_fail(e, "device error word");
  e = vsa::launch_block_mask(qp, kp, g, p, 0, row_ptr, col_idx, kept_count, workspace, err,
                             static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? VSA_OK : cuda_fail(e, "block mask launch");
}

vsa_status vsa_block_mask_topk(const double *qp, const double *kp, vsa_shape s, int32_t k,
                               vsa_mask_params p, int64_t *row_ptr, int32_t *col_idx,
                               int64_t col_capacity, int32_t *kept_count, void *workspace,
                               size_t workspace_bytes, void *stream) {
  vsa_status st = check_shape(s);
  if (st != VSA_OK) return st;
  if (k < 1) return fail(VSA_ERR_INVALID_ARG, "k=%d: at least one block per row", k);
  if (p.use_sta && (p.sta_t < 0 || p.sta_h < 0 || p.sta_w < 0))
    return fail(VSA_ERR_INVALID_ARG, "negative STA radius (%d, %d, %d)", p.sta_t, p.sta_h, p.sta_w);
  if (!row_ptr) return fail(VSA_ERR_INVALID_ARG, "null row_ptr");
  const vsa::Geometry g = vsa::geometry(s);
  const int64_t need = g.BH * g.Nb * g.Nb;
  if (col_capacity < need)
    return fail(VSA_ERR_CAPACITY, "col_capacity %lld < B*heads*Nb*Nb = %lld",
                static_cast<long long>(col_capacity), static_cast<long long>(need));
  if (empty(s)) {
    cudaError_t e = cudaMemsetAsync(row_ptr, 0, sizeof(int64_t), static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? VSA_OK : cuda_fail(e, "row_ptr reset");
  }
  if (!qp || !kp || !col_idx || !workspace)
    return fail(VSA_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(qp) || !aligned16(kp) || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      (reinterpret_cast<uintptr_t>(row_ptr) & 7u) || (reinterpret_cast<uintptr_t>(col_idx) & 3u) ||
      (kept_count && (reinterpret_cast<uintptr_t>(kept_count) & 3u)))
    return fail(VSA_ERR_UNSUPPORTED, "misaligned pointer (tensors 16 B, workspace 256 B)");
  const size_t ws = vsa::block_mask_workspace_bytes(g);
  if (workspace_bytes < ws)
    return fail(VSA_ERR_CAPACITY, "block mask workspace %zu < %zu bytes", workspace_bytes, ws);
  if (vsa::block_mask_smem_bytes(g) > kMaxSmem)
    return fail(VSA_ERR_UNSUPPORTED, "Nb=%lld blocks per head exceeds the mask kernel's shared memory",
                static_cast<long long>(g.Nb));
  cudaError_t e;
  unsigned *err = device_error_word(&e);
  if (!err) return cuda_fail(e, "device error word");
  e = vsa::launch_block_mask(qp, kp, g, p, k, row_ptr, col_idx, kept_count, workspace, err,
                             static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? VSA_OK : cuda_fail(e, "static-ratio mask launch");
}

vsa_status vsa_sta_mask(vsa_shape s, int32_t sta_t, int32_t sta_h, int32_t sta_w,
                        int64_t *row_ptr, int32_t *col_idx, int64_t col_capacity,
                        int32_t *kept_count, void *stream) {
  vsa_status st = check_shape(s);
  if (st != VSA_OK) return st;
  if (sta_t < 0 || sta_h < 0 || sta_w < 0)
    return fail(VSA_ERR_INVALID_ARG, "negative STA radius (%d, %d, %d)", sta_t, sta_h, sta_w);
  if (!row_ptr) return fail(VSA_ERR_INVALID_ARG, "null row_ptr");
  const vsa::Geometry g = vsa::geometry(s);
  const int64_t need = vsa::sta_mask_nnz(g, sta_t, sta_h, sta_w);
  if (col_capacity < need)
    return fail(VSA_ERR_CAPACITY, "col_capacity %lld < the window's %lld entries",
                static_cast<long long>(col_capacity), static_cast<long long>(need));
  if (empty(s)) {
    cudaError_t e = cudaMemsetAsync(row_ptr, 0, sizeof(int64_t), static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? VSA_OK : cuda_fail(e, "row_ptr reset");
  }
  if (!col_idx) return fail(VSA_ERR_INVALID_ARG, "null col_idx");
  if ((reinterpret_cast<uintptr_t>(row_ptr) & 7u) || (reinterpret_cast<uintptr_t>(col_idx) & 3u) ||
      (kept_count && (reinterpret_cast<uintptr_t>(kept_count) & 3u)))
    return fail(VSA_ERR_UNSUPPORTED, "misaligned pointer");
  cudaError_t e = vsa::launch_sta_mask(g, sta_t, sta_h, sta_w, row_ptr, col_idx, kept_count,
                                       static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? VSA_OK : cuda_fail(e, "STA mask launch");
}

size_t vsa_sparse_attn_workspace_size(vsa_shape s) {
  if (check_shape(s) != VSA_OK) return 0;
  return vsa::sparse_attn_workspace_bytes(vsa::geometry(s));
}

static vsa_status sparse_attn(const void *qf, const void *kf, const void *vf,
                              const int64_t *row_ptr, const int32_t *col_idx, vsa_shape s,
                              float scale, const int32_t *qblocks, int64_t n_qblocks, void *o,
                              float *lse, void *workspace, size_t workspace_bytes, void *stream,
                              int layout = 0);

vsa_status vsa_sparse_attn_fwd(const void *qf, const void *kf, const void *vf,
                               const int64_t *row_ptr, const int32_t *col_idx, vsa_shape s,
                               float scale, void *o, float *lse, void *workspace,
                               size_t workspace_bytes, void *stream) {
  return sparse_attn(qf, kf, vf, row_ptr, col_idx, s, scale, nullptr, 0, o, lse, workspace,
                     workspace_bytes, stream);
}

vsa_status vsa_sparse_attn_fwd_raster(const void *q, const void *k, const void *v,
                                      const int64_t *row_ptr, const int32_t *col_idx,
                                      vsa_shape s, float scale, void *o, float *lse,
                                      void *workspace, size_t workspace_bytes, void *stream) {
  return sparse_attn(q, k, v, row_ptr, col_idx, s, scale, nullptr, 0, o, lse, workspace,
                     workspace_bytes, stream, 1);
}

vsa_status vsa_sparse_attn_fwd_to_raster(const void *qf, const void *kf, const void *vf,
                                         const int64_t *row_ptr, const int32_t *col_idx,
                                         vsa_shape s, float scale, void *o, float *lse,
                                         void *workspace, size_t workspace_bytes,
                                         void *stream) {
  return sparse_attn(qf, kf, vf, row_ptr, col_idx, s, scale, nullptr, 0, o, lse, workspace,
                     workspace_bytes, stream, 2);
}

vsa_status vsa_sparse_attn_fwd_rows(const void *qf, const void *kf, const void *vf,
                                    const int64_t *row_ptr, const int32_t *col_idx,
                                    vsa_shape s, float scale, const int32_t *qblocks,
                                    int64_t n_qblocks, void *o, float *lse, void *workspace,
                                    size_t workspace_bytes, void *stream) {
  vsa_status st = check_shape(s);
  if (st != VSA_OK) return st;
  if (n_qblocks < 0) return fail(VSA_ERR_INVALID_ARG, "negative query-block count");
  const vsa::Geometry g = vsa::geometry(s);
  if (n_qblocks > g.BH * g.Nb)
    return fail(VSA_ERR_INVALID_ARG, "%lld query blocks listed, the shape has %lld",
                static_cast<long long>(n_qblocks), static_cast<long long>(g.BH * g.Nb));
  if (g.BH * g.Nb >= (1LL << 30))
    return fail(VSA_ERR_UNSUPPORTED, "too many query blocks for the subset planner");
  if (n_qblocks > 0 && (!qblocks || (reinterpret_cast<uintptr_t>(qblocks) & 3u)))
    return fail(VSA_ERR_INVALID_ARG, "null or misaligned query-block list");
  if (n_qblocks == 0) return VSA_OK;
  return sparse_attn(qf, kf, vf, row_ptr, col_idx, s, scale, qblocks, n_qblocks, o, lse,
                     workspace, workspace_bytes, stream);
}

static vsa_status sparse_attn(const void *qf, const void *kf, const void *vf,
                              const int64_t *row_ptr, const int32_t *col_idx, vsa_shape s,
                              float scale, const int32_t *qblocks, int64_t n_qblocks, void *o,
                              float *lse, void *workspace, size_t workspace_bytes, void *stream,
                              int layout) {
  vsa_status st = check_shape(s);
  if (st != VSA_OK) return st;
  if (empty(s)) return VSA_OK;
  if (!qf || !kf || !vf || !row_ptr || !col_idx || !o || !lse || !workspace)
    return fail(VSA_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(qf) || !aligned16(kf) || !aligned16(vf) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      (reinterpret_cast<uintptr_t>(row_ptr) & 7u) || (reinterpret_cast<uintptr_t>(col_idx) & 3u))
    return fail(VSA_ERR_UNSUPPORTED, "misaligned pointer (tensors 16 B, workspace 256 B)");
  if (!(scale == scale)) return fail(VSA_ERR_INVALID_ARG, "scale is NaN");
  const vsa::Geometry g = vsa::geometry(s);
  const size_t ws = vsa::sparse_attn_workspace_bytes(g);
  if (workspace_bytes < ws)
    return fail(VSA_ERR_CAPACITY, "attention workspace %zu < %zu bytes", workspace_bytes, ws);
  if (scale <= 0.0f) scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(s.d)));
  cudaError_t e;
  unsigned *err = device_error_word(&e);
  if (!err) return cuda_fail(e, "device error word");
  const char *why = nullptr;
  e = vsa::launch_sparse_attn(qf, kf, vf, row_ptr, col_idx, g, scale, o, lse, workspace, err,
                              static_cast<cudaStream_t>(stream), &why, qblocks, n_qblocks,
                              nullptr, layout);
  if (e != cudaSuccess)
    return why ? fail(e == cudaErrorInvalidValue ? VSA_ERR_UNSUPPORTED : VSA_ERR_CUDA, "%s", why)
               : cuda_fail(e, "sparse attention launch");
  return VSA_OK;
}

vsa_status vsa_device_status(void *stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  unsigned *err = device_error_word(&e);
  if (!err) return cuda_fail(e, "device error word");
  unsigned v = 0;
  if ((e = cudaMemcpy(&v, err, sizeof v, cudaMemcpyDeviceToHost)) != cudaSuccess)
    return cuda_fail(e, "read device error word");
  if (v == 0) return VSA_OK;
  const unsigned zero = 0;
  if ((e = cudaMemcpy(err, &zero, sizeof zero, cudaMemcpyHostToDevice)) != cudaSuccess)
    return cuda_fail(e, "clear device error word");
  return fail(VSA_ERR_DEVICE_TIMEOUT,
              "device error word 0x%x (1: TMA wait, 2: MMA wait, 4: softmax wait, 8: bad block index, 16: shared memory misaligned, 32: wait probe)",
              v);
}

vsa_status vsa_wait_probe(int64_t wait_cycles, void *stream) {
  if (wait_cycles < 1 || wait_cycles > (1LL << 32))
    return fail(VSA_ERR_INVALID_ARG, "wait_cycles %lld outside [1, 2^32]",
                static_cast<long long>(wait_cycles));
  cudaError_t e;
  unsigned *err = device_error_word(&e);
  if (!err) return cuda_fail(e, "device error word");
  if ((e = vsa::launch_wait_probe(wait_cycles, err, static_cast<cudaStream_t>(stream))) !=
      cudaSuccess)
    return cuda_fail(e, "wait probe launch");
  return VSA_OK;
}

}  // extern "C"
