// k_sta.cu -- the sliding-tile window as a block mask on its own (NABLA,
// Methodology item 3: the STA component M_STA of M = M_nabla OR M_STA, here
// without the content-adaptive part; also a plain local-window mask).
//
// Query block r = (t, y, x) keeps the key blocks within the Chebyshev radii
// (rt, rh, rw), clipped at the grid edges, listed frame-major, so ascending.
// Its count is a product of per-axis window widths w_t(t) w_y(y) w_x(x), so
// the number of entries before row r is a sum of per-axis prefix sums:
//   P_t(t) S_y S_x + w_t(t) P_y(y) S_x + w_t(t) w_y(y) P_x(x)
// (S = sum over the axis, P = sum over the coordinates below).  Every thread
// writes its row's offset, count and columns directly; no scan, no workspace.
#include "vsa_device.cuh"
#include "vsa_internal.h"

namespace vsa {
namespace {

__host__ __device__ inline int64_t width(int c, int r, int n) {
  const int lo = c - r > 0 ? c - r : 0;
  const int hi = c + r < n - 1 ? c + r : n - 1;
  return hi - lo + 1;
}

__host__ __device__ inline int64_t width_prefix(int c, int r, int n) {
  int64_t s = 0;
  for (int i = 0; i < c; ++i) s += width(i, r, n);
  return s;
}

__global__ void __launch_bounds__(256)
    sta_mask_kernel(int64_t rows, int Nb, int T, int Hb, int Wb, int rt, int rh, int rw,
                    int64_t Sy, int64_t Sx, int64_t per_head, int64_t *__restrict__ row_ptr,
                    int32_t *__restrict__ col_idx, int32_t *__restrict__ kept_count) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < rows;
       g += stride) {
    const int64_t bh = g / Nb;
    const int r = static_cast<int>(g % Nb);
    const int t = r / (Hb * Wb), y = (r / Wb) % Hb, x = r % Wb;
    const int64_t wt = width(t, rt, T), wy = width(y, rh, Hb), wx = width(x, rw, Wb);
    const int64_t off = bh * per_head + width_prefix(t, rt, T) * Sy * Sx +
                        wt * width_prefix(y, rh, Hb) * Sx + wt * wy * width_prefix(x, rw, Wb);
    row_ptr[g] = off;
    if (kept_count) kept_count[g] = static_cast<int32_t>(wt * wy * wx);
    if (g == rows - 1) row_ptr[rows] = off + wt * wy * wx;
    int64_t p = off;
    const int t1 = t + rt < T - 1 ? t + rt : T - 1, y1 = y + rh < Hb - 1 ? y + rh : Hb - 1;
    const int x1 = x + rw < Wb - 1 ? x + rw : Wb - 1;
    for (int tt = t - rt > 0 ? t - rt : 0; tt <= t1; ++tt)
      for (int yy = y - rh > 0 ? y - rh : 0; yy <= y1; ++yy)
        for (int xx = x - rw > 0 ? x - rw : 0; xx <= x1; ++xx)
          col_idx[p++] = (tt * Hb + yy) * Wb + xx;
  }
}

}  // namespace

int64_t sta_mask_nnz(const Geometry &g, int rt, int rh, int rw) {
  const int T = static_cast<int>(g.Nb / (static_cast<int64_t>(g.Hb) * g.Wb));
  return g.BH * width_prefix(T, rt, T) * width_prefix(g.Hb, rh, g.Hb) *
         width_prefix(g.Wb, rw, g.Wb);
}

cudaError_t launch_sta_mask(const Geometry &g, int rt, int rh, int rw, int64_t *row_ptr,
                            int32_t *col_idx, int32_t *kept_count, cudaStream_t st) {
  const int64_t rows = g.BH * g.Nb;
  if (rows == 0) return cudaMemsetAsync(row_ptr, 0, sizeof(int64_t), st);
  const int T = static_cast<int>(g.Nb / (static_cast<int64_t>(g.Hb) * g.Wb));
  const int64_t Sy = width_prefix(g.Hb, rh, g.Hb), Sx = width_prefix(g.Wb, rw, g.Wb);
  const int64_t per_head = width_prefix(T, rt, T) * Sy * Sx;
  const int64_t want = (rows + 255) / 256;
  const int grid = static_cast<int>(want < 8LL * num_sms() ? want : 8LL * num_sms());
  sta_mask_kernel<<<grid, 256, 0, st>>>(rows, static_cast<int>(g.Nb), T, g.Hb, g.Wb, rt, rh, rw,
                                        Sy, Sx, per_head, row_ptr, col_idx, kept_count);
  return cudaGetLastError();
}

}  // namespace vsa
