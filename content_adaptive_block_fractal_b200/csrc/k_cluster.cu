// k_cluster.cu -- semantic-aware permutation and centroid top-p (Sparse
// VideoGen2 summary, sections 2A-2C): k-means on Q and on K, tokens of one
// cluster made contiguous, key clusters chosen per query cluster by the
// centroids' estimated attention until its mass reaches p, then the block-
// sparse attention kernel over the permuted tensors.
//
// Layout: every cluster starts on a 64-token block boundary of a padded
// per-head sequence of Np = N + 64*max(Cq, Ck) rows (a static bound, so the
// host never waits for the cluster sizes); padding rows are zero and the
// attention kernel masks the padding keys of a cluster's last block with a
// per-key-block valid count.
//
// Kernels, per k-means iteration and tensor:
//   centroid_prep_kernel   fp32 centroids -> bf16 table (the tensor-core
//                          operand) and fp32 squared norms of the bf16 values
//   kmeans_assign_kernel   one CTA per 128 tokens: tcgen05.mma of the token
//                          tile against 128-centroid tiles into TMEM, argmin of
//                          ||c||^2 - 2 x.c per row (ties to the lower cluster)
//   tile_hist_kernel, tile_scan_kernel, cluster_start_kernel, position_kernel
//                          a stable counting sort: positions in cluster order,
//                          token order inside a cluster, 64-aligned starts
//   centroid_update_kernel member means in fp64, members read through the
//                          inverse map of the permutation
// and after the final assignment gather_rows_kernel (the permuted rows;
// padding rows zero)
// and once: centroid_topp_kernel (fp64 estimated attention, sort, top-p),
// cluster_csr kernels (block CSR + valid keys), the attention launch, and
// unpermute_kernel (O and LSE back to token order).
#include "vsa_device.cuh"
#include "vsa_internal.h"
#include "vsa_tma.h"

#include <cmath>

namespace vsa {
namespace {

constexpr int kTile = 256;       // tokens per counting-sort tile
constexpr int kMaxClusters = 1024;

// ------------------------------------------------------------------ centroids
__global__ void centroid_prep_kernel(const float *__restrict__ cent, int64_t rows, int C,
                                     int Cpad, int d, __nv_bfloat16 *__restrict__ cbf,
                                     float *__restrict__ cnorm) {
  const int lane = threadIdx.x & 31;
  const int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (w >= rows) return;                      // rows = BH * Cpad
  const int64_t bh = w / Cpad;
  const int j = static_cast<int>(w % Cpad);
  float s = 0.0f;
  for (int i = lane; i < d; i += 32) {
    float v = 0.0f;
    if (j < C) v = cent[(bh * C + j) * d + i];
    const __nv_bfloat16 b = __float2bfloat16_rn(v);
    cbf[w * d + i] = b;
    const float bv = __bfloat162float(b);
    s = fmaf(bv, bv, s);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
  if (lane == 0) cnorm[w] = j < C ? s : INFINITY;
}

// ------------------------------------------------------------------ assignment
template <int D>
struct AssignSmem {
  static constexpr int kTileBytes = 128 * D * 2;   // 128 rows, K-major, 4-D box layout
  static constexpr int kX = 0;
  static constexpr int kC = kTileBytes;
  static constexpr int kNorm = 2 * kTileBytes;     // [2][128] fp32
  static constexpr int kBar = kNorm + 1024;        // x_full, c_full, mma_done
  static constexpr int kSlot = kBar + 32;
  static constexpr int kBytes = kSlot + 16;
};

template <int D>
__global__ void __launch_bounds__(128)
    kmeans_assign_kernel(const __grid_constant__ CUtensorMap tx,
                         const __grid_constant__ CUtensorMap tc, const float *__restrict__ cnorm,
                         int64_t N, int Cpad, int tiles_per_head, int32_t *__restrict__ label,
                         float2 *__restrict__ diag, unsigned *err) {
  using L = AssignSmem<D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicOr(err, kErrSmemAlign);
    return;
  }
  const uint32_t sbase = smem_u32(smem_raw);
  float *s_norm = reinterpret_cast<float *>(smem_raw + L::kNorm);
  const uint32_t x_full = sbase + L::kBar, c_full = x_full + 8, mma_done = x_full + 16;
  uint32_t *slot = reinterpret_cast<uint32_t *>(smem_raw + L::kSlot);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t bh = blockIdx.x / tiles_per_head;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x % tiles_per_head) * 128;
  if (threadIdx.x == 0) {
    mbar_init(x_full, 1);
    mbar_init(c_full, 1);
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(slot), 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tx);
    tma_prefetch_desc(&tc);
    mbar_arrive_expect_tx(x_full, L::kTileBytes);
    const int grp = static_cast<int>((bh * N + row0) / 8);
    tma_load_4d(sbase + L::kX, &tx, x_full, 0, 0, 0, grp);
    tma_load_4d(sbase + L::kX + L::kTileBytes / 2, &tx, x_full, 0, 0, 0, grp + 8);
  }
  constexpr uint32_t kIdesc = idesc_bf16(128, 128, false, false);
  const uint64_t x_desc = smem_desc(sbase + L::kX, 16, 16 * D);
  const uint64_t c_desc = smem_desc(sbase + L::kC, 16, 16 * D);
  const int row = warp * 32 + lane;
  const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
  float best = INFINITY, second = INFINITY;
  int arg = 0;
  bool ok = true;
  const int ntiles = Cpad / 128;
  // The centroid tile buffer is free once its MMA has completed, so the next
  // tile's TMA load (and its norms, double-buffered) run under this tile's
  // argmin; the single TMEM accumulator is reused after the block barrier.
  s_norm[threadIdx.x] = cnorm[bh * Cpad + threadIdx.x];
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(c_full, L::kTileBytes);
    const int grp = static_cast<int>((bh * Cpad) / 8);
    tma_load_4d(sbase + L::kC, &tc, c_full, 0, 0, 0, grp);
    tma_load_4d(sbase + L::kC + L::kTileBytes / 2, &tc, c_full, 0, 0, 0, grp + 8);
  }
  __syncthreads();          // norms of tile 0 visible
  for (int ct = 0; ct < ntiles && ok; ++ct) {
    if (threadIdx.x == 0) {
      bool good = (ct > 0 || mbar_wait(x_full, 0, err, kErrWaitTma)) &&
                  mbar_wait(c_full, ct & 1, err, kErrWaitTma);
      if (good) {
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k >> 2) * 64 + (k & 3) * 2;
          mma_bf16_ss(tmem, x_desc + off, c_desc + off, kIdesc, k > 0);
        }
      }
      mma_commit(mma_done);   // arrives even when nothing was issued
      if (!good) ok = false;
    }
    if (!mbar_wait(mma_done, ct & 1, err, kErrWaitMma)) ok = false;
    tc_fence_after();
    if (ct + 1 < ntiles) {
      s_norm[((ct + 1) & 1) * 128 + threadIdx.x] = cnorm[bh * Cpad + (ct + 1) * 128 + threadIdx.x];
      if (threadIdx.x == 0 && ok) {
        mbar_arrive_expect_tx(c_full, L::kTileBytes);
        const int grp = static_cast<int>((bh * Cpad + (ct + 1) * 128) / 8);
        tma_load_4d(sbase + L::kC, &tc, c_full, 0, 0, 0, grp);
        tma_load_4d(sbase + L::kC + L::kTileBytes / 2, &tc, c_full, 0, 0, 0, grp + 8);
      }
    }
    const float *nrm = s_norm + (ct & 1) * 128;
    float s[64];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      tmem_ld64(lane_addr + 64 * h, s);
#pragma unroll
      for (int j = 0; j < 64; ++j) {
        const int c = 64 * h + j;
        const float dist = fmaf(-2.0f, s[j], nrm[c]);
        if (dist < best) {
          second = best;
          best = dist;
          arg = ct * 128 + c;
        } else if (dist < second) {
          second = dist;
        }
      }
    }
    tc_fence_before();
    ok = __syncthreads_and(ok) != 0;   // TMEM and the next tile's norms
  }
  // always a label in [0, C) (0 after a failed wait, recorded in the error
  // word), so the counting sort that follows never indexes out of range
  if (row0 + row < N) {
    label[bh * N + row0 + row] = ok ? arg : 0;
    if (diag) diag[bh * N + row0 + row] = make_float2(best, second);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// ------------------------------------------------------------------ counting sort
// Per-tile label histograms: hist[bh][tile][C].
__global__ void __launch_bounds__(kTile) tile_hist_kernel(const int32_t *__restrict__ label,
                                                          int64_t N, int C, int ntile,
                                                          int32_t *__restrict__ hist) {
  __shared__ int h[kMaxClusters];
  const int64_t bh = blockIdx.x / ntile;
  const int tile = blockIdx.x % ntile;
  for (int j = threadIdx.x; j < C; j += blockDim.x) h[j] = 0;
  __syncthreads();
  const int64_t t = static_cast<int64_t>(tile) * kTile + threadIdx.x;
  if (t < N) atomicAdd(&h[label[bh * N + t]], 1);
  __syncthreads();
  int32_t *out = hist + (bh * ntile + tile) * C;
  for (int j = threadIdx.x; j < C; j += blockDim.x) out[j] = h[j];
}

// In place: hist[bh][tile][j] -> members of cluster j in the tiles before;
// count[bh][j] = cluster size.  One thread per (bh, j).
__global__ void tile_scan_kernel(int32_t *__restrict__ hist, int64_t BH, int C, int ntile,
                                 int32_t *__restrict__ count) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= BH * C) return;
  const int64_t bh = i / C;
  const int j = static_cast<int>(i % C);
  int32_t run = 0;
  int32_t *col = hist + bh * ntile * C + j;
  int tile = 0;
  for (; tile + 8 <= ntile; tile += 8) {     // eight loads in flight, then the prefix
    int32_t v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = col[static_cast<int64_t>(tile + u) * C];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      col[static_cast<int64_t>(tile + u) * C] = run;
      run += v[u];
    }
  }
  for (; tile < ntile; ++tile) {
    const int32_t v = col[static_cast<int64_t>(tile) * C];
    col[static_cast<int64_t>(tile) * C] = run;
    run += v;
  }
  count[i] = run;
}

// start[bh][j] = first padded row of cluster j (64-aligned); start[bh][C] = end.
__global__ void __launch_bounds__(1024) cluster_start_kernel(const int32_t *__restrict__ count,
                                                             int C, int32_t *__restrict__ start) {
  __shared__ int32_t warp_tot[32];
  const int64_t bh = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int j = threadIdx.x;                 // C <= 1024
  const int32_t v = j < C ? ((count[bh * C + j] + 63) / 64) * 64 : 0;
  int32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int32_t w = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xFFFFFFFFu, w, o);
      if (lane >= o) w += y;
    }
    warp_tot[lane] = w;
  }
  __syncthreads();
  const int32_t excl = x - v + (warp ? warp_tot[warp - 1] : 0);
  if (j < C) start[bh * (C + 1) + j] = excl;
  if (j == C - 1) start[bh * (C + 1) + C] = excl + v;
}

// pos[bh][t] = padded row of token t: its cluster's start, the members in
// earlier tiles, and the members before it in its own tile (stable).
__global__ void __launch_bounds__(kTile) position_kernel(const int32_t *__restrict__ label,
                                                         int64_t N, int C, int ntile,
                                                         const int32_t *__restrict__ hist,
                                                         const int32_t *__restrict__ start,
                                                         int32_t *__restrict__ pos,
                                                         int32_t *__restrict__ inv, int64_t Np) {
  __shared__ int32_t lab[kTile];
  const int64_t bh = blockIdx.x / ntile;
  const int tile = blockIdx.x % ntile;
  const int64_t t = static_cast<int64_t>(tile) * kTile + threadIdx.x;
  lab[threadIdx.x] = t < N ? label[bh * N + t] : -1;
  __syncthreads();
  if (t >= N) return;
  const int32_t l = lab[threadIdx.x];
  int rank = 0;
  for (int i = 0; i < static_cast<int>(threadIdx.x); ++i) rank += lab[i] == l;
  const int32_t p = start[bh * (C + 1) + l] + hist[(bh * ntile + tile) * C + l] + rank;
  pos[bh * N + t] = p;
  inv[bh * Np + p] = static_cast<int32_t>(t);
}

// xp[bh][r] = x[bh][inv[r]] (16-byte vectors; vec = d/8 lanes per row, so a
// warp moves 32/vec rows at a time); padding rows zero.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4 *__restrict__ x,
                                                          const int32_t *__restrict__ inv,
                                                          int64_t BH, int64_t N, int64_t Np,
                                                          int vec, uint4 *__restrict__ xp) {
  const int lane = threadIdx.x & 31;
  const int per = 32 / vec, sub = lane / vec, col = lane % vec;
  const int64_t warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t r0 = ((static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5) * per;
       r0 < BH * Np; r0 += warps * per) {
    const int64_t r = r0 + sub;
    if (r < BH * Np) {
      const int64_t bh = r / Np;
      const int32_t t = inv[r];
      xp[r * vec + col] = t >= 0 ? __ldg(x + (bh * N + t) * vec + col) : make_uint4(0, 0, 0, 0);
    }
  }
}

// Member means in fp64, the members read through the inverse map of the
// permutation (position -> token); an empty cluster keeps its centroid.  A
// CTA per cluster: each of its 8 warps sums a contiguous eighth of the
// members (d/8 lanes read a row's 16-byte vectors, so a warp covers 256/d
// rows per step, four steps in flight), each lane keeping 8 fp64 column
// sums; the warps' partial sums are added in warp order, so the result does
// not depend on scheduling.
template <int D>
__global__ void __launch_bounds__(256)
    centroid_update_kernel(const uint4 *__restrict__ x, const int32_t *__restrict__ inv,
                           const int32_t *__restrict__ start, const int32_t *__restrict__ count,
                           int64_t BH, int64_t N, int C, int64_t Np, float *__restrict__ cent) {
  constexpr int kLanesPerRow = D / 8;
  constexpr int kRowsPerStep = 32 / kLanesPerRow;
  constexpr int kWarps = 8;
  __shared__ double part[kWarps][D];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane / kLanesPerRow, col = lane % kLanesPerRow;
  const int64_t w = blockIdx.x;                 // cluster bh * C + j
  if (w >= BH * C) return;
  const int64_t bh = w / C;
  const int j = static_cast<int>(w % C);
  const int32_t n = count[w];
  if (n == 0) return;
  const int32_t s0 = start[bh * (C + 1) + j];
  const int32_t chunk = (n + kWarps - 1) / kWarps;
  const int32_t lo = warp * chunk < n ? warp * chunk : n;
  const int32_t hi = lo + chunk < n ? lo + chunk : n;
  double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  const int32_t *members = inv + bh * Np + s0;      // token of each member, in order
  const uint4 *head = x + bh * N * kLanesPerRow + col;
  auto add = [&](const uint4 v) {
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[2 * e] += static_cast<double>(__uint_as_float(u[e] << 16));
      acc[2 * e + 1] += static_cast<double>(__uint_as_float(u[e] & 0xFFFF0000u));
    }
  };
  int32_t m = lo + sub;
  for (; m + 3 * kRowsPerStep < hi; m += 4 * kRowsPerStep) {
    int32_t t[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) t[k] = members[m + k * kRowsPerStep];
    uint4 v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] = __ldg(head + static_cast<int64_t>(t[k]) * kLanesPerRow);
#pragma unroll
    for (int k = 0; k < 4; ++k) add(v[k]);
  }
  for (; m < hi; m += kRowsPerStep)
    add(__ldg(head + static_cast<int64_t>(members[m]) * kLanesPerRow));
#pragma unroll
  for (int off = kLanesPerRow; off < 32; off <<= 1)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xFFFFFFFFu, acc[e], off);
  if (sub == 0) {
#pragma unroll
    for (int e = 0; e < 8; ++e) part[warp][col * 8 + e] = acc[e];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < D; i += blockDim.x) {
    double t = 0.0;
#pragma unroll
    for (int k = 0; k < kWarps; ++k) t += part[k][i];
    cent[w * D + i] = static_cast<float>(t / n);
  }
}

// ------------------------------------------------------------------ centroid top-p
// One CTA per (bh, query cluster): fp64 estimated attention over the key
// clusters, a_j = n_j exp(cq.ck_j / sqrt(d) - max), sorted by (a desc, j asc)
// with a bitonic sort in SMEM, kept while the mass before stays below p (all
// when p >= 1).  keep[bh][i][j].
__global__ void __launch_bounds__(256)
    centroid_topp_kernel(const float *__restrict__ cq, const float *__restrict__ ck,
                         const int32_t *__restrict__ nk, int Cq, int Ck, int d, double p,
                         uint8_t *__restrict__ keep) {
  __shared__ double s_q[256];
  __shared__ double s_a[kMaxClusters];
  __shared__ int32_t s_j[kMaxClusters];
  __shared__ double s_red[8];
  const int64_t bh = blockIdx.x / Cq;
  const int i = blockIdx.x % Cq;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int e = threadIdx.x; e < d; e += blockDim.x) s_q[e] = cq[(bh * Cq + i) * d + e];
  __syncthreads();
  int n2 = 1;
  while (n2 < Ck) n2 <<= 1;
  const double inv_sqrt_d = 1.0 / sqrt(static_cast<double>(d));
  // a warp per key cluster: coalesced reads of its centroid, fp64 products
  for (int j = warp; j < n2; j += 8) {
    double a = -INFINITY;
    if (j < Ck && nk[bh * Ck + j] > 0) {
      const float *kr = ck + (bh * Ck + j) * d;
      double dot = 0.0;
      for (int e = lane; e < d; e += 32) dot += s_q[e] * static_cast<double>(kr[e]);
#pragma unroll
      for (int o = 16; o; o >>= 1) dot += __shfl_xor_sync(0xFFFFFFFFu, dot, o);
      a = dot * inv_sqrt_d;
    }
    if (lane == 0) {
      s_a[j] = a;
      s_j[j] = j;
    }
  }
  __syncthreads();
  double m = -INFINITY;
  for (int j = threadIdx.x; j < n2; j += blockDim.x) m = fmax(m, s_a[j]);
#pragma unroll
  for (int o = 16; o; o >>= 1) m = fmax(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if (lane == 0) s_red[warp] = m;
  __syncthreads();
  m = s_red[0];
  for (int w = 1; w < 8; ++w) m = fmax(m, s_red[w]);
  __syncthreads();
  for (int j = threadIdx.x; j < n2; j += blockDim.x)
    s_a[j] = (j < Ck && s_a[j] != -INFINITY) ? static_cast<double>(nk[bh * Ck + j]) * exp(s_a[j] - m)
                                               : 0.0;
  __syncthreads();
  // sort by (a desc, j asc); padding entries (a = 0, j >= Ck) sort last
  for (int size = 2; size <= n2; size <<= 1)
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int x = threadIdx.x; x < n2; x += blockDim.x) {
        const int y = x ^ stride;
        if (y > x) {
          const bool up = (x & size) == 0;
          const bool x_first = s_a[x] > s_a[y] || (s_a[x] == s_a[y] && s_j[x] < s_j[y]);
          if (x_first != up) {
            const double ta = s_a[x];
            s_a[x] = s_a[y];
            s_a[y] = ta;
            const int32_t tj = s_j[x];
            s_j[x] = s_j[y];
            s_j[y] = tj;
          }
        }
      }
      __syncthreads();
    }
  uint8_t *kr = keep + (bh * Cq + i) * static_cast<int64_t>(Ck);
  if (threadIdx.x == 0) {
    double z = 0.0;
    for (int x = 0; x < Ck; ++x) z += s_a[x];
    const double target = p * z;
    double mass = 0.0;
    for (int x = 0; x < Ck; ++x) kr[x] = 0;
    for (int x = 0; x < Ck; ++x) {
      if (p < 1.0 && mass >= target) break;
      kr[s_j[x]] = 1;
      mass += s_a[x];
    }
  }
}

// ------------------------------------------------------------------ block CSR
// Blocks of one query cluster share a row list: the blocks of its kept key
// clusters, ascending.  rowcnt[bh][b] for every padded query block b.
__global__ void cluster_rowcount_kernel(const uint8_t *__restrict__ keep,
                                        const int32_t *__restrict__ startq,
                                        const int32_t *__restrict__ countk, int64_t BH, int Cq,
                                        int Ck, int Nbp, int32_t *__restrict__ rowcnt) {
  const int64_t r = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (r >= BH * Nbp) return;
  const int64_t bh = r / Nbp;
  const int b = static_cast<int>(r % Nbp);
  const int32_t *sq = startq + bh * (Cq + 1);
  int cnt = 0;
  if (b * 64 < sq[Cq]) {
    int lo = 0, hi = Cq;                       // last cluster with start <= 64 b
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (sq[mid] <= b * 64) lo = mid; else hi = mid;
    }
    const uint8_t *kr = keep + (bh * Cq + lo) * static_cast<int64_t>(Ck);
    for (int j = 0; j < Ck; ++j)
      if (kr[j]) cnt += (countk[bh * Ck + j] + 63) / 64;
  }
  rowcnt[r] = cnt;
}

__global__ void __launch_bounds__(1024) exclusive_scan_kernel(const int32_t *__restrict__ in,
                                                              int64_t n,
                                                              int64_t *__restrict__ out) {
  __shared__ int64_t warp_tot[32];
  __shared__ int64_t carry;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int64_t base = 0; base < n; base += 1024) {
    const int64_t i = base + threadIdx.x;
    const int64_t v = i < n ? in[i] : 0;
    int64_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t y = __shfl_up_sync(0xFFFFFFFFu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int64_t w = warp_tot[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int64_t y = __shfl_up_sync(0xFFFFFFFFu, w, o);
        if (lane >= o) w += y;
      }
      warp_tot[lane] = w;
    }
    __syncthreads();
    const int64_t incl = x + (warp ? warp_tot[warp - 1] : 0);
    if (i < n) out[i] = carry + incl - v;
    __syncthreads();
    if (threadIdx.x == 1023) carry += incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) out[n] = carry;
}

__global__ void cluster_cols_kernel(const uint8_t *__restrict__ keep,
                                    const int32_t *__restrict__ startq,
                                    const int32_t *__restrict__ startk,
                                    const int32_t *__restrict__ countk,
                                    const int64_t *__restrict__ row_ptr, int64_t BH, int Cq,
                                    int Ck, int Nbp, int32_t *__restrict__ col_idx) {
  const int64_t r = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (r >= BH * Nbp) return;
  int64_t p = row_ptr[r];
  if (row_ptr[r + 1] == p) return;
  const int64_t bh = r / Nbp;
  const int b = static_cast<int>(r % Nbp);
  const int32_t *sq = startq + bh * (Cq + 1);
  int lo = 0, hi = Cq;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (sq[mid] <= b * 64) lo = mid; else hi = mid;
  }
  const uint8_t *kr = keep + (bh * Cq + lo) * static_cast<int64_t>(Ck);
  for (int j = 0; j < Ck; ++j) {
    if (!kr[j]) continue;
    const int first = startk[bh * (Ck + 1) + j] / 64;
    const int nblk = (countk[bh * Ck + j] + 63) / 64;
    for (int k = 0; k < nblk; ++k) col_idx[p++] = first + k;
  }
}

// valid keys of each padded key block: 64, a cluster's partial last block, or
// 0 past the last cluster.
__global__ void key_valid_kernel(const int32_t *__restrict__ startk,
                                 const int32_t *__restrict__ countk, int64_t BH, int Ck, int Nbp,
                                 int32_t *__restrict__ kvalid) {
  const int64_t r = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (r >= BH * Nbp) return;
  const int64_t bh = r / Nbp;
  const int b = static_cast<int>(r % Nbp);
  const int32_t *sk = startk + bh * (Ck + 1);
  int v = 0;
  if (b * 64 < sk[Ck]) {
    int lo = 0, hi = Ck;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (sk[mid] <= b * 64) lo = mid; else hi = mid;
    }
    const int rem = countk[bh * Ck + lo] - (b * 64 - sk[lo]);
    v = rem >= 64 ? 64 : (rem > 0 ? rem : 0);
  }
  kvalid[r] = v;
}

// o[bh][t] = op[bh][pos[t]], lse likewise (a warp per token).
__global__ void __launch_bounds__(256) unpermute_kernel(const uint4 *__restrict__ op,
                                                        const float *__restrict__ lsep,
                                                        const int32_t *__restrict__ pos,
                                                        int64_t BH, int64_t N, int64_t Np,
                                                        int vec, uint4 *__restrict__ o,
                                                        float *__restrict__ lse) {
  const int lane = threadIdx.x & 31;
  const int per = 32 / vec, sub = lane / vec, col = lane % vec;   // 32/vec rows per warp
  const int64_t warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t r0 = ((static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5) * per;
       r0 < BH * N; r0 += warps * per) {
    const int64_t r = r0 + sub;
    if (r < BH * N) {
      const int64_t bh = r / N;
      const int64_t src = bh * Np + pos[r];
      o[r * vec + col] = op[src * vec + col];
      if (col == 0) lse[r] = lsep[src];
    }
  }
}

// Initial centroids: the token floor(j*N/C) of each head, widened to fp32.
__global__ void init_centroids_kernel(const __nv_bfloat16 *__restrict__ x, int64_t BH, int64_t N,
                                      int C, int d, float *__restrict__ cent) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= BH * C * d) return;
  const int e = static_cast<int>(i % d);
  const int64_t j = (i / d) % C, bh = i / (static_cast<int64_t>(C) * d);
  const int64_t t = j * N / C;
  cent[i] = __bfloat162float(x[(bh * N + t) * d + e]);
}

// ------------------------------------------------------------------ layout
size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct ClusterLayout {
  int Cmax, Cpad, ntile, Nbp;
  int64_t Np;
  size_t cbf, cnorm, label_q, label_k, count_q, count_k, hist, start_q, start_k, pos_q, pos_k,
      inv, xq, xk, xv, cent_q, cent_k, keep, rowcnt, row_ptr, col_idx, kvalid, op, lsep, attn,
      total;
  Geometry gp;   // the padded sequence as a token grid (T = Np/64 frames of 8 x 8)
};

ClusterLayout cluster_layout(const Geometry &g, const vsa_cluster_params &c) {
  ClusterLayout L;
  L.Cmax = c.Cq > c.Ck ? c.Cq : c.Ck;
  L.Cpad = ((L.Cmax + 127) / 128) * 128;
  L.ntile = static_cast<int>((g.N + kTile - 1) / kTile);
  L.Np = g.N + 64LL * L.Cmax;
  L.Nbp = static_cast<int>(L.Np / 64);
  vsa_shape sp{static_cast<int32_t>(g.BH), 1, static_cast<int32_t>(L.Nbp), 8, 8, g.d, 8};
  L.gp = geometry(sp);
  const size_t BH = static_cast<size_t>(g.BH), N = static_cast<size_t>(g.N),
               Np = static_cast<size_t>(L.Np), d = static_cast<size_t>(g.d);
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t o = off; off = align256(off + bytes); return o; };
  L.cbf = take(BH * L.Cpad * d * 2);
  L.cnorm = take(BH * L.Cpad * 4);
  L.label_q = take(BH * N * 4);
  L.label_k = take(BH * N * 4);
  L.count_q = take(BH * c.Cq * 4);
  L.count_k = take(BH * c.Ck * 4);
  L.hist = take(BH * L.ntile * L.Cmax * 4);
  L.start_q = take(BH * (c.Cq + 1) * 4);
  L.start_k = take(BH * (c.Ck + 1) * 4);
  L.pos_q = take(BH * N * 4);
  L.pos_k = take(BH * N * 4);
  L.inv = take(BH * Np * 4);
  L.xq = take(BH * Np * d * 2);
  L.xk = take(BH * Np * d * 2);
  L.xv = take(BH * Np * d * 2);
  L.cent_q = take(BH * c.Cq * d * 4);
  L.cent_k = take(BH * c.Ck * d * 4);
  L.keep = take(BH * c.Cq * c.Ck);
  L.rowcnt = take(BH * L.Nbp * 4);
  L.row_ptr = take((BH * L.Nbp + 1) * 8);
  L.col_idx = take(BH * static_cast<size_t>(L.Nbp) * L.Nbp * 4);
  L.kvalid = take(BH * L.Nbp * 4);
  L.op = take(BH * Np * d * 2);
  L.lsep = take(BH * Np * 4);
  L.attn = take(sparse_attn_workspace_bytes(L.gp));
  L.total = off;
  return L;
}

int grid_for(int64_t warps_or_threads, int per_block, int cap_per_sm) {
  const int64_t want = (warps_or_threads + per_block - 1) / per_block;
  const int64_t cap = static_cast<int64_t>(cap_per_sm) * num_sms();
  return static_cast<int>(want < cap ? want : cap);
}

}  // namespace

size_t cluster_workspace_bytes(const Geometry &g, const vsa_cluster_params &c) {
  return cluster_layout(g, c).total;
}

// One tensor through k-means from the centroids already in the workspace:
// `iters` rounds of assign + permute + update, then the final assignment and
// permutation.  Leaves labels, counts, starts, positions, the
// permuted tensor and the centroids in the workspace.
static cudaError_t run_kmeans(const void *x, const Geometry &g, int C, int iters,
                              const ClusterLayout &L, unsigned char *w,
                              size_t label_off, size_t count_off, size_t start_off,
                              size_t pos_off, size_t xp_off, size_t cent_off, unsigned *err,
                              cudaStream_t st) {
  const int64_t BH = g.BH, N = g.N, Np = L.Np;
  const int d = g.d;
  float *cent = reinterpret_cast<float *>(w + cent_off);
  int32_t *label = reinterpret_cast<int32_t *>(w + label_off);
  int32_t *count = reinterpret_cast<int32_t *>(w + count_off);
  int32_t *start = reinterpret_cast<int32_t *>(w + start_off);
  int32_t *pos = reinterpret_cast<int32_t *>(w + pos_off);
  int32_t *inv = reinterpret_cast<int32_t *>(w + L.inv);
  int32_t *hist = reinterpret_cast<int32_t *>(w + L.hist);
  __nv_bfloat16 *cbf = reinterpret_cast<__nv_bfloat16 *>(w + L.cbf);
  float *cnorm = reinterpret_cast<float *>(w + L.cnorm);
  void *xp = w + xp_off;
  cudaError_t e;
  CUtensorMap tx, tc;
  if (!make_map4(&tx, x, BH * N, d) || !make_map4(&tc, cbf, BH * L.Cpad, d))
    return cudaErrorInvalidValue;
  const int tiles_per_head = static_cast<int>((N + 127) / 128);
  const int smem = d == 128 ? AssignSmem<128>::kBytes : AssignSmem<64>::kBytes;
  const void *fn = d == 128 ? reinterpret_cast<const void *>(kmeans_assign_kernel<128>)
                            : reinterpret_cast<const void *>(kmeans_assign_kernel<64>);
  if ((e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem + 1024)) !=
      cudaSuccess)
    return e;
  const int vec = d / 8;
  for (int it = 0; it <= iters; ++it) {
    centroid_prep_kernel<<<static_cast<int>((BH * L.Cpad * 32 + 255) / 256), 256, 0, st>>>(
        cent, BH * L.Cpad, C, L.Cpad, d, cbf, cnorm);
    if (d == 128)
      kmeans_assign_kernel<128><<<static_cast<int>(BH * tiles_per_head), 128, smem + 1024, st>>>(
          tx, tc, cnorm, N, L.Cpad, tiles_per_head, label, nullptr, err);
    else
      kmeans_assign_kernel<64><<<static_cast<int>(BH * tiles_per_head), 128, smem + 1024, st>>>(
          tx, tc, cnorm, N, L.Cpad, tiles_per_head, label, nullptr, err);
    tile_hist_kernel<<<static_cast<int>(BH * L.ntile), kTile, 0, st>>>(label, N, C, L.ntile,
                                                                        hist);
    tile_scan_kernel<<<static_cast<int>((BH * C + 255) / 256), 256, 0, st>>>(hist, BH, C, L.ntile,
                                                                          count);
    cluster_start_kernel<<<static_cast<int>(BH), 1024, 0, st>>>(count, C, start);
    if ((e = cudaMemsetAsync(inv, 0xFF, static_cast<size_t>(BH) * Np * 4, st)) != cudaSuccess)
      return e;
    position_kernel<<<static_cast<int>(BH * L.ntile), kTile, 0, st>>>(label, N, C, L.ntile, hist,
                                                                       start, pos, inv, Np);
    if (it < iters) {
      const int ub = static_cast<int>(BH * C);      // a CTA per cluster
      const uint4 *x4 = static_cast<const uint4 *>(x);
      if (d == 128)
        centroid_update_kernel<128><<<ub, 256, 0, st>>>(x4, inv, start, count, BH, N, C, Np,
                                                          cent);
      else
        centroid_update_kernel<64><<<ub, 256, 0, st>>>(x4, inv, start, count, BH, N, C, Np,
                                                         cent);
    } else {
      // the final permutation: the permuted, padded tensor itself
      gather_rows_kernel<<<grid_for(BH * Np * 32, 256, 32), 256, 0, st>>>(
          static_cast<const uint4 *>(x), inv, BH, N, Np, vec, static_cast<uint4 *>(xp));
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}


cudaError_t launch_cluster_attn(const void *q, const void *k, const void *v, const Geometry &g,
                                const vsa_cluster_params &c, float scale, const float *init_q,
                                const float *init_k, void *o, float *lse,
                                const vsa_cluster_state *out_state, void *ws, unsigned *err,
                                cudaStream_t st, const char **why) {
  const ClusterLayout L = cluster_layout(g, c);
  unsigned char *w = static_cast<unsigned char *>(ws);
  const int64_t BH = g.BH, N = g.N, Np = L.Np;
  const int d = g.d;
  cudaError_t e;
  float *cent_q = reinterpret_cast<float *>(w + L.cent_q);
  float *cent_k = reinterpret_cast<float *>(w + L.cent_k);
  // initial centroids: the given ones (a cache from an earlier call), else
  // evenly spaced tokens
  const struct { const float *init; const void *x; int C; float *cent; } inits[2] = {
      {init_q, q, c.Cq, cent_q}, {init_k, k, c.Ck, cent_k}};
  for (const auto &in : inits) {
    if (in.init)
      e = cudaMemcpyAsync(in.cent, in.init, static_cast<size_t>(BH) * in.C * d * 4,
                          cudaMemcpyDeviceToDevice, st);
    else {
      init_centroids_kernel<<<static_cast<int>((BH * in.C * d + 255) / 256), 256, 0, st>>>(
          static_cast<const __nv_bfloat16 *>(in.x), BH, N, in.C, d, in.cent);
      e = cudaGetLastError();
    }
    if (e != cudaSuccess) return e;
  }
  if ((e = run_kmeans(q, g, c.Cq, c.iters, L, w, L.label_q, L.count_q, L.start_q, L.pos_q,
                      L.xq, L.cent_q, err, st)) != cudaSuccess) {
    *why = "cluster attention: k-means on Q";
    return e;
  }
  if ((e = run_kmeans(k, g, c.Ck, c.iters, L, w, L.label_k, L.count_k, L.start_k, L.pos_k,
                      L.xk, L.cent_k, err, st)) != cudaSuccess) {
    *why = "cluster attention: k-means on K";
    return e;
  }
  // V follows K's permutation (inv still holds K's inverse map)
  int32_t *inv = reinterpret_cast<int32_t *>(w + L.inv);
  gather_rows_kernel<<<grid_for(BH * Np * 32, 256, 32), 256, 0, st>>>(
      static_cast<const uint4 *>(v), inv, BH, N, Np, d / 8, reinterpret_cast<uint4 *>(w + L.xv));
  // the centroids that the final labels were assigned with
  const int32_t *count_k = reinterpret_cast<const int32_t *>(w + L.count_k);
  const int32_t *start_q = reinterpret_cast<const int32_t *>(w + L.start_q);
  const int32_t *start_k = reinterpret_cast<const int32_t *>(w + L.start_k);
  uint8_t *keep = reinterpret_cast<uint8_t *>(w + L.keep);
  centroid_topp_kernel<<<static_cast<int>(BH * c.Cq), 256, 0, st>>>(
      cent_q, cent_k, count_k, c.Cq, c.Ck, d, static_cast<double>(c.p), keep);
  int32_t *rowcnt = reinterpret_cast<int32_t *>(w + L.rowcnt);
  int64_t *row_ptr = reinterpret_cast<int64_t *>(w + L.row_ptr);
  int32_t *col_idx = reinterpret_cast<int32_t *>(w + L.col_idx);
  int32_t *kvalid = reinterpret_cast<int32_t *>(w + L.kvalid);
  const int64_t rows = BH * L.Nbp;
  cluster_rowcount_kernel<<<static_cast<int>((rows + 255) / 256), 256, 0, st>>>(
      keep, start_q, count_k, BH, c.Cq, c.Ck, L.Nbp, rowcnt);
  exclusive_scan_kernel<<<1, 1024, 0, st>>>(rowcnt, rows, row_ptr);
  cluster_cols_kernel<<<static_cast<int>((rows + 255) / 256), 256, 0, st>>>(
      keep, start_q, start_k, count_k, row_ptr, BH, c.Cq, c.Ck, L.Nbp, col_idx);
  key_valid_kernel<<<static_cast<int>((rows + 255) / 256), 256, 0, st>>>(start_k, count_k, BH,
                                                                        c.Ck, L.Nbp, kvalid);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  e = launch_sparse_attn(w + L.xq, w + L.xk, w + L.xv, row_ptr, col_idx, L.gp, scale, w + L.op,
                         reinterpret_cast<float *>(w + L.lsep), w + L.attn, err, st, why, nullptr,
                         0, kvalid);
  if (e != cudaSuccess) return e;
  unpermute_kernel<<<grid_for(BH * N * 32, 256, 32), 256, 0, st>>>(
      reinterpret_cast<const uint4 *>(w + L.op), reinterpret_cast<const float *>(w + L.lsep),
      reinterpret_cast<const int32_t *>(w + L.pos_q), BH, N, Np, d / 8, static_cast<uint4 *>(o),
      lse);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (out_state) {
    struct Copy { void *dst; size_t off, bytes; } copies[] = {
        {out_state->q_labels, L.label_q, static_cast<size_t>(BH) * N * 4},
        {out_state->k_labels, L.label_k, static_cast<size_t>(BH) * N * 4},
        {out_state->q_counts, L.count_q, static_cast<size_t>(BH) * c.Cq * 4},
        {out_state->k_counts, L.count_k, static_cast<size_t>(BH) * c.Ck * 4},
        {out_state->q_centroids, L.cent_q, static_cast<size_t>(BH) * c.Cq * d * 4},
        {out_state->k_centroids, L.cent_k, static_cast<size_t>(BH) * c.Ck * d * 4},
        {out_state->keep, L.keep, static_cast<size_t>(BH) * c.Cq * c.Ck},
    };
    for (const Copy &cp : copies)
      if (cp.dst &&
          (e = cudaMemcpyAsync(cp.dst, w + cp.off, cp.bytes, cudaMemcpyDeviceToDevice, st)) !=
              cudaSuccess)
        return e;
  }
  return cudaSuccess;
}

}  // namespace vsa
