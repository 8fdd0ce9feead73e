// k_mask.cu -- content-adaptive block mask (NABLA, Methodology item 2:
// reduced attention over pooled blocks and the per-row CDF threshold; item 3:
// union with the sliding-tile window; Sparse VideoGen2 section 2B: top-p).
//
// Four kernels:
//   mask_scores_kernel  persistent; one work unit = 64 query blocks x 128 key
//                       blocks of one (batch, head), units split evenly over
//                       the CTAs.  Forms the pooled scores with fp64
//                       tensor-core MMAs (m8n8k4), K streamed in slices,
//                       writes each tile's row maxima in fp64 and
//                       2^(t - tile max) as fp32 to the workspace slab.
//   mask_select_kernel  one warp per row: rescales the slab row to the row
//                       maximum, finds the CDF cut (histogram of the top 8
//                       octaves + exact fp64 check + warp sort of the cut
//                       bin, or bisection on the fp32 bit pattern with fp64
//                       mass tests), breaks ties by index, ORs in the STA
//                       window and writes a kept-bit row and its count.  Small
//                       SMEM per warp, so many rows are in flight per SM.
//   chunk_sums_kernel, chunk_scan_kernel
//                       exclusive scan of the counts into row_ptr (int64).
//   expand_bits_kernel  kept bits -> ascending col_idx lists.
//
// Precision: scores are exact fp64 dot products of exact pooled means; each
// probability carries a relative error of a few 1e-7 (fp32 storage and the
// hardware exp2 on a reduced argument), so the kept set equals the exact one
// except for rows whose cut is within that of 1 - thr or of a tie.
#include "vsa_device.cuh"
#include "vsa_internal.h"

#include <cmath>
#include <type_traits>

namespace vsa {
namespace {

constexpr int kRT = 64;       // query blocks per work item
constexpr int kCT = 128;      // key blocks per phase-A column tile
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kPad = 4;       // fp64 padding per smem row (conflict-free fragments)
constexpr int kKS = 32;       // columns of d per K slice in the score kernel
constexpr int kLdK = kKS + kPad;
constexpr int kCand = 256;    // per-warp candidate list capacity
constexpr int kBins = 64;     // 1/8-octave probability bins (8 octaves below the max)
constexpr int kMaxWords = 256;  // kept-bit words per row held in SMEM (Nb <= 8192)
constexpr int kOctaves = 256;   // fp32 exponent bins of the static-ratio selection
constexpr int kMaxGrid = 160; // persistent score CTAs

struct MaskArgs {
  const double *qp, *kp;
  int64_t BH;
  int Nb, d, Hb, Wb;
  float thr;
  int use_sta, rt, rh, rw;
  double c;          // scale * log2(e)
  float *slab;       // [BH*Nb][ld_slab]
  double *tmax;      // [BH*Nb][ntiles]
  int ld_slab, ntiles;
  uint32_t *bits;    // [BH*Nb][words]
  int words;
  int32_t *counts;   // [BH*Nb]
  int64_t items, tiles_per_head;
  int k;             // static-ratio selection: blocks kept per row (0: top-p)
};

__device__ __forceinline__ void dmma(double (&c)[2], double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
               : "+d"(c[0]), "+d"(c[1])
               : "d"(a), "d"(b));
}

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, bool valid) {
  const uint32_t s = smem_u32(smem);
  const int n = valid ? 16 : 0;  // src size 0 -> zero fill
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}
__device__ __forceinline__ double warp_max(double v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmax(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}
__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// 2^x for x <= 0 in fp64 argument, fp32 result with relative error ~2e-7:
// split x = n + f with f in [0, 1), hardware exp2 of f, exact scaling by 2^n.
__device__ __forceinline__ float exp2_split(double x) {
  if (!(x > -126.0)) return 0.0f;  // also maps -inf / NaN to 0
  const double n = floor(x);
  const float f = static_cast<float>(x - n);
  return ex2(f) * __int_as_float((static_cast<int>(n) + 127) << 23);
}

// key = bits of a probability in [0, 1]; bin 0 holds (7/8, 1], each bin is
// 1/8 octave; kBins (the tail) collects everything more than 8 octaves down.
__device__ __forceinline__ int prob_bin(uint32_t key) {
  const uint32_t d = key < 0x3F800000u ? 0x3F800000u - key : 0u;
  const uint32_t b = d >> 20;
  return b < static_cast<uint32_t>(kBins) ? static_cast<int>(b) : kBins;
}

// A row's probabilities relative to the row maximum: the slab entry (fp32
// 2^(s - tile max), L2-resident) times its tile's fp32 rescale factor.  Read
// again wherever a pass needs them rather than kept in SMEM, so that many
// more rows fit on an SM; the product is the same every time.
struct RowView {
  const float *slab;
  const float *ts;
  __device__ __forceinline__ float operator()(int c) const { return slab[c] * ts[c / kCT]; }
};
// The same values kept in SMEM by the first pass (rows short enough that the
// copy costs little occupancy).
struct SmemRow {
  const float *e;
  __device__ __forceinline__ float operator()(int c) const { return e[c]; }
};
constexpr int kSmemRowMaxNb = 2048;   // rows up to this many blocks stay in SMEM

// The cut by bisection on the fp32 bit pattern, mass tests in fp64.  Sets
// vkey (cut value) and need_ties, or keep_all when the sums never reach the
// target.  General path; used when the histogram path cannot decide.
template <class Row>
__device__ void cut_by_bisection(int Nb, Row ebuf, uint32_t kmax, double target,
                                 uint32_t *cand_key, int32_t *cand_idx, uint32_t &vkey,
                                 int &need_ties, bool &keep_all) {
  const int lane = threadIdx.x & 31;
  // Invariant: the cut key lies in [lo, hi); mass(key >= hi) = base < target.
  uint32_t lo = 0, hi = kmax + 1;
  double base = 0.0;
  int ncand = -1;  // -1: scan the whole row
  for (int it = 0; hi - lo > 1; ++it) {
    const uint32_t mid = lo + ((hi - lo) >> 1);
    double up = 0.0;
    if (ncand < 0) {
      for (int c = lane; c < Nb; c += 32) {
        const float e = ebuf(c);
        const uint32_t k = __float_as_uint(e);
        if (k >= mid && k < hi) up += static_cast<double>(e);
      }
    } else {
      for (int i = lane; i < ncand; i += 32) {
        const uint32_t k = cand_key[i];
        if (k >= mid && k < hi) up += static_cast<double>(__uint_as_float(k));
      }
    }
    up = warp_sum(up);
    if (base + up >= target) {
      lo = mid;
    } else {
      base += up;
      hi = mid;
    }
    if (ncand < 0 && it >= 5) {
      int cnt = 0;
      for (int c = lane; c < Nb; c += 32) {
        const uint32_t k = __float_as_uint(ebuf(c));
        cnt += (k >= lo && k < hi);
      }
      cnt = warp_sum_i(cnt);
      if (cnt <= kCand) {
        int pos = 0;
        for (int c0 = 0; c0 < Nb; c0 += 32) {
          const int c = c0 + lane;
          const uint32_t k = c < Nb ? __float_as_uint(ebuf(c)) : 0u;
          const bool in = c < Nb && k >= lo && k < hi;
          const uint32_t m = __ballot_sync(0xFFFFFFFFu, in);
          if (in) {
            const int p = pos + __popc(m & ((1u << lane) - 1u));
            cand_key[p] = k;
            cand_idx[p] = c;
          }
          pos += __popc(m);
        }
        ncand = pos;
        __syncwarp();
      }
    }
  }
  vkey = lo;
  if (vkey == 0u) {
    keep_all = true;  // the sums never reach 1 - thr: keep every block
  } else {
    const double v = static_cast<double>(__uint_as_float(vkey));
    int j = static_cast<int>(ceil((target - base) / v));
    if (j < 1) j = 1;
    while (j > 1 && base + (j - 1) * v >= target) --j;
    while (base + j * v < target && j < Nb) ++j;
    need_ties = j;
  }
}

// Phase B for one row: selection and kept bits.  ebuf: the row's probabilities
// relative to the row max, re-read from the slab (RowView).
//   1. those probabilities, their fp64 sum, and a
//      histogram of counts / fp32 masses over 1/8-octave bins;
//   2. the bin b where the cumulative mass reaches 1 - thr; an exact fp64 pass
//      confirms base = mass above b < target <= base + mass of b and collects
//      the bin's entries;
//   3. with at most 32 entries: a warp bitonic sort on (probability desc,
//      index asc) and an fp64 prefix scan mark the kept ones.  Otherwise (or
//      if the fp32 histogram misled step 2) the bisection path decides.
// Shared end of both selections: OR in the STA window, write the kept-bit
// row and its count.  wbits holds the selection's bits (warp-synchronised).
__device__ void finish_row(const MaskArgs &a, int64_t grow, int r, uint32_t *wbits) {
  const int lane = threadIdx.x & 31;
  const int Nb = a.Nb;
  if (a.use_sta) {
    // the window: at most (2rt+1)(2rh+1)(2rw+1) blocks around the row's own
    const int hw = a.Hb * a.Wb;
    const int tr = r / hw, yr = (r / a.Wb) % a.Hb, xr = r % a.Wb;
    const int nt = 2 * a.rt + 1, ny = 2 * a.rh + 1, nx = 2 * a.rw + 1;
    const int T = Nb / hw;
    for (int i = lane; i < nt * ny * nx; i += 32) {
      const int t = tr - a.rt + i / (ny * nx);
      const int y = yr - a.rh + (i / nx) % ny;
      const int x = xr - a.rw + i % nx;
      if (t >= 0 && t < T && y >= 0 && y < a.Hb && x >= 0 && x < a.Wb) {
        const int c = (t * a.Hb + y) * a.Wb + x;
        atomicOr(&wbits[c >> 5], 1u << (c & 31));
      }
    }
    __syncwarp();
  }
  uint32_t *out = a.bits + grow * a.words;
  int count = 0;
  for (int w = lane; w < a.words; w += 32) {
    const uint32_t word = wbits[w];
    out[w] = word;
    count += __popc(word);
  }
  count = warp_sum_i(count);
  if (lane == 0) a.counts[grow] = count;
  __syncwarp();
}

template <bool kSmemRow>
__device__ void select_row(const MaskArgs &a, int64_t grow, int r, const float *slab_row,
                           const double *tmax_row, float *erow, uint32_t *cand_key,
                           int32_t *cand_idx, float *tscale, int *hcnt, float *hmass,
                           uint32_t *wbits) {
  const int lane = threadIdx.x & 31;
  const int Nb = a.Nb;
  // row maximum over the tile maxima, per-tile rescale factors in fp64
  double M = -INFINITY;
  for (int t = lane; t < a.ntiles; t += 32) M = fmax(M, tmax_row[t]);
  M = warp_max(M);
  for (int t = lane; t < a.ntiles; t += 32) tscale[t] = static_cast<float>(exp2(tmax_row[t] - M));
  for (int b = lane; b < kBins; b += 32) {
    hcnt[b] = 0;
    hmass[b] = 0.0f;
  }
  __syncwarp();
  using Row = typename std::conditional<kSmemRow, SmemRow, RowView>::type;
  Row ebuf;
  if constexpr (kSmemRow) ebuf = SmemRow{erow}; else ebuf = RowView{slab_row, tscale};
  const bool need_cut = a.thr > 0.0f;
  double z = 0.0;
  uint32_t kmax = 0;
  // the slab row sits in L2: 16-byte loads, four in flight per lane, before
  // any use (the row is padded to a multiple of 4 floats)
  constexpr int kU = 4;
  for (int c0 = 4 * lane; c0 < Nb; c0 += 128 * kU) {
    float4 v[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u)
      if (c0 + 128 * u < Nb) v[u] = *reinterpret_cast<const float4 *>(slab_row + c0 + 128 * u);
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const float x4[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
      // the four entries share a 128-column tile (c0 is a multiple of 4)
      const float ts = c0 + 128 * u < Nb ? tscale[(c0 + 128 * u) / kCT] : 0.0f;
      float e4[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) e4[j] = c0 + 128 * u + j < Nb ? x4[j] * ts : 0.0f;
      // row mass: fp32 sums of four, fp64 across (relative error ~1e-7)
      z += static_cast<double>((e4[0] + e4[1]) + (e4[2] + e4[3]));
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = c0 + 128 * u + j;
        if (c < Nb) {
          const float e = e4[j];
          if constexpr (kSmemRow) erow[c] = e;
          const uint32_t k = __float_as_uint(e);
          kmax = max(kmax, k);
          if (need_cut) {
            const int b = prob_bin(k);
            if (b < kBins) {         // the tail needs no histogram
              atomicAdd(&hcnt[b], 1);
              atomicAdd(&hmass[b], e);
            }
          }
        }
      }
    }
  }
  z = warp_sum(z);
#pragma unroll
  for (int o = 16; o; o >>= 1) kmax = max(kmax, __shfl_xor_sync(0xFFFFFFFFu, kmax, o));
  __syncwarp();

  bool keep_all = !need_cut;
  uint32_t vkey = 0;
  int need_ties = 0;
  int cut_bin = -1;       // >= 0: the histogram path wrote the kept bits
  if (!keep_all) {
    const double target = (1.0 - static_cast<double>(a.thr)) * z;
    // 2. cumulative bin masses (8 bins per lane, then a warp scan)
    double loc = 0.0;
#pragma unroll
    for (int i = 0; i < kBins / 32; ++i) loc += static_cast<double>(hmass[lane * (kBins / 32) + i]);
    double incl = loc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += y;
    }
    double run = incl - loc;
    int found = kBins;
#pragma unroll
    for (int i = 0; i < kBins / 32; ++i) {
      const int b = lane * (kBins / 32) + i;
      run += static_cast<double>(hmass[b]);
      if (found == kBins && run >= target) found = b;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) found = min(found, __shfl_xor_sync(0xFFFFFFFFu, found, o));
    bool decided = false;
    if (found < kBins && hcnt[found] <= 32) {
      // exact mass above the bin and the bin's entries
      double base = 0.0;
      int pos = 0;
      for (int c0 = 0; c0 < Nb; c0 += 32) {
        const int c = c0 + lane;
        const float e = c < Nb ? ebuf(c) : 0.0f;
        const int b = c < Nb ? prob_bin(__float_as_uint(e)) : kBins;
        if (b < found) base += static_cast<double>(e);
        // entries above the cut bin are kept whatever the bin's order
        const uint32_t above = __ballot_sync(0xFFFFFFFFu, b < found);
        if (lane == 0) wbits[c0 >> 5] = above;
        const bool in = b == found;
        const uint32_t m = __ballot_sync(0xFFFFFFFFu, in);
        if (in) {
          const int p = pos + __popc(m & ((1u << lane) - 1u));
          if (p < 32) {
            cand_key[p] = __float_as_uint(e);
            cand_idx[p] = c;
          }
        }
        pos += __popc(m);
      }
      base = warp_sum(base);
      __syncwarp();
      if (pos <= 32 && base < target) {
        // one entry per lane; sort by (probability desc, index asc)
        uint64_t key = ~0ull;
        if (lane < pos)
          key = (static_cast<uint64_t>(0xFFFFFFFFu - cand_key[lane]) << 32) |
                static_cast<uint32_t>(cand_idx[lane]);
#pragma unroll
        for (int size = 2; size <= 32; size <<= 1)
#pragma unroll
          for (int stride = size >> 1; stride > 0; stride >>= 1) {
            const uint64_t other = __shfl_xor_sync(0xFFFFFFFFu, key, stride);
            const bool up = (lane & size) == 0;
            const bool lower = (lane & stride) == 0;
            const uint64_t lo_v = key < other ? key : other;
            const uint64_t hi_v = key < other ? other : key;
            key = (lower == up) ? lo_v : hi_v;
          }
        const bool valid = key != ~0ull;
        const double p = valid ? static_cast<double>(__uint_as_float(0xFFFFFFFFu - static_cast<uint32_t>(key >> 32)))
                               : 0.0;
        double inc = p;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const double y = __shfl_up_sync(0xFFFFFFFFu, inc, o);
          if (lane >= o) inc += y;
        }
        const double total = __shfl_sync(0xFFFFFFFFu, inc, 31);
        if (base + total >= target) {
          // kept while the mass before the entry is still below the target
          __syncwarp();
          if (valid && base + (inc - p) < target) {
            const int c = static_cast<int>(key & 0xFFFFFFFFu);
            atomicOr(&wbits[c >> 5], 1u << (c & 31));
          }
          cut_bin = found;
          decided = true;
        }
        __syncwarp();
      }
    }
    if (!decided)
      cut_by_bisection(Nb, ebuf, kmax, target, cand_key, cand_idx, vkey, need_ties, keep_all);
  }

  // kept bits (the histogram path wrote them already): everything, or above
  // the bisection cut with ties by index
  int ties_seen = 0;
  for (int w = 0; cut_bin < 0 && w < a.words; ++w) {
    const int c = w * 32 + lane;
    const bool valid = c < Nb;
    const uint32_t k = valid ? __float_as_uint(ebuf(c)) : 0u;
    bool kept;
    if (keep_all) {
      kept = valid;
    } else {
      kept = valid && k > vkey;
      const bool tie = valid && k == vkey;
      const uint32_t tm = __ballot_sync(0xFFFFFFFFu, tie);
      if (tie && ties_seen + __popc(tm & ((1u << lane) - 1u)) < need_ties) kept = true;
      ties_seen += __popc(tm);
    }
    const uint32_t word = __ballot_sync(0xFFFFFFFFu, kept);
    if (lane == 0) wbits[w] = word;
  }
  __syncwarp();
  finish_row(a, grow, r, wbits);
}

// Work unit = (batch-head, 64-row tile, 128-column tile), numbered row-tile
// major; CTA i takes the contiguous range [i*U/G, (i+1)*U/G), so the units
// are spread evenly and a CTA meets a new row tile (and reloads Q) only a few
// times.  K comes in slices of kKS columns of d through two cp.async buffers:
// the next slice (the next unit's first one at a unit's end) is in flight
// while the current one feeds the DMMAs.
__global__ void __launch_bounds__(kThreads, 1) mask_scores_kernel(const MaskArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  double *sQ = reinterpret_cast<double *>(smem_raw);
  const int ld = a.d + kPad;
  double *sK = sQ + kRT * ld;                  // [2][kCT][kLdK]
  __shared__ double sRed[kRT][4];
  __shared__ double sTileMax[kRT];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tq = lane & 3;
  const int wm = warp >> 2, wn = warp & 3;
  const int nslices = a.d / kKS;
  const int64_t units = a.items * a.ntiles;
  const int64_t u_begin = units * blockIdx.x / gridDim.x;
  const int64_t u_end = units * (blockIdx.x + 1) / gridDim.x;
  if (u_begin >= u_end) return;

  // K slice s (columns [s*kKS, s*kKS + kKS) of d) of unit u into buffer b
  auto load_slice = [&](int64_t u, int sl, int b) {
    const int64_t item = u / a.ntiles;
    const int c0 = static_cast<int>(u % a.ntiles) * kCT;
    const double *ksrc = a.kp + (item / a.tiles_per_head) * a.Nb * a.d + sl * kKS;
    double *dst = sK + b * (kCT * kLdK);
    for (int i = tid; i < kCT * (kKS / 2); i += kThreads) {
      const int row = i / (kKS / 2), ch = i % (kKS / 2);
      const bool ok = c0 + row < a.Nb;
      cp_async16(dst + row * kLdK + ch * 2,
                 ok ? ksrc + static_cast<int64_t>(c0 + row) * a.d + ch * 2 : a.kp, ok);
    }
    cp_async_commit();
  };

  load_slice(u_begin, 0, 0);
  int buf = 0;
  int64_t q_item = -1;
  for (int64_t u = u_begin; u < u_end; ++u) {
    const int64_t item = u / a.ntiles;
    const int ct = static_cast<int>(u % a.ntiles);
    const int64_t bh = item / a.tiles_per_head;
    const int r0 = static_cast<int>(item % a.tiles_per_head) * kRT;
    const int c0 = ct * kCT;
    if (item != q_item) {
      // every warp finished the previous unit (barrier at its end)
      const double *qsrc = a.qp + (bh * a.Nb + r0) * a.d;
      const int vec_per_row = a.d / 2;
      for (int i = tid; i < kRT * vec_per_row; i += kThreads) {
        const int row = i / vec_per_row, ch = i % vec_per_row;
        const bool ok = r0 + row < a.Nb;
        cp_async16(sQ + row * ld + ch * 2, ok ? qsrc + row * a.d + ch * 2 : a.qp, ok);
      }
      cp_async_commit();
      q_item = item;
    }

    double acc[4][4][2];
#pragma unroll
    for (int mi = 0; mi < 4; ++mi)
#pragma unroll
      for (int ni = 0; ni < 4; ++ni) acc[mi][ni][0] = acc[mi][ni][1] = 0.0;
    for (int sl = 0; sl < nslices; ++sl) {
      // prefetch the next slice (the next unit's first at the last slice)
      bool more = true;
      if (sl + 1 < nslices) load_slice(u, sl + 1, buf ^ 1);
      else if (u + 1 < u_end) load_slice(u + 1, 0, buf ^ 1);
      else more = false;
      // everything but the prefetch has landed: this slice (and Q)
      if (more) cp_async_wait_group<1>();
      else cp_async_wait_group<0>();
      __syncthreads();
      const double *qa = sQ + (wm * 32 + g) * ld + sl * kKS + tq;
      const double *kb = sK + buf * (kCT * kLdK) + (wn * 32 + g) * kLdK + tq;
#pragma unroll 2
      for (int k = 0; k < kKS; k += 4) {
        double af[4], bf[4];
#pragma unroll
        for (int mi = 0; mi < 4; ++mi) af[mi] = qa[mi * 8 * ld + k];
#pragma unroll
        for (int ni = 0; ni < 4; ++ni) bf[ni] = kb[ni * 8 * kLdK + k];
#pragma unroll
        for (int mi = 0; mi < 4; ++mi)
#pragma unroll
          for (int ni = 0; ni < 4; ++ni) dmma(acc[mi][ni], af[mi], bf[ni]);
      }
      __syncthreads();   // this buffer is refilled by the prefetch after next
      buf ^= 1;
    }

    // scaled log2 scores; columns past Nb do not exist
    float *slab = a.slab + (bh * a.Nb + r0) * a.ld_slab;
    double *tmax = a.tmax + (bh * a.Nb + r0) * a.ntiles;
#pragma unroll
    for (int mi = 0; mi < 4; ++mi) {
      double m = -INFINITY;
#pragma unroll
      for (int ni = 0; ni < 4; ++ni)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int col = c0 + wn * 32 + ni * 8 + 2 * tq + j;
          acc[mi][ni][j] = col < a.Nb ? acc[mi][ni][j] * a.c : -INFINITY;
          m = fmax(m, acc[mi][ni][j]);
        }
      m = fmax(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
      m = fmax(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
      if (tq == 0) sRed[wm * 32 + mi * 8 + g][wn] = m;
    }
    __syncthreads();
    if (tid < kRT) {
      const double m = fmax(fmax(sRed[tid][0], sRed[tid][1]), fmax(sRed[tid][2], sRed[tid][3]));
      sTileMax[tid] = m;
      if (r0 + tid < a.Nb) tmax[tid * a.ntiles + ct] = m;
    }
    __syncthreads();
#pragma unroll
    for (int mi = 0; mi < 4; ++mi) {
      const int row = wm * 32 + mi * 8 + g;
      const double m = sTileMax[row];
#pragma unroll
      for (int ni = 0; ni < 4; ++ni) {
        const int col = c0 + wn * 32 + ni * 8 + 2 * tq;
        if (col < a.Nb && r0 + row < a.Nb) {
          float2 e;
          e.x = exp2_split(acc[mi][ni][0] - m);
          e.y = exp2_split(acc[mi][ni][1] - m);
          *reinterpret_cast<float2 *>(slab + row * a.ld_slab + col) = e;
        }
      }
    }
    // sRed / sTileMax and sQ are reused by the next unit
    __syncthreads();
  }
}

// One warp per row of the mask: selection and kept bits.
// Static-ratio selection of one row (DynamicRad, "Dual-Mode Strategy",
// Static-Ratio mode; reading: the k most probable blocks, equal probabilities
// to the lower index, k >= Nb keeps the row).  The probabilities are positive
// fp32 values, so their bit patterns order like the values: a histogram of
// the exponent field finds the octave holding the k-th largest, a bisection
// over that octave's 2^23 patterns (on its members, compacted when there are
// at most kCand) finds the k-th largest pattern, and equal patterns at the cut
// are taken in index order.
template <bool kSmemRow>
__device__ void select_row_topk(const MaskArgs &a, int64_t grow, int r, const float *slab_row,
                                const double *tmax_row, float *erow, uint32_t *cand_key,
                                int32_t *cand_idx, float *tscale, int *hist, uint32_t *wbits) {
  const int lane = threadIdx.x & 31;
  const int Nb = a.Nb, k = a.k;
  double M = -INFINITY;
  for (int t = lane; t < a.ntiles; t += 32) M = fmax(M, tmax_row[t]);
  M = warp_max(M);
  for (int t = lane; t < a.ntiles; t += 32) tscale[t] = static_cast<float>(exp2(tmax_row[t] - M));
  for (int b = lane; b < kOctaves; b += 32) hist[b] = 0;
  __syncwarp();
  using Row = typename std::conditional<kSmemRow, SmemRow, RowView>::type;
  Row ebuf;
  if constexpr (kSmemRow) ebuf = SmemRow{erow}; else ebuf = RowView{slab_row, tscale};
  const bool keep_all = k >= Nb;
  for (int c = lane; c < Nb; c += 32) {
    const float e = slab_row[c] * tscale[c / kCT];
    if constexpr (kSmemRow) erow[c] = e;
    if (!keep_all) atomicAdd(&hist[__float_as_uint(e) >> 23], 1);
  }
  __syncwarp();

  bool bits_done = false;
  uint32_t vkey = 0;
  int need_ties = 0;
  if (!keep_all) {
    // lane l owns exponent bins 255-8l .. 248-8l: lane order = descending values
    int loc = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) loc += hist[kOctaves - 1 - 8 * lane - i];
    int incl = loc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += y;
    }
    int run = incl - loc, found = -1, above = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int b = kOctaves - 1 - 8 * lane - i;
      if (found < 0 && run + hist[b] >= k) {
        found = b;
        above = run;
      }
      run += hist[b];
    }
    // the highest such bin (the lowest lane that found one); every entry is
    // counted, so one exists as k < Nb
    const uint32_t fm = __ballot_sync(0xFFFFFFFFu, found >= 0);
    const int src = __ffs(fm) - 1;
    found = __shfl_sync(0xFFFFFFFFu, found, src);
    above = __shfl_sync(0xFFFFFFFFu, above, src);
    const bool compact = hist[found] <= kCand;
    // entries of higher octaves are kept whatever happens at the cut
    int pos = 0;
    for (int c0 = 0; c0 < Nb; c0 += 32) {
      const int c = c0 + lane;
      const int ex = c < Nb ? static_cast<int>(__float_as_uint(ebuf(c)) >> 23) : -1;
      const uint32_t hi_word = __ballot_sync(0xFFFFFFFFu, ex > found);
      if (lane == 0) wbits[c0 >> 5] = hi_word;
      if (compact) {
        const bool in = ex == found;
        const uint32_t m = __ballot_sync(0xFFFFFFFFu, in);
        if (in) {
          const int p = pos + __popc(m & ((1u << lane) - 1u));
          cand_key[p] = __float_as_uint(ebuf(c));
          cand_idx[p] = c;
        }
        pos += __popc(m);
      }
    }
    __syncwarp();
    // k-th largest pattern inside the octave: count(key >= hi) + above < k
    // <= count(key >= lo) + above
    uint32_t lo = static_cast<uint32_t>(found) << 23, hi = lo + (1u << 23);
    int cnt_hi = 0;
    while (hi - lo > 1) {
      const uint32_t mid = lo + ((hi - lo) >> 1);
      int cin = 0;
      if (compact) {
        for (int i = lane; i < pos; i += 32) cin += cand_key[i] >= mid && cand_key[i] < hi;
      } else {
        for (int c = lane; c < Nb; c += 32) {
          const uint32_t key = __float_as_uint(ebuf(c));
          cin += key >= mid && key < hi;
        }
      }
      cin = warp_sum_i(cin);
      if (above + cnt_hi + cin >= k) {
        lo = mid;
      } else {
        cnt_hi += cin;
        hi = mid;
      }
    }
    vkey = lo;
    need_ties = k - (above + cnt_hi);   // >= 1 entries equal to vkey
    if (compact) {
      // members in ascending index order: patterns above vkey, then the
      // first need_ties equal to it
      int ties_seen = 0;
      for (int i0 = 0; i0 < pos; i0 += 32) {
        const int i = i0 + lane;
        const uint32_t key = i < pos ? cand_key[i] : 0u;
        bool kept = i < pos && key > vkey;
        const bool tie = i < pos && key == vkey;
        const uint32_t tm = __ballot_sync(0xFFFFFFFFu, tie);
        if (tie && ties_seen + __popc(tm & ((1u << lane) - 1u)) < need_ties) kept = true;
        ties_seen += __popc(tm);
        if (kept) atomicOr(&wbits[cand_idx[i] >> 5], 1u << (cand_idx[i] & 31));
      }
      bits_done = true;
    }
  }
  if (!bits_done) {
    int ties_seen = 0;
    for (int w = 0; w < a.words; ++w) {
      const int c = w * 32 + lane;
      const bool valid = c < Nb;
      const uint32_t key = valid ? __float_as_uint(ebuf(c)) : 0u;
      bool kept;
      if (keep_all) {
        kept = valid;
      } else {
        kept = valid && key > vkey;
        const bool tie = valid && key == vkey;
        const uint32_t tm = __ballot_sync(0xFFFFFFFFu, tie);
        if (tie && ties_seen + __popc(tm & ((1u << lane) - 1u)) < need_ties) kept = true;
        ties_seen += __popc(tm);
      }
      const uint32_t word = __ballot_sync(0xFFFFFFFFu, kept);
      if (lane == 0) wbits[w] = word;
    }
  }
  __syncwarp();
  finish_row(a, grow, r, wbits);
}

// Per-warp SMEM of the top-p selection: candidates, tile factors, the bin
// histogram and the kept-bit row.
__host__ __device__ inline size_t select_warp_bytes(int ntiles, int row_floats) {
  return (static_cast<size_t>(kCand) * 8 + static_cast<size_t>(ntiles) * 8 + 16 + kBins * 8 +
          kMaxWords * 4 + static_cast<size_t>(row_floats) * 4 + 15) & ~static_cast<size_t>(15);
}

template <bool kSmemRow>
__global__ void __launch_bounds__(kThreads) mask_select_kernel(const MaskArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int warp = threadIdx.x >> 5;
  unsigned char *wbase = smem_raw + warp * select_warp_bytes(a.ntiles, kSmemRow ? a.Nb : 0);
  uint32_t *cand_key = reinterpret_cast<uint32_t *>(wbase);
  int32_t *cand_idx = reinterpret_cast<int32_t *>(cand_key + kCand);
  float *tscale = reinterpret_cast<float *>(
      (reinterpret_cast<uintptr_t>(cand_idx + kCand) + 15) & ~static_cast<uintptr_t>(15));
  int *hcnt = reinterpret_cast<int *>(tscale + a.ntiles);
  float *hmass = reinterpret_cast<float *>(hcnt + kBins);
  uint32_t *wbits = reinterpret_cast<uint32_t *>(hmass + kBins);
  float *erow = reinterpret_cast<float *>(wbits + kMaxWords);
  const int64_t rows = a.BH * a.Nb;
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * kWarps + warp; g < rows;
       g += static_cast<int64_t>(gridDim.x) * kWarps) {
    select_row<kSmemRow>(a, g, static_cast<int>(g % a.Nb), a.slab + g * a.ld_slab,
                         a.tmax + g * a.ntiles, erow, cand_key, cand_idx, tscale, hcnt, hmass,
                         wbits);
  }
}

// Per-warp SMEM of the static-ratio selection (all 4-byte fields).
__host__ __device__ inline size_t topk_warp_bytes(int ntiles, int row_floats) {
  return (static_cast<size_t>(2 * kCand + ntiles + kOctaves + kMaxWords + row_floats) * 4 + 15) &
         ~static_cast<size_t>(15);
}

template <bool kSmemRow>
__global__ void __launch_bounds__(kThreads) mask_select_topk_kernel(const MaskArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int warp = threadIdx.x >> 5;
  unsigned char *wbase = smem_raw + warp * topk_warp_bytes(a.ntiles, kSmemRow ? a.Nb : 0);
  uint32_t *cand_key = reinterpret_cast<uint32_t *>(wbase);
  int32_t *cand_idx = reinterpret_cast<int32_t *>(cand_key + kCand);
  float *tscale = reinterpret_cast<float *>(cand_idx + kCand);
  int *hist = reinterpret_cast<int *>(tscale + a.ntiles);
  uint32_t *wbits = reinterpret_cast<uint32_t *>(hist + kOctaves);
  float *erow = reinterpret_cast<float *>(wbits + kMaxWords);
  const int64_t rows = a.BH * a.Nb;
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * kWarps + warp; g < rows;
       g += static_cast<int64_t>(gridDim.x) * kWarps) {
    select_row_topk<kSmemRow>(a, g, static_cast<int>(g % a.Nb), a.slab + g * a.ld_slab,
                              a.tmax + g * a.ntiles, erow, cand_key, cand_idx, tscale, hist,
                              wbits);
  }
}

// Exclusive scan of n counts into row_ptr[0..n] by one CTA of 1024 threads.
// Exclusive scan of the kept counts into row_ptr in two launches: per-chunk
// sums of kScanChunk rows, then every chunk adds up the sums before it (at
// most a few hundred) and scans its own rows.  Coalesced, no serial walk.
constexpr int kScanChunk = 1024;

__global__ void __launch_bounds__(kScanChunk) chunk_sums_kernel(const int32_t *__restrict__ counts,
                                                                int64_t n,
                                                                int64_t *__restrict__ sums) {
  __shared__ int64_t warp_tot[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * kScanChunk + threadIdx.x;
  int64_t v = i < n ? counts[i] : 0;
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  if (lane == 0) warp_tot[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int64_t w = warp_tot[lane];
#pragma unroll
    for (int o = 16; o; o >>= 1) w += __shfl_xor_sync(0xFFFFFFFFu, w, o);
    if (lane == 0) sums[blockIdx.x] = w;
  }
}

__global__ void __launch_bounds__(kScanChunk) chunk_scan_kernel(const int32_t *__restrict__ counts,
                                                                int64_t n,
                                                                const int64_t *__restrict__ sums,
                                                                int64_t *__restrict__ row_ptr) {
  __shared__ int64_t warp_tot[32];
  __shared__ int64_t base;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (warp == 0) {                 // sum of the chunks before this one
    int64_t b = 0;
    for (int c = lane; c < static_cast<int>(blockIdx.x); c += 32) b += sums[c];
#pragma unroll
    for (int o = 16; o; o >>= 1) b += __shfl_xor_sync(0xFFFFFFFFu, b, o);
    if (lane == 0) base = b;
  }
  const int64_t i = static_cast<int64_t>(blockIdx.x) * kScanChunk + threadIdx.x;
  const int64_t v = i < n ? counts[i] : 0;
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
  const int64_t incl = base + x + (warp ? warp_tot[warp - 1] : 0);
  if (i < n) row_ptr[i] = incl - v;
  if (i == n - 1) row_ptr[n] = incl;
}

// Kept bits -> ascending column lists.  A warp per row, a lane per 32-bit
// word: the words' popcounts, a warp scan for their offsets, then each lane
// writes its own word's set bits in order.
__global__ void __launch_bounds__(256) expand_bits_kernel(const uint32_t *__restrict__ bits,
                                                          int words, int64_t rows,
                                                          const int64_t *__restrict__ row_ptr,
                                                          int32_t *__restrict__ col_idx) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; r < rows;
       r += warps) {
    int64_t pos = row_ptr[r];
    const uint32_t *rb = bits + r * words;
    for (int w0 = 0; w0 < words; w0 += 32) {
      const int w = w0 + lane;
      uint32_t word = w < words ? rb[w] : 0u;
      const int n = __popc(word);
      int incl = n;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
      }
      int32_t *dst = col_idx + pos + (incl - n);
      while (word) {
        const int b = __ffs(word) - 1;
        *dst++ = w * 32 + b;
        word &= word - 1u;
      }
      pos += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
  }
}

struct MaskLayout {
  int ld_slab, ntiles, words, grid;
  size_t slab_off, tmax_off, bits_off, counts_off, total;
  size_t smem, smem_a, smem_b, smem_k;
};

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

MaskLayout mask_layout(const Geometry &g, int grid) {
  MaskLayout L;
  L.ld_slab = static_cast<int>((g.Nb + 3) & ~3LL);
  L.ntiles = static_cast<int>((g.Nb + kCT - 1) / kCT);
  L.words = static_cast<int>((g.Nb + 31) / 32);
  L.grid = grid;
  size_t off = 0;
  L.slab_off = off;
  off = align256(off + static_cast<size_t>(g.BH * g.Nb) * L.ld_slab * 4);
  L.tmax_off = off;
  off = align256(off + static_cast<size_t>(g.BH * g.Nb) * L.ntiles * 8);
  L.bits_off = off;
  off = align256(off + static_cast<size_t>(g.BH * g.Nb) * L.words * 4);
  L.counts_off = off;
  off = align256(off + static_cast<size_t>(g.BH * g.Nb) * 4);
  L.total = off;
  L.smem_a = (static_cast<size_t>(kRT) * (g.d + kPad) + 2 * static_cast<size_t>(kCT) * kLdK) * 8;
  const int row_floats = g.Nb <= kSmemRowMaxNb ? static_cast<int>(g.Nb) : 0;
  L.smem_b = static_cast<size_t>(kWarps) * select_warp_bytes(L.ntiles, row_floats);
  L.smem_k = static_cast<size_t>(kWarps) * topk_warp_bytes(L.ntiles, row_floats);
  L.smem = L.smem_a > L.smem_b ? L.smem_a : L.smem_b;
  if (L.smem_k > L.smem) L.smem = L.smem_k;
  if (L.words > kMaxWords) L.smem = ~static_cast<size_t>(0) >> 1;  // reported as unsupported
  return L;
}

}  // namespace

size_t block_mask_workspace_bytes(const Geometry &g) { return mask_layout(g, kMaxGrid).total; }

size_t block_mask_smem_bytes(const Geometry &g) { return mask_layout(g, kMaxGrid).smem; }

cudaError_t launch_block_mask(const double *qp, const double *kp, const Geometry &g,
                              const vsa_mask_params &p, int topk, int64_t *row_ptr,
                              int32_t *col_idx, int32_t *kept_count, void *ws, unsigned *err,
                              cudaStream_t st) {
  (void)err;
  const int64_t rows = g.BH * g.Nb;
  if (rows == 0) {
    return cudaMemsetAsync(row_ptr, 0, sizeof(int64_t), st);
  }
  const int64_t tiles_per_head = (g.Nb + kRT - 1) / kRT;
  const int64_t items = g.BH * tiles_per_head;
  const int64_t units = items * ((g.Nb + kCT - 1) / kCT);
  int grid = num_sms();
  if (grid > kMaxGrid) grid = kMaxGrid;
  if (units < grid) grid = static_cast<int>(units);
  MaskLayout L = mask_layout(g, grid);
  unsigned char *w = static_cast<unsigned char *>(ws);
  MaskArgs a;
  a.qp = qp; a.kp = kp; a.BH = g.BH; a.Nb = static_cast<int>(g.Nb); a.d = g.d;
  a.Hb = g.Hb; a.Wb = g.Wb; a.thr = p.thr; a.use_sta = p.use_sta != 0;
  a.rt = p.sta_t; a.rh = p.sta_h; a.rw = p.sta_w;
  a.c = 1.4426950408889634 / std::sqrt(static_cast<double>(g.d));
  a.slab = reinterpret_cast<float *>(w + L.slab_off);
  a.tmax = reinterpret_cast<double *>(w + L.tmax_off);
  a.ld_slab = L.ld_slab; a.ntiles = L.ntiles;
  a.bits = reinterpret_cast<uint32_t *>(w + L.bits_off);
  a.words = L.words;
  a.counts = kept_count ? kept_count : reinterpret_cast<int32_t *>(w + L.counts_off);
  a.items = items; a.tiles_per_head = tiles_per_head;
  a.k = topk;
  cudaError_t e = cudaFuncSetAttribute(mask_scores_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(L.smem_a));
  if (e != cudaSuccess) return e;
  mask_scores_kernel<<<grid, kThreads, L.smem_a, st>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int64_t sel_blocks = (rows + kWarps - 1) / kWarps;
  const int sel_grid = static_cast<int>(sel_blocks < 64LL * num_sms() ? sel_blocks : 64LL * num_sms());
  const bool smem_row = g.Nb <= kSmemRowMaxNb;
  const void *sel = topk > 0 ? (smem_row ? reinterpret_cast<const void *>(mask_select_topk_kernel<true>)
                                         : reinterpret_cast<const void *>(mask_select_topk_kernel<false>))
                             : (smem_row ? reinterpret_cast<const void *>(mask_select_kernel<true>)
                                         : reinterpret_cast<const void *>(mask_select_kernel<false>));
  const size_t sel_smem = topk > 0 ? L.smem_k : L.smem_b;
  if ((e = cudaFuncSetAttribute(sel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(sel_smem))) != cudaSuccess)
    return e;
  if (topk > 0) {
    if (smem_row) mask_select_topk_kernel<true><<<sel_grid, kThreads, sel_smem, st>>>(a);
    else mask_select_topk_kernel<false><<<sel_grid, kThreads, sel_smem, st>>>(a);
  } else {
    if (smem_row) mask_select_kernel<true><<<sel_grid, kThreads, sel_smem, st>>>(a);
    else mask_select_kernel<false><<<sel_grid, kThreads, sel_smem, st>>>(a);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  {
    // chunk sums go to the start of the slab: the selection is done with it
    int64_t *sums = reinterpret_cast<int64_t *>(a.slab);
    const int chunks = static_cast<int>((rows + kScanChunk - 1) / kScanChunk);
    chunk_sums_kernel<<<chunks, kScanChunk, 0, st>>>(a.counts, rows, sums);
    chunk_scan_kernel<<<chunks, kScanChunk, 0, st>>>(a.counts, rows, sums, row_ptr);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int64_t want = (rows + 7) / 8;
  const int eg = static_cast<int>(want < 16LL * num_sms() ? want : 16LL * num_sms());
  expand_bits_kernel<<<eg, 256, 0, st>>>(a.bits, a.words, rows, row_ptr, col_idx);
  return cudaGetLastError();
}

}  // namespace vsa
