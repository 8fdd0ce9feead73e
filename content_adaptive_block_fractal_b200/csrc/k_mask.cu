// k_mask.cu -- content-adaptive block mask (NABLA, Methodology item 2:
// reduced attention over pooled blocks and the per-row CDF threshold; item 3:
// union with the sliding-tile window; Sparse VideoGen2 section 2B: top-p;
// DynamicRad section 2, Static-Ratio mode: a fixed number of blocks per row).
//
// Exact scores from integer tensor-core products.  Every pooled row x (fp64,
// d values) is written as y = x * 2^(6-e), max|x| < 2^e, and split into four
// signed base-2^7 digits:
//     y = D0 + D1 b + D2 b^2 + D3 b^3 + rho b^3,   b = 2^-7, |Dj| <= 64, |rho| <= 1/2
// (each step exact in fp64).  The score q.k = 2^(eq+ek-12) sum_i y_i y'_i is
// then, up to the dropped products of weight b^4 and below, the fixed-point
// value  A0 + b A1 + b^2 A2 + b^3 A3,  A_k = sum_{j+l=k} Dq_j . Dk_l, whose ten
// int8 dot products are exact int32 tcgen05.mma (kind::i8) results.  Per term
// the dropped part is at most 4096 (3 b^4 + 2 b^5 + b^6) + 64.001 b^3 < 7.7e-5,
// so |score error| <= d * 7.7e-5 * 2^(eq+ek-12): a bound that holds for every
// input, not an estimate.  With the fp32 combination of the A_k and the
// scaling, each log2-score t carries a known error bound eps (per row).
//
// Kernels, in launch order:
//   mask_digits_kernel   fp64 Qp, Kp -> int8 digit planes [4][rows][128] and
//                        per-row exponents (a warp per row).
//   mask_scores_kernel   persistent, warp-specialised; a work unit is 128
//                        query blocks of one head.  TMA loads the Q digit tile
//                        once and the K digit chunks (64 key blocks) into a
//                        4-deep ring; one thread issues the 40 int8 MMAs of a
//                        chunk into one of two TMEM accumulator sets; sixteen
//                        epilogue warps (thread = query row, 16 columns each)
//                        combine the four class accumulators into the fp32
//                        log2-score t = s log2(e) and store it to a row-major
//                        score slab, with the row's max, min and eps.
//   mask_select_kernel   a warp per row (rows in reverse, so the most recently
//                        written part of the slab is still in L2): 2^(t - R)
//                        in SMEM and their exact fp64 sum; 1/8-octave bins of
//                        those values, window by window (8 octaves each), find
//                        the bin holding the cut; one exact pass marks the
//                        blocks above it and collects the bin's blocks, which
//                        are sorted (t desc, index asc) and cut.  A row whose
//                        decision is not certain under eps (a near tie at the
//                        cut, a cut mass within the error of 1 - thr, an
//                        overfull cut bin) is listed for the recheck instead.
//                        Then the STA union, the kept-bit row and its count.
//   mask_recheck_kernel  a CTA per listed row: the oracle's computation in
//                        fp64 (scores, softmax, sort by probability then
//                        index, prefix mass), kept bits, STA union, count.
//   chunk_sums_kernel, chunk_scan_kernel, expand_bits_kernel
//                        counts -> row_ptr (int64) -> ascending col_idx.
#include "vsa_device.cuh"
#include "vsa_internal.h"
#include "vsa_tma.h"

#include <climits>
#include <cmath>

namespace vsa {
namespace {

constexpr int kDigits = 4;        // digit planes per pooled tensor
constexpr int kRowBytes = 128;    // one digit row: d int8 values, zero-padded to 128
constexpr int kTileRows = 128;    // query blocks per work unit (MMA M)
constexpr int kChunk = 64;        // key blocks per MMA chunk (MMA N)
constexpr int kStages = 4;        // K chunk ring
constexpr int kEpiWarps = 16;     // four per TMEM lane quarter, 16 columns each
constexpr int kThreadsA = (2 + kEpiWarps) * 32;
constexpr int kEpiBarrier = 1;    // named barrier of the epilogue warps
constexpr int kSelWarps = 8;      // rows in flight per select CTA
constexpr int kWin = 64;          // 1/8-octave bins per window (8 octaves)
constexpr int kCand = 64;         // cut-bin blocks sorted per row
constexpr int kMaxNb = 8192;      // blocks per head (kept-bit rows and per-warp rows in SMEM)

struct RowRec {
  float tmax, tmin;   // extremes of the row's log2-scores
  float eps;          // error bound of every t of the row (log2 units)
  int pad;
};

struct MaskArgs {
  int64_t BH, rows;
  int Nb, d, Hb, Wb, T;
  float thr;        // top-p threshold (topk == 0)
  int topk;         // static ratio: blocks per row (0: top-p)
  int use_sta, rt, rh, rw;
  float c_log2;     // log2(e) / sqrt(d)
  double scale;     // 1 / sqrt(d), the recheck's fp64 scale
  const double *qp, *kp;
  const int *qexp, *kexp;
  const float *kscale;      // [BH][ldk]: 2^(K row exponent), exact
  int ldk;
  float *slab;              // [rows][ld] log2-scores
  int ld;
  RowRec *rec;              // [rows]
  uint32_t *bits;           // [rows][words]
  int words;
  int32_t *counts;          // [rows]
  int32_t *flagged;         // rows listed for the recheck
  int *nflag;
  int tiles_per_head, nch, np2;
  int64_t units;
  unsigned *err;
};

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

__device__ __forceinline__ void epi_sync() {
  asm volatile("bar.sync %0, %1;" ::"n"(kEpiBarrier), "n"(kEpiWarps * 32) : "memory");
}

// exact int32 -> fp32 for |a| < 2^22
__device__ __forceinline__ float i2f_small(int32_t a) {
  return __int_as_float(a + 0x4B400000) - 12582912.0f;
}

// D[tmem] (+)= A[smem] . B[smem] with s8 operands, s32 accumulate.
__device__ __forceinline__ void mma_i8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(static_cast<uint32_t>(accumulate))
      : "memory");
}

// Instruction descriptor for kind::i8: s32 accumulator, s8 A and B, K-major.
__host__ __device__ constexpr uint32_t idesc_i8(int M, int N) {
  return (2u << 4)                                   // D format: s32
         | (1u << 7)                                 // A: s8
         | (1u << 10)                                // B: s8
         | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

#define VSA_R16(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), \
                   "=r"(r[i + 4]), "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7]), \
                   "=r"(r[i + 8]), "=r"(r[i + 9]), "=r"(r[i + 10]), "=r"(r[i + 11]), \
                   "=r"(r[i + 12]), "=r"(r[i + 13]), "=r"(r[i + 14]), "=r"(r[i + 15])
// 16 columns at each of two TMEM addresses, one wait for both.
__device__ __forceinline__ void tmem_ld2x16(uint32_t a0, uint32_t a1, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%32];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%33];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : VSA_R16(0), VSA_R16(16)
      : "r"(a0), "r"(a1)
      : "memory");
}
#undef VSA_R16

// ---------------------------------------------------------------- digits
// A warp per pooled row (Q rows first, then K rows); lane l converts values
// 4l .. 4l+3 and writes byte 4l.. of each digit row (zeros past d).
__global__ void __launch_bounds__(256)
    mask_digits_kernel(const double *__restrict__ qp, const double *__restrict__ kp,
                       int64_t rows, int64_t plane_rows, int d, int Nb, int ldk,
                       int8_t *__restrict__ qdig, int8_t *__restrict__ kdig,
                       int *__restrict__ qexp, int *__restrict__ kexp,
                       float *__restrict__ kscale, int *nflag) {
  const int lane = threadIdx.x & 31;
  const int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (w == 0 && lane == 0) *nflag = 0;
  if (w >= 2 * rows) return;
  const bool isk = w >= rows;
  const int64_t row = isk ? w - rows : w;
  const double *src = (isk ? kp : qp) + row * d;
  double x[4] = {0.0, 0.0, 0.0, 0.0};
  if (4 * lane < d) {
    const double2 u = *reinterpret_cast<const double2 *>(src + 4 * lane);
    const double2 v = *reinterpret_cast<const double2 *>(src + 4 * lane + 2);
    x[0] = u.x; x[1] = u.y; x[2] = v.x; x[3] = v.y;
  }
  double m = fmax(fmax(fabs(x[0]), fabs(x[1])), fmax(fabs(x[2]), fabs(x[3])));
  m = warp_max(m);
  int e = 0;
  if (m > 0.0) frexp(m, &e);           // m < 2^e
  uint32_t packed[kDigits] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    double y = ldexp(x[i], 6 - e);       // |y| < 64, exact
#pragma unroll
    for (int j = 0; j < kDigits; ++j) {
      const double dj = rint(y);         // |dj| <= 64
      packed[j] |= (static_cast<uint32_t>(static_cast<int>(dj)) & 0xFFu) << (8 * i);
      y = (y - dj) * 128.0;              // exact: |y - dj| <= 1/2
    }
  }
  int8_t *dig = isk ? kdig : qdig;
#pragma unroll
  for (int j = 0; j < kDigits; ++j)
    reinterpret_cast<uint32_t *>(dig + (static_cast<int64_t>(j) * plane_rows + row) * kRowBytes)[lane] =
        packed[j];
  if (lane == 0) {
    if (isk) {
      kexp[row] = e;
      // per head, padded to ldk entries so a chunk's scales are aligned
      kscale[(row / Nb) * ldk + row % Nb] = (e > -127 && e < 128) ? __int_as_float((e + 127) << 23) : 0.0f;
    } else {
      qexp[row] = e;
    }
  }
}

// ---------------------------------------------------------------- scores
struct SmemA {
  static constexpr int kQBytes = kDigits * kTileRows * kRowBytes;   // 64 KiB
  static constexpr int kKStage = kDigits * kChunk * kRowBytes;       // 32 KiB
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kQBytes;
  static constexpr int kX = kK + kStages * kKStage;   // per-slice max / min [2][4][128]
  static constexpr int kXBytes = 2 * 4 * kTileRows * 4 + 64;
  static constexpr int kBar = (kX + kXBytes + 7) & ~7;
  // q_full q_empty k_full[4] k_empty[4] acc_full[2] acc_empty[2]
  static constexpr int kNumBars = 2 + 2 * kStages + 4;
  static constexpr int kTmemSlot = kBar + kNumBars * 8;
  static constexpr int kAlloc = kTmemSlot + 16;
  static_assert(kAlloc <= 232448, "mask score kernel shared memory exceeds 227 KiB");
};

// 18 warps: at most five share a scheduler's 16K registers, so 96 each
__global__ void __maxnreg__(96)
    mask_scores_kernel(const __grid_constant__ CUtensorMap tq,
                       const __grid_constant__ CUtensorMap tk, const MaskArgs a) {
  using L = SmemA;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicOr(a.err, kErrSmemAlign);
    return;
  }
  unsigned char *smem = smem_raw;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar = sbase + L::kBar;
  const uint32_t q_full = bar, q_empty = bar + 8;
  auto k_full = [&](int s) { return bar + 16u + 8u * s; };
  auto k_empty = [&](int s) { return bar + 16u + 8u * (kStages + s); };
  auto acc_full = [&](int s) { return bar + 16u + 8u * (2 * kStages + s); };
  auto acc_empty = [&](int s) { return bar + 16u + 8u * (2 * kStages + 2 + s); };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kTmemSlot);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(acc_full(s), 1);
      mbar_init(acc_empty(s), kEpiWarps * 32);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tk);
      int n = 0, uu = 0;
      bool ok = true;
      for (int64_t u = blockIdx.x; ok && u < a.units; u += gridDim.x, ++uu) {
        const int64_t bh = u / a.tiles_per_head;
        const int tile = static_cast<int>(u % a.tiles_per_head);
        if (uu > 0 && !mbar_wait(q_empty, (uu - 1) & 1, a.err, kErrWaitMma)) break;
        mbar_arrive_expect_tx(q_full, L::kQBytes);
        tma_load_3d(sbase + L::kQ, &tq, q_full, 0,
                    static_cast<int>(bh * a.Nb + tile * kTileRows), 0);
        for (int j = 0; j < a.nch; ++j, ++n) {
          const int s = n % kStages;
          if (n >= kStages &&
              !mbar_wait(k_empty(s), ((n - kStages) / kStages) & 1, a.err, kErrWaitMma)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(k_full(s), L::kKStage);
          tma_load_3d(sbase + L::kK + s * L::kKStage, &tk, k_full(s), 0,
                      static_cast<int>(bh * a.Nb + j * kChunk), 0);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t kIdesc = idesc_i8(kTileRows, kChunk);
    // K-major, 128-byte swizzle: 8-row groups 1 KiB apart, K slices of 32
    // bytes (2 units of 16 B) inside the 128-byte row
    const uint64_t q_desc = smem_desc(sbase + L::kQ, 16, 1024);
    const uint64_t k_desc = smem_desc(sbase + L::kK, 16, 1024);
    constexpr uint32_t kQPlane = (kTileRows * kRowBytes) >> 4;
    constexpr uint32_t kKPlane = (kChunk * kRowBytes) >> 4;
    constexpr uint32_t kKStageU = L::kKStage >> 4;
    const int ksteps = a.d / 32;
    int n = 0, uu = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; ok && u < a.units; u += gridDim.x, ++uu) {
      if (!mbar_wait(q_full, uu & 1, a.err, kErrWaitTma)) break;
      for (int j = 0; j < a.nch; ++j, ++n) {
        const int s = n % kStages, b = n & 1;
        if (!mbar_wait(k_full(s), (n / kStages) & 1, a.err, kErrWaitTma) ||
            (n >= 2 && !mbar_wait(acc_empty(b), ((n - 2) >> 1) & 1, a.err, kErrWaitSoftmax))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t acc = tmem + static_cast<uint32_t>(b) * 256u;
          const uint64_t kd = k_desc + static_cast<uint32_t>(s) * kKStageU;
#pragma unroll
          for (int cls = 0; cls < kDigits; ++cls) {
            bool first = true;
#pragma unroll
            for (int j2 = 0; j2 <= cls; ++j2) {
              const int l = cls - j2;
              for (int ks = 0; ks < ksteps; ++ks) {
                mma_i8_ss(acc + cls * kChunk, q_desc + j2 * kQPlane + ks * 2,
                          kd + l * kKPlane + ks * 2, kIdesc, !first);
                first = false;
              }
            }
          }
          mma_commit(k_empty(s));
          mma_commit(acc_full(b));
          if (j == a.nch - 1) mma_commit(q_empty);
        }
        __syncwarp();
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int e = warp - 2;
    const int slice = e >> 2;                  // 16-column slice of each chunk
    const int quarter = warp & 3;              // TMEM lane quarter
    const int row = quarter * 32 + lane;       // query row within the tile
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    float *x_mx = reinterpret_cast<float *>(smem + L::kX);   // [4][128]
    float *x_mn = x_mx + 4 * kTileRows;                        // [4][128]
    int *x_head = reinterpret_cast<int *>(x_mn + 4 * kTileRows);
    const int tid = e * 32 + lane;
    int n = 0;
    // A wait that gives up clears ok; the warps then run the rest of their
    // loops without waiting or writing, so every epilogue warp still reaches
    // each named barrier and the CTA winds down.
    bool ok = true;
    for (int64_t u = blockIdx.x; u < a.units; u += gridDim.x) {
      const int64_t bh = u / a.tiles_per_head;
      const int tile = static_cast<int>(u % a.tiles_per_head);
      const int r_local = tile * kTileRows + row;
      const bool valid = r_local < a.Nb;
      const int64_t g = bh * a.Nb + r_local;
      // the head's largest K exponent (for the error bound)
      {
        int emax = INT_MIN;
        for (int c = tid; c < a.Nb; c += kEpiWarps * 32) emax = max(emax, a.kexp[bh * a.Nb + c]);
#pragma unroll
        for (int o = 16; o; o >>= 1) emax = max(emax, __shfl_xor_sync(0xFFFFFFFFu, emax, o));
        if (tid == 0) x_head[0] = INT_MIN;
        epi_sync();
        if (lane == 0) atomicMax(&x_head[0], emax);
        epi_sync();
      }
      const int ke_max = x_head[0];
      const int qe = valid ? a.qexp[g] : 0;
      const float rowf = ldexpf(a.c_log2, qe - 12);
      const float *ks_head = a.kscale + bh * a.ldk;
      float *srow = a.slab + g * a.ld;
      float tmx = -INFINITY, tmn = INFINITY;
      // the K scales of this thread's 16 columns, loaded one chunk ahead so
      // the load is off the path from the accumulators to the stores
      float4 ksn[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        ksn[q] = __ldg(reinterpret_cast<const float4 *>(ks_head + slice * 16) + q);
      for (int j = 0; j < a.nch; ++j, ++n) {
        const int b = n & 1;
        if (ok && !mbar_wait(acc_full(b), (n >> 1) & 1, a.err, kErrWaitMma)) ok = false;
        tc_fence_after();
        // classes 3 and 2 first, then 1 and 0 (half the registers live)
        const uint32_t base = lane_addr + static_cast<uint32_t>(b) * 256u + slice * 16;
        uint32_t A[32];
        float u[16];
        tmem_ld2x16(base + 2 * kChunk, base + 3 * kChunk, A);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          u[i] = fmaf(i2f_small(static_cast<int32_t>(A[16 + i])), 0.0078125f,
                      i2f_small(static_cast<int32_t>(A[i])));
        tmem_ld2x16(base, base + kChunk, A);
        tc_fence_before();
        mbar_arrive(acc_empty(b));
        const int c0 = j * kChunk + slice * 16;
        if (!ok || !valid || c0 >= a.Nb) continue;
        float t[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float sfix = fmaf(fmaf(u[i], 0.0078125f, i2f_small(static_cast<int32_t>(A[16 + i]))),
                                  0.0078125f, i2f_small(static_cast<int32_t>(A[i])));
          const float4 kq = ksn[i >> 2];
          const float ksi = (i & 3) == 0 ? kq.x : (i & 3) == 1 ? kq.y : (i & 3) == 2 ? kq.z : kq.w;
          t[i] = sfix * ksi * rowf;
        }
        if (j + 1 < a.nch) {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            ksn[q] = __ldg(reinterpret_cast<const float4 *>(ks_head + (j + 1) * kChunk + slice * 16) + q);
        }
        if (c0 + 16 <= a.Nb) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            tmx = fmaxf(tmx, t[i]);
            tmn = fminf(tmn, t[i]);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            if (c0 + i < a.Nb) {
              tmx = fmaxf(tmx, t[i]);
              tmn = fminf(tmn, t[i]);
            }
          }
        }
        // the row is padded to a multiple of 16 entries; padding is never read
        float4 *dst = reinterpret_cast<float4 *>(srow + c0);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          dst[q] = make_float4(t[4 * q], t[4 * q + 1], t[4 * q + 2], t[4 * q + 3]);
      }
      x_mx[slice * kTileRows + row] = tmx;
      x_mn[slice * kTileRows + row] = tmn;
      epi_sync();
      if (ok && slice == 0 && valid) {
        float mx = x_mx[row], mn = x_mn[row];
#pragma unroll
        for (int s = 1; s < 4; ++s) {
          mx = fmaxf(mx, x_mx[s * kTileRows + row]);
          mn = fminf(mn, x_mn[s * kTileRows + row]);
        }
        const double tabs = fmax(fabs(static_cast<double>(mx)), fabs(static_cast<double>(mn)));
        // error of a value 2^(t - R) in log2 units: d (7.7e-5 digit
        // truncation + 5.9e-6 fp32 combination of the classes) in y units,
        // times 2^(eq+ek-12) log2(e)/sqrt(d); the two fp32 roundings of t
        // (2^-23 |t|), the rounding of t - R (2^-24 (|t| + |R|), |R| <= |t| + 1),
        // the hardware exp2 (relative 2^-22, 3.4e-7 in log2 units) and the
        // fp32 partial sums of four values in the row total (3 * 2^-24)
        const double kr = ldexp(static_cast<double>(a.c_log2), qe + ke_max - 12);
        const double eps = a.d * 8.3e-5 * kr + ldexp(tabs + 1.0, -22) + 7e-7;
        const bool range_ok = qe > -100 && qe < 100 && ke_max < 100 && tabs < 1.0e5;
        RowRec r;
        r.tmax = mx;
        r.tmin = mn;
        r.eps = range_ok ? static_cast<float>(eps) : INFINITY;
        r.pad = 0;
        a.rec[g] = r;
      }
      // x_mx / x_mn are rewritten only after the next unit's two barriers
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- select
// Bins of a value p = 2^(t - R) in [0, 1) from its fp32 bit pattern.  The
// 1/8-octave bin: bin 0 holds [15/16, 1), larger bins smaller values, p = 0
// falls in the last bin (1015).  The fine key splits every bin into 64
// (key / 64 = bin).  Both are monotone: a larger p never has a larger key.
__device__ __forceinline__ int value_bin(float p) {
  const uint32_t k = __float_as_uint(p);
  const int ex = static_cast<int>(k >> 23);      // biased exponent, <= 126 for p < 1
  const int m3 = static_cast<int>((k >> 20) & 7u);
  return (126 - ex) * 8 + (7 - m3);
}
__device__ __forceinline__ int value_key(float p) {
  const uint32_t k = __float_as_uint(p);
  const int ex = static_cast<int>(k >> 23);
  const int m9 = static_cast<int>((k >> 14) & 511u);
  return (126 - ex) * 512 + (511 - m9);
}
// t - R implied by p = 2^(t - R), with the bound of its error: fp32 rounding
// of t - R and the hardware exp2 (relative 2^-21 at most)
__device__ __forceinline__ double log2_of(float p) { return log2(static_cast<double>(p)); }
__device__ __forceinline__ double log2_slack(double l) { return ldexp(fabs(l), -23) + 1e-6; }

// Per-warp SMEM of the selection: the row's 2^(t - R), the window histogram,
// the cut-bin candidates and the kept-bit row.
__host__ __device__ inline size_t select_warp_bytes(int ldp, int words) {
  return (static_cast<size_t>(ldp) * 4 + kWin * 4 + kCand * 8 + static_cast<size_t>(words) * 4 +
          15) & ~static_cast<size_t>(15);
}

// Cumulative scan of the 64 bins of `hist` (two per lane) from `above`: the
// first bin whose inclusive mass reaches `target`, or kWin - 1 (fp32 bin
// sums only place the cut; exact passes confirm it).
__device__ __forceinline__ int first_bin_reaching(const float *hist, double above, double target) {
  const int lane = threadIdx.x & 31;
  const double h0 = hist[2 * lane], h1 = hist[2 * lane + 1];
  double incl = h0 + h1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += y;
  }
  const double excl = incl - h0 - h1;
  int found = 1 << 30;
  if (above + excl + h0 >= target) found = 2 * lane;
  else if (above + incl >= target) found = 2 * lane + 1;
#pragma unroll
  for (int o = 16; o; o >>= 1) found = min(found, __shfl_xor_sync(0xFFFFFFFFu, found, o));
  return found < kWin ? found : kWin - 1;
}

// kCount: the static-ratio rule (the k largest), else top-p (mass 1 - thr).
template <bool kCount>
__global__ void __launch_bounds__(kSelWarps * 32) mask_select_kernel(const MaskArgs a, int ldp) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nw = blockDim.x >> 5;                 // rows in flight per CTA
  unsigned char *wb = smem_raw + warp * select_warp_bytes(ldp, a.words);
  float *ph = reinterpret_cast<float *>(wb);                   // [ldp]
  float *hist = ph + ldp;                                      // [kWin]
  int32_t *cand_c = reinterpret_cast<int32_t *>(hist + kWin);  // [kCand]
  float *cand_t = reinterpret_cast<float *>(cand_c + kCand);   // [kCand]
  uint32_t *bits = reinterpret_cast<uint32_t *>(cand_t + kCand);
  const int Nb = a.Nb;
  const bool keep_all_rule = kCount ? a.topk >= Nb : a.thr <= 0.0f;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * nw;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * nw + warp; i < a.rows; i += warps) {
    const int64_t g = a.rows - 1 - i;          // newest slab rows first
    const int r = static_cast<int>(g % Nb);
    const float *srow = a.slab + g * a.ld;
    bool recheck = false;
    if (keep_all_rule) {
      for (int w = lane; w < a.words; w += 32)
        bits[w] = (w + 1) * 32 <= Nb ? 0xFFFFFFFFu : ((1u << (Nb & 31)) - 1u);
    } else {
      const RowRec rc = a.rec[g];
      const double eps = rc.eps;
      if (!(eps < 1.0) || !(fabsf(rc.tmax) < 1.0e5f)) recheck = true;
      const int R = recheck ? 0 : static_cast<int>(floorf(rc.tmax)) + 1;   // every t < R
      const float Rf = static_cast<float>(R);
      // 1. the row's values 2^(t - R) in SMEM, their exact total and the
      // histogram of the top window (8 octaves)
      for (int b = lane; b < kWin; b += 32) hist[b] = 0.0f;
      __syncwarp();
      double z = 0.0, wmass = 0.0;
      if (!recheck) {
        // 16-byte loads, two in flight per lane (the row is padded to 16)
        for (int c0 = 4 * lane; c0 < Nb; c0 += 256) {
          float4 v[2];
#pragma unroll
          for (int u = 0; u < 2; ++u)
            if (c0 + 128 * u < Nb) v[u] = *reinterpret_cast<const float4 *>(srow + c0 + 128 * u);
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int cb = c0 + 128 * u;
            if (cb >= Nb) continue;
            const float x4[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
            float p4[4];
            float z4 = 0.0f, w4 = 0.0f;    // fp32 sums of four, fp64 across
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const bool in = cb + q < Nb;
              const float p = in ? ex2(x4[q] - Rf) : 0.0f;
              p4[q] = p;
              const float w = kCount ? (in ? 1.0f : 0.0f) : p;
              z4 += w;
              const int b = value_bin(p);
              if (in && b < kWin) {
                atomicAdd(&hist[b], w);
                w4 += w;
              }
            }
            z += static_cast<double>(z4);
            wmass += static_cast<double>(w4);
            // ph is padded to a multiple of 32 entries
            *reinterpret_cast<float4 *>(ph + cb) = make_float4(p4[0], p4[1], p4[2], p4[3]);
          }
        }
        z = warp_sum(z);
        wmass = warp_sum(wmass);
      }
      __syncwarp();
      const double target = kCount ? static_cast<double>(a.topk)
                                   : (1.0 - static_cast<double>(a.thr)) * z;
      // 2. windows of 64 bins, top down, until one holds the cut
      double above = 0.0;      // mass (count) of the windows above
      int bstar = -1;
      for (int wlo = 0; !recheck && bstar < 0 && wlo < 1024; wlo += kWin) {
        if (wlo > 0) {
          for (int b = lane; b < kWin; b += 32) hist[b] = 0.0f;
          __syncwarp();
          wmass = 0.0;
          for (int c = lane; c < Nb; c += 32) {
            const float p = ph[c];
            const int b = value_bin(p) - wlo;
            if (b >= 0 && b < kWin) {
              const float w = kCount ? 1.0f : p;
              atomicAdd(&hist[b], w);
              wmass += static_cast<double>(w);
            }
          }
          wmass = warp_sum(wmass);
          __syncwarp();
        }
        if (above + wmass >= target) bstar = wlo + first_bin_reaching(hist, above, target);
        else above += wmass;
        __syncwarp();
      }
      if (bstar < 0) recheck = true;     // the sums never reach the target
      // 3. exact passes over the fine keys: bits of the blocks above the cut
      // range [klo, khi), their exact mass, the nearest values on either
      // side and the range's blocks, with a histogram of the range's 64 fine
      // keys; a range with more blocks than the list holds is narrowed to
      // the fine key holding the cut and passed once more
      int ncand = 0;
      double above_x = 0.0;
      float pmin_above = INFINITY, pmax_below = 0.0f;
      int klo = bstar * 64, khi = klo + 64;
      auto exact_pass = [&]() {
        for (int b = lane; b < kWin; b += 32) hist[b] = 0.0f;
        __syncwarp();
        ncand = 0;
        above_x = 0.0;
        pmin_above = INFINITY;
        pmax_below = 0.0f;
        const bool fine = khi - klo == 64;
        // four consecutive columns per lane: lanes 8j .. 8j+7 cover kept-bit
        // word j of the 128-column chunk
        for (int c0 = 0; c0 < a.words * 32; c0 += 128) {
          const int cb = c0 + 4 * lane;
          float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
          if (cb < Nb) v = *reinterpret_cast<const float4 *>(ph + cb);   // cb + 3 < ldp
          const float p4[4] = {v.x, v.y, v.z, v.w};
          uint32_t nib = 0u, inm = 0u;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const bool valid = cb + q < Nb;
            const int k = valid ? value_key(p4[q]) : 1 << 30;
            if (k < klo) {
              above_x += kCount ? 1.0 : static_cast<double>(p4[q]);
              pmin_above = fminf(pmin_above, p4[q]);
              nib |= 1u << q;
            } else if (k >= khi && valid) {
              pmax_below = fmaxf(pmax_below, p4[q]);
            }
            const bool in = k >= klo && k < khi;
            inm |= (in ? 1u : 0u) << q;
            if (in && fine) atomicAdd(&hist[k - klo], kCount ? 1.0f : p4[q]);
          }
          uint32_t wv = nib << (4 * (lane & 7));
          wv |= __shfl_xor_sync(0xFFFFFFFFu, wv, 1);
          wv |= __shfl_xor_sync(0xFFFFFFFFu, wv, 2);
          wv |= __shfl_xor_sync(0xFFFFFFFFu, wv, 4);
          const int w = (c0 >> 5) + (lane >> 3);
          if ((lane & 7) == 0 && w < a.words) bits[w] = wv;
          // the range's blocks, in column order
          if (__any_sync(0xFFFFFFFFu, inm != 0u)) {
            const int ni = __popc(inm);
            int incl = ni;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
              const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
              if (lane >= o) incl += y;
            }
            int pos = ncand + incl - ni;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              if ((inm >> q) & 1u) {
                if (pos < kCand) {
                  cand_c[pos] = cb + q;
                  cand_t[pos] = srow[cb + q];
                }
                ++pos;
              }
            }
            ncand += __shfl_sync(0xFFFFFFFFu, incl, 31);
          }
        }
        above_x = warp_sum(above_x);
#pragma unroll
        for (int o = 16; o; o >>= 1) {
          pmin_above = fminf(pmin_above, __shfl_xor_sync(0xFFFFFFFFu, pmin_above, o));
          pmax_below = fmaxf(pmax_below, __shfl_xor_sync(0xFFFFFFFFu, pmax_below, o));
        }
        __syncwarp();
      };
      if (!recheck) {
        exact_pass();
        if (ncand > kCand && above_x < target) {
          klo += first_bin_reaching(hist, above_x, target);
          khi = klo + 1;
          exact_pass();
        }
        if (ncand == 0 || ncand > kCand || !(above_x < target)) recheck = true;
      }
      // 4. sort the cut bin (t desc, index asc) and cut it
      if (!recheck) {
        // sort key: t descending (fp32 patterns made to order like t, then
        // inverted), index ascending
        auto sort_key = [&](int v) -> uint64_t {
          uint32_t o = __float_as_uint(cand_t[v]);
          o = (o & 0x80000000u) ? ~o : (o | 0x80000000u);     // orders like t
          return (static_cast<uint64_t>(~o) << 32) | static_cast<uint32_t>(cand_c[v]);
        };
        uint64_t key[2];
        if (ncand <= 32) {
          // one key per lane: bitonic sort of 32, then position i to lane i/2
          uint64_t k1 = lane < ncand ? sort_key(lane) : ~0ull;
#pragma unroll
          for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
            for (int stride = size >> 1; stride > 0; stride >>= 1) {
              const uint64_t other = __shfl_xor_sync(0xFFFFFFFFu, k1, stride);
              const bool up = (lane & size) == 0;
              const bool lower = (lane & stride) == 0;
              const uint64_t lo = k1 < other ? k1 : other;
              const uint64_t hi = k1 < other ? other : k1;
              k1 = (lower == up) ? lo : hi;
            }
          }
          const uint64_t a0 = __shfl_sync(0xFFFFFFFFu, k1, (2 * lane) & 31);
          const uint64_t a1 = __shfl_sync(0xFFFFFFFFu, k1, (2 * lane + 1) & 31);
          key[0] = lane < 16 ? a0 : ~0ull;
          key[1] = lane < 16 ? a1 : ~0ull;
        } else {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int v = 2 * lane + h;
            key[h] = v < ncand ? sort_key(v) : ~0ull;
          }
          // bitonic sort of 64 keys, ascending, key h of lane l at position 2l + h
#pragma unroll
          for (int size = 2; size <= 64; size <<= 1) {
#pragma unroll
            for (int stride = size >> 1; stride > 0; stride >>= 1) {
              if (stride == 1) {
                const bool up = ((2 * lane) & size) == 0;
                const uint64_t lo = key[0] < key[1] ? key[0] : key[1];
                const uint64_t hi = key[0] < key[1] ? key[1] : key[0];
                key[0] = up ? lo : hi;
                key[1] = up ? hi : lo;
              } else {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                  const int pos = 2 * lane + h;
                  const uint64_t other = __shfl_xor_sync(0xFFFFFFFFu, key[h], stride >> 1);
                  const bool up = (pos & size) == 0;
                  const bool lower = (pos & stride) == 0;
                  const uint64_t lo = key[h] < other ? key[h] : other;
                  const uint64_t hi = key[h] < other ? other : key[h];
                  key[h] = (lower == up) ? lo : hi;
                }
              }
            }
          }
        }
        double pp[2];
        float tt[2];
        int cc[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const bool vld = key[h] != ~0ull;
          cc[h] = vld ? static_cast<int>(key[h] & 0xFFFFFFFFu) : -1;
          tt[h] = vld ? srow[cc[h]] : -INFINITY;
          pp[h] = vld ? (kCount ? 1.0 : static_cast<double>(ph[cc[h]])) : 0.0;
        }
        double incl = pp[0] + pp[1];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const double y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
          if (lane >= o) incl += y;
        }
        const double ex0 = incl - pp[0] - pp[1];
        // first position whose inclusive mass (count) reaches the target
        int first = 1 << 30;
        if (cc[0] >= 0 && above_x + ex0 + pp[0] >= target) first = 2 * lane;
        else if (cc[1] >= 0 && above_x + incl >= target) first = 2 * lane + 1;
#pragma unroll
        for (int o = 16; o; o >>= 1) first = min(first, __shfl_xor_sync(0xFFFFFFFFu, first, o));
        if (first >= ncand) {
          recheck = true;
        } else {
          const int keep_n = first + 1;
          const int la = first >> 1, ha = first & 1;
          const float ta = __shfl_sync(0xFFFFFFFFu, ha ? tt[1] : tt[0], la);
          const double pa = __shfl_sync(0xFFFFFFFFu, ha ? pp[1] : pp[0], la);
          const double mk = above_x + __shfl_sync(0xFFFFFFFFu, ha ? incl : ex0 + pp[0], la);
          // smallest kept and largest dropped log2-scores, bounded from the
          // values of the neighbouring bins where they are not in the list
          double ta_eff = ta, tb_eff = -INFINITY;
          if (pmin_above < INFINITY) {
            const double l = log2_of(pmin_above);
            ta_eff = fmin(ta_eff, R + l - log2_slack(l));
          }
          if (keep_n < ncand) {
            const int lb = keep_n >> 1, hb = keep_n & 1;
            tb_eff = __shfl_sync(0xFFFFFFFFu, hb ? tt[1] : tt[0], lb);
          }
          if (pmax_below > 0.0f) {
            const double l = log2_of(pmax_below);
            tb_eff = fmax(tb_eff, R + l + log2_slack(l));
          } else if (pmax_below == 0.0f && keep_n == ncand) {
            // dropped blocks whose value underflowed to 0 lie below 2^-126
            tb_eff = fmax(tb_eff, R - 126.0);
          }
          // the kept blocks are apart from the dropped ones by more than the
          // error of both; the kept mass reaches the target, and falls short
          // of it without its smallest member, under every admissible error
          if (!(ta_eff - tb_eff > 2.0 * eps)) recheck = true;
          if (!kCount) {
            const double grow2 = exp2(2.0 * eps);
            if (!(mk >= target * grow2) || !(mk * grow2 - pa < target)) recheck = true;
          }
          if (!recheck) {
#pragma unroll
            for (int h = 0; h < 2; ++h)
              if (2 * lane + h < keep_n) atomicOr(&bits[cc[h] >> 5], 1u << (cc[h] & 31));
          }
        }
      }
      __syncwarp();
    }
    if (recheck) {
      if (lane == 0) {
        const int pos = atomicAdd(a.nflag, 1);
        a.flagged[pos] = static_cast<int32_t>(g);
      }
      __syncwarp();
      continue;
    }
    if (a.use_sta && !keep_all_rule) {
      const int hw = a.Hb * a.Wb;
      const int tr = r / hw, yr = (r / a.Wb) % a.Hb, xr = r % a.Wb;
      const int nt = 2 * a.rt + 1, ny = 2 * a.rh + 1, nx = 2 * a.rw + 1;
      for (int v = lane; v < nt * ny * nx; v += 32) {
        const int t3 = tr - a.rt + v / (ny * nx);
        const int yy = yr - a.rh + (v / nx) % ny;
        const int xx = xr - a.rw + v % nx;
        if (t3 >= 0 && t3 < a.T && yy >= 0 && yy < a.Hb && xx >= 0 && xx < a.Wb) {
          const int c = (t3 * a.Hb + yy) * a.Wb + xx;
          atomicOr(&bits[c >> 5], 1u << (c & 31));
        }
      }
    }
    __syncwarp();
    int count = 0;
    for (int w = lane; w < a.words; w += 32) {
      const uint32_t x = bits[w];
      a.bits[g * a.words + w] = x;
      count += __popc(x);
    }
    count = warp_sum_i(count);
    if (lane == 0) a.counts[g] = count;
    __syncwarp();
  }
}

// ---------------------------------------------------------------- recheck
// The oracle's arithmetic for one listed row, a CTA per row: fp64 scores
// scaled by 1/sqrt(d), softmax against the row maximum, and the kept set of
// the sort on (probability desc, index asc) -- blocks taken while the mass
// before them is below 1 - thr (top-p), or the first k (static ratio).
// Scores: the head's K passes through a ring of three 32-key stages filled by
// bulk copies (32 consecutive key rows are contiguous), 16 threads per key
// reading consecutive doubles.  The cut: bisection over the probabilities'
// bit patterns (positive doubles order like their patterns) with fp64 mass
// (count) sums until at most 256 values remain between the bounds; those are
// sorted on (probability desc, index asc) and walked in order from the mass
// above them, as the oracle walks its sorted row.  Then the STA union, the
// kept-bit row and its count.
constexpr int kRcThreads = 256;
constexpr int kRcKeys = 32;       // keys per stage
constexpr int kRcStages = 3;
constexpr int kRcList = 256;      // values sorted at the end of the bisection

__host__ __device__ inline size_t recheck_smem_bytes(int ldp, int words, int d) {
  return static_cast<size_t>(kRcStages) * kRcKeys * d * 8 + static_cast<size_t>(ldp) * 8 +
         static_cast<size_t>(d) * 8 + static_cast<size_t>(kRcList) * 12 +
         ((static_cast<size_t>(words) * 4 + 15) & ~static_cast<size_t>(15)) + 64;
}

__global__ void __launch_bounds__(kRcThreads) mask_recheck_kernel(const MaskArgs a, int ldp) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int d = a.d, Nb = a.Nb;
  double *stage = reinterpret_cast<double *>(smem_raw);   // [3][32][d]
  double *pv = stage + kRcStages * kRcKeys * d;            // [ldp] scores, then probabilities
  double *q = pv + ldp;                                    // [d]
  double *lp = q + d;                                      // [256] listed values
  int *li = reinterpret_cast<int *>(lp + kRcList);         // [256] their indices
  uint32_t *bits = reinterpret_cast<uint32_t *>(li + kRcList);                 // [words]
  uint64_t *bar = reinterpret_cast<uint64_t *>(
      (reinterpret_cast<uintptr_t>(bits + a.words) + 15) & ~static_cast<uintptr_t>(15));  // [3]
  __shared__ double red[kRcThreads / 32], red2[kRcThreads / 32];
  __shared__ int nlist, ok_sh;
  const uint32_t stage_s = smem_u32(stage);
  auto bar_s = [&](int s) { return smem_u32(bar + s); };
  if (tid == 0) {
    for (int s = 0; s < kRcStages; ++s) mbar_init(bar_s(s), 1);
    fence_mbar_init();
    ok_sh = 1;
  }
  __syncthreads();
  const int nf = *a.nflag;
  const int ntiles = (Nb + kRcKeys - 1) / kRcKeys;
  const uint32_t stage_bytes = static_cast<uint32_t>(kRcKeys * d * 8);
  int n = 0;                     // stages consumed by this CTA so far (barrier phases)
  for (int64_t fi = blockIdx.x; fi < nf; fi += gridDim.x) {
    const int64_t g = a.flagged[fi];
    const int64_t bh = g / Nb;
    const int r = static_cast<int>(g % Nb);
    const double *kbase = a.kp + bh * Nb * d;
    for (int j = tid; j < d; j += kRcThreads) q[j] = a.qp[g * d + j];
    auto issue = [&](int t) {    // tile t into stage (n + t - done) % 3, by thread 0
      const int s = (n + t) % kRcStages;
      const int keys = Nb - t * kRcKeys < kRcKeys ? Nb - t * kRcKeys : kRcKeys;
      const uint32_t bytes = static_cast<uint32_t>(keys * d * 8);
      mbar_arrive_expect_tx(bar_s(s), bytes);
      bulk_load(stage_s + s * stage_bytes, kbase + static_cast<int64_t>(t) * kRcKeys * d, bytes,
                bar_s(s));
    };
    if (tid == 0)
      for (int t = 0; t < kRcStages && t < ntiles; ++t) issue(t);
    __syncthreads();
    const int key = tid >> 4, part = tid & 15;        // 16 threads per key
    for (int t = 0; t < ntiles; ++t) {
      const int s = (n + t) % kRcStages;
      if (!mbar_wait(bar_s(s), ((n + t) / kRcStages) & 1, a.err, kErrWaitTma)) ok_sh = 0;
      const double *ks = stage + s * kRcKeys * d;
#pragma unroll
      for (int h = 0; h < kRcKeys; h += 16) {
        const int kk = h + key;
        double acc = 0.0;
        for (int j = part; j < d; j += 16) acc = fma(q[j], ks[kk * d + j], acc);
#pragma unroll
        for (int o = 8; o; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
        const int c = t * kRcKeys + kk;
        if (part == 0 && c < Nb) pv[c] = acc * a.scale;
      }
      __syncthreads();            // stage s consumed by every thread
      if (tid == 0 && t + kRcStages < ntiles) issue(t + kRcStages);
    }
    n += ntiles;
    __syncthreads();
    // softmax against the row maximum (block reductions)
    double m = -INFINITY;
    for (int c = tid; c < Nb; c += kRcThreads) m = fmax(m, pv[c]);
    m = warp_max(m);
    if (lane == 0) red[warp] = m;
    __syncthreads();
    m = red[0];
    for (int w = 1; w < kRcThreads / 32; ++w) m = fmax(m, red[w]);
    __syncthreads();
    double z = 0.0;
    for (int c = tid; c < Nb; c += kRcThreads) {
      const double e = exp(pv[c] - m);
      pv[c] = e;
      z += e;
    }
    z = warp_sum(z);
    if (lane == 0) red[warp] = z;
    __syncthreads();
    z = 0.0;
    for (int w = 0; w < kRcThreads / 32; ++w) z += red[w];
    for (int c = tid; c < Nb; c += kRcThreads) pv[c] /= z;
    for (int w = tid; w < a.words; w += kRcThreads) bits[w] = 0u;
    __syncthreads();
    const bool count_rule = a.topk > 0;
    // mass (count) of the values with patterns in [lo, hi), and how many
    auto mass_in = [&](uint64_t lo, uint64_t hi, double &cnt) {
      double sum = 0.0, k = 0.0;
      for (int c = tid; c < Nb; c += kRcThreads) {
        const uint64_t kc = static_cast<uint64_t>(__double_as_longlong(pv[c]));
        if (kc >= lo && kc < hi) {
          sum += count_rule ? 1.0 : pv[c];
          k += 1.0;
        }
      }
      sum = warp_sum(sum);
      k = warp_sum(k);
      __syncthreads();
      if (lane == 0) {
        red[warp] = sum;
        red2[warp] = k;
      }
      __syncthreads();
      double tot = 0.0;
      cnt = 0.0;
      for (int w = 0; w < kRcThreads / 32; ++w) {
        tot += red[w];
        cnt += red2[w];
      }
      return tot;
    };
    const double target = count_rule ? static_cast<double>(a.topk) : 1.0 - static_cast<double>(a.thr);
    const uint64_t kInf = 0x7FF0000000000000ull;     // nothing is >= this pattern
    bool keep_all = count_rule ? a.topk >= Nb : !(a.thr > 0.0f);
    int kept_listed = 0;
    uint64_t lo = 0, hi = kInf;
    double above = 0.0;           // mass (count) of the values >= hi
    if (!keep_all) {
      double cnt;
      if (!(mass_in(0, kInf, cnt) >= target)) {
        keep_all = true;                 // the sums never reach 1 - thr
      } else {
        // invariant: above < target <= above + mass[lo, hi); stops at one
        // pattern (equal values) at the latest
        while (cnt > kRcList && hi - lo > 1) {
          const uint64_t mid = lo + ((hi - lo) >> 1);
          double cu;
          const double up = mass_in(mid, hi, cu);
          if (above + up >= target) {
            lo = mid;
            cnt = cu;
          } else {
            above += up;
            hi = mid;
            cnt -= cu;
          }
        }
        if (cnt > kRcList) {
          // more than the list holds, all equal to the pattern lo: the
          // first `need` of them in index order are kept
          const double v = count_rule ? 1.0 : __longlong_as_double(static_cast<long long>(lo));
          int j = static_cast<int>(fmin(ceil((target - above) / v), static_cast<double>(Nb)));
          if (j < 1) j = 1;
          while (j > 1 && above + (j - 1) * v >= target) --j;
          while (above + j * v < target && j < Nb) ++j;
          if (warp == 0) {
            int ties_seen = 0;
            for (int w = 0; w < a.words; ++w) {
              const int c = w * 32 + lane;
              const uint64_t kc = c < Nb ? static_cast<uint64_t>(__double_as_longlong(pv[c])) : 0ull;
              const bool tie = c < Nb && kc == lo;
              const uint32_t tm = __ballot_sync(0xFFFFFFFFu, tie);
              const bool kept = tie && ties_seen + __popc(tm & ((1u << lane) - 1u)) < j;
              const uint32_t word = __ballot_sync(0xFFFFFFFFu, kept);
              if (lane == 0) bits[w] |= word;
              ties_seen += __popc(tm);
            }
          }
          __syncthreads();
        } else {
        // the values in [lo, hi): list, sort on (value desc, index asc), walk
        if (tid == 0) nlist = 0;
        __syncthreads();
        for (int c = tid; c < Nb; c += kRcThreads) {
          const uint64_t kc = static_cast<uint64_t>(__double_as_longlong(pv[c]));
          if (kc >= lo && kc < hi) {
            const int pos = atomicAdd(&nlist, 1);
            lp[pos] = pv[c];
            li[pos] = c;
          }
        }
        __syncthreads();
        const int nl = nlist;
        for (int v = nl + tid; v < kRcList; v += kRcThreads) {
          lp[v] = -1.0;
          li[v] = INT_MAX;
        }
        __syncthreads();
        for (int size = 2; size <= kRcList; size <<= 1)
          for (int stride = size >> 1; stride > 0; stride >>= 1) {
            const int x = tid, y = x ^ stride;
            if (y > x) {
              const bool up = (x & size) == 0;
              const bool first = lp[x] > lp[y] || (lp[x] == lp[y] && li[x] < li[y]);
              if (first != up) {
                const double tp = lp[x]; lp[x] = lp[y]; lp[y] = tp;
                const int ti = li[x]; li[x] = li[y]; li[y] = ti;
              }
            }
            __syncthreads();
          }
        if (tid == 0) {
          // kept while the mass before the value is below the target
          double mass = above;
          int k = 0;
          while (k < nl && mass < target) {
            mass += count_rule ? 1.0 : lp[k];
            ++k;
          }
          nlist = k;
        }
        __syncthreads();
        kept_listed = nlist;
        }
      }
    }
    // kept bits: every value >= hi, and the first kept_listed of the list
    for (int c = tid; c < Nb; c += kRcThreads) {
      const uint64_t kc = static_cast<uint64_t>(__double_as_longlong(pv[c]));
      if (keep_all || kc >= hi) atomicOr(&bits[c >> 5], 1u << (c & 31));
    }
    for (int v = tid; v < kept_listed; v += kRcThreads)
      atomicOr(&bits[li[v] >> 5], 1u << (li[v] & 31));
    __syncthreads();
    if (a.use_sta) {
      const int hw = a.Hb * a.Wb;
      const int tr = r / hw, yr = (r / a.Wb) % a.Hb, xr = r % a.Wb;
      const int nt = 2 * a.rt + 1, ny = 2 * a.rh + 1, nx = 2 * a.rw + 1;
      for (int v = tid; v < nt * ny * nx; v += kRcThreads) {
        const int t3 = tr - a.rt + v / (ny * nx);
        const int yy = yr - a.rh + (v / nx) % ny;
        const int xx = xr - a.rw + v % nx;
        if (t3 >= 0 && t3 < a.T && yy >= 0 && yy < a.Hb && xx >= 0 && xx < a.Wb) {
          const int c = (t3 * a.Hb + yy) * a.Wb + xx;
          atomicOr(&bits[c >> 5], 1u << (c & 31));
        }
      }
      __syncthreads();
    }
    int count = 0;
    for (int w = tid; w < a.words; w += kRcThreads) {
      const uint32_t x = bits[w];
      a.bits[g * a.words + w] = x;
      count += __popc(x);
    }
    count = warp_sum_i(count);
    if (lane == 0) red[warp] = static_cast<double>(count);
    __syncthreads();
    if (tid == 0) {
      double tot = 0.0;
      for (int w = 0; w < kRcThreads / 32; ++w) tot += red[w];
      a.counts[g] = static_cast<int32_t>(tot);
    }
    __syncthreads();
    if (!ok_sh) break;           // a stage never arrived: stop (recorded)
  }
}

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

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct MaskLayout {
  int64_t rows, plane_rows;
  int words, np2, ld, ldk, ldp;
  size_t qdig_off, kdig_off, qexp_off, kexp_off, kscale_off, slab_off, rec_off, bits_off,
      counts_off, flag_off, nflag_off, sums_off, total;
  int sel_warps;
  size_t smem_select, smem_recheck;
};

MaskLayout mask_layout(const Geometry &g) {
  MaskLayout L;
  L.rows = g.BH * g.Nb;
  // digit planes hold at least one whole 128-row box
  L.plane_rows = L.rows > kTileRows ? L.rows : kTileRows;
  L.words = static_cast<int>((g.Nb + 31) / 32);
  L.np2 = 1;
  while (L.np2 < g.Nb) L.np2 <<= 1;
  L.ld = static_cast<int>((g.Nb + 15) & ~15LL);      // slab row: whole 16-column slices
  L.ldk = static_cast<int>((g.Nb + 63) & ~63LL);     // per-head K scales: whole chunks
  L.ldp = static_cast<int>((g.Nb + 31) & ~31LL);
  const size_t plane = static_cast<size_t>(kDigits) * L.plane_rows * kRowBytes;
  size_t off = 0;
  L.qdig_off = off; off = align256(off + plane);
  L.kdig_off = off; off = align256(off + plane);
  L.qexp_off = off; off = align256(off + static_cast<size_t>(L.rows) * 4);
  L.kexp_off = off; off = align256(off + static_cast<size_t>(L.rows) * 4);
  L.kscale_off = off; off = align256(off + static_cast<size_t>(g.BH) * L.ldk * 4);
  L.slab_off = off; off = align256(off + static_cast<size_t>(L.rows) * L.ld * 4);
  L.rec_off = off; off = align256(off + static_cast<size_t>(L.rows) * sizeof(RowRec));
  L.bits_off = off; off = align256(off + static_cast<size_t>(L.rows) * L.words * 4);
  L.counts_off = off; off = align256(off + static_cast<size_t>(L.rows) * 4);
  L.flag_off = off; off = align256(off + static_cast<size_t>(L.rows) * 4);
  L.nflag_off = off; off = align256(off + 16);
  L.sums_off = off; off = align256(off + static_cast<size_t>(L.rows / 1024 + 2) * 8);
  L.total = off;
  // as many rows per select CTA as 200 KiB of SMEM hold, at most kSelWarps
  const size_t pw = select_warp_bytes(L.ldp, L.words);
  L.sel_warps = static_cast<int>(pw <= (200u << 10) / kSelWarps ? kSelWarps : (200u << 10) / pw);
  if (L.sel_warps < 1) L.sel_warps = 1;
  L.smem_select = static_cast<size_t>(L.sel_warps) * pw;
  L.smem_recheck = recheck_smem_bytes(L.ldp, L.words, g.d);
  return L;
}

// The digit planes [4][plane_rows][128 B] as a 3-D map: one box = a whole
// row range of all four planes, 128-byte swizzled.
bool make_map_digits(CUtensorMap *m, const void *base, int64_t plane_rows, int box_rows) {
  EncodeFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {kRowBytes, static_cast<cuuint64_t>(plane_rows), kDigits};
  const cuuint64_t strides[2] = {kRowBytes, static_cast<cuuint64_t>(plane_rows) * kRowBytes};
  const cuuint32_t box[3] = {kRowBytes, static_cast<cuuint32_t>(box_rows), kDigits};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

}  // namespace

size_t block_mask_workspace_bytes(const Geometry &g) { return mask_layout(g).total; }

size_t block_mask_smem_bytes(const Geometry &g) {
  if (g.Nb > kMaxNb) return ~static_cast<size_t>(0) >> 1;   // reported as unsupported
  const MaskLayout L = mask_layout(g);
  size_t m = static_cast<size_t>(SmemA::kAlloc);
  if (L.smem_recheck > m) m = L.smem_recheck;
  if (L.smem_select > m) m = L.smem_select;
  return m;
}

cudaError_t launch_block_mask(const double *qp, const double *kp, const Geometry &g,
                              const vsa_mask_params &p, int topk, int64_t *row_ptr,
                              int32_t *col_idx, int32_t *kept_count, void *ws, unsigned *err,
                              cudaStream_t st) {
  const int64_t rows = g.BH * g.Nb;
  if (rows == 0) return cudaMemsetAsync(row_ptr, 0, sizeof(int64_t), st);
  const MaskLayout L = mask_layout(g);
  unsigned char *w = static_cast<unsigned char *>(ws);
  MaskArgs a;
  a.BH = g.BH; a.rows = rows; a.Nb = static_cast<int>(g.Nb); a.d = g.d;
  a.Hb = g.Hb; a.Wb = g.Wb; a.T = static_cast<int>(g.Nb / (static_cast<int64_t>(g.Hb) * g.Wb));
  a.thr = p.thr; a.topk = topk;
  a.use_sta = p.use_sta != 0; a.rt = p.sta_t; a.rh = p.sta_h; a.rw = p.sta_w;
  a.c_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(g.d)));
  a.scale = 1.0 / std::sqrt(static_cast<double>(g.d));
  a.qp = qp; a.kp = kp;
  int8_t *qdig = reinterpret_cast<int8_t *>(w + L.qdig_off);
  int8_t *kdig = reinterpret_cast<int8_t *>(w + L.kdig_off);
  int *qexp = reinterpret_cast<int *>(w + L.qexp_off);
  int *kexp = reinterpret_cast<int *>(w + L.kexp_off);
  float *kscale = reinterpret_cast<float *>(w + L.kscale_off);
  a.qexp = qexp; a.kexp = kexp; a.kscale = kscale; a.ldk = L.ldk;
  a.slab = reinterpret_cast<float *>(w + L.slab_off); a.ld = L.ld;
  a.rec = reinterpret_cast<RowRec *>(w + L.rec_off);
  a.bits = reinterpret_cast<uint32_t *>(w + L.bits_off);
  a.words = L.words;
  a.counts = kept_count ? kept_count : reinterpret_cast<int32_t *>(w + L.counts_off);
  a.flagged = reinterpret_cast<int32_t *>(w + L.flag_off);
  a.nflag = reinterpret_cast<int *>(w + L.nflag_off);
  a.tiles_per_head = static_cast<int>((g.Nb + kTileRows - 1) / kTileRows);
  a.nch = static_cast<int>((g.Nb + kChunk - 1) / kChunk);
  a.np2 = L.np2;
  a.units = g.BH * a.tiles_per_head;
  a.err = err;

  cudaError_t e;
  {
    const int64_t threads = 2 * rows * 32;
    mask_digits_kernel<<<static_cast<int>((threads + 255) / 256), 256, 0, st>>>(
        qp, kp, rows, L.plane_rows, g.d, a.Nb, L.ldk, qdig, kdig, qexp, kexp, kscale, a.nflag);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const bool keep_all = topk > 0 ? topk >= g.Nb : p.thr <= 0.0f;
  if (!keep_all) {
    CUtensorMap mq, mk;
    if (!make_map_digits(&mq, qdig, L.plane_rows, kTileRows) ||
        !make_map_digits(&mk, kdig, L.plane_rows, kChunk))
      return cudaErrorInvalidValue;
    int grid = num_sms();
    if (a.units < grid) grid = static_cast<int>(a.units);
    if ((e = cudaFuncSetAttribute(mask_scores_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  SmemA::kAlloc)) != cudaSuccess)
      return e;
    mask_scores_kernel<<<grid, kThreadsA, SmemA::kAlloc, st>>>(mq, mk, a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    const void *fn = topk > 0 ? reinterpret_cast<const void *>(mask_select_kernel<true>)
                              : reinterpret_cast<const void *>(mask_select_kernel<false>);
    if ((e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(L.smem_select))) != cudaSuccess)
      return e;
    const int64_t want = (rows + L.sel_warps - 1) / L.sel_warps;
    const int sg = static_cast<int>(want < 16LL * num_sms() ? want : 16LL * num_sms());
    const int threads = L.sel_warps * 32;
    if (topk > 0) mask_select_kernel<true><<<sg, threads, L.smem_select, st>>>(a, L.ldp);
    else mask_select_kernel<false><<<sg, threads, L.smem_select, st>>>(a, L.ldp);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if ((e = cudaFuncSetAttribute(mask_recheck_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(L.smem_recheck))) != cudaSuccess)
    return e;
  // a CTA per listed row, as many as fit on the GPU at once
  mask_recheck_kernel<<<2 * num_sms(), kRcThreads, L.smem_recheck, st>>>(a, L.ldp);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  {
    int64_t *sums = reinterpret_cast<int64_t *>(w + L.sums_off);
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
