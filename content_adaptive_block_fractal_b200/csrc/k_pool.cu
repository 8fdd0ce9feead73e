// k_pool.cu -- 64-token block mean pooling of Q and K (NABLA, Methodology
// item 2, "downsampling": Q and K are cut into blocks and mean-pooled).
//
// One warp reduces one block of 64 consecutive flattened tokens.  A token row
// of d bf16 is read by d/8 lanes with 16-byte loads (a warp covers 32/(d/8)
// rows per step), so every load instruction moves 512 contiguous bytes.  Each
// bf16 is widened to fp64 with integer ops (exact) and summed in fp64.  With
// 8 significant bits per bf16, a sum of 64 of them fits fp64's 53 bits when
// the nonzero magnitudes lie within 2^39 of each other, so the sum (in any
// order) and the final /64 are exact and the output is the exact block mean.
// HBM-bound: reads 2*N*d*2 bytes per (batch, head), writes 2*Nb*d*8.
#include "vsa_device.cuh"
#include "vsa_internal.h"

namespace vsa {
namespace {

// Exact bf16 -> fp64 widening.  Normal numbers are rebiased with integer ops
// (exponent + 1023 - 127, mantissa moved to the top of the fp64 fraction);
// zeros, subnormals, infinities and NaNs take the float path, also exact.
__device__ __forceinline__ double bf16_to_f64(uint32_t b) {
  const uint32_t e = b & 0x7F80u;
  if (e != 0u && e != 0x7F80u) {
    const uint32_t hi = (((b & 0x7FFFu) << 13) + 0x38000000u) | ((b & 0x8000u) << 16);
    return __hiloint2double(static_cast<int>(hi), 0);
  }
  return static_cast<double>(__uint_as_float(b << 16));
}

template <int D>
__global__ void __launch_bounds__(256) pool_kernel(const uint4 *__restrict__ q,
                                                   const uint4 *__restrict__ k,
                                                   double *__restrict__ qp,
                                                   double *__restrict__ kp, int64_t blocks) {
  constexpr int kLanesPerRow = D / 8;            // 16-byte vectors per token row
  constexpr int kRowsPerStep = 32 / kLanesPerRow;
  const int lane = threadIdx.x & 31;
  const int sub = lane / kLanesPerRow;           // which row of the step
  const int col = lane % kLanesPerRow;           // which 8 columns
  const int64_t warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
       w < 2 * blocks; w += warps) {
    const bool is_k = w >= blocks;
    const int64_t blk = is_k ? w - blocks : w;
    const uint4 *src = (is_k ? k : q) + blk * 64 * kLanesPerRow;
    double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll 8
    for (int r = sub; r < 64; r += kRowsPerStep) {
      const uint4 v = __ldcs(src + r * kLanesPerRow + col);
      const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        acc[2 * j] += bf16_to_f64(u[j] & 0xFFFFu);
        acc[2 * j + 1] += bf16_to_f64(u[j] >> 16);
      }
    }
#pragma unroll
    for (int off = kLanesPerRow; off < 32; off <<= 1)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] += __shfl_xor_sync(0xFFFFFFFFu, acc[j], off);
    if (sub == 0) {
      double *dst = (is_k ? kp : qp) + blk * D + col * 8;
      double2 *d2 = reinterpret_cast<double2 *>(dst);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        d2[j] = make_double2(acc[2 * j] * 0.015625, acc[2 * j + 1] * 0.015625);
    }
  }
}

// Steps 1 and 2 in one pass over Q and K.  One warp takes one 64-token block
// (one P x P patch of one frame): it reads the block's 8 raster runs of 8
// tokens, writes them as the block's contiguous 64 flattened tokens, and sums
// the columns on the way, so the flattened tensors are never read back.  Lane
// l always holds 16-byte column group l % (D/8) of its tokens, which keeps
// its 8 fp64 accumulators on fixed columns (the same split as pool_kernel,
// hence the same exact sums).  Units [0, blocks) are Q, [blocks, 2*blocks) K.
// kFlat false: the flattened copies are not written (the attention then reads
// the raster tensors through patch-addressed TMA boxes), only the means.
template <int D, bool kFlat>
__global__ void __launch_bounds__(256)
    flatten_pool_kernel(const uint4 *__restrict__ q, const uint4 *__restrict__ k,
                        uint4 *__restrict__ qf, uint4 *__restrict__ kf, double *__restrict__ qp,
                        double *__restrict__ kp, int64_t blocks, int64_t Nb, int H, int W) {
  constexpr int kVecPerRow = D / 8;              // 16-byte vectors per token
  constexpr int kVecPerRun = 8 * kVecPerRow;     // one patch row: 8 tokens
  constexpr int kPerLane = kVecPerRun / 32;      // vectors per lane per run
  const int lane = threadIdx.x & 31;
  const int col = lane % kVecPerRow;
  const int Wb = W >> 3;
  const int64_t per_frame = static_cast<int64_t>(H >> 3) * Wb;
  const int64_t warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
       w < 2 * blocks; w += warps) {
    const bool is_k = w >= blocks;
    const int64_t g = is_k ? w - blocks : w;     // (bh, block) flattened
    const int64_t bh = g / Nb, blk = g % Nb;
    const int64_t t = blk / per_frame, rem = blk % per_frame;
    const int py = static_cast<int>(rem / Wb), px = static_cast<int>(rem % Wb);
    const int64_t head = bh * Nb * 64;           // first token of the head
    const uint4 *src = (is_k ? k : q) + (head + (t * H + py * 8) * W + px * 8) * kVecPerRow;
    uint4 *dst = kFlat ? (is_k ? kf : qf) + (head + blk * 64) * kVecPerRow : nullptr;
    double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll 2
    for (int i = 0; i < 8; ++i) {                // patch row i: raster row py*8 + i
      const uint4 *run = src + static_cast<int64_t>(i) * W * kVecPerRow;
      uint4 v[kPerLane];
#pragma unroll
      for (int j = 0; j < kPerLane; ++j) v[j] = __ldcs(run + lane + 32 * j);
#pragma unroll
      for (int j = 0; j < kPerLane; ++j) {
        if (kFlat) __stcs(dst + i * kVecPerRun + lane + 32 * j, v[j]);
        const uint32_t u[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc[2 * e] += bf16_to_f64(u[e] & 0xFFFFu);
          acc[2 * e + 1] += bf16_to_f64(u[e] >> 16);
        }
      }
    }
#pragma unroll
    for (int off = kVecPerRow; off < 32; off <<= 1)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] += __shfl_xor_sync(0xFFFFFFFFu, acc[j], off);
    if (lane < kVecPerRow) {
      double2 *d2 = reinterpret_cast<double2 *>((is_k ? kp : qp) + g * D + col * 8);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        d2[j] = make_double2(acc[2 * j] * 0.015625, acc[2 * j + 1] * 0.015625);
    }
  }
}

}  // namespace

cudaError_t launch_flatten_pool_qk(const void *q, const void *k, void *qf, void *kf, double *qp,
                                   double *kp, const Geometry &g, cudaStream_t st) {
  const int64_t blocks = g.BH * g.Nb;
  if (blocks == 0) return cudaSuccess;
  const int64_t want = (2 * blocks + 7) / 8;
  const int grid = static_cast<int>(want < 32LL * num_sms() ? want : 32LL * num_sms());
  const uint4 *q4 = static_cast<const uint4 *>(q);
  const uint4 *k4 = static_cast<const uint4 *>(k);
  uint4 *qf4 = static_cast<uint4 *>(qf);
  uint4 *kf4 = static_cast<uint4 *>(kf);
  const bool flat = qf != nullptr;
  if (g.d == 128)
    flat ? flatten_pool_kernel<128, true><<<grid, 256, 0, st>>>(q4, k4, qf4, kf4, qp, kp, blocks,
                                                                g.Nb, g.H, g.W)
         : flatten_pool_kernel<128, false><<<grid, 256, 0, st>>>(q4, k4, qf4, kf4, qp, kp, blocks,
                                                                 g.Nb, g.H, g.W);
  else
    flat ? flatten_pool_kernel<64, true><<<grid, 256, 0, st>>>(q4, k4, qf4, kf4, qp, kp, blocks,
                                                               g.Nb, g.H, g.W)
         : flatten_pool_kernel<64, false><<<grid, 256, 0, st>>>(q4, k4, qf4, kf4, qp, kp, blocks,
                                                                g.Nb, g.H, g.W);
  return cudaGetLastError();
}

cudaError_t launch_pool_qk(const void *qf, const void *kf, double *qp, double *kp,
                           const Geometry &g, cudaStream_t st) {
  const int64_t blocks = g.BH * g.Nb;
  if (blocks == 0) return cudaSuccess;
  const int64_t want = (2 * blocks + 7) / 8;
  const int grid = static_cast<int>(want < 32LL * num_sms() ? want : 32LL * num_sms());
  const uint4 *q = static_cast<const uint4 *>(qf);
  const uint4 *k = static_cast<const uint4 *>(kf);
  if (g.d == 128)
    pool_kernel<128><<<grid, 256, 0, st>>>(q, k, qp, kp, blocks);
  else
    pool_kernel<64><<<grid, 256, 0, st>>>(q, k, qp, kp, blocks);
  return cudaGetLastError();
}

}  // namespace vsa
