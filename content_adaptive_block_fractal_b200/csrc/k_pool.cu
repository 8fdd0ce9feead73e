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

}  // namespace

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
