// k_flatten.cu -- fractal flattening and its inverse (NABLA, Methodology
// item 1: every P x P spatial patch becomes one contiguous run of tokens, the
// time axis keeps its order).
//
// With P = 8, the 8 raster tokens (t, y, 8*px .. 8*px+7) of one patch row are
// also 8 consecutive tokens in flattened order, at
//   f = t*H*W + ((y/8)*(W/8) + px)*64 + (y%8)*8.
// So the permutation moves contiguous runs of 8*d bf16 (2 KiB at d = 128):
// one warp copies one run with 16-byte vector loads and streaming stores,
// fully coalesced on both sides.  Pure HBM stream: 2*N*d*2 bytes per tensor.
#include "vsa_device.cuh"
#include "vsa_internal.h"

namespace vsa {
namespace {

template <bool kInverse>
__global__ void __launch_bounds__(256) fractal_permute_kernel(const uint4 *__restrict__ src,
                                                              uint4 *__restrict__ dst,
                                                              int64_t runs, int T, int H, int W,
                                                              int vec_per_run) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int Wp = W >> 3;
  const int64_t N = static_cast<int64_t>(T) * H * W;
  for (int64_t run = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
       run < runs; run += warps) {
    // run = ((bh*T + t)*H + y)*Wp + px
    int64_t r = run;
    const int px = static_cast<int>(r % Wp); r /= Wp;
    const int y = static_cast<int>(r % H); r /= H;
    const int t = static_cast<int>(r % T);
    const int64_t bh = r / T;
    const int64_t raster = bh * N + (static_cast<int64_t>(t) * H + y) * W + (px << 3);
    const int64_t flat = bh * N + static_cast<int64_t>(t) * H * W +
                         (static_cast<int64_t>(y >> 3) * Wp + px) * 64 + ((y & 7) << 3);
    const int64_t s0 = (kInverse ? flat : raster) * (vec_per_run >> 3);
    const int64_t d0 = (kInverse ? raster : flat) * (vec_per_run >> 3);
#pragma unroll 4
    for (int i = lane; i < vec_per_run; i += 32) __stcs(dst + d0 + i, __ldcs(src + s0 + i));
  }
}

}  // namespace

cudaError_t launch_fractal_permute(const void *src, void *dst, const Geometry &g, bool inverse,
                                   cudaStream_t st) {
  const int64_t runs = g.BH * g.T * g.H * (g.W >> 3);
  const int vec_per_run = g.d;  // 8 tokens * d bf16 * 2 B / 16 B
  if (runs == 0) return cudaSuccess;
  const int64_t want = (runs + 7) / 8;
  const int blocks = static_cast<int>(want < 32LL * num_sms() ? want : 32LL * num_sms());
  if (inverse)
    fractal_permute_kernel<true><<<blocks, 256, 0, st>>>(
        static_cast<const uint4 *>(src), static_cast<uint4 *>(dst), runs, g.T, g.H, g.W,
        vec_per_run);
  else
    fractal_permute_kernel<false><<<blocks, 256, 0, st>>>(
        static_cast<const uint4 *>(src), static_cast<uint4 *>(dst), runs, g.T, g.H, g.W,
        vec_per_run);
  return cudaGetLastError();
}

}  // namespace vsa
