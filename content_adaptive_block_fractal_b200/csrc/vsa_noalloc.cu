// vsa_noalloc.cu -- block-sparse attention forward for callers that cannot
// allocate device memory.
//
// vsa_sparse_attn_fwd needs a small caller-provided workspace for its
// persistent scheduler (a work counter and the longest-first work list).  Some
// callers have no way to provide one: plugins whose host framework hands them
// only input and output tensors, processes that reserve all device memory at
// start-up and forbid allocation afterwards, and latency-critical paths where
// cudaMalloc/cudaFree would implicitly synchronise the device and stall other
// streams.  This entry point serves them from a fixed array in the library's
// own device memory instead.
//
// Limits and behaviour:
//   - the array holds kNoAllocScratchBytes (8 MiB): enough for about two
//     million 128-row query tiles; larger shapes are rejected with
//     VSA_ERR_CAPACITY before anything is launched;
//   - every GPU that loads the library holds the array until the process
//     exits;
//   - all calls on a device share the one array, and it keeps the contents of
//     the last call.  The scheduler's planning kernel rewrites the work list
//     and resets the work counter to zero at the start of every call, so no
//     state leaks from one call to the next -- but two calls whose work
//     overlaps on the GPU (different streams, or different host threads
//     without ordering) race on the array and give wrong results;
//   - the first call on each device looks up the array's device address
//     (cudaGetSymbolAddress, with that device current); make that first call
//     before capturing any stream.
// Nothing here calls cudaMalloc, cudaFree or an allocating library routine.
#include "vsa_internal.h"

#include <cstdio>
#include <mutex>

namespace vsa {
void set_last_error(const char *msg);
}

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on the current device, looked up once
// per device.  In host code the symbol is only a host-side stand-in: it must
// never be passed to a kernel directly.
void *scratch_address(cudaError_t *err) {
  static void *addr[kMaxDevices] = {};
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
    if ((*err = cudaGetSymbolAddress(&p, g_noalloc_scratch)) != cudaSuccess) return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace

extern "C" vsa_status vsa_sparse_attn_fwd_noalloc(const void *qf, const void *kf, const void *vf,
                                                  const int64_t *row_ptr, const int32_t *col_idx,
                                                  vsa_shape s, float scale, void *o, float *lse,
                                                  void *stream) {
  const size_t need = vsa_sparse_attn_workspace_size(s);
  if (need == 0) {
    // invalid shape: let the regular entry point report the reason
    return vsa_sparse_attn_fwd(qf, kf, vf, row_ptr, col_idx, s, scale, o, lse, nullptr, 0,
                               stream);
  }
  if (need > kNoAllocScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof msg,
             "no-alloc sparse attention: this shape needs %zu bytes of scheduler scratch, "
             "the built-in array holds %zu; use vsa_sparse_attn_fwd with a workspace",
             need, kNoAllocScratchBytes);
    vsa::set_last_error(msg);
    return VSA_ERR_CAPACITY;
  }
  cudaError_t e;
  void *ws = scratch_address(&e);
  if (!ws) {
    char msg[256];
    snprintf(msg, sizeof msg, "no-alloc sparse attention: scratch address lookup: %s",
             cudaGetErrorString(e));
    vsa::set_last_error(msg);
    return VSA_ERR_CUDA;
  }
  return vsa_sparse_attn_fwd(qf, kf, vf, row_ptr, col_idx, s, scale, o, lse, ws,
                             kNoAllocScratchBytes, stream);
}
