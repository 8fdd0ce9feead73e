// k_probe.cu -- the bounded-wait path, exercised on purpose.
//
// Every mbarrier wait of the library gives up after a cycle limit, records a
// code in the per-device error word and lets its kernel unwind, so that a
// protocol fault surfaces as a status on the host instead of a hung GPU.
// This kernel makes such a wait run out: one thread initialises an mbarrier
// that expects one arrival and waits for its first phase, which nothing ever
// completes.  The wait polls with a suspend hint until the limit passes, then
// records kErrWaitProbe and the kernel returns; no fault, no trap.
#include "vsa_device.cuh"
#include "vsa_internal.h"

namespace vsa {
namespace {

__global__ void wait_probe_kernel(long long limit, unsigned *err) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  fence_mbar_init();
  // phase 0 never completes: nobody arrives
  mbar_wait_for(b, 0, limit, err, kErrWaitProbe);
}

}  // namespace

cudaError_t launch_wait_probe(int64_t wait_cycles, unsigned *err, cudaStream_t st) {
  wait_probe_kernel<<<1, 1, 0, st>>>(static_cast<long long>(wait_cycles), err);
  return cudaGetLastError();
}

}  // namespace vsa
