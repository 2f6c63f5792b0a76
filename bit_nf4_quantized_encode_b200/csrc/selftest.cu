// selftest.cu -- a self-test of the library's failure path: the bounded
// mbarrier wait that every pipeline kernel uses, run out on purpose.
//
// One CTA initialises an mbarrier that nothing ever arrives on and waits for
// its first phase through mbar_wait_for() with a short, caller-given limit.
// No TMA copy, MMA or other asynchronous operation is in flight, and no other
// thread or CTA waits on anything, so the wait can only end by giving up: the
// kernel then records kErrWaitTimeout in the library's device error flag (the
// same flag and bit a stuck pipeline would set) and returns.  The host reads
// the flag with qlora_read_device_errors(); the context stays usable.
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "qlora.h"
#include "sm100_ptx.cuh"

namespace qlora {

namespace {

// Longest limit the self-test accepts: about 50 ms at the B200's clocks.
constexpr long long kMaxSelftestCycles = 100000000ll;

__global__ void k_wait_selftest(long long limit_cycles, uint32_t* err, uint32_t* outcome) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool completed = mbar_wait_for(&bar, 0u, err, limit_cycles);
    if (outcome) *outcome = completed ? 2u : 1u;       // 1: gave up, as it must
  }
}

}  // namespace
}  // namespace qlora

using namespace qlora;

extern "C" qlora_status qlora_selftest_bounded_wait(int64_t limit_cycles, uint32_t* outcome,
                                                    qlora_stream_t stream) {
  if (limit_cycles < 0 || limit_cycles > kMaxSelftestCycles) return QLORA_ERR_SHAPE;
  if (outcome && (reinterpret_cast<uintptr_t>(outcome) & 3u) != 0) return QLORA_ERR_ALIGN;
  uint32_t* err = nullptr;
  const qlora_status st = device_error_flag(&err);
  if (st != QLORA_OK) return st;
  k_wait_selftest<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_cycles, err, outcome);
  return counted(cudaGetLastError()) == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}
