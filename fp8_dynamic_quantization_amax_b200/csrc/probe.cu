// probe.cu -- a test hook for the failure path of the bounded waits.
//
// Every wait in the library's kernels gives up after a time limit, records
// kDevErrTimeout in the device error word and lets the kernel return, so that
// a stalled barrier never hangs the GPU and the context stays usable.  This
// kernel runs one such wait on an mbarrier that nothing completes, with a
// short limit, so that tests can exercise that path without a fault.  The
// whole warp waits, each lane with its own limit, and then agrees on giving
// up before a warp-wide step, the way the GEMM's MMA and epilogue warps do
// before their warp-wide tensor-memory instructions.
#include "hq_internal.cuh"
#include "ptx.cuh"

namespace hq {
namespace {

__global__ void k_bounded_wait_probe(unsigned long long limit_ns, unsigned* err) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    abort_flag = 0;
    ptx::fence_mbarrier_init();
  }
  __syncthreads();
  // phase 0 of a fresh barrier with one expected arrival: nothing arrives.
  // Lane l gives up after limit_ns * (1 + l / 32); the first lane to give up
  // raises abort_flag, which ends the other lanes' waits early.
  const unsigned long long mine = limit_ns + (limit_ns >> 5) * (threadIdx.x & 31u);
  const bool give_up = __any_sync(0xFFFFFFFFu, !ptx::mbar_wait(&bar, 0, &abort_flag, err, kDevErrTimeout, mine));
  // a warp-wide step that every lane reaches together
  const unsigned all = __ballot_sync(0xFFFFFFFFu, give_up);
  if (threadIdx.x == 0 && all != 0xFFFFFFFFu) atomicOr(err, kDevErrTimeout);
}

}  // namespace

cudaError_t launch_bounded_wait_probe(unsigned long long limit_ns, cudaStream_t stream) {
  unsigned* err = device_error_word();
  if (err == nullptr) return cudaErrorUnknown;
  k_bounded_wait_probe<<<1, 32, 0, stream>>>(limit_ns, err);
  return cudaGetLastError();
}

}  // namespace hq
