// Diagnostics: exercise the bounded-wait machinery every kernel uses, without
// faulting, trapping or hanging the GPU.  One CTA waits on an mbarrier that
// nothing arrives on; the wait gives up after the configured wall-clock limit
// and the kernel records DSA_ERR_TIMEOUT in the device error word, exactly as
// a real kernel would when a producer or a peer CTA stops making progress.
#include "internal.h"
#include "sm100.cuh"

namespace dsa {
namespace {

using namespace sm100;

__global__ void wait_timeout_probe_kernel(long long wait_ns, DevErr* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const AbortSources ab{&abort_flag, &err->code};
  // phase 0 never completes: nobody arrives
  const bool ok = mbar_wait(&bar, 0, wait_ns, ab);
  if (!ok) report_error(err, DSA_ERR_TIMEOUT, 0x50u | (threadIdx.x << 8));
  __syncthreads();
  // complete the phase so the barrier is left in a consistent state
  if (threadIdx.x == 0) mbar_arrive(&bar);
}

}  // namespace

cudaError_t launch_wait_timeout_probe(const LaunchCtx& c) {
  wait_timeout_probe_kernel<<<1, 32, 0, c.stream>>>(c.wait_ns, c.err);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace dsa
