// diag.cu -- diagnostic of the bounded device-side wait.
//
// Every mbarrier wait in the library's kernels gives up after a limit, sets
// CSA_DEV_TIMEOUT in the device error word, and the CTA winds down (issued
// asynchronous work drains, TMEM is freed, the kernel returns) instead of
// hanging the GPU.  bounded_wait_probe runs that path on purpose, on a
// barrier no thread arrives at, with a short limit and nothing asynchronous
// in flight, so that a test can see the kernel return and the error word
// report the timeout while the context stays usable.
#include "common.cuh"
#include "sm100.cuh"

namespace csa {

using namespace sm100;

// One CTA of two warps.  Warp 0 holds a TMEM allocation across the wait
// (the resource a real kernel must release when it winds down); thread 0
// waits on the barrier.  With `arrive` set, thread 32 arrives after a tenth
// of the limit, so the wait completes; otherwise nothing arrives and the
// wait gives up after limit_ns.  waited_ns (nullable) receives the time
// thread 0 spent waiting.
__global__ void __launch_bounds__(64, 1)
    bounded_wait_probe(uint64_t limit_ns, int arrive, unsigned* err,
                       unsigned long long* waited_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t tbase_sm;
  __shared__ int abort_flag;
  volatile int* abort_sm = &abort_flag;
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    *abort_sm = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tbase_sm, 32);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tbase_sm;
  if (threadIdx.x == 0) {
    const uint64_t t0 = globaltimer();
    mbar_wait(&bar, 0, abort_sm, limit_ns);
    if (waited_ns) *waited_ns = (unsigned long long)(globaltimer() - t0);
  } else if (threadIdx.x == 32 && arrive) {
    const uint64_t t0 = globaltimer();
    while (globaltimer() - t0 < limit_ns / 10) __nanosleep(1000);
    mbar_arrive(&bar);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // the wind-down of the library's kernels
  if (*abort_sm && threadIdx.x == 0) atomicOr(err, CSA_DEV_TIMEOUT);
  if (warp == 0) tmem_dealloc(tbase, 32);
}

}  // namespace csa

using namespace csa;

extern "C" csa_status csa_diag_bounded_wait(uint64_t limit_ns, int arrive,
                                            uint64_t* waited_ns, csa_stream_t stream) {
  if (limit_ns == 0 || limit_ns > sm100::kWaitLimitNs) return CSA_ERR_ARG;
  if (arrive != 0 && arrive != 1) return CSA_ERR_ARG;
  unsigned* err = device_error_word();
  if (err == nullptr) return CSA_ERR_CUDA;
  cudaStream_t st = (cudaStream_t)stream;
  CSA_LAUNCH(KK_DIAG, st,
             bounded_wait_probe<<<1, 64, 0, st>>>(limit_ns, arrive, err,
                                                  (unsigned long long*)waited_ns));
  return last_launch_status();
}
