// wait_probe.cu -- test kernel for the bounded mbarrier wait that every
// tensor-core kernel of libdla uses (mbar_wait in tc_ptx.cuh).
//
// One CTA initialises an mbarrier with an arrival count of 1.  Unless
// `arrive` is set, nothing ever arrives on it and no asynchronous copy or MMA
// is issued, so the wait can only end through its poll limit: it must return
// false, raise the CTA's abort flag, and a second wait must then return at
// once.  The kernel reports DLA_ERR_TIMEOUT through the status word, as the
// library's kernels do.  With `arrive` set, the phase completes and the wait
// must return true.  Test infrastructure only (built by the tests).
#include "../../dynamic_state_memory_b200/csrc/dla_internal.cuh"
#include "../../dynamic_state_memory_b200/csrc/tc_ptx.cuh"

namespace {

__global__ void k_wait_probe(int arrive, uint32_t limit, int32_t *status, int32_t *out) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    dla::tc::mbar_init(&bar, 1);
    dla::tc::fence_mbar_init();
    abort_flag = 0;
  }
  __syncthreads();
  if (threadIdx.x == 0 && arrive) dla::tc::mbar_arrive(&bar);
  __syncthreads();
  const bool ok = dla::tc::mbar_wait(&bar, 0, &abort_flag, limit);
  __syncthreads();
  // once the flag is up, a later wait gives up at its first poll
  const long long t0 = clock64();
  const bool ok2 = dla::tc::mbar_wait(&bar, 0, &abort_flag, limit);
  const long long dt = clock64() - t0;
  __syncthreads();
  if (threadIdx.x == 0) {
    out[0] = ok ? 1 : 0;
    out[1] = abort_flag;
    out[2] = ok2 ? 1 : 0;
    out[3] = (int32_t)(dt < 0x7fffffffLL ? dt : 0x7fffffffLL);
    if (abort_flag) dla::set_status(status, DLA_ERR_TIMEOUT);
  }
}

}  // namespace

// out[0]: first wait's result, out[1]: abort flag, out[2]: second wait's
// result, out[3]: cycles the second wait took (thread 0).
extern "C" int dla_probe_bounded_wait(int arrive, unsigned limit, int32_t *status, int32_t *out,
                                      void *stream) {
  k_wait_probe<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(arrive, limit, status, out);
  return static_cast<int>(cudaGetLastError());
}
