// lime_debug_wait_timeout: a test hook for the failure detection of the
// tensor-core kernels.  Every mbarrier wait in them is bounded: after two
// seconds of the global timer it raises LIME_FLAG_TIMEOUT in the workspace's
// status word, raises the CTA's abort flag and returns, so the kernel ends and
// the context stays usable.  This entry point runs one kernel whose wait
// nothing can complete (a barrier that expects one arrival and never gets
// it), which exercises exactly that path: no fault, no trap, no unbounded
// loop.
#include "lime.h"
#include "sm100.cuh"

namespace lime {
namespace {

using namespace sm100;

__global__ void k_wait_never(unsigned* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  mbar_init(&bar, 1);
  abort_flag = 0;
  fence_mbar_init();
  // nothing arrives on `bar`: the wait gives up at its time limit
  mbar_wait(&bar, 0, status, &abort_flag);
}

}  // namespace
}  // namespace lime

extern "C" int lime_debug_wait_timeout(void* workspace, cudaStream_t stream) {
  if (!workspace || ((uintptr_t)workspace & 255)) return LIME_ERR_ARG;
  lime::k_wait_never<<<1, 1, 0, stream>>>(reinterpret_cast<unsigned*>(workspace));
  lime::note_launches(1);
  return cudaGetLastError() == cudaSuccess ? LIME_OK : LIME_ERR_CUDA;
}
