// selftest.cu -- a check of the error path that every streamed kernel and the GEMM share: a
// bounded wait that runs out records kErrTimeout in the workspace error word, which
// qlora_workspace_check reports. The kernel waits, with the library's bounded flag wait, on a
// workspace word that nothing sets; it faults and hangs nothing (the wait ends by itself after
// its poll limit, about a second).
#include "kernels.h"
#include "stream_common.cuh"

namespace qn {

namespace {

constexpr size_t kSelftestFlag = 192;  // a workspace word no kernel writes

__global__ void k_wait_timeout_selftest(int *err, const unsigned *flag) {
    if (threadIdx.x == 0 && !stream::wait_flag(flag)) stream::record_error(err, stream::kErrTimeout);
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(void *ws, cudaStream_t st) {
    char *b = static_cast<char *>(ws);
    k_wait_timeout_selftest<<<1, 32, 0, st>>>(reinterpret_cast<int *>(b),
                                                reinterpret_cast<const unsigned *>(b + kSelftestFlag));
    count_launch();
    return cudaGetLastError();
}

}  // namespace qn
