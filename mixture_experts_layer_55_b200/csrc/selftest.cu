// selftest.cu -- exercises the failure path that every pipelined kernel of the
// library relies on: a bounded mbarrier wait that gives up, records the
// timeout flag and its location in the workspace status word, and lets the
// kernel return normally (no trap, the context stays usable).
#include "common.cuh"
#include "internal.h"

namespace moe {

constexpr int kSelftestWhere = 900;

// One thread waits on an mbarrier that nothing arrives at, with the given
// limit; the wait must give up.  `done` receives 1 once the kernel got past
// the wait (so the host can tell a clean return from a kernel that never ran).
__global__ void selftest_wait_kernel(int* status, uint64_t limit_ns, int* done)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_mbar_init();
    const bool ok = mbar_wait(&bar, 0, status, kSelftestWhere, nullptr, limit_ns);
    done[0] = ok ? 2 : 1;  // 1: gave up as designed; 2: the phase completed (impossible)
}

}  // namespace moe

using namespace moe;

extern "C" moe_status moe_selftest_wait_timeout(void* workspace, size_t workspace_bytes,
                                                int64_t limit_ns, void* stream)
{
    // the status word (words 0-1) and a "done" word (word 2) of the workspace
    if (workspace == nullptr || workspace_bytes < 64 * sizeof(int)) return MOE_ERR_WORKSPACE;
    if (((uintptr_t)workspace & (kAlign - 1)) != 0) return MOE_ERR_ALIGN;
    if (limit_ns < 1000 || limit_ns > 1000000000LL) return MOE_ERR_ARG;  // 1 us .. 1 s
    int* st = static_cast<int*>(workspace);
    selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(st, (uint64_t)limit_ns,
                                                                          st + 2);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
