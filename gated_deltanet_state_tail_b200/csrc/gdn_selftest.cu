// gdn_selftest.cu -- self-tests of the device-side failure paths.  Every
// kernel's bounded waits: a wait that runs out sets kStatusTimeout and the
// wait site in the workspace header, and the kernel returns instead of hanging
// or trapping, so the context stays usable and the host reads the status with
// gdn_workspace_status().  The debug build's index checks: a failing check
// sets kStatusBounds and skips the access it guards.
#include <cuda_runtime.h>

#include "gdn_internal.h"
#include "gdn_sm100.h"
#include "gdn_tail_replay.h"

namespace gdn {
namespace {

constexpr unsigned int kSelftestWhere = 99u;   // wait-site code reported by the self-test

// One thread waits, bounded by limit_ns, on an mbarrier that nothing arrives on.
__global__ void bounded_wait_selftest_kernel(WorkspaceHeader* ws, unsigned int epoch, unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    ws->epoch = epoch;
    sm100::mbar_init(&bar, 1);
    sm100::mbar_fence_init();
    if (!sm100::mbar_wait_bounded(&bar, 0u, limit_ns)) {
        tag_merge(&ws->status, epoch, kStatusTimeout, false);
        tag_merge(&ws->where, epoch, kSelftestWhere, true);
    }
}

// The debug build's index check on an index one past a stated 4-element extent:
// the check records kStatusBounds and skips the store it guards.  (The index
// is still inside the header's pad array, so even an unchecked store would
// stay in the caller's workspace.)
__global__ void index_check_selftest_kernel(WorkspaceHeader* ws, unsigned int epoch) {
    const long long extent = 4, idx = extent;   // one past the end
    ws->epoch = epoch;
    if (index_ok(ws, epoch, idx < extent)) ws->pad[idx] = 1u;
}

}  // namespace
}  // namespace gdn

extern "C" gdn_status gdn_selftest_bounded_wait(uint64_t limit_ns, void* workspace, void* stream) {
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 15u) != 0) return GDN_ERR_INVALID_ARG;
    if (limit_ns == 0 || limit_ns > 1000000000ull) return GDN_ERR_INVALID_ARG;   // at most 1 s
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    auto* ws = static_cast<gdn::WorkspaceHeader*>(workspace);
    gdn::bounded_wait_selftest_kernel<<<1, 1, 0, st>>>(ws, gdn::next_call_number(), (unsigned long long)limit_ns);
    if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
    return GDN_OK;
}

extern "C" gdn_status gdn_selftest_index_check(void* workspace, void* stream) {
    if (!gdn::kDebugBounds) return GDN_ERR_UNSUPPORTED;   // the release build has no index checks
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 15u) != 0) return GDN_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    auto* ws = static_cast<gdn::WorkspaceHeader*>(workspace);
    gdn::index_check_selftest_kernel<<<1, 1, 0, st>>>(ws, gdn::next_call_number());
    if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
    return GDN_OK;
}

extern "C" int32_t gdn_debug_bounds_enabled(void) { return gdn::kDebugBounds ? 1 : 0; }
