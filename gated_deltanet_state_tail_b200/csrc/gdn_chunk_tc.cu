// gdn_chunk_tc.cu -- chunked WY/UT kernel on tcgen05 tensor cores (bf16, d = 128).
#include "gdn_internal.h"

namespace gdn {

bool chunk_tc_supported(int dtype, int dk, int dv) {
    (void)dtype; (void)dk; (void)dv;
    return false;
}

cudaError_t launch_chunk_tc(const CallArgs& a, cudaStream_t stream) {
    (void)a; (void)stream;
    return cudaErrorNotSupported;
}

}  // namespace gdn
