// KDA chunked prefill on tcgen05 tensor cores (sm_100a).  Not built yet: the
// entry point reports KDA_ERR_UNSUPPORTED until the kernel lands.
#pragma once

#include "kda_common.cuh"

namespace kda {
namespace tc {

inline size_t workspace_bytes(int num_seqs) {
    (void)num_seqs;
    return 0;
}

inline int launch(const void *, const void *, const void *, const float *, const float *, const float *,
                  void *, float *, const int32_t *, int, int, int, int, int, int, void *, cudaStream_t,
                  char *msg, size_t msg_len) {
    snprintf(msg, msg_len, "tensor-core prefill is not available in this build");
    return KDA_ERR_UNSUPPORTED;
}

}  // namespace tc
}  // namespace kda
