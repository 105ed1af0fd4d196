// kla_chunk_tc.cu -- tensor-core (tcgen05) chunk forward; placeholder until written.
#include "kla_launch.h"

namespace kla {

bool chunk_fwd_tc_supported(const FwdArgs&) { return false; }

cudaError_t launch_chunk_fwd_tc(const FwdArgs&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace kla
