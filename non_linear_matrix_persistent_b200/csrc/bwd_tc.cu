// tcgen05 backward (placeholder until the tensor-core BPTT kernel lands).
#include "kernels.h"

namespace m2rnn {

size_t bwd_tc_workspace(int, int, int, int, int) { return 0; }

cudaError_t launch_bwd_tc(const Params&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace m2rnn
