// index_score_tc.cu -- tensor-core (tcgen05) index score; filled in below.
#include "kernels.h"

namespace hsa {
bool index_score_tc_supported(const IndexScoreArgs&) { return false; }
cudaError_t launch_index_score_tc(const IndexScoreArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace hsa
