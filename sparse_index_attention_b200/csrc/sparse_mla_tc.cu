// sparse_mla_tc.cu -- tensor-core (tcgen05) sparse MLA attention; filled in below.
#include "kernels.h"

namespace hsa {
bool sparse_mla_tc_supported(const SparseMlaArgs&) { return false; }
size_t sparse_mla_tc_workspace(int32_t, int32_t) { return 0; }
cudaError_t launch_sparse_mla_tc(const SparseMlaArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace hsa
