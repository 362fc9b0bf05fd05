// Tensor-core decode instantiations for K format id 2 (all V formats).
#include "kvq_tc_launch.cuh"

namespace kvq {
namespace tc {
template <>
cudaError_t launch_for_k<2>(int vf, const Args& a, dim3 grid, size_t smem, cudaStream_t st) {
    KVQ_TC_V_CASES(2)
}
}  // namespace tc
}  // namespace kvq
