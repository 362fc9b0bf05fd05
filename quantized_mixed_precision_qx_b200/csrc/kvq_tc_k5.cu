// Tensor-core decode instantiations for K format id 5 (all V formats).
#include "kvq_tc_launch.cuh"

namespace kvq {
namespace tc {
template <>
cudaError_t launch_for_k<5>(int vf, const Args& a, dim3 grid, size_t smem, cudaStream_t st) {
    KVQ_TC_V_CASES(5)
}
}  // namespace tc
}  // namespace kvq
