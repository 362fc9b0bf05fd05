// Dispatch of the tensor-core decode kernel over (K format, V format), plus the
// 16-bit float ring instantiations.
#include "kvq_tc_launch.cuh"

namespace kvq {
namespace tc {

cudaError_t launch_tc(int kf, int vf, const Args& a, dim3 grid, size_t smem, cudaStream_t st) {
    if (kf == F_F16 && vf == F_F16) return launch_one<F_F16, F_F16>(a, grid, smem, st);
    if (kf == F_BF16 && vf == F_BF16) return launch_one<F_BF16, F_BF16>(a, grid, smem, st);
    switch (kf) {
        case 0: return launch_for_k<0>(vf, a, grid, smem, st);
        case 1: return launch_for_k<1>(vf, a, grid, smem, st);
        case 2: return launch_for_k<2>(vf, a, grid, smem, st);
        case 3: return launch_for_k<3>(vf, a, grid, smem, st);
        case 4: return launch_for_k<4>(vf, a, grid, smem, st);
        case 5: return launch_for_k<5>(vf, a, grid, smem, st);
        case 6: return launch_for_k<6>(vf, a, grid, smem, st);
        case 7: return launch_for_k<7>(vf, a, grid, smem, st);
        case 8: return launch_for_k<8>(vf, a, grid, smem, st);
        case 9: return launch_for_k<9>(vf, a, grid, smem, st);
        case 10: return launch_for_k<10>(vf, a, grid, smem, st);
        case 11: return launch_for_k<11>(vf, a, grid, smem, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace tc
}  // namespace kvq
