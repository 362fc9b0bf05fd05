// kvq_tc_launch.cuh -- launch helpers of the tensor-core decode kernel; one translation
// unit per K format instantiates it for every V format (kvq_tc_k*.cu).
#pragma once
#include "kvq_decode_tc.cuh"

namespace kvq {
namespace tc {

template <int KF, int VF, int NB>
cudaError_t launch_nb(const Args& a, dim3 grid, size_t smem, cudaStream_t st) {
    static bool smem_raised = false;      // raise the dynamic shared memory limit once per kernel
    if (!smem_raised) {
        cudaError_t e = cudaFuncSetAttribute(decode_tc<KF, VF, NB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             227 * 1024);
        if (e != cudaSuccess) return e;
        smem_raised = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.dependent ? 1 : 0;
    cudaError_t e = cudaLaunchKernelEx(&cfg, decode_tc<KF, VF, NB>, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// head_dim 256 (8 blocks) or 128 (4 blocks)
template <int KF, int VF>
cudaError_t launch_one(const Args& a, dim3 grid, size_t smem, cudaStream_t st) {
    if (a.D == 256) return launch_nb<KF, VF, 8>(a, grid, smem, st);
    if (a.D == 128) return launch_nb<KF, VF, 4>(a, grid, smem, st);
    return cudaErrorInvalidValue;
}

template <int KF>
cudaError_t launch_for_k(int vf, const Args& a, dim3 grid, size_t smem, cudaStream_t st);

#define KVQ_TC_V_CASES(KF)                                          \
    switch (vf) {                                                   \
        case 0: return launch_one<KF, 0>(a, grid, smem, st);        \
        case 1: return launch_one<KF, 1>(a, grid, smem, st);        \
        case 2: return launch_one<KF, 2>(a, grid, smem, st);        \
        case 3: return launch_one<KF, 3>(a, grid, smem, st);        \
        case 4: return launch_one<KF, 4>(a, grid, smem, st);        \
        case 5: return launch_one<KF, 5>(a, grid, smem, st);        \
        case 6: return launch_one<KF, 6>(a, grid, smem, st);        \
        case 7: return launch_one<KF, 7>(a, grid, smem, st);        \
        case 8: return launch_one<KF, 8>(a, grid, smem, st);        \
        case 9: return launch_one<KF, 9>(a, grid, smem, st);        \
        case 10: return launch_one<KF, 10>(a, grid, smem, st);      \
        case 11: return launch_one<KF, 11>(a, grid, smem, st);      \
    }                                                               \
    return cudaErrorInvalidValue;

// dispatch over (K format, V format); float ring formats pair with themselves
cudaError_t launch_tc(int kf, int vf, const Args& a, dim3 grid, size_t smem, cudaStream_t st);

}  // namespace tc
}  // namespace kvq
