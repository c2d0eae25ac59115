// kq_inst_mma.cu — explicit instantiations of the tensor-core GEMV kernel
// (2..8 activation columns).
#include "kq_mma.cuh"

namespace kq {
template cudaError_t launch_mma<1, 1>(const GemvArgs&, const LaunchPlan&, cudaStream_t);
template cudaError_t launch_mma<1, 2>(const GemvArgs&, const LaunchPlan&, cudaStream_t);
template cudaError_t launch_mma<2, 1>(const GemvArgs&, const LaunchPlan&, cudaStream_t);
template cudaError_t launch_mma<2, 2>(const GemvArgs&, const LaunchPlan&, cudaStream_t);
template cudaError_t mma_active_clusters<1, 1>(int, size_t, int*);
template cudaError_t mma_active_clusters<1, 2>(int, size_t, int*);
template cudaError_t mma_active_clusters<2, 1>(int, size_t, int*);
template cudaError_t mma_active_clusters<2, 2>(int, size_t, int*);
}  // namespace kq
