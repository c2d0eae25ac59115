// kq_inst_mma_q3k.cu — explicit instantiations of the tensor-core GEMV kernel
// (2..8 activation columns), Q3_K.
#include "kq_mma.cuh"

namespace kq {
#define KQ_MMA_INST(F, T, G)                                                                    \
    template cudaError_t launch_mma<F, T, G>(const GemvArgs&, const LaunchPlan&, cudaStream_t); \
    template cudaError_t mma_active_clusters<F, T, G>(int, size_t, bool, int*);
KQ_MMA_INST(5, 1, 1)
KQ_MMA_INST(5, 1, 2)
#undef KQ_MMA_INST
}  // namespace kq
