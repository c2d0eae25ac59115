// kq_inst_q6k_a.cu — explicit instantiations of the fused GEMV kernel (Q6_K).
#include "kq_gemv.cuh"

namespace kq {
template cudaError_t launch_one<2, 1, 2>(const GemvArgs&, const LaunchPlan&, cudaStream_t);
template cudaError_t launch_one<2, 2, 1>(const GemvArgs&, const LaunchPlan&, cudaStream_t);
}  // namespace kq
