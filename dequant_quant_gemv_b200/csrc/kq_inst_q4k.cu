// kq_inst_q4k.cu — explicit instantiations of the fused GEMV kernel (Q4_K).
#include "kq_gemv.cuh"

namespace kq {
template cudaError_t launch_one<1, 1, 2>(const GemvArgs&, const LaunchPlan&, cudaStream_t);
template cudaError_t launch_one<1, 2, 1>(const GemvArgs&, const LaunchPlan&, cudaStream_t);
template cudaError_t launch_one<1, 4, 1>(const GemvArgs&, const LaunchPlan&, cudaStream_t);
template cudaError_t launch_one<1, 8, 1>(const GemvArgs&, const LaunchPlan&, cudaStream_t);
}  // namespace kq
