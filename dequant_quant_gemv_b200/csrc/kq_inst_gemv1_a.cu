// kq_inst_gemv1_a.cu — explicit instantiations of the single-matrix kernel (Q4_K, Q6_K).
#include "kq_gemv1.cuh"

namespace kq {
template cudaError_t launch_gemv1<1, false>(const GemvArgs&, const LaunchPlan&, cudaStream_t);
template cudaError_t launch_gemv1<1, true>(const GemvArgs&, const LaunchPlan&, cudaStream_t);
template cudaError_t launch_gemv1<2, false>(const GemvArgs&, const LaunchPlan&, cudaStream_t);
template cudaError_t launch_gemv1<2, true>(const GemvArgs&, const LaunchPlan&, cudaStream_t);
}  // namespace kq
