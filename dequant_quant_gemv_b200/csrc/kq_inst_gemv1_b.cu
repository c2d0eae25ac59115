// kq_inst_gemv1_b.cu — explicit instantiations of the single-matrix kernel (Q5_K, Q2_K, Q3_K, Q8_0).
#include "kq_gemv1.cuh"

namespace kq {
template cudaError_t launch_gemv1<3, false>(const GemvArgs&, const LaunchPlan&, cudaStream_t);
template cudaError_t launch_gemv1<3, true>(const GemvArgs&, const LaunchPlan&, cudaStream_t);
template cudaError_t launch_gemv1<4, false>(const GemvArgs&, const LaunchPlan&, cudaStream_t);
template cudaError_t launch_gemv1<4, true>(const GemvArgs&, const LaunchPlan&, cudaStream_t);
template cudaError_t launch_gemv1<5, false>(const GemvArgs&, const LaunchPlan&, cudaStream_t);
template cudaError_t launch_gemv1<5, true>(const GemvArgs&, const LaunchPlan&, cudaStream_t);
template cudaError_t launch_gemv1<6, false>(const GemvArgs&, const LaunchPlan&, cudaStream_t);
template cudaError_t launch_gemv1<6, true>(const GemvArgs&, const LaunchPlan&, cudaStream_t);
}  // namespace kq
