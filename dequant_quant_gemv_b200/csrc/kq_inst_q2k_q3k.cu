// kq_inst_q2k_q3k.cu — explicit instantiations of the fused GEMV kernel for
// Q2_K, Q3_K and Q8_0 (one column; several columns run one launch per
// column).
#include "kq_gemv.cuh"

namespace kq {
template cudaError_t launch_one<4, 1, 2>(const GemvArgs&, const LaunchPlan&, cudaStream_t);
template cudaError_t launch_one<5, 1, 2>(const GemvArgs&, const LaunchPlan&, cudaStream_t);
template cudaError_t launch_one<6, 1, 2>(const GemvArgs&, const LaunchPlan&, cudaStream_t);
}  // namespace kq
