// kq_inst_q6k_c.cu — explicit instantiations of the fused GEMV kernel (Q6_K).
#include "kq_gemv.cuh"

namespace kq {
template cudaError_t launch_one<2, 8, 1>(const GemvArgs&, const LaunchPlan&, cudaStream_t);
}  // namespace kq
