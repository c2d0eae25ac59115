// kq_inst_q5k.cu — explicit instantiation of the fused GEMV kernel (Q5_K,
// one column; several columns run on the tensor-core kernel).
#include "kq_gemv.cuh"

namespace kq {
template cudaError_t launch_one<3, 1, 2>(const GemvArgs&, const LaunchPlan&, cudaStream_t);
}  // namespace kq
