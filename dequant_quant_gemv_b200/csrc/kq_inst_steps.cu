// kq_inst_steps.cu — instantiation of the multi-step single-column kernel.
#include "kq_steps.cuh"

namespace kq {
template cudaError_t launch_steps<2>(const StepsArgs&, int, size_t, bool, cudaStream_t);
}  // namespace kq
