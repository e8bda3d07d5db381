// Prefill grouped GEMM on the tensor cores (placeholder until the tcgen05
// kernel lands: reports unsupported, so prefill uses the grouped GEMV).
#include "ft_internal.cuh"

namespace ft {
bool prefill_tc_supported(const Shape&) { return false; }
cudaError_t prefill_tc_init(const Shape&, int) { return cudaSuccess; }
void launch_prefill_tc(const Shape&, int, const void*, int, DevState&, cudaStream_t) {}
}  // namespace ft
