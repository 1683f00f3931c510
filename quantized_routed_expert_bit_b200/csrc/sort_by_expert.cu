// The stand-alone grouping kernel (moe_sort_by_expert, and the batched paths
// of moe_expert_ffn, whose selection comes from the caller): one CTA of 32
// warps runs the counting sort of sort_pairs.cuh. moe_layer_forward and
// moe_stack_forward run the same sort in the tail of the router kernel
// instead (route_topk.cu).

#include "sort_pairs.cuh"

namespace moe {

namespace {

constexpr int kThreads = 1024;

__global__ void __launch_bounds__(kThreads) sort_by_expert_kernel(const __grid_constant__ SortParams p, bool cache) {
  extern __shared__ int sh[];
  sort_pairs(p, sh, cache);
}

}  // namespace

cudaError_t launch_sort_by_expert(const SortParams& p, cudaStream_t stream) {
  // the selection is copied to shared memory when it fits in 96 KB
  const bool cache = sort_pairs_smem(p.E, p.with_shared, kThreads / 32, p.T, p.k, true) <= 96 * 1024;
  const size_t smem = sort_pairs_smem(p.E, p.with_shared, kThreads / 32, p.T, p.k, cache);
  cudaError_t e = cudaFuncSetAttribute(sort_by_expert_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  sort_by_expert_kernel<<<1, kThreads, smem, stream>>>(p, cache);
  return cudaGetLastError();
}

}  // namespace moe
