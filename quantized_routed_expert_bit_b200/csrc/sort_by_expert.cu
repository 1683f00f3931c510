// Grouping step of the batched path: the T*k (token, slot) pairs of a
// routing decision, grouped by expert in a stable (token, slot) order, with
// the shared expert as pseudo-expert E taken by every token. This is the
// counting sort the grouped expert GEMM consumes: experts become contiguous
// runs of pairs, so each expert's weights are read once for all of its
// tokens.
//
// One CTA: a shared-memory histogram, a scan into run offsets, then a
// stable scatter in pair order by one warp (match_any ranks equal experts
// inside each batch of 32 pairs, a per-expert cursor carries the order
// across batches).

#include "moe_common.cuh"
#include "moe_launch.h"

namespace moe {

namespace {

constexpr int kThreads = 1024;

__global__ void __launch_bounds__(kThreads) sort_by_expert_kernel(SortParams p) {
  extern __shared__ int sh[];  // counts / cursors [nbins]
  const int nbins = p.E + (p.with_shared ? 1 : 0);
  const int npairs = p.T * p.k + (p.with_shared ? p.T : 0);
  for (int i = threadIdx.x; i < nbins; i += blockDim.x) sh[i] = 0;
  __syncthreads();
  for (int q = threadIdx.x; q < npairs; q += blockDim.x) {
    const int e = (q < p.T * p.k) ? p.idx[q] : p.E;
    if (e < 0 || e >= nbins || (q < p.T * p.k && e >= p.E)) {
      report(p.hdr, MOE_ERR_BOUNDS, e);
      continue;
    }
    atomicAdd(&sh[e], 1);
  }
  __syncthreads();
  // exclusive scan by warp 0 (lane-strided blocks of bins)
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int per = (nbins + 31) / 32;
    const int b0 = lane * per, b1 = min(nbins, b0 + per);
    int local = 0;
    for (int b = b0; b < b1; ++b) local += sh[b];
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - local;
    for (int b = b0; b < b1; ++b) {
      const int c = sh[b];
      sh[b] = run;
      p.offsets[b] = run;
      run += c;
    }
    if (lane == 31) p.offsets[nbins] = incl;
    if (p.chunks) {
      // GEMM work list: every expert's run of pairs cut into chunks of <= chunk_tokens
      __syncwarp();
      int nloc = 0;
      for (int b = b0; b < b1; ++b) {
        const int cnt = (b + 1 < nbins ? sh[b + 1] : incl) - sh[b];
        nloc += (cnt + p.chunk_tokens - 1) / p.chunk_tokens;
      }
      int cin = nloc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, cin, o);
        if (lane >= o) cin += v;
      }
      int ci = cin - nloc;
      for (int b = b0; b < b1; ++b) {
        const int first = sh[b];
        const int cnt = (b + 1 < nbins ? sh[b + 1] : incl) - first;
        for (int s0 = 0; s0 < cnt; s0 += p.chunk_tokens, ++ci) {
          p.chunks[3 * ci] = b;
          p.chunks[3 * ci + 1] = first + s0;
          p.chunks[3 * ci + 2] = min(p.chunk_tokens, cnt - s0);
        }
      }
      if (lane == 31) *p.nchunks = cin;
    }
  }
  __syncthreads();
  if (threadIdx.x >= 32) return;
  const int lane = threadIdx.x;
  const unsigned lt = (1u << lane) - 1u;
  for (int q0 = 0; q0 < npairs; q0 += 32) {
    const int q = q0 + lane;
    int e = -1;
    if (q < npairs) {
      e = (q < p.T * p.k) ? p.idx[q] : p.E;
      if (e < 0 || e >= p.E + (q < p.T * p.k ? 0 : 1)) e = -1;
    }
    const unsigned same = __match_any_sync(0xffffffffu, e);
    if (e >= 0) {
      const int rank = __popc(same & lt);
      p.perm[sh[e] + rank] = q;
    }
    __syncwarp();
    if (e >= 0 && (same & lt) == 0) sh[e] += __popc(same);
    __syncwarp();
  }
}

}  // namespace

cudaError_t launch_sort_by_expert(const SortParams& p, cudaStream_t stream) {
  const int nbins = p.E + (p.with_shared ? 1 : 0);
  sort_by_expert_kernel<<<1, kThreads, nbins * sizeof(int), stream>>>(p);
  return cudaGetLastError();
}

}  // namespace moe
