// Grouping step of the batched path: the T*k (token, slot) pairs of a
// routing decision, grouped by expert in a stable (token, slot) order, with
// the shared expert as pseudo-expert E taken by every token. This is the
// counting sort the grouped expert GEMM consumes: experts become contiguous
// runs of pairs, so each expert's weights are read once for all of its
// tokens.
//
// One CTA of 32 warps. Warp w owns the w-th contiguous slice of the pairs:
//   1. per-warp histograms in shared memory (shared atomics);
//   2. for every expert, the runs of the warps are laid out in warp order
//      (so the result is stable) after the runs of all smaller experts: a
//      scan over warps per expert, then a block scan over experts;
//   3. every warp scatters its slice in pair order, 32 pairs at a time
//      (match_any ranks equal experts inside a batch, the warp's per-expert
//      cursor carries the order across batches).
// Warp 0 also cuts every expert's run into chunks of <= chunk_tokens pairs
// (the GEMM work list).

#include "moe_common.cuh"
#include "moe_launch.h"

namespace moe {

namespace {

constexpr int kThreads = 1024;
constexpr int kSortWarps = kThreads / 32;

__global__ void __launch_bounds__(kThreads) sort_by_expert_kernel(SortParams p) {
  extern __shared__ int sh[];  // [kSortWarps][nbins] counts, then cursors; [nbins + 1] run starts
  const int nbins = p.E + (p.with_shared ? 1 : 0);
  const int npairs = p.T * p.k + (p.with_shared ? p.T : 0);
  int* cnt = sh;
  int* starts = sh + kSortWarps * nbins;
  __shared__ int s_tot[kSortWarps];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q0 = static_cast<int>(static_cast<int64_t>(warp) * npairs / kSortWarps);
  const int q1 = static_cast<int>(static_cast<int64_t>(warp + 1) * npairs / kSortWarps);

  auto expert_of = [&](int q) -> int {  // -1: out of range (reported)
    const int e = (q < p.T * p.k) ? p.idx[q] : p.E;
    if (e < 0 || e >= nbins || (q < p.T * p.k && e >= p.E)) return -1;
    return e;
  };

  for (int i = tid; i < kSortWarps * nbins; i += kThreads) cnt[i] = 0;
  __syncthreads();
  // 1. histogram of each warp's slice
  for (int q = q0 + lane; q < q1; q += 32) {
    const int e = expert_of(q);
    if (e < 0) {
      report(p.hdr, MOE_ERR_BOUNDS, q < p.T * p.k ? p.idx[q] : -1);
      continue;
    }
    atomicAdd(&cnt[warp * nbins + e], 1);
  }
  __syncthreads();
  // 2a. per expert: the warps' runs in warp order (cnt becomes the warp's offset inside the
  // expert's run); the expert's total
  int my_tot = 0;
  for (int e = tid; e < nbins; e += kThreads) {
    int run = 0;
    for (int w = 0; w < kSortWarps; ++w) {
      const int c = cnt[w * nbins + e];
      cnt[w * nbins + e] = run;
      run += c;
    }
    starts[e] = run;  // total for now
  }
  __syncthreads();
  // 2b. block-wide exclusive scan of the totals over experts (each thread a contiguous block of bins)
  const int per = (nbins + kThreads - 1) / kThreads;
  const int b0 = min(nbins, tid * per), b1 = min(nbins, b0 + per);
  for (int b = b0; b < b1; ++b) my_tot += starts[b];
  int incl = my_tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) s_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int v = s_tot[lane];
    int wincl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, wincl, o);
      if (lane >= o) wincl += u;
    }
    s_tot[lane] = wincl - v;  // exclusive prefix of the warps' sums
  }
  __syncthreads();
  {
    int run = s_tot[warp] + incl - my_tot;
    for (int b = b0; b < b1; ++b) {
      const int c = starts[b];
      starts[b] = run;
      p.offsets[b] = run;
      run += c;
    }
    if (tid == kThreads - 1) {
      starts[nbins] = run;
      p.offsets[nbins] = run;
    }
  }
  __syncthreads();
  // 2c. cursors: the run start of the expert plus the warp's offset inside it
  for (int i = tid; i < kSortWarps * nbins; i += kThreads) cnt[i] += starts[i % nbins];
  __syncthreads();
  // chunk list (warp 0): every expert's run cut into chunks of <= chunk_tokens
  if (warp == 0 && p.chunks) {
    const int pb = (nbins + 31) / 32;
    const int e0 = min(nbins, lane * pb), e1 = min(nbins, e0 + pb);
    int nloc = 0;
    for (int b = e0; b < e1; ++b) nloc += (starts[b + 1] - starts[b] + p.chunk_tokens - 1) / p.chunk_tokens;
    int cin = nloc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, cin, o);
      if (lane >= o) cin += v;
    }
    int ci = cin - nloc;
    for (int b = e0; b < e1; ++b) {
      const int first = starts[b];
      const int cnt_b = starts[b + 1] - first;
      for (int s0 = 0; s0 < cnt_b; s0 += p.chunk_tokens, ++ci) {
        p.chunks[3 * ci] = b;
        p.chunks[3 * ci + 1] = first + s0;
        p.chunks[3 * ci + 2] = min(p.chunk_tokens, cnt_b - s0);
      }
    }
    if (lane == 31) *p.nchunks = cin;
  }
  // 3. scatter each warp's slice in order
  const unsigned lt = (1u << lane) - 1u;
  int* cur = cnt + warp * nbins;
  for (int qb = q0; qb < q1; qb += 32) {
    const int q = qb + lane;
    const int e = (q < q1) ? expert_of(q) : -1;
    const unsigned same = __match_any_sync(0xffffffffu, e);
    if (e >= 0) p.perm[cur[e] + __popc(same & lt)] = q;
    __syncwarp();
    if (e >= 0 && (same & lt) == 0) cur[e] += __popc(same);
    __syncwarp();
  }
}

}  // namespace

size_t sort_by_expert_smem(int E, int with_shared) {
  const int nbins = E + (with_shared ? 1 : 0);
  return static_cast<size_t>(kSortWarps * nbins + nbins + 1) * sizeof(int);
}

cudaError_t launch_sort_by_expert(const SortParams& p, cudaStream_t stream) {
  const size_t smem = sort_by_expert_smem(p.E, p.with_shared);
  cudaError_t e = cudaFuncSetAttribute(sort_by_expert_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  sort_by_expert_kernel<<<1, kThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace moe
