// Grouping step of the batched paths: the T*k (token, slot) pairs of a
// routing decision, grouped by expert in a stable (token, slot) order, with
// the shared expert as pseudo-expert E taken by every token. This is the
// counting sort the grouped expert kernels consume: experts become contiguous
// runs of pairs, so each expert's weights are read once for all of its
// tokens.
//
// One CTA of W warps (W <= 32). Warp w owns the w-th contiguous slice of the
// pairs:
//   1. per-warp histograms in shared memory (shared atomics);
//   2. for every expert, the runs of the warps are laid out in warp order
//      (so the result is stable) after the runs of all smaller experts: a
//      scan over warps per expert, then a block scan over experts;
//   3. every warp scatters its slice in pair order, 32 pairs at a time
//      (match_any ranks equal experts inside a batch, the warp's per-expert
//      cursor carries the order across batches).
// Warp 0 also cuts every expert's run into chunks of <= chunk_tokens pairs
// (the work list of the grouped kernels).
//
// The selection is read through L2 (ld.global.cg): inside the router kernel
// it was written moments earlier by other CTAs.
#pragma once

#include "moe_common.cuh"
#include "moe_launch.h"

namespace moe {

// Shared memory of sort_pairs for a CTA of nwarps warps, in bytes; with cache_idx, also a copy of
// the T*k selected experts (read once, with every load of a thread in flight together).
__host__ __device__ inline size_t sort_pairs_smem(int E, int with_shared, int nwarps, int T = 0, int k = 0,
                                                  bool cache_idx = false) {
  const int nbins = E + (with_shared ? 1 : 0);
  return static_cast<size_t>(nwarps * nbins + nbins + 1 + 32 + (cache_idx ? T * k : 0)) * sizeof(int);
}

// The whole CTA runs it (blockDim.x a multiple of 32, at most 1024); sh holds sort_pairs_smem bytes
// (with the same cache_idx). p is taken by value: its fields stay in registers across the stores.
static __device__ __forceinline__ void sort_pairs(const SortParams p, int* sh, bool cache_idx) {
  const int nw = static_cast<int>(blockDim.x >> 5);
  const int nthr = static_cast<int>(blockDim.x);
  const int nbins = p.E + (p.with_shared ? 1 : 0);
  const int npairs = p.T * p.k + (p.with_shared ? p.T : 0);
  int* cnt = sh;                                // [nw][nbins] counts, then cursors
  int* starts = sh + nw * nbins;                // [nbins + 1] run starts
  int* s_tot = starts + nbins + 1;              // [32] warp totals of the scan
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q0 = static_cast<int>(static_cast<int64_t>(warp) * npairs / nw);
  const int q1 = static_cast<int>(static_cast<int64_t>(warp + 1) * npairs / nw);

  const int ntk = p.T * p.k;
  int* sidx = cache_idx ? s_tot + 32 : nullptr;  // [T*k] copy of the selection
  if (sidx) {
    constexpr int kStage = 8;
    for (int i0 = tid; i0 < ntk; i0 += kStage * nthr) {
      int v[kStage];
#pragma unroll
      for (int j = 0; j < kStage; ++j)
        if (i0 + j * nthr < ntk) v[j] = __ldcg(p.idx + i0 + j * nthr);
#pragma unroll
      for (int j = 0; j < kStage; ++j)
        if (i0 + j * nthr < ntk) sidx[i0 + j * nthr] = v[j];
    }
  }
  auto sel = [&](int q) -> int { return sidx ? sidx[q] : __ldcg(p.idx + q); };

  auto expert_of = [&](int q) -> int {  // -1: out of range (reported)
    const int e = (q < ntk) ? sel(q) : p.E;
    if (e < 0 || e >= nbins || (q < ntk && e >= p.E)) {
      report(p.hdr, MOE_ERR_BOUNDS, e);
      return -1;
    }
    return e;
  };

  for (int i = tid; i < nw * nbins; i += nthr) cnt[i] = 0;
  if (tid < 32) s_tot[tid] = 0;
  __syncthreads();
  // 1. histogram of each warp's slice
  for (int q = q0 + lane; q < q1; q += 32) {
    const int e = expert_of(q);
    if (e >= 0) atomicAdd(&cnt[warp * nbins + e], 1);
  }
  __syncthreads();
  // 2a. per expert: the warps' runs in warp order (cnt becomes the warp's offset inside the
  // expert's run); the expert's total
  for (int e = tid; e < nbins; e += nthr) {
    int run = 0;
    for (int w = 0; w < nw; ++w) {
      const int c = cnt[w * nbins + e];
      cnt[w * nbins + e] = run;
      run += c;
    }
    starts[e] = run;  // total for now
  }
  __syncthreads();
  // 2b. block-wide exclusive scan of the totals over experts (each thread a contiguous block of bins)
  const int per = (nbins + nthr - 1) / nthr;
  const int b0 = min(nbins, tid * per), b1 = min(nbins, b0 + per);
  int my_tot = 0;
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
    const int v = s_tot[lane];  // 0 past the last warp
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
    if (tid == nthr - 1) {
      starts[nbins] = run;
      p.offsets[nbins] = run;
    }
  }
  __syncthreads();
  // 2c. cursors: the run start of the expert plus the warp's offset inside it
  for (int i = tid; i < nw * nbins; i += nthr) cnt[i] += starts[i % nbins];
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
    const int e = (q < q1 && q < ntk) ? sel(q) : -1;
    const int ev = (q < q1) ? ((q < ntk) ? ((e >= 0 && e < p.E) ? e : -1) : p.E) : -1;
    const unsigned same = __match_any_sync(0xffffffffu, ev);
    if (ev >= 0) p.perm[cur[ev] + __popc(same & lt)] = q;
    __syncwarp();
    if (ev >= 0 && (same & lt) == 0) cur[ev] += __popc(same);
    __syncwarp();
  }
}

}  // namespace moe
