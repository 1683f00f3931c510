// Kernel (a): router GEMV fused with softmax and top-k.
//
// Routing as described for the Qwen3-Next / Qwen3.5 MoE models: each token
// goes to k of E experts (8 of 256, 10 of 512: Swiftlet article on xix.ai,
// paragraph 4; Runnel README, "Target"). The weights are the softmax over
// all E logits restricted to the k largest and renormalised to sum to 1
// (or the plain softmax probabilities when renorm = 0).
//
// Grid: (router row blocks) x (token tiles of TT). Each warp computes R
// router rows (experts' logits) for the tile's tokens, which are staged once
// in shared memory (eight 16-byte loads in flight per thread). A warp issues
// all of its rows' 16-byte loads (kLd per row and lane, a whole 2048-wide
// row) before the first multiply, so a row costs one memory round trip; with
// R = 2 every shared-memory read of x feeds two rows. The last CTA to finish
// a token tile (an arrival counter in the workspace, reset by that CTA for
// the next call) runs softmax and top-k, one warp per token (topk_sorted:
// each lane sorts its E/32 keys, k rounds of a warp-wide max; larger logit
// first, equal logits to the lower index).
//
// The grouping of the pairs by expert (sort_by_expert.cu) is a kernel of its
// own: run in the tail of this one, by the CTA that finishes the last tile,
// it measured slower than the separate 32-warp launch from 8 tokens up (one
// CTA's 8 warps walk the whole decision while the rest of the GPU idles), and
// no faster at 2 tokens.

#include <cfloat>
#include <climits>

#include "decode_common.cuh"

namespace moe {

namespace {

constexpr int kLd = 8;  // 16-byte loads in flight per router row and lane (256 segments of 8 bf16)

__device__ __forceinline__ float dot8_bf16(const uint4& w, const uint4& x, float a) {
  a = fmaf(bf16_lo(w.x), bf16_lo(x.x), a);
  a = fmaf(bf16_hi(w.x), bf16_hi(x.x), a);
  a = fmaf(bf16_lo(w.y), bf16_lo(x.y), a);
  a = fmaf(bf16_hi(w.y), bf16_hi(x.y), a);
  a = fmaf(bf16_lo(w.z), bf16_lo(x.z), a);
  a = fmaf(bf16_hi(w.z), bf16_hi(x.z), a);
  a = fmaf(bf16_lo(w.w), bf16_lo(x.w), a);
  a = fmaf(bf16_hi(w.w), bf16_hi(x.w), a);
  return a;
}

// Softmax + top-k of one token (one warp): lane l reads the logits of experts l + 32 i.
template <int PER>
__device__ __forceinline__ void topk_token(const float* lg, int E, int k, int renorm, int32_t* idx_out,
                                           float* w_out, int lane) {
  uint32_t wl[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = lane + 32 * i;
    wl[i] = (e < E) ? __float_as_uint(__ldcg(lg + e)) : 0u;
  }
  unsigned my_k, kmax;
  int my_e;
  topk_sorted<PER>(wl, E, k, lane, my_k, my_e, kmax);
  const float mx = fkey_inv(kmax);
  float z = 0.f;
  if (!renorm) {
#pragma unroll
    for (int i = 0; i < PER; ++i)
      if (lane + 32 * i < E) z += expf(__uint_as_float(wl[i]) - mx);
    z = warp_sum(z);
  }
  const float ex = (lane < k) ? expf(fkey_inv(my_k) - mx) : 0.f;
  const float den = renorm ? warp_sum(ex) : z;
  if (lane < k) {
    idx_out[lane] = my_e;
    w_out[lane] = ex / den;
  }
}

template <int TT, int WPC, int R>
__global__ void __launch_bounds__(WPC * 32) route_topk_kernel(const __grid_constant__ RouteParams p) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint4* sx = reinterpret_cast<uint4*>(smem);  // [tile tokens][H/8] bf16x8
  const int tile = blockIdx.y;
  const int t0 = tile * TT;
  const int nt = min(TT, p.T - t0);
  const int nseg = p.H / 8;
  const uint4* xg = reinterpret_cast<const uint4*>(p.x + static_cast<size_t>(t0) * p.H);
  {
    constexpr int kStage = 8;  // loads in flight per thread while staging the tile
    const int n = nt * nseg;
    for (int i0 = threadIdx.x; i0 < n; i0 += kStage * WPC * 32) {
      uint4 v[kStage];
#pragma unroll
      for (int j = 0; j < kStage; ++j)
        if (i0 + j * WPC * 32 < n) v[j] = __ldg(xg + i0 + j * WPC * 32);
#pragma unroll
      for (int j = 0; j < kStage; ++j)
        if (i0 + j * WPC * 32 < n) sx[i0 + j * WPC * 32] = v[j];
    }
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = (blockIdx.x * WPC + warp) * R;
  if (row0 < p.E) {
    const uint16_t* wrow[R];
#pragma unroll
    for (int r = 0; r < R; ++r) wrow[r] = p.wr + static_cast<size_t>(min(row0 + r, p.E - 1)) * p.H;
    float acc[R][TT];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int t = 0; t < TT; ++t) acc[r][t] = 0.f;
#pragma unroll 1
    for (int base = 0; base < nseg; base += 32 * kLd) {
      uint4 wv[R][kLd];
#pragma unroll
      for (int j = 0; j < kLd; ++j) {
        const int s = base + lane + 32 * j;
#pragma unroll
        for (int r = 0; r < R; ++r) wv[r][j] = (s < nseg) ? ldg_stream(wrow[r] + static_cast<size_t>(s) * 8) : uint4{};
      }
#pragma unroll
      for (int j = 0; j < kLd; ++j) {
        const int s = base + lane + 32 * j;
        if (s < nseg) {
#pragma unroll
          for (int t = 0; t < TT; ++t) {
            if (t < nt) {
              const uint4 xv = sx[t * nseg + s];
#pragma unroll
              for (int r = 0; r < R; ++r) acc[r][t] = dot8_bf16(wv[r][j], xv, acc[r][t]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int row = row0 + r;
      const float bias = (p.rbias && row < p.E) ? p.rbias[row] : 0.f;
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        const float a = warp_sum(acc[r][t]);
        if (lane == 0 && t < nt && row < p.E) p.ws.logits[static_cast<size_t>(t0 + t) * p.E + row] = a + bias;
      }
    }
    __threadfence();  // the logits before this CTA's arrival
  }
  // Arrival: the last CTA of this token tile finishes the routing. Every writer of logits has
  // fenced its stores before the barrier.
  __shared__ int is_last;
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned prev = atomicAdd(&p.ws.counters[tile], 1u);
    is_last = (prev == gridDim.x - 1);
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  for (int t = warp; t < nt; t += WPC) {
    const size_t tok = static_cast<size_t>(t0 + t);
    if (p.E <= 256) topk_token<8>(p.ws.logits + tok * p.E, p.E, p.k, p.renorm, p.idx_out + tok * p.k,
                                  p.w_out + tok * p.k, lane);
    else topk_token<16>(p.ws.logits + tok * p.E, p.E, p.k, p.renorm, p.idx_out + tok * p.k,
                        p.w_out + tok * p.k, lane);
  }
  if (threadIdx.x == 0) p.ws.counters[tile] = 0u;  // ready for the next call
}

template <int TT, int WPC, int R>
cudaError_t launch_t(const RouteParams& p, cudaStream_t stream) {
  constexpr int kRowsPerCta = WPC * R;
  dim3 grid((p.E + kRowsPerCta - 1) / kRowsPerCta, (p.T + TT - 1) / TT);
  const size_t smem = static_cast<size_t>(TT) * p.H * 2;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(route_topk_kernel<TT, WPC, R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  route_topk_kernel<TT, WPC, R><<<grid, WPC * 32, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route_topk(const RouteParams& p, cudaStream_t stream) {
  static_assert(kRouteTokTile == 8, "the arrival counters are sized for 8-token tiles (a superset for 16)");
  // 16-token tiles stage 16 rows of x (at most 128 KB); two rows per warp once the FMAs, not the
  // row loads, dominate and there are tiles enough to fill the GPU with half the row blocks
  if (p.T >= 256 && p.H <= 4096) return launch_t<16, 8, 2>(p, stream);
  if (p.T > 8 && p.H <= 4096) return launch_t<16, 8, 1>(p, stream);
  return launch_t<8, 8, 1>(p, stream);
}

}  // namespace moe
