// Kernel (a): router GEMV fused with softmax and warp-shuffle top-k.
//
// Routing as described for the Qwen3-Next / Qwen3.5 MoE models: each token
// goes to k of E experts (8 of 256, 10 of 512: Swiftlet article on xix.ai,
// paragraph 4; Runnel README, "Target"). The weights are the softmax over
// all E logits restricted to the k largest and renormalised to sum to 1
// (or the plain softmax probabilities when renorm = 0).
//
// One warp computes one router row (one expert's logit) for a tile of up to
// TT tokens (8 tokens and 4 warps a CTA for small batches; 16 tokens and 32
// warps from 16 tokens up, so a token tile is read by fewer CTAs). The
// tile's tokens are staged once in shared memory; router rows stream through
// with 128-bit loads. The last CTA to finish a token tile (an arrival counter in
// the workspace, reset by that CTA for the next call) then runs softmax and
// top-k: one warp per token, each lane holding E/32 logits, k rounds of a
// shuffle arg-max (larger logit wins, equal logits go to the lower index).

#include <cfloat>
#include <climits>

#include "moe_common.cuh"
#include "moe_launch.h"

namespace moe {

namespace {

constexpr int kMaxPerLane = 16;  // E <= 512

__device__ void topk_one_token(const float* lg, int E, int k, int renorm, int32_t* idx_out,
                               float* w_out) {
  const int lane = threadIdx.x & 31;
  float v[kMaxPerLane];
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i) {
    const int e = lane + 32 * i;
    v[i] = (e < E) ? __ldcg(lg + e) : -FLT_MAX;
  }
  float mx = -FLT_MAX;
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i) mx = fmaxf(mx, v[i]);
  mx = warp_max(mx);
  float z = 0.f;
  if (!renorm) {
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i)
      if (lane + 32 * i < E) z += expf(v[i] - mx);
    z = warp_sum(z);
  }
  float sel_v = 0.f;
  int sel_e = 0;
  for (int j = 0; j < k; ++j) {
    float bv = -FLT_MAX;
    int be = INT_MAX;
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
      const int e = lane + 32 * i;
      if (e < E && v[i] > bv) {  // strict: the lowest index of equal values in this lane
        bv = v[i];
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i)
      if (lane + 32 * i == be) v[i] = -FLT_MAX;  // taken
    if (lane == j) {
      sel_v = bv;
      sel_e = be;
    }
  }
  // sel_v of lane 0 is the largest logit overall, which equals mx.
  const float ex = (lane < k) ? expf(sel_v - mx) : 0.f;
  const float denom = renorm ? warp_sum(ex) : z;
  if (lane < k) {
    idx_out[lane] = sel_e;
    w_out[lane] = ex / denom;
  }
}

template <int TT, int WPC>
__global__ void __launch_bounds__(WPC * 32)
    route_topk_kernel(RouteParams p) {
  extern __shared__ uint4 sx[];  // [tile tokens][H/8] bf16x8
  const int tile = blockIdx.y;
  const int t0 = tile * TT;
  const int nt = min(TT, p.T - t0);
  const int nseg = p.H / 8;
  const uint4* xg = reinterpret_cast<const uint4*>(p.x + static_cast<size_t>(t0) * p.H);
  for (int i = threadIdx.x; i < nt * nseg; i += blockDim.x) sx[i] = xg[i];
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * WPC + warp;
  if (row < p.E) {
    const uint16_t* wrow = p.wr + static_cast<size_t>(row) * p.H;
    float acc[TT];
#pragma unroll
    for (int t = 0; t < TT; ++t) acc[t] = 0.f;
    for (int s = lane; s < nseg; s += 32) {
      const uint4 wv = ldg_stream(wrow + static_cast<size_t>(s) * 8);
      const float w8[8] = {bf16_lo(wv.x), bf16_hi(wv.x), bf16_lo(wv.y), bf16_hi(wv.y),
                           bf16_lo(wv.z), bf16_hi(wv.z), bf16_lo(wv.w), bf16_hi(wv.w)};
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        if (t < nt) {
          const uint4 xv = sx[t * nseg + s];
          float a = acc[t];
          a = fmaf(w8[0], bf16_lo(xv.x), a);
          a = fmaf(w8[1], bf16_hi(xv.x), a);
          a = fmaf(w8[2], bf16_lo(xv.y), a);
          a = fmaf(w8[3], bf16_hi(xv.y), a);
          a = fmaf(w8[4], bf16_lo(xv.z), a);
          a = fmaf(w8[5], bf16_hi(xv.z), a);
          a = fmaf(w8[6], bf16_lo(xv.w), a);
          a = fmaf(w8[7], bf16_hi(xv.w), a);
          acc[t] = a;
        }
      }
    }
    const float bias = p.rbias ? p.rbias[row] : 0.f;
#pragma unroll
    for (int t = 0; t < TT; ++t) {
      const float a = warp_sum(acc[t]);
      if (lane == 0 && t < nt) p.ws.logits[static_cast<size_t>(t0 + t) * p.E + row] = a + bias;
    }
    if (lane == 0) __threadfence();
  }

  // Arrival: the last CTA of this token tile finishes the routing.
  __shared__ int is_last;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned prev = atomicAdd(&p.ws.counters[tile], 1u);
    is_last = (prev == gridDim.x - 1);
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  for (int t = warp; t < nt; t += WPC) {
    const size_t tok = static_cast<size_t>(t0 + t);
    const float* lg = p.ws.logits + tok * p.E;
    topk_one_token(lg, p.E, p.k, p.renorm, p.idx_out + tok * p.k, p.w_out + tok * p.k);
  }
  if (threadIdx.x == 0) p.ws.counters[tile] = 0u;  // ready for the next call
}

template <int TT, int WPC>
cudaError_t launch_t(const RouteParams& p, cudaStream_t stream) {
  dim3 grid((p.E + WPC - 1) / WPC, (p.T + TT - 1) / TT);
  const size_t smem = static_cast<size_t>(TT) * p.H * 2;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(route_topk_kernel<TT, WPC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  route_topk_kernel<TT, WPC><<<grid, WPC * 32, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route_topk(const RouteParams& p, cudaStream_t stream) {
  static_assert(kRouteTokTile == 8, "the arrival counters are sized for 8-token tiles (a superset for 16)");
  if (p.T >= 16) return launch_t<16, 32>(p, stream);
  return launch_t<8, 4>(p, stream);
}

}  // namespace moe
