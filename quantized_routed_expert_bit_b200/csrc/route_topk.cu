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

// ---------------------------------------------------------------- tensor-core router (many tokens)
//
// From kRouteMmaMinTokens tokens the router is a GEMM worth the tensor cores: logits[t][e] =
// x[t] . Wr[e] with mma.sync m16n8k16 (bf16 products exact, fp32 accumulation), CTA tile 16 tokens
// x 64 experts (4 warps, 16 experts each), K in chunks of kMmaK through double-buffered shared
// memory (16-byte cp.async; rows padded to kMmaLd elements so the fragment loads hit 32 distinct
// banks), then softmax + top-k by a second kernel, one warp per token. The logits come out of a
// different summation order than the CUDA-core kernel's, so selections agree with it wherever the
// k-th/(k+1)-th gap is not within the last bits of fp32.

constexpr int kMmaK = 128;          // K per shared-memory chunk
constexpr int kMmaLd = kMmaK + 8;   // row stride of the chunks (elements): 68 words, rows 4 banks apart
constexpr int kMmaTokens = 16;
constexpr int kMmaExperts = 64;

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(128) route_mma_kernel(const __grid_constant__ RouteParams p) {
  __shared__ __align__(16) uint16_t sx[2][kMmaTokens * kMmaLd];
  __shared__ __align__(16) uint16_t sw[2][kMmaExperts * kMmaLd];
  const int t0 = blockIdx.y * kMmaTokens, e0 = blockIdx.x * kMmaExperts;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, q = lane & 3;
  const int nch = (p.H + kMmaK - 1) / kMmaK;
  // one K chunk of the tile's x rows and router rows into buffer b (rows past T or E, and K past H,
  // read as zeros: their products are never stored)
  auto load = [&](int ch, int b) {
    const int k0 = ch * kMmaK;
    for (int i = tid; i < (kMmaTokens + kMmaExperts) * (kMmaK / 8); i += 128) {
      const int row = i / (kMmaK / 8), seg = i % (kMmaK / 8);
      const int k = k0 + seg * 8;
      const bool isx = row < kMmaTokens;
      const int r = isx ? row : row - kMmaTokens;
      uint16_t* dst = isx ? &sx[b][r * kMmaLd + seg * 8] : &sw[b][r * kMmaLd + seg * 8];
      const int grow = isx ? t0 + r : e0 + r;
      const bool ok = k < p.H && grow < (isx ? p.T : p.E);
      if (ok) {
        const uint16_t* src = isx ? p.x + static_cast<size_t>(grow) * p.H + k : p.wr + static_cast<size_t>(grow) * p.H + k;
        cp_async16(dst, src);
      } else {
        *reinterpret_cast<uint4*>(dst) = uint4{};
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  float acc[2][4];
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[j][i] = 0.f;
  load(0, 0);
  for (int ch = 0; ch < nch; ++ch) {
    const int b = ch & 1;
    if (ch + 1 < nch) {
      load(ch + 1, b ^ 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    const uint16_t* xa = sx[b];
    const uint16_t* wb = sw[b] + warp * 16 * kMmaLd;
#pragma unroll
    for (int kk = 0; kk < kMmaK; kk += 16) {
      const uint32_t a0 = *reinterpret_cast<const uint32_t*>(&xa[g * kMmaLd + kk + 2 * q]);
      const uint32_t a1 = *reinterpret_cast<const uint32_t*>(&xa[(g + 8) * kMmaLd + kk + 2 * q]);
      const uint32_t a2 = *reinterpret_cast<const uint32_t*>(&xa[g * kMmaLd + kk + 8 + 2 * q]);
      const uint32_t a3 = *reinterpret_cast<const uint32_t*>(&xa[(g + 8) * kMmaLd + kk + 8 + 2 * q]);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const uint16_t* wr = wb + (j * 8 + g) * kMmaLd + kk + 2 * q;
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(wr);
        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(wr + 8);
        mma_bf16_16816(acc[j], a0, a1, a2, a3, b0, b1);
      }
    }
    __syncthreads();  // the buffer is refilled by the next iteration's load
  }
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int e = e0 + warp * 16 + j * 8 + 2 * q;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int t = t0 + g + 8 * h;
      if (t >= p.T) continue;
#pragma unroll
      for (int c = 0; c < 2; ++c)
        if (e + c < p.E)
          p.ws.logits[static_cast<size_t>(t) * p.E + e + c] = acc[j][2 * h + c] + (p.rbias ? p.rbias[e + c] : 0.f);
    }
  }
}

// Softmax + top-k of every token from the logits, one warp per token.
__global__ void __launch_bounds__(256) topk_kernel(const __grid_constant__ RouteParams p) {
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= p.T) return;
  const int lane = threadIdx.x & 31;
  const size_t tok = static_cast<size_t>(t);
  if (p.E <= 256) topk_token<8>(p.ws.logits + tok * p.E, p.E, p.k, p.renorm, p.idx_out + tok * p.k, p.w_out + tok * p.k,
                                lane);
  else topk_token<16>(p.ws.logits + tok * p.E, p.E, p.k, p.renorm, p.idx_out + tok * p.k, p.w_out + tok * p.k,
                      lane);
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
  if (p.T >= kRouteMmaMinTokens) {  // tensor cores, then top-k
    dim3 grid((p.E + kMmaExperts - 1) / kMmaExperts, (p.T + kMmaTokens - 1) / kMmaTokens);
    route_mma_kernel<<<grid, 128, 0, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    topk_kernel<<<(p.T + 7) / 8, 256, 0, stream>>>(p);
    return cudaGetLastError();
  }
  // 16-token tiles stage 16 rows of x (at most 128 KB); two rows per warp once the FMAs, not the
  // row loads, dominate and there are tiles enough to fill the GPU with half the row blocks
  if (p.T >= 256 && p.H <= 4096) return launch_t<16, 8, 2>(p, stream);
  if (p.T > 8 && p.H <= 4096) return launch_t<16, 8, 1>(p, stream);
  return launch_t<8, 8, 1>(p, stream);
}

}  // namespace moe
