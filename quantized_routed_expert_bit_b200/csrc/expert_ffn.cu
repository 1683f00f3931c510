// Kernel (b): the decode-time expert path, for one token at a time.
//
// Phase 1 (gate/up + SwiGLU): for every selected expert and the shared
// expert, the packed [2I][H] gate/up matrix (Runnel README, introduction:
// the routed gate and up projections run as one packed matrix; gate rows
// [0,I), up rows [I,2I)) is walked row pair by row pair:
//   h_i = silu(gate_i . x) * (up_i . x).
// Phase 2 (down + combine): every output row r sums, over the k selected
// experts and the shared expert, w_j * (D_j[r] . h_j), with w for the shared
// expert its sigmoid gate, and rounds once to bf16.
//
// Weights are MLX-style affine groups (Swiftlet article on xix.ai,
// paragraph 8): w = s*q + b per group of `group` elements along K. Codes
// stream with 128-bit loads that skip L1; each CTA's scales and biases are
// staged into shared memory by bulk copies (TMA engine) completing on an
// mbarrier, overlapping the code loads. A group's share of a dot product is
// s * sum(q x) + b * sum(x), with sum(x) over each 16-byte segment computed
// once per CTA; codes become exact fp32 integers in registers without
// int->float conversion (see dot_seg in moe_common.cuh).

#include "moe_common.cuh"
#include "moe_launch.h"

namespace moe {

namespace {

constexpr int kWarps = 8;
constexpr int kRowsPerWarp = 2;
constexpr int kRB = kWarps * kRowsPerWarp;  // rows per CTA (both phases)
constexpr int kChunkGU = 4;                 // 16-byte segments per lane per pass, phase 1
constexpr int kChunkD = 5;                  // same for phase 2

__host__ __device__ constexpr size_t align16(size_t v) { return (v + 15) & ~size_t(15); }

__device__ __forceinline__ float silu_f(float z) { return z / (1.f + expf(-z)); }

// Stage one token's activations v[0..n) (fp32 or bf16 source) into shared
// memory permuted by 16-byte code segment: element (s*PS + 4*q + c) goes to
// dst[(q*nseg + s)*4 + c], so lanes reading consecutive segments read
// consecutive float4s. seg_sum[s] = sum of the segment's PS elements.
template <int PS, typename Load>
__device__ void stage_permuted(float* dst, float* seg_sum, int n, Load load) {
  const int nseg = n / PS;
  for (int i = threadIdx.x; i < n / 4; i += blockDim.x) {
    const int s = (4 * i) / PS, q = ((4 * i) % PS) / 4;
    reinterpret_cast<float4*>(dst)[q * nseg + s] = load(i);
  }
  __syncthreads();
  for (int s = threadIdx.x; s < nseg; s += blockDim.x) {
    float a = 0.f;
#pragma unroll
    for (int q = 0; q < PS / 4; ++q) {
      const float4 f = reinterpret_cast<const float4*>(dst)[q * nseg + s];
      a += (f.x + f.y) + (f.z + f.w);
    }
    seg_sum[s] = a;
  }
}

template <int PS>
__device__ __forceinline__ void load_seg_x(const float* xs, int nseg, int s, float* xv) {
#pragma unroll
  for (int q = 0; q < PS / 4; ++q) {
    const float4 f = reinterpret_cast<const float4*>(xs)[q * nseg + s];
    xv[4 * q + 0] = f.x;
    xv[4 * q + 1] = f.y;
    xv[4 * q + 2] = f.z;
    xv[4 * q + 3] = f.w;
  }
}

// ------------------------------------------------------------------ phase 1

template <int BITS>
__global__ void __launch_bounds__(kWarps * 32)
    gateup_swiglu_kernel(FfnParams p) {
  using CT = CodeTraits<BITS>;
  constexpr int PS = CT::kPerSeg;
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ __align__(8) uint64_t bar;

  const int H = p.H;
  const int nseg = H * BITS / 128;
  const int ng = H / p.group;
  const int blk_r = p.I / kRB;
  const int blk_s = p.Is / kRB;
  const int per_tok = p.k * blk_r + blk_s;
  const int t = blockIdx.x / per_tok;
  const int r = blockIdx.x % per_tok;
  int j, rb, e = 0;
  QMat m;
  if (r < p.k * blk_r) {
    j = r / blk_r;
    rb = r % blk_r;
    m = p.gate_up;
    e = p.idx[static_cast<size_t>(t) * p.k + j];
    if (e < 0 || e >= p.E) {
      if (threadIdx.x == 0 && rb == 0) report(p.ws.hdr, MOE_ERR_BOUNDS, e);
      return;
    }
  } else {
    j = p.k;
    rb = r - p.k * blk_r;
    m = p.sh_gate_up;
    if (rb == 0 && threadIdx.x < 32) {
      // The shared expert's gate, sigmoid(x . w_sg), for phase 2.
      const uint4* xv = reinterpret_cast<const uint4*>(p.x + static_cast<size_t>(t) * p.H);
      const uint4* wv = reinterpret_cast<const uint4*>(p.wsg);
      float a = 0.f;
      for (int s = threadIdx.x; s < p.H / 8; s += 32) {
        const uint4 xa = xv[s], wa = wv[s];
        a = fmaf(bf16_lo(xa.x), bf16_lo(wa.x), a);
        a = fmaf(bf16_hi(xa.x), bf16_hi(wa.x), a);
        a = fmaf(bf16_lo(xa.y), bf16_lo(wa.y), a);
        a = fmaf(bf16_hi(xa.y), bf16_hi(wa.y), a);
        a = fmaf(bf16_lo(xa.z), bf16_lo(wa.z), a);
        a = fmaf(bf16_hi(xa.z), bf16_hi(wa.z), a);
        a = fmaf(bf16_lo(xa.w), bf16_lo(wa.w), a);
        a = fmaf(bf16_hi(xa.w), bf16_hi(wa.w), a);
      }
      a = warp_sum(a);
      if (threadIdx.x == 0) p.ws.sgate[t] = 1.f / (1.f + expf(-a));
    }
  }

  float* xs = reinterpret_cast<float*>(smem);
  float* xsum = xs + H;
  uint16_t* sb = reinterpret_cast<uint16_t*>(smem + align16(static_cast<size_t>(H) * 4 + nseg * 4));
  const int sb_elems = kRB * ng;
  const uint32_t sb_bytes = static_cast<uint32_t>(sb_elems) * 2;
  const int i0 = rb * kRB;
  const uint8_t* qbase = m.q + static_cast<size_t>(e) * m.q_stride;
  const uint16_t* sbase = m.s + static_cast<size_t>(e) * m.sb_stride;
  const uint16_t* bbase = m.b + static_cast<size_t>(e) * m.sb_stride;

  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&bar, 4 * sb_bytes);
    bulk_g2s(sb + 0 * sb_elems, sbase + static_cast<size_t>(i0) * ng, sb_bytes, &bar);
    bulk_g2s(sb + 1 * sb_elems, sbase + m.up_s + static_cast<size_t>(i0) * ng, sb_bytes, &bar);
    bulk_g2s(sb + 2 * sb_elems, bbase + static_cast<size_t>(i0) * ng, sb_bytes, &bar);
    bulk_g2s(sb + 3 * sb_elems, bbase + m.up_b + static_cast<size_t>(i0) * ng, sb_bytes, &bar);
  }

  const uint16_t* xt = p.x + static_cast<size_t>(t) * H;
  stage_permuted<PS>(xs, xsum, H, [&](int i) {
    const uint2 raw = *reinterpret_cast<const uint2*>(xt + 4 * i);
    return make_float4(bf16_lo(raw.x), bf16_hi(raw.x), bf16_lo(raw.y), bf16_hi(raw.y));
  });
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t row_bytes = static_cast<size_t>(H) * BITS / 8;
  float ag[kRowsPerWarp], au[kRowsPerWarp];
#pragma unroll
  for (int rr = 0; rr < kRowsPerWarp; ++rr) ag[rr] = au[rr] = 0.f;
  bool waited = false;
  for (int c0 = 0; c0 < nseg; c0 += 32 * kChunkGU) {
    uint4 cg[kRowsPerWarp][kChunkGU], cu[kRowsPerWarp][kChunkGU];
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
      const int i = i0 + warp * kRowsPerWarp + rr;
      const uint8_t* qg = qbase + static_cast<size_t>(i) * row_bytes;
      const uint8_t* qu = qbase + m.up_q + static_cast<size_t>(i) * row_bytes;
#pragma unroll
      for (int c = 0; c < kChunkGU; ++c) {
        const int s = c0 + 32 * c + lane;
        if (s < nseg) {
          cg[rr][c] = ldg_stream(qg + 16 * static_cast<size_t>(s));
          cu[rr][c] = ldg_stream(qu + 16 * static_cast<size_t>(s));
        }
      }
    }
    if (!waited) {
      if (!mbar_wait(&bar, 0, p.ws.hdr, 1)) return;
      waited = true;
    }
#pragma unroll
    for (int c = 0; c < kChunkGU; ++c) {
      const int s = c0 + 32 * c + lane;
      if (s < nseg) {
        float xv[PS];
        load_seg_x<PS>(xs, nseg, s, xv);
        const float xsm = xsum[s];
        const int g = s * PS / p.group;
#pragma unroll
        for (int rr = 0; rr < kRowsPerWarp; ++rr) {
          const int il = warp * kRowsPerWarp + rr;
          const float sg = bf16_to_f32(sb[0 * sb_elems + il * ng + g]);
          const float su = bf16_to_f32(sb[1 * sb_elems + il * ng + g]);
          const float bg = bf16_to_f32(sb[2 * sb_elems + il * ng + g]);
          const float bu = bf16_to_f32(sb[3 * sb_elems + il * ng + g]);
          ag[rr] = fmaf(sg, dot_seg<BITS>(cg[rr][c], xv), fmaf(bg, xsm, ag[rr]));
          au[rr] = fmaf(su, dot_seg<BITS>(cu[rr][c], xv), fmaf(bu, xsm, au[rr]));
        }
      }
    }
  }
#pragma unroll
  for (int rr = 0; rr < kRowsPerWarp; ++rr) {
    const float g = warp_sum(ag[rr]);
    const float u = warp_sum(au[rr]);
    if (lane == 0) {
      const int i = i0 + warp * kRowsPerWarp + rr;
      p.ws.h[(static_cast<size_t>(t) * (p.k + 1) + j) * p.Imax + i] = silu_f(g) * u;
    }
  }
}

// ------------------------------------------------------------------ phase 2

template <int BITS>
__global__ void __launch_bounds__(kWarps * 32)
    down_combine_kernel(FfnParams p) {
  using CT = CodeTraits<BITS>;
  constexpr int PS = CT::kPerSeg;
  constexpr int kMaxSlots = 17;
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ __align__(8) uint64_t bar;
  __shared__ float wslot[kMaxSlots];
  __shared__ int eslot[kMaxSlots];

  const int nblk = p.H / kRB;
  const int t = blockIdx.x / nblk;
  const int r0 = (blockIdx.x % nblk) * kRB;
  const int nslots = p.k + (p.Is > 0 ? 1 : 0);
  const int Imax = p.Imax;
  const int nseg_r = p.I * BITS / 128, nseg_s = p.Is * BITS / 128;
  const int ng_r = p.I / p.group, ng_s = p.Is / p.group;
  const int nseg_max = Imax * BITS / 128;
  const int ng_max = Imax / p.group;

  float* hs = reinterpret_cast<float*>(smem);                  // [nslots][Imax], permuted
  float* hsum = hs + static_cast<size_t>(nslots) * Imax;       // [nslots][nseg_max]
  uint16_t* sb = reinterpret_cast<uint16_t*>(
      smem + align16((static_cast<size_t>(nslots) * Imax + static_cast<size_t>(nslots) * nseg_max) * 4));
  const int sb_slot = 2 * kRB * ng_max;  // scales then biases of one slot

  if (threadIdx.x == 0) {
    uint32_t bytes = 0;
    int nvalid = 0;
    for (int j = 0; j < nslots; ++j) {
      int e = 0;
      float w;
      if (j < p.k) {
        e = p.idx[static_cast<size_t>(t) * p.k + j];
        w = p.w[static_cast<size_t>(t) * p.k + j];
        if (e < 0 || e >= p.E) {
          if (r0 == 0) report(p.ws.hdr, MOE_ERR_BOUNDS, e);
          e = -1;
          w = 0.f;
        }
      } else {
        w = __ldcg(p.ws.sgate + t);
      }
      eslot[j] = e;
      wslot[j] = w;
      if (e >= 0) {
        ++nvalid;
        bytes += 2u * kRB * (j < p.k ? ng_r : ng_s) * 2u;
      }
    }
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&bar, bytes);
    for (int j = 0; j < nslots; ++j) {
      if (eslot[j] < 0) continue;
      const QMat m = (j < p.k) ? p.down : p.sh_down;
      const int ng = (j < p.k) ? ng_r : ng_s;
      const size_t off = static_cast<size_t>(eslot[j]) * m.sb_stride + static_cast<size_t>(r0) * ng;
      const uint32_t nb = static_cast<uint32_t>(kRB * ng) * 2u;
      bulk_g2s(sb + j * sb_slot, m.s + off, nb, &bar);
      bulk_g2s(sb + j * sb_slot + kRB * ng, m.b + off, nb, &bar);
    }
    (void)nvalid;
  }
  __syncthreads();

  for (int j = 0; j < nslots; ++j) {
    const int Ij = (j < p.k) ? p.I : p.Is;
    const float* hg = p.ws.h + (static_cast<size_t>(t) * (p.k + 1) + (j < p.k ? j : p.k)) * Imax;
    stage_permuted<PS>(hs + static_cast<size_t>(j) * Imax, hsum + static_cast<size_t>(j) * nseg_max, Ij,
                       [&](int i) { return __ldcg(reinterpret_cast<const float4*>(hg) + i); });
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nflat = p.k * nseg_r + (p.Is > 0 ? nseg_s : 0);
  float acc[kRowsPerWarp];
#pragma unroll
  for (int rr = 0; rr < kRowsPerWarp; ++rr) acc[rr] = 0.f;
  bool waited = false;
  for (int f0 = 0; f0 < nflat; f0 += 32 * kChunkD) {
    uint4 cd[kRowsPerWarp][kChunkD];
#pragma unroll
    for (int c = 0; c < kChunkD; ++c) {
      const int f = f0 + 32 * c + lane;
      if (f < nflat) {
        const bool routed = f < p.k * nseg_r;
        const int j = routed ? f / nseg_r : p.k;
        const int s = routed ? f % nseg_r : f - p.k * nseg_r;
        const int e = eslot[j];
        if (e >= 0) {
          const QMat& m = routed ? p.down : p.sh_down;
          const size_t rowb = static_cast<size_t>(routed ? p.I : p.Is) * BITS / 8;
          const uint8_t* qb = m.q + static_cast<size_t>(e) * m.q_stride + 16 * static_cast<size_t>(s);
#pragma unroll
          for (int rr = 0; rr < kRowsPerWarp; ++rr) {
            const int row = r0 + warp * kRowsPerWarp + rr;
            cd[rr][c] = ldg_stream(qb + static_cast<size_t>(row) * rowb);
          }
        }
      }
    }
    if (!waited) {
      if (!mbar_wait(&bar, 0, p.ws.hdr, 2)) return;
      waited = true;
    }
#pragma unroll
    for (int c = 0; c < kChunkD; ++c) {
      const int f = f0 + 32 * c + lane;
      if (f < nflat) {
        const bool routed = f < p.k * nseg_r;
        const int j = routed ? f / nseg_r : p.k;
        const int s = routed ? f % nseg_r : f - p.k * nseg_r;
        if (eslot[j] >= 0) {
          const int nseg = routed ? nseg_r : nseg_s;
          const int ng = routed ? ng_r : ng_s;
          float xv[PS];
          load_seg_x<PS>(hs + static_cast<size_t>(j) * Imax, nseg, s, xv);
          const float hsm = hsum[static_cast<size_t>(j) * nseg_max + s];
          const float wj = wslot[j];
          const int g = s * PS / p.group;
#pragma unroll
          for (int rr = 0; rr < kRowsPerWarp; ++rr) {
            const int il = warp * kRowsPerWarp + rr;
            const float sc = bf16_to_f32(sb[j * sb_slot + il * ng + g]);
            const float bi = bf16_to_f32(sb[j * sb_slot + kRB * ng + il * ng + g]);
            const float part = fmaf(sc, dot_seg<BITS>(cd[rr][c], xv), bi * hsm);
            acc[rr] = fmaf(wj, part, acc[rr]);
          }
        }
      }
    }
  }
  if (!waited) mbar_wait(&bar, 0, p.ws.hdr, 2);  // never leave with copies in flight
#pragma unroll
  for (int rr = 0; rr < kRowsPerWarp; ++rr) {
    const float v = warp_sum(acc[rr]);
    if (lane == 0) p.y[static_cast<size_t>(t) * p.H + r0 + warp * kRowsPerWarp + rr] = f32_to_bf16(v);
  }
}

// ------------------------------------------------------------------ stack glue

// One CTA per token, 256 threads, each thread runs of 8 elements (H <= 8192): every load of the
// token is issued before the first add, then r += y (or r = x), the sum of squares, and x_out.
constexpr int kGlueRuns = 4;  // runs of 8 per thread: 4 * 256 * 8 = 8192 elements
__global__ void __launch_bounds__(256) glue_kernel(GlueParams p) {
  const int t = blockIdx.x;
  float* r = p.r + static_cast<size_t>(t) * p.H;
  const size_t row = static_cast<size_t>(t) * p.H;
  const int n8 = p.H / 8;
  float4 ra[kGlueRuns][2];
  uint4 ya[kGlueRuns];
#pragma unroll
  for (int c = 0; c < kGlueRuns; ++c) {
    const int i8 = threadIdx.x + 256 * c;
    if (i8 < n8) {
      if (p.y) {
        ra[c][0] = *reinterpret_cast<const float4*>(r + 8 * i8);
        ra[c][1] = *reinterpret_cast<const float4*>(r + 8 * i8 + 4);
        ya[c] = *reinterpret_cast<const uint4*>(p.y + row + 8 * i8);
      } else {
        ya[c] = *reinterpret_cast<const uint4*>(p.x_in + row + 8 * i8);
      }
    }
  }
  float ss = 0.f;
#pragma unroll
  for (int c = 0; c < kGlueRuns; ++c) {
    const int i8 = threadIdx.x + 256 * c;
    if (i8 < n8) {
      const uint4 v = ya[c];
      float a[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                    bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
      if (p.y) {
        a[0] += ra[c][0].x;
        a[1] += ra[c][0].y;
        a[2] += ra[c][0].z;
        a[3] += ra[c][0].w;
        a[4] += ra[c][1].x;
        a[5] += ra[c][1].y;
        a[6] += ra[c][1].z;
        a[7] += ra[c][1].w;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) ss = fmaf(a[u], a[u], ss);
      ra[c][0] = make_float4(a[0], a[1], a[2], a[3]);
      ra[c][1] = make_float4(a[4], a[5], a[6], a[7]);
      *reinterpret_cast<float4*>(r + 8 * i8) = ra[c][0];
      *reinterpret_cast<float4*>(r + 8 * i8 + 4) = ra[c][1];
    }
  }
  if (!p.x_out) return;
  __shared__ float red[8];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) tot += red[w];
  const float inv = 1.f / sqrtf(tot / static_cast<float>(p.H) + p.eps);
#pragma unroll
  for (int c = 0; c < kGlueRuns; ++c) {
    const int i8 = threadIdx.x + 256 * c;
    if (i8 < n8) {
      uint4 o;
      o.x = static_cast<uint32_t>(f32_to_bf16(ra[c][0].x * inv)) | (static_cast<uint32_t>(f32_to_bf16(ra[c][0].y * inv)) << 16);
      o.y = static_cast<uint32_t>(f32_to_bf16(ra[c][0].z * inv)) | (static_cast<uint32_t>(f32_to_bf16(ra[c][0].w * inv)) << 16);
      o.z = static_cast<uint32_t>(f32_to_bf16(ra[c][1].x * inv)) | (static_cast<uint32_t>(f32_to_bf16(ra[c][1].y * inv)) << 16);
      o.w = static_cast<uint32_t>(f32_to_bf16(ra[c][1].z * inv)) | (static_cast<uint32_t>(f32_to_bf16(ra[c][1].w * inv)) << 16);
      *reinterpret_cast<uint4*>(p.x_out + row + 8 * i8) = o;
    }
  }
}

template <typename K>
cudaError_t set_smem(K kernel, size_t smem) {
  if (smem <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
}

template <int BITS>
cudaError_t launch_ffn_bits(const FfnParams& p, cudaStream_t stream) {
  constexpr int PS = CodeTraits<BITS>::kPerSeg;
  const int nseg = p.H * BITS / 128;
  const int ng = p.H / p.group;
  const size_t smem1 = align16(static_cast<size_t>(p.H) * 4 + nseg * 4) + 4ull * kRB * ng * 2;
  const int per_tok = p.k * (p.I / kRB) + p.Is / kRB;
  cudaError_t err = set_smem(gateup_swiglu_kernel<BITS>, smem1);
  if (err != cudaSuccess) return err;
  gateup_swiglu_kernel<BITS><<<p.T * per_tok, kWarps * 32, smem1, stream>>>(p);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;

  const int nslots = p.k + (p.Is > 0 ? 1 : 0);
  const size_t nseg_max = static_cast<size_t>(p.Imax) / PS;
  const size_t smem2 = align16((static_cast<size_t>(nslots) * p.Imax + nslots * nseg_max) * 4) +
                       static_cast<size_t>(nslots) * 2 * kRB * (p.Imax / p.group) * 2;
  err = set_smem(down_combine_kernel<BITS>, smem2);
  if (err != cudaSuccess) return err;
  down_combine_kernel<BITS><<<p.T * (p.H / kRB), kWarps * 32, smem2, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_expert_ffn(const FfnParams& p, int bits, cudaStream_t stream) {
  return bits == 4 ? launch_ffn_bits<4>(p, stream) : launch_ffn_bits<8>(p, stream);
}

cudaError_t launch_glue(const GlueParams& p, cudaStream_t stream) {
  glue_kernel<<<p.T, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- group-major down scales

namespace {

// out[((e * ng + g) * rows + r) * 2 + {0, 1}] = (scale, bias) of row r, group g of expert e:
// one thread per (e, g, r), 4 bytes out.
__global__ void prepare_down_sb_kernel(const uint16_t* __restrict__ s, const uint16_t* __restrict__ b, int64_t stride,
                                       int n, int rows, int ng, uint32_t* __restrict__ out) {
  const int64_t total = static_cast<int64_t>(n) * ng * rows;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int r = static_cast<int>(i % rows);
    const int64_t eg = i / rows;
    const int g = static_cast<int>(eg % ng);
    const int64_t e = eg / ng;
    const int64_t src = e * stride + static_cast<int64_t>(r) * ng + g;
    out[i] = static_cast<uint32_t>(s[src]) | (static_cast<uint32_t>(b[src]) << 16);
  }
}

}  // namespace

namespace {

// One thread per 16 bytes of the output: out[((e * nu + u) * rows + r) * ub + b] = q[e][r][u * ub + b].
__global__ void prepare_down_units_kernel(const uint8_t* __restrict__ q, int64_t q_stride, int n, int rows, int rowb,
                                          int ub, uint8_t* __restrict__ out) {
  const int nu = rowb / ub, per = ub / 16;
  const int64_t total = static_cast<int64_t>(n) * nu * rows * per;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int part = static_cast<int>(i % per);
    const int64_t eur = i / per;
    const int r = static_cast<int>(eur % rows);
    const int64_t eu = eur / rows;
    const int u = static_cast<int>(eu % nu);
    const int64_t e = eu / nu;
    const uint4 v = *reinterpret_cast<const uint4*>(q + e * q_stride + static_cast<int64_t>(r) * rowb + u * ub + 16 * part);
    *reinterpret_cast<uint4*>(out + 16 * i) = v;
  }
}

}  // namespace

cudaError_t launch_prepare_down_units(const uint8_t* q, int64_t q_stride, int n, int rows, int rowb, int ub,
                                      uint8_t* out, cudaStream_t stream) {
  const int64_t total = static_cast<int64_t>(n) * rows * (rowb / 16);
  const int64_t blocks = (total + 255) / 256;
  prepare_down_units_kernel<<<static_cast<int>(blocks < 65535 ? blocks : 65535), 256, 0, stream>>>(
      q, q_stride, n, rows, rowb, ub, out);
  return cudaGetLastError();
}

cudaError_t launch_prepare_down_sb(const uint16_t* scales, const uint16_t* biases, int64_t stride, int n, int rows,
                                   int ngroups, uint16_t* out, cudaStream_t stream) {
  const int64_t total = static_cast<int64_t>(n) * ngroups * rows;
  const int64_t blocks = (total + 255) / 256;
  prepare_down_sb_kernel<<<static_cast<int>(blocks < 65535 ? blocks : 65535), 256, 0, stream>>>(
      scales, biases, stride, n, rows, ngroups, reinterpret_cast<uint32_t*>(out));
  return cudaGetLastError();
}

}  // namespace moe
