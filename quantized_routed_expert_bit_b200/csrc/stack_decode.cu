// Persistent single-token decode of a whole MoE stack in one launch.
//
// One CTA per SM, all co-resident (cooperative launch), walks every layer:
//   1. router rows: each CTA owns E/G rows of the router (plus the shared
//      expert's gate vector as row E), prefetched into shared memory by bulk
//      copies one layer ahead, and writes their logits;
//   2. grid barrier, then every CTA runs softmax + top-k itself (one warp);
//   3. the CTA's share of the selected experts' packed gate/up row pairs
//      (k*I + Is pairs split evenly over the grid) streams through registers
//      with 128-bit loads while one thread issues bulk copies of their scales
//      and biases and of the CTA's down-projection rows of every selected
//      expert (fetched now, used after the next barrier);
//   4. grid barrier on h, then every CTA computes its H/G output rows: the
//      weighted combine of the k routed experts and the gated shared expert;
//   5. grid barrier on y, then every CTA applies the residual and the
//      parameter-free RMSNorm to the full vector itself (identical arithmetic
//      in every CTA), giving the next layer's input without another pass.
// Routing fan-out and shared experts: Swiftlet article (xix.ai), paragraphs
// 4 and 8; Runnel README, "Target". Low-bit groups: same article, paragraph
// 8. Packed gate/up: Runnel README, introduction and "Streaming CLI".
//
// Grid barriers are per-CTA flags in global memory holding a rising epoch:
// a CTA publishes its epoch with a release store after __syncthreads, and
// waits until every flag has reached it. Every wait is bounded (time and
// polls); a CTA that gives up records MOE_ERR_TIMEOUT, and the others see the
// status word and leave too, after draining their own bulk copies.

#include <cfloat>
#include <climits>

#include "moe_common.cuh"
#include "moe_launch.h"

namespace moe {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;

__host__ __device__ constexpr uint32_t al128(uint32_t v) { return (v + 127u) & ~127u; }
__host__ __device__ constexpr int cdiv(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ constexpr int al8(int v) { return (v + 7) & ~7; }

// Shared-memory carve-up; identical on host (sizing) and device.
struct Carve {
  int PS, nseg_x, nslots, Imax, npc_max, ng, nr_max, ng_dmax, rowb_dmax, d_sc_el, rr_max, rowb;
  uint32_t xs, xsum, xn, r, dred, gsb, dbuf, d_slot_bytes, rbuf, total;
};

__host__ __device__ inline Carve carve(int H, int E, int k, int I, int Is, int group, int bits, int G) {
  Carve c{};
  c.PS = 128 / bits;
  c.nseg_x = H / c.PS;
  c.nslots = k + (Is > 0 ? 1 : 0);
  c.Imax = I > Is ? I : Is;
  const int NP = k * I + Is;
  c.npc_max = cdiv(NP, G) + 1;
  c.ng = H / group;
  c.nr_max = cdiv(H, G) + 1;
  c.ng_dmax = c.Imax / group;
  c.rowb_dmax = c.Imax * bits / 8;
  c.d_sc_el = al8(c.nr_max * c.ng_dmax + 16);
  c.rr_max = cdiv(E + (Is > 0 ? 1 : 0), G);
  uint32_t o = 0;
  c.xs = o;    o = al128(o + H * 4);
  c.xsum = o;  o = al128(o + c.nseg_x * 4);
  c.xn = o;    o = al128(o + H * 4);
  c.r = o;     o = al128(o + H * 4);
  c.dred = o;  o = al128(o + c.nslots * c.nr_max * 4);
  c.gsb = o;   o = al128(o + 4 * c.npc_max * c.ng * 2);
  c.d_slot_bytes = al128(c.nr_max * c.rowb_dmax + 2 * c.d_sc_el * 2);
  c.rowb = H * bits / 8;
  // one buffer, used first for this CTA's gate/up code rows ([gate rows][up rows]),
  // then for its down rows of every slot
  const uint32_t gu_bytes = 2u * c.npc_max * c.rowb;
  const uint32_t dn_bytes = c.nslots * c.d_slot_bytes;
  c.dbuf = o;  o = al128(o + (gu_bytes > dn_bytes ? gu_bytes : dn_bytes));
  c.rbuf = o;  o = al128(o + 2 * c.rr_max * H * 2);
  c.total = o;
  return c;
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void copy_tx(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  mbar_expect_tx(bar, bytes);
  bulk_g2s(dst, src, bytes, bar);
}

__device__ __forceinline__ float silu_f(float z) { return z / (1.f + expf(-z)); }

// All CTAs reach `epoch`. Returns false if this CTA must stop (a wait ran
// out here or elsewhere). One counter in global memory: every CTA adds 1
// with release semantics after __syncthreads; thread 0 alone polls it with
// acquire loads and a short sleep, so the barrier puts almost no load on the
// L2 slice that holds it.
__device__ bool grid_barrier(const DecodeParams& p, unsigned epoch, volatile int* s_abort) {
  __syncthreads();
  if (threadIdx.x == 0) {
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(p.flags) : "memory");
    const unsigned target = epoch * gridDim.x;
    bool ok = false;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 0; it < kWaitIters; ++it) {
      unsigned v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p.flags) : "memory");
      if (v >= target) {
        ok = true;
        break;
      }
      __nanosleep(32);
      if ((it & 15u) == 0) {
        const int st = *reinterpret_cast<volatile int*>(&p.hdr->status);
        if (st != 0 || globaltimer_ns() - t0 > kWaitNs) break;
      }
    }
    __threadfence();
    if (!ok) {
      report(p.hdr, MOE_ERR_TIMEOUT, 1000 + static_cast<int>(epoch));
      *s_abort = 1;
    }
  }
  __syncthreads();
  return *s_abort == 0;
}

// Order-preserving map of a float to an unsigned key (larger float, larger key).
__device__ __forceinline__ unsigned fkey(float f) {
  const unsigned u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float fkey_inv(unsigned k) {
  return __uint_as_float((k & 0x80000000u) ? (k ^ 0x80000000u) : ~k);
}

// Softmax + top-k of one token by one warp: larger logit first, equal
// logits to the lower expert index; weights renormalised over the k (or the
// plain softmax probabilities when renorm == 0). Each lane sorts its PER
// logits once (largest first, then lower index); every round one warp-wide
// max over the lanes' heads picks the winner, whose lane pops its head.
template <int PER>
__device__ void topk_warp(const float* lg, int E, int k, int renorm, int* s_idx, float* s_w) {
  const int lane = threadIdx.x & 31;
  unsigned key[PER];
  int idx[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = lane + 32 * i;
    key[i] = (e < E) ? fkey(__ldcg(lg + e)) : 0u;
    idx[i] = e;
  }
  // odd-even transposition sort: key descending, index ascending among equal keys
#pragma unroll
  for (int r = 0; r < PER; ++r) {
#pragma unroll
    for (int i = (r & 1); i + 1 < PER; i += 2) {
      const bool sw = key[i + 1] > key[i] || (key[i + 1] == key[i] && idx[i + 1] < idx[i]);
      const unsigned k0 = key[i], k1 = key[i + 1];
      const int i0 = idx[i], i1 = idx[i + 1];
      key[i] = sw ? k1 : k0;
      key[i + 1] = sw ? k0 : k1;
      idx[i] = sw ? i1 : i0;
      idx[i + 1] = sw ? i0 : i1;
    }
  }
  const float mx = fkey_inv(__reduce_max_sync(0xffffffffu, key[0]));
  float z = 0.f;
  if (!renorm) {
#pragma unroll
    for (int i = 0; i < PER; ++i)
      if (key[i] != 0u) z += expf(fkey_inv(key[i]) - mx);
    z = warp_sum(z);
  }
  unsigned my_k = 0u;
  int my_e = 0;
  for (int j = 0; j < k; ++j) {
    const unsigned wk = __reduce_max_sync(0xffffffffu, key[0]);
    const unsigned we = __reduce_min_sync(0xffffffffu, key[0] == wk ? static_cast<unsigned>(idx[0]) : 0xffffffffu);
    if (lane == j) {
      my_k = wk;
      my_e = static_cast<int>(we);
    }
    if (idx[0] == static_cast<int>(we) && key[0] == wk) {  // pop the head
#pragma unroll
      for (int i = 0; i + 1 < PER; ++i) {
        key[i] = key[i + 1];
        idx[i] = idx[i + 1];
      }
      key[PER - 1] = 0u;
    }
  }
  const float ex = (lane < k) ? expf(fkey_inv(my_k) - mx) : 0.f;
  const float den = renorm ? warp_sum(ex) : z;
  if (lane < k) {
    s_idx[lane] = my_e;
    s_w[lane] = ex / den;
  }
}

// x (bf16 bits, natural order) into the three shared views the layer uses.
template <int PS>
__device__ void set_x(float* xn, float* xs, float* xsum, int H, int i, float v) {
  const int nseg = H / PS;
  xn[i] = v;
  const int s = i / PS, q = (i % PS) / 4, c4 = i % 4;
  xs[(q * nseg + s) * 4 + c4] = v;
}

template <int PS>
__device__ void finish_xsum(const float* xs, float* xsum, int H) {
  const int nseg = H / PS;
  for (int s = threadIdx.x; s < nseg; s += blockDim.x) {
    float a = 0.f;
#pragma unroll
    for (int q = 0; q < PS / 4; ++q) {
      const float4 f = reinterpret_cast<const float4*>(xs)[q * nseg + s];
      a += (f.x + f.y) + (f.z + f.w);
    }
    xsum[s] = a;
  }
}

template <int BITS, int CH, int RB>
__global__ void __launch_bounds__(kThreads, 1) decode_stack_kernel(const __grid_constant__ DecodeParams p) {
  using CT = CodeTraits<BITS>;
  constexpr int PS = CT::kPerSeg;
  extern __shared__ __align__(128) unsigned char sm[];
  __shared__ __align__(8) uint64_t bar_r[2];
  __shared__ __align__(8) uint64_t bar_g, bar_d;
  __shared__ __align__(8) uint64_t bar_gc[3];  // gate/up code rows of pairs [0,16), [16,32), [32,48)
  __shared__ int s_idx[16];
  __shared__ float s_w[16];
  __shared__ float s_sg;
  __shared__ int s_abort;
  __shared__ float s_red[kWarps];
  __shared__ int s_pend[5];  // outstanding copy phases: router[0], router[1], gate/up scales, down rows, gate/up codes

  const int H = p.H, E = p.E, k = p.k, I = p.I, Is = p.Is, group = p.group;
  const int G = gridDim.x, c = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const Carve cv = carve(H, E, k, I, Is, group, BITS, G);
  float* xs = reinterpret_cast<float*>(sm + cv.xs);
  float* xsum = reinterpret_cast<float*>(sm + cv.xsum);
  float* xn = reinterpret_cast<float*>(sm + cv.xn);
  float* rr = reinterpret_cast<float*>(sm + cv.r);
  uint16_t* gsb = reinterpret_cast<uint16_t*>(sm + cv.gsb);
  unsigned char* dbuf = sm + cv.dbuf;
  uint16_t* rbuf = reinterpret_cast<uint16_t*>(sm + cv.rbuf);

  // ---- static assignment of this CTA's work
  const int NP = k * I + Is;
  const int gp0 = static_cast<int>(static_cast<int64_t>(c) * NP / G);
  const int gp1 = static_cast<int>(static_cast<int64_t>(c + 1) * NP / G);
  const int npc = gp1 - gp0;
  const int r0 = static_cast<int>(static_cast<int64_t>(c) * H / G);
  const int r1 = static_cast<int>(static_cast<int64_t>(c + 1) * H / G);
  const int nr = r1 - r0;
  const int nrows_rt = E + (Is > 0 ? 1 : 0);
  const int rr_cnt = (c < nrows_rt) ? cdiv(nrows_rt - c, G) : 0;
  const int nseg_x = cv.nseg_x;
  const int nslots = cv.nslots;
  const size_t rowb = static_cast<size_t>(H) * BITS / 8;

  if (tid == 0) {
    mbar_init(&bar_r[0], 1);
    mbar_init(&bar_r[1], 1);
    mbar_init(&bar_g, 1);
    mbar_init(&bar_d, 1);
    for (int b = 0; b < 3; ++b) mbar_init(&bar_gc[b], 1);
    fence_mbar_init();
    s_abort = 0;
    s_pend[0] = s_pend[1] = s_pend[2] = s_pend[3] = s_pend[4] = -1;
  }
  __syncthreads();

  auto issue_router = [&](int l) {  // thread 0 only
    const LayerDesc& Ld = p.layers[l];
    const int b = l & 1;
    for (int m = 0; m < rr_cnt; ++m) {
      const int row = c + m * G;
      const uint16_t* src = (row < E) ? Ld.wr + static_cast<size_t>(row) * H : Ld.wsg;
      copy_tx(rbuf + (static_cast<size_t>(b) * cv.rr_max + m) * H, src, static_cast<uint32_t>(H) * 2, &bar_r[b]);
    }
    mbar_arrive(&bar_r[b]);
    s_pend[b] = (l >> 1) & 1;
  };
  // Waits out every copy this CTA still has in flight (used before leaving early).
  auto drain = [&]() {
    __syncthreads();
    if (tid == 0) {
      if (s_pend[0] >= 0) mbar_wait(&bar_r[0], s_pend[0], p.hdr, 90);
      if (s_pend[1] >= 0) mbar_wait(&bar_r[1], s_pend[1], p.hdr, 91);
      if (s_pend[2] >= 0) mbar_wait(&bar_g, s_pend[2], p.hdr, 92);
      if (s_pend[3] >= 0) mbar_wait(&bar_d, s_pend[3], p.hdr, 93);
      if (s_pend[4] >= 0)
        for (int b = 0; b < 3; ++b) mbar_wait(&bar_gc[b], s_pend[4], p.hdr, 94);
    }
    __syncthreads();
  };

  if (tid == 0) issue_router(0);

  // ---- layer-0 input and residual
  for (int i = tid; i < H; i += kThreads) {
    const float v = bf16_to_f32(p.x0[i]);
    set_x<PS>(xn, xs, xsum, H, i, v);
    rr[i] = p.r_in ? p.r_in[i] : v;
    if (c == 0 && p.tr_x) p.tr_x[static_cast<size_t>(p.l0) * H + i] = p.x0[i];
  }
  __syncthreads();
  finish_xsum<PS>(xs, xsum, H);
  __syncthreads();

  unsigned epoch = p.epoch0;
  for (int l = 0; l < p.L; ++l) {
    const LayerDesc& Ld = p.layers[l];
    const int lg = p.l0 + l;  // layer index within the whole stack (trace rows)
    auto stamp = [&](int slot) {
      if (p.tr_t && c == 0 && tid == 0) p.tr_t[static_cast<size_t>(lg) * 8 + slot] = globaltimer_ns();
    };
    stamp(0);
    if (tid == 0 && l + 1 < p.L) issue_router(l + 1);

    // ---------------- 1. router rows
    if (!mbar_wait(&bar_r[l & 1], (l >> 1) & 1, p.hdr, 10)) { s_abort = 1; }
    if (tid == 0) s_pend[l & 1] = -1;
    if (warp < rr_cnt) {
      const int row = c + warp * G;
      const uint4* wv = reinterpret_cast<const uint4*>(rbuf + (static_cast<size_t>(l & 1) * cv.rr_max + warp) * H);
      float acc = 0.f;
      for (int s = lane; s < H / 8; s += 32) {
        const uint4 w8 = wv[s];
        const float4 a = reinterpret_cast<const float4*>(xn)[2 * s];
        const float4 b = reinterpret_cast<const float4*>(xn)[2 * s + 1];
        acc = fmaf(bf16_lo(w8.x), a.x, acc);
        acc = fmaf(bf16_hi(w8.x), a.y, acc);
        acc = fmaf(bf16_lo(w8.y), a.z, acc);
        acc = fmaf(bf16_hi(w8.y), a.w, acc);
        acc = fmaf(bf16_lo(w8.z), b.x, acc);
        acc = fmaf(bf16_hi(w8.z), b.y, acc);
        acc = fmaf(bf16_lo(w8.w), b.z, acc);
        acc = fmaf(bf16_hi(w8.w), b.w, acc);
      }
      acc = warp_sum(acc);
      if (lane == 0) p.logits[row] = acc + ((row < E && Ld.rbias) ? Ld.rbias[row] : 0.f);
    }
    stamp(1);
    if (!grid_barrier(p, ++epoch, &s_abort)) { drain(); return; }
    stamp(2);

    // ---------------- 2. softmax + top-k (every CTA)
    if (warp == 0) {
      if (E <= 256) topk_warp<8>(p.logits, E, k, p.renorm, s_idx, s_w);
      else topk_warp<16>(p.logits, E, k, p.renorm, s_idx, s_w);
      if (lane == 0) s_sg = (Is > 0) ? 1.f / (1.f + expf(-__ldcg(p.logits + E))) : 0.f;
      __syncwarp();
      if (c == 0 && lane < k) {
        if (p.tr_idx) p.tr_idx[static_cast<size_t>(lg) * k + lane] = s_idx[lane];
        if (p.tr_w) p.tr_w[static_cast<size_t>(lg) * k + lane] = s_w[lane];
      }
    }
    __syncthreads();
    stamp(3);

    // ---------------- 3. bulk copies: gate/up scales+biases of this CTA's pairs, down rows
    // (issued by the 32 lanes of warp 0 in parallel; lane 0 arrives once all are armed)
    if (warp == 0) {
      const int ng = cv.ng;
      // gate/up scale and bias rows: the CTA's pairs fall in at most 3 slots
      int P = gp0, seg = 0;
      while (P < gp1) {
        const bool routed = P < k * I;
        const int j = routed ? P / I : k;
        const int sstart = routed ? j * I : k * I;
        const int send = routed ? (j + 1) * I : k * I + Is;
        const int n = min(gp1, send) - P;
        if (lane >= 4 * seg && lane < 4 * seg + 4) {
          const int which = lane - 4 * seg;  // 0 gate scales, 1 up scales, 2 gate biases, 3 up biases
          const int i0 = P - sstart;
          const int q0 = P - gp0;
          const QMat m = routed ? Ld.gu : Ld.sgu;
          const int Ij = routed ? I : Is;
          const size_t eoff = static_cast<size_t>(routed ? s_idx[j] : 0) * m.sb_stride;
          const uint16_t* src = ((which & 2) ? m.b : m.s) + eoff + static_cast<size_t>((which & 1) ? Ij + i0 : i0) * ng;
          copy_tx(gsb + (which * cv.npc_max + q0) * ng, src, static_cast<uint32_t>(n * ng) * 2u, &bar_g);
        }
        P += n;
        ++seg;
      }
      // gate/up code rows of this CTA's pairs, in batches of 16 pairs (one
      // mbarrier each): per batch and slot segment one copy of gate rows, one of up rows
      {
        int c2 = 0;
        for (int b = 0; b < 3; ++b) {
          const int q_lo = 16 * b, q_hi = min(npc, 16 * b + 16);
          int P2 = gp0 + q_lo;
          while (P2 < gp0 + q_hi) {
            const bool routed = P2 < k * I;
            const int j = routed ? P2 / I : k;
            const int sstart = routed ? j * I : k * I;
            const int send = routed ? (j + 1) * I : k * I + Is;
            const int n = min(gp0 + q_hi, send) - P2;
            const int qq = P2 - gp0;
            for (int gu = 0; gu < 2; ++gu, ++c2) {
              if (lane == 16 + (c2 & 15)) {
                const QMat m = routed ? Ld.gu : Ld.sgu;
                const int Ij = routed ? I : Is;
                const uint8_t* src = m.q + static_cast<size_t>(routed ? s_idx[j] : 0) * m.q_stride +
                                     static_cast<size_t>(gu * Ij + (P2 - sstart)) * rowb;
                copy_tx(dbuf + (static_cast<size_t>(gu) * cv.npc_max + qq) * rowb, src,
                        static_cast<uint32_t>(n * rowb), &bar_gc[b]);
              }
            }
            P2 += n;
          }
        }
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bar_g);
        for (int b = 0; b < 3; ++b) mbar_arrive(&bar_gc[b]);
        s_pend[2] = l & 1;
        s_pend[4] = l & 1;
      }
      __syncwarp();
    }

    // ---------------- 4. gate/up + SwiGLU of this CTA's row pairs
    {
      const int ng = cv.ng;
      bool waited = false;
      for (int m0 = warp; m0 < npc; m0 += kWarps * RB) {
        uint4 cg[RB][CH], cu[RB][CH];
        int qv[RB];
        if (!waited) {
          if (!mbar_wait(&bar_g, l & 1, p.hdr, 11)) s_abort = 1;
          waited = true;
        }
#pragma unroll
        for (int b = 0; b < RB; ++b) {
          const int q = m0 + b * kWarps;
          qv[b] = q;
          if (q < npc) {
            if (!mbar_wait(&bar_gc[q >> 4], l & 1, p.hdr, 14)) s_abort = 1;
            const unsigned char* qg = dbuf + static_cast<size_t>(q) * rowb;
            const unsigned char* qu = dbuf + (static_cast<size_t>(cv.npc_max) + q) * rowb;
#pragma unroll
            for (int ch = 0; ch < CH; ++ch) {
              const int s = lane + 32 * ch;
              if (s < nseg_x) {
                cg[b][ch] = *reinterpret_cast<const uint4*>(qg + 16 * s);
                cu[b][ch] = *reinterpret_cast<const uint4*>(qu + 16 * s);
              }
            }
          }
        }
        float ag[RB], au[RB];
#pragma unroll
        for (int b = 0; b < RB; ++b) ag[b] = au[b] = 0.f;
#pragma unroll
        for (int ch = 0; ch < CH; ++ch) {
          const int s = lane + 32 * ch;
          if (s < nseg_x) {
            float xv[PS];
#pragma unroll
            for (int q4 = 0; q4 < PS / 4; ++q4) {
              const float4 f = reinterpret_cast<const float4*>(xs)[q4 * nseg_x + s];
              xv[4 * q4] = f.x;
              xv[4 * q4 + 1] = f.y;
              xv[4 * q4 + 2] = f.z;
              xv[4 * q4 + 3] = f.w;
            }
            const float xsm = xsum[s];
            const int g = s * PS / group;
#pragma unroll
            for (int b = 0; b < RB; ++b) {
              if (qv[b] < npc) {
                const int q = qv[b];
                const float sg = bf16_to_f32(gsb[(0 * cv.npc_max + q) * ng + g]);
                const float su = bf16_to_f32(gsb[(1 * cv.npc_max + q) * ng + g]);
                const float bg = bf16_to_f32(gsb[(2 * cv.npc_max + q) * ng + g]);
                const float bu = bf16_to_f32(gsb[(3 * cv.npc_max + q) * ng + g]);
                ag[b] = fmaf(sg, dot_seg<BITS>(cg[b][ch], xv), fmaf(bg, xsm, ag[b]));
                au[b] = fmaf(su, dot_seg<BITS>(cu[b][ch], xv), fmaf(bu, xsm, au[b]));
              }
            }
          }
        }
#pragma unroll
        for (int b = 0; b < RB; ++b) {
          const float gsum = warp_sum(ag[b]);
          const float usum = warp_sum(au[b]);
          if (lane == 0 && qv[b] < npc) {
            const int P = gp0 + qv[b];
            const bool routed = P < k * I;
            const int j = routed ? P / I : k;
            const int i = routed ? P - j * I : P - k * I;
            __stcg(p.hbuf + static_cast<size_t>(j) * cv.Imax + i, silu_f(gsum) * usum);
          }
        }
      }
      if (!waited && npc > 0 && warp == 0) {
        if (!mbar_wait(&bar_g, l & 1, p.hdr, 12)) s_abort = 1;
      }
    }
    __syncthreads();
    if (tid == 0) {
      s_pend[2] = -1;
      s_pend[4] = -1;
    }
    // down rows of every slot into the same buffer (codes, scales, biases: 3 copies
    // per slot, by warp 0's lanes); they travel while the grid waits on h
    if (warp == 0) {
      for (int c3 = lane; c3 < 3 * nslots && nr > 0; c3 += 32) {
        const int j = c3 / 3, which = c3 % 3;
        const bool routed = j < k;
        const QMat m = routed ? Ld.dn : Ld.sdn;
        const int Ij = routed ? I : Is;
        const int ngd = Ij / group;
        const size_t rowbd = static_cast<size_t>(Ij) * BITS / 8;
        const int e = routed ? s_idx[j] : 0;
        unsigned char* slot = dbuf + static_cast<size_t>(j) * cv.d_slot_bytes;
        if (which == 0) {
          copy_tx(slot, m.q + static_cast<size_t>(e) * m.q_stride + static_cast<size_t>(r0) * rowbd,
                  static_cast<uint32_t>(nr * rowbd), &bar_d);
        } else {
          const int el0 = (r0 * ngd) & ~7;
          const int el1 = al8(r1 * ngd);
          uint16_t* sc = reinterpret_cast<uint16_t*>(slot + static_cast<size_t>(cv.nr_max) * cv.rowb_dmax);
          const size_t eo = static_cast<size_t>(e) * m.sb_stride + el0;
          copy_tx(sc + (which == 2 ? cv.d_sc_el : 0), (which == 2 ? m.b : m.s) + eo,
                  static_cast<uint32_t>(el1 - el0) * 2u, &bar_d);
        }
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bar_d);
        s_pend[3] = l & 1;
      }
    }
    stamp(4);
    if (!grid_barrier(p, ++epoch, &s_abort)) { drain(); return; }
    stamp(5);

    // ---------------- 5+6. down rows + weighted combine + shared expert
    // Warp w owns slots w, w+16: its lanes keep one 16-byte code segment's
    // worth of that slot's h (read once from L2) and walk the CTA's rows; the
    // per-slot row sums meet in shared memory and are combined in slot order.
    if (!mbar_wait(&bar_d, l & 1, p.hdr, 13)) s_abort = 1;
    if (tid == 0) s_pend[3] = -1;
    const bool last_layer_out = p.layer_mode && (l == p.L - 1);
    {
      float* dred = reinterpret_cast<float*>(sm + cv.dred);  // [nslots][nr_max]
      for (int j = warp; j < nslots; j += kWarps) {
        const bool routed = j < k;
        const int Ij = routed ? I : Is;
        const int nsg = Ij / PS;                   // code segments per row (16 or 32 at I = 512)
        const int rows_per_step = 32 / nsg;        // 2 rows at a time for 16 segments
        const int s = lane % nsg;
        const int sub = lane / nsg;                // which of the rows of this step
        const int ngd = Ij / group;
        const int rowbd = Ij * BITS / 8;
        const float* hg = p.hbuf + static_cast<size_t>(j) * cv.Imax + s * PS;
        float hv[PS];
        float hsm = 0.f;
#pragma unroll
        for (int q4 = 0; q4 < PS / 4; ++q4) {
          const float4 f = __ldcg(reinterpret_cast<const float4*>(hg) + q4);
          hv[4 * q4] = f.x;
          hv[4 * q4 + 1] = f.y;
          hv[4 * q4 + 2] = f.z;
          hv[4 * q4 + 3] = f.w;
          hsm += (f.x + f.y) + (f.z + f.w);
        }
        const unsigned char* slot = dbuf + static_cast<size_t>(j) * cv.d_slot_bytes;
        const uint16_t* sc = reinterpret_cast<const uint16_t*>(slot + static_cast<size_t>(cv.nr_max) * cv.rowb_dmax);
        const int off = r0 * ngd - ((r0 * ngd) & ~7);
        const int g = s * PS / group;
        for (int rl0 = 0; rl0 < nr; rl0 += rows_per_step) {
          const int rl = rl0 + sub;
          float part = 0.f;
          if (rl < nr) {
            const uint4 cd = *reinterpret_cast<const uint4*>(slot + static_cast<size_t>(rl) * rowbd + 16 * s);
            const int ei = off + rl * ngd + g;
            part = fmaf(bf16_to_f32(sc[ei]), dot_seg<BITS>(cd, hv), bf16_to_f32(sc[cv.d_sc_el + ei]) * hsm);
          }
          // sum over the nsg lanes of each row
          for (int o = nsg >> 1; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
          if (s == 0 && rl < nr) dred[j * cv.nr_max + rl] = part;
        }
      }
      __syncthreads();
      if (tid < nr) {
        const int row = r0 + tid;
        float acc = 0.f;
        for (int j = 0; j < k; ++j) acc = fmaf(s_w[j], dred[j * cv.nr_max + tid], acc);
        if (Is > 0) acc = fmaf(s_sg, dred[k * cv.nr_max + tid], acc);
        const uint16_t yb = f32_to_bf16(acc);
        if (last_layer_out) {
          p.out[row] = yb;
        } else {
          p.ybuf[row] = yb;
        }
        if (p.tr_y) p.tr_y[static_cast<size_t>(lg) * H + row] = yb;
      }
    }
    stamp(6);
    if (last_layer_out) break;
    if (!grid_barrier(p, ++epoch, &s_abort)) { drain(); return; }
    stamp(7);

    // ---------------- 7. residual + RMSNorm of the whole vector (every CTA)
    float ss = 0.f;
    for (int i = tid; i < H; i += kThreads) {
      const float v = rr[i] + bf16_to_f32(__ldcg(p.ybuf + i));
      rr[i] = v;
      ss = fmaf(v, v, ss);
    }
    ss = warp_sum(ss);
    if (lane == 0) s_red[warp] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) tot += s_red[w];
    const float inv = 1.f / sqrtf(tot / static_cast<float>(H) + p.eps);
    const bool final_x = (l == p.L - 1);
    for (int i = tid; i < H; i += kThreads) {
      const uint16_t xb = f32_to_bf16(rr[i] * inv);
      set_x<PS>(xn, xs, xsum, H, i, bf16_to_f32(xb));
      if (c == 0) {
        if (final_x) p.out[i] = xb;
        else if (p.tr_x) p.tr_x[static_cast<size_t>(lg + 1) * H + i] = xb;
        if (final_x && p.r_out) p.r_out[i] = rr[i];
      }
    }
    __syncthreads();
    finish_xsum<PS>(xs, xsum, H);
    __syncthreads();
  }
  drain();
}

template <int BITS, int CH, int RB>
cudaError_t launch_t(const DecodeParams& p, size_t smem, int grid, cudaStream_t stream) {
  auto kern = decode_stack_kernel<BITS, CH, RB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorCooperativeLaunchTooLarge;
  void* args[] = {const_cast<DecodeParams*>(&p)};
  return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(kern), dim3(grid), dim3(kThreads), args, smem,
                                     stream);
}

}  // namespace

size_t decode_stack_smem(int H, int E, int k, int I, int Is, int group, int bits, int grid) {
  // the gate/up code rows of a CTA are staged in three batches of 16 pairs
  if (cdiv(k * I + Is, grid) > 48) return ~size_t(0);
  return carve(H, E, k, I, Is, group, bits, grid).total;
}

bool decode_stack_supported(int H, int E, int k, int I, int Is, int group, int bits) {
  const int nseg = H * bits / 128;
  if (nseg > 128) return false;          // at most 4 code segments per lane per row
  if ((H / group) % 8 != 0) return false;  // gate/up scale rows are whole 16-byte chunks
  if (k > 16 || E > 512) return false;
  (void)I;
  (void)Is;
  return true;
}

cudaError_t launch_decode_stack(const DecodeParams& p, int bits, int grid, cudaStream_t stream) {
  const size_t smem = decode_stack_smem(p.H, p.E, p.k, p.I, p.Is, p.group, bits, grid);
  const int nseg = p.H * bits / 128;
  if (bits == 4) {
    if (nseg <= 32) return launch_t<4, 1, 3>(p, smem, grid, stream);
    if (nseg <= 64) return launch_t<4, 2, 3>(p, smem, grid, stream);
    return launch_t<4, 4, 2>(p, smem, grid, stream);
  }
  if (nseg <= 32) return launch_t<8, 1, 3>(p, smem, grid, stream);
  if (nseg <= 64) return launch_t<8, 2, 3>(p, smem, grid, stream);
  return launch_t<8, 4, 2>(p, smem, grid, stream);
}

}  // namespace moe
