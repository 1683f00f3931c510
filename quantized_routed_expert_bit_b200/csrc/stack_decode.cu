// Persistent single-token decode of a whole MoE stack in one launch.
//
// One CTA per SM, all co-resident (cooperative launch), walks every layer:
//   1. residual + parameter-free RMSNorm of the previous layer's output
//      (every CTA redundantly, identical arithmetic), giving this layer's x;
//   2. router rows: each CTA owns E/G rows of the router (plus the shared
//      expert's gate vector as row E), prefetched into shared memory by bulk
//      copies one layer ahead, and publishes their logits;
//   3. softmax + top-k in every CTA from all published logits (one warp);
//   4. the CTA's share of the selected experts' packed gate/up row pairs
//      (k*I + Is pairs split evenly over the grid) lands in shared memory by
//      bulk copies in batches of 8 pairs; the dot products dequantize in
//      registers; SwiGLU of each pair is published as h;
//   5. every CTA computes its H/G output rows from all published h: the
//      weighted combine of the k routed down projections and the gated shared
//      expert, and publishes them as y.
// Routing fan-out and shared experts: Swiftlet article (xix.ai), paragraphs
// 4 and 8; Runnel README, "Target". Low-bit groups: same article, paragraph
// 8. Packed gate/up: Runnel README, introduction and "Streaming CLI".
//
// Exchanges between CTAs carry their own layer tag, so no grid barrier and no
// memory fence is needed: every exchanged value is one 32-bit word written
// once per layer with a relaxed store, and a reader polls the words
// themselves until every one carries the current layer's tag.
//  - logits and h are fp32 whose least significant mantissa bit is replaced
//    by the layer parity (a change of at most one unit in the last place);
//  - y is a bf16 in the high half with a 16-bit layer tag in the low half.
// One bit of parity is enough for logits and h: every word is rewritten in
// every layer, a writer of layer l+1 has necessarily seen all of layer l's
// exchanges (so every reader of layer l is done with it), and the host
// zeroes the exchange words before each launch (layer tags start at 1).
// Every poll and every mbarrier wait is bounded (time and polls); a CTA that
// gives up records MOE_ERR_TIMEOUT, the others see the status word and leave
// too, each after draining its own bulk copies.

#include <cfloat>
#include <climits>

#include "moe_common.cuh"
#include "moe_launch.h"

namespace moe {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBatch = 8;        // gate/up pairs per code batch (one mbarrier each)
constexpr int kMaxBatches = 8;   // at most 64 pairs per CTA
constexpr int kHChunks = 4;      // 16-byte chunks of h each thread reads: (k+1)*I <= 4*4*512
constexpr int kTopPer = 16;      // logits per lane in the top-k warp: E <= 512

__host__ __device__ constexpr uint32_t al128(uint32_t v) { return (v + 127u) & ~127u; }
__host__ __device__ constexpr int cdiv(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ constexpr int al8(int v) { return (v + 7) & ~7; }

// Shared-memory carve-up; identical on host (sizing) and device.
struct Carve {
  int PS, nsg, nsgd, nslots, npc_max, ng, nr_max, ngd, rowb, rowbd, d_sc_el, rr_max;
  uint32_t xs, xn, rr, hs, dred, guv, gsb, dbuf, d_slot_bytes, rbuf, total;
};

__host__ __device__ inline Carve carve(int H, int E, int k, int I, int Is, int group, int bits, int G) {
  Carve c{};
  c.PS = 128 / bits;
  c.nsg = H / c.PS;
  c.nsgd = I / c.PS;
  c.nslots = k + (Is > 0 ? 1 : 0);
  c.npc_max = cdiv(k * I + Is, G) + 1;
  c.ng = H / group;
  c.nr_max = cdiv(H, G) + 1;
  c.ngd = I / group;
  c.rowb = H * bits / 8;
  c.rowbd = I * bits / 8;
  c.d_sc_el = al8(c.nr_max * c.ngd + 16);
  c.rr_max = cdiv(E + (Is > 0 ? 1 : 0), G);
  uint32_t o = 0;
  c.xs = o;    o = al128(o + H * 4);
  c.xn = o;    o = al128(o + H * 4);
  c.rr = o;    o = al128(o + H * 4);
  c.hs = o;    o = al128(o + c.nslots * I * 4);
  c.dred = o;  o = al128(o + c.nslots * c.nr_max * 4);
  c.guv = o;   o = al128(o + 2 * c.npc_max * 4);
  c.gsb = o;   o = al128(o + 4 * c.npc_max * c.ng * 2);
  c.d_slot_bytes = al128(c.nr_max * c.rowbd + 2 * c.d_sc_el * 2);
  // one buffer, used first for this CTA's gate/up code rows ([gate rows][up rows]),
  // then for its down rows of every slot
  const uint32_t gu_bytes = 2u * c.npc_max * c.rowb;
  const uint32_t dn_bytes = c.nslots * c.d_slot_bytes;
  c.dbuf = o;  o = al128(o + (gu_bytes > dn_bytes ? gu_bytes : dn_bytes));
  c.rbuf = o;  o = al128(o + 2 * c.rr_max * H * 2);
  c.total = o;
  return c;
}

__device__ __forceinline__ void copy_tx(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("mbarrier.expect_tx.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
  bulk_g2s(dst, src, bytes, bar);
}

__device__ __forceinline__ void mbar_arrive1(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ void st_word(uint32_t* a, uint32_t v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(a), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_word(const uint32_t* a) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
  return v;
}

__device__ __forceinline__ uint4 ld_words4(const uint32_t* a) {
  uint4 v;
  asm volatile("ld.relaxed.gpu.global.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(a)
               : "memory");
  return v;
}

// fp32 with its last mantissa bit replaced by the layer parity.
__device__ __forceinline__ uint32_t tag_f32(float v, uint32_t par) {
  return (__float_as_uint(v) & ~1u) | par;
}

// Checked every 16 polls of a tagged-word wait that started at t0: true once
// the wait must end, because its time or poll limit ran out here
// (MOE_ERR_TIMEOUT recorded) or some CTA has already recorded an error.
__device__ __noinline__ bool give_up(uint64_t t0, uint32_t it, WsHeader* hdr, int where) {
  if (*reinterpret_cast<volatile int*>(&hdr->status) != 0) return true;
  if (globaltimer_ns() - t0 > kWaitNs || it >= kWaitIters) {
    report(hdr, MOE_ERR_TIMEOUT, where);
    return true;
  }
  return false;
}

// Between two polls that found a word not yet written: sleep a little; every
// 16 polls ask give_up.
#define MOE_POLL_BACKOFF(it, t0, hdr, where, fail) \
  {                                                \
    if ((it) == 0) (t0) = globaltimer_ns();        \
    __nanosleep(128);                              \
    if (((it) & 15u) == 15u && give_up((t0), (it), (hdr), (where))) { \
      fail = true;                                 \
      break;                                       \
    }                                              \
  }

__device__ __noinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity, WsHeader* hdr, int where) {
  return mbar_wait(bar, parity, hdr, where);
}

__device__ __forceinline__ bool mbar_ready(uint64_t* bar, uint32_t parity, WsHeader* hdr, int where) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, hdr, where);
}

__device__ __forceinline__ float silu_f(float z) { return z / (1.f + expf(-z)); }

// Order-preserving map of a float to an unsigned key (larger float, larger key).
__device__ __forceinline__ unsigned fkey(float f) {
  const unsigned u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float fkey_inv(unsigned k) {
  return __uint_as_float((k & 0x80000000u) ? (k ^ 0x80000000u) : ~k);
}

// Copy-phase bookkeeping for leaving early: parities of the phases this CTA
// still has bulk copies in flight on (-1 = none).
struct Pending {
  int r[2], g, d, gc;
};

__device__ __noinline__ void drain(Pending* pend, uint64_t* bar_r, uint64_t* bar_g, uint64_t* bar_d,
                                   uint64_t* bar_gc, int nb, WsHeader* hdr) {
  __syncthreads();
  if (threadIdx.x == 0) {
    if (pend->r[0] >= 0) mbar_wait(&bar_r[0], pend->r[0], hdr, 90);
    if (pend->r[1] >= 0) mbar_wait(&bar_r[1], pend->r[1], hdr, 91);
    if (pend->g >= 0) mbar_wait(bar_g, pend->g, hdr, 92);
    if (pend->d >= 0) mbar_wait(bar_d, pend->d, hdr, 93);
    if (pend->gc >= 0)
      for (int b = 0; b < nb; ++b) mbar_wait(&bar_gc[b], pend->gc, hdr, 94);
  }
  __syncthreads();
}

template <int BITS, int CH>
__global__ void __launch_bounds__(kThreads, 1) decode_stack_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int PS = 128 / BITS;  // codes per 16-byte segment
  extern __shared__ __align__(128) unsigned char sm[];
  __shared__ __align__(8) uint64_t bar_r[2];
  __shared__ __align__(8) uint64_t bar_g, bar_d;
  __shared__ __align__(8) uint64_t bar_gc[kMaxBatches];
  __shared__ __align__(16) LayerDesc s_ld[2];
  __shared__ int s_idx[16];
  __shared__ float s_w[16];
  __shared__ float s_sg;
  __shared__ float s_red[kWarps];
  __shared__ Pending s_pend;

  const int H = p.H, E = p.E, k = p.k, I = p.I, Is = p.Is, group = p.group;
  const int G = gridDim.x, c = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  bool ab = false;  // a wait of this thread gave up; combined over the CTA at each phase end
  const Carve cv = carve(H, E, k, I, Is, group, BITS, G);
  float* xs = reinterpret_cast<float*>(sm + cv.xs);  // x by 16-byte code segment (conflict-free float4 reads)
  float* xn = reinterpret_cast<float*>(sm + cv.xn);  // x in natural order
  float* rr = reinterpret_cast<float*>(sm + cv.rr);  // residual stream, fp32
  float* hs = reinterpret_cast<float*>(sm + cv.hs);  // h of every slot, by down code segment
  float* dred = reinterpret_cast<float*>(sm + cv.dred);
  float* guv = reinterpret_cast<float*>(sm + cv.guv);
  uint16_t* gsb = reinterpret_cast<uint16_t*>(sm + cv.gsb);
  unsigned char* dbuf = sm + cv.dbuf;
  uint16_t* rbuf = reinterpret_cast<uint16_t*>(sm + cv.rbuf);

  // ---- static assignment of this CTA's work
  const int NP = k * I + Is;
  const int gp0 = static_cast<int>(static_cast<int64_t>(c) * NP / G);
  const int gp1 = static_cast<int>(static_cast<int64_t>(c + 1) * NP / G);
  const int npc = gp1 - gp0;
  const int nb = cdiv(npc, kBatch);
  // the pair range covers at most two slots: [0, nA) in slot jA from slot row iA, then [nA, npc) in slot jA + 1
  const int jA = gp0 < k * I ? gp0 / I : k;
  const int endA = jA < k ? (jA + 1) * I : NP;
  const int nA = min(gp1, endA) - gp0;
  const int iA = gp0 - (jA < k ? jA * I : k * I);
  const int r0 = static_cast<int>(static_cast<int64_t>(c) * H / G);
  const int r1 = static_cast<int>(static_cast<int64_t>(c + 1) * H / G);
  const int nr = r1 - r0;
  const int nrows_rt = E + (Is > 0 ? 1 : 0);
  const int rr_cnt = (c < nrows_rt) ? cdiv(nrows_rt - c, G) : 0;
  const int nslots = cv.nslots;
  const int rowb = cv.rowb, rowbd = cv.rowbd, ng = cv.ng, ngd = cv.ngd;
  const int lgI = 31 - __clz(I);          // I and group are powers of two
  const int lgG = 31 - __clz(group);

  if (tid == 0) {
    mbar_init(&bar_r[0], 1);
    mbar_init(&bar_r[1], 1);
    mbar_init(&bar_g, 1);
    mbar_init(&bar_d, 1);
    for (int b = 0; b < kMaxBatches; ++b) mbar_init(&bar_gc[b], 1);
    fence_mbar_init();
    s_pend.r[0] = s_pend.r[1] = s_pend.g = s_pend.d = s_pend.gc = -1;
  }
  constexpr int kDescWords = sizeof(LayerDesc) / 8;
  static_assert(sizeof(LayerDesc) % 8 == 0 && kDescWords <= 32, "layer descriptor copy");
  if (warp == 1 && lane < kDescWords)
    reinterpret_cast<uint64_t*>(&s_ld[0])[lane] = reinterpret_cast<const uint64_t*>(&p.layers[0])[lane];
  __syncthreads();

  auto issue_router = [&](int l) {  // thread 0; s_ld[l & 1] holds layer l
    const LayerDesc& Ld = s_ld[l & 1];
    const int b = l & 1;
#pragma unroll 1
    for (int m = 0; m < rr_cnt; ++m) {
      const int row = c + m * G;
      const uint16_t* src = (row < E) ? Ld.wr + static_cast<size_t>(row) * H : Ld.wsg;
      copy_tx(rbuf + (static_cast<size_t>(b) * cv.rr_max + m) * H, src, static_cast<uint32_t>(H) * 2, &bar_r[b]);
    }
    mbar_arrive1(&bar_r[b]);
    s_pend.r[b] = (l >> 1) & 1;
  };
  auto leave = [&]() { drain(&s_pend, bar_r, &bar_g, &bar_d, bar_gc, nb, p.hdr); };

  if (tid == 0) issue_router(0);

  // lane roles in the dot products: a row of nsg 16-byte code segments is
  // covered by 32/nsg rows per warp step (nsg < 32) or by CH segments per lane
  const int nsg = cv.nsg;
  const int rps = nsg >= 32 ? 1 : 32 / nsg;
  const int gsub = nsg >= 32 ? 0 : lane / nsg;
  const int gs0 = nsg >= 32 ? lane : lane % nsg;
  const int nsgd = cv.nsgd;
  const int rpsd = 32 / nsgd;
  const int dsub = lane / nsgd;
  const int ds = lane % nsgd;
  // this warp's share of the down work: units (slot, row step), slot-major
  const int dn_upj = cdiv(nr, rpsd);
  const int dn_u0 = warp * nslots * dn_upj / kWarps, dn_u1 = (warp + 1) * nslots * dn_upj / kWarps;
  const int dn_j0 = dn_upj > 0 ? dn_u0 / dn_upj : 0;
  const int dn_t0 = dn_u0 - dn_j0 * dn_upj;

  for (int l = 0; l < p.L; ++l) {
    const int lg = p.l0 + l;  // layer index within the whole stack (trace rows)
    const uint32_t tag = static_cast<uint32_t>(l + 1);
    const uint32_t par = tag & 1u;
    auto stamp = [&](int slot) {
      if (p.tr_t && c == 0 && tid == 0) p.tr_t[static_cast<size_t>(lg) * 8 + slot] = globaltimer_ns();
    };
    stamp(0);
    // next layer's descriptor, then its router rows
    if (warp == 1 && lane < kDescWords && l + 1 < p.L)
      reinterpret_cast<uint64_t*>(&s_ld[(l + 1) & 1])[lane] =
          reinterpret_cast<const uint64_t*>(&p.layers[l + 1])[lane];

    // ---------------- 1. this layer's x (and residual)
    if (l == 0) {
#pragma unroll 1
      for (int i = tid; i < H; i += kThreads) {
        const float v = bf16_to_f32(p.x0[i]);
        xn[i] = v;
        rr[i] = p.r_in ? p.r_in[i] : v;
        if (c == 0 && p.tr_x) p.tr_x[static_cast<size_t>(p.l0) * H + i] = p.x0[i];
      }
    } else {
      // y of the previous layer: 4 rows per thread
      float ss = 0.f;
      const int i4 = 4 * tid;
      if (i4 < H) {
        const uint32_t ytag = (tag - 1u) & 0xffffu;
        uint4 w;
        uint64_t t0 = 0;
        for (uint32_t it = 0;; ++it) {
          w = ld_words4(p.ybuf + i4);
          if ((w.x & 0xffffu) == ytag && (w.y & 0xffffu) == ytag && (w.z & 0xffffu) == ytag &&
              (w.w & 0xffffu) == ytag)
            break;
          MOE_POLL_BACKOFF(it, t0, p.hdr, 20, ab)
        }
        const uint32_t wy[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float v = rr[i4 + u] + __uint_as_float(wy[u] & 0xffff0000u);
          rr[i4 + u] = v;
          ss = fmaf(v, v, ss);
        }
      }
      ss = warp_sum(ss);
      if (lane == 0) s_red[warp] = ss;
      if (__syncthreads_or(ab)) { leave(); return; }
      float tot = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) tot += s_red[w];
      const float inv = 1.f / sqrtf(tot / static_cast<float>(H) + p.eps);
#pragma unroll 1
      for (int i = tid; i < H; i += kThreads) {
        const uint16_t xb = f32_to_bf16(rr[i] * inv);
        xn[i] = bf16_to_f32(xb);
        if (c == 0 && p.tr_x) p.tr_x[static_cast<size_t>(lg) * H + i] = xb;
      }
    }
    __syncthreads();
    // x by code segment: xs[(q4 * nsg + s) * 4 + c4] = x[s * PS + q4 * 4 + c4]
#pragma unroll 1
    for (int i4 = tid; i4 < H / 4; i4 += kThreads) {
      const int s = (4 * i4) / PS, q4 = ((4 * i4) % PS) / 4;
      reinterpret_cast<float4*>(xs)[q4 * nsg + s] = reinterpret_cast<const float4*>(xn)[i4];
    }
    if (tid == 0 && l + 1 < p.L) issue_router(l + 1);
    stamp(1);

    // ---------------- 2. router rows -> logits
    if (warp < rr_cnt) {
      if (!mbar_ready(&bar_r[l & 1], (l >> 1) & 1, p.hdr, 10)) ab = true;
      const int row = c + warp * G;
      const uint4* wv = reinterpret_cast<const uint4*>(rbuf + (static_cast<size_t>(l & 1) * cv.rr_max + warp) * H);
      float acc = 0.f;
#pragma unroll 1
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
      const LayerDesc& Ld = s_ld[l & 1];
      if (lane == 0) st_word(p.logits + row, tag_f32(acc + ((row < E && Ld.rbias) ? Ld.rbias[row] : 0.f), par));
    }
    if (tid == 0) s_pend.r[l & 1] = -1;
    stamp(2);

    // ---------------- 3. softmax + top-k (every CTA, warp 0)
    if (warp == 0) {
      uint32_t wl[kTopPer];
      uint32_t wsg = par;
      {
        uint64_t t0 = 0;
        bool fail = false;
        for (uint32_t it = 0;; ++it) {
          bool ok = true;
#pragma unroll
          for (int i = 0; i < kTopPer; ++i) {
            const int e = lane + 32 * i;
            wl[i] = (e < E) ? ld_word(p.logits + e) : par;
            ok &= (wl[i] & 1u) == par;
          }
          if (Is > 0 && lane == 0) {
            wsg = ld_word(p.logits + E);
            ok &= (wsg & 1u) == par;
          }
          if (__all_sync(0xffffffffu, ok)) break;
          // warp-uniform give-up decision (lane 0 checks)
          if (it == 0) t0 = globaltimer_ns();
          __nanosleep(128);
          if ((it & 15u) == 15u && __any_sync(0xffffffffu, lane == 0 && give_up(t0, it, p.hdr, 21))) {
            fail = true;
            break;
          }
        }
        ab |= fail;
      }
      unsigned key[kTopPer];
      unsigned bk = 0u;
      int bi = 0;
#pragma unroll
      for (int i = 0; i < kTopPer; ++i) {
        key[i] = (lane + 32 * i < E) ? fkey(__uint_as_float(wl[i])) : 0u;
        if (key[i] > bk) {
          bk = key[i];
          bi = i;
        }
      }
      const float mx = fkey_inv(__reduce_max_sync(0xffffffffu, bk));
      float z = 0.f;
      if (!p.renorm) {  // softmax over all E: the words are re-read (complete and tagged by now)
#pragma unroll 1
        for (int e = lane; e < E; e += 32) z += expf(__uint_as_float(ld_word(p.logits + e)) - mx);
        z = warp_sum(z);
      }
      unsigned my_k = 0u;
      int my_e = 0;
#pragma unroll 1
      for (int j = 0; j < k; ++j) {
        // winner: largest key, then lowest expert index
        const unsigned wk = __reduce_max_sync(0xffffffffu, bk);
        const unsigned we =
            __reduce_min_sync(0xffffffffu, bk == wk ? static_cast<unsigned>(lane + 32 * bi) : 0xffffffffu);
        if (lane == j) {
          my_k = wk;
          my_e = static_cast<int>(we);
        }
        if (static_cast<int>(we & 31u) == lane) {
          const int wi = static_cast<int>(we >> 5);
          bk = 0u;
          bi = 0;
#pragma unroll
          for (int i = 0; i < kTopPer; ++i) {
            if (i == wi) key[i] = 0u;
            if (key[i] > bk) {
              bk = key[i];
              bi = i;
            }
          }
        }
      }
      const float ex = (lane < k) ? expf(fkey_inv(my_k) - mx) : 0.f;
      const float den = p.renorm ? warp_sum(ex) : z;
      if (lane < k) {
        s_idx[lane] = my_e;
        s_w[lane] = ex / den;
        if (c == 0) {
          if (p.tr_idx) p.tr_idx[static_cast<size_t>(lg) * k + lane] = my_e;
          if (p.tr_w) p.tr_w[static_cast<size_t>(lg) * k + lane] = ex / den;
        }
      }
      if (lane == 0) s_sg = (Is > 0) ? 1.f / (1.f + expf(-__uint_as_float(wsg))) : 0.f;
    }
    if (__syncthreads_or(ab)) { leave(); return; }
    stamp(3);

    const LayerDesc& Ld = s_ld[l & 1];
    // ---------------- 4a. bulk copies of this CTA's gate/up rows (warp 0), L2 prefetch of its down rows (warp 1)
    if (warp == 0) {
      {  // codes: lane = (batch, segment, gate|up)
        const int b = lane >> 2, sg = (lane >> 1) & 1, gu = lane & 1;
        const int lo = max(sg == 0 ? 0 : nA, b * kBatch);
        const int hi = min(sg == 0 ? nA : npc, b * kBatch + kBatch);
        if (hi > lo) {
          const int j = jA + sg;
          const bool routed = j < k;
          const QMat m = routed ? Ld.gu : Ld.sgu;
          const int Ij = routed ? I : Is;
          const int row = (sg == 0 ? iA : -nA) + lo;
          const uint8_t* src = m.q + static_cast<size_t>(routed ? s_idx[j] : 0) * m.q_stride +
                               static_cast<size_t>(gu * Ij + row) * rowb;
          copy_tx(dbuf + static_cast<size_t>(gu * cv.npc_max + lo) * rowb, src, static_cast<uint32_t>((hi - lo) * rowb),
                  &bar_gc[b]);
        }
      }
      if (lane < 8) {  // scales and biases: lane = (segment, kind); kind 0/1 gate/up scales, 2/3 gate/up biases
        const int sg = lane >> 2, kind = lane & 3;
        const int lo = sg == 0 ? 0 : nA, hi = sg == 0 ? nA : npc;
        if (hi > lo) {
          const int j = jA + sg;
          const bool routed = j < k;
          const QMat m = routed ? Ld.gu : Ld.sgu;
          const int Ij = routed ? I : Is;
          const int row = (sg == 0 ? iA : -nA) + lo;
          const uint16_t* src = ((kind & 2) ? m.b : m.s) + static_cast<size_t>(routed ? s_idx[j] : 0) * m.sb_stride +
                                static_cast<size_t>((kind & 1) * Ij + row) * ng;
          copy_tx(gsb + static_cast<size_t>(kind * cv.npc_max + lo) * ng, src, static_cast<uint32_t>((hi - lo) * ng) * 2u,
                  &bar_g);
        }
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive1(&bar_g);
#pragma unroll 1
        for (int b = 0; b < nb; ++b) mbar_arrive1(&bar_gc[b]);
        s_pend.g = l & 1;
        s_pend.gc = l & 1;
      }
      __syncwarp();
    } else if (warp == 1 && nr > 0) {
#pragma unroll 1
      for (int t = lane; t < 3 * nslots; t += 32) {
        const int j = t / 3, which = t % 3;
        const bool routed = j < k;
        const QMat m = routed ? Ld.dn : Ld.sdn;
        const size_t e = routed ? static_cast<size_t>(s_idx[j]) : 0;
        if (which == 0) {
          prefetch_l2(m.q + e * m.q_stride + static_cast<size_t>(r0) * rowbd, static_cast<uint32_t>(nr * rowbd));
        } else {
          const int el0 = (r0 * ngd) & ~7, el1 = al8(r1 * ngd);
          prefetch_l2((which == 2 ? m.b : m.s) + e * m.sb_stride + el0, static_cast<uint32_t>(el1 - el0) * 2u);
        }
      }
    }

    // ---------------- 4b. gate/up rows + SwiGLU
    {
      float xv[CH][PS];
      float xsm[CH];
#pragma unroll
      for (int ch = 0; ch < CH; ++ch) {
        const int s = gs0 + 32 * ch;
        float a = 0.f;
#pragma unroll
        for (int q4 = 0; q4 < PS / 4; ++q4) {
          const float4 f = reinterpret_cast<const float4*>(xs)[q4 * nsg + s];
          xv[ch][4 * q4] = f.x;
          xv[ch][4 * q4 + 1] = f.y;
          xv[ch][4 * q4 + 2] = f.z;
          xv[ch][4 * q4 + 3] = f.w;
          a += (f.x + f.y) + (f.z + f.w);
        }
        xsm[ch] = a;
      }
      bool scales_ready = false;
#pragma unroll 1
      for (int b = 0; b < nb; ++b) {
        const int lo = b * kBatch, n = min(kBatch, npc - lo);
        if (warp * rps >= 2 * n) continue;  // no row of this batch for this warp
        if (!scales_ready) {
          if (!mbar_ready(&bar_g, l & 1, p.hdr, 11)) ab = true;
          scales_ready = true;
        }
        if (!mbar_ready(&bar_gc[b], l & 1, p.hdr, 12)) ab = true;
        const int rho = warp * rps + gsub;  // [0, n) gate rows, [n, 2n) up rows of the batch
        const int gu = rho >= n ? 1 : 0;
        const int q = lo + rho - gu * n;
        float acc = 0.f;
        if (rho < 2 * n) {
          const unsigned char* row = dbuf + static_cast<size_t>(gu * cv.npc_max + q) * rowb;
          const uint16_t* sc = gsb + static_cast<size_t>(gu * cv.npc_max + q) * ng;
          const uint16_t* bi = gsb + static_cast<size_t>((2 + gu) * cv.npc_max + q) * ng;
#pragma unroll
          for (int ch = 0; ch < CH; ++ch) {
            const int s = gs0 + 32 * ch;
            const uint4 cd = *reinterpret_cast<const uint4*>(row + 16 * s);
            const int g = (s * PS) >> lgG;
            acc = fmaf(bf16_to_f32(sc[g]), dot_seg<BITS>(cd, xv[ch]), fmaf(bf16_to_f32(bi[g]), xsm[ch], acc));
          }
        }
        if (nsg >= 32) {
          acc = warp_sum(acc);
        } else {
#pragma unroll 1
          for (int o = nsg >> 1; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        }
        if (gs0 == 0 && rho < 2 * n) guv[gu * cv.npc_max + q] = acc;
      }
    }
    const bool gu_failed = __syncthreads_or(ab);
    if (tid == 0) {
      s_pend.g = -1;
      s_pend.gc = -1;
    }
    if (gu_failed) { leave(); return; }
    if (tid < npc) {
      const int P = gp0 + tid;
      const int j = P < k * I ? (P >> lgI) : k;
      const int i = P - (j << lgI);
      const float h = silu_f(guv[tid]) * guv[cv.npc_max + tid];
      st_word(p.hbuf + static_cast<size_t>(j) * I + i, tag_f32(h, par));
    }
    // down rows of every slot into the (now free) same buffer: codes, scales, biases
    if (warp == 0) {
#pragma unroll 1
      for (int t = lane; t < (nr > 0 ? 3 * nslots : 0); t += 32) {
        const int j = t / 3, which = t % 3;
        const bool routed = j < k;
        const QMat m = routed ? Ld.dn : Ld.sdn;
        const size_t e = routed ? static_cast<size_t>(s_idx[j]) : 0;
        unsigned char* slot = dbuf + static_cast<size_t>(j) * cv.d_slot_bytes;
        if (which == 0) {
          copy_tx(slot, m.q + e * m.q_stride + static_cast<size_t>(r0) * rowbd, static_cast<uint32_t>(nr * rowbd), &bar_d);
        } else {
          const int el0 = (r0 * ngd) & ~7, el1 = al8(r1 * ngd);
          uint16_t* sc = reinterpret_cast<uint16_t*>(slot + static_cast<size_t>(cv.nr_max) * rowbd);
          copy_tx(sc + (which == 2 ? cv.d_sc_el : 0), (which == 2 ? m.b : m.s) + e * m.sb_stride + el0,
                  static_cast<uint32_t>(el1 - el0) * 2u, &bar_d);
        }
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive1(&bar_d);
        s_pend.d = l & 1;
      }
    }
    stamp(4);

    // ---------------- 5a. every slot's h, by down code segment
    {
      const int nch = nslots * I / 4;
      uint4 hv[kHChunks];
      uint64_t t0 = 0;
      for (uint32_t it = 0;; ++it) {
        bool ok = true;
#pragma unroll
        for (int u = 0; u < kHChunks; ++u) {
          const int ci = tid + u * kThreads;
          if (ci < nch) {
            hv[u] = ld_words4(p.hbuf + 4 * ci);
            ok &= ((hv[u].x & hv[u].y & hv[u].z & hv[u].w & 1u) == par) && (((hv[u].x | hv[u].y | hv[u].z | hv[u].w) & 1u) == par);
          }
        }
        if (ok) break;
        MOE_POLL_BACKOFF(it, t0, p.hdr, 22, ab)
      }
#pragma unroll
      for (int u = 0; u < kHChunks; ++u) {
        const int ci = tid + u * kThreads;
        if (ci < nch) {
          const int j = (4 * ci) >> lgI, i = (4 * ci) & (I - 1);
          const int s = i / PS, q4 = (i % PS) / 4;
          reinterpret_cast<uint4*>(hs + static_cast<size_t>(j) * I)[q4 * nsgd + s] = hv[u];
        }
      }
    }
    if (__syncthreads_or(ab)) { leave(); return; }
    stamp(5);

    // ---------------- 5b. down rows of every slot for this CTA's output rows
    if (!mbar_ready(&bar_d, l & 1, p.hdr, 13)) ab = true;
    {
      const int off = r0 * ngd - ((r0 * ngd) & ~7);
      const int g = (ds * PS) >> lgG;
      int cur = -1;
      float hv[PS];
      float hsm = 0.f;
      int j = dn_j0, t = dn_t0;
#pragma unroll 1
      for (int u = dn_u0; u < dn_u1; ++u, ++t) {
        if (t == dn_upj) {
          t = 0;
          ++j;
        }
        if (j != cur) {
          cur = j;
          hsm = 0.f;
          const float4* hj = reinterpret_cast<const float4*>(hs + static_cast<size_t>(j) * I);
#pragma unroll
          for (int q4 = 0; q4 < PS / 4; ++q4) {
            const float4 f = hj[q4 * nsgd + ds];
            hv[4 * q4] = f.x;
            hv[4 * q4 + 1] = f.y;
            hv[4 * q4 + 2] = f.z;
            hv[4 * q4 + 3] = f.w;
            hsm += (f.x + f.y) + (f.z + f.w);
          }
        }
        const int rl = t * rpsd + dsub;
        float part = 0.f;
        if (rl < nr) {
          const unsigned char* slot = dbuf + static_cast<size_t>(j) * cv.d_slot_bytes;
          const uint16_t* sc = reinterpret_cast<const uint16_t*>(slot + static_cast<size_t>(cv.nr_max) * rowbd);
          const uint4 cd = *reinterpret_cast<const uint4*>(slot + static_cast<size_t>(rl) * rowbd + 16 * ds);
          const int ei = off + rl * ngd + g;
          part = fmaf(bf16_to_f32(sc[ei]), dot_seg<BITS>(cd, hv), bf16_to_f32(sc[cv.d_sc_el + ei]) * hsm);
        }
#pragma unroll 1
        for (int o = nsgd >> 1; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if (ds == 0 && rl < nr) dred[j * cv.nr_max + rl] = part;
      }
    }
    const bool dn_failed = __syncthreads_or(ab);
    if (tid == 0) s_pend.d = -1;
    if (dn_failed) { leave(); return; }
    if (tid < nr) {
      const int row = r0 + tid;
      float acc = 0.f;
#pragma unroll 1
      for (int j = 0; j < k; ++j) acc = fmaf(s_w[j], dred[j * cv.nr_max + tid], acc);
      if (Is > 0) acc = fmaf(s_sg, dred[k * cv.nr_max + tid], acc);
      const uint16_t yb = f32_to_bf16(acc);
      st_word(p.ybuf + row, (static_cast<uint32_t>(yb) << 16) | (tag & 0xffffu));
      if (p.tr_y) p.tr_y[static_cast<size_t>(lg) * H + row] = yb;
    }
    stamp(6);
  }

  // ---------------- the stack's output: residual + RMSNorm after the last layer (CTA 0)
  if (c == 0) {
    const uint32_t ytag = static_cast<uint32_t>(p.L) & 0xffffu;
    float ss = 0.f;
    const int i4 = 4 * tid;
    if (i4 < H) {
      uint4 w;
      uint64_t t0 = 0;
      for (uint32_t it = 0;; ++it) {
        w = ld_words4(p.ybuf + i4);
        if ((w.x & 0xffffu) == ytag && (w.y & 0xffffu) == ytag && (w.z & 0xffffu) == ytag && (w.w & 0xffffu) == ytag)
          break;
        MOE_POLL_BACKOFF(it, t0, p.hdr, 23, ab)
      }
      const uint32_t wy[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float v = rr[i4 + u] + __uint_as_float(wy[u] & 0xffff0000u);
        rr[i4 + u] = v;
        ss = fmaf(v, v, ss);
      }
    }
    ss = warp_sum(ss);
    if (lane == 0) s_red[warp] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) tot += s_red[w];
    const float inv = 1.f / sqrtf(tot / static_cast<float>(H) + p.eps);
#pragma unroll 1
    for (int i = tid; i < H; i += kThreads) {
      p.out[i] = f32_to_bf16(rr[i] * inv);
      if (p.r_out) p.r_out[i] = rr[i];
    }
  }
  leave();
}

template <int BITS, int CH>
cudaError_t launch_t(const DecodeParams& p, size_t smem, int grid, cudaStream_t stream) {
  auto kern = decode_stack_kernel<BITS, CH>;
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

bool pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

}  // namespace

size_t decode_stack_smem(int H, int E, int k, int I, int Is, int group, int bits, int grid) {
  const int npc_max = cdiv(k * I + Is, grid) + 1;
  // at most kMaxBatches batches of pairs, spanning at most two slots
  if (npc_max > kBatch * kMaxBatches || npc_max > I) return ~size_t(0);
  if (cdiv(E + (Is > 0 ? 1 : 0), grid) > kWarps) return ~size_t(0);  // one router row per warp
  if (cdiv(H, grid) > kThreads) return ~size_t(0);
  return carve(H, E, k, I, Is, group, bits, grid).total;
}

bool decode_stack_supported(int H, int E, int k, int I, int Is, int group, int bits) {
  const int PS = 128 / bits;
  const int nsg = H / PS, nsgd = I / PS;
  if (H % PS || I % PS || H > 2048 || H % 4) return false;  // x of a lane's segments stays in registers
  if (!(pow2(nsg) && nsg <= 32) && !(nsg % 32 == 0 && nsg / 32 <= (bits == 4 ? 2 : 4))) return false;
  if (!pow2(nsgd) || nsgd > 32) return false;           // a down row is one warp step or less
  if (Is != 0 && Is != I) return false;                 // every slot has the same down row length
  if ((H / group) % 8 != 0) return false;               // gate/up scale rows are whole 16-byte chunks
  if (k > 16 || E > 32 * kTopPer) return false;
  if ((k + 1) * I > 4 * kHChunks * kThreads) return false;
  return true;
}

cudaError_t launch_decode_stack(const DecodeParams& p, int bits, int grid, cudaStream_t stream) {
  const size_t smem = decode_stack_smem(p.H, p.E, p.k, p.I, p.Is, p.group, bits, grid);
  const int nsg = p.H * bits / 128;
  const int ch = nsg >= 32 ? nsg / 32 : 1;
  if (bits == 4) {
    if (ch == 1) return launch_t<4, 1>(p, smem, grid, stream);
    return launch_t<4, 2>(p, smem, grid, stream);
  }
  if (ch == 1) return launch_t<8, 1>(p, smem, grid, stream);
  if (ch == 2) return launch_t<8, 2>(p, smem, grid, stream);
  return launch_t<8, 4>(p, smem, grid, stream);
}

}  // namespace moe
