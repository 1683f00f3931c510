// Persistent single-token decode of a whole MoE stack in one launch, with
// each CTA's part of h kept inside the CTA ("split" over the intermediate).
//
// One CTA per SM, all co-resident (cooperative launch), walks every layer:
//   1. residual + parameter-free RMSNorm of the previous layer's output
//      (every CTA redundantly, identical arithmetic), giving this layer's x;
//   2. router rows: each CTA owns E/G rows of the router (plus the shared
//      expert's gate vector as row E), prefetched into shared memory by bulk
//      copies one layer ahead, and publishes their logits;
//   3. softmax + top-k in every CTA from all published logits (one warp);
//   4. the CTA's unit: 32 consecutive columns of one selected expert's
//      intermediate (the k*I + Is columns of the selected experts, one unit
//      per CTA, the remaining CTAs idle here). Its 32 packed gate/up row pairs
//      land in shared memory by bulk copies, the dot products dequantize in
//      registers, and SwiGLU gives the unit's 32 values of h;
//   5. the unit's 32 columns of all H down rows arrive alongside the gate/up
//      rows: 256-row tiles by the tensor memory accelerator (one 3D map per
//      layer over the experts' down codes) and the expert's whole down scale
//      and bias matrices by two bulk copies (where they do not fit beside
//      the gate/up rows, into the gate/up buffer once gate/up is done: the
//      late-copy mode). Thread t takes output rows t, t + 512, t + 1024,
//      t + 1536, forms the unit's routing-weighted partial of y for them, and
//      adds it to a replicated fp32 accumulator (reductions in L2).
// The y of a layer is then the sum of the k*I/32 + Is/32 partials: no h
// exchange between CTAs, and no CTA reads more than its own unit of any
// expert. Routing fan-out and shared experts: Swiftlet article (xix.ai),
// paragraphs 4 and 8; Runnel README, "Target". Low-bit groups: same article,
// paragraph 8. Packed gate/up: Runnel README, introduction and "Streaming CLI".
//
// Two exchanges between CTAs per layer, neither a grid barrier:
//  - logits are fp32 words whose least significant mantissa bit is replaced
//    by the layer parity (a change of at most one unit in the last place),
//    written once per layer with relaxed stores; a reader polls the words
//    until every one carries the current parity. One bit is enough: a writer
//    of layer l+1 has necessarily seen all of layer l's arrivals, so every
//    reader of layer l's logits is done with them.
//  - y: layer l's partials go to accumulator buffer l % 3 by red.add; each
//    CTA then raises one arrival counter (after a fence), and a reader waits
//    for G * (l + 1) arrivals, fences, and sums the replicas. A CTA zeroes its
//    slice of buffer (l + 1) % 3 during layer l: after the logit exchange
//    (every CTA has by then read that buffer's last contents, y of layer
//    l - 2) and before its own arrival (so the zeroes are visible before any
//    CTA's layer l + 1 reductions, which start after all layer l arrivals).
// The host zeroes the logits, the accumulators and the counter before each
// launch. Every poll and every mbarrier wait is bounded (time and polls); a
// CTA that gives up records MOE_ERR_TIMEOUT, the others see the status word
// and leave too, each after draining its own copies. The fp32 partials of y
// are added in whatever order they reach L2, so y can differ from run to run
// in its last fp32 bits before its one bf16 rounding.

#include <cfloat>
#include <climits>

#include "decode_common.cuh"
#include "moe_common.cuh"
#include "moe_launch.h"

namespace moe {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBatch = 16;                    // gate/up pairs per code batch (one mbarrier each)
constexpr int kUnit = 32;                     // columns of the intermediate per CTA
constexpr int kMaxBatches = kUnit / kBatch;
constexpr int kTopPer = 16;                   // logits per lane in the top-k warp: E <= 512
constexpr int kBoxRows = 256;                 // down rows per tensor copy

__host__ __device__ constexpr uint32_t al128(uint32_t v) { return (v + 127u) & ~127u; }
__host__ __device__ constexpr int cdiv(int a, int b) { return (a + b - 1) / b; }

// Shared-memory carve-up; identical on host (sizing) and device.
struct Carve {
  int PS, nsg, npc_max, ng, ngd, rowb, rr_max, HT, UB;
  uint32_t xs, xn, rr, hl, guv, gsb, dbuf, dcd, dss, rbuf, desc, total;
};

__host__ __device__ inline Carve carve(int H, int E, int I, int Is, int group, int bits, int G, int L, int late) {
  Carve c{};
  c.PS = 128 / bits;
  c.nsg = H / c.PS;
  c.npc_max = kUnit;
  c.ng = H / group;
  c.ngd = I / group;
  c.rowb = H * bits / 8;
  c.rr_max = cdiv(E + (Is > 0 ? 1 : 0), G);
  c.HT = H / 4;
  c.UB = kUnit * bits / 8;  // bytes of one down row inside the unit
  uint32_t o = 0;
  c.xs = o;    o = al128(o + H * 4);
  c.xn = o;    o = al128(o + H * 4);
  c.rr = o;    o = al128(o + H * 4);
  c.hl = o;    o = al128(o + kUnit * 4);
  c.guv = o;   o = al128(o + 2 * kUnit * 4);
  c.gsb = o;   o = al128(o + 4 * kUnit * c.ng * 2);
  const uint32_t gu_bytes = 2 * kUnit * c.rowb;                 // gate/up code rows
  const uint32_t dn_bytes = al128(H * c.UB) + 2 * H * c.ngd * 2;  // the unit's down codes [row][UB], then
                                                                  // the expert's down scales and biases
  if (late) {  // the down data reuses the gate/up buffer once gate/up is done
    c.dbuf = o;  o = al128(o + (gu_bytes > dn_bytes ? gu_bytes : dn_bytes));
    c.dcd = c.dbuf;
    c.dss = c.dbuf + al128(H * c.UB);
  } else {
    c.dbuf = o;  o = al128(o + gu_bytes);
    c.dcd = o;   o = al128(o + H * c.UB);
    c.dss = o;   o = al128(o + 2 * H * c.ngd * 2);
  }
  c.rbuf = o;  o = al128(o + 2 * c.rr_max * H * 2);
  c.desc = o;  o = al128(o + L * sizeof(LayerDesc));             // the launch's layer descriptors
  c.total = o;
  return c;
}

// An fp32 accumulator += v, in L2 (a reduction: no value comes back).
__device__ __forceinline__ void red_add(float* a, float v) {
  asm volatile("red.relaxed.gpu.global.add.f32 [%0], %1;" ::"l"(a), "f"(v) : "memory");
}

// 3D tiled tensor copy (x innermost) into this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void tma_3d(void* dst, const CUtensorMap* m, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
          smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_addr(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Copy-phase bookkeeping for leaving early: parities of the phases this CTA
// still has bulk copies in flight on (-1 = none).
struct Pending {
  int r[2], gc, dn;
};

__device__ __noinline__ void drain(Pending* pend, uint64_t* bar_r, uint64_t* bar_gc, uint64_t* bar_dn, int nb,
                                   WsHeader* hdr) {
  __syncthreads();
  if (threadIdx.x == 0) {
    if (pend->r[0] >= 0) mbar_wait(&bar_r[0], pend->r[0], hdr, 90);
    if (pend->r[1] >= 0) mbar_wait(&bar_r[1], pend->r[1], hdr, 91);
    if (pend->gc >= 0)
      for (int b = 0; b < nb; ++b) mbar_wait(&bar_gc[b], pend->gc, hdr, 94);
    if (pend->dn >= 0) mbar_wait(bar_dn, pend->dn, hdr, 95);
  }
  __syncthreads();
}

template <int BITS, int CH>
__global__ void __launch_bounds__(kThreads, 1) decode_split_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int PS = 128 / BITS;  // codes per 16-byte segment
  extern __shared__ __align__(128) unsigned char sm[];
  __shared__ __align__(8) uint64_t bar_r[2];
  __shared__ __align__(8) uint64_t bar_gc[kMaxBatches];
  __shared__ __align__(8) uint64_t bar_dn;
  __shared__ int s_idx[16];
  __shared__ float s_w[16];
  __shared__ float s_sg;
  __shared__ float s_red[kWarps];
  __shared__ Pending s_pend;

  const int H = p.H, E = p.E, k = p.k, I = p.I, Is = p.Is, group = p.group;
  const int G = gridDim.x, c = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  bool ab = false;  // a wait of this thread gave up; combined over the CTA at each phase end
  const Carve cv = carve(H, E, I, Is, group, BITS, G, p.L, p.split_late);
  float* xs = reinterpret_cast<float*>(sm + cv.xs);  // x by 16-byte code segment (conflict-free float4 reads)
  float* xn = reinterpret_cast<float*>(sm + cv.xn);  // x in natural order
  float* rr = reinterpret_cast<float*>(sm + cv.rr);  // residual stream, fp32
  float* hl = reinterpret_cast<float*>(sm + cv.hl);  // the unit's h, in code order
  float* guv = reinterpret_cast<float*>(sm + cv.guv);
  uint16_t* gsb = reinterpret_cast<uint16_t*>(sm + cv.gsb);
  unsigned char* dbuf = sm + cv.dbuf;
  unsigned char* dcd = sm + cv.dcd;
  unsigned char* dss = sm + cv.dss;
  uint16_t* rbuf = reinterpret_cast<uint16_t*>(sm + cv.rbuf);
  const LayerDesc* s_layers = reinterpret_cast<const LayerDesc*>(sm + cv.desc);

  // ---- static assignment of this CTA's work: unit c (if any) = columns [32c, 32c + 32) of the
  // flattened (slot, column) space, slot j at [j * I, (j + 1) * I), the shared expert last
  const int NP = k * I + Is;
  const int gp0 = c < NP / kUnit ? c * kUnit : 0;
  const int npc = c < NP / kUnit ? kUnit : 0;
  const int gp1 = gp0 + npc;
  const int nb = cdiv(npc, kBatch);
  // gate/up code of the batches below handles a pair range over up to two slots; a unit is in one
  const int jA = gp0 < k * I ? gp0 / I : k;
  const int nA = npc;
  const int iA = gp0 - (jA < k ? jA * I : k * I);
  const bool u_routed = jA < k;
  const int u_g = iA / group;  // the unit's quantisation group along the down rows
  const int nrows_rt = E + (Is > 0 ? 1 : 0);
  const int rr_cnt = (c < nrows_rt) ? cdiv(nrows_rt - c, G) : 0;
  const uint32_t* lg_in = p.logits + (c % kDecodeReplicas) * p.logits_rep;  // this CTA's copy of the logits
  const int rowb = cv.rowb, ng = cv.ng, ngd = cv.ngd, HT = cv.HT;
  const int lgG = 31 - __clz(group);  // group is a power of two
  (void)gp1;

  if (tid == 0) {
    mbar_init(&bar_r[0], 1);
    mbar_init(&bar_r[1], 1);
    for (int b = 0; b < kMaxBatches; ++b) mbar_init(&bar_gc[b], 1);
    mbar_init(&bar_dn, 1);
    fence_mbar_init();
    s_pend.r[0] = s_pend.r[1] = s_pend.gc = s_pend.dn = -1;
  }
  // every layer descriptor of the launch into shared memory, once (parameter-space reads
  // with a runtime index would otherwise miss the constant cache in the middle of a layer)
  static_assert(sizeof(LayerDesc) % 8 == 0, "layer descriptor copy");
#pragma unroll 1
  for (int i = tid; i < p.L * static_cast<int>(sizeof(LayerDesc) / 8); i += kThreads)
    reinterpret_cast<uint64_t*>(sm + cv.desc)[i] = reinterpret_cast<const uint64_t*>(p.layers)[i];
  __syncthreads();

  auto issue_router = [&](int l) {  // one thread
    const LayerDesc& Ld = s_layers[l];
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
  auto leave = [&]() { drain(&s_pend, bar_r, bar_gc, &bar_dn, nb, p.hdr); };

  if (tid == 0) issue_router(0);

  // lane roles in the gate/up dot products: a row of nsg 16-byte code segments is
  // covered by 32/nsg rows per warp step (nsg < 32) or by CH segments per lane
  const int nsg = cv.nsg;
  const int rps = nsg >= 32 ? 1 : 32 / nsg;
  const int gsub = nsg >= 32 ? 0 : lane / nsg;
  const int gs0 = nsg >= 32 ? lane : lane % nsg;

  // y of layer lp (all CTAs' partials in): rows 4t .. 4t+3, the replicas summed in order
  auto read_y = [&](int lp, float (&y)[4]) {
    const float* yb = p.yacc + static_cast<size_t>(lp % kDecodeYBufs) * p.ybuf_stride + 4 * tid;
    y[0] = y[1] = y[2] = y[3] = 0.f;
#pragma unroll
    for (int r = 0; r < kDecodeReplicas; ++r) {
      const uint4 w = ld_words4(reinterpret_cast<const uint32_t*>(yb + static_cast<size_t>(r) * p.yrep));
      y[0] += __uint_as_float(w.x);
      y[1] += __uint_as_float(w.y);
      y[2] += __uint_as_float(w.z);
      y[3] += __uint_as_float(w.w);
    }
  };
  // thread 0: wait until `target` arrivals are in, then an acquire fence
  auto wait_arrivals = [&](uint32_t target, int where) {
    if (tid != 0) return;
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
      if (ld_word(p.arrive) >= target) break;
      MOE_POLL_BACKOFF(it, t0, p.hdr, where, ab)
    }
    __threadfence();
  };

  // the unit's down data (thread 32): 256-row tiles of its 32 columns of the down codes, and
  // the expert's whole down scale and bias matrices
  auto issue_down = [&](const LayerDesc& Ld, int l) {
    const QMat& m = u_routed ? Ld.dn : Ld.sdn;
    const CUtensorMap* tm = u_routed ? &p.tm_dn[l] : &p.tm_sdn[l];
    const int e = u_routed ? s_idx[jA] : 0;
    const uint32_t sbytes = static_cast<uint32_t>(H) * ngd * 2;
    // the buffer may last have been read by ordinary loads (gate/up or the previous layer's down)
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    mbar_arrive_expect_tx(&bar_dn, static_cast<uint32_t>(H) * cv.UB + 2 * sbytes);
#pragma unroll 1
    for (int r0 = 0; r0 < H; r0 += kBoxRows) tma_3d(dcd + r0 * cv.UB, tm, iA * BITS / 8, r0, e, &bar_dn);
    bulk_g2s(dss, m.s + static_cast<size_t>(e) * m.sb_stride, sbytes, &bar_dn);
    bulk_g2s(dss + sbytes, m.b + static_cast<size_t>(e) * m.sb_stride, sbytes, &bar_dn);
    s_pend.dn = l & 1;
  };

  for (int l = 0; l < p.L; ++l) {
    const int lg = p.l0 + l;  // layer index within the whole stack (trace rows)
    const uint32_t tag = static_cast<uint32_t>(l + 1);
    const uint32_t par = tag & 1u;
    auto stamp = [&](int slot) {
      if (p.tr_t && c == 0 && tid == 0) p.tr_t[static_cast<size_t>(lg) * 8 + slot] = globaltimer_ns();
    };
    stamp(0);

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
      wait_arrivals(static_cast<uint32_t>(G) * static_cast<uint32_t>(l), 20);
      if (__syncthreads_or(ab)) { leave(); return; }
      float ss = 0.f;
      if (tid < HT) {
        float y[4];
        read_y(l - 1, y);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint16_t yb = f32_to_bf16(y[u]);
          const float v = rr[4 * tid + u] + bf16_to_f32(yb);
          rr[4 * tid + u] = v;
          ss = fmaf(v, v, ss);
          if (c == 0 && p.tr_y) p.tr_y[static_cast<size_t>(lg - 1) * H + 4 * tid + u] = yb;
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
        const uint16_t xb = f32_to_bf16(rr[i] * inv);
        xn[i] = bf16_to_f32(xb);
        if (c == 0 && p.tr_x) p.tr_x[static_cast<size_t>(lg) * H + i] = xb;
      }
    }
    __syncthreads();
    // x by code segment: xs[(q4 * nsg + s) * 4 + c4] = x[s * PS + o], q4 * 4 + c4 = seg_pos(o)
#pragma unroll 1
    for (int i = tid; i < H; i += kThreads) {
      const int s = i / PS, op = seg_pos<BITS>(i % PS);
      xs[((op >> 2) * nsg + s) * 4 + (op & 3)] = xn[i];
    }
    if (tid == kThreads - 32 && l + 1 < p.L) issue_router(l + 1);  // a warp without router rows
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
      const LayerDesc& Ld = s_layers[l];
      if (lane < kDecodeReplicas)
        st_word(p.logits + lane * p.logits_rep + row, tag_f32(acc + ((row < E && Ld.rbias) ? Ld.rbias[row] : 0.f), par));
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
            wl[i] = (e < E) ? ld_word(lg_in + e) : par;
            ok &= (wl[i] & 1u) == par;
          }
          if (Is > 0 && lane == 0) {
            wsg = ld_word(lg_in + E);
            ok &= (wsg & 1u) == par;
          }
          if (__all_sync(0xffffffffu, ok)) break;
          // warp-uniform give-up decision (lane 0 checks)
          if (it == 0) t0 = globaltimer_ns();
          if ((it & 15u) == 15u && __any_sync(0xffffffffu, lane == 0 && give_up(t0, it, p.hdr, 21))) {
            fail = true;
            break;
          }
        }
        ab |= fail;
      }
      unsigned my_k, kmax;
      int my_e;
      if (E <= 256) topk_sorted<8>(wl, E, k, lane, my_k, my_e, kmax);
      else topk_sorted<kTopPer>(wl, E, k, lane, my_k, my_e, kmax);
      const float mx = fkey_inv(kmax);
      float z = 0.f;
      if (!p.renorm) {  // softmax over all E: the words are re-read (complete and tagged by now)
#pragma unroll 1
        for (int e = lane; e < E; e += 32) z += expf(__uint_as_float(ld_word(lg_in + e)) - mx);
        z = warp_sum(z);
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

    // ---------------- 4a. the unit's gate/up code rows: bulk copies by warp 0 (lane = batch,
    // segment, gate|up), issued after the barrier that publishes the selection; its gate/up
    // scales and biases: one 16-byte load per thread into shared memory; its down codes (tensor
    // tiles) and the expert's down scales and biases (bulk copies): thread 32
    const LayerDesc& Ld = s_layers[l];
    if (warp == 0) {
      // the buffer was last read and written by ordinary loads and per-thread copies
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      const int b = lane >> 2, sg = (lane >> 1) & 1, gu = lane & 1;
      const int lo = max(sg == 0 ? 0 : nA, b * kBatch);
      const int hi = min(sg == 0 ? nA : npc, b * kBatch + kBatch);
      if (b < kMaxBatches && hi > lo) {
        const int j = jA + sg;
        const bool routed = j < k;
        const QMat& m = routed ? Ld.gu : Ld.sgu;
        const int Ij = routed ? I : Is;
        const int row = (sg == 0 ? iA : -nA) + lo;
        const uint8_t* src = m.q + static_cast<size_t>(routed ? s_idx[j] : 0) * m.q_stride +
                             static_cast<size_t>(gu * Ij + row) * rowb;
        copy_tx(dbuf + static_cast<size_t>(gu * cv.npc_max + lo) * rowb, src, static_cast<uint32_t>((hi - lo) * rowb),
                &bar_gc[b]);
      }
      __syncwarp();
      if (lane == 0) {
#pragma unroll 1
        for (int bb = 0; bb < nb; ++bb) mbar_arrive1(&bar_gc[bb]);
        s_pend.gc = l & 1;
      }
      __syncwarp();
    }
    {
      // scales and biases, in 16-byte chunks q = (kind * npc + pair) * cpr + part;
      // kind 0/1 gate/up scales, 2/3 gate/up biases
      const int cpr = ng >> 3;
      const int per_kind = npc * cpr;
#pragma unroll 1
      for (int q = tid; q < 4 * per_kind; q += kThreads) {
        const int kind = q / per_kind, rem = q - kind * per_kind;
        const int pair = rem / cpr, part = rem - pair * cpr;
        const int sg = pair < nA ? 0 : 1;
        const int j = jA + sg;
        const bool routed = j < k;
        const QMat& m = routed ? Ld.gu : Ld.sgu;
        const int Ij = routed ? I : Is;
        const int row = sg == 0 ? iA + pair : pair - nA;
        const uint16_t* src = ((kind & 2) ? m.b : m.s) + static_cast<size_t>(routed ? s_idx[j] : 0) * m.sb_stride +
                              static_cast<size_t>((kind & 1) * Ij + row) * ng + part * 8;
        *reinterpret_cast<uint4*>(gsb + static_cast<size_t>(kind * cv.npc_max + pair) * ng + part * 8) =
            __ldg(reinterpret_cast<const uint4*>(src));
      }
    }
    if (!p.split_late && tid == 32 && npc > 0) issue_down(Ld, l);
    {
      // this CTA's slice of the accumulators of layer l + 1
      const int nz = kDecodeReplicas * p.yrep;
      uint32_t* zb = reinterpret_cast<uint32_t*>(p.yacc + static_cast<size_t>((l + 1) % kDecodeYBufs) * p.ybuf_stride);
      const int z1 = static_cast<int>(static_cast<int64_t>(c + 1) * nz / G);
#pragma unroll 1
      for (int i = static_cast<int>(static_cast<int64_t>(c) * nz / G) + tid; i < z1; i += kThreads) st_word(zb + i, 0u);
    }
    __syncthreads();  // the gate/up scales are in shared memory

    // ---------------- 4b. gate/up rows + SwiGLU, batch by batch as the codes land
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
#pragma unroll 1
      for (int b = 0; b < nb; ++b) {
        const int lo = b * kBatch, n = min(kBatch, npc - lo);
        if (warp * rps >= 2 * n) continue;  // no row of this batch for this warp
        if (!mbar_ready(&bar_gc[b], l & 1, p.hdr, 12)) ab = true;
        // two rows of the batch at a time (rows rw and rw + 16 * rps), for independent work in flight
#pragma unroll 1
        for (int rw = warp * rps; rw < 2 * n; rw += 2 * kWarps * rps) {
          float acc[2];
          int qv[2], guv_i[2];
#pragma unroll
          for (int r2 = 0; r2 < 2; ++r2) {
            const int rho = rw + r2 * kWarps * rps + gsub;  // [0, n) gate rows, [n, 2n) up rows of the batch
            const int gu = rho >= n ? 1 : 0;
            const int q = lo + rho - gu * n;
            qv[r2] = rho < 2 * n ? q : -1;
            guv_i[r2] = gu * cv.npc_max + q;
            acc[r2] = 0.f;
            if (rho < 2 * n) {
              const unsigned char* row = dbuf + static_cast<size_t>(gu * cv.npc_max + q) * rowb;
              const uint16_t* sc = gsb + static_cast<size_t>(gu * cv.npc_max + q) * ng;
              const uint16_t* bi = gsb + static_cast<size_t>((2 + gu) * cv.npc_max + q) * ng;
#pragma unroll
              for (int ch = 0; ch < CH; ++ch) {
                const int s = gs0 + 32 * ch;
                const uint4 cd = *reinterpret_cast<const uint4*>(row + 16 * s);
                const int g = (s * PS) >> lgG;
                acc[r2] = fmaf(bf16_to_f32(sc[g]), dot_seg_dec<BITS>(cd, xv[ch]), fmaf(bf16_to_f32(bi[g]), xsm[ch], acc[r2]));
              }
            }
          }
          if (nsg >= 32) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
              acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], o);
              acc[1] += __shfl_xor_sync(0xffffffffu, acc[1], o);
            }
          } else {
#pragma unroll 1
            for (int o = nsg >> 1; o > 0; o >>= 1) {
              acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], o);
              acc[1] += __shfl_xor_sync(0xffffffffu, acc[1], o);
            }
          }
          if (gs0 == 0) {
            if (qv[0] >= 0) guv[guv_i[0]] = acc[0];
            if (qv[1] >= 0) guv[guv_i[1]] = acc[1];
          }
        }
      }
    }
    const bool gu_failed = __syncthreads_or(ab);
    if (tid == 0) s_pend.gc = -1;
    if (gu_failed) { leave(); return; }
    if (tid < npc) hl[(tid & ~15) | seg_pos<BITS>(tid & 15)] = silu_f(guv[tid]) * guv[cv.npc_max + tid];
    if (p.split_late && tid == 32 && npc > 0) issue_down(s_layers[l], l);  // into the freed gate/up buffer
    if (npc > 0 && tid < HT && !mbar_ready(&bar_dn, l & 1, p.hdr, 13)) ab = true;
    if (__syncthreads_or(ab)) { leave(); return; }
    if (tid == 0) s_pend.dn = -1;
    stamp(4);

    // ---------------- 5. the unit's partial of y for rows t, t + 512, t + 1024, t + 1536 (a warp
    // reads 32 consecutive rows of codes, and reduces into 32 consecutive words of y):
    // routing weight x (scale x codes . h + bias x sum h)
    if (npc > 0) {
      float hv[kUnit];
      float hsum = 0.f;
#pragma unroll
      for (int q4 = 0; q4 < kUnit / 4; ++q4) {
        const float4 f = reinterpret_cast<const float4*>(hl)[q4];
        hv[4 * q4] = f.x;
        hv[4 * q4 + 1] = f.y;
        hv[4 * q4 + 2] = f.z;
        hv[4 * q4 + 3] = f.w;
        hsum += (f.x + f.y) + (f.z + f.w);
      }
      const float wgt = u_routed ? s_w[jA] : s_sg;
      const uint16_t* dsc = reinterpret_cast<const uint16_t*>(dss);
      const uint16_t* dbi = dsc + static_cast<size_t>(H) * ngd;
      float* yrow = p.yacc + static_cast<size_t>(l % kDecodeYBufs) * p.ybuf_stride +
                    static_cast<size_t>(c % kDecodeReplicas) * p.yrep;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int r = tid + q * kThreads;
        if (r < H) {
          float d;
          if constexpr (BITS == 4) {
            d = dot_seg_dec<4>(*reinterpret_cast<const uint4*>(dcd + r * cv.UB), hv);
          } else {
            d = dot_seg<8>(*reinterpret_cast<const uint4*>(dcd + r * cv.UB), hv) +
                dot_seg<8>(*reinterpret_cast<const uint4*>(dcd + r * cv.UB + 16), hv + 16);
          }
          red_add(yrow + r, wgt * fmaf(bf16_to_f32(dsc[r * ngd + u_g]), d, bf16_to_f32(dbi[r * ngd + u_g]) * hsum));
        }
      }
    }
    if (__syncthreads_or(ab)) { leave(); return; }
    if (tid == 0) {
      __threadfence();  // this CTA's reductions and zeroes, ordered by the barrier, before its arrival
      atomicAdd(p.arrive, 1u);
    }
    stamp(6);
  }

  // ---------------- the stack's output: residual + RMSNorm after the last layer (CTA 0)
  if (c == 0) {
    wait_arrivals(static_cast<uint32_t>(G) * static_cast<uint32_t>(p.L), 23);
    if (__syncthreads_or(ab)) { leave(); return; }
    float ss = 0.f;
    if (tid < HT) {
      float y[4];
      read_y(p.L - 1, y);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint16_t yb = f32_to_bf16(y[u]);
        const float v = rr[4 * tid + u] + bf16_to_f32(yb);
        rr[4 * tid + u] = v;
        ss = fmaf(v, v, ss);
        if (p.tr_y) p.tr_y[static_cast<size_t>(p.l0 + p.L - 1) * H + 4 * tid + u] = yb;
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
  auto kern = decode_split_kernel<BITS, CH>;
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

bool decode_split_plan(int H, int E, int k, int I, int Is, int group, int bits, int grid, int L, size_t smem_limit,
                       size_t* smem, int* late) {
  if (grid < 1 || L < 1) return false;
  if (L > kMaxDecodeLayers) L = kMaxDecodeLayers;
  const int PS = 128 / bits;
  const int nsg = H / PS;
  if (H % PS || H > 2048 || H % kBoxRows) return false;  // x of a lane's segments in registers; whole tiles
  if (!(pow2(nsg) && nsg <= 32) && !(nsg % 32 == 0 && nsg / 32 <= (bits == 4 ? 2 : 4))) return false;
  if (Is != 0 && Is != I) return false;          // one down row length (and scale row) for every slot
  if (I % kUnit || !pow2(group) || group % kUnit || I % group) return false;  // a unit lies in one group
  if ((H / group) % 8 != 0) return false;        // gate/up scale rows are whole 16-byte chunks
  if (k > 16 || E > 32 * kTopPer) return false;
  if ((k * I + Is) / kUnit > grid) return false;  // at most one unit per CTA
  if (cdiv(E + (Is > 0 ? 1 : 0), grid) > kWarps) return false;  // one router row per warp
  for (int lt = 0; lt < 2; ++lt) {  // down data in a region of its own if it fits, else after gate/up
    const size_t need = carve(H, E, I, Is, group, bits, grid, L, lt).total;
    if (need <= smem_limit) {
      *smem = need;
      *late = lt;
      return true;
    }
  }
  return false;
}

cudaError_t launch_decode_split(const DecodeParams& p, int bits, int grid, cudaStream_t stream) {
  const size_t smem = carve(p.H, p.E, p.I, p.Is, p.group, bits, grid, p.L, p.split_late).total;
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
