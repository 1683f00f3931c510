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

#include "decode_common.cuh"
#include "moe_common.cuh"
#include "moe_launch.h"

namespace moe {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBatch = 16;       // gate/up pairs per code batch (one mbarrier each)
constexpr int kMaxBatches = 4;   // at most 64 pairs per CTA
constexpr int kHChunks = 4;      // 16-byte chunks of h each thread reads: (k+1)*I <= 4*4*512
constexpr int kTopPer = 16;      // logits per lane in the top-k warp: E <= 512

__host__ __device__ constexpr uint32_t al128(uint32_t v) { return (v + 127u) & ~127u; }
__host__ __device__ constexpr int cdiv(int a, int b) { return (a + b - 1) / b; }

// Shared-memory carve-up; identical on host (sizing) and device.
struct Carve {
  int PS, nsg, nsgd, nslots, npc_max, ng, nr_max, ngd, rowb, rowbd, rr_max, nunits, d_sc_el;
  uint32_t xs, xn, rr, hs, dred, guv, gsb, dbuf, dsc, rbuf, desc, total;
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
  c.rr_max = cdiv(E + (Is > 0 ? 1 : 0), G);
  c.nunits = c.nslots * cdiv(c.nr_max, 32 / c.nsgd);  // down work units (slot, row step) of a CTA, at most
  c.d_sc_el = (c.nr_max * c.ngd + 16 + 7) & ~7;       // a slot's down scales (or biases) of the CTA's rows
  uint32_t o = 0;
  c.xs = o;    o = al128(o + H * 4);
  c.xn = o;    o = al128(o + H * 4);
  c.rr = o;    o = al128(o + H * 4);
  c.hs = o;    o = al128(o + c.nslots * I * 4);
  c.dred = o;  o = al128(o + c.nslots * c.nr_max * 4);
  c.guv = o;   o = al128(o + 2 * c.npc_max * 4);
  c.gsb = o;   o = al128(o + 4 * c.npc_max * c.ng * 2);
  // one buffer: first this CTA's gate/up code rows ([gate rows][up rows]), then (once gate/up
  // is done) its down code segments by work unit ([unit][lane] x 16 bytes) and its down scales
  // and biases by slot. (Copying the down rows into a region of their own right after top-k
  // was measured slower: they compete with the gate/up stream, which is on the critical path.)
  const uint32_t gu_bytes = 2u * c.npc_max * c.rowb;
  const uint32_t dn_bytes = c.nunits * 512u + c.nslots * 4u * c.d_sc_el;
  c.dsc = c.nunits * 512u;  // offset of the down scales inside the buffer
  c.dbuf = o;  o = al128(o + (gu_bytes > dn_bytes ? gu_bytes : dn_bytes));
  c.rbuf = o;  o = al128(o + 2 * c.rr_max * H * 2);
  c.desc = o;  o = al128(o + kMaxDecodeLayers * sizeof(LayerDesc));  // the launch's layer descriptors
  c.total = o;
  return c;
}

// Copy-phase bookkeeping for leaving early: parities of the phases this CTA
// still has bulk copies in flight on (-1 = none).
struct Pending {
  int r[2], gc;
};

__device__ __noinline__ void drain(Pending* pend, uint64_t* bar_r, uint64_t* bar_gc, int nb, WsHeader* hdr) {
  __syncthreads();
  if (threadIdx.x == 0) {
    if (pend->r[0] >= 0) mbar_wait(&bar_r[0], pend->r[0], hdr, 90);
    if (pend->r[1] >= 0) mbar_wait(&bar_r[1], pend->r[1], hdr, 91);
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
  __shared__ __align__(8) uint64_t bar_gc[kMaxBatches];
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
  const LayerDesc* s_layers = reinterpret_cast<const LayerDesc*>(sm + cv.desc);

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
  // this CTA's copy of the exchange words
  const uint32_t* lg_in = p.logits + (c % kDecodeReplicas) * p.logits_rep;
  const uint32_t* h_in = p.hbuf + (c % kDecodeReplicas) * p.h_rep;
  const uint32_t* y_in = p.ybuf + (c % kDecodeReplicas) * p.y_rep;
  const int rowb = cv.rowb, rowbd = cv.rowbd, ng = cv.ng, ngd = cv.ngd;
  const int lgI = 31 - __clz(I);          // I and group are powers of two
  const int lgG = 31 - __clz(group);

  if (tid == 0) {
    mbar_init(&bar_r[0], 1);
    mbar_init(&bar_r[1], 1);
    for (int b = 0; b < kMaxBatches; ++b) mbar_init(&bar_gc[b], 1);
    fence_mbar_init();
    s_pend.r[0] = s_pend.r[1] = s_pend.gc = -1;
  }
  // every layer descriptor of the launch into shared memory, once (parameter-space reads
  // with a runtime index would otherwise miss the constant cache in the middle of a layer)
  static_assert(sizeof(LayerDesc) % 8 == 0, "layer descriptor copy");
#pragma unroll 1
  for (int i = tid; i < p.L * static_cast<int>(sizeof(LayerDesc) / 8); i += kThreads)
    reinterpret_cast<uint64_t*>(sm + cv.desc)[i] = reinterpret_cast<const uint64_t*>(p.layers)[i];
  __syncthreads();

  auto issue_router = [&](int l) {  // thread 0
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
  auto leave = [&]() { drain(&s_pend, bar_r, bar_gc, nb, p.hdr); };

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
  const int dn_j0 = dn_upj > 0 ? dn_u0 / dn_upj : 0, dn_t0 = dn_u0 - dn_j0 * dn_upj;  // first unit = (slot, step)
  unsigned char* const dnbuf = sm + cv.dbuf;
  // this CTA's down rows into shared memory by per-thread asynchronous copies: the code
  // segment of every work unit u = (slot, row step) of this warp ([u][lane] x 16 bytes), and
  // (warp j % 16) slot j's scales and biases of the CTA's rows
  auto issue_down = [&](const LayerDesc& Ld) {
    uint16_t* dscl = reinterpret_cast<uint16_t*>(dnbuf + cv.dsc);
#pragma unroll 1
    for (int u = dn_u0; u < dn_u1; ++u) {
      const int j = u / dn_upj, t = u - j * dn_upj;
      const int rl = t * rpsd + dsub;
      if (rl < nr) {
        const bool routed = j < k;
        const QMat& m = routed ? Ld.dn : Ld.sdn;
        const size_t e = routed ? static_cast<size_t>(s_idx[j]) : 0;
        cp_async16(dnbuf + (static_cast<size_t>(u) * 32 + lane) * 16,
                   m.q + e * m.q_stride + static_cast<size_t>(r0 + rl) * rowbd + 16 * ds);
      }
    }
    const int el0 = (r0 * ngd) & ~7, nel = (((r1 * ngd) + 7) & ~7) - el0;
#pragma unroll 1
    for (int j = warp; j < (nr > 0 ? nslots : 0); j += kWarps) {
      const bool routed = j < k;
      const QMat& m = routed ? Ld.dn : Ld.sdn;
      const size_t e = routed ? static_cast<size_t>(s_idx[j]) : 0;
#pragma unroll 1
      for (int q = lane; q < 2 * (nel / 8); q += 32) {
        const int which = q / (nel / 8), part = q - which * (nel / 8);
        cp_async16(dscl + (2 * j + which) * cv.d_sc_el + 8 * part, (which ? m.b : m.s) + e * m.sb_stride + el0 + 8 * part);
      }
    }
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
        if (c == 0 && p.tr_x) p.tr_x[static_cast<size_t>(p.l0) * p.tr_rows * H + i] = p.x0[i];
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
          w = ld_words4(y_in + i4);
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
        if (c == 0 && p.tr_x) p.tr_x[static_cast<size_t>(lg) * p.tr_rows * H + i] = xb;
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
          if (p.tr_idx) p.tr_idx[static_cast<size_t>(lg) * p.tr_rows * k + lane] = my_e;
          if (p.tr_w) p.tr_w[static_cast<size_t>(lg) * p.tr_rows * k + lane] = ex / den;
        }
      }
      if (lane == 0) s_sg = (Is > 0) ? 1.f / (1.f + expf(-__uint_as_float(wsg))) : 0.f;
    }
    if (__syncthreads_or(ab)) { leave(); return; }
    stamp(3);

    // ---------------- 4a. this CTA's gate/up code rows: bulk copies by warp 0 (lane = batch,
    // segment, gate|up), issued after the barrier that publishes the selection (issued by the
    // top-k warp before it, the early CTAs' copies measurably slowed the logit exchange of the
    // others); its gate/up scales and biases: one 16-byte load per thread into shared memory;
    // its down rows: prefetched into L2 for phase 5
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
        const int row = (sg == 0 ? iA : -nA) + lo;
        const uint8_t* src = m.q + static_cast<size_t>(routed ? s_idx[j] : 0) * m.q_stride + (gu ? m.up_q : 0) +
                             static_cast<size_t>(row) * rowb;
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
        const int row = sg == 0 ? iA + pair : pair - nA;
        const uint16_t* src = ((kind & 2) ? m.b : m.s) + static_cast<size_t>(routed ? s_idx[j] : 0) * m.sb_stride +
                              ((kind & 1) ? ((kind & 2) ? m.up_b : m.up_s) : 0) + static_cast<size_t>(row) * ng +
                              part * 8;
        *reinterpret_cast<uint4*>(gsb + static_cast<size_t>(kind * cv.npc_max + pair) * ng + part * 8) =
            __ldg(reinterpret_cast<const uint4*>(src));
      }
    }
    {
      // down rows of every slot (codes, scales, biases) into L2: warp w takes slots w, w + 16, ...
#pragma unroll 1
      for (int j = warp; j < (nr > 0 ? nslots : 0); j += kWarps) {
        const bool routed = j < k;
        const QMat& m = routed ? Ld.dn : Ld.sdn;
        const size_t e = routed ? static_cast<size_t>(s_idx[j]) : 0;
        const uintptr_t a0 = reinterpret_cast<uintptr_t>(m.q + e * m.q_stride + static_cast<size_t>(r0) * rowbd);
        const int nl = static_cast<int>(((a0 & 127) + static_cast<uintptr_t>(nr) * rowbd + 127) >> 7);
#pragma unroll 1
        for (int t = lane; t < nl; t += 32) prefetch_line_l2(reinterpret_cast<const void*>((a0 & ~uintptr_t(127)) + 128u * t));
        if (lane < 2) {
          const uintptr_t s0 =
              reinterpret_cast<uintptr_t>((lane ? m.b : m.s) + e * m.sb_stride + static_cast<size_t>(r0) * ngd);
          const int ns = static_cast<int>(((s0 & 127) + static_cast<uintptr_t>(nr) * ngd * 2 + 127) >> 7);
#pragma unroll 1
          for (int t = 0; t < ns; ++t) prefetch_line_l2(reinterpret_cast<const void*>((s0 & ~uintptr_t(127)) + 128u * t));
        }
      }
    }
    __syncthreads();  // the scales are in shared memory

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
    if (tid < npc) {
      const int P = gp0 + tid;
      const int j = P < k * I ? (P >> lgI) : k;
      const int i = P - (j << lgI);
      const float h = silu_f(guv[tid]) * guv[cv.npc_max + tid];
#pragma unroll
      for (int r = 0; r < kDecodeReplicas; ++r)
        st_word(p.hbuf + r * p.h_rep + static_cast<size_t>(j) * I + i, tag_f32(h, par));
    }
    stamp(4);

    // ---------------- 5a. this CTA's down rows, L2 hits by now, into the (now free) gate/up
    // buffer, issued before the wait on h
    issue_down(Ld);

    // ---------------- 5b. every slot's h, by down code segment
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
            hv[u] = ld_words4(h_in + 4 * ci);
            ok &= ((hv[u].x & hv[u].y & hv[u].z & hv[u].w & 1u) == par) && (((hv[u].x | hv[u].y | hv[u].z | hv[u].w) & 1u) == par);
          }
        }
        if (ok) break;
        MOE_POLL_BACKOFF(it, t0, p.hdr, 22, ab)
      }
      cp_async_wait_all();  // this thread's down copies (visible to all after the barrier below)
#pragma unroll
      for (int u = 0; u < kHChunks; ++u) {
        const int ci = tid + u * kThreads;
        if (ci < nch) {
          const int j = (4 * ci) >> lgI, i = (4 * ci) & (I - 1);
          const int s = i / PS;
          float* hj = hs + static_cast<size_t>(j) * I;
          const uint32_t hw[4] = {hv[u].x, hv[u].y, hv[u].z, hv[u].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int op = seg_pos<BITS>((i + e) % PS);
            hj[((op >> 2) * nsgd + s) * 4 + (op & 3)] = __uint_as_float(hw[e]);
          }
        }
      }
    }
    if (__syncthreads_or(ab)) { leave(); return; }
    stamp(5);

    // ---------------- 5c. down rows of every slot for this CTA's output rows
    {
      const uint4* dcodes = reinterpret_cast<const uint4*>(dnbuf);
      const uint16_t* dscl = reinterpret_cast<const uint16_t*>(dnbuf + cv.dsc);
      const int off = r0 * ngd - ((r0 * ngd) & ~7);
      const int dg = (ds * PS) >> lgG;
      int cur = -1;
      float hv[PS];
      float hsm = 0.f;
      // two units of the same slot at a time where possible (independent work in flight)
      int u = dn_u0;
#pragma unroll 1
      while (u < dn_u1) {
        const int j = u / dn_upj, t = u - j * dn_upj;
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
        const int nu = (u + 1 < dn_u1 && t + 1 < dn_upj) ? 2 : 1;  // warp-uniform
        float part[2] = {0.f, 0.f};
        int rlv[2];
#pragma unroll
        for (int v = 0; v < 2; ++v) {
          const int rl = (t + v) * rpsd + dsub;
          rlv[v] = rl;
          if (v < nu && rl < nr) {
            const int ei = off + rl * ngd + dg;
            part[v] = fmaf(bf16_to_f32(dscl[2 * j * cv.d_sc_el + ei]), dot_seg_dec<BITS>(dcodes[(u + v) * 32 + lane], hv),
                           bf16_to_f32(dscl[(2 * j + 1) * cv.d_sc_el + ei]) * hsm);
          }
        }
#pragma unroll 1
        for (int o = nsgd >> 1; o > 0; o >>= 1) {
          part[0] += __shfl_xor_sync(0xffffffffu, part[0], o);
          part[1] += __shfl_xor_sync(0xffffffffu, part[1], o);
        }
        if (ds == 0) {
          if (rlv[0] < nr) dred[j * cv.nr_max + rlv[0]] = part[0];
          if (nu == 2 && rlv[1] < nr) dred[j * cv.nr_max + rlv[1]] = part[1];
        }
        u += nu;
      }
    }
    if (__syncthreads_or(ab)) { leave(); return; }
    if (tid < nr) {
      const int row = r0 + tid;
      float acc = 0.f;
#pragma unroll 1
      for (int j = 0; j < k; ++j) acc = fmaf(s_w[j], dred[j * cv.nr_max + tid], acc);
      if (Is > 0) acc = fmaf(s_sg, dred[k * cv.nr_max + tid], acc);
      const uint16_t yb = f32_to_bf16(acc);
#pragma unroll
      for (int r = 0; r < kDecodeReplicas; ++r)
        st_word(p.ybuf + r * p.y_rep + row, (static_cast<uint32_t>(yb) << 16) | (tag & 0xffffu));
      if (p.tr_y) p.tr_y[static_cast<size_t>(lg) * p.tr_rows * H + row] = yb;
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
        w = ld_words4(y_in + i4);
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

// Both forms of bounded wait this file uses, run on things that never
// happen: warp 0 polls a word nothing writes (MOE_POLL_BACKOFF / give_up),
// warp 1 waits on an mbarrier nobody arrives at (mbar_wait_slow). Each must
// give up within the library's limits, record MOE_ERR_TIMEOUT and return;
// bit 0 / bit 1 of *gave_up say which of the two ended without its event.
__global__ void __launch_bounds__(64) wait_limit_kernel(WsHeader* hdr, uint32_t* never_set, int32_t* gave_up) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int s_mask;
  const int tid = threadIdx.x;
  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    s_mask = 0;
  }
  __syncthreads();
  if (tid == 0) {
    bool fail = false;
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
      if (ld_word(never_set) != 0u) break;
      MOE_POLL_BACKOFF(it, t0, hdr, 91, fail);
    }
    if (fail) atomicOr(&s_mask, 1);
  } else if (tid == 32) {
    if (!mbar_wait_slow(&bar, 0, hdr, 92)) atomicOr(&s_mask, 2);
  }
  __syncthreads();
  if (tid == 0) *gave_up = s_mask;
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
  if (ch == 3) return launch_t<8, 3>(p, smem, grid, stream);  // 1536-wide 8-bit rows
  return launch_t<8, 4>(p, smem, grid, stream);
}

cudaError_t launch_wait_limit_check(WsHeader* hdr, uint32_t* never_set, int32_t* gave_up, cudaStream_t stream) {
  wait_limit_kernel<<<1, 64, 0, stream>>>(hdr, never_set, gave_up);
  return cudaGetLastError();
}

}  // namespace moe
