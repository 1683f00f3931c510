// Persistent single-token decode of a whole MoE stack in one launch, with
// each CTA's part of h kept inside the CTA ("split" over the intermediate).
//
// One CTA per SM, all co-resident (cooperative launch), walks every layer:
//   1. residual + parameter-free RMSNorm of the previous layer's output
//      (every CTA redundantly, identical arithmetic), giving this layer's x,
//      kept as fp32 for the router and as a fixed-point integer vector for
//      the expert dot products (below);
//   2. router rows: each CTA owns E/G rows of the router (plus the shared
//      expert's gate vector as row E), prefetched into shared memory by bulk
//      copies one layer ahead, and publishes their logits;
//   3. softmax + top-k in every CTA from all published logits (one warp),
//      which at once issues the bulk copies of its CTA's unit (4.);
//   4. the CTA's unit: 32 consecutive columns of one selected expert's
//      intermediate (the k*I + Is columns of the selected experts, one unit
//      per CTA, the remaining CTAs idle here). Its 32 packed gate/up row pairs
//      with their scales and biases land in shared memory in two batches of
//      16 pairs, the dot products run on integer dot-product instructions,
//      and SwiGLU gives the unit's 32 values of h;
//   5. the unit's 32 columns of all H down rows and their scales and biases
//      (bulk copies of the contiguous blocks that moe_prepare_down_units and
//      moe_prepare_down_sb lay out; without those copies, 256-row tiles of the
//      canonical codes by the tensor memory accelerator) are requested right
//      behind the gate/up batches, or, where they do not fit beside the
//      gate/up rows, into the first batch's space as soon as every warp is
//      done with it (the mid-copy mode). Thread t takes output rows t,
//      t + 512, ..., forms the unit's routing-weighted partial of y for them,
//      and adds it to a replicated fp32 accumulator (reductions in L2).
// The y of a layer is then the sum of the k*I/32 + Is/32 partials: no h
// exchange between CTAs, and no CTA reads more than its own unit of any
// expert. Routing fan-out and shared experts: Swiftlet article (xix.ai),
// paragraphs 4 and 8; Runnel README, "Target". Low-bit groups: same article,
// paragraph 8. Packed gate/up: Runnel README, introduction and "Streaming CLI".
//
// Integer dot products. A group's share of a row's dot product is
// s_g * sum(q x) + b_g * sum(x). The activations (x, and the unit's h) are
// turned into one fixed-point vector per layer: X_i = rint(x_i * 2^S) with S
// chosen from max|x| so that |X_i| < 2^22, which is exact for every x_i
// within 14 binades of the largest (bf16 x has 8 significant bits; h is
// rounded to 22 bits below its largest element, finer than an fp32 sum of
// the products). X is split into three bytes, X = 65536*X2 + 256*X1 + X0
// (X2 signed, X1 and X0 unsigned), and sum(q X) is three exact integer sums
// of byte products (dp4a: four byte products and an add per instruction),
// recombined in fp32 once per 16-byte segment of codes and scaled back by
// 2^-S. 4-bit codes are split into even and odd nibbles as bytes first (two
// masks), so x is laid out in the same even/odd order.
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
constexpr int kNB = kUnit / kBatch;           // batches per unit
constexpr int kTopPer = 16;                   // logits per lane in the top-k warp: E <= 512
constexpr int kBoxRows = 256;                 // down rows per tensor copy
constexpr int kQ = 24;                        // u32 words of fixed-point quads per 32 codes (8 quads x 3 bytes)

__host__ __device__ constexpr uint32_t al128(uint32_t v) { return (v + 127u) & ~127u; }
__host__ __device__ constexpr int cdiv(int a, int b) { return (a + b - 1) / b; }

// Shared-memory carve-up; identical on host (sizing) and device.
struct Carve {
  int PS, nsg, QS, QSP, ng, ngd, rowb, rr_max, HT, UB;
  uint32_t xn, xq, hq, guv, gsb, gcd, dcd, dhi, dsb, dcd2, dsb2, rbuf, desc, total;
};

__host__ __device__ inline Carve carve(int H, int E, int I, int Is, int group, int bits, int G, int L, int late,
                                       int two) {
  Carve c{};
  c.PS = 128 / bits;          // codes per 16-byte segment
  c.nsg = H / c.PS;           // segments per gate/up row
  c.QS = 3 * (c.PS / 4);      // quad words of x per segment (3 bytes x PS/4 quads)
  c.QSP = c.QS + 1;           // + the segment's sum of X (odd stride: conflict-free by segment)
  c.ng = H / group;
  c.ngd = I / group;
  c.rowb = H * bits / 8;
  c.rr_max = cdiv(E + (Is > 0 ? 1 : 0), G);
  c.HT = H / 4;
  c.UB = kUnit * bits / 8;  // bytes of one down row inside the unit
  uint32_t o = 0;
  c.xn = o;    o = al128(o + H * 4);                       // x, fp32, natural order (router)
  c.xq = o;    o = al128(o + c.QSP * c.nsg * 4);           // x quads [nsg][QS] + sum of X, per segment
  c.hq = o;    o = al128(o + kQ * 4);                      // the unit's h quads
  c.guv = o;   o = al128(o + 2 * kUnit * 4);
  c.gsb = o;   o = al128(o + 4 * kUnit * c.ng * 2);        // [gate sc, up sc, gate bi, up bi][pair][ng]
  const uint32_t gu_bytes = 2 * kUnit * c.rowb;             // [gate|up][pair][rowb]
  c.gcd = o;   o = al128(o + gu_bytes);
  if (late) {
    // mid-copy mode: down rows [0, H/2) take the first batch's gate rows, [H/2, H) its up rows
    // (H/2 rows of 32 codes are exactly 16 rows of H codes)
    c.dcd = c.gcd;
    c.dhi = c.gcd + kUnit * c.rowb;
  } else {
    c.dcd = o;  o = al128(o + H * c.UB);
    c.dhi = c.dcd + (H / 2) * c.UB;
  }
  c.dsb = o;   o = al128(o + H * 4);                       // down (scale, bias) of the unit's group, [H][2]
  if (two) {  // a CTA with a second unit: its down data has a buffer of its own
    c.dcd2 = o;  o = al128(o + H * c.UB);
    c.dsb2 = o;  o = al128(o + H * 4);
  }
  c.rbuf = o;  o = al128(o + 2 * c.rr_max * H * 2);
  c.desc = o;  o = al128(o + L * sizeof(LayerDesc));       // the launch's layer descriptors
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

// Top-k of one token's logits by one warp for 16 logits per lane (E <= 512): the lane's logits of
// experts lane + 32i, i < 8 and i >= 8, are sorted as two lists of 8 (larger logit first, then
// lower expert index); each round the lane offers the better of its two heads, one warp-wide max
// picks the winner (lowest index among equal keys) and its lane pops that head. Lane j < k ends
// with the j-th pick. The same result as topk_sorted<16>, with two 8-sorts instead of a 16-sort.
__device__ __forceinline__ void topk_halves(const uint32_t* wl, int E, int k, int lane, unsigned& my_k, int& my_e,
                                            unsigned& kmax) {
  unsigned ka[8], kb[8];
  int ia[8], ib[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    ia[i] = lane + 32 * i;
    ib[i] = lane + 32 * (i + 8);
    ka[i] = (ia[i] < E) ? fkey(__uint_as_float(wl[i])) : 0u;
    kb[i] = (ib[i] < E) ? fkey(__uint_as_float(wl[i + 8])) : 0u;
  }
  auto sort8 = [](unsigned (&key)[8], int (&idx)[8]) {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
#pragma unroll
      for (int i = (r & 1); i + 1 < 8; i += 2) {
        const bool sw = key[i + 1] > key[i] || (key[i + 1] == key[i] && idx[i + 1] < idx[i]);
        const unsigned k0 = key[i], k1 = key[i + 1];
        const int i0 = idx[i], i1 = idx[i + 1];
        key[i] = sw ? k1 : k0;
        key[i + 1] = sw ? k0 : k1;
        idx[i] = sw ? i1 : i0;
        idx[i + 1] = sw ? i0 : i1;
      }
    }
  };
  sort8(ka, ia);
  sort8(kb, ib);
  my_k = 0u;
  my_e = 0;
  kmax = 0u;
#pragma unroll 1
  for (int j = 0; j < k; ++j) {
    const bool fb = kb[0] > ka[0] || (kb[0] == ka[0] && ib[0] < ia[0]);  // the lane's better head
    const unsigned hk = fb ? kb[0] : ka[0];
    const int hi = fb ? ib[0] : ia[0];
    const unsigned wk = __reduce_max_sync(0xffffffffu, hk);
    const unsigned we = __reduce_min_sync(0xffffffffu, hk == wk ? static_cast<unsigned>(hi) : 0xffffffffu);
    if (j == 0) kmax = wk;
    if (lane == j) {
      my_k = wk;
      my_e = static_cast<int>(we);
    }
    if (static_cast<unsigned>(hi) == we) {  // the owner pops the head it offered
      if (fb) {
#pragma unroll
        for (int i = 0; i + 1 < 8; ++i) {
          kb[i] = kb[i + 1];
          ib[i] = ib[i + 1];
        }
        kb[7] = 0u;
      } else {
#pragma unroll
        for (int i = 0; i + 1 < 8; ++i) {
          ka[i] = ka[i + 1];
          ia[i] = ia[i + 1];
        }
        ka[7] = 0u;
      }
    }
  }
}

// One unit of work: 32 consecutive columns of one slot's intermediate.
struct Unit {
  int j;       // slot: 0..k-1 the selected experts in rank order, k the shared expert
  int i0;      // first column inside the slot
  int g;       // its quantisation group along the down rows
  bool routed;
};

__device__ __forceinline__ Unit unit_of(int u, int k, int I, int group) {
  const int gp0 = u * 32;
  Unit U;
  U.j = gp0 < k * I ? gp0 / I : k;
  U.i0 = gp0 - (U.j < k ? U.j * I : k * I);
  U.g = U.i0 / group;
  U.routed = U.j < k;
  return U;
}

// Copy-phase bookkeeping for leaving early: parities of the phases this CTA
// still has bulk copies in flight on (-1 = none).
struct Pending {
  int r[2], gc, dn[2];
};

__device__ __noinline__ void drain(Pending* pend, uint64_t* bar_r, uint64_t* bar_gc, uint64_t* bar_dn, int nb,
                                   WsHeader* hdr) {
  __syncthreads();
  if (threadIdx.x == 0) {
    if (pend->r[0] >= 0) mbar_wait(&bar_r[0], pend->r[0], hdr, 90);
    if (pend->r[1] >= 0) mbar_wait(&bar_r[1], pend->r[1], hdr, 91);
    if (pend->gc >= 0)
      for (int b = 0; b < nb; ++b) mbar_wait(&bar_gc[b], pend->gc, hdr, 94);
    if (pend->dn[0] >= 0) mbar_wait(&bar_dn[0], pend->dn[0], hdr, 95);
    if (pend->dn[1] >= 0) mbar_wait(&bar_dn[1], pend->dn[1], hdr, 96);
  }
  __syncthreads();
}

template <int BITS, int CH, bool TWO>
__global__ void __launch_bounds__(kThreads, 1) decode_split_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int PS = 128 / BITS;  // codes per 16-byte segment
  constexpr int QW = PS / 4;      // quads per segment per byte plane
  extern __shared__ __align__(128) unsigned char sm[];
  __shared__ __align__(8) uint64_t bar_r[2];
  __shared__ __align__(8) uint64_t bar_gc[kNB];
  __shared__ __align__(8) uint64_t bar_dn[2];  // down data of the CTA's first and second unit
  __shared__ int s_idx[16];
  __shared__ float s_w[16];
  __shared__ float s_sg;
  __shared__ float s_red[2][kWarps];
  __shared__ float s_hx[2];  // the unit's sum of X_h, and 2^-S_h
  __shared__ int s_b0;       // mid-copy mode: warps done with the first gate/up batch
  __shared__ Pending s_pend;

  const int H = p.H, E = p.E, k = p.k, I = p.I, Is = p.Is, group = p.group;
  const int G = gridDim.x, c = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  bool ab = false;  // a wait of this thread gave up; combined over the CTA at each phase end
  const Carve cv = carve(H, E, I, Is, group, BITS, G, p.L, p.split_late, p.split_two);
  float* xn = reinterpret_cast<float*>(sm + cv.xn);
  uint32_t* xq = reinterpret_cast<uint32_t*>(sm + cv.xq);
  uint32_t* hq = reinterpret_cast<uint32_t*>(sm + cv.hq);
  float* guv = reinterpret_cast<float*>(sm + cv.guv);
  uint16_t* gsb = reinterpret_cast<uint16_t*>(sm + cv.gsb);
  unsigned char* gcd = sm + cv.gcd;
  unsigned char* dcd = sm + cv.dcd;    // down rows [0, H/2)
  unsigned char* dhi = sm + cv.dhi;    // down rows [H/2, H)
  const int H2 = H / 2;
  const uint32_t* dsb = reinterpret_cast<const uint32_t*>(sm + cv.dsb);
  uint16_t* rbuf = reinterpret_cast<uint16_t*>(sm + cv.rbuf);
  const LayerDesc* s_layers = reinterpret_cast<const LayerDesc*>(sm + cv.desc);

  // ---- static assignment of this CTA's work: units c and c + G (where they exist) of the
  // flattened (slot, column) space cut into 32-column units, slot j at [j * I, (j + 1) * I), the
  // shared expert last. A CTA with two units does them one after the other.
  const int NU = (k * I + Is) / kUnit;
  const int nu = (c < NU ? 1 : 0) + (TWO && c + G < NU ? 1 : 0);
  const bool has_unit = nu > 0;
  const Unit U0 = unit_of(c, k, I, group);
  const Unit U1 = unit_of(c + G, k, I, group);
  const int nrows_rt = E + (Is > 0 ? 1 : 0);
  const int rr_cnt = (c < nrows_rt) ? cdiv(nrows_rt - c, G) : 0;
  const uint32_t* lg_in = p.logits + (c % kDecodeReplicas) * p.logits_rep;  // this CTA's copy of the logits
  const int rowb = cv.rowb, ng = cv.ng, HT = cv.HT, nsg = cv.nsg;
  const int lgG = 31 - __clz(group);  // group is a power of two
  const int nb = has_unit ? kNB : 0;

  if (tid == 0) {
    mbar_init(&bar_r[0], 1);
    mbar_init(&bar_r[1], 1);
    for (int b = 0; b < kNB; ++b) mbar_init(&bar_gc[b], 1);
    mbar_init(&bar_dn[0], 1);
    mbar_init(&bar_dn[1], 1);
    fence_mbar_init();
    s_pend.r[0] = s_pend.r[1] = s_pend.gc = s_pend.dn[0] = s_pend.dn[1] = -1;
    s_b0 = 0;
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
  auto leave = [&]() { drain(&s_pend, bar_r, bar_gc, bar_dn, nb, p.hdr); };

  if (tid == 0) issue_router(0);

  // lane roles in the gate/up dot products: a row of nsg 16-byte code segments is
  // covered by 32/nsg rows per warp step (nsg < 32) or by CH segments per lane
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
  // thread 0: wait until `target` arrivals are in (acquire loads: what the arriving CTAs wrote
  // before their release arrivals is visible after)
  auto wait_arrivals = [&](uint32_t target, int where) {
    if (tid != 0) return;
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
      uint32_t v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p.arrive) : "memory");
      if (v >= target) break;
      MOE_POLL_BACKOFF(it, t0, p.hdr, where, ab)
    }
  };
  // block-wide sum of a and max of b (all threads call; every thread gets both)
  auto block_sum_max = [&](float a, float b, float& sa, float& mb) {
    a = warp_sum(a);
    b = warp_max(b);
    if (lane == 0) {
      s_red[0][warp] = a;
      s_red[1][warp] = b;
    }
    __syncthreads();
    sa = 0.f;
    mb = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      sa += s_red[0][w];
      mb = fmaxf(mb, s_red[1][w]);
    }
  };

  // a unit's down data (one thread) into down buffer `db` (0, or 1 for a CTA's second unit): its
  // 32 columns of all H down rows (one contiguous block of the unit-major copy, else 256-row tiles
  // of the canonical codes) and the (scale, bias) pairs of its group for all H rows from the
  // group-major copy (when the layer has one; else the down phase reads the canonical layout)
  auto issue_down = [&](const LayerDesc& Ld, int l, const Unit& U, int e, int db) {
    const uint16_t* sbm = U.routed ? Ld.dsb : Ld.sdsb;
    const uint8_t* cdm = U.routed ? Ld.dcu : Ld.sdcu;
    const size_t eu = U.routed ? e : 0;
    unsigned char* lo = db ? sm + cv.dcd2 : dcd;
    unsigned char* hi = db ? sm + cv.dcd2 + H2 * cv.UB : dhi;
    uint64_t* bar = &bar_dn[db];
    // the buffers may last have been read by ordinary loads (gate/up or the previous layer's down)
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(H) * (cv.UB + (sbm ? 4 : 0)));
    if (cdm) {  // the unit's 32 columns of all rows: one contiguous block, in two halves
      const uint8_t* src = cdm + ((eu * (U.routed ? I : Is) / kUnit) + U.i0 / kUnit) * H * cv.UB;
      bulk_g2s(lo, src, static_cast<uint32_t>(H2) * cv.UB, bar);
      bulk_g2s(hi, src + static_cast<size_t>(H2) * cv.UB, static_cast<uint32_t>(H2) * cv.UB, bar);
    } else {
      const CUtensorMap* tm = U.routed ? &p.tm_dn[l] : &p.tm_sdn[l];
#pragma unroll 1
      for (int r0 = 0; r0 < H; r0 += kBoxRows)
        tma_3d(r0 < H2 ? lo + r0 * cv.UB : hi + (r0 - H2) * cv.UB, tm, U.i0 * BITS / 8, r0, static_cast<int>(eu), bar);
    }
    if (sbm)
      bulk_g2s(sm + (db ? cv.dsb2 : cv.dsb), sbm + (eu * cv.ngd + U.g) * H * 2, static_cast<uint32_t>(H) * 4, bar);
    s_pend.dn[db] = l & 1;
  };

  // a unit's gate/up data (one whole warp, converged): batch 0's code rows with the scales and
  // biases of the whole unit, then batch 1's code rows, completing phase `gpar` of the batch
  // barriers; then (unless in mid-copy mode) its down data into down buffer db
  auto issue_unit = [&](const LayerDesc& Ld, int l, const Unit& U, int e, int gpar, int db) {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    const QMat& mq = U.routed ? Ld.gu : Ld.sgu;
    const int iA = U.i0;
    const uint8_t* qb = mq.q + static_cast<size_t>(e) * mq.q_stride;
    const uint16_t* sb = mq.s + static_cast<size_t>(e) * mq.sb_stride;
    const uint16_t* bb = mq.b + static_cast<size_t>(e) * mq.sb_stride;
    const uint32_t cb = static_cast<uint32_t>(kBatch) * rowb, sbb = static_cast<uint32_t>(kUnit) * ng * 2;
#pragma unroll 1
    for (int b = 0; b < kNB; ++b) {
      const int r0 = iA + b * kBatch;  // first gate row of the batch; its up row r0 starts at up_q
      if (lane == 0) mbar_arrive_expect_tx(&bar_gc[b], 2 * cb + (b == 0 ? 4 * sbb : 0u));
      __syncwarp();
      if (lane < (b == 0 ? 6 : 2)) {
        const int gu = lane & 1, kind = lane >> 1;  // kind 0 codes, 1 scales, 2 biases
        if (kind == 0)
          bulk_g2s(gcd + static_cast<size_t>(gu * kUnit + b * kBatch) * rowb,
                   qb + (gu ? mq.up_q : 0) + static_cast<size_t>(r0) * rowb, cb, &bar_gc[b]);
        else
          bulk_g2s(gsb + static_cast<size_t>(((kind - 1) * 2 + gu) * kUnit) * ng,
                   (kind == 1 ? sb + (gu ? mq.up_s : 0) : bb + (gu ? mq.up_b : 0)) + static_cast<size_t>(iA) * ng, sbb, &bar_gc[b]);
      }
    }
    if (lane == 0) {
      s_pend.gc = gpar;
      if (!p.split_late) issue_down(Ld, l, U, e, db);
    }
    __syncwarp();
  };

  float rr4[4] = {0.f, 0.f, 0.f, 0.f};  // residual stream, rows 4t .. 4t+3 (t < H/4)
  uint32_t gph = 0;  // completed phases of the gate/up batch barriers (one per unit processed)

  for (int l = 0; l < p.L; ++l) {
    const int lg = p.l0 + l;  // layer index within the whole stack (trace rows)
    const uint32_t tag = static_cast<uint32_t>(l + 1);
    const uint32_t par = tag & 1u;
    auto stamp = [&](int slot) {
      if (p.tr_t && c == 0 && tid == 0) p.tr_t[static_cast<size_t>(lg) * 8 + slot] = globaltimer_ns();
    };
    stamp(0);

    // ---------------- 1. this layer's x (and residual), fp32 and fixed point
    float xv[4] = {0.f, 0.f, 0.f, 0.f};
    float m;
    if (l == 0) {
      float mx = 0.f;
      if (tid < HT) {
        const uint2 w = *reinterpret_cast<const uint2*>(p.x0 + 4 * tid);
        xv[0] = bf16_lo(w.x);
        xv[1] = bf16_hi(w.x);
        xv[2] = bf16_lo(w.y);
        xv[3] = bf16_hi(w.y);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          rr4[u] = p.r_in ? p.r_in[4 * tid + u] : xv[u];
          mx = fmaxf(mx, fabsf(xv[u]));
        }
        if (c == 0 && p.tr_x) *reinterpret_cast<uint2*>(p.tr_x + static_cast<size_t>(p.l0) * p.tr_rows * H + 4 * tid) = w;
      }
      float unused;
      block_sum_max(0.f, mx, unused, m);
    } else {
      wait_arrivals(static_cast<uint32_t>(G) * static_cast<uint32_t>(l), 20);
      if (__syncthreads_or(ab)) { leave(); return; }
      float ss = 0.f, mx = 0.f;
      if (tid < HT) {
        float y[4];
        read_y(l - 1, y);
        uint16_t yb[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          yb[u] = f32_to_bf16(y[u]);
          rr4[u] += bf16_to_f32(yb[u]);
          ss = fmaf(rr4[u], rr4[u], ss);
          mx = fmaxf(mx, fabsf(rr4[u]));
        }
        if (c == 0 && p.tr_y)
          *reinterpret_cast<uint2*>(p.tr_y + static_cast<size_t>(lg - 1) * p.tr_rows * H + 4 * tid) =
              make_uint2(yb[0] | (static_cast<uint32_t>(yb[1]) << 16), yb[2] | (static_cast<uint32_t>(yb[3]) << 16));
      }
      float tot;
      block_sum_max(ss, mx, tot, m);
      const float inv = 1.f / sqrtf(tot / static_cast<float>(H) + p.eps);
      m *= inv;
      // bf16 rounding of the largest |r * inv| can reach the next power of two: fix_exp leaves one bit for it
      if (tid < HT) {
        uint16_t xb[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          xb[u] = f32_to_bf16(rr4[u] * inv);
          xv[u] = bf16_to_f32(xb[u]);
        }
        if (c == 0 && p.tr_x)
          *reinterpret_cast<uint2*>(p.tr_x + static_cast<size_t>(lg) * p.tr_rows * H + 4 * tid) =
              make_uint2(xb[0] | (static_cast<uint32_t>(xb[1]) << 16), xb[2] | (static_cast<uint32_t>(xb[3]) << 16));
      }
    }
    const int S = fix_exp(m);
    const float sx = pow2f(S), isx = pow2f(-S);
    if (tid < HT) {
      *reinterpret_cast<float4*>(xn + 4 * tid) = make_float4(xv[0], xv[1], xv[2], xv[3]);
    }
    __syncthreads();
    if (tid == kThreads - 32 && l + 1 < p.L) issue_router(l + 1);  // a warp without router rows
    stamp(1);

    // ---------------- 2. router rows -> logits
    if (warp < rr_cnt) {
      if (!mbar_ready(&bar_r[l & 1], (l >> 1) & 1, p.hdr, 10)) ab = true;
      const int row = c + warp * G;
      const uint4* wv = reinterpret_cast<const uint4*>(rbuf + (static_cast<size_t>(l & 1) * cv.rr_max + warp) * H);
      float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
#pragma unroll 4
      for (int s = lane; s < H / 8; s += 32) {
        const uint4 w8 = wv[s];
        const float4 a = reinterpret_cast<const float4*>(xn)[2 * s];
        const float4 b = reinterpret_cast<const float4*>(xn)[2 * s + 1];
        acc0 = fmaf(bf16_lo(w8.x), a.x, acc0);
        acc1 = fmaf(bf16_hi(w8.x), a.y, acc1);
        acc2 = fmaf(bf16_lo(w8.y), a.z, acc2);
        acc3 = fmaf(bf16_hi(w8.y), a.w, acc3);
        acc0 = fmaf(bf16_lo(w8.z), b.x, acc0);
        acc1 = fmaf(bf16_hi(w8.z), b.y, acc1);
        acc2 = fmaf(bf16_lo(w8.w), b.z, acc2);
        acc3 = fmaf(bf16_hi(w8.w), b.w, acc3);
      }
      const float acc = warp_sum((acc0 + acc1) + (acc2 + acc3));
      const LayerDesc& Ld = s_layers[l];
      if (lane < kDecodeReplicas)
        st_word(p.logits + lane * p.logits_rep + row, tag_f32(acc + ((row < E && Ld.rbias) ? Ld.rbias[row] : 0.f), par));
    }
    if (tid == 0) s_pend.r[l & 1] = -1;
    stamp(2);
    // this layer's x in fixed point (needed from the gate/up phase on, after the top-k barrier)
    if (tid < HT) {
      // fixed point; this thread's rows 4t..4t+3 give one quad of every byte plane
      int X[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) X[u] = __float2int_rn(xv[u] * sx);
      int xs = (X[0] + X[1]) + (X[2] + X[3]);
      int e[4], qi, sg;
      if constexpr (BITS == 4) {
        // rows 4t..4t+3 are positions 4h..4h+3 of word w (h = t & 1) of segment t / 8: thread h = 0
        // builds the word's even quad (its positions 0, 2 and the partner's 4, 6), h = 1 the odd
        // quad (the partner's positions 1, 3 and its own 5, 7)
        const int h = tid & 1;
        const int r0 = __shfl_xor_sync(0xffffffffu, h ? X[0] : X[1], 1);
        const int r1 = __shfl_xor_sync(0xffffffffu, h ? X[2] : X[3], 1);
        e[0] = h ? r0 : X[0];
        e[1] = h ? r1 : X[2];
        e[2] = h ? X[1] : r0;
        e[3] = h ? X[3] : r1;
        qi = ((tid >> 1) & 3) * 2 + h;
        sg = tid >> 3;
      } else {
        e[0] = X[0];
        e[1] = X[1];
        e[2] = X[2];
        e[3] = X[3];
        qi = tid & 3;
        sg = tid >> 2;
      }
#pragma unroll
      for (int j = 0; j < 3; ++j)
        xq[sg * cv.QSP + j * QW + qi] =
            xbyte(e[0], j) | (xbyte(e[1], j) << 8) | (xbyte(e[2], j) << 16) | (xbyte(e[3], j) << 24);
      // PS / 4 threads per segment
#pragma unroll
      for (int o = 1; o < PS / 4; o <<= 1) xs += __shfl_xor_sync(0xffffffffu, xs, o);
      if ((tid & (PS / 4 - 1)) == 0) xq[sg * cv.QSP + cv.QS] = __float_as_uint(static_cast<float>(xs));
    }


    // ---------------- 3. softmax + top-k (every CTA, warp 0), then the unit's copies
    const LayerDesc& Ld = s_layers[l];
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
      else topk_halves(wl, E, k, lane, my_k, my_e, kmax);
      // the unit's copies, at once (lane jA holds slot jA's pick). Issuing a routed unit's copies in
      // the round that picks its expert, or the shared expert's one layer ahead, measured slower:
      // their traffic delays the other CTAs' polls of the logits
      if (has_unit && !__any_sync(0xffffffffu, ab))  // warp-uniform: issue_unit has __syncwarp
        issue_unit(Ld, l, U0, U0.routed ? __shfl_sync(0xffffffffu, my_e, U0.j) : 0, gph & 1, 0);
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
    if (tid >= 32) {
      // this CTA's slice of the accumulators of layer l + 1
      const int nz = kDecodeReplicas * p.yrep;
      uint32_t* zb = reinterpret_cast<uint32_t*>(p.yacc + static_cast<size_t>((l + 1) % kDecodeYBufs) * p.ybuf_stride);
      const int z1 = static_cast<int>(static_cast<int64_t>(c + 1) * nz / G);
#pragma unroll 1
      for (int i = static_cast<int>(static_cast<int64_t>(c) * nz / G) + tid - 32; i < z1; i += kThreads - 32)
        st_word(zb + i, 0u);
    }

    // ---------------- 4./5. the CTA's units in turn (a lambda: without TWO it is called once, with
    // ui = 0, so that the single-unit kernel is straight-line code); false = leave the kernel
    auto unit_body = [&](const int ui, const Unit& U) -> bool {
      // ---------------- 4. gate/up rows + SwiGLU, batch by batch as the codes land
      {
        uint32_t xr[CH][3 * QW];  // this lane's segments of X, by byte plane
        float xsm[CH];
#pragma unroll
        for (int ch = 0; ch < CH; ++ch) {
          const int s = gs0 + 32 * ch;
#pragma unroll
          for (int q = 0; q < 3 * QW; ++q) xr[ch][q] = xq[s * cv.QSP + q];
          xsm[ch] = __uint_as_float(xq[s * cv.QSP + cv.QS]);
        }
#pragma unroll 1
        for (int b = 0; b < kNB; ++b) {
          if (warp * rps >= 2 * kBatch) continue;  // no row of this batch for this warp
          if (!mbar_ready(&bar_gc[b], gph & 1, p.hdr, 12)) ab = true;
          if (b == 0) stamp(4);
          // two rows of the batch at a time (rows rw and rw + 16 * rps), for independent work in flight
#pragma unroll 1
          for (int rw = warp * rps; rw < 2 * kBatch; rw += 2 * kWarps * rps) {
            float acc[2];
            int gi[2];
#pragma unroll
            for (int r2 = 0; r2 < 2; ++r2) {
              const int rho = rw + r2 * kWarps * rps + gsub;  // [0, 16) gate rows, [16, 32) up rows of the batch
              const int gu = rho >= kBatch ? 1 : 0;
              const int q = b * kBatch + rho - gu * kBatch;  // pair within the unit
              gi[r2] = rho < 2 * kBatch ? gu * kUnit + q : -1;
              acc[r2] = 0.f;
              if (rho < 2 * kBatch) {
                const unsigned char* row = gcd + static_cast<size_t>(gu * kUnit + q) * rowb;
                const uint16_t* sc = gsb + static_cast<size_t>(gu * kUnit + q) * ng;
                const uint16_t* bi = gsb + static_cast<size_t>((2 + gu) * kUnit + q) * ng;
#pragma unroll
                for (int ch = 0; ch < CH; ++ch) {
                  const int s = gs0 + 32 * ch;
                  const uint4 cd = *reinterpret_cast<const uint4*>(row + 16 * s);
                  const int g = (s * PS) >> lgG;
                  const float d = seg_dot<BITS>(cd, xr[ch] + 2 * QW, xr[ch] + QW, xr[ch]);
                  acc[r2] = fmaf(bf16_to_f32(sc[g]), d, fmaf(bf16_to_f32(bi[g]), xsm[ch], acc[r2]));
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
              if (gi[0] >= 0) guv[gi[0]] = acc[0] * isx;
              if (gi[1] >= 0) guv[gi[1]] = acc[1] * isx;
            }
          }
          if (p.split_late && b == 0) {
            // mid-copy mode: the last warp done with the first batch's rows issues the down copies
            // into their space (the other warps go on with the second batch)
            __syncwarp();
            if (lane == 0) {
              __threadfence_block();
              const int nw0 = min(kWarps, cdiv(2 * kBatch, rps));
              if (atomicAdd(&s_b0, 1) == nw0 - 1) {
                __threadfence_block();
                s_b0 = 0;
                issue_down(s_layers[l], l, U, U.routed ? s_idx[U.j] : 0, 0);
              }
            }
          }
        }
      }
      const bool gu_failed = __syncthreads_or(ab);
      if (tid == 0) s_pend.gc = -1;
      ++gph;
      if (gu_failed) { leave(); return false; }
      // the second unit's copies go out as soon as the first's gate/up rows are read
      if (TWO && ui + 1 < nu && warp == 0) issue_unit(s_layers[l], l, U1, U1.routed ? s_idx[U1.j] : 0, gph & 1, 1);
      if (warp == 0) {
        // SwiGLU, then the unit's h in fixed point (its own exponent) as quads for the down rows
        const float h = silu_f(guv[lane]) * guv[kUnit + lane];
        const int Sh = fix_exp(warp_max(fabsf(h)));
        const int X = __float2int_rn(h * pow2f(Sh));
        int hs = X;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) hs += __shfl_xor_sync(0xffffffffu, hs, o);
        // one down row of the unit = 32 codes: 4-bit, one segment of 8 quads; 8-bit, two segments of 4
        const int qp = (BITS == 4) ? quad_pos<4>(lane) : lane;
        unsigned char* hqb = reinterpret_cast<unsigned char*>(hq);
#pragma unroll
        for (int j = 0; j < 3; ++j) hqb[(j * 8 + (qp >> 2)) * 4 + (qp & 3)] = static_cast<unsigned char>(xbyte(X, j));
        if (lane == 0) {
          s_hx[0] = static_cast<float>(hs);
          s_hx[1] = pow2f(-Sh);
        }
      }
      if (tid < HT && !mbar_ready(&bar_dn[ui], l & 1, p.hdr, 13)) ab = true;
      if (__syncthreads_or(ab)) { leave(); return false; }
      if (tid == 0) s_pend.dn[ui] = -1;
      stamp(5);

      // ---------------- 5. the unit's partial of y for rows t, t + 512, ... (a warp reads 32
      // consecutive rows of codes, and reduces into 32 consecutive words of y):
      // routing weight x 2^-S_h x (scale x codes . X_h + bias x sum X_h)
      {
        uint32_t hr[kQ];
#pragma unroll
        for (int q = 0; q < kQ; ++q) hr[q] = hq[q];
        const float hsX = s_hx[0];
        const float wgt = (U.routed ? s_w[U.j] : s_sg) * s_hx[1];
        const LayerDesc& Ld5 = s_layers[l];
        const bool gm = (U.routed ? Ld5.dsb : Ld5.sdsb) != nullptr;
        const QMat& dm = U.routed ? Ld5.dn : Ld5.sdn;
        const size_t sb0 = static_cast<size_t>(U.routed ? s_idx[U.j] : 0) * dm.sb_stride + U.g;
        const unsigned char* dlo = ui ? sm + cv.dcd2 : dcd;
        const unsigned char* dhh = ui ? sm + cv.dcd2 + H2 * cv.UB : dhi;
        const uint32_t* dsbu = ui ? reinterpret_cast<const uint32_t*>(sm + cv.dsb2) : dsb;
        float* yrow = p.yacc + static_cast<size_t>(l % kDecodeYBufs) * p.ybuf_stride +
                      static_cast<size_t>(c % kDecodeReplicas) * p.yrep;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int r = tid + q * kThreads;
          if (r < H) {
            float d;
            const unsigned char* drow = r < H2 ? dlo + r * cv.UB : dhh + (r - H2) * cv.UB;
            if constexpr (BITS == 4) {
              d = seg_dot<4>(*reinterpret_cast<const uint4*>(drow), hr + 16, hr + 8, hr);
            } else {
              d = seg_dot<8>(*reinterpret_cast<const uint4*>(drow), hr + 16, hr + 8, hr) +
                  seg_dot<8>(*reinterpret_cast<const uint4*>(drow + 16), hr + 20, hr + 12, hr + 4);
            }
            float sc, bi;
            if (gm) {
              const uint32_t sbw = dsbu[r];
              sc = bf16_lo(sbw);
              bi = bf16_hi(sbw);
            } else {
              sc = bf16_to_f32(__ldg(dm.s + sb0 + static_cast<size_t>(r) * cv.ngd));
              bi = bf16_to_f32(__ldg(dm.b + sb0 + static_cast<size_t>(r) * cv.ngd));
            }
            red_add(yrow + r, wgt * fmaf(sc, d, bi * hsX));
          }
        }
      }
      if (__syncthreads_or(ab)) { leave(); return false; }
      return true;
    };
    if constexpr (TWO) {
#pragma unroll 1
      for (int ui = 0; ui < nu; ++ui)
        if (!unit_body(ui, ui == 0 ? U0 : U1)) return;
    } else {
      if (has_unit && !unit_body(0, U0)) return;
    }

    stamp(6);
    // the arrival: a release reduction (this CTA's reductions and zeroes, ordered before it by
    // the barrier, are visible to whoever acquires the count)
    if (tid == 0) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(p.arrive) : "memory");
    stamp(7);
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
        rr4[u] += bf16_to_f32(yb);
        ss = fmaf(rr4[u], rr4[u], ss);
        if (p.tr_y) p.tr_y[static_cast<size_t>(p.l0 + p.L - 1) * p.tr_rows * H + 4 * tid + u] = yb;
      }
    }
    float tot, unused;
    block_sum_max(ss, 0.f, tot, unused);
    const float inv = 1.f / sqrtf(tot / static_cast<float>(H) + p.eps);
    if (tid < HT) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        p.out[4 * tid + u] = f32_to_bf16(rr4[u] * inv);
        if (p.r_out) p.r_out[4 * tid + u] = rr4[u];
      }
    }
  }
  leave();
}

template <int BITS, int CH, bool TWO>
cudaError_t launch_t(const DecodeParams& p, size_t smem, int grid, cudaStream_t stream) {
  auto kern = decode_split_kernel<BITS, CH, TWO>;
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
                       size_t* smem, int* late, int* two_out) {
  if (grid < 1 || L < 1) return false;
  if (L > kMaxDecodeLayers) L = kMaxDecodeLayers;
  const int PS = 128 / bits;
  const int nsg = H / PS;
  if (H % PS || H > 4 * kThreads || H % kBoxRows) return false;  // rows 4t..4t+3 per thread; whole tiles
  if (!(pow2(nsg) && nsg <= 32) && !(nsg % 32 == 0 && nsg / 32 <= (bits == 4 ? 2 : 4))) return false;
  if (Is != 0 && Is != I) return false;          // one down row length (and scale row) for every slot
  if (I % kUnit || !pow2(group) || group % kUnit || I % group) return false;  // a unit lies in one group
  if (k > 16 || E > 32 * kTopPer) return false;
  const int nunits = (k * I + Is) / kUnit;
  if (nunits > 2 * grid) return false;  // at most two units per CTA
  if (cdiv(E + (Is > 0 ? 1 : 0), grid) > kWarps) return false;  // one router row per warp
  const int two = nunits > grid ? 1 : 0;
  for (int lt = 0; lt < 2; ++lt) {  // down codes in a region of their own if they fit, else mid-copy mode
    if (lt == 1 && (two || H % (2 * kBoxRows))) break;  // the halves hold whole 256-row tiles; one unit
    const size_t need = carve(H, E, I, Is, group, bits, grid, L, lt, two).total;
    if (need <= smem_limit) {
      *smem = need;
      *late = lt;
      if (two_out) *two_out = two;
      return true;
    }
  }
  return false;
}

cudaError_t launch_decode_split(const DecodeParams& p, int bits, int grid, cudaStream_t stream) {
  const size_t smem = carve(p.H, p.E, p.I, p.Is, p.group, bits, grid, p.L, p.split_late, p.split_two).total;
  const int nsg = p.H * bits / 128;
  const int ch = nsg >= 32 ? nsg / 32 : 1;
  if (p.split_two) {  // more units than CTAs: the loop over a CTA's two units
    if (bits == 4) {
      if (ch == 1) return launch_t<4, 1, true>(p, smem, grid, stream);
      return launch_t<4, 2, true>(p, smem, grid, stream);
    }
    if (ch == 1) return launch_t<8, 1, true>(p, smem, grid, stream);
    if (ch == 2) return launch_t<8, 2, true>(p, smem, grid, stream);
    if (ch == 3) return launch_t<8, 3, true>(p, smem, grid, stream);
    return launch_t<8, 4, true>(p, smem, grid, stream);
  }
  if (bits == 4) {
    if (ch == 1) return launch_t<4, 1, false>(p, smem, grid, stream);
    return launch_t<4, 2, false>(p, smem, grid, stream);
  }
  if (ch == 1) return launch_t<8, 1, false>(p, smem, grid, stream);
  if (ch == 2) return launch_t<8, 2, false>(p, smem, grid, stream);
  if (ch == 3) return launch_t<8, 3, false>(p, smem, grid, stream);  // 1536-wide 8-bit rows
  return launch_t<8, 4, false>(p, smem, grid, stream);
}

}  // namespace moe
