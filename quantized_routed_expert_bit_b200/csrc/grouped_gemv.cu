// The batched path for a few tokens per expert: a grouped matrix-vector
// product on the CUDA cores. Tokens are grouped by expert (counting sort,
// sort_by_expert.cu, in chunks of at most kGvTPI pairs), and each chunk's
// expert weights are read once for all of the chunk's tokens, 32 columns of
// the intermediate (a unit) at a time:
//
//   xquant   every token's x as the fixed-point quads of the integer dot
//            products (X = rint(x * 2^S) in 16 bits, two byte planes: see
//            fix_exp16), per token its own S; also the shared expert's
//            sigmoid gate;
//   gemv     per work item (chunk, group of upi units, upi = 1, 2 or 4 as
//            gemv_units_per_item picks for the batch size): the item's
//            tokens' quads (bulk copies, issued while the previous item's
//            down rows are computed); for each unit, the 32 gate/up row pairs
//            and their scales and biases (bulk copies, two buffers so that
//            the next unit's rows stream in while this one is computed),
//            h = silu(gate) * up for each of the chunk's tokens, then the
//            unit's 32 columns of all H down rows (one contiguous block of
//            the unit-major down copy) against each token's h; each thread
//            keeps its rows' sums for every token of the chunk in registers
//            over the item's units and stores them once, as the item's
//            partial of each pair's expert output;
//   combine  y = sum_j w_j (sum over items of o_j) + gate * o_shared, rank
//            order, one bf16 rounding.
// With 1-4 tokens per expert (batches of up to about a hundred tokens over
// 256 experts) the tensor cores would multiply mostly padding; the dot
// products run as in the single-token decode kernel (stack_split.cu), so
// with more than a token or two per chunk the kernel is bound by its integer
// instruction issue rather than by reading every selected expert once.
// MLX-style affine groups (Swiftlet article on xix.ai, paragraph 8), packed
// routed gate/up (Runnel README, introduction and "Streaming CLI"), shared
// expert (same article, paragraph 8; Runnel README, "Target").

#include "decode_common.cuh"
#include "moe_common.cuh"
#include "moe_launch.h"

namespace moe {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kUnit = 32;            // columns of the intermediate per unit
constexpr int kBatch = 16;           // gate/up pairs per code batch (one mbarrier each)
constexpr int kNB = kUnit / kBatch;  // batches per unit
constexpr int kQ = 24;               // u32 words of h quads per token (32 codes x 3 bytes / 4)
constexpr int kBoxRows = 256;        // down rows per tensor copy (canonical down layout)

__host__ __device__ constexpr uint32_t al128(uint32_t v) { return (v + 127u) & ~127u; }

// x in 16-bit fixed point. With one to four tokens per chunk the kernel is bound by its integer
// instruction issue, one dp4a per byte plane per four codes and token, and the gate/up rows carry
// two thirds of the codes: so x is held in two byte planes (X = 256 X1 + X0, X1 signed) instead of
// the decode kernel's three, X = rint(x 2^S) with S from the token's largest |x|. Elements within
// 7 binades of the largest are exact (bf16 has 8 significant bits); smaller ones are rounded to
// 2^-S, an error below 2^-15 of the largest element, which enters the gate/up outputs as
// sum_i w_i e_i (w the dequantised weights). tests/test_fixed_point_reading.py emulates this
// rounding around the oracle: on 400 tokens of the 256-wide top-2 layer the bf16 outputs stay
// within rel-L2 9.2e-4 of the oracle's (6.2e-4 with x exact: one-ulp flips of a few outputs
// dominate at that width), under the bound of 1e-3. The unit's h keeps three planes (a unit's 32
// h values are few and heavy-tailed: in two planes as well, 12 of the 400 tokens exceed the bound).
// The largest bf16 below 2^(e+1), times 2^(14-e), is 32640 < 2^15: no overflow.
__device__ __forceinline__ int fix_exp16(float m) {
  if (!(m > 0.f)) return 0;
  int e = ((__float_as_uint(m) >> 23) & 0xFF) - 127;  // floor(log2 m) for normal m
  if (e < -100) e = -100;
  return 14 - e;
}

// sum over one 16-byte segment of codes of q * X for X in two byte planes (q1[.] the signed high
// bytes, q0[.] the low bytes, laid out as for seg_dot): two exact integer sums, one fp32 rounding
template <int BITS>
__device__ __forceinline__ float seg_dot2(const uint4& c, const uint32_t* q1, const uint32_t* q0) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  int a1 = 0;
  uint32_t a0 = 0u;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if constexpr (BITS == 4) {
      const uint32_t lo = w[i] & 0x0F0F0F0Fu, hi = (w[i] >> 4) & 0x0F0F0F0Fu;
      a1 = dp4a_us(lo, q1[2 * i], a1);
      a1 = dp4a_us(hi, q1[2 * i + 1], a1);
      a0 = dp4a_uu(lo, q0[2 * i], a0);
      a0 = dp4a_uu(hi, q0[2 * i + 1], a0);
    } else {
      a1 = dp4a_us(w[i], q1[i], a1);
      a0 = dp4a_uu(w[i], q0[i], a0);
    }
  }
  return fmaf(static_cast<float>(a1), 256.f, static_cast<float>(a0));
}

// Shared-memory carve-up; identical on host (sizing) and device.
struct GvCarve {
  int PS, nsg, QS, QSP, ng, ngd, rowb, UB;
  uint32_t gub[2], xqs, hq, guv, dcd, dsb, total;
  uint32_t gu_bytes;  // one gate/up buffer: [gate 32][up 32] code rows, then [4][32][ng] scales and biases
};

__host__ __device__ inline GvCarve gv_carve(int H, int I, int group, int bits) {
  GvCarve c{};
  c.PS = 128 / bits;
  c.nsg = H / c.PS;
  c.QS = 2 * (c.PS / 4);
  c.QSP = bits == 4 ? xq_stride<4>() : xq_stride<8>();  // quads + sum, padded for 16-byte loads
  c.ng = H / group;
  c.ngd = I / group;
  c.rowb = H * bits / 8;
  c.UB = kUnit * bits / 8;
  c.gu_bytes = 2 * kUnit * c.rowb + 4 * kUnit * c.ng * 2;
  uint32_t o = 0;
  c.gub[0] = o;  o = al128(o + c.gu_bytes);
  c.gub[1] = o;  o = al128(o + c.gu_bytes);
  c.dcd = o;     o = al128(o + H * c.UB);
  c.dsb = o;     o = al128(o + H * 4);
  c.xqs = o;     o = al128(o + kGvTPI * c.nsg * c.QSP * 4);  // the item's tokens' quads
  c.hq = o;      o = al128(o + kGvTPI * (kQ + 2) * 4);       // per token: h quads, sum of X_h, 2^-S_h
  c.guv = o;     o = al128(o + kGvTPI * 2 * kUnit * 4);
  c.total = o;
  return c;
}

__device__ __forceinline__ void tma_3d(void* dst, const CUtensorMap* m, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
          smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_addr(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// One unit of one work item: the expert, which matrix set, and the unit's first column.
struct GvUnit {
  int e;       // expert (0 for the shared expert)
  bool routed;
  int i0;      // first column of the unit inside the expert's intermediate
  int ci;      // chunk (pairs of the item)
  int q;       // unit group of the item (which partial of the outputs)
  int uu;      // unit inside the group
};

template <int BITS, int CH>
__global__ void __launch_bounds__(kThreads, 1) grouped_gemv_kernel(const __grid_constant__ GemvParams p) {
  constexpr int PS = 128 / BITS;
  constexpr int QW = PS / 4;
  extern __shared__ __align__(128) unsigned char sm[];
  __shared__ __align__(8) uint64_t bar_gc[2][kNB];  // gate/up batches of buffer 0 / 1
  __shared__ __align__(8) uint64_t bar_dn;
  __shared__ __align__(8) uint64_t bar_x;           // the item's tokens' quads
  __shared__ int s_pend_gc[2], s_pend_dn, s_pend_x; // copies in flight (phase parity, -1 = none)
  __shared__ float s_xsc[kGvTPI];                   // 2^-S of the item's tokens' x
  __shared__ int s_first, s_cnt;                    // the item's pairs: first sorted position, count

  const int H = p.H, I = p.I, group = p.group;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const GvCarve cv = gv_carve(H, I, group, BITS);
  const int rowb = cv.rowb, ng = cv.ng, nsg = cv.nsg;
  const int lgG = 31 - __clz(group);
  const int upi = p.upi;                     // units per item
  const int NQ = I / (kUnit * upi);          // unit groups per expert
  const int nitems = *p.nchunks * NQ;
  bool ab = false;

  if (tid == 0) {
    for (int b = 0; b < 2; ++b)
      for (int i = 0; i < kNB; ++i) mbar_init(&bar_gc[b][i], 1);
    mbar_init(&bar_dn, 1);
    mbar_init(&bar_x, 1);
    fence_mbar_init();
    s_pend_gc[0] = s_pend_gc[1] = s_pend_dn = s_pend_x = -1;
  }
  __syncthreads();

  // the CTA's stream of units: unit m belongs to item blockIdx.x + (m / upi) * gridDim.x
  auto unit_of = [&](int m, GvUnit& u) -> bool {
    const int it = blockIdx.x + (m / upi) * gridDim.x;
    if (it >= nitems) return false;
    u.ci = it / NQ;
    u.q = it - u.ci * NQ;
    u.uu = m % upi;
    const int e = p.chunks[3 * u.ci];
    u.routed = e < p.E;
    u.e = u.routed ? e : 0;
    u.i0 = (u.q * upi + u.uu) * kUnit;
    return true;
  };
  // gate/up rows of unit u into buffer b (one thread): batch 0 (16 gate + 16 up rows, every
  // scale and bias of the unit), batch 1 (the other 32 rows); phase parity `par` of the batches
  auto issue_gu = [&](const GvUnit& u, int b, int par) {
    const QMat& mq = u.routed ? p.gu : p.sgu;
    const uint8_t* qb = mq.q + static_cast<size_t>(u.e) * mq.q_stride;
    const uint16_t* sb = mq.s + static_cast<size_t>(u.e) * mq.sb_stride;
    const uint16_t* bb = mq.b + static_cast<size_t>(u.e) * mq.sb_stride;
    unsigned char* base = sm + cv.gub[b];
    uint16_t* gsb = reinterpret_cast<uint16_t*>(base + 2 * kUnit * rowb);
    const uint32_t cb = static_cast<uint32_t>(kBatch) * rowb, sbb = static_cast<uint32_t>(kUnit) * ng * 2;
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
#pragma unroll 1
    for (int bt = 0; bt < kNB; ++bt) {
      mbar_arrive_expect_tx(&bar_gc[b][bt], 2 * cb + (bt == 0 ? 4 * sbb : 0u));
      for (int gu = 0; gu < 2; ++gu)
        bulk_g2s(base + static_cast<size_t>(gu * kUnit + bt * kBatch) * rowb,
                 qb + (gu ? mq.up_q : 0) + static_cast<size_t>(u.i0 + bt * kBatch) * rowb, cb, &bar_gc[b][bt]);
      if (bt == 0)
        for (int kind = 0; kind < 4; ++kind)  // gate sc, up sc, gate bi, up bi
          bulk_g2s(gsb + static_cast<size_t>(kind * kUnit) * ng,
                   ((kind & 2) ? bb : sb) + ((kind & 1) ? ((kind & 2) ? mq.up_b : mq.up_s) : 0) +
                       static_cast<size_t>(u.i0) * ng, sbb,
                   &bar_gc[b][bt]);
    }
    s_pend_gc[b] = par;
  };
  // down data of unit u (one thread): its 32 columns of all H rows and its group's scales and biases
  auto issue_dn = [&](const GvUnit& u, int par) {
    const uint16_t* sbm = u.routed ? p.dsb : p.sdsb;
    const uint8_t* cdm = u.routed ? p.dcu : p.sdcu;
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    mbar_arrive_expect_tx(&bar_dn, static_cast<uint32_t>(H) * (cv.UB + (sbm ? 4 : 0)));
    if (cdm) {
      bulk_g2s(sm + cv.dcd, cdm + (static_cast<size_t>(u.e) * (I / kUnit) + u.i0 / kUnit) * H * cv.UB,
               static_cast<uint32_t>(H) * cv.UB, &bar_dn);
    } else {
      const CUtensorMap* tm = u.routed ? &p.tm_dn : &p.tm_sdn;
      for (int r0 = 0; r0 < H; r0 += kBoxRows) tma_3d(sm + cv.dcd + r0 * cv.UB, tm, u.i0 * BITS / 8, r0, u.e, &bar_dn);
    }
    if (sbm)
      bulk_g2s(sm + cv.dsb, sbm + (static_cast<size_t>(u.e) * cv.ngd + u.i0 / group) * H * 2,
               static_cast<uint32_t>(H) * 4, &bar_dn);
    s_pend_dn = par;
  };
  // the item of unit u: its pairs (one thread) and its tokens' quads (one bulk copy per token, rows of
  // the per-token table xquant_kernel wrote) with their 2^-S; phase `par` of bar_x
  const int xwords = nsg * cv.QSP;
  auto issue_x = [&](const GvUnit& u, int par) {
    const int first = p.chunks[3 * u.ci + 1], cnt_u = p.chunks[3 * u.ci + 2];
    int tok[kGvTPI];
#pragma unroll
    for (int t = 0; t < kGvTPI; ++t) {
      const int pid = t < cnt_u ? p.perm[first + t] : 0;
      tok[t] = pid < p.T * p.k ? pid / p.k : pid - p.T * p.k;
    }
    s_first = first;
    s_cnt = cnt_u;
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // the buffer was read by ordinary loads
    mbar_arrive_expect_tx(&bar_x, static_cast<uint32_t>(cnt_u * xwords * 4));
#pragma unroll
    for (int t = 0; t < kGvTPI; ++t)
      if (t < cnt_u) {
        bulk_g2s(sm + cv.xqs + t * xwords * 4, p.xq + static_cast<size_t>(tok[t]) * xwords,
                 static_cast<uint32_t>(xwords * 4), &bar_x);
        s_xsc[t] = p.xsc[tok[t]];
      }
    s_pend_x = par;
  };
  constexpr int kXThread = kThreads - 32;  // lane 0 of the last warp (idle in SwiGLU for <= kGvTPI tokens)
  auto drain = [&]() {
    __syncthreads();
    if (tid == 0) {
      for (int b = 0; b < 2; ++b)
        if (s_pend_gc[b] >= 0)
          for (int i = 0; i < kNB; ++i) mbar_wait(&bar_gc[b][i], s_pend_gc[b], p.hdr, 70);
      if (s_pend_dn >= 0) mbar_wait(&bar_dn, s_pend_dn, p.hdr, 71);
      if (s_pend_x >= 0) mbar_wait(&bar_x, s_pend_x, p.hdr, 74);
    }
    __syncthreads();
  };

  // prologue: the first two units' gate/up rows, the first unit's down data, the first item's x
  GvUnit u0;
  if (!unit_of(0, u0)) return;
  if (tid == 0) {
    issue_gu(u0, 0, 0);
    GvUnit u1;
    if (unit_of(1, u1)) issue_gu(u1, 1, 0);
    issue_dn(u0, 0);
  }
  if (tid == kXThread) issue_x(u0, 0);
  __syncthreads();

  // lane roles in the gate/up dot products (as in the decode kernel)
  const int rps = nsg >= 32 ? 1 : 32 / nsg;
  const int gsub = nsg >= 32 ? 0 : lane / nsg;
  const int gs0 = nsg >= 32 ? lane : lane % nsg;
  uint32_t* xqs = reinterpret_cast<uint32_t*>(sm + cv.xqs);
  uint32_t* hqs = reinterpret_cast<uint32_t*>(sm + cv.hq);
  float* guv = reinterpret_cast<float*>(sm + cv.guv);
  float acc[kGvTPI][4];  // this thread's rows t + 512 r of every token of the item
  int cnt = 0, first = 0;

#pragma unroll 1
  for (int m = 0;; ++m) {
    GvUnit u;
    if (!unit_of(m, u)) break;
    const int b = m & 1;  // gate/up buffer; its phase parity (m / 2) & 1; the down phase m & 1
    if (u.uu == 0) {
      // ---- a new item (its pairs and x issued during the previous item): the accumulators cleared,
      // the x quads awaited
      first = s_first;
      cnt = s_cnt;
#pragma unroll
      for (int t = 0; t < kGvTPI; ++t)
#pragma unroll
        for (int r = 0; r < 4; ++r) acc[t][r] = 0.f;
      if (!mbar_wait(&bar_x, (m / upi) & 1, p.hdr, 75)) ab = true;
    }
    // ---- gate/up + SwiGLU of unit u for every token of the item
    {
      const unsigned char* base = sm + cv.gub[b];
      const uint16_t* gsb = reinterpret_cast<const uint16_t*>(base + 2 * kUnit * rowb);
#pragma unroll 1
      for (int bt = 0; bt < kNB; ++bt) {
        if (warp * rps >= 2 * kBatch) continue;
        if (!mbar_wait(&bar_gc[b][bt], (m >> 1) & 1, p.hdr, 72)) ab = true;
#pragma unroll 1
        for (int rw = warp * rps; rw < 2 * kBatch; rw += 2 * kWarps * rps) {
          // two rows (gate and up of one pair when rps == 1): their codes in registers once
          int gi[2];
          uint4 cd[2][CH];
          float scv[2][CH], biv[2][CH];
#pragma unroll
          for (int r2 = 0; r2 < 2; ++r2) {
            const int rho = rw + r2 * kWarps * rps + gsub;
            const int gu = rho >= kBatch ? 1 : 0;
            const int q = bt * kBatch + rho - gu * kBatch;
            gi[r2] = rho < 2 * kBatch ? gu * kUnit + q : -1;
            const int qq = gi[r2] < 0 ? 0 : q;
            const unsigned char* row = base + static_cast<size_t>(gu * kUnit + qq) * rowb;
#pragma unroll
            for (int ch = 0; ch < CH; ++ch) {
              const int s = gs0 + 32 * ch;
              const int g = (s * PS) >> lgG;
              cd[r2][ch] = *reinterpret_cast<const uint4*>(row + 16 * s);
              scv[r2][ch] = bf16_to_f32(gsb[(gu * kUnit + qq) * ng + g]);
              biv[r2][ch] = bf16_to_f32(gsb[((2 + gu) * kUnit + qq) * ng + g]);
            }
          }
#pragma unroll 1
          for (int t = 0; t < cnt; ++t) {
            const uint32_t* xt = xqs + t * nsg * cv.QSP;
            float a2[2] = {0.f, 0.f};
#pragma unroll
            for (int ch = 0; ch < CH; ++ch) {
              const int s = gs0 + 32 * ch;
              uint32_t xr[2 * QW];
#pragma unroll
              for (int w = 0; w < 2 * QW; w += 4) {
                const uint4 v4 = *reinterpret_cast<const uint4*>(xt + s * cv.QSP + w);
                xr[w] = v4.x;
                xr[w + 1] = v4.y;
                xr[w + 2] = v4.z;
                xr[w + 3] = v4.w;
              }
              const float xsm = __uint_as_float(xt[s * cv.QSP + cv.QS]);
#pragma unroll
              for (int r2 = 0; r2 < 2; ++r2) {
                const float d = seg_dot2<BITS>(cd[r2][ch], xr + QW, xr);
                a2[r2] = fmaf(scv[r2][ch], d, fmaf(biv[r2][ch], xsm, a2[r2]));
              }
            }
            if (nsg >= 32) {
#pragma unroll
              for (int o = 16; o > 0; o >>= 1) {
                a2[0] += __shfl_xor_sync(0xffffffffu, a2[0], o);
                a2[1] += __shfl_xor_sync(0xffffffffu, a2[1], o);
              }
            } else {
#pragma unroll 1
              for (int o = nsg >> 1; o > 0; o >>= 1) {
                a2[0] += __shfl_xor_sync(0xffffffffu, a2[0], o);
                a2[1] += __shfl_xor_sync(0xffffffffu, a2[1], o);
              }
            }
            if (gs0 == 0) {
              const float isx = s_xsc[t];
              if (gi[0] >= 0) guv[t * 2 * kUnit + gi[0]] = a2[0] * isx;
              if (gi[1] >= 0) guv[t * 2 * kUnit + gi[1]] = a2[1] * isx;
            }
          }
        }
      }
    }
    if (__syncthreads_or(ab)) { drain(); return; }
    if (tid == 0) s_pend_gc[b] = -1;
    // buffer b is free: the unit two ahead goes into it
    if (tid == 0) {
      GvUnit un;
      if (unit_of(m + 2, un)) issue_gu(un, b, ((m + 2) >> 1) & 1);
    }
    // after the item's last gate/up the x buffer is free: the next item's pairs and x
    if (tid == kXThread && u.uu == upi - 1) {
      s_pend_x = -1;
      GvUnit un;
      if (unit_of(m + 1, un)) issue_x(un, ((m + 1) / upi) & 1);
    }
    // SwiGLU; each token's h as fixed point (its own exponent), quads for the down rows
    if (warp < cnt) {
      const int t = warp;
      const float h = silu_f(guv[t * 2 * kUnit + lane]) * guv[t * 2 * kUnit + kUnit + lane];
      const int Sh = fix_exp(warp_max(fabsf(h)));
      const int X = __float2int_rn(h * pow2f(Sh));
      int hs = X;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) hs += __shfl_xor_sync(0xffffffffu, hs, o);
      const int qp = (BITS == 4) ? quad_pos<4>(lane) : lane;
      unsigned char* hqb = reinterpret_cast<unsigned char*>(hqs + t * (kQ + 2));
#pragma unroll
      for (int j = 0; j < 3; ++j) hqb[(j * 8 + (qp >> 2)) * 4 + (qp & 3)] = static_cast<unsigned char>(xbyte(X, j));
      if (lane == 0) {
        hqs[t * (kQ + 2) + kQ] = __float_as_uint(static_cast<float>(hs));
        hqs[t * (kQ + 2) + kQ + 1] = __float_as_uint(pow2f(-Sh));
      }
    }
    if (tid < H && !mbar_wait(&bar_dn, m & 1, p.hdr, 73)) ab = true;
    if (__syncthreads_or(ab)) { drain(); return; }
    if (tid == 0) s_pend_dn = -1;
    // ---- down: thread tid's rows tid + 512 r, every token of the item
    {
      const uint16_t* sbm = u.routed ? p.dsb : p.sdsb;
      const QMat& dm = u.routed ? p.dn : p.sdn;
      const size_t sb0 = static_cast<size_t>(u.e) * dm.sb_stride + u.i0 / group;
      const uint32_t* dsb = reinterpret_cast<const uint32_t*>(sm + cv.dsb);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int row = tid + r * kThreads;
        if (row < H) {
          const unsigned char* drow = sm + cv.dcd + row * cv.UB;
          float sc, bi;
          if (sbm) {
            const uint32_t w = dsb[row];
            sc = bf16_lo(w);
            bi = bf16_hi(w);
          } else {
            sc = bf16_to_f32(__ldg(dm.s + sb0 + static_cast<size_t>(row) * cv.ngd));
            bi = bf16_to_f32(__ldg(dm.b + sb0 + static_cast<size_t>(row) * cv.ngd));
          }
          const uint4 c0 = *reinterpret_cast<const uint4*>(drow);
          uint4 c1 = c0;
          if constexpr (BITS == 8) c1 = *reinterpret_cast<const uint4*>(drow + 16);
#pragma unroll
          for (int t = 0; t < kGvTPI; ++t) {
            if (t < cnt) {
              const uint32_t* hr = hqs + t * (kQ + 2);
              float d;
              if constexpr (BITS == 4) {
                d = seg_dot<4>(c0, hr + 16, hr + 8, hr);
              } else {
                d = seg_dot<8>(c0, hr + 16, hr + 8, hr) + seg_dot<8>(c1, hr + 20, hr + 12, hr + 4);
              }
              acc[t][r] += __uint_as_float(hr[kQ + 1]) * fmaf(sc, d, bi * __uint_as_float(hr[kQ]));
            }
          }
        }
      }
    }
    if (__syncthreads_or(ab)) { drain(); return; }
    // the down buffer is free: the next unit's down data
    if (tid == 0) {
      GvUnit un;
      if (unit_of(m + 1, un)) issue_dn(un, (m + 1) & 1);
    }
    // ---- the item's last unit: its partial of each pair's expert output
    if (u.uu == upi - 1) {
      float* ob = p.o + static_cast<size_t>(u.q) * p.npairs * H;
#pragma unroll
      for (int t = 0; t < kGvTPI; ++t) {
        if (t < cnt) {
          const int pid = p.perm[first + t];
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int row = tid + r * kThreads;
            if (row < H) ob[static_cast<size_t>(pid) * H + row] = acc[t][r];
          }
        }
      }
    }
  }
  drain();
}

// Every token's x as the fixed-point quads the gate/up dot products read ([T][nsg][QSP] words,
// QSP = xq_stride: per segment the two byte planes' quads, the segment's sum of X, padding), its
// 2^-S, and the shared expert's sigmoid gate. One CTA per token, H/4 threads, each thread 4
// consecutive elements (element group g = thread g: its partner group g ^ 1 is the neighbouring
// lane, the PS / 4 groups of a segment are consecutive lanes).
template <int BITS>
__global__ void xquant_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ wsg, int H, int Is,
                              uint32_t* __restrict__ xq, float* __restrict__ xsc, float* __restrict__ sgate) {
  constexpr int PS = 128 / BITS;
  constexpr int QW = PS / 4;
  const int t = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int QSP = xq_stride<BITS>();
  const int nsg = H / PS;
  __shared__ float s_red[2][16];
  const uint2 wv = *reinterpret_cast<const uint2*>(x + static_cast<size_t>(t) * H + 4 * tid);
  const float xv[4] = {bf16_lo(wv.x), bf16_hi(wv.x), bf16_lo(wv.y), bf16_hi(wv.y)};
  float mx = fmaxf(fmaxf(fabsf(xv[0]), fabsf(xv[1])), fmaxf(fabsf(xv[2]), fabsf(xv[3])));
  float dg = 0.f;
  if (Is > 0) {
    const uint2 gw = *reinterpret_cast<const uint2*>(wsg + 4 * tid);
    dg = fmaf(xv[0], bf16_lo(gw.x), fmaf(xv[1], bf16_hi(gw.x), fmaf(xv[2], bf16_lo(gw.y), xv[3] * bf16_hi(gw.y))));
  }
  mx = warp_max(mx);
  dg = warp_sum(dg);
  if (lane == 0) {
    s_red[0][warp] = mx;
    s_red[1][warp] = dg;
  }
  __syncthreads();
  float m = 0.f, sg = 0.f;
  for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) {
    m = fmaxf(m, s_red[0][w]);
    sg += s_red[1][w];
  }
  const int S = fix_exp16(m);
  const float sx = pow2f(S);
  int X[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) X[u] = __float2int_rn(xv[u] * sx);
  int xs = (X[0] + X[1]) + (X[2] + X[3]);
  int e[4], qi, sgi;
  if constexpr (BITS == 4) {
    const int h = tid & 1;
    const int r0 = __shfl_xor_sync(0xffffffffu, h ? X[0] : X[1], 1);
    const int r1 = __shfl_xor_sync(0xffffffffu, h ? X[2] : X[3], 1);
    e[0] = h ? r0 : X[0];
    e[1] = h ? r1 : X[2];
    e[2] = h ? X[1] : r0;
    e[3] = h ? X[3] : r1;
    qi = ((tid >> 1) & 3) * 2 + h;
    sgi = tid >> 3;
  } else {
    e[0] = X[0];
    e[1] = X[1];
    e[2] = X[2];
    e[3] = X[3];
    qi = tid & 3;
    sgi = tid >> 2;
  }
  uint32_t* dst = xq + static_cast<size_t>(t) * nsg * QSP;
#pragma unroll
  for (int j = 0; j < 2; ++j)
    dst[sgi * QSP + j * QW + qi] =
        xbyte(e[0], j) | (xbyte(e[1], j) << 8) | (xbyte(e[2], j) << 16) | (xbyte(e[3], j) << 24);
#pragma unroll
  for (int o = 1; o < PS / 4; o <<= 1) xs += __shfl_xor_sync(0xffffffffu, xs, o);
  if ((tid & (PS / 4 - 1)) == 0) dst[sgi * QSP + 2 * QW] = __float_as_uint(static_cast<float>(xs));
  if (tid == 0) {
    xsc[t] = pow2f(-S);
    if (Is > 0) sgate[t] = 1.f / (1.f + expf(-sg));
  }
}

// y[t][r] = bf16( sum_j w[t][j] * sum_q O[q][t*k+j][r] + gate[t] * sum_q O[q][T*k+t][r] ), rank order,
// the partials of each pair summed in order, the shared expert last. Each thread four consecutive rows
// (16-byte loads); the (pair, partial) terms are walked in that order 16 loads at a time, across pair
// boundaries, so a thread waits for ceil((k + 1) * nq / 16) round trips.
__global__ void __launch_bounds__(256) gv_combine_kernel(const float* __restrict__ o, const float* __restrict__ w,
                                                         const float* __restrict__ sgate, int T, int k, int H, int Is,
                                                         int nq, int npairs, uint16_t* __restrict__ y) {
  constexpr int kBatchLoads = 16;
  const size_t n4 = static_cast<size_t>(T) * H / 4;
  const size_t plane = static_cast<size_t>(npairs) * H;
  const int nslot = k + (Is > 0 ? 1 : 0);
  const int nterm = nslot * nq;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>((4 * i) / H), r = static_cast<int>((4 * i) % H);
    auto term_addr = [&](int j, int q) -> const float4* {  // slot j, partial q
      const size_t pid = j < k ? static_cast<size_t>(t) * k + j : static_cast<size_t>(T) * k + t;
      return reinterpret_cast<const float4*>(o + q * plane + pid * H + r);
    };
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f), s = acc;
    int jl = 0, ql = 0;  // next term to load
    int jc = 0, qc = 0;  // next term to add
#pragma unroll 1
    for (int f0 = 0; f0 < nterm; f0 += kBatchLoads) {
      float4 v[kBatchLoads];
#pragma unroll
      for (int b = 0; b < kBatchLoads; ++b)
        if (f0 + b < nterm) {
          v[b] = __ldg(term_addr(jl, ql));
          if (++ql == nq) {
            ql = 0;
            ++jl;
          }
        }
#pragma unroll
      for (int b = 0; b < kBatchLoads; ++b)
        if (f0 + b < nterm) {
          if (qc == 0) {
            s = v[b];
          } else {
            s.x += v[b].x;
            s.y += v[b].y;
            s.z += v[b].z;
            s.w += v[b].w;
          }
          if (++qc == nq) {  // the pair's sum is complete
            const float c = jc < k ? w[static_cast<size_t>(t) * k + jc] : sgate[t];
            acc.x = fmaf(c, s.x, acc.x);
            acc.y = fmaf(c, s.y, acc.y);
            acc.z = fmaf(c, s.z, acc.z);
            acc.w = fmaf(c, s.w, acc.w);
            qc = 0;
            ++jc;
          }
        }
    }
    uint2 packed;
    packed.x = static_cast<uint32_t>(f32_to_bf16(acc.x)) | (static_cast<uint32_t>(f32_to_bf16(acc.y)) << 16);
    packed.y = static_cast<uint32_t>(f32_to_bf16(acc.z)) | (static_cast<uint32_t>(f32_to_bf16(acc.w)) << 16);
    *reinterpret_cast<uint2*>(y + 4 * i) = packed;
  }
}

template <int BITS, int CH>
cudaError_t launch_gv(const GemvParams& p, int grid, cudaStream_t st) {
  const GvCarve cv = gv_carve(p.H, p.I, p.group, BITS);
  auto kern = grouped_gemv_kernel<BITS, CH>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(cv.total));
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, cv.total, st>>>(p);
  return cudaGetLastError();
}

bool pow2i(int v) { return v > 0 && (v & (v - 1)) == 0; }

}  // namespace

size_t grouped_gemv_smem(int H, int I, int group, int bits) { return gv_carve(H, I, group, bits).total; }

bool grouped_gemv_supported(int H, int I, int Is, int group, int bits, size_t smem_limit) {
  const int PS = 128 / bits, nsg = H / PS;
  if (H % PS || H > 4 * kThreads || H % kBoxRows) return false;
  if (!(pow2i(nsg) && nsg <= 32) && !(nsg % 32 == 0 && nsg / 32 <= (bits == 4 ? 2 : 4))) return false;
  if (Is != 0 && Is != I) return false;
  if (I % (kUnit * kGvUPI) || !pow2i(group) || group % kUnit || I % group) return false;
  return gv_carve(H, I, group, bits).total <= smem_limit;
}

cudaError_t launch_xquant(const uint16_t* x, const uint16_t* wsg, int T, int H, int Is, int bits, uint32_t* xq,
                          float* xsc, float* sgate, cudaStream_t st) {
  if (bits == 4) xquant_kernel<4><<<T, H / 4, 0, st>>>(x, wsg, H, Is, xq, xsc, sgate);
  else xquant_kernel<8><<<T, H / 4, 0, st>>>(x, wsg, H, Is, xq, xsc, sgate);
  return cudaGetLastError();
}

cudaError_t launch_grouped_gemv(const GemvParams& p, int bits, int grid, cudaStream_t st) {
  const int nsg = p.H * bits / 128;
  const int ch = nsg >= 32 ? nsg / 32 : 1;
  if (bits == 4) return ch == 1 ? launch_gv<4, 1>(p, grid, st) : launch_gv<4, 2>(p, grid, st);
  if (ch == 1) return launch_gv<8, 1>(p, grid, st);
  if (ch == 2) return launch_gv<8, 2>(p, grid, st);
  if (ch == 3) return launch_gv<8, 3>(p, grid, st);  // 1536-wide 8-bit rows
  return launch_gv<8, 4>(p, grid, st);
}

cudaError_t launch_gv_combine(const float* o, const float* w, const float* sgate, int T, int k, int H, int Is, int nq,
                              int npairs, uint16_t* y, int grid, cudaStream_t st) {
  gv_combine_kernel<<<grid, 256, 0, st>>>(o, w, sgate, T, k, H, Is, nq, npairs, y);
  return cudaGetLastError();
}

}  // namespace moe
