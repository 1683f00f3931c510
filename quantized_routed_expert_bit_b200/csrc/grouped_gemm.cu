// Kernel (c): the batched path. Tokens are grouped by expert (counting sort,
// sort_by_expert.cu), so each selected expert's weights are read once for
// all of its tokens, and each expert's gate/up and down products become
// small GEMMs run on the tensor cores (tcgen05, accumulators in TMEM).
//
//   gather   x (bf16) of every (token, expert) pair, in expert order, as
//            fp16 rows: the B operand of the gate/up GEMM; also the shared
//            expert's sigmoid gate per token;
//   GEMM gu  per (expert chunk of <=64 pairs, 64 intermediate indices):
//            A = the integer codes of the 64 gate rows and 64 up rows, as
//            exact fp16 integers, B = the chunk's gathered tokens; epilogue
//            h = silu(gate) * up, stored as an fp16 hi/lo pair, plus the
//            sum of h over each group of 64 intermediate indices;
//   GEMM dn  per (expert chunk, 128 output rows): A = the down rows' codes,
//            B = h hi and h lo (two MMAs, so h keeps ~22 bits); epilogue
//            writes each pair's output row (fp32);
//   combine  y = sum_j w_j o_j + sigmoid-gate * o_shared, in rank order,
//            one bf16 rounding.
// MLX-style affine groups (Swiftlet article on xix.ai, paragraph 8), packed
// routed gate/up (Runnel README, introduction and "Streaming CLI"), shared
// expert (same article, paragraph 8; Runnel README, "Target").
//
// GEMM CTA (one per SM, persistent over tiles), 16 warps:
//   warp 5      TMA producer: codes (3D map over the expert stack);
//   warp 9      TMA producer: scales and biases (per tile), B tiles (128-byte swizzled);
//   warps 1,11  MMA issuers: lane 0 issues tcgen05.mma (M=128, N=16/32, K=16) for
//               even / odd k-blocks (a single issuing thread spends ~0.6 us of
//               waits, MMAs and commits per k-block; two halve that); warp 1 owns TMEM;
//   warps 0,2,3,4,6,7,8,10  unpack codes into exact fp16 integers, swizzled A tiles;
//   warps 12-15 scale and accumulate, then the epilogue.
// The weight of code q in group g is s*q + b (MLX-style affine groups), so
// a row's dot product with a column x is  sum_g ( s_g * P_g + b_g * X_g ),
// P_g = sum_{k in g} q_k x_k,  X_g = sum_{k in g} x_k.  One k-block is one
// group of 64: the tensor cores form P_g from exact integer codes and exact
// fp16 activations with fp32 accumulation, each group into its own TMEM
// buffer (4 in rotation), and the scaling warps add s_g * P_g + b_g * X_g
// into fp32 registers. No weight is ever rounded to 16 bits. A stage ring
// of NS k-blocks decouples the roles; every wait is bounded and an abort
// drains copies and MMAs before TMEM is freed.
//
// Unpacking: 4-bit codes become fp16 (1024 + q) / (64 + q) by one lop3 per
// pair of codes and subtracting the offset gives q exactly. The pairs come
// out as (k, k+4) within each 8 codes, so the A tile holds K in the order
// 0,4,1,5,2,6,3,7 inside every 8; the B operands (gathered x, h) are
// written in the same order (a dot product does not depend on the order).

#include <cuda_fp16.h>

#include "moe_common.cuh"
#include "moe_launch.h"
#include "tc.cuh"

namespace moe {

namespace {

constexpr int kThreads = 512;
constexpr int kBM = 128;           // tile rows
constexpr int kGK = 64;            // K of one quantisation group: one 128-byte swizzle row of fp16
constexpr int kSG = 2;             // groups per pipeline stage (every wait and arrive covers two)
constexpr int kNT = kChunkTokens;  // columns (pairs) per tile
constexpr int kPS = 4;             // stages of per-group products in TMEM (kPS * kSG buffers)
constexpr int kNA = 2;             // stages of unpacked A tiles in flight (a third one, paid for with
                                   // a shallower codes ring, measured slower)
constexpr int kNB = 4;             // stages of B tiles in flight
constexpr int kATileBytes = kBM * kGK * 2;          // one group's A tile (16 KiB)
constexpr int kAStageBytes = kSG * kATileBytes;
// Warp roles. Warp w runs on sub-partition w % 4; the MMA issuer is a single
// latency-bound thread, so its sub-partition (1) holds only light roles besides
// one scaler (the scalers must cover the four TMEM lane quarters, w % 4).
constexpr int kMmaWarp = 1;        // TMEM owner; issues the MMAs of even k-blocks
constexpr int kMmaWarp2 = 11;      // issues the MMAs of odd k-blocks (its own commits and drain)
constexpr int kCodesWarp = 5;      // TMA producer of the codes
constexpr int kBWarp = 9;          // TMA producer of the B tiles, scales and biases
constexpr int kEpiWarp0 = 12;      // warps 12..15: scalers + epilogue
// unpacker index (0..7) of warp w, or -1
__host__ __device__ constexpr int unpack_index(int w) {
  return w == 0 ? 0 : w == 2 ? 1 : w == 3 ? 2 : w == 4 ? 3 : w == 6 ? 4 : w == 7 ? 5 : w == 8 ? 6 : w == 10 ? 7 : -1;
}

__host__ __device__ constexpr uint32_t al1k(uint32_t v) { return (v + 1023u) & ~1023u; }

// Position p of an 8-block of K holds element kPerm8[p] (4-bit codes only).
__host__ __device__ constexpr int perm8_pos(int k) {  // position of element k
  return (k & 4) ? ((k & 3) * 2 + 1) : ((k & 3) * 2);
}

struct GemmSmem {
  uint32_t a, b, codes, sc, xs, bar, total;
  int nc, b_stage_bytes, codes_stage_bytes, sc_buf_bytes;
};

// Rings, in stages of kSG groups: codes (nc stages, freed once unpacked), B
// tiles (kNB, freed by the MMAs), unpacked A tiles (kNA, freed by the MMAs).
__host__ __device__ inline GemmSmem gemm_smem(int mode, int bits, int K) {
  GemmSmem s{};
  const int ng = K / kGK;
  s.b_stage_bytes = kSG * (mode == 0 ? 1 : 2) * kNT * 128;  // per group kNT rows x 128 B (x2: h hi and lo)
  s.codes_stage_bytes = kBM * kSG * (kGK * bits / 8);
  s.nc = (64 * 1024) / s.codes_stage_bytes;                 // 64 KiB of codes in flight
  s.sc_buf_bytes = 2 * kBM * ng * 2;                        // scales and biases of 128 rows
  uint32_t o = 0;
  s.a = o;     o = al1k(o + kNA * kAStageBytes);
  s.b = o;     o = al1k(o + kNB * s.b_stage_bytes);
  s.codes = o; o = al1k(o + s.nc * s.codes_stage_bytes);
  s.sc = o;    o = al1k(o + 2 * s.sc_buf_bytes);
  s.xs = o;    o = al1k(o + 4 * ng * kNT * 4);        // group sums of the tile's columns, one copy per scaling warp
  s.bar = o;   o += 1024;  // the mbarriers (~45), the TMEM slot and the abort flag
  s.total = o + 1024;  // slack to align the dynamic base to 1 KiB
  return s;
}

__device__ __forceinline__ int b_box_index(int n) { return n <= 16 ? 0 : 1; }
__device__ __forceinline__ int b_box_rows(int i) { return 16 << i; }

__device__ __forceinline__ float silu_f(float z) { return z / (1.f + expf(-z)); }

// Bounded wait that also gives up as soon as another role has aborted.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, WsHeader* hdr, volatile int* abort,
                                              int where) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0; it < kWaitIters; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > kWaitNs) break;
  }
  report(hdr, MOE_ERR_TIMEOUT, where);
  *abort = 1;
  return false;
}

// Warp-uniform wait: lane 0 waits, every lane gets the same answer.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, WsHeader* hdr, volatile int* abort,
                                         int where) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = wait_or_abort(bar, parity, hdr, abort, where);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

__device__ __forceinline__ bool warp_aborted(volatile int* abort) {
  return __shfl_sync(0xffffffffu, ((threadIdx.x & 31) == 0) ? *abort : 0, 0) != 0;
}

// 32 4-bit codes (16 bytes) of one row -> 4 16-byte chunks of exact fp16 integers.
__device__ __forceinline__ void unpack32_u4(const uint4 c, uint4* out) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  const __half2 k1024 = __half2half2(__ushort_as_half(0x6400));
  const __half2 k64 = __half2half2(__ushort_as_half(0x5400));
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t x = w[i], y = w[i] >> 8;
    uint32_t v0 = (x & 0x000F000Fu) | 0x64006400u;  // (1024 + q0, 1024 + q4)
    uint32_t v1 = (x & 0x00F000F0u) | 0x54005400u;  // (  64 + q1,   64 + q5)
    uint32_t v2 = (y & 0x000F000Fu) | 0x64006400u;  // (1024 + q2, 1024 + q6)
    uint32_t v3 = (y & 0x00F000F0u) | 0x54005400u;  // (  64 + q3,   64 + q7)
    __half2 d0 = __hsub2(*reinterpret_cast<__half2*>(&v0), k1024);
    __half2 d1 = __hsub2(*reinterpret_cast<__half2*>(&v1), k64);
    __half2 d2 = __hsub2(*reinterpret_cast<__half2*>(&v2), k1024);
    __half2 d3 = __hsub2(*reinterpret_cast<__half2*>(&v3), k64);
    out[i] = make_uint4(*reinterpret_cast<uint32_t*>(&d0), *reinterpret_cast<uint32_t*>(&d1),
                        *reinterpret_cast<uint32_t*>(&d2), *reinterpret_cast<uint32_t*>(&d3));
  }
}

// 32 8-bit codes (32 bytes) of one row -> 4 16-byte chunks of exact fp16 integers (natural K order).
__device__ __forceinline__ void unpack32_u8(const uint4 c0, const uint4 c1, uint4* out) {
  const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  const __half2 k1024 = __half2half2(__ushort_as_half(0x6400));
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t r[4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t x = w[2 * i + h];
      uint32_t v0 = __byte_perm(x, 0x64646464u, 0x5140);  // (1024 + b0, 1024 + b1)
      uint32_t v1 = __byte_perm(x, 0x64646464u, 0x5342);  // (1024 + b2, 1024 + b3)
      __half2 d0 = __hsub2(*reinterpret_cast<__half2*>(&v0), k1024);
      __half2 d1 = __hsub2(*reinterpret_cast<__half2*>(&v1), k1024);
      r[2 * h] = *reinterpret_cast<uint32_t*>(&d0);
      r[2 * h + 1] = *reinterpret_cast<uint32_t*>(&d1);
    }
    out[i] = make_uint4(r[0], r[1], r[2], r[3]);
  }
}

// ------------------------------------------------------------------ GEMM kernel

template <int MODE, int BITS>
__global__ void __launch_bounds__(kThreads, 1) grouped_gemm_kernel(const __grid_constant__ GemmParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const GemmSmem L = gemm_smem(MODE, BITS, p.K);
  const int NC = L.nc;
  uint64_t* cfull = reinterpret_cast<uint64_t*>(sm + L.bar);  // [NC] codes landed
  uint64_t* cempty = cfull + NC;                              // [NC] codes unpacked
  uint64_t* bfull = cempty + NC;                              // [kNB] B tiles landed
  uint64_t* bempty = bfull + kNB;                             // [kNB] MMAs done with the B tiles
  uint64_t* afull = bempty + kNB;                             // [kNA] A tiles written
  uint64_t* aempty = afull + kNA;                             // [kNA] MMAs done with the A tiles
  uint64_t* scfull = aempty + kNA;                            // [2] scales of a tile landed
  uint64_t* scempty = scfull + 2;                             // [2] scalers done with them
  uint64_t* pfull = scempty + 2;                              // [kPS] a stage's products are in TMEM
  uint64_t* pempty = pfull + kPS;                             // [kPS] scalers have read them
  uint64_t* drain = pempty + kPS;                             // [2] MMA issuers: everything issued has finished
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 2);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int CB = kGK * BITS / 8;          // code bytes per row per group
  const int ng = p.K / kGK;               // groups per row
  const int nst = ng / kSG;               // stages per tile (ng is a multiple of 8)
  const int MT = (MODE == 0) ? p.I / 64 : p.H / kBM;
  const int nchunks = *p.nchunks;
  const int ntiles = nchunks * MT;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NC; ++i) {
      mbar_init(&cfull[i], 1);
      mbar_init(&cempty[i], 8);
    }
    for (int i = 0; i < kNB; ++i) {
      mbar_init(&bfull[i], 1);
      mbar_init(&bempty[i], 1);
    }
    for (int i = 0; i < kNA; ++i) {
      mbar_init(&afull[i], 8);
      mbar_init(&aempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&scfull[i], 1);
      mbar_init(&scempty[i], 4);
    }
    for (int i = 0; i < kPS; ++i) {
      mbar_init(&pfull[i], 1);
      mbar_init(&pempty[i], 4);
    }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tc::tmem_alloc(tmem_slot, kPS * kSG * kNT);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == kCodesWarp) {
    // ------------------------------------------------ codes producer (deep ring, freed by the unpackers)
    if (lane == 0) {
      for (int i = 0; i < 2; ++i) tc::prefetch_tmap(&p.tm_codes[i]);
      int sg = 0, last = -1;
      for (int t = blockIdx.x; t < ntiles && !*abort; t += gridDim.x) {
        const int ci = t / MT, mt = t % MT;
        const int e = p.chunks[3 * ci];
        const bool shared = (e == p.E);
        const int ez = shared ? 0 : e, mi = shared ? 1 : 0;
        const int r0 = (MODE == 0) ? mt * 64 : mt * kBM;
        const int r1 = (MODE == 0) ? p.rows / 2 + mt * 64 : mt * kBM + 64;
        bool ok = true;
        for (int st = 0; st < nst; ++st, ++sg) {
          const int s = sg % NC, u = sg / NC;
          if (u >= 1 && !wait_or_abort(&cempty[s], (u - 1) & 1, p.hdr, abort, 31)) { ok = false; break; }
          unsigned char* cs = sm + L.codes + s * L.codes_stage_bytes;
          tc::mbar_expect_tx(&cfull[s], static_cast<uint32_t>(L.codes_stage_bytes));
          tc::tma_load_3d(cs, &p.tm_codes[mi], st * kSG * CB, r0, ez, &cfull[s]);
          tc::tma_load_3d(cs + 64 * kSG * CB, &p.tm_codes[mi], st * kSG * CB, r1, ez, &cfull[s]);
          tc::mbar_arrive(&cfull[s]);
          last = sg;
        }
        if (!ok) break;
      }
      // leave no copy in flight
      for (int j = (last - NC + 1 > 0 ? last - NC + 1 : 0); j <= last; ++j) mbar_wait(&cfull[j % NC], (j / NC) & 1, p.hdr, 39);
    }
  } else if (warp == kBWarp) {
    // ------------------------------------------------ B tiles and scales producer (freed by MMAs / scalers)
    if (lane == 0) {
      for (int i = 0; i < 2; ++i) {
        tc::prefetch_tmap(&p.tm_scales[i]);
        tc::prefetch_tmap(&p.tm_biases[i]);
      }
      int sg = 0, it = 0, last = -1;
      int sc_armed[2] = {-1, -1};
      for (int t = blockIdx.x; t < ntiles && !*abort; t += gridDim.x, ++it) {
        const int ci = t / MT, mt = t % MT;
        const int e = p.chunks[3 * ci], start = p.chunks[3 * ci + 1], cnt = p.chunks[3 * ci + 2];
        const bool shared = (e == p.E);
        const int ez = shared ? 0 : e, mi = shared ? 1 : 0;
        const int bi = b_box_index(cnt);
        const int brows = b_box_rows(bi);
        const int tb = it & 1, tu = it >> 1;
        if (tu >= 1 && !wait_or_abort(&scempty[tb], (tu - 1) & 1, p.hdr, abort, 30)) break;
        unsigned char* scb = sm + L.sc + tb * L.sc_buf_bytes;
        const uint32_t half_bytes = 64u * ng * 2u;
        tc::mbar_expect_tx(&scfull[tb], 4u * half_bytes);
        const int r0 = (MODE == 0) ? mt * 64 : mt * kBM;
        const int r1 = (MODE == 0) ? p.rows / 2 + mt * 64 : mt * kBM + 64;
        tc::tma_load_3d(scb, &p.tm_scales[mi], 0, r0, ez, &scfull[tb]);
        tc::tma_load_3d(scb + half_bytes, &p.tm_scales[mi], 0, r1, ez, &scfull[tb]);
        tc::tma_load_3d(scb + 2 * half_bytes, &p.tm_biases[mi], 0, r0, ez, &scfull[tb]);
        tc::tma_load_3d(scb + 3 * half_bytes, &p.tm_biases[mi], 0, r1, ez, &scfull[tb]);
        tc::mbar_arrive(&scfull[tb]);
        sc_armed[tb] = tu;
        bool ok = true;
        for (int st = 0; st < nst; ++st, ++sg) {
          const int s = sg % kNB, u = sg / kNB;
          if (u >= 1 && !wait_or_abort(&bempty[s], (u - 1) & 1, p.hdr, abort, 32)) { ok = false; break; }
          unsigned char* bs = sm + L.b + s * L.b_stage_bytes;
          tc::mbar_expect_tx(&bfull[s], static_cast<uint32_t>(brows) * 128u * kSG * (MODE == 0 ? 1u : 2u));
#pragma unroll
          for (int g = 0; g < kSG; ++g) {
            tc::tma_load_2d(bs + g * kNT * 128, &p.tm_b[bi], (st * kSG + g) * kGK, start, &bfull[s]);
            if (MODE == 1) tc::tma_load_2d(bs + (kSG + g) * kNT * 128, &p.tm_b2[bi], (st * kSG + g) * kGK, start, &bfull[s]);
          }
          tc::mbar_arrive(&bfull[s]);
          last = sg;
        }
        if (!ok) break;
      }
      for (int j = (last - kNB + 1 > 0 ? last - kNB + 1 : 0); j <= last; ++j) mbar_wait(&bfull[j % kNB], (j / kNB) & 1, p.hdr, 37);
      for (int b = 0; b < 2; ++b)
        if (sc_armed[b] >= 0) mbar_wait(&scfull[b], sc_armed[b] & 1, p.hdr, 38);
    }
  } else if (warp == kMmaWarp || warp == kMmaWarp2) {
    // ------------------------------------------------ MMA issuers: each group of a stage into its own TMEM buffer
    const int par = (warp == kMmaWarp) ? 0 : 1;  // stages of this parity (nst is even)
    if (lane == 0) {
      int sg = 0;
      for (int t = blockIdx.x; t < ntiles && !*abort; t += gridDim.x) {
        const int ci = t / MT;
        const int cnt = p.chunks[3 * ci + 2];
        const int npad = (cnt + 15) & ~15;
        const uint32_t idesc = tc::idesc_f16_f32(kBM, npad);
        bool ok = true;
        for (int st = 0; st < nst; ++st, ++sg) {
          if ((sg & 1) != par) continue;
          const int as = sg % kNA, au = sg / kNA;
          const int bs = sg % kNB, bu = sg / kNB;
          const int ps = sg % kPS, pu = sg / kPS;
          if (!wait_or_abort(&afull[as], au & 1, p.hdr, abort, 41) || !wait_or_abort(&bfull[bs], bu & 1, p.hdr, abort, 42) ||
              (pu >= 1 && !wait_or_abort(&pempty[ps], (pu - 1) & 1, p.hdr, abort, 43))) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          // descriptors built once per stage; inside the stage they step by their start-address
          // field (16-byte units): +2 per K step of 16 (32 bytes), +1024 per A tile, +kNT*8 per B tile
          const uint64_t ad0 = tc::smem_desc_sw128(smem_addr(sm + L.a + as * kAStageBytes));
          const uint64_t bd0 = tc::smem_desc_sw128(smem_addr(sm + L.b + bs * L.b_stage_bytes));
#pragma unroll
          for (int g = 0; g < kSG; ++g) {
            const uint32_t dt = tmem + (ps * kSG + g) * kNT;
            const uint64_t ag = ad0 + static_cast<uint64_t>(g * (kATileBytes >> 4));
            const uint64_t bg = bd0 + static_cast<uint64_t>(g * (kNT * 128 >> 4));
#pragma unroll
            for (int kk = 0; kk < kGK / 16; ++kk) {
              tc::mma_f16(dt, ag + 2 * kk, bg + 2 * kk, idesc, kk != 0);
              if (MODE == 1) tc::mma_f16(dt, ag + 2 * kk, bg + (kSG * kNT * 128 >> 4) + 2 * kk, idesc, 1);
            }
          }
          tc::commit(&aempty[as]);
          tc::commit(&bempty[bs]);
          tc::commit(&pfull[ps]);
        }
        if (!ok) break;
      }
      // every MMA issued must be finished before TMEM is released
      tc::commit(&drain[par]);
      mbar_wait(&drain[par], 0, p.hdr, 49);
    }
  } else if (unpack_index(warp) >= 0) {
    // ------------------------------------------------ unpackers: 2 threads per row, both groups of a stage
    const int d = unpack_index(warp) * 32 + lane;  // 0..255
    const int m = d >> 1, half = d & 1;              // A-tile row, which 32 codes of each group's 64
    // A row m <- staging row: gate/up interleaved for mode 0, identity for mode 1
    const int srow = (MODE == 0) ? ((m & 1) * 64 + (m >> 1)) : m;
    int sg = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
      if (warp_aborted(abort)) break;
      bool ok = true;
      for (int st = 0; st < nst; ++st, ++sg) {
        const int cs = sg % NC, cu = sg / NC;
        const int as = sg % kNA, au = sg / kNA;
        if (!warp_wait(&cfull[cs], cu & 1, p.hdr, abort, 51)) { ok = false; break; }
        if (au >= 1 && !warp_wait(&aempty[as], (au - 1) & 1, p.hdr, abort, 52)) { ok = false; break; }
        const unsigned char* crow = sm + L.codes + cs * L.codes_stage_bytes + srow * (kSG * CB) + half * (CB / 2);
        uint4 outv[kSG][4];
#pragma unroll
        for (int g = 0; g < kSG; ++g) {
          if (BITS == 4) {
            unpack32_u4(*reinterpret_cast<const uint4*>(crow + g * CB), outv[g]);
          } else {
            unpack32_u8(*reinterpret_cast<const uint4*>(crow + g * CB), *reinterpret_cast<const uint4*>(crow + g * CB + 16),
                        outv[g]);
          }
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&cempty[cs]);  // codes read: the slot can be refilled
#pragma unroll
        for (int g = 0; g < kSG; ++g) {
          unsigned char* arow = sm + L.a + as * kAStageBytes + g * kATileBytes + (m >> 3) * 1024 + (m & 7) * 128;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int chunk = half * 4 + q;
            *reinterpret_cast<uint4*>(arow + ((chunk ^ (m & 7)) << 4)) = outv[g][q];
          }
        }
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&afull[as]);
      }
      if (!ok) break;
    }
  } else if (warp >= kEpiWarp0) {
    // ------------------------------------------------ scalers + epilogue (four independent warps)
    const int q = warp & 3;         // TMEM lane quarter
    const int m = 32 * q + lane;    // accumulator row held by this thread
    const int srow = (MODE == 0) ? ((m & 1) * 64 + (m >> 1)) : m;
    float* xs = reinterpret_cast<float*>(sm + L.xs) + q * ng * kNT;  // this warp's [ng][kNT]
    int sg = 0, it = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++it) {
      if (warp_aborted(abort)) break;
      const int ci = t / MT, mt = t % MT;
      const int start = p.chunks[3 * ci + 1], cnt = p.chunks[3 * ci + 2];
      const int tb = it & 1, tu = it >> 1;
      // group sums of the tile's columns (the down GEMM's come as 4 partial sums, added in order)
      // (the chunk's sums are contiguous: [cnt][ng] floats, or [cnt][ng][4] partials; 8 vector
      // loads per lane in flight at a time)
      __syncwarp();
      {
        const float4* src = reinterpret_cast<const float4*>(p.xs_in + static_cast<size_t>(start) * ng * (MODE == 0 ? 1 : 4));
        const int nvec = (MODE == 0) ? (cnt * ng) / 4 : cnt * ng;
#pragma unroll 1
        for (int v0 = 0; v0 < nvec; v0 += 32 * 8) {
          float4 f[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int qq = v0 + u * 32 + lane;
            if (qq < nvec) f[u] = __ldg(src + qq);
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int qq = v0 + u * 32 + lane;
            if (qq < nvec) {
              if (MODE == 0) {
                const int n = (4 * qq) / ng, g = (4 * qq) % ng;
                xs[g * kNT + n] = f[u].x;
                xs[(g + 1) * kNT + n] = f[u].y;
                xs[(g + 2) * kNT + n] = f[u].z;
                xs[(g + 3) * kNT + n] = f[u].w;
              } else {
                const int n = qq / ng, g = qq % ng;
                xs[g * kNT + n] = (f[u].x + f[u].y) + (f[u].z + f[u].w);
              }
            }
          }
        }
      }
      __syncwarp();
      if (!warp_wait(&scfull[tb], tu & 1, p.hdr, abort, 60)) break;
      const uint16_t* scs = reinterpret_cast<const uint16_t*>(sm + L.sc + tb * L.sc_buf_bytes);
      const uint16_t* bis = scs + 2 * 64 * ng;
      float acc[kNT];
#pragma unroll
      for (int n = 0; n < kNT; ++n) acc[n] = 0.f;
      bool ok = true;
      for (int st = 0; st < nst; ++st, ++sg) {
        const int ps = sg % kPS, pu = sg / kPS;
        if (!warp_wait(&pfull[ps], pu & 1, p.hdr, abort, 61)) { ok = false; break; }
        tc::fence_after_sync();
        const uint32_t tq = tmem + (static_cast<uint32_t>(32 * q) << 16) + ps * kSG * kNT;
        const int g0 = st * kSG;
        const float sc0 = bf16_to_f32(scs[srow * ng + g0]);
        const float bi0 = bf16_to_f32(bis[srow * ng + g0]);
        const float sc1 = bf16_to_f32(scs[srow * ng + g0 + 1]);
        const float bi1 = bf16_to_f32(bis[srow * ng + g0 + 1]);
        const float* x0 = xs + g0 * kNT;
        // columns in halves of 16 (the upper half only when the chunk has more than 16 pairs)
#pragma unroll
        for (int hf = 0; hf < kNT / 16; ++hf) {
          if (hf * 16 < cnt) {
            uint32_t v0[16], v1[16];
            tc::tmem_ld16(tq + hf * 16, v0);
            tc::tmem_ld16(tq + kNT + hf * 16, v1);
            tc::tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const int n = hf * 16 + c;
              if (n < cnt) {
                acc[n] = fmaf(sc0, __uint_as_float(v0[c]), fmaf(bi0, x0[n], acc[n]));
                acc[n] = fmaf(sc1, __uint_as_float(v1[c]), fmaf(bi1, x0[kNT + n], acc[n]));
              }
            }
          }
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&pempty[ps]);
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&scempty[tb]);
      if (MODE == 0) {
        // rows 2i (gate) and 2i+1 (up) of intermediate index mt*64 + i
        const int i = mt * 64 + (m >> 1);
        const int ip = (BITS == 4) ? ((i & ~7) | perm8_pos(i & 7)) : i;
        float* hv = acc;  // h replaces the accumulators column by column
#pragma unroll
        for (int n = 0; n < kNT; ++n) {
          const float u = __shfl_xor_sync(0xffffffffu, acc[n], 1);
          float h = 0.f;
          if (!(m & 1) && n < cnt) {
            h = silu_f(acc[n]) * u;
            const __half hi = __float2half_rn(h);
            const __half lo = __float2half_rn(h - __half2float(hi));
            const size_t o = static_cast<size_t>(start + n) * p.ldh + ip;
            p.h_hi[o] = __half_as_ushort(hi);
            p.h_lo[o] = __half_as_ushort(lo);
          }
          hv[n] = h;
        }
        // this warp's share (16 intermediate indices) of the group sum of h, every column at
        // once: a butterfly reduce-scatter leaves lane n with the sum of column n
        static_assert(kNT == 32, "one column per lane");
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
          const bool upper = (lane & o) != 0;
#pragma unroll
          for (int i2 = 0; i2 < o; ++i2) {
            const float send = upper ? hv[i2] : hv[i2 + o];
            const float keep = upper ? hv[i2 + o] : hv[i2];
            hv[i2] = keep + __shfl_xor_sync(0xffffffffu, send, o);
          }
        }
        if (lane < cnt) p.hsum_out[(static_cast<size_t>(start + lane) * (p.I / 64) + mt) * 4 + q] = hv[0];
      } else {
        const int r = mt * kBM + m;
#pragma unroll
        for (int n = 0; n < kNT; ++n) {
          if (n < cnt) {
            const int pid = __ldg(p.perm + start + n);
            p.out[static_cast<size_t>(pid) * p.H + r] = acc[n];
          }
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kPS * kSG * kNT);
  }
}

// ------------------------------------------------------------------ gather, combine

// X16[pos][:] = fp16(x[token(pos)][:]) for every sorted pair, K order permuted for
// 4-bit codes; gate[t] = sigmoid(x[t] . w_sg) for the shared expert.
__global__ void __launch_bounds__(256) gather_kernel(BatchParams p) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  const int npairs = p.T * p.k + (p.Is > 0 ? p.T : 0);
  constexpr int kRun = 8;  // segments of a row loaded by a lane before any is converted
  for (int pos = warp; pos < npairs; pos += nwarps) {
    const int pid = p.perm[pos];
    const int t = (pid < p.T * p.k) ? pid / p.k : pid - p.T * p.k;
    const uint4* xr = reinterpret_cast<const uint4*>(p.x + static_cast<size_t>(t) * p.H);
    uint4* dst = reinterpret_cast<uint4*>(p.x16 + static_cast<size_t>(pos) * p.H);
    for (int s0 = lane; s0 < p.H / 8; s0 += 32 * kRun) {  // H % 256 == 0: every lane has a segment
      uint4 v[kRun];
#pragma unroll
      for (int u = 0; u < kRun; ++u)
        if (s0 + 32 * u < p.H / 8) v[u] = __ldg(xr + s0 + 32 * u);
#pragma unroll
      for (int u = 0; u < kRun; ++u) {
        const int s = s0 + 32 * u;
        if (s < p.H / 8) {  // the same for all lanes of the warp (H / 8 is a multiple of 32)
          const float f[8] = {bf16_lo(v[u].x), bf16_hi(v[u].x), bf16_lo(v[u].y), bf16_hi(v[u].y),
                              bf16_lo(v[u].z), bf16_hi(v[u].z), bf16_lo(v[u].w), bf16_hi(v[u].w)};
          __half o[8];
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) o[p.perm8 ? perm8_pos(kk) : kk] = __float2half_rn(f[kk]);
          dst[s] = *reinterpret_cast<const uint4*>(o);
          // sum of each group of 64 (8 segments, 8 consecutive lanes)
          float g = ((f[0] + f[1]) + (f[2] + f[3])) + ((f[4] + f[5]) + (f[6] + f[7]));
          g += __shfl_xor_sync(0xffffffffu, g, 1);
          g += __shfl_xor_sync(0xffffffffu, g, 2);
          g += __shfl_xor_sync(0xffffffffu, g, 4);
          if ((lane & 7) == 0) p.xs[static_cast<size_t>(pos) * (p.H / 64) + s / 8] = g;
        }
      }
    }
  }
  if (p.Is > 0) {
    for (int t = warp; t < p.T; t += nwarps) {
      const uint4* xr = reinterpret_cast<const uint4*>(p.x + static_cast<size_t>(t) * p.H);
      const uint4* wr = reinterpret_cast<const uint4*>(p.wsg);
      float a = 0.f;
      for (int s = lane; s < p.H / 8; s += 32) {
        const uint4 xa = xr[s], wa = wr[s];
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
      if (lane == 0) p.sgate[t] = 1.f / (1.f + expf(-a));
    }
  }
}

// y[t][r] = bf16( sum_j w[t][j] * O[t*k+j][r] + gate[t] * O[T*k+t][r] ), rank order, shared last.
// Each thread four consecutive rows of one token (16-byte loads), all k (+1) pair rows loaded before
// the first multiply; the sum in rank order, the shared expert last, as one fma chain per row.
__global__ void __launch_bounds__(256) combine_kernel(BatchParams p) {
  constexpr int kMaxSlots = 17;  // k <= 16, plus the shared expert
  const size_t n4 = static_cast<size_t>(p.T) * p.H / 4;
  const int ns = p.k + (p.Is > 0 ? 1 : 0);
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>((4 * i) / p.H), r = static_cast<int>((4 * i) % p.H);
    float4 v[kMaxSlots];
#pragma unroll
    for (int j = 0; j < kMaxSlots; ++j)
      if (j < ns) {
        const size_t pid = j < p.k ? static_cast<size_t>(t) * p.k + j : static_cast<size_t>(p.T) * p.k + t;
        v[j] = __ldg(reinterpret_cast<const float4*>(p.o + pid * p.H + r));
      }
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < kMaxSlots; ++j)
      if (j < ns) {
        const float c = j < p.k ? p.w[static_cast<size_t>(t) * p.k + j] : p.sgate[t];
        acc.x = fmaf(c, v[j].x, acc.x);
        acc.y = fmaf(c, v[j].y, acc.y);
        acc.z = fmaf(c, v[j].z, acc.z);
        acc.w = fmaf(c, v[j].w, acc.w);
      }
    uint2 packed;
    packed.x = static_cast<uint32_t>(f32_to_bf16(acc.x)) | (static_cast<uint32_t>(f32_to_bf16(acc.y)) << 16);
    packed.y = static_cast<uint32_t>(f32_to_bf16(acc.z)) | (static_cast<uint32_t>(f32_to_bf16(acc.w)) << 16);
    *reinterpret_cast<uint2*>(p.y + 4 * i) = packed;
  }
}

template <int MODE, int BITS>
cudaError_t launch_gemm_t(const GemmParams& g, int grid, cudaStream_t st) {
  const GemmSmem L = gemm_smem(MODE, BITS, g.K);
  auto kern = grouped_gemm_kernel<MODE, BITS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(L.total));
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, L.total, st>>>(g);
  return cudaGetLastError();
}

}  // namespace

size_t grouped_gemm_smem(int mode, int bits, int K, int group) {
  (void)group;
  return gemm_smem(mode, bits, K).total;
}

cudaError_t launch_grouped_gemm(const GemmParams& g, int mode, int bits, int grid, cudaStream_t st) {
  if (mode == 0) return bits == 4 ? launch_gemm_t<0, 4>(g, grid, st) : launch_gemm_t<0, 8>(g, grid, st);
  return bits == 4 ? launch_gemm_t<1, 4>(g, grid, st) : launch_gemm_t<1, 8>(g, grid, st);
}

cudaError_t launch_gather(const BatchParams& p, int grid, cudaStream_t st) {
  gather_kernel<<<grid, 256, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_combine(const BatchParams& p, int grid, cudaStream_t st) {
  combine_kernel<<<grid, 256, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace moe
