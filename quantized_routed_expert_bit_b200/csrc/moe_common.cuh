// Device helpers shared by the sm_100a kernels of the routed-MoE library:
// bf16 bit handling, warp reductions, the workspace status word, mbarrier
// waits with a time limit, and bulk (TMA engine) global->shared copies.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_b200.h"

namespace moe {

constexpr int kWarp = 32;

// Workspace header: status word, the routing counters, then the buffers.
struct WsHeader {
  int32_t status;          // first device error (moe_status), 0 = none
  int32_t detail;          // kernel-specific detail of that error
  int32_t pad[14];
};

// Device-side view of the parts of the workspace the kernels touch.
struct WsView {
  WsHeader* hdr;
  uint32_t* counters;     // [n_counters], self-resetting arrival counters
  float* logits;          // [T][E] router logits
  float* sgate;           // [T] sigmoid gate of the shared expert
  float* h;               // [T][k+1][Imax] SwiGLU outputs
};

// ---------------------------------------------------------------- bf16

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// fp32 -> bf16, round to nearest even (NaN kept quiet).
__device__ __forceinline__ uint16_t f32_to_bf16(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) return static_cast<uint16_t>((u >> 16) | 0x40u);
  u += 0x7fffu + ((u >> 16) & 1u);
  return static_cast<uint16_t>(u >> 16);
}

// ---------------------------------------------------------------- warps

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// ---------------------------------------------------------------- status

__device__ __forceinline__ void report(WsHeader* hdr, int code, int detail) {
  if (atomicCAS(&hdr->status, 0, code) == 0) atomicExch(&hdr->detail, detail);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Upper bounds of every spin in this library: a wait gives up after
// kWaitNs of wall time or kWaitIters polls, whichever comes first.
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s
constexpr uint32_t kWaitIters = 1u << 26;

// ---------------------------------------------------------------- mbarrier + bulk copies

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Makes mbarrier initialisation visible to the async proxy (bulk copies).
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

// One test of phase `parity`; if it is not complete the thread may be
// suspended (up to the hint, 0.5 ms) until it completes, instead of spinning
// and taking issue slots from the warps doing the work.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity), "r"(500000u)
      : "memory");
  return ok != 0;
}

// Bounded wait on phase `parity` of an mbarrier. Returns false (and records
// MOE_ERR_TIMEOUT with `where`) if the limit ran out.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, WsHeader* hdr, int where) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0; it < kWaitIters; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > kWaitNs) break;
  }
  report(hdr, MOE_ERR_TIMEOUT, where);
  return false;
}

// Bulk copy of `bytes` (multiple of 16, both addresses 16-byte aligned) from
// global to this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// 128-bit global load that bypasses L1 allocation (streamed weights).
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// ---------------------------------------------------------------- dequant dot products
//
// The weight of a code q in group g is s_g*q + b_g, so a group's share of a
// dot product is  s_g * sum(q x) + b_g * sum(x),  with sum(x) per 16-byte
// segment of codes computed once. sum(q x) is formed from exact integers:
// a code sitting at bits [p, p+w) of a word becomes the fp32 number M + q,
// M = 2^(23-p), by OR-ing the masked word into the bits of M (one lop3/prmt,
// no int->float conversion); subtracting M gives q exactly, and q*x is an
// exact product accumulated in fp32. Pairs of codes go through the packed
// fp32x2 add and fma of sm_100.

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }
__device__ __forceinline__ float fb(uint32_t u) { return __uint_as_float(u); }

// sum over the 8 codes of one 32-bit word of 4-bit codes of q * x (x: 8 floats),
// accumulated into the pair acc.
__device__ __forceinline__ float2 dot8_u4(uint32_t w, const float* x, float2 acc) {
  const uint32_t v = w >> 12;  // codes 5, 6, 7 move to bits 8, 12, 16
  // M + q for code positions 0, 4, 8, 12, 16: M = 2^23, 2^19, 2^15, 2^11, 2^7
  const float2 f01 = f2(fb((w & 0xFu) | 0x4B000000u), fb((w & 0xF0u) | 0x49000000u));
  const float2 f23 = f2(fb((w & 0xF00u) | 0x47000000u), fb((w & 0xF000u) | 0x45000000u));
  const float2 f45 = f2(fb((w & 0xF0000u) | 0x43000000u), fb((v & 0xF00u) | 0x47000000u));
  const float2 f67 = f2(fb((v & 0xF000u) | 0x45000000u), fb((v & 0xF0000u) | 0x43000000u));
  acc = __ffma2_rn(__fadd2_rn(f01, f2(-8388608.f, -524288.f)), f2(x[0], x[1]), acc);
  acc = __ffma2_rn(__fadd2_rn(f23, f2(-32768.f, -2048.f)), f2(x[2], x[3]), acc);
  acc = __ffma2_rn(__fadd2_rn(f45, f2(-128.f, -32768.f)), f2(x[4], x[5]), acc);
  acc = __ffma2_rn(__fadd2_rn(f67, f2(-2048.f, -128.f)), f2(x[6], x[7]), acc);
  return acc;
}

// sum over the 4 codes of one 32-bit word of 8-bit codes of q * x (x: 4 floats).
// Each byte is permuted into bits 8..15 under the exponent of 2^15.
__device__ __forceinline__ float2 dot4_u8(uint32_t w, const float* x, float2 acc) {
  constexpr uint32_t kM = 0x47000000u;  // 2^15, exponent byte in byte 3
  const float2 f01 = f2(fb(__byte_perm(w, kM, 0x7504)), fb(__byte_perm(w, kM, 0x7514)));
  const float2 f23 = f2(fb(__byte_perm(w, kM, 0x7524)), fb(__byte_perm(w, kM, 0x7534)));
  acc = __ffma2_rn(__fadd2_rn(f01, f2(-32768.f, -32768.f)), f2(x[0], x[1]), acc);
  acc = __ffma2_rn(__fadd2_rn(f23, f2(-32768.f, -32768.f)), f2(x[2], x[3]), acc);
  return acc;
}

template <int BITS>
struct CodeTraits;
template <>
struct CodeTraits<4> {
  static constexpr int kPerSeg = 32;  // codes per 16-byte segment
};
template <>
struct CodeTraits<8> {
  static constexpr int kPerSeg = 16;
};

// sum over one 16-byte segment of codes of q * x[i] (x: kPerSeg floats).
template <int BITS>
__device__ __forceinline__ float dot_seg(const uint4& c, const float* x) {
  float2 acc = f2(0.f, 0.f);
  if constexpr (BITS == 4) {
    acc = dot8_u4(c.x, x + 0, acc);
    acc = dot8_u4(c.y, x + 8, acc);
    acc = dot8_u4(c.z, x + 16, acc);
    acc = dot8_u4(c.w, x + 24, acc);
  } else {
    acc = dot4_u8(c.x, x + 0, acc);
    acc = dot4_u8(c.y, x + 4, acc);
    acc = dot4_u8(c.z, x + 8, acc);
    acc = dot4_u8(c.w, x + 12, acc);
  }
  return acc.x + acc.y;
}

}  // namespace moe
