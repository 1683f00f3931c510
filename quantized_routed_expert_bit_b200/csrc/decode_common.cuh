// Device helpers of the two persistent decode kernels (stack_decode.cu,
// stack_split.cu): bulk and per-thread copies, relaxed exchange words, the
// bounded poll, the dequantising dot products of one 16-byte code segment,
// and the warp top-k.
#pragma once

#include "moe_common.cuh"
#include "moe_launch.h"

namespace moe {
namespace {

__device__ __forceinline__ void copy_tx(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("mbarrier.expect_tx.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
  bulk_g2s(dst, src, bytes, bar);
}

__device__ __forceinline__ void mbar_arrive1(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Per-thread asynchronous 16-byte global -> shared copy (L2 only), and the wait for all of this
// thread's outstanding ones.
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void prefetch_line_l2(const void* a) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(a));
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

// Between two polls that found a word not yet written (each poll is one L2
// round trip, no sleep): every 16 polls ask give_up.
#define MOE_POLL_BACKOFF(it, t0, hdr, where, fail) \
  {                                                \
    if ((it) == 0) (t0) = globaltimer_ns();        \
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

// Dot products of one 16-byte code segment with the matching x (or h) values.
// 8-bit codes: dot_seg<8> (each byte permuted under the exponent of 2^15).
// 4-bit codes: each 32-bit word is first split into its even and odd nibbles
// as bytes (two lop3), then every byte goes under the exponent of 2^15 like an
// 8-bit code: one shared magic constant, so pairs of codes take the packed
// fp32x2 subtract and fma with no register shuffling. The codes of a word
// then come out in the order 0,2,4,6,1,3,5,7, and the values they multiply
// are stored in that order (seg_pos): a dot product does not depend on the
// order of its terms, and each q*x stays exact.
template <int BITS>
__host__ __device__ constexpr int seg_pos(int o) {
  return BITS == 4 ? ((o & ~7) | (((o & 7) >> 1) + 4 * (o & 1))) : o;
}

__device__ __forceinline__ float2 dot8_u4_split(uint32_t w, const float* x, float2 acc) {
  constexpr uint32_t kM = 0x47000000u;  // 2^15
  const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
  const float2 km = f2(-32768.f, -32768.f);
  acc = __ffma2_rn(__fadd2_rn(f2(fb(__byte_perm(lo, kM, 0x7504)), fb(__byte_perm(lo, kM, 0x7514))), km), f2(x[0], x[1]), acc);
  acc = __ffma2_rn(__fadd2_rn(f2(fb(__byte_perm(lo, kM, 0x7524)), fb(__byte_perm(lo, kM, 0x7534))), km), f2(x[2], x[3]), acc);
  acc = __ffma2_rn(__fadd2_rn(f2(fb(__byte_perm(hi, kM, 0x7504)), fb(__byte_perm(hi, kM, 0x7514))), km), f2(x[4], x[5]), acc);
  acc = __ffma2_rn(__fadd2_rn(f2(fb(__byte_perm(hi, kM, 0x7524)), fb(__byte_perm(hi, kM, 0x7534))), km), f2(x[6], x[7]), acc);
  return acc;
}

template <int BITS>
__device__ __forceinline__ float dot_seg_dec(const uint4& c, const float* x) {
  if constexpr (BITS == 4) {
    float2 acc = f2(0.f, 0.f);
    acc = dot8_u4_split(c.x, x + 0, acc);
    acc = dot8_u4_split(c.y, x + 8, acc);
    acc = dot8_u4_split(c.z, x + 16, acc);
    acc = dot8_u4_split(c.w, x + 24, acc);
    return acc.x + acc.y;
  } else {
    return dot_seg<8>(c, x);
  }
}

// Order-preserving map of a float to an unsigned key (larger float, larger key).
__device__ __forceinline__ unsigned fkey(float f) {
  const unsigned u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float fkey_inv(unsigned k) {
  return __uint_as_float((k & 0x80000000u) ? (k ^ 0x80000000u) : ~k);
}

// Top-k of one token's logits by one warp: lane l holds the logits of experts
// l, l+32, ... (PER of them, tagged fp32 words). Each lane sorts its keys once
// (larger logit first, then lower expert index); every round one warp-wide
// max over the lanes' heads picks the winner (lowest index among equal
// keys), whose lane pops its head. Lane j < k ends with the j-th pick.
template <int PER>
__device__ __forceinline__ void topk_sorted(const uint32_t* wl, int E, int k, int lane, unsigned& my_k, int& my_e,
                                            unsigned& kmax) {
  unsigned key[PER];
  int idx[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    idx[i] = lane + 32 * i;
    key[i] = (idx[i] < E) ? fkey(__uint_as_float(wl[i])) : 0u;
  }
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
  kmax = __reduce_max_sync(0xffffffffu, key[0]);
  my_k = 0u;
  my_e = 0;
#pragma unroll 1
  for (int j = 0; j < k; ++j) {
    const unsigned wk = __reduce_max_sync(0xffffffffu, key[0]);
    const unsigned we = __reduce_min_sync(0xffffffffu, key[0] == wk ? static_cast<unsigned>(idx[0]) : 0xffffffffu);
    if (lane == j) {
      my_k = wk;
      my_e = static_cast<int>(we);
    }
    if (static_cast<unsigned>(idx[0]) == we) {  // expert indices are unique across lanes: the owner pops
#pragma unroll
      for (int i = 0; i + 1 < PER; ++i) {
        key[i] = key[i + 1];
        idx[i] = idx[i + 1];
      }
      key[PER - 1] = 0u;
    }
  }
}

// ---------------------------------------------------------------- fixed-point dot products
//
// A group's share of a row's dot product is s_g * sum(q x) + b_g * sum(x). The activations are
// turned into integers X_i = rint(x_i * 2^S), S chosen from max|x| (fix_exp) so that |X| <= 2^22,
// split into three bytes X = 65536*X2 + 256*X1 + X0 (X2 signed), and sum(q X) is three exact
// integer sums of byte products (dp4a), recombined in fp32 once per 16-byte segment of codes.
// 4-bit codes are split into even and odd nibbles as bytes (two masks), so the activations are laid
// out in the same order: quad_pos gives where code position o of a segment sits among its quad bytes.

// Byte dot products: 4 unsigned code bytes times 4 signed (.s32) or unsigned (.u32) bytes, plus c.
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ uint32_t dp4a_uu(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("dp4a.u32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// sum over one 16-byte segment of codes of q * X (X given as its quads: q3[j][.] byte j of X; for
// 4-bit codes quads (2w, 2w+1) hold the even and odd elements of word w), as an fp32 number.
template <int BITS>
__device__ __forceinline__ float seg_dot(const uint4& c, const uint32_t* q2, const uint32_t* q1, const uint32_t* q0) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  int a2 = 0;
  uint32_t a1 = 0u, a0 = 0u;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if constexpr (BITS == 4) {
      const uint32_t lo = w[i] & 0x0F0F0F0Fu, hi = (w[i] >> 4) & 0x0F0F0F0Fu;
      a2 = dp4a_us(lo, q2[2 * i], a2);
      a2 = dp4a_us(hi, q2[2 * i + 1], a2);
      a1 = dp4a_uu(lo, q1[2 * i], a1);
      a1 = dp4a_uu(hi, q1[2 * i + 1], a1);
      a0 = dp4a_uu(lo, q0[2 * i], a0);
      a0 = dp4a_uu(hi, q0[2 * i + 1], a0);
    } else {
      a2 = dp4a_us(w[i], q2[i], a2);
      a1 = dp4a_uu(w[i], q1[i], a1);
      a0 = dp4a_uu(w[i], q0[i], a0);
    }
  }
  // |a2| < 2^20, a1 * 256 + a0 < 2^29: both exact in int, one fp32 rounding each
  return fmaf(static_cast<float>(a2), 65536.f, static_cast<float>(a1 * 256u + a0));
}

// Byte j (0, 1, 2) of the fixed-point value X (|X| < 2^23; byte 2 is the signed top byte).
__device__ __forceinline__ uint32_t xbyte(int X, int j) { return static_cast<uint32_t>(X >> (8 * j)) & 0xFFu; }

// Where code position o (0..PS-1) of a segment sits among the segment's quad bytes:
// quad index (word*2 + odd for 4-bit, word for 8-bit) * 4 + byte.
template <int BITS>
__host__ __device__ constexpr int quad_pos(int o) {
  return BITS == 4 ? ((o >> 3) * 2 + (o & 1)) * 4 + ((o & 7) >> 1) : o;
}

// 2^S with S chosen so that |x| < 2^22 * 2^-S for |x| <= m (a power of two, clamped to fp32 range).
__device__ __forceinline__ int fix_exp(float m) {
  if (!(m > 0.f)) return 0;
  int e = ((__float_as_uint(m) >> 23) & 0xFF) - 127;  // floor(log2 m) for normal m
  if (e < -100) e = -100;
  return 21 - e;
}
__device__ __forceinline__ float pow2f(int s) { return __uint_as_float(static_cast<uint32_t>(s + 127) << 23); }

}  // namespace
}  // namespace moe
