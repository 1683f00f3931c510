// Host-side launch interfaces between the C-ABI layer (moe_api.cu) and the
// kernels. Parameter blocks are passed by value to the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_common.cuh"

namespace moe {

constexpr int kRouteTokTile = 8;  // tokens per router CTA tile (one counter each)
constexpr int kRouteMmaMinTokens = 64;  // from this many tokens the router runs on the tensor cores

struct SortParams {
  const int32_t* idx;    // [T][k]
  int T, k, E, with_shared;
  int32_t* perm;         // [T*k (+T)]
  int32_t* offsets;      // [E+1 (+1)]
  int32_t* chunks;       // optional [max][3]: expert, first sorted position, pair count (<= chunk_tokens)
  int32_t* nchunks;      // optional scalar
  int chunk_tokens;
  WsHeader* hdr;
};

struct RouteParams {
  const uint16_t* x;     // bf16 [T][H]
  const uint16_t* wr;    // bf16 [E][H]
  const float* rbias;    // fp32 [E] or null
  int T, H, E, k, renorm;
  int32_t* idx_out;      // [T][k]
  float* w_out;          // [T][k]
  WsView ws;
};

// One group of E quantised matrices [rows][K] (device pointers).
struct QMat {
  const uint8_t* q;
  const uint16_t* s;
  const uint16_t* b;
  int64_t q_stride;   // bytes per expert
  int64_t sb_stride;  // elements per expert
  // gate/up matrices: where an expert's up rows start, from its gate rows (codes in bytes, scales
  // and biases in elements): I rows further on in the packed layout, the distance to the separate
  // up tensors in the stock layout (moe_layer_weights.up); 0 for the down matrices
  int64_t up_q;
  int64_t up_s;
  int64_t up_b;
};

struct FfnParams {
  const uint16_t* x;        // bf16 [T][H]
  const int32_t* idx;       // [T][k]
  const float* w;           // [T][k]
  uint16_t* y;              // bf16 [T][H]
  QMat gate_up, down, sh_gate_up, sh_down;
  const uint16_t* wsg;      // bf16 [H] shared-expert gate vector (when Is > 0)
  int T, H, E, k, I, Is, group, Imax;
  WsView ws;
};

struct GlueParams {
  float* r;              // fp32 [T][H] residual stream (updated in place)
  const uint16_t* y;     // bf16 [T][H] layer output (null: initialise r from x_in)
  const uint16_t* x_in;  // bf16 [T][H] initial input (only when y is null)
  uint16_t* x_out;       // bf16 [T][H] next layer input
  int T, H;
  float eps;
};


constexpr int kChunkTokens = 32;  // pairs per GEMM chunk (the MMA N dimension)

// Batched path: gather of the sorted pairs' activations and the final combine.
struct BatchParams {
  const uint16_t* x;     // bf16 [T][H]
  const uint16_t* wsg;   // bf16 [H] shared-expert gate vector (when Is > 0)
  const int32_t* perm;   // [npairs] sorted position -> pair id
  int T, k, H, Is, perm8;
  uint16_t* x16;         // fp16 [npairs][H], K permuted in blocks of 8 when perm8
  float* xs;             // fp32 [npairs][H/64] sums of x over each group of 64
  float* sgate;          // [T]
  const float* w;        // [T][k] routing weights
  const float* o;        // fp32 [npairs by pair id][H] expert outputs
  uint16_t* y;           // bf16 [T][H]
};

// One grouped GEMM launch (gate/up + SwiGLU, or down) over expert chunks.
struct GemmParams {
  CUtensorMap tm_codes[2];   // 3D codes maps: [0] routed experts, [1] shared expert
  CUtensorMap tm_scales[2];
  CUtensorMap tm_biases[2];
  CUtensorMap tm_b[4];       // B operand [npairs][K] fp16, box rows 16/32/64/128, 128-byte swizzle
  CUtensorMap tm_b2[4];      // second B operand (h lo) of the down GEMM
  const int32_t* chunks;
  const int32_t* nchunks;
  const int32_t* perm;
  const float* xs_in;        // group sums of the B operand: x [npairs][K/64], or h as 4 partials [npairs][K/64][4]
  int K, rows, I, H, E, group, ldh;
  uint16_t* h_hi;            // gate/up output [npairs][ldh] fp16 hi / lo
  uint16_t* h_lo;
  float* hsum_out;           // gate/up output [npairs][I/64][4] partial group sums of h (one per epilogue warp)
  float* out;                // down output [pair id][H] fp32
  WsHeader* hdr;
};

// One layer's weights for the persistent decode kernel.
struct LayerDesc {
  const uint16_t* wr;    // bf16 [E][H]
  const float* rbias;    // fp32 [E] or null
  const uint16_t* wsg;   // bf16 [H] shared-expert gate vector (when Is > 0)
  QMat gu, dn, sgu, sdn;
  const uint16_t* dsb;   // split kernel: group-major down (scale, bias) [E][I/group][H][2] (moe_prepare_down_sb)
  const uint16_t* sdsb;  // the same for the shared expert [1][Is/group][H][2]
  const uint8_t* dcu;    // split kernel: unit-major down codes [E][I/32][H][32*bits/8] (moe_prepare_down_units)
  const uint8_t* sdcu;   // the same for the shared expert
};

constexpr int kMaxDecodeLayers = 48;   // layers per launch (kernel parameter space)
constexpr int kDecodeReplicas = 4;     // copies of each exchange word (spreads the readers over more lines)
constexpr int kDecodeYBufs = 3;        // y accumulator buffers of the split kernel, used by layers in turn

// Parameters of both persistent decode kernels: decode_stack_kernel (exchanges
// h between CTAs) and decode_split_kernel (keeps h in the CTA and reduces y).
struct DecodeParams {
  int L, l0;             // layers in this launch; index of its first layer in the stack
  int H, E, k, I, Is, group, renorm;
  float eps;
  const uint16_t* x0;    // bf16 [H] input of the first layer
  const float* r_in;     // fp32 [H] residual at the first layer, or null (= x0)
  uint16_t* out;         // bf16 [H]
  float* r_out;          // fp32 [H] residual after the last layer, or null
  uint16_t* tr_x;        // bf16 [layers][H] or null
  int32_t* tr_idx;       // [layers][k] or null
  float* tr_w;           // [layers][k] or null
  uint16_t* tr_y;        // bf16 [layers][H] or null
  uint64_t* tr_t;        // [layers][8] phase timestamps of CTA 0, or null
  int tr_rows;           // trace rows per layer (the call's tokens, run one launch each; 1 for one token)
  // exchange words between CTAs (workspace), zero at launch; each written to
  // kDecodeReplicas copies (`*_rep` words apart), CTA c reads copy c % kDecodeReplicas
  uint32_t* logits;      // [E+1] fp32 logits, last mantissa bit = layer parity
  uint32_t* hbuf;        // [k+1][I] fp32 SwiGLU outputs, last mantissa bit = layer parity (exchange kernel)
  uint32_t* ybuf;        // [H] bf16 layer output << 16 | 16-bit layer tag (exchange kernel)
  int logits_rep, h_rep, y_rep;
  // split kernel: y partial sums [kDecodeYBufs][kDecodeReplicas][yrep] fp32 (16-byte aligned;
  // CTA c adds into copy c % kDecodeReplicas, readers sum the copies) and the arrival counter
  float* yacc;
  int yrep;
  int split_late;        // split kernel: down codes copied into the first gate/up batch's space once it is read
  int split_two;         // split kernel: more units than CTAs (some CTAs take two: a second down buffer)
  int64_t ybuf_stride;   // floats between buffers (kDecodeReplicas * yrep)
  uint32_t* arrive;
  WsHeader* hdr;
  LayerDesc layers[kMaxDecodeLayers];
  // split kernel: 3D maps (row bytes, H rows, experts) over the down codes of the routed and
  // the shared experts, box (one unit's bytes, 256 rows, 1)
  CUtensorMap tm_dn[kMaxDecodeLayers];
  CUtensorMap tm_sdn[kMaxDecodeLayers];
};

// Grouped GEMV (csrc/grouped_gemv.cu): the batched path on the CUDA cores for a few tokens per
// expert. A work item is (chunk of <= kGvTPI pairs of one expert, group of upi 32-column units);
// upi (1, 2 or kGvUPI) is gemv_units_per_item's choice for the batch size.
constexpr int kGvTPI = 4;  // pairs per chunk

// Words per 16-byte code segment in the per-token quad table of the grouped GEMV (xq_token): the
// 2 * 32 / BITS quad words (two byte planes of 16-bit fixed point) and the segment's sum, padded
// to 4 m words with m odd, so that each segment starts on 16 bytes and the 16-byte loads of 8
// consecutive segments (one shared-memory phase) hit distinct banks.
template <int BITS>
__host__ __device__ constexpr int xq_stride() {
  return 4 * ((((2 * (32 / BITS) + 1) + 3) / 4) | 1);
}
constexpr int kGvUPI = 4;  // most units per item
constexpr int kGvItemsTarget = 128;  // work items wanted per launch: about one per SM of a 148-SM part

// Units per work item for T tokens: the largest of 4, 2, 1 whose item count reaches
// kGvItemsTarget with one chunk per distinct expert (fewer units per item split the experts of a
// small batch over more CTAs, at the cost of more partial outputs to combine).
inline int gemv_units_per_item(int T, int k, int E, int I, int Is) {
  const long np = static_cast<long>(T) * k + (Is > 0 ? T : 0);
  const long est = np < E + (Is > 0 ? 1 : 0) ? np : E + (Is > 0 ? 1 : 0);
  for (int u = kGvUPI; u > 1; u >>= 1)
    if (est * (I / (32 * u)) >= kGvItemsTarget) return u;
  return 1;
}
struct GemvParams {
  const int32_t* chunks;   // [nchunks][3]: expert (E = shared), first sorted position, pair count
  const int32_t* nchunks;
  const int32_t* perm;     // sorted position -> pair id
  const uint32_t* xq;      // [T][H / codes-per-16-bytes][quad words + 1] fixed-point x of every token
  const float* xsc;        // [T] 2^-S of every token's x
  QMat gu, dn, sgu, sdn;
  const uint8_t* dcu;      // unit-major down codes (moe_prepare_down_units) or null
  const uint8_t* sdcu;
  const uint16_t* dsb;     // group-major down scales and biases (moe_prepare_down_sb) or null
  const uint16_t* sdsb;
  CUtensorMap tm_dn, tm_sdn;  // canonical down codes (when dcu / sdcu are null)
  float* o;                // [I / (32 upi)][npairs][H] partial expert outputs by pair id
  int T, k, H, E, I, group, npairs, upi;
  WsHeader* hdr;
};
bool grouped_gemv_supported(int H, int I, int Is, int group, int bits, size_t smem_limit);
size_t grouped_gemv_smem(int H, int I, int group, int bits);
cudaError_t launch_xquant(const uint16_t* x, const uint16_t* wsg, int T, int H, int Is, int bits, uint32_t* xq,
                          float* xsc, float* sgate, cudaStream_t st);
cudaError_t launch_grouped_gemv(const GemvParams& p, int bits, int grid, cudaStream_t st);
cudaError_t launch_gv_combine(const float* o, const float* w, const float* sgate, int T, int k, int H, int Is, int nq,
                              int npairs, uint16_t* y, int grid, cudaStream_t st);

cudaError_t launch_route_topk(const RouteParams& p, cudaStream_t stream);
cudaError_t launch_expert_ffn(const FfnParams& p, int bits, cudaStream_t stream);
cudaError_t launch_glue(const GlueParams& p, cudaStream_t stream);
cudaError_t launch_sort_by_expert(const SortParams& p, cudaStream_t stream);

size_t grouped_gemm_smem(int mode, int bits, int K, int group);
cudaError_t launch_grouped_gemm(const GemmParams& g, int mode, int bits, int grid, cudaStream_t st);
cudaError_t launch_gather(const BatchParams& p, int grid, cudaStream_t st);
cudaError_t launch_combine(const BatchParams& p, int grid, cudaStream_t st);

bool decode_stack_supported(int H, int E, int k, int I, int Is, int group, int bits);
size_t decode_stack_smem(int H, int E, int k, int I, int Is, int group, int bits, int grid);
// The split kernel: whether it runs this shape on `grid` CTAs within `smem_limit` bytes of
// shared memory for launches of up to L layers, and its shared memory.
bool decode_split_plan(int H, int E, int k, int I, int Is, int group, int bits, int grid, int L, size_t smem_limit,
                       size_t* smem, int* late, int* two = nullptr);
cudaError_t launch_decode_split(const DecodeParams& p, int bits, int grid, cudaStream_t stream);
cudaError_t launch_decode_stack(const DecodeParams& p, int bits, int grid, cudaStream_t stream);
cudaError_t launch_wait_limit_check(WsHeader* hdr, uint32_t* never_set, int32_t* gave_up, cudaStream_t stream);
// Group-major copy of one down tensor's scales and biases: out[e][g][r][0..1] = (scale, bias) of row r,
// group g of expert e (n experts of `rows` rows and ngroups groups, expert stride `stride` elements).
// Unit-major copy of one down tensor's codes: out[e][u][r][0..ub) = codes of columns [32u, 32u+32) of row r
// (ub = 32*bits/8 bytes; n experts of `rows` rows of rowb bytes, expert stride q_stride bytes).
cudaError_t launch_prepare_down_units(const uint8_t* q, int64_t q_stride, int n, int rows, int rowb, int ub,
                                      uint8_t* out, cudaStream_t stream);
cudaError_t launch_prepare_down_sb(const uint16_t* scales, const uint16_t* biases, int64_t stride, int n, int rows,
                                   int ngroups, uint16_t* out, cudaStream_t stream);

}  // namespace moe
