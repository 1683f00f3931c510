// Host-side launch interfaces between the C-ABI layer (moe_api.cu) and the
// kernels. Parameter blocks are passed by value to the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_common.cuh"

namespace moe {

constexpr int kRouteTokTile = 8;  // tokens per router CTA tile (one counter each)

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

struct SortParams {
  const int32_t* idx;    // [T][k]
  int T, k, E, with_shared;
  int32_t* perm;         // [T*k (+T)]
  int32_t* offsets;      // [E+1 (+1)]
  WsHeader* hdr;
};

cudaError_t launch_route_topk(const RouteParams& p, cudaStream_t stream);
cudaError_t launch_expert_ffn(const FfnParams& p, int bits, cudaStream_t stream);
cudaError_t launch_glue(const GlueParams& p, cudaStream_t stream);
cudaError_t launch_sort_by_expert(const SortParams& p, cudaStream_t stream);

}  // namespace moe
