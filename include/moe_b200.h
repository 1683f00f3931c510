/*
 * moe_b200.h -- C ABI of the routed Mixture-of-Experts FFN for NVIDIA B200
 * (sm_100a), at decode time and for batches of tokens.
 *
 * What the library computes, per token x (bf16, hidden size H):
 *   1. router logits   l_e = x . Wr[e] (+ bias[e]) for all E experts;
 *   2. routing         softmax over all E, keep the k largest, renormalise
 *                      the k weights to sum to 1 (ties: lower expert index);
 *   3. per selected expert e: gu = dequant(GU_e) x with GU_e the packed
 *                      [2I][H] gate/up matrix (gate rows [0,I), up rows
 *                      [I,2I)), h = silu(gu[0:I]) * gu[I:2I], o_e = dequant(D_e) h;
 *   4. shared expert   o_s the same way with its own [2Is][H] and [H][Is]
 *                      matrices, gated by s = sigmoid(x . w_sg);
 *   5. combine         y = sum_j w_j o_{e_j} + s o_s, rounded once to bf16.
 * Sources: the routing fan-out (8 of 256 experts for the 35B model, 10 of
 * 512 for the 80B model; routers and shared experts resident) is in the
 * Swiftlet article (xix.ai, "Pacotes de Swiftlet 80B Qwen no Mac ..."),
 * paragraph 4, and the Runnel README, section "Target" (256 routed
 * experts, top-8, plus one shared expert); the MLX-style int4/int8 group
 * quantisation and the sparse MoE with shared experts are in the same
 * article, paragraph 8; the packed routed gate/up projection is in the
 * Runnel README, introduction and "Streaming CLI". The pages give no
 * formula; the steps above are the plain reading of them.
 *
 * Quantised matrices ("moe_qtensor"): E matrices [rows][K] at fixed
 * strides, one expert after the other (fixed-stride expert blocks: the
 * Swiftlet article, paragraph 4). Element k of a row belongs to group
 * k / group; its weight is  w = scale[g] * q + bias[g]  (bf16 scale and
 * bias, no zero-point). Codes run along K: 8-bit is one byte per element;
 * 4-bit is two elements per byte, the even element in the low nibble.
 * Row r of expert e starts at  q + e*q_expert_stride + r*K*bits/8  and its
 * scales/biases at  scales + e*sb_expert_stride + r*(K/group).
 *
 * Conventions for every call:
 *   - Tensor pointers are DEVICE pointers owned by the caller. The library
 *     allocates nothing; its scratch is the caller's workspace (`ws`,
 *     sized by moe_workspace_size and set up once by moe_workspace_init).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and is asynchronous; outputs are valid once the stream has
 *     reached that point.
 *   - Argument errors return at once, before anything is enqueued. Errors
 *     the device finds (an expert index outside [0,E) in the caller's
 *     topk_idx, a bounded wait that ran out) are recorded in a status word
 *     inside the workspace and read with moe_get_device_status; the kernel
 *     that found one skips the offending work and returns.
 *   - T = 0 is a no-op returning MOE_OK.
 *   - Calls that share a workspace must not run concurrently on the GPU.
 * Limits (else MOE_ERR_UNSUPPORTED): bits in {4, 8}; group in {32, 64};
 * H, I and Is multiples of group; 64 <= H <= 8192; I, Is <= 2048;
 * 1 <= k <= 16; k <= E <= 512; renorm in {0, 1}.
 * Alignment (else MOE_ERR_INVALID_ARG): x, y, router_w, shared_gate_w,
 * q, scales and biases 16-byte aligned; q_expert_stride a multiple of 16
 * bytes and sb_expert_stride a multiple of 8 elements, each at least one
 * expert's size.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ABI-identical to cudaStream_t; spelled out so this header needs no CUDA headers. */
typedef struct CUstream_st* moe_stream_t;

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* null/misaligned pointer, negative size, bad stride */
  MOE_ERR_UNSUPPORTED = 2, /* shape or format outside the limits above */
  MOE_ERR_WORKSPACE = 3,   /* workspace missing or smaller than moe_workspace_size */
  MOE_ERR_CUDA = 4,        /* a CUDA runtime call failed; see moe_last_error_string */
  MOE_ERR_TIMEOUT = 5,     /* (device) a bounded wait gave up */
  MOE_ERR_BOUNDS = 6       /* (device) an expert index outside [0, E) was skipped */
} moe_status;

/* Shape of one MoE layer. */
typedef struct {
  int32_t hidden;       /* H */
  int32_t num_experts;  /* E routed experts */
  int32_t top_k;        /* k experts per token */
  int32_t inter;        /* I, routed expert intermediate size */
  int32_t shared_inter; /* Is, shared expert intermediate size; 0 = no shared expert */
  int32_t bits;         /* 4 or 8 */
  int32_t group;        /* 32 or 64 elements per (scale, bias) along K */
  int32_t renorm;       /* 1: renormalise the k weights; 0: keep softmax probabilities */
} moe_config;

/* E quantised matrices [rows][K]; see the layout above. */
typedef struct {
  const uint8_t* q;          /* codes */
  const uint16_t* scales;    /* bf16 bit patterns [E][rows][K/group] */
  const uint16_t* biases;    /* bf16 bit patterns [E][rows][K/group] */
  int64_t q_expert_stride;   /* bytes from expert e to e+1 (64-bit: stacks exceed 2 GiB) */
  int64_t sb_expert_stride;  /* elements from expert e to e+1, scales and biases */
} moe_qtensor;

/* One layer's weights (all device memory). */
typedef struct {
  const uint16_t* router_w;      /* bf16 [E][H] */
  const float* router_bias;      /* fp32 [E] added to the logits before the softmax, or NULL */
  moe_qtensor gate_up;           /* E matrices [2I][H]: gate rows [0,I), up rows [I,2I) */
  moe_qtensor down;              /* E matrices [H][I] */
  moe_qtensor shared_gate_up;    /* 1 matrix [2Is][H] (ignored when shared_inter == 0) */
  moe_qtensor shared_down;       /* 1 matrix [H][Is] */
  const uint16_t* shared_gate_w; /* bf16 [H], the shared expert's sigmoid gate */
  /* Optional decode-ready copies of the down projections, written once at
   * load time (16-byte aligned). The single-token decode splits the
   * intermediate into units of 32 columns and reads, per unit, those 32
   * columns of all H down rows and their quantisation group's scale and
   * bias; in these layouts both are contiguous blocks:
   *   down_units     codes [E][I/32][H][32*bits/8]   (moe_prepare_down_units)
   *   down_sb        bf16 (scale, bias) [E][I/group][H][2] (moe_prepare_down_sb)
   * and shared_down_units / shared_down_sb the same for the shared expert
   * (E = 1, Is in place of I). NULL: the decode reads `down` / `shared_down`
   * in their canonical layout instead (same results, slower). The other
   * paths never read them. */
  const uint16_t* down_sb;
  const uint16_t* shared_down_sb;
  const uint8_t* down_units;
  const uint8_t* shared_down_units;
  /* Optional stock (unpacked) gate/up layout, the A/B baseline of the packed
   * routed gate/up (Runnel README, "Streaming CLI": --stock-mlp). When
   * up.q is non-NULL, gate_up holds only the gate rows, E matrices [I][H],
   * and up the up rows, E matrices [I][H], with the same expert strides as
   * gate_up (codes, and scales/biases); likewise shared_up / shared_gate_up
   * for the shared expert (shared_up.q non-NULL exactly when up.q is; a
   * mismatch, or strides that differ, is MOE_ERR_INVALID_ARG). Results are
   * the same as with the packed layout.
   * The tensor-core path reads the packed layout only: a call with stock
   * weights runs the grouped GEMV where it would run the tensor cores. */
  moe_qtensor up;
  moe_qtensor shared_up;
} moe_layer_weights;

/* Per-layer record of a stack run; any member may be NULL (not recorded). */
typedef struct {
  uint16_t* x;   /* bf16 [L][T][H] input of each layer */
  int32_t* idx;  /* [L][T][k] selected experts */
  float* w;      /* [L][T][k] routing weights */
  uint16_t* y;   /* bf16 [L][T][H] output of each layer */
  uint64_t* t;   /* [L][8] device clock (ns) at the phase boundaries of each layer as CTA 0 sees
                    them, single-token persistent path only. decode_split_kernel: 0 layer start,
                    1 x ready, 2 router rows done, 3 top-k done, 4 first gate/up batch landed,
                    5 down data landed, 6 down done, 7 arrival counted. decode_stack_kernel:
                    0 layer start, 1 router done, 2 routing barrier passed, 3 top-k done,
                    4 gate/up done, 5 h barrier passed, 6 down done, 7 y barrier passed */
} moe_trace;

/* Bytes of workspace the calls below need for T tokens (L is unused and
 * kept for callers that size one workspace per stack). 0 on bad config. */
MOE_API size_t moe_workspace_size(const moe_config* cfg, int32_t T, int32_t L);

/* Zeroes the workspace's status word and counters (asynchronously on
 * `stream`). Call once per new workspace before its first use. */
MOE_API moe_status moe_workspace_init(void* ws, size_t ws_bytes, moe_stream_t stream);

/* Steps 1-2 for T tokens. x bf16 [T][H]; router_w bf16 [E][H];
 * router_bias fp32 [E] or NULL. Writes topk_idx [T][k] and topk_w [T][k]
 * (fp32), each token's experts in descending weight. */
MOE_API moe_status moe_route_topk(const moe_config* cfg, const uint16_t* x, int32_t T,
                          const uint16_t* router_w, const float* router_bias,
                          int32_t* topk_idx, float* topk_w,
                          void* ws, size_t ws_bytes, moe_stream_t stream);

/* Steps 3-5 for T tokens given a selection: x bf16 [T][H], topk_idx [T][k],
 * topk_w [T][k] (fp32) -> y bf16 [T][H]. Indices outside [0, E) are
 * skipped and reported as MOE_ERR_BOUNDS by moe_get_device_status. */
MOE_API moe_status moe_expert_ffn(const moe_config* cfg, const moe_layer_weights* w,
                          const uint16_t* x, int32_t T,
                          const int32_t* topk_idx, const float* topk_w, uint16_t* y,
                          void* ws, size_t ws_bytes, moe_stream_t stream);

/* Steps 1-5: x bf16 [T][H] -> y bf16 [T][H], plus the selection
 * (topk_idx, topk_w [T][k]; either may be NULL if not wanted). */
MOE_API moe_status moe_layer_forward(const moe_config* cfg, const moe_layer_weights* w,
                             const uint16_t* x, int32_t T, uint16_t* y,
                             int32_t* topk_idx, float* topk_w,
                             void* ws, size_t ws_bytes, moe_stream_t stream);

/* L stacked layers (`layers` is a HOST array of L moe_layer_weights, one
 * configuration for all) joined by a residual stream with a parameter-free
 * RMSNorm, the pre-norm decoder the MoE block sits in:
 *   r_0 = x_0;  y_l = MoE_l(x_l);  r_{l+1} = r_l + y_l (fp32);
 *   x_{l+1} = bf16(r_{l+1} / sqrt(mean(r_{l+1}^2) + 1e-6)).
 * x0 bf16 [T][H] in, x_out = x_L bf16 [T][H] out. `trace` (host struct of
 * device pointers, may be NULL) records every layer. */
MOE_API moe_status moe_stack_forward(const moe_config* cfg, const moe_layer_weights* layers, int32_t L,
                             const uint16_t* x0, int32_t T, uint16_t* x_out,
                             const moe_trace* trace, void* ws, size_t ws_bytes,
                             moe_stream_t stream);

/* Number of kernel launches moe_stack_forward makes for T tokens and L
 * layers on the current device: up to the decode threshold
 * (moe_set_decode_max_tokens) each token runs the whole stack as one
 * persistent kernel (T launches per 48 layers) when the shape fits it; from
 * the batched threshold up (moe_set_batched_min_tokens) the batched path
 * (1 + 7*L) where it applies; from the GEMV threshold up
 * (moe_set_gemv_min_tokens) the grouped GEMV (1 + 6*L) where it applies;
 * otherwise 1 + 4*L. -1 on a bad configuration. */
MOE_API int32_t moe_stack_kernel_launches(const moe_config* cfg, int32_t T, int32_t L);

/* Name of the path moe_stack_forward takes for T tokens and L layers on the
 * current device (a static string): "decode_split_kernel" or
 * "decode_stack_kernel" (the persistent kernels, a token at a time), "batched" (the
 * grouped tensor-core path), "grouped_gemv" (a few tokens per expert, CUDA
 * cores), "per_layer" (four kernels per layer), "none"
 * (T or L is 0); NULL on a bad configuration. */
MOE_API const char* moe_stack_path_name(const moe_config* cfg, int32_t T, int32_t L);

/* Sets the token count from which moe_layer_forward, moe_expert_ffn and
 * moe_stack_forward take the batched tensor-core path (where the shape
 * supports it) instead of the per-token kernels, for the whole process and
 * every device; T < 1 restores the default (128). Returns the previous value.
 * A single token through a stack keeps its persistent kernel whatever the
 * value. Meant for measuring the two paths against each other (bench.py
 * --sweep); calls already enqueued are not affected. Not on the pages. */
MOE_API int32_t moe_set_batched_min_tokens(int32_t T);

/* Sets the token count from which those calls take the grouped GEMV path
 * (a few tokens per expert: each selected expert's weights read once for
 * all of its tokens, dot products on the CUDA cores, each token's x rounded
 * to 16-bit fixed point: within the same tolerance as the other paths, not
 * bit-identical to them) instead of the per-token kernels, below the batched
 * threshold; T < 1 restores the default (8). Returns the previous value.
 * Process-wide, as above. Not on the pages. */
MOE_API int32_t moe_set_gemv_min_tokens(int32_t T);

/* Sets the token count up to which moe_stack_forward runs its tokens one
 * at a time through the single-token persistent kernel (one launch per
 * token and 48 layers; each token's result as if it were called alone),
 * where the shape has that kernel; 1 keeps it to single tokens, T < 1
 * restores the default (7). Takes precedence over the two thresholds
 * above. Process-wide, as above. Not on the pages. */
MOE_API int32_t moe_set_decode_max_tokens(int32_t T);

/* The batched path's grouping step on its own: the T*k (token, slot) pairs
 * of topk_idx [T][k] grouped by expert, stable in (token, slot) order, with
 * the shared expert (if cfg->shared_inter > 0) as expert E taken by every
 * token. perm [T*k (+T)] receives pair ids (t*k + slot; T*k + t for shared
 * pairs); offsets [E+2] (or [E+1] without a shared expert) the first
 * position of each expert and, last, the pair count. */
MOE_API moe_status moe_sort_by_expert(const moe_config* cfg, const int32_t* topk_idx, int32_t T,
                              int32_t* perm, int32_t* offsets,
                              void* ws, size_t ws_bytes, moe_stream_t stream);

/* Bytes of the group-major copy of the scales and biases of n_experts down
 * matrices [H][K] (K = inter for the routed experts, shared_inter for the
 * shared one): n_experts * (K/group) * H * 4. 0 on a bad configuration or K
 * that is not a positive multiple of the group. */
MOE_API size_t moe_down_sb_size(const moe_config* cfg, int32_t n_experts, int32_t K);

/* Writes the group-major copy of `down`'s scales and biases into `out`
 * (caller-owned device memory of moe_down_sb_size bytes, 16-byte aligned):
 * out[((e*(K/group) + g)*H + r)*2 + 0] = scale of row r, group g of expert e,
 * and + 1 the bias. A pure re-layout (no arithmetic), meant to run once when
 * the weights are loaded; the result goes into moe_layer_weights.down_sb
 * (or .shared_down_sb with n_experts = 1 and K = shared_inter). Asynchronous
 * on `stream`. Not on the pages: a layout of this library's decode kernel. */
MOE_API moe_status moe_prepare_down_sb(const moe_config* cfg, const moe_qtensor* down, int32_t n_experts,
                                       int32_t K, uint16_t* out, moe_stream_t stream);

/* Bytes of the unit-major copy of the codes of n_experts down matrices
 * [H][K]: n_experts * K * H * bits / 8 (the size of the codes themselves).
 * 0 on a bad configuration or K that is not a positive multiple of 32 and
 * of the group. */
MOE_API size_t moe_down_units_size(const moe_config* cfg, int32_t n_experts, int32_t K);

/* Writes the unit-major copy of `down`'s codes into `out` (caller-owned
 * device memory of moe_down_units_size bytes, 16-byte aligned): the codes of
 * columns [32u, 32u+32) of row r of expert e go to
 * out + ((e*(K/32) + u)*H + r) * (32*bits/8). A pure re-layout, meant to run
 * once when the weights are loaded; the result goes into
 * moe_layer_weights.down_units (or .shared_down_units with n_experts = 1
 * and K = shared_inter). Asynchronous on `stream`. Not on the pages: a
 * layout of this library's decode kernel. */
MOE_API moe_status moe_prepare_down_units(const moe_config* cfg, const moe_qtensor* down, int32_t n_experts,
                                          int32_t K, uint8_t* out, moe_stream_t stream);

/* moe_layer_forward without a workspace, for callers that cannot allocate
 * device memory or pass a scratch buffer of their own: code inside a host
 * framework that owns all device memory and forbids allocation after
 * start-up, plugins that are handed only their inputs and outputs, and
 * latency-critical paths where an allocation (which may synchronise the
 * device) is not allowed. The pages have no counterpart of this call; it
 * exists for those callers only.
 * It runs the per-token kernels of moe_layer_forward (router + top-k,
 * gate/up + SwiGLU, down + combine) for every T; it never takes the batched
 * tensor-core path that moe_layer_forward uses from 8 tokens up. Its scratch
 * is a fixed 2 MiB array inside the library that every GPU that loads the
 * library holds until the process exits. The scratch a call needs is the
 * per-token part of the workspace layout (status word, routing counters,
 * logits, gate values, h, and the buffers of the single-token decode), which
 * grows with T; a call whose part exceeds 2 MiB returns MOE_ERR_WORKSPACE
 * before anything is enqueued. At H=2048, E=256, k=8, I=Is=512 that admits
 * T <= 46 tokens; at H=2048, E=512, k=10, I=Is=512, T <= 41. The call
 * allocates nothing. The first call on a device looks up the array's device
 * address (with that device current) and keeps it; make that first call
 * before any stream capture. The kept address is that of the device's
 * current context: after cudaDeviceReset (or any teardown of the primary
 * context) it is stale, so do not call this entry point again in that
 * process. Every call shares the one array: calls that overlap on the GPU
 * (other streams, other threads) race and must be serialised by the caller.
 * Each call clears the status word and counters it needs. Arguments as
 * moe_layer_forward; device_status (optional, device int32) receives the
 * call's device status (0 = MOE_OK, else a moe_status) when the stream gets
 * there. */
MOE_API moe_status moe_layer_forward_static(const moe_config* cfg, const moe_layer_weights* w,
                                            const uint16_t* x, int32_t T, uint16_t* y,
                                            int32_t* topk_idx, float* topk_w, int32_t* device_status,
                                            moe_stream_t stream);

/* Self-check of the bounded waits. Every wait inside the kernels of this
 * library (on an mbarrier, or on a word another CTA writes) gives up after
 * 2 s or 2^26 polls, records MOE_ERR_TIMEOUT in the workspace status and
 * returns, so that the context stays usable. This call runs both forms of
 * wait on events that never happen: it clears the workspace's 64-byte
 * header (status word included), then one CTA polls a header word that
 * nothing writes while a second warp waits on an mbarrier that nobody
 * arrives at. Asynchronous on `stream`; the kernel takes about 2 s. When it
 * has run, gave_up (device int32, caller-owned) holds bit 0 = the word poll
 * ended without its word, bit 1 = the mbarrier wait ended without its phase,
 * and moe_get_device_status returns MOE_ERR_TIMEOUT. Returns
 * MOE_ERR_WORKSPACE for a NULL, misaligned or smaller-than-64-byte ws,
 * MOE_ERR_INVALID_ARG for a NULL or misaligned gave_up. Not part of the
 * method; it exists to test the failure path without faulting the GPU. */
MOE_API moe_status moe_check_wait_limit(void* ws, size_t ws_bytes, int32_t* gave_up, moe_stream_t stream);

/* Waits for `stream`, then returns and clears the workspace's device status
 * (MOE_OK if no kernel reported an error since the last read). */
MOE_API moe_status moe_get_device_status(void* ws, moe_stream_t stream);

/* Static text for a status code. */
MOE_API const char* moe_status_string(moe_status s);

/* Text of the last error raised in this thread by a library call. */
MOE_API const char* moe_last_error_string(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
