// C ABI of the routed-MoE library (declared in include/moe_b200.h):
// argument validation, the workspace layout, and the stream-ordered launch
// sequence of each call. Nothing here allocates device memory.

#include <cstdarg>
#include <cstdio>
#include <algorithm>
#include <atomic>
#include <cstring>
#include <memory>
#include <mutex>
#include <string>

#include <cudaTypedefs.h>

#include "moe_b200.h"
#include "moe_common.cuh"
#include "moe_launch.h"

namespace {

thread_local std::string g_last_error;

moe_status fail(moe_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

moe_status cuda_fail(cudaError_t e, const char* where) {
  return fail(MOE_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

constexpr size_t kAlign = 256;
size_t up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

// Byte offsets of the workspace regions for T tokens.
struct Layout {
  size_t hdr, counters, logits, sgate, h, r, xa, xb, y, idx, w;
  size_t dlogits, dh, dy, dyacc, dcnt, dr, dx;            // persistent single-token decode
  size_t base_total;                                      // end of the regions above
  size_t perm, offs, chunks, nchunks, x16, hhi, hlo, o;   // batched paths (o: one plane per unit group for
                                                          // the grouped GEMV, the first for the GEMM)
  size_t xsx, xsh;                                        // group sums of x and of h
  size_t gxq, gxsc;                                       // grouped GEMV: fixed-point x, 2^-S per token
  size_t total;
};

constexpr int kBatchMinTokens = 128;  // from this many tokens the grouped tensor-core path runs (default)
std::atomic<int> g_batch_min{kBatchMinTokens};  // moe_set_batched_min_tokens
constexpr int kGemvMinTokens = 8;  // from this many tokens the grouped GEMV runs (default)
std::atomic<int> g_gemv_min{kGemvMinTokens};  // moe_set_gemv_min_tokens
// Up to this many tokens moe_stack_forward runs the single-token persistent kernel once per token
// (where the shape has one): below the GEMV threshold it beats the per-token kernels at every
// measured batch size (default)
constexpr int kDecodeMaxTokens = 7;
std::atomic<int> g_decode_max{kDecodeMaxTokens};  // moe_set_decode_max_tokens

bool decode_tokens(int T) { return T == 1 || (T >= 1 && T <= g_decode_max.load(std::memory_order_relaxed)); }

constexpr int kMaxGrid = 1024;  // largest persistent decode grid

// Partial-output rows (planes x pairs, each H floats) the grouped GEMV needs for any call of up to T
// tokens: the units per item grow with the batch, so a smaller batch can need more planes than a
// larger one. Up to the batch size where the units per item reach kGvUPI every size is a candidate;
// from there the plane count is fixed and the rows grow with T.
long gemv_partial_rows(int T, int k, int E, int I, int Is) {
  auto rows = [&](int t) {
    const long np = static_cast<long>(t) * k + (Is > 0 ? t : 0);
    return static_cast<long>(I / (32 * moe::gemv_units_per_item(t, k, E, I, Is))) * np;
  };
  long best = rows(T);
  for (int t = 1; t < T; ++t) {
    if (rows(t) > best) best = rows(t);
    if (moe::gemv_units_per_item(t, k, E, I, Is) == moe::kGvUPI) break;
  }
  return best;
}

Layout layout(const moe_config& c, int64_t T) {
  Layout L{};
  const int64_t imax = c.inter > c.shared_inter ? c.inter : c.shared_inter;
  const int64_t tiles = (T + moe::kRouteTokTile - 1) / moe::kRouteTokTile;
  size_t o = 0;
  L.hdr = o;      o += up(sizeof(moe::WsHeader));
  L.counters = o; o += up(static_cast<size_t>(tiles) * 4);
  L.logits = o;   o += up(static_cast<size_t>(T) * c.num_experts * 4);
  L.sgate = o;    o += up(static_cast<size_t>(T) * 4);
  L.h = o;        o += up(static_cast<size_t>(T) * (c.top_k + 1) * imax * 4);
  L.r = o;        o += up(static_cast<size_t>(T) * c.hidden * 4);
  L.xa = o;       o += up(static_cast<size_t>(T) * c.hidden * 2);
  L.xb = o;       o += up(static_cast<size_t>(T) * c.hidden * 2);
  L.y = o;        o += up(static_cast<size_t>(T) * c.hidden * 2);
  L.idx = o;      o += up(static_cast<size_t>(T) * c.top_k * 4);
  L.w = o;        o += up(static_cast<size_t>(T) * c.top_k * 4);
  // decode exchange words: logits, h, y, each in kDecodeReplicas copies, then the split
  // kernel's accumulators and counter (contiguous, zeroed before each launch)
  L.dlogits = o;  o += moe::kDecodeReplicas * up(static_cast<size_t>(c.num_experts + 1) * 4);
  L.dh = o;       o += moe::kDecodeReplicas * up(static_cast<size_t>(c.top_k + 1) * imax * 4);
  L.dy = o;       o += moe::kDecodeReplicas * up(static_cast<size_t>(c.hidden) * 4);
  // the split decode kernel's y accumulators (kDecodeYBufs x kDecodeReplicas) and arrival counter
  L.dyacc = o;    o += static_cast<size_t>(moe::kDecodeYBufs) * moe::kDecodeReplicas * up(static_cast<size_t>(c.hidden) * 4);
  L.dcnt = o;     o += up(4);
  L.dr = o;       o += up(static_cast<size_t>(c.hidden) * 4);
  L.dx = o;       o += up(static_cast<size_t>(c.hidden) * 2);
  L.base_total = o;
  const size_t np = static_cast<size_t>(T) * (c.top_k + 1);
  L.perm = o;     o += up(np * 4);
  L.offs = o;     o += up(static_cast<size_t>(c.num_experts + 2) * 4);
  L.chunks = o;   o += up((static_cast<size_t>(c.num_experts) + 2 + np / moe::kGvTPI + 1) * 12);
  L.nchunks = o;  o += up(4);
  L.x16 = o;      o += up(np * c.hidden * 2);
  L.hhi = o;      o += up(np * imax * 2);
  L.hlo = o;      o += up(np * imax * 2);
  // the partial outputs of the grouped GEMV for any call of up to T tokens (at least one plane: the
  // tensor-core path's outputs)
  const size_t orow = std::max<size_t>(
      np, gemv_partial_rows(static_cast<int>(T), c.top_k, c.num_experts, c.inter, c.shared_inter));
  L.o = o;        o += up(orow * c.hidden * 4);
  L.xsx = o;      o += up(np * (c.hidden / 64 + 1) * 4);
  L.xsh = o;      o += up(np * (imax / 64 + 1) * 4 * 4);
  {
    const size_t ps = 128 / c.bits, nsg = c.hidden / ps;
    const size_t qsp = c.bits == 4 ? moe::xq_stride<4>() : moe::xq_stride<8>();
    L.gxq = o;    o += up(static_cast<size_t>(T) * nsg * qsp * 4);
    L.gxsc = o;   o += up(static_cast<size_t>(T) * 4);
  }
  L.total = o;
  return L;
}

moe::WsView view(void* ws, const Layout& L) {
  char* b = static_cast<char*>(ws);
  moe::WsView v;
  v.hdr = reinterpret_cast<moe::WsHeader*>(b + L.hdr);
  v.counters = reinterpret_cast<uint32_t*>(b + L.counters);
  v.logits = reinterpret_cast<float*>(b + L.logits);
  v.sgate = reinterpret_cast<float*>(b + L.sgate);
  v.h = reinterpret_cast<float*>(b + L.h);
  return v;
}

moe_status check_cfg(const moe_config* c) {
  if (!c) return fail(MOE_ERR_INVALID_ARG, "cfg is NULL");
  if (c->bits != 4 && c->bits != 8) return fail(MOE_ERR_UNSUPPORTED, "bits=%d (need 4 or 8)", c->bits);
  if (c->group != 32 && c->group != 64) return fail(MOE_ERR_UNSUPPORTED, "group=%d (need 32 or 64)", c->group);
  if (c->hidden < 64 || c->hidden > 8192 || c->hidden % c->group)
    return fail(MOE_ERR_UNSUPPORTED, "hidden=%d (64..8192, multiple of group)", c->hidden);
  if (c->top_k < 1 || c->top_k > 16) return fail(MOE_ERR_UNSUPPORTED, "top_k=%d (1..16)", c->top_k);
  if (c->num_experts < c->top_k || c->num_experts > 512)
    return fail(MOE_ERR_UNSUPPORTED, "num_experts=%d (top_k..512)", c->num_experts);
  if (c->inter < c->group || c->inter > 2048 || c->inter % c->group)
    return fail(MOE_ERR_UNSUPPORTED, "inter=%d (group..2048, multiple of group)", c->inter);
  if (c->shared_inter != 0 &&
      (c->shared_inter < c->group || c->shared_inter > 2048 || c->shared_inter % c->group))
    return fail(MOE_ERR_UNSUPPORTED, "shared_inter=%d (0, or group..2048, multiple of group)", c->shared_inter);
  if (c->renorm != 0 && c->renorm != 1) return fail(MOE_ERR_UNSUPPORTED, "renorm=%d (0 or 1)", c->renorm);
  return MOE_OK;
}

moe_status check_ptr(const void* p, size_t a, const char* what) {
  if (!p) return fail(MOE_ERR_INVALID_ARG, "%s is NULL", what);
  if (!aligned(p, a)) return fail(MOE_ERR_INVALID_ARG, "%s is not %zu-byte aligned", what, a);
  return MOE_OK;
}

moe_status check_qt(const moe_qtensor& q, int64_t rows, int64_t K, int bits, int group, int64_t n,
                    const char* what) {
  char name[64];
  snprintf(name, sizeof(name), "%s.q", what);
  moe_status s = check_ptr(q.q, 16, name);
  if (s) return s;
  snprintf(name, sizeof(name), "%s.scales", what);
  if ((s = check_ptr(q.scales, 16, name))) return s;
  snprintf(name, sizeof(name), "%s.biases", what);
  if ((s = check_ptr(q.biases, 16, name))) return s;
  if (n > 1) {
    if (q.q_expert_stride < rows * K * bits / 8 || q.q_expert_stride % 16)
      return fail(MOE_ERR_INVALID_ARG, "%s.q_expert_stride=%lld (>= %lld, multiple of 16)", what,
                  static_cast<long long>(q.q_expert_stride), static_cast<long long>(rows * K * bits / 8));
    if (q.sb_expert_stride < rows * (K / group) || q.sb_expert_stride % 8)
      return fail(MOE_ERR_INVALID_ARG, "%s.sb_expert_stride=%lld (>= %lld, multiple of 8)", what,
                  static_cast<long long>(q.sb_expert_stride), static_cast<long long>(rows * (K / group)));
  }
  return MOE_OK;
}

// The stock (unpacked) gate/up layout: separate gate and up tensors (moe_layer_weights.up).
bool stock_layout(const moe_layer_weights& w) { return w.up.q != nullptr; }

// The up tensor of the stock layout against its gate tensor: the same expert strides.
moe_status check_up(const moe_qtensor& g, const moe_qtensor& u, int64_t n, const char* what) {
  if (n > 1 && (u.q_expert_stride != g.q_expert_stride || u.sb_expert_stride != g.sb_expert_stride))
    return fail(MOE_ERR_INVALID_ARG, "%s: expert strides differ from the gate tensor's", what);
  return MOE_OK;
}

moe_status check_weights(const moe_config& c, const moe_layer_weights* w, bool need_router) {
  if (!w) return fail(MOE_ERR_INVALID_ARG, "weights is NULL");
  moe_status s;
  if (need_router && (s = check_ptr(w->router_w, 16, "router_w"))) return s;
  if (w->router_bias && !aligned(w->router_bias, 4)) return fail(MOE_ERR_INVALID_ARG, "router_bias misaligned");
  const bool stock = stock_layout(*w);
  const int64_t gu_rows = stock ? 1 : 2;  // gate_up rows per intermediate index
  if ((s = check_qt(w->gate_up, gu_rows * c.inter, c.hidden, c.bits, c.group, c.num_experts, "gate_up"))) return s;
  if (stock && ((s = check_qt(w->up, c.inter, c.hidden, c.bits, c.group, c.num_experts, "up")) ||
                (s = check_up(w->gate_up, w->up, c.num_experts, "up"))))
    return s;
  if ((s = check_qt(w->down, c.hidden, c.inter, c.bits, c.group, c.num_experts, "down"))) return s;
  if (c.shared_inter > 0) {
    if ((s = check_qt(w->shared_gate_up, gu_rows * c.shared_inter, c.hidden, c.bits, c.group, 1, "shared_gate_up")))
      return s;
    if (stock != (w->shared_up.q != nullptr))
      return fail(MOE_ERR_INVALID_ARG, "shared_up.q must be set exactly when up.q is");
    if (stock && ((s = check_qt(w->shared_up, c.shared_inter, c.hidden, c.bits, c.group, 1, "shared_up")) ||
                  (s = check_up(w->shared_gate_up, w->shared_up, 1, "shared_up"))))
      return s;
    if ((s = check_qt(w->shared_down, c.hidden, c.shared_inter, c.bits, c.group, 1, "shared_down"))) return s;
    if ((s = check_ptr(w->shared_gate_w, 16, "shared_gate_w"))) return s;
    if (w->shared_down_sb && !aligned(w->shared_down_sb, 16))
      return fail(MOE_ERR_INVALID_ARG, "shared_down_sb is not 16-byte aligned");
    if (w->shared_down_units && !aligned(w->shared_down_units, 16))
      return fail(MOE_ERR_INVALID_ARG, "shared_down_units is not 16-byte aligned");
  }
  if (w->down_sb && !aligned(w->down_sb, 16)) return fail(MOE_ERR_INVALID_ARG, "down_sb is not 16-byte aligned");
  if (w->down_units && !aligned(w->down_units, 16))
    return fail(MOE_ERR_INVALID_ARG, "down_units is not 16-byte aligned");
  return MOE_OK;
}

moe_status check_ws(const moe_config& c, void* ws, size_t ws_bytes, int64_t T, Layout* L) {
  if (!ws) return fail(MOE_ERR_WORKSPACE, "workspace is NULL");
  if (!aligned(ws, kAlign)) return fail(MOE_ERR_WORKSPACE, "workspace is not %zu-byte aligned", kAlign);
  *L = layout(c, T);
  if (ws_bytes < L->total)
    return fail(MOE_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, L->total);
  return MOE_OK;
}

moe::QMat qmat(const moe_qtensor& q) {
  return moe::QMat{q.q, q.scales, q.biases, q.q_expert_stride, q.sb_expert_stride, 0, 0, 0};
}

// A gate/up matrix set with the offsets of its up rows: I rows on in the packed layout, the up
// tensor in the stock layout.
moe::QMat qmat_gu(const moe_config& c, const moe_qtensor& gu, const moe_qtensor& up, bool stock, int I) {
  moe::QMat m = qmat(gu);
  if (stock) {
    m.up_q = static_cast<int64_t>(reinterpret_cast<uintptr_t>(up.q) - reinterpret_cast<uintptr_t>(gu.q));
    m.up_s = static_cast<int64_t>(reinterpret_cast<uintptr_t>(up.scales) - reinterpret_cast<uintptr_t>(gu.scales)) / 2;
    m.up_b = static_cast<int64_t>(reinterpret_cast<uintptr_t>(up.biases) - reinterpret_cast<uintptr_t>(gu.biases)) / 2;
  } else {
    m.up_q = static_cast<int64_t>(I) * c.hidden * c.bits / 8;
    m.up_s = m.up_b = static_cast<int64_t>(I) * (c.hidden / c.group);
  }
  return m;
}

moe_status route(const moe_config& c, const uint16_t* x, int T, const uint16_t* wr, const float* rbias,
                 int32_t* idx, float* w, const moe::WsView& v, cudaStream_t st) {
  moe::RouteParams p{x, wr, rbias, T, c.hidden, c.num_experts, c.top_k, c.renorm, idx, w, v};
  cudaError_t e = moe::launch_route_topk(p, st);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "route_topk launch");
}

moe_status ffn(const moe_config& c, const moe_layer_weights& wt, const uint16_t* x, int T, const int32_t* idx,
               const float* w, uint16_t* y, const moe::WsView& v, cudaStream_t st) {
  moe::FfnParams p{};
  p.x = x;
  p.idx = idx;
  p.w = w;
  p.y = y;
  const bool stock = stock_layout(wt);
  p.gate_up = qmat_gu(c, wt.gate_up, wt.up, stock, c.inter);
  p.down = qmat(wt.down);
  if (c.shared_inter > 0) {
    p.sh_gate_up = qmat_gu(c, wt.shared_gate_up, wt.shared_up, stock, c.shared_inter);
    p.sh_down = qmat(wt.shared_down);
    p.wsg = wt.shared_gate_w;
  }
  p.T = T;
  p.H = c.hidden;
  p.E = c.num_experts;
  p.k = c.top_k;
  p.I = c.inter;
  p.Is = c.shared_inter;
  p.group = c.group;
  p.Imax = c.inter > c.shared_inter ? c.inter : c.shared_inter;
  p.ws = v;
  cudaError_t e = moe::launch_expert_ffn(p, c.bits, st);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "expert_ffn launch");
}

// ---------------------------------------------------------------- batched tensor-core path

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  std::call_once(g_encode_once, []() {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

// 3D map over E matrices [rows][inner] (inner contiguous, `esize` bytes per element),
// box = (box_inner, box_rows, 1 expert).
bool map_3d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, int64_t inner, int64_t rows,
            int64_t E, int64_t expert_stride_bytes, int box_inner, int box_rows = 64) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(E)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(inner * esize), static_cast<cuuint64_t>(expert_stride_bytes)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_rows), 1u};
  cuuint32_t es[3] = {1u, 1u, 1u};
  return encode_fn()(m, dt, 3, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2D fp16 map over [rows][K] with a (64 x box_rows) box in the 128-byte swizzle.
bool map_b(CUtensorMap* m, const void* base, int64_t K, int64_t rows, int box_rows) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K * 2)};
  cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t es[2] = {1u, 1u};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int device_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  return n;
}

bool batched_eligible(const moe_config& c, int T) {
  if (T < g_batch_min.load(std::memory_order_relaxed)) return false;
  if (c.group != 64) return false;  // one quantisation group per GEMM k-block
  if (c.shared_inter != 0 && c.shared_inter != c.inter) return false;
  if ((c.hidden / c.group) % 8 || (c.inter / c.group) % 8 || c.hidden % 256 || c.inter % 64) return false;
  if (!encode_fn()) return false;
  int dev = 0, optin = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return false;
  const size_t need = std::max(moe::grouped_gemm_smem(0, c.bits, c.hidden, c.group),
                               moe::grouped_gemm_smem(1, c.bits, c.inter, c.group));
  return need <= static_cast<size_t>(optin);
}

// Experts' gate/up and down for T tokens given their selection, on the tensor cores.
moe_status batched_ffn(const moe_config& c, const moe_layer_weights& wt, const uint16_t* x, int T, const int32_t* idx,
                       const float* w, uint16_t* y, void* ws, const Layout& Ly, cudaStream_t st) {
  if (stock_layout(wt)) return fail(MOE_ERR_UNSUPPORTED, "the tensor-core path reads the packed gate/up layout");
  char* b = static_cast<char*>(ws);
  const moe::WsView v = view(ws, Ly);
  const int H = c.hidden, I = c.inter, k = c.top_k, E = c.num_experts;
  const bool shared = c.shared_inter > 0;
  const int np = T * k + (shared ? T : 0);
  int32_t* perm = reinterpret_cast<int32_t*>(b + Ly.perm);
  int32_t* offs = reinterpret_cast<int32_t*>(b + Ly.offs);
  int32_t* chunks = reinterpret_cast<int32_t*>(b + Ly.chunks);
  int32_t* nchunks = reinterpret_cast<int32_t*>(b + Ly.nchunks);
  uint16_t* x16 = reinterpret_cast<uint16_t*>(b + Ly.x16);
  uint16_t* hhi = reinterpret_cast<uint16_t*>(b + Ly.hhi);
  uint16_t* hlo = reinterpret_cast<uint16_t*>(b + Ly.hlo);
  float* o = reinterpret_cast<float*>(b + Ly.o);
  float* xsx = reinterpret_cast<float*>(b + Ly.xsx);
  float* xsh = reinterpret_cast<float*>(b + Ly.xsh);
  const int sms = device_sms();
  if (sms < 1) return fail(MOE_ERR_CUDA, "no device");

  moe::SortParams sp{idx, T, k, E, shared ? 1 : 0, perm, offs, chunks, nchunks, moe::kChunkTokens, v.hdr};
  cudaError_t e = moe::launch_sort_by_expert(sp, st);
  if (e != cudaSuccess) return cuda_fail(e, "sort launch");
  moe::BatchParams bp{};
  bp.x = x;
  bp.wsg = wt.shared_gate_w;
  bp.perm = perm;
  bp.T = T;
  bp.k = k;
  bp.H = H;
  bp.Is = c.shared_inter;
  bp.perm8 = (c.bits == 4) ? 1 : 0;
  bp.x16 = x16;
  bp.xs = xsx;
  bp.sgate = v.sgate;
  bp.w = w;
  bp.o = o;
  bp.y = y;
  if ((e = moe::launch_gather(bp, sms * 4, st)) != cudaSuccess) return cuda_fail(e, "gather launch");

  auto gp = std::make_unique<moe::GemmParams>();
  const int bits = c.bits, g = c.group;
  const moe_qtensor& sgu = shared ? wt.shared_gate_up : wt.gate_up;
  const moe_qtensor& sdn = shared ? wt.shared_down : wt.down;
  // gate/up: K = H, rows = 2I
  bool ok = map_3d(&gp->tm_codes[0], wt.gate_up.q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, H * bits / 8, 2 * I, E,
                   wt.gate_up.q_expert_stride, 128 * bits / 8) &&
            map_3d(&gp->tm_codes[1], sgu.q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, H * bits / 8, 2 * I, 1,
                   static_cast<int64_t>(2) * I * H * bits / 8, 128 * bits / 8) &&
            map_3d(&gp->tm_scales[0], wt.gate_up.scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, H / g, 2 * I, E,
                   wt.gate_up.sb_expert_stride * 2, H / g) &&
            map_3d(&gp->tm_scales[1], sgu.scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, H / g, 2 * I, 1,
                   static_cast<int64_t>(2) * I * (H / g) * 2, H / g) &&
            map_3d(&gp->tm_biases[0], wt.gate_up.biases, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, H / g, 2 * I, E,
                   wt.gate_up.sb_expert_stride * 2, H / g) &&
            map_3d(&gp->tm_biases[1], sgu.biases, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, H / g, 2 * I, 1,
                   static_cast<int64_t>(2) * I * (H / g) * 2, H / g);
  for (int i = 0; i < 4 && ok; ++i) ok = map_b(&gp->tm_b[i], x16, H, np, i < 3 ? 16 << i : 64) && map_b(&gp->tm_b2[i], x16, H, np, i < 3 ? 16 << i : 64);
  if (!ok) return fail(MOE_ERR_CUDA, "tensor map encoding failed (gate/up)");
  gp->chunks = chunks;
  gp->nchunks = nchunks;
  gp->perm = perm;
  gp->xs_in = xsx;
  gp->hsum_out = xsh;
  gp->K = H;
  gp->rows = 2 * I;
  gp->I = I;
  gp->H = H;
  gp->E = E;
  gp->group = g;
  gp->ldh = I;
  gp->h_hi = hhi;
  gp->h_lo = hlo;
  gp->out = o;
  gp->hdr = v.hdr;
  if ((e = moe::launch_grouped_gemm(*gp, 0, bits, sms, st)) != cudaSuccess) return cuda_fail(e, "gate/up GEMM launch");
  // down: K = I, rows = H
  ok = map_3d(&gp->tm_codes[0], wt.down.q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, I * bits / 8, H, E,
              wt.down.q_expert_stride, 128 * bits / 8) &&
       map_3d(&gp->tm_codes[1], sdn.q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, I * bits / 8, H, 1,
              static_cast<int64_t>(H) * I * bits / 8, 128 * bits / 8) &&
       map_3d(&gp->tm_scales[0], wt.down.scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, I / g, H, E,
              wt.down.sb_expert_stride * 2, I / g) &&
       map_3d(&gp->tm_scales[1], sdn.scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, I / g, H, 1,
              static_cast<int64_t>(H) * (I / g) * 2, I / g) &&
       map_3d(&gp->tm_biases[0], wt.down.biases, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, I / g, H, E,
              wt.down.sb_expert_stride * 2, I / g) &&
       map_3d(&gp->tm_biases[1], sdn.biases, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, I / g, H, 1,
              static_cast<int64_t>(H) * (I / g) * 2, I / g);
  for (int i = 0; i < 4 && ok; ++i) ok = map_b(&gp->tm_b[i], hhi, I, np, i < 3 ? 16 << i : 64) && map_b(&gp->tm_b2[i], hlo, I, np, i < 3 ? 16 << i : 64);
  if (!ok) return fail(MOE_ERR_CUDA, "tensor map encoding failed (down)");
  gp->K = I;
  gp->rows = H;
  gp->xs_in = xsh;
  if ((e = moe::launch_grouped_gemm(*gp, 1, bits, sms, st)) != cudaSuccess) return cuda_fail(e, "down GEMM launch");
  if ((e = moe::launch_combine(bp, sms * 4, st)) != cudaSuccess) return cuda_fail(e, "combine launch");
  return MOE_OK;
}

// ---------------------------------------------------------------- grouped GEMV path

int device_smem_optin() {
  int dev = 0, optin = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return 0;
  return optin;
}

// Whether T tokens take the grouped GEMV (a few tokens per expert, CUDA cores): from
// moe_set_gemv_min_tokens tokens up, below the batched tensor-core path's threshold (or where that
// path does not apply), for shapes whose units of 32 columns come in whole groups of kGvUPI.
// stock: the layer is in the stock gate/up layout, which the tensor-core path does not read; the
// grouped GEMV then also takes the token counts the tensor cores would.
bool gemv_eligible(const moe_config& c, int T, bool stock = false) {
  if (T < g_gemv_min.load(std::memory_order_relaxed)) return false;
  if (!stock && batched_eligible(c, T)) return false;
  if (!encode_fn()) return false;
  const int optin = device_smem_optin();
  if (optin < 1024) return false;
  return moe::grouped_gemv_supported(c.hidden, c.inter, c.shared_inter, c.group, c.bits,
                                     static_cast<size_t>(optin) - 1024);
}

// Experts' gate/up and down for T tokens given their selection, as grouped matrix-vector products.
moe_status gemv_ffn(const moe_config& c, const moe_layer_weights& wt, const uint16_t* x, int T, const int32_t* idx,
                    const float* w, uint16_t* y, void* ws, const Layout& Ly, cudaStream_t st) {
  char* b = static_cast<char*>(ws);
  const moe::WsView v = view(ws, Ly);
  const int H = c.hidden, I = c.inter, k = c.top_k, E = c.num_experts;
  const bool shared = c.shared_inter > 0;
  const int np = T * k + (shared ? T : 0);
  int32_t* perm = reinterpret_cast<int32_t*>(b + Ly.perm);
  int32_t* chunks = reinterpret_cast<int32_t*>(b + Ly.chunks);
  int32_t* nchunks = reinterpret_cast<int32_t*>(b + Ly.nchunks);
  uint32_t* xq = reinterpret_cast<uint32_t*>(b + Ly.gxq);
  float* xsc = reinterpret_cast<float*>(b + Ly.gxsc);
  float* o = reinterpret_cast<float*>(b + Ly.o);
  const int sms = device_sms();
  if (sms < 1) return fail(MOE_ERR_CUDA, "no device");
  moe::SortParams sp{idx, T, k, E, shared ? 1 : 0, perm, reinterpret_cast<int32_t*>(b + Ly.offs), chunks, nchunks,
                     moe::kGvTPI, v.hdr};
  cudaError_t e = moe::launch_sort_by_expert(sp, st);
  if (e != cudaSuccess) return cuda_fail(e, "sort launch");
  if ((e = moe::launch_xquant(x, wt.shared_gate_w, T, H, c.shared_inter, c.bits, xq, xsc, v.sgate, st)) != cudaSuccess)
    return cuda_fail(e, "xquant launch");
  auto gp = std::make_unique<moe::GemvParams>();
  gp->chunks = chunks;
  gp->nchunks = nchunks;
  gp->perm = perm;
  gp->xq = xq;
  gp->xsc = xsc;
  const bool stock = stock_layout(wt);
  gp->gu = qmat_gu(c, wt.gate_up, wt.up, stock, I);
  gp->dn = qmat(wt.down);
  gp->sgu = shared ? qmat_gu(c, wt.shared_gate_up, wt.shared_up, stock, c.shared_inter) : gp->gu;
  gp->sdn = qmat(shared ? wt.shared_down : wt.down);
  gp->dcu = wt.down_units;
  gp->dsb = wt.down_sb;
  gp->sdcu = shared ? wt.shared_down_units : nullptr;
  gp->sdsb = shared ? wt.shared_down_sb : nullptr;
  const int64_t rb = static_cast<int64_t>(I) * c.bits / 8;
  const int ub = 32 * c.bits / 8;
  if (!wt.down_units &&
      !map_3d(&gp->tm_dn, wt.down.q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, rb, H, E, wt.down.q_expert_stride, ub, 256))
    return fail(MOE_ERR_CUDA, "tensor map of the down codes");
  if (shared && !wt.shared_down_units &&
      !map_3d(&gp->tm_sdn, wt.shared_down.q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, rb, H, 1, rb * H, ub, 256))
    return fail(MOE_ERR_CUDA, "tensor map of the shared down codes");
  gp->o = o;
  gp->T = T;
  gp->k = k;
  gp->H = H;
  gp->E = E;
  gp->I = I;
  gp->group = c.group;
  gp->npairs = np;
  gp->upi = moe::gemv_units_per_item(T, k, E, I, c.shared_inter);
  gp->hdr = v.hdr;
  if ((e = moe::launch_grouped_gemv(*gp, c.bits, sms, st)) != cudaSuccess) return cuda_fail(e, "grouped GEMV launch");
  const int nq = I / (32 * gp->upi);
  if ((e = moe::launch_gv_combine(o, w, v.sgate, T, k, H, c.shared_inter, nq, np, y, sms * 4, st)) != cudaSuccess)
    return cuda_fail(e, "combine launch");
  return MOE_OK;
}

// Device facts the persistent decode needs, looked up once per device.
struct DevInfo {
  bool ok = false;
  int sms = 0, coop = 0, smem_optin = 0;
};

std::mutex g_dev_mu;
DevInfo g_dev[128];

bool dev_info(DevInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return false;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DevInfo& d = g_dev[dev];
  if (!d.ok) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
      return false;
    d.ok = true;
  }
  *out = d;
  return true;
}

// Whether one token through a stack runs as a persistent kernel (one launch
// per up to kMaxDecodeLayers layers) rather than four kernels per layer, and
// which: the split kernel where it fits, else the exchange kernel.
bool decode_eligible(const moe_config& c, int L, int* grid, bool* split = nullptr, int* split_late = nullptr,
                     int* split_two = nullptr) {
  DevInfo d;
  if (!dev_info(&d) || !d.coop || d.sms < 1 || d.sms > kMaxGrid || d.smem_optin < 1024) return false;
  const size_t limit = static_cast<size_t>(d.smem_optin) - 1024;
  size_t ss = 0;
  int late = 0, two = 0;
  const bool sp = encode_fn() && moe::decode_split_plan(c.hidden, c.num_experts, c.top_k, c.inter, c.shared_inter,
                                                        c.group, c.bits, d.sms, L, limit, &ss, &late, &two);
  if (!sp) {
    if (!moe::decode_stack_supported(c.hidden, c.num_experts, c.top_k, c.inter, c.shared_inter, c.group, c.bits))
      return false;
    const size_t smem =
        moe::decode_stack_smem(c.hidden, c.num_experts, c.top_k, c.inter, c.shared_inter, c.group, c.bits, d.sms);
    if (smem > limit) return false;
  }
  *grid = d.sms;
  if (split) *split = sp;
  if (split_late) *split_late = late;
  if (split_two) *split_two = two;
  return true;
}

moe::LayerDesc layer_desc(const moe_config& c, const moe_layer_weights& w) {
  moe::LayerDesc d{};
  d.wr = w.router_w;
  d.rbias = w.router_bias;
  d.wsg = w.shared_gate_w;
  const bool stock = stock_layout(w);
  d.gu = qmat_gu(c, w.gate_up, w.up, stock, c.inter);
  d.dn = qmat(w.down);
  d.sgu = qmat_gu(c, w.shared_gate_up, w.shared_up, stock, c.shared_inter);
  d.sdn = qmat(w.shared_down);
  d.dsb = w.down_sb;
  d.sdsb = w.shared_down_sb;
  d.dcu = w.down_units;
  d.sdcu = w.shared_down_units;
  return d;
}

// One token at a time through the stack on the persistent kernel: T launches (per 48 layers), token t
// from row t of x0 into row t of x_out, its trace in row t of each layer's [T] rows.
moe_status stack_decode(const moe_config& c, const moe_layer_weights* layers, int L, int T, const uint16_t* x0,
                        uint16_t* x_out, const moe_trace* trace, void* ws, const Layout& Ly, int grid, bool split,
                        int split_late, int split_two, cudaStream_t st) {
  char* b = static_cast<char*>(ws);
  auto P = std::make_unique<moe::DecodeParams>();
  P->H = c.hidden;
  P->E = c.num_experts;
  P->k = c.top_k;
  P->I = c.inter;
  P->Is = c.shared_inter;
  P->group = c.group;
  P->renorm = c.renorm;
  P->eps = 1e-6f;
  P->tr_rows = T;
  P->logits = reinterpret_cast<uint32_t*>(b + Ly.dlogits);
  P->hbuf = reinterpret_cast<uint32_t*>(b + Ly.dh);
  P->ybuf = reinterpret_cast<uint32_t*>(b + Ly.dy);
  P->logits_rep = static_cast<int>((Ly.dh - Ly.dlogits) / moe::kDecodeReplicas / 4);
  P->h_rep = static_cast<int>((Ly.dy - Ly.dh) / moe::kDecodeReplicas / 4);
  P->y_rep = static_cast<int>((Ly.dyacc - Ly.dy) / moe::kDecodeReplicas / 4);
  P->yacc = reinterpret_cast<float*>(b + Ly.dyacc);
  P->yrep = static_cast<int>(up(static_cast<size_t>(c.hidden) * 4) / 4);
  P->ybuf_stride = static_cast<int64_t>(moe::kDecodeReplicas) * P->yrep;
  P->arrive = reinterpret_cast<uint32_t*>(b + Ly.dcnt);
  P->split_late = split_late;
  P->split_two = split_two;
  P->hdr = reinterpret_cast<moe::WsHeader*>(b + Ly.hdr);
  uint16_t* xmid = reinterpret_cast<uint16_t*>(b + Ly.dx);
  float* rmid = reinterpret_cast<float*>(b + Ly.dr);
  const size_t H = static_cast<size_t>(c.hidden), k = static_cast<size_t>(c.top_k);
  const bool one_launch = L <= moe::kMaxDecodeLayers;  // the layer descriptors are built once
  for (int t = 0; t < T; ++t)
  for (int l0 = 0; l0 < L; l0 += moe::kMaxDecodeLayers) {
    const int n = (L - l0 < moe::kMaxDecodeLayers) ? L - l0 : moe::kMaxDecodeLayers;
    const bool last = (l0 + n == L);
    P->L = n;
    P->l0 = l0;
    P->x0 = (l0 == 0) ? x0 + t * H : xmid;
    P->r_in = (l0 == 0) ? nullptr : rmid;
    P->out = last ? x_out + t * H : xmid;
    P->r_out = last ? nullptr : rmid;
    P->tr_x = (trace && trace->x) ? trace->x + t * H : nullptr;
    P->tr_idx = (trace && trace->idx) ? trace->idx + t * k : nullptr;
    P->tr_w = (trace && trace->w) ? trace->w + t * k : nullptr;
    P->tr_y = (trace && trace->y) ? trace->y + t * H : nullptr;
    P->tr_t = (trace && t == 0) ? trace->t : nullptr;  // phase timestamps: the first token's
    if (t == 0 || !one_launch) {  // else the previous token's launch had the same layers
    for (int i = 0; i < n; ++i) P->layers[i] = layer_desc(c, layers[l0 + i]);
    if (split) {
      // down codes as (row bytes, H rows, experts), one unit's 32 columns x 256 rows per copy
      const int64_t rb = static_cast<int64_t>(c.inter) * c.bits / 8;
      const int ub = 32 * c.bits / 8;
      for (int i = 0; i < n; ++i) {
        const moe_layer_weights& w = layers[l0 + i];
        if (!map_3d(&P->tm_dn[i], w.down.q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, rb, c.hidden, c.num_experts,
                    w.down.q_expert_stride, ub, 256))
          return fail(MOE_ERR_CUDA, "tensor map of layer %d's down codes", l0 + i);
        if (c.shared_inter > 0 &&
            !map_3d(&P->tm_sdn[i], w.shared_down.q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, rb, c.hidden, 1,
                    rb * c.hidden, ub, 256))
          return fail(MOE_ERR_CUDA, "tensor map of layer %d's shared down codes", l0 + i);
      }
    }
    }
    cudaError_t e = cudaMemsetAsync(b + Ly.dlogits, 0, Ly.dr - Ly.dlogits, st);
    if (e != cudaSuccess) return cuda_fail(e, "exchange word reset");
    e = split ? moe::launch_decode_split(*P, c.bits, grid, st) : moe::launch_decode_stack(*P, c.bits, grid, st);
    if (e != cudaSuccess) return cuda_fail(e, "decode_stack launch");
  }
  return MOE_OK;
}

}  // namespace

extern "C" {

int32_t moe_stack_kernel_launches(const moe_config* cfg, int32_t T, int32_t L) {
  if (check_cfg(cfg) != MOE_OK || T < 0 || L < 0) return -1;
  if (T == 0 || L == 0) return 0;
  int grid = 0;
  if (decode_tokens(T) && decode_eligible(*cfg, L, &grid))
    return T * ((L + moe::kMaxDecodeLayers - 1) / moe::kMaxDecodeLayers);
  if (batched_eligible(*cfg, T)) return 1 + 7 * L;  // route, sort, gather, 2 GEMMs, combine, glue
  if (gemv_eligible(*cfg, T)) return 1 + 6 * L;     // route, sort, xquant, GEMV, combine, glue
  return 1 + 4 * L;
}

const char* moe_stack_path_name(const moe_config* cfg, int32_t T, int32_t L) {
  if (check_cfg(cfg) != MOE_OK || T < 0 || L < 0) return nullptr;
  if (T == 0 || L == 0) return "none";
  int grid = 0;
  bool split = false;
  if (decode_tokens(T) && decode_eligible(*cfg, L, &grid, &split))
    return split ? "decode_split_kernel" : "decode_stack_kernel";
  if (batched_eligible(*cfg, T)) return "batched";
  if (gemv_eligible(*cfg, T)) return "grouped_gemv";
  return "per_layer";
}

size_t moe_workspace_size(const moe_config* cfg, int32_t T, int32_t L) {
  (void)L;
  if (check_cfg(cfg) != MOE_OK || T < 0) return 0;
  return layout(*cfg, T < 1 ? 1 : T).total;
}

moe_status moe_workspace_init(void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (!ws || !aligned(ws, kAlign)) return fail(MOE_ERR_WORKSPACE, "workspace NULL or misaligned");
  if (ws_bytes < 2 * kAlign) return fail(MOE_ERR_WORKSPACE, "workspace too small");
  cudaError_t e = cudaMemsetAsync(ws, 0, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "workspace memset");
}

moe_status moe_route_topk(const moe_config* cfg, const uint16_t* x, int32_t T, const uint16_t* router_w,
                          const float* router_bias, int32_t* topk_idx, float* topk_w, void* ws,
                          size_t ws_bytes, moe_stream_t stream) {
  moe_status s;
  if ((s = check_cfg(cfg))) return s;
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T=%d", T);
  if (T == 0) return MOE_OK;
  if ((s = check_ptr(x, 16, "x")) || (s = check_ptr(router_w, 16, "router_w")) ||
      (s = check_ptr(topk_idx, 4, "topk_idx")) || (s = check_ptr(topk_w, 4, "topk_w")))
    return s;
  if (router_bias && !aligned(router_bias, 4)) return fail(MOE_ERR_INVALID_ARG, "router_bias misaligned");
  Layout L;
  if ((s = check_ws(*cfg, ws, ws_bytes, T, &L))) return s;
  return route(*cfg, x, T, router_w, router_bias, topk_idx, topk_w, view(ws, L),
               reinterpret_cast<cudaStream_t>(stream));
}

moe_status moe_expert_ffn(const moe_config* cfg, const moe_layer_weights* w, const uint16_t* x, int32_t T,
                          const int32_t* topk_idx, const float* topk_w, uint16_t* y, void* ws, size_t ws_bytes,
                          moe_stream_t stream) {
  moe_status s;
  if ((s = check_cfg(cfg))) return s;
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T=%d", T);
  if (T == 0) return MOE_OK;
  if ((s = check_weights(*cfg, w, false))) return s;
  if ((s = check_ptr(x, 16, "x")) || (s = check_ptr(y, 16, "y")) || (s = check_ptr(topk_idx, 4, "topk_idx")) ||
      (s = check_ptr(topk_w, 4, "topk_w")))
    return s;
  Layout L;
  if ((s = check_ws(*cfg, ws, ws_bytes, T, &L))) return s;
  const bool stock = stock_layout(*w);
  if (!stock && batched_eligible(*cfg, T))
    return batched_ffn(*cfg, *w, x, T, topk_idx, topk_w, y, ws, L, reinterpret_cast<cudaStream_t>(stream));
  if (gemv_eligible(*cfg, T, stock))
    return gemv_ffn(*cfg, *w, x, T, topk_idx, topk_w, y, ws, L, reinterpret_cast<cudaStream_t>(stream));
  return ffn(*cfg, *w, x, T, topk_idx, topk_w, y, view(ws, L), reinterpret_cast<cudaStream_t>(stream));
}

moe_status moe_layer_forward(const moe_config* cfg, const moe_layer_weights* w, const uint16_t* x, int32_t T,
                             uint16_t* y, int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes,
                             moe_stream_t stream) {
  moe_status s;
  if ((s = check_cfg(cfg))) return s;
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T=%d", T);
  if (T == 0) return MOE_OK;
  if ((s = check_weights(*cfg, w, true))) return s;
  if ((s = check_ptr(x, 16, "x")) || (s = check_ptr(y, 16, "y"))) return s;
  if ((topk_idx && !aligned(topk_idx, 4)) || (topk_w && !aligned(topk_w, 4)))
    return fail(MOE_ERR_INVALID_ARG, "topk_idx/topk_w misaligned");
  Layout L;
  if ((s = check_ws(*cfg, ws, ws_bytes, T, &L))) return s;
  char* b = static_cast<char*>(ws);
  int32_t* idx = topk_idx ? topk_idx : reinterpret_cast<int32_t*>(b + L.idx);
  float* wt = topk_w ? topk_w : reinterpret_cast<float*>(b + L.w);
  const moe::WsView v = view(ws, L);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if ((s = route(*cfg, x, T, w->router_w, w->router_bias, idx, wt, v, st))) return s;
  const bool stock = stock_layout(*w);
  if (!stock && batched_eligible(*cfg, T)) return batched_ffn(*cfg, *w, x, T, idx, wt, y, ws, L, st);
  if (gemv_eligible(*cfg, T, stock)) return gemv_ffn(*cfg, *w, x, T, idx, wt, y, ws, L, st);
  return ffn(*cfg, *w, x, T, idx, wt, y, v, st);
}

moe_status moe_stack_forward(const moe_config* cfg, const moe_layer_weights* layers, int32_t L, const uint16_t* x0,
                             int32_t T, uint16_t* x_out, const moe_trace* trace, void* ws, size_t ws_bytes,
                             moe_stream_t stream) {
  moe_status s;
  if ((s = check_cfg(cfg))) return s;
  if (T < 0 || L < 0) return fail(MOE_ERR_INVALID_ARG, "T=%d L=%d", T, L);
  if (T == 0 || L == 0) return MOE_OK;
  if (!layers) return fail(MOE_ERR_INVALID_ARG, "layers is NULL");
  for (int l = 0; l < L; ++l)
    if ((s = check_weights(*cfg, &layers[l], true))) return fail(s, "layer %d: %s", l, g_last_error.c_str());
  if ((s = check_ptr(x0, 16, "x0")) || (s = check_ptr(x_out, 16, "x_out"))) return s;
  if (trace && ((trace->x && !aligned(trace->x, 16)) || (trace->y && !aligned(trace->y, 16)) ||
                (trace->idx && !aligned(trace->idx, 4)) || (trace->w && !aligned(trace->w, 4))))
    return fail(MOE_ERR_INVALID_ARG, "trace buffers misaligned");
  Layout Ly;
  if ((s = check_ws(*cfg, ws, ws_bytes, T, &Ly))) return s;
  char* b = static_cast<char*>(ws);
  const moe::WsView v = view(ws, Ly);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int grid = 0;
  bool split = false;
  int split_late = 0, split_two = 0;
  if (decode_tokens(T) && decode_eligible(*cfg, L, &grid, &split, &split_late, &split_two))
    return stack_decode(*cfg, layers, L, T, x0, x_out, trace, ws, Ly, grid, split, split_late, split_two, st);
  bool stock = false;  // any layer in the stock gate/up layout keeps the stack off the tensor cores
  for (int l = 0; l < L; ++l) stock = stock || stock_layout(layers[l]);
  const bool batched = !stock && batched_eligible(*cfg, T);
  const bool gemv = !batched && gemv_eligible(*cfg, T, stock);
  const size_t TH = static_cast<size_t>(T) * cfg->hidden;
  const size_t Tk = static_cast<size_t>(T) * cfg->top_k;
  float* r = reinterpret_cast<float*>(b + Ly.r);
  uint16_t* xbuf[2] = {reinterpret_cast<uint16_t*>(b + Ly.xa), reinterpret_cast<uint16_t*>(b + Ly.xb)};

  if (trace && trace->x) {
    cudaError_t e = cudaMemcpyAsync(trace->x, x0, TH * 2, cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e, "trace copy");
  }
  moe::GlueParams g0{r, nullptr, x0, nullptr, T, cfg->hidden, 1e-6f};
  cudaError_t e = moe::launch_glue(g0, st);
  if (e != cudaSuccess) return cuda_fail(e, "glue launch");
  const uint16_t* xcur = x0;
  for (int l = 0; l < L; ++l) {
    int32_t* idx = (trace && trace->idx) ? trace->idx + l * Tk : reinterpret_cast<int32_t*>(b + Ly.idx);
    float* wt = (trace && trace->w) ? trace->w + l * Tk : reinterpret_cast<float*>(b + Ly.w);
    uint16_t* y = (trace && trace->y) ? trace->y + l * TH : reinterpret_cast<uint16_t*>(b + Ly.y);
    if ((s = route(*cfg, xcur, T, layers[l].router_w, layers[l].router_bias, idx, wt, v, st))) return s;
    if (batched) s = batched_ffn(*cfg, layers[l], xcur, T, idx, wt, y, ws, Ly, st);
    else if (gemv) s = gemv_ffn(*cfg, layers[l], xcur, T, idx, wt, y, ws, Ly, st);
    else s = ffn(*cfg, layers[l], xcur, T, idx, wt, y, v, st);
    if (s) return s;
    uint16_t* xnext;
    if (l == L - 1) xnext = x_out;
    else if (trace && trace->x) xnext = trace->x + (l + 1) * TH;
    else xnext = xbuf[l & 1];
    moe::GlueParams g{r, y, nullptr, xnext, T, cfg->hidden, 1e-6f};
    if ((e = moe::launch_glue(g, st)) != cudaSuccess) return cuda_fail(e, "glue launch");
    xcur = xnext;
  }
  return MOE_OK;
}

moe_status moe_sort_by_expert(const moe_config* cfg, const int32_t* topk_idx, int32_t T, int32_t* perm,
                              int32_t* offsets, void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status s;
  if ((s = check_cfg(cfg))) return s;
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T=%d", T);
  if ((s = check_ptr(offsets, 4, "offsets"))) return s;
  if (T > 0 && ((s = check_ptr(topk_idx, 4, "topk_idx")) || (s = check_ptr(perm, 4, "perm")))) return s;
  Layout L;
  if ((s = check_ws(*cfg, ws, ws_bytes, T, &L))) return s;
  moe::SortParams p{topk_idx, T, cfg->top_k, cfg->num_experts, cfg->shared_inter > 0 ? 1 : 0, perm, offsets,
                    nullptr, nullptr, 0, view(ws, L).hdr};
  cudaError_t e = moe::launch_sort_by_expert(p, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "sort_by_expert launch");
}

size_t moe_down_sb_size(const moe_config* cfg, int32_t n_experts, int32_t K) {
  if (check_cfg(cfg) != MOE_OK || n_experts < 1 || K < cfg->group || K % cfg->group) return 0;
  return static_cast<size_t>(n_experts) * (K / cfg->group) * cfg->hidden * 4;
}

moe_status moe_prepare_down_sb(const moe_config* cfg, const moe_qtensor* down, int32_t n_experts, int32_t K,
                               uint16_t* out, moe_stream_t stream) {
  moe_status s;
  if ((s = check_cfg(cfg))) return s;
  if (!down) return fail(MOE_ERR_INVALID_ARG, "down is NULL");
  if (n_experts < 1 || K < cfg->group || K % cfg->group)
    return fail(MOE_ERR_INVALID_ARG, "n_experts=%d K=%d (K a positive multiple of group %d)", n_experts, K,
                cfg->group);
  if ((s = check_qt(*down, cfg->hidden, K, cfg->bits, cfg->group, n_experts, "down"))) return s;
  if ((s = check_ptr(out, 16, "out"))) return s;
  const int64_t stride = n_experts > 1 ? down->sb_expert_stride : static_cast<int64_t>(cfg->hidden) * (K / cfg->group);
  cudaError_t e = moe::launch_prepare_down_sb(down->scales, down->biases, stride, n_experts, cfg->hidden,
                                              K / cfg->group, out, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "prepare_down_sb launch");
}

size_t moe_down_units_size(const moe_config* cfg, int32_t n_experts, int32_t K) {
  if (check_cfg(cfg) != MOE_OK || n_experts < 1 || K < cfg->group || K % cfg->group || K % 32) return 0;
  return static_cast<size_t>(n_experts) * K * cfg->hidden * cfg->bits / 8;
}

moe_status moe_prepare_down_units(const moe_config* cfg, const moe_qtensor* down, int32_t n_experts, int32_t K,
                                  uint8_t* out, moe_stream_t stream) {
  moe_status s;
  if ((s = check_cfg(cfg))) return s;
  if (!down) return fail(MOE_ERR_INVALID_ARG, "down is NULL");
  if (n_experts < 1 || K < cfg->group || K % cfg->group || K % 32)
    return fail(MOE_ERR_INVALID_ARG, "n_experts=%d K=%d (K a positive multiple of 32 and of group %d)", n_experts, K,
                cfg->group);
  if ((s = check_qt(*down, cfg->hidden, K, cfg->bits, cfg->group, n_experts, "down"))) return s;
  if ((s = check_ptr(out, 16, "out"))) return s;
  const int rowb = K * cfg->bits / 8;
  const int64_t stride = n_experts > 1 ? down->q_expert_stride : static_cast<int64_t>(cfg->hidden) * rowb;
  cudaError_t e = moe::launch_prepare_down_units(down->q, stride, n_experts, cfg->hidden, rowb, 32 * cfg->bits / 8,
                                                 out, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "prepare_down_units launch");
}

int32_t moe_set_batched_min_tokens(int32_t T) {
  return g_batch_min.exchange(T < 1 ? kBatchMinTokens : T);
}

int32_t moe_set_gemv_min_tokens(int32_t T) {
  return g_gemv_min.exchange(T < 1 ? kGemvMinTokens : T);
}

int32_t moe_set_decode_max_tokens(int32_t T) {
  return g_decode_max.exchange(T < 1 ? kDecodeMaxTokens : T);
}

moe_status moe_check_wait_limit(void* ws, size_t ws_bytes, int32_t* gave_up, moe_stream_t stream) {
  if (!ws || !aligned(ws, kAlign)) return fail(MOE_ERR_WORKSPACE, "workspace NULL or misaligned");
  if (ws_bytes < sizeof(moe::WsHeader)) return fail(MOE_ERR_WORKSPACE, "workspace too small");
  moe_status s;
  if ((s = check_ptr(gave_up, 4, "gave_up"))) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  moe::WsHeader* hdr = static_cast<moe::WsHeader*>(ws);
  cudaError_t e = cudaMemsetAsync(hdr, 0, sizeof(moe::WsHeader), st);
  if (e == cudaSuccess)
    e = moe::launch_wait_limit_check(hdr, reinterpret_cast<uint32_t*>(&hdr->pad[0]), gave_up, st);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "wait limit check");
}

moe_status moe_get_device_status(void* ws, moe_stream_t stream) {
  if (!ws || !aligned(ws, kAlign)) return fail(MOE_ERR_WORKSPACE, "workspace NULL or misaligned");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t hdr[2] = {0, 0};
  cudaError_t e = cudaMemcpyAsync(hdr, ws, sizeof(hdr), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  if (hdr[0] != 0) {
    fail(static_cast<moe_status>(hdr[0]), "device reported %s (detail %d)",
         moe_status_string(static_cast<moe_status>(hdr[0])), hdr[1]);
    e = cudaMemsetAsync(ws, 0, sizeof(hdr), st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "status clear");
    return static_cast<moe_status>(hdr[0]);
  }
  return MOE_OK;
}

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
    case MOE_ERR_BOUNDS: return "MOE_ERR_BOUNDS";
  }
  return "MOE_ERR_UNKNOWN";
}

const char* moe_last_error_string(void) { return g_last_error.c_str(); }

}  // extern "C"

// ---------------------------------------------------------------- allocation-free layer call
//
// moe_layer_forward_static runs the per-token kernels of moe_layer_forward
// (never the batched tensor-core path) and takes no workspace: its scratch
// (status word, routing counters, logits, gate activations: the regions of
// the workspace layout below `base_total`) lives in the fixed array below,
// which every GPU that loads this library holds until the process exits. It serves callers that
// cannot call cudaMalloc or hand the library a buffer of their own: code
// running inside a host framework that owns all device memory and forbids
// allocation after start-up, plugins that are handed only their inputs and
// outputs, and latency-critical paths where an allocation (which may
// synchronise the device) is not allowed.

namespace {

constexpr size_t kStaticScratchBytes = size_t(2) << 20;  // 2 MiB per GPU
constexpr int kMaxDevices = 128;

__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_static_mu;
void* g_static_ptr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device. In host code the
// symbol's name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and kept. The kept address
// belongs to the device's primary context as it was at that first call; it
// is stale after cudaDeviceReset, which the header tells callers.
moe_status static_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(MOE_ERR_UNSUPPORTED, "device ordinal %d >= %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (!g_static_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
    g_static_ptr[dev] = p;
  }
  *out = g_static_ptr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_layer_forward_static(const moe_config* cfg, const moe_layer_weights* w,
                                               const uint16_t* x, int32_t T, uint16_t* y, int32_t* topk_idx,
                                               float* topk_w, int32_t* device_status, moe_stream_t stream) {
  moe_status s;
  if ((s = check_cfg(cfg))) return s;
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T=%d", T);
  if (T == 0) return MOE_OK;
  if ((s = check_weights(*cfg, w, true))) return s;
  if ((s = check_ptr(x, 16, "x")) || (s = check_ptr(y, 16, "y"))) return s;
  if ((topk_idx && !aligned(topk_idx, 4)) || (topk_w && !aligned(topk_w, 4)) ||
      (device_status && !aligned(device_status, 4)))
    return fail(MOE_ERR_INVALID_ARG, "topk_idx/topk_w/device_status misaligned");
  const Layout L = layout(*cfg, T);
  if (L.base_total > kStaticScratchBytes)
    return fail(MOE_ERR_WORKSPACE, "T=%d needs %zu bytes of scratch; the static scratch holds %zu", T, L.base_total,
                kStaticScratchBytes);
  void* ws = nullptr;
  if ((s = static_scratch(&ws))) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // Status word and arrival counters must start at zero; the rest is overwritten.
  cudaError_t e = cudaMemsetAsync(ws, 0, L.logits, st);
  if (e != cudaSuccess) return cuda_fail(e, "static scratch clear");
  char* b = static_cast<char*>(ws);
  int32_t* idx = topk_idx ? topk_idx : reinterpret_cast<int32_t*>(b + L.idx);
  float* wt = topk_w ? topk_w : reinterpret_cast<float*>(b + L.w);
  const moe::WsView v = view(ws, L);
  if ((s = route(*cfg, x, T, w->router_w, w->router_bias, idx, wt, v, st))) return s;
  if ((s = ffn(*cfg, *w, x, T, idx, wt, y, v, st))) return s;
  if (device_status) {
    e = cudaMemcpyAsync(device_status, ws, sizeof(int32_t), cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e, "device status copy");
  }
  return MOE_OK;
}
