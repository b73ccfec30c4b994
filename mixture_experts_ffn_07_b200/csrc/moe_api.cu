// The C ABI of libmoe (declared in include/moe.h): argument checks, the
// workspace layout, the order of kernel launches for each entry point, the
// device status word, and the host-side launch counter and event trace.
//
// Path choice: bf16 activations with bf16 expert weights and T >= 16 (moe_set_tensor_min_tokens) take the
// tensor-core path (row gather + tcgen05 grouped GEMMs); everything else takes
// the weight-streaming path (expert-major GEMV kernels), which reads each
// touched expert's weights once and is the bandwidth-optimal form for small T.
#include <atomic>
#include <mutex>
#include <tuple>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "kernels.h"

namespace {

__device__ int g_device_status;  // one per device; first error wins, cleared by moe_last_device_status

constexpr int kMaxDevices = 64;
constexpr int kMaxT = 1 << 20;
constexpr int kTraceCap = 4096;

struct DeviceInfo {
  bool ready = false;
  int* status = nullptr;
  int num_sms = 0;
  int smem_optin = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

std::atomic<uint64_t> g_launches{0};
std::atomic<long long> g_wait_limit{1LL << 31};
std::atomic<int> g_skip_stage{0};
std::atomic<long long> g_barrier_delay{0};
std::atomic<int> g_fused_decode{1};
std::atomic<int> g_fused_front{1};
std::atomic<int> g_pair_gemm{1};
std::atomic<int> g_decode_stream{1};
std::atomic<int> g_tma_gather{0};

struct TraceRec {
  const char* name;
  cudaEvent_t start, stop;
};
std::mutex g_trace_mu;
bool g_trace_on = false;
int g_trace_n = 0;
TraceRec g_trace[kTraceCap];

bool make_ctx(cudaStream_t s, moe::Ctx* c) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DeviceInfo& d = g_dev[dev];
    if (!d.ready) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return false;
      int sms = 0, optin = 0;
      if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) return false;
      if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return false;
      d.status = static_cast<int*>(p);
      d.num_sms = sms;
      d.smem_optin = optin;
      d.ready = true;
    }
    c->status = d.status;
    c->num_sms = d.num_sms;
    c->smem_optin = d.smem_optin;
  }
  c->stream = s;
  c->wait_limit = g_wait_limit.load();
  c->skip_stage = g_skip_stage.load();
  c->barrier_delay = g_barrier_delay.load();
  c->pdl = 1;
  return true;
}

inline size_t align256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Fewest tokens for which a bf16 layer takes the tensor-core path (moe_set_tensor_min_tokens).  Measured
// on B200 (bench.py --op crossover): the decode stream is faster up to 8 tokens on every measured shape,
// the tensor-core path from 16 on two of the three, so 16.
std::atomic<int> g_tensor_min_tokens{16};

bool tensor_path(const moe_desc& d) {
  return d.act_dtype == MOE_BF16 && d.w_dtype == MOE_BF16 && d.T >= g_tensor_min_tokens.load();
}

bool tensor_router(const moe_desc& d) {
  return d.act_dtype == MOE_BF16 && d.router_dtype == MOE_BF16 && d.T >= g_tensor_min_tokens.load() && d.E % 32 == 0;
}

// Selection, permutation and row gather as one cooperative kernel after the
// tensor-core router GEMM (prefill_front.cu).
bool fused_front(const moe_desc& d) { return tensor_path(d) && tensor_router(d); }

// The whole layer as one cooperative kernel (decode_fused.cu): the streaming
// path with at most 64 tokens.
bool fused_decode(const moe_desc& d) {
  return !tensor_path(d) && d.T >= 1 && d.T <= moe::kMaxDecodeT && d.T * d.top_k <= moe::kMaxDecodePairs;
}

// Ranges the router GEMM splits the hidden dimension into, so that small batches
// still occupy the GPU: about 160 CTAs over the 128-token tiles, at most 16.
// A function of T alone, so logits do not depend on the device's SM count.
int router_ksplit(const moe_desc& d) {
  const int mtiles = (d.T + 127) / 128;
  return std::max(1, std::min(16, 160 / std::max(1, mtiles)));
}

bool shared_gated(const moe_desc& d) { return d.shared_I > 0 && d.has_shared_gate; }

moe_status check_desc(const moe_desc* d) {
  if (!d) return MOE_ERR_INVALID_ARG;
  if (d->T < 0 || d->T > kMaxT || d->H <= 0 || d->I <= 0 || d->E < 1 || d->E > 256 || d->top_k < 1 ||
      d->top_k > d->E || d->top_k > 32 || d->shared_I < 0)
    return MOE_ERR_INVALID_ARG;
  if ((d->act != MOE_ACT_SILU && d->act != MOE_ACT_GELU_TANH) || (d->renormalize != 0 && d->renormalize != 1) ||
      (d->has_router_bias != 0 && d->has_router_bias != 1) || (d->has_shared_gate != 0 && d->has_shared_gate != 1))
    return MOE_ERR_INVALID_ARG;
  if ((d->act_dtype != MOE_F32 && d->act_dtype != MOE_BF16) ||
      (d->w_dtype != MOE_F32 && d->w_dtype != MOE_BF16 && d->w_dtype != MOE_Q8_0 && d->w_dtype != MOE_Q4_K &&
       d->w_dtype != MOE_Q4_K_Q6_K) ||
      (d->router_dtype != MOE_F32 && d->router_dtype != MOE_BF16))
    return MOE_ERR_INVALID_ARG;
  if (d->H % 32 || d->I % 32 || d->shared_I % 32) return MOE_ERR_UNSUPPORTED;
  if ((d->w_dtype == MOE_Q4_K || d->w_dtype == MOE_Q4_K_Q6_K) && (d->H % 256 || d->I % 256 || d->shared_I % 256))
    return MOE_ERR_UNSUPPORTED;
  if (d->gating != MOE_GATING_SOFTMAX && d->gating != MOE_GATING_SIGMOID) return MOE_ERR_INVALID_ARG;
  if (d->n_groups < 0 || d->n_groups > 32) return MOE_ERR_INVALID_ARG;
  if (d->n_groups > 1) {
    if (d->E % d->n_groups || d->topk_groups < 1 || d->topk_groups > d->n_groups ||
        d->top_k > d->topk_groups * (d->E / d->n_groups))
      return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

moe::RouteCfg route_cfg(const moe_desc& d) {
  moe::RouteCfg r{};
  r.E = d.E;
  r.K = d.top_k;
  r.renorm = d.renormalize;
  r.gating = d.gating;
  r.n_groups = d.n_groups > 1 ? d.n_groups : 1;
  r.topk_groups = d.n_groups > 1 ? d.topk_groups : 1;
  return r;
}

struct Layout {
  size_t logits, logit_parts, router_parts, stream_sync, front_hist, ids, w, shared_gate, counts, offsets, sorted_pairs, pair_pos,
      y_slots, x_perm, h, h_s, y_s, total;
};

Layout layout_of(const moe_desc& d) {
  Layout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  const size_t T = d.T, H = d.H, E = d.E, I = d.I, P = T * d.top_k, Is = d.shared_I;
  const bool tc = tensor_path(d);
  L.logits = take(T * E * 4);
  L.logit_parts = tensor_router(d) ? take(router_ksplit(d) * T * E * 4) : 0;
  L.router_parts = fused_decode(d) ? take(moe::decode_router_parts_floats(d.T, d.H, d.E, shared_gated(d)) * 4) : 0;
  L.stream_sync = fused_decode(d) ? take(moe::decode_stream_sync_bytes()) : 0;
  L.front_hist = fused_front(d) ? take(static_cast<size_t>(moe::kMaxFrontCtas) * E * 4) : 0;
  L.ids = take(P * 4);
  L.w = take(P * 4);
  L.shared_gate = take(T * 4);
  L.counts = take(E * 4);
  L.offsets = take((E + 1) * 4);
  L.sorted_pairs = take(P * 4);
  L.pair_pos = take(P * 4);
  L.y_slots = take(P * H * 4);
  L.x_perm = tc && !g_tma_gather.load() ? take(P * H * 2) : 0;
  L.h = take(P * I * (tc ? 2 : 4));
  L.h_s = Is ? take(T * Is * (tc ? 2 : 4)) : 0;
  L.y_s = Is ? take(T * H * 4) : 0;
  L.total = off;
  return L;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

moe_status from_cuda(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

#define MOE_TRY(expr)                          \
  do {                                         \
    const cudaError_t e_ = (expr);             \
    if (e_ != cudaSuccess) return MOE_ERR_CUDA; \
  } while (0)

// ---------------------------------------------------------------- stages
// parts: scratch for the split-K partial logits (nullptr: no split).
// The tensor-core router GEMM: logits (or, with `parts`, split-K partials
// that the selection adds in order).  Returns the number of partial arrays
// (0: the logits are complete) through *nparts.
moe_status router_gemm(const moe::Ctx& c, const moe_desc& d, const void* x, const moe_weights& w, float* logits,
                       float* parts, int* nparts) {
  const int ksplit = parts ? moe::effective_ksplit(router_ksplit(d), d.H) : 1;
  moe::GemmArgs a{};
  a.A = static_cast<const __nv_bfloat16*>(x);
  a.rows_A = d.T;
  a.Kdim = d.H;
  a.B0 = static_cast<const __nv_bfloat16*>(w.router);
  a.N = d.E;
  a.G = 1;
  a.max_rows = d.T;
  a.dual = false;
  a.out_f32 = ksplit > 1 ? parts : logits;
  a.ksplit = ksplit;
  a.part_stride = static_cast<size_t>(d.T) * d.E;
  a.name = "router_gemm";
  MOE_TRY(moe::launch_grouped_gemm(c, a));
  *nparts = ksplit > 1 ? ksplit : 0;
  return MOE_OK;
}

moe_status route_impl(const moe::Ctx& c, const moe_desc& d, const void* x, const moe_weights& w, float* logits,
                      float* parts, int32_t* ids, float* tw, float* shared_gate) {
  const void* w_s = shared_gated(d) ? w.sh_gate_w : nullptr;
  if (tensor_router(d)) {
    const int ksplit = parts ? moe::effective_ksplit(router_ksplit(d), d.H) : 1;
    moe::GemmArgs a{};
    a.A = static_cast<const __nv_bfloat16*>(x);
    a.rows_A = d.T;
    a.Kdim = d.H;
    a.B0 = static_cast<const __nv_bfloat16*>(w.router);
    a.N = d.E;
    a.G = 1;
    a.max_rows = d.T;
    a.dual = false;
    a.out_f32 = ksplit > 1 ? parts : logits;
    a.ksplit = ksplit;
    a.part_stride = static_cast<size_t>(d.T) * d.E;
    a.name = "router_gemm";
    MOE_TRY(moe::launch_grouped_gemm(c, a));
    MOE_TRY(moe::launch_router_topk(c, parts, ksplit > 1 ? ksplit : 0, a.part_stride, logits,
                                    d.has_router_bias ? w.router_bias : nullptr, d.T, route_cfg(d), ids, tw, x,
                                    d.act_dtype, w_s, d.router_dtype, d.H, shared_gate));
  } else {
    MOE_TRY(moe::launch_router_fused(c, x, d.act_dtype, w.router, w_s, d.router_dtype,
                                     d.has_router_bias ? w.router_bias : nullptr, d.T, d.H, route_cfg(d), logits, ids,
                                     tw, shared_gate));
  }
  return MOE_OK;
}

// bf16_slots (tensor-core path of moe_layer): the slot rows hold the experts' unweighted outputs in bf16 and
// the combine applies the routing weights (mlx-native moe_dispatch.rs, moe_weighted_sum_seq_bf16_input);
// otherwise they hold topk_w-weighted f32 rows, as moe_expert_ffn documents.
moe_status expert_impl(const moe::Ctx& c, const moe_desc& d, const void* x, const moe_weights& w,
                       const int32_t* offsets, const int32_t* sorted_pairs, const float* tw, float* y_slots, void* ws,
                       const Layout& L, bool rows_gathered = false, bool bf16_slots = false) {
  const int P = d.T * d.top_k;
  if (tensor_path(d)) {
    __nv_bfloat16* h = at<__nv_bfloat16>(ws, L.h);
    moe::GemmArgs a{};
    if (L.x_perm == 0) {  // the GEMM gathers each pair's x row itself (TMA tile::gather4)
      a.gather_rows = sorted_pairs;
      a.gather_div = d.top_k;
      a.A_src = static_cast<const __nv_bfloat16*>(x);
      a.rows_src = d.T;
    } else {  // x rows copied into expert order first
      __nv_bfloat16* xp = at<__nv_bfloat16>(ws, L.x_perm);
      if (!rows_gathered)
        MOE_TRY(moe::launch_gather_rows(c, static_cast<const __nv_bfloat16*>(x), sorted_pairs, offsets, d.E,
                                        d.top_k, P, d.H, xp));
      a.A = xp;
    }
    a.rows_A = P;
    a.Kdim = d.H;
    a.B0 = static_cast<const __nv_bfloat16*>(w.gate);
    a.B1 = static_cast<const __nv_bfloat16*>(w.up);
    a.N = d.I;
    a.G = d.E;
    a.offsets = offsets;
    a.max_rows = P;
    a.dual = true;
    a.act = d.act;
    a.out_bf16 = h;
    a.name = "expert_gate_up_gemm";
    MOE_TRY(moe::launch_grouped_gemm(c, a));
    moe::GemmArgs b{};
    b.A = h;
    b.rows_A = P;
    b.Kdim = d.I;
    b.B0 = static_cast<const __nv_bfloat16*>(w.down);
    b.N = d.H;
    b.G = d.E;
    b.offsets = offsets;
    b.max_rows = P;
    b.dual = false;
    if (bf16_slots) {
      b.out_bf16 = reinterpret_cast<__nv_bfloat16*>(y_slots);
    } else {
      b.out_f32 = y_slots;
      b.row_scale = tw;
    }
    b.row_map = sorted_pairs;
    b.name = "expert_down_gemm";
    MOE_TRY(moe::launch_grouped_gemm(c, b));
  } else {
    float* h = at<float>(ws, L.h);
    MOE_TRY(moe::launch_stream_gate_up(c, x, d.act_dtype, d.T, d.H, d.I, d.top_k, w.gate, w.up, w.gate_scale,
                                       w.up_scale, d.w_dtype, offsets, d.E, sorted_pairs, P, d.act, h));
    MOE_TRY(moe::launch_stream_down(c, h, d.I, d.H, w.down, w.down_scale, d.w_dtype, offsets, d.E, sorted_pairs, P,
                                    tw, y_slots));
  }
  return MOE_OK;
}

moe_status combine_impl(const moe::Ctx& c, const moe_desc& d, const float* y_slots, const void* x,
                        const moe_weights& w, const float* shared_gate, void* out, void* ws, const Layout& L,
                        const float* bf16_slot_weights = nullptr) {
  float* y_s = nullptr;
  if (d.shared_I > 0) {
    y_s = at<float>(ws, L.y_s);
    const float* gate = shared_gated(d) ? shared_gate : nullptr;
    if (tensor_path(d)) {
      __nv_bfloat16* hs = at<__nv_bfloat16>(ws, L.h_s);
      moe::GemmArgs a{};
      a.A = static_cast<const __nv_bfloat16*>(x);
      a.rows_A = d.T;
      a.Kdim = d.H;
      a.B0 = static_cast<const __nv_bfloat16*>(w.sh_gate);
      a.B1 = static_cast<const __nv_bfloat16*>(w.sh_up);
      a.N = d.shared_I;
      a.G = 1;
      a.max_rows = d.T;
      a.dual = true;
      a.act = d.act;
      a.out_bf16 = hs;
      a.name = "shared_gate_up_gemm";
      MOE_TRY(moe::launch_grouped_gemm(c, a));
      moe::GemmArgs b{};
      b.A = hs;
      b.rows_A = d.T;
      b.Kdim = d.shared_I;
      b.B0 = static_cast<const __nv_bfloat16*>(w.sh_down);
      b.N = d.H;
      b.G = 1;
      b.max_rows = d.T;
      b.dual = false;
      b.out_f32 = y_s;
      b.row_scale = gate;
      b.name = "shared_down_gemm";
      MOE_TRY(moe::launch_grouped_gemm(c, b));
    } else {
      float* hs = at<float>(ws, L.h_s);
      MOE_TRY(moe::launch_stream_gate_up(c, x, d.act_dtype, d.T, d.H, d.shared_I, 1, w.sh_gate, w.sh_up,
                                         w.sh_gate_scale, w.sh_up_scale, d.w_dtype, nullptr, 1, nullptr, d.T, d.act,
                                         hs));
      MOE_TRY(moe::launch_stream_down(c, hs, d.shared_I, d.H, w.sh_down, w.sh_down_scale, d.w_dtype, nullptr, 1,
                                      nullptr, d.T, gate, y_s));
    }
  }
  if (bf16_slot_weights)
    MOE_TRY(moe::launch_combine_weighted(c, reinterpret_cast<const __nv_bfloat16*>(y_slots), bf16_slot_weights, y_s,
                                         d.T, d.top_k, d.H, out));
  else
    MOE_TRY(moe::launch_combine(c, y_slots, y_s, d.T, d.top_k, d.H, out, d.act_dtype));
  return MOE_OK;
}

// ---------------------------------------------------------------- argument checks
moe_status check_router_args(const moe_desc& d, const void* x, const moe_weights* w) {
  if (!x || !w || !w->router || !aligned16(x) || !aligned16(w->router)) return MOE_ERR_INVALID_ARG;
  if (d.has_router_bias && !w->router_bias) return MOE_ERR_INVALID_ARG;
  if (shared_gated(d) && (!w->sh_gate_w || !aligned16(w->sh_gate_w))) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

// The weight-streaming kernels stage whole token rows in shared memory:
// x rows (H elements) and hidden rows (I or shared_I f32) of at most 64 KB.
bool stream_rows_fit(const moe_desc& d, int inner) {
  const long long xb = static_cast<long long>(d.H) * (d.act_dtype == MOE_F32 ? 4 : 2);
  return xb <= 65536 && static_cast<long long>(inner) * 4 <= 65536;
}

moe_status check_expert_weights(const moe_desc& d, const moe_weights* w) {
  if (!tensor_path(d) && !stream_rows_fit(d, d.I)) return MOE_ERR_UNSUPPORTED;
  if (!w || !w->gate || !w->up || !w->down) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w->gate) || !aligned16(w->up) || !aligned16(w->down)) return MOE_ERR_INVALID_ARG;
  if (d.w_dtype == MOE_Q8_0 && (!w->gate_scale || !w->up_scale || !w->down_scale)) return MOE_ERR_INVALID_ARG;
  if (d.w_dtype == MOE_Q4_K_Q6_K && (!w->down_scale || !aligned16(w->down_scale))) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

moe_status check_shared_weights(const moe_desc& d, const moe_weights* w) {
  if (d.shared_I == 0) return MOE_OK;
  if (!tensor_path(d) && !stream_rows_fit(d, d.shared_I)) return MOE_ERR_UNSUPPORTED;
  if (!w || !w->sh_gate || !w->sh_up || !w->sh_down) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w->sh_gate) || !aligned16(w->sh_up) || !aligned16(w->sh_down)) return MOE_ERR_INVALID_ARG;
  if (d.w_dtype == MOE_Q8_0 && (!w->sh_gate_scale || !w->sh_up_scale || !w->sh_down_scale))
    return MOE_ERR_INVALID_ARG;
  if (d.w_dtype == MOE_Q4_K_Q6_K && (!w->sh_down_scale || !aligned16(w->sh_down_scale))) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

}  // namespace

// ---------------------------------------------------------------- instrumentation
namespace moe {

cudaError_t allow_dynamic_smem(const void* kernel, int bytes) {
  static std::mutex mu;
  static std::vector<std::tuple<const void*, int, int>> done;  // (kernel, device, bytes)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(mu);
  for (const auto& d : done)
    if (std::get<0>(d) == kernel && std::get<1>(d) == dev && std::get<2>(d) >= bytes) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.emplace_back(kernel, dev, bytes);
  return e;
}

// Every launch also opens an NVTX range named after its kernel, so a profiler's
// timeline groups the launches by step; without a profiler attached the NVTX
// calls return at once.
bool pair_gemm_enabled() { return g_pair_gemm.load() != 0; }

int stream_path_mode() { return g_decode_stream.load(); }

KernelScope::KernelScope(const Ctx& c, const char* name) : ctx(c), slot(-1) {
  g_launches.fetch_add(1);
  nvtxRangePushA(name);
  std::lock_guard<std::mutex> lk(g_trace_mu);
  if (g_trace_on && g_trace_n < kTraceCap) {
    TraceRec& r = g_trace[g_trace_n];
    if (!r.start) {
      cudaEventCreate(&r.start);
      cudaEventCreate(&r.stop);
    }
    r.name = name;
    slot = g_trace_n++;
    cudaEventRecord(r.start, c.stream);
  }
}

KernelScope::~KernelScope() {
  if (slot >= 0) cudaEventRecord(g_trace[slot].stop, ctx.stream);
  nvtxRangePop();
}

}  // namespace moe

// ---------------------------------------------------------------- C ABI
extern "C" {

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported size or format";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_TIMEOUT: return "device wait timed out";
    case MOE_ERR_DEVICE_INDEX: return "expert id out of range";
  }
  return "unknown status";
}

const char* moe_version(void) { return "moe-b200 0.1 (sm_100a)"; }

size_t moe_workspace_bytes(const moe_desc* d) {
  if (check_desc(d) != MOE_OK) return 0;
  return layout_of(*d).total;
}

moe_status moe_workspace_regions(const moe_desc* d, moe_ws_regions* r) {
  if (!r || check_desc(d) != MOE_OK) return MOE_ERR_INVALID_ARG;
  const Layout L = layout_of(*d);
  r->logits = L.logits;
  r->topk_ids = L.ids;
  r->topk_w = L.w;
  r->shared_gate = L.shared_gate;
  r->counts = L.counts;
  r->offsets = L.offsets;
  r->sorted_pairs = L.sorted_pairs;
  r->pair_pos = L.pair_pos;
  return MOE_OK;
}

moe_status moe_route(const moe_desc* d, const void* x, const moe_weights* w, float* logits, int32_t* topk_ids,
                     float* topk_w, float* shared_gate, void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status st = check_desc(d);
  if (st != MOE_OK) return st;
  if (d->T == 0) return MOE_OK;
  if ((st = check_router_args(*d, x, w)) != MOE_OK) return st;
  if (!logits || !topk_ids || !topk_w || !aligned16(logits)) return MOE_ERR_INVALID_ARG;
  if (shared_gated(*d) && !shared_gate) return MOE_ERR_INVALID_ARG;
  const Layout L = layout_of(*d);
  if (ws && ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  if (ws && !aligned16(ws)) return MOE_ERR_INVALID_ARG;
  moe::Ctx c;
  if (!make_ctx(reinterpret_cast<cudaStream_t>(stream), &c)) return MOE_ERR_CUDA;
  float* parts = (ws && L.logit_parts) ? at<float>(ws, L.logit_parts) : nullptr;
  return route_impl(c, *d, x, *w, logits, parts, topk_ids, topk_w, shared_gate);
}

moe_status moe_permute(const moe_desc* d, const int32_t* topk_ids, int32_t* counts, int32_t* offsets,
                       int32_t* sorted_pairs, int32_t* pair_pos, moe_stream_t stream) {
  moe_status st = check_desc(d);
  if (st != MOE_OK) return st;
  if (d->T == 0) return MOE_OK;
  if (!topk_ids || !counts || !offsets || !sorted_pairs || !pair_pos) return MOE_ERR_INVALID_ARG;
  moe::Ctx c;
  if (!make_ctx(reinterpret_cast<cudaStream_t>(stream), &c)) return MOE_ERR_CUDA;
  return from_cuda(moe::launch_permute(c, topk_ids, d->T * d->top_k, d->E, counts, offsets, sorted_pairs, pair_pos));
}

moe_status moe_expert_ffn(const moe_desc* d, const void* x, const moe_weights* w, const int32_t* offsets,
                          const int32_t* sorted_pairs, const float* topk_w, float* y_slots, void* ws,
                          size_t ws_bytes, moe_stream_t stream) {
  moe_status st = check_desc(d);
  if (st != MOE_OK) return st;
  if (d->T == 0) return MOE_OK;
  if ((st = check_expert_weights(*d, w)) != MOE_OK) return st;
  if (!x || !aligned16(x) || !offsets || !sorted_pairs || !topk_w || !y_slots || !aligned16(y_slots))
    return MOE_ERR_INVALID_ARG;
  const Layout L = layout_of(*d);
  if (!ws || ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  if (!aligned16(ws)) return MOE_ERR_INVALID_ARG;
  moe::Ctx c;
  if (!make_ctx(reinterpret_cast<cudaStream_t>(stream), &c)) return MOE_ERR_CUDA;
  return expert_impl(c, *d, x, *w, offsets, sorted_pairs, topk_w, y_slots, ws, L);
}

moe_status moe_combine(const moe_desc* d, const float* y_slots, const void* x, const moe_weights* w,
                       const float* shared_gate, void* out, void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status st = check_desc(d);
  if (st != MOE_OK) return st;
  if (d->T == 0) return MOE_OK;
  if (!y_slots || !out || !aligned16(y_slots) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  if (d->shared_I > 0) {
    if ((st = check_shared_weights(*d, w)) != MOE_OK) return st;
    if (!x || !aligned16(x)) return MOE_ERR_INVALID_ARG;
    if (shared_gated(*d) && !shared_gate) return MOE_ERR_INVALID_ARG;
  }
  const Layout L = layout_of(*d);
  if (d->shared_I > 0 && (!ws || ws_bytes < L.total)) return MOE_ERR_WORKSPACE;
  if (ws && !aligned16(ws)) return MOE_ERR_INVALID_ARG;
  moe::Ctx c;
  if (!make_ctx(reinterpret_cast<cudaStream_t>(stream), &c)) return MOE_ERR_CUDA;
  return combine_impl(c, *d, y_slots, x, *w, shared_gate, out, ws, L);
}

moe_status moe_layer(const moe_desc* d, const void* x, const moe_weights* w, void* out, void* ws, size_t ws_bytes,
                     moe_stream_t stream) {
  moe_status st = check_desc(d);
  if (st != MOE_OK) return st;
  if (d->T == 0) return MOE_OK;
  if ((st = check_router_args(*d, x, w)) != MOE_OK) return st;
  if ((st = check_expert_weights(*d, w)) != MOE_OK) return st;
  if ((st = check_shared_weights(*d, w)) != MOE_OK) return st;
  if (!out || !aligned16(out) || out == x) return MOE_ERR_INVALID_ARG;
  const Layout L = layout_of(*d);
  if (!ws || ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  if (!aligned16(ws)) return MOE_ERR_INVALID_ARG;
  moe::Ctx c;
  if (!make_ctx(reinterpret_cast<cudaStream_t>(stream), &c)) return MOE_ERR_CUDA;
  float* logits = at<float>(ws, L.logits);
  int32_t* ids = at<int32_t>(ws, L.ids);
  float* tw = at<float>(ws, L.w);
  float* sg = at<float>(ws, L.shared_gate);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* sorted_pairs = at<int32_t>(ws, L.sorted_pairs);
  float* y_slots = at<float>(ws, L.y_slots);
  float* parts = L.logit_parts ? at<float>(ws, L.logit_parts) : nullptr;
  if (fused_decode(*d) && g_fused_decode.load()) {
    moe::DecodeLayer f{};
    f.x = x;
    f.x_dtype = d->act_dtype;
    f.router = w->router;
    f.router_dtype = d->router_dtype;
    f.bias = d->has_router_bias ? w->router_bias : nullptr;
    f.w_s = shared_gated(*d) ? w->sh_gate_w : nullptr;
    f.T = d->T;
    f.H = d->H;
    f.E = d->E;
    f.K = d->top_k;
    f.I = d->I;
    f.Is = d->shared_I;
    f.act = d->act;
    f.renorm = d->renormalize;
    f.rc = route_cfg(*d);
    f.w_dtype = d->w_dtype;
    f.gate = w->gate;
    f.up = w->up;
    f.down = w->down;
    f.gate_scale = w->gate_scale;
    f.up_scale = w->up_scale;
    f.down_scale = w->down_scale;
    f.sh_gate = w->sh_gate;
    f.sh_up = w->sh_up;
    f.sh_down = w->sh_down;
    f.sh_gate_scale = w->sh_gate_scale;
    f.sh_up_scale = w->sh_up_scale;
    f.sh_down_scale = w->sh_down_scale;
    f.router_parts = at<float>(ws, L.router_parts);
    f.stream_sync = at<void>(ws, L.stream_sync);
    f.logits = logits;
    f.ids = ids;
    f.w = tw;
    f.shared_gate = sg;
    f.counts = at<int32_t>(ws, L.counts);
    f.offsets = offsets;
    f.sorted_pairs = sorted_pairs;
    f.pair_pos = at<int32_t>(ws, L.pair_pos);
    f.h = at<float>(ws, L.h);
    f.h_s = d->shared_I ? at<float>(ws, L.h_s) : nullptr;
    f.y_slots = y_slots;
    f.y_s = d->shared_I ? at<float>(ws, L.y_s) : nullptr;
    f.out = out;
    const cudaError_t e = moe::launch_decode_layer(c, f);
    if (e == cudaSuccess) return MOE_OK;
    // the grid cannot be made resident (or the shape does not fit one CTA per SM):
    // clear the launch error and take the step-by-step path
    if (e != cudaErrorCooperativeLaunchTooLarge && e != cudaErrorInvalidValue) return MOE_ERR_CUDA;
    cudaGetLastError();
  }
  if (fused_front(*d) && g_fused_front.load()) {
    int nparts = 0;
    if ((st = router_gemm(c, *d, x, *w, logits, parts, &nparts)) != MOE_OK) return st;
    moe::PrefillFront f{};
    f.parts = parts;
    f.nparts = nparts;
    f.part_stride = static_cast<size_t>(d->T) * d->E;
    f.logits = logits;
    f.bias = d->has_router_bias ? w->router_bias : nullptr;
    f.T = d->T;
    f.E = d->E;
    f.K = d->top_k;
    f.renorm = d->renormalize;
    f.H = d->H;
    f.rc = route_cfg(*d);
    f.ids = ids;
    f.w = tw;
    f.x = static_cast<const __nv_bfloat16*>(x);
    f.w_s = shared_gated(*d) ? static_cast<const __nv_bfloat16*>(w->sh_gate_w) : nullptr;
    f.shared_gate = sg;
    f.counts = at<int32_t>(ws, L.counts);
    f.offsets = offsets;
    f.sorted_pairs = sorted_pairs;
    f.pair_pos = at<int32_t>(ws, L.pair_pos);
    f.x_perm = L.x_perm ? at<__nv_bfloat16>(ws, L.x_perm) : nullptr;
    f.hist = at<int32_t>(ws, L.front_hist);
    const cudaError_t e = moe::launch_prefill_front(c, f);
    bool gathered = e == cudaSuccess;
    if (!gathered) {  // the grid cannot be made resident: the three steps as separate launches
      if (e != cudaErrorCooperativeLaunchTooLarge && e != cudaErrorInvalidValue) return MOE_ERR_CUDA;
      cudaGetLastError();
      const void* w_s = shared_gated(*d) ? w->sh_gate_w : nullptr;
      MOE_TRY(moe::launch_router_topk(c, parts, nparts, f.part_stride, logits, f.bias, d->T, f.rc, ids, tw, x,
                                      d->act_dtype, w_s, d->router_dtype, d->H, sg));
      MOE_TRY(moe::launch_permute(c, ids, d->T * d->top_k, d->E, f.counts, offsets, sorted_pairs, f.pair_pos));
    }
    if ((st = expert_impl(c, *d, x, *w, offsets, sorted_pairs, tw, y_slots, ws, L, gathered, true)) != MOE_OK)
      return st;
    return combine_impl(c, *d, y_slots, x, *w, sg, out, ws, L, tw);
  }
  if ((st = route_impl(c, *d, x, *w, logits, parts, ids, tw, sg)) != MOE_OK) return st;
  MOE_TRY(moe::launch_permute(c, ids, d->T * d->top_k, d->E, at<int32_t>(ws, L.counts), offsets, sorted_pairs,
                              at<int32_t>(ws, L.pair_pos)));
  const bool bf16_slots = tensor_path(*d);
  if ((st = expert_impl(c, *d, x, *w, offsets, sorted_pairs, tw, y_slots, ws, L, false, bf16_slots)) != MOE_OK)
    return st;
  return combine_impl(c, *d, y_slots, x, *w, sg, out, ws, L, bf16_slots ? tw : nullptr);
}

moe_status moe_layer_host(const moe_desc* d, const void* x_host, const moe_weights* w, void* out_host, void* x_dev,
                          void* out_dev, void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status st = check_desc(d);
  if (st != MOE_OK) return st;
  if (d->T == 0) return MOE_OK;
  if (!x_host || !out_host || !x_dev || !out_dev) return MOE_ERR_INVALID_ARG;
  const size_t bytes = static_cast<size_t>(d->T) * d->H * (d->act_dtype == MOE_F32 ? 4 : 2);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (d->T > 0 && cudaMemcpyAsync(x_dev, x_host, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if ((st = moe_layer(d, x_dev, w, out_dev, ws, ws_bytes, stream)) != MOE_OK) return st;
  if (d->T > 0 && cudaMemcpyAsync(out_host, out_dev, bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status moe_q8_0_split(const void* blocks, int64_t rows, int64_t cols, int8_t* q, void* scales,
                          moe_stream_t stream) {
  if (rows < 0 || cols < 0 || cols % 32) return MOE_ERR_INVALID_ARG;
  if (rows * cols == 0) return MOE_OK;
  if (!blocks || !q || !scales || !aligned16(q) || (reinterpret_cast<uintptr_t>(scales) & 1u))
    return MOE_ERR_INVALID_ARG;
  moe::Ctx c;
  if (!make_ctx(reinterpret_cast<cudaStream_t>(stream), &c)) return MOE_ERR_CUDA;
  return from_cuda(moe::launch_q8_0_split(c, blocks, rows, cols, q, scales));
}

namespace {
bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}
}  // namespace

moe_status moe_combine_backward(int64_t T, int64_t K, int64_t H, const float* y, const float* w, const float* d_out,
                                float* d_y, float* d_w, moe_stream_t stream) {
  if (T < 0 || K < 1 || H < 1 || T > 0x7fffffffLL || K > 0x7fffffffLL || T * K > 0x1ffffffffLL)
    return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!y || !w || !d_out || !d_y || !d_w) return MOE_ERR_INVALID_ARG;
  const size_t ny = static_cast<size_t>(T) * K * H * 4, nw = static_cast<size_t>(T) * K * 4,
               nd = static_cast<size_t>(T) * H * 4;
  for (const void* out : {static_cast<const void*>(d_y), static_cast<const void*>(d_w)}) {
    const size_t no = out == d_y ? ny : nw;
    if (overlaps(out, no, y, ny) || overlaps(out, no, w, nw) || overlaps(out, no, d_out, nd))
      return MOE_ERR_INVALID_ARG;
  }
  if (overlaps(d_y, ny, d_w, nw)) return MOE_ERR_INVALID_ARG;
  moe::Ctx c;
  if (!make_ctx(reinterpret_cast<cudaStream_t>(stream), &c)) return MOE_ERR_CUDA;
  return from_cuda(moe::launch_combine_backward(c, y, w, d_out, T, static_cast<int>(K), H, d_y, d_w));
}

moe_status moe_act_up_backward(int64_t P, int64_t I, int32_t act, const float* gate_up, const float* d_h,
                               float* d_gate_up, moe_stream_t stream) {
  if (P < 0 || I < 1 || (act != MOE_ACT_SILU && act != MOE_ACT_GELU_TANH)) return MOE_ERR_INVALID_ARG;
  if (P == 0) return MOE_OK;
  if (!gate_up || !d_h || !d_gate_up) return MOE_ERR_INVALID_ARG;
  const size_t ng = static_cast<size_t>(P) * 2 * I * 4, nh = static_cast<size_t>(P) * I * 4;
  if (overlaps(d_gate_up, ng, gate_up, ng) || overlaps(d_gate_up, ng, d_h, nh)) return MOE_ERR_INVALID_ARG;
  moe::Ctx c;
  if (!make_ctx(reinterpret_cast<cudaStream_t>(stream), &c)) return MOE_ERR_CUDA;
  return from_cuda(moe::launch_act_up_backward(c, gate_up, d_h, P, I, act, d_gate_up));
}

moe_status moe_q6_k_split(const void* blocks, int64_t rows, int64_t cols, void* q, void* scales,
                          moe_stream_t stream) {
  if (rows < 0 || cols < 0 || cols % 256 || cols > (1LL << 30)) return MOE_ERR_INVALID_ARG;
  if (rows * cols == 0) return MOE_OK;
  if (!blocks || !q || !scales || !aligned16(q) || !aligned16(scales)) return MOE_ERR_INVALID_ARG;
  moe::Ctx c;
  if (!make_ctx(reinterpret_cast<cudaStream_t>(stream), &c)) return MOE_ERR_CUDA;
  return from_cuda(moe::launch_q6_k_split(c, blocks, rows, cols, q, scales));
}

moe_status moe_last_device_status(moe_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
  int v = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  return static_cast<moe_status>(v);
}

uint64_t moe_launch_count(void) { return g_launches.load(); }

void moe_trace_enable(int on) {
  std::lock_guard<std::mutex> lk(g_trace_mu);
  g_trace_on = on != 0;
  if (g_trace_on) g_trace_n = 0;
}

int moe_trace_read(const char** names, float* ms, int max) {
  std::lock_guard<std::mutex> lk(g_trace_mu);
  for (int i = 0; i < g_trace_n && i < max; ++i) {
    float t = -1.f;
    if (cudaEventSynchronize(g_trace[i].stop) == cudaSuccess) cudaEventElapsedTime(&t, g_trace[i].start, g_trace[i].stop);
    if (names) names[i] = g_trace[i].name;
    if (ms) ms[i] = t;
  }
  return g_trace_n;
}

// ---------------------------------------------------------------- moe_layer without allocation
// The scratch of moe_layer_noalloc.  In host code this name is only a stand-in
// for the device symbol; the kernels get the address that cudaGetSymbolAddress
// returns for the current device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];
static void* g_noalloc_addr[kMaxDevices];
static std::mutex g_noalloc_mu;

// Device address of the static scratch on the current device, looked up once per device.
static void* noalloc_scratch() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_noalloc_addr[dev] = p;
  }
  return g_noalloc_addr[dev];
}

moe_status moe_layer_noalloc(const moe_desc* d, const void* x, const moe_weights* w, void* out,
                             moe_stream_t stream) {
  moe_status st = check_desc(d);
  if (st != MOE_OK) return st;
  if (d->T == 0) return MOE_OK;
  if (layout_of(*d).total > MOE_NOALLOC_SCRATCH_BYTES) return MOE_ERR_WORKSPACE;
  void* ws = noalloc_scratch();
  if (!ws) return MOE_ERR_CUDA;
  return moe_layer(d, x, w, out, ws, MOE_NOALLOC_SCRATCH_BYTES, stream);
}

void moe_debug_set_wait_limit(int64_t cycles) { g_wait_limit.store(cycles > 0 ? cycles : (1LL << 31)); }

void moe_debug_set_skip_stage(int enable) { g_skip_stage.store(enable ? 1 : 0); }

void moe_debug_set_barrier_delay(int64_t cycles) { g_barrier_delay.store(cycles > 0 ? cycles : 0); }

void moe_set_fused_decode(int enable) { g_fused_decode.store(enable ? 1 : 0); }

void moe_set_fused_front(int enable) { g_fused_front.store(enable ? 1 : 0); }

void moe_set_pair_gemm(int enable) { g_pair_gemm.store(enable ? 1 : 0); }

void moe_set_decode_stream(int enable) { g_decode_stream.store(enable ? 1 : 0); }

void moe_set_tma_gather(int enable) { g_tma_gather.store(enable ? 1 : 0); }

void moe_set_tensor_min_tokens(int tokens) { g_tensor_min_tokens.store(std::max(1, tokens)); }

}  // extern "C"
