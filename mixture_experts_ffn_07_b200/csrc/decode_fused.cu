// The whole MoE layer for a small batch (T <= 64) in one cooperative launch.
//
// Decode is bandwidth-bound on the touched experts' weights (a few hundred MB
// at most), so the cost that remains after streaming them at full speed is the
// chain of dependent launches: router, permutation, gate/up, down, combine,
// each with its launch latency, pipeline ramp and tail.  Here one persistent
// grid (one CTA per SM, all resident: cooperative launch) runs the steps as
// phases separated by grid barriers:
//   R  router logits: the (router row, hidden chunk, token group) dot products
//      spread over every warp of the grid; partial sums per chunk go to the
//      workspace.                                                  -- barrier
//   S  every CTA adds the chunk partials in chunk order (the same arithmetic
//      order as the router kernels, so logits and routing are bit-identical to
//      moe_route), runs the warp top-K for all tokens and the stable counting
//      sort of the pairs into shared memory.  CTA 0 also writes them out.
//   G  gate/up of every touched expert (and the shared expert) by the
//      weight-streaming GEMV of stream_core.cuh.                   -- barrier
//   D  down, same GEMV, scaled by the routing weights (the shared expert by
//      its gate).                                                  -- barrier
//   C  combine: out[t] = sum_k y_slot[t, k] (+ y_shared[t]) in that order.
//
// The grid barrier is the bounded counter barrier of common.cuh (a 64-bit
// counter per device that grows by 2^32 per completed barrier).  Waits are
// bounded; a CTA that gives up still arrives at the later barriers, so every
// barrier of a launch sees all G arrivals and the counter is consistent for
// the next launch.  The launch asks for more than half of an SM's shared
// memory and checks on the host that one CTA per SM is the most that fits, so
// only one such grid runs on a device at a time and one counter serves all.
#include <atomic>

#include <mutex>

#include "decode_stream.cuh"
#include "route_util.cuh"
#include "stream_core.cuh"

namespace moe {

namespace {

using namespace stream;

constexpr int kTokGroup = 8;  // tokens per router work item
constexpr int kDecodeTok = 4;  // token rows per expert batch in the GEMV phases
constexpr int kMaxRouterRows = 257;
constexpr int kRouterSteps = kRouterChunk / 256;  // 8-element steps of a lane per chunk

__device__ unsigned long long g_decode_barrier;

struct DecodeArgs {
  const void* x;
  const void* router;
  int router_bf16;
  const float* bias;
  const void* w_s;  // shared-gate row (router dtype) or nullptr
  int T, H, E, K, renorm, has_shared;
  RouteCfg rc;
  Phase g, d;       // gate/up and down; pairs and row scales are set in the kernel
  int stage_bytes;  // dynamic shared memory before the pair arrays
  float* parts;     // [nch, T, R] chunk partials of the logits
  float* logits;    // [T, E] biased logits
  int32_t* ids;
  float* w;
  float* shared_gate;
  int32_t* counts;
  int32_t* offsets;
  int32_t* sorted_pairs;
  int32_t* pair_pos;
  const float* y_slots;
  const float* y_s;
  void* out;
  int* status;
  long long wait_limit;
  long long barrier_delay;
  int tma;                 // gate/up and down as one TMA-fed stream (decode_stream.cuh), else the two phases
  dstream::Sync* sync;     // queue and per-group counters of the stream (workspace)
};

// The formats the stream serves: one format for gate/up and down, f32, bf16 or Q8_0 (the k-quant stacks
// keep the two phases).
template <int WKG, int WKD>
__host__ __device__ constexpr bool stream_format() {
  return WKG == WKD && (WKG == WK_F32 || WKG == WK_BF16 || WKG == WK_Q8);
}

__device__ __forceinline__ bool cta_grid_sync(const DecodeArgs& a, int* s_abort, int* s_flag) {
  return grid_sync(&g_decode_barrier, a.wait_limit, a.status, s_abort, s_flag);
}

// Router row r0 + warp's chunk ch into registers (requested whole; zeros past the row or past R).
template <typename WT>
__device__ __forceinline__ void router_load(const DecodeArgs& a, int r0, int ch, int R, Raw8<WT> (&wr)[kRouterSteps]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r = r0 + warp;
  if (r >= R) return;
  const int h0 = ch * kRouterChunk, hc = min(kRouterChunk, a.H - h0);
  const WT* wrow = (r < a.E ? static_cast<const WT*>(a.router) + static_cast<size_t>(r) * a.H
                            : static_cast<const WT*>(a.w_s)) +
                   h0;
#pragma unroll
  for (int u = 0; u < kRouterSteps; ++u)
    if (lane * 8 + 256 * u < hc) raw_load(wrow + lane * 8 + 256 * u, wr[u]);
}

// Partial logits of a block of router rows for one (hidden chunk, token group):
// the CTA has staged the group's x chunk in shared memory as f32 (xs, rows of
// kRouterChunk); warp w takes row r0 + w, whose chunk it loaded into wr (router_load) before the
// staging, so both loads are in flight together.  The chunk arithmetic is that of route_util.cuh.
template <typename WT>
__device__ __forceinline__ void router_rows(const DecodeArgs& a, const float* xs, int r0, int ch, int t0, int nt,
                                            int R, const Raw8<WT> (&wr)[kRouterSteps]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r = r0 + warp;
  if (r >= R) return;
  const int hc = min(kRouterChunk, a.H - ch * kRouterChunk);
  float acc[kTokGroup];
#pragma unroll
  for (int c = 0; c < kTokGroup; ++c) acc[c] = 0.f;
#pragma unroll
  for (int u = 0; u < kRouterSteps; ++u) {
    const int j = lane * 8 + 256 * u;
    if (j < hc) {
      float wv[8];
      raw_decode(wr[u], wv);
#pragma unroll
      for (int c = 0; c < kTokGroup; ++c) {
        if (c < nt) {
          const float4 x0 = *reinterpret_cast<const float4*>(xs + c * kRouterChunk + j);
          const float4 x1 = *reinterpret_cast<const float4*>(xs + c * kRouterChunk + j + 4);
          const float xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
          for (int q = 0; q < 8; ++q) acc[c] = fmaf(wv[q], xv[q], acc[c]);
        }
      }
    }
  }
#pragma unroll
  for (int c = 0; c < kTokGroup; ++c) {
    if (c < nt) {
      const float v = warp_sum(acc[c]);
      if (lane == 0) a.parts[(static_cast<size_t>(ch) * a.T + t0 + c) * R + r] = v;
    }
  }
}

// Stages x[t0 .. t0+nt) [h0 .. h0+hc) as f32 rows of kRouterChunk.  All threads.
template <typename XT>
__device__ __forceinline__ void router_stage_x(const DecodeArgs& a, float* xs, int ch, int t0, int nt) {
  const int h0 = ch * kRouterChunk, hc = min(kRouterChunk, a.H - h0);
  const int g8 = hc / 8;
  for (int i = threadIdx.x; i < nt * g8; i += blockDim.x) {
    const int c = i / g8, q = i - c * g8;
    Raw8<XT> r;
    raw_load(static_cast<const XT*>(a.x) + static_cast<size_t>(t0 + c) * a.H + h0 + 8 * q, r);
    float v[8];
    raw_decode(r, v);
    float4* dst = reinterpret_cast<float4*>(xs + c * kRouterChunk + 8 * q);
    dst[0] = make_float4(v[0], v[1], v[2], v[3]);
    dst[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
}

// One R work item of a CTA: the row block's chunk requested, the x chunk staged (when it differs from the
// one staged last), then the partial logits.  All threads.
template <typename XT, typename WT>
__device__ __forceinline__ void router_item(const DecodeArgs& a, float* xs, int rb, int cg, int ch, int t0, int nt,
                                            int R, int& staged) {
  Raw8<WT> wr[kRouterSteps];
  router_load<WT>(a, rb * kWarps, ch, R, wr);
  if (cg != staged) {
    __syncthreads();
    router_stage_x<XT>(a, xs, ch, t0, nt);
    __syncthreads();
    staged = cg;
  }
  router_rows<WT>(a, xs, rb * kWarps, ch, t0, nt, R, wr);
}

// MAXT: the most tokens of one expert batch (1 when T = 1: only single-token code, more loads in flight).
template <typename XT, int WKG, int WKD, int MAXT>
__global__ void __launch_bounds__(kThreads, 1)
    decode_layer_kernel(const DecodeArgs a, const __grid_constant__ dstream::Maps maps) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int s_expert[kMaxGroups], s_first[kMaxGroups], s_count[kMaxGroups], s_poff[kMaxGroups + 1];
  __shared__ long long s_coff[kMaxGroups + 1];
  __shared__ int s_cnt[256], s_off[257];
  __shared__ float s_sgate[kMaxDecodeT];
  __shared__ Phase s_ph[2];
  __shared__ int s_arow[kMaxTok], s_dest[kMaxTok];
  __shared__ float s_scale[kMaxTok];
  __shared__ float s_part[kMaxUnits * kMaxTok * 2];
  __shared__ int s_warp[8];
  __shared__ int s_n, s_flag, s_abort;
  __shared__ int s_gi[kMaxGroups + 1], s_di[kMaxGroups + 1];
  __shared__ dstream::Ring s_ring;
  __shared__ float s_bias[256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = a.T, E = a.E, K = a.K, P = T * K;
  const int R = E + (a.w_s ? 1 : 0);
  float* s_rows = reinterpret_cast<float*>(smem);  // phase S: one logit row per warp (stage area)
  int32_t* s_ids = reinterpret_cast<int32_t*>(smem + a.stage_bytes);
  float* s_w = reinterpret_cast<float*>(s_ids + P);
  int32_t* s_sorted = reinterpret_cast<int32_t*>(s_w + P);
  int32_t* s_rank = s_sorted + P;
  const Smem sm{smem, s_arow, s_dest, s_scale, s_part};

  if (threadIdx.x == 0) {
    s_abort = 0;
    s_ph[0] = a.g;
    s_ph[1] = a.d;
    s_ph[0].pairs = s_sorted;
    s_ph[1].pairs = s_sorted;
    s_ph[1].src[0].row_scale = s_w;
    s_ph[1].src[1].row_scale = a.w_s ? s_sgate : nullptr;
  }

  if (blockIdx.x == 0 && a.tma)  // the stream's queue and counters start at zero (visible after the barrier)
    for (int i = threadIdx.x; i < 1 + dstream::kMaxGroups; i += blockDim.x) reinterpret_cast<unsigned*>(a.sync)[i] = 0;

  // the stream's tensor maps into the copy engine's descriptor cache while R and S run, by the warp that
  // will issue the copies (only the maps this layer uses)
  if constexpr (stream_format<WKG, WKD>()) {
    using namespace dstream;
    if (a.tma && warp == kCW && lane < M_COUNT) {
      const bool sh = lane == M_SGATE || lane == M_SUP || lane == M_SDOWN || lane == M_HS;
      if (!sh || a.has_shared) {
        prefetch_tensormap(&maps.w[lane]);
        if (WKG == WK_Q8 && lane <= M_SDOWN) prefetch_tensormap(&maps.s[lane]);
      }
    }
  }

  // the routing bias, copied to shared memory while R runs (it is read in S)
  if (a.bias)
    for (int e = threadIdx.x; e < E; e += blockDim.x) cp_async4(&s_bias[e], a.bias + e);

  // ---- R: partial router logits; a CTA item is (hidden chunk, token group, block of kWarps rows).  Token
  // groups are as small as spreads the items over the grid (a warp's work is one row for each token of its
  // group, so fewer tokens per item is a shorter phase), at most kTokGroup tokens.
  {
    const int nch = (a.H + kRouterChunk - 1) / kRouterChunk;
    const int nrb = (R + kWarps - 1) / kWarps;
    const int groups_fit = max(1, static_cast<int>(gridDim.x) / (nch * nrb));
    const int tgs = min(kTokGroup, (T + groups_fit - 1) / groups_fit);
    const int ntg = (T + tgs - 1) / tgs;
    const int items = nch * ntg * nrb;
    float* xs = reinterpret_cast<float*>(smem);
    int staged = -1;
    for (int i = blockIdx.x; i < items; i += gridDim.x) {
      const int rb = i % nrb, cg = i / nrb;  // consecutive items of a CTA share their x chunk when they can
      const int ch = cg % nch, tg = cg / nch;
      const int t0 = tg * tgs, nt = min(tgs, T - t0);
      if (a.router_bf16)
        router_item<XT, __nv_bfloat16>(a, xs, rb, cg, ch, t0, nt, R, staged);
      else
        router_item<XT, float>(a, xs, rb, cg, ch, t0, nt, R, staged);
    }
  }
  cp_async_wait_all();  // the bias copies (long done); the barrier's block sync publishes them
  debug_delay_cta0(a.barrier_delay);
  cta_grid_sync(a, &s_abort, &s_flag);

  // ---- S: logits, top-K and the pair permutation, in every CTA
  {
    const int nch = (a.H + kRouterChunk - 1) / kRouterChunk;
    for (int t = warp; t < T; t += kWarps) {
      float* row = s_rows + warp * kMaxRouterRows;
      float l[9];  // experts lane + 32 i; chunk partials requested together, added in chunk order
#pragma unroll
      for (int i = 0; i < 9; ++i) l[i] = 0.f;
      for (int ch0 = 0; ch0 < nch; ch0 += 4) {
        float v[4][9];
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int i = 0; i < 9; ++i)
            v[j][i] = (ch0 + j < nch && lane + 32 * i < R)
                          ? __ldcg(a.parts + (static_cast<size_t>(ch0 + j) * T + t) * R + lane + 32 * i)
                          : 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int i = 0; i < 9; ++i)
            if (ch0 + j < nch) l[i] += v[j][i];
      }
#pragma unroll
      for (int i = 0; i < 9; ++i)
        if (lane + 32 * i < R) row[lane + 32 * i] = l[i];
      __syncwarp();
      float* lout = blockIdx.x == 0 ? a.logits + static_cast<size_t>(t) * E : row;
      warp_topk(row, a.bias ? s_bias : nullptr, a.rc, lout, s_ids + t * K, s_w + t * K);
      if (a.w_s && lane == 0) {
        const float sg = 1.0f / (1.0f + expf(-row[E]));
        s_sgate[t] = sg;
        if (blockIdx.x == 0) a.shared_gate[t] = sg;
      }
      __syncwarp();
    }
    __syncthreads();
    if (warp == 0) {  // stable counting sort: ranks within each expert in pair order
      for (int e = lane; e < E; e += 32) s_cnt[e] = 0;
      __syncwarp();
      for (int base = 0; base < P; base += 32) {
        const int p = base + lane;
        const int e = p < P ? s_ids[p] : -1;
        const unsigned m = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(m & ((1u << lane) - 1u));
        const int before = p < P ? s_cnt[e] : 0;
        __syncwarp();
        if (p < P) {
          s_rank[p] = before + rank;
          if (rank == 0) s_cnt[e] = before + __popc(m);
        }
        __syncwarp();
      }
      int loc[8], sum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = lane * 8 + i;
        loc[i] = e < E ? s_cnt[e] : 0;
        sum += loc[i];
      }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      int run = incl - sum;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = lane * 8 + i;
        if (e < E) s_off[e] = run;
        run += loc[i];
      }
      if (lane == 31) s_off[E] = incl;
    }
    __syncthreads();
    for (int p = threadIdx.x; p < P; p += blockDim.x) {
      const int pos = s_off[s_ids[p]] + s_rank[p];
      s_sorted[pos] = p;
      if (blockIdx.x == 0) {
        a.pair_pos[p] = pos;
        a.sorted_pairs[pos] = p;
        a.ids[p] = s_ids[p];
        a.w[p] = s_w[p];
      }
    }
    if (blockIdx.x == 0)
      for (int e = threadIdx.x; e <= E; e += blockDim.x) {
        a.offsets[e] = s_off[e];
        if (e < E) a.counts[e] = s_cnt[e];
      }
    // groups: touched experts in order, then the shared expert
    if (threadIdx.x < 256) {
      const int e = threadIdx.x;
      const bool f = e < E && s_cnt[e] > 0;
      const unsigned bal = __ballot_sync(0xffffffffu, f);
      if (lane == 0) s_warp[warp] = __popc(bal);
      asm volatile("bar.sync 1, 256;" ::: "memory");
      int base = 0, n = 0;
      for (int w = 0; w < 8; ++w) {
        if (w < warp) base += s_warp[w];
        n += s_warp[w];
      }
      if (f) {
        const int i = base + __popc(bal & ((1u << lane) - 1u));
        s_expert[i] = e;
        s_first[i] = s_off[e];
        s_count[i] = s_cnt[e];
      }
      if (threadIdx.x == 0) {
        if (a.has_shared) {
          s_expert[n] = -1;
          s_first[n] = 0;
          s_count[n] = T;
          ++n;
        }
        s_n = n;
      }
    }
    __syncthreads();
  }

  bool ok;
  bool streamed = false;
  if constexpr (stream_format<WKG, WKD>()) {
    if (a.tma) {
      // ---- G + D as one stream of items (decode_stream.cuh); then one barrier before the combine
      constexpr int NT = dstream::item_tokens(MAXT);
      dstream::Params dp;
      dp.H = a.H;
      dp.K = a.K;
      dp.I = a.g.plan[0].Nout;
      dp.Is = a.has_shared ? a.g.plan[1].Nout : 0;
      dp.act = a.g.act_fn;
      dp.h = a.g.src[0].out;
      dp.h_s = a.g.src[1].out;
      dp.y_slots = a.d.src[0].out;
      dp.y_s = a.d.src[1].out;
      dp.sync = a.sync;
      dp.wait_limit = a.wait_limit;
      dp.status = a.status;
      if (warp == 0) dstream::build_items<NT>(dp, s_expert, s_count, s_n, s_gi, s_di);
      __syncthreads();
      const dstream::Items its{s_expert, s_first, s_count, s_gi, s_di, s_n};
      if (!s_abort) {
        uint8_t* stages = smem + ((128u - (smem_addr(smem) & 127u)) & 127u);  // copy destinations: 128-aligned
        const bool c_ok = dstream::run_stream<XT, WKG, NT>(maps, dp, its, stages, s_ring, s_sorted, s_w,
                                                          a.w_s ? s_sgate : nullptr);
        if (!c_ok) s_abort = 1;
      }
      ok = cta_grid_sync(a, &s_abort, &s_flag);
      streamed = true;
    }
  }
  if (!streamed) {
    // ---- G: gate/up
    {
      const Tables tb{s_expert, s_first, s_count, s_poff, s_coff, s_n};
      if (warp == 0) build_prefix(tb, s_ph[0]);
      __syncthreads();
      int p0, p1;
      cta_pairs(tb, s_ph[0], p0, p1);
      if (!s_abort) run_phase<XT, WKG, true, MAXT>(s_ph[0], tb, p0, p1, sm);
    }
    cta_grid_sync(a, &s_abort, &s_flag);

    // ---- D: down
    {
      const Tables tb{s_expert, s_first, s_count, s_poff, s_coff, s_n};
      if (warp == 0) build_prefix(tb, s_ph[1]);
      __syncthreads();
      int p0, p1;
      cta_pairs(tb, s_ph[1], p0, p1);
      if (!s_abort) run_phase<float, WKD, false, MAXT>(s_ph[1], tb, p0, p1, sm);
    }
    ok = cta_grid_sync(a, &s_abort, &s_flag);
  }

  // ---- C: combine.  A warp takes 32 consecutive float4 of the output (the warps of the grid in turn, CTA
  // first, so a small batch spreads over many SMs); each lane asks for its first kCombineK slot rows (and the
  // shared expert's row) at once, then adds them in k order.
  if (ok) {
    constexpr int kCombineK = 8;
    const int H4 = a.H / 4;
    const long long total = static_cast<long long>(T) * H4;
    const long long nchunk = (total + 31) / 32;
    const float4* ys = reinterpret_cast<const float4*>(a.y_slots);
    const float4* sh = reinterpret_cast<const float4*>(a.y_s);
    for (long long u = blockIdx.x + static_cast<long long>(gridDim.x) * warp; u < nchunk;
         u += static_cast<long long>(gridDim.x) * kWarps) {
      const long long idx = u * 32 + lane;
      if (idx >= total) continue;
      const long long t = idx / H4;
      const int c = static_cast<int>(idx - t * H4);
      const float4* yt = ys + (t * K) * H4 + c;
      float4 v[kCombineK];
#pragma unroll
      for (int k = 0; k < kCombineK; ++k)
        if (k < K) v[k] = __ldcg(yt + k * H4);
      const float4 vs = a.has_shared ? __ldcg(sh + t * H4 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
      float4 acc = v[0];
#pragma unroll
      for (int k = 1; k < kCombineK; ++k)
        if (k < K) {
          acc.x += v[k].x;
          acc.y += v[k].y;
          acc.z += v[k].z;
          acc.w += v[k].w;
        }
      for (int k = kCombineK; k < K; ++k) {
        const float4 w = __ldcg(yt + k * H4);
        acc.x += w.x;
        acc.y += w.y;
        acc.z += w.z;
        acc.w += w.w;
      }
      if (a.has_shared) {
        acc.x += vs.x;
        acc.y += vs.y;
        acc.z += vs.z;
        acc.w += vs.w;
      }
      if constexpr (sizeof(XT) == 4) {
        reinterpret_cast<float4*>(a.out)[idx] = acc;
      } else {
        const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
        uint2 pk;
        pk.x = *reinterpret_cast<const uint32_t*>(&lo);
        pk.y = *reinterpret_cast<const uint32_t*>(&hi);
        reinterpret_cast<uint2*>(a.out)[idx] = pk;
      }
    }
  }
  if (threadIdx.x == 0 && s_abort) record_status(a.status, MOE_ERR_TIMEOUT);
}

// Static shared memory of a kernel instance (queried once).
template <typename XT, int WKG, int WKD, int MAXT>
int static_smem() {
  static std::atomic<int> bytes{-1};
  int b = bytes.load();
  if (b < 0) {
    cudaFuncAttributes fa{};
    if (cudaFuncGetAttributes(&fa, decode_layer_kernel<XT, WKG, WKD, MAXT>) != cudaSuccess) return -1;
    b = static_cast<int>(fa.sharedSizeBytes);
    bytes.store(b);
  }
  return b;
}

template <typename XT, int WKG, int WKD, int MAXT>
cudaError_t launch_fused_t(const Ctx& c, const DecodeArgs& a0, int P, const dstream::Maps& maps) {
  auto kern = decode_layer_kernel<XT, WKG, WKD, MAXT>;
  DecodeArgs a = a0;
  if (!stream_format<WKG, WKD>()) a.tma = 0;
  const int st = static_smem<XT, WKG, WKD, MAXT>();
  // the stream's ring reuses the stage area (the two phases take over if it does not fit)
  const int ring = dstream::ring_bytes(WKG) + 128;
  if (a.tma && std::max(a.stage_bytes, ring) + 16 * P + st > c.smem_optin) a.tma = 0;
  if (a.tma) a.stage_bytes = std::max(a.stage_bytes, ring);
  // more than half of an SM's shared memory, so one CTA per SM whatever the register count: a CTA of a later
  // grid then starts only after this grid's last barrier (the barrier counter is shared by all launches)
  const int smem = std::max(a.stage_bytes + 16 * P, c.smem_optin / 2 + 1024);
  if (st < 0 || smem + st > c.smem_optin) return cudaErrorInvalidValue;
  cudaError_t e = allow_dynamic_smem(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm != 1) return cudaErrorInvalidValue;  // the step-by-step launches run instead
  KernelScope ks(c, "decode_layer");
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(c.num_sms);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = c.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a, maps);
}

template <typename XT, int WKG, int WKD>
cudaError_t launch_fused(const Ctx& c, const DecodeArgs& a, int P, const dstream::Maps& maps) {
  if (a.T == 1) return launch_fused_t<XT, WKG, WKD, 1>(c, a, P, maps);
  return launch_fused_t<XT, WKG, WKD, kDecodeTok>(c, a, P, maps);
}

template <typename XT>
cudaError_t launch_kinds(const Ctx& c, const DecodeArgs& a, int P, int wkg, int wkd, const dstream::Maps& maps) {
  if (wkg == WK_F32) return launch_fused<XT, WK_F32, WK_F32>(c, a, P, maps);
  if (wkg == WK_BF16) return launch_fused<XT, WK_BF16, WK_BF16>(c, a, P, maps);
  if (wkg == WK_Q8) return launch_fused<XT, WK_Q8, WK_Q8>(c, a, P, maps);
  if (wkd == WK_Q6K) return launch_fused<XT, WK_Q4K, WK_Q6K>(c, a, P, maps);
  return launch_fused<XT, WK_Q4K, WK_Q4K>(c, a, P, maps);
}

cudaError_t launch_by_kind(const Ctx& c, const DecodeArgs& a, int P, bool x_f32, int wkg, int wkd,
                           const dstream::Maps& maps) {
  return x_f32 ? launch_kinds<float>(c, a, P, wkg, wkd, maps) : launch_kinds<__nv_bfloat16>(c, a, P, wkg, wkd, maps);
}

// ---- tensor maps of the stream, encoded once per (tensor, shape) and kept
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

struct MapKey {
  const void* base;
  int dtype;
  uint64_t rows, cols;
  uint32_t box_rows;
  int dev;
  bool operator==(const MapKey& o) const {
    return base == o.base && dtype == o.dtype && rows == o.rows && cols == o.cols && box_rows == o.box_rows &&
           dev == o.dev;
  }
};

// A row-major matrix [rows, cols] of `dtype` elements read in boxes of box_cols x box_rows
// (zero fill past the edges).  The last few maps are kept, keyed by pointer, shape and box.
bool stream_map(CUtensorMap* m, const void* base, CUtensorMapDataType dtype, int esize, uint64_t rows, uint64_t cols,
                uint32_t box_cols, uint32_t box_rows) {
  constexpr int kCache = 64;
  static std::mutex mu;
  static MapKey keys[kCache];
  static CUtensorMap vals[kCache];
  static int used = 0, next = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  const MapKey key{base, static_cast<int>(dtype), rows, cols, box_cols * 1024u + box_rows, dev};
  {
    std::lock_guard<std::mutex> lk(mu);
    for (int i = 0; i < used; ++i)
      if (keys[i] == key) {
        *m = vals[i];
        return true;
      }
  }
  EncodeTiledFn enc = encode_fn();
  if (!enc || (reinterpret_cast<uintptr_t>(base) & 15u) || (cols * esize) % 16) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * esize};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(m, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
      CUDA_SUCCESS)
    return false;
  std::lock_guard<std::mutex> lk(mu);
  keys[next] = key;
  vals[next] = *m;
  next = (next + 1) % kCache;
  used = std::max(used, next == 0 ? kCache : next);
  return true;
}

// The map of one weight matrix [rows, K] for the stream, in boxes of 256 elements (Q8_0: 256 32-bit words
// of codes) x box_rows, and for Q8_0 the map of its fp16 scale plane [rows, K / 32] in boxes of 32 x box_rows;
// false if the layout does not fit (misaligned pointer, K not whole 256-code units for Q8_0).
bool weight_map(int wk, const void* w, const void* scale, uint64_t rows, uint64_t K, uint32_t box_rows,
                CUtensorMap* mw, CUtensorMap* ms) {
  if (wk == WK_F32) return stream_map(mw, w, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, rows, K, 256, box_rows);
  if (wk == WK_BF16) return stream_map(mw, w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows, K, 256, box_rows);
  if (K % 256) return false;
  return stream_map(mw, w, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, rows, K / 4, 256, box_rows) &&
         stream_map(ms, scale, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, rows, K / 32, 32, box_rows);
}

}  // namespace

size_t decode_router_parts_floats(int T, int H, int E, bool shared_gate) {
  const size_t nch = (static_cast<size_t>(H) + kRouterChunk - 1) / kRouterChunk;
  return nch * T * (E + (shared_gate ? 1 : 0));
}

cudaError_t launch_decode_layer(const Ctx& c, const DecodeLayer& L) {
  if (L.T <= 0) return cudaSuccess;
  const int P = L.T * L.K;
  if (L.T > kMaxDecodeT || P > kMaxDecodePairs || L.E > 256 || (L.H % 4)) return cudaErrorInvalidValue;
  const int wkg = wk_gate_up(L.w_dtype), wkd = wk_down(L.w_dtype);
  const int ab = L.x_dtype == MOE_F32 ? 4 : 2;
  DecodeArgs a{};
  // gate/up: routed experts read x rows through the pair list, the shared expert reads x row r
  a.g.plan[0] = make_plan(wkg, true, L.H, L.I, ab, L.T, kDecodeTok);
  a.g.plan[1] = L.Is > 0 ? make_plan(wkg, true, L.H, L.Is, ab, L.T, kDecodeTok) : a.g.plan[0];
  a.d.plan[0] = make_plan(wkd, false, L.I, L.H, 4, L.T, kDecodeTok);
  a.d.plan[1] = L.Is > 0 ? make_plan(wkd, false, L.Is, L.H, 4, L.T, kDecodeTok) : a.d.plan[0];
  // phases R and S use the stage area for an f32 x chunk of a token group and one logit row per warp
  int stage = std::max(kTokGroup * kRouterChunk * 4, kWarps * kMaxRouterRows * 4);
  for (const Plan* p : {&a.g.plan[0], &a.g.plan[1], &a.d.plan[0], &a.d.plan[1]}) {
    if (p->xrow_bytes > kMaxTokenRowBytes) return cudaErrorInvalidValue;
    stage = std::max(stage, p->TS * p->xrow_bytes);
  }
  a.stage_bytes = (stage + 127) / 128 * 128;
  a.x = L.x;
  a.router = L.router;
  a.router_bf16 = L.router_dtype == MOE_BF16;
  a.bias = L.bias;
  a.w_s = L.w_s;
  a.T = L.T;
  a.H = L.H;
  a.E = L.E;
  a.K = L.K;
  a.renorm = L.renorm;
  a.rc = L.rc;
  a.has_shared = L.Is > 0;
  a.g.K = L.K;
  a.g.act_fn = L.act;
  GroupSrc& gr = a.g.src[0];
  gr.w0 = static_cast<const uint8_t*>(L.gate);
  gr.w1 = static_cast<const uint8_t*>(L.up);
  gr.s0 = static_cast<const uint8_t*>(L.gate_scale);
  gr.s1 = static_cast<const uint8_t*>(L.up_scale);
  gr.act = static_cast<const uint8_t*>(L.x);
  gr.out = L.h;
  gr.act_via_pairs = 1;
  GroupSrc& gs = a.g.src[1];
  gs.w0 = static_cast<const uint8_t*>(L.sh_gate);
  gs.w1 = static_cast<const uint8_t*>(L.sh_up);
  gs.s0 = static_cast<const uint8_t*>(L.sh_gate_scale);
  gs.s1 = static_cast<const uint8_t*>(L.sh_up_scale);
  gs.act = static_cast<const uint8_t*>(L.x);
  gs.out = L.h_s;
  // down: routed rows go to their pair's slot scaled by its weight; the shared expert by its gate
  a.d.K = 1;
  GroupSrc& dr = a.d.src[0];
  dr.w0 = static_cast<const uint8_t*>(L.down);
  dr.s0 = static_cast<const uint8_t*>(L.down_scale);
  dr.act = reinterpret_cast<const uint8_t*>(L.h);
  dr.out = L.y_slots;
  dr.out_via_pairs = 1;
  dr.scale_via_pairs = 1;
  GroupSrc& ds = a.d.src[1];
  ds.w0 = static_cast<const uint8_t*>(L.sh_down);
  ds.s0 = static_cast<const uint8_t*>(L.sh_down_scale);
  ds.act = reinterpret_cast<const uint8_t*>(L.h_s);
  ds.out = L.y_s;
  a.parts = L.router_parts;
  a.logits = L.logits;
  a.ids = L.ids;
  a.w = L.w;
  a.shared_gate = L.shared_gate;
  a.counts = L.counts;
  a.offsets = L.offsets;
  a.sorted_pairs = L.sorted_pairs;
  a.pair_pos = L.pair_pos;
  a.y_slots = L.y_slots;
  a.y_s = L.y_s;
  a.out = L.out;
  a.status = c.status;
  a.wait_limit = c.wait_limit;
  a.barrier_delay = c.barrier_delay;
  // gate/up and down as one TMA-fed stream: f32 or bf16 in both projections, every matrix mappable
  dstream::Maps maps;
  memset(&maps, 0, sizeof(maps));
  a.sync = static_cast<dstream::Sync*>(L.stream_sync);
  const int sw = stream_path_mode();
  a.tma = L.stream_sync != nullptr && wkg == wkd && (wkg == WK_F32 || wkg == WK_BF16 || wkg == WK_Q8);
  if (a.tma) {
    using namespace dstream;
    const uint64_t E = L.E, H = L.H, I = L.I, Is = L.Is;
    constexpr uint32_t GR = kRows / 2, DR = kRows;  // boxes of 16 gate (or up) rows, 32 down rows
    bool ok = weight_map(wkg, L.gate, L.gate_scale, E * I, H, GR, &maps.w[M_GATE], &maps.s[M_GATE]) &&
              weight_map(wkg, L.up, L.up_scale, E * I, H, GR, &maps.w[M_UP], &maps.s[M_UP]) &&
              weight_map(wkd, L.down, L.down_scale, E * H, I, DR, &maps.w[M_DOWN], &maps.s[M_DOWN]);
    if (ok && Is > 0)
      ok = weight_map(wkg, L.sh_gate, L.sh_gate_scale, Is, H, GR, &maps.w[M_SGATE], &maps.s[M_SGATE]) &&
           weight_map(wkg, L.sh_up, L.sh_up_scale, Is, H, GR, &maps.w[M_SUP], &maps.s[M_SUP]) &&
           weight_map(wkd, L.sh_down, L.sh_down_scale, H, Is, DR, &maps.w[M_SDOWN], &maps.s[M_SDOWN]);
    const uint64_t T = L.T, P = T * L.K;
    const bool xf = L.x_dtype == MOE_F32;
    const CUtensorMapDataType xdt = xf ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const int xes = xf ? 4 : 2;
    if (wkg == WK_Q8) {
      // activations as rows of 256 values, four of them (one token's 1024 values) per box
      ok = ok && H % 256 == 0 && I % 256 == 0 && Is % 256 == 0;
      if (ok)
        ok = stream_map(&maps.w[M_X], L.x, xdt, xes, T * H / 256, 256, 256, 4) &&
             stream_map(&maps.w[M_H], L.h, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, P * I / 256, 256, 256, 4);
      if (ok && Is > 0)
        ok = stream_map(&maps.w[M_HS], L.h_s, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, T * Is / 256, 256, 256, 4);
    } else {
      // x in boxes of one row; h and h_s in boxes of the item's tokens (no taller than the matrix), the same
      // kernel instance launch_fused picks for T
      const uint32_t nt = static_cast<uint32_t>(item_tokens(L.T == 1 ? 1 : kDecodeTok));
      maps.h_box = static_cast<int>(std::min<uint64_t>(nt, P));
      maps.hs_box = static_cast<int>(std::min<uint64_t>(nt, T));
      if (ok)
        ok = stream_map(&maps.w[M_X], L.x, xdt, xes, T, H, 256, 1) &&
             stream_map(&maps.w[M_H], L.h, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, P, I, 256, maps.h_box);
      if (ok && Is > 0)
        ok = stream_map(&maps.w[M_HS], L.h_s, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, T, Is, 256, maps.hs_box);
    }
    a.tma = ok && sw != 0;
  }
  return launch_by_kind(c, a, P, L.x_dtype == MOE_F32, wkg, wkd, maps);
}

}  // namespace moe
