// Router: logits, softmax, top-K and renormalisation.
//
// Selection follows hf2q qwen35/gpu_ffn.rs, softmax_topk_renorm_cpu (a full
// stable sort by probability, first K) and the route kernel of ferrum-kernels
// vnext_ops/moe.rs (one 32-thread group per token, E <= 256, K <= 32).  Here a
// warp owns one token: each lane keeps up to 8 logits in registers and K
// rounds of a warp arg-max with a lower-index tie-break produce the K experts
// in (logit desc, index asc) order -- the order the stable sort yields,
// compared on logits (softmax is monotone, so the selection is the same).
//
// Two ways to get the logits:
//  * router_cluster_kernel (small batches, any dtype): a cluster of 8 CTAs
//    owns 16 tokens; each CTA computes the dot products of one eighth of the
//    router rows on CUDA cores and writes them straight into the leader CTA's
//    shared memory (distributed shared memory); after a cluster barrier the
//    leader's warps run the top-K.  One launch for the whole router.
//  * the tensor-core grouped GEMM (bf16, large batches) writes f32 logits and
//    router_topk_kernel selects from them, computing the shared-gate dot
//    product of its token on the way when there is one.
#include <cooperative_groups.h>

#include "route_util.cuh"

namespace cg = cooperative_groups;

namespace moe {

namespace {

constexpr int kCluster = 8;   // CTAs per cluster in router_cluster_kernel
constexpr int kClusterTok = 16;
constexpr int kMaxRows = 257; // E <= 256 router rows + the shared-gate row

// Loads 8 consecutive x values from shared memory as f32.
__device__ __forceinline__ void smem8(const float* p, float (&v)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// acc[c] += W[row, h0 + j] . xs[c, j] for j in [0, hc) and tokens c < nt, where xs
// is the token block staged in shared memory (row stride `ld`).  The weight
// chunks of a lane (up to kRowUnroll x 8 elements) are all requested before any
// is used, so a row costs one or two memory round trips instead of one per chunk.
constexpr int kRowUnroll = 8;
template <int NT, typename XT, typename WT>
__device__ __forceinline__ void row_dots_smem(const WT* __restrict__ wrow, const XT* xs, int ld, int hc, int nt,
                                              float (&acc)[NT]) {
  const int lane = threadIdx.x & 31;
  for (int base = lane * 8; base < hc; base += 256 * kRowUnroll) {
    Raw8<WT> w[kRowUnroll];
#pragma unroll
    for (int u = 0; u < kRowUnroll; ++u)
      if (base + 256 * u < hc) raw_load(wrow + base + 256 * u, w[u]);
#pragma unroll
    for (int u = 0; u < kRowUnroll; ++u) {
      const int j = base + 256 * u;
      if (j < hc) {
        float wv[8];
        raw_decode(w[u], wv);
#pragma unroll
        for (int c = 0; c < NT; ++c) {
          if (c < nt) {
            float xv[8];
            smem8(xs + c * ld + j, xv);
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[c] = fmaf(wv[q], xv[q], acc[c]);
          }
        }
      }
    }
  }
}

constexpr int kStageBytes = 64 * 1024;  // x staging per chunk of the hidden dimension
static_assert(kStageBytes / (kClusterTok * 4) == kRouterChunk, "router chunking must match route_util.cuh");

template <typename XT, typename WT>
__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(256)
    router_cluster_kernel(const XT* __restrict__ x, const WT* __restrict__ W, const WT* __restrict__ w_s,
                          const float* __restrict__ bias, int T, int H, const RouteCfg rc,
                          float* __restrict__ logits, int32_t* __restrict__ ids, float* __restrict__ wout,
                          float* __restrict__ shared_gate) {
  const int E = rc.E, K = rc.K;
  constexpr int kHc = kStageBytes / (kClusterTok * 4);                // hidden elements per chunk (f32 staging)
  constexpr int kRowsPerCta = (kMaxRows + kCluster - 1) / kCluster;  // 33
  extern __shared__ __align__(16) uint8_t x_stage_raw[];
  float* xs = reinterpret_cast<float*>(x_stage_raw);  // token rows widened to f32 once, read by every router row
  __shared__ float s_logits[kClusterTok * kMaxRows];
  __shared__ float s_part[kClusterTok * kRowsPerCta];
  cg::cluster_group cluster = cg::this_cluster();
  const unsigned rank = cluster.block_rank();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_trigger();
  cluster.sync();  // every CTA of the cluster is running before shared memory is written remotely
  pdl_wait();
  const int t0 = (blockIdx.x / kCluster) * kClusterTok;
  const int nt = min(kClusterTok, T - t0);
  const int R = E + (w_s ? 1 : 0);
  const int rpc = (R + kCluster - 1) / kCluster;
  const int r_begin = rank * rpc, r_end = min(R, r_begin + rpc);
  for (int i = threadIdx.x; i < kClusterTok * kRowsPerCta; i += blockDim.x) s_part[i] = 0.f;
  for (int h0 = 0; h0 < H; h0 += kHc) {
    const int hc = min(kHc, H - h0);
    __syncthreads();  // previous chunk consumed
    const int opr = hc / 8;  // 8-element groups per staged row
    for (int i = threadIdx.x; i < nt * opr; i += blockDim.x) {
      const int c = i / opr, q = i - c * opr;
      Raw8<XT> r;
      raw_load(x + static_cast<size_t>(t0 + c) * H + h0 + 8 * q, r);
      float v[8];
      raw_decode(r, v);
      float4* dst = reinterpret_cast<float4*>(xs + c * kHc + 8 * q);
      dst[0] = make_float4(v[0], v[1], v[2], v[3]);
      dst[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
    __syncthreads();
    for (int r = r_begin + warp; r < r_end; r += 8) {
      const WT* wrow = ((r < E) ? W + static_cast<size_t>(r) * H : w_s) + h0;
      float acc[kClusterTok];
#pragma unroll
      for (int c = 0; c < kClusterTok; ++c) acc[c] = 0.f;
      row_dots_smem<kClusterTok>(wrow, xs, kHc, hc, nt, acc);
#pragma unroll
      for (int c = 0; c < kClusterTok; ++c) {
        const float v = warp_sum(acc[c]);
        if (lane == c) s_part[c * kRowsPerCta + (r - r_begin)] += v;
      }
    }
  }
  __syncwarp();
  float* lead = cluster.map_shared_rank(s_logits, 0);
  for (int r = r_begin + warp; r < r_end; r += 8)
    if (lane < nt) lead[lane * kMaxRows + r] = s_part[lane * kRowsPerCta + (r - r_begin)];
  cluster.sync();  // remote writes into the leader's shared memory are complete and visible
  if (rank != 0) return;
  for (int tt = warp; tt < nt; tt += 8) {
    const size_t t = static_cast<size_t>(t0 + tt);
    warp_topk(s_logits + tt * kMaxRows, bias, rc, logits + t * E, ids + t * K, wout + t * K);
    if (w_s && lane == 0) shared_gate[t] = 1.0f / (1.0f + expf(-s_logits[tt * kMaxRows + E]));
  }
}

// Top-K from logits in global memory (the tensor-core router), one warp per
// token.  The GEMM may leave the logits as `nparts` partial sums over ranges of
// the hidden dimension; they are added in range order (a fixed order, so the
// result is deterministic) into `logits` before selection.  With w_s the warp
// also computes the shared gate sigmoid(w_s . x[t]).
template <typename XT, typename WT>
__global__ void __launch_bounds__(256) router_topk_kernel(const float* __restrict__ parts, int nparts,
                                                          size_t part_stride, float* __restrict__ logits,
                                                          const float* __restrict__ bias, int T,
                                                          const RouteCfg rc, int32_t* __restrict__ ids,
                                                          float* __restrict__ wout, const XT* __restrict__ x,
                                                          const WT* __restrict__ w_s, int H,
                                                          float* __restrict__ shared_gate) {
  __shared__ float s_row[8][256];  // one logit row per warp
  const int warp = threadIdx.x >> 5;
  pdl_trigger();
  pdl_wait();
  const int t = blockIdx.x * (blockDim.x >> 5) + warp;
  if (t >= T) return;
  topk_token(parts, nparts, part_stride, logits, bias, rc, ids, wout, x, w_s, H, shared_gate, t, s_row[warp]);
}

template <typename XT, typename WT>
cudaError_t cluster_typed(const Ctx& c, const void* x, const void* W, const void* w_s, const float* bias, int T,
                          int H, const RouteCfg& rc, float* logits, int32_t* ids, float* w,
                          float* shared_gate) {
  const int clusters = (T + kClusterTok - 1) / kClusterTok;
  const cudaError_t e =
      allow_dynamic_smem(reinterpret_cast<const void*>(router_cluster_kernel<XT, WT>), kStageBytes);
  if (e != cudaSuccess) return e;
  KernelScope ks(c, "router_fused");
  return launch_kernel(c, router_cluster_kernel<XT, WT>, dim3(clusters * kCluster), dim3(256), kStageBytes,
                       static_cast<const XT*>(x), static_cast<const WT*>(W), static_cast<const WT*>(w_s), bias, T,
                       H, rc, logits, ids, w, shared_gate);
}

}  // namespace

template <typename XT, typename WT>
cudaError_t topk_typed(const Ctx& c, const float* parts, int nparts, size_t part_stride, float* logits,
                       const float* bias, int T, const RouteCfg& rc, int32_t* ids, float* w, const void* x,
                       const void* w_s, int H, float* shared_gate) {
  KernelScope ks(c, "router_topk");
  return launch_kernel(c, router_topk_kernel<XT, WT>, dim3((T + 7) / 8), dim3(256), 0, parts, nparts, part_stride,
                       logits, bias, T, rc, ids, w, static_cast<const XT*>(x), static_cast<const WT*>(w_s),
                       H, shared_gate);
}

cudaError_t launch_router_topk(const Ctx& c, const float* parts, int nparts, size_t part_stride, float* logits,
                               const float* bias, int T, const RouteCfg& rc, int32_t* ids, float* w,
                               const void* x, int x_dtype, const void* w_s, int w_dtype, int H, float* shared_gate) {
  if (T == 0) return cudaSuccess;
  if (x_dtype == MOE_F32 && w_dtype == MOE_F32)
    return topk_typed<float, float>(c, parts, nparts, part_stride, logits, bias, T, rc, ids, w, x, w_s, H,
                                    shared_gate);
  if (x_dtype == MOE_F32 && w_dtype == MOE_BF16)
    return topk_typed<float, __nv_bfloat16>(c, parts, nparts, part_stride, logits, bias, T, rc, ids, w, x,
                                            w_s, H, shared_gate);
  if (x_dtype == MOE_BF16 && w_dtype == MOE_F32)
    return topk_typed<__nv_bfloat16, float>(c, parts, nparts, part_stride, logits, bias, T, rc, ids, w, x,
                                            w_s, H, shared_gate);
  return topk_typed<__nv_bfloat16, __nv_bfloat16>(c, parts, nparts, part_stride, logits, bias, T, rc, ids,
                                                  w, x, w_s, H, shared_gate);
}

cudaError_t launch_router_fused(const Ctx& c, const void* x, int x_dtype, const void* W, const void* w_s,
                                int w_dtype, const float* bias, int T, int H, const RouteCfg& rc,
                                float* logits, int32_t* ids, float* w, float* shared_gate) {
  if (T == 0) return cudaSuccess;
  if (x_dtype == MOE_F32 && w_dtype == MOE_F32)
    return cluster_typed<float, float>(c, x, W, w_s, bias, T, H, rc, logits, ids, w, shared_gate);
  if (x_dtype == MOE_F32 && w_dtype == MOE_BF16)
    return cluster_typed<float, __nv_bfloat16>(c, x, W, w_s, bias, T, H, rc, logits, ids, w,
                                               shared_gate);
  if (x_dtype == MOE_BF16 && w_dtype == MOE_F32)
    return cluster_typed<__nv_bfloat16, float>(c, x, W, w_s, bias, T, H, rc, logits, ids, w,
                                               shared_gate);
  return cluster_typed<__nv_bfloat16, __nv_bfloat16>(c, x, W, w_s, bias, T, H, rc, logits, ids, w,
                                                     shared_gate);
}

}  // namespace moe
