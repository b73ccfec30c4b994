// Router: logits on CUDA cores for the weight-streaming path and the shared
// gate, and the per-token softmax + top-K + renormalisation.
//
// Selection follows hf2q qwen35/gpu_ffn.rs, softmax_topk_renorm_cpu (a full
// stable sort by probability, first K) and the route kernel of ferrum-kernels
// vnext_ops/moe.rs (one 32-thread group per token, E <= 256, K <= 32).  Here a
// warp owns one token: each lane keeps up to 8 logits in registers and K
// rounds of a warp arg-max with a lower-index tie-break produce the K experts
// in (logit desc, index asc) order -- the order the stable sort yields,
// compared on logits (softmax is monotone, so the selection is the same).
#include "kernels.h"

namespace moe {

namespace {

constexpr int kTok = 8;  // tokens per warp item in the logits kernel

__device__ __forceinline__ void load8(const float* __restrict__ p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void load8(const __nv_bfloat16* __restrict__ p, float (&v)[8]) {
  const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
    v[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
  }
}

// One warp per (row, chunk of kTok tokens); rows [row0, row0 + nrows) where
// row E means the shared-gate vector w_s.
template <typename XT, typename WT>
__global__ void __launch_bounds__(256) router_logits_kernel(const XT* __restrict__ x, const WT* __restrict__ W,
                                                            const WT* __restrict__ w_s, int T, int H, int E,
                                                            int row0, int nrows, float* __restrict__ logits,
                                                            float* __restrict__ shared_gate) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nchunks = (T + kTok - 1) / kTok;
  const long long item = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + warp;
  if (item >= static_cast<long long>(nrows) * nchunks) return;
  const int r = row0 + static_cast<int>(item % nrows);
  const int t0 = static_cast<int>(item / nrows) * kTok;
  const int nt = min(kTok, T - t0);
  const WT* wrow = (r < E) ? W + static_cast<size_t>(r) * H : w_s;
  float acc[kTok];
#pragma unroll
  for (int c = 0; c < kTok; ++c) acc[c] = 0.f;
  for (int j = lane * 8; j < H; j += 256) {
    float wv[8];
    load8(wrow + j, wv);
#pragma unroll
    for (int c = 0; c < kTok; ++c) {
      if (c < nt) {
        float xv[8];
        load8(x + static_cast<size_t>(t0 + c) * H + j, xv);
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[c] = fmaf(wv[q], xv[q], acc[c]);
      }
    }
  }
  float mine = 0.f;
#pragma unroll
  for (int c = 0; c < kTok; ++c) {
    const float s = warp_sum(acc[c]);
    if (lane == c) mine = s;
  }
  if (lane < nt) {
    if (r < E)
      logits[static_cast<size_t>(t0 + lane) * E + r] = mine;
    else
      shared_gate[t0 + lane] = 1.0f / (1.0f + expf(-mine));
  }
}

__global__ void __launch_bounds__(256) router_topk_kernel(float* __restrict__ logits, const float* __restrict__ bias,
                                                          int T, int E, int K, int renorm, int32_t* __restrict__ ids,
                                                          float* __restrict__ wout) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + warp;
  if (t >= T) return;
  float* row = logits + static_cast<size_t>(t) * E;
  float v[8];
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    v[i] = -INFINITY;
    if (e < E) {
      float l = row[e];
      if (bias) {
        l += bias[e];
        row[e] = l;
      }
      v[i] = l;
      m = fmaxf(m, l);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));

  uint32_t taken = 0;
  int my_e = 0;
  float my_v = 0.f;
  for (int k = 0; k < K; ++k) {
    float bv = -INFINITY;
    int be = 0x7FFFFFFF;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1u) && (v[i] > bv || (v[i] == bv && e < be))) {
        bv = v[i];
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
    if (lane == k) {
      my_e = be;
      my_v = bv;
    }
  }
  const float ev = (lane < K) ? expf(my_v - m) : 0.f;
  float denom;
  if (renorm) {
    denom = warp_sum(ev);
  } else {
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (lane + 32 * i < E) s += expf(v[i] - m);
    denom = warp_sum(s);
  }
  const float inv = denom > 1e-20f ? 1.0f / denom : (renorm ? 1.0f / K : 1.0f);
  if (lane < K) {
    ids[static_cast<size_t>(t) * K + lane] = my_e;
    wout[static_cast<size_t>(t) * K + lane] = ev * inv;
  }
}

template <typename XT, typename WT>
cudaError_t logits_typed(const Ctx& c, const void* x, const void* W, const void* w_s, int T, int H, int E, int row0,
                         int nrows, float* logits, float* shared_gate) {
  const long long items = static_cast<long long>(nrows) * ((T + kTok - 1) / kTok);
  if (items == 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>((items + 7) / 8);
  KernelScope ks(c, "router_logits");
  router_logits_kernel<XT, WT><<<blocks, 256, 0, c.stream>>>(
      static_cast<const XT*>(x), static_cast<const WT*>(W), static_cast<const WT*>(w_s), T, H, E, row0, nrows,
      logits, shared_gate);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router_logits(const Ctx& c, const void* x, int x_dtype, const void* W, const void* w_s,
                                 int w_dtype, int T, int H, int E, bool rows_from_router, float* logits,
                                 float* shared_gate) {
  const int row0 = rows_from_router ? 0 : E;
  const int nrows = (rows_from_router ? E : 0) + (w_s ? 1 : 0);
  if (x_dtype == MOE_F32 && w_dtype == MOE_F32)
    return logits_typed<float, float>(c, x, W, w_s, T, H, E, row0, nrows, logits, shared_gate);
  if (x_dtype == MOE_F32 && w_dtype == MOE_BF16)
    return logits_typed<float, __nv_bfloat16>(c, x, W, w_s, T, H, E, row0, nrows, logits, shared_gate);
  if (x_dtype == MOE_BF16 && w_dtype == MOE_F32)
    return logits_typed<__nv_bfloat16, float>(c, x, W, w_s, T, H, E, row0, nrows, logits, shared_gate);
  return logits_typed<__nv_bfloat16, __nv_bfloat16>(c, x, W, w_s, T, H, E, row0, nrows, logits, shared_gate);
}

cudaError_t launch_router_topk(const Ctx& c, float* logits, const float* bias, int T, int E, int K, int renorm,
                               int32_t* ids, float* w) {
  if (T == 0) return cudaSuccess;
  KernelScope ks(c, "router_topk");
  router_topk_kernel<<<(T + 7) / 8, 256, 0, c.stream>>>(logits, bias, T, E, K, renorm, ids, w);
  return cudaGetLastError();
}

}  // namespace moe
