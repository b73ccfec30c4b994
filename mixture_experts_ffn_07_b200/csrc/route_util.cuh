// Routing helpers shared by the router kernels (router.cu) and the fused
// decode kernel (decode_fused.cu): raw 8-element loads of x / router rows,
// the chunked order in which a router logit is accumulated, and the warp
// top-K.  Both kernels use exactly this arithmetic order, so for the same
// inputs they produce bit-identical logits and routing.
#pragma once

#include "kernels.h"

namespace moe {
namespace {

// A router logit l[t, e] = sum_h x[t, h] * W_r[e, h] is accumulated in chunks of
// kRouterChunk hidden elements: inside a chunk lane l sums (fmaf, in order)
// the products at h0 + 8*l + 256*u + q for u = 0.. and q = 0..7; the 32 lane
// partials are added by warp_sum; the chunk totals are added in chunk order
// starting from 0.
constexpr int kRouterChunk = 1024;

template <typename T>
struct Raw8;  // 8 elements as raw 16-byte words
template <>
struct Raw8<float> {
  uint4 a, b;
};
template <>
struct Raw8<__nv_bfloat16> {
  uint4 a;
};
__device__ __forceinline__ void raw_load(const float* p, Raw8<float>& r) {
  r.a = __ldg(reinterpret_cast<const uint4*>(p));
  r.b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
}
__device__ __forceinline__ void raw_load(const __nv_bfloat16* p, Raw8<__nv_bfloat16>& r) {
  r.a = __ldg(reinterpret_cast<const uint4*>(p));
}
__device__ __forceinline__ void raw_decode(const Raw8<float>& r, float (&v)[8]) {
  v[0] = __uint_as_float(r.a.x); v[1] = __uint_as_float(r.a.y); v[2] = __uint_as_float(r.a.z);
  v[3] = __uint_as_float(r.a.w); v[4] = __uint_as_float(r.b.x); v[5] = __uint_as_float(r.b.y);
  v[6] = __uint_as_float(r.b.z); v[7] = __uint_as_float(r.b.w);
}
__device__ __forceinline__ void raw_decode(const Raw8<__nv_bfloat16>& r, float (&v)[8]) {
  const uint32_t w[4] = {r.a.x, r.a.y, r.a.z, r.a.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
    v[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
  }
}

// An order-preserving 32-bit key of a non-NaN float (a > b as floats iff key(a) > key(b); -0 and +0 share
// the key of +0; -inf is 0x007FFFFF, so key 0 stays below every value), and the value of a key.
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f == 0.f ? 0.f : f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float order_key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Routing weights of one token, by one warp: lane k < K holds the k-th selected expert my_e and its biased
// logit my_v; v[i] are the lane's biased logits of experts lane + 32 i (NaN as -inf; used by the softmax
// over all E experts), m their maximum.  Softmax or sigmoid gate values, renormalised over the K selected
// when asked; lane k writes ids[k] and wout[k].
__device__ __forceinline__ void warp_weights(int my_e, float my_v, const float (&v)[8], float m, const RouteCfg& rc,
                                             int32_t* __restrict__ ids, float* __restrict__ wout) {
  const int lane = threadIdx.x & 31;
  const int E = rc.E, K = rc.K;
  float ev, denom;
  if (rc.gating == MOE_GATING_SIGMOID) {
    ev = (lane < K) ? 1.0f / (1.0f + expf(-my_v)) : 0.f;
    denom = rc.renorm ? warp_sum(ev) : 1.0f;
  } else {
    ev = (lane < K) ? expf(my_v - m) : 0.f;
    if (rc.renorm) {
      denom = warp_sum(ev);
    } else {
      float s = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (lane + 32 * i < E) s += expf(v[i] - m);
      denom = warp_sum(s);
    }
  }
  const float inv = denom > 1e-20f ? 1.0f / denom : (rc.renorm ? 1.0f / K : 1.0f);
  if (lane < K) {
    ids[lane] = my_e;
    wout[lane] = ev * inv;
  }
}

// Top-K (+ renormalisation) of one token, by one warp, from the lane's biased
// logits v[i] of experts e = lane + 32 i (NaN already mapped to -inf; entries
// beyond E are -inf) and m, their maximum over the warp.  With n_groups > 1 the
// experts form n_groups contiguous groups, a group scores its largest logit,
// and only the topk_groups best groups (lower index on ties) are eligible.
// Weights: softmax gate values over all E experts, or sigmoid gate values;
// renormalised over the K selected when asked.
__device__ __forceinline__ void warp_select(const float (&v)[8], float m, const RouteCfg& rc,
                                            int32_t* __restrict__ ids, float* __restrict__ wout) {
  const int lane = threadIdx.x & 31;
  const int E = rc.E, K = rc.K;
  uint32_t taken = 0;  // bit i: v[i] not eligible (its group is not among the kept ones)
  if (rc.n_groups > 1) {
    const int gs = E / rc.n_groups;
    float my_gs = -INFINITY;  // lane g: score of group g
    for (int g = 0; g < rc.n_groups; ++g) {
      float gm = -INFINITY;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        if (e < E && e / gs == g) gm = fmaxf(gm, v[i]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, o));
      if (lane == g) my_gs = gm;
    }
    uint32_t kept = 0;
    for (int j = 0; j < rc.topk_groups; ++j) {
      float bv = ((kept >> lane) & 1u) || lane >= rc.n_groups ? -INFINITY : my_gs;
      int bg = ((kept >> lane) & 1u) || lane >= rc.n_groups ? 0x7FFFFFFF : lane;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int og = __shfl_xor_sync(0xffffffffu, bg, o);
        if (ov > bv || (ov == bv && og < bg)) {
          bv = ov;
          bg = og;
        }
      }
      kept |= 1u << bg;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((kept >> (e / gs)) & 1u)) taken |= 1u << i;
    }
  }

  // Candidates as order-preserving 32-bit keys (-0 counts as +0, as in a float compare; -inf is 0x007FFFFF)
  // and an ineligible one (past E, or in an excluded group) as key 0, below every expert.  Each lane sorts
  // its eight once (key descending, lower expert first: a strict order, the experts differ), so its best
  // remaining candidate is always its first.  Then K rounds: the largest first key over the warp (one
  // redux); when one lane holds it that lane wins, else the lowest expert among the holders (a second
  // redux, only on equal values); the winner drops its first candidate.  The same selection as a pairwise
  // (value, lower index) maximum.
  uint32_t ck[8];
  int ce[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    ce[i] = lane + 32 * i;
    ck[i] = (ce[i] < E && !((taken >> i) & 1u)) ? order_key(v[i]) : 0u;
  }
  auto cas = [&](int i, int j) {  // the better of candidates i and j to i
    const bool sw = ck[j] > ck[i] || (ck[j] == ck[i] && ce[j] < ce[i]);
    const uint32_t ki = ck[i], kj = ck[j];
    const int ei = ce[i], ej = ce[j];
    ck[i] = sw ? kj : ki;
    ck[j] = sw ? ki : kj;
    ce[i] = sw ? ej : ei;
    ce[j] = sw ? ei : ej;
  };
  // Batcher's odd-even merge sort of 8: 19 compare-exchanges in 6 layers
  cas(0, 2); cas(1, 3); cas(4, 6); cas(5, 7);
  cas(0, 4); cas(1, 5); cas(2, 6); cas(3, 7);
  cas(0, 1); cas(2, 3); cas(4, 5); cas(6, 7);
  cas(2, 4); cas(3, 5);
  cas(1, 4); cas(3, 6);
  cas(1, 2); cas(3, 4); cas(5, 6);
  int my_e = 0;
  float my_v = 0.f;
  for (int k = 0; k < K; ++k) {
    const uint32_t km = __reduce_max_sync(0xffffffffu, ck[0]);
    const unsigned holders = __ballot_sync(0xffffffffu, ck[0] == km);
    int wl;
    if (holders & (holders - 1u))  // equal values in several lanes (uniform branch)
      wl = static_cast<int>(__reduce_min_sync(0xffffffffu, ck[0] == km ? static_cast<uint32_t>(ce[0]) : 0xFFFFFFFFu)) & 31;
    else
      wl = __ffs(holders) - 1;
    const int be = __shfl_sync(0xffffffffu, ce[0], wl);
    if (lane == k) {
      my_e = be;
      my_v = order_key_value(km);
    }
    const bool w = lane == wl;
#pragma unroll
    for (int i = 0; i < 7; ++i) {
      ck[i] = w ? ck[i + 1] : ck[i];
      ce[i] = w ? ce[i + 1] : ce[i];
    }
    ck[7] = w ? 0u : ck[7];
  }
  warp_weights(my_e, my_v, v, m, rc, ids, wout);
}

// warp_select on the E raw logits of `row` (global or shared memory) plus the
// bias; the biased logits go to logits_out (a different array than row).
__device__ __forceinline__ void warp_topk(const float* __restrict__ row, const float* __restrict__ bias,
                                          const RouteCfg& rc, float* __restrict__ logits_out,
                                          int32_t* __restrict__ ids, float* __restrict__ wout) {
  const int lane = threadIdx.x & 31;
  float v[8];
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    v[i] = -INFINITY;
    if (e < rc.E) {
      float l = row[e];
      if (bias) l += bias[e];
      logits_out[e] = l;
      v[i] = l == l ? l : -INFINITY;  // a NaN logit ranks last, so K valid experts are always chosen
      m = fmaxf(m, l);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  warp_select(v, m, rc, ids, wout);
}

// srow[e] = the sum of the `nparts` (<= 16 / EP) split-K partial logits of
// expert e of token t (T*E floats each, `stride` apart), added in part order.
// A lane takes EP of its experts per round, all their parts requested together.
template <int EP>
__device__ __forceinline__ void sum_parts(const float* __restrict__ parts, int nparts, size_t stride, int E, int t,
                                          float* srow) {
  constexpr int KP = 16 / EP;
  const int lane = threadIdx.x & 31;
  const float* src = parts + static_cast<size_t>(t) * E;
  for (int e0 = lane; e0 < E; e0 += 32 * EP) {
    float r[EP][KP];
#pragma unroll
    for (int q = 0; q < EP; ++q)
#pragma unroll
      for (int k = 0; k < KP; ++k)
        r[q][k] = (e0 + 32 * q < E && k < nparts) ? src[e0 + 32 * q + k * stride] : 0.f;
#pragma unroll
    for (int q = 0; q < EP; ++q) {
      if (e0 + 32 * q < E) {
        float sum = r[q][0];
#pragma unroll
        for (int k = 1; k < KP; ++k)
          if (k < nparts) sum += r[q][k];
        srow[e0 + 32 * q] = sum;
      }
    }
  }
}

// Selection for token t by one warp, from logits in global memory: `nparts`
// (<= 16) partial logit arrays of T*E floats, part_stride apart starting at
// `parts`, are added in order into `srow`, the warp's row of E floats in
// shared memory (nparts == 0: logits[t] already holds the sums and is copied
// there); warp_topk then writes the biased logits to logits[t].  With w_s the warp also writes shared_gate[t] = sigmoid(w_s . x[t])
// (lane l accumulates elements 8l + 256u + q in order; warp_sum).
template <typename XT, typename WT>
__device__ __forceinline__ void topk_token(const float* parts, int nparts, size_t part_stride, float* logits,
                                           const float* bias, const RouteCfg& rc, int32_t* ids, float* wout,
                                           const XT* x, const WT* w_s, int H, float* shared_gate, int t,
                                           float* srow) {
  constexpr int kUnroll = 4;
  const int lane = threadIdx.x & 31;
  const int E = rc.E, K = rc.K;
  float* row = logits + static_cast<size_t>(t) * E;
  if (nparts > 0) {
    if (nparts <= 4)
      sum_parts<4>(parts, nparts, part_stride, E, t, srow);
    else if (nparts <= 8)
      sum_parts<2>(parts, nparts, part_stride, E, t, srow);
    else
      sum_parts<1>(parts, nparts, part_stride, E, t, srow);
  } else {
    for (int e = lane; e < E; e += 32) srow[e] = row[e];
  }
  __syncwarp();
  warp_topk(srow, bias, rc, row, ids + static_cast<size_t>(t) * K, wout + static_cast<size_t>(t) * K);
  __syncwarp();
  if (w_s) {
    const XT* xr = x + static_cast<size_t>(t) * H;
    float acc = 0.f;
    for (int base = lane * 8; base < H; base += 256 * kUnroll) {
      Raw8<XT> xv[kUnroll];
      Raw8<WT> wv[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u)
        if (base + 256 * u < H) {
          raw_load(xr + base + 256 * u, xv[u]);
          raw_load(w_s + base + 256 * u, wv[u]);
        }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u)
        if (base + 256 * u < H) {
          float a[8], b[8];
          raw_decode(xv[u], a);
          raw_decode(wv[u], b);
#pragma unroll
          for (int q = 0; q < 8; ++q) acc = fmaf(a[q], b[q], acc);
        }
    }
    acc = warp_sum(acc);
    if (lane == 0) shared_gate[t] = 1.0f / (1.0f + expf(-acc));
  }
}

}  // namespace
}  // namespace moe
