// Weight-streaming expert FFN for small batches (T <= 64) and non-bf16
// formats, the weighted combine, and the Q8_0 block split.
//
// Decode is bound by reading expert weights from HBM (hf2q qwen35/gpu_ffn.rs:
// mat-vec beats tiled mat-mat at one row; DS4Server qwen_mtplx.rs,
// fused_experts: moe_glu_h then moe_down_y).  The kernels here are
// expert-major: a warp takes one output row of one touched expert and streams
// that weight row once with 16-byte loads per lane, computing the dot product
// for every token routed to the expert (up to 8 at a time from registers),
// then reduces across the warp with shuffles.  Q8_0 weights are dequantised in
// registers (value = fp16 scale * int8) and never widened in memory.
#include "kernels.h"

namespace moe {

namespace {

constexpr int kRows = 8;    // tokens (rows) per register block
constexpr int kUnroll = 4;  // 16-byte weight chunks in flight per lane and row
constexpr int kThreads = 256;

enum { WK_F32 = 0, WK_BF16 = 1, WK_Q8 = 2 };

template <int WK>
struct WTraits;
template <>
struct WTraits<WK_F32> {
  static constexpr int VEC = 4;
};
template <>
struct WTraits<WK_BF16> {
  static constexpr int VEC = 8;
};
template <>
struct WTraits<WK_Q8> {
  static constexpr int VEC = 16;
};

template <int WK>
__device__ __forceinline__ void decode_w(const uint4 u, float scale, float (&v)[WTraits<WK>::VEC]) {
  if constexpr (WK == WK_F32) {
    v[0] = __uint_as_float(u.x);
    v[1] = __uint_as_float(u.y);
    v[2] = __uint_as_float(u.z);
    v[3] = __uint_as_float(u.w);
  } else if constexpr (WK == WK_BF16) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
      v[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
    }
  } else {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
      for (int b = 0; b < 4; ++b) v[4 * i + b] = scale * static_cast<float>(static_cast<int8_t>((w[i] >> (8 * b)) & 0xFFu));
    }
  }
}

template <int VEC>
__device__ __forceinline__ void load_vec(const float* __restrict__ p, float (&v)[VEC]) {
#pragma unroll
  for (int i = 0; i < VEC / 4; ++i) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p) + i);
    v[4 * i] = a.x;
    v[4 * i + 1] = a.y;
    v[4 * i + 2] = a.z;
    v[4 * i + 3] = a.w;
  }
}

template <int VEC>
__device__ __forceinline__ void load_vec(const __nv_bfloat16* __restrict__ p, float (&v)[VEC]) {
  if constexpr (VEC == 4) {
    const uint2 a = __ldg(reinterpret_cast<const uint2*>(p));
    v[0] = bf16_bits_to_f32(a.x & 0xFFFFu);
    v[1] = bf16_bits_to_f32(a.x >> 16);
    v[2] = bf16_bits_to_f32(a.y & 0xFFFFu);
    v[3] = bf16_bits_to_f32(a.y >> 16);
  } else {
#pragma unroll
    for (int i = 0; i < VEC / 8; ++i) {
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(p) + i);
      const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[8 * i + 2 * j] = bf16_bits_to_f32(w[j] & 0xFFFFu);
        v[8 * i + 2 * j + 1] = bf16_bits_to_f32(w[j] >> 16);
      }
    }
  }
}

// Builds the list of experts with at least one row (offsets == nullptr: one group).
__device__ __forceinline__ int active_experts(const int32_t* offsets, int E, int* s_active, int* s_warp) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = threadIdx.x;
  const bool f = offsets && e < E && offsets[e + 1] > offsets[e];
  const unsigned b = __ballot_sync(0xffffffffu, f);
  if (lane == 0) s_warp[warp] = __popc(b);
  __syncthreads();
  int base = 0, n = 0;
  for (int w = 0; w < kThreads / 32; ++w) {
    if (w < warp) base += s_warp[w];
    n += s_warp[w];
  }
  if (f) s_active[base + __popc(b & ((1u << lane) - 1u))] = e;
  if (!offsets) {
    if (threadIdx.x == 0) s_active[0] = 0;
    n = 1;
  }
  __syncthreads();
  return n;
}

template <typename XT, int WK>
__global__ void __launch_bounds__(kThreads) stream_gate_up_kernel(
    const XT* __restrict__ x, int T, int H, int I, int K, const uint8_t* __restrict__ gate,
    const uint8_t* __restrict__ up, const __half* __restrict__ gate_s, const __half* __restrict__ up_s,
    const int32_t* __restrict__ offsets, int E, const int32_t* __restrict__ pairs, int act, float* __restrict__ h) {
  constexpr int VEC = WTraits<WK>::VEC;
  constexpr int EB = (WK == WK_F32) ? 4 : (WK == WK_BF16 ? 2 : 1);
  __shared__ int s_active[kThreads];
  __shared__ int s_warp[kThreads / 32];
  const int n_active = active_experts(offsets, E, s_active, s_warp);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nchunk = H / VEC;
  const long long total = static_cast<long long>(n_active) * I;
  const long long stride = static_cast<long long>(gridDim.x) * (kThreads / 32);
  for (long long item = static_cast<long long>(blockIdx.x) * (kThreads / 32) + warp; item < total; item += stride) {
    const int a = static_cast<int>(item / I);
    const int i = static_cast<int>(item - static_cast<long long>(a) * I);
    const int e = s_active[a];
    const int r0 = offsets ? offsets[e] : 0;
    const int r1 = offsets ? offsets[e + 1] : T;
    const size_t wrow = static_cast<size_t>(e) * I + i;
    const uint4* grow = reinterpret_cast<const uint4*>(gate + wrow * H * EB);
    const uint4* urow = reinterpret_cast<const uint4*>(up + wrow * H * EB);
    const __half* gsr = (WK == WK_Q8) ? gate_s + wrow * (H / 32) : nullptr;
    const __half* usr = (WK == WK_Q8) ? up_s + wrow * (H / 32) : nullptr;
    for (int rc = r0; rc < r1; rc += kRows) {
      const int nr = min(kRows, r1 - rc);
      int tok[kRows];
#pragma unroll
      for (int c = 0; c < kRows; ++c) tok[c] = (c < nr) ? (pairs ? pairs[rc + c] / K : rc + c) : 0;
      float ag[kRows], au[kRows];
#pragma unroll
      for (int c = 0; c < kRows; ++c) ag[c] = au[c] = 0.f;
      for (int ch0 = lane; ch0 < nchunk; ch0 += 32 * kUnroll) {
        uint4 wg[kUnroll], wu[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int ch = ch0 + 32 * u;
          if (ch < nchunk) {
            wg[u] = __ldg(grow + ch);
            wu[u] = __ldg(urow + ch);
          }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int ch = ch0 + 32 * u;
          if (ch < nchunk) {
            float vg[VEC], vu[VEC];
            const float sg = (WK == WK_Q8) ? __half2float(gsr[ch >> 1]) : 1.f;
            const float su = (WK == WK_Q8) ? __half2float(usr[ch >> 1]) : 1.f;
            decode_w<WK>(wg[u], sg, vg);
            decode_w<WK>(wu[u], su, vu);
#pragma unroll
            for (int c = 0; c < kRows; ++c) {
              if (c < nr) {
                float xv[VEC];
                load_vec<VEC>(x + static_cast<size_t>(tok[c]) * H + static_cast<size_t>(ch) * VEC, xv);
#pragma unroll
                for (int q = 0; q < VEC; ++q) {
                  ag[c] = fmaf(vg[q], xv[q], ag[c]);
                  au[c] = fmaf(vu[q], xv[q], au[c]);
                }
              }
            }
          }
        }
      }
#pragma unroll
      for (int c = 0; c < kRows; ++c) {
        const float g = warp_sum(ag[c]);
        const float u = warp_sum(au[c]);
        if (lane == c && c < nr) h[static_cast<size_t>(rc + c) * I + i] = act_fn(act, g) * u;
      }
    }
  }
}

template <int WK>
__global__ void __launch_bounds__(kThreads) stream_down_kernel(
    const float* __restrict__ h, int I, int H, int T, const uint8_t* __restrict__ down,
    const __half* __restrict__ down_s, const int32_t* __restrict__ offsets, int E, const int32_t* __restrict__ pairs,
    const float* __restrict__ row_scale, float* __restrict__ y) {
  constexpr int VEC = WTraits<WK>::VEC;
  constexpr int EB = (WK == WK_F32) ? 4 : (WK == WK_BF16 ? 2 : 1);
  __shared__ int s_active[kThreads];
  __shared__ int s_warp[kThreads / 32];
  const int n_active = active_experts(offsets, E, s_active, s_warp);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nchunk = I / VEC;
  const long long total = static_cast<long long>(n_active) * H;
  const long long stride = static_cast<long long>(gridDim.x) * (kThreads / 32);
  for (long long item = static_cast<long long>(blockIdx.x) * (kThreads / 32) + warp; item < total; item += stride) {
    const int a = static_cast<int>(item / H);
    const int j = static_cast<int>(item - static_cast<long long>(a) * H);
    const int e = s_active[a];
    const int r0 = offsets ? offsets[e] : 0;
    const int r1 = offsets ? offsets[e + 1] : T;
    const size_t wrow = static_cast<size_t>(e) * H + j;
    const uint4* drow = reinterpret_cast<const uint4*>(down + wrow * I * EB);
    const __half* dsr = (WK == WK_Q8) ? down_s + wrow * (I / 32) : nullptr;
    for (int rc = r0; rc < r1; rc += kRows) {
      const int nr = min(kRows, r1 - rc);
      float acc[kRows];
#pragma unroll
      for (int c = 0; c < kRows; ++c) acc[c] = 0.f;
      for (int ch0 = lane; ch0 < nchunk; ch0 += 32 * kUnroll) {
        uint4 wd[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int ch = ch0 + 32 * u;
          if (ch < nchunk) wd[u] = __ldg(drow + ch);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int ch = ch0 + 32 * u;
          if (ch < nchunk) {
            float vd[VEC];
            decode_w<WK>(wd[u], (WK == WK_Q8) ? __half2float(dsr[ch >> 1]) : 1.f, vd);
#pragma unroll
            for (int c = 0; c < kRows; ++c) {
              if (c < nr) {
                float hv[VEC];
                load_vec<VEC>(h + static_cast<size_t>(rc + c) * I + static_cast<size_t>(ch) * VEC, hv);
#pragma unroll
                for (int q = 0; q < VEC; ++q) acc[c] = fmaf(vd[q], hv[q], acc[c]);
              }
            }
          }
        }
      }
#pragma unroll
      for (int c = 0; c < kRows; ++c) {
        const float s = warp_sum(acc[c]);
        if (lane == c && c < nr) {
          const int dest = pairs ? pairs[rc + c] : rc + c;
          const float sc = row_scale ? row_scale[dest] : 1.f;
          y[static_cast<size_t>(dest) * H + j] = sc * s;
        }
      }
    }
  }
}

template <typename OT>
__global__ void __launch_bounds__(256) combine_kernel(const float4* __restrict__ y_slots,
                                                      const float4* __restrict__ y_shared, int T, int K, int H4,
                                                      OT* __restrict__ out) {
  const long long total = static_cast<long long>(T) * H4;
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long t = idx / H4;
    const int c = static_cast<int>(idx - t * H4);
    float4 acc = __ldg(y_slots + (t * K) * H4 + c);
    for (int k = 1; k < K; ++k) {
      const float4 v = __ldg(y_slots + (t * K + k) * H4 + c);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    if (y_shared) {
      const float4 v = __ldg(y_shared + t * H4 + c);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    if constexpr (sizeof(OT) == 4) {
      reinterpret_cast<float4*>(out)[idx] = acc;
    } else {
      const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
      const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
      uint2 pk;
      pk.x = *reinterpret_cast<const uint32_t*>(&lo);
      pk.y = *reinterpret_cast<const uint32_t*>(&hi);
      reinterpret_cast<uint2*>(out)[idx] = pk;
    }
  }
}

__global__ void __launch_bounds__(256) q8_0_split_kernel(const uint8_t* __restrict__ blocks, long long nblocks,
                                                         int8_t* __restrict__ q, uint16_t* __restrict__ scales) {
  for (long long b = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; b < nblocks;
       b += static_cast<long long>(gridDim.x) * blockDim.x) {
    const uint8_t* src = blocks + b * 34;
    scales[b] = static_cast<uint16_t>(src[0] | (src[1] << 8));
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      w[i] = src[2 + 4 * i] | (src[3 + 4 * i] << 8) | (src[4 + 4 * i] << 16) | (static_cast<uint32_t>(src[5 + 4 * i]) << 24);
    uint4* dst = reinterpret_cast<uint4*>(q + b * 32);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
  }
}

template <typename KernelT>
int resident_blocks(KernelT kernel, int num_sms) {
  int per_sm = 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, 0) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  return per_sm * num_sms;
}

template <typename XT, int WK>
cudaError_t gate_up_typed(const Ctx& c, const void* x, int T, int H, int I, int K, const void* gate, const void* up,
                          const void* gs, const void* us, const int32_t* offsets, int E, const int32_t* pairs,
                          int rows_bound, int act, float* h) {
  const long long items = static_cast<long long>(offsets ? std::min(E, rows_bound) : 1) * I;
  const int grid = static_cast<int>(std::max(
      1LL, std::min<long long>((items + 7) / 8, resident_blocks(stream_gate_up_kernel<XT, WK>, c.num_sms))));
  KernelScope ks(c, "stream_gate_up");
  stream_gate_up_kernel<XT, WK><<<grid, kThreads, 0, c.stream>>>(
      static_cast<const XT*>(x), T, H, I, K, static_cast<const uint8_t*>(gate), static_cast<const uint8_t*>(up),
      static_cast<const __half*>(gs), static_cast<const __half*>(us), offsets, E, pairs, act, h);
  return cudaGetLastError();
}

template <int WK>
cudaError_t down_typed(const Ctx& c, const float* h, int I, int H, int T, const void* down, const void* ds,
                       const int32_t* offsets, int E, const int32_t* pairs, int rows_bound, const float* row_scale,
                       float* y) {
  const long long items = static_cast<long long>(offsets ? std::min(E, rows_bound) : 1) * H;
  const int grid = static_cast<int>(
      std::max(1LL, std::min<long long>((items + 7) / 8, resident_blocks(stream_down_kernel<WK>, c.num_sms))));
  KernelScope ks(c, "stream_down");
  stream_down_kernel<WK><<<grid, kThreads, 0, c.stream>>>(h, I, H, T, static_cast<const uint8_t*>(down),
                                                          static_cast<const __half*>(ds), offsets, E, pairs,
                                                          row_scale, y);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_stream_gate_up(const Ctx& c, const void* x, int x_dtype, int T, int H, int I, int K,
                                  const void* gate, const void* up, const void* gate_scale, const void* up_scale,
                                  int w_dtype, const int32_t* offsets, int E, const int32_t* pairs, int rows_bound,
                                  int act, float* h) {
  if (rows_bound <= 0) return cudaSuccess;
  // offsets == nullptr means one group whose rows are the T tokens
  const int TT = offsets ? 0 : rows_bound;
  if (x_dtype == MOE_F32) {
    if (w_dtype == MOE_F32)
      return gate_up_typed<float, WK_F32>(c, x, TT, H, I, K, gate, up, nullptr, nullptr, offsets, E, pairs,
                                          rows_bound, act, h);
    if (w_dtype == MOE_BF16)
      return gate_up_typed<float, WK_BF16>(c, x, TT, H, I, K, gate, up, nullptr, nullptr, offsets, E, pairs,
                                           rows_bound, act, h);
    return gate_up_typed<float, WK_Q8>(c, x, TT, H, I, K, gate, up, gate_scale, up_scale, offsets, E, pairs,
                                       rows_bound, act, h);
  }
  if (w_dtype == MOE_F32)
    return gate_up_typed<__nv_bfloat16, WK_F32>(c, x, TT, H, I, K, gate, up, nullptr, nullptr, offsets, E, pairs,
                                                rows_bound, act, h);
  if (w_dtype == MOE_BF16)
    return gate_up_typed<__nv_bfloat16, WK_BF16>(c, x, TT, H, I, K, gate, up, nullptr, nullptr, offsets, E, pairs,
                                                 rows_bound, act, h);
  return gate_up_typed<__nv_bfloat16, WK_Q8>(c, x, TT, H, I, K, gate, up, gate_scale, up_scale, offsets, E, pairs,
                                             rows_bound, act, h);
}

cudaError_t launch_stream_down(const Ctx& c, const float* h, int I, int H, const void* down, const void* down_scale,
                               int w_dtype, const int32_t* offsets, int E, const int32_t* pairs, int rows_bound,
                               const float* row_scale, float* y) {
  if (rows_bound <= 0) return cudaSuccess;
  const int TT = offsets ? 0 : rows_bound;
  if (w_dtype == MOE_F32)
    return down_typed<WK_F32>(c, h, I, H, TT, down, nullptr, offsets, E, pairs, rows_bound, row_scale, y);
  if (w_dtype == MOE_BF16)
    return down_typed<WK_BF16>(c, h, I, H, TT, down, nullptr, offsets, E, pairs, rows_bound, row_scale, y);
  return down_typed<WK_Q8>(c, h, I, H, TT, down, down_scale, offsets, E, pairs, rows_bound, row_scale, y);
}

cudaError_t launch_combine(const Ctx& c, const float* y_slots, const float* y_shared, int T, int K, int H, void* out,
                           int out_dtype) {
  if (T == 0) return cudaSuccess;
  const int H4 = H / 4;
  const long long total = static_cast<long long>(T) * H4;
  const int blocks = static_cast<int>(std::max(1LL, std::min<long long>((total + 255) / 256, 16LL * c.num_sms)));
  KernelScope ks(c, "combine");
  if (out_dtype == MOE_F32)
    combine_kernel<float><<<blocks, 256, 0, c.stream>>>(reinterpret_cast<const float4*>(y_slots),
                                                        reinterpret_cast<const float4*>(y_shared), T, K, H4,
                                                        static_cast<float*>(out));
  else
    combine_kernel<__nv_bfloat16><<<blocks, 256, 0, c.stream>>>(reinterpret_cast<const float4*>(y_slots),
                                                                reinterpret_cast<const float4*>(y_shared), T, K,
                                                                H4, static_cast<__nv_bfloat16*>(out));
  return cudaGetLastError();
}

cudaError_t launch_q8_0_split(const Ctx& c, const void* blocks, int64_t rows, int64_t cols, int8_t* q,
                              void* scales) {
  const long long nb = static_cast<long long>(rows) * (cols / 32);
  if (nb == 0) return cudaSuccess;
  const int grid = static_cast<int>(std::max(1LL, std::min<long long>((nb + 255) / 256, 16LL * c.num_sms)));
  KernelScope ks(c, "q8_0_split");
  q8_0_split_kernel<<<grid, 256, 0, c.stream>>>(static_cast<const uint8_t*>(blocks), nb, q,
                                                static_cast<uint16_t*>(scales));
  return cudaGetLastError();
}

}  // namespace moe
