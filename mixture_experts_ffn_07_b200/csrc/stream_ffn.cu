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

template <int VEC>
__device__ __forceinline__ void load_vec_smem(const float* p, float (&v)[VEC]) {
#pragma unroll
  for (int i = 0; i < VEC / 4; ++i) {
    const float4 a = reinterpret_cast<const float4*>(p)[i];
    v[4 * i] = a.x;
    v[4 * i + 1] = a.y;
    v[4 * i + 2] = a.z;
    v[4 * i + 3] = a.w;
  }
}

template <int VEC>
__device__ __forceinline__ void load_vec_smem(const __nv_bfloat16* p, float (&v)[VEC]) {
  if constexpr (VEC == 4) {
    const uint2 a = *reinterpret_cast<const uint2*>(p);
    v[0] = bf16_bits_to_f32(a.x & 0xFFFFu);
    v[1] = bf16_bits_to_f32(a.x >> 16);
    v[2] = bf16_bits_to_f32(a.y & 0xFFFFu);
    v[3] = bf16_bits_to_f32(a.y >> 16);
  } else {
#pragma unroll
    for (int i = 0; i < VEC / 8; ++i) {
      const uint4 a = reinterpret_cast<const uint4*>(p)[i];
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

// Chunks of 16 weight bytes a lane requests before it computes on any of them.
template <int WK>
struct Unroll {
  static constexpr int U = (WK == WK_Q8) ? 4 : 8;
};

constexpr int kStageBytes = 96 * 1024;  // shared memory for the staged token rows of one CTA item

// Copies rows src[row(c)] (c < n, `len` elements of T each) into dst[c * len].
template <typename T, typename RowFn>
__device__ __forceinline__ void stage_rows(T* dst, const T* __restrict__ src, int n, int len, RowFn row) {
  const int vpr = len * static_cast<int>(sizeof(T)) / 16;
  for (int i = threadIdx.x; i < n * vpr; i += blockDim.x) {
    const int c = i / vpr, q = i - c * vpr;
    reinterpret_cast<uint4*>(dst + static_cast<size_t>(c) * len)[q] =
        __ldg(reinterpret_cast<const uint4*>(src + static_cast<size_t>(row(c)) * len) + q);
  }
}

// gate/up: a CTA item is (touched expert, block of RB intermediate rows).  The
// CTA stages the expert's token rows of x in shared memory (TS at a time),
// then each warp streams its gate and up rows once against all staged tokens.
template <typename XT, int WK>
__global__ void __launch_bounds__(kThreads, 2) stream_gate_up_kernel(
    const XT* __restrict__ x, int T, int H, int I, int K, const uint8_t* __restrict__ gate,
    const uint8_t* __restrict__ up, const __half* __restrict__ gate_s, const __half* __restrict__ up_s,
    const int32_t* __restrict__ offsets, int E, const int32_t* __restrict__ pairs, int act, float* __restrict__ h,
    int RB, int TS) {
  constexpr int VEC = WTraits<WK>::VEC;
  constexpr int EB = (WK == WK_F32) ? 4 : (WK == WK_BF16 ? 2 : 1);
  constexpr int U = Unroll<WK>::U;
  extern __shared__ __align__(16) uint8_t stage_raw[];
  XT* xs = reinterpret_cast<XT*>(stage_raw);
  __shared__ int s_active[kThreads];
  __shared__ int s_warp[kThreads / 32];
  pdl_trigger();
  pdl_wait();
  const int n_active = active_experts(offsets, E, s_active, s_warp);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nchunk = H / VEC;
  const int blocks_per_expert = (I + RB - 1) / RB;
  const int total = n_active * blocks_per_expert;
  for (int item = blockIdx.x; item < total; item += gridDim.x) {
    const int a = item / blocks_per_expert;
    const int i0 = (item - a * blocks_per_expert) * RB;
    const int i1 = min(I, i0 + RB);
    const int e = s_active[a];
    const int r0 = offsets ? offsets[e] : 0;
    const int r1 = offsets ? offsets[e + 1] : T;
    for (int rc = r0; rc < r1; rc += TS) {
      const int nr = min(TS, r1 - rc);
      __syncthreads();  // the previous token rows are no longer read
      stage_rows(xs, x, nr, H, [&](int c) { return pairs ? pairs[rc + c] / K : rc + c; });
      __syncthreads();
      for (int i = i0 + warp; i < i1; i += kThreads / 32) {
        const size_t wrow = static_cast<size_t>(e) * I + i;
        const uint4* grow = reinterpret_cast<const uint4*>(gate + wrow * H * EB);
        const uint4* urow = reinterpret_cast<const uint4*>(up + wrow * H * EB);
        const __half* gsr = (WK == WK_Q8) ? gate_s + wrow * (H / 32) : nullptr;
        const __half* usr = (WK == WK_Q8) ? up_s + wrow * (H / 32) : nullptr;
        float ag[kRows], au[kRows];
#pragma unroll
        for (int c = 0; c < kRows; ++c) ag[c] = au[c] = 0.f;
        for (int ch0 = lane; ch0 < nchunk; ch0 += 32 * U) {
          uint4 wg[U], wu[U];
          float sg[U], su[U];
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const int ch = ch0 + 32 * u;
            if (ch < nchunk) {
              wg[u] = __ldg(grow + ch);
              wu[u] = __ldg(urow + ch);
              if (WK == WK_Q8) {
                sg[u] = __half2float(gsr[ch >> 1]);
                su[u] = __half2float(usr[ch >> 1]);
              }
            }
          }
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const int ch = ch0 + 32 * u;
            if (ch < nchunk) {
              float vg[VEC], vu[VEC];
              decode_w<WK>(wg[u], WK == WK_Q8 ? sg[u] : 1.f, vg);
              decode_w<WK>(wu[u], WK == WK_Q8 ? su[u] : 1.f, vu);
#pragma unroll
              for (int c = 0; c < kRows; ++c) {
                if (c < nr) {
                  float xv[VEC];
                  load_vec_smem<VEC>(xs + static_cast<size_t>(c) * H + static_cast<size_t>(ch) * VEC, xv);
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
          if (c < nr) {  // warp-uniform
            const float g = warp_sum(ag[c]);
            const float u = warp_sum(au[c]);
            if (lane == c) h[static_cast<size_t>(rc + c) * I + i] = act_fn(act, g) * u;
          }
        }
      }
    }
  }
}

// down: a CTA item is (touched expert, block of RB output rows).  The CTA stages
// the expert's h rows (TS at a time); a warp takes RPI rows at once and its
// lanes share their (row, chunk) index space, so short rows still give every
// lane several 16-byte loads to keep in flight.
template <int WK, int RPI>
__global__ void __launch_bounds__(kThreads, 2) stream_down_kernel(
    const float* __restrict__ h, int I, int H, int T, const uint8_t* __restrict__ down,
    const __half* __restrict__ down_s, const int32_t* __restrict__ offsets, int E, const int32_t* __restrict__ pairs,
    const float* __restrict__ row_scale, float* __restrict__ y, int RB, int TS) {
  constexpr int VEC = WTraits<WK>::VEC;
  constexpr int EB = (WK == WK_F32) ? 4 : (WK == WK_BF16 ? 2 : 1);
  constexpr int U = Unroll<WK>::U;
  extern __shared__ __align__(16) uint8_t stage_raw[];
  float* hs = reinterpret_cast<float*>(stage_raw);
  __shared__ int s_active[kThreads];
  __shared__ int s_warp[kThreads / 32];
  __shared__ int s_dest[kRows];    // output row of each staged row
  __shared__ float s_scale[kRows]; // and its routing weight
  pdl_trigger();
  pdl_wait();
  const int n_active = active_experts(offsets, E, s_active, s_warp);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nchunk = I / VEC;
  const int blocks_per_expert = (H + RB - 1) / RB;
  const int total = n_active * blocks_per_expert;
  for (int item = blockIdx.x; item < total; item += gridDim.x) {
    const int a = item / blocks_per_expert;
    const int jb0 = (item - a * blocks_per_expert) * RB;
    const int jb1 = min(H, jb0 + RB);
    const int e = s_active[a];
    const int r0 = offsets ? offsets[e] : 0;
    const int r1 = offsets ? offsets[e + 1] : T;
    for (int rc = r0; rc < r1; rc += TS) {
      const int nr = min(TS, r1 - rc);
      __syncthreads();
      stage_rows(hs, h, nr, I, [&](int c) { return rc + c; });
      if (threadIdx.x < nr) {
        const int dest = pairs ? pairs[rc + threadIdx.x] : rc + threadIdx.x;
        s_dest[threadIdx.x] = dest;
        s_scale[threadIdx.x] = row_scale ? row_scale[dest] : 1.f;
      }
      __syncthreads();
      for (int j0 = jb0 + warp * RPI; j0 < jb1; j0 += (kThreads / 32) * RPI) {
        const int nrow = min(RPI, jb1 - j0);
        const size_t wrow0 = static_cast<size_t>(e) * H + j0;
        const uint8_t* dbase = down + wrow0 * I * EB;
        const __half* sbase = (WK == WK_Q8) ? down_s + wrow0 * (I / 32) : nullptr;
        const int span = nrow * nchunk;
        float acc[RPI][kRows];
#pragma unroll
        for (int r = 0; r < RPI; ++r)
#pragma unroll
          for (int c = 0; c < kRows; ++c) acc[r][c] = 0.f;
        for (int k0 = lane; k0 < span; k0 += 32 * U) {
          uint4 wd[U];
          float sd[U];
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const int k = k0 + 32 * u;
            if (k < span) {
              const int r = k / nchunk, ch = k - r * nchunk;
              wd[u] = __ldg(reinterpret_cast<const uint4*>(dbase + static_cast<size_t>(r) * I * EB) + ch);
              if (WK == WK_Q8) sd[u] = __half2float(sbase[static_cast<size_t>(r) * (I / 32) + (ch >> 1)]);
            }
          }
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const int k = k0 + 32 * u;
            if (k < span) {
              const int r = k / nchunk, ch = k - r * nchunk;
              float vd[VEC];
              decode_w<WK>(wd[u], WK == WK_Q8 ? sd[u] : 1.f, vd);
#pragma unroll
              for (int c = 0; c < kRows; ++c) {
                if (c < nr) {
                  float hv[VEC];
                  load_vec_smem<VEC>(hs + static_cast<size_t>(c) * I + static_cast<size_t>(ch) * VEC, hv);
                  float part = 0.f;
#pragma unroll
                  for (int q = 0; q < VEC; ++q) part = fmaf(vd[q], hv[q], part);
#pragma unroll
                  for (int rr = 0; rr < RPI; ++rr)
                    if (rr == r) acc[rr][c] += part;
                }
              }
            }
          }
        }
#pragma unroll
        for (int rr = 0; rr < RPI; ++rr) {
          if (rr < nrow) {
#pragma unroll
            for (int c = 0; c < kRows; ++c) {
              if (c < nr) {
                const float sv = warp_sum(acc[rr][c]);
                if (lane == c) y[static_cast<size_t>(s_dest[c]) * H + j0 + rr] = s_scale[c] * sv;
              }
            }
          }
        }
      }
    }
  }
}

template <typename OT>
__global__ void __launch_bounds__(256) combine_kernel(const float4* __restrict__ y_slots,
                                                      const float4* __restrict__ y_shared, int T, int K, int H4,
                                                      OT* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
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
  pdl_trigger();
  pdl_wait();
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
int resident_blocks(KernelT kernel, int num_sms, size_t smem) {
  int per_sm = 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, smem) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  return per_sm * num_sms;
}

// Rows per CTA item: a multiple of 8 between 8 and 64, aiming at ~4 items per SM.
int rows_per_item(long long rows_bound, int num_sms, int lo) {
  long long rb = rows_bound / (4LL * num_sms);
  rb = std::max<long long>(lo, std::min<long long>(64, rb));
  return static_cast<int>(rb / 8 * 8);
}

template <typename XT, int WK>
cudaError_t gate_up_typed(const Ctx& c, const void* x, int T, int H, int I, int K, const void* gate, const void* up,
                          const void* gs, const void* us, const int32_t* offsets, int E, const int32_t* pairs,
                          int rows_bound, int act, float* h) {
  const long long experts = offsets ? std::min(E, rows_bound) : 1;
  const int RB = rows_per_item(experts * I, c.num_sms, 8);
  const int TS = static_cast<int>(std::max<long long>(1, std::min<long long>(kRows, kStageBytes / (1LL * H * sizeof(XT)))));
  const size_t smem = static_cast<size_t>(TS) * H * sizeof(XT);
  auto kern = stream_gate_up_kernel<XT, WK>;
  cudaError_t e = allow_dynamic_smem(reinterpret_cast<const void*>(kern), kStageBytes);
  if (e != cudaSuccess) return e;
  const long long items = experts * ((I + RB - 1) / RB);
  const int grid = static_cast<int>(std::max(1LL, std::min<long long>(items, resident_blocks(kern, c.num_sms, smem))));
  KernelScope ks(c, "stream_gate_up");
  return launch_kernel(c, kern, dim3(grid), dim3(kThreads), smem, static_cast<const XT*>(x), T, H, I, K,
                       static_cast<const uint8_t*>(gate), static_cast<const uint8_t*>(up),
                       static_cast<const __half*>(gs), static_cast<const __half*>(us), offsets, E, pairs, act, h, RB,
                       TS);
}

template <int WK, int RPI>
cudaError_t down_rpi(const Ctx& c, const float* h, int I, int H, int T, const void* down, const void* ds,
                     const int32_t* offsets, int E, const int32_t* pairs, int rows_bound, const float* row_scale,
                     float* y) {
  const long long experts = offsets ? std::min(E, rows_bound) : 1;
  const int RB = rows_per_item(experts * H, c.num_sms, 8 * RPI);
  const int TS = static_cast<int>(std::max<long long>(1, std::min<long long>(kRows, kStageBytes / (4LL * I))));
  const size_t smem = static_cast<size_t>(TS) * I * sizeof(float);
  auto kern = stream_down_kernel<WK, RPI>;
  cudaError_t e = allow_dynamic_smem(reinterpret_cast<const void*>(kern), kStageBytes);
  if (e != cudaSuccess) return e;
  const long long items = experts * ((H + RB - 1) / RB);
  const int grid = static_cast<int>(std::max(1LL, std::min<long long>(items, resident_blocks(kern, c.num_sms, smem))));
  KernelScope ks(c, "stream_down");
  return launch_kernel(c, kern, dim3(grid), dim3(kThreads), smem, h, I, H, T, static_cast<const uint8_t*>(down),
                       static_cast<const __half*>(ds), offsets, E, pairs, row_scale, y, RB, TS);
}

// Rows per warp pass so that a lane has about Unroll<WK>::U chunks of a pass to request at once.
template <int WK>
cudaError_t down_typed(const Ctx& c, const float* h, int I, int H, int T, const void* down, const void* ds,
                       const int32_t* offsets, int E, const int32_t* pairs, int rows_bound, const float* row_scale,
                       float* y) {
  const int per_row = I / WTraits<WK>::VEC;
  const int want = 32 * Unroll<WK>::U;
  if (per_row * 2 > want)
    return down_rpi<WK, 1>(c, h, I, H, T, down, ds, offsets, E, pairs, rows_bound, row_scale, y);
  if (per_row * 4 > want)
    return down_rpi<WK, 2>(c, h, I, H, T, down, ds, offsets, E, pairs, rows_bound, row_scale, y);
  return down_rpi<WK, 4>(c, h, I, H, T, down, ds, offsets, E, pairs, rows_bound, row_scale, y);
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
    return launch_kernel(c, combine_kernel<float>, dim3(blocks), dim3(256), 0,
                         reinterpret_cast<const float4*>(y_slots), reinterpret_cast<const float4*>(y_shared), T, K,
                         H4, static_cast<float*>(out));
  return launch_kernel(c, combine_kernel<__nv_bfloat16>, dim3(blocks), dim3(256), 0,
                       reinterpret_cast<const float4*>(y_slots), reinterpret_cast<const float4*>(y_shared), T, K, H4,
                       static_cast<__nv_bfloat16*>(out));
}

cudaError_t launch_q8_0_split(const Ctx& c, const void* blocks, int64_t rows, int64_t cols, int8_t* q,
                              void* scales) {
  const long long nb = static_cast<long long>(rows) * (cols / 32);
  if (nb == 0) return cudaSuccess;
  const int grid = static_cast<int>(std::max(1LL, std::min<long long>((nb + 255) / 256, 16LL * c.num_sms)));
  KernelScope ks(c, "q8_0_split");
  return launch_kernel(c, q8_0_split_kernel, dim3(grid), dim3(256), 0, static_cast<const uint8_t*>(blocks), nb, q,
                       static_cast<uint16_t*>(scales));
}

}  // namespace moe
