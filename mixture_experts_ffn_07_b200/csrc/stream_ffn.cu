// The weighted combine of the slot rows (plus the shared expert) and the
// one-time splits of GGML Q8_0 and Q6_K blocks into quant and scale planes.
#include "stream_core.cuh"

namespace moe {

namespace {

// One thread per (token, float4 column) item, grid-stride; IT is the index
// type (32-bit whenever the item count allows, which keeps the row division cheap).
template <typename OT, typename IT>
__global__ void __launch_bounds__(256) combine_kernel(const float4* __restrict__ y_slots,
                                                      const float4* __restrict__ y_shared, int T, int K, int H4,
                                                      OT* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  const IT total = static_cast<IT>(T) * H4;
  for (IT idx = static_cast<IT>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<IT>(gridDim.x) * blockDim.x) {
    const IT t = idx / H4;
    const IT c = idx - t * H4;
    const float4* ys = y_slots + (t * K) * H4 + c;
    float4 v[8];
    float4 acc = __ldg(ys);
    for (int k0 = 1; k0 < K; k0 += 8) {  // up to eight slot rows in flight, added in k order
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (k0 + j < K) v[j] = __ldg(ys + static_cast<IT>(k0 + j) * H4);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (k0 + j < K) {
          acc.x += v[j].x;
          acc.y += v[j].y;
          acc.z += v[j].z;
          acc.w += v[j].w;
        }
    }
    if (y_shared) {
      const float4 w = __ldg(y_shared + t * H4 + c);
      acc.x += w.x;
      acc.y += w.y;
      acc.z += w.z;
      acc.w += w.w;
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

// The combine of the tensor-core layer, whose slot rows hold the experts' bf16
// outputs (mlx-native moe_dispatch.rs, moe_weighted_sum_seq_bf16_input: bf16
// expert outputs, f32 weights, f32 accumulator): out[t] = w[t,0] y[t,0] +
// w[t,1] y[t,1] + ... in k order (a product, then fused multiply-adds), plus
// the shared expert's f32 row; one thread per (token, 4 columns), grid-stride.
__device__ __forceinline__ float4 bf16x4_f4(uint2 v) {
  return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u), __uint_as_float(v.y << 16),
                     __uint_as_float(v.y & 0xFFFF0000u));
}

template <typename IT>
__global__ void __launch_bounds__(256) combine_w_kernel(const uint2* __restrict__ ys, const float* __restrict__ w,
                                                        const float4* __restrict__ y_shared, int T, int K, int H4,
                                                        __nv_bfloat16* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  const IT total = static_cast<IT>(T) * H4;
  for (IT idx = static_cast<IT>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<IT>(gridDim.x) * blockDim.x) {
    const IT t = idx / H4;
    const IT c = idx - t * H4;
    const uint2* base = ys + (t * K) * H4 + c;
    const float* wt = w + t * K;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k0 = 0; k0 < K; k0 += 8) {  // up to eight slot rows in flight, added in k order
      uint2 v[8];
      float wk[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (k0 + j < K) {
          v[j] = __ldg(base + static_cast<IT>(k0 + j) * H4);
          wk[j] = __ldg(wt + k0 + j);
        }
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (k0 + j < K) {
          const float4 y = bf16x4_f4(v[j]);
          if (k0 + j == 0) {
            acc = make_float4(wk[j] * y.x, wk[j] * y.y, wk[j] * y.z, wk[j] * y.w);
          } else {
            acc.x = fmaf(wk[j], y.x, acc.x);
            acc.y = fmaf(wk[j], y.y, acc.y);
            acc.z = fmaf(wk[j], y.z, acc.z);
            acc.w = fmaf(wk[j], y.w, acc.w);
          }
        }
    }
    if (y_shared) {
      const float4 s4 = __ldg(y_shared + t * H4 + c);
      acc.x += s4.x;
      acc.y += s4.y;
      acc.z += s4.z;
      acc.w += s4.w;
    }
    const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 pk;
    pk.x = *reinterpret_cast<const uint32_t*>(&lo);
    pk.y = *reinterpret_cast<const uint32_t*>(&hi);
    reinterpret_cast<uint2*>(out)[idx] = pk;
  }
}

// One thread per Q6_K block: ql|qh (192 bytes) to the quant plane, the 16
// scales and the fp16 d to the block's places in its row of the scale plane;
// the last block of a row also zeroes the row's padding.
__global__ void __launch_bounds__(256) q6_k_split_kernel(const uint8_t* __restrict__ blocks, long long nblocks,
                                                         int nb, int srow, uint8_t* __restrict__ q,
                                                         uint8_t* __restrict__ scales) {
  pdl_trigger();
  pdl_wait();
  for (long long b = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; b < nblocks;
       b += static_cast<long long>(gridDim.x) * blockDim.x) {
    const uint8_t* src = blocks + b * 210;
    uint4* dq = reinterpret_cast<uint4*>(q + b * 192);
    for (int i = 0; i < 12; ++i) {
      uint32_t w[4];
      for (int j = 0; j < 4; ++j) {
        const uint8_t* p = src + 16 * i + 4 * j;
        w[j] = p[0] | (p[1] << 8) | (p[2] << 16) | (static_cast<uint32_t>(p[3]) << 24);
      }
      dq[i] = make_uint4(w[0], w[1], w[2], w[3]);
    }
    const long long r = b / nb;
    const int j = static_cast<int>(b - r * nb);
    uint8_t* row = scales + r * srow;
    for (int i = 0; i < 16; ++i) row[16 * j + i] = src[192 + i];
    row[16 * nb + 2 * j] = src[208];
    row[16 * nb + 2 * j + 1] = src[209];
    if (j == nb - 1)
      for (int i = 18 * nb; i < srow; ++i) row[i] = 0;
  }
}

}  // namespace

template <typename OT, typename IT>
cudaError_t combine_typed(const Ctx& c, const float* y_slots, const float* y_shared, int T, int K, int H4, void* out) {
  auto kern = combine_kernel<OT, IT>;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, 0) != cudaSuccess || per_sm < 1) per_sm = 1;
  const long long total = static_cast<long long>(T) * H4;
  const int blocks = static_cast<int>(std::max(1LL, std::min<long long>((total + 255) / 256, 1LL * per_sm * c.num_sms)));
  return launch_kernel(c, kern, dim3(blocks), dim3(256), 0, reinterpret_cast<const float4*>(y_slots),
                       reinterpret_cast<const float4*>(y_shared), T, K, H4, static_cast<OT*>(out));
}

cudaError_t launch_combine(const Ctx& c, const float* y_slots, const float* y_shared, int T, int K, int H, void* out,
                           int out_dtype) {
  if (T == 0) return cudaSuccess;
  const int H4 = H / 4;
  // 32-bit indices while every slot row offset fits
  const bool narrow = static_cast<long long>(T) * K * H4 < (1LL << 31) - 256LL * 1024 * 148;
  KernelScope ks(c, "combine");
  if (out_dtype == MOE_F32)
    return narrow ? combine_typed<float, int>(c, y_slots, y_shared, T, K, H4, out)
                  : combine_typed<float, long long>(c, y_slots, y_shared, T, K, H4, out);
  return narrow ? combine_typed<__nv_bfloat16, int>(c, y_slots, y_shared, T, K, H4, out)
                : combine_typed<__nv_bfloat16, long long>(c, y_slots, y_shared, T, K, H4, out);
}

template <typename IT>
cudaError_t combine_w_typed(const Ctx& c, const __nv_bfloat16* y_slots, const float* w, const float* y_shared, int T,
                            int K, int H4, void* out) {
  auto kern = combine_w_kernel<IT>;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, 0) != cudaSuccess || per_sm < 1) per_sm = 1;
  const long long total = static_cast<long long>(T) * H4;
  const int blocks = static_cast<int>(std::max(1LL, std::min<long long>((total + 255) / 256, 1LL * per_sm * c.num_sms)));
  return launch_kernel(c, kern, dim3(blocks), dim3(256), 0, reinterpret_cast<const uint2*>(y_slots), w,
                       reinterpret_cast<const float4*>(y_shared), T, K, H4, static_cast<__nv_bfloat16*>(out));
}

cudaError_t launch_combine_weighted(const Ctx& c, const __nv_bfloat16* y_slots, const float* w, const float* y_shared,
                                    int T, int K, int H, void* out) {
  if (T == 0) return cudaSuccess;
  const int H4 = H / 4;
  const bool narrow = static_cast<long long>(T) * K * H4 < (1LL << 31) - 256LL * 1024 * 148;
  KernelScope ks(c, "combine");
  return narrow ? combine_w_typed<int>(c, y_slots, w, y_shared, T, K, H4, out)
                : combine_w_typed<long long>(c, y_slots, w, y_shared, T, K, H4, out);
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

cudaError_t launch_q6_k_split(const Ctx& c, const void* blocks, int64_t rows, int64_t cols, void* q, void* scales) {
  const int nb = static_cast<int>(cols / 256);
  const long long nblk = static_cast<long long>(rows) * nb;
  if (nblk == 0) return cudaSuccess;
  const int srow = stream::q6k_srow_bytes(static_cast<int>(cols));
  const int grid = static_cast<int>(std::max(1LL, std::min<long long>((nblk + 255) / 256, 16LL * c.num_sms)));
  KernelScope ks(c, "q6_k_split");
  return launch_kernel(c, q6_k_split_kernel, dim3(grid), dim3(256), 0, static_cast<const uint8_t*>(blocks), nblk, nb,
                       srow, static_cast<uint8_t*>(q), static_cast<uint8_t*>(scales));
}

}  // namespace moe
