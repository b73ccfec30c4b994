// Backward of two steps of the layer, for training callers (mlx-native
// moe_dispatch.rs, the backward kernels of moe_weighted_sum_seq and
// moe_swiglu_seq):
//
//   combine   out[t,:] = sum_k w[t,k] y[t,k,:]
//             d_y[t,k,:] = w[t,k] d_out[t,:]        d_w[t,k] = <y[t,k,:], d_out[t,:]>
//   act * up  h[p,i] = act(g[p,i]) u[p,i]  with gate_up row p = [g | u]
//             d_g = d_h u act'(g)                   d_u = d_h act(g)
//
// Both read and write every element once and do a few flops per element, so
// they are HBM-bound: wide coalesced loads that bypass L1 for the streams read
// once, streaming stores, grids sized to the SM count.
//
// Combine backward: one warp per (token, slot) pair, four pairs per 128-thread
// CTA (so the CTAs spread evenly over the SMs in one wave).  A lane takes
// float4 columns, four at a time in flight from the slot row and from the
// token's d_out row (which the token's other slots read too, mostly from L2),
// writes w * d_out and keeps a partial dot product; the warp adds the partials
// with a fixed shuffle tree, so d_w is the same on every run.
#include "kernels.h"

namespace moe {

namespace {

constexpr int kBwdThreads = 256;
constexpr int kCombineThreads = 128;
constexpr int kColsInFlight = 4;

__device__ __forceinline__ float4 ld_once4(const float4* p) {
  float4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ float ld_once(const float* p) {
  float v;
  asm volatile("ld.global.nc.L1::no_allocate.f32 %0, [%1];" : "=f"(v) : "l"(p));
  return v;
}

// Loads of VEC-wide column j of a row, as float4 (VEC == 4) or one float in .x.
template <int VEC>
__device__ __forceinline__ float4 ld_col(const float* row, long long j) {
  if constexpr (VEC == 4) return ld_once4(reinterpret_cast<const float4*>(row) + j);
  return make_float4(ld_once(row + j), 0.f, 0.f, 0.f);
}
// d_out rows are read by each of the token's K slots: keep them cacheable.
template <int VEC>
__device__ __forceinline__ float4 ld_col_l2(const float* row, long long j) {
  if constexpr (VEC == 4) return __ldg(reinterpret_cast<const float4*>(row) + j);
  return make_float4(__ldg(row + j), 0.f, 0.f, 0.f);
}
template <int VEC>
__device__ __forceinline__ void st_col(float* row, long long j, float4 v) {
  if constexpr (VEC == 4)
    __stcs(reinterpret_cast<float4*>(row) + j, v);
  else
    __stcs(row + j, v.x);
}

__device__ __forceinline__ float dot4(float4 a, float4 b, float acc) {
  acc = fmaf(a.x, b.x, acc);
  acc = fmaf(a.y, b.y, acc);
  acc = fmaf(a.z, b.z, acc);
  return fmaf(a.w, b.w, acc);
}
__device__ __forceinline__ float4 scale4(float s, float4 v) { return make_float4(s * v.x, s * v.y, s * v.z, s * v.w); }

template <int VEC>
__global__ void __launch_bounds__(kCombineThreads) combine_backward_kernel(const float* __restrict__ y,
                                                                           const float* __restrict__ w,
                                                                           const float* __restrict__ d_out, long long P,
                                                                           int K, long long H, float* __restrict__ d_y,
                                                                           float* __restrict__ d_w) {
  pdl_trigger();
  pdl_wait();
  const long long p = blockIdx.x * static_cast<long long>(kCombineThreads / 32) + (threadIdx.x >> 5);
  if (p >= P) return;
  const int lane = threadIdx.x & 31;
  const long long ncol = H / VEC;
  const float* yrow = y + p * H;
  const float* drow = d_out + (p / K) * H;
  float* orow = d_y + p * H;
  const float wk = __ldg(w + p);
  float acc = 0.f;
  for (long long j0 = lane; j0 < ncol; j0 += 32 * kColsInFlight) {
    float4 yv[kColsInFlight], dv[kColsInFlight];
#pragma unroll
    for (int u = 0; u < kColsInFlight; ++u) {
      const long long j = j0 + 32 * u;
      if (j < ncol) {
        yv[u] = ld_col<VEC>(yrow, j);
        dv[u] = ld_col_l2<VEC>(drow, j);
      }
    }
#pragma unroll
    for (int u = 0; u < kColsInFlight; ++u) {
      const long long j = j0 + 32 * u;
      if (j < ncol) {
        acc = dot4(yv[u], dv[u], acc);
        st_col<VEC>(orow, j, scale4(wk, dv[u]));
      }
    }
  }
  acc = warp_sum(acc);
  if (lane == 0) d_w[p] = acc;
}

// act(g) and act'(g) together (SiLU, or the tanh GELU with sqrt(2/pi) and 0.044715).
__device__ __forceinline__ void act_and_grad(int act, float g, float& a, float& da) {
  if (act == MOE_ACT_SILU) {
    const float s = 1.0f / (1.0f + expf(-g));
    a = g * s;
    da = s * (1.0f + g * (1.0f - s));
  } else {
    const float c = 0.7978845608028654f, k3 = 0.044715f;
    const float th = tanhf(c * (g + k3 * g * g * g));
    a = 0.5f * g * (1.0f + th);
    da = 0.5f * (1.0f + th) + 0.5f * g * (1.0f - th * th) * c * (1.0f + 3.0f * k3 * g * g);
  }
}

template <int VEC>
__device__ __forceinline__ void act_up_cols(int act, float4 g, float4 u, float4 dh, float4& dg, float4& du) {
  float a, da;
  act_and_grad(act, g.x, a, da);
  dg.x = dh.x * u.x * da;
  du.x = dh.x * a;
  if constexpr (VEC == 4) {
    act_and_grad(act, g.y, a, da);
    dg.y = dh.y * u.y * da;
    du.y = dh.y * a;
    act_and_grad(act, g.z, a, da);
    dg.z = dh.z * u.z * da;
    du.z = dh.z * a;
    act_and_grad(act, g.w, a, da);
    dg.w = dh.w * u.w * da;
    du.w = dh.w * a;
  }
}

// Elementwise over the P x I/VEC column groups; each thread takes two groups
// (its index and the one a grid further on) per iteration, loads first.
template <int VEC>
__global__ void __launch_bounds__(kBwdThreads) act_up_backward_kernel(const float* __restrict__ gate_up,
                                                                      const float* __restrict__ d_h, long long P,
                                                                      long long I, int act,
                                                                      float* __restrict__ d_gate_up) {
  pdl_trigger();
  pdl_wait();
  const long long ncol = I / VEC, total = P * ncol;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i0 = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i0 < total; i0 += 2 * stride) {
    float4 g[2], u[2], dh[2];
    long long p[2], j[2];
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const long long idx = i0 + s * stride;
      if (idx < total) {
        p[s] = idx / ncol;
        j[s] = idx - p[s] * ncol;
        const float* row = gate_up + p[s] * 2 * I;
        g[s] = ld_col<VEC>(row, j[s]);
        u[s] = ld_col<VEC>(row + I, j[s]);
        dh[s] = ld_col<VEC>(d_h + p[s] * I, j[s]);
      }
    }
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      if (i0 + s * stride < total) {
        float4 dg, du;
        act_up_cols<VEC>(act, g[s], u[s], dh[s], dg, du);
        float* orow = d_gate_up + p[s] * 2 * I;
        st_col<VEC>(orow, j[s], dg);
        st_col<VEC>(orow + I, j[s], du);
      }
    }
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <typename Kern, typename... Args>
cudaError_t launch_pdl(const Ctx& c, Kern kern, dim3 grid, int threads, Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads);
  cfg.stream = c.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = c.pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

}  // namespace

cudaError_t launch_combine_backward(const Ctx& c, const float* y, const float* w, const float* d_out, long long T,
                                    int K, long long H, float* d_y, float* d_w) {
  if (T <= 0) return cudaSuccess;
  const long long P = T * K, per = kCombineThreads / 32;
  if ((P + per - 1) / per > 0x7fffffffLL) return cudaErrorInvalidValue;
  const bool vec = H % 4 == 0 && aligned16(y) && aligned16(d_out) && aligned16(d_y);
  KernelScope ks(c, "combine_backward");
  const dim3 grid(static_cast<unsigned>((P + per - 1) / per));
  return vec ? launch_pdl(c, combine_backward_kernel<4>, grid, kCombineThreads, y, w, d_out, P, K, H, d_y, d_w)
             : launch_pdl(c, combine_backward_kernel<1>, grid, kCombineThreads, y, w, d_out, P, K, H, d_y, d_w);
}

// A grid of whole waves: the SM count times the CTAs of `kern` one SM holds.
template <typename Kern>
unsigned wave_grid(const Ctx& c, Kern kern, long long items) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kBwdThreads, 0) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  const long long want = (items + kBwdThreads - 1) / kBwdThreads;
  return static_cast<unsigned>(std::max(1LL, std::min(want, static_cast<long long>(c.num_sms) * per_sm)));
}

cudaError_t launch_act_up_backward(const Ctx& c, const float* gate_up, const float* d_h, long long P, long long I,
                                   int act, float* d_gate_up) {
  if (P <= 0) return cudaSuccess;
  const bool vec = I % 4 == 0 && aligned16(gate_up) && aligned16(d_h) && aligned16(d_gate_up);
  const long long items = P * (vec ? I / 4 : I);
  KernelScope ks(c, "act_up_backward");
  if (vec)
    return launch_pdl(c, act_up_backward_kernel<4>, dim3(wave_grid(c, act_up_backward_kernel<4>, items)), kBwdThreads,
                      gate_up, d_h, P, I, act, d_gate_up);
  return launch_pdl(c, act_up_backward_kernel<1>, dim3(wave_grid(c, act_up_backward_kernel<1>, items)), kBwdThreads,
                    gate_up, d_h, P, I, act, d_gate_up);
}

}  // namespace moe
