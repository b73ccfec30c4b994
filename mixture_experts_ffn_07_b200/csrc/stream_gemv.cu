// Standalone weight-streaming kernels for the expert FFN when the tensor-core
// path does not apply (f32 or Q8_0 weights, or small bf16 batches) and the
// whole layer does not run as one fused decode kernel: one launch per
// operation (gate/up, down).  The GEMV itself is in stream_core.cuh.
#include "stream_core.cuh"

namespace moe {

namespace {

using namespace stream;

struct Launch {
  const int32_t* offsets;  // [E+1] rows per expert (nullptr: one group of T rows)
  int E, T;
};

template <typename AT, int WK, bool DUAL>
__global__ void __launch_bounds__(kThreads, 1) stream_gemv_kernel(const Phase ph, const Launch a) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int s_expert[kMaxGroups], s_first[kMaxGroups], s_count[kMaxGroups], s_poff[kMaxGroups + 1];
  __shared__ long long s_coff[kMaxGroups + 1];
  __shared__ int s_arow[kMaxTok], s_dest[kMaxTok];
  __shared__ float s_scale[kMaxTok];
  __shared__ float s_part[kMaxUnits * kMaxTok * 2];
  __shared__ int s_warp[8];
  __shared__ int s_n;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_trigger();
  pdl_wait();
  if (threadIdx.x < 256) {  // touched experts in order, with their rows
    const int e = threadIdx.x;
    const bool f = a.offsets ? (e < a.E && a.offsets[e + 1] > a.offsets[e]) : (e == 0);
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
      s_first[i] = a.offsets ? a.offsets[e] : 0;
      s_count[i] = a.offsets ? a.offsets[e + 1] - a.offsets[e] : a.T;
    }
    if (threadIdx.x == 0) s_n = n;
  }
  __syncthreads();
  const Tables tb{s_expert, s_first, s_count, s_poff, s_coff, s_n};
  if (warp == 0) build_prefix(tb, ph);
  __syncthreads();
  int p0, p1;
  cta_pairs(tb, ph, p0, p1);
  const Smem sm{smem, s_arow, s_dest, s_scale, s_part};
  run_phase<AT, WK, DUAL, kMaxTok>(ph, tb, p0, p1, sm);
}

template <typename AT, int WK, bool DUAL>
cudaError_t launch_typed(const Ctx& c, const Phase& ph, const Launch& a, const char* name) {
  auto kern = stream_gemv_kernel<AT, WK, DUAL>;
  if (ph.plan[0].xrow_bytes > kMaxTokenRowBytes) return cudaErrorInvalidValue;
  const int smem = ph.plan[0].TS * ph.plan[0].xrow_bytes;
  const cudaError_t e = allow_dynamic_smem(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  KernelScope ks(c, name);
  return launch_kernel(c, kern, dim3(c.num_sms), dim3(kThreads), smem, ph, a);
}

}  // namespace

cudaError_t launch_stream_gate_up(const Ctx& c, const void* x, int x_dtype, int T, int H, int I, int K,
                                  const void* gate, const void* up, const void* gate_scale, const void* up_scale,
                                  int w_dtype, const int32_t* offsets, int E, const int32_t* pairs, int rows_bound,
                                  int act, float* h) {
  if (rows_bound <= 0) return cudaSuccess;
  Phase ph{};
  GroupSrc& s = ph.src[0];
  s.w0 = static_cast<const uint8_t*>(gate);
  s.w1 = static_cast<const uint8_t*>(up);
  s.s0 = static_cast<const uint8_t*>(gate_scale);
  s.s1 = static_cast<const uint8_t*>(up_scale);
  s.act = static_cast<const uint8_t*>(x);
  s.out = h;
  s.act_via_pairs = pairs != nullptr;
  ph.pairs = pairs;
  ph.K = K;
  ph.act_fn = act;
  const Launch a{offsets, offsets ? E : 1, offsets ? 0 : rows_bound};
  const int wk = wk_gate_up(w_dtype);
  // an expert owns at most one row per token: at most P / K rows
  const int max_tok = offsets ? std::max(1, rows_bound / std::max(1, K)) : rows_bound;
  ph.plan[0] = ph.plan[1] = make_plan(wk, true, H, I, x_dtype == MOE_F32 ? 4 : 2, max_tok);
  const char* n = "stream_gate_up";
  if (x_dtype == MOE_F32) {
    if (wk == WK_F32) return launch_typed<float, WK_F32, true>(c, ph, a, n);
    if (wk == WK_BF16) return launch_typed<float, WK_BF16, true>(c, ph, a, n);
    if (wk == WK_Q4K) return launch_typed<float, WK_Q4K, true>(c, ph, a, n);
    return launch_typed<float, WK_Q8, true>(c, ph, a, n);
  }
  if (wk == WK_F32) return launch_typed<__nv_bfloat16, WK_F32, true>(c, ph, a, n);
  if (wk == WK_BF16) return launch_typed<__nv_bfloat16, WK_BF16, true>(c, ph, a, n);
  if (wk == WK_Q4K) return launch_typed<__nv_bfloat16, WK_Q4K, true>(c, ph, a, n);
  return launch_typed<__nv_bfloat16, WK_Q8, true>(c, ph, a, n);
}

cudaError_t launch_stream_down(const Ctx& c, const float* h, int I, int H, const void* down, const void* down_scale,
                               int w_dtype, const int32_t* offsets, int E, const int32_t* pairs, int rows_bound,
                               const float* row_scale, float* y) {
  if (rows_bound <= 0) return cudaSuccess;
  Phase ph{};
  GroupSrc& s = ph.src[0];
  s.w0 = static_cast<const uint8_t*>(down);
  s.s0 = static_cast<const uint8_t*>(down_scale);
  s.act = reinterpret_cast<const uint8_t*>(h);
  s.out = y;
  s.row_scale = row_scale;
  s.out_via_pairs = 1;
  s.scale_via_pairs = 1;
  ph.pairs = pairs;
  ph.K = 1;
  const Launch a{offsets, offsets ? E : 1, offsets ? 0 : rows_bound};
  const int wk = wk_down(w_dtype);
  ph.plan[0] = ph.plan[1] = make_plan(wk, false, I, H, 4, kMaxTok);
  const char* n = "stream_down";
  if (wk == WK_F32) return launch_typed<float, WK_F32, false>(c, ph, a, n);
  if (wk == WK_BF16) return launch_typed<float, WK_BF16, false>(c, ph, a, n);
  if (wk == WK_Q4K) return launch_typed<float, WK_Q4K, false>(c, ph, a, n);
  if (wk == WK_Q6K) return launch_typed<float, WK_Q6K, false>(c, ph, a, n);
  return launch_typed<float, WK_Q8, false>(c, ph, a, n);
}

}  // namespace moe
