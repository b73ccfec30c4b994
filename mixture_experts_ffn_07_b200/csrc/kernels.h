// Host-side launchers of the MoE kernels (internal to libmoe; the public
// interface is include/moe.h).  Every launcher enqueues on ctx.stream and
// returns cudaSuccess or the launch error.
#pragma once

#include "common.cuh"

namespace moe {

// Router logits on CUDA cores: logits[t, r] = x[t] . W[r] for rows r in
// [0, E) of the router and, when w_s != nullptr, shared_gate[t] =
// sigmoid(x[t] . w_s).  rows_from_router = false computes only the w_s row.
cudaError_t launch_router_logits(const Ctx& c, const void* x, int x_dtype, const void* W, const void* w_s,
                                 int w_dtype, int T, int H, int E, bool rows_from_router, float* logits,
                                 float* shared_gate);

// Softmax + top-K (+renorm) per token, one warp per token.  Adds the optional
// bias to the logits in place; writes ids and weights.
cudaError_t launch_router_topk(const Ctx& c, float* logits, const float* bias, int T, int E, int K, int renorm,
                               int32_t* ids, float* w);

// Single-CTA stable counting sort of the P pair ids by expert.
cudaError_t launch_permute(const Ctx& c, const int32_t* ids, int P, int E, int32_t* counts, int32_t* offsets,
                           int32_t* sorted_pairs, int32_t* pair_pos);

// X_perm[r] = x[sorted_pairs[r] / K] for r < offsets[E] (bf16 rows of H).
cudaError_t launch_gather_rows(const Ctx& c, const __nv_bfloat16* x, const int32_t* sorted_pairs,
                               const int32_t* offsets, int E, int K, int P, int H, __nv_bfloat16* x_perm);

// Grouped GEMM on tcgen05 tensor cores.  A: [rows_A, Kdim] bf16 row-major.
// Groups g in [0, G): rows [off[g], off[g+1]) of A (off == nullptr: one group
// of rows_A rows).  B0/B1: [G*N, Kdim] bf16 (group g owns rows g*N..).
//  dual = true : D = [A B0^T | A B1^T] per 128-column tile; out_bf16[row, n] = act(D0) * D1
//  dual = false: out_f32[dest, n] = scale * (A B0^T)[row, n],
//                dest = row_map ? row_map[row] : row, scale = row_scale ? row_scale[dest] : 1
struct GemmArgs {
  const __nv_bfloat16* A;
  int64_t rows_A;
  int Kdim;
  const __nv_bfloat16* B0;
  const __nv_bfloat16* B1;
  int N;
  int G;
  const int32_t* offsets;
  int max_rows;            // host bound on the rows actually used (sizes the grid)
  bool dual;
  int act;
  __nv_bfloat16* out_bf16;
  float* out_f32;
  const int32_t* row_map;
  const float* row_scale;
  const char* name;        // trace label
};
cudaError_t launch_grouped_gemm(const Ctx& c, const GemmArgs& a);

// Weight-streaming expert FFN (any T; f32/bf16 activations, f32/bf16/Q8_0 weights).
// Groups as above (offsets == nullptr: one group of rows [0, T) with identity rows).
// h[r, i] = act(W_gate[e,i] . x[tok(r)]) * (W_up[e,i] . x[tok(r)]), tok(r) = pairs ? pairs[r] / K : r.
cudaError_t launch_stream_gate_up(const Ctx& c, const void* x, int x_dtype, int T, int H, int I, int K,
                                  const void* gate, const void* up, const void* gate_scale, const void* up_scale,
                                  int w_dtype, const int32_t* offsets, int E, const int32_t* pairs, int rows_bound,
                                  int act, float* h);
// y[dest, j] = scale * (W_down[e,j] . h[r]), dest = pairs ? pairs[r] : r, scale = row_scale ? row_scale[dest] : 1.
cudaError_t launch_stream_down(const Ctx& c, const float* h, int I, int H, const void* down, const void* down_scale,
                               int w_dtype, const int32_t* offsets, int E, const int32_t* pairs, int rows_bound,
                               const float* row_scale, float* y);

// out[t, :] = sum_k y_slots[t*K + k, :] (+ y_shared[t, :]) -> out_dtype.
cudaError_t launch_combine(const Ctx& c, const float* y_slots, const float* y_shared, int T, int K, int H,
                           void* out, int out_dtype);

// GGML Q8_0 blocks -> int8 plane + fp16 scale plane.
cudaError_t launch_q8_0_split(const Ctx& c, const void* blocks, int64_t rows, int64_t cols, int8_t* q,
                              void* scales);

}  // namespace moe
