// Host-side launchers of the MoE kernels (internal to libmoe; the public
// interface is include/moe.h).  Every launcher enqueues on ctx.stream and
// returns cudaSuccess or the launch error.
#pragma once

#include "common.cuh"

namespace moe {

// How a token's experts are chosen and weighted.
struct RouteCfg {
  int E, K, renorm;
  int gating;       // MOE_GATING_SOFTMAX | MOE_GATING_SIGMOID
  int n_groups;     // > 1: group-limited selection (E % n_groups == 0, n_groups <= 32)
  int topk_groups;  // groups kept
};


// Softmax + top-K (+renorm) per token from logits in global memory, one warp
// per token.  Adds the optional bias to the logits in place; with w_s also
// writes shared_gate[t] = sigmoid(w_s . x[t]).
// `nparts` partial logit arrays of T*E floats, part_stride apart starting at
// `parts`, are summed in order into `logits` first.
cudaError_t launch_router_topk(const Ctx& c, const float* parts, int nparts, size_t part_stride, float* logits,
                               const float* bias, int T, const RouteCfg& rc, int32_t* ids, float* w,
                               const void* x, int x_dtype, const void* w_s, int w_dtype, int H, float* shared_gate);

// Router in one launch for small batches: logits (+ the shared-gate row when
// w_s != nullptr) by clusters of 8 CTAs, then softmax + top-K (+renorm) per token.
cudaError_t launch_router_fused(const Ctx& c, const void* x, int x_dtype, const void* W, const void* w_s,
                                int w_dtype, const float* bias, int T, int H, const RouteCfg& rc,
                                float* logits, int32_t* ids, float* w, float* shared_gate);

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
  int ksplit = 1;          // single mode without row_map/row_scale only: K split into ranges whose
  size_t part_stride = 0;  // f32 results go to out_f32 + range * part_stride (summed by the caller)
  // Row gather (the routed gate/up projection): A row r is row gather_rows[r] / gather_div of A_src
  // [rows_src, Kdim]; rows_A then counts the logical rows.  nullptr: A is read as it is.
  const int32_t* gather_rows = nullptr;
  int gather_div = 1;
  const __nv_bfloat16* A_src = nullptr;
  int64_t rows_src = 0;
};
cudaError_t launch_grouped_gemm(const Ctx& c, const GemmArgs& a);
bool pair_gemm_enabled();  // moe_set_pair_gemm

// The number of K ranges a split request really produces for a reduction of
// Kdim: at most one per 64-wide k-block, and no empty range.  The caller sums
// exactly this many partial results.
inline int effective_ksplit(int requested, int Kdim) {
  const int nkb = (Kdim + 63) / 64;
  const int want = std::max(1, std::min(requested, nkb));
  const int per = (nkb + want - 1) / want;
  return (nkb + per - 1) / per;
}

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
// out[t] = sum_k w[t,k] y_slots[t*K+k] in f32 (bf16 expert outputs), + y_shared[t] (f32), as bf16.
cudaError_t launch_combine_weighted(const Ctx& c, const __nv_bfloat16* y_slots, const float* w, const float* y_shared,
                                    int T, int K, int H, void* out);
cudaError_t launch_combine(const Ctx& c, const float* y_slots, const float* y_shared, int T, int K, int H,
                           void* out, int out_dtype);

// GGML Q8_0 blocks -> int8 plane + fp16 scale plane.
// Backward of the combine and of act(gate) * up (backward.cu).
cudaError_t launch_combine_backward(const Ctx& c, const float* y, const float* w, const float* d_out, long long T,
                                    int K, long long H, float* d_y, float* d_w);
cudaError_t launch_act_up_backward(const Ctx& c, const float* gate_up, const float* d_h, long long P, long long I,
                                   int act, float* d_gate_up);
cudaError_t launch_q6_k_split(const Ctx& c, const void* blocks, int64_t rows, int64_t cols, void* q, void* scales);
cudaError_t launch_q8_0_split(const Ctx& c, const void* blocks, int64_t rows, int64_t cols, int8_t* q,
                              void* scales);


// The whole layer for a small batch in one cooperative launch (decode_fused.cu):
// router, top-K, permutation, gate/up, down and combine as phases of one
// persistent grid separated by grid barriers.  Writes the same workspace
// outputs as the step-by-step path (logits, ids, w, shared_gate, counts,
// offsets, sorted_pairs, pair_pos, h, h_s, y_slots, y_s) and `out`.
constexpr int kMaxDecodeT = 64;
constexpr int kMaxDecodePairs = 2048;
struct DecodeLayer {
  const void* x;
  int x_dtype;
  const void* router;
  int router_dtype;
  const float* bias;   // router bias or nullptr
  const void* w_s;     // shared-gate row or nullptr
  int T, H, E, K, I, Is, act, renorm, w_dtype;
  RouteCfg rc;  // E, K, renorm repeated with the gating and groups
  const void *gate, *up, *down, *gate_scale, *up_scale, *down_scale;
  const void *sh_gate, *sh_up, *sh_down, *sh_gate_scale, *sh_up_scale, *sh_down_scale;
  float* router_parts;  // decode_router_parts_floats(...) floats
  float* logits;
  int32_t* ids;
  float* w;
  float* shared_gate;
  int32_t* counts;
  int32_t* offsets;
  int32_t* sorted_pairs;
  int32_t* pair_pos;
  float* h;
  float* h_s;
  float* y_slots;
  float* y_s;
  void* out;
  void* stream_sync;  // decode_stream_sync_bytes() of workspace for the gate/up + down stream (nullptr: two phases)
};
size_t decode_router_parts_floats(int T, int H, int E, bool shared_gate);
constexpr size_t decode_stream_sync_bytes() { return 4 * (1 + 257); }
int stream_path_mode();  // moe_set_decode_stream: 0 two phases, 1 the stream (f32 / bf16 / Q8_0 weights)
cudaError_t launch_decode_layer(const Ctx& c, const DecodeLayer& L);


// Top-K selection (from the router GEMM's output), stable permutation and
// x-row gather of the tensor-core path in one cooperative launch
// (prefill_front.cu).  Writes the same workspace regions as
// router_topk + permute + gather_rows, and the same values.
constexpr int kMaxFrontCtas = 256;
struct PrefillFront {
  const float* parts;  // split-K partial logits (nparts > 0), part_stride apart; else logits already complete
  int nparts;
  size_t part_stride;
  float* logits;
  const float* bias;
  int T, E, K, renorm, H;
  RouteCfg rc;
  int32_t* ids;
  float* w;
  const __nv_bfloat16* x;
  const __nv_bfloat16* w_s;  // shared-gate row or nullptr
  float* shared_gate;
  int32_t* counts;
  int32_t* offsets;
  int32_t* sorted_pairs;
  int32_t* pair_pos;
  __nv_bfloat16* x_perm;
  int32_t* hist;  // kMaxFrontCtas * E ints of scratch
};
cudaError_t launch_prefill_front(const Ctx& c, const PrefillFront& f);

}  // namespace moe
