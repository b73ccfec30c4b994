/*
 * libmoe -- a Mixture-of-Experts FFN layer for NVIDIA B200 (sm_100a).
 *
 * The layer: router logits, softmax + top-K (+ renormalisation), dispatch of
 * each token to its K experts, per expert act(x W_gate^T) * (x W_up^T) then
 * W_down, a routing-weighted combine, and an optional sigmoid-gated shared
 * expert.  Notation: T tokens, H hidden, E experts, K = top_k, I expert
 * intermediate, Is shared intermediate, P = T*K (token, slot) pairs with pair
 * id p = t*K + k.
 *
 * Conventions for every entry point
 *  - Pointers to tensors are DEVICE pointers owned by the caller (moe_layer_host
 *    is the one exception, see there).  The library never allocates, frees or
 *    retains device memory; scratch comes from the caller's workspace.
 *  - Tensors are dense and row-major.  Weights are stored out x in (the
 *    nn.Linear convention): rows are contiguous along the input dimension.
 *  - Calls are asynchronous on `stream` (0 = legacy default stream): they
 *    return after enqueueing.  Arguments are checked on the host first; any
 *    error return means nothing was launched and nothing was written.
 *  - Device-side problems (an expert id out of range, a pipeline wait that ran
 *    past its time limit) do not trap: kernels record a status word that
 *    moe_last_device_status() reads.
 *  - Limits: 1 <= E <= 256, 1 <= K <= min(E, 32), H, I and Is multiples of 32,
 *    T <= 2^20.  T == 0 is valid and does nothing (pointers may then be NULL).
 *    Every tensor pointer must be 16-byte aligned.  Outputs may not alias inputs.
 *  - The library keeps no per-call state; it is safe to call from several host
 *    threads on different streams.
 *
 * Citations name the page (crate and file) and the function the operation
 * follows.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* a cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* a size, flag or pointer is out of contract */
  MOE_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. H not a multiple of 32) */
  MOE_ERR_WORKSPACE = 3,   /* workspace smaller than moe_workspace_bytes() */
  MOE_ERR_CUDA = 4,        /* a CUDA runtime call failed (launch, attribute, copy) */
  MOE_ERR_TIMEOUT = 5,     /* device: a pipeline wait ran past its limit (kernel gave up cleanly) */
  MOE_ERR_DEVICE_INDEX = 6 /* device: an expert id outside [0, E) reached the permutation */
} moe_status;

/* Storage formats.  MOE_Q4_K and MOE_Q4_K_Q6_K are expert-weight formats only
 * (the k-quant stacks of the Metal MoE providers, ferrum-kernels vnext MoE:
 * "q4k" for all projections, "q4k_q6k" for Q4_K gate/up with Q6_K down). */
typedef enum { MOE_F32 = 0, MOE_BF16 = 1, MOE_Q8_0 = 2, MOE_Q4_K = 3, MOE_Q4_K_Q6_K = 4 } moe_dtype;

/* SiLU(g) = g / (1 + e^-g)  (hf2q qwen35/gpu_ffn.rs, silu_mul_cpu);
 * GELU_TANH(g) = 0.5 g (1 + tanh(sqrt(2/pi) (g + 0.044715 g^3)))
 * (mlx-native moe_dispatch.rs, fused_gelu_mul and its test oracle cpu_gelu). */
typedef enum { MOE_ACT_SILU = 0, MOE_ACT_GELU_TANH = 1 } moe_act;

/* Gate values from the (biased) logits l_e: softmax over all E experts
 * (hf2q softmax_topk_renorm_cpu), or sigmoid 1/(1+e^-l_e) per expert (the
 * other GatingFunction ferrox-models decoder.rs passes to its routers). */
typedef enum { MOE_GATING_SOFTMAX = 0, MOE_GATING_SIGMOID = 1 } moe_gating;

typedef struct moe_desc {
  int32_t T, H, E, I, top_k;
  int32_t act;             /* moe_act, used by routed and shared experts */
  int32_t renormalize;     /* 1: selected gate values divided by their sum; 0: the gate values themselves */
  int32_t act_dtype;       /* MOE_F32 | MOE_BF16: x and out */
  int32_t w_dtype;         /* MOE_F32 | MOE_BF16 | MOE_Q8_0 | MOE_Q4_K | MOE_Q4_K_Q6_K: expert and shared
                              projections (the k-quant formats need H, I and shared_I multiples of 256) */
  int32_t router_dtype;    /* MOE_F32 | MOE_BF16: router W and the shared-gate vector w_s */
  int32_t has_router_bias; /* 1: logits += b_e before selection (ferrox-models decoder.rs, gpt_oss_ffn) */
  int32_t shared_I;        /* 0: no shared expert */
  int32_t has_shared_gate; /* 1: shared output scaled by sigmoid(w_s . x); 0: scale 1 */
  int32_t gating;          /* moe_gating (0: softmax) */
  int32_t n_groups;        /* 0 or 1: plain top-K.  > 1: group-limited selection (ferrox-models decoder.rs,
                              route_top_k_grouped): the experts form n_groups contiguous groups of E/n_groups,
                              a group scores its largest logit and only the topk_groups best groups (lower
                              index on ties) are eligible.  E % n_groups == 0, n_groups <= 32. */
  int32_t topk_groups;     /* groups kept: 1 <= topk_groups <= n_groups, top_k <= topk_groups * E / n_groups */
} moe_desc;

/*
 * Weights.  Shapes (out x in):
 *   router [E,H], router_bias [E] f32, gate [E,I,H], up [E,I,H], down [E,H,I],
 *   sh_gate [Is,H], sh_up [Is,H], sh_down [H,Is], sh_gate_w [H].
 * For w_dtype == MOE_Q8_0 the projection pointers hold int8 quants with the
 * same shapes and the *_scale pointers hold one fp16 scale per 32 consecutive
 * inputs ([E,I,H/32], [E,H,I/32], [Is,H/32], [H,Is/32]); value = scale * q.
 * moe_q8_0_split() converts GGML Q8_0 blocks into this split form.
 * For MOE_Q4_K every projection holds GGML Q4_K blocks in place, row by row:
 * a row of n inputs is n/256 blocks of 144 bytes {fp16 d; fp16 dmin;
 * u8 scales[12]; u8 qs[128]}, so gate is [E,I,H/256,144] bytes; the *_scale
 * pointers are unused.  For MOE_Q4_K_Q6_K gate/up (and sh_gate/sh_up) are Q4_K
 * as above and down / sh_down hold GGML Q6_K blocks {u8 ql[128]; u8 qh[64];
 * i8 scales[16]; fp16 d} in the split form of moe_q6_k_split(): down is
 * [E*H, I/256, 192] bytes (ql then qh of each block) and down_scale
 * [E*H, srow] bytes with srow = ceil(18 * I/256 / 16) * 16: the 16 scales of
 * every block of the row, then the fp16 d of every block, then zeros.
 * All weight pointers are 16-byte aligned.  Unused pointers may be NULL.
 */
typedef struct moe_weights {
  const void* router;
  const float* router_bias;
  const void* gate;
  const void* up;
  const void* down;
  const void* sh_gate;
  const void* sh_up;
  const void* sh_down;
  const void* sh_gate_w;
  const void* gate_scale;
  const void* up_scale;
  const void* down_scale;
  const void* sh_gate_scale;
  const void* sh_up_scale;
  const void* sh_down_scale;
} moe_weights;

/* Human-readable name of a status code (static string). */
const char* moe_status_string(moe_status s);

/* Library version string (static). */
const char* moe_version(void);

/*
 * Bytes of caller-provided device workspace moe_layer needs for `d`: linear in
 * T for fixed sizes, plus the bf16 router's split-K partial logits (at most
 * 20480*E*4 bytes) and 256*E*4 bytes of per-CTA expert counts for T > 64, or
 * for 1 <= T <= 64 on the streaming path the fused decode kernel's per-chunk
 * partial logits (ceil(H/1024)*T*(E+1)*4 bytes), in 256-byte aligned regions.  Returns 0 for an invalid
 * descriptor.  moe_route, moe_expert_ffn and moe_combine need no more than this.
 */
size_t moe_workspace_bytes(const moe_desc* d);

/*
 * Where moe_layer leaves its routing inside the workspace: byte offsets from
 * `ws` (each 256-byte aligned) of logits [T,E] f32 (with the bias),
 * topk_ids [T,K] int32, topk_w [T,K] f32, shared_gate [T] f32 (written only
 * when shared_I > 0 and has_shared_gate), counts [E] int32, offsets [E+1]
 * int32, sorted_pairs [P] int32 and pair_pos [P] int32, with the meanings of
 * moe_route and moe_permute.  Readable once the stream has passed the
 * moe_layer call.  Host only.  MOE_ERR_INVALID_ARG for an invalid descriptor
 * or r == NULL.
 */
typedef struct moe_ws_regions {
  size_t logits, topk_ids, topk_w, shared_gate, counts, offsets, sorted_pairs, pair_pos;
} moe_ws_regions;
moe_status moe_workspace_regions(const moe_desc* d, moe_ws_regions* r);

/*
 * Router: logits, softmax, top-K with renormalisation.
 * (hf2q qwen35/gpu_ffn.rs, softmax_topk_renorm_cpu and dispatch_moe_softmax_topk;
 *  ferrum-kernels vnext_ops/moe.rs, route kernel, one 32-thread group per token)
 *  x        [T,H] act_dtype
 *  logits   [T,E] f32 out: x W_r^T (+ b), the values selection compared
 *  topk_ids [T,K] int32 out: experts in order (logit desc, index asc)
 *  topk_w   [T,K] f32 out: the selected experts' gate values (moe_gating), divided by their sum
 *           when renormalize
 *  shared_gate [T] f32 out: sigmoid(w_s . x); required iff shared_I > 0 and has_shared_gate
 *  ws, ws_bytes: optional workspace (NULL, or >= moe_workspace_bytes(d)).  With it,
 *           a bf16 batch splits the logits GEMM over the hidden dimension into
 *           partial sums added in a fixed order (the split moe_layer uses, so the
 *           logits, and hence the selection, are identical to moe_layer's);
 *           without it the GEMM is not split.
 */
moe_status moe_route(const moe_desc* d, const void* x, const moe_weights* w, float* logits, int32_t* topk_ids,
                     float* topk_w, float* shared_gate, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Histogram, exclusive scan and stable permutation of the P pairs by expert
 * (DS4Server qwen_mtplx.rs, gather_sort: argsort of the flat expert ids and
 *  its inverse; ferrox-models decoder.rs, moe_ffn_batch buckets in token order).
 *  topk_ids     [P] int32 in
 *  counts       [E] int32 out: pairs routed to each expert
 *  offsets      [E+1] int32 out: exclusive prefix sum, offsets[E] = P
 *  sorted_pairs [P] int32 out: pair ids grouped by expert, ascending within an expert
 *  pair_pos     [P] int32 out: inverse, sorted_pairs[pair_pos[p]] = p
 * Ids outside [0,E) are skipped and reported as MOE_ERR_DEVICE_INDEX.
 */
moe_status moe_permute(const moe_desc* d, const int32_t* topk_ids, int32_t* counts, int32_t* offsets,
                       int32_t* sorted_pairs, int32_t* pair_pos, moe_stream_t stream);

/*
 * Routed experts: for every expert e and each of its rows r in
 * [offsets[e], offsets[e+1]) with pair p = sorted_pairs[r], token t = p / K:
 *   y_slots[p,:] = topk_w[p] * W_down[e] (act(W_gate[e] x_t) * (W_up[e] x_t))
 * (mlx-native moe_dispatch.rs, moe_dispatch per-expert loop; hf2q
 *  qwen35/gpu_ffn.rs, quantized_matmul_id gate/up, silu_mul, down;
 *  ferrum-kernels vnext_ops/moe.rs, routed_down_slots)
 *  y_slots [P,H] f32 out.  Uses ws (>= moe_workspace_bytes(d) bytes).
 */
moe_status moe_expert_ffn(const moe_desc* d, const void* x, const moe_weights* w, const int32_t* offsets,
                          const int32_t* sorted_pairs, const float* topk_w, float* y_slots, void* ws,
                          size_t ws_bytes, moe_stream_t stream);

/*
 * Combine: out[t,:] = sum_{k=0..K-1} y_slots[t*K+k,:] + s_t * shared(x_t), in
 * that order, in f32, then converted to act_dtype; s_t = shared_gate[t] or 1.
 * (mlx-native moe_dispatch.rs, moe_weighted_sum; hf2q qwen35/gpu_ffn.rs,
 *  moe_weighted_reduce and the sigmoid-gated shared expert)
 *  shared_gate [T] f32 from moe_route (ignored unless shared_I > 0 and has_shared_gate)
 *  out [T,H] act_dtype out.  Runs the shared expert first when shared_I > 0 (uses ws).
 */
moe_status moe_combine(const moe_desc* d, const float* y_slots, const void* x, const moe_weights* w,
                       const float* shared_gate, void* out, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * The whole layer in one call: route, permute, experts, shared expert, combine.
 * Picks the tensor-core path (tcgen05 grouped GEMMs) when x and the expert
 * weights are bf16 and T > 64, else the weight-streaming path.  The
 * streaming path stages whole token rows in shared memory and returns
 * MOE_ERR_UNSUPPORTED (also from moe_expert_ffn / moe_combine) when
 * H * sizeof(act) > 65536 or I * 4 > 65536 or shared_I * 4 > 65536.
 * On the tensor-core path each expert's output row is kept in bf16 and the
 * combine adds w_k * y_k in f32 in slot order (mlx-native moe_dispatch.rs,
 * moe_weighted_sum_seq_bf16_input), so the result may differ in the last bits
 * from moe_expert_ffn + moe_combine, whose f32 slot rows are weighted first.
 *  x [T,H] act_dtype in, out [T,H] act_dtype out, ws >= moe_workspace_bytes(d).
 */
moe_status moe_layer(const moe_desc* d, const void* x, const moe_weights* w, void* out, void* ws, size_t ws_bytes,
                     moe_stream_t stream);

/*
 * moe_layer with HOST activations: copies x_host (T*H elements of act_dtype)
 * into x_dev, runs moe_layer, copies out_dev back into out_host, all on
 * `stream` (one cudaMemcpyAsync per copy; pinned host memory makes them
 * asynchronous).  x_dev and out_dev are caller-owned device buffers of the
 * same size.  Returns after enqueueing; synchronise `stream` before reading
 * out_host.
 */
moe_status moe_layer_host(const moe_desc* d, const void* x_host, const moe_weights* w, void* out_host, void* x_dev,
                          void* out_dev, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * moe_layer for callers that cannot allocate device memory when they call the
 * layer: for example a host whose HBM is already handed out to its own pool,
 * code that must not pay cudaMalloc's implicit device synchronisation, or a
 * plain C caller with no allocator at hand.  The pages have no counterpart of
 * this entry point; it exists for such callers only.
 *
 * Same inputs, outputs and results as moe_layer, but the scratch is a static
 * device array of MOE_NOALLOC_SCRATCH_BYTES (32 MiB) inside libmoe, present on
 * every GPU that loads the library until the process exits; nothing is
 * allocated or freed.  Descriptors with moe_workspace_bytes(d) above that size
 * are rejected with MOE_ERR_WORKSPACE before anything is launched (every
 * decode batch, T <= 64, of the layer shapes this library is measured on fits).
 * The first call on a device looks up the array's device address with that
 * device current; make that first call before any stream capture.  All calls
 * share the one array and it keeps the previous call's contents (nothing in
 * it has to start at zero: each call writes every region before reading it),
 * so calls that can overlap on the GPU -- other streams, other host threads --
 * race on it: serialise them.
 */
#define MOE_NOALLOC_SCRATCH_BYTES (32u << 20)
moe_status moe_layer_noalloc(const moe_desc* d, const void* x, const moe_weights* w, void* out, moe_stream_t stream);

/*
 * Split GGML Q8_0 blocks ({fp16 d; int8 q[32]}, 34 bytes, along the input
 * dimension) of a [rows, cols] matrix into int8 quants [rows, cols] and fp16
 * scales [rows, cols/32], the form moe_weights expects for MOE_Q8_0.  A
 * one-time load step (the pages repack weights at load: hf2q qwen35/gpu_ffn.rs,
 * pre-cast to bf16; ferrox-models decoder.rs, MoePackedQ4Planes).
 */
moe_status moe_q8_0_split(const void* blocks, int64_t rows, int64_t cols, int8_t* q, void* scales,
                          moe_stream_t stream);

/*
 * Backward of the routing-weighted combine out[t,:] = sum_k w[t,k] y[t,k,:],
 * for a loss L with d_out = dL/dout given (mlx-native moe_dispatch.rs, the
 * backward kernels of moe_weighted_sum_seq):
 *   d_y[t,k,:] = w[t,k] d_out[t,:]          d_w[t,k] = sum_h y[t,k,h] d_out[t,h]
 *  y     [T,K,H] f32 device: the expert outputs BEFORE weighting (row t*K+k);
 *        moe_expert_ffn's y_slots are already weighted by topk_w
 *  w     [T,K]   f32 device: the routing weights
 *  d_out [T,H]   f32 device
 *  d_y   [T,K,H] f32 device out;  d_w [T,K] f32 device out
 * d_w is summed in a fixed order (the same bits on every run).  T == 0 does
 * nothing.  MOE_ERR_INVALID_ARG: T < 0, K < 1, H < 1, T or K > 2^31-1,
 * T*K > 2^33-1, a null pointer, or an output range that overlaps an input range.  Caller-owned
 * memory; asynchronous on `stream`.
 */
moe_status moe_combine_backward(int64_t T, int64_t K, int64_t H, const float* y, const float* w, const float* d_out,
                                float* d_y, float* d_w, moe_stream_t stream);

/*
 * Backward of h = act(gate) * up (mlx-native moe_dispatch.rs, the backward
 * kernel of moe_swiglu_seq, which writes both gradients into one buffer laid
 * out like its input):
 *   d_gate = d_h * up * act'(gate)          d_up = d_h * act(gate)
 *   act'(g) = s (1 + g (1 - s)), s = 1/(1+e^-g), for MOE_ACT_SILU;
 *   0.5 (1 + tanh z) + 0.5 g (1 - tanh^2 z) sqrt(2/pi) (1 + 3 * 0.044715 g^2),
 *   z = sqrt(2/pi) (g + 0.044715 g^3), for MOE_ACT_GELU_TANH
 *  gate_up   [P, 2I] f32 device: row p = [gate (I values) | up (I values)]
 *  d_h       [P, I]  f32 device
 *  d_gate_up [P, 2I] f32 device out: row p = [d_gate | d_up]
 * P == 0 does nothing.  MOE_ERR_INVALID_ARG: P < 0, I < 1, an unknown act, a
 * null pointer, or an output range that overlaps an input range.
 * Caller-owned memory; asynchronous on `stream`.
 */
moe_status moe_act_up_backward(int64_t P, int64_t I, int32_t act, const float* gate_up, const float* d_h,
                               float* d_gate_up, moe_stream_t stream);

/*
 * Split GGML Q6_K blocks (210 bytes {u8 ql[128]; u8 qh[64]; i8 scales[16];
 * fp16 d} per 256 inputs, along the input dimension) of a [rows, cols] matrix
 * into the 16-byte aligned form moe_weights expects for the down projections
 * of MOE_Q4_K_Q6_K: q [rows, cols/256, 192] bytes (ql, qh of each block) and
 * scales [rows, srow] bytes, srow = ceil(18 * cols/256 / 16) * 16 (the int8
 * scales of the row's blocks, then their fp16 d, then zero padding).  Every
 * byte is moved unchanged: a one-time load step (ferrum-kernels vnext MoE,
 * prepare_q6_expert_part, prepares the Q6_K expert planes at load).
 * blocks: device, any alignment; q and scales: device, 16-byte aligned,
 * caller-owned.  cols % 256 != 0, negative sizes, null pointers or unaligned
 * outputs: MOE_ERR_INVALID_ARG.  rows * cols == 0 does nothing.
 */
moe_status moe_q6_k_split(const void* blocks, int64_t rows, int64_t cols, void* q, void* scales,
                          moe_stream_t stream);

/*
 * Synchronises `stream`, then returns and clears the device status word of
 * the current device (MOE_OK, MOE_ERR_TIMEOUT, MOE_ERR_DEVICE_INDEX), or
 * MOE_ERR_CUDA if the synchronisation failed.
 */
moe_status moe_last_device_status(moe_stream_t stream);

/* ---- instrumentation (host side only; no device memory) ---- */

/* Total kernels this library has launched in this process. */
uint64_t moe_launch_count(void);

/* Per-kernel CUDA-event timing of later calls: on != 0 starts recording (and
 * clears earlier records), 0 stops.  Records are kept for up to 4096 launches. */
void moe_trace_enable(int on);

/* Synchronises the recorded events and copies up to `max` records: kernel name
 * (static string) and duration in milliseconds.  Returns the number of
 * records available. */
int moe_trace_read(const char** names, float* ms, int max);

/* Debug: per-wait time limit in SM clock cycles for the pipeline waits of the
 * tensor-core kernels (default 2^31, about a second); and a fault switch that
 * makes the TMA producer of the next grouped-GEMM launches skip one stage's
 * loads, so the consumer's wait runs out and MOE_ERR_TIMEOUT is reported.
 * Used by the failure-detection test; never set in normal use. */
void moe_debug_set_wait_limit(int64_t cycles);
void moe_debug_set_skip_stage(int enable);

/* Debug: CTA 0 of the cooperative kernels (the prefill front and the fused
 * decode layer) spins `cycles` SM cycles before its first grid-barrier
 * arrival (0: off).  With a wait limit below the delay the other CTAs give
 * up on that barrier and report MOE_ERR_TIMEOUT; CTA 0 still arrives, so the
 * barrier counter stays consistent for later launches.  Failure-detection
 * tests only. */
void moe_debug_set_barrier_delay(int64_t cycles);

/* How moe_layer runs a batch of 1..64 tokens on the weight-streaming path:
 * enable = 1 (default) as one cooperative kernel ("decode_layer": router,
 * top-K, permutation, gate/up, down and combine as phases of one persistent
 * grid, one CTA per SM); 0 as the step-by-step launches.  Both write the same
 * workspace regions and `out`, and give the same routing.  If the cooperative
 * grid cannot be made resident, moe_layer takes the step-by-step path by
 * itself.  Process-wide; takes effect at the next call. */
void moe_set_fused_decode(int enable);

/* How moe_layer runs the selection, permutation and row gather of the
 * tensor-core path (bf16, T > 64, bf16 router with E % 32 == 0): enable = 1
 * (default) as one cooperative kernel ("route_permute_gather") after the
 * router GEMM; 0 as three launches (router_topk, permute, gather_rows).  Same
 * values either way; if the cooperative grid cannot be made resident,
 * moe_layer takes the three launches by itself.  Process-wide. */
void moe_set_fused_front(int enable);

/* How the tensor-core expert GEMMs run compute-bound launches (groups that
 * average at least 200 rows): enable = 1 (default) puts every group's full
 * 256-row tiles on pairs of CTAs (clusters of two SMs sharing one
 * tcgen05.mma.cta_group::2 of M = 256, N = 256) and the rows left in each group
 * on the single-CTA kernel; 0 runs all rows on the single-CTA kernel
 * (M = 128).  Same arithmetic per output element either way (one f32
 * accumulator per element, K in the same order), so the same bits.
 * Process-wide; takes effect at the next call. */
void moe_set_pair_gemm(int enable);

/* How the cooperative decode kernel (moe_set_fused_decode) runs gate/up and
 * down for f32, bf16 and Q8_0 weights: enable = 1 (default) as one stream of
 * work items (32 weight rows each, fed through the copy engine by one issuing
 * warp into a ring of stages per CTA, taken from a device-wide queue that
 * hands out all gate/up items, expert by expert, before the down items; a down
 * item waits only for its own expert's gate/up items); 0 as two phases
 * separated by a grid barrier, each CTA streaming a contiguous slice of the
 * rows, which is how the k-quant stacks always run (and Q8_0 whose H, I or
 * shared I is not a multiple of 256).  Same routing and the same values up to
 * the order of f32 additions.  Process-wide; takes effect at the next call. */
void moe_set_decode_stream(int enable);

/* How the tensor-core path feeds the routed gate/up GEMM its x rows in expert
 * order: enable = 0 (default) first copies them into a workspace array of
 * P x H bf16 rows (in the fused selection kernel, or a gather kernel), which
 * the GEMM reads with 128-row box loads; 1 gathers them inside the GEMM, each
 * pair's row straight from x by the copy engine (tile::gather4 loads of four
 * rows, 32 per 128-row tile and k-block), which saves the copy's traffic and
 * workspace but measured slower on B200 (the skewed layer's gate/up GEMM
 * 3.0 -> 7.4 ms: the copy engine's cost per small load bounds it).  Same values.
 * moe_workspace_bytes follows the current setting (the copy needs
 * P * H * 2 more bytes), so size workspaces after changing it.  Process-wide. */
void moe_set_tma_gather(int enable);

/* The fewest tokens for which a bf16 layer (bf16 activations and expert
 * weights) takes the tensor-core path (router GEMM, grouped tcgen05 GEMMs)
 * instead of the weight-streaming path; default 16 (the streaming path for 1..15
 * tokens), where the two paths cross on B200 (between 8 and 16 tokens on the
 * measured shapes).  Values below 1 count as 1.  moe_workspace_bytes follows
 * the current setting, so size workspaces after changing it.  Process-wide. */
void moe_set_tensor_min_tokens(int tokens);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
