// Selection, permutation and row gather of the tensor-core path in one
// cooperative launch, after the router GEMM.
//
// The three steps are the ones of router_topk_kernel, permute_kernel and
// gather_rows_kernel (hf2q softmax_topk_renorm_cpu for the selection;
// DS4Server gather_sort for the stable expert order and the gathered rows),
// which as separate launches each pay a launch and a ramp for a few
// microseconds of work.  Here CTA c owns a contiguous block of tokens:
//   A  a warp per token adds the router GEMM's split-K partials in order and
//      selects (topk_token, shared with router_topk_kernel, so the ids equal
//      moe_route's bit for bit); the CTA counts its pairs per expert and
//      publishes the counts in hist[c][*];                         -- barrier
//   B  every CTA adds the published counts (totals, and the counts of the
//      CTAs before it; J = 512 / E threads per expert, register sums over a
//      fixed subset of CTAs each, no atomics), scans them into expert offsets, places its own pairs
//      in pair order (a stable counting sort, so the permutation is unique),
//      writes sorted_pairs / pair_pos and copies each pair's x row into its
//      place in x_perm.
// The grid barrier is the bounded counter barrier of common.cuh on a counter
// of its own; the kernel asks for more than half of an SM's shared memory so
// that no two of these grids are ever resident on one device together.
#include <atomic>

#include "route_util.cuh"

namespace moe {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
// dynamic shared memory: [kWarps][256] f32 logit rows (A), [2][kThreads] count partials (B), then the
// positions of this CTA's pairs (B)
constexpr int kPosOff = kWarps * 256 * 4 + 2 * kThreads * 4;

__device__ unsigned long long g_front_barrier;

struct FrontArgs {
  const float* parts;  // split-K partial logits (nparts > 0) or nullptr
  int nparts;
  size_t part_stride;
  float* logits;  // [T, E]
  const float* bias;
  int T, E, K, renorm, H;
  RouteCfg rc;
  int32_t* ids;
  float* w;
  const __nv_bfloat16* x;
  const __nv_bfloat16* w_s;
  float* shared_gate;
  int32_t* counts;
  int32_t* offsets;
  int32_t* sorted_pairs;
  int32_t* pair_pos;
  __nv_bfloat16* x_perm;
  int32_t* hist;  // [gridDim.x, E]
  int pos_cap;    // pair positions the shared-memory area after the count partials holds (0: none)
  int* status;
  long long wait_limit;
  long long barrier_delay;
};

__global__ void __launch_bounds__(kThreads, 1) front_kernel(const FrontArgs a) {
  extern __shared__ __align__(16) uint8_t fsmem[];  // logit rows, count partials, pair positions (kPosOff)
  __shared__ int s_hist[256], s_run[256], s_tot[256], s_off[257];
  __shared__ int s_abort, s_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, c = blockIdx.x, E = a.E, K = a.K;
  const int t0 = static_cast<int>(static_cast<long long>(a.T) * c / G);
  const int t1 = static_cast<int>(static_cast<long long>(a.T) * (c + 1) / G);
  const int p0 = t0 * K, p1 = t1 * K;
  if (threadIdx.x == 0) s_abort = 0;
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_hist[e] = 0;
  pdl_trigger();
  pdl_wait();  // the router GEMM's logits are complete and visible

  // ---- A: selection of this CTA's tokens, and its pair counts
  for (int t = t0 + warp; t < t1; t += kWarps)
    topk_token<__nv_bfloat16, __nv_bfloat16>(a.parts, a.nparts, a.part_stride, a.logits, a.bias, a.rc, a.ids, a.w,
                                             a.x, a.w_s, a.H, a.shared_gate, t,
                                             reinterpret_cast<float*>(fsmem) + warp * 256);
  __syncthreads();
  for (int p = p0 + threadIdx.x; p < p1; p += blockDim.x) atomicAdd(&s_hist[a.ids[p]], 1);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) a.hist[static_cast<size_t>(c) * E + e] = s_hist[e];
  debug_delay_cta0(a.barrier_delay);
  if (!grid_sync(&g_front_barrier, a.wait_limit, a.status, &s_abort, &s_flag)) {
    // some CTA's counts may be missing: placing pairs could go out of range.  Leave tables the next kernels
    // can follow without leaving their buffers: this CTA's pairs map to themselves, and CTA 0 (which writes
    // the offsets when it gets through) gives every expert no rows.
    if (threadIdx.x == 0) record_status(a.status, MOE_ERR_TIMEOUT);
    for (int p = p0 + threadIdx.x; p < p1; p += blockDim.x) {
      a.sorted_pairs[p] = p;
      a.pair_pos[p] = p;
    }
    if (c == 0)
      for (int e = threadIdx.x; e <= E; e += blockDim.x) {
        a.offsets[e] = 0;
        if (e < E) a.counts[e] = 0;
      }
    return;
  }

  // ---- B: offsets, this CTA's pair positions and rows
  {  // totals and the counts of the CTAs before this one: J = 512 / E threads per expert, each summing the
     // counts of CTAs j, j + J, ... in registers (16 loads in flight), then a fixed-order sum over j
    int* red_tot = reinterpret_cast<int*>(fsmem + kWarps * 256 * 4);
    int* red_run = red_tot + kThreads;
    const int J = kThreads / E;
    if (threadIdx.x < J * E) {
      const int e = threadIdx.x % E, j = threadIdx.x / E;
      int tot = 0, run = 0;
      for (int c0 = j; c0 < G; c0 += 16 * J) {
        int v[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const int cc = c0 + q * J;
          v[q] = cc < G ? __ldcg(a.hist + static_cast<size_t>(cc) * E + e) : 0;
        }
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          tot += v[q];
          if (c0 + q * J < c) run += v[q];
        }
      }
      red_tot[j * E + e] = tot;
      red_run[j * E + e] = run;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      int tot = 0, run = 0;
      for (int j = 0; j < J; ++j) {
        tot += red_tot[j * E + e];
        run += red_run[j * E + e];
      }
      s_tot[e] = tot;
      s_run[e] = run;
    }
  }
  __syncthreads();
  if (warp == 0) {  // exclusive scan of the totals (E <= 256: 8 per lane)
    int loc[8], sum = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane * 8 + i;
      loc[i] = e < E ? s_tot[e] : 0;
      sum += loc[i];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - sum;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane * 8 + i;
      if (e < E) s_off[e] = run;
      run += loc[i];
    }
    if (lane == 31) s_off[E] = incl;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    s_run[e] += s_off[e];  // where this CTA's first pair of expert e goes
    if (c == 0) {
      a.counts[e] = s_tot[e];
      a.offsets[e] = s_off[e];
    }
  }
  if (c == 0 && threadIdx.x == 0) a.offsets[E] = s_off[E];
  __syncthreads();
  int* s_pos = reinterpret_cast<int*>(fsmem + kPosOff);
  const bool pos_in_smem = p1 - p0 <= a.pos_cap;
  if (warp == 0) {  // in pair order, 32 at a time; equal experts ranked by lane
    for (int base = p0; base < p1; base += 32) {
      const int p = base + lane;
      const int e = p < p1 ? a.ids[p] : -1;
      const unsigned m = __match_any_sync(0xffffffffu, e);
      const int rank = __popc(m & ((1u << lane) - 1u));
      const int before = p < p1 ? s_run[e] : 0;
      __syncwarp();
      if (p < p1) {
        const int pos = before + rank;
        a.sorted_pairs[pos] = p;
        a.pair_pos[p] = pos;
        if (pos_in_smem) s_pos[p - p0] = pos;
        if (rank == 0) s_run[e] = before + __popc(m);
      }
      __syncwarp();
    }
  }
  if (a.x_perm == nullptr) return;  // the expert GEMM gathers the rows itself
  __syncthreads();
  const int n16 = a.H / 8;  // 16-byte groups of a bf16 row
  const uint4* src = reinterpret_cast<const uint4*>(a.x);
  uint4* dst = reinterpret_cast<uint4*>(a.x_perm);
  // a warp per token: each 4 KB of its row is loaded once and stored at the places of all the token's pairs
  // in this CTA's range (a token's K pairs are consecutive in pair order)
  for (int t = p0 / K + warp; t * K < p1; t += kWarps) {
    const int q0 = max(p0, t * K), q1 = min(p1, t * K + K);
    const uint4* s = src + static_cast<size_t>(t) * n16;
    for (int o = lane; o < n16; o += 32 * 8) {  // a 4 KB row (H = 2048) in one round of loads
      uint4 v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (o + 32 * j < n16) v[j] = __ldg(s + o + 32 * j);
      for (int q = q0; q < q1; ++q) {
        uint4* d = dst + static_cast<size_t>(pos_in_smem ? s_pos[q - p0] : a.pair_pos[q]) * n16;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (o + 32 * j < n16) d[o + 32 * j] = v[j];
      }
    }
  }
}

}  // namespace

cudaError_t launch_prefill_front(const Ctx& c, const PrefillFront& f) {
  if (f.T <= 0) return cudaSuccess;
  if (f.E > 256 || (f.H % 8)) return cudaErrorInvalidValue;
  FrontArgs a{};
  a.parts = f.parts;
  a.nparts = f.nparts;
  a.part_stride = f.part_stride;
  a.logits = f.logits;
  a.bias = f.bias;
  a.T = f.T;
  a.E = f.E;
  a.K = f.K;
  a.renorm = f.renorm;
  a.H = f.H;
  a.rc = f.rc;
  a.ids = f.ids;
  a.w = f.w;
  a.x = f.x;
  a.w_s = f.w_s;
  a.shared_gate = f.shared_gate;
  a.counts = f.counts;
  a.offsets = f.offsets;
  a.sorted_pairs = f.sorted_pairs;
  a.pair_pos = f.pair_pos;
  a.x_perm = f.x_perm;
  a.hist = f.hist;
  a.status = c.status;
  a.wait_limit = c.wait_limit;
  a.barrier_delay = c.barrier_delay;
  // more than half of an SM's shared memory: one CTA per SM, one such grid per device (and room for the
  // warps' logit rows, the count partials and, when they fit, the positions of a CTA's pairs)
  const int grid = std::min(c.num_sms, kMaxFrontCtas);
  const long long max_pairs = (static_cast<long long>(f.T) + grid - 1) / grid * f.K;
  a.pos_cap = kPosOff + max_pairs * 4 <= c.smem_optin ? static_cast<int>(max_pairs) : 0;
  const int smem = std::max(c.smem_optin / 2 + 1024, kPosOff + a.pos_cap * 4);
  cudaError_t e = allow_dynamic_smem(reinterpret_cast<const void*>(front_kernel), smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, front_kernel, kThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm != 1) return cudaErrorInvalidValue;  // the separate launches run instead
  KernelScope ks(c, "route_permute_gather");
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = c.stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // the launch overlaps the router GEMM's tail
  attr[1].val.programmaticStreamSerializationAllowed = c.pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, front_kernel, a);
}

}  // namespace moe
