// Expert histogram, exclusive scan and stable permutation of the (token, slot)
// pairs, plus the row gather that lays the routed activations out expert by
// expert for the tensor-core GEMM.
//
// Semantics: DS4Server qwen_mtplx.rs, gather_sort (order = argsort of the
// flat expert ids, inverse = argsort(order), token row = order / top_k) and
// ferrox-models decoder.rs, moe_ffn_batch (per-expert buckets keep token
// order).  Here: one CTA of 32 warps; warp w owns a contiguous segment of the
// pairs, counts it per expert, and after a scan over (expert, warp) scatters
// it again in order, ranking equal experts inside a 32-pair chunk with
// __match_any_sync.  The result is a stable sort, so it is unique and is
// compared bit-exactly with the oracle.
#include "kernels.h"

namespace moe {

namespace {

constexpr int kWarps = 32;
constexpr int kMaxE = 256;

__global__ void __launch_bounds__(kWarps * 32) permute_kernel(const int32_t* __restrict__ ids, int P, int E,
                                                               int32_t* __restrict__ counts,
                                                               int32_t* __restrict__ offsets,
                                                               int32_t* __restrict__ sorted_pairs,
                                                               int32_t* __restrict__ pair_pos, int* status) {
  __shared__ int hist[kWarps][kMaxE];  // per (warp segment, expert): count, later running base
  __shared__ int tot[kMaxE];
  __shared__ int excl[kMaxE + 1];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kWarps * kMaxE; i += blockDim.x) (&hist[0][0])[i] = 0;
  __syncthreads();

  const int seg = (P + kWarps - 1) / kWarps;
  const int p0 = min(P, warp * seg), p1 = min(P, p0 + seg);
  bool bad = false;
  for (int base = p0; base < p1; base += 32) {
    const int p = base + lane;
    if (p < p1) {
      const int e = ids[p];
      if (e >= 0 && e < E)
        atomicAdd(&hist[warp][e], 1);
      else
        bad = true;
    }
  }
  if (bad) record_status(status, MOE_ERR_DEVICE_INDEX);
  __syncthreads();

  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int s = 0;
    for (int w = 0; w < kWarps; ++w) s += hist[w][e];
    tot[e] = s;
  }
  __syncthreads();
  if (warp == 0) {  // exclusive scan over experts: lane owns experts [8*lane, 8*lane+8)
    int v[8], local = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane * 8 + i;
      v[i] = e < E ? tot[e] : 0;
      local += v[i];
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    int run = incl - local;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane * 8 + i;
      if (e < E) excl[e] = run;
      run += v[i];
    }
    if (lane == 31) excl[E] = incl;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = excl[e];
    for (int w = 0; w < kWarps; ++w) {
      const int c = hist[w][e];
      hist[w][e] = run;
      run += c;
    }
    counts[e] = tot[e];
    offsets[e] = excl[e];
  }
  if (threadIdx.x == 0) offsets[E] = excl[E];
  __syncthreads();

  for (int base = p0; base < p1; base += 32) {
    const int p = base + lane;
    const int e = (p < p1) ? ids[p] : -1;
    const bool ok = e >= 0 && e < E;
    const unsigned peers = __match_any_sync(0xffffffffu, ok ? e : -1);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    int pos = 0;
    if (ok) pos = hist[warp][e] + rank;
    __syncwarp();
    if (ok) {
      if (lane == __ffs(peers) - 1) hist[warp][e] += __popc(peers);
      sorted_pairs[pos] = p;
      pair_pos[p] = pos;
    }
    __syncwarp();
  }
}

// One thread per 16-byte chunk of a destination row.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ x,
                                                          const int32_t* __restrict__ sorted_pairs,
                                                          const int32_t* __restrict__ offsets, int E, int K, int P,
                                                          int chunks_per_row, uint4* __restrict__ out) {
  const int rows = min(P, offsets[E]);
  const long long total = static_cast<long long>(rows) * chunks_per_row;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = i / chunks_per_row;
    const int c = static_cast<int>(i - r * chunks_per_row);
    const int t = sorted_pairs[r] / K;
    out[r * chunks_per_row + c] = __ldg(x + static_cast<long long>(t) * chunks_per_row + c);
  }
}

}  // namespace

cudaError_t launch_permute(const Ctx& c, const int32_t* ids, int P, int E, int32_t* counts, int32_t* offsets,
                           int32_t* sorted_pairs, int32_t* pair_pos) {
  KernelScope ks(c, "permute");
  permute_kernel<<<1, kWarps * 32, 0, c.stream>>>(ids, P, E, counts, offsets, sorted_pairs, pair_pos, c.status);
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const Ctx& c, const __nv_bfloat16* x, const int32_t* sorted_pairs,
                               const int32_t* offsets, int E, int K, int P, int H, __nv_bfloat16* x_perm) {
  if (P == 0) return cudaSuccess;
  const int cpr = H / 8;
  const long long total = static_cast<long long>(P) * cpr;
  const int blocks = static_cast<int>(std::min<long long>((total + 255) / 256, 8LL * c.num_sms));
  KernelScope ks(c, "gather_rows");
  gather_rows_kernel<<<blocks, 256, 0, c.stream>>>(reinterpret_cast<const uint4*>(x), sorted_pairs, offsets, E, K,
                                                   P, cpr, reinterpret_cast<uint4*>(x_perm));
  return cudaGetLastError();
}

}  // namespace moe
