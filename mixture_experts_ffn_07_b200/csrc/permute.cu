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
// compared bit-exactly with the oracle.  Up to 65536 pairs the same sort runs
// on a cluster of CTAs (permute_cluster_kernel); beyond that one CTA loops.
#include <cooperative_groups.h>

#include "kernels.h"

namespace cg = cooperative_groups;

namespace moe {

namespace {

constexpr int kWarps = 32;
constexpr int kMaxE = 256;
constexpr int kBatch = 8;  // 32-pair rounds whose ids are loaded together
constexpr int kCluster = 8;

__global__ void __launch_bounds__(kWarps * 32) permute_kernel(const int32_t* __restrict__ ids, int P, int E,
                                                               int32_t* __restrict__ counts,
                                                               int32_t* __restrict__ offsets,
                                                               int32_t* __restrict__ sorted_pairs,
                                                               int32_t* __restrict__ pair_pos, int* status) {
  __shared__ int hist[kWarps][kMaxE];  // per (warp segment, expert): count, later running base
  __shared__ int tot[kMaxE];
  __shared__ int excl[kMaxE + 1];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_trigger();
  for (int i = threadIdx.x; i < kWarps * kMaxE; i += blockDim.x) (&hist[0][0])[i] = 0;
  pdl_wait();
  __syncthreads();

  const int seg = (P + kWarps - 1) / kWarps;
  const int p0 = min(P, warp * seg), p1 = min(P, p0 + seg);
  bool bad = false;
  for (int base = p0; base < p1; base += 32 * kBatch) {
    int e[kBatch];  // all loads of the batch in flight before any is used
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int p = base + 32 * j + lane;
      e[j] = (p < p1) ? ids[p] : -1;
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      if (base + 32 * j + lane < p1) {
        if (e[j] >= 0 && e[j] < E)
          atomicAdd(&hist[warp][e[j]], 1);
        else
          bad = true;
      }
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

  for (int base = p0; base < p1; base += 32 * kBatch) {
    int eb[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int p = base + 32 * j + lane;
      eb[j] = (p < p1) ? ids[p] : -1;
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {  // rounds in pair order keep the sort stable
      const int p = base + 32 * j + lane;
      const int e = eb[j];
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
}

// The same stable counting sort for up to 8 x 8192 pairs, by a cluster of up to
// 8 CTAs.  CTA b owns pairs [8192 b, 8192 (b+1)), each thread 8 of them held in
// registers (warp w: 256 consecutive pairs in 8 rounds of 32).  CTA-level
// expert counts are exchanged through distributed shared memory, so the pairs
// are read from memory once and no global scratch is needed.
constexpr int kPerThread = 8;
constexpr int kClusterChunk = kWarps * 32 * kPerThread;  // 8192 pairs per CTA

__global__ void __launch_bounds__(kWarps * 32) permute_cluster_kernel(const int32_t* __restrict__ ids, int P, int E,
                                                                       int32_t* __restrict__ counts,
                                                                       int32_t* __restrict__ offsets,
                                                                       int32_t* __restrict__ sorted_pairs,
                                                                       int32_t* __restrict__ pair_pos, int* status) {
  __shared__ int hist[kWarps][kMaxE];
  __shared__ int tot[kMaxE];   // this CTA's pairs per expert (read by the other CTAs)
  __shared__ int excl[kMaxE + 1];
  __shared__ int cta_base[kMaxE];
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int ncta = static_cast<int>(cluster.num_blocks());
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_trigger();
  for (int i = threadIdx.x; i < kWarps * kMaxE; i += blockDim.x) (&hist[0][0])[i] = 0;
  pdl_wait();
  const int base = rank * kClusterChunk + warp * 32 * kPerThread;
  int e[kPerThread];
#pragma unroll
  for (int j = 0; j < kPerThread; ++j) {
    const int p = base + 32 * j + lane;
    e[j] = (p < P) ? ids[p] : -1;
  }
  __syncthreads();
  bool bad = false;
#pragma unroll
  for (int j = 0; j < kPerThread; ++j) {
    if (base + 32 * j + lane < P) {
      if (e[j] >= 0 && e[j] < E)
        atomicAdd(&hist[warp][e[j]], 1);
      else
        bad = true;
    }
  }
  if (bad) record_status(status, MOE_ERR_DEVICE_INDEX);
  __syncthreads();
  for (int x = threadIdx.x; x < E; x += blockDim.x) {
    int s = 0;
    for (int w = 0; w < kWarps; ++w) s += hist[w][x];
    tot[x] = s;
  }
  cluster.sync();  // every CTA's totals are ready
  for (int x = threadIdx.x; x < E; x += blockDim.x) {
    int all = 0, before = 0;
    for (int b = 0; b < ncta; ++b) {
      const int v = cluster.map_shared_rank(tot, b)[x];
      all += v;
      if (b < rank) before += v;
    }
    cta_base[x] = before;
    excl[x] = all;  // per-expert totals, scanned below
  }
  __syncthreads();
  if (warp == 0) {  // exclusive scan of the totals over experts
    int v[8], local = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int x = lane * 8 + i;
      v[i] = x < E ? excl[x] : 0;
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
      const int x = lane * 8 + i;
      if (x < E) {
        if (rank == 0) {
          counts[x] = v[i];
          offsets[x] = run;
        }
        excl[x] = run;
      }
      run += v[i];
    }
    if (lane == 31 && rank == 0) offsets[E] = incl;
  }
  __syncthreads();
  for (int x = threadIdx.x; x < E; x += blockDim.x) {
    int run = excl[x] + cta_base[x];
    for (int w = 0; w < kWarps; ++w) {
      const int c = hist[w][x];
      hist[w][x] = run;
      run += c;
    }
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < kPerThread; ++j) {  // rounds in pair order keep the sort stable
    const int p = base + 32 * j + lane;
    const bool ok = p < P && e[j] >= 0 && e[j] < E;
    const unsigned peers = __match_any_sync(0xffffffffu, ok ? e[j] : -1);
    const int rk = __popc(peers & ((1u << lane) - 1u));
    int pos = 0;
    if (ok) pos = hist[warp][e[j]] + rk;
    __syncwarp();
    if (ok) {
      if (lane == __ffs(peers) - 1) hist[warp][e[j]] += __popc(peers);
      sorted_pairs[pos] = p;
      pair_pos[p] = pos;
    }
    __syncwarp();
  }
  cluster.sync();  // no CTA leaves while another may still read its totals
}

// One warp per destination row; each lane moves 16-byte chunks, four in flight.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ x,
                                                          const int32_t* __restrict__ sorted_pairs,
                                                          const int32_t* __restrict__ offsets, int E, int K, int P,
                                                          int chunks_per_row, uint4* __restrict__ out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_trigger();
  pdl_wait();
  const int rows = min(P, offsets[E]);
  const int nwarps = gridDim.x * (blockDim.x >> 5);
  for (int r = blockIdx.x * (blockDim.x >> 5) + warp; r < rows; r += nwarps) {
    const int t = sorted_pairs[r] / K;
    const uint4* src = x + static_cast<size_t>(t) * chunks_per_row;
    uint4* dst = out + static_cast<size_t>(r) * chunks_per_row;
    for (int c0 = lane; c0 < chunks_per_row; c0 += 128) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (c0 + 32 * u < chunks_per_row) v[u] = __ldg(src + c0 + 32 * u);
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (c0 + 32 * u < chunks_per_row) dst[c0 + 32 * u] = v[u];
    }
  }
}

}  // namespace

cudaError_t launch_permute(const Ctx& c, const int32_t* ids, int P, int E, int32_t* counts, int32_t* offsets,
                           int32_t* sorted_pairs, int32_t* pair_pos) {
  if (P <= kCluster * kClusterChunk) {
    const int ncta = std::max(1, (P + kClusterChunk - 1) / kClusterChunk);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ncta);
    cfg.blockDim = dim3(kWarps * 32);
    cfg.stream = c.stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = c.pdl ? 1 : 0;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = ncta;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    KernelScope ks(c, "permute");
    const cudaError_t e = cudaLaunchKernelEx(&cfg, permute_cluster_kernel, ids, P, E, counts, offsets, sorted_pairs,
                                             pair_pos, c.status);
    return e != cudaSuccess ? e : cudaGetLastError();
  }
  KernelScope ks(c, "permute");
  return launch_kernel(c, permute_kernel, dim3(1), dim3(kWarps * 32), 0, ids, P, E, counts, offsets, sorted_pairs,
                       pair_pos, c.status);
}

cudaError_t launch_gather_rows(const Ctx& c, const __nv_bfloat16* x, const int32_t* sorted_pairs,
                               const int32_t* offsets, int E, int K, int P, int H, __nv_bfloat16* x_perm) {
  if (P == 0) return cudaSuccess;
  const int cpr = H / 8;
  const int blocks = std::max(1, std::min((P + 7) / 8, 8 * c.num_sms));
  KernelScope ks(c, "gather_rows");
  return launch_kernel(c, gather_rows_kernel, dim3(blocks), dim3(256), 0, reinterpret_cast<const uint4*>(x),
                       sorted_pairs, offsets, E, K, P, cpr, reinterpret_cast<uint4*>(x_perm));
}

}  // namespace moe
