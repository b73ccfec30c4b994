// Gate/up and down of the fused decode layer as one continuous weight stream.
//
// The layer's weight rows (every touched expert's gate, up and down rows, and
// the shared expert's) are cut into work items that run in one queue: first
// all gate/up items, expert by expert, then all down items in the same expert
// order (the role of DS4Server qwen_mtplx.rs, fused_experts: moe_glu_h then
// moe_down_y, here without a pause between the two).  An item is 32 weight
// rows over the whole reduction length, for a chunk of up to NT tokens of one
// group:
//   gate/up: gate rows j..j+15 and up rows j..j+15 of an expert (16 features);
//   down:    down rows n..n+31.
// Every CTA takes the next item from a device-wide counter; lane 0 of warp 0
// streams the items' rows through the copy engine (cp.async.bulk.tensor.2d,
// one box of 16 or 32 rows x 256 elements per copy -- 16 to 32 KB, so the
// copy engine's cost per copy stays small -- no multicast) into a ring of
// kStages stages, each on its own pair of mbarriers (full: the copies landed;
// empty: all 16 warps are done with it).  Warp w takes two rows of every
// stage (gate/up: gate row w and up row 16 + w, i.e. feature j + w; down: rows
// 2w and 2w + 1); lane l owns 16-byte chunks l and 32 + l of each row (512
// bytes apart, so every shared-memory load of the warp reads 512 contiguous
// bytes), loads its activation values for those elements once per token (x
// from the input through L1, h from L2) and uses them for both rows,
// accumulating 2 x NT partial sums in registers.  At the item's last stage
// the warp adds its lanes' partial sums (a butterfly over the 2*NT values)
// and writes
//   gate/up: h[r, j + w] = act(g) * u   (f32 rows of the hidden activation)
//   down:    y[dest_r, n + 2w + i] = scale_r * d_i (the pairs' slot rows
//            weighted by the routing weight, or the shared expert's rows by
//            its gate).
// A down item of expert e needs the whole h rows of e: when all 16 warps of a
// gate/up item have stored their h values (counted in shared memory), the
// last one fences and adds 1 to the group's counter; a down item's warps wait
// (bounded) until the count is complete before they read h, and remember
// groups found complete, so later items of the group do not ask again.  The queue hands out all gate/up items first, expert by expert, so
// the first down items find their experts finished long before; there is no
// grid barrier between the two projections, and a CTA moves from gate/up rows
// to down rows without draining its ring.  (Asking L2 for a batch of items
// ahead of their copies measured slower: the prefetched rows of 148 CTAs
// evict one another.)  A group with more than NT tokens
// has one item per chunk of NT tokens, the chunks of a row block next to each
// other in the queue so that the repeated weight rows come from L2.
//
// Formats: f32 and bf16 weight rows, f32 or bf16 activations.  (A Q8_0 form
// of the stream measured slower than the row-pair GEMV of stream_core.cuh,
// so Q8_0 and the k-quant stacks keep the two phases.)
#pragma once

#include "stream_core.cuh"

namespace moe {
namespace dstream {

using stream::kWarps;
using stream::WK_BF16;
using stream::WK_F32;

constexpr int kStages = 4;            // ring depth
constexpr int kRows = 32;             // weight rows per stage (and per item)
constexpr int kRowBytes = 1024;       // bytes of one weight row in a stage (f32: 256 values)
constexpr int kStageBytes = kRows * kRowBytes;    // 32 KB
constexpr int kRingBytes = kStages * kStageBytes;
static_assert(kStageBytes % 128 == 0 && (kRows / 2) * 512 % 128 == 0,
              "every copy into the ring starts at a 128-byte boundary");

// Elements of a row per stage (KC: 256, the widest box), bytes of a row per
// stage (RB) and 16-byte chunks per lane and row (NCH).
template <int WK>
struct Fmt {
  static_assert(WK == WK_F32 || WK == WK_BF16, "the stream serves f32 and bf16 weights");
  static constexpr int EB = WK == WK_F32 ? 4 : 2;
  static constexpr int KC = 256;                       // row elements per stage
  static constexpr int RB = KC * EB;                   // bytes of a row in a stage
  static constexpr int NCH = RB / 512;                 // 16-byte chunks per lane and row
  static constexpr int E16 = 16 / EB;                  // elements per chunk
  static_assert(RB % 512 == 0 && RB <= kRowBytes, "a stage row is whole 512-byte runs");
};

// Tensor maps of one layer: the weights of gate, up, down, shared gate, shared
// up, shared down, in boxes 256 elements wide, 16 rows high for gate/up and
// 32 for down.
enum { M_GATE = 0, M_UP, M_DOWN, M_SGATE, M_SUP, M_SDOWN, M_COUNT };
struct Maps {
  CUtensorMap w[M_COUNT];
};

// Per-launch synchronisation words in the caller's workspace, zeroed by the
// kernel before the grid barrier that precedes the stream.
constexpr int kMaxGroups = 257;
struct Sync {
  unsigned queue;               // next batch of items to hand out
  unsigned done[kMaxGroups];    // finished gate/up items per group
};

struct Params {
  int H, K, I, Is, act;
  const void* x;       // [T, H] activations (XT)
  float* h;            // [P, I] hidden rows in expert-sorted order
  float* h_s;          // [T, Is] shared expert hidden rows
  float* y_slots;      // [P, H] weighted expert outputs, row = pair id
  float* y_s;          // [T, H] shared expert output (scaled by its gate)
  Sync* sync;
  long long wait_limit;
  int* status;
};

// Item tables of the layer (shared memory, filled once per CTA after routing).
struct Items {
  const int* expert;  // group g: expert id, -1 = shared expert
  const int* first;   // first sorted row of the group
  const int* count;   // tokens of the group
  const int* gi;      // [n + 1] prefix of gate/up items per group
  const int* di;      // [n + 1] prefix of down items per group
  int n;
};

__device__ __forceinline__ int nchunks(int count, int nt) { return (count + nt - 1) / nt; }

// Items of a group: gate/up (features / 16) x chunks, down (H / 32) x chunks.
__device__ __forceinline__ int g_items(const Params& p, int expert, int count, int nt) {
  return ((expert < 0 ? p.Is : p.I) / (kRows / 2)) * nchunks(count, nt);
}
__device__ __forceinline__ int d_items(const Params& p, int count, int nt) {
  return (p.H / kRows) * nchunks(count, nt);
}

// One warp fills gi / di (prefix sums over the n groups).
template <int NT>
__device__ __forceinline__ void build_items(const Params& p, const int* expert, const int* count, int n, int* gi,
                                            int* di) {
  const int lane = threadIdx.x & 31;
  const int per = (n + 31) / 32;
  const int g0 = min(n, lane * per), g1 = min(n, g0 + per);
  int sg = 0, sd = 0;
  for (int g = g0; g < g1; ++g) {
    sg += g_items(p, expert[g], count[g], NT);
    sd += d_items(p, count[g], NT);
  }
  int eg = sg, ed = sd;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, eg, o);
    const int b = __shfl_up_sync(0xffffffffu, ed, o);
    if (lane >= o) {
      eg += a;
      ed += b;
    }
  }
  int rg = eg - sg, rd = ed - sd;
  for (int g = g0; g < g1; ++g) {
    gi[g] = rg;
    di[g] = rd;
    rg += g_items(p, expert[g], count[g], NT);
    rd += d_items(p, count[g], NT);
  }
  if (lane == 31) {
    gi[n] = eg;
    di[n] = ed;
  }
  __syncwarp();
}

// What one item covers.
struct Item {
  int down;   // 0: gate/up, 1: down
  int g;      // group
  int e;      // expert (-1: shared)
  int r0;     // gate/up: the first of 16 features; down: the first of 32 rows
  int t0;     // first token of the chunk within the group
  int nt;     // tokens of the chunk
  int kdim;   // reduction length
  int nkc;    // stages of the item
};

template <int NT, int WK>
__device__ __forceinline__ Item decode_item(const Params& p, const Items& it, int idx) {
  Item m;
  const int ng = it.gi[it.n];
  m.down = idx >= ng;
  const int* off = m.down ? it.di : it.gi;
  const int v = m.down ? idx - ng : idx;
  int lo = 0, hi = it.n - 1;  // largest g with off[g] <= v
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= v)
      lo = mid;
    else
      hi = mid - 1;
  }
  m.g = lo;
  m.e = it.expert[lo];
  const int cnt = it.count[lo];
  const int nch = nchunks(cnt, NT);
  const int local = v - off[lo];
  const int rb = local / nch, tc = local - rb * nch;
  m.r0 = m.down ? rb * kRows : rb * (kRows / 2);
  m.t0 = tc * NT;
  m.nt = min(NT, cnt - m.t0);
  m.kdim = m.down ? (m.e < 0 ? p.Is : p.I) : p.H;
  m.nkc = (m.kdim + Fmt<WK>::KC - 1) / Fmt<WK>::KC;
  return m;
}

// Thread 0: requests stage kc of item m (its 32 rows) into `st`, completing on `bar`.
template <int WK>
__device__ __forceinline__ void issue_stage(const Maps& maps, const Params& p, const Item& m, int kc, uint8_t* st,
                                            uint64_t* bar) {
  constexpr int RB = Fmt<WK>::RB;
  const int kx = kc * Fmt<WK>::KC;
  mbar_arrive_expect_tx(bar, kRows * RB);
  const uint64_t pol = l2_policy_evict_first();  // weight rows are read once (a repeated chunk: from L2 at once)
  if (!m.down) {
    const int row = (m.e < 0 ? 0 : m.e * p.I) + m.r0;
    tma_load_2d_hint(st, &maps.w[m.e < 0 ? M_SGATE : M_GATE], bar, kx, row, pol);
    tma_load_2d_hint(st + (kRows / 2) * RB, &maps.w[m.e < 0 ? M_SUP : M_UP], bar, kx, row, pol);
  } else {
    tma_load_2d_hint(st, &maps.w[m.e < 0 ? M_SDOWN : M_DOWN], bar, kx, (m.e < 0 ? 0 : m.e * p.H) + m.r0, pol);
  }
}

// E16 activation values of a row at element k, as f32 pairs (L1 for the
// layer's input x, L2 only for the h rows this kernel writes).
template <typename AT, bool L2ONLY, int E16>
__device__ __forceinline__ void act_chunk(const AT* row, int k, float2 (&x)[E16 / 2]) {
  if constexpr (sizeof(AT) == 4) {
#pragma unroll
    for (int q = 0; q < E16 / 4; ++q) {
      const float4* p4 = reinterpret_cast<const float4*>(row + k) + q;
      const float4 a = L2ONLY ? __ldcg(p4) : __ldg(p4);
      x[2 * q] = make_float2(a.x, a.y);
      x[2 * q + 1] = make_float2(a.z, a.w);
    }
  } else if constexpr (E16 == 4) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(row + k));
    x[0] = stream::bf16x2_f2(v.x);
    x[1] = stream::bf16x2_f2(v.y);
  } else {
#pragma unroll
    for (int q = 0; q < E16 / 8; ++q) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(row + k) + q);
      x[4 * q] = stream::bf16x2_f2(v.x);
      x[4 * q + 1] = stream::bf16x2_f2(v.y);
      x[4 * q + 2] = stream::bf16x2_f2(v.z);
      x[4 * q + 3] = stream::bf16x2_f2(v.w);
    }
  }
}

// The 16-byte chunk of a stage row at shared address `a`, widened to E16 f32 values (as pairs).
template <int WK>
__device__ __forceinline__ void w_chunk(uint32_t a, float2 (&w)[Fmt<WK>::E16 / 2]) {
  const uint4 v = stream::lds16(a);
  if constexpr (WK == WK_F32) {
    w[0] = make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
    w[1] = make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
  } else {
    w[0] = stream::bf16x2_f2(v.x);
    w[1] = stream::bf16x2_f2(v.y);
    w[2] = stream::bf16x2_f2(v.z);
    w[3] = stream::bf16x2_f2(v.w);
  }
}

// Sums of V values over the warp: afterwards lane l holds the total of value
// l / (32 / V) (each total in 32 / V lanes).  V is a power of two <= 32.
template <int V>
__device__ __forceinline__ float warp_reduce_many(float (&v)[V]) {
  const int lane = threadIdx.x & 31;
  int n = V;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    if (n > 1) {
      const bool upper = (lane & off) != 0;
#pragma unroll
      for (int i = 0; i < V / 2; ++i) {
        if (i < n / 2) {
          const float keep = upper ? v[i + n / 2] : v[i];
          const float send = upper ? v[i] : v[i + n / 2];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
      }
      n >>= 1;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
    }
  }
  return v[0];
}

// Wait until phase `parity` of `bar` completed; false after `limit` cycles
// (decided by lane 0, so the outcome is warp-uniform).  All lanes.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, long long limit) {
  if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
  const long long t0 = clock64();
  for (;;) {
    if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
    if (__shfl_sync(0xffffffffu, static_cast<int>(clock64() - t0 > limit), 0)) return false;
  }
}

// Shared state of the stream in one CTA (shared memory).
constexpr int kMaxBatch = 4;  // most items handed out per queue step (fewer when there are few items per warp)
struct Ring {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  Item item[kStages];      // the item a stage belongs to (decoded once, by the producer)
  int kc[kStages];         // the stage's index within its item; -1: the queue is empty
  int done_warps[kStages]; // warps of the gate/up item ending in this stage that have stored their h values
  unsigned gdone[(kMaxGroups + 31) / 32];  // groups whose gate/up items are all finished (known to this CTA)
};

// The stream of one CTA, until the queue is empty.  All threads of the CTA
// (16 warps).  Returns false if a wait gave up (MOE_ERR_TIMEOUT recorded).
//   stages: kRingBytes of shared memory, 128-byte aligned
//   pairs:  sorted pair ids;  wpair: routing weight per pair id;  sgate: shared-expert gate per token or nullptr
template <typename XT, int WK, int NT>
__device__ __forceinline__ bool run_stream(const Maps& maps, const Params& p, const Items& it, uint8_t* stages,
                                           Ring& ring, const int32_t* pairs, const float* wpair, const float* sgate) {
  constexpr int KC = Fmt<WK>::KC;
  constexpr int RB = Fmt<WK>::RB;
  constexpr int NCH = Fmt<WK>::NCH;
  constexpr int E16 = Fmt<WK>::E16;
  constexpr int NV = 2 * NT;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int total = it.gi[it.n] + it.di[it.n];
  const bool producer = threadIdx.x == 0;
  // items per queue step: about 16 steps per CTA, at most kMaxBatch (large items are few: batching them
  // would leave the CTAs unevenly loaded)
  const int kBatch = max(1, min(kMaxBatch, total / (static_cast<int>(gridDim.x) * 16)));

  // ---- issue side (thread 0): a cursor over (item, stage of the item) in queue order; items come in
  // batches of kBatch consecutive ones, the next batch asked for while the current one is issued
  int is_item = 0, is_end = 0, is_next = 0, is_kc = 0;
  Item is_m{};
  if (producer) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ring.full[s], 1);
      mbar_init(&ring.empty[s], kWarps);
    }
    for (int s = 0; s < kStages; ++s) ring.done_warps[s] = 0;
    for (int i = 0; i < (kMaxGroups + 31) / 32; ++i) ring.gdone[i] = 0;
    fence_mbar_init();
    is_item = static_cast<int>(atomicAdd(&p.sync->queue, 1u)) * kBatch;
    is_end = min(total, is_item + kBatch);
    is_next = static_cast<int>(atomicAdd(&p.sync->queue, 1u)) * kBatch;
    if (is_item < is_end) is_m = decode_item<NT, WK>(p, it, is_item);
  }
  auto issue = [&](int s) {  // thread 0: the next stage in queue order into ring stage s, or an end mark
    while (is_item < is_end && is_kc >= is_m.nkc) {
      if (++is_item >= is_end) {
        is_item = is_next;
        is_end = min(total, is_item + kBatch);
        if (is_item < is_end)  // the batch after it, asked for now
          is_next = static_cast<int>(atomicAdd(&p.sync->queue, 1u)) * kBatch;
      }
      is_kc = 0;
      if (is_item < is_end) is_m = decode_item<NT, WK>(p, it, is_item);
    }
    if (is_item >= is_end) {
      ring.kc[s] = -1;
      mbar_arrive(&ring.full[s]);  // the end mark is published through the same barrier
      return;
    }
    ring.item[s] = is_m;
    ring.kc[s] = is_kc;
    issue_stage<WK>(maps, p, is_m, is_kc, stages + s * kStageBytes, &ring.full[s]);
    ++is_kc;
  };
  if (producer)
    for (int s = 0; s < kStages; ++s) issue(s);
  __syncthreads();

  // ---- compute side (every warp)
  Item m{};
  int arow[NT];  // activation row of each token of the chunk (x row for gate/up, h row for down)
  float2 acc_a[NT], acc_b[NT];
  bool ok = true;
  for (uint32_t q = 0;; ++q) {
    const int s = static_cast<int>(q % kStages);
    const uint32_t par = (q / kStages) & 1u;
    if (!warp_wait(&ring.full[s], par, p.wait_limit)) {
      record_status(p.status, MOE_ERR_TIMEOUT);
      ok = false;
      break;
    }
    const int kc = ring.kc[s];
    if (kc < 0) break;
    if (kc == 0) {  // ---- the item begins
      m = ring.item[s];
      const int first = it.first[m.g];
#pragma unroll
      for (int c = 0; c < NT; ++c) {
        const int t = m.t0 + min(c, m.nt - 1);
        arow[c] = m.e < 0 ? t : (m.down ? first + t : pairs[first + t] / p.K);
        acc_a[c] = acc_b[c] = make_float2(0.f, 0.f);
      }
      if (m.down && !(ring.gdone[m.g >> 5] >> (m.g & 31) & 1u)) {
        // the group's gate/up items are not known to be finished here: wait until the count is complete
        const unsigned need = static_cast<unsigned>(g_items(p, m.e, it.count[m.g], NT));
        int waited = 1;
        if (lane == 0) {
          const long long t0 = clock64();
          for (;;) {
            unsigned v;
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(&p.sync->done[m.g]) : "memory");
            if (v >= need) break;
            if (clock64() - t0 > p.wait_limit) {
              waited = 0;
              break;
            }
          }
          if (waited) atomicOr_block(&ring.gdone[m.g >> 5], 1u << (m.g & 31));
        }
        waited = __shfl_sync(0xffffffffu, waited, 0);
        __syncwarp();
        if (!waited) {
          record_status(p.status, MOE_ERR_TIMEOUT);
          ok = false;
        }
      }
    }
    // ---- this stage: the warp's rows a and b, lane chunks ch = 0..NCH-1 at bytes ch*512 + lane*16
    const uint32_t st = smem_addr(stages + s * kStageBytes);
    const int ra = m.down ? 2 * warp : warp, rb = m.down ? 2 * warp + 1 : kRows / 2 + warp;
    const uint32_t wa_s = st + ra * RB, wb_s = st + rb * RB;
#pragma unroll
    for (int ch = 0; ch < NCH; ++ch) {
      const int k = kc * KC + (ch * 512 + lane * 16) / Fmt<WK>::EB;
      if (ok && k < m.kdim) {  // past the row (the last stage's tail): nothing to add
        float2 wa[E16 / 2], wb[E16 / 2];
        w_chunk<WK>(wa_s + ch * 512 + lane * 16, wa);
        w_chunk<WK>(wb_s + ch * 512 + lane * 16, wb);
#pragma unroll
        for (int c = 0; c < NT; ++c) {
          if (c < m.nt) {
            float2 xv[E16 / 2];
            if (m.down)
              act_chunk<float, true, E16>(m.e >= 0 ? p.h + static_cast<size_t>(arow[c]) * p.I
                                                    : p.h_s + static_cast<size_t>(arow[c]) * p.Is,
                                          k, xv);
            else
              act_chunk<XT, false, E16>(static_cast<const XT*>(p.x) + static_cast<size_t>(arow[c]) * p.H, k, xv);
#pragma unroll
            for (int i = 0; i < E16 / 2; ++i) {
              acc_a[c] = __ffma2_rn(wa[i], xv[i], acc_a[c]);
              acc_b[c] = __ffma2_rn(wb[i], xv[i], acc_b[c]);
            }
          }
        }
      }
    }
    if (ok && kc == m.nkc - 1) {  // ---- the item ends: add the lanes' sums and store
      float v[NV];
#pragma unroll
      for (int c = 0; c < NT; ++c) {
        v[c] = acc_a[c].x + acc_a[c].y;
        v[NT + c] = acc_b[c].x + acc_b[c].y;
      }
      const float tot = warp_reduce_many<NV>(v);
      constexpr int per = 32 / NV;  // lanes holding each total; value i sits in lanes [i*per, i*per + per)
      const int vi = lane / per;
      const int c = vi % NT;
      const int first = it.first[m.g];
      const int t = m.t0 + min(c, m.nt - 1);
      const int pr = m.e < 0 ? t : pairs[first + t];
      if (!m.down) {
        // row a (gate) totals are values [0, NT), row b (up) [NT, 2 NT): 16 lanes higher
        const float u = __shfl_down_sync(0xffffffffu, tot, 16);
        if (lane < 16 && lane % per == 0 && c < m.nt) {
          const float hv = act_fn(p.act, tot) * u;
          const int f = m.r0 + warp;
          if (m.e < 0)
            p.h_s[static_cast<size_t>(t) * p.Is + f] = hv;
          else
            p.h[static_cast<size_t>(first + t) * p.I + f] = hv;
        }
        // the item's 16 warps count themselves in shared memory; the last one makes all their h stores
        // visible GPU-wide (the fence is cumulative over what it observed) and counts the item for its group
        __threadfence_block();
        __syncwarp();
        if (lane == 0 && atomicAdd_block(&ring.done_warps[s], 1) == kWarps - 1) {
          ring.done_warps[s] = 0;  // ready for the next item ending in this stage (after the refill)
          __threadfence();
          atomicAdd(&p.sync->done[m.g], 1u);
        }
      } else if (lane % per == 0 && c < m.nt) {
        const int n = m.r0 + 2 * warp + vi / NT;  // rows 2w, 2w + 1 of the block
        if (m.e < 0)
          p.y_s[static_cast<size_t>(t) * p.H + n] = (sgate ? sgate[t] : 1.f) * tot;
        else
          p.y_slots[static_cast<size_t>(pr) * p.H + n] = wpair[pr] * tot;
      }
    }
    // the warp is done with the stage (its shared memory, and the item-end count kept for it)
    __syncwarp();
    if (lane == 0) mbar_arrive(&ring.empty[s]);
    // thread 0 refills the stage once every warp has released it
    if (producer) {
      const long long t0 = clock64();
      while (!mbar_try_wait(&ring.empty[s], par)) {
        if (clock64() - t0 > p.wait_limit) {
          record_status(p.status, MOE_ERR_TIMEOUT);
          ok = false;
          break;
        }
      }
      if (ok) issue(s);
    }
    ok = __shfl_sync(0xffffffffu, static_cast<int>(ok), 0) != 0;
    if (!ok) break;
  }
  return ok;
}

}  // namespace dstream
}  // namespace moe
