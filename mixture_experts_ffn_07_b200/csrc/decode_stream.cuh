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
// Every CTA takes its next batch of items from a device-wide counter.  The
// CTA is warp specialised: lane 0 of warp 8 streams each item's weight rows
// through the copy engine (cp.async.bulk.tensor.2d, one box of 16 or 32 rows x
// 256 elements per copy; no multicast) into a ring of kStages stages of 32 KB,
// each on a full and an empty mbarrier, and the same stage receives the item's
// activation rows for its 256 elements (the x rows of the chunk's tokens for
// gate/up, a box of h rows for down), so no consumer waits on a global load.
// The issuing thread sleeps on a stage's empty barrier until the 8 consumer
// warps have released it and the consumers sleep on the full barriers:
// nothing polls (a polling issuer measured ~4.3 TB/s on a bare stream of such
// stages, a sleeping one ~5.1).  Consumer warp w takes four rows of every
// stage as two row pairs -- gate/up: features 2w and 2w + 1 (gate row f with
// up row 16 + f); down: rows 4w .. 4w + 3 -- lane l owns 16-byte chunks l and
// 32 + l of each row (512 bytes apart, so every shared-memory load of the
// warp reads 512 contiguous bytes), reads its activation values for those
// elements once per token and uses them for all four rows, accumulating
// 2 x 2 x NT partial sums in registers.  At the item's last stage the warp
// adds its lanes' partial sums (a butterfly over the 2*NT values of each pair)
// and writes
//   gate/up: h[r, j + f] = act(g) * u   (f32 rows of the hidden activation)
//   down:    y[dest_r, n] = scale_r * d  (the pairs' slot rows weighted by
//            the routing weight, or the shared expert's rows by its gate).
// A down item of expert e needs the whole h rows of e: when the 8 consumer
// warps of a gate/up item have stored their h values (counted in shared
// memory), the last one fences and adds 1 to the group's counter.  Before the
// issuing thread requests the first stage of a down item it waits (bounded)
// until its group's count is complete, with an acquiring load; a proxy fence
// then orders the copy engine's reads of h after the stores that count
// published, and the group is remembered as complete.  While it waits, the
// consumers go on with the stages already in the ring.  The queue hands out
// all gate/up items first, expert by expert, and each CTA takes its items in
// queue order, so a down item only waits for gate/up items ahead of it:
// there is no grid barrier between the two projections, and a CTA moves from
// gate/up rows to down rows without draining its ring.  (Asking L2 for a
// batch of items ahead of their copies measured slower: the prefetched rows
// of 148 CTAs evict one another.)  A group with more than NT tokens has one
// item per chunk of NT tokens, the chunks of a row block next to each other
// in the queue so that the repeated weight rows come from L2.
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
using stream::WK_Q8;

constexpr int kStages = 4;            // ring depth
constexpr int kRows = 32;             // weight rows per stage (and per item)
constexpr int kRowBytes = 1024;       // bytes of one weight row in a stage (f32: 256 values, Q8_0: 1024 codes)
constexpr int kMaxNT = 4;             // most tokens per item
constexpr int kStageWBytes = kRows * kRowBytes;  // 32 KB of weight rows

// Tokens per item of a kernel instance built for at most maxt tokens (host and device).
__host__ __device__ constexpr int item_tokens(int maxt) { return maxt == 1 ? 1 : kMaxNT; }

// Geometry of a stage by weight format.  KC: row elements per stage (256 f32, 512 bf16 values in two
// 256-wide boxes, 1024 Q8_0 codes as 256 words); RB: bytes of a row in a stage (kRowBytes for all three);
// NCH: 16-byte chunks per lane and row; E16: elements per chunk;
// AR: bytes of one activation row of the stage (KC values, room for f32); SR: bytes of the fp16 scales of
// one row (Q8_0: 32 blocks).  A stage is [kRows weight rows][kMaxNT activation rows][kRows scale rows].
template <int WK>
struct Fmt {
  static_assert(WK == WK_F32 || WK == WK_BF16 || WK == WK_Q8, "the stream serves f32, bf16 and Q8_0 weights");
  static constexpr int EB = WK == WK_F32 ? 4 : (WK == WK_BF16 ? 2 : 1);
  static constexpr int KC = WK == WK_Q8 ? 1024 : (WK == WK_BF16 ? 512 : 256);
  static constexpr int RB = KC * EB;
  // bf16: a stage holds two 256-column chunks, each as its own plane of kRows rows of 512 bytes (a box is
  // at most 256 wide), and the activation rows likewise as two planes of kMaxNT rows of 1 KB
  static constexpr bool SPLIT = WK == WK_BF16;
  static constexpr int PLANE = kRows * 512;
  static constexpr int APLANE = kMaxNT * 1024;
  static constexpr int NCH = RB / 512;
  static constexpr int E16 = 16 / EB;
  static constexpr int AR = KC * 4;
  static constexpr int SR = WK == WK_Q8 ? KC / 32 * 2 : 0;
  static constexpr int ACT = kStageWBytes;                  // offset of the activation rows
  static constexpr int SCL = ACT + kMaxNT * AR;             // offset of the scale rows
  static constexpr int SB = (SCL + kRows * SR + 127) / 128 * 128;  // stage bytes
  static_assert(RB % 512 == 0 && RB <= kRowBytes && AR % 128 == 0 && SCL % 128 == 0 && (kRows / 2) * SR % 64 == 0,
                "every copy into the ring starts at a 128-byte boundary (scale halves at 64)");
};

// Shared memory of the ring by weight format (host and device).
__host__ __device__ constexpr int ring_bytes(int wk) {
  return kStages * (wk == WK_Q8 ? Fmt<WK_Q8>::SB : (wk == WK_BF16 ? Fmt<WK_BF16>::SB : Fmt<WK_F32>::SB));
}

// Tensor maps of one layer: the weights of gate, up, down, shared gate, shared
// up, shared down, in boxes 256 elements wide (Q8_0: 256 32-bit words of codes),
// 16 rows high for gate/up and 32 for down, and for Q8_0 their fp16 scale
// planes in boxes of 32 x as many rows; the input x; the hidden rows h [P, I]
// and h_s [T, Is] (f32).  For f32 / bf16 weights x comes in boxes of 256 x 1
// row and h (h_s) in boxes of 256 x h_box (hs_box) rows; for Q8_0 all three are
// seen as rows of 256 values ([T * H / 256, 256] and so on) in boxes of 4 such
// rows: the 1024 values of one token that a stage needs.
enum { M_GATE = 0, M_UP, M_DOWN, M_SGATE, M_SUP, M_SDOWN, M_X, M_H, M_HS, M_COUNT };
struct Maps {
  CUtensorMap w[M_COUNT];
  CUtensorMap s[M_SDOWN + 1];
  int h_box, hs_box;
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

// Item idx of the queue; `hint` is a group to try before searching (the previous item's: consecutive items
// of a CTA are mostly in one group).
template <int NT, int WK>
__device__ __forceinline__ Item decode_item(const Params& p, const Items& it, int idx, int hint = 0) {
  Item m;
  const int ng = it.gi[it.n];
  m.down = idx >= ng;
  const int* off = m.down ? it.di : it.gi;
  const int v = m.down ? idx - ng : idx;
  int lo = 0, hi = it.n - 1;  // largest g with off[g] <= v
  if (hint >= 0 && hint < it.n && off[hint] <= v && v < off[hint + 1]) {
    lo = hint;
  } else {
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (off[mid] <= v)
        lo = mid;
      else
        hi = mid - 1;
    }
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

// The issuing thread: requests stage kc of item m into `st`, completing on
// `bar`: its 32 weight rows (wrow: first row of the item in its matrix; Q8_0
// also their scales) and its activation rows -- gate/up: the x rows xrow[0..nt)
// of the item's tokens; down: the h (or h_s) rows from row xrow[0].
//   pol: L2 policy of the weight rows (evict first: read once; a repeated chunk comes from L2 at once);
//   apol: of the activation rows (evict last: read by many items)
template <typename XT, int WK, int NT>
__device__ __forceinline__ void issue_stage(const Maps& maps, const Params& p, const Item& m, int kc, int wrow,
                                            const int (&xrow)[NT], uint8_t* st, uint64_t* bar, uint64_t pol,
                                            uint64_t apol) {
  using F = Fmt<WK>;
  constexpr bool Q8 = WK == WK_Q8;
  const int kx = kc * (Q8 ? F::KC / 4 : F::KC);  // Q8_0 codes as 32-bit words
  uint8_t* act = st + F::ACT;
  uint8_t* sc = st + F::SCL;
  const int ax = Q8 ? 0 : kx;  // activation copies: Q8_0 reads 4 rows of the 256-value view
  if constexpr (F::SPLIT) {
    if (!m.down) {
      mbar_arrive_expect_tx(bar, kRows * F::RB + m.nt * 2 * 256 * static_cast<int>(sizeof(XT)));
      const int mg = m.e < 0 ? M_SGATE : M_GATE, mu = m.e < 0 ? M_SUP : M_UP;
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        const int kxc = kx + ch * 256;
        tma_load_2d_hint(st + ch * F::PLANE, &maps.w[mg], bar, kxc, wrow, pol);
        tma_load_2d_hint(st + ch * F::PLANE + (kRows / 2) * 512, &maps.w[mu], bar, kxc, wrow, pol);
#pragma unroll
        for (int c = 0; c < NT; ++c)
          if (c < m.nt) tma_load_2d_hint(act + ch * F::APLANE + c * 1024, &maps.w[M_X], bar, kxc, xrow[c], apol);
      }
    } else {
      const int hb = m.e < 0 ? maps.hs_box : maps.h_box;
      mbar_arrive_expect_tx(bar, kRows * F::RB + 2 * hb * 256 * 4);
      const int md = m.e < 0 ? M_SDOWN : M_DOWN, mh = m.e < 0 ? M_HS : M_H;
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        tma_load_2d_hint(st + ch * F::PLANE, &maps.w[md], bar, kx + ch * 256, wrow, pol);
        tma_load_2d_hint(act + ch * F::APLANE, &maps.w[mh], bar, kx + ch * 256, xrow[0], apol);
      }
    }
    return;
  }
  if (!m.down) {
    const int xb = F::KC * static_cast<int>(sizeof(XT));
    mbar_arrive_expect_tx(bar, kRows * F::RB + kRows * F::SR + m.nt * xb);
    const int mg = m.e < 0 ? M_SGATE : M_GATE, mu = m.e < 0 ? M_SUP : M_UP;
    tma_load_2d_hint(st, &maps.w[mg], bar, kx, wrow, pol);
    tma_load_2d_hint(st + (kRows / 2) * F::RB, &maps.w[mu], bar, kx, wrow, pol);
    if constexpr (Q8) {
      tma_load_2d_hint(sc, &maps.s[mg], bar, kc * 32, wrow, pol);
      tma_load_2d_hint(sc + (kRows / 2) * F::SR, &maps.s[mu], bar, kc * 32, wrow, pol);
    }
#pragma unroll
    for (int c = 0; c < NT; ++c)
      if (c < m.nt)
        tma_load_2d_hint(act + c * F::AR, &maps.w[M_X], bar, ax, Q8 ? xrow[c] * (p.H / 256) + kc * 4 : xrow[c], apol);
  } else {
    const int md = m.e < 0 ? M_SDOWN : M_DOWN, mh = m.e < 0 ? M_HS : M_H;
    if constexpr (Q8) {
      mbar_arrive_expect_tx(bar, kRows * F::RB + kRows * F::SR + m.nt * F::AR);
      tma_load_2d_hint(st, &maps.w[md], bar, kx, wrow, pol);
      tma_load_2d_hint(sc, &maps.s[md], bar, kc * 32, wrow, pol);
      const int per = (m.e < 0 ? p.Is : p.I) / 256;
#pragma unroll
      for (int c = 0; c < NT; ++c)
        if (c < m.nt) tma_load_2d_hint(act + c * F::AR, &maps.w[mh], bar, 0, (xrow[0] + c) * per + kc * 4, apol);
    } else {
      const int hb = m.e < 0 ? maps.hs_box : maps.h_box;
      mbar_arrive_expect_tx(bar, kRows * F::RB + hb * F::KC * 4);
      tma_load_2d_hint(st, &maps.w[md], bar, kx, wrow, pol);
      tma_load_2d_hint(act, &maps.w[mh], bar, kx, xrow[0], apol);
    }
  }
}

// E16 activation values (type AT) at shared address `a`, as f32 pairs.
template <typename AT, int E16>
__device__ __forceinline__ void act_smem(uint32_t a, float2 (&x)[E16 / 2]) {
  if constexpr (sizeof(AT) == 4) {
#pragma unroll
    for (int q = 0; q < E16 / 4; ++q) {
      const uint4 v = stream::lds16(a + 16 * q);
      x[2 * q] = make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
      x[2 * q + 1] = make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
    }
  } else if constexpr (E16 == 4) {
    uint32_t v0, v1;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v0), "=r"(v1) : "r"(a));
    x[0] = stream::bf16x2_f2(v0);
    x[1] = stream::bf16x2_f2(v1);
  } else {
#pragma unroll
    for (int q = 0; q < E16 / 8; ++q) {
      const uint4 v = stream::lds16(a + 16 * q);
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
  } else if constexpr (WK == WK_BF16) {
    w[0] = stream::bf16x2_f2(v.x);
    w[1] = stream::bf16x2_f2(v.y);
    w[2] = stream::bf16x2_f2(v.z);
    w[3] = stream::bf16x2_f2(v.w);
  } else {  // Q8_0 codes, widened exactly
    stream::q8_quad(v.x, w[0], w[1]);
    stream::q8_quad(v.y, w[2], w[3]);
    stream::q8_quad(v.z, w[4], w[5]);
    stream::q8_quad(v.w, w[6], w[7]);
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

// Shared state of the stream in one CTA (shared memory).
constexpr int kMaxBatch = 4;  // most items handed out per queue step (fewer when there are few items per warp)
constexpr int kCW = 8;        // consumer warps; warp kCW issues the copies; the rest sit the stream out
constexpr int kDoneQ = 32;    // finished gate/up items waiting to be counted (at most one per stage in flight)
struct Ring {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  Item item[kStages];      // the item a stage belongs to
  int kc[kStages];         // the stage's index within its item; -1: the queue is empty
  int done_warps[kStages]; // consumer warps done with the gate/up item ending in this stage
  int dq[kDoneQ];          // group + 1 of each finished gate/up item, in claim order (0: not yet written)
  int dq_tail;             // items claimed a place in dq (consumers)
};

// Waits (bounded) until phase `parity` of `bar` completes, asleep on the barrier.  Every lane of the warp;
// false (warp-uniform) if the wait gave up.
__device__ __forceinline__ bool warp_sleep_wait(uint64_t* bar, uint32_t parity, long long limit) {
  const long long t0 = clock64();
  for (;;) {
    if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
    if (__shfl_sync(0xffffffffu, static_cast<int>(clock64() - t0 > limit), 0)) return false;
  }
}

// The stream of one CTA, until the queue is empty.  All threads of the CTA
// (16 warps).  Returns false if a wait gave up (MOE_ERR_TIMEOUT recorded).
//   stages: ring_bytes(WK) of shared memory, 128-byte aligned
//   pairs:  sorted pair ids;  wpair: routing weight per pair id;  sgate: shared-expert gate per token or nullptr
//
// Warp specialised: lane 0 of warp kCW issues every copy, asleep on a stage's empty barrier until the kCW
// consumer warps have released it; the consumers sleep on the full barriers.  Nothing polls, and the
// issuing thread may wait for the device-wide counters (the queue, a group's gate/up count) without
// holding up the consumers, which go on with the stages already in the ring.  The queue puts every gate/up
// item before every down item and each CTA takes items in queue order, so a down item only ever waits for
// gate/up items that are ahead of it in some CTA's ring or queue order: none waits on a stage that waits
// on it.
template <typename XT, int WK, int NT>
__device__ __forceinline__ bool run_stream(const Maps& maps, const Params& p, const Items& it, uint8_t* stages,
                                           Ring& ring, const int32_t* pairs, const float* wpair, const float* sgate) {
  constexpr int KC = Fmt<WK>::KC;
  constexpr int RB = Fmt<WK>::RB;
  constexpr int NCH = Fmt<WK>::NCH;
  constexpr int E16 = Fmt<WK>::E16;
  constexpr int EB = Fmt<WK>::EB;
  constexpr int NV = 2 * NT;
  static_assert(NT <= kMaxNT, "an item's activation rows fit its stage");
  static_assert(kCW * 4 == kRows && kCW < kWarps, "a consumer warp takes four rows of a stage");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int total = it.gi[it.n] + it.di[it.n];
  // items per queue step: about 16 steps per CTA, at most kMaxBatch (large items are few: batching them
  // would leave the CTAs unevenly loaded).  The first batch is the CTA's own (batch blockIdx.x), the next
  // ones come from the counter.
  const int batch = max(1, min(kMaxBatch, total / (static_cast<int>(gridDim.x) * 16)));
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ring.full[s], 1);
      mbar_init(&ring.empty[s], kCW);
      ring.done_warps[s] = 0;
    }
    for (int i = 0; i < kDoneQ; ++i) ring.dq[i] = 0;
    ring.dq_tail = 0;
    fence_mbar_init();
  }
  __syncthreads();
  bool ok = true;

  if (warp == kCW) {
    // ---- the issuing thread: items in queue order, each batch's successor claimed when the batch starts
    if (lane == 0) {
      auto claim = [&]() {
        return (static_cast<int>(gridDim.x) + static_cast<int>(atomicAdd(&p.sync->queue, 1u))) * batch;
      };
      int item = static_cast<int>(blockIdx.x) * batch;
      int end = min(total, item + batch);
      // the batch after this one, claimed when this one starts, so that the counter's answer is there when
      // needed (claims of one CTA only grow: a claim past the end ends its stream)
      int next = item < end ? claim() : total;
      const uint64_t pol = l2_policy_evict_first(), apol = l2_policy_evict_last();
      const int kshift = (p.K & (p.K - 1)) == 0 ? __ffs(p.K) - 1 : -1;  // pair -> token without a division
      unsigned gdone[(kMaxGroups + 31) / 32];  // groups whose gate/up items are all finished (known here)
#pragma unroll
      for (int i = 0; i < (kMaxGroups + 31) / 32; ++i) gdone[i] = 0;
      Item m{};
      int kc = 0, wrow = 0;
      int xr[NT];
      bool have = false;
      int dq_head = 0;
      // finished gate/up items, counted for their groups: the consumers' last warp of an item wrote the
      // entry after its item's h stores (ordered by a block fence); this thread observes the entry, and its
      // GPU fence, cumulative over what it observed, makes those stores visible before the count
      auto drain = [&]() {
        for (;;) {
          const int g1 = *reinterpret_cast<volatile int*>(&ring.dq[dq_head % kDoneQ]);
          if (g1 == 0) return;
          __threadfence_block();
          *reinterpret_cast<volatile int*>(&ring.dq[dq_head % kDoneQ]) = 0;
          ++dq_head;
          __threadfence();
          atomicAdd(&p.sync->done[g1 - 1], 1u);
        }
      };
      const long long t0 = clock64();
      // no CTA issues more stages than the whole queue holds: a bound that ends the loop whatever happens
      const long long most = static_cast<long long>(total) * ((max(p.H, max(p.I, p.Is)) + KC - 1) / KC) + kStages;
      for (uint32_t seq = 0;; ++seq) {
        const int s = static_cast<int>(seq % kStages);
        if (seq > most) {
          ok = false;
          break;
        }
        if (seq >= kStages) {
          while (!mbar_try_wait(&ring.empty[s], (seq / kStages - 1) & 1u))
            if (clock64() - t0 > p.wait_limit) {
              ok = false;
              break;
            }
          if (!ok) break;
        }
        drain();
        if (!have || kc >= m.nkc) {  // the next item, from this batch or the next
          if (have && ++item >= end) {
            item = next;
            end = min(total, item + batch);
            next = item < total ? claim() : total;
          }
          const int hint = have ? m.g : 0;
          have = true;
          kc = 0;
          if (item < end) {
            m = decode_item<NT, WK>(p, it, item, hint);
            const int first = it.first[m.g];
            if (!m.down) {
              wrow = (m.e < 0 ? 0 : m.e * p.I) + m.r0;
#pragma unroll
              for (int k = 0; k < NT; ++k) {
                const int t = m.t0 + min(k, m.nt - 1);
                const int pr = pairs[first + t];
                xr[k] = m.e < 0 ? t : (kshift >= 0 ? pr >> kshift : pr / p.K);
              }
            } else {
              wrow = (m.e < 0 ? 0 : m.e * p.H) + m.r0;
#pragma unroll
              for (int k = 0; k < NT; ++k) xr[k] = m.e < 0 ? m.t0 : first + m.t0;
              if (!(gdone[m.g >> 5] >> (m.g & 31) & 1u)) {
                // the item reads the h rows of its group: once every gate/up item of the group has counted
                // itself; then a proxy fence orders the copy engine's reads after the stores it published
                const unsigned need = static_cast<unsigned>(g_items(p, m.e, it.count[m.g], NT));
                for (;;) {
                  drain();  // this CTA's own finished items may be what the group waits for
                  unsigned v;
                  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(&p.sync->done[m.g]) : "memory");
                  if (v >= need) break;
                  if (clock64() - t0 > p.wait_limit) {
                    ok = false;
                    break;
                  }
                  __nanosleep(200);
                }
                if (!ok) {  // the slot is free: an end mark stops the consumers at once
                  ring.kc[s] = -1;
                  mbar_arrive(&ring.full[s]);
                  break;
                }
                fence_proxy_async_global();
                gdone[m.g >> 5] |= 1u << (m.g & 31);
              }
            }
          }
        }
        if (item >= end) {
          ring.kc[s] = -1;
          mbar_arrive(&ring.full[s]);  // the end mark is published through the same barrier
          // the stages still in flight may end gate/up items: once the consumers have released every one
          // of them, count the last finished items
          for (uint32_t n = seq > kStages ? seq - kStages : 0; n < seq && ok; ++n)
            while (!mbar_try_wait(&ring.empty[n % kStages], (n / kStages) & 1u))
              if (clock64() - t0 > p.wait_limit) {
                ok = false;
                break;
              }
          drain();
          break;
        }
        ring.item[s] = m;
        ring.kc[s] = kc;
        issue_stage<XT, WK, NT>(maps, p, m, kc, wrow, xr, stages + s * Fmt<WK>::SB, &ring.full[s], pol, apol);
        ++kc;
      }
      if (!ok) record_status(p.status, MOE_ERR_TIMEOUT);
    }
    __syncwarp();
    return ok;
  }
  if (warp > kCW) return true;

  // ---- consumers (warps 0 .. kCW-1): rows of pairs pi = 0, 1 -- gate/up: features f = 2w + pi (gate row f,
  // up row 16 + f); down: rows 4w + 2pi and 4w + 2pi + 1
  Item m{};
  float2 acc_a[2][NT], acc_b[2][NT];
  for (uint32_t q = 0;; ++q) {
    const int s = static_cast<int>(q % kStages);
    const uint32_t par = (q / kStages) & 1u;
    if (!warp_sleep_wait(&ring.full[s], par, p.wait_limit)) {
      record_status(p.status, MOE_ERR_TIMEOUT);
      ok = false;
      break;
    }
    const int kc = ring.kc[s];
    if (kc < 0) break;
    if (kc == 0) {  // ---- the item begins
      m = ring.item[s];
#pragma unroll
      for (int pi = 0; pi < 2; ++pi)
#pragma unroll
        for (int c = 0; c < NT; ++c) acc_a[pi][c] = acc_b[pi][c] = make_float2(0.f, 0.f);
    }
    // ---- this stage: lane chunks ch = 0..NCH-1 at bytes ch*512 + lane*16 of the warp's rows; the
    // activation rows of the item's tokens follow the weight rows, then (Q8_0) the rows' scales
    const uint32_t st = smem_addr(stages + s * Fmt<WK>::SB);
    const uint32_t act = st + Fmt<WK>::ACT;
    if constexpr (WK == WK_Q8) {
      // In each 512-code half of a row, lane l takes the 4-code groups at 4l + 128q (q = 0..3): the loads of
      // the codes (32-bit words) and of the activations (4 values) of a group are then adjacent across the
      // lanes, free of shared-memory bank conflicts (16 contiguous codes per lane would put the lanes' f32
      // activations 64 bytes apart, four to a bank).  Each group lies in one block: partial = sum q * x over
      // it, then acc += d * partial.  Token by token, the four rows' chains side by side (the codes are
      // widened again per token: most items have one or two tokens).
      const int r0 = m.down ? 4 * warp : 2 * warp, r1 = m.down ? r0 + 1 : kRows / 2 + r0;
      const int r2 = m.down ? r0 + 2 : r0 + 1, r3 = m.down ? r0 + 3 : kRows / 2 + r0 + 1;
      const int rows[4] = {r0, r1, r2, r3};
      constexpr int AB = 4 * sizeof(XT);  // activation bytes of a group (gate/up); down reads f32 h
#pragma unroll
      for (int ch = 0; ch < NCH; ++ch) {
        if (kc * KC + ch * 512 >= m.kdim) break;  // past the row: nothing to add (rows are whole 256-code units)
#pragma unroll
        for (int c = 0; c < NT; ++c) {
          if (c >= m.nt) break;
          float2 sj[4] = {};  // the four rows' sums over this half, as pairs
#pragma unroll
          for (int qh = 0; qh < 2; ++qh) {  // two groups' activations at a time
            // groups q = 2 qh, 2 qh + 1 lie in the stage's 256-code unit 2 ch + qh: past the row, nothing to add
            // (their codes are zero fill, but the activations there belong to other rows and may be anything)
            if (kc * KC + ch * 512 + qh * 256 >= m.kdim) break;
            float2 xv[2][2];
#pragma unroll
            for (int qq = 0; qq < 2; ++qq) {
              const int e = ch * 512 + 4 * lane + 128 * (2 * qh + qq);  // the group's first code
              if (m.down || sizeof(XT) == 4) {
                const uint4 v = stream::lds16(act + c * Fmt<WK>::AR + e * 4);
                xv[qq][0] = make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
                xv[qq][1] = make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
              } else {
                uint32_t v0, v1;
                asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];"
                             : "=r"(v0), "=r"(v1)
                             : "r"(act + c * Fmt<WK>::AR + e * AB / 4));
                xv[qq][0] = stream::bf16x2_f2(v0);
                xv[qq][1] = stream::bf16x2_f2(v1);
              }
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
#pragma unroll
              for (int qq = 0; qq < 2; ++qq) {
                const int q = 2 * qh + qq;
                uint16_t hv;  // the group's block scale
                asm volatile("ld.shared.u16 %0, [%1];"
                             : "=h"(hv)
                             : "r"(st + Fmt<WK>::SCL + rows[j] * Fmt<WK>::SR + (ch * 16 + (lane >> 3) + 4 * q) * 2));
                uint32_t wv;
                asm volatile("ld.shared.u32 %0, [%1];" : "=r"(wv) : "r"(st + rows[j] * RB + ch * 512 + 4 * lane + 128 * q));
                float2 lo, hi;
                stream::q8_quad(wv, lo, hi);
                const float2 pq = __ffma2_rn(hi, xv[qq][1], __fmul2_rn(lo, xv[qq][0]));
                const float d = __half2float(__ushort_as_half(hv));
                sj[j] = __ffma2_rn(make_float2(d, d), pq, sj[j]);
              }
            }
          }
          // Q8_0 sums in the .x halves of the accumulators (the .y halves stay zero)
          acc_a[0][c].x += sj[0].x + sj[0].y;
          acc_b[0][c].x += sj[1].x + sj[1].y;
          acc_a[1][c].x += sj[2].x + sj[2].y;
          acc_b[1][c].x += sj[3].x + sj[3].y;
        }
      }
    } else {
#pragma unroll
      for (int ch = 0; ch < NCH; ++ch) {
        const int kl = (ch * 512 + lane * 16) / EB;  // element within the stage
        if (kc * KC + kl < m.kdim) {  // past the row (the last stage's tail): nothing to add
          float2 xv[NT][E16 / 2];
          // bf16: chunk ch is its own plane (element kl = 256 ch + 8 lane)
          const uint32_t arow = Fmt<WK>::SPLIT ? act + ch * Fmt<WK>::APLANE : act;
          const int apitch = Fmt<WK>::SPLIT ? 1024 : Fmt<WK>::AR;
          const int ael = Fmt<WK>::SPLIT ? lane * 8 : kl;
#pragma unroll
          for (int c = 0; c < NT; ++c) {
            if (c < m.nt) {
              if (m.down)
                act_smem<float, E16>(arow + c * apitch + ael * 4, xv[c]);
              else
                act_smem<XT, E16>(arow + c * apitch + ael * static_cast<int>(sizeof(XT)), xv[c]);
            }
          }
#pragma unroll
          for (int pi = 0; pi < 2; ++pi) {
            const int ra = m.down ? 4 * warp + 2 * pi : 2 * warp + pi;
            const int rb = m.down ? ra + 1 : kRows / 2 + ra;
            float2 wa[E16 / 2], wb[E16 / 2];
            if constexpr (Fmt<WK>::SPLIT) {
              w_chunk<WK>(st + ch * Fmt<WK>::PLANE + ra * 512 + lane * 16, wa);
              w_chunk<WK>(st + ch * Fmt<WK>::PLANE + rb * 512 + lane * 16, wb);
            } else {
              w_chunk<WK>(st + ra * RB + ch * 512 + lane * 16, wa);
              w_chunk<WK>(st + rb * RB + ch * 512 + lane * 16, wb);
            }
#pragma unroll
            for (int c = 0; c < NT; ++c) {
              if (c < m.nt) {
#pragma unroll
                for (int i = 0; i < E16 / 2; ++i) {
                  acc_a[pi][c] = __ffma2_rn(wa[i], xv[c][i], acc_a[pi][c]);
                  acc_b[pi][c] = __ffma2_rn(wb[i], xv[c][i], acc_b[pi][c]);
                }
              }
            }
          }
        }
      }
    }
    if (kc == m.nkc - 1) {  // ---- the item ends: add the lanes' sums and store
      const int first = it.first[m.g];
      if (NT == 1 || m.nt == 1) {
        // one token: the four rows' sums in one butterfly; rows a0, b0, a1, b1 land in lanes 0, 8, 16, 24
        float v[4] = {acc_a[0][0].x + acc_a[0][0].y, acc_b[0][0].x + acc_b[0][0].y, acc_a[1][0].x + acc_a[1][0].y,
                      acc_b[1][0].x + acc_b[1][0].y};
        const float tot = warp_reduce_many<4>(v);
        const int t = m.t0;
        if (!m.down) {
          const float u = __shfl_down_sync(0xffffffffu, tot, 8);  // the up row's sum beside its gate row's
          if ((lane & 15) == 0) {
            const float hv = act_fn(p.act, tot) * u;
            const int f = m.r0 + 2 * warp + (lane >> 4);
            if (m.e < 0)
              p.h_s[static_cast<size_t>(t) * p.Is + f] = hv;
            else
              p.h[static_cast<size_t>(first + t) * p.I + f] = hv;
          }
        } else if ((lane & 7) == 0) {
          const int n = m.r0 + 4 * warp + (lane >> 3);
          if (m.e < 0) {
            p.y_s[static_cast<size_t>(t) * p.H + n] = (sgate ? sgate[t] : 1.f) * tot;
          } else {
            const int pr = pairs[first + t];
            p.y_slots[static_cast<size_t>(pr) * p.H + n] = wpair[pr] * tot;
          }
        }
      } else {
#pragma unroll
        for (int pi = 0; pi < 2; ++pi) {
          float v[NV];
#pragma unroll
          for (int c = 0; c < NT; ++c) {
            v[c] = acc_a[pi][c].x + acc_a[pi][c].y;
            v[NT + c] = acc_b[pi][c].x + acc_b[pi][c].y;
          }
          const float tot = warp_reduce_many<NV>(v);
          constexpr int per = 32 / NV;  // lanes holding each total; value i sits in lanes [i*per, i*per + per)
          const int vi = lane / per;
          const int c = vi % NT;
          const int t = m.t0 + min(c, m.nt - 1);
          const int pr = m.e < 0 ? t : pairs[first + t];
          if (!m.down) {
            // row a (gate) totals are values [0, NT), row b (up) [NT, 2 NT): 16 lanes higher
            const float u = __shfl_down_sync(0xffffffffu, tot, 16);
            if (lane < 16 && lane % per == 0 && c < m.nt) {
              const float hv = act_fn(p.act, tot) * u;
              const int f = m.r0 + 2 * warp + pi;
              if (m.e < 0)
                p.h_s[static_cast<size_t>(t) * p.Is + f] = hv;
              else
                p.h[static_cast<size_t>(first + t) * p.I + f] = hv;
            }
          } else if (lane % per == 0 && c < m.nt) {
            const int n = m.r0 + 4 * warp + 2 * pi + vi / NT;  // rows 4w + 2pi, 4w + 2pi + 1 of the block
            if (m.e < 0)
              p.y_s[static_cast<size_t>(t) * p.H + n] = (sgate ? sgate[t] : 1.f) * tot;
            else
              p.y_slots[static_cast<size_t>(pr) * p.H + n] = wpair[pr] * tot;
          }
        }
      }
      if (!m.down) {
        // the item's consumer warps count themselves in shared memory; the last one (which has observed
        // the others' h stores through the count) queues the item for the issuing thread to count
        __syncwarp();
        if (lane == 0) {
          __threadfence_block();
          if (atomicAdd_block(&ring.done_warps[s], 1) == kCW - 1) {
            ring.done_warps[s] = 0;  // ready for the next item ending in this stage (after the refill)
            const int slot = atomicAdd_block(&ring.dq_tail, 1);
            __threadfence_block();
            *reinterpret_cast<volatile int*>(&ring.dq[slot % kDoneQ]) = m.g + 1;
          }
        }
      }
    }
    // the warp is done with the stage
    __syncwarp();
    if (lane == 0) mbar_arrive(&ring.empty[s]);
  }
  return ok;
}

}  // namespace dstream
}  // namespace moe
