// Weight-streaming expert GEMV, shared by the standalone streaming kernels
// (stream_gemv.cu) and the fused decode kernel (decode_fused.cu).
//
// Decode reads every touched expert's weights once and does little arithmetic
// per byte (hf2q qwen35/gpu_ffn.rs: mat-vec beats tiled mat-mat at one row;
// DS4Server qwen_mtplx.rs, fused_experts: moe_glu_h then moe_down_y).  The
// work is a list of row pairs -- gate row i with up row i (gate/up), or down
// rows 2i and 2i+1 -- for each token batch of each group of rows (a touched
// expert, or the shared expert).  A persistent CTA per SM takes a contiguous
// slice of that list, balanced by cost (bytes, plus arithmetic per token for
// Q8_0).  For each token batch in its slice the CTA stages the batch's token
// rows (x for gate/up, h for down) in shared memory once; then its 16 warps
// take row pairs in turn (a CTA with few pairs splits each along K first, so
// every warp gets several units).  A warp streams its rows straight from HBM
// with coalesced 16- or 8-byte loads per lane (read once, no L1 allocation),
// a burst of loads per row in flight, after asking L2 to fetch the pair it
// will take two turns later; it dots them with the staged rows using packed
// f32x2 FMAs.  Partial sums of split pairs are added in K order.  f32 token rows are staged with their 16-byte
// groups permuted within each run of eight (group j at j ^ ((j >> 3) & 7)), so
// that lanes reading 16, 32 or 64 consecutive bytes each hit distinct banks.
// Q8_0 codes are widened exactly in registers (the exponent-bias trick: with
// the sign bit flipped, byte b is u = b + 128 and the word 0x4B0000uu is the
// float 2^23 + u) and the fp16 block scale is applied to each 8-value
// partial sum.  The k-quant stacks (Q4_K read in place, Q6_K in the split form
// of moe_q6_k_split) give each lane one 32-value chunk of a 256-value block per
// step; their codes are widened the same way and each weight is formed with one
// rounding (d s q - dmin m for Q4_K, d s (q - 32) for Q6_K) before the dots.
//
//  gate/up (DUAL): h[r, i] = act(W_gate[e,i] . a_r) * (W_up[e,i] . a_r)
//  down          : y[dest_r, j] = scale_r * (W_down[e,j] . a_r)
#pragma once

#include <algorithm>

#include "kernels.h"

namespace moe {
namespace stream {

enum { WK_F32 = 0, WK_BF16 = 1, WK_Q8 = 2, WK_Q4K = 3, WK_Q6K = 4 };

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxTok = 8;                   // token rows per batch
constexpr int kXStageBytes = 128 * 1024;     // staged token rows per CTA
constexpr int kMaxTokenRowBytes = 64 * 1024; // one staged token row
constexpr int kMaxGroups = 257;              // E <= 256 experts + the shared expert
// A CTA with fewer than kChunkPairs row pairs in a token batch splits each
// pair along K into S segments (starting at multiples of kKSegAlign) so that
// every warp has about kUnitsPerWarp units; the partial sums (at most
// kMaxUnits) are added in K order afterwards.
constexpr int kUnitsPerWarp = 3;
constexpr int kChunkPairs = kUnitsPerWarp * kWarps;
constexpr int kMaxUnits = 2 * kChunkPairs;
constexpr int kKSegAlign = 512;

// One kind of group (routed experts or the shared expert) in one phase.
struct Plan {
  int Kdim;        // reduction length (H for gate/up, I for down)
  int Nout;        // output rows per expert (I for gate/up, H for down)
  int TS;          // token rows per batch
  int npairs;      // row pairs per token batch
  int row_bytes;   // bytes of one weight row (Q8_0: the int8 codes)
  int srow_bytes;  // bytes of one row of Q8_0 scales (0 otherwise)
  int xrow_bytes;  // bytes of one staged token row
  int cost_base;   // cost of a row pair: cost_base + tokens * cost_tok
  int cost_tok;
};

// Where one kind of group reads its rows and writes its outputs.
struct GroupSrc {
  const uint8_t* w0;  // gate or down [*, Nout, Kdim] (expert e starts at row e * Nout)
  const uint8_t* w1;  // up (gate/up only)
  const uint8_t* s0;  // Q8_0 scales of w0 / w1 [*, Nout, Kdim / 32] fp16
  const uint8_t* s1;
  const uint8_t* act;      // token rows, xrow_bytes apart
  float* out;              // output rows of Nout f32
  const float* row_scale;  // down: weight per row (nullptr: 1)
  int act_via_pairs;       // token row of row r = pairs[r] / K (else r)
  int out_via_pairs;       // output row of row r = pairs[r] (else r)
  int scale_via_pairs;     // scale of row r = row_scale[pairs[r]] (else row_scale[r])
};

struct Phase {
  GroupSrc src[2];       // [0] routed experts, [1] the shared expert
  Plan plan[2];
  const int32_t* pairs;  // sorted pair ids (global or shared memory); nullptr = identity
  int K;
  int act_fn;
};

// Per-CTA tables in shared memory.  Group g: expert[g] (-1 = shared expert),
// rows [first[g], first[g] + count[g]); its row pairs are [poff[g], poff[g+1])
// of the phase's list (batch-major), its cost [coff[g], coff[g+1]).
struct Tables {
  int* expert;
  int* first;
  int* count;
  int* poff;
  long long* coff;
  int n;
};

// Shared memory a streaming CTA uses.
struct Smem {
  uint8_t* xs;   // kXStageBytes of staged token rows
  int* arow;     // [kMaxTok] source row of each staged token row
  int* dest;     // [kMaxTok] output row of each token row
  float* scale;  // [kMaxTok] down: weight of each token row
  float* part;   // [kMaxUnits][kMaxTok][2] partial dot products of split row pairs
};

// ---------------------------------------------------------------- host planning
// Weight kinds of the gate/up and of the down projections of a layer format.
inline int wk_gate_up(int w_dtype) {
  switch (w_dtype) {
    case MOE_F32: return WK_F32;
    case MOE_BF16: return WK_BF16;
    case MOE_Q8_0: return WK_Q8;
    default: return WK_Q4K;  // MOE_Q4_K, MOE_Q4_K_Q6_K
  }
}
inline int wk_down(int w_dtype) { return w_dtype == MOE_Q4_K_Q6_K ? WK_Q6K : wk_gate_up(w_dtype); }

// Bytes of the scale row of a Q6_K split matrix with Kdim inputs: 16 int8
// scales per block, then one fp16 d per block, padded to 16 bytes.
__host__ __device__ constexpr int q6k_srow_bytes(int Kdim) { return ((Kdim / 256) * 18 + 15) / 16 * 16; }

inline Plan make_plan(int wk, bool dual, int Kdim, int Nout, int act_bytes_per_elem, int max_tokens,
                      int tok_cap = kMaxTok) {
  Plan p{};
  p.Kdim = Kdim;
  p.Nout = Nout;
  const int eb = wk == WK_F32 ? 4 : (wk == WK_BF16 ? 2 : 1);
  p.row_bytes = wk == WK_Q4K ? (Kdim / 256) * 144 : (wk == WK_Q6K ? (Kdim / 256) * 192 : Kdim * eb);
  p.srow_bytes = wk == WK_Q8 ? (Kdim / 32) * 2 : (wk == WK_Q6K ? q6k_srow_bytes(Kdim) : 0);
  p.xrow_bytes = Kdim * act_bytes_per_elem;
  p.TS = std::max(1, std::min(std::min(kMaxTok, tok_cap), max_tokens));
  while (p.TS > 1 && p.TS * p.xrow_bytes > kXStageBytes) --p.TS;
  p.npairs = dual ? Nout : (Nout + 1) / 2;
  // a pair streams 2 rows of weights; Q8_0 spends about 1 ALU op per weight
  // per token on top of the widening, f32 / bf16 far less than the bytes cost
  p.cost_base = 2 * (p.row_bytes + p.srow_bytes) / 64 + 1;
  const bool kq = wk == WK_Q4K || wk == WK_Q6K;
  if (kq) p.cost_base += 2 * Kdim / 128;  // forming the weights costs ALU work of its own
  p.cost_tok = (wk == WK_Q8 || kq) ? std::max(1, 2 * Kdim / 256) : std::max(1, 2 * Kdim / 2048);
  return p;
}

// ---------------------------------------------------------------- device side
// ---- loads ----
__device__ __forceinline__ uint4 ld_stream16(const void* p) {  // read once: no L1 allocation
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ uint2 ld_stream8(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];"
               : "=r"(v.x), "=r"(v.y)
               : "l"(p));
  return v;
}
__device__ __forceinline__ uint16_t ld_stream2(const void* p) {
  uint16_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ uint4 lds16(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ uint2 lds8(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }
__device__ __forceinline__ float2 bf16x2_f2(uint32_t w) {
  return f2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// ---- one weight chunk per lane and step ----
// F32: 4 weights (16 bytes); BF16: 4 weights (8 bytes); Q8: 8 codes (8 bytes,
// within one scale block).
__host__ __device__ constexpr int chunk_v(int wk, int nt) { return (void)nt, wk == WK_Q8 ? 8 : 4; }

template <int WK, int NT>
struct Chunk;
template <int NT>
struct Chunk<WK_F32, NT> {
  static constexpr int V = chunk_v(WK_F32, NT);
  uint4 r;
  __device__ __forceinline__ void load(const uint8_t* row, int k) { r = ld_stream16(row + 4 * k); }
};
template <int NT>
struct Chunk<WK_BF16, NT> {
  static constexpr int V = chunk_v(WK_BF16, NT);
  uint2 r;
  __device__ __forceinline__ void load(const uint8_t* row, int k) { r = ld_stream8(row + 2 * k); }
};
template <int NT>
struct Chunk<WK_Q8, NT> {
  static constexpr int V = chunk_v(WK_Q8, NT);
  uint32_t r[V / 4];
  uint16_t s;
  __device__ __forceinline__ void load(const uint8_t* row, int k) {
    if constexpr (V == 16) {
      const uint4 v = ld_stream16(row + k);
      r[0] = v.x;
      r[1] = v.y;
      r[2] = v.z;
      r[3] = v.w;
    } else {
      const uint2 v = ld_stream8(row + k);
      r[0] = v.x;
      r[1] = v.y;
    }
  }
};

// Position of 16-byte group j of a staged f32 row.
__device__ __forceinline__ int swz(int j) { return j ^ ((j >> 3) & 7); }

// V token values of one staged row at element k (a multiple of V), as f32 pairs.
template <typename AT, int V>
__device__ __forceinline__ void x_chunk(uint32_t row, int k, float2 (&x)[V / 2]) {
  if constexpr (sizeof(AT) == 4) {
#pragma unroll
    for (int q = 0; q < V / 4; ++q) {
      const uint4 a = lds16(row + 16 * swz(k / 4 + q));
      x[2 * q] = f2(__uint_as_float(a.x), __uint_as_float(a.y));
      x[2 * q + 1] = f2(__uint_as_float(a.z), __uint_as_float(a.w));
    }
  } else if constexpr (V == 4) {
    const uint2 a = lds8(row + 2 * k);
    x[0] = bf16x2_f2(a.x);
    x[1] = bf16x2_f2(a.y);
  } else {
#pragma unroll
    for (int q = 0; q < V / 8; ++q) {
      const uint4 a = lds16(row + 2 * k + 16 * q);
      x[4 * q] = bf16x2_f2(a.x);
      x[4 * q + 1] = bf16x2_f2(a.y);
      x[4 * q + 2] = bf16x2_f2(a.z);
      x[4 * q + 3] = bf16x2_f2(a.w);
    }
  }
}

// Widens a chunk to f32 pairs, in element order.
__device__ __forceinline__ void q8_quad(uint32_t w, float2& lo, float2& hi) {
  const uint32_t u = w ^ 0x80808080u;
  const float2 bias = f2(-8388736.0f, -8388736.0f);  // -(2^23 + 128)
  lo = __fadd2_rn(f2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7650)),
                     __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7651))), bias);
  hi = __fadd2_rn(f2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7652)),
                     __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7653))), bias);
}

template <int WK, int NT>
__device__ __forceinline__ void w_chunk(const Chunk<WK, NT>& c, float2 (&w)[Chunk<WK, NT>::V / 2]) {
  if constexpr (WK == WK_F32) {
    w[0] = f2(__uint_as_float(c.r.x), __uint_as_float(c.r.y));
    w[1] = f2(__uint_as_float(c.r.z), __uint_as_float(c.r.w));
  } else if constexpr (WK == WK_BF16) {
    w[0] = bf16x2_f2(c.r.x);
    w[1] = bf16x2_f2(c.r.y);
  } else {
#pragma unroll
    for (int i = 0; i < Chunk<WK, NT>::V / 4; ++i) q8_quad(c.r[i], w[2 * i], w[2 * i + 1]);
  }
}

// ---- work list ----
__device__ __forceinline__ int batches_of(const Plan& pl, int count) { return (count + pl.TS - 1) / pl.TS; }

__device__ __forceinline__ long long group_cost(const Plan& pl, int count) {
  const int nb = batches_of(pl, count);
  const int last = count - (nb - 1) * pl.TS;
  return static_cast<long long>(pl.npairs) *
         ((nb - 1) * static_cast<long long>(pl.cost_base + pl.TS * pl.cost_tok) + pl.cost_base + last * pl.cost_tok);
}

// Fills tb.poff / tb.coff (prefix sums of pairs and cost over the groups).
// Called by one whole warp.
__device__ __forceinline__ void build_prefix(const Tables& tb, const Phase& ph) {
  const int lane = threadIdx.x & 31;
  const int per = (tb.n + 31) / 32;
  const int g0 = min(tb.n, lane * per), g1 = min(tb.n, g0 + per);
  int sp = 0;
  long long sc = 0;
  for (int g = g0; g < g1; ++g) {
    const Plan& pl = ph.plan[tb.expert[g] < 0 ? 1 : 0];
    sp += batches_of(pl, tb.count[g]) * pl.npairs;
    sc += group_cost(pl, tb.count[g]);
  }
  int ep = sp;
  long long ec = sc;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, ep, o);
    const long long b = __shfl_up_sync(0xffffffffu, ec, o);
    if (lane >= o) {
      ep += a;
      ec += b;
    }
  }
  int rp = ep - sp;
  long long rc = ec - sc;
  for (int g = g0; g < g1; ++g) {
    tb.poff[g] = rp;
    tb.coff[g] = rc;
    const Plan& pl = ph.plan[tb.expert[g] < 0 ? 1 : 0];
    rp += batches_of(pl, tb.count[g]) * pl.npairs;
    rc += group_cost(pl, tb.count[g]);
  }
  if (lane == 31) {
    tb.poff[tb.n] = ep;
    tb.coff[tb.n] = ec;
  }
  __syncwarp();
}

// Last index g in [0, n] with off[g] <= v.
template <typename T>
__device__ __forceinline__ int last_le(const T* off, int n, T v) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= v)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

// First pair of the list whose cost starts at or after `x`.
__device__ __forceinline__ int first_pair_at(const Tables& tb, const Phase& ph, long long x) {
  const int g = last_le(tb.coff, tb.n, x);
  if (g >= tb.n) return tb.poff[tb.n];
  const Plan& pl = ph.plan[tb.expert[g] < 0 ? 1 : 0];
  const long long full = static_cast<long long>(pl.npairs) * (pl.cost_base + pl.TS * pl.cost_tok);
  const int nb = batches_of(pl, tb.count[g]);
  long long r = x - tb.coff[g];
  const int b = static_cast<int>(min(static_cast<long long>(nb - 1), r / full));
  r -= b * full;
  const int nt = min(pl.TS, tb.count[g] - b * pl.TS);
  const long long per = pl.cost_base + nt * pl.cost_tok;
  const int i = static_cast<int>((r + per - 1) / per);
  return min(tb.poff[g] + b * pl.npairs + i, tb.poff[g + 1]);
}

// This CTA's pairs: those whose cost starts in its even share of the total.
__device__ __forceinline__ void cta_pairs(const Tables& tb, const Phase& ph, int& p0, int& p1) {
  const long long c = tb.coff[tb.n];
  p0 = first_pair_at(tb, ph, c * blockIdx.x / gridDim.x);
  p1 = first_pair_at(tb, ph, c * (blockIdx.x + 1) / gridDim.x);
}

// Stages the token rows of one batch (nr rows from row rc of group kind
// `kind`) into shared memory, f32 rows permuted by swz().  All threads of the
// CTA; ends synchronised.
__device__ __forceinline__ void stage_rows(const Phase& ph, int kind, int rc, int nr, const Smem& sm, bool f32) {
  const GroupSrc& src = ph.src[kind];
  const Plan& pl = ph.plan[kind];
  if (threadIdx.x < nr) {
    const int r = rc + threadIdx.x;
    const bool need = ph.pairs && (src.act_via_pairs | src.out_via_pairs | src.scale_via_pairs);
    const int dest = need ? ph.pairs[r] : r;
    sm.arow[threadIdx.x] = src.act_via_pairs ? dest / ph.K : r;
    sm.dest[threadIdx.x] = src.out_via_pairs ? dest : r;
    sm.scale[threadIdx.x] = src.row_scale ? src.row_scale[src.scale_via_pairs ? dest : r] : 1.f;
  }
  __syncthreads();
  const int n16 = pl.xrow_bytes / 16;
  for (int i = threadIdx.x; i < nr * n16; i += blockDim.x) {
    const int c = i / n16, o = i - c * n16;
    const uint4 v =
        __ldcg(reinterpret_cast<const uint4*>(src.act + static_cast<size_t>(sm.arow[c]) * pl.xrow_bytes) + o);
    reinterpret_cast<uint4*>(sm.xs + c * pl.xrow_bytes)[f32 ? swz(o) : o] = v;
  }
  __syncthreads();
}

// Writes the outputs of row pair pi for token row c (of the staged batch).
template <bool DUAL>
__device__ __forceinline__ void pair_out(const Phase& ph, int kind, int pi, int c, float va, float vb,
                                         const Smem& sm) {
  const GroupSrc& src = ph.src[kind];
  const Plan& pl = ph.plan[kind];
  float* orow = src.out + static_cast<size_t>(sm.dest[c]) * pl.Nout;
  if (DUAL) {
    orow[pi] = act_fn(ph.act_fn, va) * vb;
  } else {
    orow[2 * pi] = sm.scale[c] * va;
    if (2 * pi + 1 < pl.Nout) orow[2 * pi + 1] = sm.scale[c] * vb;
  }
}

// Dot products of elements [kb, ke) of weight rows A and B (in HBM) with NT
// staged token rows (shared memory at `xs`, xrow_bytes apart); kb is a
// multiple of kKSegAlign.  Lane partial sums are reduced over the warp; lane
// c < NT returns token c's values in va, vb.
// U1: loads in flight per lane and row for one token (8 in code compiled for one token per batch, whose
// registers allow it; 4 otherwise).
template <int NT, int WK, typename AT, int U1 = 4>
__device__ __forceinline__ void pair_dot(const uint8_t* wa, const uint8_t* wb, const uint8_t* sa, const uint8_t* sb,
                                         uint32_t xs, int xrow_bytes, int kb, int ke, float& va, float& vb) {
  constexpr int V = Chunk<WK, NT>::V;
  constexpr int U = NT == 1 ? U1 : (NT == 2 ? 2 : 1);  // loads in flight per lane and row in each round
  const int lane = threadIdx.x & 31;
  float2 acc_a[NT], acc_b[NT];
#pragma unroll
  for (int c = 0; c < NT; ++c) acc_a[c] = acc_b[c] = f2(0.f, 0.f);
  for (int k0 = kb + lane * V; k0 < ke; k0 += 32 * V * U) {
    Chunk<WK, NT> ca[U], cb[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int k = k0 + 32 * V * u;
      if (k < ke) {
        ca[u].load(wa, k);
        cb[u].load(wb, k);
        if constexpr (WK == WK_Q8) {
          ca[u].s = ld_stream2(sa + 2 * (k >> 5));
          cb[u].s = ld_stream2(sb + 2 * (k >> 5));
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int k = k0 + 32 * V * u;
      if (k < ke) {
        float2 wva[V / 2], wvb[V / 2];
        w_chunk<WK, NT>(ca[u], wva);
        w_chunk<WK, NT>(cb[u], wvb);
        float2 sca, scb;
        if constexpr (WK == WK_Q8) {
          const float s_a = __half2float(__ushort_as_half(ca[u].s));
          const float s_b = __half2float(__ushort_as_half(cb[u].s));
          sca = f2(s_a, s_a);
          scb = f2(s_b, s_b);
        }
#pragma unroll
        for (int c = 0; c < NT; ++c) {
          float2 xv[V / 2];
          x_chunk<AT, V>(xs + c * xrow_bytes, k, xv);
          if constexpr (WK == WK_Q8) {
            float2 pa = __fmul2_rn(wva[0], xv[0]);
            float2 pb = __fmul2_rn(wvb[0], xv[0]);
#pragma unroll
            for (int i = 1; i < V / 2; ++i) {
              pa = __ffma2_rn(wva[i], xv[i], pa);
              pb = __ffma2_rn(wvb[i], xv[i], pb);
            }
            acc_a[c] = __ffma2_rn(sca, pa, acc_a[c]);
            acc_b[c] = __ffma2_rn(scb, pb, acc_b[c]);
          } else {
#pragma unroll
            for (int i = 0; i < V / 2; ++i) {
              acc_a[c] = __ffma2_rn(wva[i], xv[i], acc_a[c]);
              acc_b[c] = __ffma2_rn(wvb[i], xv[i], acc_b[c]);
            }
          }
        }
      }
    }
  }
  va = vb = 0.f;
#pragma unroll
  for (int c = 0; c < NT; ++c) {
    const float sa_ = warp_sum(acc_a[c].x + acc_a[c].y);
    const float sb_ = warp_sum(acc_b[c].x + acc_b[c].y);
    if (lane == c) {
      va = sa_;
      vb = sb_;
    }
  }
}

// ---- k-quant stacks ----
// Four unsigned bytes (codes below 2^8) widened exactly and offset by `bias`
// (-2^23 gives the code, -(2^23 + 32) the centred Q6_K code).
__device__ __forceinline__ void u8x4(uint32_t v, float bias, float2& lo, float2& hi) {
  const float2 b = f2(bias, bias);
  lo = __fadd2_rn(f2(__uint_as_float(__byte_perm(v, 0x4B000000u, 0x7650)),
                     __uint_as_float(__byte_perm(v, 0x4B000000u, 0x7651))), b);
  hi = __fadd2_rn(f2(__uint_as_float(__byte_perm(v, 0x4B000000u, 0x7652)),
                     __uint_as_float(__byte_perm(v, 0x4B000000u, 0x7653))), b);
}

// Token values [p, p + 4) of a staged row (p a multiple of 4).
template <typename AT>
__device__ __forceinline__ void x4(uint32_t row, int p, float2& a, float2& b) {
  if constexpr (sizeof(AT) == 4) {
    const uint4 v = lds16(row + 16 * swz(p >> 2));
    a = f2(__uint_as_float(v.x), __uint_as_float(v.y));
    b = f2(__uint_as_float(v.z), __uint_as_float(v.w));
  } else {
    const uint2 v = lds8(row + 2 * p);
    a = bf16x2_f2(v.x);
    b = bf16x2_f2(v.y);
  }
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int i) {
  return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

// Scale d s_j and offset dmin m_j of sub-block j (32 values) of a Q4_K block
// whose 16-byte head is h = {d, dmin | scales[0..3] | scales[4..7] | scales[8..11]}.
__device__ __forceinline__ void q4k_sub(const uint4& h, int j, float& dsc, float& dm) {
  const float d = __half2float(__ushort_as_half(static_cast<unsigned short>(h.x & 0xFFFFu)));
  const float dmin = __half2float(__ushort_as_half(static_cast<unsigned short>(h.x >> 16)));
  uint32_t sc, mn;
  if (j < 4) {
    sc = (h.y >> (8 * j)) & 63u;
    mn = (h.z >> (8 * j)) & 63u;
  } else {
    const int sh = 8 * (j - 4);
    const uint32_t lo = h.w >> sh;
    sc = (lo & 15u) | (((h.y >> sh) >> 6 & 3u) << 4);
    mn = (lo >> 4 & 15u) | (((h.z >> sh) >> 6 & 3u) << 4);
  }
  dsc = d * static_cast<float>(sc);  // exact: 11 x 6 bits
  dm = dmin * static_cast<float>(mn);
}

// Q4_K dot of two rows (blocks of 144 bytes read in place).  Chunk q of a
// block holds qs bytes [16q, 16q + 16): low nibbles are values
// 64c + 16h + [0, 16) of sub-block 2c, high nibbles values 64c + 32 + 16h +
// [0, 16) of sub-block 2c + 1 (c = q / 2, h = q % 2).
template <int NT, typename AT>
__device__ __forceinline__ void q4k_pair_dot(const uint8_t* wa, const uint8_t* wb, uint32_t xs, int xrow_bytes,
                                             int kb, int ke, float2 (&acc_a)[NT], float2 (&acc_b)[NT]) {
  const int lane = threadIdx.x & 31;
  const float bias = -8388608.0f;  // -2^23
  for (int k = kb + 32 * lane; k < ke; k += 32 * 32) {
    const int blk = k >> 8, q = (k >> 5) & 7, c2 = q >> 1;
    const uint8_t* ba = wa + blk * 144;
    const uint8_t* bb = wb + blk * 144;
    const uint4 ha = ld_stream16(ba), hb = ld_stream16(bb);
    const uint4 qa = ld_stream16(ba + 16 + 16 * q), qb = ld_stream16(bb + 16 + 16 * q);
    float sa0, ma0, sa1, ma1, sb0, mb0, sb1, mb1;
    q4k_sub(ha, 2 * c2, sa0, ma0);
    q4k_sub(ha, 2 * c2 + 1, sa1, ma1);
    q4k_sub(hb, 2 * c2, sb0, mb0);
    q4k_sub(hb, 2 * c2 + 1, sb1, mb1);
    const int p0 = (blk << 8) + 64 * c2 + 16 * (q & 1);
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
      float2 a[4], b[4];  // [low run: 2 pairs | high run: 2 pairs]
      const uint32_t va = word_of(qa, wi), vb = word_of(qb, wi);
      u8x4(va & 0x0F0F0F0Fu, bias, a[0], a[1]);
      u8x4((va >> 4) & 0x0F0F0F0Fu, bias, a[2], a[3]);
      u8x4(vb & 0x0F0F0F0Fu, bias, b[0], b[1]);
      u8x4((vb >> 4) & 0x0F0F0F0Fu, bias, b[2], b[3]);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        a[i] = __ffma2_rn(f2(sa0, sa0), a[i], f2(-ma0, -ma0));
        a[2 + i] = __ffma2_rn(f2(sa1, sa1), a[2 + i], f2(-ma1, -ma1));
        b[i] = __ffma2_rn(f2(sb0, sb0), b[i], f2(-mb0, -mb0));
        b[2 + i] = __ffma2_rn(f2(sb1, sb1), b[2 + i], f2(-mb1, -mb1));
      }
#pragma unroll
      for (int c = 0; c < NT; ++c) {
        float2 x[4];
        x4<AT>(xs + c * xrow_bytes, p0 + 4 * wi, x[0], x[1]);
        x4<AT>(xs + c * xrow_bytes, p0 + 32 + 4 * wi, x[2], x[3]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc_a[c] = __ffma2_rn(a[i], x[i], acc_a[c]);
          acc_b[c] = __ffma2_rn(b[i], x[i], acc_b[c]);
        }
      }
    }
  }
}

// Q6_K dot of two rows in the split form: quant rows of 192-byte blocks
// (ql[128] | qh[64]) and scale rows (16 int8 scales per block, then the fp16
// d of each block).  Chunk q of a block is half n = q / 4 and l-range
// [8m, 8m + 8) (m = q % 4): values 128n + 32i + 8m + [0, 8), i = 0..3, with
// low bits from ql[64n + 8m + 32 (i & 1)] (low nibbles for i < 2, high for
// i >= 2), high bits (qh[32n + 8m] >> 2i) & 3, scale sc[8n + 2i + m / 2].
template <int NT, typename AT>
__device__ __forceinline__ void q6k_pair_dot(const uint8_t* wa, const uint8_t* wb, const uint8_t* sa,
                                             const uint8_t* sb, int Kdim, uint32_t xs, int xrow_bytes, int kb, int ke,
                                             float2 (&acc_a)[NT], float2 (&acc_b)[NT]) {
  const int lane = threadIdx.x & 31;
  const int nb = Kdim >> 8;
  const float bias = -8388640.0f;  // -(2^23 + 32)
  for (int k = kb + 32 * lane; k < ke; k += 32 * 32) {
    const int blk = k >> 8, q = (k >> 5) & 7, n = q >> 2, m = q & 3;
    const uint8_t* ba = wa + blk * 192 + 64 * n + 8 * m;
    const uint8_t* bb = wb + blk * 192 + 64 * n + 8 * m;
    const uint2 la = ld_stream8(ba), ha = ld_stream8(ba + 32), qa = ld_stream8(ba + 128 - 32 * n);
    const uint2 lb = ld_stream8(bb), hb = ld_stream8(bb + 32), qb = ld_stream8(bb + 128 - 32 * n);
    const uint2 sca = ld_stream8(sa + 16 * blk + 8 * n), scb = ld_stream8(sb + 16 * blk + 8 * n);
    const float da = __half2float(__ushort_as_half(ld_stream2(sa + 16 * nb + 2 * blk)));
    const float db = __half2float(__ushort_as_half(ld_stream2(sb + 16 * nb + 2 * blk)));
    float dsa[4], dsb[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int bi = 2 * i + (m >> 1);  // scale byte within sc[8n .. 8n + 8)
      const uint32_t wsa = bi < 4 ? sca.x : sca.y, wsb = bi < 4 ? scb.x : scb.y;
      dsa[i] = da * static_cast<float>(static_cast<int8_t>((wsa >> (8 * (bi & 3))) & 0xFFu));  // exact: 11 x 8 bits
      dsb[i] = db * static_cast<float>(static_cast<int8_t>((wsb >> (8 * (bi & 3))) & 0xFFu));
    }
    const int p0 = (blk << 8) + 128 * n + 8 * m;
#pragma unroll
    for (int wi = 0; wi < 2; ++wi) {
      const uint32_t L_a = wi ? la.y : la.x, H_a = wi ? ha.y : ha.x, Q_a = wi ? qa.y : qa.x;
      const uint32_t L_b = wi ? lb.y : lb.x, H_b = wi ? hb.y : hb.x, Q_b = wi ? qb.y : qb.x;
      const uint32_t ca[4] = {(L_a & 0x0F0F0F0Fu) | ((Q_a << 4) & 0x30303030u),
                              (H_a & 0x0F0F0F0Fu) | ((Q_a << 2) & 0x30303030u),
                              ((L_a >> 4) & 0x0F0F0F0Fu) | (Q_a & 0x30303030u),
                              ((H_a >> 4) & 0x0F0F0F0Fu) | ((Q_a >> 2) & 0x30303030u)};
      const uint32_t cb[4] = {(L_b & 0x0F0F0F0Fu) | ((Q_b << 4) & 0x30303030u),
                              (H_b & 0x0F0F0F0Fu) | ((Q_b << 2) & 0x30303030u),
                              ((L_b >> 4) & 0x0F0F0F0Fu) | (Q_b & 0x30303030u),
                              ((H_b >> 4) & 0x0F0F0F0Fu) | ((Q_b >> 2) & 0x30303030u)};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float2 a0, a1, b0, b1;
        u8x4(ca[i], bias, a0, a1);
        u8x4(cb[i], bias, b0, b1);
        a0 = __fmul2_rn(f2(dsa[i], dsa[i]), a0);
        a1 = __fmul2_rn(f2(dsa[i], dsa[i]), a1);
        b0 = __fmul2_rn(f2(dsb[i], dsb[i]), b0);
        b1 = __fmul2_rn(f2(dsb[i], dsb[i]), b1);
#pragma unroll
        for (int c = 0; c < NT; ++c) {
          float2 x0, x1;
          x4<AT>(xs + c * xrow_bytes, p0 + 32 * i + 4 * wi, x0, x1);
          acc_a[c] = __ffma2_rn(a0, x0, acc_a[c]);
          acc_a[c] = __ffma2_rn(a1, x1, acc_a[c]);
          acc_b[c] = __ffma2_rn(b0, x0, acc_b[c]);
          acc_b[c] = __ffma2_rn(b1, x1, acc_b[c]);
        }
      }
    }
  }
}

// Warp sums of the lane accumulators: lane c < NT receives token c's values.
template <int NT>
__device__ __forceinline__ void pair_reduce(const float2 (&acc_a)[NT], const float2 (&acc_b)[NT], float& va,
                                            float& vb) {
  const int lane = threadIdx.x & 31;
  va = vb = 0.f;
#pragma unroll
  for (int c = 0; c < NT; ++c) {
    const float sa_ = warp_sum(acc_a[c].x + acc_a[c].y);
    const float sb_ = warp_sum(acc_b[c].x + acc_b[c].y);
    if (lane == c) {
      va = sa_;
      vb = sb_;
    }
  }
}

__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Asks L2 to fetch the weight rows (and 16-byte multiples of Q8_0 scale rows)
// of row pair pi: lane 0 of a warp.
template <int WK, bool DUAL>
__device__ __forceinline__ void prefetch_pair(const Phase& ph, int kind, int e, int pi) {
  const GroupSrc& src = ph.src[kind];
  const Plan& pl = ph.plan[kind];
  const size_t row0 = static_cast<size_t>(e < 0 ? 0 : e) * pl.Nout;
  const int ia = DUAL ? pi : 2 * pi;
  const int nb = DUAL ? 1 : min(2, pl.Nout - ia);  // down: rows ia, ia+1 are contiguous
  prefetch_l2(src.w0 + (row0 + ia) * pl.row_bytes, nb * pl.row_bytes);
  if (DUAL) prefetch_l2(src.w1 + (row0 + ia) * pl.row_bytes, pl.row_bytes);
  if ((WK == WK_Q8 || WK == WK_Q6K) && (pl.srow_bytes % 16) == 0) {
    prefetch_l2(src.s0 + (row0 + ia) * pl.srow_bytes, nb * pl.srow_bytes);
    if (DUAL) prefetch_l2(src.s1 + (row0 + ia) * pl.srow_bytes, pl.srow_bytes);
  }
}

// Elements [kb, ke) of row pair pi for NT tokens.  part == nullptr: the whole
// row, outputs written; else the partial sums go to part[c][0..1].
template <int NT, typename AT, int WK, bool DUAL, int MAXNT>
__device__ __forceinline__ void run_unit(const Phase& ph, int kind, int e, int pi, int kb, int ke, float* part,
                                         const Smem& sm) {
  const GroupSrc& src = ph.src[kind];
  const Plan& pl = ph.plan[kind];
  const int lane = threadIdx.x & 31;
  const size_t row0 = static_cast<size_t>(e < 0 ? 0 : e) * pl.Nout;
  const int ia = DUAL ? pi : 2 * pi;
  const int ib = DUAL ? pi : min(2 * pi + 1, pl.Nout - 1);
  const uint8_t* wa = src.w0 + (row0 + ia) * pl.row_bytes;
  const uint8_t* wb = (DUAL ? src.w1 : src.w0) + (row0 + ib) * pl.row_bytes;
  constexpr bool scaled = WK == WK_Q8 || WK == WK_Q6K;  // weights with a scale plane
  const uint8_t* sa = scaled ? src.s0 + (row0 + ia) * pl.srow_bytes : nullptr;
  const uint8_t* sb = scaled ? (DUAL ? src.s1 : src.s0) + (row0 + ib) * pl.srow_bytes : nullptr;
  float va, vb;
  if constexpr (WK == WK_Q4K || WK == WK_Q6K) {
    float2 acc_a[NT], acc_b[NT];
#pragma unroll
    for (int c = 0; c < NT; ++c) acc_a[c] = acc_b[c] = f2(0.f, 0.f);
    if constexpr (WK == WK_Q4K)
      q4k_pair_dot<NT, AT>(wa, wb, smem_addr(sm.xs), pl.xrow_bytes, kb, ke, acc_a, acc_b);
    else
      q6k_pair_dot<NT, AT>(wa, wb, sa, sb, pl.Kdim, smem_addr(sm.xs), pl.xrow_bytes, kb, ke, acc_a, acc_b);
    pair_reduce<NT>(acc_a, acc_b, va, vb);
  } else {
    pair_dot<NT, WK, AT, MAXNT == 1 ? 8 : 4>(wa, wb, sa, sb, smem_addr(sm.xs), pl.xrow_bytes, kb, ke, va, vb);
  }
  if (lane < NT) {
    if (part) {
      part[2 * lane] = va;
      part[2 * lane + 1] = vb;
    } else {
      pair_out<DUAL>(ph, kind, pi, lane, va, vb, sm);
    }
  }
}

// Straight-line code for each token count up to MAXNT (the plans' TS bound).
template <typename AT, int WK, bool DUAL, int MAXNT>
__device__ __forceinline__ void unit_nt(int nr, const Phase& ph, int kind, int e, int pi, int kb, int ke, float* part,
                                        const Smem& sm) {
  if constexpr (MAXNT == 1) {
    (void)nr;
    run_unit<1, AT, WK, DUAL, MAXNT>(ph, kind, e, pi, kb, ke, part, sm);
  } else {
    if (MAXNT <= 4 || nr <= 4) {
      switch (nr) {
        case 1: run_unit<1, AT, WK, DUAL, MAXNT>(ph, kind, e, pi, kb, ke, part, sm); break;
        case 2: run_unit<2, AT, WK, DUAL, MAXNT>(ph, kind, e, pi, kb, ke, part, sm); break;
        case 3: run_unit<3, AT, WK, DUAL, MAXNT>(ph, kind, e, pi, kb, ke, part, sm); break;
        default: run_unit<4, AT, WK, DUAL, MAXNT>(ph, kind, e, pi, kb, ke, part, sm); break;
      }
    } else if constexpr (MAXNT > 4) {
      switch (nr) {
        case 5: run_unit<5, AT, WK, DUAL, MAXNT>(ph, kind, e, pi, kb, ke, part, sm); break;
        case 6: run_unit<6, AT, WK, DUAL, MAXNT>(ph, kind, e, pi, kb, ke, part, sm); break;
        case 7: run_unit<7, AT, WK, DUAL, MAXNT>(ph, kind, e, pi, kb, ke, part, sm); break;
        default: run_unit<8, AT, WK, DUAL, MAXNT>(ph, kind, e, pi, kb, ke, part, sm); break;
      }
    }
  }
}

// Runs this CTA's slice [p0, p1) of a phase's pair list.  All threads.
template <typename AT, int WK, bool DUAL, int MAXNT>
__device__ __forceinline__ void run_phase(const Phase& ph, const Tables& tb, int p0, int p1, const Smem& sm) {
  const int warp = threadIdx.x >> 5;
  int p = p0;
  while (p < p1) {
    const int g = last_le(tb.poff, tb.n - 1, p);
    const int e = tb.expert[g];
    const int kind = e < 0 ? 1 : 0;
    const Plan& pl = ph.plan[kind];
    const int local = p - tb.poff[g];
    const int b = local / pl.npairs;
    const int pi0 = local - b * pl.npairs;
    const int rc = tb.first[g] + b * pl.TS;
    const int nr = min(pl.TS, tb.first[g] + tb.count[g] - rc);
    const int seg = min(p1 - p, pl.npairs - pi0);  // pairs of this batch in the slice
    // K segments per pair so that the warps get about kUnitsPerWarp units each
    const int S = seg >= kChunkPairs ? 1 : max(1, min((kChunkPairs + seg - 1) / seg, pl.Kdim / kKSegAlign));
    const int kseg = S == 1 ? pl.Kdim : ((pl.Kdim + S - 1) / S + kKSegAlign - 1) / kKSegAlign * kKSegAlign;
    const int units = seg * S;  // S > 1 only when seg < kChunkPairs, so then units < kMaxUnits
    if ((threadIdx.x & 31) == 0)  // the warp's first two pairs; each unit then asks for the one two turns on
      for (int u = warp; u < min(units, warp + 2 * kWarps); u += kWarps)
        if (u % S == 0) prefetch_pair<WK, DUAL>(ph, kind, e, pi0 + u / S);
    stage_rows(ph, kind, rc, nr, sm, sizeof(AT) == 4);
    for (int u = warp; u < units; u += kWarps) {
      const int un = u + 2 * kWarps;
      if ((threadIdx.x & 31) == 0 && un < units && un % S == 0) prefetch_pair<WK, DUAL>(ph, kind, e, pi0 + un / S);
      const int i = u / S, sgi = u - i * S;
      const int kb = sgi * kseg, ke = min(pl.Kdim, kb + kseg);
      unit_nt<AT, WK, DUAL, MAXNT>(nr, ph, kind, e, pi0 + i, kb, ke, S == 1 ? nullptr : sm.part + u * kMaxTok * 2,
                                   sm);
    }
    if (S > 1) {
      __syncthreads();
      for (int t = threadIdx.x; t < seg * nr; t += blockDim.x) {  // add the segments in K order
        const int i = t / nr, c = t - i * nr;
        float va = 0.f, vb = 0.f;
        for (int sgi = 0; sgi < S; ++sgi) {
          const float* q = sm.part + ((i * S + sgi) * kMaxTok + c) * 2;
          va += q[0];
          vb += q[1];
        }
        pair_out<DUAL>(ph, kind, pi0 + i, c, va, vb, sm);
      }
    }
    p += seg;
    __syncthreads();  // every warp is done with the staged rows and the partial sums
  }
}

}  // namespace stream
}  // namespace moe
