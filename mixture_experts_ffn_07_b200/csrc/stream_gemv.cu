// Weight-streaming expert FFN for small batches (T <= 64) and for f32 / Q8_0
// weights: the bandwidth-bound decode path.
//
// Decode reads every touched expert's weights once and does little arithmetic
// per byte (hf2q qwen35/gpu_ffn.rs: mat-vec beats tiled mat-mat at one row;
// DS4Server qwen_mtplx.rs, fused_experts: moe_glu_h then moe_down_y).  Here the
// copy engine does all the moving.  A persistent CTA per SM walks a contiguous
// range of work items (touched expert, block of R output rows) split into token
// batches.  One producer warp copies, with cp.async.bulk:
//   * each item's weight rows (contiguous: rows are out x in) into a ring of
//     weight stages, Q8_0 scale rows alongside;
//   * each expert's token rows (x for gate/up, h for down) into a two-slot ring,
//     with the rows' output index and routing weight.
// Eight consumer warps never wait for one another: row pairs (gate row i with
// up row i; or two down rows) are dealt round-robin over the whole walk, each
// warp dots its pairs with the staged token rows, writes its outputs and
// arrives on the stage's release barrier.  Lanes take 4 consecutive weights at
// a time, so the token rows are read 16 bytes per lane at consecutive
// addresses (no bank conflicts).  Q8_0 weights are widened in registers: exact
// int8 -> f32 through the exponent-bias trick, the fp16 block scale applied to
// each 4-value partial sum.
//
//  gate/up (DUAL): h[r, i] = act(W_gate[e,i] . a_r) * (W_up[e,i] . a_r)
//  down          : y[dest_r, j] = scale_r * (W_down[e,j] . a_r)
#include "kernels.h"

namespace moe {

namespace {

enum { WK_F32 = 0, WK_BF16 = 1, WK_Q8 = 2 };

constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 1) * 32;  // + one producer warp
constexpr int kMaxStages = 4;
constexpr int kMaxTok = 8;  // token rows per batch
constexpr int kMaxPairsPerWarp = 2;
constexpr int kMaxTokenRowBytes = 64 * 1024;  // one staged token row
constexpr int kSmemBudget = 216 * 1024;
constexpr uint32_t kPiece = 32768;  // largest single bulk copy issued

struct Plan {
  int PPW;          // row pairs per consumer warp per item
  int NP;           // row pairs per item (kConsumerWarps * PPW)
  int RPM;          // rows per matrix per item (NP for gate/up, 2 NP for down)
  int KR;           // reduction elements per item (a multiple of 32)
  int nkr;          // items per row block (K ranges)
  int TS;           // token rows per batch (and per token slot)
  int Kdim;         // reduction length (H for gate/up, I for down)
  int Nout;         // output rows per expert (I for gate/up, H for down)
  int row_bytes;    // bytes of one full weight row (quants only for Q8_0)
  int srow_bytes;   // bytes of one full row of Q8_0 scales (0 otherwise)
  int seg_bytes;    // bytes of one row segment of KR weights
  int sseg_bytes;   // bytes of one row segment of KR/32 scales
  int tile_bytes;   // bytes of one weight stage
  int stages;       // weight stages (2..4)
  int xrow_bytes;   // bytes of one staged token row
  int xslot_bytes;  // bytes of one token slot
};

struct Args {
  const void* act;         // token rows: x [T, H] (gate/up) or h [rows, I] f32 (down)
  const uint8_t* w0;       // gate or down [*, Nout, Kdim] in the weight format
  const uint8_t* w1;       // up (gate/up only)
  const uint8_t* s0;       // Q8_0 scales of w0 / w1
  const uint8_t* s1;
  const int32_t* offsets;  // [E+1] rows per expert (nullptr: one group of T rows)
  int E, T, K;
  const int32_t* pairs;    // sorted pair ids (nullptr: identity)
  int act_fn;
  float* out;              // h [rows, I] (gate/up) or y [*, H] (down)
  const float* row_scale;  // down: per pair (or per token) weight
  int* status;
  long long wait_limit;
};

// ---- four weights at a time ----
template <int WK>
struct Quad;
template <>
struct Quad<WK_F32> {
  using raw = float4;
};
template <>
struct Quad<WK_BF16> {
  using raw = uint2;
};
template <>
struct Quad<WK_Q8> {
  using raw = uint32_t;
};

template <int WK>
__device__ __forceinline__ void quad_f32(const typename Quad<WK>::raw r, float (&v)[4]) {
  if constexpr (WK == WK_F32) {
    v[0] = r.x;
    v[1] = r.y;
    v[2] = r.z;
    v[3] = r.w;
  } else if constexpr (WK == WK_BF16) {
    v[0] = bf16_bits_to_f32(r.x & 0xFFFFu);
    v[1] = bf16_bits_to_f32(r.x >> 16);
    v[2] = bf16_bits_to_f32(r.y & 0xFFFFu);
    v[3] = bf16_bits_to_f32(r.y >> 16);
  } else {
    // Exact int8 -> f32 without conversion instructions: with the sign bit
    // flipped, byte b is u = b + 128; the word 0x4B0000uu is the float 2^23 + u,
    // so subtracting 2^23 + 128 leaves b.
    const uint32_t u = r ^ 0x80808080u;
    v[0] = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7650)) - 8388736.0f;
    v[1] = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7651)) - 8388736.0f;
    v[2] = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7652)) - 8388736.0f;
    v[3] = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7653)) - 8388736.0f;
  }
}

template <typename XT>
__device__ __forceinline__ void x_quad(const XT* row, int q, float (&v)[4]) {
  if constexpr (sizeof(XT) == 4) {
    const float4 a = reinterpret_cast<const float4*>(row)[q];
    v[0] = a.x;
    v[1] = a.y;
    v[2] = a.z;
    v[3] = a.w;
  } else {
    const uint2 a = reinterpret_cast<const uint2*>(row)[q];
    v[0] = bf16_bits_to_f32(a.x & 0xFFFFu);
    v[1] = bf16_bits_to_f32(a.x >> 16);
    v[2] = bf16_bits_to_f32(a.y & 0xFFFFu);
    v[3] = bf16_bits_to_f32(a.y >> 16);
  }
}

// Adds the quad q of rows A and B dotted with the NT token rows to acc_a / acc_b.
template <int NT, int WK, typename XT>
__device__ __forceinline__ void quad_step(const typename Quad<WK>::raw* ra, const typename Quad<WK>::raw* rb,
                                          const __half* sa, const __half* sb, const XT* xs, int Kdim, int q,
                                          float (&acc_a)[NT], float (&acc_b)[NT]) {
  float va[4], vb[4];
  quad_f32<WK>(ra[q], va);
  quad_f32<WK>(rb[q], vb);
  float sca = 1.f, scb = 1.f;
  if constexpr (WK == WK_Q8) {  // 8 quads per 32-value block
    sca = __half2float(sa[q >> 3]);
    scb = __half2float(sb[q >> 3]);
  }
#pragma unroll
  for (int c = 0; c < NT; ++c) {
    float xv[4];
    x_quad<XT>(xs + c * Kdim, q, xv);
    const float pa = fmaf(va[0], xv[0], va[1] * xv[1]) + fmaf(va[2], xv[2], va[3] * xv[3]);
    const float pb = fmaf(vb[0], xv[0], vb[1] * xv[1]) + fmaf(vb[2], xv[2], vb[3] * xv[3]);
    acc_a[c] = fmaf(sca, pa, acc_a[c]);
    acc_b[c] = fmaf(scb, pb, acc_b[c]);
  }
}

// Adds to per-lane partial sums the dot products of row segments A and B (nq
// quads in shared memory) with NT token rows (shared memory, row stride xstride
// elements, starting at quad q0 of the rows).  Lane l takes quads l, l+32, ...,
// two per iteration into separate sums.
template <int NT, int WK, typename XT>
__device__ __forceinline__ void dot_pair_acc(const uint8_t* wa, const __half* sa, const uint8_t* wb,
                                             const __half* sb, const XT* xs, int xstride, int q0, int nq,
                                             float (&a0)[NT], float (&b0)[NT], float (&a1)[NT], float (&b1)[NT]) {
  using R = typename Quad<WK>::raw;
  const int lane = threadIdx.x & 31;
  const R* ra = reinterpret_cast<const R*>(wa);
  const R* rb = reinterpret_cast<const R*>(wb);
  const XT* x0 = xs + 4 * q0;
  int q = lane;
  for (; q + 32 < nq; q += 64) {
    quad_step<NT, WK, XT>(ra, rb, sa, sb, x0, xstride, q, a0, b0);
    quad_step<NT, WK, XT>(ra, rb, sa, sb, x0, xstride, q + 32, a1, b1);
  }
  if (q < nq) quad_step<NT, WK, XT>(ra, rb, sa, sb, x0, xstride, q, a0, b0);
}

__device__ __forceinline__ void bulk_copy(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(smem_dst)),
      "l"(gsrc), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void bulk_copy_split(uint8_t* dst, const uint8_t* src, uint32_t bytes, uint64_t* bar) {
  for (uint32_t off = 0; off < bytes; off += kPiece) bulk_copy(dst + off, src + off, min(kPiece, bytes - off), bar);
}

// One step of the walk over (work item, token batch) that producer and consumers share.
struct Walk {
  int e, b;         // expert, token batch
  int j0, nrow;     // first output row, rows (per matrix) in the block
  int rc, nr;       // first token row of the batch, rows in the batch
};

// One unit for one consumer warp: its PPW row pairs of the block, over the nkr
// K-range items (waiting for and releasing each stage), partial sums kept in
// registers across the ranges, then reduced and written.
template <int NT, typename AT, int WK, bool DUAL>
__device__ __forceinline__ bool consume_unit(const Args& a, const Plan& pl, const Walk& w, const uint8_t* tiles,
                                             const uint8_t* xslots, int slot, int& it, uint64_t* full,
                                             uint64_t* empty, volatile int* abort_flag,
                                             const int (*s_dest)[kMaxTok], const float (*s_scale)[kMaxTok]) {
  constexpr int NMAT = DUAL ? 2 : 1;
  constexpr int PPW_MAX = kMaxPairsPerWarp;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const AT* xs = reinterpret_cast<const AT*>(xslots + slot * pl.xslot_bytes);
  const int npairs = DUAL ? w.nrow : (w.nrow + 1) / 2;
  float a0[PPW_MAX][NT], b0[PPW_MAX][NT], a1[PPW_MAX][NT], b1[PPW_MAX][NT];
#pragma unroll
  for (int p = 0; p < PPW_MAX; ++p)
#pragma unroll
    for (int c = 0; c < NT; ++c) a0[p][c] = b0[p][c] = a1[p][c] = b1[p][c] = 0.f;
  for (int kr = 0; kr < pl.nkr; ++kr, ++it) {
    const int s = it % pl.stages;
    const bool ok = mbar_wait_bounded(&full[s], (it / pl.stages) & 1u, a.wait_limit, abort_flag);
    if (!__all_sync(0xffffffffu, ok)) return false;
    const uint8_t* t = tiles + s * pl.tile_bytes;
    const __half* sbase = reinterpret_cast<const __half*>(t + NMAT * pl.RPM * pl.seg_bytes);
    const int kre = min(pl.KR, pl.Kdim - kr * pl.KR);
#pragma unroll
    for (int p = 0; p < PPW_MAX; ++p) {
      const int pr = warp * pl.PPW + p;
      if (p < pl.PPW && pr < npairs) {
        const int ra_row = DUAL ? pr : 2 * pr;
        const int rb_row = DUAL ? pr : min(2 * pr + 1, w.nrow - 1);
        const int mb = DUAL ? 1 : 0;
        const uint8_t* wa = t + ra_row * pl.seg_bytes;
        const uint8_t* wb = t + (mb * pl.RPM + rb_row) * pl.seg_bytes;
        const __half* sa = WK == WK_Q8 ? sbase + ra_row * (pl.sseg_bytes / 2) : nullptr;
        const __half* sb = WK == WK_Q8 ? sbase + (mb * pl.RPM + rb_row) * (pl.sseg_bytes / 2) : nullptr;
        dot_pair_acc<NT, WK, AT>(wa, sa, wb, sb, xs, pl.Kdim, (kr * pl.KR) >> 2, kre >> 2, a0[p], b0[p], a1[p],
                                 b1[p]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
#pragma unroll
  for (int p = 0; p < PPW_MAX; ++p) {
    const int pr = warp * pl.PPW + p;
    if (p < pl.PPW && pr < npairs) {
      float va = 0.f, vb = 0.f;
#pragma unroll
      for (int c = 0; c < NT; ++c) {
        const float sa_ = warp_sum(a0[p][c] + a1[p][c]);
        const float sb_ = warp_sum(b0[p][c] + b1[p][c]);
        if (lane == c) {
          va = sa_;
          vb = sb_;
        }
      }
      if (lane < NT) {
        if (DUAL) {
          a.out[static_cast<size_t>(s_dest[slot][lane]) * pl.Nout + w.j0 + pr] = act_fn(a.act_fn, va) * vb;
        } else {
          float* yrow = a.out + static_cast<size_t>(s_dest[slot][lane]) * pl.Nout + w.j0;
          yrow[2 * pr] = s_scale[slot][lane] * va;
          if (2 * pr + 1 < w.nrow) yrow[2 * pr + 1] = s_scale[slot][lane] * vb;
        }
      }
    }
  }
  return true;
}

template <typename AT, int WK, bool DUAL>
__global__ void __launch_bounds__(kThreads, 1) stream_gemv_kernel(const Args a, const Plan pl) {
  constexpr int NMAT = DUAL ? 2 : 1;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t full[kMaxStages], empty[kMaxStages], xfull[2], xempty[2];
  __shared__ int s_active[256], s_first[256], s_count[256], s_uoff[257];
  __shared__ int s_warp[8];
  __shared__ int s_n;
  __shared__ int s_dest[2][kMaxTok];
  __shared__ float s_scale[2][kMaxTok];
  __shared__ int s_abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* tiles = smem;
  uint8_t* xslots = smem + pl.stages * pl.tile_bytes;

  if (threadIdx.x == 0) {
    for (int s = 0; s < pl.stages; ++s) {
      mbar_init(&full[s], 2);  // byte-counted arrival + producer warp's arrival
      mbar_init(&empty[s], kConsumerWarps);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&xfull[s], 2);
      mbar_init(&xempty[s], kConsumerWarps);
    }
    s_abort = 0;
    fence_mbar_init();
  }
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
      s_active[i] = e;
      s_first[i] = a.offsets ? a.offsets[e] : 0;
      s_count[i] = a.offsets ? a.offsets[e + 1] - a.offsets[e] : a.T;
    }
    if (threadIdx.x == 0) s_n = n;
  }
  __syncthreads();
  volatile int* abort_flag = &s_abort;
  // Work units: (touched expert, token batch, block of NP row pairs); each unit
  // is nkr items (K ranges) in a row.  CTAs take contiguous ranges of units.
  const int rblocks = (pl.Nout + pl.RPM - 1) / pl.RPM;
  if (threadIdx.x == 0) {
    int run = 0;
    for (int i = 0; i < s_n; ++i) {
      s_uoff[i] = run;
      run += ((s_count[i] + pl.TS - 1) / pl.TS) * rblocks;
    }
    s_uoff[s_n] = run;
  }
  __syncthreads();
  const int total = s_uoff[s_n];
  const int u0 = static_cast<int>(static_cast<long long>(blockIdx.x) * total / gridDim.x);
  const int u1 = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * total / gridDim.x);
  auto locate = [&](int u, Walk& w) {
    int lo = 0, hi = s_n - 1;  // last active expert whose units start at or before u
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_uoff[mid] <= u)
        lo = mid;
      else
        hi = mid - 1;
    }
    const int local = u - s_uoff[lo];
    const int b = local / rblocks;
    w.e = s_active[lo];
    w.b = b;
    w.j0 = (local - b * rblocks) * pl.RPM;
    w.nrow = min(pl.RPM, pl.Nout - w.j0);
    w.rc = s_first[lo] + b * pl.TS;
    w.nr = min(pl.TS, s_first[lo] + s_count[lo] - w.rc);
  };

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer warp
    int it = 0, xit = -1, key_e = -1, key_b = -1;
    uint32_t issued = 0, issued_ph = 0, xissued = 0, xissued_ph = 0;
    bool stop = false;
    for (int u = u0; u < u1 && !stop; ++u) {
      Walk w;
      locate(u, w);
      if (w.e != key_e || w.b != key_b) {  // next token batch: fill the next token slot
        ++xit;
        const int xs = xit & 1;
        const uint32_t xph = (xit >> 1) & 1u;
        bool ok = true;
        if (lane == 0) ok = mbar_wait_bounded(&xempty[xs], xph ^ 1u, a.wait_limit, abort_flag);
        if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) break;
        xissued &= ~(1u << xs);
        int arow = 0;
        if (lane < w.nr) {
          const int r = w.rc + lane;
          const int dest = a.pairs ? a.pairs[r] : r;
          arow = DUAL ? (a.pairs ? dest / a.K : r) : r;
          s_dest[xs][lane] = DUAL ? r : dest;  // gate/up writes h row r; down writes y row dest
          s_scale[xs][lane] = (!DUAL && a.row_scale) ? a.row_scale[dest] : 1.f;
        }
        if (lane == 0) mbar_arrive_expect_tx(&xfull[xs], static_cast<uint32_t>(w.nr) * pl.xrow_bytes);
        __syncwarp();
        if (lane < w.nr)
          bulk_copy_split(xslots + xs * pl.xslot_bytes + lane * pl.xrow_bytes,
                          static_cast<const uint8_t*>(a.act) + static_cast<size_t>(arow) * pl.xrow_bytes,
                          pl.xrow_bytes, &xfull[xs]);
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&xfull[xs]);
          xissued |= 1u << xs;
          xissued_ph = (xissued_ph & ~(1u << xs)) | (xph << xs);
        }
        key_e = w.e;
        key_b = w.b;
      }
      const size_t row0 = static_cast<size_t>(w.e) * pl.Nout + w.j0;
      for (int kr = 0; kr < pl.nkr; ++kr, ++it) {
        const int s = it % pl.stages;
        const uint32_t ph = (it / pl.stages) & 1u;
        bool ok = true;
        if (lane == 0) ok = mbar_wait_bounded(&empty[s], ph ^ 1u, a.wait_limit, abort_flag);
        if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) {
          stop = true;
          break;
        }
        issued &= ~(1u << s);
        uint8_t* t = tiles + s * pl.tile_bytes;
        uint8_t* ts = t + NMAT * pl.RPM * pl.seg_bytes;
        const int k0e = kr * pl.KR;                          // first element of the range
        const int kre = min(pl.KR, pl.Kdim - k0e);           // elements in the range
        const uint32_t segb = static_cast<uint32_t>(kre) * (pl.row_bytes / pl.Kdim);
        const bool whole = pl.nkr == 1;                      // rows contiguous in memory and in the tile
        const bool bulk_scales = WK == WK_Q8 && whole && (pl.srow_bytes % 16) == 0;
        const uint32_t qbytes = static_cast<uint32_t>(w.nrow) * (whole ? pl.row_bytes : segb);
        const uint32_t sbytes = static_cast<uint32_t>(w.nrow) * pl.srow_bytes;
        if (lane == 0) mbar_arrive_expect_tx(&full[s], NMAT * (qbytes + (bulk_scales ? sbytes : 0u)));
        __syncwarp();
        for (int m = 0; m < NMAT; ++m) {
          const uint8_t* wsrc = (m ? a.w1 : a.w0) + row0 * pl.row_bytes;
          uint8_t* wdst = t + m * pl.RPM * pl.seg_bytes;
          if (whole) {
            if (lane == 0) bulk_copy_split(wdst, wsrc, qbytes, &full[s]);
          } else {
            for (int r = lane; r < w.nrow; r += 32)
              bulk_copy(wdst + r * pl.seg_bytes, wsrc + static_cast<size_t>(r) * pl.row_bytes + k0e * (pl.row_bytes / pl.Kdim),
                        segb, &full[s]);
          }
        }
        if (WK == WK_Q8) {
          if (bulk_scales) {
            if (lane == 0)
              for (int m = 0; m < NMAT; ++m)
                bulk_copy_split(ts + m * pl.RPM * pl.sseg_bytes, (m ? a.s1 : a.s0) + row0 * pl.srow_bytes, sbytes,
                                &full[s]);
          } else {  // 2-byte granules: the warp copies them, 8 loads in flight per lane
            const int hpr = kre / 32;  // scales per row in this range
            const int nh = w.nrow * hpr;
            for (int m = 0; m < NMAT; ++m) {
              const uint16_t* g = reinterpret_cast<const uint16_t*>(m ? a.s1 : a.s0) + row0 * (pl.srow_bytes / 2) + k0e / 32;
              uint16_t* d = reinterpret_cast<uint16_t*>(ts + m * pl.RPM * pl.sseg_bytes);
              for (int i0 = lane; i0 < nh; i0 += 256) {
                uint16_t v[8];
#pragma unroll
                for (int uu = 0; uu < 8; ++uu) {
                  const int i = i0 + 32 * uu;
                  if (i < nh) v[uu] = __ldg(g + (i / hpr) * (pl.srow_bytes / 2) + (i % hpr));
                }
#pragma unroll
                for (int uu = 0; uu < 8; ++uu) {
                  const int i = i0 + 32 * uu;
                  if (i < nh) d[(i / hpr) * (pl.sseg_bytes / 2) + (i % hpr)] = v[uu];
                }
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&full[s]);
          issued |= 1u << s;
          issued_ph = (issued_ph & ~(1u << s)) | (ph << s);
        }
      }
    }
    if (lane == 0 && *abort_flag) {  // let issued copies land before the CTA exits
      const long long t0 = clock64();
      for (int s = 0; s < pl.stages; ++s)
        if (issued & (1u << s))
          while (!mbar_try_wait(&full[s], (issued_ph >> s) & 1u) && clock64() - t0 < a.wait_limit) {
          }
      for (int s = 0; s < 2; ++s)
        if (xissued & (1u << s))
          while (!mbar_try_wait(&xfull[s], (xissued_ph >> s) & 1u) && clock64() - t0 < a.wait_limit) {
          }
    }
  } else {
    // ------------------------------------------------------------ consumer warps
    int it = 0, xit = -1, key_e = -1, key_b = -1;
    bool stop = false;
    for (int u = u0; u < u1 && !stop; ++u) {
      Walk w;
      locate(u, w);
      if (w.e != key_e || w.b != key_b) {
        if (xit >= 0 && lane == 0) mbar_arrive(&xempty[xit & 1]);  // done with the previous token rows
        ++xit;
        const bool ok = mbar_wait_bounded(&xfull[xit & 1], (xit >> 1) & 1u, a.wait_limit, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) break;
        key_e = w.e;
        key_b = w.b;
      }
      bool ok = true;
      switch (w.nr) {  // straight-line code for the token count
        case 1: ok = consume_unit<1, AT, WK, DUAL>(a, pl, w, tiles, xslots, xit & 1, it, full, empty, abort_flag, s_dest, s_scale); break;
        case 2: ok = consume_unit<2, AT, WK, DUAL>(a, pl, w, tiles, xslots, xit & 1, it, full, empty, abort_flag, s_dest, s_scale); break;
        case 3: ok = consume_unit<3, AT, WK, DUAL>(a, pl, w, tiles, xslots, xit & 1, it, full, empty, abort_flag, s_dest, s_scale); break;
        case 4: ok = consume_unit<4, AT, WK, DUAL>(a, pl, w, tiles, xslots, xit & 1, it, full, empty, abort_flag, s_dest, s_scale); break;
        case 5: ok = consume_unit<5, AT, WK, DUAL>(a, pl, w, tiles, xslots, xit & 1, it, full, empty, abort_flag, s_dest, s_scale); break;
        case 6: ok = consume_unit<6, AT, WK, DUAL>(a, pl, w, tiles, xslots, xit & 1, it, full, empty, abort_flag, s_dest, s_scale); break;
        case 7: ok = consume_unit<7, AT, WK, DUAL>(a, pl, w, tiles, xslots, xit & 1, it, full, empty, abort_flag, s_dest, s_scale); break;
        default: ok = consume_unit<8, AT, WK, DUAL>(a, pl, w, tiles, xslots, xit & 1, it, full, empty, abort_flag, s_dest, s_scale); break;
      }
      if (!ok) stop = true;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && s_abort) record_status(a.status, MOE_ERR_TIMEOUT);
}

// Shapes of the items.  Every consumer warp owns PPW row pairs of each item;
// a row block is split into K ranges when its full rows would not fit ~48 KB
// stages (f32 rows of a few thousand elements), otherwise PPW grows while an
// item stays within ~48 KB.  Token slots take at most a third of the budget
// unless a single token row needs more (up to kMaxTokenRowBytes).
Plan make_plan(int wk, bool dual, int Kdim, int Nout, int act_bytes_per_elem, int max_tokens) {
  Plan p{};
  p.Kdim = Kdim;
  p.Nout = Nout;
  const int eb = wk == WK_F32 ? 4 : (wk == WK_BF16 ? 2 : 1);
  p.row_bytes = Kdim * eb;
  p.srow_bytes = wk == WK_Q8 ? (Kdim / 32) * 2 : 0;
  p.xrow_bytes = Kdim * act_bytes_per_elem;
  const int nmat = dual ? 2 : 1;
  p.TS = std::max(1, std::min(kMaxTok, max_tokens));
  while (p.TS > 1 && 2 * p.TS * p.xrow_bytes > kSmemBudget / 3) --p.TS;
  p.xslot_bytes = (p.TS * p.xrow_bytes + 127) / 128 * 128;
  const int left = kSmemBudget - 2 * p.xslot_bytes;
  const int target = std::min(48 * 1024, left / 2);  // at least two stages
  const int rows_per_pair = 2;  // gate+up, or two down rows
  const int full_pair = rows_per_pair * (p.row_bytes + p.srow_bytes);
  p.PPW = 1;
  if (kConsumerWarps * full_pair <= target) {  // whole rows; grow pairs per warp
    p.KR = Kdim;
    while (p.PPW < kMaxPairsPerWarp && kConsumerWarps * (p.PPW + 1) * full_pair <= target) ++p.PPW;
  } else {  // split rows into nearly equal K ranges, multiples of 32 elements
    const long long per_elem = static_cast<long long>(rows_per_pair) * kConsumerWarps * eb;
    const int nkr = static_cast<int>((Kdim * per_elem + target - 1) / target);
    p.KR = std::min(Kdim, ((Kdim + nkr - 1) / nkr + 31) / 32 * 32);
  }
  p.nkr = (Kdim + p.KR - 1) / p.KR;
  p.NP = kConsumerWarps * p.PPW;
  p.RPM = dual ? p.NP : 2 * p.NP;
  p.seg_bytes = p.KR * eb;
  p.sseg_bytes = wk == WK_Q8 ? (p.KR / 32) * 2 : 0;
  p.tile_bytes = ((nmat * p.RPM * (p.seg_bytes + p.sseg_bytes)) + 127) / 128 * 128;
  p.stages = std::max(2, std::min(kMaxStages, left / p.tile_bytes));
  return p;
}

template <typename AT, int WK, bool DUAL>
cudaError_t launch_typed(const Ctx& c, const Args& a, const Plan& p, const char* name) {
  auto kern = stream_gemv_kernel<AT, WK, DUAL>;
  if (p.xrow_bytes > kMaxTokenRowBytes) return cudaErrorInvalidValue;
  const int smem = p.stages * p.tile_bytes + 2 * p.xslot_bytes;
  const cudaError_t e = allow_dynamic_smem(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  KernelScope ks(c, name);
  return launch_kernel(c, kern, dim3(c.num_sms), dim3(kThreads), smem, a, p);
}

}  // namespace

cudaError_t launch_stream_gate_up(const Ctx& c, const void* x, int x_dtype, int T, int H, int I, int K,
                                  const void* gate, const void* up, const void* gate_scale, const void* up_scale,
                                  int w_dtype, const int32_t* offsets, int E, const int32_t* pairs, int rows_bound,
                                  int act, float* h) {
  if (rows_bound <= 0) return cudaSuccess;
  Args a{};
  a.act = x;
  a.w0 = static_cast<const uint8_t*>(gate);
  a.w1 = static_cast<const uint8_t*>(up);
  a.s0 = static_cast<const uint8_t*>(gate_scale);
  a.s1 = static_cast<const uint8_t*>(up_scale);
  a.offsets = offsets;
  a.E = offsets ? E : 1;
  a.T = offsets ? 0 : rows_bound;
  a.K = K;
  a.pairs = pairs;
  a.act_fn = act;
  a.out = h;
  a.status = c.status;
  a.wait_limit = c.wait_limit;
  const int wk = w_dtype == MOE_F32 ? WK_F32 : (w_dtype == MOE_BF16 ? WK_BF16 : WK_Q8);
  // an expert owns at most one row per token: at most P / K rows
  const int max_tok = offsets ? std::max(1, rows_bound / std::max(1, K)) : rows_bound;
  const Plan p = make_plan(wk, true, H, I, x_dtype == MOE_F32 ? 4 : 2, max_tok);
  const char* n = "stream_gate_up";
  if (x_dtype == MOE_F32) {
    if (wk == WK_F32) return launch_typed<float, WK_F32, true>(c, a, p, n);
    if (wk == WK_BF16) return launch_typed<float, WK_BF16, true>(c, a, p, n);
    return launch_typed<float, WK_Q8, true>(c, a, p, n);
  }
  if (wk == WK_F32) return launch_typed<__nv_bfloat16, WK_F32, true>(c, a, p, n);
  if (wk == WK_BF16) return launch_typed<__nv_bfloat16, WK_BF16, true>(c, a, p, n);
  return launch_typed<__nv_bfloat16, WK_Q8, true>(c, a, p, n);
}

cudaError_t launch_stream_down(const Ctx& c, const float* h, int I, int H, const void* down, const void* down_scale,
                               int w_dtype, const int32_t* offsets, int E, const int32_t* pairs, int rows_bound,
                               const float* row_scale, float* y) {
  if (rows_bound <= 0) return cudaSuccess;
  Args a{};
  a.act = h;
  a.w0 = static_cast<const uint8_t*>(down);
  a.s0 = static_cast<const uint8_t*>(down_scale);
  a.offsets = offsets;
  a.E = offsets ? E : 1;
  a.T = offsets ? 0 : rows_bound;
  a.K = 1;
  a.pairs = pairs;
  a.out = y;
  a.row_scale = row_scale;
  a.status = c.status;
  a.wait_limit = c.wait_limit;
  const int wk = w_dtype == MOE_F32 ? WK_F32 : (w_dtype == MOE_BF16 ? WK_BF16 : WK_Q8);
  const Plan p = make_plan(wk, false, I, H, 4, kMaxTok);
  const char* n = "stream_down";
  if (wk == WK_F32) return launch_typed<float, WK_F32, false>(c, a, p, n);
  if (wk == WK_BF16) return launch_typed<float, WK_BF16, false>(c, a, p, n);
  return launch_typed<float, WK_Q8, false>(c, a, p, n);
}

}  // namespace moe
