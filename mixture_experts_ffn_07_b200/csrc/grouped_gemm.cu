// Grouped GEMM on Blackwell tensor cores for the expert projections.
//
// Role of the pages' id-indexed matmuls (hf2q qwen35/gpu_ffn.rs,
// quantized_matmul_id for gate/up and down; DS4Server qwen_mtplx.rs,
// GatherQMM over expert-sorted rows) with the activation product fused into
// the gate/up epilogue (hf2q, fused_gate_up_silu; ferrum-kernels
// vnext_ops/moe.rs, gate_up_silu) and the routing weight fused into the down
// epilogue (ferrum-kernels, routed_down_slots; mlx-native moe_dispatch.rs,
// moe_weighted_sum).
//
// Design (sm_100a):
//  * persistent grid, one CTA per SM; work items (group, n-tile, m-tile) with
//    the m-tile fastest so CTAs running at the same time share weight tiles
//    in L2; in single mode, for memory-bound groups of more than one row tile,
//    an item covers two row tiles against one weight tile (two accumulators),
//    so each weight tile is loaded once per group;
//  * warp 0: TMA producer (one lane) into a shared-memory ring of 128x64 A
//    tiles and BNx64 B tiles, 128-byte swizzle (6 stages at BN = 128, 4 at 256);
//  * warp 1: allocates 2*BN TMEM columns and issues tcgen05.mma (M=128, N=BN,
//    K=16, bf16 in, f32 accumulate) from one lane; two accumulators so the
//    epilogue of one tile overlaps the main loop of the next;
//  * warps 2-5: epilogue, one TMEM lane (= output row) per thread;
//  * dual mode (gate/up): the BN-row B tile is BN/2 rows of W_gate followed
//    by the same BN/2 rows of W_up, so TMEM columns [0,BN/2) hold x W_gate^T and
//    [BN/2,BN) hold x W_up^T for the same outputs; the epilogue writes
//    act(g) * u as bf16;
//  * single mode (down, router): the epilogue scales row r by row_scale and
//    stores it at row row_map[r] (the slot row of the pair), f32 or bf16;
//  * both epilogues pass each row's output through the warp's staging rows in
//    shared memory, 128 bytes per row at a time, and the warp writes them out
//    as whole 128-byte row segments (four rows per store instruction) instead
//    of 16-byte pieces of 32 rows, or one small bulk copy per row segment;
//  * every mbarrier wait is bounded; on expiry the CTA records
//    MOE_ERR_TIMEOUT, lets in-flight copies and MMAs land, frees TMEM and exits.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>

#include "kernels.h"

namespace moe {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int A_BYTES = BM * BK * 2;
constexpr int MAX_G = 256;
constexpr int THREADS = 192;
constexpr int kMaxPairDevices = 64;

// Tile shape per instantiation: the MMA is M=128 x N=BN; an item covers MT
// (1 or 2) row tiles of one group against the same BN weight rows, so a stage
// holds MT A tiles (128x64) and one B tile (BNx64); ~192 KB of stages either way.
template <int BN, int MT>
struct Tile {
  static_assert(MT == 1 || BN == 128, "two row tiles per item need 4*BN <= 512 TMEM columns");
  static constexpr int STAGES = MT == 2 ? 4 : (BN == 128 ? 6 : 4);
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = MT * A_BYTES + B_BYTES;
  static constexpr uint32_t TMEM_COLS = 2 * MT * BN;  // two accumulator sets of MT tiles
};

template <int STAGES>
struct Aux {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t done;
  uint32_t tmem_base;
  int abort;
  int item_off[MAX_G + 1];
  int row_off[MAX_G];
  int cnt[MAX_G];
};

// Epilogue staging: each epilogue warp owns 32 rows x 128 bytes of shared
// memory (a 144-byte pitch keeps both the row writes and the row-segment
// reads free of bank conflicts).
constexpr int kOutPitch = 144;
constexpr int kOutStage = 4 * 32 * kOutPitch;

template <int BN, int MT>
constexpr size_t smem_bytes() {
  return 1024 + static_cast<size_t>(Tile<BN, MT>::STAGES) * Tile<BN, MT>::STAGE_BYTES +
         (sizeof(Aux<Tile<BN, MT>::STAGES>) + 127) / 128 * 128 + kOutStage;
}

struct KParams {
  const int32_t* offsets;
  int G;
  int ksplit;          // K ranges per output tile (plain f32 mode only)
  int kb_per_split;    // k-blocks per range
  size_t part_stride;  // elements between the f32 outputs of consecutive ranges
  int rows_single;
  int N;
  int Kdim;
  int n_tiles;
  int col_step;
  int act;
  __nv_bfloat16* out_bf16;
  float* out_f32;
  const int32_t* row_map;
  const float* row_scale;
  int* status;
  long long wait_limit;
  int skip_stage;
  int head_mult;       // single-CTA kernel: skip each group's first floor(rows / head_mult) * head_mult rows
                       // (the CTA-pair kernel's full 256-row tiles); 0: all rows
  const int32_t* gather_rows;  // A row r = row gather_rows[r] / gather_div of the map's tensor (nullptr: row r)
  int gather_div;
};

// Token rows of A rows [a_row + 4 lane, a_row + 4 lane + 4) for a gathered A operand (rows past the last
// logical row read the last one; the epilogue never writes them).
__device__ __forceinline__ void gather_tokens(const KParams& p, int a_row, int (&tr)[4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < 4; ++j) tr[j] = p.gather_rows[min(a_row + 4 * lane + j, p.rows_single - 1)] / p.gather_div;
}

// Wait ignoring the abort flag (used to drain in-flight work before exit).
__device__ __forceinline__ bool wait_cycles(uint64_t* bar, uint32_t parity, long long limit) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > limit) return false;
  return true;
}

// Item w -> group g, first row tile mt and the number nm (1..MT) of row tiles
// it covers, column tile nt, K range ks.
template <int MT, typename AuxT>
__device__ __forceinline__ void decode_item(const AuxT& aux, int G, int ksplit, int w, int& g, int& mt, int& nm,
                                            int& nt, int& ks) {
  int lo = 0, hi = G - 1;  // largest g with item_off[g] <= w
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (aux.item_off[mid] <= w)
      lo = mid;
    else
      hi = mid - 1;
  }
  g = lo;
  const int tiles = (aux.cnt[g] + BM - 1) / BM;
  const int mitems = (tiles + MT - 1) / MT;
  const int local = w - aux.item_off[g];
  ks = local % ksplit;
  const int rest = local / ksplit;
  nt = rest / mitems;
  mt = (rest - nt * mitems) * MT;
  nm = min(MT, tiles - mt);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}

// Epilogue of one accumulator tile: TMEM lane q*32 + lane (this thread's row)
// holds BN f32 columns from `tbase`.  The output goes out in slabs of 128 bytes
// per row: each thread writes its row's slab into the warp's staging rows, then
// the warp copies the 32 staged rows out with 16-byte stores, 8 lanes per row,
// so each store instruction writes four whole 128-byte row segments wherever
// the rows go (rows are scattered through row_map in the down projection).
//  DUAL: h[dest, col0 + c] = act(g_c) * u_c as bf16, c < BN/2 (g: columns
//        [0, BN/2), u: [BN/2, BN));
//  else: out[dest, col0 + c] = scale * acc_c, bf16 (out_bf16) or f32.
// dest < 0: the row is not written.  Column chunks at or beyond p.N are not
// written (N is a multiple of 32, so a 16-byte chunk is all in or all out).
// All lanes of the warp; the TMEM loads are .sync.aligned.
template <bool DUAL, int BN>
__device__ __forceinline__ void epilogue_tile(const KParams& p, uint32_t tbase, uint8_t* wstage, int dest, float scale,
                                              int col0, int ks) {
  const int lane = threadIdx.x & 31;
  uint8_t* srow = wstage + lane * kOutPitch;
  const uint32_t stage_s = smem_addr(wstage);
  const bool f32_out = !DUAL && p.out_bf16 == nullptr;
  const int ocols = DUAL ? BN / 2 : BN;      // output columns of the tile
  const int slab = f32_out ? 32 : 64;        // output columns per 128-byte slab
  for (int s0 = 0; s0 < ocols; s0 += slab) {
    if (col0 + s0 >= p.N) break;  // warp-uniform
    if (f32_out) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(tbase + s0, v);
      tmem_ld_wait();
      uint4* s4 = reinterpret_cast<uint4*>(srow);
#pragma unroll
      for (int jj = 0; jj < 8; ++jj)
        s4[jj] = make_uint4(__float_as_uint(scale * __uint_as_float(v[4 * jj])),
                            __float_as_uint(scale * __uint_as_float(v[4 * jj + 1])),
                            __float_as_uint(scale * __uint_as_float(v[4 * jj + 2])),
                            __float_as_uint(scale * __uint_as_float(v[4 * jj + 3])));
    } else {
#pragma unroll
      for (int half = 0; half < 2; ++half) {  // 32 output columns = 64 bytes of the slab each
        const int c = s0 + 32 * half;
        uint32_t packed[16];
        if (DUAL) {
          uint32_t gr[32], ur[32];
          tmem_ld_32x32b_x32(tbase + c, gr);
          tmem_ld_32x32b_x32(tbase + BN / 2 + c, ur);
          tmem_ld_wait();
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const float h0 = act_fn(p.act, __uint_as_float(gr[2 * jj])) * __uint_as_float(ur[2 * jj]);
            const float h1 = act_fn(p.act, __uint_as_float(gr[2 * jj + 1])) * __uint_as_float(ur[2 * jj + 1]);
            packed[jj] = pack_bf16x2(h0, h1);
          }
        } else {
          uint32_t v[32];
          tmem_ld_32x32b_x32(tbase + c, v);
          tmem_ld_wait();
#pragma unroll
          for (int jj = 0; jj < 16; ++jj)
            packed[jj] = pack_bf16x2(scale * __uint_as_float(v[2 * jj]), scale * __uint_as_float(v[2 * jj + 1]));
        }
        uint4* s4 = reinterpret_cast<uint4*>(srow + 64 * half);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
          s4[jj] = make_uint4(packed[4 * jj], packed[4 * jj + 1], packed[4 * jj + 2], packed[4 * jj + 3]);
      }
    }
    __syncwarp();
    // copy out: lane -> staged row 4 i + lane / 8, 16-byte chunk lane % 8
    const int ch = lane & 7;
    const int cpe = f32_out ? 4 : 8;  // output columns per 16-byte chunk
    const int col = col0 + s0 + ch * cpe;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int rr = 4 * i + (lane >> 3);
      const int d = __shfl_sync(0xffffffffu, dest, rr);
      const uint4 v = lds128(stage_s + rr * kOutPitch + ch * 16);
      if (d >= 0 && col < p.N) {
        if (f32_out)
          *reinterpret_cast<uint4*>(p.out_f32 + ks * p.part_stride + static_cast<size_t>(d) * p.N + col) = v;
        else
          *reinterpret_cast<uint4*>(p.out_bf16 + static_cast<size_t>(d) * p.N + col) = v;
      }
    }
    __syncwarp();  // the staged rows are read before the next slab overwrites them
  }
}

template <bool DUAL, int BN, int MT>
__global__ void __launch_bounds__(THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB0,
                        const __grid_constant__ CUtensorMap mapB1, const KParams p) {
  constexpr int STAGES = Tile<BN, MT>::STAGES;
  constexpr int STAGE_BYTES = Tile<BN, MT>::STAGE_BYTES;
  constexpr int B_BYTES = Tile<BN, MT>::B_BYTES;
  constexpr uint32_t TMEM_COLS = Tile<BN, MT>::TMEM_COLS;
  constexpr int BN_MMA = BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Aux<STAGES>& aux = *reinterpret_cast<Aux<STAGES>*>(smem + STAGES * STAGE_BYTES);
  uint8_t* out_stage = smem + STAGES * STAGE_BYTES + ((sizeof(Aux<STAGES>) + 127) / 128) * 128;
  volatile int* abort_flag = &aux.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // prologue that reads nothing earlier kernels write: overlaps their tail under programmatic launch
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&aux.full[s], 1);
      mbar_init(&aux.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&aux.tfull[b], 1);
      mbar_init(&aux.tempty[b], 4);
    }
    mbar_init(&aux.done, 1);
    aux.abort = 0;
    fence_mbar_init();
  } else if (threadIdx.x == 32) {
    prefetch_tensormap(&mapA);
    prefetch_tensormap(&mapB0);
    if (DUAL) prefetch_tensormap(&mapB1);
  }
  if (warp == 1) {
    tmem_alloc(&aux.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  pdl_trigger();
  // The tail launch after the CTA-pair kernel (head_mult > 0) reads only what the kernels before the pair
  // kernel wrote, which the pair kernel's CTAs waited for before they let this launch start, and writes rows
  // the pair kernel does not: it starts at once (filling the pair kernel's last wave) and waits for the pair
  // kernel only before it exits, so that the launches after it see both kernels' output.
  if (p.head_mult == 0) pdl_wait();
  for (int g = threadIdx.x; g < p.G; g += THREADS) {
    const int o0 = p.offsets ? p.offsets[g] : 0;
    const int o1 = p.offsets ? p.offsets[g + 1] : p.rows_single;
    // a group's rows stay inside the A tensor (and so inside every output indexed by them), whatever the
    // offsets hold; offsets outside it are reported
    const int r0 = min(max(o0, 0), p.rows_single), r1 = min(max(o1, r0), p.rows_single);
    if (r0 != o0 || r1 != o1) record_status(p.status, MOE_ERR_DEVICE_INDEX);
    const int head = p.head_mult > 0 ? (r1 - r0) / p.head_mult * p.head_mult : 0;
    aux.row_off[g] = r0 + head;
    aux.cnt[g] = r1 - r0 - head;
  }
  __syncthreads();
  if (warp == 0) {  // exclusive scan of work items per group; lane owns groups [8*lane, 8*lane+8)
    int v[8], local = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int g = lane * 8 + i;
      v[i] = g < p.G ? ((aux.cnt[g] + MT * BM - 1) / (MT * BM)) * p.n_tiles * p.ksplit : 0;
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
      const int g = lane * 8 + i;
      if (g < p.G) aux.item_off[g] = run;
      run += v[i];
    }
    if (lane == 31) aux.item_off[p.G] = incl;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem_base = aux.tmem_base;
  const int total = aux.item_off[p.G];
  const int nkb = (p.Kdim + BK - 1) / BK;
  const long long limit = p.wait_limit;

  if (warp == 0) {
    if (MT == 1 && p.gather_rows != nullptr) {
      // ------------------------------------------------------------ TMA producer, gathered A rows (whole warp)
      // Lane l gathers rows [4 l, 4 l + 4) of each 128-row A tile straight from the token rows
      // (tile::gather4, one row per coordinate, into the 128-byte-swizzled tile as a box load would);
      // lane 0 waits for the stage, expects its bytes and loads the weight tile.
      uint32_t kbg = 0, outstanding = 0, out_phase = 0;
      bool skipped = false;
      const uint64_t pol_w = l2_policy_evict_first();
      const uint64_t pol_a = l2_policy_evict_last();
      for (int w = blockIdx.x; w < total; w += gridDim.x) {
        if (__shfl_sync(0xffffffffu, *abort_flag, 0)) break;
        int g, mt, nm, nt, ks;
        decode_item<MT>(aux, p.G, p.ksplit, w, g, mt, nm, nt, ks);
        const int a_row = aux.row_off[g] + mt * BM;
        int tr[4];
        gather_tokens(p, a_row, tr);
        const bool one_mtile = aux.cnt[g] <= BM;
        const int b_row = g * p.N + nt * p.col_step;
        const int kb0 = ks * p.kb_per_split, kb1 = min(nkb, kb0 + p.kb_per_split);
        for (int kb = kb0; kb < kb1; ++kb, ++kbg) {
          const int s = kbg % STAGES;
          const uint32_t ph = (kbg / STAGES) & 1u;
          int ok = 1;
          if (lane == 0) ok = mbar_wait_bounded(&aux.empty[s], ph ^ 1u, limit, abort_flag);
          if (!__shfl_sync(0xffffffffu, ok, 0)) break;
          outstanding &= ~(1u << s);
          if (p.skip_stage && !skipped && blockIdx.x == 0) {  // debug: leave this stage unfilled
            skipped = true;
            continue;
          }
          uint8_t* sa = smem + s * STAGE_BYTES;
          uint8_t* sb = sa + A_BYTES;
          if (lane == 0) mbar_arrive_expect_tx(&aux.full[s], A_BYTES + B_BYTES);
          __syncwarp();
          tma_gather4(sa + lane * 4 * 128, &mapA, &aux.full[s], kb * BK, tr[0], tr[1], tr[2], tr[3], pol_a);
          if (lane == 0) {
            if (one_mtile) {
              tma_load_2d_hint(sb, &mapB0, &aux.full[s], kb * BK, b_row, pol_w);
              if (DUAL) tma_load_2d_hint(sb + B_BYTES / 2, &mapB1, &aux.full[s], kb * BK, b_row, pol_w);
            } else {
              tma_load_2d(sb, &mapB0, &aux.full[s], kb * BK, b_row);
              if (DUAL) tma_load_2d(sb + B_BYTES / 2, &mapB1, &aux.full[s], kb * BK, b_row);
            }
          }
          outstanding |= 1u << s;
          out_phase = (out_phase & ~(1u << s)) | (ph << s);
        }
      }
      if (lane == 0 && *abort_flag) {  // let issued copies land before the CTA exits
        for (int s = 0; s < STAGES; ++s)
          if (outstanding & (1u << s)) wait_cycles(&aux.full[s], (out_phase >> s) & 1u, limit);
      }
    } else if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      uint32_t kbg = 0, outstanding = 0, out_phase = 0;
      bool skipped = false;
      const uint64_t pol_w = l2_policy_evict_first();  // weights of a group with one row tile: read once
      const uint64_t pol_a = l2_policy_evict_last();   // activation rows: read by every column tile
      for (int w = blockIdx.x; w < total && !*abort_flag; w += gridDim.x) {
        int g, mt, nm, nt, ks;
        decode_item<MT>(aux, p.G, p.ksplit, w, g, mt, nm, nt, ks);
        const int a_row = aux.row_off[g] + mt * BM;
        const bool one_mtile = aux.cnt[g] <= MT * BM;  // this item covers every row tile of the group
        const int b_row = g * p.N + nt * p.col_step;
        const int kb0 = ks * p.kb_per_split, kb1 = min(nkb, kb0 + p.kb_per_split);
        for (int kb = kb0; kb < kb1; ++kb, ++kbg) {
          const int s = kbg % STAGES;
          const uint32_t ph = (kbg / STAGES) & 1u;
          if (!mbar_wait_bounded(&aux.empty[s], ph ^ 1u, limit, abort_flag)) break;
          outstanding &= ~(1u << s);
          if (p.skip_stage && !skipped && blockIdx.x == 0) {  // debug: leave this stage unfilled
            skipped = true;
            continue;
          }
          uint8_t* sa = smem + s * STAGE_BYTES;
          uint8_t* sb = sa + MT * A_BYTES;
          mbar_arrive_expect_tx(&aux.full[s], nm * A_BYTES + B_BYTES);
          for (int j = 0; j < nm; ++j)
            tma_load_2d_hint(sa + j * A_BYTES, &mapA, &aux.full[s], kb * BK, a_row + j * BM, pol_a);
          if (one_mtile) {  // the weight tile is not needed again
            tma_load_2d_hint(sb, &mapB0, &aux.full[s], kb * BK, b_row, pol_w);
            if (DUAL) tma_load_2d_hint(sb + B_BYTES / 2, &mapB1, &aux.full[s], kb * BK, b_row, pol_w);
          } else {  // the group's other row tiles read it again: default L2 policy
            tma_load_2d(sb, &mapB0, &aux.full[s], kb * BK, b_row);
            if (DUAL) tma_load_2d(sb + B_BYTES / 2, &mapB1, &aux.full[s], kb * BK, b_row);
          }
          outstanding |= 1u << s;
          out_phase = (out_phase & ~(1u << s)) | (ph << s);
        }
      }
      if (*abort_flag) {  // let issued copies land before the CTA exits
        for (int s = 0; s < STAGES; ++s)
          if (outstanding & (1u << s)) wait_cycles(&aux.full[s], (out_phase >> s) & 1u, limit);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      const uint32_t idesc = idesc_bf16_f32(BM, BN_MMA);
      uint32_t kbg = 0;
      int it = 0;
      for (int w = blockIdx.x; w < total; w += gridDim.x, ++it) {
        int g, mt, nm, nt, ks;
        decode_item<MT>(aux, p.G, p.ksplit, w, g, mt, nm, nt, ks);
        const int kb0 = ks * p.kb_per_split, kb1 = min(nkb, kb0 + p.kb_per_split);
        const int acc = it & 1;
        const uint32_t acc_ph = (it >> 1) & 1u;
        if (!mbar_wait_bounded(&aux.tempty[acc], acc_ph ^ 1u, limit, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * MT * BN_MMA;  // row tile j accumulates at + j * BN
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb, ++kbg) {
          const int s = kbg % STAGES;
          const uint32_t ph = (kbg / STAGES) & 1u;
          if (!mbar_wait_bounded(&aux.full[s], ph, limit, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_addr(smem + s * STAGE_BYTES);
          const uint64_t bdesc = sw128_kmajor_desc(a_addr + MT * A_BYTES);
          for (int j = 0; j < nm; ++j) {
            const uint64_t adesc = sw128_kmajor_desc(a_addr + j * A_BYTES);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              umma_bf16(d_tmem + j * BN_MMA, adesc + static_cast<uint64_t>(kk * 2),
                        bdesc + static_cast<uint64_t>(kk * 2), idesc, (kb > kb0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&aux.empty[s]);
        }
        if (!ok) break;
        umma_commit(&aux.tfull[acc]);
      }
      umma_commit(&aux.done);  // every MMA issued above completes before TMEM is released
      wait_cycles(&aux.done, 0, limit);
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lanes [32q, 32q+32) are reachable from this warp
    const int r = q * 32 + lane;
    int it = 0;
    for (int w = blockIdx.x; w < total; w += gridDim.x, ++it) {
      int g, mt0, nm, nt, ks;
      decode_item<MT>(aux, p.G, p.ksplit, w, g, mt0, nm, nt, ks);
      const int acc = it & 1;
      const uint32_t acc_ph = (it >> 1) & 1u;
      // every lane waits; the outcome is made warp-uniform because the TMEM loads below are .sync.aligned
      const bool ok = mbar_wait_bounded(&aux.tfull[acc], acc_ph, limit, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      for (int j = 0; j < nm; ++j) {
      const int mt = mt0 + j;
      const int rows_valid = min(BM, aux.cnt[g] - mt * BM);
      const int a_row = aux.row_off[g] + mt * BM;
      const int col0 = nt * p.col_step;
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + (acc * MT + j) * BN_MMA;
      int dest = -1;
      float scale = 1.f;
      if (r < rows_valid) {
        const int src = a_row + r;
        if (DUAL) {
          dest = src;
        } else {
          dest = p.row_map ? p.row_map[src] : src;
          if (dest < 0 || dest >= p.rows_single) {  // output rows number the A rows: a bad map entry is skipped
            record_status(p.status, MOE_ERR_DEVICE_INDEX);
            dest = -1;
          } else {
            scale = p.row_scale ? p.row_scale[dest] : 1.f;
          }
        }
      }
      epilogue_tile<DUAL, BN_MMA>(p, tbase, out_stage + q * 32 * kOutPitch, dest, scale, col0, ks);
      }  // row tiles of the item
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&aux.tempty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
  if (threadIdx.x == 0 && aux.abort) record_status(p.status, MOE_ERR_TIMEOUT);
  if (p.head_mult > 0) pdl_wait();  // complete only after the pair kernel (see above)
}

// ------------------------------------------------------------------ CTA-pair kernel
// For compute-bound launches: the full 256-row tiles of each group run on
// pairs of CTAs (clusters of two) that share one tcgen05.mma.cta_group::2 of
// M = 256, N = 256.  CTA r of a pair loads rows [128 r, 128 r + 128) of the
// tile's A rows and 128 rows of B: in dual mode CTA 0 the W_gate rows and CTA 1
// the same W_up rows (TMEM columns [0,128) are then gate, [128,256) up); in
// single mode rows [128 r, 128 r + 128) of the 256 output columns.  Per MMA
// flop each CTA stages half the B bytes of the single-CTA 128 x 256 tile.  Both
// CTAs' loads complete on CTA 0's stage barrier (CTA 0 expects both CTAs'
// bytes); CTA 0's MMA thread issues the MMAs and its commits arrive on the
// stage-empty and accumulator-full barriers of both CTAs; each CTA's epilogue
// drains its own 128 TMEM lanes (epilogue_tile) and arrives on CTA 0's
// accumulator-empty barrier.  No load is multicast.  The rows of a group past
// its last full 256-row tile are left to the single-CTA kernel (head_mult).
constexpr int PAIR_M = 256;
constexpr int PAIR_STAGES = 6;
constexpr int PAIR_B_BYTES = 128 * BK * 2;
constexpr int PAIR_STAGE_BYTES = A_BYTES + PAIR_B_BYTES;
constexpr uint32_t PAIR_TMEM_COLS = 512;  // two accumulators of 256 columns

constexpr size_t pair_smem_bytes() {
  return 1024 + static_cast<size_t>(PAIR_STAGES) * PAIR_STAGE_BYTES + (sizeof(Aux<PAIR_STAGES>) + 127) / 128 * 128 +
         kOutStage;
}

// Item w of the pair kernel -> group g, 256-row tile mt, column tile nt.
template <typename AuxT>
__device__ __forceinline__ void decode_pair_item(const AuxT& aux, int G, int w, int& g, int& mt, int& nt) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (aux.item_off[mid] <= w)
      lo = mid;
    else
      hi = mid - 1;
  }
  g = lo;
  const int tiles = aux.cnt[g] / PAIR_M;
  const int local = w - aux.item_off[g];
  nt = local / tiles;
  mt = local - nt * tiles;
}

template <bool DUAL>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB0,
                             const __grid_constant__ CUtensorMap mapB1, const KParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Aux<PAIR_STAGES>& aux = *reinterpret_cast<Aux<PAIR_STAGES>*>(smem + PAIR_STAGES * PAIR_STAGE_BYTES);
  uint8_t* out_stage = smem + PAIR_STAGES * PAIR_STAGE_BYTES + ((sizeof(Aux<PAIR_STAGES>) + 127) / 128) * 128;
  volatile int* abort_flag = &aux.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: the CTA that issues the MMAs
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < PAIR_STAGES; ++s) {
      mbar_init(&aux.full[s], 1);
      mbar_init(&aux.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&aux.tfull[b], 1);
      mbar_init(&aux.tempty[b], 8);  // the four epilogue warps of both CTAs
    }
    mbar_init(&aux.done, 1);
    aux.abort = 0;
    fence_mbar_init();
  } else if (threadIdx.x == 32) {
    prefetch_tensormap(&mapA);
    prefetch_tensormap(&mapB0);
    if (DUAL) prefetch_tensormap(&mapB1);
  }
  if (warp == 1) {
    tmem_alloc_pair(&aux.tmem_base, PAIR_TMEM_COLS);
    tmem_relinquish_pair();
  }
  pdl_wait();
  pdl_trigger();  // after the wait: the tail launch relies on this grid having waited for its predecessors
  for (int g = threadIdx.x; g < p.G; g += THREADS) {
    const int o0 = p.offsets ? p.offsets[g] : 0;
    const int o1 = p.offsets ? p.offsets[g + 1] : p.rows_single;
    const int r0 = min(max(o0, 0), p.rows_single), r1 = min(max(o1, r0), p.rows_single);
    if (r0 != o0 || r1 != o1) record_status(p.status, MOE_ERR_DEVICE_INDEX);
    aux.row_off[g] = r0;
    aux.cnt[g] = (r1 - r0) / PAIR_M * PAIR_M;
  }
  __syncthreads();
  if (warp == 0) {  // exclusive scan of work items per group; lane owns groups [8*lane, 8*lane+8)
    int v[8], local = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int g = lane * 8 + i;
      v[i] = g < p.G ? (aux.cnt[g] / PAIR_M) * p.n_tiles : 0;
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
      const int g = lane * 8 + i;
      if (g < p.G) aux.item_off[g] = run;
      run += v[i];
    }
    if (lane == 31) aux.item_off[p.G] = incl;
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers and TMEM are ready before any load, MMA or remote arrive
  tc_fence_after();

  const uint32_t tmem_base = aux.tmem_base;
  const int total = aux.item_off[p.G];
  const int nkb = (p.Kdim + BK - 1) / BK;
  const long long limit = p.wait_limit;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs; with gathered A
    // rows the whole warp: lane l gathers rows [4 l, 4 l + 4) of the CTA's 128 A rows, as in the single-CTA
    // kernel, and lane 0 does the rest)
    const bool gather = p.gather_rows != nullptr;
    if (gather || lane == 0) {
      uint32_t kbg = 0, outstanding = 0, out_phase = 0;
      const uint64_t pol_a = l2_policy_evict_last();    // activation rows: read by every column tile
      const uint64_t pol_b = l2_policy_evict_normal();  // weight tiles: read by each row tile of the group
      const CUtensorMap* mb = (DUAL && rank == 1) ? &mapB1 : &mapB0;
      const unsigned mask = gather ? 0xffffffffu : 1u;
      for (int w = pair; w < total; w += npairs) {
        if (__shfl_sync(mask, *abort_flag, 0)) break;
        int g, mt, nt;
        decode_pair_item(aux, p.G, w, g, mt, nt);
        const int a_row = aux.row_off[g] + mt * PAIR_M + static_cast<int>(rank) * BM;
        const int b_row = g * p.N + nt * p.col_step + (DUAL ? 0 : static_cast<int>(rank) * 128);
        int tr[4] = {0, 0, 0, 0};
        if (gather) gather_tokens(p, a_row, tr);
        for (int kb = 0; kb < nkb; ++kb, ++kbg) {
          const int s = kbg % PAIR_STAGES;
          const uint32_t ph = (kbg / PAIR_STAGES) & 1u;
          int ok = 1;
          if (lane == 0) ok = mbar_wait_bounded(&aux.empty[s], ph ^ 1u, limit, abort_flag);
          if (!__shfl_sync(mask, ok, 0)) break;
          outstanding &= ~(1u << s);
          uint8_t* sa = smem + s * PAIR_STAGE_BYTES;
          const uint32_t full_s = cluster_addr(&aux.full[s], 0);
          if (lane == 0 && rank == 0) mbar_arrive_expect_tx(&aux.full[s], 2 * PAIR_STAGE_BYTES);
          if (gather) {
            __syncwarp();
            tma_gather4_pair(sa + lane * 4 * 128, &mapA, full_s, kb * BK, tr[0], tr[1], tr[2], tr[3], pol_a);
          } else {
            tma_load_2d_pair(sa, &mapA, full_s, kb * BK, a_row, pol_a);
          }
          if (lane == 0) tma_load_2d_pair(sa + A_BYTES, mb, full_s, kb * BK, b_row, pol_b);
          outstanding |= 1u << s;
          out_phase = (out_phase & ~(1u << s)) | (ph << s);
        }
      }
      if (lane == 0 && *abort_flag && rank == 0) {  // let issued copies land before the pair exits
        for (int s = 0; s < PAIR_STAGES; ++s)
          if (outstanding & (1u << s)) wait_cycles(&aux.full[s], (out_phase >> s) & 1u, limit);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------------------ MMA issuer (CTA 0 of the pair)
      const uint32_t idesc = idesc_bf16_f32(PAIR_M, 256);
      uint32_t kbg = 0;
      int it = 0;
      for (int w = pair; w < total; w += npairs, ++it) {
        const int acc = it & 1;
        const uint32_t acc_ph = (it >> 1) & 1u;
        if (!mbar_wait_bounded(&aux.tempty[acc], acc_ph ^ 1u, limit, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * 256;
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb, ++kbg) {
          const int s = kbg % PAIR_STAGES;
          const uint32_t ph = (kbg / PAIR_STAGES) & 1u;
          if (!mbar_wait_bounded(&aux.full[s], ph, limit, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_addr(smem + s * PAIR_STAGE_BYTES);
          const uint64_t adesc = sw128_kmajor_desc(a_addr);
          const uint64_t bdesc = sw128_kmajor_desc(a_addr + A_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            umma_bf16_pair(d_tmem, adesc + static_cast<uint64_t>(kk * 2), bdesc + static_cast<uint64_t>(kk * 2), idesc,
                           (kb > 0 || kk > 0) ? 1u : 0u);
          umma_commit_pair(&aux.empty[s], 0x3);
        }
        if (!ok) break;
        umma_commit_pair(&aux.tfull[acc], 0x3);
      }
      umma_commit_pair(&aux.done, 0x3);  // every MMA issued above completes before TMEM is released
      wait_cycles(&aux.done, 0, limit);
    }
  } else {
    // -------------------------------------------------------------- epilogue (both CTAs)
    const int q = warp & 3;
    const int r = q * 32 + lane;
    int it = 0;
    for (int w = pair; w < total; w += npairs, ++it) {
      int g, mt, nt;
      decode_pair_item(aux, p.G, w, g, mt, nt);
      const int acc = it & 1;
      const uint32_t acc_ph = (it >> 1) & 1u;
      const bool ok = mbar_wait_bounded(&aux.tfull[acc], acc_ph, limit, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const int src = aux.row_off[g] + mt * PAIR_M + static_cast<int>(rank) * BM + r;  // full tiles: every row valid
      int dest = src;
      float scale = 1.f;
      if (!DUAL) {
        dest = p.row_map ? p.row_map[src] : src;
        if (dest < 0 || dest >= p.rows_single) {
          record_status(p.status, MOE_ERR_DEVICE_INDEX);
          dest = -1;
        } else {
          scale = p.row_scale ? p.row_scale[dest] : 1.f;
        }
      }
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * 256;
      epilogue_tile<DUAL, 256>(p, tbase, out_stage + q * 32 * kOutPitch, dest, scale, nt * p.col_step, 0);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(cluster_addr(&aux.tempty[acc], 0));
    }
  }

  tc_fence_before();
  __syncwarp();
  cluster_sync_all();  // both CTAs are done with each other's barriers, shared memory and TMEM
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, PAIR_TMEM_COLS);
  }
  if (threadIdx.x == 0 && aux.abort) record_status(p.status, MOE_ERR_TIMEOUT);
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}

// Row-major bf16 matrix [rows, cols] read in boxes of box_rows x 64 columns, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(BK), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

KParams make_params(const Ctx& c, const GemmArgs& a, int col_step, int head_mult) {
  KParams p;
  p.offsets = a.offsets;
  p.G = a.G;
  const int nkb = (a.Kdim + BK - 1) / BK;
  p.ksplit = effective_ksplit(a.ksplit, a.Kdim);
  p.kb_per_split = (nkb + p.ksplit - 1) / p.ksplit;
  p.part_stride = a.part_stride;
  p.rows_single = static_cast<int>(a.rows_A);
  p.N = a.N;
  p.Kdim = a.Kdim;
  p.col_step = col_step;
  p.n_tiles = (a.N + p.col_step - 1) / p.col_step;
  p.act = a.act;
  p.out_bf16 = a.out_bf16;
  p.out_f32 = a.out_f32;
  p.row_map = a.row_map;
  p.row_scale = a.row_scale;
  p.status = c.status;
  p.wait_limit = c.wait_limit;
  p.skip_stage = c.skip_stage;
  p.head_mult = head_mult;
  p.gather_rows = a.gather_rows;
  p.gather_div = a.gather_div > 0 ? a.gather_div : 1;
  return p;
}

// The A map: the operand's rows in 128-row boxes, or, for a gathered operand, the source rows one at a time
// (tile::gather4 boxes are one row high).
bool make_a_map(CUtensorMap* m, const GemmArgs& a) {
  if (a.gather_rows)
    return make_map(m, a.A_src, static_cast<uint64_t>(a.rows_src), static_cast<uint64_t>(a.Kdim), 1);
  return make_map(m, a.A, static_cast<uint64_t>(a.rows_A), static_cast<uint64_t>(a.Kdim), BM);
}

template <bool DUAL, int BN, int MT>
cudaError_t launch_tiled(const Ctx& c, const GemmArgs& a, int head_mult = 0) {
  CUtensorMap mA, mB0, mB1;
  const uint32_t brows = DUAL ? BN / 2 : BN;
  if (!make_a_map(&mA, a) ||
      !make_map(&mB0, a.B0, static_cast<uint64_t>(a.G) * a.N, static_cast<uint64_t>(a.Kdim), brows))
    return cudaErrorInvalidValue;
  if (DUAL) {
    if (!make_map(&mB1, a.B1, static_cast<uint64_t>(a.G) * a.N, static_cast<uint64_t>(a.Kdim), brows))
      return cudaErrorInvalidValue;
  } else {
    mB1 = mB0;
  }
  const KParams p = make_params(c, a, DUAL ? BN / 2 : BN, head_mult);
  // rows left after the pair kernel's full tiles: fewer than head_mult per group
  const long long rows = head_mult > 0 ? std::min<long long>(a.max_rows, static_cast<long long>(a.G) * (head_mult - 1))
                                       : a.max_rows;
  const long long tiles_bound = rows / BM + std::min<long long>(a.G, rows);
  const long long items_bound = tiles_bound * p.n_tiles * p.ksplit;
  const int grid = static_cast<int>(std::max(1LL, std::min<long long>(c.num_sms, items_bound)));
  auto kern = grouped_gemm_kernel<DUAL, BN, MT>;
  const cudaError_t e =
      allow_dynamic_smem(reinterpret_cast<const void*>(kern), static_cast<int>(smem_bytes<BN, MT>()));
  if (e != cudaSuccess) return e;
  KernelScope ks(c, a.name ? a.name : (DUAL ? "grouped_gemm_dual" : "grouped_gemm"));
  return launch_kernel(c, kern, dim3(grid), dim3(THREADS), smem_bytes<BN, MT>(), mA, mB0, mB1, p);
}

// Clusters of two that fit on the device at once (0 if none), once per device and kernel.
template <bool DUAL>
int pair_clusters(const Ctx& c) {
  static std::atomic<int> cached[kMaxPairDevices];
  static std::atomic<bool> init[kMaxPairDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxPairDevices) return 0;
  if (init[dev].load()) return cached[dev].load();
  auto kern = grouped_gemm_pair_kernel<DUAL>;
  int n = 0;
  if (allow_dynamic_smem(reinterpret_cast<const void*>(kern), static_cast<int>(pair_smem_bytes())) == cudaSuccess) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2 * (c.num_sms / 2));
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = pair_smem_bytes();
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();
  cached[dev].store(n);
  init[dev].store(true);
  return n;
}

// The trace name of a CTA-pair launch's tail launch ("<name>_tail").
inline const char* tail_name(const char* name) {
  if (!std::strcmp(name, "expert_gate_up_gemm")) return "expert_gate_up_gemm_tail";
  if (!std::strcmp(name, "expert_down_gemm")) return "expert_down_gemm_tail";
  if (!std::strcmp(name, "shared_gate_up_gemm")) return "shared_gate_up_gemm_tail";
  if (!std::strcmp(name, "shared_down_gemm")) return "shared_down_gemm_tail";
  return "grouped_gemm_tail";
}

// The full 256-row tiles of every group on CTA pairs (M = 256, N = 256 per
// MMA), then the rows left in each group on the single-CTA kernel.
template <bool DUAL>
cudaError_t launch_pair(const Ctx& c, const GemmArgs& a, int clusters) {
  CUtensorMap mA, mB0, mB1;
  if (!make_a_map(&mA, a) ||
      !make_map(&mB0, a.B0, static_cast<uint64_t>(a.G) * a.N, static_cast<uint64_t>(a.Kdim), 128))
    return cudaErrorInvalidValue;
  if (DUAL) {
    if (!make_map(&mB1, a.B1, static_cast<uint64_t>(a.G) * a.N, static_cast<uint64_t>(a.Kdim), 128))
      return cudaErrorInvalidValue;
  } else {
    mB1 = mB0;
  }
  const KParams p = make_params(c, a, DUAL ? 128 : 256, 0);
  const long long items_bound = static_cast<long long>(a.max_rows / PAIR_M) * p.n_tiles;
  const int pairs = static_cast<int>(std::max(1LL, std::min<long long>(clusters, items_bound)));
  auto kern = grouped_gemm_pair_kernel<DUAL>;
  {
    KernelScope ks(c, a.name ? a.name : (DUAL ? "grouped_gemm_dual" : "grouped_gemm"));
    const cudaError_t e = launch_kernel(c, kern, dim3(2 * pairs), dim3(THREADS), pair_smem_bytes(), mA, mB0, mB1, p);
    if (e != cudaSuccess) return e;
  }
  GemmArgs tail = a;
  if (a.name) tail.name = tail_name(a.name);
  return launch_tiled<DUAL, 256, 1>(c, tail, PAIR_M);
}

}  // namespace

// Tail of the last wave when `items` equal work items run on `sms` persistent CTAs.
double wave_waste(double items, int sms) {
  const double waves = items / sms;
  const double full = std::ceil(waves);
  return full > 0 ? (full - waves) / full : 0.0;
}

// Narrow tiles (N = 128) for weight-streaming (memory-bound) shapes whose last
// wave would leave many SMs idle with wide tiles; wide tiles (N = 256) for
// compute-bound shapes, where they halve the A-tile traffic per flop.
cudaError_t launch_grouped_gemm(const Ctx& c, const GemmArgs& a) {
  if (a.G <= 0 || a.max_rows <= 0 || a.N <= 0 || a.rows_A <= 0) return cudaSuccess;
  if (a.G > MAX_G || a.N % 32) return cudaErrorInvalidValue;  // the epilogue writes whole 16-byte column chunks
  if (a.gather_rows && (!a.dual || a.ksplit > 1 || !a.A_src)) return cudaErrorInvalidValue;
  const int groups = std::min(a.G, a.max_rows);
  const double rows_per_group = static_cast<double>(a.max_rows) / groups;
  // about half an M tile of padding per group
  const double tiles = static_cast<double>(a.max_rows) / BM + 0.5 * groups;
  const double cols_wide = a.dual ? 128.0 : 256.0;
  const double items_wide = tiles * std::ceil(a.N / cols_wide);
  const double items_narrow = tiles * std::ceil(a.N / (cols_wide / 2));
  // weights are streamed once per group; rows per group sets flops per weight byte (ridge ~200)
  const bool memory_bound = rows_per_group < 200.0;
  // single mode (the down projection: short K) with memory-bound groups that often span two row tiles: narrow
  // tiles covering two row tiles per item, so each item is twice as long and each weight tile is loaded once per
  // group.  The gate/up projection keeps one row tile per item: its long K rows already share weight tiles
  // through L2 between the CTAs running a group's row tiles side by side, and it keeps 6 stages.
  if (!a.dual && memory_bound && rows_per_group > 96.0) return launch_tiled<false, 128, 2>(c, a);
  // at most 128 output columns (the router: N = E): a 256-column tile would be three quarters zero fill
  if (!a.dual && a.N <= 128) return launch_tiled<false, 128, 1>(c, a);
  // compute-bound launches with at least one full 256-row tile: CTA pairs for the full tiles
  if (!memory_bound && a.ksplit <= 1 && a.max_rows >= PAIR_M && pair_gemm_enabled()) {
    const int clusters = a.dual ? pair_clusters<true>(c) : pair_clusters<false>(c);
    if (clusters > 0) return a.dual ? launch_pair<true>(c, a, clusters) : launch_pair<false>(c, a, clusters);
  }
  // narrow tiles waste less of the last wave, but every column tile re-reads the activation rows: with more than
  // 96 rows per group (activations well beyond L2 on such launches) the dual launch keeps wide tiles
  const bool narrow = memory_bound && !(a.dual && rows_per_group > 96.0) &&
                      wave_waste(items_wide, c.num_sms) - wave_waste(items_narrow, c.num_sms) > 0.03;
  if (a.dual) return narrow ? launch_tiled<true, 128, 1>(c, a) : launch_tiled<true, 256, 1>(c, a);
  return narrow ? launch_tiled<false, 128, 1>(c, a) : launch_tiled<false, 256, 1>(c, a);
}

}  // namespace moe
