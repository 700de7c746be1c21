// decode_tc.cu -- grouped-query paged decode attention on the 5th-generation
// tensor cores (tcgen05, accumulators in tensor memory), for 16-bit K/V with
// head size 128, G = Hq / Hkv in {4, 8} query heads per KV head, and KV
// heads in groups of HG = 4. (G = 16 would need 640 tensor-memory columns for
// the double-buffered accumulators below; it runs on the CUDA-core kernel.)
//
// Why tensor cores here: the G query heads that share a KV head turn the
// per-token work into a small dense contraction. On the CUDA cores that is ~4
// FMAs per byte of K/V at G = 8, close to the FP32 pipe's limit at HBM speed;
// on tcgen05 it is a few MMAs per tile.
//
// Tile = 128 rows of K (or V): HG heads x Rt = 128 / HG tokens, taken from
// whole physical blocks. A 5-D TMA tensor map views the pool as
// [num_blocks][2 d-halves][Hkv][block_size][64 d] (strides of the real
// [num_blocks, block_size, Hkv, D] layout), so one TMA box brings Rb token
// rows of all HG heads for one 64-wide d-half: 8-16 KB per instruction, in the
// canonical 128-byte-swizzled layout the MMA reads (rows = (head, token),
// 128 B each; the two d-halves 16 KB apart). Bigger boxes matter: streaming
// the same bytes as 2-4 KB per-head boxes is limited by TMA issue, not HBM.
//
// Work split: the tiles of all (sequence b, group h of HG KV heads) pairs,
// in (b, h, tile) order, form one list of T tiles, and the CTAs take equal
// shares of its cost: a tile costs kCostTile, and each pair adds
// DecodeArgs::pair_cost for the work of starting and finishing a unit (the
// query load, the first tile's reduction, the epilogue), so a CTA whose share
// crosses many short pairs streams fewer tiles. Tile x of the p-th pair with
// tiles sits at cost position kCostTile * x + pair_cost * (p + 1), and CTA c
// takes the tiles whose positions lie in [floor(c C / grid),
// floor((c + 1) C / grid)), C the total cost: every CTA does about the same
// work whatever the mix of context lengths, so no CTA finishes a long
// sequence alone at the end. A CTA's share is a run of units:
// whole pairs in the middle, and at each end possibly a piece of a pair that
// continues in the neighbouring CTA. A whole pair is written to the output
// directly. A piece is written as (reference max, exp-sum, unnormalised
// output) into its CTA's piece slot, then takes a ticket on its pair; the
// piece that finishes last reads every piece of the pair back (from L2) and
// merges them: M = max m_p, L = sum l_p 2^(m_p - M), o = sum 2^(m_p - M) o_p / L.
// No CTA waits for another, and no separate merge launch is needed.
//
// Per tile (swap-AB, rows of the tile on the MMA's M = 128):
//   scores  S^T[128 x HG*G]   = K_tile . Q_grp^T         (all query heads of the group)
//   output  O^T_h[128 d x 2G] += V_h^T . [P_hi; P_lo]_h^T  one MMA per head and 16 tokens
// Each row (head h, token) keeps only its own head's G scores. The softmax
// weights enter the output product as two 16-bit parts, p = hi + lo with
// hi = RN(p), lo = RN(p - hi), so the products keep ~16 significant bits
// instead of 8 (bf16); O accumulates in fp32 in TMEM for the whole unit.
// The online softmax rescales O lazily: a query head's reference max moves
// only when a tile's max exceeds it by more than 2^64 (weights up to 2^64 are
// far from fp32 overflow in l and O, and relative precision does not depend
// on scale), which after the first tile is rare; then the affected TMEM
// columns are read, scaled and written back. Exact in real arithmetic: O and
// l always share the same reference.
//
// CTA = 10 warps, persistent over its share:
//   warps 0-7  two softmax groups; group w takes tiles t with t % 2 == w, so
//              every SM sub-partition runs two independent softmax warps; at
//              the end of a unit the group that did not take its last tile
//              hands its reference maxima and exp-sums to the other (mbarrier
//              hand-off), which merges both TMEM accumulators into a shared-
//              memory staging buffer and sends the unit's rows (contiguous in
//              the output and in the workspace) out with bulk asynchronous
//              copies; the accumulators are double-buffered by unit parity,
//              so the next unit's products do not wait for this merge;
//   warp 8     TMA producer (one lane): Q of the unit, K and V tiles through a
//              ring of 32 KB stages;
//   warp 9     MMA issuer (one lane): S(t), then O(t-1).
// Every pipeline wait is bounded (DecodeArgs::wait_ns, 1 s unless a test
// shortens it; the timeout-path test also withholds one query load, so that a
// wait can only run out); a wait that gives up sets the PA_DEV_TIMEOUT bit, raises
// a CTA-wide abort flag, and all roles leave their loops (the softmax warps
// of a group only together, at a named-barrier vote), wait for their own
// asynchronous work (those waits keep the full 1 s bound, so no copy or MMA is
// left in flight), free tensor memory and return.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math_constants.h>

#include <cfloat>

#include "pa_internal.h"
#include "tc_ptx.cuh"

namespace pa {

namespace {

using namespace tc;

constexpr int kD = 128;
constexpr int kRows = 128;                      // rows per tile (the MMA's M)
constexpr int kHalf = kRows * 128;              // bytes of one 64-wide d-half of a tile
constexpr int kStageBytes = 2 * kHalf;          // one K or V tile: 32 KB
constexpr int kHG = 4;                          // KV heads per unit
constexpr int kRt = kRows / kHG;                // tokens per head per tile (32)
constexpr int kThreads = 320;
constexpr int kScanChunk = 1024;                // sequences per pass of the first prologue scan
constexpr float kRescaleLog2 = 64.f;            // lazy rescale threshold (log2 units): p <= 2^64,
                                                // far from fp32 overflow in l and O
constexpr int kEpochShift = 24;                 // ticket word: epoch << 24 | pieces arrived
constexpr unsigned long long kCountMask = (1ull << kEpochShift) - 1;

// 16-bit pools: a ring of 32 KB stages, each the K or V operand of one tile.
// FP8 pools (KV8): a ring of 16 KB stages of codes (K or V of one tile, one
// 128-byte line per row) and, per softmax group, a 32 KB buffer that holds the
// V operand of the group's current tile widened to f16; the query buffer holds
// the 16-bit query as loaded, then its E4M3 pieces.
template <int G, bool KV8 = false> struct TcShape {
  static constexpr int NS = kHG * G;                         // N of the score MMA
  static constexpr int NOH = ((2 * G + 15) / 16) * 16;       // N of a head's output MMA
  static constexpr int NO = kHG * NOH;                       // output columns per group
  static constexpr int kStages = 5;
  static constexpr int kStage = KV8 ? kHalf : kStageBytes;   // bytes per ring stage
  static constexpr int kTmemCols = 512;                      // S x2, O x (2 units x 2 groups)
  static constexpr int kNP = 3;                              // E4M3 pieces of the query at most
  static constexpr int kQBytes = (KV8 ? kNP : 2) * NS * 128; // Q operand: 2 d-halves x NS rows
  static constexpr int kPBytes = 2 * NOH * 128;              // P operand of one tile: 2 lines
  static constexpr int kStgBytes = NS * kD * 4;              // one group's merged rows (fp32)
  static constexpr int OFF_VOP = kStages * kStage;           // [2 groups] widened V (FP8 pools)
  static constexpr int OFF_Q = OFF_VOP + (KV8 ? 2 * kStageBytes : 0);
  static constexpr int OFF_P = OFF_Q + 2 * kQBytes;
  static constexpr int OFF_STG = OFF_P + 2 * kPBytes;        // [2 groups] output staging
  static constexpr int OFF_X = OFF_STG + 2 * kStgBytes;      // [2][2][NS] reference max, exp-sum
  static constexpr int OFF_BAR = OFF_X + 2 * 2 * NS * 4 + 16;
  static constexpr int NBAR = 2 * kStages + 23;
  static constexpr int GP = G < 8 ? 8 : G;                  // per-chunk stride of the reductions
  static constexpr int OFF_RED = (OFF_BAR + 8 * NBAR + 15) / 16 * 16;  // [group][2][8][GP] maxima
  static constexpr int OFF_REDL = OFF_RED + 2 * 2 * 8 * GP * 4;   // [group][2][8][GP] sums
  static constexpr int OFF_MREF = OFF_REDL + 2 * 2 * 8 * GP * 4;  // [group][3][NS] references
  static constexpr int OFF_COEF = OFF_MREF + 2 * 3 * NS * 4;   // [group][2][NS] merge weights
  static constexpr int OFF_QSC = OFF_COEF + 2 * 2 * NS * 4;      // [2 query buffers][NS] score scales
  static constexpr int OFF_MISC = (OFF_QSC + 2 * NS * 4 + 15) / 16 * 16;
  static constexpr int BYTES = OFF_MISC + 64;
  static constexpr int SMEM = BYTES + 1024;                  // + alignment slack
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
  // an S buffer: NS columns, or one block of NS per query piece (FP8 pools)
  static constexpr int SW = (KV8 ? kNP : 1) * NS;
  static_assert(2 * SW + 4 * NO <= kTmemCols, "tensor memory columns");
  static_assert(OFF_STG % 128 == 0, "bulk-copy source alignment");
  static_assert(OFF_COEF % 16 == 0, "vector loads of the merge weights");
  static_assert(OFF_Q % 1024 == 0 && kQBytes % 1024 == 0 && (NS * 128) % 1024 == 0,
                "128-byte-swizzled operands start on 1024-byte boundaries");
};

// barrier indices (the ring's full/empty pairs come first)
template <int NST> struct Bars {
  static constexpr int FULL = 0, EMPTY = NST, QFULL = 2 * NST, QEMPTY = QFULL + 2,
                       SFULL = QEMPTY + 2, SFREE = SFULL + 2, PREADY = SFREE + 2,
                       OFULL = PREADY + 2, XFULL = OFULL + 2, XFREE = XFULL + 2,
                       ODONE = XFREE + 2, DONE = ODONE + 2, QCONV = DONE + 1,
                       QSREAD = QCONV + 2;
};

// Shared words written by the prologue (OFF_MISC).
struct Misc {
  uint32_t tmem;        // tensor-memory base address
  uint32_t abort_flag;
  int32_t valid;        // this CTA's share holds tiles
  int32_t b0, h0, k0;   // first unit: sequence, KV-head group, first tile in the pair
  int32_t found;        // prologue scan: bit 0 the share's start located, bit 1 its end
  int32_t last[2];      // per softmax group: this piece was the last of its pair
  int32_t p0;           // first unit's pair: its index among the pairs with tiles
  long long r0, r1;     // the share: global tiles [r0, r1)
  long long C;          // cost of all pairs
};
static_assert(sizeof(Misc) <= 64, "misc words");

// ---------------------------------------------------------------- the work list
constexpr long long kCostTile = 16;             // cost of one tile (pair_cost is in these units)

// First cost position of CTA c's share: floor(c * C / grid), without 64-bit overflow.
__device__ __forceinline__ long long share_begin(long long c, long long C, long long grid) {
  return (C / grid) * c + ((C % grid) * c) / grid;
}
// The CTA whose share holds cost position x (the largest c with share_begin(c) <= x).
__device__ __forceinline__ int share_owner(long long x, long long C, long long grid) {
  return (int)(((x + 1) * grid - 1) / C);
}
// Cost position of global tile x of the p-th pair with tiles.
__device__ __forceinline__ long long tile_cost(long long x, long long p, long long pair_cost) {
  return kCostTile * x + pair_cost * (p + 1);
}

// The shares that hold tiles of one pair (tiles [pair0, pair0 + ntp), the p-th
// pair with tiles): CTAs c0 .. c1, the owners of its first and last tile, and
// each one's piece slot. A CTA between them whose share falls between two of
// the pair's tiles holds no piece. c0's share starts before the pair when it
// also holds the previous pair's last tile (global tile pair0 - 1, p - 1).
struct PairShares {
  long long pos0;       // cost position of the pair's first tile
  long long pair0;
  int ntp, c0, c1;
  bool c0_before;       // the pair is c0's last unit (slot 2 c0 + 1), else its first
};
__device__ __forceinline__ PairShares pair_shares(long long pair0, int ntp, long long p,
                                                  long long C, int grid, long long pair_cost) {
  PairShares r;
  r.pos0 = tile_cost(pair0, p, pair_cost);
  r.pair0 = pair0;
  r.ntp = ntp;
  r.c0 = share_owner(r.pos0, C, grid);
  r.c1 = share_owner(r.pos0 + kCostTile * (ntp - 1), C, grid);
  r.c0_before = p > 0 && share_begin(r.c0, C, grid) <= tile_cost(pair0 - 1, p - 1, pair_cost);
  return r;
}
// First tile of share c (c0 < c <= c1 + 1) inside the pair; the pair's end for c1 + 1.
__device__ __forceinline__ long long share_first_tile(const PairShares& r, int c, long long C,
                                                      int grid) {
  if (c > r.c1) return r.pair0 + r.ntp;
  return r.pair0 + (share_begin(c, C, grid) - r.pos0 + kCostTile - 1) / kCostTile;
}
// Does share c (c0 <= c <= c1) hold a tile of the pair?
__device__ __forceinline__ bool share_holds(const PairShares& r, int c, long long C, int grid) {
  return c == r.c0 || share_first_tile(r, c, C, grid) < share_first_tile(r, c + 1, C, grid);
}
__device__ __forceinline__ int pair_pieces(const PairShares& r, long long C, int grid) {
  int n = 0;
  for (int c = r.c0; c <= r.c1; ++c) n += share_holds(r, c, C, grid);
  return n;
}

// Tiles of sequence b in this pass (0 for an empty pass or a bad length).
template <int BS>
__device__ __forceinline__ int seq_tiles(const DecodeArgs& a, int b, int& ctx, int& start) {
  ctx = __ldg(a.context_lens + b);
  start = a.start_blocks ? __ldg(a.start_blocks + b) * BS : 0;
  if (ctx < 0 || ctx > a.max_blocks * BS || ctx > a.max_context_len || start < 0 || start > ctx)
    return 0;
  return (ctx - start + kRt - 1) / kRt;
}
template <int BS>
__device__ __forceinline__ bool seq_bad(const DecodeArgs& a, int ctx, int start) {
  return ctx < 0 || ctx > a.max_blocks * BS || ctx > a.max_context_len || start < 0 ||
         start > ctx;
}

// A walk over this CTA's share, one unit (a pair, or a piece of one) at a time.
struct Cursor {
  int b, h;             // current pair
  int p;                // its index among the pairs with tiles
  int k0, k1;           // tiles [k0, k1) of the pair in this unit
  int ntp;              // tiles of the pair
  int ctx, start;       // the sequence's length and the first token of the pass
  long long g0;         // global index of the unit's first tile
  long long left;       // tiles of the share after this unit
  bool valid;
};

__device__ __forceinline__ void cur_fill(Cursor& c, int k0, long long budget) {
  c.k0 = k0;
  const long long n = min((long long)(c.ntp - k0), budget);
  c.k1 = k0 + (int)n;
  c.left = budget - n;
}

template <int BS>
__device__ __forceinline__ void cur_init(const DecodeArgs& a, Cursor& c, const Misc* ms) {
  c.valid = ms->valid != 0;
  if (!c.valid) return;
  c.b = ms->b0;
  c.h = ms->h0;
  c.p = ms->p0;
  c.ntp = seq_tiles<BS>(a, c.b, c.ctx, c.start);
  c.g0 = ms->r0;
  cur_fill(c, ms->k0, ms->r1 - ms->r0);
}

// Move to the next unit of the share (pairs with no tiles are skipped).
template <int BS>
__device__ __forceinline__ void cur_next(const DecodeArgs& a, int nhg, Cursor& c) {
  if (!c.valid) return;
  if (c.left <= 0) { c.valid = false; return; }
  c.g0 += c.k1 - c.k0;
  ++c.p;
  if (++c.h >= nhg) {
    c.h = 0;
    int n = 0;
    do {
      if (++c.b >= a.B) { c.valid = false; return; }
      n = seq_tiles<BS>(a, c.b, c.ctx, c.start);
    } while (n == 0);
    c.ntp = n;
  }
  cur_fill(c, 0, c.left);
}

struct Unit {
  int b, h, ctx, t0, t1, ntiles, ntp;
  bool whole;           // the unit is its whole pair
  long long g0;         // global index of its first tile
  long long pair0;      // global index of the pair's first tile
  int p;                // the pair's index among the pairs with tiles
};

__device__ __forceinline__ Unit unit_of(const Cursor& c) {
  Unit x;
  x.b = c.b; x.h = c.h; x.ctx = c.ctx; x.ntp = c.ntp;
  x.t0 = c.start + c.k0 * kRt;
  x.t1 = min(c.ctx, c.start + c.k1 * kRt);
  x.ntiles = c.k1 - c.k0;
  x.whole = c.k0 == 0 && c.k1 == c.ntp;
  x.g0 = c.g0;
  x.pair0 = c.g0 - c.k0;
  x.p = c.p;
  return x;
}

// A tile position of the walk (for look-ahead of block ids).
struct TilePos {
  Cursor c;
  int k;                // tile within the unit
};
template <int BS>
__device__ __forceinline__ void next_tile(const DecodeArgs& a, int nhg, TilePos& p) {
  if (!p.c.valid) return;
  if (++p.k >= p.c.k1 - p.c.k0) { p.k = 0; cur_next<BS>(a, nhg, p.c); }
}

// Prologue (the 128 threads of warps 0-3; stage 0 as scratch): count the
// tiles and the pairs with tiles, zero the output rows of sequences with none
// (CTA b % grid owns sequence b's rows), and find the global tiles where this
// CTA's share starts and ends. Two short passes over context_lens, each a
// block-wide reduction or scan.
template <int BS>
__device__ void plan_share(const DecodeArgs& a, int nhg, uint8_t* scratch, Misc* ms) {
  constexpr int PER = kScanChunk / 128;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int grid = (int)gridDim.x, cta = (int)blockIdx.x;
  int* empty_s = reinterpret_cast<int*>(scratch);                   // [kScanChunk]
  int* nempty = empty_s + kScanChunk;
  long long* wsum = reinterpret_cast<long long*>(scratch + 4 * kScanChunk + 64);   // [2][4 warps]
  auto bar = [] { asm volatile("bar.sync 1, 128;" ::: "memory"); };

  // pass 1: tiles of every sequence (per KV-head group), sequences with tiles;
  // rows of empty ones
  long long mine = 0, mine_ne = 0;
  for (int b0 = 0; b0 < a.B; b0 += kScanChunk) {
    if (tid == 0) *nempty = 0;
    bar();
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      const int b = b0 + e * 128 + tid;
      if (b >= a.B) break;
      int ctx, st;
      const int n = seq_tiles<BS>(a, b, ctx, st);
      mine += n;
      mine_ne += n > 0;
      if (n == 0 && (b % grid) == cta) empty_s[atomicAdd(nempty, 1)] = b;
    }
    bar();
    for (int k = 0; k < *nempty; ++k) {
      const int b = empty_s[k];
      int ctx, st;
      (void)seq_tiles<BS>(a, b, ctx, st);
      if (seq_bad<BS>(a, ctx, st) && tid == 0) flag_error(a.err_flag, PA_DEV_BAD_CTX);
      if (!a.force_split)                 // the split-only pass leaves every row to the merge
        for (int i = tid; i < a.Hq * kD; i += 128)
          store_out(a.out, (size_t)b * a.Hq * kD + i, 0.f, a.out_dtype);
    }
    bar();
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    mine += __shfl_xor_sync(0xffffffffu, mine, o);
    mine_ne += __shfl_xor_sync(0xffffffffu, mine_ne, o);
  }
  if (lane == 0) { wsum[warp] = mine; wsum[4 + warp] = mine_ne; }
  bar();
  const long long T = (long long)nhg * (wsum[0] + wsum[1] + wsum[2] + wsum[3]);
  const long long NP = (long long)nhg * (wsum[4] + wsum[5] + wsum[6] + wsum[7]);
  const long long pc = a.pair_cost;
  const long long C = kCostTile * T + pc * NP;
  // the share: tiles whose cost positions lie in [t0, t1)
  const long long t0 = T > 0 ? share_begin(cta, C, grid) : 0;
  const long long t1 = T > 0 ? share_begin(cta + 1, C, grid) : 0;
  bar();
  if (tid == 0) {
    ms->C = C; ms->r0 = T; ms->r1 = T;
    ms->valid = 0; ms->found = 0;
  }
  bar();
  if (T == 0 || t0 >= t1) return;

  // pass 2: the first tile whose position is >= t0 (the share's first) and the
  // first whose position is >= t1 (the next share's first), a scan over the
  // sequences, 128 a round; each sequence with tiles holds the targets that
  // lie after its predecessor's last tile position and up to its own last.
  long long carry = 0, carry_ne = 0;      // tiles per group, sequences with tiles, before this round
  for (int b0 = 0; b0 < a.B; b0 += 128) {
    const int b = b0 + tid;
    int ctx = 0, st = 0;
    const int n = b < a.B ? seq_tiles<BS>(a, b, ctx, st) : 0;
    long long incl = n, incl_ne = n > 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long t = __shfl_up_sync(0xffffffffu, incl, o);
      const long long u = __shfl_up_sync(0xffffffffu, incl_ne, o);
      if (lane >= o) { incl += t; incl_ne += u; }
    }
    if (lane == 31) { wsum[warp] = incl; wsum[4 + warp] = incl_ne; }
    bar();
    long long wpre = 0, wpre_ne = 0;
    for (int w = 0; w < warp; ++w) { wpre += wsum[w]; wpre_ne += wsum[4 + w]; }
    if (n > 0) {
      const long long x0 = (long long)nhg * (carry + wpre + incl - n);     // its first global tile
      const long long p0 = (long long)nhg * (carry_ne + wpre_ne + incl_ne - 1);   // its first pair
      const long long last = tile_cost(x0 + (long long)nhg * n - 1, p0 + nhg - 1, pc);
      const long long prev = p0 > 0 ? tile_cost(x0 - 1, p0 - 1, pc) : -1;
      // the first tile of this sequence at position >= t (prev < t <= last)
      auto locate = [&](long long t, int& h, int& k) {
        h = 0;
        while (h + 1 < nhg && tile_cost(x0 + (long long)(h + 1) * n - 1, p0 + h, pc) < t) ++h;
        const long long first = tile_cost(x0 + (long long)h * n, p0 + h, pc);
        k = t <= first ? 0 : (int)((t - first + kCostTile - 1) / kCostTile);
      };
      if (prev < t0 && t0 <= last) {
        int h, k;
        locate(t0, h, k);
        ms->b0 = b;
        ms->h0 = h;
        ms->k0 = k;
        ms->p0 = (int32_t)(p0 + h);
        ms->r0 = x0 + (long long)h * n + k;
        ms->valid = 1;
        atomicOr(&ms->found, 1);
      }
      if (prev < t1 && t1 <= last) {
        int h, k;
        locate(t1, h, k);
        ms->r1 = x0 + (long long)h * n + k;
        atomicOr(&ms->found, 2);
      }
    }
    carry += wsum[0] + wsum[1] + wsum[2] + wsum[3];
    carry_ne += wsum[4] + wsum[5] + wsum[6] + wsum[7];
    bar();
    if (ms->found == 3) break;
  }
  bar();
  // no tile at or after t1: the share runs to the end of the list
  if (tid == 0 && ms->valid && ms->r0 >= ms->r1) ms->valid = 0;
  bar();
}

// Take a ticket on a pair: true for the piece that arrives last. Lock-free
// (every failed exchange means another piece succeeded), bounded anyway.
__device__ __forceinline__ bool take_ticket(unsigned long long* word, unsigned long long epoch,
                                            int npieces, uint32_t* err_flag) {
  unsigned long long cur = atomicAdd(word, 0ull);
#pragma unroll 1
  for (int it = 0; it < (1 << 20); ++it) {
    const unsigned long long cnt = (cur >> kEpochShift) == epoch ? (cur & kCountMask) : 0ull;
    const unsigned long long want = (epoch << kEpochShift) | (cnt + 1);
    const unsigned long long prev = atomicCAS(word, cur, want);
    if (prev == cur) return (int)(cnt + 1) == npieces;
    cur = prev;
  }
  flag_error(err_flag, PA_DEV_TIMEOUT);
  return false;
}

// The last piece of a pair: merge every piece's (m, l, o) of the group's NS
// query heads. 128 threads: thread `row` takes query head n = row / TPR and
// DPT consecutive d. A piece's loads (m, l and its DPT values) are issued
// together, and with DPT <= 16 two pieces' (more would cost registers the
// CTA does not have). Writes the staging buffer (normalised output rows in
// the output type, or, in the split-only pass, fp32 rows plus M and L).
template <int G>
__device__ __forceinline__ void merge_pieces(const DecodeArgs& a, const Unit& x, int row,
                                             uint8_t* stg, long long C, int grid, bool final_out,
                                             size_t cas_row0) {
  constexpr int NS = kHG * G, TPR = 128 / NS, DPT = kD / TPR;
  constexpr int NB = DPT <= 16 ? 2 : 1;          // pieces whose loads are in flight together
  const int n = row / TPR, d0 = (row % TPR) * DPT;
  const PairShares ps = pair_shares(x.pair0, x.ntp, x.p, C, grid, a.pair_cost);
  float M = -CUDART_INF_F, L = 0.f, o[DPT];
#pragma unroll
  for (int e = 0; e < DPT; ++e) o[e] = 0.f;
#pragma unroll 1
  for (int c = ps.c0; c <= ps.c1; c += NB) {
    float m[NB], l[NB];
    float4 v[NB][DPT / 4];
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      const int cj = c + j;
      const bool has = cj <= ps.c1 && share_holds(ps, cj, C, grid);   // else no piece there
      const size_t s = 2 * (size_t)cj + (cj == ps.c0 && ps.c0_before ? 1 : 0);
      m[j] = has ? __ldcg(a.sk_m + s * NS + n) : -CUDART_INF_F;
      l[j] = has ? __ldcg(a.sk_l + s * NS + n) : 0.f;
      const float4* src = reinterpret_cast<const float4*>(a.sk_acc + (s * NS + n) * kD + d0);
#pragma unroll
      for (int e = 0; e < DPT / 4; ++e) v[j][e] = has ? __ldcg(src + e) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      if (m[j] == -CUDART_INF_F) continue;    // no piece, or no valid token in it
      const float Mn = fmaxf(M, m[j]);
      const float ca = exp2f(M - Mn), cb = exp2f(m[j] - Mn);   // M = -inf gives ca = 0
      L = fmaf(L, ca, l[j] * cb);
#pragma unroll
      for (int e = 0; e < DPT / 4; ++e) {
        o[4 * e + 0] = fmaf(o[4 * e + 0], ca, v[j][e].x * cb);
        o[4 * e + 1] = fmaf(o[4 * e + 1], ca, v[j][e].y * cb);
        o[4 * e + 2] = fmaf(o[4 * e + 2], ca, v[j][e].z * cb);
        o[4 * e + 3] = fmaf(o[4 * e + 3], ca, v[j][e].w * cb);
      }
      M = Mn;
    }
  }
  if (final_out) {
    const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
    for (int e = 0; e < DPT; ++e) store_out(stg, (size_t)n * kD + d0 + e, o[e] * inv, a.out_dtype);
  } else {
#pragma unroll
    for (int e = 0; e < DPT; ++e) reinterpret_cast<float*>(stg)[n * kD + d0 + e] = o[e];
    if (row % TPR == 0) {
      a.ws_m[cas_row0 + n] = M;
      a.ws_l[cas_row0 + n] = L;
    }
  }
}

// Two 16-bit query elements of a 32-bit word (element 0 in the low half) as fp32.
template <int FMT>
__device__ __forceinline__ float2 q_pair(uint32_t w) {
  if (FMT == 1) return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
  return __half22float2(*reinterpret_cast<const __half2*>(&w));
}

// KV8: the pools hold FP8 E4M3 codes (K times k_scale, folded into the score
// scale; V times v_scale, folded into the output weights). TMA brings a tile's
// codes into 16 KB stages; the score product reads the K codes as they are,
// and the softmax group that owns the tile, once it has written the tile's
// weights, widens the V codes into the group's V buffer and frees the stage.
template <int FMT, int BS, int G, bool KV8>
__global__ void __launch_bounds__(kThreads, 1)
decode_tc_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmQ) {
  using S = TcShape<G, KV8>;
  constexpr int NST = S::kStages;
  using Bx = Bars<NST>;
  constexpr int NS = S::NS, NOH = S::NOH, NO = S::NO;
  constexpr int RB = BS < kRt ? BS : kRt;        // token rows per TMA box (per head)
  constexpr int NQ = kRt / RB;                   // boxes per d-half per tile
  constexpr int KS = kRt / 16;                   // output-MMA K steps per head per tile
  constexpr int NCH = NQ * kHG;                  // (box, head) row chunks per tile
  // FP8 pools. The score product runs on the K codes themselves
  // (kind::f8f6f4): the query of each head is scaled by an exact power of two
  // and split into E4M3 pieces, q = 2^e (q1 + q2 [+ q3]), each the rounding of
  // what the earlier ones leave; two pieces hold a bf16 value exactly (4 + 4
  // significant bits), three an f16 value, unless an element lies below the
  // E4M3 grid (2^-17 of the head's largest element). The scores take 2^e back.
  // The output product runs on f16 operands whatever the query type: E4M3 ->
  // f16 is one conversion per pair of codes (bf16 would take several).
  constexpr int CF = KV8 ? 0 : FMT;             // element type of the output product
  constexpr bool QCNV = KV8;                    // the query becomes E4M3 pieces
  constexpr int NPU = FMT == 1 ? 2 : 3;         // pieces the score product uses
  constexpr uint32_t IDESC_S = make_idesc(CF, 0, 0, KV8 ? NPU * NS : NS, 128);
  constexpr uint32_t IDESC_O = make_idesc(CF, 1, 0, NOH, 128);
  static_assert(NCH * RB == kRows && NCH <= 8, "tile geometry");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + S::OFF_BAR;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  Misc* ms = reinterpret_cast<Misc*>(smem + S::OFF_MISC);
  volatile uint32_t* abort_flag = &ms->abort_flag;
  const int nhg = a.Hkv / kHG;
  const uint64_t wait_ns = a.wait_ns;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_trigger();

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(bar(Bx::FULL + s), 1);
      mbar_init(bar(Bx::EMPTY + s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(Bx::QFULL + i), 1);
      mbar_init(bar(Bx::QEMPTY + i), 1);
      mbar_init(bar(Bx::SFULL + i), 1);
      mbar_init(bar(Bx::SFREE + i), 128);
      mbar_init(bar(Bx::PREADY + i), 128);
      mbar_init(bar(Bx::OFULL + i), 1);
      mbar_init(bar(Bx::XFULL + i), 128);
      mbar_init(bar(Bx::XFREE + i), 128);
    }
    mbar_init(bar(Bx::ODONE), 128);
    mbar_init(bar(Bx::ODONE + 1), 128);
    mbar_init(bar(Bx::DONE), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(Bx::QCONV + i), 128);
      mbar_init(bar(Bx::QSREAD + i), 256);
    }
    ms->abort_flag = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 8) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(&ms->tmem)),
                 "r"(S::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  pdl_wait();                            // global memory from here on
  if (warp < 4) {
    plan_share<BS>(a, nhg, smem, ms);
    fence_proxy_async();                 // stage 0 served as scratch; TMA writes it next
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms->tmem;
  const uint32_t tmem_s = tmem;                 // S buffers: [0, NS) and [NS, 2NS)
  // O accumulators from column 2NS: [unit parity][group], NO columns each, so the
  // next unit accumulates while the previous one is merged
  const uint32_t tmem_o = tmem + 2 * S::SW;
  auto obuf = [&](int ui, int g) { return tmem_o + (uint32_t)((2 * (ui & 1) + g) * NO); };
  const long long C = ms->C, r0 = ms->r0;
  const int grid = (int)gridDim.x, cta = (int)blockIdx.x;
  auto give_up = [&]() {
    *abort_flag = 1u;
    flag_error(a.err_flag, PA_DEV_TIMEOUT);
  };
  // K of a tile is ready for the tensor cores when TMA has filled its stage. V
  // is ready when TMA has filled its stage (16-bit pools), or, with FP8 pools,
  // when the group that owns the tile has widened its codes into the group's V
  // buffer, which it does before it hands over the tile's P (PREADY).
  auto k_ready_bar = [&](int s) { return bar(Bx::FULL + s); };
  // token range of tile k of a unit, and how many of its boxes hold tokens
  auto tile_span = [&](const Unit& x, int k, int& ts, int& te, int& nql) {
    ts = x.t0 + k * kRt;
    te = min(x.t1, ts + kRt);
    nql = (te - ts + RB - 1) / RB;
  };

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int tc = 0, issued = 0;
      int q_last[2] = {-1, -1};                    // last unit whose query went to buffer 0 / 1
      int phys_next[NQ];
      // block ids of the tile at p (-1 past the share's end)
      auto load_ids = [&](const TilePos& p, int* ph) {
        if (!p.c.valid) {
#pragma unroll
          for (int q = 0; q < NQ; ++q) ph[q] = -1;
          return;
        }
        const Unit x = unit_of(p.c);
        int ts, te, nql;
        tile_span(x, p.k, ts, te, nql);
        const int32_t* table = a.block_tables + (size_t)x.b * a.max_blocks;
#pragma unroll
        for (int q = 0; q < NQ; ++q) ph[q] = q < nql ? __ldg(table + (ts + q * RB) / BS) : -1;
      };
      Cursor cur;
      cur_init<BS>(a, cur, ms);
      TilePos ahead{cur, 0};
      load_ids(ahead, phys_next);
      for (int i = 0; cur.valid; ++i, cur_next<BS>(a, nhg, cur)) {
        const Unit x = unit_of(cur);
        const int qi = i & 1;
        if (!mbar_wait(bar(Bx::QEMPTY + qi), ((i >> 1) & 1) ^ 1, abort_flag, wait_ns)) { give_up(); goto prod_done; }
        if (!(a.test_withhold_q && i == 0)) {
          mbar_expect_tx(bar(Bx::QFULL + qi), 2u * NS * 128u);
          for (int hh = 0; hh < 2; ++hh)
            tma_load_2d(sbase + S::OFF_Q + qi * S::kQBytes + hh * (NS * 128), &tmQ, hh * 64,
                        x.b * a.Hq + x.h * kHG * G, bar(Bx::QFULL + qi));
          q_last[qi] = i;
        }
        for (int k = 0; k < x.ntiles; ++k) {
          int ts, te, nql;
          tile_span(x, k, ts, te, nql);
          int phys[NQ];
          uint32_t bytes = 0;
#pragma unroll
          for (int q = 0; q < NQ; ++q) {
            phys[q] = phys_next[q];
            if (phys[q] >= 0 && phys[q] < a.num_blocks) bytes += (KV8 ? 1u : 2u) * RB * kHG * 128u;
          }
          next_tile<BS>(a, nhg, ahead);
          load_ids(ahead, phys_next);
          for (int kv = 0; kv < 2; ++kv) {
            const int seq = 2 * tc + kv, s = seq % NST;
            if (!mbar_wait(bar(Bx::EMPTY + s), ((seq / NST) & 1) ^ 1, abort_flag, wait_ns)) { give_up(); goto prod_done; }
            mbar_expect_tx(bar(Bx::FULL + s), bytes);
            const uint32_t dst = sbase + s * S::kStage;
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
              if (phys[q] < 0 || phys[q] >= a.num_blocks) continue;
              const int rr0 = (ts + q * RB) % BS;
              if (KV8) {
                // all 128 codes of a row in one 128-byte line
                tma_load_4d(dst + q * (kHG * RB * 128), kv ? &tmV : &tmK, 0, rr0,
                            x.h * kHG, phys[q], bar(Bx::FULL + s));
              } else {
                for (int hh = 0; hh < 2; ++hh)
                  tma_load_5d(dst + hh * kHalf + q * (kHG * RB * 128), kv ? &tmV : &tmK, 0, rr0,
                              x.h * kHG, hh, phys[q], bar(Bx::FULL + s));
              }
            }
            ++issued;
          }
          ++tc;
        }
      }
    prod_done:
      // never leave with copies in flight: wait (bounded) for the last loads of
      // every stage and of both query buffers
      for (int seq = max(0, issued - NST); seq < issued; ++seq) {
        const int s = seq % NST;
        const uint64_t t0 = globaltimer();
        while (!mbar_try(bar(Bx::FULL + s), (seq / NST) & 1) && globaltimer() - t0 < kWaitNs) {}
      }
      for (int qb = 0; qb < 2; ++qb) {
        if (q_last[qb] < 0) continue;
        const uint64_t t0 = globaltimer();
        while (!mbar_try(bar(Bx::QFULL + qb), (q_last[qb] >> 1) & 1) && globaltimer() - t0 < kWaitNs) {}
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int tc = 0;
      bool ok = true;
      // output product of tile tt (unit ui, tile kk of the unit, nql boxes with tokens)
      auto issue_pv = [&](int tt, int ui, int kk, int nql) -> bool {
        const int pb = tt & 1;
        if (!mbar_wait(bar(Bx::PREADY + pb), (tt >> 1) & 1, abort_flag, wait_ns)) return false;
        const bool first = kk <= 1;                   // this group's first tile of the unit
        // the unit's accumulators were last used by unit ui - 2: wait for its merge
        if (first && ui >= 2 &&
            !mbar_wait(bar(Bx::ODONE + (ui & 1)), ((ui - 2) >> 1) & 1, abort_flag, wait_ns))
          return false;
        const int seq = 2 * tt + 1, s = seq % NST;
        // FP8 pools: the group widened V into its buffer before handing over P
        if (!KV8 && !mbar_wait(bar(Bx::FULL + s), (seq / NST) & 1, abort_flag, wait_ns)) return false;
        tc_fence_after();
        const uint32_t vst = KV8 ? sbase + S::OFF_VOP + pb * kStageBytes : sbase + s * S::kStage;
        const uint32_t pst = sbase + S::OFF_P + pb * S::kPBytes;
#pragma unroll
        for (int h = 0; h < kHG; ++h) {
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) {
            if (ks * 16 >= nql * RB) continue;       // no tokens loaded there
            const int q = (ks * 16) / RB;
            const int row0 = q * (kHG * RB) + h * RB + (ks * 16) % RB;
            const int c = h * KS + ks;                // 32-byte chunk of the P operand
            // A = V^T (MN-major): 16 rows of head h from row0; d-halves 16 KB apart
            const uint64_t ad = sw128_desc(vst + row0 * 128, kHalf, 1024);
            // B = [P_hi; P_lo] of head h, K-major, chunk c of the 2-line P tile
            const uint64_t bd = sw128_desc(pst + (c >> 2) * (NOH * 128) + (c & 3) * 32, 16, 1024);
            mma_f16(obuf(ui, pb) + h * NOH, ad, bd, IDESC_O, (first && ks == 0) ? 0u : 1u);
          }
        }
        if (!KV8) mma_commit(bar(Bx::EMPTY + s));   // FP8: the group freed the code stage
        mma_commit(bar(Bx::OFULL + pb));
        return true;
      };
      int pui = 0, pkk = 0, pnql = 0;                // the tile waiting for its output product
      bool pending = false;                          // tile tc - 1 still needs its output product
      Cursor cur;
      cur_init<BS>(a, cur, ms);
      for (int i = 0; cur.valid && ok; ++i, cur_next<BS>(a, nhg, cur)) {
        const Unit x = unit_of(cur);
        const int qi = i & 1;
        if (!mbar_wait(bar(Bx::QFULL + qi), (i >> 1) & 1, abort_flag, wait_ns)) { ok = false; break; }
        if (QCNV && !mbar_wait(bar(Bx::QCONV + qi), (i >> 1) & 1, abort_flag, wait_ns)) { ok = false; break; }
        const uint32_t qst = sbase + S::OFF_Q + qi * S::kQBytes;
        for (int k = 0; k < x.ntiles; ++k) {
          int ts, te, nql;
          tile_span(x, k, ts, te, nql);
          const int sb = tc & 1;
          const int seq = 2 * tc, s = seq % NST;
          if (pending) {
            // whichever comes first: the softmax of tile tc - 1 (issue its output
            // product now, so its V stage and its group are released early) or
            // the inputs of S(tc)
            const uint64_t t0 = globaltimer();
            while (true) {
              if (mbar_test(bar(Bx::PREADY + ((tc - 1) & 1)), ((tc - 1) >> 1) & 1)) {
                if (!issue_pv(tc - 1, pui, pkk, pnql)) ok = false;
                pending = false;
                break;
              }
              if (mbar_test(bar(Bx::SFREE + sb), ((tc >> 1) & 1) ^ 1) &&
                  mbar_test(k_ready_bar(s), (seq / NST) & 1))
                break;
              if (*abort_flag || globaltimer() - t0 > wait_ns) { ok = false; break; }
            }
            if (!ok) break;
          }
          if (!mbar_wait(bar(Bx::SFREE + sb), ((tc >> 1) & 1) ^ 1, abort_flag, wait_ns)) { ok = false; break; }
          if (!mbar_wait(k_ready_bar(s), (seq / NST) & 1, abort_flag, wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t kst = sbase + s * S::kStage;
          if constexpr (QCNV) {
            // K codes (one 128-byte line per row) times the query pieces, which
            // stand one after another as NPU * NS rows of B: each piece's scores
            // land in their own NS columns (4 steps of 32 codes)
#pragma unroll
            for (int ks = 0; ks < kD / 32; ++ks) {
              const uint64_t ad = sw128_desc(kst + ks * 32, 16, 1024);
              const uint64_t bd = sw128_desc(qst + ks * 32, 16, 1024);
              mma_f8(tmem_s + sb * S::SW, ad, bd, IDESC_S, ks > 0 ? 1u : 0u);
            }
          } else {
#pragma unroll
            for (int ks = 0; ks < kD / 16; ++ks) {
              const uint64_t ad = sw128_desc(kst + (ks >> 2) * kHalf + (ks & 3) * 32, 16, 1024);
              const uint64_t bd = sw128_desc(qst + (ks >> 2) * (NS * 128) + (ks & 3) * 32, 16, 1024);
              mma_f16(tmem_s + sb * S::SW, ad, bd, IDESC_S, ks > 0 ? 1u : 0u);
            }
          }
          mma_commit(bar(Bx::EMPTY + s));
          mma_commit(bar(Bx::SFULL + sb));
          if (k == x.ntiles - 1) mma_commit(bar(Bx::QEMPTY + qi));
          if (pending && !issue_pv(tc - 1, pui, pkk, pnql)) { ok = false; break; }
          pending = true;
          pui = i; pkk = k; pnql = nql;
          ++tc;
        }
      }
      if (ok && pending && !issue_pv(tc - 1, pui, pkk, pnql)) ok = false;
      if (!ok) give_up();
      // all issued MMAs must finish before tensor memory is released
      mma_commit(bar(Bx::DONE));
      const uint64_t t0 = globaltimer();
      while (!mbar_try(bar(Bx::DONE), 0) && globaltimer() - t0 < kWaitNs) {}
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax / output groups
    const int grp = warp >> 2;                     // group: tiles t with t % 2 == grp
    const int wq = warp & 3;                       // TMEM lane quadrant of this warp
    const int row = threadIdx.x & 127;             // tile row (head, token) for S; d row for O
    const uint32_t lane_off = (uint32_t)(32 * wq) << 16;
    const int rq = row / (kHG * RB), rh = (row / RB) % kHG, rr = row % RB;
    const int tt_row = rq * RB + rr;               // this row's token within its head's tile
    const int col0 = ((32 * wq / RB) % kHG) * G;   // first S column this warp reads
    float* red = reinterpret_cast<float*>(smem + S::OFF_RED) + grp * 16 * S::GP;     // [2][8][GP]
    float* red_l = reinterpret_cast<float*>(smem + S::OFF_REDL) + grp * 16 * S::GP;  // [2][8][GP]
    float* mold = reinterpret_cast<float*>(smem + S::OFF_MREF) + grp * 3 * NS;      // [NS]
    float* mnew = mold + NS;                                                         // [NS]
    float* mown = mnew + NS;                                                         // [NS]
    float* xbuf = reinterpret_cast<float*>(smem + S::OFF_X);                   // [2][2][NS] + flags
    int* xflag = reinterpret_cast<int*>(smem + S::OFF_X + 2 * 2 * NS * 4);    // [2]
    uint8_t* pbuf = smem + S::OFF_P + grp * S::kPBytes;
    // P address of this row: head rh, K step tt_row / 16, element tt_row % 16
    const int pc = rh * KS + tt_row / 16, pe = tt_row % 16;
    uint8_t* prow = pbuf + (pc >> 2) * (NOH * 128);
    const int pchunk = (pc & 3) * 2 + (pe >> 3), pbyte = (pe & 7) * 2;
    bool failed = false;
    int tc = 0;                                    // global tile index
    // Wait for the output product of this group's tile t, the latest tile it
    // handed over. A parity wait is exact here: the barrier cannot pass t's
    // phase before the group hands over tile t + 2, and it has already passed
    // the phase before t's (the group has seen S of a tile >= t, and the
    // issuer puts S(t) after O(t - 2) on the same in-order tensor pipe).
    auto wait_pv = [&](int t) {
      if (!mbar_wait(bar(Bx::OFULL + grp), (t >> 1) & 1, abort_flag, wait_ns)) failed = true;
    };
    auto row_id = [&](const TilePos& p) -> int {
      if (!p.c.valid) return -1;
      const Unit x = unit_of(p.c);
      int ts, te, nql;
      tile_span(x, p.k, ts, te, nql);
      return rq < nql ? __ldg(a.block_tables + (size_t)x.b * a.max_blocks + (ts + rq * RB) / BS) : -1;
    };
    Cursor cur;
    cur_init<BS>(a, cur, ms);
    TilePos ahead{cur, 0};
    if (grp == 1) next_tile<BS>(a, nhg, ahead);              // group 1 starts at tile 1
    int phys_next = row_id(ahead);
    bool stop = false;
    for (int i = 0; cur.valid && !stop; ++i, cur_next<BS>(a, nhg, cur)) {
      const Unit x = unit_of(cur);
      float mo[G], l[G];                           // this row's head: reference max, exp-sum
#pragma unroll
      for (int g = 0; g < G; ++g) { mo[g] = -CUDART_INF_F; l[g] = 0.f; }
      int my_last = -1;
      float qcs[G];                                // score scale of each query head of this row's head
      if constexpr (QCNV) {
        // the group that takes the unit's first tile turns its 16-bit query into
        // E4M3 pieces in place: query head n is scaled by 2^-e_n (its largest |q|
        // lands in [2^7, 2^8), below the E4M3 maximum 448) and split as
        // q1 = RN(q), q2 = RN(q - q1), q3 = RN(q - q1 - q2); the head's score
        // scale takes 2^e_n
        const int qi = i & 1;
        float* qsc = reinterpret_cast<float*>(smem + S::OFF_QSC) + qi * NS;
        if ((tc & 1) == grp) {
          if (!mbar_wait(bar(Bx::QFULL + qi), (i >> 1) & 1, abort_flag, wait_ns)) failed = true;
          // the scales of unit i - 2 (same buffer) have been read by both groups
          if (i >= 2 && !mbar_wait(bar(Bx::QSREAD + qi), ((i - 2) >> 1) & 1, abort_flag, wait_ns))
            failed = true;
          constexpr int TPQ = 128 / NS, CPT = 16 / TPQ;       // threads per query head, chunks each
          const int n = row / TPQ, part = row % TPQ;
          uint8_t* qb = smem + S::OFF_Q + qi * S::kQBytes;
          // the 16-bit query: [2 d-halves][NS rows][128 B], 128-byte swizzled
          uint4 v[CPT];
          float mx = 0.f;
#pragma unroll
          for (int j = 0; j < CPT; ++j) {
            const int ch = part * CPT + j, hh = ch >> 3, c = ch & 7;
            v[j] = *reinterpret_cast<const uint4*>(qb + hh * (NS * 128) + n * 128 + ((c ^ (n & 7)) << 4));
            const uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = q_pair<FMT>(w[e]);
              mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
            }
          }
#pragma unroll
          for (int o = TPQ / 2; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          // every row has been read before the pieces overwrite the buffer
          if (!wg_vote_or(failed, grp)) {
            int e2 = 0;
            if (mx > 0.f && mx <= FLT_MAX)
              e2 = min(max((int)((__float_as_uint(mx) >> 23) & 0xff) - 127 - 7, -100), 100);
            const float down = __uint_as_float((uint32_t)(127 - e2) << 23);   // 2^-e2
            // the pieces: [NPU][NS rows][128 codes], 128-byte swizzled (K-major)
#pragma unroll
            for (int j = 0; j < CPT; ++j) {
              const int ch = part * CPT + j, hh = ch >> 3, c = ch & 7;
              const int d0 = hh * 64 + c * 8;                   // first of the chunk's 8 elements
              const uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
              uint32_t pw[NPU][2];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 f = q_pair<FMT>(w[e]);
                float r0 = f.x * down, r1 = f.y * down;        // exact: a power of two
#pragma unroll
                for (int pc = 0; pc < NPU; ++pc) {
                  const __nv_fp8x2_storage_t h =
                      __nv_cvt_float2_to_fp8x2(make_float2(r0, r1), __NV_SATFINITE, __NV_E4M3);
                  if ((e & 1) == 0) pw[pc][e >> 1] = 0u;
                  pw[pc][e >> 1] |= (uint32_t)h << ((e & 1) * 16);
                  if (pc + 1 < NPU) {                          // what this piece leaves (exact)
                    const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(h, __NV_E4M3);
                    const float2 hf = __half22float2(*reinterpret_cast<const __half2*>(&hr));
                    r0 -= hf.x;
                    r1 -= hf.y;
                  }
                }
              }
              const int off = n * 128 + (((d0 >> 4) ^ (n & 7)) << 4) + (d0 & 15);
#pragma unroll
              for (int pc = 0; pc < NPU; ++pc)
                *reinterpret_cast<uint2*>(qb + pc * (NS * 128) + off) = make_uint2(pw[pc][0], pw[pc][1]);
            }
            if (part == 0) qsc[n] = a.scale_log2 * __uint_as_float((uint32_t)(127 + e2) << 23);
          } else {
            failed = true;
          }
          fence_proxy_async();                     // the pieces -> the tensor cores
          mbar_arrive(bar(Bx::QCONV + qi));
        }
        if (!mbar_wait(bar(Bx::QCONV + qi), (i >> 1) & 1, abort_flag, wait_ns)) failed = true;
#pragma unroll
        for (int g = 0; g < G; ++g) qcs[g] = qsc[rh * G + g];
        mbar_arrive(bar(Bx::QSREAD + qi));
      } else {
#pragma unroll
        for (int g = 0; g < G; ++g) qcs[g] = a.scale_log2;
      }
      for (int k = 0; k < x.ntiles; ++k, ++tc) {
        if ((tc & 1) != grp) continue;
        int ts, te, nql;
        tile_span(x, k, ts, te, nql);
        const bool in_range = rq < nql;
        const int phys = phys_next;
        next_tile<BS>(a, nhg, ahead);                         // two tiles ahead: the next own tile
        next_tile<BS>(a, nhg, ahead);
        phys_next = row_id(ahead);
        const bool blk_ok = phys >= 0 && phys < a.num_blocks;
        const bool valid = in_range && blk_ok && ts + tt_row < te;
        if (in_range && !blk_ok && rr == 0 && rh == 0) flag_error(a.err_flag, PA_DEV_BAD_BLOCK_ID);
        const bool first = my_last < 0;

        const int par = (tc >> 1) & 1;                        // use count of this group's buffers
        if (!mbar_wait(bar(Bx::SFULL + grp), par, abort_flag, wait_ns)) failed = true;
        tc_fence_after();
        constexpr int SVN = ((32 / RB) * G + 15) / 16 * 16;  // S columns this warp loads
        float sv[SVN];
#pragma unroll
        for (int c = 0; c < SVN; c += 16) tmem_ld16(tmem_s + lane_off + grp * S::SW + col0 + c, sv + c);
        if constexpr (KV8) {
          // the query pieces' scores: S = S(q1) + S(q2) [+ S(q3)]
#pragma unroll
          for (int pc = 1; pc < NPU; ++pc) {
            float sp[SVN];
#pragma unroll
            for (int c = 0; c < SVN; c += 16)
              tmem_ld16(tmem_s + lane_off + grp * S::SW + pc * NS + col0 + c, sp + c);
#pragma unroll
            for (int c = 0; c < SVN; ++c) sv[c] += sp[c];
          }
        }
        tc_fence_before();
        mbar_arrive(bar(Bx::SFREE + grp));

        float s[G];
        const bool second = rh * G != col0;                   // this row's head is the 2nd loaded
        float* rb = red + par * 8 * S::GP;
        bool exceed = false;                                  // a score passed its reference
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float raw = (RB < 32 && second) ? sv[(RB < 32 ? G : 0) + g] : sv[g];
          s[g] = valid ? raw * (QCNV ? qcs[g] : a.scale_log2) : -CUDART_INF_F;
          exceed |= s[g] > mo[g] + kRescaleLog2;
        }
        // The references (uniform per query head over the group): the unit's first
        // tile sets them to its maxima, a reduction over the group; a later tile
        // only votes on whether some score passed its reference by 2^64, and
        // reduces (then rescales) only in that rare case.
        const bool reduce = wg_vote_or(failed || first || exceed, grp);
        if (reduce && wg_vote_or(failed, grp)) { stop = true; break; }
        float tm[G], ao[G];
#pragma unroll
        for (int g = 0; g < G; ++g) { tm[g] = -CUDART_INF_F; ao[g] = 1.f; }
        if (reduce) {
#pragma unroll
          for (int g = 0; g < G; ++g) {
            float v = s[g];
#pragma unroll
            for (int o = RB / 2; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
            if (rr == 0) rb[(rq * kHG + rh) * S::GP + g] = v;
          }
          wg_sync(grp);
#pragma unroll
          for (int g = 0; g < G; ++g) {
#pragma unroll
            for (int q = 0; q < NQ; ++q) tm[g] = fmaxf(tm[g], rb[(q * kHG + rh) * S::GP + g]);
            if (first) mo[g] = tm[g];
          }
        }
        if (!first && reduce) {
          // rare: O holds earlier tiles' products; publish old and new references,
          // wait for the last product, rescale the moved columns in TMEM
          if (rq == 0 && rr == 0) {
#pragma unroll
            for (int g = 0; g < G; ++g) {
              mold[rh * G + g] = mo[g];
              mnew[rh * G + g] = tm[g] > mo[g] + kRescaleLog2 ? tm[g] : mo[g];
            }
          }
          wg_sync(grp);
          wait_pv(tc - 2);
          tc_fence_after();
#pragma unroll
          for (int h = 0; h < kHG; ++h) {
#pragma unroll
            for (int c = 0; c < NOH; c += 16) {
              float o[16];
              const uint32_t ta = obuf(i, grp) + lane_off + h * NOH + c;
              tmem_ld16(ta, o);
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const int cc = c + e;             // hi columns [0, G), lo columns [G, 2G)
                if (cc >= 2 * G) continue;
                const int n = h * G + (cc < G ? cc : cc - G);
                if (mnew[n] != mold[n] && mold[n] != -CUDART_INF_F) o[e] *= exp2f(mold[n] - mnew[n]);
              }
              tmem_st16(ta, o);
            }
          }
          tc_fence_before();
#pragma unroll
          for (int g = 0; g < G; ++g) {
            if (tm[g] > mo[g] + kRescaleLog2) {
              ao[g] = mo[g] == -CUDART_INF_F ? 1.f : exp2f(mo[g] - tm[g]);
              mo[g] = tm[g];
            }
          }
          wg_sync(grp);                           // mold / mnew may be rewritten next tile
        }
        // this group's P buffer (and, with FP8 pools, its V buffer) was last read
        // by the output product of its previous tile: the issuer put S(tc) after
        // it on the in-order tensor pipe, so seeing S(tc) means it is complete
        // (the wait below then returns at once; it keeps the order explicit)
        if (tc >= 2) wait_pv(tc - 2);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float p = valid ? exp2f(s[g] - mo[g]) : 0.f;
          l[g] = fmaf(l[g], ao[g], p);
          uint16_t hi, lo;
          split_16<CF>(p, hi, lo);
          *reinterpret_cast<uint16_t*>(prow + g * 128 + ((pchunk ^ (g & 7)) << 4) + pbyte) = hi;
          *reinterpret_cast<uint16_t*>(prow + (G + g) * 128 + ((pchunk ^ ((G + g) & 7)) << 4) + pbyte) = lo;
        }
        if (!KV8 && in_range && !valid) {
          // this V row enters the output product with weight 0: it must hold finite values
          const int seq = 2 * tc + 1, sv_ = seq % NST;
          if (!mbar_wait(bar(Bx::FULL + sv_), (seq / NST) & 1, abort_flag, wait_ns)) failed = true;
          uint4* z0 = reinterpret_cast<uint4*>(smem + sv_ * S::kStage + row * 128);
          uint4* z1 = reinterpret_cast<uint4*>(smem + sv_ * S::kStage + kHalf + row * 128);
#pragma unroll
          for (int c = 0; c < 8; ++c) { z0[c] = make_uint4(0, 0, 0, 0); z1[c] = make_uint4(0, 0, 0, 0); }
        }
        if constexpr (KV8) {
          // V of this tile: its codes become the group's V buffer, widened to f16
          // (zeros for rows that must not count); the output product of the
          // group's previous tile, which read the buffer last, is complete (see
          // above). The code stage is free again once every row has been read.
          const int seq = 2 * tc + 1, s = seq % NST;
          if (!mbar_wait(bar(Bx::FULL + s), (seq / NST) & 1, abort_flag, wait_ns)) failed = true;
          if (in_range && !failed)
            widen_row_fp8_to<CF>(smem + s * S::kStage, smem + S::OFF_VOP + grp * kStageBytes, row,
                                 !valid);
          wg_sync(grp);
          if (row == 0) mbar_arrive(bar(Bx::EMPTY + s));
        }
        fence_proxy_async();                      // P (and the widened V) -> the tensor cores
        mbar_arrive(bar(Bx::PREADY + grp));
        my_last = tc;
      }
      if (stop) break;

      // ---- end of unit i: exp-sums per query head, then one group merges both accumulators
      float* rl = red_l + (i & 1) * 8 * S::GP;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float v = l[g];
#pragma unroll
        for (int o = RB / 2; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (rr == 0) rl[(rq * kHG + rh) * S::GP + g] = v;
      }
      if (wg_vote_or(failed, grp)) break;
      const int xi = i & 1, xpar = (i >> 1) & 1;
      float* xm = xbuf + xi * 2 * NS;
      float* xl = xm + NS;
      const int last_grp = (tc - 1) & 1;                    // group of the unit's last tile
      if (grp != last_grp) {
        if (my_last >= 0) wait_pv(my_last);
        if (!mbar_wait(bar(Bx::XFREE + xi), xpar ^ 1, abort_flag, wait_ns)) failed = true;
        if (row < NS) {
          float L = 0.f;
#pragma unroll
          for (int q = 0; q < NQ; ++q) L += rl[(q * kHG + row / G) * S::GP + row % G];
          xl[row] = L;
        }
        if (rq == 0 && rr == 0) {
#pragma unroll
          for (int g = 0; g < G; ++g) xm[rh * G + g] = mo[g];
        }
        if (row == 0) xflag[xi] = my_last >= 0 ? 1 : 0;
        tc_fence_before();
        mbar_arrive(bar(Bx::XFULL + xi));
      } else {
        wait_pv(my_last);
        if (!mbar_wait(bar(Bx::XFULL + xi), xpar, abort_flag, wait_ns)) failed = true;
        if (rq == 0 && rr == 0) {
#pragma unroll
          for (int g = 0; g < G; ++g) mown[rh * G + g] = mo[g];
        }
        if (row == 0) bulk_wait_read();           // the group's previous rows have left staging
        wg_sync(grp);
        const bool has_p = xflag[xi] != 0;
        // Where the unit's rows go: a whole pair to the output (normalised), or,
        // in the split-only pass, to its workspace slot; a piece to its CTA's
        // piece slot. The NS rows are contiguous in each.
        const bool piece = !x.whole;
        const bool final_out = !piece && !a.force_split;
        const int osz = final_out && a.out_dtype != PA_F32 ? 2 : 4;
        uint8_t* stg = smem + S::OFF_STG + grp * S::kStgBytes;
        const size_t out_row0 = (size_t)x.b * a.Hq + (size_t)x.h * NS;
        const size_t cas_row0 = ((size_t)x.b * a.P + a.slot_base) * a.Hq + (size_t)x.h * NS;
        const size_t piece_row0 = (2 * (size_t)cta + (x.g0 == r0 ? 0 : 1)) * NS;
        float* wm = piece ? a.sk_m : a.ws_m;
        float* wl = piece ? a.sk_l : a.ws_l;
        const size_t wrow0 = piece ? piece_row0 : cas_row0;
        float* coef = reinterpret_cast<float*>(smem + S::OFF_COEF) + grp * 2 * NS;
        if (row < NS) {
          // query head n: combined max and exp-sum, and the weights of the two
          // accumulators (divided by the exp-sum when this is the final output)
          const int n = row, h = n / G, g = n - h * G;
          float L = 0.f;
#pragma unroll
          for (int q = 0; q < NQ; ++q) L += rl[(q * kHG + h) * S::GP + g];
          const float mp = has_p ? xm[n] : -CUDART_INF_F;
          const float mine = mown[n];
          const float M = fmaxf(mine, mp);
          float c = 0.f, cp = 0.f;
          if (M != -CUDART_INF_F) {
            c = exp2f(mine - M);
            if (has_p) cp = exp2f(mp - M);
          }
          const float Lt = L * c + (has_p ? xl[n] * cp : 0.f);
          c *= a.v_scale;                       // 1 unless V holds FP8 codes
          cp *= a.v_scale;
          if (final_out) {
            const float inv = Lt > 0.f ? 1.f / Lt : 0.f;
            c *= inv;
            cp *= inv;
          } else {
            wm[wrow0 + n] = M;
            wl[wrow0 + n] = Lt;
          }
          coef[n] = c;
          coef[NS + n] = cp;
        }
        wg_sync(grp);
        tc_fence_after();
#pragma unroll 1
        for (int h = 0; h < kHG; ++h) {
          float own[16 > NOH ? 16 : NOH], part[16 > NOH ? 16 : NOH], w[G], wp[G];
#pragma unroll
          for (int c = 0; c < NOH; c += 16) {
            tmem_ld16(obuf(i, grp) + lane_off + h * NOH + c, own + c);
            tmem_ld16(obuf(i, 1 - grp) + lane_off + h * NOH + c, part + c);
          }
#pragma unroll
          for (int g = 0; g < G; g += 4) {
            *reinterpret_cast<float4*>(w + g) = *reinterpret_cast<const float4*>(coef + h * G + g);
            *reinterpret_cast<float4*>(wp + g) = *reinterpret_cast<const float4*>(coef + NS + h * G + g);
          }
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const int n = h * G + g;
            float v = (own[g] + own[G + g]) * w[g];
            if (has_p) v = fmaf(part[g] + part[G + g], wp[g], v);   // no partner: its TMEM is stale
            if (final_out) store_out(stg, (size_t)n * kD + row, v, a.out_dtype);
            else reinterpret_cast<float*>(stg)[n * kD + row] = v;
          }
        }
        tc_fence_before();
        mbar_arrive(bar(Bx::XFREE + xi));
        mbar_arrive(bar(Bx::ODONE + (i & 1)));
        fence_proxy_async();                      // staging writes -> the bulk copy's proxy
        wg_sync(grp);                             // (mown is rewritten at the next merge, too)
        const uint32_t hb = (uint32_t)(G * kD * osz);
        if (row == 0) {
          uint8_t* dst = final_out ? static_cast<uint8_t*>(a.out) + out_row0 * kD * osz
                       : piece     ? reinterpret_cast<uint8_t*>(a.sk_acc) + piece_row0 * kD * 4
                                   : reinterpret_cast<uint8_t*>(a.ws_acc) + cas_row0 * kD * 4;
#pragma unroll
          for (int h = 0; h < kHG; ++h) bulk_store(dst + h * hb, smem_addr(stg) + h * hb, hb);
          bulk_commit();
        }
        if (piece) {
          // publish the piece (its m, l stores and its bulk copy), then take a
          // ticket; the last piece of the pair merges all of them
          __threadfence();
          wg_sync(grp);
          if (row == 0) {
            bulk_wait_all();
            fence_proxy_async_global();
            __threadfence();
            const int np = pair_pieces(pair_shares(x.pair0, x.ntp, x.p, C, grid, a.pair_cost), C, grid);
            ms->last[grp] =
                take_ticket(a.tickets + (size_t)x.b * nhg + x.h, a.epoch, np, a.err_flag) ? 1 : 0;
          }
          wg_sync(grp);
          if (ms->last[grp]) {
            __threadfence();
            merge_pieces<G>(a, x, row, stg, C, grid, !a.force_split, cas_row0);
            fence_proxy_async();
            wg_sync(grp);
            if (row == 0) {
              const int osz2 = a.force_split || a.out_dtype == PA_F32 ? 4 : 2;
              const uint32_t hb2 = (uint32_t)(G * kD * osz2);
              uint8_t* dst = a.force_split ? reinterpret_cast<uint8_t*>(a.ws_acc) + cas_row0 * kD * 4
                                           : static_cast<uint8_t*>(a.out) + out_row0 * kD * osz2;
#pragma unroll
              for (int h = 0; h < kHG; ++h) bulk_store(dst + h * hb2, smem_addr(stg) + h * hb2, hb2);
              bulk_commit();
              // every piece has arrived: leave the ticket at zero for this epoch
              atomicExch(a.tickets + (size_t)x.b * nhg + x.h, a.epoch << kEpochShift);
            }
          }
        }
      }
    }
    if (row == 0) bulk_wait_all();               // no copy outlives the kernel
    if (failed) give_up();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(S::kTmemCols)
                 : "memory");
  }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

bool make_maps(const DecodeArgs& a, int dtype, bool kv8, int G, CUtensorMap* k, CUtensorMap* v,
               CUtensorMap* q) {
  auto enc = encode_fn();
  if (!enc || a.num_blocks <= 0) return false;
  const CUtensorMapDataType dt =
      dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const int rb = a.bs < kRt ? a.bs : kRt;
  for (int i = 0; i < 2; ++i) {
    CUresult r;
    void* pool = const_cast<void*>(i == 0 ? a.k_cache : a.v_cache);
    if (kv8) {
      // FP8 pool [num_blocks][bs][Hkv][128 codes]: a box of RB rows x kHG heads
      // lands head-major, one 128-byte line per row, 128-byte swizzled
      const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)a.bs, (cuuint64_t)a.Hkv,
                                  (cuuint64_t)a.num_blocks};
      const cuuint64_t strides[3] = {(cuuint64_t)a.Hkv * kD, (cuuint64_t)kD,
                                     (cuuint64_t)a.bs * a.Hkv * kD};
      const cuuint32_t box[4] = {(cuuint32_t)kD, (cuuint32_t)rb, (cuuint32_t)kHG, 1};
      const cuuint32_t es[4] = {1, 1, 1, 1};
      r = enc(i == 0 ? k : v, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, pool, dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    } else {
      // the pool [num_blocks][bs][Hkv][D] seen as [num_blocks][2][Hkv][bs][64]: a box of
      // RB rows x kHG heads x 64 d lands head-major, 128 B per row, 128-byte swizzled
      const cuuint64_t dims[5] = {64, (cuuint64_t)a.bs, (cuuint64_t)a.Hkv, 2,
                                  (cuuint64_t)a.num_blocks};
      const cuuint64_t strides[4] = {(cuuint64_t)a.Hkv * kD * 2, (cuuint64_t)kD * 2, 128,
                                     (cuuint64_t)a.bs * a.Hkv * kD * 2};
      const cuuint32_t box[5] = {64, (cuuint32_t)rb, (cuuint32_t)kHG, 1, 1};
      const cuuint32_t es[5] = {1, 1, 1, 1, 1};
      r = enc(i == 0 ? k : v, dt, 5, pool, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    }
    if (r != CUDA_SUCCESS) return false;
  }
  const cuuint64_t qdims[2] = {(cuuint64_t)kD, (cuuint64_t)a.B * a.Hq};
  const cuuint64_t qstr[1] = {(cuuint64_t)kD * 2};
  const cuuint32_t qbox[2] = {64, (cuuint32_t)(kHG * G)};
  const cuuint32_t qes[2] = {1, 1};
  return enc(q, dt, 2, const_cast<void*>(a.q), qdims, qstr, qbox, qes,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Upper bound of the tiles of a call (every sequence at max_context_len).
long long max_tiles(const DecodeArgs& a) {
  const long long per = ((long long)(a.max_context_len > 0 ? a.max_context_len : 1) + kRt - 1) / kRt;
  return (long long)a.B * (a.Hkv / kHG) * per;
}

template <int FMT, int BS, int G, bool KV8>
int launch_tc_t(const DecodeArgs& a, const CUtensorMap& k, const CUtensorMap& v,
                const CUtensorMap& q, cudaStream_t stream) {
  auto kern = decode_tc_kernel<FMT, BS, G, KV8>;
  constexpr int smem = TcShape<G, KV8>::SMEM;
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return PA_ERR_CUDA;
    attr = true;
  }
  // one CTA per SM (at most one per tile): the workspace's piece slots are sized for that
  const long long tiles = max_tiles(a);
  const long long grid = tiles < sm_count_cached() ? tiles : sm_count_cached();
  if (grid <= 0) return PA_OK;
  return launch_k(kern, dim3((unsigned)grid), dim3(kThreads), smem, stream, a, k, v, q) ==
                 cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

template <int FMT, int BS, bool KV8>
int launch_tc_g(const DecodeArgs& a, const CUtensorMap& k, const CUtensorMap& v,
                const CUtensorMap& q, cudaStream_t stream) {
  switch (a.Hq / a.Hkv) {
    case 4: return launch_tc_t<FMT, BS, 4, KV8>(a, k, v, q, stream);
    case 8: return launch_tc_t<FMT, BS, 8, KV8>(a, k, v, q, stream);
  }
  return PA_ERR_UNSUPPORTED;
}

template <bool KV8>
int launch_tc_all(const DecodeArgs& a, int dtype, const CUtensorMap& k, const CUtensorMap& v,
                  const CUtensorMap& q, cudaStream_t stream) {
  if (dtype == PA_BF16)
    return a.bs == 16 ? launch_tc_g<1, 16, KV8>(a, k, v, q, stream)
                      : launch_tc_g<1, 32, KV8>(a, k, v, q, stream);
  return a.bs == 16 ? launch_tc_g<0, 16, KV8>(a, k, v, q, stream)
                    : launch_tc_g<0, 32, KV8>(a, k, v, q, stream);
}

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

bool tc_shape(int Hq, int Hkv, int D) {
  if (D != kD || Hkv <= 0 || Hq % Hkv || Hkv % kHG) return false;
  const int G = Hq / Hkv;
  return G == 4 || G == 8;
}

bool tc_supported(int dtype, int Hq, int Hkv, int D, int bs) {
  // 16-bit pools, or FP8 pools (with a 16-bit query: the caller checks that)
  if (dtype != PA_F16 && dtype != PA_BF16 && dtype != PA_FP8_E4M3) return false;
  return (bs == 16 || bs == 32) && tc_shape(Hq, Hkv, D);
}

// Piece slots for every CTA of the largest grid, then one ticket word per pair.
size_t tc_workspace_bytes(int B, int Hq, int Hkv, int D) {
  if (B <= 0 || !tc_shape(Hq, Hkv, D)) return 0;
  const size_t ns = (size_t)kHG * (Hq / Hkv);
  const size_t slots = 2 * (size_t)sm_count_cached();
  return up256(slots * ns * kD * 4) + 2 * up256(slots * ns * 4) +
         up256((size_t)B * (Hkv / kHG) * 8);
}

void tc_carve(DecodeArgs& a, char* base) {
  const size_t ns = (size_t)kHG * (a.Hq / a.Hkv);
  const size_t slots = 2 * (size_t)sm_count_cached();
  a.sk_acc = reinterpret_cast<float*>(base);
  base += up256(slots * ns * kD * 4);
  a.sk_m = reinterpret_cast<float*>(base);
  base += up256(slots * ns * 4);
  a.sk_l = reinterpret_cast<float*>(base);
  base += up256(slots * ns * 4);
  a.tickets = reinterpret_cast<unsigned long long*>(base);
}

int launch_decode_tc(const DecodeArgs& a, int dtype, bool kv8, cudaStream_t stream) {
  const int G = a.Hq / a.Hkv;
  CUtensorMap k, v, q;
  if (!make_maps(a, dtype, kv8, G, &k, &v, &q))
    return kv8 ? launch_decode_simt_kv(a, dtype, PA_FP8_E4M3, PA_FP8_E4M3, stream)
               : launch_decode_simt(a, dtype, stream);
  return kv8 ? launch_tc_all<true>(a, dtype, k, v, q, stream)
             : launch_tc_all<false>(a, dtype, k, v, q, stream);
}

}  // namespace pa
