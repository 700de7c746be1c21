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
// Work unit = (sequence, partition of the context, group of HG KV heads).
// Tile = 128 rows of K (or V): HG heads x Rt = 128 / HG tokens, taken from
// whole physical blocks. A 5-D TMA tensor map views the pool as
// [num_blocks][2 d-halves][Hkv][block_size][64 d] (strides of the real
// [num_blocks, block_size, Hkv, D] layout), so one TMA box brings Rb token
// rows of all HG heads for one 64-wide d-half: 8-16 KB per instruction, in the
// canonical 128-byte-swizzled layout the MMA reads (rows = (head, token),
// 128 B each; the two d-halves 16 KB apart). Bigger boxes matter: streaming
// the same bytes as 2-4 KB per-head boxes is limited by TMA issue, not HBM.
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
// CTA = 10 warps, persistent over its list of units:
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
// Every pipeline wait is bounded (1 s); a wait that gives up sets the
// PA_DEV_TIMEOUT bit, raises a CTA-wide abort flag, and all roles leave their
// loops (the softmax warps of a group only together, at a named-barrier vote),
// wait for their own asynchronous work, free tensor memory and return.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math_constants.h>

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
constexpr int kMaxUnits = 320;                  // work units one CTA can hold in its list
constexpr int kScanChunk = 1024;                // sequences scanned per pass (stage 0 as scratch)
constexpr float kRescaleLog2 = 64.f;            // lazy rescale threshold (log2 units): p <= 2^64,
                                                // far from fp32 overflow in l and O

template <int G> struct TcShape {
  static constexpr int NS = kHG * G;                         // N of the score MMA
  static constexpr int NOH = ((2 * G + 15) / 16) * 16;       // N of a head's output MMA
  static constexpr int NO = kHG * NOH;                       // output columns per group
  static constexpr int kStages = 5;
  static constexpr int kTmemCols = 512;                      // S x2, O x (2 units x 2 groups)
  static constexpr int kQBytes = 2 * NS * 128;               // Q operand: 2 d-halves x NS rows
  static constexpr int kPBytes = 2 * NOH * 128;              // P operand of one tile: 2 lines
  static constexpr int kStgBytes = NS * kD * 4;              // one group's merged rows (fp32)
  static constexpr int OFF_Q = kStages * kStageBytes;
  static constexpr int OFF_P = OFF_Q + 2 * kQBytes;
  static constexpr int OFF_STG = OFF_P + 2 * kPBytes;        // [2 groups] output staging
  static constexpr int OFF_X = OFF_STG + 2 * kStgBytes;      // [2][2][NS] reference max, exp-sum
  static constexpr int OFF_BAR = OFF_X + 2 * 2 * NS * 4 + 16;
  static constexpr int NBAR = 2 * kStages + 20;
  static constexpr int GP = G < 8 ? 8 : G;                  // per-chunk stride of the reductions
  static constexpr int OFF_RED = OFF_BAR + 8 * NBAR;         // [group][2][8 chunks][GP] maxima
  static constexpr int OFF_REDL = OFF_RED + 2 * 2 * 8 * GP * 4;   // [group][2][8][GP] sums
  static constexpr int OFF_MREF = OFF_REDL + 2 * 2 * 8 * GP * 4;  // [group][3][NS] references
  static constexpr int OFF_COEF = OFF_MREF + 2 * 3 * NS * 4;   // [group][2][NS] merge weights
  static constexpr int OFF_REC = (OFF_COEF + 2 * 2 * NS * 4 + 15) / 16 * 16;
  static constexpr int OFF_MISC = OFF_REC + kMaxUnits * 16;
  static constexpr int BYTES = OFF_MISC + 32;
  static constexpr int SMEM = BYTES + 1024;                  // + alignment slack
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
  static_assert(2 * NS + 4 * NO <= kTmemCols, "tensor memory columns");
  static_assert(OFF_STG % 128 == 0, "bulk-copy source alignment");
  static_assert(OFF_COEF % 16 == 0, "vector loads of the merge weights");
};

// barrier indices (the ring's full/empty pairs come first)
template <int NST> struct Bars {
  static constexpr int FULL = 0, EMPTY = NST, QFULL = 2 * NST, QEMPTY = QFULL + 2,
                       SFULL = QEMPTY + 2, SFREE = SFULL + 2, PREADY = SFREE + 2,
                       OFULL = PREADY + 2, XFULL = OFULL + 2, XFREE = XFULL + 2,
                       ODONE = XFREE + 2, DONE = ODONE + 2;
};

// ---------------------------------------------------------------- work units
// A unit is (sequence b, partition j, group h of kHG KV heads). Units exist
// only for partitions that hold tokens. Units are spread over the CTAs like
// longest-first list scheduling: they are ranked by size class (16 classes of
// tile count, whole partitions first), and rank r goes to round r / grid of a
// zig-zag over the CTAs (even rounds CTA 0, 1, ..., odd rounds backwards), so
// every CTA gets its big units first and the small ones even out the end.
// Every CTA builds its own list at start, in shared memory, so the roles never
// touch global memory to find their next unit.
struct __align__(16) URec {
  int b, hj, ctx, start;      // hj = KV-head group | partition << 16; start = first token of the pass
};

struct Unit {
  int b, h, j, ctx, t0, t1, ntiles, nparts;
};

__device__ __forceinline__ Unit unit_from(const URec& r, int psize) {
  Unit x;
  x.b = r.b; x.h = r.hj & 0xffff; x.j = r.hj >> 16; x.ctx = r.ctx;
  x.t0 = r.start + x.j * psize;
  x.t1 = min(r.ctx, x.t0 + psize);
  x.ntiles = (x.t1 - x.t0 + kRt - 1) / kRt;
  x.nparts = (r.ctx - r.start + psize - 1) / psize;
  return x;
}

// Build this CTA's unit list (128 threads of warps 0-3, stage 0 as scratch).
// Sequences with no tokens (or a context length the table cannot hold) get no
// units; their output rows are zeroed here by CTA b % grid. Thread t of a pass
// over kScanChunk sequences owns sequences t, t + 128, ... of the chunk, and
// ranks within a class follow (pass, thread, sequence) order. Every loop here
// is short and independent across threads: this runs before any K/V moves.
template <int BS>
__device__ void build_unit_list(const DecodeArgs& a, int nhg, uint8_t* scratch, URec* recs,
                                int* my_units) {
  constexpr int NC = 16;                                  // size classes
  constexpr int PER = kScanChunk / 128;                   // sequences per thread and pass
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int grid = (int)gridDim.x, cta = (int)blockIdx.x;
  int* ctx_s = reinterpret_cast<int*>(scratch);           // [kScanChunk]
  int* start_s = ctx_s + kScanChunk;                      // [kScanChunk] first token of the pass
  int* next_s = start_s + kScanChunk;                     // [NC][128] next rank per class
  int* hist = next_s + NC * 128;                          // [NC] units per class
  int* cbase = hist + NC;                                 // [NC] first rank of each class
  int* carry = cbase + NC;                                // [NC] ranks used by earlier passes
  int* wsum = carry + NC;                                 // [4][NC]
  int* nempty = wsum + 4 * NC;                            // sequences to zero in this pass
  int* empty_s = nempty + 4;                              // [kScanChunk]
  const int TP = (a.psize + kRt - 1) / kRt;               // tiles of a whole partition
  // a context length (or pass start) the table cannot hold
  auto bad = [&](int ctx, int start) {
    return ctx < 0 || ctx > a.max_blocks * BS || ctx > a.max_context_len || start < 0 ||
           start > ctx;
  };
  // partitions of the pass [start, ctx) and tiles of its last one; false: no units
  auto shape = [&](int ctx, int start, int& np, int& tl) -> bool {
    if (bad(ctx, start) || ctx == start) return false;
    np = (ctx - start + a.psize - 1) / a.psize;
    tl = (ctx - start - (np - 1) * a.psize + kRt - 1) / kRt;
    return true;
  };
  auto start_of = [&](int b) { return a.start_blocks ? __ldg(a.start_blocks + b) * BS : 0; };
  auto cls = [&](int nt) { return min(NC - 1, (nt * NC + TP - 1) / TP - 1); };
  auto bar = [] { asm volatile("bar.sync 1, 128;" ::: "memory"); };

  if (tid < NC) { hist[tid] = 0; carry[tid] = 0; }
  bar();
  for (int b = tid; b < a.B; b += 128) {
    int np, tl;
    if (!shape(__ldg(a.context_lens + b), start_of(b), np, tl)) continue;
    if (np > 1) atomicAdd(&hist[NC - 1], (np - 1) * nhg);
    atomicAdd(&hist[cls(tl)], nhg);
  }
  bar();
  if (tid == 0) {
    int r = 0;
    for (int q = NC - 1; q >= 0; --q) { cbase[q] = r; r += hist[q]; }
    const int full = r / grid, rem = r - full * grid;
    const bool extra = rem > 0 && ((full & 1) ? cta >= grid - rem : cta < rem);
    *my_units = min(full + (extra ? 1 : 0), kMaxUnits);
  }
  for (int b0 = 0; b0 < a.B; b0 += kScanChunk) {
    const int n = min(kScanChunk, a.B - b0);
    if (tid == 0) *nempty = 0;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      const int i = e * 128 + tid;
      ctx_s[i] = i < n ? __ldg(a.context_lens + b0 + i) : 0;
      start_s[i] = i < n ? start_of(b0 + i) : 0;
    }
    bar();
    // units per class of this thread's sequences, then a block-wide scan per class
    int v[NC];
#pragma unroll
    for (int q = 0; q < NC; ++q) v[q] = 0;
    for (int e = 0; e < PER; ++e) {
      int np, tl;
      const int i = e * 128 + tid;
      if (!shape(ctx_s[i], start_s[i], np, tl)) {
        if (i < n && ((b0 + i) % grid) == cta) empty_s[atomicAdd(nempty, 1)] = i;
        continue;
      }
      const int c = cls(tl);
#pragma unroll
      for (int q = 0; q < NC; ++q) v[q] += (q == NC - 1 ? (np - 1) * nhg : 0) + (q == c ? nhg : 0);
    }
    int incl[NC];
#pragma unroll
    for (int q = 0; q < NC; ++q) {
      incl[q] = v[q];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl[q], o);
        if (lane >= o) incl[q] += t;
      }
      if (lane == 31) wsum[warp * NC + q] = incl[q];
    }
    bar();
#pragma unroll
    for (int q = 0; q < NC; ++q) {
      int wpre = 0;
      for (int w = 0; w < warp; ++w) wpre += wsum[w * NC + q];
      next_s[q * 128 + tid] = cbase[q] + carry[q] + wpre + incl[q] - v[q];
    }
    bar();
    if (tid < NC) carry[tid] += wsum[tid] + wsum[NC + tid] + wsum[2 * NC + tid] + wsum[3 * NC + tid];
    // walk the units in the order they were counted; keep the ones that land here
    for (int e = 0; e < PER; ++e) {
      const int li = e * 128 + tid;
      int np, tl;
      if (!shape(ctx_s[li], start_s[li], np, tl)) continue;
      if (np > 1) {
        // whole partitions: consecutive ranks r0 .. r0 + nf - 1 (unit j * nhg + h);
        // visit only the rounds they span and this CTA's slot in each
        int* nx = next_s + (NC - 1) * 128 + tid;
        const int r0 = *nx, nf = (np - 1) * nhg;
        *nx = r0 + nf;
        for (int round = r0 / grid; round * grid < r0 + nf && round < kMaxUnits; ++round) {
          const int r = round * grid + ((round & 1) ? grid - 1 - cta : cta);
          if (r < r0 || r >= r0 + nf) continue;
          recs[round] = URec{b0 + li, ((r - r0) % nhg) | (((r - r0) / nhg) << 16), ctx_s[li],
                             start_s[li]};
        }
      }
      int* nx = next_s + cls(tl) * 128 + tid;               // the last partition
      for (int h = 0; h < nhg; ++h) {
        const int r = (*nx)++;
        const int round = r / grid, pos = r - round * grid;
        const int owner = (round & 1) ? grid - 1 - pos : pos;
        if (owner == cta && round < kMaxUnits)
          recs[round] = URec{b0 + li, h | ((np - 1) << 16), ctx_s[li], start_s[li]};
      }
    }
    // zero the output rows of empty / bad sequences this CTA owns
    bar();
    for (int k = 0; k < *nempty; ++k) {
      const int li = empty_s[k], b = b0 + li;
      if (bad(ctx_s[li], start_s[li]) && tid == 0) flag_error(a.err_flag, PA_DEV_BAD_CTX);
      if (!a.force_split)                 // the split-only pass leaves every row to the merge
        for (int i = tid; i < a.Hq * kD; i += 128)
          store_out(a.out, (size_t)b * a.Hq * kD + i, 0.f, a.out_dtype);
    }
    bar();
  }
}

// Advance (i, k) to the next tile of the CTA's unit list (i == nu: past the end).
__device__ __forceinline__ void next_tile(const URec* recs, int nu, int psize, int& i, int& k) {
  if (i >= nu) return;
  const Unit x = unit_from(recs[i], psize);
  if (++k >= x.ntiles) { k = 0; ++i; }
}


template <int FMT, int BS, int G>
__global__ void __launch_bounds__(kThreads, 1)
decode_tc_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmQ) {
  using S = TcShape<G>;
  constexpr int NST = S::kStages;
  using Bx = Bars<NST>;
  constexpr int NS = S::NS, NOH = S::NOH, NO = S::NO;
  constexpr int RB = BS < kRt ? BS : kRt;        // token rows per TMA box (per head)
  constexpr int NQ = kRt / RB;                   // boxes per d-half per tile
  constexpr int KS = kRt / 16;                   // output-MMA K steps per head per tile
  constexpr int NCH = NQ * kHG;                  // (box, head) row chunks per tile
  constexpr uint32_t IDESC_S = make_idesc(FMT, 0, 0, NS, 128);
  constexpr uint32_t IDESC_O = make_idesc(FMT, 1, 0, NOH, 128);
  static_assert(NCH * RB == kRows && NCH <= 8, "tile geometry");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + S::OFF_BAR;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  const URec* recs = reinterpret_cast<const URec*>(smem + S::OFF_REC);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + S::OFF_MISC + 4);
  int* my_units_s = reinterpret_cast<int*>(smem + S::OFF_MISC + 8);
  const int nhg = a.Hkv / kHG;

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
    *abort_flag = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 8) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(S::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  pdl_wait();                            // global memory from here on
  if (warp < 4) {
    build_unit_list<BS>(a, nhg, smem, const_cast<URec*>(recs), my_units_s);
    fence_proxy_async();                 // stage 0 served as scratch; TMA writes it next
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_s = tmem;                 // S buffers: [0, NS) and [NS, 2NS)
  // O accumulators from column 2NS: [unit parity][group], NO columns each, so the
  // next unit accumulates while the previous one is merged
  const uint32_t tmem_o = tmem + 2 * NS;
  auto obuf = [&](int ui, int g) { return tmem_o + (uint32_t)((2 * (ui & 1) + g) * NO); };
  const int nu = *my_units_s;
  auto give_up = [&]() {
    *abort_flag = 1u;
    flag_error(a.err_flag, PA_DEV_TIMEOUT);
  };
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
      int phys_next[NQ];
      auto load_ids = [&](int i, int k, int* ph) {
        const Unit x = unit_from(recs[i], a.psize);
        int ts, te, nql;
        tile_span(x, k, ts, te, nql);
        const int32_t* table = a.block_tables + (size_t)x.b * a.max_blocks;
#pragma unroll
        for (int q = 0; q < NQ; ++q) ph[q] = q < nql ? __ldg(table + (ts + q * RB) / BS) : -1;
      };
      if (nu > 0) load_ids(0, 0, phys_next);
      for (int i = 0; i < nu; ++i) {
        const Unit x = unit_from(recs[i], a.psize);
        const int qi = i & 1;
        if (!mbar_wait(bar(Bx::QEMPTY + qi), ((i >> 1) & 1) ^ 1, abort_flag)) { give_up(); goto prod_done; }
        mbar_expect_tx(bar(Bx::QFULL + qi), 2u * NS * 128u);
        for (int hh = 0; hh < 2; ++hh)
          tma_load_2d(sbase + S::OFF_Q + qi * S::kQBytes + hh * (NS * 128), &tmQ, hh * 64,
                      x.b * a.Hq + x.h * kHG * G, bar(Bx::QFULL + qi));
        for (int k = 0; k < x.ntiles; ++k) {
          int ts, te, nql;
          tile_span(x, k, ts, te, nql);
          int phys[NQ];
          uint32_t bytes = 0;
#pragma unroll
          for (int q = 0; q < NQ; ++q) {
            phys[q] = phys_next[q];
            if (phys[q] >= 0 && phys[q] < a.num_blocks) bytes += 2u * RB * kHG * 128u;
          }
          if (k + 1 < x.ntiles) load_ids(i, k + 1, phys_next);
          else if (i + 1 < nu) load_ids(i + 1, 0, phys_next);
          for (int kv = 0; kv < 2; ++kv) {
            const int seq = 2 * tc + kv, s = seq % NST;
            if (!mbar_wait(bar(Bx::EMPTY + s), ((seq / NST) & 1) ^ 1, abort_flag)) { give_up(); goto prod_done; }
            mbar_expect_tx(bar(Bx::FULL + s), bytes);
            const uint32_t dst = sbase + s * kStageBytes;
#pragma unroll
            for (int q = 0; q < NQ; ++q) {
              if (phys[q] < 0 || phys[q] >= a.num_blocks) continue;
              const int r0 = (ts + q * RB) % BS;
              for (int hh = 0; hh < 2; ++hh)
                tma_load_5d(dst + hh * kHalf + q * (kHG * RB * 128), kv ? &tmV : &tmK, 0, r0,
                            x.h * kHG, hh, phys[q], bar(Bx::FULL + s));
            }
            ++issued;
          }
          ++tc;
        }
      }
    prod_done:
      // never leave with copies in flight: wait (bounded) for the last loads of every stage
      for (int seq = max(0, issued - NST); seq < issued; ++seq) {
        const int s = seq % NST;
        const uint64_t t0 = globaltimer();
        while (!mbar_try(bar(Bx::FULL + s), (seq / NST) & 1) && globaltimer() - t0 < kWaitNs) {}
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
        if (!mbar_wait(bar(Bx::PREADY + pb), (tt >> 1) & 1, abort_flag)) return false;
        const bool first = kk <= 1;                   // this group's first tile of the unit
        // the unit's accumulators were last used by unit ui - 2: wait for its merge
        if (first && ui >= 2 && !mbar_wait(bar(Bx::ODONE + (ui & 1)), ((ui - 2) >> 1) & 1, abort_flag))
          return false;
        const int seq = 2 * tt + 1, s = seq % NST;
        if (!mbar_wait(bar(Bx::FULL + s), (seq / NST) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t vst = sbase + s * kStageBytes;
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
        mma_commit(bar(Bx::EMPTY + s));
        mma_commit(bar(Bx::OFULL + pb));
        return true;
      };
      int pui = 0, pkk = 0, pnql = 0;                // the tile waiting for its output product
      bool pending = false;                          // tile tc - 1 still needs its output product
      for (int i = 0; i < nu && ok; ++i) {
        const Unit x = unit_from(recs[i], a.psize);
        const int qi = i & 1;
        if (!mbar_wait(bar(Bx::QFULL + qi), (i >> 1) & 1, abort_flag)) { ok = false; break; }
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
                  mbar_test(bar(Bx::FULL + s), (seq / NST) & 1))
                break;
              if (*abort_flag || globaltimer() - t0 > kWaitNs) { ok = false; break; }
            }
            if (!ok) break;
          }
          if (!mbar_wait(bar(Bx::SFREE + sb), ((tc >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
          if (!mbar_wait(bar(Bx::FULL + s), (seq / NST) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t kst = sbase + s * kStageBytes;
#pragma unroll
          for (int ks = 0; ks < kD / 16; ++ks) {
            const uint64_t ad = sw128_desc(kst + (ks >> 2) * kHalf + (ks & 3) * 32, 16, 1024);
            const uint64_t bd = sw128_desc(qst + (ks >> 2) * (NS * 128) + (ks & 3) * 32, 16, 1024);
            mma_f16(tmem_s + sb * NS, ad, bd, IDESC_S, ks > 0 ? 1u : 0u);
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
      if (!mbar_wait(bar(Bx::OFULL + grp), (t >> 1) & 1, abort_flag)) failed = true;
    };
    auto row_id = [&](int i, int k) -> int {
      const Unit x = unit_from(recs[i], a.psize);
      int ts, te, nql;
      tile_span(x, k, ts, te, nql);
      return rq < nql ? __ldg(a.block_tables + (size_t)x.b * a.max_blocks + (ts + rq * RB) / BS) : -1;
    };
    int ni = 0, nk = 0;
    if (nu > 0 && grp == 1) next_tile(recs, nu, a.psize, ni, nk);       // group 1 starts at tile 1
    int phys_next = (nu > 0 && ni < nu) ? row_id(ni, nk) : -1;
    bool stop = false;
    for (int i = 0; i < nu && !stop; ++i) {
      const Unit x = unit_from(recs[i], a.psize);
      float mo[G], l[G];                           // this row's head: reference max, exp-sum
#pragma unroll
      for (int g = 0; g < G; ++g) { mo[g] = -CUDART_INF_F; l[g] = 0.f; }
      int my_last = -1;
      for (int k = 0; k < x.ntiles; ++k, ++tc) {
        if ((tc & 1) != grp) continue;
        int ts, te, nql;
        tile_span(x, k, ts, te, nql);
        const bool in_range = rq < nql;
        const int phys = phys_next;
        next_tile(recs, nu, a.psize, ni, nk);                 // two tiles ahead: the next own tile
        next_tile(recs, nu, a.psize, ni, nk);
        if (ni < nu) phys_next = row_id(ni, nk);
        const bool blk_ok = phys >= 0 && phys < a.num_blocks;
        const bool valid = in_range && blk_ok && ts + tt_row < te;
        if (in_range && !blk_ok && rr == 0 && rh == 0) flag_error(a.err_flag, PA_DEV_BAD_BLOCK_ID);
        const bool first = my_last < 0;

        const int par = (tc >> 1) & 1;                        // use count of this group's buffers
        if (!mbar_wait(bar(Bx::SFULL + grp), par, abort_flag)) failed = true;
        tc_fence_after();
        constexpr int SVN = ((32 / RB) * G + 15) / 16 * 16;  // S columns this warp loads
        float sv[SVN];
#pragma unroll
        for (int c = 0; c < SVN; c += 16) tmem_ld16(tmem_s + lane_off + grp * NS + col0 + c, sv + c);
        tc_fence_before();
        mbar_arrive(bar(Bx::SFREE + grp));

        float s[G];
        const bool second = rh * G != col0;                   // this row's head is the 2nd loaded
        float* rb = red + par * 8 * S::GP;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float raw = (RB < 32 && second) ? sv[(RB < 32 ? G : 0) + g] : sv[g];
          s[g] = valid ? raw * a.scale_log2 : -CUDART_INF_F;
          float v = s[g];
#pragma unroll
          for (int o = RB / 2; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
          if (rr == 0) rb[(rq * kHG + rh) * S::GP + g] = v;
        }
        if (wg_vote_or(failed, grp)) { stop = true; break; }
        // this head's tile maxima; lazy update of the references (uniform per group)
        float tm[G], ao[G];
        bool exceed = false;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          tm[g] = -CUDART_INF_F;
#pragma unroll
          for (int q = 0; q < NQ; ++q) tm[g] = fmaxf(tm[g], rb[(q * kHG + rh) * S::GP + g]);
          ao[g] = 1.f;
          if (first) mo[g] = tm[g];
          else exceed |= tm[g] > mo[g] + kRescaleLog2;
        }
        if (!first && wg_vote_or(exceed, grp)) {
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
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float p = valid ? exp2f(s[g] - mo[g]) : 0.f;
          l[g] = fmaf(l[g], ao[g], p);
          uint16_t hi, lo;
          split_16<FMT>(p, hi, lo);
          *reinterpret_cast<uint16_t*>(prow + g * 128 + ((pchunk ^ (g & 7)) << 4) + pbyte) = hi;
          *reinterpret_cast<uint16_t*>(prow + (G + g) * 128 + ((pchunk ^ ((G + g) & 7)) << 4) + pbyte) = lo;
        }
        if (in_range && !valid) {
          // this V row enters the output product with weight 0: it must hold finite values
          const int seq = 2 * tc + 1, sv_ = seq % NST;
          if (!mbar_wait(bar(Bx::FULL + sv_), (seq / NST) & 1, abort_flag)) failed = true;
          uint4* r0 = reinterpret_cast<uint4*>(smem + sv_ * kStageBytes + row * 128);
          uint4* r1 = reinterpret_cast<uint4*>(smem + sv_ * kStageBytes + kHalf + row * 128);
#pragma unroll
          for (int c = 0; c < 8; ++c) { r0[c] = make_uint4(0, 0, 0, 0); r1[c] = make_uint4(0, 0, 0, 0); }
        }
        fence_proxy_async();
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
        if (!mbar_wait(bar(Bx::XFREE + xi), xpar ^ 1, abort_flag)) failed = true;
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
        if (!mbar_wait(bar(Bx::XFULL + xi), xpar, abort_flag)) failed = true;
        if (rq == 0 && rr == 0) {
#pragma unroll
          for (int g = 0; g < G; ++g) mown[rh * G + g] = mo[g];
        }
        if (row == 0) bulk_wait_read();           // the group's previous rows have left staging
        wg_sync(grp);
        const bool has_p = xflag[xi] != 0;
        // merged rows go to shared memory first, then out in one bulk copy per head:
        // the unit's NS output rows are contiguous in out [B, Hq, D] and in the
        // workspace [B, P, Hq, D]
        const bool final_out = x.nparts == 1 && !a.force_split;
        const int osz = final_out && a.out_dtype != PA_F32 ? 2 : 4;
        uint8_t* stg = smem + S::OFF_STG + grp * S::kStgBytes;
        const size_t row0 = final_out ? (size_t)x.b * a.Hq + (size_t)x.h * NS
                                      : ((size_t)x.b * a.P + a.slot_base + x.j) * a.Hq +
                                            (size_t)x.h * NS;
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
          if (final_out) {
            const float inv = Lt > 0.f ? 1.f / Lt : 0.f;
            c *= inv;
            cp *= inv;
          } else {
            a.ws_m[row0 + n] = M;
            a.ws_l[row0 + n] = Lt;
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
        if (row == 0) {
          uint8_t* dst = final_out ? static_cast<uint8_t*>(a.out) + row0 * kD * osz
                                   : reinterpret_cast<uint8_t*>(a.ws_acc) + row0 * kD * 4;
          const uint32_t hb = (uint32_t)(G * kD * osz);
#pragma unroll
          for (int h = 0; h < kHG; ++h) bulk_store(dst + h * hb, smem_addr(stg) + h * hb, hb);
          bulk_commit();
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

bool make_maps(const DecodeArgs& a, int dtype, int G, CUtensorMap* k, CUtensorMap* v,
               CUtensorMap* q) {
  auto enc = encode_fn();
  if (!enc || a.num_blocks <= 0) return false;
  const CUtensorMapDataType dt =
      dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  // the pool [num_blocks][bs][Hkv][D] seen as [num_blocks][2][Hkv][bs][64]: a box of
  // RB rows x kHG heads x 64 d lands head-major, 128 B per row, 128-byte swizzled
  const int rb = a.bs < kRt ? a.bs : kRt;
  const cuuint64_t dims[5] = {64, (cuuint64_t)a.bs, (cuuint64_t)a.Hkv, 2, (cuuint64_t)a.num_blocks};
  const cuuint64_t strides[4] = {(cuuint64_t)a.Hkv * kD * 2, (cuuint64_t)kD * 2, 128,
                                 (cuuint64_t)a.bs * a.Hkv * kD * 2};
  const cuuint32_t box[5] = {64, (cuuint32_t)rb, (cuuint32_t)kHG, 1, 1};
  const cuuint32_t es[5] = {1, 1, 1, 1, 1};
  for (int i = 0; i < 2; ++i) {
    CUresult r = enc(i == 0 ? k : v, dt, 5, const_cast<void*>(i == 0 ? a.k_cache : a.v_cache), dims,
                     strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
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

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return kSMs;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return kSMs;
  return n;
}

template <int FMT, int BS, int G>
int launch_tc_t(const DecodeArgs& a, const CUtensorMap& k, const CUtensorMap& v,
                const CUtensorMap& q, cudaStream_t stream) {
  auto kern = decode_tc_kernel<FMT, BS, G>;
  constexpr int smem = TcShape<G>::SMEM;
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return PA_ERR_CUDA;
    attr = true;
  }
  // Units that hold tokens number at most B * (Hkv / kHG) * P; a CTA's list holds kMaxUnits.
  const long long units = (long long)a.B * (a.Hkv / kHG) * a.P;
  if (units <= 0) return PA_OK;
  long long grid = units < sm_count() ? units : sm_count();
  if ((units + grid - 1) / grid > kMaxUnits) grid = (units + kMaxUnits - 1) / kMaxUnits;
  if (grid > 0x7fffffffLL) return PA_ERR_UNSUPPORTED;
  return launch_k(kern, dim3((unsigned)grid), dim3(kThreads), smem, stream, a, k, v, q) ==
                 cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

template <int FMT, int BS>
int launch_tc_g(const DecodeArgs& a, const CUtensorMap& k, const CUtensorMap& v,
                const CUtensorMap& q, cudaStream_t stream) {
  switch (a.Hq / a.Hkv) {
    case 4: return launch_tc_t<FMT, BS, 4>(a, k, v, q, stream);
    case 8: return launch_tc_t<FMT, BS, 8>(a, k, v, q, stream);
  }
  return PA_ERR_UNSUPPORTED;
}

}  // namespace

bool tc_supported(int dtype, int Hq, int Hkv, int D, int bs) {
  if (dtype != PA_F16 && dtype != PA_BF16) return false;
  if (D != kD || (bs != 16 && bs != 32) || Hkv <= 0 || Hq % Hkv || Hkv % kHG) return false;
  const int G = Hq / Hkv;
  return G == 4 || G == 8;
}

int launch_decode_tc(const DecodeArgs& a, int dtype, cudaStream_t stream) {
  const int G = a.Hq / a.Hkv;
  CUtensorMap k, v, q;
  if (!make_maps(a, dtype, G, &k, &v, &q)) return launch_decode_simt(a, dtype, stream);
  if (dtype == PA_BF16)
    return a.bs == 16 ? launch_tc_g<1, 16>(a, k, v, q, stream) : launch_tc_g<1, 32>(a, k, v, q, stream);
  return a.bs == 16 ? launch_tc_g<0, 16>(a, k, v, q, stream) : launch_tc_g<0, 32>(a, k, v, q, stream);
}

}  // namespace pa
