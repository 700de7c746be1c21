// prefill_tc.cu -- paged (chunked) prefill attention on the 5th-generation
// tensor cores with the query rows on the MMA's M.
//
// A chunk of a sequence's new query tokens attends, causally, to the
// sequence's cached tokens through its block table ("推理引擎内部机制——
// PagedAttention、连续批处理、分块预填充", chunked prefill: a long prompt is cut
// into chunks that run between decode steps). New token i of a chunk of n at
// the end of a context of ctx tokens sits at position ctx - n + i and attends
// positions 0 .. ctx - n + i.
//
// Work unit = (sequence b, chunk of TPU = 128 / G new tokens, KV head h).
// Its 128 query rows are (token t, query head g of the group of h), row
// r = t * G + g: one TMA box of the query [T][Hq][128] brings them in that
// order. Tile = 128 keys of head h: one TMA box per physical block and 64-wide
// d-half, 128-byte swizzled (block-sized boxes; a head's rows of a block are
// contiguous, the heads of a block are not). Per tile:
//   S[128 rows x 128 keys]  = Q . K_tile^T          (tensor memory, fp32)
//   O[128 rows x 128 d]    += P_hi . V_tile + P_lo . V_tile
// where the weights P (in tensor memory, written over S) enter as two 16-bit
// parts, p = hi + lo, hi = RN(p), lo = RN(p - hi) (~16 significant bits, as
// in the decode kernels), and the A operand of the output products is read
// from tensor memory: each 32-key chunk of S becomes 16 columns of hi parts
// followed by 16 columns of lo parts (two keys per 32-bit column).
//
// Two softmax groups share a unit's 128 query rows: thread (group hf, row r)
// owns row r's keys [64 hf, 64 hf + 64) of every tile and O's columns [64 hf,
// 64 hf + 64), so a row needs only its two threads to agree: they exchange the
// tile's row maximum (and, at the unit's end, their parts of the row sum)
// through shared memory. A thread reads its scores twice, 32 columns at a
// time: once for the maximum, once for the weights, which it writes over the
// chunk it has just read. (Holding all of a row's scores in registers made the
// loop body four times longer; a per-key mask branch inside the loops cost
// more than the rest of the tile's softmax: the mask is one bit per key of a
// 32-key chunk, and whole chunks take a loop without it.) The reference
// maximum of a row is its first tile's maximum
// and moves only when a later tile exceeds it by 2^64 (then the row's O is
// rescaled in tensor memory, each half by its thread); references are
// floored at -FLT_MAX so masked scores (-inf) give weight 0 without a guard.
// Keys past a row's position are masked; the V rows of keys that no row of
// the unit attends (past its last position, or in a block with a bad id) are
// zeroed in shared memory before the output product, so they add exact zeros.
//
// CTA = 10 warps, persistent over rounds of units taken in alternating
// directions (fa_unit_of_cta; the chunks late in their sequences, which
// attend the most keys, come first):
//   warps 0-7  softmax and epilogue, two groups (thread = query row = TMEM
//              lane; warps w and w + 4 reach the same lanes);
//   warp 8     TMA producer: the unit's query (double-buffered by unit), the
//              K and V tiles through a ring of 32 KB stages (its lanes issue
//              the copies of a tile's blocks together);
//   warp 9     MMA issuer and owner of the tensor memory: S(t), then the
//              output product of tile t - 1 (S is double-buffered by tile, O
//              by unit, so a unit's epilogue overlaps the next unit's tiles).
// Every pipeline wait is bounded (1 s); one that gives up sets PA_DEV_TIMEOUT,
// raises the CTA's abort flag, and every role drains its asynchronous work,
// frees tensor memory and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math_constants.h>

#include <cfloat>
#include <cstdlib>

#include "pa_internal.h"
#include "tc_ptx.cuh"

namespace pa {

namespace {

using namespace tc;

constexpr int kD = 128;
constexpr int kM = 128;                         // query rows per unit (the MMA's M)
constexpr int kTile = 128;                      // keys per tile
constexpr int kHalf = 128 * 128;                // one 64-wide d-half of a 128-row operand
constexpr int kOp = 2 * kHalf;                  // one 128 x 128 16-bit operand: 32 KB
constexpr int kNST = 5;                         // K / V ring stages (odd: a stage serves K and V in turn)
constexpr int kThreads = 320;                   // two softmax groups, producer, MMA
constexpr int kProdWarp = 8, kMmaWarp = 9;
constexpr float kRescaleLog2 = 64.f;

constexpr int OFF_Q = 0;                        // [2 units][32 KB]
constexpr int OFF_KV = 2 * kOp;                 // [kNST][32 KB]
constexpr int OFF_BAR = OFF_KV + kNST * kOp;
enum { B_FULL = 0, B_EMPTY = kNST, B_QFULL = 2 * kNST, B_QEMPTY = B_QFULL + 2,
       B_SFULL = B_QEMPTY + 2, B_PREADY = B_SFULL + 2, B_OSTEP = B_PREADY + 2,
       B_ODONE = B_OSTEP + 2, B_DONE = B_ODONE + 2, B_CONV = B_DONE + 1,
       B_COUNT = B_CONV + kNST };
constexpr int OFF_MISC = OFF_BAR + 8 * B_COUNT;
constexpr int OFF_XCH = OFF_MISC + 16;          // [2 groups][128 rows]: row maxima, then row sums
constexpr int kSmem = OFF_XCH + 2 * 128 * 4 + 1024;   // + alignment slack
static_assert(kSmem <= 227 * 1024, "shared memory per CTA");
constexpr int kTmemCols = 512;                  // S/P x2 (by tile), O x2 (by unit)

struct FaArgs {
  void* out;
  int out_dtype;
  const int32_t* block_tables;
  int max_blocks;
  const int32_t* context_lens;
  const int32_t* query_start;
  int B, Hq, Hkv, bs, num_blocks, chunks;
  float scale_log2;
  float v_scale;        // value of one V unit (FP8 V pool; 1 otherwise)
  int max_context_len;
  uint32_t* err_flag;
};

struct FUnit {
  int b, c, h;
  int qrow0;            // first query row (token) of the chunk in [T]
  int ntok;             // new tokens of the chunk (0: nothing to do)
  int pos0;             // position of the chunk's first token
  int t1;               // keys [0, t1) are attended by some row
  int ntiles;
  bool bad;             // the sequence's lengths are inconsistent
};

template <int G>
__device__ __forceinline__ FUnit fa_unit(const FaArgs& a, long long u) {
  constexpr int TPU = kM / G;
  FUnit x;
  x.h = (int)(u % a.Hkv);
  const long long t = u / a.Hkv;
  x.b = (int)(t % a.B);
  x.c = a.chunks - 1 - (int)(t / a.B);
  const int qs = __ldg(a.query_start + x.b), qe = __ldg(a.query_start + x.b + 1);
  const int n = qe - qs, ctx = __ldg(a.context_lens + x.b);
  x.bad = n < 0 || ctx < n || ctx > a.max_blocks * a.bs || ctx > a.max_context_len;
  x.ntok = x.bad ? 0 : max(0, min(TPU, n - x.c * TPU));
  x.qrow0 = qs + x.c * TPU;
  x.pos0 = ctx - n + x.c * TPU;
  x.t1 = x.ntok > 0 ? x.pos0 + x.ntok : 0;
  x.ntiles = (x.t1 + kTile - 1) / kTile;
  return x;
}

// The k-th unit of CTA cta: rounds of grid units, taken in alternating
// directions (CTA c gets unit c of even rounds and unit grid - 1 - c of odd
// ones). Units come longest first, so plain round-robin would hand CTA 0 the
// largest unit of every round.
__device__ __forceinline__ long long fa_unit_of_cta(long long k, int cta, int grid) {
  return k * grid + ((k & 1) ? grid - 1 - cta : cta);
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two fp32 weights -> packed 16-bit hi parts and lo parts (element 0 in the low half).
template <int FMT>
__device__ __forceinline__ void split2(float p0, float p1, uint32_t& hi, uint32_t& lo) {
  if (FMT == 1) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(p0 - hf.x, p1 - hf.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&l);
  } else {
    const __half2 h = __floats2half2_rn(p0, p1);
    const float2 hf = __half22float2(h);
    const __half2 l = __floats2half2_rn(p0 - hf.x, p1 - hf.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&l);
  }
}

// K8 / V8: that pool holds FP8 E4M3 codes. TMA brings a tile's codes (one
// 128-byte line per row, at the stage's upper half) and the softmax thread
// that owns the tile row widens it in place to the query's 16-bit type
// (exact) before the tile is released to the tensor cores. A unit's first
// tile is widened before its scores; each later tile right after the weights
// of the tile before it are handed over, beside that tile's output product.
template <int FMT, int BS, int G, bool K8, bool V8>
__global__ void __launch_bounds__(kThreads, 1)
prefill_fa_kernel(const FaArgs a, const __grid_constant__ CUtensorMap tmQ,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV) {
  constexpr int NB_T = kTile / BS;               // physical blocks per tile
  constexpr uint32_t kBlkBits = (uint32_t)((1ull << BS) - 1ull);   // one block's keys in a chunk mask
  constexpr uint32_t IDESC_S = make_idesc(FMT, 0, 0, kTile, kM);
  constexpr uint32_t IDESC_O = make_idesc(FMT, 0, 1, kD, kM);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_addr(smem);
  auto bar = [&](int i) { return sbase + OFF_BAR + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long U = (long long)a.B * a.chunks * a.Hkv;
  pdl_trigger();

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNST; ++s) {
      mbar_init(bar(B_FULL + s), 1);
      mbar_init(bar(B_EMPTY + s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(B_QFULL + i), 1);
      mbar_init(bar(B_QEMPTY + i), 1);
      mbar_init(bar(B_SFULL + i), 1);
      mbar_init(bar(B_PREADY + i), 256);
      mbar_init(bar(B_OSTEP + i), 1);
      mbar_init(bar(B_ODONE + i), 256);
    }
    mbar_init(bar(B_DONE), 1);
    for (int s = 0; s < kNST; ++s) mbar_init(bar(B_CONV + s), 128);
    *abort_flag = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  pdl_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_s = tmem;                  // S/P: [0, 128), [128, 256)
  const uint32_t tmem_o = tmem + 2 * kTile;      // O: [256, 384), [384, 512)
  auto give_up = [&]() {
    *abort_flag = 1u;
    flag_error(a.err_flag, PA_DEV_TIMEOUT);
  };
  // a stage holding K (kv = 0) or V (kv = 1) is ready for the tensor cores when
  // TMA filled it (16-bit pool) or when the softmax group widened it (FP8 pool)
  auto ready_bar = [&](int kv, int s) {
    return bar(((kv ? V8 : K8) ? B_CONV : B_FULL) + s);
  };
  // Phase parity of ring position seq on its ready barrier. FULL completes a
  // phase on every use of the stage, and so does CONV when both pools hold
  // codes. With one FP8 pool only its uses are widened: the ring has an odd
  // number of stages, so a stage's uses alternate K and V, and use u = seq /
  // kNST of a stage is the (u / 2)-th of its kind.
  static_assert(kNST % 2 == 1, "uses of a stage alternate K and V");
  auto ready_parity = [&](int kv, int seq) -> uint32_t {
    const int u = seq / kNST;
    return (uint32_t)(((kv ? V8 : K8) && K8 != V8) ? u >> 1 : u) & 1u;
  };

  if (warp == kProdWarp) {
    // ------------------------------------------------------------ producer
    // The warp's lanes share a tile's copies: lane q < NB_T issues those of the
    // tile's q-th block (one instruction starts them all, instead of one
    // thread issuing 16-32 in a row) and reads that block's id a tile ahead;
    // lane 0 waits for free stages, sets the expected bytes and loads the query.
    int tc_ = 0, issued = 0, ui = 0;
    int q_last[2] = {-1, -1};
    bool stop = false;
    for (long long kk = 0; !stop; ++kk) {
      const long long u = fa_unit_of_cta(kk, blockIdx.x, gridDim.x);
      if (u >= U) break;
      const FUnit x = fa_unit<G>(a, u);
      if (lane == 0 && x.bad && x.c == 0 && x.h == 0) flag_error(a.err_flag, PA_DEV_BAD_CTX);
      if (x.ntok <= 0) continue;
      const int qi = ui & 1;
      bool ok = true;
      if (lane == 0) {
        ok = mbar_wait(bar(B_QEMPTY + qi), ((ui >> 1) & 1) ^ 1, abort_flag);
        if (ok) {
          mbar_expect_tx(bar(B_QFULL + qi), (uint32_t)kOp);
          for (int hh = 0; hh < 2; ++hh)
            tma_load_4d(sbase + OFF_Q + qi * kOp + hh * kHalf, &tmQ, 0, hh, x.h * G, x.qrow0,
                        bar(B_QFULL + qi));
          q_last[qi] = ui;
        }
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) { stop = true; break; }
      const int32_t* table = a.block_tables + (size_t)x.b * a.max_blocks;
      // this lane's block of tile k (-1 for none)
      auto fetch = [&](int k) -> int {
        const int ts = k * kTile;
        const int nblk = (min(x.t1, ts + kTile) - ts + BS - 1) / BS;
        return lane < nblk ? __ldg(table + ts / BS + lane) : -1;
      };
      int ahead = fetch(0);
      for (int k = 0; k < x.ntiles && !stop; ++k, ++tc_) {
        const int ts = k * kTile;
        const int nblk = (min(x.t1, ts + kTile) - ts + BS - 1) / BS;
        int phys = ahead;
        if (k + 1 < x.ntiles) ahead = fetch(k + 1);     // latency overlaps this tile's copies
        if (lane < nblk && (phys < 0 || phys >= a.num_blocks)) {
          flag_error(a.err_flag, PA_DEV_BAD_BLOCK_ID);
          phys = -1;
        }
        // per 128-byte line of rows of the blocks that are loaded
        const uint32_t bytes = (uint32_t)__popc(__ballot_sync(0xffffffffu, phys >= 0)) * (BS * 128u);
        for (int kv = 0; kv < 2; ++kv) {
          const int seq = 2 * tc_ + kv, s = seq % kNST;
          const bool codes = kv ? V8 : K8;
          bool ok2 = true;
          if (lane == 0) {
            ok2 = mbar_wait(bar(B_EMPTY + s), ((seq / kNST) & 1) ^ 1, abort_flag);
            if (ok2) mbar_expect_tx(bar(B_FULL + s), codes ? bytes : 2u * bytes);
          }
          if (!__shfl_sync(0xffffffffu, ok2, 0)) { stop = true; break; }
          const uint32_t dst = sbase + OFF_KV + s * kOp;
          if (phys >= 0) {
            if (codes) {
              tma_load_4d(dst + kHalf + lane * (BS * 128), kv ? &tmV : &tmK, 0, 0, x.h, phys,
                          bar(B_FULL + s));
            } else {
              for (int hh = 0; hh < 2; ++hh)
                tma_load_5d(dst + hh * kHalf + lane * (BS * 128), kv ? &tmV : &tmK, 0, 0, x.h, hh,
                            phys, bar(B_FULL + s));
            }
          }
          ++issued;
        }
      }
      ++ui;
    }
    if (lane == 0) {
      if (stop) give_up();
      // never leave with copies in flight: the last loads of every stage and query buffer
      for (int seq = max(0, issued - kNST); seq < issued; ++seq) {
        const int s = seq % kNST;
        const uint64_t t0 = globaltimer();
        while (!mbar_try(bar(B_FULL + s), (seq / kNST) & 1) && globaltimer() - t0 < kWaitNs) {}
      }
      for (int qb = 0; qb < 2; ++qb) {
        if (q_last[qb] < 0) continue;
        const uint64_t t0 = globaltimer();
        while (!mbar_try(bar(B_QFULL + qb), (q_last[qb] >> 1) & 1) && globaltimer() - t0 < kWaitNs) {}
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int tc_ = 0, ui = 0;
      bool ok = true;
      // output product of tile tt (the unit's first if first) into O buffer ob
      auto issue_pv = [&](int tt, bool first, int ob) -> bool {
        const int pb = tt & 1;
        if (!mbar_wait(bar(B_PREADY + pb), (tt >> 1) & 1, abort_flag)) return false;
        // the O buffer was last used by unit ui - 2: wait for its epilogue
        if (first && ui >= 2 && !mbar_wait(bar(B_ODONE + ob), ((ui - 2) >> 1) & 1, abort_flag))
          return false;
        const int seq = 2 * tt + 1, s = seq % kNST;
        if (!mbar_wait(ready_bar(1, s), ready_parity(1, seq), abort_flag)) return false;
        tc_fence_after();
        const uint32_t vst = sbase + OFF_KV + s * kOp;
#pragma unroll
        for (int part = 0; part < 2; ++part) {
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk) {
            const uint64_t bd = sw128_desc(vst + kk * 16 * 128, kHalf, 1024);
            mma_f16_ta(tmem_o + ob * kD,
                       tmem_s + pb * kTile + (kk >> 1) * 32 + part * 16 + (kk & 1) * 8, bd, IDESC_O,
                       (first && part == 0 && kk == 0) ? 0u : 1u);
          }
        }
        mma_commit(bar(B_EMPTY + s));
        mma_commit(bar(B_OSTEP + pb));
        return true;
      };
      for (long long kk = 0; ok; ++kk) {
        const long long u = fa_unit_of_cta(kk, blockIdx.x, gridDim.x);
        if (u >= U) break;
        const FUnit x = fa_unit<G>(a, u);
        if (x.ntok <= 0) continue;
        const int qi = ui & 1, ob = ui & 1;
        if (!mbar_wait(bar(B_QFULL + qi), (ui >> 1) & 1, abort_flag)) { ok = false; break; }
        const uint32_t qst = sbase + OFF_Q + qi * kOp;
        for (int k = 0; k < x.ntiles; ++k, ++tc_) {
          const int sb = tc_ & 1;
          const int seq = 2 * tc_, s = seq % kNST;
          if (!mbar_wait(ready_bar(0, s), ready_parity(0, seq), abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t kst = sbase + OFF_KV + s * kOp;
#pragma unroll
          for (int ks = 0; ks < kD / 16; ++ks) {
            const uint64_t ad = sw128_desc(qst + (ks >> 2) * kHalf + (ks & 3) * 32, 16, 1024);
            const uint64_t bd = sw128_desc(kst + (ks >> 2) * kHalf + (ks & 3) * 32, 16, 1024);
            mma_f16(tmem_s + sb * kTile, ad, bd, IDESC_S, ks > 0 ? 1u : 0u);
          }
          mma_commit(bar(B_EMPTY + s));
          mma_commit(bar(B_SFULL + sb));
          if (k == x.ntiles - 1) mma_commit(bar(B_QEMPTY + qi));
          if (k > 0 && !issue_pv(tc_ - 1, k == 1, ob)) { ok = false; break; }
        }
        if (ok && !issue_pv(tc_ - 1, x.ntiles == 1, ob)) ok = false;
        ++ui;
      }
      if (!ok) give_up();
      mma_commit(bar(B_DONE));                   // every issued MMA done before TMEM is freed
      const uint64_t t0 = globaltimer();
      while (!mbar_try(bar(B_DONE), 0) && globaltimer() - t0 < kWaitNs) {}
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    // Two groups of four warps share the 128 query rows: thread (hf, r) owns row
    // r's keys [64 hf, 64 hf + 64) of each tile and its O columns [64 hf, 64 hf +
    // 64) (warps w and w + 4 reach the same tensor-memory lanes). The groups
    // exchange each tile's row maxima and, at a unit's end, the row sums.
    const int r = threadIdx.x & 127;             // query row = TMEM lane
    const int hf = threadIdx.x >> 7;             // which half of the keys and of O
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const int tl = r / G, g = r - (r / G) * G;   // token of the unit, head of the group
    float* xch = reinterpret_cast<float*>(smem + OFF_XCH);    // [2][128]
    auto sync256 = [] { asm volatile("bar.sync 1, 256;" ::: "memory"); };
    auto vote256 = [](bool v) -> bool {
      uint32_t o;
      asm volatile("{ .reg .pred pi, po; setp.ne.u32 pi, %1, 0; bar.red.or.pred po, 1, 256, pi;"
                   " selp.u32 %0, 1, 0, po; }"
                   : "=r"(o) : "r"((uint32_t)v) : "memory");
      return o != 0;
    };
    bool failed = false;
    int tc_ = 0, ui = 0;                         // tiles seen, units done
    // Wait for the output product of tile t. Products alternate between two
    // barriers by tile parity, so a parity wait is exact: the barrier of t has
    // passed the phase before t's (this group has seen S of tile t or a later
    // one, and the issuer puts S(t) after O(t - 2) on the in-order tensor pipe)
    // and cannot pass t's own before the group hands over tile t + 2. (One
    // barrier for every product could pass two phases while a slow warp had
    // not yet looked, and a parity wait would then take the wrong phase.)
    auto wait_o = [&](int t) {
      if (!mbar_wait(bar(B_OSTEP + (t & 1)), (t >> 1) & 1, abort_flag)) failed = true;
    };
    for (long long kk = 0; !failed; ++kk) {
      const long long u = fa_unit_of_cta(kk, blockIdx.x, gridDim.x);
      if (u >= U) break;
      const FUnit x = fa_unit<G>(a, u);
      if (x.ntok <= 0) continue;
      const int ob = ui & 1;
      const bool row_ok = tl < x.ntok;
      const int pos = x.pos0 + tl;               // this row attends keys [0, pos]
      const int32_t* table = a.block_tables + (size_t)x.b * a.max_blocks;
      float m = -CUDART_INF_F, l = 0.f;          // l: this half's part of the row sum
      // blocks of tile j with a bad id (the producer loaded nothing there)
      auto tile_bad = [&](int j) {
        const int tsj = j * kTile;
        const int nb = (min(x.t1, tsj + kTile) - tsj + BS - 1) / BS;
        uint32_t bb = 0;
#pragma unroll
        for (int q = 0; q < NB_T; ++q) {
          if (q >= nb) continue;
          const int ph = __ldg(table + tsj / BS + q);
          if (ph < 0 || ph >= a.num_blocks) bb |= 1u << q;
        }
        return bb;
      };
      // FP8 pools: widen row r of tile j's K stage (group 0) or V stage (group 1)
      // (global tile tj); a V row no row of the unit attends becomes zeros
      auto widen_tile = [&](int j, int tj) {
        if constexpr (K8 || V8) {
          const int kv = hf;
          if (kv ? V8 : K8) {
            const bool zv = kv == 1 && (j * kTile + r >= x.t1 || ((tile_bad(j) >> (r / BS)) & 1u));
            const int seq = 2 * tj + kv, s = seq % kNST;
            if (!mbar_wait(bar(B_FULL + s), (seq / kNST) & 1, abort_flag)) failed = true;
            if (!failed) widen_row_fp8<FMT>(smem + OFF_KV + s * kOp, r, zv);
            fence_proxy_async();
            mbar_arrive(bar(B_CONV + s));
          }
        }
      };
      widen_tile(0, tc_);
      for (int k = 0; k < x.ntiles; ++k, ++tc_) {
        const int sb = tc_ & 1;
        const int ts = k * kTile;
        const uint32_t badblk = tile_bad(k);
        // V row r of the stage: zero if no row of the unit attends key ts + r
        const bool zero_v = ts + r >= x.t1 || ((badblk >> (r / BS)) & 1u);
        if (!mbar_wait(bar(B_SFULL + sb), (tc_ >> 1) & 1, abort_flag)) failed = true;
        tc_fence_after();
        const uint32_t srow = tmem_s + lane_off + sb * kTile;
        // scores in the log2 domain, masked: keys past the row's position and
        // keys of blocks with a bad id get -inf. The visibility of a 32-key
        // chunk is one bit per key, computed without branches; a chunk every
        // row of the warp sees whole takes the loop without the mask (most
        // chunks), so no per-key branch or select is left in the hot loops.
        auto chunk_mask = [&](int c) -> uint32_t {
          const int n = min(max(pos - (ts + c) + 1, 0), 32);      // keys up to the position
          uint32_t msk = n >= 32 ? 0xffffffffu : ((1u << n) - 1u);
#pragma unroll
          for (int q = 0; q < 32 / BS; ++q)
            msk &= ((badblk >> (c / BS + q)) & 1u) ? ~(kBlkBits << (q * BS)) : 0xffffffffu;
          return row_ok ? msk : 0u;
        };
        const float sl2 = a.scale_log2;
        const int c_lo = 64 * hf;                // this half's first key column
        // pass 1: the maximum over this half's 64 keys, 32 columns of S at a time
        float tm = -CUDART_INF_F;
#pragma unroll 1
        for (int c = c_lo; c < c_lo + 64; c += 32) {
          uint32_t raw[32];
          tmem_ld32(srow + c, raw);
          tmem_wait_ld();
          const uint32_t vm = chunk_mask(c);
          float t0 = -CUDART_INF_F, t1 = -CUDART_INF_F, t2 = -CUDART_INF_F, t3 = -CUDART_INF_F;
          if (__all_sync(0xffffffffu, vm == 0xffffffffu)) {
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              t0 = fmaxf(t0, __uint_as_float(raw[j]) * sl2);
              t1 = fmaxf(t1, __uint_as_float(raw[j + 1]) * sl2);
              t2 = fmaxf(t2, __uint_as_float(raw[j + 2]) * sl2);
              t3 = fmaxf(t3, __uint_as_float(raw[j + 3]) * sl2);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              t0 = fmaxf(t0, ((vm >> j) & 1u) ? __uint_as_float(raw[j]) * sl2 : -CUDART_INF_F);
              t1 = fmaxf(t1, ((vm >> (j + 1)) & 1u) ? __uint_as_float(raw[j + 1]) * sl2 : -CUDART_INF_F);
              t2 = fmaxf(t2, ((vm >> (j + 2)) & 1u) ? __uint_as_float(raw[j + 2]) * sl2 : -CUDART_INF_F);
              t3 = fmaxf(t3, ((vm >> (j + 3)) & 1u) ? __uint_as_float(raw[j + 3]) * sl2 : -CUDART_INF_F);
            }
          }
          tm = fmaxf(tm, fmaxf(fmaxf(t0, t1), fmaxf(t2, t3)));
        }
        // the row's tile maximum: both halves (the second barrier keeps the
        // buffer until both have read it)
        xch[hf * 128 + r] = tm;
        sync256();
        tm = fmaxf(xch[r], xch[128 + r]);
        sync256();
        float alpha = 1.f;
        bool resc = false;
        if (k == 0) {
          m = fmaxf(tm, -FLT_MAX);
        } else if (tm > m + kRescaleLog2) {
          resc = true;
          alpha = ex2(m - tm);
          m = tm;
        }
        if (__any_sync(0xffffffffu, resc)) {
          // rare: this warp's rows move their reference; O holds the products of
          // tiles up to k - 1: wait for the last one, rescale this half of the
          // rows in TMEM (both halves of a row take the same decision)
          wait_o(tc_ - 1);
          tc_fence_after();
#pragma unroll 1
          for (int c = c_lo; c < c_lo + 64; c += 32) {
            uint32_t o[32];
            tmem_ld32(tmem_o + lane_off + ob * kD + c, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(tmem_o + lane_off + ob * kD + c, o);
          }
          tmem_wait_st();
          l *= alpha;
        }
        // pass 2: weights and this half's part of the row sum; each 32-column
        // chunk of S is read again and overwritten by its weights' 16-bit parts,
        // hi in the chunk's first 16 columns and lo in the next 16
#pragma unroll 1
        for (int c = c_lo; c < c_lo + 64; c += 32) {
          uint32_t raw[32];
          tmem_ld32(srow + c, raw);
          tmem_wait_ld();
          const uint32_t vm = chunk_mask(c);
          uint32_t pk[32];
          float l0 = 0.f, l1 = 0.f;
          if (__all_sync(0xffffffffu, vm == 0xffffffffu)) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float p0 = ex2(__uint_as_float(raw[2 * e]) * sl2 - m);
              const float p1 = ex2(__uint_as_float(raw[2 * e + 1]) * sl2 - m);
              l0 += p0;
              l1 += p1;
              split2<FMT>(p0, p1, pk[e], pk[16 + e]);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float x0 = __uint_as_float(raw[2 * e]) * sl2 - m;
              const float x1 = __uint_as_float(raw[2 * e + 1]) * sl2 - m;
              const float p0 = ex2(((vm >> (2 * e)) & 1u) ? x0 : -CUDART_INF_F);
              const float p1 = ex2(((vm >> (2 * e + 1)) & 1u) ? x1 : -CUDART_INF_F);
              l0 += p0;
              l1 += p1;
              split2<FMT>(p0, p1, pk[e], pk[16 + e]);
            }
          }
          l += l0 + l1;
          tmem_st32(srow + c, pk);
        }
        if (!V8 && zero_v) {
          // this V row enters the output product with weight 0: it must hold
          // finite values (each group zeroes one d-half of the row)
          const int seq = 2 * tc_ + 1, s = seq % kNST;
          if (!mbar_wait(bar(B_FULL + s), (seq / kNST) & 1, abort_flag)) failed = true;
          uint4* z = reinterpret_cast<uint4*>(smem + OFF_KV + s * kOp + hf * kHalf + r * 128);
#pragma unroll
          for (int q = 0; q < 8; ++q) z[q] = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async();
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(B_PREADY + sb));
        if (k + 1 < x.ntiles) widen_tile(k + 1, tc_ + 1);
      }
      // ---- epilogue: O / l of this row to the output, each half its 64
      // columns. The products of the last two tiles may both be pending; the
      // last one's commit tracks every earlier MMA, so one wait covers both.
      xch[hf * 128 + r] = l;
      sync256();
      const float lrow = xch[r] + xch[128 + r];
      sync256();
      wait_o(tc_ - 1);
      tc_fence_after();
      const float inv = lrow > 0.f ? a.v_scale / lrow : 0.f;
      const size_t orow = ((size_t)(x.qrow0 + tl) * a.Hq + (size_t)x.h * G + g) * kD;
#pragma unroll 1
      for (int c = 64 * hf; c < 64 * hf + 64; c += 32) {
        uint32_t o[32];
        tmem_ld32(tmem_o + lane_off + ob * kD + c, o);
        tmem_wait_ld();
        if (row_ok && !failed) {
          if (a.out_dtype == PA_F32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.out) + orow + c);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[e] = make_float4(__uint_as_float(o[4 * e]) * inv, __uint_as_float(o[4 * e + 1]) * inv,
                                   __uint_as_float(o[4 * e + 2]) * inv, __uint_as_float(o[4 * e + 3]) * inv);
          } else {
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float f0 = __uint_as_float(o[2 * e]) * inv, f1 = __uint_as_float(o[2 * e + 1]) * inv;
              if (a.out_dtype == PA_BF16) {
                const __nv_bfloat162 h = __floats2bfloat162_rn(f0, f1);
                pk[e] = *reinterpret_cast<const uint32_t*>(&h);
              } else {
                const __half2 h = __floats2half2_rn(f0, f1);
                pk[e] = *reinterpret_cast<const uint32_t*>(&h);
              }
            }
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.out) + orow + c);
#pragma unroll
            for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar(B_ODONE + ob));
      ++ui;
      // the warps of both groups leave together
      failed = vote256(failed);
    }
    if (failed) give_up();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

PFN_cuTensorMapEncodeTiled_v12000 fa_encode_fn() {
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

// Query [T][Hq][128] seen as [T][Hq][2 d-halves][64]: a box of TPU tokens x G
// heads x one d-half lands as 128 rows (token-major, then head) of 128 B,
// 128-byte swizzled. Pools [NB][bs][Hkv][128] seen as [NB][2][Hkv][bs][64]: a
// box of one block's bs rows of one head and one d-half.
bool make_fa_maps(const PrefillLaunch& p, int G, bool k8, bool v8, CUtensorMap* q, CUtensorMap* k,
                  CUtensorMap* v) {
  auto enc = fa_encode_fn();
  if (!enc || p.num_blocks <= 0) return false;
  const CUtensorMapDataType dt =
      p.dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const cuuint64_t qdims[4] = {64, 2, (cuuint64_t)p.Hq, (cuuint64_t)p.T};
  const cuuint64_t qstr[3] = {128, (cuuint64_t)kD * 2, (cuuint64_t)p.Hq * kD * 2};
  const cuuint32_t qbox[4] = {64, 1, (cuuint32_t)G, (cuuint32_t)(kM / G)};
  const cuuint32_t es4[4] = {1, 1, 1, 1};
  if (enc(q, dt, 4, const_cast<void*>(p.q), qdims, qstr, qbox, es4, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  const cuuint64_t dims[5] = {64, (cuuint64_t)p.bs, (cuuint64_t)p.Hkv, 2, (cuuint64_t)p.num_blocks};
  const cuuint64_t strides[4] = {(cuuint64_t)p.Hkv * kD * 2, (cuuint64_t)kD * 2, 128,
                                 (cuuint64_t)p.bs * p.Hkv * kD * 2};
  const cuuint32_t box[5] = {64, (cuuint32_t)p.bs, 1, 1, 1};
  const cuuint32_t es5[5] = {1, 1, 1, 1, 1};
  // FP8 pool [NB][bs][Hkv][128 codes]: a box of one block's bs rows of one head,
  // one 128-byte line per row
  const cuuint64_t cdims[4] = {(cuuint64_t)kD, (cuuint64_t)p.bs, (cuuint64_t)p.Hkv,
                               (cuuint64_t)p.num_blocks};
  const cuuint64_t cstr[3] = {(cuuint64_t)p.Hkv * kD, (cuuint64_t)kD, (cuuint64_t)p.bs * p.Hkv * kD};
  const cuuint32_t cbox[4] = {(cuuint32_t)kD, (cuuint32_t)p.bs, 1, 1};
  for (int i = 0; i < 2; ++i) {
    void* pool = const_cast<void*>(i == 0 ? p.k_cache : p.v_cache);
    const bool codes = i == 0 ? k8 : v8;
    const CUresult r =
        codes ? enc(i == 0 ? k : v, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, pool, cdims, cstr, cbox, es4,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE)
              : enc(i == 0 ? k : v, dt, 5, pool, dims, strides, box, es5,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
  }
  return true;
}

template <int FMT, int BS, int G, bool K8, bool V8>
int launch_fa_t(const FaArgs& a, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                cudaStream_t stream) {
  auto kern = prefill_fa_kernel<FMT, BS, G, K8, V8>;
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) !=
        cudaSuccess)
      return PA_ERR_CUDA;
    attr = true;
  }
  const long long U = (long long)a.B * a.chunks * a.Hkv;
  if (U <= 0) return PA_OK;
  const long long grid = U < sm_count_cached() ? U : sm_count_cached();
  return launch_k(kern, dim3((unsigned)grid), dim3(kThreads), kSmem, stream, a, q, k, v) ==
                 cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

template <int FMT, int BS, bool K8, bool V8>
int launch_fa_g(const FaArgs& a, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                cudaStream_t stream) {
  switch (a.Hq / a.Hkv) {
    case 1: return launch_fa_t<FMT, BS, 1, K8, V8>(a, q, k, v, stream);
    case 2: return launch_fa_t<FMT, BS, 2, K8, V8>(a, q, k, v, stream);
    case 4: return launch_fa_t<FMT, BS, 4, K8, V8>(a, q, k, v, stream);
    case 8: return launch_fa_t<FMT, BS, 8, K8, V8>(a, q, k, v, stream);
    case 16: return launch_fa_t<FMT, BS, 16, K8, V8>(a, q, k, v, stream);
  }
  return PA_ERR_UNSUPPORTED;
}

template <bool K8, bool V8>
int launch_fa_kv(const FaArgs& a, int dtype, int bs, const CUtensorMap& q, const CUtensorMap& k,
                 const CUtensorMap& v, cudaStream_t stream) {
  if (dtype == PA_BF16)
    return bs == 16 ? launch_fa_g<1, 16, K8, V8>(a, q, k, v, stream)
                    : launch_fa_g<1, 32, K8, V8>(a, q, k, v, stream);
  return bs == 16 ? launch_fa_g<0, 16, K8, V8>(a, q, k, v, stream)
                  : launch_fa_g<0, 32, K8, V8>(a, q, k, v, stream);
}

}  // namespace

bool prefill_fa_supported(int dtype, int Hq, int Hkv, int D, int bs) {
  if (dtype != PA_F16 && dtype != PA_BF16) return false;
  if (D != kD || (bs != 16 && bs != 32) || Hkv <= 0 || Hq % Hkv) return false;
  const int G = Hq / Hkv;
  return G == 1 || G == 2 || G == 4 || G == 8 || G == 16;
}

int launch_prefill_fa(const PrefillLaunch& p, cudaStream_t stream) {
  const int G = p.Hq / p.Hkv;
  const bool k8 = p.k_dtype == PA_FP8_E4M3, v8 = p.v_dtype == PA_FP8_E4M3;
  CUtensorMap q, k, v;
  if (!make_fa_maps(p, G, k8, v8, &q, &k, &v)) return PA_ERR_CUDA;
  FaArgs a{};
  a.out = p.out;
  a.out_dtype = p.out_dtype;
  a.block_tables = p.block_tables;
  a.max_blocks = p.max_blocks;
  a.context_lens = p.context_lens;
  a.query_start = p.query_start;
  a.B = p.B; a.Hq = p.Hq; a.Hkv = p.Hkv; a.bs = p.bs; a.num_blocks = p.num_blocks;
  a.chunks = (p.max_query_len + kM / G - 1) / (kM / G);
  a.scale_log2 = p.scale_log2;
  a.v_scale = v8 ? p.v_scale : 1.f;
  a.max_context_len = p.max_context_len;
  a.err_flag = p.err_flag;
  if (k8 && v8) return launch_fa_kv<true, true>(a, p.dtype, p.bs, q, k, v, stream);
  if (k8) return launch_fa_kv<true, false>(a, p.dtype, p.bs, q, k, v, stream);
  if (v8) return launch_fa_kv<false, true>(a, p.dtype, p.bs, q, k, v, stream);
  return launch_fa_kv<false, false>(a, p.dtype, p.bs, q, k, v, stream);
}

}  // namespace pa
