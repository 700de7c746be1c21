// decode_prefix_tc.cu -- decode attention of a group of sequences over the
// blocks they share (the group's common prefix), on the 5th-generation tensor
// cores: every shared block is streamed once per group, not once per sequence.
//
// Parallel sampling forks one prompt into sequences that share its physical
// blocks ("五十三：vLLM-PagedAttention" section 17; the copy-on-write sharing of
// "vLLM 与 LLM 推理部署实战" section 2.2). The decode queries of all of them
// attend those blocks. For every query row of a group this kernel computes the
// softmax state (m, l, acc) of each prefix partition (a multiple of 128 tokens);
// the merge kernel combines it with the partials of each sequence's own
// suffix (decode_simt.cu / decode_tc.cu in their split-only mode).
//
// Work unit = (group g, chunk c of the group's members, KV head h, prefix
// partition j). Rows of a unit = the chunk's members x the G query heads of
// KV head h, NQ <= kNQ = 64 (padded to NQP, a multiple of 16). Tile = 128
// tokens of KV head h: one TMA box per physical block and 64-wide d-half.
//   S^T[128 tokens x NQP] = K_tile . Q^T
//   O^T[128 d x NQP]     += V^T . P_hi^T + V^T . P_lo^T   (weights split in two
//                           16-bit parts, as in the per-sequence kernel)
// A softmax thread owns one token row of S^T. The reference max of a query
// column is set on the unit's first tile (an exact column max) and moves only
// when a score passes it by 2^64 (then O's columns are rescaled in TMEM), so a
// tile needs no reduction across threads; the column sums l are per-thread
// partial sums reduced once per unit. A score enters as one FMA against its
// column's reference (s * scale - m, log2 units); a 16-bit mask per token row
// says which of the thread's columns see the key (all of them on most tiles,
// one warp-uniform test), and references are floored at -FLT_MAX so a masked
// score stays -inf and its weight 2^-inf = 0 needs no guard.
//
// The same kernel runs paged prefill (PF = true): a chunk of a sequence's new
// query tokens attends, causally, to the sequence's own blocks — the prompt
// phase before decode (the lesson, "分块预填充": long prompts are cut into
// chunks that run beside decode steps). There a unit is (sequence b, chunk c
// of up to kNQ / G new tokens, KV head h); row q = (token q / G, query head
// q % G) at position pos0 + q / G attends keys [0, pos0 + q / G]; the unit
// covers all of them and writes the normalised output rows directly.
//
// CTA = 18 warps, persistent over units u = blockIdx.x + k * gridDim.x:
// warps 0-15 softmax and epilogue (warp w: TMEM lanes 32 (w % 4) .. + 31, query
// columns 16 (w / 4) .. + 15, so each row's columns are split among four
// warps and every scheduler runs four softmax warps), warp 16 TMA producer,
// warp 17 MMA issuer (it also owns the tensor memory). Every wait is bounded;
// one that gives up sets PA_DEV_TIMEOUT and the CTA drains and returns.
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
constexpr int kHalf = 128 * 128;                // one 64-wide d-half of a 128-row tile
constexpr int kStage = 2 * kHalf;               // one K or V tile: 32 KB
constexpr int kNST = 4;                         // ring stages
constexpr int kNQ = 64;                         // query rows per unit (max)
constexpr int kTile = 128;                      // tokens per tile
constexpr int kSplit = 4;                       // softmax threads per row of S^T
constexpr int kSoft = 128 * kSplit;             // softmax threads
constexpr int kHalfCols = kNQ / kSplit;         // query columns per softmax thread
constexpr int kSoftWarps = kSoft / 32;
constexpr int kThreads = kSoft + 64;            // + TMA producer warp + MMA warp
constexpr float kRescaleLog2 = 64.f;

constexpr int OFF_Q = kNST * kStage;            // Q: 2 d-halves x kNQ rows x 128 B
constexpr int kQBytes = 2 * kNQ * 128;
constexpr int OFF_P = OFF_Q + kQBytes;          // P: [2 buffers][hi, lo][2 token halves][kNQ][128 B]
constexpr int kPPart = 2 * kNQ * 128;
constexpr int kPBuf = 2 * kPPart;
constexpr int OFF_MREF = OFF_P + 2 * kPBuf;     // [3][kNQ] reference, old, new maxima
constexpr int OFF_RED = OFF_MREF + 3 * kNQ * 4; // [4 warps][kNQ]
constexpr int OFF_BAR = OFF_RED + 4 * kNQ * 4;
enum { B_FULL = 0, B_EMPTY = kNST, B_QFULL = 2 * kNST, B_QEMPTY, B_SFULL, B_SFREE = B_SFULL + 2,
       B_PREADY = B_SFREE + 2, B_OFULL = B_PREADY + 2, B_ODONE = B_OFULL + 2, B_DONE,
       B_CONV, B_COUNT = B_CONV + kNST };
constexpr int OFF_MISC = OFF_BAR + 8 * B_COUNT;
constexpr int kSmem = OFF_MISC + 32 + 1024;
static_assert(kSmem <= 227 * 1024, "shared memory per CTA");
constexpr int kTmemCols = 256;                  // S x2 (2 * kNQ) + O (kNQ), rounded up

struct PrefixArgs {
  const void* q;
  const int32_t* block_tables;
  int max_blocks;
  const int32_t* shared_blocks;                 // [B] blocks each sequence shares with its group
  const int32_t* group_offsets;                 // [num_groups + 1]
  const int32_t* group_members;                 // [B]
  int num_groups, chunks, parts;                // chunks per group, prefix partitions
  int part_tokens;                              // tokens per prefix partition (multiple of 128)
  int B, Hq, Hkv, bs, num_blocks;
  float scale_log2;
  float v_scale;                                // value of one V unit (FP8 V pool; 1 otherwise)
  int P;                                        // workspace slots per sequence
  float* ws_acc;
  float* ws_m;
  float* ws_l;
  uint32_t* err_flag;
  // prefill mode
  const int32_t* query_start;                   // [B + 1]: new tokens of b are query rows [qs_b, qs_{b+1})
  const int32_t* context_lens;                  // [B]: tokens in the cache, the new ones included
  int max_context_len;
  void* out;                                    // [T, Hq, D] of out_dtype
  int out_dtype;
};

struct PUnit {
  int g, mbeg, nm, h, j, b0, t0, t1, ntiles, nq, nqp;
  int qrow0, pos0;                              // prefill: first query row, its position
  bool bad;                                     // prefill: the sequence's lengths are inconsistent
};

// Prefill unit u = (sequence b, chunk c, KV head h): nm = tokens of the chunk.
__device__ __forceinline__ PUnit prefill_unit(const PrefixArgs& a, int G, int mc, long long u) {
  PUnit x;
  x.h = (int)(u % a.Hkv);
  const long long t = u / a.Hkv;
  const int c = (int)(t % a.chunks);
  const int b = (int)(t / a.chunks);
  const int qs = __ldg(a.query_start + b), qe = __ldg(a.query_start + b + 1);
  const int n = qe - qs, ctx = __ldg(a.context_lens + b);
  x.bad = n < 0 || ctx < n || ctx > a.max_blocks * a.bs || ctx > a.max_context_len;
  x.g = b; x.mbeg = 0; x.j = 0; x.b0 = b; x.t0 = 0;
  x.nm = x.bad ? 0 : min(mc, n - c * mc);
  x.qrow0 = qs + c * mc;
  x.pos0 = ctx - n + c * mc;
  x.t1 = x.nm > 0 ? x.pos0 + x.nm : 0;          // keys of the chunk's last token, inclusive
  x.ntiles = (x.t1 + kTile - 1) / kTile;
  x.nq = x.nm * G;
  x.nqp = (x.nq + 15) / 16 * 16;
  return x;
}

// Decode unit u; nm <= 0 means the unit has no rows (every role skips it).
__device__ __forceinline__ PUnit prefix_unit(const PrefixArgs& a, int G, int mc, long long u) {
  PUnit x;
  x.j = (int)(u % a.parts);
  long long t = u / a.parts;
  x.h = (int)(t % a.Hkv);
  t /= a.Hkv;
  const int c = (int)(t % a.chunks);
  x.g = (int)(t / a.chunks);
  const int gb = __ldg(a.group_offsets + x.g), ge = __ldg(a.group_offsets + x.g + 1);
  x.mbeg = gb + c * mc;
  x.nm = min(ge, x.mbeg + mc) - x.mbeg;
  x.b0 = gb < ge ? __ldg(a.group_members + gb) : 0;
  int sb = x.nm > 0 ? __ldg(a.shared_blocks + x.b0) : 0;
  if (sb < 0 || sb > a.max_blocks) sb = 0;      // never read past the table (the suffix pass flags it)
  const int ptoks = sb * a.bs;
  x.t0 = x.j * a.part_tokens;
  x.t1 = min(ptoks, x.t0 + a.part_tokens);
  x.ntiles = x.t1 > x.t0 ? (x.t1 - x.t0 + kTile - 1) / kTile : 0;
  x.nq = x.nm * G;
  x.nqp = (x.nq + 15) / 16 * 16;
  x.qrow0 = 0; x.pos0 = 0; x.bad = false;
  return x;
}

template <bool PF>
__device__ __forceinline__ PUnit mq_unit(const PrefixArgs& a, int G, int mc, long long u) {
  return PF ? prefill_unit(a, G, mc, u) : prefix_unit(a, G, mc, u);
}

// 2^x by the multi-function unit's approximation (relative error ~2^-22, flushes
// subnormal results to 0; -inf gives +0): the weights then go through the hi/lo
// 16-bit split, which keeps far less than that.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Named barrier of the kSoft softmax threads; vote = OR of every thread's flag.
__device__ __forceinline__ void sm_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kSoft) : "memory"); }
__device__ __forceinline__ bool sm_vote(bool x) {
  uint32_t r;
  asm volatile(
      "{ .reg .pred pi, po; setp.ne.u32 pi, %1, 0; bar.red.or.pred po, 1, %2, pi;"
      " selp.u32 %0, 1, 0, po; }"
      : "=r"(r)
      : "r"((uint32_t)x), "n"(kSoft)
      : "memory");
  return r != 0;
}

// K8 / V8 (shared-prefix mode): that pool holds FP8 E4M3 codes. TMA brings a
// tile's codes (one 128-byte line per row, at the stage's upper half) and the
// threads of the first query columns (one per tile row) widen them in place
// to the query's 16-bit type, exactly, before the tile goes to the tensor cores.
template <int FMT, int BS, bool PF, bool K8 = false, bool V8 = false>
__global__ void __launch_bounds__(kThreads, 1)
multi_query_tc_kernel(const PrefixArgs a, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV) {
  constexpr int NB_T = kTile / BS;              // physical blocks per tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_addr(smem);
  auto bar = [&](int i) { return sbase + OFF_BAR + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.Hq / a.Hkv;
  const int mc = kNQ / G;                       // members (prefill: tokens) per chunk
  const long long U = PF ? (long long)a.B * a.chunks * a.Hkv
                         : (long long)a.num_groups * a.chunks * a.Hkv * a.parts;
  pdl_trigger();

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNST; ++s) {
      mbar_init(bar(B_FULL + s), 1);
      mbar_init(bar(B_EMPTY + s), 1);
    }
    mbar_init(bar(B_QFULL), kSoft);
    mbar_init(bar(B_QEMPTY), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(B_SFULL + i), 1);
      mbar_init(bar(B_SFREE + i), kSoft);
      mbar_init(bar(B_PREADY + i), kSoft);
      mbar_init(bar(B_OFULL + i), 1);
    }
    mbar_init(bar(B_ODONE), kSoft);
    mbar_init(bar(B_DONE), 1);
    for (int s = 0; s < kNST; ++s) mbar_init(bar(B_CONV + s), 128);
    *abort_flag = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kSoftWarps + 1) {
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
  const uint32_t tmem_s = tmem;                 // S buffers: columns [0, kNQ), [kNQ, 2 kNQ)
  const uint32_t tmem_o = tmem + 2 * kNQ;       // O: [2 kNQ, 3 kNQ)
  auto give_up = [&]() {
    *abort_flag = 1u;
    flag_error(a.err_flag, PA_DEV_TIMEOUT);
  };
  // a stage holding K (kv = 0) or V (kv = 1) is ready for the tensor cores when
  // TMA filled it (16-bit pool) or when its rows were widened (FP8 pool)
  auto ready_bar = [&](int kv, int s) {
    return bar(((kv ? V8 : K8) ? B_CONV : B_FULL) + s);
  };

  if (warp == kSoftWarps) {
    // ------------------------------------------------------------ producer
    // The warp's lanes share a tile's copies: lane q < NB_T issues those of the
    // tile's q-th block (one instruction starts them all) and reads that
    // block's id a tile ahead; lane 0 waits for free stages and sets the
    // expected bytes.
    {
      int tc_ = 0, issued = 0;
      bool stop = false;
      for (long long u = blockIdx.x; u < U && !stop; u += gridDim.x) {
        const PUnit x = mq_unit<PF>(a, G, mc, u);
        if (x.nm <= 0 || x.ntiles == 0) continue;
        const int32_t* table = a.block_tables + (size_t)x.b0 * a.max_blocks;
        // this lane's block of tile k of the unit (-1 for none)
        auto load_id = [&](int k) -> int {
          const int ts = x.t0 + k * kTile;
          const int nblk = (min(x.t1, ts + kTile) - ts + BS - 1) / BS;
          return lane < nblk ? __ldg(table + ts / BS + lane) : -1;
        };
        int phys_next = load_id(0);
        for (int k = 0; k < x.ntiles && !stop; ++k, ++tc_) {
          const int ts = x.t0 + k * kTile;
          const int nblk = (min(x.t1, ts + kTile) - ts + BS - 1) / BS;
          int phys = phys_next;
          if (k + 1 < x.ntiles) phys_next = load_id(k + 1);   // a tile ahead: off the issue path
          if (lane < nblk && (phys < 0 || phys >= a.num_blocks)) {
            flag_error(a.err_flag, PA_DEV_BAD_BLOCK_ID);
            phys = -1;
          }
          // per 128-byte line of rows of the blocks that are loaded
          const uint32_t bytes = (uint32_t)__popc(__ballot_sync(0xffffffffu, phys >= 0)) * (BS * 128u);
          for (int kv = 0; kv < 2; ++kv) {
            const int seq = 2 * tc_ + kv, s = seq % kNST;
            const bool codes = kv ? V8 : K8;
            bool ok = true;
            if (lane == 0) {
              ok = mbar_wait(bar(B_EMPTY + s), ((seq / kNST) & 1) ^ 1, abort_flag);
              if (ok) mbar_expect_tx(bar(B_FULL + s), codes ? bytes : 2u * bytes);
            }
            if (!__shfl_sync(0xffffffffu, ok, 0)) { stop = true; break; }
            const uint32_t dst = sbase + s * kStage;
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
      }
      if (lane == 0) {
        if (stop) give_up();
        for (int seq = max(0, issued - kNST); seq < issued; ++seq) {
          const int s = seq % kNST;
          const uint64_t t0 = globaltimer();
          while (!mbar_try(bar(B_FULL + s), (seq / kNST) & 1) && globaltimer() - t0 < kWaitNs) {}
        }
      }
    }
  } else if (warp == kSoftWarps + 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int tc_ = 0, ua = 0;
      bool ok = true;
      for (long long u = blockIdx.x; u < U && ok; u += gridDim.x) {
        const PUnit x = mq_unit<PF>(a, G, mc, u);
        if (x.nm <= 0 || x.ntiles == 0) continue;
        const uint32_t idesc_s = make_idesc(FMT, 0, 0, x.nqp, 128);
        const uint32_t idesc_o = make_idesc(FMT, 1, 0, x.nqp, 128);
        if (!mbar_wait(bar(B_QFULL), ua & 1, abort_flag)) { ok = false; break; }
        const uint32_t qst = sbase + OFF_Q;
        auto issue_pv = [&](int tt, bool first) -> bool {
          const int pb = tt & 1;
          if (!mbar_wait(bar(B_PREADY + pb), (tt >> 1) & 1, abort_flag)) return false;
          if (first && ua > 0 && !mbar_wait(bar(B_ODONE), (ua - 1) & 1, abort_flag)) return false;
          const int seq = 2 * tt + 1, s = seq % kNST;
          if (!mbar_wait(ready_bar(1, s), (seq / kNST) & 1, abort_flag)) return false;
          tc_fence_after();
          const uint32_t vst = sbase + s * kStage;
          const uint32_t pst = sbase + OFF_P + pb * kPBuf;
#pragma unroll
          for (int ks = 0; ks < kTile / 16; ++ks) {
            const uint64_t ad = sw128_desc(vst + ks * 16 * 128, kHalf, 1024);
#pragma unroll
            for (int part = 0; part < 2; ++part) {
              const uint64_t bd =
                  sw128_desc(pst + part * kPPart + (ks >> 2) * (kNQ * 128) + (ks & 3) * 32, 16, 1024);
              mma_f16(tmem_o, ad, bd, idesc_o, (first && ks == 0 && part == 0) ? 0u : 1u);
            }
          }
          mma_commit(bar(B_EMPTY + s));
          mma_commit(bar(B_OFULL + pb));
          return true;
        };
        for (int k = 0; k < x.ntiles; ++k) {
          const int sb = tc_ & 1;
          if (!mbar_wait(bar(B_SFREE + sb), ((tc_ >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
          const int seq = 2 * tc_, s = seq % kNST;
          if (!mbar_wait(ready_bar(0, s), (seq / kNST) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t kst = sbase + s * kStage;
#pragma unroll
          for (int ks = 0; ks < kD / 16; ++ks) {
            const uint64_t ad = sw128_desc(kst + (ks >> 2) * kHalf + (ks & 3) * 32, 16, 1024);
            const uint64_t bd = sw128_desc(qst + (ks >> 2) * (kNQ * 128) + (ks & 3) * 32, 16, 1024);
            mma_f16(tmem_s + sb * kNQ, ad, bd, idesc_s, ks > 0 ? 1u : 0u);
          }
          mma_commit(bar(B_EMPTY + s));
          mma_commit(bar(B_SFULL + sb));
          if (k == x.ntiles - 1) mma_commit(bar(B_QEMPTY));
          if (k > 0 && !issue_pv(tc_ - 1, k == 1)) { ok = false; break; }
          ++tc_;
        }
        if (ok && !issue_pv(tc_ - 1, x.ntiles == 1)) ok = false;
        ++ua;
      }
      if (!ok) give_up();
      mma_commit(bar(B_DONE));
      const uint64_t t0 = globaltimer();
      while (!mbar_try(bar(B_DONE), 0) && globaltimer() - t0 < kWaitNs) {}
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int r = threadIdx.x & 127;             // token row of S^T; d row of O^T
    const int c0 = (warp >> 2) * kHalfCols;      // first query column of this thread
    const int st = threadIdx.x;                  // 0 .. kSoft - 1
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    float* mref = reinterpret_cast<float*>(smem + OFF_MREF);
    float* mold = mref + kNQ;
    float* mnew = mold + kNQ;
    float* red = reinterpret_cast<float*>(smem + OFF_RED);
    bool failed = false, stop = false;
    int tc_ = 0, ua = 0;
    auto wait_pv = [&](int t) {                  // output product of tile t has completed
      if (!mbar_wait(bar(B_OFULL + (t & 1)), (t >> 1) & 1, abort_flag)) failed = true;
    };
    // column maxima of s[] (this thread's columns c0 + i) over the 128 rows -> dst[q],
    // floored at -FLT_MAX: a column with no visible key keeps a finite reference, so
    // score - reference is -inf exactly where the score is masked
    auto col_max = [&](const float* s, float* dst) {
#pragma unroll
      for (int i = 0; i < kHalfCols; ++i) {
        float v = s[i];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0) red[(warp & 3) * kNQ + c0 + i] = v;
      }
      sm_sync();
      if (st < kNQ)
        dst[st] = fmaxf(fmaxf(fmaxf(red[st], red[kNQ + st]), fmaxf(red[2 * kNQ + st], red[3 * kNQ + st])),
                        -FLT_MAX);
      sm_sync();
    };
    for (long long u = blockIdx.x; u < U && !stop; u += gridDim.x) {
      const PUnit x = mq_unit<PF>(a, G, mc, u);
      if (PF && x.bad && x.h == 0 && st == 0 && (u / a.Hkv) % a.chunks == 0)
        flag_error(a.err_flag, PA_DEV_BAD_CTX);
      if (x.nm <= 0) continue;
      // the (query token, head) row q of the unit in the query matrix
      auto q_row = [&](int q) -> size_t {
        const int tokrow = PF ? x.qrow0 + q / G : __ldg(a.group_members + x.mbeg + q / G);
        return (size_t)tokrow * a.Hq + (size_t)x.h * G + (q % G);
      };
      // rows of the unit: q = m * G + gg -> (sequence, query head) slot of partition j
      auto slot_row = [&](int q) -> size_t {
        const int b = __ldg(a.group_members + x.mbeg + q / G);
        return ((size_t)b * a.P + x.j) * a.Hq + (size_t)x.h * G + (q % G);
      };
      if (!PF && x.ntiles == 0) {
        // this partition of the prefix holds no tokens: an empty partial
        for (int i = 0; i < kHalfCols; ++i)
          if (c0 + i < x.nq) a.ws_acc[slot_row(c0 + i) * kD + r] = 0.f;
        if (st < x.nq) {
          a.ws_m[slot_row(st)] = -CUDART_INF_F;
          a.ws_l[slot_row(st)] = 0.f;
        }
        continue;
      }
      // Q rows of the unit into the K-major 128-byte-swizzled operand
      if (ua > 0 && !mbar_wait(bar(B_QEMPTY), (ua - 1) & 1, abort_flag)) failed = true;
      for (int c = st; c < x.nqp * 16; c += kSoft) {
        const int q = c >> 4, k16 = c & 15, hh = k16 >> 3, kk = k16 & 7;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (q < x.nq)
          v = *reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(a.q) + q_row(q) * (kD * 2) +
                                              k16 * 16);
        *reinterpret_cast<uint4*>(smem + OFF_Q + hh * (kNQ * 128) + q * 128 + ((kk ^ (q & 7)) << 4)) = v;
      }
      fence_proxy_async();
      mbar_arrive(bar(B_QFULL));

      float l[kHalfCols];                        // partial exp-sums of columns c0 + i
#pragma unroll
      for (int i = 0; i < kHalfCols; ++i) l[i] = 0.f;
      const int32_t* table = a.block_tables + (size_t)x.b0 * a.max_blocks;
      for (int k = 0; k < x.ntiles; ++k, ++tc_) {
        const int ts = x.t0 + k * kTile;
        const int tok = ts + r;
        bool valid = tok < x.t1;
        if (valid) {
          const int32_t p = __ldg(table + tok / BS);
          valid = p >= 0 && p < a.num_blocks;
        }
        // bit i of mk: column c0 + i is a real query row that sees this key (prefill:
        // column q, at position pos0 + q / G, sees key tok iff q >= (tok - pos0) * G)
        const int qlo = PF ? min(max((tok - x.pos0) * G - c0, 0), kHalfCols) : 0;
        const int qhi = valid ? min(max(x.nq - c0, 0), kHalfCols) : 0;
        const uint32_t mk = qhi > qlo ? ((1u << qhi) - 1u) & ~((1u << qlo) - 1u) : 0u;
        const bool full = __all_sync(0xffffffffu, mk == (1u << kHalfCols) - 1u);
        if constexpr (K8 || V8) {
          // widen this tile's rows (threads of the first column block, one per row);
          // a V row that must not count becomes zeros
          if (c0 == 0) {
#pragma unroll 1
            for (int kv = 0; kv < 2; ++kv) {
              if (!(kv ? V8 : K8)) continue;
              const int seq = 2 * tc_ + kv, s = seq % kNST;
              if (!mbar_wait(bar(B_FULL + s), (seq / kNST) & 1, abort_flag)) failed = true;
              if (!failed) widen_row_fp8<FMT>(smem + s * kStage, r, kv == 1 && !valid);
              fence_proxy_async();
              mbar_arrive(bar(B_CONV + s));
            }
          }
        }
        if (!mbar_wait(bar(B_SFULL + (tc_ & 1)), (tc_ >> 1) & 1, abort_flag)) failed = true;
        tc_fence_after();
        float s[kHalfCols];
#pragma unroll
        for (int c = 0; c < kHalfCols; c += 16)
          tmem_ld16(tmem_s + lane_off + (tc_ & 1) * kNQ + c0 + c, s + c);
        tc_fence_before();
        mbar_arrive(bar(B_SFREE + (tc_ & 1)));
        if (sm_vote(failed)) { stop = true; break; }
        // s[i] becomes the scaled score of column c0 + i minus the column's reference
        // maximum (log2 units): -inf where the key is masked
        if (k == 0) {
#pragma unroll
          for (int i = 0; i < kHalfCols; ++i)
            s[i] = ((mk >> i) & 1u) ? s[i] * a.scale_log2 : -CUDART_INF_F;
          col_max(s, mref);
#pragma unroll
          for (int i = 0; i < kHalfCols; ++i) s[i] -= mref[c0 + i];
        } else {
          const float4* m4 = reinterpret_cast<const float4*>(mref + c0);
#pragma unroll
          for (int j = 0; j < kHalfCols / 4; ++j) {
            const float4 m = m4[j];
            s[4 * j] = fmaf(s[4 * j], a.scale_log2, -m.x);
            s[4 * j + 1] = fmaf(s[4 * j + 1], a.scale_log2, -m.y);
            s[4 * j + 2] = fmaf(s[4 * j + 2], a.scale_log2, -m.z);
            s[4 * j + 3] = fmaf(s[4 * j + 3], a.scale_log2, -m.w);
          }
          if (!full) {
#pragma unroll
            for (int i = 0; i < kHalfCols; ++i)
              if (!((mk >> i) & 1u)) s[i] = -CUDART_INF_F;
          }
          float mx = s[0];
#pragma unroll
          for (int i = 1; i < kHalfCols; ++i) mx = fmaxf(mx, s[i]);
          if (sm_vote(mx > kRescaleLog2)) {
            // rare: some column passed its reference by more than 2^64. Its reference
            // moves up by the tile's maximum d of that column (relative to it), and its
            // O (all earlier products included) and l are scaled by 2^-d
            col_max(s, mnew);
            if (st < kNQ) mold[st] = mnew[st] > kRescaleLog2 ? mnew[st] : 0.f;
            sm_sync();
            wait_pv(tc_ - 1);
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < kHalfCols; c += 16) {
              float o[16];
              tmem_ld16(tmem_o + lane_off + c0 + c, o);
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const float d = mold[c0 + c + e];
                if (d != 0.f) {
                  const float f = exp2f(-d);
                  o[e] *= f;
                  l[c + e] *= f;
                }
              }
              tmem_st16(tmem_o + lane_off + c0 + c, o);
            }
            tc_fence_before();
#pragma unroll
            for (int i = 0; i < kHalfCols; ++i) s[i] -= mold[c0 + i];
            sm_sync();
            if (st < kNQ) mref[st] += mold[st];
            sm_sync();
          }
        }
        // the P buffer of this tile was last read by the output product of tile tc - 2
        if (tc_ >= 2) wait_pv(tc_ - 2);
        uint8_t* pb = smem + OFF_P + (tc_ & 1) * kPBuf + (r >> 6) * (kNQ * 128);
        const int pc = (r & 63) >> 3, pbyte = (r & 7) * 2;
#pragma unroll
        for (int i = 0; i < kHalfCols; ++i) {
          const int q = c0 + i;
          const float p = fast_exp2(s[i]);        // 0 where masked
          l[i] += p;
          uint16_t hi, lo;
          split_16<FMT>(p, hi, lo);
          const int off = q * 128 + ((pc ^ (q & 7)) << 4) + pbyte;
          *reinterpret_cast<uint16_t*>(pb + off) = hi;
          *reinterpret_cast<uint16_t*>(pb + kPPart + off) = lo;
        }
        if (!V8 && !valid && c0 == 0) {
          // a row with weight 0 still enters the product: it must hold finite values
          const int seq = 2 * tc_ + 1, sv = seq % kNST;
          if (!mbar_wait(bar(B_FULL + sv), (seq / kNST) & 1, abort_flag)) failed = true;
          uint4* r0 = reinterpret_cast<uint4*>(smem + sv * kStage + r * 128);
          uint4* r1 = reinterpret_cast<uint4*>(smem + sv * kStage + kHalf + r * 128);
#pragma unroll
          for (int c = 0; c < 8; ++c) { r0[c] = make_uint4(0, 0, 0, 0); r1[c] = make_uint4(0, 0, 0, 0); }
        }
        fence_proxy_async();
        mbar_arrive(bar(B_PREADY + (tc_ & 1)));
      }
      if (stop) break;

      // ---- end of the unit: column sums, then O and (m, l) to the workspace
      wait_pv(tc_ - 1);
      if (sm_vote(failed)) break;
#pragma unroll
      for (int i = 0; i < kHalfCols; ++i) {
        float v = l[i];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red[(warp & 3) * kNQ + c0 + i] = v;
      }
      sm_sync();
      if (PF) {
        // prefill: each column's exp-sum, then normalised rows straight to the output
        if (st < kNQ) mold[st] = red[st] + red[kNQ + st] + red[2 * kNQ + st] + red[3 * kNQ + st];
        sm_sync();
      } else if (st < x.nq) {
        const size_t sr = slot_row(st);
        a.ws_m[sr] = mref[st] == -FLT_MAX ? -CUDART_INF_F : mref[st];
        a.ws_l[sr] = red[st] + red[kNQ + st] + red[2 * kNQ + st] + red[3 * kNQ + st];
      }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < kHalfCols; c += 16) {
        float o[16];
        tmem_ld16(tmem_o + lane_off + c0 + c, o);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int q = c0 + c + e;
          if (q >= x.nq) continue;
          if (PF) {
            const float L = mold[q];
            store_out(a.out, q_row(q) * kD + r, L > 0.f ? o[e] / L : 0.f, a.out_dtype);
          } else {
            a.ws_acc[slot_row(q) * kD + r] = o[e] * a.v_scale;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar(B_ODONE));
      sm_sync();                                 // red and mref are rewritten by the next unit
      ++ua;
    }
    if (failed) give_up();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kSoftWarps + 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

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

// The pool [NB][bs][Hkv][D] seen as [NB][2][Hkv][bs][64]: a box of one block's
// bs rows of one head and one d-half, 128-byte swizzled.
bool make_prefix_maps(const void* k_cache, const void* v_cache, int dtype, int bs, int Hkv,
                      int num_blocks, CUtensorMap* k, CUtensorMap* v, bool k8 = false,
                      bool v8 = false) {
  auto enc = encode_fn();
  if (!enc || num_blocks <= 0) return false;
  const CUtensorMapDataType dt =
      dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const cuuint64_t dims[5] = {64, (cuuint64_t)bs, (cuuint64_t)Hkv, 2, (cuuint64_t)num_blocks};
  const cuuint64_t strides[4] = {(cuuint64_t)Hkv * kD * 2, (cuuint64_t)kD * 2, 128,
                                 (cuuint64_t)bs * Hkv * kD * 2};
  const cuuint32_t box[5] = {64, (cuuint32_t)bs, 1, 1, 1};
  const cuuint32_t es[5] = {1, 1, 1, 1, 1};
  // FP8 pool [NB][bs][Hkv][128 codes]: a box of one block's bs rows of one head
  const cuuint64_t cdims[4] = {(cuuint64_t)kD, (cuuint64_t)bs, (cuuint64_t)Hkv,
                               (cuuint64_t)num_blocks};
  const cuuint64_t cstr[3] = {(cuuint64_t)Hkv * kD, (cuuint64_t)kD, (cuuint64_t)bs * Hkv * kD};
  const cuuint32_t cbox[4] = {(cuuint32_t)kD, (cuuint32_t)bs, 1, 1};
  for (int i = 0; i < 2; ++i) {
    void* pool = const_cast<void*>(i == 0 ? k_cache : v_cache);
    const CUresult r =
        (i == 0 ? k8 : v8)
            ? enc(i == 0 ? k : v, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, pool, cdims, cstr, cbox, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE)
            : enc(i == 0 ? k : v, dt, 5, pool, dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
  }
  return true;
}

template <int FMT, int BS, bool PF, bool K8 = false, bool V8 = false>
int launch_mq_t(const PrefixArgs& a, const CUtensorMap& k, const CUtensorMap& v,
                cudaStream_t stream) {
  auto kern = multi_query_tc_kernel<FMT, BS, PF, K8, V8>;
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) !=
        cudaSuccess)
      return PA_ERR_CUDA;
    attr = true;
  }
  const long long U = PF ? (long long)a.B * a.chunks * a.Hkv
                         : (long long)a.num_groups * a.chunks * a.Hkv * a.parts;
  if (U <= 0) return PA_OK;
  int dev = 0, sms = kSMs;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long grid = U < sms ? U : sms;
  return launch_k(kern, dim3((unsigned)grid), dim3(kThreads), kSmem, stream, a, k, v) ==
                 cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace

bool prefix_tc_supported(int dtype, int Hq, int Hkv, int D, int bs) {
  if (dtype != PA_F16 && dtype != PA_BF16) return false;
  if (D != kD || (bs != 16 && bs != 32) || Hkv <= 0 || Hq % Hkv) return false;
  return Hq / Hkv <= kNQ;
}

int prefix_chunks(int max_group_size, int G) {
  const int mc = kNQ / G;
  return (max_group_size + mc - 1) / mc;
}

template <int FMT, int BS>
int launch_prefix_kv(const PrefixArgs& a, bool k8, bool v8, const CUtensorMap& k,
                     const CUtensorMap& v, cudaStream_t stream) {
  if (k8 && v8) return launch_mq_t<FMT, BS, false, true, true>(a, k, v, stream);
  if (k8) return launch_mq_t<FMT, BS, false, true, false>(a, k, v, stream);
  if (v8) return launch_mq_t<FMT, BS, false, false, true>(a, k, v, stream);
  return launch_mq_t<FMT, BS, false>(a, k, v, stream);
}

int launch_prefix_tc(const DecodeArgs& d, int dtype, const int32_t* group_offsets,
                     const int32_t* group_members, int num_groups, int max_group_size,
                     int parts, int part_tokens, cudaStream_t stream, bool k8, bool v8) {
  CUtensorMap k, v;
  if (!make_prefix_maps(d.k_cache, d.v_cache, dtype, d.bs, d.Hkv, d.num_blocks, &k, &v, k8, v8))
    return PA_ERR_CUDA;
  PrefixArgs a{};
  a.q = d.q;
  a.block_tables = d.block_tables;
  a.max_blocks = d.max_blocks;
  a.shared_blocks = d.start_blocks;
  a.group_offsets = group_offsets;
  a.group_members = group_members;
  a.num_groups = num_groups;
  a.chunks = prefix_chunks(max_group_size, d.Hq / d.Hkv);
  a.parts = parts;
  a.part_tokens = part_tokens;
  a.B = d.B; a.Hq = d.Hq; a.Hkv = d.Hkv; a.bs = d.bs; a.num_blocks = d.num_blocks;
  a.scale_log2 = d.scale_log2;
  a.P = d.P;
  a.ws_acc = d.ws_acc; a.ws_m = d.ws_m; a.ws_l = d.ws_l;
  a.err_flag = d.err_flag;
  a.v_scale = d.v_scale;
  if (dtype == PA_BF16)
    return d.bs == 16 ? launch_prefix_kv<1, 16>(a, k8, v8, k, v, stream)
                      : launch_prefix_kv<1, 32>(a, k8, v8, k, v, stream);
  return d.bs == 16 ? launch_prefix_kv<0, 16>(a, k8, v8, k, v, stream)
                    : launch_prefix_kv<0, 32>(a, k8, v8, k, v, stream);
}

int launch_prefill_tc(const PrefillLaunch& p, cudaStream_t stream) {
  CUtensorMap k, v;
  if (!make_prefix_maps(p.k_cache, p.v_cache, p.dtype, p.bs, p.Hkv, p.num_blocks, &k, &v))
    return PA_ERR_CUDA;
  PrefixArgs a{};
  a.q = p.q;
  a.block_tables = p.block_tables;
  a.max_blocks = p.max_blocks;
  a.query_start = p.query_start;
  a.context_lens = p.context_lens;
  a.max_context_len = p.max_context_len;
  a.out = p.out;
  a.out_dtype = p.out_dtype;
  a.B = p.B; a.Hq = p.Hq; a.Hkv = p.Hkv; a.bs = p.bs; a.num_blocks = p.num_blocks;
  a.scale_log2 = p.scale_log2;
  a.chunks = (p.max_query_len + kNQ / (p.Hq / p.Hkv) - 1) / (kNQ / (p.Hq / p.Hkv));
  a.parts = 1;
  a.err_flag = p.err_flag;
  a.v_scale = 1.f;
  if (p.dtype == PA_BF16)
    return p.bs == 16 ? launch_mq_t<1, 16, true>(a, k, v, stream)
                      : launch_mq_t<1, 32, true>(a, k, v, stream);
  return p.bs == 16 ? launch_mq_t<0, 16, true>(a, k, v, stream)
                    : launch_mq_t<0, 32, true>(a, k, v, stream);
}

}  // namespace pa
