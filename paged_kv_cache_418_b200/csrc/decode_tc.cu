// decode_tc.cu -- grouped-query paged decode attention on the 5th-generation
// tensor cores (tcgen05, accumulators in tensor memory), for 16-bit K/V with
// head size 128 and G = Hq / Hkv in {4, 8, 16} query heads per KV head.
//
// Why tensor cores here: the G query heads that share a KV head turn the
// per-token work into a small dense contraction (G x 128 against 128-token
// tiles). On the CUDA cores that is ~4 FMAs per byte of K/V at G = 8, close to
// the FP32 pipe's limit at HBM speed; on tcgen05 it is a few MMAs per tile.
//
// Shapes (swap-AB, so the 128-token tile fills the MMA's M = 128):
//   scores  S^T[128 tok x 16]  = K_tile[128 tok x 128 d] . Q^T      (Q rows padded to 16)
//   output  O^T[128 d x NO]   += V_tile^T[128 d x 128 tok] . P^T     (P = [P_hi; P_lo])
// P is split into two 16-bit parts, p = hi + lo with hi = RN(p), lo = RN(p - hi),
// stacked as 2G rows of the B operand, so the products keep ~16 significant
// bits of the softmax weights instead of 8 (bf16); the two column groups of O
// are summed in fp32 afterwards. K/V products are exact and accumulate in fp32.
//
// Data movement: a 4-D TMA tensor map over the pool [num_blocks, bs, Hkv, D]
// loads, for one physical block and one KV head, bs rows x 64 d (128 bytes)
// with 128-byte swizzling, which is exactly the canonical SW128 K-major
// layout the MMA reads for K, and the MN-major layout it reads for V^T. One
// tile = 128 / bs such block loads per d-half, written side by side.
//
// CTA = 6 warps, persistent over work units (sequence, KV head, partition):
//   warps 0-3  softmax + output: read S from TMEM (one token row per thread),
//              online softmax over the tile (running max per head), write
//              P_hi/P_lo to shared memory, then fold the tile's O (one d row
//              per thread) into fp32 registers with the rescale factor;
//   warp 4     TMA producer (one lane): Q of the unit, then K and V tiles
//              through a 6-stage ring (192 KB in flight per SM);
//   warp 5     MMA issuer (one lane): S(t), then O(t-1), committing each to
//              mbarriers that release ring stages and hand results over.
// S and O each have two TMEM buffers and P two shared buffers, so the softmax
// of tile t overlaps the PV product of tile t-1 and the loads of later tiles.
//
// Every pipeline wait is bounded (1 s); a wait that gives up sets the
// PA_DEV_TIMEOUT bit, raises a CTA-wide abort flag, and all roles leave their
// loops (the softmax warps only together, at a named-barrier vote), wait for
// their own asynchronous work, free tensor memory and return.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math_constants.h>

#include "pa_internal.h"

namespace pa {

namespace {

constexpr int kD = 128;
constexpr int kTile = 128;                      // tokens per tile
constexpr int kHalf = kTile * 128;              // bytes of one 64-wide d-half of a tile
constexpr int kStageBytes = 2 * kHalf;          // one K or V tile: 32 KB
constexpr int kStages = 6;
constexpr int kNS = 16;                         // N of the score MMA
constexpr int kQBytes = 2 * kNS * 128;          // Q operand: 2 d-halves x 16 rows x 128 B
constexpr int kThreads = 192;
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr int kTmemCols = 128;
constexpr int kMaxUnits = 512;                  // work units one CTA can hold in its list
constexpr int kScanChunk = 4096;                // sequences scanned per pass (stage 0 as scratch)

template <int G> struct TcShape {
  static constexpr int NO = ((2 * G + 15) / 16) * 16;      // N of the PV MMA
  static constexpr int kPBytes = NO * 2 * 128;               // per tile: 2 token-halves
  static constexpr int OFF_Q = kStages * kStageBytes;
  static constexpr int OFF_P = OFF_Q + 2 * kQBytes;
  static constexpr int OFF_BAR = OFF_P + 2 * kPBytes;
  static constexpr int NBAR = 2 * kStages + 15;
  static constexpr int OFF_RED = OFF_BAR + 8 * NBAR;
  static constexpr int OFF_REDL = OFF_RED + 2 * 4 * 16 * 4;
  static constexpr int OFF_REC = (OFF_REDL + 4 * 16 * 4 + 15) / 16 * 16;
  static constexpr int OFF_MISC = OFF_REC + kMaxUnits * 16;
  static constexpr int BYTES = OFF_MISC + 32;
  static constexpr int SMEM = BYTES + 1024;                  // + alignment slack
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

// barrier indices
constexpr int B_FULL = 0, B_EMPTY = kStages, B_QFULL = 2 * kStages, B_QEMPTY = B_QFULL + 2,
              B_SFULL = B_QEMPTY + 2, B_SFREE = B_SFULL + 2, B_PREADY = B_SFREE + 2,
              B_OFULL = B_PREADY + 2, B_OFREE = B_OFULL + 2, B_DONE = B_OFREE + 2;

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for the phase with the given parity; false = gave up (timeout or abort).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          volatile uint32_t* abort_flag) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kWaitNs) return false;
  }
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, int c3, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}
// Shared-memory matrix descriptor, 128-byte swizzle (tcgen05 format: version 1 at bit 46).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor of kind::f16 with fp32 accumulation.
__host__ __device__ constexpr uint32_t make_idesc(int fmt, int a_mn, int b_mn, int N, int M) {
  return (1u << 4) | ((uint32_t)fmt << 7) | ((uint32_t)fmt << 10) | ((uint32_t)a_mn << 15) |
         ((uint32_t)b_mn << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void mma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p; setp.ne.u32 p, %4, 0;"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
// 16 consecutive fp32 columns of this thread's TMEM lane; waits for the load.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  __syncwarp();
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15},"
      " [%16];\n\ttcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
// Vote over the 128 softmax threads (named barrier 1): OR of every thread's flag.
__device__ __forceinline__ bool wg_vote_or(bool x) {
  uint32_t r;
  asm volatile(
      "{ .reg .pred pi, po; setp.ne.u32 pi, %1, 0; bar.red.or.pred po, 1, 128, pi;"
      " selp.u32 %0, 1, 0, po; }"
      : "=r"(r)
      : "r"((uint32_t)x)
      : "memory");
  return r != 0;
}

template <int FMT> __device__ __forceinline__ void split_16(float p, uint16_t& hi, uint16_t& lo) {
  if (FMT == 1) {
    __nv_bfloat16 h = __float2bfloat16_rn(p);
    __nv_bfloat16 l = __float2bfloat16_rn(p - __bfloat162float(h));
    hi = __bfloat16_as_ushort(h);
    lo = __bfloat16_as_ushort(l);
  } else {
    __half h = __float2half_rn(p);
    __half l = __float2half_rn(p - __half2float(h));
    hi = __half_as_ushort(h);
    lo = __half_as_ushort(l);
  }
}

// ---------------------------------------------------------------- work units
// A unit is (sequence b, KV head h, partition j). Units exist only for
// partitions that hold tokens; they are numbered sequence by sequence
// (k = (units before b) * Hkv + j * Hkv + h) and CTA c takes k = c, c + grid,
// ... Every CTA builds its own list at start, in shared memory, so the roles
// never touch global memory to find their next unit.
struct __align__(16) URec {
  int b, h, j, ctx;
};

struct Unit {
  int b, h, j, ctx, t0, t1, ntiles, nparts;
};

__device__ __forceinline__ Unit unit_from(const URec& r, int psize) {
  Unit x;
  x.b = r.b; x.h = r.h; x.j = r.j; x.ctx = r.ctx;
  x.t0 = r.j * psize;
  x.t1 = min(r.ctx, x.t0 + psize);
  x.ntiles = (x.t1 - x.t0 + kTile - 1) / kTile;
  x.nparts = (r.ctx + psize - 1) / psize;
  return x;
}

// Build this CTA's unit list (128 threads of warps 0-3). Sequences with no
// tokens (or a context length the table cannot hold) get no units; their
// output rows are zeroed here by the CTA that owns them.
template <int BS>
__device__ void build_unit_list(const DecodeArgs& a, uint8_t* scratch, URec* recs, int* carry_s,
                                int* wsum, int* my_units) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int* np_s = reinterpret_cast<int*>(scratch);
  int* ctx_s = np_s + kScanChunk;
  constexpr int PER = kScanChunk / 128;
  if (tid == 0) *carry_s = 0;
  asm volatile("bar.sync 1, 128;" ::: "memory");
  for (int b0 = 0; b0 < a.B; b0 += kScanChunk) {
    const int n = min(kScanChunk, a.B - b0);
    for (int i = tid; i < kScanChunk; i += 128) {
      int np = 0, ctx = 0;
      if (i < n) {
        ctx = __ldg(a.context_lens + b0 + i);
        const bool bad = ctx < 0 || ctx > a.max_blocks * BS || ctx > a.max_context_len;
        np = (bad || ctx == 0) ? 0 : (ctx + a.psize - 1) / a.psize;
        if (bad && ((b0 + i) % (int)gridDim.x) == (int)blockIdx.x) flag_error(a.err_flag, PA_DEV_BAD_CTX);
      }
      np_s[i] = np;
      ctx_s[i] = ctx;
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    int sum = 0;
    for (int e = 0; e < PER; ++e) sum += np_s[tid * PER + e];
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) wsum[warp] = incl;
    asm volatile("bar.sync 1, 128;" ::: "memory");
    int wpre = 0;
    for (int w = 0; w < warp; ++w) wpre += wsum[w];
    const int base = *carry_s;
    int pre = base + wpre + incl - sum;                 // partitions before my first sequence
    for (int e = 0; e < PER; ++e) {
      const int li = tid * PER + e, np = np_s[li];
      if (np > 0) {
        const long long start = (long long)pre * a.Hkv, end = start + (long long)np * a.Hkv;
        long long k = start + (((long long)blockIdx.x - start % gridDim.x) + gridDim.x) % gridDim.x;
        for (; k < end; k += gridDim.x) {
          const int idx = (int)((k - blockIdx.x) / gridDim.x);
          const int local = (int)(k - start);
          if (idx < kMaxUnits) recs[idx] = URec{b0 + li, local % a.Hkv, local / a.Hkv, ctx_s[li]};
        }
      }
      pre += np;
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    // zero the output rows of empty / bad sequences this CTA owns
    for (int li = 0; li < n; ++li) {
      const int b = b0 + li;
      if (np_s[li] != 0 || (b % (int)gridDim.x) != (int)blockIdx.x) continue;
      for (int i = tid; i < a.Hq * kD; i += 128)
        store_out(a.out, (size_t)b * a.Hq * kD + i, 0.f, a.out_dtype);
    }
    if (tid == 127) *carry_s = pre;
    asm volatile("bar.sync 1, 128;" ::: "memory");
  }
  if (tid == 0) {
    const long long U = (long long)(*carry_s) * a.Hkv;
    const long long mine = U > blockIdx.x ? (U - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    *my_units = (int)(mine < kMaxUnits ? mine : kMaxUnits);
  }
}

template <int FMT, int BS, int G>
__global__ void __launch_bounds__(kThreads, 1)
decode_tc_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmQ) {
  using S = TcShape<G>;
  constexpr int NO = S::NO;
  constexpr uint32_t IDESC_S = make_idesc(FMT, 0, 0, kNS, 128);
  constexpr uint32_t IDESC_O = make_idesc(FMT, 1, 0, NO, 128);
  constexpr int BPT = kTile / BS;                       // physical blocks per tile

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + S::OFF_BAR;
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  float* red = reinterpret_cast<float*>(smem + S::OFF_RED);     // [2][4][16]
  float* red_l = reinterpret_cast<float*>(smem + S::OFF_REDL);  // [4][16]
  const URec* recs = reinterpret_cast<const URec*>(smem + S::OFF_REC);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::OFF_MISC);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + S::OFF_MISC + 4);
  int* my_units_s = reinterpret_cast<int*>(smem + S::OFF_MISC + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(B_FULL + s), 1);
      mbar_init(bar(B_EMPTY + s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(B_QFULL + i), 1);
      mbar_init(bar(B_QEMPTY + i), 1);
      mbar_init(bar(B_SFULL + i), 1);
      mbar_init(bar(B_SFREE + i), 128);
      mbar_init(bar(B_PREADY + i), 128);
      mbar_init(bar(B_OFULL + i), 1);
      mbar_init(bar(B_OFREE + i), 128);
    }
    mbar_init(bar(B_DONE), 1);
    *abort_flag = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp < 4) {
    build_unit_list<BS>(a, smem, const_cast<URec*>(recs), reinterpret_cast<int*>(smem + S::OFF_MISC + 12),
                        reinterpret_cast<int*>(smem + S::OFF_MISC + 16), my_units_s);
    fence_proxy_async();                 // stage 0 served as scratch; TMA writes it next
  } else if (warp == 4) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_s = tmem;                 // S buffers: columns [0,16) and [16,32)
  const uint32_t tmem_o = tmem + 2 * kNS;       // O buffers: [32, 32+NO) and [32+NO, 32+2NO)
  const int nu = *my_units_s;
  auto give_up = [&]() {
    *abort_flag = 1u;
    flag_error(a.err_flag, PA_DEV_TIMEOUT);
  };

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int tc = 0, issued = 0;
      int phys_next[BPT];
      // block ids of tile k of unit i, loaded one tile ahead of their use
      auto load_ids = [&](int i, int k, int* ph) {
        const Unit x = unit_from(recs[i], a.psize);
        const int ts = x.t0 + k * kTile, te = min(x.t1, ts + kTile);
        const int nb = (te - ts + BS - 1) / BS;
        const int32_t* table = a.block_tables + (size_t)x.b * a.max_blocks + ts / BS;
#pragma unroll
        for (int q = 0; q < BPT; ++q) ph[q] = q < nb ? __ldg(table + q) : -1;
      };
      if (nu > 0) load_ids(0, 0, phys_next);
      for (int i = 0; i < nu; ++i) {
        const Unit x = unit_from(recs[i], a.psize);
        const int qi = i & 1;
        if (!mbar_wait(bar(B_QEMPTY + qi), ((i >> 1) & 1) ^ 1, abort_flag)) { give_up(); goto prod_done; }
        mbar_expect_tx(bar(B_QFULL + qi), 2u * G * 128u);
        for (int hh = 0; hh < 2; ++hh)
          tma_load_2d(sbase + S::OFF_Q + qi * kQBytes + hh * (kNS * 128), &tmQ, hh * 64,
                      x.b * a.Hq + x.h * G, bar(B_QFULL + qi));
        for (int k = 0; k < x.ntiles; ++k) {
          int phys[BPT];
          uint32_t bytes = 0;
#pragma unroll
          for (int q = 0; q < BPT; ++q) {
            phys[q] = phys_next[q];
            if (phys[q] >= 0 && phys[q] < a.num_blocks) bytes += 2u * BS * 128u;
          }
          if (k + 1 < x.ntiles) load_ids(i, k + 1, phys_next);
          else if (i + 1 < nu) load_ids(i + 1, 0, phys_next);
          for (int kv = 0; kv < 2; ++kv) {
            const int seq = 2 * tc + kv, s = seq % kStages;
            if (!mbar_wait(bar(B_EMPTY + s), ((seq / kStages) & 1) ^ 1, abort_flag)) { give_up(); goto prod_done; }
            mbar_expect_tx(bar(B_FULL + s), bytes);
            const uint32_t dst = sbase + s * kStageBytes;
#pragma unroll
            for (int q = 0; q < BPT; ++q) {
              if (phys[q] < 0 || phys[q] >= a.num_blocks) continue;
              for (int hh = 0; hh < 2; ++hh)
                tma_load_4d(dst + hh * kHalf + q * BS * 128, kv ? &tmV : &tmK, hh * 64, x.h, 0,
                            phys[q], bar(B_FULL + s));
            }
            ++issued;
          }
          ++tc;
        }
      }
    prod_done:
      // never leave with copies in flight: wait (bounded) for the last loads of every stage
      for (int seq = max(0, issued - kStages); seq < issued; ++seq) {
        const int s = seq % kStages;
        const uint64_t t0 = globaltimer();
        while (!mbar_try(bar(B_FULL + s), (seq / kStages) & 1) && globaltimer() - t0 < kWaitNs) {}
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int tc = 0;
      bool ok = true;
      auto issue_pv = [&](int tt, int nb) -> bool {
        const int pb = tt & 1;
        if (!mbar_wait(bar(B_PREADY + pb), (tt >> 1) & 1, abort_flag)) return false;
        if (!mbar_wait(bar(B_OFREE + pb), ((tt >> 1) & 1) ^ 1, abort_flag)) return false;
        const int seq = 2 * tt + 1, s = seq % kStages;
        if (!mbar_wait(bar(B_FULL + s), (seq / kStages) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t vst = sbase + s * kStageBytes;
        const uint32_t pst = sbase + S::OFF_P + pb * S::kPBytes;
        const int nsteps = nb * BS / 16;
        for (int ks = 0; ks < nsteps; ++ks) {
          // A = V^T, MN-major: 16 token rows (2 KB) per K step, d-halves 16 KB apart
          const uint64_t ad = sw128_desc(vst + ks * 2048, kHalf, 1024);
          // B = [P_hi; P_lo], K-major: token-halves NO*128 B apart, 32 B per K step
          const uint64_t bd = sw128_desc(pst + (ks >> 2) * (NO * 128) + (ks & 3) * 32, 16, 1024);
          mma_f16(tmem_o + pb * NO, ad, bd, IDESC_O, ks > 0 ? 1u : 0u);
        }
        mma_commit(bar(B_EMPTY + s));
        mma_commit(bar(B_OFULL + pb));
        return true;
      };
      for (int i = 0; i < nu && ok; ++i) {
        const Unit x = unit_from(recs[i], a.psize);
        const int qi = i & 1;
        if (!mbar_wait(bar(B_QFULL + qi), (i >> 1) & 1, abort_flag)) { ok = false; break; }
        const uint32_t qst = sbase + S::OFF_Q + qi * kQBytes;
        int prev_nb = 0;
        for (int k = 0; k < x.ntiles; ++k) {
          const int ts = x.t0 + k * kTile, te = min(x.t1, ts + kTile);
          const int sb = tc & 1;
          if (!mbar_wait(bar(B_SFREE + sb), ((tc >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
          const int seq = 2 * tc, s = seq % kStages;
          if (!mbar_wait(bar(B_FULL + s), (seq / kStages) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t kst = sbase + s * kStageBytes;
#pragma unroll
          for (int ks = 0; ks < kD / 16; ++ks) {
            const uint64_t ad = sw128_desc(kst + (ks >> 2) * kHalf + (ks & 3) * 32, 16, 1024);
            const uint64_t bd = sw128_desc(qst + (ks >> 2) * (kNS * 128) + (ks & 3) * 32, 16, 1024);
            mma_f16(tmem_s + sb * kNS, ad, bd, IDESC_S, ks > 0 ? 1u : 0u);
          }
          mma_commit(bar(B_EMPTY + s));
          mma_commit(bar(B_SFULL + sb));
          if (k == x.ntiles - 1) mma_commit(bar(B_QEMPTY + qi));
          if (k > 0 && !issue_pv(tc - 1, prev_nb)) { ok = false; break; }
          prev_nb = (te - ts + BS - 1) / BS;
          ++tc;
        }
        if (!ok) break;
        if (!issue_pv(tc - 1, prev_nb)) { ok = false; break; }
      }
      if (!ok) give_up();
      // all issued MMAs must finish before tensor memory is released
      mma_commit(bar(B_DONE));
      const uint64_t t0 = globaltimer();
      while (!mbar_try(bar(B_DONE), 0) && globaltimer() - t0 < kWaitNs) {}
    }
  } else {
    // ------------------------------------------------------------ softmax / output warps
    const int row = threadIdx.x;                   // token row of S, d row of O
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
    int tc = 0;
    bool failed = false;
    // this thread's block id for tile k of unit i (its token row), one tile ahead
    auto row_id = [&](int i, int k) -> int {
      const Unit x = unit_from(recs[i], a.psize);
      const int ts = x.t0 + k * kTile, te = min(x.t1, ts + kTile);
      const int nb = (te - ts + BS - 1) / BS;
      return row < nb * BS ? __ldg(a.block_tables + (size_t)x.b * a.max_blocks + ts / BS + row / BS)
                           : -1;
    };
    int phys_next = nu > 0 ? row_id(0, 0) : -1;
    for (int i = 0; i < nu; ++i) {
      const Unit x = unit_from(recs[i], a.psize);
      float m[G], l[G], O[G], al_prev[G], al[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        m[g] = -CUDART_INF_F; l[g] = 0.f; O[g] = 0.f; al_prev[g] = 0.f;
      }
      auto accumulate = [&](int tt, const float* alpha) {
        const int pb = tt & 1;
        if (!mbar_wait(bar(B_OFULL + pb), (tt >> 1) & 1, abort_flag)) failed = true;
        tc_fence_after();
        float o[NO];
#pragma unroll
        for (int c = 0; c < NO; c += 16) tmem_ld16(tmem_o + lane_off + pb * NO + c, o + c);
        tc_fence_before();
        mbar_arrive(bar(B_OFREE + pb));
#pragma unroll
        for (int g = 0; g < G; ++g) O[g] = fmaf(O[g], alpha[g], o[g] + o[G + g]);
      };
      bool stop = false;
      for (int k = 0; k < x.ntiles; ++k) {
        const int ts = x.t0 + k * kTile, te = min(x.t1, ts + kTile);
        const int nb = (te - ts + BS - 1) / BS;
        const bool in_range = row < nb * BS;
        const int phys = phys_next;
        if (k + 1 < x.ntiles) phys_next = row_id(i, k + 1);
        else if (i + 1 < nu) phys_next = row_id(i + 1, 0);
        const bool blk_ok = phys >= 0 && phys < a.num_blocks;
        const bool valid = in_range && blk_ok && ts + row < te;
        if (in_range && !blk_ok && (row % BS) == 0) flag_error(a.err_flag, PA_DEV_BAD_BLOCK_ID);

        const int sb = tc & 1;
        if (!mbar_wait(bar(B_SFULL + sb), (tc >> 1) & 1, abort_flag)) failed = true;
        tc_fence_after();
        float s[16];
        tmem_ld16(tmem_s + lane_off + sb * kNS, s);
        tc_fence_before();
        mbar_arrive(bar(B_SFREE + sb));

        float* rb = red + (tc & 1) * 64;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          s[g] = valid ? s[g] * a.scale_log2 : -CUDART_INF_F;
          float v = s[g];
#pragma unroll
          for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
          if (lane == 0) rb[warp * 16 + g] = v;
        }
        if (wg_vote_or(failed)) { stop = true; break; }
        const int pb = tc & 1;
        uint8_t* pbase = smem + S::OFF_P + pb * S::kPBytes + (row >> 6) * (NO * 128);
        const int chunk = (row & 63) >> 3, e = row & 7;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float tmax = fmaxf(fmaxf(rb[g], rb[16 + g]), fmaxf(rb[32 + g], rb[48 + g]));
          const float m_new = fmaxf(m[g], tmax);
          al[g] = m_new == -CUDART_INF_F ? 1.f : exp2f(m[g] - m_new);
          const float p = valid ? exp2f(s[g] - m_new) : 0.f;
          l[g] = fmaf(l[g], al[g], p);
          m[g] = m_new;
          uint16_t hi, lo;
          split_16<FMT>(p, hi, lo);
          *reinterpret_cast<uint16_t*>(pbase + g * 128 + ((chunk ^ (g & 7)) << 4) + e * 2) = hi;
          *reinterpret_cast<uint16_t*>(pbase + (G + g) * 128 + (((chunk ^ ((G + g) & 7))) << 4) + e * 2) = lo;
        }
        if (in_range && !valid) {
          // this V row enters the PV product with weight 0: it must hold finite values
          const int seq = 2 * tc + 1, sv = seq % kStages;
          if (!mbar_wait(bar(B_FULL + sv), (seq / kStages) & 1, abort_flag)) failed = true;
          uint4* r0 = reinterpret_cast<uint4*>(smem + sv * kStageBytes + row * 128);
          uint4* r1 = reinterpret_cast<uint4*>(smem + sv * kStageBytes + kHalf + row * 128);
#pragma unroll
          for (int c = 0; c < 8; ++c) { r0[c] = make_uint4(0, 0, 0, 0); r1[c] = make_uint4(0, 0, 0, 0); }
        }
        fence_proxy_async();
        mbar_arrive(bar(B_PREADY + pb));
        if (k > 0) accumulate(tc - 1, al_prev);
#pragma unroll
        for (int g = 0; g < G; ++g) al_prev[g] = al[g];
        ++tc;
      }
      if (stop) break;
      accumulate(tc - 1, al_prev);

      // epilogue: total exp-sum per head, then the unit's output rows
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float v = l[g];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red_l[warp * 16 + g] = v;
      }
      if (wg_vote_or(failed)) break;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float L = red_l[g] + red_l[16 + g] + red_l[32 + g] + red_l[48 + g];
        const size_t orow = (size_t)x.b * a.Hq + x.h * G + g;
        if (x.nparts == 1) {
          store_out(a.out, orow * kD + row, L > 0.f ? O[g] / L : 0.f, a.out_dtype);
        } else {
          const size_t pj = orow * a.P + x.j;
          a.ws_acc[pj * kD + row] = O[g];
          if (row == 0) { a.ws_m[pj] = m[g]; a.ws_l[pj] = L; }
        }
      }
    }
    if (failed) give_up();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
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
  const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)a.Hkv, (cuuint64_t)a.bs,
                              (cuuint64_t)a.num_blocks};
  const cuuint64_t strides[3] = {(cuuint64_t)kD * 2, (cuuint64_t)a.Hkv * kD * 2,
                                 (cuuint64_t)a.bs * a.Hkv * kD * 2};
  const cuuint32_t box[4] = {64, 1, (cuuint32_t)a.bs, 1};
  const cuuint32_t es[4] = {1, 1, 1, 1};
  for (int i = 0; i < 2; ++i) {
    CUresult r = enc(i == 0 ? k : v, dt, 4, const_cast<void*>(i == 0 ? a.k_cache : a.v_cache), dims,
                     strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
  }
  const cuuint64_t qdims[2] = {(cuuint64_t)kD, (cuuint64_t)a.B * a.Hq};
  const cuuint64_t qstr[1] = {(cuuint64_t)kD * 2};
  const cuuint32_t qbox[2] = {64, (cuuint32_t)G};
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
  // Units that hold tokens number at most B * Hkv * P; a CTA's list holds kMaxUnits.
  const long long units = (long long)a.B * a.Hkv * a.P;
  if (units <= 0) return PA_OK;
  long long grid = units < sm_count() ? units : sm_count();
  if ((units + grid - 1) / grid > kMaxUnits) grid = (units + kMaxUnits - 1) / kMaxUnits;
  if (grid > 0x7fffffffLL) return PA_ERR_UNSUPPORTED;
  kern<<<(unsigned)grid, kThreads, smem, stream>>>(a, k, v, q);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

template <int FMT, int BS>
int launch_tc_g(const DecodeArgs& a, const CUtensorMap& k, const CUtensorMap& v,
                const CUtensorMap& q, cudaStream_t stream) {
  switch (a.Hq / a.Hkv) {
    case 4: return launch_tc_t<FMT, BS, 4>(a, k, v, q, stream);
    case 8: return launch_tc_t<FMT, BS, 8>(a, k, v, q, stream);
    case 16: return launch_tc_t<FMT, BS, 16>(a, k, v, q, stream);
  }
  return PA_ERR_UNSUPPORTED;
}

}  // namespace

bool tc_supported(int dtype, int Hq, int Hkv, int D, int bs) {
  if (dtype != PA_F16 && dtype != PA_BF16) return false;
  if (D != kD || (bs != 16 && bs != 32) || Hkv <= 0 || Hq % Hkv) return false;
  const int G = Hq / Hkv;
  return G == 4 || G == 8 || G == 16;
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
