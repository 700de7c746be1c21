// decode_simt.cu -- paged decode attention on the CUDA cores.
//
// One CTA = one (partition j, KV head h, chunk of GC query heads, sequence b).
// Its four warps walk the partition's tokens in tiles; a tile is TILE rows of
// one physical block (the whole block for 16-bit D=128, half of it for fp32
// D=128). For every tile a warp
//   1. reads the physical block id from the block table (prefetched one tile
//      ahead, so the table read is off the critical path),
//   2. issues all of the tile's K and V row loads at once: 16-byte vectors,
//      LPR lanes per row, RPI rows per warp instruction, so each row is one
//      fully used, contiguous 128 / 256-byte segment,
//   3. forms the GC scores of each row as fp32 partial dots reduced over the
//      row's LPR lanes with xor shuffles,
//   4. applies the online-softmax update (running max m, running sum l,
//      rescale by exp2(m_old - m_new)) and accumulates p * V in fp32.
// Rows past the context length are never loaded and never enter the sums (a
// select, not a multiply by zero, because unused slots may hold NaN).
// At the end the four warps' (m, l, acc) are merged through shared memory.
// A sequence whose context fits in one partition is written to the output
// directly; otherwise the partition's (m, l, acc) go to the workspace and the
// merge kernel combines them.
//
// The pages describe this kernel only as FlashAttention changed to read
// non-contiguous blocks ("vLLM 与 LLM 推理部署实战", section 2.3) and list
// block prefetch, shared-memory reuse and asynchronous copies as its
// optimisations ("vLLM与PagedAttention：大模型推理内存优化技术解析", section
// 3.2); the tiling and vector layout here are this library's own.
#include <math_constants.h>

#include <cstdlib>

#include "pa_internal.h"

namespace pa {

namespace {

constexpr int kWarps = 4;

// Packed fp32x2 FMA (two lanes of fp32 per instruction on sm_100).
__device__ __forceinline__ void fma2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  uint64_t d = (uint64_t)__float_as_uint(d0) | ((uint64_t)__float_as_uint(d1) << 32);
  const uint64_t a = (uint64_t)__float_as_uint(a0) | ((uint64_t)__float_as_uint(a1) << 32);
  const uint64_t b = (uint64_t)__float_as_uint(b0) | ((uint64_t)__float_as_uint(b1) << 32);
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(d) : "l"(a), "l"(b));
  d0 = __uint_as_float((uint32_t)d);
  d1 = __uint_as_float((uint32_t)(d >> 32));
}

// VEC consecutive query elements of type TQ, widened to fp32 (16-byte loads).
template <typename TQ, int VEC>
__device__ __forceinline__ void load_q(const TQ* p, float* f) {
  constexpr int N = Vec<TQ>::N;
  static_assert(VEC % N == 0, "query chunk");
#pragma unroll
  for (int c = 0; c < VEC / N; ++c) widen16<TQ>(*reinterpret_cast<const uint4*>(p + c * N), f + c * N);
}

// TQ: query element type; TK, TV: K and V pool element types (TQ, or FP8
// E4M3 codes; the two may differ); PF: issue the loads of each warp's next
// tile before computing the current one.
template <typename TQ, typename TK, typename TV, int D, int BS, int GC, bool PF>
__global__ void __launch_bounds__(kWarps * 32)
decode_simt_kernel(const DecodeArgs a) {
  // elements per lane and row: a 16-byte slice of the wider pool's row (the
  // narrower pool's slice is then 8 bytes)
  constexpr int ESZ = sizeof(TK) > sizeof(TV) ? sizeof(TK) : sizeof(TV);
  constexpr int VEC = 16 / ESZ;
  constexpr int NBK = VEC * sizeof(TK), NBV = VEC * sizeof(TV);
  using RK = typename Raw<NBK>::T;
  using RV = typename Raw<NBV>::T;
  constexpr int LPR = D / VEC;                 // lanes per K/V row: 4, 8, 16 or 32
  constexpr int RPI = 32 / LPR;                // rows per warp instruction: 8, 4, 2 or 1
  constexpr int RGMAX = VEC == 16 ? 4 : 8;     // registers: 16 floats per slice for FP8 pools
  constexpr int RG = (BS / RPI) < RGMAX ? (BS / RPI) : RGMAX;   // row groups per tile
  constexpr int TILE = RG * RPI;               // tokens per tile (divides BS)
  static_assert(BS % TILE == 0, "tile must divide the block");

  __shared__ float sm_acc[kWarps][GC][D];
  __shared__ float sm_m[kWarps][GC];
  __shared__ float sm_l[kWarps][GC];
  pdl_trigger();
  pdl_wait();

  const int G = a.Hq / a.Hkv;
  const int chunks = G / GC;
  const int j = blockIdx.x / chunks;
  const int chunk = blockIdx.x - j * chunks;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int hq0 = h * G + chunk * GC;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int ctx = a.context_lens[b];
  const int start = a.start_blocks ? a.start_blocks[b] * BS : 0;   // first token of this pass
  const bool bad_ctx = ctx < 0 || ctx > a.max_blocks * BS || ctx > a.max_context_len ||
                       start < 0 || start > ctx;
  const int tok_begin = start + j * a.psize;
  if (bad_ctx || ctx == start) {
    // zero rows, written once (by partition 0); the merge kernel skips them
    // (in the split-only pass the merge writes every row)
    if (j == 0) {
      if (bad_ctx && threadIdx.x == 0 && chunk == 0 && h == 0) flag_error(a.err_flag, PA_DEV_BAD_CTX);
      if (!a.force_split)
        for (int i = threadIdx.x; i < GC * D; i += blockDim.x)
          store_out(a.out, ((size_t)b * a.Hq + hq0 + i / D) * D + i % D, 0.f, a.out_dtype);
    }
    return;
  }
  if (tok_begin >= ctx) return;                 // partition past this sequence's end
  const int tok_end = min(ctx, tok_begin + a.psize);
  const int nparts = (ctx - start + a.psize - 1) / a.psize;

  // query vectors of this chunk, pre-scaled so scores come out as scale*log2(e)*q.k
  const int ci = lane % LPR;                    // which 16-byte vector of a row
  const int rs = lane / LPR;                    // which row of an RPI-row group
  float qf[GC][VEC];
#pragma unroll
  for (int g = 0; g < GC; ++g) {
    load_q<TQ, VEC>(reinterpret_cast<const TQ*>(a.q) + ((size_t)b * a.Hq + hq0 + g) * D + ci * VEC,
                    qf[g]);
#pragma unroll
    for (int e = 0; e < VEC; ++e) qf[g][e] *= a.scale_log2;
  }

  float m[GC], l[GC], acc[GC][VEC];
#pragma unroll
  for (int g = 0; g < GC; ++g) {
    m[g] = -CUDART_INF_F;
    l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[g][e] = 0.f;
  }

  const int32_t* table = a.block_tables + (size_t)b * a.max_blocks;
  const TK* kc = reinterpret_cast<const TK*>(a.k_cache);
  const TV* vc = reinterpret_cast<const TV*>(a.v_cache);
  const size_t row_stride = (size_t)a.Hkv * D;          // elements between token rows
  const int tile_begin = tok_begin / TILE;
  const int tile_end = (tok_end + TILE - 1) / TILE;

  // rows of tile tt of block ph into k / v (zeros past the context or for a bad block)
  auto issue = [&](int tt, int ph, RK* k, RV* v) {
    const int token0 = tt * TILE;
    const bool ok = ph >= 0 && ph < a.num_blocks;
    const size_t base =
        ((size_t)(ok ? ph : 0) * BS + (token0 % BS)) * row_stride + (size_t)h * D + ci * VEC;
#pragma unroll
    for (int r = 0; r < RG; ++r) {
      const int row = r * RPI + rs;
      if (ok && token0 + row < tok_end) {
        k[r] = ld_stream<NBK>(kc + base + row * row_stride);
        v[r] = ld_stream<NBV>(vc + base + row * row_stride);
      } else {
        k[r] = raw_zero<NBK>();
        v[r] = raw_zero<NBV>();
      }
    }
  };
  // scores, online softmax and P.V of tile tt
  auto consume = [&](int tt, const RK* kr, const RV* vr) {
    const int token0 = tt * TILE;
    // scores of the lane's RG rows, reduced over the row's LPR lanes
    float s[RG][GC];
#pragma unroll
    for (int r = 0; r < RG; ++r) {
      float kf[VEC];
      widen_raw<TK, VEC>(kr[r], kf);
#pragma unroll
      for (int g = 0; g < GC; ++g) {
        if constexpr (VEC == 16) {
          // FP8 rows carry twice the elements per byte: packed FMAs halve the issue
          float d0 = 0.f, d1 = 0.f;
#pragma unroll
          for (int e = 0; e < VEC; e += 2) fma2(d0, d1, qf[g][e], qf[g][e + 1], kf[e], kf[e + 1]);
          s[r][g] = d0 + d1;
        } else {
          float d0 = 0.f;
#pragma unroll
          for (int e = 0; e < VEC; ++e) d0 = fmaf(qf[g][e], kf[e], d0);
          s[r][g] = d0;
        }
      }
    }
#pragma unroll
    for (int o = LPR / 2; o >= 1; o >>= 1)
#pragma unroll
      for (int r = 0; r < RG; ++r)
#pragma unroll
        for (int g = 0; g < GC; ++g) s[r][g] += __shfl_xor_sync(0xffffffffu, s[r][g], o);

    // online softmax over the tile (max over all TILE rows of the warp)
#pragma unroll
    for (int g = 0; g < GC; ++g) {
      float tmax = -CUDART_INF_F;
#pragma unroll
      for (int r = 0; r < RG; ++r)
        if (token0 + r * RPI + rs < tok_end) tmax = fmaxf(tmax, s[r][g]);
#pragma unroll
      for (int o = LPR; o < 32; o <<= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
      const float m_new = fmaxf(m[g], tmax);
      const float alpha = exp2f(m[g] - m_new);
      m[g] = m_new;
      l[g] *= alpha;
#pragma unroll
      for (int e = 0; e < VEC; ++e) acc[g][e] *= alpha;
#pragma unroll
      for (int r = 0; r < RG; ++r) {
        const bool valid = token0 + r * RPI + rs < tok_end;
        s[r][g] = valid ? exp2f(s[r][g] - m_new) : 0.f;
        l[g] += s[r][g];
      }
    }
#pragma unroll
    for (int r = 0; r < RG; ++r) {
      float vf[VEC];
      widen_raw<TV, VEC>(vr[r], vf);
#pragma unroll
      for (int g = 0; g < GC; ++g) {
        if constexpr (VEC == 16) {
#pragma unroll
          for (int e = 0; e < VEC; e += 2)
            fma2(acc[g][e], acc[g][e + 1], s[r][g], s[r][g], vf[e], vf[e + 1]);
        } else {
#pragma unroll
          for (int e = 0; e < VEC; ++e) acc[g][e] = fmaf(s[r][g], vf[e], acc[g][e]);
        }
      }
    }
  };
  auto block_of = [&](int tt) { return __ldg(table + (tt * TILE) / BS); };
  auto bad_block = [&](int ph) {
    if (ph < 0 || ph >= a.num_blocks) {
      if (lane == 0) flag_error(a.err_flag, PA_DEV_BAD_BLOCK_ID);
      return true;
    }
    return false;
  };

  int t = tile_begin + warp;
  if constexpr (PF) {
    // Loads of the warp's next tile are issued before this tile is computed, so
    // each warp always has a tile's K and V in flight (block ids two tiles ahead).
    RK kr[RG];
    RV vr[RG];
    int phys = t < tile_end ? block_of(t) : -1;
    int phys_n = t + kWarps < tile_end ? block_of(t + kWarps) : -1;
    if (t < tile_end) issue(t, phys, kr, vr);
    for (; t < tile_end; t += kWarps) {
      const int tn = t + kWarps;
      const int ph = phys;
      RK kn[RG];
      RV vn[RG];
      if (tn < tile_end) issue(tn, phys_n, kn, vn);
      phys = phys_n;
      phys_n = tn + kWarps < tile_end ? block_of(tn + kWarps) : -1;
      if (!bad_block(ph)) consume(t, kr, vr);
#pragma unroll
      for (int r = 0; r < RG; ++r) { kr[r] = kn[r]; vr[r] = vn[r]; }
    }
  } else {
    int phys_next = t < tile_end ? block_of(t) : 0;
    for (; t < tile_end; t += kWarps) {
      const int phys = phys_next;
      const int tn = t + kWarps;
      if (tn < tile_end) phys_next = block_of(tn);
      if (bad_block(phys)) continue;
      RK kr[RG];
      RV vr[RG];
      issue(t, phys, kr, vr);
      consume(t, kr, vr);
    }
  }

  // combine the RPI row slots of the warp (same vector index, different rows)
#pragma unroll
  for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
    for (int g = 0; g < GC; ++g) {
      l[g] += __shfl_xor_sync(0xffffffffu, l[g], o);
#pragma unroll
      for (int e = 0; e < VEC; ++e) acc[g][e] += __shfl_xor_sync(0xffffffffu, acc[g][e], o);
    }
  if (lane < LPR) {
#pragma unroll
    for (int g = 0; g < GC; ++g)
#pragma unroll
      for (int e = 0; e < VEC; ++e) sm_acc[warp][g][ci * VEC + e] = acc[g][e];
  }
  if (lane == 0) {
#pragma unroll
    for (int g = 0; g < GC; ++g) { sm_m[warp][g] = m[g]; sm_l[warp][g] = l[g]; }
  }
  __syncthreads();

  // merge the warps: M = max m_w, L = sum l_w 2^(m_w - M), O = sum acc_w 2^(m_w - M)
  for (int i = threadIdx.x; i < GC * D; i += blockDim.x) {
    const int g = i / D, d = i - g * D;
    float M = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm_m[w][g]);
    float L = 0.f, O = 0.f;
    if (M != -CUDART_INF_F) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float c = exp2f(sm_m[w][g] - M);
        L = fmaf(sm_l[w][g], c, L);
        O = fmaf(sm_acc[w][g][d], c, O);
      }
    }
    const size_t row = (size_t)b * a.Hq + hq0 + g;
    O *= a.v_scale;                              // 1 unless the V pool holds FP8 codes
    if (nparts == 1 && !a.force_split) {
      store_out(a.out, row * D + d, L > 0.f ? O / L : 0.f, a.out_dtype);
    } else {
      const size_t pj = ((size_t)b * a.P + a.slot_base + j) * a.Hq + hq0 + g;   // [B][P][Hq] slot
      a.ws_acc[pj * D + d] = O;
      if (d == 0) { a.ws_m[pj] = M; a.ws_l[pj] = L; }
    }
  }
}

// Prefetching the next tile (PF) keeps two tiles of loads in flight per warp:
// it pays where a warp's tile carries few bytes (FP8 pools: half the bytes of a
// 16-bit tile per load) and on the MHA shape (one query head per CTA), where
// the extra registers still leave enough warps per SM; PA_SIMT_PREFETCH=0/1
// overrides the choice, for measurements.
int prefetch_override() {
  const char* s = std::getenv("PA_SIMT_PREFETCH");
  if (!s || !*s) return -1;
  return s[0] == '1' ? 1 : 0;
}

template <typename TQ, typename TK, typename TV, int D, int BS, int GC>
int launch_t(const DecodeArgs& a, cudaStream_t stream) {
  const int chunks = (a.Hq / a.Hkv) / GC;
  dim3 grid((unsigned)(a.P * chunks), (unsigned)a.Hkv, (unsigned)a.B);
  const int ov = prefetch_override();
  // loads of the next tile issued before the current one is computed: the default
  // for one query head per CTA (MHA: the extra registers leave enough warps) and
  // for pools of codes (half the bytes per row, so a warp needs two tiles in flight)
  const bool pf = ov >= 0 ? ov == 1 : (GC == 1 || sizeof(TK) == 1 || sizeof(TV) == 1);
  const cudaError_t e =
      pf ? launch_k(decode_simt_kernel<TQ, TK, TV, D, BS, GC, true>, grid, dim3(kWarps * 32), 0,
                    stream, a)
         : launch_k(decode_simt_kernel<TQ, TK, TV, D, BS, GC, false>, grid, dim3(kWarps * 32), 0,
                    stream, a);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

template <typename TQ, typename TK, typename TV, int D, int BS>
int launch_gc(const DecodeArgs& a, cudaStream_t stream) {
  const int G = a.Hq / a.Hkv;
  if (G == 1) return launch_t<TQ, TK, TV, D, BS, 1>(a, stream);
  if constexpr (sizeof(TK) == 1 && sizeof(TV) == 1) {
    return launch_t<TQ, TK, TV, D, BS, 2>(a, stream);   // FP8: pairs of heads (registers)
  } else {
    if (G == 2) return launch_t<TQ, TK, TV, D, BS, 2>(a, stream);
    return launch_t<TQ, TK, TV, D, BS, 4>(a, stream);   // G = 4, 8, 16: chunks of 4 heads
  }
}

template <typename TQ, typename TK, typename TV, int D>
int launch_bs(const DecodeArgs& a, cudaStream_t stream) {
  return a.bs == 16 ? launch_gc<TQ, TK, TV, D, 16>(a, stream)
                    : launch_gc<TQ, TK, TV, D, 32>(a, stream);
}

template <typename TQ, typename TK, typename TV>
int launch_d(const DecodeArgs& a, cudaStream_t stream) {
  return a.D == 64 ? launch_bs<TQ, TK, TV, 64>(a, stream) : launch_bs<TQ, TK, TV, 128>(a, stream);
}

// Merge of the split pass, for each (b, hq) row with more than one partition:
// M = max_j m_j, L = sum_j l_j 2^(m_j - M), o = sum_j 2^(m_j - M) acc_j / L.
// NW warps share a row (NW = 4 when rows have many partitions, else 1); warp w
// takes partitions w, w + NW, ... Its lanes first find the maximum over the
// warp's partitions (one partition per lane), then each lane computes the
// weight of its partition and the warp streams the acc rows eight partitions
// at a time, so eight loads are in flight per lane. The NW warps of a row
// combine their (M, L, o) through shared memory.
template <int PER> struct VecF;
template <> struct VecF<4> { using T = float4; };
template <> struct VecF<2> { using T = float2; };

template <int D, int NW>
__global__ void __launch_bounds__(128) merge_kernel(const DecodeArgs a) {
  constexpr int PER = D / 32;                  // floats per lane: one 16- or 8-byte vector
  constexpr int RPB = 4 / NW;                  // rows per block
  using V = typename VecF<PER>::T;
  __shared__ float sm_m[NW], sm_l[NW];
  __shared__ float sm_o[NW][D];
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * RPB + warp / NW;
  const int sub = warp % NW;
  // the NW warps of a row take the same branch here (for NW > 1 the block is one row)
  if (row >= a.B * a.Hq) return;
  const int b = row / a.Hq, hq = row - b * a.Hq;
  // partials of (b, hq) sit at [B][P][Hq] slots: partition stride Hq
  const size_t base = (size_t)b * a.P * a.Hq + hq;
  const float* pm = a.ws_m + base;
  const float* pl = a.ws_l + base;
  // when one batch of lanes covers every partition of the grid (the usual
  // case), each lane loads its partition's m and l together with the context
  // length, and partitions past this row's end are masked once it is known
  const bool one = a.P <= 32 * NW;
  const int jl = sub + lane * NW;
  float M = -CUDART_INF_F, mj = -CUDART_INF_F, lj = 0.f;
  if (one && jl < a.P) { mj = pm[(size_t)jl * a.Hq]; lj = pl[(size_t)jl * a.Hq]; }
  const int ctx = a.context_lens[b];
  const int start = a.start_blocks ? a.start_blocks[b] * a.bs : 0;
  if (ctx < 0 || ctx > a.max_blocks * a.bs || ctx > a.max_context_len || start < 0 || start > ctx ||
      (!a.force_split && ctx == 0)) {
    if (a.force_split && sub == 0)                 // split-only pass: the merge owns every row
      for (int e = lane; e < D; e += 32) store_out(a.out, (size_t)row * D + e, 0.f, a.out_dtype);
    return;
  }
  // partitions of this row: slots [0, slot_base) hold earlier passes' partials
  // (the shared prefix), then ceil((ctx - start) / psize) of this pass
  const int nparts = a.slot_base + (ctx - start + a.psize - 1) / a.psize;
  if (nparts <= 1 && !a.force_split) return;
  if (one) {
    if (jl >= nparts) { mj = -CUDART_INF_F; lj = 0.f; }
    M = mj;
  } else {
    for (int jj = sub + lane * NW; jj < nparts; jj += 32 * NW) M = fmaxf(M, pm[(size_t)jj * a.Hq]);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float L = 0.f, O[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) O[e] = 0.f;
  if (M != -CUDART_INF_F) {                    // a warp with no partitions keeps M = -inf
    for (int j0 = sub; j0 < nparts; j0 += 32 * NW) {
      const int jl = j0 + lane * NW;           // this lane's partition of the batch
      float c = 0.f;
      if (jl < nparts) {
        c = exp2f((one ? mj : pm[(size_t)jl * a.Hq]) - M);
        L = fmaf(one ? lj : pl[(size_t)jl * a.Hq], c, L);
      }
      const int cnt = min(32, (nparts - j0 + NW - 1) / NW);
      for (int t0 = 0; t0 < cnt; t0 += 8) {
        V v[8];
        float ct[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          ct[u] = __shfl_sync(0xffffffffu, c, (t0 + u) & 31);
          if (t0 + u < cnt)
            v[u] = *reinterpret_cast<const V*>(
                a.ws_acc + (base + (size_t)(j0 + (t0 + u) * NW) * a.Hq) * D + lane * PER);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (t0 + u < cnt) {
            const float* f = reinterpret_cast<const float*>(&v[u]);
#pragma unroll
            for (int e = 0; e < PER; ++e) O[e] = fmaf(f[e], ct[u], O[e]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
  if (NW > 1) {
    if (lane == 0) { sm_m[sub] = M; sm_l[sub] = L; }
#pragma unroll
    for (int e = 0; e < PER; ++e) sm_o[sub][lane * PER + e] = O[e];
    __syncthreads();
    if (sub != 0) return;
    float Mx = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < NW; ++w) Mx = fmaxf(Mx, sm_m[w]);
    L = 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) O[e] = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float c = sm_m[w] == -CUDART_INF_F ? 0.f : exp2f(sm_m[w] - Mx);
      L = fmaf(sm_l[w], c, L);
#pragma unroll
      for (int e = 0; e < PER; ++e) O[e] = fmaf(sm_o[w][lane * PER + e], c, O[e]);
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
  for (int e = 0; e < PER; ++e) store_out(a.out, (size_t)row * D + lane * PER + e, O[e] * inv, a.out_dtype);
}

template <int D>
int launch_merge_d(const DecodeArgs& a, cudaStream_t stream) {
  const long long rows = (long long)a.B * a.Hq;
  if (a.P >= 16) {
    return launch_k(merge_kernel<D, 4>, dim3((unsigned)rows), dim3(128), 0, stream, a) ==
                   cudaSuccess ? PA_OK : PA_ERR_CUDA;
  }
  return launch_k(merge_kernel<D, 1>, dim3((unsigned)((rows + 3) / 4)), dim3(128), 0, stream, a) ==
                 cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace

int launch_decode_simt(const DecodeArgs& a, int dtype, cudaStream_t stream) {
  switch (dtype) {
    case PA_F32: return launch_d<float, float, float>(a, stream);
    case PA_F16: return launch_d<__half, __half, __half>(a, stream);
    case PA_BF16: return launch_d<__nv_bfloat16, __nv_bfloat16, __nv_bfloat16>(a, stream);
  }
  return PA_ERR_DTYPE;
}

// Pools of other types than the query's: both FP8 (any query type), or one FP8
// and the other of the query's 16-bit type.
int launch_decode_simt_kv(const DecodeArgs& a, int q_dtype, int k_dtype, int v_dtype,
                          cudaStream_t stream) {
  using F8 = __nv_fp8_e4m3;
  const bool kf = k_dtype == PA_FP8_E4M3, vf = v_dtype == PA_FP8_E4M3;
  if (kf && vf) {
    switch (q_dtype) {
      case PA_F32: return launch_d<float, F8, F8>(a, stream);
      case PA_F16: return launch_d<__half, F8, F8>(a, stream);
      case PA_BF16: return launch_d<__nv_bfloat16, F8, F8>(a, stream);
    }
    return PA_ERR_DTYPE;
  }
  if (q_dtype == PA_F16) {
    if (kf && v_dtype == PA_F16) return launch_d<__half, F8, __half>(a, stream);
    if (vf && k_dtype == PA_F16) return launch_d<__half, __half, F8>(a, stream);
  } else if (q_dtype == PA_BF16) {
    if (kf && v_dtype == PA_BF16) return launch_d<__nv_bfloat16, F8, __nv_bfloat16>(a, stream);
    if (vf && k_dtype == PA_BF16) return launch_d<__nv_bfloat16, __nv_bfloat16, F8>(a, stream);
  }
  if (!kf && !vf && k_dtype == q_dtype && v_dtype == q_dtype) return launch_decode_simt(a, q_dtype, stream);
  return PA_ERR_DTYPE;
}

int launch_merge(const DecodeArgs& a, cudaStream_t stream) {
  return a.D == 64 ? launch_merge_d<64>(a, stream) : launch_merge_d<128>(a, stream);
}

}  // namespace pa
