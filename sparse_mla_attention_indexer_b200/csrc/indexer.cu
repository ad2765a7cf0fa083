// DSA indexer scores over a paged FP8 indexer cache, on the sm_100a tensor cores.
//
// vLLM blog "vLLM 首日支持 Mistral Large 4", section "实现细节 / 模型架构":
// the sparse indexer reads an FP8 indexer cache and has its own SSMax; section
// "ROCm 实现细节": one FP8 scale per key, 132 B per token.  Score of query
// token t against cached token s < n_t:
//   I[t, s] = c_t * sq_t * sk_s * sum_h w[t, h] * ReLU(q8[t, h, :] . k8[s, :])
//
// Design (one persistent CTA per SM, warp-specialised):
//   * a work item is (request, query group of <= 4 tokens, 128-token tile);
//     items are counted on the device from cu_q / ctx_len (one round of
//     parallel loads per 192 requests) and split evenly over the CTAs, so the
//     host never reads device data;
//   * warp 0 moves the tile's two 64-token key pages into shared memory with
//     3-D TMA loads (128-B swizzle) over the paged pool, and the pages'
//     per-token scales with plain bulk copies, into a 9-stage ring;
//   * warp 1 issues tcgen05.mma kind::f8f6f4: D[128 tokens, 64 x Qg] =
//     K[128, 128] . Q[64 x Qg, 128]^T, E4M3 x E4M3 with fp32 accumulation in
//     TMEM (eight 64-column accumulators for one-query groups, else two of
//     256, so MMA and epilogue overlap);
//   * two epilogue warpgroups (one thread per token row, alternate items)
//     read D from TMEM, apply ReLU, the head weights and sq * sk * c_t, and
//     store the scores of visible positions.
// Every wait is bounded; a wait that gives up sets SML_FAULT_TIMEOUT and the
// CTA winds down (no trap).
#include <cudaTypedefs.h>
#include <math.h>

#include <mutex>

#include "ptx.cuh"
#include "sml_internal.cuh"

namespace sml {
namespace {

constexpr int kTile = 128;       // tokens per tile = MMA M
constexpr int kPageKeyBytes = SML_PAGE_TOKENS * SML_INDEX_DIM;   // 8,192
constexpr int kQRowsBytes = SML_INDEX_HEADS * SML_INDEX_DIM;      // 8,192 per query token

// Two shapes of the same kernel:
//   general: 9-stage ring, query groups of up to 4 tokens (N <= 256), two
//            256-column accumulators, four epilogue warpgroups (one per query
//            of the group, all on every item), one CTA per SM;
//   decode (every request has one query token): 5-stage ring, one-token groups
//            (N = 64), four 64-column accumulators, one epilogue warpgroup, and
//            half the shared memory and TMEM, so two CTAs share each SM and
//            keep twice the loads in flight.
template <int kStages_, int kGroup_, int kAccBufs_, int kEpiGroups_, int kCtasPerSm_, bool kQueryPerWg_,
          int kQBufs_>
struct Cfg {
  static constexpr int kStages = kStages_;
  static constexpr int kGroup = kGroup_;          // query tokens per group: N = 64 * Qg
  static constexpr int kAccBufs = kAccBufs_;
  static constexpr int kAccCols = 64 * kGroup_;
  static constexpr int kTmemCols = kAccBufs_ * 64 * kGroup_;
  static constexpr int kEpiGroups = kEpiGroups_;  // epilogue warpgroups, taking alternate items
  static constexpr int kThreads = 64 + 128 * kEpiGroups_;   // warp 0 TMA, warp 1 MMA, then the epilogue
  static constexpr int kCtasPerSm = kCtasPerSm_;
  // true: every epilogue warpgroup works on every item, warpgroup g on
  // queries [g kWgQ, (g + 1) kWgQ) of the group; false: the warpgroups take
  // alternate items, all their queries.
  static constexpr bool kQueryPerWg = kQueryPerWg_;
  static constexpr int kWgQ = kQueryPerWg_ ? kGroup_ / kEpiGroups_ : kGroup_;
  static_assert(!kQueryPerWg_ || kGroup_ % kEpiGroups_ == 0, "whole query shares per warpgroup");
  static constexpr int kQBufs = kQBufs_;   // query-group buffers
};
using CfgGeneral = Cfg<9, 4, 2, 4, 1, true, 2>;
using CfgDecode = Cfg<5, 1, 4, 1, 2, false, 2>;

template <class C>
struct __align__(1024) Smem {
  static constexpr int kStages = C::kStages, kGroup = C::kGroup, kEpiGroups = C::kEpiGroups;
  uint8_t keys[kStages][2 * kPageKeyBytes];      // [stage][128 rows x 128 B], SW128
  uint8_t q[C::kQBufs][kGroup * kQRowsBytes];    // [buffer][256 rows x 128 B], SW128
  float ksc[kStages][kTile];
  // per epilogue warpgroup: head weights, sq_t * c_t and n_t of its queries
  // (the whole group, or its one query of the group when kQueryPerWg)
  static constexpr int kWgQueries = C::kWgQ;
  __align__(16) float w[kEpiGroups][kWgQueries * SML_INDEX_HEADS];
  float qf[kEpiGroups][kWgQueries];
  int nv[kEpiGroups][kWgQueries];
  uint64_t full[kStages], empty[kStages];
  uint64_t qfull[C::kQBufs], qempty[C::kQBufs];
  uint64_t accfull[C::kAccBufs], accempty[C::kAccBufs];
  uint64_t drain;
  int valid[kStages];                            // bit p: page p of the tile was loaded
  uint32_t tmem_base;
  int abort;
  int sched[4];   // beg, end, first request, offset in it
  int red[C::kThreads / 32];
};

struct Params {
  int B, T, max_ctx, max_pages, ssmax;
  float s_index;
  const int32_t* cu_q;
  const int32_t* ctx_len;
  const int32_t* block_table;
  const int32_t* vis_len;     // optional n_t per token (non-decreasing within a request)
  const int32_t* ssmax_len;   // optional SSMax n per token
  const float* iq_scale;
  const float* iw;
  const uint8_t* index_base;
  int64_t index_pages;
  float* scores;
  int32_t* status;
};

// Walks the work items (request r, query group g, tile) in order.
template <int kGroup>
struct Walker {
  const Params* P;
  int r, g, tile, ngroups, ntiles;
  Req rq;

  __device__ void load_req() {
    rq = load_request(P->cu_q, P->ctx_len, r, P->T, P->max_ctx, P->max_pages, P->vis_len != nullptr);
    ngroups = rq.ok ? (rq.Q + kGroup - 1) / kGroup : 0;
  }
  __device__ int group_tiles() const {
    const int last = min(rq.Q, kGroup * g + kGroup);   // the group's queries: [4g, last)
    bool bad = false;                                  // (reported by the epilogue)
    const int n_last = visible_len(P->vis_len, rq, rq.q0 + last - 1, &bad);   // the largest of the group's
    return (n_last + kTile - 1) / kTile;
  }
  __device__ int qg() const { return min(kGroup, rq.Q - kGroup * g); }
  // Position on item `off` of request r0 (which has more than `off` items).
  __device__ void start(int r0, int off) {
    r = r0;
    load_req();
    for (g = 0; g < ngroups; ++g) {
      ntiles = group_tiles();
      if (off < ntiles) break;
      off -= ntiles;
    }
    tile = off;
  }
  // Items of the current request.
  __device__ int request_items() {
    int total = 0;
    for (g = 0; g < ngroups; ++g) total += group_tiles();
    return total;
  }
  __device__ void advance() {
    if (++tile < ntiles) return;
    tile = 0;
    if (++g < ngroups) {
      ntiles = group_tiles();
      return;
    }
    g = 0;
    for (++r; r < P->B; ++r) {
      load_req();
      if (ngroups > 0) {
        ntiles = group_tiles();
        return;
      }
    }
  }
};

// Block-wide sum of one int per thread (all kThreads threads call it).
template <int kThreads>
__device__ __forceinline__ int block_sum(int v, int* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  int s = 0;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) s += red[w];
  return s;
}

// Block-wide inclusive scan of one int per thread; *sum gets the block total.
template <int kThreads>
__device__ __forceinline__ int block_scan(int v, int* red, int* sum) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  __syncthreads();
  if (lane == 31) red[warp] = v;
  __syncthreads();
  int before = 0, s = 0;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) {
    before += w < warp ? red[w] : 0;
    s += red[w];
  }
  *sum = s;
  return v + before;
}

// This CTA's share of the work items and where it starts (request, offset),
// with every thread loading one request at a time: a round of parallel loads
// per kThreads requests instead of one dependent load chain per request.
template <int kThreads, int kGroup>
__device__ void schedule(const Params& P, int* red, int* out /* beg, end, r0, off0 */) {
  if (P.B <= kThreads) {
    // One request per thread: one round of loads and one scan give both the
    // total and where this CTA's share starts.
    Walker<kGroup> w{&P};
    w.r = threadIdx.x;
    int cnt = 0;
    if (w.r < P.B) {
      w.load_req();
      if (!w.rq.ok && blockIdx.x == 0) raise_fault(P.status, SML_FAULT_LENGTHS);
      cnt = w.request_items();
    }
    int total;
    const int incl = block_scan<kThreads>(cnt, red, &total);
    const long long G = gridDim.x;
    const int beg = (int)((long long)total * blockIdx.x / G);
    const int end = (int)((long long)total * (blockIdx.x + 1) / G);
    if (threadIdx.x == 0) {
      out[0] = beg;
      out[1] = end;
      out[2] = P.B;
      out[3] = 0;
    }
    __syncthreads();
    if (beg < end && cnt > 0 && beg >= incl - cnt && beg < incl) {
      out[2] = w.r;
      out[3] = beg - (incl - cnt);
    }
    return;
  }
  int total = 0;
  for (int base = 0; base < P.B; base += kThreads) {
    Walker<kGroup> w{&P};
    w.r = base + threadIdx.x;
    int cnt = 0;
    if (w.r < P.B) {
      w.load_req();
      if (!w.rq.ok && blockIdx.x == 0) raise_fault(P.status, SML_FAULT_LENGTHS);
      cnt = w.request_items();
    }
    total += block_sum<kThreads>(cnt, red);
  }
  const long long G = gridDim.x;
  const int beg = (int)((long long)total * blockIdx.x / G);
  const int end = (int)((long long)total * (blockIdx.x + 1) / G);
  if (threadIdx.x == 0) {
    out[0] = beg;
    out[1] = end;
    out[2] = P.B;
    out[3] = 0;
  }
  if (beg >= end) return;
  int acc = 0;
  for (int base = 0; base < P.B && acc <= beg; base += kThreads) {
    Walker<kGroup> w{&P};
    w.r = base + threadIdx.x;
    int cnt = 0;
    if (w.r < P.B) {
      w.load_req();
      cnt = w.request_items();
    }
    int sum;
    const int incl = block_scan<kThreads>(cnt, red, &sum);
    if (cnt > 0 && beg >= acc + incl - cnt && beg < acc + incl) {
      out[2] = w.r;
      out[3] = beg - (acc + incl - cnt);
    }
    acc += sum;
  }
}

// Warp-uniform bounded wait: every lane polls, the warp agrees on the result.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const volatile int* abort) {
  const bool ok = ptx::mbar_wait(bar, parity, abort);
  return __all_sync(0xffffffffu, ok);
}

template <class C>
__global__ void __launch_bounds__(C::kThreads, C::kCtasPerSm)
indexer_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                  const Params P) {
  constexpr int kStages = C::kStages, kGroup = C::kGroup, kAccBufs = C::kAccBufs, kTmemCols = C::kTmemCols;
  constexpr int kEpiGroups = C::kEpiGroups, kThreads = C::kThreads;
  extern __shared__ uint8_t smem_raw[];
  Smem<C>& S = *reinterpret_cast<Smem<C>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      ptx::mbar_init(&S.full[i], 1);
      // MMA commit + one arrive per epilogue warp that reads the stage
      ptx::mbar_init(&S.empty[i], 1 + (C::kQueryPerWg ? 4 * kEpiGroups : 4));
    }
    for (int i = 0; i < C::kQBufs; ++i) {
      ptx::mbar_init(&S.qfull[i], 1);
      ptx::mbar_init(&S.qempty[i], 1);
    }
    for (int i = 0; i < kAccBufs; ++i) {
      ptx::mbar_init(&S.accfull[i], 1);
      ptx::mbar_init(&S.accempty[i], C::kQueryPerWg ? 4 * kEpiGroups : 4);   // the warps that read it
    }
    ptx::mbar_init(&S.drain, 1);
    S.abort = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tensormap(&kmap);
    ptx::prefetch_tensormap(&qmap);
  }
  if (warp == 1) {
    ptx::tmem_alloc(&S.tmem_base, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::griddep_wait();   // inputs may come from the previous kernel of the stream
  schedule<kThreads, kGroup>(P, S.red, S.sched);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  // This CTA holds its tensor memory now, so a dependent grid scheduled on the
  // same SM cannot starve it of columns.
  if (threadIdx.x == 0) ptx::griddep_launch_dependents();
  const int beg = S.sched[0], end = S.sched[1];
  volatile int* abort = &S.abort;

  if (warp == 0) {
    // ---------------- TMA producer (one lane) ----------------
    if (lane == 0 && beg < end) {
      Walker<kGroup> w{&P};
      w.start(S.sched[2], S.sched[3]);
      int stage = 0;
      uint32_t phase = 0;
      int qcount = 0, last_r = -1, last_g = -1;
      for (int it = beg; it < end; ++it, w.advance()) {
        if (w.r != last_r || w.g != last_g) {
          const int qb = qcount % C::kQBufs;
          if (!ptx::mbar_wait(&S.qempty[qb], ((qcount / C::kQBufs) & 1) ^ 1, abort)) { *abort = 1; break; }
          const int qg = w.qg();
          ptx::mbar_arrive_expect_tx(&S.qfull[qb], qg * kQRowsBytes);
          for (int j = 0; j < qg; ++j)
            ptx::tma_load_2d(&S.q[qb][j * kQRowsBytes], &qmap, &S.qfull[qb], 0,
                             (w.rq.q0 + kGroup * w.g + j) * SML_INDEX_HEADS);
          ++qcount;
          last_r = w.r;
          last_g = w.g;
        }
        if (!ptx::mbar_wait(&S.empty[stage], phase ^ 1, abort)) { *abort = 1; break; }
        int valid = 0;
        uint32_t bytes = 0;
        int phys[2];
        for (int pg = 0; pg < 2; ++pg) {
          const int lp = w.tile * 2 + pg;
          phys[pg] = -1;
          if (lp * SML_PAGE_TOKENS < w.rq.L) {
            const int ph = __ldg(P.block_table + (size_t)w.r * P.max_pages + lp);
            if (ph >= 0 && ph < P.index_pages) {
              phys[pg] = ph;
              valid |= 1 << pg;
              bytes += kPageKeyBytes + SML_PAGE_TOKENS * 4;
            } else {
              raise_fault(P.status, SML_FAULT_PAGE);
            }
          }
        }
        S.valid[stage] = valid;
        ptx::mbar_arrive_expect_tx(&S.full[stage], bytes);
        for (int pg = 0; pg < 2; ++pg) {
          if (phys[pg] < 0) continue;
          ptx::tma_load_3d(&S.keys[stage][pg * kPageKeyBytes], &kmap, &S.full[stage], 0, 0, phys[pg]);
          ptx::bulk_load(&S.ksc[stage][pg * SML_PAGE_TOKENS],
                         P.index_base + (size_t)phys[pg] * SML_INDEX_PAGE_BYTES + kPageKeyBytes,
                         SML_PAGE_TOKENS * 4, &S.full[stage]);
        }
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (*abort) {
        // Let copies already issued land before the CTA's shared memory goes away.
        for (int i = 0; i < kStages; ++i) ptx::mbar_wait(&S.full[i], phase ^ (i >= stage ? 1u : 0u), nullptr, 100000u);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer (one lane) ----------------
    if (lane == 0 && beg < end) {
      Walker<kGroup> w{&P};
      w.start(S.sched[2], S.sched[3]);
      int stage = 0, acc = 0;
      uint32_t phase = 0, accphase = 0;
      int qcount = 0, last_r = -1, last_g = -1, qb = 0;
      for (int it = beg; it < end; ++it, w.advance()) {
        if (w.r != last_r || w.g != last_g) {
          if (qcount > 0) ptx::mma_commit(&S.qempty[qb]);   // previous group's queries free once read
          qb = qcount % C::kQBufs;
          if (!ptx::mbar_wait(&S.qfull[qb], (qcount / C::kQBufs) & 1, abort)) { *abort = 1; break; }
          ++qcount;
          last_r = w.r;
          last_g = w.g;
        }
        if (!ptx::mbar_wait(&S.accempty[acc], accphase ^ 1, abort)) { *abort = 1; break; }
        if (!ptx::mbar_wait(&S.full[stage], phase, abort)) { *abort = 1; break; }
        ptx::tc_fence_after();
        const uint32_t idesc = ptx::idesc_m128(SML_INDEX_HEADS * w.qg(), 0);
        const uint32_t d = S.tmem_base + acc * C::kAccCols;
        const uint32_t a0 = ptx::smem_u32(S.keys[stage]);
        const uint32_t b0 = ptx::smem_u32(S.q[qb]);
#pragma unroll
        for (int k = 0; k < SML_INDEX_DIM / 32; ++k)
          ptx::mma_f8f6f4_ss(d, ptx::sdesc_sw128(a0 + 32 * k), ptx::sdesc_sw128(b0 + 32 * k), idesc, k > 0);
        ptx::mma_commit(&S.empty[stage]);
        ptx::mma_commit(&S.accfull[acc]);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
        if (++acc == kAccBufs) {
          acc = 0;
          accphase ^= 1;
        }
      }
    }
    if (lane == 0) {
      // Every MMA this thread issued has finished before TMEM is released.
      ptx::mma_commit(&S.drain);
      ptx::mbar_wait(&S.drain, 0, nullptr, 100000u);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue: kEpiGroups warpgroups, one thread per token row ----------------
    // kQueryPerWg: warpgroup eg takes query eg of every item.  Otherwise
    // warpgroup eg takes the items with ordinal (it - beg) = eg mod kEpiGroups,
    // all the group's queries.
    const int eg = (warp - 2) >> 2;
    const int quarter = warp & 3;               // TMEM lanes 32 * quarter .. + 31
    const int row = quarter * 32 + lane;
    const int et = threadIdx.x - 64 - 128 * eg; // 0..127 within the warpgroup
    constexpr int kWq = Smem<C>::kWgQueries;
    float* wsm = S.w[eg];
    float* qfs = S.qf[eg];
    int* nvs = S.nv[eg];
    Walker<kGroup> w{&P};
    if (beg < end) w.start(S.sched[2], S.sched[3]);
    int last_r = -1, last_g = -1;
    for (int it = beg; it < end; ++it, w.advance()) {
      const int j_it = it - beg;
      if (!C::kQueryPerWg && j_it % kEpiGroups != eg) continue;
      const int stage = j_it % kStages, acc = j_it % kAccBufs;
      const uint32_t phase = (j_it / kStages) & 1, accphase = (j_it / kAccBufs) & 1;
      const int qg = w.qg();
      const int j0 = kGroup * w.g;
      // this warpgroup's queries of the group: [jb, jb + jn)
      const int jb = C::kQueryPerWg ? eg * kWq : 0;
      const int jn = C::kQueryPerWg ? max(0, min(kWq, qg - jb)) : qg;
      if (w.r != last_r || w.g != last_g) {
        asm volatile("bar.sync %0, 128;" ::"r"(1 + eg) : "memory");
        for (int i = et; i < jn * SML_INDEX_HEADS; i += 128)
          wsm[i] = __ldg(P.iw + (size_t)(w.rq.q0 + j0 + jb) * SML_INDEX_HEADS + i);
        if (et < jn) {
          const int t = w.rq.q0 + j0 + jb + et;
          bool bad = false;
          const int n = visible_len(P.vis_len, w.rq, t, &bad);
          if (bad) raise_fault(P.status, SML_FAULT_LENGTHS);
          const float c = P.ssmax ? P.s_index * logf((float)ssmax_len_of(P.ssmax_len, t, n)) : 1.f;
          qfs[et] = __ldg(P.iq_scale + t) * c;
          nvs[et] = n;
        }
        asm volatile("bar.sync %0, 128;" ::"r"(1 + eg) : "memory");
        last_r = w.r;
        last_g = w.g;
      }
      if (!warp_wait(&S.accfull[acc], accphase, abort)) { *abort = 1; break; }
      if (!warp_wait(&S.full[stage], phase, abort)) { *abort = 1; break; }
      ptx::tc_fence_after();
      const float sk = S.ksc[stage][row];
      const bool row_ok = (S.valid[stage] >> (row >> 6)) & 1;
      const int s = w.tile * kTile + row;
      const uint32_t tbase = S.tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * C::kAccCols;
      for (int jj = 0; jj < jn && jj < kWq; ++jj) {
        const int j = jb + jj;
        uint32_t v0[32], v1[32];
        ptx::tmem_ld32(tbase + j * SML_INDEX_HEADS, v0);
        ptx::tmem_ld32(tbase + j * SML_INDEX_HEADS + 32, v1);
        ptx::tmem_wait_ld(v0, v1);
        const float4* wj = reinterpret_cast<const float4*>(wsm + jj * SML_INDEX_HEADS);
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float4 wa = wj[i], wb = wj[8 + i];
          s0 = fmaf(wa.x, fmaxf(__uint_as_float(v0[4 * i]), 0.f), s0);
          s0 = fmaf(wa.y, fmaxf(__uint_as_float(v0[4 * i + 1]), 0.f), s0);
          s0 = fmaf(wa.z, fmaxf(__uint_as_float(v0[4 * i + 2]), 0.f), s0);
          s0 = fmaf(wa.w, fmaxf(__uint_as_float(v0[4 * i + 3]), 0.f), s0);
          s1 = fmaf(wb.x, fmaxf(__uint_as_float(v1[4 * i]), 0.f), s1);
          s1 = fmaf(wb.y, fmaxf(__uint_as_float(v1[4 * i + 1]), 0.f), s1);
          s1 = fmaf(wb.z, fmaxf(__uint_as_float(v1[4 * i + 2]), 0.f), s1);
          s1 = fmaf(wb.w, fmaxf(__uint_as_float(v1[4 * i + 3]), 0.f), s1);
        }
        if (row_ok && s < nvs[jj]) P.scores[(size_t)(w.rq.q0 + j0 + j) * P.max_ctx + s] = (s0 + s1) * qfs[jj] * sk;
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        ptx::mbar_arrive(&S.accempty[acc]);
        ptx::mbar_arrive(&S.empty[stage]);
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && S.abort) raise_fault(P.status, SML_FAULT_TIMEOUT);
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(S.tmem_base, kTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// Encoded tensor maps depend only on the address, the shape and the device:
// the last few are kept so that a call with the same caches and batch shape
// (every decode step) does not re-encode them.
struct MapCache {
  struct Entry {
    const void* base;
    int64_t n;
    int dev;
    CUtensorMap map;
  };
  std::mutex mu;
  Entry e[8] = {};
  int next = 0;
  template <typename Encode>
  bool get(const void* base, int64_t n, CUtensorMap* out, Encode&& encode) {
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> g(mu);
    for (const Entry& x : e)
      if (x.base == base && x.n == n && x.dev == dev && base != nullptr) {
        *out = x.map;
        return true;
      }
    if (!encode(out)) return false;
    e[next] = Entry{base, n, dev, *out};
    next = (next + 1) % 8;
    return true;
  }
};

template <class C>
cudaError_t launch_cfg(const CUtensorMap& kmap, const CUtensorMap& qmap, const Params& P, cudaStream_t stream) {
  const size_t smem = sizeof(Smem<C>) + 1024;
  cudaError_t e = set_max_smem(reinterpret_cast<const void*>(indexer_tc_kernel<C>), smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(indexer_tc_kernel<C>, dim3(device_sm_count() * C::kCtasPerSm), dim3(C::kThreads), smem, stream, 0,
                    kmap, qmap, P);
}

}  // namespace

cudaError_t launch_indexer(const sml_problem& p, const uint8_t* iq8, const float* iq_scale,
                           const float* iw, const uint8_t* index_base, int64_t index_pages,
                           float* scores, int32_t* status, cudaStream_t stream) {
  auto enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap kmap, qmap;
  static MapCache kcache, qcache;
  const bool kok = kcache.get(index_base, index_pages, &kmap, [&](CUtensorMap* m) {
    // The pool as [pages][64 rows][128 B]: one box = the 64 keys of one page.
    cuuint64_t dims[3] = {SML_INDEX_DIM, SML_PAGE_TOKENS, (cuuint64_t)index_pages};
    cuuint64_t strides[2] = {SML_INDEX_DIM, SML_INDEX_PAGE_BYTES};
    cuuint32_t box[3] = {SML_INDEX_DIM, SML_PAGE_TOKENS, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(index_base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  });
  if (!kok) return cudaErrorInvalidValue;
  const bool qok = qcache.get(iq8, p.num_tokens, &qmap, [&](CUtensorMap* m) {
    // Indexer queries as [T * 64 rows][128 B]: one box = the 64 heads of a token.
    cuuint64_t dims[2] = {SML_INDEX_DIM, (cuuint64_t)p.num_tokens * SML_INDEX_HEADS};
    cuuint64_t strides[1] = {SML_INDEX_DIM};
    cuuint32_t box[2] = {SML_INDEX_DIM, SML_INDEX_HEADS};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(iq8), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  });
  if (!qok) return cudaErrorInvalidValue;
  Params P;
  P.B = p.num_requests;
  P.T = p.num_tokens;
  P.max_ctx = p.max_ctx;
  P.max_pages = p.max_pages;
  P.ssmax = p.ssmax;
  P.s_index = p.ssmax_s_index;
  P.cu_q = p.cu_q;
  P.ctx_len = p.ctx_len;
  P.block_table = p.block_table;
  P.vis_len = p.vis_len;
  P.ssmax_len = p.ssmax_len;
  P.iq_scale = iq_scale;
  P.iw = iw;
  P.index_base = index_base;
  P.index_pages = index_pages;
  P.scores = scores;
  P.status = status;
  // When every request has one query token (T == B) every group is one token.
  if (p.num_tokens == p.num_requests) return launch_cfg<CfgDecode>(kmap, qmap, P, stream);
  return launch_cfg<CfgGeneral>(kmap, qmap, P, stream);
}

}  // namespace sml
