// Absorbed-query sparse MLA over a paged fp8_ds_mla (or plain E4M3) latent
// cache on the sm_100a tensor cores, split over the selected keys, then a
// log-sum-exp merge.
//
// vLLM blog "vLLM 首日支持 Mistral Large 4": highlights list (MLA, KV LoRA
// rank 512, RoPE dim 64, top-2048 keys per query); section "实现细节 / 模型架构"
// (sparse MLA over the fp8_ds_mla latent cache; NoPE = RoPE dim 0 on the same
// cache; SSMax on the MLA query); section "长上下文" (partial results merged by
// their LSE); section "ROCm 实现细节", paragraph "FP8 潜在缓存" (the plain
// per-tensor E4M3 cache, 576 B per token).  For token t, head h over the
// selected set S_t:
//   z_i = sm_scale * c_t * (q_nope . c_hat_i + q_pe . k_pe_i)
//   out = sum_i softmax(z)_i c_hat_i,   lse = ln sum_i exp(z_i)
// with c_hat_i = e4m3 latent x its 128-element block scale.
//
// Work: a unit is (query token, group of 16 heads, tile of 128 selected keys).
// Each CTA serves one head group (blockIdx.x % groups) and takes an equal
// contiguous range of that group's (token, tile) units, token-major, as few
// CTAs per group as give the same longest range; the CTAs of the different
// groups with the same blockIdx.x / groups walk the same tokens' tiles at the
// same time, so a row gathered for one group is still in L2 for the others.
// Where a range crosses a token boundary the CTA writes one partial result
// per (token, head group), and a merge kernel combines them by their LSE.  Keys are
// the MMA M dimension of QK^T and the K dimension of PV, the 16 heads N (16
// heads as M would waste 3/4 of the smallest M); both products run on
// kind::f8f6f4 straight from the gathered E4M3 tile: the latent is never
// converted.
//   * warps 17-31 fill the two tile buffers: they turn the tile's selected
//     positions into pool rows (block table, bounds checks), then copy the
//     rows with 16-B cp.async straight into place, 128-B-swizzled, a masked
//     row as zeros; the copies arrive on the buffer's barrier by themselves,
//     so the loaders go on to the next tile at once.  (Random 656-B rows are
//     bound by the requests in flight per SM: measured on B200, cp.async
//     reaches about 20 GB/s per SM whatever the shared-memory size and the
//     number of SMs gathering, while register loads lose a quarter of that
//     rate when the kernel's shared memory leaves L1 small, and TMA
//     tile::gather4 reaches about half of it.);
//   * warp 16 issues the MMAs (one thread):
//       S_b^T = C_b . [Qhi_b; Qlo_b]^T   (K-major; N = 32: both query terms),
//       S_pe^T = K_pe . Q_pe^T           (bf16; plain E4M3: both terms),
//       O_b^T += C_b^T . [Bhi_b; Bmid_b; Blo_b]^T  (C_b^T read MN-major from
//       the same tile; N = 48: the three weight terms),
//     each as soon as its inputs are ready: a tile's PV (which frees its
//     buffer) does not wait for the next tile's QK^T, nor the reverse;
//   * warps 0-15 (four per TMEM lane quarter: keys 32q..32q+31, heads
//     4 hq .. 4 hq + 3) run the softmax on S^T and build the weights
//     B_b[i, h] = 2^(z_ih - M_h) scale_ib as three E4M3 terms whose sum
//     carries 12 significant bits; M_h is a per-head integer exponent that
//     keeps every weight at most 440, raised (and O rescaled, exactly) only
//     when a tile would exceed that; at the end of a (token, head group) they
//     read O^T back and write its partial output and LSE.  Warps 0-7 also
//     stage each (token, head group)'s query.  The softmax is split over
//     sixteen warps so that a tile's weights are ready well within the time
//     the next tile's rows take to arrive: the tile buffer is then free again
//     before the loaders need it.
// The query is split exactly into two E4M3 terms sharing a power-of-two scale
// per head; products of E4M3 values are exact and accumulate in fp32.
// Every wait is bounded; a wait that gives up sets SML_FAULT_TIMEOUT and the
// CTA winds down (no trap).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <math.h>

#include "ptx.cuh"
#include "sml_internal.cuh"

namespace sml {
namespace {

constexpr int kHC = 16;          // heads per unit
constexpr int kKT = 128;         // keys per tile
constexpr int kSoftmaxWarps = 16;      // warps 0-15
constexpr int kSoftmaxThreads = 32 * kSoftmaxWarps;
constexpr int kStageWarps = 8;         // warps 0-7 stage the query (thread = head x 32-dim part)
constexpr int kWarpMma = 16;
constexpr int kWarpLoad = 17;          // warps 17-31 copy the rows
constexpr int kLoadWarps = 15;
constexpr int kLoadThreads = 32 * kLoadWarps;
constexpr int kThreads = 32 * (kWarpLoad + kLoadWarps);   // 1024: eight warpgroups
static_assert(kLoadThreads >= kKT, "one loader thread per key of a tile looks up its pool row");
// Registers: the kernel launches with kRegsLaunch per thread; the four softmax
// warpgroups then raise theirs to kRegsSoftmax and the other four (MMA and
// loaders) lower theirs to kRegsOther.  setmaxnreg.inc draws on what the
// block launched with, so the shares must add up to it exactly.
constexpr int kRegsLaunch = 64, kRegsSoftmax = 80, kRegsOther = 48;
static_assert(kThreads * kRegsLaunch == kSoftmaxThreads * kRegsSoftmax + (kThreads - kSoftmaxThreads) * kRegsOther,
              "warpgroup register shares must add up to the launch allocation");
static_assert(kThreads % 128 == 0 && kSoftmaxThreads % 128 == 0 && kWarpMma == kSoftmaxWarps,
              "roles are whole warpgroups: 0-3 softmax, 4-7 the rest");
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// Weight exponents: a key's weights are capped at 440 (E4M3's largest value
// is 448; the margin covers the approximate 2^x and log2); an exponent that
// has to move puts the tile's largest possible weight in (56, 112].
constexpr float kLog2Cap = 8.78135971f;    // log2(440)
constexpr float kLog2Head = 6.80735492f;   // log2(112)
// bf16 weights have fp32's range: the exponent only keeps 2^(z - M_h) within
// 2^16 (a raise sets M_h at the tile's largest logit).
constexpr float kBfLog2Cap = 16.f;

// TMEM columns
constexpr uint32_t kColS = 0;       // S_b^T (lanes = keys): 32 columns per block b (hi | lo query term)
constexpr uint32_t kColSpe = 128;   // S_pe^T: 16 columns (bf16), or 32 (plain E4M3: hi | lo)
constexpr uint32_t kColO = 256;     // O_b^T (lanes = dims of block b): 48 columns (hi | mid | lo) ...
constexpr uint32_t kOStride = 64;   // ... at kColO + kOStride b
constexpr int kPBytes = kKT * 3 * kHC;   // one block's weight terms: 128 keys x 48 E4M3
constexpr int kLatBlock = kKT * 128;     // one 128-dim latent block of a tile

// Latent formats of the kernel's template parameter.
constexpr int kFmtDsMla = 0, kFmtPlain = 1, kFmtBf16 = 2;
// Tile buffers and 128-B latent blocks per tile of a format: the E4M3 tiles
// (64 KB of latent) are double-buffered; a bf16 tile is 128 KB (eight blocks
// of 64 dims), so one buffer is all shared memory holds.
template <int kFmt>
struct FmtDims {
  static constexpr int kBufs = kFmt == kFmtBf16 ? 1 : 2;
  static constexpr int kBlocks = kFmt == kFmtBf16 ? 8 : 4;
  static constexpr int kTerms = kFmt == kFmtBf16 ? 2 : 3;   // weight terms (PV N = 16 kTerms)
};

template <int kFmt>
struct __align__(1024) Smem {
  static constexpr int kBufs = FmtDims<kFmt>::kBufs, kBlocks = FmtDims<kFmt>::kBlocks;
  uint8_t lat[kBufs][kBlocks][kLatBlock];  // [buffer][block b][128 keys x 128 B] E4M3 (128 dims) or bf16 (64 dims), SW128
  uint8_t pe[kBufs][kKT * 128];  // [buffer][128 keys x 128 B] RoPE key (64 bf16, or 64 E4M3 + 64 zeros), SW128
  // E4M3: [block] 32 rows x 128 B, SW128, rows 0-15 high term, 16-31 low
  // term; bf16: the same bytes as 8 blocks of 16 rows x 128 B (64 dims)
  uint8_t q8[4][2 * kHC * 128];
  uint8_t qpe[2 * kHC * 128];    // RoPE query, SW128: bf16 rows 0-15; plain E4M3: rows 0-15 high, 16-31 low
  // E4M3: weight terms of block b, MN-major 8-key x 16-B core matrices; bf16:
  // the first 8 KB, the two terms of the weights (no block scales)
  uint8_t pb[4][kPBytes];
  float sc[kBufs][kKT][4];       // [buffer][key] the four block scales of the staged row
  float xmax[2][4][4][8];        // [tile parity][head quarter][key quarter]: 4 head maxima, largest scale
  float xsum[4][4][4];           // [head quarter][key quarter][head]: row-sum exchange
  float qs[kHC];                 // power-of-two query scale per head
  int32_t rowid[4][kKT];         // [tile % 4] pool row of each key, -1 = masked
  uint64_t full[kBufs], lat_free[kBufs];
  uint64_t q_ready, s_full, s_free, p_full, pv_done, o_free, drain;
  uint32_t tmem_base;
  int abort;
};

struct Params {
  int B, T, H, K, rope_dim, max_ctx, max_pages, ssmax;
  float sm_scale, ssmax_s;
  const int32_t* cu_q;
  const int32_t* ctx_len;
  const int32_t* block_table;
  const int32_t* vis_len;     // optional n_t per token
  const int32_t* ssmax_len;   // optional SSMax n per token
  const uint16_t* q;
  const uint8_t* latent;
  int64_t latent_pages;
  float latent_scale;   // plain E4M3 pool: its scale
  const int32_t* idx;
  const int32_t* idx_len;
  MlaWs ws;
  int32_t* status;
};

// Byte address of (row, 16-B chunk) in a 128-B-swizzled tile of 128-B rows.
__device__ __forceinline__ uint32_t sw128(uint32_t base, int row, int chunk) {
  return base + (row >> 3) * 1024 + (row & 7) * 128 + ((chunk ^ (row & 7)) << 4);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
__device__ __forceinline__ void st_shared_v2(uint32_t addr, uint32_t a, uint32_t b) {
  asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}
__device__ __forceinline__ void st_shared_b32(uint32_t addr, uint32_t a) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(a) : "memory");
}

// Round two floats to E4M3 (nearest even, saturating); the codes, low byte = a.
__device__ __forceinline__ uint32_t f2_to_e4m3x2(float a, float b) {
  return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3) & 0xffffu;
}

__device__ __forceinline__ float2 e4m3x2_to_f2(uint32_t two) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two & 0xffffu), __NV_E4M3);
  return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

// x (two values) -> E4M3 codes of the nearest value and the exact residual.
__device__ __forceinline__ uint32_t split_e4m3x2(float& x0, float& x1) {
  const uint32_t c = f2_to_e4m3x2(x0, x1);
  const float2 r = e4m3x2_to_f2(c);
  x0 -= r.x;
  x1 -= r.y;
  return c;
}

// x rounded to 4 significant bits, nearest even, by integer arithmetic on
// its fp32 bits: the E4M3 value nearest to x wherever x is in E4M3's normal
// range (|x| in [2^-6, 448]).  Below 2^-6 the result is finer than E4M3's
// subnormal step 2^-9, and the code the conversion then picks is within
// 2^-10 of it.
__device__ __forceinline__ float round_e4m3_normal(float x) {
  const uint32_t b = __float_as_uint(x);
  return __uint_as_float((b + 0x7ffffu + ((b >> 20) & 1u)) & 0xfff00000u);
}

// Three E4M3 terms of two weights (each at most 448), low byte = first
// weight: x = hi + mid + lo to 12 significant bits; the residuals are exact
// in fp32.
__device__ __forceinline__ void split3_e4m3x2(float x0, float x1, uint32_t& hi, uint32_t& mid, uint32_t& lo) {
  const float h0 = round_e4m3_normal(x0), h1 = round_e4m3_normal(x1);
  const float r0 = x0 - h0, r1 = x1 - h1;
  const float m0 = round_e4m3_normal(r0), m1 = round_e4m3_normal(r1);
  hi = f2_to_e4m3x2(h0, h1);
  mid = f2_to_e4m3x2(m0, m1);
  lo = f2_to_e4m3x2(r0 - m0, r1 - m1);
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const volatile int* abort) {
  const bool ok = ptx::mbar_wait(bar, parity, abort);
  return __all_sync(0xffffffffu, ok);
}

// AND of a flag over the softmax threads (named barrier 5).  Every wait
// outcome reaches this before the next named barrier of the softmax warps, so
// a wait that gave up ends all of them together instead of leaving some
// blocked at a barrier.
__device__ __forceinline__ bool softmax_all(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, 5, %2, p;\n selp.u32 %0, 1, 0, q;\n}"
      : "=r"(r)
      : "r"((uint32_t)ok), "n"(kSoftmaxThreads)
      : "memory");
  return r != 0;
}

// AND of a flag over the loader threads (named barrier 6); also orders their
// shared-memory writes before it against reads after it.
__device__ __forceinline__ bool loader_all(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, 6, %2, p;\n selp.u32 %0, 1, 0, q;\n}"
      : "=r"(r)
      : "r"((uint32_t)ok), "n"(kLoadThreads)
      : "memory");
  return r != 0;
}

// 2^x (the hardware approximation; relative error about 2^-22).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// OR of a flag over the four warps of one head quarter (named barrier 1 +
// quarter; also a barrier for them).
__device__ __forceinline__ bool group_any(int hq, bool v) {
  uint32_t r;
  asm volatile("{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, %2, 128, p;\n selp.u32 %0, 1, 0, q;\n}"
               : "=r"(r)
               : "r"((uint32_t)v), "r"(1 + hq)
               : "memory");
  return r != 0;
}

// log2(x) (the hardware approximation), x > 0.
__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// The four warps of one head quarter (named barrier 1 + quarter).
__device__ __forceinline__ void group_sync(int hq) { asm volatile("bar.sync %0, 128;" ::"r"(1 + hq) : "memory"); }

// First unit of the i-th CTA of a head group (units of one head group).
__device__ __forceinline__ long long unit_begin(const MlaPlan& m, int i) { return m.units * i / m.cpg; }
// Index, within its head group's CTAs, of the CTA whose range holds unit u.
__device__ __forceinline__ int cta_of(const MlaPlan& m, long long u) {
  return (int)(((u + 1) * m.cpg - 1) / m.units);
}

// One (token, head group) of a CTA's range: tiles [j0, j0 + nj) of it, of
// which the first ne hold selected keys (tile j holds keys [128 j, 128 j +
// 128) of the token's selection, len of them valid).
struct Seg {
  int tg, t, g, j0, nj, ne;
  int r, n, len, nss;   // request, visible length, selected count, SSMax n
  bool req_ok, len_bad;
  size_t slot;
};

// Warp-collective (the request lookup is a 32-way search).
__device__ __forceinline__ Seg segment_at(const Params& P, long long u, long long e) {
  const MlaPlan& m = P.ws.plan;
  Seg s;
  s.t = (int)(u / m.tpt);
  s.j0 = (int)(u % m.tpt);
  s.g = blockIdx.x % m.hg;
  s.tg = s.t * m.hg + s.g;
  const long long seg_end = min(e, (long long)(s.t + 1) * m.tpt);
  s.nj = (int)(seg_end - u);
  s.r = request_of_warp(P.cu_q, P.B, s.t);
  const Req rq = load_request(P.cu_q, P.ctx_len, s.r, P.T, P.max_ctx, P.max_pages, P.vis_len != nullptr);
  s.req_ok = rq.ok && s.t >= rq.q0 && s.t - rq.q0 < rq.Q;
  bool bad_n = false;
  s.n = s.req_ok ? visible_len(P.vis_len, rq, s.t, &bad_n) : 0;
  s.req_ok = s.req_ok && !bad_n;
  s.nss = ssmax_len_of(P.ssmax_len, s.t, s.n);
  // Everything above reads the problem's request arrays, which no call of this
  // library produces for a sparse-MLA call (the interface requires it); the
  // selection comes from the previous kernel (a no-op after the first call).
  ptx::griddep_wait();
  const int len = s.req_ok ? __ldg(P.idx_len + s.t) : 0;
  const int len_max = min(P.K, s.n);
  s.len_bad = len < 0 || len > len_max;
  s.len = max(0, min(len, len_max));
  const int tiles = (s.len + kKT - 1) / kKT;
  s.ne = max(0, min(s.nj, tiles - s.j0));
  s.slot = (size_t)s.tg * m.smax + ((int)blockIdx.x / m.hg - cta_of(m, (long long)s.t * m.tpt));
  return s;
}

// A cursor over the non-empty tiles of a CTA's range, in order: tile jj of
// segment s (the seg-th non-empty (token, head group) of the range), the
// k-th tile overall.  Warp-collective, like segment_at.
struct Cur {
  long long u;   // the unit after segment s
  int ne;        // segment s's non-empty tiles
  int jj, seg, k;
  bool valid;
};

__device__ __forceinline__ void cur_seek(Cur& c, const Params& P, long long ue) {
  while (c.u < ue) {
    const Seg s = segment_at(P, c.u, ue);
    c.u += s.nj;
    c.ne = s.ne;
    if (s.ne > 0) {
      c.jj = 0;
      c.valid = true;
      return;
    }
  }
  c.valid = false;
}

__device__ __forceinline__ void cur_start(Cur& c, const Params& P, long long ub, long long ue) {
  c.u = ub;
  c.seg = 0;
  c.k = 0;
  cur_seek(c, P, ue);
}

__device__ __forceinline__ void cur_next(Cur& c, const Params& P, long long ue) {
  ++c.k;
  if (++c.jj < c.ne) return;
  ++c.seg;
  cur_seek(c, P, ue);
}

// Stage the query of (token t, head group g) for QK^T (the 256 softmax
// threads; thread = head h, part p of 16).  Nope part: q = s_h (hi + lo), hi
// and lo E4M3 and s_h a power of two >= amax_h / 448, so q / s_h, its
// rounding to hi and the residual lo are exact in fp32, and lo is exact in
// E4M3 (a bf16 has 8 significant bits, hi takes 4, the residual the other 4)
// down to E4M3's subnormal step.  RoPE part: copied as bf16; for a plain E4M3
// pool split the same way (its products are E4M3 x E4M3).  A bf16 pool takes
// the bf16 query as it is (bf16 x bf16 products), s_h = 1.
template <int kFmt>
__device__ __forceinline__ void stage_query(const Params& P, Smem<kFmt>& S, int t, int g, int tid) {
  constexpr bool kPlain = kFmt == kFmtPlain;
  const int h = tid >> 4, p = tid & 15;
  if constexpr (kFmt == kFmtBf16) {
    // 16-B chunk c of the head's row: c < 64 latent dims [8 c, 8 c + 8)
    // (block c / 8 of 64 dims, 2 KB of 16 rows each), 64-71 the RoPE part
    const uint16_t* qh = P.q + ((size_t)t * P.H + g * kHC + h) * (SML_LATENT_DIM + P.rope_dim);
    const int nc = P.rope_dim ? 72 : 64;
    const uint32_t q0 = ptx::smem_u32(&S.q8[0][0]), qp = ptx::smem_u32(S.qpe);
    for (int c = p; c < nc; c += 16) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(qh) + c);
      const uint32_t dst = c < 64 ? sw128(q0 + (c >> 3) * (kHC * 128), h, c & 7) : sw128(qp, h, c - 64);
      st_shared_v4(dst, v.x, v.y, v.z, v.w);
    }
    if (p == 0) S.qs[h] = 1.f;
    return;
  }
  const int Dq = SML_LATENT_DIM + P.rope_dim;
  const uint16_t* qh = P.q + ((size_t)t * P.H + g * kHC + h) * Dq;
  uint4 v[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = __ldg(reinterpret_cast<const uint4*>(qh + 32 * p) + i);
  uint2 pv = make_uint2(0u, 0u);
  if (P.rope_dim) pv = __ldg(reinterpret_cast<const uint2*>(qh + SML_LATENT_DIM + 4 * p));
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
    for (int k = 0; k < 4; ++k)
      amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w[k] << 16)), fabsf(__uint_as_float(w[k] & 0xffff0000u))));
  }
  if (kPlain) {
    amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(pv.x << 16)), fabsf(__uint_as_float(pv.x & 0xffff0000u))));
    amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(pv.y << 16)), fabsf(__uint_as_float(pv.y & 0xffff0000u))));
  }
#pragma unroll
  for (int o = 1; o < 16; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  int e2 = 0;
  if (amax > 0.f) frexpf(amax / 448.f, &e2);   // amax / 448 < 2^e2
  const float inv = ldexpf(1.f, -e2);
  if (p == 0) S.qs[h] = ldexpf(1.f, e2);
  // dims [32 p, 32 p + 32) -> block p / 4, 16-B chunks 2 (p % 4) and 2 (p % 4) + 1
  const int b = p >> 2;
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint4 vv = v[2 * c + (k >> 1)];
      const uint32_t wa = (k & 1) ? vv.z : vv.x, wb = (k & 1) ? vv.w : vv.y;
      float x0 = __uint_as_float(wa << 16) * inv, x1 = __uint_as_float(wa & 0xffff0000u) * inv;
      float x2 = __uint_as_float(wb << 16) * inv, x3 = __uint_as_float(wb & 0xffff0000u) * inv;
      const uint32_t h01 = split_e4m3x2(x0, x1), h23 = split_e4m3x2(x2, x3);
      hw[k] = h01 | (h23 << 16);
      lw[k] = f2_to_e4m3x2(x0, x1) | (f2_to_e4m3x2(x2, x3) << 16);
    }
    const int chunk = 2 * (p & 3) + c;
    st_shared_v4(sw128(ptx::smem_u32(S.q8[b]), h, chunk), hw[0], hw[1], hw[2], hw[3]);
    st_shared_v4(sw128(ptx::smem_u32(S.q8[b]), h + kHC, chunk), lw[0], lw[1], lw[2], lw[3]);
  }
  if (P.rope_dim) {
    const uint32_t qb = ptx::smem_u32(S.qpe);
    if (kPlain) {
      // 4 E4M3 codes per term: bytes 4 p .. 4 p + 3 of rows h (high) and h + 16 (low)
      float x0 = __uint_as_float(pv.x << 16) * inv, x1 = __uint_as_float(pv.x & 0xffff0000u) * inv;
      float x2 = __uint_as_float(pv.y << 16) * inv, x3 = __uint_as_float(pv.y & 0xffff0000u) * inv;
      const uint32_t h01 = split_e4m3x2(x0, x1), h23 = split_e4m3x2(x2, x3);
      const uint32_t lo = f2_to_e4m3x2(x0, x1) | (f2_to_e4m3x2(x2, x3) << 16);
      st_shared_b32(sw128(qb, h, p >> 2) + 4 * (p & 3), h01 | (h23 << 16));
      st_shared_b32(sw128(qb, h + kHC, p >> 2) + 4 * (p & 3), lo);
    } else {
      // 4 bf16: bytes 8 p .. 8 p + 7 of row h
      st_shared_v2(sw128(qb, h, p >> 1) + 8 * (p & 1), pv.x, pv.y);
    }
  }
}

// kPlain: the latent pool is plain E4M3 (576-B rows under one scale); else
// fp8_ds_mla.  A template parameter, so that each path is compiled for its
// own row layout.
template <int kFmt>
__global__ void __launch_bounds__(kThreads, 1) sparse_mla_kernel(const __grid_constant__ Params P) {
  constexpr bool kPlain = kFmt == kFmtPlain, kBf = kFmt == kFmtBf16;
  constexpr int kBufs = FmtDims<kFmt>::kBufs, kTerms = FmtDims<kFmt>::kTerms;
  using Sm = Smem<kFmt>;
  extern __shared__ uint8_t smem_raw[];
  Sm& S = *reinterpret_cast<Sm*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const MlaPlan& plan = P.ws.plan;
  // this CTA serves head group blockIdx.x % hg: its units are that group's
  const int gi = (int)blockIdx.x / plan.hg;
  const long long ub = unit_begin(plan, gi), ue = unit_begin(plan, gi + 1);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kBufs; ++i) {
      // every loader thread's copies (asynchronous arrivals) + one ordinary arrival
      ptx::mbar_init(&S.full[i], kLoadThreads + 1);
      ptx::mbar_init(&S.lat_free[i], 1);   // PV of the tile done (its last reader)
    }
    ptx::mbar_init(&S.q_ready, kStageWarps);
    ptx::mbar_init(&S.s_full, 1);
    ptx::mbar_init(&S.s_free, kSoftmaxWarps);
    ptx::mbar_init(&S.p_full, kSoftmaxWarps);
    ptx::mbar_init(&S.pv_done, 1);
    ptx::mbar_init(&S.o_free, kSoftmaxWarps);
    ptx::mbar_init(&S.drain, 1);
    S.abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == kWarpMma) {
    ptx::tmem_alloc(&S.tmem_base, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  // This CTA holds its tensor memory now, so a dependent grid scheduled on the
  // same SM cannot starve it of columns.  Each thread waits for the previous
  // kernel (the selection) just before its first read of idx_len (in
  // segment_at): the request lookups and the first query overlap that kernel.
  if (threadIdx.x == 0) ptx::griddep_launch_dependents();
  volatile int* abort = &S.abort;
  const uint32_t T0 = S.tmem_base;

  // Each role moves its warpgroup's register share first (the lowering ones
  // free what the raising ones take; every warpgroup takes exactly one branch).
  if (warp >= kWarpLoad) {
    // ================= loaders: pool rows, then row copies =================
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
    const int lt = threadIdx.x - 32 * kWarpLoad;   // 0 .. kLoadThreads - 1
    constexpr int kRow = kBf ? SML_LATENT_BF16_ROW_BYTES : kPlain ? SML_LATENT_E4M3_ROW_BYTES : SML_LATENT_ROW_BYTES;
    // A row as 16-B chunks: 0-31 the 512-B latent (chunk c: block c / 8,
    // 16-B column c % 8); fp8_ds_mla, 32 the four block scales and 33-40 the
    // bf16 RoPE key; plain E4M3, 32-35 the 64 RoPE codes (the only bytes of
    // the row the RoPE MMA reads).  The tile's chunks are numbered row-major
    // and dealt out to the loader threads in order (chunk lt + kLoadThreads
    // i), so a warp's 32 chunks are mostly of one row.
    // bf16: chunks 0-63 the 1,024-B latent (block c / 8 of 64 dims), 64-71
    // the RoPE key.
    const int parts = kBf ? (P.rope_dim ? 72 : 64) : kPlain ? (P.rope_dim ? 36 : 32) : (P.rope_dim ? 41 : 33);
    const int drow = kLoadThreads / parts, dpart = kLoadThreads - drow * parts;
    const int row0 = lt / parts, part0 = lt - row0 * parts;
    int k = 0;   // tiles so far
    bool ok = true;
    for (long long u = ub; ok && u < ue;) {
      const Seg s = segment_at(P, u, ue);
      u += s.nj;
      if (lt == 0) {
        if (!s.req_ok) raise_fault(P.status, SML_FAULT_LENGTHS);
        else if (s.len_bad) raise_fault(P.status, SML_FAULT_TOPK_LEN);
      }
      for (int jj = 0; jj < s.ne; ++jj, ++k) {
        const int j = s.j0 + jj, buf = k % kBufs;
        int32_t* rowid = S.rowid[k & 3];   // last used by tile k - 4, whose softmax is done
        // pool row of the tile's key lt (loaded before the buffer is free)
        if (lt < kKT) {
          int rid = -1;
          const int key = j * kKT + lt;
          if (key < s.len) {
            const int pos = __ldg(P.idx + (size_t)s.t * P.K + key);
            if (pos >= 0 && pos < s.n) {
              const int ph = __ldg(P.block_table + (size_t)s.r * P.max_pages + pos / SML_PAGE_TOKENS);
              if (ph >= 0 && ph < P.latent_pages) rid = ph * SML_PAGE_TOKENS + pos % SML_PAGE_TOKENS;
              else raise_fault(P.status, SML_FAULT_PAGE);
            } else {
              raise_fault(P.status, SML_FAULT_INDEX);
            }
          }
          rowid[lt] = rid;
        }
        // the buffer's last tile (k - kBufs) has been read by its PV
        if (k >= kBufs) ok = warp_wait(&S.lat_free[buf], ((k / kBufs) - 1) & 1, abort);
        ok = loader_all(ok);   // the tile's row ids written, and the wait's outcome shared
        if (!ok) break;
        // the row ids are generic writes the softmax reads: released by this
        // arrival (after the barrier above); the copies arrive by themselves
        if (lt == 0) ptx::mbar_arrive(&S.full[buf]);
        const uint32_t lat0 = ptx::smem_u32(S.lat[buf][0]);
        const uint32_t pe0 = ptx::smem_u32(S.pe[buf]);
        const uint32_t sc0 = ptx::smem_u32(&S.sc[buf][0][0]);
        int row = row0, part = part0;
        for (; row < kKT; row += drow, part += dpart) {
          if (part >= parts) {
            part -= parts;
            ++row;
            if (row >= kKT) break;
          }
          const int id = rowid[row];
          const uint8_t* src = P.latent + (size_t)(id >= 0 ? id : 0) * kRow + 16 * part;
          uint32_t dst;
          if (part < (kBf ? 64 : 32)) dst = sw128(lat0 + (part >> 3) * kLatBlock, row, part & 7);
          else if (kBf) dst = sw128(pe0, row, part - 64);
          else if (kPlain) dst = sw128(pe0, row, part - 32);
          else if (part == 32) dst = sc0 + 16 * row;
          else dst = sw128(pe0, row, part - 33);
          ptx::cp_async16(dst, src, id >= 0 ? 16u : 0u);   // a masked row is zero-filled, nothing read
        }
        // This thread's copies arrive on the buffer's barrier once they have
        // landed (generic-proxy writes: the MMA thread fences them for its
        // async-proxy reads after it sees the barrier complete).
        ptx::cp_async_arrive_noinc(&S.full[buf]);
      }
    }
    if (!ok) *abort = 1;
    ptx::cp_async_wait_all();   // nothing in flight when the CTA's shared memory goes away
    __syncwarp();
  } else if (warp == kWarpMma) {
    // ================= MMA issuer =================
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
    // E4M3 x E4M3 (bf16 pool: bf16 x bf16), both K-major, N = 32 (bf16: 16)
    const uint32_t id_qk = kBf ? ptx::idesc_f16(kHC, 1, 0, 0) : ptx::idesc_f16(2 * kHC, 0, 0, 0);
    const uint32_t id_pe = ptx::idesc_f16(kHC, 1, 0, 0);   // bf16, N = 16
    // both MN-major, N = 16 x the weight terms
    const uint32_t id_pv = kBf ? ptx::idesc_f16(2 * kHC, 1, 1, 1) : ptx::idesc_f16(3 * kHC, 0, 1, 1);
    auto issue_qk = [&](int buf) {
      if constexpr (kBf) {
        // S^T = C . Q^T + K_pe . Q_pe^T, all into one accumulator (no block
        // scales), 16 dims per step: 8 blocks of 64 latent dims, then RoPE.
        const uint32_t q0 = ptx::smem_u32(&S.q8[0][0]);
#pragma unroll
        for (int b = 0; b < 8; ++b) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            ptx::mma_f16_ss(T0 + kColS, ptx::sdesc_sw128(ptx::smem_u32(S.lat[buf][b]) + 32 * kk),
                            ptx::sdesc_sw128(q0 + b * (kHC * 128) + 32 * kk), id_qk, (b | kk) != 0);
        }
        if (P.rope_dim) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            ptx::mma_f16_ss(T0 + kColS, ptx::sdesc_sw128(ptx::smem_u32(S.pe[buf]) + 32 * kk),
                            ptx::sdesc_sw128(ptx::smem_u32(S.qpe) + 32 * kk), id_qk, 1);
        }
        ptx::mma_commit(&S.s_full);
        return;
      }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {   // 32 latent dims per step
#pragma unroll
        for (int b = 0; b < 4; ++b)
          ptx::mma_f8f6f4_ss(T0 + kColS + 32 * b, ptx::sdesc_sw128(ptx::smem_u32(S.lat[buf][b]) + 32 * kk),
                             ptx::sdesc_sw128(ptx::smem_u32(S.q8[b]) + 32 * kk), id_qk, kk > 0);
        if (P.rope_dim) {
          if (!kPlain)
            ptx::mma_f16_ss(T0 + kColSpe, ptx::sdesc_sw128(ptx::smem_u32(S.pe[buf]) + 32 * kk),
                            ptx::sdesc_sw128(ptx::smem_u32(S.qpe) + 32 * kk), id_pe, kk > 0);
          else if (kk < 2)   // 64 E4M3 RoPE codes: two steps of 32
            ptx::mma_f8f6f4_ss(T0 + kColSpe, ptx::sdesc_sw128(ptx::smem_u32(S.pe[buf]) + 32 * kk),
                               ptx::sdesc_sw128(ptx::smem_u32(S.qpe) + 32 * kk), id_qk, kk > 0);
        }
      }
      ptx::mma_commit(&S.s_full);
    };
    // O_b^T (+)= C_b^T . B_b^T, 32 keys per step.  A: the latent tile read
    // MN-major (dims contiguous; 8-key swizzle atoms 1,024 B apart).  B: 8-key
    // x 16-B core matrices, the three terms 128 B apart, 8-key groups 384 B
    // apart.  The first tile of a (token, head group) overwrites O; it waits
    // until the epilogue of the one before has read O.
    auto issue_pv = [&](int kk, bool first) {
      const int buf = kk % kBufs;
      if constexpr (kBf) {
        // bf16: O_m^T (+)= C_m^T . [Bhi; Blo]^T for output block m (dims
        // 128 m .. 128 m + 127: latent blocks 2 m and 2 m + 1, whose 64-dim
        // swizzle atoms are 16 KB apart), 16 keys per step.  B: 8-key x 16-B
        // core matrices (8 heads of one term), the four (term, head half)
        // ones 128 B apart, 8-key groups 512 B apart.
        const uint32_t pb0 = ptx::smem_u32(&S.pb[0][0]);
#pragma unroll
        for (int st = 0; st < kKT / 16; ++st) {
#pragma unroll
          for (int m = 0; m < 4; ++m)
            ptx::mma_f16_ss(T0 + kColO + kOStride * m,
                            ptx::sdesc(ptx::smem_u32(S.lat[buf][2 * m]) + 2048 * st, 16384, 1024, 2),
                            ptx::sdesc(pb0 + 1024 * st, 512, 128, 0), id_pv, !first || st > 0);
        }
        ptx::mma_commit(&S.pv_done);
        ptx::mma_commit(&S.lat_free[buf]);
        return;
      }
#pragma unroll
      for (int st = 0; st < kKT / 32; ++st) {
#pragma unroll
        for (int b = 0; b < 4; ++b)
          ptx::mma_f8f6f4_ss(T0 + kColO + kOStride * b,
                             ptx::sdesc(ptx::smem_u32(S.lat[buf][b]) + 4096 * st, 16384, 1024, 2),
                             ptx::sdesc(ptx::smem_u32(S.pb[b]) + 1536 * st, 384, 128, 0), id_pv,
                             !first || st > 0);
      }
      ptx::mma_commit(&S.pv_done);
      ptx::mma_commit(&S.lat_free[buf]);
    };
    // Two cursors over the CTA's tiles: the next QK^T and the next PV.  A
    // tile's QK^T needs its rows, the softmax done reading the last S (S is
    // one accumulator) and, for the first tile of a (token, head group), the
    // staged query; its PV needs its weights and, for the first tile of a
    // (token, head group) after the first, the epilogue of the one before
    // done reading O.  Whichever is ready goes first; QK^T runs at most one
    // tile ahead of PV.
    Cur cq, cv;
    cur_start(cq, P, ub, ue);
    cur_start(cv, P, ub, ue);
    bool ok = true;
    uint32_t idle = 0;
    while (ok && cv.valid) {
      int act = 0;   // 1: PV of cv, 2: QK^T of cq, -1: gave up
      if (lane == 0) {
        const bool pv_first = cv.jj == 0 && cv.seg > 0;
        const bool pv_ready = cv.k < cq.k && ptx::mbar_test_wait(&S.p_full, cv.k & 1) &&
                              (!pv_first || ptx::mbar_test_wait(&S.o_free, (cv.seg - 1) & 1));
        if (pv_ready) {
          act = 1;
        } else if (cq.valid && cq.k <= cv.k + 1 && (cq.jj > 0 || ptx::mbar_test_wait(&S.q_ready, cq.seg & 1)) &&
                   ptx::mbar_test_wait(&S.full[cq.k % kBufs], (cq.k / kBufs) & 1) &&
                   (cq.k == 0 || ptx::mbar_test_wait(&S.s_free, (cq.k - 1) & 1))) {
          act = 2;
        } else if (*abort || ++idle > (1u << 22)) {
          act = -1;
        } else {
          // sleep on the barrier the next step most likely waits for
          if (cv.k < cq.k) ptx::mbar_try_wait_ns(&S.p_full, cv.k & 1, 200);
          else if (cq.valid) ptx::mbar_try_wait_ns(&S.full[cq.k % kBufs], (cq.k / kBufs) & 1, 200);
        }
        if (act == 1) {
          ptx::tc_fence_after();
          issue_pv(cv.k, cv.jj == 0);
        } else if (act == 2) {
          // the copies are generic-proxy writes: order them before the MMAs' reads
          ptx::fence_proxy_async();
          ptx::tc_fence_after();
          issue_qk(cq.k % kBufs);
        }
      }
      act = __shfl_sync(0xffffffffu, act, 0);
      if (act == 1) {
        cur_next(cv, P, ue);
        idle = 0;
      } else if (act == 2) {
        cur_next(cq, P, ue);
        idle = 0;
      } else if (act < 0) {
        ok = false;
      }
    }
    if (lane == 0) {
      if (!ok) *abort = 1;
      // every MMA this thread issued has finished before TMEM is released
      ptx::mma_commit(&S.drain);
      ptx::mbar_wait(&S.drain, 0, nullptr, 100000u);
    }
    __syncwarp();
  } else {
    // ================= softmax: warps 0-15 =================
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    // TMEM lane quarter (keys, and latent dims in the epilogue) and head
    // quarter: this thread owns key (or dim) `row` for heads 4 hq .. 4 hq + 3.
    const int q4 = warp & 3, hq = warp >> 2;
    const int row = 32 * q4 + lane;
    const int tid = threadIdx.x;                // 0 .. 511
    const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
    // The query of a (token, head group) is staged (by warps 0-7), and
    // q_ready signalled, before the epilogue of the non-empty one before it:
    // the MMA issues the first QK^T of the next before the last PV of the
    // current, and that PV is what the epilogue waits for.
    auto signal_query = [&]() {
      if (warp < kStageWarps) {
        ptx::fence_proxy_async();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&S.q_ready);
      }
    };
    auto stage = [&](const Seg& s) {
      if (warp < kStageWarps) stage_query<kFmt>(P, S, s.t, s.g, tid);
      signal_query();
    };
    // The query of the range's first (token, head group) is an input, not
    // the selection: staged before the previous kernel has finished, and
    // signalled once that (token, head group) turns out to hold keys.
    long long pre_tg = (ub / plan.tpt) * plan.hg + (int)blockIdx.x % plan.hg;
    if (warp < kStageWarps) stage_query<kFmt>(P, S, (int)(ub / plan.tpt), (int)blockIdx.x % plan.hg, tid);
    int k = 0;
    bool ok = true, staged = false;
    for (long long u = ub; u < ue;) {
      const Seg s = segment_at(P, u, ue);
      u += s.nj;
      // every softmax thread is done with the last (token, head group): its S.qs and S.xsum
      ok = softmax_all(ok);
      if (!ok) break;
      float* pout = P.ws.part_out + s.slot * kHC * SML_LATENT_DIM;
      float* plse = P.ws.part_lse + s.slot * kHC;
      if (s.ne == 0) {
        // no selected key in this CTA's tiles of it: an empty partial (lse = -inf drops out of the merge)
        for (int i = tid; i < kHC * SML_LATENT_DIM; i += kSoftmaxThreads) pout[i] = 0.f;
        if (tid < kHC) plse[tid] = -INFINITY;
        continue;
      }
      if (!staged) {
        if (s.tg == pre_tg) signal_query();
        else stage(s);
      }
      pre_tg = -1;
      staged = false;
      ok = softmax_all(ok);   // S.qs visible to every softmax thread
      float qsh[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) qsh[h] = S.qs[4 * hq + h];
      // logits in log2 units: z log2(e), so that p = 2^(z - M)
      const float zscale = P.sm_scale * (P.ssmax ? P.ssmax_s * logf((float)s.nss) : 1.f) * kLog2e;
      // Per head of this quarter (identical in all its threads): the integer
      // exponent M_h the weights are taken against (-inf until the head's
      // first key), and this key row's share of the row sum, in units of 2^M_h.
      float M[4], lrow[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        M[h] = -INFINITY;
        lrow[h] = 0.f;
      }
      for (int jj = 0; jj < s.ne; ++jj, ++k) {
        const int buf = k % kBufs;
        ok = ok && warp_wait(&S.full[buf], (k / kBufs) & 1, abort) && warp_wait(&S.s_full, k & 1, abort);
        if (!ok) *abort = 1;
        ok = softmax_all(ok);
        if (!ok) break;
        ptx::tc_fence_after();
        const bool valid = S.rowid[k & 3][row] >= 0;
        // this key's block scales (plain pool: one scale, 0 for a masked key)
        const float* scr = &S.sc[buf][row][0];
        const float psc = valid ? P.latent_scale : 0.f;
        // z = zscale * (s_h * sum_b scale_b (S_b,hi + S_b,lo) + S_pe), fp32
        float z[4] = {0.f, 0.f, 0.f, 0.f};
        if constexpr (kBf) {
          // bf16: one accumulator holds the whole dot product, RoPE included
          uint32_t v[4];
          ptx::tmem_ld4(T0 + kColS + 4 * hq + lane_off, v);
          ptx::tmem_wait_ld(v);
#pragma unroll
          for (int h = 0; h < 4; ++h) z[h] = __uint_as_float(v[h]);
        }
#pragma unroll
        for (int b = 0; b < (kBf ? 0 : 4); ++b) {
          uint32_t vh[4], vl[4];
          ptx::tmem_ld4(T0 + kColS + 32 * b + 4 * hq + lane_off, vh);
          ptx::tmem_ld4(T0 + kColS + 32 * b + kHC + 4 * hq + lane_off, vl);
          ptx::tmem_wait_ld(vh, vl);
          const float scb = kPlain ? psc : scr[b];
#pragma unroll
          for (int h = 0; h < 4; ++h) z[h] = fmaf(scb, __uint_as_float(vh[h]) + __uint_as_float(vl[h]), z[h]);
        }
#pragma unroll
        for (int h = 0; h < 4; ++h) z[h] *= qsh[h];
        if (P.rope_dim && !kBf) {
          if (kPlain) {
            // RoPE codes under the pool scale, both query terms
            uint32_t vh[4], vl[4];
            ptx::tmem_ld4(T0 + kColSpe + 4 * hq + lane_off, vh);
            ptx::tmem_ld4(T0 + kColSpe + kHC + 4 * hq + lane_off, vl);
            ptx::tmem_wait_ld(vh, vl);
#pragma unroll
            for (int h = 0; h < 4; ++h)
              z[h] = fmaf(qsh[h] * P.latent_scale, __uint_as_float(vh[h]) + __uint_as_float(vl[h]), z[h]);
          } else {
            uint32_t v[4];
            ptx::tmem_ld4(T0 + kColSpe + 4 * hq + lane_off, v);
            ptx::tmem_wait_ld(v);
#pragma unroll
            for (int h = 0; h < 4; ++h) z[h] += __uint_as_float(v[h]);
          }
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&S.s_free);   // S read: the next tile's QK^T may overwrite it
#pragma unroll
        for (int h = 0; h < 4; ++h) z[h] = valid ? z[h] * zscale : -INFINITY;
        // This key's weights x_b = 2^(z - M_h) scale_b must stay within
        // E4M3's 448: with this key's largest scale, each head's bound is
        // 2^(z - M_h + lk).  A bound above the cap, or a head without M_h yet,
        // sends the quarter's four warps through the exact update (a vote:
        // after the first tile it is rare, so most tiles exchange nothing
        // between warps here).
        // (bf16: no scales and no overflow: the bound only keeps 2^(z - M_h)
        // within 2^kBfCap, M_h set at the tile's maximum)
        const float kmax = kBf ? 1.f : kPlain ? psc : fmaxf(fmaxf(scr[0], scr[1]), fmaxf(scr[2], scr[3]));
        const float lk = kBf ? 0.f : kmax > 0.f ? lg2(kmax) : -INFINITY;
        constexpr float kCap = kBf ? kBfLog2Cap : kLog2Cap, kHead = kBf ? 0.f : kLog2Head;
        bool need = false;
#pragma unroll
        for (int h = 0; h < 4; ++h) need = need || (z[h] != -INFINITY && !(z[h] - M[h] + lk <= kCap));
        need = group_any(hq, need);
        float f[4] = {1.f, 1.f, 1.f, 1.f};
        bool any = false;
        if (need) {
          // Exact tile statistics: each head's largest logit over the 128
          // keys and the tile's largest block scale (masked rows: scale 0).
          float* xm = S.xmax[k & 1][hq][q4];
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const float w = ptx::warp_max_f32(z[h]);
            if (lane == 0) xm[h] = w;
          }
          const float scw = ptx::warp_max_f32(kmax);
          if (lane == 0) xm[4] = scw;
          group_sync(hq);
          float tm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY}, SC = 0.f;
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            const float* x = S.xmax[k & 1][hq][qq];
#pragma unroll
            for (int h = 0; h < 4; ++h) tm[h] = fmaxf(tm[h], x[h]);
            SC = fmaxf(SC, x[4]);
          }
          // A head whose bound 2^(tmax_h - M_h) SC exceeds the cap (or that
          // has no M_h) takes the integer M_h that puts it in (56, 112]: 4x
          // headroom for later tiles, and the dominant weights keep all 12
          // bits of the three-term split (a weight of at least 4 does).  M_h
          // is never lowered.  O and the row sums scale by f_h =
          // 2^(M_old - M_new), exactly.
          const float lsc = SC > 0.f ? lg2(SC) : -INFINITY;
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const float e = tm[h] + lsc;
            if (tm[h] != -INFINITY && !(e - M[h] <= kCap)) {
              const float Mn = ceilf(e - kHead);
              if (M[h] != -INFINITY) {
                const float d = M[h] - Mn;   // a negative integer
                f[h] = d < -126.f ? 0.f : __int_as_float((127 + (int)d) << 23);
                lrow[h] *= f[h];
                any = true;
              }
              M[h] = Mn;
            }
          }
        }
        // The previous tile's PV reads the weight tiles and accumulates into
        // O: wait for it before rescaling O or overwriting the weights (the
        // previous (token, head group)'s last PV was waited for by its
        // epilogue).
        if (jj > 0) {
          ok = warp_wait(&S.pv_done, (k - 1) & 1, abort);
          if (!ok) {
            *abort = 1;
            continue;   // the next softmax_all ends every softmax warp
          }
          if (any) {
            ptx::tc_fence_after();   // TMEM accesses after the wait (none when nothing is rescaled)
#pragma unroll 1
            for (int b = 0; b < 4; ++b) {   // this thread: latent dim 128 b + row, this quarter's heads
              uint32_t ov[3][4];
              const uint32_t a = T0 + kColO + kOStride * b + 4 * hq + lane_off;
#pragma unroll
              for (int term = 0; term < kTerms; ++term) ptx::tmem_ld4(a + kHC * term, ov[term]);
              ptx::tmem_wait_ld(ov[0], ov[1]);
              if (kTerms > 2) ptx::reg_fence(ov[2]);
#pragma unroll
              for (int term = 0; term < kTerms; ++term) {
#pragma unroll
                for (int h = 0; h < 4; ++h) ov[term][h] = __float_as_uint(__uint_as_float(ov[term][h]) * f[h]);
                ptx::tmem_st4(a + kHC * term, ov[term]);
              }
            }
            ptx::tmem_wait_st();
          }
        }
        // p = 2^(z - M) (0 for a masked key); weights x = p * scale_b as hi + mid + lo (E4M3)
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float p = z[h] == -INFINITY ? 0.f : ex2(z[h] - M[h]);
          lrow[h] += p;
          z[h] = p;
        }
        if constexpr (kBf) {
          // bf16 weights as hi + lo (bf16 each: 16 significant bits): B is
          // 8-key x 16-B core matrices of 8 heads, (term, head half) 128 B
          // apart, 8-key groups 512 B apart
          uint32_t hi[2], lo[2];
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const __nv_bfloat162 hv = __floats2bfloat162_rn(z[2 * i], z[2 * i + 1]);
            const float2 hf = __bfloat1622float2(hv);
            const __nv_bfloat162 lv = __floats2bfloat162_rn(z[2 * i] - hf.x, z[2 * i + 1] - hf.y);
            hi[i] = *reinterpret_cast<const uint32_t*>(&hv);
            lo[i] = *reinterpret_cast<const uint32_t*>(&lv);
          }
          const uint32_t pb = ptx::smem_u32(&S.pb[0][0]) + (row >> 3) * 512 + (hq >> 1) * 128 + (row & 7) * 16 + (hq & 1) * 8;
          st_shared_v2(pb, hi[0], hi[1]);
          st_shared_v2(pb + 256, lo[0], lo[1]);
        }
        const uint32_t pb_off = (row >> 3) * 384 + (row & 7) * 16 + 4 * hq;
#pragma unroll
        for (int b = 0; b < (kBf ? 0 : 4); ++b) {
          const float scb = kPlain ? psc : scr[b];
          uint32_t h01, m01, l01, h23, m23, l23;
          split3_e4m3x2(z[0] * scb, z[1] * scb, h01, m01, l01);
          split3_e4m3x2(z[2] * scb, z[3] * scb, h23, m23, l23);
          const uint32_t pb = ptx::smem_u32(S.pb[b]) + pb_off;
          st_shared_b32(pb, h01 | (h23 << 16));
          st_shared_b32(pb + 128, m01 | (m23 << 16));
          st_shared_b32(pb + 256, l01 | (l23 << 16));
        }
        ptx::fence_proxy_async();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&S.p_full);
      }
      // the next non-empty (token, head group)'s query
      for (long long v = u; ok && v < ue;) {
        const Seg nx = segment_at(P, v, ue);
        v += nx.nj;
        if (nx.ne > 0) {
          stage(nx);
          staged = true;
          break;
        }
      }
      // ---- epilogue of this (token, head group) ----
      ok = ok && warp_wait(&S.pv_done, (k - 1) & 1, abort);
      if (!ok) *abort = 1;
      ok = softmax_all(ok);
      if (!ok) break;
      ptx::tc_fence_after();
      // row sums over the 128 keys (the quarter's four warps)
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        float v = lrow[h];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) S.xsum[hq][q4][h] = v;
      }
      group_sync(hq);
      float osc[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float l = S.xsum[hq][0][h] + S.xsum[hq][1][h] + S.xsum[hq][2][h] + S.xsum[hq][3][h];
        osc[h] = l > 0.f ? 1.f / l : 0.f;
        if (q4 == 0 && lane == h) plse[4 * hq + h] = l > 0.f ? (M[h] + log2f(l)) * kLn2 : -INFINITY;
      }
      // out = (hi + mid + lo) / l_h: this thread's latent dim 128 b + row
#pragma unroll 1
      for (int b = 0; b < 4; ++b) {
        uint32_t o3[3][4];
        const uint32_t a = T0 + kColO + kOStride * b + 4 * hq + lane_off;
#pragma unroll
        for (int term = 0; term < kTerms; ++term) ptx::tmem_ld4(a + kHC * term, o3[term]);
        ptx::tmem_wait_ld(o3[0], o3[1]);
        if (kTerms > 2) ptx::reg_fence(o3[2]);
        const int dim = 128 * b + row;
#pragma unroll
        for (int h = 0; h < 4; ++h)
          pout[(size_t)(4 * hq + h) * SML_LATENT_DIM + dim] =
              (__uint_as_float(o3[0][h]) + __uint_as_float(o3[1][h]) + (kTerms > 2 ? __uint_as_float(o3[2][h]) : 0.f)) *
              osc[h];
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&S.o_free);
    }
    if (!ok) *abort = 1;
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && S.abort) raise_fault(P.status, SML_FAULT_TIMEOUT);
  if (warp == kWarpMma) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(S.tmem_base, 512);
  }
}

static_assert(SML_MAX_TOPK / kKT + 1 <= 32, "a (token, head group) has at most one partial per lane");

// out[t,h,:] = sum_s exp(lse_s - lse) O_s,  lse = ln sum_s exp(lse_s), over
// the partials of every CTA whose range touched (t, h's head group).  One
// block per (head, token); every warp works out the partials' weights (lane s
// holds partial s, at most 32 of them), then each thread gathers its four
// dims of all partials with the loads issued four partials at a time.
__global__ void __launch_bounds__(128)
lse_merge_kernel(int H, MlaWs ws, float* __restrict__ out, float* __restrict__ lse) {
  const int h = blockIdx.x, t = blockIdx.y, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) ptx::griddep_launch_dependents();
  ptx::griddep_wait();   // the partials come from the previous kernel
  const MlaPlan& m = ws.plan;
  const int tg = t * m.hg + h / kHC, hl = h % kHC;
  const long long u0 = (long long)t * m.tpt;   // the token's first unit in its head group
  const int n = cta_of(m, u0 + m.tpt - 1) - cta_of(m, u0) + 1;   // <= tiles per token + 1 <= 32
  const size_t base = (size_t)tg * m.smax;
  const float ls = lane < n ? __ldcg(ws.part_lse + (base + lane) * kHC + hl) : -INFINITY;
  float mx = ls;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const float w = (mx == -INFINITY || ls == -INFINITY) ? 0.f : expf(ls - mx);
  float den = w;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  const float inv = den > 0.f ? 1.f / den : 0.f;
  const float4* po = reinterpret_cast<const float4*>(ws.part_out + (base * kHC + hl) * SML_LATENT_DIM) + threadIdx.x;
  const size_t pstride = (size_t)kHC * SML_LATENT_DIM / 4;   // float4s from one partial to the next
  float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < n; s0 += 4) {
    float4 v[4];
    float ws4[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      ws4[i] = __shfl_sync(0xffffffffu, w, (s0 + i) & 31);
      v[i] = (s0 + i < n && ws4[i] != 0.f) ? __ldcg(po + (size_t)(s0 + i) * pstride) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float wi = s0 + i < n ? ws4[i] : 0.f;
      o.x = fmaf(wi, v[i].x, o.x);
      o.y = fmaf(wi, v[i].y, o.y);
      o.z = fmaf(wi, v[i].z, o.z);
      o.w = fmaf(wi, v[i].w, o.w);
    }
  }
  o.x *= inv;
  o.y *= inv;
  o.z *= inv;
  o.w *= inv;
  reinterpret_cast<float4*>(out + ((size_t)t * H + h) * SML_LATENT_DIM)[threadIdx.x] = o;
  if (threadIdx.x == 0) lse[(size_t)t * H + h] = den > 0.f ? mx + logf(den) : -INFINITY;
}

}  // namespace

MlaPlan mla_plan(const sml_problem& p) {
  MlaPlan m;
  m.hg = p.num_heads / kHC;
  m.tpt = (p.topk + kKT - 1) / kKT;
  m.units = (long long)p.num_tokens * m.tpt;
  if (m.units < 1) {
    m.cpg = 0;
    m.ctas = 0;
    m.smax = 1;
    return m;
  }
  // Per head group, as few CTAs as give the same longest range: ceil(units /
  // its share of the SMs) units per CTA at most.  (On decode, all SMs
  // gathering at once only adds contention at the memory for the same
  // finishing time.)
  const long long sms = device_sm_count();
  const long long share = sms / m.hg > 0 ? sms / m.hg : 1;
  const long long most = (m.units + share - 1) / share;
  m.cpg = (int)((m.units + most - 1) / most);
  m.ctas = m.hg * m.cpg;
  // every CTA holds at least `per` units, so a run of tpt units touches at
  // most 1 + ceil((tpt - 1) / per) CTAs
  const long long per = m.units / m.cpg;
  m.smax = (int)((m.tpt - 1 + per - 1) / per) + 1;
  return m;
}

cudaError_t launch_sparse_mla(const sml_problem& p, const uint16_t* q, const sml_cache& latent,
                              const int32_t* idx, const int32_t* idx_len,
                              float* out, float* lse, const MlaWs& ws, int32_t* status,
                              cudaStream_t stream) {
  if (latent.num_pages > (int64_t)(INT32_MAX / SML_PAGE_TOKENS)) return cudaErrorInvalidValue;   // int32 row ids
  Params P;
  P.B = p.num_requests;
  P.T = p.num_tokens;
  P.H = p.num_heads;
  P.K = p.topk;
  P.rope_dim = p.rope_dim;
  P.max_ctx = p.max_ctx;
  P.max_pages = p.max_pages;
  P.ssmax = p.ssmax;
  P.sm_scale = p.sm_scale;
  P.ssmax_s = p.ssmax_s;
  P.cu_q = p.cu_q;
  P.ctx_len = p.ctx_len;
  P.block_table = p.block_table;
  P.vis_len = p.vis_len;
  P.ssmax_len = p.ssmax_len;
  P.q = q;
  P.latent = static_cast<const uint8_t*>(latent.base);
  P.latent_pages = latent.num_pages;
  const bool plain = latent.format == SML_LATENT_E4M3;
  P.latent_scale = plain ? latent.scale : 1.f;
  P.idx = idx;
  P.idx_len = idx_len;
  P.ws = ws;
  P.status = status;
  const bool bf16 = latent.format == SML_LATENT_BF16;
  const size_t smem = (bf16 ? sizeof(Smem<kFmtBf16>) : plain ? sizeof(Smem<kFmtPlain>) : sizeof(Smem<kFmtDsMla>)) + 1024;
  auto kernel = bf16 ? sparse_mla_kernel<kFmtBf16> : plain ? sparse_mla_kernel<kFmtPlain> : sparse_mla_kernel<kFmtDsMla>;
  cudaError_t e = set_max_smem(reinterpret_cast<const void*>(kernel), smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kernel, dim3(ws.plan.ctas), dim3(kThreads), smem, stream, 0, P);
  if (e != cudaSuccess) return e;
  return launch_pdl(lse_merge_kernel, dim3(p.num_heads, p.num_tokens), dim3(128), 0, stream, 0, p.num_heads, ws,
                    out, lse);
}

}  // namespace sml
