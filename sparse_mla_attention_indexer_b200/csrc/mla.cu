// Absorbed-query sparse MLA over a paged fp8_ds_mla latent cache on the sm_100a
// tensor cores, split over the selected keys, then a log-sum-exp merge.
//
// vLLM blog "vLLM 首日支持 Mistral Large 4": highlights list (MLA, KV LoRA
// rank 512, RoPE dim 64, top-2048 keys per query); section "实现细节 / 模型架构"
// (sparse MLA over the fp8_ds_mla latent cache; NoPE = RoPE dim 0 on the same
// cache; SSMax on the MLA query); section "长上下文" (partial results merged by
// their LSE).  For token t, head h over the selected set S_t:
//   z_i = sm_scale * c_t * (q_nope . c_hat_i + q_pe . k_pe_i)
//   out = sum_i softmax(z)_i c_hat_i,   lse = ln sum_i exp(z_i)
// with c_hat_i = e4m3 latent x its 128-element block scale.
//
// One CTA = (query token, group of 16 heads, split of up to 512 selected keys),
// in tiles of 128 keys; keys are the MMA M dimension of QK^T and its K
// dimension of PV, the 16 heads N (an MMA costs at least ~45 cycles whatever
// its N, and 16 heads as M would waste 3/4 of the smallest M).  Both products
// run on kind::f8f6f4 straight from the gathered E4M3 latent tile: nothing of
// the latent is ever converted.
//   * warps 4-14 gather the selected 656-B rows, eight rows per warp batch
//     (16-B register loads, one row per warp instruction), into
//     128-B-swizzled tiles: E4M3 latent, bf16 RoPE key, block scales aside;
//     two tile buffers.  Random rows need many loads in flight per SM, hence
//     many gather warps and deep batches;
//   * warp 15 issues the MMAs:
//       S_b^T = C_b . [Qhi_b; Qlo_b]^T  (K-major; N = 32: both query terms),
//       S_pe^T = K_pe . Q_pe^T          (kind::f16, bf16),
//       O_b^T += C_b^T . [Bhi_b; Bmid_b; Blo_b]^T  (C_b^T read MN-major from
//       the same tile; N = 48: the three weight terms);
//     the next tile's QK^T goes in ahead of this tile's PV, as soon as its
//     rows have landed and the softmax has read S;
//   * warps 0-3 (one thread per key) run the softmax on S^T and build the
//     weights B_b[i, h] = p_ih scale_ib / sigma_h as three E4M3 terms whose
//     sum carries 12 significant bits (finer than fp16); sigma_h is a per-head
//     power of two that keeps the terms in range, raised (and O rescaled,
//     exactly) only when a tile would overflow; at the end they read O^T back
//     (one thread per latent dim) and write the split's output and LSE.
// The query is split exactly into two E4M3 terms sharing a power-of-two scale
// per head; products of E4M3 values are exact and accumulate in fp32.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <math.h>

#include "ptx.cuh"
#include "sml_internal.cuh"

namespace sml {
namespace {

constexpr int kHC = 16;          // heads per CTA
constexpr int kKT = 128;         // keys per tile
constexpr int kMaxSplit = 512;   // keys per split (4 tiles)
constexpr int kThreads = 512;    // warps 0-3 softmax, 4-14 gather, 15 MMA
constexpr int kGatherWarps = 11;
constexpr int kBatchRows = 8;                     // rows per gather batch (16 loads in flight per thread)
constexpr int kBatchesPerTile = 128 / kBatchRows;  // >= kGatherWarps: every gather warp has a batch in every tile
static_assert(kBatchesPerTile >= kGatherWarps, "a gather warp without a batch in a tile would never signal it");
constexpr int kWarpMma = 15;
constexpr float kLazyRescale = 8.f;   // nats

// TMEM columns
constexpr uint32_t kColS = 0;       // S_b^T (lanes = keys): 32 columns per block b (hi | lo query term)
constexpr uint32_t kColSpe = 128;   // S_pe^T
constexpr uint32_t kColO = 256;     // O_b^T (lanes = dims of block b): 48 columns (hi | mid | lo) ...
constexpr uint32_t kOStride = 64;   // ... at kColO + kOStride b
constexpr int kPBytes = kKT * 3 * kHC;   // one block's weight terms: 128 keys x 48 E4M3

struct __align__(1024) Smem {
  uint8_t lat[2][4][kKT * 128];  // [buffer][block b][128 keys x 128 B] E4M3, SW128
  uint8_t pe[2][kKT * 128];      // [buffer][128 keys x 64 bf16], SW128
  uint8_t q8[4][2 * kHC * 128];  // [block] 32 rows x 128 B, SW128: rows 0-15 high term, 16-31 low term
  uint8_t qpe[kHC * 128];        // query RoPE bf16 [16 heads x 64], SW128
  uint8_t pb[4][kPBytes];        // weight terms of block b, MN-major 8-key x 16-B core matrices
  float xch[kKT * kHC];          // softmax column-reduction exchange
  float sc[2][kKT][4];           // [buffer][key][block] scales of the staged tile
  float qs[kHC];                 // power-of-two query scale per head
  float hstat[kHC];              // per-head row sum (epilogue)
  float hm[kHC];                 // per-head running max m_h
  float hsig[kHC];               // per-head weight scale sigma_h (a power of two; 0 = not set yet)
  float halpha[kHC];             // this tile's exp(m_old - m_new)
  float hf[kHC];                 // this tile's rescale factor of O
  float hinv[kHC];               // 1 / sigma_h (0 while unset)
  float hosc[kHC];               // epilogue: sigma_h / l_h, the output scale of head h
  float scw[2][4];               // per-warp max of the tile's scales (double-buffered by tile)
  int32_t rowid[kMaxSplit];      // pool row (page * 64 + row) of each key, -1 = masked
  uint64_t e_full[2], e_free[2];
  uint64_t q_ready, s_full, s_free, p_full, pv_done, drain;
  uint32_t tmem_base;
  int abort;
};

struct Params {
  int B, T, H, K, rope_dim, max_ctx, max_pages, ssmax;
  float sm_scale, ssmax_s;
  const int32_t* cu_q;
  const int32_t* ctx_len;
  const int32_t* block_table;
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

// 16-B global load that does not allocate in L1 (each row is read once).
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Round two floats to E4M3 (nearest even, saturating); the codes, low byte = a.
__device__ __forceinline__ uint32_t f2_to_e4m3x2(float a, float b) {
  return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3) & 0xffffu;
}

__device__ __forceinline__ float2 e4m3x2_to_f2(uint32_t two) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two & 0xffffu), __NV_E4M3);
  return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

// Two floats that are bf16 values -> their bf16 bits, low half = a.
__device__ __forceinline__ uint32_t bf16x2_bits(float a, float b) {
  return (__float_as_uint(a) >> 16) | (__float_as_uint(b) & 0xffff0000u);
}

// x (two values) -> E4M3 codes of the nearest value and the exact residual.
__device__ __forceinline__ uint32_t split_e4m3x2(float& x0, float& x1) {
  const uint32_t c = f2_to_e4m3x2(x0, x1);
  const float2 r = e4m3x2_to_f2(c);
  x0 -= r.x;
  x1 -= r.y;
  return c;
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const volatile int* abort) {
  const bool ok = ptx::mbar_wait(bar, parity, abort);
  return __all_sync(0xffffffffu, ok);
}

// AND of a flag over the four softmax warps (named barrier 1): every wait
// outcome is made uniform across them before the next named barrier, so a
// timed-out wait ends all four together instead of leaving three behind.
__device__ __forceinline__ bool softmax_all(bool ok) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, 1, 128, p;\n selp.u32 %0, 1, 0, q;\n}"
      : "=r"(r)
      : "r"((uint32_t)ok)
      : "memory");
  return r != 0;
}

// Softmax exchange buffer: [128 keys][16] floats, columns XOR-swizzled by key.
__device__ __forceinline__ float* xbuf(Smem& S, int key, int col) {
  return S.xch + key * kHC + (col ^ (key & 15));
}

// Sum (or max) over the 128 keys of 16 per-key values (warps 0-3); every
// softmax thread reads the 16 results from S.hstat afterwards.  Shared writes
// made before the call are visible to all four warps after it.
template <bool kMax>
__device__ __forceinline__ void column_reduce(Smem& S, int row, const float (&v)[kHC]) {
#pragma unroll
  for (int h = 0; h < kHC; ++h) *xbuf(S, row, h) = v[h];
  asm volatile("bar.sync 1, 128;" ::: "memory");
  const int hh = row >> 3, part = row & 7;   // head hh, keys part + 8 j
  float acc = kMax ? -INFINITY : 0.f;
#pragma unroll
  for (int j = 0; j < kKT / 8; ++j) {
    const float x = *xbuf(S, part + 8 * j, hh);
    acc = kMax ? fmaxf(acc, x) : acc + x;
  }
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) {
    const float y = __shfl_xor_sync(0xffffffffu, acc, o);
    acc = kMax ? fmaxf(acc, y) : acc + y;
  }
  if (part == 0) S.hstat[hh] = acc;
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

// Per-tile softmax statistics (warps 0-3).  Max over the 128 keys of z; then
// the thread owning head h updates, for that head, the lazily raised running
// max m_h and the weight scale sigma_h: the tile's weights are at most
// exp(tmax_h - m_h) * SC (SC = largest block scale in the tile) and must stay
// <= 448 sigma_h; sigma_h is reset to the next power of two >= U_h / 448
// (U_h below) whenever U_h leaves [28, 448] sigma_h.  O holds
// sum(weights / sigma), so both changes rescale it by
// f_h = exp(m_old - m_new) * sigma_old / sigma_new (exact for the sigma
// part).  Returns whether any f_h != 1.
__device__ __forceinline__ bool tile_stats(Smem& S, int row, const float (&z)[kHC], int tile) {
#pragma unroll
  for (int h = 0; h < kHC; ++h) *xbuf(S, row, h) = z[h];
  asm volatile("bar.sync 1, 128;" ::: "memory");
  const int hh = row >> 3, part = row & 7;
  float tm = -INFINITY;
#pragma unroll
  for (int j = 0; j < kKT / 8; ++j) tm = fmaxf(tm, *xbuf(S, part + 8 * j, hh));
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, o));
  uint32_t changed = 0;
  if (part == 0) {
    const float* w = S.scw[tile & 1];
    const float SC = fmaxf(fmaxf(w[0], w[1]), fmaxf(w[2], w[3]));
    float m = S.hm[hh], sig = S.hsig[hh];
    float alpha = 1.f;
    if (tm > m + kLazyRescale || (m == -INFINITY && tm != -INFINITY)) {
      alpha = m == -INFINITY ? 0.f : expf(m - tm);
      m = tm;
    }
    // Weights that matter are ~SC (p ~ 1 against the running max) or, in a
    // tile above the running max, up to exp(tmax - m) SC; sigma keeps the
    // largest of them within [28, 448] sigma, so the dominant weights keep all
    // 12 bits of the three-term split, and moves only when they leave it.
    const float U = tm == -INFINITY ? 0.f : fmaxf(expf(tm - m), 1.f) * SC;
    float beta = 1.f;
    if (U > 0.f && (U > 448.f * sig || U < 28.f * sig)) {
      int e = 0;
      frexpf(U * (1.f / 448.f), &e);   // U / 448 < 2^e
      const float ns = ldexpf(1.f, e);
      beta = sig > 0.f ? sig / ns : 1.f;
      sig = ns;
    }
    S.hm[hh] = m;
    S.hsig[hh] = sig;
    S.halpha[hh] = alpha;
    S.hf[hh] = alpha * beta;
    S.hinv[hh] = sig > 0.f ? 1.f / sig : 0.f;
    changed = alpha * beta != 1.f;
  }
  uint32_t any;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, 1, 128, p;\n selp.u32 %0, 1, 0, q;\n}"
      : "=r"(any)
      : "r"(changed)
      : "memory");
  return any != 0;
}

// kPlain: the latent pool is plain E4M3 (576-B rows under one scale); else
// fp8_ds_mla.  A template parameter, so that each gather loop is compiled for
// its own row layout.
template <bool kPlain>
__global__ void __launch_bounds__(kThreads, 1) sparse_mla_tc_kernel(const Params P) {
  extern __shared__ uint8_t smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, hg = blockIdx.y, t = blockIdx.z;
  ptx::griddep_wait();   // the selection comes from the previous kernel

  // ---- this split's key range (uniform across the CTA) ----
  const int r = request_of_warp(P.cu_q, P.B, t);
  const Req rq = load_request(P.cu_q, P.ctx_len, r, P.T, P.max_ctx, P.max_pages);
  const bool req_ok = rq.ok && t >= rq.q0 && t - rq.q0 < rq.Q;
  const int n = req_ok ? rq.L - rq.Q + (t - rq.q0) + 1 : 0;
  int len = req_ok ? __ldg(P.idx_len + t) : 0;
  const int len_max = min(P.K, n);
  if (len < 0 || len > len_max) {
    if (split == 0 && hg == 0 && threadIdx.x == 0) raise_fault(P.status, SML_FAULT_TOPK_LEN);
    len = max(0, min(len, len_max));
  }
  if (!req_ok && split == 0 && hg == 0 && threadIdx.x == 0) raise_fault(P.status, SML_FAULT_LENGTHS);
  const int kb = split * P.ws.keys_per_split;
  const int ke = min(len, kb + P.ws.keys_per_split);
  const size_t slot0 = ((size_t)t * P.H + hg * kHC) * P.ws.splits + split;   // + h * splits
  if (kb >= ke) {
    // No selected key in this split: an empty partial (lse = -inf drops out of the merge).
    for (int e = threadIdx.x; e < kHC * SML_LATENT_DIM; e += kThreads)
      P.ws.part_out[(slot0 + (size_t)(e / SML_LATENT_DIM) * P.ws.splits) * SML_LATENT_DIM + e % SML_LATENT_DIM] = 0.f;
    if (threadIdx.x < kHC) P.ws.part_lse[slot0 + (size_t)threadIdx.x * P.ws.splits] = -INFINITY;
    return;
  }
  const int nkeys = ke - kb;
  const int ntiles = (nkeys + kKT - 1) / kKT;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&S.e_full[i], kGatherWarps);   // one arrival per gather warp
      ptx::mbar_init(&S.e_free[i], 1);   // PV of the tile done (it is the tile's last reader)
    }
    ptx::mbar_init(&S.q_ready, 4);
    ptx::mbar_init(&S.s_full, 1);
    ptx::mbar_init(&S.s_free, 4);
    ptx::mbar_init(&S.p_full, 4);
    ptx::mbar_init(&S.pv_done, 1);
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
  // same SM cannot starve it of columns.
  if (threadIdx.x == 0) ptx::griddep_launch_dependents();
  volatile int* abort = &S.abort;
  const uint32_t T0 = S.tmem_base;
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;

  if (warp >= 4 && warp < 4 + kGatherWarps) {
    // ================= gather warps: row offsets, then rows -> swizzled tiles =================
    constexpr int kGT = 32 * kGatherWarps;
    const int ct = threadIdx.x - 128;   // 0 .. kGT - 1
    // Pool rows of the split's keys.
    for (int k = ct; k < kMaxSplit; k += kGT) {
      int32_t id = -1;
      if (k < nkeys) {
        const int pos = __ldg(P.idx + (size_t)t * P.K + kb + k);
        if (pos >= 0 && pos < n) {
          const int ph = __ldg(P.block_table + (size_t)r * P.max_pages + pos / SML_PAGE_TOKENS);
          if (ph >= 0 && ph < P.latent_pages)
            id = ph * SML_PAGE_TOKENS + pos % SML_PAGE_TOKENS;
          else
            raise_fault(P.status, SML_FAULT_PAGE);
        } else {
          raise_fault(P.status, SML_FAULT_INDEX);
        }
      }
      S.rowid[k] = id;
    }
    asm volatile("bar.sync 2, %0;" ::"n"(kGT) : "memory");
    // Rows -> tiles in batches of kBatchRows rows per warp (a tile is
    // kKT / kBatchRows batches; batch i goes to warp i % kGatherWarps): the
    // batch's loads go into registers first (lane l: 16-B latent chunk l, then
    // lane 0 the four scales and lanes 1-8 the RoPE key), then the warp waits
    // for the tile's buffer to be free and stores them 128-B-swizzled, so the
    // loads are in flight while the buffer drains.  A masked row is zeros.  A
    // warp signals a tile after storing its last batch of it.
    const int gw = warp - 4;
    const int nb_total = ntiles * kBatchesPerTile;
    bool ok = true;
    for (int bi = gw; bi < nb_total; bi += kGatherWarps) {
      const int tile = bi / kBatchesPerTile, buf = tile & 1;
      const int row0 = (bi % kBatchesPerTile) * kBatchRows;
      uint4 va[kBatchRows], vb[kBatchRows];
      uint32_t live = 0;   // bit u: row u of the batch is a selected row (plain E4M3 only)
#pragma unroll
      for (int u = 0; u < kBatchRows; ++u) {
        const int32_t id = S.rowid[tile * kKT + row0 + u];
        const uint8_t* src =
            P.latent + (size_t)(id >= 0 ? id : 0) * (kPlain ? SML_LATENT_E4M3_ROW_BYTES : SML_LATENT_ROW_BYTES);
        va[u] = make_uint4(0u, 0u, 0u, 0u);
        vb[u] = make_uint4(0u, 0u, 0u, 0u);
        if (id >= 0) {
          if (kPlain) live |= 1u << u;
          va[u] = ldg_stream(src + 16 * lane);
          // fp8_ds_mla: lane 0 the four block scales, lanes 1-8 the bf16 RoPE
          // key; plain E4M3: lanes 0-3 the 64 RoPE codes
          if (kPlain ? (lane < 4 && P.rope_dim) : (lane == 0 || (lane <= 8 && P.rope_dim)))
            vb[u] = ldg_stream(src + SML_LATENT_DIM + 16 * lane);
        }
      }
      // first batch of this tile for this warp: the buffer must be free (PV of tile - 2 done)
      if (tile >= 2 && bi - kGatherWarps < tile * kBatchesPerTile &&
          !warp_wait(&S.e_free[buf], ((tile >> 1) - 1) & 1, abort)) {
        ok = false;
        break;
      }
      const uint32_t lat_l = ptx::smem_u32(S.lat[buf][lane >> 3]);
      const uint32_t pe_b = ptx::smem_u32(S.pe[buf]);
      const uint32_t sc_b = ptx::smem_u32(&S.sc[buf][0][0]);
#pragma unroll
      for (int u = 0; u < kBatchRows; ++u) {
        const int row = row0 + u;
        st_shared_v4(sw128(lat_l, row, lane & 7), va[u].x, va[u].y, va[u].z, va[u].w);
        if (kPlain) {
          // one scale for every block (zero for a masked row); RoPE codes
          // widened to bf16 (exact: E4M3 values are bf16 values)
          if (lane == 0) {
            const uint32_t sb = (live >> u) & 1 ? __float_as_uint(P.latent_scale) : 0u;
            st_shared_v4(sc_b + row * 16, sb, sb, sb, sb);
          }
          if (lane < 4 && P.rope_dim) {
            const uint32_t w[4] = {vb[u].x, vb[u].y, vb[u].z, vb[u].w};
            uint32_t o[8];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float2 lo = e4m3x2_to_f2(w[k]), hi = e4m3x2_to_f2(w[k] >> 16);
              o[2 * k] = bf16x2_bits(lo.x, lo.y);
              o[2 * k + 1] = bf16x2_bits(hi.x, hi.y);
            }
            st_shared_v4(sw128(pe_b, row, 2 * lane), o[0], o[1], o[2], o[3]);
            st_shared_v4(sw128(pe_b, row, 2 * lane + 1), o[4], o[5], o[6], o[7]);
          }
        } else if (lane == 0) {
          st_shared_v4(sc_b + row * 16, vb[u].x, vb[u].y, vb[u].z, vb[u].w);
        } else if (lane <= 8 && P.rope_dim) {
          st_shared_v4(sw128(pe_b, row, lane - 1), vb[u].x, vb[u].y, vb[u].z, vb[u].w);
        }
      }
      if (bi + kGatherWarps >= (tile + 1) * kBatchesPerTile) {   // this warp's last batch of the tile
        ptx::fence_proxy_async();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&S.e_full[buf]);
      }
    }
    if (!ok) *abort = 1;
  } else if (warp == kWarpMma) {
    // ================= MMA issuer =================
    if (lane == 0) {
      const uint32_t id_qk = ptx::idesc_f16(2 * kHC, 0, 0, 0);   // E4M3 x E4M3, both K-major, N = 32
      const uint32_t id_pe = ptx::idesc_f16(kHC, 1, 0, 0);       // bf16, N = 16
      const uint32_t id_pv = ptx::idesc_f16(3 * kHC, 0, 1, 1);   // E4M3 x E4M3, both MN-major, N = 48
      auto issue_qk = [&](int buf) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {   // 32 latent dims per step
#pragma unroll
          for (int b = 0; b < 4; ++b)
            ptx::mma_f8f6f4_ss(T0 + kColS + 32 * b, ptx::sdesc_sw128(ptx::smem_u32(S.lat[buf][b]) + 32 * k),
                               ptx::sdesc_sw128(ptx::smem_u32(S.q8[b]) + 32 * k), id_qk, k > 0);
          if (P.rope_dim)
            ptx::mma_f16_ss(T0 + kColSpe, ptx::sdesc_sw128(ptx::smem_u32(S.pe[buf]) + 32 * k),
                            ptx::sdesc_sw128(ptx::smem_u32(S.qpe) + 32 * k), id_pe, k > 0);
        }
        ptx::mma_commit(&S.s_full);
      };
      bool ok = ptx::mbar_wait(&S.q_ready, 0, abort) && ptx::mbar_wait(&S.e_full[0], 0, abort);
      if (ok) {
        ptx::tc_fence_after();
        issue_qk(0);
      }
      for (int tile = 0; ok && tile < ntiles; ++tile) {
        const int buf = tile & 1;
        if (tile + 1 < ntiles) {
          // next tile's QK^T once its rows have landed and the softmax has read S
          if (!ptx::mbar_wait(&S.e_full[buf ^ 1], ((tile + 1) >> 1) & 1, abort) ||
              !ptx::mbar_wait(&S.s_free, tile & 1, abort)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          issue_qk(buf ^ 1);
        }
        if (!ptx::mbar_wait(&S.p_full, tile & 1, abort)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        // O_b^T += C_b^T . B_b^T, 32 keys per step.  A: the latent tile read
        // MN-major (dims contiguous; 8-key swizzle atoms 1,024 B apart).  B:
        // 8-key x 16-B core matrices, the three terms 128 B apart, 8-key
        // groups 384 B apart.
#pragma unroll
        for (int k = 0; k < kKT / 32; ++k) {
#pragma unroll
          for (int b = 0; b < 4; ++b)
            ptx::mma_f8f6f4_ss(T0 + kColO + kOStride * b, ptx::sdesc(ptx::smem_u32(S.lat[buf][b]) + 4096 * k, 16384, 1024, 2),
                               ptx::sdesc(ptx::smem_u32(S.pb[b]) + 1536 * k, 384, 128, 0), id_pv, (tile | k) != 0);
        }
        ptx::mma_commit(&S.pv_done);
        ptx::mma_commit(&S.e_free[buf]);
      }
      if (!ok) *abort = 1;
      ptx::mma_commit(&S.drain);
      ptx::mbar_wait(&S.drain, 0, nullptr, 1u << 20);
    }
    __syncwarp();
  } else {
    // ================= softmax: warps 0-3, thread = key row / latent dim =================
    const int row = warp * 32 + lane;
    {
      // Query of the 16 heads.  Nope part: q = s_h (hi + lo), hi and lo E4M3 and
      // s_h a power of two >= amax_h / 448, so q / s_h, its rounding to hi and
      // the residual lo are exact in fp32, and lo is exact in E4M3 (a bf16 has
      // 8 significant bits, hi takes 4, the residual the other 4) down to
      // E4M3's subnormal step.  RoPE part copied as bf16.
      const int Dq = SML_LATENT_DIM + P.rope_dim;
      const int h = row >> 3, part = row & 7;   // 8 threads per head, 64 nope dims each
      const uint16_t* qh = P.q + ((size_t)t * P.H + hg * kHC + h) * Dq;
      uint4 v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = __ldg(reinterpret_cast<const uint4*>(qh + 64 * part) + i);
      uint4 pv = make_uint4(0u, 0u, 0u, 0u);
      if (P.rope_dim) pv = __ldg(reinterpret_cast<const uint4*>(qh + SML_LATENT_DIM) + part);   // 8 bf16
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
        for (int k = 0; k < 4; ++k)
          amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w[k] << 16)), fabsf(__uint_as_float(w[k] & 0xffff0000u))));
      }
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
      int e2 = 0;
      if (amax > 0.f) frexpf(amax / 448.f, &e2);        // amax / 448 < 2^e2
      const float qscale = ldexpf(1.f, e2), inv = ldexpf(1.f, -e2);
      if (part == 0) S.qs[h] = qscale;
      // dims [64 part, 64 part + 64) -> block part / 2, 16-B chunks 4 (part % 2) + c
      const int b = part >> 1;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          // elements 16 c + 4 k .. + 3 of this thread's 64
          const uint4 vv = v[2 * c + (k >> 1)];
          const uint32_t wa = (k & 1) ? vv.z : vv.x, wb = (k & 1) ? vv.w : vv.y;
          float x0 = __uint_as_float(wa << 16) * inv, x1 = __uint_as_float(wa & 0xffff0000u) * inv;
          float x2 = __uint_as_float(wb << 16) * inv, x3 = __uint_as_float(wb & 0xffff0000u) * inv;
          const uint32_t h01 = split_e4m3x2(x0, x1), h23 = split_e4m3x2(x2, x3);
          hw[k] = h01 | (h23 << 16);
          lw[k] = f2_to_e4m3x2(x0, x1) | (f2_to_e4m3x2(x2, x3) << 16);
        }
        const int chunk = 4 * (part & 1) + c;
        st_shared_v4(sw128(ptx::smem_u32(S.q8[b]), h, chunk), hw[0], hw[1], hw[2], hw[3]);
        st_shared_v4(sw128(ptx::smem_u32(S.q8[b]), h + kHC, chunk), lw[0], lw[1], lw[2], lw[3]);
      }
      st_shared_v4(sw128(ptx::smem_u32(S.qpe), h, part), pv.x, pv.y, pv.z, pv.w);
      ptx::fence_proxy_async();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&S.q_ready);
    }
    const float zscale = P.sm_scale * (P.ssmax ? P.ssmax_s * logf((float)max(n, 1)) : 1.f);
    float lrow[kHC];   // this key row's share of the row sums
#pragma unroll
    for (int h = 0; h < kHC; ++h) lrow[h] = 0.f;
    if (row < kHC) {
      S.hm[row] = -INFINITY;
      S.hsig[row] = 0.f;
    }
    bool ok = softmax_all(warp_wait(&S.q_ready, 0, abort));   // S.qs; orders the init above
    for (int tile = 0; ok && tile < ntiles; ++tile) {
      const int buf = tile & 1;
      if (!softmax_all(warp_wait(&S.e_full[buf], (tile >> 1) & 1, abort) && warp_wait(&S.s_full, tile & 1, abort))) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const bool valid = S.rowid[tile * kKT + row] >= 0;
      float sc[4];
#pragma unroll
      for (int b = 0; b < 4; ++b) sc[b] = S.sc[buf][row][b];
      // z = zscale * (s_h * sum_b scale_b (S_b,hi + S_b,lo) + S_pe), fp32
      float z[kHC];
      {
#pragma unroll
        for (int h = 0; h < kHC; ++h) z[h] = 0.f;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          uint32_t v[32];
          ptx::tmem_ld32(T0 + kColS + 32 * b + lane_off, v);
          ptx::tmem_wait_ld(v);
#pragma unroll
          for (int h = 0; h < kHC; ++h) z[h] = fmaf(sc[b], __uint_as_float(v[h]) + __uint_as_float(v[kHC + h]), z[h]);
        }
#pragma unroll
        for (int h = 0; h < kHC; ++h) z[h] *= S.qs[h];
        if (P.rope_dim) {
          // plain E4M3 keys hold codes: their scale multiplies the RoPE term
          const float pe_scale = kPlain ? P.latent_scale : 1.f;
          uint32_t v[16];
          ptx::tmem_ld16(T0 + kColSpe + lane_off, v);
          ptx::tmem_wait_ld(v);
#pragma unroll
          for (int h = 0; h < kHC; ++h) z[h] = fmaf(pe_scale, __uint_as_float(v[h]), z[h]);
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&S.s_free);   // S read: the next tile's QK^T may overwrite it
#pragma unroll
        for (int h = 0; h < kHC; ++h) z[h] = valid ? z[h] * zscale : -INFINITY;
      }
      // the tile's largest block scale (masked rows were zero-filled: scale 0)
      float scm = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) scm = fmaxf(scm, __shfl_xor_sync(0xffffffffu, scm, o));
      if (lane == 0) S.scw[tile & 1][warp] = scm;
      const bool any = tile_stats(S, row, z, tile);
#pragma unroll
      for (int h = 0; h < kHC; ++h) lrow[h] *= S.halpha[h];
      // The previous tile's PV reads the weight tiles and accumulates into O:
      // wait for it before rescaling O or overwriting the weights.
      if (tile > 0) {
        if (!softmax_all(warp_wait(&S.pv_done, (tile - 1) & 1, abort))) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        if (any) {
#pragma unroll 1
          for (int b = 0; b < 4; ++b) {   // this thread: latent dim 128 b + row
            uint32_t ov[32], ow[16];
            ptx::tmem_ld32(T0 + kColO + kOStride * b + lane_off, ov);
            ptx::tmem_ld16(T0 + kColO + kOStride * b + 32 + lane_off, ow);
            ptx::tmem_wait_ld(ov, ow);
#pragma unroll
            for (int h = 0; h < kHC; ++h) {
              const float f = S.hf[h];
              ov[h] = __float_as_uint(__uint_as_float(ov[h]) * f);
              ov[kHC + h] = __float_as_uint(__uint_as_float(ov[kHC + h]) * f);
              ow[h] = __float_as_uint(__uint_as_float(ow[h]) * f);
            }
            ptx::tmem_st32(T0 + kColO + kOStride * b + lane_off, ov);
            ptx::tmem_st16(T0 + kColO + kOStride * b + 32 + lane_off, ow);
          }
          ptx::tmem_wait_st();
        }
      }
      // p = exp(z - m); weights x = p * scale_b / sigma as hi + mid + lo (E4M3)
#pragma unroll
      for (int h = 0; h < kHC; ++h) {
        const float p = z[h] == -INFINITY ? 0.f : expf(z[h] - S.hm[h]);
        lrow[h] += p;
        z[h] = p * S.hinv[h];
      }
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        uint32_t wh[4], wm[4], wl[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {   // heads 4 q .. 4 q + 3
          float x0 = z[4 * q] * sc[b], x1 = z[4 * q + 1] * sc[b];
          float x2 = z[4 * q + 2] * sc[b], x3 = z[4 * q + 3] * sc[b];
          const uint32_t h01 = split_e4m3x2(x0, x1), h23 = split_e4m3x2(x2, x3);
          const uint32_t m01 = split_e4m3x2(x0, x1), m23 = split_e4m3x2(x2, x3);
          wh[q] = h01 | (h23 << 16);
          wm[q] = m01 | (m23 << 16);
          wl[q] = f2_to_e4m3x2(x0, x1) | (f2_to_e4m3x2(x2, x3) << 16);
        }
        const uint32_t pb = ptx::smem_u32(S.pb[b]) + (row >> 3) * 384 + (row & 7) * 16;
        st_shared_v4(pb, wh[0], wh[1], wh[2], wh[3]);
        st_shared_v4(pb + 128, wm[0], wm[1], wm[2], wm[3]);
        st_shared_v4(pb + 256, wl[0], wl[1], wl[2], wl[3]);
      }
      ptx::fence_proxy_async();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&S.p_full);
    }
    ok = softmax_all(ok && warp_wait(&S.pv_done, (ntiles - 1) & 1, abort));
    if (!ok) *abort = 1;
    ptx::tc_fence_after();
    // Row sums over the 128 key lanes, then each head's output scale
    // sigma_h / l_h and its log-sum-exp.
    column_reduce<false>(S, row, lrow);
    if (row < kHC) {
      const float lsum = S.hstat[row];
      S.hosc[row] = lsum > 0.f ? S.hsig[row] / lsum : 0.f;
      P.ws.part_lse[slot0 + (size_t)row * P.ws.splits] = lsum > 0.f ? S.hm[row] + logf(lsum) : -INFINITY;
    }
  }

  // Output, sigma_h (hi + mid + lo) / l_h per head, by every warp but the MMA
  // issuer (the gather warps are idle by now): unit (block b, TMEM lane
  // quarter q) goes to a warp whose quarter is q.  The named barrier orders
  // the last PV (the softmax warps waited for it) and S.hosc before the reads;
  // every path of warps 0-14, a timed-out one included, reaches it.
  if (warp != kWarpMma) {
    asm volatile("bar.sync 3, %0;" ::"n"(32 * kWarpMma) : "memory");
    ptx::tc_fence_after();
    const int q = warp & 3;
    const int nq = (kWarpMma - 1 - q) / 4 + 1;   // warps 0..14 with quarter q
    float osc[kHC];
#pragma unroll
    for (int h = 0; h < kHC; ++h) osc[h] = S.hosc[h];
#pragma unroll 1
    for (int b = warp >> 2; b < 4; b += nq) {
      uint32_t ov[32], ow[16];
      ptx::tmem_ld32(T0 + kColO + kOStride * b + lane_off, ov);
      ptx::tmem_ld16(T0 + kColO + kOStride * b + 32 + lane_off, ow);
      ptx::tmem_wait_ld(ov, ow);
      const int dim = 128 * b + 32 * q + lane;
#pragma unroll
      for (int h = 0; h < kHC; ++h) {
        const float o = __uint_as_float(ov[h]) + __uint_as_float(ov[kHC + h]) + __uint_as_float(ow[h]);
        P.ws.part_out[(slot0 + (size_t)h * P.ws.splits) * SML_LATENT_DIM + dim] = o * osc[h];
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && S.abort) raise_fault(P.status, SML_FAULT_TIMEOUT);
  if (warp == kWarpMma) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(S.tmem_base, 512);
  }
}

// out[t,h,:] = sum_s exp(lse_s - lse) O_s,  lse = ln sum_s exp(lse_s).
__global__ void __launch_bounds__(128)
lse_merge_kernel(int H, MlaWs ws, float* __restrict__ out, float* __restrict__ lse) {
  const int h = blockIdx.x, t = blockIdx.y, S = ws.splits;
  if (threadIdx.x == 0) ptx::griddep_launch_dependents();
  ptx::griddep_wait();   // the partials come from the previous kernel
  const size_t base = ((size_t)t * H + h) * S;
  float mx = -INFINITY;
  for (int s = 0; s < S; ++s) mx = fmaxf(mx, ws.part_lse[base + s]);
  float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
  float den = 0.f;
  if (mx != -INFINITY) {
    for (int s = 0; s < S; ++s) {
      const float ls = ws.part_lse[base + s];
      if (ls == -INFINITY) continue;
      const float w = expf(ls - mx);
      den += w;
      const float4 v = reinterpret_cast<const float4*>(ws.part_out + (base + s) * SML_LATENT_DIM)[threadIdx.x];
      o.x = fmaf(w, v.x, o.x);
      o.y = fmaf(w, v.y, o.y);
      o.z = fmaf(w, v.z, o.z);
      o.w = fmaf(w, v.w, o.w);
    }
    const float inv = 1.f / den;
    o.x *= inv;
    o.y *= inv;
    o.z *= inv;
    o.w *= inv;
  }
  reinterpret_cast<float4*>(out + ((size_t)t * H + h) * SML_LATENT_DIM)[threadIdx.x] = o;
  if (threadIdx.x == 0) lse[(size_t)t * H + h] = den > 0.f ? mx + logf(den) : -INFINITY;
}

}  // namespace

int mla_splits(const sml_problem& p, int* keys_per_split) {
  // Splits of whole 128-key tiles, at most 512 keys: about one CTA per SM for
  // the whole problem, so the per-CTA set-up is paid once per SM and the
  // staging of a tile overlaps the math of the one before.
  const int tiles = (p.topk + kKT - 1) / kKT;
  const int ctas = p.num_tokens * (p.num_heads / kHC);
  int tps = (int)(((long long)ctas * tiles + 148 - 1) / 148);
  tps = tps < 1 ? 1 : (tps > kMaxSplit / kKT ? kMaxSplit / kKT : tps);
  if (tps > tiles) tps = tiles;
  const int kps = tps * kKT;
  if (keys_per_split) *keys_per_split = kps;
  return (p.topk + kps - 1) / kps;
}

cudaError_t launch_sparse_mla(const sml_problem& p, const uint16_t* q, const sml_cache& latent,
                              const int32_t* idx, const int32_t* idx_len,
                              float* out, float* lse, const MlaWs& ws, int32_t* status,
                              cudaStream_t stream) {
  if (latent.num_pages > (int64_t)(INT32_MAX / SML_PAGE_TOKENS)) return cudaErrorInvalidValue;
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
  P.q = q;
  P.latent = static_cast<const uint8_t*>(latent.base);
  P.latent_pages = latent.num_pages;
  const bool plain = latent.format == SML_LATENT_E4M3;
  P.latent_scale = plain ? latent.scale : 1.f;
  P.idx = idx;
  P.idx_len = idx_len;
  P.ws = ws;
  P.status = status;
  const size_t smem = sizeof(Smem) + 1024;
  auto kernel = plain ? sparse_mla_tc_kernel<true> : sparse_mla_tc_kernel<false>;
  cudaError_t e = set_max_smem(reinterpret_cast<const void*>(kernel), smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(kernel, dim3(ws.splits, p.num_heads / kHC, p.num_tokens), dim3(kThreads), smem, stream, 0, P);
  if (e != cudaSuccess) return e;
  return launch_pdl(lse_merge_kernel, dim3(p.num_heads, p.num_tokens), dim3(128), 0, stream, 0, p.num_heads, ws, out,
                    lse);
}

}  // namespace sml
