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
// in tiles of 128 keys; keys are the MMA M dimension and the 16 heads N (an
// MMA costs at least ~45 cycles whatever its N, and 16 heads as M would waste
// 3/4 of the smallest M).
//   * warp 11 gathers the selected 656-B rows, one bulk copy per row, into a
//     ring of 16-row chunks that holds a whole tile;
//   * warps 4-5 copy each row's E4M3 latent and bf16 RoPE key into
//     128-B-swizzled MMA tiles (and the block scales aside);
//   * warps 6-9 (one thread per latent dim) write V^T into TMEM as fp16
//     (E4M3 -> fp16 is exact): the A operand of the PV MMA;
//   * warp 10 issues tcgen05.mma: S_b^T = C_b . Q_b^T per 128-dim block b with
//     kind::f8f6f4 straight from the E4M3 tile (the bf16 query split exactly
//     into two E4M3 terms sharing a power-of-two scale per head, so both
//     accumulate into one fp32 accumulator), the RoPE part with kind::f16
//     (bf16), and after the softmax O_b^T += V_b^T . P'_b^T;
//   * warps 0-3 (one thread per key) run the softmax on S^T: z = sm_scale c_t
//     (sum_b scale_b s_h S_b + S_pe) in fp32, column maxima through shared
//     memory, a lazily raised running max (O rescaled in TMEM only when a
//     head's max grows by more than 8), P'_b = fp16(p x scale_b) and per-block
//     row sums of exactly those weights divided by the scale (so a dominant
//     key's rounding cancels in the normalisation); at the end they read O^T
//     back (one thread per latent dim) and write the split's output and LSE.
// The E4M3 tile is free again as soon as QK^T has read it, so the next tile is
// staged while this one's softmax and PV run.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <math.h>

#include "ptx.cuh"
#include "sml_internal.cuh"

namespace sml {
namespace {

constexpr int kHC = 16;          // heads per CTA (MMA N)
constexpr int kKT = 128;         // keys per tile (MMA M)
constexpr int kMaxSplit = 512;   // keys per split (4 tiles)
constexpr int kChunk = 16;       // rows per gather chunk
constexpr int kRing = kKT / kChunk;   // ring slots: one whole tile
constexpr int kThreads = 384;    // warps 0-3 softmax, 4-5 stage, 6-9 V^T, 10 MMA, 11 gather
constexpr int kStageWarps = 2;
constexpr float kLazyRescale = 8.f;   // nats

// TMEM columns
constexpr uint32_t kColVT = 0;      // V_b^T, fp16 pairs: 64 columns per block b (lanes = dims)
constexpr uint32_t kColS = 256;     // S_b^T (lanes = keys): 16 columns per block b
constexpr uint32_t kColSpe = 320;   // S_pe^T
constexpr uint32_t kColO = 384;     // O_b^T (lanes = dims of block b): 16 columns per block
constexpr uint32_t kColL = 448;     // per-key row-sum partials of block b (lanes = keys)

struct __align__(1024) Smem {
  uint8_t lat[4][kKT * 128];     // [block b][128 keys x 128 B] E4M3, SW128
  uint8_t pe[kKT * 128];         // [128 keys x 64 bf16], SW128
  uint8_t qhi[4][kHC * 128];     // query nope, high E4M3 term [block][16 heads x 128 B], SW128
  uint8_t qlo[4][kHC * 128];     // low E4M3 term
  uint8_t qpe[kHC * 128];        // query RoPE bf16 [16 heads x 64], SW128
  uint8_t p[4][kKT * kHC * 2];   // P'_b fp16, MN-major 8x8 core matrices; p[2..3] double as the exchange buffer
  uint8_t raw[kRing][kChunk * SML_LATENT_ROW_BYTES];
  float sc[kKT][4];              // [key][block] scales of the staged tile
  float qs[kHC];                 // power-of-two query scale per head
  float hstat[kHC];              // per-head tile max / row sum
  int32_t rowid[kMaxSplit];      // pool row (page * 64 + row) of each key, -1 = masked
  uint64_t q_ready, rows_ready, e_full, e_free, s_full, p_full, vt_full, pv_done, drain;
  uint64_t raw_full[kRing], raw_empty[kRing];
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
  const int32_t* idx;
  const int32_t* idx_len;
  MlaWs ws;
  int32_t* status;
};

// Byte address of (row, 16-B chunk) in a 128-B-swizzled K-major tile.
__device__ __forceinline__ uint32_t sw128(uint32_t base, int row, int chunk) {
  return base + (row >> 3) * 1024 + (row & 7) * 128 + ((chunk ^ (row & 7)) << 4);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Two E4M3 codes (low byte first) -> two fp16 values (exact), packed.
__device__ __forceinline__ uint32_t e4m3x2_to_h2(uint32_t two) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two & 0xffffu), __NV_E4M3);
  return (uint32_t)h.x | ((uint32_t)h.y << 16);
}

// Round two floats to E4M3 (nearest even, saturating); the codes, low byte = a.
__device__ __forceinline__ uint32_t f2_to_e4m3x2(float a, float b) {
  return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ float2 e4m3x2_to_f2(uint32_t two) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two & 0xffffu), __NV_E4M3);
  return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const volatile int* abort) {
  const bool ok = ptx::mbar_wait(bar, parity, abort);
  return __all_sync(0xffffffffu, ok);
}

// Softmax exchange buffer: [128 keys][16] floats in P'_2 / P'_3, columns
// XOR-swizzled by key.
__device__ __forceinline__ float* xbuf(Smem& S, int key, int col) {
  return reinterpret_cast<float*>(S.p[2]) + key * kHC + (col ^ (key & 15));
}

// Sum (or max) over the 128 keys of 16 per-key values (warps 0-3); every
// softmax thread reads the 16 results from S.hstat afterwards.
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

__global__ void __launch_bounds__(kThreads, 1) sparse_mla_tc_kernel(const Params P) {
  extern __shared__ uint8_t smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, hg = blockIdx.y, t = blockIdx.z;

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
    ptx::mbar_init(&S.q_ready, 4);
    ptx::mbar_init(&S.rows_ready, kStageWarps);
    ptx::mbar_init(&S.e_full, kStageWarps);
    ptx::mbar_init(&S.e_free, 1 + 4);     // QK done + softmax warps read the scales
    ptx::mbar_init(&S.s_full, 1);
    ptx::mbar_init(&S.p_full, 4);
    ptx::mbar_init(&S.vt_full, 4);
    ptx::mbar_init(&S.pv_done, 1);
    ptx::mbar_init(&S.drain, 1);
    for (int i = 0; i < kRing; ++i) {
      ptx::mbar_init(&S.raw_full[i], 1);
      ptx::mbar_init(&S.raw_empty[i], kStageWarps + 4);   // stage warps + V^T warps
    }
    S.abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 10) {
    ptx::tmem_alloc(&S.tmem_base, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  volatile int* abort = &S.abort;
  const uint32_t T0 = S.tmem_base;
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;

  if (warp >= 4 && warp < 4 + kStageWarps) {
    // ================= stage warps: row offsets, then rows -> swizzled tiles =================
    constexpr int kST = 32 * kStageWarps;
    const int ct = threadIdx.x - 128;   // 0 .. kST - 1
    {
      // Pool rows of the split's keys: all position loads, then all block-table loads.
      constexpr int kPer = kMaxSplit / kST;
      int pos[kPer], ph[kPer];
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int k = ct + j * kST;
        pos[j] = k < nkeys ? __ldg(P.idx + (size_t)t * P.K + kb + k) : -1;
      }
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int k = ct + j * kST;
        const bool in = k < nkeys && pos[j] >= 0 && pos[j] < n;
        if (k < nkeys && !in) raise_fault(P.status, SML_FAULT_INDEX);
        ph[j] = in ? __ldg(P.block_table + (size_t)r * P.max_pages + pos[j] / SML_PAGE_TOKENS) : -1;
        if (!in) pos[j] = -1;
      }
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        int32_t id = -1;
        if (pos[j] >= 0) {
          if (ph[j] >= 0 && ph[j] < P.latent_pages)
            id = ph[j] * SML_PAGE_TOKENS + pos[j] % SML_PAGE_TOKENS;
          else
            raise_fault(P.status, SML_FAULT_PAGE);
        }
        S.rowid[ct + j * kST] = id;
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&S.rows_ready);
    }
    // Rows -> tiles: stage warp w takes rows kRowsPerWarp w .. of each chunk.
    constexpr int kRowsPerWarp = kChunk / kStageWarps;
    const int sw = warp - 4;
    int chunk = 0;
    for (int tile = 0; tile < ntiles; ++tile) {
      if (tile > 0 && !warp_wait(&S.e_free, (tile - 1) & 1, abort)) { *abort = 1; break; }
      bool ok = true;
      for (int cc = 0; cc < kRing; ++cc, ++chunk) {
        const int slot = chunk % kRing;
        if (!warp_wait(&S.raw_full[slot], (chunk / kRing) & 1, abort)) { ok = false; break; }
#pragma unroll
        for (int rr = 0; rr < kRowsPerWarp; ++rr) {
          const int j = kRowsPerWarp * sw + rr; // row within the chunk
          const int row = cc * kChunk + j;      // row within the tile
          const bool valid = S.rowid[tile * kKT + row] >= 0;
          const uint8_t* src = S.raw[slot] + j * SML_LATENT_ROW_BYTES;
          uint4 v = make_uint4(0u, 0u, 0u, 0u);
          if (valid) v = *reinterpret_cast<const uint4*>(src + 16 * lane);
          st_shared_v4(sw128(ptx::smem_u32(S.lat[lane >> 3]), row, lane & 7), v.x, v.y, v.z, v.w);
          if (lane < 8) {
            uint4 e = make_uint4(0u, 0u, 0u, 0u);
            if (valid && P.rope_dim) e = *reinterpret_cast<const uint4*>(src + SML_LATENT_DIM + 16 + 16 * lane);
            st_shared_v4(sw128(ptx::smem_u32(S.pe), row, lane), e.x, e.y, e.z, e.w);
          } else if (lane < 12) {
            S.sc[row][lane - 8] = valid ? reinterpret_cast<const float*>(src + SML_LATENT_DIM)[lane - 8] : 1.f;
          }
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&S.raw_empty[slot]);
      }
      if (!ok) { *abort = 1; break; }
      ptx::fence_proxy_async();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&S.e_full);
    }
  } else if (warp >= 4 + kStageWarps && warp < 8 + kStageWarps) {
    // ================= V^T warps: one thread per latent dim of every block =================
    const int d = (warp & 3) * 32 + lane;   // = TMEM lane (a warp reaches lanes 32 (warp % 4) ..)
    int chunk = 0;
    for (int tile = 0; tile < ntiles; ++tile) {
      if (tile > 0 && !warp_wait(&S.pv_done, (tile - 1) & 1, abort)) { *abort = 1; break; }
      ptx::tc_fence_after();
      bool ok = true;
      for (int cc = 0; cc < kRing; ++cc, ++chunk) {
        const int slot = chunk % kRing;
        if (!warp_wait(&S.raw_full[slot], (chunk / kRing) & 1, abort)) { ok = false; break; }
        const uint8_t* src = S.raw[slot];
        uint32_t vb[4][8];
#pragma unroll
        for (int jp = 0; jp < kChunk / 2; ++jp) {   // key pairs of the chunk
          const int k0 = cc * kChunk + 2 * jp;
          const bool v0 = S.rowid[tile * kKT + k0] >= 0, v1 = S.rowid[tile * kKT + k0 + 1] >= 0;
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const uint32_t lo8 = v0 ? src[(2 * jp) * SML_LATENT_ROW_BYTES + 128 * b + d] : 0u;
            const uint32_t hi8 = v1 ? src[(2 * jp + 1) * SML_LATENT_ROW_BYTES + 128 * b + d] : 0u;
            vb[b][jp] = e4m3x2_to_h2(lo8 | (hi8 << 8));
          }
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&S.raw_empty[slot]);
#pragma unroll
        for (int b = 0; b < 4; ++b) ptx::tmem_st8(T0 + kColVT + 64 * b + 8 * cc + lane_off, vb[b]);
      }
      if (!ok) { *abort = 1; break; }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&S.vt_full);
    }
  } else if (warp == 11) {
    // ================= gather: one bulk copy per selected row =================
    if (lane == 0) {
      bool ok = ptx::mbar_wait(&S.rows_ready, 0, abort);
      const int nchunks = ntiles * kRing;
      int chunk = 0;
      for (; ok && chunk < nchunks; ++chunk) {
        const int slot = chunk % kRing;
        if (!ptx::mbar_wait(&S.raw_empty[slot], ((chunk / kRing) & 1) ^ 1, abort)) { ok = false; break; }
        uint32_t bytes = 0;
        for (int j = 0; j < kChunk; ++j) bytes += S.rowid[chunk * kChunk + j] >= 0 ? SML_LATENT_ROW_BYTES : 0;
        ptx::mbar_arrive_expect_tx(&S.raw_full[slot], bytes);
        for (int j = 0; j < kChunk; ++j) {
          const int32_t id = S.rowid[chunk * kChunk + j];
          if (id >= 0)
            ptx::bulk_load(S.raw[slot] + j * SML_LATENT_ROW_BYTES, P.latent + (size_t)id * SML_LATENT_ROW_BYTES,
                           SML_LATENT_ROW_BYTES, &S.raw_full[slot]);
        }
      }
      if (!ok) {
        *abort = 1;
        // Let copies already issued land before shared memory goes away.
        for (int c = max(0, chunk - kRing); c < chunk; ++c)
          ptx::mbar_wait(&S.raw_full[c % kRing], (c / kRing) & 1, nullptr, 1u << 16);
      }
    }
    __syncwarp();
  } else if (warp == 10) {
    // ================= MMA issuer =================
    if (lane == 0) {
      bool ok = ptx::mbar_wait(&S.q_ready, 0, abort);
      const uint32_t id_qk = ptx::idesc_m128(kHC, 0);         // E4M3 x E4M3, K-major
      const uint32_t id_pe = ptx::idesc_f16(kHC, 1, 0, 0);    // bf16
      const uint32_t id_pv = ptx::idesc_f16(kHC, 0, 0, 1);    // f16; A (TMEM) K-major, B MN-major
      for (int tile = 0; ok && tile < ntiles; ++tile) {
        if (!ptx::mbar_wait(&S.e_full, tile & 1, abort)) { ok = false; break; }
        ptx::tc_fence_after();
        // S_b^T = C_b . (Qhi_b + Qlo_b)^T: four accumulators, 32 dims per step, interleaved
#pragma unroll
        for (int k = 0; k < 4; ++k) {
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const uint64_t a = ptx::sdesc_sw128(ptx::smem_u32(S.lat[b]) + 32 * k);
            ptx::mma_f8f6f4_ss(T0 + kColS + 16 * b, a, ptx::sdesc_sw128(ptx::smem_u32(S.qhi[b]) + 32 * k), id_qk, k > 0);
            ptx::mma_f8f6f4_ss(T0 + kColS + 16 * b, a, ptx::sdesc_sw128(ptx::smem_u32(S.qlo[b]) + 32 * k), id_qk, 1);
          }
          if (P.rope_dim)
            ptx::mma_f16_ss(T0 + kColSpe, ptx::sdesc_sw128(ptx::smem_u32(S.pe) + 32 * k),
                            ptx::sdesc_sw128(ptx::smem_u32(S.qpe) + 32 * k), id_pe, k > 0);
        }
        ptx::mma_commit(&S.s_full);
        ptx::mma_commit(&S.e_free);
        if (!ptx::mbar_wait(&S.p_full, tile & 1, abort) || !ptx::mbar_wait(&S.vt_full, tile & 1, abort)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        // O_b^T += V_b^T . P'_b^T: A = V_b^T in TMEM (16 keys = 8 columns per step);
        // B = P'_b^T, MN-major core matrices (8-head blocks 128 B apart, 8-key groups 256 B apart).
#pragma unroll
        for (int k = 0; k < kKT / 16; ++k) {
#pragma unroll
          for (int b = 0; b < 4; ++b)
            ptx::mma_f16_ts(T0 + kColO + 16 * b, T0 + kColVT + 64 * b + 8 * k,
                            ptx::sdesc(ptx::smem_u32(S.p[b]) + 512 * k, 256, 128, 0), id_pv, (tile | k) != 0);
        }
        ptx::mma_commit(&S.pv_done);
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
          const float x0 = __uint_as_float(wa << 16) * inv, x1 = __uint_as_float(wa & 0xffff0000u) * inv;
          const float x2 = __uint_as_float(wb << 16) * inv, x3 = __uint_as_float(wb & 0xffff0000u) * inv;
          const uint32_t h01 = f2_to_e4m3x2(x0, x1), h23 = f2_to_e4m3x2(x2, x3);
          const float2 r01 = e4m3x2_to_f2(h01), r23 = e4m3x2_to_f2(h23);
          const uint32_t l01 = f2_to_e4m3x2(x0 - r01.x, x1 - r01.y), l23 = f2_to_e4m3x2(x2 - r23.x, x3 - r23.y);
          hw[k] = (h01 & 0xffffu) | (h23 << 16);
          lw[k] = (l01 & 0xffffu) | (l23 << 16);
        }
        const int chunk = 4 * (part & 1) + c;
        st_shared_v4(sw128(ptx::smem_u32(S.qhi[b]), h, chunk), hw[0], hw[1], hw[2], hw[3]);
        st_shared_v4(sw128(ptx::smem_u32(S.qlo[b]), h, chunk), lw[0], lw[1], lw[2], lw[3]);
      }
      st_shared_v4(sw128(ptx::smem_u32(S.qpe), h, part), pv.x, pv.y, pv.z, pv.w);
      ptx::fence_proxy_async();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&S.q_ready);
    }
    const float zscale = P.sm_scale * (P.ssmax ? P.ssmax_s * logf((float)max(n, 1)) : 1.f);
    float m[kHC];
#pragma unroll
    for (int h = 0; h < kHC; ++h) m[h] = -INFINITY;
    bool ok = warp_wait(&S.q_ready, 0, abort);   // S.qs
    float qs[kHC];
#pragma unroll
    for (int h = 0; h < kHC; ++h) qs[h] = S.qs[h];
    for (int tile = 0; ok && tile < ntiles; ++tile) {
      if (!warp_wait(&S.e_full, tile & 1, abort) || !warp_wait(&S.s_full, tile & 1, abort)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const bool valid = S.rowid[tile * kKT + row] >= 0;
      float sc[4];
#pragma unroll
      for (int b = 0; b < 4; ++b) sc[b] = S.sc[row][b];
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&S.e_free);   // scales read
      // z = zscale * (sum_b scale_b * s_h * S_b + S_pe), fp32
      float z[kHC];
      {
        uint32_t v[16];
        float acc[kHC];
#pragma unroll
        for (int h = 0; h < kHC; ++h) acc[h] = 0.f;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          ptx::tmem_ld16(T0 + kColS + 16 * b + lane_off, v);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < kHC; ++h) acc[h] = fmaf(sc[b], __uint_as_float(v[h]), acc[h]);
        }
        if (P.rope_dim) {
          ptx::tmem_ld16(T0 + kColSpe + lane_off, v);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < kHC; ++h) z[h] = __uint_as_float(v[h]);
        } else {
#pragma unroll
          for (int h = 0; h < kHC; ++h) z[h] = 0.f;
        }
#pragma unroll
        for (int h = 0; h < kHC; ++h) z[h] = valid ? fmaf(acc[h], qs[h], z[h]) * zscale : -INFINITY;
      }
      column_reduce<true>(S, row, z);
      // lazily raised running max; rescale O and the row-sum partials when it moves
      float alpha[kHC];
      bool any = false;
#pragma unroll
      for (int h = 0; h < kHC; ++h) {
        const float tm = S.hstat[h];
        alpha[h] = 1.f;
        if (tm > m[h] + kLazyRescale || (m[h] == -INFINITY && tm != -INFINITY)) {
          alpha[h] = m[h] == -INFINITY ? 0.f : expf(m[h] - tm);
          m[h] = tm;
          any = true;
        }
      }
      if (any && tile > 0) {
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          uint32_t ov[16];
          ptx::tmem_ld16(T0 + kColO + 16 * b + lane_off, ov);    // this thread: latent dim 128 b + row
          ptx::tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < kHC; ++h) ov[h] = __float_as_uint(__uint_as_float(ov[h]) * alpha[h]);
          ptx::tmem_st16(T0 + kColO + 16 * b + lane_off, ov);
          ptx::tmem_ld16(T0 + kColL + 16 * b + lane_off, ov);    // this thread: key row's partials
          ptx::tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < kHC; ++h) ov[h] = __float_as_uint(__uint_as_float(ov[h]) * alpha[h]);
          ptx::tmem_st16(T0 + kColL + 16 * b + lane_off, ov);
        }
        ptx::tmem_wait_st();
      }
      float p[kHC];
#pragma unroll
      for (int h = 0; h < kHC; ++h) p[h] = z[h] == -INFINITY ? 0.f : expf(z[h] - m[h]);
      // P'_b = fp16(p * scale_b); row-sum partial of block b += P'_b / scale_b
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        uint32_t lv[16], pw[8];
        const float inv_sc = sc[b] > 0.f ? 1.f / sc[b] : 0.f;   // an all-zero block has scale 0
        if (tile > 0) {
          ptx::tmem_ld16(T0 + kColL + 16 * b + lane_off, lv);
          ptx::tmem_wait_ld();
        } else {
#pragma unroll
          for (int h = 0; h < kHC; ++h) lv[h] = 0u;
        }
#pragma unroll
        for (int h = 0; h < kHC; h += 2) {
          const __half2 ph = __floats2half2_rn(p[h] * sc[b], p[h + 1] * sc[b]);
          const float2 pr = __half22float2(ph);
          const float w0 = inv_sc > 0.f ? pr.x * inv_sc : p[h];
          const float w1 = inv_sc > 0.f ? pr.y * inv_sc : p[h + 1];
          lv[h] = __float_as_uint(__uint_as_float(lv[h]) + w0);
          lv[h + 1] = __float_as_uint(__uint_as_float(lv[h + 1]) + w1);
          pw[h >> 1] = *reinterpret_cast<const uint32_t*>(&ph);
        }
        ptx::tmem_st16(T0 + kColL + 16 * b + lane_off, lv);
        const uint32_t pb = ptx::smem_u32(S.p[b]) + (row >> 3) * 256 + (row & 7) * 16;
        st_shared_v4(pb, pw[0], pw[1], pw[2], pw[3]);          // heads 0-7
        st_shared_v4(pb + 128, pw[4], pw[5], pw[6], pw[7]);    // heads 8-15
      }
      ptx::tmem_wait_st();
      ptx::fence_proxy_async();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&S.p_full);
    }
    if (ok && !warp_wait(&S.pv_done, (ntiles - 1) & 1, abort)) ok = false;
    if (!ok) *abort = 1;
    ptx::tc_fence_after();
    // Per block: row sums over the 128 key lanes, then the normalised output.
    float lsum0[kHC];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      uint32_t lv[16];
      ptx::tmem_ld16(T0 + kColL + 16 * b + lane_off, lv);
      ptx::tmem_wait_ld();
      float lf[kHC];
#pragma unroll
      for (int h = 0; h < kHC; ++h) lf[h] = __uint_as_float(lv[h]);
      column_reduce<false>(S, row, lf);
      float inv[kHC];
#pragma unroll
      for (int h = 0; h < kHC; ++h) {
        const float ls = S.hstat[h];
        inv[h] = ls > 0.f ? 1.f / ls : 0.f;
        if (b == 0) lsum0[h] = ls;
      }
      uint32_t ov[16];
      ptx::tmem_ld16(T0 + kColO + 16 * b + lane_off, ov);
      ptx::tmem_wait_ld();
      const int dim = 128 * b + row;
#pragma unroll
      for (int h = 0; h < kHC; ++h)
        P.ws.part_out[(slot0 + (size_t)h * P.ws.splits) * SML_LATENT_DIM + dim] = __uint_as_float(ov[h]) * inv[h];
    }
    // lse from block 0's row sums: sum_i fp16(p_i * scale_i0) / scale_i0 ~ sum_i p_i.
    if (row < kHC) {
      float mrow = 0.f, lrow = 0.f;   // m[row], lsum0[row] without dynamic register indexing
#pragma unroll
      for (int h = 0; h < kHC; ++h) {
        mrow = (h == row) ? m[h] : mrow;
        lrow = (h == row) ? lsum0[h] : lrow;
      }
      P.ws.part_lse[slot0 + (size_t)row * P.ws.splits] = lrow > 0.f ? mrow + logf(lrow) : -INFINITY;
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && S.abort) raise_fault(P.status, SML_FAULT_TIMEOUT);
  if (warp == 10) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(S.tmem_base, 512);
  }
}

// out[t,h,:] = sum_s exp(lse_s - lse) O_s,  lse = ln sum_s exp(lse_s).
__global__ void __launch_bounds__(128)
lse_merge_kernel(int H, MlaWs ws, float* __restrict__ out, float* __restrict__ lse) {
  const int h = blockIdx.x, t = blockIdx.y, S = ws.splits;
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

cudaError_t launch_sparse_mla(const sml_problem& p, const uint16_t* q, const uint8_t* latent_base,
                              int64_t latent_pages, const int32_t* idx, const int32_t* idx_len,
                              float* out, float* lse, const MlaWs& ws, int32_t* status,
                              cudaStream_t stream) {
  if (latent_pages > (int64_t)(INT32_MAX / SML_PAGE_TOKENS)) return cudaErrorInvalidValue;
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
  P.latent = latent_base;
  P.latent_pages = latent_pages;
  P.idx = idx;
  P.idx_len = idx_len;
  P.ws = ws;
  P.status = status;
  const size_t smem = sizeof(Smem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(sparse_mla_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(ws.splits, p.num_heads / kHC, p.num_tokens);
  sparse_mla_tc_kernel<<<grid, kThreads, smem, stream>>>(P);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  lse_merge_kernel<<<dim3(p.num_heads, p.num_tokens), 128, 0, stream>>>(p.num_heads, ws, out, lse);
  return cudaGetLastError();
}

}  // namespace sml
