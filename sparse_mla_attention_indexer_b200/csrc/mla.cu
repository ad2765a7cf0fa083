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
//
// One CTA = (query token, group of 16 heads, split of up to 512 selected keys),
// processed in tiles of 128 keys, with the keys as the MMA M dimension and the
// heads as N (16 heads would waste 3/4 of an M >= 64 tile the other way round):
//   * warp 5 gathers the selected 656-B rows with one bulk copy per row into a
//     4-slot ring of 16-row chunks;
//   * warps 6-9 dequantise each row (E4M3 x its block scale -> fp16; the bf16
//     RoPE key is copied as is) into a 128-B-swizzled tile C [128 keys x 576];
//   * warp 4 issues tcgen05.mma kind::f16: S^T[128 x 16] = C . Q^T (nope in
//     fp16, RoPE part in bf16, one fp32 accumulator), then after the softmax
//     O_b^T[128 dims x 16] += C_b^T . P^T for the four 128-dim blocks b -- the
//     same shared tile read K-major for QK^T and MN-major for PV;
//   * warps 0-3 (one thread per key) run the softmax on S^T: column maxima
//     through shared memory, a lazily raised running max (O in TMEM is
//     rescaled only when a head's max grows by more than 8, so P stays below
//     e^8 in fp16), P in fp16, per-thread partial row sums; at the end they read
//     O^T back (one thread per latent dim) and write the split's normalised
//     output and LSE.
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
constexpr int kRing = 4;         // gather ring slots
constexpr int kConvWarps = 4;
constexpr int kThreads = (6 + kConvWarps) * 32;   // warps 0-3 softmax, 4 MMA, 5 gather, 6.. dequantise
constexpr float kLazyRescale = 8.f;   // nats

struct __align__(1024) Smem {
  uint8_t c[8][kKT * 128];       // latent sub-tile d: dims [64d, 64d + 64), fp16 E4M3 values, [128 keys x 128 B], SW128
  uint8_t pe[kKT * 128];         // RoPE key bf16 [128 keys x 64], SW128
  uint8_t q[8][kHC * 128];       // q nope fp16 sub-tiles [16 heads x 64], SW128
  uint8_t qpe[kHC * 128];        // q RoPE bf16 [16 heads x 64], SW128
  uint8_t p[4][kKT * kHC * 2];   // P'_b fp16, MN-major 8x8 core matrices [key/8][head/8][key%8][head%8];
                                 // p[2..3] double as the softmax exchange buffer
  uint8_t raw[kRing][kChunk * SML_LATENT_ROW_BYTES];
  float sc[kKT][4];              // block scales of the tile's keys
  float hstat[kHC];              // per-head tile max / row sum
  int32_t rowid[kMaxSplit];      // pool row (page * 64 + row) of each key, -1 = masked
  uint64_t q_ready, rows_ready, e_full, s_full, p_full, pv_done, drain;
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

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Two E4M3 codes (low byte first) -> two fp16 values (exact).
__device__ __forceinline__ uint32_t e4m3x2_to_h2(uint32_t two) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two & 0xffffu), __NV_E4M3);
  return (uint32_t)h.x | ((uint32_t)h.y << 16);
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const volatile int* abort) {
  const bool ok = ptx::mbar_wait(bar, parity, abort);
  return __all_sync(0xffffffffu, ok);
}

// Softmax exchange: [128 keys][16] floats in the P'_2 / P'_3 buffers, columns
// XOR-swizzled by key to spread banks.
__device__ __forceinline__ float* xbuf(Smem& S, int key, int col) {
  return reinterpret_cast<float*>(S.p[2]) + key * kHC + (col ^ (key & 15));
}

// Sum (or max) over the 128 keys of 16 per-key values, one call per 16 columns;
// every softmax thread gets the 16 results in S.hstat.  Threads: warps 0-3.
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
  const int Dq = SML_LATENT_DIM + P.rope_dim;

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
  const int nchunks = ntiles * (kKT / kChunk);

  if (threadIdx.x == 0) {
    ptx::mbar_init(&S.q_ready, 4);
    ptx::mbar_init(&S.rows_ready, kConvWarps);
    ptx::mbar_init(&S.e_full, kConvWarps);
    ptx::mbar_init(&S.s_full, 1);
    ptx::mbar_init(&S.p_full, 4);
    ptx::mbar_init(&S.pv_done, 1);
    ptx::mbar_init(&S.drain, 1);
    for (int i = 0; i < kRing; ++i) {
      ptx::mbar_init(&S.raw_full[i], 1);
      ptx::mbar_init(&S.raw_empty[i], kConvWarps);
    }
    S.abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 4) {
    ptx::tmem_alloc(&S.tmem_base, 256);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  volatile int* abort = &S.abort;
  // TMEM columns: S_b^T (b = 0..3, lanes = keys) at 16 b; S_pe^T at 64;
  // O_b^T (lanes = dims of block b) at 128 + 16 b; per-key row-sum partials
  // of block b (lanes = keys) at 192 + 16 b.
  const uint32_t tS = S.tmem_base, tO = S.tmem_base + 128, tL = S.tmem_base + 192;

  if (warp >= 6) {
    // ================= dequantise (kConvWarps warps) =================
    constexpr int kCT = kConvWarps * 32;
    constexpr int kRowsPerWarp = kChunk / kConvWarps;
    const int cw = warp - 6, ct = threadIdx.x - 6 * 32;
    // Pool rows of the split's keys: all position loads first, then all
    // block-table loads, so each thread waits for two latencies, not eight.
    constexpr int kPer = kMaxSplit / kCT;
    int pos[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int k = ct + j * kCT;
      pos[j] = k < nkeys ? __ldg(P.idx + (size_t)t * P.K + kb + k) : -1;
    }
    int ph[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int k = ct + j * kCT;
      const bool in = k < nkeys && pos[j] >= 0 && pos[j] < n;
      if (k < nkeys && !in) raise_fault(P.status, SML_FAULT_INDEX);
      ph[j] = in ? __ldg(P.block_table + (size_t)r * P.max_pages + pos[j] / SML_PAGE_TOKENS) : -1;
      if (!in) pos[j] = -1;
    }
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int k = ct + j * kCT;
      int32_t id = -1;
      if (pos[j] >= 0) {
        if (ph[j] >= 0 && ph[j] < P.latent_pages)
          id = ph[j] * SML_PAGE_TOKENS + pos[j] % SML_PAGE_TOKENS;
        else
          raise_fault(P.status, SML_FAULT_PAGE);
      }
      S.rowid[k] = id;
    }
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(&S.rows_ready);

    int chunk = 0;
    for (int tile = 0; tile < ntiles; ++tile) {
      if (tile > 0 && !warp_wait(&S.pv_done, (tile - 1) & 1, abort)) { *abort = 1; break; }
      bool ok = true;
      for (int cc = 0; cc < kKT / kChunk; ++cc, ++chunk) {
        const int slot = chunk % kRing;
        if (!warp_wait(&S.raw_full[slot], (chunk / kRing) & 1, abort)) { ok = false; break; }
        for (int rr = 0; rr < kRowsPerWarp; ++rr) {
          const int j = cw * kRowsPerWarp + rr;      // row within the chunk
          const int row = cc * kChunk + j;           // row within the tile
          const bool valid = S.rowid[tile * kKT + row] >= 0;
          const uint8_t* src = S.raw[slot] + j * SML_LATENT_ROW_BYTES;
          // latent: lane l holds dims [16 l, 16 l + 16) as exact fp16 E4M3 values
          uint32_t o[8];
          if (valid) {
            const uint4 v = *reinterpret_cast<const uint4*>(src + 16 * lane);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              o[2 * i] = e4m3x2_to_h2(w[i] & 0xffffu);
              o[2 * i + 1] = e4m3x2_to_h2(w[i] >> 16);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) o[i] = 0u;
          }
          const int d = lane >> 2, ch = (lane & 3) * 2;
          const uint32_t tb = ptx::smem_u32(S.c[d]);
          st_shared_v4(sw128(tb, row, ch), o[0], o[1], o[2], o[3]);
          st_shared_v4(sw128(tb, row, ch + 1), o[4], o[5], o[6], o[7]);
          if (lane < 8) {
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (valid && P.rope_dim) v = *reinterpret_cast<const uint4*>(src + SML_LATENT_DIM + 16 + 16 * lane);
            st_shared_v4(sw128(ptx::smem_u32(S.pe), row, lane), v.x, v.y, v.z, v.w);
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
  } else if (warp == 5) {
    // ================= gather: one bulk copy per selected row =================
    if (lane == 0) {
      bool ok = ptx::mbar_wait(&S.rows_ready, 0, abort);
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
  } else if (warp == 4) {
    // ================= MMA issuer =================
    if (lane == 0) {
      bool ok = ptx::mbar_wait(&S.q_ready, 0, abort);
      const uint32_t id_qk = ptx::idesc_f16(kHC, 0, 0, 0);   // f16, K-major A and B
      const uint32_t id_pe = ptx::idesc_f16(kHC, 1, 0, 0);   // bf16
      const uint32_t id_pv = ptx::idesc_f16(kHC, 0, 1, 1);   // f16, MN-major A (C_b^T) and B (P'_b^T)
      for (int tile = 0; ok && tile < ntiles; ++tile) {
        if (!ptx::mbar_wait(&S.e_full, tile & 1, abort)) { ok = false; break; }
        ptx::tc_fence_after();
        // S_b^T = C_b . Q_b^T, one accumulator per 128-dim scale block b
        // (2 sub-tiles x 4 steps of 16 dims each) ...
        for (int d = 0; d < 8; ++d) {
          const uint32_t a = ptx::smem_u32(S.c[d]), b = ptx::smem_u32(S.q[d]);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            ptx::mma_f16_ss(tS + 16 * (d >> 1), ptx::sdesc(a + 32 * k, 16, 1024, 2),
                            ptx::sdesc(b + 32 * k, 16, 1024, 2), id_qk, ((d & 1) | k) != 0);
        }
        // ... and the RoPE part (bf16) in its own accumulator.
        if (P.rope_dim) {
          const uint32_t a = ptx::smem_u32(S.pe), b = ptx::smem_u32(S.qpe);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            ptx::mma_f16_ss(tS + 64, ptx::sdesc(a + 32 * k, 16, 1024, 2), ptx::sdesc(b + 32 * k, 16, 1024, 2), id_pe,
                            k != 0);
        }
        ptx::mma_commit(&S.s_full);
        if (!ptx::mbar_wait(&S.p_full, tile & 1, abort)) { ok = false; break; }
        ptx::tc_fence_after();
        // O_b^T += C_b^T . P'_b^T: A = dims [128 b, 128 b + 128) of the tile read MN-major
        // (64-dim blocks 16 KB apart, 8-key groups 1 KB apart); B = P'_b^T, MN-major core
        // matrices (8-head blocks 128 B apart, 8-key groups 256 B apart).
        for (int b = 0; b < 4; ++b) {
          const uint32_t a = ptx::smem_u32(S.c[2 * b]), pb = ptx::smem_u32(S.p[b]);
#pragma unroll
          for (int k = 0; k < kKT / 16; ++k)
            ptx::mma_f16_ss(tO + 16 * b, ptx::sdesc(a + 2048 * k, 16384, 1024, 2),
                            ptx::sdesc(pb + 512 * k, 256, 128, 0), id_pv, (tile | k) != 0);
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
      // Query heads of this group, while the other warps resolve the key rows:
      // nope bf16 -> fp16 (exact in fp16's normal range), RoPE part copied as bf16.
      const uint16_t* qbase = P.q + ((size_t)t * P.H + hg * kHC) * Dq;
      for (int e = row; e < kHC * (Dq / 8); e += 128) {
        const int h = e / (Dq / 8), c8 = e % (Dq / 8);    // 8 elements = one 16-B chunk
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(qbase + (size_t)h * Dq) + c8);
        if (c8 < 64) {
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
          uint32_t o[4];
#pragma unroll
          for (int i = 0; i < 4; ++i)
            o[i] = pack_half2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u));
          st_shared_v4(sw128(ptx::smem_u32(S.q[c8 >> 3]), h, c8 & 7), o[0], o[1], o[2], o[3]);
        } else {
          st_shared_v4(sw128(ptx::smem_u32(S.qpe), h, c8 - 64), v.x, v.y, v.z, v.w);
        }
      }
      ptx::fence_proxy_async();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&S.q_ready);
    }
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const float zscale = P.sm_scale * (P.ssmax ? P.ssmax_s * logf((float)max(n, 1)) : 1.f);
    float m[kHC];
#pragma unroll
    for (int h = 0; h < kHC; ++h) m[h] = -INFINITY;
    bool ok = true;
    for (int tile = 0; tile < ntiles; ++tile) {
      if (!warp_wait(&S.s_full, tile & 1, abort)) { ok = false; break; }
      ptx::tc_fence_after();
      const bool valid = S.rowid[tile * kKT + row] >= 0;
      float sc[4];
#pragma unroll
      for (int b = 0; b < 4; ++b) sc[b] = S.sc[row][b];
      // z = zscale * (sum_b scale_b * S_b + S_pe), fp32
      float z[kHC];
      {
        uint32_t v[16];
        if (P.rope_dim) {
          ptx::tmem_ld16(tS + 64 + lane_off, v);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < kHC; ++h) z[h] = __uint_as_float(v[h]);
        } else {
#pragma unroll
          for (int h = 0; h < kHC; ++h) z[h] = 0.f;
        }
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          ptx::tmem_ld16(tS + 16 * b + lane_off, v);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < kHC; ++h) z[h] = fmaf(sc[b], __uint_as_float(v[h]), z[h]);
        }
      }
#pragma unroll
      for (int h = 0; h < kHC; ++h) z[h] = valid ? z[h] * zscale : -INFINITY;
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
          ptx::tmem_ld16(tO + 16 * b + lane_off, ov);    // this thread: latent dim 128 b + row
          ptx::tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < kHC; ++h) ov[h] = __float_as_uint(__uint_as_float(ov[h]) * alpha[h]);
          ptx::tmem_st16(tO + 16 * b + lane_off, ov);
          ptx::tmem_ld16(tL + 16 * b + lane_off, ov);    // this thread: key row's partials
          ptx::tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < kHC; ++h) ov[h] = __float_as_uint(__uint_as_float(ov[h]) * alpha[h]);
          ptx::tmem_st16(tL + 16 * b + lane_off, ov);
        }
        ptx::tmem_wait_st();
      }
      float p[kHC];
#pragma unroll
      for (int h = 0; h < kHC; ++h) p[h] = z[h] == -INFINITY ? 0.f : expf(z[h] - m[h]);
      // P'_b = fp16(p * scale_b); row-sum partial of block b += P'_b / scale_b, so a
      // block's normalisation uses exactly the weights its MMA used.
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        uint32_t lv[16], pw[8];
        const float inv_sc = sc[b] > 0.f ? 1.f / sc[b] : 0.f;   // an all-zero block has scale 0
        if (tile > 0) {
          ptx::tmem_ld16(tL + 16 * b + lane_off, lv);
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
        ptx::tmem_st16(tL + 16 * b + lane_off, lv);
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
      ptx::tmem_ld16(tL + 16 * b + lane_off, lv);
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
      ptx::tmem_ld16(tO + 16 * b + lane_off, ov);
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
  if (warp == 4) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(S.tmem_base, 256);
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
  // gather of a tile overlaps the math of the one before.
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
