// Exact per-row top-k over the indexer scores.
//
// The pages (vLLM blog on Mistral Large 4, section "ROCm 实现细节", paragraph on
// the persistent fused decode) require an exact top-2048; the DCP paragraph of
// section "长上下文" mentions the radix select that vLLM's candidate exchange
// replaced.  This is a single-GPU select written for sm_100a:
//
//  * scores become order-preserving 32-bit keys (-0 -> +0, NaN lowest);
//  * a 1,024-key sample places a floor below the k-th largest value; one pass
//    histograms the values at or above it into 2,048 buckets linear in value
//    up to the row's maximum (so the shared-memory atomics touch about k values
//    and spread over the bins) and finds the bucket that holds the k-th
//    largest value; if the sample misjudged, the pass covers every value;
//  * only that bucket's keys (a handful, typically) go through an exact radix
//    select (11 / 11 / 10 key bits) to find the k-th largest key tau and how
//    many keys equal to tau are taken; a row whose threshold bucket is huge
//    (heavy ties) runs the radix select over all its keys instead;
//  * a last pass in position order, one warp per contiguous range, emits every
//    key > tau and the lowest positions among keys == tau: the output is in
//    ascending position order and ties go to the lower position;
//  * rows longer than one chunk (16,384 positions) are cut into chunks, each
//    selected by its own CTA into a candidate list; the last CTA of the row to
//    finish (an arrival counter, no waiting) selects again over the
//    concatenated candidates.  The global top-k is a subset of the union of
//    the chunk top-ks, so the result is exact.
#include "sml_internal.cuh"

namespace sml {
namespace {

constexpr int kBuckets = 2048;
constexpr int kCandCap = 4096;
constexpr int kSmallCand = 256;   // threshold by direct rank counting up to this many candidates
constexpr int kSample = 1024;     // keys sampled to place the histogram floor

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t b = __float_as_uint(f);
  if ((b & 0x7fffffffu) > 0x7f800000u) return 0u;  // NaN ranks below -inf
  if (b == 0x80000000u) b = 0u;                     // -0.0 ties with +0.0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Inverse of order_key (NaN comes back as a NaN).
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

struct SelectShared {
  int hist[kBuckets];
  uint32_t cand[kCandCap];
  int warp_a[32], warp_b[32];
  float red_lo[32], red_hi[32];
  int ncand;
  int bcast[2];
  uint32_t bcast_tau;
  float bcast_f;
};

// Inclusive block-wide scan of one int per thread; *total gets the block sum.
__device__ __forceinline__ int block_scan_incl(int v, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) warp_tot[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int n = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += n;
    }
    warp_tot[lane] = w;
  }
  __syncthreads();
  if (warp > 0) v += warp_tot[warp - 1];
  *total = warp_tot[nw - 1];
  __syncthreads();
  return v;
}

// Over the histogram sh.hist[0, nb): the bin holding the `need`-th largest
// element, and how many elements lie in the bins above it.
__device__ __forceinline__ void find_bin(int nb, int need, SelectShared& sh, int* bin, int* above_out) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int bpt = nb / nt;   // nb is a multiple of nt
  int local = 0;
  for (int j = 0; j < bpt; ++j) local += sh.hist[nb - 1 - (tid * bpt + j)];
  int total;
  const int incl = block_scan_incl(local, sh.warp_a, &total);
  int above = incl - local;
  for (int j = 0; j < bpt; ++j) {
    const int b = nb - 1 - (tid * bpt + j);
    const int h = sh.hist[b];
    if (above < need && need <= above + h) {
      sh.bcast[0] = b;
      sh.bcast[1] = above;
    }
    above += h;
  }
  __syncthreads();
  *bin = sh.bcast[0];
  *above_out = sh.bcast[1];
  __syncthreads();
}

// Radix select over n keys: the k-th largest key tau (1 <= k <= n) and how
// many keys equal to tau belong to the top k (*take).
template <typename KeyAt>
__device__ void radix_threshold(int n, int k, KeyAt key_at, SelectShared& sh, uint32_t* tau, int* take) {
  const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31;
  uint32_t prefix = 0, pmask = 0;
  int remaining = k;
#pragma unroll
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);   // 11 / 11 / 10 key bits
    const int nb = pass == 2 ? 1024 : 2048;
    for (int b = tid; b < nb; b += nt) sh.hist[b] = 0;
    __syncthreads();
    for (int base = 0; base < n; base += nt) {
      const int i = base + tid;
      int bin = -1;
      if (i < n) {
        const uint32_t key = key_at(i);
        if ((key & pmask) == prefix) bin = (int)((key >> shift) & (uint32_t)(nb - 1));
      }
      const unsigned peers = __match_any_sync(0xffffffffu, bin);
      if (bin >= 0 && lane == __ffs(peers) - 1) atomicAdd(&sh.hist[bin], __popc(peers));
    }
    __syncthreads();
    int b, above;
    find_bin(nb, remaining, sh, &b, &above);
    remaining -= above;
    prefix |= (uint32_t)b << shift;
    pmask |= (uint32_t)(nb - 1) << shift;
  }
  *tau = prefix;
  *take = remaining;
}

// Warp 0 only: over sh.hist[0, kBuckets), the bucket holding the `need`-th
// largest element and the count above it, into sh.bcast.
__device__ __forceinline__ void find_bucket_warp(int need, SelectShared& sh) {
  const int lane = threadIdx.x & 31;
  constexpr int kPer = kBuckets / 32;           // lane l owns buckets [top - kPer l, ...) descending
  const int top = kBuckets - 1 - lane * kPer;
  int local = 0;
  for (int j = 0; j < kPer; ++j) local += sh.hist[top - j];
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const int before = incl - local;
  if (before < need && need <= incl) {
    int above = before;
    for (int j = 0; j < kPer; ++j) {
      const int h = sh.hist[top - j];
      if (need <= above + h) {
        sh.bcast[0] = top - j;
        sh.bcast[1] = above;
        break;
      }
      above += h;
    }
  }
}

// Select the k largest of n keys (key_at(i), i in [0, n)); call emit(pos, i)
// for each selected i, pos = its rank in ascending i order.  All threads of the
// block call it; blockDim.x == kTopkThreads.
template <typename KeyAt, typename Emit>
__device__ void select_topk(int n, int k, KeyAt key_at, Emit emit, SelectShared& sh) {
  const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
  if (n <= k) {
    for (int i = tid; i < n; i += nt) emit(i, i);
    return;
  }
  // 1. finite range of the values
  float lo = INFINITY, hi = -INFINITY;
#pragma unroll 4
  for (int i = tid; i < n; i += nt) {
    const float v = key_value(key_at(i));
    if (isfinite(v)) {
      lo = fminf(lo, v);
      hi = fmaxf(hi, v);
    }
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (lane == 0) {
    sh.red_lo[warp] = lo;
    sh.red_hi[warp] = hi;
  }
  for (int b = tid; b < kBuckets; b += nt) sh.hist[b] = 0;
  if (tid == 0) sh.ncand = 0;
  __syncthreads();
  lo = INFINITY;
  hi = -INFINITY;
  for (int w = 0; w < nt / 32; ++w) {
    lo = fminf(lo, sh.red_lo[w]);
    hi = fmaxf(hi, sh.red_hi[w]);
  }
  // 2. A floor below which fewer than k values can lie above: a sample of
  // kSample evenly spaced keys, histogrammed into 256 value bins, gives the bin
  // holding its k * kSample / n-th largest key, plus a 4-sigma margin.  Only
  // values at or above the floor go into the fine histogram, so its atomics
  // touch about k values instead of n.  If the sample misjudged (fewer than k
  // values at or above the floor) every value is histogrammed instead.
  const float width = hi - lo;
  const bool finite_range = hi > lo && width < INFINITY;
  float floor_v = -INFINITY;
  if (finite_range && n > 2 * k) {
    const int stride = n / kSample;
    for (int b = tid; b < 256; b += nt) sh.hist[b] = 0;
    __syncthreads();
    const float cscale = 254.f / width;
    for (int j = tid; j < kSample; j += nt) {
      const float v = key_value(key_at(j * stride));
      const int cb = !(v > -INFINITY) ? 0 : (v == INFINITY ? 255 : 1 + (int)fminf(fmaxf((v - lo) * cscale, 0.f), 253.f));
      atomicAdd(&sh.hist[cb], 1);
    }
    __syncthreads();
    if (warp == 0) {
      const float mu = (float)k * kSample / (float)n;
      const int need_s = min(kSample, (int)ceilf(mu + 4.f * sqrtf(mu) + 4.f));
      // 8 coarse bins per lane, descending
      const int top = 255 - 8 * lane;
      int local = 0;
      for (int j = 0; j < 8; ++j) local += sh.hist[top - j];
      int incl = local;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int above = incl - local;
      if (above < need_s && need_s <= incl) {
        for (int j = 0; j < 8; ++j) {
          above += sh.hist[top - j];
          if (need_s <= above) {
            const int cb = top - j;   // coarse bin 1..254 covers [lo + (cb-1)/cscale, ...)
            sh.bcast_f = cb <= 1 ? -INFINITY : lo + (float)(cb - 1) / cscale;
            break;
          }
        }
      }
      if (lane == 0 && incl < need_s) sh.bcast_f = -INFINITY;   // unreachable: all samples counted
    }
    __syncthreads();
    floor_v = sh.bcast_f;
  }
  // Fine buckets: 0 = NaN / -inf (full mode only), 1 .. kBuckets-2 finite, top = +inf;
  // -1 = below the floor.
  int full = !(floor_v > -INFINITY);
  float base_v = full ? lo : floor_v;
  float scale = finite_range && hi > base_v ? (float)(kBuckets - 3) / (hi - base_v) : 0.f;
  auto bucket = [&](uint32_t key) -> int {
    const float v = key_value(key);
    if (v == INFINITY) return kBuckets - 1;
    if (!full && !(v >= base_v)) return -1;
    if (!(v > -INFINITY)) return 0;                               // NaN or -inf
    const float x = fminf(fmaxf((v - base_v) * scale, 0.f), (float)(kBuckets - 3));   // monotone in v
    return 1 + (int)x;
  };
  for (int attempt = 0; attempt < 2; ++attempt) {
    for (int b = tid; b < kBuckets; b += nt) sh.hist[b] = 0;
    __syncthreads();
    int counted = 0;
#pragma unroll 4
    for (int i = tid; i < n; i += nt) {
      const int b = bucket(key_at(i));
      if (b >= 0) {
        atomicAdd(&sh.hist[b], 1);
        ++counted;
      }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) counted += __shfl_xor_sync(0xffffffffu, counted, o);
    if (lane == 0) sh.warp_a[warp] = counted;
    __syncthreads();
    int total = 0;
    for (int w = 0; w < nt / 32; ++w) total += sh.warp_a[w];
    if (full || total >= k) break;   // uniform across the block
    full = 1;                        // the sample misjudged: histogram every value
    base_v = lo;
    scale = finite_range ? (float)(kBuckets - 3) / width : 0.f;
    __syncthreads();
  }
  if (warp == 0) find_bucket_warp(k, sh);
  __syncthreads();
  const int bk = sh.bcast[0], above = sh.bcast[1];
  // 3. the keys of the threshold bucket
#pragma unroll 4
  for (int i = tid; i < n; i += nt) {
    const uint32_t key = key_at(i);
    if (bucket(key) == bk) {
      const int slot = atomicAdd(&sh.ncand, 1);
      if (slot < kCandCap) sh.cand[slot] = key;
    }
  }
  __syncthreads();
  const int nc = sh.ncand;
  const int need = k - above;   // 1 <= need <= nc
  uint32_t tau;
  int take;
  if (nc <= kSmallCand) {
    // tau = the candidate with fewer than `need` candidates above it and at
    // least `need` at or above it; every thread holding that key agrees.
    if (tid < nc) {
      const uint32_t key = sh.cand[tid];
      int gt = 0, ge = 0;
      for (int j = 0; j < nc; ++j) {
        const uint32_t c = sh.cand[j];
        gt += c > key;
        ge += c >= key;
      }
      if (gt < need && need <= ge) {
        sh.bcast_tau = key;
        sh.bcast[1] = need - gt;
      }
    }
    __syncthreads();
    tau = sh.bcast_tau;
    take = sh.bcast[1];
  } else if (nc <= kCandCap) {
    radix_threshold(nc, need, [&](int i) { return sh.cand[i]; }, sh, &tau, &take);
  } else {
    radix_threshold(n, k, key_at, sh, &tau, &take);   // heavy ties: over every key
  }
  // 4. emission in position order; warp w owns a contiguous range
  const int nw = nt / 32;
  const int seg = ((n + nw - 1) / nw + 31) & ~31;
  const int beg = min(n, warp * seg), end = min(n, beg + seg);
  int cgt = 0, ceq = 0;
  for (int i0 = beg; i0 < end; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t key = i < end ? key_at(i) : 0u;
    cgt += __popc(__ballot_sync(0xffffffffu, i < end && key > tau));
    ceq += __popc(__ballot_sync(0xffffffffu, i < end && key == tau));
  }
  if (lane == 0) {
    sh.warp_a[warp] = cgt;
    sh.warp_b[warp] = ceq;
  }
  __syncthreads();
  if (warp == 0) {
    int a = sh.warp_a[lane], b = sh.warp_b[lane];
    const int a0 = a, b0 = b;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, a, o), y = __shfl_up_sync(0xffffffffu, b, o);
      if (lane >= o) {
        a += x;
        b += y;
      }
    }
    sh.warp_a[lane] = a - a0;   // exclusive prefix over the warps
    sh.warp_b[lane] = b - b0;
  }
  __syncthreads();
  int g = sh.warp_a[warp], e = sh.warp_b[warp];
  const unsigned below = (1u << lane) - 1u;
  for (int i0 = beg; i0 < end; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t key = i < end ? key_at(i) : 0u;
    const bool gt = i < end && key > tau, eq = i < end && key == tau;
    const unsigned bg = __ballot_sync(0xffffffffu, gt), be = __ballot_sync(0xffffffffu, eq);
    const int gb = g + __popc(bg & below), eb = e + __popc(be & below);
    if (gt || (eq && eb < take)) emit(gb + min(eb, take), i);
    g += __popc(bg);
    e += __popc(be);
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kTopkThreads, 1)
topk_kernel(int B, int T, int K, int max_ctx, int max_pages, const int32_t* __restrict__ cu_q,
            const int32_t* __restrict__ ctx_len, const float* __restrict__ scores,
            int32_t* __restrict__ idx, int32_t* __restrict__ idx_len, TopkWs ws,
            int32_t* status) {
  extern __shared__ uint32_t skeys[];  // kTopkChunk keys
  __shared__ SelectShared sh;
  __shared__ int is_last;
  const int tid = threadIdx.x, nt = blockDim.x;
  const int t = blockIdx.y, c = blockIdx.x;
  const int r = request_of_warp(cu_q, B, t);
  const Req rq = load_request(cu_q, ctx_len, r, T, max_ctx, max_pages);
  const int q0 = rq.q0, Q = rq.Q, L = rq.L;
  int32_t* out = idx + (size_t)t * K;
  if (!rq.ok || t < q0 || t - q0 >= Q) {
    if (c == 0) {
      for (int i = tid; i < K; i += nt) out[i] = -1;
      if (tid == 0) {
        idx_len[t] = 0;
        raise_fault(status, SML_FAULT_LENGTHS);
      }
    }
    return;
  }
  const int n = L - Q + (t - q0) + 1;
  const int nch = (n + kTopkChunk - 1) / kTopkChunk;
  if (c >= nch) return;
  const int c0 = c * kTopkChunk;
  const int cn = min(kTopkChunk, n - c0);
  const float* row = scores + (size_t)t * max_ctx + c0;
#pragma unroll 32
  for (int i = tid; i < cn; i += nt) skeys[i] = order_key(__ldcg(row + i));
  __syncthreads();
  auto smem_key = [&](int i) { return skeys[i]; };

  if (nch == 1) {
    select_topk(cn, K, smem_key, [&](int pos, int i) { out[pos] = i; }, sh);
    const int len = min(K, n);
    for (int i = len + tid; i < K; i += nt) out[i] = -1;
    if (tid == 0) idx_len[t] = len;
    return;
  }

  // Level 1: this chunk's top-k, as candidates in position order.
  const size_t row_base = (size_t)t * ws.chunks * K;
  uint32_t* ck = ws.cand_key + row_base + (size_t)c * K;
  int32_t* ci = ws.cand_idx + row_base + (size_t)c * K;
  select_topk(cn, K, smem_key, [&](int pos, int i) { ck[pos] = skeys[i]; ci[pos] = c0 + i; }, sh);
  __threadfence();  // this thread's candidates are visible device-wide ...
  __syncthreads();  // ... before the row's arrival counter moves
  if (tid == 0) {
    const int old = atomicAdd(ws.counters + t, 1);
    is_last = (old == nch - 1);
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();

  // Level 2 (last CTA of the row): every chunk but the last holds exactly K
  // candidates (a chunk has kTopkChunk >= K positions), so the candidates are
  // contiguous and still in position order.
  const int total = (nch - 1) * K + min(K, n - (nch - 1) * kTopkChunk);
  const uint32_t* tk = ws.cand_key + row_base;
  const int32_t* ti = ws.cand_idx + row_base;
  if (total <= kTopkChunk) {
#pragma unroll 16
    for (int i = tid; i < total; i += nt) skeys[i] = __ldcg(tk + i);
    __syncthreads();
    select_topk(total, K, smem_key, [&](int pos, int i) { out[pos] = __ldcg(ti + i); }, sh);
  } else {
    select_topk(total, K, [&](int i) { return __ldcg(tk + i); },
                [&](int pos, int i) { out[pos] = __ldcg(ti + i); }, sh);
  }
  if (tid == 0) {
    idx_len[t] = K;  // n > kTopkChunk >= K
    ws.counters[t] = 0;
  }
}

}  // namespace

cudaError_t launch_topk(const sml_problem& p, const float* scores, int32_t* idx, int32_t* idx_len,
                        const TopkWs& ws, int32_t* status, cudaStream_t stream) {
  const size_t smem = (size_t)kTopkChunk * sizeof(uint32_t);
  cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(ws.chunks, p.num_tokens);
  topk_kernel<<<grid, kTopkThreads, smem, stream>>>(p.num_requests, p.num_tokens, p.topk,
                                                    p.max_ctx, p.max_pages, p.cu_q, p.ctx_len,
                                                    scores, idx, idx_len, ws, status);
  return cudaGetLastError();
}

}  // namespace sml
