// Exact per-row top-k over the indexer scores.
//
// The pages (vLLM blog on Mistral Large 4, section "ROCm 实现细节", paragraph on
// the persistent fused decode) require an exact top-2048; the DCP paragraph of
// section "长上下文" mentions the radix select that vLLM's candidate exchange
// replaced.  This is a single-GPU select written for sm_100a:
//
//  * scores become order-preserving 32-bit keys (-0 -> +0, NaN lowest);
//  * a 1,024-key sample places a floor below the k-th largest value; one pass
//    histograms the values at or above it into 2,048 buckets (512 where one
//    cluster selects a row) linear in value up to the row's maximum (so the
//    shared-memory atomics touch about k values and spread over the bins) and
//    finds the bucket that holds the k-th largest value; if the sample
//    misjudged, the pass covers every value;
//  * only that bucket's keys (a handful, typically) go through an exact radix
//    select (11 / 11 / 10 key bits) to find the k-th largest key tau and how
//    many keys equal to tau are taken; a row whose threshold bucket is huge
//    (heavy ties) runs the radix select over all its keys instead;
//  * a last pass in position order, one warp per contiguous range, emits every
//    key > tau and the lowest positions among keys == tau: the output is in
//    ascending position order and ties go to the lower position;
//  * rows longer than one chunk (16,384 positions) are cut into chunks, each
//    turned by its own CTA into a candidate list; the last CTA of the row to
//    finish (an arrival counter, no waiting) selects again over the
//    concatenated candidates.  A chunk's candidates are its keys at or above a
//    floor placed by a strided sample of the whole row (the same in every CTA
//    of the row), or its own top k when more than k keys pass the floor or the
//    sample gives none; a row whose candidates fall short of k (the sample
//    misjudged) is selected again over all its positions.  Either way every
//    key of the global top k is a candidate, so the result is exact.
#include "ptx.cuh"
#include "sml_internal.cuh"

namespace sml {
namespace {

constexpr int kBuckets = 2048;
constexpr int kCandCap = 4096;
constexpr int kSmallCand = 256;   // threshold by direct rank counting up to this many candidates
constexpr int kSample = 1024;     // keys sampled to place the histogram floor
constexpr int kMaxSegChunks = 4096;   // longest row (in chunks) whose candidates are floor-cut segments
constexpr int kLevel2Keys = 2 * kTopkChunk;   // candidate keys the last CTA of a row holds in shared memory

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
template <typename Sh>
__device__ __forceinline__ void find_bin(int nb, int need, const int* hist, Sh& sh, int* bin, int* above_out) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int bpt = nb / nt;   // nb is a multiple of nt
  int local = 0;
  for (int j = 0; j < bpt; ++j) local += hist[nb - 1 - (tid * bpt + j)];
  int total;
  const int incl = block_scan_incl(local, sh.warp_a, &total);
  int above = incl - local;
  for (int j = 0; j < bpt; ++j) {
    const int b = nb - 1 - (tid * bpt + j);
    const int h = hist[b];
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
template <typename KeyAt, typename Sh>
__device__ void radix_threshold(int n, int k, KeyAt key_at, Sh& sh, uint32_t* tau, int* take) {
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
    find_bin(nb, remaining, sh.hist, sh, &b, &above);
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

// The row's floor from a strided sample of up to kSample keys, the same in
// every CTA of the row so that all agree: the sample's ceil(mu + 4 sqrt(mu) +
// 4)-th largest value (mu = k ns / n), found through a 256-bin coarse
// histogram and then exactly among the samples of its bin, so that about
// k (1 + a margin) keys of the row lie at or above it; -inf when the sample's
// finite range is empty or the row is short.  All threads of the block call
// it; the result is uniform.
__device__ float row_floor(const float* row, int n, int k, SelectShared& sh) {
  const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
  const int ns = min(kSample, n);
  constexpr int kPer = kSample / kTopkThreads;
  float sv[kPer];
  float lo = INFINITY, hi = -INFINITY;
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int j = tid + u * nt;
    sv[u] = NAN;
    if (j < ns) {
      sv[u] = key_value(order_key(__ldcg(row + (int)((long long)j * n / ns))));
      if (isfinite(sv[u])) {
        lo = fminf(lo, sv[u]);
        hi = fmaxf(hi, sv[u]);
      }
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
  for (int b = tid; b < 256; b += nt) sh.hist[b] = 0;
  if (tid == 0) {
    sh.bcast_f = -INFINITY;
    sh.bcast[0] = 0;   // no bin found: no floor
  }
  __syncthreads();
  lo = INFINITY;
  hi = -INFINITY;
  for (int w = 0; w < nt / 32; ++w) {
    lo = fminf(lo, sh.red_lo[w]);
    hi = fmaxf(hi, sh.red_hi[w]);
  }
  const float width = hi - lo;
  if (!(hi > lo && width < INFINITY) || n <= 2 * k) return -INFINITY;
  const float cscale = 254.f / width;
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const float v = sv[u];
    if (tid + u * nt < ns) {
      const int cb = !(v > -INFINITY) ? 0 : (v == INFINITY ? 255 : 1 + (int)fminf(fmaxf((v - lo) * cscale, 0.f), 253.f));
      atomicAdd(&sh.hist[cb], 1);
    }
  }
  __syncthreads();
  if (warp == 0) {
    const float mu = (float)k * ns / (float)n;
    const int need_s = min(ns, (int)ceilf(mu + 4.f * sqrtf(mu) + 4.f));
    const int top = 255 - 8 * lane;   // 8 coarse bins per lane, descending
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
        const int h = sh.hist[top - j];
        if (need_s <= above + h) {
          sh.bcast[0] = top - j;            // the bin
          sh.bcast[1] = need_s - above;     // rank of the floor within it (1 = its largest)
          break;
        }
        above += h;
      }
    }
  }
  if (tid == 0) sh.ncand = 0;
  __syncthreads();
  const int fb = sh.bcast[0], rank = sh.bcast[1];
  if (fb <= 1) return -INFINITY;            // the floor would sit in the -inf / lowest bin
  // the bin's samples into shared memory, then the one with `rank - 1` larger
  // ones (ties: the value itself is the floor whichever copy is taken)
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const float v = sv[u];
    if (tid + u * nt < ns && v > -INFINITY && v < INFINITY &&
        1 + (int)fminf(fmaxf((v - lo) * cscale, 0.f), 253.f) == fb)
      sh.cand[atomicAdd(&sh.ncand, 1)] = __float_as_uint(v);
  }
  __syncthreads();
  const int m = sh.ncand;
  for (int i = tid; i < m; i += nt) {
    const float v = __uint_as_float(sh.cand[i]);
    int gt = 0, ge = 0;
    for (int j = 0; j < m; ++j) {
      const float w = __uint_as_float(sh.cand[j]);
      gt += w > v;
      ge += w >= v;
    }
    if (gt < rank && rank <= ge) sh.bcast_f = v;   // every writer writes the same value
  }
  __syncthreads();
  return sh.bcast_f;
}

__global__ void __launch_bounds__(kTopkThreads, 1)
topk_kernel(int B, int T, int K, int max_ctx, int max_pages, const int32_t* __restrict__ cu_q,
            const int32_t* __restrict__ ctx_len, const int32_t* __restrict__ vis_len, const float* __restrict__ scores,
            int32_t* __restrict__ idx, int32_t* __restrict__ idx_len, TopkWs ws,
            int32_t* status) {
  extern __shared__ uint32_t skeys[];  // kTopkChunk keys
  __shared__ SelectShared sh;
  __shared__ int is_last;
  const int tid = threadIdx.x, nt = blockDim.x;
  const int t = blockIdx.y, c = blockIdx.x;
  if (tid == 0) ptx::griddep_launch_dependents();
  ptx::griddep_wait();   // the scores come from the previous kernel
  const int r = request_of_warp(cu_q, B, t);
  const Req rq = load_request(cu_q, ctx_len, r, T, max_ctx, max_pages, vis_len != nullptr);
  const int q0 = rq.q0, Q = rq.Q;
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
  bool bad_n = false;
  const int n = visible_len(vis_len, rq, t, &bad_n);
  if (bad_n && c == 0 && tid == 0) raise_fault(status, SML_FAULT_LENGTHS);
  if (n == 0) {   // nothing visible: an empty selection
    if (c == 0) {
      for (int i = tid; i < K; i += nt) out[i] = -1;
      if (tid == 0) idx_len[t] = 0;
    }
    return;
  }
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

  // Level 1: this chunk's candidates, in position order.  With a sampled
  // floor, the chunk's keys at or above it when there are at most K of them;
  // otherwise (and in rows too long for segment offsets in shared memory) the
  // chunk's own top K.
  constexpr int kW = kTopkThreads / 32;
  const size_t row_base = (size_t)t * ws.chunks * K;
  uint32_t* ck = ws.cand_key + row_base + (size_t)c * K;
  int32_t* ci = ws.cand_idx + row_base + (size_t)c * K;
  const float* full_row = scores + (size_t)t * max_ctx;
  const bool segmented = nch <= kMaxSegChunks;
  int count = -1;
  if (segmented) {
    const float fl = row_floor(full_row, n, K, sh);
    if (fl > -INFINITY) {
      const uint32_t fkey = order_key(fl);
      const int lane = tid & 31, warp = tid >> 5;
      const int seg = ((cn + kW - 1) / kW + 31) & ~31;
      const int wb = min(cn, warp * seg), we = min(cn, wb + seg);
      int cnt = 0;
      for (int i0 = wb; i0 < we; i0 += 32) {
        const int i = i0 + lane;
        cnt += __popc(__ballot_sync(0xffffffffu, i < we && skeys[i] >= fkey));
      }
      if (lane == 0) sh.warp_a[warp] = cnt;
      __syncthreads();
      int total = 0, before = 0;
      for (int w = 0; w < kW; ++w) {
        total += sh.warp_a[w];
        before += w < warp ? sh.warp_a[w] : 0;
      }
      if (total <= K) {
        const unsigned below = (1u << lane) - 1u;
        int off = before;
        for (int i0 = wb; i0 < we; i0 += 32) {
          const int i = i0 + lane;
          const bool cand = i < we && skeys[i] >= fkey;
          const unsigned m = __ballot_sync(0xffffffffu, cand);
          if (cand) {
            const int p = off + __popc(m & below);
            ck[p] = skeys[i];
            ci[p] = c0 + i;
          }
          off += __popc(m);
        }
        count = total;
      }
      __syncthreads();   // every warp has read warp_a before sh is reused
    }
  }
  if (count < 0) {
    select_topk(cn, K, smem_key, [&](int pos, int i) { ck[pos] = skeys[i]; ci[pos] = c0 + i; }, sh);
    count = min(K, cn);
  }
  if (segmented && tid == 0) ws.cand_cnt[(size_t)t * ws.chunks + c] = count;
  __threadfence();  // this thread's candidates are visible device-wide ...
  __syncthreads();  // ... before the row's arrival counter moves
  if (tid == 0) {
    const int old = atomicAdd(ws.counters + t, 1);
    is_last = (old == nch - 1);
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();

  // Level 2 (last CTA of the row).
  const uint32_t* tk = ws.cand_key + row_base;
  const int32_t* ti = ws.cand_idx + row_base;
  if (!segmented) {
    // every chunk but the last holds exactly K candidates (a chunk has
    // kTopkChunk >= K positions), so they are contiguous and in position order
    const int total = (nch - 1) * K + min(K, n - (nch - 1) * kTopkChunk);
    select_topk(total, K, [&](int i) { return __ldcg(tk + i); },
                [&](int pos, int i) { out[pos] = __ldcg(ti + i); }, sh);
  } else {
    // segment starts (candidates before chunk c) into shared memory, after
    // room for kLevel2Keys candidate keys
    int* soff = reinterpret_cast<int*>(skeys + kLevel2Keys);
    const int32_t* cnt = ws.cand_cnt + (size_t)t * ws.chunks;
    int total = 0;
    for (int base = 0; base < nch; base += nt) {
      const int c2 = base + tid;
      const int v = c2 < nch ? __ldcg(cnt + c2) : 0;
      int tot;
      const int incl = block_scan_incl(v, sh.warp_b, &tot);
      if (c2 < nch) soff[c2] = total + incl - v;
      total += tot;
    }
    if (tid == 0) soff[nch] = total;
    __syncthreads();
    if (total < K) {
      // the sample misjudged (fewer than K keys at or above its floor): every
      // position of the row
      select_topk(n, K, [&](int i) { return order_key(__ldcg(full_row + i)); },
                  [&](int pos, int i) { out[pos] = i; }, sh);
    } else {
      // candidate i lies in the last chunk whose segment starts at or before i
      auto seg_of = [&](int i) {
        int a = 0, b = nch - 1;
        while (a < b) {
          const int mid = (a + b + 1) >> 1;
          if (soff[mid] <= i) a = mid;
          else b = mid - 1;
        }
        return a;
      };
      if (total <= kLevel2Keys) {
        // the keys into shared memory (one warp per chunk); positions are read
        // from global memory for the K selected only
        const int lane = tid & 31, warp = tid >> 5;
        for (int c2 = warp; c2 < nch; c2 += kW) {
          const int o = soff[c2], m2 = soff[c2 + 1] - o;
          for (int j = lane; j < m2; j += 32) skeys[o + j] = __ldcg(tk + (size_t)c2 * K + j);
        }
        __syncthreads();
        select_topk(total, K, smem_key,
                    [&](int pos, int i) {
                      const int g = seg_of(i);
                      out[pos] = __ldcg(ti + (size_t)g * K + (i - soff[g]));
                    },
                    sh);
      } else {
      select_topk(total, K,
                  [&](int i) {
                    const int g = seg_of(i);
                    return __ldcg(tk + (size_t)g * K + (i - soff[g]));
                  },
                  [&](int pos, int i) {
                    const int g = seg_of(i);
                    out[pos] = __ldcg(ti + (size_t)g * K + (i - soff[g]));
                  },
                  sh);
      }
    }
  }
  if (tid == 0) {
    idx_len[t] = K;  // n > kTopkChunk >= K
    ws.counters[t] = 0;
  }
}

// ---- one cluster per row --------------------------------------------------------
//
// Rows of up to kClusterMax chunks: the chunks' CTAs form one thread-block
// cluster and select together, in one level, exchanging histograms, the keys
// of the threshold bucket and the selected counts through distributed shared
// memory at hardware cluster barriers.  Each CTA lands its chunk's raw scores
// in shared memory with one bulk asynchronous copy (a CTA's plain loads top out
// near 20 GB/s), places a floor from a strided sample meanwhile, then makes one
// pass over the chunk that compacts the values at or above the floor, in
// position order, into per-warp candidate lists in place; the histogram (512
// buckets linear in value from the floor) and every later step touch only
// those candidates.

constexpr int kClusterMax = 8;
constexpr int kWarps = kTopkThreads / 32;
constexpr int kSegMax = kTopkChunk / kWarps;   // positions per warp segment
constexpr int kLinBuckets = 512;              // value-linear buckets of the candidate histogram
static_assert(kLinBuckets <= kBuckets && kLinBuckets % kTopkThreads == 0, "one pass of bins per thread");
constexpr int kBulkPiece = 4096;              // positions per bulk copy instruction (16 KB)
constexpr uint32_t kBulkWaitUs = 200000;      // limit on the wait for the chunk's copy
static_assert(kSegMax % 128 == 0, "warp segments are whole 128-position steps");

struct ClusterShared {
  uint64_t full;                   // the chunk's bulk copy has landed
  int hist[kBuckets];              // this CTA's histogram (read by the whole cluster)
  int gh[kBuckets];                // the cluster's histogram
  uint16_t cpos[kWarps][kSegMax];  // candidate positions (chunk-local) per warp, ascending
  int wcnt[kWarps];                // candidates per warp
  uint32_t bkeys[kCandCap];        // this CTA's keys in the threshold bucket (read by the cluster)
  uint32_t gkeys[kCandCap];        // the cluster's keys in the threshold bucket
  int nbk;                         // this CTA's count of them (read by the cluster)
  int above;                       // this CTA's keys in buckets above it (read by the cluster)
  int nbq[kClusterMax], abq[kClusterMax];   // every CTA's nbk and above, copied here
  int sel[2];                      // this CTA's keys > tau and == tau (read by the cluster)
  int samp_hist[256];
  int warp_a[32], warp_b[32];
  float red_lo[32], red_hi[32];
  int bcast[2];
  int bcast_tot;
  uint32_t bcast_tau;
  float bcast_f;
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
// Every thread of every CTA of the cluster; shared-memory writes before it are
// visible to the cluster's reads after it.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Split form of cluster_sync: arrive once this CTA is done reading the others'
// shared memory, wait before leaving (so no CTA's shared memory goes away
// while another may still read it).
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }
// Load a 32-bit word at `p`'s offset in the shared memory of cluster CTA `rank`.
__device__ __forceinline__ uint32_t ld_cluster(const void* p, uint32_t rank) {
  uint32_t a, v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"((uint32_t)__cvta_generic_to_shared(p)), "r"(rank));
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
  return v;
}

// S.gh = the sum over the cluster of every CTA's S.hist[0, nb).  The caller
// passes a cluster barrier before any CTA rebuilds S.hist.
__device__ __forceinline__ void cluster_hist_sum(ClusterShared& S, int nb, int C) {
  cluster_sync();   // covers this CTA's threads too
  // up to kBuckets / blockDim.x bins per thread, every remote load in flight at once
  constexpr int kPer = kBuckets / kTopkThreads;
  uint32_t v[kPer][kClusterMax];
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int b = threadIdx.x + u * kTopkThreads;
#pragma unroll
    for (int r = 0; r < kClusterMax; ++r) v[u][r] = (b < nb && r < C) ? ld_cluster(&S.hist[b], r) : 0u;
  }
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int b = threadIdx.x + u * kTopkThreads;
    int s = 0;
#pragma unroll
    for (int r = 0; r < kClusterMax; ++r) s += (int)v[u][r];
    if (b < nb) S.gh[b] = s;
  }
  __syncthreads();
}

// One warp: over hist[0, NB) (NB a multiple of 32), the bin holding the
// need-th largest element and how many lie in the bins above it, into
// sh.bcast[0] and sh.bcast[1] (left alone when the histogram holds fewer than
// need); returns the histogram's total in every lane.
template <int NB, typename Sh>
__device__ __forceinline__ int bin_scan_warp(int need, const int* hist, Sh& sh) {
  const int lane = threadIdx.x & 31;
  constexpr int kPer = NB / 32;
  const int top = NB - 1 - lane * kPer;   // lane l holds bins top, top - 1, ..., descending
  int h[kPer];
  int local = 0;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    h[j] = hist[top - j];
    local += h[j];
  }
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  int above = incl - local;
  if (above < need && need <= incl) {
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      if (above < need && need <= above + h[j]) {
        sh.bcast[0] = top - j;
        sh.bcast[1] = above;
      }
      above += h[j];
    }
  }
  return __shfl_sync(0xffffffffu, incl, 31);
}

__global__ void __launch_bounds__(kTopkThreads, 1)
topk_cluster_kernel(int B, int T, int K, int max_ctx, int max_pages, const int32_t* __restrict__ cu_q,
                    const int32_t* __restrict__ ctx_len, const int32_t* __restrict__ vis_len,
                    const float* __restrict__ scores,
                    int32_t* __restrict__ idx, int32_t* __restrict__ idx_len, int32_t* status) {
  extern __shared__ __align__(16) uint8_t tk_smem[];
  uint32_t* keys = reinterpret_cast<uint32_t*>(tk_smem);
  ClusterShared& S = *reinterpret_cast<ClusterShared*>(tk_smem + kTopkChunk * sizeof(uint32_t));
  const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
  const int C = (int)cluster_size(), c = (int)cluster_rank();
  const int t = blockIdx.y;
  if (tid == 0) {
    ptx::griddep_launch_dependents();
    ptx::mbar_init(&S.full, 1);
    ptx::fence_mbar_init();
  }
  // The scores come from the previous kernel, and so may the lengths (the
  // candidate merge of context parallelism writes the merged rows' lengths,
  // which its global selection passes as ctx_len): every global read follows
  // the wait.  Everything up to the first cluster barrier depends only on the
  // row, so an early return is taken by the whole cluster or by none of it.
  ptx::griddep_wait();
  const int r = request_of_warp(cu_q, B, t);
  const Req rq = load_request(cu_q, ctx_len, r, T, max_ctx, max_pages, vis_len != nullptr);
  const bool row_ok = rq.ok && t >= rq.q0 && t - rq.q0 < rq.Q;
  bool bad_n = false;
  const int n = row_ok ? visible_len(vis_len, rq, t, &bad_n) : 0;
  int32_t* out = idx + (size_t)t * K;
  if (!row_ok) {
    if (c == 0) {
      for (int i = tid; i < K; i += nt) out[i] = -1;
      if (tid == 0) {
        idx_len[t] = 0;
        raise_fault(status, SML_FAULT_LENGTHS);
      }
    }
    return;
  }
  if (bad_n && c == 0 && tid == 0) raise_fault(status, SML_FAULT_LENGTHS);
  if (n <= K) {
    if (c == 0) {
      for (int i = tid; i < K; i += nt) out[i] = i < n ? i : -1;
      if (tid == 0) idx_len[t] = n;
    }
    return;
  }
  // Balanced chunks, multiples of 32 positions (n <= C * kTopkChunk).
  const int per = ((n + C - 1) / C + 31) & ~31;
  const int c0 = min(n, c * per), cn = min(n, c0 + per) - c0;
  const float* row = scores + (size_t)t * max_ctx;

  // 1. this chunk's raw scores into shared memory (keys[] holds float bits
  //    until the candidate pass turns them into keys): one bulk asynchronous
  //    copy of its 16-B aligned part where the row allows it, plain loads
  //    otherwise; the row's sample straight from global memory (every CTA
  //    takes the same sample, so all agree on it) while the copy flies.
  const bool bulk = (reinterpret_cast<uintptr_t>(row + c0) & 15) == 0;
  const int n_bulk = bulk ? (cn & ~3) : 0;
  if (tid == 0) {
    ptx::mbar_arrive_expect_tx(&S.full, (uint32_t)n_bulk * 4u);
    for (int o = 0; o < n_bulk; o += kBulkPiece)
      ptx::bulk_load(keys + o, row + c0 + o, (uint32_t)min(kBulkPiece, n_bulk - o) * 4u, &S.full);
  }
  for (int i = n_bulk + tid; i < cn; i += nt) keys[i] = __float_as_uint(__ldcg(row + c0 + i));
  const int ns = min(kSample, n);
  float sraw[kSample / kTopkThreads];
#pragma unroll
  for (int u = 0; u < kSample / kTopkThreads; ++u) {
    const int j = tid + u * nt;
    sraw[u] = j < ns ? __ldcg(row + (int)((long long)j * n / ns)) : NAN;
  }
  float sv[kSample / kTopkThreads];
  float lo = INFINITY, hi = -INFINITY;
#pragma unroll
  for (int u = 0; u < kSample / kTopkThreads; ++u) {
    const int j = tid + u * nt;
    sv[u] = NAN;
    if (j < ns) {
      sv[u] = key_value(order_key(sraw[u]));
      if (isfinite(sv[u])) {
        lo = fminf(lo, sv[u]);
        hi = fmaxf(hi, sv[u]);
      }
    }
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (lane == 0) {
    S.red_lo[warp] = lo;
    S.red_hi[warp] = hi;
  }
  for (int b = tid; b < 256; b += nt) S.samp_hist[b] = 0;
  for (int b = tid; b < kLinBuckets; b += nt) S.hist[b] = 0;
  if (tid == 0) S.bcast_f = -INFINITY;
  __syncthreads();
  lo = INFINITY;
  hi = -INFINITY;
  for (int w = 0; w < kWarps; ++w) {
    lo = fminf(lo, S.red_lo[w]);
    hi = fmaxf(hi, S.red_hi[w]);
  }
  // 2. floor: the sample's ceil(mu + 4 sqrt(mu) + 4)-th largest value's coarse
  //    bin (mu = k ns / n), so that about k (1 + a margin) values lie above it.
  const float width = hi - lo;
  const bool finite_range = hi > lo && width < INFINITY;
  float floor_v = -INFINITY;
  if (finite_range && n > 2 * K) {
    const float cscale = 254.f / width;
#pragma unroll
    for (int u = 0; u < kSample / kTopkThreads; ++u) {
      const float v = sv[u];
      if (tid + u * nt < ns) {
        const int cb = !(v > -INFINITY) ? 0 : (v == INFINITY ? 255 : 1 + (int)fminf(fmaxf((v - lo) * cscale, 0.f), 253.f));
        atomicAdd(&S.samp_hist[cb], 1);
      }
    }
    __syncthreads();
    if (warp == 0) {
      const float mu = (float)K * ns / (float)n;
      const int need_s = min(ns, (int)ceilf(mu + 4.f * sqrtf(mu) + 4.f));
      const int top = 255 - 8 * lane;
      int local = 0;
      for (int j = 0; j < 8; ++j) local += S.samp_hist[top - j];
      int incl = local;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int above = incl - local;
      if (above < need_s && need_s <= incl) {
        for (int j = 0; j < 8; ++j) {
          above += S.samp_hist[top - j];
          if (need_s <= above) {
            const int cb = top - j;
            S.bcast_f = cb <= 1 ? -INFINITY : lo + (float)(cb - 1) / cscale;
            break;
          }
        }
      }
    }
    __syncthreads();
    floor_v = S.bcast_f;
  }
  // Fine buckets: 0 = NaN / -inf, 1 .. kLinBuckets-2 linear in value from the
  // floor (or the sample's minimum) to the sample's maximum, clamped at both
  // ends, kLinBuckets-1 = +inf: monotone in the key.
  bool full = !(floor_v > -INFINITY);
  float base_v = full ? lo : floor_v;
  float scale = finite_range && hi > base_v ? (float)(kLinBuckets - 3) / (hi - base_v) : 0.f;
  auto bucket = [&](uint32_t key) -> int {
    const float v = key_value(key);
    if (v == INFINITY) return kLinBuckets - 1;
    if (!(v > -INFINITY)) return 0;
    return 1 + (int)fminf(fmaxf((v - base_v) * scale, 0.f), (float)(kLinBuckets - 3));
  };
  // 3. one pass over the chunk, each warp over its own segment (a multiple of
  //    128 positions, 4 per lane), 4 values per lane at a time: the candidates
  //    (key >= the floor's key; every key when there is no floor) are
  //    compacted in place, keys to the front of the warp's segment of keys[]
  //    (a candidate's slot never lies after its own position, and every lane
  //    has read its values before the ballots let any lane write) and their
  //    chunk positions to cpos, both in position order; then the histogram of
  //    the candidates' buckets.  Afterwards candidate j of a warp is key
  //    keys[wb + j] at chunk position cpos[warp][j].
  if (n_bulk > 0 && !ptx::mbar_wait(&S.full, 0, nullptr, kBulkWaitUs)) {
    // The copy outlived its limit: flag the row and give the copy one more
    // bounded wait, so that no copy is left writing when the CTA goes on.
    if (tid == 0) raise_fault(status, SML_FAULT_TIMEOUT);
    ptx::mbar_wait(&S.full, 0, nullptr, kBulkWaitUs);
  }
  __syncthreads();   // the plain-loaded tail, and every lane past the copy
  const int seg = ((cn + kWarps - 1) / kWarps + 127) & ~127;
  const int wb = min(cn, warp * seg), we = min(cn, wb + seg);
  const unsigned below = (1u << lane) - 1u;
  int total = 0;
  for (int attempt = 0; attempt < 2; ++attempt) {
    // key >= the floor's key is value >= the floor for every non-NaN value
    // (order_key is monotone and ties -0 with +0); NaN passes only when full
    const float fv = base_v;
    int cnt = 0;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (wb + 4 * lane < we) v = *reinterpret_cast<const float4*>(keys + wb + 4 * lane);
    for (int i0 = wb; i0 < we; i0 += 128) {
      const int i = i0 + 4 * lane;
      // the next window's values before this window's writes, which land at
      // or before this window's positions and so never in the next window
      float4 vn = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i + 128 < we) vn = *reinterpret_cast<const float4*>(keys + i + 128);
      const bool cx = i < we && (full || v.x >= fv), cy = i + 1 < we && (full || v.y >= fv);
      const bool cz = i + 2 < we && (full || v.z >= fv), cw = i + 3 < we && (full || v.w >= fv);
      // the lanes' candidate counts (0..4) bit by bit: ranks without a scan
      const int nc = (int)cx + (int)cy + (int)cz + (int)cw;
      const unsigned b0 = __ballot_sync(0xffffffffu, nc & 1), b1 = __ballot_sync(0xffffffffu, nc & 2),
                     b2 = __ballot_sync(0xffffffffu, nc & 4);
      const int px = cnt + __popc(b0 & below) + 2 * __popc(b1 & below) + 4 * __popc(b2 & below);
      const int py = px + (int)cx, pz = py + (int)cy, pw = pz + (int)cz;
      cnt += __popc(b0) + 2 * __popc(b1) + 4 * __popc(b2);
      if (cx) { keys[wb + px] = order_key(v.x); S.cpos[warp][px] = (uint16_t)i; }
      if (cy) { keys[wb + py] = order_key(v.y); S.cpos[warp][py] = (uint16_t)(i + 1); }
      if (cz) { keys[wb + pz] = order_key(v.z); S.cpos[warp][pz] = (uint16_t)(i + 2); }
      if (cw) { keys[wb + pw] = order_key(v.w); S.cpos[warp][pw] = (uint16_t)(i + 3); }
      v = vn;
    }
    __syncwarp();
    for (int j = lane; j < cnt; j += 32) atomicAdd(&S.hist[bucket(keys[wb + j])], 1);
    if (lane == 0) S.wcnt[warp] = cnt;
    cluster_hist_sum(S, kLinBuckets, C);
    // the cluster's total, and (when it reaches K) the threshold bucket
    if (warp == 0) {
      const int tot = bin_scan_warp<kLinBuckets>(K, S.gh, S);
      if (lane == 0) {
        S.bcast_tot = tot;
        S.nbk = 0;
        S.above = 0;
      }
    }
    __syncthreads();
    total = S.bcast_tot;
    if (full || total >= K) break;   // the same in every CTA of the cluster
    full = true;                     // the sample misjudged: every key is a candidate
    base_v = lo;
    scale = finite_range ? (float)(kLinBuckets - 3) / width : 0.f;
    __syncthreads();
    cluster_sync();                  // every CTA has read this histogram before it is rebuilt
    // the compaction overwrote the chunk: its raw scores again, and a clean histogram
    for (int i = tid; i < cn; i += nt) keys[i] = __float_as_uint(__ldcg(row + c0 + i));
    for (int b = tid; b < kLinBuckets; b += nt) S.hist[b] = 0;
    __syncthreads();
  }
  // 4. the threshold bucket (the same in every CTA), and this CTA's count of
  //    keys above it
  const int bk = S.bcast[0], need = K - S.bcast[1];
  const int wn = S.wcnt[warp];
  {
    int part = 0;
    for (int b = bk + 1 + tid; b < kLinBuckets; b += nt) part += S.hist[b];
    part = __reduce_add_sync(0xffffffffu, part);
    if (lane == 0 && part > 0) atomicAdd(&S.above, part);
  }
  // 5. this CTA's keys in the threshold bucket, published with that count
  for (int j = lane; j < wn; j += 32) {
    const uint32_t key = keys[wb + j];
    if (bucket(key) == bk) {
      const int slot = atomicAdd(&S.nbk, 1);
      if (slot < kCandCap) S.bkeys[slot] = key;
    }
  }
  cluster_sync();   // S.nbk, S.above, S.bkeys complete; every CTA is done reading the others' histograms
  // every CTA's bucket-key count and count above, one round of remote loads
  if (warp == 0 && lane < C) {
    S.nbq[lane] = (int)ld_cluster(&S.nbk, lane);
    S.abq[lane] = (int)ld_cluster(&S.above, lane);
  }
  __syncthreads();
  int nbt = 0;
  bool fits = true;
  for (int q = 0; q < C; ++q) {
    nbt += S.nbq[q];
    fits = fits && S.nbq[q] <= kCandCap;
  }
  fits = fits && nbt <= kCandCap;
  // tau = the need-th largest key of the bucket over the cluster, take = how
  // many keys equal to tau are selected; out0 = where this CTA's selection
  // starts in the row's output, my_take = the ties this CTA may take (ties go
  // to the lowest positions, so to the CTAs before this one first).
  uint32_t tau;
  int take, out0 = 0, my_take = 0;
  if (fits) {
    // all the cluster's bucket keys, CTA by CTA: element i of the
    // concatenation is key i - o_q of CTA q (o_q = the counts before q)
    for (int i = tid; i < nbt; i += nt) {
      int q = 0, o = 0;
      while (i >= o + S.nbq[q]) o += S.nbq[q++];
      S.gkeys[i] = ld_cluster(&S.bkeys[i - o], q);
    }
    __syncthreads();
    cluster_arrive();   // done reading the other CTAs' shared memory: no remote access after this
    if (nbt <= kSmallCand) {
      if (tid < nbt) {
        const uint32_t key = S.gkeys[tid];
        int gt = 0, ge = 0;
        for (int j = 0; j < nbt; ++j) {
          const uint32_t x = S.gkeys[j];
          gt += x > key;
          ge += x >= key;
        }
        if (gt < need && need <= ge) {
          S.bcast_tau = key;
          S.bcast[1] = need - gt;
        }
      }
      __syncthreads();
      tau = S.bcast_tau;
      take = S.bcast[1];
    } else {
      radix_threshold(nbt, need, [&](int i) { return S.gkeys[i]; }, S, &tau, &take);
    }
    __syncthreads();
    if (warp == 0) {
      // The CTAs before this one select their keys above the bucket, their
      // bucket keys > tau, and the ties in CTA order until take runs out:
      // min(E, take) ties in all, E = their keys == tau.
      int o = 0, ab = 0;
      for (int q = 0; q < c; ++q) {
        o += S.nbq[q];
        ab += S.abq[q];
      }
      int gt = 0, eq = 0;
      for (int j = lane; j < o; j += 32) {
        const uint32_t x = S.gkeys[j];
        gt += x > tau;
        eq += x == tau;
      }
      gt = __reduce_add_sync(0xffffffffu, gt);
      eq = __reduce_add_sync(0xffffffffu, eq);
      if (lane == 0) {
        S.bcast[0] = ab + gt + min(eq, take);
        S.bcast[1] = max(0, take - eq);
      }
    }
  } else {
    // Heavy ties: a radix select (11 / 11 / 10 key bits) over the threshold
    // bucket's keys where they lie, the histograms summed over the cluster.
    uint32_t prefix = 0, pmask = 0;
    int remaining = need;
    for (int pass = 0; pass < 3; ++pass) {
      const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
      const int nb = pass == 2 ? 1024 : 2048;
      for (int b = tid; b < nb; b += nt) S.hist[b] = 0;
      __syncthreads();
      for (int j = lane; j < wn; j += 32) {
        const uint32_t key = keys[wb + j];
        if (bucket(key) == bk && (key & pmask) == prefix) atomicAdd(&S.hist[(key >> shift) & (uint32_t)(nb - 1)], 1);
      }
      cluster_hist_sum(S, nb, C);
      int b, above;
      find_bin(nb, remaining, S.gh, S, &b, &above);
      remaining -= above;
      prefix |= (uint32_t)b << shift;
      pmask |= (uint32_t)(nb - 1) << shift;
      cluster_sync();   // every CTA has read this histogram before it is rebuilt
    }
    tau = prefix;
    take = remaining;
    // this CTA's counts of keys > tau and == tau, exchanged over the cluster
    int cg = 0, ce = 0;
    for (int j0 = 0; j0 < wn; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t key = j < wn ? keys[wb + j] : 0u;
      cg += __popc(__ballot_sync(0xffffffffu, j < wn && key > tau));
      ce += __popc(__ballot_sync(0xffffffffu, j < wn && key == tau));
    }
    if (lane == 0) {
      S.warp_a[warp] = cg;
      S.warp_b[warp] = ce;
    }
    __syncthreads();
    if (tid == 0) {
      int a = 0, b = 0;
      for (int w = 0; w < kWarps; ++w) {
        a += S.warp_a[w];
        b += S.warp_b[w];
      }
      S.sel[0] = a;
      S.sel[1] = b;
    }
    __syncthreads();
    cluster_sync();
    if (tid == 0) {
      int off = 0, eq_before = 0;
      for (int q = 0; q < c; ++q) {
        const int g = (int)ld_cluster(&S.sel[0], q), e = (int)ld_cluster(&S.sel[1], q);
        off += g + max(0, min(e, take - eq_before));
        eq_before += e;
      }
      S.bcast[0] = off;
      S.bcast[1] = max(0, take - eq_before);
    }
    __syncthreads();
    cluster_arrive();
  }
  __syncthreads();
  out0 = S.bcast[0];
  my_take = S.bcast[1];
  // 6. this CTA's counts per warp (exclusive prefixes over the warps)
  int cgt = 0, ceq = 0;
  for (int j0 = 0; j0 < wn; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t key = j < wn ? keys[wb + j] : 0u;
    cgt += __popc(__ballot_sync(0xffffffffu, j < wn && key > tau));
    ceq += __popc(__ballot_sync(0xffffffffu, j < wn && key == tau));
  }
  __syncthreads();
  if (lane == 0) {
    S.warp_a[warp] = cgt;
    S.warp_b[warp] = ceq;
  }
  __syncthreads();
  if (warp == 0) {
    int a = lane < kWarps ? S.warp_a[lane] : 0, b = lane < kWarps ? S.warp_b[lane] : 0;
    const int a0 = a, b0 = b;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, a, o), y = __shfl_up_sync(0xffffffffu, b, o);
      if (lane >= o) {
        a += x;
        b += y;
      }
    }
    if (lane < kWarps) {
      S.warp_a[lane] = a - a0;
      S.warp_b[lane] = b - b0;
    }
  }
  __syncthreads();
  // 7. emission in position order
  int g = S.warp_a[warp], e = S.warp_b[warp];
  for (int j0 = 0; j0 < wn; j0 += 32) {
    const int j = j0 + lane;
    const int pos = j < wn ? S.cpos[warp][j] : 0;
    const uint32_t key = j < wn ? keys[wb + j] : 0u;
    const bool gt = j < wn && key > tau, eq = j < wn && key == tau;
    const unsigned bg = __ballot_sync(0xffffffffu, gt), be = __ballot_sync(0xffffffffu, eq);
    const int gb = g + __popc(bg & below), eb = e + __popc(be & below);
    if (gt || (eq && eb < my_take)) out[out0 + gb + min(eb, my_take)] = c0 + pos;
    g += __popc(bg);
    e += __popc(be);
  }
  if (c == 0 && tid == 0) idx_len[t] = K;
  cluster_wait();   // shared memory stays until every CTA of the cluster is done reading it
}

}  // namespace

cudaError_t launch_topk(const sml_problem& p, const float* scores, int32_t* idx, int32_t* idx_len,
                        const TopkWs& ws, int32_t* status, cudaStream_t stream) {
  if (ws.chunks <= kClusterMax) {
    // one cluster of ws.chunks CTAs per row
    const size_t smem = (size_t)kTopkChunk * sizeof(uint32_t) + sizeof(ClusterShared);
    cudaError_t e = set_max_smem(reinterpret_cast<const void*>(topk_cluster_kernel), smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(topk_cluster_kernel, dim3(ws.chunks, p.num_tokens), dim3(kTopkThreads), smem, stream, ws.chunks,
                      p.num_requests, p.num_tokens, p.topk, p.max_ctx, p.max_pages, p.cu_q, p.ctx_len, p.vis_len,
                      scores, idx, idx_len, status);
  }
  // chunk keys, or (last CTA of a row) candidate keys, then segment starts
  const size_t smem = (size_t)kLevel2Keys * sizeof(uint32_t) + (kMaxSegChunks + 1) * sizeof(int);
  cudaError_t e = set_max_smem(reinterpret_cast<const void*>(topk_kernel), smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(topk_kernel, dim3(ws.chunks, p.num_tokens), dim3(kTopkThreads), smem, stream, 0, p.num_requests,
                    p.num_tokens, p.topk, p.max_ctx, p.max_pages, p.cu_q, p.ctx_len, p.vis_len, scores, idx, idx_len,
                    ws, status);
}

}  // namespace sml
