// Exact per-row top-k by radix select in shared memory.
//
// The pages (vLLM blog on Mistral Large 4, section "ROCm 实现细节", paragraph on
// the persistent fused decode) require an exact top-2048; the DCP paragraph of
// section "长上下文" mentions the radix select that vLLM's candidate exchange
// replaced.  This is a single-GPU radix select written for sm_100a:
//
//  * scores become order-preserving 32-bit keys (-0 -> +0, NaN lowest);
//  * three histogram passes over 11 / 11 / 10 key bits find the k-th largest
//    key tau and how many keys equal to tau are taken;
//  * a final pass in position order emits every key > tau and the lowest
//    positions among keys == tau, so the output is in ascending position
//    order and ties go to the lower position by construction;
//  * a row longer than one chunk (32,768 positions) is cut into chunks, each
//    selected by its own CTA into a candidate list; the last CTA of the row to
//    finish (an arrival counter, no waiting) selects again over the
//    concatenated candidates.  The global top-k is a subset of the union of
//    the chunk top-ks, so the result is exact.
#include "sml_internal.cuh"

namespace sml {
namespace {

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t b = __float_as_uint(f);
  if ((b & 0x7fffffffu) > 0x7f800000u) return 0u;  // NaN ranks below -inf
  if (b == 0x80000000u) b = 0u;                     // -0.0 ties with +0.0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

struct SelectShared {
  int hist[2048];
  int warp_tot[32];
  int bcast[2];
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

// Select the k largest of n keys (key_at(i), i in [0, n)); call emit(pos, i)
// for each selected i, pos = its rank in ascending i order.  All threads of the
// block must call it.  Requires blockDim.x == kTopkThreads.
template <typename KeyAt, typename Emit>
__device__ void select_topk(int n, int k, KeyAt key_at, Emit emit, SelectShared& sh) {
  const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31;
  if (n <= k) {
    for (int i = tid; i < n; i += nt) emit(i, i);
    return;
  }
  uint32_t prefix = 0, pmask = 0;
  int remaining = k;
  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = shifts[pass];
    const int nb = 1 << widths[pass];
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
    // Bins in descending order, nb / nt consecutive bins per thread.
    const int bpt = nb / nt;
    int local = 0;
    for (int j = 0; j < bpt; ++j) local += sh.hist[nb - 1 - (tid * bpt + j)];
    int total;
    const int incl = block_scan_incl(local, sh.warp_tot, &total);
    int above = incl - local;  // keys in bins higher than this thread's bins
    for (int j = 0; j < bpt; ++j) {
      const int b = nb - 1 - (tid * bpt + j);
      const int h = sh.hist[b];
      if (above < remaining && remaining <= above + h) {
        sh.bcast[0] = b;
        sh.bcast[1] = above;
      }
      above += h;
    }
    __syncthreads();
    const int b = sh.bcast[0];
    remaining -= sh.bcast[1];
    prefix |= (uint32_t)b << shift;
    pmask |= (uint32_t)(nb - 1) << shift;
    __syncthreads();
  }
  const uint32_t tau = prefix;
  int gt_run = 0, eq_run = 0;
  for (int base = 0; base < n; base += nt) {
    const int i = base + tid;
    const uint32_t key = i < n ? key_at(i) : 0u;
    const int gt = (i < n) && key > tau;
    const int eq = (i < n) && key == tau;
    const int packed = (gt << 16) | eq;
    int total;
    const int incl = block_scan_incl(packed, sh.warp_tot, &total);
    const int excl = incl - packed;
    const int gt_before = gt_run + (excl >> 16);
    const int eq_before = eq_run + (excl & 0xffff);
    if (gt || (eq && eq_before < remaining)) emit(gt_before + min(eq_before, remaining), i);
    gt_run += total >> 16;
    eq_run += total & 0xffff;
    if (gt_run + min(eq_run, remaining) >= k) break;  // uniform across the block
  }
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
  const int r = request_of(cu_q, B, t);
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
                                                    p.max_ctx, p.max_pages, p.cu_q,
                                                    p.ctx_len, scores, idx, idx_len, ws, status);
  return cudaGetLastError();
}

}  // namespace sml
