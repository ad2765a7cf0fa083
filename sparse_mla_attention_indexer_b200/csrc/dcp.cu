// Decode context parallelism (DCP) over R ranks with token-sharded caches:
// the steps between the ranks' own indexer / top-k and their own sparse MLA.
//
// vLLM blog "vLLM 首日支持 Mistral Large 4", section "长上下文：解码和预填充的上下文
// 并行", paragraph "DCP" and the list after it: the cache is sharded by token;
// each rank's top-k candidates are exchanged as (score, id) pairs and merged
// with a stable top-k; each rank attends over the selected tokens it holds
// (its top-k slots compacted, their count bounding the attention); the
// partial outputs are combined by their log-sum-exp.
//
// Token s of a request lives on rank (s / I) % R at local position
// (s / (I R)) I + s % I, so a rank's tokens keep their order.  The merge
// places every candidate at its rank in global position order across all
// ranks (one binary search per other rank), so that the exact top-k of this
// library, whose ties go to the lower index, resolves ties to the lower global
// position over the merged row.
#include "ptx.cuh"
#include "sml_internal.cuh"

namespace sml {
namespace {

struct RankArrays {
  const float* scores[SML_DCP_MAX_RANKS];
  const int32_t* idx[SML_DCP_MAX_RANKS];
  const int32_t* len[SML_DCP_MAX_RANKS];
  int64_t stride[SML_DCP_MAX_RANKS];
  int packed;   // scores[r] is [T, K], aligned with idx[r]
};

struct RankOut {
  int32_t* idx[SML_DCP_MAX_RANKS];
  int32_t* len[SML_DCP_MAX_RANKS];
};

// The host checks that every rank's score stride times R fits in int32, so a
// valid local position's global position does; the arithmetic runs in int64
// all the same, so that an invalid one cannot wrap into range.
__device__ __forceinline__ long long global_pos(int local, int rank, int R, int I) {
  return ((long long)(local / I) * R + rank) * I + local % I;
}

// Candidates of query t whose global position is below g on rank r (the
// rank's list is ascending in local, hence in global, position).
__device__ __forceinline__ int count_below(const int32_t* list, int n, long long g, int r, int R, int I) {
  int a = 0, b = n;
  while (a < b) {
    const int mid = (a + b) >> 1;
    if (global_pos(__ldg(list + mid), r, R, I) < g) a = mid + 1;
    else b = mid;
  }
  return a;
}

constexpr int kMergeThreads = 256;

__global__ void __launch_bounds__(kMergeThreads)
dcp_merge_kernel(RankArrays ra, int R, int I, int K, float* __restrict__ mscore, int32_t* __restrict__ mpos,
                 int32_t* __restrict__ mlen, int32_t* status) {
  ptx::griddep_wait();
  if (threadIdx.x == 0) ptx::griddep_launch_dependents();
  const int t = blockIdx.x;
  int n[SML_DCP_MAX_RANKS];
  int total = 0;
  for (int r = 0; r < R; ++r) {
    int v = __ldg(ra.len[r] + t);
    if (v < 0 || v > K) {
      if (threadIdx.x == 0) raise_fault(status, SML_FAULT_TOPK_LEN);
      v = max(0, min(v, K));
    }
    n[r] = v;
    total += v;
  }
  const size_t row = (size_t)t * R * K;
  // Every slot of the merged row starts as (NaN, -1): a NaN ranks below every
  // score in the top-k, and the split skips position -1.  Valid ascending
  // lists overwrite every slot; an invalid entry (reported) leaves its slot so.
  for (int m = threadIdx.x; m < total; m += kMergeThreads) {
    mscore[row + m] = __int_as_float(0x7fc00000);
    mpos[row + m] = -1;
  }
  __syncthreads();
  for (int r = 0; r < R; ++r) {
    const int32_t* list = ra.idx[r] + (size_t)t * K;
    for (int i = threadIdx.x; i < n[r]; i += kMergeThreads) {
      const int l = __ldg(list + i);
      const long long g = l >= 0 ? global_pos(l, r, R, I) : -1;
      if (l < 0 || (!ra.packed && l >= ra.stride[r]) || g > INT32_MAX) {
        raise_fault(status, SML_FAULT_INDEX);
        continue;
      }
      int m = i;
      for (int r2 = 0; r2 < R; ++r2)
        if (r2 != r) m += count_below(ra.idx[r2] + (size_t)t * K, n[r2], g, r2, R, I);
      if (m < total) {
        mscore[row + m] = ra.packed ? __ldg(ra.scores[r] + (size_t)t * K + i)
                                    : __ldg(ra.scores[r] + (size_t)t * ra.stride[r] + l);
        mpos[row + m] = (int32_t)g;
      }
    }
  }
  if (threadIdx.x == 0) mlen[t] = total;
}

// One warp per query: the selected merged slots, in ascending global
// position, go to their rank's list in order (ballot compaction per rank).
__global__ void __launch_bounds__(32)
dcp_split_kernel(int R, int I, int K, const int32_t* __restrict__ sel, const int32_t* __restrict__ sel_len,
                 const int32_t* __restrict__ mpos, int mstride, RankOut out, int32_t* status) {
  ptx::griddep_wait();
  if (threadIdx.x == 0) ptx::griddep_launch_dependents();
  const int t = blockIdx.x, lane = threadIdx.x;
  int n = __ldg(sel_len + t);
  if (n < 0 || n > K) {
    if (lane == 0) raise_fault(status, SML_FAULT_TOPK_LEN);
    n = max(0, min(n, K));
  }
  int cnt[SML_DCP_MAX_RANKS];
  for (int r = 0; r < R; ++r) cnt[r] = 0;
  const unsigned below = (1u << lane) - 1u;
  for (int i0 = 0; i0 < n; i0 += 32) {
    const int i = i0 + lane;
    int owner = -1, local = 0;
    if (i < n) {
      const int m = __ldg(sel + (size_t)t * K + i);
      const int g = m >= 0 && m < mstride ? __ldg(mpos + (size_t)t * mstride + m) : -1;
      if (g >= 0) {
        owner = (g / I) % R;
        local = (int)(((long long)g / ((long long)I * R)) * I + g % I);
      } else {
        raise_fault(status, SML_FAULT_INDEX);   // a selection outside the row, or an unfilled merge slot
      }
    }
    for (int r = 0; r < R; ++r) {
      const unsigned mk = __ballot_sync(0xffffffffu, owner == r);
      if (owner == r) out.idx[r][(size_t)t * K + cnt[r] + __popc(mk & below)] = local;
      cnt[r] += __popc(mk);
    }
  }
  for (int r = 0; r < R; ++r) {
    for (int i = cnt[r] + lane; i < K; i += 32) out.idx[r][(size_t)t * K + i] = -1;
    if (lane == 0) out.len[r][t] = cnt[r];
  }
}

// cand[t, i] = scores[t, idx[t, i]] for i < len[t], NaN past it and for a
// position outside the row.
__global__ void __launch_bounds__(256)
dcp_pack_kernel(int K, const float* __restrict__ scores, int64_t stride, const int32_t* __restrict__ idx,
                const int32_t* __restrict__ len, float* __restrict__ cand, int32_t* status) {
  ptx::griddep_wait();
  if (threadIdx.x == 0) ptx::griddep_launch_dependents();
  const int t = blockIdx.x;
  int n = __ldg(len + t);
  if (n < 0 || n > K) {
    if (threadIdx.x == 0) raise_fault(status, SML_FAULT_TOPK_LEN);
    n = max(0, min(n, K));
  }
  for (int i = threadIdx.x; i < K; i += blockDim.x) {
    float v = __int_as_float(0x7fc00000);
    if (i < n) {
      const int l = __ldg(idx + (size_t)t * K + i);
      if (l >= 0 && l < stride) v = __ldg(scores + (size_t)t * stride + l);
      else raise_fault(status, SML_FAULT_INDEX);
    }
    cand[(size_t)t * K + i] = v;
  }
}

struct PartArrays {
  const float* out[SML_DCP_MAX_RANKS];
  const float* lse[SML_DCP_MAX_RANKS];
};

// out[t,h,:] = sum_r exp(lse_r - lse) out_r,  lse = ln sum_r exp(lse_r); a
// part with lse_r = -inf (no selected token on that rank) drops out.
__global__ void __launch_bounds__(128)
lse_combine_kernel(PartArrays pa, int R, int H, float* __restrict__ out, float* __restrict__ lse) {
  ptx::griddep_wait();
  if (threadIdx.x == 0) ptx::griddep_launch_dependents();
  const int t = blockIdx.x, h = blockIdx.y;   // tokens on x: gridDim.y is limited to 65,535
  const size_t th = (size_t)t * H + h;
  float mx = -INFINITY;
  for (int r = 0; r < R; ++r) mx = fmaxf(mx, __ldg(pa.lse[r] + th));
  float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
  float den = 0.f;
  if (mx != -INFINITY) {
    for (int r = 0; r < R; ++r) {
      const float ls = __ldg(pa.lse[r] + th);
      if (ls == -INFINITY) continue;
      const float w = expf(ls - mx);
      den += w;
      const float4 v = __ldg(reinterpret_cast<const float4*>(pa.out[r] + th * SML_LATENT_DIM) + threadIdx.x);
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
  reinterpret_cast<float4*>(out + th * SML_LATENT_DIM)[threadIdx.x] = o;
  if (threadIdx.x == 0) lse[th] = den > 0.f ? mx + logf(den) : -INFINITY;
}

}  // namespace

cudaError_t launch_dcp_merge(const sml_dcp_ranks& rk, int T, int K, float* mscore, int32_t* mpos, int32_t* mlen,
                             int32_t* status, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  RankArrays ra{};
  for (int r = 0; r < rk.num_ranks; ++r) {
    ra.scores[r] = rk.scores[r];
    ra.idx[r] = rk.idx[r];
    ra.len[r] = rk.idx_len[r];
    ra.stride[r] = rk.score_stride[r];
  }
  ra.packed = rk.packed;
  return launch_pdl(dcp_merge_kernel, dim3(T), dim3(kMergeThreads), 0, stream, 0, ra, rk.num_ranks, rk.interleave, K,
                    mscore, mpos, mlen, status);
}

cudaError_t launch_dcp_pack(int T, int K, const float* scores, int64_t stride, const int32_t* idx,
                            const int32_t* len, float* cand, int32_t* status, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  return launch_pdl(dcp_pack_kernel, dim3(T), dim3(256), 0, stream, 0, K, scores, stride, idx, len, cand, status);
}

cudaError_t launch_dcp_split(int R, int I, int T, int K, const int32_t* sel, const int32_t* sel_len,
                             const int32_t* mpos, int32_t* const* local_idx, int32_t* const* local_len,
                             int32_t* status, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  RankOut out{};
  for (int r = 0; r < R; ++r) {
    out.idx[r] = local_idx[r];
    out.len[r] = local_len[r];
  }
  return launch_pdl(dcp_split_kernel, dim3(T), dim3(32), 0, stream, 0, R, I, K, sel, sel_len, mpos, R * K, out,
                    status);
}

cudaError_t launch_lse_combine(int R, int T, int H, const float* const* part_out, const float* const* part_lse,
                               float* out, float* lse, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  PartArrays pa{};
  for (int r = 0; r < R; ++r) {
    pa.out[r] = part_out[r];
    pa.lse[r] = part_lse[r];
  }
  return launch_pdl(lse_combine_kernel, dim3(T, H), dim3(128), 0, stream, 0, pa, R, H, out, lse);
}

}  // namespace sml
