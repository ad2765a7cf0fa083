// Internal declarations shared by the libsml.so translation units.
#pragma once
#include <utility>

#include <cuda_runtime.h>
#include <stdint.h>

#include <string>

#include "sml.h"

namespace sml {

// ---- workspace -----------------------------------------------------------------
// Every stage's workspace starts with a 256-B header whose first word is the
// sticky device status (SML_FAULT_* bits), then the per-row arrival counters of
// the two-level top-k.  Regions are 256-B aligned.
struct WsHeader {
  int32_t status;
  int32_t pad[63];
};

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Top-k: one CTA selects over a chunk of up to kTopkChunk positions held in
// shared memory; longer rows are cut into chunks whose candidates the last
// arriving CTA of the row merges.
constexpr int kTopkChunk = 16384;
constexpr int kTopkThreads = 512;

struct TopkWs {
  int32_t* counters;   // [T] arrival counters, zero between calls
  uint32_t* cand_key;  // [T, chunks, K]
  int32_t* cand_idx;   // [T, chunks, K]
  int32_t* cand_cnt;   // [T, chunks] candidates per chunk
  int chunks;          // ceil(max_ctx / kTopkChunk)
};

// Sparse MLA work split.  A unit is (query token, group of 16 heads, tile of
// 128 selected keys); units are numbered token-major, then head group, then
// tile, and a persistent grid of `ctas` CTAs takes equal contiguous ranges of
// them.  A CTA writes one partial result (per head: output and LSE) for every
// (token, head group) its range touches; a (token, head group) has at most
// `smax` such CTAs, and its partials sit in slots [tg * smax, tg * smax + n)
// in CTA order, n = the CTAs that touch it.
// Sparse-MLA work plan.  Head group g is served by the CTAs with blockIdx.x
// % hg == g; those cpg CTAs split its T * tpt (token, tile) units into equal
// contiguous ranges (token-major), so the hg CTAs with the same blockIdx.x /
// hg walk the same tokens' tiles together and read each row while it is in L2.
struct MlaPlan {
  int hg;              // head groups, H / 16
  int tpt;             // tiles per (token, head group), ceil(topk / 128)
  long long units;     // units of one head group: T * tpt
  int cpg;             // CTAs per head group
  int ctas;            // hg * cpg
  int smax;            // slots per (token, head group)
};

struct MlaWs {
  float* part_out;     // [T * hg * smax * 16, 512]
  float* part_lse;     // [T * hg * smax * 16]
  MlaPlan plan;
};

// Message returned by sml_last_error() on this host thread.
void set_last_error(const std::string& msg);

// Region sizes, in bytes (host).
size_t topk_region_bytes(const sml_problem& p);
size_t mla_region_bytes(const sml_problem& p);
// The plan of a problem on the current device (its SM count sets `ctas`).
MlaPlan mla_plan(const sml_problem& p);
// Partial slots of a plan (16 heads each): T * hg * smax.
inline size_t mla_slots(const MlaPlan& m, int T) { return (size_t)T * m.hg * m.smax; }

// ---- device helpers ---------------------------------------------------------------
__device__ __forceinline__ void raise_fault(int32_t* status, int bits) {
  if (status) atomicOr(status, bits);
}

// Request owning query token t (cu_q non-decreasing, cu_q[0] = 0).
__device__ __forceinline__ int request_of(const int32_t* __restrict__ cu_q, int B, int t) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (__ldg(cu_q + mid) <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// The same lookup by one full warp: a 32-way search, one round of parallel
// loads for B <= 32 (log32(B) rounds in general) instead of log2(B) dependent
// loads.  Every lane returns the same request.
__device__ __forceinline__ int request_of_warp(const int32_t* __restrict__ cu_q, int B, int t) {
  const int lane = threadIdx.x & 31;
  int lo = 0, hi = B;   // answer in [lo, hi)
  while (hi - lo > 1) {
    const int step = (hi - lo + 31) / 32;
    const int j = lo + lane * step;
    const bool le = j < hi && __ldg(cu_q + j) <= t;
    const unsigned mask = __ballot_sync(0xffffffffu, le);
    const int last = mask ? 31 - __clz(mask) : 0;
    lo = lo + last * step;
    hi = min(hi, lo + step);
  }
  return lo;
}

// Query range, context length and visible length of request r, checked against
// the problem: 0 <= q0, Q >= 1, q0 + Q <= T, Q <= L <= max_ctx (0 <= L when
// the visible lengths are given per token) and ceil(L / 64) <= max_pages.
// Anything else is SML_FAULT_LENGTHS and the request is skipped, so no index
// derived from it leaves its buffer.
struct Req {
  int q0, Q, L;
  bool ok;
};

__device__ __forceinline__ Req load_request(const int32_t* __restrict__ cu_q,
                                            const int32_t* __restrict__ ctx_len, int r, int T,
                                            int max_ctx, int max_pages, bool given_vis = false) {
  Req q;
  q.q0 = __ldg(cu_q + r);
  q.Q = __ldg(cu_q + r + 1) - q.q0;
  q.L = __ldg(ctx_len + r);
  q.ok = q.q0 >= 0 && q.Q >= 1 && q.q0 <= T - q.Q && q.L >= (given_vis ? 0 : q.Q) && q.L <= max_ctx &&
         (q.L + SML_PAGE_TOKENS - 1) / SML_PAGE_TOKENS <= max_pages;
  return q;
}

// n_t of query token t of request rq (rq.ok, t in its range): vis[t] when the
// problem gives the visible lengths (clamped into [0, L]; a value outside it
// is reported through *bad), else the causal rule L - Q + j + 1.
__device__ __forceinline__ int visible_len(const int32_t* __restrict__ vis, const Req& rq, int t, bool* bad) {
  if (!vis) return rq.L - rq.Q + (t - rq.q0) + 1;
  const int n = __ldg(vis + t);
  if (n < 0 || n > rq.L) {
    *bad = true;
    return n < 0 ? 0 : rq.L;
  }
  return n;
}

// The n of token t's SSMax factors: ssmax_len[t] (at least 1) when given, else n_t.
__device__ __forceinline__ int ssmax_len_of(const int32_t* __restrict__ ssl, int t, int n) {
  const int m = ssl ? __ldg(ssl + t) : n;
  return m < 1 ? 1 : m;
}

// Host-side per-device caches for the launchers (thread-safe): the SM count,
// and the dynamic shared-memory attribute, set once per kernel and device.
int device_sm_count();
cudaError_t set_max_smem(const void* func, size_t bytes);

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous kernel of the stream finishes, and reads nothing that
// kernel may write before griddep_wait().  cluster_x > 0 also sets a cluster
// of cluster_x CTAs along x.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, int cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute at[2];
  int na = 0;
  at[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (cluster_x > 0) {
    at[na].id = cudaLaunchAttributeClusterDimension;
    at[na].val.clusterDim.x = (unsigned)cluster_x;
    at[na].val.clusterDim.y = 1;
    at[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = at;
  cfg.numAttrs = na;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  return e != cudaSuccess ? e : cudaGetLastError();
}

// ---- launchers (one per kernel family; all enqueue on `stream`) --------------------
cudaError_t launch_indexer(const sml_problem& p, const uint8_t* iq8, const float* iq_scale,
                           const float* iw, const uint8_t* index_base, int64_t index_pages,
                           float* scores, int32_t* status, cudaStream_t stream);
cudaError_t launch_topk(const sml_problem& p, const float* scores, int32_t* idx, int32_t* idx_len,
                        const TopkWs& ws, int32_t* status, cudaStream_t stream);
cudaError_t launch_sparse_mla(const sml_problem& p, const uint16_t* q, const sml_cache& latent,
                              const int32_t* idx, const int32_t* idx_len,
                              float* out, float* lse, const MlaWs& ws, int32_t* status,
                              cudaStream_t stream);
cudaError_t launch_indexer_k_write(const void* k, const int32_t* slot, int n, void* cache, int64_t num_pages,
                                   int32_t* status, cudaStream_t stream);
cudaError_t launch_latent_write(const void* c, const void* kpe, const int32_t* slot, int n, const sml_cache& cache,
                                int32_t* status, cudaStream_t stream);
cudaError_t launch_dcp_merge(const sml_dcp_ranks& rk, int T, int K, float* mscore, int32_t* mpos, int32_t* mlen,
                             int32_t* status, cudaStream_t stream);
cudaError_t launch_dcp_pack(int T, int K, const float* scores, int64_t stride, const int32_t* idx,
                            const int32_t* len, float* cand, int32_t* status, cudaStream_t stream);
cudaError_t launch_dcp_split(int R, int I, int T, int K, const int32_t* sel, const int32_t* sel_len,
                             const int32_t* mpos, int32_t* const* local_idx, int32_t* const* local_len,
                             int32_t* status, cudaStream_t stream);
cudaError_t launch_lse_combine(int R, int T, int H, const float* const* part_out, const float* const* part_lse,
                               float* out, float* lse, cudaStream_t stream);
cudaError_t launch_indexer_q_quant(const void* iq, int T, void* iq8, float* iq_scale, cudaStream_t stream);

}  // namespace sml
