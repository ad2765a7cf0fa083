// C ABI of libsml.so: argument validation, workspace layout and launches.
//
// Validation is default-deny and reports every failed check at once, the
// start-up rule of the fused decode path in the vLLM blog "vLLM 首日支持
// Mistral Large 4", section "ROCm 实现细节" ("the path is default-deny ... fails
// with an error listing all reasons").  Checks that need device data run in the
// kernels and set the sticky status word instead of trapping.
#include <math.h>
#include <stdio.h>

#include <map>
#include <mutex>
#include <string>

#include "sml_internal.cuh"

namespace sml {

static thread_local std::string g_last_error;

void set_last_error(const std::string& msg) { g_last_error = msg; }

namespace {

struct Checker {
  std::string msg;
  int code = SML_OK;
  void fail(int c, const char* what) {
    if (!msg.empty()) msg += "; ";
    msg += what;
    // UNSUPPORTED only if nothing is plainly invalid.
    if (code == SML_OK || (code == SML_ERR_UNSUPPORTED && c != SML_ERR_UNSUPPORTED)) code = c;
  }
  void check(bool ok, int c, const char* what) {
    if (!ok) fail(c, what);
  }
  int done(const char* fn) {
    if (code != SML_OK) {
      g_last_error = std::string(fn) + ": " + msg;
    } else {
      g_last_error.clear();
    }
    return code;
  }
};

bool aligned(const void* ptr, size_t a) { return ((uintptr_t)ptr % a) == 0; }

void check_problem(Checker& c, const sml_problem* p) {
  if (!p) {
    c.fail(SML_ERR_INVALID_ARG, "problem is NULL");
    return;
  }
  c.check(p->num_requests >= 1, SML_ERR_INVALID_ARG, "num_requests < 1");
  c.check(p->num_requests <= 65535, SML_ERR_UNSUPPORTED, "num_requests > 65535");
  c.check(p->num_tokens >= p->num_requests, SML_ERR_INVALID_ARG,
          "num_tokens < num_requests (every request needs a query token)");
  c.check(p->num_tokens <= 65535, SML_ERR_UNSUPPORTED, "num_tokens > 65535");
  c.check(p->num_heads == 16 || p->num_heads == 32 || p->num_heads == 64 || p->num_heads == 128,
          SML_ERR_UNSUPPORTED, "num_heads not in {16, 32, 64, 128}");
  c.check(p->topk >= 1 && p->topk <= SML_MAX_TOPK, SML_ERR_UNSUPPORTED, "topk not in [1, 2048]");
  c.check(p->rope_dim == 0 || p->rope_dim == SML_ROPE_DIM, SML_ERR_UNSUPPORTED,
          "rope_dim not in {0, 64}");
  c.check(p->max_pages >= 1, SML_ERR_INVALID_ARG, "max_pages < 1");
  c.check(p->max_ctx >= 1, SML_ERR_INVALID_ARG, "max_ctx < 1");
  c.check(p->max_ctx <= (1 << 30), SML_ERR_UNSUPPORTED, "max_ctx > 2^30");
  c.check(p->ssmax == 0 || p->ssmax == 1, SML_ERR_INVALID_ARG, "ssmax not 0 or 1");
  c.check(isfinite(p->sm_scale) && p->sm_scale > 0.f, SML_ERR_INVALID_ARG,
          "sm_scale not finite and positive");
  c.check(isfinite(p->ssmax_s) && isfinite(p->ssmax_s_index), SML_ERR_INVALID_ARG,
          "ssmax_s / ssmax_s_index not finite");
  c.check(p->cu_q != nullptr, SML_ERR_INVALID_ARG, "cu_q is NULL");
  c.check(p->ctx_len != nullptr, SML_ERR_INVALID_ARG, "ctx_len is NULL");
  c.check(p->block_table != nullptr, SML_ERR_INVALID_ARG, "block_table is NULL");
}

void check_cache(Checker& c, sml_cache cache, const char* what, bool latent) {
  std::string w(what);
  if (!cache.base) c.fail(SML_ERR_INVALID_ARG, (w + ".base is NULL").c_str());
  else if (!aligned(cache.base, 256)) c.fail(SML_ERR_INVALID_ARG, (w + ".base not 256-B aligned").c_str());
  if (cache.num_pages < 1) c.fail(SML_ERR_INVALID_ARG, (w + ".num_pages < 1").c_str());
  if (!latent) {
    if (cache.format != 0) c.fail(SML_ERR_UNSUPPORTED, (w + ".format not 0").c_str());
  } else if (cache.format == SML_LATENT_E4M3) {
    if (!(isfinite(cache.scale) && cache.scale > 0.f))
      c.fail(SML_ERR_INVALID_ARG, (w + ".scale not finite and positive").c_str());
  } else if (cache.format != SML_LATENT_FP8_DS_MLA && cache.format != SML_LATENT_BF16) {
    c.fail(SML_ERR_UNSUPPORTED, (w + ".format not an SML_LATENT_* format").c_str());
  }
}

struct Layout {
  size_t header = 0, counters = 0, cand_key = 0, cand_idx = 0, cand_cnt = 0, part_out = 0, part_lse = 0,
         scores = 0, total = 0;
};

int topk_chunks(const sml_problem& p) { return (p.max_ctx + kTopkChunk - 1) / kTopkChunk; }

// One fixed layout for every stage: [header][top-k counters][top-k candidates]
// [MLA partials][scores].  A stage's size is the end of the last region it
// uses, so a workspace sized for a later stage serves every earlier one, and
// the top-k arrival counters (which must stay zero between calls) are never
// overwritten by another stage.
Layout layout(const sml_problem& p, int stage) {
  Layout L;
  size_t off = align_up(sizeof(WsHeader));
  L.counters = off;  // sized for the largest T, so no problem's other regions overlap it
  off += align_up((size_t)65536 * sizeof(int32_t));
  const int ch = topk_chunks(p);
  if (ch > 1) {
    const size_t n = (size_t)p.num_tokens * ch * p.topk;
    L.cand_key = off;
    off += align_up(n * sizeof(uint32_t));
    L.cand_idx = off;
    off += align_up(n * sizeof(int32_t));
    L.cand_cnt = off;
    off += align_up((size_t)p.num_tokens * ch * sizeof(int32_t));
  }
  const size_t end_topk = off;
  const size_t slots = mla_slots(mla_plan(p), p.num_tokens) * 16;   // 16 heads per slot
  L.part_out = off;
  off += align_up(slots * SML_LATENT_DIM * sizeof(float));
  L.part_lse = off;
  off += align_up(slots * sizeof(float));
  const size_t end_mla = off;
  L.scores = off;
  off += align_up((size_t)p.num_tokens * p.max_ctx * sizeof(float));
  switch (stage) {
    case SML_STAGE_INDEXER: L.total = align_up(sizeof(WsHeader)); break;
    case SML_STAGE_TOPK: L.total = end_topk; break;
    case SML_STAGE_MLA: L.total = end_mla; break;
    default: L.total = off; break;
  }
  return L;
}

void check_workspace(Checker& c, const sml_problem* p, int stage, void* ws, size_t bytes) {
  if (!ws) {
    c.fail(SML_ERR_WORKSPACE, "workspace is NULL");
    return;
  }
  if (!aligned(ws, 256)) c.fail(SML_ERR_WORKSPACE, "workspace not 256-B aligned");
  if (p && c.code == SML_OK) {
    const size_t need = layout(*p, stage).total;
    if (bytes < need) {
      char buf[128];
      snprintf(buf, sizeof buf, "workspace has %zu bytes, needs %zu", bytes, need);
      c.fail(SML_ERR_WORKSPACE, buf);
    }
  }
}

int32_t* status_of(void* ws) { return &static_cast<WsHeader*>(ws)->status; }

TopkWs topk_ws(const sml_problem& p, const Layout& L, void* ws) {
  char* b = static_cast<char*>(ws);
  TopkWs t;
  t.counters = reinterpret_cast<int32_t*>(b + L.counters);
  t.cand_key = L.cand_key ? reinterpret_cast<uint32_t*>(b + L.cand_key) : nullptr;
  t.cand_idx = L.cand_idx ? reinterpret_cast<int32_t*>(b + L.cand_idx) : nullptr;
  t.cand_cnt = L.cand_cnt ? reinterpret_cast<int32_t*>(b + L.cand_cnt) : nullptr;
  t.chunks = topk_chunks(p);
  return t;
}

MlaWs mla_ws(const sml_problem& p, const Layout& L, void* ws) {
  char* b = static_cast<char*>(ws);
  MlaWs m;
  m.plan = mla_plan(p);
  m.part_out = reinterpret_cast<float*>(b + L.part_out);
  m.part_lse = reinterpret_cast<float*>(b + L.part_lse);
  return m;
}

int cuda_fail(cudaError_t e, const char* fn) {
  g_last_error = std::string(fn) + ": " + cudaGetErrorString(e);
  return SML_ERR_CUDA;
}

}  // namespace

int device_sm_count() {
  static std::mutex mu;
  static int count[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  std::lock_guard<std::mutex> g(mu);
  if (count[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    count[dev] = n > 0 ? n : 148;
  }
  return count[dev];
}

cudaError_t set_max_smem(const void* func, size_t bytes) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, size_t> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> g(mu);
  size_t& have = done[{func, dev}];
  if (have >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) have = bytes;
  return e;
}

size_t topk_region_bytes(const sml_problem& p) { return layout(p, SML_STAGE_TOPK).total; }
size_t mla_region_bytes(const sml_problem& p) { return layout(p, SML_STAGE_MLA).total; }

}  // namespace sml

using namespace sml;

extern "C" {

size_t sml_workspace_size(const sml_problem* p, int stage) {
  Checker c;
  check_problem(c, p);
  c.check(stage >= SML_STAGE_INDEXER && stage <= SML_STAGE_LAYER, SML_ERR_INVALID_ARG,
          "stage not one of SML_STAGE_*");
  if (c.done("sml_workspace_size") != SML_OK) return 0;
  return layout(*p, stage).total;
}

int sml_workspace_init(void* workspace, size_t ws_bytes, void* stream) {
  Checker c;
  c.check(workspace != nullptr, SML_ERR_WORKSPACE, "workspace is NULL");
  c.check(workspace == nullptr || aligned(workspace, 256), SML_ERR_WORKSPACE,
          "workspace not 256-B aligned");
  c.check(ws_bytes >= sizeof(WsHeader), SML_ERR_WORKSPACE, "workspace smaller than its header");
  if (c.done("sml_workspace_init") != SML_OK) return c.code;
  // Header plus the largest counter array any problem using this workspace can
  // have: zero the whole buffer, which is what the callers allocate anyway.
  cudaError_t e = cudaMemsetAsync(workspace, 0, ws_bytes, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SML_OK : cuda_fail(e, "sml_workspace_init");
}

int sml_indexer_scores(const sml_problem* p, const void* iq8, const float* iq_scale, const float* iw,
                       sml_cache index_cache, float* scores, void* workspace, size_t ws_bytes,
                       void* stream) {
  Checker c;
  check_problem(c, p);
  c.check(iq8 != nullptr && aligned(iq8, 16), SML_ERR_INVALID_ARG, "iq8 NULL or not 16-B aligned");
  c.check(iq_scale != nullptr, SML_ERR_INVALID_ARG, "iq_scale is NULL");
  c.check(iw != nullptr, SML_ERR_INVALID_ARG, "iw is NULL");
  c.check(scores != nullptr, SML_ERR_INVALID_ARG, "scores is NULL");
  check_cache(c, index_cache, "index_cache", false);
  check_workspace(c, p, SML_STAGE_INDEXER, workspace, ws_bytes);
  if (c.done("sml_indexer_scores") != SML_OK) return c.code;
  cudaError_t e = launch_indexer(*p, static_cast<const uint8_t*>(iq8), iq_scale, iw,
                                 static_cast<const uint8_t*>(index_cache.base), index_cache.num_pages,
                                 scores, status_of(workspace), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SML_OK : cuda_fail(e, "sml_indexer_scores");
}

int sml_topk(const sml_problem* p, const float* scores, int32_t* idx, int32_t* idx_len,
             void* workspace, size_t ws_bytes, void* stream) {
  Checker c;
  check_problem(c, p);
  c.check(scores != nullptr, SML_ERR_INVALID_ARG, "scores is NULL");
  c.check(idx != nullptr, SML_ERR_INVALID_ARG, "idx is NULL");
  c.check(idx_len != nullptr, SML_ERR_INVALID_ARG, "idx_len is NULL");
  check_workspace(c, p, SML_STAGE_TOPK, workspace, ws_bytes);
  if (c.done("sml_topk") != SML_OK) return c.code;
  const Layout L = layout(*p, SML_STAGE_TOPK);
  cudaError_t e = launch_topk(*p, scores, idx, idx_len, topk_ws(*p, L, workspace),
                              status_of(workspace), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SML_OK : cuda_fail(e, "sml_topk");
}

int sml_sparse_mla_decode(const sml_problem* p, const void* q, sml_cache latent,
                          const int32_t* idx, const int32_t* idx_len, float* out, float* lse,
                          void* workspace, size_t ws_bytes, void* stream) {
  Checker c;
  check_problem(c, p);
  c.check(q != nullptr && aligned(q, 16), SML_ERR_INVALID_ARG, "q NULL or not 16-B aligned");
  c.check(idx != nullptr, SML_ERR_INVALID_ARG, "idx is NULL");
  c.check(idx_len != nullptr, SML_ERR_INVALID_ARG, "idx_len is NULL");
  c.check(out != nullptr && aligned(out, 16), SML_ERR_INVALID_ARG, "out NULL or not 16-B aligned");
  c.check(lse != nullptr, SML_ERR_INVALID_ARG, "lse is NULL");
  check_cache(c, latent, "latent", true);
  check_workspace(c, p, SML_STAGE_MLA, workspace, ws_bytes);
  if (c.done("sml_sparse_mla_decode") != SML_OK) return c.code;
  const Layout L = layout(*p, SML_STAGE_MLA);
  cudaError_t e = launch_sparse_mla(*p, static_cast<const uint16_t*>(q), latent, idx,
                                    idx_len, out, lse, mla_ws(*p, L, workspace), status_of(workspace),
                                    static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SML_OK : cuda_fail(e, "sml_sparse_mla_decode");
}

int sml_run_layer(const sml_problem* p, const void* q, const void* iq8, const float* iq_scale,
                  const float* iw, sml_cache latent, sml_cache index_cache,
                  const int32_t* reuse_idx, const int32_t* reuse_len, int32_t* idx_out,
                  int32_t* len_out, float* out, float* lse, void* workspace, size_t ws_bytes,
                  void* stream) {
  Checker c;
  check_problem(c, p);
  const bool reuse = reuse_idx != nullptr;
  c.check(q != nullptr && aligned(q, 16), SML_ERR_INVALID_ARG, "q NULL or not 16-B aligned");
  c.check(out != nullptr && aligned(out, 16), SML_ERR_INVALID_ARG, "out NULL or not 16-B aligned");
  c.check(lse != nullptr, SML_ERR_INVALID_ARG, "lse is NULL");
  check_cache(c, latent, "latent", true);
  if (reuse) {
    c.check(reuse_len != nullptr, SML_ERR_INVALID_ARG, "reuse_idx given without reuse_len");
  } else {
    c.check(reuse_len == nullptr, SML_ERR_INVALID_ARG, "reuse_len given without reuse_idx");
    c.check(iq8 != nullptr && aligned(iq8, 16), SML_ERR_INVALID_ARG, "iq8 NULL or not 16-B aligned");
    c.check(iq_scale != nullptr, SML_ERR_INVALID_ARG, "iq_scale is NULL");
    c.check(iw != nullptr, SML_ERR_INVALID_ARG, "iw is NULL");
    c.check(idx_out != nullptr, SML_ERR_INVALID_ARG, "idx_out is NULL");
    c.check(len_out != nullptr, SML_ERR_INVALID_ARG, "len_out is NULL");
    check_cache(c, index_cache, "index_cache", false);
  }
  check_workspace(c, p, SML_STAGE_LAYER, workspace, ws_bytes);
  if (c.done("sml_run_layer") != SML_OK) return c.code;
  const Layout L = layout(*p, SML_STAGE_LAYER);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* status = status_of(workspace);
  cudaError_t e = cudaSuccess;
  const int32_t* use_idx = reuse_idx;
  const int32_t* use_len = reuse_len;
  if (!reuse) {
    float* scores = reinterpret_cast<float*>(static_cast<char*>(workspace) + L.scores);
    e = launch_indexer(*p, static_cast<const uint8_t*>(iq8), iq_scale, iw,
                       static_cast<const uint8_t*>(index_cache.base), index_cache.num_pages, scores,
                       status, st);
    if (e == cudaSuccess) e = launch_topk(*p, scores, idx_out, len_out, topk_ws(*p, L, workspace), status, st);
    use_idx = idx_out;
    use_len = len_out;
  }
  if (e == cudaSuccess)
    e = launch_sparse_mla(*p, static_cast<const uint16_t*>(q), latent, use_idx, use_len, out, lse,
                          mla_ws(*p, L, workspace), status,
                          st);
  return e == cudaSuccess ? SML_OK : cuda_fail(e, "sml_run_layer");
}

// ---- producers ------------------------------------------------------------------

namespace {

void check_producer(Checker& c, int32_t n, const int32_t* slot, sml_cache cache, const char* what,
                    int64_t max_pages, void* workspace, bool latent) {
  c.check(n >= 0, SML_ERR_INVALID_ARG, "n < 0");
  c.check(n == 0 || (slot != nullptr && aligned(slot, 4)), SML_ERR_INVALID_ARG, "slot NULL or not 4-B aligned");
  check_cache(c, cache, what, latent);
  c.check(cache.num_pages <= max_pages, SML_ERR_UNSUPPORTED, "num_pages * 64 slots exceed int32");
  c.check(workspace == nullptr || aligned(workspace, 256), SML_ERR_WORKSPACE, "workspace not 256-B aligned");
}

constexpr int64_t kMaxSlotPages = ((int64_t)1 << 31) / SML_PAGE_TOKENS;

}  // namespace

int sml_indexer_k_cache_write(const void* k, const int32_t* slot, int32_t n, sml_cache index_cache,
                              void* workspace, void* stream) {
  Checker c;
  check_producer(c, n, slot, index_cache, "index_cache", kMaxSlotPages, workspace, false);
  c.check(n == 0 || (k != nullptr && aligned(k, 16)), SML_ERR_INVALID_ARG, "k NULL or not 16-B aligned");
  if (c.done("sml_indexer_k_cache_write") != SML_OK) return c.code;
  cudaError_t e = launch_indexer_k_write(k, slot, n, const_cast<void*>(index_cache.base), index_cache.num_pages,
                                         workspace ? status_of(workspace) : nullptr,
                                         static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SML_OK : cuda_fail(e, "sml_indexer_k_cache_write");
}

int sml_latent_cache_write(const void* cl, const void* k_pe, const int32_t* slot, int32_t n, sml_cache latent,
                           void* workspace, void* stream) {
  Checker c;
  check_producer(c, n, slot, latent, "latent", kMaxSlotPages, workspace, true);
  c.check(n == 0 || (cl != nullptr && aligned(cl, 16)), SML_ERR_INVALID_ARG, "c NULL or not 16-B aligned");
  c.check(aligned(k_pe, 16), SML_ERR_INVALID_ARG, "k_pe not 16-B aligned");
  if (c.done("sml_latent_cache_write") != SML_OK) return c.code;
  cudaError_t e = launch_latent_write(cl, k_pe, slot, n, latent, workspace ? status_of(workspace) : nullptr,
                                      static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SML_OK : cuda_fail(e, "sml_latent_cache_write");
}

int sml_indexer_q_quant(const void* iq, int32_t num_tokens, void* iq8, float* iq_scale, void* stream) {
  Checker c;
  c.check(num_tokens >= 0, SML_ERR_INVALID_ARG, "num_tokens < 0");
  const bool any = num_tokens > 0;
  c.check(!any || (iq != nullptr && aligned(iq, 16)), SML_ERR_INVALID_ARG, "iq NULL or not 16-B aligned");
  c.check(!any || (iq8 != nullptr && aligned(iq8, 16)), SML_ERR_INVALID_ARG, "iq8 NULL or not 16-B aligned");
  c.check(!any || (iq_scale != nullptr && aligned(iq_scale, 4)), SML_ERR_INVALID_ARG,
          "iq_scale NULL or not 4-B aligned");
  if (c.done("sml_indexer_q_quant") != SML_OK) return c.code;
  cudaError_t e = launch_indexer_q_quant(iq, num_tokens, iq8, iq_scale, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SML_OK : cuda_fail(e, "sml_indexer_q_quant");
}

// ---- decode context parallelism -------------------------------------------------------

int sml_dcp_merge_candidates(const sml_dcp_ranks* ranks, int32_t num_tokens, int32_t topk, float* merged_scores,
                             int32_t* merged_pos, int32_t* merged_len, void* workspace, void* stream) {
  Checker c;
  c.check(ranks != nullptr, SML_ERR_INVALID_ARG, "ranks is NULL");
  c.check(num_tokens >= 0, SML_ERR_INVALID_ARG, "num_tokens < 0");
  c.check(topk >= 1 && topk <= SML_MAX_TOPK, SML_ERR_UNSUPPORTED, "topk not in [1, 2048]");
  c.check(workspace == nullptr || aligned(workspace, 256), SML_ERR_WORKSPACE, "workspace not 256-B aligned");
  if (ranks) {
    c.check(ranks->num_ranks >= 1 && ranks->num_ranks <= SML_DCP_MAX_RANKS, SML_ERR_UNSUPPORTED,
            "num_ranks not in [1, SML_DCP_MAX_RANKS]");
    c.check(ranks->interleave >= 1, SML_ERR_INVALID_ARG, "interleave < 1");
    const int R = ranks->num_ranks >= 1 && ranks->num_ranks <= SML_DCP_MAX_RANKS ? ranks->num_ranks : 0;
    c.check(ranks->packed == 0 || ranks->packed == 1, SML_ERR_INVALID_ARG, "ranks->packed not 0 or 1");
    for (int r = 0; r < R && num_tokens > 0; ++r) {
      c.check(ranks->scores[r] != nullptr, SML_ERR_INVALID_ARG, "ranks->scores[r] is NULL");
      c.check(ranks->idx[r] != nullptr, SML_ERR_INVALID_ARG, "ranks->idx[r] is NULL");
      c.check(ranks->idx_len[r] != nullptr, SML_ERR_INVALID_ARG, "ranks->idx_len[r] is NULL");
      if (ranks->packed) continue;   // positions past int32 are reported by the kernel
      c.check(ranks->score_stride[r] >= 1 && ranks->score_stride[r] <= (1 << 30), SML_ERR_INVALID_ARG,
              "ranks->score_stride[r] not in [1, 2^30]");
      c.check(ranks->score_stride[r] * (int64_t)R <= INT32_MAX, SML_ERR_UNSUPPORTED,
              "ranks->score_stride[r] * num_ranks exceeds int32 (global positions are int32)");
    }
  }
  const bool any = num_tokens > 0;
  c.check(!any || merged_scores != nullptr, SML_ERR_INVALID_ARG, "merged_scores is NULL");
  c.check(!any || merged_pos != nullptr, SML_ERR_INVALID_ARG, "merged_pos is NULL");
  c.check(!any || merged_len != nullptr, SML_ERR_INVALID_ARG, "merged_len is NULL");
  if (c.done("sml_dcp_merge_candidates") != SML_OK) return c.code;
  cudaError_t e = launch_dcp_merge(*ranks, num_tokens, topk, merged_scores, merged_pos, merged_len,
                                   workspace ? status_of(workspace) : nullptr, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SML_OK : cuda_fail(e, "sml_dcp_merge_candidates");
}

int sml_dcp_pack_candidates(int32_t num_tokens, int32_t topk, const float* scores, int64_t score_stride,
                            const int32_t* idx, const int32_t* idx_len, float* cand_scores, void* workspace,
                            void* stream) {
  Checker c;
  c.check(num_tokens >= 0, SML_ERR_INVALID_ARG, "num_tokens < 0");
  c.check(topk >= 1 && topk <= SML_MAX_TOPK, SML_ERR_UNSUPPORTED, "topk not in [1, 2048]");
  c.check(score_stride >= 1 && score_stride <= (1 << 30), SML_ERR_INVALID_ARG, "score_stride not in [1, 2^30]");
  c.check(workspace == nullptr || aligned(workspace, 256), SML_ERR_WORKSPACE, "workspace not 256-B aligned");
  const bool any = num_tokens > 0;
  c.check(!any || (scores && idx && idx_len && cand_scores), SML_ERR_INVALID_ARG,
          "scores, idx, idx_len or cand_scores is NULL");
  if (c.done("sml_dcp_pack_candidates") != SML_OK) return c.code;
  cudaError_t e = launch_dcp_pack(num_tokens, topk, scores, score_stride, idx, idx_len, cand_scores,
                                  workspace ? status_of(workspace) : nullptr, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SML_OK : cuda_fail(e, "sml_dcp_pack_candidates");
}

int sml_dcp_split_selection(int32_t num_ranks, int32_t interleave, int32_t num_tokens, int32_t topk,
                            const int32_t* sel, const int32_t* sel_len, const int32_t* merged_pos,
                            int32_t* const* local_idx, int32_t* const* local_len, void* workspace, void* stream) {
  Checker c;
  c.check(num_ranks >= 1 && num_ranks <= SML_DCP_MAX_RANKS, SML_ERR_UNSUPPORTED,
          "num_ranks not in [1, SML_DCP_MAX_RANKS]");
  c.check(interleave >= 1, SML_ERR_INVALID_ARG, "interleave < 1");
  c.check(num_tokens >= 0, SML_ERR_INVALID_ARG, "num_tokens < 0");
  c.check(topk >= 1 && topk <= SML_MAX_TOPK, SML_ERR_UNSUPPORTED, "topk not in [1, 2048]");
  c.check(workspace == nullptr || aligned(workspace, 256), SML_ERR_WORKSPACE, "workspace not 256-B aligned");
  const bool any = num_tokens > 0;
  c.check(!any || (sel && sel_len && merged_pos), SML_ERR_INVALID_ARG, "sel, sel_len or merged_pos is NULL");
  c.check(!any || (local_idx && local_len), SML_ERR_INVALID_ARG, "local_idx or local_len is NULL");
  if (any && local_idx && local_len && num_ranks >= 1 && num_ranks <= SML_DCP_MAX_RANKS)
    for (int r = 0; r < num_ranks; ++r)
      c.check(local_idx[r] && local_len[r], SML_ERR_INVALID_ARG, "local_idx[r] or local_len[r] is NULL");
  if (c.done("sml_dcp_split_selection") != SML_OK) return c.code;
  cudaError_t e = launch_dcp_split(num_ranks, interleave, num_tokens, topk, sel, sel_len, merged_pos, local_idx,
                                   local_len, workspace ? status_of(workspace) : nullptr,
                                   static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SML_OK : cuda_fail(e, "sml_dcp_split_selection");
}

int sml_lse_combine(int32_t num_parts, int32_t num_tokens, int32_t num_heads, const float* const* part_out,
                    const float* const* part_lse, float* out, float* lse, void* stream) {
  Checker c;
  c.check(num_parts >= 1 && num_parts <= SML_DCP_MAX_RANKS, SML_ERR_UNSUPPORTED,
          "num_parts not in [1, SML_DCP_MAX_RANKS]");
  c.check(num_tokens >= 0, SML_ERR_INVALID_ARG, "num_tokens < 0");
  c.check(num_heads >= 1 && num_heads <= 65535, SML_ERR_INVALID_ARG, "num_heads not in [1, 65535]");
  const bool any = num_tokens > 0;
  c.check(!any || (part_out && part_lse), SML_ERR_INVALID_ARG, "part_out or part_lse is NULL");
  if (any && part_out && part_lse && num_parts >= 1 && num_parts <= SML_DCP_MAX_RANKS)
    for (int r = 0; r < num_parts; ++r)
      c.check(part_out[r] && aligned(part_out[r], 16) && part_lse[r], SML_ERR_INVALID_ARG,
              "part_out[r] NULL or not 16-B aligned, or part_lse[r] NULL");
  c.check(!any || (out && aligned(out, 16)), SML_ERR_INVALID_ARG, "out NULL or not 16-B aligned");
  c.check(!any || lse, SML_ERR_INVALID_ARG, "lse is NULL");
  if (c.done("sml_lse_combine") != SML_OK) return c.code;
  cudaError_t e = launch_lse_combine(num_parts, num_tokens, num_heads, part_out, part_lse, out, lse,
                                     static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SML_OK : cuda_fail(e, "sml_lse_combine");
}

int sml_read_device_status(void* workspace, int clear, int32_t* bits, void* stream) {
  Checker c;
  c.check(workspace != nullptr, SML_ERR_WORKSPACE, "workspace is NULL");
  if (c.done("sml_read_device_status") != SML_OK) return c.code;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, status_of(workspace), sizeof word, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess && clear) e = cudaMemsetAsync(status_of(workspace), 0, sizeof word, st);
  if (e != cudaSuccess) return cuda_fail(e, "sml_read_device_status");
  if (bits) *bits = word;
  if (word & SML_FAULT_TIMEOUT) return SML_ERR_TIMEOUT;
  return word ? SML_ERR_DEVICE_FAULT : SML_OK;
}

const char* sml_status_string(int code) {
  switch (code) {
    case SML_OK: return "ok";
    case SML_ERR_INVALID_ARG: return "invalid argument";
    case SML_ERR_UNSUPPORTED: return "unsupported shape or option";
    case SML_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case SML_ERR_CUDA: return "CUDA runtime error";
    case SML_ERR_DEVICE_FAULT: return "a device-side check failed";
    case SML_ERR_TIMEOUT: return "a bounded device wait gave up";
    default: return "unknown status";
  }
}

const char* sml_last_error(void) { return g_last_error.c_str(); }

const char* sml_version(void) { return "sml 0.1.0 sm_100a"; }

}  // extern "C"
