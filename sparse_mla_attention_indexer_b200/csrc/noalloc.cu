// sml_sparse_mla_decode_noalloc: sparse MLA decode whose split partials live in
// a fixed scratch array compiled into the library, for callers that cannot
// hand the library a workspace (see include/sml.h).
#include <math.h>
#include <stdio.h>

#include <mutex>
#include <string>

#include "sml_internal.cuh"

namespace sml {

// Scratch for the per-split partial outputs and LSEs.  Every GPU that loads
// libsml.so holds these bytes until the process exits.
constexpr size_t kNoallocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];
// The sticky device status word of this entry point (SML_FAULT_* bits), in
// place of the one a workspace would hold; zero when the library loads.
static __device__ __align__(256) int32_t g_noalloc_status;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
struct DeviceAddrs {
  void* scratch;
  int32_t* status;
};
DeviceAddrs g_addr[kMaxDevices] = {};

// Device addresses of the scratch array and the status word on the current
// device, looked up once per device (the host-side names of the arrays are not
// device addresses).
cudaError_t device_addresses(DeviceAddrs* out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev].scratch) {
    void* p = nullptr;
    void* st = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    e = cudaGetSymbolAddress(&st, g_noalloc_status);
    if (e != cudaSuccess) return e;
    g_addr[dev].scratch = p;
    g_addr[dev].status = static_cast<int32_t*>(st);
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace sml

using namespace sml;

extern "C" int sml_sparse_mla_decode_noalloc(const sml_problem* p, const void* q, sml_cache latent,
                                             const int32_t* idx, const int32_t* idx_len, float* out,
                                             float* lse, void* stream) {
  std::string msg;
  int code = SML_OK;
  auto fail = [&](int c, const std::string& what) {
    if (!msg.empty()) msg += "; ";
    msg += what;
    if (code == SML_OK || (code == SML_ERR_UNSUPPORTED && c != SML_ERR_UNSUPPORTED)) code = c;
  };
  // Same argument checks as sml_sparse_mla_decode: validate through its sizing
  // helper, which records every failed problem check.
  const size_t mla_bytes = p ? sml_workspace_size(p, SML_STAGE_MLA) : 0;
  if (!p || mla_bytes == 0) fail(SML_ERR_INVALID_ARG, p ? sml_last_error() : "problem is NULL");
  if (!q || ((uintptr_t)q % 16)) fail(SML_ERR_INVALID_ARG, "q NULL or not 16-B aligned");
  if (!idx) fail(SML_ERR_INVALID_ARG, "idx is NULL");
  if (!idx_len) fail(SML_ERR_INVALID_ARG, "idx_len is NULL");
  if (!out || ((uintptr_t)out % 16)) fail(SML_ERR_INVALID_ARG, "out NULL or not 16-B aligned");
  if (!lse) fail(SML_ERR_INVALID_ARG, "lse is NULL");
  if (!latent.base || ((uintptr_t)latent.base % 256)) fail(SML_ERR_INVALID_ARG, "latent.base NULL or not 256-B aligned");
  if (latent.num_pages < 1) fail(SML_ERR_INVALID_ARG, "latent.num_pages < 1");
  if (latent.format == SML_LATENT_E4M3) {
    if (!(isfinite(latent.scale) && latent.scale > 0.f)) fail(SML_ERR_INVALID_ARG, "latent.scale not finite and positive");
  } else if (latent.format != SML_LATENT_FP8_DS_MLA && latent.format != SML_LATENT_BF16) {
    fail(SML_ERR_UNSUPPORTED, "latent.format not an SML_LATENT_* format");
  }
  MlaWs ws{};
  size_t need = 0;
  if (code == SML_OK) {
    ws.plan = mla_plan(*p);
    const size_t slots = mla_slots(ws.plan, p->num_tokens) * 16;
    const size_t out_bytes = align_up(slots * SML_LATENT_DIM * sizeof(float));
    need = out_bytes + align_up(slots * sizeof(float));
    if (need > kNoallocScratchBytes) {
      char buf[200];
      snprintf(buf, sizeof buf,
               "problem needs %zu bytes of split scratch (T=%d x H=%d x %d slots per 16 heads), the built-in "
               "scratch holds %zu; use sml_sparse_mla_decode with a workspace",
               need, p->num_tokens, p->num_heads, ws.plan.smax, kNoallocScratchBytes);
      fail(SML_ERR_UNSUPPORTED, buf);
    }
  }
  if (code != SML_OK) {
    set_last_error(std::string("sml_sparse_mla_decode_noalloc: ") + msg);
    return code;
  }
  DeviceAddrs addr{};
  cudaError_t e = device_addresses(&addr);
  if (e == cudaSuccess) {
    char* b = static_cast<char*>(addr.scratch);
    const size_t slots = mla_slots(ws.plan, p->num_tokens) * 16;
    ws.part_out = reinterpret_cast<float*>(b);
    ws.part_lse = reinterpret_cast<float*>(b + align_up(slots * SML_LATENT_DIM * sizeof(float)));
    e = launch_sparse_mla(*p, static_cast<const uint16_t*>(q), latent, idx, idx_len, out, lse, ws, addr.status,
                          static_cast<cudaStream_t>(stream));
  }
  if (e != cudaSuccess) {
    set_last_error(std::string("sml_sparse_mla_decode_noalloc: ") + cudaGetErrorString(e));
    return SML_ERR_CUDA;
  }
  set_last_error("");
  return SML_OK;
}

extern "C" int sml_noalloc_read_status(int clear, int32_t* bits, void* stream) {
  DeviceAddrs addr{};
  cudaError_t e = device_addresses(&addr);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t word = 0;
  if (e == cudaSuccess) e = cudaMemcpyAsync(&word, addr.status, sizeof word, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess && clear) e = cudaMemsetAsync(addr.status, 0, sizeof word, st);
  if (e != cudaSuccess) {
    set_last_error(std::string("sml_noalloc_read_status: ") + cudaGetErrorString(e));
    return SML_ERR_CUDA;
  }
  set_last_error("");
  if (bits) *bits = word;
  if (word & SML_FAULT_TIMEOUT) return SML_ERR_TIMEOUT;
  return word ? SML_ERR_DEVICE_FAULT : SML_OK;
}
