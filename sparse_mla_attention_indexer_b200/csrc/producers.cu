// Producers just before the decode step: FP8 quantisation of new tokens into
// the indexer cache and the fp8_ds_mla latent cache, and of the indexer
// queries.
//
// vLLM blog "vLLM 首日支持 Mistral Large 4", paragraph "可断开的 CUDA 图和融合":
// the indexer Q path and K path are hand-written fused kernels, and the
// indexer K goes straight into the FP8 cache.  A block x becomes E4M3 codes of
// x / s with s = amax|x| / 448 (s = 1 for an all-zero block); s and the
// quotients are IEEE fp32 divisions and the codes round to nearest even with
// saturation (the hardware conversion), so a code is a pure function of the
// block's bf16 bits.
//
// All three are streaming copies with a little arithmetic, bound by how many
// bytes are in flight: every thread issues all of its loads before it uses
// any of them (the slot check does not hold back the data load).  The cache writes take two new
// tokens per warp (a token's 128-B key or 512-B codes are one coalesced store
// per warp, at a slot the block table scatters anywhere in the pool); the
// query quantiser takes one 16-KB token per 256-thread CTA (its loads are all
// in flight at once; staging them through shared memory with bulk copies
// measured slower).
#include <cuda_fp8.h>

#include "ptx.cuh"
#include "sml_internal.cuh"

namespace sml {
namespace {

constexpr int kWarpsPerCta = 8;
constexpr int kTokPerWarp = 2;
constexpr float kE4m3Max = 448.f;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float absmax2(uint32_t w) { return fmaxf(fabsf(bf16_lo(w)), fabsf(bf16_hi(w))); }

__device__ __forceinline__ float block_scale(float amax) {
  return amax > 0.f ? __fdiv_rn(amax, kE4m3Max) : 1.f;
}

__device__ __forceinline__ uint32_t code(float x, float s) {
  return __nv_cvt_float_to_fp8(__fdiv_rn(x, s), __NV_SATFINITE, __NV_E4M3);
}

// Two bf16 values (little-endian pair) -> two codes in the low 16 bits.
__device__ __forceinline__ uint32_t quant2(uint32_t w, float s) {
  return code(bf16_lo(w), s) | (code(bf16_hi(w), s) << 8);
}

// Eight bf16 values -> eight codes, byte i = value i.
__device__ __forceinline__ uint2 quant8(uint4 v, float s) {
  return make_uint2(quant2(v.x, s) | (quant2(v.y, s) << 16), quant2(v.z, s) | (quant2(v.w, s) << 16));
}

__device__ __forceinline__ bool slot_ok(int s, long long slots, int lane, int32_t* status) {
  if (s >= 0 && s < slots) return true;
  if (s != -1 && lane == 0) raise_fault(status, SML_FAULT_PAGE);
  return false;
}

// Two new tokens per warp: 128 bf16 in (256 B) and 128 codes + one scale out each.
__global__ void __launch_bounds__(32 * kWarpsPerCta)
indexer_k_write_kernel(const uint2* __restrict__ k, const int32_t* __restrict__ slot, int n,
                       uint8_t* __restrict__ cache, long long slots, int32_t* status) {
  ptx::griddep_wait();
  if (threadIdx.x == 0) ptx::griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int step = gridDim.x * kWarpsPerCta * kTokPerWarp;
  for (int i0 = (blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5)) * kTokPerWarp; i0 < n; i0 += step) {
    int s[kTokPerWarp];
    uint2 v[kTokPerWarp];
#pragma unroll
    for (int u = 0; u < kTokPerWarp; ++u) {
      const int i = i0 + u;
      s[u] = i < n ? __ldg(slot + i) : -1;
      if (i < n) v[u] = __ldg(k + (size_t)i * (SML_INDEX_DIM / 4) + lane);
    }
#pragma unroll
    for (int u = 0; u < kTokPerWarp; ++u) {
      if (!slot_ok(s[u], slots, lane, status)) continue;
      float a = fmaxf(absmax2(v[u].x), absmax2(v[u].y));
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
      const float sc = block_scale(a);
      uint8_t* page = cache + (size_t)(s[u] / SML_PAGE_TOKENS) * SML_INDEX_PAGE_BYTES;
      const int row = s[u] % SML_PAGE_TOKENS;
      reinterpret_cast<uint32_t*>(page + row * SML_INDEX_DIM)[lane] =
          quant2(v[u].x, sc) | (quant2(v[u].y, sc) << 16);
      if (lane == 0) reinterpret_cast<float*>(page + SML_PAGE_TOKENS * SML_INDEX_DIM)[row] = sc;
    }
  }
}

// Two new tokens per warp: lane l quantises latent values [16 l, 16 l + 16)
// of each, eight lanes per 128-value block; lanes 0..7 copy the 128-B RoPE key.
__global__ void __launch_bounds__(32 * kWarpsPerCta)
latent_write_kernel(const uint4* __restrict__ c, const uint4* __restrict__ kpe, const int32_t* __restrict__ slot,
                    int n, uint8_t* __restrict__ cache, long long slots, int32_t* status) {
  ptx::griddep_wait();
  if (threadIdx.x == 0) ptx::griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int step = gridDim.x * kWarpsPerCta * kTokPerWarp;
  for (int i0 = (blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5)) * kTokPerWarp; i0 < n; i0 += step) {
    int s[kTokPerWarp];
    uint4 v0[kTokPerWarp], v1[kTokPerWarp], pe[kTokPerWarp];
#pragma unroll
    for (int u = 0; u < kTokPerWarp; ++u) {
      const int i = i0 + u;
      s[u] = i < n ? __ldg(slot + i) : -1;
      pe[u] = make_uint4(0, 0, 0, 0);
      if (i < n) {
        const uint4* src = c + (size_t)i * (SML_LATENT_DIM / 8) + 2 * lane;
        v0[u] = __ldg(src);
        v1[u] = __ldg(src + 1);
        if (kpe && lane < 8) pe[u] = __ldg(kpe + (size_t)i * (SML_ROPE_DIM / 8) + lane);
      }
    }
#pragma unroll
    for (int u = 0; u < kTokPerWarp; ++u) {
      if (!slot_ok(s[u], slots, lane, status)) continue;
      const uint4 a0 = v0[u], a1 = v1[u];
      float a = fmaxf(fmaxf(fmaxf(absmax2(a0.x), absmax2(a0.y)), fmaxf(absmax2(a0.z), absmax2(a0.w))),
                      fmaxf(fmaxf(absmax2(a1.x), absmax2(a1.y)), fmaxf(absmax2(a1.z), absmax2(a1.w))));
#pragma unroll
      for (int o = 4; o >= 1; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
      const float sc = block_scale(a);
      uint8_t* row = cache + (size_t)(s[u] / SML_PAGE_TOKENS) * SML_LATENT_PAGE_BYTES +
                     (size_t)(s[u] % SML_PAGE_TOKENS) * SML_LATENT_ROW_BYTES;
      const uint2 q0 = quant8(a0, sc), q1 = quant8(a1, sc);
      reinterpret_cast<uint4*>(row)[lane] = make_uint4(q0.x, q0.y, q1.x, q1.y);
      if ((lane & 7) == 0) reinterpret_cast<float*>(row + SML_LATENT_DIM)[lane >> 3] = sc;
      if (lane < 8) reinterpret_cast<uint4*>(row + SML_LATENT_DIM + 16)[lane] = pe[u];
    }
  }
}

// The plain E4M3 pool (blog, section "ROCm 实现细节", paragraph "FP8 潜在缓存"):
// every one of a row's 576 values becomes the code of x / scale with the
// pool's given scale.  Two new tokens per warp: lane l codes latent values
// [16 l, 16 l + 16) into bytes [16 l, 16 l + 16) of the 576-B row; lanes 0..7
// code RoPE values [8 l, 8 l + 8) into bytes 512 + 8 l.
__global__ void __launch_bounds__(32 * kWarpsPerCta)
latent_write_plain_kernel(const uint4* __restrict__ c, const uint4* __restrict__ kpe,
                          const int32_t* __restrict__ slot, int n, float scale, uint8_t* __restrict__ cache,
                          long long slots, int32_t* status) {
  ptx::griddep_wait();
  if (threadIdx.x == 0) ptx::griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int step = gridDim.x * kWarpsPerCta * kTokPerWarp;
  for (int i0 = (blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5)) * kTokPerWarp; i0 < n; i0 += step) {
    int s[kTokPerWarp];
    uint4 v0[kTokPerWarp], v1[kTokPerWarp], pe[kTokPerWarp];
#pragma unroll
    for (int u = 0; u < kTokPerWarp; ++u) {
      const int i = i0 + u;
      s[u] = i < n ? __ldg(slot + i) : -1;
      pe[u] = make_uint4(0, 0, 0, 0);
      if (i < n) {
        const uint4* src = c + (size_t)i * (SML_LATENT_DIM / 8) + 2 * lane;
        v0[u] = __ldg(src);
        v1[u] = __ldg(src + 1);
        if (kpe && lane < 8) pe[u] = __ldg(kpe + (size_t)i * (SML_ROPE_DIM / 8) + lane);
      }
    }
#pragma unroll
    for (int u = 0; u < kTokPerWarp; ++u) {
      if (!slot_ok(s[u], slots, lane, status)) continue;
      uint8_t* row = cache + (size_t)(s[u] / SML_PAGE_TOKENS) * SML_LATENT_E4M3_PAGE_BYTES +
                     (size_t)(s[u] % SML_PAGE_TOKENS) * SML_LATENT_E4M3_ROW_BYTES;
      const uint2 q0 = quant8(v0[u], scale), q1 = quant8(v1[u], scale);
      reinterpret_cast<uint4*>(row)[lane] = make_uint4(q0.x, q0.y, q1.x, q1.y);
      if (lane < 8) reinterpret_cast<uint2*>(row + SML_LATENT_DIM)[lane] = kpe ? quant8(pe[u], scale) : make_uint2(0, 0);
    }
  }
}

// The bf16 pool (blog, section "ROCm 实现细节", paragraph "FP8 潜在缓存": 1,152 B
// per token per layer in bf16): a row is the token's 512 latent and 64 RoPE
// values as given, no quantisation.  Two new tokens per warp: lane l copies
// latent bytes [32 l, 32 l + 32); lanes 0..7 the RoPE bytes 1,024 + 16 l
// (zeros without a RoPE key).
__global__ void __launch_bounds__(32 * kWarpsPerCta)
latent_write_bf16_kernel(const uint4* __restrict__ c, const uint4* __restrict__ kpe,
                         const int32_t* __restrict__ slot, int n, uint8_t* __restrict__ cache, long long slots,
                         int32_t* status) {
  ptx::griddep_wait();
  if (threadIdx.x == 0) ptx::griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int step = gridDim.x * kWarpsPerCta * kTokPerWarp;
  for (int i0 = (blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5)) * kTokPerWarp; i0 < n; i0 += step) {
    int s[kTokPerWarp];
    uint4 v0[kTokPerWarp], v1[kTokPerWarp], pe[kTokPerWarp];
#pragma unroll
    for (int u = 0; u < kTokPerWarp; ++u) {
      const int i = i0 + u;
      s[u] = i < n ? __ldg(slot + i) : -1;
      pe[u] = make_uint4(0, 0, 0, 0);
      if (i < n) {
        const uint4* src = c + (size_t)i * (SML_LATENT_DIM / 8) + 2 * lane;
        v0[u] = __ldg(src);
        v1[u] = __ldg(src + 1);
        if (kpe && lane < 8) pe[u] = __ldg(kpe + (size_t)i * (SML_ROPE_DIM / 8) + lane);
      }
    }
#pragma unroll
    for (int u = 0; u < kTokPerWarp; ++u) {
      if (!slot_ok(s[u], slots, lane, status)) continue;
      uint8_t* row = cache + (size_t)(s[u] / SML_PAGE_TOKENS) * SML_LATENT_BF16_PAGE_BYTES +
                     (size_t)(s[u] % SML_PAGE_TOKENS) * SML_LATENT_BF16_ROW_BYTES;
      reinterpret_cast<uint4*>(row)[2 * lane] = v0[u];
      reinterpret_cast<uint4*>(row)[2 * lane + 1] = v1[u];
      if (lane < 8) reinterpret_cast<uint4*>(row + 2 * SML_LATENT_DIM)[lane] = pe[u];
    }
  }
}

// One CTA per query token: 64 x 128 bf16 in (16 KB), one block.
constexpr int kQThreads = 256;
constexpr int kQVec = SML_INDEX_HEADS * SML_INDEX_DIM / 8 / kQThreads;   // uint4 loads per thread: 4

__global__ void __launch_bounds__(kQThreads)
indexer_q_quant_kernel(const uint4* __restrict__ iq, int T, uint2* __restrict__ iq8, float* __restrict__ scale) {
  __shared__ float red[kQThreads / 32];
  ptx::griddep_wait();
  if (threadIdx.x == 0) ptx::griddep_launch_dependents();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int kPerToken = SML_INDEX_HEADS * SML_INDEX_DIM / 8;
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    uint4 v[kQVec];
    float a = 0.f;
#pragma unroll
    for (int j = 0; j < kQVec; ++j) {
      v[j] = __ldg(iq + (size_t)t * kPerToken + j * kQThreads + threadIdx.x);
      a = fmaxf(a, fmaxf(fmaxf(absmax2(v[j].x), absmax2(v[j].y)), fmaxf(absmax2(v[j].z), absmax2(v[j].w))));
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if (lane == 0) red[warp] = a;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < kQThreads / 32; ++w) a = fmaxf(a, red[w]);
    const float sc = block_scale(a);
#pragma unroll
    for (int j = 0; j < kQVec; ++j) iq8[(size_t)t * kPerToken + j * kQThreads + threadIdx.x] = quant8(v[j], sc);
    if (threadIdx.x == 0) scale[t] = sc;
    __syncthreads();   // red is reused by the next token
  }
}

int token_grid(int n, int per_cta, int ctas_per_sm) {
  const int want = (n + per_cta - 1) / per_cta;
  const int cap = device_sm_count() * ctas_per_sm;
  return want < cap ? want : cap;
}

}  // namespace

cudaError_t launch_indexer_k_write(const void* k, const int32_t* slot, int n, void* cache, int64_t num_pages,
                                   int32_t* status, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  return launch_pdl(indexer_k_write_kernel, dim3(token_grid(n, kWarpsPerCta * kTokPerWarp, 8)), dim3(32 * kWarpsPerCta), 0,
                    stream, 0, static_cast<const uint2*>(k), slot, n, static_cast<uint8_t*>(cache),
                    (long long)num_pages * SML_PAGE_TOKENS, status);
}

cudaError_t launch_latent_write(const void* c, const void* kpe, const int32_t* slot, int n, const sml_cache& cache,
                                int32_t* status, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const dim3 grid(token_grid(n, kWarpsPerCta * kTokPerWarp, 8)), block(32 * kWarpsPerCta);
  uint8_t* base = static_cast<uint8_t*>(const_cast<void*>(cache.base));
  const long long slots = (long long)cache.num_pages * SML_PAGE_TOKENS;
  if (cache.format == SML_LATENT_BF16)
    return launch_pdl(latent_write_bf16_kernel, grid, block, 0, stream, 0, static_cast<const uint4*>(c),
                      static_cast<const uint4*>(kpe), slot, n, base, slots, status);
  if (cache.format == SML_LATENT_E4M3)
    return launch_pdl(latent_write_plain_kernel, grid, block, 0, stream, 0, static_cast<const uint4*>(c),
                      static_cast<const uint4*>(kpe), slot, n, cache.scale, base, slots, status);
  return launch_pdl(latent_write_kernel, grid, block, 0, stream, 0, static_cast<const uint4*>(c),
                    static_cast<const uint4*>(kpe), slot, n, base, slots, status);
}

cudaError_t launch_indexer_q_quant(const void* iq, int T, void* iq8, float* iq_scale, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  return launch_pdl(indexer_q_quant_kernel, dim3(token_grid(T, 1, 8)), dim3(kQThreads), 0, stream, 0,
                    static_cast<const uint4*>(iq), T, static_cast<uint2*>(iq8), iq_scale);
}

}  // namespace sml
