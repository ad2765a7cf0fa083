// DSA indexer scores over a paged FP8 indexer cache.
//
// vLLM blog "vLLM 首日支持 Mistral Large 4", section "实现细节 / 模型架构":
// the sparse indexer reads an FP8 indexer cache and has its own SSMax; section
// "ROCm 实现细节": one FP8 scale per key, 132 B per token.  Score of query
// token t against cached token s < n_t:
//   I[t, s] = c_t * sq_t * sk_s * sum_h w[t, h] * ReLU(q8[t, h, :] . k8[s, :])
//
// One CTA scores one 64-token page of one request for up to kQChunk of its
// query tokens.  FP8 codes are widened exactly to fp32; each product of two
// E4M3 values is exact in fp32 and the sums accumulate in fp32.
#include <cuda_fp8.h>

#include "sml_internal.cuh"

namespace sml {
namespace {

constexpr int kQChunk = 16;
constexpr int kThreads = 256;
constexpr int kPad = 129;  // row pitch in floats: conflict-free column reads

__device__ __forceinline__ void e4m3x16_to_f32(uint4 v, float* dst) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[i] & 0xffffu), __NV_E4M3);
    const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[i] >> 16), __NV_E4M3);
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&lo));
    const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&hi));
    dst[4 * i + 0] = a.x;
    dst[4 * i + 1] = a.y;
    dst[4 * i + 2] = b.x;
    dst[4 * i + 3] = b.y;
  }
}

__global__ void __launch_bounds__(kThreads)
indexer_page_kernel(int B, int T, int max_pages, int max_ctx, int ssmax, float s_index,
                    const int32_t* __restrict__ cu_q, const int32_t* __restrict__ ctx_len,
                    const int32_t* __restrict__ block_table, const uint8_t* __restrict__ iq8,
                    const float* __restrict__ iq_scale, const float* __restrict__ iw,
                    const uint8_t* __restrict__ index_base, int64_t index_pages,
                    float* __restrict__ scores, int32_t* status) {
  extern __shared__ float dsm[];
  float (*ks)[kPad] = reinterpret_cast<float (*)[kPad]>(dsm);                      // [64][kPad]
  float (*qs)[kPad] = reinterpret_cast<float (*)[kPad]>(dsm + SML_PAGE_TOKENS * kPad);
  __shared__ float ksc[SML_PAGE_TOKENS];
  __shared__ float wsh[SML_INDEX_HEADS];
  __shared__ float part[4][SML_PAGE_TOKENS];
  const int tid = threadIdx.x;
  const int pg = blockIdx.x, r = blockIdx.y;
  const Req rq = load_request(cu_q, ctx_len, r, T, max_ctx, max_pages);
  const int q0 = rq.q0, Q = rq.Q, L = rq.L;
  if (!rq.ok) {
    if (pg == 0 && blockIdx.z == 0 && tid == 0) raise_fault(status, SML_FAULT_LENGTHS);
    return;
  }
  if (pg * SML_PAGE_TOKENS >= L) return;
  const int jb = blockIdx.z * kQChunk;
  if (jb >= Q) return;
  const int je = min(Q, jb + kQChunk);
  const int phys = __ldg(block_table + (size_t)r * max_pages + pg);
  if (phys < 0 || phys >= index_pages) {
    if (tid == 0) raise_fault(status, SML_FAULT_PAGE);
    return;
  }
  const uint8_t* page = index_base + (size_t)phys * SML_INDEX_PAGE_BYTES;
  for (int v = tid; v < SML_PAGE_TOKENS * SML_INDEX_DIM / 16; v += kThreads) {
    float tmp[16];
    e4m3x16_to_f32(__ldg(reinterpret_cast<const uint4*>(page) + v), tmp);
    const int row = v / 8, col = (v % 8) * 16;
#pragma unroll
    for (int i = 0; i < 16; ++i) ks[row][col + i] = tmp[i];
  }
  if (tid < SML_PAGE_TOKENS)
    ksc[tid] = __ldg(reinterpret_cast<const float*>(page + SML_PAGE_TOKENS * SML_INDEX_DIM) + tid);

  const int tok = tid & 63, hg = tid >> 6;
  for (int j = jb; j < je; ++j) {
    const int n = L - Q + j + 1;
    if (pg * SML_PAGE_TOKENS >= n) continue;  // uniform: page not visible to query j
    const int t = q0 + j;
    __syncthreads();
    const uint8_t* qrow = iq8 + (size_t)t * SML_INDEX_HEADS * SML_INDEX_DIM;
    for (int v = tid; v < SML_INDEX_HEADS * SML_INDEX_DIM / 16; v += kThreads) {
      float tmp[16];
      e4m3x16_to_f32(__ldg(reinterpret_cast<const uint4*>(qrow) + v), tmp);
      const int row = v / 8, col = (v % 8) * 16;
#pragma unroll
      for (int i = 0; i < 16; ++i) qs[row][col + i] = tmp[i];
    }
    if (tid < SML_INDEX_HEADS) wsh[tid] = __ldg(iw + (size_t)t * SML_INDEX_HEADS + tid);
    __syncthreads();
    float acc = 0.f;
    for (int h = hg * 16; h < hg * 16 + 16; ++h) {
      float dot = 0.f;
#pragma unroll 8
      for (int d = 0; d < SML_INDEX_DIM; ++d) dot = fmaf(qs[h][d], ks[tok][d], dot);
      acc = fmaf(wsh[h], fmaxf(dot, 0.f), acc);
    }
    part[hg][tok] = acc;
    __syncthreads();
    if (tid < SML_PAGE_TOKENS) {
      const int s = pg * SML_PAGE_TOKENS + tid;
      if (s < n) {
        const float c = ssmax ? s_index * logf((float)n) : 1.f;
        const float sum = (part[0][tid] + part[1][tid]) + (part[2][tid] + part[3][tid]);
        scores[(size_t)t * max_ctx + s] = sum * __ldg(iq_scale + t) * ksc[tid] * c;
      }
    }
  }
}

}  // namespace

cudaError_t launch_indexer(const sml_problem& p, const uint8_t* iq8, const float* iq_scale,
                           const float* iw, const uint8_t* index_base, int64_t index_pages,
                           float* scores, int32_t* status, cudaStream_t stream) {
  // Query chunks: enough for the request with the most query tokens (<= T).
  const int qchunks = (p.num_tokens - p.num_requests + 1 + kQChunk - 1) / kQChunk;
  dim3 grid(p.max_pages, p.num_requests, qchunks);
  const size_t smem = (size_t)(SML_PAGE_TOKENS + SML_INDEX_HEADS) * kPad * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(indexer_page_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  indexer_page_kernel<<<grid, kThreads, smem, stream>>>(
      p.num_requests, p.num_tokens, p.max_pages, p.max_ctx, p.ssmax, p.ssmax_s_index, p.cu_q, p.ctx_len,
      p.block_table, iq8, iq_scale, iw, index_base, index_pages, scores, status);
  return cudaGetLastError();
}

}  // namespace sml
