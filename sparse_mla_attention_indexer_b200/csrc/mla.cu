// Absorbed-query sparse MLA over a paged fp8_ds_mla latent cache, split over
// the selected keys, followed by a log-sum-exp merge of the splits.
//
// vLLM blog "vLLM 首日支持 Mistral Large 4": highlights list (MLA, KV LoRA
// rank 512, RoPE dim 64, top-2048 keys per query); section "实现细节 / 模型架构"
// (sparse MLA over the fp8_ds_mla latent cache; NoPE = RoPE dim 0 on the same
// cache; SSMax on the MLA query); section "长上下文" (partial results merged by
// their LSE).  For token t, head h over the selected set S_t:
//   z_i = sm_scale * c_t * (q_nope . c_hat_i + q_pe . k_pe_i)
//   out = sum_i softmax(z)_i c_hat_i,   lse = ln sum_i exp(z_i)
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <math.h>

#include "sml_internal.cuh"

namespace sml {
namespace {

constexpr int kHG = 16;       // heads per CTA
constexpr int kTile = 16;     // keys per shared-memory tile
constexpr int kThreads = 256;
constexpr int kPitch = 577;   // floats per smem row (576 + 1: conflict-free)

__global__ void __launch_bounds__(kThreads, 1)
sparse_mla_split_kernel(int B, int T, int H, int K, int rope_dim, int max_pages, int max_ctx, int ssmax,
                        float sm_scale, float ssmax_s, const int32_t* __restrict__ cu_q,
                        const int32_t* __restrict__ ctx_len, const int32_t* __restrict__ block_table,
                        const uint16_t* __restrict__ q, const uint8_t* __restrict__ latent,
                        int64_t latent_pages, const int32_t* __restrict__ idx,
                        const int32_t* __restrict__ idx_len, MlaWs ws, int32_t* status) {
  extern __shared__ float smem[];
  float* qf = smem;                     // [kHG][kPitch]
  float* kf = qf + kHG * kPitch;        // [kTile][kPitch]
  float* ps = kf + kTile * kPitch;      // [kHG][kTile]
  __shared__ int rowvalid[kTile];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x, hg = blockIdx.y, t = blockIdx.z;
  const int S = ws.splits;
  const int Dq = SML_LATENT_DIM + rope_dim;
  const int r = request_of(cu_q, B, t);
  const Req rq = load_request(cu_q, ctx_len, r, T, max_ctx, max_pages);
  const int q0 = rq.q0, Q = rq.Q, L = rq.L;
  const bool ok = rq.ok && t >= q0 && t - q0 < Q;
  if (!ok && split == 0 && hg == 0 && tid == 0) raise_fault(status, SML_FAULT_LENGTHS);
  const int n = ok ? L - Q + (t - q0) + 1 : 0;
  int len = ok ? __ldg(idx_len + t) : 0;
  const int len_max = min(K, n);
  if (len < 0 || len > len_max) {
    if (split == 0 && hg == 0 && tid == 0) raise_fault(status, SML_FAULT_TOPK_LEN);
    len = max(0, min(len, len_max));
  }
  const int kb = split * ws.keys_per_split;
  const int ke = min(len, kb + ws.keys_per_split);
  const float zscale = sm_scale * (ssmax ? ssmax_s * logf((float)max(n, 1)) : 1.f);

  // Query heads hg*16 .. +16, bf16 -> fp32.
  for (int e = tid; e < kHG * Dq; e += kThreads) {
    const int h = e / Dq, d = e % Dq;
    const uint16_t bits = __ldg(q + ((size_t)t * H + hg * kHG + h) * Dq + d);
    qf[h * kPitch + d] = __uint_as_float((uint32_t)bits << 16);
  }

  const int oh = tid >> 4;      // head owned in the softmax and the output
  const int ok_lane = tid & 15; // key (logits) / dim group (output)
  float m = -INFINITY, l = 0.f;
  float acc[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) acc[j] = 0.f;

  for (int tile = kb; tile < ke; tile += kTile) {
    const int nk = min(kTile, ke - tile);
    __syncthreads();  // previous tile fully consumed (and qf written)
    // Gather: each warp loads 2 rows.
    for (int rr = warp * 2; rr < warp * 2 + 2; ++rr) {
      bool valid = false;
      const uint8_t* row = nullptr;
      if (rr < nk) {
        const int pos = __ldg(idx + (size_t)t * K + tile + rr);
        if (pos >= 0 && pos < n) {
          const int phys = __ldg(block_table + (size_t)r * max_pages + pos / SML_PAGE_TOKENS);
          if (phys >= 0 && phys < latent_pages) {
            valid = true;
            row = latent + (size_t)phys * SML_LATENT_PAGE_BYTES +
                  (size_t)(pos % SML_PAGE_TOKENS) * SML_LATENT_ROW_BYTES;
          } else if (lane == 0) {
            raise_fault(status, SML_FAULT_PAGE);
          }
        } else if (lane == 0) {
          raise_fault(status, SML_FAULT_INDEX);
        }
      }
      if (lane == 0) rowvalid[rr] = valid;
      float* dst = kf + rr * kPitch;
      if (valid) {
        const float4 sc = __ldg(reinterpret_cast<const float4*>(row + SML_LATENT_DIM));
        const float scale = (lane < 8) ? sc.x : (lane < 16) ? sc.y : (lane < 24) ? sc.z : sc.w;
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(row) + lane);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[i] & 0xffffu), __NV_E4M3);
          const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[i] >> 16), __NV_E4M3);
          const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&lo));
          const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&hi));
          dst[lane * 16 + 4 * i + 0] = a.x * scale;
          dst[lane * 16 + 4 * i + 1] = a.y * scale;
          dst[lane * 16 + 4 * i + 2] = b.x * scale;
          dst[lane * 16 + 4 * i + 3] = b.y * scale;
        }
        if (rope_dim && lane < 8) {
          const uint4 pe = __ldg(reinterpret_cast<const uint4*>(row + SML_LATENT_DIM + 16) + lane);
          const uint32_t pw[4] = {pe.x, pe.y, pe.z, pe.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            dst[SML_LATENT_DIM + lane * 8 + 2 * i + 0] = __uint_as_float(pw[i] << 16);
            dst[SML_LATENT_DIM + lane * 8 + 2 * i + 1] = __uint_as_float(pw[i] & 0xffff0000u);
          }
        }
      } else if (rr < kTile) {
        for (int d = lane; d < Dq; d += 32) dst[d] = 0.f;
      }
    }
    __syncthreads();
    // Logits: thread (head oh, key ok_lane).
    float z = -INFINITY;
    if (ok_lane < nk && rowvalid[ok_lane]) {
      const float* qv = qf + oh * kPitch;
      const float* kv = kf + ok_lane * kPitch;
      float dot = 0.f;
#pragma unroll 8
      for (int d = 0; d < Dq; ++d) dot = fmaf(qv[d], kv[d], dot);
      z = dot * zscale;
    }
    float tmax = z;
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
    const float m_new = fmaxf(m, tmax);
    float alpha = 1.f, p = 0.f;
    if (m_new != -INFINITY) {
      alpha = (m == -INFINITY) ? 0.f : expf(m - m_new);
      p = (z == -INFINITY) ? 0.f : expf(z - m_new);
    }
    float psum = p;
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
    l = l * alpha + psum;
    m = m_new;
    ps[oh * kTile + ok_lane] = p;
    __syncthreads();
    // Output: thread (head oh, dims ok_lane + 16 j).
    const float* prow = ps + oh * kTile;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int d = ok_lane + 16 * j;
      float a = acc[j] * alpha;
      for (int k = 0; k < nk; ++k) a = fmaf(prow[k], kf[k * kPitch + d], a);
      acc[j] = a;
    }
  }

  const int h = hg * kHG + oh;
  const size_t slot = ((size_t)t * H + h) * S + split;
  float* po = ws.part_out + slot * SML_LATENT_DIM;
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int j = 0; j < 32; ++j) po[ok_lane + 16 * j] = acc[j] * inv;
  if (ok_lane == 0) ws.part_lse[slot] = l > 0.f ? m + logf(l) : -INFINITY;
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
  // Enough (token, head-group, split) CTAs to fill the GPU twice, splits of
  // whole 64-key groups.
  const int ctas = p.num_tokens * (p.num_heads / kHG);
  int S = (2 * 148 + ctas - 1) / ctas;
  const int groups = (p.topk + 63) / 64;
  S = S < 1 ? 1 : (S > groups ? groups : S);
  const int kps = ((groups + S - 1) / S) * 64;
  S = (p.topk + kps - 1) / kps;
  if (keys_per_split) *keys_per_split = kps;
  return S;
}

cudaError_t launch_sparse_mla(const sml_problem& p, const uint16_t* q, const uint8_t* latent_base,
                              int64_t latent_pages, const int32_t* idx, const int32_t* idx_len,
                              float* out, float* lse, const MlaWs& ws, int32_t* status,
                              cudaStream_t stream) {
  const size_t smem = (size_t)(kHG * kPitch + kTile * kPitch + kHG * kTile) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(sparse_mla_split_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(ws.splits, p.num_heads / kHG, p.num_tokens);
  sparse_mla_split_kernel<<<grid, kThreads, smem, stream>>>(
      p.num_requests, p.num_tokens, p.num_heads, p.topk, p.rope_dim, p.max_pages, p.max_ctx, p.ssmax,
      p.sm_scale, p.ssmax_s, p.cu_q, p.ctx_len, p.block_table, q, latent_base, latent_pages, idx,
      idx_len, ws, status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  lse_merge_kernel<<<dim3(p.num_heads, p.num_tokens), 128, 0, stream>>>(p.num_heads, ws, out, lse);
  return cudaGetLastError();
}

}  // namespace sml
