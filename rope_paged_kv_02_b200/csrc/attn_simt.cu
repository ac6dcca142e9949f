// Paged attention for float32 caches: one thread per (query row, head), exact fp32
// online softmax over the visible keys.  [3DRoPE-KV] "Attention Computation with Cached
// RoPE": the keys are the visible patch pages in page-table order, then the special stream.
// This path serves small float32 streams (correctness-first); bf16 caches use the tcgen05
// kernel in attn_tc.cu.
#include "../../include/lbm.h"
#include "lbm_internal.h"

namespace lbm {
namespace {

template <int D>
__global__ void __launch_bounds__(64) attn_simt_kernel(const __grid_constant__ SimtParams p) {
  const int h = blockIdx.y;
  const int row = blockIdx.x * blockDim.x + threadIdx.x;
  const bool active = row < p.tokens;
  const float* q = static_cast<const float*>(p.q);
  float qv[D], o[D];
#pragma unroll
  for (int d = 0; d < D; ++d) {
    qv[d] = active ? q[((long long)row * p.heads + h) * D + d] * p.scale : 0.f;
    o[d] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  auto visit = [&](const float* kr, const float* vr) {
    float s = 0.f;
#pragma unroll
    for (int d = 0; d < D; d += 4) {
      const float4 kk = *reinterpret_cast<const float4*>(kr + d);
      s = fmaf(qv[d], kk.x, s);
      s = fmaf(qv[d + 1], kk.y, s);
      s = fmaf(qv[d + 2], kk.z, s);
      s = fmaf(qv[d + 3], kk.w, s);
    }
    const float mn = fmaxf(m, s);
    const float alpha = expf(m - mn);
    const float pe = expf(s - mn);
    l = l * alpha + pe;
#pragma unroll
    for (int d = 0; d < D; d += 4) {
      const float4 vv = *reinterpret_cast<const float4*>(vr + d);
      o[d] = fmaf(o[d], alpha, pe * vv.x);
      o[d + 1] = fmaf(o[d + 1], alpha, pe * vv.y);
      o[d + 2] = fmaf(o[d + 2], alpha, pe * vv.z);
      o[d + 3] = fmaf(o[d + 3], alpha, pe * vv.w);
    }
    m = mn;
  };
  const float* kp = static_cast<const float*>(p.k_patch);
  const float* vp = static_cast<const float*>(p.v_patch);
  const long long head_rows = (long long)p.pool_pages * p.page_stride;
  for (int i = 0; i < p.n_pages; ++i) {
    const long long row0 = (long long)h * head_rows + (long long)p.pages[i] * p.page_stride;
    for (int j = 0; j < p.patches; ++j) visit(kp + (row0 + j) * D, vp + (row0 + j) * D);
  }
  const float* ks = static_cast<const float*>(p.k_special);
  const float* vs = static_cast<const float*>(p.v_special);
  for (int j = 0; j < p.n_special; ++j) {
    const long long r = (long long)h * p.spec_cap + j;
    visit(ks + r * D, vs + r * D);
  }
  if (active) {
    float* out = static_cast<float*>(p.out) + ((long long)row * p.heads + h) * D;
    const float inv = 1.f / l;
#pragma unroll
    for (int d = 0; d < D; ++d) out[d] = o[d] * inv;
  }
}

}  // namespace

cudaError_t launch_attn_simt(const SimtParams& p, cudaStream_t s) {
  dim3 grid((p.tokens + 63) / 64, p.heads, 1);
  if (p.head_dim == 64)
    attn_simt_kernel<64><<<grid, 64, 0, s>>>(p);
  else if (p.head_dim == 128)
    attn_simt_kernel<128><<<grid, 64, 0, s>>>(p);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace lbm
