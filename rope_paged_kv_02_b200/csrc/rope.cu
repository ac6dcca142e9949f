// 3D RoPE kernels: expanded-table writer and the fused rotate + append pass.
//
// [3DRoPE-KV] "Complex-Valued Tensor Application": the rotation is a complex product
// written in real arithmetic; [3DRoPE-KV] "Frame Appending and Position Encoding
// Integration": the rotated k and the plain v are written into the frame's patch page and
// the special stream.  One pass over q, k, v: every 16-byte chunk is loaded once with a
// 128-bit load, its feature pairs rotated in fp32 registers (q and k only), rounded once
// to the storage type and stored with a 128-bit store straight into its destination
// (q in place; k and v into the pools).
#include <cuda_bf16.h>

#include "../../include/lbm.h"
#include "lbm_internal.h"

namespace lbm {
namespace {

struct alignas(16) U4 {
  uint32_t x, y, z, w;
};

__device__ __forceinline__ U4 ld_stream(const void* p) {
  U4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ U4 ld_plain(const void* p) {
  U4 r;
  asm volatile("ld.global.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void st_plain(void* p, const U4& r) {
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(r.x), "r"(r.y),
               "r"(r.z), "r"(r.w)
               : "memory");
}

// (cos, sin) of feature pair i for a token at (t, hh, ww): pairs [0, nt) use the t table,
// [nt, nt+nh) the h table, the rest the w table.  Branch-free (one load), because the lanes
// of a warp cover different pairs of the same token.
__device__ __forceinline__ float2 pair_cs(const RopeTables& rt, int i, int t, int hh, int ww) {
  const bool in_t = i < rt.nt;
  const bool in_h = !in_t && i < rt.nt + rt.nh;
  const float2* base = in_t ? rt.tab_t : (in_h ? rt.tab_h : rt.tab_w);
  const int pairs = in_t ? rt.nt : (in_h ? rt.nh : rt.nw);
  const int row = in_t ? t : (in_h ? hh : ww);
  const int col = in_t ? i : (in_h ? i - rt.nt : i - rt.nt - rt.nh);
  return __ldg(base + row * pairs + col);
}

__device__ __forceinline__ void rot(float& x0, float& x1, float2 cs) {
  const float y0 = fmaf(x0, cs.x, -x1 * cs.y);
  const float y1 = fmaf(x0, cs.y, x1 * cs.x);
  x0 = y0;
  x1 = y1;
}

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);  // .x (low half) = lo
  return *reinterpret_cast<uint32_t*>(&b);
}

// Rotates the 16-byte chunk starting at feature d0 of a token at (t, hh, ww).
template <typename T>
__device__ __forceinline__ U4 rotate_chunk(const RopeTables& rt, U4 in, int d0, int t, int hh,
                                           int ww);

template <>
__device__ __forceinline__ U4 rotate_chunk<__nv_bfloat16>(const RopeTables& rt, U4 in, int d0,
                                                          int t, int hh, int ww) {
  // 8 bf16 = 4 pairs; pair u lives in word u (low half = x[2i], high half = x[2i+1]).
  uint32_t w[4] = {in.x, in.y, in.z, in.w};
  const int i0 = d0 >> 1;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    float x0 = bf_lo(w[u]), x1 = bf_hi(w[u]);
    rot(x0, x1, pair_cs(rt, i0 + u, t, hh, ww));
    w[u] = pack_bf(x0, x1);
  }
  return U4{w[0], w[1], w[2], w[3]};
}

template <>
__device__ __forceinline__ U4 rotate_chunk<float>(const RopeTables& rt, U4 in, int d0, int t,
                                                  int hh, int ww) {
  float x[4] = {__uint_as_float(in.x), __uint_as_float(in.y), __uint_as_float(in.z),
                __uint_as_float(in.w)};
  const int i0 = d0 >> 1;
  rot(x[0], x[1], pair_cs(rt, i0, t, hh, ww));
  rot(x[2], x[3], pair_cs(rt, i0 + 1, t, hh, ww));
  return U4{__float_as_uint(x[0]), __float_as_uint(x[1]), __float_as_uint(x[2]),
            __float_as_uint(x[3])};
}

constexpr int kAppendThreads = 256;
constexpr int kAppendUnroll = 1;

// One pass over the 3 * T * H * (D / EPC) 16-byte chunks of q, k, v (32-bit indices: a
// frame is far below 2^31 chunks): tensor-major (q, k, v), then token, head, chunk, so
// neighbouring threads touch neighbouring 16-byte chunks.  CPR = chunks per (token, head)
// row is a compile-time power of two, so only the division by the head count is a real one.
template <typename T, int CPR>
__global__ void __launch_bounds__(kAppendThreads)
    rope_append_kernel(RopeTables rt, Pools pools, AppendArgs a) {
  constexpr int EPC = 16 / sizeof(T);
  // launched as a programmatic dependent of the previous kernel on the stream (the previous
  // frame's attention may still read the page and slots written here): wait for it to
  // finish before touching memory; the launch itself already overlapped its tail
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const uint32_t per_tensor = (uint32_t)a.tokens * a.heads * CPR;
  const uint32_t total = 3u * per_tensor;
  const uint32_t stride_all = gridDim.x * blockDim.x * kAppendUnroll;
  for (uint32_t base = blockIdx.x * blockDim.x * kAppendUnroll + threadIdx.x; base < total;
       base += stride_all) {
    U4 val[kAppendUnroll];
    // issue every load of this round before any arithmetic (memory-level parallelism)
#pragma unroll
    for (int u = 0; u < kAppendUnroll; ++u) {
      const uint32_t idx = base + u * blockDim.x;
      if (idx < total) {
        const uint32_t tensor = idx >= per_tensor ? (idx >= 2 * per_tensor ? 2u : 1u) : 0u;
        const uint32_t rem = idx - tensor * per_tensor;
        const char* src = tensor == 0 ? (const char*)a.q : tensor == 1 ? (const char*)a.k
                                                                       : (const char*)a.v;
        src += (size_t)rem * 16;
        val[u] = tensor == 0 ? ld_plain(src) : ld_stream(src);
      }
    }
#pragma unroll
    for (int u = 0; u < kAppendUnroll; ++u) {
      const uint32_t idx = base + u * blockDim.x;
      if (idx >= total) continue;
      const uint32_t tensor = idx >= per_tensor ? (idx >= 2 * per_tensor ? 2u : 1u) : 0u;
      const uint32_t rem = idx - tensor * per_tensor;
      const int c = (int)(rem % CPR);
      const uint32_t th = rem / CPR;
      const int j = (int)(th / (uint32_t)a.heads);
      const int h = (int)(th - (uint32_t)j * a.heads);
      const int d0 = c * EPC;
      U4 out = val[u];
      if (tensor < 2) {
        int hh = 0, ww = 0;
        if (j >= a.psi) {
          const int pj = j - a.psi;
          hh = 1 + pj / rt.ppw;
          ww = 1 + pj - (hh - 1) * rt.ppw;
        }
        out = rotate_chunk<T>(rt, out, d0, a.frame, hh, ww);
      }
      char* dst;
      if (tensor == 0) {
        dst = (char*)a.q + (size_t)rem * 16;
      } else {
        const bool special = j < a.psi;
        void* pool = special ? (tensor == 1 ? pools.k_special : pools.v_special)
                             : (tensor == 1 ? pools.k_patch : pools.v_patch);
        size_t row;
        if (special)
          row = (size_t)h * pools.spec_cap + a.special_slot + j;
        else
          row = ((size_t)h * pools.num_pages + a.page) * pools.page_stride + (j - a.psi);
        dst = (char*)pool + (row * CPR + c) * 16;
      }
      st_plain(dst, out);
    }
  }
}

__global__ void rope_expand_kernel(RopeTables rt, float* cos_out, float* sin_out) {
  const int half = rt.head_dim / 2;
  const int T = rt.psi + rt.pph * rt.ppw;
  const long long total = (long long)rt.ppf * T * half;
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const int i = (int)(idx % half);
    const long long r = idx / half;
    const int t = (int)(r / T);
    const int j = (int)(r % T);
    int hh = 0, ww = 0;
    if (j >= rt.psi) {
      hh = 1 + (j - rt.psi) / rt.ppw;
      ww = 1 + (j - rt.psi) % rt.ppw;
    }
    const float2 cs = pair_cs(rt, i, t, hh, ww);
    cos_out[idx] = cs.x;
    sin_out[idx] = cs.y;
  }
}

}  // namespace

cudaError_t launch_rope_expand(const RopeTables& rt, float* cos_out, float* sin_out,
                               cudaStream_t s) {
  const long long total = (long long)rt.ppf * (rt.psi + rt.pph * rt.ppw) * (rt.head_dim / 2);
  long long blocks = (total + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  rope_expand_kernel<<<(unsigned)blocks, 256, 0, s>>>(rt, cos_out, sin_out);
  return cudaGetLastError();
}

cudaError_t launch_rope_append(const RopeTables& rt, const Pools& pools, const AppendArgs& a,
                               cudaStream_t s) {
  const int esz = a.dtype == LBM_BF16 ? 2 : 4;
  const int cpr = a.head_dim * esz / 16;
  const long long chunks = 3LL * a.tokens * a.heads * cpr;
  if (chunks >= (1LL << 31)) return cudaErrorInvalidValue;
  const long long per_block = (long long)kAppendThreads * kAppendUnroll;
  long long blocks = (chunks + per_block - 1) / per_block;
  if (blocks > 148 * 64) blocks = 148 * 64;
  if (blocks < 1) blocks = 1;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(kAppendThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (a.dtype == LBM_BF16 && cpr == 8)
    return cudaLaunchKernelEx(&cfg, rope_append_kernel<__nv_bfloat16, 8>, rt, pools, a);
  if (a.dtype == LBM_BF16 && cpr == 16)
    return cudaLaunchKernelEx(&cfg, rope_append_kernel<__nv_bfloat16, 16>, rt, pools, a);
  if (a.dtype == LBM_F32 && cpr == 16)
    return cudaLaunchKernelEx(&cfg, rope_append_kernel<float, 16>, rt, pools, a);
  if (a.dtype == LBM_F32 && cpr == 32)
    return cudaLaunchKernelEx(&cfg, rope_append_kernel<float, 32>, rt, pools, a);
  return cudaErrorInvalidValue;
}

}  // namespace lbm
