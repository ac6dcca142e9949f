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

// Rotates the feature pairs of one 16-byte chunk by the given (cos, sin) per pair.
template <typename T>
__device__ __forceinline__ U4 rotate_chunk(U4 in, const float2* cs);

template <>
__device__ __forceinline__ U4 rotate_chunk<__nv_bfloat16>(U4 in, const float2* cs) {
  // 8 bf16 = 4 pairs; pair u lives in word u (low half = x[2i], high half = x[2i+1]).
  uint32_t w[4] = {in.x, in.y, in.z, in.w};
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    float x0 = bf_lo(w[u]), x1 = bf_hi(w[u]);
    rot(x0, x1, cs[u]);
    w[u] = pack_bf(x0, x1);
  }
  return U4{w[0], w[1], w[2], w[3]};
}

template <>
__device__ __forceinline__ U4 rotate_chunk<float>(U4 in, const float2* cs) {
  float x[4] = {__uint_as_float(in.x), __uint_as_float(in.y), __uint_as_float(in.z),
                __uint_as_float(in.w)};
  rot(x[0], x[1], cs[0]);
  rot(x[2], x[3], cs[1]);
  return U4{__float_as_uint(x[0]), __float_as_uint(x[1]), __float_as_uint(x[2]),
            __float_as_uint(x[3])};
}

constexpr int kAppendThreads = 256;

// Thread (token j, 16-byte chunk c) of head group blockIdx.y handles HG consecutive heads:
// the chunk's (cos, sin) pairs depend only on the token and the feature, so they and all the
// index arithmetic are computed once and reused for q and k of every head of the group.
// Lanes run over chunks first, then tokens, so a warp reads whole 128-byte rows of q, k, v
// and, per head, writes consecutive rows of the frame's page.  All 3 * HG loads of a thread
// are issued before the first rotation, to keep enough bytes in flight to cover HBM latency.
// WITH_Q = false: q is left to the attention kernel, which rotates it as it loads it; the
// pass then reads k, v and writes the pools only (4 instead of 6 T H D element moves).
template <typename T, int CPR, int HG, bool WITH_Q>
__global__ void __launch_bounds__(kAppendThreads)
    rope_append_kernel(RopeTables rt, Pools pools, AppendArgs a) {
  constexpr int EPC = 16 / sizeof(T);  // elements per 16-byte chunk
  constexpr int NPC = EPC / 2;         // feature pairs per chunk
  // launched as a programmatic dependent of the previous kernel on the stream (the previous
  // frame's attention may still read the page and slots written here): wait for it to
  // finish before touching memory; the launch itself already overlapped its tail
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const uint32_t items = (uint32_t)a.tokens * CPR;
  const uint32_t idx = blockIdx.x * kAppendThreads + threadIdx.x;
  if (idx >= items) return;
  const int c = (int)(idx % CPR);
  const int j = (int)(idx / CPR);
  const int h0 = blockIdx.y * HG;

  // sources: [tokens][heads][CPR] chunks
  const size_t row_chunks = (size_t)a.heads * CPR;
  const size_t src0 = (size_t)j * row_chunks + (size_t)h0 * CPR + c;
  U4 vq[HG], vk[HG], vv[HG];
#pragma unroll
  for (int u = 0; u < HG; ++u) {
    if (WITH_Q) vq[u] = ld_plain((const char*)a.q + (src0 + u * CPR) * 16);
    vk[u] = ld_stream((const char*)a.k + (src0 + u * CPR) * 16);
    vv[u] = ld_stream((const char*)a.v + (src0 + u * CPR) * 16);
  }

  int hh = 0, ww = 0;
  const bool special = j < a.psi;
  if (!special) {
    const int pj = j - a.psi;
    hh = 1 + pj / rt.ppw;
    ww = 1 + pj - (hh - 1) * rt.ppw;
  }
  float2 cs[NPC];
  const int i0 = c * NPC;
#pragma unroll
  for (int u = 0; u < NPC; ++u) cs[u] = pair_cs(rt, i0 + u, a.frame, hh, ww);

  // destinations: the special stream [heads][spec_cap] or the frame's page
  // [heads][num_pages * page_stride] rows of CPR chunks
  size_t dst0, head_step;
  char *kpool, *vpool;
  if (special) {
    kpool = (char*)pools.k_special;
    vpool = (char*)pools.v_special;
    head_step = (size_t)pools.spec_cap * CPR;
    dst0 = ((size_t)h0 * pools.spec_cap + a.special_slot + j) * CPR + c;
  } else {
    kpool = (char*)pools.k_patch;
    vpool = (char*)pools.v_patch;
    head_step = (size_t)pools.num_pages * pools.page_stride * CPR;
    dst0 = (((size_t)h0 * pools.num_pages + a.page) * pools.page_stride + (j - a.psi)) * CPR + c;
  }
#pragma unroll
  for (int u = 0; u < HG; ++u) {
    if (WITH_Q) st_plain((char*)a.q + (src0 + u * CPR) * 16, rotate_chunk<T>(vq[u], cs));
    st_plain(kpool + (dst0 + u * head_step) * 16, rotate_chunk<T>(vk[u], cs));
    st_plain(vpool + (dst0 + u * head_step) * 16, vv[u]);
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
  const long long items = (long long)a.tokens * cpr;
  if (items <= 0 || 3LL * items * a.heads >= (1LL << 31)) return cudaErrorInvalidValue;
  // heads per thread: the most (4, 2, 1) that still leaves two blocks of 256 threads per SM
  // in flight (small frames need the threads to cover HBM latency more than the reuse)
  const long long min_threads = 148LL * 2 * kAppendThreads;
  int hg = 1;
  if (a.heads % 4 == 0 && items * (a.heads / 4) >= min_threads)
    hg = 4;
  else if (a.heads % 2 == 0 && items * (a.heads / 2) >= min_threads)
    hg = 2;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3((unsigned)((items + kAppendThreads - 1) / kAppendThreads),
                     (unsigned)(a.heads / hg));
  cfg.blockDim = dim3(kAppendThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
#define LBM_APPEND_LAUNCH_Q(T, C, Q)                                                        \
  if (hg == 4) return cudaLaunchKernelEx(&cfg, rope_append_kernel<T, C, 4, Q>, rt, pools, a); \
  if (hg == 2) return cudaLaunchKernelEx(&cfg, rope_append_kernel<T, C, 2, Q>, rt, pools, a); \
  return cudaLaunchKernelEx(&cfg, rope_append_kernel<T, C, 1, Q>, rt, pools, a);
#define LBM_APPEND_LAUNCH(T, C)             \
  if (a.q != nullptr) {                     \
    LBM_APPEND_LAUNCH_Q(T, C, true)         \
  } else {                                  \
    LBM_APPEND_LAUNCH_Q(T, C, false)        \
  }
  if (a.dtype == LBM_BF16 && cpr == 8) { LBM_APPEND_LAUNCH(__nv_bfloat16, 8) }
  if (a.dtype == LBM_BF16 && cpr == 16) { LBM_APPEND_LAUNCH(__nv_bfloat16, 16) }
  if (a.dtype == LBM_F32 && cpr == 16) { LBM_APPEND_LAUNCH(float, 16) }
  if (a.dtype == LBM_F32 && cpr == 32) { LBM_APPEND_LAUNCH(float, 32) }
#undef LBM_APPEND_LAUNCH
#undef LBM_APPEND_LAUNCH_Q
  return cudaErrorInvalidValue;
}

}  // namespace lbm
