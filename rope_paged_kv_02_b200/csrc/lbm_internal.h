// Internal interfaces between the C ABI glue (lbm.cpp) and the CUDA kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <vector>

namespace lbm {

// Per-axis cos/sin tables on the device, float2 (cos, sin), rounded once from double.
struct RopeTables {
  int head_dim, ppf, pph, ppw, psi;
  int nt, nh, nw;          // pairs of the t, h, w axes (d_t/2, d_h/2, d_w/2)
  const float2* tab_t;     // [ppf][nt]
  const float2* tab_h;     // [pph + 1][nh]
  const float2* tab_w;     // [ppw + 1][nw]
};

// Device pools of one cache.  Patch pools: [heads][num_pages * page_stride][head_dim];
// special pools: [heads][spec_cap][head_dim].
struct Pools {
  void* k_patch;
  void* v_patch;
  void* k_special;
  void* v_special;
  int num_pages;
  int page_stride;  // tokens per page slot (patches_per_frame rounded up to 128)
  int spec_cap;     // special stream capacity in tokens (multiple of 128)
};

struct AppendArgs {
  int dtype;  // LBM_F32 / LBM_BF16
  int heads, head_dim, tokens, psi;
  int frame;          // absolute frame index (t coordinate)
  int page;           // patch page of this frame
  int special_slot;   // first special slot of this frame
  void* q;            // rotated in place
  const void* k;
  const void* v;
};

constexpr int kMaxPages = 1024;

// Kernel parameter block of the paged attention (passed by value).
// Stream-K partition of one frame's attention over `grid` persistent CTAs.  A unit is one
// (pair of 128-row query tiles, head), unit u = head * n_pairs + pair; its key tiles are the
// global work items [u * n_tiles, (u + 1) * n_tiles).  CTA c processes the contiguous items
// [sk_lo(c), sk_lo(c + 1)), i.e. a run of segments (unit, key-tile range); a segment that
// is a whole unit writes the final output, any other writes a partial (O, LSE) into slot
// unit + c (dense: at most units + grid slots), merged by the combine kernel.
__host__ __device__ inline long long sk_lo(long long work, int grid, int c) {
  return (long long)c * work / grid;
}

struct AttnParams {
  CUtensorMap tm_q;      // q   {head_dim, heads, T}
  CUtensorMap tm_kp;     // K patch pool {head_dim, P*stride, heads}
  CUtensorMap tm_vp;
  CUtensorMap tm_ks;     // K special pool {head_dim, spec_cap, heads}
  CUtensorMap tm_vs;
  void* out;             // [T][heads][head_dim] bf16
  float* part_o;         // [units + grid slots][256 rows][head_dim] fp32 partial outputs
  float* part_lse;       // [units + grid slots][256 rows] log2-domain LSE
  int* err;              // device error word (bounded waits)
  int tokens;            // T
  int heads;
  int patches;           // valid tokens per patch page
  int page_stride;
  int tiles_per_page;    // key tiles per patch page: ceil(patches / 128)
  int n_pages;           // visible patch pages
  int n_special;         // visible special tokens
  int n_tiles;           // n_pages * tiles_per_page + ceil(n_special / 128)
  int n_pairs;           // ceil(ceil(T / 128) / 2) query-tile pairs
  long long work;        // n_pairs * heads * n_tiles
  int grid;              // persistent CTAs
  float scale_log2;      // log2(e) / sqrt(head_dim)
  uint16_t pages[kMaxPages];
};

struct SimtParams {
  const void* q;
  void* out;
  const void* k_patch;
  const void* v_patch;
  const void* k_special;
  const void* v_special;
  int tokens, heads, head_dim;
  int patches, page_stride, pool_pages, spec_cap;
  int n_pages, n_special;
  float scale;
  uint16_t pages[kMaxPages];  // visible patch pages, visible order
};

// rope.cu
cudaError_t launch_rope_expand(const RopeTables& rt, float* cos_out, float* sin_out,
                               cudaStream_t s);
cudaError_t launch_rope_append(const RopeTables& rt, const Pools& pools,
                               const AppendArgs& a, cudaStream_t s);

// attn_tc.cu (bf16, tcgen05)
size_t attn_tc_smem_bytes(int head_dim);
cudaError_t launch_attn_tc(const AttnParams& p, int head_dim, cudaStream_t s);
// merges the partial results of every unit that spans more than one CTA
cudaError_t launch_attn_combine(const AttnParams& p, int head_dim, cudaStream_t s);
// floats of partial results a frame may write: (units + grid) slots of 256 rows x (D + 1)
inline size_t sk_scratch_floats(long long units, int grid, int head_dim) {
  return (size_t)(units + grid) * 256 * (size_t)(head_dim + 1);
}
// true when some unit is shared by two CTAs (then the combine kernel must run)
inline bool sk_has_split(long long work, int grid, int n_tiles) {
  for (int c = 1; c < grid; ++c)
    if (sk_lo(work, grid, c) % n_tiles != 0) return true;
  return false;
}

// attn_static.cu: device address of the file-scope split-KV scratch on `device` (current)
int noalloc_scratch(int device, float** ptr, size_t* floats);

// attn_simt.cu (fp32)
cudaError_t launch_attn_simt(const SimtParams& p, cudaStream_t s);

}  // namespace lbm
