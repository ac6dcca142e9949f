// Internal interfaces between the C ABI glue (lbm.cpp) and the CUDA kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <vector>

namespace lbm {

// Per-axis cos/sin tables on the device, float2 (cos, sin), rounded once from double.
// Feature pair i of a token at (t, h, w) takes the t table for i < nt, the h table for
// nt <= i < nt + nh and the w table after.  The 2D (y, x) variant has nt = 0, its h and w
// tables being the y and x halves (one row per token of a frame).
struct RopeTables {
  int head_dim, ppf, pph, ppw, psi;
  int nt, nh, nw;          // pairs of the t, h, w axes (d_t/2, d_h/2, d_w/2)
  const float2* tab_t;     // [ppf][nt] (no rows when nt = 0)
  const float2* tab_h;     // [pph + 1][nh] (2D: [psi + pph * ppw][nh])
  const float2* tab_w;     // [ppw + 1][nw] (2D: [psi + pph * ppw][nw])
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
  void* q;            // rotated in place; NULL: left to the attention kernel
  const void* k;
  const void* v;
};

constexpr int kMaxPages = 1024;

// Keys per K/V tile of the tensor-core attention: 128 at head_dim 64; 64 at head_dim 128,
// where two score buffers of a query tile then fit next to its 128 output columns in tensor
// memory.  Host (tile counts, tensor-map boxes) and kernel use this one definition.
__host__ __device__ constexpr int attn_key_tile(int head_dim) { return head_dim == 64 ? 128 : 64; }

constexpr int kMaxGrid = 1024;  // persistent attention CTAs per launch, at most
constexpr int kMaxUnits = 1024;  // units whose key order the planner rotates (see AttnParams)

// Shared memory the attention kernel sets aside for the RoPE tables of its in-kernel q
// rotation: the frame's t row and the h and w tables, (nt + (pph+1) nh + (ppw+1) nw) float2.
// Larger tables are read from global memory instead.
constexpr int kRopeStageBytes = 24 * 1024;
inline bool rope_fits_stage(const RopeTables& rt) {
  return ((long long)rt.nt + (long long)(rt.pph + 1) * rt.nh + (long long)(rt.ppw + 1) * rt.nw) *
             8 <= kRopeStageBytes;
}

// Kernel parameter block of the paged attention (passed by value).
// Stream-K partition of one frame's attention over `grid` persistent CTAs.  A unit is one
// (pair of 128-row query tiles, head), unit u = head * n_pairs + pair; its key tiles are the
// global work items [u * n_tiles, (u + 1) * n_tiles).  CTA c processes the contiguous items
// [sk_start[c], sk_start[c + 1]) (never empty), i.e. a run of segments (unit, key-tile
// range); a segment that is a whole unit writes the final output, any other writes a
// partial (O, LSE) into slot unit + c (dense: at most units + grid slots), merged by the
// combine kernel.  The host places the boundaries by cost (sk_partition).
struct AttnParams {
  CUtensorMap tm_q;      // q   {head_dim, heads, T}: raw (rotate_q) or already rotated
  CUtensorMap tm_kp;     // K patch pool {head_dim, P*stride, heads}
  CUtensorMap tm_vp;
  CUtensorMap tm_ks;     // K special pool {head_dim, spec_cap, heads}
  CUtensorMap tm_vs;
  void* q_rot_out;       // nullable [T][heads][head_dim] bf16: the rotated q the kernel used
  RopeTables rope;       // tables of the in-kernel rotation of q
  int rotate_q;          // 1: rotate q at its tokens' positions before Q.K^T
  int rope_staged;       // 1: the kernel copies the tables to shared memory (they fit)
  int frame;             // t coordinate of the frame (absolute frame index)
  void* out;             // [T][heads][head_dim] bf16
  float* part_o;         // [units + grid slots][256 rows][head_dim] fp32 partial outputs
  float* part_lse;       // [units + grid slots][256 rows] log2-domain LSE
  int* err;              // device error word (bounded waits)
  unsigned long long wait_limit_ns;  // limit of one wait of the kernel's roles
  int tokens;            // T
  int heads;
  int patches;           // valid tokens per patch page
  int page_stride;
  int tiles_per_page;    // key tiles per patch page: ceil(patches / attn_key_tile(D))
  uint32_t tpp_magic;    // ceil(2^32 / tiles_per_page) (tiles_per_page > 1): division by it
  int n_pages;           // visible patch pages
  int n_special;         // visible special tokens
  int n_tiles;           // n_pages * tiles_per_page + ceil(n_special / attn_key_tile(D))
  int n_pairs;           // ceil(ceil(T / 128) / 2) query-tile pairs
  long long work;        // n_pairs * heads * n_tiles
  int grid;              // persistent CTAs
  float scale_log2;      // log2(e) / sqrt(head_dim)
  uint16_t pages[kMaxPages];
  int sk_start[kMaxGrid + 1];  // first work item of CTA c; sk_start[grid] = work
  // Key-tile order inside each unit: item i of unit u reads key tile (i + rot[u]) mod n_tiles.
  // The 2 n_pairs query tiles of a head read the same keys; rotating each unit so that the CTA
  // entering it is at key tile ~tau at time tau keeps the CTAs of a head (and of all heads) on
  // nearly the same key tiles at the same time, so each K/V tile comes from DRAM about once
  // and from L2 for the other query tiles.  When units > kMaxUnits no unit is rotated (the
  // kernel reads rot[u] only for u < kMaxUnits).
  int rot[kMaxUnits];
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
// dynamic shared memory of one attention CTA (checked against the device at cache creation)
size_t attn_tc_smem_bytes(int head_dim, bool fold);
cudaError_t launch_attn_tc(const AttnParams& p, int head_dim, cudaStream_t s);
// merges the partial results of every unit that spans more than one CTA
cudaError_t launch_attn_combine(const AttnParams& p, int head_dim, cudaStream_t s);
// floats of partial results a frame may write: (units + grid) slots of 256 rows x (D + 1)
inline size_t sk_scratch_floats(long long units, int grid, int head_dim) {
  return (size_t)(units + grid) * 256 * (size_t)(head_dim + 1);
}
// Relative costs of the stream-K partition, measured on the tensor-core kernel: a key-tile
// step of a pair with two query tiles (both softmax warpgroups busy), a step of a pair with
// a single query tile, and the pipeline refill at the start of every segment.
constexpr long long kCostPairStep = 6;
constexpr long long kCostSingleStep = 5;
constexpr long long kCostSegment = 10;

// Fills p.sk_start[0 .. p.grid] (needs p.n_tiles, n_pairs, heads, tokens, work, grid with
// 1 <= grid <= min(work, kMaxGrid)): CTA c starts at the first item whose cost offset reaches
// c / grid of the frame's total cost; then every CTA is given at least one item.
inline void sk_partition(AttnParams& p) {
  const int q_tiles = (p.tokens + 127) / 128;
  const bool last_single = (q_tiles & 1) != 0;
  const long long nt = p.n_tiles;
  auto unit_cost = [&](int pair) {
    const bool single = last_single && pair == p.n_pairs - 1;
    return kCostSegment + nt * (single ? kCostSingleStep : kCostPairStep);
  };
  const long long per_head = (long long)(p.n_pairs - 1) * unit_cost(0) + unit_cost(p.n_pairs - 1);
  const long long total = per_head * p.heads;
  for (int c = 0; c <= p.grid; ++c) {
    const long long v = (long long)((__int128)c * total / p.grid);
    long long x;
    if (c == p.grid) {
      x = p.work;
    } else {
      const long long head = v / per_head;
      long long r = v - head * per_head;
      int pair = 0;
      while (pair < p.n_pairs - 1 && r >= unit_cost(pair)) r -= unit_cost(pair++);
      const long long w = last_single && pair == p.n_pairs - 1 ? kCostSingleStep : kCostPairStep;
      // item t > 0 of the unit starts at cost kCostSegment + t * w (item 0 at 0)
      long long t = r <= 0 ? 0 : (r - kCostSegment + w - 1) / w;
      if (r > 0 && t < 1) t = 1;
      if (t > nt) t = nt;
      x = ((long long)head * p.n_pairs + pair) * nt + t;
    }
    p.sk_start[c] = (int)x;
  }
  // non-empty shares: strictly increasing starts, each leaving room for the CTAs after it
  for (int c = 1; c < p.grid; ++c) {
    long long x = p.sk_start[c];
    if (x < (long long)p.sk_start[c - 1] + 1) x = p.sk_start[c - 1] + 1;
    if (x > p.work - (p.grid - c)) x = p.work - (p.grid - c);
    p.sk_start[c] = (int)x;
  }
}

// Fills p.rot (needs p.sk_start).  Unit u starts in exactly one CTA's range [S_c, S_{c+1});
// that CTA reaches the unit's first item after u * n_tiles - S_c items of its own, so rotating
// the unit by that amount (mod n_tiles) has it read key tile tau at its step tau.  When the
// next CTA holds a longer part of the unit (from item a = S_{c+1} - u * n_tiles, at its step
// 0), the unit is rotated for that CTA instead (by -a), so the larger part of every unit is
// read in phase; the other part is off by less than n_tiles.
inline void sk_rotations(AttnParams& p) {
  const long long units = (long long)p.n_pairs * p.heads;
  if (units > kMaxUnits) {
    for (int u = 0; u < kMaxUnits; ++u) p.rot[u] = 0;
    return;
  }
  const long long n = p.n_tiles;
  int c = 0;
  for (long long u = 0; u < units; ++u) {
    const long long first = u * n, end = first + n;
    while (c + 1 < p.grid && p.sk_start[c + 1] <= first) ++c;
    const long long own = std::min<long long>(p.sk_start[c + 1], end) - first;
    const long long next = c + 1 < p.grid ? std::min<long long>(p.sk_start[c + 2], end) -
                                                std::min<long long>(p.sk_start[c + 1], end)
                                          : 0;
    if (next > own)
      p.rot[u] = (int)((n - (p.sk_start[c + 1] - first) % n) % n);
    else
      p.rot[u] = (int)((first - p.sk_start[c]) % n);
  }
}

// Multiplier m = ceil(2^32 / d) with which floor(t * m / 2^32) = t / d for every t < n
// (exact while n * d <= 2^32: the error t * (m - 2^32/d) / 2^32 stays below 1/d); 0 when that
// does not hold or d == 1, and the kernel then divides.
inline uint32_t tile_div_magic(int d, long long n) {
  if (d <= 1 || (unsigned long long)n * (unsigned long long)d > (1ull << 32)) return 0u;
  return (uint32_t)(((1ull << 32) + (unsigned long long)d - 1) / (unsigned long long)d);
}

// true when some unit is shared by two CTAs (then the combine kernel must run)
inline bool sk_has_split(const AttnParams& p) {
  for (int c = 1; c < p.grid; ++c)
    if (p.sk_start[c] % p.n_tiles != 0) return true;
  return false;
}

// attn_static.cu: device address of the file-scope stream-K scratch on `device` (current)
int noalloc_scratch(int device, float** ptr, size_t* floats);

// attn_simt.cu (fp32)
cudaError_t launch_attn_simt(const SimtParams& p, cudaStream_t s);

}  // namespace lbm
