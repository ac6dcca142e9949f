// C ABI glue: RoPE table objects, the cache object (pools, scratch, tensor maps, page
// manager) and the per-frame calls.  All validation happens here, before any state changes
// or launches; the kernels trust their arguments.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstdint>
#include <cstring>
#include <new>
#include <vector>

#include "../../include/lbm.h"
#include "lbm_internal.h"
#include "pager.h"

struct lbm_rope {
  lbm::RopeTables t;
  float2* d_tables = nullptr;
  int device = 0;
};

// K/V pools of one transformer block and their tensor maps.
struct CacheBlock {
  lbm::Pools pools{};
  CUtensorMap tm_kp, tm_vp, tm_ks, tm_vs;
};

constexpr unsigned long long kDefaultWaitLimitNs = 2000000000ull;

struct lbm_cache {
  int heads, head_dim, patches, psi, scale_frames, sliding_window, max_frames, dtype;
  int device = 0;
  int num_sms = 148;
  const lbm_rope* rope = nullptr;
  std::vector<CacheBlock> blocks;  // one per transformer block, sharing the page table
  int next_block = 0;           // block whose append / attention comes next in this frame
  bool block_appended = false;  // next_block has appended this frame and not yet attended
  int frame_mode = 0;           // is_keyframe of the frame in flight (0, 1, deferred)
  void* pool_mem = nullptr;     // one allocation holding every block's four pools
  float* part_o = nullptr;      // partial outputs of units shared by several CTAs
  float* part_lse = nullptr;
  size_t scratch_floats = 0;    // capacity of part_o + part_lse in floats
  int forced_grid = 0;          // LBM_ATTN_GRID at create time (0: one CTA per SM)
  unsigned long long wait_limit_ns = kDefaultWaitLimitNs;  // lbm_cache_set_wait_limit
  int* d_err = nullptr;
  long long device_bytes = 0;
  long long launches = 0;       // kernels launched so far
  bool q_rotated = false;       // the pending block's q was rotated by its append
  CUtensorMap tm_q;             // cached for the last q pointer seen
  const void* tm_q_ptr = nullptr;
  lbm::Pager pager;
  cudaEvent_t ev = nullptr;     // recorded after every launch; orders calls across streams
  cudaStream_t last_stream = nullptr;
  bool ev_valid = false;
  lbm_cache(int s, int w, int m, int psi_) : pager(s, w, m, psi_) {}
};

namespace {

constexpr int kKeyTile = 128;  // page strides are multiples (of every attention key tile)

int elem_size(int dtype) { return dtype == LBM_BF16 ? 2 : 4; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 3-D bf16 tensor map {d0 (contiguous), d1, d2} with strides (bytes) s1, s2 and box
// {64, b1, b2}, 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
              uint64_t s1, uint64_t s2, uint32_t b1, uint32_t b2) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1, s2};
  cuuint32_t box[3] = {64, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

int use_device(int dev) {
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) return LBM_ERR_CUDA;
  if (cur != dev && cudaSetDevice(dev) != cudaSuccess) return LBM_ERR_CUDA;
  return LBM_OK;
}

void order_before(lbm_cache* c, cudaStream_t s) {
  if (c->ev_valid && s != c->last_stream) cudaStreamWaitEvent(s, c->ev, 0);
}

void order_after(lbm_cache* c, cudaStream_t s) {
  cudaEventRecord(c->ev, s);
  c->last_stream = s;
  c->ev_valid = true;
}

// Fills everything of the attention parameters but the partial-result scratch: the visible
// page list (no container), tensor maps, and the stream-K partition of the frame's work
// over the persistent CTAs.  Returns LBM_OK or an error status.
int fill_attn_params(lbm_cache* c, int block, const void* q, void* out, void* q_rot_out,
                     lbm::AttnParams& p) {
  const CacheBlock& bk = c->blocks[block];
  int n_pages = 0;
  for (const auto& e : c->pager.scale()) p.pages[n_pages++] = (uint16_t)e.page;
  for (const auto& e : c->pager.window()) p.pages[n_pages++] = (uint16_t)e.page;
  p.pages[n_pages++] = (uint16_t)c->pager.pending_page();
  const int n_sp = c->pager.n_special() + c->psi;
  const int T = c->psi + c->patches;
  if (q != c->tm_q_ptr) {
    const uint64_t row = (uint64_t)c->head_dim * 2;
    if (!make_map(&c->tm_q, q, c->head_dim, c->heads, T, row, row * c->heads, 1, 128))
      return LBM_ERR_CUDA;
    c->tm_q_ptr = q;
  }
  p.tm_q = c->tm_q;
  p.q_rot_out = q_rot_out;
  p.rope = c->rope->t;
  p.rotate_q = c->q_rotated ? 0 : 1;
  p.rope_staged = p.rotate_q && lbm::rope_fits_stage(c->rope->t) ? 1 : 0;
  p.frame = (int)c->pager.pending_frame();
  p.tm_kp = bk.tm_kp;
  p.tm_vp = bk.tm_vp;
  p.tm_ks = bk.tm_ks;
  p.tm_vs = bk.tm_vs;
  p.out = out;
  p.err = c->d_err;
  p.wait_limit_ns = c->wait_limit_ns;
  p.tokens = T;
  p.heads = c->heads;
  p.patches = c->patches;
  p.page_stride = bk.pools.page_stride;
  const int kt = lbm::attn_key_tile(c->head_dim);  // keys per attention key tile
  p.tiles_per_page = (c->patches + kt - 1) / kt;
  p.tpp_magic = 0u;  // set below once n_tiles is known
  p.n_pages = n_pages;
  p.n_special = n_sp;
  p.n_tiles = p.n_pages * p.tiles_per_page + (n_sp + kt - 1) / kt;
  p.tpp_magic = lbm::tile_div_magic(p.tiles_per_page, p.n_tiles);
  p.n_pairs = ((T + 127) / 128 + 1) / 2;
  p.work = (long long)p.n_pairs * c->heads * p.n_tiles;
  if (p.work >= (1LL << 31)) return LBM_ERR_UNSUPPORTED;  // the kernel counts in 32 bits
  const long long want = c->forced_grid ? c->forced_grid : c->num_sms;
  p.grid = (int)std::min<long long>(std::min<long long>(want, p.work), lbm::kMaxGrid);
  lbm::sk_partition(p);
  lbm::sk_rotations(p);
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)c->head_dim));
  return LBM_OK;
}

// The attention of block next_block has been issued: the next block's turn, and after the
// last block the frame is committed or rolled back (or, decided later, marked attended).
void block_attended(lbm_cache* c) {
  c->block_appended = false;
  if (++c->next_block == (int)c->blocks.size()) {
    c->next_block = 0;
    int evicted = -1;
    c->pager.finish(&evicted);
  }
}

// One axis of a rope object: a table of `rows` positions for the feature pairs of d_axis
// features, angle(p, i) = p * base^(-2i / d_axis).
struct AxisSpec {
  int rows;
  int d_axis;
  double base;
};

// Fills the t, h and w tables (angles in double, cos/sin rounded once to float), uploads them
// and returns the rope object.  An axis with d_axis 0 has no pairs (the 2D variant's t).
int build_rope(lbm::RopeTables t, AxisSpec at, AxisSpec ah, AxisSpec aw, lbm_rope_t** out) {
  t.nt = at.d_axis / 2;
  t.nh = ah.d_axis / 2;
  t.nw = aw.d_axis / 2;
  const size_t n_t = (size_t)at.rows * t.nt, n_h = (size_t)ah.rows * t.nh,
               n_w = (size_t)aw.rows * t.nw;
  std::vector<float2> host(std::max<size_t>(n_t + n_h + n_w, 1));
  auto fill = [&](float2* dst, const AxisSpec& ax) {
    const int pairs = ax.d_axis / 2;
    for (int i = 0; i < pairs; ++i) {
      const double inv = std::pow(ax.base, -(2.0 * i) / (double)ax.d_axis);
      for (int p = 0; p < ax.rows; ++p) {
        const double a = (double)p * inv;
        dst[(size_t)p * pairs + i] = make_float2((float)std::cos(a), (float)std::sin(a));
      }
    }
  };
  fill(host.data(), at);
  fill(host.data() + n_t, ah);
  fill(host.data() + n_t + n_h, aw);
  auto* r = new (std::nothrow) lbm_rope;
  if (!r) return LBM_ERR_NOMEM;
  if (cudaGetDevice(&r->device) != cudaSuccess ||
      cudaMalloc(&r->d_tables, host.size() * sizeof(float2)) != cudaSuccess) {
    delete r;
    cudaGetLastError();
    return LBM_ERR_NOMEM;
  }
  if (cudaMemcpy(r->d_tables, host.data(), host.size() * sizeof(float2),
                 cudaMemcpyHostToDevice) != cudaSuccess) {
    cudaFree(r->d_tables);
    delete r;
    return LBM_ERR_CUDA;
  }
  t.tab_t = r->d_tables;
  t.tab_h = r->d_tables + n_t;
  t.tab_w = r->d_tables + n_t + n_h;
  r->t = t;
  *out = r;
  return LBM_OK;
}

// Attention of block `block` of the pending frame, then its commit / rollback when it is the
// last block.  q_rot_out: where the kernel also writes the q it rotated (nullable; only when
// it rotates).  noalloc: partial results in the library's file-scope array instead of the
// cache's scratch (lbm_attend_frame_noalloc).
int attend(lbm_cache* c, int block, const void* q, void* out, void* q_rot_out, bool noalloc,
           void* stream) {
  if (!c || !q || !out || !aligned16(q) || !aligned16(out)) return LBM_ERR_INVALID;
  if (block < 0 || block >= (int)c->blocks.size()) return LBM_ERR_INVALID;
  if (block != c->next_block || !c->block_appended || !c->pager.awaiting_attention())
    return LBM_ERR_SEQUENCE;
  if (q_rot_out && (c->q_rotated || c->dtype != LBM_BF16)) return LBM_ERR_INVALID;
  const lbm::Pools& pl = c->blocks[block].pools;
  if (use_device(c->device) != LBM_OK) return LBM_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int T = c->psi + c->patches;
  if (c->dtype == LBM_BF16) {
    // nothing on this path touches the heap (the no-allocation call relies on it): the
    // parameter block (~7 KB) lives on the stack and the page list is read in place
    float* scratch = c->part_o;
    size_t scratch_floats = c->scratch_floats;
    if (noalloc) {
      const int st = lbm::noalloc_scratch(c->device, &scratch, &scratch_floats);
      if (st != LBM_OK) return st;
    }
    lbm::AttnParams p;
    const int st = fill_attn_params(c, block, q, out, q_rot_out, p);
    if (st != LBM_OK) return st;
    const long long units = (long long)p.n_pairs * c->heads;
    const bool split = lbm::sk_has_split(p);
    if (split && lbm::sk_scratch_floats(units, p.grid, c->head_dim) > scratch_floats)
      return LBM_ERR_CAPACITY;
    p.part_o = scratch;
    p.part_lse = noalloc ? scratch + (size_t)(units + p.grid) * 256 * c->head_dim : c->part_lse;
    order_before(c, s);
    if (lbm::launch_attn_tc(p, c->head_dim, s) != cudaSuccess) return LBM_ERR_CUDA;
    ++c->launches;
    if (split) {
      if (lbm::launch_attn_combine(p, c->head_dim, s) != cudaSuccess) return LBM_ERR_CUDA;
      ++c->launches;
    }
  } else {
    std::vector<int> pages;
    int n_sp = 0, last_len = 0;
    if (c->pager.visible(&pages, &n_sp, &last_len) != lbm::PagerStatus::kOk)
      return LBM_ERR_SEQUENCE;
    static thread_local lbm::SimtParams p;
    p.q = q;
    p.out = out;
    p.k_patch = pl.k_patch;
    p.v_patch = pl.v_patch;
    p.k_special = pl.k_special;
    p.v_special = pl.v_special;
    p.tokens = T;
    p.heads = c->heads;
    p.head_dim = c->head_dim;
    p.patches = c->patches;
    p.page_stride = pl.page_stride;
    p.pool_pages = pl.num_pages;
    p.spec_cap = pl.spec_cap;
    p.n_pages = (int)pages.size();
    p.n_special = n_sp;
    p.scale = (float)(1.0 / std::sqrt((double)c->head_dim));
    for (size_t i = 0; i < pages.size(); ++i) p.pages[i] = (uint16_t)pages[i];
    order_before(c, s);
    if (lbm::launch_attn_simt(p, s) != cudaSuccess) return LBM_ERR_CUDA;
    ++c->launches;
  }
  order_after(c, s);
  block_attended(c);
  return LBM_OK;
}

}  // namespace

extern "C" {

const char* lbm_status_string(int status) {
  switch (status) {
    case LBM_OK: return "ok";
    case LBM_ERR_INVALID: return "invalid argument";
    case LBM_ERR_UNSUPPORTED: return "unsupported configuration";
    case LBM_ERR_SEQUENCE: return "call out of sequence";
    case LBM_ERR_CAPACITY: return "capacity exceeded";
    case LBM_ERR_NOMEM: return "out of memory";
    case LBM_ERR_CUDA: return "CUDA error";
    case LBM_ERR_TIMEOUT: return "device wait timed out";
    default: return "unknown status";
  }
}

int lbm_rope3d_tables(int head_dim, int ppf, int pph, int ppw, int patch_start_idx,
                      double theta, lbm_rope_t** out) {
  return lbm_rope3d_tables_fhw(head_dim, 0, 0, 0, ppf, pph, ppw, patch_start_idx, theta, 1.0,
                               out);
}

int lbm_rope3d_tables_fhw(int head_dim, int dt, int dh, int dw, int ppf, int pph, int ppw,
                          int patch_start_idx, double theta, double ntk_factor,
                          lbm_rope_t** out) {
  if (!out) return LBM_ERR_INVALID;
  *out = nullptr;
  if (head_dim < 6 || head_dim % 2) return LBM_ERR_INVALID;
  if (dt == 0 && dh == 0 && dw == 0) {
    // default split: d_h = d_w = 2 * (head_dim / 6), d_t = the rest; pairs ordered t, h, w
    dh = dw = 2 * (head_dim / 6);
    dt = head_dim - 2 * dh;
  }
  if (dt < 2 || dh < 2 || dw < 2 || dt % 2 || dh % 2 || dw % 2 || dt + dh + dw != head_dim ||
      ppf < 1 || pph < 1 ||
      ppw < 1 || patch_start_idx < 0 || !(ntk_factor > 0.0) || !(theta * ntk_factor > 1.0) ||
      (long long)pph * ppw > (1 << 20) || ppf > (1 << 24))
    return LBM_ERR_INVALID;
  theta *= ntk_factor;  // [VideoRoPE] "NTK-Aware Frequency Scaling": theta * ntk_factor
  lbm::RopeTables t{};
  t.head_dim = head_dim;
  t.ppf = ppf;
  t.pph = pph;
  t.ppw = ppw;
  t.psi = patch_start_idx;
  return build_rope(t, {ppf, dt, theta}, {pph + 1, dh, theta}, {ppw + 1, dw, theta}, out);
}

int lbm_rope2d_tables(int head_dim, int ppf, int pph, int ppw, int patch_start_idx,
                      double frequency, lbm_rope_t** out) {
  if (!out) return LBM_ERR_INVALID;
  *out = nullptr;
  // two halves (y, x) of whole feature pairs: head_dim divisible by 4
  if (head_dim < 4 || head_dim % 4 || ppf < 1 || pph < 1 || ppw < 1 || patch_start_idx < 0 ||
      !(frequency > 1.0) || (long long)pph * ppw > (1 << 20) || ppf > (1 << 24))
    return LBM_ERR_INVALID;
  lbm::RopeTables t{};
  t.head_dim = head_dim;
  t.ppf = ppf;
  t.pph = pph;
  t.ppw = ppw;
  t.psi = patch_start_idx;
  // [RoPERange] "Deriving Size from Token Count": each half's table has one row per token of
  // a frame (positions 0 .. T-1), which covers the coordinates 0 .. max(pph, ppw) in use
  const int rows = patch_start_idx + pph * ppw;
  const int d_half = head_dim / 2;
  return build_rope(t, {0, 0, frequency}, {rows, d_half, frequency}, {rows, d_half, frequency},
                    out);
}

int lbm_rope3d_expand(const lbm_rope_t* rope, float* cos_out, float* sin_out, void* stream) {
  if (!rope || !cos_out || !sin_out) return LBM_ERR_INVALID;
  if (use_device(rope->device) != LBM_OK) return LBM_ERR_CUDA;
  return lbm::launch_rope_expand(rope->t, cos_out, sin_out, (cudaStream_t)stream) == cudaSuccess
             ? LBM_OK
             : LBM_ERR_CUDA;
}

void lbm_rope_destroy(lbm_rope_t* rope) {
  if (!rope) return;
  cudaFree(rope->d_tables);
  delete rope;
}

int lbm_cache_create(int heads, int head_dim, int patches_per_frame, int specials_per_frame,
                     int scale_frames, int sliding_window, int max_frames, int dtype,
                     const lbm_rope_t* rope, lbm_cache_t** out) {
  return lbm_cache_create_blocks(1, heads, head_dim, patches_per_frame, specials_per_frame,
                                 scale_frames, sliding_window, max_frames, dtype, rope, out);
}

int lbm_cache_create_blocks(int num_blocks, int heads, int head_dim, int patches_per_frame,
                            int specials_per_frame, int scale_frames, int sliding_window,
                            int max_frames, int dtype, const lbm_rope_t* rope,
                            lbm_cache_t** out) {
  if (!out) return LBM_ERR_INVALID;
  *out = nullptr;
  if (num_blocks < 1 || num_blocks > 1024) return LBM_ERR_INVALID;
  if (!rope || heads < 1 || heads > 65535 || patches_per_frame < 1 || scale_frames < 0 ||
      sliding_window < 0 || max_frames < 1 ||
      scale_frames + sliding_window + 1 > LBM_MAX_PAGES)
    return LBM_ERR_INVALID;
  if (dtype != LBM_BF16 && dtype != LBM_F32) return LBM_ERR_UNSUPPORTED;
  if (head_dim != 64 && head_dim != 128) return LBM_ERR_UNSUPPORTED;
  if (specials_per_frame != 6 || rope->t.psi != specials_per_frame ||
      rope->t.head_dim != head_dim || rope->t.pph * rope->t.ppw != patches_per_frame)
    return LBM_ERR_INVALID;

  auto* c = new (std::nothrow) lbm_cache(scale_frames, sliding_window, max_frames, 6);
  if (!c) return LBM_ERR_NOMEM;
  c->heads = heads;
  c->head_dim = head_dim;
  c->patches = patches_per_frame;
  c->psi = specials_per_frame;
  c->scale_frames = scale_frames;
  c->sliding_window = sliding_window;
  c->max_frames = max_frames;
  c->dtype = dtype;
  c->rope = rope;
  cudaGetDevice(&c->device);
  cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device);
  if (dtype == LBM_BF16) {
    // the bf16 attention is tcgen05 code built for sm_100a: it runs on compute capability
    // 10.0 only, with the dynamic shared memory of its larger (folded) instance
    int major = 0, minor = 0, optin = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, c->device);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, c->device);
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, c->device);
    const size_t need = std::max(lbm::attn_tc_smem_bytes(head_dim, false),
                                 lbm::attn_tc_smem_bytes(head_dim, true));
    if (major != 10 || minor != 0 || (size_t)optin < need) {
      cudaGetLastError();
      delete c;
      return LBM_ERR_UNSUPPORTED;
    }
  }
  if (const char* env = std::getenv("LBM_ATTN_GRID")) {
    const int v = std::atoi(env);
    if (v >= 1 && v <= 4 * c->num_sms && v <= lbm::kMaxGrid) c->forced_grid = v;
  }

  const int P = scale_frames + sliding_window + 1;
  const int stride = (patches_per_frame + kKeyTile - 1) / kKeyTile * kKeyTile;
  const long long cap = (6LL * (max_frames + 1) + 127) / 128 * 128;
  const int e = elem_size(dtype);
  const size_t patch_bytes = (size_t)heads * P * stride * head_dim * e;
  const size_t spec_bytes = (size_t)heads * cap * head_dim * e;
  const size_t per_block = 2 * patch_bytes + 2 * spec_bytes;
  const size_t total = per_block * (size_t)num_blocks;
  const int T = specials_per_frame + patches_per_frame;
  // partial results: (units + persistent CTAs) slots of 256 rows x (head_dim + 1) floats
  const long long units = (long long)(((T + 127) / 128 + 1) / 2) * heads;
  const int grid_max = c->forced_grid ? c->forced_grid : c->num_sms;
  c->scratch_floats = lbm::sk_scratch_floats(units, grid_max, head_dim);
  const size_t part_o_bytes = (size_t)(units + grid_max) * 256 * head_dim * sizeof(float);
  const size_t part_lse_bytes = (size_t)(units + grid_max) * 256 * sizeof(float);
  auto fail = [&](int st) {
    cudaFree(c->pool_mem);
    cudaFree(c->part_o);
    cudaFree(c->part_lse);
    cudaFree(c->d_err);
    if (c->ev) cudaEventDestroy(c->ev);
    cudaGetLastError();
    delete c;
    return st;
  };
  if (cap > (1LL << 31) / 2) return fail(LBM_ERR_INVALID);
  if (cudaMalloc(&c->pool_mem, total) != cudaSuccess) return fail(LBM_ERR_NOMEM);
  if (cudaMemset(c->pool_mem, 0, total) != cudaSuccess) return fail(LBM_ERR_CUDA);
  if (dtype == LBM_BF16) {
    if (cudaMalloc(&c->part_o, part_o_bytes) != cudaSuccess ||
        cudaMalloc(&c->part_lse, part_lse_bytes) != cudaSuccess)
      return fail(LBM_ERR_NOMEM);
  }
  if (cudaMalloc(&c->d_err, sizeof(int)) != cudaSuccess) return fail(LBM_ERR_NOMEM);
  if (cudaMemset(c->d_err, 0, sizeof(int)) != cudaSuccess) return fail(LBM_ERR_CUDA);
  if (cudaEventCreateWithFlags(&c->ev, cudaEventDisableTiming) != cudaSuccess)
    return fail(LBM_ERR_CUDA);
  c->blocks.resize(num_blocks);
  for (int b = 0; b < num_blocks; ++b) {
    char* base = static_cast<char*>(c->pool_mem) + per_block * (size_t)b;
    lbm::Pools& pl = c->blocks[b].pools;
    pl.k_patch = base;
    pl.v_patch = base + patch_bytes;
    pl.k_special = base + 2 * patch_bytes;
    pl.v_special = base + 2 * patch_bytes + spec_bytes;
    pl.num_pages = P;
    pl.page_stride = stride;
    pl.spec_cap = (int)cap;
  }
  c->device_bytes = (long long)(total + (dtype == LBM_BF16 ? part_o_bytes + part_lse_bytes : 0) +
                                sizeof(int));
  if (dtype == LBM_BF16) {
    const uint64_t row = (uint64_t)head_dim * 2;
    const uint64_t prow = (uint64_t)P * stride;
    const uint32_t kt = (uint32_t)lbm::attn_key_tile(head_dim);  // tensor-map box rows
    for (CacheBlock& bk : c->blocks) {
      const lbm::Pools& pl = bk.pools;
      if (!make_map(&bk.tm_kp, pl.k_patch, head_dim, prow, heads, row, prow * row, kt, 1) ||
          !make_map(&bk.tm_vp, pl.v_patch, head_dim, prow, heads, row, prow * row, kt, 1) ||
          !make_map(&bk.tm_ks, pl.k_special, head_dim, cap, heads, row, cap * row, kt, 1) ||
          !make_map(&bk.tm_vs, pl.v_special, head_dim, cap, heads, row, cap * row, kt, 1))
        return fail(LBM_ERR_CUDA);
    }
  }
  if (cudaDeviceSynchronize() != cudaSuccess) return fail(LBM_ERR_CUDA);
  *out = c;
  return LBM_OK;
}

int lbm_append_frame(lbm_cache_t* c, void* q, const void* k, const void* v, long long frame_idx,
                     int is_keyframe, void* stream) {
  if (!c) return LBM_ERR_INVALID;
  return lbm_append_frame_block(c, c->next_block, q, k, v, frame_idx, is_keyframe, stream);
}

int lbm_append_frame_block(lbm_cache_t* c, int block, void* q, const void* k, const void* v,
                           long long frame_idx, int is_keyframe, void* stream) {
  if (!c || !k || !v || !aligned16(q) || !aligned16(k) || !aligned16(v))
    return LBM_ERR_INVALID;
  // q = NULL leaves the rotation of q to the attention kernel (tensor-core path only)
  if (!q && c->dtype != LBM_BF16) return LBM_ERR_UNSUPPORTED;
  if (is_keyframe < 0 || is_keyframe > LBM_KEYFRAME_DEFERRED) return LBM_ERR_INVALID;
  if (block < 0 || block >= (int)c->blocks.size()) return LBM_ERR_INVALID;
  if (block != c->next_block || c->block_appended) return LBM_ERR_SEQUENCE;
  if (frame_idx < 0 || frame_idx >= c->rope->t.ppf) return LBM_ERR_SEQUENCE;
  int page = -1, slot = -1;
  if (block == 0) {
    switch (c->pager.peek_append(frame_idx, is_keyframe, &page, &slot)) {
      case lbm::PagerStatus::kOk: break;
      case lbm::PagerStatus::kSequence: return LBM_ERR_SEQUENCE;
      case lbm::PagerStatus::kCapacity: return LBM_ERR_CAPACITY;
    }
  } else {
    // a later block writes the same frame into its own pools, at the page and special
    // slots block 0 took
    if (!c->pager.pending() || frame_idx != c->pager.pending_frame()) return LBM_ERR_SEQUENCE;
    if (is_keyframe != c->frame_mode) return LBM_ERR_INVALID;
    page = c->pager.pending_page();
    slot = c->pager.n_special();
  }
  if (use_device(c->device) != LBM_OK) return LBM_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  lbm::AppendArgs a{};
  a.dtype = c->dtype;
  a.heads = c->heads;
  a.head_dim = c->head_dim;
  a.tokens = c->psi + c->patches;
  a.psi = c->psi;
  a.frame = (int)frame_idx;
  a.page = page;
  a.special_slot = slot;
  a.q = q;
  a.k = k;
  a.v = v;
  order_before(c, s);
  if (lbm::launch_rope_append(c->rope->t, c->blocks[block].pools, a, s) != cudaSuccess)
    return LBM_ERR_CUDA;
  ++c->launches;
  order_after(c, s);
  if (block == 0) {
    c->pager.append(frame_idx, is_keyframe, &page, &slot);
    c->frame_mode = is_keyframe;
  }
  c->block_appended = true;
  c->q_rotated = q != nullptr;
  return LBM_OK;
}

int lbm_commit_frame(lbm_cache_t* c, int keep) {
  if (!c) return LBM_ERR_INVALID;
  int evicted = -1;
  switch (c->pager.commit(keep != 0, &evicted)) {
    case lbm::PagerStatus::kOk: return LBM_OK;
    case lbm::PagerStatus::kSequence: return LBM_ERR_SEQUENCE;
    case lbm::PagerStatus::kCapacity: return LBM_ERR_CAPACITY;
  }
  return LBM_ERR_INVALID;
}

int lbm_attend_frame(lbm_cache_t* c, const void* q, void* out, void* stream) {
  if (!c) return LBM_ERR_INVALID;
  return attend(c, c->next_block, q, out, nullptr, false, stream);
}

int lbm_attend_frame_block(lbm_cache_t* c, int block, const void* q, void* out, void* stream) {
  return attend(c, block, q, out, nullptr, false, stream);
}

int lbm_attend_frame_qrot(lbm_cache_t* c, const void* q, void* out, void* q_rot_out,
                          void* stream) {
  if (!c) return LBM_ERR_INVALID;
  if (!q_rot_out || !aligned16(q_rot_out)) return LBM_ERR_INVALID;
  return attend(c, c->next_block, q, out, q_rot_out, false, stream);
}

int lbm_attend_frame_noalloc(lbm_cache_t* c, const void* q, void* out, void* stream) {
  if (!c) return LBM_ERR_INVALID;
  if (c->dtype != LBM_BF16) return LBM_ERR_UNSUPPORTED;
  return attend(c, c->next_block, q, out, nullptr, true, stream);
}

int lbm_cache_reset(lbm_cache_t* c) {
  if (!c) return LBM_ERR_INVALID;
  c->pager.reset();
  c->next_block = 0;
  c->block_appended = false;
  return LBM_OK;
}

int lbm_cache_state(const lbm_cache_t* c, lbm_cache_state_t* st) {
  if (!c || !st) return LBM_ERR_INVALID;
  st->device_bytes = c->device_bytes;
  st->kernel_launches = c->launches;
  return lbm::fill_state(c->pager, st);
}

int lbm_cache_read_kv(const lbm_cache_t* c, int which, int index, int count, void* host_out) {
  return lbm_cache_read_kv_block(c, 0, which, index, count, host_out);
}

int lbm_cache_read_kv_block(const lbm_cache_t* c, int block, int which, int index, int count,
                            void* host_out) {
  if (!c || !host_out || block < 0 || block >= (int)c->blocks.size()) return LBM_ERR_INVALID;
  const lbm::Pools& pl = c->blocks[block].pools;
  const int e = elem_size(c->dtype);
  const size_t row = (size_t)c->head_dim * e;
  const void* src;
  size_t pitch, width;
  if (which == LBM_K_PATCH || which == LBM_V_PATCH) {
    if (index < 0 || index >= pl.num_pages) return LBM_ERR_INVALID;
    const char* pool = static_cast<const char*>(which == LBM_K_PATCH ? pl.k_patch
                                                                     : pl.v_patch);
    src = pool + (size_t)index * pl.page_stride * row;
    pitch = (size_t)pl.num_pages * pl.page_stride * row;
    width = (size_t)c->patches * row;
  } else if (which == LBM_K_SPECIAL || which == LBM_V_SPECIAL) {
    if (index < 0 || count < 1 || index + count > pl.spec_cap) return LBM_ERR_INVALID;
    const char* pool = static_cast<const char*>(which == LBM_K_SPECIAL ? pl.k_special
                                                                       : pl.v_special);
    src = pool + (size_t)index * row;
    pitch = (size_t)pl.spec_cap * row;
    width = (size_t)count * row;
  } else {
    return LBM_ERR_INVALID;
  }
  if (use_device(c->device) != LBM_OK) return LBM_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return LBM_ERR_CUDA;
  if (cudaMemcpy2D(host_out, width, src, pitch, width, c->heads, cudaMemcpyDeviceToHost) !=
      cudaSuccess)
    return LBM_ERR_CUDA;
  return LBM_OK;
}

int lbm_cache_set_wait_limit(lbm_cache_t* c, unsigned long long ns) {
  if (!c || ns > kDefaultWaitLimitNs) return LBM_ERR_INVALID;
  c->wait_limit_ns = ns == 0 ? kDefaultWaitLimitNs : ns;
  return LBM_OK;
}

int lbm_cache_check(lbm_cache_t* c) {
  if (!c) return LBM_ERR_INVALID;
  if (use_device(c->device) != LBM_OK) return LBM_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return LBM_ERR_CUDA;
  int err = 0;
  if (cudaMemcpy(&err, c->d_err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return LBM_ERR_CUDA;
  if (err != 0) {
    cudaMemset(c->d_err, 0, sizeof(int));
    return LBM_ERR_TIMEOUT;
  }
  return LBM_OK;
}

void lbm_cache_destroy(lbm_cache_t* c) {
  if (!c) return;
  use_device(c->device);
  cudaDeviceSynchronize();
  cudaFree(c->pool_mem);
  cudaFree(c->part_o);
  cudaFree(c->part_lse);
  cudaFree(c->d_err);
  if (c->ev) cudaEventDestroy(c->ev);
  delete c;
}

}  // extern "C"
