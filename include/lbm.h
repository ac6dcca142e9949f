/*
 * lbm.h - C ABI of the streaming-frame step: 3D RoPE, dual-stream paged KV cache, paged
 * attention, for one NVIDIA B200 (sm_100a).
 *
 * The operations follow five articles about the lingbot-map project, cited by title and
 * section:
 *   [3DRoPE-KV]  "How 3D RoPE Positional Encoding Works with the Paged KV Cache in
 *                 LingBot-Map"
 *   [VideoRoPE]  "Video RoPE Positional Encoding: 3D Rotary Embeddings for Long-Sequence
 *                 Video in Ling-Bot-Map"
 *   [RealTime3D] "How LingBot-Map Achieves Real-Time 3D Reconstruction: Streaming
 *                 Transformers and KV Caching"
 *   [KVBenefits] "KV Caching Benefits in Ling Bot-Map: 7 Advantages for Streaming Vision
 *                 Models"
 *   [RoPERange]  "How to Handle Sequences Exceeding the RoPE Training Range in LingBot-Map"
 *
 * Conventions common to every call
 * --------------------------------
 *  - Every call returns an lbm status (LBM_OK == 0, errors < 0).  Nothing throws or aborts
 *    across the ABI.  A call that fails leaves the library state as it was.
 *  - q, k, v and out are DEVICE pointers owned by the caller, contiguous [T][heads][head_dim]
 *    (token-major), T = specials_per_frame + patches_per_frame, 16-byte aligned, element type
 *    the cache's dtype (LBM_F32: float, LBM_BF16: bfloat16).
 *  - stream is a cudaStream_t (NULL = the legacy default stream).  Work is only enqueued;
 *    nothing synchronises the host except the calls that say so.  Calls on one cache from
 *    several streams are ordered by the library through an event it records after each launch.
 *  - The library owns the RoPE tables, the K/V page pools, stream-K scratch and the page
 *    table.  The caller owns its q/k/v/out buffers and the streams.
 *  - Host bookkeeping (page table, free list, deferred eviction) runs at call time on the
 *    host; the only host->device traffic of a frame is kernel launch parameters.
 */
#ifndef LBM_H
#define LBM_H

#if defined(__GNUC__)
#define LBM_API __attribute__((visibility("default")))
#else
#define LBM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---------------------------------------------------------------------- */
enum {
  LBM_OK = 0,
  LBM_ERR_INVALID = -1,      /* bad argument: null/misaligned pointer, size out of range    */
  LBM_ERR_UNSUPPORTED = -2,  /* valid but not implemented (head_dim not 64/128, dtype)        */
  LBM_ERR_SEQUENCE = -3,     /* call out of order (append twice, attend first, frame order)  */
  LBM_ERR_CAPACITY = -4,     /* special stream full: max_frames keyframes already committed  */
  LBM_ERR_NOMEM = -5,        /* device or host allocation failed                             */
  LBM_ERR_CUDA = -6,         /* a CUDA runtime / driver call or kernel launch failed         */
  LBM_ERR_TIMEOUT = -7       /* a kernel gave up a bounded wait and flagged an error         */
};

enum { LBM_F32 = 0, LBM_BF16 = 1 };

/* which pool lbm_cache_read_kv copies */
enum { LBM_K_PATCH = 0, LBM_V_PATCH = 1, LBM_K_SPECIAL = 2, LBM_V_SPECIAL = 3 };

/* Tokens per page of the special stream.  [3DRoPE-KV] "Attention Computation with Cached
 * RoPE" passes the valid length of the last, partly filled special page; the pages give no
 * page size, this library uses the attention tile height. */
#define LBM_SPECIAL_PAGE 128
/* Most patch pages one frame can see (scale_frames + sliding_window + 1). */
#define LBM_MAX_PAGES 1024

typedef struct lbm_rope lbm_rope_t;
typedef struct lbm_cache lbm_cache_t;
typedef struct lbm_pager lbm_pager_t;

/* ---- 3D RoPE tables ---------------------------------------------------------------------
 * [3DRoPE-KV] "Multi-Axis Frequency Generation"; [VideoRoPE] "The Three Rotary Dimensions".
 * One 1D table per axis a in (t, h, w): angle(p, i) = p * theta^(-2i/d_a), i < d_a/2, with
 * d_h = d_w = 2*(head_dim/6) and d_t = head_dim - 2*d_h; pairs ordered t, h, w along
 * head_dim/2.  Angles and cos/sin are computed in double on the host and rounded once to
 * float.  Rows: t in [0, ppf), h in [0, pph], w in [0, ppw].  Token j of frame t sits at
 * (t, 0, 0) for j < patch_start_idx (special tokens) and at (t, 1 + r, 1 + c) for patch
 * (r, c) = divmod(j - patch_start_idx, ppw).  Feature pair i is (x[2i], x[2i+1]).
 *   head_dim       64 or 128 (any even value >= 6 is accepted here; caches take 64/128)
 *   ppf            frames covered by the t table (frame_idx must stay below it)
 *   pph, ppw       patch grid of a frame
 *   patch_start_idx special tokens before the patches of each frame (6)
 *   theta          base (10000.0); NTK scaling is theta * ntk_factor, passed pre-multiplied
 *   out            receives the table object; the caller frees it with lbm_rope_destroy
 *                  after every cache that uses it is destroyed.
 * Allocates device memory on the current device; synchronous. */
LBM_API int lbm_rope3d_tables(int head_dim, int ppf, int pph, int ppw, int patch_start_idx,
                      double theta, lbm_rope_t** out);

/* The same tables with an explicit (t, h, w) split of head_dim = d_t + d_h + d_w (the pages'
 * fhw_dim, e.g. [20, 22, 22] for head_dim 64 in [3DRoPE-KV] "Implementation Example" and
 * [40, 44, 44] for 128 in [VideoRoPE] "Enabling 3D RoPE for Video Heads") and an NTK factor
 * that multiplies theta ([VideoRoPE] "NTK-Aware Frequency Scaling").
 *   head_dim       even, >= 6
 *   d_t, d_h, d_w  each even and >= 2, summing to head_dim; or all three 0 for the default
 *                  split of lbm_rope3d_tables (d_h = d_w = 2*(head_dim/6), d_t = the rest)
 *   ntk_factor     > 0, with theta * ntk_factor > 1
 * Otherwise LBM_ERR_INVALID.  lbm_rope3d_tables is this call with the default split and
 * ntk_factor 1.  Allocates device memory on the current device; synchronous. */
LBM_API int lbm_rope3d_tables_fhw(int head_dim, int d_t, int d_h, int d_w, int ppf, int pph,
                                  int ppw, int patch_start_idx, double theta, double ntk_factor,
                                  lbm_rope_t** out);

/* The 2D (y, x) variant of [RoPERange] "How to Handle Sequences Exceeding the RoPE Training
 * Range in LingBot-Map", sections "Spatial Position Encoding" and "Dynamic Frequency Caching
 * for Arbitrary Sequence Lengths": the features split into two halves of head_dim/2, the
 * first rotated by a 1D rotary embedding of the row y, the second by one of the column x,
 * angle(p, i) = p * frequency^(-2i/(head_dim/2)), i < head_dim/4, frequency 100.0 on the
 * page; each half's table has one row per token of a frame (sized from the token count, not
 * from the largest coordinate).  Token j of a frame sits at (0, 0) for j < patch_start_idx and
 * at (1 + r, 1 + c) for patch (r, c); the frame index plays no part in the rotation (frames
 * are still told apart by the cache).  Feature pair i is (x[2i], x[2i+1]); pairs
 * [0, head_dim/4) take y, the rest x.  The page's scaling_factor (1.0, undefined there) is not
 * modelled.
 *   head_dim       a multiple of 4 (caches take 64 / 128)
 *   ppf            frames a cache using these tables may stream (frame_idx < ppf)
 *   pph, ppw, patch_start_idx   as for lbm_rope3d_tables
 *   frequency      > 1
 * The result is used exactly like a 3D table object (caches, lbm_rope3d_expand,
 * lbm_rope_destroy).  LBM_ERR_INVALID for bad sizes.  Allocates device memory on the
 * current device; synchronous. */
LBM_API int lbm_rope2d_tables(int head_dim, int ppf, int pph, int ppw, int patch_start_idx,
                              double frequency, lbm_rope_t** out);

/* Writes the expanded table of [3DRoPE-KV] "Multi-Axis Frequency Generation" (the one the
 * page prints as [ppf * (patch_start_idx + pph*ppw)][head_dim/2]), for parity checks of the
 * tables a rope object holds.
 *   rope            from lbm_rope3d_tables / lbm_rope3d_tables_fhw / lbm_rope2d_tables
 *   cos_out, sin_out  DEVICE pointers, caller-owned, float [ppf * (patch_start_idx +
 *                  pph*ppw)][head_dim/2] each: row = frame * tokens_per_frame + token, frames
 *                  0..ppf-1 in order, a frame's tokens in the order above (specials, then
 *                  patches row-major); column = feature pair
 *   stream          cudaStream_t the kernel is enqueued on (nothing waits for it)
 * LBM_ERR_INVALID for a null argument, LBM_ERR_CUDA if the launch fails. */
LBM_API int lbm_rope3d_expand(const lbm_rope_t* rope, float* cos_out, float* sin_out, void* stream);

LBM_API void lbm_rope_destroy(lbm_rope_t* rope);

/* ---- the dual-stream paged KV cache -----------------------------------------------------
 * [3DRoPE-KV] "Dual-Stream Memory Layout": the patch stream keeps one page of
 * patches_per_frame tokens per frame; the first scale_frames keyframes' pages stay, the next
 * sliding_window pages are recycled, the oldest window page returns to a free list when the
 * window overflows (after the attention of the frame that overflows it: deferred eviction).
 * The special stream is append-only, specials_per_frame tokens per committed keyframe.
 *   heads, head_dim    head_dim 64 or 128 (else LBM_ERR_UNSUPPORTED)
 *   patches_per_frame  must equal rope's pph*ppw
 *   specials_per_frame must equal rope's patch_start_idx and be 6
 *   scale_frames, sliding_window  >= 0; scale_frames + sliding_window + 1 <= LBM_MAX_PAGES
 *   max_frames         keyframes the special stream can hold (>= 1)
 *   dtype              LBM_BF16 (tensor-core path) or LBM_F32 (exact SIMT path); a bf16
 *                      cache needs a compute capability 10.0 device (B200) with the
 *                      attention kernel's shared memory, else LBM_ERR_UNSUPPORTED
 *   rope               tables built for the same head_dim / grid; must outlive the cache
 * Device memory: K and V patch pools [heads][P*stride][head_dim] with P = scale_frames +
 * sliding_window + 1 pages and stride = patches_per_frame rounded up to 128 (zero-filled);
 * K and V special pools [heads][cap][head_dim], cap = 6*(max_frames+1) rounded up to 128;
 * stream-K scratch: partial results of (units + persistent CTAs) x 256 rows x (head_dim + 1)
 * floats, a unit being one (pair of 128-row query tiles, head).  Synchronous. */
LBM_API int lbm_cache_create(int heads, int head_dim, int patches_per_frame, int specials_per_frame,
                     int scale_frames, int sliding_window, int max_frames, int dtype,
                     const lbm_rope_t* rope, lbm_cache_t** out);

/* A cache for num_blocks transformer blocks (1..1024) that share one page table
 * ([3DRoPE-KV] "Implementation Example": the cache manager is created for num_blocks blocks,
 * and appending and attention take a block_idx).  Every block has its own K/V pools (the
 * sizes of lbm_cache_create, times num_blocks) and tensor maps; the page table, free list and
 * special-stream count are shared, since every block sees the same frames.  A frame visits
 * the blocks in order: for b = 0 .. num_blocks-1, append (block b) then attend (block b).
 * Block 0's append takes the frame's page and special slots, later blocks write theirs at the
 * same places, and the frame is committed or rolled back after the last block's attention.
 * lbm_cache_create is num_blocks = 1; lbm_append_frame / lbm_attend_frame act on the next
 * block in that order.  Synchronous. */
LBM_API int lbm_cache_create_blocks(int num_blocks, int heads, int head_dim,
                                    int patches_per_frame, int specials_per_frame,
                                    int scale_frames, int sliding_window, int max_frames,
                                    int dtype, const lbm_rope_t* rope, lbm_cache_t** out);

/* Rotate and append one frame.  [3DRoPE-KV] "Frame Appending and Position Encoding
 * Integration" and "Complex-Valued Tensor Application"; [VideoRoPE] "Temporal Consistency
 * in KV-Cache Streaming" (t = absolute frame index).
 *   q      device, [T][heads][head_dim], or NULL.  Non-NULL: rotated IN PLACE by this call
 *          (read, rotated, written back), and the attention then uses it as it is.  NULL
 *          (bf16 caches only, else LBM_ERR_UNSUPPORTED): the rotation of q is folded into
 *          the attention, which rotates the raw q as it loads it ([3DRoPE-KV] FAQ "Where does
 *          the RoPE application occur relative to the KV cache write?": q is rotated before
 *          the attention, k before the cache write) and leaves q unchanged; this call then
 *          moves only k and v (4 instead of 6 x T x heads x head_dim elements).
 *   k, v   device, [T][heads][head_dim]; k is rotated, v is not; both are written into the
 *          frame's patch page (tokens >= 6) and the next 6 slots of the special stream
 *   frame_idx    strictly greater than the previous frame's, and < rope's ppf
 *   is_keyframe  1: the frame is kept after its attention; 0: rolled back after it
 *                ([KVBenefits] "Reduced KV Growth via Keyframe Streaming");
 *                LBM_KEYFRAME_DEFERRED: decided after the attention by lbm_commit_frame
 *                ([KVBenefits] "Dynamic Keyframe Selection": selection by what the frame
 *                shows); other values: LBM_ERR_INVALID
 * One kernel launch.  Errors: LBM_ERR_SEQUENCE if a frame is already pending or frame_idx
 * does not increase or is >= ppf; LBM_ERR_CAPACITY for a keyframe when max_frames keyframes
 * are committed. */
#define LBM_KEYFRAME_DEFERRED 2
LBM_API int lbm_append_frame(lbm_cache_t* cache, void* q, const void* k, const void* v,
                     long long frame_idx, int is_keyframe, void* stream);
/* The same for block block_idx of a multi-block cache.  Errors: LBM_ERR_INVALID for a block
 * out of range or (blocks > 0) an is_keyframe different from block 0's; LBM_ERR_SEQUENCE
 * unless block_idx is the next block of the frame in flight (block 0: no frame in flight;
 * later blocks: the previous block has attended) and, for blocks > 0, frame_idx is that
 * frame's. */
LBM_API int lbm_append_frame_block(lbm_cache_t* cache, int block_idx, void* q, const void* k,
                                   const void* v, long long frame_idx, int is_keyframe,
                                   void* stream);

/* Attention of the pending frame's queries over what the cache retains: scale pages ->
 * window pages (oldest first) -> the frame's own page -> all special tokens ([3DRoPE-KV]
 * "Attention Computation with Cached RoPE"); a frame's own tokens all see each other; softmax
 * scale 1/sqrt(head_dim).  Then commits the frame (keyframe; deferred eviction) or rolls it
 * back ([KVBenefits] "Dynamic Keyframe Selection"); a frame appended with
 * LBM_KEYFRAME_DEFERRED stays pending until lbm_commit_frame.
 *   q    device [T][heads][head_dim]: the q lbm_append_frame rotated, or, when the append
 *        was given q = NULL, the raw q, which the kernel rotates as it loads it (q is not
 *        written)
 *   out  device [T][heads][head_dim], written
 * bf16: one tcgen05 kernel launch, plus one combine launch when the keys are split across
 * CTAs.  Errors: LBM_ERR_SEQUENCE if no frame is pending or the pending frame has already
 * been attended. */
LBM_API int lbm_attend_frame(lbm_cache_t* cache, const void* q, void* out, void* stream);
/* As lbm_attend_frame for a frame whose append left q to the attention (q = NULL there),
 * and the kernel also writes the rotated q it used, rounded to bf16, into q_rot_out (device
 * [T][heads][head_dim], caller-owned): what lbm_append_frame would have written into q in
 * place.  For checks of the folded rotation.  LBM_ERR_INVALID if q_rot_out is NULL or
 * misaligned, or the frame's q was rotated by its append, or the cache is not bf16. */
LBM_API int lbm_attend_frame_qrot(lbm_cache_t* cache, const void* q, void* out, void* q_rot_out,
                                  void* stream);
/* The same for block block_idx (LBM_ERR_SEQUENCE unless it has just appended). */
LBM_API int lbm_attend_frame_block(lbm_cache_t* cache, int block_idx, const void* q, void* out,
                                   void* stream);

/* Keep (keep != 0) or drop the pending frame appended with LBM_KEYFRAME_DEFERRED, after its
 * attention ([KVBenefits] "Dynamic Keyframe Selection": a kept frame triggers the deferred
 * eviction, a dropped frame's tentative entry is rolled back).  The resulting page table is
 * the one an up-front is_keyframe = keep would have given.  Host-only; no GPU work.
 * Errors: LBM_ERR_SEQUENCE unless such a frame is pending and attended; LBM_ERR_CAPACITY
 * when keep and max_frames keyframes are committed (the frame stays pending: drop it). */
LBM_API int lbm_commit_frame(lbm_cache_t* cache, int keep);

/* Like lbm_attend_frame, for callers that may not allocate device memory while frames
 * stream (a runtime that owns the whole GPU through its own pool and budget, or a real-time
 * loop where cudaMalloc / cudaFree would synchronise the device).  The pages describe no such
 * call; it has no counterpart there.  Same arguments, same result and same page-table update
 * as lbm_attend_frame, but the stream-K partial results go to a file-scope device array of
 * LBM_NOALLOC_SCRATCH_BYTES (16 MiB) that every GPU loading the library holds until exit,
 * instead of the cache's own scratch; the call allocates nothing (device or host heap).
 *   - bf16 caches only (LBM_ERR_UNSUPPORTED otherwise).
 *   - The first call on a device looks up the array's device address with that device
 *     current; make that first call before any stream capture.  Host threads may make their
 *     first calls at the same time (the lookup is guarded), but calls on one cache must not
 *     run concurrently, as for every call on a cache.
 *   - With one CTA per SM (148 on a B200): a head_dim 64 frame fits while units + 148 <= 252
 *     (16 heads: up to 12 query tiles, 1536 tokens); a head_dim 128 frame whose keys are
 *     split needs at least 149 x 256 x 129 x 4 bytes (19.5 MB) and is always refused.
 *   - A frame whose units are shared by CTAs and whose partial results need more than
 *     LBM_NOALLOC_SCRATCH_BYTES ((units + CTAs) x 256 x (head_dim + 1) x 4 bytes) is refused
 *     with LBM_ERR_CAPACITY and the cache is left as it was.
 *   - Every call shares the array and leaves its last contents there; nothing in it needs
 *     to start at zero.  Calls whose kernels overlap on the GPU (several streams or caches
 *     at once) race on it: order them. */
#define LBM_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
LBM_API int lbm_attend_frame_noalloc(lbm_cache_t* cache, const void* q, void* out,
                                     void* stream);

/* Forget every frame: all pages free, special stream empty ([KVBenefits] "Cross-Window
 * Alignment for Long Videos": clean_kv_cache).  Host-only; pool contents are left as they
 * are (nothing reads them before they are written again). */
LBM_API int lbm_cache_reset(lbm_cache_t* cache);

/* Host snapshot of the page table, for tests and monitoring ([KVBenefits] "Working with
 * the KV Cache API": get_kv_cache_info).  The caller sets capacity and the five array
 * pointers (each with room for capacity entries, or NULL to skip); counts are always set. */
typedef struct {
  int num_pages;          /* P = scale_frames + sliding_window + 1                          */
  int n_scale;            /* scale pages held                                                */
  int n_window;           /* window pages held                                               */
  int n_free;             /* pages on the free stack                                         */
  int n_special;          /* committed special tokens                                        */
  int special_pages;      /* ceil(n_special / LBM_SPECIAL_PAGE)                              */
  int last_page_len;      /* valid tokens in the last committed special page (0 if none)    */
  int pending;            /* 1 between lbm_append_frame and lbm_attend_frame                 */
  int pending_page;       /* page of the pending frame (-1 if none)                         */
  int pending_is_keyframe;
  long long pending_frame;
  long long last_frame;   /* last appended frame_idx, -1 if none                             */
  long long device_bytes; /* pool + scratch bytes held on the device                         */
  long long kernel_launches; /* kernels this cache has launched since it was created         */
  int capacity;           /* in: entries each array below can take                           */
  int* scale_pages;       /* out: scale pages in commit order                                */
  long long* scale_frames;
  int* window_pages;      /* out: window pages oldest first                                  */
  long long* window_frames;
  int* free_pages;        /* out: free stack bottom .. top (top is popped next)              */
} lbm_cache_state_t;

LBM_API int lbm_cache_state(const lbm_cache_t* cache, lbm_cache_state_t* state);

/* Copies part of a pool to host memory (synchronises the device; for tests).
 *   which  LBM_K_PATCH / LBM_V_PATCH: index = page id, count ignored; host_out receives
 *          [heads][patches_per_frame][head_dim]
 *          LBM_K_SPECIAL / LBM_V_SPECIAL: tokens [index, index+count) of the special
 *          stream; host_out receives [heads][count][head_dim]
 * Elements are the cache's dtype. */
LBM_API int lbm_cache_read_kv(const lbm_cache_t* cache, int which, int index, int count,
                      void* host_out);
/* The same for block block_idx (lbm_cache_read_kv reads block 0). */
LBM_API int lbm_cache_read_kv_block(const lbm_cache_t* cache, int block_idx, int which,
                                    int index, int count, void* host_out);

/* Synchronises the device and reports a bounded wait that ran out in an earlier kernel
 * (LBM_ERR_TIMEOUT, after which the error word is cleared) or LBM_OK. */
LBM_API int lbm_cache_check(lbm_cache_t* cache);

/* Time limit of each wait inside the attention kernel's roles (the producer waiting for a
 * free ring stage, the MMA issuers for loaded tiles and softmax results, the softmax threads
 * for scores), in nanoseconds of %globaltimer: a wait that runs out sets the device error
 * word and makes every role of the CTA leave; lbm_cache_check then reports LBM_ERR_TIMEOUT
 * and the frame's output is not valid.  The waits at the kernel's exit, for copies and
 * tensor-core operations already issued, keep their own 2 s bound, so nothing is left in
 * flight when the tensor memory is freed.  Below 1000 ns a wait that is not satisfied at its
 * first test runs out at once (a waiting thread may sleep longer than that inside one test,
 * so shorter limits are not honoured literally): the way to exercise the failure path.
 * ns = 0 restores the default, 2 s (2e9); values above it are LBM_ERR_INVALID.  Host-only;
 * applies to attention calls made after it. */
LBM_API int lbm_cache_set_wait_limit(lbm_cache_t* cache, unsigned long long ns);

LBM_API void lbm_cache_destroy(lbm_cache_t* cache);

LBM_API const char* lbm_status_string(int status);

/* ---- host-only page manager -------------------------------------------------------------
 * The page table / free list / deferred-eviction state machine the cache drives, exposed on
 * its own so that it can be checked without a GPU.  Same rules as the cache:
 * [3DRoPE-KV] "Dual-Stream Memory Layout"; [KVBenefits] "Dynamic Keyframe Selection".
 * A fresh manager pops pages 0, 1, ..., P-1; evicted and rolled-back pages are pushed on
 * top of the free stack (LIFO). */
LBM_API int lbm_pager_create(int scale_frames, int sliding_window, int max_frames,
                     int specials_per_frame, lbm_pager_t** out);
/* Pops the frame's page and reserves its special slots; *page and *special_slot receive them. */
LBM_API int lbm_pager_append(lbm_pager_t* pager, long long frame_idx, int is_keyframe, int* page,
                     int* special_slot);
/* The pending frame's visible patch pages (scale, window oldest first, own page) into
 * pages[0..capacity), their count, and the visible special tokens (committed + own). */
LBM_API int lbm_pager_visible(const lbm_pager_t* pager, int* pages, int capacity, int* n_pages,
                      int* n_special, int* last_page_len);
/* The pending frame's attention is done: commit (keyframe) or roll back (non-keyframe) it;
 * *evicted receives the page returned to the free list by deferred eviction, or -1.  A frame
 * appended with LBM_KEYFRAME_DEFERRED only becomes attended (*evicted = -1). */
LBM_API int lbm_pager_finish(lbm_pager_t* pager, int* evicted);
/* Keep or drop an attended LBM_KEYFRAME_DEFERRED frame, as lbm_commit_frame. */
LBM_API int lbm_pager_commit(lbm_pager_t* pager, int keep, int* evicted);
LBM_API int lbm_pager_reset(lbm_pager_t* pager);
LBM_API int lbm_pager_state(const lbm_pager_t* pager, lbm_cache_state_t* state);
LBM_API void lbm_pager_destroy(lbm_pager_t* pager);

#ifdef __cplusplus
}
#endif
#endif /* LBM_H */
