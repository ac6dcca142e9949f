// Paged attention of one frame's queries over the retained keys, bf16 in / fp32 softmax,
// on the 5th-generation tensor cores (tcgen05, accumulators in tensor memory).
//
// [3DRoPE-KV] "Attention Computation with Cached RoPE": the queries of the frame attend
// over the visible page table (scale pages -> window pages -> own page -> special pages,
// the last special page partly filled), with K/V that already carry their rotation.
//
// One CTA = two query tiles of 128 rows of one head, over one split of the key tiles.
// Both query tiles share every K/V tile the CTA loads.  Warp roles (12 warps):
//   warp 0      TMA producer: the two Q tiles once per segment, then K/V tiles gathered
//               page by page through the page table into a ring of shared-memory stages
//               (128B swizzle).
//   warp 1, 2   allocate tensor memory (warp 1); one lane of warp 1+g issues every
//               tcgen05.mma of query tile g:
//                 S = Q_g K_j^T   (A, B from shared memory)      -> TMEM S_g
//                 O_g += P V_j    (A = P from TMEM, B = V smem)   -> TMEM O_g
//               S_{j+1} is issued before PV_j, so scores and softmax overlap: at head_dim 64
//               as soon as the softmax warps have read S_j (one S buffer); at head_dim 128
//               into the other of two S buffers once PV_{j-1} has read the P it held.
//   warps 4..7  softmax of query tile 0, warps 8..11 of tile 1: each thread owns one query
//               row (its TMEM lane); reads S_j, row max, exp2, row sum in fp32, writes P_j
//               (bf16) into TMEM, and rescales O only when the running max grew by more than
//               2^8 (lazy rescale; exact because O and l share one reference max).
//               When the frame's q is raw (its append left q alone), each softmax thread
//               also rotates its own query row in place in shared memory at the token's
//               (t, h, w) position before Q.K^T reads it ([3DRoPE-KV] FAQ "Where does the
//               RoPE application occur relative to the KV cache write?"): the next segment's
//               rows are rotated while the current segment's last P.V runs.
//   The two softmax warpgroups run concurrently, so one's exponentials overlap the other's
//   tensor-core work.
// Tensor memory: 256 columns per query tile g at 256 g.  head_dim 64, 128-key tiles: S [0,128),
// P [128,192), O [192,256).  head_dim 128, 64-key tiles: S_0 [0,64), S_1 [64,128) with P_b
// written over S_b, O [128,256).
// Every mbarrier wait is bounded (about 2 s); a wait that runs out sets the device error
// word, raises a CTA-wide abort flag, and every role falls through to the common exit,
// which drains outstanding copies / MMAs (bounded) and frees tensor memory.
#include <cuda_bf16.h>

#include <mutex>

#include "../../include/lbm.h"
#include "lbm_internal.h"

namespace lbm {
namespace {

constexpr int BM = 128;         // query rows per CTA
constexpr int kThreads = 384;   // 12 warps
constexpr uint32_t kTmemCols = 512;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;
constexpr unsigned long long kImmediateLimitNs = 1000ull;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale when max grows by > 2^8
constexpr unsigned kFull = 0xffffffffu;

constexpr int kMaxStages = 6;  // K/V ring stages the barrier block has room for

template <int D, bool FOLD>
struct Cfg {
  static constexpr int BN = attn_key_tile(D);            // keys per K/V tile
  // K/V pipeline stages: six 16 KB stages fill the room left next to the query tiles at
  // head_dim 64 (measured 1-2 % faster than four there; five at head_dim 128 were not)
  static constexpr int NS = (D == 64 && !FOLD) ? 6 : 4;
  static_assert(NS <= kMaxStages, "the barrier block holds kMaxStages ring barriers");
  static constexpr int ATOMS = D / 64;                   // 64-feature swizzle atom columns
  static constexpr int Q_ATOM = BM * 128;                // 128 query rows x 64 bf16
  static constexpr int KV_ATOM = BN * 128;               // BN key rows x 64 bf16
  static constexpr int Q_TILE = ATOMS * Q_ATOM;          // one query tile
  static constexpr int KV_TILE = ATOMS * KV_ATOM;        // one K or V tile
  static constexpr int OFF_Q = 0;                        // two query tiles
  static constexpr int OFF_K = OFF_Q + 2 * Q_TILE;
  static constexpr int OFF_V = OFF_K + NS * KV_TILE;
  static constexpr int OFF_BAR = OFF_V + NS * KV_TILE;
  static constexpr int BAR_BYTES = 512;
  static constexpr int OFF_TAB = OFF_BAR + BAR_BYTES;    // RoPE tables for the q rotation
  static constexpr int TAB_BYTES = FOLD ? kRopeStageBytes : 0;
  static constexpr int SMEM = OFF_TAB + TAB_BYTES + 1024;  // + slack to align the base to 1 KB
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

// ---- PTX wrappers -----------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// The issue helpers below (expect_tx, TMA, MMA, commit) are called by a whole warp in
// warp-uniform control flow; one elected lane issues the instruction.  Keeping the loop
// warp-uniform lets the compiler hold descriptors and addresses in uniform registers.
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n\t}" ::"r"(bar),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// try_wait without a suspend-time hint: the thread may be suspended for a short,
// system-defined time and resumes as soon as the phase completes.  (A long hint delayed the
// wake-up by several hundred cycles after the completing arrival, on the critical path
// between the softmax and MMA roles; spinning on test_wait took issue slots instead.)
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-suspending check of a phase (no wait at all).
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ unsigned long long global_timer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// What a bounded wait needs: the CTA's abort flag, the device error word and the time limit
// of one wait (roles' waits: the cache's wait limit, 2 s unless set; the drains at the exit
// always use kWaitLimitNs).
struct WaitCtx {
  volatile int* abort_flag;
  int* err;
  unsigned long long limit_ns;
};

// Bounded wait for the phase of `bar` with the given parity to complete.  Returns false
// when the CTA is aborting or the limit ran out (then the error word and abort flag are set).
__device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, WaitCtx wa,
                                            int where) {
  if (wa.limit_ns < kImmediateLimitNs) {
    // a limit below the resolution a suspended try_wait can honour: a wait that is not
    // satisfied at its first test runs out at once (how the failure path is exercised)
    *wa.abort_flag = 1;
    atomicExch(wa.err, where);
    return false;
  }
  const unsigned long long t0 = global_timer();
  while (true) {
    if (mbar_try(bar, parity)) return true;
    if (*wa.abort_flag) return false;
    if (global_timer() - t0 > wa.limit_ns) {
      *wa.abort_flag = 1;
      atomicExch(wa.err, where);
      return false;
    }
  }
}

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, const WaitCtx& wa,
                                          int where) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  if (ok) return true;
  return mbar_wait_slow(bar, parity, wa, where);
}

// Whole-warp wait: every lane waits, and the vote makes the outcome warp-uniform, so the
// warp-collective issue helpers after it always run with the full warp.
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity, const WaitCtx& wa,
                                               int where) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, wa, where));
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* tm, int x, int y,
                                            int z, uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];\n\t}" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor (sm100 format, version 1, 128-byte swizzle).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::f16: bf16 x bf16 -> f32, K-major A, B K- or MN-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accum)
      : "memory");
}

__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accum)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}"
      ::"r"(bar)
      : "memory");
}

// 32 consecutive 32-bit columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Pins registers after tcgen05.wait::ld so no use is scheduled before the wait.
template <int N>
__device__ __forceinline__ void reg_fence(uint32_t* r) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i])::"memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
      "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]),
      "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&b);
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ uint64_t pack_f2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}

__device__ __forceinline__ void unpack_f2(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}

// (a0, a1) * (b, b) + (c, c) on the paired fp32 pipe
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.ftz.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.ftz.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// The eight floats of four packed pairs, summed pairwise.
__device__ __forceinline__ float sum_f2x4(const uint64_t* v) {
  float a0, a1, b0, b1, c0, c1, d0, d1;
  unpack_f2(v[0], a0, a1);
  unpack_f2(v[1], b0, b1);
  unpack_f2(v[2], c0, c1);
  unpack_f2(v[3], d0, d1);
  return ((a0 + a1) + (b0 + b1)) + ((c0 + c1) + (d0 + d1));
}

// Key tile t of the visible list: pool (patch or special), first pool row, valid keys.
struct TileRef {
  bool special;
  int row0;
  int valid;
};

// Page index of patch tile t, t / tiles_per_page: a multiply-high with the host's
// tpp_magic = ceil(2^32 / tiles_per_page), exact while t * tiles_per_page < 2^32 (the host
// sets tpp_magic = 0 for frames where that could fail, and then this divides).
__device__ __forceinline__ int tile_page(const AttnParams& p, int t) {
  if (p.tiles_per_page == 1) return t;
  return p.tpp_magic ? (int)__umulhi((uint32_t)t, p.tpp_magic) : t / p.tiles_per_page;
}
__device__ __forceinline__ int tile_in_page(const AttnParams& p, int t) {
  return t - tile_page(p, t) * p.tiles_per_page;
}

template <int BN>
__device__ __forceinline__ TileRef tile_ref(const AttnParams& p, int t) {
  const int npt = p.n_pages * p.tiles_per_page;
  TileRef r;
  if (t < npt) {
    const int pi = tile_page(p, t);
    const int i = t - pi * p.tiles_per_page;
    r.special = false;
    r.row0 = (int)p.pages[pi] * p.page_stride + BN * i;
    r.valid = min(BN, p.patches - BN * i);
  } else {
    const int i = t - npt;
    r.special = true;
    r.row0 = BN * i;
    r.valid = min(BN, p.n_special - BN * i);
  }
  return r;
}

// Valid keys of key tile t (see tile_ref), without a division when every patch tile is full.
template <int BN>
__device__ __forceinline__ int tile_valid(const AttnParams& p, int t) {
  const int npt = p.n_pages * p.tiles_per_page;
  if (t >= npt) return min(BN, p.n_special - BN * (t - npt));
  if (p.patches % BN == 0) return BN;
  return min(BN, p.patches - BN * tile_in_page(p, t));
}

struct Bars {
  uint64_t q_loaded;       // the query tiles of the current segment landed (TMA)
  uint64_t q_full[2];      // per tile g: its rows rotated in place and visible to the MMA (128)
  uint64_t q_empty;        // both MMA issuers are done with them (count 2)
  uint64_t s_full[2][2];   // per query tile g and S buffer: S_j landed in TMEM
  uint64_t s_free[2];      // per g: the softmax warps have read S_j
  uint64_t p_full[2][2];   // per g and buffer: P_j written to TMEM (and O rescaled if needed)
  uint64_t pv_done[2][2];  // per g and buffer: PV_j finished (its P buffer is free again)
  uint64_t o_free[2];      // per g: the epilogue has read O of the segment
  uint64_t drain[2];
  uint64_t kv_full[kMaxStages];
  uint64_t kv_empty[kMaxStages];  // one arrival per MMA issuer (count 2)
  uint32_t tmem_base;
  int abort_flag;
};

static_assert(sizeof(Bars) <= 512, "barrier block exceeds its shared-memory slot");

// Tensor-memory columns of query tile g (256 columns at 256 g).  head_dim 64 (128-key tiles):
// S [0,128), P [128,192), O [192,256), one S/P buffer.  head_dim 128 (64-key tiles): two
// buffers S_b [64 b, 64 b + 64) with P_b written over the first 32 columns of S_b after S_b
// is read into registers, O [128,256); tile j uses buffer j % 2, so S_{j+1} can be computed
// while PV_j still reads P_j.
template <int D>
struct TmemMap {
  static constexpr int NB = D == 64 ? 1 : 2;  // S/P buffers
  __host__ __device__ static constexpr uint32_t S(int b) { return D == 64 ? 0 : 64 * b; }
  __host__ __device__ static constexpr uint32_t P(int b) { return D == 64 ? 128 : 64 * b; }
  static constexpr uint32_t O = D == 64 ? 192 : 128;
  // buffer of tile t, and the phase parity of that buffer's barriers at tile t
  __device__ static int buf(int t) { return NB == 1 ? 0 : (t & 1); }
  __device__ static uint32_t par(int t) { return (uint32_t)(NB == 1 ? t : (t >> 1)) & 1u; }
};

// One run of key tiles of one unit, as a CTA walks its share of the work.
struct Segment {
  int unit, a, b;   // items [a, b) of the unit
};

// Rotation of unit `unit`'s key order (units past the rotation table, kMaxUnits, keep the
// natural order).  Read once per segment: an indexed read of the parameter block.
__device__ __forceinline__ int unit_rot(const AttnParams& p, int unit) {
  return unit < kMaxUnits ? p.rot[unit] : 0;
}
// Key tile read by item i of a unit rotated by rot.
__device__ __forceinline__ int key_tile(const AttnParams& p, int rot, int i) {
  const int t = i + rot;
  return t >= p.n_tiles ? t - p.n_tiles : t;
}

// Work items are counted in 32-bit integers: the host keeps a frame's work below 2^31.
__device__ __forceinline__ Segment segment_at(const AttnParams& p, int x, int hi) {
  Segment sg;
  sg.unit = x / p.n_tiles;
  sg.a = x - sg.unit * p.n_tiles;
  sg.b = min(hi, (sg.unit + 1) * p.n_tiles) - sg.unit * p.n_tiles;
  return sg;
}
__device__ __forceinline__ int seg_pair(const AttnParams& p, const Segment& sg) {
  return sg.unit % p.n_pairs;
}
__device__ __forceinline__ int seg_head(const AttnParams& p, const Segment& sg) {
  return sg.unit / p.n_pairs;
}
__device__ __forceinline__ int seg_nq(const AttnParams& p, const Segment& sg, int q_tiles) {
  return min(2, q_tiles - 2 * seg_pair(p, sg));
}

// One query row in shared memory (K-major, 128-byte swizzle as the TMA box leaves it: the
// 16-byte chunk c of row r of an atom sits at chunk position c ^ (r % 8); the next 64
// features are one atom further) put in final form by its own thread.  With p.rotate_q the
// row's feature pairs are rotated at the token's (t, h, w) position in fp32 and rounded once
// to bf16 ([3DRoPE-KV] "Complex-Valued Tensor Application"), the same arithmetic as the
// append kernel's, and written back in place; with p.q_rot_out (first segment of the unit
// only: one writer per row) the rotated row is also stored there.  The (cos, sin) pairs come
// from the CTA's shared-memory copy of the tables (tab: t row of the frame, then the h and w
// tables) when p.rope_staged, else from global memory.  Rows past the frame are zeros from
// the TMA and stay zeros.  Ends with the fence that makes the generic-proxy writes visible to
// the tensor core.  Not inlined: it runs once per segment, and its registers stay out of the
// softmax loop's budget.
template <int D, int Q_ATOM>
__device__ __noinline__ void place_q_row(const AttnParams& p, const float2* tab, uint32_t q_row,
                                         int row, int head, bool writer) {
  if (!p.rotate_q || row >= p.tokens) return;
  const RopeTables& rt = p.rope;
  int hh = 0, ww = 0;
  if (row >= rt.psi) {
    const int pj = row - rt.psi;
    hh = 1 + pj / rt.ppw;
    ww = 1 + pj - (hh - 1) * rt.ppw;
  }
  // the row of each axis table this token uses
  const bool staged = p.rope_staged != 0;
  const float2* bt = staged ? tab : rt.tab_t + (size_t)p.frame * rt.nt;
  const float2* bh = staged ? tab + rt.nt + hh * rt.nh : rt.tab_h + (size_t)hh * rt.nh;
  const float2* bw = staged ? tab + rt.nt + (rt.pph + 1) * rt.nh + ww * rt.nw
                            : rt.tab_w + (size_t)ww * rt.nw;
  const int nth = rt.nt + rt.nh;
  const uint32_t sw = (uint32_t)(row & 7);  // the swizzle phase of this row (row % 8 of the tile)
  uint4* out = p.q_rot_out != nullptr && writer
                   ? reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.q_rot_out) +
                                              ((size_t)row * p.heads + head) * D)
                   : nullptr;
#pragma unroll
  for (int a = 0; a < D / 64; ++a) {
    float2 cs[32];
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      const int i = 32 * a + u;
      cs[u] = i < rt.nt ? bt[i] : (i < nth ? bh[i - rt.nt] : bw[i - nth]);
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint32_t addr = q_row + a * Q_ATOM + ((c ^ sw) << 4);
      uint32_t w[4];
      asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                   : "r"(addr));
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 r = cs[4 * c + u];
        const float x0 = __uint_as_float(w[u] << 16), x1 = __uint_as_float(w[u] & 0xffff0000u);
        w[u] = pack_bf16(fmaf(x0, r.x, -x1 * r.y), fmaf(x0, r.y, x1 * r.x));
      }
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w[0]),
                   "r"(w[1]), "r"(w[2]), "r"(w[3])
                   : "memory");
      if (out != nullptr) out[8 * a + c] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
  // generic-proxy writes, read by the tensor core through the async proxy
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Persistent CTA c of p.grid walks the global work items [sk_start[c], sk_start[c+1]).  Every role
// walks the same segments; barrier phases run on across segments (counters per role).
// FOLD: the frame's q is raw and every softmax thread rotates its query row in place after the
// TMA load (the append left q alone); without it the q rows are used as loaded.
template <int D, bool FOLD>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ AttnParams p) {
  using C = Cfg<D, FOLD>;
  using TM = TmemMap<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + C::OFF_BAR);
  volatile int* abort_flag = &bars->abort_flag;
  const WaitCtx wa{abort_flag, p.err, p.wait_limit_ns};

  // warp index through a shuffle: provably warp-uniform, so role-dependent descriptors and
  // addresses stay in uniform registers
  const int warp = __shfl_sync(0xffffffffu, (int)(threadIdx.x >> 5), 0);
  const int lane = threadIdx.x & 31;
  const int q_tiles = (p.tokens + BM - 1) / BM;
  const int lo = p.sk_start[blockIdx.x];
  const int hi = p.sk_start[blockIdx.x + 1];

  const uint32_t sQ = smem_u32(smem + C::OFF_Q);
  const uint32_t sK = smem_u32(smem + C::OFF_K);
  const uint32_t sV = smem_u32(smem + C::OFF_V);
  auto bar = [&](const uint64_t& b) { return smem_u32(&b); };

  if (threadIdx.x == 0) {
    mbar_init(bar(bars->q_loaded), 1);
    mbar_init(bar(bars->q_full[0]), 128);
    mbar_init(bar(bars->q_full[1]), 128);
    mbar_init(bar(bars->q_empty), 2);
    for (int g = 0; g < 2; ++g) {
      for (int b = 0; b < 2; ++b) {
        mbar_init(bar(bars->s_full[g][b]), 1);
        mbar_init(bar(bars->p_full[g][b]), 128);
        mbar_init(bar(bars->pv_done[g][b]), 1);
      }
      mbar_init(bar(bars->s_free[g]), 128);
      mbar_init(bar(bars->o_free[g]), 128);
      mbar_init(bar(bars->drain[g]), 1);
    }
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(bar(bars->kv_full[s]), 1);
      mbar_init(bar(bars->kv_empty[s]), 2);
    }
    bars->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // the frame's row of the t table and the whole h and w tables, for the in-kernel rotation
  // of q (constant inputs, so this may overlap the previous kernel's tail)
  float2* tab = reinterpret_cast<float2*>(smem + C::OFF_TAB);
  if (FOLD && p.rope_staged) {
    const RopeTables& rt = p.rope;
    const int n_h = (rt.pph + 1) * rt.nh, n_w = (rt.ppw + 1) * rt.nw;
    for (int i = threadIdx.x; i < rt.nt + n_h + n_w; i += kThreads)
      tab[i] = i < rt.nt ? __ldg(rt.tab_t + (size_t)p.frame * rt.nt + i)
                         : (i < rt.nt + n_h ? __ldg(rt.tab_h + (i - rt.nt))
                                            : __ldg(rt.tab_w + (i - rt.nt - n_h)));
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&bars->tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = __shfl_sync(0xffffffffu, bars->tmem_base, 0);
  // launched as a programmatic dependent of the append kernel: the set-up above overlapped
  // its tail; the pages it writes are read only after it has finished
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == 0) {
    // ---------------- TMA producer (whole warp, elected lane issues) ----------------
    int issued = 0;        // key tiles issued so far (ring position)
    int seg_i = 0;
    bool ok = true;
    for (int x = lo; ok && x < hi; ++seg_i) {
      const Segment sg = segment_at(p, x, hi);
      x = sg.unit * p.n_tiles + sg.b;
      // the query buffers are free once both MMA issuers are done with the last segment
      if (seg_i > 0 &&
          !mbar_wait_warp(bar(bars->q_empty), (seg_i - 1) & 1, wa, 12)) {
        ok = false;
        break;
      }
      const int n_q = seg_nq(p, sg, q_tiles);
      const int head = seg_head(p, sg);
      const int rot = unit_rot(p, sg.unit);
      mbar_expect_tx(bar(bars->q_loaded), n_q * C::Q_TILE);
      for (int g = 0; g < n_q; ++g) {
#pragma unroll
        for (int a = 0; a < C::ATOMS; ++a)
          tma_load_3d(sQ + g * C::Q_TILE + a * C::Q_ATOM, &p.tm_q, 64 * a, head,
                      (2 * seg_pair(p, sg) + g) * BM, bar(bars->q_loaded));
      }
      for (int t = sg.a; t < sg.b; ++t, ++issued) {
        const int s = issued % C::NS;
        if (issued >= C::NS &&
            !mbar_wait_warp(bar(bars->kv_empty[s]), ((issued - C::NS) / C::NS) & 1, wa,
                             1)) {
          ok = false;
          break;
        }
        const TileRef tr = tile_ref<C::BN>(p, key_tile(p, rot, t));
        const CUtensorMap* tk = tr.special ? &p.tm_ks : &p.tm_kp;
        const CUtensorMap* tv = tr.special ? &p.tm_vs : &p.tm_vp;
        mbar_expect_tx(bar(bars->kv_full[s]), 2 * C::KV_TILE);
#pragma unroll
        for (int a = 0; a < C::ATOMS; ++a) {
          tma_load_3d(sK + s * C::KV_TILE + a * C::KV_ATOM, tk, 64 * a, tr.row0, head,
                      bar(bars->kv_full[s]));
          tma_load_3d(sV + s * C::KV_TILE + a * C::KV_ATOM, tv, 64 * a, tr.row0, head,
                      bar(bars->kv_full[s]));
        }
      }
    }
    if (*abort_flag) {
      // drain: wait (bounded) for the copies this warp issued that may still be landing
      if (seg_i > 0) {
        const unsigned long long t0 = global_timer();
        while (!mbar_try(bar(bars->q_loaded), (seg_i - 1) & 1) &&
               global_timer() - t0 < kWaitLimitNs) {
        }
      }
      for (int j = max(0, issued - C::NS); j < issued; ++j) {
        const unsigned long long t0 = global_timer();
        while (!mbar_try(bar(bars->kv_full[j % C::NS]), (j / C::NS) & 1) &&
               global_timer() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else if (warp == 1 || warp == 2) {
    // ---------------- MMA issuers: warp 1 for query tile 0, warp 2 for tile 1 ----------------
    const int g = warp - 1;
    constexpr uint32_t idesc_s = idesc_bf16(BM, C::BN, false);
    constexpr uint32_t idesc_o = idesc_bf16(BM, D, true);
    const uint32_t tg = tmem + 256 * g;
    const uint32_t tO = tg + TM::O;
    const uint32_t q_base = sQ + g * C::Q_TILE;
    int ring = 0;     // key tiles consumed from the ring (all segments)
    int jg = 0;       // key tiles processed by this query tile (all segments)
    int segs = 0;     // segments this query tile took part in
    int seg_i = 0;
    bool ok = true;
    for (int x = lo; ok && x < hi; ++seg_i) {
      const Segment sg = segment_at(p, x, hi);
      x = sg.unit * p.n_tiles + sg.b;
      const int n = sg.b - sg.a;
      if (!mbar_wait_warp(bar(bars->q_loaded), seg_i & 1, wa, 2)) {
        ok = false;
        break;
      }
      if (g >= seg_nq(p, sg, q_tiles)) {
        // no second query tile in this pair: release each ring stage and the query buffers
        // after the tile has landed, so no arrival can run a phase ahead
        for (int t = 0; t < n; ++t, ++ring) {
          const int s = ring % C::NS;
          if (!mbar_wait_warp(bar(bars->kv_full[s]), (ring / C::NS) & 1, wa, 4)) {
            ok = false;
            break;
          }
          if (lane == 0) mbar_arrive(bar(bars->kv_empty[s]));
        }
        if (lane == 0) mbar_arrive(bar(bars->q_empty));
        continue;
      }
      // this tile's rows are in final form: rotated in place by the softmax threads when q is
      // raw (when it was rotated by the append, the TMA load alone is enough)
      if (FOLD && !mbar_wait_warp(bar(bars->q_full[g]), segs & 1, wa, 14)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int j0 = jg;  // first tile of this segment in this query tile's count
      auto issue_qk = [&](int j) -> bool {
        const int s = (ring + (j - j0)) % C::NS;
        const int r = ring + (j - j0);
        if (!mbar_wait_warp(bar(bars->kv_full[s]), (r / C::NS) & 1, wa, 4))
          return false;
        // the S buffer of tile j is free: one buffer, the softmax has read S_{j-1}; two
        // buffers, PV_{j-2} has read P_{j-2}, which was written after S_{j-2} was read
        if (TM::NB == 1) {
          if (j >= 1 &&
              !mbar_wait_warp(bar(bars->s_free[g]), (j - 1) & 1, wa, 5))
            return false;
        } else if (j >= 2 && !mbar_wait_warp(bar(bars->pv_done[g][TM::buf(j)]), TM::par(j - 2),
                                             wa, 5)) {
          return false;
        }
        tc_fence_after();
        const uint32_t k_base = sK + s * C::KV_TILE;
        const uint32_t tS = tg + TM::S(TM::buf(j));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t qo = (kk >> 2) * C::Q_ATOM + (kk & 3) * 32;
          const uint32_t ko = (kk >> 2) * C::KV_ATOM + (kk & 3) * 32;
          mma_ss(tS, sdesc(q_base + qo, 16, 1024), sdesc(k_base + ko, 16, 1024), idesc_s,
                 kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(bars->s_full[g][TM::buf(j)]));
        return true;
      };
      auto issue_pv = [&](int i) -> bool {
        if (!mbar_wait_warp(bar(bars->p_full[g][TM::buf(i)]), TM::par(i), wa, 3))
          return false;
        // O of the previous segment must have been read out before the first PV overwrites it
        if (i == j0 && segs > 0 &&
            !mbar_wait_warp(bar(bars->o_free[g]), (segs - 1) & 1, wa, 13))
          return false;
        tc_fence_after();
        const int s = (ring + (i - j0)) % C::NS;
        const uint32_t v_base = sV + s * C::KV_TILE;
        const uint32_t tP = tg + TM::P(TM::buf(i));
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk) {
          // B = V tile [keys][D], MN-major: 16 keys = 2 groups of 8 rows of 128 B; the next
          // 64 features are one atom column (KV_ATOM bytes) further
          const uint64_t bd = sdesc(v_base + kk * 2048, C::KV_ATOM, 1024);
          mma_ts(tO, tP + 8 * kk, bd, idesc_o, (i > j0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar(bars->pv_done[g][TM::buf(i)]));
        mma_commit(bar(bars->kv_empty[s]));
        return true;
      };
      // S_j is issued before PV_{j-1}, so the softmax can start on it early
      ok = ok && issue_qk(j0);
      for (int j = j0 + 1; ok && j < j0 + n; ++j) ok = issue_qk(j) && issue_pv(j - 1);
      if (ok) {
        // the last QK of the segment has been issued: the query buffers can be refilled once
        // it completes
        mma_commit(bar(bars->q_empty));
        ok = issue_pv(j0 + n - 1);
      }
      jg += n;
      ring += n;
      ++segs;
    }
    // every MMA issued by this warp has completed once `drain` flips
    mma_commit(bar(bars->drain[g]));
    const unsigned long long t0 = global_timer();
    while (!mbar_try(bar(bars->drain[g]), 0) && global_timer() - t0 < kWaitLimitNs) {
    }
  } else if (warp >= 4) {
    // ---------------- softmax + epilogue: warps 4..7 tile 0, warps 8..11 tile 1 ----------------
    const int g = (warp - 4) >> 2;
    const int quad = warp & 3;                  // TMEM lane quadrant this warp may access
    const int row_in_pair = g * BM + quad * 32 + lane;
    const uint32_t lane_base = tmem + 256 * g + ((uint32_t)(quad * 32) << 16);
    const uint32_t tO = lane_base + TM::O;
    constexpr int BN = C::BN;
    int jg = 0;
    int seg_i = 0;
    bool ok = true;
    bool q_placed = false;  // this segment's rows were placed ahead, during the last one
    // waits for segment k's query tiles and, if this tile takes part, puts its row in final
    // form; every segment's q_loaded phase is waited, so its parity stays unambiguous
    auto place_q = [&](const Segment& qs, int k) -> bool {
      if (!FOLD) return true;  // q rotated by the append: nothing to place
      if (!__all_sync(kFull, mbar_wait(bar(bars->q_loaded), k & 1, wa, 15)))
        return false;
      if (g < seg_nq(p, qs, q_tiles)) {
        // this thread's row of tile g (recomputed here: nothing of it stays live in the loop)
        const uint32_t q_row = smem_u32(smem + C::OFF_Q) + g * C::Q_TILE +
                               ((threadIdx.x - 128u) & 127u) * 128u;
        place_q_row<D, C::Q_ATOM>(p, reinterpret_cast<const float2*>(smem + C::OFF_TAB), q_row,
                                   (2 * seg_pair(p, qs)) * BM + row_in_pair, seg_head(p, qs),
                                   qs.a == 0);
        mbar_arrive(bar(bars->q_full[g]));
      }
      return true;
    };
    uint32_t S[BN];
    for (int x = lo; ok && x < hi; ++seg_i) {
      const Segment sg = segment_at(p, x, hi);
      x = sg.unit * p.n_tiles + sg.b;
      if (FOLD && !q_placed && !place_q(sg, seg_i)) {
        ok = false;
        break;
      }
      q_placed = false;
      if (g >= seg_nq(p, sg, q_tiles)) continue;
      const int n = sg.b - sg.a;
      const int j0 = jg;
      // head_dim 128 reads the unit's rotation once per segment (the valid-key count is
      // computed before the score wait); head_dim 64 per tile (measured faster there)
      const int rot = D == 128 ? unit_rot(p, sg.unit) : 0;
      float m = -INFINITY;  // running max (log2 domain) the P values and O are relative to
      float l = 0.f;
      for (int j = j0; ok && j < j0 + n; ++j) {
        // every wait in these warps is made warp-uniform, so warp-collective tcgen05 ops and
        // votes below always run with the whole warp
        const int sb = TM::buf(j);
        const uint32_t tS = lane_base + TM::S(sb);
        const uint32_t tP = lane_base + TM::P(sb);
        // keys of this tile: at head_dim 128 computed before the wait, off the score -> max
        // chain; at head_dim 64 (every register taken) after the scores are in
        int valid = D == 128 ? tile_valid<BN>(p, key_tile(p, rot, sg.a + (j - j0))) : BN;
        if (!__all_sync(kFull, mbar_wait(bar(bars->s_full[g][sb]), TM::par(j), wa, 6))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) tmem_ld32(tS + 32 * c, S + 32 * c);
        tmem_wait_ld();
        reg_fence<BN>(S);
        if (TM::NB == 1) {
          // one S buffer: the next Q.K^T may overwrite it once every thread has read it
          tc_fence_before();
          mbar_arrive(bar(bars->s_free[g]));
        }

        if (D == 64) valid = tile_valid<BN>(p, key_tile(p, unit_rot(p, sg.unit), sg.a + (j - j0)));
        if (valid != BN) {
          // keys past the end of a page / of the special stream: -inf scores, zero weight
#pragma unroll
          for (int i = 0; i < BN; ++i)
            if (i >= valid) S[i] = 0xff800000u;
        }
        float mx8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          mx8[i] = fmaxf(__uint_as_float(S[2 * i]), __uint_as_float(S[2 * i + 1]));
#pragma unroll
        for (int i = 16; i < BN; i += 2)
          mx8[(i >> 1) & 7] = max3f(mx8[(i >> 1) & 7], __uint_as_float(S[i]),
                                    __uint_as_float(S[i + 1]));
        const float mx = max3f(max3f(mx8[0], mx8[1], mx8[2]), max3f(mx8[3], mx8[4], mx8[5]),
                               fmaxf(mx8[6], mx8[7]));
        const float m_tile = mx * p.scale_log2;
        bool rescale = false;
        float alpha = 1.f;
        if (m_tile > m + kRescaleThreshold) {
          alpha = fast_exp2(m - m_tile);  // 0 on the first tile (m = -inf)
          m = m_tile;
          l *= alpha;
          rescale = true;
        }
        // one P buffer: P_j overwrites P_{j-1}, so PV_{j-1} must have finished (two buffers:
        // P_j goes to its own S buffer; PV_{j-1} is waited for only before rescaling O)
        if (TM::NB == 1 && j >= 1 &&
            !__all_sync(kFull, mbar_wait(bar(bars->pv_done[g][0]), (j - 1) & 1, wa,
                                          7))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t c2 = pack_f2(p.scale_log2, p.scale_log2);
        const uint64_t nm2 = pack_f2(-m, -m);
        uint64_t l4[4] = {0, 0, 0, 0};
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int i0 = 32 * c + 2 * i;
            float x0, x1;
            unpack_f2(ffma2(pack_f2(__uint_as_float(S[i0]), __uint_as_float(S[i0 + 1])), c2,
                            nm2),
                      x0, x1);
            const float p0 = fast_exp2(x0);
            const float p1 = fast_exp2(x1);
            l4[i & 3] = fadd2(l4[i & 3], pack_f2(p0, p1));
            pk[i] = pack_bf16(p0, p1);
          }
          tmem_st16(tP + 16 * c, pk);
        }
        l += sum_f2x4(l4);
        if (__any_sync(kFull, rescale) && j > j0) {
          // O holds sum_{i<j} P_i V_i relative to the old max: scale it before PV_j lands
          if (TM::NB == 2 &&
              !__all_sync(kFull, mbar_wait(bar(bars->pv_done[g][TM::buf(j - 1)]),
                                           TM::par(j - 1), wa, 7))) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + 32 * c, o);
            tmem_wait_ld();
            reg_fence<32>(o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st16(tO + 32 * c, o);
            tmem_st16(tO + 32 * c + 16, o + 16);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(bars->p_full[g][sb]));
      }
      // the next segment's query tiles land once both Q.K^T of this one are done: if they
      // are there, put them in final form now, while the last P.V of this segment runs
      // (otherwise at the top of the next segment, after this one's epilogue)
      if (FOLD && ok && x < hi &&
          __all_sync(kFull, mbar_test(bar(bars->q_loaded), (seg_i + 1) & 1))) {
        if (!place_q(segment_at(p, x, hi), seg_i + 1)) {
          ok = false;
          break;
        }
        q_placed = true;
      }
      jg += n;
      if (!ok ||
          !__all_sync(kFull, mbar_wait(bar(bars->pv_done[g][TM::buf(jg - 1)]), TM::par(jg - 1),
                                       wa, 
                                       9))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float inv_l = 1.f / l;
      const int row = (2 * seg_pair(p, sg)) * BM + row_in_pair;
      const bool store = row < p.tokens;
      if (sg.a == 0 && sg.b == p.n_tiles) {   // the whole unit: write the final output
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) +
                             ((long long)row * p.heads + seg_head(p, sg)) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + 32 * c, o);
          tmem_wait_ld();
          reg_fence<32>(o);
          if (store) {
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              w[i] = pack_bf16(__uint_as_float(o[2 * i]) * inv_l,
                               __uint_as_float(o[2 * i + 1]) * inv_l);
            uint4* dst = reinterpret_cast<uint4*>(out + 32 * c);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
          }
        }
      } else {
        // slot unit + c: one per (CTA, unit it touches), dense over CTAs in order
        const long long slot = (long long)sg.unit + blockIdx.x;
        const long long r = slot * (2 * BM) + row_in_pair;
        float* po = p.part_o + r * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + 32 * c, o);
          tmem_wait_ld();
          reg_fence<32>(o);
          if (store) {
            float4* dst = reinterpret_cast<float4*>(po + 32 * c);
#pragma unroll
            for (int v = 0; v < 8; ++v)
              dst[v] = make_float4(__uint_as_float(o[4 * v]) * inv_l,
                                   __uint_as_float(o[4 * v + 1]) * inv_l,
                                   __uint_as_float(o[4 * v + 2]) * inv_l,
                                   __uint_as_float(o[4 * v + 3]) * inv_l);
          }
        }
        if (store) p.part_lse[r] = m + __log2f(l);
      }
      // O of this segment has been read: the next segment's first PV may overwrite it
      tc_fence_before();
      mbar_arrive(bar(bars->o_free[g]));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

// Largest c in [0, grid) with sk_start[c] <= x (binary search, warp-uniform).
__device__ __forceinline__ int last_start_at_or_before(const AttnParams& p, int x) {
  int lo = 0, hi = p.grid - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.sk_start[mid] <= x)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

// Merges the partial results of the units that span more than one CTA:
// out[row][h] = sum_s w_s o_s / sum_s w_s with w_s = 2^(lse_s - max_s lse_s).
// One warp per (unit, four rows of the pair): each quarter-warp owns one row, its 8 lanes
// hold D / 8 features each.  Lane s of a quarter loads the LSE of segment s (8 at a time),
// the quarter reduces max and weights with shuffles, then the O rows of four segments (two
// for head_dim 128) are loaded before any is used, so a row costs about two L2 round trips,
// and the index work of a warp is shared by four rows.  32-bit indices: a frame's partials are far below 2^31
// floats.
template <int D>
__global__ void __launch_bounds__(256) attn_combine_kernel(const __grid_constant__ AttnParams p) {
  constexpr int VPL = D / 8;   // features per lane
  constexpr int V4 = VPL / 4;  // float4 loads per lane and segment
  constexpr int RPW = 4;       // rows per warp
  constexpr int SB = D == 64 ? 4 : 2;  // segments whose O rows are loaded before use
  const unsigned gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int quarter = lane >> 3;
  const int ql = lane & 7;
  const unsigned units = (unsigned)(p.n_pairs * p.heads);
  constexpr unsigned kWarpsPerUnit = 2 * BM / RPW;
  if (gw >= units * kWarpsPerUnit) return;
  const int unit = (int)(gw / kWarpsPerUnit);
  const int row_in_pair = (int)(gw - (unsigned)unit * kWarpsPerUnit) * RPW + quarter;
  const int head = unit / p.n_pairs;
  const int pair = unit - head * p.n_pairs;
  const int row = 2 * pair * BM + row_in_pair;
  const int first = unit * p.n_tiles;
  const int last = first + p.n_tiles - 1;
  // CTAs whose share [sk_start[c], sk_start[c+1]) meets this unit: c0 .. c1 (the shares are
  // non-empty and increasing: c0 is the last CTA starting at or before the unit's first
  // item, c1 the last starting at or before its last item, a few CTAs after c0)
  const int c0 = last_start_at_or_before(p, first);
  int c1 = c0;
  while (c1 + 1 < p.grid && p.sk_start[c1 + 1] <= last) ++c1;
  if (c1 == c0) return;  // one CTA did the whole unit and wrote the output itself
  // the index arithmetic above reads only kernel parameters and overlapped the attention
  // kernel's tail; its partials are read only after it has completed
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const bool valid = row < p.tokens;  // rows past the frame have no partials
  const int nseg = c1 - c0 + 1;
  // partial row of segment (CTA c0 + s): slot unit + c
  const int r0 = (unit + c0) * (2 * BM) + row_in_pair;
  float mx = -INFINITY;
  for (int s0 = 0; s0 < nseg; s0 += 8) {
    const float v = valid && s0 + ql < nseg ? p.part_lse[r0 + (s0 + ql) * (2 * BM)] : -INFINITY;
    mx = fmaxf(mx, v);
  }
#pragma unroll
  for (int o = 4; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float acc[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) acc[i] = 0.f;
  float wsum = 0.f;
  for (int s0 = 0; s0 < nseg; s0 += 8) {
    const float w_lane =
        valid && s0 + ql < nseg ? fast_exp2(p.part_lse[r0 + (s0 + ql) * (2 * BM)] - mx) : 0.f;
    const int cnt = min(8, nseg - s0);  // the same for every quarter (one unit per warp)
    for (int k0 = 0; k0 < cnt; k0 += SB) {
      float4 v[SB][V4];
      float w[SB];
#pragma unroll
      for (int u = 0; u < SB; ++u) {
        const int k = min(k0 + u, cnt - 1);
        w[u] = __shfl_sync(0xffffffffu, w_lane, (quarter << 3) + k);
        const float4* po = reinterpret_cast<const float4*>(
            p.part_o + (size_t)(r0 + (s0 + k) * (2 * BM)) * D + ql * VPL);
#pragma unroll
        for (int q = 0; q < V4; ++q)
          v[u][q] = valid && k0 + u < cnt ? po[q] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < SB; ++u) {
        if (k0 + u >= cnt) break;
        wsum += w[u];
#pragma unroll
        for (int q = 0; q < V4; ++q) {
          acc[4 * q] = fmaf(w[u], v[u][q].x, acc[4 * q]);
          acc[4 * q + 1] = fmaf(w[u], v[u][q].y, acc[4 * q + 1]);
          acc[4 * q + 2] = fmaf(w[u], v[u][q].z, acc[4 * q + 2]);
          acc[4 * q + 3] = fmaf(w[u], v[u][q].w, acc[4 * q + 3]);
        }
      }
    }
  }
  if (!valid) return;
  const float inv = 1.f / wsum;
  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) + ((size_t)row * p.heads + head) * D +
                     ql * VPL;
#pragma unroll
  for (int q = 0; q < V4; ++q)
    *reinterpret_cast<uint2*>(o + 4 * q) =
        make_uint2(pack_bf16(acc[4 * q] * inv, acc[4 * q + 1] * inv),
                   pack_bf16(acc[4 * q + 2] * inv, acc[4 * q + 3] * inv));
}

}  // namespace

size_t attn_tc_smem_bytes(int head_dim, bool fold) {
  if (head_dim == 64) return fold ? Cfg<64, true>::SMEM : Cfg<64, false>::SMEM;
  return fold ? Cfg<128, true>::SMEM : Cfg<128, false>::SMEM;
}

namespace {

constexpr int kMaxAttnDevices = 64;

// The shared-memory opt-in of a kernel is set per device: once for every device this process
// launches the kernel on (thread-safe, no allocation).
template <int D, bool FOLD>
cudaError_t prepare_attn_tc() {
  static std::once_flag once[kMaxAttnDevices];
  static cudaError_t state[kMaxAttnDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxAttnDevices)
    return cudaErrorInvalidDevice;
  std::call_once(once[dev], [dev] {
    state[dev] = cudaFuncSetAttribute(attn_tc_kernel<D, FOLD>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      Cfg<D, FOLD>::SMEM);
  });
  return state[dev];
}

}  // namespace

namespace {

// Launch with programmatic stream serialisation: the kernel may be scheduled while the
// previous kernel on the stream drains; it waits for it (griddepcontrol.wait) before
// touching that kernel's results.
template <typename K>
cudaError_t launch_pdl(K kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       const AttnParams& p) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, p);
}

template <int D, bool FOLD>
cudaError_t launch_attn_tc_t(const AttnParams& p, cudaStream_t s) {
  cudaError_t e;
  if ((e = prepare_attn_tc<D, FOLD>()) != cudaSuccess) return e;
  return launch_pdl(attn_tc_kernel<D, FOLD>, dim3(p.grid), dim3(kThreads), Cfg<D, FOLD>::SMEM,
                    s, p);
}

}  // namespace

cudaError_t launch_attn_tc(const AttnParams& p, int head_dim, cudaStream_t s) {
  const bool fold = p.rotate_q != 0;
  if (head_dim == 64) return fold ? launch_attn_tc_t<64, true>(p, s) : launch_attn_tc_t<64, false>(p, s);
  if (head_dim == 128)
    return fold ? launch_attn_tc_t<128, true>(p, s) : launch_attn_tc_t<128, false>(p, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_attn_combine(const AttnParams& p, int head_dim, cudaStream_t s) {
  const long long warps = (long long)p.n_pairs * p.heads * (2 * BM / 4);  // four rows a warp
  const dim3 blocks((unsigned)((warps * 32 + 255) / 256));
  if (head_dim == 64) return launch_pdl(attn_combine_kernel<64>, blocks, dim3(256), 0, s, p);
  if (head_dim == 128) return launch_pdl(attn_combine_kernel<128>, blocks, dim3(256), 0, s, p);
  return cudaErrorInvalidValue;
}

}  // namespace lbm
