// Host page manager of the dual-stream paged KV cache (pure integer code, no CUDA).
//
// [3DRoPE-KV] "Dual-Stream Memory Layout": one patch page per frame; the first
// scale_frames committed keyframes keep their pages, later ones enter a sliding window of
// sliding_window pages whose oldest page returns to the free list when it overflows.  The
// special stream is append-only.  [KVBenefits] "Dynamic Keyframe Selection": a frame is
// placed tentatively, attends, and is then kept (deferred eviction) or rolled back -- decided
// at append, or after the attention when the frame is appended undecided.
#pragma once

#include <cstdint>
#include <deque>
#include <vector>

#include "../../include/lbm.h"

namespace lbm {

constexpr int kSpecialPage = 128;

enum class PagerStatus { kOk, kSequence, kCapacity };

struct PageEntry {
  int page;
  long long frame;
};

class Pager {
 public:
  Pager(int scale_frames, int sliding_window, int max_frames, int specials_per_frame);

  int num_pages() const { return scale_frames_ + sliding_window_ + 1; }
  void reset();

  // Pops a page for frame_idx and reserves the next specials_per_frame special slots.
  // mode: 0 drop after attention, 1 keep, LBM_KEYFRAME_DEFERRED decide with commit().
  PagerStatus append(long long frame_idx, int mode, int* page, int* special_slot);
  // What append would return, without changing any state.
  PagerStatus peek_append(long long frame_idx, int mode, int* page, int* special_slot) const;
  // Visible patch pages of the pending frame, in scale -> window -> own order.
  PagerStatus visible(std::vector<int>* pages, int* n_special, int* last_page_len) const;
  // After the pending frame's attention: commit or roll back a decided frame (*evicted =
  // page freed by deferred eviction or -1); an undecided frame only becomes attended.
  PagerStatus finish(int* evicted);
  // Keep or drop an undecided frame after its attention (kCapacity: keeping it would exceed
  // max_frames; the frame stays pending).
  PagerStatus commit(bool keep, int* evicted);
  // True while a pending frame can still be attended.
  bool awaiting_attention() const { return pending_ && !attended_; }

  bool pending() const { return pending_; }
  int pending_page() const { return pending_page_; }
  bool pending_is_keyframe() const { return pending_key_; }
  bool pending_deferred() const { return pending_ && deferred_; }
  long long pending_frame() const { return pending_frame_; }
  long long last_frame() const { return last_frame_; }
  int n_special() const { return n_special_; }
  int committed() const { return committed_; }
  const std::vector<PageEntry>& scale() const { return scale_; }
  const std::deque<PageEntry>& window() const { return window_; }
  const std::vector<int>& free_stack() const { return free_; }

 private:
  int scale_frames_, sliding_window_, max_frames_, specials_;
  std::vector<PageEntry> scale_;
  std::deque<PageEntry> window_;
  std::vector<int> free_;  // stack, top = back()
  int n_special_ = 0;
  int committed_ = 0;
  bool pending_ = false;
  int pending_page_ = -1;
  bool pending_key_ = false;
  bool deferred_ = false;   // the pending frame waits for commit()
  bool attended_ = false;   // ... and its attention has been issued
  long long pending_frame_ = -1;
  long long last_frame_ = -1;

  PagerStatus settle(int* evicted);  // commit / roll back the pending frame by pending_key_
};

// Fills the counts and, where the caller gave room, the arrays of a state snapshot.
int fill_state(const Pager& p, lbm_cache_state_t* st);

}  // namespace lbm
