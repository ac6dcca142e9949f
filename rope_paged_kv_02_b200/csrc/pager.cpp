// Host page manager and its C ABI (lbm_pager_*).  See pager.h for the rules it follows.
#include "pager.h"

#include <algorithm>
#include <new>

#include "../../include/lbm.h"

namespace lbm {

Pager::Pager(int scale_frames, int sliding_window, int max_frames, int specials_per_frame)
    : scale_frames_(scale_frames),
      sliding_window_(sliding_window),
      max_frames_(max_frames),
      specials_(specials_per_frame) {
  reset();
}

void Pager::reset() {
  scale_.clear();
  window_.clear();
  free_.clear();
  // A fresh cache pops pages 0, 1, ..., P-1: push them in reverse.
  for (int p = num_pages() - 1; p >= 0; --p) free_.push_back(p);
  n_special_ = 0;
  committed_ = 0;
  pending_ = false;
  pending_page_ = -1;
  pending_key_ = false;
  deferred_ = false;
  attended_ = false;
  pending_frame_ = -1;
  last_frame_ = -1;
}

PagerStatus Pager::peek_append(long long frame_idx, int mode, int* page,
                               int* special_slot) const {
  if (pending_ || frame_idx <= last_frame_) return PagerStatus::kSequence;
  if (mode == 1 && committed_ >= max_frames_) return PagerStatus::kCapacity;
  *page = free_.back();
  *special_slot = n_special_;
  return PagerStatus::kOk;
}

PagerStatus Pager::append(long long frame_idx, int mode, int* page, int* special_slot) {
  if (pending_ || frame_idx <= last_frame_) return PagerStatus::kSequence;
  if (mode == 1 && committed_ >= max_frames_) return PagerStatus::kCapacity;
  // There is always a free page here: at most scale_frames + sliding_window are held
  // between frames, and P = scale_frames + sliding_window + 1.
  pending_page_ = free_.back();
  free_.pop_back();
  pending_ = true;
  pending_key_ = mode == 1;
  deferred_ = mode == LBM_KEYFRAME_DEFERRED;
  attended_ = false;
  pending_frame_ = frame_idx;
  last_frame_ = frame_idx;
  *page = pending_page_;
  *special_slot = n_special_;
  return PagerStatus::kOk;
}

PagerStatus Pager::visible(std::vector<int>* pages, int* n_special, int* last_page_len) const {
  if (!pending_) return PagerStatus::kSequence;
  pages->clear();
  for (const auto& e : scale_) pages->push_back(e.page);
  for (const auto& e : window_) pages->push_back(e.page);
  pages->push_back(pending_page_);
  const int n_sp = n_special_ + specials_;
  const int sp_pages = (n_sp + kSpecialPage - 1) / kSpecialPage;
  *n_special = n_sp;
  *last_page_len = n_sp - kSpecialPage * (sp_pages - 1);
  return PagerStatus::kOk;
}

PagerStatus Pager::finish(int* evicted) {
  if (!pending_ || attended_) return PagerStatus::kSequence;
  *evicted = -1;
  if (deferred_) {
    attended_ = true;  // the decision comes with commit()
    return PagerStatus::kOk;
  }
  return settle(evicted);
}

PagerStatus Pager::commit(bool keep, int* evicted) {
  if (!pending_ || !deferred_ || !attended_) return PagerStatus::kSequence;
  if (keep && committed_ >= max_frames_) return PagerStatus::kCapacity;
  pending_key_ = keep;
  return settle(evicted);
}

PagerStatus Pager::settle(int* evicted) {
  *evicted = -1;
  if (pending_key_) {
    const PageEntry e{pending_page_, pending_frame_};
    if (static_cast<int>(scale_.size()) < scale_frames_) {
      scale_.push_back(e);
    } else {
      window_.push_back(e);
      if (static_cast<int>(window_.size()) > sliding_window_) {
        *evicted = window_.front().page;  // deferred eviction: after this frame's attention
        window_.pop_front();
        free_.push_back(*evicted);
      }
    }
    n_special_ += specials_;
    ++committed_;
  } else {
    free_.push_back(pending_page_);  // rollback: the tentative page goes back on top
  }
  pending_ = false;
  pending_page_ = -1;
  pending_key_ = false;
  deferred_ = false;
  attended_ = false;
  pending_frame_ = -1;
  return PagerStatus::kOk;
}

}  // namespace lbm

struct lbm_pager {
  lbm::Pager p;
};

namespace {

int to_status(lbm::PagerStatus s) {
  switch (s) {
    case lbm::PagerStatus::kOk: return LBM_OK;
    case lbm::PagerStatus::kSequence: return LBM_ERR_SEQUENCE;
    case lbm::PagerStatus::kCapacity: return LBM_ERR_CAPACITY;
  }
  return LBM_ERR_INVALID;
}

}  // namespace

namespace lbm {

// Fills the counts and (where the caller gave room) the arrays of a state snapshot.
int fill_state(const Pager& p, lbm_cache_state_t* st) {
  if (!st) return LBM_ERR_INVALID;
  const int cap = st->capacity;
  st->num_pages = p.num_pages();
  st->n_scale = static_cast<int>(p.scale().size());
  st->n_window = static_cast<int>(p.window().size());
  st->n_free = static_cast<int>(p.free_stack().size());
  st->n_special = p.n_special();
  st->special_pages = (p.n_special() + kSpecialPage - 1) / kSpecialPage;
  st->last_page_len =
      st->special_pages ? p.n_special() - kSpecialPage * (st->special_pages - 1) : 0;
  st->pending = p.pending() ? 1 : 0;
  st->pending_page = p.pending_page();
  st->pending_is_keyframe = p.pending_deferred() ? LBM_KEYFRAME_DEFERRED
                                                 : (p.pending_is_keyframe() ? 1 : 0);
  st->pending_frame = p.pending_frame();
  st->last_frame = p.last_frame();
  if (cap < 0) return LBM_ERR_INVALID;
  if ((st->scale_pages || st->scale_frames) && st->n_scale > cap) return LBM_ERR_CAPACITY;
  if ((st->window_pages || st->window_frames) && st->n_window > cap) return LBM_ERR_CAPACITY;
  if (st->free_pages && st->n_free > cap) return LBM_ERR_CAPACITY;
  for (int i = 0; i < st->n_scale; ++i) {
    if (st->scale_pages) st->scale_pages[i] = p.scale()[i].page;
    if (st->scale_frames) st->scale_frames[i] = p.scale()[i].frame;
  }
  for (int i = 0; i < st->n_window; ++i) {
    if (st->window_pages) st->window_pages[i] = p.window()[i].page;
    if (st->window_frames) st->window_frames[i] = p.window()[i].frame;
  }
  if (st->free_pages)
    std::copy(p.free_stack().begin(), p.free_stack().end(), st->free_pages);
  return LBM_OK;
}

}  // namespace lbm

extern "C" {

int lbm_pager_create(int scale_frames, int sliding_window, int max_frames,
                     int specials_per_frame, lbm_pager_t** out) {
  if (!out) return LBM_ERR_INVALID;
  *out = nullptr;
  if (scale_frames < 0 || sliding_window < 0 || max_frames < 1 || specials_per_frame < 1 ||
      scale_frames + sliding_window + 1 > LBM_MAX_PAGES)
    return LBM_ERR_INVALID;
  auto* p = new (std::nothrow)
      lbm_pager{lbm::Pager(scale_frames, sliding_window, max_frames, specials_per_frame)};
  if (!p) return LBM_ERR_NOMEM;
  *out = p;
  return LBM_OK;
}

int lbm_pager_append(lbm_pager_t* pager, long long frame_idx, int is_keyframe, int* page,
                     int* special_slot) {
  if (!pager || !page || !special_slot) return LBM_ERR_INVALID;
  if (is_keyframe < 0 || is_keyframe > LBM_KEYFRAME_DEFERRED) return LBM_ERR_INVALID;
  return to_status(pager->p.append(frame_idx, is_keyframe, page, special_slot));
}

int lbm_pager_visible(const lbm_pager_t* pager, int* pages, int capacity, int* n_pages,
                      int* n_special, int* last_page_len) {
  if (!pager || !n_pages || !n_special || !last_page_len) return LBM_ERR_INVALID;
  std::vector<int> v;
  const int st = to_status(pager->p.visible(&v, n_special, last_page_len));
  if (st != LBM_OK) return st;
  *n_pages = static_cast<int>(v.size());
  if (pages) {
    if (capacity < *n_pages) return LBM_ERR_CAPACITY;
    std::copy(v.begin(), v.end(), pages);
  }
  return LBM_OK;
}

int lbm_pager_finish(lbm_pager_t* pager, int* evicted) {
  if (!pager || !evicted) return LBM_ERR_INVALID;
  return to_status(pager->p.finish(evicted));
}

int lbm_pager_commit(lbm_pager_t* pager, int keep, int* evicted) {
  if (!pager || !evicted) return LBM_ERR_INVALID;
  return to_status(pager->p.commit(keep != 0, evicted));
}

int lbm_pager_reset(lbm_pager_t* pager) {
  if (!pager) return LBM_ERR_INVALID;
  pager->p.reset();
  return LBM_OK;
}

int lbm_pager_state(const lbm_pager_t* pager, lbm_cache_state_t* state) {
  if (!pager) return LBM_ERR_INVALID;
  if (state) {
    state->device_bytes = 0;
    state->kernel_launches = 0;
  }
  return lbm::fill_state(pager->p, state);
}

void lbm_pager_destroy(lbm_pager_t* pager) { delete pager; }

}  // extern "C"
