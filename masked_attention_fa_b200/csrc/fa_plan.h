// Host-only planning interface (validation, geometry decode, work list).
#pragma once

#include <vector>

#include "../../include/fa.h"
#include "fa_internal.h"

namespace fa {

fa_status_t fail(fa_status_t st, const char* fmt, ...);
void clear_error();
const char* last_error();

fa_status_t validate_desc(const fa_desc_t* d);
fa_status_t validate_call(const fa_desc_t* d, const int64_t* prefix, const int64_t* cu_q,
                          const int64_t* cu_kv, int has_mask);
std::vector<SeqRec> decode_geometry(const fa_desc_t* d, const int64_t* prefix,
                                    const int64_t* cu_q, const int64_t* cu_kv, int has_mask);
// Longest-first key of a work item from its two sub-tiles' key-tile ranges,
// in eighths of a kernel step. One step runs both sub-tiles on one key tile,
// so an item takes about as many steps as its longer sub-tile has tiles; the
// shorter sub-tile adds about an eighth of a step per tile (measured on
// B200: ~1.9 us per step of the longer one, ~0.2 us per tile of the shorter).
// An item whose second sub-tile is empty therefore costs nearly as much as a
// full one of the same length, not half.
inline int32_t lpt_key(const TileRange& a, const TileRange& b) {
  const int32_t ta = a.hi > a.lo ? a.hi - a.lo : 0;
  const int32_t tb = b.hi > b.lo ? b.hi - b.lo : 0;
  return ta > tb ? 8 * ta + tb : 8 * tb + ta;
}
std::vector<WorkItem> build_items(const fa_desc_t* d, const std::vector<SeqRec>& recs);
// Whether a closed-form list of n_items is claimed at run time on num_sms
// SMs (the kernel's claiming instance, at least kClaimMinItemsPerCta items
// per SM).
bool claims_items(int64_t n_items, int num_sms);
// Orders a closed-form work list in place, allocating nothing. Strict
// longest first (ties in (sequence, block, head) order) for lists each CTA
// takes a fixed share of; for claimed lists (locality = true), longest
// first by buckets of kLocalityTiles key tiles, and inside a bucket the
// items of one (sequence, head) together, so that the CTAs claiming
// consecutive items read the same K/V tiles at about the same time and
// share them through L2 (with strict order the ~148 items in flight come
// from as many (sequence, head) pairs, whose K/V outgrow L2 and are read
// from DRAM by every item: 3.7x the algorithmic bytes on a causal-prefix
// problem of 8k tokens, 4.5x on 16 varlen sequences). Items without a key
// tile come last either way (claiming relies on it). On those two problems
// buckets of 24 tiles measured 1-1.3 % faster than 16 (8: 2.5-4 % slower;
// 64: the 16 sequences +3 %, the 8k-token problem -2 %).
constexpr int32_t kLocalityTiles = 24;
void order_work_list(WorkItem* first, WorkItem* last, bool locality);
int64_t visible_pairs(const fa_desc_t* d, const std::vector<SeqRec>& recs);
int32_t tile_class(const SeqRec& s, int64_t qt, int64_t kt);

// Paged K/V calls: the extra checks (TND, no dense mask, block geometry) and
// the group / unit lists.
fa_status_t validate_paged(const fa_desc_t* d, const int64_t* prefix, const int64_t* cu_q,
                           const int64_t* cu_kv, int64_t num_blocks, int32_t block_size,
                           int32_t max_blocks);
// slots: CTAs of the partial kernel resident at once; heads_per_unit: heads
// one unit (CTA) covers.
void build_paged(const fa_desc_t* d, const std::vector<SeqRec>& recs, int64_t slots,
                 int32_t heads_per_unit, std::vector<PagedGroup>* groups,
                 std::vector<PagedUnit>* units);

}  // namespace fa
