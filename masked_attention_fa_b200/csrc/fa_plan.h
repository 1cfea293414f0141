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
std::vector<WorkItem> build_items(const fa_desc_t* d, const std::vector<SeqRec>& recs);
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
