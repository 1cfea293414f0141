// Internal structures shared by the host scheduler and the sm_100a kernel.
//
// Geometry: every sparseMode of the Ascend "sparseMode参数说明" page reduces,
// per sequence, to one closed-form interval of visible keys per query row:
//
//     row i sees key j  <=>  max(0, i + lo_off) <= j <= min(Skv-1, max(i + hi_off, prefix-1))
//
// (and, in modes 0/1 with an attenMask, the mask entry must be 0). Both ends
// are non-decreasing in i, which is what lets the scheduler skip whole
// 128x128 tiles and mask elements on boundary tiles only.
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define FA_HD __host__ __device__ __forceinline__
#else
#define FA_HD inline
#endif

namespace fa {

constexpr int kTileM = 128;       // query rows per sub-tile (one TMEM lane each)
constexpr int kTileN = 128;       // keys per KV tile
constexpr int kSubTiles = 2;      // query sub-tiles per work item (ping-pong)
constexpr int kBlockM = kTileM * kSubTiles;
constexpr int64_t kUnbounded = int64_t(1) << 30;  // "no bound" offset (|sizes| < 2^30)

enum SeqFlags : int32_t { kSeqDenseMask = 1 };

// One sequence (BNSD/BSND: the single shared shape; TND: one varlen entry).
struct SeqRec {
  int32_t q_off;    // first query token of the sequence (TND), else 0
  int32_t kv_off;   // first key token of the sequence (TND), else 0
  int32_t sq;       // query rows
  int32_t skv;      // keys
  int32_t lo_off;   // row i sees j >= i + lo_off      (-2^30: no lower bound)
  int32_t hi_off;   // row i sees j <= i + hi_off ...   (+2^30: no upper bound)
  int32_t prefix;   // ... or j <= prefix - 1 (modes 5/6), else 0
  int32_t flags;    // kSeqDenseMask: the attenMask must be read
};
static_assert(sizeof(SeqRec) == 32, "SeqRec layout");

// Work item: one (sequence, head, block of 256 query rows).
struct WorkItem {
  int32_t b;
  int32_t h;
  int32_t qblk;
  int32_t cost;  // longest-first key: lpt_key on the host, the tile sum in the device rebuild
};
static_assert(sizeof(WorkItem) == 16, "WorkItem layout");

// Paged K/V forward (decode-shaped calls): a group is (sequence, head, up
// to kPagedRows query rows); its visible keys are cut into chunks. A unit
// is one chunk of one row block of one sequence for a run of heads (one CTA
// reads whole token rows of the cache); its partial results are merged per
// group in chunk order.
constexpr int kPagedRows = 4;

struct PagedGroup {
  int32_t b, h;          // sequence, head
  int32_t row0, nrows;   // query rows [row0, row0 + nrows) of the sequence
  int32_t unit0, nunits; // its units: unit0 + c * ustride, c < nunits
  int32_t ustride;       // units between consecutive chunks of the group
  int32_t hslot;         // the head's slot in those units' partial results
};
static_assert(sizeof(PagedGroup) == 32, "PagedGroup layout");

struct PagedUnit {
  int32_t b;             // sequence
  int32_t row0, nrows;   // query rows of the sequence
  int32_t h0;            // first head (the unit covers heads h0 .. h0 + heads per unit - 1)
  int32_t key0, key1;    // keys [key0, key1) of the sequence
};
static_assert(sizeof(PagedUnit) == 24, "PagedUnit layout");

// KV tiles of one 128-row query sub-tile: [lo, hi) holds every tile with a
// visible key; tiles in [full_lo, full_hi) need no element mask.
struct TileRange {
  int32_t lo, hi, full_lo, full_hi;
};

FA_HD int64_t imin64(int64_t a, int64_t b) { return a < b ? a : b; }
FA_HD int64_t imax64(int64_t a, int64_t b) { return a > b ? a : b; }

// Last visible key of row i (before clamping to Skv-1).
FA_HD int64_t row_hi(const SeqRec& s, int64_t i) {
  return imax64(i + s.hi_off, int64_t(s.prefix) - 1);
}
// First visible key of row i (before clamping to 0).
FA_HD int64_t row_lo(const SeqRec& s, int64_t i) { return i + s.lo_off; }

// Tile range of query rows [r0, r0 + 128) of sequence s.
FA_HD TileRange tile_range(const SeqRec& s, int64_t r0) {
  TileRange t{0, 0, 0, 0};
  if (r0 >= s.sq || s.skv <= 0) return t;
  int64_t r1 = imin64(r0 + kTileM, s.sq);  // one past the last stored row
  // Rows whose clamped interval is non-empty form one run [i_first, i_last].
  int64_t i_first = (s.prefix >= 1) ? r0 : imax64(r0, -int64_t(s.hi_off));
  int64_t i_last = imin64(r1 - 1, int64_t(s.skv) - 1 - s.lo_off);
  if (i_first > i_last) return t;
  int64_t jlo = imax64(0, row_lo(s, i_first));
  int64_t jhi = imin64(int64_t(s.skv) - 1, row_hi(s, i_last));
  if (jlo > jhi) return t;
  t.lo = int32_t(jlo / kTileN);
  t.hi = int32_t(jhi / kTileN + 1);
  t.full_lo = t.full_hi = t.lo;
  if (s.flags & kSeqDenseMask) return t;
  // A tile [c0, c0+128) is FULL when every stored row sees all of it:
  // lo(r1-1) <= c0 and min(hi(r0), Skv-1) >= c0 + 127.
  int64_t need_lo = imax64(0, row_lo(s, r1 - 1));
  int64_t f_lo = (need_lo + kTileN - 1) / kTileN;
  int64_t top = imin64(row_hi(s, r0), int64_t(s.skv) - 1);
  int64_t f_hi = top < 0 ? 0 : (top + 1) / kTileN;
  f_lo = imax64(f_lo, t.lo);
  f_hi = imin64(f_hi, t.hi);
  if (f_hi > f_lo) {
    t.full_lo = int32_t(f_lo);
    t.full_hi = int32_t(f_hi);
  }
  return t;
}

}  // namespace fa
