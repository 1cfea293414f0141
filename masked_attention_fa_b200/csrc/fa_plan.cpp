// Host side of the C ABI that needs no device: argument validation, the
// per-sequence geometry decode and the tile scheduler's work list.
//
// Validation rules come from the Ascend CANN page "sparseMode参数说明":
//   sparseMode=0 (the two 说明 notes on negative nextTokens / preTokens),
//   sparseMode=4 (pre and next must intersect),
//   sparseMode=7 and sparseMode=8 (the band-piece conditions and Sq <= Skv
//   for the other batches).
#include "fa_plan.h"
#include "fa_kernel.h"

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

namespace fa {

static thread_local std::string g_last_error;

fa_status_t fail(fa_status_t st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

void clear_error() { g_last_error.clear(); }
const char* last_error() { return g_last_error.c_str(); }

static int64_t clamp_off(__int128 x) {
  if (x < -(__int128)kUnbounded) return -kUnbounded;
  if (x > (__int128)kUnbounded) return kUnbounded;
  return (int64_t)x;
}

fa_status_t validate_desc(const fa_desc_t* d) {
  if (!d) return fail(FA_ERR_NULLPTR, "desc is NULL");
  if (d->layout < FA_BNSD || d->layout > FA_TND)
    return fail(FA_ERR_PARAM_INVALID, "layout %d is not BNSD(0), BSND(1) or TND(2)", d->layout);
  if (d->sparse_mode < 0 || d->sparse_mode > 8)
    return fail(FA_ERR_PARAM_INVALID, "sparse_mode %d is outside 0..8", d->sparse_mode);
  if (d->alibi < FA_ALIBI_NONE || d->alibi > FA_ALIBI_LEFT)
    return fail(FA_ERR_PARAM_INVALID, "alibi %d is not NONE(0), RIGHT(1), SQRT(2) or LEFT(3)",
                d->alibi);
  if (d->B < 1 || d->N < 1 || d->D < 1)
    return fail(FA_ERR_SHAPE, "B, N and D must be >= 1 (got %lld, %lld, %lld)", (long long)d->B,
                (long long)d->N, (long long)d->D);
  if (d->Sq < 0 || d->Skv < 0)
    return fail(FA_ERR_SHAPE, "Sq and Skv must be >= 0 (got %lld, %lld)", (long long)d->Sq,
                (long long)d->Skv);
  if (d->Sq >= kUnbounded || d->Skv >= kUnbounded || d->B >= kUnbounded || d->N >= 65536)
    return fail(FA_ERR_UNSUPPORTED, "sizes too large (Sq, Skv, B < 2^30, N < 65536)");
  if (d->D != 64 && d->D != 128)
    return fail(FA_ERR_UNSUPPORTED, "head dim D=%lld: this build supports D in {64, 128}",
                (long long)d->D);
  // Element counts of the largest operand must stay well inside TMA's
  // 2^40-byte stride range.
  const __int128 rows_q = (d->layout == FA_TND) ? (__int128)d->Sq : (__int128)d->B * d->Sq;
  const __int128 rows_kv = (d->layout == FA_TND) ? (__int128)d->Skv : (__int128)d->B * d->Skv;
  if (std::max(rows_q, rows_kv) * d->N * d->D * 2 >= ((__int128)1 << 39))
    return fail(FA_ERR_UNSUPPORTED, "operands larger than 2^39 bytes");
  if (!(d->scale > 0.0) || !std::isfinite(d->scale))
    return fail(FA_ERR_PARAM_INVALID, "scale must be finite and > 0 (got %g)", d->scale);
  if (d->mask_kind < FA_MASK_NONE || d->mask_kind > FA_MASK_BNSS)
    return fail(FA_ERR_PARAM_INVALID, "mask_kind %d is not NONE/SS/B1SS/BNSS", d->mask_kind);
  const int m = d->sparse_mode;
  if (m >= 2 && d->mask_kind != FA_MASK_NONE)
    return fail(FA_ERR_PARAM_INVALID,
                "sparse_mode %d derives its mask from the geometry; mask_kind must be NONE", m);
  if (m == 1 && d->mask_kind == FA_MASK_NONE)
    return fail(FA_ERR_PARAM_INVALID, "sparse_mode 1 (allMask) needs a mask_kind");
  if (d->alibi != FA_ALIBI_NONE && d->mask_kind != FA_MASK_NONE)
    return fail(FA_ERR_UNSUPPORTED, "an ALiBi bias with an attenMask is not supported");
  if (d->layout == FA_TND && d->mask_kind != FA_MASK_NONE)
    return fail(FA_ERR_UNSUPPORTED, "an attenMask with the TND layout is not supported");
  if ((m == 7 || m == 8) && d->layout != FA_TND)
    return fail(FA_ERR_PARAM_INVALID, "sparse_mode %d is a varlen mode and needs layout TND", m);
  if (m == 0 && d->mask_kind != FA_MASK_NONE) {
    const int64_t pre = d->pre_tokens, nxt = d->next_tokens;
    if (nxt < 0) {
      if ((__int128)pre < -(__int128)nxt)
        return fail(FA_ERR_PARAM_INVALID,
                    "sparse_mode 0: next_tokens < 0 needs pre_tokens >= |next_tokens|");
      if (-(__int128)nxt >= d->Skv)
        return fail(FA_ERR_PARAM_INVALID, "sparse_mode 0: |next_tokens| must be < Skv");
    }
    if (pre < 0) {
      if ((__int128)nxt < -(__int128)pre)
        return fail(FA_ERR_PARAM_INVALID,
                    "sparse_mode 0: pre_tokens < 0 needs next_tokens >= |pre_tokens|");
      if (-(__int128)pre >= d->Sq)
        return fail(FA_ERR_PARAM_INVALID, "sparse_mode 0: |pre_tokens| must be < Sq");
    }
  }
  if (m == 4 && (__int128)d->pre_tokens + (__int128)d->next_tokens < 0)
    return fail(FA_ERR_PARAM_INVALID,
                "sparse_mode 4: the pre/next band must intersect (pre_tokens + next_tokens >= 0)");
  return FA_OK;
}

static void seq_extent(const fa_desc_t* d, const int64_t* cu_q, const int64_t* cu_kv, int64_t b,
                       int64_t* q_off, int64_t* kv_off, int64_t* sq, int64_t* skv) {
  if (d->layout == FA_TND) {
    *q_off = b == 0 ? 0 : cu_q[b - 1];
    *kv_off = b == 0 ? 0 : cu_kv[b - 1];
    *sq = cu_q[b] - *q_off;
    *skv = cu_kv[b] - *kv_off;
  } else {
    *q_off = *kv_off = 0;
    *sq = d->Sq;
    *skv = d->Skv;
  }
}

fa_status_t validate_call(const fa_desc_t* d, const int64_t* prefix, const int64_t* cu_q,
                          const int64_t* cu_kv, int has_mask) {
  fa_status_t st = validate_desc(d);
  if (st != FA_OK) return st;
  const int m = d->sparse_mode;
  if (m == 1 && !has_mask) return fail(FA_ERR_NULLPTR, "sparse_mode 1 (allMask) needs atten_mask");
  if (m == 0 && has_mask && d->mask_kind == FA_MASK_NONE)
    return fail(FA_ERR_PARAM_INVALID, "atten_mask given but mask_kind is NONE");
  if (d->layout == FA_TND) {
    if (!cu_q || !cu_kv)
      return fail(FA_ERR_NULLPTR, "TND needs actual_seq_qlen and actual_seq_kvlen");
    int64_t pq = 0, pk = 0;
    for (int64_t b = 0; b < d->B; ++b) {
      if (cu_q[b] < pq || cu_kv[b] < pk)
        return fail(FA_ERR_SHAPE, "actual_seq lengths must be non-decreasing cumulative ends "
                    "(entry %lld)", (long long)b);
      pq = cu_q[b];
      pk = cu_kv[b];
    }
    if (pq != d->Sq || pk != d->Skv)
      return fail(FA_ERR_SHAPE,
                  "last actual_seq_qlen/kvlen (%lld, %lld) must equal Sq/Skv (%lld, %lld)",
                  (long long)pq, (long long)pk, (long long)d->Sq, (long long)d->Skv);
  }
  if (m == 5 || m == 6) {
    if (!prefix) return fail(FA_ERR_NULLPTR, "sparse_mode %d needs the prefix array", m);
    for (int64_t b = 0; b < d->B; ++b) {
      int64_t qo, ko, sq, skv;
      seq_extent(d, cu_q, cu_kv, b, &qo, &ko, &sq, &skv);
      if (prefix[b] < 0 || prefix[b] > skv)
        return fail(FA_ERR_PARAM_INVALID, "prefix[%lld]=%lld must be in [0, Skv_b=%lld]",
                    (long long)b, (long long)prefix[b], (long long)skv);
    }
  }
  if (m == 7 || m == 8) {
    int64_t band = -1;
    for (int64_t i = 0; i < d->B; ++i) {
      int64_t b = (m == 7) ? d->B - 1 - i : i;
      int64_t qo, ko, sq, skv;
      seq_extent(d, cu_q, cu_kv, b, &qo, &ko, &sq, &skv);
      if (sq > 0) {
        band = b;
        break;
      }
    }
    if (band >= 0) {
      int64_t qo, ko, sq, skv;
      seq_extent(d, cu_q, cu_kv, band, &qo, &ko, &sq, &skv);
      const __int128 pre = d->pre_tokens, nxt = d->next_tokens;
      if (pre < skv)
        return fail(FA_ERR_PARAM_INVALID,
                    "sparse_mode %d: pre_tokens (%lld) must be >= Skv of the band sequence (%lld)",
                    m, (long long)d->pre_tokens, (long long)skv);
      if (m == 7 && (nxt > 0 || nxt < (__int128)(sq - skv)))
        return fail(FA_ERR_PARAM_INVALID,
                    "sparse_mode 7: need last_Sq - last_Skv (%lld) <= next_tokens (%lld) <= 0",
                    (long long)(sq - skv), (long long)d->next_tokens);
      if (m == 8 && nxt < (__int128)(sq - skv))
        return fail(FA_ERR_PARAM_INVALID,
                    "sparse_mode 8: need next_tokens (%lld) >= first_Sq - first_Skv (%lld)",
                    (long long)d->next_tokens, (long long)(sq - skv));
      if (m == 7) {
        for (int64_t b = 0; b < d->B; ++b) {
          if (b == band) continue;
          seq_extent(d, cu_q, cu_kv, b, &qo, &ko, &sq, &skv);
          if (sq > skv)
            return fail(FA_ERR_PARAM_INVALID,
                        "sparse_mode 7: non-band sequence %lld has Sq (%lld) > Skv (%lld)",
                        (long long)b, (long long)sq, (long long)skv);
        }
      }
    }
  }
  return FA_OK;
}

// Rows of sequence b see keys [max(0, i + lo), min(Skv-1, max(i + hi, prefix-1))].
std::vector<SeqRec> decode_geometry(const fa_desc_t* d, const int64_t* prefix,
                                    const int64_t* cu_q, const int64_t* cu_kv, int has_mask) {
  const int m = d->sparse_mode;
  const bool dense = (m == 1) || (m == 0 && has_mask);
  int64_t first_ne = -1, last_ne = -1;
  for (int64_t b = 0; b < d->B; ++b) {
    int64_t qo, ko, sq, skv;
    seq_extent(d, cu_q, cu_kv, b, &qo, &ko, &sq, &skv);
    if (sq > 0) {
      if (first_ne < 0) first_ne = b;
      last_ne = b;
    }
  }
  std::vector<SeqRec> recs((size_t)d->B);
  for (int64_t b = 0; b < d->B; ++b) {
    int64_t qo, ko, sq, skv;
    seq_extent(d, cu_q, cu_kv, b, &qo, &ko, &sq, &skv);
    const __int128 delta = (__int128)skv - sq;
    int64_t lo = -kUnbounded, hi = kUnbounded, pfx = 0;
    int rule = m;
    if (m == 7) rule = (b == last_ne) ? 4 : 3;
    if (m == 8) rule = (b == first_ne) ? 4 : 2;
    switch (rule) {
      case 0:
        if (has_mask) {  // band from the top-left, inclusive bounds
          lo = clamp_off(-(__int128)d->pre_tokens);
          hi = clamp_off((__int128)d->next_tokens);
        }
        break;
      case 1:
        break;
      case 2:  // leftUpCausal
        hi = 0;
        break;
      case 3:  // rightDownCausal
        hi = clamp_off(delta);
        break;
      case 4:  // band from the bottom-right
        lo = clamp_off(delta - d->pre_tokens);
        hi = clamp_off(delta + d->next_tokens);
        break;
      case 5:
      case 6:  // rightDownCausal plus prefix[b] leading columns
        hi = clamp_off(delta);
        pfx = prefix[b];
        break;
    }
    SeqRec& r = recs[(size_t)b];
    r.q_off = (int32_t)qo;
    r.kv_off = (int32_t)ko;
    r.sq = (int32_t)sq;
    r.skv = (int32_t)skv;
    r.lo_off = (int32_t)lo;
    r.hi_off = (int32_t)hi;
    r.prefix = (int32_t)pfx;
    r.flags = dense ? kSeqDenseMask : 0;
  }
  return recs;
}


// One item per (sequence, head, 256-row block). Items are sorted by
// descending lpt_key (longest-processing-time first), ties in index order.
std::vector<WorkItem> build_items(const fa_desc_t* d, const std::vector<SeqRec>& recs) {
  std::vector<WorkItem> items;
  for (int64_t b = 0; b < d->B; ++b) {
    const SeqRec& s = recs[(size_t)b];
    if (s.sq <= 0) continue;
    const int32_t nblk = (s.sq + kBlockM - 1) / kBlockM;
    for (int32_t qb = 0; qb < nblk; ++qb) {
      const int32_t cost = lpt_key(tile_range(s, (int64_t)qb * kBlockM),
                                   tile_range(s, (int64_t)qb * kBlockM + kTileM));
      for (int64_t h = 0; h < d->N; ++h)
        items.push_back(WorkItem{(int32_t)b, (int32_t)h, qb, cost});
    }
  }
  order_work_list(items.data(), items.data() + items.size(), false);
  return items;
}

bool claims_items(int64_t n_items, int num_sms) {
  return n_items >= (int64_t)kClaimMinItemsPerCta * num_sms && n_items < 0x7fff0000;
}

void order_work_list(WorkItem* first, WorkItem* last, bool locality) {
  // The cost key is 8 x (the longer sub-tile's key tiles) + (the
  // shorter's); 8 x kLocalityTiles of it make one bucket.
  constexpr int32_t kBucket = 8 * kLocalityTiles;
  if (!locality) {
    std::sort(first, last, [](const WorkItem& a, const WorkItem& c) {
      if (a.cost != c.cost) return a.cost > c.cost;
      if (a.b != c.b) return a.b < c.b;
      if (a.qblk != c.qblk) return a.qblk < c.qblk;
      return a.h < c.h;
    });
    return;
  }
  std::sort(first, last, [](const WorkItem& a, const WorkItem& c) {
    const bool ea = a.cost == 0, ec = c.cost == 0;  // no key tile: last
    if (ea != ec) return ec;
    const int32_t ba = a.cost / kBucket, bc = c.cost / kBucket;
    if (ba != bc) return ba > bc;
    if (a.b != c.b) return a.b < c.b;
    if (a.h != c.h) return a.h < c.h;
    if (a.cost != c.cost) return a.cost > c.cost;
    return a.qblk < c.qblk;
  });
}

fa_status_t validate_paged(const fa_desc_t* d, const int64_t* prefix, const int64_t* cu_q,
                           const int64_t* cu_kv, int64_t num_blocks, int32_t block_size,
                           int32_t max_blocks) {
  fa_status_t st = validate_call(d, prefix, cu_q, cu_kv, 0);
  if (st != FA_OK) return st;
  if (d->layout != FA_TND)
    return fail(FA_ERR_UNSUPPORTED, "paged K/V needs a TND handle (packed query tokens)");
  if (d->sparse_mode == 1 || d->mask_kind != FA_MASK_NONE)
    return fail(FA_ERR_UNSUPPORTED, "paged K/V reads no attenMask (dense-mask modes need BNSD/BSND)");
  if (d->alibi != FA_ALIBI_NONE)
    return fail(FA_ERR_UNSUPPORTED, "paged K/V does not add an ALiBi bias");
  if (block_size < 1 || block_size > (1 << 20))
    return fail(FA_ERR_PARAM_INVALID, "block_size %d outside [1, 2^20]", block_size);
  if (max_blocks < 1) return fail(FA_ERR_PARAM_INVALID, "max_blocks %d < 1", max_blocks);
  if (num_blocks < 1) return fail(FA_ERR_PARAM_INVALID, "num_blocks %lld < 1", (long long)num_blocks);
  if (num_blocks > (int64_t(1) << 40) / block_size)
    return fail(FA_ERR_PARAM_INVALID, "num_blocks * block_size beyond 2^40 tokens");
  for (int64_t b = 0; b < d->B; ++b) {
    const int64_t skv = cu_kv[b] - (b ? cu_kv[b - 1] : 0);
    if ((skv + block_size - 1) / block_size > max_blocks)
      return fail(FA_ERR_SHAPE, "sequence %lld has %lld keys: more than max_blocks (%d) blocks of %d",
                  (long long)b, (long long)skv, max_blocks, block_size);
  }
  return FA_OK;
}

// Groups in (sequence, head, row block) order; the visible key range of a
// row block is [lo(first row), hi(last row)] (the row intervals are
// monotone). Units are listed in (sequence, row block, chunk, head run)
// order; a group's chunks are therefore `runs` units apart. The chunk
// length is chosen so that all units fit in one wave of `slots` resident
// CTAs (each span adds at most one short chunk per run), which keeps every
// SM busy to the end; when there are too many spans for that, chunks of
// total / (4 slots) keys spread the work over several waves.
void build_paged(const fa_desc_t* d, const std::vector<SeqRec>& recs, int64_t slots,
                 int32_t heads_per_unit, std::vector<PagedGroup>* groups,
                 std::vector<PagedUnit>* units) {
  groups->clear();
  units->clear();
  const int64_t N = d->N;
  const int64_t runs = (N + heads_per_unit - 1) / heads_per_unit;
  struct Span { int64_t lo, hi; };
  std::vector<Span> spans;
  int64_t total = 0;  // keys over all row blocks, times head runs (per run: one unit each)
  for (const SeqRec& s : recs) {
    for (int64_t r0 = 0; r0 < s.sq; r0 += kPagedRows) {
      const int64_t r1 = imin64(r0 + kPagedRows, s.sq) - 1;
      const int64_t lo = imax64(0, row_lo(s, r0));
      const int64_t hi = imin64(int64_t(s.skv) - 1, row_hi(s, r1));
      spans.push_back(Span{lo, hi});
      if (hi >= lo) total += (hi - lo + 1) * runs;
    }
  }
  int64_t tails = 0;  // spans with keys, times runs: the most short chunks
  for (const Span& sp : spans)
    if (sp.hi >= sp.lo) tails += runs;
  slots = imax64(slots, 1);
  int64_t chunk = slots > tails ? (total + (slots - tails) - 1) / (slots - tails)
                                : (total + 4 * slots - 1) / (4 * slots);
  chunk = imax64(chunk, 64);
  size_t si = 0;
  for (size_t b = 0; b < recs.size(); ++b) {
    const SeqRec& s = recs[b];
    const int64_t nrb = (s.sq + kPagedRows - 1) / kPagedRows;
    const size_t gbase = groups->size();  // group (b, h, rb) at gbase + h * nrb + rb
    for (int64_t h = 0; h < N; ++h) {
      for (int64_t rb = 0; rb < nrb; ++rb) {
        PagedGroup g;
        g.b = (int32_t)b;
        g.h = (int32_t)h;
        g.row0 = (int32_t)(rb * kPagedRows);
        g.nrows = (int32_t)(imin64((rb + 1) * kPagedRows, s.sq) - rb * kPagedRows);
        g.unit0 = 0;
        g.nunits = 0;
        g.ustride = (int32_t)runs;
        g.hslot = (int32_t)(h % heads_per_unit);
        groups->push_back(g);
      }
    }
    for (int64_t rb = 0; rb < nrb; ++rb, ++si) {
      const Span sp = spans[si];
      const int32_t first = (int32_t)units->size();
      const int32_t row0 = (int32_t)(rb * kPagedRows);
      const int32_t nrows = (int32_t)(imin64((rb + 1) * kPagedRows, s.sq) - rb * kPagedRows);
      int32_t nchunks = 0;
      for (int64_t k0 = sp.lo; k0 <= sp.hi; k0 += chunk, ++nchunks)
        for (int64_t run = 0; run < runs; ++run)
          units->push_back(PagedUnit{(int32_t)b, row0, nrows, (int32_t)(run * heads_per_unit),
                                     (int32_t)k0, (int32_t)imin64(k0 + chunk, sp.hi + 1)});
      for (int64_t h = 0; h < N; ++h) {
        PagedGroup& g = (*groups)[gbase + h * nrb + rb];
        g.unit0 = first + (int32_t)(h / heads_per_unit);
        g.nunits = nchunks;
      }
    }
  }
}

int64_t visible_pairs(const fa_desc_t* d, const std::vector<SeqRec>& recs) {
  int64_t total = 0;
  for (const SeqRec& s : recs) {
    int64_t per_head = 0;
    for (int64_t i = 0; i < s.sq; ++i) {
      int64_t jlo = imax64(0, row_lo(s, i));
      int64_t jhi = imin64((int64_t)s.skv - 1, row_hi(s, i));
      if (jhi >= jlo) per_head += jhi - jlo + 1;
    }
    total += per_head * d->N;
  }
  return total;
}

int32_t tile_class(const SeqRec& s, int64_t qt, int64_t kt) {
  const int64_t r0 = qt * kTileM;
  if (r0 >= s.sq || kt < 0 || kt * kTileN >= s.skv) return FA_TILE_EMPTY;
  const TileRange t = tile_range(s, r0);
  if (kt < t.lo || kt >= t.hi) return FA_TILE_EMPTY;
  if (kt >= t.full_lo && kt < t.full_hi) return FA_TILE_FULL;
  return FA_TILE_PARTIAL;
}


// Query split across devices: see fa_split_queries in fa.h. The unsplit job
// is TND in mode 2 or 3; a part keeps every key of the sequences it touches.
static int64_t row_cost(int mode, int64_t i, int64_t sq, int64_t skv) {
  // visible keys of row i: mode 3 sees j <= i + (skv - sq), mode 2 sees j <= i
  const int64_t hi = (mode == 3) ? i + (skv - sq) : i;
  return imax64(0, imin64(hi + 1, skv));
}

fa_status_t split_queries(const fa_desc_t* d, const int64_t* cu_q, const int64_t* cu_kv,
                          int32_t n_parts, const int64_t* cuts, int32_t part,
                          fa_split_part_t* out, int64_t* oq, int64_t* okv) {
  if (!out || !oq || !okv) return fail(FA_ERR_NULLPTR, "out arrays are required");
  fa_status_t st = validate_call(d, nullptr, cu_q, cu_kv, 0);
  if (st != FA_OK) return st;
  if (d->layout != FA_TND || (d->sparse_mode != 2 && d->sparse_mode != 3))
    return fail(FA_ERR_UNSUPPORTED, "query split needs a TND job in sparse_mode 2 or 3");
  if (n_parts < 1 || part < 0 || part >= n_parts)
    return fail(FA_ERR_PARAM_INVALID, "part %d of %d parts", part, n_parts);
  const int mode = d->sparse_mode;
  const int64_t T = d->Sq;
  auto seq = [&](int64_t b, int64_t* qo, int64_t* ko, int64_t* sq, int64_t* skv) {
    *qo = b ? cu_q[b - 1] : 0;
    *ko = b ? cu_kv[b - 1] : 0;
    *sq = cu_q[b] - *qo;
    *skv = cu_kv[b] - *ko;
  };
  if (mode == 3) {
    for (int64_t b = 0; b < d->B; ++b) {
      int64_t qo, ko, sq, skv;
      seq(b, &qo, &ko, &sq, &skv);
      if (sq > skv)
        return fail(FA_ERR_UNSUPPORTED,
                    "splitting a rightDownCausal job needs Sq_b <= Skv_b (sequence %lld)",
                    (long long)b);
    }
  }
  // The part's query tokens [a, e).
  int64_t a = 0, e = T;
  if (cuts) {
    int64_t prev = 0;
    for (int32_t k = 0; k + 1 < n_parts; ++k) {
      if (cuts[k] < prev || cuts[k] > T)
        return fail(FA_ERR_PARAM_INVALID, "cuts must be increasing positions in [0, T_q]");
      prev = cuts[k];
    }
    a = part ? cuts[part - 1] : 0;
    e = part + 1 < n_parts ? cuts[part] : T;
  } else {
    // Balance the visible pairs: cut where the running cost crosses k/n of it.
    int64_t total = 0;
    for (int64_t b = 0; b < d->B; ++b) {
      int64_t qo, ko, sq, skv;
      seq(b, &qo, &ko, &sq, &skv);
      for (int64_t i = 0; i < sq; ++i) total += row_cost(mode, i, sq, skv);
    }
    auto cut_at = [&](int32_t k) -> int64_t {  // first token whose prefix cost >= k/n of total
      if (k <= 0) return 0;
      if (k >= n_parts) return T;
      const __int128 target = (__int128)total * k;
      __int128 run = 0;
      for (int64_t b = 0; b < d->B; ++b) {
        int64_t qo, ko, sq, skv;
        seq(b, &qo, &ko, &sq, &skv);
        for (int64_t i = 0; i < sq; ++i) {
          if (run * n_parts >= target) return qo + i;
          run += row_cost(mode, i, sq, skv);
        }
      }
      return T;
    };
    a = cut_at(part);
    e = cut_at(part + 1);
  }
  std::memset(out, 0, sizeof(*out));
  out->desc = *d;
  out->desc.sparse_mode = mode;
  out->desc.pre_tokens = 0;
  out->desc.next_tokens = 0;
  out->q_begin = a;
  out->q_end = e;
  if (a >= e) {  // empty part
    out->desc.B = 1;
    out->desc.Sq = out->desc.Skv = 0;
    out->kv_begin = out->kv_end = 0;
    oq[0] = okv[0] = 0;
    return FA_OK;
  }
  int64_t b0 = 0;
  while (cu_q[b0] <= a) ++b0;  // sequence holding token a
  int64_t b1 = b0;
  while (cu_q[b1] < e) ++b1;   // sequence holding token e - 1
  int64_t qo0, ko0, sq0, skv0, qo1, ko1, sq1, skv1;
  seq(b0, &qo0, &ko0, &sq0, &skv0);
  seq(b1, &qo1, &ko1, &sq1, &skv1);
  int64_t nq = 0, nk = 0;
  for (int64_t b = b0; b <= b1; ++b) {
    int64_t qo, ko, sq, skv;
    seq(b, &qo, &ko, &sq, &skv);
    const int64_t r0 = imax64(a, qo) - qo, r1 = imin64(e, qo + sq) - qo;
    nq += imax64(0, r1 - r0);
    nk += skv;
    oq[b - b0] = nq;
    okv[b - b0] = nk;
  }
  out->desc.B = b1 - b0 + 1;
  out->desc.Sq = nq;
  out->desc.Skv = nk;
  out->kv_begin = ko0;
  out->kv_end = ko1 + skv1;
  const int64_t c0 = a - qo0;             // first kept row of sequence b0
  const int64_t c1 = imin64(e, qo1 + sq1) - qo1;  // one past the last kept row of b1
  if (mode == 3 && c1 < sq1) {
    // The last sequence keeps rows [.., c1) of a rightDownCausal block: a band
    // anchored at the bottom-right with next = c1 - Sq_b, pre = Skv_b.
    out->desc.sparse_mode = 7;
    out->desc.pre_tokens = skv1;
    out->desc.next_tokens = c1 - sq1;
  } else if (mode == 2 && c0 > 0) {
    // The first sequence keeps rows [c0, ..) of a leftUpCausal block: a band
    // with next = (last kept row + 1) - Skv_b, pre = Skv_b.
    const int64_t c0_end = (b0 == b1) ? c1 : sq0;
    out->desc.sparse_mode = 8;
    out->desc.pre_tokens = skv0;
    out->desc.next_tokens = c0_end - skv0;
  }
  return validate_call(&out->desc, nullptr, oq, okv, 0);
}

}  // namespace fa

using namespace fa;

extern "C" {

const char* fa_last_error(void) { return last_error(); }

int32_t fa_version(void) { return FA_VERSION; }

fa_status_t fa_validate(const fa_desc_t* desc, const int64_t* prefix,
                        const int64_t* actual_seq_qlen, const int64_t* actual_seq_kvlen,
                        int32_t has_mask) {
  clear_error();
  return validate_call(desc, prefix, actual_seq_qlen, actual_seq_kvlen, has_mask);
}

fa_status_t fa_visible_pairs(const fa_desc_t* desc, const int64_t* prefix,
                             const int64_t* actual_seq_qlen, const int64_t* actual_seq_kvlen,
                             int32_t has_mask, int64_t* pairs_out) {
  clear_error();
  if (!pairs_out) return fail(FA_ERR_NULLPTR, "pairs_out is NULL");
  fa_status_t st = validate_call(desc, prefix, actual_seq_qlen, actual_seq_kvlen, has_mask);
  if (st != FA_OK) return st;
  if (desc->sparse_mode == 1 || (desc->sparse_mode == 0 && has_mask))
    return fail(FA_ERR_UNSUPPORTED, "visible pairs of a dense-mask call depend on the mask data");
  auto recs = decode_geometry(desc, prefix, actual_seq_qlen, actual_seq_kvlen, has_mask);
  *pairs_out = visible_pairs(desc, recs);
  return FA_OK;
}

int32_t fa_tile_class(const fa_desc_t* desc, const int64_t* prefix,
                      const int64_t* actual_seq_qlen, const int64_t* actual_seq_kvlen,
                      int32_t has_mask, int64_t b, int64_t qt, int64_t kt) {
  clear_error();
  if (validate_call(desc, prefix, actual_seq_qlen, actual_seq_kvlen, has_mask) != FA_OK) return -1;
  if (b < 0 || b >= desc->B || qt < 0) {
    fail(FA_ERR_PARAM_INVALID, "tile index out of range");
    return -1;
  }
  auto recs = decode_geometry(desc, prefix, actual_seq_qlen, actual_seq_kvlen, has_mask);
  return tile_class(recs[(size_t)b], qt, kt);
}

fa_status_t fa_split_queries(const fa_desc_t* desc, const int64_t* actual_seq_qlen,
                             const int64_t* actual_seq_kvlen, int32_t n_parts,
                             const int64_t* cuts, int32_t part, fa_split_part_t* out,
                             int64_t* out_seq_qlen, int64_t* out_seq_kvlen) {
  clear_error();
  return split_queries(desc, actual_seq_qlen, actual_seq_kvlen, n_parts, cuts, part, out,
                       out_seq_qlen, out_seq_kvlen);
}

fa_status_t fa_plan_stats(const fa_desc_t* desc, const int64_t* prefix,
                          const int64_t* actual_seq_qlen, const int64_t* actual_seq_kvlen,
                          int32_t has_mask, int64_t* out) {
  clear_error();
  if (!out) return fail(FA_ERR_NULLPTR, "out is NULL");
  fa_status_t st = validate_call(desc, prefix, actual_seq_qlen, actual_seq_kvlen, has_mask);
  if (st != FA_OK) return st;
  auto recs = decode_geometry(desc, prefix, actual_seq_qlen, actual_seq_kvlen, has_mask);
  auto items = build_items(desc, recs);
  int64_t counts[3] = {0, 0, 0};
  for (const SeqRec& s : recs) {
    const int64_t nqt = (s.sq + kTileM - 1) / kTileM;
    const int64_t nkt = (s.skv + kTileN - 1) / kTileN;
    for (int64_t qt = 0; qt < nqt; ++qt) {
      const TileRange t = tile_range(s, qt * kTileM);
      const int64_t nonempty = t.hi - t.lo;
      const int64_t full = t.full_hi - t.full_lo;
      counts[FA_TILE_FULL] += full * desc->N;
      counts[FA_TILE_PARTIAL] += (nonempty - full) * desc->N;
      counts[FA_TILE_EMPTY] += (nkt - nonempty) * desc->N;
    }
  }
  out[0] = (int64_t)items.size();
  out[1] = counts[FA_TILE_EMPTY];
  out[2] = counts[FA_TILE_PARTIAL];
  out[3] = counts[FA_TILE_FULL];
  return FA_OK;
}

fa_status_t fa_plan_items(const fa_desc_t* desc, const int64_t* prefix,
                          const int64_t* actual_seq_qlen, const int64_t* actual_seq_kvlen,
                          int32_t num_sms, int64_t capacity, int32_t* out, int64_t* n_items) {
  clear_error();
  if (!n_items) return fail(FA_ERR_NULLPTR, "n_items is NULL");
  if (capacity < 0) return fail(FA_ERR_PARAM_INVALID, "capacity %lld < 0", (long long)capacity);
  if (capacity > 0 && !out) return fail(FA_ERR_NULLPTR, "out is NULL");
  if (num_sms < 1) return fail(FA_ERR_PARAM_INVALID, "num_sms %d < 1", num_sms);
  fa_status_t st = validate_call(desc, prefix, actual_seq_qlen, actual_seq_kvlen, 0);
  if (st != FA_OK) return st;
  auto recs = decode_geometry(desc, prefix, actual_seq_qlen, actual_seq_kvlen, 0);
  auto items = build_items(desc, recs);
  if (claims_items((int64_t)items.size(), num_sms))
    order_work_list(items.data(), items.data() + items.size(), true);
  *n_items = (int64_t)items.size();
  if ((int64_t)items.size() > capacity)
    return fail(FA_ERR_SHAPE, "the work list has %zu items, capacity %lld", items.size(),
                (long long)capacity);
  for (size_t m = 0; m < items.size(); ++m) {
    out[4 * m] = items[m].b;
    out[4 * m + 1] = items[m].h;
    out[4 * m + 2] = items[m].qblk;
    out[4 * m + 3] = items[m].cost;
  }
  return FA_OK;
}

}  // extern "C"
