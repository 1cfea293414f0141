/*
 * fa.h — C ABI of the B200 (sm_100a) masked attention forward.
 *
 *   O = softmax(scale * Q K^T masked by the sparseMode geometry) V
 *
 * computed tile by tile with an online softmax (running row max m_i and
 * running row sum l_i), never materialising the Sq x Skv score matrix.
 * Operation: the "FlashAttention tiling & online softmax" exercise page
 * (section "Mục tiêu kiến thức": running maximum m_i, running sum l_i).
 * Mask geometry: the Ascend CANN page "sparseMode参数说明", sections
 * sparseMode=0 .. sparseMode=8, and its attenMask rule (a True entry hides
 * the QK^T position).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Two stages, as the aclnnScatterPaKvCache page's host flow does: a
 *    descriptor is validated and turned into a handle once (fa_create),
 *    then the handle runs calls on a caller-supplied CUDA stream (fa_fwd).
 *  - All validation happens on the host before any device work; a call that
 *    returns a non-OK status has touched no output and enqueued nothing.
 *    fa_last_error() then returns a message for the calling thread.
 *  - Status codes follow the null-pointer / invalid-parameter split of the
 *    aclnnScatterPaKvCache page's "返回值" table.
 *  - Results are bitwise deterministic: every output row is produced by one
 *    CTA, visiting its key tiles in a fixed order (no split-K atomics), as
 *    the aclnnScatterPaKvCache page's "确定性计算" note asks of that op.
 *  - A handle is not thread-safe; distinct handles are independent. The
 *    calls of one handle must not overlap on the GPU (enqueue them on one
 *    stream, or order them with events): they share its device workspace,
 *    including the counter from which long work lists are claimed.
 */
#ifndef FA_B200_FA_H
#define FA_B200_FA_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FA_VERSION 1

typedef struct fa_handle_s* fa_handle_t;

/* Memory layouts of Q, K, V and O (bf16, dense, innermost dimension D):
 *   FA_BNSD  Q/O [B, N, Sq, D],  K/V [B, N, Skv, D]
 *   FA_BSND  Q/O [B, Sq, N, D],  K/V [B, Skv, N, D]
 *   FA_TND   Q/O [T_q, N, D],    K/V [T_kv, N, D]  (varlen, packed tokens)
 * lse is fp32 [B, N, Sq] for BNSD/BSND and [N, T_q] for TND. */
typedef enum { FA_BNSD = 0, FA_BSND = 1, FA_TND = 2 } fa_layout_t;

/* Shapes of the optional attenMask (uint8, nonzero = masked), read only in
 * sparseMode 0 and 1:  SS [Sq, Skv], B1SS [B, 1, Sq, Skv], BNSS [B, N, Sq, Skv]. */
typedef enum {
    FA_MASK_NONE = 0,
    FA_MASK_SS = 1,
    FA_MASK_B1SS = 2,
    FA_MASK_BNSS = 3
} fa_mask_kind_t;

typedef enum {
    FA_OK = 0,
    FA_ERR_NULLPTR = 1,        /* a required pointer is NULL */
    FA_ERR_PARAM_INVALID = 2,  /* a value breaks a documented constraint */
    FA_ERR_SHAPE = 3,          /* sizes or length arrays are inconsistent */
    FA_ERR_UNSUPPORTED = 4,    /* valid request outside this build (e.g. D) */
    FA_ERR_ALLOC = 5,          /* host or device allocation failed */
    FA_ERR_CUDA = 6,           /* a CUDA runtime call failed */
    FA_ERR_TIMEOUT = 7,        /* a device-side wait gave up (kernel aborted) */
    FA_ERR_DEVICE = 8          /* the kernel reported an internal error */
} fa_status_t;

/* ALiBi bias added to the scores (the Ascend ATB page "压缩mask", alibi
 * section: the alibi mask is a per-head coefficient, slopes[h], times an
 * alibi bias, plus the triangular mask, in a right-aligned, a square-root and
 * a left-aligned variant). The page's formula is lost; the reading taken, with
 * delta_b = Skv_b - Sq_b and positions inside the sequence:
 *   FA_ALIBI_RIGHT  bias(i, j) = j - (i + delta_b): the key's signed distance
 *                   from the row's diagonal anchored at the bottom-right
 *                   corner (0 on it, negative to its left);
 *   FA_ALIBI_SQRT   the square root of that distance's size, sign kept;
 *   FA_ALIBI_LEFT   bias(i, j) = j (a constant per row away from RIGHT: the
 *                   same O, lse larger by slopes[h] * (i + delta_b)).
 * The score of a visible pair is scale * q.k + slopes[h] * bias(i, j); the
 * visibility rule is the sparseMode geometry, unchanged. */
typedef enum {
    FA_ALIBI_NONE = 0,
    FA_ALIBI_RIGHT = 1,
    FA_ALIBI_SQRT = 2,
    FA_ALIBI_LEFT = 3
} fa_alibi_t;

/* Problem descriptor. For FA_TND, B is the number of sequences and Sq / Skv
 * are the token totals T_q / T_kv. */
typedef struct {
    int32_t layout;        /* fa_layout_t */
    int32_t sparse_mode;   /* 0..8 */
    int32_t mask_kind;     /* fa_mask_kind_t; must be NONE unless mode 0/1 */
    int32_t alibi;         /* fa_alibi_t; FA_ALIBI_NONE (0) unless the call is fa_fwd_alibi */
    int64_t B, N, Sq, Skv, D;
    int64_t pre_tokens;    /* preTokens  (modes 0, 4, 7, 8; ignored otherwise) */
    int64_t next_tokens;   /* nextTokens (modes 0, 4, 7, 8; ignored otherwise) */
    double scale;          /* multiplies q.k before the softmax; > 0, finite */
} fa_desc_t;

/*
 * fa_create — validate the static part of a descriptor and make a handle.
 *
 * desc: host pointer, read during the call only. out: receives the handle.
 * Constraints checked here (the rest needs the per-call arrays, see fa_fwd):
 *   layout in {BNSD, BSND, TND}; sparse_mode in 0..8; B, N, D >= 1;
 *   Sq, Skv >= 0 and < 2^30; D in {64, 128} (FA_ERR_UNSUPPORTED otherwise);
 *   scale finite and > 0; mask_kind is NONE for modes 2..8; mode 1 needs a
 *   mask kind; a mask with TND is FA_ERR_UNSUPPORTED (the sparseMode page
 *   gives no TND mask shape); modes 7 and 8 need TND; in mode 0 with a mask,
 *   next < 0 needs pre >= |next| and |next| < Skv, pre < 0 needs
 *   next >= |pre| and |pre| < Sq (sparseMode=0 section, the two 说明 notes);
 *   in mode 4 the band must intersect: pre + next >= 0 (sparseMode=4);
 *   alibi in 0..3, and an ALiBi bias only without an attenMask (mask_kind
 *   NONE; FA_ERR_UNSUPPORTED otherwise).
 * Ownership: the handle owns a small device workspace (work list, counters,
 * error word) and a pinned staging buffer, released by fa_destroy. The
 * workspace is allocated on the current device at the first fa_fwd.
 */
fa_status_t fa_create(const fa_desc_t* desc, fa_handle_t* out);

/*
 * fa_fwd — enqueue one masked attention forward on `cuda_stream`.
 *
 * q, k, v      device, bf16, dense in the handle's layout; 16-byte aligned.
 * atten_mask   device uint8 in the handle's mask_kind shape, nonzero =
 *              masked; read in modes 0 and 1 only (NULL in mode 0 means
 *              "no mask": nothing is masked and pre/next are ignored, as the
 *              sparseMode=0 section states). Ignored for modes 2..8.
 * prefix       host int64[B]; modes 5/6 only: prefix[b] leading key columns
 *              are visible to every query row of batch b; 0 <= prefix[b] <=
 *              Skv_b.
 * actual_seq_qlen, actual_seq_kvlen
 *              host int64[B], TND only: cumulative end offsets without a
 *              leading 0 ({3,5} means lengths 3 and 2), non-decreasing, last
 *              entries equal to Sq and Skv of the descriptor.
 * o            device bf16, same layout and shape as q.
 * lse          device fp32, natural-log sum of exp(scale q.k) over the
 *              visible keys of each row; -inf (and O = 0) for a row with no
 *              visible key.
 * cuda_stream  a cudaStream_t (NULL = legacy default stream).
 *
 * Per-call constraints (sparseMode=7/8 sections): mode 7 needs, for the last
 * sequence with Sq_b > 0: pre >= Skv_b and Sq_b - Skv_b <= next <= 0, and
 * Sq_b <= Skv_b for every other sequence; mode 8 needs, for the first
 * sequence with Sq_b > 0: pre >= Skv_b and next >= Sq_b - Skv_b. Violations
 * return FA_ERR_PARAM_INVALID before any device work.
 *
 * Dense masks (mode 1, or mode 0 with atten_mask): the call first runs the
 * occupancy pre-pass of fa_mask_occupancy into the handle's workspace (two
 * small kernels on the same stream), so that key tiles the mask hides
 * entirely are skipped and tiles it leaves entirely visible are computed
 * without reading it, then a one-block kernel that rebuilds the work list
 * from the pre-pass's ranges, longest item first by its real number of key
 * tiles; fa_fwd_with_ranges skips the pre-pass but not the rebuild.
 *
 * Work distribution: items (sequence, head, 256 query rows) are sorted
 * longest first. A closed-form call whose list holds at least 8 items per
 * SM lets each CTA claim its next item from a counter in the workspace
 * while it loads its current one (the last CTA resets it), with the list
 * grouped by (sequence, head) inside buckets of similar length so that the
 * items in flight share K/V through L2 (see fa_plan_items); otherwise each
 * CTA takes a fixed share. Every output row is produced by one CTA either
 * way, so results do not depend on which CTA computed them.
 *
 * Asynchronous: returns once the kernel is enqueued. The host arrays are
 * read during the call only. Device-side problems (a wait that gave up) are
 * reported by fa_sync_status. The device must be sm_100 (B200 class);
 * otherwise FA_ERR_UNSUPPORTED.
 */
fa_status_t fa_fwd(fa_handle_t h, const void* q, const void* k, const void* v,
                   const uint8_t* atten_mask, const int64_t* prefix,
                   const int64_t* actual_seq_qlen, const int64_t* actual_seq_kvlen,
                   void* o, float* lse, void* cuda_stream);

/*
 * fa_fwd_alibi — fa_fwd for a handle whose descriptor names an ALiBi
 * variant (alibi != FA_ALIBI_NONE): every visible score gets
 * slopes[h] * bias(i, j) added before the softmax (see fa_alibi_t).
 *
 * slopes  device fp32 [N], 4-byte aligned, finite; read by the kernel.
 * The other arguments and the asynchronous behaviour are fa_fwd's. Errors:
 * FA_ERR_NULLPTR (NULL slopes), FA_ERR_PARAM_INVALID (a handle without an
 * ALiBi variant, unaligned slopes), and fa_fwd's. fa_fwd on an ALiBi handle
 * returns FA_ERR_PARAM_INVALID (it has no slopes). The lse is fp32: in the
 * left-aligned variant it grows like slopes[h] * (i + delta_b), and its
 * absolute rounding error with it.
 */
fa_status_t fa_fwd_alibi(fa_handle_t h, const void* q, const void* k, const void* v,
                         const float* slopes, const int64_t* prefix,
                         const int64_t* actual_seq_qlen, const int64_t* actual_seq_kvlen,
                         void* o, float* lse, void* cuda_stream);

/* fa_sync_status — wait for the handle's last call and read its device error
 * word: FA_OK, FA_ERR_TIMEOUT (a bounded wait in the kernel gave up, its
 * outputs are undefined) or FA_ERR_DEVICE. The error word is cleared. */
fa_status_t fa_sync_status(fa_handle_t h);

/* fa_destroy — wait for the handle's work and free everything it owns.
 * NULL is accepted. */
fa_status_t fa_destroy(fa_handle_t h);

/* Message of the calling thread's last non-OK status ("" if none). Valid
 * until the thread's next fa_* call. */
const char* fa_last_error(void);

/* Library version (FA_VERSION). */
int32_t fa_version(void);

/*
 * fa_fwd_noalloc — the same forward as fa_fwd for callers that cannot
 * allocate memory (for example code running inside a framework that owns
 * every device allocation through its own pool, a real-time loop that must
 * not allocate after start-up, or a plugin called from another library's
 * memory callbacks). The pages have no counterpart of this entry point.
 *
 * No handle: the descriptor and all arrays are passed on every call, with
 * the meaning, layout and validation of fa_create + fa_fwd. A descriptor
 * with an ALiBi variant is FA_ERR_UNSUPPORTED here (there are no slopes). The work list
 * and the error word live in one fixed device array of 1 MiB per device,
 * held from library load until process exit, instead of a cudaMalloc'd
 * workspace: the call makes no cudaMalloc, cudaFree or pinned allocation.
 * Capacity: 256 + 32 * B (rounded up to 256) + 16 * items bytes, where items
 * = N * sum over sequences of ceil(Sq_b / 256); a problem beyond 1 MiB returns
 * FA_ERR_UNSUPPORTED before any device work (use fa_create/fa_fwd then).
 * A dense-mask call puts each item's two key-tile ranges (32 bytes per item,
 * rounded up to 256) and the occupancy pre-pass's scratch (16 bytes per mask
 * plane and 128-row query block, rounded up to 256, plus 1 byte per plane
 * and 128 x 128 tile) behind the work list when they fit; when they do not,
 * the call runs without the pre-pass (every tile of the band with the
 * element mask) and gives the same result.
 * A closed-form call puts each item's two key-tile ranges behind the list
 * when they fit, and then, with at least 8 items per SM, claims its items
 * through two counters in the array's 256-byte header, cleared with the
 * error word (see fa_fwd, work distribution).
 * Sharing: every call shares the array and leaves its work list there; the
 * header (error word and claim counters) is cleared at the start of each
 * call. Calls whose kernels
 * overlap on the GPU race on the array: order them on one stream. Host calls
 * are serialised internally.
 * Set-up: the first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) and the device's attributes with that device
 * current; make that first call before any stream capture begins.
 * Graphs: calls cannot be captured into a CUDA graph. Each call uploads its
 * work list from one static host buffer that the next call overwrites, so a
 * replay would read another call's list; a call on a capturing stream
 * returns FA_ERR_UNSUPPORTED and enqueues nothing.
 * Device-side failures: a bounded wait in the kernel that gives up leaves
 * the outputs undefined and sets an error word in the array's header, which
 * fa_noalloc_sync_status reports. Each call clears the header first, so the
 * word describes the most recent call.
 */
fa_status_t fa_fwd_noalloc(const fa_desc_t* desc, const void* q, const void* k, const void* v,
                           const uint8_t* atten_mask, const int64_t* prefix,
                           const int64_t* actual_seq_qlen, const int64_t* actual_seq_kvlen,
                           void* o, float* lse, void* cuda_stream);

/*
 * fa_noalloc_sync_status — the fa_sync_status of the allocation-free entry
 * point (which has no handle to hold its status). The pages have no
 * counterpart of it.
 *
 * Waits for `cuda_stream` (the stream of the last fa_fwd_noalloc call on
 * the current device), then reads the error word in the fixed array's
 * header: FA_OK, FA_ERR_TIMEOUT (a bounded wait in the kernel gave up; that
 * call's O and lse are undefined) or FA_ERR_DEVICE. A non-zero word is
 * cleared, with the rest of the header. Allocates nothing (the word is read
 * into a static host variable). FA_OK when no call has run on the device.
 * Errors: FA_ERR_CUDA if the synchronisation or the read fails (for example
 * after a fault that ended the CUDA context).
 */
fa_status_t fa_noalloc_sync_status(void* cuda_stream);

/*
 * fa_fwd_paged — forward of a TND handle with the keys and values read from
 * paged caches instead of packed tensors, for decode-shaped calls (a few
 * query rows per sequence against a long cached context).
 *
 * Cache layout: the "Norm" cache of the aclnnScatterPaKvCache page
 * (scenario 2): k_cache and v_cache are device bf16 [num_blocks, block_size,
 * N, D], a token written at slot s sitting in block s / block_size at offset
 * s % block_size. Key j of sequence b is in block block_table[b][j /
 * block_size] at offset j % block_size.
 * q, o         device bf16 [T_q, N, D] (the handle's Sq = T_q), 16-byte aligned.
 * lse          device fp32 [N, T_q], 4-byte aligned.
 * block_table  device int32 [B, max_blocks], 4-byte aligned; only the first
 *              ceil(Skv_b / block_size) entries of row b are read. An entry
 *              outside [0, num_blocks) is not dereferenced: its keys are
 *              left out and fa_sync_status reports FA_ERR_DEVICE.
 * actual_seq_qlen, actual_seq_kvlen
 *              host int64[B], cumulative as in fa_fwd: query rows per
 *              sequence and cached keys per sequence (the handle's Skv =
 *              the last kvlen entry).
 * prefix       host int64[B] for modes 5/6, else ignored.
 * Visibility: the handle's sparseMode row intervals per sequence (modes 0
 * without a mask, 2..8), exactly as fa_fwd applies them to TND.
 * Constraints (FA_ERR_* before any device work): a TND handle with no mask
 * kind, no ALiBi variant and sparse_mode != 1; 1 <= block_size <= 2^20; num_blocks >= 1;
 * ceil(Skv_b / block_size) <= max_blocks for every b.
 * The work is split over the keys (units of one sequence, one head, up to 4
 * query rows and one chunk of keys) and each row's chunks are merged in a
 * fixed order, so results are bitwise deterministic. Asynchronous, on
 * cuda_stream; the handle's workspace holds the work list and the partial
 * results.
 */
fa_status_t fa_fwd_paged(fa_handle_t h, const void* q, const void* k_cache, const void* v_cache,
                         const int32_t* block_table, int64_t num_blocks, int32_t block_size,
                         int32_t max_blocks, const int64_t* prefix, const int64_t* actual_seq_qlen,
                         const int64_t* actual_seq_kvlen, void* o, float* lse, void* cuda_stream);

/*
 * fa_mask_occupancy — the dense-mask pre-pass that fa_fwd and
 * fa_fwd_noalloc run before the attention kernel in sparseMode 1 (allMask)
 * and in sparseMode 0 with an attenMask ("sparseMode参数说明" page,
 * sparseMode=0 and sparseMode=1 sections: the operator computes the pairs
 * the mask leaves visible, in mode 0 only those inside the preTokens /
 * nextTokens band), enqueued on its own on `cuda_stream`.
 *
 * The mask has P planes of Sq x Skv bytes (SS: P = 1, B1SS: P = B, BNSS:
 * P = B * N; nonzero = masked). For plane p, query rows [128 qt, 128 qt + 128)
 * and keys [128 kt, 128 kt + 128), a pair (i, j) is visible when i < Sq,
 * j < Skv, the mode's band admits it and the mask byte is 0. Outputs:
 * tile_class  device uint8 [P, ceil(Sq/128), ceil(Skv/128)]:
 *             FA_TILE_EMPTY (no visible pair), FA_TILE_FULL (every row
 *             i < Sq of the tile sees all 128 keys, each < Skv) or
 *             FA_TILE_PARTIAL.
 * ranges      device int32 [P, ceil(Sq/128), 4], 16-byte aligned: per query
 *             sub-tile {lo, hi, full_lo, full_hi}: [lo, hi) runs from the
 *             first to the last non-EMPTY tile ({0, 0, 0, 0} when all are
 *             EMPTY) and [full_lo, full_hi) is the longest run of FULL tiles,
 *             the first one on ties (full_lo = full_hi = lo when there is
 *             none). fa_fwd visits the tiles of [lo, hi) and applies the
 *             element mask outside [full_lo, full_hi).
 * desc        layout BNSD or BSND, sparse_mode 0 or 1 with a mask_kind;
 *             the other checks are fa_create's. atten_mask: device, in the
 *             mask_kind shape. All buffers belong to the caller.
 * Errors: FA_ERR_NULLPTR, FA_ERR_PARAM_INVALID (other modes, no mask kind,
 * unaligned ranges), FA_ERR_UNSUPPORTED (not sm_100, TND), FA_ERR_CUDA
 * (launch). Asynchronous like fa_fwd; it reads the whole mask inside the
 * band once (1 byte per element).
 */
fa_status_t fa_mask_occupancy(const fa_desc_t* desc, const uint8_t* atten_mask,
                              uint8_t* tile_class, int32_t* ranges, void* cuda_stream);

/*
 * fa_fwd_with_ranges — fa_fwd for a dense-mask handle (sparse_mode 1, or 0
 * with a mask_kind) that takes the pre-pass's ranges from the caller instead
 * of running the pre-pass: one fa_mask_occupancy can then serve every call
 * that uses the same mask (for example every layer of a model); the call
 * launches the one-block work-list rebuild and the attention kernel.
 *
 * ranges  device int32, 16-byte aligned, exactly as fa_mask_occupancy wrote
 *         them for this descriptor's shape and this atten_mask, which must
 *         not have changed since; other values give undefined O and lse
 *         (every memory access stays inside the operands all the same).
 * The other arguments are fa_fwd's (no prefix or length arrays: modes 0/1
 * take none). Errors as fa_fwd, plus FA_ERR_PARAM_INVALID for a handle
 * without a dense mask or unaligned ranges and FA_ERR_NULLPTR for NULL
 * ranges or atten_mask.
 */
fa_status_t fa_fwd_with_ranges(fa_handle_t h, const void* q, const void* k, const void* v,
                               const uint8_t* atten_mask, const int32_t* ranges, void* o,
                               float* lse, void* cuda_stream);

/* ---------------- host-only helpers (no device work) ------------------- */

/*
 * fa_validate — every check that fa_create and fa_fwd make, without a
 * handle and without touching any device. has_mask: whether atten_mask would
 * be non-NULL. Arrays as in fa_fwd (host).
 */
fa_status_t fa_validate(const fa_desc_t* desc, const int64_t* prefix,
                        const int64_t* actual_seq_qlen, const int64_t* actual_seq_kvlen,
                        int32_t has_mask);

/*
 * fa_visible_pairs — number of visible (b, h, i, j) pairs of a valid call,
 * from the closed-form row intervals of the geometry (the FLOP count of the
 * throughput metric is 4 * D * pairs). Modes with a dense mask (mode 1, mode 0
 * with a mask) are FA_ERR_UNSUPPORTED: their count depends on the mask data.
 */
fa_status_t fa_visible_pairs(const fa_desc_t* desc, const int64_t* prefix,
                             const int64_t* actual_seq_qlen,
                             const int64_t* actual_seq_kvlen, int32_t has_mask,
                             int64_t* pairs_out);

/* Tile classes of the scheduler (tiles are 128 query rows x 128 keys). */
typedef enum { FA_TILE_EMPTY = 0, FA_TILE_PARTIAL = 1, FA_TILE_FULL = 2 } fa_tile_class_t;

/*
 * fa_tile_class — how the scheduler classifies the tile of sequence b with
 * query rows [128 qt, 128 qt + 128) and keys [128 kt, 128 kt + 128) (rows and
 * keys inside the sequence): EMPTY tiles are skipped, PARTIAL tiles get an
 * element mask, FULL tiles none. Returns the class, or -1 on invalid input.
 */
int32_t fa_tile_class(const fa_desc_t* desc, const int64_t* prefix,
                      const int64_t* actual_seq_qlen, const int64_t* actual_seq_kvlen,
                      int32_t has_mask, int64_t b, int64_t qt, int64_t kt);

/*
 * fa_plan_stats — size of the work list a call would run: out[0] = work
 * items (one per (sequence, head, block of 256 query rows) with at least one
 * query row), out[1] = EMPTY, out[2] = PARTIAL, out[3] = FULL 128x128 tiles
 * over all items and heads. out: host int64[4].
 */
fa_status_t fa_plan_stats(const fa_desc_t* desc, const int64_t* prefix,
                          const int64_t* actual_seq_qlen, const int64_t* actual_seq_kvlen,
                          int32_t has_mask, int64_t* out);

/*
 * fa_plan_items — the work list of a closed-form call (no attenMask) in the
 * order the kernel takes it on a device with num_sms SMs (148 on B200).
 * The cost key of an item is 8 x (the longer sub-tile's key tiles) + (the
 * shorter's). A list each CTA takes a fixed share of (fewer than 8 items
 * per SM) is longest first, ties in (sequence, block, head) order. A list
 * that is claimed at run time (at least 8 items per SM) is longest first by
 * buckets of 24 key tiles (key / 192), and inside a bucket ordered by
 * (sequence, head), then longest first, then block: the items in flight
 * then share their K/V tiles through L2. Items without a key tile come last
 * in both orders. Item m is out[4m .. 4m+3] = (sequence b, head h, block of
 * 256 query rows, cost key). out: host int32[4 * capacity], may be NULL when
 * capacity is 0. *n_items receives the list's length also when it exceeds
 * capacity (then FA_ERR_SHAPE and out is not written). num_sms < 1 is
 * FA_ERR_PARAM_INVALID. Host only; dense-mask calls rebuild their list on
 * the device from the mask.
 */
fa_status_t fa_plan_items(const fa_desc_t* desc, const int64_t* prefix,
                          const int64_t* actual_seq_qlen, const int64_t* actual_seq_kvlen,
                          int32_t num_sms, int64_t capacity, int32_t* out, int64_t* n_items);

/* ---------------- query split across devices (host only) ---------------- */

/* One part of a query split: its own problem and where it sits in the
 * unsplit tensors. */
typedef struct {
    fa_desc_t desc;            /* the part's problem: TND, sparse_mode 7/3 or 8/2 */
    int64_t q_begin, q_end;    /* its query tokens [q_begin, q_end) of the unsplit Q, O, lse */
    int64_t kv_begin, kv_end;  /* its key tokens [kv_begin, kv_end) of the unsplit K, V */
} fa_split_part_t;

/*
 * fa_split_queries — the multi-card scheme of the sparseMode page
 * (sparseMode=7 / sparseMode=8 sections): the query tokens of a varlen job
 * are cut into n_parts contiguous ranges, key/value are not cut, and each
 * part becomes an independent call whose outputs are exactly the unsplit
 * call's rows [q_begin, q_end). A rightDownCausal job (mode 3) gives parts in
 * mode 7 (the last sequence of a part, cut at its top, is the band with
 * preTokens = Skv_b, nextTokens = rows kept - Sq_b) or mode 3; a leftUpCausal
 * job (mode 2) gives parts in mode 8 (the first sequence, cut at its bottom,
 * is the band with preTokens = Skv_b, nextTokens = Sq_b - Skv_b for a bottom
 * piece) or mode 2.
 *
 * desc: TND, sparse_mode 2 or 3 (mode 3 needs Sq_b <= Skv_b for every
 * sequence, as the sparseMode=7 section requires of its non-band batches).
 * cuts: host int64[n_parts - 1], increasing query-token positions in
 * [0, T_q]; NULL = balance the visible-pair count of the parts.
 * part: 0 .. n_parts-1. out: the part; out_seq_qlen / out_seq_kvlen: host
 * int64[desc->B], receive the part's cumulative arrays (out->desc.B entries).
 * An empty part has Sq = Skv = 0 and one empty sequence.
 */
fa_status_t fa_split_queries(const fa_desc_t* desc, const int64_t* actual_seq_qlen,
                             const int64_t* actual_seq_kvlen, int32_t n_parts,
                             const int64_t* cuts, int32_t part, fa_split_part_t* out,
                             int64_t* out_seq_qlen, int64_t* out_seq_kvlen);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_FA_H */
