// Launch interface of the sm_100a masked attention forward kernel.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fa_internal.h"

namespace fa {

// Device error word bits (written by the kernel, read by fa_sync_status).
enum : uint32_t {
  kErrTimeout = 1u,      // a bounded mbarrier wait gave up
  kErrWhereShift = 8u,   // bits 8..15: which wait gave up first (WaitSite)
};

// Kernel arguments (passed by value as a __grid_constant__ parameter; the
// tensor maps must stay 64-byte aligned inside it).
struct __align__(64) FwdParams {
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  const SeqRec* seqs;
  const WorkItem* items;
  void* o;                 // bf16
  float* lse;
  const uint8_t* mask;     // dense attenMask (modes 0/1), else unused
  unsigned int* err_word;
  int64_t o_sb, o_sh, o_st;  // O element strides: batch, head, token
  int64_t l_sb, l_sh;        // lse element strides: batch, head (token stride 1)
  int64_t m_sb, m_sh, m_si;  // mask element strides: batch, head, row (column stride 1)
  // Dense-mask calls (or null): the key-tile ranges of sub-tiles 0 and 1
  // of work item idx are item_tr[2 idx] and item_tr[2 idx + 1].
  const TileRange* item_tr;
  // Work claiming (or null: each CTA takes the fixed snake of positions
  // c, 2G-1-c, 2G+c, ... of the list). With a counter, CTA c starts at
  // position c and every later item is the next unclaimed position G + n,
  // n from atomicAdd(claim, 1), taken while the CTA still loads its current
  // item; the last CTA to finish sets claim and claim_done back to 0. Needs
  // every item without a key tile after every item with one (a list sorted
  // by descending cost), and calls that do not overlap on the GPU.
  unsigned int* claim;
  unsigned int* claim_done;
  // ALiBi (or null): per-head slopes [N], fp32; alibi is the fa_alibi_t
  // variant. Only the closed-form instances with item_tr add the bias.
  const float* slopes;
  int32_t alibi;
  int32_t n_items;
  int32_t tnd;             // packed tokens: TMA batch coordinate 0, token = offset + row
  float scale_log2;        // scale * log2(e)
  uint32_t debug_flags;
  uint64_t timeout_ns;     // limit of every device-side wait
};

// Closed-form calls claim their items at run time (FwdParams::claim, a
// kernel instance of its own) when the list holds at least this many items
// per CTA: claims even out the differences in speed between SMs and the
// error of the cost key, which the fixed snake cannot, at a small cost per
// item. With fewer, each CTA's share is a few long items that the snake
// balances as well.
constexpr int kClaimMinItemsPerCta = 8;

enum DebugFlags : uint32_t {
  // The TMA warp of CTA 0 never loads its first Q tile, so the MMA warp's
  // wait on it runs out: exercises the bounded-wait abort path.
  kDebugDropFirstQ = 1u,
};

// Dense-mask tile occupancy (sparseMode 0 with an attenMask, sparseMode 1).
// Pass 1 classifies every 128 x 128 tile of every mask plane as EMPTY (no
// visible pair), FULL (every stored row sees all 128 keys) or PARTIAL; pass
// 2 reduces each plane's row of tiles (one 128-row query sub-tile) to the
// TileRange the attention kernel walks.
struct OccParams {
  const uint8_t* mask;   // planes of Sq x Skv bytes, nonzero = masked
  uint8_t* cls;          // out: [plane][qt][kt] tile classes (fa_tile_class_t values)
  TileRange* ranges;     // out: [plane][qt]
  SeqRec geo;            // the geometry every sequence shares (BNSD/BSND)
  int64_t m_plane;       // bytes per mask plane (Sq * Skv)
  int64_t n_planes;
  int32_t n_qt, n_kt;    // 128-row query sub-tiles, 128-key tiles
  int32_t vec16;         // mask base and rows 16-byte aligned: 16-byte loads
};

// Scratch bytes of the pre-pass for `n_planes` planes of Sq x Skv: the
// ranges (16 bytes per sub-tile, rounded up to 256) then the classes.
size_t occupancy_bytes(int64_t n_planes, int64_t sq, int64_t skv);
// Fill the pointer-free fields of `a` (the caller sets mask, cls, ranges).
void occupancy_shape(OccParams* a, const SeqRec& geo, int64_t n_planes);
// Enqueue both passes on `stream`.
cudaError_t launch_occupancy(const OccParams& a, int num_sms, cudaStream_t stream);

// The work list of a dense-mask call (BNSD/BSND: items (b, block of 256
// rows, h) for every b, block and h), rebuilt on the device from the
// pre-pass's ranges: longest first by the real key-tile count (ties in the
// host list's (b, block, h) order), each item's two sub-tile ranges beside
// it in item_tr. Lists longer than kSortMaxItems keep the (b, block, h)
// order.
struct SchedParams {
  const TileRange* ranges;  // [plane][qt] from the pre-pass
  WorkItem* items;          // out: [n]
  TileRange* item_tr;       // out: [2 n]
  int64_t occ_sb, occ_sh;   // plane = b * occ_sb + h * occ_sh
  int32_t B, N, nblk;       // items = B * nblk * N
  int32_t n_qt, sq;         // 128-row sub-tiles per plane, query rows
  int32_t n_kt;             // key tiles (a sub-tile's cost is at most n_kt)
};
constexpr int64_t kSortMaxItems = 65536;  // 2 bytes each in shared memory
cudaError_t launch_schedule(const SchedParams& s, cudaStream_t stream);

// ---------------------------------------------------------------- paged K/V
// Decode-shaped forward over paged caches [num_blocks, block_size, N, D]:
// work is split into groups (sequence, head, up to kPagedRows query rows)
// and each group's visible keys into units (chunks) that run in parallel;
// a merge pass combines each group's units in order.
enum : uint32_t { kErrBadBlock = 1u << 16 };  // a block_table entry outside [0, num_blocks)

struct PagedParams {
  const void* q;               // bf16 [T_q, N, D]
  const void* k_cache;         // bf16 [num_blocks, block_size, N, D]
  const void* v_cache;
  const int32_t* block_table;  // [B, max_blocks]
  const SeqRec* seqs;
  const PagedGroup* groups;
  const PagedUnit* units;
  float* part;                 // per (unit, head, row): o[D], m (log2 units), l, 2 pad (D + 4 floats)
  void* o;                     // bf16 [T_q, N, D]
  float* lse;                  // [N, T_q]
  unsigned int* err_word;
  int64_t num_blocks;
  int64_t t_q;
  int64_t n_units;
  int32_t n_heads, block_size, max_blocks, n_groups;
  int32_t heads_per_unit;      // heads one unit (CTA) covers; part is [unit][head][row][D + 4]
  int32_t bs_shift;            // log2(block_size) when it is a power of two, else -1
  float scale_log2;
};

// Heads one paged unit covers for N heads of dimension D: whole warps of
// D / 16 threads per head, at most 256 threads.
int paged_heads_per_unit(int64_t n_heads, int D);
// CTAs of the partial kernel resident at once on num_sms SMs.
int paged_slots(int D, int max_rows, int heads_per_unit, int num_sms);

// Enqueue the partial and merge kernels for head dim D (64 or 128);
// max_rows: the most query rows any group holds.
cudaError_t launch_paged(int D, int max_rows, const PagedParams& p, cudaStream_t stream);

// Build a 4-D bf16 tensor map over (D, S, N, B) with the given element
// strides of S, N and B, boxes of 64 x 128 x 1 x 1, 128-byte swizzle.
bool encode_operand_map(CUtensorMap* tm, const void* base, int64_t D, int64_t S, int64_t N,
                        int64_t B, int64_t st_s, int64_t st_n, int64_t st_b);

// Enqueue the kernel for head dim D on `stream` with `grid` persistent CTAs.
// Returns cudaSuccess or the launch error; `why` gets a reason for refusals.
cudaError_t launch_fwd(int D, const FwdParams& p, int grid, cudaStream_t stream,
                       const char** why);

}  // namespace fa
