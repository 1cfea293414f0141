// C ABI front end: handles, per-call plan caching and the kernel launch.
//
// Two-stage use as the aclnnScatterPaKvCache page's host flow describes it:
// the descriptor is checked once (fa_create), then each fa_fwd validates its
// per-call arrays, reuses or rebuilds the cached work list, copies it to the
// handle's device workspace through pinned staging memory and enqueues the
// persistent kernel on the caller's stream.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "../../include/fa.h"
#include "fa_kernel.h"
#include "fa_plan.h"

using namespace fa;

struct fa_handle_s {
  fa_desc_t desc{};
  int device = -1;
  int num_sms = 0;
  // plan cache: the per-call arrays the current work list was built from
  std::vector<int64_t> plan_key;
  bool plan_valid = false;
  int32_t n_items = 0;
  int32_t n_seqs = 0;
  SeqRec geo0{};  // geometry of sequence 0 (every sequence's, outside TND)
  // paged K/V calls: [header][SeqRec x B][PagedGroup x n_groups][PagedUnit x
  // n_units] then the units' partial results (the plan key starts with -2)
  int32_t n_groups = 0;
  int64_t n_units = 0;
  int32_t paged_rows = 0;  // most query rows in one group
  // device workspace: [error word | claim counter at 128 | claim_done at 192 |
  // pad to 256 B][SeqRec x B][WorkItem x n]
  // [item_tr: 2 x TileRange per item] then, for a dense attenMask, the
  // occupancy pre-pass's ranges and classes
  void* d_ws = nullptr;
  size_t ws_bytes = 0;
  // pinned staging of the work list and the event of its last upload
  void* h_stage = nullptr;
  size_t stage_bytes = 0;
  cudaEvent_t stage_done = nullptr;
  cudaEvent_t last_call = nullptr;
  bool any_call = false;
  // tensor maps of the last call's operands
  const void* tm_key[3] = {nullptr, nullptr, nullptr};
  CUtensorMap tm[3];
  uint64_t timeout_ns = 2000000000ull;
  uint32_t debug_flags = 0;
};

namespace {

constexpr size_t kHeaderBytes = 256;
constexpr size_t kClaimOffset = 128;  // two work-claim counters, 64 bytes apart

bool env_flag(const char* name) {
  const char* v = std::getenv(name);
  return v != nullptr && v[0] != '\0' && v[0] != '0';
}

fa_status_t cuda_fail(cudaError_t e, const char* what) {
  return fail(FA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Planes of the attenMask the occupancy pre-pass reduces: SS one plane for
// every batch and head, B1SS one per batch, BNSS one per batch and head; 0
// when the call reads no mask.
int64_t mask_planes(const fa_desc_t* d, int has_mask) {
  if (!has_mask) return 0;
  if (d->mask_kind == FA_MASK_SS) return 1;
  if (d->mask_kind == FA_MASK_B1SS) return d->B;
  return d->B * d->N;
}

// Dense-mask calls keep, after the work list, each item's two ranges
// (item_tr, 32 bytes per item) and then the pre-pass's scratch.
size_t item_tr_offset(int32_t n_seqs, int32_t n_items) {
  return align_up(kHeaderBytes + align_up((size_t)n_seqs * sizeof(SeqRec), 256) +
                      (size_t)n_items * sizeof(WorkItem),
                  256);
}
size_t occupancy_offset(int32_t n_seqs, int32_t n_items) {
  return item_tr_offset(n_seqs, n_items) +
         align_up((size_t)n_items * 2 * sizeof(TileRange), 256);
}

// Point the pre-pass at `scratch`: the ranges, then (256-byte aligned) the
// classes; `a` already has its shape.
void occupancy_bind(OccParams* a, uint8_t* scratch) {
  a->ranges = reinterpret_cast<TileRange*>(scratch);
  a->cls = scratch + align_up((size_t)(a->n_planes * a->n_qt) * sizeof(TileRange), 256);
}

fa_status_t bind_device(fa_handle_t h) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (h->device >= 0) {
    if (dev != h->device)
      return fail(FA_ERR_PARAM_INVALID, "handle is bound to device %d, current device is %d",
                  h->device, dev);
    return FA_OK;
  }
  cudaDeviceProp prop;
  e = cudaGetDeviceProperties(&prop, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
  if (prop.major != 10 || prop.minor != 0)
    return fail(FA_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library runs on sm_100 (B200)", dev,
                prop.major, prop.minor);
  e = cudaEventCreateWithFlags(&h->stage_done, cudaEventDisableTiming);
  if (e != cudaSuccess) return cuda_fail(e, "cudaEventCreate");
  e = cudaEventCreateWithFlags(&h->last_call, cudaEventDisableTiming);
  if (e != cudaSuccess) return cuda_fail(e, "cudaEventCreate");
  h->device = dev;
  h->num_sms = prop.multiProcessorCount;
  return FA_OK;
}

// Make sure the device workspace holds `bytes`; the error word is zeroed
// whenever the workspace is (re)allocated.
fa_status_t ensure_workspace(fa_handle_t h, size_t bytes) {
  if (h->d_ws != nullptr && h->ws_bytes >= bytes) return FA_OK;
  if (env_flag("FA_TEST_FAIL_ALLOC")) return fail(FA_ERR_ALLOC, "device workspace (test hook)");
  if (h->d_ws != nullptr) {
    if (h->any_call) cudaEventSynchronize(h->last_call);
    cudaFree(h->d_ws);
    h->d_ws = nullptr;
    h->ws_bytes = 0;
  }
  size_t want = align_up(bytes < 4096 ? 4096 : bytes, 4096);
  cudaError_t e = cudaMalloc(&h->d_ws, want);
  if (e != cudaSuccess) {
    h->d_ws = nullptr;
    return fail(FA_ERR_ALLOC, "cudaMalloc(%zu): %s", want, cudaGetErrorString(e));
  }
  e = cudaMemset(h->d_ws, 0, kHeaderBytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemset");
  h->ws_bytes = want;
  return FA_OK;
}

fa_status_t ensure_stage(fa_handle_t h, size_t bytes) {
  if (h->h_stage != nullptr && h->stage_bytes >= bytes) return FA_OK;
  if (h->h_stage != nullptr) {
    cudaEventSynchronize(h->stage_done);
    cudaFreeHost(h->h_stage);
    h->h_stage = nullptr;
    h->stage_bytes = 0;
  }
  size_t want = align_up(bytes < 4096 ? 4096 : bytes, 4096);
  cudaError_t e = cudaMallocHost(&h->h_stage, want);
  if (e != cudaSuccess) {
    h->h_stage = nullptr;
    return fail(FA_ERR_ALLOC, "cudaMallocHost(%zu): %s", want, cudaGetErrorString(e));
  }
  h->stage_bytes = want;
  return FA_OK;
}

std::vector<int64_t> make_key(const fa_desc_t* d, const int64_t* prefix, const int64_t* cu_q,
                              const int64_t* cu_kv, int has_mask) {
  std::vector<int64_t> key;
  key.push_back(has_mask);
  if (d->sparse_mode == 5 || d->sparse_mode == 6) key.insert(key.end(), prefix, prefix + d->B);
  if (d->layout == FA_TND) {
    key.insert(key.end(), cu_q, cu_q + d->B);
    key.insert(key.end(), cu_kv, cu_kv + d->B);
  }
  return key;
}

fa_status_t refresh_plan(fa_handle_t h, const int64_t* prefix, const int64_t* cu_q,
                         const int64_t* cu_kv, int has_mask, cudaStream_t stream) {
  std::vector<int64_t> key = make_key(&h->desc, prefix, cu_q, cu_kv, has_mask);
  if (h->plan_valid && key == h->plan_key) return FA_OK;
  std::vector<SeqRec> recs = decode_geometry(&h->desc, prefix, cu_q, cu_kv, has_mask);
  std::vector<WorkItem> items = build_items(&h->desc, recs);
  if (items.size() > (size_t)0x7fffffff) return fail(FA_ERR_UNSUPPORTED, "too many work items");
  // Claimed lists (closed form only) take the L2-locality order.
  if (!has_mask && claims_items((int64_t)items.size(), h->num_sms))
    order_work_list(items.data(), items.data() + items.size(), true);
  const size_t seq_bytes = recs.size() * sizeof(SeqRec);
  const size_t item_bytes = items.size() * sizeof(WorkItem);
  const int64_t planes = mask_planes(&h->desc, has_mask);
  // Each item's two sub-tile ranges follow the list (item_tr): computed
  // here from the closed form and uploaded with it, or for a dense mask
  // written on the device by the rebuild kernel, followed by the pre-pass's
  // scratch. The kernel then reads a range with one load that does not wait
  // for the item record (computing it took ~1-2k cycles at each boundary).
  const size_t tr_off = item_tr_offset((int32_t)recs.size(), (int32_t)items.size());
  const size_t tr_bytes = items.size() * 2 * sizeof(TileRange);
  const size_t payload = planes ? align_up(seq_bytes, 256) + item_bytes
                                : tr_off - kHeaderBytes + tr_bytes;
  const size_t occ = planes ? occupancy_bytes(planes, h->desc.Sq, h->desc.Skv) : 0;
  fa_status_t st = ensure_workspace(
      h, planes ? occupancy_offset((int32_t)recs.size(), (int32_t)items.size()) + occ
                : kHeaderBytes + payload);
  if (st != FA_OK) return st;
  st = ensure_stage(h, payload);
  if (st != FA_OK) return st;
  cudaError_t e = cudaEventSynchronize(h->stage_done);  // previous upload has left staging
  if (e != cudaSuccess) return cuda_fail(e, "cudaEventSynchronize");
  if (h->any_call) {  // a kernel of this handle on another stream may still read the old list
    e = cudaStreamWaitEvent(stream, h->last_call, 0);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
  }
  uint8_t* hs = static_cast<uint8_t*>(h->h_stage);
  std::memcpy(hs, recs.data(), seq_bytes);
  if (item_bytes) std::memcpy(hs + align_up(seq_bytes, 256), items.data(), item_bytes);
  if (!planes) {  // each item's two sub-tile ranges, from the closed form
    TileRange* tr = reinterpret_cast<TileRange*>(hs + (tr_off - kHeaderBytes));
    for (size_t n = 0; n < items.size(); ++n) {
      const SeqRec& sr = recs[(size_t)items[n].b];
      for (int st = 0; st < kSubTiles; ++st) {
        const int64_t r0 = (int64_t)items[n].qblk * kBlockM + st * kTileM;
        tr[2 * n + st] = r0 < sr.sq ? tile_range(sr, r0) : TileRange{0, 0, 0, 0};
      }
    }
  }
  e = cudaMemcpyAsync(static_cast<uint8_t*>(h->d_ws) + kHeaderBytes, hs, payload,
                      cudaMemcpyHostToDevice, stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyAsync(work list)");
  e = cudaEventRecord(h->stage_done, stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  h->plan_key.swap(key);
  h->plan_valid = true;
  h->n_items = (int32_t)items.size();
  h->n_seqs = (int32_t)recs.size();
  if (!recs.empty()) h->geo0 = recs[0];
  return FA_OK;
}

// Element strides (batch, head, token) of Q/O or K/V in the handle's layout.
void operand_strides(const fa_desc_t* d, int64_t S, int64_t* sb, int64_t* sh, int64_t* st) {
  const int64_t N = d->N, D = d->D;
  switch (d->layout) {
    case FA_BNSD:
      *sb = N * S * D;
      *sh = S * D;
      *st = D;
      break;
    case FA_BSND:
      *sb = S * N * D;
      *sh = D;
      *st = N * D;
      break;
    default:  // TND: batch stride unused (tokens are global)
      *sb = 0;
      *sh = D;
      *st = N * D;
      break;
  }
}

fa_status_t encode_maps(fa_handle_t h, const void* q, const void* k, const void* v) {
  const void* ptrs[3] = {q, k, v};
  const fa_desc_t* d = &h->desc;
  for (int i = 0; i < 3; ++i) {
    if (h->tm_key[i] == ptrs[i]) continue;
    const int64_t S = (i == 0) ? d->Sq : d->Skv;
    int64_t sb, sh, st;
    operand_strides(d, S, &sb, &sh, &st);
    const bool tnd = d->layout == FA_TND;
    // dims (D, S, N, B); TND: (D, T, N, 1) with a dummy (valid) batch stride
    const int64_t b_extent = tnd ? 1 : d->B;
    const int64_t b_stride = tnd ? (S > 0 ? S : 1) * d->N * d->D : sb;
    if (!encode_operand_map(&h->tm[i], ptrs[i], d->D, S, d->N, b_extent, st, sh, b_stride)) {
      h->tm_key[i] = nullptr;
      return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled failed for operand %d", i);
    }
    h->tm_key[i] = ptrs[i];
  }
  return FA_OK;
}

}  // namespace

extern "C" {

fa_status_t fa_create(const fa_desc_t* desc, fa_handle_t* out) {
  clear_error();
  if (!out) return fail(FA_ERR_NULLPTR, "out is NULL");
  *out = nullptr;
  fa_status_t st = validate_desc(desc);
  if (st != FA_OK) return st;
  if (env_flag("FA_TEST_FAIL_ALLOC")) return fail(FA_ERR_ALLOC, "handle (test hook)");
  fa_handle_t h = new (std::nothrow) fa_handle_s();
  if (!h) return fail(FA_ERR_ALLOC, "handle");
  h->desc = *desc;
  if (const char* t = std::getenv("FA_WAIT_TIMEOUT_MS")) {
    long long ms = std::atoll(t);
    if (ms > 0) h->timeout_ns = (uint64_t)ms * 1000000ull;
  }
  if (env_flag("FA_TEST_DROP_FIRST_Q")) h->debug_flags |= kDebugDropFirstQ;
  *out = h;
  return FA_OK;
}

}  // extern "C"

namespace {

// fa_fwd and fa_fwd_with_ranges. `ranges` (or null): the dense-mask
// occupancy of this mask, already computed by fa_mask_occupancy.
fa_status_t forward(fa_handle_t h, const void* q, const void* k, const void* v,
                    const uint8_t* atten_mask, const int32_t* ranges, const float* slopes,
                    const int64_t* prefix, const int64_t* actual_seq_qlen,
                    const int64_t* actual_seq_kvlen, void* o, float* lse, void* cuda_stream) {
  if (!h) return fail(FA_ERR_NULLPTR, "handle is NULL");
  if (!q || !k || !v || !o || !lse) return fail(FA_ERR_NULLPTR, "q, k, v, o and lse are required");
  const fa_desc_t* d = &h->desc;
  if (d->alibi != FA_ALIBI_NONE && !slopes)
    return fail(FA_ERR_PARAM_INVALID,
                "the handle names an ALiBi variant: call fa_fwd_alibi with the slopes");
  if (slopes && ((uintptr_t)slopes & 3u))
    return fail(FA_ERR_PARAM_INVALID, "slopes must be 4-byte aligned");
  const int m = d->sparse_mode;
  const int has_mask = (m <= 1) && atten_mask != nullptr;
  fa_status_t st = validate_call(d, prefix, actual_seq_qlen, actual_seq_kvlen, has_mask);
  if (st != FA_OK) return st;
  const uintptr_t align = (uintptr_t)q | (uintptr_t)k | (uintptr_t)v | (uintptr_t)o;
  if (align & 15u) return fail(FA_ERR_PARAM_INVALID, "q, k, v and o must be 16-byte aligned");
  if ((uintptr_t)lse & 3u) return fail(FA_ERR_PARAM_INVALID, "lse must be 4-byte aligned");
  st = bind_device(h);
  if (st != FA_OK) return st;
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  st = refresh_plan(h, prefix, actual_seq_qlen, actual_seq_kvlen, has_mask, stream);
  if (st != FA_OK) return st;
  if (h->n_items == 0) return FA_OK;  // no query rows: nothing to write
  st = encode_maps(h, q, k, v);
  if (st != FA_OK) return st;

  FwdParams p;
  std::memset(&p, 0, sizeof(p));
  p.tm_q = h->tm[0];
  p.tm_k = h->tm[1];
  p.tm_v = h->tm[2];
  uint8_t* ws = static_cast<uint8_t*>(h->d_ws);
  p.err_word = reinterpret_cast<unsigned int*>(ws);
  p.seqs = reinterpret_cast<const SeqRec*>(ws + kHeaderBytes);
  p.items = reinterpret_cast<const WorkItem*>(
      ws + kHeaderBytes + align_up((size_t)h->n_seqs * sizeof(SeqRec), 256));
  p.o = o;
  p.lse = lse;
  p.mask = atten_mask;
  operand_strides(d, d->Sq, &p.o_sb, &p.o_sh, &p.o_st);
  if (d->layout == FA_TND) {
    p.l_sb = 0;
    p.l_sh = d->Sq;
  } else {
    p.l_sb = d->N * d->Sq;
    p.l_sh = d->Sq;
  }
  if (has_mask) {
    const int64_t plane = d->Sq * d->Skv;
    p.m_si = d->Skv;
    p.m_sb = (d->mask_kind == FA_MASK_SS) ? 0 : (d->mask_kind == FA_MASK_B1SS ? plane : d->N * plane);
    p.m_sh = (d->mask_kind == FA_MASK_BNSS) ? plane : 0;
  }
  if (has_mask) {
    // Reduce the mask to per-sub-tile key-tile ranges (unless the caller
    // already did), then rebuild the work list from them on the device, all
    // on the same stream ahead of the attention kernel.
    OccParams a;
    std::memset(&a, 0, sizeof(a));
    occupancy_shape(&a, h->geo0, mask_planes(d, has_mask));
    a.mask = atten_mask;
    SchedParams sp;
    std::memset(&sp, 0, sizeof(sp));
    sp.B = (int32_t)d->B;
    sp.N = (int32_t)d->N;
    sp.nblk = (int32_t)((d->Sq + kBlockM - 1) / kBlockM);
    if ((int64_t)sp.B * sp.N * sp.nblk != h->n_items)
      return fail(FA_ERR_DEVICE, "internal: dense-mask work list has %d items, expected %lld",
                  h->n_items, (long long)sp.B * sp.N * sp.nblk);
    // The list, item_tr and the pre-pass's table are rewritten every call:
    // a kernel of this handle on another stream may still be reading them.
    if (h->any_call) {
      cudaError_t e = cudaStreamWaitEvent(stream, h->last_call, 0);
      if (e != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
    }
    if (ranges != nullptr) {
      a.ranges = reinterpret_cast<TileRange*>(const_cast<int32_t*>(ranges));
    } else {
      occupancy_bind(&a, ws + occupancy_offset(h->n_seqs, h->n_items));
      cudaError_t e = launch_occupancy(a, h->num_sms, stream);
      if (e != cudaSuccess) return cuda_fail(e, "occupancy pre-pass launch");
    }
    sp.ranges = a.ranges;
    sp.items = const_cast<WorkItem*>(p.items);
    sp.item_tr = reinterpret_cast<TileRange*>(ws + item_tr_offset(h->n_seqs, h->n_items));
    sp.occ_sb = (d->mask_kind == FA_MASK_SS) ? 0 : (d->mask_kind == FA_MASK_B1SS ? 1 : d->N);
    sp.occ_sh = (d->mask_kind == FA_MASK_BNSS) ? 1 : 0;
    sp.n_qt = a.n_qt;
    sp.sq = (int32_t)d->Sq;
    sp.n_kt = a.n_kt;
    cudaError_t e = launch_schedule(sp, stream);
    if (e != cudaSuccess) return cuda_fail(e, "work list schedule launch");
    p.item_tr = sp.item_tr;
  }
  if (!has_mask)
    p.item_tr = reinterpret_cast<const TileRange*>(ws + item_tr_offset(h->n_seqs, h->n_items));
  p.n_items = h->n_items;
  // Closed-form lists (descending lpt_key: items without a key tile last)
  // with many items per CTA are claimed at run time.
  if (!has_mask && claims_items(h->n_items, h->num_sms)) {
    p.claim = reinterpret_cast<unsigned int*>(ws + kClaimOffset);
    p.claim_done = reinterpret_cast<unsigned int*>(ws + kClaimOffset + 64);
  }
  if (d->alibi != FA_ALIBI_NONE) {
    p.slopes = slopes;
    p.alibi = d->alibi;
  }
  p.tnd = d->layout == FA_TND ? 1 : 0;
  p.scale_log2 = (float)(d->scale * 1.4426950408889634073599);
  p.debug_flags = h->debug_flags;
  p.timeout_ns = h->timeout_ns;
  const int grid = h->n_items < h->num_sms ? h->n_items : h->num_sms;
  const char* why = nullptr;
  cudaError_t e = launch_fwd((int)d->D, p, grid, stream, &why);
  if (e != cudaSuccess) {
    if (why) return fail(FA_ERR_UNSUPPORTED, "launch refused: %s", why);
    return cuda_fail(e, "kernel launch");
  }
  e = cudaEventRecord(h->last_call, stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  h->any_call = true;
  return FA_OK;
}

}  // namespace

extern "C" {

fa_status_t fa_fwd(fa_handle_t h, const void* q, const void* k, const void* v,
                   const uint8_t* atten_mask, const int64_t* prefix,
                   const int64_t* actual_seq_qlen, const int64_t* actual_seq_kvlen, void* o,
                   float* lse, void* cuda_stream) {
  clear_error();
  return forward(h, q, k, v, atten_mask, nullptr, nullptr, prefix, actual_seq_qlen,
                 actual_seq_kvlen, o, lse, cuda_stream);
}

fa_status_t fa_fwd_alibi(fa_handle_t h, const void* q, const void* k, const void* v,
                         const float* slopes, const int64_t* prefix,
                         const int64_t* actual_seq_qlen, const int64_t* actual_seq_kvlen,
                         void* o, float* lse, void* cuda_stream) {
  clear_error();
  if (!h) return fail(FA_ERR_NULLPTR, "handle is NULL");
  if (!slopes) return fail(FA_ERR_NULLPTR, "slopes is NULL");
  if (h->desc.alibi == FA_ALIBI_NONE)
    return fail(FA_ERR_PARAM_INVALID, "fa_fwd_alibi needs a handle with an ALiBi variant");
  return forward(h, q, k, v, nullptr, nullptr, slopes, prefix, actual_seq_qlen,
                 actual_seq_kvlen, o, lse, cuda_stream);
}

fa_status_t fa_fwd_with_ranges(fa_handle_t h, const void* q, const void* k, const void* v,
                               const uint8_t* atten_mask, const int32_t* ranges, void* o,
                               float* lse, void* cuda_stream) {
  clear_error();
  if (!h) return fail(FA_ERR_NULLPTR, "handle is NULL");
  if (h->desc.sparse_mode > 1 || h->desc.mask_kind == FA_MASK_NONE || !atten_mask)
    return fail(FA_ERR_PARAM_INVALID,
                "fa_fwd_with_ranges needs sparse_mode 0 or 1 with a mask kind and atten_mask");
  if (!ranges) return fail(FA_ERR_NULLPTR, "ranges is NULL");
  if ((uintptr_t)ranges & 15u) return fail(FA_ERR_PARAM_INVALID, "ranges must be 16-byte aligned");
  return forward(h, q, k, v, atten_mask, ranges, nullptr, nullptr, nullptr, nullptr, o, lse,
                 cuda_stream);
}

fa_status_t fa_fwd_paged(fa_handle_t h, const void* q, const void* k_cache, const void* v_cache,
                         const int32_t* block_table, int64_t num_blocks, int32_t block_size,
                         int32_t max_blocks, const int64_t* prefix, const int64_t* actual_seq_qlen,
                         const int64_t* actual_seq_kvlen, void* o, float* lse,
                         void* cuda_stream) {
  clear_error();
  if (!h) return fail(FA_ERR_NULLPTR, "handle is NULL");
  if (!q || !k_cache || !v_cache || !block_table || !o || !lse)
    return fail(FA_ERR_NULLPTR, "q, k_cache, v_cache, block_table, o and lse are required");
  const fa_desc_t* d = &h->desc;
  fa_status_t st = validate_paged(d, prefix, actual_seq_qlen, actual_seq_kvlen, num_blocks,
                                  block_size, max_blocks);
  if (st != FA_OK) return st;
  const uintptr_t align = (uintptr_t)q | (uintptr_t)k_cache | (uintptr_t)v_cache | (uintptr_t)o;
  if (align & 15u)
    return fail(FA_ERR_PARAM_INVALID, "q, k_cache, v_cache and o must be 16-byte aligned");
  if (((uintptr_t)lse | (uintptr_t)block_table) & 3u)
    return fail(FA_ERR_PARAM_INVALID, "lse and block_table must be 4-byte aligned");
  st = bind_device(h);
  if (st != FA_OK) return st;
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  const int64_t D = d->D;
  std::vector<int64_t> key = {-2, block_size, max_blocks};
  key.insert(key.end(), actual_seq_qlen, actual_seq_qlen + d->B);
  key.insert(key.end(), actual_seq_kvlen, actual_seq_kvlen + d->B);
  if (d->sparse_mode == 5 || d->sparse_mode == 6) key.insert(key.end(), prefix, prefix + d->B);
  const int32_t hpu = paged_heads_per_unit(d->N, (int)D);
  const size_t part_unit = (size_t)hpu * kPagedRows * (size_t)(D + 4) * sizeof(float);
  if (!h->plan_valid || key != h->plan_key) {
    std::vector<SeqRec> recs = decode_geometry(d, prefix, actual_seq_qlen, actual_seq_kvlen, 0);
    std::vector<PagedGroup> groups;
    std::vector<PagedUnit> units;
    int32_t max_rows = 0;
    for (const SeqRec& r : recs) max_rows = std::max(max_rows, std::min(r.sq, (int32_t)kPagedRows));
    build_paged(d, recs, paged_slots((int)D, max_rows, hpu, h->num_sms), hpu, &groups, &units);
    if (units.size() > (size_t)0x7fffffff || groups.size() > (size_t)0x7fffffff)
      return fail(FA_ERR_UNSUPPORTED, "too many paged work units");
    const size_t seq_bytes = align_up(recs.size() * sizeof(SeqRec), 256);
    const size_t group_bytes = align_up(groups.size() * sizeof(PagedGroup), 256);
    const size_t payload = seq_bytes + group_bytes + units.size() * sizeof(PagedUnit);
    st = ensure_workspace(h, align_up(kHeaderBytes + payload, 256) + units.size() * part_unit);
    if (st != FA_OK) return st;
    st = ensure_stage(h, payload);
    if (st != FA_OK) return st;
    cudaError_t e = cudaEventSynchronize(h->stage_done);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventSynchronize");
    if (h->any_call) {
      e = cudaStreamWaitEvent(stream, h->last_call, 0);
      if (e != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
    }
    uint8_t* hs = static_cast<uint8_t*>(h->h_stage);
    std::memcpy(hs, recs.data(), recs.size() * sizeof(SeqRec));
    if (!groups.empty()) std::memcpy(hs + seq_bytes, groups.data(), groups.size() * sizeof(PagedGroup));
    if (!units.empty())
      std::memcpy(hs + seq_bytes + group_bytes, units.data(), units.size() * sizeof(PagedUnit));
    e = cudaMemcpyAsync(static_cast<uint8_t*>(h->d_ws) + kHeaderBytes, hs, payload,
                        cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyAsync(paged work list)");
    e = cudaEventRecord(h->stage_done, stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    h->plan_key.swap(key);
    h->plan_valid = true;
    h->n_seqs = (int32_t)recs.size();
    h->n_groups = (int32_t)groups.size();
    h->n_units = (int64_t)units.size();
    h->n_items = 0;
    h->paged_rows = 0;
    for (const PagedGroup& g : groups) h->paged_rows = std::max(h->paged_rows, g.nrows);
  } else if (h->any_call) {
    // The partial buffer is rewritten: order after the handle's last call.
    cudaError_t e = cudaStreamWaitEvent(stream, h->last_call, 0);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
  }
  if (h->n_groups == 0) return FA_OK;  // no query rows
  uint8_t* ws = static_cast<uint8_t*>(h->d_ws);
  const size_t seq_bytes = align_up((size_t)h->n_seqs * sizeof(SeqRec), 256);
  const size_t group_bytes = align_up((size_t)h->n_groups * sizeof(PagedGroup), 256);
  const size_t payload = seq_bytes + group_bytes + (size_t)h->n_units * sizeof(PagedUnit);
  PagedParams pp;
  std::memset(&pp, 0, sizeof(pp));
  pp.q = q;
  pp.k_cache = k_cache;
  pp.v_cache = v_cache;
  pp.block_table = block_table;
  pp.seqs = reinterpret_cast<const SeqRec*>(ws + kHeaderBytes);
  pp.groups = reinterpret_cast<const PagedGroup*>(ws + kHeaderBytes + seq_bytes);
  pp.units = reinterpret_cast<const PagedUnit*>(ws + kHeaderBytes + seq_bytes + group_bytes);
  pp.part = reinterpret_cast<float*>(ws + align_up(kHeaderBytes + payload, 256));
  pp.o = o;
  pp.lse = lse;
  pp.err_word = reinterpret_cast<unsigned int*>(ws);
  pp.num_blocks = num_blocks;
  pp.t_q = d->Sq;
  pp.n_units = h->n_units;
  pp.n_heads = (int32_t)d->N;
  pp.block_size = block_size;
  pp.max_blocks = max_blocks;
  pp.n_groups = h->n_groups;
  pp.heads_per_unit = hpu;
  pp.bs_shift = -1;
  if ((block_size & (block_size - 1)) == 0)
    for (int sh = 0; sh < 31; ++sh)
      if ((1 << sh) == block_size) pp.bs_shift = sh;
  pp.scale_log2 = (float)(d->scale * 1.4426950408889634073599);
  cudaError_t e = launch_paged((int)D, h->paged_rows, pp, stream);
  if (e != cudaSuccess) return cuda_fail(e, "paged kernel launch");
  e = cudaEventRecord(h->last_call, stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  h->any_call = true;
  return FA_OK;
}

fa_status_t fa_mask_occupancy(const fa_desc_t* desc, const uint8_t* atten_mask,
                              uint8_t* tile_class, int32_t* ranges, void* cuda_stream) {
  clear_error();
  if (!desc) return fail(FA_ERR_NULLPTR, "desc is NULL");
  if (!atten_mask || !tile_class || !ranges)
    return fail(FA_ERR_NULLPTR, "atten_mask, tile_class and ranges are required");
  fa_status_t st = validate_desc(desc);
  if (st != FA_OK) return st;
  if (desc->sparse_mode > 1 || desc->mask_kind == FA_MASK_NONE)
    return fail(FA_ERR_PARAM_INVALID, "the occupancy pre-pass needs sparse_mode 0 or 1 with a mask");
  st = validate_call(desc, nullptr, nullptr, nullptr, 1);
  if (st != FA_OK) return st;
  if ((uintptr_t)ranges & 15u) return fail(FA_ERR_PARAM_INVALID, "ranges must be 16-byte aligned");
  int dev = 0, major = 0, minor = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e, "device query");
  if (major != 10 || minor != 0)
    return fail(FA_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library runs on sm_100 (B200)", dev,
                major, minor);
  std::vector<SeqRec> recs = decode_geometry(desc, nullptr, nullptr, nullptr, 1);
  if (recs.empty()) return FA_OK;
  OccParams a;
  std::memset(&a, 0, sizeof(a));
  occupancy_shape(&a, recs[0], mask_planes(desc, 1));
  a.mask = atten_mask;
  a.cls = tile_class;
  a.ranges = reinterpret_cast<TileRange*>(ranges);
  e = launch_occupancy(a, sms, static_cast<cudaStream_t>(cuda_stream));
  if (e != cudaSuccess) return cuda_fail(e, "occupancy pre-pass launch");
  return FA_OK;
}

fa_status_t fa_sync_status(fa_handle_t h) {
  clear_error();
  if (!h) return fail(FA_ERR_NULLPTR, "handle is NULL");
  if (!h->any_call) return FA_OK;
  cudaError_t e = cudaEventSynchronize(h->last_call);
  if (e != cudaSuccess) return cuda_fail(e, "cudaEventSynchronize");
  unsigned int word = 0;
  e = cudaMemcpy(&word, h->d_ws, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(error word)");
  if (word == 0) return FA_OK;
  // Clear the whole header: the error word and, should an aborted launch
  // have left them set, the claim counters.
  e = cudaMemset(h->d_ws, 0, kHeaderBytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemset(header)");
  if (word & kErrTimeout)
    return fail(FA_ERR_TIMEOUT, "a device-side wait gave up (site %u); outputs are undefined",
                (word >> kErrWhereShift) & 0xffu);
  if (word & kErrBadBlock)
    return fail(FA_ERR_DEVICE,
                "a block_table entry was outside [0, num_blocks); its keys were left out");
  return fail(FA_ERR_DEVICE, "device error word 0x%08x", word);
}

fa_status_t fa_destroy(fa_handle_t h) {
  clear_error();
  if (!h) return FA_OK;
  if (h->any_call) cudaEventSynchronize(h->last_call);
  if (h->stage_done) cudaEventSynchronize(h->stage_done);
  if (h->d_ws) cudaFree(h->d_ws);
  if (h->h_stage) cudaFreeHost(h->h_stage);
  if (h->stage_done) cudaEventDestroy(h->stage_done);
  if (h->last_call) cudaEventDestroy(h->last_call);
  delete h;
  return FA_OK;
}

}  // extern "C"
