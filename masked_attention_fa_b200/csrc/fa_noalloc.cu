// fa_fwd_noalloc: the forward for callers that must not allocate memory.
//
// Who needs this: code that runs where allocating is not allowed or not
// safe, for example inside a framework that owns all device memory through
// its own pool and forbids cudaMalloc/cudaFree behind its back, a real-time
// inference loop that must not allocate after start-up, or a plugin that is
// called from inside another library's allocator or memory callbacks. The
// handle-based fa_create/fa_fwd path allocates a device workspace (and pinned
// staging memory) for its work list; this entry point instead keeps the work
// list and the error word in a fixed, file-scope device array that exists
// from the moment the library is loaded onto a device until the process exits.
//
// Limits and sharing:
//   - The array holds kNoAllocScratchBytes (1 MiB): a 256-byte header (error
//     word and the kernel's two work-claim counters), the per-sequence records (32 bytes per sequence, rounded up to
//     256 bytes) and the work list (16 bytes per (sequence, head, block of
//     256 query rows)). Larger problems are rejected with FA_ERR_UNSUPPORTED
//     before any device work.
//   - A dense-mask call (sparseMode 1, or 0 with an attenMask) also puts
//     each work item's two key-tile ranges (32 bytes per item) and the
//     occupancy pre-pass's scratch (16 bytes per mask plane and 128-row query
//     sub-tile, rounded up to 256, plus 1 byte per plane and 128 x 128 tile)
//     behind the work list when they fit; when they do not, the call still
//     runs, without the pre-pass (every tile of the band is visited with the
//     element mask), and gives the same result.
//   - Every call, on every stream, shares the one array per device and leaves
//     its own work list in it. Calls whose kernels overlap on the GPU (for
//     example on two streams without ordering between them) race on the
//     array; order them on one stream, or use fa_create/fa_fwd handles.
//   - The first call on a device does the per-device set-up (it looks up the
//     array's device address with cudaGetSymbolAddress, reads the device's
//     attributes and sets the kernel's shared-memory attribute). Make that
//     first call before any stream capture begins.
//   - Calls cannot be recorded into a CUDA graph: each call uploads its work
//     list from one static host image that the next call overwrites, so a
//     replayed copy would pair this call's outputs with another call's list.
//     A call on a stream that is capturing returns FA_ERR_UNSUPPORTED before
//     doing anything.
//   - A device-side wait that gives up leaves an error word in the array's
//     header; fa_noalloc_sync_status reads it (and clears the header). The
//     next call clears it too, so check after each call that needs checking.
//   - No cudaMalloc, cudaFree, pinned or host-heap allocation happens on the
//     success path: the work list is built in a static host buffer, copied
//     with cudaMemcpyAsync from pageable memory (the call returns once the
//     driver has taken the bytes) and the error word is cleared with
//     cudaMemsetAsync. Host calls are serialised by a mutex.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/fa.h"
#include "fa_kernel.h"
#include "fa_plan.h"

// Size of the fixed device array (and of its host image).
#define FA_NOALLOC_SCRATCH_BYTES (1u << 20)

// The device scratch: header | SeqRec[B] | WorkItem[n]. In host code this
// name denotes a host-side shadow, never a device address: the address that
// kernels get comes from cudaGetSymbolAddress at set-up.
static __device__ __align__(256) unsigned char g_fa_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

namespace fa {
namespace {

constexpr size_t kNoAllocScratchBytes = FA_NOALLOC_SCRATCH_BYTES;
constexpr size_t kNoAllocHeaderBytes = 256;
constexpr int kNoAllocMaxDevices = 64;

// Host copy of the same layout, filled before each upload.
alignas(256) unsigned char g_host_image[kNoAllocScratchBytes];
std::mutex g_mutex;

struct DeviceSlot {
  bool ready;
  void* scratch;  // device address of g_fa_noalloc_scratch on that device
  int num_sms;
};
DeviceSlot g_devices[kNoAllocMaxDevices];

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// The test hooks the handle path reads at fa_create (a dropped first Q load
// that makes a bounded wait run out, and a shorter wait limit), read here at
// every call: reading the environment allocates nothing.
bool env_flag(const char* name) {
  const char* v = std::getenv(name);
  return v != nullptr && v[0] != '\0' && v[0] != '0';
}
uint64_t wait_limit_ns() {
  if (const char* t = std::getenv("FA_WAIT_TIMEOUT_MS")) {
    const long long ms = std::atoll(t);
    if (ms > 0) return (uint64_t)ms * 1000000ull;
  }
  return 2000000000ull;
}

fa_status_t cuda_err(cudaError_t e, const char* what) {
  return fail(FA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Per-device set-up, once per device, with that device current.
fa_status_t device_slot(DeviceSlot** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_err(e, "cudaGetDevice");
  if (dev < 0 || dev >= kNoAllocMaxDevices)
    return fail(FA_ERR_UNSUPPORTED, "device index %d beyond %d", dev, kNoAllocMaxDevices);
  DeviceSlot& s = g_devices[dev];
  if (!s.ready) {
    int major = 0, minor = 0, sms = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_err(e, "cudaDeviceGetAttribute");
    if (major != 10 || minor != 0)
      return fail(FA_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library runs on sm_100 (B200)",
                  dev, major, minor);
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_fa_noalloc_scratch);
    if (e != cudaSuccess || ptr == nullptr)
      return cuda_err(e == cudaSuccess ? cudaErrorInvalidSymbol : e, "cudaGetSymbolAddress");
    s.scratch = ptr;
    s.num_sms = sms;
    s.ready = true;
  }
  *out = &s;
  return FA_OK;
}

void strides_of(const fa_desc_t* d, int64_t S, int64_t* sb, int64_t* sh, int64_t* st) {
  const int64_t N = d->N, D = d->D;
  if (d->layout == FA_BNSD) {
    *sb = N * S * D, *sh = S * D, *st = D;
  } else if (d->layout == FA_BSND) {
    *sb = S * N * D, *sh = D, *st = N * D;
  } else {
    *sb = 0, *sh = D, *st = N * D;
  }
}

}  // namespace
}  // namespace fa

using namespace fa;

extern "C" fa_status_t fa_fwd_noalloc(const fa_desc_t* desc, const void* q, const void* k,
                                      const void* v, const uint8_t* atten_mask,
                                      const int64_t* prefix, const int64_t* actual_seq_qlen,
                                      const int64_t* actual_seq_kvlen, void* o, float* lse,
                                      void* cuda_stream) {
  clear_error();
  if (!desc) return fail(FA_ERR_NULLPTR, "desc is NULL");
  if (!q || !k || !v || !o || !lse) return fail(FA_ERR_NULLPTR, "q, k, v, o and lse are required");
  const int has_mask = (desc->sparse_mode <= 1) && atten_mask != nullptr;
  fa_status_t st = validate_call(desc, prefix, actual_seq_qlen, actual_seq_kvlen, has_mask);
  if (st != FA_OK) return st;
  if (desc->alibi != FA_ALIBI_NONE)
    return fail(FA_ERR_UNSUPPORTED, "fa_fwd_noalloc takes no ALiBi slopes; use fa_fwd_alibi");
  const uintptr_t align = (uintptr_t)q | (uintptr_t)k | (uintptr_t)v | (uintptr_t)o;
  if (align & 15u) return fail(FA_ERR_PARAM_INVALID, "q, k, v and o must be 16-byte aligned");
  if ((uintptr_t)lse & 3u) return fail(FA_ERR_PARAM_INVALID, "lse must be 4-byte aligned");

  // Size of the work list, checked against the fixed array before anything else.
  size_t n_items = 0;
  for (int64_t b = 0; b < desc->B; ++b) {
    int64_t sq = desc->Sq;
    if (desc->layout == FA_TND) sq = actual_seq_qlen[b] - (b ? actual_seq_qlen[b - 1] : 0);
    if (sq > 0) n_items += (size_t)((sq + kBlockM - 1) / kBlockM) * (size_t)desc->N;
  }
  const size_t seq_bytes = round256((size_t)desc->B * sizeof(SeqRec));
  const size_t need = kNoAllocHeaderBytes + seq_bytes + n_items * sizeof(WorkItem);
  if (need > kNoAllocScratchBytes)
    return fail(FA_ERR_UNSUPPORTED,
                "fa_fwd_noalloc: the work list needs %zu bytes but its fixed device array holds "
                "%zu (%lld sequences, %zu work items); use fa_create/fa_fwd for this problem",
                need, kNoAllocScratchBytes, (long long)desc->B, n_items);
  if (n_items == 0) return FA_OK;

  // A graph replay of this call would re-read the static host image after
  // later calls rewrote it: refuse capture outright.
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  cudaStreamCaptureStatus capturing = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(stream, &capturing);
  if (e != cudaSuccess) return cuda_err(e, "cudaStreamIsCapturing");
  if (capturing != cudaStreamCaptureStatusNone)
    return fail(FA_ERR_UNSUPPORTED,
                "fa_fwd_noalloc cannot be captured into a CUDA graph (its work list is uploaded "
                "from a host buffer that later calls overwrite); call it outside capture");

  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceSlot* slot = nullptr;
  st = device_slot(&slot);
  if (st != FA_OK) return st;

  // Per-sequence records and work items, built in the static host image with
  // the same rules and order as the handle path.
  SeqRec* recs = reinterpret_cast<SeqRec*>(g_host_image + kNoAllocHeaderBytes);
  WorkItem* items = reinterpret_cast<WorkItem*>(g_host_image + kNoAllocHeaderBytes + seq_bytes);
  int64_t first_ne = -1, last_ne = -1;
  for (int64_t b = 0; b < desc->B; ++b) {
    int64_t sq = desc->Sq;
    if (desc->layout == FA_TND) sq = actual_seq_qlen[b] - (b ? actual_seq_qlen[b - 1] : 0);
    if (sq > 0) {
      if (first_ne < 0) first_ne = b;
      last_ne = b;
    }
  }
  for (int64_t b = 0; b < desc->B; ++b) {
    int64_t qo = 0, ko = 0, sq = desc->Sq, skv = desc->Skv;
    if (desc->layout == FA_TND) {
      qo = b ? actual_seq_qlen[b - 1] : 0;
      ko = b ? actual_seq_kvlen[b - 1] : 0;
      sq = actual_seq_qlen[b] - qo;
      skv = actual_seq_kvlen[b] - ko;
    }
    const __int128 delta = (__int128)skv - sq;
    auto clampo = [](__int128 x) -> int64_t {
      return x < -(__int128)kUnbounded ? -kUnbounded
                                       : (x > (__int128)kUnbounded ? kUnbounded : (int64_t)x);
    };
    int64_t lo = -kUnbounded, hi = kUnbounded, pfx = 0;
    int rule = desc->sparse_mode;
    if (rule == 7) rule = (b == last_ne) ? 4 : 3;
    if (rule == 8) rule = (b == first_ne) ? 4 : 2;
    if (rule == 0 && has_mask) {  // band from the top-left
      lo = clampo(-(__int128)desc->pre_tokens);
      hi = clampo((__int128)desc->next_tokens);
    } else if (rule == 2) {  // leftUpCausal
      hi = 0;
    } else if (rule == 3) {  // rightDownCausal
      hi = clampo(delta);
    } else if (rule == 4) {  // band from the bottom-right
      lo = clampo(delta - desc->pre_tokens);
      hi = clampo(delta + desc->next_tokens);
    } else if (rule == 5 || rule == 6) {  // rightDownCausal plus prefix columns
      hi = clampo(delta);
      pfx = prefix[b];
    }
    recs[b] = SeqRec{(int32_t)qo, (int32_t)ko, (int32_t)sq, (int32_t)skv, (int32_t)lo, (int32_t)hi,
                     (int32_t)pfx,
                     (desc->sparse_mode == 1 || (desc->sparse_mode == 0 && has_mask))
                         ? (int32_t)kSeqDenseMask : 0};
  }
  size_t n = 0;
  for (int64_t b = 0; b < desc->B; ++b) {
    const SeqRec& s = recs[b];
    if (s.sq <= 0) continue;
    const int32_t nblk = (s.sq + kBlockM - 1) / kBlockM;
    for (int32_t qb = 0; qb < nblk; ++qb) {
      const int32_t cost = lpt_key(tile_range(s, (int64_t)qb * kBlockM),
                                   tile_range(s, (int64_t)qb * kBlockM + kTileM));
      for (int64_t h = 0; h < desc->N; ++h) items[n++] = WorkItem{(int32_t)b, (int32_t)h, qb, cost};
    }
  }
  // The handle path's order (in place, no temporary buffer): strict longest
  // first, or the L2-locality order for a list that is claimed at run time
  // (a closed-form list with room for its ranges, see below).
  const size_t tr_need = round256(need) + n * 2 * sizeof(TileRange);
  const bool claimed = !has_mask && tr_need <= kNoAllocScratchBytes &&
                       claims_items((int64_t)n, slot->num_sms);
  order_work_list(items, items + n, claimed);

  unsigned char* dscr = static_cast<unsigned char*>(slot->scratch);
  e = cudaMemsetAsync(dscr, 0, kNoAllocHeaderBytes, stream);  // error word = 0
  if (e != cudaSuccess) return cuda_err(e, "cudaMemsetAsync");
  e = cudaMemcpyAsync(dscr + kNoAllocHeaderBytes, g_host_image + kNoAllocHeaderBytes,
                      need - kNoAllocHeaderBytes, cudaMemcpyHostToDevice, stream);
  if (e != cudaSuccess) return cuda_err(e, "cudaMemcpyAsync");

  FwdParams p;
  std::memset(&p, 0, sizeof(p));
  const fa_desc_t* d = desc;
  const bool tnd = d->layout == FA_TND;
  const void* ptrs[3] = {q, k, v};
  CUtensorMap* maps[3] = {&p.tm_q, &p.tm_k, &p.tm_v};
  for (int i = 0; i < 3; ++i) {
    const int64_t S = i == 0 ? d->Sq : d->Skv;
    int64_t sb, sh, stt;
    strides_of(d, S, &sb, &sh, &stt);
    const int64_t b_stride = tnd ? (S > 0 ? S : 1) * d->N * d->D : sb;
    if (!encode_operand_map(maps[i], ptrs[i], d->D, S, d->N, tnd ? 1 : d->B, stt, sh, b_stride))
      return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled failed for operand %d", i);
  }
  p.err_word = reinterpret_cast<unsigned int*>(dscr);
  p.seqs = reinterpret_cast<const SeqRec*>(dscr + kNoAllocHeaderBytes);
  p.items = reinterpret_cast<const WorkItem*>(dscr + kNoAllocHeaderBytes + seq_bytes);
  p.o = o;
  p.lse = lse;
  p.mask = atten_mask;
  strides_of(d, d->Sq, &p.o_sb, &p.o_sh, &p.o_st);
  p.l_sb = tnd ? 0 : d->N * d->Sq;
  p.l_sh = d->Sq;
  if (has_mask) {
    const int64_t plane = d->Sq * d->Skv;
    p.m_si = d->Skv;
    p.m_sb = (d->mask_kind == FA_MASK_SS) ? 0 : (d->mask_kind == FA_MASK_B1SS ? plane : d->N * plane);
    p.m_sh = (d->mask_kind == FA_MASK_BNSS) ? plane : 0;
  }
  if (!has_mask && n > 0) {
    // Each item's two sub-tile ranges beside the list when they fit, as the
    // handle path keeps them (else the kernel computes them per item).
    const size_t tr_off = round256(need);
    if (tr_off + n * 2 * sizeof(TileRange) <= kNoAllocScratchBytes) {
      TileRange* tr = reinterpret_cast<TileRange*>(g_host_image + tr_off);
      for (size_t m = 0; m < n; ++m) {
        const SeqRec& sr = recs[items[m].b];
        for (int st = 0; st < kSubTiles; ++st) {
          const int64_t r0 = (int64_t)items[m].qblk * kBlockM + st * kTileM;
          tr[2 * m + st] = r0 < sr.sq ? tile_range(sr, r0) : TileRange{0, 0, 0, 0};
        }
      }
      e = cudaMemcpyAsync(dscr + tr_off, g_host_image + tr_off, n * 2 * sizeof(TileRange),
                          cudaMemcpyHostToDevice, stream);
      if (e != cudaSuccess) return cuda_err(e, "cudaMemcpyAsync(item ranges)");
      p.item_tr = reinterpret_cast<const TileRange*>(dscr + tr_off);
      // Claimed work as in fa_fwd; the counters sit in the header, which
      // was zeroed above.
      if (claimed) {
        p.claim = reinterpret_cast<unsigned int*>(dscr + 128);
        p.claim_done = reinterpret_cast<unsigned int*>(dscr + 192);
      }
    }
  }
  if (has_mask && n > 0) {
    // The occupancy pre-pass and the device-side list rebuild run when their
    // scratch (each item's ranges, the pre-pass's table and classes) fits
    // behind the work list; otherwise the kernel visits every tile of the
    // band with the element mask, which gives the same result more slowly.
    const int64_t planes = d->mask_kind == FA_MASK_SS ? 1
                           : d->mask_kind == FA_MASK_B1SS ? d->B
                                                          : d->B * d->N;
    const size_t tr_off = round256(need);
    const size_t occ_off = tr_off + round256(n * 2 * sizeof(TileRange));
    if (occ_off + occupancy_bytes(planes, d->Sq, d->Skv) <= kNoAllocScratchBytes) {
      OccParams a;
      std::memset(&a, 0, sizeof(a));
      occupancy_shape(&a, recs[0], planes);
      a.mask = atten_mask;
      a.ranges = reinterpret_cast<TileRange*>(dscr + occ_off);
      a.cls = dscr + occ_off + round256((size_t)(planes * a.n_qt) * sizeof(TileRange));
      e = launch_occupancy(a, slot->num_sms, stream);
      if (e != cudaSuccess) return cuda_err(e, "occupancy pre-pass launch");
      SchedParams sp;
      std::memset(&sp, 0, sizeof(sp));
      sp.ranges = a.ranges;
      sp.items = reinterpret_cast<WorkItem*>(dscr + kNoAllocHeaderBytes + seq_bytes);
      sp.item_tr = reinterpret_cast<TileRange*>(dscr + tr_off);
      sp.occ_sb = (d->mask_kind == FA_MASK_SS) ? 0 : (d->mask_kind == FA_MASK_B1SS ? 1 : d->N);
      sp.occ_sh = (d->mask_kind == FA_MASK_BNSS) ? 1 : 0;
      sp.B = (int32_t)d->B;
      sp.N = (int32_t)d->N;
      sp.nblk = (int32_t)((d->Sq + kBlockM - 1) / kBlockM);
      sp.n_qt = a.n_qt;
      sp.sq = (int32_t)d->Sq;
      sp.n_kt = a.n_kt;
      if ((size_t)sp.B * sp.N * sp.nblk != n)
        return fail(FA_ERR_DEVICE, "internal: dense-mask work list has %zu items", n);
      e = launch_schedule(sp, stream);
      if (e != cudaSuccess) return cuda_err(e, "work list schedule launch");
      p.item_tr = sp.item_tr;
    }
  }
  p.n_items = (int32_t)n;
  p.tnd = tnd ? 1 : 0;
  p.scale_log2 = (float)(d->scale * 1.4426950408889634073599);
  p.debug_flags = env_flag("FA_TEST_DROP_FIRST_Q") ? kDebugDropFirstQ : 0u;
  p.timeout_ns = wait_limit_ns();
  const int grid = (int)std::min<size_t>(n, (size_t)slot->num_sms);
  const char* why = nullptr;
  e = launch_fwd((int)d->D, p, grid, stream, &why);
  if (e != cudaSuccess) {
    if (why) return fail(FA_ERR_UNSUPPORTED, "launch refused: %s", why);
    return cuda_err(e, "kernel launch");
  }
  return FA_OK;
}

extern "C" fa_status_t fa_noalloc_sync_status(void* cuda_stream) {
  clear_error();
  std::lock_guard<std::mutex> lock(g_mutex);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_err(e, "cudaGetDevice");
  if (dev < 0 || dev >= kNoAllocMaxDevices || !g_devices[dev].ready)
    return FA_OK;  // no call has run on this device
  e = cudaStreamSynchronize(static_cast<cudaStream_t>(cuda_stream));
  if (e != cudaSuccess) return cuda_err(e, "cudaStreamSynchronize");
  // A 4-byte read into a static host word: no allocation.
  static unsigned int word;
  e = cudaMemcpy(&word, g_devices[dev].scratch, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_err(e, "cudaMemcpy(error word)");
  if (word == 0) return FA_OK;
  // Clear the whole header: the error word and, should an aborted launch
  // have left them set, the claim counters.
  e = cudaMemset(g_devices[dev].scratch, 0, kNoAllocHeaderBytes);
  if (e != cudaSuccess) return cuda_err(e, "cudaMemset(header)");
  if (word & kErrTimeout)
    return fail(FA_ERR_TIMEOUT,
                "a device-side wait gave up (site %u); the last call's outputs are undefined",
                (word >> kErrWhereShift) & 0xffu);
  return fail(FA_ERR_DEVICE, "device error word 0x%08x", word);
}
