// Dense-mask tile occupancy: the pre-pass of sparseMode 0 (with an attenMask)
// and sparseMode 1 (allMask).
//
// The "sparseMode参数说明" page (sparseMode=1, allMask) has the caller pass
// the whole mask and the operator compute every pair the mask leaves
// visible; with sparseMode=0 the visible part is further cut to the band
// between preTokens and nextTokens. The closed-form geometry therefore only
// bounds where visible pairs can be, and without this pass the attention
// kernel would visit every 128 x 128 tile inside that bound and read the
// mask byte of every element. The masks the pages draw (the lower triangle
// of the causal case, the band) are mostly whole tiles that are all hidden
// or all visible, so the pass reduces the mask, once per call, to:
//
//   pass 1  the class of every tile of every mask plane: EMPTY (no visible
//           pair), FULL (every stored query row of the tile sees all 128 of
//           its keys, each key < Skv) or PARTIAL;
//   pass 2  per mask plane and 128-row query sub-tile, the TileRange the
//           attention kernel walks: [lo, hi) from the first to the last
//           non-EMPTY tile and [full_lo, full_hi) the longest run of FULL
//           tiles (the first such run on ties; lo..lo when there is none);
//   pass 3  the work list rebuilt from those ranges, longest item first by
//           its real number of key tiles (the host, which never sees the
//           mask, can only order items by the band), each item's two ranges
//           stored beside it so the attention kernel reads them by item
//           index, with no dependent load at an item boundary.
//
// EMPTY tiles at either end are skipped; FULL tiles of the run are computed
// without the element mask; every other tile of [lo, hi) (EMPTY ones in the
// middle too) keeps the element mask, so the result is exactly that of the
// unreduced mask. Passes 1 and 2 run as one launch (a thread-block cluster
// per strip), bound by reading the mask once (1 byte per element inside the
// band); pass 3 reads 32 bytes per item.
#include <cuda_runtime.h>

#include <cooperative_groups.h>

#include "fa_kernel.h"

namespace fa {
namespace {

enum : uint8_t { kOccEmpty = 0, kOccPartial = 1, kOccFull = 2 };

constexpr int kClassThreads = 256;  // 32 rows x 8 chunks of 16 keys per pass

// Bit b set when byte b of the 16 is zero (an unmasked key).
__device__ __forceinline__ uint32_t zero_bytes16(const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t bits = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t e = __vcmpeq4(w[q], 0u);  // 0xff in every zero byte
    const uint32_t nib = (e & 1u) | ((e >> 7) & 2u) | ((e >> 14) & 4u) | ((e >> 21) & 8u);
    bits |= nib << (4 * q);
  }
  return bits;
}

// Passes 1 and 2 in one launch: a cluster of kClusterCtas blocks per
// (plane, 128-row query sub-tile) strip. Each block classifies groups of kG
// consecutive tiles (rank r takes tiles [kG (8 i + r), kG (8 i + r) + kG)),
// with the 16-byte loads of all kG tiles in flight at once: thread t reads
// keys [16 (t % 8), 16 (t % 8) + 16) of rows t / 8 + 32 p, p = 0..3, so each
// warp load covers four whole 128-byte rows. The classes go to global memory;
// after the cluster barrier the leader block's first warp reads the strip's
// classes back (from L2) and writes its range.
constexpr int kClusterCtas = 8;
constexpr int kG = 4;
constexpr int kWarps = kClassThreads / 32;

__global__ void __cluster_dims__(kClusterCtas, 1, 1) __launch_bounds__(kClassThreads)
    occupancy_strips(const OccParams a) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  __shared__ uint32_t red_any[kG][kWarps], red_all[kG][kWarps];
  const int chunk = threadIdx.x & 7;
  const int rsub = threadIdx.x >> 3;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = (int)cluster.block_rank();
  const int64_t strip = blockIdx.x / kClusterCtas;
  const int64_t plane = strip / a.n_qt;
  const int qt = (int)(strip - plane * a.n_qt);
  const SeqRec& s = a.geo;
  const int64_t r0 = (int64_t)qt * kTileM;
  const uint8_t* base = a.mask + plane * a.m_plane;
  uint8_t* cls = a.cls + strip * a.n_kt;
  // The band bounds every visible pair: tiles outside it are EMPTY without
  // reading the mask.
  const TileRange g = tile_range(s, r0);
  // Visible keys [jlo, jhi] of this thread's four rows (empty past Sq).
  int jlo[kTileM / 32], jhi[kTileM / 32];
#pragma unroll
  for (int ps = 0; ps < kTileM / 32; ++ps) {
    const int64_t i = r0 + ps * 32 + rsub;
    jlo[ps] = 1;
    jhi[ps] = 0;
    if (i < s.sq) {
      jlo[ps] = (int)imax64(0, row_lo(s, i));
      jhi[ps] = (int)imin64((int64_t)s.skv - 1, row_hi(s, i));
    }
  }
  for (int kt0 = rank * kG; kt0 < a.n_kt; kt0 += kClusterCtas * kG) {
    uint32_t win[kG][kTileM / 32];  // keys of the chunk inside the row's band
    uint4 v[kG][kTileM / 32];
#pragma unroll
    for (int j = 0; j < kG; ++j) {
      const int kt = kt0 + j;
      const int j0 = kt * kTileN + chunk * 16;
#pragma unroll
      for (int ps = 0; ps < kTileM / 32; ++ps) {
        const int64_t i = r0 + ps * 32 + rsub;
        win[j][ps] = 0u;
        v[j][ps] = make_uint4(0u, 0u, 0u, 0u);
        if (kt < a.n_kt && kt >= g.lo && kt < g.hi) {
          const int lo = max(jlo[ps], j0);
          const int hi = min(jhi[ps], j0 + 15);
          if (lo <= hi) {
            win[j][ps] = ((1u << (uint32_t)(hi - lo + 1)) - 1u) << (uint32_t)(lo - j0);
            // With 16-byte rows the chunk lies inside the row: j0 <= hi < Skv
            // and both are multiples of 16.
            if (a.vec16) v[j][ps] = __ldg(reinterpret_cast<const uint4*>(base + i * s.skv + j0));
          }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kG; ++j) {
      const int kt = kt0 + j;
      const int j0 = kt * kTileN + chunk * 16;
      bool any = false, all = true;
#pragma unroll
      for (int ps = 0; ps < kTileM / 32; ++ps) {
        const int64_t i = r0 + ps * 32 + rsub;
        if (i >= s.sq) continue;  // rows past the sequence are not stored
        uint32_t zero = 0u;
        if (a.vec16) {
          zero = zero_bytes16(v[j][ps]);
        } else if (win[j][ps] != 0u) {
          const uint8_t* row = base + i * s.skv + j0;
          for (int b = 0; b < 16; ++b)
            if (((win[j][ps] >> b) & 1u) && row[b] == 0) zero |= 1u << b;
        }
        const uint32_t vis = zero & win[j][ps];
        any = any || vis != 0u;
        all = all && vis == 0xffffu;  // a key outside the band or >= Skv breaks FULL
      }
      const uint32_t wa = __any_sync(0xffffffffu, any), wl = __all_sync(0xffffffffu, all);
      if (lane == 0) {
        red_any[j][warp] = wa;
        red_all[j][warp] = wl;
      }
    }
    __syncthreads();
    if (threadIdx.x < kG && kt0 + (int)threadIdx.x < a.n_kt) {
      const int j = threadIdx.x;
      uint32_t any = 0u, all = 1u;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        any |= red_any[j][w];
        all &= red_all[j][w];
      }
      cls[kt0 + j] = all ? kOccFull : (any ? kOccPartial : kOccEmpty);
    }
    __syncthreads();
  }
  // Every block's classes are written; the writers' fence and the barrier's
  // release / acquire make them visible to the leader.
  if (threadIdx.x < kG) __threadfence();
  cluster.sync();
  if (rank != 0 || warp != 0) return;
  int lo = -1, hi = 0, run_lo = 0, run = 0, best_lo = 0, best = 0;
  for (int k0 = 0; k0 < a.n_kt; k0 += 32) {
    const int kt = k0 + lane;
    const uint32_t c = kt < a.n_kt ? cls[kt] : (uint32_t)kOccEmpty;
    const uint32_t nonempty = __ballot_sync(0xffffffffu, c != kOccEmpty);
    const uint32_t full = __ballot_sync(0xffffffffu, c == kOccFull);
    if (nonempty) {
      if (lo < 0) lo = k0 + __ffs(nonempty) - 1;
      hi = k0 + 32 - __clz(nonempty);
    }
    for (int b = 0; b < 32; ++b) {
      if ((full >> b) & 1u) {
        if (run == 0) run_lo = k0 + b;
        if (++run > best) {
          best = run;
          best_lo = run_lo;
        }
      } else {
        run = 0;
      }
    }
  }
  if (lane == 0) {
    TileRange r{0, 0, 0, 0};
    if (lo >= 0) {
      r.lo = lo;
      r.hi = hi;
      r.full_lo = best > 0 ? best_lo : lo;
      r.full_hi = best > 0 ? best_lo + best : lo;
    }
    a.ranges[strip] = r;
  }
}

// Pass 3: the work list in longest-first order by the real tile counts.
constexpr int kSchedThreads = 1024;
constexpr int kSchedBuckets = 4096;  // cost buckets; larger costs share the last one
constexpr int kWarpsSched = kSchedThreads / 32;
constexpr int kRankBuckets = 128;     // buckets of the parallel rank (at most 1024 items)

struct ItemCoord {
  int b, h, qb;
};

// Item c of the (b, block, h) enumeration the host list is built in.
__device__ __forceinline__ ItemCoord item_coord(const SchedParams& s, int64_t c) {
  const int64_t per_b = (int64_t)s.nblk * s.N;
  const int b = (int)(c / per_b);
  const int64_t rem = c - (int64_t)b * per_b;
  const int qb = (int)(rem / s.N);
  return ItemCoord{b, (int)(rem - (int64_t)qb * s.N), qb};
}

__device__ __forceinline__ TileRange sub_tr(const SchedParams& s, const ItemCoord& ic, int st) {
  const int qt = ic.qb * kSubTiles + st;
  if ((int64_t)qt * kTileM >= s.sq) return TileRange{0, 0, 0, 0};
  const int64_t plane = ic.b * s.occ_sb + ic.h * s.occ_sh;
  return s.ranges[plane * s.n_qt + qt];
}

__device__ __forceinline__ int item_cost(const SchedParams& s, const ItemCoord& ic) {
  int cost = 0;
#pragma unroll
  for (int st = 0; st < kSubTiles; ++st) {
    const TileRange tr = sub_tr(s, ic, st);
    cost += tr.hi > tr.lo ? tr.hi - tr.lo : 0;
  }
  return cost;
}

// Counts of buckets 0..nb-1 in cnt become their starts when the buckets are
// laid out from the highest down (one warp; lane l scans ranks
// [l * per, (l + 1) * per) of r = nb - 1 - k).
__device__ __forceinline__ void descending_offsets(int* cnt, int nb, int lane) {
  const int per = (nb + 31) / 32;
  const int r0 = min(lane * per, nb), r1 = min(r0 + per, nb);
  int sum = 0;
  for (int r = r0; r < r1; ++r) sum += cnt[nb - 1 - r];
  int incl = sum;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += v;
  }
  int acc = incl - sum;
  for (int r = r0; r < r1; ++r) {
    const int k = nb - 1 - r;
    const int c = cnt[k];
    cnt[k] = acc;
    acc += c;
  }
  __syncwarp();
}

// One block: a counting sort of the items by cost (descending). Warp 0
// places 32 items at a time in enumeration order, so equal costs keep it and
// the list is the same on every call. With at most one item per thread the
// item and its ranges stay in registers and warp 0 only hands out positions;
// otherwise warp 0 writes the items and the ranges are looked up again.
__global__ void __launch_bounds__(kSchedThreads) occupancy_schedule(const SchedParams s) {
  extern __shared__ uint16_t bucket_sm[];  // bucket of every item (sorted lists)
  __shared__ int start[kSchedBuckets];
  __shared__ int pos_sm[kSchedThreads];  // position of item c (one item per thread)
  __shared__ int wcount[kWarpsSched][kRankBuckets];  // items per (warp, cost bucket)
  const int tid = threadIdx.x, lane = tid & 31;
  const int64_t n = (int64_t)s.B * s.nblk * s.N;
  const bool one_each = n <= kSchedThreads;
  // This thread's item when one_each.
  ItemCoord mine{0, 0, 0};
  TileRange tr0{0, 0, 0, 0}, tr1{0, 0, 0, 0};
  int my_cost = 0;
  if (one_each && tid < n) {
    mine = item_coord(s, tid);
    tr0 = sub_tr(s, mine, 0);
    tr1 = sub_tr(s, mine, 1);
    my_cost = (tr0.hi > tr0.lo ? tr0.hi - tr0.lo : 0) + (tr1.hi > tr1.lo ? tr1.hi - tr1.lo : 0);
  }
  const int nb = min(s.n_kt * kSubTiles + 1, kSchedBuckets);
  if (one_each && nb <= kRankBuckets) {
    // Stable rank in parallel: within a warp from the lanes of equal cost
    // below this one, across warps from per-warp bucket counts.
    for (int k = tid; k < kWarpsSched * kRankBuckets; k += kSchedThreads)
      (&wcount[0][0])[k] = 0;
    __syncthreads();
    const int warp = tid >> 5;
    const int bk = tid < n ? min(my_cost, nb - 1) : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, bk);
    const int below = __popc(peers & ((1u << lane) - 1u));
    if (bk >= 0 && below == 0) wcount[warp][bk] = __popc(peers);
    __syncthreads();
    if (tid < nb) {  // exclusive prefix over warps per bucket, bucket totals
      int acc = 0;
      for (int w2 = 0; w2 < kWarpsSched; ++w2) {
        const int c = wcount[w2][tid];
        wcount[w2][tid] = acc;
        acc += c;
      }
      start[tid] = acc;
    }
    __syncthreads();
    if (tid < 32) descending_offsets(start, nb, lane);  // bucket k after every bucket > k
    __syncthreads();
    if (tid < n) {
      const int pos = start[bk] + wcount[warp][bk] + below;
      s.items[pos] = WorkItem{mine.b, mine.h, mine.qb, my_cost};
      s.item_tr[2 * pos] = tr0;
      s.item_tr[2 * pos + 1] = tr1;
    }
    return;
  }
  if (n <= kSortMaxItems) {
    for (int k = tid; k < nb; k += kSchedThreads) start[k] = 0;
    __syncthreads();
    for (int64_t c = tid; c < n; c += kSchedThreads) {
      const int cost = one_each ? my_cost : item_cost(s, item_coord(s, c));
      const int bk = min(cost, nb - 1);
      bucket_sm[c] = (uint16_t)bk;
      atomicAdd(&start[bk], 1);
    }
    __syncthreads();
    if (tid < 32) {
      descending_offsets(start, nb, lane);
      for (int64_t base = 0; base < n; base += 32) {
        const int64_t c = base + lane;
        const bool valid = c < n;
        const int bk = valid ? (int)bucket_sm[c] : -1;
        const unsigned peers = __match_any_sync(0xffffffffu, bk);
        const int leader = __ffs(peers) - 1;
        int pos0 = 0;
        if (valid && lane == leader) {
          pos0 = start[bk];
          start[bk] = pos0 + __popc(peers);
        }
        pos0 = __shfl_sync(0xffffffffu, pos0, leader);
        if (valid) {
          const int pos = pos0 + __popc(peers & ((1u << lane) - 1u));
          if (one_each) {
            pos_sm[c] = pos;
          } else {
            const ItemCoord ic = item_coord(s, c);
            s.items[pos] = WorkItem{ic.b, ic.h, ic.qb, bk};
          }
        }
        __syncwarp();
      }
    }
  } else {
    for (int64_t c = tid; c < n; c += kSchedThreads) {
      const ItemCoord ic = item_coord(s, c);
      s.items[c] = WorkItem{ic.b, ic.h, ic.qb, item_cost(s, ic)};
    }
  }
  __syncthreads();
  if (one_each) {
    if (tid < n) {
      const int pos = pos_sm[tid];
      s.items[pos] = WorkItem{mine.b, mine.h, mine.qb, my_cost};
      s.item_tr[2 * pos] = tr0;
      s.item_tr[2 * pos + 1] = tr1;
    }
    return;
  }
  for (int64_t pos = tid; pos < n; pos += kSchedThreads) {
    const WorkItem it = s.items[pos];
    const ItemCoord ic{it.b, it.h, it.qblk};
    s.item_tr[2 * pos] = sub_tr(s, ic, 0);
    s.item_tr[2 * pos + 1] = sub_tr(s, ic, 1);
  }
}

size_t round_up(size_t x, size_t m) { return (x + m - 1) / m * m; }

}  // namespace

cudaError_t launch_schedule(const SchedParams& s, cudaStream_t stream) {
  const int64_t n = (int64_t)s.B * s.nblk * s.N;
  if (n <= 0) return cudaSuccess;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(occupancy_schedule,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(kSortMaxItems * sizeof(uint16_t)));
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const size_t dyn = n <= kSortMaxItems ? (size_t)n * sizeof(uint16_t) : 0;
  occupancy_schedule<<<1, kSchedThreads, dyn, stream>>>(s);
  return cudaGetLastError();
}

size_t occupancy_bytes(int64_t n_planes, int64_t sq, int64_t skv) {
  const int64_t n_qt = (sq + kTileM - 1) / kTileM, n_kt = (skv + kTileN - 1) / kTileN;
  return round_up((size_t)(n_planes * n_qt) * sizeof(TileRange), 256) +
         (size_t)(n_planes * n_qt * n_kt);
}

void occupancy_shape(OccParams* a, const SeqRec& geo, int64_t n_planes) {
  a->geo = geo;
  a->n_planes = n_planes;
  a->m_plane = (int64_t)geo.sq * geo.skv;
  a->n_qt = (geo.sq + kTileM - 1) / kTileM;
  a->n_kt = (geo.skv + kTileN - 1) / kTileN;
  a->vec16 = 0;
}

cudaError_t launch_occupancy(const OccParams& a_in, int num_sms, cudaStream_t stream) {
  (void)num_sms;
  OccParams a = a_in;
  a.vec16 = (a.geo.skv % 16 == 0 && ((uintptr_t)a.mask & 15u) == 0) ? 1 : 0;
  const int64_t strips = a.n_planes * a.n_qt;
  if (strips <= 0) return cudaSuccess;
  if (strips > 0x7fffffff / kClusterCtas) return cudaErrorInvalidValue;
  occupancy_strips<<<(int)(strips * kClusterCtas), kClassThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace fa
