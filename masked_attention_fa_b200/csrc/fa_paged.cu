// Forward with keys and values read from paged caches, for decode-shaped
// calls (a few query rows per sequence against a long cached context).
//
// Cache layout: the "Norm" cache of the aclnnScatterPaKvCache page
// (scenario 2), [num_blocks, block_size, N, D] bf16, where a token written
// at slot s sits in block s / block_size at offset s % block_size. Key j of
// sequence b is in block block_table[b][j / block_size] at offset
// j % block_size. Visibility is the closed-form row interval of the
// sequence's sparseMode (the same SeqRec rule as the packed kernel).
//
// With one to four query rows per (sequence, head) there is no dense
// contraction to feed the tensor cores: every cached key and value byte is
// read once and used for a handful of FMAs, so the path is bound by HBM
// bandwidth. It is split over the keys so that a few long sequences still
// fill the GPU:
//
//   paged_partial  one CTA per (sequence, row block of up to kPagedRows
//                  query rows, chunk of keys, run of up to 256 * 16 / D
//                  heads). D / 16 threads share a head, each with 16
//                  dimensions of q, k, v and o, so for every key the CTA reads
//                  whole token rows of the cache (a token's heads are adjacent
//                  in the layout) with 32-byte loads, several keys in flight.
//                  A score is a sum over the head's threads (xor shuffles);
//                  each (head, row) runs the online softmax (running max m,
//                  running sum l) over the whole chunk and writes its partial
//                  (o, m, l) in fp32. The unit's block ids are staged in
//                  shared memory.
//   paged_merge    one warp per (group, row) combines the chunks of its group
//                  in chunk order (a fixed order, so the result is the same
//                  on every run), divides by l and writes O (bf16) and lse.
//
// Every block-table entry is checked against [0, num_blocks) before it is
// used; a bad one sets kErrBadBlock in the error word and masks that key.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "fa_kernel.h"

namespace fa {
namespace {

constexpr int kSlice = 16;        // dimensions per thread
constexpr int kPartPad = 4;       // a partial row: o[D], m, l, two pad floats (16-byte rows)
constexpr int kTableStage = 512;  // block ids of a unit staged in shared memory
constexpr float kLn2 = 0.69314718055994530942f;

__device__ __forceinline__ void unpack8(const uint4& v, float* f) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// Rescale an accumulator to a larger running maximum (log2 units).
__device__ __forceinline__ float rescale(float m_old, float m_new) {
  return m_old == -INFINITY ? 0.f : exp2f(m_old - m_new);
}

// One CTA per unit: heads [h0, h0 + HC) of one row block of one sequence
// over the keys [key0, key1). Thread t serves head h0 + t / L (L = D / 16
// threads per head) and dimensions [16 (t % L), 16 (t % L) + 16), so for
// every key the CTA reads whole token rows of the cache (all heads are
// adjacent in the layout). R: rows a unit may hold (1 for decode calls);
// KEYS: keys whose loads are in flight together.
template <int D, int R, int KEYS>
__global__ void __launch_bounds__(256) paged_partial(const PagedParams p) {
  constexpr int L = D / kSlice;
  __shared__ int32_t sm_blk[kTableStage];
  const PagedUnit u = p.units[blockIdx.x];
  const SeqRec sr = p.seqs[u.b];
  const int hl = threadIdx.x / L, sl = threadIdx.x % L;
  const int h = u.h0 + hl;
  const bool live = h < p.n_heads;
  const __nv_bfloat16* qb = reinterpret_cast<const __nv_bfloat16*>(p.q);
  float q[R][kSlice];
  int jlo[R], jhi[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    jlo[r] = 1, jhi[r] = 0;
#pragma unroll
    for (int x = 0; x < kSlice; ++x) q[r][x] = 0.f;
    if (r < u.nrows) {
      const int64_t i = (int64_t)u.row0 + r;  // row inside the sequence
      jlo[r] = (int)imax64(0, row_lo(sr, i));
      jhi[r] = (int)imin64((int64_t)sr.skv - 1, row_hi(sr, i));
      if (live) {
        const uint4* src = reinterpret_cast<const uint4*>(
            qb + (((int64_t)sr.q_off + i) * p.n_heads + h) * D + sl * kSlice);
        unpack8(src[0], q[r]);
        unpack8(src[1], q[r] + 8);
#pragma unroll
        for (int x = 0; x < kSlice; ++x) q[r][x] *= p.scale_log2;
      }
    }
  }
  float m[R], l[R], o[R][kSlice];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    m[r] = -INFINITY, l[r] = 0.f;
#pragma unroll
    for (int x = 0; x < kSlice; ++x) o[r][x] = 0.f;
  }
  const __nv_bfloat16* kc = reinterpret_cast<const __nv_bfloat16*>(p.k_cache);
  const __nv_bfloat16* vc = reinterpret_cast<const __nv_bfloat16*>(p.v_cache);
  const int32_t* table = p.block_table + (int64_t)u.b * p.max_blocks;
  // Block and offset of key j: a shift and a mask for power-of-two block sizes.
  const int bs_shift = p.bs_shift;
  auto block_of = [&](int j) { return bs_shift >= 0 ? j >> bs_shift : j / p.block_size; };
  auto offset_of = [&](int j) {
    return bs_shift >= 0 ? j & (p.block_size - 1) : j % p.block_size;
  };
  // This thread's elements inside a token row (all heads of a token are adjacent).
  const int64_t row_elems = (int64_t)p.n_heads * D;
  const int64_t my_off = (int64_t)h * D + sl * kSlice;
  // The unit's block ids, read once into shared memory (units hold keys, so
  // key1 > key0 and the blocks are table entries [blk0, blk0 + nblk)).
  const int blk0 = block_of(u.key0);
  const int nblk = block_of(u.key1 - 1) - blk0 + 1;
  const bool staged = nblk <= kTableStage;
  if (staged)
    for (int t = threadIdx.x; t < nblk; t += blockDim.x) sm_blk[t] = __ldg(table + blk0 + t);
  __syncthreads();
  bool bad = false;
  for (int j0 = u.key0; j0 < u.key1; j0 += KEYS) {
    uint4 kv[KEYS][2], vv[KEYS][2];
    bool ok[KEYS];
#pragma unroll
    for (int e = 0; e < KEYS; ++e) {
      const int j = j0 + e;
      ok[e] = false;
      if (j < u.key1) {
        const int bi = block_of(j);
        const int32_t blk = staged ? sm_blk[bi - blk0] : __ldg(table + bi);
        if (blk >= 0 && (int64_t)blk < p.num_blocks) {
          ok[e] = true;
          if (live) {
            const int64_t slot = (int64_t)blk * p.block_size + offset_of(j);
            const int64_t off = slot * row_elems + my_off;
            const uint4* ks = reinterpret_cast<const uint4*>(kc + off);
            const uint4* vs = reinterpret_cast<const uint4*>(vc + off);
            kv[e][0] = __ldg(ks);
            kv[e][1] = __ldg(ks + 1);
            vv[e][0] = __ldg(vs);
            vv[e][1] = __ldg(vs + 1);
          } else {
            kv[e][0] = kv[e][1] = vv[e][0] = vv[e][1] = make_uint4(0u, 0u, 0u, 0u);
          }
        } else {
          bad = true;
        }
      }
    }
#pragma unroll
    for (int e = 0; e < KEYS; ++e) {
      if (!ok[e]) continue;  // the same for every thread: one block id per key
      const int j = j0 + e;
      float kf[kSlice], vf[kSlice];
      unpack8(kv[e][0], kf);
      unpack8(kv[e][1], kf + 8);
      unpack8(vv[e][0], vf);
      unpack8(vv[e][1], vf + 8);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if (r >= u.nrows) break;
        float s = 0.f;
#pragma unroll
        for (int x = 0; x < kSlice; ++x) s = fmaf(q[r][x], kf[x], s);
#pragma unroll
        for (int d = 1; d < L; d <<= 1) s += __shfl_xor_sync(0xffffffffu, s, d);
        if (j < jlo[r] || j > jhi[r]) continue;
        if (s > m[r]) {
          const float a = rescale(m[r], s);
          l[r] *= a;
#pragma unroll
          for (int x = 0; x < kSlice; ++x) o[r][x] *= a;
          m[r] = s;
        }
        const float pj = exp2f(s - m[r]);
        l[r] += pj;
#pragma unroll
        for (int x = 0; x < kSlice; ++x) o[r][x] = fmaf(pj, vf[x], o[r][x]);
      }
    }
  }
  if (bad && threadIdx.x == 0) atomicOr(p.err_word, kErrBadBlock);
  if (!live) return;
  float* out = p.part + ((int64_t)blockIdx.x * p.heads_per_unit + hl) * kPagedRows * (D + kPartPad);
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (r >= u.nrows) break;
    float4* dst = reinterpret_cast<float4*>(out + r * (D + kPartPad) + sl * kSlice);
#pragma unroll
    for (int x = 0; x < kSlice / 4; ++x)
      dst[x] = make_float4(o[r][4 * x], o[r][4 * x + 1], o[r][4 * x + 2], o[r][4 * x + 3]);
    if (sl == 0) {
      out[r * (D + kPartPad) + D] = m[r];
      out[r * (D + kPartPad) + D + 1] = l[r];
    }
  }
}

// One warp per (group, row): the group's chunks in chunk order.
template <int D>
__global__ void __launch_bounds__(128) paged_merge(const PagedParams p) {
  const int lane = threadIdx.x & 31;
  const int64_t w = ((int64_t)blockIdx.x * 128 + threadIdx.x) >> 5;  // (group, row)
  if (w >= (int64_t)p.n_groups * kPagedRows) return;  // whole warps
  const int gi = (int)(w / kPagedRows), r = (int)(w % kPagedRows);
  const PagedGroup g = p.groups[gi];
  if (r >= g.nrows) return;
  const SeqRec sr = p.seqs[g.b];
  const int64_t t = (int64_t)sr.q_off + g.row0 + r;  // query token
  auto part_of = [&](int c) {
    const int64_t unit = (int64_t)g.unit0 + (int64_t)c * g.ustride;
    return p.part + ((unit * p.heads_per_unit + g.hslot) * kPagedRows + r) * (D + kPartPad);
  };
  float mm = -INFINITY;
  for (int c = 0; c < g.nunits; ++c) mm = fmaxf(mm, part_of(c)[D]);
  float acc[D / 32], ll = 0.f;
#pragma unroll
  for (int x = 0; x < D / 32; ++x) acc[x] = 0.f;
  for (int c = 0; c < g.nunits; ++c) {
    const float* part = part_of(c);
    const float a = rescale(part[D], mm);
    ll += part[D + 1] * a;
#pragma unroll
    for (int x = 0; x < D / 32; ++x) acc[x] += part[lane + 32 * x] * a;
  }
  const float inv = ll > 0.f ? 1.f / ll : 0.f;
  __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) + (t * p.n_heads + g.h) * D;
#pragma unroll
  for (int x = 0; x < D / 32; ++x) orow[lane + 32 * x] = __float2bfloat16_rn(acc[x] * inv);
  if (lane == 0)
    p.lse[(int64_t)g.h * p.t_q + t] = ll > 0.f ? (mm + log2f(ll)) * kLn2 : -INFINITY;
}

template <int D>
cudaError_t launch_d(int max_rows, const PagedParams& p, cudaStream_t stream) {
  const int threads = p.heads_per_unit * (D / kSlice);
  const int units = (int)p.n_units;
  if (units > 0) {
    if (max_rows <= 1) paged_partial<D, 1, 4><<<units, threads, 0, stream>>>(p);
    else paged_partial<D, kPagedRows, 2><<<units, threads, 0, stream>>>(p);
  }
  const int64_t merge_blocks = ((int64_t)p.n_groups * kPagedRows + 3) / 4;
  if (merge_blocks > 0) paged_merge<D><<<(int)merge_blocks, 128, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

int paged_heads_per_unit(int64_t n_heads, int D) {
  const int lanes = D / kSlice;           // threads per head
  const int cap = 256 / lanes;            // heads in a 256-thread CTA
  const int per_warp = 32 / lanes;        // heads per warp
  const int64_t h = n_heads < cap ? n_heads : cap;
  return (int)((h + per_warp - 1) / per_warp * per_warp);  // whole warps
}

int paged_slots(int D, int max_rows, int heads_per_unit, int num_sms) {
  const int threads = heads_per_unit * (D / kSlice);
  int per_sm = 0;
  cudaError_t e = cudaErrorInvalidValue;
  if (D == 128)
    e = max_rows <= 1 ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                            &per_sm, paged_partial<128, 1, 4>, threads, 0)
                      : cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                            &per_sm, paged_partial<128, kPagedRows, 2>, threads, 0);
  else if (D == 64)
    e = max_rows <= 1 ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                            &per_sm, paged_partial<64, 1, 4>, threads, 0)
                      : cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                            &per_sm, paged_partial<64, kPagedRows, 2>, threads, 0);
  if (e != cudaSuccess || per_sm < 1) per_sm = 1;
  return per_sm * (num_sms > 0 ? num_sms : 1);
}

cudaError_t launch_paged(int D, int max_rows, const PagedParams& p, cudaStream_t stream) {
  if (p.n_units > 0x7fffffff || (int64_t)p.n_groups * kPagedRows > 0x7fffffffLL)
    return cudaErrorInvalidValue;
  if (D == 128) return launch_d<128>(max_rows, p, stream);
  if (D == 64) return launch_d<64>(max_rows, p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace fa
