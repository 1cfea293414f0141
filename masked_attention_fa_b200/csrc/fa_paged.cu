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
//   paged_partial  one CTA (4 warps) per (sequence, head, group of up to
//                  kPagedRows query rows, chunk of keys). Lane l of a warp
//                  owns D/32 consecutive dimensions of q, k, v and o; a warp
//                  takes 8 keys per step with all their loads in flight, forms
//                  each score with a butterfly sum over the warp and runs
//                  the online softmax (running max m, running sum l) per row.
//                  The four warps' (m, l, o) are combined in shared memory
//                  and the chunk's partial is written in fp32.
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

constexpr int kPagedWarps = 4;
constexpr int kPagedKeys = 8;  // keys per warp step (loads in flight)
constexpr float kLn2 = 0.69314718055994530942f;

template <int D>
struct PagedVec;
template <>
struct PagedVec<128> {  // 4 bf16 per lane
  using T = uint2;
  static __device__ __forceinline__ void unpack(const T& v, float (&f)[4]) {
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&v.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&v.y);
    const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    f[0] = fa.x, f[1] = fa.y, f[2] = fb.x, f[3] = fb.y;
  }
};
template <>
struct PagedVec<64> {  // 2 bf16 per lane
  using T = uint32_t;
  static __device__ __forceinline__ void unpack(const T& v, float (&f)[2]) {
    const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v));
    f[0] = fa.x, f[1] = fa.y;
  }
};

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int d = 16; d >= 1; d >>= 1) x += __shfl_xor_sync(0xffffffffu, x, d);
  return x;
}

// Rescale an accumulator to a larger running maximum (log2 units).
__device__ __forceinline__ float rescale(float m_old, float m_new) {
  return m_old == -INFINITY ? 0.f : exp2f(m_old - m_new);
}

template <int D>
__global__ void __launch_bounds__(kPagedWarps * 32) paged_partial(const PagedParams p) {
  constexpr int V = D / 32;  // dimensions per lane
  using Vec = PagedVec<D>;
  using T = typename Vec::T;
  __shared__ float sm_m[kPagedWarps][kPagedRows], sm_l[kPagedWarps][kPagedRows];
  __shared__ float sm_o[kPagedWarps][kPagedRows][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const PagedUnit u = p.units[blockIdx.x];
  const PagedGroup g = p.groups[u.group];
  const SeqRec sr = p.seqs[g.b];
  // This lane's slice of q for the group's rows, pre-multiplied by scale * log2(e).
  float q[kPagedRows][V];
  int jlo[kPagedRows], jhi[kPagedRows];
#pragma unroll
  for (int r = 0; r < kPagedRows; ++r) {
    jlo[r] = 1, jhi[r] = 0;
#pragma unroll
    for (int x = 0; x < V; ++x) q[r][x] = 0.f;
    if (r < g.nrows) {
      const int64_t i = (int64_t)g.row0 + r;  // row inside the sequence
      jlo[r] = (int)imax64(0, row_lo(sr, i));
      jhi[r] = (int)imin64((int64_t)sr.skv - 1, row_hi(sr, i));
      const T qv = *reinterpret_cast<const T*>(
          reinterpret_cast<const __nv_bfloat16*>(p.q) +
          (((int64_t)sr.q_off + i) * p.n_heads + g.h) * D + lane * V);
      float f[V];
      Vec::unpack(qv, f);
#pragma unroll
      for (int x = 0; x < V; ++x) q[r][x] = f[x] * p.scale_log2;
    }
  }
  float m[kPagedRows], l[kPagedRows], o[kPagedRows][V];
#pragma unroll
  for (int r = 0; r < kPagedRows; ++r) {
    m[r] = -INFINITY, l[r] = 0.f;
#pragma unroll
    for (int x = 0; x < V; ++x) o[r][x] = 0.f;
  }
  const __nv_bfloat16* kc = reinterpret_cast<const __nv_bfloat16*>(p.k_cache);
  const __nv_bfloat16* vc = reinterpret_cast<const __nv_bfloat16*>(p.v_cache);
  const int32_t* table = p.block_table + (int64_t)g.b * p.max_blocks;
  bool bad = false;
  // Keys [key0, key1): warp w takes steps of kPagedKeys keys, round robin.
  for (int j0 = u.key0 + warp * kPagedKeys; j0 < u.key1; j0 += kPagedWarps * kPagedKeys) {
    T kv[kPagedKeys], vv[kPagedKeys];
    bool ok[kPagedKeys];
#pragma unroll
    for (int e = 0; e < kPagedKeys; ++e) {
      const int j = j0 + e;
      ok[e] = false;
      if (j < u.key1) {
        const int32_t blk = __ldg(table + j / p.block_size);
        if (blk >= 0 && (int64_t)blk < p.num_blocks) {
          const int64_t slot = (int64_t)blk * p.block_size + j % p.block_size;
          const int64_t off = (slot * p.n_heads + g.h) * D + lane * V;
          kv[e] = __ldg(reinterpret_cast<const T*>(kc + off));
          vv[e] = __ldg(reinterpret_cast<const T*>(vc + off));
          ok[e] = true;
        } else {
          bad = true;
        }
      }
    }
#pragma unroll
    for (int e = 0; e < kPagedKeys; ++e) {
      if (!ok[e]) continue;  // warp-uniform: every lane saw the same block id
      const int j = j0 + e;
      float kf[V], vf[V];
      Vec::unpack(kv[e], kf);
      Vec::unpack(vv[e], vf);
#pragma unroll
      for (int r = 0; r < kPagedRows; ++r) {
        if (r >= g.nrows) break;
        float part = 0.f;
#pragma unroll
        for (int x = 0; x < V; ++x) part = fmaf(q[r][x], kf[x], part);
        const float s = warp_sum(part);
        if (j < jlo[r] || j > jhi[r]) continue;
        if (s > m[r]) {
          const float a = rescale(m[r], s);
          l[r] *= a;
#pragma unroll
          for (int x = 0; x < V; ++x) o[r][x] *= a;
          m[r] = s;
        }
        const float pj = exp2f(s - m[r]);
        l[r] += pj;
#pragma unroll
        for (int x = 0; x < V; ++x) o[r][x] = fmaf(pj, vf[x], o[r][x]);
      }
    }
  }
  if (bad && lane == 0) atomicOr(p.err_word, kErrBadBlock);
  // Combine the four warps.
#pragma unroll
  for (int r = 0; r < kPagedRows; ++r) {
    if (lane == 0) {
      sm_m[warp][r] = m[r];
      sm_l[warp][r] = l[r];
    }
#pragma unroll
    for (int x = 0; x < V; ++x) sm_o[warp][r][lane * V + x] = o[r][x];
  }
  __syncthreads();
  // Thread t writes dimension (t % D) of rows t / D, t / D + 128 / D, ...
  float* out = p.part + (int64_t)blockIdx.x * kPagedRows * (D + 2);
  for (int idx = threadIdx.x; idx < kPagedRows * D; idx += kPagedWarps * 32) {
    const int r = idx / D, x = idx % D;
    float mm = -INFINITY;
#pragma unroll
    for (int w = 0; w < kPagedWarps; ++w) mm = fmaxf(mm, sm_m[w][r]);
    float acc = 0.f, ll = 0.f;
#pragma unroll
    for (int w = 0; w < kPagedWarps; ++w) {
      const float a = rescale(sm_m[w][r], mm);
      acc += sm_o[w][r][x] * a;
      ll += sm_l[w][r] * a;
    }
    out[r * (D + 2) + x] = acc;
    if (x == 0) {
      out[r * (D + 2) + D] = mm;
      out[r * (D + 2) + D + 1] = ll;
    }
  }
}

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
  float mm = -INFINITY;
  for (int c = 0; c < g.nunits; ++c)
    mm = fmaxf(mm, p.part[((int64_t)(g.unit0 + c) * kPagedRows + r) * (D + 2) + D]);
  float acc[D / 32], ll = 0.f;
#pragma unroll
  for (int x = 0; x < D / 32; ++x) acc[x] = 0.f;
  for (int c = 0; c < g.nunits; ++c) {
    const float* part = p.part + ((int64_t)(g.unit0 + c) * kPagedRows + r) * (D + 2);
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

}  // namespace

cudaError_t launch_paged(int D, const PagedParams& p, cudaStream_t stream) {
  if (p.n_units <= 0 && p.n_groups <= 0) return cudaSuccess;
  const int64_t merge_warps = (int64_t)p.n_groups * kPagedRows;
  const int64_t merge_blocks = (merge_warps + 3) / 4;
  if (p.n_units > 0x7fffffff || merge_blocks > 0x7fffffff) return cudaErrorInvalidValue;
  if (D == 128) {
    if (p.n_units > 0) paged_partial<128><<<(int)p.n_units, kPagedWarps * 32, 0, stream>>>(p);
    if (merge_blocks > 0) paged_merge<128><<<(int)merge_blocks, 128, 0, stream>>>(p);
  } else if (D == 64) {
    if (p.n_units > 0) paged_partial<64><<<(int)p.n_units, kPagedWarps * 32, 0, stream>>>(p);
    if (merge_blocks > 0) paged_merge<64><<<(int)merge_blocks, 128, 0, stream>>>(p);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace fa
