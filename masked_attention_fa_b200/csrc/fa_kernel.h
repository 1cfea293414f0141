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
  int32_t n_items;
  int32_t tnd;             // packed tokens: TMA batch coordinate 0, token = offset + row
  float scale_log2;        // scale * log2(e)
  uint32_t debug_flags;
  uint64_t timeout_ns;     // limit of every device-side wait
};

enum DebugFlags : uint32_t {
  // The TMA warp of CTA 0 never loads its first Q tile, so the MMA warp's
  // wait on it runs out: exercises the bounded-wait abort path.
  kDebugDropFirstQ = 1u,
};

// Build a 4-D bf16 tensor map over (D, S, N, B) with the given element
// strides of S, N and B, boxes of 64 x 128 x 1 x 1, 128-byte swizzle.
bool encode_operand_map(CUtensorMap* tm, const void* base, int64_t D, int64_t S, int64_t N,
                        int64_t B, int64_t st_s, int64_t st_n, int64_t st_b);

// Enqueue the kernel for head dim D on `stream` with `grid` persistent CTAs.
// Returns cudaSuccess or the launch error; `why` gets a reason for refusals.
cudaError_t launch_fwd(int D, const FwdParams& p, int grid, cudaStream_t stream,
                       const char** why);

}  // namespace fa
