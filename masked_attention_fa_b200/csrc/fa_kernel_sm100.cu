// Masked attention forward for B200 (sm_100a).
//
// Computes O = softmax(scale * Q K^T, restricted to the visible keys) V and
// the per-row log-sum-exp, with the online softmax of the "FlashAttention
// tiling & online softmax" exercise page (running max m_i, running sum l_i,
// section "Mục tiêu kiến thức"), never writing the score matrix out. Which
// keys are visible follows the Ascend "sparseMode参数说明" page, reduced per
// sequence to one interval of keys per query row (fa_internal.h).
//
// One persistent CTA per SM, 16 warps, warp-specialised:
//   warps 0-3   softmax of query sub-tile 0 (rows 0..127 of the item)
//   warps 4-7   softmax of query sub-tile 1 (rows 128..255)
//   warps 8-11  epilogue: O / l of both sub-tiles to global memory
//   warp 12     S = Q K^T issuer (one thread; owns TMEM)
//   warp 13     TMA producer (one thread)
//   warp 14     O += P V issuer (one thread)
//   warp 15     idle
// Tensor memory (512 columns): S0 | S1 | O0 | O1 (fp32 scores and output
// accumulators of the two sub-tiles). P = exp(S - m) in bf16 goes to its own
// buffer (shared memory at D = 128, free tensor memory columns at D = 64), so
// the softmax releases S_s as soon as it has read it and the next QK of the
// sub-tile runs while the softmax exponentiates.
// The two MMA streams are issued by two threads, so that one thread's
// barrier waits and commits (each of which stalls the tensor pipe while the
// issuing thread handles it) overlap the other thread's MMAs. The softmax
// waits for PV_s(t-1) before it overwrites the P buffer and before it
// rescales O_s in place; the epilogue waits for the item's last PV.
// Every mbarrier wait is bounded (globaltimer); on expiry the CTA records
// the site in the error word, drains its in-flight copies and MMAs, frees
// its tensor memory and exits. The two softmax warpgroups pass the
// exponential unit back and forth through hardware named barriers, which
// cannot time out: a warpgroup that leaves on an error releases the other
// one (see turn_wait).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "fa_internal.h"
#include "fa_kernel.h"
#include "fa_tmem_asm.h"

namespace fa {
namespace dev {

// Trace builds only (-DFA_TRACE=<cta>, made by masked_attention_fa_b200/
// trace.py): clock64 stamps of CTA <cta> at the points where the roles wait
// and hand work over, per key tile; compiled out of the library itself. The
// traced CTA is a compile-time constant so a stamp costs no load.
#ifdef FA_TRACE
constexpr int kTraceN = 1024;
__device__ unsigned long long g_fa_trace[8][8][kTraceN];   // [row][event][tile]
__device__ unsigned long long g_fa_wtrace[8][4][kTraceN];  // [softmax warp][event][turn]
__device__ __forceinline__ unsigned long long trace_clock() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%clock64;" : "=l"(t));
  return t;
}
#define FA_STAMP(r, e, n)                                                          \
  do {                                                                             \
    if ((int)blockIdx.x == (FA_TRACE) && (uint32_t)(n) < (uint32_t)kTraceN)      \
      g_fa_trace[r][e][n] = trace_clock();                                         \
  } while (0)
#define FA_WSTAMP(e, n)                                                                 \
  do {                                                                                  \
    if ((threadIdx.x & 31) == 0 && (int)blockIdx.x == (FA_TRACE) &&                    \
        (uint32_t)(n) < (uint32_t)kTraceN)                                              \
      g_fa_wtrace[threadIdx.x >> 5][e][n] = trace_clock();                             \
  } while (0)
// A stamp taken once the 32-bit value v exists (a load of it has landed).
#define FA_STAMP_DEP(r, e, n, v)                                                   \
  do {                                                                             \
    if ((int)blockIdx.x == (FA_TRACE) && (uint32_t)(n) < (uint32_t)kTraceN) {    \
      asm volatile("" ::"r"((uint32_t)(v)));                                       \
      g_fa_trace[r][e][n] = trace_clock();                                         \
    }                                                                              \
  } while (0)
#else
#define FA_STAMP(r, e, n) \
  do {                    \
  } while (0)
#define FA_WSTAMP(e, n) \
  do {                  \
  } while (0)
#define FA_STAMP_DEP(r, e, n, v) \
  do {                           \
  } while (0)
#endif

constexpr int kThreads = 512;
constexpr int kWarpMma = 12;
constexpr int kWarpLoad = 13;
constexpr int kWarpPv = 14;
// Register split (setmaxnreg) over the 512 x 128 registers of the launch:
// softmax warpgroups 0-1 take 192, the epilogue warpgroup 2 and the
// warpgroup of the MMA and TMA warps keep 64 each.
constexpr int kRegsSoftmax = 192;
constexpr int kRegsEpi = 64;
constexpr int kRegsControl = 64;
constexpr int kRegsTotal = 2 * 128 * kRegsSoftmax + 128 * kRegsEpi + 128 * kRegsControl;
static_assert(kRegsTotal == kThreads * 128, "register split must equal the launch allocation");
constexpr float kRescaleLog2 = 8.0f;  // rescale O only when the max grows by > 2^8

// Where a wait gave up (error word bits 8..15).
enum WaitSite : uint32_t {
  kSiteQEmpty = 1, kSiteKvEmpty = 2, kSiteQFull = 3, kSiteKvFull = 4, kSitePFull = 5,
  kSiteSFull = 6, kSiteOPv = 7, kSiteDrain = 8, kSiteSFree = 9, kSiteOFree = 10,
  kSiteMufu = 11 /* no longer waited on: the turn is a named barrier */, kSiteEpi = 12, kSiteStatFree = 13, kSiteIdxFull = 14, kSiteIdxEmpty = 15,
};

// Claimed work (the kClaim instance): the TMA thread claims the CTA's items
// and passes their indices to the other roles through a ring of kIdxSlots
// shared-memory slots, read by the QK and PV threads, the 8 softmax warps
// and the 4 epilogue warps. A claim is taken kClaimLead key tiles before
// the TMA thread's last loads of its current item.
constexpr int kIdxSlots = 8;
constexpr int kIdxReaders = 14;
constexpr int kClaimLead = 2;

template <int D>
struct Cfg {
  static constexpr int kChunks = D / 64;                 // 64-column (128-byte) chunks per row
  static constexpr uint32_t kChunkBytes = 128u * 128u;   // 128 rows x 128 bytes
  static constexpr uint32_t kTileBytes = 128u * D * 2u;  // 128 rows of Q, K or V
  // P = exp(S - m) in bf16 feeds the P.V MMA from shared memory at D = 128
  // (tensor memory is full with S0 | S1 | O0 | O1) and from its own tensor
  // memory columns at D = 64.
  static constexpr bool kPInTmem = (D == 64);
  static constexpr int kStages = (D == 128) ? 3 : 8;     // K/V ring depth
  static constexpr uint32_t kQBytes = 2u * kTileBytes;
  static constexpr uint32_t kKVBytes = kStages * kTileBytes;
  static constexpr uint32_t kPTileBytes = 128u * 128u * 2u;  // P of one sub-tile (bf16)
  static constexpr uint32_t kPBytes = kPInTmem ? 0u : 2u * kPTileBytes;
  static constexpr uint32_t kCtlBytes = 1024u;   // barriers
  static constexpr uint32_t kStatBytes = 1024u;  // 1/l of the 2 x 128 rows
  static constexpr uint32_t kSmemBytes =
      1024u + kQBytes + kKVBytes + kPBytes + kCtlBytes + kStatBytes;
  static constexpr uint32_t kTmemCols = 512u;
  // TMEM columns of S_s and of O_s
  __host__ __device__ static constexpr uint32_t col_s(int s) { return s ? 128u : 0u; }
  __host__ __device__ static constexpr uint32_t col_o(int s) { return s ? 256u + D : 256u; }
  // TMEM columns of P_s when kPInTmem (64 columns of bf16 pairs each)
  __host__ __device__ static constexpr uint32_t col_p(int s) { return 256u + 2u * D + 64u * s; }
  static_assert(!kPInTmem || 256u + 2u * D + 128u <= kTmemCols, "tensor memory budget");
  static_assert(kSmemBytes <= 227u * 1024u, "shared memory budget");
};

template <int NS>
struct Ctl {
  uint64_t q_full[2], q_empty[2];  // Q sub-tile s loaded / no longer read
  uint64_t kv_full[NS], kv_empty[NS];
  uint64_t s_full[2];  // S_s in TMEM
  uint64_t s_free[2];  // S_s read into registers: the next QK_s may overwrite it
  uint64_t p_full[2];  // P_s in shared memory
  uint64_t o_pv[2];    // one PV_s finished (O_s updated, P_s buffer free again)
  uint64_t epi_full[2];   // 1/l of sub-tile s written for the epilogue (every item)
  uint64_t stat_free[2];  // epilogue has read that 1/l (every item)
  uint64_t o_free[2];     // epilogue has read O_s (items that visit a key tile)
  uint64_t drain[2];  // one per MMA-issuing thread
  uint32_t tmem_base;
  volatile int abort_flag;
  uint64_t idx_full[kIdxSlots];   // slot holds the index of this CTA's next item
  uint64_t idx_empty[kIdxSlots];  // every reader has taken it
  int idx_ring[kIdxSlots];
};

// ----------------------------------------------------------------- basics

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 1/x and log2(x) on the exponential unit (one instruction each; relative
// error a few ulp, far inside the tolerances of O and lse).
__device__ __forceinline__ float rcp_fast(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2_fast(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// bf16x2 with `lo` in the low half (the even column of the pair).
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Three-input maximum (sm_100).
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ uint64_t pack_f32x2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}

// (a, b) <- (a, b) * m2 + c2, two lanes per instruction.
__device__ __forceinline__ void fma_x2(float& a, float& b, uint64_t m2, uint64_t c2) {
  asm("{\n\t.reg .b64 r;\n\t"
      "mov.b64 r, {%0, %1};\n\t"
      "fma.rn.f32x2 r, r, %2, %3;\n\t"
      "mov.b64 {%0, %1}, r;\n\t}"
      : "+f"(a), "+f"(b)
      : "l"(m2), "l"(c2));
}

// (a, b) += (x, y), two lanes per instruction.
__device__ __forceinline__ void add_x2(float& a, float& b, float x, float y) {
  asm("{\n\t.reg .b64 r, s;\n\t"
      "mov.b64 r, {%0, %1};\n\t"
      "mov.b64 s, {%2, %3};\n\t"
      "add.rn.f32x2 r, r, s;\n\t"
      "mov.b64 {%0, %1}, r;\n\t}"
      : "+f"(a), "+f"(b)
      : "f"(x), "f"(y));
}

// 2^x for two values on the FMA pipe instead of the MUFU unit. Cody-Waite
// reduction x = n + f with n = round(x) (adding 1.5 * 2^23 leaves n in the
// low mantissa bits), a degree-3 minimax polynomial for 2^f on [-1/2, 1/2]
// (Remez, relative error 7.5e-5; coefficients from gen_exp2_poly.py), and n
// added into the exponent field. Inputs are clamped to >= -126.
__device__ __forceinline__ void ex2_poly_x2(float& a, float& b) {
  constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
  a = fmaxf(a, -126.0f);
  b = fmaxf(b, -126.0f);
  float ta = a, tb = b;
  add_x2(ta, tb, kShift, kShift);   // t = x + shift (rounded: n in the low bits)
  float na = ta, nb = tb;
  add_x2(na, nb, -kShift, -kShift); // n = t - shift
  float fa = -na, fb = -nb;
  add_x2(fa, fb, a, b);             // f = x - n, |f| <= 1/2
  float pa = 0.05517167f, pb = 0.05517167f;
  fma_x2(pa, pb, pack_f32x2(fa, fb), pack_f32x2(0.24261113f, 0.24261113f));
  fma_x2(pa, pb, pack_f32x2(fa, fb), pack_f32x2(0.69326097f, 0.69326097f));
  fma_x2(pa, pb, pack_f32x2(fa, fb), pack_f32x2(0.99992806f, 0.99992806f));
  a = __int_as_float(__float_as_int(pa) + (__float_as_int(ta) << 23));
  b = __int_as_float(__float_as_int(pb) + (__float_as_int(tb) << 23));
}

// Columns c with (c % 8) < kPolyPer8 take the FMA-pipe exponential on tiles
// without masked entries; the rest use ex2.approx on the MUFU unit.
constexpr int kPolyPer8 = 0;

// Keys of a row exponentiated before the exponential-unit turn passes on.
constexpr int kTokenCol = 128;

// Row maximum of 128 scores: eight independent chains of 3-input maxima.
__device__ __forceinline__ float row_max128(const float (&x)[128]) {
  float m[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    float a = x[j];
#pragma unroll
    for (int r = 1; r < 15; r += 2) a = max3f(a, x[8 * r + j], x[8 * (r + 1) + j]);
    m[j] = fmaxf(a, x[120 + j]);
  }
  return max3f(max3f(m[0], m[1], m[2]), max3f(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
}

// ----------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

struct WaitCtx {
  volatile int* abort_flag;
  unsigned int* err_word;
  uint64_t timeout_ns;
};

// Wait for the phase with the given parity; false if the CTA is aborting or
// the wait outlived the limit (then the error word records the site).
// `honor_abort` = false is used by the drain waits of the abort path.
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, const WaitCtx& w,
                                          uint32_t site, bool honor_abort = true) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t spin = 1;; ++spin) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((spin & 63u) == 0u) {
      if (honor_abort && *w.abort_flag) return false;
      if (globaltimer_ns() - t0 > w.timeout_ns) {
        if (honor_abort) {
          *w.abort_flag = 1;
          atomicOr(w.err_word, kErrTimeout | (site << kErrWhereShift));
        }
        return false;
      }
    }
  }
}

// Turn of softmax warpgroup s on the exponential unit: a hardware named
// barrier (id 1 + s) over both warpgroups (256 threads). Warpgroup s waits
// on it (bar.sync); the other warpgroup hands the turn over (bar.arrive)
// once its exponentials are done. Measured against an mbarrier token polled
// with try_wait, the hand-over is ~200 cycles shorter, twice per key tile
// (+3 to +7 % on every workload).
//  - `dep` (the row maximum) is an input of the wait, so the work that
//    produces it cannot sink past it; `zero`, produced after it, is added
//    into the exponent offset, so no exponential can be hoisted above it.
//  - A named barrier cannot time out. Every wait that fails elsewhere sets
//    the abort flag, and a warpgroup leaving its loop with the flag set
//    arrives once more on the other warpgroup's barrier (turn_release), so
//    a warpgroup blocked in its turn is released; every turn re-reads the
//    flag after the barrier, so the released warpgroup leaves too. The two
//    warpgroups cannot both block: each waits only for a turn the other
//    hands over after the turn it took itself.
__device__ __forceinline__ bool turn_wait(int s, float dep, float& zero,
                                          const volatile int* abort_flag) {
  asm volatile("bar.sync %0, 256;" ::"r"(1 + s), "f"(dep));
  uint32_t f;
  asm volatile("ld.volatile.shared.u32 %0, [%1];"
               : "=r"(f)
               : "r"(smem_u32(const_cast<const int*>(abort_flag))));
  asm volatile("mov.b32 %0, 0f00000000;" : "=f"(zero));
  return __all_sync(0xffffffffu, f == 0u);
}

// Hands the exponential unit to warpgroup s_other once `dep` (a value
// computed from every exponential of this turn) exists. Whole warps.
__device__ __forceinline__ void turn_pass(int s_other, float dep) {
  asm volatile("bar.arrive %0, 256;" ::"r"(1 + s_other), "f"(dep));
}

// Called by a whole warp as it leaves the softmax loop: after an error,
// release the other warpgroup from a turn it may be waiting for.
__device__ __forceinline__ void turn_release(int s_other, const volatile int* abort_flag) {
  __syncwarp();
  if (__any_sync(0xffffffffu, *abort_flag != 0)) turn_pass(s_other, 0.f);
}

// Whole-warp wait: every lane waits, the warp proceeds only if all did.
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, const WaitCtx& w,
                                          uint32_t site) {
  const bool ok = wait_bounded(bar, parity, w, site);
  return __all_sync(0xffffffffu, ok);
}

// k-th item index of this CTA into the ring (TMA thread). The arrive
// releases the store; the readers' wait acquires it.
template <int NS>
__device__ __forceinline__ bool idx_publish(Ctl<NS>* ctl, int k, int idx, const WaitCtx& w) {
  const int slot = k % kIdxSlots;
  if (k >= kIdxSlots &&
      !wait_bounded(&ctl->idx_empty[slot], ((k / kIdxSlots) - 1) & 1u, w, kSiteIdxEmpty))
    return false;
  ctl->idx_ring[slot] = idx;
  mbar_arrive(&ctl->idx_full[slot]);
  return true;
}

// k-th item index of this CTA (one thread); INT_MAX, which ends every role's
// list, when the wait gave up.
template <int NS>
__device__ __forceinline__ int idx_take(Ctl<NS>* ctl, int k, const WaitCtx& w) {
  const int slot = k % kIdxSlots;
  if (!wait_bounded(&ctl->idx_full[slot], (k / kIdxSlots) & 1u, w, kSiteIdxFull))
    return 0x7fffffff;
  const int idx = *reinterpret_cast<volatile int*>(&ctl->idx_ring[slot]);
  mbar_arrive(&ctl->idx_empty[slot]);
  return idx;
}

// The same for a whole warp: one release per warp, after every lane read.
template <int NS>
__device__ __forceinline__ int idx_take_warp(Ctl<NS>* ctl, int k, const WaitCtx& w) {
  const int slot = k % kIdxSlots;
  if (!wait_warp(&ctl->idx_full[slot], (k / kIdxSlots) & 1u, w, kSiteIdxFull)) return 0x7fffffff;
  const int idx = *reinterpret_cast<volatile int*>(&ctl->idx_ring[slot]);
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(&ctl->idx_empty[slot]);
  return idx;
}

// ----------------------------------------------------------------- tcgen05

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (SM100 layout type 2,
// descriptor version 1). Byte offsets lbo/sbo as the canonical layouts use:
//   K-major:  rows 128 B apart, 8-row groups sbo = 1024 B apart (lbo unused);
//   MN-major: 64-element MN blocks lbo apart, 8-row K groups sbo apart.
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, kind::f16: bf16 x bf16 -> fp32, A K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(uint32_t M, uint32_t N, bool b_mn_major) {
  return (1u << 4)     // D format: f32
         | (1u << 7)   // A format: bf16
         | (1u << 10)  // B format: bf16
         | ((b_mn_major ? 1u : 0u) << 16) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b,
                                       uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

// Arrive on `bar` once every tcgen05.mma issued so far by this thread is done.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* tm, uint64_t* bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
      "r"(smem_u32(bar))
      : "memory");
}

// ----------------------------------------------------------------- schedule

// k-th item of this CTA: items are in descending-cost order and dealt out
// in a snake (0..G-1, G-1..0, ...), which evens out the per-CTA sums.
__device__ __forceinline__ int item_index(int k) {
  const int G = gridDim.x, c = blockIdx.x;
  return k * G + ((k & 1) ? (G - 1 - c) : c);
}

// Walk over an item's key tiles [lo, hi): ascending, or, with kRev (the
// ALiBi instances), descending from the diagonal. ALiBi raises a row's
// scores towards the diagonal by up to slope * 128 per tile, so an
// ascending walk raises the running maximum on almost every tile, and every
// raise by more than the rescale threshold rescales O; walking down from the
// diagonal meets the largest bias first. Written so that the ascending walk
// compiles to the plain loop.
template <bool kRev>
__device__ __forceinline__ int walk_first(int lo, int hi) { return kRev ? hi - 1 : lo; }
template <bool kRev>
__device__ __forceinline__ bool walk_in(int t, int lo, int hi) { return kRev ? t >= lo : t < hi; }
template <bool kRev>
__device__ __forceinline__ int walk_last(int lo, int hi) { return kRev ? lo : hi - 1; }
template <bool kRev>
constexpr int kWalkStep = kRev ? -1 : 1;

struct ItemPlan {
  TileRange tr[2];
  int lo, hi;      // union of the two sub-tiles' tile ranges
  int nsub;        // sub-tiles with at least one stored row
};

// Key-tile range of query sub-tile st of item it. With kOcc (p.item_tr set:
// the host's closed-form ranges, or for a dense attenMask the ranges the
// occupancy pre-pass reduced the mask to) it is read from beside work item
// idx, one load that does not wait for the item record; without, it is
// computed from the sequence record (the allocation-free fallback). Every
// role derives its tile sequence from this one function.
template <bool kOcc>
__device__ __forceinline__ TileRange sub_range(const FwdParams& p, int idx, const WorkItem& it,
                                               const SeqRec& s, int st) {
  if constexpr (kOcc) {
    // item_tr is 256-byte aligned and 16 bytes per entry: one vector load.
    const int4 v = __ldg(reinterpret_cast<const int4*>(p.item_tr) + 2 * (int64_t)idx + st);
    return TileRange{v.x, v.y, v.z, v.w};
  } else {
    return tile_range(s, (int64_t)it.qblk * kBlockM + st * kTileM);
  }
}

template <bool kOcc>
__device__ __forceinline__ ItemPlan plan_item(const FwdParams& p, int idx, const WorkItem& it,
                                              const SeqRec& s) {
  ItemPlan ip;
  ip.lo = 0x7fffffff;
  ip.hi = 0;
  ip.nsub = 0;
#pragma unroll
  for (int st = 0; st < 2; ++st) {
    const int64_t r0 = (int64_t)it.qblk * kBlockM + st * kTileM;
    ip.tr[st] = sub_range<kOcc>(p, idx, it, s, st);
    if (r0 < s.sq) ip.nsub = st + 1;
    if (ip.tr[st].hi > ip.tr[st].lo) {
      ip.lo = min(ip.lo, ip.tr[st].lo);
      ip.hi = max(ip.hi, ip.tr[st].hi);
    }
  }
  if (ip.hi == 0) ip.lo = 0;
  return ip;
}

__device__ __forceinline__ bool active(const TileRange& t, int j) { return j >= t.lo && j < t.hi; }

// ----------------------------------------------------------------- roles

// TMA producer (one thread). The ring carries K and V tiles in exactly the
// order the MMA warp consumes them: K(t+1) ahead of V(t) (the scores of tile
// t+1 are computed before P(t) is multiplied by V(t)), and an item's first K
// ahead of the previous item's last V. Per item: Q of sub-tile 0, the first
// K tile, Q of sub-tile 1, the previous item's last V, then K(t+1), V(t)
// for the item's key tiles but the last, whose V waits for the next item's
// first K (or the end of the work list). A Q tile is loaded once its buffer
// is released by the last QK of the previous item on that sub-tile; placing
// Q1 after the first K keeps a late Q1 release from holding back K.
// With kClaim this thread also takes the CTA's items: it publishes the index
// of each into the ring, the next one once its claim returns, before the
// loads the other roles need to finish the current item.
template <int D, bool kOcc, bool kClaim, bool kRev>
__device__ void load_role(const FwdParams& p, Ctl<Cfg<D>::kStages>* ctl, uint8_t* sQ,
                          uint8_t* sKV, const WaitCtx& w) {
  using C = Cfg<D>;
  constexpr int NS = C::kStages;
  uint32_t ring = 0;
  uint32_t nq[2] = {0u, 0u};
  bool ok = true;
  auto load_q = [&](const WorkItem& it, const SeqRec& sr, int st, int bc) -> bool {
    if (nq[st] > 0 && !wait_bounded(&ctl->q_empty[st], (nq[st] - 1) & 1u, w, kSiteQEmpty))
      return false;
    const bool drop = (p.debug_flags & kDebugDropFirstQ) && blockIdx.x == 0 && nq[0] + nq[1] == 0;
    if (!drop) {
      mbar_expect_tx(&ctl->q_full[st], C::kTileBytes);
      const int row = sr.q_off + it.qblk * kBlockM + st * kTileM;
#pragma unroll
      for (int c = 0; c < C::kChunks; ++c)
        tma_load_4d(sQ + st * C::kTileBytes + c * C::kChunkBytes, &p.tm_q, &ctl->q_full[st],
                    c * 64, row, it.h, bc);
    }
    ++nq[st];
    return true;
  };
  auto load_kv = [&](const CUtensorMap* tm, int row, int h, int bc) -> bool {
    const uint32_t st = ring % NS;
    FA_STAMP(6, 0, ring);
    if (ring >= (uint32_t)NS &&
        !wait_bounded(&ctl->kv_empty[st], ((ring / NS) - 1) & 1u, w, kSiteKvEmpty))
      return false;
    FA_STAMP(6, 1, ring);
    mbar_expect_tx(&ctl->kv_full[st], C::kTileBytes);
#pragma unroll
    for (int c = 0; c < C::kChunks; ++c)
      tma_load_4d(sKV + st * C::kTileBytes + c * C::kChunkBytes, tm, &ctl->kv_full[st], c * 64,
                  row, h, bc);
    ++ring;
    return true;
  };
  struct PendingV {
    int row, h, bc;
  } pend{0, -1, 0};
  if constexpr (!kClaim) {
  for (int k = 0; ok; ++k) {
    const int idx = item_index(k);
    if (idx >= p.n_items) break;
    const WorkItem it = p.items[idx];
    const SeqRec sr = p.seqs[it.b];
    const ItemPlan ip = plan_item<kOcc>(p, idx, it, sr);
    if (ip.hi <= ip.lo) continue;
    const int bc = p.tnd ? 0 : it.b;
    constexpr int st = kWalkStep<kRev>;
    if (ip.tr[0].hi > ip.tr[0].lo) ok = load_q(it, sr, 0, bc);
    if (ok) ok = load_kv(&p.tm_k, sr.kv_off + walk_first<kRev>(ip.lo, ip.hi) * kTileN, it.h, bc);
    if (ok && ip.tr[1].hi > ip.tr[1].lo) ok = load_q(it, sr, 1, bc);
    // The previous item's last V follows this item's first K: the MMA warp
    // computes those scores before it finishes the previous item.
    if (ok && pend.h >= 0) ok = load_kv(&p.tm_v, pend.row, pend.h, pend.bc);
    for (int t = walk_first<kRev>(ip.lo, ip.hi); walk_in<kRev>(t + st, ip.lo, ip.hi) && ok;
         t += st) {
      ok = load_kv(&p.tm_k, sr.kv_off + (t + st) * kTileN, it.h, bc);
      if (ok) ok = load_kv(&p.tm_v, sr.kv_off + t * kTileN, it.h, bc);
    }
    pend = PendingV{sr.kv_off + walk_last<kRev>(ip.lo, ip.hi) * kTileN, it.h, bc};
  }
  } else {
  int idx = item_index(0);
  ok = idx_publish(ctl, 0, idx, w);
  for (int k = 0; ok && idx < p.n_items; ++k) {
    const WorkItem it = p.items[idx];
    const SeqRec sr = p.seqs[it.b];
    const ItemPlan ip = plan_item<kOcc>(p, idx, it, sr);
    // Items without a key tile come last: the first one this CTA claims ends
    // its loads, so the last V goes now, not after the remaining claims (the
    // PV thread needs it before the other roles can finish the current item
    // and free the ring slots those claims need).
    if (ip.hi <= ip.lo && pend.h >= 0) {
      ok = load_kv(&p.tm_v, pend.row, pend.h, pend.bc);
      pend.h = -1;
    }
    unsigned int ticket = 0u;
    bool claimed = false;
    if (ok && ip.hi > ip.lo) {
      const int bc = p.tnd ? 0 : it.b;
      constexpr int st = kWalkStep<kRev>;
      // kClaimLead tiles before the walk's last
      const int claim_at = kRev ? min(ip.hi - 1, ip.lo + kClaimLead)
                                : max(ip.lo, ip.hi - 1 - kClaimLead);
      if (ip.tr[0].hi > ip.tr[0].lo) ok = load_q(it, sr, 0, bc);
      if (ok) ok = load_kv(&p.tm_k, sr.kv_off + walk_first<kRev>(ip.lo, ip.hi) * kTileN, it.h, bc);
      if (ok && ip.tr[1].hi > ip.tr[1].lo) ok = load_q(it, sr, 1, bc);
      if (ok && pend.h >= 0) ok = load_kv(&p.tm_v, pend.row, pend.h, pend.bc);
      for (int t = walk_first<kRev>(ip.lo, ip.hi); walk_in<kRev>(t + st, ip.lo, ip.hi) && ok;
           t += st) {
        // The claim's result is first used after this loop, so its round
        // trip overlaps the item's last loads.
        if (!claimed && (kRev ? t <= claim_at : t >= claim_at)) {
          ticket = atomicAdd(p.claim, 1u);
          claimed = true;
        }
        ok = load_kv(&p.tm_k, sr.kv_off + (t + st) * kTileN, it.h, bc);
        if (ok) ok = load_kv(&p.tm_v, sr.kv_off + t * kTileN, it.h, bc);
      }
      pend = PendingV{sr.kv_off + walk_last<kRev>(ip.lo, ip.hi) * kTileN, it.h, bc};
    }
    if (!ok) break;
    if (!claimed) ticket = atomicAdd(p.claim, 1u);
    const int next = (int)(gridDim.x + ticket);  // at most n_items + gridDim.x - 1
    if (next < p.n_items) {
      asm volatile("prefetch.global.L1 [%0];" ::"l"(p.items + next));
      if constexpr (kOcc) asm volatile("prefetch.global.L1 [%0];" ::"l"(p.item_tr + 2 * next));
    }
    ok = idx_publish(ctl, k + 1, next, w);
    idx = next;
  }
  }
  if (ok && pend.h >= 0) ok = load_kv(&p.tm_v, pend.row, pend.h, pend.bc);
  if (!ok) {
    // Abort: let every copy this thread started land before the CTA exits.
    const uint32_t first = ring > (uint32_t)NS ? ring - NS : 0u;
    for (uint32_t r = first; r < ring; ++r)
      wait_bounded(&ctl->kv_full[r % NS], (r / NS) & 1u, w, kSiteDrain, false);
    for (int st = 0; st < 2; ++st)
      if (nq[st] > 0) wait_bounded(&ctl->q_full[st], (nq[st] - 1) & 1u, w, kSiteDrain, false);
  }
}

template <int D>
__device__ __forceinline__ void issue_qk(uint32_t tmem, const uint8_t* sQ, const uint8_t* sKV,
                                         int sub, uint32_t kst) {
  using C = Cfg<D>;
  constexpr uint32_t idesc = idesc_bf16(128, 128, false);
  // K-major, 128-byte swizzle: step k advances 32 bytes inside a 128-byte
  // row, every 4 steps move to the next 64-column chunk.
  const uint64_t a0 = sdesc(smem_u32(sQ) + sub * C::kTileBytes, 16u, 1024u);
  const uint64_t b0 = sdesc(smem_u32(sKV) + kst * C::kTileBytes, 16u, 1024u);
  const uint32_t d = tmem + C::col_s(sub);
#pragma unroll 1
  for (int k = 0; k < D / 16; ++k) {
    const uint64_t off = (uint64_t)(((k >> 2) * C::kChunkBytes + (k & 3) * 32u) >> 4);
    mma_ss(d, a0 + off, b0 + off, idesc, k > 0 ? 1u : 0u);
  }
}

template <int D>
__device__ __forceinline__ void issue_pv(uint32_t tmem, const uint8_t* sP, const uint8_t* sKV,
                                         int sub, uint32_t vst, bool accumulate) {
  using C = Cfg<D>;
  constexpr uint32_t idesc = idesc_bf16(128, D, true);
  // V is MN-major (D contiguous): step k moves 16 key rows = 2048 bytes.
  const uint64_t b0 = sdesc(smem_u32(sKV) + vst * C::kTileBytes, C::kChunkBytes, 1024u);
  const uint32_t d = tmem + C::col_o(sub);
  if constexpr (C::kPInTmem) {
    // P in tensor memory: 16 keys = 8 columns of bf16 pairs per step.
    const uint32_t a = tmem + C::col_p(sub);
#pragma unroll
    for (int k = 0; k < kTileN / 16; ++k)
      mma_ts(d, a + k * 8u, b0 + (uint64_t)(k * (2048u >> 4)), idesc,
             (accumulate || k > 0) ? 1u : 0u);
  } else {
    // P in shared memory, K-major like Q: step k advances 32 bytes in a
    // 128-byte row, every 4 steps the next 64-key chunk.
    const uint64_t a0 = sdesc(smem_u32(sP) + sub * C::kPTileBytes, 16u, 1024u);
#pragma unroll
    for (int k = 0; k < kTileN / 16; ++k) {
      const uint64_t a_off = (uint64_t)(((k >> 2) * C::kChunkBytes + (k & 3) * 32u) >> 4);
      mma_ss(d, a0 + a_off, b0 + (uint64_t)(k * (2048u >> 4)), idesc,
             (accumulate || k > 0) ? 1u : 0u);
    }
  }
}

// Key-tile ranges of an item as the MMA warps need them: sub-tile s visits
// [lo[s], hi[s]), the item visits [lo[2], hi[2]); `pos` is the item's
// position in this CTA's list.
struct MmaPlan {
  int lo[3], hi[3];
  int pos;
};

// Key-tile ranges of item idx; false when it has no key tile.
template <bool kOcc>
__device__ __forceinline__ bool mma_plan(const FwdParams& p, int idx, MmaPlan& mp) {
  const WorkItem it = p.items[idx];
  const ItemPlan ip = plan_item<kOcc>(p, idx, it, p.seqs[it.b]);
  if (ip.hi <= ip.lo) return false;
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    mp.lo[s] = ip.tr[s].lo;
    mp.hi[s] = ip.tr[s].hi;
  }
  mp.lo[2] = ip.lo;
  mp.hi[2] = ip.hi;
  return true;
}

// Next item of this CTA with at least one key tile, from position k on:
// computed from the snake, or (kRing) read from the index ring, every slot
// up to the one that ends the list.
template <bool kOcc, bool kRing, int NS>
__device__ __forceinline__ bool next_item(const FwdParams& p, Ctl<NS>* ctl, const WaitCtx& w,
                                          int& k, MmaPlan& mp) {
  for (;; ++k) {
    int idx;
    if constexpr (kRing) idx = idx_take(ctl, k, w);
    else idx = item_index(k);
    if (idx >= p.n_items) return false;
    if (mma_plan<kOcc>(p, idx, mp)) {
      mp.pos = k;
      ++k;
      return true;
    }
  }
}

__device__ __forceinline__ bool act(const MmaPlan& mp, int s, int t) {
  return t >= mp.lo[s] && t < mp.hi[s];
}

// Ring position of the K and V tiles of the g-th key tile this CTA visits
// (counted over its items in order). The TMA producer loads K(g+1) ahead of
// V(g): K(0), K(1), V(0), K(2), V(1), ..., K(last), V(last-1), V(last).
__device__ __forceinline__ uint32_t ring_k(uint32_t g) { return g == 0 ? 0u : 2u * g - 1u; }
__device__ __forceinline__ uint32_t ring_v(uint32_t g, bool last) {
  return last ? 2u * g + 1u : 2u * g + 2u;
}

// S = Q K^T issue (one thread). Walks the CTA's key tiles in order; for each
// tile t of an item and each sub-tile s that visits it, waits until the
// softmax has read S_s of the previous tile and issues S_s = Q_s K(t)^T.
// It runs ahead of the P.V stream (another thread), limited only by the
// softmax releasing S, so the scores of the next tile, also across item
// boundaries, are ready when the softmax wants them.
template <int D, bool kOcc, bool kClaim, bool kRev>
__device__ void qk_role(const FwdParams& p, Ctl<Cfg<D>::kStages>* ctl, uint32_t tmem,
                        const uint8_t* sQ, const uint8_t* sKV, const WaitCtx& w) {
  using C = Cfg<D>;
  constexpr int NS = C::kStages;
  uint32_t g = 0;                  // key tiles visited so far
  uint32_t nq[2] = {0u, 0u};       // Q loads awaited per sub-tile
  uint32_t n_qk[2] = {0u, 0u};     // QK MMAs issued per sub-tile
  bool ok = true;
  int k = 0;
  MmaPlan cur;
  while (ok && next_item<kOcc, kClaim>(p, ctl, w, k, cur)) {
    bool q_ready[2] = {false, false};
    for (int t = walk_first<kRev>(cur.lo[2], cur.hi[2]); walk_in<kRev>(t, cur.lo[2], cur.hi[2]) && ok;
         t += kWalkStep<kRev>, ++g) {
      const uint32_t r = ring_k(g);
      FA_STAMP(2, 0, g);
      if (!wait_bounded(&ctl->kv_full[r % NS], (r / NS) & 1u, w, kSiteKvFull)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        if (!act(cur, s, t)) continue;
        if (!q_ready[s]) {
          if (!wait_bounded(&ctl->q_full[s], nq[s] & 1u, w, kSiteQFull)) {
            ok = false;
            break;
          }
          ++nq[s];
          q_ready[s] = true;
        }
        FA_STAMP(2, 2 + s, g);
        if (n_qk[s] > 0 &&
            !wait_bounded(&ctl->s_free[s], (n_qk[s] - 1) & 1u, w, kSiteSFree)) {
          ok = false;
          break;
        }
        tc_fence_after();
        FA_STAMP(2, 4 + s, g);
        issue_qk<D>(tmem, sQ, sKV, s, r % NS);
        mma_commit(&ctl->s_full[s]);
        ++n_qk[s];
        // last read of this Q
        if (t == walk_last<kRev>(cur.lo[s], cur.hi[s])) mma_commit(&ctl->q_empty[s]);
      }
      if (ok) mma_commit(&ctl->kv_empty[r % NS]);
    }
  }
  // Wait until every MMA this thread issued (and its commits) has finished
  // with tensor and shared memory.
  mma_commit(&ctl->drain[0]);
  wait_bounded(&ctl->drain[0], 0u, w, kSiteDrain, false);
}

// O += P V issue (one thread). For each key tile t and each sub-tile that
// visits it, waits for P_s(t) from the softmax and issues O_s += P_s V(t);
// the commit after it tells the softmax that O_s is updated and that the P
// buffer may be rewritten. The first PV of an item overwrites O_s, so it
// waits until the epilogue has read O_s of the previous item that had one.
template <int D, bool kOcc, bool kClaim, bool kRev>
__device__ void pv_role(const FwdParams& p, Ctl<Cfg<D>::kStages>* ctl, uint32_t tmem,
                        const uint8_t* sP, const uint8_t* sKV, const WaitCtx& w) {
  using C = Cfg<D>;
  constexpr int NS = C::kStages;
  uint32_t g = 0;
  uint32_t p_count[2] = {0u, 0u};  // P tiles consumed per sub-tile
  uint32_t n_act[2] = {0u, 0u};    // items so far in which sub-tile s visits a key tile
  bool ok = true;
  int k = 0;
  MmaPlan cur;
  bool have = next_item<kOcc, kClaim>(p, ctl, w, k, cur);
  bool at_end = !have;  // kClaim: the slot that ends the list has been read
  while (ok && have) {
    MmaPlan nxt;
    bool have_next = false;
    if constexpr (!kClaim) have_next = next_item<kOcc, false>(p, ctl, w, k, nxt);
    bool first[2] = {true, true};
    for (int t = walk_first<kRev>(cur.lo[2], cur.hi[2]); walk_in<kRev>(t, cur.lo[2], cur.hi[2]) && ok;
         t += kWalkStep<kRev>, ++g) {
      const bool last_t = t == walk_last<kRev>(cur.lo[2], cur.hi[2]);
      if constexpr (kClaim) {
        // A claimed next item is known once the TMA thread's claim returns,
        // published before it loads this item's last V: look at one slot at
        // the last key tile. Items without a key tile come last, so one of
        // them (or the end of the list) ends this thread's MMAs; the slots
        // after it are read once those are issued.
        if (last_t) {
          const int nidx = idx_take(ctl, k, w);
          ++k;
          if (nidx >= p.n_items) at_end = true;
          else have_next = mma_plan<kOcc>(p, nidx, nxt);
        }
      }
      const uint32_t r = ring_v(g, !have_next && last_t);
      FA_STAMP(3, 0, g);
      if (!wait_bounded(&ctl->kv_full[r % NS], (r / NS) & 1u, w, kSiteKvFull)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        if (!act(cur, s, t)) continue;
        FA_STAMP(3, 2 + s, g);
        if (!wait_bounded(&ctl->p_full[s], p_count[s] & 1u, w, kSitePFull)) {
          ok = false;
          break;
        }
        ++p_count[s];
        // o_free[s] completes one phase per item that visits a key tile of
        // sub-tile s: wait for the one of the previous such item.
        if (first[s]) {
          if (n_act[s] > 0 &&
              !wait_bounded(&ctl->o_free[s], (n_act[s] - 1) & 1u, w, kSiteOFree)) {
            ok = false;
            break;
          }
          ++n_act[s];
        }
        tc_fence_after();
        FA_STAMP(3, 4 + s, g);
        issue_pv<D>(tmem, sP, sKV, s, r % NS, !first[s]);
        first[s] = false;
        mma_commit(&ctl->o_pv[s]);
      }
      if (ok) mma_commit(&ctl->kv_empty[r % NS]);
    }
    cur = nxt;
    have = have_next;
  }
  if constexpr (kClaim) {
    if (ok && !at_end)
      while (idx_take(ctl, k++, w) < p.n_items) {
      }
  }
  mma_commit(&ctl->drain[1]);
  wait_bounded(&ctl->drain[1], 0u, w, kSiteDrain, false);
}

// Scores of this thread's row (128 keys of S_s) with the element mask of a
// boundary tile applied (-inf where the key is not visible). The visible
// columns [c_lo, c_hi] and, for a dense mask, its bits become four words of
// one bit per key, and each score is kept or replaced by one bit test (a
// quarter of the cost of a range compare per key, measured).
__device__ __forceinline__ void load_scores(uint32_t tS, float (&x)[128], bool partial, int c_lo,
                                            int c_hi, bool dense, const uint32_t (&mbits)[4]) {
  uint32_t sv[128];
  tmem_ld128_wait(tS, sv);
#pragma unroll
  for (int c = 0; c < 128; ++c) x[c] = __uint_as_float(sv[c]);
  if (partial) {
    // One bit per key: visible = inside [c_lo, c_hi] and (dense) unmasked.
    uint32_t wm[4];
#pragma unroll
    for (int wd = 0; wd < 4; ++wd) {
      const int a = c_lo - 32 * wd, b = c_hi - 32 * wd;  // visible bits [a, b] of this word
      const uint32_t upto = b >= 31 ? 0xffffffffu : (b < 0 ? 0u : (0xffffffffu >> (31 - b)));
      const uint32_t from = a <= 0 ? 0xffffffffu : (a > 31 ? 0u : (0xffffffffu << a));
      wm[wd] = upto & from & ~(dense ? mbits[wd] : 0u);
    }
#pragma unroll
    for (int c = 0; c < 128; ++c)
      x[c] = ((wm[c >> 5] >> (c & 31)) & 1u) ? x[c] : -INFINITY;
  }
}

// x <- 2^(x * scale_log2 - ref) for the 128 keys of the row, packed into 64
// bf16 pairs (even key in the low half); returns the row sum of the fp32
// values (eight independent partial sums).
template <bool kPoly, int kC0 = 0, int kC1 = 128>
__device__ __forceinline__ void exp_pack_part(const float (&x)[128], uint64_t m2, uint64_t c2,
                                              float (&acc)[8], uint32_t (&pk)[64]) {
#pragma unroll
  for (int c = kC0; c < kC1; c += 2) {
    float a = x[c], b = x[c + 1];
    fma_x2(a, b, m2, c2);
    if (kPoly && (c & 7) < kPolyPer8) {
      ex2_poly_x2(a, b);
    } else {
      a = ex2(a);
      b = ex2(b);
    }
    const int k = (c >> 1) & 3;
    add_x2(acc[2 * k], acc[2 * k + 1], a, b);
    pk[c >> 1] = pack_bf16(a, b);
  }
}

// ALiBi: scores of the row's 128 keys of this tile in log2 units with the
// bias added, a2 = slope * log2(e). d0 is the signed distance of the tile's
// first key from the row's diagonal anchored at the bottom-right corner (key
// c is d0 + c away). The linear bias (right-aligned; the left-aligned one
// differs by a constant per row, applied to lse at the end) leaves
// x <- x * scale_log2 + a2 * c, without the tile's offset a2 * d0; the
// square-root variant adds its whole bias, x <- x * scale_log2 +
// a2 * sign(d) sqrt|d|, with sqrt on the MUFU unit. Hidden keys stay -inf.
__device__ __forceinline__ void apply_alibi(float (&x)[128], float scale_log2, float a2, int d0,
                                            bool sqrt_bias) {
  if (sqrt_bias) {
#pragma unroll
    for (int c = 0; c < 128; ++c) {
      const float d = (float)(d0 + c);
      float r;
      asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(fabsf(d)));
      x[c] = fmaf(x[c], scale_log2, a2 * copysignf(r, d));
    }
  } else {
    // The ramp a2 * c only: the tile's offset a2 * d0 is one scalar per row
    // that the caller adds to the row maximum and to the exponent offset, so
    // the ramp stays small and is built by additions (four interleaved chains
    // of sixteen steps of 8 a2), one packed add per two keys.
    const uint64_t s2 = pack_f32x2(scale_log2, scale_log2);
    const float st = 8.f * a2;
    float r[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) r[q] = a2 * (float)q;
#pragma unroll
    for (int c = 0; c < 128; c += 8) {
#pragma unroll
      for (int q = 0; q < 8; q += 2) {
        fma_x2(x[c + q], x[c + q + 1], s2, pack_f32x2(r[q], r[q + 1]));
        add_x2(r[q], r[q + 1], st, st);
      }
    }
  }
}

__device__ __forceinline__ float sum_acc(float (&acc)[8]) {
  add_x2(acc[0], acc[1], acc[2], acc[3]);
  add_x2(acc[4], acc[5], acc[6], acc[7]);
  add_x2(acc[0], acc[1], acc[4], acc[5]);
  return acc[0] + acc[1];
}

// O and lse stores that do not allocate in L1. The SM keeps only ~28 KB of
// L1 beside 227 KB of shared memory; 64 KB of O per item written through it
// evicts the work-item and sequence records every role reads at the next
// item boundary (measured: +5 % causal, +2 % on the other workloads).
__device__ __forceinline__ void st_global_na_v4(void* ptr, const uint4& v) {
  asm volatile("st.global.L1::no_allocate.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(ptr), "r"(v.x),
               "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
// 32 bytes in one access (ptr 32-byte aligned): a row of O leaves the SM in
// half as many accesses as with 16-byte stores. Each 16-byte store of the
// epilogue's warp touches 32 rows, and the load/store unit is shared with
// the softmax warps, whose shared-memory traffic (P) and item-boundary
// accesses wait behind the epilogue's burst: measured +2 to +4 % on causal,
// band and ALiBi, +1 % on the long-item workloads.
__device__ __forceinline__ void st_global_na_v8(void* ptr, const uint4& a, const uint4& b) {
  asm volatile("st.global.L1::no_allocate.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(
                   ptr),
               "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
               : "memory");
}
__device__ __forceinline__ void st_global_na_f32(float* ptr, float v) {
  asm volatile("st.global.L1::no_allocate.f32 [%0], %1;" ::"l"(ptr), "f"(v) : "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// Row `row` of a 128 x 128 bf16 P tile at `base` (1024-byte aligned), in the
// layout a TMA load with 128-byte swizzle gives a 64-column box and the MMA
// reads as K-major: two 64-key chunks of 16 KB, rows 128 bytes apart, and
// the 16-byte unit u of row r at unit position u ^ (r % 8). Eight
// consecutive rows cover all 32 banks, so every store is conflict-free.
__device__ __forceinline__ void store_p_smem(uint32_t base, int row, const uint32_t (&pk)[64]) {
  const uint32_t rb = base + (uint32_t)row * 128u;
  const uint32_t sw = (uint32_t)row & 7u;
#pragma unroll
  for (int u = 0; u < 16; ++u)
    st_shared_v4(rb + (uint32_t)(u >> 3) * 16384u + ((((uint32_t)u & 7u) ^ sw) << 4),
                 pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
}

// The same exponentials for all 128 keys, with P stored to shared memory as
// it is produced: each 16-byte unit (8 keys) of row `row` of the P tile at
// `base` (the layout of store_p_smem) is written as soon as it is
// packed, so the stores overlap the exponential unit's work instead of
// following it. Same sums as exp_pack_part.
__device__ __forceinline__ void exp_pack_store(const float (&x)[128], uint64_t m2, uint64_t c2,
                                               float (&acc)[8], uint32_t base, int row) {
  const uint32_t rb = base + (uint32_t)row * 128u;
  const uint32_t sw = (uint32_t)row & 7u;
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float a = x[8 * u + 2 * q], b = x[8 * u + 2 * q + 1];
      fma_x2(a, b, m2, c2);
      a = ex2(a);
      b = ex2(b);
      add_x2(acc[2 * q], acc[2 * q + 1], a, b);
      w[q] = pack_bf16(a, b);
    }
    st_shared_v4(rb + (uint32_t)(u >> 3) * 16384u + ((((uint32_t)u & 7u) ^ sw) << 4), w[0], w[1],
                 w[2], w[3]);
  }
}

// Make this thread's generic-proxy shared-memory writes visible to the
// tensor core's (async-proxy) reads that follow the next barrier.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Softmax of query sub-tile `sub` (one warpgroup, one row per thread). Per
// key tile: read S_s, release it to the next QK, row maximum, then - in
// strict alternation with the other softmax warpgroup, so that the two
// never compete for the exponential unit - exponentiate and pack P; then
// wait for the previous PV (it still reads the P buffer and O_s must hold
// it before a rescale), rescale O_s if the reference maximum moved, store P.
// Every tile of the item's union range is one turn for both warpgroups; a
// warpgroup that does not visit the tile passes its turn on. At the end of
// an item it writes the row's log-sum-exp and hands 1/l to the epilogue
// warpgroup.
// kDense: the dense-mask extras (the next mask line prefetched a tile ahead,
// 16-byte mask gathers), compiled only into the dense-mask instance.
// kAlibi: the ALiBi bias added to the scores before the row maximum.
template <int D, bool kOcc, bool kDense, bool kClaim, bool kAlibi>
__device__ void softmax_role(const FwdParams& p, Ctl<Cfg<D>::kStages>* ctl, float* inv_l_sm,
                             uint32_t tmem, uint8_t* sP, int sub, const WaitCtx& w) {
  using C = Cfg<D>;
  const int wq = (threadIdx.x >> 5) & 3;           // TMEM lane quarter of this warp
  const int lane = threadIdx.x & 31;
  const int row = wq * 32 + lane;                  // row of the sub-tile = TMEM lane
  const uint32_t lane_bits = (uint32_t)(wq * 32) << 16;
  const uint32_t tS = tmem + lane_bits + C::col_s(sub);
  const uint32_t tO = tmem + lane_bits + C::col_o(sub);
  const uint32_t tP = tmem + lane_bits + C::col_p(sub);
  const uint32_t sPs = smem_u32(sP) + sub * C::kPTileBytes;
  const float scale_log2 = p.scale_log2;
  // Dense-mask rows start on 16-byte boundaries (base and row stride); the
  // 16-byte gather below is compiled into the dense-mask variant only.
  const bool mask_vec =
      kDense && ((reinterpret_cast<uintptr_t>(p.mask) | (uintptr_t)p.m_si) & 15u) == 0;
  uint32_t s_count = 0;   // S tiles consumed
  uint32_t pv_count = 0;  // P tiles produced = PV MMAs of this sub-tile
  uint32_t turn = 0;      // exponential-unit turns taken
  bool ok = true;
  for (int k = 0; ok; ++k) {
    int idx;
    if constexpr (kClaim) idx = idx_take_warp(ctl, k, w);
    else idx = item_index(k);
    if (idx >= p.n_items) break;
    // Item boundary stamps: warpgroup 0 in row 5, warpgroup 1 in row 7.
    [[maybe_unused]] const bool stamper = (threadIdx.x & 127) == 0;
    if (stamper) FA_STAMP(sub ? 7 : 5, 0, k);
    const WorkItem it = p.items[idx];
    if (stamper) FA_STAMP_DEP(sub ? 7 : 5, 1, k, it.b ^ it.qblk);
    const SeqRec sr = p.seqs[it.b];
    if (stamper) FA_STAMP_DEP(sub ? 7 : 5, 2, k, sr.q_off ^ sr.flags);
    // The next item's record is read at the item boundary, on the critical
    // path of the exponential-unit turns: pull it into L1 now (a claimed
    // item is prefetched by the TMA thread once its claim returns).
    if (!kClaim && lane == 0 && item_index(k + 1) < p.n_items) {
      asm volatile("prefetch.global.L1 [%0];" ::"l"(p.items + item_index(k + 1)));
      if constexpr (kOcc)
        asm volatile("prefetch.global.L1 [%0];" ::"l"(p.item_tr + 2 * item_index(k + 1)));
    }
    const ItemPlan ip = plan_item<kOcc>(p, idx, it, sr);
    // sub is a run-time value: select, so the plan stays in registers (an
    // indexed copy would live on the stack, in the SM's small L1).
    const TileRange tr = sub == 0 ? ip.tr[0] : ip.tr[1];
    if (stamper) FA_STAMP_DEP(sub ? 7 : 5, 3, k, ip.lo ^ tr.hi);
    const int64_t r0 = (int64_t)it.qblk * kBlockM + sub * kTileM;
    const int i = (int)(r0 + row);  // query row inside the sequence
    const bool row_valid = i < sr.sq;
    // Visible keys of this row: [jlo, jhi] (empty when jlo > jhi).
    int jlo = 1, jhi = 0;
    if (row_valid) {
      jlo = (int)imax64(0, row_lo(sr, i));
      jhi = (int)imin64((int64_t)sr.skv - 1, row_hi(sr, i));
    }
    // ALiBi: slope of the head, in log2 units, and the distance of key 0
    // from this row's bottom-right-anchored diagonal.
    float slope = 0.f, a2 = 0.f;
    int dbase = 0;
    if constexpr (kAlibi) {
      slope = __ldg(p.slopes + it.h);
      a2 = slope * 1.4426950408889634f;
      dbase = -(i + (sr.skv - sr.sq));
    }
    const uint8_t* mrow = nullptr;
    if ((sr.flags & kSeqDenseMask) && row_valid)
      mrow = p.mask + it.b * p.m_sb + it.h * p.m_sh + (int64_t)i * p.m_si;
    float m_used = -INFINITY;  // reference max (log2 units, scaled)
    float l = 0.f;             // running sum relative to m_used
    // Dense-mask variant: the mask line of the next tile that needs it is
    // pulled into L1 a tile ahead, so the gather after S arrives hits L1.
    auto prefetch_mask = [&](int tn) {
      if constexpr (kDense) {
        if (mrow != nullptr && tn >= tr.lo && tn < tr.hi && !(tn >= tr.full_lo && tn < tr.full_hi))
          asm volatile("prefetch.global.L1 [%0];" ::"l"(mrow + (int64_t)tn * kTileN));
      }
    };
    prefetch_mask(walk_first<kAlibi>(tr.lo, tr.hi));
    if (stamper) FA_STAMP_DEP(sub ? 7 : 5, 4, k, jlo ^ jhi);
    // The ALiBi instances walk the tiles down from the diagonal (walk_first).
    for (int t = walk_first<kAlibi>(ip.lo, ip.hi); walk_in<kAlibi>(t, ip.lo, ip.hi);
         t += kWalkStep<kAlibi>) {
      // Turn on the exponential unit: warpgroup 0 goes first in every tile.
      const bool first_turn = sub == 0 && turn == 0;
      ++turn;
      if (t < tr.lo || t >= tr.hi) {
        // Not visited by this sub-tile: pass the turn on.
        float zero = 0.f;
        if (!first_turn && !turn_wait(sub, 0.f, zero, w.abort_flag)) {
          ok = false;
          break;
        }
        turn_pass(sub ^ 1, zero);
        continue;
      }
      prefetch_mask(t + kWalkStep<kAlibi>);
      if ((threadIdx.x & 127) == 0) FA_STAMP(sub, 0, turn - 1);
      if (!wait_warp(&ctl->s_full[sub], s_count & 1u, w, kSiteSFull)) {
        ok = false;
        break;
      }
      ++s_count;
      const bool partial = !(t >= tr.full_lo && t < tr.full_hi);
      const int c_lo = jlo - t * kTileN, c_hi = jhi - t * kTileN;
      // Dense attenMask bits of this row's 128 keys (1 = hidden), gathered
      // before the scores are loaded so they cost no score registers.
      uint32_t mbits[4] = {0u, 0u, 0u, 0u};
      if (partial && mrow != nullptr) {
        const uint8_t* mt = mrow + (int64_t)t * kTileN;
        bool vec = false;
        if constexpr (kDense) vec = mask_vec && (t + 1) * kTileN <= sr.skv;
        if (vec) {
          // The whole 128-byte tile row lies inside the mask row and is
          // 16-byte aligned: eight 16-byte loads in flight at once, one bit
          // per nonzero byte. Bits outside [c_lo, c_hi] are harmless, those
          // keys are hidden by the window anyway.
          uint4 v[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) v[q] = __ldg(reinterpret_cast<const uint4*>(mt) + q);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint32_t wv[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              const uint32_t e = __vcmpne4(wv[r], 0u);  // 0xff in every nonzero byte
              const uint32_t nib =
                  (e & 1u) | ((e >> 7) & 2u) | ((e >> 14) & 4u) | ((e >> 21) & 8u);
              mbits[q >> 1] |= nib << (16 * (q & 1) + 4 * r);
            }
          }
        } else {
#pragma unroll
          for (int wd = 0; wd < 4; ++wd) {
            uint32_t bits = 0u;
#pragma unroll 1
            for (int c = wd * 32; c < wd * 32 + 32; ++c)
              if (c >= c_lo && c <= c_hi && mt[c] != 0) bits |= 1u << (c & 31);
            mbits[wd] = bits;
          }
        }
      }
      if ((threadIdx.x & 127) == 0) FA_STAMP(sub, 1, turn - 1);
      tc_fence_after();
      float x[128];
      load_scores(tS, x, partial, c_lo, c_hi, mrow != nullptr, mbits);
      if ((threadIdx.x & 127) == 0) FA_STAMP(sub, 2, turn - 1);
      // S_s is in registers: the next QK of this sub-tile may overwrite it.
      tc_fence_before();
      mbar_arrive(&ctl->s_free[sub]);
      // Without ALiBi the scale is applied inside the exponential (the max
      // of the raw scores scales, scale > 0); with it x holds the biased
      // scores in log2 units already.
      // Linear ALiBi: the tile's bias offset, a2 * (distance of its first key).
      const float abase = (kAlibi && p.alibi != 2) ? a2 * (float)(t * kTileN + dbase) : 0.f;
      if constexpr (kAlibi) apply_alibi(x, scale_log2, a2, t * kTileN + dbase, p.alibi == 2);
      const float m_new = kAlibi ? row_max128(x) + abase : row_max128(x) * scale_log2;
      const bool resc = m_new > m_used + kRescaleLog2;
      float alpha = 1.f;
      if (resc) {
        alpha = (m_used == -INFINITY) ? 0.f : ex2(m_used - m_new);
        l *= alpha;
        m_used = m_new;
      }
      float zero = 0.f;
      if ((threadIdx.x & 127) == 0) FA_STAMP(sub, 3, turn - 1);
      FA_WSTAMP(2, turn - 1);
      // With ALiBi the bias makes this warpgroup's work between two of its
      // turns longer than the other warpgroup's exponentials, so P goes to
      // shared memory while this turn's exponentials run (exp_pack_store),
      // and the wait for the previous PV moves ahead of the turn. Without it
      // that work fits, and stores inside the loop would only slow the
      // exponentials: P is stored after the turn is handed over.
      constexpr bool kStoreInTurn = kAlibi && !C::kPInTmem && kPolyPer8 == 0 && kTokenCol == 128;
      auto pv_done = [&]() -> bool {
        // The previous PV of this sub-tile must be done: it still reads the
        // P buffer, and O_s must hold it before it is rescaled.
        if (!wait_warp(&ctl->o_pv[sub], (pv_count - 1) & 1u, w, kSiteOPv)) return false;
        tc_fence_after();
        if ((threadIdx.x & 127) == 0) FA_STAMP(sub, 6, turn - 1);
        // Not on the sub-tile's first tile of the item: the first PV of an
        // item overwrites O_s.
        if ((kAlibi ? t < tr.hi - 1 : t > tr.lo) && __any_sync(0xffffffffu, resc)) {
#pragma unroll 1
          for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t ov[32];
            tmem_ld32_wait(tO + ch * 32u, ov);
#pragma unroll
            for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
            tmem_st32(tO + ch * 32u, ov);
          }
        }
        return true;
      };
      if constexpr (kStoreInTurn) {
        if (pv_count > 0 && !pv_done()) {
          ok = false;
          break;
        }
      }
      if (!first_turn && !turn_wait(sub, m_new, zero, w.abort_flag)) {
        ok = false;
        break;
      }
      if ((threadIdx.x & 127) == 0) FA_STAMP(sub, 4, turn - 1);
      FA_WSTAMP(0, turn - 1);
      const float ref = ((m_used == -INFINITY) ? 0.f : m_used) + zero;
      const float mul = kAlibi ? 1.f : scale_log2;
      const uint64_t m2 = pack_f32x2(mul, mul);
      const float off = kAlibi ? abase - ref : -ref;
      const uint64_t c2 = pack_f32x2(off, off);
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if constexpr (kStoreInTurn) {
        exp_pack_store(x, m2, c2, acc, sPs, row);
        __syncwarp();
        turn_pass(sub ^ 1, ((acc[0] + acc[1]) + (acc[2] + acc[3])) +
                               ((acc[4] + acc[5]) + (acc[6] + acc[7])));
        l += sum_acc(acc);
        fence_proxy_async_smem();
        if ((threadIdx.x & 127) == 0) FA_STAMP(sub, 5, turn - 1);
        FA_WSTAMP(1, turn - 1);
      } else {
        uint32_t pk[64];
        // The other warpgroup gets its turn once the first kTokenCol keys
        // are done, so both feed the exponential unit across the handover.
        // One instance of the exponential loop serves every tile while the
        // FMA-pipe polynomial is off: a second copy for the (rarer) boundary
        // tiles is cold in the instruction cache each time it runs.
        if constexpr (kPolyPer8 > 0) {
          if (partial) exp_pack_part<false, 0, kTokenCol>(x, m2, c2, acc, pk);
          else exp_pack_part<true, 0, kTokenCol>(x, m2, c2, acc, pk);
        } else {
          exp_pack_part<false, 0, kTokenCol>(x, m2, c2, acc, pk);
        }
        __syncwarp();
        turn_pass(sub ^ 1, ((acc[0] + acc[1]) + (acc[2] + acc[3])) +
                               ((acc[4] + acc[5]) + (acc[6] + acc[7])));
        if constexpr (kPolyPer8 > 0) {
          if (partial) exp_pack_part<false, kTokenCol, 128>(x, m2, c2, acc, pk);
          else exp_pack_part<true, kTokenCol, 128>(x, m2, c2, acc, pk);
        } else {
          exp_pack_part<false, kTokenCol, 128>(x, m2, c2, acc, pk);
        }
        l += sum_acc(acc);
        if ((threadIdx.x & 127) == 0) FA_STAMP(sub, 5, turn - 1);
        FA_WSTAMP(1, turn - 1);
        if (pv_count > 0 && !pv_done()) {
          ok = false;
          break;
        }
        if constexpr (C::kPInTmem) {
          tmem_st32(tP, *reinterpret_cast<const uint32_t(*)[32]>(&pk[0]));
          tmem_st32(tP + 32u, *reinterpret_cast<const uint32_t(*)[32]>(&pk[32]));
        } else {
          store_p_smem(sPs, row, pk);
          fence_proxy_async_smem();
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&ctl->p_full[sub]);
      if ((threadIdx.x & 127) == 0) FA_STAMP(sub, 7, turn - 1);
      FA_WSTAMP(3, turn - 1);
      ++pv_count;
    }
    if (!ok) break;
    if (stamper) FA_STAMP(sub ? 7 : 5, 5, k);
    // lse = ln(sum exp(scale q.k)); 1/l goes to the epilogue once it has
    // taken the previous item's value.
    if (k > 0 && !wait_warp(&ctl->stat_free[sub], (k - 1) & 1u, w, kSiteStatFree)) {
      ok = false;
      break;
    }
    if (stamper) FA_STAMP(sub ? 7 : 5, 6, k);
    inv_l_sm[sub * kTileM + row] = l > 0.f ? rcp_fast(l) : 0.f;
    mbar_arrive(&ctl->epi_full[sub]);
    if (row_valid) {
      float lse = l > 0.f ? (m_used + lg2_fast(l)) * 0.69314718055994530942f : -INFINITY;
      // Left-aligned ALiBi: the same weights, every score larger by
      // slope * (i + Skv - Sq) than the right-aligned one computed here.
      if constexpr (kAlibi)
        if (p.alibi == 3 && l > 0.f) lse = fmaf(slope, (float)(-dbase), lse);
      st_global_na_f32(p.lse + it.b * p.l_sb + it.h * p.l_sh + sr.q_off + i, lse);
    }
    if (stamper) FA_STAMP(sub ? 7 : 5, 7, k);
  }
  turn_release(sub ^ 1, w.abort_flag);
}

// Epilogue (one warpgroup, one row of each sub-tile per thread): for every
// item and sub-tile, once the softmax has handed over 1/l and the item's last
// PV is done, O_s / l -> bf16 rows in global memory (zeros for rows that see
// no key); 1/l is released as soon as it is read, O_s once it is read.
template <int D, bool kOcc, bool kClaim>
__device__ void epilogue_role(const FwdParams& p, Ctl<Cfg<D>::kStages>* ctl,
                              const float* inv_l_sm, uint32_t tmem, const WaitCtx& w) {
  using C = Cfg<D>;
  const int wq = (threadIdx.x >> 5) & 3;
  const int row = wq * 32 + (threadIdx.x & 31);
  const uint32_t lane_bits = (uint32_t)(wq * 32) << 16;
  uint32_t n_pv0 = 0u, n_pv1 = 0u;  // PVs of each sub-tile so far (registers, not an indexed array)
  // Rows start 32-byte aligned when O does (row strides are multiples of 128
  // bytes at D = 64 and 128); O itself need only be 16-byte aligned.
  const bool o_v8 = (reinterpret_cast<uintptr_t>(p.o) & 31u) == 0;
  for (int k = 0;; ++k) {
    int idx;
    if constexpr (kClaim) idx = idx_take_warp(ctl, k, w);
    else idx = item_index(k);
    if (idx >= p.n_items) break;
    const WorkItem it = p.items[idx];
    const SeqRec sr = p.seqs[it.b];
#pragma unroll 1
    for (int sub = 0; sub < 2; ++sub) {
      const int64_t r0 = (int64_t)it.qblk * kBlockM + sub * kTileM;
      const TileRange tr = sub_range<kOcc>(p, idx, it, sr, sub);
      const int i = (int)(r0 + row);
      const bool row_valid = i < sr.sq;
      if (threadIdx.x == 256) FA_STAMP(4, 3 * sub, k);
      if (!wait_warp(&ctl->epi_full[sub], k & 1u, w, kSiteEpi)) return;
      const float inv_l = inv_l_sm[sub * kTileM + row];
      mbar_arrive(&ctl->stat_free[sub]);
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) + it.b * p.o_sb +
                            it.h * p.o_sh + ((int64_t)sr.q_off + i) * p.o_st;
      if (tr.hi > tr.lo) {
        const uint32_t npv = (sub ? n_pv1 : n_pv0) + (uint32_t)(tr.hi - tr.lo);
        if (sub) n_pv1 = npv;
        else n_pv0 = npv;
        if (threadIdx.x == 256) FA_STAMP(4, 1 + 3 * sub, k);
        if (!wait_warp(&ctl->o_pv[sub], (npv - 1) & 1u, w, kSiteOPv)) return;
        tc_fence_after();
        if (threadIdx.x == 256) FA_STAMP(4, 2 + 3 * sub, k);
        const uint32_t tO = tmem + lane_bits + C::col_o(sub);
#pragma unroll 1
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t ov[32];
          tmem_ld32_wait(tO + ch * 32u, ov);
          uint4 pkd[4];
          uint32_t* pw = reinterpret_cast<uint32_t*>(pkd);
#pragma unroll
          for (int c = 0; c < 16; ++c)
            pw[c] = pack_bf16(__uint_as_float(ov[2 * c]) * inv_l,
                              __uint_as_float(ov[2 * c + 1]) * inv_l);
          if (row_valid) {
            uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
            if (o_v8) {
              st_global_na_v8(dst, pkd[0], pkd[1]);
              st_global_na_v8(dst + 2, pkd[2], pkd[3]);
            } else {
#pragma unroll
              for (int v = 0; v < 4; ++v) st_global_na_v4(dst + v, pkd[v]);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&ctl->o_free[sub]);
      } else if (row_valid) {
        uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll 1
        for (int v = 0; v < D / 8; ++v) st_global_na_v4(dst + v, make_uint4(0u, 0u, 0u, 0u));
      }
    }
  }
}

template <int D, bool kOcc, bool kDense, bool kClaim, bool kAlibi>
__global__ void __launch_bounds__(kThreads, 1) fa_fwd_sm100(const __grid_constant__ FwdParams p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + C::kQBytes;
  uint8_t* sP = sKV + C::kKVBytes;
  auto* ctl = reinterpret_cast<Ctl<C::kStages>*>(sP + C::kPBytes);
  static_assert(sizeof(Ctl<C::kStages>) <= C::kCtlBytes, "barrier area");
  float* inv_l_sm = reinterpret_cast<float*>(sP + C::kPBytes + C::kCtlBytes);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) FA_STAMP(6, 7, 0);
  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ctl->q_full[s], 1);
      mbar_init(&ctl->q_empty[s], 1);
    }
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&ctl->kv_full[s], 1);
      mbar_init(&ctl->kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ctl->s_full[s], 1);
      mbar_init(&ctl->s_free[s], 128);
      mbar_init(&ctl->p_full[s], 128);
      mbar_init(&ctl->o_pv[s], 1);
      mbar_init(&ctl->epi_full[s], 128);
      mbar_init(&ctl->stat_free[s], 128);
      mbar_init(&ctl->o_free[s], 128);
    }
    mbar_init(&ctl->drain[0], 1);
    mbar_init(&ctl->drain[1], 1);
    if constexpr (kClaim) {
      for (int r = 0; r < kIdxSlots; ++r) {
        mbar_init(&ctl->idx_full[r], 1);
        mbar_init(&ctl->idx_empty[r], kIdxReaders);
      }
    }
    ctl->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kWarpMma) {
    asm volatile(
        "tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
            smem_u32(&ctl->tmem_base)),
        "r"(C::kTmemCols)
        : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const WaitCtx w{&ctl->abort_flag, p.err_word, p.timeout_ns};

  if (warp < 8) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    softmax_role<D, kOcc, kDense, kClaim, kAlibi>(p, ctl, inv_l_sm, tmem, sP, warp >> 2, w);
  } else if (warp < 12) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsEpi));
    epilogue_role<D, kOcc, kClaim>(p, ctl, inv_l_sm, tmem, w);
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
    if (warp == kWarpMma && lane == 0) qk_role<D, kOcc, kClaim, kAlibi>(p, ctl, tmem, sQ, sKV, w);
    if (warp == kWarpPv && lane == 0) pv_role<D, kOcc, kClaim, kAlibi>(p, ctl, tmem, sP, sKV, w);
    if (warp == kWarpLoad && lane == 0) load_role<D, kOcc, kClaim, kAlibi>(p, ctl, sQ, sKV, w);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpMma) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(C::kTmemCols)
                 : "memory");
  }
  if constexpr (kClaim) {
    // Every claim of this CTA has returned (its TMA thread has left its
    // list): the last CTA out leaves the counters at 0 for the next launch.
    if (threadIdx.x == 0) {
      __threadfence();
      if (atomicAdd(p.claim_done, 1u) == gridDim.x - 1) {
        atomicExch(p.claim, 0u);
        atomicExch(p.claim_done, 0u);
      }
    }
  }
}

}  // namespace dev

// ----------------------------------------------------------------- host

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

bool encode_operand_map(CUtensorMap* tm, const void* base, int64_t D, int64_t S, int64_t N,
                        int64_t B, int64_t st_s, int64_t st_n, int64_t st_b) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)(S > 0 ? S : 1), (cuuint64_t)N,
                              (cuuint64_t)(B > 0 ? B : 1)};
  const cuuint64_t strides[3] = {(cuuint64_t)st_s * 2u, (cuuint64_t)st_n * 2u,
                                 (cuuint64_t)st_b * 2u};
  const cuuint32_t box[4] = {64u, 128u, 1u, 1u};
  const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, bool kOcc, bool kDense, bool kClaim = false, bool kAlibi = false>
static cudaError_t launch_d(const FwdParams& p, int grid, cudaStream_t stream, const char** why) {
  using C = dev::Cfg<D>;
  auto kern = dev::fa_fwd_sm100<D, kOcc, kDense, kClaim, kAlibi>;
  static bool configured = false;
  static bool regs_ok = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)C::kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaFuncAttributes attr;
    e = cudaFuncGetAttributes(&attr, kern);
    if (e != cudaSuccess) return e;
    // setmaxnreg redistributes the registers the CTA was launched with; a
    // split larger than that allocation would never be granted.
    regs_ok = attr.numRegs * dev::kThreads >= dev::kRegsTotal;
    configured = true;
  }
  if (!regs_ok) {
    if (why) *why = "kernel compiled with fewer registers than its warpgroup split needs";
    return cudaErrorInvalidConfiguration;
  }
  kern<<<grid, dev::kThreads, C::kSmemBytes, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_fwd(int D, const FwdParams& p, int grid, cudaStream_t stream,
                       const char** why) {
  // Six instances per head dim: ranges beside the items with the
  // dense-mask extras, without them (fixed snake or claimed work, each also
  // with the ALiBi bias), and ranges from the closed form (no item_tr). Only
  // the claiming instances read p.claim.
  const bool occ = p.item_tr != nullptr;
  const bool dense = occ && p.mask != nullptr && p.m_si > 0;
  const bool claim = occ && !dense && p.claim != nullptr;
  const bool alibi = p.slopes != nullptr;
  if (alibi && (!occ || dense)) {
    if (why) *why = "an ALiBi bias needs a closed-form call with per-item ranges";
    return cudaErrorInvalidValue;
  }
  if (D == 128) {
    if (alibi)
      return claim ? launch_d<128, true, false, true, true>(p, grid, stream, why)
                   : launch_d<128, true, false, false, true>(p, grid, stream, why);
    return dense   ? launch_d<128, true, true>(p, grid, stream, why)
           : claim ? launch_d<128, true, false, true>(p, grid, stream, why)
           : occ   ? launch_d<128, true, false>(p, grid, stream, why)
                   : launch_d<128, false, false>(p, grid, stream, why);
  }
  if (D == 64) {
    if (alibi)
      return claim ? launch_d<64, true, false, true, true>(p, grid, stream, why)
                   : launch_d<64, true, false, false, true>(p, grid, stream, why);
    return dense   ? launch_d<64, true, true>(p, grid, stream, why)
           : claim ? launch_d<64, true, false, true>(p, grid, stream, why)
           : occ   ? launch_d<64, true, false>(p, grid, stream, why)
                   : launch_d<64, false, false>(p, grid, stream, why);
  }
  if (why) *why = "unsupported head dim";
  return cudaErrorInvalidValue;
}

}  // namespace fa

#ifdef FA_TRACE
// Trace builds only: the traced CTA, and clearing and reading the stamps.
extern "C" int fa_trace_cta(void) { return FA_TRACE; }
extern "C" int fa_trace_clear(void) {
  static unsigned long long zero[8 * 8 * fa::dev::kTraceN];
  cudaError_t e = cudaMemcpyToSymbol(fa::dev::g_fa_trace, zero, sizeof(zero));
  if (e == cudaSuccess)
    e = cudaMemcpyToSymbol(fa::dev::g_fa_wtrace, zero, sizeof(fa::dev::g_fa_wtrace));
  return (int)e;
}
extern "C" int fa_trace_read(void* tiles, void* warps) {
  cudaError_t e = cudaMemcpyFromSymbol(tiles, fa::dev::g_fa_trace, sizeof(fa::dev::g_fa_trace));
  if (e == cudaSuccess)
    e = cudaMemcpyFromSymbol(warps, fa::dev::g_fa_wtrace, sizeof(fa::dev::g_fa_wtrace));
  return (int)e;
}
#endif
