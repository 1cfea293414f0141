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
//   warp 12     tcgen05.mma issuer (one thread; owns TMEM)
//   warp 13     TMA producer (one thread)
//   other warps idle (they give their registers to the softmax warps)
// Tensor memory (512 columns): S0 | S1 | O0 | O1. S_s holds the fp32 scores
// of sub-tile s; the softmax overwrites its first 64 columns with P (bf16
// pairs), which feeds the P.V MMA directly from TMEM. O_s accumulates fp32.
// MMA issue order per key tile t:  PV0(t), QK0(t+1), PV1(t), QK1(t+1), so
// each softmax warpgroup has the time of two MMA groups to turn S into P,
// and every S_s(t+1) commit also proves PV_s(t) complete (commits track all
// earlier MMAs), which is what lets the softmax rescale O_s in place.
// Every mbarrier wait is bounded (globaltimer); on expiry the CTA records
// the site in the error word, drains its in-flight copies and MMAs, frees
// its tensor memory and exits.
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

constexpr int kThreads = 512;
constexpr int kWarpMma = 12;
constexpr int kWarpLoad = 13;
// Register split (setmaxnreg) over the 512 x 128 registers of the launch:
// softmax warpgroups 0-1 take 208, the idle warpgroup 2 keeps 24, the
// warpgroup of the MMA and TMA warps keeps 72.
constexpr int kRegsSoftmax = 208;
constexpr int kRegsIdle = 24;
constexpr int kRegsControl = 72;
constexpr int kRegsTotal = 2 * 128 * kRegsSoftmax + 128 * kRegsIdle + 128 * kRegsControl;
static_assert(kRegsTotal == kThreads * 128, "register split must equal the launch allocation");
constexpr float kRescaleLog2 = 8.0f;  // rescale O only when the max grows by > 2^8
constexpr int kPChunks = 4;           // P is exponentiated and stored 32 keys at a time

// Where a wait gave up (error word bits 8..15).
enum WaitSite : uint32_t {
  kSiteQEmpty = 1, kSiteKvEmpty = 2, kSiteQFull = 3, kSiteKvFull = 4, kSitePFull = 5,
  kSiteSFull = 6, kSiteODone = 7, kSiteDrain = 8,
};

template <int D>
struct Cfg {
  static constexpr int kChunks = D / 64;                 // 64-column (128-byte) chunks per row
  static constexpr uint32_t kChunkBytes = 128u * 128u;   // 128 rows x 128 bytes
  static constexpr uint32_t kTileBytes = 128u * D * 2u;  // 128 rows of Q, K or V
  static constexpr int kStages = (D == 128) ? 4 : 8;     // K/V ring depth
  static constexpr uint32_t kQBytes = 2u * kTileBytes;
  static constexpr uint32_t kKVBytes = kStages * kTileBytes;
  static constexpr uint32_t kCtlBytes = 512u;
  static constexpr uint32_t kSmemBytes = 1024u + kQBytes + kKVBytes + kCtlBytes;
  static constexpr uint32_t kTmemCols = 512u;
  // TMEM columns of S_s / P_s and of O_s
  __host__ __device__ static constexpr uint32_t col_s(int s) { return s ? 128u : 0u; }
  __host__ __device__ static constexpr uint32_t col_o(int s) { return s ? 256u + D : 256u; }
  static_assert(kSmemBytes <= 227u * 1024u, "shared memory budget");
};

template <int NS>
struct Ctl {
  uint64_t q_full, q_empty;
  uint64_t kv_full[NS], kv_empty[NS];
  uint64_t s_full[2], p_full[2], o_done[2];
  uint64_t drain[1];
  uint32_t tmem_base;
  volatile int abort_flag;
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

// x <- 2^(x * scale_log2 - ref) in place; returns the row sum (eight
// independent partial sums). kPoly: some columns use ex2_poly_x2.
template <bool kPoly>
__device__ __forceinline__ float exp_rows(float (&x)[128], float scale_log2, float ref) {
  const uint64_t m2 = pack_f32x2(scale_log2, scale_log2);
  const uint64_t c2 = pack_f32x2(-ref, -ref);
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int c = 0; c < 128; c += 2) {
    float a = x[c], b = x[c + 1];
    fma_x2(a, b, m2, c2);
    if (kPoly && (c & 7) < kPolyPer8) {
      ex2_poly_x2(a, b);
    } else {
      a = ex2(a);
      b = ex2(b);
    }
    x[c] = a;
    x[c + 1] = b;
    const int k = (c >> 1) & 3;
    add_x2(acc[2 * k], acc[2 * k + 1], a, b);
  }
  add_x2(acc[0], acc[1], acc[2], acc[3]);
  add_x2(acc[4], acc[5], acc[6], acc[7]);
  add_x2(acc[0], acc[1], acc[4], acc[5]);
  return acc[0] + acc[1];
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

// Whole-warp wait: every lane waits, the warp proceeds only if all did.
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity, const WaitCtx& w,
                                          uint32_t site) {
  const bool ok = wait_bounded(bar, parity, w, site);
  return __all_sync(0xffffffffu, ok);
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

struct ItemPlan {
  TileRange tr[2];
  int lo, hi;      // union of the two sub-tiles' tile ranges
  int nsub;        // sub-tiles with at least one stored row
};

__device__ __forceinline__ ItemPlan plan_item(const SeqRec& s, int qblk) {
  ItemPlan ip;
  ip.lo = 0x7fffffff;
  ip.hi = 0;
  ip.nsub = 0;
#pragma unroll
  for (int st = 0; st < 2; ++st) {
    const int64_t r0 = (int64_t)qblk * kBlockM + st * kTileM;
    ip.tr[st] = tile_range(s, r0);
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

template <int D>
__device__ void load_role(const FwdParams& p, Ctl<Cfg<D>::kStages>* ctl, uint8_t* sQ,
                          uint8_t* sKV, const WaitCtx& w) {
  using C = Cfg<D>;
  constexpr int NS = C::kStages;
  uint32_t ring = 0, q_loads = 0;
  bool ok = true;
  for (int k = 0; ok; ++k) {
    const int idx = item_index(k);
    if (idx >= p.n_items) break;
    const WorkItem it = p.items[idx];
    const SeqRec sr = p.seqs[it.b];
    const ItemPlan ip = plan_item(sr, it.qblk);
    if (ip.hi <= ip.lo) continue;
    const int bc = p.tnd ? 0 : it.b;
    if (q_loads > 0 && !wait_bounded(&ctl->q_empty, (q_loads - 1) & 1u, w, kSiteQEmpty)) {
      ok = false;
      break;
    }
    const bool drop = (p.debug_flags & kDebugDropFirstQ) && blockIdx.x == 0 && q_loads == 0;
    if (!drop) {
      mbar_expect_tx(&ctl->q_full, ip.nsub * C::kTileBytes);
      for (int st = 0; st < ip.nsub; ++st) {
        const int row = sr.q_off + it.qblk * kBlockM + st * kTileM;
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_4d(sQ + st * C::kTileBytes + c * C::kChunkBytes, &p.tm_q, &ctl->q_full, c * 64,
                      row, it.h, bc);
      }
    }
    ++q_loads;
    for (int t = ip.lo; t < ip.hi && ok; ++t) {
#pragma unroll 1
      for (int kv = 0; kv < 2; ++kv) {
        const uint32_t st = ring % NS;
        if (ring >= (uint32_t)NS &&
            !wait_bounded(&ctl->kv_empty[st], ((ring / NS) - 1) & 1u, w, kSiteKvEmpty)) {
          ok = false;
          break;
        }
        mbar_expect_tx(&ctl->kv_full[st], C::kTileBytes);
        const CUtensorMap* tm = kv == 0 ? &p.tm_k : &p.tm_v;
        const int row = sr.kv_off + t * kTileN;
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_4d(sKV + st * C::kTileBytes + c * C::kChunkBytes, tm, &ctl->kv_full[st],
                      c * 64, row, it.h, bc);
        ++ring;
      }
    }
  }
  if (!ok) {
    // Abort: let every copy this thread started land before the CTA exits.
    const uint32_t first = ring > (uint32_t)NS ? ring - NS : 0u;
    for (uint32_t r = first; r < ring; ++r)
      wait_bounded(&ctl->kv_full[r % NS], (r / NS) & 1u, w, kSiteDrain, false);
    if (q_loads > 0) wait_bounded(&ctl->q_full, (q_loads - 1) & 1u, w, kSiteDrain, false);
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
__device__ __forceinline__ void issue_pv(uint32_t tmem, const uint8_t* sKV, int sub, uint32_t vst,
                                         bool accumulate) {
  using C = Cfg<D>;
  constexpr uint32_t idesc = idesc_bf16(128, D, true);
  // V is MN-major (D contiguous): step k moves 16 key rows = 2048 bytes.
  const uint64_t b0 = sdesc(smem_u32(sKV) + vst * C::kTileBytes, C::kChunkBytes, 1024u);
  const uint32_t a = tmem + C::col_s(sub);  // P: 128 bf16 = 64 columns
  const uint32_t d = tmem + C::col_o(sub);
#pragma unroll
  for (int k = 0; k < kTileN / 16; ++k)
    mma_ts(d, a + k * 8u, b0 + (uint64_t)(k * (2048u >> 4)), idesc,
           (accumulate || k > 0) ? 1u : 0u);
}

// MMA issue (one thread). Per key tile t, in this order:
//   O_0 += P_0(t) V(t); S_0(t+1) = Q_0 K(t+1)^T; O_1 += P_1(t) V(t);
//   S_1(t+1) = Q_1 K(t+1)^T
// so each softmax warpgroup has two MMA groups' time to turn S into P. Both
// ring waits come before the first group and the commits follow the QK
// groups, so consecutive groups go out with only the P wait between them:
// the tensor pipe queues few instructions and any gap in issue idles it.
template <int D>
__device__ void mma_role(const FwdParams& p, Ctl<Cfg<D>::kStages>* ctl, uint32_t tmem,
                         const uint8_t* sQ, const uint8_t* sKV, const WaitCtx& w) {
  using C = Cfg<D>;
  constexpr int NS = C::kStages;
  uint32_t ring = 0, q_loads = 0;
  uint32_t p_count[2] = {0u, 0u};
  bool ok = true;
  for (int k = 0; ok; ++k) {
    const int idx = item_index(k);
    if (idx >= p.n_items) break;
    const WorkItem it = p.items[idx];
    const SeqRec sr = p.seqs[it.b];
    const ItemPlan ip = plan_item(sr, it.qblk);
    if (ip.hi <= ip.lo) continue;
    if (!wait_bounded(&ctl->q_full, q_loads & 1u, w, kSiteQFull)) {
      ok = false;
      break;
    }
    ++q_loads;
    uint32_t kst = ring % NS;
    if (!wait_bounded(&ctl->kv_full[kst], (ring / NS) & 1u, w, kSiteKvFull)) {
      ok = false;
      break;
    }
    ++ring;
#pragma unroll
    for (int s = 0; s < 2; ++s)
      if (active(ip.tr[s], ip.lo)) {
        issue_qk<D>(tmem, sQ, sKV, s, kst);
        mma_commit(&ctl->s_full[s]);
      }
    mma_commit(&ctl->kv_empty[kst]);
    if (ip.lo + 1 == ip.hi) mma_commit(&ctl->q_empty);
    bool first[2] = {true, true};
    for (int t = ip.lo; t < ip.hi && ok; ++t) {
      const uint32_t vst = ring % NS;
      if (!wait_bounded(&ctl->kv_full[vst], (ring / NS) & 1u, w, kSiteKvFull)) {
        ok = false;
        break;
      }
      ++ring;
      const bool nxt = t + 1 < ip.hi;
      if (nxt) {
        kst = ring % NS;
        if (!wait_bounded(&ctl->kv_full[kst], (ring / NS) & 1u, w, kSiteKvFull)) {
          ok = false;
          break;
        }
        ++ring;
      }
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        if (active(ip.tr[s], t)) {
          if (!wait_bounded(&ctl->p_full[s], p_count[s] & 1u, w, kSitePFull)) {
            ok = false;
            break;
          }
          ++p_count[s];
          tc_fence_after();
          issue_pv<D>(tmem, sKV, s, vst, !first[s]);
          first[s] = false;
          if (t == ip.tr[s].hi - 1) mma_commit(&ctl->o_done[s]);
        }
        if (nxt && active(ip.tr[s], t + 1)) {
          issue_qk<D>(tmem, sQ, sKV, s, kst);
          mma_commit(&ctl->s_full[s]);
        }
      }
      if (!ok) break;
      mma_commit(&ctl->kv_empty[vst]);
      if (nxt) {
        mma_commit(&ctl->kv_empty[kst]);
        if (t + 2 == ip.hi) mma_commit(&ctl->q_empty);
      }
    }
  }
  if (!ok) {
    // Abort: wait until every MMA issued so far has finished with TMEM/SMEM.
    mma_commit(&ctl->drain[0]);
    wait_bounded(&ctl->drain[0], 0u, w, kSiteDrain, false);
  }
}

// Scores of this thread's row (128 keys of S_s) with the element mask of a
// boundary tile applied (-inf where the key is not visible). The visible
// columns [c_lo, c_hi] are tested as one unsigned range compare per element;
// dense-mask bits (modes 0/1) are applied only when present.
__device__ __forceinline__ void load_scores(uint32_t tS, float (&x)[128], bool partial, int c_lo,
                                            int c_hi, bool dense, const uint32_t (&mbits)[4]) {
  uint32_t sv[128];
  tmem_ld128_wait(tS, sv);
#pragma unroll
  for (int c = 0; c < 128; ++c) x[c] = __uint_as_float(sv[c]);
  if (partial) {
    int lo = c_lo, width = c_hi - c_lo;
    if (width < 0) lo = 1 << 20, width = 0;  // nothing visible
#pragma unroll
    for (int c = 0; c < 128; ++c)
      x[c] = ((unsigned)(c - lo) <= (unsigned)width) ? x[c] : -INFINITY;
    if (dense) {
#pragma unroll
      for (int c = 0; c < 128; ++c)
        x[c] = ((mbits[c >> 5] >> (c & 31)) & 1u) ? -INFINITY : x[c];
    }
  }
}

// Exponentiate keys [32 c, 32 c + 32) of the row against `ref`, add them to
// the eight partial sums and pack P into 16 bf16 pairs.
template <bool kPoly>
__device__ __forceinline__ void exp_chunk(float (&x)[128], int chunk, uint64_t m2, uint64_t c2,
                                          float (&acc)[8], uint32_t (&pk)[16]) {
#pragma unroll
  for (int j = 0; j < 32; j += 2) {
    const int c = chunk * 32 + j;
    float a = x[c], b = x[c + 1];
    fma_x2(a, b, m2, c2);
    if (kPoly && (c & 7) < kPolyPer8) {
      ex2_poly_x2(a, b);
    } else {
      a = ex2(a);
      b = ex2(b);
    }
    const int k = (j >> 1) & 3;
    add_x2(acc[2 * k], acc[2 * k + 1], a, b);
    pk[j >> 1] = pack_bf16(a, b);
  }
}

// Exponentiate the row chunk by chunk, storing each chunk of P as soon as it
// is packed; one arrival on p_full once every store has landed.
template <bool kPoly>
__device__ __forceinline__ float exp_store_p(float (&x)[128], float scale_log2, float ref,
                                             uint32_t tS, uint64_t* p_full) {
  const uint64_t m2 = pack_f32x2(scale_log2, scale_log2);
  const uint64_t c2 = pack_f32x2(-ref, -ref);
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int c = 0; c < kPChunks; ++c) {
    uint32_t pk[16];
    exp_chunk<kPoly>(x, c, m2, c2, acc, pk);
    tmem_st16(tS + 16u * c, pk);
  }
  tmem_st_wait();
  tc_fence_before();
  mbar_arrive(p_full);
  add_x2(acc[0], acc[1], acc[2], acc[3]);
  add_x2(acc[4], acc[5], acc[6], acc[7]);
  add_x2(acc[0], acc[1], acc[4], acc[5]);
  return acc[0] + acc[1];
}

template <int D>
__device__ void softmax_role(const FwdParams& p, Ctl<Cfg<D>::kStages>* ctl, uint32_t tmem,
                             int sub, const WaitCtx& w) {
  using C = Cfg<D>;
  const int wq = (threadIdx.x >> 5) & 3;           // TMEM lane quarter of this warp
  const int row = wq * 32 + (threadIdx.x & 31);    // row of the sub-tile = TMEM lane
  const uint32_t lane_bits = (uint32_t)(wq * 32) << 16;
  const uint32_t tS = tmem + lane_bits + C::col_s(sub);
  const uint32_t tO = tmem + lane_bits + C::col_o(sub);
  const float scale_log2 = p.scale_log2;
  uint32_t s_count = 0, o_count = 0;
  bool ok = true;
  for (int k = 0; ok; ++k) {
    const int idx = item_index(k);
    if (idx >= p.n_items) break;
    const WorkItem it = p.items[idx];
    const SeqRec sr = p.seqs[it.b];
    const int64_t r0 = (int64_t)it.qblk * kBlockM + sub * kTileM;
    const TileRange tr = tile_range(sr, r0);
    const int i = (int)(r0 + row);  // query row inside the sequence
    const bool row_valid = i < sr.sq;
    // Visible keys of this row: [jlo, jhi] (empty when jlo > jhi).
    int jlo = 1, jhi = 0;
    if (row_valid) {
      jlo = (int)imax64(0, row_lo(sr, i));
      jhi = (int)imin64((int64_t)sr.skv - 1, row_hi(sr, i));
    }
    const uint8_t* mrow = nullptr;
    if ((sr.flags & kSeqDenseMask) && row_valid)
      mrow = p.mask + it.b * p.m_sb + it.h * p.m_sh + (int64_t)i * p.m_si;
    float m_used = -INFINITY;  // reference max (log2 units, scaled)
    float l = 0.f;             // running sum relative to m_used
    for (int t = tr.lo; t < tr.hi; ++t) {
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
#pragma unroll
        for (int wd = 0; wd < 4; ++wd) {
          uint32_t bits = 0u;
#pragma unroll 1
          for (int c = wd * 32; c < wd * 32 + 32; ++c)
            if (c >= c_lo && c <= c_hi && mt[c] != 0) bits |= 1u << (c & 31);
          mbits[wd] = bits;
        }
      }
      tc_fence_after();
      float x[128];
      load_scores(tS, x, partial, c_lo, c_hi, mrow != nullptr, mbits);
      const float m_new = row_max128(x) * scale_log2;
      const bool resc = m_new > m_used + kRescaleLog2;
      float alpha = 1.f;
      if (resc) {
        alpha = (m_used == -INFINITY) ? 0.f : ex2(m_used - m_new);
        l *= alpha;
        m_used = m_new;
      }
      // O_s already holds PV(t-1) (the S_s(t) commit tracked it); rescale it
      // in place when this row's reference max moved, before the first P
      // chunk lets PV(t) accumulate. Not on the item's first tile: its PV
      // overwrites O_s.
      if (t > tr.lo && __any_sync(0xffffffffu, resc)) {
#pragma unroll 1
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t ov[32];
          tmem_ld32_wait(tO + ch * 32u, ov);
#pragma unroll
          for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
          tmem_st32(tO + ch * 32u, ov);
        }
      }
      const float ref = (m_used == -INFINITY) ? 0.f : m_used;
      l += partial ? exp_store_p<false>(x, scale_log2, ref, tS, &ctl->p_full[sub])
                   : exp_store_p<true>(x, scale_log2, ref, tS, &ctl->p_full[sub]);
    }
    if (!ok) break;
    // Epilogue: O / l -> bf16, lse = ln(sum exp(scale q.k)).
    __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) + it.b * p.o_sb +
                          it.h * p.o_sh + ((int64_t)sr.q_off + i) * p.o_st;
    float lse = -INFINITY;
    if (tr.hi > tr.lo) {
      if (!wait_warp(&ctl->o_done[sub], o_count & 1u, w, kSiteODone)) {
        ok = false;
        break;
      }
      ++o_count;
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
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
#pragma unroll
          for (int v = 0; v < 4; ++v) dst[v] = pkd[v];
        }
      }
      if (l > 0.f) lse = (m_used + log2f(l)) * 0.69314718055994530942f;
    } else if (row_valid) {
      uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll 1
      for (int v = 0; v < D / 8; ++v) dst[v] = make_uint4(0u, 0u, 0u, 0u);
    }
    if (row_valid) p.lse[it.b * p.l_sb + it.h * p.l_sh + sr.q_off + i] = lse;
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) fa_fwd_sm100(const __grid_constant__ FwdParams p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + C::kQBytes;
  auto* ctl = reinterpret_cast<Ctl<C::kStages>*>(sKV + C::kKVBytes);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&ctl->q_full, 1);
    mbar_init(&ctl->q_empty, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&ctl->kv_full[s], 1);
      mbar_init(&ctl->kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ctl->s_full[s], 1);
      mbar_init(&ctl->p_full[s], 128);
      mbar_init(&ctl->o_done[s], 1);
    }
    mbar_init(&ctl->drain[0], 1);
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
    softmax_role<D>(p, ctl, tmem, warp >> 2, w);
  } else if (warp < 12) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsIdle));
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
    if (warp == kWarpMma && lane == 0) mma_role<D>(p, ctl, tmem, sQ, sKV, w);
    if (warp == kWarpLoad && lane == 0) load_role<D>(p, ctl, sQ, sKV, w);
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

template <int D>
static cudaError_t launch_d(const FwdParams& p, int grid, cudaStream_t stream, const char** why) {
  using C = dev::Cfg<D>;
  auto kern = dev::fa_fwd_sm100<D>;
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
  if (D == 128) return launch_d<128>(p, grid, stream, why);
  if (D == 64) return launch_d<64>(p, grid, stream, why);
  if (why) *why = "unsupported head dim";
  return cudaErrorInvalidValue;
}

}  // namespace fa
