// Cycles per 128-key row of the softmax's exponential loop for several
// instruction mixes: one row per thread, W warps per SM sub-partition (4 W
// warps per CTA, one CTA per SM). A measurement probe, not part of the
// library; built and run by `python -m masked_attention_fa_b200.trace
// --exp-probe`. The loop mirrors the attention kernel's: per key pair one
// f32x2 FMA (scale, offset), two ex2.approx, one f32x2 add into the row sum
// and one bf16x2 pack; the variants swap or drop parts of it.
#include <cstdio>
#include <cstdint>
#include <cuda_runtime.h>
__device__ __forceinline__ uint64_t clk() { uint64_t t; asm volatile("mov.u64 %0, %%clock64;" : "=l"(t)); return t; }
__device__ __forceinline__ float ex2(float x) { float y; asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x)); return y; }
__device__ __forceinline__ uint32_t cvt2(float lo, float hi) { uint32_t r; asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo)); return r; }
__device__ __forceinline__ uint32_t pack_int(float lo, float hi) {
  // round half up to bf16 with integer adds, then take the two high halves
  uint32_t a = __float_as_uint(lo) + 0x8000u, b = __float_as_uint(hi) + 0x8000u, r;
  asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ void fma_x2(float& a, float& b, uint64_t m2, uint64_t c2) {
  asm("{\n\t.reg .b64 r;\n\tmov.b64 r, {%0, %1};\n\tfma.rn.f32x2 r, r, %2, %3;\n\tmov.b64 {%0, %1}, r;\n\t}" : "+f"(a), "+f"(b) : "l"(m2), "l"(c2));
}
__device__ __forceinline__ void add_x2(float& a, float& b, float x, float y) {
  asm("{\n\t.reg .b64 r, s;\n\tmov.b64 r, {%0, %1};\n\tmov.b64 s, {%2, %3};\n\tadd.rn.f32x2 r, r, s;\n\tmov.b64 {%0, %1}, r;\n\t}" : "+f"(a), "+f"(b) : "f"(x), "f"(y));
}
__device__ __forceinline__ uint64_t pk2(float a, float b) { uint64_t r; asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b)); return r; }
__device__ __forceinline__ void ex2_poly_x2(float& a, float& b) {
  constexpr float kShift = 12582912.0f;
  a = fmaxf(a, -126.0f);
  b = fmaxf(b, -126.0f);
  float ta = a, tb = b;
  add_x2(ta, tb, kShift, kShift);
  float na = ta, nb = tb;
  add_x2(na, nb, -kShift, -kShift);
  float fa = -na, fb = -nb;
  add_x2(fa, fb, a, b);
  float pa = 0.05517167f, pb = 0.05517167f;
  fma_x2(pa, pb, pk2(fa, fb), pk2(0.24261113f, 0.24261113f));
  fma_x2(pa, pb, pk2(fa, fb), pk2(0.69326097f, 0.69326097f));
  fma_x2(pa, pb, pk2(fa, fb), pk2(0.99992806f, 0.99992806f));
  a = __int_as_float(__float_as_int(pa) + (__float_as_int(ta) << 23));
  b = __int_as_float(__float_as_int(pb) + (__float_as_int(tb) << 23));
}
__device__ __forceinline__ float ex2_lean(float x) {
  x = fmaxf(x, -126.0f);
  const float t = x + 12582912.0f;           // n in the low mantissa bits
  const float f = x - (t - 12582912.0f);     // |f| <= 1/2
  const float p = fmaf(fmaf(fmaf(0.05517167f, f, 0.24261113f), f, 0.69326097f), f, 0.99992806f);
  return __int_as_float(__float_as_int(t) * (1 << 23) + __float_as_int(p));
}
__device__ __forceinline__ uint32_t ex2h2(uint32_t x) { uint32_t y; asm("ex2.approx.f16x2 %0, %1;" : "=r"(y) : "r"(x)); return y; }
__device__ __forceinline__ uint32_t ex2bf2(uint32_t x) { uint32_t y; asm("ex2.approx.ftz.bf16x2 %0, %1;" : "=r"(y) : "r"(x)); return y; }

template <int MODE>
__global__ void __launch_bounds__(256, 1) kern(const float* in, uint32_t* out, long long* cyc, int reps) {
  float x[128];
  for (int c = 0; c < 128; ++c) x[c] = in[(threadIdx.x * 131 + c) & 4095];
  uint32_t pk[64];
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  const uint64_t m2 = pk2(0.0883883f, 0.0883883f), c2 = pk2(-1.5f, -1.5f);
  __syncthreads();
  uint64_t t0 = clk();
  for (int r = 0; r < reps; ++r) {
#pragma unroll
    for (int c = 0; c < 128; c += 2) {
      float a = x[c], b = x[c + 1];
      if (MODE == 0) {          // ex2 only
        a = ex2(a); b = ex2(b); acc[c & 7] += a; acc[(c + 1) & 7] += b;
      } else if (MODE == 1) {   // cvt only
        pk[c >> 1] ^= cvt2(a, b);
      } else if (MODE == 2) {   // kernel loop: fma2, ex2 x2, add2, cvt
        fma_x2(a, b, m2, c2);
        a = ex2(a); b = ex2(b);
        const int k = (c >> 1) & 3;
        add_x2(acc[2 * k], acc[2 * k + 1], a, b);
        pk[c >> 1] ^= cvt2(a, b);
      } else if (MODE == 3) {   // kernel loop with the integer pack
        fma_x2(a, b, m2, c2);
        a = ex2(a); b = ex2(b);
        const int k = (c >> 1) & 3;
        add_x2(acc[2 * k], acc[2 * k + 1], a, b);
        pk[c >> 1] ^= pack_int(a, b);
      } else if (MODE == 4) {   // fma2 + pack to f16x2 + ex2.f16x2 + unpack + add (exp in half)
        fma_x2(a, b, m2, c2);
        uint32_t h; asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(h) : "f"(b), "f"(a));
        uint32_t e = ex2h2(h);
        pk[c >> 1] ^= e;
      } else if (MODE == 5) {   // bf16x2 ex2
        fma_x2(a, b, m2, c2);
        uint32_t h = cvt2(a, b);
        pk[c >> 1] ^= ex2bf2(h);
      } else if (MODE >= 40) {  // MODE = 40 + polyper8, lean scalar poly, cvt pack
        constexpr int kp = MODE - 40;
        fma_x2(a, b, m2, c2);
        if ((c & 7) < kp) { a = ex2_lean(a); b = ex2_lean(b); }
        else { a = ex2(a); b = ex2(b); }
        const int k = (c >> 1) & 3;
        add_x2(acc[2 * k], acc[2 * k + 1], a, b);
        pk[c >> 1] ^= cvt2(a, b);
      } else if (MODE >= 10) {  // MODE = 10 + 8*intpack + polyper8
        constexpr int kp = (MODE - 10) % 8, ip = (MODE - 10) / 8;
        fma_x2(a, b, m2, c2);
        if ((c & 7) < kp) ex2_poly_x2(a, b);
        else { a = ex2(a); b = ex2(b); }
        const int k = (c >> 1) & 3;
        add_x2(acc[2 * k], acc[2 * k + 1], a, b);
        pk[c >> 1] ^= ip ? pack_int(a, b) : cvt2(a, b);
      } else if (MODE == 6) {   // kernel loop without the pack
        fma_x2(a, b, m2, c2);
        a = ex2(a); b = ex2(b);
        const int k = (c >> 1) & 3;
        add_x2(acc[2 * k], acc[2 * k + 1], a, b);
        pk[c >> 1] ^= __float_as_uint(a) ^ __float_as_uint(b);
      }
    }
#pragma unroll
    for (int c = 0; c < 128; ++c) x[c] = x[c] * 0.999f + 0.0001f;
  }
  uint64_t t1 = clk();
  uint32_t s = 0;
  for (int c = 0; c < 64; ++c) s ^= pk[c];
  for (int c = 0; c < 8; ++c) s ^= __float_as_uint(acc[c]);
  out[blockIdx.x * blockDim.x + threadIdx.x] = s;
  if ((threadIdx.x & 31) == 0) cyc[blockIdx.x * 16 + (threadIdx.x >> 5)] = (long long)(t1 - t0);
}

template <int MODE> void run(const char* name, int warps_per_smsp, const float* din, uint32_t* dout, long long* dcyc) {
  const int threads = 128 * warps_per_smsp, reps = 200;
  kern<MODE><<<148, threads>>>(din, dout, dcyc, reps);
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) { printf("%s error %s\n", name, cudaGetErrorString(e)); return; }
  long long h[148 * 16];
  cudaMemcpy(h, dcyc, sizeof(h), cudaMemcpyDeviceToHost);
  double s = 0; int n = 0;
  for (int b = 0; b < 148; ++b) for (int w = 0; w < threads / 32; ++w) { s += h[b * 16 + w]; ++n; }
  printf("| %-44s | %d | %.0f |\n", name, warps_per_smsp, s / n / reps);
}

int main() {
  float* din; uint32_t* dout; long long* dcyc;
  cudaMalloc(&din, 4096 * 4); cudaMalloc(&dout, 148 * 512 * 4); cudaMalloc(&dcyc, 148 * 16 * 8);
  float h[4096]; for (int i = 0; i < 4096; ++i) h[i] = -(float)(i % 97) * 0.13f;
  cudaMemcpy(din, h, sizeof(h), cudaMemcpyHostToDevice);
  cudaMemset(dcyc, 0, 148 * 16 * 8);
  printf("| loop | warps per sub-partition | cycles per row per warp |\n|---|---|---|\n");
  for (int w = 1; w <= 2; ++w) {
    run<0>("ex2 only (with the row sum)", w, din, dout, dcyc);
    run<1>("bf16x2 pack only", w, din, dout, dcyc);
    run<2>("kernel loop (bf16x2 pack)", w, din, dout, dcyc);
    run<3>("kernel loop, integer round + byte-permute pack", w, din, dout, dcyc);
    run<6>("kernel loop without the pack", w, din, dout, dcyc);
    run<4>("ex2.approx.f16x2", w, din, dout, dcyc);
    run<5>("ex2.approx.ftz.bf16x2", w, din, dout, dcyc);
    run<12>("FMA-pipe exp2 on 25% of keys (f32x2)", w, din, dout, dcyc);
    run<14>("FMA-pipe exp2 on 50% of keys (f32x2)", w, din, dout, dcyc);
    run<42>("FMA-pipe exp2 on 25% of keys (scalar)", w, din, dout, dcyc);
  }
  cudaFree(din); cudaFree(dout); cudaFree(dcyc);
  return 0;
}
