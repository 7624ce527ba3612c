// Memory-bound kernels of the DiT block path: flow-matching Euler update,
// token merge / unmerge, RoPE table, RMSNorm (to bf16, or fused with per-token
// int8 quantisation) and per-row int8 quantisation.
//
// All of them stream HBM with 16-byte vector accesses, consecutive threads on
// consecutive 16-byte words, and grids sized in multiples of the SM count.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace h3b {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block-wide reduction (sum or max) for up to 32 warps; all threads get the result.
template <bool MAX>
__device__ __forceinline__ float block_reduce(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = MAX ? warp_max(v) : warp_sum(v);
  __syncthreads();  // protect `red` from the previous use
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = lane < nw ? red[lane] : (MAX ? 0.f : 0.f);
  r = MAX ? warp_max(r) : warp_sum(r);
  return r;
}

// Code of v for row scale s: rint(v / s) with the IEEE fp32 quotient,
// half-even, clamped to [-127, 127].  rs = 1/s.  v*rs is within a few ulp of
// v/s (|v/s| <= 127), so it rounds to the same integer unless the quotient lies
// within 1e-4 of a half-integer; only then is the exact quotient computed.
__device__ __forceinline__ int8_t quant1(float v, float s, float rs) {
  if (!(s > 0.f)) return 0;
  const float y = v * rs;
  float q = rintf(y);
  if (fabsf(fabsf(y - q) - 0.5f) < 1e-4f) q = rintf(v / s);
  q = fminf(fmaxf(q, -127.f), 127.f);
  return static_cast<int8_t>(static_cast<int>(q));
}

// Packed fp32 pairs with explicit round-to-nearest (never contracted into an FMA).
__device__ __forceinline__ uint64_t p2(float a, float b) {
  return (static_cast<uint64_t>(__float_as_uint(b)) << 32) | __float_as_uint(a);
}
__device__ __forceinline__ uint32_t lo32(uint64_t v) { return static_cast<uint32_t>(v); }
__device__ __forceinline__ uint32_t hi32(uint64_t v) { return static_cast<uint32_t>(v >> 32); }
__device__ __forceinline__ uint64_t mul2_rn(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t add2_rn(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t sub2_rn(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// max of three, NaN if any operand is NaN
__device__ __forceinline__ float max3_nan(float a, float b, float c) {
  float d;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Four codes (byte i = code of element i), identical to quant1 on each, in
// about a quarter of its instructions and none on the conversion pipe.  y =
// v*rs is rounded half-even to an integer by adding 1.5*2^23 (exact for
// |y| < 2^22), and the code is the low byte of the sum's bit pattern
// (two's complement: the constant's low byte is 0).  quant1 departs from
// rint(y) only when y lies within 1e-4 of a half-integer (it then takes the
// IEEE quotient) or rounds past +-127 (clamp); a group with such an element,
// |y| > 127.25 or a NaN goes through quant1.  y - rint(y) is exact, so the
// tie test is quant1's own comparison.
__device__ __forceinline__ uint32_t quant4(float a, float b, float c, float d, float s, float rs) {
  if (!(s > 0.f)) return 0u;
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  const uint64_t r2 = p2(rs, rs), k2 = p2(kRound, kRound);
  const uint64_t y01 = mul2_rn(p2(a, b), r2), y23 = mul2_rn(p2(c, d), r2);
  const uint64_t z01 = add2_rn(y01, k2), z23 = add2_rn(y23, k2);
  const uint64_t t01 = sub2_rn(y01, sub2_rn(z01, k2)), t23 = sub2_rn(y23, sub2_rn(z23, k2));
  const float tm = max3_nan(fabsf(__uint_as_float(lo32(t01))), fabsf(__uint_as_float(hi32(t01))),
                            fmaxf(fabsf(__uint_as_float(lo32(t23))), fabsf(__uint_as_float(hi32(t23)))));
  const float ym = max3_nan(fabsf(__uint_as_float(lo32(y01))), fabsf(__uint_as_float(hi32(y01))),
                            fmaxf(fabsf(__uint_as_float(lo32(y23))), fabsf(__uint_as_float(hi32(y23)))));
  if (!(0.5f - tm >= 1e-4f) || !(ym <= 127.25f))
    return static_cast<uint32_t>(static_cast<uint8_t>(quant1(a, s, rs))) |
           static_cast<uint32_t>(static_cast<uint8_t>(quant1(b, s, rs))) << 8 |
           static_cast<uint32_t>(static_cast<uint8_t>(quant1(c, s, rs))) << 16 |
           static_cast<uint32_t>(static_cast<uint8_t>(quant1(d, s, rs))) << 24;
  return __byte_perm(__byte_perm(lo32(z01), hi32(z01), 0x0040), __byte_perm(lo32(z23), hi32(z23), 0x0040), 0x5410);
}

// ------------------------------------------------------------------ Euler step
__global__ void k_flow(float* __restrict__ x, const float* __restrict__ v, float dt, size_t n,
                       float* __restrict__ xc, int* err) {
  pdl_trigger();
  pdl_wait();
  const size_t n4 = n >> 2;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  float4* x4 = reinterpret_cast<float4*>(x);
  const float4* v4 = reinterpret_cast<const float4*>(v);
  float4* c4 = reinterpret_cast<float4*>(xc);
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
    if (!idx_ok(err, 4 * i, 4, n, 1)) continue;
    float4 a = x4[i];
    const float4 b = __ldcs(v4 + i);
    a.x = fmaf(dt, b.x, a.x);
    a.y = fmaf(dt, b.y, a.y);
    a.z = fmaf(dt, b.z, a.z);
    a.w = fmaf(dt, b.w, a.w);
    x4[i] = a;
    if (xc) c4[i] = a;
  }
  for (size_t i = (n4 << 2) + static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
    if (!idx_ok(err, i, 1, n, 2)) continue;
    const float a = fmaf(dt, v[i], x[i]);
    x[i] = a;
    if (xc) xc[i] = a;
  }
}

// ------------------------------------------------------------------ token reduction
// Video token (f, r, 2c'+k) is row 2*((f*H + r)*(W/2) + c') + k of the full
// sequence, so merged row i averages full rows 2i and 2i+1; audio rows follow.
__global__ void k_merge(const float4* __restrict__ x, float4* __restrict__ xm, float4* __restrict__ xm_copy,
                        int half_video, int n_audio, int d4, int* err) {
  pdl_trigger();
  pdl_wait();
  const size_t total = static_cast<size_t>(half_video + n_audio) * d4;
  const long long full = (2ll * half_video + n_audio) * d4;  // float4 units of x
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t e = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total; e += stride) {
    const size_t row = e / d4, col = e - row * d4;
    if (!idx_ok(err, e, 1, total, 4)) continue;
    float4 o;
    if (row < static_cast<size_t>(half_video)) {
      if (!idx_ok(err, (2 * row) * d4 + col, d4 + 1, full, 3)) continue;  // rows 2 row and 2 row + 1
      const float4 a = __ldcs(x + (2 * row) * d4 + col);
      const float4 b = __ldcs(x + (2 * row + 1) * d4 + col);
      o.x = __fmul_rn(__fadd_rn(a.x, b.x), 0.5f);
      o.y = __fmul_rn(__fadd_rn(a.y, b.y), 0.5f);
      o.z = __fmul_rn(__fadd_rn(a.z, b.z), 0.5f);
      o.w = __fmul_rn(__fadd_rn(a.w, b.w), 0.5f);
    } else {
      if (!idx_ok(err, (row + half_video) * d4 + col, 1, full, 3)) continue;
      o = __ldcs(x + (row + half_video) * d4 + col);  // audio: full row = V + a = merged row + V/2
    }
    xm[e] = o;
    if (xm_copy) xm_copy[e] = o;
  }
}

__global__ void k_unmerge(const float4* __restrict__ xm, float4* __restrict__ x, int n_video, int n_audio, int d4,
                          int* err) {
  pdl_trigger();
  pdl_wait();
  const size_t total = static_cast<size_t>(n_video + n_audio) * d4;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  const int half = n_video / 2;
  for (size_t e = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total; e += stride) {
    const size_t row = e / d4, col = e - row * d4;
    const size_t src = row < static_cast<size_t>(n_video) ? row / 2 : row - half;
    if (!idx_ok(err, src * d4 + col, 1, (static_cast<long long>(half) + n_audio) * d4, 5)) continue;
    x[e] = xm[src * d4 + col];
  }
}

// Delta-broadcast unmerge: full video row r gains ym[r/2] - xm0[r/2] (the
// merged blocks' update); audio rows take ym.
__global__ void k_unmerge_delta(float4* __restrict__ x, const float4* __restrict__ ym,
                                const float4* __restrict__ xm0, int n_video, int n_audio, int d4, int* err) {
  pdl_trigger();
  pdl_wait();
  const size_t total = static_cast<size_t>(n_video + n_audio) * d4;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  const int half = n_video / 2;
  for (size_t e = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total; e += stride) {
    const size_t row = e / d4, col = e - row * d4;
    const long long merged = (static_cast<long long>(half) + n_audio) * d4;
    if (row < static_cast<size_t>(n_video)) {
      const size_t src = (row / 2) * d4 + col;
      if (!idx_ok(err, src, 1, merged, 6)) continue;
      const float4 y = ym[src], m = xm0[src];
      float4 v = x[e];
      v.x += y.x - m.x;
      v.y += y.y - m.y;
      v.z += y.z - m.z;
      v.w += y.w - m.w;
      x[e] = v;
    } else {
      if (!idx_ok(err, (row - half) * d4 + col, 1, merged, 7)) continue;
      x[e] = ym[(row - half) * d4 + col];
    }
  }
}

// ------------------------------------------------------------------ RoPE table
// table[s][j] = (cos, sin) of pos * theta^(-2 jl / n) for pair j of token s,
// jl the pair's index inside its section of width n (fp64 angle, fp32 store).
// The D/2 frequencies of the video sections and of the audio section are
// computed once per block (fp64) into shared memory; each element then costs
// one fp64 product and a fp64 reduction modulo 2 pi before the fp32 sincos.
constexpr int kMaxHalfHead = 64;  // head_dim <= 128
__global__ void k_rope_table(float2* __restrict__ table, int F, int H, int Wc, int A, int D, float theta,
                             int merged, int* err) {
  pdl_trigger();
  __shared__ double f_video[kMaxHalfHead], f_audio[kMaxHalfHead];
  const int half = D / 2;
  const int nf = D / 4, nr = 3 * D / 8, nc = D - nf - nr;
  const double l2t = log2(static_cast<double>(theta));
  for (int j = threadIdx.x; j < half; j += blockDim.x) {
    int jl, n;
    if (j < nf / 2) {
      jl = j; n = nf;
    } else if (j < (nf + nr) / 2) {
      jl = j - nf / 2; n = nr;
    } else {
      jl = j - (nf + nr) / 2; n = nc;
    }
    f_video[j] = exp2(-2.0 * jl / n * l2t);
    f_audio[j] = exp2(-2.0 * j / D * l2t);
  }
  __syncthreads();
  pdl_wait();  // the table may still be read by the previous block's QKV GEMM
  const int n_video = F * H * Wc;
  const size_t total = static_cast<size_t>(n_video + A) * half;
  for (size_t e = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int s = static_cast<int>(e / half), j = static_cast<int>(e % half);
    double ang;
    if (s < n_video) {
      const int f = s / (H * Wc), rem = s % (H * Wc), r = rem / Wc, c = rem % Wc;
      const double pos = j < nf / 2 ? f : j < (nf + nr) / 2 ? r : (merged ? 2.0 * c + 0.5 : static_cast<double>(c));
      ang = pos * f_video[j];
    } else {
      ang = static_cast<double>(s - n_video) * f_audio[j];
    }
    // reduce to about [-pi, pi] in fp64, then fp32 sin/cos of the remainder
    const double two_pi = 6.283185307179586, inv_two_pi = 0.15915494309189535;
    const float red = static_cast<float>(fma(-rint(ang * inv_two_pi), two_pi, ang));
    float sn, cs;
    sincosf(red, &sn, &cs);
    if (!idx_ok(err, e, 1, total, 8)) continue;
    table[e] = make_float2(cs, sn);
  }
}

// ------------------------------------------------------------------ GELU (the FC1 epilogue's function)
__global__ void k_gelu(const float* __restrict__ x, float* __restrict__ y, size_t n, int* err) {
  pdl_trigger();
  pdl_wait();
  // pairs through the same packed form the GEMM epilogue uses; an odd last element alone
  const size_t pairs = n / 2;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < pairs;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    if (!idx_ok(err, 2 * i, 2, n, 9)) continue;
    float a = x[2 * i], b = x[2 * i + 1];
    gelu_erf2(a, b);
    y[2 * i] = a;
    y[2 * i + 1] = b;
  }
  if ((n & 1) && blockIdx.x == 0 && threadIdx.x == 0) y[n - 1] = gelu_erf(x[n - 1]);
}

// ------------------------------------------------------------------ RMSNorm (+ quant)
// One CTA per token row; the row stays in registers between the statistics and
// the output pass (x is read from HBM exactly once).
template <int VPT, bool INT8>
__global__ void __launch_bounds__(kThreads) k_rmsnorm(const float* __restrict__ x, const float* __restrict__ g, int d,
                                                      float eps, void* __restrict__ out, float* __restrict__ out_scale,
                                                      const Mod mod, int* err) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[32];
  const int row = blockIdx.x, d4 = d >> 2;
  const long long n4 = static_cast<long long>(gridDim.x) * d4;  // float4 units of x (and of the output rows)
  const float4* xr = reinterpret_cast<const float4*>(x + static_cast<size_t>(row) * d);
  const float4* g4 = reinterpret_cast<const float4*>(g);
  float4 v[VPT];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int c = threadIdx.x + i * blockDim.x;
    if (c < d4 && idx_ok(err, static_cast<long long>(row) * d4 + c, 1, n4, 10)) {
      v[i] = xr[c];
      ss += v[i].x * v[i].x + v[i].y * v[i].y + v[i].z * v[i].z + v[i].w * v[i].w;
    } else {
      v[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  ss = block_reduce<false>(ss, red);
  const float r = 1.0f / sqrtf(ss / static_cast<float>(d) + eps);
  const size_t cls = mod.shift && row >= mod.split ? static_cast<size_t>(mod.stride) : 0;
  const float4* sh4 = reinterpret_cast<const float4*>(mod.shift + cls);
  const float4* sc4 = reinterpret_cast<const float4*>(mod.scale + cls);
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int c = threadIdx.x + i * blockDim.x;
    if (c < d4) {
      const float4 gg = g4[c];
      v[i].x = v[i].x * r * gg.x;
      v[i].y = v[i].y * r * gg.y;
      v[i].z = v[i].z * r * gg.z;
      v[i].w = v[i].w * r * gg.w;
      if (mod.shift) {
        const float4 sh = __ldg(sh4 + c), sc = __ldg(sc4 + c);
        v[i].x = fmaf(v[i].x, 1.0f + sc.x, sh.x);
        v[i].y = fmaf(v[i].y, 1.0f + sc.y, sh.y);
        v[i].z = fmaf(v[i].z, 1.0f + sc.z, sh.z);
        v[i].w = fmaf(v[i].w, 1.0f + sc.w, sh.w);
      }
      if (INT8) amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v[i].x), fabsf(v[i].y)), fmaxf(fabsf(v[i].z), fabsf(v[i].w))));
      else {
        uint2 p;
        p.x = pack_bf16x2(v[i].x, v[i].y);
        p.y = pack_bf16x2(v[i].z, v[i].w);
        if (idx_ok(err, static_cast<long long>(row) * d4 + c, 1, n4, 11))
          reinterpret_cast<uint2*>(out)[static_cast<size_t>(row) * d4 + c] = p;
      }
    }
  }
  if (INT8) {
    amax = block_reduce<true>(amax, red);
    const float s = amax / 127.0f, rs = 1.0f / s;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int c = threadIdx.x + i * blockDim.x;
      if (c < d4 && idx_ok(err, static_cast<long long>(row) * d4 + c, 1, n4, 11))
        reinterpret_cast<uint32_t*>(out)[static_cast<size_t>(row) * d4 + c] = quant4(v[i].x, v[i].y, v[i].z, v[i].w, s, rs);
    }
    if (threadIdx.x == 0 && idx_ok(err, row, 1, gridDim.x, 12)) out_scale[row] = s;
  }
}

// ------------------------------------------------------------------ row quantisation
__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ uint2 quant8(const float (&f)[8], float s, float rs) {
  return make_uint2(quant4(f[0], f[1], f[2], f[3], s, rs), quant4(f[4], f[5], f[6], f[7], s, rs));
}

// max |.| of 8 bf16 on packed pairs: the sign bits cleared, then bf16x2 max
// (exact: the max of bf16 magnitudes is one of them), widened once.
__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a & 0x7fff7fffu), "r"(b & 0x7fff7fffu));
  return r;
}
__device__ __forceinline__ float bf16x8_absmax(const uint4& u) {
  const uint32_t m = bf16x2_absmax(bf16x2_absmax(u.x, u.y), bf16x2_absmax(u.z, u.w));
  return fmaxf(__uint_as_float(m << 16), __uint_as_float(m & 0xffff0000u));
}

// One CTA per row: max |row| then codes, row held in registers.
template <int VPT>
__global__ void __launch_bounds__(kThreads) k_quant_rows(const uint4* __restrict__ a, int k8, int8_t* __restrict__ q,
                                                         float* __restrict__ scale, int* err) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[32];
  const int row = blockIdx.x;
  const uint4* ar = a + static_cast<size_t>(row) * k8;
  uint4 v[VPT];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int c = threadIdx.x + i * blockDim.x;
    v[i] = c < k8 && idx_ok(err, static_cast<long long>(row) * k8 + c, 1, static_cast<long long>(gridDim.x) * k8, 13)
               ? ar[c]
               : make_uint4(0, 0, 0, 0);
    amax = fmaxf(amax, bf16x8_absmax(v[i]));
  }
  amax = block_reduce<true>(amax, red);
  const float s = amax / 127.0f, rs = 1.0f / s;
  uint2* qr = reinterpret_cast<uint2*>(q + static_cast<size_t>(row) * k8 * 8);
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int c = threadIdx.x + i * blockDim.x;
    if (c < k8 && idx_ok(err, static_cast<long long>(row) * k8 + c, 1, static_cast<long long>(gridDim.x) * k8, 14)) {
      float f[8];
      bf16x8_to_f32(v[i], f);
      qr[c] = quant8(f, s, rs);
    }
  }
  if (threadIdx.x == 0 && idx_ok(err, row, 1, gridDim.x, 14)) scale[row] = s;
}

// Known row maxima: purely elementwise.  One CTA per row; thread t takes the
// 16-element chunks t, t + 256, ... (CPT of them), issues all their loads
// (two 16 bytes each) before the row scale's two divisions and before it
// converts any, and writes 16 codes per chunk in one 16-byte store.  Against
// a grid of one 16-element chunk per thread: 269 -> 237 us for the
// 20640 x 20480 FC2 input (0.72 -> 0.82 of the measured copy bandwidth).
template <int CPT>
__global__ void __launch_bounds__(kThreads) k_quant_absmax(const uint4* __restrict__ a,
                                                           const float* __restrict__ absmax, int k16,
                                                           int8_t* __restrict__ q, float* __restrict__ scale,
                                                           int* err) {
  pdl_trigger();
  pdl_wait();
  const int row = blockIdx.x;
  const long long n16 = static_cast<long long>(gridDim.x) * k16;  // 16-element chunks of a and q
  const uint4* ar = a + static_cast<size_t>(row) * k16 * 2;
  uint4* qr = reinterpret_cast<uint4*>(q) + static_cast<size_t>(row) * k16;
  uint4 v[2 * CPT];
#pragma unroll
  for (int i = 0; i < CPT; ++i) {
    const int c = threadIdx.x + i * kThreads;
    if (c < k16 && idx_ok(err, 2 * (static_cast<long long>(row) * k16 + c), 2, 2 * n16, 15)) {
      v[2 * i] = __ldcs(ar + 2 * c);
      v[2 * i + 1] = __ldcs(ar + 2 * c + 1);
    }
  }
  const float s = idx_ok(err, row, 1, gridDim.x, 17) ? absmax[row] / 127.0f : 0.f, rs = 1.0f / s;
#pragma unroll
  for (int i = 0; i < CPT; ++i) {
    const int c = threadIdx.x + i * kThreads;
    if (c < k16 && idx_ok(err, static_cast<long long>(row) * k16 + c, 1, n16, 16)) {
      float f0[8], f1[8];
      bf16x8_to_f32(v[2 * i], f0);
      bf16x8_to_f32(v[2 * i + 1], f1);
      const uint2 lo = quant8(f0, s, rs), hi = quant8(f1, s, rs);
      qr[c] = make_uint4(lo.x, lo.y, hi.x, hi.y);
    }
  }
  if (threadIdx.x == 0 && idx_ok(err, row, 1, gridDim.x, 17)) scale[row] = s;
}

// Same with 8 elements per thread (k a multiple of 8 but not of 16).
__global__ void k_quant_absmax8(const uint4* __restrict__ a, const float* __restrict__ absmax, int k8,
                                int8_t* __restrict__ q, float* __restrict__ scale, int* err) {
  pdl_trigger();
  pdl_wait();
  const int row = blockIdx.y;
  const long long n8 = static_cast<long long>(gridDim.y) * k8;  // 8-element chunks of a and q (this launch)
  const float s = idx_ok(err, row, 1, gridDim.y, 17) ? absmax[row] / 127.0f : 0.f, rs = 1.0f / s;
  const uint4* ar = a + static_cast<size_t>(row) * k8;
  uint2* qr = reinterpret_cast<uint2*>(q) + static_cast<size_t>(row) * k8;
  for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < k8; c += gridDim.x * blockDim.x) {
    if (!idx_ok(err, static_cast<long long>(row) * k8 + c, 1, n8, 15)) continue;
    float f[8];
    bf16x8_to_f32(__ldcs(ar + c), f);
    qr[c] = quant8(f, s, rs);
  }
  if (blockIdx.x == 0 && threadIdx.x == 0 && idx_ok(err, row, 1, gridDim.y, 17)) scale[row] = s;
}

// Self-test of the index checks: one thread passes index i of an extent n
// through idx_ok as every checked access does, without touching memory.  In
// the index-checked build an i outside [0, n) records (EK_INDEX << 8) | 99.
__global__ void k_selftest_index(int* err, long long i, long long n) {
  pdl_trigger();
  pdl_wait();
  if (idx_ok(err, i, 1, n, 99)) {
  }
}

// Failure-path self-test: wait on an mbarrier that nothing will complete,
// with a short limit; the bounded wait must give up, record its code in the
// device error word and let the kernel exit normally.
__global__ void k_selftest_wait(int* err, unsigned long long timeout_ns) {
  pdl_trigger();
  pdl_wait();
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, &abort_flag, err, (EK_SELFTEST << 8) | 1, timeout_ns);
  __syncthreads();
}

int grid_for(size_t work_items, int num_sms, int per_sm = 8) {
  const size_t want = (work_items + kThreads - 1) / kThreads;
  const size_t cap = static_cast<size_t>(num_sms) * per_sm;
  return static_cast<int>(want < cap ? (want > 0 ? want : 1) : cap);
}

}  // namespace

cudaError_t launch_flow_step(const Ctx& c, float* x, const float* v, float dt, size_t n, float* x_copy) {
  if (n == 0) return cudaSuccess;
  return launch_pdl(c.stream, k_flow, dim3(grid_for((n + 3) / 4, c.num_sms)), dim3(kThreads), 0, 1u, x, v, dt, n,
                    x_copy, c.err);
}

cudaError_t launch_merge(const Ctx& c, const float* x, float* xm, int n_video, int n_audio, int d, float* xm_copy) {
  const int d4 = d / 4;
  const size_t total = static_cast<size_t>(n_video / 2 + n_audio) * d4;
  if (total == 0) return cudaSuccess;
  return launch_pdl(c.stream, k_merge, dim3(grid_for(total, c.num_sms)), dim3(kThreads), 0, 1u,
                    reinterpret_cast<const float4*>(x), reinterpret_cast<float4*>(xm),
                    reinterpret_cast<float4*>(xm_copy), n_video / 2, n_audio, d4, c.err);
}

cudaError_t launch_unmerge_delta(const Ctx& c, float* x, const float* ym, const float* xm0, int n_video, int n_audio,
                                 int d) {
  const int d4 = d / 4;
  const size_t total = static_cast<size_t>(n_video + n_audio) * d4;
  if (total == 0) return cudaSuccess;
  return launch_pdl(c.stream, k_unmerge_delta, dim3(grid_for(total, c.num_sms)), dim3(kThreads), 0, 1u,
                    reinterpret_cast<float4*>(x), reinterpret_cast<const float4*>(ym),
                    reinterpret_cast<const float4*>(xm0), n_video, n_audio, d4, c.err);
}

cudaError_t launch_unmerge(const Ctx& c, const float* xm, float* x, int n_video, int n_audio, int d) {
  const int d4 = d / 4;
  const size_t total = static_cast<size_t>(n_video + n_audio) * d4;
  if (total == 0) return cudaSuccess;
  return launch_pdl(c.stream, k_unmerge, dim3(grid_for(total, c.num_sms)), dim3(kThreads), 0, 1u,
                    reinterpret_cast<const float4*>(xm), reinterpret_cast<float4*>(x), n_video, n_audio, d4, c.err);
}

cudaError_t launch_rope_table(const Ctx& c, const h3b_dims& dm, int merged, float* table) {
  const int wc = merged ? dm.cols / 2 : dm.cols;
  const size_t total = static_cast<size_t>(dm.frames * dm.rows * wc + dm.n_audio) * (dm.head_dim / 2);
  if (total == 0) return cudaSuccess;
  return launch_pdl(c.stream, k_rope_table, dim3(grid_for(total, c.num_sms, 8)), dim3(kThreads), 0, 1u,
                    reinterpret_cast<float2*>(table), dm.frames, dm.rows, wc, dm.n_audio, dm.head_dim, dm.rope_theta,
                    merged, c.err);
}

cudaError_t launch_gelu(const Ctx& c, const float* x, float* y, size_t n) {
  if (n == 0) return cudaSuccess;
  return launch_pdl(c.stream, k_gelu, dim3(grid_for(n, c.num_sms)), dim3(kThreads), 0, 1u, x, y, n, c.err);
}

cudaError_t launch_rmsnorm(const Ctx& c, const float* x, const float* g, int rows, int d, float eps, void* out,
                           float* out_scale, int out_int8, const Mod& mod) {
  if (rows == 0) return cudaSuccess;
  const int d4 = d / 4;
  int threads = d4 >= kThreads ? kThreads : ((d4 + 31) / 32) * 32;
  // The int8 variant does two block reductions per row; at d = 4096..6144
  // four warps per row (more rows in flight per SM) measured fastest at
  // d = 5120, S = 20640: 116 us with 256 threads, 110 with 128, 125 with 160,
  // 172 with 64.
  if (out_int8 && d4 % 128 == 0 && d4 / 128 >= 8 && d4 / 128 <= 12) threads = 128;
  const int vpt = (d4 + threads - 1) / threads;
  cudaError_t e;
#define H3B_NORM_CASE(V)                                                                                       \
  case V:                                                                                                      \
    e = out_int8 ? launch_pdl(c.stream, k_rmsnorm<V, true>, dim3(rows), dim3(threads), 0, 1u, x, g, d, eps, out,  \
                              out_scale, mod, c.err)                                                           \
                 : launch_pdl(c.stream, k_rmsnorm<V, false>, dim3(rows), dim3(threads), 0, 1u, x, g, d, eps, out, \
                              out_scale, mod, c.err);                                                          \
    break;
  switch (vpt) {
    H3B_NORM_CASE(1) H3B_NORM_CASE(2) H3B_NORM_CASE(3) H3B_NORM_CASE(4)
    H3B_NORM_CASE(5) H3B_NORM_CASE(6) H3B_NORM_CASE(7) H3B_NORM_CASE(8)
    H3B_NORM_CASE(9) H3B_NORM_CASE(10) H3B_NORM_CASE(11) H3B_NORM_CASE(12)
    default: return cudaErrorInvalidValue;
  }
#undef H3B_NORM_CASE
  return e;
}

cudaError_t launch_quant_rows(const Ctx& c, const void* a, int rows, int k, int8_t* q, float* s) {
  if (rows == 0) return cudaSuccess;
  const int k8 = k / 8;
  // the most warps (8 down to 5) that give every thread the same number of
  // 16-byte units (no idle lanes: k = 5120 takes 160 threads x 4), else 256
  int threads = k8 >= kThreads ? kThreads : ((k8 + 31) / 32) * 32;
  for (int w = 8; w >= 5 && k8 > kThreads; --w)
    if (k8 % (32 * w) == 0 && k8 / (32 * w) <= 16) {
      threads = 32 * w;
      break;
    }
  const int vpt = (k8 + threads - 1) / threads;
  const uint4* a4 = reinterpret_cast<const uint4*>(a);
  cudaError_t e;
#define H3B_Q_CASE(V) \
  case V: e = launch_pdl(c.stream, k_quant_rows<V>, dim3(rows), dim3(threads), 0, 1u, a4, k8, q, s, c.err); break;
  switch (vpt) {
    H3B_Q_CASE(1) H3B_Q_CASE(2) H3B_Q_CASE(3) H3B_Q_CASE(4) H3B_Q_CASE(5) H3B_Q_CASE(6)
    H3B_Q_CASE(7) H3B_Q_CASE(8) H3B_Q_CASE(9) H3B_Q_CASE(10) H3B_Q_CASE(11) H3B_Q_CASE(12)
    H3B_Q_CASE(13) H3B_Q_CASE(14) H3B_Q_CASE(15) H3B_Q_CASE(16)
    default: return cudaErrorInvalidValue;
  }
#undef H3B_Q_CASE
  return e;
}

cudaError_t launch_quant_absmax(const Ctx& c, const void* a, const float* absmax, int rows, int k, int8_t* q,
                                float* s) {
  if (rows == 0 || k == 0) return cudaSuccess;
  const uint4* a4 = reinterpret_cast<const uint4*>(a);
  const int k16 = k / 16, cpt = (k16 + kThreads - 1) / kThreads;
  if (k % 16 == 0 && cpt <= 8) {  // k <= 32768: one CTA per row
    cudaError_t e = cudaErrorInvalidValue;
#define H3B_QA_CASE(V) \
  case V:                                                                                                          \
    e = launch_pdl(c.stream, k_quant_absmax<V>, dim3(rows), dim3(kThreads), 0, 1u, a4, absmax, k16, q, s, c.err); \
    break;
    switch (cpt) {
      H3B_QA_CASE(1) H3B_QA_CASE(2) H3B_QA_CASE(3) H3B_QA_CASE(4) H3B_QA_CASE(5) H3B_QA_CASE(6)
      H3B_QA_CASE(7) H3B_QA_CASE(8)
    }
#undef H3B_QA_CASE
    return e != cudaSuccess ? e : cudaGetLastError();
  }
  // k a multiple of 8 only, or beyond 32768: 8 elements per thread, grid (chunks, rows)
  const int chunks = k / 8;
  const int bx = (chunks + kThreads - 1) / kThreads;
  for (int r0 = 0; r0 < rows; r0 += 65535) {  // grid.y limit
    const int nr = rows - r0 < 65535 ? rows - r0 : 65535;
    const dim3 grid(bx, nr);
    const uint4* ar = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a) + static_cast<size_t>(r0) * k);
    const cudaError_t e = launch_pdl(c.stream, k_quant_absmax8, grid, dim3(kThreads), 0, 1u, ar, absmax + r0, chunks,
                                     q + static_cast<size_t>(r0) * k, s + r0, c.err);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

cudaError_t launch_selftest_index(const Ctx& c, long long i, long long n) {
  return launch_pdl(c.stream, k_selftest_index, dim3(1), dim3(1), 0, 1u, c.err, i, n);
}

cudaError_t launch_selftest_wait(const Ctx& c, unsigned long long timeout_ns) {
  return launch_pdl(c.stream, k_selftest_wait, dim3(1), dim3(32), 0, 1u, c.err, timeout_ns);
}

}  // namespace h3b
