// Tensor-core GEMM C = A B^T for the DiT block's four linear layers, on the
// sm_100a tcgen05 path: TMA (128-byte swizzle) -> shared-memory ring ->
// tcgen05.mma (bf16 -> fp32, or int8 -> int32) with the accumulator in TMEM ->
// epilogue warps read TMEM and apply the fused epilogue.
//
// Two variants, both persistent over output tiles with one CTA per SM: the
// single-CTA kernel below (128x256 tiles) and a CTA-pair kernel (256x256
// tiles, tcgen05 cta_group::2, further down) used when the pair tiles fill at
// least one wave.  Single-CTA structure:
//   warp 0      TMA producer (one elected thread): A tile [128 x 128 B] and
//               B tile [256 x 128 B] per stage, 4 stages.
//   warp 1      MMA issuer (one thread): 4 MMAs of 128x256xK16 (bf16) or
//               128x256xK32 (int8) per stage; commits free the stage.
//   warps 2..9  epilogue: warp w reads TMEM lanes 32*(w%4).. (one output row
//               per thread) and writes half of the tile's columns (warps 2..5
//               the first 128, warps 6..9 the rest), 32 columns at a time.
// Two 256-column accumulators (all 512 TMEM columns) let the epilogue of
// tile i overlap the MMAs of tile i+1.
//
// Epilogues fused into the store (h3b.h H3B_EPI_*): plain fp32 / bf16, QKV
// with RoPE applied to the Q and K columns, fp32 residual add (x += acc),
// GELU (+ per-row max |GELU| for the next int8 quantisation), raw int32.
// INT8 inputs are dequantised as float(acc) * s_a[m] * s_w[n] first.
#include "common.cuh"
#include "kernels.h"

namespace h3b {

namespace {

constexpr int BM = 128, BN = 256, KBYTES = 128, STAGES = 4;
constexpr int A_STAGE = BM * KBYTES;  // 16 KB
constexpr int B_STAGE = BN * KBYTES;  // 32 KB
constexpr int TMEM_COLS = 2 * BN;     // two fp32 / int32 accumulators
constexpr int EPI_WARPS = 8;  // two warps per TMEM lane quarter, each half of the columns
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr int NUM_BARS = 2 * STAGES + 5;
constexpr int SMEM_BYTES = 1024 + STAGES * (A_STAGE + B_STAGE) + NUM_BARS * 8 + 16;
#ifndef H3B_GEMM_GROUP
#define H3B_GEMM_GROUP 0  // > 0: a fixed raster group width (tuning builds) instead of the measured rule
#endif

// Tile t -> (m block, n block): groups of group_n n-blocks, m-major inside a
// group, so the tiles in flight share a band of B and sweep A.
__device__ __forceinline__ void tile_coords(int t, int num_m, int num_n, int group_n, int& mb, int& nb) {
  const int per_group = num_m * group_n;
  const int g = t / per_group;
  const int first_n = g * group_n;
  const int gs = min(group_n, num_n - first_n);
  const int local = t - g * per_group;
  mb = local / gs;
  nb = first_n + local % gs;
}

// Work unit u -> (tile t, k-block range [kb0, kb1), split part or -1).  Units
// below full_tiles are whole tiles; when split > 1 the tiles left after the
// last full wave are cut into `split` consecutive K ranges each.
__device__ __forceinline__ void unit_range(int u, int full_tiles, int split, int num_kb, int& t, int& kb0, int& kb1,
                                           int& part) {
  if (split <= 1 || u < full_tiles) {
    t = u;
    kb0 = 0;
    kb1 = num_kb;
    part = -1;
    return;
  }
  const int v = u - full_tiles;
  t = full_tiles + v / split;
  part = v % split;
  kb0 = part * num_kb / split;
  kb1 = (part + 1) * num_kb / split;
}

// Residual epilogue through shared memory.  TMEM hands each thread one row of
// a 32x32 chunk; stored straight to global memory, every 16-byte access of a
// warp would touch 32 rows (32 cache lines).  Each epilogue warp instead parks
// the chunk in a 4 KB buffer of its own (16-byte groups XOR-swizzled by row:
// conflict-free both ways) and reads it back four rows per instruction, eight
// lanes covering one 128-byte row segment, so the residual read and write
// touch 4 lines per instruction.
constexpr int STG_FLOATS = 32 * 32;                   // one warp's buffer
constexpr int STG_BYTES = EPI_WARPS * STG_FLOATS * 4;  // 32 KB per CTA

__device__ __forceinline__ int stg_off(int row, int grp) { return row * 32 + ((grp ^ (row & 7)) << 2); }

// Row-per-thread values -> the warp's buffer (all lanes).
__device__ __forceinline__ void stage_put(float* stg, int lane, const float (&v)[32]) {
  __syncwarp();  // the previous chunk has been read back
#pragma unroll
  for (int j = 0; j < 8; ++j)
    *reinterpret_cast<float4*>(stg + stg_off(lane, j)) = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
  __syncwarp();
}

// Element group i of this lane: chunk row 4i + lane/8, columns 4(lane%8) .. +4.
__device__ __forceinline__ float4 stage_get(const float* stg, int lane, int i) {
  return *reinterpret_cast<const float4*>(stg + stg_off(4 * i + (lane >> 3), lane & 7));
}

// The residual values of a chunk in the same row-contiguous lane order
// (rows row0 .. row0+32 of C, columns n .. n+32; rows >= M read as 0).
__device__ __forceinline__ void load_resid_rows(const GemmArgs& p, int row0, int n, int lane, float4 (&dst)[8]) {
  const float* C = static_cast<const float*>(p.C) + n + 4 * (lane & 7);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = row0 + 4 * i + (lane >> 3);
    dst[i] = m < p.M && idx_ok(p.err, static_cast<long long>(m) * p.N + n + 4 * (lane & 7), 4,
                               static_cast<long long>(p.M) * p.N, 20)
                 ? *reinterpret_cast<const float4*>(C + static_cast<size_t>(m) * p.N)
                 : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// Row-per-thread fp32 values of one chunk (dequantised for INT8; row m >= M gives 0 scale).
template <bool INT8>
__device__ __forceinline__ void chunk_values(const GemmArgs& p, int m, int n, const uint32_t (&r)[32], float (&v)[32]) {
  if (INT8) {
    const float sa = m < p.M ? p.sa[m] : 0.f;
    const float4* sb4 = reinterpret_cast<const float4*>(p.sb + n);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 sb = __ldg(sb4 + i);
      v[4 * i + 0] = static_cast<float>(static_cast<int>(r[4 * i + 0])) * sa * sb.x;
      v[4 * i + 1] = static_cast<float>(static_cast<int>(r[4 * i + 1])) * sa * sb.y;
      v[4 * i + 2] = static_cast<float>(static_cast<int>(r[4 * i + 2])) * sa * sb.z;
      v[4 * i + 3] = static_cast<float>(static_cast<int>(r[4 * i + 3])) * sa * sb.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
  }
}

// Folded RMSNorm factor of row m (1 when the GEMM has none).
__device__ __forceinline__ float norm_row_scale(const GemmArgs& p, int m) {
  return p.row_scale && m < p.M ? p.row_scale[m] : 1.f;
}

// Sums of squares of the rows a warp wrote (ssq[i] for row row0 + 4i + lane/8,
// over this lane's columns) -> one partial per row and tile half.
__device__ __forceinline__ void store_row_squares(const GemmArgs& p, int row0, int lane, int part, float (&ssq)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float v = ssq[i];
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    const int m = row0 + 4 * i + (lane >> 3);
    if ((lane & 7) == 0 && m < p.M &&
        idx_ok(p.err, static_cast<long long>(m) * p.ss_parts + part, 1, static_cast<long long>(p.M) * p.ss_parts, 22))
      p.ss_out[static_cast<size_t>(m) * p.ss_parts + part] = v;
  }
}

// C[m, n .. n+32) += gate[class(m), n ..] * staged values (gate 1 when absent;
// fmaf(1, v, c) rounds exactly like c + v), res = the prefetched C values.
// With p.xb: also the bf16 copy of the new C times xb_gain, and each row's
// sum of squares added to ssq.
__device__ __forceinline__ void resid_rows(const GemmArgs& p, const float* stg, int row0, int n, int lane,
                                           const float4 (&res)[8], float (&ssq)[8]) {
  const int col = n + 4 * (lane & 7);
  float4 g0 = make_float4(1.f, 1.f, 1.f, 1.f), g1 = g0;
  if (p.gate) {
    g0 = __ldg(reinterpret_cast<const float4*>(p.gate + col));
    if (p.gate_split < p.M) g1 = __ldg(reinterpret_cast<const float4*>(p.gate + static_cast<size_t>(p.gate_stride) + col));
  }
  float* C = static_cast<float*>(p.C) + col;
  const float4 gn = p.xb ? __ldg(reinterpret_cast<const float4*>(p.xb_gain + col)) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = row0 + 4 * i + (lane >> 3);
    if (m < p.M && idx_ok(p.err, static_cast<long long>(m) * p.N + col, 4, static_cast<long long>(p.M) * p.N, 21)) {
      const float4 v = stage_get(stg, lane, i);
      const float4 g = m >= p.gate_split ? g1 : g0;
      float4 a = res[i];
      a.x = fmaf(g.x, v.x, a.x);
      a.y = fmaf(g.y, v.y, a.y);
      a.z = fmaf(g.z, v.z, a.z);
      a.w = fmaf(g.w, v.w, a.w);
      *reinterpret_cast<float4*>(C + static_cast<size_t>(m) * p.N) = a;
      if (p.xb) {
        *reinterpret_cast<uint2*>(p.xb + static_cast<size_t>(m) * p.N + col) =
            make_uint2(pack_bf16x2(a.x * gn.x, a.y * gn.y), pack_bf16x2(a.z * gn.z, a.w * gn.w));
        ssq[i] += a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w;
      }
    }
  }
}

// Staged chunk -> rows trow0 .. trow0+32 of a tile-shaped fp32 partial (row stride BN).
__device__ __forceinline__ void partial_rows(const GemmArgs& p, float* part, const float* stg, int trow0, int ccol,
                                             int lane) {
  float* dst = part + ccol + 4 * (lane & 7);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const long long off = static_cast<long long>(trow0 + 4 * i + (lane >> 3)) * BN;
    if (idx_ok(p.err, (dst - p.partial) + off, 4, static_cast<long long>(p.partial_elems), 24))
      *reinterpret_cast<float4*>(dst + off) = stage_get(stg, lane, i);
  }
}

// One chunk of a residual tile (whole tile or K-part), all lanes of the warp.
template <bool INT8>
__device__ __forceinline__ void resid_chunk(const GemmArgs& p, float* stg, int lane, int row0, int n, int ccol,
                                            const uint32_t (&r)[32], float* part, int trow0, float4 (&cnext)[8],
                                            bool more, float (&ssq)[8]) {
  float v[32];
  chunk_values<INT8>(p, row0 + lane, n, r, v);
  stage_put(stg, lane, v);
  if (part) {
    partial_rows(p, part, stg, trow0, ccol, lane);
    return;
  }
  float4 cur[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) cur[i] = cnext[i];
  if (more) load_resid_rows(p, row0, n + 32, lane, cnext);
  resid_rows(p, stg, row0, n, lane, cur, ssq);
}

// One 32-column chunk of one row (every epilogue but the residual one).
template <bool INT8, int EPI>
__device__ __forceinline__ void epilogue_chunk(const GemmArgs& p, int m, int n, const uint32_t (&r)[32],
                                               float& row_amax, float rs) {
  const size_t off = static_cast<size_t>(m) * p.N + n;
  if (!idx_ok(p.err, n, 32, p.N, 23) || !idx_ok(p.err, off, 32, static_cast<long long>(p.M) * p.N, 23)) return;
  if (EPI == H3B_EPI_I32) {
    int4* c = reinterpret_cast<int4*>(static_cast<int*>(p.C) + off);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      c[i] = make_int4(static_cast<int>(r[4 * i]), static_cast<int>(r[4 * i + 1]), static_cast<int>(r[4 * i + 2]),
                       static_cast<int>(r[4 * i + 3]));
    return;
  }
  float v[32];
  if (INT8) {
    const float sa = p.sa[m];
    const float4* sb4 = reinterpret_cast<const float4*>(p.sb + n);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 sb = __ldg(sb4 + i);
      v[4 * i + 0] = static_cast<float>(static_cast<int>(r[4 * i + 0])) * sa * sb.x;
      v[4 * i + 1] = static_cast<float>(static_cast<int>(r[4 * i + 1])) * sa * sb.y;
      v[4 * i + 2] = static_cast<float>(static_cast<int>(r[4 * i + 2])) * sa * sb.z;
      v[4 * i + 3] = static_cast<float>(static_cast<int>(r[4 * i + 3])) * sa * sb.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
  }
  if (p.row_scale) {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] *= rs;
  }

  if (EPI == H3B_EPI_F32) {
    float4* c = reinterpret_cast<float4*>(static_cast<float*>(p.C) + off);
#pragma unroll
    for (int i = 0; i < 8; ++i) c[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    return;
  }
  if (EPI == H3B_EPI_QKV_ROPE) {
    const int j0 = (n % p.head_dim) >> 1;
    if (n < 2 * p.d && m < p.rope_rows &&
        idx_ok(p.err, static_cast<long long>(m) * (p.head_dim >> 1) + j0, 16,
               static_cast<long long>(p.rope_rows) * (p.head_dim >> 1), 23)) {  // Q or K block: rotate 16 pairs
      const float4* t4 = reinterpret_cast<const float4*>(p.rope + static_cast<size_t>(m) * (p.head_dim >> 1) + j0);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 cs = __ldg(t4 + i);  // (cos, sin) of pairs 2i and 2i+1
        const float a0 = v[4 * i], a1 = v[4 * i + 1], b0 = v[4 * i + 2], b1 = v[4 * i + 3];
        v[4 * i] = a0 * cs.x - a1 * cs.y;
        v[4 * i + 1] = a0 * cs.y + a1 * cs.x;
        v[4 * i + 2] = b0 * cs.z - b1 * cs.w;
        v[4 * i + 3] = b0 * cs.w + b1 * cs.z;
      }
    }
  }
  if (EPI == H3B_EPI_GELU) {
#pragma unroll
    for (int i = 0; i < 32; i += 2) gelu_erf2(v[i], v[i + 1]);
  }
  // bf16 store (BF16, QKV_ROPE, GELU)
  uint32_t w[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
  if (EPI == H3B_EPI_GELU && INT8) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xffff0000u);
      row_amax = fmaxf(row_amax, fmaxf(fabsf(lo), fabsf(hi)));
    }
  }
  uint4* c = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.C) + off);
#pragma unroll
  for (int i = 0; i < 4; ++i) c[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
}

template <bool INT8, int EPI>
__global__ void __launch_bounds__(THREADS, 1)
    k_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const GemmArgs p) {
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_STAGE;
  float* stg_all = reinterpret_cast<float*>(sB + STAGES * B_STAGE);  // residual staging (RESID only)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + STAGES * B_STAGE + (EPI == H3B_EPI_RESID ? STG_BYTES : 0));
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t bar0 = smem_u32(bars);
  // barrier map: full[s], empty[s], tmem_full[2], tmem_empty[2], mma_done
  const uint32_t full0 = bar0, empty0 = bar0 + 8 * STAGES, tfull0 = bar0 + 16 * STAGES,
                 tempty0 = tfull0 + 16, mma_done = tempty0 + 16;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull0 + 8 * a, 1);
      mbar_init(tempty0 + 8 * a, EPI_WARPS);  // one arrival per epilogue warp
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  const uint32_t tmem_base = *tmem_slot;

  const int num_m = (p.M + BM - 1) / BM, num_n = (p.N + BN - 1) / BN, num_tiles = num_m * num_n;
  const int num_units = p.split > 1 ? p.full_tiles + (num_tiles - p.full_tiles) * p.split : num_tiles;
  constexpr int KE = INT8 ? 128 : 64;  // K elements per stage
  const int num_kb = p.K / KE;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_par = 0;
      for (int u = blockIdx.x; u < num_units; u += gridDim.x) {
        int t, kb0, kb1, part, mb, nb;
        unit_range(u, p.full_tiles, p.split, num_kb, t, kb0, kb1, part);
        tile_coords(t, num_m, num_n, p.group_n, mb, nb);
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1, abort_flag, p.err, (EK_GEMM << 8) | 1)) {
            ok = false;
            break;
          }
          const uint32_t fb = full0 + 8 * stage;
          mbar_arrive_expect_tx(fb, A_STAGE + B_STAGE);
          tma_load_2d(smem_u32(sA + stage * A_STAGE), &tmA, fb, kb * KE, mb * BM);
          tma_load_2d(smem_u32(sB + stage * B_STAGE), &tmB, fb, kb * KE, nb * BN);
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
      }
      // every copy this thread issued lands before the CTA may exit
      for (int s = 0; s < STAGES; ++s)
        if ((issued >> s) & 1) mbar_drain(full0 + 8 * s, (issued_par >> s) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = INT8 ? idesc_i8(BM, BN) : idesc_bf16(BM, BN, false);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      for (int u = blockIdx.x; u < num_units; u += gridDim.x) {
        int t, kb0, kb1, part;
        unit_range(u, p.full_tiles, p.split, num_kb, t, kb0, kb1, part);
        if (!mbar_wait(tempty0 + 8 * acc, acc_phase ^ 1, abort_flag, p.err, (EK_GEMM << 8) | 2)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(full0 + 8 * stage, phase, abort_flag, p.err, (EK_GEMM << 8) | 3)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * A_STAGE), b0 = smem_u32(sB + stage * B_STAGE);
#pragma unroll
          for (int k = 0; k < KBYTES / 32; ++k) {
            const uint64_t ad = desc_sw128_k(a0 + 32 * k), bd = desc_sw128_k(b0 + 32 * k);
            if (INT8)
              mma_i8_ss(d_tmem, ad, bd, idesc, (kb > kb0) || k != 0);
            else
              mma_bf16_ss(d_tmem, ad, bd, idesc, (kb > kb0) || k != 0);
          }
          tc_commit(empty0 + 8 * stage);  // frees the stage once these MMAs have read it
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        tc_commit(tfull0 + 8 * acc);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
      // all issued MMAs complete before TMEM can be released
      tc_commit(mma_done);
      mbar_drain(mma_done, 0);
    }
  } else {
    const int q = warp & 3;              // TMEM lane quarter this warp may access
    const int ch = (warp - 2) >> 2;      // column half of the tile this warp writes
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int u = blockIdx.x; u < num_units; u += gridDim.x) {
      int t, kb0, kb1, part, mb, nb;
      unit_range(u, p.full_tiles, p.split, num_kb, t, kb0, kb1, part);
      tile_coords(t, num_m, num_n, p.group_n, mb, nb);
      const bool ok = mbar_wait(tfull0 + 8 * acc, acc_phase, abort_flag, p.err, (EK_GEMM << 8) | 4);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const int m = mb * BM + q * 32 + lane;
      float row_amax = 0.f;
      // residual tiles: the next chunk's C values are in flight while this chunk is processed
      const int c0 = ch * (BN / 64), c1 = (ch + 1) * (BN / 64);
      float* const stg = stg_all + (warp - 2) * STG_FLOATS;
      float* const part_dst =
          EPI == H3B_EPI_RESID && part >= 0
              ? p.partial + (static_cast<size_t>(t - p.full_tiles) * p.split + part) * (BM * BN)
              : nullptr;
      float4 cnext[8];
      float ssq[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      const float rs = EPI == H3B_EPI_RESID ? 1.f : norm_row_scale(p, m);
      if (EPI == H3B_EPI_RESID && !part_dst && nb * BN + c0 * 32 < p.N)
        load_resid_rows(p, m - lane, nb * BN + c0 * 32, lane, cnext);
#pragma unroll 1
      for (int c = c0; c < c1; ++c) {
        const int n = nb * BN + c * 32;
        if (n >= p.N) break;
        uint32_t r[32];
        tmem_ld32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN + c * 32, r);
        tmem_ld_wait();
        if (EPI == H3B_EPI_RESID) {
          // K-parts of tail tiles write fp32 partials (added into C later, in part order)
          resid_chunk<INT8>(p, stg, lane, m - lane, n, c * 32, r, part_dst, q * 32, cnext,
                            c + 1 < c1 && n + 32 < p.N, ssq);
        } else if (m < p.M) {
          epilogue_chunk<INT8, EPI>(p, m, n, r, row_amax, rs);
        }
      }
      if (EPI == H3B_EPI_RESID && p.xb && !part_dst) store_row_squares(p, m - lane, lane, 2 * nb + ch, ssq);
      if (INT8 && EPI == H3B_EPI_GELU && m < p.M && idx_ok(p.err, m, 1, p.M, 25))
        atomicMax(reinterpret_cast<int*>(p.row_absmax) + m, __float_as_int(row_amax));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
  }

  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// C[m, n] += sum over parts of the tail tiles' fp32 partials, in part order
// (deterministic).  One CTA per (tail tile, row), one thread per column.
// With xb set (folded RMSNorm): also the bf16 copy of C times xb_gain and the
// row's sums of squares per 128-column tile half (the values the residual
// epilogue writes for whole tiles).
template <int TM>
__global__ void __launch_bounds__(BN) k_splitk_add(float* __restrict__ C, const float* __restrict__ partial, int M,
                                                   int N, int full_tiles, int split, int num_m, int num_n,
                                                   int group_n, const float* __restrict__ gate, int gate_split,
                                                   int gate_stride, __nv_bfloat16* __restrict__ xb,
                                                   const float* __restrict__ xb_gain, float* __restrict__ ss_out,
                                                   int ss_parts, int* err, size_t partial_elems) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[BN / 32];
  const int i = blockIdx.x / TM, r = blockIdx.x % TM, col = threadIdx.x;
  int mb, nb;
  tile_coords(full_tiles + i, num_m, num_n, group_n, mb, nb);
  const int m = mb * TM + r, n = nb * BN + col;
  if (m >= M) return;  // the whole CTA: m depends on the block only
  float sq = 0.f;
  const long long src0 = static_cast<long long>(i) * split * (TM * BN) + r * BN + col;
  if (n < N && idx_ok(err, src0, static_cast<long long>(split - 1) * (TM * BN) + 1,
                      static_cast<long long>(partial_elems), 26) &&
      idx_ok(err, static_cast<long long>(m) * N + n, 1, static_cast<long long>(M) * N, 27)) {
    const float* src = partial + src0;
    float acc = 0.f;
    for (int q = 0; q < split; ++q) acc += src[static_cast<size_t>(q) * (TM * BN)];
    float c = C[static_cast<size_t>(m) * N + n];
    c = gate ? fmaf(gate[(m >= gate_split ? static_cast<size_t>(gate_stride) : 0) + n], acc, c) : c + acc;
    C[static_cast<size_t>(m) * N + n] = c;
    if (xb) {
      xb[static_cast<size_t>(m) * N + n] = __float2bfloat16_rn(c * xb_gain[n]);
      sq = c * c;
    }
  }
  if (!xb) return;  // uniform: a kernel argument
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  if ((col & 31) == 0) red[col >> 5] = sq;
  __syncthreads();
  if (col < 2 && idx_ok(err, static_cast<long long>(m) * ss_parts + 2 * nb + col, 1,
                         static_cast<long long>(M) * ss_parts, 28)) {
    // warps 0-3 hold columns 0-127 of the tile, warps 4-7 columns 128-255
    const float h = red[4 * col] + red[4 * col + 1] + red[4 * col + 2] + red[4 * col + 3];
    ss_out[static_cast<size_t>(m) * ss_parts + 2 * nb + col] = h;
  }
}

// ---------------------------------------------------------------------------
// 2-SM variant: a cluster of two CTAs computes a 256x256 tile with
// tcgen05.mma.cta_group::2.  CTA rank r loads rows [128r, 128r+128) of the A
// tile and rows [128r, 128r+128) of the B tile (its half of N) into its own
// shared memory; the pair's MMA (issued by rank 0) reads both halves and
// leaves rows [128r, 128r+128) x all 256 columns of D in rank r's TMEM.  Per
// SM this feeds 32 KB per 64-wide K step instead of 48 KB.  Both ranks' TMA
// loads complete on rank 0's stage barrier; rank 0's commits arrive on both
// ranks' barriers (multicast commit); rank 1's epilogue releases the
// accumulator on rank 0's barrier.  No TMA load uses multicast.
constexpr int BM2 = 256;
constexpr int HALF_STAGE = 128 * KBYTES;  // 16 KB: 128 rows of A or B, one 128-byte K atom
constexpr int ATOMS_RING = 6;              // K atoms of A (and of B) in the ring
// K atoms per pipeline stage.  Two (128 bf16 / 256 int8 elements: eight MMAs
// per barrier wait and commit) leave the issuing thread slack to absorb the
// ALU-heavy GELU and RoPE epilogue warps that share its SM sub-partition; the
// residual GEMMs keep one atom per stage (finer release: more bytes in flight
// for their streamed A operand).
__host__ __device__ constexpr int pair_atoms(int epi) { return epi == H3B_EPI_RESID ? 1 : 2; }
constexpr int STAGES2 = ATOMS_RING;  // barrier slots (the most stages any epilogue uses)
constexpr int NUM_BARS2 = 2 * STAGES2 + 5;
constexpr int SMEM2_BYTES = 1024 + ATOMS_RING * 2 * HALF_STAGE + NUM_BARS2 * 8 + 16;
static_assert(SMEM2_BYTES + STG_BYTES <= 232448 && SMEM_BYTES + STG_BYTES <= 232448, "shared memory per CTA");
constexpr uint32_t PEER_BIT_CLEAR = 0xFEFFFFFFu;  // shared::cluster address of the same offset in rank 0

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
__device__ __forceinline__ uint32_t smem_in_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar_rank0, int x,
                                                 int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
      "[%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_rank0), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void mma2_bf16(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void mma2_i8(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
// arrive (once the issued MMAs complete) on the barrier at this offset in both ranks
__device__ __forceinline__ void commit2_both(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                   bar),
               "h"(static_cast<uint16_t>(3))
               : "memory");
}
__device__ __forceinline__ void commit2_local(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

template <bool INT8, int EPI>
__global__ void __launch_bounds__(THREADS, 1)
    k_gemm2(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const GemmArgs p) {
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  constexpr int AT = pair_atoms(EPI), NST = ATOMS_RING / AT, STAGE2 = AT * HALF_STAGE;
  uint8_t* sB = smem + ATOMS_RING * HALF_STAGE;
  float* stg_all = reinterpret_cast<float*>(sB + ATOMS_RING * HALF_STAGE);  // residual staging (RESID only)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + ATOMS_RING * HALF_STAGE + (EPI == H3B_EPI_RESID ? STG_BYTES : 0));
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NUM_BARS2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int cid = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
  const uint32_t bar0 = smem_u32(bars);
  // full[s] (rank 0's are used), empty[s], tmem_full[2], tmem_empty[2] (rank 0's are used), mma_done
  const uint32_t full0 = bar0, empty0 = bar0 + 8 * STAGES2, tfull0 = bar0 + 16 * STAGES2, tempty0 = tfull0 + 16,
                 mma_done = tempty0 + 16;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES2; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull0 + 8 * a, 1);
      mbar_init(tempty0 + 8 * a, 2 * EPI_WARPS);  // epilogue warps of both ranks
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both ranks' barriers exist before any cross-rank arrival
  tc_fence_after();
  pdl_wait();
  const uint32_t tmem_base = *tmem_slot;

  const int num_m = (p.M + BM2 - 1) / BM2, num_n = (p.N + BN - 1) / BN, num_tiles = num_m * num_n;
  const int num_units = p.split > 1 ? p.full_tiles + (num_tiles - p.full_tiles) * p.split : num_tiles;
  constexpr int KE = INT8 ? 128 : 64;
  constexpr int KS = AT * KE;         // K elements per stage
  const int num_kb = (p.K + KS - 1) / KS;  // stages; the last may hold one atom (K is a multiple of KE)

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, issued = 0, issued_par = 0;
      for (int u = cid; u < num_units; u += nclusters) {
        int t, kb0, kb1, part, mb, nb;
        unit_range(u, p.full_tiles, p.split, num_kb, t, kb0, kb1, part);
        tile_coords(t, num_m, num_n, p.group_n, mb, nb);
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1, abort_flag, p.err, (EK_GEMM << 8) | 5)) {
            ok = false;
            break;
          }
          const uint32_t fb = full0 + 8 * stage;
          const int na = AT == 1 ? 1 : min(AT, (p.K - kb * KS) / KE);
          if (leader) mbar_arrive_expect_tx(fb, 4 * HALF_STAGE * na);  // both ranks' A and B halves
          for (int a = 0; a < na; ++a) {
            tma_load_2d_pair(smem_u32(sA + stage * STAGE2 + a * HALF_STAGE), &tmA, fb & PEER_BIT_CLEAR,
                             kb * KS + a * KE, mb * BM2 + 128 * rank);
            tma_load_2d_pair(smem_u32(sB + stage * STAGE2 + a * HALF_STAGE), &tmB, fb & PEER_BIT_CLEAR,
                             kb * KS + a * KE, nb * BN + 128 * rank);
          }
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == NST) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
      }
      if (leader)  // rank 0's stage barriers count both ranks' bytes
        for (int s = 0; s < NST; ++s)
          if ((issued >> s) & 1) mbar_drain(full0 + 8 * s, (issued_par >> s) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      constexpr uint32_t idesc = INT8 ? idesc_i8(BM2, BN) : idesc_bf16(BM2, BN, false);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      for (int u = cid; u < num_units; u += nclusters) {
        int t, kb0, kb1, part;
        unit_range(u, p.full_tiles, p.split, num_kb, t, kb0, kb1, part);
        if (!mbar_wait(tempty0 + 8 * acc, acc_phase ^ 1, abort_flag, p.err, (EK_GEMM << 8) | 6)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(full0 + 8 * stage, phase, abort_flag, p.err, (EK_GEMM << 8) | 7)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * STAGE2), b0 = smem_u32(sB + stage * STAGE2);
          const int nk = AT == 1 ? KBYTES / 32 : min(AT, (p.K - kb * KS) / KE) * (KBYTES / 32);
#pragma unroll
          for (int k = 0; k < AT * (KBYTES / 32); ++k) {
            if (AT == 1 || k < nk) {
              const uint32_t off = (k / (KBYTES / 32)) * HALF_STAGE + 32 * (k % (KBYTES / 32));
              const uint64_t ad = desc_sw128_k(a0 + off), bd = desc_sw128_k(b0 + off);
              if (INT8)
                mma2_i8(d_tmem, ad, bd, idesc, (kb > kb0) || k != 0);
              else
                mma2_bf16(d_tmem, ad, bd, idesc, (kb > kb0) || k != 0);
            }
          }
          commit2_both(empty0 + 8 * stage);  // frees the stage in both ranks
          if (++stage == NST) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        commit2_both(tfull0 + 8 * acc);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
      commit2_local(mma_done);
      mbar_drain(mma_done, 0);
    }
  } else {
    const int q = warp & 3;
    const int ch = (warp - 2) >> 2;
    const uint32_t tempty_rank0 = smem_in_rank(tempty0, 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int u = cid; u < num_units; u += nclusters) {
      int t, kb0, kb1, part, mb, nb;
      unit_range(u, p.full_tiles, p.split, num_kb, t, kb0, kb1, part);
      tile_coords(t, num_m, num_n, p.group_n, mb, nb);
      const bool ok = mbar_wait(tfull0 + 8 * acc, acc_phase, abort_flag, p.err, (EK_GEMM << 8) | 8);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const int trow = 128 * rank + q * 32 + lane;  // row inside the 256-row tile
      const int m = mb * BM2 + trow;
      float row_amax = 0.f;
      const int c0 = ch * (BN / 64), c1 = (ch + 1) * (BN / 64);
      float* const stg = stg_all + (warp - 2) * STG_FLOATS;
      float* const part_dst =
          EPI == H3B_EPI_RESID && part >= 0
              ? p.partial + (static_cast<size_t>(t - p.full_tiles) * p.split + part) * (BM2 * BN)
              : nullptr;
      float4 cnext[8];
      float ssq[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      const float rs = EPI == H3B_EPI_RESID ? 1.f : norm_row_scale(p, m);
      if (EPI == H3B_EPI_RESID && !part_dst && nb * BN + c0 * 32 < p.N)
        load_resid_rows(p, m - lane, nb * BN + c0 * 32, lane, cnext);
#pragma unroll 1
      for (int c = c0; c < c1; ++c) {
        const int n = nb * BN + c * 32;
        if (n >= p.N) break;
        uint32_t r[32];
        tmem_ld32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN + c * 32, r);
        tmem_ld_wait();
        if (EPI == H3B_EPI_RESID) {
          resid_chunk<INT8>(p, stg, lane, m - lane, n, c * 32, r, part_dst, trow - lane, cnext,
                            c + 1 < c1 && n + 32 < p.N, ssq);
        } else if (m < p.M) {
          epilogue_chunk<INT8, EPI>(p, m, n, r, row_amax, rs);
        }
      }
      if (EPI == H3B_EPI_RESID && p.xb && !part_dst) store_row_squares(p, m - lane, lane, 2 * nb + ch, ssq);
      if (INT8 && EPI == H3B_EPI_GELU && m < p.M && idx_ok(p.err, m, 1, p.M, 25))
        atomicMax(reinterpret_cast<int*>(p.row_absmax) + m, __float_as_int(row_amax));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader)
          mbar_arrive(tempty0 + 8 * acc);
        else
          mbar_arrive_remote(tempty_rank0 + 8 * acc);
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // rank 0's MMAs are done and rank 1 no longer touches rank 0's barriers
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS) : "memory");
  }
}

using GemmKernel = void (*)(const CUtensorMap, const CUtensorMap, const GemmArgs);

template <bool INT8>
GemmKernel pick2(int epi) {
  switch (epi) {
    case H3B_EPI_F32: return k_gemm2<INT8, H3B_EPI_F32>;
    case H3B_EPI_BF16: return k_gemm2<INT8, H3B_EPI_BF16>;
    case H3B_EPI_QKV_ROPE: return k_gemm2<INT8, H3B_EPI_QKV_ROPE>;
    case H3B_EPI_RESID: return k_gemm2<INT8, H3B_EPI_RESID>;
    case H3B_EPI_GELU: return k_gemm2<INT8, H3B_EPI_GELU>;
    case H3B_EPI_I32: return INT8 ? k_gemm2<INT8, H3B_EPI_I32> : nullptr;
    default: return nullptr;
  }
}

template <bool INT8>
GemmKernel pick(int epi) {
  switch (epi) {
    case H3B_EPI_F32: return k_gemm<INT8, H3B_EPI_F32>;
    case H3B_EPI_BF16: return k_gemm<INT8, H3B_EPI_BF16>;
    case H3B_EPI_QKV_ROPE: return k_gemm<INT8, H3B_EPI_QKV_ROPE>;
    case H3B_EPI_RESID: return k_gemm<INT8, H3B_EPI_RESID>;
    case H3B_EPI_GELU: return k_gemm<INT8, H3B_EPI_GELU>;
    case H3B_EPI_I32: return INT8 ? k_gemm<INT8, H3B_EPI_I32> : nullptr;
    default: return nullptr;
  }
}

// One thread per row: the row's partial sums of squares in order -> factor.
__global__ void k_norm_scale(const float* __restrict__ ss, int rows, int parts, int d, float eps,
                             float* __restrict__ r, int* err) {
  pdl_trigger();
  pdl_wait();
  const int m = blockIdx.x * blockDim.x + threadIdx.x;
  if (m >= rows) return;
  if (!idx_ok(err, static_cast<long long>(m) * parts, parts, static_cast<long long>(rows) * parts, 29)) return;
  const float* q = ss + static_cast<size_t>(m) * parts;
  float s = 0.f;
  for (int i = 0; i < parts; ++i) s += q[i];
  r[m] = 1.0f / sqrtf(s / static_cast<float>(d) + eps);
}

}  // namespace

cudaError_t launch_norm_scale(const Ctx& c, const float* ss, int rows, int parts, int d, float eps, float* r) {
  if (rows == 0) return cudaSuccess;
  const cudaError_t e = launch_pdl(c.stream, k_norm_scale, dim3((rows + 127) / 128), dim3(128), 0, 1u, ss, rows,
                                   parts, d, eps, r, c.err);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_gemm(const Ctx& c, const void* A, const void* B, int ab_int8, int epi, const GemmArgs& args_in,
                        float* scratch, size_t scratch_bytes) {
  GemmArgs args = args_in;
  const int eb = ab_int8 ? 1 : 2;
  const CUtensorMapDataType dt = ab_int8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  // CTA pairs (256x256 tiles) when they fill at least one wave of pairs;
  // single CTAs (128x256 tiles) otherwise, for more parallelism.
  const int tiles2 = ((args.M + BM2 - 1) / BM2) * ((args.N + BN - 1) / BN);
  const bool pair = c.num_sms >= 2 && tiles2 >= c.num_sms / 2;
  const int TM = pair ? BM2 : BM;
  GemmKernel kern = pair ? (ab_int8 ? pick2<true>(epi) : pick2<false>(epi))
                         : (ab_int8 ? pick<true>(epi) : pick<false>(epi));
  if (!kern) return cudaErrorInvalidValue;
  CUtensorMap ta, tb;
  if (!encode_tmap_2d(&ta, dt, eb, A, args.K, args.M, static_cast<uint64_t>(args.K) * eb, KBYTES / eb, 128) ||
      !encode_tmap_2d(&tb, dt, eb, B, args.K, args.N, static_cast<uint64_t>(args.K) * eb, KBYTES / eb,
                      pair ? 128 : BN))
    return cudaErrorInvalidValue;
  const int smem = (pair ? SMEM2_BYTES : SMEM_BYTES) + (epi == H3B_EPI_RESID ? STG_BYTES : 0);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int num_m = (args.M + TM - 1) / TM, num_n = (args.N + BN - 1) / BN;
  const int tiles = num_m * num_n;
  // Raster group width: A is read from HBM about once per group of group_n
  // N tiles while the group's band of B stays in L2.  Measured HBM reads at
  // d = 5120 (widths 1, 8, 16, 19, 40): 16 for B rows of at most 1.5 MB per
  // N tile (the K = 5120 int8 GEMMs: FC1 at S = 20640 reads 652 MB at 16
  // against 1167 MB at 8), 8 otherwise (bf16 FC1 958-969 MB at 8-16 but
  // 1269 MB at 19; FC2 at K = 20480 1730 MB at 8, 2102 at 4, 1916 at 16).
  {
    int g = static_cast<double>(BN) * args.K * eb <= 1.5 * 1024 * 1024 ? 16 : 8;
    if (H3B_GEMM_GROUP > 0) g = H3B_GEMM_GROUP;
    args.group_n = g > num_n ? num_n : g;
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  int slots = c.num_sms;  // tiles in flight at once
  if (pair) {
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = c.stream;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // pairs must sit in one GPC: ask how many can be resident at once
    cfg.gridDim = dim3(c.num_sms);
    int active = 0;
    e = cudaOccupancyMaxActiveClusters(&active, kern, &cfg);
    if (e != cudaSuccess) return e;
    slots = active > 0 ? active : 1;
  }
  const int grid = tiles < slots ? tiles : slots;
  if (grid == 0) return cudaSuccess;
  // Residual GEMMs whose last wave is at most a third full: cut the tail
  // tiles along K over the idle SMs (partials in the caller's scratch).
  args.split = 1;
  args.full_tiles = tiles;
  args.partial = nullptr;
  args.partial_elems = 0;
  // K steps (stages) of the kernel that runs: two atoms per stage for pairs
  const int ke = (pair ? pair_atoms(epi) : 1) * (KBYTES / eb);
  const int num_kb = (args.K + ke - 1) / ke;
  const int rem = tiles % grid;
  if (epi == H3B_EPI_RESID && scratch && tiles > grid && rem > 0 && 3 * rem <= grid) {
    int split = grid / rem;
    if (split > num_kb / 2) split = num_kb / 2;
    const size_t per_split = static_cast<size_t>(rem) * TM * BN * sizeof(float);
    if (static_cast<size_t>(split) * per_split > scratch_bytes) split = static_cast<int>(scratch_bytes / per_split);
    if (split >= 2) {
      args.split = split;
      args.full_tiles = tiles - rem;
      args.partial = scratch;
      args.partial_elems = scratch_bytes / sizeof(float);
    }
  }
  e = launch_pdl(c.stream, kern, dim3(pair ? 2 * grid : grid), dim3(THREADS), smem, pair ? 2u : 1u, ta, tb, args);
  if (e != cudaSuccess) return e;
  e = cudaGetLastError();
  if (e != cudaSuccess || args.split <= 1) return e;
  if (pair)
    e = launch_pdl(c.stream, k_splitk_add<BM2>, dim3(rem * BM2), dim3(BN), 0, 1u, static_cast<float*>(args.C),
                   static_cast<const float*>(args.partial), args.M, args.N, args.full_tiles, args.split, num_m, num_n,
                   args.group_n, args.gate, args.gate_split, args.gate_stride, args.xb, args.xb_gain, args.ss_out,
                   args.ss_parts, args.err, args.partial_elems);
  else
    e = launch_pdl(c.stream, k_splitk_add<BM>, dim3(rem * BM), dim3(BN), 0, 1u, static_cast<float*>(args.C),
                   static_cast<const float*>(args.partial), args.M, args.N, args.full_tiles, args.split, num_m, num_n,
                   args.group_n, args.gate, args.gate_split, args.gate_stride, args.xb, args.xb_gain, args.ss_out,
                   args.ss_parts, args.err, args.partial_elems);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace h3b
