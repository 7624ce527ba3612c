// Bidirectional flash attention over the joint video + audio sequence,
// o = softmax(q k^T / sqrt(D)) v per head, on the sm_100a tcgen05 path.
//
// One CTA per (pair of 128-query tiles A and B, head); both tiles share every
// K/V tile loaded into shared memory.  12 warps (warps 10, 11 idle):
//   warps 0..3  softmax of tile A, warps 4..7 softmax of tile B: thread t of a
//               warpgroup owns query row t (= TMEM lane t); it reads the score
//               row S from TMEM, keeps the running max m and sum l, and writes
//               P (bf16 pairs) back into the same TMEM columns, where the PV
//               MMA reads it as its A operand.  O is rescaled in TMEM only when
//               the running max grows by more than 2^8 (lazy rescale: o = O/l
//               is exact for any reference max, the threshold bounds P <= 256).
//   warp 8      TMA producer: Q_A, Q_B once; K tiles of 128 keys through a
//               three-stage ring, V tiles through a two-stage ring.
//   warp 9      MMA issuer: per key tile j, PV_A(j), S_A(j+1), PV_B(j),
//               S_B(j+1).  MMAs from one thread execute in issue order, so
//               S_A(j+1) may overwrite the columns PV_A(j) reads P from.
// TMEM (512 columns): S/P of A [0,128), O of A [128,256), S/P of B
// [256,384), O of B [384,512).
//
// exp2 runs on the MUFU unit (ex2.approx).  POLY_OF_8 > 0 moves that many
// key pairs of every eight to the FMA pipe, evaluated as 2^x = 2^n * p(f), n = rint(x), f = x - n in
// [-1/2, 1/2], p a degree-3 polynomial fitted to 2^f on that interval by
// iteratively reweighted least squares on relative error (max relative
// error 7.5e-5, below the bf16 rounding of P).  Keys past S in the last tile
// get score -inf before the row max, so one code path serves every tile and
// their probability is exp2(-inf) = 0; query rows past S are computed on
// zero-filled rows and not stored.
#include "common.cuh"
#include "kernels.h"

namespace h3b {

namespace {

constexpr int BQ = 128, BKV = 128, THREADS = 384, KS = 3, VS = 2;
// Register split (setmaxnreg): launch 384 x 168 = 64512; softmax warpgroups
// 2 x 128 x 216 = 55296 plus control warpgroup 128 x 56 = 7168 -> 62464.
constexpr int REG_SOFTMAX = 216, REG_CONTROL = 56;
constexpr int SOFTMAX_THREADS = 256;
constexpr int REG_SPLIT = SOFTMAX_THREADS * REG_SOFTMAX + (THREADS - SOFTMAX_THREADS) * REG_CONTROL;
constexpr float RESCALE_LOG2 = 8.0f;
constexpr int POLY_OF_8 = 0;   // key pairs (of every 8) that take the FMA-pipe exp2 (0: all on MUFU, measured fastest)
// TMEM column of tile t's S/P and O regions
__host__ __device__ constexpr uint32_t s_col(int t) { return t * 256u; }
__host__ __device__ constexpr uint32_t o_col(int t) { return t * 256u + 128u; }
constexpr int TMEM_COLS = 512;
// q_full, k_full/k_empty per K stage, v_full/v_empty per V stage, s_full x2, p_full x2x2, o_final x2, mma_done
constexpr int NUM_BARS = 1 + 2 * KS + 2 * VS + 2 + 4 + 2 + 1;

struct AttnArgs {
  int S, n_heads;
  __nv_bfloat16* out;
  int* err;
  int pairs;       // 256-row query pairs per head
  int n_full;      // work items (pair, head) run whole; the rest are split along keys
  int ks;          // key-range parts per split item
  float* partial;  // split parts: O [256][D] fp32, then m [256], l [256] per part
  size_t partial_elems;  // floats in partial (index checks)
};

template <int D>
constexpr int slot_floats() {
  return 256 * D + 2 * 256;
}

template <int D>
constexpr int smem_bytes() {
  return 1024 + (2 + KS + VS) * 128 * D * 2 + NUM_BARS * 8 + 16;
}

__device__ __forceinline__ float ex2_mufu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float m;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(a), "f"(b), "f"(c));
  return m;
}
__device__ __forceinline__ uint32_t cvt_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// 2^x for a pair, on the FMA pipe (x >= -126 after clamping; callers never pass -inf).
__device__ __forceinline__ uint64_t ex2_poly2(uint64_t x) {
  constexpr float C0 = 0.9999280571937561f, C1 = 0.6932609677314758f, C2 = 0.2426111400127411f,
                  C3 = 0.0551716685295105f;
  float x0 = fmaxf(f2_lo(x), -126.f), x1 = fmaxf(f2_hi(x), -126.f);
  const float t0 = x0 + 12582912.f, t1 = x1 + 12582912.f;  // 1.5 * 2^23: low mantissa bits = rint(x)
  const uint64_t f = f2_pack(x0 - (t0 - 12582912.f), x1 - (t1 - 12582912.f));
  uint64_t p = f2_fma(f2_pack(C3, C3), f, f2_pack(C2, C2));
  p = f2_fma(p, f, f2_pack(C1, C1));
  p = f2_fma(p, f, f2_pack(C0, C0));
  const uint32_t e0 = __float_as_uint(t0) << 23, e1 = __float_as_uint(t1) << 23;  // n << 23
  return f2_pack(__uint_as_float(__float_as_uint(f2_lo(p)) + e0), __uint_as_float(__float_as_uint(f2_hi(p)) + e1));
}

__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Probabilities of keys [64h, 64h+64) of one row, in place: pair i (keys 2i,
// 2i+1) reads r[2i], r[2i+1] and leaves its bf16 pair in r[i], a slot already
// consumed.  Partial row sums go to acc.  Keys past S hold -inf scores here
// (masked before the row max), so their exp2 is 0 on either pipe.
template <int HALF>
__device__ __forceinline__ void softmax_half(uint32_t (&r)[BKV], uint64_t c2, uint64_t nm2, uint64_t (&acc)[4]) {
#pragma unroll
  for (int i = 32 * HALF; i < 32 * HALF + 32; ++i) {
    const uint64_t x = f2_fma(f2_pack(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])), c2, nm2);
    uint64_t p;
    if ((i % 8) >= 8 - POLY_OF_8)
      p = ex2_poly2(x);
    else
      p = f2_pack(ex2_mufu(f2_lo(x)), ex2_mufu(f2_hi(x)));
    acc[i & 3] = f2_add(acc[i & 3], p);
    r[i] = cvt_bf16x2(f2_lo(p), f2_hi(p));
  }
}

template <int D>
__global__ void __launch_bounds__(THREADS, 1)
    k_attention(const __grid_constant__ CUtensorMap tm, const AttnArgs a) {
  const int S = a.S, n_heads = a.n_heads;
  int* const err = a.err;
  constexpr int KB = D / 64;         // 128-byte column blocks per head row
  constexpr int TILE = 128 * D * 2;  // bytes of a 128-row Q/K/V tile
  constexpr int BLK = 128 * 128;     // bytes of one 128-row x 128-byte block
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;               // tiles A, B
  uint8_t* sK = sQ + 2 * TILE;      // KS stages
  uint8_t* sV = sK + KS * TILE;     // VS stages
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + VS * TILE);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t b0 = smem_u32(bars);
  const uint32_t q_full = b0, k_full = b0 + 8, k_empty = k_full + 8 * KS, v_full = k_empty + 8 * KS,
                 v_empty = v_full + 8 * VS, s_full = v_empty + 8 * VS, p_full = s_full + 16, o_final = p_full + 32,
                 mma_done = o_final + 16;  // p_full: [tile][half]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d_model = n_heads * D;
  const int nkv_all = (S + BKV - 1) / BKV;
  // work item (query pair, head) and key-tile range [kv0, kv0 + nkv)
  int item, kv0 = 0, nkv = nkv_all, slot = -1;
  if (static_cast<int>(blockIdx.x) < a.n_full) {
    item = blockIdx.x;
  } else {
    slot = blockIdx.x - a.n_full;
    item = a.n_full + slot / a.ks;
    const int part = slot % a.ks;
    kv0 = part * nkv_all / a.ks;
    nkv = (part + 1) * nkv_all / a.ks - kv0;
  }
  const int q0 = (item % a.pairs) * 2 * BQ, h = item / a.pairs;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < KS; ++s) {
      mbar_init(k_full + 8 * s, 1);
      mbar_init(k_empty + 8 * s, 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(v_full + 8 * s, 1);
      mbar_init(v_empty + 8 * s, 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(s_full + 8 * t, 1);
      mbar_init(p_full + 16 * t, 4);
      mbar_init(p_full + 16 * t + 8, 4);
      mbar_init(o_final + 8 * t, 1);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  const uint32_t tmem = *tmem_slot;
  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REG_CONTROL));
  }
  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t k_issued = 0, v_issued = 0, k_par = 0, v_par = 0;
      mbar_arrive_expect_tx(q_full, 2 * TILE);
      for (int t = 0; t < 2; ++t)
        for (int kb = 0; kb < KB; ++kb)
          tma_load_2d(smem_u32(sQ + t * TILE + kb * BLK), &tm, q_full, h * D + 64 * kb, q0 + t * BQ);
      for (int jj = 0; jj < nkv; ++jj) {
        const int j = kv0 + jj;
        const int ks = jj % KS, vs = jj % VS;
        const uint32_t kph = (jj / KS) & 1, vph = (jj / VS) & 1;
        if (!mbar_wait(k_empty + 8 * ks, kph ^ 1, abort_flag, err, (EK_ATTN << 8) | 1)) break;
        mbar_arrive_expect_tx(k_full + 8 * ks, TILE);
        for (int kb = 0; kb < KB; ++kb)
          tma_load_2d(smem_u32(sK + ks * TILE + kb * BLK), &tm, k_full + 8 * ks, d_model + h * D + 64 * kb, j * BKV);
        k_issued |= 1u << ks;
        k_par = (k_par & ~(1u << ks)) | (kph << ks);
        if (!mbar_wait(v_empty + 8 * vs, vph ^ 1, abort_flag, err, (EK_ATTN << 8) | 2)) break;
        mbar_arrive_expect_tx(v_full + 8 * vs, TILE);
        for (int kb = 0; kb < KB; ++kb)
          tma_load_2d(smem_u32(sV + vs * TILE + kb * BLK), &tm, v_full + 8 * vs, 2 * d_model + h * D + 64 * kb,
                      j * BKV);
        v_issued |= 1u << vs;
        v_par = (v_par & ~(1u << vs)) | (vph << vs);
      }
      mbar_drain(q_full, 0);
      for (int s = 0; s < KS; ++s)
        if ((k_issued >> s) & 1) mbar_drain(k_full + 8 * s, (k_par >> s) & 1);
      for (int s = 0; s < VS; ++s)
        if ((v_issued >> s) & 1) mbar_drain(v_full + 8 * s, (v_par >> s) & 1);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(BQ, BKV, false);
      constexpr uint32_t idesc_o = idesc_bf16(BQ, D, true);  // V is MN-major (D contiguous)
      auto issue_s = [&](int t, int ks) {
        const uint32_t qa = smem_u32(sQ + t * TILE), ka = smem_u32(sK + ks * TILE);
#pragma unroll
        for (int i = 0; i < D / 16; ++i) {
          const uint32_t off = (i >> 2) * BLK + (i & 3) * 32;
          mma_bf16_ss(tmem + s_col(t), desc_sw128_k(qa + off), desc_sw128_k(ka + off), idesc_s, i != 0);
        }
      };
      // O_t += P_t V: keys [0,64) once the first half of P is published, then [64,128)
      auto issue_pv = [&](int t, int vs, bool acc, int j) -> bool {
        const uint32_t va = smem_u32(sV + vs * TILE);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          if (!mbar_wait(p_full + 16 * t + 8 * half, j & 1, abort_flag, err, (EK_ATTN << 8) | (6 + half)))
            return false;
          tc_fence_after();
#pragma unroll
          for (int i = 4 * half; i < 4 * half + 4; ++i)
            mma_bf16_ts(tmem + o_col(t), tmem + s_col(t) + 8 * i, desc_sw128_mn(va + i * 16 * 128, BLK), idesc_o,
                        acc || i != 0);
        }
        return true;
      };
      bool ok = mbar_wait(q_full, 0, abort_flag, err, (EK_ATTN << 8) | 3) &&
                mbar_wait(k_full, 0, abort_flag, err, (EK_ATTN << 8) | 4);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        tc_commit(s_full);
        issue_s(1, 0);
        tc_commit(s_full + 8);
        tc_commit(k_empty);
      }
      for (int j = 0; ok && j < nkv; ++j) {  // j: index inside this CTA's key range
        const int vs = j % VS, ks = (j + 1) % KS;
        const bool more = j + 1 < nkv;
        ok = mbar_wait(v_full + 8 * vs, (j / VS) & 1, abort_flag, err, (EK_ATTN << 8) | 5) &&
             issue_pv(0, vs, j > 0, j);
        if (!ok) break;
        if (more) {
          ok = mbar_wait(k_full + 8 * ks, ((j + 1) / KS) & 1, abort_flag, err, (EK_ATTN << 8) | 7);
          if (!ok) break;
          tc_fence_after();
          issue_s(0, ks);
          tc_commit(s_full);
        } else {
          tc_commit(o_final);
        }
        ok = issue_pv(1, vs, j > 0, j);
        if (!ok) break;
        tc_commit(v_empty + 8 * vs);
        if (more) {
          issue_s(1, ks);
          tc_commit(s_full + 8);
          tc_commit(k_empty + 8 * ks);
        } else {
          tc_commit(o_final + 8);
        }
      }
      tc_commit(mma_done);
      mbar_drain(mma_done, 0);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax (warps 0..7)
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REG_SOFTMAX));
    const int t = warp >> 2, q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t sc = tmem + lane_base + s_col(t), oc = tmem + lane_base + o_col(t);
    const float c = 1.4426950408889634f / sqrtf(static_cast<float>(D));  // log2(e) / sqrt(D)
    float m_use = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {  // j: index inside this CTA's key range
      ok = mbar_wait(s_full + 8 * t, j & 1, abort_flag, err, (EK_ATTN << 8) | 9);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int valid = S - (kv0 + j) * BKV;  // keys of this tile that exist (>= 1)
      // the whole score row, one TMEM round trip
      uint32_t r[BKV];
      tmem_ld32(sc + 0, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
      tmem_ld32(sc + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
      tmem_ld32(sc + 64, *reinterpret_cast<uint32_t(*)[32]>(&r[64]));
      tmem_ld32(sc + 96, *reinterpret_cast<uint32_t(*)[32]>(&r[96]));
      tmem_ld_wait();
      if (valid < BKV) {  // last tile of a ragged S: keys past S get score -inf
#pragma unroll
        for (int i = 0; i < BKV; ++i)
          if (i >= valid) r[i] = 0xff800000u;
      }
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int i = 0; i < BKV; i += 4) {
        mx0 = max3(mx0, __uint_as_float(r[i]), __uint_as_float(r[i + 1]));
        mx1 = max3(mx1, __uint_as_float(r[i + 2]), __uint_as_float(r[i + 3]));
      }
      const float m_new = fmaxf(mx0, mx1) * c;
      float alpha = 1.f;
      bool rescale = false;
      if (j == 0) {
        m_use = m_new;
      } else if (m_new > m_use + RESCALE_LOG2) {
        alpha = ex2_mufu(m_use - m_new);
        m_use = m_new;
        rescale = true;
      }
      // The commit behind s_full(j) follows PV(j-1), so O is complete here.
      if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(oc + cc * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(oc + cc * 32, o);
        }
      }
      // P of keys [0,64) -> TMEM columns [0,32), published; then keys [64,128) -> [32,64)
      const uint64_t c2 = f2_pack(c, c), nm2 = f2_pack(-m_use, -m_use);
      uint64_t acc[4] = {0, 0, 0, 0};
      softmax_half<0>(r, c2, nm2, acc);
      tmem_st32(sc + 0, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full + 16 * t);
      softmax_half<1>(r, c2, nm2, acc);
      tmem_st32(sc + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
      const uint64_t sum2 = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
      l = l * alpha + (f2_lo(sum2) + f2_hi(sum2));
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full + 16 * t + 8);
    }
    if (ok) {
      ok = mbar_wait(o_final + 8 * t, 0, abort_flag, err, (EK_ATTN << 8) | 10);
      if (__all_sync(0xffffffffu, ok) && slot >= 0) {
        // key-range part: unnormalised O, reference max m (log2 units) and sum l
        tc_fence_after();
        float* base = a.partial + static_cast<size_t>(slot) * slot_floats<D>();
        const int prow = t * BQ + row;
        const long long b0 = static_cast<long long>(slot) * slot_floats<D>(), pe = static_cast<long long>(a.partial_elems);
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(oc + cc * 32, o);
          tmem_ld_wait();
          float4* dst = reinterpret_cast<float4*>(base + static_cast<size_t>(prow) * D + cc * 32);
          if (idx_ok(err, b0 + static_cast<long long>(prow) * D + cc * 32, 32, pe, 31)) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(__uint_as_float(o[4 * i]), __uint_as_float(o[4 * i + 1]),
                                   __uint_as_float(o[4 * i + 2]), __uint_as_float(o[4 * i + 3]));
          }
        }
        if (idx_ok(err, b0 + 256 * D + prow, 257, pe, 31)) {  // m at +prow, l at +256+prow
          base[256 * D + prow] = m_use;
          base[256 * D + 256 + prow] = l;
        }
      } else if (__all_sync(0xffffffffu, ok)) {
        tc_fence_after();
        const float inv = 1.f / l;
        // Every MMA of the CTA has completed here (o_final follows the last S
        // MMA of both tiles), so the Q tiles are idle: each softmax warp stages
        // its 32 rows x D of bf16 output there (16-byte units XOR-swizzled by
        // row: conflict-free both ways) and then writes whole row segments,
        // 256/D rows per warp store instead of one 16-byte piece of 32 rows.
        constexpr int UNITS = D / 8;  // 16-byte units per output row
        uint8_t* stg = sQ + warp * (32 * D * 2);
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(oc + cc * 32, o);
          tmem_ld_wait();
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            w[i] = cvt_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            *reinterpret_cast<uint4*>(stg + lane * (D * 2) + (((cc * 4 + i) ^ (lane % UNITS)) << 4)) =
                make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
        __syncwarp();
        constexpr int RPI = 32 / UNITS;  // rows per warp store
        const int rbase = q0 + t * BQ + q * 32, u = lane % UNITS;
#pragma unroll
        for (int k = 0; k < 32 / RPI; ++k) {
          const int r = k * RPI + lane / UNITS;
          if (rbase + r < S && idx_ok(err, static_cast<long long>(rbase + r) * d_model + h * D + u * 8, 8,
                                      static_cast<long long>(S) * d_model, 30))
            *reinterpret_cast<uint4*>(a.out + static_cast<size_t>(rbase + r) * d_model + h * D + u * 8) =
                *reinterpret_cast<const uint4*>(stg + r * (D * 2) + ((u ^ (r % UNITS)) << 4));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// Merge the key-range parts of the split items: with M = max_c m_c,
// o = sum_c O_c 2^(m_c - M) / sum_c l_c 2^(m_c - M), parts in fixed order.
template <int D>
__global__ void __launch_bounds__(D) k_attn_combine(const AttnArgs a) {
  pdl_trigger();
  pdl_wait();
  const int ti = blockIdx.x / 256, r = blockIdx.x % 256, col = threadIdx.x;
  const int item = a.n_full + ti;
  const int grow = (item % a.pairs) * 2 * BQ + r, h = item / a.pairs;
  if (grow >= a.S) return;
  if (!idx_ok(a.err, static_cast<long long>(ti) * a.ks * slot_floats<D>(),
              static_cast<long long>(a.ks) * slot_floats<D>(), static_cast<long long>(a.partial_elems), 32) ||
      !idx_ok(a.err, static_cast<long long>(grow) * (a.n_heads * D) + h * D + col, 1,
              static_cast<long long>(a.S) * a.n_heads * D, 33))
    return;
  const float* base = a.partial + static_cast<size_t>(ti) * a.ks * slot_floats<D>();
  float M = -INFINITY;
  for (int c = 0; c < a.ks; ++c) M = fmaxf(M, base[static_cast<size_t>(c) * slot_floats<D>() + 256 * D + r]);
  float L = 0.f, acc = 0.f;
  for (int c = 0; c < a.ks; ++c) {
    const float* sl = base + static_cast<size_t>(c) * slot_floats<D>();
    const float w = exp2f(sl[256 * D + r] - M);
    L += sl[256 * D + 256 + r] * w;
    acc += sl[static_cast<size_t>(r) * D + col] * w;
  }
  a.out[static_cast<size_t>(grow) * (a.n_heads * D) + h * D + col] = __float2bfloat16_rn(acc / L);
}

__global__ void k_exp2_poly(const float* __restrict__ x, float* __restrict__ y, int n) {
  pdl_trigger();
  pdl_wait();
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    const uint64_t r = ex2_poly2(f2_pack(x[i], x[i + 1]));
    y[i] = f2_lo(r);
    y[i + 1] = f2_hi(r);
  } else if (i < n) {
    y[i] = f2_lo(ex2_poly2(f2_pack(x[i], 0.f)));
  }
}

}  // namespace

cudaError_t launch_exp2_poly(const Ctx& c, const float* x, float* y, int n) {
  if (n <= 0) return cudaSuccess;
  const int threads = 256, blocks = (n / 2 + threads) / threads;
  const cudaError_t e = launch_pdl(c.stream, k_exp2_poly, dim3(blocks), dim3(threads), 0, 1u, x, y, n);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_attention(const Ctx& c, const void* qkv, int S, int n_heads, int head_dim, void* o,
                             float* scratch, size_t scratch_bytes) {
  if (S == 0) return cudaSuccess;
  const int d_model = n_heads * head_dim;
  CUtensorMap tm;
  if (!encode_tmap_2d(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, qkv, 3ull * d_model, S, 3ull * d_model * 2, 64, 128))
    return cudaErrorInvalidValue;
  const bool d128 = head_dim == 128;
  auto kern = d128 ? k_attention<128> : k_attention<64>;
  // both sizes ask for the D=128 footprint: one CTA per SM (it holds all 512 TMEM columns)
  const int smem = smem_bytes<128>();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // setmaxnreg.inc waits until the registers the block was launched with cover
  // the split; a build whose register count could not grant it is refused here
  // rather than left to wait.
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.numRegs * THREADS < REG_SPLIT) return cudaErrorInvalidConfiguration;
  AttnArgs a;
  a.S = S;
  a.n_heads = n_heads;
  a.out = static_cast<__nv_bfloat16*>(o);
  a.err = c.err;
  a.pairs = (S + 2 * BQ - 1) / (2 * BQ);
  const int items = a.pairs * n_heads, nkv = (S + BKV - 1) / BKV;
  a.n_full = items;
  a.ks = 1;
  a.partial = nullptr;
  a.partial_elems = 0;
  // Items left after the last full wave, when they fill at most half of it,
  // are cut along the keys over the idle SMs and merged by a second kernel.
  const int tail = items % c.num_sms;
  const size_t slot_bytes = sizeof(float) * (d128 ? slot_floats<128>() : slot_floats<64>());
  if (scratch && items > c.num_sms && tail > 0 && 2 * tail <= c.num_sms) {
    int ks = c.num_sms / tail;
    if (ks > nkv / 2) ks = nkv / 2;
    if (static_cast<size_t>(tail) * ks * slot_bytes > scratch_bytes)
      ks = static_cast<int>(scratch_bytes / (static_cast<size_t>(tail) * slot_bytes));
    if (ks >= 2) {
      a.n_full = items - tail;
      a.ks = ks;
      a.partial = scratch;
      a.partial_elems = scratch_bytes / sizeof(float);
    }
  }
  const int grid = a.n_full + (items - a.n_full) * a.ks;
  e = launch_pdl(c.stream, kern, dim3(grid), dim3(THREADS), smem, 1u, tm, a);
  if (e != cudaSuccess) return e;
  e = cudaGetLastError();
  if (e != cudaSuccess || a.ks == 1) return e;
  if (d128)
    e = launch_pdl(c.stream, k_attn_combine<128>, dim3((items - a.n_full) * 256), dim3(128), 0, 1u, a);
  else
    e = launch_pdl(c.stream, k_attn_combine<64>, dim3((items - a.n_full) * 256), dim3(64), 0, 1u, a);
  return cudaGetLastError();
}

}  // namespace h3b
