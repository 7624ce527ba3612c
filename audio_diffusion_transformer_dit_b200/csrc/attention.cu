// Bidirectional flash attention over the joint video + audio sequence,
// o = softmax(q k^T / sqrt(D)) v per head, on the sm_100a tcgen05 path.
//
// One CTA per (128-query tile, head); 6 warps:
//   warps 0..3  softmax: thread t owns query row t (= TMEM lane t); reads the
//               score row from TMEM, keeps the running max m and sum l,
//               writes P (bf16) into shared memory in the 128-byte-swizzled
//               K-major layout the MMA reads, and rescales O in TMEM when the
//               running max grows by more than 2^8 (lazy rescale: the result
//               o = O / l is exact for any reference max, the threshold only
//               bounds P <= 256).
//   warp 4      TMA producer: Q once, then K and V tiles of 128 keys through
//               two-stage rings.
//   warp 5      MMA issuer: S_j = Q K_j^T into one of two TMEM score buffers
//               (128 columns each), then O += P_{j-1} V_{j-1} (O: D columns of
//               TMEM), so the scores of tile j are computed while the softmax
//               of tile j-1 runs.
// Keys past S in the last tile are masked to -inf; query rows past S are
// computed on zero-filled rows and not stored.
#include "common.cuh"
#include "kernels.h"

namespace h3b {

namespace {

constexpr int BQ = 128, BKV = 128, THREADS = 192;
constexpr int TILE_BYTES_MAX = BQ * 128 * 2;  // 128 rows x D=128 bf16
constexpr int SMEM_BYTES = 1024 + TILE_BYTES_MAX * 6 + 32 * 8 + 16;
constexpr float RESCALE_LOG2 = 8.0f;
constexpr int S_COL0 = 0, O_COL = 2 * BKV, TMEM_COLS = 512;

template <int D>
__global__ void __launch_bounds__(THREADS, 1)
    k_attention(const __grid_constant__ CUtensorMap tm, int S, int n_heads, __nv_bfloat16* __restrict__ out,
                int* err) {
  constexpr int KB = D / 64;                 // 64-column (128-byte) blocks per head row
  constexpr int TILE = 128 * D * 2;          // bytes of a 128-row Q/K/V tile
  constexpr int BLK = 128 * 128;             // bytes of one 128-row x 128-byte block
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + TILE;        // 2 stages
  uint8_t* sV = sK + 2 * TILE;    // 2 stages
  uint8_t* sP = sV + 2 * TILE;    // 128 x 128 bf16 = 2 blocks
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + 2 * BLK);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 32);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t b0 = smem_u32(bars);
  const uint32_t q_full = b0, k_full = b0 + 8, k_empty = b0 + 24, v_full = b0 + 40, v_empty = b0 + 56,
                 s_full = b0 + 72, s_free = b0 + 88, p_full = b0 + 104, o_done = b0 + 112, mma_done = b0 + 120;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = blockIdx.x, h = blockIdx.y;
  const int d_model = n_heads * D;
  const int nkv = (S + BKV - 1) / BKV;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(k_full + 8 * s, 1);
      mbar_init(k_empty + 8 * s, 1);
      mbar_init(v_full + 8 * s, 1);
      mbar_init(v_empty + 8 * s, 1);
      mbar_init(s_full + 8 * s, 1);
      mbar_init(s_free + 8 * s, 4);
    }
    mbar_init(p_full, 4);
    mbar_init(o_done, 1);
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
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t k_issued = 0, v_issued = 0, k_par = 0, v_par = 0;
      mbar_arrive_expect_tx(q_full, TILE);
      for (int kb = 0; kb < KB; ++kb) tma_load_2d(smem_u32(sQ + kb * BLK), &tm, q_full, h * D + 64 * kb, qb * BQ);
      for (int j = 0; j < nkv; ++j) {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!mbar_wait(k_empty + 8 * st, ph ^ 1, abort_flag, err, (EK_ATTN << 8) | 1)) break;
        mbar_arrive_expect_tx(k_full + 8 * st, TILE);
        for (int kb = 0; kb < KB; ++kb)
          tma_load_2d(smem_u32(sK + st * TILE + kb * BLK), &tm, k_full + 8 * st, d_model + h * D + 64 * kb, j * BKV);
        k_issued |= 1u << st;
        k_par = (k_par & ~(1u << st)) | (ph << st);
        if (!mbar_wait(v_empty + 8 * st, ph ^ 1, abort_flag, err, (EK_ATTN << 8) | 2)) break;
        mbar_arrive_expect_tx(v_full + 8 * st, TILE);
        for (int kb = 0; kb < KB; ++kb)
          tma_load_2d(smem_u32(sV + st * TILE + kb * BLK), &tm, v_full + 8 * st, 2 * d_model + h * D + 64 * kb,
                      j * BKV);
        v_issued |= 1u << st;
        v_par = (v_par & ~(1u << st)) | (ph << st);
      }
      mbar_drain(q_full, 0);
      for (int s = 0; s < 2; ++s) {
        if ((k_issued >> s) & 1) mbar_drain(k_full + 8 * s, (k_par >> s) & 1);
        if ((v_issued >> s) & 1) mbar_drain(v_full + 8 * s, (v_par >> s) & 1);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(BQ, BKV, false);
      constexpr uint32_t idesc_o = idesc_bf16(BQ, D, true);  // V is MN-major (D contiguous)
      const uint32_t q0 = smem_u32(sQ), p0 = smem_u32(sP);
      bool ok = mbar_wait(q_full, 0, abort_flag, err, (EK_ATTN << 8) | 3);
      tc_fence_after();
      for (int j = 0; ok && j <= nkv; ++j) {
        if (j < nkv) {  // S_j = Q K_j^T
          const int st = j & 1;
          const uint32_t ph = (j >> 1) & 1;
          ok = mbar_wait(k_full + 8 * st, ph, abort_flag, err, (EK_ATTN << 8) | 4);
          if (ok && j >= 2) ok = mbar_wait(s_free + 8 * st, ph ^ 1, abort_flag, err, (EK_ATTN << 8) | 5);
          if (!ok) break;
          tc_fence_after();
          const uint32_t k0 = smem_u32(sK + st * TILE);
#pragma unroll
          for (int i = 0; i < D / 16; ++i) {
            const uint32_t off = (i >> 2) * BLK + (i & 3) * 32;
            mma_bf16_ss(tmem + S_COL0 + st * BKV, desc_sw128_k(q0 + off), desc_sw128_k(k0 + off), idesc_s, i != 0);
          }
          tc_commit(s_full + 8 * st);
          tc_commit(k_empty + 8 * st);
        }
        if (j >= 1) {  // O += P_{j-1} V_{j-1}
          const int jj = j - 1, st = jj & 1;
          ok = mbar_wait(p_full, jj & 1, abort_flag, err, (EK_ATTN << 8) | 6);
          if (ok) ok = mbar_wait(v_full + 8 * st, (jj >> 1) & 1, abort_flag, err, (EK_ATTN << 8) | 7);
          if (!ok) break;
          tc_fence_after();
          const uint32_t v0 = smem_u32(sV + st * TILE);
#pragma unroll
          for (int i = 0; i < BKV / 16; ++i) {
            const uint64_t ad = desc_sw128_k(p0 + (i >> 2) * BLK + (i & 3) * 32);
            const uint64_t bd = desc_sw128_mn(v0 + i * 16 * 128, BLK);
            mma_bf16_ss(tmem + O_COL, ad, bd, idesc_o, (jj | i) != 0);
          }
          tc_commit(o_done);
          tc_commit(v_empty + 8 * st);
        }
      }
      tc_commit(mma_done);
      mbar_drain(mma_done, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 0..3)
    const int row = warp * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const float c = 1.4426950408889634f / sqrtf(static_cast<float>(D));  // log2(e) / sqrt(D)
    float m_use = -INFINITY, l = 0.f;
    bool ok = true;
    const uint32_t prow = smem_u32(sP) + row * 128;
    for (int j = 0; j < nkv; ++j) {
      const int st = j & 1;
      ok = mbar_wait(s_full + 8 * st, (j >> 1) & 1, abort_flag, err, (EK_ATTN << 8) | 8);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[BKV];
#pragma unroll
      for (int cc = 0; cc < BKV / 32; ++cc) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + S_COL0 + st * BKV + cc * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) s[cc * 32 + i] = __uint_as_float(r[i]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free + 8 * st);  // score buffer may be overwritten

      const int valid = S - j * BKV;  // keys of this tile that exist
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < BKV; ++i) {
        if (i >= valid) s[i] = -INFINITY;
        mx = fmaxf(mx, s[i]);
      }
      const float m_new = mx * c;
      float alpha = 1.f;
      bool rescale = false;
      if (j == 0) {
        m_use = m_new;
      } else if (m_new > m_use + RESCALE_LOG2) {
        alpha = exp2f(m_use - m_new);
        m_use = m_new;
        rescale = true;
      }
      float sum = 0.f;
      uint32_t pk[BKV / 2];
#pragma unroll
      for (int i = 0; i < BKV / 2; ++i) {
        const float p0 = exp2f(fmaf(s[2 * i], c, -m_use));
        const float p1 = exp2f(fmaf(s[2 * i + 1], c, -m_use));
        sum += p0 + p1;
        pk[i] = pack_bf16x2(p0, p1);
      }
      l = l * alpha + sum;

      if (j >= 1) {  // PV_{j-1} must be done before P is overwritten or O rescaled
        ok = mbar_wait(o_done, (j - 1) & 1, abort_flag, err, (EK_ATTN << 8) | 9);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t r[32];
            const uint32_t ta = tmem + lane_base + O_COL + cc * 32;
            tmem_ld32(ta, r);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st32(ta, r);
          }
          tmem_st_wait();
        }
      }
      // P row -> shared memory, 128-byte swizzle (16-byte chunk c of row r at c ^ (r % 8))
#pragma unroll
      for (int cc = 0; cc < BKV / 8; ++cc) {
        const uint32_t addr = prow + (cc >> 3) * BLK + ((((cc & 7) ^ (row & 7))) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[4 * cc]), "r"(pk[4 * cc + 1]),
                     "r"(pk[4 * cc + 2]), "r"(pk[4 * cc + 3])
                     : "memory");
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (ok) {
      ok = mbar_wait(o_done, (nkv - 1) & 1, abort_flag, err, (EK_ATTN << 8) | 10);
      if (__all_sync(0xffffffffu, ok)) {
        tc_fence_after();
        const int grow = qb * BQ + row;
        const float inv = 1.f / l;
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t r[32];
          tmem_ld32(tmem + lane_base + O_COL + cc * 32, r);
          tmem_ld_wait();
          if (grow < S) {
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              w[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * inv, __uint_as_float(r[2 * i + 1]) * inv);
            uint4* dst = reinterpret_cast<uint4*>(out + static_cast<size_t>(grow) * d_model + h * D + cc * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
          }
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

}  // namespace

cudaError_t launch_attention(const Ctx& c, const void* qkv, int S, int n_heads, int head_dim, void* o) {
  if (S == 0) return cudaSuccess;
  const int d_model = n_heads * head_dim;
  CUtensorMap tm;
  if (!encode_tmap_2d(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, qkv, 3ull * d_model, S, 3ull * d_model * 2, 64, 128))
    return cudaErrorInvalidValue;
  auto kern = head_dim == 128 ? k_attention<128> : k_attention<64>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid((S + BQ - 1) / BQ, n_heads);
  kern<<<grid, THREADS, SMEM_BYTES, c.stream>>>(tm, S, n_heads, static_cast<__nv_bfloat16*>(o), c.err);
  return cudaGetLastError();
}

}  // namespace h3b
