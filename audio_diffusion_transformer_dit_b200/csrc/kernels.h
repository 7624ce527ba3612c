// Internal launcher declarations shared by the h3b translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "h3b.h"

namespace h3b {

// Launch with programmatic stream serialization (the kernel overlaps its
// prologue with its predecessor's tail; see pdl_wait in common.cuh).
// cluster_x > 1 adds a thread-block-cluster dimension.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(cudaStream_t stream, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       unsigned cluster_x, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  unsigned n = 1;
  if (cluster_x > 1) {
    at[1].id = cudaLaunchAttributeClusterDimension;
    at[1].val.clusterDim.x = cluster_x;
    at[1].val.clusterDim.y = 1;
    at[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = at;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// kernel ids for tracing (names in h3b_kernel_name)
enum KernelId {
  KID_FLOW = 0,
  KID_MERGE,
  KID_UNMERGE,
  KID_ROPE_TABLE,
  KID_RMSNORM,
  KID_QUANT_ROWS,
  KID_QUANT_ABSMAX,
  KID_GEMM_QKV,
  KID_GEMM_O,
  KID_GEMM_FC1,
  KID_GEMM_FC2,
  KID_GEMM,
  KID_ATTN,
  KID_MEMSET,
  KID_UNMERGE_DELTA,
  KID_COPY,
  KID_GELU,
  KID_NORM_SCALE,
  KID_COUNT
};

struct Ctx {
  cudaStream_t stream;
  int* err;
  int num_sms;
};

// returns cudaError_t of the launch
cudaError_t launch_flow_step(const Ctx& c, float* x, const float* v, float dt, size_t n, float* x_copy);
cudaError_t launch_merge(const Ctx& c, const float* x, float* xm, int n_video, int n_audio, int d,
                         float* xm_copy = nullptr);
cudaError_t launch_unmerge_delta(const Ctx& c, float* x, const float* ym, const float* xm0, int n_video, int n_audio,
                                 int d);
cudaError_t launch_unmerge(const Ctx& c, const float* xm, float* x, int n_video, int n_audio, int d);
cudaError_t launch_rope_table(const Ctx& c, const h3b_dims& dm, int merged, float* table);
// adaLN-style modulation of a normed row, y <- y * (1 + scale[k]) + shift[k]
// for k < d; rows >= split (the condition rows) read their vectors at +stride.
// shift == nullptr: no modulation.
struct Mod {
  const float* shift = nullptr;
  const float* scale = nullptr;
  int split = 0, stride = 0;
};
cudaError_t launch_gelu(const Ctx& c, const float* x, float* y, size_t n);
cudaError_t launch_rmsnorm(const Ctx& c, const float* x, const float* g, int rows, int d, float eps, void* out,
                           float* out_scale, int out_int8, const Mod& mod = Mod{});
cudaError_t launch_quant_rows(const Ctx& c, const void* a, int rows, int k, int8_t* q, float* s);
cudaError_t launch_quant_absmax(const Ctx& c, const void* a, const float* absmax, int rows, int k, int8_t* q,
                                float* s);

struct GemmArgs {
  int M, N, K;
  void* C;
  const float* sa;
  const float* sb;
  const float2* rope;
  int d, head_dim;
  float* row_absmax;
  int* err;
  // split-K of the tail tiles (residual epilogue only; set by launch_gemm)
  int full_tiles, split;
  float* partial;
  // residual epilogue: C += gate[n] * acc when gate is set (rows >= gate_split
  // read the gate at +gate_stride); QKV epilogue: rows >= rope_rows are not rotated
  const float* gate;
  int gate_split, gate_stride;
  int rope_rows;
  // raster group width in N tiles (set by launch_gemm)
  int group_n;
  // RMSNorm folded across two GEMMs (bf16 residual stream).  Residual
  // epilogue, when xb is set: also writes xb[m, n] = bf16(C[m, n] * xb_gain[n])
  // and, per row and 128-column tile half, the sum of C^2 into
  // ss_out[m * ss_parts + 2 * tile_n + half] (launch_norm_scale turns those
  // into one factor per row).  Other epilogues, when row_scale is set: scale
  // the accumulator of row m by row_scale[m] before RoPE / GELU.
  __nv_bfloat16* xb;
  const float* xb_gain;
  float* ss_out;
  int ss_parts;
  const float* row_scale;
  // floats in the split-K partial buffer (set by launch_gemm; index checks)
  size_t partial_elems;
};
// r[m] = 1 / sqrt(sum_q ss[m * parts + q] / d + eps), q in order (deterministic).
cudaError_t launch_norm_scale(const Ctx& c, const float* ss, int rows, int parts, int d, float eps, float* r);

// A [M,K], B [N,K] K-major (bf16 or int8); C per epilogue.  scratch (may be
// NULL) lets a residual GEMM split its last partial wave along K.
cudaError_t launch_gemm(const Ctx& c, const void* A, const void* B, int ab_int8, int epi, const GemmArgs& args,
                        float* scratch = nullptr, size_t scratch_bytes = 0);

// scratch (may be NULL) lets the last partial wave of work items split along the keys.
cudaError_t launch_attention(const Ctx& c, const void* qkv, int S, int n_heads, int head_dim, void* o,
                             float* scratch = nullptr, size_t scratch_bytes = 0);
cudaError_t launch_exp2_poly(const Ctx& c, const float* x, float* y, int n);
cudaError_t launch_selftest_wait(const Ctx& c, unsigned long long timeout_ns);
cudaError_t launch_selftest_index(const Ctx& c, long long i, long long n);

// tensor-map encoding through the driver entry point (no libcuda link)
bool encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, int elem_bytes, const void* base, uint64_t inner,
                    uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer);

}  // namespace h3b
