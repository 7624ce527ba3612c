// h3b C ABI: argument validation, workspace planning (aliased activation
// arenas), the block / stack / denoise orchestration, tracing and the
// tensor-map encoder.  Every entry point only enqueues work on the caller's
// stream; nothing here allocates device memory or synchronises (except the
// explicitly synchronising h3b_device_error / h3b_trace_stop).
#include <math.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "kernels.h"

namespace h3b {

__device__ int g_device_error;  // device error word (one per device)

namespace {

constexpr int kMaxDevices = 64;

// Per-device state, filled once under the mutex.  `ready` is published with
// release order after num_sms and err are written, and read with acquire
// order on the fast path, so a thread that sees ready == true also sees them.
struct DeviceInfo {
  std::atomic<bool> ready{false};
  int num_sms = 0;
  int* err = nullptr;
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

int device_ctx(cudaStream_t stream, Ctx* c) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return H3B_ERR_DEVICE;
  DeviceInfo& di = g_dev[dev];
  if (!di.ready.load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!di.ready.load(std::memory_order_relaxed)) {
      int major = 0, sms = 0;
      if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return H3B_ERR_DEVICE;
      if (major != 10) return H3B_ERR_DEVICE;
      if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return H3B_ERR_DEVICE;
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return H3B_ERR_CUDA;
      di.num_sms = sms;
      di.err = static_cast<int*>(p);
      di.ready.store(true, std::memory_order_release);
    }
  }
  c->stream = stream;
  c->err = di.err;
  c->num_sms = di.num_sms;
  return H3B_OK;
}

// ------------------------------------------------------------------ tracing
struct TraceRec {
  int kid;
  cudaEvent_t a, b;
};
struct Trace {
  bool on = false;
  int cap = 0, n = 0;
  std::vector<TraceRec> recs;
  std::vector<float> ms;
} g_trace;

const char* kKernelNames[KID_COUNT] = {"flow_step", "token_merge", "token_unmerge", "rope_table", "rmsnorm",
                                       "quant_rows", "quant_absmax", "gemm_qkv_rope", "gemm_o_resid",
                                       "gemm_fc1_gelu", "gemm_fc2_resid", "gemm", "attention", "memset",
                                       "token_unmerge_delta", "copy", "gelu", "norm_scale"};

struct TraceScope {
  TraceRec* rec = nullptr;
  cudaStream_t s;
  TraceScope(int kid, cudaStream_t st) : s(st) {
    if (g_trace.on && g_trace.n < g_trace.cap) {
      rec = &g_trace.recs[g_trace.n++];
      rec->kid = kid;
      cudaEventRecord(rec->a, s);
    }
  }
  ~TraceScope() {
    if (rec) cudaEventRecord(rec->b, s);
  }
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// ------------------------------------------------------------------ validation
int check_dims(const h3b_dims* dm) {
  if (!dm) return H3B_ERR_NULL;
  if (dm->frames < 0 || dm->rows < 0 || dm->cols < 0 || dm->n_audio < 0) return H3B_ERR_DIMS;
  if (dm->head_dim != 64 && dm->head_dim != 128) return H3B_ERR_DIMS;
  if (dm->n_heads <= 0 || dm->d != dm->n_heads * dm->head_dim) return H3B_ERR_DIMS;
  if (dm->d % 128 != 0 || dm->d > 8192) return H3B_ERR_DIMS;
  if (dm->ffn <= 0 || dm->ffn % 128 != 0 || dm->ffn > 32768) return H3B_ERR_DIMS;
  if (!(dm->eps >= 0.f) || !(dm->rope_theta > 0.f)) return H3B_ERR_DIMS;
  const long long s = 1LL * dm->frames * dm->rows * dm->cols + dm->n_audio;
  if (s <= 0 || s > (1LL << 24)) return H3B_ERR_DIMS;
  return H3B_OK;
}

int seq_len(const h3b_dims& dm, int merged) {
  return dm.frames * dm.rows * (merged ? dm.cols / 2 : dm.cols) + dm.n_audio;
}

size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace layout.  The block's activation arenas alias across its lifetime:
//   [qkv 3d bf16 | o d bf16 | u1 (norm-1 out)] during the attention half;
//   the MLP input u2 reuses the QKV arena (offset 0) and the FC1 hidden
//   overlays the rest (qkv, o and u1 are dead by then).
struct Plan {
  size_t qkv, o, u1, oq, u2, g, gq;   // byte offsets inside the arena
  size_t xb1, ss1, ss2, r1, r2;       // folded RMSNorm: next QKV input, partial sums, row factors (bf16)
  size_t arena, naive;                // arena bytes, bytes without aliasing
  size_t s_act, s_g, amax;            // fp32 [S] scale / max vectors (INT8)
  size_t rope, rope_m, xm;            // RoPE tables, merged-sequence buffer
  size_t xm0, delta;                  // merged input (delta unmerge), cached core update
  size_t total;
  int n_cond;                         // condition rows after the audio tokens
};

// Activations cover the generated rows plus n_cond condition rows; the RoPE
// tables cover the generated rows only (condition rows are not rotated).
Plan plan(const h3b_dims& dm, int dtype, int reduction, int keep_merged_input = 0, int core = 0, int n_cond = 0) {
  Plan p{};
  p.n_cond = n_cond;
  const size_t S = seq_len(dm, 0) + n_cond, d = dm.d, f = dm.ffn;
  if (dtype == H3B_INT8) {
    p.qkv = 0;
    p.o = al256(6 * d * S);
    p.u1 = p.o + al256(2 * d * S);
    p.oq = p.u1 + al256(d * S);
    const size_t attn_end = p.oq + al256(d * S);
    p.u2 = 0;
    p.g = al256(d * S);
    p.gq = p.g + al256(2 * f * S);
    const size_t mlp_end = p.gq + al256(f * S);
    p.arena = attn_end > mlp_end ? attn_end : mlp_end;
    p.naive = al256(6 * d * S) + al256(2 * d * S) + 3 * al256(d * S) + al256(2 * f * S) + al256(f * S);
  } else {
    p.qkv = 0;
    p.o = al256(6 * d * S);
    p.u1 = p.o + al256(2 * d * S);
    const size_t attn_end = p.u1 + al256(2 * d * S);
    p.u2 = 0;
    p.g = al256(2 * d * S);
    const size_t mlp_end = p.g + al256(2 * f * S);
    p.arena = attn_end > mlp_end ? attn_end : mlp_end;
    p.oq = p.gq = 0;
    p.naive = al256(6 * d * S) + 3 * al256(2 * d * S) + al256(2 * f * S);
  }
  size_t off = al256(p.arena);
  p.s_act = off;
  off += al256(S * 4);
  p.s_g = off;
  off += al256(S * 4);
  p.amax = off;
  off += al256(S * 4);
  p.rope = off;
  off += al256(static_cast<size_t>(seq_len(dm, 0)) * (dm.head_dim / 2) * 8);
  if (reduction) {
    const size_t Sm = seq_len(dm, 1) + n_cond;
    p.rope_m = off;
    off += al256(static_cast<size_t>(seq_len(dm, 1)) * (dm.head_dim / 2) * 8);
    p.xm = off;
    off += al256(Sm * d * 4);
  } else {
    p.rope_m = p.xm = 0;
  }
  p.xm0 = p.delta = 0;
  if (reduction && keep_merged_input) {
    p.xm0 = off;
    off += al256(static_cast<size_t>(seq_len(dm, 1) + n_cond) * d * 4);
  }
  if (core) {
    p.delta = off;
    off += al256(S * d * 4);
  }
  p.xb1 = p.ss1 = p.ss2 = p.r1 = p.r2 = 0;
  if (dtype != H3B_INT8) {
    // bf16(x * g) for the next block's QKV GEMM (the arena is full while FC2
    // reads the hidden activations), and the per-row partial sums of squares
    // of both folded norms (2 per 256-column tile of d)
    const size_t parts = 2 * ((d + 255) / 256);
    p.xb1 = off;
    off += al256(2 * d * S);
    p.ss1 = off;
    off += al256(S * parts * 4);
    p.ss2 = off;
    off += al256(S * parts * 4);
    p.r1 = off;
    off += al256(S * 4);
    p.r2 = off;
    off += al256(S * 4);
  }
  p.total = off;
  return p;
}

int check_weights(const h3b_block_weights* w, int dtype) {
  if (!w) return H3B_ERR_NULL;
  if (w->dtype != dtype) return H3B_ERR_DTYPE;
  if (!w->w_qkv || !w->w_o || !w->w_fc1 || !w->w_fc2 || !w->g_attn || !w->g_mlp) return H3B_ERR_NULL;
  if (!aligned16(w->w_qkv) || !aligned16(w->w_o) || !aligned16(w->w_fc1) || !aligned16(w->w_fc2) ||
      !aligned16(w->g_attn) || !aligned16(w->g_mlp))
    return H3B_ERR_ALIGN;
  if (dtype == H3B_INT8) {
    if (!w->s_qkv || !w->s_o || !w->s_fc1 || !w->s_fc2) return H3B_ERR_NULL;
    if (!aligned16(w->s_qkv) || !aligned16(w->s_o) || !aligned16(w->s_fc1) || !aligned16(w->s_fc2))
      return H3B_ERR_ALIGN;
  }
  return H3B_OK;
}

#define H3B_TRY(expr)                 \
  do {                                \
    const int _st = (expr);           \
    if (_st != H3B_OK) return _st;    \
  } while (0)
#define H3B_CU(kid, expr)                                    \
  do {                                                       \
    TraceScope _ts((kid), c.stream);                         \
    if ((expr) != cudaSuccess) return H3B_ERR_CUDA;          \
  } while (0)

int norm_parts(const h3b_dims& dm) { return 2 * ((dm.d + 255) / 256); }

GemmArgs gemm_args(int M, int N, int K, void* C, const float* sa, const float* sb, const float* rope,
                   const h3b_dims& dm, float* amax, int* err) {
  GemmArgs a;
  a.M = M;
  a.N = N;
  a.K = K;
  a.C = C;
  a.sa = sa;
  a.sb = sb;
  a.rope = reinterpret_cast<const float2*>(rope);
  a.d = dm.d;
  a.head_dim = dm.head_dim;
  a.row_absmax = amax;
  a.err = err;
  a.full_tiles = 0;
  a.split = 1;
  a.partial = nullptr;
  a.gate = nullptr;
  a.gate_split = 0;
  a.gate_stride = 0;
  a.rope_rows = M;
  a.group_n = 1;
  a.xb = nullptr;
  a.xb_gain = nullptr;
  a.ss_out = nullptr;
  a.ss_parts = norm_parts(dm);
  a.row_scale = nullptr;
  a.partial_elems = 0;
  return a;
}

// Folded RMSNorm (bf16 blocks without modulation): the residual GEMM before
// a norm writes bf16(x * g) and per-row partial sums of x^2; the GEMM after
// it reads that copy and scales each row by 1 / sqrt(mean x^2 + eps).
GemmArgs norm_out(GemmArgs a, __nv_bfloat16* xb, const float* gain, float* ss) {
  a.xb = xb;
  a.xb_gain = gain;
  a.ss_out = ss;
  return a;
}
GemmArgs norm_in(GemmArgs a, const float* r) {
  a.row_scale = r;
  return a;
}

GemmArgs gated(GemmArgs a, const float* gate, int split, int stride) {
  a.gate = gate;
  a.gate_split = split;
  a.gate_stride = stride;
  return a;
}

// One block on x [S_eff + n_cond, d]; rope = table of this geometry (already
// filled).  mod (nullable): this block's modulation [2][6][d] fp32 -- row class
// (generated, condition) x (shift, scale, gate of the attention half, then of
// the MLP half).
// Folded norms (bf16, no modulation): norm_in -- the previous block's FC2
// left bf16(x * g_attn) in xb1 and the row sums in ss1, so RMSNorm1 is folded
// into this block's QKV GEMM; next_gain (nullable) -- this block's FC2 leaves
// the same for the next block, whose g_attn it is.  RMSNorm2 is folded into
// the O-proj / FC1 pair inside every such block.
int block_impl(const Ctx& c, const h3b_dims& dm, const h3b_block_weights& w, float* x, int merged, uint8_t* ws,
               const Plan& p, const float* rope, const float* mod = nullptr, bool norm_in_ready = false,
               const float* next_gain = nullptr) {
  const int Sg = seq_len(dm, merged), S = Sg + p.n_cond, d = dm.d, f = dm.ffn;
  Mod m1, m2;
  const float *gate1 = nullptr, *gate2 = nullptr;
  if (mod) {
    m1 = Mod{mod, mod + d, Sg, 6 * d};
    m2 = Mod{mod + 3 * d, mod + 4 * d, Sg, 6 * d};
    gate1 = mod + 2 * d;
    gate2 = mod + 5 * d;
  }
  GemmArgs qkv_args = gemm_args(S, 3 * d, d, nullptr, nullptr, nullptr, rope, dm, nullptr, c.err);
  qkv_args.rope_rows = Sg;
  uint8_t* A = ws;
  void* qkv = A + p.qkv;
  void* o = A + p.o;
  void* u1 = A + p.u1;
  void* u2 = A + p.u2;
  void* g = A + p.g;
  float* s_act = reinterpret_cast<float*>(ws + p.s_act);
  if (w.dtype == H3B_BF16) {
    const bool fold = !mod;  // the modulated norm is not a per-row scale
    float* ss1 = reinterpret_cast<float*>(ws + p.ss1);
    float* ss2 = reinterpret_cast<float*>(ws + p.ss2);
    __nv_bfloat16* xb1 = reinterpret_cast<__nv_bfloat16*>(ws + p.xb1);
    qkv_args.C = qkv;
    float* r1 = reinterpret_cast<float*>(ws + p.r1);
    float* r2 = reinterpret_cast<float*>(ws + p.r2);
    if (fold && norm_in_ready) {
      H3B_CU(KID_NORM_SCALE, launch_norm_scale(c, ss1, S, norm_parts(dm), d, dm.eps, r1));
      H3B_CU(KID_GEMM_QKV, launch_gemm(c, xb1, w.w_qkv, 0, H3B_EPI_QKV_ROPE, norm_in(qkv_args, r1)));
    } else {
      H3B_CU(KID_RMSNORM, launch_rmsnorm(c, x, w.g_attn, S, d, dm.eps, u1, nullptr, 0, m1));
      H3B_CU(KID_GEMM_QKV, launch_gemm(c, u1, w.w_qkv, 0, H3B_EPI_QKV_ROPE, qkv_args));
    }
    // the norm-1 arena is dead once the QKV GEMM has run: key-split attention partials
    H3B_CU(KID_ATTN, launch_attention(c, qkv, S, dm.n_heads, dm.head_dim, o, reinterpret_cast<float*>(u1),
                                      2 * static_cast<size_t>(d) * S));
    // O-proj: split-K partials in the dead QKV arena past the MLP-input slot,
    // where the folded norm writes bf16(x1 * g_mlp) for FC1
    GemmArgs o_args =
        gated(gemm_args(S, d, d, x, nullptr, nullptr, nullptr, dm, nullptr, c.err), gate1, Sg, 6 * d);
    if (fold) o_args = norm_out(o_args, reinterpret_cast<__nv_bfloat16*>(u2), w.g_mlp, ss2);
    const size_t o_part = p.u2 + al256(2 * static_cast<size_t>(d) * S);
    H3B_CU(KID_GEMM_O, launch_gemm(c, o, w.w_o, 0, H3B_EPI_RESID, o_args, reinterpret_cast<float*>(A + o_part),
                                   p.o - o_part));
    if (fold)
      H3B_CU(KID_NORM_SCALE, launch_norm_scale(c, ss2, S, norm_parts(dm), d, dm.eps, r2));
    else
      H3B_CU(KID_RMSNORM, launch_rmsnorm(c, x, w.g_mlp, S, d, dm.eps, u2, nullptr, 0, m2));
    GemmArgs fc1_args = gemm_args(S, f, d, g, nullptr, nullptr, nullptr, dm, nullptr, c.err);
    H3B_CU(KID_GEMM_FC1, launch_gemm(c, u2, w.w_fc1, 0, H3B_EPI_GELU, fold ? norm_in(fc1_args, r2) : fc1_args));
    // FC2: split-K partials in the dead MLP-input slot
    GemmArgs fc2_args =
        gated(gemm_args(S, d, f, x, nullptr, nullptr, nullptr, dm, nullptr, c.err), gate2, Sg, 6 * d);
    if (fold && next_gain) fc2_args = norm_out(fc2_args, xb1, next_gain, ss1);
    H3B_CU(KID_GEMM_FC2, launch_gemm(c, g, w.w_fc2, 0, H3B_EPI_RESID, fc2_args, reinterpret_cast<float*>(A + p.u2),
                                     p.g - p.u2));
  } else {
    int8_t* oq = reinterpret_cast<int8_t*>(A + p.oq);
    int8_t* gq = reinterpret_cast<int8_t*>(A + p.gq);
    float* s_g = reinterpret_cast<float*>(ws + p.s_g);
    float* amax = reinterpret_cast<float*>(ws + p.amax);
    H3B_CU(KID_RMSNORM, launch_rmsnorm(c, x, w.g_attn, S, d, dm.eps, u1, s_act, 1, m1));
    qkv_args.C = qkv;
    qkv_args.sa = s_act;
    qkv_args.sb = w.s_qkv;
    H3B_CU(KID_GEMM_QKV, launch_gemm(c, u1, w.w_qkv, 1, H3B_EPI_QKV_ROPE, qkv_args));
    H3B_CU(KID_ATTN, launch_attention(c, qkv, S, dm.n_heads, dm.head_dim, o, reinterpret_cast<float*>(u1),
                                      static_cast<size_t>(d) * S));
    H3B_CU(KID_QUANT_ROWS, launch_quant_rows(c, o, S, d, oq, s_act));
    H3B_CU(KID_GEMM_O, launch_gemm(c, oq, w.w_o, 1, H3B_EPI_RESID,
                                   gated(gemm_args(S, d, d, x, s_act, w.s_o, nullptr, dm, nullptr, c.err), gate1, Sg,
                                         6 * d),
                                   reinterpret_cast<float*>(A + p.qkv), p.o - p.qkv));
    H3B_CU(KID_RMSNORM, launch_rmsnorm(c, x, w.g_mlp, S, d, dm.eps, u2, s_act, 1, m2));
    H3B_CU(KID_MEMSET, cudaMemsetAsync(amax, 0, sizeof(float) * S, c.stream));
    H3B_CU(KID_GEMM_FC1, launch_gemm(c, u2, w.w_fc1, 1, H3B_EPI_GELU,
                                     gemm_args(S, f, d, g, s_act, w.s_fc1, nullptr, dm, amax, c.err)));
    H3B_CU(KID_QUANT_ABSMAX, launch_quant_absmax(c, g, amax, S, f, gq, s_g));
    H3B_CU(KID_GEMM_FC2, launch_gemm(c, gq, w.w_fc2, 1, H3B_EPI_RESID,
                                     gated(gemm_args(S, d, f, x, s_g, w.s_fc2, nullptr, dm, nullptr, c.err), gate2,
                                           Sg, 6 * d),
                                     reinterpret_cast<float*>(A + p.u2), p.g - p.u2));
  }
  return H3B_OK;
}

int fill_rope(const Ctx& c, const h3b_dims& dm, uint8_t* ws, const Plan& p, int reduction) {
  H3B_CU(KID_ROPE_TABLE, launch_rope_table(c, dm, 0, reinterpret_cast<float*>(ws + p.rope)));
  if (reduction) H3B_CU(KID_ROPE_TABLE, launch_rope_table(c, dm, 1, reinterpret_cast<float*>(ws + p.rope_m)));
  return H3B_OK;
}

// Blocks lo..hi on x; the token-reduction window [mf, ml] is applied when it
// lies inside [lo, hi] (merge before mf, unmerge after ml; udelta selects the
// delta-broadcast unmerge).  RoPE tables must be filled.
// mod (nullable): [n_blocks][2][6][d] for blocks 0.. of the whole stack.
int run_blocks(const Ctx& c, const h3b_dims& dm, const h3b_block_weights* blocks, int lo, int hi, int mf, int ml,
               int udelta, float* x, uint8_t* ws, const Plan& p, const float* mod = nullptr) {
  const bool on = mf >= 0 && lo <= mf && ml <= hi;
  float* rope = reinterpret_cast<float*>(ws + p.rope);
  float* rope_m = on ? reinterpret_cast<float*>(ws + p.rope_m) : nullptr;
  float* xm = on ? reinterpret_cast<float*>(ws + p.xm) : nullptr;
  float* xm0 = on && udelta ? reinterpret_cast<float*>(ws + p.xm0) : nullptr;
  const int V = dm.frames * dm.rows * dm.cols;
  const int tail = dm.n_audio + p.n_cond;  // rows after the video rows, carried through the reduction
  bool folded = false;  // block l-1's FC2 left block l's folded norm-1 input
  for (int l = lo; l <= hi; ++l) {
    if (on && l == mf) H3B_CU(KID_MERGE, launch_merge(c, x, xm, V, tail, dm.d, xm0));
    const bool merged = on && l >= mf && l <= ml;
    // the chain of folded norms runs between unmodulated bf16 blocks on the
    // same token grid (a merge or unmerge between two blocks breaks it)
    const bool chain = !mod && l < hi && blocks[l].dtype == H3B_BF16 && blocks[l + 1].dtype == H3B_BF16 &&
                       !(on && (l == ml || l + 1 == mf));
    H3B_TRY(block_impl(c, dm, blocks[l], merged ? xm : x, merged, ws, p, merged ? rope_m : rope,
                       mod ? mod + static_cast<size_t>(l) * 12 * dm.d : nullptr, folded,
                       chain ? blocks[l + 1].g_attn : nullptr));
    folded = chain;
    if (on && l == ml) {
      if (udelta)
        H3B_CU(KID_UNMERGE_DELTA, launch_unmerge_delta(c, x, xm, xm0, V, tail, dm.d));
      else
        H3B_CU(KID_UNMERGE, launch_unmerge(c, xm, x, V, tail, dm.d));
    }
  }
  return H3B_OK;
}

int stack_impl(const Ctx& c, const h3b_dims& dm, const h3b_block_weights* blocks, int n_blocks, int mf, int ml,
               float* x, uint8_t* ws, const Plan& p, int udelta = 0, const float* mod = nullptr) {
  H3B_TRY(fill_rope(c, dm, ws, p, mf >= 0));
  return run_blocks(c, dm, blocks, 0, n_blocks - 1, mf, ml, udelta, x, ws, p, mod);
}

int check_stack_args(const h3b_dims* dims, const h3b_block_weights* blocks, int n_blocks, int mf, int ml, float* x,
                     void* ws, size_t ws_bytes, Plan* out, int udelta = 0, int cf = -1, int cl = -1, int n_cond = 0) {
  H3B_TRY(check_dims(dims));
  if (n_cond < 0 || seq_len(*dims, 0) + static_cast<long long>(n_cond) > (1LL << 24)) return H3B_ERR_DIMS;
  if (!blocks || !x || !ws) return H3B_ERR_NULL;
  if (!aligned16(x) || !aligned16(ws)) return H3B_ERR_ALIGN;
  if (n_blocks < 0) return H3B_ERR_DIMS;
  if (mf >= 0) {
    if (ml < mf || ml >= n_blocks || (dims->cols & 1)) return H3B_ERR_DIMS;
  }
  const int dtype = n_blocks > 0 ? blocks[0].dtype : H3B_BF16;
  if (dtype != H3B_BF16 && dtype != H3B_INT8) return H3B_ERR_DTYPE;
  for (int l = 0; l < n_blocks; ++l) H3B_TRY(check_weights(&blocks[l], dtype));
  if (cf >= 0) {
    if (cl < cf || cl >= n_blocks) return H3B_ERR_DIMS;
    // the reduction window lies inside the core window or outside it
    if (mf >= 0 && !(cf <= mf && ml <= cl) && !(ml < cf || mf > cl)) return H3B_ERR_DIMS;
  }
  *out = plan(*dims, dtype, mf >= 0, mf >= 0 && udelta, cf >= 0, n_cond);
  if (ws_bytes < out->total) return H3B_ERR_WORKSPACE;
  return H3B_OK;
}

// Flow-matching loop.  Whole-velocity reuse: the stack runs on steps with
// i % reuse == 0 or the last one.  Core reuse (cf >= 0, reuse == 1): the core
// blocks run on steps with i % core_reuse == 0 or the last one; their update
// is cached (as its negative, in ws at p.delta) and added on the other steps.
// Condition rows (p.n_cond): v holds [generated ; condition] rows; every
// evaluation refills the condition rows from cond, the Euler update covers
// the generated rows only.  mod: [mod_steps][n_blocks][2][6][d] or NULL.
int denoise_impl(const Ctx& c, const h3b_dims& dm, const h3b_block_weights* blocks, int n_blocks, int mf, int ml,
                 int udelta, int cf, int cl, int n_steps, int reuse, int core_reuse, float* x, float* v, uint8_t* ws,
                 const Plan& p, int* n_fresh, int* n_core, const float* cond = nullptr, const float* mod = nullptr,
                 int mod_steps = 1) {
  const size_t n = static_cast<size_t>(seq_len(dm, 0)) * dm.d;    // generated rows
  const size_t n_all = n + static_cast<size_t>(p.n_cond) * dm.d;  // + condition rows
  auto fresh = [&](int i, int r) { return i % r == 0 || i == n_steps - 1; };
  float* neg_delta = cf >= 0 ? reinterpret_cast<float*>(ws + p.delta) : nullptr;
  const size_t mod_step = static_cast<size_t>(n_blocks) * 12 * dm.d;
  int count = 0, core_count = 0;
  H3B_TRY(fill_rope(c, dm, ws, p, mf >= 0));
  H3B_CU(KID_COPY, cudaMemcpyAsync(v, x, n * sizeof(float), cudaMemcpyDeviceToDevice, c.stream));
  for (int i = 0; i < n_steps; ++i) {
    const float* m = mod ? mod + (mod_steps > 1 ? static_cast<size_t>(i) * mod_step : 0) : nullptr;
    if (fresh(i, reuse)) {
      if (p.n_cond)
        H3B_CU(KID_COPY,
               cudaMemcpyAsync(v + n, cond, (n_all - n) * sizeof(float), cudaMemcpyDeviceToDevice, c.stream));
      if (cf < 0) {
        H3B_TRY(run_blocks(c, dm, blocks, 0, n_blocks - 1, mf, ml, udelta, v, ws, p, m));
      } else {
        H3B_TRY(run_blocks(c, dm, blocks, 0, cf - 1, mf, ml, udelta, v, ws, p, m));
        if (fresh(i, core_reuse)) {
          H3B_CU(KID_COPY, cudaMemcpyAsync(neg_delta, v, n_all * sizeof(float), cudaMemcpyDeviceToDevice, c.stream));
          H3B_TRY(run_blocks(c, dm, blocks, cf, cl, mf, ml, udelta, v, ws, p, m));
          H3B_CU(KID_FLOW, launch_flow_step(c, neg_delta, v, -1.0f, n_all, nullptr));  // input - output
          ++core_count;
        } else {
          H3B_CU(KID_FLOW, launch_flow_step(c, v, neg_delta, -1.0f, n_all, nullptr));  // + cached update
        }
        H3B_TRY(run_blocks(c, dm, blocks, cl + 1, n_blocks - 1, mf, ml, udelta, v, ws, p, m));
      }
      ++count;
    }
    const float s0 = static_cast<float>(1.0 - static_cast<double>(i) / n_steps);
    const float s1 = static_cast<float>(1.0 - static_cast<double>(i + 1) / n_steps);
    const bool next_fresh = i + 1 < n_steps && fresh(i + 1, reuse);
    H3B_CU(KID_FLOW, launch_flow_step(c, x, v, s1 - s0, n, next_fresh ? v : nullptr));
  }
  if (n_fresh) *n_fresh = count;
  if (n_core) *n_core = core_count;
  return H3B_OK;
}

}  // namespace

// ------------------------------------------------------------------ tensor maps
bool encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, int elem_bytes, const void* base, uint64_t inner,
                    uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer) {
  typedef CUresult (*EncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                               const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                               CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
  static EncodeFn fn = nullptr;
  if (!fn) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!fn) {
      void* p = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !p)
        return false;
      fn = reinterpret_cast<EncodeFn>(p);
    }
  }
  (void)elem_bytes;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace h3b

using namespace h3b;

// Options of the extended entry points: the condition-row count and the
// modulation array (16-byte aligned; mod_steps >= 1 slices of [n_blocks][2][6][d]).
static int check_opts(const h3b_stack_opts* o) {
  if (!o) return H3B_ERR_NULL;
  if (o->n_cond < 0) return H3B_ERR_DIMS;
  if (o->modulation) {
    if (!aligned16(o->modulation)) return H3B_ERR_ALIGN;
    if (o->mod_steps < 1) return H3B_ERR_DIMS;
  }
  return H3B_OK;
}

// ====================================================================== C ABI
extern "C" {

const char* h3b_status_string(int s) {
  switch (s) {
    case H3B_OK: return "ok";
    case H3B_ERR_NULL: return "a required pointer is NULL";
    case H3B_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case H3B_ERR_DIMS: return "unsupported or inconsistent sizes";
    case H3B_ERR_DTYPE: return "unknown dtype or epilogue";
    case H3B_ERR_WORKSPACE: return "workspace smaller than required";
    case H3B_ERR_CUDA: return "a CUDA call failed";
    case H3B_ERR_DEVICE: return "no usable sm_100 device";
    case H3B_ERR_TIMEOUT: return "a bounded device-side wait gave up";
    default: return "unknown status";
  }
}

int h3b_seq_len(const h3b_dims* dims, int merged) {
  if (check_dims(dims) != H3B_OK) return -1;
  if (merged && (dims->cols & 1)) return -1;
  return seq_len(*dims, merged);
}

size_t h3b_workspace_bytes(const h3b_dims* dims, int dtype, int token_reduction) {
  if (check_dims(dims) != H3B_OK || (dtype != H3B_BF16 && dtype != H3B_INT8)) return 0;
  if (token_reduction && (dims->cols & 1)) return 0;
  return plan(*dims, dtype, token_reduction != 0).total;
}

size_t h3b_workspace_saved_bytes(const h3b_dims* dims, int dtype) {
  if (check_dims(dims) != H3B_OK || (dtype != H3B_BF16 && dtype != H3B_INT8)) return 0;
  const Plan p = plan(*dims, dtype, 0);
  return p.naive - p.arena;
}

int h3b_block_forward(const h3b_dims* dims, const h3b_block_weights* w, float* x, int merged, void* ws,
                      size_t ws_bytes, void* stream) {
  H3B_TRY(check_dims(dims));
  if (!w || !x || !ws) return H3B_ERR_NULL;
  if (!aligned16(x) || !aligned16(ws)) return H3B_ERR_ALIGN;
  if (merged && (dims->cols & 1)) return H3B_ERR_DIMS;
  if (w->dtype != H3B_BF16 && w->dtype != H3B_INT8) return H3B_ERR_DTYPE;
  H3B_TRY(check_weights(w, w->dtype));
  const Plan p = plan(*dims, w->dtype, 0);
  if (ws_bytes < p.total) return H3B_ERR_WORKSPACE;
  Ctx c;
  H3B_TRY(device_ctx(static_cast<cudaStream_t>(stream), &c));
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  float* rope = reinterpret_cast<float*>(wsb + p.rope);
  H3B_CU(KID_ROPE_TABLE, launch_rope_table(c, *dims, merged, rope));
  return block_impl(c, *dims, *w, x, merged, wsb, p, rope);
}

int h3b_stack_forward(const h3b_dims* dims, const h3b_block_weights* blocks, int n_blocks, int merge_first,
                      int merge_last, float* x, void* ws, size_t ws_bytes, void* stream) {
  Plan p;
  H3B_TRY(check_stack_args(dims, blocks, n_blocks, merge_first, merge_last, x, ws, ws_bytes, &p));
  Ctx c;
  H3B_TRY(device_ctx(static_cast<cudaStream_t>(stream), &c));
  return stack_impl(c, *dims, blocks, n_blocks, merge_first, merge_last, x, static_cast<uint8_t*>(ws), p);
}

int h3b_denoise(const h3b_dims* dims, const h3b_block_weights* blocks, int n_blocks, int merge_first,
                int merge_last, int n_steps, int reuse, float* x, float* v, void* ws, size_t ws_bytes, int* n_fresh,
                void* stream) {
  Plan p;
  H3B_TRY(check_stack_args(dims, blocks, n_blocks, merge_first, merge_last, x, ws, ws_bytes, &p));
  if (!v) return H3B_ERR_NULL;
  if (!aligned16(v)) return H3B_ERR_ALIGN;
  if (n_steps <= 0 || reuse <= 0) return H3B_ERR_DIMS;
  Ctx c;
  H3B_TRY(device_ctx(static_cast<cudaStream_t>(stream), &c));
  return denoise_impl(c, *dims, blocks, n_blocks, merge_first, merge_last, 0, -1, -1, n_steps, reuse, 1, x, v,
                      static_cast<uint8_t*>(ws), p, n_fresh, nullptr);
}

size_t h3b_workspace_bytes_ex(const h3b_dims* dims, int dtype, const h3b_stack_opts* o) {
  if (!o || check_dims(dims) != H3B_OK || (dtype != H3B_BF16 && dtype != H3B_INT8)) return 0;
  if (check_opts(o) != H3B_OK) return 0;
  const int red = o->merge_first >= 0;
  if (red && (dims->cols & 1)) return 0;
  return plan(*dims, dtype, red, red && o->unmerge_delta, o->core_first >= 0, o->n_cond).total;
}

int h3b_stack_forward_ex(const h3b_dims* dims, const h3b_block_weights* blocks, int n_blocks,
                         const h3b_stack_opts* o, float* x, void* ws, size_t ws_bytes, void* stream) {
  if (!o) return H3B_ERR_NULL;
  H3B_TRY(check_opts(o));
  Plan p;
  H3B_TRY(check_stack_args(dims, blocks, n_blocks, o->merge_first, o->merge_last, x, ws, ws_bytes, &p,
                           o->unmerge_delta, -1, -1, o->n_cond));
  Ctx c;
  H3B_TRY(device_ctx(static_cast<cudaStream_t>(stream), &c));
  return stack_impl(c, *dims, blocks, n_blocks, o->merge_first, o->merge_last, x, static_cast<uint8_t*>(ws), p,
                    o->unmerge_delta, o->modulation);
}

int h3b_denoise_ex(const h3b_dims* dims, const h3b_block_weights* blocks, int n_blocks, const h3b_stack_opts* o,
                   int n_steps, int reuse, int core_reuse, float* x, float* v, void* ws, size_t ws_bytes,
                   int* n_fresh, int* n_core_fresh, void* stream) {
  if (!o) return H3B_ERR_NULL;
  H3B_TRY(check_opts(o));
  Plan p;
  H3B_TRY(check_stack_args(dims, blocks, n_blocks, o->merge_first, o->merge_last, x, ws, ws_bytes, &p,
                           o->unmerge_delta, o->core_first, o->core_last, o->n_cond));
  if (!v) return H3B_ERR_NULL;
  if (!aligned16(v)) return H3B_ERR_ALIGN;
  if (n_steps <= 0 || reuse <= 0 || core_reuse <= 0) return H3B_ERR_DIMS;
  if (o->core_first >= 0 && reuse != 1) return H3B_ERR_DIMS;  // core reuse excludes whole-velocity reuse
  if (o->modulation && o->mod_steps != 1 && o->mod_steps != n_steps) return H3B_ERR_DIMS;
  if (o->n_cond > 0) {
    if (!o->cond_rows) return H3B_ERR_NULL;
    if (!aligned16(o->cond_rows)) return H3B_ERR_ALIGN;
  }
  Ctx c;
  H3B_TRY(device_ctx(static_cast<cudaStream_t>(stream), &c));
  return denoise_impl(c, *dims, blocks, n_blocks, o->merge_first, o->merge_last, o->unmerge_delta, o->core_first,
                      o->core_last, n_steps, reuse, core_reuse, x, v, static_cast<uint8_t*>(ws), p, n_fresh,
                      n_core_fresh, o->cond_rows, o->modulation, o->modulation ? o->mod_steps : 1);
}

int h3b_quantize_weights(const void* w, int rows, int k, int8_t* q, float* scale, void* stream) {
  if (rows != 0 && (!w || !q || !scale)) return H3B_ERR_NULL;
  if (!aligned16(w) || !aligned16(q) || !aligned16(scale)) return H3B_ERR_ALIGN;
  if (rows < 0 || k <= 0 || k % 8 != 0 || k > 32768) return H3B_ERR_DIMS;
  if (rows == 0) return H3B_OK;
  Ctx c;
  H3B_TRY(device_ctx(static_cast<cudaStream_t>(stream), &c));
  H3B_CU(KID_QUANT_ROWS, launch_quant_rows(c, w, rows, k, q, scale));
  return H3B_OK;
}

int h3b_quantize_rows_absmax(const void* a, const float* absmax, int rows, int k, int8_t* q, float* scale,
                             void* stream) {
  if (rows != 0 && (!a || !absmax || !q || !scale)) return H3B_ERR_NULL;
  if (!aligned16(a) || !aligned16(q) || !aligned16(scale) || !aligned16(absmax)) return H3B_ERR_ALIGN;
  if (rows < 0 || k <= 0 || k % 8 != 0) return H3B_ERR_DIMS;
  if (rows == 0) return H3B_OK;
  Ctx c;
  H3B_TRY(device_ctx(static_cast<cudaStream_t>(stream), &c));
  H3B_CU(KID_QUANT_ABSMAX, launch_quant_absmax(c, a, absmax, rows, k, q, scale));
  return H3B_OK;
}

int h3b_token_merge(const h3b_dims* dims, const float* x, float* xm, void* stream) {
  H3B_TRY(check_dims(dims));
  if (!x || !xm) return H3B_ERR_NULL;
  if (!aligned16(x) || !aligned16(xm)) return H3B_ERR_ALIGN;
  if (dims->cols & 1) return H3B_ERR_DIMS;
  Ctx c;
  H3B_TRY(device_ctx(static_cast<cudaStream_t>(stream), &c));
  H3B_CU(KID_MERGE, launch_merge(c, x, xm, dims->frames * dims->rows * dims->cols, dims->n_audio, dims->d));
  return H3B_OK;
}

int h3b_token_unmerge(const h3b_dims* dims, const float* xm, float* x, void* stream) {
  H3B_TRY(check_dims(dims));
  if (!x || !xm) return H3B_ERR_NULL;
  if (!aligned16(x) || !aligned16(xm)) return H3B_ERR_ALIGN;
  if (dims->cols & 1) return H3B_ERR_DIMS;
  Ctx c;
  H3B_TRY(device_ctx(static_cast<cudaStream_t>(stream), &c));
  H3B_CU(KID_UNMERGE, launch_unmerge(c, xm, x, dims->frames * dims->rows * dims->cols, dims->n_audio, dims->d));
  return H3B_OK;
}

int h3b_token_unmerge_delta(const h3b_dims* dims, float* x, const float* ym, const float* xm0, void* stream) {
  H3B_TRY(check_dims(dims));
  if (!x || !ym || !xm0) return H3B_ERR_NULL;
  if (!aligned16(x) || !aligned16(ym) || !aligned16(xm0)) return H3B_ERR_ALIGN;
  if (dims->cols & 1) return H3B_ERR_DIMS;
  Ctx c;
  H3B_TRY(device_ctx(static_cast<cudaStream_t>(stream), &c));
  H3B_CU(KID_UNMERGE_DELTA,
         launch_unmerge_delta(c, x, ym, xm0, dims->frames * dims->rows * dims->cols, dims->n_audio, dims->d));
  return H3B_OK;
}

int h3b_flow_step(float* x, const float* v, float sigma_cur, float sigma_next, size_t n, float* x_copy,
                  void* stream) {
  if (n == 0) return H3B_OK;  // nothing to update; empty buffers may be NULL
  if (!x || !v) return H3B_ERR_NULL;
  if (!aligned16(x) || !aligned16(v) || (x_copy && !aligned16(x_copy))) return H3B_ERR_ALIGN;
  Ctx c;
  H3B_TRY(device_ctx(static_cast<cudaStream_t>(stream), &c));
  H3B_CU(KID_FLOW, launch_flow_step(c, x, v, sigma_next - sigma_cur, n, x_copy));
  return H3B_OK;
}

int h3b_rope_table(const h3b_dims* dims, int merged, float* table, void* stream) {
  H3B_TRY(check_dims(dims));
  if (!table) return H3B_ERR_NULL;
  if (!aligned16(table)) return H3B_ERR_ALIGN;
  if (merged && (dims->cols & 1)) return H3B_ERR_DIMS;
  Ctx c;
  H3B_TRY(device_ctx(static_cast<cudaStream_t>(stream), &c));
  H3B_CU(KID_ROPE_TABLE, launch_rope_table(c, *dims, merged, table));
  return H3B_OK;
}

int h3b_rmsnorm(const float* x, const float* g, int rows, int d, float eps, void* out, float* out_scale,
                int out_dtype, void* stream) {
  if (rows != 0 && (!x || !g || !out || (out_dtype == H3B_INT8 && !out_scale))) return H3B_ERR_NULL;
  if (!aligned16(x) || !aligned16(g) || !aligned16(out)) return H3B_ERR_ALIGN;
  if (out_dtype != H3B_BF16 && out_dtype != H3B_INT8) return H3B_ERR_DTYPE;
  if (rows < 0 || d <= 0 || d % 4 != 0 || d > 8192 || !(eps >= 0.f)) return H3B_ERR_DIMS;
  if (rows == 0) return H3B_OK;
  Ctx c;
  H3B_TRY(device_ctx(static_cast<cudaStream_t>(stream), &c));
  H3B_CU(KID_RMSNORM, launch_rmsnorm(c, x, g, rows, d, eps, out, out_scale, out_dtype == H3B_INT8));
  return H3B_OK;
}

int h3b_gemm(const void* A, const void* B, int M, int N, int K, int ab_dtype, int epilogue, void* C,
             const float* scale_a, const float* scale_b, const float* rope_table, const h3b_dims* dims,
             float* row_absmax, void* scratch, size_t scratch_bytes, void* stream) {
  if (M != 0 && (!A || !C)) return H3B_ERR_NULL;
  if (!B) return H3B_ERR_NULL;
  if (!aligned16(A) || !aligned16(B) || !aligned16(C)) return H3B_ERR_ALIGN;
  if (ab_dtype != H3B_BF16 && ab_dtype != H3B_INT8) return H3B_ERR_DTYPE;
  if (epilogue < H3B_EPI_F32 || epilogue > H3B_EPI_I32) return H3B_ERR_DTYPE;
  if (epilogue == H3B_EPI_I32 && ab_dtype != H3B_INT8) return H3B_ERR_DTYPE;
  if (M < 0 || N <= 0 || K <= 0 || N % 32 != 0 || K % (ab_dtype == H3B_INT8 ? 128 : 64) != 0) return H3B_ERR_DIMS;
  if (ab_dtype == H3B_INT8 && epilogue != H3B_EPI_I32) {
    if (!scale_a || !scale_b) return H3B_ERR_NULL;
    if (!aligned16(scale_b)) return H3B_ERR_ALIGN;
  }
  h3b_dims dm{};
  if (epilogue == H3B_EPI_QKV_ROPE) {
    H3B_TRY(check_dims(dims));
    if (!rope_table) return H3B_ERR_NULL;
    if (!aligned16(rope_table)) return H3B_ERR_ALIGN;
    if (N != 3 * dims->d) return H3B_ERR_DIMS;
    dm = *dims;
  }
  if (epilogue == H3B_EPI_GELU && ab_dtype == H3B_INT8 && !row_absmax) return H3B_ERR_NULL;
  if (M == 0) return H3B_OK;
  Ctx c;
  H3B_TRY(device_ctx(static_cast<cudaStream_t>(stream), &c));
  if (scratch && !aligned16(scratch)) return H3B_ERR_ALIGN;
  H3B_CU(KID_GEMM, launch_gemm(c, A, B, ab_dtype == H3B_INT8, epilogue,
                               gemm_args(M, N, K, C, scale_a, scale_b, rope_table, dm, row_absmax, c.err),
                               static_cast<float*>(scratch), scratch ? scratch_bytes : 0));
  return H3B_OK;
}

int h3b_attention(const void* qkv, int S, int n_heads, int head_dim, void* o, void* scratch, size_t scratch_bytes,
                  void* stream) {
  if (S != 0 && (!qkv || !o)) return H3B_ERR_NULL;
  if (!aligned16(qkv) || !aligned16(o) || (scratch && !aligned16(scratch))) return H3B_ERR_ALIGN;
  if (S < 0 || n_heads <= 0 || (head_dim != 64 && head_dim != 128)) return H3B_ERR_DIMS;
  if (S == 0) return H3B_OK;
  Ctx c;
  H3B_TRY(device_ctx(static_cast<cudaStream_t>(stream), &c));
  H3B_CU(KID_ATTN, launch_attention(c, qkv, S, n_heads, head_dim, o, static_cast<float*>(scratch),
                                    scratch ? scratch_bytes : 0));
  return H3B_OK;
}

int h3b_exp2_poly(const float* x, float* y, int n, void* stream) {
  if (n < 0) return H3B_ERR_DIMS;
  if (n == 0) return H3B_OK;
  if (!x || !y) return H3B_ERR_NULL;
  if (!aligned16(x) || !aligned16(y)) return H3B_ERR_ALIGN;
  Ctx c;
  H3B_TRY(device_ctx(static_cast<cudaStream_t>(stream), &c));
  H3B_CU(KID_ATTN, launch_exp2_poly(c, x, y, n));
  return H3B_OK;
}

int h3b_gelu(const float* x, float* y, size_t n, void* stream) {
  if (n == 0) return H3B_OK;
  if (!x || !y) return H3B_ERR_NULL;
  Ctx c;
  H3B_TRY(device_ctx(static_cast<cudaStream_t>(stream), &c));
  H3B_CU(KID_GELU, launch_gelu(c, x, y, n));
  return H3B_OK;
}

int h3b_selftest_wait_timeout(int timeout_us, void* stream) {
  if (timeout_us <= 0 || timeout_us > 1000000) return H3B_ERR_DIMS;
  Ctx c;
  H3B_TRY(device_ctx(static_cast<cudaStream_t>(stream), &c));
  H3B_CU(KID_MEMSET, launch_selftest_wait(c, 1000ull * static_cast<unsigned long long>(timeout_us)));
  return H3B_OK;
}

int h3b_selftest_index_check(long long i, long long n, void* stream) {
  if (n <= 0) return H3B_ERR_DIMS;
  Ctx c;
  H3B_TRY(device_ctx(static_cast<cudaStream_t>(stream), &c));
  H3B_CU(KID_MEMSET, launch_selftest_index(c, i, n));
  return H3B_OK;
}

int h3b_index_checked(void) { return H3B_CHECK; }

int h3b_device_error(void* stream) {
  Ctx c;
  H3B_TRY(device_ctx(static_cast<cudaStream_t>(stream), &c));
  int v = 0;
  if (cudaMemcpyAsync(&v, c.err, sizeof(int), cudaMemcpyDeviceToHost, c.stream) != cudaSuccess) return H3B_ERR_CUDA;
  if (cudaStreamSynchronize(c.stream) != cudaSuccess) return H3B_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyAsync(c.err, &zero, sizeof(int), cudaMemcpyHostToDevice, c.stream) != cudaSuccess ||
        cudaStreamSynchronize(c.stream) != cudaSuccess)
      return H3B_ERR_CUDA;
  }
  return v;
}

int h3b_trace_start(int capacity) {
  if (capacity < 0) return H3B_ERR_DIMS;
  std::lock_guard<std::mutex> lk(g_mu);
  if (static_cast<int>(g_trace.recs.size()) < capacity) {
    const size_t old = g_trace.recs.size();
    g_trace.recs.resize(capacity);
    for (size_t i = old; i < g_trace.recs.size(); ++i) {
      if (cudaEventCreate(&g_trace.recs[i].a) != cudaSuccess || cudaEventCreate(&g_trace.recs[i].b) != cudaSuccess) {
        g_trace.recs.resize(i);
        return H3B_ERR_CUDA;
      }
    }
  }
  g_trace.cap = capacity;
  g_trace.n = 0;
  g_trace.on = true;
  return H3B_OK;
}

int h3b_trace_stop(int* n_records) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_trace.on = false;
  g_trace.ms.assign(g_trace.n, 0.f);
  for (int i = 0; i < g_trace.n; ++i) {
    if (cudaEventSynchronize(g_trace.recs[i].b) != cudaSuccess) return H3B_ERR_CUDA;
    if (cudaEventElapsedTime(&g_trace.ms[i], g_trace.recs[i].a, g_trace.recs[i].b) != cudaSuccess)
      return H3B_ERR_CUDA;
  }
  if (n_records) *n_records = g_trace.n;
  return H3B_OK;
}

int h3b_trace_read(int* kernel_ids, float* ms, int max_records) {
  std::lock_guard<std::mutex> lk(g_mu);
  const int n = g_trace.n < max_records ? g_trace.n : max_records;
  for (int i = 0; i < n && i < static_cast<int>(g_trace.ms.size()); ++i) {
    if (kernel_ids) kernel_ids[i] = g_trace.recs[i].kid;
    if (ms) ms[i] = g_trace.ms[i];
  }
  return n;
}

const char* h3b_kernel_name(int kid) { return (kid >= 0 && kid < KID_COUNT) ? kKernelNames[kid] : "unknown"; }

}  // extern "C"
