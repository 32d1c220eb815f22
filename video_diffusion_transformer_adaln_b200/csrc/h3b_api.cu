// The C ABI of the h3b library (declared in include/h3b.h): argument
// validation, workspace planning, TMA descriptor encoding and the launch
// sequence of one gated-AdaLN DiT block forward.
//
// Method references (web pages on the h3.c / h3-metal engine):
//   "h3-metal: Apple Silicon을 위한 네이티브 MiniMax-H3 추론", sections
//     "Int8 양자화" (gated AdaLN with the activation quantizer fused ahead of
//     the int8 QKV and MLP projections), "Metal 4 및 TensorOps" (head-major
//     Q/K/V) and "속도 및 품질 트레이드오프" (Token Reduction, Active DiT Blocks).
//   "h3.c與MLX路線對比：MiniMax-H3在Apple Silicon上的兩種推理實現工程取捨",
//     section "性能上限" (AdaLN gating, RoPE and quantization folded into the
//     preceding kernels; activation memory reused by lifetime).
#include <algorithm>
#include <atomic>
#include <cstdlib>
#include <mutex>
#include <string>
#include <vector>

#include "h3b.h"
#include "h3b_common.cuh"
#include "h3b_internal.h"

// Device error word: kernels OR a nonzero code into it when a bounded wait
// runs out. Host code reaches it through its device address (per device).
__device__ unsigned int g_h3b_error_word;

// Test hook for the bounded waits: one thread waits, with the same bounded
// mbarrier wait every pipeline uses, on a phase that nothing completes, so the
// wait runs out after limit_ns, records ERR_WAIT_PROBE in the error word and
// returns. Result: 1 when the wait ran out, 0 if the phase completed.
__device__ int g_h3b_probe_result;

static __global__ void bounded_wait_probe_kernel(unsigned* err, unsigned long long limit_ns) {
  __shared__ __align__(8) unsigned long long bar;
  if (threadIdx.x != 0) return;
  const uint32_t b = h3b::smem_u32(&bar);
  h3b::mbar_init(b, 1);
  h3b::fence_barrier_init();
  const bool completed = h3b::mbar_wait(b, 0, err, h3b::ERR_WAIT_PROBE, limit_ns);
  g_h3b_probe_result = completed ? 0 : 1;
}

namespace h3b {
namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool init = false;
  bool arch_ok = false;
  int sms = 0;
  unsigned* err = nullptr;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;
thread_local std::string g_detail;

h3b_status cuda_fail(cudaError_t e, const char* where) {
  g_detail = std::string(where) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")";
  return H3B_ERR_CUDA;
}
h3b_status fail(h3b_status s, const std::string& why) {
  g_detail = why;
  return s;
}

// Per-device facts, read once: compute capability (10.0 required), SM count,
// and the device address of the error word.
h3b_status device_info(DeviceInfo** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(H3B_ERR_ARG, "device index out of range");
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& di = g_dev[dev];
  if (!di.init) {
    int major = 0, minor = 0, sms = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute");
    di.arch_ok = (major == 10 && minor == 0);
    di.sms = sms;
    if (di.arch_ok) {
      void* p = nullptr;
      if ((e = cudaGetSymbolAddress(&p, g_h3b_error_word)) != cudaSuccess)
        return cuda_fail(e, "cudaGetSymbolAddress(error word)");
      di.err = static_cast<unsigned*>(p);
    }
    di.init = true;
  }
  if (!di.arch_ok) return fail(H3B_ERR_ARCH, "device is not compute capability 10.0 (sm_100a)");
  *out = &di;
  return H3B_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Tokens of a T x H x W latent grid, or -1 when an extent is below 1 or the count
// reaches 2^31. The product is formed one factor at a time, each step below 2^62,
// so no extents a caller can pass make it overflow.
long long grid_tokens(long long T, long long H, long long W) {
  const long long lim = 1LL << 31;
  if (T < 1 || H < 1 || W < 1 || T >= lim || H >= lim || W >= lim) return -1;
  if (T * H >= lim) return -1;
  const long long L = T * H * W;
  return L >= lim ? -1 : L;
}

h3b_status check_dims(const h3b_dims* d) {
  if (!d) return fail(H3B_ERR_ARG, "dims is NULL");
  if (d->B < 1 || d->T < 1 || d->H < 1 || d->W < 1) return fail(H3B_ERR_SHAPE, "B, T, H, W must be >= 1");
  if (d->B > 8) return fail(H3B_ERR_SHAPE, "B must be <= 8");
  if (d->head_dim != 64 && d->head_dim != 128) return fail(H3B_ERR_SHAPE, "head_dim must be 64 or 128");
  if (d->n_heads < 1 || (long long)d->d != (long long)d->n_heads * d->head_dim)
    return fail(H3B_ERR_SHAPE, "d != n_heads * head_dim");
  if (d->d < 256 || d->d % 256 != 0 || d->d > 8192) return fail(H3B_ERR_SHAPE, "d must be a multiple of 256 in [256, 8192]");
  if (d->d_ff < 256 || d->d_ff % 256 != 0 || d->d_ff > 32768)
    return fail(H3B_ERR_SHAPE, "d_ff must be a multiple of 256 in [256, 32768]");
  if (d->rope_t < 0 || d->rope_h < 0 || d->rope_w < 0 || (d->rope_t | d->rope_h | d->rope_w) & 1 ||
      d->rope_t + d->rope_h + d->rope_w != d->head_dim)
    return fail(H3B_ERR_SHAPE, "rope split must be even parts summing to head_dim");
  if (!(d->rope_theta > 0.0f) || !(d->ln_eps >= 0.0f)) return fail(H3B_ERR_ARG, "rope_theta > 0 and ln_eps >= 0");
  const long long L = grid_tokens(d->T, d->H, d->W);
  if (L < 0 || L * d->B >= (1LL << 31)) return fail(H3B_ERR_SHAPE, "too many tokens");
  if (L * d->B * (long long)d->d_ff > (1LL << 40)) return fail(H3B_ERR_SHAPE, "problem too large");
  return H3B_OK;
}

struct WsLayout {
  size_t mod, rope, sA, absmax, act, r1, total;
};

size_t rope_bytes(const h3b_dims& d) {
  return sizeof(float2) * ((size_t)d.T * (d.rope_t / 2) + (size_t)d.H * (d.rope_h / 2) +
                           (size_t)d.W * (d.rope_w / 2));
}

WsLayout ws_layout(const h3b_dims& d) {
  WsLayout w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  const size_t R = (size_t)d.B * d.T * d.H * d.W;
  const size_t D = d.d, F = d.d_ff;
  w.mod = take((size_t)d.B * 6 * D * 4);
  w.rope = take(rope_bytes(d));
  w.sA = take(R * 4);
  w.absmax = take(R * 4);
  // int8 activations (A1..A4 in turn, up to R x F), or the bf16 QKV input.
  w.act = take(std::max(R * std::max(D, F), d.qkv_int8 ? (size_t)0 : R * D * 2));
  // Q/K/V + attention output, later reused for the GELU output.
  w.r1 = take(std::max(3 * R * D * 2 + R * D * 2, R * F * 2));
  w.total = off;
  return w;
}

h3b_status check_weights(const h3b_dims& d, const h3b_block_weights* w) {
  if (!w) return fail(H3B_ERR_ARG, "weights is NULL");
  const void* req[] = {w->w_ada, w->w1, w->s1, w->w2, w->s2};
  for (const void* p : req) {
    if (!p) return fail(H3B_ERR_ARG, "a required weight pointer is NULL");
    if (!aligned16(p)) return fail(H3B_ERR_ALIGN, "weight pointer not 16-byte aligned");
  }
  if (d.wo_bf16) {
    if (!w->wo_bf16) return fail(H3B_ERR_ARG, "wo_bf16 NULL");
    if (!aligned16(w->wo_bf16)) return fail(H3B_ERR_ALIGN, "wo_bf16 alignment");
  } else {
    if (!w->wo || !w->so) return fail(H3B_ERR_ARG, "wo/so NULL");
    if (!aligned16(w->wo) || !aligned16(w->so)) return fail(H3B_ERR_ALIGN, "wo/so alignment");
  }
  if (d.qkv_int8) {
    if (!w->wqkv || !w->sqkv) return fail(H3B_ERR_ARG, "wqkv/sqkv NULL");
    if (!aligned16(w->wqkv) || !aligned16(w->sqkv)) return fail(H3B_ERR_ALIGN, "wqkv/sqkv alignment");
  } else {
    if (!w->wqkv_bf16) return fail(H3B_ERR_ARG, "wqkv_bf16 NULL");
    if (!aligned16(w->wqkv_bf16)) return fail(H3B_ERR_ALIGN, "wqkv_bf16 alignment");
  }
  const void* opt[] = {w->b_ada, w->bqkv, w->bo, w->b1, w->b2};
  for (const void* p : opt)
    if (p && !aligned16(p)) return fail(H3B_ERR_ALIGN, "bias pointer not 16-byte aligned");
  return H3B_OK;
}

// ---------------------------------------------------------------------------
// Kernel-level timing (h3b_profile_*): event pairs around each launch.
// ---------------------------------------------------------------------------
struct ProfRec {
  const char* name;
  cudaEvent_t a, b;
};
std::mutex g_prof_mu;
std::atomic<bool> g_prof_on{false};  // read by every launch without the lock
std::vector<ProfRec> g_prof_recs;
std::vector<cudaEvent_t> g_prof_free;

}  // namespace

bool profiling_enabled() { return g_prof_on.load(); }

bool pdl_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("H3B_PDL");
    return !(v && v[0] == '0');
  }();
  return on;
}

namespace {

cudaEvent_t prof_event() {
  if (!g_prof_free.empty()) {
    cudaEvent_t e = g_prof_free.back();
    g_prof_free.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// Scoped bracket: records a start event now and an end event when the launch
// has been enqueued (only while profiling is on).
struct ProfScope {
  const char* name;
  cudaStream_t st;
  cudaEvent_t a = nullptr;
  ProfScope(const char* n, cudaStream_t s) : name(n), st(s) {
    if (!g_prof_on) return;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    a = prof_event();
    if (a) cudaEventRecord(a, st);
  }
  ~ProfScope() {
    if (!a) return;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    cudaEvent_t b = prof_event();
    if (!b) {
      g_prof_free.push_back(a);  // no end event: drop this launch's record, keep the event
      return;
    }
    cudaEventRecord(b, st);
    g_prof_recs.push_back({name, a, b});
  }
};

#define H3B_CK(call, where)                                 \
  do {                                                      \
    ProfScope prof_scope_(where, st);                       \
    cudaError_t e_ = (call);                                \
    if (e_ != cudaSuccess) return cuda_fail(e_, where);     \
  } while (0)

GemmArgs base_args(int M, int N, int K, unsigned* err) {
  GemmArgs a{};
  a.M = M;
  a.N = N;
  a.K = K;
  a.rows_per_item = M > 0 ? M : 1;
  a.err = err;
  return a;
}

// The block's launch sequence on one stream (workspace regions per ws_layout).
h3b_status run_block(const h3b_dims& d, const h3b_block_weights& w, const float* c, void* x,
                     uint8_t* ws, const WsLayout& lay, bool rope_ready, const DeviceInfo& di,
                     cudaStream_t st) {
  const int D = d.d, F = d.d_ff, L = d.T * d.H * d.W, R = d.B * L;
  float* mod = reinterpret_cast<float*>(ws + lay.mod);
  float2* rope = reinterpret_cast<float2*>(ws + lay.rope);
  float* sA = reinterpret_cast<float*>(ws + lay.sA);
  float* absmax = reinterpret_cast<float*>(ws + lay.absmax);
  int8_t* act = reinterpret_cast<int8_t*>(ws + lay.act);
  uint8_t* r1 = ws + lay.r1;
  void* qkv = r1;
  void* o = r1 + (size_t)3 * R * D * 2;
  void* g = r1;

  // a1: AdaLN modulation vectors (the same launch fills the RoPE table when needed)
  H3B_CK(launch_adaln_gemv(w.w_ada, w.b_ada, c, d.B, D, mod, rope_ready ? nullptr : rope, d.T, d.H, d.W,
                           d.rope_t, d.rope_h, d.rope_w, d.rope_theta, di.sms, st), "adaln_gemv");
  // a2: LN + modulation + quantization (or the bf16 activation for bf16 QKV)
  if (d.qkv_int8)
    H3B_CK(launch_ln_mod_quant(x, R, D, d.ln_eps, mod, mod + D, L, 6 * D, act, sA, nullptr, absmax, 1, di.err, di.sms, st), "ln_mod_quant");
  else
    H3B_CK(launch_ln_mod_quant(x, R, D, d.ln_eps, mod, mod + D, L, 6 * D, nullptr, nullptr, act, absmax, 0, di.err, di.sms, st), "ln_mod");
  // a3: QKV projection + 3D RoPE, head-major
  {
    GemmArgs a = base_args(R, 3 * D, D, di.err);
    a.sA = sA;
    a.sW = w.sqkv;
    a.bias = w.bqkv;
    a.out = qkv;
    a.B = d.B; a.L = L; a.T = d.T; a.H = d.H; a.W = d.W; a.d = D;
    a.n_heads = d.n_heads; a.head_dim = d.head_dim;
    a.rope_t = d.rope_t; a.rope_h = d.rope_h; a.rope_w = d.rope_w; a.rope = rope;
    H3B_CK(launch_gemm(d.qkv_int8 != 0, EPI_QKV, act, d.qkv_int8 ? (const void*)w.wqkv : w.wqkv_bf16, a, di.sms, st), "gemm_qkv");
  }
  // a4: attention; a5: quantize its output
  {
    AttnArgs a{d.B, L, d.n_heads, d.head_dim, qkv, o, absmax, di.err};
    H3B_CK(launch_attention(a, st), "attention");
  }
  // a6: output projection + gated residual (gate_attn = chunk 2): int8 on the quantized
  // attention output (a5), or bf16 directly on the bf16 attention output
  if (!d.wo_bf16) {
    H3B_CK(launch_quant_rows_bf16(o, R, D, absmax, act, sA, di.sms, st), "quant_o");
    GemmArgs a = base_args(R, D, D, di.err);
    a.sA = sA; a.sW = w.so; a.bias = w.bo; a.out = x;
    a.gate = mod + 2 * D; a.rows_per_item = L; a.gate_stride = 6 * D;
    H3B_CK(launch_gemm(true, EPI_RESID, act, w.wo, a, di.sms, st), "gemm_wo");
  } else {
    GemmArgs a = base_args(R, D, D, di.err);
    a.bias = w.bo; a.out = x;
    a.gate = mod + 2 * D; a.rows_per_item = L; a.gate_stride = 6 * D;
    H3B_CK(launch_gemm(false, EPI_RESID, o, w.wo_bf16, a, di.sms, st), "gemm_wo");
  }
  // a7: LN + modulation + quantization for the MLP (chunks 3, 4)
  H3B_CK(launch_ln_mod_quant(x, R, D, d.ln_eps, mod + 3 * D, mod + 4 * D, L, 6 * D, act, sA, nullptr, absmax, 1, di.err, di.sms, st), "ln_mod_quant_mlp");
  // a8: W1 + GELU (+ row absmax), then requantize
  {
    GemmArgs a = base_args(R, F, D, di.err);
    a.sA = sA; a.sW = w.s1; a.bias = w.b1; a.out = g; a.absmax = absmax;
    H3B_CK(launch_gemm(true, EPI_GELU, act, w.w1, a, di.sms, st), "gemm_w1");
  }
  H3B_CK(launch_quant_rows_bf16(g, R, F, absmax, act, sA, di.sms, st), "quant_g");
  // a9: W2 + gated residual (gate_mlp = chunk 5)
  {
    GemmArgs a = base_args(R, D, F, di.err);
    a.sA = sA; a.sW = w.s2; a.bias = w.b2; a.out = x;
    a.gate = mod + 5 * D; a.rows_per_item = L; a.gate_stride = 6 * D;
    H3B_CK(launch_gemm(true, EPI_RESID, act, w.w2, a, di.sms, st), "gemm_w2");
  }
  return H3B_OK;
}

}  // namespace

// ---------------------------------------------------------------------------
// TMA descriptors (driver entry point fetched through the runtime).
// ---------------------------------------------------------------------------
void set_error_detail(const std::string& why) { g_detail = why; }
int check_current_device() {
  DeviceInfo* di = nullptr;
  return device_info(&di);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool make_tmap_2d(CUtensorMap* map, const void* base, int elem_bytes, uint64_t cols, uint64_t rows,
                  uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows, int swizzle_bytes) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  CUtensorMapSwizzle sw;
  switch (swizzle_bytes) {
    case 128: sw = CU_TENSOR_MAP_SWIZZLE_128B; break;
    case 64: sw = CU_TENSOR_MAP_SWIZZLE_64B; break;
    case 32: sw = CU_TENSOR_MAP_SWIZZLE_32B; break;
    case 0: sw = CU_TENSOR_MAP_SWIZZLE_NONE; break;
    default: return false;
  }
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt = elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  return fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_3d(CUtensorMap* map, const void* base, int elem_bytes, uint64_t d0, uint64_t d1, uint64_t d2,
                  uint32_t box0, uint32_t box1) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {d0 * elem_bytes, d0 * d1 * elem_bytes};
  const cuuint32_t box[3] = {box0, box1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapDataType dt = elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  return fn(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace h3b

using namespace h3b;

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

const char* h3b_status_string(h3b_status s) {
  switch (s) {
    case H3B_OK: return "ok";
    case H3B_ERR_ARG: return "invalid argument";
    case H3B_ERR_SHAPE: return "unsupported shape";
    case H3B_ERR_ALIGN: return "pointer not 16-byte aligned";
    case H3B_ERR_WORKSPACE: return "workspace too small";
    case H3B_ERR_ARCH: return "device is not sm_100a (compute capability 10.0)";
    case H3B_ERR_CUDA: return "CUDA error";
    case H3B_ERR_DEVICE_CHECK: return "device error word set";
  }
  return "unknown status";
}

const char* h3b_last_error_detail(void) { return g_detail.c_str(); }

h3b_status h3b_workspace_size(const h3b_dims* dims, size_t* bytes) {
  h3b_status s = check_dims(dims);
  if (s != H3B_OK) return s;
  if (!bytes) return fail(H3B_ERR_ARG, "bytes is NULL");
  *bytes = ws_layout(*dims).total;
  return H3B_OK;
}

size_t h3b_rope_table_bytes(const h3b_dims* dims) {
  if (check_dims(dims) != H3B_OK) return 0;
  return rope_bytes(*dims);
}

// Host checks shared by the block entry points (no device query).
static h3b_status block_common(const h3b_dims* dims, const float* c, void* x, void* ws, size_t ws_bytes,
                               WsLayout* lay) {
  h3b_status s = check_dims(dims);
  if (s != H3B_OK) return s;
  if (!c || !x || !ws) return fail(H3B_ERR_ARG, "c, x and ws must be non-NULL");
  if (!aligned16(c) || !aligned16(x)) return fail(H3B_ERR_ALIGN, "c/x not 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return fail(H3B_ERR_ALIGN, "workspace not 256-byte aligned");
  *lay = ws_layout(*dims);
  if (ws_bytes < lay->total) return fail(H3B_ERR_WORKSPACE, "workspace smaller than h3b_workspace_size");
  return H3B_OK;
}

h3b_status h3b_block_forward(const h3b_dims* dims, const h3b_block_weights* w, const float* c, void* x,
                             void* ws, size_t ws_bytes, h3b_stream stream) {
  WsLayout lay;
  h3b_status s = block_common(dims, c, x, ws, ws_bytes, &lay);
  if (s != H3B_OK) return s;
  if ((s = check_weights(*dims, w)) != H3B_OK) return s;
  DeviceInfo* di = nullptr;
  if ((s = device_info(&di)) != H3B_OK) return s;
  return run_block(*dims, *w, c, x, static_cast<uint8_t*>(ws), lay, false, *di, stream);
}

h3b_status h3b_blocks_forward(const h3b_dims* dims, const h3b_block_weights* w, int n_blocks, const float* c,
                              void* x, void* ws, size_t ws_bytes, h3b_stream stream) {
  WsLayout lay;
  h3b_status s = block_common(dims, c, x, ws, ws_bytes, &lay);
  if (s != H3B_OK) return s;
  if (n_blocks < 0 || (n_blocks > 0 && !w)) return fail(H3B_ERR_ARG, "n_blocks < 0 or weights NULL");
  for (int i = 0; i < n_blocks; ++i)
    if ((s = check_weights(*dims, &w[i])) != H3B_OK) return s;
  DeviceInfo* di = nullptr;
  if ((s = device_info(&di)) != H3B_OK) return s;
  const size_t c_stride = (size_t)dims->B * dims->d;
  for (int i = 0; i < n_blocks; ++i) {
    s = run_block(*dims, w[i], c + i * c_stride, x, static_cast<uint8_t*>(ws), lay, i > 0, *di, stream);
    if (s != H3B_OK) return s;
  }
  return H3B_OK;
}

h3b_status h3b_blocks_forward_cached(const h3b_dims* dims, const h3b_block_weights* w, int n_blocks, int first,
                                     int last, int fresh, const float* c, void* x, void* x_save, float* delta,
                                     void* ws, size_t ws_bytes, h3b_stream stream) {
  // host-only checks of the range arguments first, then the common block checks
  if (n_blocks < 0 || (n_blocks > 0 && !w)) return fail(H3B_ERR_ARG, "n_blocks < 0 or weights NULL");
  if (first < 0 || first > last || last > n_blocks) return fail(H3B_ERR_ARG, "need 0 <= first <= last <= n_blocks");
  const bool range = first < last;
  if (range && !delta) return fail(H3B_ERR_ARG, "delta NULL");
  if (range && fresh && !x_save) return fail(H3B_ERR_ARG, "x_save NULL");
  if ((range && !aligned16(delta)) || (range && fresh && !aligned16(x_save)))
    return fail(H3B_ERR_ALIGN, "delta / x_save not 16-byte aligned");
  WsLayout lay;
  h3b_status s = block_common(dims, c, x, ws, ws_bytes, &lay);
  if (s != H3B_OK) return s;
  for (int i = 0; i < n_blocks; ++i)
    if ((s = check_weights(*dims, &w[i])) != H3B_OK) return s;
  DeviceInfo* di = nullptr;
  if ((s = device_info(&di)) != H3B_OK) return s;
  cudaStream_t st = stream;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  const size_t c_stride = (size_t)dims->B * dims->d;
  const long long n = (long long)dims->B * dims->T * dims->H * dims->W * dims->d;
  bool rope_done = false;  // the first block that runs fills the RoPE table
  auto run = [&](int i) {
    const h3b_status r = run_block(*dims, w[i], c + i * c_stride, x, wsb, lay, rope_done, *di, st);
    rope_done = true;
    return r;
  };
  for (int i = 0; i < first; ++i)
    if ((s = run(i)) != H3B_OK) return s;
  if (range) {
    if (fresh) {
      const cudaError_t e = cudaMemcpyAsync(x_save, x, (size_t)n * 2, cudaMemcpyDeviceToDevice, st);
      if (e != cudaSuccess) return cuda_fail(e, "save range input");
      for (int i = first; i < last; ++i)
        if ((s = run(i)) != H3B_OK) return s;
      H3B_CK(launch_range_delta(x_save, x, delta, n, di->sms, st), "range_delta");
    } else {
      H3B_CK(launch_range_apply(x, delta, n, di->sms, st), "range_apply");
    }
  }
  for (int i = last; i < n_blocks; ++i)
    if ((s = run(i)) != H3B_OK) return s;
  return H3B_OK;
}

h3b_status h3b_range_delta(const void* before, const void* after, float* delta, long long n, h3b_stream stream) {
  cudaStream_t st = stream;
  if (n < 0 || n % 8 != 0) return fail(H3B_ERR_SHAPE, "n must be a non-negative multiple of 8");
  if (n == 0) return H3B_OK;  // empty problem: nothing to launch
  if (!before || !after || !delta) return fail(H3B_ERR_ARG, "NULL pointer");
  if (!aligned16(before) || !aligned16(after) || !aligned16(delta)) return fail(H3B_ERR_ALIGN, "alignment");
  DeviceInfo* di = nullptr;
  h3b_status s = device_info(&di);
  if (s != H3B_OK) return s;
  H3B_CK(launch_range_delta(before, after, delta, n, di->sms, st), "range_delta");
  return H3B_OK;
}

h3b_status h3b_range_apply(void* x, const float* delta, long long n, h3b_stream stream) {
  cudaStream_t st = stream;
  if (n < 0 || n % 8 != 0) return fail(H3B_ERR_SHAPE, "n must be a non-negative multiple of 8");
  if (n == 0) return H3B_OK;  // empty problem: nothing to launch
  if (!x || !delta) return fail(H3B_ERR_ARG, "NULL pointer");
  if (!aligned16(x) || !aligned16(delta)) return fail(H3B_ERR_ALIGN, "alignment");
  DeviceInfo* di = nullptr;
  h3b_status s = device_info(&di);
  if (s != H3B_OK) return s;
  H3B_CK(launch_range_apply(x, delta, n, di->sms, st), "range_apply");
  return H3B_OK;
}

h3b_status h3b_blocks_forward_reduced(const h3b_dims* full, const h3b_block_weights* w, int n_blocks,
                                      int first, int last, const float* c, void* x, void* xm, void* ym,
                                      void* ws, size_t ws_bytes, h3b_stream stream) {
  WsLayout lay_full;
  h3b_status s = block_common(full, c, x, ws, ws_bytes, &lay_full);
  if (s != H3B_OK) return s;
  if (n_blocks < 0 || (n_blocks > 0 && !w)) return fail(H3B_ERR_ARG, "n_blocks < 0 or weights NULL");
  if (first < 0 || first > last || last > n_blocks) return fail(H3B_ERR_ARG, "need 0 <= first <= last <= n_blocks");
  const bool reduced = first < last;
  h3b_dims merged = *full;
  WsLayout lay_merged = lay_full;
  if (reduced) {
    if (full->W % 2 != 0) return fail(H3B_ERR_SHAPE, "W must be even for token pairing");
    if (!ym) return fail(H3B_ERR_ARG, "ym must be non-NULL");
    if (!aligned16(ym)) return fail(H3B_ERR_ALIGN, "ym not 16-byte aligned");
    (void)xm;  // the merged input is recomputed from x by the unpairing
    merged.W = full->W / 2;
    if ((s = check_dims(&merged)) != H3B_OK) return s;
    lay_merged = ws_layout(merged);
  }
  for (int i = 0; i < n_blocks; ++i)
    if ((s = check_weights(*full, &w[i])) != H3B_OK) return s;
  DeviceInfo* di = nullptr;
  if ((s = device_info(&di)) != H3B_OK) return s;
  cudaStream_t st = stream;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  const size_t c_stride = (size_t)full->B * full->d;
  const long long lines = (long long)full->B * full->T * full->H;
  for (int i = 0; i < first; ++i)
    if ((s = run_block(*full, w[i], c + i * c_stride, x, wsb, lay_full, i > 0, *di, st)) != H3B_OK) return s;
  if (reduced) {
    H3B_CK(launch_token_pair(x, ym, nullptr, lines, full->W, full->d, di->sms, st), "token_pair");
    for (int i = first; i < last; ++i)
      if ((s = run_block(merged, w[i], c + i * c_stride, ym, wsb, lay_merged, i > first, *di, st)) != H3B_OK)
        return s;
    H3B_CK(launch_token_unpair(x, nullptr, ym, x, lines, full->W, full->d, di->sms, st), "token_unpair");
  }
  for (int i = last; i < n_blocks; ++i)
    if ((s = run_block(*full, w[i], c + i * c_stride, x, wsb, lay_full, i > last || (!reduced && i > 0), *di, st)) !=
        H3B_OK)
      return s;
  return H3B_OK;
}

static h3b_status check_pair_dims(const h3b_dims* full) {
  if (!full) return fail(H3B_ERR_ARG, "dims is NULL");
  if (full->B < 1 || full->T < 1 || full->H < 1 || full->W < 2) return fail(H3B_ERR_SHAPE, "bad grid");
  if (full->W % 2 != 0) return fail(H3B_ERR_SHAPE, "W must be even for token pairing");
  if (full->d < 8 || full->d % 8 != 0 || full->d > 65536)
    return fail(H3B_ERR_SHAPE, "d must be a multiple of 8, <= 65536");
  const long long L = grid_tokens(full->T, full->H, full->W);
  if (L < 0 || L * full->B >= (1LL << 31)) return fail(H3B_ERR_SHAPE, "too many tokens");
  return H3B_OK;
}

h3b_status h3b_token_pair(const h3b_dims* full, const void* x, void* xm, void* xm_copy, h3b_stream stream) {
  h3b_status s = check_pair_dims(full);
  if (s != H3B_OK) return s;
  if (!x || !xm) return fail(H3B_ERR_ARG, "x and xm must be non-NULL");
  if (!aligned16(x) || !aligned16(xm) || (xm_copy && !aligned16(xm_copy))) return fail(H3B_ERR_ALIGN, "alignment");
  DeviceInfo* di = nullptr;
  if ((s = device_info(&di)) != H3B_OK) return s;
  const long long lines = (long long)full->B * full->T * full->H;
  cudaStream_t st = stream;
  H3B_CK(launch_token_pair(x, xm, xm_copy, lines, full->W, full->d, di->sms, stream), "token_pair");
  return H3B_OK;
}

h3b_status h3b_token_unpair(const h3b_dims* full, const void* x, const void* xm, const void* ym, void* out,
                            h3b_stream stream) {
  h3b_status s = check_pair_dims(full);
  if (s != H3B_OK) return s;
  if (!x || !ym || !out) return fail(H3B_ERR_ARG, "NULL pointer");
  if (!aligned16(x) || (xm && !aligned16(xm)) || !aligned16(ym) || !aligned16(out))
    return fail(H3B_ERR_ALIGN, "alignment");
  DeviceInfo* di = nullptr;
  if ((s = device_info(&di)) != H3B_OK) return s;
  const long long lines = (long long)full->B * full->T * full->H;
  cudaStream_t st = stream;
  H3B_CK(launch_token_unpair(x, xm, ym, out, lines, full->W, full->d, di->sms, stream), "token_unpair");
  return H3B_OK;
}

h3b_status h3b_quantize_weights(const float* w, int rows, int cols, int8_t* q, float* s, h3b_stream stream) {
  cudaStream_t st = stream;
  if (rows < 0 || cols < 16 || cols % 16 != 0) return fail(H3B_ERR_SHAPE, "cols must be a positive multiple of 16");
  if (rows == 0) return H3B_OK;  // empty problem: nothing to launch
  if (!w || !q || !s) return fail(H3B_ERR_ARG, "NULL pointer");
  if (!aligned16(w) || !aligned16(q)) return fail(H3B_ERR_ALIGN, "alignment");
  DeviceInfo* di = nullptr;
  h3b_status hs = device_info(&di);
  if (hs != H3B_OK) return hs;
  H3B_CK(launch_quant_rows_f32(w, rows, cols, q, s, stream), "quantize_weights");
  return H3B_OK;
}

h3b_status h3b_test_bounded_wait(unsigned long long limit_ns, int* waited_out) {
  if (!waited_out) return fail(H3B_ERR_ARG, "waited_out is NULL");
  if (limit_ns < 1000ull || limit_ns > 1000000000ull) return fail(H3B_ERR_ARG, "limit_ns must be in [1 us, 1 s]");
  DeviceInfo* di = nullptr;
  h3b_status s = device_info(&di);
  if (s != H3B_OK) return s;
  cudaStream_t st = nullptr;
  H3B_CK((bounded_wait_probe_kernel<<<1, 32>>>(di->err, limit_ns), cudaGetLastError()), "bounded_wait_probe");
  int r = -1;
  H3B_CK(cudaMemcpyFromSymbol(&r, g_h3b_probe_result, sizeof(int)), "read probe result");  // waits for the kernel
  *waited_out = r;
  return H3B_OK;
}

h3b_status h3b_device_error(unsigned int* code, int clear) {
  cudaStream_t st = nullptr;
  if (!code) return fail(H3B_ERR_ARG, "code is NULL");
  DeviceInfo* di = nullptr;
  h3b_status s = device_info(&di);
  if (s != H3B_OK) return s;
  H3B_CK(cudaDeviceSynchronize(), "cudaDeviceSynchronize");
  H3B_CK(cudaMemcpy(code, di->err, sizeof(unsigned), cudaMemcpyDeviceToHost), "read error word");
  if (clear) H3B_CK(cudaMemset(di->err, 0, sizeof(unsigned)), "clear error word");
#ifdef H3B_CHECKED
  // the row kernels' bounds word (they take no error-word argument)
  if (unsigned* bw = rowops_bounds_word()) {
    unsigned b = 0;
    H3B_CK(cudaMemcpy(&b, bw, sizeof(unsigned), cudaMemcpyDeviceToHost), "read bounds word");
    if (clear) H3B_CK(cudaMemset(bw, 0, sizeof(unsigned)), "clear bounds word");
    *code |= b;
  }
#endif
  return *code ? H3B_ERR_DEVICE_CHECK : H3B_OK;
}

int h3b_checked_build(void) {
#ifdef H3B_CHECKED
  return 1;
#else
  return 0;
#endif
}

// ---- step entry points ------------------------------------------------------

h3b_status h3b_adaln_modulation(const h3b_dims* dims, const void* w_ada, const float* b_ada, const float* c,
                                float* mod, h3b_stream stream) {
  cudaStream_t st = stream;
  h3b_status s = check_dims(dims);
  if (s != H3B_OK) return s;
  if (!w_ada || !c || !mod) return fail(H3B_ERR_ARG, "NULL pointer");
  if (!aligned16(w_ada) || !aligned16(c) || !aligned16(mod)) return fail(H3B_ERR_ALIGN, "alignment");
  DeviceInfo* di = nullptr;
  if ((s = device_info(&di)) != H3B_OK) return s;
  H3B_CK(launch_adaln_gemv(w_ada, b_ada, c, dims->B, dims->d, mod, nullptr, 0, 0, 0, 0, 0, 0, 0.0, di->sms, stream),
         "adaln_gemv");
  return H3B_OK;
}

h3b_status h3b_ln_modulate_quantize(const void* x, int rows, int d, float eps, const float* shift,
                                    const float* scale, int rows_per_item, int mod_stride, int8_t* q, float* s,
                                    void* h_out, float* absmax_zero, int write_codes, h3b_stream stream) {
  cudaStream_t st = stream;
  if (rows < 0 || d < 256 || d % 256 != 0 || d > 8192) return fail(H3B_ERR_SHAPE, "d must be a multiple of 256, <= 8192");
  if (rows_per_item < 1 || mod_stride < 0 || mod_stride % 4 != 0) return fail(H3B_ERR_ARG, "rows_per_item/mod_stride");
  if (rows == 0) return H3B_OK;  // empty problem: nothing to launch
  if (!x || !shift || !scale || (write_codes && (!q || !s))) return fail(H3B_ERR_ARG, "NULL pointer");
  if (!aligned16(x) || !aligned16(shift) || !aligned16(scale) || (q && !aligned16(q)) || (h_out && !aligned16(h_out)))
    return fail(H3B_ERR_ALIGN, "alignment");
  DeviceInfo* di = nullptr;
  h3b_status hs = device_info(&di);
  if (hs != H3B_OK) return hs;
  H3B_CK(launch_ln_mod_quant(x, rows, d, eps, shift, scale, rows_per_item, mod_stride, q, s, h_out, absmax_zero,
                             write_codes, di->err, di->sms, stream), "ln_mod_quant");
  return H3B_OK;
}

h3b_status h3b_quantize_rows(const void* h, int rows, int cols, const float* absmax, int8_t* q, float* s,
                             h3b_stream stream) {
  cudaStream_t st = stream;
  if (rows < 0 || cols < 16 || cols % 16 != 0) return fail(H3B_ERR_SHAPE, "cols must be a positive multiple of 16");
  if (rows == 0) return H3B_OK;  // empty problem: nothing to launch
  if (!h || !q || !s) return fail(H3B_ERR_ARG, "NULL pointer");
  if (!aligned16(h) || !aligned16(q)) return fail(H3B_ERR_ALIGN, "alignment");
  DeviceInfo* di = nullptr;
  h3b_status hs = device_info(&di);
  if (hs != H3B_OK) return hs;
  H3B_CK(launch_quant_rows_bf16(h, rows, cols, absmax, q, s, di->sms, stream), "quantize_rows");
  return H3B_OK;
}

// Host checks shared by the GEMM entry points (no device query). An empty problem
// (M == 0) sets *empty and returns as soon as the sizes are checked: its pointers
// are not inspected.
static h3b_status gemm_checks(const void* A, const void* W, const void* out, int M, int N, int K, bool* empty) {
  *empty = false;
  if (M < 0 || N < 16 || N % 16 != 0 || K < 16 || K % 16 != 0)
    return fail(H3B_ERR_SHAPE, "need M >= 0, N and K positive multiples of 16");
  const long long lim = 1LL << 40;  // elements of any operand or result; keeps every tile count in int
  if ((long long)M * N > lim || (long long)M * K > lim || (long long)N * K > lim)
    return fail(H3B_ERR_SHAPE, "problem too large (an operand or the result exceeds 2^40 elements)");
  if (M == 0) {
    *empty = true;
    return H3B_OK;
  }
  if (!A || !W || !out) return fail(H3B_ERR_ARG, "NULL pointer");
  if (!aligned16(A) || !aligned16(W) || !aligned16(out)) return fail(H3B_ERR_ALIGN, "alignment");
  return H3B_OK;
}

h3b_status h3b_gemm_i8_s32(const int8_t* A, const int8_t* W, int32_t* C, int M, int N, int K, h3b_stream stream) {
  cudaStream_t st = stream;
  bool empty = false;
  h3b_status s = gemm_checks(A, W, C, M, N, K, &empty);
  if (s != H3B_OK || empty) return s;
  DeviceInfo* di = nullptr;
  if ((s = device_info(&di)) != H3B_OK) return s;
  GemmArgs a = base_args(M, N, K, di->err);
  a.out = C;
  H3B_CK(launch_gemm(true, EPI_S32, A, W, a, di->sms, stream), "gemm_i8_s32");
  return H3B_OK;
}

h3b_status h3b_gemm_i8_dequant(const int8_t* A, const float* sA, const int8_t* W, const float* sW,
                               const float* bias, void* out, int M, int N, int K, h3b_stream stream) {
  cudaStream_t st = stream;
  bool empty = false;
  h3b_status s = gemm_checks(A, W, out, M, N, K, &empty);
  if (s != H3B_OK || empty) return s;
  if (!sA || !sW) return fail(H3B_ERR_ARG, "scales NULL");
  if (!aligned16(sW) || (bias && !aligned16(bias))) return fail(H3B_ERR_ALIGN, "alignment");
  DeviceInfo* di = nullptr;
  if ((s = device_info(&di)) != H3B_OK) return s;
  GemmArgs a = base_args(M, N, K, di->err);
  a.sA = sA; a.sW = sW; a.bias = bias; a.out = out;
  H3B_CK(launch_gemm(true, EPI_DEQ, A, W, a, di->sms, stream), "gemm_i8_dequant");
  return H3B_OK;
}

h3b_status h3b_qkv_projection(const h3b_dims* dims, const void* A, const float* sA, const h3b_block_weights* w,
                              void* qkv, void* rope_ws, h3b_stream stream) {
  cudaStream_t st = stream;
  h3b_status s = check_dims(dims);
  if (s != H3B_OK) return s;
  if (!A || !w || !qkv || !rope_ws) return fail(H3B_ERR_ARG, "NULL pointer");
  if (dims->qkv_int8 && (!w->wqkv || !w->sqkv || !sA)) return fail(H3B_ERR_ARG, "int8 QKV needs wqkv, sqkv, sA");
  if (!dims->qkv_int8 && !w->wqkv_bf16) return fail(H3B_ERR_ARG, "bf16 QKV needs wqkv_bf16");
  if (!aligned16(A) || !aligned16(qkv) || !aligned16(rope_ws) || (w->bqkv && !aligned16(w->bqkv)) ||
      (w->sqkv && !aligned16(w->sqkv)))
    return fail(H3B_ERR_ALIGN, "alignment");
  DeviceInfo* di = nullptr;
  if ((s = device_info(&di)) != H3B_OK) return s;
  const int L = dims->T * dims->H * dims->W, D = dims->d;
  float2* rope = static_cast<float2*>(rope_ws);
  H3B_CK(launch_rope_table(rope, dims->T, dims->H, dims->W, dims->rope_t, dims->rope_h, dims->rope_w,
                           dims->rope_theta, stream), "rope_table");
  GemmArgs a = base_args(dims->B * L, 3 * D, D, di->err);
  a.sA = sA; a.sW = w->sqkv; a.bias = w->bqkv; a.out = qkv;
  a.B = dims->B; a.L = L; a.T = dims->T; a.H = dims->H; a.W = dims->W; a.d = D;
  a.n_heads = dims->n_heads; a.head_dim = dims->head_dim;
  a.rope_t = dims->rope_t; a.rope_h = dims->rope_h; a.rope_w = dims->rope_w; a.rope = rope;
  H3B_CK(launch_gemm(dims->qkv_int8 != 0, EPI_QKV, A, dims->qkv_int8 ? (const void*)w->wqkv : w->wqkv_bf16, a,
                     di->sms, stream), "qkv_projection");
  return H3B_OK;
}

h3b_status h3b_attention(const h3b_dims* dims, const void* qkv, void* o, float* absmax, h3b_stream stream) {
  cudaStream_t st = stream;
  // Attention alone needs only the grid, the batch and the head shape.
  if (!dims) return fail(H3B_ERR_ARG, "dims is NULL");
  if (dims->B < 1 || dims->T < 1 || dims->H < 1 || dims->W < 1 || dims->n_heads < 1)
    return fail(H3B_ERR_SHAPE, "B, T, H, W, n_heads must be >= 1");
  if (dims->head_dim != 64 && dims->head_dim != 128) return fail(H3B_ERR_SHAPE, "head_dim must be 64 or 128");
  if ((long long)dims->B * dims->n_heads > 65535) return fail(H3B_ERR_SHAPE, "B * n_heads must be <= 65535");
  const long long L_tokens = grid_tokens(dims->T, dims->H, dims->W);
  if (L_tokens < 0 || L_tokens * dims->B >= (1LL << 31)) return fail(H3B_ERR_SHAPE, "too many tokens");
  h3b_status s = H3B_OK;
  if (!qkv || !o || !absmax) return fail(H3B_ERR_ARG, "NULL pointer");
  if (!aligned16(qkv) || !aligned16(o)) return fail(H3B_ERR_ALIGN, "alignment");
  DeviceInfo* di = nullptr;
  if ((s = device_info(&di)) != H3B_OK) return s;
  AttnArgs a{dims->B, dims->T * dims->H * dims->W, dims->n_heads, dims->head_dim, qkv, o, absmax, di->err};
  H3B_CK(launch_attention(a, stream), "attention");
  return H3B_OK;
}

h3b_status h3b_gemm_i8_gated_residual(const int8_t* A, const float* sA, const int8_t* W, const float* sW,
                                      const float* bias, const float* gate, int rows_per_item, int gate_stride,
                                      void* x, int M, int N, int K, h3b_stream stream) {
  cudaStream_t st = stream;
  bool empty = false;
  h3b_status s = gemm_checks(A, W, x, M, N, K, &empty);
  if (s != H3B_OK || empty) return s;
  if (!sA || !sW || !gate) return fail(H3B_ERR_ARG, "scales/gate NULL");
  if (rows_per_item < 1 || gate_stride < 0 || gate_stride % 4 != 0) return fail(H3B_ERR_ARG, "rows_per_item/gate_stride");
  if (!aligned16(sW) || !aligned16(gate) || (bias && !aligned16(bias))) return fail(H3B_ERR_ALIGN, "alignment");
  DeviceInfo* di = nullptr;
  if ((s = device_info(&di)) != H3B_OK) return s;
  GemmArgs a = base_args(M, N, K, di->err);
  a.sA = sA; a.sW = sW; a.bias = bias; a.out = x;
  a.gate = gate; a.rows_per_item = rows_per_item; a.gate_stride = gate_stride;
  H3B_CK(launch_gemm(true, EPI_RESID, A, W, a, di->sms, stream), "gemm_i8_gated_residual");
  return H3B_OK;
}

h3b_status h3b_gemm_bf16_gated_residual(const void* A, const void* W, const float* bias, const float* gate,
                                        int rows_per_item, int gate_stride, void* x, int M, int N, int K,
                                        h3b_stream stream) {
  cudaStream_t st = stream;
  bool empty = false;
  h3b_status s = gemm_checks(A, W, x, M, N, K, &empty);
  if (s != H3B_OK || empty) return s;
  if (!gate) return fail(H3B_ERR_ARG, "gate NULL");
  if (rows_per_item < 1 || gate_stride < 0 || gate_stride % 4 != 0) return fail(H3B_ERR_ARG, "rows_per_item/gate_stride");
  if (!aligned16(gate) || (bias && !aligned16(bias))) return fail(H3B_ERR_ALIGN, "alignment");
  DeviceInfo* di = nullptr;
  if ((s = device_info(&di)) != H3B_OK) return s;
  GemmArgs a = base_args(M, N, K, di->err);
  a.bias = bias; a.out = x;
  a.gate = gate; a.rows_per_item = rows_per_item; a.gate_stride = gate_stride;
  H3B_CK(launch_gemm(false, EPI_RESID, A, W, a, di->sms, stream), "gemm_bf16_gated_residual");
  return H3B_OK;
}

h3b_status h3b_gemm_i8_gelu(const int8_t* A, const float* sA, const int8_t* W, const float* sW, const float* bias,
                            void* g, float* absmax, int M, int N, int K, h3b_stream stream) {
  cudaStream_t st = stream;
  bool empty = false;
  h3b_status s = gemm_checks(A, W, g, M, N, K, &empty);
  if (s != H3B_OK || empty) return s;
  if (!sA || !sW || !absmax) return fail(H3B_ERR_ARG, "scales/absmax NULL");
  if (!aligned16(sW) || (bias && !aligned16(bias))) return fail(H3B_ERR_ALIGN, "alignment");
  DeviceInfo* di = nullptr;
  if ((s = device_info(&di)) != H3B_OK) return s;
  GemmArgs a = base_args(M, N, K, di->err);
  a.sA = sA; a.sW = sW; a.bias = bias; a.out = g; a.absmax = absmax;
  H3B_CK(launch_gemm(true, EPI_GELU, A, W, a, di->sms, stream), "gemm_i8_gelu");
  return H3B_OK;
}

h3b_status h3b_profile_enable(int enable) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = enable != 0;
  return H3B_OK;
}

int h3b_profile_read(h3b_kernel_time* out, int max_entries) {
  if (!out || max_entries < 0) return H3B_ERR_ARG;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  int n = 0;
  for (const ProfRec& r : g_prof_recs) {
    float ms = 0.0f;
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, r.a, r.b);
    if (e != cudaSuccess) return cuda_fail(e, "profile event");
    int k = 0;
    while (k < n && std::string(out[k].name) != r.name) ++k;
    if (k == n) {
      if (n == max_entries) continue;
      out[n].name = r.name;
      out[n].launches = 0;
      out[n].total_ms = 0.0;
      ++n;
    }
    out[k].launches += 1;
    out[k].total_ms += ms;
  }
  for (const ProfRec& r : g_prof_recs) {
    g_prof_free.push_back(r.a);
    g_prof_free.push_back(r.b);
  }
  g_prof_recs.clear();
  return n;
}

}  // extern "C"
