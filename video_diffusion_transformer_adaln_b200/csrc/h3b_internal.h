// Internal launcher interface between the C ABI (h3b_api.cu) and the kernel
// translation units. Host-only declarations; every launcher enqueues on `st`
// and returns the launch status.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>

namespace h3b {

// ---- memory-bound row kernels (k_rowops.cu)
// rope_tab (optional): the same launch also fills the RoPE table (see launch_rope_table).
cudaError_t launch_adaln_gemv(const void* W_ada, const float* bias, const float* c, int B, int d,
                              float* mod, float2* rope_tab, int T, int H, int W, int rt, int rh, int rw,
                              double theta, int sms, cudaStream_t st);
cudaError_t launch_ln_mod_quant(const void* x, int rows, int d, float eps, const float* shift,
                                const float* scale, int rows_per_item, int mod_stride, int8_t* q,
                                float* s, void* h_out, float* absmax_zero, int write_codes, unsigned* err,
                                int sms, cudaStream_t st);
cudaError_t launch_quant_rows_bf16(const void* h, int rows, int cols, const float* absmax,
                                   int8_t* q, float* s, int sms, cudaStream_t st);
cudaError_t launch_quant_rows_f32(const float* w, int rows, int cols, int8_t* q, float* s,
                                  cudaStream_t st);
cudaError_t launch_token_pair(const void* x, void* xm, void* xm2, long long lines, int W, int d,
                              int sms, cudaStream_t st);
// delta fp32 [n] = after - before (bf16 [n]); x bf16 [n] = bf16(x + delta). n % 8 == 0.
cudaError_t launch_range_delta(const void* before, const void* after, float* delta, long long n, int sms,
                               cudaStream_t st);
cudaError_t launch_range_apply(void* x, const float* delta, long long n, int sms, cudaStream_t st);
// xm may be nullptr: the merged input is then recomputed from x.
cudaError_t launch_token_unpair(const void* x, const void* xm, const void* ym, void* out,
                                long long lines, int W, int d, int sms, cudaStream_t st);
cudaError_t launch_rope_table(float2* tab, int T, int H, int W, int rt, int rh, int rw,
                              double theta, cudaStream_t st);
// Device address of the row kernels' bounds word (checked build), or nullptr.
unsigned* rowops_bounds_word();

// ---- tensor-core GEMM (k_gemm.cu)
enum GemmEpilogue : int {
  EPI_S32 = 0,    // int32 accumulators out
  EPI_DEQ = 1,    // bf16(acc * sA * sW + bias)
  EPI_QKV = 2,    // dequant + 3D RoPE on Q, K; head-major Q/K/V
  EPI_RESID = 3,  // x = bf16(x + gate * (acc * sA * sW + bias))
  EPI_GELU = 4,   // g = bf16(gelu_tanh(acc * sA * sW + bias)), row absmax
};

struct GemmArgs {
  int M, N, K;
  const float* sA;  // [M] per-row activation scales (int8 operands only)
  const float* sW;  // [N] per-output-channel weight scales (int8 operands only)
  const float* bias;
  void* out;
  float* absmax;      // EPI_GELU
  const float* gate;  // EPI_RESID: gate[item * gate_stride + n]
  int rows_per_item, gate_stride;
  // EPI_QKV
  int B, L, T, H, W, d, n_heads, head_dim, rope_t, rope_h, rope_w;
  const float2* rope;  // table from launch_rope_table
  int rope_smem_entries;  // set by launch_gemm: table entries staged in shared memory (0: none)
  unsigned* err;       // device error word
  // tile raster (set by launch_gemm): groups of `group` M-tiles (raster_n == 0)
  // or of `group` N-tiles (raster_n == 1)
  int raster_n, group;
};

// A [M][K] and W [N][K] row-major, int8 (kInt8) or bf16.
cudaError_t launch_gemm(bool int8_operands, GemmEpilogue epi, const void* A, const void* W,
                        const GemmArgs& args, int sms, cudaStream_t st);

// ---- attention (k_attention.cu)
struct AttnArgs {
  int B, L, n_heads, head_dim;
  const void* qkv;  // bf16 [3][B][n_heads][L][head_dim]
  void* o;          // bf16 [B][L][n_heads*head_dim]
  float* absmax;    // [B*L]
  unsigned* err;
};
cudaError_t launch_attention(const AttnArgs& a, cudaStream_t st);

// ---- error detail reported by h3b_last_error_detail (h3b_api.cu)
void set_error_detail(const std::string& why);
// ---- H3B_OK when the current device is compute capability 10.0, else the status
//      (H3B_ERR_ARCH, H3B_ERR_CUDA) the block entry points return (h3b_api.cu)
int check_current_device();
// ---- whether h3b_profile_enable(1) is in effect (h3b_api.cu)
bool profiling_enabled();

// ---- TMA descriptor construction (h3b_api.cu)
// Row-major 2D tensor of `rows` x `cols` elements of `elem_bytes` each,
// `row_stride_bytes` apart; box of box_cols x box_rows with a 128-, 64- or 32-byte
// swizzle (0: none).
bool make_tmap_2d(CUtensorMap* map, const void* base, int elem_bytes, uint64_t cols,
                  uint64_t rows, uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows,
                  int swizzle_bytes = 128);
// 3D tensor [d2][d1][d0] (d0 innermost), box of box0 x box1 x 1, 128-byte swizzle.
bool make_tmap_3d(CUtensorMap* map, const void* base, int elem_bytes, uint64_t d0, uint64_t d1,
                  uint64_t d2, uint32_t box0, uint32_t box1);

// ---- launches with programmatic stream serialization (each kernel calls
//      griddepcontrol.wait before touching global data); off when the
//      environment variable H3B_PDL is "0" (h3b_api.cu)
bool pdl_enabled();
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k, args...);
}

}  // namespace h3b
