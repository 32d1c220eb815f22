// Memory-bound kernels of the block: AdaLN modulation GEMV, the fused
// LayerNorm + modulation + per-row int8 quantizer, the quant-only pass, the
// per-output-channel weight quantizer, token pairing and the RoPE table.
//
// All of them stream rows with 16-byte vector accesses, one warp (or block)
// per row, with warp-shuffle reductions; none keeps state between launches.
//
// Method references (web pages on the h3.c / h3-metal engine):
//   "h3-metal: Apple Silicon을 위한 네이티브 MiniMax-H3 추론", section "Int8 양자화":
//     dynamic per-row activation quantization, per-output-channel weight scales,
//     the activation quantizer fused into the preceding gated-AdaLN kernel.
//   "맥북에서 AI 영상 생성 모델 돌리기 - MiniMax H3 로컬 실행과 30초 애니메이션 만들기",
//     section "int8 이 뭔가요": one F32 scale per row / per output channel.
//   "h3-metal: ...", section "속도 및 품질 트레이드오프", Token Reduction row:
//     horizontally adjacent video tokens are paired.
#include "h3b_common.cuh"
#include "h3b_internal.h"

namespace h3b {

// ---------------------------------------------------------------------------
// Warp / block reductions
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// The quantizer decision, in binary32 exactly as the method states it:
// scale = absmax / 127, code = round-half-even(v / scale) clamped to [-127, 127];
// absmax == 0 gives code 0.
__device__ __forceinline__ int quant_code(float v, float scale, float absmax) {
  if (absmax == 0.0f) return 0;
  int c = __float2int_rn(__fdiv_rn(v, scale));
  return max(-127, min(127, c));
}
__device__ __forceinline__ uint32_t pack4_i8(int a, int b, int c, int d) {
  return (uint32_t)(a & 0xFF) | ((uint32_t)(b & 0xFF) << 8) | ((uint32_t)(c & 0xFF) << 16) |
         ((uint32_t)(d & 0xFF) << 24);
}

// ---------------------------------------------------------------------------
// AdaLN modulation Linear: mod[b][j] = sum_k W[j][k] c[b][k] + bias[j].
// One warp per output row j, all batch items at once (W is read once); c is
// staged in shared memory as fp32.
// ---------------------------------------------------------------------------
constexpr int kGemvMaxB = 8;

__global__ void __launch_bounds__(256) adaln_gemv_kernel(const __nv_bfloat16* __restrict__ W,
                                                         const float* __restrict__ bias,
                                                         const float* __restrict__ c, int B, int d,
                                                         float* __restrict__ mod) {
  extern __shared__ float cs[];  // [B][d]
  for (int i = threadIdx.x; i < B * d; i += blockDim.x) cs[i] = c[i];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x * 8 + warp;
  if (j >= 6 * d) return;
  const uint4* wr = reinterpret_cast<const uint4*>(W + (size_t)j * d);
  const int nvec = d / 8;
  float acc[kGemvMaxB];
#pragma unroll
  for (int b = 0; b < kGemvMaxB; ++b) acc[b] = 0.0f;
  for (int v0 = lane; v0 < nvec; v0 += 32 * 4) {
    uint4 w4[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int v = v0 + 32 * u;
      if (v < nvec) w4[u] = __ldcs(wr + v);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int v = v0 + 32 * u;
      if (v >= nvec) break;
      const uint32_t ww[4] = {w4[u].x, w4[u].y, w4[u].z, w4[u].w};
#pragma unroll
      for (int b = 0; b < kGemvMaxB; ++b) {
        if (b >= B) break;
        const float* cb = cs + b * d + v * 8;
        float a = acc[b];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          a = fmaf(bf16_lo(ww[e]), cb[2 * e], a);
          a = fmaf(bf16_hi(ww[e]), cb[2 * e + 1], a);
        }
        acc[b] = a;
      }
    }
  }
#pragma unroll
  for (int b = 0; b < kGemvMaxB; ++b) {
    if (b >= B) break;
    const float r = warp_sum(acc[b]);
    if (lane == 0) mod[(size_t)b * 6 * d + j] = r + (bias ? bias[j] : 0.0f);
  }
}

// ---------------------------------------------------------------------------
// Fused LayerNorm + modulation + per-row int8 quantization. One warp per row;
// the row stays in registers (NV 16-byte vectors per lane, d = 256*NV).
//   y = (x - mean) * rsqrt(var + eps)          (fp32, two-pass variance)
//   h = bf16(y * (1 + scale) + shift)
//   s = absmax(h) / 127, q = rint(h / s)       (binary32 decision)
// ---------------------------------------------------------------------------
template <int NV>
__global__ void __launch_bounds__(256, (NV <= 4 ? 4 : (NV <= 12 ? 2 : 1))) ln_mod_quant_kernel(
    const __nv_bfloat16* __restrict__ x, int rows, float eps, const float* __restrict__ shift,
    const float* __restrict__ scale, int rows_per_item, int mod_stride, int8_t* __restrict__ q,
    float* __restrict__ s, __nv_bfloat16* __restrict__ h_out, float* __restrict__ absmax_zero,
    int write_codes) {
  constexpr int d = NV * 256;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + warp;
  if (row >= rows) return;
  const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)row * d);
  uint4 v[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) v[i] = __ldcs(xr + lane + 32 * i);

  float sum = 0.0f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const uint32_t u[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) sum += bf16_lo(u[e]) + bf16_hi(u[e]);
  }
  const float mean = warp_sum(sum) * (1.0f / d);
  float sq = 0.0f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const uint32_t u[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float a = bf16_lo(u[e]) - mean, b = bf16_hi(u[e]) - mean;
      sq = fmaf(a, a, sq);
      sq = fmaf(b, b, sq);
    }
  }
  const float rstd = 1.0f / sqrtf(warp_sum(sq) * (1.0f / d) + eps);

  const int item = row / rows_per_item;
  const float4* sh4 = reinterpret_cast<const float4*>(shift + (size_t)item * mod_stride);
  const float4* sc4 = reinterpret_cast<const float4*>(scale + (size_t)item * mod_stride);
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int vec = lane + 32 * i;
    const float4 sa = __ldg(sh4 + 2 * vec), sb = __ldg(sh4 + 2 * vec + 1);
    const float4 ca = __ldg(sc4 + 2 * vec), cb = __ldg(sc4 + 2 * vec + 1);
    const float shv[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
    const float scv[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
    uint32_t u[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float h0 = round_bf16(fmaf((bf16_lo(u[e]) - mean) * rstd, 1.0f + scv[2 * e], shv[2 * e]));
      const float h1 =
          round_bf16(fmaf((bf16_hi(u[e]) - mean) * rstd, 1.0f + scv[2 * e + 1], shv[2 * e + 1]));
      amax = fmaxf(amax, fmaxf(fabsf(h0), fabsf(h1)));
      u[e] = pack_bf16x2(h0, h1);
    }
    v[i] = make_uint4(u[0], u[1], u[2], u[3]);
  }
  amax = warp_max(amax);
  if (h_out) {
    uint4* hr = reinterpret_cast<uint4*>(h_out + (size_t)row * d);
#pragma unroll
    for (int i = 0; i < NV; ++i) hr[lane + 32 * i] = v[i];
  }
  if (absmax_zero && lane == 0) absmax_zero[row] = 0.0f;
  if (!write_codes) return;
  const float sc = __fdiv_rn(amax, 127.0f);
  if (lane == 0) s[row] = sc;
  uint2* qr = reinterpret_cast<uint2*>(q + (size_t)row * d);
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const uint32_t u[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
    int c[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      c[2 * e] = quant_code(bf16_lo(u[e]), sc, amax);
      c[2 * e + 1] = quant_code(bf16_hi(u[e]), sc, amax);
    }
    qr[lane + 32 * i] = make_uint2(pack4_i8(c[0], c[1], c[2], c[3]), pack4_i8(c[4], c[5], c[6], c[7]));
  }
}

// ---------------------------------------------------------------------------
// Per-row quantization of bf16 or fp32 rows; one block per row. With a
// precomputed absmax the row is read once.
// ---------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&f)[8]);
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&f)[8]) {
  const uint4 u = __ldcs(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    f[2 * e] = bf16_lo(w[e]);
    f[2 * e + 1] = bf16_hi(w[e]);
  }
}
template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&f)[8]) {
  const float4 a = __ldcs(reinterpret_cast<const float4*>(p));
  const float4 b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

template <typename T>
__global__ void __launch_bounds__(256) quant_rows_kernel(const T* __restrict__ in, int cols,
                                                         const float* __restrict__ absmax_in,
                                                         int8_t* __restrict__ q,
                                                         float* __restrict__ s) {
  __shared__ float red[8];
  const int row = blockIdx.x;
  const T* r = in + (size_t)row * cols;
  const int nvec = cols / 8;
  float amax;
  if (absmax_in) {
    amax = absmax_in[row];
  } else {
    float m = 0.0f;
    for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
      float f[8];
      load8<T>(r + v * 8, f);
#pragma unroll
      for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(f[e]));
    }
    m = warp_max(m);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    m = red[0];
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, red[w]);
    amax = m;
  }
  const float sc = __fdiv_rn(amax, 127.0f);
  if (threadIdx.x == 0) s[row] = sc;
  uint2* qr = reinterpret_cast<uint2*>(q + (size_t)row * cols);
  for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
    float f[8];
    load8<T>(r + v * 8, f);
    int c[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) c[e] = quant_code(f[e], sc, amax);
    qr[v] = make_uint2(pack4_i8(c[0], c[1], c[2], c[3]), pack4_i8(c[4], c[5], c[6], c[7]));
  }
}

// ---------------------------------------------------------------------------
// Token pairing. Rows are the B*T*H (t, h) lines of W tokens of d channels.
//   pair:   xm[line][k] = bf16((x[line][2k] + x[line][2k+1]) / 2)
//   unpair: out[line][w] = bf16(x[line][w] + (ym[line][w/2] - xm[line][w/2]))
// The fp32 sum of two bf16 values followed by the halving and one rounding to
// bf16 gives the correctly rounded mean.
// ---------------------------------------------------------------------------
__global__ void token_pair_kernel(const __nv_bfloat16* __restrict__ x, __nv_bfloat16* __restrict__ xm,
                                  __nv_bfloat16* __restrict__ xm2, long long n_out_vec, int Wm,
                                  int dvec) {
  for (long long o = blockIdx.x * (long long)blockDim.x + threadIdx.x; o < n_out_vec;
       o += (long long)gridDim.x * blockDim.x) {
    const long long rp = o / dvec;
    const int cv = (int)(o - rp * dvec);
    const long long line = rp / Wm;
    const int k = (int)(rp - line * Wm);
    const long long in0 = ((line * (2LL * Wm) + 2 * k) * dvec + cv);
    const uint4 a = __ldcs(reinterpret_cast<const uint4*>(x) + in0);
    const uint4 b = __ldcs(reinterpret_cast<const uint4*>(x) + in0 + dvec);
    const uint32_t ua[4] = {a.x, a.y, a.z, a.w}, ub[4] = {b.x, b.y, b.z, b.w};
    uint32_t r[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      r[e] = pack_bf16x2((bf16_lo(ua[e]) + bf16_lo(ub[e])) * 0.5f,
                         (bf16_hi(ua[e]) + bf16_hi(ub[e])) * 0.5f);
    const uint4 out = make_uint4(r[0], r[1], r[2], r[3]);
    reinterpret_cast<uint4*>(xm)[o] = out;
    if (xm2) reinterpret_cast<uint4*>(xm2)[o] = out;
  }
}

__global__ void token_unpair_kernel(const __nv_bfloat16* __restrict__ x,
                                    const __nv_bfloat16* __restrict__ xm,
                                    const __nv_bfloat16* __restrict__ ym, __nv_bfloat16* out,
                                    long long n_vec, int W, int dvec) {
  for (long long o = blockIdx.x * (long long)blockDim.x + threadIdx.x; o < n_vec;
       o += (long long)gridDim.x * blockDim.x) {
    const long long tok = o / dvec;
    const int cv = (int)(o - tok * dvec);
    const long long line = tok / W;
    const int w = (int)(tok - line * W);
    const long long m = (line * (W / 2) + w / 2) * dvec + cv;
    const uint4 a = __ldcs(reinterpret_cast<const uint4*>(x) + o);
    const uint4 p = __ldg(reinterpret_cast<const uint4*>(xm) + m);
    const uint4 y = __ldg(reinterpret_cast<const uint4*>(ym) + m);
    const uint32_t ua[4] = {a.x, a.y, a.z, a.w}, up[4] = {p.x, p.y, p.z, p.w},
                   uy[4] = {y.x, y.y, y.z, y.w};
    uint32_t r[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      r[e] = pack_bf16x2(bf16_lo(ua[e]) + (bf16_lo(uy[e]) - bf16_lo(up[e])),
                         bf16_hi(ua[e]) + (bf16_hi(uy[e]) - bf16_hi(up[e])));
    reinterpret_cast<uint4*>(out)[o] = make_uint4(r[0], r[1], r[2], r[3]);
  }
}

// ---------------------------------------------------------------------------
// RoPE table: for each axis (t, h, w) with n positions and segment length r,
// entry [pos * (r/2) + j] = (cos, sin)(pos * theta^(-2j/r)), evaluated in fp64
// and stored as fp32. Axis blocks are stored one after the other (t, h, w).
// ---------------------------------------------------------------------------
__global__ void rope_table_kernel(float2* __restrict__ tab, int T, int H, int W, int rt, int rh,
                                  int rw, double theta) {
  const int nt = T * (rt / 2), nh = H * (rh / 2), nw = W * (rw / 2);
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nt + nh + nw; i += gridDim.x * blockDim.x) {
    int idx = i, r = rt;
    if (idx >= nt + nh) { idx -= nt + nh; r = rw; }
    else if (idx >= nt) { idx -= nt; r = rh; }
    const int half = r / 2, pos = idx / half, j = idx % half;
    const double ang = (double)pos * pow(theta, -2.0 * (double)j / (double)r);
    tab[i] = make_float2((float)cos(ang), (float)sin(ang));
  }
}

// ---------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------
cudaError_t launch_adaln_gemv(const void* W, const float* bias, const float* c, int B, int d,
                              float* mod, cudaStream_t st) {
  if (B > kGemvMaxB) return cudaErrorInvalidValue;
  const size_t smem = (size_t)B * d * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(adaln_gemv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  adaln_gemv_kernel<<<(6 * d + 7) / 8, 256, smem, st>>>(static_cast<const __nv_bfloat16*>(W), bias, c,
                                                        B, d, mod);
  return cudaGetLastError();
}

template <int NV>
static cudaError_t ln_dispatch(const void* x, int rows, float eps, const float* shift,
                               const float* scale, int rpi, int ms, int8_t* q, float* s, void* h,
                               float* az, int wc, cudaStream_t st) {
  ln_mod_quant_kernel<NV><<<(rows + 7) / 8, 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(x), rows, eps, shift, scale, rpi, ms, q, s,
      static_cast<__nv_bfloat16*>(h), az, wc);
  return cudaGetLastError();
}

cudaError_t launch_ln_mod_quant(const void* x, int rows, int d, float eps, const float* shift,
                                const float* scale, int rows_per_item, int mod_stride, int8_t* q,
                                float* s, void* h_out, float* absmax_zero, int write_codes,
                                cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
#define H3B_LN_CASE(nv) \
  case nv:              \
    return ln_dispatch<nv>(x, rows, eps, shift, scale, rows_per_item, mod_stride, q, s, h_out, absmax_zero, write_codes, st);
  switch (d / 256) {
    H3B_LN_CASE(1) H3B_LN_CASE(2) H3B_LN_CASE(3) H3B_LN_CASE(4) H3B_LN_CASE(5) H3B_LN_CASE(6)
    H3B_LN_CASE(7) H3B_LN_CASE(8) H3B_LN_CASE(9) H3B_LN_CASE(10) H3B_LN_CASE(11) H3B_LN_CASE(12)
    H3B_LN_CASE(13) H3B_LN_CASE(14) H3B_LN_CASE(15) H3B_LN_CASE(16) H3B_LN_CASE(17) H3B_LN_CASE(18)
    H3B_LN_CASE(19) H3B_LN_CASE(20) H3B_LN_CASE(21) H3B_LN_CASE(22) H3B_LN_CASE(23) H3B_LN_CASE(24)
    H3B_LN_CASE(25) H3B_LN_CASE(26) H3B_LN_CASE(27) H3B_LN_CASE(28) H3B_LN_CASE(29) H3B_LN_CASE(30)
    H3B_LN_CASE(31) H3B_LN_CASE(32)
    default:
      return cudaErrorInvalidValue;
  }
#undef H3B_LN_CASE
}

cudaError_t launch_quant_rows_bf16(const void* h, int rows, int cols, const float* absmax,
                                   int8_t* q, float* s, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  quant_rows_kernel<__nv_bfloat16><<<rows, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(h), cols,
                                                        absmax, q, s);
  return cudaGetLastError();
}

cudaError_t launch_quant_rows_f32(const float* w, int rows, int cols, int8_t* q, float* s,
                                  cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  quant_rows_kernel<float><<<rows, 256, 0, st>>>(w, cols, nullptr, q, s);
  return cudaGetLastError();
}

static int grid_for(long long n, int sms) {
  const long long want = (n + 255) / 256;
  const long long cap = (long long)sms * 16;
  return (int)(want < cap ? (want > 0 ? want : 1) : cap);
}

cudaError_t launch_token_pair(const void* x, void* xm, void* xm2, long long lines, int W, int d,
                              int sms, cudaStream_t st) {
  const long long n = lines * (W / 2) * (d / 8);
  if (n == 0) return cudaSuccess;
  token_pair_kernel<<<grid_for(n, sms), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(x), static_cast<__nv_bfloat16*>(xm),
      static_cast<__nv_bfloat16*>(xm2), n, W / 2, d / 8);
  return cudaGetLastError();
}

cudaError_t launch_token_unpair(const void* x, const void* xm, const void* ym, void* out,
                                long long lines, int W, int d, int sms, cudaStream_t st) {
  const long long n = lines * W * (d / 8);
  if (n == 0) return cudaSuccess;
  token_unpair_kernel<<<grid_for(n, sms), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(xm),
      static_cast<const __nv_bfloat16*>(ym), static_cast<__nv_bfloat16*>(out), n, W, d / 8);
  return cudaGetLastError();
}

cudaError_t launch_rope_table(float2* tab, int T, int H, int W, int rt, int rh, int rw,
                              double theta, cudaStream_t st) {
  const int n = T * (rt / 2) + H * (rh / 2) + W * (rw / 2);
  rope_table_kernel<<<(n + 255) / 256, 256, 0, st>>>(tab, T, H, W, rt, rh, rw, theta);
  return cudaGetLastError();
}

}  // namespace h3b
