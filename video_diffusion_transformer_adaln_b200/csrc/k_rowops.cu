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
// The same decision without a division per element: t = v * RN(1/scale)
// differs from RN(v / scale) by less than 2^-15.4 for |t| <= 127.5, so when t
// is farther than 2^-14 from a half-integer both round to the same integer;
// only then-near ties take the correctly rounded division. Bit-identical to
// quant_code for every input (absmax > 0).
constexpr float kTieGuard = 0.5f - 1.0f / 16384.0f;
__device__ __forceinline__ int quant_code_fast(float v, float scale, float rcp) {
  float t = v * rcp;
  float c = rintf(t);
  if (fabsf(t - c) > kTieGuard) c = rintf(__fdiv_rn(v, scale));
  return max(-127, min(127, (int)c));
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

// One warp per output row j; the row's d/8 16-byte vectors (NV per lane) are
// all requested before any is used, so each warp keeps its whole row in flight.
template <int NV>
__global__ void __launch_bounds__(256) adaln_gemv_kernel(const __nv_bfloat16* __restrict__ W,
                                                         const float* __restrict__ bias,
                                                         const float* __restrict__ c, int B,
                                                         float* __restrict__ mod) {
  constexpr int d = NV * 256;
  extern __shared__ float cs[];  // [B][d]
  for (int i = threadIdx.x; i < B * d; i += blockDim.x) cs[i] = c[i];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x * 8 + warp;
  const bool valid = j < 6 * d;
  const uint4* wr = reinterpret_cast<const uint4*>(W + (size_t)(valid ? j : 0) * d);
  uint4 w4[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) w4[i] = __ldcs(wr + lane + 32 * i);
  __syncthreads();
  if (!valid) return;
  float acc[kGemvMaxB];
#pragma unroll
  for (int b = 0; b < kGemvMaxB; ++b) acc[b] = 0.0f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const uint32_t ww[4] = {w4[i].x, w4[i].y, w4[i].z, w4[i].w};
    const int v = lane + 32 * i;
#pragma unroll
    for (int b = 0; b < kGemvMaxB; ++b) {
      if (b >= B) break;
      const float4 c0 = *reinterpret_cast<const float4*>(cs + b * d + v * 8);
      const float4 c1 = *reinterpret_cast<const float4*>(cs + b * d + v * 8 + 4);
      float a = acc[b];
      a = fmaf(bf16_lo(ww[0]), c0.x, a); a = fmaf(bf16_hi(ww[0]), c0.y, a);
      a = fmaf(bf16_lo(ww[1]), c0.z, a); a = fmaf(bf16_hi(ww[1]), c0.w, a);
      a = fmaf(bf16_lo(ww[2]), c1.x, a); a = fmaf(bf16_hi(ww[2]), c1.y, a);
      a = fmaf(bf16_lo(ww[3]), c1.z, a); a = fmaf(bf16_hi(ww[3]), c1.w, a);
      acc[b] = a;
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
// Fused LayerNorm + modulation + per-row int8 quantization. A row of
// d = 8 * VPT * G channels is held in registers by a group of G threads
// (VPT 16-byte vectors each); a 256-thread block serves 256 / G rows.
//   y = (x - mean) * rsqrt(var + eps)          (fp32, two-pass variance)
//   h = bf16(y * (1 + scale) + shift)
//   s = absmax(h) / 127, q = rint(h / s)       (binary32 decision)
// ---------------------------------------------------------------------------
template <int G>
__device__ __forceinline__ float group_sum(float v, float* red) {
  v = warp_sum(v);
  if (G == 32) return v;
  constexpr int NW = G / 32;
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[warp] = v;
  __syncthreads();
  const int first = (warp / NW) * NW;
  float t = 0.0f;
#pragma unroll
  for (int i = 0; i < NW; ++i) t += red[first + i];
  __syncthreads();
  return t;
}
template <int G>
__device__ __forceinline__ float group_max(float v, float* red) {
  v = warp_max(v);
  if (G == 32) return v;
  constexpr int NW = G / 32;
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[warp] = v;
  __syncthreads();
  const int first = (warp / NW) * NW;
  float t = 0.0f;
#pragma unroll
  for (int i = 0; i < NW; ++i) t = fmaxf(t, red[first + i]);
  __syncthreads();
  return t;
}

__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t u) { return make_float2(bf16_lo(u), bf16_hi(u)); }

template <int VPT, int G>
__global__ void __launch_bounds__(256) ln_mod_quant_kernel(
    const __nv_bfloat16* __restrict__ x, int rows, float eps, const float* __restrict__ shift,
    const float* __restrict__ scale, int rows_per_item, int mod_stride, int8_t* __restrict__ q,
    float* __restrict__ s, __nv_bfloat16* __restrict__ h_out, float* __restrict__ absmax_zero,
    int write_codes) {
  constexpr int RPB = 256 / G;
  constexpr int d = VPT * G * 8;
  __shared__ float red[8];
  const int gt = threadIdx.x % G;
  const int row = blockIdx.x * RPB + threadIdx.x / G;
  const bool valid = row < rows;
  const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)(valid ? row : 0) * d);
  uint4 v[VPT];
#pragma unroll
  for (int i = 0; i < VPT; ++i) v[i] = valid ? __ldcs(xr + gt + G * i) : make_uint4(0, 0, 0, 0);

  float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    acc = __fadd2_rn(acc, bf16x2_to_f2(v[i].x));
    acc = __fadd2_rn(acc, bf16x2_to_f2(v[i].y));
    acc = __fadd2_rn(acc, bf16x2_to_f2(v[i].z));
    acc = __fadd2_rn(acc, bf16x2_to_f2(v[i].w));
  }
  const float mean = group_sum<G>(acc.x + acc.y, red) * (1.0f / d);
  const float2 nmean = make_float2(-mean, -mean);
  acc = make_float2(0.0f, 0.0f);
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const uint32_t u[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 c = __fadd2_rn(bf16x2_to_f2(u[e]), nmean);
      acc = __ffma2_rn(c, c, acc);
    }
  }
  const float rstd = 1.0f / sqrtf(group_sum<G>(acc.x + acc.y, red) * (1.0f / d) + eps);
  const float2 rstd2 = make_float2(rstd, rstd);

  const int item = (valid ? row : 0) / rows_per_item;
  const float2* sh2 = reinterpret_cast<const float2*>(shift + (size_t)item * mod_stride);
  const float2* sc2 = reinterpret_cast<const float2*>(scale + (size_t)item * mod_stride);
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int c0 = (gt + G * i) * 4;  // float2 index of the vector's first channel pair
    uint32_t u[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 sh = __ldg(sh2 + c0 + e);
      const float2 sc = __ldg(sc2 + c0 + e);
      const float2 y = __fmul2_rn(__fadd2_rn(bf16x2_to_f2(u[e]), nmean), rstd2);
      const float2 h = __ffma2_rn(y, make_float2(1.0f + sc.x, 1.0f + sc.y), sh);
      u[e] = pack_bf16x2(h.x, h.y);
      amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(u[e])), fabsf(bf16_hi(u[e]))));
    }
    v[i] = make_uint4(u[0], u[1], u[2], u[3]);
  }
  amax = group_max<G>(amax, red);
  if (!valid) return;
  if (h_out) {
    uint4* hr = reinterpret_cast<uint4*>(h_out + (size_t)row * d);
#pragma unroll
    for (int i = 0; i < VPT; ++i) hr[gt + G * i] = v[i];
  }
  if (absmax_zero && gt == 0) absmax_zero[row] = 0.0f;
  if (!write_codes) return;
  const float sc = __fdiv_rn(amax, 127.0f);
  const float rcp = __frcp_rn(sc);
  if (gt == 0) s[row] = sc;
  uint2* qr = reinterpret_cast<uint2*>(q + (size_t)row * d);
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const uint32_t u[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
    int c[8];
    if (!(rcp < INFINITY)) {  // absmax == 0 (codes 0) or a subnormal scale: exact division
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        c[2 * e] = quant_code(bf16_lo(u[e]), sc, amax);
        c[2 * e + 1] = quant_code(bf16_hi(u[e]), sc, amax);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        c[2 * e] = quant_code_fast(bf16_lo(u[e]), sc, rcp);
        c[2 * e + 1] = quant_code_fast(bf16_hi(u[e]), sc, rcp);
      }
    }
    qr[gt + G * i] = make_uint2(pack4_i8(c[0], c[1], c[2], c[3]), pack4_i8(c[4], c[5], c[6], c[7]));
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
  const float rcp = __frcp_rn(sc);
  if (threadIdx.x == 0) s[row] = sc;
  uint2* qr = reinterpret_cast<uint2*>(q + (size_t)row * cols);
  constexpr int U = 4;  // vectors in flight per thread
  for (int v0 = threadIdx.x; v0 < nvec; v0 += U * blockDim.x) {
    float f[U][8];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + u * blockDim.x;
      if (v < nvec) load8<T>(r + v * 8, f[u]);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + u * blockDim.x;
      if (v >= nvec) break;
      int c[8];
#pragma unroll
      for (int e = 0; e < 8; ++e)
        c[e] = (rcp < INFINITY) ? quant_code_fast(f[u][e], sc, rcp) : quant_code(f[u][e], sc, amax);
      qr[v] = make_uint2(pack4_i8(c[0], c[1], c[2], c[3]), pack4_i8(c[4], c[5], c[6], c[7]));
    }
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
template <int NV>
static cudaError_t gemv_dispatch(const void* W, const float* bias, const float* c, int B, float* mod,
                                 cudaStream_t st) {
  constexpr int d = NV * 256;
  const size_t smem = (size_t)B * d * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(adaln_gemv_kernel<NV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  adaln_gemv_kernel<NV><<<(6 * d + 7) / 8, 256, smem, st>>>(static_cast<const __nv_bfloat16*>(W), bias, c, B,
                                                            mod);
  return cudaGetLastError();
}

cudaError_t launch_adaln_gemv(const void* W, const float* bias, const float* c, int B, int d,
                              float* mod, cudaStream_t st) {
  if (B > kGemvMaxB || d % 256 != 0) return cudaErrorInvalidValue;
#define H3B_GV(nv) \
  case nv:         \
    return gemv_dispatch<nv>(W, bias, c, B, mod, st);
  switch (d / 256) {
    H3B_GV(1) H3B_GV(2) H3B_GV(3) H3B_GV(4) H3B_GV(5) H3B_GV(6) H3B_GV(7) H3B_GV(8)
    H3B_GV(9) H3B_GV(10) H3B_GV(11) H3B_GV(12) H3B_GV(13) H3B_GV(14) H3B_GV(15) H3B_GV(16)
    H3B_GV(17) H3B_GV(18) H3B_GV(19) H3B_GV(20) H3B_GV(21) H3B_GV(22) H3B_GV(23) H3B_GV(24)
    H3B_GV(25) H3B_GV(26) H3B_GV(27) H3B_GV(28) H3B_GV(29) H3B_GV(30) H3B_GV(31) H3B_GV(32)
    default:
      return cudaErrorInvalidValue;
  }
#undef H3B_GV
}

template <int VPT, int G>
static cudaError_t ln_dispatch(const void* x, int rows, float eps, const float* shift,
                               const float* scale, int rpi, int ms, int8_t* q, float* s, void* h,
                               float* az, int wc, cudaStream_t st) {
  constexpr int RPB = 256 / G;
  ln_mod_quant_kernel<VPT, G><<<(rows + RPB - 1) / RPB, 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(x), rows, eps, shift, scale, rpi, ms, q, s,
      static_cast<__nv_bfloat16*>(h), az, wc);
  return cudaGetLastError();
}

// d = 256 k: a row is split over G = 128 (k % 4 == 0), 64 (k % 2 == 0) or 32
// threads holding VPT = 32 k / G vectors of 8 channels each.
cudaError_t launch_ln_mod_quant(const void* x, int rows, int d, float eps, const float* shift,
                                const float* scale, int rows_per_item, int mod_stride, int8_t* q,
                                float* s, void* h_out, float* absmax_zero, int write_codes,
                                cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  const int k = d / 256;
#define H3B_LN(vpt, g) \
  return ln_dispatch<vpt, g>(x, rows, eps, shift, scale, rows_per_item, mod_stride, q, s, h_out, absmax_zero, write_codes, st)
  if (k % 4 == 0) {
    switch (k / 4) {
      case 1: H3B_LN(1, 128); case 2: H3B_LN(2, 128); case 3: H3B_LN(3, 128); case 4: H3B_LN(4, 128);
      case 5: H3B_LN(5, 128); case 6: H3B_LN(6, 128); case 7: H3B_LN(7, 128); case 8: H3B_LN(8, 128);
      default: return cudaErrorInvalidValue;
    }
  } else if (k % 2 == 0) {
    switch (k / 2) {
      case 1: H3B_LN(1, 64); case 3: H3B_LN(3, 64); case 5: H3B_LN(5, 64); case 7: H3B_LN(7, 64);
      case 9: H3B_LN(9, 64); case 11: H3B_LN(11, 64); case 13: H3B_LN(13, 64); case 15: H3B_LN(15, 64);
      default: return cudaErrorInvalidValue;
    }
  } else {
    switch (k) {
      case 1: H3B_LN(1, 32); case 3: H3B_LN(3, 32); case 5: H3B_LN(5, 32); case 7: H3B_LN(7, 32);
      case 9: H3B_LN(9, 32); case 11: H3B_LN(11, 32); case 13: H3B_LN(13, 32); case 15: H3B_LN(15, 32);
      case 17: H3B_LN(17, 32); case 19: H3B_LN(19, 32); case 21: H3B_LN(21, 32); case 23: H3B_LN(23, 32);
      case 25: H3B_LN(25, 32); case 27: H3B_LN(27, 32); case 29: H3B_LN(29, 32); case 31: H3B_LN(31, 32);
      default: return cudaErrorInvalidValue;
    }
  }
#undef H3B_LN
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
