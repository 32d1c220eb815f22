// Memory-bound kernels of the block: AdaLN modulation GEMV, the fused
// LayerNorm + modulation + per-row int8 quantizer, the quant-only pass, the
// per-output-channel weight quantizer, token pairing, the residual-reuse delta
// and its re-application, and the RoPE table.
//
// All of them stream with 16-byte vector accesses and keep no state between
// launches. The GEMV gives a warp one output row; the LN quantizer spreads a
// row over 1-8 warps (warp shuffles, then one shared slot per warp) and stages
// its next rows with cp.async; the quant pass and the elementwise kernels
// stream whole rows or flat ranges.
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

// Bounds word of this file's kernels in the checked build (H3B_IDX_OK); the host
// reads it together with the device error word.
__device__ unsigned g_h3b_rowops_bounds;

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
// Eight codes of one 16-byte bf16 vector without a branch per element:
// a = fma(v, RN(1/scale), 1.5 * 2^23) rounds the exact product p = v * RN(1/scale)
// to the nearest integer c (ties to even) in the low mantissa bits, whose low
// byte is the int8 code (|p| <= 127.5 never yields -128), and
// dd = fma(v, RN(1/scale), -c) is p - c to within 2^-25. p differs from v / scale
// by at most 127.5 * 2^-24 = 2^-17 and RN(v / scale) from v / scale by at most
// 2^-18, so where |dd| <= 0.5 - 2^-14 the binary32 decision rint(RN(v / scale))
// is c. The largest |dd| is tracked and the dd are returned; if an element lies
// closer to a half-integer the caller patches those elements with quant8_slow.
__device__ __forceinline__ uint2 quant8_fast(uint4 v, float rcp, float& worst, float2 (&dds)[4]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  const float2 r2 = make_float2(rcp, rcp), M2 = make_float2(12582912.0f, 12582912.0f);
  const float2 nM2 = make_float2(-12582912.0f, -12582912.0f);
  uint32_t b[8];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 x = make_float2(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xFFFF0000u));
    const float2 a = __ffma2_rn(x, r2, M2);
    const float2 c = __fadd2_rn(a, nM2);  // exact
    const float2 dd = __ffma2_rn(x, r2, make_float2(-c.x, -c.y));
    worst = fmaxf(worst, fmaxf(fabsf(dd.x), fabsf(dd.y)));
    dds[e] = dd;
    b[2 * e] = __float_as_uint(a.x);
    b[2 * e + 1] = __float_as_uint(a.y);
  }
  const uint32_t lo = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
  const uint32_t hi = __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410);
  return make_uint2(lo, hi);
}
__device__ __forceinline__ uint32_t pack4_i8(int a, int b, int c, int d) {
  return (uint32_t)(a & 0xFF) | ((uint32_t)(b & 0xFF) << 8) | ((uint32_t)(c & 0xFF) << 16) |
         ((uint32_t)(d & 0xFF) << 24);
}
// Scales below this take the division for every element (quant8_slow); at or
// above it RN(1/scale) is finite and every quantity below is a normal number.
constexpr float kMinFastScale = 0x1p-100f;
// The codes of a vector whose fast path saw a near tie, patched element by
// element. On bf16 rows a few elements in a thousand have v * RN(1/scale) within
// 2^-14 of a half-integer (bf16 values over a bf16 absmax put many quotients on
// or next to one, most of them exactly), so only those elements, found from the
// fast path's distances dd, are decided again, without a division: with h the
// half-integer next to the product and r = v - h * scale,
//   r is exact in binary32 (one fma): v and h * scale are multiples of
//     ulp(scale) / 2, and |r| < 2^-13 scale (|v / scale - h| < 2^-14 + 2^-17)
//     needs fewer than 13 bits of them;
//   RN(v / scale) == h exactly when |r| <= scale * ulp(h) / 2 (h has at most 9
//     significant bits, so a quotient midway to h's neighbour rounds to h; the
//     smaller spacing just below |h| = 0.5 changes no code), and then the code
//     is the even integer next to h (rint(h));
//   otherwise the code is h + 0.5 when r > 0 and h - 0.5 when r < 0.
// A zero, subnormal or tiny scale (the whole row) takes the division itself.
// kGivenDd: the fast path's dd are passed in (d0..d3); otherwise they are
// recomputed here, which keeps the caller's live registers down.
template <bool kGivenDd>
__device__ __noinline__ uint2 quant8_slow(uint4 v, float scale, float rcp, float absmax, uint2 code, float2 d0,
                                         float2 d1, float2 d2, float2 d3) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  if (!(scale >= kMinFastScale)) {
    int c[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      c[2 * e] = quant_code(bf16_lo(w[e]), scale, absmax);
      c[2 * e + 1] = quant_code(bf16_hi(w[e]), scale, absmax);
    }
    return make_uint2(pack4_i8(c[0], c[1], c[2], c[3]), pack4_i8(c[4], c[5], c[6], c[7]));
  }
  uint32_t word[2] = {code.x, code.y};
  const float given[8] = {d0.x, d0.y, d1.x, d1.y, d2.x, d2.y, d3.x, d3.y};
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float x = (e & 1) ? bf16_hi(w[e >> 1]) : bf16_lo(w[e >> 1]);
    const float c0 = fmaf(x, rcp, 12582912.0f) - 12582912.0f;  // as quant8_fast
    const float dd = kGivenDd ? given[e] : fmaf(x, rcp, -c0);
    if (fabsf(dd) > kTieGuard) {
      const float h = c0 + copysignf(0.5f, dd);
      const float r = fmaf(-h, scale, x);
      const float us = __uint_as_float((__float_as_uint(h) & 0x7F800000u) - (24u << 23)) * scale;
      const float c = fabsf(r) <= us ? rintf(h) : (r > 0.0f ? h + 0.5f : h - 0.5f);
      const uint32_t byte = (uint32_t)max(-127, min(127, (int)c)) & 0xFFu;
      const int k = e >> 2, sh = 8 * (e & 3);
      word[k] = (word[k] & ~(0xFFu << sh)) | (byte << sh);
    }
  }
  return make_uint2(word[0], word[1]);
}
// Eight codes of one bf16 vector, bit-identical to quant_code on each element.
template <bool kGivenDd>
__device__ __forceinline__ uint2 quant8(uint4 v, float scale, float rcp, float absmax) {
  float worst = scale >= kMinFastScale ? 0.0f : 1.0f;  // zero, tiny or NaN scale: the slow path decides
  float2 dd[4];
  uint2 code = quant8_fast(v, rcp, worst, dd);
  if (worst > kTieGuard) code = quant8_slow<kGivenDd>(v, scale, rcp, absmax, code, dd[0], dd[1], dd[2], dd[3]);
  return code;
}

// ---------------------------------------------------------------------------
// AdaLN modulation Linear: mod[b][j] = sum_k W[j][k] c[b][k] + bias[j].
// One warp per output row j, all batch items at once (W is read once); c is
// staged in shared memory as fp32.
// ---------------------------------------------------------------------------
constexpr int kGemvMaxB = 8;

// Persistent blocks: c is staged in shared memory once per block, then each
// warp walks groups of kGemvRows consecutive output rows, j0 = (block * 8 +
// warp) * kGemvRows + k * (blocks * 8 * kGemvRows). A group is read in chunks of
// kGemvChunk 16-byte vectors per lane and row, all requested before any is used;
// each c vector read from shared memory then serves all rows of the group, so
// shared-memory traffic is a quarter of one row at a time.
struct RopeTableArgs {
  float2* tab;  // nullptr: no table this launch
  int T, H, W, rt, rh, rw;
  double theta;
};

__device__ void rope_table_entries(const RopeTableArgs& r, int first, int stride);

constexpr int kGemvRows = 4;
constexpr int kGemvChunk = 4;

// MB: the largest batch the instance handles (1, or kGemvMaxB), so one latent keeps few accumulators.
template <int NV, int MB>
__global__ void __launch_bounds__(256) adaln_gemv_kernel(const __nv_bfloat16* __restrict__ W,
                                                         const float* __restrict__ bias,
                                                         const float* __restrict__ c, int B,
                                                         float* __restrict__ mod, const RopeTableArgs rope,
                                                         int gemv_blocks) {
  griddep_wait();
  griddep_launch_dependents();
  constexpr int d = NV * 256;
  constexpr int R = kGemvRows, CH = kGemvChunk;
  if ((int)blockIdx.x >= gemv_blocks) {  // trailing blocks fill the RoPE table
    rope_table_entries(rope, ((int)blockIdx.x - gemv_blocks) * blockDim.x + threadIdx.x,
                       ((int)gridDim.x - gemv_blocks) * blockDim.x);
    return;
  }
  extern __shared__ float cs[];  // [B][d]
  for (int i = threadIdx.x; i < B * d; i += blockDim.x) cs[i] = c[i];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int j0 = (blockIdx.x * 8 + warp) * R; j0 < 6 * d; j0 += gemv_blocks * 8 * R) {  // warp-uniform
    float acc[R][MB];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int b = 0; b < MB; ++b) acc[r][b] = 0.0f;
#pragma unroll 1
    for (int i0 = 0; i0 < NV; i0 += CH) {
      uint4 w4[R][CH];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const uint4* wr = reinterpret_cast<const uint4*>(W + (size_t)(j0 + r) * d);
#pragma unroll
        for (int i = 0; i < CH; ++i)
          if (i0 + i < NV) w4[r][i] = __ldcs(wr + lane + 32 * (i0 + i));
      }
#pragma unroll
      for (int i = 0; i < CH; ++i) {
        if (i0 + i >= NV) break;
        const int v = lane + 32 * (i0 + i);
#pragma unroll
        for (int b = 0; b < MB; ++b) {
          if (b >= B) break;
          const float4 c0 = *reinterpret_cast<const float4*>(cs + b * d + v * 8);
          const float4 c1 = *reinterpret_cast<const float4*>(cs + b * d + v * 8 + 4);
#pragma unroll
          for (int r = 0; r < R; ++r) {
            const uint32_t ww[4] = {w4[r][i].x, w4[r][i].y, w4[r][i].z, w4[r][i].w};
            float a = acc[r][b];
            a = fmaf(bf16_lo(ww[0]), c0.x, a); a = fmaf(bf16_hi(ww[0]), c0.y, a);
            a = fmaf(bf16_lo(ww[1]), c0.z, a); a = fmaf(bf16_hi(ww[1]), c0.w, a);
            a = fmaf(bf16_lo(ww[2]), c1.x, a); a = fmaf(bf16_hi(ww[2]), c1.y, a);
            a = fmaf(bf16_lo(ww[3]), c1.z, a); a = fmaf(bf16_hi(ww[3]), c1.w, a);
            acc[r][b] = a;
          }
        }
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int b = 0; b < MB; ++b) {
        if (b >= B) break;
        const float sum = warp_sum(acc[r][b]);
        const int j = j0 + r;
        if (lane == 0 && H3B_IDX_OK((long long)b * 6 * d + j, (long long)B * 6 * d, &g_h3b_rowops_bounds))
          mod[(size_t)b * 6 * d + j] = sum + (bias ? bias[j] : 0.0f);
      }
  }
}

// ---------------------------------------------------------------------------
// Fused LayerNorm + modulation + per-row int8 quantization.
//   y = (x - mean) * rsqrt(var + eps)          (fp32, two-pass variance)
//   h = bf16(y * (1 + scale) + shift)
//   s = absmax(h) / 127, q = rint(h / s)       (binary32 decision)
// A row of d = 256 NV channels (32 NV 16-byte vectors) is held in registers by
// tpr = 32 NV / VPT threads, VPT vectors each; a block holds rpp = blockDim /
// tpr rows at a time and walks its share of the rows in passes of rpp rows,
// all of one batch item, staging the next pass's rows in shared memory with
// cp.async while it works on the current ones. The item's (1 + scale, shift) pairs sit in shared
// memory, loaded when the item changes, laid out [4][vectors] so that a warp's
// 16-byte reads of one channel pair per vector fall in distinct banks.
// Reductions: warp shuffles, then one shared slot per warp and a named barrier
// of the row group (slots alternate between passes, so no barrier guards their
// reuse; a one-warp row needs only the warp's own sync). The row absmax is taken
// in fp32 before the bf16 rounding: rounding to nearest is monotone, so the
// rounded fp32 absmax is the absmax of the rounded h.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t u) { return make_float2(bf16_lo(u), bf16_hi(u)); }
__device__ __forceinline__ float max3f_row(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

constexpr int kLnMaxWarps = 32;

// Named barrier `id` over `count` threads (a multiple of 32).
__device__ __forceinline__ void named_barrier(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// 16-byte asynchronous copy global -> shared (L2 only), and the wait for all of
// this thread's outstanding copies.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Threads per block of the LN quantizer: the row's tpr threads, times as many
// rows as fit in 512 threads (or one row of up to 1024 threads).
__host__ __device__ constexpr int ln_block(int vpr, int vpt) {
  return vpr / vpt >= 512 ? vpr / vpt : (512 / (vpr / vpt)) * (vpr / vpt);
}

// VPT vectors per thread; NV > 0 fixes the row at 32 NV vectors (d = 256 NV) at
// compile time, so that strides and the block shape are constants; NV = 0 takes
// the row length from vpr_arg.
template <int VPT, int NV>
__global__ void __launch_bounds__(1024, 1) ln_mod_quant_kernel(
    const __nv_bfloat16* __restrict__ x, int rows, int vpr_arg, float eps, const float* __restrict__ shift,
    const float* __restrict__ scale, int rows_per_item, int mod_stride, int8_t* __restrict__ q,
    float* __restrict__ s, __nv_bfloat16* __restrict__ h_out, float* __restrict__ absmax_zero,
    int write_codes) {
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ float4 modp[];  // [4][vpr]: (1+sc[2c], 1+sc[2c+1], sh[2c], sh[2c+1]), c = 4 vec + e
  // then the staging rows of the next pass: [rpp][vpr] 16-byte vectors, each written and read
  // back by the same thread (cp.async), so no barrier guards them
  __shared__ float red[2][3][kLnMaxWarps];
  const int vpr = NV ? 32 * NV : vpr_arg;
  const int nthreads = NV ? ln_block(32 * NV, VPT) : (int)blockDim.x;
  const int tpr = vpr / VPT;
  const int rpp = nthreads / tpr;
  const int sub = threadIdx.x / tpr;
  const int t = threadIdx.x - sub * tpr;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wpr = tpr >> 5, w0 = sub * wpr;
  const float inv_d = 1.0f / (float)(vpr * 8);
  const int items = (rows + rows_per_item - 1) / rows_per_item;
  const unsigned gpi = (unsigned)((rows_per_item + rpp - 1) / rpp);
  const unsigned total = (unsigned)items * gpi;  // passes; at most rows, so 32 bits suffice
  int cur = -1, par = 0;
  unsigned item = blockIdx.x / gpi, g_in = blockIdx.x % gpi;  // pass = (item, pass within item)
  uint4* stage = reinterpret_cast<uint4*>(modp + 4 * vpr) + (size_t)sub * vpr;
  // row-group barrier: a named barrier per group (ids 1..rpp), or the warp itself
  auto group_sync = [&]() {
    if (wpr > 1) named_barrier(1 + sub, tpr);
    else __syncwarp();
  };
  // this thread's vectors of its row in pass (it, gi) -> staging, when that row exists
  auto prefetch = [&](unsigned gg, unsigned it, unsigned gi) {
    const int r = (int)gi * rpp + sub, rw = (int)it * rows_per_item + r;
    if (gg >= total || r >= rows_per_item || rw >= rows) return;
    const uint4* src = reinterpret_cast<const uint4*>(x) + (size_t)rw * vpr;
#pragma unroll
    for (int i = 0; i < VPT; ++i)
      if (H3B_IDX_OK((long long)rw * vpr + t + tpr * i, (long long)rows * vpr, &g_h3b_rowops_bounds))
        cp_async16(stage + t + tpr * i, src + t + tpr * i);
  };
  prefetch(blockIdx.x, item, g_in);
  cp_async_commit();
  for (unsigned g = blockIdx.x; g < total; g += gridDim.x) {
    if ((int)item != cur) {  // block-uniform
      __syncthreads();
      const float2* sc2 = reinterpret_cast<const float2*>(scale + (size_t)item * mod_stride);
      const float2* sh2 = reinterpret_cast<const float2*>(shift + (size_t)item * mod_stride);
      for (int c = threadIdx.x; c < 4 * vpr; c += nthreads) {
        const float2 a = __ldg(sc2 + c), b = __ldg(sh2 + c);
        modp[(c & 3) * vpr + (c >> 2)] = make_float4(1.0f + a.x, 1.0f + a.y, b.x, b.y);
      }
      cur = item;
      __syncthreads();
    }
    const int r_in = (int)g_in * rpp + sub;
    const int row = (int)item * rows_per_item + r_in;
    const bool valid = r_in < rows_per_item && row < rows;
    cp_async_wait_all();
    uint4 v[VPT];
#pragma unroll
    for (int i = 0; i < VPT; ++i) v[i] = valid ? stage[t + tpr * i] : make_uint4(0, 0, 0, 0);

    float* rd = red[par][0];
    par ^= 1;
    // the row in fp32 pairs, converted once
    float2 f[VPT * 4];
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      f[4 * i + 0] = bf16x2_to_f2(v[i].x);
      f[4 * i + 1] = bf16x2_to_f2(v[i].y);
      f[4 * i + 2] = bf16x2_to_f2(v[i].z);
      f[4 * i + 3] = bf16x2_to_f2(v[i].w);
    }
    // the staged vectors are in registers now: start the next pass's loads
    unsigned n_in = g_in + gridDim.x, n_item = item;
    while (n_in >= gpi) {  // (item, pass within item) of the next pass, without a division
      n_in -= gpi;
      ++n_item;
    }
    prefetch(g + gridDim.x, n_item, n_in);
    cp_async_commit();
    float2 acc = f[0];
#pragma unroll
    for (int e = 1; e < VPT * 4; ++e) acc = __fadd2_rn(acc, f[e]);
    float r = warp_sum(acc.x + acc.y);
    if (lane == 0) rd[warp] = r;
    group_sync();
    r = 0.0f;
    for (int k = 0; k < wpr; ++k) r += rd[w0 + k];
    const float mean = r * inv_d;
    const float2 nmean = make_float2(-mean, -mean);

#pragma unroll
    for (int e = 0; e < VPT * 4; ++e) f[e] = __fadd2_rn(f[e], nmean);  // x - mean
    acc = __fmul2_rn(f[0], f[0]);
#pragma unroll
    for (int e = 1; e < VPT * 4; ++e) acc = __ffma2_rn(f[e], f[e], acc);
    r = warp_sum(acc.x + acc.y);
    if (lane == 0) rd[kLnMaxWarps + warp] = r;
    group_sync();
    r = 0.0f;
    for (int k = 0; k < wpr; ++k) r += rd[kLnMaxWarps + w0 + k];
    const float rstd = 1.0f / sqrtf(r * inv_d + eps);
    const float2 rstd2 = make_float2(rstd, rstd);

    // h = bf16((x - mean) * rstd * (1 + scale) + shift); max |h| in fp32 before the rounding
    float am = 0.0f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int vec = t + tpr * i;
      uint32_t u[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float4 m = modp[e * vpr + vec];
        const float2 y = __fmul2_rn(f[4 * i + e], rstd2);
        const float2 h = __ffma2_rn(y, make_float2(m.x, m.y), make_float2(m.z, m.w));
        u[e] = pack_bf16x2(h.x, h.y);
        am = max3f_row(am, fabsf(h.x), fabsf(h.y));
      }
      v[i] = make_uint4(u[0], u[1], u[2], u[3]);
    }
    float amax = warp_max(am);
    if (lane == 0) rd[2 * kLnMaxWarps + warp] = amax;
    group_sync();
    amax = 0.0f;
    for (int k = 0; k < wpr; ++k) amax = fmaxf(amax, rd[2 * kLnMaxWarps + w0 + k]);
    amax = round_bf16(amax);  // = the max of the rounded |h|
    if (valid) {
      if (h_out) {
        uint4* hr = reinterpret_cast<uint4*>(h_out) + (size_t)row * vpr;
#pragma unroll
        for (int i = 0; i < VPT; ++i)
          if (H3B_IDX_OK((long long)row * vpr + t + tpr * i, (long long)rows * vpr, &g_h3b_rowops_bounds))
            hr[t + tpr * i] = v[i];
      }
      if (absmax_zero && t == 0 && H3B_IDX_OK(row, rows, &g_h3b_rowops_bounds)) absmax_zero[row] = 0.0f;
      if (write_codes) {
        const float sc = __fdiv_rn(amax, 127.0f);
        const float rcp = __frcp_rn(sc);
        if (t == 0 && H3B_IDX_OK(row, rows, &g_h3b_rowops_bounds)) s[row] = sc;
        uint2* qr = reinterpret_cast<uint2*>(q) + (size_t)row * vpr;
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
          const uint2 code = quant8<true>(v[i], sc, rcp, amax);
          if (H3B_IDX_OK((long long)row * vpr + t + tpr * i, (long long)rows * vpr, &g_h3b_rowops_bounds))
            qr[t + tpr * i] = code;
        }
      }
    }
    item = n_item;
    g_in = n_in;
  }
  cp_async_wait_all();
}

// Per-row quantization with each row's absmax already known: a block covers
// whole rows (rpb rows of vpr 16-byte vectors, rpb * vpr <= 4096 unless one row
// is longer, rpb <= 32). Each thread walks the block's vectors in rounds of
// four, loading the next round into the other of two register sets before it
// quantizes the current one (the first round's loads are issued before the
// scales are derived), so eight vectors per thread are in flight. Each row's
// scale and its reciprocal are derived once, into shared memory.
constexpr int kQuantMaxRowsPerBlock = 32;
constexpr int kQuantThreads = 256;
// VPR > 0 fixes the row at VPR vectors at compile time (the widths of the block's O and
// G rows); VPR = 0 takes it from vpr_arg.
template <int VPR>
__global__ void __launch_bounds__(kQuantThreads, 4) quant_rows_known_absmax_kernel(const __nv_bfloat16* __restrict__ in,
                                                                               int rows, int vpr_arg, int rpb,
                                                                               const float* __restrict__ absmax_in,
                                                                               int8_t* __restrict__ q,
                                                                               float* __restrict__ s) {
  griddep_wait();
  griddep_launch_dependents();
  constexpr int U = 4, T = kQuantThreads;
  const unsigned vpr = VPR ? (unsigned)VPR : (unsigned)vpr_arg;
  __shared__ float2 srow[kQuantMaxRowsPerBlock];  // (scale, RN(1/scale)) of the block's rows
  __shared__ float samax[kQuantMaxRowsPerBlock];
  const unsigned row0 = blockIdx.x * (unsigned)rpb;
  const unsigned nr = min((unsigned)rpb, (unsigned)rows - row0);
  const unsigned span = nr * vpr;  // vectors covered by this block
  const size_t base = (size_t)row0 * vpr;
  const uint4* src = reinterpret_cast<const uint4*>(in) + base;
  uint2* dst = reinterpret_cast<uint2*>(q) + base;
  auto load_round = [&](unsigned k0, uint4(&buf)[U]) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const unsigned k = k0 + u * T;
      buf[u] = k < span && H3B_IDX_OK(base + k, (long long)rows * vpr, &g_h3b_rowops_bounds)
                   ? __ldcs(src + k)
                   : make_uint4(0, 0, 0, 0);
    }
  };
  uint4 ra[U], rb[U];
  load_round(threadIdx.x, ra);
  if (threadIdx.x < nr) {
    const float amax = __ldg(absmax_in + row0 + threadIdx.x);
    const float sc = __fdiv_rn(amax, 127.0f);
    srow[threadIdx.x] = make_float2(sc, __frcp_rn(sc));
    samax[threadIdx.x] = amax;
    if (H3B_IDX_OK(row0 + threadIdx.x, rows, &g_h3b_rowops_bounds)) s[row0 + threadIdx.x] = sc;
  }
  __syncthreads();
  // row of vector k: a division by the constant row length, or advanced incrementally
  // (k only grows) when the length is known only at run time
  unsigned r = 0, row_end = vpr;
  auto quant_round = [&](unsigned k0, const uint4(&buf)[U]) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const unsigned k = k0 + u * T;
      if (k >= span) break;
      if (VPR) {
        r = k / (unsigned)(VPR ? VPR : 1);
      } else {
        while (k >= row_end) {
          ++r;
          row_end += vpr;
        }
      }
      const float2 sr = srow[r];
      const uint2 code = quant8<false>(buf[u], sr.x, sr.y, samax[r]);
      if (H3B_IDX_OK(base + k, (long long)rows * vpr, &g_h3b_rowops_bounds)) dst[k] = code;
    }
  };
  for (unsigned k0 = threadIdx.x; k0 < span; k0 += 2 * U * T) {
    load_round(k0 + U * T, rb);
    quant_round(k0, ra);
    if (k0 + U * T >= span) break;
    load_round(k0 + 2 * U * T, ra);
    quant_round(k0 + U * T, rb);
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
  griddep_wait();
  griddep_launch_dependents();
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
  griddep_wait();
  griddep_launch_dependents();
  for (long long o = blockIdx.x * (long long)blockDim.x + threadIdx.x; o < n_out_vec;
       o += (long long)gridDim.x * blockDim.x) {
    const long long rp = o / dvec;
    const int cv = (int)(o - rp * dvec);
    const long long line = rp / Wm;
    const int k = (int)(rp - line * Wm);
    const long long in0 = ((line * (2LL * Wm) + 2 * k) * dvec + cv);
    if (!H3B_IDX_OK(in0 + dvec, 2 * n_out_vec, &g_h3b_rowops_bounds)) continue;
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

// One thread per 16-byte vector of a merged token: it reads both unmerged
// tokens of the pair and the block's merged output, and writes both positions,
// so each byte is read and written once. Without xm the merged input is
// recomputed from the pair by the same rounding token_pair_kernel applies.
__global__ void token_unpair_kernel(const __nv_bfloat16* __restrict__ x,
                                    const __nv_bfloat16* __restrict__ xm,
                                    const __nv_bfloat16* __restrict__ ym, __nv_bfloat16* out,
                                    long long n_out_vec, int Wm, int dvec) {
  griddep_wait();
  griddep_launch_dependents();
  for (long long o = blockIdx.x * (long long)blockDim.x + threadIdx.x; o < n_out_vec;
       o += (long long)gridDim.x * blockDim.x) {
    const long long rp = o / dvec;
    const int cv = (int)(o - rp * dvec);
    const long long line = rp / Wm;
    const int k = (int)(rp - line * Wm);
    const long long in0 = ((line * (2LL * Wm) + 2 * k) * dvec + cv);
    if (!H3B_IDX_OK(in0 + dvec, 2 * n_out_vec, &g_h3b_rowops_bounds)) continue;
    const uint4 a = __ldcs(reinterpret_cast<const uint4*>(x) + in0);
    const uint4 b = __ldcs(reinterpret_cast<const uint4*>(x) + in0 + dvec);
    const uint4 y = __ldcs(reinterpret_cast<const uint4*>(ym) + o);
    const uint32_t ua[4] = {a.x, a.y, a.z, a.w}, ub[4] = {b.x, b.y, b.z, b.w}, uy[4] = {y.x, y.y, y.z, y.w};
    uint32_t up[4];
    if (xm) {
      const uint4 p = __ldcs(reinterpret_cast<const uint4*>(xm) + o);
      up[0] = p.x; up[1] = p.y; up[2] = p.z; up[3] = p.w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e)
        up[e] = pack_bf16x2((bf16_lo(ua[e]) + bf16_lo(ub[e])) * 0.5f, (bf16_hi(ua[e]) + bf16_hi(ub[e])) * 0.5f);
    }
    uint32_t ra[4], rb[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float dl = bf16_lo(uy[e]) - bf16_lo(up[e]), dh = bf16_hi(uy[e]) - bf16_hi(up[e]);
      ra[e] = pack_bf16x2(bf16_lo(ua[e]) + dl, bf16_hi(ua[e]) + dh);
      rb[e] = pack_bf16x2(bf16_lo(ub[e]) + dl, bf16_hi(ub[e]) + dh);
    }
    reinterpret_cast<uint4*>(out)[in0] = make_uint4(ra[0], ra[1], ra[2], ra[3]);
    reinterpret_cast<uint4*>(out)[in0 + dvec] = make_uint4(rb[0], rb[1], rb[2], rb[3]);
  }
}

// ---------------------------------------------------------------------------
// Residual reuse across denoise steps ([README] control table, core-residual
// reuse): the delta of a block range, delta = x_after - x_before in fp32 (the
// difference of two bf16 values), and its re-application x = bf16(x + delta).
// Eight channels per thread: one 16-byte bf16 vector and two 16-byte fp32 ones.
// ---------------------------------------------------------------------------
__global__ void range_delta_kernel(const __nv_bfloat16* __restrict__ before, const __nv_bfloat16* __restrict__ after,
                                   float* __restrict__ delta, long long n_vec) {
  griddep_wait();
  griddep_launch_dependents();
  for (long long o = blockIdx.x * (long long)blockDim.x + threadIdx.x; o < n_vec;
       o += (long long)gridDim.x * blockDim.x) {
    const uint4 a = __ldcs(reinterpret_cast<const uint4*>(before) + o);
    const uint4 b = __ldcs(reinterpret_cast<const uint4*>(after) + o);
    const uint32_t ua[4] = {a.x, a.y, a.z, a.w}, ub[4] = {b.x, b.y, b.z, b.w};
    float r[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      r[2 * e] = bf16_lo(ub[e]) - bf16_lo(ua[e]);
      r[2 * e + 1] = bf16_hi(ub[e]) - bf16_hi(ua[e]);
    }
    float4* d4 = reinterpret_cast<float4*>(delta) + 2 * o;
    __stcs(d4, make_float4(r[0], r[1], r[2], r[3]));
    __stcs(d4 + 1, make_float4(r[4], r[5], r[6], r[7]));
  }
}

__global__ void range_apply_kernel(__nv_bfloat16* __restrict__ x, const float* __restrict__ delta, long long n_vec) {
  griddep_wait();
  griddep_launch_dependents();
  for (long long o = blockIdx.x * (long long)blockDim.x + threadIdx.x; o < n_vec;
       o += (long long)gridDim.x * blockDim.x) {
    const uint4 a = __ldcs(reinterpret_cast<const uint4*>(x) + o);
    const float4 d0 = __ldcs(reinterpret_cast<const float4*>(delta) + 2 * o);
    const float4 d1 = __ldcs(reinterpret_cast<const float4*>(delta) + 2 * o + 1);
    const float dd[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
    const uint32_t ua[4] = {a.x, a.y, a.z, a.w};
    uint32_t r[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) r[e] = pack_bf16x2(bf16_lo(ua[e]) + dd[2 * e], bf16_hi(ua[e]) + dd[2 * e + 1]);
    reinterpret_cast<uint4*>(x)[o] = make_uint4(r[0], r[1], r[2], r[3]);
  }
}

// ---------------------------------------------------------------------------
// RoPE table: for each axis (t, h, w) with n positions and segment length r,
// entry [pos * (r/2) + j] = (cos, sin)(pos * theta^(-2j/r)), evaluated in fp64
// and stored as fp32. Axis blocks are stored one after the other (t, h, w).
// ---------------------------------------------------------------------------
__device__ void rope_table_entries(const RopeTableArgs& r, int first, int stride) {
  if (!r.tab) return;
  const int nt = r.T * (r.rt / 2), nh = r.H * (r.rh / 2), nw = r.W * (r.rw / 2);
  for (int i = first; i < nt + nh + nw; i += stride) {
    int idx = i, len = r.rt;
    if (idx >= nt + nh) { idx -= nt + nh; len = r.rw; }
    else if (idx >= nt) { idx -= nt; len = r.rh; }
    const int half = len / 2, pos = idx / half, j = idx % half;
    const double ang = (double)pos * pow(r.theta, -2.0 * (double)j / (double)len);
    r.tab[i] = make_float2((float)cos(ang), (float)sin(ang));
  }
}

__global__ void rope_table_kernel(const RopeTableArgs r) {
  griddep_wait();
  griddep_launch_dependents();
  rope_table_entries(r, blockIdx.x * blockDim.x + threadIdx.x, gridDim.x * blockDim.x);
}

// ---------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------
template <int NV, int MB>
static cudaError_t gemv_launch(const void* W, const float* bias, const float* c, int B, float* mod,
                               const RopeTableArgs& rope, int sms, cudaStream_t st) {
  constexpr int d = NV * 256;
  auto kern = adaln_gemv_kernel<NV, MB>;
  const size_t smem = (size_t)B * d * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, smem);
  if (e != cudaSuccess) return e;
  per_sm = per_sm < 1 ? 1 : per_sm;
  // persistent blocks, as many as are resident at once, at most one per 8 row groups
  const int gemv_blocks = std::min((6 * d + 8 * kGemvRows - 1) / (8 * kGemvRows), sms * per_sm);
  int rope_blocks = 0;
  if (rope.tab) {
    const int n = rope.T * (rope.rt / 2) + rope.H * (rope.rh / 2) + rope.W * (rope.rw / 2);
    rope_blocks = (n + 255) / 256;
  }
  return launch_pdl(kern, dim3(gemv_blocks + rope_blocks), dim3(256), smem, st,
                    static_cast<const __nv_bfloat16*>(W), bias, c, B, mod, rope, gemv_blocks);
}

template <int NV>
static cudaError_t gemv_dispatch(const void* W, const float* bias, const float* c, int B, float* mod,
                                 const RopeTableArgs& rope, int sms, cudaStream_t st) {
  return B == 1 ? gemv_launch<NV, 1>(W, bias, c, B, mod, rope, sms, st)
                : gemv_launch<NV, kGemvMaxB>(W, bias, c, B, mod, rope, sms, st);
}

cudaError_t launch_adaln_gemv(const void* W, const float* bias, const float* c, int B, int d,
                              float* mod, float2* rope_tab, int T, int H, int Wd, int rt, int rh, int rw,
                              double theta, int sms, cudaStream_t st) {
  if (B > kGemvMaxB || d % 256 != 0) return cudaErrorInvalidValue;
  const RopeTableArgs rope{rope_tab, T, H, Wd, rt, rh, rw, theta};
#define H3B_GV(nv) \
  case nv:         \
    return gemv_dispatch<nv>(W, bias, c, B, mod, rope, sms, st);
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

// Threads per row: the fewest warps w dividing NV with NV / w <= 6 vectors per
// thread; the block holds as many rows as fit in 512 threads (at least one), so
// one copy of the modulation table serves more rows.
template <int VPT, int NV>
static cudaError_t ln_dispatch(const void* x, int rows, int nv, float eps, const float* shift,
                               const float* scale, int rpi, int ms, int8_t* q, float* s, void* h,
                               float* az, int wc, int sms, cudaStream_t st) {
  const int vpr = 32 * nv;
  const int tpr = vpr / VPT;
  const int block = ln_block(vpr, VPT);
  const int rpp_d = block / tpr;
  const size_t smem = (size_t)vpr * 4 * sizeof(float4) + (size_t)rpp_d * vpr * sizeof(uint4);
  auto kern = ln_mod_quant_kernel<VPT, NV>;
  // the attribute belongs to the current device, so it is set on every launch (a host-side call)
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, block, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  const int rpp = block / tpr;
  const long long passes = (long long)((rows + rpi - 1) / rpi) * ((rpi + rpp - 1) / rpp);
  const long long grid = std::min<long long>(passes, (long long)sms * per_sm);
  return launch_pdl(kern, dim3((unsigned)grid), dim3(block), smem, st, static_cast<const __nv_bfloat16*>(x), rows,
                    vpr, eps, shift, scale, rpi, ms, q, s, static_cast<__nv_bfloat16*>(h), az, wc);
}

cudaError_t launch_ln_mod_quant(const void* x, int rows, int d, float eps, const float* shift,
                                const float* scale, int rows_per_item, int mod_stride, int8_t* q,
                                float* s, void* h_out, float* absmax_zero, int write_codes, unsigned* err,
                                int sms, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  const int nv = d / 256;
  if (nv < 1 || nv > 32 || d % 256) return cudaErrorInvalidValue;
  // the widths of the workloads get kernels with the row length built in
  if (nv == 20) return ln_dispatch<5, 20>(x, rows, nv, eps, shift, scale, rows_per_item, mod_stride, q, s, h_out, absmax_zero, write_codes, sms, st);
  if (nv == 8) return ln_dispatch<4, 8>(x, rows, nv, eps, shift, scale, rows_per_item, mod_stride, q, s, h_out, absmax_zero, write_codes, sms, st);
  if (nv == 1) return ln_dispatch<1, 1>(x, rows, nv, eps, shift, scale, rows_per_item, mod_stride, q, s, h_out, absmax_zero, write_codes, sms, st);
  int w = 1;
  while (nv % w || nv / w > 6) ++w;
  switch (nv / w) {
    case 1: return ln_dispatch<1, 0>(x, rows, nv, eps, shift, scale, rows_per_item, mod_stride, q, s, h_out, absmax_zero, write_codes, sms, st);
    case 2: return ln_dispatch<2, 0>(x, rows, nv, eps, shift, scale, rows_per_item, mod_stride, q, s, h_out, absmax_zero, write_codes, sms, st);
    case 3: return ln_dispatch<3, 0>(x, rows, nv, eps, shift, scale, rows_per_item, mod_stride, q, s, h_out, absmax_zero, write_codes, sms, st);
    case 4: return ln_dispatch<4, 0>(x, rows, nv, eps, shift, scale, rows_per_item, mod_stride, q, s, h_out, absmax_zero, write_codes, sms, st);
    case 5: return ln_dispatch<5, 0>(x, rows, nv, eps, shift, scale, rows_per_item, mod_stride, q, s, h_out, absmax_zero, write_codes, sms, st);
    case 6: return ln_dispatch<6, 0>(x, rows, nv, eps, shift, scale, rows_per_item, mod_stride, q, s, h_out, absmax_zero, write_codes, sms, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_quant_rows_bf16(const void* h, int rows, int cols, const float* absmax,
                                   int8_t* q, float* s, int sms, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  if (absmax) {
    const int vpr = cols / 8;
    // about 4096 vectors (64 KB of input) per block: each thread keeps four 16-byte loads in
    // flight over four rounds, and the per-block setup is amortized over several rows
    int rpb = 4096 / vpr;
    rpb = std::min(rpb, rows / (4 * sms));  // but at least about four blocks per SM
    rpb = rpb < 1 ? 1 : (rpb > kQuantMaxRowsPerBlock ? kQuantMaxRowsPerBlock : rpb);
    const int grid = (rows + rpb - 1) / rpb;
    const auto* in = static_cast<const __nv_bfloat16*>(h);
    auto kern = vpr == 640    ? quant_rows_known_absmax_kernel<640>
                : vpr == 2560 ? quant_rows_known_absmax_kernel<2560>
                              : quant_rows_known_absmax_kernel<0>;
    return launch_pdl(kern, dim3(grid), dim3(kQuantThreads), 0, st, in, rows, vpr, rpb, absmax, q, s);
  }
  return launch_pdl(quant_rows_kernel<__nv_bfloat16>, dim3(rows), dim3(256), 0, st,
                    static_cast<const __nv_bfloat16*>(h), cols, absmax, q, s);
}

cudaError_t launch_quant_rows_f32(const float* w, int rows, int cols, int8_t* q, float* s,
                                  cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  return launch_pdl(quant_rows_kernel<float>, dim3(rows), dim3(256), 0, st, w, cols, (const float*)nullptr, q, s);
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
  return launch_pdl(token_pair_kernel, dim3(grid_for(n, sms)), dim3(256), 0, st, static_cast<const __nv_bfloat16*>(x),
                    static_cast<__nv_bfloat16*>(xm), static_cast<__nv_bfloat16*>(xm2), n, W / 2, d / 8);
}

cudaError_t launch_range_delta(const void* before, const void* after, float* delta, long long n, int sms,
                               cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const long long nv = n / 8;
  return launch_pdl(range_delta_kernel, dim3(grid_for(nv, sms)), dim3(256), 0, st,
                    static_cast<const __nv_bfloat16*>(before), static_cast<const __nv_bfloat16*>(after), delta, nv);
}

cudaError_t launch_range_apply(void* x, const float* delta, long long n, int sms, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const long long nv = n / 8;
  return launch_pdl(range_apply_kernel, dim3(grid_for(nv, sms)), dim3(256), 0, st, static_cast<__nv_bfloat16*>(x),
                    delta, nv);
}

cudaError_t launch_token_unpair(const void* x, const void* xm, const void* ym, void* out,
                                long long lines, int W, int d, int sms, cudaStream_t st) {
  const long long n = lines * (W / 2) * (d / 8);
  if (n == 0) return cudaSuccess;
  return launch_pdl(token_unpair_kernel, dim3(grid_for(n, sms)), dim3(256), 0, st, static_cast<const __nv_bfloat16*>(x),
                    static_cast<const __nv_bfloat16*>(xm), static_cast<const __nv_bfloat16*>(ym),
                    static_cast<__nv_bfloat16*>(out), n, W / 2, d / 8);
}

unsigned* rowops_bounds_word() {
  void* p = nullptr;
  return cudaGetSymbolAddress(&p, g_h3b_rowops_bounds) == cudaSuccess ? static_cast<unsigned*>(p) : nullptr;
}

cudaError_t launch_rope_table(float2* tab, int T, int H, int W, int rt, int rh, int rw,
                              double theta, cudaStream_t st) {
  const int n = T * (rt / 2) + H * (rh / 2) + W * (rw / 2);
  return launch_pdl(rope_table_kernel, dim3((n + 255) / 256), dim3(256), 0, st, RopeTableArgs{tab, T, H, W, rt, rh, rw, theta});
}

}  // namespace h3b
